/*
 * attn.h -- C ABI of libattn, the B200 (sm_100a) fused exact-attention forward.
 *
 * The operation (page "FlashAttention (SV)", section "Problematik med
 * standard-attention", the attention formula; tiled with the online softmax
 * of section "Online-beräkning av Softmax" and fused into one kernel as in
 * section "Sammanslagning av operationer till en enda CUDA-kärna"):
 *
 *   S = scale * Q K^T  (+ causal mask),   O = softmax(S) V,
 *   LSE[i] = ln sum_j exp(S[i, j])        (natural log of the scaled scores)
 *
 * Head sizes 64, 128 and 256 and grouped/multi-query heads follow page
 * "FlashAttention-4震撼发布：性能再攀新高" (the FlashAttention-2 list: head
 * size up to 256, MQA and GQA).  The FP8 entry points follow page
 * "FlashAttention-3 — 闪电注意力-3", section 3 (FP8 with incoherent
 * processing: rotate Q and K by a random orthogonal Hadamard matrix, then
 * quantise).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers:  every tensor pointer is a DEVICE pointer owned by the caller
 *            (for example torch.empty(...).data_ptr()).  The library keeps no
 *            reference after the call returns and allocates no device memory
 *            for the caller's data.  Tensor pointers must be 16-byte aligned
 *            (the tiles are moved by the Tensor Memory Accelerator).
 * Layout:    Q and O are [B, Nq, Hq, d]; K and V are [B, Nk, Hkv, d]; all
 *            contiguous row-major with d innermost.  LSE is [B, Hq, Nq] fp32.
 * Heads:     query head h reads key/value head h / (Hq / Hkv); Hq % Hkv == 0
 *            (Hkv == Hq is multi-head, Hkv == 1 multi-query).
 * Causal:    bottom-right aligned.  Query row i sees key j iff
 *            j <= i + (Nk - Nq).  With Nq == Nk this is j <= i.  A row that
 *            sees no key (only when Nq > Nk) gets O = 0 and LSE = -inf.
 * Stream:    `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *            stream).  Every call is asynchronous on that stream and returns
 *            after the launch; device results are ready when the stream is.
 * Errors:    argument errors are returned synchronously as attn_status_t and
 *            nothing is launched.  A launch failure returns ATTN_ERR_CUDA.
 *            Every device-side wait is bounded: a wait that runs out records
 *            an error word on the device instead of hanging; read it with
 *            attn_get_last_device_error().
 * Threads:   all entry points are thread-safe.
 * Empty:     B == 0, Hq == 0 or Nq == 0 is a no-op returning ATTN_OK.  Nk == 0
 *            gives O = 0 and LSE = -inf for every row.
 * Environment (read once, at the first call):
 *            ATTN_LOG=1 prints one line per kernel launch to stderr: the
 *            kernel, its template configuration (head size, key tile, query
 *            tiles per block, ring stages, causal, dtype, software-exp share,
 *            score buffers, separate P, streams, staged output), grid, block,
 *            shared memory and problem size.  The library is silent otherwise.
 *            ATTN_WAIT_TIMEOUT_NS=<n> sets the limit of every device-side wait
 *            in nanoseconds (default 2 s).
 */
#ifndef LIBATTN_ATTN_H_
#define LIBATTN_ATTN_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = 1,    /* null pointer, negative size, Hq % Hkv != 0, non-finite scale */
    ATTN_ERR_UNSUPPORTED = 2,    /* head size or dtype not built, or not an sm_100 device */
    ATTN_ERR_MISALIGNED = 3,     /* a tensor pointer is not 16-byte aligned */
    ATTN_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
    ATTN_ERR_DEVICE_TIMEOUT = 5  /* a device-side wait ran out (see attn_get_last_device_error) */
} attn_status_t;

typedef enum {
    ATTN_BF16 = 0,     /* Q, K, V in bfloat16 */
    ATTN_FP8_E4M3 = 1  /* Q, K, V in OCP FP8 E4M3 with unit scales */
} attn_dtype_t;

/*
 * attn_fwd -- fused attention forward.
 *   q      [B, Nq, Hq, d]  bf16 (or e4m3 bytes when dtype == ATTN_FP8_E4M3)
 *   k, v   [B, Nk, Hkv, d] same dtype as q
 *   o      [B, Nq, Hq, d]  bf16 output (always bf16)
 *   lse    [B, Hq, Nq]     fp32 output, natural log; may be NULL to skip it
 *   d      64, 128 or 256 for bf16; 128 for FP8
 *   causal 0 or 1
 *   scale  finite multiplier of Q K^T (1/sqrt(d) for the usual attention)
 *   dtype  attn_dtype_t
 * Returns ATTN_OK or an error code; see the conventions above.
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
             int dtype, void *stream);

/*
 * attn_fwd_part -- attn_fwd restricted to batches [b_begin, b_end) and the
 * query heads of key/value heads [kvh_begin, kvh_end) (query heads
 * [kvh_begin * g, kvh_end * g) with g = Hq / Hkv, so a grouped-query group is
 * never split).  Every (batch, head) of the problem is independent (page
 * "FlashAttention (SV)", the attention formula is applied per head), so
 * several devices can each compute a part of one call on the same full
 * tensors, with no exchange of data between them.
 *   q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dtype, stream
 *                as attn_fwd: the FULL tensors and sizes of the call
 *   b_begin, b_end      0 <= b_begin <= b_end <= B
 *   kvh_begin, kvh_end  0 <= kvh_begin <= kvh_end <= Hkv
 * Only the O rows and LSE entries of the part are written; the rest of o and
 * lse is left as it was.  An empty range is a no-op.  attn_fwd is this call
 * with the whole range.  Returns ATTN_ERR_INVALID_ARG for a range outside the
 * problem; otherwise as attn_fwd.
 */
int attn_fwd_part(const void *q, const void *k, const void *v, void *o, float *lse,
                  int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                  int dtype, int b_begin, int b_end, int kvh_begin, int kvh_end, void *stream);

/*
 * attn_shard_units -- the share of one call that rank `rank` of `world`
 * computes when the call is split over devices: the B * Hkv units (batch,
 * key/value head) are cut in batch-major order into `world` contiguous runs
 * whose lengths differ by at most one; rank r takes run r.  The run is
 * written to rects as up to three rectangles, rectangle i being
 * rects[4i .. 4i+3] = {b_begin, b_end, kvh_begin, kvh_end}, each one
 * attn_fwd_part call (rects must hold 12 ints).  Returns the number of
 * rectangles (0 when the rank has no unit), or -1 for invalid arguments
 * (B < 0, Hkv < 0, world < 1, rank outside [0, world), rects NULL).
 * Host-only; no CUDA call.
 */
int attn_shard_units(int B, int Hkv, int world, int rank, int *rects);

/*
 * attn_fwd_host -- attn_fwd (bf16) with its inputs and outputs in HOST memory:
 * the call copies Q, K and V in, computes, and copies O (and LSE) out, all
 * enqueued on `stream`.  The work is cut into n_chunks runs of the B * Hkv
 * (batch, key/value head) units (the split of attn_shard_units, so a
 * grouped-query group stays whole) and pipelined: the copies in of chunk
 * c + 1 and the copies out of chunk c - 1 run while chunk c computes.  The
 * copies run on two streams of the library's own (one per direction), made to
 * wait for the work already on `stream` and joined back to it, so the host
 * outputs are complete when `stream` is.  Each chunk moves strided rows (its
 * heads of every sequence row) with one 2-D copy per tensor and rectangle.
 *   q_h, k_h, v_h    host inputs, layouts as attn_fwd.  Page-locked memory
 *                    (cudaHostAlloc, cudaHostRegister, torch pin_memory) lets
 *                    the copies overlap; pageable memory works but serialises.
 *   o_h, lse_h       host outputs; lse_h may be NULL (then LSE stays on the
 *                    device, if lse_d is given, or is not computed).
 *   q_d, k_d, v_d, o_d, lse_d
 *                    caller-owned DEVICE buffers of the full tensors, as for
 *                    attn_fwd (16-byte aligned; lse_d may be NULL only when
 *                    lse_h is NULL).  They hold the inputs and results after
 *                    the call as attn_fwd's tensors would.
 *   n_chunks         pipeline depth, >= 1; 0 picks 8.  Clamped to B * Hkv.
 *   B, Hq, Hkv, Nq, Nk, d, causal, scale, stream   as attn_fwd.
 * Host buffers must not overlap the device ones.  The library allocates no
 * memory for the data; its two streams and a few events per device are
 * created at the first call and kept.  Calls from several host threads are
 * serialised while they enqueue.  Returns as attn_fwd (ATTN_ERR_INVALID_ARG
 * also for a NULL host pointer, n_chunks < 0, or lse_h without lse_d);
 * ATTN_ERR_CUDA if an enqueue fails part way (the stream may then hold part
 * of the work).
 */
int attn_fwd_host(const void *q_h, const void *k_h, const void *v_h, void *o_h, float *lse_h,
                  void *q_d, void *k_d, void *v_d, void *o_d, float *lse_d,
                  int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                  int n_chunks, void *stream);

/*
 * attn_fwd_fp8 -- FP8 E4M3 attention forward with per-tensor scales.
 * Page "FlashAttention-3 — 闪电注意力-3", section 3: the inputs are quantised
 * (Q and K after the Hadamard rotation, see attn_hadamard_quant_fp8) and the
 * products run on FP8 tensor cores.  The real inputs are q8*dq, k8*dk, v8*dv:
 *   S = scale * dq * dk * (q8 k8^T);  P = softmax weights rounded to E4M3;
 *   O = dv * (P v8) / rowsum,  bf16.
 *   q8, k8, v8   e4m3 bytes, layouts as attn_fwd; d must be 128
 *   descale_q/k/v  DEVICE pointers to one fp32 each (dq, dk, dv), as written
 *                  by attn_hadamard_quant_fp8, so no host synchronisation is
 *                  needed between quantisation and attention
 * Returns ATTN_OK or an error code.
 */
int attn_fwd_fp8(const void *q8, const void *k8, const void *v8, void *o, float *lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                 const float *descale_q, const float *descale_k, const float *descale_v,
                 void *stream);

/*
 * attn_hadamard_quant_fp8 -- FP8 input preparation (page "FlashAttention-3 —
 * 闪电注意力-3", section 3, items 1-3).
 *   x          [rows, d] bf16 input (any leading shape flattened to rows)
 *   x8         [rows, d] e4m3 output
 *   descale    DEVICE pointer to one fp32 output: amax / 448, where amax is
 *              the largest |value| of the (rotated) tensor
 *   workspace  DEVICE scratch of attn_hadamard_quant_fp8_workspace_bytes()
 *              bytes, owned by the caller; its contents on entry do not matter
 *   signs      DEVICE pointer to d fp32 values, each +1 or -1 (the random
 *              diagonal), or NULL for no rotation (plain per-tensor FP8)
 *   d          128 (a power of two the rotation is built for)
 * With signs != NULL each row is replaced by x diag(signs) H_d / sqrt(d)
 * (Sylvester Hadamard H_d, computed as a fast Walsh-Hadamard transform in
 * fp32), which is orthogonal, so (QM)(KM)^T = QK^T.  Then every element is
 * quantised as E4M3(x * (448/amax)) with round-to-nearest-even and
 * saturation (fp32 arithmetic).
 */
int attn_hadamard_quant_fp8(const void *x, void *x8, float *descale, void *workspace,
                            long long rows, int d, const float *signs, void *stream);

/* Bytes of device workspace attn_hadamard_quant_fp8 needs. */
long long attn_hadamard_quant_fp8_workspace_bytes(void);

/*
 * attn_hadamard_quant_fp8_noalloc -- attn_hadamard_quant_fp8 without the
 * workspace argument, for callers that cannot allocate device memory: code
 * whose device memory is owned by another allocator it has no handle to, and
 * real-time or plug-in code that must not call cudaMalloc on its hot path.
 * The pages have no counterpart; this is a packaging of the same operation.
 *   x, x8, descale, rows, d, signs, stream  as attn_hadamard_quant_fp8.
 * Scratch: a 256-byte file-scope device array inside the library (every GPU
 * that loads the library holds it until the process exits).  The call needs
 * attn_hadamard_quant_fp8_workspace_bytes() of it (currently 256 bytes, for
 * any rows); a build whose need exceeded 256 bytes would return
 * ATTN_ERR_UNSUPPORTED.  Nothing is allocated: no cudaMalloc/cudaFree and no
 * allocating library routine.
 * Set-up: the first call on a device looks up the array's device address with
 * that device current; make that first call before any stream capture.
 * Sharing: all calls on a device use the same array, which keeps the last
 * call's contents; each call clears the part that must start at zero.  Calls
 * that overlap on the GPU (for example on two streams) race on the array and
 * must be ordered by the caller.
 * Returns ATTN_OK or an error code, as attn_hadamard_quant_fp8.
 */
int attn_hadamard_quant_fp8_noalloc(const void *x, void *x8, float *descale, long long rows, int d,
                                    const float *signs, void *stream);

/*
 * attn_get_last_device_error -- synchronises `stream`, then reads and clears
 * the device error word of the current device.  Returns ATTN_OK,
 * ATTN_ERR_DEVICE_TIMEOUT (a bounded wait ran out inside a kernel) or
 * ATTN_ERR_CUDA (the synchronisation itself failed).  If `detail` is not
 * NULL it receives the raw word: bit 0 timeout, bits 8..15 the wait site,
 * bits 16..31 the low bits of the block index.
 */
int attn_get_last_device_error(void *stream, unsigned int *detail);

/* Human-readable name of a status code (static storage). */
const char *attn_status_string(int status);

/*
 * Causal tile plan (host and device share this logic; exported for tests).
 * For the query rows [row0, row1) of one query tile, against Nk keys cut
 * into tiles of bn keys:
 *   attn_kv_tile_count  number of leading key tiles that hold at least one
 *                       visible (row, key) pair (key tiles after that are
 *                       skipped entirely; 0 if the rows see no key);
 *   attn_tile_kind      0 = skip (no visible pair), 1 = full (every pair
 *                       visible: no mask needed), 2 = partial (mask per
 *                       element), for key tile kt.
 * row1 is clipped to Nq.  Returns -1 on invalid arguments.
 */
int attn_kv_tile_count(int row0, int row1, int Nq, int Nk, int bn, int causal);
int attn_tile_kind(int row0, int row1, int kt, int Nq, int Nk, int bn, int causal);

/*
 * Split-KV forward (decode-shaped calls: few query rows, long key ranges).
 * The same operation as attn_fwd (BF16, d in {64, 128, 256}, same layouts,
 * causal rule and outputs), computed as n_splits partial attentions over
 * contiguous key windows and merged by attn_combine's LSE-weighted sum; page
 * "FlashAttention (SV)", section "Online-beräkning av Softmax" (the rescaling
 * by exp(m_old - m_new) that lets partial results over key blocks merge);
 * the pages name FlashDecoding for the decode setting but give no method, so
 * the window split and the combine formula are this library's reading.
 *   n_splits        requested number of key windows; <= 0 chooses one that
 *                   fills the GPU about twice (windows of >= 512 keys).  The
 *                   windows hold a multiple of 128 keys; fewer windows than
 *                   requested may result.  One window runs attn_fwd itself.
 *   workspace       DEVICE scratch, 16-byte aligned, of at least
 *                   attn_splitkv_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, n_splits)
 *                   bytes (0 when no split results: workspace may be NULL);
 *                   owned by the caller, not retained after the call.
 * Returns ATTN_ERR_INVALID_ARG for a missing or short workspace and
 * ATTN_ERR_UNSUPPORTED when B * windows exceeds 65535; otherwise as attn_fwd.
 * When the group size g = Hq / Hkv > 1 divides 128, the g query heads of a
 * key/value head share query tiles (row i of head h at tile row i * g + h % g),
 * so each key/value tile is read once per group and short query ranges fill
 * the 128-row tiles.
 * attn_splitkv_workspace_bytes returns -1 for invalid sizes (and, with
 * n_splits <= 0, when no sm_100 device is current).
 */
long long attn_splitkv_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int n_splits);
int attn_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     int n_splits, void *workspace, long long workspace_bytes, void *stream);

/*
 * LSE-weighted merge of S partial results over disjoint key windows:
 *   LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) * O_s
 * (windows with LSE_s = -inf weigh nothing; a row whose every LSE_s is -inf
 * gets O = 0, LSE = -inf).
 *   o_parts    DEVICE fp32 [S, B, Nq, Hq, d]: O_s, each normalised by its own
 *              row sum; 16-byte aligned
 *   lse_parts  DEVICE fp32 [S, B, Hq, Nq]: LSE_s (natural log)
 *   o          DEVICE bf16 [B, Nq, Hq, d], 16-byte aligned; lse DEVICE fp32
 *              [B, Hq, Nq] or NULL
 * Exported for callers that shard keys across devices and for the tests;
 * attn_fwd_splitkv uses it on its own partials.
 */
int attn_combine(const float *o_parts, const float *lse_parts, int n_splits, int B, int Hq, int Nq,
                 int d, void *o, float *lse, void *stream);

/*
 * The tile plan for a key window (split-KV): the window holds Nk keys and
 * `shift` further keys follow it, so that in window-local indices query row i
 * sees key j iff j < Nk and (!causal || j <= i + (Nk - Nq) + shift).
 * shift = 0 is attn_kv_tile_count / attn_tile_kind.  Host-only; -1 on
 * invalid arguments.
 */
int attn_kv_tile_count_window(int row0, int row1, int Nq, int Nk, int shift, int bn, int causal);
int attn_tile_kind_window(int row0, int row1, int kt, int Nq, int Nk, int shift, int bn, int causal);

/*
 * attn_gemm_add -- D = A B + C for small reduction sizes K (page
 * "FlashAttention-4震撼发布": an A@B+C kernel on Blackwell that overlaps its
 * epilogue with the next products through two accumulation buffers; the page
 * gives no sizes or method, so layouts and tiling are this library's).
 *   a  [M, K] bf16, b [K, N] bf16, c [M, N] bf16 or NULL (no addition),
 *   d  [M, N] bf16 output; all row-major DEVICE pointers, 16-byte aligned.
 * Products accumulate in fp32; D = bf16(A B + C), round to nearest even.
 * Sizes: any M >= 0; N and K multiples of 8 (ATTN_ERR_UNSUPPORTED
 * otherwise), with the row strides 2N and 2K bytes and the matrix extents
 * within the Tensor Memory Accelerator's limits (ATTN_ERR_CUDA when a tensor
 * map cannot be encoded).  K = 0 gives D = C (or 0).  The design targets
 * small K (the kernel is then HBM-bound on reading C and writing D).
 * Aliasing: c == d is allowed (an in-place D += A B); a c that overlaps d
 * any other way returns ATTN_ERR_INVALID_ARG.  a and b must not overlap d.
 */
int attn_gemm_add(const void *a, const void *b, const void *c, void *d, int M, int N, int K, void *stream);

/*
 * Which kernel attn_fwd / attn_fwd_fp8 launch for a key range of Nk keys at
 * head size d (64, 128, 256) with the causal flag: 1 = the persistent kernel
 * (one block per SM looping over the work items; used for short key ranges,
 * Nk <= 1024, whose items are short), 0 = one block per work item (longer
 * ranges, and causal launches at d = 128, where the blocks of uneven causal
 * items are handed out longest first).  Both compute the same result.
 * Host-only; -1 for invalid arguments.  The page set describes one block per
 * (batch, head, query block); the persistent schedule is this library's own.
 */
int attn_fwd_schedule(int Nk, int d, int causal);

/*
 * Debug hook for the failure path: launches one block that waits, with the
 * given limit in nanoseconds, on a device barrier nothing ever completes, so
 * the bounded wait runs out and records ATTN_ERR_DEVICE_TIMEOUT in the
 * device error word.  Used by the tests to show that a wait that cannot
 * finish ends with an error status and leaves the context usable.
 */
int attn_debug_unsatisfied_wait(long long limit_ns, void *stream);

/*
 * Counters of the library's tensor-map cache (host only, never fails for
 * non-NULL arguments): `hits` counts tensor maps taken from the cache,
 * `encodes` those encoded afresh.  Every launch needs one map per Q/K/V
 * operand (A/B for attn_gemm_add); a map is a pure function of the tensor's
 * base address, shape and tile box, so calls that reuse the same tensors skip
 * the encoding.  The cache holds 256 maps (64 sets of 4) and is guarded by a
 * mutex.
 */
int attn_debug_map_cache_stats(unsigned long long *hits, unsigned long long *encodes);

/*
 * Debug hook for the softmax exponential: y[i] = 2^x[i] for n values, as the
 * attention kernel computes it: mode 0 the hardware approximation
 * (ex2.approx), mode 1 the software polynomial (page "FlashAttention-4震撼发布",
 * software emulation of the exponential).  x and y are device pointers.
 */
int attn_debug_exp2(const float *x, float *y, long long n, int mode, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBATTN_ATTN_H_ */
