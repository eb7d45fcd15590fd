// attn_api.cu -- the C ABI of libattn (declared in include/attn.h): argument
// checks, TMA descriptor encoding, choice of kernel instantiation, launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_fwd_kernel.cuh"
#include "attn_fwd_persistent_kernel.cuh"
#include "combine.cuh"
#include "fp8_prep.cuh"
#include "gemm_add.cuh"
#include "tiles.h"

namespace attn {
namespace {

__device__ unsigned int g_err_word;     // device error word (bounded waits that ran out)

// Scratch of attn_hadamard_quant_fp8_noalloc: a fixed 256-byte array that every
// device loading this library holds until process exit.  Only word 0 (the
// running absolute maximum) is used; the rest pads it to the 256 bytes the
// workspace-taking entry point asks for.
constexpr int kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned int g_noalloc_scratch[kNoAllocScratchBytes / 4];
__device__ float g_unit_descale = 1.0f;  // descale used when attn_fwd is given e4m3 inputs

constexpr int kMaxDevices = 64;
constexpr int kMaxSplits = 1024;  // key windows of one split-KV call
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait

struct DeviceState {
  bool init = false;
  int status = ATTN_OK;
  unsigned int* err = nullptr;
  unsigned int* noalloc_scratch = nullptr;  // device address of g_noalloc_scratch
  const float* unit_descale = nullptr;      // device address of g_unit_descale
  int num_sms = 0;
  CUcontext ctx = nullptr;  // context the addresses above belong to
  unsigned gen = 0;         // bumped whenever the state is (re)built
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
EncodeTiledFn g_encode = nullptr;
CtxGetCurrentFn g_ctx_current = nullptr;

// ATTN_LOG=1 in the environment: every launch prints its kernel, template
// configuration, grid and problem size to stderr (read once; silent otherwise).
bool log_on() {
  static const bool v = [] {
    const char* e = std::getenv("ATTN_LOG");
    return e != nullptr && std::atoi(e) > 0;
  }();
  return v;
}
#define ATTN_LOGF(...)                        \
  do {                                        \
    if (log_on()) std::fprintf(stderr, __VA_ARGS__); \
  } while (0)
template <class Cfg>
void log_launch(const char* kernel, dim3 grid, int B, int Hq, int Hkv, int Nq, int Nk, const char* extra = "") {
  if (!log_on()) return;
  std::fprintf(stderr,
               "attn: %s<D=%d BN=%d NQT=%d KST=%d VST=%d causal=%d fp8=%d EMU=%d SB=%d PSEP=%d NS=%d OST=%d> "
               "grid=(%u,%u,%u) block=%d smem=%u B=%d Hq=%d Hkv=%d Nq=%d Nk=%d%s\n",
               kernel, Cfg::D, Cfg::BN, Cfg::NQT, Cfg::KST, Cfg::VST, (int)Cfg::CAUSAL, (int)Cfg::FP8, Cfg::EMU, Cfg::SB,
               (int)Cfg::PSEP, Cfg::NS, (int)Cfg::OST, grid.x, grid.y, grid.z, Cfg::NTHREADS, Cfg::SMEM_BYTES, B, Hq,
               Hkv, Nq, Nk, extra);
}

unsigned long long timeout_ns() {
  static unsigned long long v = [] {
    const char* e = std::getenv("ATTN_WAIT_TIMEOUT_NS");
    if (e == nullptr) return kDefaultTimeoutNs;
    const unsigned long long x = std::strtoull(e, nullptr, 10);
    return x > 0 ? x : kDefaultTimeoutNs;
  }();
  return v;
}

template <class Fn>
bool driver_entry(const char* name, Fn* out) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess ||
      fn == nullptr)
    return false;
  *out = reinterpret_cast<Fn>(fn);
  return true;
}

// Per-device setup: checks for an sm_100 device and finds the device
// addresses of the library's own device variables.  The state belongs to the
// device's current context: when that context changes (a cudaDeviceReset
// destroys it) the state is rebuilt, so no address of an old context is used.
// Only a verdict that cannot change (not an sm_100 device) is cached; a failed
// CUDA call is retried on the next entry.
int device_state(int* dev_out, DeviceState** st_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_dev[dev];
  *dev_out = dev;
  *st_out = &st;
  if (st.init && st.status == ATTN_OK) {
    CUcontext cur = nullptr;
    if (g_ctx_current(&cur) == CUDA_SUCCESS && cur == st.ctx) return ATTN_OK;
    st.init = false;  // new context: look everything up again
  }
  if (st.init) return st.status;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (major != 10 || minor != 0) {  // built for sm_100a only
    st.init = true;
    st.status = ATTN_ERR_UNSUPPORTED;
    return st.status;
  }
  if ((g_encode == nullptr && !driver_entry("cuTensorMapEncodeTiled", &g_encode)) ||
      (g_ctx_current == nullptr && !driver_entry("cuCtxGetCurrent", &g_ctx_current)))
    return ATTN_ERR_CUDA;
  unsigned int *err = nullptr, *scratch = nullptr;
  float* one = nullptr;
  // (these calls also create the device's context if it does not exist yet)
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_err_word) != cudaSuccess ||
      cudaGetSymbolAddress(reinterpret_cast<void**>(&scratch), g_noalloc_scratch) != cudaSuccess ||
      cudaGetSymbolAddress(reinterpret_cast<void**>(&one), g_unit_descale) != cudaSuccess || err == nullptr ||
      scratch == nullptr || one == nullptr)
    return ATTN_ERR_CUDA;
  CUcontext cur = nullptr;
  if (g_ctx_current(&cur) != CUDA_SUCCESS || cur == nullptr) return ATTN_ERR_CUDA;
  st.err = err;
  st.noalloc_scratch = scratch;
  st.unit_descale = one;
  st.num_sms = sms;
  st.ctx = cur;
  ++st.gen;
  st.status = ATTN_OK;
  st.init = true;
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Cache of encoded tensor maps.  A map is a pure function of the encoding's
// arguments (base address, data type, dims, strides, box; the other fields
// are the same for every map here), so a hit returns exactly what a fresh
// encoding would; calls that reuse the same tensors skip the host-side
// encoding.  kMapSets sets of kMapWays entries (round-robin replacement within
// a set, so the few maps of one call never evict each other), guarded by a
// mutex.
struct MapKey {
  uint64_t ptr;
  uint32_t dtype, rank;
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5];
};
constexpr int kMapSets = 64, kMapWays = 4;
struct MapEntry {
  bool valid = false;
  MapKey key;
  CUtensorMap map;
};
struct MapSet {
  MapEntry way[kMapWays];
  int next = 0;
};
MapSet g_maps[kMapSets];
std::mutex g_maps_mu;
std::atomic<unsigned long long> g_map_hits{0}, g_map_encodes{0};

int encode_cached(CUtensorMap* m, CUtensorMapDataType dt, uint32_t rank, const void* ptr, const cuuint64_t* dims,
                  const cuuint64_t* strides, const cuuint32_t* box) {
  MapKey key;
  std::memset(&key, 0, sizeof(key));  // padding bytes take part in the comparison
  key.ptr = reinterpret_cast<uint64_t>(ptr);
  key.dtype = (uint32_t)dt;
  key.rank = rank;
  for (uint32_t i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides[i];
  }
  uint64_t h = 1469598103934665603ull;  // FNV-1a over the key bytes
  const unsigned char* kb = reinterpret_cast<const unsigned char*>(&key);
  for (size_t i = 0; i < sizeof(key); ++i) h = (h ^ kb[i]) * 1099511628211ull;
  MapSet& set = g_maps[h % kMapSets];
  {
    std::lock_guard<std::mutex> lk(g_maps_mu);
    for (int w = 0; w < kMapWays; ++w)
      if (set.way[w].valid && std::memcmp(&set.way[w].key, &key, sizeof(key)) == 0) {
        *m = set.way[w].map;
        g_map_hits.fetch_add(1, std::memory_order_relaxed);
        return ATTN_OK;
      }
  }
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  const CUresult r = g_encode(m, dt, rank, const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ATTN_ERR_CUDA;
  g_map_encodes.fetch_add(1, std::memory_order_relaxed);
  std::lock_guard<std::mutex> lk(g_maps_mu);
  MapEntry& e = set.way[set.next];
  set.next = (set.next + 1) % kMapWays;
  e.valid = true;
  std::memcpy(&e.key, &key, sizeof(key));
  e.map = *m;
  return ATTN_OK;
}

int encode_bnhd(CUtensorMap* m, const void* ptr, bool fp8, int B, int N, int H, int d, int rows) {
  const cuuint64_t es = fp8 ? 1 : 2;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)N * H * d * es};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / es), 1u, (cuuint32_t)rows, 1u};
  return encode_cached(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ptr, dims,
                       strides, box);
}

// Q viewed as (d, g, Hkv, Nq, B) for head packing: a box of g heads x
// rows / g query rows of one key/value head lands in shared memory as `rows`
// packed 128-byte rows (row i * g + head-in-group), the layout of an unpacked
// Q tile.
int encode_q_packed(CUtensorMap* m, const void* ptr, int B, int Nq, int Hkv, int g, int d, int rows) {
  const cuuint64_t es = 2;
  const cuuint64_t Hq = (cuuint64_t)Hkv * g;
  const cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)g, (cuuint64_t)Hkv, (cuuint64_t)Nq, (cuuint64_t)B};
  const cuuint64_t strides[4] = {(cuuint64_t)d * es, (cuuint64_t)g * d * es, Hq * d * es,
                                 (cuuint64_t)Nq * Hq * d * es};
  const cuuint32_t box[5] = {(cuuint32_t)(128 / es), (cuuint32_t)g, 1u, (cuuint32_t)(rows / g), 1u};
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, ptr, dims, strides, box);
}

// 2-D row-major bf16 matrix [rows, cols] as a 4-D map (cols, rows, 1, 1), box
// (64 columns = 128 bytes, box_rows), 128-byte swizzle, zero fill out of range.
int encode_rows(CUtensorMap* m, const void* ptr, int rows, int cols, int box_rows) {
  const cuuint64_t es = 2;
  const cuuint64_t dims[4] = {(cuuint64_t)cols, (cuuint64_t)rows, 1, 1};
  const cuuint64_t row_bytes = (cuuint64_t)cols * es, all = (cuuint64_t)rows * row_bytes;
  const cuuint64_t strides[3] = {row_bytes, all, all};
  const cuuint32_t box[4] = {64u, (cuuint32_t)box_rows, 1u, 1u};
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ptr, dims, strides, box);
}

// The same matrix as a rank-2 map (cols, rows), for the 2-D tiled loads and
// stores of the A@B+C epilogue.
int encode_rows_2d(CUtensorMap* m, const void* ptr, int rows, int cols, int box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box);
}

// Rows that see no key (Nk == 0): O = 0 and LSE = -inf for batches
// [b0, b0 + nb) and query heads [h0, h0 + nh) of the [B, Nq, Hq, d] output.
__global__ void empty_rows_kernel(__nv_bfloat16* o, float* lse, int Nq, int Hq, int d, int b0, int nb, int h0,
                                  int nh) {
  const long long rows = (long long)nb * Nq * nh;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < rows * d; i += stride) {
    const long long r = i / d;
    const int c = (int)(i - r * d), h = h0 + (int)(r % nh);
    const long long bi = r / nh;
    const int b = b0 + (int)(bi / Nq), row = (int)(bi % Nq);
    o[(((long long)b * Nq + row) * Hq + h) * d + c] = __float2bfloat16(0.f);
    if (lse != nullptr && c == 0) lse[((long long)b * Hq + h) * Nq + row] = -INFINITY;
  }
}

__global__ void unsatisfied_wait_kernel(unsigned int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t mbar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&mbar), 1);  // one arrival expected; none ever comes
    abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{&abort_flag, err, limit_ns};
    wait_bar(ptx::smem_u32(&mbar), 0u, wc, kSiteProbe);
  }
  __syncthreads();
}

__global__ void exp2_probe_kernel(const float* x, float* y, long long n, int mode) {
  const long long i = 2 * (blockIdx.x * (long long)blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  float ya, yb;
  if (mode == 1) {
    exp2_soft2(a, b, ya, yb);
  } else {
    ya = ptx::ex2(a);
    yb = ptx::ex2(b);
  }
  y[i] = ya;
  if (i + 1 < n) y[i + 1] = yb;
}

// The part of a call's problem one launch computes: batches [b0, b0 + nb) and
// query heads [h0, h0 + nh) (whole key/value groups).
struct Part {
  int b0, nb, h0, nh;
};

// Fills the parameters both kernels share; false when the work items do not
// fit the kernels' int indexing.
template <class Cfg>
bool fill_params(FwdParams* p, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                 const float* dq, const float* dk, const float* dv, DeviceState* st, const Part& part) {
  p->o = o;
  p->lse = lse;
  p->B = B;
  p->Hq = Hq;
  p->Hkv = Hkv;
  p->Nq = Nq;
  p->Nk = Nk;
  p->group = Hq / Hkv;
  p->b0 = part.b0;
  p->nb = part.nb;
  p->h0 = part.h0;
  p->nh = part.nh;
  p->n_qblocks = (Nq + Cfg::BM * Cfg::NQT - 1) / (Cfg::BM * Cfg::NQT);
  const long long items = (long long)part.nb * part.nh * p->n_qblocks;
  if (items > 0x7FFFFFFFll) return false;
  p->n_items = (int)items;
  // causal blocks differ in length: the persistent kernel orders them
  // longest-first across heads when all of K and V fits comfortably in L2;
  // otherwise it keeps a head's query blocks together so that they share its
  // K/V tiles through L2
  const long long kv_bytes = 2ll * part.nb * Nk * (part.nh / p->group) * Cfg::D * Cfg::ELEM;
  p->qb_major = (Cfg::CAUSAL && kv_bytes <= (48ll << 20)) ? 1 : 0;
  p->band = 0;
  p->sl2 = scale * 1.4426950408889634f;
  p->dq = dq;
  p->dk = dk;
  p->dv = dv;
  p->err = st->err;
  p->timeout_ns = timeout_ns();
  p->n_splits = 1;
  p->kv_chunk = Nk;
  p->pack = 1;
  p->o_part = nullptr;
  p->lse_part = nullptr;
  return true;
}

template <class Cfg>
int encode_qkv(CUtensorMap* tq, CUtensorMap* tk, CUtensorMap* tv, const void* q, const void* k, const void* v,
               int B, int Hq, int Hkv, int Nq, int Nk) {
  if (encode_bnhd(tq, q, Cfg::FP8, B, Nq, Hq, Cfg::D, Cfg::BM) != ATTN_OK ||
      encode_bnhd(tk, k, Cfg::FP8, B, Nk, Hkv, Cfg::D, Cfg::BN) != ATTN_OK ||
      encode_bnhd(tv, v, Cfg::FP8, B, Nk, Hkv, Cfg::D, Cfg::BN) != ATTN_OK)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// Raises the kernel's dynamic shared memory limit once per device state (the
// attribute belongs to the context, so a rebuilt state sets it again;
// concurrent first calls from several host threads both set the same
// attribute, which is harmless).
template <class Kernel>
int set_smem_once(Kernel kernel, int bytes, std::atomic<unsigned> (&done)[kMaxDevices], const DeviceState* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  if (done[dev].load(std::memory_order_acquire) != st->gen) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return ATTN_ERR_CUDA;
    done[dev].store(st->gen, std::memory_order_release);
  }
  return ATTN_OK;
}

// One block per work item (batch, query head, query block).
template <class Cfg>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
               int Nk, float scale, const float* dq, const float* dk, const float* dv, DeviceState* st,
               cudaStream_t stream, const Part& part) {
  static std::atomic<unsigned> attr_set[kMaxDevices];
  int rc = set_smem_once(attn_fwd_kernel<Cfg>, (int)Cfg::SMEM_BYTES, attr_set, st);
  if (rc != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = encode_qkv<Cfg>(&tq, &tk, &tv, q, k, v, B, Hq, Hkv, Nq, Nk)) != ATTN_OK) return rc;
  FwdParams p;
  if (!fill_params<Cfg>(&p, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, part)) return ATTN_ERR_UNSUPPORTED;
  dim3 grid((unsigned)p.n_qblocks, (unsigned)part.nh, (unsigned)part.nb);
  if (Cfg::CAUSAL) {
    // causal blocks differ in length: longest first within bands of (batch,
    // head) pairs whose K and V together fit in about 48 MB of L2 (query heads
    // of one key/value group are adjacent, so a band holds whole groups'
    // worth of K/V); one 1-D grid
    const long long kv_pair = 2ll * Nk * Cfg::D * Cfg::ELEM / p.group;  // K/V bytes per query head
    long long band = (48ll << 20) / (kv_pair > 0 ? kv_pair : 1);
    const long long nbh = (long long)part.nb * part.nh;
    band = band < 1 ? 1 : (band > nbh ? nbh : band);
    p.band = (int)band;
    grid = dim3((unsigned)p.n_items, 1u, 1u);
  }
  log_launch<Cfg>("attn_fwd_kernel", grid, B, Hq, Hkv, Nq, Nk, Cfg::CAUSAL ? " (1-D grid, head bands)" : "");
  attn_fwd_kernel<Cfg><<<grid, Cfg::NTHREADS, Cfg::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// One block per SM, each looping over work items.
template <class Cfg>
int launch_fwd_persistent(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int Nq, int Nk, float scale, const float* dq, const float* dk, const float* dv,
                          DeviceState* st, cudaStream_t stream, const Part& part) {
  static std::atomic<unsigned> attr_set[kMaxDevices];
  int rc = set_smem_once(attn_fwd_persistent_kernel<Cfg>, (int)Cfg::SMEM_BYTES, attr_set, st);
  if (rc != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = encode_qkv<Cfg>(&tq, &tk, &tv, q, k, v, B, Hq, Hkv, Nq, Nk)) != ATTN_OK) return rc;
  FwdParams p;
  if (!fill_params<Cfg>(&p, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, part)) return ATTN_ERR_UNSUPPORTED;
  // the output map (staged output only; otherwise an unused copy of Q's)
  CUtensorMap to = tq;
  if (Cfg::OST && encode_bnhd(&to, o, false, B, Nq, Hq, Cfg::D, Cfg::BM) != ATTN_OK) return ATTN_ERR_CUDA;
  const int nstreams = (p.n_items + Cfg::NS - 1) / Cfg::NS;  // blocks that find work
  const int nblk = nstreams < st->num_sms ? nstreams : st->num_sms;
  log_launch<Cfg>("attn_fwd_persistent_kernel", dim3((unsigned)nblk), B, Hq, Hkv, Nq, Nk);
  attn_fwd_persistent_kernel<Cfg><<<dim3((unsigned)nblk), Cfg::NTHREADS, Cfg::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Split-KV partials: one block per (query block, head, batch x window),
// fp32 O_s and LSE_s into the caller's workspace.
template <class Cfg>
int launch_fwd_split(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int Hq,
                     int Hkv, int Nq, int Nk, float scale, int n_splits, int kv_chunk, int pack, DeviceState* st,
                     cudaStream_t stream) {
  static std::atomic<unsigned> attr_set[kMaxDevices];
  int rc = set_smem_once(attn_fwd_kernel<Cfg>, (int)Cfg::SMEM_BYTES, attr_set, st);
  if (rc != ATTN_OK) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = encode_qkv<Cfg>(&tq, &tk, &tv, q, k, v, B, Hq, Hkv, Nq, Nk)) != ATTN_OK) return rc;
  if (pack > 1 && (rc = encode_q_packed(&tq, q, B, Nq, Hkv, pack, Cfg::D, Cfg::BM)) != ATTN_OK) return rc;
  FwdParams p;
  if (!fill_params<Cfg>(&p, nullptr, nullptr, B, Hq, Hkv, Nq, Nk, scale, nullptr, nullptr, nullptr, st,
                        Part{0, B, 0, Hq}))
    return ATTN_ERR_UNSUPPORTED;
  p.n_splits = n_splits;
  p.kv_chunk = kv_chunk;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.pack = pack;
  if (pack > 1) p.n_qblocks = (int)(((long long)Nq * pack + Cfg::BM * Cfg::NQT - 1) / (Cfg::BM * Cfg::NQT));
  const dim3 grid((unsigned)p.n_qblocks, (unsigned)(pack > 1 ? Hkv : Hq), (unsigned)(B * n_splits));
  if (log_on()) {
    char extra[64];
    std::snprintf(extra, sizeof extra, " split-KV windows=%d chunk=%d pack=%d", n_splits, kv_chunk, pack);
    log_launch<Cfg>("attn_fwd_kernel", grid, B, Hq, Hkv, Nq, Nk, extra);
  }
  attn_fwd_kernel<Cfg><<<grid, Cfg::NTHREADS, Cfg::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// the long-range configurations with head packing compiled in; when a key/
// value group's (packed) query rows fit one 128-row tile, a block holds one
// query tile with two score buffers instead (Q K_{j+1}^T under the softmax of
// tile j), measured faster on decode shapes
template <bool C> using CfgSplitD64 = FwdCfg<64, 128, 2, 3, 3, C, false, 3, 1, false, 1, true>;
template <bool C> using CfgSplitD128 = FwdCfg<128, 128, 2, 2, 2, C, false, 2, 1, false, 1, true>;
template <bool C> using CfgSplitD64One = FwdCfg<64, 128, 1, 3, 3, C, false, 3, 2, false, 1, true>;
template <bool C> using CfgSplitD128One = FwdCfg<128, 128, 1, 2, 2, C, false, 2, 2, false, 1, true>;
template <bool C> using CfgSplitD256 = FwdCfg<256, 64, 1, 2, 2, C, false, 0, 2, false, 1, true>;

template <template <bool> class Cfg>
int launch_split_causal(bool causal, const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                        int B, int Hq, int Hkv, int Nq, int Nk, float scale, int n_splits, int kv_chunk, int pack,
                        DeviceState* st, cudaStream_t s) {
  return causal ? launch_fwd_split<Cfg<true>>(q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale, n_splits,
                                              kv_chunk, pack, st, s)
                : launch_fwd_split<Cfg<false>>(q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale, n_splits,
                                               kv_chunk, pack, st, s);
}

// Head packing for split-KV: the query heads of a key/value group share one
// query tile when the group size divides the 128-row tile.
int pack_factor(int Hq, int Hkv) {
  const int g = Hq / Hkv;
  return (g > 1 && 128 % g == 0) ? g : 1;
}

int launch_combine(const float* o_part, const float* lse_part, int S, int B, int Hq, int Nq, int d, void* o,
                   float* lse, cudaStream_t s) {
  const long long rows = (long long)B * Nq * Hq;
  const long long blocks = (rows * 32 + 255) / 256;
  if (blocks > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  auto* ob = reinterpret_cast<__nv_bfloat16*>(o);
  ATTN_LOGF("attn: attn_combine_kernel<%d> grid=(%lld) block=256 windows=%d B=%d Hq=%d Nq=%d\n", d, blocks, S, B, Hq,
            Nq);
  switch (d) {
    case 64: attn_combine_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(o_part, lse_part, S, B, Hq, Nq, ob, lse); break;
    case 128: attn_combine_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(o_part, lse_part, S, B, Hq, Nq, ob, lse); break;
    default: attn_combine_kernel<256><<<(unsigned)blocks, 256, 0, s>>>(o_part, lse_part, S, B, Hq, Nq, ob, lse); break;
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Split plan: windows of kv_chunk keys (a multiple of 128, so of every key
// tile) and the number of non-empty windows.  n_splits <= 0 asks for enough
// blocks to fill the GPU about twice, with windows of at least 512 keys.
struct SplitPlan {
  int n_splits, kv_chunk;
};
SplitPlan split_plan(int B, int Hq, int Hkv, int Nq, int Nk, int n_splits, int num_sms) {
  if (n_splits <= 0) {
    const int g = pack_factor(Hq, Hkv);
    const long long blocks = (long long)B * (Hq / g) * (((long long)Nq * g + 255) / 256);
    long long want = (2ll * num_sms + blocks - 1) / (blocks > 0 ? blocks : 1);
    const long long cap = Nk / 512 > 1 ? Nk / 512 : 1;
    want = want < 1 ? 1 : (want > cap ? cap : want);
    n_splits = (int)(want > 256 ? 256 : want);
  }
  if (n_splits > kMaxSplits) n_splits = kMaxSplits;
  const long long per = (Nk + n_splits - 1) / n_splits;
  const int chunk = (int)(((per + 127) / 128) * 128);
  const int eff = chunk > 0 ? (int)((Nk + chunk - 1) / chunk) : 1;
  return SplitPlan{eff < 1 ? 1 : eff, chunk > 0 ? chunk : 128};
}
long long splitkv_bytes(long long S, long long B, long long Hq, long long Nq, long long d) {
  const long long o_bytes = ((S * B * Nq * Hq * d * 4) + 255) / 256 * 256;
  return o_bytes + S * B * Hq * Nq * 4;
}

// Key ranges up to this length use the persistent kernel: their work items
// are short, and a persistent block overlaps an item's fixed costs (first
// loads, epilogue) with the neighbouring items instead of paying a block
// start for each.  Longer items run one block per item.
constexpr int kPersistentMaxNk = 1024;

// The kernel a key range runs on: persistent for short ranges, except causal
// launches at d = 128, where one block per item in longest-first order
// (the hardware hands the blocks out as SMs free up) balances the uneven
// causal items better (measured on B200: N = 512 causal 271 -> 323 TFLOP/s,
// N = 1024 causal 466 -> 524; d = 64 keeps the persistent kernel, 262 vs 232
// on the GPT-2 shape).
bool use_persistent(int Nk, int d, bool causal) { return Nk <= kPersistentMaxNk && !(causal && d == 128); }

// Kernel configurations, FwdCfg<D, BN, NQT, KST, VST, CAUSAL, FP8, EMU, SB,
// PSEP, NS>: per head size a long-range one (one block per item) and a
// short-range one (persistent).  EMU is the share of softmax exponentials
// computed in software (out of 8 element pairs), chosen by measurement.
//   d = 64 short: two independent streams of one 128-row query tile each; P
//   in columns of its own (S 128 + P 64 + O 64 = 256 columns per stream);
//   each output tile staged in shared memory for one TMA store (K ring of 2
//   and V ring of 3 stages leave room for it); every exponential on the
//   hardware unit (a software share measured slower at d = 64, where the
//   exponentials are a small part of a key tile's time).
template <bool C> using CfgD64 = FwdCfg<64, 128, 2, 3, 3, C, false, 3>;
template <bool C> using CfgD64Short = FwdCfg<64, 128, 1, 2, 3, C, false, 0, 1, true, 2, false, true>;
template <bool C> using CfgD128 = FwdCfg<128, 128, 2, 2, 2, C, false, C ? 2 : 1>;
template <bool C> using CfgD128Short = FwdCfg<128, 128, 2, 2, 2, C, false, 0>;
template <bool C> using CfgD256 = FwdCfg<256, 64, 1, 2, 2, C, false, 0>;
template <bool C> using CfgFP8 = FwdCfg<128, 128, 2, 3, 3, C, true, 2>;

template <template <bool> class Long, template <bool> class Short>
int launch_sched(bool causal, const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                 int Hkv, int Nq, int Nk, float scale, const float* dq, const float* dk, const float* dv,
                 DeviceState* st, cudaStream_t s, const Part& pt) {
  const bool persist = use_persistent(Nk, Long<false>::D, causal);
  if (causal)
    return persist
               ? launch_fwd_persistent<Short<true>>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, s, pt)
               : launch_fwd<Long<true>>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, s, pt);
  return persist
             ? launch_fwd_persistent<Short<false>>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, s, pt)
             : launch_fwd<Long<false>>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, s, pt);
}

int check_common(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                 int Nk, int causal, float scale) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || Nq == 0) return -1;  // nothing to compute
  if (Hkv == 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (o == nullptr || (Nk > 0 && (q == nullptr || k == nullptr || v == nullptr))) return ATTN_ERR_INVALID_ARG;
  if (B > 65535 || Hq > 65535) return ATTN_ERR_UNSUPPORTED;  // grid y / z limits
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  return ATTN_OK;
}

__global__ void set_float_kernel(float* p, float v) { *p = v; }

// FP8 preparation of one tensor [rows, 128] (both entry points): clear the
// amax word, the amax pass, the quantising pass.  `amax` is one word of
// device scratch (the caller's workspace or the library's static array).
template <bool ROT>
int launch_prep_passes(const CUtensorMap& tx, const CUtensorMap& tx8, const PrepParams& p, DeviceState* st,
                       cudaStream_t s) {
  static std::atomic<unsigned> attr_a[kMaxDevices], attr_q[kMaxDevices];
  int rc;
  if ((rc = set_smem_once(fp8_prep_kernel<ROT, false>, (int)PrepCfg<false>::SMEM_BYTES, attr_a, st)) != ATTN_OK ||
      (rc = set_smem_once(fp8_prep_kernel<ROT, true>, (int)PrepCfg<true>::SMEM_BYTES, attr_q, st)) != ATTN_OK)
    return rc;
  const int ga = p.n_tiles < PrepCfg<false>::BLOCKS_PER_SM * st->num_sms ? p.n_tiles
                                                                        : PrepCfg<false>::BLOCKS_PER_SM * st->num_sms;
  const int gq = p.n_tiles < PrepCfg<true>::BLOCKS_PER_SM * st->num_sms ? p.n_tiles
                                                                       : PrepCfg<true>::BLOCKS_PER_SM * st->num_sms;
  ATTN_LOGF("attn: fp8_prep_kernel<rotate=%d> amax pass grid=(%d) + quantising pass grid=(%d) block=%d rows=%lld\n",
            (int)ROT, ga, gq, kPrepRows, (long long)p.rows);
  fp8_prep_kernel<ROT, false><<<ga, kPrepRows, PrepCfg<false>::SMEM_BYTES, s>>>(tx, tx8, p);
  fp8_prep_kernel<ROT, true><<<gq, kPrepRows, PrepCfg<true>::SMEM_BYTES, s>>>(tx, tx8, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int launch_prep(const void* x, void* x8, float* descale, unsigned int* amax, long long rows, const float* signs,
                DeviceState* st, cudaStream_t s) {
  if (rows == 0) {  // amax of nothing is 0: descale 1, as for an all-zero tensor
    set_float_kernel<<<1, 1, 0, s>>>(descale, 1.0f);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
  }
  if (rows > 0x7FFFFFFFll - kPrepRows) return ATTN_ERR_UNSUPPORTED;  // tile coordinates are int
  CUtensorMap tx, tx8;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kPrepD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kPrepD * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)kPrepRows};
    if (encode_cached(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, strides, box) != ATTN_OK)
      return ATTN_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)kPrepD, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kPrepD};
    const cuuint32_t box[2] = {(cuuint32_t)kPrepD, (cuuint32_t)kPrepRows};
    if (encode_cached(&tx8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, x8, dims, strides, box) != ATTN_OK)
      return ATTN_ERR_CUDA;
  }
  PrepParams p;
  p.rows = rows;
  p.n_tiles = (int)((rows + kPrepRows - 1) / kPrepRows);
  p.signs = signs;
  p.amax_bits = amax;
  p.descale = descale;
  p.err = st->err;
  p.timeout_ns = timeout_ns();
  if (cudaMemsetAsync(amax, 0, sizeof(unsigned int), s) != cudaSuccess) return ATTN_ERR_CUDA;
  return signs != nullptr ? launch_prep_passes<true>(tx, tx8, p, st, s) : launch_prep_passes<false>(tx, tx8, p, st, s);
}

int fill_empty(void* o, float* lse, int B, int Hq, int Nq, int d, const Part& pt, cudaStream_t s) {
  empty_rows_kernel<<<256, 256, 0, s>>>(reinterpret_cast<__nv_bfloat16*>(o), lse, Nq, Hq, d, pt.b0, pt.nb, pt.h0,
                                        pt.nh);
  (void)B;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The forward over one part of the problem, after the argument checks: the
// kernel configuration for (d, dtype), short key ranges on the persistent
// kernel.  fp8: E4M3 inputs with device descales dq, dk, dv.
int fwd_checked(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                int Nk, int d, bool causal, float scale, bool fp8, const float* dq, const float* dk,
                const float* dv, const Part& pt, DeviceState* st, cudaStream_t s) {
  if (pt.nb == 0 || pt.nh == 0) return ATTN_OK;
  if (Nk == 0) return fill_empty(o, lse, B, Hq, Nq, d, pt, s);
  if (fp8) return launch_sched<CfgFP8, CfgFP8>(causal, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, dq, dk, dv, st, s, pt);
  switch (d) {
    case 64:
      return launch_sched<CfgD64, CfgD64Short>(causal, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, nullptr, nullptr,
                                               nullptr, st, s, pt);
    case 128:
      return launch_sched<CfgD128, CfgD128Short>(causal, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, nullptr, nullptr,
                                                 nullptr, st, s, pt);
    default:
      return launch_sched<CfgD256, CfgD256>(causal, q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, nullptr, nullptr,
                                            nullptr, st, s, pt);
  }
}

// Contiguous share of the B x Hkv (batch, key/value head) units, batch-major,
// as up to three rectangles [b0, b1) x [g0, g1).
int shard_rects(int B, int Hkv, int world, int rank, int* r) {
  const long long U = (long long)B * Hkv;
  const long long u0 = U * rank / world, u1 = U * (rank + 1) / world;
  if (u0 >= u1) return 0;
  const int bs = (int)(u0 / Hkv), gs = (int)(u0 % Hkv);
  const int be = (int)((u1 - 1) / Hkv), ge = (int)((u1 - 1) % Hkv) + 1;
  int n = 0;
  auto put = [&](int b0, int b1, int g0, int g1) {
    r[4 * n] = b0;
    r[4 * n + 1] = b1;
    r[4 * n + 2] = g0;
    r[4 * n + 3] = g1;
    ++n;
  };
  if (bs == be) {
    put(bs, bs + 1, gs, ge);
    return n;
  }
  int full0 = bs, full1 = be + 1;
  if (gs > 0) {
    put(bs, bs + 1, gs, Hkv);
    full0 = bs + 1;
  }
  if (ge < Hkv) full1 = be;
  if (full0 < full1) put(full0, full1, 0, Hkv);
  if (ge < Hkv) put(be, be + 1, 0, ge);
  return n;
}

// Streams and events of the host-buffer pipeline (attn_fwd_host), one set per
// device, created at the first call in the device's current context and
// rebuilt when the context changes (the old handles died with it).  The
// events are shared by successive calls: each call enqueues under the
// device's pipeline mutex, and a stream wait binds to the record made just
// before it, so a later call re-recording an event cannot disturb an earlier
// call's dependencies.
constexpr int kMaxChunks = 64;
struct Pipe {
  CUcontext ctx = nullptr;
  cudaStream_t in = nullptr, out = nullptr;  // host-to-device and device-to-host copies
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_done[kMaxChunks] = {}, comp_done[kMaxChunks] = {};
};
Pipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu[kMaxDevices];

int pipe_get(int dev, const DeviceState* st, Pipe** out) {
  Pipe& pp = g_pipe[dev];
  if (pp.ctx != st->ctx) {
    Pipe fresh;
    auto ev = [](cudaEvent_t* e) { return cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess; };
    bool ok = cudaStreamCreateWithFlags(&fresh.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&fresh.out, cudaStreamNonBlocking) == cudaSuccess && ev(&fresh.start) &&
              ev(&fresh.end);
    for (int c = 0; ok && c < kMaxChunks; ++c) ok = ev(&fresh.in_done[c]) && ev(&fresh.comp_done[c]);
    if (!ok) return ATTN_ERR_CUDA;
    fresh.ctx = st->ctx;
    pp = fresh;
  }
  *out = &pp;
  return ATTN_OK;
}

// One strided block of rows between host and device: `rows` rows of `width`
// bytes, `pitch` bytes apart in both buffers, starting `off` bytes in.
cudaError_t copy_rows(void* dst, const void* src, size_t off, size_t width, size_t pitch, size_t rows,
                      cudaMemcpyKind kind, cudaStream_t s) {
  if (width == 0 || rows == 0) return cudaSuccess;
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + off, pitch, static_cast<const char*>(src) + off, pitch, width,
                           rows, kind, s);
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case ATTN_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int attn_kv_tile_count(int row0, int row1, int Nq, int Nk, int bn, int causal) {
  if (row0 < 0 || row1 < row0 || Nq < 0 || Nk < 0 || bn <= 0 || (causal != 0 && causal != 1)) return -1;
  return kv_tile_count(row0, row1, Nq, Nk, bn, causal != 0);
}

int attn_fwd_schedule(int Nk, int d, int causal) {
  if (Nk < 0 || (d != 64 && d != 128 && d != 256) || (causal != 0 && causal != 1)) return -1;
  return use_persistent(Nk, d, causal != 0) ? 1 : 0;
}

int attn_tile_kind(int row0, int row1, int kt, int Nq, int Nk, int bn, int causal) {
  if (row0 < 0 || row1 < row0 || kt < 0 || Nq < 0 || Nk < 0 || bn <= 0 || (causal != 0 && causal != 1)) return -1;
  return tile_kind(row0, row1, kt, Nq, Nk, bn, causal != 0);
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk,
             int d, int causal, float scale, int dtype, void* stream) {
  return attn_fwd_part(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dtype, 0, B, 0, Hkv, stream);
}

int attn_fwd_part(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                  int Nk, int d, int causal, float scale, int dtype, int b_begin, int b_end, int kvh_begin,
                  int kvh_end, void* stream) {
  if (dtype != ATTN_BF16 && dtype != ATTN_FP8_E4M3) return ATTN_ERR_INVALID_ARG;
  int rc = check_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, causal, scale);
  if (rc == -1) return ATTN_OK;
  if (rc != ATTN_OK) return rc;
  if (b_begin < 0 || b_end < b_begin || b_end > B || kvh_begin < 0 || kvh_end < kvh_begin || kvh_end > Hkv)
    return ATTN_ERR_INVALID_ARG;
  const bool fp8 = dtype == ATTN_FP8_E4M3;
  if (fp8 ? d != 128 : (d != 64 && d != 128 && d != 256)) return ATTN_ERR_UNSUPPORTED;
  int dev = 0;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  const int g = Hq / Hkv;
  const Part pt{b_begin, b_end - b_begin, kvh_begin * g, (kvh_end - kvh_begin) * g};
  // e4m3 inputs with unit scales read the library's device constant 1.0
  const float* u = fp8 ? st->unit_descale : nullptr;
  return fwd_checked(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal != 0, scale, fp8, u, u, u, pt, st,
                     static_cast<cudaStream_t>(stream));
}

int attn_shard_units(int B, int Hkv, int world, int rank, int* rects) {
  if (B < 0 || Hkv < 0 || world < 1 || rank < 0 || rank >= world || rects == nullptr) return -1;
  return shard_rects(B, Hkv, world, rank, rects);
}

int attn_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h, void* q_d, void* k_d,
                  void* v_d, void* o_d, float* lse_d, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                  float scale, int n_chunks, void* stream) {
  if (q_h == nullptr || o_h == nullptr || (Nk > 0 && (k_h == nullptr || v_h == nullptr)) || n_chunks < 0 ||
      (lse_h != nullptr && lse_d == nullptr))
    return ATTN_ERR_INVALID_ARG;
  int rc = check_common(q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, Nq, Nk, causal, scale);
  if (rc == -1) return ATTN_OK;
  if (rc != ATTN_OK) return rc;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  int dev = 0;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  std::lock_guard<std::mutex> lk(g_pipe_mu[dev]);
  Pipe* pp = nullptr;
  if ((rc = pipe_get(dev, st, &pp)) != ATTN_OK) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long units = (long long)B * Hkv;
  long long nc = n_chunks == 0 ? 8 : n_chunks;
  nc = nc > units ? units : nc;
  nc = nc > kMaxChunks ? kMaxChunks : nc;
  const int C = (int)nc, g = Hq / Hkv;
  const size_t es = 2;  // bf16
  const size_t qpitch = (size_t)Hq * d * es, kpitch = (size_t)Hkv * d * es, lpitch = (size_t)Hq * Nq * 4;
#define ATTN_CK(x)                                   \
  do {                                               \
    if ((x) != cudaSuccess) return ATTN_ERR_CUDA; \
  } while (0)
  // the copies start after the work already on `stream`
  ATTN_CK(cudaEventRecord(pp->start, s));
  ATTN_CK(cudaStreamWaitEvent(pp->in, pp->start, 0));
  ATTN_CK(cudaStreamWaitEvent(pp->out, pp->start, 0));
  for (int c = 0; c < C; ++c) {
    int r[12];
    const int nr = shard_rects(B, Hkv, C, c, r);
    for (int i = 0; i < nr; ++i) {  // in: this chunk's heads of every row of Q, K, V
      const size_t b0 = (size_t)r[4 * i], nb = (size_t)(r[4 * i + 1] - r[4 * i]);
      const size_t g0 = (size_t)r[4 * i + 2], ng = (size_t)(r[4 * i + 3] - r[4 * i + 2]);
      ATTN_CK(copy_rows(q_d, q_h, (b0 * Nq * Hq + g0 * g) * d * es, ng * g * d * es, qpitch, nb * Nq,
                        cudaMemcpyHostToDevice, pp->in));
      if (Nk > 0) {
        const size_t koff = (b0 * Nk * Hkv + g0) * d * es;
        ATTN_CK(copy_rows(k_d, k_h, koff, ng * d * es, kpitch, nb * Nk, cudaMemcpyHostToDevice, pp->in));
        ATTN_CK(copy_rows(v_d, v_h, koff, ng * d * es, kpitch, nb * Nk, cudaMemcpyHostToDevice, pp->in));
      }
    }
    ATTN_CK(cudaEventRecord(pp->in_done[c], pp->in));
    ATTN_CK(cudaStreamWaitEvent(s, pp->in_done[c], 0));
    for (int i = 0; i < nr; ++i) {
      const Part pt{r[4 * i], r[4 * i + 1] - r[4 * i], r[4 * i + 2] * g, (r[4 * i + 3] - r[4 * i + 2]) * g};
      if ((rc = fwd_checked(q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, Nq, Nk, d, causal != 0, scale, false, nullptr,
                            nullptr, nullptr, pt, st, s)) != ATTN_OK)
        return rc;
    }
    ATTN_CK(cudaEventRecord(pp->comp_done[c], s));
    ATTN_CK(cudaStreamWaitEvent(pp->out, pp->comp_done[c], 0));
    for (int i = 0; i < nr; ++i) {  // out: this chunk's O rows (and LSE entries)
      const size_t b0 = (size_t)r[4 * i], nb = (size_t)(r[4 * i + 1] - r[4 * i]);
      const size_t g0 = (size_t)r[4 * i + 2], ng = (size_t)(r[4 * i + 3] - r[4 * i + 2]);
      ATTN_CK(copy_rows(o_h, o_d, (b0 * Nq * Hq + g0 * g) * d * es, ng * g * d * es, qpitch, nb * Nq,
                        cudaMemcpyDeviceToHost, pp->out));
      if (lse_h != nullptr)
        ATTN_CK(copy_rows(lse_h, lse_d, (b0 * Hq + g0 * g) * Nq * 4, ng * g * Nq * 4, lpitch, nb,
                          cudaMemcpyDeviceToHost, pp->out));
    }
  }
  // `stream` completes only after the last copy out
  ATTN_CK(cudaEventRecord(pp->end, pp->out));
  ATTN_CK(cudaStreamWaitEvent(s, pp->end, 0));
#undef ATTN_CK
  return ATTN_OK;
}

int attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                 int Nk, int d, int causal, float scale, const float* descale_q, const float* descale_k,
                 const float* descale_v, void* stream) {
  int rc = check_common(q8, k8, v8, o, lse, B, Hq, Hkv, Nq, Nk, causal, scale);
  if (rc == -1) return ATTN_OK;
  if (rc != ATTN_OK) return rc;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Nk > 0 && (descale_q == nullptr || descale_k == nullptr || descale_v == nullptr)) return ATTN_ERR_INVALID_ARG;
  int dev = 0;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  return fwd_checked(q8, k8, v8, o, lse, B, Hq, Hkv, Nq, Nk, d, causal != 0, scale, true, descale_q, descale_k,
                     descale_v, Part{0, B, 0, Hq}, st, static_cast<cudaStream_t>(stream));
}

long long attn_splitkv_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int n_splits) {
  if (B < 0 || Hq < 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq < 0 || Nk < 0 || (d != 64 && d != 128 && d != 256))
    return -1;
  if (B == 0 || Hq == 0 || Nq == 0 || Nk == 0) return 0;
  int num_sms = 148;
  if (n_splits <= 0) {
    int dev = 0;
    DeviceState* st = nullptr;
    if (device_state(&dev, &st) != ATTN_OK) return -1;
    num_sms = st->num_sms;
  }
  const SplitPlan sp = split_plan(B, Hq, Hkv, Nq, Nk, n_splits, num_sms);
  if (sp.n_splits == 1) return 0;
  return splitkv_bytes(sp.n_splits, B, Hq, Nq, d);
}

int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int Nq, int Nk, int d, int causal, float scale, int n_splits, void* workspace,
                     long long workspace_bytes, void* stream) {
  int rc = check_common(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, causal, scale);
  if (rc == -1) return ATTN_OK;
  if (rc != ATTN_OK) return rc;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  int dev = 0;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (Nk == 0) return fill_empty(o, lse, B, Hq, Nq, d, Part{0, B, 0, Hq}, s);
  const SplitPlan sp = split_plan(B, Hq, Hkv, Nq, Nk, n_splits, st->num_sms);
  if (sp.n_splits == 1) return attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, ATTN_BF16, stream);
  if ((long long)B * sp.n_splits > 65535) return ATTN_ERR_UNSUPPORTED;  // grid z
  const long long need = splitkv_bytes(sp.n_splits, B, Hq, Nq, d);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             ((long long)sp.n_splits * B * Nq * Hq * d * 4 + 255) / 256 * 256);
  const bool c = causal != 0;
  const int g = pack_factor(Hq, Hkv);
  const bool one_tile = (long long)Nq * g <= 128;
  switch (d) {
    case 64:
      rc = one_tile ? launch_split_causal<CfgSplitD64One>(c, q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale,
                                                          sp.n_splits, sp.kv_chunk, g, st, s)
                    : launch_split_causal<CfgSplitD64>(c, q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale,
                                                       sp.n_splits, sp.kv_chunk, g, st, s);
      break;
    case 128:
      rc = one_tile ? launch_split_causal<CfgSplitD128One>(c, q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale,
                                                           sp.n_splits, sp.kv_chunk, g, st, s)
                    : launch_split_causal<CfgSplitD128>(c, q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale,
                                                        sp.n_splits, sp.kv_chunk, g, st, s);
      break;
    default:
      rc = launch_split_causal<CfgSplitD256>(c, q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, scale, sp.n_splits,
                                             sp.kv_chunk, g, st, s);
      break;
  }
  if (rc != ATTN_OK) return rc;
  return launch_combine(o_part, lse_part, sp.n_splits, B, Hq, Nq, d, o, lse, s);
}

int attn_combine(const float* o_parts, const float* lse_parts, int n_splits, int B, int Hq, int Nq, int d, void* o,
                 float* lse, void* stream) {
  if (n_splits < 1 || B < 0 || Hq < 0 || Nq < 0) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || Hq == 0 || Nq == 0) return ATTN_OK;
  if (o_parts == nullptr || lse_parts == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse_parts) & 3u) != 0 ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0))
    return ATTN_ERR_MISALIGNED;
  int dev = 0;
  DeviceState* st = nullptr;
  int rc = device_state(&dev, &st);
  if (rc != ATTN_OK) return rc;
  return launch_combine(o_parts, lse_parts, n_splits, B, Hq, Nq, d, o, lse, static_cast<cudaStream_t>(stream));
}

int attn_kv_tile_count_window(int row0, int row1, int Nq, int Nk, int shift, int bn, int causal) {
  if (row0 < 0 || row1 < row0 || Nq < 0 || Nk < 0 || shift < 0 || bn <= 0 || (causal != 0 && causal != 1)) return -1;
  return kv_tile_count(row0, row1, Nq, Nk, bn, causal != 0, shift);
}

int attn_tile_kind_window(int row0, int row1, int kt, int Nq, int Nk, int shift, int bn, int causal) {
  if (row0 < 0 || row1 < row0 || kt < 0 || Nq < 0 || Nk < 0 || shift < 0 || bn <= 0 ||
      (causal != 0 && causal != 1))
    return -1;
  return tile_kind(row0, row1, kt, Nq, Nk, bn, causal != 0, shift);
}

int attn_gemm_add(const void* a, const void* b, const void* c, void* d, int M, int N, int K, void* stream) {
  if (M < 0 || N < 0 || K < 0) return ATTN_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return ATTN_OK;
  if (d == nullptr || (K > 0 && (a == nullptr || b == nullptr))) return ATTN_ERR_INVALID_ARG;
  if (N % 8 != 0 || K % 8 != 0) return ATTN_ERR_UNSUPPORTED;  // 16-byte row strides for TMA and vector access
  if ((K > 0 && (!aligned16(a) || !aligned16(b))) || (c != nullptr && !aligned16(c)) || !aligned16(d))
    return ATTN_ERR_MISALIGNED;
  if (c != nullptr && c != d) {  // C may be D itself, but not partly overlap it
    const uintptr_t cb = reinterpret_cast<uintptr_t>(c), db = reinterpret_cast<uintptr_t>(d);
    const uintptr_t bytes = (uintptr_t)M * (uintptr_t)N * 2u;
    if (cb < db + bytes && db < cb + bytes) return ATTN_ERR_INVALID_ARG;
  }
  int dev = 0;
  DeviceState* st = nullptr;
  int rc = device_state(&dev, &st);
  if (rc != ATTN_OK) return rc;
  static std::atomic<unsigned> attr_set[kMaxDevices];
  if ((rc = set_smem_once(gemm_add_kernel, (int)GemmCfg::SMEM_BYTES, attr_set, st)) != ATTN_OK) return rc;
  CUtensorMap ta, tb, tc, td;
  std::memset(&ta, 0, sizeof(ta));
  std::memset(&tb, 0, sizeof(tb));
  std::memset(&tc, 0, sizeof(tc));
  if (K > 0 && (encode_rows(&ta, a, M, K, GemmCfg::BM) != ATTN_OK || encode_rows(&tb, b, K, N, GemmCfg::BK) != ATTN_OK))
    return ATTN_ERR_CUDA;
  // C and D move by 2-D tiled TMA (the kernel's loads and stores of them are
  // .2d operations): rank-2 maps, boxes of 64 columns x 128 rows
  if ((c != nullptr && encode_rows_2d(&tc, c, M, N, GemmCfg::BM) != ATTN_OK) ||
      encode_rows_2d(&td, d, M, N, GemmCfg::BM) != ATTN_OK)
    return ATTN_ERR_CUDA;
  GemmParams p;
  p.has_c = c != nullptr ? 1 : 0;
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_m = (M + GemmCfg::BM - 1) / GemmCfg::BM;
  const long long tiles = (long long)p.tiles_m * ((N + GemmCfg::BN - 1) / GemmCfg::BN);
  if (tiles > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  p.n_tiles = (int)tiles;
  p.k_steps = (K + GemmCfg::BK - 1) / GemmCfg::BK;
  p.err = st->err;
  p.timeout_ns = timeout_ns();
  const int nblk = p.n_tiles < st->num_sms ? p.n_tiles : st->num_sms;
  ATTN_LOGF("attn: gemm_add_kernel grid=(%d) block=%d smem=%u M=%d N=%d K=%d C=%s tiles=%d\n", nblk, GemmCfg::NTHREADS,
            (unsigned)GemmCfg::SMEM_BYTES, M, N, K, c != nullptr ? "yes" : "no", p.n_tiles);
  gemm_add_kernel<<<dim3((unsigned)nblk), GemmCfg::NTHREADS, GemmCfg::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(
      ta, tb, tc, td, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

long long attn_hadamard_quant_fp8_workspace_bytes(void) { return 256; }

int attn_hadamard_quant_fp8(const void* x, void* x8, float* descale, void* workspace, long long rows, int d,
                            const float* signs, void* stream) {
  if (rows < 0) return ATTN_ERR_INVALID_ARG;
  if (d != kPrepD) return ATTN_ERR_UNSUPPORTED;
  if (x == nullptr || x8 == nullptr || descale == nullptr || workspace == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(workspace) || !aligned16(signs) ||
      (reinterpret_cast<uintptr_t>(descale) & 3u) != 0)
    return ATTN_ERR_MISALIGNED;
  int dev = 0, rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  return launch_prep(x, x8, descale, static_cast<unsigned int*>(workspace), rows, signs, st,
                     static_cast<cudaStream_t>(stream));
}

int attn_hadamard_quant_fp8_noalloc(const void* x, void* x8, float* descale, long long rows, int d,
                                    const float* signs, void* stream) {
  // Same checks as attn_hadamard_quant_fp8, minus the workspace.
  if (rows < 0) return ATTN_ERR_INVALID_ARG;
  if (d != kPrepD) return ATTN_ERR_UNSUPPORTED;
  if (x == nullptr || x8 == nullptr || descale == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(signs) || (reinterpret_cast<uintptr_t>(descale) & 3u) != 0)
    return ATTN_ERR_MISALIGNED;
  // The scratch this call needs must fit the static array.
  if (attn_hadamard_quant_fp8_workspace_bytes() > (long long)kNoAllocScratchBytes) return ATTN_ERR_UNSUPPORTED;
  int dev = 0, rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  // Host code cannot use g_noalloc_scratch's name as a device address: its
  // address was looked up by device_state, once per device (and context), with
  // that device current (the first call on a device does this).
  // launch_prep clears the word it uses (the array keeps the previous call's
  // maximum) before the amax pass.
  return launch_prep(x, x8, descale, st->noalloc_scratch, rows, signs, st, static_cast<cudaStream_t>(stream));
}

int attn_get_last_device_error(void* stream, unsigned int* detail) {
  int dev = 0, rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpy(&word, st->err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  const unsigned int zero = 0;
  if (word != 0 && cudaMemcpy(st->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (detail != nullptr) *detail = word;
  return word != 0 ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
}

int attn_debug_map_cache_stats(unsigned long long* hits, unsigned long long* encodes) {
  if (hits == nullptr || encodes == nullptr) return ATTN_ERR_INVALID_ARG;
  *hits = g_map_hits.load(std::memory_order_relaxed);
  *encodes = g_map_encodes.load(std::memory_order_relaxed);
  return ATTN_OK;
}

int attn_debug_exp2(const float* x, float* y, long long n, int mode, void* stream) {
  if (n < 0 || (mode != 0 && mode != 1) || (n > 0 && (x == nullptr || y == nullptr))) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  int dev = 0, rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  const long long pairs = (n + 1) / 2;
  exp2_probe_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, mode);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int attn_debug_unsatisfied_wait(long long limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 10000000000ll) return ATTN_ERR_INVALID_ARG;
  int dev = 0, rc;
  DeviceState* st = nullptr;
  if ((rc = device_state(&dev, &st)) != ATTN_OK) return rc;
  unsatisfied_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(st->err, (unsigned long long)limit_ns);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"
