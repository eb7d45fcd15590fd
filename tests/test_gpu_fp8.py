"""FP8 path (page "FlashAttention-3 — 闪电注意力-3", section 3): the Hadamard
rotation + per-tensor E4M3 quantiser, and the FP8 attention kernel, against the
fp64 oracle.

* quantiser without rotation: bit-exact against the oracle's fp32 quantiser
  on the same fp32 inputs (the bf16 values, exactly representable);
* quantiser with rotation: the oracle rotates in fp64, the kernel in fp32,
  so a code may differ by one step where the value sits at a rounding midpoint;
* attention: the kernel (quantising on the GPU) against the oracle running
  the same method in fp64 (rotate, quantise per tensor, attend on the
  dequantised values): mean |dO| <= 3e-2, the stated FP8 bar.  What is left
  between the two is P rounded to E4M3 in the kernel (relative <= 2^-4 per
  weight) and the rare one-step code differences above.
* accuracy of the method itself against exact attention of the original bf16
  inputs is reported (rotated and unrotated, workload with 1 % outlier
  channels x20); the rotation must lower it.  It is not held to 3e-2: on this
  workload the fp64 oracle of the same method is itself about 3-4e-2 away from
  exact attention (per-tensor E4M3 keeps 3 mantissa bits; where Q and K share
  an outlier channel the scores reach ~35 and the softmax is nearly one-hot).
"""
import math

import numpy as np
import pytest

import attn_inputs as gen
import oracle
from gpu_util import bf16_dev_to_f64, bf16_ulp, to_dev_bf16

pytestmark = pytest.mark.gpu

# mean |dO| of the FP8 kernel against the fp64 definition on the kernel's own
# codes, relative to the mean of the |V| attention A (see check_fp8_parity)
FP8_PARITY_MEAN_REL = 1e-2


def torch():
    import torch as t
    return t


def quantise_gpu(xb, signs=None):
    """xb: bf16 bits [..., 128] -> (codes uint8 [...,128], descale float)."""
    import exact_attention_140_b200 as ea
    T = torch()
    x = to_dev_bf16(xb)
    rows = x.numel() // 128
    x8 = T.empty(x.shape, dtype=T.uint8, device="cuda")
    desc = T.empty(1, dtype=T.float32, device="cuda")
    ws = T.empty(ea.attn_hadamard_quant_fp8_workspace_bytes(), dtype=T.uint8, device="cuda")
    sg = None if signs is None else T.from_numpy(np.ascontiguousarray(signs, dtype=np.float32)).cuda()
    ea.attn_hadamard_quant_fp8(x, x8, desc, ws, rows, 128, sg)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    return x8.cpu().numpy(), float(desc.cpu().item())


def test_quantiser_no_rotation_bit_exact():
    xb = gen.normal_bf16(21, (2, 333, 4, 128), column_scale=gen.outlier_scale(22, 4, 128))
    codes, desc = quantise_gpu(xb)
    xf = gen.bf16_bits_to_f32(xb)
    amax = np.float32(np.max(np.abs(xf)))
    assert desc == np.float32(amax / np.float32(448.0))
    ref = oracle.quant_e4m3_f32(xf, float(amax))
    assert np.array_equal(codes, ref)


def test_quantiser_with_rotation():
    d = 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    xb = gen.normal_bf16(23, (1, 515, 3, d), column_scale=gen.outlier_scale(24, 3, d))
    codes, desc = quantise_gpu(xb, signs)
    ref_codes, ref_desc = oracle.fp8_prepare(gen.bf16_bits_to_f64(xb), signs.astype(np.float64))
    assert abs(desc - ref_desc) <= 1e-6 * ref_desc
    diff = codes != ref_codes
    assert diff.mean() <= 1e-3, diff.mean()
    # where they differ it is by one code step (same sign, adjacent magnitude)
    a, b = codes[diff].astype(int), ref_codes[diff].astype(int)
    assert np.all((a & 0x80) == (b & 0x80)) and np.all(np.abs((a & 0x7F) - (b & 0x7F)) == 1)


def test_rotation_preserves_scores_on_gpu_codes():
    """(QM)(KM)^T = QK^T: dequantised rotated codes reproduce the scores within FP8 error."""
    d = 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb = gen.normal_bf16(31, (64, d))
    kb = gen.normal_bf16(32, (64, d))
    q8, dq = quantise_gpu(qb, signs)
    k8, dk = quantise_gpu(kb, signs)
    s_fp8 = (oracle.e4m3_decode(q8) * dq) @ (oracle.e4m3_decode(k8) * dk).T
    s_ref = gen.bf16_bits_to_f64(qb) @ gen.bf16_bits_to_f64(kb).T
    assert np.sqrt(np.mean((s_fp8 - s_ref) ** 2)) <= 0.1 * np.sqrt(np.mean(s_ref ** 2))


def fp8_attention(qb, kb, vb, causal, signs, rotate=True, scale=None):
    """Quantise on the GPU (Q, K rotated when rotate; V plain) and run attn_fwd_fp8.
    Returns O, LSE (fp64) and the kernel's own inputs: the codes of Q, K, V and
    their three descales."""
    import exact_attention_140_b200 as ea
    T = torch()
    B, Nq, Hq, d = qb.shape
    Nk, Hkv = kb.shape[1], kb.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = {n: to_dev_bf16(a) for n, a in (("q", qb), ("k", kb), ("v", vb))}
    q8, k8, v8 = (T.empty(dev[n].shape, dtype=T.uint8, device="cuda") for n in "qkv")
    desc = T.empty(3, dtype=T.float32, device="cuda")
    wsb = ea.attn_hadamard_quant_fp8_workspace_bytes()
    ws = T.empty(3 * wsb, dtype=T.uint8, device="cuda")
    sg = T.from_numpy(np.ascontiguousarray(signs, dtype=np.float32)).cuda() if rotate else None
    ea.attn_hadamard_quant_fp8(dev["q"], q8, desc.data_ptr(), ws.data_ptr(), B * Nq * Hq, d, sg)
    ea.attn_hadamard_quant_fp8(dev["k"], k8, desc.data_ptr() + 4, ws.data_ptr() + wsb, B * Nk * Hkv, d, sg)
    ea.attn_hadamard_quant_fp8(dev["v"], v8, desc.data_ptr() + 8, ws.data_ptr() + 2 * wsb, B * Nk * Hkv, d, None)
    o = T.full((B, Nq, Hq, d), float("nan"), dtype=T.bfloat16, device="cuda")
    lse = T.empty((B, Hq, Nq), dtype=T.float32, device="cuda")
    ea.attn_fwd_fp8(q8, k8, v8, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, desc.data_ptr(),
                    desc.data_ptr() + 4, desc.data_ptr() + 8)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    codes = tuple(x.cpu().numpy() for x in (q8, k8, v8))
    return bf16_dev_to_f64(o), lse.double().cpu().numpy(), codes, desc.double().cpu().numpy()


def dequantised(codes, desc):
    """The real inputs the FP8 kernel attends over: code values times descales, fp64."""
    return tuple(oracle.e4m3_decode(c) * float(s) for c, s in zip(codes, desc))


def oracle_fp8_inputs(qb, kb, vb, signs, rotate=True):
    """The oracle's own FP8 preparation, dequantised: what the FP8 kernel should see."""
    sg = signs.astype(np.float64) if rotate else None
    q8, dq = oracle.fp8_prepare(gen.bf16_bits_to_f64(qb), sg)
    k8, dk = oracle.fp8_prepare(gen.bf16_bits_to_f64(kb), sg)
    v8, dv = oracle.fp8_prepare(gen.bf16_bits_to_f64(vb), None)
    return oracle.e4m3_decode(q8) * dq, oracle.e4m3_decode(k8) * dk, oracle.e4m3_decode(v8) * dv


def rounding_terms(qd, kd, vd, causal, scale, rows=None):
    """Per output element, the two sums that bound the effect of rounding the
    softmax weights to E4M3 (fp64, from the dequantised inputs):
        A  = sum_j w_j |v_j| / l                (l = sum_j w_j)
        A2 = sum_j min(w_j, 2^-10) |v_j| / l
    with w_j = exp(s_j - max s) over the visible keys.  rows: flat
    (b*Hq + h)*Nq + i indices (all rows when None).  Returns A, A2 shaped
    like O (or [len(rows), d])."""
    B, Nq, Hq, d = qd.shape
    Nk, Hkv = kd.shape[1], kd.shape[2]
    g = Hq // Hkv
    if rows is None:
        rows = np.arange(B * Hq * Nq)
    rows = np.asarray(rows)
    A = np.zeros((rows.size, d))
    A2 = np.zeros((rows.size, d))
    b, h, i = rows // (Hq * Nq), (rows // Nq) % Hq, rows % Nq
    for bb in np.unique(b):
        for hh in np.unique(h[b == bb]):
            sel = np.nonzero((b == bb) & (h == hh))[0]
            kh = hh // g
            s_ = scale * (qd[bb, i[sel], hh, :] @ kd[bb, :, kh, :].T)  # [rows, Nk]
            if causal:
                vis = np.arange(Nk)[None, :] <= (i[sel] + (Nk - Nq))[:, None]
                s_ = np.where(vis, s_, -np.inf)
            m = np.max(s_, axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            w = np.exp(s_ - m)
            l = np.sum(w, axis=1, keepdims=True)
            l = np.where(l > 0, l, 1.0)
            va = np.abs(vd[bb, :, kh, :])
            A[sel] = (w @ va) / l
            A2[sel] = (np.minimum(w, 2.0 ** -10) @ va) / l
    if rows.size == B * Hq * Nq and np.array_equal(rows, np.arange(rows.size)):
        # flat row order (b, h, i) -> O layout [B, Nq, Hq, d]
        A = A.reshape(B, Hq, Nq, d).transpose(0, 2, 1, 3)
        A2 = A2.reshape(B, Hq, Nq, d).transpose(0, 2, 1, 3)
    return A, A2


def fp8_max_bound(a_abs, a_sub, o_ref):
    """The E4M3 rounding of each kernel weight x (relative to the kernel's lazy
    reference max, x = c w with c in [1, 2^8]) errs by at most 2^-4 x
    (normal range) plus min(x, 2^-10) (subnormal range or flushed to zero);
    divided by the kernel's row sum c l that is at most 2^-4 w / l +
    min(w, 2^-10) / l.  On top: the exp2 approximations and the fp32 scores
    (relative 1e-3 of a weight, generously) and the final bf16 rounding of O
    (one ulp: the kernel value may sit on the other side of a midpoint)."""
    return (2.0 ** -4 + 1e-3) * a_abs + a_sub + bf16_ulp(o_ref)


def check_fp8_parity(o, lse, codes, desc, causal, scale):
    """The FP8 attention kernel against the fp64 definition evaluated on the
    kernel's own inputs (its codes and descales).  What separates the two is
    the kernel's P rounded to E4M3 before P V (round to nearest even), the
    exp2 approximations (relative <= 1.1e-4) and fp32 arithmetic; l sums the
    unrounded weights, so LSE carries only the exp2 and score errors.
    Bounds: every element within fp8_max_bound; mean |dO| <=
    FP8_PARITY_MEAN_REL * mean A (unbiased rounding averages out over the
    keys); |dLSE| <= 1e-3 (the BF16 bar)."""
    qd, kd, vd = dequantised(codes, desc)
    o_ref, lse_ref = oracle.attn_fwd(qd, kd, vd, causal, scale)
    a_abs, a_sub = rounding_terms(qd, kd, vd, causal, scale)
    assert np.all(np.isfinite(o))
    err = np.abs(o - o_ref)
    bound = fp8_max_bound(a_abs, a_sub, o_ref)
    rel_mean = err.mean() / a_abs.mean()
    empty = np.isneginf(lse_ref)
    dl = np.abs(lse[~empty] - lse_ref[~empty])
    print(f"FP8 parity: mean |dO| {err.mean():.3e} (mean A {a_abs.mean():.3e}, ratio {rel_mean:.3e}; "
          f"mean A2 {a_sub.mean():.3e}), max |dO|/bound {np.max(err / bound):.3f}, max |dLSE| {dl.max():.3e}")
    worst = np.argmax(err - bound)
    assert err.flat[worst] <= bound.flat[worst], (err.flat[worst], bound.flat[worst])
    assert np.array_equal(np.isneginf(lse), empty)
    assert rel_mean <= FP8_PARITY_MEAN_REL, rel_mean
    assert dl.max() <= 1e-3, dl.max()
    return err, o_ref


# Nk <= 1024 runs the persistent kernel, longer key ranges the one-block-per-item
# kernel (the one the full-size benchmark times); both, causal and not, ragged.
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 1024, 1100, 2048])
def test_fp8_attention_against_oracle(causal, N):
    d = 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb, kb, vb = gen.qkv_bf16(1, 4, 2, N, N, d, outliers=True)
    scale = 1.0 / math.sqrt(d)
    o, lse, codes, desc = fp8_attention(qb, kb, vb, causal, signs, scale=scale)
    err, o_q = check_fp8_parity(o, lse, codes, desc, causal, scale)
    o_x, _ = oracle.attn_fwd(*(gen.bf16_bits_to_f64(a) for a in (qb, kb, vb)), causal, scale)
    print(f"N={N} causal={causal}: kernel vs exact {np.abs(o - o_x).mean():.2e}, "
          f"fp64 on the kernel's codes vs exact {np.abs(o_q - o_x).mean():.2e}")


@pytest.mark.parametrize("N", [300, 1100])
def test_fp8_negative_scale(N):
    """A negative scale makes the kernel track the row minimum of the raw
    scores; full and diagonal (masked) tiles of both kernels."""
    d = 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb, kb, vb = gen.qkv_bf16(1, 2, 1, N, N, d)
    scale = -1.0 / math.sqrt(d)
    for causal in (False, True):
        o, lse, codes, desc = fp8_attention(qb, kb, vb, causal, signs, scale=scale)
        check_fp8_parity(o, lse, codes, desc, causal, scale)


def test_fp8_method_oracle_agrees_with_kernel_codes():
    """The GPU quantiser and the oracle's fp64 preparation give the same method:
    attention on the oracle's own codes is within the parity bound of the
    kernel's output too (the codes differ by at most one step in <= 1e-3 of
    the elements)."""
    d, N = 128, 600
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb, kb, vb = gen.qkv_bf16(1, 4, 2, N, N, d, outliers=True)
    scale = 1.0 / math.sqrt(d)
    o, _, codes, desc = fp8_attention(qb, kb, vb, True, signs, scale=scale)
    o_q, _ = oracle.attn_fwd(*oracle_fp8_inputs(qb, kb, vb, signs), True, scale)
    o_k, _ = oracle.attn_fwd(*dequantised(codes, desc), True, scale)
    print(f"method oracle vs kernel-codes oracle {np.abs(o_q - o_k).mean():.2e}, kernel vs method oracle "
          f"{np.abs(o - o_q).mean():.2e}")
    assert np.abs(o_q - o_k).mean() <= 0.25 * np.abs(o - o_k).mean() + 1e-4


def test_fp8_fullsize_outliers_rotation_sampled():
    """B=4, H=16, N=8192, d=128, 1 % outlier channels x20, rotated Q/K, e4m3,
    in the launch configuration the benchmark times: sampled rows against the
    fp64 oracle of the same FP8 method (stated bar), and the accuracy against
    exact attention with and without the rotation (reported; the rotation must
    lower the error, page "FlashAttention-3 — 闪电注意力-3" section 3)."""
    B, H, N, d = 4, 16, 8192, 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb, kb, vb = gen.qkv_bf16(B, H, H, N, N, d, outliers=True)
    o_rot, _, codes, desc = fp8_attention(qb, kb, vb, False, signs, rotate=True)
    o_plain, _, _, _ = fp8_attention(qb, kb, vb, False, signs, rotate=False)
    rng = np.random.default_rng(7)
    rows = np.unique(rng.integers(0, B * H * N, size=96))
    o_x, _ = oracle.attn_fwd_rows(*(gen.bf16_bits_to_f64(a) for a in (qb, kb, vb)), False, 1 / math.sqrt(d), rows)
    qd, kd, vd = dequantised(codes, desc)
    o_q, _ = oracle.attn_fwd_rows(qd, kd, vd, False, 1 / math.sqrt(d), rows)
    a_abs, a_sub = rounding_terms(qd, kd, vd, False, 1 / math.sqrt(d), rows)
    b, h, i = rows // (H * N), (rows // N) % H, rows % N
    err = np.abs(o_rot[b, i, h] - o_q)
    print(f"full-size FP8: max |dO|/bound {np.max(err / fp8_max_bound(a_abs, a_sub, o_q)):.3f}")
    assert np.all(err <= fp8_max_bound(a_abs, a_sub, o_q))
    e_par = err.mean()
    e_rot = np.abs(o_rot[b, i, h] - o_x).mean()
    e_plain = np.abs(o_plain[b, i, h] - o_x).mean()
    print(f"FP8 kernel vs fp64 on its codes {e_par:.3e} (ratio to mean A {e_par / a_abs.mean():.3e}); "
          f"vs exact: rotated {e_rot:.3e}, unrotated {e_plain:.3e}, ratio {e_plain / e_rot:.2f}")
    assert np.all(np.isfinite(o_rot))
    assert e_par <= FP8_PARITY_MEAN_REL * a_abs.mean()
    assert e_plain > 1.5 * e_rot
