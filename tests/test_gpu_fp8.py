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
from gpu_util import bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu

FP8_TRUTH_MEAN = 3e-2


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


def fp8_attention(qb, kb, vb, causal, signs, rotate=True):
    """Quantise on the GPU (Q, K rotated when rotate; V plain) and run attn_fwd_fp8."""
    import exact_attention_140_b200 as ea
    T = torch()
    B, Nq, Hq, d = qb.shape
    Nk, Hkv = kb.shape[1], kb.shape[2]
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
    ea.attn_fwd_fp8(q8, k8, v8, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, 1.0 / math.sqrt(d), desc.data_ptr(),
                    desc.data_ptr() + 4, desc.data_ptr() + 8)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    return bf16_dev_to_f64(o), lse.double().cpu().numpy()


def oracle_fp8_inputs(qb, kb, vb, signs, rotate=True):
    """The oracle's own FP8 preparation, dequantised: what the FP8 kernel should see."""
    sg = signs.astype(np.float64) if rotate else None
    q8, dq = oracle.fp8_prepare(gen.bf16_bits_to_f64(qb), sg)
    k8, dk = oracle.fp8_prepare(gen.bf16_bits_to_f64(kb), sg)
    v8, dv = oracle.fp8_prepare(gen.bf16_bits_to_f64(vb), None)
    return oracle.e4m3_decode(q8) * dq, oracle.e4m3_decode(k8) * dk, oracle.e4m3_decode(v8) * dv


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 1024])
def test_fp8_attention_against_oracle(causal, N):
    d = 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb, kb, vb = gen.qkv_bf16(1, 4, 2, N, N, d, outliers=True)
    o, lse = fp8_attention(qb, kb, vb, causal, signs)
    assert np.all(np.isfinite(o))
    qd, kd, vd = oracle_fp8_inputs(qb, kb, vb, signs)
    o_q, lse_q = oracle.attn_fwd(qd, kd, vd, causal, 1.0 / math.sqrt(d))
    # same quantised inputs: the difference is P rounded to E4M3 (relative
    # error <= 2^-4 per weight, averaging out over keys) and fp32 accumulation
    err = np.abs(o - o_q)
    assert err.mean() <= FP8_TRUTH_MEAN, err.mean()
    assert np.max(np.abs(lse - lse_q)) <= 2e-2
    o_x, _ = oracle.attn_fwd(*(gen.bf16_bits_to_f64(a) for a in (qb, kb, vb)), causal, 1.0 / math.sqrt(d))
    print(f"N={N} causal={causal}: kernel vs FP8 oracle {err.mean():.2e}, vs exact {np.abs(o - o_x).mean():.2e}, "
          f"FP8 oracle vs exact {np.abs(o_q - o_x).mean():.2e}")


def test_fp8_fullsize_outliers_rotation_sampled():
    """B=4, H=16, N=8192, d=128, 1 % outlier channels x20, rotated Q/K, e4m3,
    in the launch configuration the benchmark times: sampled rows against the
    fp64 oracle of the same FP8 method (stated bar), and the accuracy against
    exact attention with and without the rotation (reported; the rotation must
    lower the error, page "FlashAttention-3 — 闪电注意力-3" section 3)."""
    B, H, N, d = 4, 16, 8192, 128
    signs = gen.hadamard_signs(gen.BASE_SEED + 3, d)
    qb, kb, vb = gen.qkv_bf16(B, H, H, N, N, d, outliers=True)
    o_rot, _ = fp8_attention(qb, kb, vb, False, signs, rotate=True)
    o_plain, _ = fp8_attention(qb, kb, vb, False, signs, rotate=False)
    rng = np.random.default_rng(7)
    rows = np.unique(rng.integers(0, B * H * N, size=96))
    o_x, _ = oracle.attn_fwd_rows(*(gen.bf16_bits_to_f64(a) for a in (qb, kb, vb)), False, 1 / math.sqrt(d), rows)
    qd, kd, vd = oracle_fp8_inputs(qb, kb, vb, signs)
    o_q, _ = oracle.attn_fwd_rows(qd, kd, vd, False, 1 / math.sqrt(d), rows)
    b, h, i = rows // (H * N), (rows // N) % H, rows % N
    e_par = np.abs(o_rot[b, i, h] - o_q).mean()
    e_rot = np.abs(o_rot[b, i, h] - o_x).mean()
    e_plain = np.abs(o_plain[b, i, h] - o_x).mean()
    print(f"FP8 kernel vs FP8 oracle {e_par:.3e}; vs exact: rotated {e_rot:.3e}, unrotated {e_plain:.3e}, "
          f"ratio {e_plain / e_rot:.2f}")
    assert np.all(np.isfinite(o_rot))
    assert e_par <= FP8_TRUTH_MEAN
    assert e_plain > 1.5 * e_rot
