"""Parity of the CUDA path with the fp64 oracle, element by element, on seeded
inputs; plus the special cases the mathematics fixes.  Tolerances: BF16
max|dO| <= 1e-2, mean|dO| <= 1e-3, |dLSE| <= 1e-3 (N(0,1) inputs)."""
import math

import numpy as np
import pytest

import attn_inputs as gen
import oracle
from gpu_util import BF16_TOL, compare, run_attn

pytestmark = pytest.mark.gpu


def qkv(B, Hq, Hkv, Nq, Nk, d, seed=gen.BASE_SEED):
    return gen.qkv_bf16(B, Hq, Hkv, Nq, Nk, d, seed=seed)


def f64(x):
    return gen.bf16_bits_to_f64(x)


def full_check(B, Hq, Hkv, Nq, Nk, d, causal, seed=gen.BASE_SEED, scale=None):
    qb, kb, vb = qkv(B, Hq, Hkv, Nq, Nk, d, seed)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = run_attn(qb, kb, vb, causal, scale)
    o_ref, lse_ref = oracle.attn_fwd(f64(qb), f64(kb), f64(vb), causal, scale)
    return compare(o, lse, o_ref, lse_ref)


def test_config1_tiny():
    """B=1, H=1, N=128, d=64, non-causal, scale 1/8."""
    full_check(1, 1, 1, 128, 128, 64, False)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_several_tiles_ragged_tail(d, causal):
    # 300 = 2 full 128-row tiles + a ragged tail; GQA group of 2
    full_check(2, 4, 2, 300, 300, d, causal)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [1, 2, 17, 127, 129, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_odd_lengths(d, N, causal):
    full_check(1, 2, 2, N, N, d, causal)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Nq,Nk", [(200, 333), (333, 200), (1, 700), (700, 5), (128, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_unequal_lengths(d, Nq, Nk, causal):
    # causal with Nq > Nk leaves rows with no visible key: O = 0, LSE = -inf
    full_check(1, 2, 1, Nq, Nk, d, causal)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (8, 1)])
def test_gqa_mqa_against_oracle(Hq, Hkv):
    full_check(2, Hq, Hkv, 257, 257, 128, True)


# Key ranges up to 1024 run on the persistent kernel, longer ones on the
# one-block-per-item kernel; these cases sit on both sides of that boundary.
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Nq,Nk", [(1024, 1024), (300, 1025), (1100, 1100), (129, 1500)])
@pytest.mark.parametrize("causal", [False, True])
def test_both_schedules(d, Nq, Nk, causal):
    full_check(1, 2, 1, Nq, Nk, d, causal)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [200, 1100])
def test_gqa_equals_repeated_heads_bitwise(d, N):
    """Grouped heads read the shared K/V head: identical to MHA on repeated K/V."""
    qb, kb, vb = qkv(1, 8, 2, N, N, d)
    o1, l1 = run_attn(qb, kb, vb, True)
    o2, l2 = run_attn(qb, np.repeat(kb, 4, axis=2), np.repeat(vb, 4, axis=2), True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_v_all_ones_gives_ones(d, causal):
    qb, kb, _ = qkv(1, 2, 2, 300, 300, d)
    vb = gen.f32_to_bf16_bits(np.ones((1, 300, 2, d), dtype=np.float32))
    o, _ = run_attn(qb, kb, vb, causal)
    assert np.max(np.abs(o - 1.0)) <= 4e-3


@pytest.mark.parametrize("d", [64, 128, 256])
def test_constant_v_rows(d):
    qb, kb, _ = qkv(1, 2, 1, 260, 260, d)
    c = np.linspace(-2.0, 3.0, d).astype(np.float32)
    vb = gen.f32_to_bf16_bits(np.broadcast_to(c, (1, 260, 1, d)))
    cb = f64(gen.f32_to_bf16_bits(c))
    for causal in (False, True):
        o, _ = run_attn(qb, kb, vb, causal)
        assert np.max(np.abs(o - cb)) <= 1e-2 * np.max(np.abs(cb))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_causal_row0_is_v0(d):
    qb, kb, vb = qkv(2, 2, 2, 256, 256, d)
    o, lse = run_attn(qb, kb, vb, True, 0.2)
    assert np.array_equal(o[:, 0], f64(vb)[:, 0])  # weight 2^0 = 1 exactly, O = V_0 / 1
    s00 = 0.2 * np.einsum("bhd,bhd->bh", f64(qb)[:, 0], f64(kb)[:, 0])
    assert np.max(np.abs(lse[:, :, 0] - s00)) <= 1e-5 * max(1.0, np.max(np.abs(s00)))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_single_key(d):
    qb, kb, vb = qkv(1, 2, 2, 200, 1, d)
    o, lse = run_attn(qb, kb, vb, False, 0.3)
    assert np.array_equal(o, np.broadcast_to(f64(vb)[:, 0:1], o.shape))
    s = 0.3 * np.einsum("bihd,bjhd->bhi", f64(qb), f64(kb))
    assert np.max(np.abs(lse - s)) <= 1e-5 * max(1.0, np.max(np.abs(s)))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_scale_zero_closed_form(d, causal):
    Nq, Nk = 190, 300
    qb, kb, vb = qkv(1, 1, 1, Nq, Nk, d)
    o, lse = run_attn(qb, kb, vb, causal, 0.0)
    v = f64(vb)[0, :, 0]
    csum = np.cumsum(v, axis=0)
    for i in range(Nq):
        n = Nk if not causal else min(Nk, i + (Nk - Nq) + 1)
        assert abs(lse[0, 0, i] - math.log(n)) <= 1e-5
        assert np.max(np.abs(o[0, i, 0] - csum[n - 1] / n)) <= 1e-3 + 1e-2 * np.max(np.abs(csum[n - 1] / n))


@pytest.mark.parametrize("d", [64, 128, 256])
def test_key_permutation_invariance(d):
    qb, kb, vb = qkv(1, 2, 2, 130, 390, d)
    perm = np.random.default_rng(1).permutation(390)
    o1, l1 = run_attn(qb, kb, vb, False)
    o2, l2 = run_attn(qb, kb[:, perm], vb[:, perm], False)
    ref, lref = oracle.attn_fwd(f64(qb), f64(kb), f64(vb), False, 1 / math.sqrt(d))
    compare(o1, l1, ref, lref)
    compare(o2, l2, ref, lref)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_large_scores_and_dominant_key(d):
    """Q x 30 pushes scores to ~1e3 (many rescales, one dominant key per row).
    This is outside the N(0,1) condition the 1e-2 bar is stated for: a weight
    near 1 rounded to bf16 (relative 2^-9) while the row sum keeps the fp32
    weight moves O by up to 2^-9 |v| (|v| <= 4: 0.008), plus the output
    rounding (0.008), so the max bound here is 2e-2."""
    qb, kb, vb = qkv(1, 2, 2, 257, 515, d)
    q30 = gen.f32_to_bf16_bits((f64(qb) * 30.0).astype(np.float32))
    for causal in (False, True):
        o, lse = run_attn(q30, kb, vb, causal)
        o_ref, lse_ref = oracle.attn_fwd(f64(q30), f64(kb), f64(vb), causal, 1 / math.sqrt(d))
        # LSE of scores ~1e3 in fp32: allow relative 1e-6 on top of the absolute bar
        tol = dict(BF16_TOL, max_abs=2e-2,
                   lse=max(BF16_TOL["lse"], 1e-6 * float(np.max(np.abs(lse_ref[np.isfinite(lse_ref)])))))
        compare(o, lse, o_ref, lse_ref, tol)


def test_lse_optional_and_outputs_fully_written():
    qb, kb, vb = qkv(1, 3, 1, 333, 333, 128)
    o, _ = run_attn(qb, kb, vb, True, with_lse=False)
    o_ref, _ = oracle.attn_fwd(f64(qb), f64(kb), f64(vb), True, 1 / math.sqrt(128))
    compare(o, None, o_ref, None)


def test_empty_key_set():
    import exact_attention_140_b200 as ea
    from gpu_util import torch_mod
    torch = torch_mod()
    o = torch.full((1, 5, 2, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, 5), dtype=torch.float32, device="cuda")
    q = torch.zeros((1, 5, 2, 64), dtype=torch.bfloat16, device="cuda")
    ea.attn_fwd(q, None, None, o, lse, 1, 2, 2, 5, 0, 64, 0, 0.125)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


@pytest.mark.parametrize("N", [512, 1300])
def test_repeatable(N):
    qb, kb, vb = qkv(2, 4, 4, N, N, 128)
    a = run_attn(qb, kb, vb, True)
    b = run_attn(qb, kb, vb, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# A negative scale turns the row maximum of the raw scores into the row
# minimum (a separate branch in both kernels); full and diagonal tiles, on the
# persistent kernel (key ranges <= 1024) and the one-block-per-item kernel.
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [300, 1100])
@pytest.mark.parametrize("causal", [False, True])
def test_negative_scale(d, N, causal):
    full_check(1, 2, 1, N, N, d, causal, scale=-1.0 / math.sqrt(d))
