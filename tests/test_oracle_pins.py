"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix,
never against the oracle's own code path.

* brute force in long double with a different algebra (no max subtraction);
* the online recurrence of page "FlashAttention (SV)", section "Online-beräkning
  av Softmax", which the page says gives the exact result, for many block sizes
  and lazy thresholds;
* closed forms: rows sum to one, constant V, causal row 0, a single key,
  scale = 0, the hand-derived fixtures in tests/golden/;
* invariants: grouped heads equal repeated heads, joint key/value permutation;
* the rotation of page "FlashAttention-3 — 闪电注意力-3" section 3 is orthogonal
  and leaves Q K^T unchanged;
* the E4M3 codec against the OCP FP8 definition.
"""
import math
import os

import numpy as np
import pytest

import attn_inputs as gen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_qkv(B, Hq, Hkv, Nq, Nk, d, seed=7):
    q, k, v = gen.qkv_bf16(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    return gen.bf16_bits_to_f64(q), gen.bf16_bits_to_f64(k), gen.bf16_bits_to_f64(v)


def rel_close(a, b, tol):
    a = np.asarray(a)
    b = np.asarray(b)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin)
    assert np.array_equal(a[~fin], b[~fin])
    scale = max(1.0, float(np.max(np.abs(b[fin])))) if fin.any() else 1.0
    assert float(np.max(np.abs(a[fin] - b[fin]), initial=0.0)) <= tol * scale


SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d
    (1, 1, 1, 1, 1, 1),
    (1, 1, 1, 5, 5, 2),
    (2, 2, 1, 7, 7, 4),
    (1, 4, 2, 16, 16, 64),
    (1, 2, 2, 5, 11, 4),   # Nq < Nk
    (1, 2, 1, 13, 6, 2),   # Nq > Nk: causal rows with no key
    (1, 1, 1, 16, 3, 1),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_two_pass_equals_bruteforce(shape, causal):
    B, Hq, Hkv, Nq, Nk, d = shape
    q, k, v = rand_qkv(*shape)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    ob, lseb = oracle.attn_bruteforce(q, k, v, causal, scale)
    rel_close(o, ob, 1e-12)
    rel_close(lse, lseb, 1e-12)


@pytest.mark.parametrize("block", [1, 3, 16, 128])
@pytest.mark.parametrize("tau_log2", [0.0, 2.0, 8.0, 20.0])
@pytest.mark.parametrize("causal", [False, True])
def test_online_recurrence_is_exact(block, tau_log2, causal):
    shape = (2, 4, 2, 37, 150, 16)
    q, k, v = rand_qkv(*shape, seed=11)
    q = q * 3.0  # spread the scores so the max moves across blocks
    scale = 1.0 / 4.0
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    oo, lso, _ = oracle.attn_online(q, k, v, causal, scale, block, tau_log2 * math.log(2.0))
    rel_close(oo, o, 1e-12)
    rel_close(lso, lse, 1e-12)


def test_lazy_threshold_skips_rescales():
    """A larger threshold moves the reference max less often (the page on
    FlashAttention-4 reports about 90 % of output rescalings skipped)."""
    q, k, v = rand_qkv(1, 2, 2, 64, 2048, 64, seed=3)
    scale = 1.0 / 8.0
    _, _, eager = oracle.attn_online(q, k, v, False, scale, 128, 0.0)
    _, _, lazy = oracle.attn_online(q, k, v, False, scale, 128, 8.0 * math.log(2.0))
    assert eager > 0
    assert lazy < eager


@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):
    q, k, v = rand_qkv(1, 2, 2, 33, 33, 8)
    o, _ = oracle.attn_fwd(q, k, np.ones_like(v), causal, 0.5)
    assert np.max(np.abs(o - 1.0)) <= 1e-14


def test_constant_v_rows():
    q, k, _ = rand_qkv(2, 2, 1, 19, 23, 8)
    c = np.linspace(-3.0, 5.0, 8)
    v = np.broadcast_to(c, (2, 23, 1, 8)).copy()
    for causal in (False, True):
        o, _ = oracle.attn_fwd(q * 4, k, v, causal, 1.0)
        assert np.max(np.abs(o - c)) <= 1e-12


def test_causal_row_zero_is_v0():
    q, k, v = rand_qkv(2, 3, 3, 12, 12, 16)
    scale = 0.25
    o, lse = oracle.attn_fwd(q, k, v, True, scale)
    assert np.array_equal(o[:, 0], v[:, 0])  # weight exactly exp(0)/exp(0) = 1
    s00 = scale * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0])
    assert np.max(np.abs(lse[:, :, 0] - s00)) <= 1e-12


def test_single_key():
    q, k, v = rand_qkv(1, 2, 1, 9, 1, 8)
    scale = 0.3
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, scale)
        s = scale * np.einsum("bihd,bjd->bhi", q, k[:, :, 0])
        if causal:  # bottom-right: row i sees key 0 iff 0 <= i + (1 - 9)
            vis = np.arange(9) >= 8
            assert np.all(o[:, ~vis] == 0.0) and np.all(np.isneginf(lse[:, :, ~vis]))
            assert np.array_equal(o[:, vis], np.broadcast_to(v[:, 0:1, 0:1, :], o[:, vis].shape))
            assert np.max(np.abs(lse[:, :, vis] - s[:, :, vis])) <= 1e-12
        else:
            assert np.array_equal(o, np.broadcast_to(v[:, 0:1, 0:1, :], o.shape))
            assert np.max(np.abs(lse - s)) <= 1e-12


@pytest.mark.parametrize("Nq,Nk", [(8, 8), (5, 9), (9, 5)])
def test_scale_zero_uniform_weights(Nq, Nk):
    q, k, v = rand_qkv(1, 1, 1, Nq, Nk, 4)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, 0.0)
        for i in range(Nq):
            n_allowed = Nk if not causal else max(0, min(Nk, i + (Nk - Nq) + 1))
            if n_allowed == 0:
                assert np.all(o[0, i, 0] == 0.0) and np.isneginf(lse[0, 0, i])
                continue
            mean_v = v[0, :n_allowed, 0].mean(axis=0)
            assert np.max(np.abs(o[0, i, 0] - mean_v)) <= 1e-12
            assert abs(lse[0, 0, i] - math.log(n_allowed)) <= 1e-12


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = (x.strip() for x in line.split("=", 1))
            out[key] = [part.strip() for part in val.split("|")]
    return out


def _ev(expr):
    return float(eval(expr, {"__builtins__": {}}, {"e": math.e, "log": math.log}))


def test_golden_two_keys():
    g = _read_golden("closed_form_two_keys.txt")
    q = np.array([[float(x) for x in g["q"][0].split()]]).reshape(1, 1, 1, 2)
    k = np.array([[float(x) for x in r.split()] for r in g["k"]]).reshape(1, 2, 1, 2)
    v = np.array([[float(x) for x in r.split()] for r in g["v"]]).reshape(1, 2, 1, 2)
    exp_o = np.array([_ev(x) for x in g["O"]])
    exp_lse = _ev(g["LSE"][0])
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, _ev(g["scale"][0]))
        assert np.max(np.abs(o.reshape(-1) - exp_o)) <= 1e-15
        assert abs(lse.reshape(-1)[0] - exp_lse) <= 1e-15


def test_golden_scale_zero_causal():
    g = _read_golden("closed_form_scale_zero.txt")
    vals = np.array([float(x) for x in g["v"][0].split()])
    Nk, Nq = vals.size, len(g["O"])
    v = vals.reshape(1, Nk, 1, 1)
    q = np.ones((1, Nq, 1, 1))
    k = np.ones((1, Nk, 1, 1))
    o, lse = oracle.attn_fwd(q, k, v, True, 0.0)
    assert np.max(np.abs(o.reshape(-1) - np.array([_ev(x) for x in g["O"]]))) <= 1e-14
    assert np.max(np.abs(lse.reshape(-1) - np.array([_ev(x) for x in g["LSE"]]))) <= 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_repeated_heads(causal):
    q, k, v = rand_qkv(2, 8, 2, 21, 21, 8)
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.35)
    kr, vr = np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2)
    o2, lse2 = oracle.attn_fwd(q, kr, vr, causal, 0.35)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_key_permutation_invariance():
    q, k, v = rand_qkv(1, 2, 2, 17, 40, 8)
    perm = np.random.default_rng(0).permutation(40)
    o, lse = oracle.attn_fwd(q, k, v, False, 0.4)
    o2, lse2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], False, 0.4)
    rel_close(o2, o, 1e-12)
    rel_close(lse2, lse, 1e-12)


def test_scores_are_scaled_not_values():
    """A plausible slip: applying scale after softmax or to V.  Doubling the scale
    must sharpen the weights, and O must stay within the convex hull of V rows."""
    q, k, v = rand_qkv(1, 1, 1, 4, 6, 4)
    o1, _ = oracle.attn_fwd(q, k, v, False, 0.1)
    o2, _ = oracle.attn_fwd(q, k, v, False, 5.0)
    assert not np.allclose(o1, o2)
    assert np.all(o2 <= v.max(axis=1, keepdims=True) + 1e-12)
    assert np.all(o2 >= v.min(axis=1, keepdims=True) - 1e-12)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_hadamard_orthogonal_and_preserves_scores(d):
    signs = gen.hadamard_signs(143, d).astype(np.float64)
    M = oracle.hadamard(d, signs)
    assert np.max(np.abs(M @ M.T - np.eye(d))) <= 1e-15
    x = gen.bf16_bits_to_f64(gen.normal_bf16(5, (9, d)))
    y = gen.bf16_bits_to_f64(gen.normal_bf16(6, (13, d)))
    xr, yr = oracle.rotate_rows(x, M), oracle.rotate_rows(y, M)
    ref = x @ y.T
    assert np.max(np.abs(xr @ yr.T - ref)) <= 1e-12 * np.linalg.norm(x) * np.linalg.norm(y)
    # Sylvester structure: entries are +-1/sqrt(d), first column carries the signs
    assert np.allclose(np.abs(M), 1.0 / math.sqrt(d), rtol=0, atol=1e-15)
    assert np.array_equal(np.sign(M[:, 0]), signs)


def test_hadamard_rotation_spreads_outliers():
    """Incoherent processing: a single large coordinate is spread over all d."""
    d = 128
    signs = gen.hadamard_signs(143, d).astype(np.float64)
    M = oracle.hadamard(d, signs)
    x = np.zeros((1, d))
    x[0, 5] = 20.0
    xr = oracle.rotate_rows(x, M)
    assert np.allclose(np.abs(xr), 20.0 / math.sqrt(d), rtol=0, atol=1e-12)


def test_e4m3_codec():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    nan = np.isnan(vals)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    # known values from the OCP FP8 E4M3 definition
    assert vals[0x7E] == 448.0 and vals[0xFE] == -448.0
    assert vals[0x01] == 2.0 ** -9 and vals[0x08] == 2.0 ** -6 and vals[0x38] == 1.0
    assert vals[0x07] == 7 * 2.0 ** -9 and vals[0x3C] == 1.5
    # round trip of every finite code (-0 keeps its sign bit)
    fin = ~nan
    re = oracle.e4m3_encode(vals[fin])
    assert np.array_equal(re, codes[fin])
    # saturation
    assert oracle.e4m3_encode(np.array([1e6, -1e6, 449.0, 464.0]))[0:4].tolist() == \
        [0x7E, 0xFE, 0x7E, 0x7E]
    # ties to even on midpoints between consecutive positive codes
    pos = vals[0:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2.0
    got = oracle.e4m3_encode(mids)
    lo = np.arange(0, 0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want.astype(np.uint8))
    # just off the midpoint goes to the nearer code
    assert np.array_equal(oracle.e4m3_encode(mids * (1 + 1e-9)), (lo + 1).astype(np.uint8))
    assert np.array_equal(oracle.e4m3_encode(mids * (1 - 1e-9)), lo.astype(np.uint8))


def test_quant_e4m3_f32_maps_amax_to_448():
    x = np.array([0.5, -2.0, 1.0, 0.0], dtype=np.float32)
    c = oracle.quant_e4m3_f32(x, 2.0)
    # 0.5*224 = 112 = 1.75*2^6 -> exponent field 13, mantissa 6 -> 0x6E;
    # -2*224 = -448 -> 0xFE;  224 = 1.75*2^7 -> 0x76;  0 -> 0x00
    assert c.tolist() == [0x6E, 0xFE, 0x76, 0x00]


def test_fp8_prepare_roundtrip_error_small():
    x = gen.bf16_bits_to_f64(gen.normal_bf16(9, (64, 128)))
    signs = gen.hadamard_signs(10, 128).astype(np.float64)
    codes, desc = oracle.fp8_prepare(x, signs)
    xr = oracle.rotate_rows(x, oracle.hadamard(128, signs))
    back = oracle.e4m3_decode(codes) * desc
    # E4M3 keeps 3 mantissa bits: relative rounding error <= 2^-4 for normals
    big = np.abs(xr) > 2.0 ** -6 * desc
    assert np.max(np.abs(back[big] - xr[big]) / np.abs(xr[big])) <= 2.0 ** -4 + 1e-12


def test_mask_bottom_right():
    m = oracle.mask(3, 5, True)
    assert m.tolist() == [[1, 1, 1, 0, 0], [1, 1, 1, 1, 0], [1, 1, 1, 1, 1]]
    m = oracle.mask(5, 3, True)
    assert m.tolist() == [[0, 0, 0], [0, 0, 0], [1, 0, 0], [1, 1, 0], [1, 1, 1]]
    assert oracle.mask(4, 6, False).all()


def test_generator_is_seeded_and_standard_normal():
    a = gen.normal(140, 200000)
    assert np.array_equal(a, gen.normal(140, 200000))
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    # SplitMix64 published first output for seed 0 (state advanced once)
    assert int(gen.splitmix64(0, 1)[0]) == 0xE220A8397B1DCDAF
    bits = gen.f32_to_bf16_bits(np.array([1.0, 1.00390625, 1.01171875, -2.5], dtype=np.float32))
    # 1.00390625 = 1 + 2^-8 is a tie between bf16 1.0 and 1.0078125 -> even (1.0)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020]


ROWS_SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d: GQA groups, Nq < Nk, Nq > Nk (empty causal rows)
    (2, 6, 3, 23, 23, 8),
    (3, 4, 1, 11, 29, 4),
    (2, 4, 2, 31, 9, 16),
]


@pytest.mark.parametrize("shape", ROWS_SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_rows_variant_equals_full_definition(shape, causal):
    """oracle.attn_fwd_rows decodes a flat row index r = (b*Hq + h)*Nq + i on its
    own; the sampled full-size checks rest on it.  Every selected row must be
    the same bits as that row of the (pinned) full definition, and a decode
    that swaps b/h/i or uses a wrong output stride fails here: the rows are
    scattered over every batch, head and position, in shuffled order, with
    repeats."""
    B, Hq, Hkv, Nq, Nk, d = shape
    q, k, v = rand_qkv(*shape, seed=29)
    scale = 0.37
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    rng = np.random.default_rng(5)
    total = B * Hq * Nq
    rows = np.concatenate([rng.permutation(total), rng.integers(0, total, size=17)])
    ro, rl = oracle.attn_fwd_rows(q, k, v, causal, scale, rows)
    b, h, i = rows // (Hq * Nq), (rows // Nq) % Hq, rows % Nq
    assert np.array_equal(ro, o[b, i, h, :])
    assert np.array_equal(rl, lse[b, h, i])
    if causal and Nq > Nk:
        assert np.isneginf(rl).any()  # the empty rows are among those checked
