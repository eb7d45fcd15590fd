"""Split-KV on the GPU: the attention over key windows (fp32 partials) merged
by the LSE-weighted combine, against the fp64 oracle of the unsplit
definition (BF16 bar: max |dO| <= 1e-2, mean <= 1e-3, |dLSE| <= 1e-3); and the
combine kernel alone against the oracle's merge.  Grouped heads whose group
size divides 128 run with their query heads stacked in one tile (head
packing); the cases cover packed and unpacked groups."""
import math

import numpy as np
import pytest

import attn_inputs as gen
import oracle
from gpu_util import bf16_dev_to_f64, bf16_ulp, compare, to_dev_bf16, torch_mod

pytestmark = pytest.mark.gpu


def f64(x):
    return gen.bf16_bits_to_f64(x)


def run_splitkv(qb, kb, vb, causal, scale, n_splits):
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Nq, Hq, d = qb.shape
    Nk, Hkv = kb.shape[1], kb.shape[2]
    q, k, v = (to_dev_bf16(x) for x in (qb, kb, vb))
    o = T.full((B, Nq, Hq, d), float("nan"), dtype=T.bfloat16, device="cuda")
    lse = T.full((B, Hq, Nq), float("nan"), dtype=T.float32, device="cuda")
    nbytes = ea.attn_splitkv_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, n_splits)
    assert nbytes >= 0
    ws = T.empty(max(nbytes, 16), dtype=T.uint8, device="cuda")
    ea.attn_fwd_splitkv(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, n_splits, ws, nbytes)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    return bf16_dev_to_f64(o), lse.double().cpu().numpy()


CASES = [  # d, B, Hq, Hkv, Nq, Nk, requested windows
    (128, 2, 4, 2, 1, 1000, 4),
    (128, 1, 8, 2, 7, 4097, 5),
    (64, 2, 2, 1, 300, 700, 3),
    (256, 1, 2, 2, 33, 2000, 6),
    (64, 2, 4, 1, 16, 3000, 0),      # window count chosen by the library
    (128, 1, 2, 2, 128, 1024, 64),   # more windows asked than key tiles exist
    (128, 1, 2, 1, 200, 129, 2),     # causal: rows before the diagonal see nothing
    (128, 1, 24, 8, 5, 3000, 4),     # group of 3 does not divide the tile: heads not packed
    (64, 1, 16, 2, 9, 2500, 3),      # groups of 8 packed: 16 query rows per tile
    (128, 1, 32, 1, 3, 1500, 2),     # MQA, group of 32: 96 packed rows in one tile
    (256, 2, 8, 2, 40, 1200, 3),     # d = 256 with packing (one query tile per block)
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_splitkv_against_oracle(case, causal):
    d, B, Hq, Hkv, Nq, Nk, S = case
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, Nq, Nk, d, seed=gen.BASE_SEED + 20)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_splitkv(qb, kb, vb, causal, scale, S)
    o_ref, lse_ref = oracle.attn_fwd(f64(qb), f64(kb), f64(vb), causal, scale)
    compare(o, lse, o_ref, lse_ref)


def test_splitkv_matches_unsplit_kernel():
    """The same call with and without windows: both within the bar of the
    oracle, and close to each other (only rounding differs)."""
    from gpu_util import run_attn
    qb, kb, vb = gen.qkv_bf16(2, 8, 2, 64, 5000, 128, seed=gen.BASE_SEED + 21)
    o1, l1 = run_attn(qb, kb, vb, True, 1 / math.sqrt(128))
    o2, l2 = run_splitkv(qb, kb, vb, True, 1 / math.sqrt(128), 8)
    assert np.max(np.abs(o1 - o2)) <= 2e-2 and np.max(np.abs(l1 - l2)) <= 1e-3


@pytest.mark.parametrize("S", [5, 40])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_combine_kernel_against_oracle(d, S):
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Nq, Hq = 2, 37, 3
    rng = np.random.default_rng(d)
    o_parts = rng.standard_normal((S, B, Nq, Hq, d)).astype(np.float32)
    lse_parts = (rng.standard_normal((S, B, Hq, Nq)) * 4).astype(np.float32)
    lse_parts[2, :, :, :5] = -np.inf        # some windows empty for some rows
    lse_parts[:, 1, 0, 7] = -np.inf         # one row with every window empty
    op = T.from_numpy(o_parts).cuda()
    lp = T.from_numpy(lse_parts).cuda()
    o = T.full((B, Nq, Hq, d), float("nan"), dtype=T.bfloat16, device="cuda")
    lse = T.full((B, Hq, Nq), float("nan"), dtype=T.float32, device="cuda")
    ea.attn_combine(op, lp, S, B, Hq, Nq, d, o, lse)
    T.cuda.synchronize()
    o_ref, lse_ref = oracle.combine_bnhd(o_parts, lse_parts)
    og, lg = bf16_dev_to_f64(o), lse.double().cpu().numpy()
    assert np.all(og[1, 7, 0] == 0) and np.isneginf(lg[1, 0, 7])
    # fp32 merge then one bf16 rounding: within one bf16 ulp (+ fp32 noise)
    assert np.all(np.abs(og - o_ref) <= bf16_ulp(o_ref) + 1e-6)
    fin = ~np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lg), ~fin)
    assert np.max(np.abs(lg[fin] - lse_ref[fin]) / np.maximum(1.0, np.abs(lse_ref[fin]))) <= 1e-5


def test_splitkv_decode_shape_sampled_rows():
    """The decode-shaped benchmark workload (B=4, Hq=32, Hkv=8, Nq=16,
    Nk=32768, d=128, non-causal) in the launch configuration the benchmark
    times (windows chosen by the library): sampled rows against the fp64
    oracle."""
    B, Hq, Hkv, Nq, Nk, d = 4, 32, 8, 16, 32768, 128
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, Nq, Nk, d)
    o, lse = run_splitkv(qb, kb, vb, False, 1 / math.sqrt(d), 0)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, Nq - 1, B * Hq * Nq - 1], rng.integers(0, B * Hq * Nq, size=40)]))
    o_ref, lse_ref = oracle.attn_fwd_rows(f64(qb), f64(kb), f64(vb), False, 1 / math.sqrt(d), rows)
    b, h, i = rows // (Hq * Nq), (rows // Nq) % Hq, rows % Nq
    compare(o[b, i, h, :], lse[b, h, i], o_ref, lse_ref)


def test_splitkv_argument_errors():
    import exact_attention_140_b200 as ea
    T = torch_mod()
    q = T.zeros((1, 4, 2, 128), dtype=T.bfloat16, device="cuda")
    k = T.zeros((1, 4096, 2, 128), dtype=T.bfloat16, device="cuda")
    o = T.empty_like(q)
    need = ea.attn_splitkv_workspace_bytes(1, 2, 2, 4, 4096, 128, 4)
    assert need > 0
    ws = T.empty(need, dtype=T.uint8, device="cuda")
    assert ea.attn_fwd_splitkv(q, k, k, o, None, 1, 2, 2, 4, 4096, 128, 0, 0.1, 4, ws, need - 1,
                               raise_on_error=False) == 1   # workspace too small
    assert ea.attn_fwd_splitkv(q, k, k, o, None, 1, 2, 2, 4, 4096, 128, 0, 0.1, 4, None, need,
                               raise_on_error=False) == 1   # no workspace
    assert ea.attn_fwd_splitkv(q, k, k, o, None, 1, 2, 2, 4, 4096, 96, 0, 0.1, 4, ws, need,
                               raise_on_error=False) == 2   # head size
