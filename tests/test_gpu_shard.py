"""One call split over devices by (batch, key/value head) units: attn_fwd_part
computes a rectangle of batches x key/value groups on the full tensors and
writes only those rows.  With one GPU here, the ranks of a world run one
after another on the same device and write into one output: their union must
be bit-identical to a single attn_fwd (every (batch, head) is computed by the
same kernel either way), and a rank's call must leave every other row as it
was."""
import math

import numpy as np
import pytest

import attn_inputs as gen
from gpu_util import bf16_dev_to_f64, to_dev_bf16, torch_mod

pytestmark = pytest.mark.gpu


def dev_inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, Nq, Nk, d, seed=seed)
    return to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb)


@pytest.mark.parametrize("world", [2, 3, 5])
@pytest.mark.parametrize("N,d,causal", [(300, 128, True), (1100, 64, False), (700, 256, True), (1500, 128, False)])
def test_shards_reassemble_to_the_whole_call(world, N, d, causal):
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Hq, Hkv = 3, 8, 4
    q, k, v = dev_inputs(B, Hq, Hkv, N, N, d, seed=300 + N)
    scale = 1.0 / math.sqrt(d)
    o_ref = T.empty((B, N, Hq, d), dtype=T.bfloat16, device="cuda")
    l_ref = T.empty((B, Hq, N), dtype=T.float32, device="cuda")
    ea.attn_fwd(q, k, v, o_ref, l_ref, B, Hq, Hkv, N, N, d, causal, scale, ea.ATTN_BF16)
    o = T.full((B, N, Hq, d), float("nan"), dtype=T.bfloat16, device="cuda")
    lse = T.full((B, Hq, N), float("nan"), dtype=T.float32, device="cuda")
    g = Hq // Hkv
    for rank in range(world):
        before = bf16_dev_to_f64(o)
        rects = ea.attention_shard(q, k, v, o, lse, rank, world, causal=causal, scale=scale)
        rc, word = ea.attn_get_last_device_error()
        assert rc == 0, hex(word)
        after = bf16_dev_to_f64(o)
        mine = np.zeros((B, N, Hq, d), dtype=bool)
        for (b0, b1, g0, g1) in rects:
            mine[b0:b1, :, g0 * g:g1 * g, :] = True
        # rows outside this rank's rectangles are untouched (NaN stays NaN,
        # values written by earlier ranks stay bit-identical)
        assert np.array_equal(np.isnan(after[~mine]), np.isnan(before[~mine]))
        fin = ~np.isnan(before) & ~mine
        assert np.array_equal(after[fin], before[fin])
    assert np.array_equal(bf16_dev_to_f64(o), bf16_dev_to_f64(o_ref))
    assert T.equal(lse, l_ref)


def test_part_with_no_keys_fills_only_its_rows():
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Hq, Hkv, Nq, d = 2, 4, 2, 5, 64
    q = T.zeros((B, Nq, Hq, d), dtype=T.bfloat16, device="cuda")
    o = T.full((B, Nq, Hq, d), 7.0, dtype=T.bfloat16, device="cuda")
    lse = T.zeros((B, Hq, Nq), dtype=T.float32, device="cuda")
    ea.attn_fwd_part(q, None, None, o, lse, B, Hq, Hkv, Nq, 0, d, 0, 0.125, ea.ATTN_BF16, 1, 2, 1, 2)
    T.cuda.synchronize()
    # batch 1, query heads 2..3 (key/value head 1): O = 0, LSE = -inf; the rest untouched
    assert T.all(o[1, :, 2:4] == 0) and T.all(T.isneginf(lse[1, 2:4]))
    o[1, :, 2:4] = 7.0
    lse[1, 2:4] = 0.0
    assert T.all(o == 7.0) and T.all(lse == 0.0)
