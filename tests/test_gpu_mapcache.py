"""The tensor-map cache of the C ABI: a second call with the same tensors
takes its three maps (Q, K, V) from the cache instead of encoding them, and
its result is bit-identical to the first call's."""
import math

import numpy as np
import pytest

import attn_inputs as gen
from gpu_util import bf16_dev_to_f64, to_dev_bf16, torch_mod

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N", [300, 1500])  # the persistent and the one-block-per-item kernel
def test_second_call_reuses_cached_maps(N):
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Hq, Hkv, d = 1, 4, 2, 128
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, N, N, d, seed=77 + N)
    q, k, v = to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb)
    outs = []
    stats = []
    for _ in range(2):
        o = T.empty((B, N, Hq, d), dtype=T.bfloat16, device="cuda")
        stats.append(ea.attn_debug_map_cache_stats())
        ea.attn_fwd(q, k, v, o, None, B, Hq, Hkv, N, N, d, True, 1 / math.sqrt(d))
        rc, word = ea.attn_get_last_device_error()
        assert rc == 0, hex(word)
        outs.append(bf16_dev_to_f64(o))
    stats.append(ea.attn_debug_map_cache_stats())
    (h0, e0), (h1, e1), (h2, e2) = stats
    assert e2 == e1 and h2 - h1 == 3, stats  # the second call encoded nothing
    assert np.array_equal(outs[0], outs[1])
