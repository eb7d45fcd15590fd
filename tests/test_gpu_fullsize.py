"""Full-size workloads in the launch configuration the benchmark times: the whole
output is computed on the GPU and sampled rows are recomputed one by one by
the fp64 oracle; every output must be finite and every LSE finite (no empty
rows at Nq == Nk)."""
import math
import zlib

import numpy as np
import pytest

import attn_inputs as gen
import oracle
from gpu_util import compare, run_attn

pytestmark = pytest.mark.gpu

CONFIGS = {
    "gpt2": (8, 12, 12, 1024, 64, True),
    "gqa": (4, 32, 8, 4096, 128, True),
    "mqa": (4, 32, 1, 4096, 128, True),
    "d256": (2, 8, 8, 4096, 256, False),
}
for _n in (512, 1024, 2048, 4096, 8192, 16384):
    for _c in (False, True):
        CONFIGS[f"sweep{_n}{'c' if _c else ''}"] = (16384 // _n, 16, 16, _n, 128, _c)


def sample_rows(B, Hq, N, rng, n=40):
    """Rows at tile edges (0, 127, 128, 255, 256, N-1) of a few heads, plus random rows."""
    picks = []
    heads = [(0, 0), (B - 1, Hq - 1), (B // 2, Hq // 2)]
    for b, h in heads:
        for i in (0, 1, 127, 128, 255, 256, N // 2, N - 2, N - 1):
            if 0 <= i < N:
                picks.append((b * Hq + h) * N + i)
    picks += list(rng.integers(0, B * Hq * N, size=n))
    return np.unique(np.array(picks, dtype=np.int64))


@pytest.mark.parametrize("name", list(CONFIGS))
def test_fullsize_sampled_rows(name):
    B, Hq, Hkv, N, d, causal = CONFIGS[name]
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, N, N, d)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_attn(qb, kb, vb, causal, scale)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    rows = sample_rows(B, Hq, N, np.random.default_rng(zlib.crc32(name.encode())))
    o_ref, lse_ref = oracle.attn_fwd_rows(gen.bf16_bits_to_f64(qb), gen.bf16_bits_to_f64(kb),
                                          gen.bf16_bits_to_f64(vb), causal, scale, rows)
    b, h, i = rows // (Hq * N), (rows // N) % Hq, rows % N
    emax, emean, dlse = compare(o[b, i, h, :], lse[b, h, i], o_ref, lse_ref)
    print(f"{name}: {rows.size} rows, max |dO| {emax:.3e}, mean |dO| {emean:.3e}, max |dLSE| {dlse:.3e}")
