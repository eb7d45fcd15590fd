"""The causal tile plan of the kernels (which key tiles a query tile visits,
which are full and which need an element mask) against the oracle's
elementwise visibility predicate: bit-exact over many shapes, ragged and
Nq != Nk included."""
import numpy as np
import pytest

import exact_attention_140_b200 as ea
import oracle

EDGE = [1, 2, 3, 63, 64, 65, 127, 128, 129, 191, 200, 255, 256, 257, 300]


def expected_plan(mask, row0, row1, bn):
    Nq, Nk = mask.shape
    rows = mask[row0:min(row1, Nq)]
    n_tiles = (Nk + bn - 1) // bn
    kinds = []
    for kt in range(n_tiles + 2):  # two tiles past the end must read as skip
        blk_full = np.zeros((rows.shape[0], bn), dtype=bool)
        lo, hi = kt * bn, min((kt + 1) * bn, Nk)
        if lo < Nk:
            blk_full[:, : hi - lo] = rows[:, lo:hi]
        if rows.shape[0] == 0 or not blk_full.any():
            kinds.append(0)
        elif blk_full.all():
            kinds.append(1)
        else:
            kinds.append(2)
    count = 0
    for kt, kd in enumerate(kinds):
        if kd != 0:
            count = kt + 1
    # visible tiles form a prefix
    assert all(kd != 0 for kd in kinds[:count])
    return count, kinds


def check(Nq, Nk, bm, bn, causal):
    mask = oracle.mask(Nq, Nk, causal)
    n_q = (Nq + bm - 1) // bm + 1  # one tile past the end too
    for qt in range(n_q):
        row0, row1 = qt * bm, (qt + 1) * bm
        count, kinds = expected_plan(mask, row0, row1, bn)
        assert ea.attn_kv_tile_count(row0, row1, Nq, Nk, bn, causal) == count, (Nq, Nk, bm, bn, causal, qt)
        for kt, kd in enumerate(kinds):
            assert ea.attn_tile_kind(row0, row1, kt, Nq, Nk, bn, causal) == kd, (Nq, Nk, bm, bn, causal, qt, kt)


@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("bm,bn", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_edge_shapes(bm, bn, causal):
    for Nq in EDGE:
        for Nk in EDGE:
            check(Nq, Nk, bm, bn, causal)


def test_random_shapes():
    rng = np.random.default_rng(140)
    for _ in range(150):
        Nq, Nk = (int(x) for x in rng.integers(1, 301, size=2))
        bm, bn = int(rng.choice([64, 128])), int(rng.choice([64, 128]))
        check(Nq, Nk, bm, bn, int(rng.integers(0, 2)))


def test_invalid_arguments():
    assert ea.attn_kv_tile_count(-1, 5, 10, 10, 64, 0) == -1
    assert ea.attn_kv_tile_count(0, 5, 10, 10, 0, 0) == -1
    assert ea.attn_tile_kind(0, 5, -1, 10, 10, 64, 1) == -1
    assert ea.attn_tile_kind(0, 5, 0, 10, 10, 64, 3) == -1
