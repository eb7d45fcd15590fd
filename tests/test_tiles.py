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


@pytest.mark.parametrize("bn", [128, 64])
@pytest.mark.parametrize("causal", [0, 1])
def test_all_lengths_up_to_300(bn, causal):
    """Exhaustive over Nq, Nk in [1, 300] for the kernels' tile shapes (128 query
    rows; 128 keys, or 64 at d = 256)."""
    for nq in range(1, 301):
        for nk in range(1, 301):
            check(nq, nk, 128, bn, causal)


def test_random_shapes():
    rng = np.random.default_rng(140)
    for _ in range(1500):
        Nq, Nk = (int(x) for x in rng.integers(1, 301, size=2))
        bm, bn = int(rng.choice([64, 128])), int(rng.choice([64, 128]))
        check(Nq, Nk, bm, bn, int(rng.integers(0, 2)))


def test_invalid_arguments():
    assert ea.attn_kv_tile_count(-1, 5, 10, 10, 64, 0) == -1
    assert ea.attn_kv_tile_count(0, 5, 10, 10, 0, 0) == -1
    assert ea.attn_tile_kind(0, 5, -1, 10, 10, 64, 1) == -1
    assert ea.attn_tile_kind(0, 5, 0, 10, 10, 64, 3) == -1


def check_window(Nq, nk, kv0, shift, bm, bn, causal):
    """Keys [kv0, kv0 + nk) of a range of kv0 + nk + shift keys: the window's
    plan against the window's columns of the full elementwise mask."""
    mask = oracle.mask(Nq, kv0 + nk + shift, causal)[:, kv0:kv0 + nk]
    n_q = (Nq + bm - 1) // bm + 1
    for qt in range(n_q):
        row0, row1 = qt * bm, (qt + 1) * bm
        count, kinds = expected_plan(mask, row0, row1, bn)
        got = ea.attn_kv_tile_count_window(row0, row1, Nq, nk, shift, bn, causal)
        assert got == count, (Nq, nk, kv0, shift, bm, bn, causal, qt)
        for kt, kd in enumerate(kinds):
            assert ea.attn_tile_kind_window(row0, row1, kt, Nq, nk, shift, bn, causal) == kd, \
                (Nq, nk, kv0, shift, bm, bn, causal, qt, kt)


def test_key_windows():
    rng = np.random.default_rng(141)
    for _ in range(200):
        Nq = int(rng.integers(1, 260))
        nk = int(rng.integers(1, 300))
        kv0, shift = int(rng.integers(0, 300)), int(rng.integers(0, 300))
        bm, bn = int(rng.choice([64, 128])), int(rng.choice([64, 128]))
        check_window(Nq, nk, kv0, shift, bm, bn, int(rng.integers(0, 2)))


def test_window_without_shift_is_the_plain_plan():
    for Nq, Nk in ((1, 1), (70, 300), (300, 70), (128, 256)):
        for causal in (0, 1):
            for kt in range(4):
                assert ea.attn_tile_kind_window(0, 128, kt, Nq, Nk, 0, 64, causal) == \
                    ea.attn_tile_kind(0, 128, kt, Nq, Nk, 64, causal)
            assert ea.attn_kv_tile_count_window(0, 128, Nq, Nk, 0, 64, causal) == \
                ea.attn_kv_tile_count(0, 128, Nq, Nk, 64, causal)
    assert ea.attn_kv_tile_count_window(0, 5, 10, 10, -1, 64, 0) == -1
    assert ea.attn_tile_kind_window(0, 5, 0, 10, 10, 0, 64, 2) == -1
