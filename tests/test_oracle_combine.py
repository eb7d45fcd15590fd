"""The split-KV merge in the oracle: partial results over disjoint key windows
(oracle.attn_fwd_window) merged by oracle.combine must reproduce the unsplit
definition (oracle.attn_fwd), whatever the partition; plus a worked example
and the merge's own identities.  CPU only."""
import math
import os

import numpy as np
import pytest

import attn_inputs as gen
import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def f64(x):
    return gen.bf16_bits_to_f64(x)


def windows_merge(q, k, v, causal, scale, cuts):
    parts = [oracle.attn_fwd_window(q, k, v, causal, scale, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    return oracle.combine_bnhd(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk,Hq,Hkv,d", [(70, 200, 2, 1, 16), (200, 70, 2, 2, 8), (1, 500, 4, 2, 32),
                                          (33, 33, 1, 1, 64)])
def test_merge_of_windows_equals_definition(causal, Nq, Nk, Hq, Hkv, d):
    qb, kb, vb = gen.qkv_bf16(2, Hq, Hkv, Nq, Nk, d, seed=11)
    q, k, v = f64(qb), f64(kb), f64(vb)
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.3)
    rng = np.random.default_rng(Nq * 7 + Nk)
    for n_cuts in (1, 2, 3, 7):
        inner = sorted(rng.choice(np.arange(1, Nk), size=min(n_cuts - 1, Nk - 1), replace=False).tolist())
        cuts = [0] + inner + [Nk]
        om, lm = windows_merge(q, k, v, causal, 0.3, cuts)
        assert np.array_equal(np.isneginf(lm), np.isneginf(lse))
        fin = ~np.isneginf(lse)
        assert np.max(np.abs(om - o)) <= 1e-12
        assert np.max(np.abs(lm[fin] - lse[fin]), initial=0.0) <= 1e-12


def test_windows_with_no_visible_key_weigh_nothing():
    """Causal, Nq < Nk: the first rows see none of the last window's keys."""
    qb, kb, vb = gen.qkv_bf16(1, 1, 1, 40, 300, 16, seed=12)
    q, k, v = f64(qb), f64(kb), f64(vb)
    o_last, l_last = oracle.attn_fwd_window(q, k, v, True, 0.25, 280, 300)
    assert np.all(np.isneginf(l_last[0, 0, :20])) and np.all(o_last[0, :20] == 0)
    om, lm = windows_merge(q, k, v, True, 0.25, [0, 100, 280, 300])
    o, lse = oracle.attn_fwd(q, k, v, True, 0.25)
    assert np.max(np.abs(om - o)) <= 1e-12 and np.max(np.abs(lm - lse)) <= 1e-12


def test_merge_identities():
    rng = np.random.default_rng(3)
    o_parts = rng.standard_normal((4, 5, 6, 3, 8))
    lse_parts = rng.standard_normal((4, 5, 3, 6)) * 3
    lse_parts[1, 0, :, :] = -np.inf  # an empty window for batch 0
    o1, l1 = oracle.combine_bnhd(o_parts[:1], lse_parts[:1])
    assert np.array_equal(o1, o_parts[0]) and np.array_equal(l1, lse_parts[0])  # one window: identity
    o, lse = oracle.combine_bnhd(o_parts, lse_parts)
    perm = [2, 0, 3, 1]
    op, lp = oracle.combine_bnhd(o_parts[perm], lse_parts[perm])
    assert np.max(np.abs(op - o)) <= 1e-12 and np.max(np.abs(lp - lse)) <= 1e-12  # order does not matter
    # equal LSE everywhere: the plain mean of the partial outputs, LSE + ln S
    same = np.zeros_like(lse_parts)
    om, lm = oracle.combine_bnhd(o_parts, same)
    assert np.max(np.abs(om - o_parts.mean(axis=0))) <= 1e-12 and np.max(np.abs(lm - math.log(4))) <= 1e-12
    # every window empty: O = 0, LSE = -inf
    oe, le = oracle.combine_bnhd(o_parts, np.full_like(lse_parts, -np.inf))
    assert np.all(oe == 0) and np.all(np.isneginf(le))


def read_fixture(name):
    vals = {}
    for line in open(os.path.join(HERE, "golden", name)):
        line = line.split("#")[0].split()
        if not line:
            continue
        conv = {"ln3": math.log(3.0), "ln4": math.log(4.0), "ln8": math.log(8.0)}
        vals[line[0]] = np.array([conv.get(t, None) if t in conv else float(t) for t in line[1:]])
    return vals


def test_worked_example_two_windows():
    g = read_fixture("combine_two_windows.txt")
    q = g["q"].reshape(1, 1, 1, 2)
    k = np.stack([g["k0"], g["k1"], g["k2"]]).reshape(1, 3, 1, 2)
    v = np.stack([g["v0"], g["v1"], g["v2"]]).reshape(1, 3, 1, 2)
    oa, la = oracle.attn_fwd_window(q, k, v, False, 1.0, 0, 2)
    ob, lb = oracle.attn_fwd_window(q, k, v, False, 1.0, 2, 3)
    assert np.max(np.abs(oa.ravel() - g["o_a"])) <= 1e-14 and abs(la.item() - g["lse_a"][0]) <= 1e-14
    assert np.max(np.abs(ob.ravel() - g["o_b"])) <= 1e-14 and abs(lb.item() - g["lse_b"][0]) <= 1e-14
    o, lse = oracle.combine_bnhd(np.stack([oa, ob]), np.stack([la, lb]))
    assert np.max(np.abs(o.ravel() - g["o"])) <= 1e-14 and abs(lse.item() - g["lse"][0]) <= 1e-14
    of, lf = oracle.attn_fwd(q, k, v, False, 1.0)
    assert np.max(np.abs(of.ravel() - g["o"])) <= 1e-14 and abs(lf.item() - g["lse"][0]) <= 1e-14
