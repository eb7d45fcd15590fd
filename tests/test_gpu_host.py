"""attn_fwd_host: inputs and outputs in host memory, the copies in, the kernels
and the copies out pipelined over chunks of (batch, key/value head) units.
Its host O and LSE must equal, bit for bit, attn_fwd's on the same device
tensors (the same kernels on the same data), for every chunking, and its
device buffers must hold what attn_fwd's would."""
import math

import numpy as np
import pytest

import attn_inputs as gen
from gpu_util import torch_mod

pytestmark = pytest.mark.gpu

CASES = [  # B, Hq, Hkv, Nq, Nk, d, causal
    (2, 4, 4, 300, 300, 64, True),     # persistent kernel, ragged tail
    (2, 8, 2, 1100, 1100, 128, True),  # per-item kernel, GQA groups of 4
    (3, 4, 1, 257, 700, 128, False),   # MQA, Nq != Nk
    (1, 2, 2, 520, 520, 256, False),
    (2, 2, 2, 200, 0, 64, False),      # no keys: O = 0, LSE = -inf
]


def _host_bf16(T, bits, pinned):
    t = T.from_numpy(bits.view(np.int16).copy()).view(T.bfloat16)
    return t.pin_memory() if pinned else t


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("n_chunks", [0, 1, 3, 64])
def test_host_pipeline_matches_device_call(case, n_chunks):
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Hq, Hkv, Nq, Nk, d, causal = case
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, Nq, max(Nk, 1), d, seed=900 + Nq + d)
    kb, vb = kb[:, :Nk], vb[:, :Nk]
    scale = 1 / math.sqrt(d)
    q_h, k_h, v_h = (_host_bf16(T, x, True) for x in (qb, kb, vb))
    o_h = T.empty((B, Nq, Hq, d), dtype=T.bfloat16).pin_memory()
    lse_h = T.empty((B, Hq, Nq), dtype=T.float32).pin_memory()
    q_d, k_d, v_d = (T.empty(x.shape, dtype=T.bfloat16, device="cuda") for x in (q_h, k_h, v_h))
    o_d = T.empty((B, Nq, Hq, d), dtype=T.bfloat16, device="cuda")
    lse_d = T.empty((B, Hq, Nq), dtype=T.float32, device="cuda")
    ea.attn_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                     n_chunks=n_chunks)
    T.cuda.synchronize()
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    # reference: the device entry point on device copies of the same inputs
    q2, k2, v2 = (x.cuda() for x in (q_h, k_h, v_h))
    o2 = T.empty_like(o_d)
    l2 = T.empty_like(lse_d)
    ea.attn_fwd(q2, k2, v2, o2, l2, B, Hq, Hkv, Nq, Nk, d, causal, scale)
    T.cuda.synchronize()
    assert T.equal(o_h.view(T.int16), o2.cpu().view(T.int16))
    assert T.equal(lse_h, l2.cpu())
    assert T.equal(o_d.view(T.int16), o2.view(T.int16))
    assert T.equal(q_d.view(T.int16), q2.view(T.int16)) and T.equal(v_d.view(T.int16), v2.view(T.int16))


def test_host_pipeline_pageable_memory_and_no_lse():
    """Pageable host buffers work (the copies serialise), and lse_h = NULL leaves
    the host without LSE while O is still complete."""
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Hq, Hkv, N, d = 2, 4, 2, 640, 128
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, N, N, d, seed=931)
    q_h, k_h, v_h = (_host_bf16(T, x, False) for x in (qb, kb, vb))
    o_h = T.zeros((B, N, Hq, d), dtype=T.bfloat16)
    q_d, k_d, v_d = (T.empty(x.shape, dtype=T.bfloat16, device="cuda") for x in (q_h, k_h, v_h))
    o_d = T.empty((B, N, Hq, d), dtype=T.bfloat16, device="cuda")
    ea.attn_fwd_host(q_h, k_h, v_h, o_h, None, q_d, k_d, v_d, o_d, None, B, Hq, Hkv, N, N, d, False,
                     1 / math.sqrt(d), n_chunks=2)
    T.cuda.synchronize()
    o2 = T.empty_like(o_d)
    ea.attn_fwd(q_h.cuda(), k_h.cuda(), v_h.cuda(), o2, None, B, Hq, Hkv, N, N, d, False, 1 / math.sqrt(d))
    T.cuda.synchronize()
    assert T.equal(o_h.view(T.int16), o2.cpu().view(T.int16))


def test_host_pipeline_on_a_side_stream_orders_after_prior_work():
    """Work already on the caller's stream (here: writing the host-visible
    device buffers) completes before the pipeline's copies start, and the
    stream's completion covers the copies out."""
    import exact_attention_140_b200 as ea
    T = torch_mod()
    B, Hq, Hkv, N, d = 1, 8, 8, 1024, 64
    qb, kb, vb = gen.qkv_bf16(B, Hq, Hkv, N, N, d, seed=932)
    q_h, k_h, v_h = (_host_bf16(T, x, True) for x in (qb, kb, vb))
    o_h = T.empty((B, N, Hq, d), dtype=T.bfloat16).pin_memory()
    s = T.cuda.Stream()
    with T.cuda.stream(s):
        q_d, k_d, v_d = (T.full(x.shape, 7.0, dtype=T.bfloat16, device="cuda") for x in (q_h, k_h, v_h))
        o_d = T.full((B, N, Hq, d), 3.0, dtype=T.bfloat16, device="cuda")
        for _ in range(3):  # queue more prior work on the stream
            o_d.mul_(1.0)
        ea.attn_fwd_host(q_h, k_h, v_h, o_h, None, q_d, k_d, v_d, o_d, None, B, Hq, Hkv, N, N, d, True,
                         1 / math.sqrt(d), n_chunks=4, stream=s)
    s.synchronize()
    o2 = T.empty_like(o_d)
    ea.attn_fwd(q_h.cuda(), k_h.cuda(), v_h.cuda(), o2, None, B, Hq, Hkv, N, N, d, True, 1 / math.sqrt(d))
    T.cuda.synchronize()
    assert T.equal(o_h.view(T.int16), o2.cpu().view(T.int16))
