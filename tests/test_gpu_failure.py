"""Failure detection without a GPU fault: a device-side wait that can never be
satisfied (a barrier nothing arrives at) runs out after its limit, records a
timeout in the device error word, and the context stays usable."""
import math

import numpy as np
import pytest

import attn_inputs as gen
import oracle
from gpu_util import compare, run_attn

pytestmark = pytest.mark.gpu

SITE_PROBE = 10  # wait-site code of the probe kernel (bits 8..15 of the word)


def test_unsatisfied_wait_reports_timeout_and_context_survives():
    import exact_attention_140_b200 as ea
    rc0, _ = ea.attn_get_last_device_error()  # start from a clear word
    assert rc0 == 0
    ea.attn_debug_unsatisfied_wait(2_000_000)  # 2 ms limit
    rc, word = ea.attn_get_last_device_error()
    assert rc == 5, (rc, hex(word))  # ATTN_ERR_DEVICE_TIMEOUT
    assert word & 1 and ((word >> 8) & 0xFF) == SITE_PROBE
    # the word is cleared by the read, and the context still runs attention
    rc2, word2 = ea.attn_get_last_device_error()
    assert rc2 == 0 and word2 == 0
    qb, kb, vb = gen.qkv_bf16(1, 2, 2, 200, 200, 64)
    o, lse = run_attn(qb, kb, vb, True)
    ref = oracle.attn_fwd(*(gen.bf16_bits_to_f64(x) for x in (qb, kb, vb)), True, 1 / math.sqrt(64))
    compare(o, lse, *ref)


def test_status_strings_on_device_error():
    import exact_attention_140_b200 as ea
    assert "timed out" in ea.attn_status_string(5)
