"""ATTN_LOG=1: every launch prints its kernel and template configuration to
stderr; without it the library prints nothing.  Runs in a child process,
since the library reads the variable once."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import math, torch
import exact_attention_140_b200 as ea
for N, d, causal in ((300, 64, True), (1500, 128, True), (1500, 128, False)):
    q = torch.randn(1, N, 2, d, device="cuda").to(torch.bfloat16)
    k = torch.randn(1, N, 2, d, device="cuda").to(torch.bfloat16)
    v = torch.randn(1, N, 2, d, device="cuda").to(torch.bfloat16)
    o = torch.empty_like(q)
    ea.attn_fwd(q, k, v, o, None, 1, 2, 2, N, N, d, causal, 1 / math.sqrt(d))
torch.cuda.synchronize()
rc, word = ea.attn_get_last_device_error()
assert rc == 0, hex(word)
"""


def _run(env_extra):
    env = dict(os.environ)
    env.pop("ATTN_LOG", None)
    env.update(env_extra)
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stderr


def test_log_prints_each_launch():
    err = [l for l in _run({"ATTN_LOG": "1"}).splitlines() if l.startswith("attn: ")]
    assert len(err) == 3, err
    assert "attn_fwd_persistent_kernel<D=64 " in err[0] and "causal=1" in err[0] and "Nk=300" in err[0]
    assert "attn_fwd_kernel<D=128 " in err[1] and "causal=1" in err[1] and "head bands" in err[1]
    assert "attn_fwd_kernel<D=128 " in err[2] and "causal=0" in err[2]


def test_silent_by_default():
    assert not any(l.startswith("attn: ") for l in _run({}).splitlines())
