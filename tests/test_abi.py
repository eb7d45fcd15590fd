"""CPU checks of the C boundary: the library loads, exports every symbol that
include/attn.h declares, and rejects bad arguments with the documented status
before touching the GPU (no compute calls are made here)."""
import ctypes
import os
import re

import numpy as np
import pytest

import exact_attention_140_b200 as ea

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3
FAKE = 1 << 20  # 16-byte aligned non-null fake device address; never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|long long|char\s*\*|const char\s*\*)\s*\*?\s*(attn_\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert set(names) == set(ea.EXPORTS), names
    lib = ctypes.CDLL(ea.lib_path)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    assert ea.attn_status_string(0) == "ok"
    for s in range(1, 6):
        assert ea.attn_status_string(s) and ea.attn_status_string(s) != "unknown status"
    assert ea.attn_status_string(99) == "unknown status"


def call(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, Nq=128, Nk=128, d=128, causal=0,
                scale=0.125, dtype=0)
    args.update(kw)
    return ea.attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Hq"],
                       args["Hkv"], args["Nq"], args["Nk"], args["d"], args["causal"], args["scale"],
                       args["dtype"], stream=0, raise_on_error=False)


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), INVALID), (dict(Nq=-3), INVALID), (dict(Nk=-1), INVALID), (dict(Hq=3, Hkv=2), INVALID),
    (dict(Hkv=0), INVALID), (dict(causal=2), INVALID), (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID), (dict(o=0), INVALID), (dict(q=0), INVALID), (dict(dtype=7), INVALID),
    (dict(d=96), UNSUPPORTED), (dict(d=32), UNSUPPORTED), (dict(d=512), UNSUPPORTED),
    (dict(dtype=1, d=64), UNSUPPORTED),
    (dict(q=FAKE + 8), MISALIGNED), (dict(o=FAKE + 2), MISALIGNED), (dict(lse=FAKE + 2), MISALIGNED),
    (dict(B=0), OK), (dict(Nq=0), OK), (dict(Hq=0), OK),
])
def test_argument_errors_before_any_cuda_call(kw, status):
    assert call(**kw) == status


def test_fp8_argument_errors():
    f = lambda **kw: ea.attn_fwd_fp8(kw.get("q", FAKE), FAKE, FAKE, FAKE, None, 1, 1, 1, 128, 128,
                                     kw.get("d", 128), 0, 0.1, kw.get("dq", FAKE), FAKE, FAKE, stream=0,
                                     raise_on_error=False)
    assert f(d=64) == UNSUPPORTED
    assert f(dq=0) == INVALID
    assert f(q=FAKE + 1) == MISALIGNED


def test_quant_argument_errors():
    f = lambda **kw: ea.attn_hadamard_quant_fp8(kw.get("x", FAKE), FAKE, FAKE, kw.get("ws", FAKE),
                                                kw.get("rows", 4), kw.get("d", 128), kw.get("signs"), stream=0,
                                                raise_on_error=False)
    assert f(d=64) == UNSUPPORTED
    assert f(rows=-1) == INVALID
    assert f(ws=0) == INVALID
    assert f(x=FAKE + 4) == MISALIGNED
    assert f(signs=FAKE + 4) == MISALIGNED
    assert ea.attn_hadamard_quant_fp8_workspace_bytes() >= 4


def test_debug_probe_rejects_bad_limits():
    assert ea.attn_debug_unsatisfied_wait(0, stream=0, raise_on_error=False) == INVALID
    assert ea.attn_debug_unsatisfied_wait(10 ** 11, stream=0, raise_on_error=False) == INVALID


def test_error_raises():
    with pytest.raises(ea.AttnError):
        ea.attn_fwd(FAKE, FAKE, FAKE, FAKE, None, 1, 3, 2, 8, 8, 128, 0, 0.1, 0, stream=0)


def test_schedule_boundary():
    # persistent kernel for key ranges up to 1024, one block per item above
    assert ea.attn_fwd_schedule(-1, 128, 0) == -1
    assert ea.attn_fwd_schedule(64, 96, 0) == -1
    for d in (64, 128, 256):
        assert [ea.attn_fwd_schedule(n, d, 0) for n in (0, 1, 1024, 1025, 8192)] == [1, 1, 1, 0, 0]
    # causal: persistent up to 1024 keys at d = 64 and 256; never at d = 128
    assert [ea.attn_fwd_schedule(n, 64, 1) for n in (1, 1024, 1025)] == [1, 1, 0]
    assert [ea.attn_fwd_schedule(n, 128, 1) for n in (1, 1024, 1025)] == [0, 0, 0]


def test_splitkv_argument_errors_before_any_cuda_call():
    def split(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8, Nk=4096, d=128, causal=0,
                 scale=0.1, S=4, ws=FAKE, wsb=1 << 20)
        a.update(kw)
        return ea.attn_fwd_splitkv(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"],
                                   a["Nk"], a["d"], a["causal"], a["scale"], a["S"], a["ws"], a["wsb"], stream=0,
                                   raise_on_error=False)
    assert split(B=-1) == INVALID
    assert split(Hq=3) == INVALID
    assert split(causal=2) == INVALID
    assert split(scale=float("nan")) == INVALID
    assert split(o=0) == INVALID
    assert split(q=FAKE + 8) == MISALIGNED
    assert split(Nq=0) == OK  # nothing to compute


def test_splitkv_workspace_sizes():
    # windows of a multiple of 128 keys: 4096 keys in 4 windows of 1024
    S, B, Hq, Nq, d = 4, 1, 4, 8, 128
    o_bytes = (S * B * Nq * Hq * d * 4 + 255) // 256 * 256
    assert ea.attn_splitkv_workspace_bytes(B, Hq, 2, Nq, 4096, d, S) == o_bytes + S * B * Hq * Nq * 4
    # 300 keys asked for 8 windows: windows of 128 keys, 3 of them
    assert ea.attn_splitkv_workspace_bytes(1, 2, 2, 4, 300, 64, 8) == (3 * 4 * 2 * 64 * 4 + 255) // 256 * 256 + 3 * 2 * 4 * 4
    assert ea.attn_splitkv_workspace_bytes(1, 2, 2, 4, 100, 64, 8) == 0   # one window: no partials
    assert ea.attn_splitkv_workspace_bytes(1, 2, 2, 4, 0, 64, 4) == 0     # no keys
    assert ea.attn_splitkv_workspace_bytes(1, 3, 2, 4, 100, 64, 4) == -1  # Hq % Hkv != 0
    assert ea.attn_splitkv_workspace_bytes(1, 2, 2, 4, 100, 96, 4) == -1  # head size


def test_combine_argument_errors_before_any_cuda_call():
    def comb(**kw):
        a = dict(op=FAKE, lp=FAKE, S=3, B=1, Hq=2, Nq=5, d=128, o=FAKE, lse=FAKE)
        a.update(kw)
        return ea.attn_combine(a["op"], a["lp"], a["S"], a["B"], a["Hq"], a["Nq"], a["d"], a["o"], a["lse"],
                               stream=0, raise_on_error=False)
    assert comb(S=0) == INVALID
    assert comb(B=-1) == INVALID
    assert comb(d=96) == UNSUPPORTED
    assert comb(op=0) == INVALID
    assert comb(o=FAKE + 2) == MISALIGNED
    assert comb(lse=FAKE + 2) == MISALIGNED
    assert comb(Nq=0) == OK


def test_gemm_add_argument_errors_before_any_cuda_call():
    def g(**kw):
        a = dict(a=FAKE, b=FAKE, c=FAKE, d=FAKE, M=128, N=256, K=64)
        a.update(kw)
        return ea.attn_gemm_add(a["a"], a["b"], a["c"], a["d"], a["M"], a["N"], a["K"], stream=0,
                                raise_on_error=False)
    assert g(M=-1) == INVALID
    assert g(d=0) == INVALID
    assert g(a=0) == INVALID
    assert g(N=12) == UNSUPPORTED
    assert g(K=60) == UNSUPPORTED
    assert g(a=FAKE + 8) == MISALIGNED
    assert g(c=FAKE + 2) == MISALIGNED
    assert g(M=0) == OK and g(N=0) == OK


def test_gemm_add_partial_overlap_of_c_and_d_rejected():
    """C may be D itself (an in-place update) but may not partly overlap it:
    another thread's store to D could then land before C is read."""
    def g(c, d, M=128, N=256):
        return ea.attn_gemm_add(FAKE, FAKE, c, d, M, N, 64, stream=0, raise_on_error=False)
    nbytes = 128 * 256 * 2
    assert g(FAKE + 16, FAKE) == INVALID
    assert g(FAKE, FAKE + nbytes - 16) == INVALID
    # disjoint ranges and the exact alias pass the argument checks (and then
    # fail only for want of a GPU here)
    assert g(FAKE + nbytes, FAKE) != INVALID
    assert g(FAKE, FAKE) != INVALID


@pytest.mark.parametrize("B,Hkv", [(1, 1), (2, 8), (3, 5), (4, 1), (7, 3), (1, 16), (0, 4)])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_units_cover_every_unit_once(B, Hkv, world):
    """The B x Hkv (batch, key/value head) units of one call split over `world`
    ranks: every unit belongs to exactly one rank, the ranks' shares differ by
    at most one unit, and each rank's share is a contiguous batch-major run."""
    owner = np.full((B, Hkv), -1)
    sizes = []
    for r in range(world):
        rects = ea.attn_shard_units(B, Hkv, world, r)
        assert len(rects) <= 3
        units = []
        for (b0, b1, g0, g1) in rects:
            assert 0 <= b0 < b1 <= B and 0 <= g0 < g1 <= Hkv
            assert np.all(owner[b0:b1, g0:g1] == -1)
            owner[b0:b1, g0:g1] = r
            units += [b * Hkv + g for b in range(b0, b1) for g in range(g0, g1)]
        units.sort()
        if units:
            assert units == list(range(units[0], units[-1] + 1))
        sizes.append(len(units))
    assert np.all(owner >= 0)
    assert max(sizes) - min(sizes) <= 1
    # ranks in order: rank r's run precedes rank r+1's
    firsts = [min((b * Hkv + g for b, g in zip(*np.nonzero(owner == r))), default=None) for r in range(world)]
    got = [f for f in firsts if f is not None]
    assert got == sorted(got)


def test_shard_units_invalid():
    with pytest.raises(ea.AttnError):
        ea.attn_shard_units(2, 2, 0, 0)
    with pytest.raises(ea.AttnError):
        ea.attn_shard_units(2, 2, 2, 2)
    with pytest.raises(ea.AttnError):
        ea.attn_shard_units(-1, 2, 2, 0)


def test_fwd_part_range_errors_before_any_cuda_call():
    def part(b0, b1, g0, g1, **kw):
        a = dict(B=2, Hq=8, Hkv=4, Nq=64, Nk=64, d=128)
        a.update(kw)
        return ea.attn_fwd_part(FAKE, FAKE, FAKE, FAKE, None, a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"],
                                0, 0.1, ea.ATTN_BF16, b0, b1, g0, g1, stream=0, raise_on_error=False)
    assert part(-1, 1, 0, 4) == INVALID
    assert part(1, 0, 0, 4) == INVALID
    assert part(0, 3, 0, 4) == INVALID
    assert part(0, 2, 2, 1) == INVALID
    assert part(0, 2, 0, 5) == INVALID
    assert part(0, 2, 0, 4, d=96) == UNSUPPORTED
    assert part(0, 2, 0, 4, Nq=0) == OK  # nothing to compute


def test_fwd_host_argument_errors_before_any_cuda_call():
    host = np.zeros(16, dtype=np.uint8)  # stands in for every host buffer; never touched
    H = host.ctypes.data

    def call(q_h=H, k_h=H, v_h=H, o_h=H, lse_h=None, lse_d=None, n_chunks=0, **kw):
        a = dict(B=2, Hq=8, Hkv=4, Nq=64, Nk=64, d=128, causal=0, scale=0.1)
        a.update(kw)
        return ea.attn_fwd_host(q_h, k_h, v_h, o_h, lse_h, FAKE, FAKE, FAKE, FAKE, lse_d, a["B"], a["Hq"], a["Hkv"],
                                a["Nq"], a["Nk"], a["d"], a["causal"], a["scale"], n_chunks=n_chunks, stream=0,
                                raise_on_error=False)
    assert call(q_h=None) == INVALID
    assert call(o_h=None) == INVALID
    assert call(k_h=None) == INVALID
    assert call(v_h=None) == INVALID
    assert call(n_chunks=-1) == INVALID
    assert call(lse_h=H) == INVALID            # a host LSE needs a device LSE buffer
    assert call(Hq=6) == INVALID               # Hq % Hkv != 0
    assert call(scale=float("nan")) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(B=0) == OK                     # nothing to compute
    assert call(Nq=0) == OK
