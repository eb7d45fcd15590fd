"""D = A B + C on tcgen05 (attn_gemm_add) against the fp64 oracle on the same
bf16 inputs.  Products accumulate in fp32 and D is rounded once to bf16, so
an element may differ from the exact value by the fp32 summation error,
bounded by K * u * (sum_k |a_k b_k| + |c|) (u = 2^-23, allowing for rounding
inside the tensor core's 16-wide steps), plus one bf16 ulp of the result
(a value near a rounding midpoint may round either way after the fp32 sum);
the mean error stays below half an ulp plus the mean summation bound."""
import numpy as np
import pytest

import attn_inputs as gen
import oracle
from gpu_util import bf16_dev_to_f64, bf16_ulp, to_dev_bf16, torch_mod

pytestmark = pytest.mark.gpu


def run_gemm(ab, bb, cb):
    import exact_attention_140_b200 as ea
    T = torch_mod()
    M, K = ab.shape
    N = bb.shape[1]
    a, b = to_dev_bf16(ab), to_dev_bf16(bb)
    c = None if cb is None else to_dev_bf16(cb)
    d = T.full((M, N), float("nan"), dtype=T.bfloat16, device="cuda")
    ea.attn_gemm_add(a if K > 0 else None, b if K > 0 else None, c, d, M, N, K)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    return bf16_dev_to_f64(d)


def check(M, N, K, with_c, seed=7):
    ab = gen.normal_bf16(seed, (M, K))
    bb = gen.normal_bf16(seed + 1, (K, N))
    cb = gen.normal_bf16(seed + 2, (M, N)) if with_c else None
    d = run_gemm(ab, bb, cb)
    a64, b64 = gen.bf16_bits_to_f64(ab), gen.bf16_bits_to_f64(bb)
    c64 = None if cb is None else gen.bf16_bits_to_f64(cb)
    ref = oracle.gemm_add(a64, b64, c64)
    assert np.all(np.isfinite(d))
    err = np.abs(d - ref)
    ulp = bf16_ulp(ref)
    acc = K * 2.0 ** -23 * oracle.gemm_add(np.abs(a64), np.abs(b64), None if c64 is None else np.abs(c64))
    assert np.all(err <= ulp + acc), float(np.max(err - ulp - acc))
    assert err.mean() <= 0.5 * ulp.mean() + acc.mean(), (err.mean(), ulp.mean(), acc.mean())


@pytest.mark.parametrize("with_c", [True, False])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (1, 256, 64), (300, 520, 200), (1000, 1000, 8),
                                   (257, 264, 1024), (64, 8, 72), (2048, 4096, 128)])
def test_gemm_add_against_oracle(M, N, K, with_c):
    check(M, N, K, with_c)


def test_zero_k_gives_c():
    cb = gen.normal_bf16(9, (200, 40))
    d = run_gemm(np.zeros((200, 0), dtype=np.uint16), np.zeros((0, 40), dtype=np.uint16), cb)
    assert np.array_equal(d, gen.bf16_bits_to_f64(cb))
    d0 = run_gemm(np.zeros((200, 0), dtype=np.uint16), np.zeros((0, 40), dtype=np.uint16), None)
    assert np.all(d0 == 0)


def test_bench_shape_sampled_rows():
    """The benchmark's shape (M = N = 8192, K = 128): sampled rows against the oracle."""
    M, N, K = 8192, 8192, 128
    ab = gen.normal_bf16(11, (M, K))
    bb = gen.normal_bf16(12, (K, N))
    cb = gen.normal_bf16(13, (M, N))
    d = run_gemm(ab, bb, cb)
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], np.random.default_rng(3).integers(0, M, 28)]))
    a64, b64, c64 = gen.bf16_bits_to_f64(ab[rows]), gen.bf16_bits_to_f64(bb), gen.bf16_bits_to_f64(cb[rows])
    ref = oracle.gemm_add(a64, b64, c64)
    acc = K * 2.0 ** -23 * oracle.gemm_add(np.abs(a64), np.abs(b64), np.abs(c64))
    err = np.abs(d[rows] - ref)
    assert np.all(err <= bf16_ulp(ref) + acc)


def test_in_place_c_is_d():
    """c == d: D += A B in place (each epilogue thread reads its C elements
    before it stores the same elements of D)."""
    import exact_attention_140_b200 as ea
    M, N, K = 300, 520, 64
    ab, bb, cb = gen.normal_bf16(21, (M, K)), gen.normal_bf16(22, (K, N)), gen.normal_bf16(23, (M, N))
    T = torch_mod()
    a, b, cd = to_dev_bf16(ab), to_dev_bf16(bb), to_dev_bf16(cb)
    ea.attn_gemm_add(a, b, cd, cd, M, N, K)
    rc, word = ea.attn_get_last_device_error()
    assert rc == 0, hex(word)
    got = bf16_dev_to_f64(cd)
    ref_out = run_gemm(ab, bb, cb)  # the same product into a separate D
    assert np.array_equal(got, ref_out)
    T.cuda.synchronize()
