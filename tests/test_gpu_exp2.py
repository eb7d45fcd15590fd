"""The softmax exponential as the kernel computes it, against 2^x in fp64:
the hardware approximation and the software polynomial (Cody-Waite split +
degree-3 polynomial fitted by exact_attention_140_b200/csrc/fit_exp2_poly.py)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def run(x, mode):
    import torch

    import exact_attention_140_b200 as ea
    xd = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    yd = torch.empty_like(xd)
    ea.attn_debug_exp2(xd, yd, xd.numel(), mode)
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def inputs():
    rng = np.random.default_rng(5)
    x = rng.uniform(-125.0, 8.0, size=1 << 22).astype(np.float32)
    edges = np.array([0.0, -0.0, 1.0, -1.0, 0.5, -0.5, 0.49999997, -0.50000006, 8.0, -125.0, -124.5,
                      1e-8, -1e-8, 3.25, -7.75], dtype=np.float32)
    return np.concatenate([edges, x])


@pytest.mark.parametrize("mode,bound", [(0, 2.0 ** -20), (1, 1.2e-4)])
def test_exp2_relative_error(mode, bound):
    x = inputs()
    y = run(x, mode)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= bound, (mode, rel.max(), x[np.argmax(rel)])


@pytest.mark.parametrize("mode", [0, 1])
def test_exp2_of_zero_is_one(mode):
    y = run(np.array([0.0, -0.0], dtype=np.float32), mode)
    assert y.tolist() == [1.0, 1.0]


def test_exp2_integers_exact_in_software():
    x = np.arange(-120, 9, dtype=np.float32)
    y = run(x, 1)
    assert np.array_equal(y, np.exp2(x.astype(np.float64)))


def test_exp2_below_range():
    x = np.array([-np.inf, -1000.0, -130.0, -126.5], dtype=np.float32)
    assert np.all(run(x, 0) == 0.0)  # hardware path flushes to zero (masked keys use it)
    ys = run(x, 1)  # software path clamps at 2^-125: negligible next to a row sum >= 1
    assert np.all(ys <= 2.0 ** -124) and np.all(ys >= 0.0)
