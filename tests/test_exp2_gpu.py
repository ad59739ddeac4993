"""The FMA-pipe exp2 of the prompt-phase softmax, on the GPU, against the
exact 2^x (computed in fp64 on the host).

Bound: at most 3 ulp of the fp32 result over [-125, 10] (the minimax
polynomial's own relative error is 1.6e-7, about a third of an ulp at the
top of a binade; the fp32 Horner steps add the rest).  The exponential unit's
ex2.approx is measured beside it for comparison.  Closed forms: 2^n exact at
integers n >= -125, 2^0 = 1, and 2^-125 for every input below -125."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from paged_kv_cache_326_b200 import build
    build.build()
    import paged_kv_cache_326_b200 as P
    P.lib()
    return P


def _run(P, x, method):
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    P.binding.pa_exp2_probe(xd, yd, method)
    torch.cuda.synchronize()
    return yd.cpu().numpy()


def _ulp_err(y, x):
    ex = np.exp2(x.astype(np.float64))
    ulp = np.exp2(np.floor(np.log2(ex)) - 23)
    return np.abs(y.astype(np.float64) - ex) / ulp


def test_polynomial_within_3_ulp_of_exact(P):
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-125, 10, 1 << 22), rng.uniform(-1, 1, 1 << 20),
                        np.arange(-250, 21) / 2.0]).astype(np.float32)
    poly = _ulp_err(_run(P, x, 0), x)
    mufu = _ulp_err(_run(P, x, 1), x)
    print(f"polynomial: max {poly.max():.2f} ulp, mean {poly.mean():.3f}; "
          f"ex2.approx: max {mufu.max():.2f} ulp, mean {mufu.mean():.3f}")
    assert poly.max() <= 3.0


def test_polynomial_closed_forms(P):
    n = np.arange(-125, 11).astype(np.float32)
    assert np.array_equal(_run(P, n, 0), np.exp2(n.astype(np.float64)).astype(np.float32))
    assert _run(P, np.array([0.0, -0.0], dtype=np.float32), 0).tolist() == [1.0, 1.0]
    low = np.array([-125.5, -126, -200, -1e30, -np.inf], dtype=np.float32)
    assert np.all(_run(P, low, 0) == np.float32(2.0 ** -125))
