"""Pins of the oracle's projected layer (projections around the Lighthouse
layer, Sec. 3.1): central finite differences of <y, dy> with the selection
frozen (pure fp64 mode) against projected_backward, for the input and for
every weight; and the plain products themselves on exact small-integer
data."""
import numpy as np
import pytest

from oracle import lighthouse_oracle as lo


def _setup(seed=0, B=1, N=32, H=2, d=4, Dm=6, L=2, p=2, k=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, N, Dm))
    w = [rng.standard_normal((H * d, Dm)) * 0.5 for _ in range(3)] + [rng.standard_normal((Dm, H * d)) * 0.5]
    dy = rng.standard_normal((B, N, Dm))
    y, st = lo.projected_forward(x, *w, H, L, p, k, parity=False)
    flags = {key: s["flags"] for key, s in st["states"].items()}
    return x, w, dy, st, flags, (H, L, p, k)


def _loss(x, w, dy, flags, cfg):
    y, _ = lo.projected_forward(x, *w, *cfg, parity=False, flags=flags)
    return float(np.sum(y * dy))


@pytest.mark.parametrize("which", ["x", "wq", "wk", "wv", "wo"])
def test_projected_gradients_match_finite_differences(which):
    x, w, dy, st, flags, cfg = _setup()
    dx, dwq, dwk, dwv, dwo = lo.projected_backward(st, dy)
    analytic = dict(x=dx, wq=dwq, wk=dwk, wv=dwv, wo=dwo)[which]
    rng = np.random.default_rng(1)
    eps = 1e-6
    for _ in range(6):
        idx = tuple(rng.integers(0, n) for n in analytic.shape)
        xs, ws = x.copy(), [a.copy() for a in w]
        target = xs if which == "x" else ws[["wq", "wk", "wv", "wo"].index(which)]
        target[idx] += eps
        lp = _loss(xs, ws, dy, flags, cfg)
        target[idx] -= 2 * eps
        lm = _loss(xs, ws, dy, flags, cfg)
        fd = (lp - lm) / (2 * eps)
        assert abs(fd - analytic[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, analytic[idx])


def test_projection_products_on_exact_data():
    # with identity projections Q = K = V = x and y = O: the layer alone
    B, N, H, d, L, p, k = 1, 64, 2, 4, 3, 2, 2
    Dm = H * d
    x = np.random.default_rng(2).integers(-4, 5, size=(B, N, Dm)).astype(float)
    eye = np.eye(Dm)
    y, st = lo.projected_forward(x, eye, eye, eye, eye, H, L, p, k, parity=False)
    o_ref, _ = lo.forward(x.reshape(B, N, H, d), x.reshape(B, N, H, d), x.reshape(B, N, H, d),
                          L, p, k, parity=False)
    assert np.allclose(y, o_ref.reshape(B, N, Dm), rtol=0, atol=1e-12)
