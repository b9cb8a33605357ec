"""The layer with its projections (LighthouseProjectedLayer: lh_gemm around
lh_forward / lh_backward) against the oracle's projected layer.

The weights are sparse with entries in {1, -1/2} (two per row), so every
forward projection is a sum of two exact products: the library's fp32 sum and
the oracle's fp64 sum round to the same bf16 Q, K, V, and the selection can
be compared bit for bit.  Outputs and gradients are compared within the bf16
tolerance, with envelopes propagated through the final products."""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_bwd_envelopes, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def _sparse_weight(rows, cols, shift):
    w = np.zeros((rows, cols))
    for r in range(rows):
        w[r, (r + shift) % cols] += 1.0
        w[r, (7 * r + 3 + shift) % cols] -= 0.5
    return w


@pytest.mark.parametrize("B,N,H,d,Dm,Lv,p,k,seed", [
    (1, 2048, 2, 64, 128, 3, 4, 32, 0),
    (1, 1024, 2, 128, 256, 3, 4, 16, 1),
])
def test_projected_layer_matches_oracle(L, B, N, H, d, Dm, Lv, p, k, seed):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(B, N, Dm, generator=gen).to(torch.bfloat16)
    dy = torch.randn(B, N, Dm, generator=gen).to(torch.bfloat16)
    w64 = [_sparse_weight(H * d, Dm, s) for s in (0, 5, 11)] + [_sparse_weight(Dm, H * d, 17)]
    w = [torch.tensor(a, dtype=torch.bfloat16).cuda() for a in w64]
    layer = L.LighthouseProjectedLayer(B, N, H, d, Dm, Lv, p, k)
    y = layer.forward(x.cuda(), *w)
    dx, dwq, dwk, dwv, dwo = layer.backward(dy.cuda())
    torch.cuda.synchronize()
    L.check_device_status()

    x64, dy64 = f64(x), f64(dy)
    y_ref, st = lo.projected_forward(x64, *w64, H, Lv, p, k, parity=True)
    # exact forward projections, hence the same selection bit for bit
    for name, got in (("q", layer.q), ("k", layer.k), ("v", layer.v)):
        np.testing.assert_array_equal(f64(got), st[name], err_msg=name)
    sel = layer.core.views()["sel_idx"].cpu().numpy()
    for (b, h), sh in st["states"].items():
        np.testing.assert_array_equal(sel[b, h], sh["sel_idx"])

    # envelopes of O and of dQ, dK, dV (per head), then through the products
    env_o = np.zeros_like(st["o"])
    env_g = [np.zeros_like(st["o"]) for _ in range(3)]
    do_ref = lo.round_bf16(dy64 @ w64[3]).reshape(st["o"].shape)
    for (b, h), sh in st["states"].items():
        e = lo.attention(sh["qg"], sh["kg"], np.abs(sh["vg"]), sh["scale"])[0]
        env_o[b, :, h, :] = lo.scatter(e, sh["slot_map"], N, Lv, p)
        dog = lo.round_bf16(lo.scatter_bwd(do_ref[b, :, h, :], sh["sel_idx"], N, Lv, p))
        for a, eg in enumerate(attn_bwd_envelopes(sh["qg"], sh["kg"], sh["vg"], dog, sh["scale"])):
            env_g[a][b, :, h, :] = lo.pyramid_bwd(eg, sh["slot_map"], N, Lv, p)
    T = B * N
    o_mag = (np.abs(st["o"]) + env_o).reshape(T, -1)
    assert_close(f64(y).reshape(T, Dm), y_ref.reshape(T, Dm), "y", env=o_mag @ np.abs(w64[3]).T)

    ref = lo.projected_backward(st, dy64)
    grads_ref = lo.backward(st["states"], do_ref)
    g_mag = [(np.abs(lo.round_bf16(g)) + e).reshape(T, -1) for g, e in zip(grads_ref, env_g)]
    env_dx = sum(gm @ np.abs(wi) for gm, wi in zip(g_mag, w64[:3]))
    assert_close(f64(dx).reshape(T, Dm), ref[0].reshape(T, Dm), "dx", env=env_dx)
    xm = np.abs(x64).reshape(T, Dm)
    for name, got, want, gm in zip(("dwq", "dwk", "dwv"), (dwq, dwk, dwv), ref[1:4], g_mag):
        assert_close(f64(got), want, name, env=gm.T @ xm)
    assert_close(f64(dwo), ref[4], "dwo", env=np.abs(dy64).reshape(T, Dm).T @ o_mag)
