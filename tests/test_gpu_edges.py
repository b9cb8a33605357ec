"""Degenerate shapes of the method on the GPU against the oracle: no finer
entry selected (k = 0 with L > 1, so the gathered sequence is the coarsest
level alone), in both selection modes, with several batch rows and an odd
number of heads."""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_bwd_envelopes, f64, head
from hierarchical_selection_attention_b200.inputs import make_dout, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


@pytest.mark.parametrize("B,N,H,d,Lv,p,k,mode,seed", [
    (2, 1024, 3, 64, 3, 4, 0, 0, 11),    # S = N / 16: the coarsest level only
    (1, 2048, 1, 128, 2, 2, 0, 1, 12),   # quota mode with nothing to take
    (3, 512, 1, 64, 3, 2, 1, 1, 13),     # one entry per finer level per head
])
def test_degenerate_selection(L, B, N, H, d, Lv, p, k, mode, seed):
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    dout = make_dout(B, N, H, d, seed).cuda()
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, select_mode=mode)
    assert layer.S == N // p ** (Lv - 1) + (Lv - 1) * p * k
    o = layer.forward(q, kk, v)
    dq, dk, dv = layer.backward(dout)
    torch.cuda.synchronize()
    L.check_device_status()
    sv = layer.views()
    for b in range(B):
        for h in range(H):
            st = lo.forward_head(head(q, b, h), head(kk, b, h), head(v, b, h), Lv, p, k,
                                 parity=True, select_mode=mode)
            np.testing.assert_array_equal(sv["sel_idx"][b, h].cpu().numpy(), st["sel_idx"])
            env_og = lo.attention(st["qg"], st["kg"], np.abs(st["vg"]), st["scale"])[0]
            assert_close(f64(o[b, :, h, :]), st["o"], "o",
                         env=lo.scatter(env_og, st["slot_map"], N, Lv, p))
            # uncovered base positions (before the first coarse entry ends) stay 0
            if k == 0:
                assert np.all(f64(o[b, :p ** (Lv - 1) - 1, h, :]) == 0)
            dog = lo.round_bf16(lo.scatter_bwd(head(dout, b, h), st["sel_idx"], N, Lv, p))
            grads = lo.attention_bwd(st["qg"], st["kg"], st["vg"], dog, st["scale"])
            envs = attn_bwd_envelopes(st["qg"], st["kg"], st["vg"], dog, st["scale"])
            for name, gpu, gg, eg in zip(("dq", "dk", "dv"), (dq, dk, dv), grads, envs):
                want = lo.pyramid_bwd(lo.round_bf16(gg), st["slot_map"], N, Lv, p)
                assert_close(f64(gpu[b, :, h, :]), want, name,
                             env=lo.pyramid_bwd(eg, st["slot_map"], N, Lv, p))
