"""Backward parity of the CUDA path with the CPU oracle.

Stage by stage through the C ABI: the scatter adjoint (dO~ and D), the
attention backward (dQ~, dK~, dV~) and the gather/pooling adjoint, then the
whole lh_backward.  The oracle's gradient is the exact fp64 gradient with the
selection frozen (itself pinned by finite differences), rounded only where
the library stores bf16.
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_bwd_envelopes, close_report, f64, head
from hierarchical_selection_attention_b200.inputs import make_dout, make_qkv

pytestmark = pytest.mark.gpu

CASES = [
    (1, 4096, 2, 64, 3, 4, 64, 0),
    (2, 2048, 3, 128, 3, 4, 40, 1),     # ragged S = 448
    (1, 640, 2, 128, 1, 4, 0, 2),       # dense causal
    (1, 1000, 2, 64, 2, 2, 50, 3),
    (1, 1024, 2, 128, 4, 2, 20, 4),
    (1, 256, 1, 64, 3, 4, 3, 5),        # S = 40
    (1, 972, 2, 64, 3, 3, 20, 6),       # p = 3: one token per scatter thread, window 9, S = 228
    (1, 515, 1, 128, 1, 2, 0, 7),       # L = 1 with odd N: dense causal over 515
]


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def oracle_backward(st, doh):
    N, Lv, p = st["N"], st["L"], st["p"]
    dog = lo.round_bf16(lo.scatter_bwd(doh, st["sel_idx"], N, Lv, p))
    dqg, dkg, dvg = lo.attention_bwd(st["qg"], st["kg"], st["vg"], dog, st["scale"])
    grads_g = [lo.round_bf16(x) for x in (dqg, dkg, dvg)]
    grads = [lo.pyramid_bwd(x, st["slot_map"], N, Lv, p) for x in grads_g]
    envs_g = attn_bwd_envelopes(st["qg"], st["kg"], st["vg"], dog, st["scale"])
    envs = [lo.pyramid_bwd(e, st["slot_map"], N, Lv, p) for e in envs_g]
    o_exact = lo.attention(st["qg"], st["kg"], st["vg"], st["scale"])[0]
    return dict(dog=dog, delta=np.sum(dog * o_exact, axis=1),
                delta_env=np.sum(np.abs(dog * o_exact), axis=1), grads_g=(dqg, dkg, dvg),
                envs_g=envs_g, grads=grads, envs=envs)


@pytest.mark.parametrize("B,N,H,d,Lv,p,k,seed", CASES)
def test_backward_matches_oracle(L, B, N, H, d, Lv, p, k, seed):
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    dout = make_dout(B, N, H, d, seed).cuda()
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    layer.forward(q, kk, v)
    sv = layer.views()
    cfg = layer.cfg
    S = layer.S
    dev = q.device
    # stage by stage
    dog = torch.empty(B, H, S, d, dtype=torch.bfloat16, device=dev)
    delta = torch.empty(B, H, S, dtype=torch.float32, device=dev)
    L.lh_scatter_bwd(cfg, dout, sv["og"], sv["sel_idx"], dog, delta, og_lo=sv["og_lo"])
    dqg, dkg, dvg = (torch.empty(B, H, S, d, dtype=torch.bfloat16, device=dev) for _ in range(3))
    _, bwd_ws, _ = L.lh_workspace_bytes(cfg)
    ws = torch.empty(bwd_ws, dtype=torch.uint8, device=dev)
    L.lh_attn_bwd(cfg, sv["qg"], sv["kg"], sv["vg"], sv["og"], sv["lse"], dog, dqg, dkg, dvg, ws,
                  og_lo=sv["og_lo"])
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    L.lh_gather_bwd(cfg, dqg, dkg, dvg, sv["slot_map"], dq, dk, dv)
    # whole backward
    g2 = layer.backward(dout)
    torch.cuda.synchronize()
    L.check_device_status()
    for a, b2 in zip((dq, dk, dv), g2):
        assert torch.equal(a, b2)
    for b in range(B):
        for h in range(H):
            st = lo.forward_head(head(q, b, h), head(kk, b, h), head(v, b, h), Lv, p, k, parity=True)
            ref = oracle_backward(st, head(dout, b, h))
            assert_close(f64(dog[b, h]), ref["dog"], "dog")
            assert_close(delta[b, h].cpu().numpy(), ref["delta"], "delta", env=ref["delta_env"])
            for name, got, want, env in zip(("dqg", "dkg", "dvg"), (dqg, dkg, dvg), ref["grads_g"],
                                            ref["envs_g"]):
                print(name, b, h, "max-abs(scaled|y|) %.2e rel-L2 %.2e" % close_report(f64(got[b, h]), want),
                      "envelope-scaled %.2e" % close_report(f64(got[b, h]), want, env)[0])
                assert_close(f64(got[b, h]), want, name, env=env)
            for name, got, want, env in zip(("dq", "dk", "dv"), (dq, dk, dv), ref["grads"], ref["envs"]):
                assert_close(f64(got[b, :, h, :]), want, name, env=env)


def test_backward_is_deterministic(L):
    B, N, H, d, Lv, p, k, seed = 1, 4096, 2, 64, 3, 4, 64, 0
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    dout = make_dout(B, N, H, d, seed).cuda()
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    layer.forward(q, kk, v)
    a = [t.clone() for t in layer.backward(dout)]
    b = layer.backward(dout)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_autograd_wrapper(L):
    B, N, H, d, Lv, p, k, seed = 1, 1024, 2, 64, 3, 4, 16, 7
    q, kk, v = (t.cuda().requires_grad_() for t in make_qkv(B, N, H, d, seed))
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    o = L.LighthouseAttention.apply(q, kk, v, layer)
    dout = make_dout(B, N, H, d, seed).cuda()
    o.backward(dout)
    ref = layer.backward(dout)
    torch.cuda.synchronize()
    assert torch.equal(q.grad, ref[0]) and torch.equal(kk.grad, ref[1]) and torch.equal(v.grad, ref[2])
