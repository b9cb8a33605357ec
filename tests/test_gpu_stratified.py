"""The stratified selection (select_mode 2) on the GPU against the oracle:
selection, gather order and slot map bit for bit, the layer output and the
gradients within the bf16 tolerance, through lh_forward and lh_backward
(LighthouseLayer); the selection alone at the 64K workload's full size."""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_bwd_envelopes, f64, head
from hierarchical_selection_attention_b200.inputs import WORKLOADS, make_dout, make_qkv

pytestmark = pytest.mark.gpu

# B, N, H, d, L, p, k, chunk quota m, seed
CASES = [
    (1, 4096, 2, 64, 3, 4, 64, 64, 0),      # 8 chunks of 640
    (2, 2048, 3, 128, 3, 4, 40, 20, 1),     # 16 chunks of 160, ragged S = 448
    (1, 1024, 2, 128, 4, 2, 20, 8, 4),      # 15 chunks over 1792 candidates (119 / 120)
    (1, 256, 1, 64, 3, 4, 3, 1, 5),         # 24 chunks of 13 / 14, one entry each
]


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


@pytest.mark.parametrize("B,N,H,d,Lv,p,k,m,seed", CASES)
def test_stratified_layer_matches_oracle(L, B, N, H, d, Lv, p, k, m, seed):
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    dout = make_dout(B, N, H, d, seed).cuda()
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, select_mode=2, select_chunk=m)
    o = layer.forward(q, kk, v)
    dq, dk, dv = layer.backward(dout)
    torch.cuda.synchronize()
    L.check_device_status()
    sv = layer.views()
    C, n = lo.n_candidates(N, Lv, p), lo.n_select(Lv, p, k) // m
    for b in range(B):
        for h in range(H):
            st = lo.forward_head(head(q, b, h), head(kk, b, h), head(v, b, h), Lv, p, k,
                                 parity=True, select_mode=2, select_chunk=m)
            np.testing.assert_array_equal(sv["sel_idx"][b, h].cpu().numpy(), st["sel_idx"])
            np.testing.assert_array_equal(sv["slot_map"][b, h].cpu().numpy(), st["slot_map"])
            for s in range(n):   # exactly m entries from each chunk
                assert int(st["flags"][s * C // n:(s + 1) * C // n].sum()) == m
            env_og = lo.attention(st["qg"], st["kg"], np.abs(st["vg"]), st["scale"])[0]
            env = lo.scatter(env_og, st["slot_map"], N, Lv, p)
            assert_close(f64(o[b, :, h, :]), st["o"], "o", env=env)
            dog = lo.round_bf16(lo.scatter_bwd(head(dout, b, h), st["sel_idx"], N, Lv, p))
            grads_g = lo.attention_bwd(st["qg"], st["kg"], st["vg"], dog, st["scale"])
            envs_g = attn_bwd_envelopes(st["qg"], st["kg"], st["vg"], dog, st["scale"])
            for name, gpu, gg, eg in zip(("dq", "dk", "dv"), (dq, dk, dv), grads_g, envs_g):
                want = lo.pyramid_bwd(lo.round_bf16(gg), st["slot_map"], N, Lv, p)
                env_t = lo.pyramid_bwd(eg, st["slot_map"], N, Lv, p)
                assert_close(f64(gpu[b, :, h, :]), want, name, env=env_t)


def test_stratified_selection_full_size(L):
    # the 64K workload (H = 8, d = 128, k = 1024): 8192 entries in 64 chunks of 1280
    w = WORKLOADS[1]
    B, N, H, d, Lv, p, k = (w[x] for x in ("B", "N", "H", "d", "L", "p", "k"))
    m = 128
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed=1))
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, select_mode=2, select_chunk=m)
    layer.forward(q, kk, v)
    torch.cuda.synchronize()
    L.check_device_status()
    sv = layer.views()
    for b in range(B):
        for h in range(H):
            st = lo.select_head(head(q, b, h), head(kk, b, h), Lv, p, k,
                                select_mode=2, select_chunk=m)
            np.testing.assert_array_equal(sv["sel_idx"][b, h].cpu().numpy(), st["sel_idx"])
            np.testing.assert_array_equal(sv["slot_map"][b, h].cpu().numpy(), st["slot_map"])


def test_one_chunk_equals_joint(L):
    # m = n_sel: a single chunk over all candidates is the joint selection, bit for bit
    B, N, H, d, Lv, p, k, seed = 1, 4096, 2, 64, 3, 4, 64, 6
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    outs = []
    for mode, m in ((0, 0), (2, lo.n_select(Lv, p, k))):
        layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, select_mode=mode, select_chunk=m)
        outs.append((layer.forward(q, kk, v).clone(), layer.views()["sel_idx"].clone()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][0], outs[1][0])
