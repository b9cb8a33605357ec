"""The per-level-quota selection (select_mode 1) on the GPU against the
oracle: selection, gather order and slot map bit for bit, the layer output
and the gradients within the bf16 tolerance, through lh_forward and
lh_backward (LighthouseLayer)."""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_bwd_envelopes, f64, head
from hierarchical_selection_attention_b200.inputs import make_dout, make_qkv

pytestmark = pytest.mark.gpu

# B, N, H, d, L, p, k, seed: p k fits the coarsest finer level in each
CASES = [
    (1, 4096, 2, 64, 3, 4, 64, 0),
    (2, 2048, 3, 128, 3, 4, 40, 1),     # ragged S = 448
    (1, 1024, 2, 128, 4, 2, 20, 4),     # three finer levels
    (1, 256, 1, 64, 3, 4, 3, 5),        # S = 40
]


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


@pytest.mark.parametrize("B,N,H,d,Lv,p,k,seed", CASES)
def test_quota_layer_matches_oracle(L, B, N, H, d, Lv, p, k, seed):
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    dout = make_dout(B, N, H, d, seed).cuda()
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, select_mode=1)
    o = layer.forward(q, kk, v)
    dq, dk, dv = layer.backward(dout)
    torch.cuda.synchronize()
    L.check_device_status()
    sv = layer.views()
    for b in range(B):
        for h in range(H):
            st = lo.forward_head(head(q, b, h), head(kk, b, h), head(v, b, h), Lv, p, k,
                                 parity=True, select_mode=1)
            np.testing.assert_array_equal(sv["sel_idx"][b, h].cpu().numpy(), st["sel_idx"])
            np.testing.assert_array_equal(sv["slot_map"][b, h].cpu().numpy(), st["slot_map"])
            # exactly p k entries from each finer level
            offs = lo.level_offsets(N, Lv, p)
            for l in range(Lv - 1):
                assert int(st["flags"][offs[l]:offs[l] + N // p**l].sum()) == p * k
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


def test_two_levels_quota_equals_joint(L):
    # one finer level: the quota is the whole budget, so both modes agree bit for bit
    B, N, H, d, Lv, p, k, seed = 1, 1000, 2, 64, 2, 2, 50, 3
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    outs = []
    for mode in (0, 1):
        layer = L.LighthouseLayer(B, N, H, d, Lv, p, k, select_mode=mode)
        outs.append((layer.forward(q, kk, v).clone(), layer.views()["sel_idx"].clone()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][0], outs[1][0])
