"""Complete parity of one head at every full workload size, in the launch
configuration the benchmark times (lh_forward + lh_backward on [B, N, H, d]
bf16).

For one (b, h) per workload the oracle runs the whole layer, forward and
backward, over all S gathered rows and all N tokens ("Long Context
Pre-Training with Lighthouse Attention", Sec. 3.3-3.6; the backward as
Sec. 3.2 prescribes), and every value is compared:

- the gathered sub-sequence results the layer leaves behind: the attention
  output og and its LSE (saved buffer), the scatter adjoint dog and the
  gathered gradients dqg, dkg, dvg (backward scratch).  dkg and dvg of the
  first slots are the longest reductions of the backward (a key row of slot
  m sums over all S - m query rows), which is why the whole head is checked
  rather than a sample;
- the token outputs O, dQ, dK and dV at all N positions.

Each comparison records its plain max-abs, its envelope-scaled max-abs and
its rel-L2 (tests/parity.py writes them to tests/results/).
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_envelopes_full, head, record
from hierarchical_selection_attention_b200.inputs import WORKLOADS, make_dout, make_qkv

pytestmark = pytest.mark.gpu

# fp32 LSE of the kernel (fp32 scores and row sums, ex2.approx) against the
# oracle's fp64 one: an absolute bound; the pages fix no precision for it
LSE_ABS = 1e-3


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


@pytest.mark.parametrize("wi", [1, 2, 3, 4])
def test_fullsize_one_head_complete(L, wi):
    w = WORKLOADS[wi]
    B, N, H, d, Lv, p, k = (w[x] for x in ("B", "N", "H", "d", "L", "p", "k"))
    qh, kh, vh = make_qkv(B, N, H, d, seed=wi)
    doh = make_dout(B, N, H, d, seed=wi)
    q, kk, v, dout = (t.cuda() for t in (qh, kh, vh, doh))
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    o = layer.forward(q, kk, v)
    dq, dk, dv = layer.backward(dout)
    torch.cuda.synchronize()
    L.check_device_status()
    sv, bv = layer.views(), layer.bwd_views()
    b, h = B - 1, (3 * wi) % H
    gat = lambda t: t[b, h].double().cpu().numpy()
    tok = lambda t: t[b, :, h, :].double().cpu().numpy()
    tag = f"{w['name']}[b={b},h={h}]"

    # ---- oracle, whole head
    qx, kx, vx, dox = (head(x, b, h) for x in (qh, kh, vh, doh))
    st = lo.forward_head(qx, kx, vx, Lv, p, k, parity=True)
    np.testing.assert_array_equal(sv["sel_idx"][b, h].cpu().numpy(), st["sel_idx"])
    np.testing.assert_array_equal(sv["slot_map"][b, h].cpu().numpy(), st["slot_map"])
    scale = st["scale"]
    dog = lo.round_bf16(lo.scatter_bwd(dox, st["sel_idx"], N, Lv, p))
    dqg, dkg, dvg = lo.attention_bwd(st["qg"], st["kg"], st["vg"], dog, scale)
    grads = [lo.pyramid_bwd(lo.round_bf16(g), st["slot_map"], N, Lv, p) for g in (dqg, dkg, dvg)]
    eo, eq, ek, ev = attn_envelopes_full(st["qg"], st["kg"], st["vg"], dog, scale)

    # ---- gathered sub-sequence (S rows)
    assert_close(gat(sv["og"]), st["og"], f"og {tag}", env=eo)
    lse = sv["lse"][b, h].double().cpu().numpy()
    record(lse, st["lse"], f"lse {tag}")
    assert np.max(np.abs(lse - st["lse"])) <= LSE_ABS, f"lse {tag}"
    assert_close(gat(bv["dog"]), dog, f"dog {tag}")
    assert_close(gat(bv["dqg"]), dqg, f"dqg {tag}", env=eq)
    assert_close(gat(bv["dkg"]), dkg, f"dkg {tag}", env=ek)
    assert_close(gat(bv["dvg"]), dvg, f"dvg {tag}", env=ev)

    # ---- token outputs (N rows); envelopes pushed through the same linear maps
    env_o = lo.scatter(eo, st["slot_map"], N, Lv, p)
    assert_close(tok(o), st["o"], f"O {tag}", env=env_o)
    for name, gpu, want, env in (("dQ", dq, grads[0], eq), ("dK", dk, grads[1], ek),
                                 ("dV", dv, grads[2], ev)):
        env_t = lo.pyramid_bwd(env, st["slot_map"], N, Lv, p)
        assert_close(tok(gpu), want, f"{name} {tag}", env=env_t)
