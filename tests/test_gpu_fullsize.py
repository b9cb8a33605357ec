"""Parity at the full workload sizes, in the launch configuration the
benchmark times (lh_forward + lh_backward on [B, N, H, d] bf16).

The oracle cannot run these layers whole, so:
- selection, gather order and slot map: every (b, h), bit for bit;
- layer output O: sampled base positions of two heads, through the oracle
  attention rows that reach them;
- dQ: sampled positions (a dQ~ row needs only its own attention row);
- dK, dV: positions near the end of the sequence, whose gathered entries sit
  in the last slots, so the oracle needs only the attention rows after them.
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, attn_bwd_envelopes, head
from hierarchical_selection_attention_b200.inputs import WORKLOADS, make_dout, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def _slots_of(t, sm, N, Lv, p, shifted):
    """Slots of the entries that reach base position t (scatter: shifted
    window; gather adjoint: plain window), level by level."""
    offs = lo.level_offsets(N, Lv, p)
    out = []
    for lvl in range(Lv):
        j = (t + 1) // p**lvl - 1 if shifted else t // p**lvl
        if j >= 0:
            s = int(sm[offs[lvl] + j])
            if s >= 0:
                out.append((lvl, s))
    return out


@pytest.mark.parametrize("wi", [1, 2, 3, 4])
def test_fullsize_parity(L, wi):
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
    sv = layer.views()
    S = layer.S
    sel_gpu = sv["sel_idx"].cpu().numpy()
    sm_gpu = sv["slot_map"].cpu().numpy()
    rng = np.random.default_rng(1000 + wi)
    checked = 0
    for b in range(B):
        for h in range(H):
            qx, kx = head(qh, b, h), head(kh, b, h)
            sel = lo.select_head(qx, kx, Lv, p, k)
            np.testing.assert_array_equal(sel_gpu[b, h], sel["sel_idx"])
            np.testing.assert_array_equal(sm_gpu[b, h], sel["slot_map"])
            if checked >= 2:
                continue
            checked += 1
            vx, dox = head(vh, b, h), head(doh, b, h)
            # --- O at sampled positions (both ends, heavy middle)
            ts = np.unique(np.concatenate([[0, 1, 15, 16, N - 1, N - 2],
                                           rng.integers(0, N, 26)]))
            want, aux = lo.outputs_at(qx, kx, vx, Lv, p, k, ts, sel=sel)
            env_rows = lo.attention(aux["qg"], aux["kg"], np.abs(aux["vg"]), 1.0 / np.sqrt(d),
                                    rows=aux["rows"])[0]
            pos = {int(s): n for n, s in enumerate(aux["rows"])}
            env = np.zeros_like(want)
            for n, t in enumerate(ts):
                for _, s in _slots_of(int(t), sel["slot_map"], N, Lv, p, shifted=True):
                    env[n] += env_rows[pos[s]]
            got = o[b, ts, h, :].double().cpu().numpy()
            assert_close(got, want, f"O[{b},{h}]", env=env)
            # --- gradients
            qg, kg, vg = aux["qg"], aux["kg"], aux["vg"]
            scale = 1.0 / np.sqrt(d)
            dog = lo.round_bf16(lo.scatter_bwd(dox, sel["sel_idx"], N, Lv, p))
            # dQ at sampled positions: dQ~ rows of the slots that contain them
            tq = np.unique(rng.integers(0, N, 24))
            need = sorted({s for t in tq for _, s in _slots_of(int(t), sel["slot_map"], N, Lv, p, False)})
            dqg_rows, _, _ = lo.attention_bwd(qg, kg, vg, dog, scale, rows=np.array(need))
            env_q, _, _ = attn_bwd_envelopes(qg, kg, vg, dog, scale, rows=np.array(need))
            want_dq, env_dq = np.zeros((len(tq), d)), np.zeros((len(tq), d))
            for n, t in enumerate(tq):
                for lvl, s in _slots_of(int(t), sel["slot_map"], N, Lv, p, False):
                    want_dq[n] += lo.round_bf16(dqg_rows[s]) / p**lvl
                    env_dq[n] += env_q[s] / p**lvl
            got_dq = dq[b, tq, h, :].double().cpu().numpy()
            assert_close(got_dq, want_dq, f"dQ[{b},{h}]", env=env_dq)
            # dK, dV at the last positions: their entries occupy the last slots
            tk = np.arange(N - 48, N)
            need = sorted({s for t in tk for _, s in _slots_of(int(t), sel["slot_map"], N, Lv, p, False)})
            m0 = min(need)
            _, dkg, dvg = lo.attention_bwd(qg, kg, vg, dog, scale, rows=np.arange(m0, S))
            _, env_k, env_v = attn_bwd_envelopes(qg, kg, vg, dog, scale, rows=np.arange(m0, S))
            for name, gg, ee, gpu in (("dK", dkg, env_k, dk), ("dV", dvg, env_v, dv)):
                want_g, env_g = np.zeros((len(tk), d)), np.zeros((len(tk), d))
                for n, t in enumerate(tk):
                    for lvl, s in _slots_of(int(t), sel["slot_map"], N, Lv, p, False):
                        want_g[n] += lo.round_bf16(gg[s]) / p**lvl
                        env_g[n] += ee[s] / p**lvl
                got_g = gpu[b, tk, h, :].double().cpu().numpy()
                assert_close(got_g, want_g, f"{name}[{b},{h}]", env=env_g)
