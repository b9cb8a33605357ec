"""Forward parity of the CUDA path with the CPU oracle, stage by stage.

Every call goes through the C ABI (ctypes binding).  Indices (selection,
gather order, slot map) must match bit for bit; fp32 scores bit for bit;
pooled values within one bf16 ulp; attention outputs, LSE and the layer
output within the bf16 tolerance of ``parity.py``.
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, bf16_ulp, close_report, f64, head
from hierarchical_selection_attention_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

# B, N, H, d, L, p, k, seed: span several 128-row tiles, ragged tails (S % 128),
# both head dims, one to four levels, p = 2 and p = 4.
CASES = [
    (1, 4096, 2, 64, 3, 4, 64, 0),      # the tiny workload (S = 768)
    (2, 2048, 3, 128, 3, 4, 40, 1),     # S = 448: ragged last tile
    (1, 640, 2, 128, 1, 4, 0, 2),       # L = 1: dense causal attention, S = N
    (1, 1000, 2, 64, 2, 2, 50, 3),      # S = 700
    (1, 1024, 2, 128, 4, 2, 20, 4),     # S = 248
    (1, 256, 1, 64, 3, 4, 3, 5),        # S = 40: one partial tile
    (1, 972, 2, 64, 3, 3, 20, 6),       # p = 3: one token per scatter thread, window 9, S = 228
    (1, 515, 1, 128, 1, 2, 0, 7),       # L = 1 with odd N: dense causal over 515
]


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def run_stages(L, cfg, q, k, v):
    B, N, H, d = q.shape
    S, P, R = L.lh_subseq_len(cfg), L.lh_total_entries(cfg), L.lh_pooled_rows(cfg)
    dev = q.device
    e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=dev)
    out = dict(q_lv=e(B * R * H * d), k_lv=e(B * R * H * d), v_lv=e(B * R * H * d),
               qk=e(B, H, P, dt=torch.float32), kq=e(B, H, P, dt=torch.float32),
               sel_idx=e(B, H, S, dt=torch.int32), slot_map=e(B, H, P, dt=torch.int32),
               qg=e(B, H, S, d), kg=e(B, H, S, d), vg=e(B, H, S, d), og=e(B, H, S, d),
               og_lo=e(B, H, S, d), lse=e(B, H, S, dt=torch.float32), o=torch.empty_like(q))
    fwd_ws, _, _ = L.lh_workspace_bytes(cfg)
    ws = torch.empty(fwd_ws, dtype=torch.uint8, device=dev)
    lv = [out[n] if R else None for n in ("q_lv", "k_lv", "v_lv")]
    L.lh_pyramid(cfg, q, k, v, *lv, out["qk"], out["kq"])
    L.lh_score_topk(cfg, out["qk"], out["kq"], out["sel_idx"], out["slot_map"], ws)
    L.lh_gather(cfg, q, k, v, *lv, out["sel_idx"], out["qg"], out["kg"], out["vg"])
    L.lh_attn_fwd(cfg, out["qg"], out["kg"], out["vg"], out["og"], out["lse"], og_lo=out["og_lo"])
    L.lh_scatter(cfg, out["og"], out["slot_map"], out["o"])
    torch.cuda.synchronize()
    L.check_device_status()
    return out


def level_view(x, B, N, H, d, Lv, p, lvl):
    """Level lvl (>= 1) of a pooled buffer as [B, N/p^l, H, d]."""
    start = sum(N // p**j for j in range(1, lvl))
    n = N // p**lvl
    return x.view(-1)[B * start * H * d:B * (start + n) * H * d].view(B, n, H, d)


@pytest.mark.parametrize("B,N,H,d,Lv,p,k,seed", CASES)
def test_forward_stages_match_oracle(L, B, N, H, d, Lv, p, k, seed):
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    cfg = L.make_config(B, N, H, d, Lv, p, k)
    g = run_stages(L, cfg, q, kk, v)
    mism = 0
    for b in range(B):
        for h in range(H):
            st = lo.forward_head(head(q, b, h), head(kk, b, h), head(v, b, h), Lv, p, k, parity=True)
            # scores: fp32 keys bit for bit
            np.testing.assert_array_equal(g["qk"][b, h].cpu().numpy(), st["qk"])
            np.testing.assert_array_equal(g["kq"][b, h].cpu().numpy(), st["kq"])
            # pooled entries within one bf16 ulp of the exactly rounded mean
            for lvl in range(1, Lv):
                for name, idx in (("q_lv", 0), ("k_lv", 1), ("v_lv", 2)):
                    got = f64(level_view(g[name], B, N, H, d, Lv, p, lvl)[b, :, h, :])
                    want = st["levels"][idx][lvl]
                    diff = np.abs(got - want)
                    assert np.all(diff <= bf16_ulp(want) + 1e-300), (name, lvl)
                    mism += int(np.count_nonzero(diff))
            # selection, order and slot map bit for bit
            np.testing.assert_array_equal(g["sel_idx"][b, h].cpu().numpy(), st["sel_idx"])
            np.testing.assert_array_equal(g["slot_map"][b, h].cpu().numpy(), st["slot_map"])
            # gathered rows are the pyramid rows the slots name
            assert_close(f64(g["qg"][b, h]), st["qg"], "qg", max_abs=1e-2, rel_l2=1e-3)
            # og is a convex combination of V rows: its rounding envelope is P |V|
            env_og = lo.attention(st["qg"], st["kg"], np.abs(st["vg"]), st["scale"])[0]
            assert_close(f64(g["og"][b, h]), st["og"], "og", env=env_og)
            # og + og_lo carries the fp32 result: closer to the exact output than og
            o_hi_lo = f64(g["og"][b, h]) + f64(g["og_lo"][b, h])
            o_exact = lo.attention(st["qg"], st["kg"], st["vg"], st["scale"])[0]
            _, rel_hi = close_report(f64(g["og"][b, h]), o_exact)
            _, rel_hl = assert_close(o_hi_lo, o_exact, "og + og_lo", env=env_og)
            assert rel_hl < 0.8 * rel_hi, (rel_hl, rel_hi)
            assert_close(g["lse"][b, h].cpu().numpy(), st["lse"], "lse")
            env = lo.scatter(env_og, st["slot_map"], N, Lv, p)
            assert_close(f64(g["o"][b, :, h, :]), st["o"], "o", env=env)
    # exact-rounding disagreements of pooled values must stay rare
    assert mism <= max(8, B * H * N * d // 2000)


def test_all_equal_scores_take_lowest_indices(L):
    """Constant rows: every key ties, the lower flat index decides."""
    B, N, H, d, Lv, p, k = 1, 1024, 2, 64, 3, 4, 10
    q = torch.full((B, N, H, d), 0.5, dtype=torch.bfloat16, device="cuda")
    cfg = L.make_config(B, N, H, d, Lv, p, k)
    g = run_stages(L, cfg, q, q.clone(), q.clone())
    n_sel = lo.n_select(Lv, p, k)
    sm = g["slot_map"].cpu().numpy()
    C = lo.n_candidates(N, Lv, p)
    for h in range(H):
        assert np.all(sm[0, h, :n_sel] >= 0) and np.all(sm[0, h, n_sel:C] < 0)
        assert np.all(sm[0, h, C:] >= 0)
    # uniform V: every reached position gets V times its fan-in
    st = lo.forward_head(head(q, 0, 0), head(q, 0, 0), head(q, 0, 0), Lv, p, k, parity=True)
    assert_close(f64(g["o"][0, :, 0, :]), st["o"], "o",
                 env=lo.scatter(np.abs(st["og"]), st["slot_map"], N, Lv, p))


def test_forward_entry_point_matches_stages_and_is_deterministic(L):
    B, N, H, d, Lv, p, k, seed = 2, 2048, 3, 128, 3, 4, 40, 1
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    cfg = L.make_config(B, N, H, d, Lv, p, k)
    g = run_stages(L, cfg, q, kk, v)
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    o1 = layer.forward(q, kk, v).clone()
    views = {n: t.clone() for n, t in layer.views().items()}
    o2 = layer.forward(q, kk, v)
    torch.cuda.synchronize()
    L.check_device_status()
    assert torch.equal(o1, o2)
    assert torch.equal(o1, g["o"])
    for n in ("sel_idx", "slot_map", "qg", "kg", "vg", "og", "og_lo", "lse"):
        assert torch.equal(views[n], g[n]), n


def test_integer_atomic_scatter_places_like_pull(L):
    B, N, H, d, Lv, p, k, seed = 1, 4096, 2, 64, 3, 4, 64, 0
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
    cfg = L.make_config(B, N, H, d, Lv, p, k)
    g = run_stages(L, cfg, q, kk, v)
    cfg1 = L.make_config(B, N, H, d, Lv, p, k, scatter_mode=1)
    fwd_ws, _, _ = L.lh_workspace_bytes(cfg1)
    ws = torch.empty(fwd_ws, dtype=torch.uint8, device="cuda")
    o1 = torch.empty_like(q)
    L.lh_scatter(cfg1, g["og"], g["slot_map"], o1, ws)
    o2 = torch.empty_like(q)
    L.lh_scatter(cfg1, g["og"], g["slot_map"], o2, ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert_close(f64(o1), f64(g["o"]), "o atomic vs pull", max_abs=1e-2, rel_l2=1e-3)
    assert torch.equal(o1 == 0, g["o"] == 0)     # same placement


def test_bad_arguments_fail_before_launch(L):
    cfg = L.make_config(1, 100, 2, 64, 3, 4, 1)
    x = torch.empty(1, 100, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LighthouseError):
        L.lh_attn_fwd(cfg, x, x, x, x, torch.empty(10, device="cuda"))
    cfg = L.make_config(1, 4096, 2, 64, 3, 4, 64)
    with pytest.raises(L.LighthouseError):
        L.lh_score_topk(cfg, torch.empty(8, device="cuda"), torch.empty(8, device="cuda"),
                        torch.empty(8, dtype=torch.int32, device="cuda"),
                        torch.empty(8, dtype=torch.int32, device="cuda"),
                        torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert L.lh_get_device_status()[0] == 0
