"""lh_score_topk_noalloc: the top-k and order for callers that cannot
allocate device memory (their memory belongs to another allocator, or their
interface has no room for a scratch pointer).  Its scratch is a fixed device
array inside the library instead of a caller workspace.

Checked through the C ABI against lh_score_topk with a workspace, on calls
in a row with different shapes, so that whatever one call leaves in the
shared array cannot change the next one's result.  Indices must match bit
for bit.  This file is collected last on purpose.
"""
import pytest
import torch

from hierarchical_selection_attention_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

# B, N, H, d, L, p, k, seed, select_mode, select_chunk: every selection mode,
# with a shape change between calls so no call can lean on the last one's
# leftovers
SHAPES = [(1, 4096, 2, 64, 3, 4, 64, 0, 0, 0), (2, 2048, 3, 128, 3, 4, 40, 1, 0, 0),
          (1, 4096, 2, 64, 3, 4, 64, 0, 1, 0), (1, 8192, 2, 64, 4, 4, 32, 2, 1, 0),
          (1, 4096, 2, 64, 3, 4, 64, 0, 2, 32), (2, 2048, 3, 128, 3, 4, 40, 1, 2, 20),
          (1, 4096, 2, 64, 3, 4, 64, 0, 0, 0)]


def _scores(L, cfg, q, k, v):
    B, N, H, d = q.shape
    P, R = L.lh_total_entries(cfg), L.lh_pooled_rows(cfg)
    lv = [torch.empty(max(B * R * H * d, 1), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    qk = torch.empty(B, H, P, dtype=torch.float32, device="cuda")
    kq = torch.empty_like(qk)
    L.lh_pyramid(cfg, q, k, v, *lv, qk, kq)
    return qk, kq


def test_noalloc_topk_matches_workspace_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse as L

    assert L.lh_score_topk_noalloc_max_bytes() == 8 << 20
    for B, N, H, d, Lv, p, k, seed, mode, chunk in SHAPES:
        q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed))
        cfg = L.make_config(B, N, H, d, Lv, p, k, select_mode=mode, select_chunk=chunk)
        S, P = L.lh_subseq_len(cfg), L.lh_total_entries(cfg)
        qk, kq = _scores(L, cfg, q, kk, v)
        fws, _, _ = L.lh_workspace_bytes(cfg)
        ws = torch.empty(fws, dtype=torch.uint8, device="cuda")
        sel_ref = torch.empty(B, H, S, dtype=torch.int32, device="cuda")
        sm_ref = torch.empty(B, H, P, dtype=torch.int32, device="cuda")
        L.lh_score_topk(cfg, qk, kq, sel_ref, sm_ref, ws)
        for _ in range(2):  # two calls in a row on the same shared array
            sel = torch.full((B, H, S), -7, dtype=torch.int32, device="cuda")
            sm = torch.full((B, H, P), -7, dtype=torch.int32, device="cuda")
            L.lh_score_topk_noalloc(cfg, qk, kq, sel, sm)
            torch.cuda.synchronize()
            assert torch.equal(sel, sel_ref)
            assert torch.equal(sm, sm_ref)
    L.check_device_status()


def test_noalloc_topk_rejects_shapes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse as L

    x = torch.empty(16, dtype=torch.float32, device="cuda")
    i = torch.empty(16, dtype=torch.int32, device="cuda")
    # B*H = 512 heads: ~27 MB of scratch; and the per-level quota at B*H = 128,
    # L = 3, N = 2^20, whose two segments per head need ~13 MB
    for cfg in (L.make_config(64, 1 << 20, 8, 128, 3, 4, 1024),
                L.make_config(16, 1 << 20, 8, 128, 3, 4, 1024, select_mode=1)):
        with pytest.raises(L.LighthouseError) as e:
            L.lh_score_topk_noalloc(cfg, x, x, i, i)
        assert e.value.code == 3  # LH_ERR_WORKSPACE, raised before any launch
