"""The C ABI library loads, exports every symbol the header declares, and its
host-side size and config logic agrees with the oracle's formulas (no GPU
needed: none of these calls launches a kernel)."""
import os
import re
import subprocess

import pytest

from oracle import lighthouse_oracle as lo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lighthouse.h")


@pytest.fixture(scope="module")
def L():
    from hierarchical_selection_attention_b200 import build
    build.build()
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lh_[a-z0-9_]+)\s*\(", text)))


def test_header_and_library_exports_agree(L):
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (lh_[a-z0-9_]+)", out))
    decl = declared_symbols()
    assert decl, "no declarations parsed"
    missing = [s for s in decl if s not in exported]
    assert not missing, missing
    assert set(L.EXPORTED) == set(decl)


@pytest.mark.parametrize("B,N,H,d,Lv,p,k", [(1, 4096, 2, 64, 3, 4, 64), (1, 65536, 8, 128, 3, 4, 1024),
                                            (2, 131072, 8, 128, 3, 4, 2048),
                                            (1, 524288, 8, 128, 3, 4, 4096),
                                            (1, 1048576, 8, 128, 4, 4, 4096),
                                            (3, 2048, 3, 128, 3, 4, 40), (1, 640, 2, 128, 1, 4, 0),
                                            (1, 729, 1, 64, 4, 3, 5)])
def test_sizes_match_oracle(L, B, N, H, d, Lv, p, k):
    cfg = L.make_config(B, N, H, d, Lv, p, k)
    assert L.lh_config_check(cfg) == 0
    assert L.lh_subseq_len(cfg) == lo.subseq_len(N, Lv, p, k)
    assert L.lh_total_entries(cfg) == lo.total_entries(N, Lv, p)
    assert L.lh_pooled_rows(cfg) == lo.total_entries(N, Lv, p) - N
    fwd, bwd, saved = L.lh_workspace_bytes(cfg)
    S, P = lo.subseq_len(N, Lv, p, k), lo.total_entries(N, Lv, p)
    assert saved >= B * H * (S * 4 + P * 4 + 5 * S * d * 2 + S * 4)
    offs = L.lh_saved_offsets(cfg)
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert bwd >= B * H * S * (4 * d * 2 + 4)
    assert fwd >= 2 * B * H * P * 4 + 3 * B * (P - N) * H * d * 2


@pytest.mark.parametrize("args,code", [
    ((1, 100, 2, 64, 3, 4, 1), 1),      # 16 does not divide 100
    ((1, 64, 2, 64, 3, 4, 100), 1),     # budget larger than the candidates
    ((1, 64, 2, 96, 3, 4, 1), 2),       # head dim not built
    ((1, 64, 2, 64, 3, 1, 1), 1),       # p < 2
    ((0, 64, 2, 64, 3, 4, 1), 1),       # empty batch
    ((1, 4096, 2, 64, 7, 2, 1), 2),     # more levels than built
])
def test_config_rejections(L, args, code):
    assert L.lh_config_check(L.make_config(*args)) == code
    assert L.lh_subseq_len(L.make_config(*args)) == -1


def test_launch_counts(L):
    cfg = L.make_config(1, 4096, 2, 64, 3, 4, 64)
    assert L.lh_forward_launches(cfg) > 5
    assert L.lh_backward_launches(cfg) >= 3
    assert L.lh_forward_launches(L.make_config(1, 100, 2, 64, 3, 4, 1)) == -1


@pytest.mark.parametrize("mode,N,L_,p,k,chunk,code", [
    (1, 4096, 3, 4, 64, 0, 0),     # per-level quota: p k = 256 <= N / p = 1024
    (1, 64, 3, 4, 4, 0, 0),        # p k = 16 == the coarsest finer level
    (1, 64, 3, 4, 5, 0, 1),        # p k = 20 > 16 (the joint mode accepts it)
    (0, 64, 3, 4, 5, 0, 0),
    (2, 4096, 3, 4, 64, 64, 0),    # stratified: 512 / 64 = 8 chunks
    (2, 4096, 3, 4, 64, 512, 0),   # one chunk (the joint selection)
    (2, 4096, 3, 4, 64, 0, 1),     # no chunk quota
    (2, 4096, 3, 4, 64, 48, 1),    # 48 does not divide 512
    (2, 4096, 3, 4, 0, 0, 0),      # nothing to select: no chunks needed
    (3, 4096, 3, 4, 64, 0, 2),     # no such mode
    (1, 640, 1, 4, 0, 0, 0),       # one level: nothing to select in any mode
])
def test_select_mode_config(L, mode, N, L_, p, k, chunk, code):
    cfg = L.make_config(1, N, 2, 64, L_, p, k, select_mode=mode, select_chunk=chunk)
    assert L.lh_config_check(cfg) == code
    if code == 0:
        # S does not depend on the selection mode
        assert L.lh_subseq_len(cfg) == lo.subseq_len(N, L_, p, k)
        lo.check_config(N, L_, p, k, mode, chunk)   # the oracle accepts it too
    elif code == 1:
        with pytest.raises(ValueError):
            lo.check_config(N, L_, p, k, mode, chunk)


def test_quota_mode_needs_a_larger_selection_workspace(L):
    # one radix-selection state per finer level instead of one per head
    f0, _, _ = L.lh_workspace_bytes(L.make_config(1, 4096, 2, 64, 3, 4, 64))
    f1, _, _ = L.lh_workspace_bytes(L.make_config(1, 4096, 2, 64, 3, 4, 64, select_mode=1))
    assert f1 > f0


def test_stratified_mode_needs_no_histograms(L):
    # a chunk keeps only its threshold state: no per-pass global histograms
    f0, _, _ = L.lh_workspace_bytes(L.make_config(1, 4096, 2, 64, 3, 4, 64))
    f2, _, _ = L.lh_workspace_bytes(L.make_config(1, 4096, 2, 64, 3, 4, 64, select_mode=2,
                                                  select_chunk=64))
    assert f2 < f0
    assert L.lh_forward_launches(L.make_config(1, 4096, 2, 64, 3, 4, 64, select_mode=2,
                                               select_chunk=64)) == \
        L.lh_forward_launches(L.make_config(1, 4096, 2, 64, 3, 4, 64)) - 11


def test_gemm_argument_checks(L):
    """lh_gemm rejects bad shapes and layouts before any launch (no GPU needed)."""
    import ctypes
    op = L.lh_gemm_operand
    P = ctypes.c_void_p

    def call(M, N, ops, c=0x1000, ldc=None, a_mn=0, b_mn=0, splits=1, ws=None, nb=0):
        arr = (op * max(1, len(ops)))(*ops)
        return L._lib.lh_gemm(M, N, len(ops), arr, a_mn, b_mn, P(c), N if ldc is None else ldc,
                              splits, P(ws), nb, P(0))

    ok_op = op(0x2000, 0x3000, 64, 64, 64)
    assert call(128, 256, []) == 1                                   # no pairs
    assert call(128, 250, [ok_op]) == 1                              # N not a multiple of 8
    assert call(128, 256, [op(0x2000, 0x3000, 60, 64, 64)]) == 1     # K not a multiple of 8
    assert call(128, 256, [op(0x2008, 0x3000, 64, 64, 64)]) == 1     # misaligned A
    assert call(128, 256, [op(0x2000, 0x3000, 64, 32, 64)]) == 1     # lda < K (K-major A)
    assert call(128, 256, [op(0x2000, 0x3000, 64, 64, 64)], a_mn=1) == 1   # lda < M (MN-major A)
    assert call(128, 256, [ok_op], ldc=200) == 1                     # ldc < N
    assert call(128, 256, [ok_op] * 4) == 1                          # more than three pairs
    assert call(128, 256, [ok_op], a_mn=2) == 1                      # unknown layout
    big = op(0x2000, 0x3000, 8192, 8192, 8192)
    assert call(128, 256, [big], splits=4) == 3                      # split K without a workspace
    assert L.lh_gemm_ws_bytes(128, 256, 4) == 4 * 128 * 256 * 4
    assert L.lh_gemm_ws_bytes(128, 256, 1) == 0


def test_gemm_binding_checks_operand_shapes(L):
    """The binding refuses operands whose extents differ from (M or N) x k, so
    the kernel never reads past an allocation (CPU tensors fail the device
    check first, the shape rule is the same)."""
    import torch
    c = torch.empty(128, 256, dtype=torch.bfloat16)
    a = torch.empty(128, 64, dtype=torch.bfloat16)
    b = torch.empty(256, 64, dtype=torch.bfloat16)
    with pytest.raises(L.LighthouseError):
        L.lh_gemm(c, [(a, b, 64)])      # host tensors are refused before any call


def test_grid_limits_rejected_before_launch(L):
    """(b, h) pairs (times the L-1 segments of the per-level quota) index the
    y dimension of the selection grids, which stops at 65535: such configs
    are refused up front (LH_ERR_UNSUPPORTED), not left to fail at launch."""
    assert L.lh_config_check(L.make_config(1, 4096, 65535, 64, 3, 4, 64)) == 0
    assert L.lh_config_check(L.make_config(2, 4096, 40000, 64, 3, 4, 64)) == 2
    assert L.lh_config_check(L.make_config(1, 4096, 40000, 64, 3, 4, 64, select_mode=1)) == 2
    assert L.lh_config_check(L.make_config(1, 4096, 30000, 64, 3, 4, 64, select_mode=1)) == 0


def test_bwd_ws_offsets_fit_the_scratch(L):
    cfg = L.make_config(2, 2048, 3, 128, 3, 4, 40)
    _, bwd, _ = L.lh_workspace_bytes(cfg)
    offs = L.lh_bwd_ws_offsets(cfg)
    S, d, BH = L.lh_subseq_len(cfg), 128, 6
    sizes = [BH * S * 4] + [BH * S * d * 2] * 4
    assert all(o % 256 == 0 for o in offs)
    spans = sorted(zip(offs, sizes))
    for (a, n), (b, _) in zip(spans, spans[1:]):
        assert a + n <= b
    assert spans[-1][0] + spans[-1][1] <= bwd
