"""The plain GEMM (lh_gemm) on the GPU against fp64 products of the same bf16
inputs: every operand layout, one to three summed pairs, split K, ragged
tiles.  Tolerance: the bf16 rounding of the output plus fp32 accumulation,
max-abs scaled by the envelope sum |a||b| (see tests/parity.py)."""
import numpy as np
import pytest
import torch

from tests.parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def _operand(rows, k, mn, gen):
    # logical [rows, k]; stored K-major ([rows, k]) or MN-major ([k, rows])
    x = torch.randn(rows, k, generator=gen).to(torch.bfloat16)
    stored = x.t().contiguous() if mn else x.contiguous()
    return x.double().numpy(), stored.cuda()


@pytest.mark.parametrize("M,N,ks,a_mn,b_mn,splits", [
    (256, 256, (128,), 0, 0, 1),
    (300, 264, (136,), 0, 0, 1),          # ragged in M, N and K
    (200, 520, (64, 72, 200), 0, 1, 1),   # three summed pairs, B MN-major
    (136, 256, (1024,), 1, 1, 4),         # long K split over CTAs
    (384, 136, (96,), 1, 0, 1),
    (1024, 512, (512, 512), 0, 1, 3),
])
def test_gemm_matches_fp64(L, M, N, ks, a_mn, b_mn, splits):
    gen = torch.Generator().manual_seed(M * 7 + N + len(ks))
    ref = np.zeros((M, N))
    env = np.zeros((M, N))
    pairs, keep = [], []
    for k in ks:
        a64, a = _operand(M, k, a_mn, gen)
        b64, b = _operand(N, k, b_mn, gen)
        ref += a64 @ b64.T
        env += np.abs(a64) @ np.abs(b64).T
        pairs.append((a, b, k))
        keep += [a, b]
    c = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(1, L.lh_gemm_ws_bytes(M, N, splits)), dtype=torch.uint8, device="cuda")
    L.lh_gemm(c, pairs, a_mn=a_mn, b_mn=b_mn, splits=splits, ws=ws)
    torch.cuda.synchronize()
    L.check_device_status()
    assert_close(c.double().cpu().numpy(), ref, "gemm", env=env)
    # deterministic: the same bits again (split K sums the partials in order)
    c2 = torch.empty_like(c)
    L.lh_gemm(c2, pairs, a_mn=a_mn, b_mn=b_mn, splits=splits, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(c, c2)


def test_gemm_writes_into_a_row_slice(L):
    # C may be a column block of a wider matrix (its own leading dimension)
    gen = torch.Generator().manual_seed(5)
    a64, a = _operand(128, 64, 0, gen)
    b64, b = _operand(256, 64, 0, gen)
    big = torch.zeros(128, 512, dtype=torch.bfloat16, device="cuda")
    L.lh_gemm(big[:, 128:384], [(a, b, 64)])
    torch.cuda.synchronize()
    got = big.double().cpu().numpy()
    assert np.all(got[:, :128] == 0) and np.all(got[:, 384:] == 0)
    assert_close(got[:, 128:384], a64 @ b64.T, "gemm slice", env=np.abs(a64) @ np.abs(b64).T)
