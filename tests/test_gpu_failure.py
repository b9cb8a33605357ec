"""Failure detection on the GPU, without a fault: a bounded wait that runs
out must come back to the host as LH_ERR_DEVICE_TIMEOUT through the device
status word, and the context must stay usable afterwards."""
import time

import pytest
import torch

from oracle import lighthouse_oracle as lo
from tests.parity import assert_close, f64, head
from hierarchical_selection_attention_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import lighthouse
    return lighthouse


def test_wait_that_runs_out_reports_timeout_and_the_context_survives(L):
    L.lh_get_device_status()                             # start from a cleared status word
    t0 = time.monotonic()
    L.lh_check_wait_timeout()                            # one warp, an mbarrier nothing completes
    code, detail = L.lh_get_device_status()              # synchronises, reads and clears
    waited = time.monotonic() - t0
    assert code == L.LH_ERR_DEVICE_TIMEOUT and detail == L.LH_WAIT_TIMEOUT_CHECK_DETAIL
    assert 0.2 < waited < 30.0, waited                   # ~4e9 SM cycles: bounded, not instant
    assert L.lh_get_device_status() == (L.LH_OK, 0)      # the read cleared it

    # the context is intact: a small layer still runs and matches the oracle
    B, N, H, d, Lv, p, k = 1, 1024, 1, 64, 3, 4, 8
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed=9))
    layer = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    o = layer.forward(q, kk, v)
    torch.cuda.synchronize()
    L.check_device_status()
    st = lo.forward_head(head(q, 0, 0), head(kk, 0, 0), head(v, 0, 0), Lv, p, k, parity=True)
    env = lo.scatter(lo.attention(st["qg"], st["kg"], abs(st["vg"]), st["scale"])[0],
                     st["slot_map"], N, Lv, p)
    assert_close(f64(o[0, :, 0, :]), st["o"], "o", env=env)
