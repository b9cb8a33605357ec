"""The head split on one GPU: the layer run rank by rank on each rank's head
range (heads.HeadShardedLayer, no collective) gives exactly the whole
layer's output and gradients, bit for bit (Sec. 3.4: everything after the
per-head scores runs per head)."""
import pytest
import torch

from hierarchical_selection_attention_b200.inputs import make_dout, make_qkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R", [2, 3])
def test_head_slices_assemble_to_the_whole_layer(R):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_selection_attention_b200 import heads, lighthouse as L
    B, N, H, d, Lv, p, k = 2, 8192, 8, 128, 3, 4, 64
    q, kk, v = (t.cuda() for t in make_qkv(B, N, H, d, seed=11))
    dout = make_dout(B, N, H, d, seed=11).cuda()
    whole = L.LighthouseLayer(B, N, H, d, Lv, p, k)
    o = whole.forward(q, kk, v)
    g = whole.backward(dout)
    for r in range(R):
        part = heads.HeadShardedLayer(B, N, H, d, Lv, p, k, R, r)
        h0, h1 = part.h0, part.h1
        assert torch.equal(part.forward(q, kk, v), o[:, :, h0:h1])
        for a, b in zip(part.backward(dout), g):
            assert torch.equal(a, b[:, :, h0:h1])
    torch.cuda.synchronize()
    L.check_device_status()
