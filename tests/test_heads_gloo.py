"""One layer's heads split over ranks (heads.HeadShardedLayer), on 2 and 3
gloo ranks on the host.  Each rank runs the layer on its own head range and
one all-gather assembles the output and the gradients; the result must be
the single-rank layer's, bit for bit.  The per-rank layer here is the
oracle (fp64, per head), since the host has no GPU: what is checked is the
partition and the gather (Sec. 3.4: selection and everything after it run
per head, so a head split changes no value)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_selection_attention_b200 import heads
from oracle import lighthouse_oracle as lo

B, N, H, d, L, p, k = 2, 256, 5, 8, 3, 2, 6


def _inputs():
    rng = np.random.default_rng(5)
    return [torch.from_numpy(rng.standard_normal((B, N, H, d))) for _ in range(4)]


class OracleLayer:
    """forward / backward of the layer on [B, N, h, d] fp64 tensors."""

    def __init__(self, Hr):
        self.states = None

    def forward(self, q, kk, v):
        o, self.states = lo.forward(q.numpy(), kk.numpy(), v.numpy(), L, p, k, parity=False)
        return torch.from_numpy(o)

    def backward(self, dout):
        return tuple(torch.from_numpy(g) for g in lo.backward(self.states, dout.numpy()))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, R, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        q, kk, v, g = _inputs()
        lay = heads.HeadShardedLayer(B, N, H, d, L, p, k, R, rank, make_layer=OracleLayer)
        o = lay.forward(q, kk, v, gather=True)
        grads = lay.backward(g, gather=True)
        local = lay.forward(q, kk, v)                  # the rank's own slice, no collective
        out.put((rank, o.numpy(), [x.numpy() for x in grads], local.numpy(), (lay.h0, lay.h1)))
    finally:
        dist.destroy_process_group()


def test_head_ranges_cover_every_head_once():
    for Hh, R in ((8, 8), (8, 3), (5, 2), (16, 4)):
        got = [heads.head_range(Hh, R, r) for r in range(R)]
        assert got[0][0] == 0 and got[-1][1] == Hh
        assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
        assert max(b - a for a, b in got) - min(b - a for a, b in got) <= 1
    with pytest.raises(ValueError):
        heads.head_range(2, 3, 0)


@pytest.mark.parametrize("R", [2, 3])
def test_head_split_over_gloo_ranks_is_the_single_rank_layer(R):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, R, port, out)) for r in range(R)]
    for pr in procs:
        pr.start()
    got = [out.get(timeout=180) for _ in range(R)]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    q, kk, v, g = _inputs()
    ref = OracleLayer(H)
    o_ref = ref.forward(q, kk, v).numpy()
    g_ref = [x.numpy() for x in ref.backward(g)]
    for rank, o, grads, local, (h0, h1) in got:
        np.testing.assert_array_equal(o, o_ref)
        for a, b in zip(grads, g_ref):
            np.testing.assert_array_equal(a, b)
        np.testing.assert_array_equal(local, o_ref[:, :, h0:h1])
