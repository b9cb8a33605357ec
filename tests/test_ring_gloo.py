"""The context-parallel ring on real processes: 2-4 ranks over gloo
(127.0.0.1), each holding one shard's gathered Q, K, V, passing the K/V
blocks (and, backward, their dK/dV sums) to the next rank with the
library's transport and schedule (ring.ring_forward / ring.ring_backward).

The step arithmetic here is plain fp64 torch on the host, so what is
checked is the ring itself: blocks reach the right rank at the right step,
the log-sum-exp merges and the gradient sums open and close where they
should, and after the last hop the dK/dV sums are home.  The result must be
the oracle's attention over the shards' sub-sequences concatenated in shard
order (cp_forward_head; its gradients by attention_bwd)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_selection_attention_b200 import ring
from oracle import lighthouse_oracle as lo

# N, L, p, k, d, R: shard sub-sequences of 72 / 40 / 44 rows
CASES = [(384, 3, 2, 5, 8, 2), (384, 3, 2, 5, 8, 3), (512, 2, 4, 3, 16, 4)]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(N, d):
    rng = np.random.default_rng(N + d)
    q, k, v, g = (rng.standard_normal((N, d)) * 0.7 for _ in range(4))
    return q, k, v, g


def _rank_main(rank, R, case, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=R)
    try:
        N, L, p, k, d, _ = case
        q, kk, v, g = _inputs(N, d)
        st = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)
        Sr = lo.subseq_len(N // R, L, p, k)
        rows = slice(rank * Sr, (rank + 1) * Sr)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        Q, K, V = t(st["qg"][rows]), t(st["kg"][rows]), t(st["vg"][rows])
        scale = st["scale"]
        tri = torch.ones(Sr, Sr, dtype=torch.bool).tril()
        o_acc, lse_acc = torch.zeros(Sr, d, dtype=torch.float64), torch.zeros(Sr, dtype=torch.float64)

        def scores(step, kb):
            s = scale * Q @ kb.T
            return s.masked_fill(~tri, -math.inf) if step.mode == ring.DIAG else s

        def fwd_step(step, kv):
            s = scores(step, kv[0])
            m = s.max(dim=1).values
            e = torch.exp(s - m[:, None])
            lsum = e.sum(dim=1)
            o_b, l_b = (e @ kv[1]) / lsum[:, None], m + torch.log(lsum)
            if step.first:
                o_acc.copy_(o_b)
                lse_acc.copy_(l_b)
            else:
                new = torch.logaddexp(lse_acc, l_b)
                o_acc.copy_(o_acc * torch.exp(lse_acc - new)[:, None] + o_b * torch.exp(l_b - new)[:, None])
                lse_acc.copy_(new)

        tp = ring.P2PTransport()
        new_like = lambda ts: [torch.empty_like(x) for x in ts]
        ring.ring_forward(R, rank, [K, V], fwd_step, tp, new_like)

        # backward: the shard's scatter adjoint, D from its own final output
        Ns = N // R
        sh = st["shards"][rank]
        dog = t(lo.scatter_bwd(g[rank * Ns:(rank + 1) * Ns], sh["sel_idx"], Ns, L, p))
        D = (dog * o_acc).sum(dim=1)
        dq = torch.zeros(Sr, d, dtype=torch.float64)

        def p_ds(step, kv):
            P = torch.exp(scores(step, kv[0]) - lse_acc[:, None])
            return P, P * (dog @ kv[1].T - D[:, None])

        def dq_step(step, kv):
            _, dS = p_ds(step, kv)
            gq = scale * dS @ kv[0]
            dq.copy_(gq if step.first else dq + gq)

        def dkdv_step(step, kv, acc):
            P, dS = p_ds(step, kv)
            gk, gv = scale * dS.T @ Q, P.T @ dog
            acc[0].copy_(gk if step.first else acc[0] + gk)
            acc[1].copy_(gv if step.first else acc[1] + gv)

        acc0 = [torch.zeros(Sr, d, dtype=torch.float64) for _ in range(2)]
        kv_home, acc = ring.ring_backward(R, rank, [K, V], acc0, dq_step, dkdv_step, tp, new_like)
        out.put((rank, o_acc.numpy(), lse_acc.numpy(), dq.numpy(), acc[0].numpy(), acc[1].numpy(),
                 bool(torch.equal(kv_home[0], K) and torch.equal(kv_home[1], V))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES)
def test_ring_over_gloo_ranks_matches_the_concatenated_attention(case):
    N, L, p, k, d, R = case
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, R, case, port, out)) for r in range(R)]
    for pr in procs:
        pr.start()
    got = {}
    for _ in range(R):
        item = out.get(timeout=180)
        got[item[0]] = item[1:]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    q, kk, v, g = _inputs(N, d)
    st = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)
    dog = np.concatenate([lo.scatter_bwd(g[r * (N // R):(r + 1) * (N // R)], s["sel_idx"], N // R, L, p)
                          for r, s in enumerate(st["shards"])])
    dqg, dkg, dvg = lo.attention_bwd(st["qg"], st["kg"], st["vg"], dog, st["scale"])
    Sr = lo.subseq_len(N // R, L, p, k)
    for r in range(R):
        o, lse, dq, dk, dv, home = got[r]
        rows = slice(r * Sr, (r + 1) * Sr)
        assert home, "the K/V block did not come home unchanged"
        for name, x, y in (("og", o, st["og"][rows]), ("lse", lse, st["lse"][rows]),
                           ("dqg", dq, dqg[rows]), ("dkg", dk, dkg[rows]), ("dvg", dv, dvg[rows])):
            np.testing.assert_allclose(x, y, rtol=1e-10, atol=1e-10, err_msg=f"{name} rank {r}")
