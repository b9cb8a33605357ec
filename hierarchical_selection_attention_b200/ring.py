"""Context parallelism for the Lighthouse layer: the sequence cut into R
contiguous shards, one per rank.

"Long Context Pre-Training with Lighthouse Attention", single-B200 latency
benchmark paragraph (multi-GPU training note, App. D.4 cited): pyramid
pooling, scoring and top-k run shard-locally, and the gathered sub-sequence
rotates through ring attention, with no sparsity-aware collective.  Shard r
runs stages (i)-(iii) on its own N/R tokens with the layer's p and k, so its
sub-sequence has S rows.  Every entry of shard r' < r ends before any entry
of shard r, so over the sub-sequences concatenated in shard order the plain
causal mask applies: shard r's rows see every earlier shard's whole block and
their own block causally.  Each shard scatters its own rows.

This module holds the ring's schedule and its drivers:

* forward_steps / dq_steps / dkdv_steps(R, rank): which K/V block a rank
  works on at which step, in which mode, and whether the step opens or
  closes a sum.  The K/V block of shard src starts at rank src and moves one
  rank on (r -> r + 1 mod R) after every step, so at step s rank r holds
  block (r - s) mod R.
    forward and dQ: steps 0..r; step 0 is the rank's own block (causal,
      opens the sum), step r is block 0 (closes it).
    dK, dV of a block: they travel with it, as fp32 sums; rank r adds its
      share of block src = r - s at steps 1..r (every key visible; the first
      rank after the owner opens the sum), and after R moves the block is
      home, where the owner adds its own causal share last and writes the
      bf16 result ("home step" R).
* ring_forward / ring_backward: one rank's part, over a transport that
  moves blocks to the next rank (torch.distributed point-to-point: NCCL on
  GPUs, gloo on the host), with the step arithmetic passed in as callables.
* LighthouseRingLayer: all R shards in one process on one GPU, the K/V
  blocks read where they lie (the transport is the identity), the step
  arithmetic in the library's ring-step kernels (lh_attn_*_block).

A block that arrives from another rank always lands in a local buffer before
any kernel reads it; no kernel reads another GPU's memory.
"""
from __future__ import annotations

from dataclasses import dataclass

DIAG, FULL = 0, 1          # LH_BLOCK_DIAG, LH_BLOCK_FULL


@dataclass(frozen=True)
class Step:
    step: int      # 0 .. R (R: the home step of the dK/dV sums)
    rank: int      # the query shard, i.e. the rank that computes
    src: int       # the shard whose K/V block it computes against
    mode: int      # DIAG (own block, causal) or FULL (an earlier block)
    first: bool    # opens the sum it adds to
    last: bool     # closes it (writes the bf16 result)


def _check(R: int, rank: int) -> None:
    if R < 1 or not 0 <= rank < R:
        raise ValueError(f"rank {rank} of a ring of {R}")


def block_at(R: int, rank: int, step: int) -> int:
    """The K/V block rank `rank` holds at step `step`."""
    return (rank - step) % R


def forward_steps(R: int, rank: int) -> list[Step]:
    """Forward (and dQ) steps of one rank: its own block first (causal), then
    each earlier shard's block as it arrives, ending with block 0."""
    _check(R, rank)
    return [Step(s, rank, rank - s, DIAG if s == 0 else FULL, s == 0, s == rank)
            for s in range(rank + 1)]


def dq_steps(R: int, rank: int) -> list[Step]:
    return forward_steps(R, rank)


def dkdv_steps(R: int, rank: int) -> list[Step]:
    """dK/dV steps computed by one rank: its share of each earlier block at
    steps 1..rank (the block's sum opens at the rank right after its owner),
    then, at the home step R, its own block, causal, closing that block's
    sum (and opening it too if no later rank exists)."""
    _check(R, rank)
    out = [Step(s, rank, rank - s, FULL, s == 1, False) for s in range(1, rank + 1)]
    out.append(Step(R, rank, rank, DIAG, rank == R - 1, True))
    return out


def schedule(R: int) -> dict[str, list[Step]]:
    """Every step of every rank, ordered by step and then rank."""
    key = lambda st: (st.step, st.rank)
    return {"forward": sorted((st for r in range(R) for st in forward_steps(R, r)), key=key),
            "dq": sorted((st for r in range(R) for st in dq_steps(R, r)), key=key),
            "dkdv": sorted((st for r in range(R) for st in dkdv_steps(R, r)), key=key)}


# ------------------------------------------------------------ transports --

class P2PTransport:
    """Moves tensors one rank on around the ring with torch.distributed
    point-to-point operations: send to rank + 1, receive from rank - 1 into
    the caller's (local) buffers.  Works with NCCL on GPUs and gloo on the
    host."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.R = dist.get_world_size(group)

    def start(self, send: list, recv: list):
        d = self.dist
        nxt, prv = (self.rank + 1) % self.R, (self.rank - 1) % self.R
        nxt_g = d.get_global_rank(self.group, nxt) if self.group is not None else nxt
        prv_g = d.get_global_rank(self.group, prv) if self.group is not None else prv
        ops = [d.P2POp(d.isend, t, nxt_g, self.group) for t in send]
        ops += [d.P2POp(d.irecv, t, prv_g, self.group) for t in recv]
        return d.batch_isend_irecv(ops)

    @staticmethod
    def wait(reqs):
        for r in reqs:
            r.wait()


def ring_forward(R: int, rank: int, kv: list, fwd_step, transport, new_like):
    """One rank's forward ring.  kv: its own K/V block tensors; fwd_step(step,
    kv_block) runs the step's arithmetic into this rank's accumulators;
    new_like(kv) makes receive buffers.  The next block's transfer runs while
    the current one is being computed on (blocks are read-only here)."""
    steps = {st.step: st for st in forward_steps(R, rank)}
    cur = kv
    for s in range(R):
        reqs, nxt = None, None
        if s < R - 1:                        # blocks still needed further on
            nxt = new_like(cur)
            reqs = transport.start(cur, nxt)
        if s in steps:
            fwd_step(steps[s], cur)
        if reqs is not None:
            transport.wait(reqs)
            cur = nxt


def ring_backward(R: int, rank: int, kv: list, dkv_acc: list, dq_step, dkdv_step, transport,
                  new_like):
    """One rank's backward ring.  The payload that moves is the K/V block
    with its fp32 dK/dV sums; dq_step(step, kv) adds to this rank's dQ,
    dkdv_step(step, kv, acc) to the travelling sums (or, at the home step,
    closes this rank's own block).  Returns the payload after it has come
    home."""
    dq = {st.step: st for st in dq_steps(R, rank)}
    dkdv = {st.step: st for st in dkdv_steps(R, rank)}
    kv, acc = list(kv), list(dkv_acc)
    for s in range(R):
        if s in dq:
            dq_step(dq[s], kv)
        if s in dkdv:
            dkdv_step(dkdv[s], kv, acc)
        if R == 1:                           # a ring of one: the block never leaves
            continue
        payload = kv + acc
        nxt = new_like(payload)
        transport.wait(transport.start(payload, nxt))   # the sums are final for this hop
        kv, acc = nxt[:len(kv)], nxt[len(kv):]
    dkdv_step(dkdv[R], kv, acc)               # home: own block, closing the sums
    return kv, acc


# ------------------------------------------------- one process, one GPU --

class LighthouseRingLayer:
    """The context-parallel layer with its R shards in one process: shard r
    holds tokens r N/R .. (r+1) N/R - 1 and runs stages (i)-(iii) and (iv) on
    them with its own buffers (a LighthouseLayer of N/R tokens), and the
    ring attention runs over the shards' gathered sub-sequences in the order
    the ring schedule gives, reading each K/V block where it lies.

    forward(q, k, v) -> o and backward(dout) -> (dq, dk, dv) on [B, N, H, d]
    bf16 tensors (torch's current stream).  A shard of a B = 1 tensor is a
    contiguous view; for B > 1 it is copied out and back."""

    def __init__(self, B, N, H, d, L, p, k, R, scale: float = 0.0, device="cuda",
                 select_mode: int = 0, select_chunk: int = 0, scatter_mode: int = 0):
        import torch
        from hierarchical_selection_attention_b200 import lighthouse as lh
        if R < 1 or N % R:
            raise ValueError("the shard count must divide N")
        self.lh, self.torch = lh, torch
        self.B, self.N, self.H, self.d, self.R, self.Ns = B, N, H, d, R, N // R
        self.shards = [lh.LighthouseLayer(B, self.Ns, H, d, L, p, k, scale, device=device,
                                          select_mode=select_mode, select_chunk=select_chunk,
                                          scatter_mode=scatter_mode)
                       for _ in range(R)]
        self.cfg = self.shards[0].cfg
        self.S = self.shards[0].S
        dev = self.shards[0].device
        f32 = lambda *s: torch.empty(*s, dtype=torch.float32, device=dev)
        shape = (B, H, self.S, d)
        self.o_acc = [f32(*shape) for _ in range(R)]
        self.lse2_acc = [f32(B, H, self.S) for _ in range(R)]
        self.dq_acc = [f32(*shape) for _ in range(R)]
        self.dk_acc = [f32(*shape) for _ in range(R)]
        self.dv_acc = [f32(*shape) for _ in range(R)]

    def _tok(self, x, r):
        sl = x[:, r * self.Ns:(r + 1) * self.Ns]
        return sl if sl.is_contiguous() else sl.contiguous()

    def forward(self, q, k, v, out=None):
        lh, R = self.lh, self.R
        o = self.torch.empty_like(q) if out is None else out
        for r, sh in enumerate(self.shards):
            lh.lh_forward_gather(self.cfg, self._tok(q, r), self._tok(k, r), self._tok(v, r),
                                 sh.saved, sh.ws_fwd)
        views = [sh.views() for sh in self.shards]
        for st in schedule(R)["forward"]:
            a, b = views[st.rank], views[st.src]
            lh.lh_attn_fwd_block(self.cfg, st.mode, st.first, st.last, a["qg"], b["kg"], b["vg"],
                                 self.o_acc[st.rank], self.lse2_acc[st.rank], a["og"], a["lse"],
                                 og_lo=a["og_lo"])
        for r, sh in enumerate(self.shards):
            sl = o[:, r * self.Ns:(r + 1) * self.Ns]
            dst = sl if sl.is_contiguous() else self.torch.empty_like(sl.contiguous())
            lh.lh_forward_scatter(self.cfg, sh.saved, dst, sh.ws_fwd)
            if dst is not sl:
                sl.copy_(dst)
        return o

    def backward(self, dout, grads=None):
        lh, R = self.lh, self.R
        if grads is None:
            grads = tuple(self.torch.empty_like(dout) for _ in range(3))
        for r, sh in enumerate(self.shards):
            lh.lh_backward_scatter(self.cfg, sh.saved, self._tok(dout, r), sh.ws_bwd)
        views = [sh.views() for sh in self.shards]
        bviews = [sh.bwd_views() for sh in self.shards]
        sched = schedule(R)
        steps = sorted([("dq", st) for st in sched["dq"]] + [("dkdv", st) for st in sched["dkdv"]],
                       key=lambda x: (x[1].step, x[1].rank, x[0]))
        for kind, st in steps:
            a, b = views[st.rank], views[st.src]
            ga = bviews[st.rank]
            if kind == "dq":
                lh.lh_attn_bwd_dq_block(self.cfg, st.mode, st.first, st.last, a["qg"], b["kg"],
                                        b["vg"], ga["dog"], a["lse"], ga["delta"],
                                        self.dq_acc[st.rank], ga["dqg"])
            else:
                gb = bviews[st.src]
                lh.lh_attn_bwd_dkdv_block(self.cfg, st.mode, st.first, st.last, a["qg"], b["kg"],
                                          b["vg"], ga["dog"], a["lse"], ga["delta"],
                                          self.dk_acc[st.src], self.dv_acc[st.src], gb["dkg"],
                                          gb["dvg"])
        for r, sh in enumerate(self.shards):
            outs = []
            for g in grads:
                sl = g[:, r * self.Ns:(r + 1) * self.Ns]
                outs.append(sl if sl.is_contiguous() else self.torch.empty_like(sl.contiguous()))
            lh.lh_backward_gather(self.cfg, sh.saved, sh.ws_bwd, *outs)
            for g, t in zip(grads, outs):
                sl = g[:, r * self.Ns:(r + 1) * self.Ns]
                if t is not sl:
                    sl.copy_(t)
        return grads


# ------------------------------------------------ one rank of a real ring --

class LighthouseRingRank:
    """One rank's part of the context-parallel layer across R processes (one
    GPU each): this rank holds shard `rank` of the sequence ([B, N/R, H, d]
    tensors), runs stages (i)-(iii) and (iv) on it, and the ring attention
    with the other ranks through `transport` (P2PTransport over the default
    process group by default: NCCL point-to-point into local receive
    buffers).  The step arithmetic is the library's ring-step kernels; the
    schedule and the drivers are the ones above.

    Every rank must call forward and backward in the same order (each one is
    a sequence of point-to-point exchanges with both neighbours)."""

    def __init__(self, B, N_shard, H, d, L, p, k, R, rank, scale: float = 0.0, device="cuda",
                 transport=None, select_mode: int = 0, select_chunk: int = 0):
        import torch
        from hierarchical_selection_attention_b200 import lighthouse as lh
        self.lh, self.torch, self.R, self.rank = lh, torch, R, rank
        self.layer = lh.LighthouseLayer(B, N_shard, H, d, L, p, k, scale, device=device,
                                        select_mode=select_mode, select_chunk=select_chunk)
        self.cfg, self.S = self.layer.cfg, self.layer.S
        dev = self.layer.device
        shape = (B, H, self.S, d)
        self.o_acc = torch.empty(*shape, dtype=torch.float32, device=dev)
        self.lse2_acc = torch.empty(B, H, self.S, dtype=torch.float32, device=dev)
        self.dq_acc = torch.empty(*shape, dtype=torch.float32, device=dev)
        self.transport = transport

    def _tp(self):
        if self.transport is None:
            self.transport = P2PTransport()
        return self.transport

    @staticmethod
    def _new_like(ts):
        return [t.new_empty(t.shape) for t in ts]

    def forward(self, q, k, v, out=None):
        lh = self.lh
        o = self.torch.empty_like(q) if out is None else out
        lay = self.layer
        lh.lh_forward_gather(self.cfg, q, k, v, lay.saved, lay.ws_fwd)
        a = lay.views()

        def step(st, kv):
            lh.lh_attn_fwd_block(self.cfg, st.mode, st.first, st.last, a["qg"], kv[0], kv[1],
                                 self.o_acc, self.lse2_acc, a["og"], a["lse"], og_lo=a["og_lo"])

        # the stream orders the kernels against the exchanges NCCL enqueues on it
        ring_forward(self.R, self.rank, [a["kg"], a["vg"]], step, self._tp(), self._new_like)
        lh.lh_forward_scatter(self.cfg, lay.saved, o, lay.ws_fwd)
        return o

    def backward(self, dout, grads=None):
        lh, torch = self.lh, self.torch
        lay = self.layer
        if grads is None:
            grads = tuple(torch.empty_like(dout) for _ in range(3))
        lh.lh_backward_scatter(self.cfg, lay.saved, dout, lay.ws_bwd)
        a, g = lay.views(), lay.bwd_views()
        acc = [torch.empty_like(self.dq_acc), torch.empty_like(self.dq_acc)]

        def dq_step(st, kv):
            lh.lh_attn_bwd_dq_block(self.cfg, st.mode, st.first, st.last, a["qg"], kv[0], kv[1],
                                    g["dog"], a["lse"], g["delta"], self.dq_acc, g["dqg"])

        def dkdv_step(st, kv, acc_):
            lh.lh_attn_bwd_dkdv_block(self.cfg, st.mode, st.first, st.last, a["qg"], kv[0], kv[1],
                                      g["dog"], a["lse"], g["delta"], acc_[0], acc_[1], g["dkg"],
                                      g["dvg"])

        ring_backward(self.R, self.rank, [a["kg"], a["vg"]], acc, dq_step, dkdv_step, self._tp(),
                      self._new_like)
        lh.lh_backward_gather(self.cfg, lay.saved, lay.ws_bwd, *grads)
        return grads
