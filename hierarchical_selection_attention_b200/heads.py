"""One layer's heads split across ranks (one GPU each).

"Long Context Pre-Training with Lighthouse Attention", Sec. 3.4: scores are
per-head l2 norms and the selection runs per head, so every (b, h) pair goes
through all stages on its own and a layer partitions over heads with no
exchange during the layer.  Rank `rank` of R takes the contiguous head range
head_range(H, R, rank) and runs the whole layer (lh_forward / lh_backward)
on it; only a caller who wants the full [B, N, H, d] output on every rank
needs a collective: one all-gather of the head slices.
"""
from __future__ import annotations


def head_range(H: int, R: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank`: H split into R contiguous, near-equal ranges
    (the first H mod R ranks take one more)."""
    if R < 1 or not 0 <= rank < R or H < R:
        raise ValueError(f"cannot split {H} heads over rank {rank} of {R}")
    base, extra = divmod(H, R)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


class HeadShardedLayer:
    """The Lighthouse layer on this rank's heads of a [B, N, H, d] problem.

    forward(q, k, v) takes either the full tensors (the rank's heads are
    sliced out and made contiguous) or the rank's own [B, N, H_r, d] slice,
    and returns the rank's output slice, or with gather=True the full
    output assembled by one all-gather over `group`.  backward(dout) does the
    same for the three gradients.

    `make_layer(H_r)` builds the per-rank layer (default: a LighthouseLayer
    of H_r heads on `device`); anything with forward(q, k, v) -> o and
    backward(dout) -> (dq, dk, dv) on [B, N, H_r, d] tensors works."""

    def __init__(self, B, N, H, d, L, p, k, R, rank, device="cuda", group=None, make_layer=None,
                 **layer_kw):
        self.B, self.N, self.H, self.d, self.R, self.rank = B, N, H, d, R, rank
        self.h0, self.h1 = head_range(H, R, rank)
        self.group = group
        if make_layer is None:
            from hierarchical_selection_attention_b200 import lighthouse as lh
            make_layer = lambda Hr: lh.LighthouseLayer(B, N, Hr, d, L, p, k, device=device,
                                                       **layer_kw)
        self.layer = make_layer(self.h1 - self.h0)

    def _mine(self, x):
        if x.shape[2] == self.h1 - self.h0 and x.shape[2] != self.H:
            return x if x.is_contiguous() else x.contiguous()
        return x[:, :, self.h0:self.h1].contiguous()

    def _gather(self, x):
        """All ranks' head slices into [B, N, H, d], in head order.  Slices
        of unequal size are padded to the largest for the collective."""
        import torch
        import torch.distributed as dist
        width = max(b - a for a, b in (head_range(self.H, self.R, r) for r in range(self.R)))
        pad = x.new_zeros(x.shape[0], x.shape[1], width, x.shape[3])
        pad[:, :, :x.shape[2]] = x
        parts = [torch.empty_like(pad) for _ in range(self.R)]
        dist.all_gather(parts, pad.contiguous(), group=self.group)
        out = x.new_empty(x.shape[0], x.shape[1], self.H, x.shape[3])
        for r, t in enumerate(parts):
            a, b = head_range(self.H, self.R, r)
            out[:, :, a:b] = t[:, :, :b - a]
        return out

    def forward(self, q, k, v, gather=False):
        o = self.layer.forward(self._mine(q), self._mine(k), self._mine(v))
        return self._gather(o) if gather else o

    def backward(self, dout, gather=False):
        grads = self.layer.backward(self._mine(dout))
        return tuple(self._gather(g) for g in grads) if gather else grads
