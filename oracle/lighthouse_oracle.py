"""Plain, slow fp64 CPU oracle of the Lighthouse Attention layer's hot path.

TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
CPU-baseline leg of the benchmark may import this module.  The library's
product path never calls it, and this module imports nothing of the library.

Everything follows "Long Context Pre-Training with Lighthouse Attention"
(arXiv 2605.06554, HTML version), whose display equations were lost from the
text we have; each step below is rebuilt from the prose around them:

* Sec. 3.3, pyramid: window W_i^(l) = [i p^l, (i+1) p^l - 1]; entry (l, i) is
  the mean of Q, K and V over that window; p^(L-1) must divide N; the
  number of entries is sum_l N / p^l <= N p / (p - 1).
* Sec. 3.4, scoring and selection: the level-0 query and key scores are the
  per-head l2 norms of Q_t and K_t; a coarser entry's score is the maximum
  of the level-0 scores inside its window; one top-k runs jointly over the
  concatenated QK and KQ streams of every level but the coarsest, which is
  always kept whole.
* Sec. 3.5, Eq. 8 and 9: the selected triples form a sub-sequence of length
  S = N / p^(L-1) + (L-1) p k, sorted by pyramid coordinate so that a plain
  S x S causal mask applies; standard softmax attention runs over it.
* Sec. 3.6, scatter-back: the output of entry (l, i) goes to the window
  shifted right by p^l - 1 (it starts at the last token the entry
  summarises); contributions of different levels are summed.
* Sec. 3.2 and Sec. 3.4: the selection is discrete; gradients flow through
  the scatter, the attention and the gather (and the mean pooling) into Q,
  K and V, never through indices or scores.

Readings where the text is silent (each is listed with its reason in the
design notes of the repository):

* budget: exactly n_sel = (L-1) p k distinct entries from levels 0..L-2 are
  chosen jointly, plus all N / p^(L-1) entries of level L-1, so the length
  is exactly S;
* the joint top-k over the two streams takes distinct entries from the
  concatenated stream sorted by score (descending) until n_sel are found;
* ties: the lower flat pyramid index f(l, i) = sum_{l'<l} N/p^l' + i wins;
* the ranking key is the fp32 rounding of the fp64 norm;
* an entry's position for the causal mask is its last token e = (i+1)p^l - 1;
  entries ending on the same token are ordered child before parent
  (ascending level);
* softmax scale 1/sqrt(d); positions no entry reaches get 0;
* selection is per (batch, head);
* the stratified selection (mode 2) cuts the finer-level stream, in flat
  index order, into n_sel / m near-equal contiguous chunks and keeps the top
  m of each; the pages leave the chunk size to an appendix they do not
  include, so m is a parameter;
* context parallelism (cp_forward_head) cuts the sequence into R contiguous
  shards, runs the pyramid, scores and selection per shard with the layer's
  p and k, and attends over the shards' sub-sequences concatenated in shard
  order under the plain causal mask (what a ring over the shards computes).

``parity=True`` rounds values to bf16 where the library stores them (pooled
entries, the gathered output, its gradient and the gathered gradients) and
keeps every computation in fp64; ``parity=False`` never rounds and is what
the self-checks use.
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------
# Sizes (Sec. 3.3 and Eq. 8)
# --------------------------------------------------------------------------


def level_sizes(N: int, L: int, p: int) -> list[int]:
    """Entries per level: N / p^l for l = 0..L-1 (Sec. 3.3)."""
    return [N // p**lvl for lvl in range(L)]


def level_offsets(N: int, L: int, p: int) -> list[int]:
    """Flat index of entry (l, 0): sum_{l' < l} N / p^l'."""
    out, acc = [], 0
    for n in level_sizes(N, L, p):
        out.append(acc)
        acc += n
    return out


def total_entries(N: int, L: int, p: int) -> int:
    return sum(level_sizes(N, L, p))


def n_candidates(N: int, L: int, p: int) -> int:
    """Entries of levels 0..L-2, the ones that compete in the top-k."""
    return sum(level_sizes(N, L, p)[:-1])


def n_select(L: int, p: int, k: int) -> int:
    """Finer-level budget: each of the L-1 finer levels is charged p*k (Eq. 8)."""
    return (L - 1) * p * k


def subseq_len(N: int, L: int, p: int, k: int) -> int:
    """S = N / p^(L-1) + (L-1) p k (Eq. 8)."""
    return N // p ** (L - 1) + n_select(L, p, k)


def check_config(N: int, L: int, p: int, k: int, mode: int = 0, chunk: int = 0) -> None:
    if p < 2 or L < 1 or N < 1 or k < 0:
        raise ValueError("need p >= 2, L >= 1, N >= 1, k >= 0")
    if N % p ** (L - 1):
        raise ValueError("p^(L-1) must divide N (Sec. 3.3)")
    if n_select(L, p, k) > n_candidates(N, L, p):
        raise ValueError("(L-1) p k exceeds the number of finer-level entries")
    if mode == 1 and L > 1 and p * k > N // p ** (L - 2):
        raise ValueError("per-level quota: p k exceeds the entries of the coarsest finer level")
    if mode == 2 and n_select(L, p, k) and (chunk < 1 or n_select(L, p, k) % chunk):
        raise ValueError("stratified selection: the chunk quota must be >= 1 and divide (L-1) p k")
    if mode not in (0, 1, 2):
        raise ValueError("select mode must be 0 (joint), 1 (per-level quota) or 2 (stratified)")


def entry_level_index(f: np.ndarray, N: int, L: int, p: int):
    """Map flat pyramid indices to (level, index within level)."""
    f = np.asarray(f, dtype=np.int64)
    offs = np.asarray(level_offsets(N, L, p), dtype=np.int64)
    lvl = np.searchsorted(offs, f, side="right") - 1
    return lvl, f - offs[lvl]


# --------------------------------------------------------------------------
# bf16 rounding (storage points of the library)
# --------------------------------------------------------------------------

_BF16_MAX = (2.0 - 2.0**-7) * 2.0**127


def round_bf16(x) -> np.ndarray:
    """Round fp64 values once to the nearest bf16 value (ties to even).

    bf16 keeps 8 significant bits; the smallest subnormal is 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0)
    _, e = np.frexp(x[fin])                       # x = m 2^e, 0.5 <= |m| < 1
    q = np.maximum(e - 8, -133)                   # exponent of one unit in the last place
    r = np.ldexp(np.rint(np.ldexp(x[fin], -q)), q)  # rint: half to even
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


# --------------------------------------------------------------------------
# (i) Pyramid, Sec. 3.3
# --------------------------------------------------------------------------


def pyramid(xh: np.ndarray, L: int, p: int) -> list[np.ndarray]:
    """Levels of one head: level l row i = mean of base rows in W_i^(l).

    xh: [N, d] fp64.  Each level is the direct mean over its p^l base rows.
    """
    N, d = xh.shape
    levels = [xh]
    for lvl in range(1, L):
        w = p**lvl
        levels.append(xh.reshape(N // w, w, d).mean(axis=1))
    return levels


# --------------------------------------------------------------------------
# (ii) Scores and joint top-k, Sec. 3.4
# --------------------------------------------------------------------------


def token_norms(xh: np.ndarray) -> np.ndarray:
    """||x_t||_2 per row: squares summed in fp64 in ascending order of the
    feature index, fp64 square root, then one rounding to fp32 (the ranking
    key)."""
    ss = np.cumsum(xh * xh, axis=1)[:, -1]
    return np.sqrt(ss).astype(np.float32)


def scores(qh: np.ndarray, kh: np.ndarray, L: int, p: int):
    """QK and KQ streams of one head over all levels, flat-indexed, fp32.

    Level 0: the l2 norms of Q_t (query score) and K_t (key score).  Level
    l: the max of the level-0 scores inside W_i^(l).
    """
    qk0, kq0 = token_norms(qh), token_norms(kh)
    qk, kq = [], []
    for lvl in range(L):
        w = p**lvl
        qk.append(qk0.reshape(-1, w).max(axis=1))
        kq.append(kq0.reshape(-1, w).max(axis=1))
    return np.concatenate(qk), np.concatenate(kq)


def select(qk: np.ndarray, kq: np.ndarray, N: int, L: int, p: int, k: int,
           mode: int = 0, chunk: int = 0) -> np.ndarray:
    """Selection flags over all flat pyramid indices of one head.

    mode 0 (joint, Sec. 3.4): the QK and KQ streams of the finer levels are
    concatenated and sorted by score (descending), ties by lower flat index;
    distinct entries are taken from the front until n_sel are found.

    mode 1 (per-level quota, the Eq. 8 accounting read literally: each of
    the L-1 finer levels contributes p k entries): the same walk, but over
    one finer level at a time, taking p k distinct entries from each.

    mode 2 (stratified, the implementation note of Sec. 3: the score stream
    is partitioned into chunks and each chunk keeps its own top m): the
    finer-level entries, in flat-index order, are cut into n_sel / m
    contiguous chunks, chunk s covering [floor(s C / n), floor((s+1) C / n))
    for C candidates and n chunks; each chunk takes m = ``chunk`` distinct
    entries by the same walk.

    Level L-1 is kept whole in every mode.
    """
    C = n_candidates(N, L, p)
    flags = np.zeros(total_entries(N, L, p), dtype=bool)
    if mode == 0:
        ranges = [(0, C, n_select(L, p, k))]
    elif mode == 1:
        offs = level_offsets(N, L, p)
        ranges = [(offs[l], offs[l] + N // p**l, p * k) for l in range(L - 1)]
    elif mode == 2:
        n_sel = n_select(L, p, k)
        if n_sel and (chunk < 1 or n_sel % chunk):
            raise ValueError("stratified selection: the chunk quota must be >= 1 and divide (L-1) p k")
        n = n_sel // chunk if n_sel else 0      # nothing to take: no chunks
        ranges = [(s * C // n, (s + 1) * C // n, chunk) for s in range(n)]
    else:
        raise ValueError("select mode must be 0 (joint), 1 (per-level quota) or 2 (stratified)")
    for lo, hi, take in ranges:
        f = np.arange(lo, hi, dtype=np.int64)
        stream_f = np.concatenate([f, f])
        stream_s = np.concatenate([qk[lo:hi], kq[lo:hi]]).astype(np.float64)
        walk = stream_f[np.lexsort((stream_f, -stream_s))]
        _, first = np.unique(walk, return_index=True)   # where each entry first shows up
        flags[walk[np.sort(first)[:take]]] = True
    flags[C:] = True
    return flags


def gather_order(flags: np.ndarray, N: int, L: int, p: int):
    """Topological order of the selected entries (Sec. 3.5).

    Entries are sorted by the last base token they summarise,
    e = (i+1) p^l - 1, then by level (a child before its parent).
    Returns (sel_idx [S] flat indices in order, slot_map [P] slot or -1).
    """
    sel = np.nonzero(flags)[0].astype(np.int64)
    lvl, i = entry_level_index(sel, N, L, p)
    e = (i + 1) * (np.int64(p) ** lvl) - 1
    perm = np.lexsort((lvl, e))
    sel_idx = sel[perm]
    slot_map = np.full(flags.shape[0], -1, dtype=np.int64)
    slot_map[sel_idx] = np.arange(sel_idx.shape[0])
    return sel_idx, slot_map


def gather_rows(levels: list[np.ndarray], sel_idx: np.ndarray, N: int, L: int, p: int) -> np.ndarray:
    lvl, i = entry_level_index(sel_idx, N, L, p)
    d = levels[0].shape[1]
    out = np.empty((sel_idx.shape[0], d))
    for lv in range(L):
        m = lvl == lv
        out[m] = levels[lv][i[m]]
    return out


# --------------------------------------------------------------------------
# (iii) Causal softmax attention over the sub-sequence, Eq. 9
# --------------------------------------------------------------------------


def attention(qg, kg, vg, scale: float, rows=None, chunk: int = 256):
    """O_m = sum_{m' <= m} softmax_m'(scale q_m . k_m') v_m' and the natural-log
    LSE of each row, for the requested rows (all by default).

    A block of rows only multiplies against the keys up to its last row:
    later keys are masked for every row of the block (weight exactly 0)."""
    S = qg.shape[0]
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.empty((rows.shape[0], vg.shape[1]))
    lse = np.empty(rows.shape[0])
    cols = np.arange(S)
    for a in range(0, rows.shape[0], chunk):
        r = rows[a:a + chunk]
        hi = int(r.max()) + 1
        s = (qg[r] @ kg[:hi].T) * scale
        s[cols[None, :hi] > r[:, None]] = -np.inf
        mx = s.max(axis=1)
        ex = np.exp(s - mx[:, None])
        z = ex.sum(axis=1)
        lse[a:a + chunk] = mx + np.log(z)
        o[a:a + chunk] = (ex / z[:, None]) @ vg[:hi]
    return o, lse


def attention_bwd(qg, kg, vg, dog, scale: float, chunk: int = 256, rows=None):
    """Gradients of the causal attention with respect to its three inputs.

    P = softmax rows, dP = dO V^T, dS = P * (dP - rowsum(P * dP)),
    dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
    ``rows`` restricts the sums over query rows to the given rows (dQ is then
    exact on those rows, dK and dV hold those rows' share).
    """
    S = qg.shape[0]
    dq = np.zeros_like(qg)
    dk = np.zeros_like(kg)
    dv = np.zeros_like(vg)
    cols = np.arange(S)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    for a in range(0, rows.shape[0], chunk):
        r = rows[a:a + chunk]
        hi = int(r.max()) + 1          # keys after the block's last row: P = 0
        s = (qg[r] @ kg[:hi].T) * scale
        s[cols[None, :hi] > r[:, None]] = -np.inf
        mx = s.max(axis=1)
        ex = np.exp(s - mx[:, None])
        pr = ex / ex.sum(axis=1)[:, None]
        dp = dog[r] @ vg[:hi].T
        ds = pr * (dp - (pr * dp).sum(axis=1)[:, None])
        dq[r] = scale * (ds @ kg[:hi])
        dk[:hi] += scale * (ds.T @ qg[r])
        dv[:hi] += pr.T @ dog[r]
    return dq, dk, dv


# --------------------------------------------------------------------------
# (iv) Scatter-back, Sec. 3.6, and its adjoint
# --------------------------------------------------------------------------


def _level_slots(slot_map, N, L, p, lvl):
    off = level_offsets(N, L, p)[lvl]
    return slot_map[off:off + N // p**lvl]


def scatter(og: np.ndarray, slot_map: np.ndarray, N: int, L: int, p: int) -> np.ndarray:
    """O_t = sum over levels of the output of the selected entry whose shifted
    range [(i+1)p^l - 1, (i+2)p^l - 2] holds t; 0 where none does."""
    d = og.shape[1]
    o = np.zeros((N, d))
    for lvl in range(L):
        w = p**lvl
        slots = _level_slots(slot_map, N, L, p, lvl)
        rows = np.zeros((slots.shape[0], d))
        have = slots >= 0
        rows[have] = og[slots[have]]
        spread = np.repeat(rows, w, axis=0)       # entry i covers w tokens
        o[w - 1:] += spread[:N - (w - 1)]         # shifted by p^l - 1
    return o


def scatter_bwd(do: np.ndarray, sel_idx: np.ndarray, N: int, L: int, p: int) -> np.ndarray:
    """dO~_m = sum of dO_t over the shifted range of entry m (clipped to t < N)."""
    d = do.shape[1]
    lvl, i = entry_level_index(sel_idx, N, L, p)
    dog = np.zeros((sel_idx.shape[0], d))
    for lv in range(L):
        w = p**lv
        shifted = np.concatenate([do[w - 1:], np.zeros((w - 1, d))])
        sums = shifted.reshape(N // w, w, d).sum(axis=1)
        m = lvl == lv
        dog[m] = sums[i[m]]
    return dog


def pyramid_bwd(dxg: np.ndarray, slot_map: np.ndarray, N: int, L: int, p: int) -> np.ndarray:
    """dX_t = sum_l [entry (l, floor(t/p^l)) selected] p^-l dX~_slot (mean-pool
    adjoint; the pooling window is unshifted)."""
    d = dxg.shape[1]
    dx = np.zeros((N, d))
    for lvl in range(L):
        w = p**lvl
        slots = _level_slots(slot_map, N, L, p, lvl)
        rows = np.zeros((slots.shape[0], d))
        have = slots >= 0
        rows[have] = dxg[slots[have]] / w
        dx += np.repeat(rows, w, axis=0)
    return dx


# --------------------------------------------------------------------------
# One head, whole layer
# --------------------------------------------------------------------------


def forward_head(qh, kh, vh, L, p, k, scale=None, parity=True, flags=None, select_mode=0,
                 select_chunk=0):
    """Forward of one (batch, head).  qh, kh, vh: [N, d] fp64.

    ``flags`` freezes the selection (used by gradient and causality checks).
    """
    N, d = qh.shape
    check_config(N, L, p, k, select_mode, select_chunk)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qk, kq = scores(qh, kh, L, p)
    if flags is None:
        flags = select(qk, kq, N, L, p, k, select_mode, select_chunk)
    sel_idx, slot_map = gather_order(flags, N, L, p)
    rnd = round_bf16 if parity else (lambda a: a)
    pyr = [pyramid(x, L, p) for x in (qh, kh, vh)]
    pyr = [[lv[0]] + [rnd(a) for a in lv[1:]] for lv in pyr]
    qg, kg, vg = (gather_rows(lv, sel_idx, N, L, p) for lv in pyr)
    og, lse = attention(qg, kg, vg, scale)
    og = rnd(og)
    o = scatter(og, slot_map, N, L, p)
    return dict(qk=qk, kq=kq, flags=flags, sel_idx=sel_idx, slot_map=slot_map,
                levels=pyr, qg=qg, kg=kg, vg=vg, og=og, lse=lse, o=o,
                scale=scale, L=L, p=p, k=k, N=N, parity=parity)


def backward_head(st, doh):
    """Gradients dQ, dK, dV [N, d] of one head, indices frozen."""
    N, L, p = st["N"], st["L"], st["p"]
    rnd = round_bf16 if st["parity"] else (lambda a: a)
    dog = rnd(scatter_bwd(doh, st["sel_idx"], N, L, p))
    dqg, dkg, dvg = attention_bwd(st["qg"], st["kg"], st["vg"], dog, st["scale"])
    return tuple(pyramid_bwd(rnd(g), st["slot_map"], N, L, p) for g in (dqg, dkg, dvg)) + (dog,)


# --------------------------------------------------------------------------
# Whole tensors [B, N, H, d]
# --------------------------------------------------------------------------


def _head(x, b, h) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x[b, :, h, :], dtype=np.float64))


def forward(q, k, v, L, p, kk, scale=None, parity=True, select_mode=0, select_chunk=0):
    """Forward over every (b, h).  q, k, v: arrays [B, N, H, d] (any float
    dtype; converted exactly to fp64 per head).  Returns per-head states in a
    dict keyed by (b, h) and the output O [B, N, H, d]."""
    B, N, H, d = q.shape
    states = {}
    o = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            st = forward_head(_head(q, b, h), _head(k, b, h), _head(v, b, h),
                              L, p, kk, scale, parity, select_mode=select_mode,
                              select_chunk=select_chunk)
            states[(b, h)] = st
            o[b, :, h, :] = st["o"]
    return o, states


def backward(states, do):
    B, N, H, d = do.shape
    grads = [np.zeros((B, N, H, d)) for _ in range(3)]
    for (b, h), st in states.items():
        g = backward_head(st, _head(do, b, h))
        for a in range(3):
            grads[a][b, :, h, :] = g[a]
    return tuple(grads)


# --------------------------------------------------------------------------
# Sampled outputs for inputs too large to run whole
# --------------------------------------------------------------------------


def select_head(qh, kh, L, p, k, select_mode=0, select_chunk=0):
    """Scores, flags, gather order and slot map of one head (no attention)."""
    N = qh.shape[0]
    qk, kq = scores(qh, kh, L, p)
    flags = select(qk, kq, N, L, p, k, select_mode, select_chunk)
    sel_idx, slot_map = gather_order(flags, N, L, p)
    return dict(qk=qk, kq=kq, flags=flags, sel_idx=sel_idx, slot_map=slot_map)


def outputs_at(qh, kh, vh, L, p, k, t_list, scale=None, parity=True, sel=None):
    """O_t of one head for the base positions in ``t_list`` only: the
    attention runs just for the slots that reach those positions."""
    N, d = qh.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    sel = select_head(qh, kh, L, p, k) if sel is None else sel
    rnd = round_bf16 if parity else (lambda a: a)
    pyr = [pyramid(x, L, p) for x in (qh, kh, vh)]
    pyr = [[lv[0]] + [rnd(a) for a in lv[1:]] for lv in pyr]
    qg, kg, vg = (gather_rows(lv, sel["sel_idx"], N, L, p) for lv in pyr)
    t_list = np.asarray(t_list, dtype=np.int64)
    offs = level_offsets(N, L, p)
    need = {}
    for t in t_list:
        for lvl in range(L):
            j = (t + 1) // p**lvl - 1
            if j >= 0:
                s = sel["slot_map"][offs[lvl] + j]
                if s >= 0:
                    need.setdefault(int(t), []).append(int(s))
    rows = np.array(sorted({s for v in need.values() for s in v}), dtype=np.int64)
    og_rows, lse_rows = (attention(qg, kg, vg, scale, rows=rows) if rows.size
                         else (np.zeros((0, d)), np.zeros(0)))
    og_rows = rnd(og_rows)
    pos = {int(s): n for n, s in enumerate(rows)}
    out = np.zeros((t_list.shape[0], d))
    for n, t in enumerate(t_list):
        for s in need.get(int(t), []):          # ascending level order
            out[n] += og_rows[pos[s]]
    return out, dict(sel=sel, rows=rows, og=og_rows, lse=lse_rows, qg=qg, kg=kg, vg=vg)


# --------------------------------------------------------------------------
# The projections on either side of the layer (Sec. 3.1): per-head Q, K, V
# come from the layer's own W_Q, W_K, W_V, and the output projection W_O
# follows.  Plain products; the library computes them with its own GEMM.
# --------------------------------------------------------------------------


def projected_forward(x, wq, wk, wv, wo, H, L, p, k, scale=None, parity=True, select_mode=0,
                      flags=None):
    """x [B, N, Dm]; wq, wk, wv [H d, Dm]; wo [Dm, H d].

    Q = x wq^T, K = x wk^T, V = x wv^T (split into H heads of d), the
    Lighthouse layer per head, y = O wo^T.  Parity mode rounds to bf16 where
    the library stores bf16 (Q, K, V, O, y).  ``flags`` ({(b, h): flags})
    freezes the selection."""
    B, N, Dm = x.shape
    rnd = round_bf16 if parity else (lambda a: a)
    q, kk, v = (rnd(x @ w.T).reshape(B, N, H, -1) for w in (wq, wk, wv))
    o = np.zeros_like(q)
    states = {}
    for b in range(B):
        for h in range(H):
            st = forward_head(_head(q, b, h), _head(kk, b, h), _head(v, b, h), L, p, k, scale,
                              parity, flags=None if flags is None else flags[(b, h)],
                              select_mode=select_mode)
            states[(b, h)] = st
            o[b, :, h, :] = st["o"]
    o = rnd(o)
    y = rnd(o.reshape(B, N, -1) @ wo.T)
    return y, dict(x=x, wq=wq, wk=wk, wv=wv, wo=wo, q=q, k=kk, v=v, o=o, states=states,
                   parity=parity)


def projected_backward(st, dy):
    """Gradients (dx, dwq, dwk, dwv, dwo) of <y, dy>, the selection frozen."""
    rnd = round_bf16 if st["parity"] else (lambda a: a)
    x, o = st["x"], st["o"]
    B, N, Dm = x.shape
    do = rnd(dy @ st["wo"]).reshape(o.shape)
    grads = backward(st["states"], do)
    dq, dk, dv = (rnd(g).reshape(B * N, -1) for g in grads)
    xf, of, dyf = x.reshape(B * N, Dm), o.reshape(B * N, -1), dy.reshape(B * N, -1)
    dx = rnd(dq @ st["wq"] + dk @ st["wk"] + dv @ st["wv"]).reshape(B, N, Dm)
    dwq, dwk, dwv = (rnd(g.T @ xf) for g in (dq, dk, dv))
    dwo = rnd(dyf.T @ of)
    return dx, dwq, dwk, dwv, dwo


# --------------------------------------------------------------------------
# Context parallelism: the sequence cut into shards (the pages' multi-GPU
# training note: pyramid, scores and top-k run shard-local, and the gathered
# sub-sequences go through ring attention)
# --------------------------------------------------------------------------


def cp_forward_head(qh, kh, vh, L, p, k, R, scale=None, parity=True, select_mode=0,
                    select_chunk=0, flags=None):
    """Forward of one head with the N tokens cut into R contiguous shards.

    Each shard runs the pyramid, the scores and the selection on its own N/R
    tokens with the layer's p and k, so its sub-sequence has S(N/R) entries.
    The shards' sub-sequences, in shard order, are then attended to as one
    sequence under the causal mask.  That is what a ring over the shards
    computes: every entry of shard r' < r ends before any entry of shard r,
    so shard r's rows see all earlier shards' rows, and their own causally.
    Each shard scatters its own part of the output.  ``flags`` (one array
    per shard) freezes the selection, as in forward_head.
    """
    N, d = qh.shape
    if R < 1 or N % R:
        raise ValueError("the shard count must divide N")
    Ns = N // R
    check_config(Ns, L, p, k, select_mode, select_chunk)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rnd = round_bf16 if parity else (lambda a: a)
    shards = []
    for r in range(R):
        sl = slice(r * Ns, (r + 1) * Ns)
        qk, kq = scores(qh[sl], kh[sl], L, p)
        fl = select(qk, kq, Ns, L, p, k, select_mode, select_chunk) if flags is None else flags[r]
        sel_idx, slot_map = gather_order(fl, Ns, L, p)
        pyr = [pyramid(x[sl], L, p) for x in (qh, kh, vh)]
        pyr = [[lv[0]] + [rnd(a) for a in lv[1:]] for lv in pyr]
        qg, kg, vg = (gather_rows(lv, sel_idx, Ns, L, p) for lv in pyr)
        shards.append(dict(qk=qk, kq=kq, flags=fl, sel_idx=sel_idx, slot_map=slot_map,
                           qg=qg, kg=kg, vg=vg))
    qg, kg, vg = (np.concatenate([s[n] for s in shards]) for n in ("qg", "kg", "vg"))
    og, lse = attention(qg, kg, vg, scale)
    og = rnd(og)
    Sr = subseq_len(Ns, L, p, k)
    o = np.zeros((N, d))
    for r, s in enumerate(shards):
        s["og"] = og[r * Sr:(r + 1) * Sr]
        o[r * Ns:(r + 1) * Ns] = scatter(s["og"], s["slot_map"], Ns, L, p)
    return dict(shards=shards, qg=qg, kg=kg, vg=vg, og=og, lse=lse, o=o, scale=scale, L=L,
                p=p, k=k, N=N, R=R, parity=parity)


def cp_backward_head(st, doh):
    """Gradients dQ, dK, dV [N, d] of one sharded head, indices frozen: each
    shard's scatter adjoint, the attention backward over the concatenated
    sub-sequences, each shard's gather and pooling adjoint."""
    N, R, L, p, k = st["N"], st["R"], st["L"], st["p"], st["k"]
    Ns = N // R
    Sr = subseq_len(Ns, L, p, k)
    rnd = round_bf16 if st["parity"] else (lambda a: a)
    dog = np.concatenate([rnd(scatter_bwd(doh[r * Ns:(r + 1) * Ns], s["sel_idx"], Ns, L, p))
                          for r, s in enumerate(st["shards"])])
    dxg = attention_bwd(st["qg"], st["kg"], st["vg"], dog, st["scale"])
    grads = [np.zeros((N, doh.shape[1])) for _ in range(3)]
    for r, s in enumerate(st["shards"]):
        rows = slice(r * Sr, (r + 1) * Sr)
        for a in range(3):
            grads[a][r * Ns:(r + 1) * Ns] = pyramid_bwd(rnd(dxg[a][rows]), s["slot_map"], Ns, L, p)
    return tuple(grads)
