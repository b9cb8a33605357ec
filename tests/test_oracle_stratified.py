"""Pins of the oracle's stratified selection (select_mode 2): the finer-level
entries, in flat-index order, are cut into n_sel / m contiguous chunks of
near-equal size, and each chunk keeps its own top m by the joint mode's
ordering (score desc, lower flat index first); the coarsest level is kept
whole, so S is the same as in the other modes."""
import json
import os

import numpy as np
import pytest

from oracle import lighthouse_oracle as lo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _levels_selected(flags, N, L, p):
    offs = lo.level_offsets(N, L, p)
    return [sorted(np.nonzero(flags[offs[l]:offs[l] + N // p**l])[0].tolist()) for l in range(L)]


def _scores_from_norms(qk0, N, L, p):
    q = np.zeros((N, 2)); q[:, 0] = qk0
    return lo.scores(q, np.zeros((N, 2)), L, p)


def test_hand_worked_stratified():
    g = json.load(open(os.path.join(GOLDEN, "stratified_n16_l3_p2_k1.json")))
    c, x = g["config"], g["expected"]
    N, L, p, k, m = c["N"], c["L"], c["p"], c["k"], c["chunk"]
    qk, kq = _scores_from_norms(np.array(g["inputs"]["qk0"], float), N, L, p)
    flags = lo.select(qk, kq, N, L, p, k, mode=2, chunk=m)
    sel = _levels_selected(flags, N, L, p)
    assert sel[0] == x["stratified"]["level0"] and sel[1] == x["stratified"]["level1"]
    assert sel[2] == list(range(N // p**2))
    assert int(flags.sum()) == x["S"]
    sel_idx, _ = lo.gather_order(flags, N, L, p)
    assert sel_idx.tolist() == x["stratified"]["sel_idx"]
    qk, kq = _scores_from_norms(np.ones(N), N, L, p)
    sel = _levels_selected(lo.select(qk, kq, N, L, p, k, mode=2, chunk=m), N, L, p)
    assert sel[0] == x["all_equal_stratified"]["level0"]
    assert sel[1] == x["all_equal_stratified"]["level1"]


def _brute_force(qk, kq, C, n_chunks, m):
    """Entry f of chunk s is chosen iff fewer than m entries of the same chunk
    beat it: a higher r = max(QK, KQ), or an equal r at a lower flat index."""
    chosen = set()
    r = [max(float(a), float(b)) for a, b in zip(qk[:C], kq[:C])]
    for s in range(n_chunks):
        lo_, hi_ = s * C // n_chunks, (s + 1) * C // n_chunks
        for f in range(lo_, hi_):
            beaten_by = sum(1 for g in range(lo_, hi_) if r[g] > r[f] or (r[g] == r[f] and g < f))
            if beaten_by < m:
                chosen.add(f)
    return chosen


@pytest.mark.parametrize("N,L,p,k,m,seed", [
    (64, 3, 2, 4, 2, 0),       # 8 chunks of 12
    (96, 2, 3, 5, 3, 1),       # 5 chunks, sizes 19/19/19/19/20
    (128, 4, 2, 3, 1, 2),      # 18 chunks over three finer levels, sizes 12/13
    (64, 3, 4, 3, 6, 3),       # 4 chunks crossing the level boundary at f = 64
])
def test_brute_force_and_counts(N, L, p, k, m, seed):
    rng = np.random.default_rng(seed)
    q, kk = rng.standard_normal((N, 4)), rng.standard_normal((N, 4))
    q[rng.integers(0, N, 6)] = q[0]           # exact ties between tokens and across levels
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k, mode=2, chunk=m)
    C, n_sel = lo.n_candidates(N, L, p), lo.n_select(L, p, k)
    n_chunks = n_sel // m
    assert set(np.nonzero(flags[:C])[0].tolist()) == _brute_force(qk, kq, C, n_chunks, m)
    for s in range(n_chunks):
        assert int(flags[s * C // n_chunks:(s + 1) * C // n_chunks].sum()) == m
    assert flags[C:].all()
    assert int(flags.sum()) == lo.subseq_len(N, L, p, k)


def test_one_chunk_is_the_joint_selection():
    rng = np.random.default_rng(4)
    N, L, p, k = 256, 3, 4, 6
    q, kk = rng.standard_normal((N, 8)), rng.standard_normal((N, 8))
    qk, kq = lo.scores(q, kk, L, p)
    n_sel = lo.n_select(L, p, k)
    assert np.array_equal(lo.select(qk, kq, N, L, p, k, mode=2, chunk=n_sel),
                          lo.select(qk, kq, N, L, p, k, mode=0))


def test_every_candidate_its_own_chunk_keeps_all():
    # N = 16, L = 2, p = 2, k = 8: n_sel = 16 = the 16 level-0 candidates, so
    # m = 1 makes every candidate its own chunk and every entry is kept
    N, L, p, k = 16, 2, 2, 8
    q = np.random.default_rng(5).standard_normal((N, 4))
    qk, kq = lo.scores(q, q, L, p)
    assert lo.select(qk, kq, N, L, p, k, mode=2, chunk=1).all()


def test_stratified_config_limits():
    lo.check_config(4096, 3, 4, 64, mode=2, chunk=64)
    with pytest.raises(ValueError):
        lo.check_config(4096, 3, 4, 64, mode=2, chunk=0)
    with pytest.raises(ValueError):
        lo.check_config(4096, 3, 4, 64, mode=2, chunk=48)     # 512 is not a multiple of 48
    with pytest.raises(ValueError):
        lo.check_config(4096, 3, 4, 64, mode=3)
