"""Pins of the oracle's per-level-quota selection (select_mode 1): each of
the L-1 finer levels contributes exactly p k entries, chosen within the level
by the joint mode's own ordering (score desc, lower flat index first); the
coarsest level is kept whole, so S is the same as in the joint mode."""
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
    # Q_t = (qk_t, 0), K_t = 0: the oracle's own norms and max-pooling
    q = np.zeros((N, 2)); q[:, 0] = qk0
    return lo.scores(q, np.zeros((N, 2)), L, p)


def test_hand_worked_quota_vs_joint():
    g = json.load(open(os.path.join(GOLDEN, "quota_n16_l3_p2_k1.json")))
    c, x = g["config"], g["expected"]
    N, L, p, k = c["N"], c["L"], c["p"], c["k"]
    qk, kq = _scores_from_norms(np.array(g["inputs"]["qk0"], float), N, L, p)
    fj = lo.select(qk, kq, N, L, p, k, mode=0)
    fq = lo.select(qk, kq, N, L, p, k, mode=1)
    sj, sq = _levels_selected(fj, N, L, p), _levels_selected(fq, N, L, p)
    assert sj[0] == x["joint"]["level0"] and sj[1] == x["joint"]["level1"]
    assert sq[0] == x["quota"]["level0"] and sq[1] == x["quota"]["level1"]
    assert sj[2] == sq[2] == list(range(N // p**2))
    assert int(fq.sum()) == int(fj.sum()) == x["S"]
    sel_idx, _ = lo.gather_order(fq, N, L, p)
    assert sel_idx.tolist() == x["quota"]["sel_idx"]
    # all-equal scores: every choice is made by the tie rule
    qk, kq = _scores_from_norms(np.ones(N), N, L, p)
    sj = _levels_selected(lo.select(qk, kq, N, L, p, k, mode=0), N, L, p)
    sq = _levels_selected(lo.select(qk, kq, N, L, p, k, mode=1), N, L, p)
    assert sj[0] == x["all_equal_joint"]["level0"] and sj[1] == x["all_equal_joint"]["level1"]
    assert sq[0] == x["all_equal_quota"]["level0"] and sq[1] == x["all_equal_quota"]["level1"]


@pytest.mark.parametrize("N,L,p,k,seed", [(256, 3, 4, 3, 0), (512, 4, 2, 5, 1), (192, 2, 3, 7, 2)])
def test_quota_counts_and_length(N, L, p, k, seed):
    rng = np.random.default_rng(seed)
    q, kk = rng.standard_normal((N, 8)), rng.standard_normal((N, 8))
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k, mode=1)
    per_level = [len(s) for s in _levels_selected(flags, N, L, p)]
    assert per_level[:L - 1] == [p * k] * (L - 1)
    assert per_level[L - 1] == N // p ** (L - 1)
    assert int(flags.sum()) == lo.subseq_len(N, L, p, k)
    # within each finer level the chosen entries are never beaten by an unchosen one
    offs = lo.level_offsets(N, L, p)
    r = np.maximum(qk, kq)
    for l in range(L - 1):
        f = np.arange(offs[l], offs[l] + N // p**l)
        chosen, rest = f[flags[f]], f[~flags[f]]
        if rest.size:
            worst = min(chosen, key=lambda e: (r[e], -e))
            best_rest = max(rest, key=lambda e: (r[e], -e))
            assert (r[worst], -worst) > (r[best_rest], -best_rest)


def test_two_levels_quota_equals_joint():
    # with one finer level the quota is the whole budget: both modes coincide
    rng = np.random.default_rng(3)
    N, L, p, k = 384, 2, 4, 9
    q, kk = rng.standard_normal((N, 16)), rng.standard_normal((N, 16))
    qk, kq = lo.scores(q, kk, L, p)
    assert np.array_equal(lo.select(qk, kq, N, L, p, k, mode=0), lo.select(qk, kq, N, L, p, k, mode=1))


def test_quota_config_limits():
    # p k must fit in the coarsest finer level (level L-2 has N / p^(L-2) entries)
    lo.check_config(64, 3, 4, 4, mode=1)          # 16 <= 16
    with pytest.raises(ValueError):
        lo.check_config(64, 3, 4, 5, mode=1)      # 20 > 16
    lo.check_config(64, 3, 4, 5, mode=0)          # the joint budget 40 <= 80 candidates
    with pytest.raises(ValueError):
        lo.select(np.zeros(84), np.zeros(84), 64, 3, 4, 1, mode=3)   # no such mode
    with pytest.raises(ValueError):
        lo.select(np.zeros(84), np.zeros(84), 64, 3, 4, 1, mode=2)   # stratified needs its quota
