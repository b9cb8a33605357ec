"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one part of the oracle to something other than itself: the
numbers printed in "Long Context Pre-Training with Lighthouse Attention",
a hand-worked example, closed forms, invariants, brute force, a library
routine for a special case, or finite differences.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lighthouse_oracle as lo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale_rows=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape)
    if scale_rows:
        x *= rng.lognormal(0.0, 0.5, size=shape[:-1] + (1,))
    return lo.round_bf16(x)


# ---------------------------------------------------------------- sizes ---

def test_subseq_len_printed_values():
    g = json.load(open(os.path.join(GOLDEN, "subseq_len.json")))
    for c in g["cases"]:
        S = lo.subseq_len(c["N"], c["L"], c["p"], c["k"])
        if "S_exact" in c:
            assert S == c["S_exact"], c["cite"]
        else:
            assert abs(S - c["S_printed"]) <= c["rel_tol"] * c["S_printed"], c["cite"]
    # the worked case written out: 10^6 / 4^3 + 3 * 4 * 4096
    assert lo.subseq_len(10**6, 4, 4, 4096) == 15625 + 49152


@pytest.mark.parametrize("N,L,p", [(4096, 3, 4), (524288, 3, 4), (1 << 20, 4, 4),
                                   (64, 6, 2), (729, 4, 3), (8, 1, 2)])
def test_entry_count_bound(N, L, p):
    tot = lo.total_entries(N, L, p)
    assert tot == sum(N // p**l for l in range(L))
    assert tot * (p - 1) <= N * p          # sum_l N/p^l <= N p/(p-1), Sec. 3.3
    offs = lo.level_offsets(N, L, p)
    lvl, i = lo.entry_level_index(np.arange(tot), N, L, p)
    assert np.all(offs[0] == 0) and np.all(np.diff(lvl) >= 0)
    assert np.all(i < np.asarray(lo.level_sizes(N, L, p))[lvl])


def test_check_config_rejects():
    with pytest.raises(ValueError):
        lo.check_config(100, 3, 4, 1)       # 16 does not divide 100
    with pytest.raises(ValueError):
        lo.check_config(64, 3, 4, 100)      # budget above the candidates


# ----------------------------------------------------------- bf16 round ---

def test_round_bf16_ties_and_double_rounding():
    one = 1.0
    assert lo.round_bf16(one + 2**-8) == one                 # tie -> even
    assert lo.round_bf16(one + 3 * 2**-8) == one + 2**-6     # tie -> even (up)
    # just above a tie: a detour through fp32 would land on the tie and go down
    assert lo.round_bf16(one + 2**-8 + 2**-40) == one + 2**-7
    assert lo.round_bf16(-(one + 2**-8 + 2**-40)) == -(one + 2**-7)
    assert lo.round_bf16(2.0**-133) == 2.0**-133             # smallest subnormal
    assert lo.round_bf16(2.0**-135) == 0.0
    assert np.isinf(lo.round_bf16(3.5e38))
    assert lo.round_bf16(0.0) == 0.0


def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-30, 30, 100000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = lo.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


# -------------------------------------------------------------- pyramid ---

def test_pyramid_mean_of_means_and_linearity():
    N, d, L, p = 256, 8, 4, 4
    x, y = _rand((N, d), 1), _rand((N, d), 2)
    lv = lo.pyramid(x, L, p)
    for l in range(1, L):
        prev = lv[l - 1]
        np.testing.assert_allclose(prev.reshape(-1, p, d).mean(axis=1), lv[l], rtol=0, atol=1e-12)
        assert lv[l].shape == (N // p**l, d)
    a, b = 0.3, -1.7
    lz = lo.pyramid(a * x + b * y, L, p)
    ly = lo.pyramid(y, L, p)
    for l in range(L):
        np.testing.assert_allclose(lz[l], a * lv[l] + b * ly[l], rtol=0, atol=1e-12)
    # window definition W_i^(l) = [i p^l, (i+1) p^l - 1], Sec. 3.3
    i, l = 3, 2
    np.testing.assert_allclose(lv[l][i], x[i * 16:(i + 1) * 16].mean(axis=0), atol=1e-14)


# --------------------------------------------------------------- scores ---

def test_scores_norms_and_max_of_children():
    N, d, L, p = 512, 64, 4, 2
    q, k = _rand((N, d), 3), _rand((N, d), 4)
    qk, kq = lo.scores(q, k, L, p)
    offs = lo.level_offsets(N, L, p)
    # level 0: exactly-rounded fp32 of the l2 norm (fsum gives the exact sum)
    want = np.array([math.sqrt(math.fsum(float(v) * float(v) for v in row)) for row in q],
                    dtype=np.float64).astype(np.float32)
    np.testing.assert_array_equal(qk[:N], want)
    want_k = np.linalg.norm(k, axis=1).astype(np.float32)
    assert np.max(np.abs(kq[:N].astype(np.float64) - want_k) / want_k) <= 2**-23
    # each coarse score equals the max of its p children, bitwise
    for l in range(1, L):
        n = N // p**l
        for s in (qk, kq):
            child = s[offs[l - 1]:offs[l - 1] + n * p].reshape(n, p).max(axis=1)
            np.testing.assert_array_equal(s[offs[l]:offs[l] + n], child)
    assert qk.dtype == np.float32 and qk.shape == (lo.total_entries(N, L, p),)


# ------------------------------------------------------------ selection ---

def _brute_force_flags(qk, kq, N, L, p, k):
    """Entry f is selected iff fewer than n_sel candidates beat it, where g
    beats f if max(qk, kq)_g > max(qk, kq)_f, or equal and g < f."""
    C = lo.n_candidates(N, L, p)
    r = np.maximum(qk[:C], kq[:C]).astype(np.float64)
    flags = np.zeros(lo.total_entries(N, L, p), dtype=bool)
    for f in range(C):
        beats = np.sum(r > r[f]) + np.sum((r == r[f]) & (np.arange(C) < f))
        flags[f] = beats < lo.n_select(L, p, k)
    flags[C:] = True
    return flags


@pytest.mark.parametrize("N,L,p,k,seed", [(64, 3, 2, 2, 0), (64, 3, 2, 5, 1), (81, 3, 3, 2, 2),
                                          (128, 4, 2, 3, 3), (32, 2, 4, 3, 4)])
def test_select_matches_brute_force(N, L, p, k, seed):
    rng = np.random.default_rng(seed)
    # few distinct values -> many exact ties decided by the index rule
    qk0 = rng.integers(0, 6, N).astype(np.float64)
    kq0 = rng.integers(0, 6, N).astype(np.float64)
    q = np.zeros((N, 2)); q[:, 0] = qk0
    kk = np.zeros((N, 2)); kk[:, 1] = kq0
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k)
    np.testing.assert_array_equal(flags, _brute_force_flags(qk, kq, N, L, p, k))
    assert flags.sum() == lo.subseq_len(N, L, p, k)


def test_select_all_equal_takes_lowest_indices():
    N, L, p, k = 64, 3, 2, 3
    q = np.ones((N, 4)); kk = np.ones((N, 4))
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k)
    n_sel = lo.n_select(L, p, k)
    C = lo.n_candidates(N, L, p)
    assert flags[:n_sel].all() and not flags[n_sel:C].any() and flags[C:].all()


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_n8_l2_p2_k1.json")))
    c, e = g["config"], g["expected"]
    N, L, p, k = c["N"], c["L"], c["p"], c["k"]
    q = np.zeros((N, 2)); q[:, 0] = g["inputs"]["qk0"]
    kk = np.zeros((N, 2)); kk[:, 1] = g["inputs"]["kq0"]
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k)
    np.testing.assert_array_equal(flags[:N].astype(int), e["flags_level0"])
    sel_idx, slot_map = lo.gather_order(flags, N, L, p)
    np.testing.assert_array_equal(sel_idx, e["sel_idx"])
    assert len(sel_idx) == e["S"] == lo.subseq_len(N, L, p, k)
    # scatter placement: one-hot outputs per slot reveal which slots reach t
    S = len(sel_idx)
    o = lo.scatter(np.eye(S), slot_map, N, L, p)
    for t in range(N):
        assert sorted(np.nonzero(o[t])[0].tolist()) == sorted(e["slots_per_t"][t])
    np.testing.assert_array_equal(o.sum(axis=1), e["fanin"])


# ---------------------------------------------------------------- order ---

@pytest.mark.parametrize("N,L,p,k", [(4096, 3, 4, 64), (512, 4, 2, 7), (729, 4, 3, 5), (256, 1, 4, 0)])
def test_gather_order_is_topological(N, L, p, k):
    q, kk = _rand((N, 16), 5), _rand((N, 16), 6)
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k)
    sel_idx, slot_map = lo.gather_order(flags, N, L, p)
    S = lo.subseq_len(N, L, p, k)
    assert len(sel_idx) == S and len(np.unique(sel_idx)) == S
    lvl, i = lo.entry_level_index(sel_idx, N, L, p)
    e = (i + 1) * p**lvl - 1
    assert np.all(np.diff(e) >= 0)
    same = np.diff(e) == 0
    assert np.all(np.diff(lvl)[same] > 0)
    assert np.all(slot_map[sel_idx] == np.arange(S))
    assert np.sum(slot_map >= 0) == S
    off = lo.level_offsets(N, L, p)[L - 1]
    assert np.all(slot_map[off:] >= 0)            # coarsest level whole


# -------------------------------------------------------------- scatter ---

@pytest.mark.parametrize("N,L,p,k", [(4096, 3, 4, 64), (512, 4, 2, 7), (243, 3, 3, 2)])
def test_scatter_fanin_coverage_disjoint(N, L, p, k):
    q, kk = _rand((N, 8), 7), _rand((N, 8), 8)
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k)
    sel_idx, slot_map = lo.gather_order(flags, N, L, p)
    S = len(sel_idx)
    lvl, _ = lo.entry_level_index(sel_idx, N, L, p)
    fan = np.zeros(N, dtype=int)
    for l in range(L):
        one = np.zeros((S, 1)); one[lvl == l] = 1.0
        cnt = lo.scatter(one, slot_map, N, L, p)[:, 0]
        assert np.all(cnt <= 1)                    # disjoint within a level
        fan += cnt.astype(int)
    assert np.all(fan <= L)                        # fan-in bounded by L
    assert np.all(fan[p ** (L - 1) - 1:] >= 1)     # no holes past the first coarse end


def test_scatter_adjoint_and_pyramid_adjoint():
    N, L, p, k, d = 512, 3, 4, 8, 4
    q, kk = _rand((N, d), 9), _rand((N, d), 10)
    qk, kq = lo.scores(q, kk, L, p)
    flags = lo.select(qk, kq, N, L, p, k)
    sel_idx, slot_map = lo.gather_order(flags, N, L, p)
    S = len(sel_idx)
    rng = np.random.default_rng(11)
    og, do = rng.standard_normal((S, d)), rng.standard_normal((N, d))
    lhs = np.sum(lo.scatter(og, slot_map, N, L, p) * do)
    rhs = np.sum(og * lo.scatter_bwd(do, sel_idx, N, L, p))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1)
    x, g = rng.standard_normal((N, d)), rng.standard_normal((S, d))
    gx = lo.gather_rows(lo.pyramid(x, L, p), sel_idx, N, L, p)
    lhs = np.sum(gx * g)
    rhs = np.sum(x * lo.pyramid_bwd(g, slot_map, N, L, p))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1)


# ------------------------------------------------------------ attention ---

@pytest.mark.parametrize("N,d", [(64, 8), (200, 16)])
def test_single_level_is_dense_causal_sdpa(N, d):
    """L = 1: S = N, nothing is pooled or shifted, O is causal SDPA (Eq. 1)."""
    q, k, v = (_rand((N, d), s) for s in (12, 13, 14))
    st = lo.forward_head(q, k, v, L=1, p=4, k=0, parity=False)
    assert len(st["sel_idx"]) == N and np.all(st["sel_idx"] == np.arange(N))
    want = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a)[None, None] for a in (q, k, v)), is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(st["o"], want, rtol=1e-12, atol=1e-12)


def test_attention_first_row_uniform_v_and_lse():
    N, L, p, k, d = 1024, 3, 4, 16, 8
    q, kk, v = (_rand((N, d), s) for s in (15, 16, 17))
    v[:] = 0.75
    st = lo.forward_head(q, kk, v, L, p, k, parity=False)
    np.testing.assert_allclose(st["og"][0], st["vg"][0], atol=0)      # one visible key
    lvl, _ = lo.entry_level_index(st["sel_idx"], N, L, p)
    fan = np.zeros(N)
    for l in range(L):
        one = np.zeros((len(lvl), 1)); one[lvl == l] = 1.0
        fan += lo.scatter(one, st["slot_map"], N, L, p)[:, 0]
    np.testing.assert_allclose(st["o"], 0.75 * fan[:, None] * np.ones((1, d)), atol=1e-12)
    # LSE row 1 by hand: log(exp(s00)+exp(s01))
    s = st["scale"] * np.array([st["qg"][1] @ st["kg"][0], st["qg"][1] @ st["kg"][1]])
    assert abs(st["lse"][1] - math.log(math.exp(s[0]) + math.exp(s[1]))) < 1e-12


def test_causality_with_frozen_selection():
    N, L, p, k, d = 256, 3, 4, 6, 8
    q, kk, v = (_rand((N, d), s) for s in (18, 19, 20))
    st = lo.forward_head(q, kk, v, L, p, k, parity=False)
    t0 = 137
    q2, k2, v2 = q.copy(), kk.copy(), v.copy()
    rng = np.random.default_rng(21)
    for a in (q2, k2, v2):
        a[t0 + 1:] += rng.standard_normal(a[t0 + 1:].shape)
    st2 = lo.forward_head(q2, k2, v2, L, p, k, parity=False, flags=st["flags"])
    np.testing.assert_array_equal(st2["o"][:t0 + 1], st["o"][:t0 + 1])
    assert not np.allclose(st2["o"][t0 + 1:], st["o"][t0 + 1:])


# ------------------------------------------------------------- backward ---

def test_gradients_match_finite_differences():
    N, L, p, k, d = 64, 3, 2, 3, 4
    q, kk, v = (_rand((N, d), s) for s in (22, 23, 24))
    rng = np.random.default_rng(25)
    g = rng.standard_normal((N, d))
    st = lo.forward_head(q, kk, v, L, p, k, parity=False)
    dq, dk, dv, _ = lo.backward_head(st, g)
    flags = st["flags"]

    def loss(a, b, c):
        return np.sum(lo.forward_head(a, b, c, L, p, k, parity=False, flags=flags)["o"] * g)

    eps = 1e-6
    pts = [(t, j) for t in (0, 1, 5, 17, 33, 62, 63) for j in range(d)]
    for which, grad in enumerate((dq, dk, dv)):
        for t, j in pts:
            args_p = [q.copy(), kk.copy(), v.copy()]
            args_m = [q.copy(), kk.copy(), v.copy()]
            args_p[which][t, j] += eps
            args_m[which][t, j] -= eps
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[t, j]) <= 1e-6 * max(1.0, abs(fd)), (which, t, j, fd, grad[t, j])


def test_parity_mode_rounds_only_storage_points():
    N, L, p, k, d = 256, 3, 4, 6, 8
    q, kk, v = (_rand((N, d), s) for s in (26, 27, 28))
    a = lo.forward_head(q, kk, v, L, p, k, parity=True)
    b = lo.forward_head(q, kk, v, L, p, k, parity=False)
    np.testing.assert_array_equal(a["sel_idx"], b["sel_idx"])
    np.testing.assert_array_equal(lo.round_bf16(a["og"]), a["og"])
    assert np.max(np.abs(a["o"] - b["o"])) < 0.05


def test_outputs_at_matches_full_forward():
    N, L, p, k, d = 1024, 3, 4, 16, 8
    q, kk, v = (_rand((N, d), s) for s in (29, 30, 31))
    st = lo.forward_head(q, kk, v, L, p, k, parity=True)
    ts = [0, 3, 14, 15, 16, 511, 700, 1023]
    got, _ = lo.outputs_at(q, kk, v, L, p, k, ts, parity=True)
    np.testing.assert_allclose(got, st["o"][ts], rtol=0, atol=1e-12)
