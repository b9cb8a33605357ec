"""Pins of the oracle's context-parallel layer (cp_forward_head /
cp_backward_head): the sequence cut into R contiguous shards, pyramid,
scores and selection per shard, causal attention over the shards'
sub-sequences in shard order (what a ring over the shards computes), and a
per-shard scatter."""
import numpy as np
import pytest

from oracle import lighthouse_oracle as lo


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_one_shard_is_the_layer():
    N, L, p, k, d = 256, 3, 4, 6, 8
    q, kk, v = (_rand((N, d), s) for s in (1, 2, 3))
    g = _rand((N, d), 4)
    a = lo.forward_head(q, kk, v, L, p, k, parity=True)
    c = lo.cp_forward_head(q, kk, v, L, p, k, R=1, parity=True)
    np.testing.assert_array_equal(c["o"], a["o"])
    np.testing.assert_array_equal(c["shards"][0]["sel_idx"], a["sel_idx"])
    for x, y in zip(lo.cp_backward_head(c, g), lo.backward_head(a, g)[:3]):
        np.testing.assert_array_equal(x, y)


def test_first_shard_is_the_layer_on_its_own_tokens():
    # shard 0 sees no other shard, so its output is the plain layer on its tokens
    N, L, p, k, d, R = 512, 3, 4, 5, 8, 4
    q, kk, v = (_rand((N, d), s) for s in (5, 6, 7))
    c = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=True)
    Ns = N // R
    a = lo.forward_head(q[:Ns], kk[:Ns], v[:Ns], L, p, k, parity=True)
    np.testing.assert_array_equal(c["o"][:Ns], a["o"])


def test_later_shards_do_not_reach_earlier_ones():
    N, L, p, k, d, R = 384, 2, 4, 7, 8, 3
    q, kk, v = (_rand((N, d), s) for s in (8, 9, 10))
    base = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)["o"]
    Ns = N // R
    q2, k2, v2 = q.copy(), kk.copy(), v.copy()
    for x in (q2, k2, v2):
        x[2 * Ns:] = _rand((Ns, d), 11)            # rewrite the last shard
    moved = lo.cp_forward_head(q2, k2, v2, L, p, k, R, parity=False)["o"]
    np.testing.assert_array_equal(moved[:2 * Ns], base[:2 * Ns])
    k3 = kk.copy()
    k3[:Ns] *= 3.0                                  # an earlier shard's keys do reach later ones
    later = lo.cp_forward_head(q, k3, v, L, p, k, R, parity=False)["o"]
    assert np.abs(later[Ns:] - base[Ns:]).max() > 1e-3


def test_shards_end_in_order():
    # every entry of shard r ends (last base token, global) before any entry of shard r+1,
    # which is why the concatenation in shard order takes the plain causal mask
    N, L, p, k, d, R = 512, 3, 2, 9, 4, 4
    q, kk, v = (_rand((N, d), s) for s in (12, 13, 14))
    c = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)
    Ns = N // R
    ends = []
    for r, s in enumerate(c["shards"]):
        lvl, i = lo.entry_level_index(s["sel_idx"], Ns, L, p)
        e = (i + 1) * p ** lvl - 1 + r * Ns
        assert np.all(np.diff(e) >= 0)              # topological order inside the shard
        ends.append((e.min(), e.max()))
    for (_, hi), (lo_, _) in zip(ends, ends[1:]):
        assert hi < lo_


def test_ring_of_blocks_equals_the_concatenated_attention():
    # what a ring computes: shard r's queries against each earlier shard's whole block and
    # its own block causally, merged by log-sum-exp, block by block
    N, L, p, k, d, R = 384, 3, 2, 5, 8, 3
    q, kk, v = (_rand((N, d), s, 0.7) for s in (15, 16, 17))
    c = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)
    Sr = lo.subseq_len(N // R, L, p, k)
    qg, kg, vg, sc = c["qg"], c["kg"], c["vg"], c["scale"]
    for r in range(R):
        Q = qg[r * Sr:(r + 1) * Sr]
        m = np.full(Sr, -np.inf)
        lsum = np.zeros(Sr)
        acc = np.zeros((Sr, d))
        for j in range(r + 1):                      # blocks arrive one by one
            K, V = kg[j * Sr:(j + 1) * Sr], vg[j * Sr:(j + 1) * Sr]
            s = sc * Q @ K.T
            if j == r:
                s = np.where(np.tri(Sr, dtype=bool), s, -np.inf)
            m_new = np.maximum(m, s.max(axis=1))
            w = np.exp(m - m_new)
            e = np.exp(s - m_new[:, None])
            lsum = lsum * w + e.sum(axis=1)
            acc = acc * w[:, None] + e @ V
            m = m_new
        np.testing.assert_allclose(acc / lsum[:, None], c["og"][r * Sr:(r + 1) * Sr],
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(m + np.log(lsum), c["lse"][r * Sr:(r + 1) * Sr],
                                   rtol=1e-12, atol=1e-12)


def test_cp_gradients_match_finite_differences():
    N, L, p, k, d, R = 64, 2, 2, 3, 4, 2
    q, kk, v = (_rand((N, d), s) for s in (18, 19, 20))
    g = _rand((N, d), 21)
    st = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)
    grads = lo.cp_backward_head(st, g)
    flags = [s["flags"] for s in st["shards"]]

    def loss(a, b, c):
        return np.sum(lo.cp_forward_head(a, b, c, L, p, k, R, parity=False, flags=flags)["o"] * g)

    eps = 1e-6
    pts = [(t, j) for t in (0, 3, 31, 32, 33, 50, 63) for j in range(d)]
    for which, grad in enumerate(grads):
        for t, j in pts:
            ap = [q.copy(), kk.copy(), v.copy()]
            am = [q.copy(), kk.copy(), v.copy()]
            ap[which][t, j] += eps
            am[which][t, j] -= eps
            fd = (loss(*ap) - loss(*am)) / (2 * eps)
            assert abs(fd - grad[t, j]) <= 1e-6 * max(1.0, abs(fd)), (which, t, j, fd, grad[t, j])


def test_cp_config_limits():
    q = np.zeros((96, 4))
    with pytest.raises(ValueError):
        lo.cp_forward_head(q, q, q, 2, 2, 1, R=5)      # 5 does not divide 96
    with pytest.raises(ValueError):
        lo.cp_forward_head(q, q, q, 3, 4, 1, R=4)      # a shard of 24 tokens: 16 does not divide 24


def test_uniform_values_give_each_shard_its_own_fan_in():
    # V = c everywhere: every attention row is exactly c, so O_t = c times the number of
    # levels whose selected entry reaches t (shifted window, shard-local indices)
    N, L, p, k, d, R = 192, 3, 2, 4, 4, 3
    q, kk = _rand((N, d), 22), _rand((N, d), 23)
    c = np.array([0.5, -1.0, 2.0, 0.25])
    v = np.tile(c, (N, 1))
    st = lo.cp_forward_head(q, kk, v, L, p, k, R, parity=False)
    Ns = N // R
    offs = lo.level_offsets(Ns, L, p)
    for r, s in enumerate(st["shards"]):
        for tl in range(Ns):
            fan = 0
            for lvl in range(L):
                j = (tl + 1) // p**lvl - 1
                if j >= 0 and s["flags"][offs[lvl] + j]:
                    fan += 1
            np.testing.assert_allclose(st["o"][r * Ns + tl], fan * c, rtol=0, atol=1e-12)
