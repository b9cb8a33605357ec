"""The ring schedule of the context-parallel layer (host logic, no GPU):
which K/V block each rank works on at each step, in which mode, and where
each sum opens and closes."""
import pytest

from hierarchical_selection_attention_b200 import ring


@pytest.mark.parametrize("R", [1, 2, 3, 4, 7])
def test_every_visible_pair_once_in_order(R):
    sch = ring.schedule(R)
    want = {(r, s) for r in range(R) for s in range(r + 1)}   # shard r sees shards 0..r
    for kind in ("forward", "dq", "dkdv"):
        pairs = [(st.rank, st.src) for st in sch[kind]]
        assert len(pairs) == len(set(pairs)) and set(pairs) == want, kind
        for st in sch[kind]:
            assert st.mode == (ring.DIAG if st.src == st.rank else ring.FULL)
            if st.step < R:                  # the block really is at that rank then
                assert ring.block_at(R, st.rank, st.step) == st.src
            else:                            # home step: the block is back at its owner
                assert st.step == R and st.src == st.rank == ring.block_at(R, st.rank, R)


@pytest.mark.parametrize("R", [1, 2, 3, 5])
def test_each_sum_opens_once_and_closes_last(R):
    sch = ring.schedule(R)
    for kind, key in (("forward", "rank"), ("dq", "rank"), ("dkdv", "src")):
        by = {}
        for st in sch[kind]:
            by.setdefault(getattr(st, key), []).append(st)
        assert sorted(by) == list(range(R))
        for owner, sts in by.items():
            sts.sort(key=lambda st: st.step)
            assert [st.first for st in sts] == [True] + [False] * (len(sts) - 1), (kind, owner)
            assert [st.last for st in sts] == [False] * (len(sts) - 1) + [True], (kind, owner)
    # forward / dQ open on the own (causal) block; dK/dV close on it, at home
    for r in range(R):
        assert ring.forward_steps(R, r)[0].mode == ring.DIAG
        home = ring.dkdv_steps(R, r)[-1]
        assert home.mode == ring.DIAG and home.step == R and home.last


def test_one_shard_is_one_plain_step():
    assert ring.forward_steps(1, 0) == [ring.Step(0, 0, 0, ring.DIAG, True, True)]
    assert ring.dkdv_steps(1, 0) == [ring.Step(1, 0, 0, ring.DIAG, True, True)]


def test_bad_ranks_rejected():
    with pytest.raises(ValueError):
        ring.forward_steps(3, 3)
    with pytest.raises(ValueError):
        ring.dkdv_steps(0, 0)
