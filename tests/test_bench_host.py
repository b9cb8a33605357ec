"""Host-side accounting of bench.py, on the CPU: the algorithmic bytes and
FLOPs of every stage, the written part of each HBM stage's bytes (the
read/write-aware bound divides it by the measured write-only rate), and the
captured DRAM traffic, which is reported only for the workload it was taken
on."""
import json
import os

import pytest

import bench
from hierarchical_selection_attention_b200.inputs import WORKLOADS


@pytest.mark.parametrize("w", WORKLOADS, ids=[w["name"] for w in WORKLOADS])
def test_written_bytes_are_part_of_the_algorithmic_bytes(w):
    alg = bench.algorithmic(w)
    wr = bench.algorithmic_writes(w)
    hbm = {k for k, (bound, _) in alg.items() if bound == "hbm"}
    assert set(wr) == hbm
    for k in hbm:
        assert 0 < wr[k] < alg[k][1], k
    B, N, H, d, L, p, k, S, P, R, C = bench.sizes(w)
    tok, gat = B * N * H * d * 2, B * H * S * d * 2
    # the stages whose output is one [B, N, H, d] tensor, or three
    assert wr["scatter"] == tok
    assert wr["gather_bwd"] == 3 * tok
    assert wr["gather"] == 3 * gat


def test_attention_flops_are_the_causal_triangle():
    w = WORKLOADS[3]
    B, N, H, d, L, p, k, S, P, R, C = bench.sizes(w)
    alg = bench.algorithmic(w)
    one = 2 * B * H * d * S * (S + 1) // 2          # one causal S x S x d product
    assert alg["attn_fwd"] == ("tensor", 2 * one)
    assert alg["attn_bwd_dkdv"] == ("tensor", 4 * one)
    assert alg["attn_bwd_dq"] == ("tensor", one)
    assert bench.EXECUTED_GEMMS == {"attn_fwd": 2, "attn_bwd_dkdv": 4, "attn_bwd_dq": 3}


def test_traffic_is_reported_only_for_its_workload():
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    ent = json.load(open(path))["attn_bwd_dkdv"]
    assert bench.load_traffic("attn_bwd_dkdv", ent["workload_name"]) == ent["dram_bytes_per_launch"]
    others = [w["name"] for w in WORKLOADS if w["name"] != ent["workload_name"]]
    assert others
    for name in others:
        assert bench.load_traffic("attn_bwd_dkdv", name) is None
    assert bench.load_traffic("attn_fwd", ent["workload_name"]) is None
