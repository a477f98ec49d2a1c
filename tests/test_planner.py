"""The decode planner's choices, on the host (no GPU): which cut a call gets on
a 148-SM part, and invariants of every plan.  The expected cuts are the ones
measured fastest on B200 (even tile cut for long calls, whole units or equal
pieces of units for short ones)."""
import math

import pytest

import head_sparse_decode_b200 as sha

# (B, H_q, H_kv, N_kv, d, top_k) -> (blocks, whole units: no workspace)
CUTS = {
    # long calls: the even tile cut, units split across neighbouring blocks
    "opt66b": ((64, 72, 72, 1920, 128, 22), 148, False),
    "llama2_7b": ((128, 32, 32, 2048, 128, 16), 148, False),
    "llama31_70b_gqa": ((32, 64, 8, 4096, 128, 5), 148, False),
    "llama31_70b_gqa_16k": ((8, 64, 8, 16384, 128, 5), 148, False),
    # whole units per block: no split, no merge, no workspace
    "b8_n512_k8": ((8, 32, 32, 512, 128, 8), 64, True),      # 64 blocks of 4 tiles
    "b8_n512_k16": ((8, 32, 32, 512, 128, 16), 128, True),
    "b64_n512_k8": ((64, 32, 32, 512, 128, 8), 148, True),   # 3 or 4 units per block
    # each unit in p equal pieces of at least 3 tiles
    "b1_n1920_k24": ((1, 32, 32, 1920, 128, 24), 120, False),  # p = 5
    "b1_n8192_k32": ((1, 32, 32, 8192, 128, 32), 128, False),  # p = 4
    # pieces would leave too many SMs idle or be too short: the even cut
    "b1_n1920_k16": ((1, 32, 32, 1920, 128, 16), 148, False),
    "b1_n512_k32": ((1, 32, 32, 512, 128, 32), 128, False),    # one tile per block
}


@pytest.mark.parametrize("name", sorted(CUTS))
def test_cut_of_measured_shapes(name):
    args, blocks, whole = CUTS[name]
    p = sha.sha_decode_plan(*args, num_sms=148)
    assert p["blocks"] == blocks
    assert (p["workspace_bytes"] == 0) == whole


def test_forced_split_count_is_kept():
    p = sha.sha_decode_plan(4, 8, 8, 640, 128, 2, num_splits=7, num_sms=148)
    assert p["blocks"] == 7 and p["workspace_bytes"] > 0


@pytest.mark.parametrize("G", [1, 8])
@pytest.mark.parametrize("d", [64, 128])
def test_plan_invariants(G, d):
    for B in (1, 3, 8, 32, 64, 256):
        for N in (1, 100, 512, 1920, 4096, 16384):
            for k in (1, 4, 8):
                H_kv = 8
                p = sha.sha_decode_plan(B, G * H_kv, H_kv, N, d, k, num_sms=148)
                tiles = math.ceil(N / 128)
                assert p["tiles_per_head"] == tiles and p["tile_keys"] == 128
                assert p["total_tiles"] == B * k * tiles
                assert 1 <= p["blocks"] <= min(4096, p["total_tiles"])
                # a workspace, when needed, holds the counters and two slots per block
                ws = p["workspace_bytes"]
                slot_bytes = math.ceil(G * (d + 2) / 32) * 32 * 4
                assert ws == 0 or ws >= 4096 * 4 + 2 * p["blocks"] * slot_bytes


# Clusters of c blocks of the clustered kernel that fit on a B200 at once
# (cudaOccupancyMaxActiveClusters at its shared-memory size, one block per SM).
B200_CLUSTERS = {2: 74, 3: 45, 4: 33, 5: 26, 6: 22, 7: 15, 8: 15}

# (B, H_q, H_kv, N_kv, d, top_k) -> blocks per cluster, 0 = not clustered; the
# cuts measured fastest on B200 (CUDA-graph replay, inputs rotated past L2)
CLUSTERED = {
    "b1_n512_k8": ((1, 32, 32, 512, 128, 8), 4),        # 5.5 us; 8 whole units 6.6
    "b1_n512_k32": ((1, 32, 32, 512, 128, 32), 4),      # 6.5 us; even cut 8.5
    "b1_n1920_k8": ((1, 32, 32, 1920, 128, 8), 8),      # 7.0 us; even cut 10.5
    "b1_n1920_k32": ((1, 32, 32, 1920, 128, 32), 3),    # 10.1 us; pieces 13.4
    "b1_n8192_k8": ((1, 32, 32, 8192, 128, 8), 8),      # 11.4 us; even cut 14.6
    "b8_n1920_k8": ((8, 32, 32, 1920, 128, 8), 2),      # 14.4 us; pieces 17.8
    "llama31_70b_gqa_16k": ((8, 64, 8, 16384, 128, 5), 3),   # 51.3 us; even cut 56.5
    # a few units per block: clusters of 2, each block one whole unit and half of
    # a shared one (6 tiles), against two whole units on some blocks (8 tiles)
    "b8_n512_k24": ((8, 32, 32, 512, 128, 24), 2),
    # whole units win: short units with no idle SMs to gain
    "b8_n512_k8": ((8, 32, 32, 512, 128, 8), 0),        # 7.4 us; clusters of 2 7.8
    # more units than clusters fit at once: the planner's other cuts
    "b8_n1920_k16": ((8, 32, 32, 1920, 128, 16), 0),
    "opt66b": ((64, 72, 72, 1920, 128, 22), 0),
    "llama31_70b_gqa": ((32, 64, 8, 4096, 128, 5), 0),
    # the multi-head FMA kernel's calls (d = 64) and G > 8 are never clustered
    "mha_d64": ((1, 32, 32, 1920, 64, 8), 0),
    "gqa_g16": ((1, 64, 4, 4096, 128, 2), 0),
}


@pytest.mark.parametrize("name", sorted(CLUSTERED))
def test_clustered_cut_of_measured_shapes(name):
    args, cluster = CLUSTERED[name]
    p = sha.sha_decode_plan_ex(*args, num_sms=148, cluster_capacity=B200_CLUSTERS)
    assert p["cluster"] == cluster, p
    if cluster:
        units = args[0] * args[5]
        upc = p["units_per_cluster"]
        assert p["blocks"] == -(-units // upc) * cluster
        assert p["workspace_bytes"] == 0 and p["pieces"] == 0
        if name == "b8_n512_k24":
            assert (upc, p["whole_per_block"]) == (3, 1)
        else:
            assert (upc, p["whole_per_block"]) == (1, 0)
    else:
        # without the clustered cut the plan is sha_decode_plan's
        q = sha.sha_decode_plan(*args, num_sms=148)
        assert {k: p[k] for k in q} == q


def test_no_capacities_means_no_clustered_cut():
    p = sha.sha_decode_plan_ex(1, 32, 32, 1920, 128, 8, num_sms=148)
    assert p["cluster"] == 0
    assert {k: p[k] for k in ("blocks", "workspace_bytes")} == {
        k: sha.sha_decode_plan(1, 32, 32, 1920, 128, 8, num_sms=148)[k]
        for k in ("blocks", "workspace_bytes")}


def test_forced_split_count_never_clusters():
    p = sha.sha_decode_plan_ex(1, 32, 32, 1920, 128, 8, num_splits=64, num_sms=148,
                               cluster_capacity=B200_CLUSTERS)
    assert p["cluster"] == 0 and p["blocks"] == 64


@pytest.mark.parametrize("G", [1, 2, 5, 8])
@pytest.mark.parametrize("d", [64, 128])
def test_clustered_plan_invariants(G, d):
    for B in (1, 2, 4, 8):
        for N in (1, 129, 512, 1920, 8192, 16384):
            for k in (1, 3, 8):
                H_kv = 8
                p = sha.sha_decode_plan_ex(B, G * H_kv, H_kv, N, d, k, num_sms=148,
                                           cluster_capacity=B200_CLUSTERS)
                c = p["cluster"]
                if not c:
                    continue
                units = B * k
                upc, whole = p["units_per_cluster"], p["whole_per_block"]
                clusters = -(-units // upc)
                # one wave of clusters, each splitting at least one unit into
                # pieces of at least one tile
                assert 2 <= c <= 8 and c <= p["tiles_per_head"]
                assert clusters <= B200_CLUSTERS[c] and p["blocks"] == clusters * c
                assert 0 <= c * whole < upc
                assert G <= 8 and not (G == 1 and d == 64)
                assert p["workspace_bytes"] == 0
