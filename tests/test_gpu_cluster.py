"""GPU parity of the clustered cut: units split across the blocks of a
thread-block cluster and merged in distributed shared memory, against the
float64 oracle, called through the C ABI (ctypes binding)."""
import numpy as np
import pytest
import torch

import workloads
from parity import TOLERANCE, check_against_oracle, out_bits

pytestmark = pytest.mark.gpu

W = workloads.Workload


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


def _on_gpu(w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    return q.to(dev), k.to(dev), v.to(dev), idx.to(dev)


def _clustered(sha, w, q, k, v, idx, cluster, upc, whole=0):
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_clustered(q, k, v, idx, w.scale, out, cluster, upc, whole)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    return out


# (workload, cluster sizes, units per cluster): several tiles per piece and a
# ragged last tile, pieces of one tile, G = 1 / 3 / 8, both dtypes, d = 64 / 128
CASES = [
    (W("c_mha", B=1, H_q=32, H_kv=32, N_kv=1920, d=128, top_k=8, dtype="fp16", seed=401),
     (2, 3, 4, 5, 6, 7, 8), (1, 3)),
    (W("c_mha_ragged", B=3, H_q=16, H_kv=16, N_kv=1000, d=128, top_k=5, dtype="bf16", seed=402),
     (2, 3, 8), (1, 2, 15)),
    (W("c_one_tile_pieces", B=2, H_q=8, H_kv=8, N_kv=300, d=128, top_k=4, dtype="fp16", seed=403),
     (2, 3), (1, 4)),
    (W("c_gqa8", B=2, H_q=64, H_kv=8, N_kv=1000, d=128, top_k=5, dtype="bf16", seed=404),
     (2, 4, 8), (1, 2, 10)),
    (W("c_gqa3", B=4, H_q=12, H_kv=4, N_kv=777, d=128, top_k=3, dtype="fp16", seed=405),
     (2, 5), (1, 4)),
    (W("c_gqa4_d64", B=3, H_q=16, H_kv=4, N_kv=1500, d=64, top_k=2, dtype="fp16", seed=406),
     (2, 7), (1, 3)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_clustered_matches_oracle(sha, case):
    w, clusters, upcs = case
    q, k, v, idx = _on_gpu(w)
    expected = None
    for c in clusters:
        for upc in upcs:
            out = _clustered(sha, w, q, k, v, idx, c, upc)
            check_against_oracle(w, q, k, v, idx, out, expected)


# (workload, cluster, units per cluster, whole units per block): clusters
# that hold whole units besides the ones they split, and a ragged last cluster
MIXED = [
    (W("m_mha", B=8, H_q=32, H_kv=32, N_kv=512, d=128, top_k=24, dtype="fp16", seed=421),
     2, 3, 1),
    (W("m_mha_ragged", B=5, H_q=16, H_kv=16, N_kv=900, d=128, top_k=7, dtype="bf16", seed=422),
     3, 8, 2),
    (W("m_gqa8", B=4, H_q=64, H_kv=8, N_kv=1000, d=128, top_k=5, dtype="bf16", seed=423),
     2, 5, 2),
    (W("m_gqa2_d64", B=6, H_q=8, H_kv=4, N_kv=700, d=64, top_k=3, dtype="fp16", seed=424),
     4, 7, 1),
    (W("m_all_whole", B=6, H_q=8, H_kv=8, N_kv=300, d=128, top_k=4, dtype="fp16", seed=425),
     2, 4, 2),
]


@pytest.mark.parametrize("case", MIXED, ids=lambda c: c[0].name)
def test_mixed_clustered_matches_oracle(sha, case):
    w, c, upc, whole = case
    q, k, v, idx = _on_gpu(w)
    for _ in range(2):                      # repeated calls reuse the cluster barriers
        out = _clustered(sha, w, q, k, v, idx, c, upc, whole)
        check_against_oracle(w, q, k, v, idx, out)


def test_clustered_repeat_bit_identical(sha):
    w = CASES[0][0]
    q, k, v, idx = _on_gpu(w)
    a = _clustered(sha, w, q, k, v, idx, 4, 2)
    b = _clustered(sha, w, q, k, v, idx, 4, 2)
    assert np.array_equal(out_bits(a), out_bits(b))


def test_clustered_beyond_capacity_runs_in_waves(sha):
    # 4096 blocks in clusters of 2: far more than fit on the device at once
    w = W("c_waves", B=64, H_q=32, H_kv=32, N_kv=256, d=128, top_k=32, dtype="fp16", seed=407)
    q, k, v, idx = _on_gpu(w)
    out = _clustered(sha, w, q, k, v, idx, 2, 1)
    check_against_oracle(w, q, k, v, idx, out)


def test_clustered_bad_ids_skipped_and_flagged(sha):
    w = W("c_bad", B=2, H_q=16, H_kv=16, N_kv=700, d=128, top_k=4, dtype="fp16", seed=408)
    q, k, v, idx = _on_gpu(w)
    idx[0, 1] = 99
    idx[1, 3] = -2
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_clustered(q, k, v, idx, w.scale, out, 3, 2)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_ERR_BAD_INDEX
    check_against_oracle(w, q, k, v, idx, out)      # the skipped slots write nothing


def test_clustered_argument_checks(sha):
    w = W("c_args", B=1, H_q=8, H_kv=8, N_kv=300, d=128, top_k=2, dtype="fp16", seed=409)
    q, k, v, idx = _on_gpu(w)
    out = workloads.make_out(w, "cuda")
    for c, upc, whole, status in ((1, 1, 0, sha.SHA_ERR_INVALID_ARG),
                                  (9, 1, 0, sha.SHA_ERR_INVALID_ARG),
                                  (4, 1, 0, sha.SHA_ERR_INVALID_ARG),   # 3 tiles: at most 3 pieces
                                  (2, 0, 0, sha.SHA_ERR_INVALID_ARG),
                                  (2, 3, 2, sha.SHA_ERR_INVALID_ARG),   # 4 whole units > 3
                                  (2, 1, -1, sha.SHA_ERR_INVALID_ARG)):
        with pytest.raises(sha.ShaError) as e:
            sha.sha_decode_clustered(q, k, v, idx, w.scale, out, c, upc, whole)
        assert e.value.status == status
    # clusters of 4 whose units all go whole need no piece per tile
    sha.sha_decode_clustered(q, k, v, idx, w.scale, out, 4, 4, 1)
    check_against_oracle(w, q, k, v, idx, out)
    # the multi-head FMA kernel's calls (d = 64, G = 1) and G > 8 are not served
    w64 = w.with_(d=64)
    q6, k6, v6, i6 = _on_gpu(w64)
    with pytest.raises(sha.ShaError) as e:
        sha.sha_decode_clustered(q6, k6, v6, i6, w64.scale, workloads.make_out(w64, "cuda"), 2, 1)
    assert e.value.status == sha.SHA_ERR_UNSUPPORTED
    w16 = W("c_g16", B=1, H_q=32, H_kv=2, N_kv=300, d=128, top_k=1, dtype="bf16", seed=410)
    q16, k16, v16, i16 = _on_gpu(w16)
    with pytest.raises(sha.ShaError) as e:
        sha.sha_decode_clustered(q16, k16, v16, i16, w16.scale, workloads.make_out(w16, "cuda"),
                                 2, 1)
    assert e.value.status == sha.SHA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK


def test_capacity_and_planner_choice(sha):
    caps = sha.sha_decode_cluster_capacity(128)
    assert caps[2] >= 1, caps
    assert all(caps[c] >= caps[c + 1] for c in range(2, 8)), caps
    # a short call the planner sends to the clustered cut on this device runs it
    w = workloads.sweep(1, 1920, 8)
    plan = sha.sha_decode_plan_ex(w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k,
                                  num_sms=torch.cuda.get_device_properties(0).multi_processor_count,
                                  cluster_capacity=caps)
    assert plan["cluster"] >= 2 and plan["workspace_bytes"] == 0, plan
    q, k, v, idx = _on_gpu(w)
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    check_against_oracle(w, q, k, v, idx, out)
    forced = _clustered(sha, w, q, k, v, idx, plan["cluster"], plan["units_per_cluster"],
                        plan["whole_per_block"])
    assert np.array_equal(out_bits(out), out_bits(forced))


def test_clustered_within_tolerance_of_even_cut(sha):
    w = W("c_vs_even", B=2, H_q=32, H_kv=32, N_kv=4096, d=128, top_k=6, dtype="bf16", seed=411)
    q, k, v, idx = _on_gpu(w)
    even = workloads.make_out(w, "cuda")
    ws = sha.alloc_workspace(q, k, idx, 148)
    sha.sha_decode_ex(q, k, v, idx, w.scale, even, ws, 148)
    clustered = _clustered(sha, w, q, k, v, idx, 8, 1)
    diff = (even.double() - clustered.double()).abs()
    active = ~torch.isnan(even.double())
    assert float(diff[active].max()) <= TOLERANCE[w.dtype]
