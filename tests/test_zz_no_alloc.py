"""sha_decode_noalloc: the decode for callers that cannot allocate device memory
(an engine whose allocator owns all of HBM, a step that must not pay for
cudaMalloc).  Its split-merge scratch is a fixed array inside the library; the
result must match the ordinary entry point's, call after call, since each call
reuses the array the previous one left behind.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process."""
import pytest
import torch

import workloads
from parity import TOLERANCE, check_against_oracle, out_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


def _inputs(w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    return q.cuda(), k.cuda(), v.cuda(), idx.cuda()


def _plan_on_device(sha, w, num_splits=0):
    props = torch.cuda.get_device_properties(0)
    return sha.sha_decode_plan_ex(w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k, num_splits,
                                  num_sms=props.multi_processor_count,
                                  cluster_capacity=sha.sha_decode_cluster_capacity(w.d))


def _check_twice(sha, shapes):
    dtype = shapes[0].dtype
    for w in shapes:
        # heads straddle thread blocks and merge through the static scratch
        plan = _plan_on_device(sha, w)
        assert plan["cluster"] == 0 and plan["workspace_bytes"] > 0, plan
    for w in shapes:                   # calls in a row through the static scratch
        q, k, v, idx = _inputs(w)
        ref = workloads.make_out(w, "cuda")
        sha.decode(q, k, v, idx, w.scale, ref)
        got = workloads.make_out(w, "cuda")
        sha.sha_decode_noalloc(q, k, v, idx, w.scale, got)
        torch.cuda.synchronize()
        assert sha.sha_get_device_status() == sha.SHA_OK
        written = out_bits(ref) != workloads.SENTINEL[dtype]
        assert (out_bits(got)[~written] == workloads.SENTINEL[dtype]).all()
        diff = (got.double() - ref.double()).abs().cpu().numpy()[written]
        assert diff.max() <= TOLERANCE[dtype]
        check_against_oracle(w, q, k, v, idx, got)


@pytest.mark.parametrize("dtype,d", [("fp16", 128), ("bf16", 64)])
def test_noalloc_matches_the_allocating_entry_point_twice(sha, dtype, d):
    # more units than SMs, over 32 tiles per block: the even tile cut, units
    # split between neighbouring blocks
    first = workloads.Workload("noalloc_a", B=32, H_q=16, H_kv=16, N_kv=4000, d=d, top_k=5,
                               dtype=dtype, seed=51)
    second = first.with_(name="noalloc_b", B=24, N_kv=3777, top_k=7, seed=52)
    _check_twice(sha, [first, second])


def test_noalloc_on_chip_merge_twice(sha):
    # 256 units of 16 tiles over 148 blocks, about 28 tiles each: every split
    # unit meets 2 blocks, which selects the kernel build that finishes a
    # block's last split unit on chip, copying its partner's state out of the
    # static scratch
    w = workloads.Workload("noalloc_scout", B=16, H_q=32, H_kv=32, N_kv=2048, d=128,
                           top_k=16, dtype="fp16", seed=54)
    _check_twice(sha, [w, w.with_(name="noalloc_scout_b", seed=55)])


def test_noalloc_rejects_scratch_beyond_its_limit(sha):
    w = workloads.Workload("noalloc_big", B=4, H_q=8, H_kv=8, N_kv=4096, d=128, top_k=8,
                           dtype="fp16", seed=53)
    q, k, v, idx = _inputs(w)
    out = workloads.make_out(w, "cuda")
    splits = 1000       # 2000 partial states of 640 B: beyond the 512 KiB array
    assert _plan_on_device(sha, w, splits)["workspace_bytes"] > sha.NOALLOC_SCRATCH_BYTES
    with pytest.raises(sha.ShaError) as err:
        sha.sha_decode_noalloc(q, k, v, idx, w.scale, out, num_splits=splits)
    assert err.value.status == sha.SHA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out_bits(out) == workloads.SENTINEL["fp16"]).all()
