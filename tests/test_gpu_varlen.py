"""Per-row cache lengths on the GPU against the float64 oracle (sha_decode_varlen)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import TOLERANCE, active_mask, out_bits

pytestmark = pytest.mark.gpu
W = workloads.Workload


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


def _inputs(w, device="cuda"):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    return q.to(device), k.to(device), v.to(device), idx.to(device)


def _lengths(w, seed, lo=1):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, w.N_kv + 1, (w.B,), generator=g, dtype=torch.int32)


def _check(w, q, k, v, idx, lens, out):
    want, bad = oracle.sha_decode_varlen(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(),
                                         lens.cpu().numpy(), w.scale, w.dtype)
    written = ~np.isnan(want[..., 0])
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~written] == np.uint16(workloads.SENTINEL[w.dtype])).all()
    got = out.cpu().double().numpy()
    err = np.abs(got[written] - want[written]).max()
    assert err <= TOLERANCE[w.dtype], err
    return bad


CASES = [
    W("vl_mha", B=6, H_q=8, H_kv=8, N_kv=700, d=128, top_k=3, dtype="fp16", seed=81),
    W("vl_mha64", B=9, H_q=6, H_kv=6, N_kv=300, d=64, top_k=2, dtype="bf16", seed=82),
    W("vl_gqa", B=5, H_q=32, H_kv=4, N_kv=900, d=128, top_k=2, dtype="bf16", seed=83),
    W("vl_gqa64", B=4, H_q=16, H_kv=8, N_kv=260, d=64, top_k=3, dtype="fp16", seed=84),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_varlen_parity(sha, w):
    q, k, v, idx = _inputs(w)
    lens = _lengths(w, w.seed)
    lens[0] = 1
    lens[-1] = w.N_kv
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_varlen(q, k, v, idx, lens.cuda(), w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    assert _check(w, q, k, v, idx, lens, out) == 0


@pytest.mark.parametrize("w", [CASES[1], CASES[2]], ids=lambda w: w.name)
def test_full_lengths_reproduce_the_fixed_length_bits(sha, w):
    """With every length = N_max the kernel plans the same split as the
    fixed-length path and runs the same kernel, so the results are
    bit-identical.  (Multi-head calls with d = 128 run on the tensor-core
    kernel at fixed lengths and on the FMA kernel with per-row lengths.)"""
    q, k, v, idx = _inputs(w)
    a = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, a)
    b = workloads.make_out(w, "cuda")
    lens = torch.full((w.B,), w.N_kv, dtype=torch.int32, device="cuda")
    sha.sha_decode_varlen(q, k, v, idx, lens, w.scale, b)
    torch.cuda.synchronize()
    assert np.array_equal(out_bits(a), out_bits(b))


def test_full_lengths_multi_head_d128_match_the_oracle(sha):
    """The d = 128 multi-head case of the test above: the two calls run on
    different kernels, so each is held to the oracle instead of to the other."""
    w = CASES[0]
    q, k, v, idx = _inputs(w)
    lens = torch.full((w.B,), w.N_kv, dtype=torch.int32)
    b = workloads.make_out(w, "cuda")
    sha.sha_decode_varlen(q, k, v, idx, lens.cuda(), w.scale, b)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    assert _check(w, q, k, v, idx, lens, b) == 0


@pytest.mark.parametrize("w", [CASES[1], CASES[2]], ids=lambda w: w.name)
def test_keys_past_a_row_length_are_never_used(sha, w):
    """The cache past each row's length holds NaN; results are unaffected."""
    q, k, v, idx = _inputs(w)
    lens = _lengths(w, w.seed + 1)
    k2, v2 = k.clone(), v.clone()
    for b, L in enumerate(lens.tolist()):
        k2[b, :, L:] = float("nan")
        v2[b, :, L:] = float("nan")
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_varlen(q, k2, v2, idx, lens.cuda(), w.scale, out)
    torch.cuda.synchronize()
    assert _check(w, q, k, v, idx, lens, out) == 0


def test_rows_with_bad_lengths_are_skipped(sha):
    w = CASES[0]
    q, k, v, idx = _inputs(w)
    lens = _lengths(w, 85)
    lens[1] = 0
    lens[3] = w.N_kv + 5
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_varlen(q, k, v, idx, lens.cuda(), w.scale, out)
    assert sha.sha_get_device_status() == sha.SHA_ERR_BAD_INDEX
    assert _check(w, q, k, v, idx, lens, out) == 2 * w.top_k


def test_varlen_large_batch_sampled(sha):
    """A decode batch of 128 rows with lengths spread over [1, 4096]."""
    w = workloads.CONFIGS["llama2_7b"].with_(N_kv=4096, seed=86)
    q, k, v = workloads.make_qkv(w, device="cuda")
    idx = workloads.make_index(w).cuda()
    lens = _lengths(w, 87)
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_varlen(q, k, v, idx, lens.cuda(), w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    idx_h = idx.cpu().numpy()
    mask = active_mask(idx_h, w.B, w.H_kv, 1)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == np.uint16(workloads.SENTINEL[w.dtype])).all()
    got = out.cpu().double().numpy()
    rng = np.random.default_rng(0)
    rows = sorted(set(rng.choice(w.B, 12, replace=False).tolist()) | {0, w.B - 1})
    for b in rows:
        L = int(lens[b])
        kt, vt = k[b:b + 1, :, :L].cpu().contiguous(), v[b:b + 1, :, :L].cpu().contiguous()
        ref, _ = oracle.sha_decode(q[b:b + 1].cpu(), kt, vt, idx_h[b:b + 1], w.scale, w.dtype)
        for h in idx_h[b]:
            assert np.abs(got[b, h] - ref[0, h]).max() <= TOLERANCE[w.dtype]
