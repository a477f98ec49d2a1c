"""Head x token sparsity on the GPU (sha_decode_tokens) against the float64
oracle: each selected unit attends only to its listed keys."""
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


def _run(sha, w, q, k, v, idx, tok):
    dev = torch.device("cuda")
    out = workloads.make_out(w, dev)
    sha.sha_decode_tokens(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), tok.to(dev), w.scale, out)
    torch.cuda.synchronize()
    return out, sha.sha_get_device_status()


def _check(w, q, k, v, idx, tok, out, skip=()):
    want, _ = oracle.sha_decode_tokens(q, k, v, idx.numpy(), tok.numpy(), w.scale, w.dtype)
    mask = active_mask(idx.numpy(), w.B, w.H_kv, w.G)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == np.uint16(workloads.SENTINEL[w.dtype])).all(), "an inactive row was written"
    for b, s in skip:                      # units whose output is unspecified
        h = int(idx[b, s])
        mask[b, h * w.G:(h + 1) * w.G] = False
    got = out.cpu().double().numpy()
    err = np.abs(got[mask] - want[mask]).max()
    assert err <= TOLERANCE[w.dtype], err
    return err


# (workload, keys per unit): several tiles and a ragged last one, one tile,
# a single key, more keys than the cache holds (repeats), G = 1 / 3 / 8
CASES = [
    (W("t_mha", B=4, H_q=16, H_kv=16, N_kv=1000, d=128, top_k=4, dtype="fp16", seed=801), 300),
    (W("t_mha_d64", B=3, H_q=8, H_kv=8, N_kv=777, d=64, top_k=3, dtype="bf16", seed=802), 77),
    (W("t_gqa8", B=2, H_q=64, H_kv=8, N_kv=2000, d=128, top_k=5, dtype="bf16", seed=803), 1000),
    (W("t_gqa3_d64", B=5, H_q=12, H_kv=4, N_kv=300, d=64, top_k=2, dtype="fp16", seed=804), 129),
    (W("t_one_key", B=3, H_q=8, H_kv=8, N_kv=500, d=128, top_k=2, dtype="fp16", seed=805), 1),
    (W("t_repeats", B=2, H_q=8, H_kv=8, N_kv=100, d=128, top_k=3, dtype="fp16", seed=806), 257),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_tokens_match_oracle(sha, case):
    w, n_sel = case
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    tok = workloads.make_tokens(w, n_sel)
    out, status = _run(sha, w, q, k, v, idx, tok)
    assert status == sha.SHA_OK
    _check(w, q, k, v, idx, tok, out)


def test_every_key_in_order_is_the_full_decode(sha):
    w = W("t_full", B=3, H_q=16, H_kv=16, N_kv=700, d=128, top_k=5, dtype="fp16", seed=807)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    tok = torch.arange(w.N_kv, dtype=torch.int32).expand(w.B, w.top_k, -1).contiguous()
    out, status = _run(sha, w, q, k, v, idx, tok)
    assert status == sha.SHA_OK
    _check(w, q, k, v, idx, tok, out)
    dev = torch.device("cuda")
    full = workloads.make_out(w, dev)
    sha.decode(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), w.scale, full)
    torch.cuda.synchronize()
    m = ~torch.isnan(full.double())
    assert float((out.double() - full.double()).abs()[m].max()) <= TOLERANCE[w.dtype]


def test_repeat_calls_bit_identical_and_unlisted_keys_unread(sha):
    # unlisted keys hold NaN: a single one read would poison its unit
    w = W("t_nan", B=3, H_q=32, H_kv=8, N_kv=900, d=128, top_k=4, dtype="bf16", seed=808)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    tok = workloads.make_tokens(w, 333)
    listed = torch.zeros((w.B, w.H_kv, w.N_kv), dtype=torch.bool)
    for b in range(w.B):
        for s in range(w.top_k):
            listed[b, int(idx[b, s]), tok[b, s].long()] = True
    k_nan, v_nan = k.clone(), v.clone()
    k_nan[~listed] = float("nan")
    v_nan[~listed] = float("nan")
    a, st_a = _run(sha, w, q, k_nan, v_nan, idx, tok)
    b, st_b = _run(sha, w, q, k_nan, v_nan, idx, tok)
    assert st_a == st_b == sha.SHA_OK
    assert np.array_equal(out_bits(a), out_bits(b))
    _check(w, q, k, v, idx, tok, a)


def test_out_of_range_positions_flagged_and_others_exact(sha):
    w = W("t_bad", B=3, H_q=16, H_kv=16, N_kv=600, d=128, top_k=3, dtype="fp16", seed=809)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    tok = workloads.make_tokens(w, 200)
    tok[0, 1, 17] = w.N_kv
    tok[2, 2, 0] = -5
    out, status = _run(sha, w, q, k, v, idx, tok)
    assert status == sha.SHA_ERR_BAD_INDEX
    _check(w, q, k, v, idx, tok, out, skip=((0, 1), (2, 2)))


def test_argument_checks(sha):
    w = W("t_args", B=2, H_q=8, H_kv=8, N_kv=64, d=128, top_k=2, dtype="fp16", seed=810)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    out = workloads.make_out(w, dev)
    empty = torch.zeros((w.B, w.top_k, 0), dtype=torch.int32, device=dev)
    with pytest.raises(sha.ShaError) as e:
        sha.sha_decode_tokens(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), empty, w.scale, out)
    assert e.value.status == sha.SHA_ERR_INVALID_ARG
    assert (out_bits(out) == np.uint16(workloads.SENTINEL["fp16"])).all()


def test_opt66b_shape_quarter_of_the_keys_sampled_units(sha):
    # the OPT-66B step with each selected head keeping a quarter of its keys
    w = workloads.CONFIGS["opt66b"]
    dev = torch.device("cuda")
    q, k, v = workloads.make_qkv(w, device=dev)
    idx = workloads.make_index(w)
    tok = workloads.make_tokens(w, w.N_kv // 4)
    out = workloads.make_out(w, dev)
    sha.sha_decode_tokens(q, k, v, idx.to(dev), tok.to(dev), w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    mask = active_mask(idx.numpy(), w.B, w.H_kv, w.G)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == np.uint16(workloads.SENTINEL[w.dtype])).all()
    rng = np.random.default_rng(3)
    units = [(int(u) // w.top_k, int(u) % w.top_k)
             for u in rng.choice(w.units, size=48, replace=False)]
    qu = torch.stack([q[b, idx[b, s]].cpu().unsqueeze(0) for b, s in units])
    ku = torch.stack([k[b, idx[b, s]][tok[b, s].long().to(dev)].cpu() for b, s in units])
    vu = torch.stack([v[b, idx[b, s]][tok[b, s].long().to(dev)].cpu() for b, s in units])
    ref = oracle.sha_units(qu, ku, vu, w.scale, w.dtype)
    got = out.cpu().double().numpy()
    err = max(float(np.abs(got[b, int(idx[b, s])] - ref[i][0]).max())
              for i, (b, s) in enumerate(units))
    assert err <= TOLERANCE[w.dtype], err
