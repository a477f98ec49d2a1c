"""Strided K/V caches (sha_decode_strided) against the float64 oracle: a
token-major cache [B, N, H_kv, d], a head-major cache padded past N_kv, and
the K and V views of one fused buffer [B, N, 2, H_kv, d]; the oracle reads
contiguous copies of the same values."""
import numpy as np
import pytest
import torch

import workloads
from parity import check_against_oracle

pytestmark = pytest.mark.gpu
W = workloads.Workload


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


CASES = [
    W("tok_mha", B=3, H_q=8, H_kv=8, N_kv=1000, d=128, top_k=3, dtype="fp16", seed=301),
    W("tok_mha_d64", B=2, H_q=6, H_kv=6, N_kv=333, d=64, top_k=4, dtype="bf16", seed=302),
    W("tok_gqa", B=3, H_q=64, H_kv=8, N_kv=777, d=128, top_k=5, dtype="bf16", seed=303),
    W("tok_gqa_d64", B=2, H_q=16, H_kv=4, N_kv=129, d=64, top_k=2, dtype="fp16", seed=304),
]


def _decode(sha, w, q, k, v, idx):
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_strided(q, k, v, idx, w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    return out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_token_major_cache(sha, w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    # the same values stored token-major: [B, N, H_kv, d]
    k_tok = k.permute(0, 2, 1, 3).contiguous().to(dev)
    v_tok = v.permute(0, 2, 1, 3).contiguous().to(dev)
    out = _decode(sha, w, q.to(dev), k_tok.permute(0, 2, 1, 3), v_tok.permute(0, 2, 1, 3),
                  idx.to(dev))
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("w", CASES[:3], ids=lambda w: w.name)
def test_padded_head_major_cache(sha, w):
    """Each (row, head) block is N_max = N_kv + 61 keys long; the keys past N_kv
    hold NaN and must never be read into the result."""
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    n_max = w.N_kv + 61
    k_pad = torch.full((w.B, w.H_kv, n_max, w.d), float("nan"), dtype=k.dtype)
    v_pad = torch.full_like(k_pad, float("nan"))
    k_pad[:, :, :w.N_kv] = k
    v_pad[:, :, :w.N_kv] = v
    k_pad, v_pad = k_pad.to(dev), v_pad.to(dev)
    out = _decode(sha, w, q.to(dev), k_pad[:, :, :w.N_kv], v_pad[:, :, :w.N_kv], idx.to(dev))
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("w", [CASES[0], CASES[2]], ids=lambda w: w.name)
def test_fused_kv_buffer(sha, w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    kv = torch.stack((k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3)), dim=2).contiguous().to(dev)
    out = _decode(sha, w, q.to(dev), kv[:, :, 0].permute(0, 2, 1, 3),
                  kv[:, :, 1].permute(0, 2, 1, 3), idx.to(dev))
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("w", [CASES[0], CASES[2]], ids=lambda w: w.name)
def test_contiguous_strides_match_sha_decode_bit_for_bit(sha, w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    q, k, v, idx = q.to(dev), k.to(dev), v.to(dev), idx.to(dev)
    a = _decode(sha, w, q, k, v, idx)
    b = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, b)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_k_and_v_strides_must_rank_alike(sha):
    w = CASES[0]
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    k_tok = k.permute(0, 2, 1, 3).contiguous().to(dev).permute(0, 2, 1, 3)   # token-major
    out = workloads.make_out(w, "cuda")
    with pytest.raises(sha.ShaError) as e:
        sha.sha_decode_strided(q.to(dev), k_tok, v.to(dev), idx.to(dev), w.scale, out)
    assert e.value.status == sha.SHA_ERR_UNSUPPORTED
    bits = out.cpu().view(torch.int16).numpy().view(np.uint16)
    assert (bits == workloads.SENTINEL[w.dtype]).all()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_token_major_cache_with_row_lengths(sha, w):
    """Token-major cache, row b using its first seqlens[b] keys; keys at or past a
    row's length hold NaN and must never reach the result."""
    import oracle
    from parity import TOLERANCE, out_bits

    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    g = torch.Generator().manual_seed(w.seed + 5)
    lens = torch.randint(1, w.N_kv + 1, (w.B,), generator=g, dtype=torch.int32)
    lens[0] = 1
    lens[-1] = w.N_kv
    k_poison, v_poison = k.clone(), v.clone()
    for b in range(w.B):
        k_poison[b, :, int(lens[b]):] = float("nan")
        v_poison[b, :, int(lens[b]):] = float("nan")
    dev = torch.device("cuda")
    k_tok = k_poison.permute(0, 2, 1, 3).contiguous().to(dev).permute(0, 2, 1, 3)
    v_tok = v_poison.permute(0, 2, 1, 3).contiguous().to(dev).permute(0, 2, 1, 3)
    out = workloads.make_out(w, "cuda")
    sha.sha_decode_strided(q.to(dev), k_tok, v_tok, idx.to(dev), w.scale, out,
                           seqlens=lens.to(dev))
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    want, bad = oracle.sha_decode_varlen(q, k, v, idx.numpy(), lens.numpy(), w.scale, w.dtype)
    assert bad == 0
    written = ~np.isnan(want[..., 0])
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~written] == np.uint16(workloads.SENTINEL[w.dtype])).all()
    got = out.cpu().double().numpy()
    assert np.isfinite(got[written]).all()
    assert np.abs(got[written] - want[written]).max() <= TOLERANCE[w.dtype]
