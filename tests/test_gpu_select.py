"""Device head selection (router scores -> batch_head_index) against the oracle:
integers, so bit-exact; and selection followed by decode on one stream."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_against_oracle, out_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


@pytest.mark.parametrize("B,H,top_k", [(64, 72, 22), (128, 32, 16), (32, 8, 5), (7, 256, 100),
                                       (5, 1, 1), (300, 33, 33), (9, 200, 1)])
@pytest.mark.parametrize("ties", [False, True])
def test_select_heads_bit_exact(sha, B, H, top_k, ties):
    g = torch.Generator().manual_seed(B * 7 + H)
    if ties:
        scores = torch.randint(-3, 4, (B, H), generator=g).float()
    else:
        scores = torch.randn((B, H), generator=g)
    if H > 2:
        scores[0, 1] = float("-inf")
        scores[-1, 0] = float("inf")
    got = sha.sha_select_heads(scores.cuda(), top_k)
    torch.cuda.synchronize()
    want = oracle.select_heads(scores.numpy(), top_k)
    assert np.array_equal(got.cpu().numpy(), want)


def test_select_then_decode_on_one_stream(sha):
    w = workloads.CONFIGS["opt66b"].with_(B=8, N_kv=700, seed=71)
    q, k, v = workloads.make_qkv(w)
    scores = torch.randn((w.B, w.H_kv), generator=torch.Generator().manual_seed(72))
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = workloads.make_out(w, dev)
    out, idx = sha.decode_from_scores(qd, kd, vd, scores.to(dev), w.top_k, w.scale, out)
    torch.cuda.synchronize()
    want_idx = oracle.select_heads(scores.numpy(), w.top_k)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    check_against_oracle(w, qd, kd, vd, torch.from_numpy(want_idx), out)
    # the same index given directly gives the same bits
    out2 = workloads.make_out(w, dev)
    sha.decode(qd, kd, vd, torch.from_numpy(want_idx).to(dev), w.scale, out2)
    torch.cuda.synchronize()
    assert np.array_equal(out_bits(out), out_bits(out2))


def test_select_groups_for_gqa(sha):
    w = workloads.CONFIGS["llama31_70b_gqa"].with_(N_kv=500, seed=73)
    q, k, v = workloads.make_qkv(w)
    scores = torch.randn((w.B, w.H_kv), generator=torch.Generator().manual_seed(74))
    dev = torch.device("cuda")
    out = workloads.make_out(w, dev)
    out, idx = sha.decode_from_scores(q.to(dev), k.to(dev), v.to(dev), scores.to(dev),
                                      w.top_k, w.scale, out)
    torch.cuda.synchronize()
    want_idx = oracle.select_heads(scores.numpy(), w.top_k)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    check_against_oracle(w, q, k, v, torch.from_numpy(want_idx), out)
