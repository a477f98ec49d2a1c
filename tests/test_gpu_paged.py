"""Paged KV cache on the GPU (sha_decode_paged) against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import TOLERANCE, out_bits

pytestmark = pytest.mark.gpu
W = workloads.Workload


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


def _paged(w, page_size, seed, spare=5):
    """Seeded inputs with the cache scattered over a page pool in random order
    (plus `spare` unused pages filled with NaN)."""
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(1, w.N_kv + 1, (w.B,), generator=g, dtype=torch.int32)
    P = -(-w.N_kv // page_size)
    n_pages = w.B * P + spare
    perm = torch.randperm(n_pages, generator=g)
    kp = torch.full((n_pages, w.H_kv, page_size, w.d), float("nan"), dtype=k.dtype)
    vp = kp.clone()
    table = torch.empty((w.B, P), dtype=torch.int32)
    for b in range(w.B):
        for i in range(P):
            slot = int(perm[b * P + i])
            n = min(page_size, w.N_kv - i * page_size)
            kp[slot, :, :n] = k[b, :, i * page_size:i * page_size + n]
            vp[slot, :, :n] = v[b, :, i * page_size:i * page_size + n]
            table[b, i] = slot
    return q, kp, vp, idx, lens, table


def _run_and_check(sha, w, q, kp, vp, idx, lens, table):
    dev = torch.device("cuda")
    out = workloads.make_out(w, dev)
    sha.sha_decode_paged(q.to(dev), kp.to(dev), vp.to(dev), idx.to(dev), lens.to(dev),
                         table.to(dev), w.scale, out)
    torch.cuda.synchronize()
    status = sha.sha_get_device_status()
    want, bad = oracle.sha_decode_paged(q, kp, vp, idx.numpy(), lens.numpy(), table.numpy(),
                                        w.scale, w.dtype)
    written = ~np.isnan(want[..., 0])
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~written] == np.uint16(workloads.SENTINEL[w.dtype])).all()
    got = out.cpu().double().numpy()
    assert np.abs(got[written] - want[written]).max() <= TOLERANCE[w.dtype]
    return status, bad


@pytest.mark.parametrize("page_size", [1, 16, 100, 128, 256])
def test_paged_mha(sha, page_size):
    w = W("pg_mha", B=5, H_q=8, H_kv=8, N_kv=600, d=128, top_k=3, dtype="fp16",
          seed=100 + page_size)
    status, bad = _run_and_check(sha, w, *_paged(w, page_size, w.seed))
    assert status == sha.SHA_OK and bad == 0


@pytest.mark.parametrize("page_size", [8, 16, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_paged_gqa(sha, page_size, d):
    w = W("pg_gqa", B=4, H_q=32, H_kv=4, N_kv=700, d=d, top_k=2, dtype="bf16",
          seed=200 + page_size + d)
    status, bad = _run_and_check(sha, w, *_paged(w, page_size, w.seed))
    assert status == sha.SHA_OK and bad == 0


def test_paged_bad_page_id_is_flagged(sha):
    w = W("pg_bad", B=3, H_q=8, H_kv=8, N_kv=256, d=128, top_k=2, dtype="fp16", seed=301)
    q, kp, vp, idx, lens, table = _paged(w, 64, w.seed)
    lens[1] = 200
    table[1, 2] = 10_000                              # needed by row 1
    dev = torch.device("cuda")
    out = workloads.make_out(w, dev)
    sha.sha_decode_paged(q.to(dev), kp.to(dev), vp.to(dev), idx.to(dev), lens.to(dev),
                         table.to(dev), w.scale, out)
    assert sha.sha_get_device_status() == sha.SHA_ERR_BAD_INDEX
    # the other rows are still right
    want, bad = oracle.sha_decode_paged(q, kp, vp, idx.numpy(), lens.numpy(), table.numpy(),
                                        w.scale, w.dtype)
    got = out.cpu().double().numpy()
    for b in (0, 2):
        for h in idx[b].tolist():
            assert np.abs(got[b, h] - want[b, h]).max() <= TOLERANCE[w.dtype]


def test_gqa_page_size_must_be_a_power_of_two(sha):
    w = W("pg_ps", B=1, H_q=8, H_kv=2, N_kv=48, d=128, top_k=1, dtype="bf16", seed=302)
    q, kp, vp, idx, lens, table = _paged(w, 12, w.seed)
    dev = torch.device("cuda")
    with pytest.raises(sha.ShaError) as e:
        sha.sha_decode_paged(q.to(dev), kp.to(dev), vp.to(dev), idx.to(dev), lens.to(dev),
                             table.to(dev), w.scale, workloads.make_out(w, dev))
    assert e.value.status == sha.SHA_ERR_UNSUPPORTED
