"""Seeded random shapes against the float64 oracle: decode (G = 1..16, d = 64 /
128, ragged key counts, top_k from 0 to H_kv, automatic and forced splits), head
x token sparsity (random list lengths, repeats past the cache), and the
Selective GEMM (batch 1..64 on both GEMM paths, ragged neuron counts, unions from
almost empty to full, both activations)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_against_oracle, check_sampled_units, mlp_excess

pytestmark = pytest.mark.gpu
W = workloads.Workload
M = workloads.MlpWorkload


def _decode_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        G = int(rng.choice([1, 1, 2, 4, 8, 16]))
        H_kv = int(rng.integers(1, 17)) if G < 16 else int(rng.integers(1, 5))
        d = int(rng.choice([64, 128]))
        N_kv = int(rng.integers(1, 3001))
        top_k = int(rng.integers(1, H_kv + 1)) if rng.random() > 0.1 else 0
        B = int(rng.integers(1, 13))
        dtype = str(rng.choice(["fp16", "bf16"]))
        splits = int(rng.choice([0, 0, int(rng.integers(1, 400))]))
        cases.append((W(f"rand{i}_B{B}_G{G}_Hkv{H_kv}_N{N_kv}_d{d}_k{top_k}_{dtype}", B=B,
                        H_q=G * H_kv, H_kv=H_kv, N_kv=N_kv, d=d, top_k=top_k, dtype=dtype,
                        seed=9000 + i), splits))
    return cases


def _split_regime_cases(n, seed):
    """More units than blocks and units a few tiles long: the even tile cut, with
    most blocks ending on the head of a unit split in two (merged on chip)."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        G = int(rng.integers(1, 9))
        H_kv = int(rng.choice([4, 8, 16]))
        d = int(rng.choice([64, 128]))
        N_kv = int(rng.integers(600, 3001))
        top_k = int(rng.integers(max(1, H_kv // 2), H_kv + 1))
        B = int(rng.integers(16, 49))
        dtype = str(rng.choice(["fp16", "bf16"]))
        cases.append(W(f"split{i}_B{B}_G{G}_Hkv{H_kv}_N{N_kv}_d{d}_k{top_k}_{dtype}", B=B,
                       H_q=G * H_kv, H_kv=H_kv, N_kv=N_kv, d=d, top_k=top_k, dtype=dtype,
                       seed=9700 + i))
    return cases


def _mlp_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        B = int(rng.choice([1, 3, 8, 9, 16, 23, 32, 47, 64]))
        d = int(rng.choice([256, 512, 768, 1024, 1536]))
        D = int(rng.integers(1, 3001))
        density = float(rng.choice([0.005, 0.05, 0.2, 0.5, 1.0]))
        dtype = str(rng.choice(["fp16", "bf16"]))
        act = str(rng.choice(["relu", "identity"]))
        cases.append((M(f"mrand{i}_B{B}_d{d}_D{D}_p{density}_{dtype}", B=B, d=d, D=D,
                        density=density, dtype=dtype, seed=9500 + i), act))
    return cases


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


@pytest.mark.parametrize("w,splits", _decode_cases(24, 1234), ids=lambda c: getattr(c, "name", str(c)))
def test_random_decode_shape(sha, w, splits):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    q, k, v, idx = q.to(dev), k.to(dev), v.to(dev), idx.to(dev)
    out = workloads.make_out(w, "cuda")
    if splits == 0:
        sha.decode(q, k, v, idx, w.scale, out)
    else:
        ws = sha.alloc_workspace(q, k, idx, splits)
        sha.sha_decode_ex(q, k, v, idx, w.scale, out, ws, splits)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("w", _split_regime_cases(16, 2468), ids=lambda w: w.name)
def test_random_split_regime_shape(sha, w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    q, k, v, idx = q.to(dev), k.to(dev), v.to(dev), idx.to(dev)
    outs = []
    for _ in range(2):
        out = workloads.make_out(w, "cuda")
        sha.decode(q, k, v, idx, w.scale, out)
        torch.cuda.synchronize()
        assert sha.sha_get_device_status() == sha.SHA_OK
        outs.append(out)
    check_sampled_units(w, q, k, v, idx, outs[0], n_random=32)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


@pytest.mark.parametrize("w,act", _mlp_cases(16, 4321), ids=lambda c: getattr(c, "name", str(c)))
def test_random_selective_mlp_shape(sha, w, act):
    x, W1t, W2t, active = workloads.make_mlp(w)
    dev = torch.device("cuda")
    S, n_S = sha.sha_mlp_union(active.to(dev))
    y = sha.sha_selective_mlp(x.to(dev), W1t.to(dev), W2t.to(dev), S, n_S, activation=act)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    want_S = oracle.mlp_union(active.numpy())
    n = int(n_S.item())
    assert n == len(want_S) and np.array_equal(S[:n].cpu().numpy(), want_S)
    want = oracle.selective_mlp(x, W1t, W2t, want_S, w.dtype, act=act)
    excess, err = mlp_excess(y.cpu().double().numpy(), want, w.dtype)
    assert excess <= 0, err


def _token_cases(n, seed):
    """Head x token sparsity: random G, d, cache lengths and list lengths
    (single keys, ragged last tiles, lists longer than the cache with
    repeats), so every gather warp meets full, partial and empty row blocks."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        G = int(rng.choice([1, 1, 2, 4, 8]))
        H_kv = int(rng.integers(1, 13))
        d = int(rng.choice([64, 128]))
        N_kv = int(rng.integers(1, 2501))
        top_k = int(rng.integers(1, H_kv + 1))
        B = int(rng.integers(1, 17))
        n_sel = int(rng.choice([1, int(rng.integers(1, 300)), int(rng.integers(1, 2 * N_kv + 2)),
                                int(rng.integers(100, 1200))]))
        dtype = str(rng.choice(["fp16", "bf16"]))
        cases.append((W(f"tok{i}_B{B}_G{G}_Hkv{H_kv}_N{N_kv}_d{d}_k{top_k}_s{n_sel}_{dtype}", B=B,
                        H_q=G * H_kv, H_kv=H_kv, N_kv=N_kv, d=d, top_k=top_k, dtype=dtype,
                        seed=9800 + i), n_sel))
    return cases


@pytest.mark.parametrize("w,n_sel", _token_cases(16, 4321), ids=lambda c: getattr(c, "name", str(c)))
def test_random_token_shape(sha, w, n_sel):
    from parity import TOLERANCE, active_mask, out_bits
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    tok = workloads.make_tokens(w, n_sel)
    dev = torch.device("cuda")
    out = workloads.make_out(w, dev)
    sha.sha_decode_tokens(q.to(dev), k.to(dev), v.to(dev), idx.to(dev), tok.to(dev), w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    want, _ = oracle.sha_decode_tokens(q, k, v, idx.numpy(), tok.numpy(), w.scale, w.dtype)
    mask = active_mask(idx.numpy(), w.B, w.H_kv, w.G)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == np.uint16(workloads.SENTINEL[w.dtype])).all()
    if mask.any():
        got = out.cpu().double().numpy()
        assert np.abs(got[mask] - want[mask]).max() <= TOLERANCE[w.dtype]
