"""Selective GEMM on the GPU against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import mlp_excess

pytestmark = pytest.mark.gpu
M = workloads.MlpWorkload


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


@pytest.mark.parametrize("B,D,p", [(1, 300, 0.1), (8, 5000, 0.02), (64, 2048, 0.5),
                                   (3, 1, 1.0), (5, 1024, 0.0)])
def test_union_bit_exact(sha, B, D, p):
    g = torch.Generator().manual_seed(B * 100 + D)
    active = (torch.rand((B, D), generator=g) < p).to(torch.uint8)
    S, n_S = sha.sha_mlp_union(active.cuda())
    torch.cuda.synchronize()
    want = oracle.mlp_union(active.numpy())
    n = int(n_S.item())
    assert n == len(want)
    assert np.array_equal(S[:n].cpu().numpy(), want)


CASES = [
    M("m1", B=1, d=256, D=1024, density=0.1, dtype="fp16", seed=1),
    M("m2", B=8, d=512, D=2048, density=0.3, dtype="bf16", seed=2),
    M("m3", B=64, d=256, D=1500, density=0.7, dtype="fp16", seed=3),
    M("m4", B=17, d=768, D=3072, density=1.0, dtype="bf16", seed=4),
    M("m5", B=5, d=256, D=4096, density=0.003, dtype="fp16", seed=5),
    M("m6", B=12, d=512, D=1024, density=0.4, dtype="bf16", seed=6),     # batch tiles of 16
    M("m7", B=32, d=1024, D=2048, density=0.2, dtype="fp16", seed=7),    # batch tiles of 32
]


def _run(sha, w, act="relu"):
    x, W1t, W2t, active = workloads.make_mlp(w)
    dev = torch.device("cuda")
    S, n_S = sha.sha_mlp_union(active.to(dev))
    y = sha.sha_selective_mlp(x.to(dev), W1t.to(dev), W2t.to(dev), S, n_S, activation=act)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    want_S = oracle.mlp_union(active.numpy())
    assert int(n_S.item()) == len(want_S)
    want = oracle.selective_mlp(x, W1t, W2t, want_S, w.dtype, act=act)
    return mlp_excess(y.cpu().double().numpy(), want, w.dtype)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_selective_mlp_parity(sha, w):
    excess, err = _run(sha, w)
    assert excess <= 0, err


@pytest.mark.parametrize("case", [1, 6, 2], ids=["batch8", "batch32", "batch64"])
def test_selective_mlp_identity_activation(sha, case):
    w = CASES[case].with_(seed=21)
    excess, err = _run(sha, w, act="identity")
    assert excess <= 0, err


@pytest.mark.parametrize("case", [0, 6], ids=["batch1", "batch32"])
def test_empty_union_gives_zero(sha, case):
    w = CASES[case]
    x, W1t, W2t, _ = workloads.make_mlp(w)
    dev = torch.device("cuda")
    S = torch.zeros(w.D, dtype=torch.int32, device=dev)
    n_S = torch.zeros(1, dtype=torch.int32, device=dev)
    y = sha.sha_selective_mlp(x.to(dev), W1t.to(dev), W2t.to(dev), S, n_S)
    torch.cuda.synchronize()
    assert (y == 0).all()


@pytest.mark.parametrize("case", [0, 6], ids=["batch1", "batch32"])
def test_out_of_range_ids_are_flagged_not_read(sha, case):
    w = CASES[case]
    x, W1t, W2t, _ = workloads.make_mlp(w)
    dev = torch.device("cuda")
    S = torch.tensor([3, 10**6, 7], dtype=torch.int32, device=dev)
    n_S = torch.tensor([3], dtype=torch.int32, device=dev)
    sha.sha_selective_mlp(x.to(dev), W1t.to(dev), W2t.to(dev), S, n_S)
    assert sha.sha_get_device_status() == sha.SHA_ERR_BAD_INDEX


def test_opt66b_mlp_shape_sampled(sha):
    """The OPT-66B MLP at batch 8 and a 30 % union: sampled output columns."""
    w = workloads.MLP_CONFIGS["opt66b_mlp"]
    dev = torch.device("cuda")
    x, W1t, W2t, active = workloads.make_mlp(w, device=dev)
    S, n_S = sha.sha_mlp_union(active)
    y = sha.sha_selective_mlp(x, W1t, W2t, S, n_S)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    n = int(n_S.item())
    Sh = S[:n].cpu().numpy()
    assert np.array_equal(Sh, oracle.mlp_union(active.cpu().numpy()))
    cols = np.sort(np.random.default_rng(0).choice(w.d, 256, replace=False))
    want = oracle.selective_mlp(x.cpu(), W1t.cpu(), W2t[:, cols].cpu().contiguous(), Sh, w.dtype)
    excess, err = mlp_excess(y[:, cols].cpu().double().numpy(), want, w.dtype)
    assert excess <= 0, err


@pytest.mark.parametrize("B,density,dtype", [(64, 1.0, "fp16"), (50, 0.3, "fp16"),
                                             (32, 0.05, "fp16"), (16, 0.5, "fp16"),
                                             (9, 0.2, "fp16"), (40, 0.3, "bf16")])
def test_opt66b_mlp_large_batch_sampled(sha, B, density, dtype):
    """Batches above 8 (tensor-memory up-projection) at the OPT-66B shape: a dense
    union leaves some neuron groups whole inside one block and splits others
    across blocks; sparse unions split every group.  Sampled batch rows and
    output columns against the oracle (which takes the same union S)."""
    w = workloads.MLP_CONFIGS["opt66b_mlp"].with_(B=B, density=density, dtype=dtype,
                                                  seed=5100 + B)
    dev = torch.device("cuda")
    x, W1t, W2t, active = workloads.make_mlp(w, device=dev)
    S, n_S = sha.sha_mlp_union(active)
    y = sha.sha_selective_mlp(x, W1t, W2t, S, n_S)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    n = int(n_S.item())
    Sh = S[:n].cpu().numpy()
    assert np.array_equal(Sh, oracle.mlp_union(active.cpu().numpy()))
    rows = sorted({0, B // 3, (2 * B) // 3, B - 1})
    cols = np.sort(np.random.default_rng(B).choice(w.d, 192, replace=False))
    want = oracle.selective_mlp(x[rows].cpu(), W1t.cpu(), W2t[:, cols].cpu().contiguous(), Sh,
                                w.dtype)
    excess, err = mlp_excess(y[rows][:, cols].cpu().double().numpy(), want, w.dtype)
    assert excess <= 0, err


@pytest.mark.parametrize("case", [1, 3, 6, 2], ids=["batch8", "batch17", "batch32", "batch64"])
def test_repeat_calls_are_bit_identical(sha, case):
    """Split partial sums are added in a fixed order: no dependence on timing."""
    w = CASES[case]
    x, W1t, W2t, active = workloads.make_mlp(w)
    dev = torch.device("cuda")
    x, W1t, W2t = x.to(dev), W1t.to(dev), W2t.to(dev)
    S, n_S = sha.sha_mlp_union(active.to(dev))
    ys = [sha.sha_selective_mlp(x, W1t, W2t, S, n_S) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))


@pytest.mark.parametrize("B,d,D,density,dtype,act", [
    (8, 9216, 36864, 0.1, "fp16", "relu"),      # OPT-66B MLP, 10 % union
    (8, 9216, 36864, 0.3, "bf16", "identity"),  # 30 %, no activation
    (3, 9216, 36864, 0.02, "bf16", "relu"),     # fewer neuron groups than SMs
    (1, 12288, 4096, 0.5, "fp16", "relu"),      # 12 column blocks of 1024
    (7, 768, 5000, 0.37, "bf16", "relu"),       # one unit per group (d = one stage)
    (8, 2560, 777, 1.0, "fp16", "identity"),    # union not a multiple of 16 or 128
    (6, 9216, 36864, 1.0, "fp16", "relu"),      # every neuron
])
def test_small_batch_shapes_sampled(sha, B, d, D, density, dtype, act):
    """Batches up to 8 over sparse to dense unions, a hidden size whose column
    blocks outnumber the SMs, d of one stage, unions that are not a multiple of
    the tile sizes, both activations.  Sampled output columns against the oracle,
    and a repeated call gives the same bits."""
    w = M("sk", B=B, d=d, D=D, density=density, dtype=dtype, seed=5200 + B + D % 97)
    dev = torch.device("cuda")
    x, W1t, W2t, active = workloads.make_mlp(w, device=dev)
    S, n_S = sha.sha_mlp_union(active)
    y = sha.sha_selective_mlp(x, W1t, W2t, S, n_S, activation=act)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    n = int(n_S.item())
    Sh = S[:n].cpu().numpy()
    assert np.array_equal(Sh, oracle.mlp_union(active.cpu().numpy()))
    cols = np.sort(np.random.default_rng(D).choice(d, min(d, 192), replace=False))
    want = oracle.selective_mlp(x.cpu(), W1t.cpu(), W2t[:, cols].cpu().contiguous(), Sh,
                                w.dtype, act=act)
    excess, err = mlp_excess(y[:, cols].cpu().double().numpy(), want, w.dtype)
    assert excess <= 0, err
    # a second call gives the same bits (partial sums added in a fixed order)
    y2 = sha.sha_selective_mlp(x, W1t, W2t, S, n_S, activation=act)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
