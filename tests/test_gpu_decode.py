"""GPU parity of the CUDA selective-head decode against the float64 oracle,
called through the C ABI (ctypes binding)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import TOLERANCE, active_mask, check_against_oracle, check_sampled_units, out_bits

pytestmark = pytest.mark.gpu

W = workloads.Workload


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


def _on_gpu(w):
    q, k, v = workloads.make_qkv(w)            # CPU generator: host-reproducible
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    return q.to(dev), k.to(dev), v.to(dev), idx.to(dev)


def _run(sha, w, q, k, v, idx, num_splits=None, out=None):
    out = workloads.make_out(w, "cuda") if out is None else out
    if num_splits is None:
        sha.decode(q, k, v, idx, w.scale, out)
    else:
        ws = sha.alloc_workspace(q, k, idx, num_splits)
        sha.sha_decode_ex(q, k, v, idx, w.scale, out, ws, num_splits)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    return out


def test_tiny_mha(sha):
    w = workloads.CONFIGS["tiny_mha"]
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    check_against_oracle(w, q, k, v, idx, out)


# several tiles and a ragged tail, both head dims and dtypes
CASES = [
    W("mha_a", B=3, H_q=8, H_kv=8, N_kv=200, d=128, top_k=3, dtype="fp16", seed=11),
    W("mha_b", B=5, H_q=6, H_kv=6, N_kv=1000, d=64, top_k=2, dtype="fp16", seed=12),
    W("mha_c", B=2, H_q=16, H_kv=16, N_kv=513, d=128, top_k=16, dtype="bf16", seed=13),
    W("mha_d", B=7, H_q=4, H_kv=4, N_kv=65, d=64, top_k=1, dtype="bf16", seed=14),
    W("mha_e", B=1, H_q=12, H_kv=12, N_kv=63, d=128, top_k=5, dtype="fp16", seed=15),
    W("mha_f", B=4, H_q=8, H_kv=8, N_kv=2049, d=128, top_k=4, dtype="fp16", seed=16,
      index="zipf"),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_parity_ragged(sha, w):
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 29, 148, 10_000])
def test_forced_splits_match_oracle(sha, splits):
    w = W("splits", B=3, H_q=8, H_kv=8, N_kv=777, d=128, top_k=3, dtype="fp16", seed=21)
    q, k, v, idx = _on_gpu(w)
    expected, _ = oracle.sha_decode(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(), w.scale,
                                    w.dtype)
    out = _run(sha, w, q, k, v, idx, num_splits=splits)
    check_against_oracle(w, q, k, v, idx, out, expected)


def test_block_cap_and_many_part_merges(sha):
    """Limits of the split: a forced 10 000 blocks over 8192 tiles is clamped to
    4096 (each head's 64 tiles then merge from 32 blocks), and one 64K-key head
    is spread over as many blocks as the 64-part merge cap allows."""
    for w, splits in ((W("cap4096", B=16, H_q=8, H_kv=8, N_kv=8192, d=64, top_k=8,
                         dtype="fp16", seed=23), 10_000),
                      (W("ctx64k", B=1, H_q=2, H_kv=2, N_kv=65536, d=128, top_k=1,
                         dtype="bf16", seed=24), 10_000),
                      (W("ctx64k_auto", B=1, H_q=2, H_kv=2, N_kv=65536, d=128, top_k=1,
                         dtype="bf16", seed=25), None),
                      (W("ctx64k_gqa", B=1, H_q=16, H_kv=2, N_kv=65536, d=128, top_k=1,
                         dtype="bf16", seed=26), None)):
        q, k, v, idx = _on_gpu(w)
        if splits is not None:
            plan = sha.sha_decode_plan(w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k, splits)
            assert plan["blocks"] <= 4096
        out = _run(sha, w, q, k, v, idx, num_splits=splits)
        check_against_oracle(w, q, k, v, idx, out)


def test_workspace_counters_return_to_zero(sha):
    w = W("ws", B=2, H_q=4, H_kv=4, N_kv=300, d=64, top_k=3, dtype="bf16", seed=22)
    q, k, v, idx = _on_gpu(w)
    ws = sha.alloc_workspace(q, k, idx, num_splits=5)
    out = workloads.make_out(w, "cuda")
    plan = sha.sha_decode_plan(w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k, 5)
    assert plan["workspace_bytes"] > 0
    for _ in range(3):
        sha.sha_decode_ex(q, k, v, idx, w.scale, out, ws, 5)
        torch.cuda.synchronize()
        counters = ws[: 16384].view(torch.int32)
        assert int(counters.abs().sum()) == 0
    check_against_oracle(w, q, k, v, idx, out)


def test_workspace_shared_by_calls_of_different_shapes(sha):
    """One workspace (and the library's own) serving calls whose partial states
    and counters would overlap if their layout depended on the call's shape."""
    small = W("ws_small", B=2, H_q=4, H_kv=4, N_kv=300, d=128, top_k=2, dtype="fp16", seed=30)
    large = W("ws_large", B=16, H_q=8, H_kv=8, N_kv=700, d=128, top_k=6, dtype="fp16", seed=31)
    data = {w.name: (w, *_on_gpu(w)) for w in (small, large)}
    nbytes = max(sha.sha_decode_workspace_size(w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k, 7)
                 for w in (small, large))
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    for name in ("ws_small", "ws_large", "ws_small", "ws_large"):
        w, q, k, v, idx = data[name]
        out = workloads.make_out(w, "cuda")
        sha.sha_decode_ex(q, k, v, idx, w.scale, out, ws, 7)
        torch.cuda.synchronize()
        check_against_oracle(w, q, k, v, idx, out)
        out = _run(sha, w, q, k, v, idx)
        check_against_oracle(w, q, k, v, idx, out)


def test_repeat_calls_are_bit_identical(sha):
    w = W("det", B=4, H_q=8, H_kv=8, N_kv=900, d=128, top_k=5, dtype="fp16", seed=23)
    q, k, v, idx = _on_gpu(w)
    a = out_bits(_run(sha, w, q, k, v, idx))
    b = out_bits(_run(sha, w, q, k, v, idx))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("w", [
    # even tile cut, units split between two blocks: the block holding a unit's head
    # merges it on chip when the other part is in, through the slots otherwise
    W("det_split_mha", B=32, H_q=32, H_kv=32, N_kv=1920, d=128, top_k=16, dtype="fp16",
      seed=27),
    W("det_split_gqa", B=32, H_q=64, H_kv=8, N_kv=2048, d=128, top_k=5, dtype="bf16", seed=28),
], ids=lambda w: w.name)
def test_split_unit_merges_are_bit_identical_under_contention(sha, w):
    """Which path merges a split unit depends on timing; the result must not.
    Repeats run while a large copy on another stream perturbs the blocks'
    progress, and every repeat must give the same bits (and match the oracle)."""
    q, k, v, idx = _on_gpu(w)
    ref = _run(sha, w, q, k, v, idx)
    check_sampled_units(w, q, k, v, idx, ref, n_random=48)
    ref_bits = out_bits(ref)
    src = torch.empty(1 << 28, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    side = torch.cuda.Stream()
    for i in range(12):
        if i % 3:
            with torch.cuda.stream(side):
                dst.copy_(src)
        out = workloads.make_out(w, "cuda")
        sha.decode(q, k, v, idx, w.scale, out)
        torch.cuda.synchronize()
        assert sha.sha_get_device_status() == sha.SHA_OK
        assert np.array_equal(out_bits(out), ref_bits), i


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_single_key_returns_value_rows_exactly(sha, dtype):
    w = W("n1", B=3, H_q=8, H_kv=8, N_kv=1, d=128, top_k=4, dtype=dtype, seed=24)
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    vbits = out_bits(v).reshape(w.B, w.H_kv, w.d)
    for b, row in enumerate(idx.cpu().numpy()):
        for h in row:
            assert np.array_equal(bits[b, h], vbits[b, h])


def test_top_k_zero_writes_nothing(sha):
    w = W("k0", B=2, H_q=4, H_kv=4, N_kv=64, d=64, top_k=0, dtype="fp16", seed=25)
    q, k, v, _ = _on_gpu(w.with_(top_k=1))
    idx = torch.zeros((w.B, 0), dtype=torch.int32, device="cuda")
    out = _run(sha, w, q, k, v, idx)
    assert (out_bits(out) == np.uint16(workloads.SENTINEL["fp16"])).all()


def test_all_heads_active_is_dense_attention(sha):
    """top_k = H (layer 0 runs dense): equal to dense attention everywhere."""
    w = W("dense", B=2, H_q=8, H_kv=8, N_kv=300, d=128, top_k=8, dtype="fp16", seed=26)
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.cpu().double().unsqueeze(2), k.cpu().double(), v.cpu().double(),
        scale=w.scale).squeeze(2)
    err = (out.cpu().double() - ref).abs().max().item()
    assert err <= TOLERANCE["fp16"]


def test_out_of_range_ids_skip_the_slot_and_raise_the_flag(sha):
    w = W("bad", B=3, H_q=8, H_kv=8, N_kv=130, d=64, top_k=2, dtype="fp16", seed=27)
    q, k, v, idx = _on_gpu(w)
    idx[1, 0] = 8
    idx[2, 1] = -3
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    assert sha.sha_get_device_status() == sha.SHA_ERR_BAD_INDEX
    assert sha.sha_get_device_status() == sha.SHA_OK          # read clears it
    check_against_oracle(w, q, k, v, idx, out)


def test_index_order_within_a_row_does_not_matter(sha):
    w = W("perm", B=4, H_q=8, H_kv=8, N_kv=400, d=128, top_k=4, dtype="fp16", seed=28)
    q, k, v, idx = _on_gpu(w)
    a = _run(sha, w, q, k, v, idx)
    b = _run(sha, w, q, k, v, idx.flip(1).contiguous())
    # same rows written; values agree to rounding (the block split depends on order)
    written = out_bits(a) != workloads.SENTINEL["fp16"]
    assert np.array_equal(written, out_bits(b) != workloads.SENTINEL["fp16"])
    diff = (a.double() - b.double()).abs().cpu().numpy()
    assert diff[written].max() <= TOLERANCE["fp16"]


def test_rows_of_other_tensors_are_not_read(sha):
    """Unselected heads' K/V may hold anything (here NaN): results are unaffected."""
    w = W("nan", B=2, H_q=8, H_kv=8, N_kv=256, d=128, top_k=3, dtype="fp16", seed=29)
    q, k, v, idx = _on_gpu(w)
    expected, _ = oracle.sha_decode(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(), w.scale,
                                    w.dtype)
    mask = active_mask(idx.cpu().numpy(), w.B, w.H_kv, 1)
    k2, v2 = k.clone(), v.clone()
    k2[torch.from_numpy(~mask).cuda()] = float("nan")
    v2[torch.from_numpy(~mask).cuda()] = float("nan")
    out = _run(sha, w, q, k2, v2, idx)
    check_against_oracle(w, q, k, v, idx, out, expected)


# ---------------------------------------------------------------- full-size configs

@pytest.mark.parametrize("name", ["opt66b", "opt66b_dense", "llama2_7b", "llama2_7b_ctx16k"])
def test_full_size_config_sampled(sha, name):
    w = workloads.CONFIGS[name]
    q, k, v = workloads.make_qkv(w, device="cuda")
    idx = workloads.make_index(w).cuda()
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    err, n = check_sampled_units(w, q, k, v, idx, out, n_random=48)
    assert n >= 48


# ---------------------------------------------------------------- grouped-query (G > 1)

GQA_CASES = [
    W("gqa_g8", B=3, H_q=64, H_kv=8, N_kv=300, d=128, top_k=5, dtype="bf16", seed=41),
    W("gqa_g2", B=4, H_q=8, H_kv=4, N_kv=129, d=64, top_k=2, dtype="fp16", seed=42),
    W("gqa_g4", B=2, H_q=32, H_kv=8, N_kv=1000, d=128, top_k=3, dtype="fp16", seed=43),
    W("gqa_g16", B=2, H_q=64, H_kv=4, N_kv=200, d=128, top_k=4, dtype="bf16", seed=44),
    W("gqa_g7", B=3, H_q=28, H_kv=4, N_kv=65, d=64, top_k=2, dtype="bf16", seed=45),
    W("gqa_short", B=5, H_q=16, H_kv=2, N_kv=17, d=128, top_k=1, dtype="fp16", seed=46),
]


@pytest.mark.parametrize("w", GQA_CASES, ids=lambda w: w.name)
def test_gqa_parity(sha, w):
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    check_against_oracle(w, q, k, v, idx, out)


# Odd group sizes under the even tile cut, where a block ends with the head of a unit
# split in two and merges it on chip: a part's G * (d + 2) floats are copied rounded
# up to 16 bytes.
@pytest.mark.parametrize("w", [
    W("gqa_G3_d128", B=16, H_q=24, H_kv=8, N_kv=3000, d=128, top_k=5, dtype="bf16", seed=81),
    W("gqa_G3_d64", B=16, H_q=24, H_kv=8, N_kv=3000, d=64, top_k=5, dtype="fp16", seed=82),
    W("gqa_G5_d64", B=40, H_q=40, H_kv=8, N_kv=2600, d=64, top_k=4, dtype="bf16", seed=83),
    W("gqa_G7_d128", B=32, H_q=56, H_kv=8, N_kv=2200, d=128, top_k=5, dtype="fp16", seed=84),
    W("gqa_G7_d64", B=40, H_q=28, H_kv=4, N_kv=1700, d=64, top_k=4, dtype="bf16", seed=85),
], ids=lambda w: w.name)
def test_gqa_odd_group_sizes_with_split_units(sha, w):
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    check_sampled_units(w, q, k, v, idx, out, n_random=64)
    again = _run(sha, w, q, k, v, idx)
    assert np.array_equal(out_bits(out), out_bits(again))


@pytest.mark.parametrize("splits", [1, 3, 7, 64, 10_000])
def test_gqa_forced_splits(sha, splits):
    w = W("gqa_splits", B=2, H_q=32, H_kv=4, N_kv=900, d=128, top_k=3, dtype="bf16", seed=47)
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx, num_splits=splits)
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_gqa_single_key_returns_value_rows_exactly(sha, dtype):
    w = W("gqa_n1", B=2, H_q=16, H_kv=4, N_kv=1, d=128, top_k=2, dtype=dtype, seed=48)
    q, k, v, idx = _on_gpu(w)
    out = _run(sha, w, q, k, v, idx)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    vbits = out_bits(v).reshape(w.B, w.H_kv, w.d)
    for b, row in enumerate(idx.cpu().numpy()):
        for h in row:
            for j in range(w.G):
                assert np.array_equal(bits[b, h * w.G + j], vbits[b, h])


def test_gqa_unselected_groups_are_not_read(sha):
    w = W("gqa_nan", B=2, H_q=32, H_kv=8, N_kv=190, d=128, top_k=3, dtype="bf16", seed=49)
    q, k, v, idx = _on_gpu(w)
    expected, _ = oracle.sha_decode(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(), w.scale,
                                    w.dtype)
    sel = np.zeros((w.B, w.H_kv), dtype=bool)
    for b, row in enumerate(idx.cpu().numpy()):
        sel[b, row] = True
    k2, v2 = k.clone(), v.clone()
    k2[torch.from_numpy(~sel).cuda()] = float("nan")
    v2[torch.from_numpy(~sel).cuda()] = float("nan")
    out = _run(sha, w, q, k2, v2, idx)
    check_against_oracle(w, q, k, v, idx, out, expected)


def test_gqa_out_of_range_group_ids(sha):
    w = W("gqa_bad", B=3, H_q=32, H_kv=8, N_kv=130, d=128, top_k=2, dtype="bf16", seed=50)
    q, k, v, idx = _on_gpu(w)
    idx[0, 1] = 8
    idx[2, 0] = -1
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    assert sha.sha_get_device_status() == sha.SHA_ERR_BAD_INDEX
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("name", ["llama31_70b_gqa", "llama31_70b_gqa_ctx16k"])
def test_gqa_full_size_config_sampled(sha, name):
    w = workloads.CONFIGS[name]
    q, k, v = workloads.make_qkv(w, device="cuda")
    idx = workloads.make_index(w).cuda()
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    err, n = check_sampled_units(w, q, k, v, idx, out, n_random=48)
    assert n >= min(48, w.units)


# ---------------------------------------------------------------- scaling-sweep points

@pytest.mark.parametrize("B,N_kv,top_k", [(1, 8192, 8), (256, 512, 32), (32, 4096, 24),
                                          (8, 1920, 16)])
def test_sweep_points_sampled(sha, B, N_kv, top_k):
    w = workloads.sweep(B, N_kv, top_k, point=B + N_kv + top_k)
    q, k, v = workloads.make_qkv(w, device="cuda")
    idx = workloads.make_index(w).cuda()
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    check_sampled_units(w, q, k, v, idx, out, n_random=24)


def test_long_context_16k_gqa_and_mha(sha):
    """The pages evaluate contexts up to 16K tokens."""
    for w in (W("ctx16k_mha", B=2, H_q=8, H_kv=8, N_kv=16384, d=128, top_k=3, dtype="fp16",
                seed=61),
              W("ctx16k_gqa", B=2, H_q=32, H_kv=4, N_kv=16384, d=128, top_k=2, dtype="bf16",
                seed=62)):
        q, k, v, idx = _on_gpu(w)
        out = _run(sha, w, q, k, v, idx)
        check_against_oracle(w, q, k, v, idx, out)


# ---------------------------------------------------------------- CUDA-graph capture

def test_select_and_decode_captured_in_a_cuda_graph(sha):
    """Head selection + decode captured once and replayed with new inputs copied
    into the captured buffers: every replay matches an eager call."""
    w = W("graph", B=16, H_q=32, H_kv=8, N_kv=1000, d=128, top_k=3, dtype="bf16", seed=91)
    q, k, v, _ = _on_gpu(w)
    scores = torch.randn((w.B, w.H_kv), device="cuda")
    out = workloads.make_out(w, "cuda")
    sha.decode_from_scores(q, k, v, scores, w.top_k, w.scale, out)      # warm-up, workspace
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _, idx_g = sha.decode_from_scores(q, k, v, scores, w.top_k, w.scale, out)
    for step in range(3):
        gen = torch.Generator(device="cuda").manual_seed(100 + step)
        q.copy_(torch.randn(q.shape, generator=gen, device="cuda").to(q.dtype))
        scores.copy_(torch.randn(scores.shape, generator=gen, device="cuda"))
        out.view(torch.int16).fill_(workloads.SENTINEL["bf16"])
        graph.replay()
        torch.cuda.synchronize()
        ref = workloads.make_out(w, "cuda")
        ref, idx_e = sha.decode_from_scores(q, k, v, scores, w.top_k, w.scale, ref)
        torch.cuda.synchronize()
        assert torch.equal(idx_g, idx_e)
        assert np.array_equal(out_bits(out), out_bits(ref))
    check_against_oracle(w, q, k, v, idx_e, out)
