"""Pins for the float64 oracle: checks against what the pages and the mathematics
fix, not against the oracle itself.

Each test is chosen so that a plausible slip in the oracle fails it:
  * a wrong widening of fp16/bf16 bits        -> exhaustive conversion test
  * a wrong sign in exp, a dropped scale,
    dropped normalisation, K/V swapped,
    a transposed K                             -> hand-derived golden values
  * a wrong head / group / query-row mapping  -> golden routing, SDPA with GQA
  * wrong online-softmax rescaling             -> online vs definition
  * writing inactive rows                      -> untouched-row checks
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _half_bits(values, dtype="fp16"):
    t = torch.tensor(values, dtype=torch.float64).to(workloads.TORCH_DTYPE[dtype])
    return t


def _rand(shape, seed, dtype="fp16", lo=None):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(workloads.TORCH_DTYPE[dtype])


# ---------------------------------------------------------------- widening

def test_fp16_widening_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.widen(b, "fp16") for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros too
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_widening_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (bits << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = np.array([oracle.widen(int(b), "bf16") for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- hand-derived

def _frac(s):
    return float(Fraction(s))


@pytest.mark.parametrize("tile", [0, 1, 2, 3])
def test_golden_single_unit(tile):
    with open(os.path.join(GOLDEN, "hand_single_unit.json")) as f:
        g = json.load(f)
    assert g["scale"] == "ln2"
    q = _half_bits(g["q"]).reshape(1, 1, -1)
    K = _half_bits(g["K"]).reshape(1, 1, len(g["K"]), -1)
    V = _half_bits(g["V"]).reshape(1, 1, len(g["V"]), -1)
    out, bad = oracle.sha_decode(q, K, V, [[0]], math.log(2), "fp16", tile=tile)
    assert bad == 0
    want = np.array([_frac(s) for s in g["expected"]])
    np.testing.assert_allclose(out[0, 0], want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("tile", [0, 1])
def test_golden_gqa_routing(tile):
    with open(os.path.join(GOLDEN, "hand_gqa_routing.json")) as f:
        g = json.load(f)
    Q = _half_bits(g["Q"])
    K = _half_bits(g["K"])
    V = _half_bits(g["V"])
    out, bad = oracle.sha_decode(Q, K, V, g["batch_head_index"], math.log(2), "fp16",
                                 tile=tile)
    assert bad == 0
    for key, vals in g["expected"].items():
        b, h = map(int, key.split(","))
        np.testing.assert_allclose(out[b, h], [_frac(s) for s in vals], rtol=0, atol=1e-13)
    for key in g["untouched"]:
        b, h = map(int, key.split(","))
        assert np.isnan(out[b, h]).all()


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("G", [1, 2, 8])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_all_heads_active_equals_sdpa(G, dtype):
    """With every head selected (layer 0 runs dense) the result is plain attention:
    torch's scaled_dot_product_attention in float64 on the CPU."""
    B, H_kv, N_kv, d = 3, 4, 37, 16
    H_q = H_kv * G
    q = _rand((B, H_q, d), 1, dtype)
    k = _rand((B, H_kv, N_kv, d), 2, dtype)
    v = _rand((B, H_kv, N_kv, d), 3, dtype)
    # every head, in a different order per row
    idx = np.stack([np.random.default_rng(b).permutation(H_kv) for b in range(B)])
    scale = 0.37
    out, bad = oracle.sha_decode(q, k, v, idx, scale, dtype)
    assert bad == 0
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().unsqueeze(2), k.double(), v.double(), scale=scale,
        enable_gqa=(G > 1)).squeeze(2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_sparse_rows_equal_sdpa_rows_and_rest_untouched():
    w = workloads.CONFIGS["tiny_mha"]
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    out, bad = oracle.sha_decode(q, k, v, idx, w.scale, w.dtype)
    assert bad == 0
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().unsqueeze(2), k.double(), v.double(), scale=w.scale).squeeze(2).numpy()
    active = np.zeros((w.B, w.H_q), dtype=bool)
    for b in range(w.B):
        for h in idx[b].tolist():
            active[b, h] = True
    np.testing.assert_allclose(out[active], ref[active], rtol=0, atol=1e-12)
    assert np.isnan(out[~active]).all()


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_single_key_returns_value_row(dtype):
    """N_kv = 1: softmax of one score is 1, so O = V exactly."""
    q = _rand((2, 3, 8), 4, dtype)
    k = _rand((2, 3, 1, 8), 5, dtype)
    v = _rand((2, 3, 1, 8), 6, dtype)
    out, _ = oracle.sha_decode(q, k, v, [[0, 1, 2], [2, 1, 0]], 0.5, dtype)
    assert np.array_equal(out, v.double().squeeze(2).numpy())


def test_identical_keys_give_mean_value():
    N, d = 29, 8
    q = _rand((1, 1, d), 7)
    k = _rand((1, 1, 1, d), 8).expand(1, 1, N, d).contiguous()
    v = _rand((1, 1, N, d), 9)
    out, _ = oracle.sha_decode(q, k, v, [[0]], 0.9, "fp16")
    np.testing.assert_allclose(out[0, 0], v.double()[0, 0].mean(0).numpy(), rtol=0, atol=1e-13)


def test_zero_scale_gives_mean_value():
    N, d = 31, 8
    q, k, v = _rand((1, 1, d), 10), _rand((1, 1, N, d), 11), _rand((1, 1, N, d), 12)
    out, _ = oracle.sha_decode(q, k, v, [[0]], 0.0, "fp16")
    np.testing.assert_allclose(out[0, 0], v.double()[0, 0].mean(0).numpy(), rtol=0, atol=1e-13)


def test_dominant_key_selects_its_value():
    """One score 60 above all others: O = V[n*] up to e^-60 relative weight."""
    N, d = 16, 4
    k = torch.zeros((1, 1, N, d), dtype=torch.float16)
    k[0, 0, 5, 0] = 60.0
    q = torch.tensor([[[1.0, 0, 0, 0]]], dtype=torch.float16)
    v = _rand((1, 1, N, d), 13)
    out, _ = oracle.sha_decode(q, k, v, [[0]], 1.0, "fp16")
    np.testing.assert_allclose(out[0, 0], v.double()[0, 0, 5].numpy(), rtol=0, atol=1e-20)


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("tile", [1, 3, 16, 100, 128, 500])
def test_online_recurrence_equals_definition(tile):
    """Algorithm 1's tiled recurrence (renormalised per tile) is an exact
    reorganisation of the two-pass softmax."""
    B, H, N, d = 2, 3, 128, 32
    q, k, v = _rand((B, H, d), 14), _rand((B, H, N, d), 15), _rand((B, H, N, d), 16)
    idx = [[2, 0], [1, 2]]
    two_pass, _ = oracle.sha_decode(q, k, v, idx, 0.2, "fp16", tile=0)
    online, _ = oracle.sha_decode(q, k, v, idx, 0.2, "fp16", tile=tile)
    np.testing.assert_allclose(online, two_pass, rtol=0, atol=1e-13, equal_nan=True)


def test_joint_permutation_of_keys_and_values():
    N, d = 50, 16
    q, k, v = _rand((1, 1, d), 17), _rand((1, 1, N, d), 18), _rand((1, 1, N, d), 19)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(3))
    a, _ = oracle.sha_decode(q, k, v, [[0]], 0.3, "fp16")
    b, _ = oracle.sha_decode(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(),
                             [[0]], 0.3, "fp16")
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


def test_shift_of_all_scores_changes_nothing():
    """Adding c to every key adds scale*q.c to every score: softmax is unchanged.
    Values are multiples of 1/8 so every shifted key is exact in fp16."""
    N, d = 20, 8
    g = torch.Generator().manual_seed(20)
    k = (torch.randint(-16, 16, (1, 1, N, d), generator=g) / 8.0).to(torch.float16)
    c = (torch.randint(-16, 16, (d,), generator=g) / 8.0)
    q = (torch.randint(-8, 8, (1, 1, d), generator=g) / 8.0).to(torch.float16)
    v = _rand((1, 1, N, d), 21)
    a, _ = oracle.sha_decode(q, k, v, [[0]], 0.7, "fp16")
    b, _ = oracle.sha_decode(q, (k.double() + c.double()).to(torch.float16), v, [[0]], 0.7,
                             "fp16")
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_output_is_a_convex_combination_of_values():
    N, d = 64, 32
    q, k, v = _rand((1, 1, d), 22), _rand((1, 1, N, d), 23), _rand((1, 1, N, d), 24)
    out, _ = oracle.sha_decode(q, k, v, [[0]], 2.0, "fp16")
    vv = v.double()[0, 0].numpy()
    assert (out[0, 0] >= vv.min(0) - 1e-15).all() and (out[0, 0] <= vv.max(0) + 1e-15).all()


# ---------------------------------------------------------------- routing edges

def test_out_of_range_ids_are_skipped_and_counted():
    q, k, v = _rand((2, 4, 8), 25), _rand((2, 4, 9, 8), 26), _rand((2, 4, 9, 8), 27)
    out, bad = oracle.sha_decode(q, k, v, [[0, 7], [-1, 3]], 0.5, "fp16")
    assert bad == 2
    assert not np.isnan(out[0, 0]).any() and not np.isnan(out[1, 3]).any()
    for b, h in [(0, 1), (0, 2), (0, 3), (1, 0), (1, 1), (1, 2)]:
        assert np.isnan(out[b, h]).all()


def test_zero_top_k_writes_nothing():
    q, k, v = _rand((2, 4, 8), 28), _rand((2, 4, 9, 8), 29), _rand((2, 4, 9, 8), 30)
    out, bad = oracle.sha_decode(q, k, v, np.zeros((2, 0), np.int32), 0.5, "fp16")
    assert bad == 0 and np.isnan(out).all()


def test_units_entry_matches_full_layout():
    w = workloads.CONFIGS["tiny_mha"].with_(H_q=8, H_kv=4)   # G = 2
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    full, _ = oracle.sha_decode(q, k, v, idx, w.scale, w.dtype)
    bs = np.repeat(np.arange(w.B), w.top_k)
    hs = idx.reshape(-1).numpy()
    qu = torch.stack([q[b, h * w.G:(h + 1) * w.G] for b, h in zip(bs, hs)])
    ku = torch.stack([k[b, h] for b, h in zip(bs, hs)])
    vu = torch.stack([v[b, h] for b, h in zip(bs, hs)])
    per_unit = oracle.sha_units(qu, ku, vu, w.scale, w.dtype)
    for i, (b, h) in enumerate(zip(bs, hs)):
        assert np.array_equal(per_unit[i], full[b, h * w.G:(h + 1) * w.G])


# ---------------------------------------------------------------- head selection

@pytest.mark.parametrize("B,H,top_k", [(5, 8, 3), (3, 72, 22), (4, 32, 32), (2, 256, 100),
                                       (3, 1, 1), (2, 9, 0)])
def test_select_heads_matches_stable_argsort(B, H, top_k):
    """numpy's stable argsort of -score: decreasing score, ties by head id."""
    rng = np.random.default_rng(B * 1000 + H)
    scores = rng.integers(-4, 5, size=(B, H)).astype(np.float32)   # many ties
    got = oracle.select_heads(scores, top_k)
    want = np.argsort(-scores, axis=1, kind="stable")[:, :top_k].astype(np.int32)
    assert np.array_equal(got, want)


def test_select_heads_hand_example():
    scores = np.array([[0.5, 2.0, -1.0, 2.0, 7.0]], dtype=np.float32)
    assert oracle.select_heads(scores, 3).tolist() == [[4, 1, 3]]
    neg = np.array([[-np.inf, -3.0, -np.inf]], dtype=np.float32)
    assert oracle.select_heads(neg, 3).tolist() == [[1, 0, 2]]


# ---------------------------------------------------------------- per-row lengths

def test_varlen_rows_equal_fixed_length_on_truncated_caches():
    """Row b with length L is plain decode over the first L keys (checked against
    the fixed-length path on a truncated copy, and against SDPA on that copy)."""
    B, H, N, d = 4, 6, 90, 16
    q, k, v = _rand((B, H, d), 31), _rand((B, H, N, d), 32), _rand((B, H, N, d), 33)
    idx = np.array([[0, 5], [2, 3], [1, 4], [5, 0]])
    lens = [1, 37, 90, 64]
    got, bad = oracle.sha_decode_varlen(q, k, v, idx, lens, 0.25, "fp16")
    assert bad == 0
    for b, L in enumerate(lens):
        kt, vt = k[b:b + 1, :, :L].contiguous(), v[b:b + 1, :, :L].contiguous()
        ref, _ = oracle.sha_decode(q[b:b + 1], kt, vt, idx[b:b + 1], 0.25, "fp16")
        np.testing.assert_array_equal(got[b], ref[0])
        sd = torch.nn.functional.scaled_dot_product_attention(
            q[b:b + 1].double().unsqueeze(2), kt.double(), vt.double(), scale=0.25).squeeze(2)
        for h in idx[b]:
            np.testing.assert_allclose(got[b, h], sd[0, h].numpy(), rtol=0, atol=1e-12)


def test_varlen_full_lengths_equal_fixed_and_bad_lengths_are_skipped():
    B, H, N, d = 3, 4, 20, 8
    q, k, v = _rand((B, H, d), 34), _rand((B, H, N, d), 35), _rand((B, H, N, d), 36)
    idx = np.array([[0, 1], [2, 3], [3, 0]])
    fixed, _ = oracle.sha_decode(q, k, v, idx, 0.3, "fp16")
    same, bad = oracle.sha_decode_varlen(q, k, v, idx, [N, N, N], 0.3, "fp16")
    assert bad == 0 and np.array_equal(np.isnan(fixed), np.isnan(same))
    np.testing.assert_array_equal(fixed[~np.isnan(fixed)], same[~np.isnan(same)])
    out, bad = oracle.sha_decode_varlen(q, k, v, idx, [0, N + 1, 5], 0.3, "fp16")
    assert bad == 4 and np.isnan(out[:2]).all() and not np.isnan(out[2, [3, 0]]).any()


# ---------------------------------------------------------------- paged cache

def _to_pages(k, page_size, perm):
    """[B, H, N, d] contiguous cache -> [B*N/ps, H, ps, d] pages, page i of row b stored
    at pool slot perm[b*P + i]; returns (pool, block_table)."""
    B, H, N, d = k.shape
    P = N // page_size
    pool = torch.empty((B * P, H, page_size, d), dtype=k.dtype)
    table = np.empty((B, P), dtype=np.int32)
    for b in range(B):
        for i in range(P):
            slot = int(perm[b * P + i])
            pool[slot] = k[b, :, i * page_size:(i + 1) * page_size]
            table[b, i] = slot
    return pool, table


@pytest.mark.parametrize("page_size", [1, 16, 64])
def test_paged_equals_contiguous_varlen_for_any_page_placement(page_size):
    B, H, N, d = 3, 4, 128, 16
    q, k, v = _rand((B, H, d), 41), _rand((B, H, N, d), 42), _rand((B, H, N, d), 43)
    idx = np.array([[0, 3], [2, 1], [3, 2]])
    lens = [1, 77, 128]
    perm = np.random.default_rng(page_size).permutation(B * N // page_size)
    kp, table = _to_pages(k, page_size, perm)
    vp, _ = _to_pages(v, page_size, perm)
    want, _ = oracle.sha_decode_varlen(q, k, v, idx, lens, 0.3, "fp16")
    got, bad = oracle.sha_decode_paged(q, kp, vp, idx, lens, table, 0.3, "fp16")
    assert bad == 0
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    np.testing.assert_array_equal(got[~np.isnan(got)], want[~np.isnan(want)])


def test_paged_rows_with_bad_pages_or_lengths_are_skipped():
    B, H, N, d, ps = 3, 2, 32, 8, 16
    q, k, v = _rand((B, H, d), 44), _rand((B, H, N, d), 45), _rand((B, H, N, d), 46)
    kp, table = _to_pages(k, ps, np.arange(B * N // ps))
    vp, _ = _to_pages(v, ps, np.arange(B * N // ps))
    table[1, 1] = 999                           # row 1 needs page 1 (length 20)
    out, bad = oracle.sha_decode_paged(q, kp, vp, [[0], [1], [0]], [5, 20, 33], table, 0.5,
                                       "fp16")
    assert bad == 2 and not np.isnan(out[0, 0]).any() and np.isnan(out[1:]).all()


# ---------------------------------------------------------------- selective GEMM (MLP)

def test_mlp_union_matches_numpy():
    rng = np.random.default_rng(5)
    active = rng.random((7, 300)) < 0.05
    assert np.array_equal(oracle.mlp_union(active), np.nonzero(active.any(0))[0])
    assert len(oracle.mlp_union(np.zeros((3, 10), bool))) == 0


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_selective_mlp_all_neurons_is_the_dense_mlp(dtype):
    """S = every neuron: relu(x W1) W2^T with torch in float64."""
    B, d, D = 5, 24, 40
    x, W1t, W2t = _rand((B, d), 51, dtype), _rand((D, d), 52, dtype), _rand((D, d), 53, dtype)
    y = oracle.selective_mlp(x, W1t, W2t, np.arange(D), dtype)
    ref = torch.relu(x.double() @ W1t.double().T) @ W2t.double()
    np.testing.assert_allclose(y, ref.numpy(), rtol=0, atol=1e-11)


def test_selective_mlp_equals_dense_with_unselected_neurons_removed():
    B, d, D = 4, 16, 50
    x, W1t, W2t = _rand((B, d), 54), _rand((D, d), 55), _rand((D, d), 56)
    S = np.array([1, 7, 8, 20, 49])
    y = oracle.selective_mlp(x, W1t, W2t, S, "fp16")
    keep = torch.zeros(D, dtype=torch.float64)
    keep[S] = 1.0
    ref = (torch.relu(x.double() @ W1t.double().T) * keep) @ W2t.double()
    np.testing.assert_allclose(y, ref.numpy(), rtol=0, atol=1e-12)
    # identity activation, and the empty set
    y_lin = oracle.selective_mlp(x, W1t, W2t, S, "fp16", act="identity")
    ref_lin = ((x.double() @ W1t.double().T) * keep) @ W2t.double()
    np.testing.assert_allclose(y_lin, ref_lin.numpy(), rtol=0, atol=1e-12)
    assert (oracle.selective_mlp(x, W1t, W2t, [], "fp16") == 0).all()


def test_selective_mlp_column_subset_is_the_same_sum():
    B, d, D = 3, 16, 30
    x, W1t, W2t = _rand((B, d), 57), _rand((D, d), 58), _rand((D, d), 59)
    S = [2, 5, 11, 29]
    full = oracle.selective_mlp(x, W1t, W2t, S, "fp16")
    cols = [1, 7, 15]
    sub = oracle.selective_mlp(x, W1t, W2t[:, cols].contiguous(), S, "fp16")
    np.testing.assert_array_equal(sub, full[:, cols])


# ---------------------------------------------------------------- head x token sparsity

def _token_case(seed, B=3, H_q=8, H_kv=4, N_kv=40, d=16, top_k=2, n_sel=9, dtype="fp16"):
    w = workloads.Workload("tok", B=B, H_q=H_q, H_kv=H_kv, N_kv=N_kv, d=d, top_k=top_k,
                           dtype=dtype, seed=seed)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w).numpy()
    rng = np.random.default_rng(seed)
    tok = rng.integers(0, N_kv, size=(B, top_k, n_sel)).astype(np.int32)
    return w, q, k, v, idx, tok


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_tokens_equal_the_unit_oracle_on_a_gathered_cache(dtype):
    # restricting a unit to its listed keys is the ordinary per-unit attention
    # over a cache that holds exactly those keys, in that order
    w, q, k, v, idx, tok = _token_case(11, dtype=dtype)
    got, bad = oracle.sha_decode_tokens(q, k, v, idx, tok, w.scale, dtype)
    assert bad == 0
    G = w.G
    units = [(b, s) for b in range(w.B) for s in range(w.top_k)]
    qu = torch.stack([q[b, idx[b, s] * G:(idx[b, s] + 1) * G] for b, s in units])
    ku = torch.stack([k[b, idx[b, s]][torch.from_numpy(tok[b, s]).long()] for b, s in units])
    vu = torch.stack([v[b, idx[b, s]][torch.from_numpy(tok[b, s]).long()] for b, s in units])
    ref = oracle.sha_units(qu, ku, vu, w.scale, dtype)
    for i, (b, s) in enumerate(units):
        h = idx[b, s]
        assert np.abs(got[b, h * G:(h + 1) * G] - ref[i]).max() < 1e-12


def test_tokens_brute_force_numpy():
    w, q, k, v, idx, tok = _token_case(12, B=2, H_q=2, H_kv=2, N_kv=13, d=8, top_k=1, n_sel=5)
    got, _ = oracle.sha_decode_tokens(q, k, v, idx, tok, w.scale, w.dtype)
    for b in range(w.B):
        h = idx[b, 0]
        qd = q[b, h].double().numpy()
        K = k[b, h].double().numpy()[tok[b, 0]]
        V = v[b, h].double().numpy()[tok[b, 0]]
        s = w.scale * K @ qd
        p = np.exp(s - s.max())
        want = p @ V / p.sum()
        assert np.abs(got[b, h] - want).max() < 1e-12


def test_all_positions_in_order_is_the_full_decode():
    w, q, k, v, idx, _ = _token_case(13, N_kv=23)
    tok = np.broadcast_to(np.arange(w.N_kv, dtype=np.int32), (w.B, w.top_k, w.N_kv)).copy()
    got, bad = oracle.sha_decode_tokens(q, k, v, idx, tok, w.scale, w.dtype)
    full, _ = oracle.sha_decode(q, k, v, idx, w.scale, w.dtype)
    assert bad == 0
    written = ~np.isnan(full)
    assert np.array_equal(np.isnan(got), np.isnan(full))
    assert np.abs(got[written] - full[written]).max() < 1e-12


def test_token_order_and_duplication_invariance():
    w, q, k, v, idx, tok = _token_case(14, n_sel=6)
    base, _ = oracle.sha_decode_tokens(q, k, v, idx, tok, w.scale, w.dtype)
    rng = np.random.default_rng(5)
    perm = np.stack([np.stack([rng.permutation(t) for t in row]) for row in tok])
    shuffled, _ = oracle.sha_decode_tokens(q, k, v, idx, perm, w.scale, w.dtype)
    doubled, _ = oracle.sha_decode_tokens(q, k, v, idx, np.repeat(tok, 2, axis=2), w.scale,
                                          w.dtype)
    m = ~np.isnan(base)
    assert np.abs(shuffled[m] - base[m]).max() < 1e-12
    assert np.abs(doubled[m] - base[m]).max() < 1e-12


def test_single_token_returns_its_value_row():
    w, q, k, v, idx, tok = _token_case(15, n_sel=1)
    got, _ = oracle.sha_decode_tokens(q, k, v, idx, tok, w.scale, w.dtype)
    for b in range(w.B):
        for s in range(w.top_k):
            h = idx[b, s]
            want = v[b, h, tok[b, s, 0]].double().numpy()
            for j in range(w.G):
                assert np.array_equal(got[b, h * w.G + j], want)


def test_units_with_out_of_range_tokens_are_skipped_and_counted():
    w, q, k, v, idx, tok = _token_case(16)
    tok[0, 1, 3] = w.N_kv
    tok[2, 0, 0] = -1
    got, bad = oracle.sha_decode_tokens(q, k, v, idx, tok, w.scale, w.dtype)
    assert bad == 2
    G = w.G
    for b, s in ((0, 1), (2, 0)):
        h = idx[b, s]
        assert np.isnan(got[b, h * G:(h + 1) * G]).all()
    h = idx[0, 0]
    assert not np.isnan(got[0, h * G:(h + 1) * G]).any()
