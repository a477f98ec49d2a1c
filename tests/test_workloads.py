"""The seeded input recipe (no GPU): what the generators promise about their
inputs, and the algorithmic byte counts the roofline divides by."""
import torch

import workloads


def test_head_index_rows_are_distinct_valid_and_seeded():
    for name in ("opt66b", "llama2_7b", "llama31_70b_gqa"):
        w = workloads.CONFIGS[name]
        idx = workloads.make_index(w)
        assert idx.shape == (w.B, w.top_k) and idx.dtype == torch.int32
        assert int(idx.min()) >= 0 and int(idx.max()) < w.H_kv
        for row in idx:
            assert len(set(row.tolist())) == w.top_k
        assert torch.equal(idx, workloads.make_index(w))
        assert not torch.equal(idx, workloads.make_index(w.with_(seed=w.seed + 1)))


def test_zipf_index_favours_a_few_heads():
    w = workloads.CONFIGS["llama2_7b"]
    counts = torch.bincount(workloads.make_index(w).flatten().long(), minlength=w.H_kv)
    # each of 128 rows takes 16 of 32 heads: uniform would give 64 per head
    assert int(counts.max()) > 100 and int(counts.min()) < 40


def test_token_lists_are_sorted_distinct_and_in_range():
    w = workloads.CONFIGS["opt66b"].with_(B=4)
    for n_sel in (1, 480, 1920):
        t = workloads.make_tokens(w, n_sel)
        assert t.shape == (w.B, w.top_k, n_sel) and t.dtype == torch.int32
        assert int(t.min()) >= 0 and int(t.max()) < w.N_kv
        flat = t.reshape(-1, n_sel)
        assert bool((flat[:, 1:] > flat[:, :-1]).all())      # sorted, no repeats
    # a list longer than the cache holds every position, the rest drawn again
    t = workloads.make_tokens(w.with_(N_kv=64), 100).reshape(-1, 100)
    for row in t:
        assert set(row.tolist()) == set(range(64))


def test_mlp_mask_covers_exactly_the_union():
    w = workloads.MLP_CONFIGS["opt66b_mlp"].with_(d=256, density=0.1)
    _, _, _, active = workloads.make_mlp(w)
    assert active.shape == (w.B, w.D) and active.dtype == torch.uint8
    assert int(active.any(dim=0).sum()) == w.n_union()


def test_output_is_prefilled_with_the_sentinel():
    for dtype in ("fp16", "bf16"):
        w = workloads.CONFIGS["tiny_mha"].with_(dtype=dtype)
        bits = workloads.make_out(w).view(torch.int16).to(torch.int32) & 0xFFFF
        assert bool((bits == workloads.SENTINEL[dtype]).all())


def test_algorithmic_bytes_of_the_opt66b_step():
    # 1408 units x (1920 keys x 128 x 2 B for K and V), their Q and O rows, the index
    w = workloads.CONFIGS["opt66b"]
    assert w.units == 1408
    assert w.algorithmic_bytes() == 1408 * 2 * 1920 * 128 * 2 + 2 * 1408 * 128 * 2 + 4 * 1408
    assert w.algorithmic_bytes() == 1_384_846_848
    # GQA: one K/V stream per selected group, G query and output rows per unit
    g = workloads.CONFIGS["llama31_70b_gqa"]
    assert g.algorithmic_bytes() == 160 * 2 * 4096 * 128 * 2 + 2 * 160 * 8 * 128 * 2 + 4 * 160
