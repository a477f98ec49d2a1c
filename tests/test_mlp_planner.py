"""The Selective GEMM planner's choices, on the host (no GPU): which GEMMs of a
layer run on tcgen05, how the warp-level down-projection is split, and
invariants of every plan.  The OPT-66B MLP pins are the launch shapes the ncu
captures recorded on a 148-SM B200 (for example 144 down-projection blocks at
batch 8)."""
import pytest

import head_sparse_decode_b200 as sha

OPT_D, OPT_DFF = 9216, 36864


@pytest.mark.parametrize("B,pad,tc_up,tc_down", [
    (1, 8, False, False), (8, 8, False, False),      # warp-level MMAs up to 8 rows
    (9, 16, True, False), (16, 16, True, False),     # tcgen05 up-projection from 9
    (17, 32, True, True), (32, 32, True, True),      # and the down-projection from 17
    (33, 64, True, True), (64, 64, True, True),
])
def test_opt66b_batch_tiers(B, pad, tc_up, tc_down):
    p = sha.sha_selective_mlp_plan(B, OPT_D, OPT_DFF, num_sms=148)
    assert (p["batch_pad"], p["tc_up"], p["tc_down"]) == (pad, tc_up, tc_down)
    assert p["h_rows"] == OPT_DFF                    # 36864 is a multiple of 128


@pytest.mark.parametrize("B", [1, 4, 8, 16])
def test_opt66b_warp_level_down_projection_split(B):
    # 1024-column items: 9 column chunks x 16 neuron ranges = 144 blocks of 148
    p = sha.sha_selective_mlp_plan(B, OPT_D, OPT_DFF, num_sms=148)
    assert p["down_cols"] == 1024
    assert p["down_splits"] == 16
    assert p["down_blocks"] == 144


@pytest.mark.parametrize("args,status", [
    ((0, 256, 100, 148), sha.SHA_ERR_INVALID_ARG),
    ((4, 256, 0, 148), sha.SHA_ERR_INVALID_ARG),
    ((4, 256, 100, 0), sha.SHA_ERR_INVALID_ARG),
    ((65, 256, 100, 148), sha.SHA_ERR_UNSUPPORTED),
    ((4, 300, 100, 148), sha.SHA_ERR_UNSUPPORTED),
])
def test_rejected_sizes(args, status):
    with pytest.raises(sha.ShaError) as err:
        sha.sha_selective_mlp_plan(*args)
    assert err.value.status == status


def test_plan_invariants():
    for sms in (1, 2, 16, 132, 148, 300):
        for d in (256, 512, 768, 4096, 9216, 12288):
            for D in (1, 100, 4096, 36864):
                for B in (1, 2, 7, 8, 9, 15, 16, 17, 31, 32, 33, 63, 64):
                    p = sha.sha_selective_mlp_plan(B, d, D, num_sms=sms)
                    pad = p["batch_pad"]
                    # the smallest tier that holds the batch
                    assert pad == min(t for t in (8, 16, 32, 64) if t >= B)
                    assert not p["tc_down"] or p["tc_up"]
                    assert not p["tc_up"] or (pad >= 16 and sms <= 256)
                    assert p["h_rows"] == -(-D // 128) * 128
                    wc = p["down_cols"]
                    assert wc % 256 == 0 and d % wc == 0 and wc <= (512 if pad == 64 else 1024)
                    items = d // wc * p["down_splits"]
                    assert p["down_splits"] >= 1
                    assert p["down_blocks"] == min(items, sms)
                    ws = p["workspace_bytes"]
                    assert ws % 256 == 0 and ws >= p["h_rows"] * pad * 2
