"""Bounds: no entry point writes outside its output rows or outside the
workspace it was given.  `out` is a view into a larger buffer whose padding
before and after holds a sentinel, the caller-owned workspace likewise; after
each call every padding byte must be unchanged, bit for bit, and the output
must still match the oracle (Algorithm 1 of the pages writes O only at the
selected head's rows)."""
import numpy as np
import pytest
import torch

import workloads
from parity import check_against_oracle

pytestmark = pytest.mark.gpu

W = workloads.Workload
PAD = 4096          # elements of padding on each side of out (16-byte multiple)
WS_PAD = 64 * 1024  # bytes of padding on each side of a workspace
WS_FILL = 0xA5


@pytest.fixture(scope="module")
def sha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as h
    return h


def _inputs(w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    return q.to(dev), k.to(dev), v.to(dev), idx.to(dev)


def _guarded_out(w):
    """(buffer, out): out [B, H_q, d] in the middle of a sentinel-filled buffer."""
    n = w.B * w.H_q * w.d
    buf = torch.empty(PAD + n + PAD, dtype=workloads.TORCH_DTYPE[w.dtype], device="cuda")
    buf.view(torch.int16).fill_(np.int16(np.uint16(workloads.SENTINEL[w.dtype])))
    return buf, buf[PAD:PAD + n].view(w.B, w.H_q, w.d)


def _check_out_padding(w, buf):
    bits = buf.view(torch.int16).cpu().numpy().view(np.uint16)
    s = np.uint16(workloads.SENTINEL[w.dtype])
    n = w.B * w.H_q * w.d
    assert (bits[:PAD] == s).all(), "written before out"
    assert (bits[PAD + n:] == s).all(), "written after out"


def _guarded_workspace(nbytes):
    """(buffer, workspace): a zeroed workspace between two filled guard regions."""
    buf = torch.full((WS_PAD + nbytes + WS_PAD,), WS_FILL, dtype=torch.uint8, device="cuda")
    buf[WS_PAD:WS_PAD + nbytes].zero_()
    return buf, buf[WS_PAD:WS_PAD + nbytes]


def _check_ws_padding(buf, nbytes):
    b = buf.cpu().numpy()
    assert (b[:WS_PAD] == WS_FILL).all(), "written before the workspace"
    assert (b[WS_PAD + nbytes:] == WS_FILL).all(), "written after the workspace"


def _ok(sha):
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK


DECODE_CASES = [
    # (workload, forced split count or 0)
    (W("b_mha", B=32, H_q=16, H_kv=16, N_kv=1000, d=128, top_k=5, dtype="fp16", seed=701), 0),
    (W("b_mha_short", B=1, H_q=32, H_kv=32, N_kv=1920, d=128, top_k=8, dtype="fp16",
       seed=702), 0),                                     # clustered cut
    (W("b_mha_d64", B=9, H_q=12, H_kv=12, N_kv=515, d=64, top_k=7, dtype="bf16", seed=703), 0),
    (W("b_gqa3", B=16, H_q=24, H_kv=8, N_kv=3000, d=128, top_k=5, dtype="bf16", seed=704), 0),
    (W("b_gqa7", B=12, H_q=28, H_kv=4, N_kv=2500, d=64, top_k=3, dtype="fp16", seed=705), 0),
    (W("b_gqa3_split", B=4, H_q=24, H_kv=8, N_kv=3000, d=128, top_k=5, dtype="bf16",
       seed=706), 37),
    (W("b_gqa7_split", B=3, H_q=28, H_kv=4, N_kv=2500, d=64, top_k=3, dtype="fp16",
       seed=707), 111),
    (W("b_mha_split", B=5, H_q=8, H_kv=8, N_kv=2049, d=128, top_k=4, dtype="fp16", seed=708),
     4096),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: c[0].name)
def test_decode_writes_only_its_rows_and_workspace(sha, case):
    w, splits = case
    q, k, v, idx = _inputs(w)
    # library-owned workspace (sha_decode / sha_decode_bf16)
    buf, out = _guarded_out(w)
    sha.decode(q, k, v, idx, w.scale, out)
    _ok(sha)
    _check_out_padding(w, buf)
    check_against_oracle(w, q, k, v, idx, out)
    # caller-owned workspace with guards on both sides (sha_decode_ex)
    nbytes = sha.sha_decode_workspace_size(w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k, splits)
    nbytes = max(256, (nbytes + 255) // 256 * 256)
    wbuf, ws = _guarded_workspace(nbytes)
    buf, out = _guarded_out(w)
    sha.sha_decode_ex(q, k, v, idx, w.scale, out, ws, splits)
    _ok(sha)
    _check_out_padding(w, buf)
    _check_ws_padding(wbuf, nbytes)
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("cluster", [2, 3, 8])
def test_clustered_writes_only_its_rows(sha, cluster):
    w = W("b_clustered", B=2, H_q=64, H_kv=8, N_kv=1100, d=128, top_k=3, dtype="bf16",
          seed=709)
    q, k, v, idx = _inputs(w)
    buf, out = _guarded_out(w)
    sha.sha_decode_clustered(q, k, v, idx, w.scale, out, cluster, 2)
    _ok(sha)
    _check_out_padding(w, buf)
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("G,d", [(1, 128), (1, 64), (8, 128), (3, 64)])
def test_varlen_writes_only_its_rows(sha, G, d):
    w = W("b_varlen", B=7, H_q=4 * G, H_kv=4, N_kv=700, d=d, top_k=3,
          dtype="bf16" if G > 1 else "fp16", seed=710 + G)
    q, k, v, idx = _inputs(w)
    g = torch.Generator().manual_seed(w.seed)
    lens = torch.randint(1, w.N_kv + 1, (w.B,), generator=g, dtype=torch.int32)
    # the oracle sees each row truncated to its length: keys past it are NaN here
    k_nan, v_nan = k.clone(), v.clone()
    for b, L in enumerate(lens.tolist()):
        k_nan[b, :, L:] = float("nan")
        v_nan[b, :, L:] = float("nan")
    buf, out = _guarded_out(w)
    sha.sha_decode_varlen(q, k_nan, v_nan, idx, lens.cuda(), w.scale, out)
    _ok(sha)
    _check_out_padding(w, buf)
    import oracle
    want, _ = oracle.sha_decode_varlen(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(),
                                       lens.numpy(), w.scale, w.dtype)
    written = ~np.isnan(want[..., 0])
    got = out.cpu().double().numpy()
    from parity import TOLERANCE
    assert np.abs(got[written] - want[written]).max() <= TOLERANCE[w.dtype]


@pytest.mark.parametrize("G,d,page", [(1, 128, 16), (1, 64, 7), (8, 128, 32)])
def test_paged_writes_only_its_rows(sha, G, d, page):
    w = W("b_paged", B=5, H_q=4 * G, H_kv=4, N_kv=300, d=d, top_k=2,
          dtype="fp16" if G == 1 else "bf16", seed=720 + page)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    P = -(-w.N_kv // page)
    n_pages = w.B * P
    g = torch.Generator().manual_seed(w.seed)
    perm = torch.randperm(n_pages, generator=g)
    kp = torch.zeros((n_pages, w.H_kv, page, w.d), dtype=k.dtype)
    vp = torch.zeros_like(kp)
    table = torch.empty((w.B, P), dtype=torch.int32)
    for b in range(w.B):
        for i in range(P):
            slot = int(perm[b * P + i])
            n = min(page, w.N_kv - i * page)
            kp[slot, :, :n] = k[b, :, i * page:i * page + n]
            vp[slot, :, :n] = v[b, :, i * page:i * page + n]
            table[b, i] = slot
    lens = torch.full((w.B,), w.N_kv, dtype=torch.int32)
    buf, out = _guarded_out(w)
    dev = torch.device("cuda")
    sha.sha_decode_paged(q.to(dev), kp.to(dev), vp.to(dev), idx.to(dev), lens.to(dev),
                         table.to(dev), w.scale, out)
    _ok(sha)
    _check_out_padding(w, buf)
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("G,d", [(1, 128), (8, 128), (2, 64)])
def test_strided_writes_only_its_rows(sha, G, d):
    w = W("b_strided", B=3, H_q=4 * G, H_kv=4, N_kv=555, d=d, top_k=2,
          dtype="bf16", seed=730 + G)
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    k_tok = k.permute(0, 2, 1, 3).contiguous().to(dev)
    v_tok = v.permute(0, 2, 1, 3).contiguous().to(dev)
    buf, out = _guarded_out(w)
    sha.sha_decode_strided(q.to(dev), k_tok.permute(0, 2, 1, 3), v_tok.permute(0, 2, 1, 3),
                           idx.to(dev), w.scale, out)
    _ok(sha)
    _check_out_padding(w, buf)
    check_against_oracle(w, q, k, v, idx, out)


@pytest.mark.parametrize("G,d,n_sel", [(1, 128, 300), (8, 128, 129), (3, 64, 77)])
def test_tokens_write_only_their_rows(sha, G, d, n_sel):
    w = W("b_tokens", B=4, H_q=4 * G, H_kv=4, N_kv=500, d=d, top_k=3,
          dtype="fp16" if G == 1 else "bf16", seed=740 + G)
    q, k, v, idx = _inputs(w)
    tok = workloads.make_tokens(w, n_sel).cuda()
    buf, out = _guarded_out(w)
    sha.sha_decode_tokens(q, k, v, idx, tok, w.scale, out)
    _ok(sha)
    _check_out_padding(w, buf)
    import oracle
    from parity import TOLERANCE, active_mask
    want, _ = oracle.sha_decode_tokens(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(),
                                       tok.cpu().numpy(), w.scale, w.dtype)
    mask = active_mask(idx.cpu().numpy(), w.B, w.H_kv, w.G)
    got = out.cpu().double().numpy()
    assert np.abs(got[mask] - want[mask]).max() <= TOLERANCE[w.dtype]


@pytest.mark.parametrize("B,d,D,density", [(8, 9216, 36864, 0.1), (5, 768, 5000, 0.37),
                                           (1, 12288, 4096, 0.5), (24, 512, 2048, 0.3)])
def test_selective_mlp_writes_only_y_and_its_workspace(sha, B, d, D, density):
    w = workloads.MlpWorkload("b_mlp", B=B, d=d, D=D, density=density, dtype="fp16",
                              seed=750 + B)
    dev = torch.device("cuda")
    x, W1t, W2t, active = workloads.make_mlp(w, device=dev)
    S, n_S = sha.sha_mlp_union(active)
    n = B * d
    ybuf = torch.empty(PAD + n + PAD, dtype=torch.float16, device=dev)
    ybuf.view(torch.int16).fill_(np.int16(np.uint16(workloads.SENTINEL["fp16"])))
    y = ybuf[PAD:PAD + n].view(B, d)
    nbytes = sha.sha_selective_mlp_workspace_size(B, d, D)
    nbytes = (nbytes + 255) // 256 * 256
    wbuf, ws = _guarded_workspace(nbytes)
    sha.sha_selective_mlp(x, W1t, W2t, S, n_S, y, workspace=ws)
    _ok(sha)
    bits = ybuf.view(torch.int16).cpu().numpy().view(np.uint16)
    s = np.uint16(workloads.SENTINEL["fp16"])
    assert (bits[:PAD] == s).all() and (bits[PAD + n:] == s).all(), "written outside y"
    _check_ws_padding(wbuf, nbytes)
    import oracle
    from parity import mlp_excess
    Sh = S[:int(n_S.item())].cpu().numpy()
    cols = np.sort(np.random.default_rng(D).choice(d, min(d, 128), replace=False))
    want = oracle.selective_mlp(x.cpu(), W1t.cpu(), W2t[:, cols].cpu().contiguous(), Sh, "fp16")
    excess, err = mlp_excess(y[:, cols].cpu().double().numpy(), want, "fp16")
    assert excess <= 0, err
