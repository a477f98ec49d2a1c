"""Failure detection: every pipeline wait of the decode kernels is bounded.
On a test build of the library whose wait limit the test lowers to one
nanosecond, the first wait that has to spin gives up: the kernel must
return (nothing waits forever, nothing traps), report SHA_ERR_TIMEOUT through
sha_get_device_status, leave every unselected row untouched, and leave the
library-owned workspace usable, so that the next call after the limit is
restored matches the oracle.  The product library is unaffected throughout."""
import ctypes

import pytest
import torch

import workloads
from parity import check_against_oracle, out_bits

pytestmark = pytest.mark.gpu

W = workloads.Workload
LIMIT_NS = 4_000_000_000


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import head_sparse_decode_b200 as sha
    from head_sparse_decode_b200 import build
    hooks = ctypes.CDLL(build.build_test_hooks())
    vp, i = ctypes.c_void_p, ctypes.c_int
    args = [vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp, vp]
    for name in ("sha_decode", "sha_decode_bf16"):
        getattr(hooks, name).argtypes = args
        getattr(hooks, name).restype = i
    hooks.sha_decode_clustered.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp,
                                           i, i, i, i, vp]
    hooks.sha_decode_clustered.restype = i
    hooks.sha_decode_tokens.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, ctypes.c_float,
                                        vp, i, vp]
    hooks.sha_decode_tokens.restype = i
    hooks.sha_get_device_status.argtypes = [vp]
    hooks.sha_get_device_status.restype = i
    hooks.sha_test_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    hooks.sha_test_set_wait_limit.restype = i
    yield sha, hooks
    hooks.sha_test_set_wait_limit(LIMIT_NS)


def _inputs(w):
    q, k, v = workloads.make_qkv(w)
    idx = workloads.make_index(w)
    dev = torch.device("cuda")
    return q.to(dev), k.to(dev), v.to(dev), idx.to(dev)


def _call(hooks, w, q, k, v, idx, out, cluster=0):
    s = torch.cuda.current_stream().cuda_stream
    a = (q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), w.B, w.H_q, w.H_kv, w.N_kv,
         w.d, w.top_k, w.scale, out.data_ptr())
    if cluster:
        return hooks.sha_decode_clustered(*a, 0 if w.dtype == "fp16" else 1, cluster, 1, 0, s)
    fn = hooks.sha_decode if w.dtype == "fp16" else hooks.sha_decode_bf16
    return fn(*a, s)


def _status(hooks):
    return hooks.sha_get_device_status(torch.cuda.current_stream().cuda_stream)


CASES = [
    # more units than SMs: even cut, units split between blocks, merged
    # through the library workspace's slots and arrival counters
    (W("timeout_gqa_kernel", B=32, H_q=16, H_kv=16, N_kv=4000, d=128, top_k=5, dtype="fp16",
       seed=601), 0),
    (W("timeout_fma_kernel", B=32, H_q=16, H_kv=16, N_kv=1000, d=64, top_k=5, dtype="bf16",
       seed=602), 0),
    (W("timeout_gqa_g8", B=16, H_q=64, H_kv=8, N_kv=2000, d=128, top_k=5, dtype="bf16",
       seed=603), 0),
    # the clustered cut: parts stored into other blocks' shared memory
    (W("timeout_clustered", B=1, H_q=32, H_kv=32, N_kv=1920, d=128, top_k=8, dtype="fp16",
       seed=604), 4),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_wait_gives_up_reports_and_recovers(libs, case):
    sha, hooks = libs
    w, cluster = case
    q, k, v, idx = _inputs(w)
    assert hooks.sha_get_device_status(None) == sha.SHA_OK

    assert hooks.sha_test_set_wait_limit(1) == sha.SHA_OK
    out = workloads.make_out(w, "cuda")
    assert _call(hooks, w, q, k, v, idx, out, cluster) == sha.SHA_OK
    torch.cuda.synchronize()                       # the kernel returned
    assert _status(hooks) == sha.SHA_ERR_TIMEOUT
    assert _status(hooks) == sha.SHA_OK            # read and cleared
    # rows of unselected heads stay untouched even when the call gives up
    from parity import active_mask
    mask = active_mask(idx.cpu().numpy(), w.B, w.H_kv, w.G)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == workloads.SENTINEL[w.dtype]).all()

    # limit restored: the same library (and its workspace) computes correctly
    assert hooks.sha_test_set_wait_limit(LIMIT_NS) == sha.SHA_OK
    for _ in range(2):
        out = workloads.make_out(w, "cuda")
        assert _call(hooks, w, q, k, v, idx, out, cluster) == sha.SHA_OK
        torch.cuda.synchronize()
        assert _status(hooks) == sha.SHA_OK
        check_against_oracle(w, q, k, v, idx, out)

    # and the product library was never touched by any of it
    out = workloads.make_out(w, "cuda")
    sha.decode(q, k, v, idx, w.scale, out)
    torch.cuda.synchronize()
    assert sha.sha_get_device_status() == sha.SHA_OK
    check_against_oracle(w, q, k, v, idx, out)


def test_gathered_wait_gives_up_reports_and_recovers(libs):
    """The head x token gather: four gather warps, each with its own bounded
    waits, arriving on the same stages."""
    sha, hooks = libs
    w = W("timeout_tokens", B=16, H_q=32, H_kv=32, N_kv=3000, d=128, top_k=6, dtype="fp16",
          seed=605)
    q, k, v, idx = _inputs(w)
    tok = workloads.make_tokens(w, 700).cuda()
    s = torch.cuda.current_stream().cuda_stream

    def call(out):
        return hooks.sha_decode_tokens(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(),
                                       tok.data_ptr(), w.B, w.H_q, w.H_kv, w.N_kv, w.d, w.top_k,
                                       tok.shape[2], w.scale, out.data_ptr(), 0, s)

    assert hooks.sha_get_device_status(None) == sha.SHA_OK
    assert hooks.sha_test_set_wait_limit(1) == sha.SHA_OK
    out = workloads.make_out(w, "cuda")
    assert call(out) == sha.SHA_OK
    torch.cuda.synchronize()
    assert _status(hooks) == sha.SHA_ERR_TIMEOUT
    from parity import TOLERANCE, active_mask
    mask = active_mask(idx.cpu().numpy(), w.B, w.H_kv, w.G)
    bits = out_bits(out).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == workloads.SENTINEL[w.dtype]).all()

    assert hooks.sha_test_set_wait_limit(LIMIT_NS) == sha.SHA_OK
    import numpy as np
    import oracle
    want, _ = oracle.sha_decode_tokens(q.cpu(), k.cpu(), v.cpu(), idx.cpu().numpy(),
                                       tok.cpu().numpy(), w.scale, w.dtype)
    for _ in range(2):
        out = workloads.make_out(w, "cuda")
        assert call(out) == sha.SHA_OK
        torch.cuda.synchronize()
        assert _status(hooks) == sha.SHA_OK
        got = out.cpu().double().numpy()
        assert np.abs(got[mask] - want[mask]).max() <= TOLERANCE[w.dtype]
