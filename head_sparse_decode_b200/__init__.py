"""Selective Head Attention (SHA) decode on B200 -- Python binding.

A thin ctypes layer over ``libsha_decode.so`` (the C ABI declared in
``include/sha_decode.h``): it checks tensor properties, converts them to
pointers and sizes, and calls the library.  Every step of the computation
runs in the library's CUDA kernels; there is no fallback.  Importing this
package fails loudly if the library has not been built
(``python head_sparse_decode_b200/build.py``).

    out = sha_decode(q, k, v, batch_head_index, scale, out)      # fp16
    out = sha_decode_bf16(q, k, v, batch_head_index, scale, out) # bf16
    out = decode(q, k, v, batch_head_index, out=out)             # either dtype

Shapes: q, out [B, H_q, d] (or [B, H_q, 1, d]); k, v [B, H_kv, N_kv, d];
batch_head_index [B, top_k] int32 on the same device.  Rows of out whose head
is not selected are left exactly as they were.
"""
import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# SHA_DECODE_LIBRARY names another build of the same library, e.g. one made with
# non-default tuning knobs (python head_sparse_decode_b200/build.py --define
# SHA_MHA_TENSOR_CORES=0 --output /tmp/libsha_fma.so), for measurements.
LIBRARY_PATH = os.environ.get("SHA_DECODE_LIBRARY") or os.path.join(_PKG, "libsha_decode.so")

if not os.path.exists(LIBRARY_PATH):
    raise ImportError(
        f"{LIBRARY_PATH} is missing: build the CUDA library first "
        "(python head_sparse_decode_b200/build.py)")

_lib = ctypes.CDLL(LIBRARY_PATH)

SHA_OK = 0
SHA_ERR_INVALID_ARG = 1
SHA_ERR_UNSUPPORTED = 2
SHA_ERR_MISALIGNED = 3
SHA_ERR_LAUNCH = 4
SHA_ERR_BAD_INDEX = 5
SHA_ERR_TIMEOUT = 6
SHA_ERR_WORKSPACE = 7
SHA_FP16 = 0
SHA_BF16 = 1

_vp = ctypes.c_void_p
_i = ctypes.c_int
_DECODE_ARGS = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp]
_lib.sha_decode.argtypes = _DECODE_ARGS
_lib.sha_decode.restype = _i
_lib.sha_decode_bf16.argtypes = _DECODE_ARGS
_lib.sha_decode_bf16.restype = _i
_lib.sha_decode_ex.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float, _vp,
                               _i, _vp, ctypes.c_size_t, _i, _vp]
_lib.sha_decode_ex.restype = _i
_lib.sha_decode_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i, _i]
_lib.sha_decode_workspace_size.restype = ctypes.c_size_t
_lib.sha_get_device_status.argtypes = [_vp]
_lib.sha_get_device_status.restype = _i
_lib.sha_status_string.argtypes = [_i]
_lib.sha_status_string.restype = ctypes.c_char_p
_lib.sha_last_cuda_error.argtypes = []
_lib.sha_last_cuda_error.restype = ctypes.c_char_p
_lib.sha_decode_plan.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(ctypes.c_int64)]
_lib.sha_decode_plan.restype = _i
_lib.sha_copy_bandwidth_probe.argtypes = [_vp, _vp, ctypes.c_size_t, _vp]
_lib.sha_copy_bandwidth_probe.restype = _i


class ShaError(RuntimeError):
    def __init__(self, status):
        msg = sha_status_string(status)
        if status == SHA_ERR_LAUNCH:
            msg += ": " + _lib.sha_last_cuda_error().decode()
        super().__init__(msg)
        self.status = status


def sha_status_string(status):
    return _lib.sha_status_string(int(status)).decode()


def _check(status):
    if status != SHA_OK:
        raise ShaError(status)


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _shapes(q, k, v, batch_head_index, out):
    if k.dim() != 4 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, H_kv, N_kv, d]")
    B, H_kv, N_kv, d = k.shape
    if q.dim() == 4:
        if q.shape[2] != 1:
            raise ValueError("decode takes one query token: q must be [B, H_q, 1, d]")
    elif q.dim() != 3:
        raise ValueError("q must be [B, H_q, d] or [B, H_q, 1, d]")
    if q.shape[0] != B or q.shape[-1] != d:
        raise ValueError("q does not match k's batch or head dim")
    H_q = q.shape[1]
    if out.numel() != B * H_q * d:
        raise ValueError("out must hold [B, H_q, d] elements")
    if batch_head_index.dim() != 2 or batch_head_index.shape[0] != B:
        raise ValueError("batch_head_index must be [B, top_k]")
    top_k = batch_head_index.shape[1]
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out),
                    ("batch_head_index", batch_head_index)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device != k.device:
            raise ValueError(f"{name} is on {t.device}, k on {k.device}")
    if batch_head_index.dtype != torch.int32:
        raise TypeError("batch_head_index must be int32")
    for name, t in (("q", q), ("v", v), ("out", out)):
        if t.dtype != k.dtype:
            raise TypeError(f"{name} has dtype {t.dtype}, k has {k.dtype}")
    return B, H_q, H_kv, N_kv, d, top_k


def _default_scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def _decode_args(q, k, v, batch_head_index, scale, out, stream):
    B, H_q, H_kv, N_kv, d, top_k = _shapes(q, k, v, batch_head_index, out)
    return ([q.data_ptr(), k.data_ptr(), v.data_ptr(), batch_head_index.data_ptr(),
             B, H_q, H_kv, N_kv, d, top_k, _default_scale(scale, d), out.data_ptr()],
            _stream_handle(stream, k.device))


def sha_decode(q, k, v, batch_head_index, scale, out, stream=None):
    """fp16 selective head decode into ``out`` (library-managed workspace)."""
    if k.dtype != torch.float16:
        raise TypeError("sha_decode takes float16 tensors; use sha_decode_bf16 for bfloat16")
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode(*args, s))
    return out


def sha_decode_bf16(q, k, v, batch_head_index, scale, out, stream=None):
    """bf16 selective head decode into ``out`` (library-managed workspace)."""
    if k.dtype != torch.bfloat16:
        raise TypeError("sha_decode_bf16 takes bfloat16 tensors")
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_bf16(*args, s))
    return out


_lib.sha_decode_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                   ctypes.c_float, _vp, _i, _vp]
_lib.sha_decode_varlen.restype = _i


def sha_decode_varlen(q, k, v, batch_head_index, seqlens, scale, out, stream=None):
    """Selective head decode where row b uses the first seqlens[b] keys of its
    [N_max]-long cache (seqlens: int32 [B] on the device, each in [1, N_max])."""
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    if (seqlens.dim() != 1 or seqlens.shape[0] != k.shape[0] or seqlens.dtype != torch.int32
            or not seqlens.is_contiguous() or seqlens.device != k.device):
        raise ValueError("seqlens must be a contiguous int32 [B] tensor on k's device")
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_varlen(*args[:4], seqlens.data_ptr(), *args[4:],
                                      _dtype_code(k.dtype), s))
    return out


_lib.sha_decode_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                  ctypes.c_float, _vp, _i, _vp]
_lib.sha_decode_paged.restype = _i


def sha_decode_paged(q, k_pages, v_pages, batch_head_index, seqlens, block_table, scale, out,
                     stream=None):
    """Selective head decode over a paged cache: k/v_pages [num_pages, H_kv, page_size, d],
    block_table int32 [B, max_pages], seqlens int32 [B] (all on one device)."""
    if k_pages.dim() != 4 or v_pages.shape != k_pages.shape:
        raise ValueError("k_pages and v_pages must both be [num_pages, H_kv, page_size, d]")
    num_pages, H_kv, page_size, d = k_pages.shape
    B = q.shape[0]
    H_q = q.shape[1]
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_pages]")
    max_pages = block_table.shape[1]
    for name, t, dt in (("block_table", block_table, torch.int32), ("seqlens", seqlens, torch.int32),
                        ("batch_head_index", batch_head_index, torch.int32),
                        ("q", q, k_pages.dtype), ("v_pages", v_pages, k_pages.dtype),
                        ("out", out, k_pages.dtype)):
        if t.dtype != dt or not t.is_contiguous() or t.device != k_pages.device:
            raise ValueError(f"{name} must be a contiguous {dt} tensor on {k_pages.device}")
    if seqlens.shape != (B,) or q.shape[-1] != d or out.numel() != B * H_q * d:
        raise ValueError("inconsistent shapes")
    top_k = batch_head_index.shape[1]
    with torch.cuda.device(k_pages.device):
        _check(_lib.sha_decode_paged(
            q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), batch_head_index.data_ptr(),
            seqlens.data_ptr(), block_table.data_ptr(), B, H_q, H_kv, num_pages, page_size,
            max_pages, d, top_k, _default_scale(scale, d), out.data_ptr(),
            _dtype_code(k_pages.dtype), _stream_handle(stream, k_pages.device)))
    return out


_lib.sha_decode_strided.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                                    _vp, ctypes.POINTER(ctypes.c_int64),
                                    ctypes.POINTER(ctypes.c_int64), _i, _vp]
_lib.sha_decode_strided.restype = _i


def sha_decode_strided(q, k, v, batch_head_index, scale, out, seqlens=None, stream=None):
    """Selective head decode where k and v are [B, H_kv, N_kv, d] views with any
    strides and d contiguous (e.g. a token-major [B, N_kv, H_kv, d] cache viewed
    with .permute(0, 2, 1, 3), or a padded cache sliced to N_kv keys); with
    seqlens (int32 [B] on the device) row b uses its first seqlens[b] keys."""
    if k.dim() != 4 or v.shape != k.shape:
        raise ValueError("k and v must both be [B, H_kv, N_kv, d] views")
    if k.stride(3) != 1 or v.stride(3) != 1:
        raise ValueError("k and v must have d contiguous")
    B, H_kv, N_kv, d = k.shape
    for name, t in (("q", q), ("out", out), ("batch_head_index", batch_head_index)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for name, t in (("q", q), ("v", v), ("out", out), ("batch_head_index", batch_head_index)):
        if not t.is_cuda or t.device != k.device:
            raise ValueError(f"{name} must be a CUDA tensor on {k.device}")
    for name, t in (("q", q), ("v", v), ("out", out)):
        if t.dtype != k.dtype:
            raise TypeError(f"{name} has dtype {t.dtype}, k has {k.dtype}")
    if batch_head_index.dtype != torch.int32 or batch_head_index.dim() != 2 \
            or batch_head_index.shape[0] != B:
        raise ValueError("batch_head_index must be int32 [B, top_k]")
    H_q = q.shape[1]
    if q.shape[0] != B or q.shape[-1] != d or out.numel() != B * H_q * d:
        raise ValueError("inconsistent shapes")
    if seqlens is not None and (seqlens.dim() != 1 or seqlens.shape[0] != B
                                or seqlens.dtype != torch.int32 or not seqlens.is_contiguous()
                                or seqlens.device != k.device):
        raise ValueError("seqlens must be a contiguous int32 [B] tensor on k's device")
    ks = (ctypes.c_int64 * 3)(k.stride(0), k.stride(1), k.stride(2))
    vs = (ctypes.c_int64 * 3)(v.stride(0), v.stride(1), v.stride(2))
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_strided(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), batch_head_index.data_ptr(),
            None if seqlens is None else seqlens.data_ptr(), B, H_q, H_kv,
            N_kv, d, batch_head_index.shape[1], _default_scale(scale, d), out.data_ptr(), ks, vs,
            _dtype_code(k.dtype), _stream_handle(stream, k.device)))
    return out


_lib.sha_decode_tokens.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                   ctypes.c_float, _vp, _i, _vp]
_lib.sha_decode_tokens.restype = _i


def sha_decode_tokens(q, k, v, batch_head_index, tokens, scale, out, stream=None):
    """Head x token sparsity: unit (b, slot k) attends only to the keys listed in
    tokens[b, k, :] (int32 [B, top_k, n_sel] on the device, positions in
    [0, N_kv) of the selected head's cache)."""
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    B, top_k = batch_head_index.shape
    if (tokens.dim() != 3 or tokens.shape[0] != B or tokens.shape[1] != top_k
            or tokens.dtype != torch.int32 or not tokens.is_contiguous()
            or tokens.device != k.device):
        raise ValueError("tokens must be a contiguous int32 [B, top_k, n_sel] tensor on k's device")
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_tokens(*args[:4], tokens.data_ptr(), *args[4:10],
                                      tokens.shape[2], *args[10:], _dtype_code(k.dtype), s))
    return out


def _dtype_code(dtype):
    if dtype == torch.float16:
        return SHA_FP16
    if dtype == torch.bfloat16:
        return SHA_BF16
    raise TypeError(f"unsupported dtype {dtype}")


def sha_decode_workspace_size(B, H_q, H_kv, N_kv, d, top_k, num_splits=0, device=None):
    """Workspace bytes sha_decode_ex needs for these sizes on ``device``."""
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(_lib.sha_decode_workspace_size(B, H_q, H_kv, N_kv, d, top_k, num_splits))


def alloc_workspace(q, k, batch_head_index, num_splits=0):
    """A zero-filled workspace tensor sized for sha_decode_ex with these inputs."""
    B, H_kv, N_kv, d = k.shape
    nbytes = sha_decode_workspace_size(B, q.shape[1], H_kv, N_kv, d,
                                       batch_head_index.shape[1], num_splits, k.device)
    return torch.zeros(max(nbytes, 1), dtype=torch.uint8, device=k.device)


def sha_decode_ex(q, k, v, batch_head_index, scale, out, workspace=None, num_splits=0,
                  stream=None):
    """Selective head decode with a caller-owned workspace and a forced split count
    (0 = automatic).  ``workspace`` is a zero-initialised CUDA uint8 tensor of at
    least sha_decode_workspace_size(...) bytes (see alloc_workspace); every call
    leaves it zeroed again."""
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    ws_ptr, ws_bytes = (0, 0) if workspace is None else (workspace.data_ptr(),
                                                         workspace.numel() * workspace.element_size())
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_ex(*args, _dtype_code(k.dtype), ws_ptr, ws_bytes,
                                  int(num_splits), s))
    return out


_lib.sha_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                                    _vp, _i, _i, _vp]
_lib.sha_decode_noalloc.restype = _i
_lib.sha_noalloc_scratch_bytes.argtypes = []
_lib.sha_noalloc_scratch_bytes.restype = ctypes.c_size_t
# size of the library's fixed scratch array, as the library was built
NOALLOC_SCRATCH_BYTES = int(_lib.sha_noalloc_scratch_bytes())


def sha_decode_noalloc(q, k, v, batch_head_index, scale, out, num_splits=0, stream=None):
    """Multi-head decode for callers that cannot allocate device memory: the
    library keeps the split-merge scratch in a fixed device array
    (NOALLOC_SCRATCH_BYTES) instead of a workspace, so the call allocates nothing.  Calls on one device
    share that array: do not let them overlap on the GPU."""
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_noalloc(*args, _dtype_code(k.dtype), int(num_splits), s))
    return out


def decode(q, k, v, batch_head_index, scale=None, out=None, stream=None):
    """Selective head decode for either dtype; allocates ``out`` if not given
    (rows of unselected heads are then uninitialised)."""
    if out is None:
        out = torch.empty((q.shape[0], q.shape[1], q.shape[-1]), dtype=q.dtype, device=q.device)
    if k.dtype == torch.float16:
        return sha_decode(q, k, v, batch_head_index, scale, out, stream)
    return sha_decode_bf16(q, k, v, batch_head_index, scale, out, stream)


def sha_decode_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits=0, num_sms=148):
    """Host-side plan of a call: dict with tiles_per_head, total_tiles, blocks,
    workspace_bytes, tile_keys.  Raises ShaError for sizes the library rejects."""
    plan = (ctypes.c_int64 * 5)()
    _check(_lib.sha_decode_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, num_sms, plan))
    return {"tiles_per_head": plan[0], "total_tiles": plan[1], "blocks": plan[2],
            "workspace_bytes": plan[3], "tile_keys": plan[4]}


_lib.sha_decode_plan_ex.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i,
                                    ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)]
_lib.sha_decode_plan_ex.restype = _i
_lib.sha_decode_cluster_capacity.argtypes = [_i, ctypes.POINTER(ctypes.c_int32)]
_lib.sha_decode_cluster_capacity.restype = _i
_lib.sha_decode_clustered.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                                      _vp, _i, _i, _i, _i, _vp]
_lib.sha_decode_clustered.restype = _i


def sha_decode_plan_ex(B, H_q, H_kv, N_kv, d, top_k, num_splits=0, num_sms=148,
                       cluster_capacity=None):
    """sha_decode_plan with the clustered cut: ``cluster_capacity`` maps a cluster
    size c (2..8) to the clusters of c blocks the device holds at once (None: no
    clustered cut).  Adds cluster, units_per_cluster, whole_per_block and pieces."""
    plan = (ctypes.c_int64 * 9)()
    caps = None
    if cluster_capacity is not None:
        caps = (ctypes.c_int32 * 9)(*[int(cluster_capacity.get(c, 0)) for c in range(9)])
    _check(_lib.sha_decode_plan_ex(B, H_q, H_kv, N_kv, d, top_k, num_splits, num_sms, caps, plan))
    return {"tiles_per_head": plan[0], "total_tiles": plan[1], "blocks": plan[2],
            "workspace_bytes": plan[3], "tile_keys": plan[4], "cluster": plan[5],
            "units_per_cluster": plan[6], "pieces": plan[7], "whole_per_block": plan[8]}


def sha_decode_cluster_capacity(d=128, device=None):
    """{c: clusters of c blocks of the clustered kernel that fit on the device at once}."""
    caps = (ctypes.c_int32 * 9)()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        _check(_lib.sha_decode_cluster_capacity(d, caps))
    return {c: caps[c] for c in range(2, 9)}


def sha_decode_clustered(q, k, v, batch_head_index, scale, out, cluster, units_per_cluster=1,
                         whole_per_block=0, stream=None):
    """Selective head decode under a clustered cut chosen by the caller: clusters of
    ``cluster`` blocks, each taking ``units_per_cluster`` (row, head) units, of which
    ``whole_per_block`` go whole to each block and the rest are split into pieces
    merged in distributed shared memory."""
    args, s = _decode_args(q, k, v, batch_head_index, scale, out, stream)
    with torch.cuda.device(k.device):
        _check(_lib.sha_decode_clustered(*args, _dtype_code(k.dtype), int(cluster),
                                         int(units_per_cluster), int(whole_per_block), s))
    return out


_lib.sha_select_heads.argtypes = [_vp, _i, _i, _i, _vp, _vp]
_lib.sha_select_heads.restype = _i


def sha_select_heads(scores, top_k, out=None, stream=None):
    """Per-row top-k of router scores [B, H] (float32, CUDA) into an int32
    [B, top_k] index tensor on the same device (decreasing score, ties by head id)."""
    if scores.dim() != 2 or not scores.is_cuda or not scores.is_contiguous():
        raise ValueError("scores must be a contiguous CUDA tensor [B, H]")
    if scores.dtype != torch.float32:
        raise TypeError("scores must be float32")
    B, H = scores.shape
    if out is None:
        out = torch.empty((B, top_k), dtype=torch.int32, device=scores.device)
    if out.shape != (B, top_k) or out.dtype != torch.int32 or not out.is_contiguous():
        raise ValueError("out must be a contiguous int32 [B, top_k] tensor")
    with torch.cuda.device(scores.device):
        _check(_lib.sha_select_heads(scores.data_ptr(), B, H, int(top_k), out.data_ptr(),
                                     _stream_handle(stream, scores.device)))
    return out


def decode_from_scores(q, k, v, scores, top_k, scale=None, out=None, stream=None):
    """Head selection then selective decode, both on the device and on one stream:
    the router scores [B, H_kv] pick each row's top_k heads (or groups)."""
    idx = sha_select_heads(scores, top_k, stream=stream)
    return decode(q, k, v, idx, scale, out, stream), idx


_lib.sha_mlp_union_workspace_size.argtypes = [_i]
_lib.sha_mlp_union_workspace_size.restype = ctypes.c_size_t
_lib.sha_mlp_union.argtypes = [_vp, _i, _i, _vp, _vp, _vp, ctypes.c_size_t, _vp]
_lib.sha_mlp_union.restype = _i
_lib.sha_selective_mlp_workspace_size.argtypes = [_i, _i, _i]
_lib.sha_selective_mlp_workspace_size.restype = ctypes.c_size_t
_lib.sha_selective_mlp.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp,
                                   ctypes.c_size_t, _vp]
_lib.sha_selective_mlp.restype = _i


def sha_mlp_union(active, S=None, n_S=None, workspace=None, stream=None):
    """Union of active neurons over the batch: active [B, D] uint8/bool (CUDA) ->
    (S int32 [D], n_S int32 [1]); the first n_S entries of S are the ids."""
    if active.dtype == torch.bool:
        active = active.view(torch.uint8)
    if active.dim() != 2 or active.dtype != torch.uint8 or not active.is_contiguous():
        raise ValueError("active must be a contiguous uint8/bool CUDA tensor [B, D]")
    B, D = active.shape
    dev = active.device
    S = torch.empty(D, dtype=torch.int32, device=dev) if S is None else S
    n_S = torch.empty(1, dtype=torch.int32, device=dev) if n_S is None else n_S
    with torch.cuda.device(dev):
        nbytes = int(_lib.sha_mlp_union_workspace_size(D))
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        _check(_lib.sha_mlp_union(active.data_ptr(), B, D, S.data_ptr(), n_S.data_ptr(),
                                  workspace.data_ptr(), workspace.numel(),
                                  _stream_handle(stream, dev)))
    return S, n_S


_lib.sha_selective_mlp_plan.argtypes = [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_int64)]
_lib.sha_selective_mlp_plan.restype = _i


def sha_selective_mlp_plan(B, d, D, num_sms=148):
    """Host-side plan of a Selective GEMM layer: dict with batch_pad, tc_up,
    tc_down, h_rows, down_splits, down_blocks, down_cols and workspace_bytes.
    Raises ShaError for sizes the library rejects."""
    plan = (ctypes.c_int64 * 8)()
    _check(_lib.sha_selective_mlp_plan(B, d, D, num_sms, plan))
    return {"batch_pad": plan[0], "tc_up": bool(plan[1]), "tc_down": bool(plan[2]),
            "h_rows": plan[3], "down_splits": plan[4], "down_blocks": plan[5],
            "down_cols": plan[6], "workspace_bytes": plan[7]}


def sha_selective_mlp_workspace_size(B, d, D, device=None):
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(_lib.sha_selective_mlp_workspace_size(B, d, D))


def sha_selective_mlp(x, W1t, W2t, S, n_S, y=None, activation="relu", workspace=None,
                      stream=None):
    """Selective GEMM: y = sigma(x W1t[S]^T) W2t[S] over the first n_S ids of S.
    x [B, d]; W1t, W2t [D, d] neuron-major; S int32 [>= n_S]; n_S int32 [1] (all CUDA)."""
    B, d = x.shape
    D = W1t.shape[0]
    for name, t in (("x", x), ("W1t", W1t), ("W2t", W2t)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != x.dtype:
            raise ValueError(f"{name} must be a contiguous CUDA tensor of x's dtype")
    if W1t.shape != (D, d) or W2t.shape != (D, d):
        raise ValueError("W1t and W2t must both be [D, d]")
    if S.dtype != torch.int32 or n_S.dtype != torch.int32:
        raise TypeError("S and n_S must be int32")
    dev = x.device
    if y is None:
        y = torch.empty((B, d), dtype=x.dtype, device=dev)
    with torch.cuda.device(dev):
        if workspace is None:
            nbytes = int(_lib.sha_selective_mlp_workspace_size(B, d, D))
            if nbytes == 0:
                raise ShaError(SHA_ERR_UNSUPPORTED)
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        _check(_lib.sha_selective_mlp(
            x.data_ptr(), W1t.data_ptr(), W2t.data_ptr(), S.data_ptr(), n_S.data_ptr(), B, d, D,
            1 if activation == "relu" else 0, _dtype_code(x.dtype), y.data_ptr(),
            workspace.data_ptr(), workspace.numel(), _stream_handle(stream, dev)))
    return y


def sha_get_device_status(stream=None, device=None):
    """Synchronise ``stream`` and read-and-clear the device's sticky flags; returns a
    status code (SHA_OK, SHA_ERR_BAD_INDEX or SHA_ERR_TIMEOUT)."""
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        return int(_lib.sha_get_device_status(_stream_handle(stream, dev)))


def sha_copy_bandwidth_probe(dst, src, stream=None):
    """dst.copy_(src) with the library's 16-byte vectorised copy kernel (bandwidth probe)."""
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < nbytes:
        raise ValueError("dst is smaller than src")
    with torch.cuda.device(src.device):
        _check(_lib.sha_copy_bandwidth_probe(dst.data_ptr(), src.data_ptr(), nbytes,
                                             _stream_handle(stream, src.device)))
    return dst


__all__ = [
    "sha_decode", "sha_decode_bf16", "sha_decode_ex", "sha_decode_workspace_size",
    "sha_get_device_status", "sha_status_string", "sha_decode_plan", "sha_select_heads",
    "decode_from_scores", "sha_decode_varlen", "sha_decode_paged", "sha_mlp_union",
    "sha_selective_mlp", "sha_selective_mlp_workspace_size", "sha_selective_mlp_plan",
    "sha_copy_bandwidth_probe", "decode",
    "alloc_workspace", "ShaError", "LIBRARY_PATH", "sha_decode_noalloc",
]
