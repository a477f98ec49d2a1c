"""Float64 CPU oracle for Selective Head Attention decode -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU
baseline and its ``--impl reference`` arm) may import this package.  The
CUDA library never calls it and shares no code with it; it is the
independent reference the CUDA path is compared against.

The arithmetic lives in ``sha_oracle.c`` (plain C, float64); this module only
loads it and marshals arguments.  Inputs are the 16-bit patterns of fp16 or
bf16 tensors (numpy ``uint16`` arrays, or CPU torch tensors of dtype
float16 / bfloat16).

What is computed, and which passage each function follows, is stated in
``sha_oracle.c``: the attention equation of the "Attention Head 稀疏性"
section (papernotes.org summary of Polar Sparsity), Algorithm 1 "Selective
Head Flash Attention (Decode)" (ri.k117.org reproducibility record), the
routing of the "Selective Head Attention (SHA) Kernel" section, and the
router's top-k head selection ("Router 训练").
"""
import ctypes
import os

import numpy as np

from . import build as _build

FP16 = 0
BF16 = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.sha_oracle_decode.restype = ctypes.c_longlong
        lib.sha_oracle_decode.argtypes = [
            u16p, u16p, u16p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.c_int, ctypes.c_int, f64p]
        lib.sha_oracle_units.restype = ctypes.c_int
        lib.sha_oracle_units.argtypes = [
            u16p, u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int, f64p]
        lib.sha_oracle_widen.restype = ctypes.c_double
        lib.sha_oracle_widen.argtypes = [ctypes.c_uint16, ctypes.c_int]
        lib.sha_oracle_decode_varlen.restype = ctypes.c_longlong
        lib.sha_oracle_decode_varlen.argtypes = [
            u16p, u16p, u16p, i32p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, f64p]
        lib.sha_oracle_decode_tokens.restype = ctypes.c_longlong
        lib.sha_oracle_decode_tokens.argtypes = [
            u16p, u16p, u16p, i32p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
            f64p]
        lib.sha_oracle_decode_paged.restype = ctypes.c_longlong
        lib.sha_oracle_decode_paged.argtypes = [
            u16p, u16p, u16p, i32p, i32p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, ctypes.c_int, f64p]
        lib.sha_oracle_mlp_union.restype = ctypes.c_int
        lib.sha_oracle_mlp_union.argtypes = [ctypes.POINTER(ctypes.c_uint8), ctypes.c_int,
                                             ctypes.c_int, i32p]
        lib.sha_oracle_selective_mlp.restype = ctypes.c_int
        lib.sha_oracle_selective_mlp.argtypes = [
            u16p, u16p, u16p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, f64p]
        lib.sha_oracle_select_heads.restype = ctypes.c_int
        lib.sha_oracle_select_heads.argtypes = [
            ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p]
        lib.sha_oracle_num_threads.restype = ctypes.c_int
        lib.sha_oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _bits(x):
    """uint16 bit patterns of an fp16/bf16 array, as a C-contiguous numpy array."""
    if isinstance(x, np.ndarray):
        if x.dtype == np.float16:
            x = x.view(np.uint16)
        if x.dtype != np.uint16:
            raise TypeError(f"expected uint16 bit patterns, got {x.dtype}")
        return np.ascontiguousarray(x)
    import torch  # CPU tensors only; the oracle never touches a device
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"unsupported input type {type(x)}")
    if x.device.type != "cpu":
        raise ValueError("the oracle takes host tensors only")
    if x.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError(f"expected float16/bfloat16, got {x.dtype}")
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


def _dtype_code(dtype):
    if dtype in ("fp16", "float16", FP16):
        return FP16
    if dtype in ("bf16", "bfloat16", BF16):
        return BF16
    import torch
    if dtype == torch.float16:
        return FP16
    if dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unknown dtype {dtype!r}")


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def widen(bits, dtype):
    """Exact float64 value of one fp16/bf16 bit pattern (IEEE definition)."""
    return _load().sha_oracle_widen(int(bits), _dtype_code(dtype))


def num_threads():
    """Host threads the oracle's parallel loops use."""
    return _load().sha_oracle_num_threads()


def sha_decode(q, k, v, batch_head_index, scale, dtype, out=None, tile=0):
    """Selective head decode in float64 over the full layout.

    q: [B, H_q, d], k/v: [B, H_kv, N_kv, d] (a singleton query axis
    ``[B, H_q, 1, d]`` is accepted too), batch_head_index: [B, top_k] int.
    ``out`` (float64 [B, H_q, d]) is written only at the selected heads' rows;
    when omitted it starts as all-NaN so untouched rows stay recognisable.
    ``tile`` = 0 uses the two-pass definition, ``tile`` > 0 Algorithm 1's
    online recurrence with that tile size.
    Returns (out, number_of_out_of_range_ids).
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    if kb.ndim != 4 or kb.shape != vb.shape:
        raise ValueError("k and v must be [B, H_kv, N_kv, d] of one shape")
    B, H_kv, N_kv, d = kb.shape
    qb = qb.reshape(B, -1, d)
    H_q = qb.shape[1]
    idx = np.ascontiguousarray(np.asarray(batch_head_index, dtype=np.int32).reshape(B, -1))
    top_k = idx.shape[1]
    if out is None:
        out = np.full((B, H_q, d), np.nan, dtype=np.float64)
    if out.dtype != np.float64 or not out.flags.c_contiguous or out.shape != (B, H_q, d):
        raise ValueError("out must be a C-contiguous float64 [B, H_q, d] array")
    bad = _load().sha_oracle_decode(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(idx, ctypes.c_int32), B, H_q, H_kv, N_kv, d, top_k, float(scale),
        _dtype_code(dtype), int(tile), _ptr(out, ctypes.c_double))
    if bad < 0:
        raise ValueError("inconsistent sizes")
    return out, int(bad)


def sha_units(q_units, k_units, v_units, scale, dtype, tile=0):
    """Per-unit attention on gathered units: q [n, G, d], k/v [n, N_kv, d] -> float64 [n, G, d]."""
    qb, kb, vb = _bits(q_units), _bits(k_units), _bits(v_units)
    n, N_kv, d = kb.shape
    qb = qb.reshape(n, -1, d)
    G = qb.shape[1]
    out = np.empty((n, G, d), dtype=np.float64)
    rc = _load().sha_oracle_units(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        n, G, N_kv, d, float(scale), _dtype_code(dtype), int(tile),
        _ptr(out, ctypes.c_double))
    if rc != 0:
        raise ValueError("inconsistent sizes")
    return out


def select_heads(scores, top_k):
    """Per-row top-k head ids of router scores [B, H] (float32): decreasing score,
    ties by increasing head id.  Returns int32 [B, top_k]."""
    sc = np.ascontiguousarray(np.asarray(scores, dtype=np.float32))
    if sc.ndim != 2:
        raise ValueError("scores must be [B, H]")
    B, H = sc.shape
    out = np.empty((B, top_k), dtype=np.int32)
    rc = _load().sha_oracle_select_heads(_ptr(sc, ctypes.c_float), B, H, int(top_k),
                                         _ptr(out, ctypes.c_int32))
    if rc != 0:
        raise ValueError("inconsistent sizes")
    return out


def sha_decode_varlen(q, k, v, batch_head_index, seqlens, scale, dtype, out=None):
    """Selective head decode where row b uses only the first seqlens[b] keys of its
    [N_max]-long cache.  Same conventions as sha_decode; rows with a length outside
    [1, N_max] are skipped and counted.  Returns (out, count)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H_kv, N_max, d = kb.shape
    qb = qb.reshape(B, -1, d)
    H_q = qb.shape[1]
    idx = np.ascontiguousarray(np.asarray(batch_head_index, dtype=np.int32).reshape(B, -1))
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(B))
    top_k = idx.shape[1]
    if out is None:
        out = np.full((B, H_q, d), np.nan, dtype=np.float64)
    bad = _load().sha_oracle_decode_varlen(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(idx, ctypes.c_int32), _ptr(lens, ctypes.c_int32), B, H_q, H_kv, N_max, d, top_k,
        float(scale), _dtype_code(dtype), _ptr(out, ctypes.c_double))
    if bad < 0:
        raise ValueError("inconsistent sizes")
    return out, int(bad)


def sha_decode_tokens(q, k, v, batch_head_index, tokens, scale, dtype, out=None):
    """Head x token sparsity: unit (b, slot k) attends only to the keys listed in
    tokens[b, k, :] (int32 [B, top_k, n_sel], positions in [0, N_kv) of its head).
    Units with a position out of range are skipped and counted with bad head
    ids.  Same other conventions as sha_decode.  Returns (out, count)."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, H_kv, N_kv, d = kb.shape
    qb = qb.reshape(B, -1, d)
    H_q = qb.shape[1]
    idx = np.ascontiguousarray(np.asarray(batch_head_index, dtype=np.int32).reshape(B, -1))
    top_k = idx.shape[1]
    tok = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(B, top_k, -1))
    n_sel = tok.shape[2]
    if out is None:
        out = np.full((B, H_q, d), np.nan, dtype=np.float64)
    bad = _load().sha_oracle_decode_tokens(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(idx, ctypes.c_int32), _ptr(tok, ctypes.c_int32), B, H_q, H_kv, N_kv, d, top_k,
        n_sel, float(scale), _dtype_code(dtype), _ptr(out, ctypes.c_double))
    if bad < 0:
        raise ValueError("inconsistent sizes")
    return out, int(bad)


def sha_decode_paged(q, k_pages, v_pages, batch_head_index, seqlens, block_table, scale, dtype,
                     out=None):
    """Selective head decode over a paged cache: k/v_pages [num_pages, H_kv, page_size, d],
    block_table [B, max_pages], seqlens [B].  Returns (out, count of skipped units)."""
    qb, kb, vb = _bits(q), _bits(k_pages), _bits(v_pages)
    num_pages, H_kv, page_size, d = kb.shape
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    B, max_pages = bt.shape
    qb = qb.reshape(B, -1, d)
    H_q = qb.shape[1]
    idx = np.ascontiguousarray(np.asarray(batch_head_index, dtype=np.int32).reshape(B, -1))
    lens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32).reshape(B))
    top_k = idx.shape[1]
    if out is None:
        out = np.full((B, H_q, d), np.nan, dtype=np.float64)
    bad = _load().sha_oracle_decode_paged(
        _ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16), _ptr(vb, ctypes.c_uint16),
        _ptr(idx, ctypes.c_int32), _ptr(lens, ctypes.c_int32), _ptr(bt, ctypes.c_int32),
        B, H_q, H_kv, num_pages, page_size, max_pages, d, top_k, float(scale),
        _dtype_code(dtype), _ptr(out, ctypes.c_double))
    if bad < 0:
        raise ValueError("inconsistent sizes")
    return out, int(bad)


def mlp_union(active):
    """Sorted ids of the neurons active for any row: active [B, D] (bool/uint8)."""
    a = np.ascontiguousarray(np.asarray(active).astype(np.uint8))
    B, D = a.shape
    S = np.empty(D, dtype=np.int32)
    n = _load().sha_oracle_mlp_union(_ptr(a, ctypes.c_uint8), B, D, _ptr(S, ctypes.c_int32))
    if n < 0:
        raise ValueError("inconsistent sizes")
    return S[:n].copy()


def selective_mlp(x, W1t, W2t, S, dtype, act="relu"):
    """sigma(x W1[:, S]) W2[:, S]^T in float64; x [B, d], W1t [D, d], W2t [D, d_out]
    (neuron-major; d_out < d computes a subset of output columns), S neuron ids.
    Returns float64 [B, d_out]."""
    xb, w1, w2 = _bits(x), _bits(W1t), _bits(W2t)
    B, d = xb.shape
    D = w1.shape[0]
    if w1.shape != (D, d) or w2.ndim != 2 or w2.shape[0] != D:
        raise ValueError("W1t must be [D, d] and W2t [D, d_out]")
    d_out = w2.shape[1]
    Sa = np.ascontiguousarray(np.asarray(S, dtype=np.int32))
    y = np.empty((B, d_out), dtype=np.float64)
    rc = _load().sha_oracle_selective_mlp(
        _ptr(xb, ctypes.c_uint16), _ptr(w1, ctypes.c_uint16), _ptr(w2, ctypes.c_uint16),
        _ptr(Sa, ctypes.c_int32), len(Sa), B, d, d_out, D, 1 if act == "relu" else 0,
        _dtype_code(dtype), _ptr(y, ctypes.c_double))
    if rc != 0:
        raise ValueError("inconsistent sizes")
    return y
