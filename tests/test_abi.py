"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments on the host before touching a GPU (no compute here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def _declared_functions():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(HEADER_DIR, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(sha_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    import head_sparse_decode_b200 as h
    return h._lib


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("sha_decode", "sha_decode_bf16", "sha_decode_ex", "sha_decode_workspace_size",
                 "sha_decode_plan", "sha_get_device_status", "sha_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    import head_sparse_decode_b200 as h
    raw = ctypes.CDLL(h.LIBRARY_PATH)
    for name in _declared_functions():
        assert hasattr(raw, name), f"{name} declared in include/ but not exported"


def test_status_strings(lib):
    import head_sparse_decode_b200 as h
    for code in range(8):
        assert h.sha_status_string(code).startswith("SHA_")


_P = ctypes.c_void_p


def _call(lib, B=2, H_q=4, H_kv=4, N_kv=16, d=64, top_k=2, scale=0.125, ptr=0x1000,
          dtype=0, num_splits=0):
    return lib.sha_decode_ex(ptr, ptr, ptr, ptr, B, H_q, H_kv, N_kv, d, top_k,
                             ctypes.c_float(scale), ptr, dtype, None, 0, num_splits, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(d=256), 2),                   # unsupported head dim
    (dict(H_q=6, H_kv=4), 1),                            # H_q not a multiple of H_kv
    (dict(H_q=68, H_kv=4), 2),                           # G = 17 > 16
    (dict(top_k=5), 1), (dict(top_k=-1), 1),             # top_k outside [0, H_kv]
    (dict(N_kv=0), 1), (dict(B=-1), 1),
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1),
    (dict(dtype=7), 2),
    (dict(num_splits=-3), 1),
    (dict(ptr=0x1008), 3),                               # not 16-byte aligned
    (dict(ptr=0), 1),                                    # null
])
def test_host_rejects_bad_arguments_before_any_launch(lib, kw, code):
    assert _call(lib, **kw) == code


@pytest.mark.parametrize("kw", [dict(B=0), dict(top_k=0), dict(B=0, ptr=0)])
def test_empty_problem_is_a_no_op(lib, kw):
    assert _call(lib, **kw) == 0


def test_plan_tiles_and_blocks():
    import head_sparse_decode_b200 as h
    p = h.sha_decode_plan(64, 72, 72, 1920, 128, 22, num_sms=148)
    assert p["tiles_per_head"] == -(-1920 // p["tile_keys"])
    assert p["total_tiles"] == 64 * 22 * p["tiles_per_head"]
    assert p["blocks"] == 148
    # forced splits are clamped to the number of tiles
    p = h.sha_decode_plan(1, 4, 4, 10, 64, 1, num_splits=50, num_sms=148)
    assert p["total_tiles"] == 1 and p["blocks"] == 1 and p["workspace_bytes"] == 0
    # one block per head exactly: no partial states, no workspace
    p = h.sha_decode_plan(4, 8, 8, 640, 128, 2, num_splits=8, num_sms=148)
    assert p["workspace_bytes"] == 0
    # heads straddling blocks need counters and partial states
    p = h.sha_decode_plan(4, 8, 8, 640, 128, 2, num_splits=3, num_sms=148)
    assert p["workspace_bytes"] > 0
    with pytest.raises(h.ShaError):
        h.sha_decode_plan(1, 4, 4, 10, 96, 1)


@pytest.mark.parametrize("B,H,top_k,code", [(2, 300, 3, 2), (2, 8, 9, 1), (2, 0, 0, 1),
                                             (-1, 8, 2, 1), (0, 8, 2, 0), (3, 8, 0, 0)])
def test_select_heads_host_checks(lib, B, H, top_k, code):
    lib.sha_select_heads.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_void_p, ctypes.c_void_p]
    assert lib.sha_select_heads(0x1000, B, H, top_k, 0x2000, None) == code


def test_varlen_and_paged_host_checks(lib):
    P = 0x1000
    lib.sha_decode_varlen.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    # null lengths, unsupported head dim, misaligned lengths
    assert lib.sha_decode_varlen(P, P, P, P, None, 2, 4, 4, 64, 64, 2, 0.1, P, 0, None) == 1
    assert lib.sha_decode_varlen(P, P, P, P, P, 2, 4, 4, 64, 96, 2, 0.1, P, 0, None) == 2
    assert lib.sha_decode_varlen(P, P, P, P, P + 2, 2, 4, 4, 64, 64, 2, 0.1, P, 0, None) == 3
    lib.sha_decode_paged.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 8 + [
        ctypes.c_float, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    # (B, H_q, H_kv, num_pages, page_size, max_pages, d, top_k)
    assert lib.sha_decode_paged(P, P, P, P, P, P, 2, 8, 2, 10, 12, 4, 128, 1, 0.1, P, 1,
                                None) == 2          # GQA needs a power-of-two page size
    assert lib.sha_decode_paged(P, P, P, P, P, P, 2, 8, 2, 10, 0, 4, 128, 1, 0.1, P, 1,
                                None) == 1          # page_size 0
    assert lib.sha_decode_paged(P, P, P, P, None, P, 2, 8, 8, 10, 16, 4, 128, 1, 0.1, P, 0,
                                None) == 1          # no lengths


def test_strided_host_checks(lib):
    P = 0x1000
    lib.sha_decode_strided.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64),
        ctypes.POINTER(ctypes.c_int64), ctypes.c_int, ctypes.c_void_p]
    good = (ctypes.c_int64 * 3)(4 * 64 * 128, 128, 4 * 128)    # token-major [B, N, H, d]
    odd = (ctypes.c_int64 * 3)(4 * 64 * 128, 128, 4 * 128 + 4)  # token stride not 16 bytes
    zero = (ctypes.c_int64 * 3)(4 * 64 * 128, 0, 4 * 128)

    def call(ks, vs, d=128):
        return lib.sha_decode_strided(P, P, P, P, None, 2, 4, 4, 64, d, 2, 0.1, P, ks, vs, 0,
                                      None)
    assert call(None, good) == 1
    assert call(good, zero) == 1
    assert call(good, odd) == 3
    assert call(good, good, d=96) == 2


def test_selective_mlp_host_checks(lib):
    P = 0x1000
    lib.sha_selective_mlp.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    lib.sha_selective_mlp_workspace_size.restype = ctypes.c_size_t
    # batch above 64, d not a multiple of 256, bad activation
    assert lib.sha_selective_mlp(P, P, P, P, P, 65, 256, 512, 1, 0, P, P, 1 << 30, None) == 2
    assert lib.sha_selective_mlp(P, P, P, P, P, 4, 300, 512, 1, 0, P, P, 1 << 30, None) == 2
    assert lib.sha_selective_mlp(P, P, P, P, P, 4, 256, 512, 7, 0, P, P, 1 << 30, None) == 1
    lib.sha_mlp_union.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int] + [
        ctypes.c_void_p] * 3 + [ctypes.c_size_t, ctypes.c_void_p]
    assert lib.sha_mlp_union(P, 0, 100, P, P, P, 1 << 20, None) == 1
    assert lib.sha_mlp_union(P, 2, 100, P, P, P, 1, None) == 7     # workspace too small


def test_tokens_host_checks(lib):
    P = 0x1000
    lib.sha_decode_tokens.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 + [
        ctypes.c_float, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]

    def call(tokens=P, B=2, d=128, top_k=2, n_sel=16, ptr=P):
        # (B, H_q, H_kv, N_kv, d, top_k, n_sel)
        return lib.sha_decode_tokens(ptr, ptr, ptr, ptr, tokens, B, 4, 4, 64, d, top_k, n_sel,
                                     0.1, ptr, 0, None)
    assert call(n_sel=0) == 1                        # no keys listed
    assert call(tokens=None) == 1                    # no list
    assert call(d=96) == 2                           # unsupported head dim
    assert call(top_k=5) == 1                        # top_k above H_kv
    assert call(ptr=0x1008) == 3                     # misaligned cache
    assert call(tokens=None, B=0) == 0               # empty problem: nothing to read


def test_noalloc_host_checks(lib):
    import head_sparse_decode_b200 as h
    P = 0x1000
    lib.sha_decode_noalloc.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]

    def call(H_q=4, H_kv=4, B=2, top_k=2, dtype=0, splits=0, ptr=P):
        return lib.sha_decode_noalloc(ptr, ptr, ptr, ptr, B, H_q, H_kv, 64, 128, top_k, 0.1,
                                      ptr, dtype, splits, None)
    assert call(H_q=8, H_kv=4) == 2                  # grouped queries: not this entry point
    assert call(dtype=7) == 2
    assert call(splits=-1) == 1
    assert call(ptr=0) == 1
    assert call(ptr=0x1008) == 3
    assert call(B=0, ptr=0) == 0                     # empty problem: nothing enqueued
    # the binding reads the array's size from the library as built
    assert lib.sha_noalloc_scratch_bytes() == h.NOALLOC_SCRATCH_BYTES == 512 * 1024


def test_clustered_host_checks(lib):
    P = 0x1000
    lib.sha_decode_clustered.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_void_p]

    def call(cluster=2, d=128):
        return lib.sha_decode_clustered(P, P, P, P, 2, 4, 4, 64, d, 2, 0.1, P, 0, cluster, 2, 0,
                                        None)
    assert call(cluster=1) == 1                      # a cluster holds at least two blocks
    assert call(cluster=0) == 1
    assert call(d=96) == 2
