"""The C-ABI library loads, exports every entry point include/hs2.h declares,
and rejects bad arguments on the host before touching the GPU (CPU only)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hs2():
    from long_context_bridge_b200 import build
    build.build()
    import long_context_bridge_b200 as m
    return m


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "hs2.h")).read()
    return set(re.findall(r"^\s*(?:hs2_status|size_t|const char\*|uint64_t)\s+(hs2_\w+)\s*\(",
                          text, flags=re.M))


def test_exports_match_header(hs2):
    decl = declared_symbols()
    assert {"hs2_bridge_kv", "hs2_full_attn_lse", "hs2_select_topk", "hs2_sparse_attn",
            "hs2_block_prefill", "hs2_block_decode"} <= decl
    lib = C.CDLL(hs2.LIB_PATH)
    for name in decl:
        assert hasattr(lib, name), name
    assert decl == set(hs2.EXPORTED)


def _raw(hs2):
    return hs2._lib


def test_host_side_errors(hs2):
    L = _raw(hs2)
    ok_ptr = C.c_void_p(0x10000)
    bad_ptr = C.c_void_p(0x10001)
    s = hs2.Shape.make(1024, 8, 2)
    # head_dim other than 128 is unsupported
    s64 = hs2.Shape.make(1024, 8, 2, head_dim=64)
    assert L.hs2_full_attn_lse(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s64), None) == hs2.ERR_UNSUPPORTED
    # Hq not a multiple of Hkv, G = 3, G = 32
    for hq, hkv in ((7, 2), (6, 2), (64, 2)):
        sh = hs2.Shape.make(1024, hq, hkv)
        assert L.hs2_full_attn_lse(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(sh), None) == hs2.ERR_UNSUPPORTED
    # null, misaligned, T <= 0
    assert L.hs2_full_attn_lse(None, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s), None) == hs2.ERR_INVALID_ARG
    assert L.hs2_full_attn_lse(ok_ptr, bad_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s), None) == hs2.ERR_INVALID_ARG
    s0 = hs2.Shape.make(0, 8, 2)
    assert L.hs2_full_attn_lse(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s0), None) == hs2.ERR_INVALID_ARG
    # bad selection budget
    sk = hs2.Shape.make(1024, 8, 2, k_global=-1)
    assert L.hs2_sparse_attn(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, C.byref(sk), None) == hs2.ERR_INVALID_ARG
    sw = hs2.Shape.make(1024, 8, 2, window=0)
    assert L.hs2_sparse_attn(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, C.byref(sw), None) == hs2.ERR_INVALID_ARG
    # bridge: d_model must be a positive multiple of 64
    assert L.hs2_bridge_kv(ok_ptr, 100, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s), None) == hs2.ERR_INVALID_ARG
    # bridge into the FP8 cache: null output, misaligned scale, bad d_model
    assert L.hs2_bridge_kv_fp8(ok_ptr, 128, ok_ptr, ok_ptr, None, ok_ptr, ok_ptr, C.byref(s),
                               None) == hs2.ERR_INVALID_ARG
    assert L.hs2_bridge_kv_fp8(ok_ptr, 128, ok_ptr, ok_ptr, ok_ptr, ok_ptr, bad_ptr, C.byref(s),
                               None) == hs2.ERR_INVALID_ARG
    assert L.hs2_bridge_kv_fp8(ok_ptr, 96, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s),
                               None) == hs2.ERR_INVALID_ARG
    assert L.hs2_bridge_kv_fp8(ok_ptr, 128, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, C.byref(s64),
                               None) == hs2.ERR_UNSUPPORTED
    # fused sparse layers: no layers, a null or misaligned layer pointer
    two = (C.c_void_p * 2)(0x10000, 0x20000)
    one_null = (C.c_void_p * 2)(0x10000, None)
    one_bad = (C.c_void_p * 2)(0x10000, 0x20001)
    P = C.POINTER(C.c_void_p)
    for n, q, o in ((0, two, two), (2, one_null, two), (2, two, one_bad)):
        assert L.hs2_sparse_attn_layers(n, C.cast(q, P), ok_ptr, ok_ptr, ok_ptr, C.cast(o, P), None,
                                        C.byref(s), None) == hs2.ERR_INVALID_ARG
    # workspace too small for selection
    need = hs2.workspace_size(hs2.OP_SELECT, s)
    if need > 0:
        assert L.hs2_select_topk(ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, C.byref(s), ok_ptr,
                                 need - 16, None) == hs2.ERR_WORKSPACE
        assert L.hs2_select_topk(ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, C.byref(s), None,
                                 need, None) == hs2.ERR_WORKSPACE
    # decode: sequence longer than the cache
    lens = (C.c_int64 * 2)(10, 5000)
    sd = hs2.Shape.make(4096, 8, 2)
    arr = (C.c_void_p * 1)()
    assert L.hs2_block_decode(2, lens, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                              ok_ptr, 0, C.cast(arr, C.POINTER(C.c_void_p)),
                              C.cast(arr, C.POINTER(C.c_void_p)), C.byref(sd), ok_ptr, 1 << 40,
                              None) == hs2.ERR_INVALID_ARG
    # decode limits, checked before any launch: batch > 64, batch * capacity >= 2^31
    lens65 = (C.c_int64 * 65)(*([10] * 65))
    assert L.hs2_block_decode(65, lens65, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                              ok_ptr, 0, C.cast(arr, C.POINTER(C.c_void_p)),
                              C.cast(arr, C.POINTER(C.c_void_p)), C.byref(sd), ok_ptr, 1 << 40,
                              None) == hs2.ERR_UNSUPPORTED
    big = hs2.Shape.make(1 << 28, 8, 2)
    lens8 = (C.c_int64 * 8)(*([10] * 8))
    assert L.hs2_block_decode(8, lens8, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                              ok_ptr, 0, C.cast(arr, C.POINTER(C.c_void_p)),
                              C.cast(arr, C.POINTER(C.c_void_p)), C.byref(big), ok_ptr, 1 << 40,
                              None) == hs2.ERR_UNSUPPORTED
    with pytest.raises(hs2.HS2Error):
        hs2.workspace_size(hs2.OP_BLOCK_DECODE, sd, 65)
    # context-parallel decode: a slice past the sequence, a slice longer than
    # the local cache, too many ranks for the merge of their top-k records
    i64 = lambda *v: (C.c_int64 * len(v))(*v)
    sh = hs2.Shape.make(4096, 8, 2)
    assert L.hs2_decode_cp_attn(1, i64(5000), i64(4000), i64(5001), ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                                ok_ptr, ok_ptr, C.byref(sh), ok_ptr, 1 << 40,
                                None) == hs2.ERR_INVALID_ARG
    assert L.hs2_decode_cp_attn(1, i64(9000), i64(0), i64(4097), ok_ptr, ok_ptr, ok_ptr, ok_ptr,
                                ok_ptr, ok_ptr, C.byref(sh), ok_ptr, 1 << 40,
                                None) == hs2.ERR_INVALID_ARG
    assert L.hs2_decode_cp_select(1, i64(9000), i64(0), i64(4096), 9, ok_ptr, ok_ptr, ok_ptr,
                                  ok_ptr, C.byref(sh), ok_ptr, 1 << 40, None) == hs2.ERR_UNSUPPORTED
    assert L.hs2_decode_cp_finish(1, 0, 1, ok_ptr, C.cast(arr, C.POINTER(C.c_void_p)),
                                  C.byref(sh), None) == hs2.ERR_INVALID_ARG
    assert hs2.hs2_status_string(hs2.ERR_TIMEOUT) == "device-side wait timed out"
    assert hs2.hs2_status_string(hs2.ERR_BAD_INDEX) == "index list entry out of range (skipped)"


def test_workspace_size_queries(hs2):
    s = hs2.Shape.make(32768, 16, 2)
    assert hs2.workspace_size(hs2.OP_FULL_ATTN, s) == 0
    assert hs2.workspace_size(hs2.OP_SPARSE, s) == 0
    with pytest.raises(hs2.HS2Error):
        hs2.workspace_size(hs2.OP_FULL_ATTN, hs2.Shape.make(32768, 16, 2, head_dim=96))


def test_sparse_plan_sizes_and_host_checks(hs2):
    """The union plan's size follows its layout (per item of 256/G query rows:
    a (count, mask) pair, then positions and masks for (256/G)(k+w) entries
    rounded up to 128, per KV head), and the two plan calls reject unsupported
    shapes, missing buffers and a short plan on the host."""
    L = _raw(hs2)
    ok_ptr = C.c_void_p(0x10000)
    for T, hq, hkv, k, w in ((131072, 32, 4, 1024, 128), (1000, 16, 1, 2048, 256), (700, 32, 2, 64, 16)):
        P = 256 // (hq // hkv)
        s = hs2.Shape.make(T, hq, hkv, k_global=k, window=w)
        items = -(-T // P) * hkv
        cap = -(-(P * (k + w)) // 128) * 128
        want = -(-(items * 8) // 256) * 256 + 2 * items * cap * 4
        assert hs2.workspace_size(hs2.OP_SPARSE_PLAN, s) == want
        # a plan one byte short
        assert L.hs2_sparse_plan(ok_ptr, C.byref(s), ok_ptr, want - 1, None) == hs2.ERR_WORKSPACE
        assert L.hs2_sparse_plan(None, C.byref(s), ok_ptr, want, None) == hs2.ERR_INVALID_ARG
        assert L.hs2_sparse_attn_planned(ok_ptr, ok_ptr, ok_ptr, None, ok_ptr, None, C.byref(s),
                                         None) == hs2.ERR_INVALID_ARG
    # no plan path: G outside {8, 16}, or (256/G)(k + w) above 36864
    for hq, hkv, k, w in ((8, 2, 64, 16), (8, 1, 1024, 256), (64, 4, 2048, 512)):
        s = hs2.Shape.make(4096, hq, hkv, k_global=k, window=w)
        with pytest.raises(hs2.HS2Error):
            hs2.workspace_size(hs2.OP_SPARSE_PLAN, s)
        assert L.hs2_sparse_plan(ok_ptr, C.byref(s), ok_ptr, 1 << 40, None) == hs2.ERR_UNSUPPORTED
        assert L.hs2_sparse_attn_planned(ok_ptr, ok_ptr, ok_ptr, ok_ptr, ok_ptr, None, C.byref(s),
                                         None) == hs2.ERR_UNSUPPORTED
    # the block prefill's workspace covers a plan slab (32768 rows) as well as the selection
    s = hs2.Shape.make(131072, 32, 4)
    slab_items = 32768 // 32 * 4
    slab = -(-(slab_items * 8) // 256) * 256 + 2 * slab_items * 1152 * 32 * 4
    assert hs2.workspace_size(hs2.OP_BLOCK_PREFILL, s) >= slab
