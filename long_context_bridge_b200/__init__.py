"""Python binding of libhs2 (the HySparse2 cross-decoder block for B200).

Argument marshalling only: every function checks tensor dtypes, devices and
contiguity, then calls the C entry point of the same name with raw device
pointers and the current CUDA stream.  All computation runs in the library's
CUDA kernels.  There is no fallback: if ``libhs2.so`` is missing or fails to
load, importing this package raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhs2.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_BAD_INDEX = range(7)
OP_BRIDGE, OP_FULL_ATTN, OP_SELECT, OP_SPARSE, OP_BLOCK_PREFILL, OP_BLOCK_DECODE, OP_SPARSE_PLAN = range(7)


class HS2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_lib.hs2_status_string(status).decode()} (status {status})")
        self.status = status


class Shape(C.Structure):
    """hs2_shape: T, n_q_heads, n_kv_heads, head_dim, scale, k_global, window."""
    _fields_ = [("T", C.c_int64), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32),
                ("head_dim", C.c_int32), ("scale", C.c_float), ("k_global", C.c_int32),
                ("window", C.c_int32)]

    @classmethod
    def make(cls, T, n_q_heads, n_kv_heads, head_dim=128, scale=None, k_global=1024, window=128):
        if scale is None:
            scale = head_dim ** -0.5
        return cls(int(T), int(n_q_heads), int(n_kv_heads), int(head_dim), float(scale),
                   int(k_global), int(window))


def _load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(f"libhs2.so not built at {path}: run long_context_bridge_b200/build.py")
    L = C.CDLL(path)
    P, I32, I64, SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    SP = C.POINTER(Shape)
    PP = C.POINTER(C.c_void_p)
    sigs = {
        "hs2_bridge_kv": [P, I32, P, P, P, P, SP, P],
        "hs2_bridge_kv_fp8": [P, I32, P, P, P, P, P, SP, P],
        "hs2_full_attn_lse": [P, P, P, P, P, SP, P],
        "hs2_select_topk": [P, P, P, P, P, SP, P, SZ, P],
        "hs2_select_topk_noalloc": [P, P, P, P, P, SP, P],
        "hs2_sparse_attn": [P, P, P, P, P, P, SP, P],
        "hs2_sparse_attn_layers": [I32, PP, P, P, P, PP, PP, SP, P],
        "hs2_sparse_plan": [P, SP, P, SZ, P],
        "hs2_sparse_attn_planned": [P, P, P, P, P, P, SP, P],
        "hs2_block_prefill": [P, I32, P, P, P, P, P, P, P, P, I32, PP, PP, SP, P, SZ, P],
        "hs2_block_decode": [I32, C.POINTER(C.c_int64), P, P, P, P, P, P, P, P, I32, PP, PP, SP,
                             P, SZ, P],
        "hs2_block_prefill_rows": [I64, P, P, P, P, P, P, I32, PP, PP, SP, P, SZ, P],
        "hs2_debug_read_probe": [P, SZ, I32, P, P],
        "hs2_debug_set_select_speculation": [C.c_float],
        "hs2_decode_cp_attn": [I32, C.POINTER(C.c_int64), C.POINTER(C.c_int64),
                               C.POINTER(C.c_int64), P, P, P, P, P, P, SP, P, SZ, P],
        "hs2_decode_cp_select": [I32, C.POINTER(C.c_int64), C.POINTER(C.c_int64),
                                 C.POINTER(C.c_int64), I32, P, P, P, P, SP, P, SZ, P],
        "hs2_decode_cp_sparse": [I32, C.POINTER(C.c_int64), C.POINTER(C.c_int64),
                                 C.POINTER(C.c_int64), I32, P, P, P, P, P, P, I32, PP, P, SP, P],
        "hs2_decode_cp_finish": [I32, I32, I32, P, PP, SP, P],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = C.c_int
    L.hs2_workspace_size.argtypes = [I32, SP, I32, I32]
    L.hs2_workspace_size.restype = SZ
    L.hs2_get_device_status.argtypes = [P]
    L.hs2_get_device_status.restype = C.c_int
    L.hs2_status_string.argtypes = [C.c_int]
    L.hs2_status_string.restype = C.c_char_p
    L.hs2_kernel_launches.restype = C.c_uint64
    L.hs2_debug_set_wait_budget.argtypes = [C.c_int64]
    L.hs2_debug_set_wait_budget.restype = C.c_int
    return L


_lib = _load()

EXPORTED = ["hs2_bridge_kv", "hs2_bridge_kv_fp8", "hs2_full_attn_lse", "hs2_select_topk", "hs2_select_topk_noalloc",
            "hs2_sparse_attn", "hs2_sparse_attn_layers", "hs2_sparse_plan", "hs2_sparse_attn_planned",
            "hs2_block_prefill", "hs2_block_decode", "hs2_workspace_size",
            "hs2_get_device_status", "hs2_status_string", "hs2_kernel_launches",
            "hs2_debug_set_wait_budget", "hs2_debug_read_probe", "hs2_block_prefill_rows",
            "hs2_debug_set_select_speculation",
            "hs2_decode_cp_attn",
            "hs2_decode_cp_select",
            "hs2_decode_cp_sparse", "hs2_decode_cp_finish"]


def _ptr(t, dtype, what, nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{what} is required")
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _check(status, what):
    if status != OK:
        raise HS2Error(status, what)


BF16, F32, I32T, U8 = torch.bfloat16, torch.float32, torch.int32, torch.uint8


def workspace_size(op: int, shape: Shape, batch: int = 1, d_model: int = 0) -> int:
    n = _lib.hs2_workspace_size(op, C.byref(shape), batch, d_model)
    if n == C.c_size_t(-1).value:
        raise HS2Error(ERR_INVALID_ARG, "hs2_workspace_size")
    return int(n)


def hs2_bridge_kv(H, W_k, W_v, K, V, shape: Shape, stream=None):
    _check(_lib.hs2_bridge_kv(_ptr(H, BF16, "H"), H.shape[-1], _ptr(W_k, BF16, "W_k"),
                              _ptr(W_v, BF16, "W_v"), _ptr(K, BF16, "K"), _ptr(V, BF16, "V"),
                              C.byref(shape), _stream(stream)), "hs2_bridge_kv")


def hs2_bridge_kv_fp8(H, W_k, W_v, Kc, Vc, scale, shape: Shape, stream=None):
    _check(_lib.hs2_bridge_kv_fp8(_ptr(H, BF16, "H"), H.shape[-1], _ptr(W_k, BF16, "W_k"),
                                  _ptr(W_v, BF16, "W_v"), _ptr(Kc, U8, "Kc"), _ptr(Vc, U8, "Vc"),
                                  _ptr(scale, F32, "scale"), C.byref(shape), _stream(stream)),
           "hs2_bridge_kv_fp8")


def hs2_full_attn_lse(Q, K, V, O, lse, shape: Shape, stream=None):
    _check(_lib.hs2_full_attn_lse(_ptr(Q, BF16, "Q"), _ptr(K, BF16, "K"), _ptr(V, BF16, "V"),
                                  _ptr(O, BF16, "O"), _ptr(lse, F32, "lse"), C.byref(shape),
                                  _stream(stream)), "hs2_full_attn_lse")


def hs2_select_topk(Q, K, lse, idx, kth, shape: Shape, workspace, stream=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.hs2_select_topk(_ptr(Q, BF16, "Q"), _ptr(K, BF16, "K"), _ptr(lse, F32, "lse"),
                                _ptr(idx, I32T, "idx"), _ptr(kth, F32, "kth", True),
                                C.byref(shape), _ptr(workspace, U8, "workspace", True), nbytes,
                                _stream(stream)), "hs2_select_topk")


def hs2_select_topk_noalloc(Q, K, lse, idx, kth, shape: Shape, stream=None):
    """hs2_select_topk on the library's own scratch, for callers that cannot
    allocate device memory; see include/hs2.h for its limits."""
    _check(_lib.hs2_select_topk_noalloc(_ptr(Q, BF16, "Q"), _ptr(K, BF16, "K"),
                                        _ptr(lse, F32, "lse"), _ptr(idx, I32T, "idx"),
                                        _ptr(kth, F32, "kth", True), C.byref(shape),
                                        _stream(stream)), "hs2_select_topk_noalloc")


def hs2_sparse_attn(Q, K, V, idx, O, lse, shape: Shape, stream=None):
    _check(_lib.hs2_sparse_attn(_ptr(Q, BF16, "Q"), _ptr(K, BF16, "K"), _ptr(V, BF16, "V"),
                                _ptr(idx, I32T, "idx"), _ptr(O, BF16, "O"),
                                _ptr(lse, F32, "lse", True), C.byref(shape), _stream(stream)),
           "hs2_sparse_attn")


def hs2_sparse_plan(idx, shape: Shape, plan, stream=None):
    nbytes = plan.numel() * plan.element_size()
    _check(_lib.hs2_sparse_plan(_ptr(idx, I32T, "idx"), C.byref(shape), _ptr(plan, U8, "plan"),
                                nbytes, _stream(stream)), "hs2_sparse_plan")


def hs2_sparse_attn_planned(Q, K, V, plan, O, lse, shape: Shape, stream=None):
    _check(_lib.hs2_sparse_attn_planned(_ptr(Q, BF16, "Q"), _ptr(K, BF16, "K"), _ptr(V, BF16, "V"),
                                        _ptr(plan, U8, "plan"), _ptr(O, BF16, "O"),
                                        _ptr(lse, F32, "lse", True), C.byref(shape),
                                        _stream(stream)), "hs2_sparse_attn_planned")


def _ptr_array(ts, dtype, what):
    arr = (C.c_void_p * max(1, len(ts)))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t, dtype, f"{what}[{i}]").value
    return C.cast(arr, C.POINTER(C.c_void_p)), arr


def hs2_sparse_attn_layers(Qs, K, V, idx, Os, lses, shape: Shape, stream=None):
    qs, _keep_q = _ptr_array(Qs, BF16, "Q")
    os_, _keep_o = _ptr_array(Os, BF16, "O")
    ls = None
    if lses is not None:
        ls = (C.c_void_p * max(1, len(lses)))(*[_ptr(t, F32, "lse", True) for t in lses])
    _check(_lib.hs2_sparse_attn_layers(len(Qs), qs, _ptr(K, BF16, "K"), _ptr(V, BF16, "V"),
                                       _ptr(idx, I32T, "idx"), os_, ls, C.byref(shape),
                                       _stream(stream)), "hs2_sparse_attn_layers")


def hs2_block_prefill(H, W_k, W_v, K, V, Q_full, O_full, lse, idx, Q_sparse, O_sparse,
                      shape: Shape, workspace, stream=None):
    qs, _keep_q = _ptr_array(Q_sparse, BF16, "Q_sparse")
    os_, _keep_o = _ptr_array(O_sparse, BF16, "O_sparse")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.hs2_block_prefill(
        _ptr(H, BF16, "H", True), 0 if H is None else H.shape[-1], _ptr(W_k, BF16, "W_k", True),
        _ptr(W_v, BF16, "W_v", True), _ptr(K, BF16, "K"), _ptr(V, BF16, "V"),
        _ptr(Q_full, BF16, "Q_full"), _ptr(O_full, BF16, "O_full"), _ptr(lse, F32, "lse"),
        _ptr(idx, I32T, "idx"), len(Q_sparse), qs, os_, C.byref(shape),
        _ptr(workspace, U8, "workspace", True), nbytes, _stream(stream)), "hs2_block_prefill")


def hs2_block_prefill_rows(q_begin, K, V, Q_full, O_full, lse, idx, Q_sparse, O_sparse,
                           shape: Shape, workspace, stream=None):
    qs, _keep_q = _ptr_array(Q_sparse, BF16, "Q_sparse")
    os_, _keep_o = _ptr_array(O_sparse, BF16, "O_sparse")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.hs2_block_prefill_rows(
        int(q_begin), _ptr(K, BF16, "K"), _ptr(V, BF16, "V"), _ptr(Q_full, BF16, "Q_full"),
        _ptr(O_full, BF16, "O_full"), _ptr(lse, F32, "lse"), _ptr(idx, I32T, "idx"),
        len(Q_sparse), qs, os_, C.byref(shape), _ptr(workspace, U8, "workspace", True), nbytes,
        _stream(stream)), "hs2_block_prefill_rows")


def hs2_block_decode(seq_len, q_full, Kc, Vc, k_scale, v_scale, o_full, lse, idx, q_sparse,
                     o_sparse, shape: Shape, workspace, stream=None):
    B = len(seq_len)
    lens = (C.c_int64 * B)(*[int(x) for x in seq_len])
    qs, _keep_q = _ptr_array(q_sparse, BF16, "q_sparse")
    os_, _keep_o = _ptr_array(o_sparse, BF16, "o_sparse")
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.hs2_block_decode(
        B, lens, _ptr(q_full, BF16, "q_full"), _ptr(Kc, U8, "Kc"), _ptr(Vc, U8, "Vc"),
        _ptr(k_scale, F32, "k_scale"), _ptr(v_scale, F32, "v_scale"), _ptr(o_full, BF16, "o_full"),
        _ptr(lse, F32, "lse"), _ptr(idx, I32T, "idx"), len(q_sparse), qs, os_, C.byref(shape),
        _ptr(workspace, U8, "workspace", True), nbytes, _stream(stream)), "hs2_block_decode")



def _i64s(xs):
    return (C.c_int64 * len(xs))(*[int(x) for x in xs])


DECODE_REC_FLOATS = 130   # softmax-state record: m, l, o[128]


def hs2_decode_cp_attn(seq_len, slice_lo, slice_hi, q_full, Kc, Vc, k_scale, v_scale, attn_rec,
                       shape: Shape, workspace, stream=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.hs2_decode_cp_attn(
        len(seq_len), _i64s(seq_len), _i64s(slice_lo), _i64s(slice_hi),
        _ptr(q_full, BF16, "q_full"), _ptr(Kc, U8, "Kc"), _ptr(Vc, U8, "Vc"),
        _ptr(k_scale, F32, "k_scale"), _ptr(v_scale, F32, "v_scale"),
        _ptr(attn_rec, F32, "attn_rec"), C.byref(shape), _ptr(workspace, U8, "workspace", True),
        nbytes, _stream(stream)), "hs2_decode_cp_attn")


def hs2_decode_cp_select(seq_len, slice_lo, slice_hi, n_ranks, attn_recs, o_full, lse, sel_rec,
                         shape: Shape, workspace, stream=None):
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.hs2_decode_cp_select(
        len(seq_len), _i64s(seq_len), _i64s(slice_lo), _i64s(slice_hi), int(n_ranks),
        _ptr(attn_recs, F32, "attn_recs"), _ptr(o_full, BF16, "o_full"), _ptr(lse, F32, "lse"),
        _ptr(sel_rec, I32T, "sel_rec"), C.byref(shape), _ptr(workspace, U8, "workspace", True),
        nbytes, _stream(stream)), "hs2_decode_cp_select")


def hs2_decode_cp_sparse(seq_len, slice_lo, slice_hi, n_ranks, sel_recs, idx, Kc, Vc, k_scale,
                         v_scale, q_sparse, sparse_rec, shape: Shape, stream=None):
    qs, _keep_q = _ptr_array(q_sparse, BF16, "q_sparse")
    _check(_lib.hs2_decode_cp_sparse(
        len(seq_len), _i64s(seq_len), _i64s(slice_lo), _i64s(slice_hi), int(n_ranks),
        _ptr(sel_recs, I32T, "sel_recs"), _ptr(idx, I32T, "idx"), _ptr(Kc, U8, "Kc"),
        _ptr(Vc, U8, "Vc"), _ptr(k_scale, F32, "k_scale"), _ptr(v_scale, F32, "v_scale"),
        len(q_sparse), qs, _ptr(sparse_rec, F32, "sparse_rec", True), C.byref(shape),
        _stream(stream)), "hs2_decode_cp_sparse")


def hs2_decode_cp_finish(n_ranks, sparse_recs, o_sparse, shape: Shape, stream=None):
    os_, _keep_o = _ptr_array(o_sparse, BF16, "o_sparse")
    batch = o_sparse[0].shape[0]
    _check(_lib.hs2_decode_cp_finish(batch, int(n_ranks), len(o_sparse),
                                     _ptr(sparse_recs, F32, "sparse_recs"), os_, C.byref(shape),
                                     _stream(stream)), "hs2_decode_cp_finish")


def hs2_get_device_status(stream=None) -> int:
    return int(_lib.hs2_get_device_status(_stream(stream)))


def hs2_debug_set_wait_budget(cycles: int) -> None:
    """Testing hook: spin budget of the kernels' bounded waits (<= 0: default)."""
    _check(_lib.hs2_debug_set_wait_budget(int(cycles)), "hs2_debug_set_wait_budget")


def hs2_debug_read_probe(buf, reps: int, sink, stream=None) -> None:
    """Measurement hook: `reps` passes of 16-byte loads over the uint8 buffer."""
    _check(_lib.hs2_debug_read_probe(_ptr(buf, U8, "buf"), buf.numel(), int(reps),
                                     _ptr(sink, I32T, "sink"), _stream(stream)),
           "hs2_debug_read_probe")


def hs2_debug_set_select_speculation(factor: float) -> None:
    """Testing hook: starting fraction of the selection's speculative floor."""
    _check(_lib.hs2_debug_set_select_speculation(float(factor)),
           "hs2_debug_set_select_speculation")


def hs2_kernel_launches() -> int:
    return int(_lib.hs2_kernel_launches())


def hs2_status_string(status: int) -> str:
    return _lib.hs2_status_string(status).decode()
