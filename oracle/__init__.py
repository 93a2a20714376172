"""CPU oracle of the HySparse2 cross-decoder block (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does.  The
arithmetic lives in ``hs2_oracle.c`` (plain C, fp64); this module compiles it
with gcc and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hs2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

BF16, E4M3 = 0, 1


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_LIB)
        P, I64, I32, D = C.c_void_p, C.c_int64, C.c_int, C.c_double
        L.orc_bridge.argtypes = [P, I64, I32, P, I32, P]
        L.orc_full_attn.argtypes = [I32, P, P, P, P, I32, I32, P, P, I64, I32, D, P, P]
        L.orc_select.argtypes = [I32, P, P, I32, I32, P, P, I64, I32, D, P, I32, I32, P, P]
        L.orc_scores.argtypes = [I32, P, P, I32, I32, P, I32, I32, D, P, P, I64, P]
        L.orc_sparse_attn.argtypes = [I32, P, P, P, P, I32, I32, P, I64, I32, D, P, I32, P, P]
        L.orc_e4m3_value.argtypes = [I32]
        L.orc_e4m3_value.restype = D
        L.orc_bf16_round.argtypes = [P, I64, P]
        L.orc_e4m3_encode.argtypes = [C.c_float]
        L.orc_e4m3_encode.restype = C.c_uint8
        L.orc_quantize_rows.argtypes = [P, P, I64, I32, P, P, P]
        L.orc_threads.restype = I32
        L.orc_set_threads.argtypes = [I32]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def threads() -> int:
    return int(lib().orc_threads())


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def e4m3_table() -> np.ndarray:
    L = lib()
    return np.array([L.orc_e4m3_value(c) for c in range(256)], dtype=np.float64)


def bf16_round(x) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_round(_p(x), x.size, _p(out))
    return out


def bridge(H, W) -> np.ndarray:
    """bf16(H @ W) with fp64 accumulation; H [T, dm], W [dm, N] bf16 bits."""
    H, W = _c(H, np.uint16), _c(W, np.uint16)
    T, dm = H.shape
    N = W.shape[1]
    out = np.empty((T, N), np.uint16)
    lib().orc_bridge(_p(H), T, dm, _p(W), N, _p(out))
    return out


def e4m3_encode(x) -> np.ndarray:
    """e4m3 codes of fp32 values: nearest, ties to the even code, saturated at
    448, sign kept (f1's rounding rule)."""
    L = lib()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([L.orc_e4m3_encode(C.c_float(float(v))) for v in x], dtype=np.uint8)


def bridge_fp8(H, Wk, Wv, Hkv: int, d: int = 128):
    """f1, bridge-only prefill into the FP8 cache: K/V = bf16(H W) as in S1,
    then one fp32 scale per (token, KV head) and e4m3 codes of x / scale.
    Returns (Kc, Vc uint8 [T, Hkv, d], scale float32 [T, Hkv], K, V bf16 bits)."""
    K = bridge(H, Wk)
    V = bridge(H, Wv)
    T = K.shape[0]
    rows = T * Hkv
    Kc = np.empty((T, Hkv, d), np.uint8)
    Vc = np.empty((T, Hkv, d), np.uint8)
    S = np.empty((T, Hkv), np.float32)
    lib().orc_quantize_rows(_p(K), _p(V), rows, d, _p(Kc), _p(Vc), _p(S))
    return Kc, Vc, S, K.reshape(T, Hkv, d), V.reshape(T, Hkv, d)


class KV:
    """K/V source: bf16 bits [T, Hkv, d], or e4m3 codes with scales [T, Hkv]."""

    def __init__(self, K, V, k_scale=None, v_scale=None):
        if k_scale is None:
            self.kind = BF16
            self.K, self.V = _c(K, np.uint16), _c(V, np.uint16)
            self.ks = self.vs = None
        else:
            self.kind = E4M3
            self.K, self.V = _c(K, np.uint8), _c(V, np.uint8)
            self.ks = _c(k_scale, np.float32)
            self.vs = _c(v_scale if v_scale is not None else k_scale, np.float32)
        self.T, self.Hkv, self.d = self.K.shape


def full_attn(kv: KV, Qr, rows, scale: float):
    """Full causal attention for query rows ``rows``; Qr [n, Hq, d] bf16 bits.
    Returns (O [n, Hq, d] fp64, lse [n, Hq] fp64)."""
    Qr, rows = _c(Qr, np.uint16), _c(rows, np.int64)
    n, Hq, d = Qr.shape
    assert rows.max(initial=-1) < kv.T
    O = np.empty((n, Hq, d), np.float64)
    lse = np.empty((n, Hq), np.float64)
    lib().orc_full_attn(kv.kind, _p(kv.K), _p(kv.V), _p(kv.ks), _p(kv.vs), kv.Hkv, d,
                        _p(Qr), _p(rows), n, Hq, scale, _p(O), _p(lse))
    return O, lse


def select(kv: KV, Qr, rows, scale: float, lse, k: int = 1024, w: int = 128):
    """Index lists [n, Hkv, k+w] int32 and k-th scores [n, Hkv] (NaN when every
    candidate is selected)."""
    Qr, rows, lse = _c(Qr, np.uint16), _c(rows, np.int64), _c(lse, np.float64)
    n, Hq, d = Qr.shape
    idx = np.empty((n, kv.Hkv, k + w), np.int32)
    kth = np.empty((n, kv.Hkv), np.float64)
    lib().orc_select(kv.kind, _p(kv.K), _p(kv.ks), kv.Hkv, d, _p(Qr), _p(rows), n, Hq, scale,
                     _p(lse), k, w, _p(idx), _p(kth))
    return idx, kth


def scores(kv: KV, q_row, g: int, scale: float, lse_row, js):
    """score_{i,g,j} for the given positions js; q_row [Hq, d] bf16 bits,
    lse_row [Hq] fp64."""
    q_row, lse_row, js = _c(q_row, np.uint16), _c(lse_row, np.float64), _c(js, np.int64)
    Hq, d = q_row.shape
    out = np.empty(len(js), np.float64)
    lib().orc_scores(kv.kind, _p(kv.K), _p(kv.ks), kv.Hkv, d, _p(q_row), g, Hq, scale,
                     _p(lse_row), _p(js), len(js), _p(out))
    return out


def sparse_attn(kv: KV, Qr, idx, scale: float):
    """Sparse attention of query rows Qr [n, Hq, d] over idx [n, Hkv, kw].
    Returns (O fp64 [n, Hq, d], lse fp64 [n, Hq])."""
    Qr, idx = _c(Qr, np.uint16), _c(idx, np.int32)
    n, Hq, d = Qr.shape
    kw = idx.shape[2]
    O = np.empty((n, Hq, d), np.float64)
    lse = np.empty((n, Hq), np.float64)
    lib().orc_sparse_attn(kv.kind, _p(kv.K), _p(kv.V), _p(kv.ks), _p(kv.vs), kv.Hkv, d,
                          _p(Qr), n, Hq, scale, _p(idx), kw, _p(O), _p(lse))
    return O, lse


def block_rows(kv: KV, Q, Qs, rows, scale: float, k: int = 1024, w: int = 128):
    """The whole block for the given rows: full attention, selection, and one
    sparse layer per entry of Qs (each [n, Hq, d], rows aligned with Q)."""
    O, lse = full_attn(kv, Q, rows, scale)
    idx, kth = select(kv, Q, rows, scale, lse, k, w)
    outs = [sparse_attn(kv, q, idx, scale)[0] for q in Qs]
    return {"O": O, "lse": lse, "idx": idx, "kth": kth, "O_sparse": outs}


def decode(kv_per_seq: list, q, qs: list, scale: float, k: int = 1024, w: int = 128):
    """Decode step: for each sequence b, the block at row N_b - 1 of its cache.
    q [B, Hq, d]; qs: list of [B, Hq, d]."""
    res = []
    for b, kv in enumerate(kv_per_seq):
        rows = np.array([kv.T - 1], np.int64)
        res.append(block_rows(kv, q[b:b + 1], [x[b:b + 1] for x in qs], rows, scale, k, w))
    return res
