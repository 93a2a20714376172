"""Seeded synthetic inputs for the HySparse2 cross-decoder block.

This module is shared by the CPU oracle's tests and by the GPU path's tests and
bench.  It holds no arithmetic of the method (no projection, attention, scoring
or selection): only random numbers, their rounding to the storage formats, and
the placement of planted "needle" keys.

Random numbers
--------------
A counter-based generator, so that any element of any tensor can be produced on
its own (a sampled row needs no neighbours):

* ``mix(z)`` is the SplitMix64 output function (Steele, Lea, Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014);
* the stream of tensor ``tid`` under ``seed`` has key
  ``key = mix(seed * GAMMA + tid)`` and its element ``e`` draws
  ``r(e) = mix(key + (e + 1) * GAMMA)`` (all arithmetic mod 2**64), i.e. the
  e-th output of a SplitMix64 generator started at ``key``;
* a uniform is ``u = ((r >> 11) + 0.5) * 2**-53`` in (0, 1);
* normal number ``e`` of a tensor is Box-Muller on the uniforms of draws
  ``2e`` and ``2e+1``: ``sqrt(-2 ln u1) * cos(2 pi u2)`` (fp64);
* stored bf16 values are fp64 -> fp32 (round to nearest even) -> bf16 (round
  to nearest even).

The same generator exists twice: in numpy (the definition, used for every input
the CPU oracle sees at sizes the host can generate) and in torch int64 ops (for
the full-size GPU workloads).  A test pins the two to each other bit for bit.

Workloads (the five block configurations)
-----------------------------------------
C1 tiny block, C2 32K block with bridge, C3 128K block with bridge, C4 1M block,
C5 1M-context FP8 decode over a batch of 8.  Shapes, value distributions and
needle counts follow the configuration list of the block; ``seed = 20260925 +
config number``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_U64 = np.uint64

# tensor ids of the streams
TID_H, TID_WK, TID_WV, TID_Q = 1, 2, 3, 4
TID_QS0 = 5            # sparse layer l uses TID_QS0 + l
TID_K, TID_V = 10, 11
TID_NEEDLE_POS, TID_NEEDLE_DIR = 20, 21
TID_DEC_K0, TID_DEC_V0, TID_DEC_POS0 = 100, 200, 300   # + sequence number


# ----------------------------------------------------------------------------
# numpy generator (the definition)
# ----------------------------------------------------------------------------
def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> _U64(30))) * _U64(_M1)
    z = (z ^ (z >> _U64(27))) * _U64(_M2)
    return z ^ (z >> _U64(31))


def stream_key(seed: int, tid: int) -> int:
    z = np.array([(seed * GAMMA + tid) % (1 << 64)], dtype=np.uint64)
    return int(_mix_np(z)[0])


def draws_np(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    """r(e) for e in [start, start+count) as uint64."""
    key = _U64(stream_key(seed, tid))
    e = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix_np(key + e * _U64(GAMMA))


def uniforms_np(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    r = draws_np(seed, tid, start, count)
    return ((r >> _U64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normals_np(seed: int, tid: int, start: int, count: int) -> np.ndarray:
    """Normal numbers start..start+count-1 of stream (seed, tid), fp64."""
    u = uniforms_np(seed, tid, 2 * start, 2 * count)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_np(seed: int, tid: int, start: int, count: int, sd: float = 1.0,
                   chunk: int = 1 << 24) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    for s in range(0, count, chunk):
        c = min(chunk, count - s)
        out[s:s + c] = f64_to_bf16_bits(normals_np(seed, tid, start + s, c) * sd)
    return out


# ----------------------------------------------------------------------------
# torch generator (same definition in int64 arithmetic, for device tensors)
# ----------------------------------------------------------------------------
def _s64(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


def _mix_torch(z):
    m34, m37, m33 = (1 << 34) - 1, (1 << 37) - 1, (1 << 33) - 1
    z = (z ^ ((z >> 30) & m34)) * _s64(_M1)
    z = (z ^ ((z >> 27) & m37)) * _s64(_M2)
    return z ^ ((z >> 31) & m33)


def normals_torch(seed: int, tid: int, start: int, count: int, device="cuda"):
    import torch
    key = _s64(stream_key(seed, tid))
    e = torch.arange(2 * start + 1, 2 * (start + count) + 1, dtype=torch.int64, device=device)
    r = _mix_torch(e * _s64(GAMMA) + key)
    u = (((r >> 11) & ((1 << 53) - 1)).to(torch.float64) + 0.5) * (2.0 ** -53)
    u1, u2 = u[0::2], u[1::2]
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)


def normal_bf16_torch(seed: int, tid: int, start: int, count: int, sd: float = 1.0,
                      device="cuda", chunk: int = 1 << 26):
    import torch
    out = torch.empty(count, dtype=torch.bfloat16, device=device)
    for s in range(0, count, chunk):
        c = min(chunk, count - s)
        out[s:s + c] = (normals_torch(seed, tid, start + s, c, device) * sd).float().bfloat16()
    return out


# ----------------------------------------------------------------------------
# FP8 e4m3 (OCP E4M3FN) quantiser used to build decode caches
# ----------------------------------------------------------------------------
def _e4m3_positive_values() -> np.ndarray:
    """Values of codes 0x00..0x7E (sign 0, finite), from the format: bias 7,
    3 mantissa bits, subnormals at exponent field 0, 0x7F is NaN."""
    vals = np.empty(127, dtype=np.float64)
    for c in range(127):
        e, m = c >> 3, c & 7
        vals[c] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3_POS = _e4m3_positive_values()


def e4m3_quantize_np(x: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to e4m3fn codes: nearest, ties to even code,
    magnitudes above 448 saturate to 448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    hi = np.searchsorted(_E4M3_POS, a, side="left").clip(0, 126)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - _E4M3_POS[lo], _E4M3_POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a == _E4M3_POS[hi], hi, code).astype(np.uint8)
    sign = (np.signbit(x) & (code != 0)).astype(np.uint8) << np.uint8(7)
    return code | sign


# ----------------------------------------------------------------------------
# Workload definitions
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class BlockConfig:
    name: str
    number: int
    T: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int = 128
    n_sparse: int = 3
    d_model: int = 0          # 0: K/V are inputs (no bridge)
    n_needles: int = 0        # per KV head (per sequence for decode)
    q_mix: bool = False       # Q rows = 0.5 z + 0.5 sqrt(d) u_g
    batch: int = 1            # decode batch (C5)
    fp8_cache: bool = False
    k_global: int = 1024
    window: int = 128

    @property
    def seed(self) -> int:
        return 20260925 + self.number

    @property
    def G(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


CONFIGS = {
    "C1": BlockConfig("tiny block T=2048 4q/1kv", 1, 2048, 4, 1, n_sparse=1),
    "C2": BlockConfig("block T=32768 16q/2kv bridge", 2, 32768, 16, 2, d_model=2048,
                      n_needles=64),
    "C3": BlockConfig("block T=131072 32q/4kv bridge", 3, 131072, 32, 4, d_model=2048,
                      n_needles=256, q_mix=True),
    "C4": BlockConfig("block T=1048576 32q/4kv", 4, 1 << 20, 32, 4, n_needles=1024,
                      q_mix=True),
    "C5": BlockConfig("decode 8 x 1048576 fp8 cache 32q/4kv", 5, 1 << 20, 32, 4,
                      n_needles=1024, q_mix=True, batch=8, fp8_cache=True),
}


def needle_positions(seed: int, tid: int, stream: int, n: int, T: int) -> np.ndarray:
    """n distinct positions in [0, T): successive draws r mod T of substream
    ``stream`` (counter offset stream * 2**32), duplicates skipped."""
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    assert n <= T
    seen: list[int] = []
    got = set()
    e = stream << 32
    while len(seen) < n:
        r = draws_np(seed, tid, e, 4 * n)
        for v in (r % _U64(T)).astype(np.int64):
            if int(v) not in got:
                got.add(int(v))
                seen.append(int(v))
                if len(seen) == n:
                    break
        e += 4 * n
    return np.array(seen, dtype=np.int64)


def needle_dirs(cfg: BlockConfig) -> np.ndarray:
    """Unit vectors u_g [Hkv, d] (fp64), one per KV head."""
    z = normals_np(cfg.seed, TID_NEEDLE_DIR, 0, cfg.n_kv_heads * cfg.head_dim)
    z = z.reshape(cfg.n_kv_heads, cfg.head_dim)
    return z / np.linalg.norm(z, axis=1, keepdims=True)


def needle_key_bits(cfg: BlockConfig) -> np.ndarray:
    """Planted key rows 4 * u_g as bf16 bits [Hkv, d]."""
    return f64_to_bf16_bits(4.0 * needle_dirs(cfg))


def prefill_needles(cfg: BlockConfig, T: int | None = None) -> list[np.ndarray]:
    T = cfg.T if T is None else T
    n = min(cfg.n_needles, T)
    return [needle_positions(cfg.seed, TID_NEEDLE_POS, g, n, T) for g in range(cfg.n_kv_heads)]


def q_rows_np(cfg: BlockConfig, tid: int, rows: np.ndarray) -> np.ndarray:
    """Query rows [len(rows), Hq, d] as bf16 bits, generated row by row."""
    Hq, d = cfg.n_q_heads, cfg.head_dim
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), Hq, d), dtype=np.uint16)
    u = needle_dirs(cfg) if cfg.q_mix else None
    # group contiguous runs to amortise the generator
    i = 0
    while i < len(rows):
        j = i
        while j + 1 < len(rows) and rows[j + 1] == rows[j] + 1:
            j += 1
        r0, n = int(rows[i]), j - i + 1
        z = normals_np(cfg.seed, tid, r0 * Hq * d, n * Hq * d).reshape(n, Hq, d)
        if cfg.q_mix:
            ug = np.repeat(u, cfg.G, axis=0)           # [Hq, d]
            z = 0.5 * z + 0.5 * math.sqrt(d) * ug[None]
        out[i:j + 1] = f64_to_bf16_bits(z)
        i = j + 1
    return out


def kv_np(cfg: BlockConfig, tid: int, T: int | None = None) -> np.ndarray:
    """Directly generated K or V [T, Hkv, d] bf16 bits (configs without bridge)."""
    T = cfg.T if T is None else T
    return normal_bf16_np(cfg.seed, tid, 0, T * cfg.n_kv_heads * cfg.head_dim).reshape(
        T, cfg.n_kv_heads, cfg.head_dim)


def bridge_inputs_np(cfg: BlockConfig, T: int | None = None):
    """H [T, d_model], W_k, W_v [d_model, Hkv*d] as bf16 bits."""
    T = cfg.T if T is None else T
    dm, N = cfg.d_model, cfg.n_kv_heads * cfg.head_dim
    H = normal_bf16_np(cfg.seed, TID_H, 0, T * dm).reshape(T, dm)
    sd = 1.0 / math.sqrt(dm)
    Wk = normal_bf16_np(cfg.seed, TID_WK, 0, dm * N, sd).reshape(dm, N)
    Wv = normal_bf16_np(cfg.seed, TID_WV, 0, dm * N, sd).reshape(dm, N)
    return H, Wk, Wv


# The bridge recipe on a coarse dyadic grid: H = round(2 z) / 2 clipped to
# [-8, 8] and W = round(2^9 z / sqrt(d_model)) / 2^9 clipped to [-1/8, 1/8]
# (z the same N(0,1) draws as bridge_inputs_np).  Every product H W is then
# an integer multiple of 2^-10 of magnitude <= 1, so every partial sum of a
# row's d_model <= 2^11 products is an integer multiple of 2^-10 below 2^11:
# at most 21 significant bits, exact in fp32 whatever the order of summation.
# An fp32-accumulating bridge and an fp64 one then round the same exact
# value to bf16.
def _dyadic_h(z):
    return np.clip(np.round(2.0 * z), -16, 16) / 2.0


def _dyadic_w(z, dm):
    return np.clip(np.round(z * (512.0 / math.sqrt(dm))), -64, 64) / 512.0


def bridge_inputs_dyadic_np(cfg: BlockConfig, T: int | None = None):
    """H [T, d_model], W_k, W_v [d_model, Hkv*d] bf16 bits on the dyadic grid."""
    T = cfg.T if T is None else T
    dm, N = cfg.d_model, cfg.n_kv_heads * cfg.head_dim
    H = f64_to_bf16_bits(_dyadic_h(normals_np(cfg.seed, TID_H, 0, T * dm))).reshape(T, dm)
    Wk = f64_to_bf16_bits(_dyadic_w(normals_np(cfg.seed, TID_WK, 0, dm * N), dm)).reshape(dm, N)
    Wv = f64_to_bf16_bits(_dyadic_w(normals_np(cfg.seed, TID_WV, 0, dm * N), dm)).reshape(dm, N)
    return H, Wk, Wv


def bridge_inputs_dyadic_torch(cfg: BlockConfig, T: int | None = None, device="cuda",
                               chunk: int = 1 << 26):
    """bridge_inputs_dyadic_np's tensors generated on the device (bf16)."""
    import torch
    T = cfg.T if T is None else T
    dm, N = cfg.d_model, cfg.n_kv_heads * cfg.head_dim

    def gen(tid, count, grid):
        out = torch.empty(count, dtype=torch.bfloat16, device=device)
        for s0 in range(0, count, chunk):
            c = min(chunk, count - s0)
            out[s0:s0 + c] = grid(normals_torch(cfg.seed, tid, s0, c, device)).float().bfloat16()
        return out

    h = lambda z: torch.clamp(torch.round(2.0 * z), -16, 16) / 2.0
    w = lambda z: torch.clamp(torch.round(z * (512.0 / math.sqrt(dm))), -64, 64) / 512.0
    return (gen(TID_H, T * dm, h).view(T, dm), gen(TID_WK, dm * N, w).view(dm, N),
            gen(TID_WV, dm * N, w).view(dm, N))


def plant_needles_np(cfg: BlockConfig, K: np.ndarray, positions: list[np.ndarray]) -> None:
    """Overwrite needle rows of K [T, Hkv, d] (bf16 bits) in place."""
    rows = needle_key_bits(cfg)
    for g, pos in enumerate(positions):
        pos = pos[pos < K.shape[0]]
        K[pos, g, :] = rows[g]


@dataclass
class DecodeCache:
    Kc: np.ndarray      # [B, N, Hkv, d] uint8 e4m3 codes
    Vc: np.ndarray
    scale: np.ndarray   # [B, N, Hkv] fp32, shared by the K and V rows
    needles: list = field(default_factory=list)


def decode_cache_np(cfg: BlockConfig, N: int, batch: int | None = None) -> DecodeCache:
    """FP8 cache: bf16 N(0,1) K/V plus needles, per-(token, KV head) scale
    s = max(amax|K row|, amax|V row|) / 448 (fp32), codes = e4m3(x / s)."""
    B = cfg.batch if batch is None else batch
    Hkv, d = cfg.n_kv_heads, cfg.head_dim
    Kc = np.empty((B, N, Hkv, d), np.uint8)
    Vc = np.empty((B, N, Hkv, d), np.uint8)
    S = np.empty((B, N, Hkv), np.float32)
    nrows = needle_key_bits(cfg)
    needles = []
    for b in range(B):
        K = bf16_bits_to_f32(normal_bf16_np(cfg.seed, TID_DEC_K0 + b, 0, N * Hkv * d)).reshape(N, Hkv, d)
        V = bf16_bits_to_f32(normal_bf16_np(cfg.seed, TID_DEC_V0 + b, 0, N * Hkv * d)).reshape(N, Hkv, d)
        pos_b = []
        for g in range(Hkv):
            pos = needle_positions(cfg.seed, TID_DEC_POS0 + b, g, min(cfg.n_needles, N), N)
            K[pos, g, :] = bf16_bits_to_f32(nrows[g])
            pos_b.append(pos)
        needles.append(pos_b)
        amax = np.maximum(np.abs(K).max(axis=2), np.abs(V).max(axis=2)).astype(np.float32)
        s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        S[b] = s
        Kc[b] = e4m3_quantize_np((K / s[:, :, None]).astype(np.float32))
        Vc[b] = e4m3_quantize_np((V / s[:, :, None]).astype(np.float32))
    return DecodeCache(Kc, Vc, S, needles)


def decode_cache_split_scales_np(cfg: BlockConfig, N: int, batch: int | None = None,
                                 v_gain: float = 8.0):
    """FP8 cache whose K and V rows have their own scales: bf16 N(0,1) K plus
    needles and v_gain * N(0,1) V, k_scale = amax|K row| / 448 and v_scale =
    amax|V row| / 448 per (token, KV head), codes = e4m3(x / scale).
    Returns (Kc, Vc, k_scale, v_scale)."""
    B = cfg.batch if batch is None else batch
    Hkv, d = cfg.n_kv_heads, cfg.head_dim
    Kc = np.empty((B, N, Hkv, d), np.uint8)
    Vc = np.empty((B, N, Hkv, d), np.uint8)
    KS = np.empty((B, N, Hkv), np.float32)
    VS = np.empty((B, N, Hkv), np.float32)
    nrows = needle_key_bits(cfg)
    for b in range(B):
        K = bf16_bits_to_f32(normal_bf16_np(cfg.seed, TID_DEC_K0 + b, 0, N * Hkv * d)).reshape(N, Hkv, d)
        V = bf16_bits_to_f32(normal_bf16_np(cfg.seed, TID_DEC_V0 + b, 0, N * Hkv * d,
                                            v_gain)).reshape(N, Hkv, d)
        for g in range(Hkv):
            pos = needle_positions(cfg.seed, TID_DEC_POS0 + b, g, min(cfg.n_needles, N), N)
            K[pos, g, :] = bf16_bits_to_f32(nrows[g])
        for X, S, C in ((K, KS, Kc), (V, VS, Vc)):
            amax = np.abs(X).max(axis=2).astype(np.float32)
            s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
            S[b] = s
            C[b] = e4m3_quantize_np((X / s[:, :, None]).astype(np.float32))
    return Kc, Vc, KS, VS


def q_rows_torch(cfg: BlockConfig, tid: int, T: int | None = None, device="cuda", rows: int = 4096):
    """q_rows_np's recipe for all rows [T, Hq, d] on the device (bf16 tensor)."""
    import torch
    T = cfg.T if T is None else T
    Hq, d = cfg.n_q_heads, cfg.head_dim
    out = torch.empty(T, Hq, d, dtype=torch.bfloat16, device=device)
    ug = torch.from_numpy(needle_dirs(cfg)).to(device).repeat_interleave(cfg.G, 0)[None]
    for r0 in range(0, T, rows):
        n = min(rows, T - r0)
        z = normals_torch(cfg.seed, tid, r0 * Hq * d, n * Hq * d, device).view(n, Hq, d)
        if cfg.q_mix:
            z = 0.5 * z + 0.5 * math.sqrt(d) * ug
        out[r0:r0 + n] = z.float().bfloat16()
    return out


def kv_torch(cfg: BlockConfig, tid: int, T: int | None = None, device="cuda"):
    """kv_np's recipe on the device: [T, Hkv, d] bf16 tensor."""
    T = cfg.T if T is None else T
    return normal_bf16_torch(cfg.seed, tid, 0, T * cfg.n_kv_heads * cfg.head_dim,
                             device=device).view(T, cfg.n_kv_heads, cfg.head_dim)


def bridge_inputs_torch(cfg: BlockConfig, T: int | None = None, device="cuda"):
    """bridge_inputs_np's recipe on the device: H, W_k, W_v bf16 tensors."""
    T = cfg.T if T is None else T
    dm, N = cfg.d_model, cfg.n_kv_heads * cfg.head_dim
    H = normal_bf16_torch(cfg.seed, TID_H, 0, T * dm, device=device).view(T, dm)
    sd = 1.0 / math.sqrt(dm)
    Wk = normal_bf16_torch(cfg.seed, TID_WK, 0, dm * N, sd, device=device).view(dm, N)
    Wv = normal_bf16_torch(cfg.seed, TID_WV, 0, dm * N, sd, device=device).view(dm, N)
    return H, Wk, Wv


def needle_scatter_torch(cfg: BlockConfig, T: int | None = None, device="cuda"):
    """(rows, heads, values) of the planted needle keys for K[rows, heads] = values."""
    import torch
    pos = prefill_needles(cfg, T)
    nk = torch.from_numpy(needle_key_bits(cfg).view(np.int16)).to(device).view(torch.bfloat16)
    rows = torch.cat([torch.from_numpy(p) for p in pos]).to(device)
    heads = torch.cat([torch.full((len(p),), g, dtype=torch.int64)
                       for g, p in enumerate(pos)]).to(device)
    return rows, heads, nk[heads]


def decode_cache_torch(cfg: BlockConfig, N: int, batch: int | None = None, device="cuda"):
    """decode_cache_np's recipe on the device (torch); the e4m3 rounding is
    torch's float8_e4m3fn cast of values clamped to [-448, 448], pinned to the
    numpy quantiser by the tests.  Returns (Kc, Vc, scale) as uint8/uint8/fp32
    tensors [B, N, Hkv, d], [B, N, Hkv]."""
    import torch
    B = cfg.batch if batch is None else batch
    Hkv, d = cfg.n_kv_heads, cfg.head_dim
    Kc = torch.empty(B, N, Hkv, d, dtype=torch.uint8, device=device)
    Vc = torch.empty_like(Kc)
    S = torch.empty(B, N, Hkv, dtype=torch.float32, device=device)
    nrows = torch.from_numpy(bf16_bits_to_f32(needle_key_bits(cfg))).to(device)
    for b in range(B):
        K = normal_bf16_torch(cfg.seed, TID_DEC_K0 + b, 0, N * Hkv * d, device=device).float().view(N, Hkv, d)
        V = normal_bf16_torch(cfg.seed, TID_DEC_V0 + b, 0, N * Hkv * d, device=device).float().view(N, Hkv, d)
        for g in range(Hkv):
            pos = needle_positions(cfg.seed, TID_DEC_POS0 + b, g, min(cfg.n_needles, N), N)
            K[torch.from_numpy(pos).to(device), g, :] = nrows[g]
        amax = torch.maximum(K.abs().amax(dim=2), V.abs().amax(dim=2))
        s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        S[b] = s
        Kc[b] = (K / s[:, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        Vc[b] = (V / s[:, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        del K, V
    return Kc, Vc, S


def decode_queries_np(cfg: BlockConfig, tid: int, batch: int | None = None) -> np.ndarray:
    """One query per sequence [B, Hq, d] as bf16 bits (row b of stream tid)."""
    B = cfg.batch if batch is None else batch
    return q_rows_np(cfg, tid, np.arange(B))
