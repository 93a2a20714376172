// sparse_attn.cu -- sparse attention over the shared K/V and index list.
//
// KV Reuse (javabetter.cn explainer "mimo-v3-hysparse2", KV Reuse paragraph;
// aitop.news summary): each sparse layer attends with its own queries to the
// full-attention layer's K/V cache at the positions on that layer's token list
// and keeps no K/V of its own.
//
// Tensor-core gather attention with mma.sync m16n8k16, one (query row, KV
// head) pair per warp (or per group of WPR warps that split its list):
//   S^T[16 keys x 8 heads] = K_sel Q^T   and   O^T[16 dims x 8 heads] += V_sel^T P^T
// The dot-product dimension and the output dims are permuted (a sum does not
// care about the order of its terms, and the output permutation is undone at
// the store) so that every lane's fragment words are contiguous in memory:
//   * QK^T: lane (gid, t) reads 32 dims of gathered key rows gid and gid+8 --
//     bf16: dims 64u + 16t .. +15 for u = 0, 1 (two 32-byte loads), FP8:
//     dims 32t .. 32t+31; for bf16 these words are the A registers as they are;
//   * PV: lane (gid, t) reads dims 16*gid .. +15 of gathered value rows
//     4t..4t+3 (bf16: one 32-byte load per row), paired into A registers with
//     one byte permute each.
// Each gathered row is read by four (K) or eight (V) lanes with loads that
// cover it exactly; in the bf16 layout the lanes of one load instruction read
// whole 32-byte sectors of each row.  Softmax is online and base 2; P goes through 256
// bytes of shared memory per warp to become the B operand.  The FP8 variant
// converts e4m3 codes to f16 exactly, multiplies the logits by the key's
// scale and folds the value's scale into P.
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_sparse)

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kPScale = 1024.f;  // FP8: P * v_scale * 2^10 stays in f16's normal range
constexpr int kDecodeCluster = 8;   // CTAs sharing one decode (sequence, KV head) list

template <bool F16>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two) {
  __half2_raw h =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.y) << 16);
}

template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (F16) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    return pack_bf16x2(lo, hi);
  }
}

template <bool F16>
__device__ __forceinline__ uint16_t one16(float x) {
  if constexpr (F16) {
    __half h = __float2half_rn(x);
    return *reinterpret_cast<uint16_t*>(&h);
  } else {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t*>(&h);
  }
}

template <bool F16>
__device__ __forceinline__ float from16(uint16_t v) {
  if constexpr (F16) {
    return __half2float(*reinterpret_cast<__half*>(&v));
  } else {
    return __uint_as_float(uint32_t(v) << 16);
  }
}

// A list entry as the gather uses it: -1 (no token) and positions in
// [0, bound) pass unchanged; anything else is recorded as DEV_BAD_INDEX and
// skipped like -1, so a caller's bad list never reads outside K/V.
__device__ __forceinline__ int checked_entry(int j, int bound) {
  if (j == -1 || unsigned(j) < unsigned(bound)) return j;
  set_dev_status(DEV_BAD_INDEX);
  return -1;
}

// 32 contiguous bytes (32-byte aligned) from global memory, read-only path
__device__ __forceinline__ void ldg256(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

// G query heads of one KV head; FP8: e4m3 cache with per-(token, head) scales;
// WPR warps share one (row, KV head) pair, splitting its list; with CS > 1
// the CS CTAs of a thread-block cluster share it (CS * WPR parts) and combine
// their partial softmax states through distributed shared memory.  NL > 1
// fuses NL sparse layers: the pair's NL * G heads (layer e / G, head e % G of
// pair head e) share every gathered K/V row; their Q, O and lse come from
// `lp`.
template <int G, bool FP8, int WPR, int CS = 1, int NL = 1>
__global__ void __launch_bounds__(128)
    sparse_mma_kernel(const __nv_bfloat16* __restrict__ Q, const void* __restrict__ Kp,
                      const void* __restrict__ Vp, const float* __restrict__ ks,
                      const float* __restrict__ vs, const int32_t* __restrict__ idx,
                      __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int64_t rows,
                      int Hkv, int kw, float scale_log2, int64_t cache_T,
                      const __grid_constant__ SparseLayers lp,
                      const __grid_constant__ RowSpans spans, float* __restrict__ rec) {
  constexpr int HE = NL * G;                      // heads of a pair
  constexpr int NT = (HE + 7) / 8;                // 8-head n-tiles
  static_assert(NL == 1 || (WPR == 1 && !FP8), "layers are fused on the prefill path only");
  constexpr int NW = 4;                  // warps per CTA
  constexpr int PAIRS = NW / WPR;        // (row, KV head) pairs per CTA
  constexpr bool F16 = FP8;              // FP8 path: f16 MMA; bf16 path: bf16 MMA
  __shared__ uint16_t sP[NW][NT][8 * 16];
  __shared__ float sM[NW][NT * 8], sL[NW][NT * 8];
  __shared__ float sO[WPR > 1 ? NW : 1][WPR > 1 ? NT * 8 : 1][WPR > 1 ? 128 : 1];
  // this CTA's combined state, read by the cluster's first CTA
  __shared__ float cM[CS > 1 ? NT * 8 : 1], cL[CS > 1 ? NT * 8 : 1];
  __shared__ float cO[CS > 1 ? NT * 8 : 1][CS > 1 ? 128 : 1];
  static_assert(CS == 1 || WPR == 4, "a cluster splits pairs that fill their CTAs");

  const int warp = warp_id(), lane = lane_id();
  const int gid = lane >> 2, t = lane & 3;
  const int64_t pair = int64_t(blockIdx.x / CS) * PAIRS + warp / WPR;
  const int crank = int(blockIdx.x % CS);  // rank in the cluster (CS > 1)
  const int part = crank * WPR + warp % WPR;
  const bool active = pair < rows * Hkv;
  // KV-head-major pairs: a CTA's warps take consecutive rows of one KV head,
  // whose lists share the window and much of the rest
  const int64_t r = active ? pair % rows : 0;
  const int g = active ? int(pair / rows) : 0;
  const int Hq = Hkv * G;
  const int64_t tok0 = FP8 ? r * cache_T : 0;  // decode: sequence r's cache rows,
  const int jlo = FP8 ? spans.lo[r] : 0;         // holding its positions from jlo
  const int32_t* list = idx + (r * Hkv + g) * kw;
  const int per = (kw + WPR * CS - 1) / (WPR * CS);
  const int e_lo = part * per, e_hi = min(kw, e_lo + per);
  // valid positions: rows of K/V (prefill: cache_T holds their count); in
  // decode the list holds absolute positions and the slice test below keeps
  // every read inside the cache (its slice [lo, hi) spans at most cache_T rows)
  const int jbound = FP8 ? INT32_MAX : int(cache_T);

  // query fragments: head nt*8+gid; step s uses the dims that lane t's K
  // loads hold: bf16 dims 64(s/4) + 16t + 4(s%4) + {0..3}, FP8 dims 32t + 4s + {0..3}
  uint32_t qf[NT][8][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 8 + gid;  // pair head
    const bool real = hh < HE && active;
    const __nv_bfloat16* Qh =
        NL == 1 ? Q : reinterpret_cast<const __nv_bfloat16*>(lp.Q[real ? hh / G : 0]);
    const uint4* qr = reinterpret_cast<const uint4*>(Qh + (r * Hq + g * G + (real ? hh % G : 0)) * 128 +
                                                     (FP8 ? 32 * t : 16 * t));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      // bf16: 16-byte pieces u of the lane's two 32-byte runs at 64(u/2) + 16t
      const uint4 w = real ? __ldg(qr + (FP8 ? u : (u & 1) + 8 * (u >> 1))) : make_uint4(0, 0, 0, 0);
      const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int s = 2 * u + h2;
        if constexpr (F16) {
          qf[nt][s][0] = pack2<true>(bf16lo(w4[2 * h2]), bf16hi(w4[2 * h2]));
          qf[nt][s][1] = pack2<true>(bf16lo(w4[2 * h2 + 1]), bf16hi(w4[2 * h2 + 1]));
        } else {
          qf[nt][s][0] = w4[2 * h2];
          qf[nt][s][1] = w4[2 * h2 + 1];
        }
      }
    }
  }

  float m_run[NT][2], l_run[NT][2], o[NT][8][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[nt][i][0] = o[nt][i][1] = o[nt][i][2] = o[nt][i][3] = 0.f;
  }

  // positions of a step's 16 list entries (lanes 16-31 repeat 0-15), loaded
  // one step ahead so that a step's gathers do not wait for its list load
  int jl_next = (active && e_lo + (lane & 15) < e_hi) ? __ldg(list + e_lo + (lane & 15)) : -1;
  for (int e0 = e_lo; e0 < e_hi && active; e0 += 16) {
    int jl = checked_entry(jl_next, jbound);
    // decode with the context split over ranks: only this rank's slice
    if (FP8 && (jl < spans.lo[r] || jl >= spans.hi[r])) jl = -1;
    const int en = e0 + 16 + (lane & 15);
    jl_next = en < e_hi ? __ldg(list + en) : -1;
    const int jA = __shfl_sync(0xffffffffu, jl, gid), jB = __shfl_sync(0xffffffffu, jl, gid + 8);
    int jP[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) jP[u] = __shfl_sync(0xffffffffu, jl, 4 * t + u);
    const bool vA = jA >= 0, vB = jB >= 0;
    const int64_t rowA = (tok0 + (vA ? jA - jlo : 0)) * Hkv + g;
    const int64_t rowB = (tok0 + (vB ? jB - jlo : 0)) * Hkv + g;

    // ---- gathers: K rows (this lane's 32 dims), V rows 4t+u (16 dims)
    uint32_t ka[16], kb[16];  // bf16: words; FP8: first 8 hold 32 codes
    uint32_t vw[4][8];
    float vsc[4] = {0.f, 0.f, 0.f, 0.f};
    float ksA = 1.f, ksB = 1.f;
    if constexpr (!FP8) {
      // lanes t = 0..3 of a row read 128 contiguous bytes per 32-byte load
      // (dims 64u + 16t .. +15): every sector they touch is used whole
      const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(Kp) + rowA * 128 + 16 * t;
      const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(Kp) + rowB * 128 + 16 * t;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t x[8], y[8];
        ldg256(pa + 64 * u, x);
        ldg256(pb + 64 * u, y);
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          ka[8 * u + w] = x[w];
          kb[8 * u + w] = y[w];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t rv = (tok0 + (jP[u] >= 0 ? jP[u] - jlo : 0)) * Hkv + g;
        // lanes gid = 0..7 read a whole 256-byte row, 32 bytes each: dims
        // 16*gid .. +15
        ldg256(reinterpret_cast<const __nv_bfloat16*>(Vp) + rv * 128 + 16 * gid, vw[u]);
        vsc[u] = jP[u] >= 0 ? 1.f : 0.f;
      }
    } else {
      const uint4* pa = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(Kp) +
                                                       rowA * 128 + 32 * t);
      const uint4* pb = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(Kp) +
                                                       rowB * 128 + 32 * t);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint4 x = __ldg(pa + u), y = __ldg(pb + u);
        ka[4 * u] = x.x; ka[4 * u + 1] = x.y; ka[4 * u + 2] = x.z; ka[4 * u + 3] = x.w;
        kb[4 * u] = y.x; kb[4 * u + 1] = y.y; kb[4 * u + 2] = y.z; kb[4 * u + 3] = y.w;
      }
      ksA = vA ? __ldg(ks + rowA) : 0.f;
      ksB = vB ? __ldg(ks + rowB) : 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t rv = (tok0 + (jP[u] >= 0 ? jP[u] - jlo : 0)) * Hkv + g;
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(Vp) +
                                                             rv * 128 + 16 * gid));
        vw[u][0] = x.x; vw[u][1] = x.y; vw[u][2] = x.z; vw[u][3] = x.w;
        vsc[u] = jP[u] >= 0 ? __ldg(vs + rv) * kPScale : 0.f;
      }
    }

    // ---- S^T = K Q^T
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      uint32_t a0, a1, a2, a3;
      if constexpr (!FP8) {
        a0 = ka[2 * s];      // row gid, dims 32t+4s+{0,1}
        a1 = kb[2 * s];      // row gid+8
        a2 = ka[2 * s + 1];  // row gid, dims 32t+4s+{2,3}
        a3 = kb[2 * s + 1];
      } else {
        a0 = e4m3x2_f16x2(ka[s]);
        a1 = e4m3x2_f16x2(kb[s]);
        a2 = e4m3x2_f16x2(ka[s] >> 16);
        a3 = e4m3x2_f16x2(kb[s] >> 16);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma16816<F16>(sacc[nt], a0, a1, a2, a3, qf[nt][s][0], qf[nt][s][1]);
    }

    // ---- online softmax (base 2), lane: keys gid / gid+8, heads 2t, 2t+1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h0 = nt * 8 + 2 * t;
      const float cA = scale_log2 * ksA, cB = scale_log2 * ksB;
      float s00 = vA ? sacc[nt][0] * cA : -INFINITY, s01 = vA ? sacc[nt][1] * cA : -INFINITY;
      float s10 = vB ? sacc[nt][2] * cB : -INFINITY, s11 = vB ? sacc[nt][3] * cB : -INFINITY;
      if (h0 >= HE) s00 = s10 = -INFINITY;
      if (h0 + 1 >= HE) s01 = s11 = -INFINITY;
      float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
      const float al0 = mn0 == -INFINITY ? 1.f : fast_exp2(m_run[nt][0] - mn0);
      const float al1 = mn1 == -INFINITY ? 1.f : fast_exp2(m_run[nt][1] - mn1);
      const float p00 = mn0 == -INFINITY ? 0.f : fast_exp2(s00 - mn0);
      const float p10 = mn0 == -INFINITY ? 0.f : fast_exp2(s10 - mn0);
      const float p01 = mn1 == -INFINITY ? 0.f : fast_exp2(s01 - mn1);
      const float p11 = mn1 == -INFINITY ? 0.f : fast_exp2(s11 - mn1);
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
      l_run[nt][0] = l_run[nt][0] * al0 + p00 + p10;
      l_run[nt][1] = l_run[nt][1] * al1 + p01 + p11;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[nt][i][0] *= al0;
        o[nt][i][2] *= al0;
        o[nt][i][1] *= al1;
        o[nt][i][3] *= al1;
      }
      uint16_t* sp = sP[warp][nt];  // [head][key]
      sp[(2 * t) * 16 + gid] = one16<F16>(p00);
      sp[(2 * t + 1) * 16 + gid] = one16<F16>(p01);
      sp[(2 * t) * 16 + gid + 8] = one16<F16>(p10);
      sp[(2 * t + 1) * 16 + gid + 8] = one16<F16>(p11);
    }
    __syncwarp();
    // ---- O^T += V^T P^T: K slots {2t,2t+1,2t+8,2t+9} = keys 4t+{0,1,2,3};
    // MMA i, row gid -> dim D(i) = 16*gid + 2i; row gid+8 -> D(i) + 1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint16_t* sp = sP[warp][nt] + gid * 16 + 4 * t;
      const uint32_t b0 = pack2<F16>(from16<F16>(sp[0]) * vsc[0], from16<F16>(sp[1]) * vsc[1]);
      const uint32_t b1 = pack2<F16>(from16<F16>(sp[2]) * vsc[2], from16<F16>(sp[3]) * vsc[3]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t a0, a1, a2, a3;
        if constexpr (!FP8) {
          // word i of the lane's row slices = dims D(i) (low), D(i) + 1 (high)
          a0 = __byte_perm(vw[0][i], vw[1][i], 0x5410);
          a1 = __byte_perm(vw[0][i], vw[1][i], 0x7632);
          a2 = __byte_perm(vw[2][i], vw[3][i], 0x5410);
          a3 = __byte_perm(vw[2][i], vw[3][i], 0x7632);
        } else {
          // byte 2i / 2i+1 of a row slice = dims 16*gid+2i / +1
          const int wd = i >> 1, sh = (i & 1) * 16;
          const uint32_t r0 = vw[0][wd] >> sh, r1 = vw[1][wd] >> sh;
          const uint32_t r2 = vw[2][wd] >> sh, r3 = vw[3][wd] >> sh;
          a0 = e4m3x2_f16x2(__byte_perm(r0, r1, 0x0040));
          a1 = e4m3x2_f16x2(__byte_perm(r0, r1, 0x0051));
          a2 = e4m3x2_f16x2(__byte_perm(r2, r3, 0x0040));
          a3 = e4m3x2_f16x2(__byte_perm(r2, r3, 0x0051));
        }
        mma16816<F16>(o[nt][i], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncwarp();
  }

  // ---- finish: l over the lanes of a head, then (optionally) combine the
  // WPR warps of the pair, then O = o / l, lse
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      l_run[nt][e] = l;
    }
  const float oscale = FP8 ? 1.f / kPScale : 1.f;
  if constexpr (WPR == 1) {
    if (!active) return;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int h = nt * 8 + 2 * t + e;  // pair head: layer h / G, head h % G
        if (h >= HE) continue;
        __nv_bfloat16* Oh = NL == 1 ? O : reinterpret_cast<__nv_bfloat16*>(lp.O[h / G]);
        float* lseh = NL == 1 ? lse : lp.lse[h / G];
        const float l = l_run[nt][e];
        const float inv = l > 0.f ? oscale / l : 0.f;
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(o[nt][i][e] * inv, o[nt][i][e + 2] * inv);
        __nv_bfloat16* orow = Oh + (r * Hq + g * G + h % G) * 128;
        // pk[i] holds dims D(i), D(i) + 1
        uint4* d0 = reinterpret_cast<uint4*>(orow + 16 * gid);
        uint4* d1 = reinterpret_cast<uint4*>(orow + 16 * gid + 8);
        *d0 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *d1 = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        if (lseh != nullptr && gid == 0)
          lseh[r * Hq + g * G + h % G] = l > 0.f ? (m_run[nt][e] + __log2f(l)) * kLn2 : -INFINITY;
      }
    }
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (gid == 0) {
        sM[warp][nt * 8 + 2 * t] = m_run[nt][0];
        sM[warp][nt * 8 + 2 * t + 1] = m_run[nt][1];
        sL[warp][nt * 8 + 2 * t] = l_run[nt][0];
        sL[warp][nt * 8 + 2 * t + 1] = l_run[nt][1];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int d = 16 * gid + 2 * i;
        sO[warp][nt * 8 + 2 * t][d] = o[nt][i][0];
        sO[warp][nt * 8 + 2 * t + 1][d] = o[nt][i][1];
        sO[warp][nt * 8 + 2 * t][d + 1] = o[nt][i][2];
        sO[warp][nt * 8 + 2 * t + 1][d + 1] = o[nt][i][3];
      }
    }
    __syncthreads();
    if constexpr (CS > 1) {
      // combine this CTA's warps per head (unnormalised, relative to cM)
      for (int h = warp; h < G; h += NW) {
        float M = -INFINITY;
        for (int w2 = 0; w2 < WPR; ++w2) M = fmaxf(M, sM[w2][h]);
        float L = 0.f, f[WPR];
        for (int w2 = 0; w2 < WPR; ++w2) {
          f[w2] = M == -INFINITY ? 0.f : fast_exp2(sM[w2][h] - M);
          L += sL[w2][h] * f[w2];
        }
        for (int d = lane; d < 128; d += 32) {
          float acc = 0.f;
          for (int w2 = 0; w2 < WPR; ++w2) acc += sO[w2][h][d] * f[w2];
          cO[h][d] = acc;
        }
        if (lane == 0) {
          cM[h] = M;
          cL[h] = L;
        }
      }
      namespace cg = cooperative_groups;
      cg::cluster_group cluster = cg::this_cluster();
      cluster.sync();
      if (crank == 0 && active) {
        for (int h = warp; h < G; h += NW) {
          float Mr[CS], M = -INFINITY;
#pragma unroll
          for (int q = 0; q < CS; ++q) {
            Mr[q] = *cluster.map_shared_rank(&cM[h], q);
            M = fmaxf(M, Mr[q]);
          }
          float L = 0.f;
#pragma unroll
          for (int q = 0; q < CS; ++q) {
            Mr[q] = M == -INFINITY ? 0.f : fast_exp2(Mr[q] - M);  // weight of CTA q
            L += *cluster.map_shared_rank(&cL[h], q) * Mr[q];
          }
          const float inv = L > 0.f ? oscale / L : 0.f;
          // rec: this rank's softmax state over its slice (m, l, o unnormalised)
          float* rr = rec != nullptr ? rec + (r * Hq + g * G + h) * 130 : nullptr;
          for (int d = lane; d < 128; d += 32) {
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < CS; ++q) acc += *cluster.map_shared_rank(&cO[h][d], q) * Mr[q];
            if (rr != nullptr)
              rr[2 + d] = acc * oscale;
            else
              O[(r * Hq + g * G + h) * 128 + d] = __float2bfloat16_rn(acc * inv);
          }
          if (rr != nullptr && lane == 0) {
            rr[0] = M;
            rr[1] = L;
          }
          if (rr == nullptr && lse != nullptr && lane == 0)
            lse[r * Hq + g * G + h] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
        }
      }
      cluster.sync();  // the other CTAs' shared memory stays until it has been read
    } else if (part == 0 && active) {
      const int w0 = warp;  // first warp of this pair
      for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
        for (int w2 = 0; w2 < WPR; ++w2) M = fmaxf(M, sM[w0 + w2][h]);
        float L = 0.f, f[WPR];
        for (int w2 = 0; w2 < WPR; ++w2) {
          f[w2] = M == -INFINITY ? 0.f : fast_exp2(sM[w0 + w2][h] - M);
          L += sL[w0 + w2][h] * f[w2];
        }
        const float inv = L > 0.f ? oscale / L : 0.f;
        for (int d = lane; d < 128; d += 32) {
          float acc = 0.f;
          for (int w2 = 0; w2 < WPR; ++w2) acc += sO[w0 + w2][h][d] * f[w2];
          O[(r * Hq + g * G + h) * 128 + d] = __float2bfloat16_rn(acc * inv);
        }
        if (lse != nullptr && lane == 0)
          lse[r * Hq + g * G + h] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
      }
    }
  }
}

template <int G>
cudaError_t launch_g(const SparseArgs& a, cudaStream_t stream) {
  const int64_t pairs = a.T * a.Hkv;
  const float sl2 = a.scale * kLog2e;
  if (a.Kc != nullptr) {
    // decode: few pairs, each split over a cluster of kDecodeCluster CTAs of
    // four warps
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(pairs * kDecodeCluster));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kDecodeCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, sparse_mma_kernel<G, true, 4, kDecodeCluster>,
        reinterpret_cast<const __nv_bfloat16*>(a.Q), static_cast<const void*>(a.Kc),
        static_cast<const void*>(a.Vc), static_cast<const float*>(a.ks),
        static_cast<const float*>(a.vs), static_cast<const int32_t*>(a.idx),
        reinterpret_cast<__nv_bfloat16*>(a.O), a.lse, int64_t(a.T), a.Hkv, a.kw, sl2,
        int64_t(a.cache_T), SparseLayers{}, a.spans, a.rec);
    if (e != cudaSuccess) return e;
  } else {
    sparse_mma_kernel<G, false, 1><<<unsigned((pairs + 3) / 4), 128, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(a.Q), a.K, a.V, nullptr, nullptr, a.idx,
        reinterpret_cast<__nv_bfloat16*>(a.O), a.lse, a.T, a.Hkv, a.kw, sl2,
        a.kv_rows > 0 ? a.kv_rows : a.T, SparseLayers{}, RowSpans{}, nullptr);
  }
  count_launch();
  return cudaGetLastError();
}

// L layers in one pass over the gathered rows (bf16 K/V)
template <int G, int L>
cudaError_t launch_fused(const SparseArgs& a, const SparseLayers& lp, cudaStream_t stream) {
  const int64_t pairs = a.T * a.Hkv;
  sparse_mma_kernel<G, false, 1, 1, L><<<unsigned((pairs + 3) / 4), 128, 0, stream>>>(
      nullptr, a.K, a.V, nullptr, nullptr, a.idx, nullptr, nullptr, a.T, a.Hkv, a.kw,
      a.scale * kLog2e, a.kv_rows > 0 ? a.kv_rows : a.T, lp, RowSpans{}, nullptr);
  count_launch();
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_fused_g(const SparseArgs& a, const SparseLayers& lp, int L,
                           cudaStream_t stream) {
  switch (L) {
    case 2: return launch_fused<G, 2>(a, lp, stream);
    case 3: return launch_fused<G, 3>(a, lp, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

int max_fused_layers(int G) { return G <= 8 ? kMaxFusedLayers : 1; }

cudaError_t launch_sparse_fused(const SparseArgs& a, const SparseLayers& lp, int L,
                                cudaStream_t stream) {
  if (L < 2 || L > max_fused_layers(a.Hq / a.Hkv)) return cudaErrorInvalidValue;
  switch (a.Hq / a.Hkv) {
    case 1: return launch_fused_g<1>(a, lp, L, stream);
    case 2: return launch_fused_g<2>(a, lp, L, stream);
    case 4: return launch_fused_g<4>(a, lp, L, stream);
    case 8: return launch_fused_g<8>(a, lp, L, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sparse(const SparseArgs& a, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_g<1>(a, stream);
    case 2: return launch_g<2>(a, stream);
    case 4: return launch_g<4>(a, stream);
    case 8: return launch_g<8>(a, stream);
    case 16: return launch_g<16>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hs2
