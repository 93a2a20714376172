// decode.cu -- one decode step of the cross-decoder block over an FP8 KV cache.
//
// The FP8 KV cache of the zgeo.com.cn comparison table and of the
// javabetter.cn explainer's 1M-token figures; the cross-decoder runs while
// generating (zgeo.com.cn, section 核心技术原理解析).  For each sequence b the
// new token is the last cache entry i = N_b - 1; the block runs full
// attention, token selection and the sparse layers on
//   K^[t,g,:] = e4m3(Kc[b,t,g,:]) * k_scale[b,t,g]  (likewise V).
//
// Kernels (all on `stream`):
//   decode_partial  split-KV attention of the G query heads of (b, g) over a
//                   8192-key chunk: a producer warp streams 128-row K and V
//                   tiles by TMA (128-byte swizzle) into a shared memory ring
//                   (2 stages) and their per-token scales by cp.async; four
//                   warps each take 32 keys of a stage and run mma.sync
//                   m16n8k16 (e4m3 codes -> f16 exactly, fp32 accumulation).
//                   The dot-product dimension and the output dims are
//                   permuted so every lane reads 16 contiguous bytes of a K
//                   or V row.  The KV heads of a chunk are neighbours in the
//                   grid, so the head slices of the same cache rows are read
//                   at about the same time.
//                   Writes base-2 logits (fp32) for the scoring pass and the
//                   chunk's (max, sum, unnormalised output).
//   decode_merge    merges the chunks: o (bf16), lse (natural log).
//   decode_score    score_j = sum_h exp2(logit_hj - lse2_h) for candidates
//                   j <= i - w, stored; histogram of score buckets (fp32
//                   bits >> 20: eighths of a binade) per (b, g).
//   decode_collect  every candidate in the bucket holding the k-th best score
//                   or above goes to a per-(b, g) list (about k + a few
//                   hundred entries).
//   decode_final    per (b, g): exact top k of the list on the 64-bit key
//                   (score bits << 32 | ~j), positions sorted ascending, then
//                   the window; an exact radix select over all candidates
//                   when the list overflows.
// The sparse layers then gather the FP8 rows at idx (sparse_attn.cu).
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_decode)
HS2_BUDGET_SETTER(budget_decode)

namespace {

constexpr int CH = 8192;            // keys per decode_partial CTA
constexpr int DP_WARPS = 4;         // each warp: CH / 4 keys, 16 per step
constexpr int NBUCKET = 2048;       // score buckets (bits >> 20 of fp32 < 2^8)
constexpr int CAPC = kDecodeMergeCap;  // candidate list capacity per (b, g)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int MAX_B = kDecodeMaxBatch;
constexpr float kPScale = 1024.f;   // P' = p * v_scale * 2^10 keeps f16 products normal

struct Partial {  // per (b, h, chunk)
  float m, l;
};

struct SeqLens {  // per sequence, passed by value: its length n (the new token
  int n[MAX_B];     // is n - 1) and the slice [lo, hi) of its cache this call
  int lo[MAX_B];    // covers (the whole cache, [0, n), unless the context is
  int hi[MAX_B];    // split over ranks)
};

// both e4m3 pairs of a 32-bit word -> two f16x2 (low pair, high pair)
__device__ __forceinline__ void cvt_e4m3x4_f16x2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l16, h16;\n\tmov.b32 {l16, h16}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l16;\n\tcvt.rn.f16x2.e4m3x2 %1, h16;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4-byte asynchronous copy global -> shared; src_bytes 0 writes zeros
__device__ __forceinline__ void cp_async4(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// arrive on `bar` once this thread's earlier cp.async copies have landed
// (counts as one of the barrier's expected arrivals)
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// decode_partial: grid (Hkv, chunks, B), DP_WARPS consumer warps + 1 producer
// ---------------------------------------------------------------------------
constexpr int KPW = 32;                           // keys per warp per stage
constexpr int DSTAGE_KEYS = DP_WARPS * KPW;       // keys per TMA stage
constexpr int DSTAGES = 2;                        // ring depth
constexpr int DSTAGE_BYTES = 2 * DSTAGE_KEYS * 128;  // K and V codes

template <int G>
__global__ void __launch_bounds__((DP_WARPS + 1) * 32, 3)
    decode_partial(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __nv_bfloat16* __restrict__ q, const float* __restrict__ ks,
                   const float* __restrict__ vs, SeqLens seq_len, int64_t cap,
                   int Hkv, int nch, float scale_log2, float* __restrict__ logits,
                   Partial* __restrict__ part, float* __restrict__ part_o) {
  constexpr int NT = G > 8 ? G / 8 : 1;   // 8-head n-tiles
  constexpr int GH = G < 8 ? G : 8;       // real heads per n-tile
  __shared__ uint16_t sP[DP_WARPS][NT][8 * KPW];     // P [head][key] f16 per warp
  __shared__ float sM[DP_WARPS][NT * 8], sL[DP_WARPS][NT * 8];
  __shared__ uint64_t full[DSTAGES], empty[DSTAGES];
  __shared__ float sScale[DSTAGES][2][DSTAGE_KEYS];  // K and V scales of a stage's keys
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* ring = smem_align1024(dsmem_raw);

  // the KV heads of a chunk are neighbours in the grid, so the 128-byte head
  // slices of the same cache rows are read at about the same time
  const int g = blockIdx.x, c = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int gid = lane >> 2, t = lane & 3;
  const int Hq = Hkv * G;
  // chunk c covers positions lo + c * CH .. (local rows c * CH ..) of the slice
  const int64_t c_lo = int64_t(seq_len.lo[b]) + int64_t(c) * CH;
  const int64_t c_hi = min(c_lo + CH, int64_t(seq_len.hi[b]));
  const int n_st = c_hi > c_lo ? int((c_hi - c_lo + DSTAGE_KEYS - 1) / DSTAGE_KEYS) : 0;
  // cache row of position p of sequence b: the cache holds its slice
  // [lo, hi), position lo at row b * cap
  const int64_t lo = seq_len.lo[b];
  const int64_t rowpos = int64_t(b) * cap - lo;

  if (threadIdx.x == 0) {
    for (int i = 0; i < DSTAGES; ++i) {
      mbar_init(&full[i], 1 + 32);  // the TMA issuer, plus one per producer lane's scales
      mbar_init(&empty[i], DP_WARPS);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == DP_WARPS) {
    // ---------------- producer: K and V tiles of 64 rows -> smem ring by TMA,
    // their per-token scales by cp.async (two keys per lane) ------------------
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    int issued = 0;
    for (int si = 0; si < n_st; ++si) {
      const int slot = si % DSTAGES;
      bool go = true;
      if (lane == 0 && si >= DSTAGES) go = mbar_wait(&empty[slot], ((si / DSTAGES) & 1) ^ 1);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      issued = si + 1;
      const int64_t kbase = c_lo + int64_t(si) * DSTAGE_KEYS;
#pragma unroll
      for (int u = 0; u < DSTAGE_KEYS / 32; ++u) {
        const int64_t key = kbase + lane + 32 * u;
        const bool in = key < c_hi;
        const size_t off = size_t(rowpos + (in ? key : c_lo)) * Hkv + g;
        cp_async4(&sScale[slot][0][lane + 32 * u], ks + off, in ? 4 : 0);
        cp_async4(&sScale[slot][1][lane + 32 * u], vs + off, in ? 4 : 0);
      }
      cp_async_arrive(&full[slot]);
      if (lane == 0) {
        uint8_t* st = ring + slot * DSTAGE_BYTES;
        const int z = int(rowpos + c_lo) + si * DSTAGE_KEYS;
        mbar_arrive_expect_tx(&full[slot], DSTAGE_BYTES);
        tma_load_3d(st, &tmK, &full[slot], 0, g, z);
        tma_load_3d(st + DSTAGE_KEYS * 128, &tmV, &full[slot], 0, g, z);
      }
    }
    // every issued copy (TMA tiles and every lane's scales) lands before the
    // CTA can exit
    if (lane == 0)
      for (int sl = 0; sl < DSTAGES; ++sl)
        drain_phase(&full[sl], issued > sl ? (issued - 1 - sl) / DSTAGES + 1 : 0);
    __syncwarp();
    return;
  }

  // query fragments (B operand of S^T = K q^T): dims permuted so that lane t
  // uses dims 32t .. 32t+31: MMA step s, k-slot {2t,2t+1,2t+8,2t+9} ->
  // dim 32t + 4s + {0,1,2,3}
  uint32_t qf[NT][8][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hh = nt * 8 + gid;
    const bool real = hh < G;
    const __nv_bfloat16* qr = q + (size_t(b) * Hq + g * G + (real ? hh : 0)) * 128 + 32 * t;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 w = real ? *reinterpret_cast<const uint4*>(qr + 8 * u) : make_uint4(0, 0, 0, 0);
      const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {  // two steps per 16 bytes
        const int s = 2 * u + h2;
        qf[nt][s][0] = pack_f16x2(bf16lo(ws4[2 * h2]), bf16hi(ws4[2 * h2]));
        qf[nt][s][1] = pack_f16x2(bf16lo(ws4[2 * h2 + 1]), bf16hi(ws4[2 * h2 + 1]));
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
  float* lg = logits + (size_t(b) * Hkv + g) * cap * G;
  bool ok = true;

  for (int si = 0; si < n_st; ++si) {
    const int slot = si % DSTAGES;
    ok = ok && mbar_wait(&full[slot], (si / DSTAGES) & 1);
    const uint8_t* sK = ring + slot * DSTAGE_BYTES;
    const uint8_t* sV = sK + DSTAGE_KEYS * 128;
    const int wk0 = KPW * warp;  // this warp's first row of the stage
    const int64_t key0 = c_lo + int64_t(si) * DSTAGE_KEYS + wk0;
    // ---- S^T = K q^T for the warp's two 16-key groups (independent chains);
    // rows in the swizzled tile: unit u of row r sits at r*128 + ((u ^ (r & 7)) << 4)
    float sacc[2][NT][4];
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      const int rA = wk0 + 16 * q2 + gid, rB = rA + 8;
      const uint4 ka = *reinterpret_cast<const uint4*>(sK + rA * 128 + (((2 * t) ^ (rA & 7)) << 4));
      const uint4 kb = *reinterpret_cast<const uint4*>(sK + rA * 128 + (((2 * t + 1) ^ (rA & 7)) << 4));
      const uint4 kc = *reinterpret_cast<const uint4*>(sK + rB * 128 + (((2 * t) ^ (rB & 7)) << 4));
      const uint4 kd = *reinterpret_cast<const uint4*>(sK + rB * 128 + (((2 * t + 1) ^ (rB & 7)) << 4));
      const uint32_t kw0[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
      const uint32_t kw1[8] = {kc.x, kc.y, kc.z, kc.w, kd.x, kd.y, kd.z, kd.w};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[q2][nt][e] = 0.f;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        // row gid: slots 2t,2t+1 (a0) and 2t+8,2t+9 (a2); row gid+8: a1, a3
        uint32_t a0, a1, a2, a3;
        cvt_e4m3x4_f16x2x2(kw0[s], a0, a2);
        cvt_e4m3x4_f16x2x2(kw1[s], a1, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_f16(sacc[q2][nt], a0, a1, a2, a3, qf[nt][s][0], qf[nt][s][1]);
      }
    }
    // ---- base-2 logits; lane holds, per group q2, keys 16q2+gid (c0,c1) and
    // 16q2+gid+8 (c2,c3) for heads 2t, 2t+1
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h0 = nt * 8 + 2 * t;
      float sv[2][2][2];  // [group][key gid / gid+8][head 2t / 2t+1]
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int64_t r0 = key0 + 16 * q2 + gid, r1 = r0 + 8;
        const bool v0 = r0 < c_hi, v1 = r1 < c_hi;
        const float c0 = sScale[slot][0][wk0 + 16 * q2 + gid] * scale_log2;
        const float c1 = sScale[slot][0][wk0 + 16 * q2 + gid + 8] * scale_log2;
        sv[q2][0][0] = v0 ? sacc[q2][nt][0] * c0 : -INFINITY;
        sv[q2][0][1] = v0 ? sacc[q2][nt][1] * c0 : -INFINITY;
        sv[q2][1][0] = v1 ? sacc[q2][nt][2] * c1 : -INFINITY;
        sv[q2][1][1] = v1 ? sacc[q2][nt][3] * c1 : -INFINITY;
        if (h0 >= GH + nt * 8) sv[q2][0][0] = sv[q2][1][0] = -INFINITY;  // padded heads
        if (h0 + 1 >= GH + nt * 8) sv[q2][0][1] = sv[q2][1][1] = -INFINITY;
        if (h0 + 1 < G) {
          if (v0) *reinterpret_cast<float2*>(lg + (r0 - lo) * G + h0) = make_float2(sv[q2][0][0], sv[q2][0][1]);
          if (v1) *reinterpret_cast<float2*>(lg + (r1 - lo) * G + h0) = make_float2(sv[q2][1][0], sv[q2][1][1]);
        } else if (h0 < G) {
          if (v0) lg[(r0 - lo) * G + h0] = sv[q2][0][0];
          if (v1) lg[(r1 - lo) * G + h0] = sv[q2][1][0];
        }
      }
      // online softmax over the warp's 32 keys of the stage for heads h0, h0+1
      float mx0 = fmaxf(fmaxf(sv[0][0][0], sv[0][1][0]), fmaxf(sv[1][0][0], sv[1][1][0]));
      float mx1 = fmaxf(fmaxf(sv[0][0][1], sv[0][1][1]), fmaxf(sv[1][0][1], sv[1][1][1]));
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
      const float al0 = mn0 == -INFINITY ? 1.f : fast_exp2(m_run[nt][0] - mn0);
      const float al1 = mn1 == -INFINITY ? 1.f : fast_exp2(m_run[nt][1] - mn1);
      const bool grew = mn0 != m_run[nt][0] || mn1 != m_run[nt][1];
      float pv[2][2][2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          pv[q2][kk][0] = mn0 == -INFINITY ? 0.f : fast_exp2(sv[q2][kk][0] - mn0);
          pv[q2][kk][1] = mn1 == -INFINITY ? 0.f : fast_exp2(sv[q2][kk][1] - mn1);
        }
      m_run[nt][0] = mn0;
      m_run[nt][1] = mn1;
      l_run[nt][0] = l_run[nt][0] * al0 + ((pv[0][0][0] + pv[0][1][0]) + (pv[1][0][0] + pv[1][1][0]));
      l_run[nt][1] = l_run[nt][1] * al1 + ((pv[0][0][1] + pv[0][1][1]) + (pv[1][0][1] + pv[1][1][1]));
      if (__any_sync(0xffffffffu, grew)) {  // rescale only after a new maximum
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o[nt][i][0] *= al0;
          o[nt][i][2] *= al0;
          o[nt][i][1] *= al1;
          o[nt][i][3] *= al1;
        }
      }
      // P (not yet times V's scale) to shared memory, [head][32 keys] f16
      uint16_t* sp = sP[warp][nt];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const __half hp = __float2half_rn(pv[q2][kk][e]);
            sp[(2 * t + e) * KPW + 16 * q2 + 8 * kk + gid] = *reinterpret_cast<const uint16_t*>(&hp);
          }
    }
    __syncwarp();
    // ---- O^T += V^T P'^T per 16-key group: M = 16 dims (permuted), K = 16
    // keys (4t+u), N = heads; B fragment: P'[head gid][keys 4t, 4t+1] and
    // [4t+2, 4t+3], times V's scale (which carries the 2^10 factor)
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      uint4 vr[4];
      float vsc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int rv = wk0 + 16 * q2 + 4 * t + u;
        vr[u] = *reinterpret_cast<const uint4*>(sV + rv * 128 + ((gid ^ (rv & 7)) << 4));
        vsc[u] = sScale[slot][1][rv] * kPScale;
      }
      const uint32_t vw[4][4] = {{vr[0].x, vr[0].y, vr[0].z, vr[0].w},
                                 {vr[1].x, vr[1].y, vr[1].z, vr[1].w},
                                 {vr[2].x, vr[2].y, vr[2].z, vr[2].w},
                                 {vr[3].x, vr[3].y, vr[3].z, vr[3].w}};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint16_t* sp = sP[warp][nt] + gid * KPW + 16 * q2 + 4 * t;
        const float f0 = __half2float(*reinterpret_cast<const __half*>(sp + 0)) * vsc[0];
        const float f1 = __half2float(*reinterpret_cast<const __half*>(sp + 1)) * vsc[1];
        const float f2 = __half2float(*reinterpret_cast<const __half*>(sp + 2)) * vsc[2];
        const float f3 = __half2float(*reinterpret_cast<const __half*>(sp + 3)) * vsc[3];
        const uint32_t b0 = pack_f16x2(f0, f1), b1 = pack_f16x2(f2, f3);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          // bytes 2i / 2i+1 of a row slice = dims 16*gid + 2i (MMA row gid) and
          // 16*gid + 2i + 1 (row gid+8).  One permute gathers, for two keys,
          // [key0 dim 2i, key1 dim 2i, key0 dim 2i+1, key1 dim 2i+1].
          const int wd = i >> 1, p = (i & 1) * 2;
          const uint32_t sel = uint32_t(p) | uint32_t(p + 4) << 4 | uint32_t(p + 1) << 8 |
                               uint32_t(p + 5) << 12;
          uint32_t a0, a1, a2, a3;
          cvt_e4m3x4_f16x2x2(__byte_perm(vw[0][wd], vw[1][wd], sel), a0, a1);
          cvt_e4m3x4_f16x2x2(__byte_perm(vw[2][wd], vw[3][wd], sel), a2, a3);
          mma_f16(o[nt][i], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }

  // ---- combine the warps of the CTA, then one partial per (b, h, chunk);
  // the drained ring holds the warps' outputs
  asm volatile("bar.sync 1, %0;" ::"n"(DP_WARPS * 32) : "memory");
  float (*sO)[NT * 8][128] = reinterpret_cast<float (*)[NT * 8][128]>(ring);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      l_run[nt][e] = l;
    }
    if (gid == 0) {
      sM[warp][nt * 8 + 2 * t] = m_run[nt][0];
      sM[warp][nt * 8 + 2 * t + 1] = m_run[nt][1];
      sL[warp][nt * 8 + 2 * t] = l_run[nt][0];
      sL[warp][nt * 8 + 2 * t + 1] = l_run[nt][1];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sO[warp][nt * 8 + 2 * t][16 * gid + 2 * i] = o[nt][i][0];
      sO[warp][nt * 8 + 2 * t + 1][16 * gid + 2 * i] = o[nt][i][1];
      sO[warp][nt * 8 + 2 * t][16 * gid + 2 * i + 1] = o[nt][i][2];
      sO[warp][nt * 8 + 2 * t + 1][16 * gid + 2 * i + 1] = o[nt][i][3];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(DP_WARPS * 32) : "memory");
  for (int hh = warp; hh < G; hh += DP_WARPS) {
    float M = -INFINITY;
    for (int w2 = 0; w2 < DP_WARPS; ++w2) M = fmaxf(M, sM[w2][hh]);
    float L = 0.f, f[DP_WARPS];
    for (int w2 = 0; w2 < DP_WARPS; ++w2) {
      f[w2] = M == -INFINITY ? 0.f : fast_exp2(sM[w2][hh] - M);
      L += sL[w2][hh] * f[w2];
    }
    const size_t pi = (size_t(b) * Hq + g * G + hh) * nch + c;
    for (int d = lane; d < 128; d += 32) {
      float acc = 0.f;
      for (int w2 = 0; w2 < DP_WARPS; ++w2) acc += sO[w2][hh][d] * f[w2];
      part_o[pi * 128 + d] = acc * (1.f / kPScale);
    }
    if (lane == 0) part[pi] = Partial{M, L};
  }
}

// ---------------------------------------------------------------------------
// decode_merge: grid (Hq, B), 128 threads
// ---------------------------------------------------------------------------
constexpr int MERGE_GROUPS = 4;  // groups of 128 threads, each over every 4th chunk
constexpr int REC = kDecodeRecFloats;  // a softmax-state record: m, l, o[128] (floats)

// Merges the chunk partials of each (b, h) over the chunks covering its
// slice.  rec == nullptr: the result o (bf16), lse (natural log) and lse2;
// otherwise the merged state itself as one record (m, l, o unnormalised),
// [B][Hq][REC], for a merge across ranks.
__global__ void __launch_bounds__(128 * MERGE_GROUPS)
    decode_merge(const Partial* __restrict__ part, const float* __restrict__ part_o,
                 SeqLens seq_len, int Hq, int nch, __nv_bfloat16* __restrict__ o,
                 float* __restrict__ lse, float* __restrict__ lse2_out, float* __restrict__ rec) {
  __shared__ float s_red[MERGE_GROUPS][129];
  __shared__ float s_max[128 * MERGE_GROUPS / 32];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int d = tid & 127, grp = tid >> 7;
  const int nc = (seq_len.hi[b] - seq_len.lo[b] + CH - 1) / CH;  // chunks of the slice
  const size_t base = (size_t(b) * Hq + h) * nch;
  // the largest chunk maximum
  float M = -INFINITY;
  for (int c = tid; c < nc; c += 128 * MERGE_GROUPS) M = fmaxf(M, part[base + c].m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if ((tid & 31) == 0) s_max[tid >> 5] = M;
  __syncthreads();
  M = s_max[0];
#pragma unroll
  for (int i = 1; i < 128 * MERGE_GROUPS / 32; ++i) M = fmaxf(M, s_max[i]);
  float L = 0.f, acc = 0.f;
#pragma unroll 4
  for (int c = grp; c < nc; c += MERGE_GROUPS) {
    const Partial p = part[base + c];
    const float f = p.m == -INFINITY ? 0.f : fast_exp2(p.m - M);
    L += p.l * f;
    acc += part_o[(base + c) * 128 + d] * f;
  }
  s_red[grp][d] = acc;
  if (d == 0) s_red[grp][128] = L;
  __syncthreads();
  if (grp == 0) {
    for (int q = 1; q < MERGE_GROUPS; ++q) acc += s_red[q][d];
    L = 0.f;
    for (int q = 0; q < MERGE_GROUPS; ++q) L += s_red[q][128];
    if (rec != nullptr) {
      float* r = rec + (size_t(b) * Hq + h) * REC;
      r[2 + d] = acc;
      if (d == 0) {
        r[0] = M;
        r[1] = L;
      }
      return;
    }
    o[(size_t(b) * Hq + h) * 128 + d] = __float2bfloat16_rn(acc / L);
    if (d == 0) {
      const float l2 = M + __log2f(L);
      lse[size_t(b) * Hq + h] = l2 * kLn2;
      lse2_out[size_t(b) * Hq + h] = l2;
    }
  }
}

// Merges the records of R ranks for (b, h): record r at
// recs + r * rank_stride + (b * Hq + h) * REC.  Writes o (bf16), and lse /
// lse2 where those pointers are not null.
__global__ void __launch_bounds__(128)
    decode_merge_ranks(const float* __restrict__ recs, int R, int64_t rank_stride, int Hq,
                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                       float* __restrict__ lse2_out) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const size_t off = (size_t(b) * Hq + h) * REC;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, recs[r * rank_stride + off]);
  float L = 0.f, acc = 0.f;
  for (int r = 0; r < R; ++r) {
    const float* rr = recs + r * rank_stride + off;
    const float f = rr[0] == -INFINITY ? 0.f : fast_exp2(rr[0] - M);
    L += rr[1] * f;
    acc += rr[2 + d] * f;
  }
  o[(size_t(b) * Hq + h) * 128 + d] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
  if (d == 0) {
    const float l2 = L > 0.f ? M + __log2f(L) : -INFINITY;
    if (lse != nullptr) lse[size_t(b) * Hq + h] = l2 * kLn2;
    if (lse2_out != nullptr) lse2_out[size_t(b) * Hq + h] = l2;
  }
}

// ---------------------------------------------------------------------------
// decode_score: grid (chunks, Hkv, B), 256 threads
// ---------------------------------------------------------------------------
__device__ int block_kth_bucket(const uint32_t* __restrict__ gh, uint32_t k, uint32_t* s_scan);

template <int G>
__global__ void __launch_bounds__(256)
    decode_score(const float* __restrict__ logits, const float* __restrict__ lse2,
                 SeqLens seq_len, int64_t cap, int Hkv, int k, int w,
                 float* __restrict__ score, uint32_t* __restrict__ hist,
                 uint32_t* __restrict__ done, int* __restrict__ kth_bucket) {
  __shared__ uint32_t sh[NBUCKET];
  __shared__ float sl[G];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int N = seq_len.n[b];
  // candidates j <= i - w, i.e. j < N - w, inside the slice [lo, hi)
  const int64_t j_end = min(int64_t(N) - w, int64_t(seq_len.hi[b]));
  for (int i = threadIdx.x; i < NBUCKET; i += 256) sh[i] = 0;
  if (threadIdx.x < G) sl[threadIdx.x] = lse2[size_t(b) * Hkv * G + g * G + threadIdx.x];
  __syncthreads();
  const int64_t lo = seq_len.lo[b];  // logits and scores are indexed by j - lo
  const float* lg = logits + (size_t(b) * Hkv + g) * cap * G;
  float* sc = score + (size_t(b) * Hkv + g) * cap;
  const int64_t j_hi = min(lo + int64_t(c + 1) * CH, j_end);
  for (int64_t j = lo + int64_t(c) * CH + threadIdx.x; j < j_hi; j += 256) {
    // the G logits of key j: 16-byte loads where G allows
    float x[G];
    if constexpr (G % 4 == 0) {
#pragma unroll
      for (int h = 0; h < G; h += 4) {
        const float4 v = *reinterpret_cast<const float4*>(lg + (j - lo) * G + h);
        x[h] = v.x;
        x[h + 1] = v.y;
        x[h + 2] = v.z;
        x[h + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h) x[h] = lg[(j - lo) * G + h];
    }
    float acc = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) acc += fast_exp2(x[h] - sl[h]);
    sc[j - lo] = acc;
    atomicAdd(&sh[__float_as_uint(acc) >> 20], 1u);
  }
  __syncthreads();
  uint32_t* gh = hist + (size_t(b) * Hkv + g) * NBUCKET;
  for (int i = threadIdx.x; i < NBUCKET; i += 256)
    if (sh[i]) atomicAdd(&gh[i], sh[i]);
  // the last CTA of (b, g) to finish finds the bucket of the k-th best score
  __shared__ uint32_t s_last, s_scan[256];
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&done[size_t(b) * Hkv + g], 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    const int kb = block_kth_bucket(gh, uint32_t(k), s_scan);
    if (threadIdx.x == 0) kth_bucket[size_t(b) * Hkv + g] = kb;
  }
}

// bucket holding the k-th largest count from the top (NBUCKET bins, 256
// threads); returns -1 if the total is below k
__device__ int block_kth_bucket(const uint32_t* __restrict__ gh, uint32_t k, uint32_t* s_scan) {
  // each thread sums 8 bins (highest first)
  const int tid = threadIdx.x;
  uint32_t c8[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c8[i] = __ldcg(gh + NBUCKET - 1 - 8 * tid - i);  // other CTAs' atomics, from L2
    local += c8[i];
  }
  s_scan[tid] = local;
  __syncthreads();
  // inclusive scan over 256 threads (simple Hillis-Steele)
  for (int off = 1; off < 256; off <<= 1) {
    const uint32_t v = tid >= off ? s_scan[tid - off] : 0u;
    __syncthreads();
    s_scan[tid] += v;
    __syncthreads();
  }
  __shared__ int found;
  if (tid == 0) found = -1;
  __syncthreads();
  const uint32_t incl = s_scan[tid], excl = incl - local;
  if (excl < k && k <= incl) {
    uint32_t cum = excl;
    for (int i = 0; i < 8; ++i) {
      if (cum + c8[i] >= k) {
        found = NBUCKET - 1 - 8 * tid - i;
        break;
      }
      cum += c8[i];
    }
  }
  __syncthreads();
  return found;
}

// ---------------------------------------------------------------------------
// decode_collect: grid (chunks, Hkv, B), 256 threads
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    decode_collect(const float* __restrict__ score, const int* __restrict__ kth_bucket,
                   SeqLens seq_len, int64_t cap, int Hkv, int k, int w,
                   uint2* __restrict__ cand, uint32_t* __restrict__ ccount) {
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int N = seq_len.n[b];
  const int64_t s_lo = seq_len.lo[b];
  const int64_t s_hi = min(int64_t(N) - w, int64_t(seq_len.hi[b]));  // slice candidates [s_lo, s_hi)
  if (s_hi - s_lo <= k) return;  // every candidate is selected; decode_final writes them
  const int64_t j_lo = s_lo + int64_t(c) * CH;
  const int64_t j_hi = min(j_lo + CH, s_hi);
  if (j_lo >= j_hi) return;
  const size_t bg = size_t(b) * Hkv + g;
  const int kb = kth_bucket[bg];
  const uint32_t thr = kb < 0 ? 0u : uint32_t(kb);
  const float* sc = score + bg * cap;  // score of key j at sc[j - s_lo]
  const int lane = lane_id();
  const bool vec = (cap & 3) == 0;  // rows of scores start 16-byte aligned
  // in local indices x = j - s_lo: rounds of 2048 keys from a multiple of 4
  // at or below x_lo; thread owns keys x0 .. x0+3 and x0+1024 .. x0+1027
  // (16-byte aligned when cap is a multiple of 4); all eight loads are
  // issued before any is used
  const int64_t x_lo = j_lo - s_lo, x_hi = j_hi - s_lo;
  for (int64_t base = x_lo & ~int64_t(3); base < x_hi; base += 2048) {
    float v[8];
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
      const int64_t x0 = base + 1024 * hlf + 4 * threadIdx.x;
      if (vec && x0 + 3 < x_hi) {
        const float4 x = __ldcs(reinterpret_cast<const float4*>(sc + x0));
        v[4 * hlf] = x.x;
        v[4 * hlf + 1] = x.y;
        v[4 * hlf + 2] = x.z;
        v[4 * hlf + 3] = x.w;
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) v[4 * hlf + u] = x0 + u < x_hi ? sc[x0 + u] : 0.f;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int64_t xl = base + 1024 * (e >> 2) + 4 * threadIdx.x + (e & 3);
      const int64_t j = xl + s_lo;
      const bool take = xl >= x_lo && xl < x_hi && (__float_as_uint(v[e]) >> 20) >= thr;
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (bal) {
        uint32_t pos = 0;
        if (lane == __ffs(bal) - 1) pos = atomicAdd(&ccount[bg], __popc(bal));
        pos = __shfl_sync(0xffffffffu, pos, __ffs(bal) - 1);
        const uint32_t p = pos + __popc(bal & ((1u << lane) - 1u));
        if (take && p < uint32_t(CAPC))
          cand[bg * CAPC + p] = make_uint2(__float_as_uint(v[e]), uint32_t(j));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// decode_final: grid (Hkv, B), 512 threads
// ---------------------------------------------------------------------------
__device__ void block_bitonic_u64(uint64_t* s, int np, bool descending) {
  for (int size = 2; size <= np; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < np / 2; i += blockDim.x) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool up = ((lo & size) == 0) != descending;
        const uint64_t a = s[lo], bb = s[hi];
        if ((a > bb) == up) {
          s[lo] = bb;
          s[hi] = a;
        }
      }
      __syncthreads();
    }
}

// What decode_final reads and writes.
//   FINAL_FULL   the whole block on one device: the top k of the candidate
//                list (or, when it overflowed, of every candidate's score),
//                positions ascending, then the window, into idx.
//   FINAL_LOCAL  one rank of a context split over ranks: the top k of the
//                candidates in its slice as records (score bits, position),
//                [B][Hkv][k], padded with (0, 0xFFFFFFFF) (below every real
//                candidate) when the slice has fewer.
//   FINAL_MERGE  the top k of the ranks' gathered records, positions
//                ascending, then the window, into idx.  Record e of (b, g)
//                is recs[(e / k) * rank_stride + (b * Hkv + g) * k + e % k].
enum { FINAL_FULL = 0, FINAL_LOCAL = 1, FINAL_MERGE = 2 };

struct FinalIO {
  const uint2* cand;        // decode_collect's lists [B][Hkv][CAPC]
  const uint32_t* ccount;   // and their lengths
  const uint2* recs;        // FINAL_MERGE: gathered records
  int n_ranks;
  int64_t rank_stride;      // in records
  uint2* rec_out;           // FINAL_LOCAL: this rank's records
  int32_t* idx;             // FINAL_FULL / FINAL_MERGE: [B][Hkv][k + w]
};

template <int MODE>
__global__ void __launch_bounds__(512)
    decode_final(FinalIO io, const float* __restrict__ score, SeqLens seq_len, int64_t cap,
                 int Hkv, int k, int w) {
  extern __shared__ uint64_t sk[];  // CAPC keys
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_misc[4];
  const int g = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int N = seq_len.n[b];
  const int64_t i = N - 1;
  const int64_t ncand = max(int64_t(0), i - w + 1);
  const size_t bg = size_t(b) * Hkv + g;
  int32_t* out = MODE == FINAL_LOCAL ? nullptr : io.idx + bg * (k + w);
  uint2* rec = MODE == FINAL_LOCAL ? io.rec_out + bg * k : nullptr;
  // candidates of this call: all of [0, ncand), or those of the slice
  const int64_t c_lo = MODE == FINAL_LOCAL ? min(int64_t(seq_len.lo[b]), ncand) : 0;
  const int64_t c_hi = MODE == FINAL_LOCAL ? min(int64_t(seq_len.hi[b]), ncand) : ncand;
  const int64_t nc = max(int64_t(0), c_hi - c_lo);
  // score of candidate j at sc[j - lo] (the cache holds the slice from lo)
  const int64_t lo = seq_len.lo[b];
  const float* sc = score + bg * cap;
  if (MODE != FINAL_LOCAL) {
    for (int t2 = tid; t2 < w; t2 += blockDim.x) {
      const int64_t p = i - w + 1 + t2;
      out[k + t2] = p >= 0 ? int32_t(p) : -1;
    }
  }
  if (nc <= k) {
    if (MODE == FINAL_LOCAL) {
      for (int e = tid; e < k; e += blockDim.x)
        rec[e] = e < nc ? make_uint2(__float_as_uint(sc[c_lo + e - lo]), uint32_t(c_lo + e))
                        : make_uint2(0u, 0xFFFFFFFFu);
    } else {
      for (int e = tid; e < k; e += blockDim.x) out[e] = e < nc ? e : -1;
    }
    return;
  }
  const uint32_t n = MODE == FINAL_MERGE ? uint32_t(io.n_ranks) * uint32_t(k) : io.ccount[bg];
  if (n <= uint32_t(CAPC)) {
    int np = 1;
    while (np < int(n)) np <<= 1;
    for (int e = tid; e < np; e += blockDim.x) {
      if (e < int(n)) {
        const uint2 v = MODE == FINAL_MERGE
                            ? io.recs[(e / k) * io.rank_stride + int64_t(bg) * k + e % k]
                            : io.cand[bg * CAPC + e];
        sk[e] = (uint64_t(v.x) << 32) | uint64_t(~v.y);
      } else {
        sk[e] = 0;  // below every real key
      }
    }
    __syncthreads();
    block_bitonic_u64(sk, np, true);  // best first
    if (MODE == FINAL_LOCAL) {
      for (int e = tid; e < k; e += blockDim.x)
        rec[e] = make_uint2(uint32_t(sk[e] >> 32), ~uint32_t(sk[e]));
      return;
    }
    // the k best positions, ascending
    int kp = 1;
    while (kp < k) kp <<= 1;
    __syncthreads();
    for (int e = tid; e < kp; e += blockDim.x)
      sk[e] = e < k ? uint64_t(~uint32_t(sk[e])) : ~uint64_t(0);
    __syncthreads();
    block_bitonic_u64(sk, kp, false);
    for (int e = tid; e < k; e += blockDim.x) out[e] = int32_t(sk[e]);
    return;
  }
  // overflow (FULL / LOCAL): exact radix select over every candidate's score,
  // then the selected positions in ascending order by a block-wide ordered scan
  uint64_t prefix = 0, mask = 0;
  uint32_t remaining = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int e = tid; e < 256; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
    for (int64_t j = c_lo + tid; j < c_hi; j += blockDim.x) {
      const uint64_t key = (uint64_t(__float_as_uint(sc[j - lo])) << 32) | uint64_t(~uint32_t(j));
      if ((key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & 255], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0;
      int bin = 255;
      for (; bin >= 0; --bin) {
        if (cum + s_hist[bin] >= remaining) break;
        cum += s_hist[bin];
      }
      s_misc[0] = uint32_t(bin);
      s_misc[1] = cum;
      s_misc[2] = s_hist[bin];
    }
    __syncthreads();
    const uint32_t bin = s_misc[0], above = s_misc[1], inbin = s_misc[2];
    __syncthreads();
    remaining -= above;
    prefix |= uint64_t(bin) << shift;
    mask |= uint64_t(0xFF) << shift;
    if (inbin == remaining) break;
  }
  __shared__ uint32_t s_warp[16];
  uint32_t written = 0;
  for (int64_t base = c_lo; base < c_hi; base += blockDim.x) {
    const int64_t j = base + tid;
    bool sel = false;
    float v = 0.f;
    if (j < c_hi) {
      v = sc[j - lo];
      const uint64_t key = (uint64_t(__float_as_uint(v)) << 32) | uint64_t(~uint32_t(j));
      sel = (key & mask) >= prefix;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    if (lane_id() == 0) s_warp[warp_id()] = __popc(bal);
    __syncthreads();
    uint32_t before = written;
    for (int w2 = 0; w2 < warp_id(); ++w2) before += s_warp[w2];
    uint32_t tot = 0;
    for (int w2 = 0; w2 < int(blockDim.x / 32); ++w2) tot += s_warp[w2];
    if (sel) {
      const uint32_t p = before + __popc(bal & ((1u << lane_id()) - 1u));
      if (p < uint32_t(k)) {
        if (MODE == FINAL_LOCAL)
          rec[p] = make_uint2(__float_as_uint(v), uint32_t(j));
        else
          out[p] = int32_t(j);
      }
    }
    written += tot;
    __syncthreads();
  }
}

template <int G>
cudaError_t launch_dec_g(const DecodeArgs& a, const SeqLens& d_seq, int max_len, cudaStream_t st,
                         uint8_t* w8) {
  const int Hq = a.Hq, Hkv = a.Hkv, B = a.B;
  const int nch = int((a.cap + CH - 1) / CH);
  const int nch_used = (max_len + CH - 1) / CH;  // chunks of the longest slice (<= nch)
  const bool full = a.step == DEC_FULL;
  // workspace layout (see decode_workspace_bytes); DEC_CP_ATTN leaves the
  // logits there for DEC_CP_SELECT
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = w8 + off;
    off += (bytes + 255) / 256 * 256;
    return p;
  };
  float* logits = reinterpret_cast<float*>(take(size_t(B) * Hkv * a.cap * G * 4));
  float* score = reinterpret_cast<float*>(take(size_t(B) * Hkv * a.cap * 4));
  Partial* part = reinterpret_cast<Partial*>(take(size_t(B) * Hq * nch * sizeof(Partial)));
  float* part_o = reinterpret_cast<float*>(take(size_t(B) * Hq * nch * 128 * 4));
  float* lse2 = reinterpret_cast<float*>(take(size_t(B) * Hq * 4));
  uint32_t* hist = reinterpret_cast<uint32_t*>(take(size_t(B) * Hkv * NBUCKET * 4));
  // per (b, g): candidate count, finished scoring CTAs, k-th best bucket
  uint32_t* ccount = reinterpret_cast<uint32_t*>(take(size_t(B) * Hkv * 12));
  uint32_t* done = ccount + size_t(B) * Hkv;
  int* kth_bucket = reinterpret_cast<int*>(done + size_t(B) * Hkv);
  uint2* cand = reinterpret_cast<uint2*>(take(size_t(B) * Hkv * CAPC * 8));
  const float sl2 = a.scale * kLog2e;
  cudaError_t e = cudaSuccess;
  unsigned launches = 0;

  if (full || a.step == DEC_CP_ATTN) {
    // K, V codes viewed as [B*cap tokens][Hkv][64 two-byte units]: 64-row boxes
    CUtensorMap tmK, tmV;
    const uint64_t rows = uint64_t(B) * a.cap;
    if (!make_tmap_3d(&tmK, a.Kc, 64, Hkv, rows, 128, uint64_t(Hkv) * 128, 64, 1, DSTAGE_KEYS) ||
        !make_tmap_3d(&tmV, a.Vc, 64, Hkv, rows, 128, uint64_t(Hkv) * 128, 64, 1, DSTAGE_KEYS))
      return cudaErrorInvalidValue;
    const int psmem = DSTAGES * DSTAGE_BYTES + 1024;
    e = ensure_smem_attr(reinterpret_cast<const void*>(decode_partial<G>), psmem);
    if (e != cudaSuccess) return e;
    if (nch_used > 0)
      decode_partial<G><<<dim3(Hkv, nch_used, B), (DP_WARPS + 1) * 32, psmem, st>>>(
          tmK, tmV, reinterpret_cast<const __nv_bfloat16*>(a.q), a.ks, a.vs, d_seq, a.cap, Hkv,
          nch, sl2, logits, part, part_o);
    decode_merge<<<dim3(Hq, B), 128 * MERGE_GROUPS, 0, st>>>(
        part, part_o, d_seq, Hq, nch, reinterpret_cast<__nv_bfloat16*>(a.o), a.lse, lse2,
        full ? nullptr : a.attn_rec);
    launches += 2;
    if (!full) {
      count_launch(launches);
      return cudaGetLastError();
    }
  }
  if (a.step == DEC_CP_SELECT) {
    decode_merge_ranks<<<dim3(Hq, B), 128, 0, st>>>(
        a.attn_recs, a.n_ranks, int64_t(B) * Hq * REC, Hq, reinterpret_cast<__nv_bfloat16*>(a.o),
        a.lse, lse2);
    ++launches;
  }
  if (full || a.step == DEC_CP_SELECT) {
    e = cudaMemsetAsync(hist, 0, size_t(B) * Hkv * NBUCKET * 4, st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(ccount, 0, size_t(B) * Hkv * 8, st);  // counts and tickets
    if (e != cudaSuccess) return e;
    if (nch_used > 0) {
      decode_score<G><<<dim3(nch_used, Hkv, B), 256, 0, st>>>(logits, lse2, d_seq, a.cap, Hkv,
                                                              a.k, a.w, score, hist, done,
                                                              kth_bucket);
      decode_collect<<<dim3(nch_used, Hkv, B), 256, 0, st>>>(score, kth_bucket, d_seq, a.cap,
                                                             Hkv, a.k, a.w, cand, ccount);
      launches += 2;
    }
    const int fsmem = CAPC * 8;
    FinalIO io{};
    io.cand = cand;
    io.ccount = ccount;
    if (full) {
      io.idx = a.idx;
      e = ensure_smem_attr(reinterpret_cast<const void*>(decode_final<FINAL_FULL>), fsmem);
      if (e != cudaSuccess) return e;
      decode_final<FINAL_FULL><<<dim3(Hkv, B), 512, fsmem, st>>>(io, score, d_seq, a.cap, Hkv,
                                                                 a.k, a.w);
    } else {
      io.rec_out = a.sel_rec;
      e = ensure_smem_attr(reinterpret_cast<const void*>(decode_final<FINAL_LOCAL>), fsmem);
      if (e != cudaSuccess) return e;
      decode_final<FINAL_LOCAL><<<dim3(Hkv, B), 512, fsmem, st>>>(io, score, d_seq, a.cap, Hkv,
                                                                  a.k, a.w);
    }
    ++launches;
    if (!full) {
      count_launch(launches);
      return cudaGetLastError();
    }
  }
  if (a.step == DEC_CP_SPARSE) {
    const int fsmem = CAPC * 8;
    FinalIO io{};
    io.recs = a.sel_recs;
    io.n_ranks = a.n_ranks;
    io.rank_stride = int64_t(B) * Hkv * a.k;
    io.idx = a.idx;
    e = ensure_smem_attr(reinterpret_cast<const void*>(decode_final<FINAL_MERGE>), fsmem);
    if (e != cudaSuccess) return e;
    decode_final<FINAL_MERGE><<<dim3(Hkv, B), 512, fsmem, st>>>(io, score, d_seq, a.cap, Hkv,
                                                                a.k, a.w);
    ++launches;
  }
  count_launch(launches);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (full || a.step == DEC_CP_SPARSE) {
    for (int l = 0; l < a.n_sparse; ++l) {
      SparseArgs s{};
      s.Q = a.qs[l];
      s.idx = a.idx;
      s.O = full ? a.os[l] : nullptr;
      s.lse = nullptr;
      s.T = B;
      s.Hq = Hq;
      s.Hkv = Hkv;
      s.scale = a.scale;
      s.kw = a.k + a.w;
      s.Kc = a.Kc;
      s.Vc = a.Vc;
      s.ks = a.ks;
      s.vs = a.vs;
      s.cache_T = a.cap;
      for (int b = 0; b < B; ++b) {
        s.spans.lo[b] = d_seq.lo[b];
        s.spans.hi[b] = full ? int(a.cap) : d_seq.hi[b];
      }
      s.rec = full ? nullptr : a.sparse_rec + size_t(l) * B * Hq * REC;
      e = launch_sparse(s, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  if (a.step == DEC_CP_FINISH) {
    for (int l = 0; l < a.n_sparse; ++l) {
      decode_merge_ranks<<<dim3(Hq, B), 128, 0, st>>>(
          a.sparse_recs + size_t(l) * B * Hq * REC, a.n_ranks, int64_t(a.n_sparse) * B * Hq * REC,
          Hq, reinterpret_cast<__nv_bfloat16*>(a.os[l]), nullptr, nullptr);
    }
    count_launch(a.n_sparse);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

size_t dec_ws_bytes(int B, int64_t cap, int Hq, int Hkv) {
  const int G = Hq / Hkv;
  const int nch = int((cap + CH - 1) / CH);
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  return r(size_t(B) * Hkv * cap * G * 4) + r(size_t(B) * Hkv * cap * 4) +
         r(size_t(B) * Hq * nch * sizeof(Partial)) + r(size_t(B) * Hq * nch * 128 * 4) +
         r(size_t(B) * Hq * 4) + r(size_t(B) * Hkv * NBUCKET * 4) + r(size_t(B) * Hkv * 12) +
         r(size_t(B) * Hkv * CAPC * 8);
}

}  // namespace

size_t decode_workspace_bytes(int B, int64_t cap, int Hq, int Hkv, int k, int w) {
  (void)k;
  (void)w;
  return dec_ws_bytes(B, cap, Hq, Hkv);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.B > MAX_B || a.k > CAPC / 2 || int64_t(a.B) * a.cap > INT32_MAX) return cudaErrorNotSupported;
  if (a.step != DEC_FULL && int64_t(a.n_ranks) * a.k > CAPC) return cudaErrorNotSupported;
  SeqLens d_seq{};
  int max_len = 0;  // the longest slice
  for (int b = 0; b < a.B; ++b) {
    d_seq.n[b] = int(a.seq_len_host[b]);
    d_seq.lo[b] = a.lo_host != nullptr ? int(a.lo_host[b]) : 0;
    d_seq.hi[b] = a.hi_host != nullptr ? int(a.hi_host[b]) : d_seq.n[b];
    max_len = d_seq.hi[b] - d_seq.lo[b] > max_len ? d_seq.hi[b] - d_seq.lo[b] : max_len;
  }
  uint8_t* w8 = reinterpret_cast<uint8_t*>(a.ws);
  switch (a.Hq / a.Hkv) {
    case 1: return launch_dec_g<1>(a, d_seq, max_len, st, w8);
    case 2: return launch_dec_g<2>(a, d_seq, max_len, st, w8);
    case 4: return launch_dec_g<4>(a, d_seq, max_len, st, w8);
    case 8: return launch_dec_g<8>(a, d_seq, max_len, st, w8);
    case 16: return launch_dec_g<16>(a, d_seq, max_len, st, w8);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hs2
