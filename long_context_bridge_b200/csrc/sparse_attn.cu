// sparse_attn.cu -- sparse attention over the shared K/V and index list.
//
// KV Reuse (javabetter.cn explainer "mimo-v3-hysparse2", KV Reuse paragraph;
// aitop.news summary): each sparse layer attends with its own queries to the
// full-attention layer's K/V cache at the positions on that layer's token list
// and keeps no K/V of its own.
//
// One warp handles one (query row, KV head) pair and its G query heads:
//   * the warp walks the list 32 entries at a time; lane t gathers K row
//     idx[t] with 16-byte loads and forms the G logits against the queries
//     held in shared memory (pre-scaled by scale * log2 e);
//   * online softmax per head across the warp (base-2 exponent);
//   * V rows of the batch are read coalesced (lane l owns dims 4l..4l+3) and
//     accumulated with the batch's probabilities, staged in shared memory.
// The FP8 variant reads e4m3 codes and folds the per-(token, head) scales into
// the logit (K) and into the probability weight (V).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_sparse)

namespace {

constexpr int WARPS = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// two e4m3 codes (low byte first) -> two floats, exact
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

template <int G, bool FP8>
__global__ void __launch_bounds__(WARPS * 32)
    sparse_attn_kernel(const __nv_bfloat16* __restrict__ Q, const void* __restrict__ Kp,
                       const void* __restrict__ Vp, const float* __restrict__ ks,
                       const float* __restrict__ vs, const int32_t* __restrict__ idx,
                       __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int64_t rows,
                       int Hkv, int kw, float scale_log2, int64_t cache_T) {
  __shared__ __align__(16) float sq[WARPS][G][128];
  __shared__ float sp[WARPS][G][32];
  __shared__ int sj[WARPS][32];
  __shared__ float svs[WARPS][32];

  const int w = warp_id(), lane = lane_id();
  const int64_t pair = int64_t(blockIdx.x) * WARPS + w;
  if (pair >= rows * Hkv) return;
  const int64_t r = pair / Hkv;
  const int g = int(pair % Hkv);
  const int Hq = Hkv * G;
  const int64_t tok0 = FP8 ? r * cache_T : 0;  // decode: sequence r's cache

  // queries of the group, pre-scaled to the base-2 logit domain
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint2 v = *reinterpret_cast<const uint2*>(Q + (r * Hq + g * G + h) * 128 + lane * 4);
    sq[w][h][lane * 4 + 0] = bf16lo(v.x) * scale_log2;
    sq[w][h][lane * 4 + 1] = bf16hi(v.x) * scale_log2;
    sq[w][h][lane * 4 + 2] = bf16lo(v.y) * scale_log2;
    sq[w][h][lane * 4 + 3] = bf16hi(v.y) * scale_log2;
  }
  __syncwarp();

  const int32_t* list = idx + pair * kw;
  float m[G], l[G], acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
    acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
  }

  for (int base = 0; base < kw; base += 32) {
    const int t = base + lane;
    const int j = t < kw ? list[t] : -1;
    float s[G];
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = -INFINITY;
    float vscale = 0.f;
    if (j >= 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) s[h] = 0.f;
      const int64_t row = (tok0 + j) * Hkv + g;
      if constexpr (!FP8) {
        const uint4* kr = reinterpret_cast<const uint4*>(
            reinterpret_cast<const __nv_bfloat16*>(Kp) + row * 128);
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const uint4 u = __ldg(kr + c);
          const float k8[8] = {bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y),
                               bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w)};
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float4 q0 = *reinterpret_cast<const float4*>(&sq[w][h][c * 8]);
            const float4 q1 = *reinterpret_cast<const float4*>(&sq[w][h][c * 8 + 4]);
            s[h] += q0.x * k8[0] + q0.y * k8[1] + q0.z * k8[2] + q0.w * k8[3] + q1.x * k8[4] +
                    q1.y * k8[5] + q1.z * k8[6] + q1.w * k8[7];
          }
        }
      } else {
        const uint4* kr =
            reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(Kp) + row * 128);
#pragma unroll 2
        for (int c = 0; c < 8; ++c) {
          const uint4 u = __ldg(kr + c);
          const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
          float k16[16];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 a = e4m3x2_to_float2(uint16_t(wds[q] & 0xFFFF));
            const float2 b = e4m3x2_to_float2(uint16_t(wds[q] >> 16));
            k16[4 * q + 0] = a.x;
            k16[4 * q + 1] = a.y;
            k16[4 * q + 2] = b.x;
            k16[4 * q + 3] = b.y;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float acc_h = 0.f;
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 qv = *reinterpret_cast<const float4*>(&sq[w][h][c * 16 + e]);
              acc_h += qv.x * k16[e] + qv.y * k16[e + 1] + qv.z * k16[e + 2] + qv.w * k16[e + 3];
            }
            s[h] += acc_h;
          }
        }
        const float kscale = __ldg(ks + row);
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] *= kscale;
        vscale = __ldg(vs + row);
      }
    }
    // online softmax, base 2
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float bm = warp_max(s[h]);
      const float mn = fmaxf(m[h], bm);
      float p = 0.f, alpha = 1.f;
      if (mn != -INFINITY) {
        alpha = fast_exp2(m[h] - mn);  // m = -inf -> 0
        p = j >= 0 ? fast_exp2(s[h] - mn) : 0.f;
      }
      l[h] = l[h] * alpha + warp_sum(p);
      acc[h][0] *= alpha;
      acc[h][1] *= alpha;
      acc[h][2] *= alpha;
      acc[h][3] *= alpha;
      m[h] = mn;
      sp[w][h][lane] = p;
    }
    sj[w][lane] = j;
    svs[w][lane] = vscale;
    __syncwarp();
    const int nb = min(32, kw - base);
    for (int tt = 0; tt < nb; ++tt) {
      const int jj = sj[w][tt];
      if (jj < 0) continue;
      const int64_t row = (tok0 + jj) * Hkv + g;
      float v4[4];
      if constexpr (!FP8) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(
            reinterpret_cast<const __nv_bfloat16*>(Vp) + row * 128 + lane * 4));
        v4[0] = bf16lo(u.x);
        v4[1] = bf16hi(u.x);
        v4[2] = bf16lo(u.y);
        v4[3] = bf16hi(u.y);
      } else {
        const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(
            reinterpret_cast<const uint8_t*>(Vp) + row * 128 + lane * 4));
        const float2 a = e4m3x2_to_float2(uint16_t(u & 0xFFFF));
        const float2 b = e4m3x2_to_float2(uint16_t(u >> 16));
        const float sv = svs[w][tt];
        v4[0] = a.x * sv;
        v4[1] = a.y * sv;
        v4[2] = b.x * sv;
        v4[3] = b.y * sv;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = sp[w][h][tt];
        acc[h][0] += p * v4[0];
        acc[h][1] += p * v4[1];
        acc[h][2] += p * v4[2];
        acc[h][3] += p * v4[3];
      }
    }
    __syncwarp();
  }

#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
    uint2 o;
    o.x = pack_bf16x2(acc[h][0] * inv, acc[h][1] * inv);
    o.y = pack_bf16x2(acc[h][2] * inv, acc[h][3] * inv);
    *reinterpret_cast<uint2*>(O + (r * Hq + g * G + h) * 128 + lane * 4) = o;
    if (lse != nullptr && lane == 0)
      lse[r * Hq + g * G + h] = l[h] > 0.f ? (m[h] + __log2f(l[h])) * kLn2 : -INFINITY;
  }
}

template <int G>
cudaError_t launch_g(const SparseArgs& a, cudaStream_t stream) {
  const int64_t pairs = a.T * a.Hkv;
  const dim3 grid(unsigned((pairs + WARPS - 1) / WARPS));
  const float sl2 = a.scale * kLog2e;
  if (a.Kc != nullptr) {
    sparse_attn_kernel<G, true><<<grid, WARPS * 32, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(a.Q), a.Kc, a.Vc, a.ks, a.vs, a.idx,
        reinterpret_cast<__nv_bfloat16*>(a.O), a.lse, a.T, a.Hkv, a.kw, sl2, a.cache_T);
  } else {
    sparse_attn_kernel<G, false><<<grid, WARPS * 32, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(a.Q), a.K, a.V, nullptr, nullptr, a.idx,
        reinterpret_cast<__nv_bfloat16*>(a.O), a.lse, a.T, a.Hkv, a.kw, sl2, 0);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace

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
