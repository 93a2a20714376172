// bridge_gemm.cu -- KV Bridging projection K = H W_k, V = H W_v on tcgen05.
//
// KV Bridging (javabetter.cn explainer "mimo-v3-hysparse2", KV Bridging
// paragraph; siami.tw article section 一): the cross-decoder full-attention
// layer computes its K/V from self-decoder hidden states with its own weights.
//
// One CTA computes a 128 x BN tile of [K | V] (N index n < Nkv -> K, else V):
//   warp 0     TMA producer: H tile [128 x 64] (K-major) and W tile [64 x BN]
//              (MN-major, W is row-major [d_model, Nkv]) into a STAGES ring
//   warp 1     allocates TMEM, one lane issues tcgen05.mma 128xBNx16 and
//              commits each stage back to the producer
//   warps 2-5  epilogue: TMEM -> registers -> bf16 -> global
// bridge_fp8_kernel (further down) is the same GEMM with the K and V tiles of
// one KV head in one CTA and an epilogue that writes the FP8 decode cache.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_bridge)
HS2_BUDGET_SETTER(budget_bridge)


namespace {
constexpr int BM = 128, BK = 64, STAGES = 3;
constexpr int THREADS = 192;

template <int BN>
struct BridgeCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * BN * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr uint32_t IDESC = idesc_bf16(BM, BN, /*a_mn=*/0, /*b_mn=*/1);
};

template <int BN>
__global__ void __launch_bounds__(THREADS, 1)
    bridge_gemm_kernel(const __grid_constant__ CUtensorMap tmH,
                       const __grid_constant__ CUtensorMap tmWk,
                       const __grid_constant__ CUtensorMap tmWv, __nv_bfloat16* __restrict__ K,
                       __nv_bfloat16* __restrict__ V, int T, int dm, int Nkv) {
  using C = BridgeCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accbar = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);

  const int warp = warp_id(), lane = lane_id();
  const int n0 = blockIdx.x * BN;  // column of [K | V]
  const int m0 = blockIdx.y * BM;
  const bool isV = n0 >= Nkv;
  const int nloc = isV ? n0 - Nkv : n0;
  const int num_kb = dm / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accbar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    prefetch_tmap(&tmH);
    prefetch_tmap(isV ? &tmWv : &tmWk);
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      if (kb >= STAGES && !mbar_wait(&empty[s], ((kb / STAGES) & 1) ^ 1)) break;
      uint8_t* sA = smem + s * C::STAGE_BYTES;
      uint8_t* sB = sA + C::A_BYTES;
      mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
      tma_load_2d(sA, &tmH, &full[s], kb * BK, m0);
#pragma unroll
      for (int c = 0; c < BN / 64; ++c)
        tma_load_2d(sB + c * (BK * 128), isV ? &tmWv : &tmWk, &full[s], nloc + c * 64, kb * BK);
      issued = kb + 1;
    }
    // every issued copy lands before the CTA can exit
    for (int s = 0; s < STAGES; ++s) drain_phase(&full[s], issued > s ? (issued - 1 - s) / STAGES + 1 : 0);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    bool ok = true;
    for (int kb = 0; kb < num_kb && ok; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait(&full[s], (kb / STAGES) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * C::STAGE_BYTES);
      const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
      for (int ks = 0; ks < BK / 16; ++ks) {
        // A: K-major, advance 16 elements = 32 B inside the 128 B swizzle row
        const uint64_t ad = sdesc_sw128(a0 + ks * 32, 16, 1024);
        // B: MN-major, advance 16 K-rows of 128 B; MN chunks of 64 are BK*128 B apart
        const uint64_t bd = sdesc_sw128(b0 + ks * 16 * 128, BK * 128, 1024);
        mma_ss(tmem, ad, bd, C::IDESC, (kb | ks) != 0);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(accbar);
    mbar_wait_budget(accbar, 0, kDrainBudgetCycles);  // no MMA outlives the TMEM
  } else if (warp >= 2) {
    // ---------------- epilogue ----------------
    const int sub = warp & 3;  // TMEM lanes 32*sub .. 32*sub+31
    const bool ok = mbar_wait(accbar, 0);
    tc_fence_after();
    const int row = m0 + sub * 32 + lane;
    __nv_bfloat16* out = isV ? V : K;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + (uint32_t(sub * 32) << 16) + c * 32, r);
      tmem_wait_ld();
      if (ok && row < T) {
        uint4* dst = reinterpret_cast<uint4*>(out + size_t(row) * Nkv + nloc + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
          v.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
          v.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
          v.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
          dst[q] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}
// ---------------------------------------------------------------------------
// Bridge-only prefill into the FP8 cache: one CTA = 128 tokens x one KV head,
// with both its K tile and its V tile (two TMEM accumulators of 128 columns),
// so that the epilogue holds the whole (token, head) row pair for the scale
//   s = max(amax|K row|, amax|V row|) / 448 (fp32; 1 for an all-zero pair)
// and writes codes = e4m3(bf16(x) / s) (fp32 quotient, nearest, ties to even,
// saturated) into the cache layout [T][Hkv][128] plus s into [T][Hkv].
// Two stages of {H 128x64, W_k 64x128, W_v 64x128}; two CTAs per SM, so one
// CTA's epilogue overlaps the other's MMAs.
// ---------------------------------------------------------------------------
constexpr int F_STAGES = 2;
constexpr int F_A_BYTES = BM * BK * 2;
constexpr int F_B_BYTES = BK * 128 * 2;
constexpr int F_STAGE_BYTES = F_A_BYTES + 2 * F_B_BYTES;
constexpr int F_SMEM = F_STAGES * F_STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t F_IDESC = idesc_bf16(BM, 128, /*a_mn=*/0, /*b_mn=*/1);

__device__ __forceinline__ float bf16_rounded(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ uint32_t e4m3_code(float q) {
  return uint32_t(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
}

__global__ void __launch_bounds__(THREADS, 2)
    bridge_fp8_kernel(const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmWk,
                      const __grid_constant__ CUtensorMap tmWv, uint8_t* __restrict__ Kc,
                      uint8_t* __restrict__ Vc, float* __restrict__ scale, int T, int dm,
                      int Hkv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + F_STAGES * F_STAGE_BYTES);
  uint64_t* empty = full + F_STAGES;
  uint64_t* accbar = empty + F_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);

  const int warp = warp_id(), lane = lane_id();
  const int g = blockIdx.x;  // KV head: columns 128g .. 128g+127 of W_k and W_v
  const int m0 = blockIdx.y * BM;
  const int num_kb = dm / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < F_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accbar, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // K accumulator at +0, V at +128

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmWk);
    prefetch_tmap(&tmWv);
    int issued = 0;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % F_STAGES;
      if (kb >= F_STAGES && !mbar_wait(&empty[s], ((kb / F_STAGES) & 1) ^ 1)) break;
      issued = kb + 1;
      uint8_t* sA = smem + s * F_STAGE_BYTES;
      uint8_t* sBk = sA + F_A_BYTES;
      uint8_t* sBv = sBk + F_B_BYTES;
      mbar_arrive_expect_tx(&full[s], F_STAGE_BYTES);
      tma_load_2d(sA, &tmH, &full[s], kb * BK, m0);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(sBk + c * (BK * 128), &tmWk, &full[s], g * 128 + c * 64, kb * BK);
        tma_load_2d(sBv + c * (BK * 128), &tmWv, &full[s], g * 128 + c * 64, kb * BK);
      }
    }
    for (int s = 0; s < F_STAGES; ++s)
      drain_phase(&full[s], issued > s ? (issued - 1 - s) / F_STAGES + 1 : 0);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    bool ok = true;
    for (int kb = 0; kb < num_kb && ok; ++kb) {
      const int s = kb % F_STAGES;
      if (!mbar_wait(&full[s], (kb / F_STAGES) & 1)) { ok = false; break; }
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * F_STAGE_BYTES);
      const uint32_t bk0 = a0 + F_A_BYTES, bv0 = bk0 + F_B_BYTES;
#pragma unroll
      for (int ks = 0; ks < BK / 16; ++ks) {
        const uint64_t ad = sdesc_sw128(a0 + ks * 32, 16, 1024);
        const uint64_t bkd = sdesc_sw128(bk0 + ks * 16 * 128, BK * 128, 1024);
        const uint64_t bvd = sdesc_sw128(bv0 + ks * 16 * 128, BK * 128, 1024);
        mma_ss(tmem, ad, bkd, F_IDESC, (kb | ks) != 0);
        mma_ss(tmem + 128, ad, bvd, F_IDESC, (kb | ks) != 0);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(accbar);
    mbar_wait_budget(accbar, 0, kDrainBudgetCycles);  // no MMA outlives the TMEM
  } else if (warp >= 2) {
    // ---------------- epilogue: one thread per token ----------------
    const int sub = warp & 3;  // TMEM lanes 32*sub .. 32*sub+31
    const bool ok = mbar_wait(accbar, 0);
    tc_fence_after();
    const int row = m0 + sub * 32 + lane;
    const uint32_t base = tmem + (uint32_t(sub * 32) << 16);
    // pass 1: the amax of the bf16 K and V rows
    float amax = 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t r[32];
      tmem_ld32(base + c * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(bf16_rounded(__uint_as_float(r[e]))));
    }
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    // pass 2: codes, 32 per chunk (chunks 0-3: K, 4-7: V)
    const bool store = ok && row < T;
    const size_t off = (size_t(row) * Hkv + g) * 128;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      uint32_t r[32];
      tmem_ld32(base + c * 32, r);
      tmem_wait_ld();
      uint32_t w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          word |= e4m3_code(__fdiv_rn(bf16_rounded(__uint_as_float(r[4 * q + b])), s)) << (8 * b);
        w[q] = word;
      }
      if (store) {
        uint4* dst = reinterpret_cast<uint4*>((c < 4 ? Kc : Vc) + off + (c & 3) * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    if (store) scale[size_t(row) * Hkv + g] = s;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}
}  // namespace

cudaError_t launch_bridge(const BridgeArgs& a, cudaStream_t stream) {
  constexpr int BN = 128;
  using C = BridgeCfg<BN>;
  CUtensorMap tmH, tmWk, tmWv;
  // H [T, dm]: x = feature (contiguous), y = token; box 64 x 128
  if (!make_tmap_2d(&tmH, a.H, a.dm, a.T, size_t(a.dm) * 2, 64, BM)) return cudaErrorInvalidValue;
  // W [dm, Nkv]: x = output column (contiguous), y = feature; box 64 x 64
  if (!make_tmap_2d(&tmWk, a.Wk, a.Nkv, a.dm, size_t(a.Nkv) * 2, 64, BK))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tmWv, a.Wv, a.Nkv, a.dm, size_t(a.Nkv) * 2, 64, BK))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(bridge_gemm_kernel<BN>), C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(2 * a.Nkv / BN, (a.T + BM - 1) / BM);
  bridge_gemm_kernel<BN><<<grid, THREADS, C::SMEM, stream>>>(
      tmH, tmWk, tmWv, reinterpret_cast<__nv_bfloat16*>(a.K),
      reinterpret_cast<__nv_bfloat16*>(a.V), int(a.T), a.dm, a.Nkv);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_bridge_fp8(const BridgeFp8Args& a, cudaStream_t stream) {
  CUtensorMap tmH, tmWk, tmWv;
  if (!make_tmap_2d(&tmH, a.H, a.dm, a.T, size_t(a.dm) * 2, 64, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tmWk, a.Wk, a.Nkv, a.dm, size_t(a.Nkv) * 2, 64, BK))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tmWv, a.Wv, a.Nkv, a.dm, size_t(a.Nkv) * 2, 64, BK))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(bridge_fp8_kernel), F_SMEM);
  if (e != cudaSuccess) return e;
  const int Hkv = a.Nkv / 128;
  dim3 grid(Hkv, (a.T + BM - 1) / BM);
  bridge_fp8_kernel<<<grid, THREADS, F_SMEM, stream>>>(tmH, tmWk, tmWv, a.Kc, a.Vc, a.scale,
                                                       int(a.T), a.dm, Hkv);
  count_launch();
  return cudaGetLastError();
}

}  // namespace hs2
