// full_attn.cu -- causal GQA full attention with per-row log-sum-exp.
//
// The block's full-attention layer (javabetter.cn explainer
// "mimo-v3-hysparse2", Cross-Decoder paragraph).  Its lse is what turns logits
// into the probabilities that rank tokens for the sparse layers (zgeo.com.cn
// page, section 核心技术原理解析).
//
// Layout: a Q tile is 128 "rows" = QT = 128/G consecutive queries x the G
// query heads of one KV head (row r = query q0 + r/G, head g*G + r%G), so the
// K/V tiles streamed through shared memory serve all heads of the group.  A
// CTA owns two consecutive Q tiles, A and B, and ping-pongs between them:
//   warp 0     TMA: both Q tiles once, then K_j / V_j (128 keys x 128 dims,
//              128 B swizzle) into two-stage rings
//   warp 1     TMEM owner; one lane issues, per KV tile j,
//                PV_A(j-1)  S_A(j)  PV_B(j-1)  S_B(j)
//              so the tensor core always has the other tile's work while a
//              softmax runs.  S = Q K^T (M = N = 128, K = 128) lands in TMEM;
//              P is written back over the first 64 columns of its own S and
//              PV reads it from TMEM (A operand in tensor memory).
//   warps 2-5  softmax of tile A, warps 6-9 softmax of tile B: one thread per
//              row (TMEM lane), base-2 online softmax with a lazily raised
//              reference max (O is rescaled only when the row max grows by
//              more than 2^8), scale-and-shift and row sums on packed fp32
//              pairs, P as bf16 into TMEM, epilogue O / l and lse.
// TMEM: S_A [0,128), O_A [128,256), S_B [256,384), O_B [384,512).
#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_full_attn)
HS2_BUDGET_SETTER(budget_full_attn)

namespace {

constexpr int THREADS = 320;               // producer, MMA, two softmax warpgroups
constexpr int TILE = 128;                  // keys per KV tile, rows per Q tile
constexpr int CHUNK = TILE * 128;          // bytes of one 64-column half tile
constexpr int TILE_BYTES = 2 * CHUNK;      // 128 rows x 128 dims bf16
constexpr int OFF_Q = 0;                              // Q_A, Q_B
constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;         // 2 stages
constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;         // 2 stages
constexpr int OFF_BAR = OFF_V + 2 * TILE_BYTES;
constexpr int SMEM = OFF_BAR + 512 + 1024;
constexpr uint32_t IDESC_S = idesc_bf16(128, 128, 0, 0);   // Q K^T: both K-major
constexpr uint32_t IDESC_O = idesc_bf16(128, 128, 0, 1);   // P V: V is MN-major
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];   // per Q tile
  uint64_t p_full[2];   // per Q tile (128 arrivals)
  uint64_t o_done[2];   // per Q tile (last PV)
  uint64_t drain;       // the MMA issuer's final commit
  uint32_t tmem_slot;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  // K-major operand [128 rows][128 K] as two 64-column swizzled halves
  return sdesc_sw128(tile + (ks >> 2) * CHUNK + (ks & 3) * 32, 16, 1024);
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1)
    full_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ O,
                     float* __restrict__ lse, int T, int Hkv, float scale_log2, int q_begin) {
  constexpr int QT = TILE / G;  // queries per Q tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  const int warp = warp_id(), lane = lane_id();
  const int nqb = (T + QT - 1) / QT;
  const int npair = (nqb + 1) / 2;
  const int pr = npair - 1 - int(blockIdx.x);  // heaviest pairs first
  const int g = blockIdx.y;
  int q0[2], n_t[2];
#pragma unroll
  for (int X = 0; X < 2; ++X) {
    // rows of Q/O/lse are positions q_begin + row (q_begin a multiple of
    // TILE), so a Q tile's queries share one diagonal K tile
    q0[X] = (2 * pr + X) * QT;
    n_t[X] = q0[X] < T ? (q_begin + min(q0[X] + QT, T) - 1) / TILE + 1 : 0;
  }
  const int n_max = max(n_t[0], n_t[1]);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 128);
      mbar_init(&bars->o_done[s], 1);
    }
    mbar_init(&bars->drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, 512);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ producer ------------------------------
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int nq = n_t[1] > 0 ? 2 : 1;
      mbar_arrive_expect_tx(&bars->q_full, nq * TILE_BYTES);
      for (int X = 0; X < nq; ++X)
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + OFF_Q + X * TILE_BYTES + c * CHUNK, &tmQ, &bars->q_full, c * 64,
                      g * G, q0[X]);
      int nk = 0, nv = 0;  // K and V tiles issued
      for (int j = 0; j < n_max; ++j) {
        const int s = j & 1;
        const uint32_t ph = ((j >> 1) & 1) ^ 1;
        if (j >= 2 && !mbar_wait(&bars->k_empty[s], ph)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + OFF_K + s * TILE_BYTES + c * CHUNK, &tmK, &bars->k_full[s], c * 64,
                      g, j * TILE);
        nk = j + 1;
        if (j >= 2 && !mbar_wait(&bars->v_empty[s], ph)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + OFF_V + s * TILE_BYTES + c * CHUNK, &tmV, &bars->v_full[s], c * 64,
                      g, j * TILE);
        nv = j + 1;
      }
      // every issued copy lands before the CTA can exit
      drain_phase(&bars->q_full, 1);
      for (int s = 0; s < 2; ++s) {
        drain_phase(&bars->k_full[s], nk > s ? (nk - 1 - s) / 2 + 1 : 0);
        drain_phase(&bars->v_full[s], nv > s ? (nv - 1 - s) / 2 + 1 : 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer -----------------------------
      bool ok = mbar_wait(&bars->q_full, 0);
      auto issue_s = [&](int X, int j) {
        const uint32_t sQ = smem_u32(smem + OFF_Q + X * TILE_BYTES);
        const uint32_t sK = smem_u32(smem + OFF_K + (j & 1) * TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + X * 256, kmajor_desc(sQ, ks), kmajor_desc(sK, ks), IDESC_S, ks > 0);
        mma_commit(&bars->s_full[X]);
      };
      auto issue_pv = [&](int X, int j) -> bool {
        if (!mbar_wait(&bars->p_full[X], j & 1)) return false;
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + OFF_V + (j & 1) * TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // V as the MN-major B operand: K = keys (rows of 128 B), N = dims in
          // two 64-wide chunks CHUNK bytes apart; P from TMEM, 8 columns per
          // 16 keys
          const uint64_t bd = sdesc_sw128(sV + ks * 16 * 128, CHUNK, 1024);
          mma_ts(tmem + X * 256 + 128, tmem + X * 256 + ks * 8, bd, IDESC_O, (j > 0 || ks > 0));
        }
        if (j == n_t[X] - 1) mma_commit(&bars->o_done[X]);
        return true;
      };
      if (ok && n_max > 0) {
        ok = mbar_wait(&bars->k_full[0], 0);
        tc_fence_after();
        if (ok) {
          for (int X = 0; X < 2; ++X)
            if (n_t[X] > 0) issue_s(X, 0);
          mma_commit(&bars->k_empty[0]);
        }
      }
      for (int j = 0; j < n_max && ok; ++j) {
        const int s = j & 1;
        const bool next = j + 1 < n_max;
        if (!mbar_wait(&bars->v_full[s], (j >> 1) & 1)) { ok = false; break; }
        if (j < n_t[0] && !issue_pv(0, j)) { ok = false; break; }
        if (next) {
          if (!mbar_wait(&bars->k_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          if (j + 1 < n_t[0]) issue_s(0, j + 1);
        }
        if (j < n_t[1] && !issue_pv(1, j)) { ok = false; break; }
        mma_commit(&bars->v_empty[s]);
        if (next) {
          if (j + 1 < n_t[1]) issue_s(1, j + 1);
          mma_commit(&bars->k_empty[(j + 1) & 1]);
        }
      }
      mma_drain(&bars->drain);  // no MMA outlives the TMEM
    }
  } else {
    // -------------------------------- softmax -------------------------------
    const int X = (warp - 2) >> 2;             // Q tile of this warpgroup
    const int sub = warp & 3;
    const int row = sub * 32 + lane;            // TMEM lane == tile row
    const int q0X = X ? q0[1] : q0[0];
    const int qi = q0X + row / G;               // this row of Q/O/lse
    const int qpos = q_begin + qi;              // and its position
    const int h = g * G + row % G;              // and head
    const uint32_t lane_addr = uint32_t(sub * 32) << 16;
    const uint32_t tS = tmem + lane_addr + X * 256, tO = tS + 128;
    const int n = X ? n_t[1] : n_t[0];
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      // S_X(j) is complete, and with it every earlier MMA of this tile
      ok = ok && mbar_wait(&bars->s_full[X], j & 1);
      tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]);
      }
      if (j == n - 1) {  // causal mask on the diagonal tile
        const int lim = qpos - j * TILE;  // keys with column > lim are masked
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e > lim) x[e] = -INFINITY;
      }
      float mq[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int e = 4; e < 128; e += 8)
#pragma unroll
        for (int u = 0; u < 4; ++u) mq[u] = fmax3(mq[u], x[e + u], x[e + 4 + u]);
      const float m_new = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * scale_log2;
      float alpha = 1.f;
      const bool raise = m_new > m_use + kRescaleThreshold;
      if (raise) {
        alpha = fast_exp2(m_use - m_new);  // 0 on the first tile
        m_use = m_new;
      }
      const uint64_t sc2 = f2(scale_log2, scale_log2), nm2 = f2(-m_use, -m_use);
      uint64_t sum2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
      uint32_t pk[64];
#pragma unroll
      for (int e = 0; e < 128; e += 2) {
        float a, b, p0, p1;
        f2_split(f2_fma(f2(x[e], x[e + 1]), sc2, nm2), a, b);
        p0 = fast_exp2(a);
        p1 = fast_exp2(b);
        sum2[(e >> 1) & 1] = f2_add(sum2[(e >> 1) & 1], f2(p0, p1));
        pk[e >> 1] = pack_bf16x2(p0, p1);
      }
      float s0, s1, s2, s3;
      f2_split(sum2[0], s0, s1);
      f2_split(sum2[1], s2, s3);
      const float sum = (s0 + s1) + (s2 + s3);
      l = l * alpha + sum;
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tO + c * 32, r);
        }
      }
      // P (bf16 pairs) over the first 64 columns of this tile's S
      uint32_t lo[32], hi[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        lo[e] = pk[e];
        hi[e] = pk[32 + e];
      }
      tmem_st32(tS, lo);
      tmem_st32(tS + 32, hi);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[X]);
    }
    // epilogue: O / l, lse
    if (n > 0) {
      ok = ok && mbar_wait(&bars->o_done[X], 0);
      tc_fence_after();
      const float inv = 1.f / l;
      const bool store = ok && qi < T;
      __nv_bfloat16* dst = O + (size_t(qi) * (Hkv * G) + h) * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]) * inv, __uint_as_float(r[8 * q + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]) * inv, __uint_as_float(r[8 * q + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]) * inv, __uint_as_float(r[8 * q + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]) * inv, __uint_as_float(r[8 * q + 7]) * inv);
            reinterpret_cast<uint4*>(dst + c * 32)[q] = v;
          }
        }
      }
      if (store) lse[size_t(qi) * (Hkv * G) + h] = (m_use + __log2f(l)) * kLn2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int G>
cudaError_t launch_g(const AttnArgs& a, cudaStream_t stream) {
  constexpr int QT = TILE / G;
  CUtensorMap tmQ, tmK, tmV;
  // Q [T, Hq, 128]: box 64 dims x G heads x QT tokens -> 128 rows of 128 B
  if (!make_tmap_3d(&tmQ, a.Q, 128, a.Hq, a.T, 256, uint64_t(a.Hq) * 256, 64, G, QT))
    return cudaErrorInvalidValue;
  // K, V [q_begin + T, Hkv, 128]: box 64 dims x 1 head x 128 tokens
  const uint64_t kv_rows = uint64_t(a.q_begin + a.T);
  if (!make_tmap_3d(&tmK, a.K, 128, a.Hkv, kv_rows, 256, uint64_t(a.Hkv) * 256, 64, 1, TILE))
    return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tmV, a.V, 128, a.Hkv, kv_rows, 256, uint64_t(a.Hkv) * 256, 64, 1, TILE))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(full_attn_kernel<G>), SMEM);
  if (e != cudaSuccess) return e;
  const int nqb = int((a.T + QT - 1) / QT);
  const dim3 grid(unsigned((nqb + 1) / 2), unsigned(a.Hkv));
  full_attn_kernel<G><<<grid, THREADS, SMEM, stream>>>(
      tmQ, tmK, tmV, reinterpret_cast<__nv_bfloat16*>(a.O), a.lse, int(a.T), a.Hkv,
      a.scale * kLog2e, int(a.q_begin));
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_full_attn(const AttnArgs& a, cudaStream_t stream) {
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
