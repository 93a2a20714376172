// sparse_union.cu -- sparse attention over the union of neighbouring queries'
// lists, on the 5th-generation tensor cores.
//
// The same operation as sparse_attn.cu (KV Reuse: javabetter.cn explainer
// "mimo-v3-hysparse2", KV Reuse paragraph; aitop.news summary): each sparse
// layer attends with its own queries to the shared K/V at the positions on
// its token list.  The lists of consecutive queries of one KV head overlap
// heavily (the recent windows almost entirely, the top-k sets largely), so
// this path gathers each distinct row once for a group of queries:
//
//   item = P = 256/G consecutive query rows x one KV head = two tcgen05 tiles
//          of 128 (query, head) rows, A (the first 128/G queries) and B.
//
// Plan (sparse_plan_kernel, one CTA per item): the union U of the item's P
// lists, ascending, and per union row a mask of the queries whose list holds
// it.  Positions are marked in a shared-memory bitmap one window of 2^17
// positions at a time; a block scan of the words' bit counts gives every
// position its rank in the union, so the masks (in the plan, zeroed first)
// are set with one atomic per list entry.  The order of a list does not matter; an entry
// outside [-1, kv_rows) or repeated within its list is reported as
// DEV_BAD_INDEX and used at most once.
//
// Attention (sparse_union_kernel): full_attn.cu's structure on gathered
// tiles.  A CTA owns one item; its two Q tiles share every K/V chunk:
//   warp 0     the Q tiles, then K chunk j (128 union rows, gathered four
//              rows per TMA, tile::gather4 with 128 B swizzle) and the
//              chunk's mask tiles into a two-stage ring
//   warp 10    the V chunks into a two-stage ring
//   warp 1     TMEM owner; one lane issues per chunk
//                PV_A(j) S_A(j+1) PV_B(j) S_B(j+1)
//              S = Q K^T over the 128 dims plus one more K step of 16:
//              a one-hot of each row's query within its tile (A side)
//              against the chunk's mask tile for that tile's queries (B side:
//              0 where the query's list holds the union row, -B where it
//              does not, B = 2^e with B * scale * log2 e in [2^13, 2^14)),
//              so a row's base-2 logits of rows not on its list drop by at
//              least 2^13 and their probabilities underflow to exactly 0;
//              P stays in TMEM for PV
//   warps 2-9  softmax of A and of B, one thread per (query, head) row: the
//              online base-2 softmax of full_attn.cu.  Chunks seen before a
//              row's first listed key add finite values (logits within
//              rounding of each other) that the rescale by 2^(-2^13 or less)
//              multiplies by exactly 0.  A row whose list is empty (the plan
//              records which queries have entries) writes O = 0, lse = -inf,
//              as the per-list kernel does.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_sparse_union)
HS2_BUDGET_SETTER(budget_sparse_union)

namespace {

constexpr int TILE = 128;  // union rows per chunk, rows per Q tile

// ----------------------------------------------------------------------------
// plan
// ----------------------------------------------------------------------------
constexpr int PLAN_THREADS = 512;
constexpr int PLAN_WARPS = PLAN_THREADS / 32;
constexpr int kWinWords = 4096;                  // bitmap words per window
constexpr int kWinSpan = kWinWords * 32;         // positions per window
constexpr int kWordsPerThread = kWinWords / PLAN_THREADS;

template <int P>
__global__ void __launch_bounds__(PLAN_THREADS)
    sparse_plan_kernel(const int32_t* __restrict__ idx, int T, int Hkv, int kw, int kv_rows,
                       int nqb, int qb0, int64_t cap, uint2* __restrict__ uinfo,
                       int32_t* __restrict__ urow, uint32_t* __restrict__ umask) {
  static_assert(P % PLAN_WARPS == 0 && P <= 32, "queries per item");
  __shared__ uint32_t bitmap[kWinWords];
  __shared__ uint32_t prefix[kWinWords];
  __shared__ uint32_t wsum[PLAN_WARPS];
  __shared__ int max_pos_s;
  __shared__ uint32_t total_s;
  __shared__ uint32_t qmask_s;  // queries with at least one usable entry
  const int item = blockIdx.x;         // plan entry: (KV head, query block) of this launch
  const int g = item / nqb, qb = qb0 + item % nqb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // warp w takes the lists of queries w, w + 16, ... of the item
  auto list_of = [&](int q) -> const int32_t* {
    const int64_t row = int64_t(qb) * P + q;
    return row < T ? idx + (row * Hkv + g) * kw : nullptr;
  };
  int32_t* out_row = urow + item * cap;
  uint32_t* out_mask = umask + item * cap;

  if (threadIdx.x == 0) {
    max_pos_s = -1;
    qmask_s = 0;
  }
  __syncthreads();
  // the largest listed position (windows past it hold nothing), and which
  // queries have entries
  for (int q = warp; q < P; q += PLAN_WARPS) {
    const int32_t* list = list_of(q);
    if (list == nullptr) continue;
    int mp = -1;
    for (int e = lane; e < kw; e += 32) {
      const int j = list[e];
      if (j >= 0 && j < kv_rows) {
        mp = max(mp, j);
      } else if (j != -1) {
        set_dev_status(DEV_BAD_INDEX);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mp = max(mp, __shfl_xor_sync(0xffffffffu, mp, o));
    if (lane == 0 && mp >= 0) {
      atomicMax(&max_pos_s, mp);
      atomicOr(&qmask_s, 1u << q);
    }
  }
  __syncthreads();
  const int max_pos = max_pos_s;

  uint32_t ubase = 0;
  for (int64_t W0 = 0; W0 <= max_pos; W0 += kWinSpan) {
    for (int i = threadIdx.x; i < kWinWords; i += PLAN_THREADS) bitmap[i] = 0;
    __syncthreads();
    const int64_t W1 = min(W0 + kWinSpan, int64_t(kv_rows));
    for (int q = warp; q < P; q += PLAN_WARPS) {
      const int32_t* list = list_of(q);
      if (list == nullptr) continue;
      for (int e = lane; e < kw; e += 32) {
        const int j = list[e];
        if (j >= W0 && j < W1) atomicOr(&bitmap[(j - W0) >> 5], 1u << (j & 31));
      }
    }
    __syncthreads();
    // exclusive prefix of the words' bit counts; thread t owns a run of words
    const int w0 = threadIdx.x * kWordsPerThread;
    uint32_t c[kWordsPerThread], s = 0;
#pragma unroll
    for (int i = 0; i < kWordsPerThread; ++i) {
      c[i] = __popc(bitmap[w0 + i]);
      s += c[i];
    }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t v = lane < PLAN_WARPS ? wsum[lane] : 0u;
      uint32_t x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += t;
      }
      if (lane < PLAN_WARPS) wsum[lane] = x - v;
      if (lane == 31) total_s = x;
    }
    __syncthreads();
    // the window's union rows, ascending
    uint32_t run = wsum[warp] + incl - s;
#pragma unroll
    for (int i = 0; i < kWordsPerThread; ++i) {
      prefix[w0 + i] = run;
      uint32_t bits = bitmap[w0 + i];
      uint32_t r = ubase + run;
      while (bits != 0u) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        out_row[r++] = int32_t(W0) + (w0 + i) * 32 + b;
      }
      run += c[i];
    }
    __syncthreads();
    const uint32_t total = total_s;
    for (uint32_t i = threadIdx.x; i < total; i += PLAN_THREADS) out_mask[ubase + i] = 0u;
    __syncthreads();
    // each entry's rank in the window's union marks its query there
    for (int q = warp; q < P; q += PLAN_WARPS) {
      const int32_t* list = list_of(q);
      if (list == nullptr) continue;
      for (int e = lane; e < kw; e += 32) {
        const int j = list[e];
        if (j >= W0 && j < W1) {
          const int wd = (j - W0) >> 5;
          const uint32_t r = prefix[wd] + __popc(bitmap[wd] & ((1u << (j & 31)) - 1u));
          const uint32_t old = atomicOr(&out_mask[ubase + r], 1u << q);
          if (old & (1u << q)) set_dev_status(DEV_BAD_INDEX);  // listed twice
        }
      }
    }
    __syncthreads();
    ubase += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) uinfo[item] = make_uint2(ubase, qmask_s);
}

// ----------------------------------------------------------------------------
// attention over the union
// ----------------------------------------------------------------------------
constexpr int THREADS = 352;   // K loader, MMA, two softmax warpgroups, V loader
constexpr int LOADER_V = 10;
constexpr int NST = 2;                     // K / V ring stages
constexpr int CHUNK = TILE * 128;          // bytes of one 64-column half tile
constexpr int TILE_BYTES = 2 * CHUNK;      // 128 rows x 128 dims bf16
constexpr int OFF_Q = 0;                              // Q_A, Q_B
constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;         // NST stages
constexpr int OFF_V = OFF_K + NST * TILE_BYTES;       // NST stages
// NST extra tiles (128 rows x 128 B, swizzled): 16-column blocks 1 and 2 of
// stage s hold the mask tiles of tiles A and B for the chunk in stage s;
// block 0 of stage 0 holds the one-hot of each row's query within its tile
constexpr int OFF_X = OFF_V + NST * TILE_BYTES;
constexpr int OFF_BAR = OFF_X + NST * CHUNK;
constexpr int SMEM = OFF_BAR + 512 + 1024;
static_assert(SMEM <= 232448, "shared memory per CTA");
constexpr uint32_t IDESC_S = idesc_bf16(128, 128, 0, 0);   // Q K^T: both K-major
constexpr uint32_t IDESC_O = idesc_bf16(128, 128, 0, 1);   // P V: V is MN-major
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint16_t kBf16One = 0x3F80;      // 1.0

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2];   // per Q tile
  uint64_t p_full[2];   // per Q tile (128 arrivals)
  uint64_t o_done[2];   // per Q tile (last PV)
  uint64_t drain;       // the MMA issuer's final commit
  uint32_t tmem_slot;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sdesc_sw128(tile + (ks >> 2) * CHUNK + (ks & 3) * 32, 16, 1024);
}

// byte offset of 16-byte chunk cc (0..7) of row r in a 128 B-swizzled tile
__device__ __forceinline__ uint32_t sw128_off(int r, int cc) {
  return uint32_t(r) * 128u + (uint32_t(cc ^ (r & 7)) << 4);
}

// mask tile entries of one union row for the 16 queries of a tile (bits of m)
__device__ __forceinline__ void mask_row16(uint8_t* x_tile, int r, int block, uint32_t m,
                                           uint32_t masked_bits) {
  uint32_t w[8];
#pragma unroll
  for (int c2 = 0; c2 < 8; ++c2) {
    const uint32_t lo = ((m >> (2 * c2)) & 1u) ? 0u : masked_bits;
    const uint32_t hi = ((m >> (2 * c2 + 1)) & 1u) ? 0u : masked_bits;
    w[c2] = lo | (hi << 16);
  }
  *reinterpret_cast<uint4*>(x_tile + sw128_off(r, 2 * block)) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(x_tile + sw128_off(r, 2 * block + 1)) =
      make_uint4(w[4], w[5], w[6], w[7]);
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1)
    sparse_union_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const uint2* __restrict__ uinfo, const int32_t* __restrict__ urow,
                        const uint32_t* __restrict__ umask, int64_t cap,
                        __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int T, int Hkv,
                        int nqb, int qb0, float scale_log2, uint32_t masked_bits) {
  constexpr int QT = TILE / G;   // queries per Q tile
  constexpr int P = 2 * QT;      // queries per item
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  const int warp = warp_id(), lane = lane_id();
  const int lq = nqb - 1 - int(blockIdx.x);  // latest (largest) items first
  const int g = blockIdx.y;
  const int qb = qb0 + lq;
  const int64_t entry = int64_t(g) * nqb + lq;
  const int64_t base = entry * cap;
  const uint2 info = uinfo[entry];
  const int U = int(info.x);
  const uint32_t qmask = info.y;
  // an item with an empty union still runs one chunk (all masked) to write its rows
  const int n = max(1, (U + TILE - 1) / TILE);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int X = 0; X < 2; ++X) {
      mbar_init(&bars->s_full[X], 1);
      mbar_init(&bars->p_full[X], 128);
      mbar_init(&bars->o_done[X], 1);
    }
    mbar_init(&bars->drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_slot, 512);
    tc_fence_before();
  }
  if (warp >= 2 && warp < 6) {
    // one-hot of each row's query within its tile (block 0 of the stage-0 extra tile)
    const int r = threadIdx.x - 64;
    const int qcol = r / G;
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo = (2 * i == qcol) ? kBf16One : 0u;
      const uint32_t hi = (2 * i + 1 == qcol) ? kBf16One : 0u;
      w[i] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(smem + OFF_X + sw128_off(r, 0)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(smem + OFF_X + sw128_off(r, 1)) = make_uint4(w[4], w[5], w[6], w[7]);
    fence_proxy_async_smem();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_slot;

  if (warp == 0 || warp == LOADER_V) {
    // ------------------------------- loaders -------------------------------
    // lane l gathers union rows 4l .. 4l+3 of each chunk (both 64-column
    // halves); the K loader also writes those rows of the chunk's mask tiles.
    // Each lane's positions and masks are loaded one chunk ahead.
    const bool isV = warp == LOADER_V;
    if (!isV && lane == 0) {
      prefetch_tmap(&tmQ);
      mbar_arrive_expect_tx(&bars->q_full, 2 * TILE_BYTES);
      for (int X = 0; X < 2; ++X)
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + OFF_Q + X * TILE_BYTES + c * CHUNK, &tmQ, &bars->q_full, c * 64,
                      g * G, qb * P + X * QT);
    }
    if (lane == 0) prefetch_tmap(isV ? &tmV : &tmK);
    int4 np = make_int4(0, 0, 0, 0);
    uint4 nm = make_uint4(0u, 0u, 0u, 0u);
    auto load_rows = [&](int j) {
      const int u0 = j * TILE + 4 * lane;
      np = *reinterpret_cast<const int4*>(urow + base + u0);
      if (!isV) nm = *reinterpret_cast<const uint4*>(umask + base + u0);
    };
    load_rows(0);
    int issued = 0;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const int s = j % NST;
      int pos[4] = {np.x, np.y, np.z, np.w};
      uint32_t msk[4] = {nm.x, nm.y, nm.z, nm.w};
      if (j + 1 < n) load_rows(j + 1);
      const int u0 = j * TILE + 4 * lane;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (u0 + i >= U) {  // past the union: row 0, masked for every query
          pos[i] = 0;
          msk[i] = 0u;
        }
      }
      uint64_t* full = isV ? &bars->v_full[s] : &bars->k_full[s];
      bool w_ok = true;
      if (lane == 0 && j >= NST)
        w_ok = mbar_wait(isV ? &bars->v_empty[s] : &bars->k_empty[s], ((j / NST) - 1) & 1);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
      if (!isV) {
        uint8_t* x_tile = smem + OFF_X + s * CHUNK;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mask_row16(x_tile, 4 * lane + i, 1, msk[i] & 0xFFFFu, masked_bits);          // tile A
          mask_row16(x_tile, 4 * lane + i, 2, (msk[i] >> QT) & 0xFFFFu, masked_bits);  // tile B
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(full, TILE_BYTES);
      __syncwarp();
      uint8_t* dst = smem + (isV ? OFF_V : OFF_K) + s * TILE_BYTES + (4 * lane) * 128;
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tma_gather4(dst + c * CHUNK, isV ? &tmV : &tmK, full, c * 64, pos[0] * Hkv + g,
                    pos[1] * Hkv + g, pos[2] * Hkv + g, pos[3] * Hkv + g);
      issued = j + 1;
    }
    // every issued copy lands before the CTA can exit
    if (lane == 0) {
      if (!isV) drain_phase(&bars->q_full, 1);
      for (int s = 0; s < NST; ++s)
        drain_phase(isV ? &bars->v_full[s] : &bars->k_full[s],
                    issued > s ? uint32_t((issued - 1 - s) / NST + 1) : 0u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer -----------------------------
      bool ok = mbar_wait(&bars->q_full, 0);
      const uint32_t sX0 = smem_u32(smem + OFF_X);
      auto issue_s = [&](int X, int j) {
        const int s = j % NST;
        const uint32_t sQ = smem_u32(smem + OFF_Q + X * TILE_BYTES);
        const uint32_t sK = smem_u32(smem + OFF_K + s * TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + X * 256, kmajor_desc(sQ, ks), kmajor_desc(sK, ks), IDESC_S, ks > 0);
        // the list masks: one-hot(query) . mask row
        mma_ss(tmem + X * 256, sdesc_sw128(sX0, 16, 1024),
               sdesc_sw128(sX0 + s * CHUNK + 32 * (1 + X), 16, 1024), IDESC_S, 1);
        mma_commit(&bars->s_full[X]);
      };
      auto issue_pv = [&](int X, int j) -> bool {
        if (!mbar_wait(&bars->p_full[X], j & 1)) return false;
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + OFF_V + (j % NST) * TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bd = sdesc_sw128(sV + ks * 16 * 128, CHUNK, 1024);
          mma_ts(tmem + X * 256 + 128, tmem + X * 256 + ks * 8, bd, IDESC_O, (j > 0 || ks > 0));
        }
        if (j == n - 1) mma_commit(&bars->o_done[X]);
        return true;
      };
      if (ok) {
        ok = mbar_wait(&bars->k_full[0], 0);
        tc_fence_after();
        if (ok) {
          issue_s(0, 0);
          issue_s(1, 0);
          mma_commit(&bars->k_empty[0]);
        }
      }
      for (int j = 0; j < n && ok; ++j) {
        const int s = j % NST;
        const bool next = j + 1 < n;
        if (!mbar_wait(&bars->v_full[s], (j / NST) & 1)) { ok = false; break; }
        if (!issue_pv(0, j)) { ok = false; break; }
        if (next) {
          const int s1 = (j + 1) % NST;
          if (!mbar_wait(&bars->k_full[s1], ((j + 1) / NST) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!issue_pv(1, j)) { ok = false; break; }
        mma_commit(&bars->v_empty[s]);
        if (next) {
          issue_s(1, j + 1);
          mma_commit(&bars->k_empty[(j + 1) % NST]);
        }
      }
      mma_drain(&bars->drain);  // no MMA outlives the TMEM
    }
  } else {
    // -------------------------------- softmax -------------------------------
    const int X = (warp - 2) >> 2;
    const int sub = warp & 3;
    const int row = sub * 32 + lane;            // TMEM lane == tile row
    const int qin = X * QT + row / G;           // query within the item
    const int qi = qb * P + qin;                // query row
    const int h = g * G + row % G;              // query head
    const uint32_t lane_addr = uint32_t(sub * 32) << 16;
    const uint32_t tS = tmem + lane_addr + X * 256, tO = tS + 128;
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
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
      float mq[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int e = 4; e < 128; e += 8)
#pragma unroll
        for (int u = 0; u < 4; ++u) mq[u] = fmax3(mq[u], x[e + u], x[e + 4 + u]);
      const float m_new = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * scale_log2;
      float alpha = 1.f;
      const bool raise = m_new > m_use + kRescaleThreshold;
      if (raise) {
        alpha = fast_exp2(m_use - m_new);  // 0 on the first chunk and after masked-only ones
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
    // epilogue: O / l and lse (a row of a query with an empty list: 0, -inf)
    ok = ok && mbar_wait(&bars->o_done[X], 0);
    tc_fence_after();
    const bool empty = ((qmask >> qin) & 1u) == 0u;
    const float inv = empty ? 0.f : 1.f / l;
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
    if (store && lse != nullptr)
      lse[size_t(qi) * (Hkv * G) + h] = empty ? -INFINITY : (m_use + __log2f(l)) * kLn2;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// queries per plan item (two Q tiles)
int union_p(int Hq, int Hkv) { return Hkv > 0 ? 2 * TILE / (Hq / Hkv) : 0; }

// bf16 bits of -B, B = 2^e the power of two with B * scale * log2 e in
// [2^13, 2^14): far enough below every listed logit, near enough that
// masked-only logits stay within rounding of each other after scaling
uint32_t masked_bf16_bits(float scale) {
  int e = 0;
  const double c = double(scale) * 1.4426950408889634;
  while (std::ldexp(c, e) < 8192.0 && e < 126) ++e;
  while (std::ldexp(c, e) >= 16384.0 && e > -126) --e;
  return 0x8000u | (uint32_t(e + 127) << 7);
}

template <int G>
cudaError_t launch_union_g(const SparseArgs& a, const UnionPlan& pl, cudaStream_t stream) {
  constexpr int QT = TILE / G;
  CUtensorMap tmQ, tmK, tmV;
  // Q [T, Hq, 128]: box 64 dims x G heads x QT tokens -> 128 rows of 128 B
  if (!make_tmap_3d(&tmQ, a.Q, 128, a.Hq, a.T, 256, uint64_t(a.Hq) * 256, 64, G, QT))
    return cudaErrorInvalidValue;
  // K, V as [kv_rows * Hkv] rows of 128 dims: box 64 dims x 1 row, gathered
  // four rows at a time
  const uint64_t rows = uint64_t(a.kv_rows) * a.Hkv;
  if (!make_tmap_2d(&tmK, a.K, 128, rows, 256, 64, 1)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tmV, a.V, 128, rows, 256, 64, 1)) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(sparse_union_kernel<G>), SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned(pl.nqb), unsigned(a.Hkv));
  sparse_union_kernel<G><<<grid, THREADS, SMEM, stream>>>(
      tmQ, tmK, tmV, pl.uinfo, pl.urow, pl.umask, pl.cap, reinterpret_cast<__nv_bfloat16*>(a.O),
      a.lse, int(a.T), a.Hkv, pl.nqb, pl.qb0, a.scale * kLog2e, masked_bf16_bits(a.scale));
  count_launch();
  return cudaGetLastError();
}

template <int P>
cudaError_t launch_plan_p(const SparseArgs& a, const UnionPlan& pl, cudaStream_t stream) {
  const unsigned items = unsigned(pl.nqb) * unsigned(a.Hkv);
  sparse_plan_kernel<P><<<items, PLAN_THREADS, 0, stream>>>(
      a.idx, int(a.T), a.Hkv, a.kw, int(a.kv_rows), pl.nqb, pl.qb0, pl.cap, pl.uinfo, pl.urow,
      pl.umask);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool sparse_union_supported(int64_t T, int Hq, int Hkv, int kw, int64_t kv_rows) {
  if (Hkv <= 0 || Hq % Hkv != 0) return false;
  const int G = Hq / Hkv;
  if (G != 8 && G != 16) return false;
  const int P = union_p(Hq, Hkv);
  return kw >= 1 && int64_t(P) * kw <= kUnionMaxEntries && T >= 1 && T <= INT32_MAX &&
         kv_rows >= T && kv_rows * Hkv <= INT32_MAX;
}

UnionPlan union_plan_layout(int64_t T, int Hq, int Hkv, int kw, int64_t row0, int64_t rows,
                            void* base) {
  UnionPlan pl{};
  const int P = union_p(Hq, Hkv);
  pl.qb0 = int(row0 / P);
  pl.nqb = int((rows + P - 1) / P);
  pl.cap = (int64_t(P) * kw + TILE - 1) / TILE * TILE;
  const size_t items = size_t(pl.nqb) * size_t(Hkv);
  const size_t cnt_bytes = (items * 8 + 255) / 256 * 256;
  const size_t arr_bytes = items * size_t(pl.cap) * 4;
  pl.bytes = cnt_bytes + 2 * arr_bytes;
  if (base != nullptr) {
    uint8_t* b = static_cast<uint8_t*>(base);
    pl.uinfo = reinterpret_cast<uint2*>(b);
    pl.urow = reinterpret_cast<int32_t*>(b + cnt_bytes);
    pl.umask = reinterpret_cast<uint32_t*>(b + cnt_bytes + arr_bytes);
  }
  (void)T;
  return pl;
}

cudaError_t launch_sparse_plan(const SparseArgs& a, const UnionPlan& pl, cudaStream_t stream) {
  switch (union_p(a.Hq, a.Hkv)) {
    case 32: return launch_plan_p<32>(a, pl, stream);
    case 16: return launch_plan_p<16>(a, pl, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sparse_union(const SparseArgs& a, const UnionPlan& pl, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 8: return launch_union_g<8>(a, pl, stream);
    case 16: return launch_union_g<16>(a, pl, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hs2
