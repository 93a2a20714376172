// select_topk.cu -- token scores, exact top-k and forced recent window.
//
// Token-level selection (javabetter.cn explainer "mimo-v3-hysparse2",
// selection-granularity and local-window paragraphs; siami.tw article section
// 四; the 1024 + 128 entry of the zgeo.com.cn comparison table): for query i
// and KV head g, the candidates j <= i - w are ranked by the full layer's
// attention, score = sum over the group's heads of exp(s - lse); the k best
// (equal scores: smaller j first) are kept, then the w most recent positions.
//
// Persistent kernel, one CTA per SM, work item = (128/G queries, KV head):
//   warp 0     TMA: the item's Q tile once, K tiles into a 4-stage ring
//   warp 1     TMEM owner; one lane issues S^T = K Q^T (M = 128 keys,
//              N = 128 (query, head) rows) into TMEM buffer t%2
//   warps 2-5  scorers: thread = key (TMEM lane); it reads the 128 columns of
//              its key and sums exp2(s*scale*log2e - lse2) over each query's
//              G heads in registers, so a query's score needs no shuffles.
//              A candidate passes when its score bucket (float bits >> 20:
//              eighths of a binade) is at or above the query's floor; passing
//              candidates are appended to a per-query buffer in ascending
//              position order (ballot + per-warp counts), and a reduction
//              barrier lets a tile with no passing candidate skip the append.
//              A buffer about to overflow is trimmed, by one warp, to the
//              buckets that still hold its k best (one histogram pass, one
//              stable compaction) and the floor is raised.  At the end of the
//              item an exact radix select over the 64-bit key
//              (score bits << 32 | ~j) keeps the k best, still in position order.
// Items whose every query has at most k candidates skip the scoring: all
// candidates are selected.
#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_select)

namespace {

constexpr int THREADS = 192;
constexpr int TILE = 128;
constexpr int CHUNK = TILE * 128;
constexpr int TILE_BYTES = 2 * CHUNK;
constexpr int KSTAGES = 4;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int OFF_MISC = OFF_K + KSTAGES * TILE_BYTES;
constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 0);
constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
  uint64_t q_full, q_empty;
  uint64_t k_full[KSTAGES], k_empty[KSTAGES];
  uint64_t s_full[2], s_empty[2];
  uint32_t tmem_slot;
  float lse2[128];          // base-2 lse of the item's 128 (query, head) rows
  uint32_t tot[2][128];     // entries in each query's buffer (by tile parity)
  uint32_t bmin[128];       // filter: keep candidates whose score bucket >= bmin
  uint32_t bseen[128];      // smallest bucket ever appended to each buffer
  uint32_t wcnt[4][128];    // per-warp pass counts of the current tile
  uint32_t hist[4][256];    // per-warp radix histograms
};
constexpr int SMEM = OFF_MISC + int(sizeof(Misc)) + 1024;

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sdesc_sw128(tile + (ks >> 2) * CHUNK + (ks & 3) * 32, 16, 1024);
}

// Named barrier of the 128 scorer threads; returns the OR of `pred` over them.
__device__ __forceinline__ bool scorer_sync_or(bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(pred))
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void scorer_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Score bucket: sign, exponent and 3 mantissa bits of the fp32 score (a
// non-negative float), i.e. eighths of a binade; monotone in the score.
__device__ __forceinline__ uint32_t bucket_of(uint32_t score_bits) { return score_bits >> 20; }

// Ranking key: larger is better; equal scores rank the smaller position first.
__device__ __forceinline__ uint64_t sel_key(uint2 v) {
  return (uint64_t(v.x) << 32) | uint64_t(~v.y);
}

// Warp-aggregated histogram increment (one atomic per distinct bin).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active, int lane) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

// Find, scanning bins from 255 down, the bin where the running count reaches
// `need`.  Returns the bin; `above` = entries in higher bins, `inbin` = its count.
__device__ __forceinline__ uint32_t hist_cross(const uint32_t* hist, uint32_t need, int lane,
                                               uint32_t& above, uint32_t& inbin) {
  uint32_t c8[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c8[i] = hist[255 - 8 * lane - i];
    local += c8[i];
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const uint32_t excl = incl - local;
  const uint32_t bal = __ballot_sync(0xffffffffu, excl < need && need <= incl);
  const int src = bal ? __ffs(bal) - 1 : 31;
  uint32_t bin = 0, ab = 0, ib = 0;
  if (lane == src) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (cum + c8[i] >= need) {
        bin = 255 - 8 * lane - i;
        ab = cum;
        ib = c8[i];
        break;
      }
      cum += c8[i];
    }
  }
  above = __shfl_sync(0xffffffffu, ab, src);
  inbin = __shfl_sync(0xffffffffu, ib, src);
  return __shfl_sync(0xffffffffu, bin, src);
}

__device__ __forceinline__ void hist_clear(uint32_t* hist, int lane) {
  for (int b = lane; b < 256; b += 32) hist[b] = 0;
  __syncwarp();
}

// Stable in-place compaction of buf[0..n): keep entries with keep(v).
template <class Keep>
__device__ __forceinline__ uint32_t warp_compact(uint2* buf, uint32_t n, int lane, Keep keep) {
  uint32_t out = 0;
  for (uint32_t base = 0; base < n; base += 32) {
    const uint32_t e = base + lane;
    uint2 v = make_uint2(0u, 0u);
    bool sel = false;
    if (e < n) {
      v = buf[e];
      sel = keep(v);
    }
    const uint32_t b = __ballot_sync(0xffffffffu, sel);
    if (sel) buf[out + __popc(b & ((1u << lane) - 1u))] = v;
    out += __popc(b);
  }
  __syncwarp();
  return out;
}

// Coarse trim of a full buffer: keep the entries whose bucket is at or above
// the highest bucket that still leaves >= k entries.  All entries have bucket
// >= bmin.  Returns the new bucket floor; n is updated.
__device__ uint32_t warp_trim_buckets(uint2* buf, uint32_t& n, uint32_t k, uint32_t bmin,
                                      uint32_t* hist, int lane) {
  hist_clear(hist, lane);
  for (uint32_t base = 0; base < n; base += 32) {
    const uint32_t e = base + lane;
    uint32_t bin = 0;
    if (e < n) bin = min(bucket_of(buf[e].x) - bmin, 255u);
    hist_add(hist, bin, e < n, lane);
  }
  __syncwarp();
  uint32_t above, inbin;
  const uint32_t b = hist_cross(hist, k, lane, above, inbin);
  const uint32_t floor_b = bmin + b;
  n = warp_compact(buf, n, lane, [&](uint2 v) { return bucket_of(v.x) >= floor_b; });
  return floor_b;
}

// Exact: keep the k best of buf[0..n) (n >= k) in place, in buffer order.
// The first digit is the score bucket relative to bmin (entries all have
// bucket >= bmin), then 8-bit digits of the remaining score and position bits.
__device__ void warp_keep_topk(uint2* buf, uint32_t n, uint32_t k, uint32_t bmin, uint32_t* hist,
                               int lane) {
  uint64_t prefix = 0, mask = 0;
  uint32_t remaining = k;
  int shift;
  // digit 1: bucket (key bits 63..52) relative to bmin
  hist_clear(hist, lane);
  for (uint32_t base = 0; base < n; base += 32) {
    const uint32_t e = base + lane;
    uint32_t bin = 0;
    if (e < n) bin = min(bucket_of(buf[e].x) - bmin, 255u);
    hist_add(hist, bin, e < n, lane);
  }
  __syncwarp();
  {
    uint32_t above, inbin;
    const uint32_t b = hist_cross(hist, remaining, lane, above, inbin);
    __syncwarp();
    if (b < 255) {
      prefix = uint64_t(bmin + b) << 52;
      mask = uint64_t(0xFFF) << 52;
      remaining -= above;
      if (inbin == remaining) goto select;
      shift = 44;
    } else {
      shift = 56;  // the crossing lies 32 binades above bmin: resolve from the top
    }
  }
  for (; shift >= -4; shift -= 8) {
    const int sh = shift < 0 ? 0 : shift;
    const uint64_t dmask = shift < 0 ? 0xFull : 0xFFull;
    hist_clear(hist, lane);
    for (uint32_t base = 0; base < n; base += 32) {
      const uint32_t e = base + lane;
      uint32_t bin = 0;
      bool act = false;
      if (e < n) {
        const uint64_t key = sel_key(buf[e]);
        act = (key & mask) == prefix;
        bin = uint32_t((key >> sh) & dmask);
      }
      hist_add(hist, bin, act, lane);
    }
    __syncwarp();
    uint32_t above, inbin;
    const uint32_t b = hist_cross(hist, remaining, lane, above, inbin);
    __syncwarp();
    remaining -= above;
    prefix |= uint64_t(b) << sh;
    mask |= dmask << sh;
    if (inbin == remaining) break;
  }
select:
  warp_compact(buf, n, lane, [&](uint2 v) { return (sel_key(v) & mask) >= prefix; });
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1)
    select_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const float* __restrict__ lse, int32_t* __restrict__ idx,
                  float* __restrict__ kth, uint2* __restrict__ ws, int T, int Hkv, int k, int w,
                  int cap, float scale_log2) {
  constexpr int QT = TILE / G;   // queries per item
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc* ms = reinterpret_cast<Misc*>(smem + OFF_MISC);
  const int warp = warp_id(), lane = lane_id();
  const int Hq = Hkv * G;
  const int nqb = (T + QT - 1) / QT;
  const int n_items = nqb * Hkv;

  auto item = [&](int it, int& q0, int& g, int& n_tiles, bool& score) {
    const int qb = nqb - 1 - it / Hkv;  // heaviest items first
    g = it % Hkv;
    q0 = qb * QT;
    const int q_last = min(q0 + QT, T) - 1;
    score = k > 0 && (q_last - w + 1) > k;
    n_tiles = score ? (q_last - w) / TILE + 1 : 0;
  };

  if (threadIdx.x == 0) {
    mbar_init(&ms->q_full, 1);
    mbar_init(&ms->q_empty, 1);
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(&ms->k_full[s], 1);
      mbar_init(&ms->k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ms->s_full[b], 1);
      mbar_init(&ms->s_empty[b], 128);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&ms->tmem_slot, 256);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ producer ------------------------------
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      uint32_t kt = 0, qn = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        int q0, g, n_tiles;
        bool score;
        item(it, q0, g, n_tiles, score);
        if (!score) continue;
        if (qn > 0 && !mbar_wait(&ms->q_empty, (qn - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&ms->q_full, TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + OFF_Q + c * CHUNK, &tmQ, &ms->q_full, c * 64, g * G, q0);
        for (int t = 0; t < n_tiles; ++t, ++kt) {
          const int s = kt % KSTAGES;
          if (kt >= KSTAGES && !mbar_wait(&ms->k_empty[s], ((kt / KSTAGES) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ms->k_full[s], TILE_BYTES);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(smem + OFF_K + s * TILE_BYTES + c * CHUNK, &tmK, &ms->k_full[s], c * 64,
                        g, t * TILE);
        }
        ++qn;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer -----------------------------
      const uint32_t sQ = smem_u32(smem + OFF_Q);
      uint32_t kt = 0, st = 0, qn = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        int q0, g, n_tiles;
        bool score;
        item(it, q0, g, n_tiles, score);
        if (!score) continue;
        if (!mbar_wait(&ms->q_full, qn & 1)) { ok = false; break; }
        for (int t = 0; t < n_tiles; ++t, ++kt, ++st) {
          const int s = kt % KSTAGES, b = st & 1;
          if (!mbar_wait(&ms->k_full[s], (kt / KSTAGES) & 1)) { ok = false; break; }
          if (st >= 2 && !mbar_wait(&ms->s_empty[b], ((st >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + OFF_K + s * TILE_BYTES);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + b * 128, kmajor_desc(sK, ks), kmajor_desc(sQ, ks), IDESC, ks > 0);
          mma_commit(&ms->s_full[b]);
          mma_commit(&ms->k_empty[s]);
        }
        mma_commit(&ms->q_empty);
        ++qn;
      }
    }
  } else {
    // -------------------------------- scorers -------------------------------
    // queries scored per group: at least one 32-column chunk, at most 8
    // queries (register budget) unless one chunk holds more
    constexpr int QG = (32 / G > 8) ? 32 / G : (QT < 8 ? QT : 8);
    constexpr int NG = QT / QG;            // groups per tile
    constexpr int CPG = QG * G / 32;       // 32-column chunks per group
    const int sub = warp & 3;
    const int tid = threadIdx.x - 64;  // 0..127
    const uint32_t lane_addr = uint32_t(sub * 32) << 16;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t st = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      int q0, g, n_tiles;
      bool score;
      item(it, q0, g, n_tiles, score);
      {
        const int qrow = q0 + tid / G;
        ms->lse2[tid] = qrow < T ? lse[size_t(qrow) * Hq + g * G + tid % G] * kLog2e : INFINITY;
        if (tid < QT) {
          ms->tot[0][tid] = 0;
          ms->tot[1][tid] = 0;
          ms->bmin[tid] = 0;
          ms->bseen[tid] = 0xFFFFFFFFu;
        }
      }
      scorer_sync();
      uint2* qbuf0 = ws + size_t(blockIdx.x) * QT * cap;
      for (int t = 0; t < n_tiles; ++t, ++st) {
        const int b = st & 1, par = t & 1;
        ok = ok && mbar_wait(&ms->s_full[b], (st >> 1) & 1);
        tc_fence_after();
        const int j = t * TILE + sub * 32 + lane;  // this thread's key
        // every key of the tile is a candidate of every query unless the tile
        // reaches the window of the item's first query
        const bool all_cand = (t + 1) * TILE - 1 + w <= q0;
        bool need = false;  // a buffer this thread counted may overflow next tile
#pragma unroll 1
        for (int gi = 0; gi < NG; ++gi) {
          uint32_t bal[QG];
          float sc[QG];
          bool any_pass = false;
#pragma unroll
          for (int cc = 0; cc < CPG; ++cc) {
            const int c = gi * CPG + cc;  // chunk: columns 32c .. 32c+31
            uint32_t r[32];
            tmem_ld32(tmem + lane_addr + b * 128 + c * 32, r);
            tmem_wait_ld();
            if (gi == NG - 1 && cc == CPG - 1) {
              tc_fence_before();
              mbar_arrive(&ms->s_empty[b]);
            }
#pragma unroll
            for (int qq = 0; qq < 32 / G; ++qq) {
              float acc = 0.f;
#pragma unroll
              for (int h = 0; h < G; ++h)
                acc += fast_exp2(fmaf(__uint_as_float(r[qq * G + h]), scale_log2,
                                      -ms->lse2[c * 32 + qq * G + h]));
              sc[cc * (32 / G) + qq] = acc;
            }
          }
#pragma unroll
          for (int ql = 0; ql < QG; ++ql) {
            const int q = gi * QG + ql;
            const int qpos = q0 + q;
            const bool cand = (all_cand || j + w <= qpos) && qpos < T;
            const bool pass = cand && bucket_of(__float_as_uint(sc[ql])) >= ms->bmin[q];
            bal[ql] = __ballot_sync(0xffffffffu, pass);
            if (lane == 0) ms->wcnt[sub][q] = __popc(bal[ql]);
            any_pass |= bal[ql] != 0;
          }
          // append the passing candidates of this group in ascending position
          if (scorer_sync_or(any_pass)) {
#pragma unroll
            for (int ql = 0; ql < QG; ++ql) {
              const int q = gi * QG + ql;
              if (bal[ql] == 0) continue;
              uint32_t base = ms->tot[par][q];
              for (int v = 0; v < sub; ++v) base += ms->wcnt[v][q];
              if ((bal[ql] >> lane) & 1u) {
                const uint32_t bits = __float_as_uint(sc[ql]);
                qbuf0[size_t(q) * cap + base + __popc(bal[ql] & lt_mask)] =
                    make_uint2(bits, uint32_t(j));
                const uint32_t mb = __reduce_min_sync(bal[ql], bucket_of(bits));
                if (lane == __ffs(bal[ql]) - 1) atomicMin(&ms->bseen[q], mb);
              }
            }
            if (tid < QG) {
              const int q = gi * QG + tid;
              const uint32_t nt =
                  ms->tot[par][q] + ms->wcnt[0][q] + ms->wcnt[1][q] + ms->wcnt[2][q] + ms->wcnt[3][q];
              ms->tot[par ^ 1][q] = nt;
              need |= nt > uint32_t(cap - TILE);
            }
          } else if (tid < QG) {
            ms->tot[par ^ 1][gi * QG + tid] = ms->tot[par][gi * QG + tid];
          }
        }
        // make room: a buffer that could overflow on the next tile is trimmed
        // to the score buckets that still hold its k best
        if (scorer_sync_or(need)) {
          for (int q = sub; q < QT; q += 4) {
            uint32_t n = ms->tot[par ^ 1][q];
            if (n <= uint32_t(cap - TILE)) continue;
            uint2* qb = qbuf0 + size_t(q) * cap;
            const uint32_t base = max(ms->bmin[q], ms->bseen[q]);
            uint32_t bm = warp_trim_buckets(qb, n, k, base, ms->hist[sub], lane);
            if (n > uint32_t(cap + k) / 2) {  // coarse buckets: keep exactly k
              warp_keep_topk(qb, n, k, bm, ms->hist[sub], lane);
              n = k;
            }
            if (lane == 0) {
              ms->tot[par ^ 1][q] = n;
              ms->bmin[q] = bm;
            }
          }
          scorer_sync();
        }
      }
      // ---- outputs of the item ----
      for (int q = sub; q < QT; q += 4) {
        const int qpos = q0 + q;
        if (qpos >= T) continue;
        const int ncand = max(0, qpos - w + 1);
        int32_t* out = idx + (size_t(qpos) * Hkv + g) * (k + w);
        float kv = -1.f;
        if (!score || ncand <= k) {
          for (int e = lane; e < k; e += 32) out[e] = e < ncand ? e : -1;
        } else {
          uint2* qb = qbuf0 + size_t(q) * cap;
          const uint32_t n = ms->tot[n_tiles & 1][q];
          if (ok && n > uint32_t(k))
            warp_keep_topk(qb, n, k, max(ms->bmin[q], ms->bseen[q]), ms->hist[sub], lane);
          uint32_t mn = 0xFFFFFFFFu;
          for (int e = lane; e < k; e += 32) {
            const uint2 v = qb[e];
            out[e] = int32_t(v.y);
            mn = min(mn, v.x);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          kv = __uint_as_float(mn);
        }
        for (int t2 = lane; t2 < w; t2 += 32) {
          const int p = qpos - w + 1 + t2;
          out[k + t2] = p >= 0 ? p : -1;
        }
        if (kth != nullptr && lane == 0) kth[size_t(qpos) * Hkv + g] = kv;
      }
      scorer_sync();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int buffer_cap(int k) { return 4 * k + 256; }

template <int G>
cudaError_t launch_g(const SelectArgs& a, cudaStream_t stream) {
  constexpr int QT = TILE / G;
  CUtensorMap tmQ, tmK;
  if (!make_tmap_3d(&tmQ, a.Q, 128, a.Hq, a.T, 256, uint64_t(a.Hq) * 256, 64, G, QT))
    return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tmK, a.K, 128, a.Hkv, a.T, 256, uint64_t(a.Hkv) * 256, 64, 1, TILE))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_kernel<G>), SMEM);
  if (e != cudaSuccess) return e;
  const int n_items = int((a.T + QT - 1) / QT) * a.Hkv;
  const int grid = min(sm_count(), n_items);
  select_kernel<G><<<grid, THREADS, SMEM, stream>>>(
      tmQ, tmK, a.lse, a.idx, a.kth, reinterpret_cast<uint2*>(a.ws), int(a.T), a.Hkv, a.k, a.w,
      buffer_cap(a.k), a.scale * kLog2e);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

size_t select_workspace_bytes(int64_t T, int Hq, int Hkv, int k, int w) {
  (void)T;
  (void)w;
  const int QT = TILE / (Hq / Hkv);
  return size_t(sm_count()) * QT * buffer_cap(k) * sizeof(uint2);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
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
