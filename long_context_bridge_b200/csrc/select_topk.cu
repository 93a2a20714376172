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
//   warp 0     TMA: the item's Q tile once, K tiles into a ring
//   warp 1     TMEM owner; one lane issues S^T = K Q^T (M = 128 keys,
//              N = 128 (query, head) rows) into one of four TMEM buffers
//   warps 2-17 scorers, four per TMEM lane quarter: thread = key (TMEM lane);
//              scorer warp 4s + r takes the s-th quarter of the item's queries
//              (TMEM columns 32s .. 32s + 31) for keys 32r .. 32r + 31.
// Scores: every scorer thread computes, for its key and each of its warp's
// queries, score = sum over the G heads of exp2(s * scale * log2 e - lse2_h)
// in fp32 (pairs of heads per FFMA2, one ex2.approx per head, pairwise adds).
// Candidates only enter the top k if their score reaches the query's floor F.
// Streaming exact top-k without CTA barriers in the tile loop:
//   * every scorer warp appends the candidates of its 32 keys whose score
//     reaches the floor to its own per-query sub-buffer; the four warps of a
//     query's quarter hold disjoint key sets;
//   * every append is also counted in a per-query histogram of score bins
//     (eighths of a binade below the largest possible score G) in shared
//     memory; whatever snapshot of it a warp reads, the highest bin with at
//     least k appended entries at or above it bounds the k-th best score from
//     below, so that bin's lower edge is a valid floor.  One warp owns each
//     query's floor, which only rises; it is refreshed every few tiles;
//   * speculative floor: an item starts from 0.9 of the smallest k-th best
//     score of the CTA's previous item of the same KV head (items run from
//     the latest positions backwards, and earlier queries' k-th best scores
//     are mostly larger).  Under it the histograms are not kept.  A query
//     that ends with fewer than k buffered entries shows the guess was too
//     high; the item is then listed and recomputed without speculation by a
//     second launch, so the result never depends on the guess;
//   * a sub-buffer about to overflow drops its entries below the floor, or,
//     if that is not enough, keeps its own exact k best;
//   * at the end of the item one warp per query selects the k best of the
//     union of the four sub-buffers on the 64-bit key
//     (score bits << 32 | ~position), larger score first and equal scores to
//     the smaller position: the append histogram gives the k-th best's bin
//     (a counting pass rebuilds it if entries were dropped or not counted),
//     one pass takes every entry above that bin and lists the bin's own
//     entries, an exact radix select over that short list settles the rest
//     (over every entry if the list is too long), and the chosen positions
//     are sorted ascending by a bitonic sort held lane-major in registers.
// Items whose every query has at most k candidates skip the scoring: all
// candidates are selected.
#include <cstddef>

#include "common.cuh"
#include "kernels.h"

namespace hs2 {

HS2_STATUS_ACCESSOR(status_select)
HS2_BUDGET_SETTER(budget_select)

namespace {

constexpr int SETS = 4;                      // scorer warp sets (query quarters)
constexpr int SCORER_WARPS = 4 * SETS;       // one warp per (set, TMEM lane quarter)
constexpr int SCORERS = 32 * SCORER_WARPS;
constexpr int THREADS = 64 + SCORERS;        // producer warp, MMA warp, scorers
constexpr int TILE = 128;
constexpr int CHUNK = TILE * 128;
constexpr int TILE_BYTES = 2 * CHUNK;
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int MAX_STAGES = 4;
constexpr int NSB = 4;          // S^T buffers in TMEM (128 columns each)
constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 0);
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kRefresh = 8;         // tiles between floor refreshes (a power of two)
constexpr int kBoundaryCap = 1024;  // boundary-bin entries per final select in scratch
constexpr int kSortWords = 2048 + 2 * kBoundaryCap;  // per-warp sort scratch (32-bit words)

template <int G>
struct SelCfg {
  static constexpr int QT = TILE / G;                 // queries per item
  static constexpr int QH = QT / SETS;                // queries per scorer set (32 columns)
  static constexpr int NB = QT <= 32 ? 256 : 64;      // histogram bins per query
  static constexpr int BSHIFT = QT <= 32 ? 20 : 22;   // bin width: 2^-3 or 2^-1 binade
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[MAX_STAGES], k_empty[MAX_STAGES];
  uint64_t s_full[NSB], s_empty[NSB];
  uint64_t drain;  // the MMA issuer's final commit
  uint32_t tmem_slot;
};

template <int G>
struct Misc {
  static constexpr int QT = SelCfg<G>::QT, NB = SelCfg<G>::NB;
  Bars bars;
  alignas(16) float nlse2[128];  // minus the base-2 lse of the item's 128 (query, head) rows
  uint32_t floor_bits[QT];    // candidates need score bits >= floor_bits (a bin's lower edge)
  uint32_t compacted[QT];     // a sub-buffer of the query dropped entries (hist inexact)
  uint32_t cnt[4][QT];        // entries in each sub-buffer
  alignas(16) uint32_t hist[QT][NB];  // appended entries per score bin
  uint32_t dig[SCORER_WARPS][256];    // per-warp radix histograms
  uint32_t spec_bits;   // speculative floor for the CTA's next item of head spec_g (0: none)
  int32_t spec_g;
  uint32_t spec_min;    // smallest k-th best score (bits) among the item's queries
  uint32_t item_fail;   // a query of the item ended with fewer than k buffered entries
};

// 16-byte vector accesses to the histograms and the lse rows
template <int G>
constexpr bool misc_aligned() {
  return offsetof(Misc<G>, nlse2) % 16 == 0 && offsetof(Misc<G>, hist) % 16 == 0 &&
         sizeof(Misc<G>) % 16 == 0;
}
static_assert(misc_aligned<1>() && misc_aligned<2>() && misc_aligned<4>() && misc_aligned<8>() &&
                  misc_aligned<16>(),
              "shared-memory layout of the selection kernel");

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sdesc_sw128(tile + (ks >> 2) * CHUNK + (ks & 3) * 32, 16, 1024);
}

__device__ __forceinline__ void scorer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(SCORERS) : "memory");
}

// Ranking key: larger is better; equal scores rank the smaller position first.
__device__ __forceinline__ uint64_t sel_key(uint2 v) {
  return (uint64_t(v.x) << 32) | uint64_t(~v.y);
}

template <int NB, int BSHIFT>
__device__ __forceinline__ uint32_t bin_of(uint32_t score_bits, uint32_t lo) {
  const uint32_t bk = score_bits >> BSHIFT;
  return bk >= lo ? min(bk - lo, uint32_t(NB - 1)) : 0u;
}

// Scan bins from the top: the bin where the running count reaches `need`;
// `above` = count in higher bins, `inbin` = its own count.  -1 when the total
// is below `need`.
template <int NB>
__device__ __forceinline__ int hist_cross(const uint32_t* hist, uint32_t need, int lane,
                                          uint32_t& above, uint32_t& inbin) {
  constexpr int PER = NB / 32;
  static_assert(PER == 2 || PER % 4 == 0, "bins per lane");
  // lane l owns bins NB-1-PER*l down to NB-PER*(l+1): one contiguous block,
  // read with vector loads (conflict-free) and taken highest first
  uint32_t c[PER], local = 0;
  const uint32_t* blk = hist + NB - PER * (lane + 1);
  if constexpr (PER == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(blk);
    c[0] = v.y;
    c[1] = v.x;
  } else {
#pragma unroll
    for (int i = 0; i < PER; i += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(blk + i);
      c[PER - 1 - i] = v.x;
      c[PER - 2 - i] = v.y;
      c[PER - 3 - i] = v.z;
      c[PER - 4 - i] = v.w;
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) local += c[i];
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const uint32_t excl = incl - local;
  const uint32_t bal = __ballot_sync(0xffffffffu, excl < need && need <= incl);
  if (bal == 0) {
    above = __shfl_sync(0xffffffffu, incl, 31);
    inbin = 0;
    return -1;
  }
  const int src = __ffs(bal) - 1;
  int bin = 0;
  uint32_t ab = 0, ib = 0;
  if (lane == src) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (cum + c[i] >= need) {
        bin = NB - 1 - PER * lane - i;
        ab = cum;
        ib = c[i];
        break;
      }
      cum += c[i];
    }
  }
  above = __shfl_sync(0xffffffffu, ab, src);
  inbin = __shfl_sync(0xffffffffu, ib, src);
  return __shfl_sync(0xffffffffu, bin, src);
}

// Apply fn(entry, valid) to every entry of up to four lists, eight loads in
// flight per lane.  The lane-to-entry map is the same on every call.
template <class Fn>
__device__ __forceinline__ void for_each_entry(uint2* const* sub, const uint32_t* n, int lane,
                                               Fn fn) {
  for (int w = 0; w < 4; ++w) {
    const uint2* b = sub[w];
    const uint32_t nw = n[w];
    for (uint32_t base = 0; base < nw; base += 256) {
      uint2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t e = base + u * 32 + lane;
        v[u] = e < nw ? b[e] : make_uint2(0u, 0xFFFFFFFFu);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) fn(v[u], base + u * 32 + lane < nw, w);
    }
  }
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

// Exact selection over up to four lists (total >= k): (prefix, mask) such
// that exactly the k entries with (key & mask) >= prefix are the k best.
// Digit 1 is the score bin; when that bin is exact, later digits only look at
// the entries inside it.
template <int NB, int BSHIFT>
__device__ void radix_select(uint2* const* sub, const uint32_t* n, uint32_t k, uint32_t lo,
                             uint32_t* hist, int lane, uint64_t& prefix_out,
                             uint64_t& mask_out) {
  uint64_t prefix = 0, mask = 0;
  uint32_t remaining = k;
  int shift = 56;
  for (int b = lane; b < NB; b += 32) hist[b] = 0;
  __syncwarp();
  for_each_entry(sub, n, lane, [&](uint2 v, bool act, int) {
    if (act) atomicAdd(&hist[bin_of<NB, BSHIFT>(v.x, lo)], 1u);
  });
  __syncwarp();
  {
    uint32_t above, inbin;
    const int b = hist_cross<NB>(hist, remaining, lane, above, inbin);
    __syncwarp();
    if (b > 0 && b < NB - 1) {  // an exact bucket: key bits 63 .. 32+BSHIFT
      prefix = uint64_t(lo + b) << (32 + BSHIFT);
      mask = ~uint64_t(0) << (32 + BSHIFT);
      remaining -= above;
      shift = (inbin == remaining) ? -100 : 32 + BSHIFT - 8;
    }
  }
  for (; shift > -8; shift -= 8) {
    const int sh = shift < 0 ? 0 : shift;
    const uint32_t width = shift < 0 ? 8 + shift : 8;
    const uint64_t dmask = (uint64_t(1) << width) - 1;
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for_each_entry(sub, n, lane, [&](uint2 v, bool act, int) {
      const uint64_t key = sel_key(v);
      if (act && (key & mask) == prefix) atomicAdd(&hist[uint32_t((key >> sh) & dmask)], 1u);
    });
    __syncwarp();
    uint32_t above, inbin;
    const int b = hist_cross<256>(hist, remaining, lane, above, inbin);
    __syncwarp();
    remaining -= above;
    prefix |= uint64_t(b) << sh;
    mask |= dmask << sh;
    if (inbin == remaining) break;
  }
  prefix_out = prefix;
  mask_out = mask;
}

// Ascending bitonic sort of 1024 values held lane-major: v[r] of lane l is
// element 32 l + r.  The 40 stages with strides below 32 compare registers of
// one lane; only the 15 stages with larger strides exchange across lanes.
__device__ __forceinline__ void warp_sort1024_lm(uint32_t (&v)[32], int lane) {
#pragma unroll
  for (int size = 2; size <= 1024; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride < 32) {
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          if (r & stride) continue;
          // element 32 l + r ascends iff bit `size` of its index is clear
          const bool up = size < 32 ? (r & size) == 0 : ((lane << 5) & size) == 0;
          const uint32_t a = v[r], b = v[r + stride];
          v[r] = up ? min(a, b) : max(a, b);
          v[r + stride] = up ? max(a, b) : min(a, b);
        }
      } else {
        const int ls = stride >> 5;
        const bool up = ((lane << 5) & size) == 0;
        const bool lower = (lane & ls) == 0;
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          const uint32_t o = __shfl_xor_sync(0xffffffffu, v[r], ls);
          v[r] = (lower == up) ? min(v[r], o) : max(v[r], o);
        }
      }
    }
  }
}

// Make room in a sub-buffer of n entries: drop the entries below the floor
// fl (stable), or, if that is not enough, keep its own exact k best (they
// contain its part of the top k).  Returns the new count.  Kept out of line:
// it runs rarely and would otherwise bloat the scorers' tile loop.
template <int NB, int BSHIFT>
__device__ __noinline__ uint32_t make_room(uint2* buf, uint32_t n, uint32_t fl, int k, int capw,
                                           uint32_t lo, uint32_t* dig, int lane) {
  __syncwarp();
  n = warp_compact(buf, n, lane, [&](uint2 v) { return v.x >= fl; });
  if (n + 32 > uint32_t(capw) / 2 + k / 2 && n > uint32_t(k)) {
    uint2* one[4] = {buf, buf, buf, buf};
    const uint32_t nn[4] = {n, 0, 0, 0};
    uint64_t pf, mk;
    radix_select<NB, BSHIFT>(one, nn, k, lo, dig, lane, pf, mk);
    n = warp_compact(buf, n, lane, [&](uint2 v) { return (sel_key(v) & mk) >= pf; });
  }
  __syncwarp();
  return n;
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1)
    select_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const float* __restrict__ lse, int32_t* __restrict__ idx,
                  float* __restrict__ kth, uint2* __restrict__ ws, uint32_t* __restrict__ wsort,
                  int T, int Hkv, int k, int w, int capw, int kst, float scale_log2, int q_begin,
                  float spec_factor, const int32_t* __restrict__ item_list,
                  uint32_t* __restrict__ fail_count, int32_t* __restrict__ fail_list) {
  using Cfg = SelCfg<G>;
  constexpr int QT = Cfg::QT, QH = Cfg::QH, NB = Cfg::NB, BSHIFT = Cfg::BSHIFT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_align1024(smem_raw);
  Misc<G>* ms = reinterpret_cast<Misc<G>*>(smem + OFF_K + kst * TILE_BYTES);
  Bars* br = &ms->bars;
  const int warp = warp_id(), lane = lane_id();
  const int Hq = Hkv * G;
  const int nqb = (T + QT - 1) / QT;
  // all items, or (recomputing items whose speculative floor failed) the
  // listed ones, without speculation
  const int n_items = item_list == nullptr
                          ? nqb * Hkv
                          : int(min(*const_cast<volatile uint32_t*>(fail_count), uint32_t(nqb * Hkv)));
  const bool speculate = spec_factor > 0.f && item_list == nullptr;
  // score bins: bucket (bits >> BSHIFT) relative to lo; the top bin holds the
  // largest possible score G, bin 0 everything NB-1 bins and more below it
  const uint32_t top = __float_as_uint(float(G)) >> BSHIFT;
  const uint32_t lo = top - (NB - 1);

  // rows of Q/lse/idx are positions q_begin + row (q_begin a multiple of TILE)
  auto item = [&](int it, int& q0, int& g, int& n_tiles, bool& score) {
    // KV-head-major, heaviest query blocks first within a head, so that the
    // CTAs running at one time stream the same head's K through L2
    if (item_list != nullptr) it = item_list[it];
    const int qb = nqb - 1 - it % nqb;
    g = it / nqb;
    q0 = qb * QT;
    const int q_last = q_begin + min(q0 + QT, T) - 1;  // position of the item's last query
    score = k > 0 && (q_last - w + 1) > k;
    n_tiles = score ? (q_last - w) / TILE + 1 : 0;
  };

  if (threadIdx.x == 0) {
    mbar_init(&br->q_full, 1);
    mbar_init(&br->q_empty, 1);
    for (int s = 0; s < kst; ++s) {
      mbar_init(&br->k_full[s], 1);
      mbar_init(&br->k_empty[s], 1);
    }
    for (int b = 0; b < NSB; ++b) {
      mbar_init(&br->s_full[b], 1);
      mbar_init(&br->s_empty[b], SCORERS);
    }
    mbar_init(&br->drain, 1);
    ms->spec_bits = 0;
    ms->spec_g = -1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&br->tmem_slot, NSB * 128);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = br->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ producer ------------------------------
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      uint32_t kt = 0, qn = 0, q_issued = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        int q0, g, n_tiles;
        bool score;
        item(it, q0, g, n_tiles, score);
        if (!score) continue;
        if (qn > 0 && !mbar_wait(&br->q_empty, (qn - 1) & 1)) { ok = false; break; }
        mbar_arrive_expect_tx(&br->q_full, TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(smem + OFF_Q + c * CHUNK, &tmQ, &br->q_full, c * 64, g * G, q0);
        ++q_issued;
        for (int t = 0; t < n_tiles; ++t, ++kt) {
          const int s = kt % kst;
          if (kt >= uint32_t(kst) && !mbar_wait(&br->k_empty[s], ((kt / kst) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&br->k_full[s], TILE_BYTES);
          for (int c = 0; c < 2; ++c)
            tma_load_3d(smem + OFF_K + s * TILE_BYTES + c * CHUNK, &tmK, &br->k_full[s], c * 64,
                        g, t * TILE);
        }
        ++qn;
      }
      // every issued copy lands before the CTA can exit (kt counts the K
      // tiles issued: a timed-out wait leaves the loop before the increment)
      drain_phase(&br->q_full, q_issued);
      for (int s = 0; s < kst; ++s)
        drain_phase(&br->k_full[s], kt > uint32_t(s) ? (kt - 1 - s) / kst + 1 : 0);
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
        if (!mbar_wait(&br->q_full, qn & 1)) { ok = false; break; }
        for (int t = 0; t < n_tiles; ++t, ++kt, ++st) {
          const int s = kt % kst, b = st % NSB;
          if (!mbar_wait(&br->k_full[s], (kt / kst) & 1)) { ok = false; break; }
          if (st >= NSB && !mbar_wait(&br->s_empty[b], ((st / NSB) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sK = smem_u32(smem + OFF_K + s * TILE_BYTES);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + b * 128, kmajor_desc(sK, ks), kmajor_desc(sQ, ks), IDESC, ks > 0);
          mma_commit(&br->s_full[b]);
          mma_commit(&br->k_empty[s]);
        }
        mma_commit(&br->q_empty);
        ++qn;
      }
      mma_drain(&br->drain);  // no MMA outlives the TMEM
    }
  } else {
    // -------------------------------- scorers -------------------------------
    const int sw = warp - 2;          // scorer warp 0..SCORER_WARPS-1
    const int half = sw >> 2;         // which set (quarter) of the item's queries
    const int sub = warp & 3;         // TMEM lane quarter = key quarter of a tile
    const int tid = threadIdx.x - 64; // 0..SCORERS-1
    const uint32_t lane_addr = uint32_t(sub * 32) << 16;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint2* my_bufs = ws + (size_t(blockIdx.x) * 4 + sub) * QT * capw;  // [QT][capw]
    const uint64_t c2 = f2(scale_log2, scale_log2);
    uint32_t st = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      int q0, g, n_tiles;
      bool score;
      item(it, q0, g, n_tiles, score);
      if (tid < 128) {
        const int qrow = q0 + tid / G;
        ms->nlse2[tid] = qrow < T ? -lse[size_t(qrow) * Hq + g * G + tid % G] * kLog2e : -INFINITY;
      }
      // speculative floor: a fraction of the smallest k-th best score of the
      // CTA's previous item of this head (earlier-processed items lie at
      // later positions, whose k-th best scores are not larger)
      const uint32_t spec = speculate && ms->spec_g == g ? ms->spec_bits : 0u;
      // with a speculative floor the histograms are not kept (the floor is
      // close to the final k-th best already): the final select counts
      for (int i = tid; i < QT; i += SCORERS) {
        ms->floor_bits[i] = spec;
        ms->compacted[i] = spec != 0u;
      }
      for (int i = tid; i < QT * NB; i += SCORERS) (&ms->hist[0][0])[i] = 0;
      const int qb0 = half * QH;        // this warp's queries: qb0 .. qb0 + QH - 1
      const int qvalid = T - q0 - qb0;  // of which those below qvalid exist
      uint2* qbuf = my_bufs + size_t(qb0) * capw;  // query qb0 + qq at qbuf + qq * capw
      // tiles whose every key is a candidate of every query of the set need no
      // per-key test: keys up to q0 + qb0 - w are candidates of query qb0
      const bool all_exist = qvalid >= QH;
      const int last_free = q_begin + q0 + qb0 - w;
      const float* nlw = &ms->nlse2[half * 32];
      uint32_t n[QH], fl[QH];  // appended entries and floors of this warp's queries
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) {
        n[qq] = 0;
        fl[qq] = spec;
      }
      scorer_sync();
      if (tid == 0) {
        ms->spec_min = 0xFFFFFFFFu;
        ms->item_fail = 0;
      }
      for (int t = 0; t < n_tiles; ++t, ++st) {
        const int b = st % NSB;
        ok = ok && mbar_wait(&br->s_full[b], (st / NSB) & 1);
        tc_fence_after();
        const int j = t * TILE + sub * 32 + lane;  // this thread's key
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + b * 128 + half * 32, r);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&br->s_empty[b]);
        // score of each query: sum over its G heads of exp2(s * scale_log2 - lse2)
        float sc[QH];
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) {
          if constexpr (G == 1) {
            sc[qq] = fast_exp2(fmaf(__uint_as_float(r[qq]), scale_log2, nlw[qq]));
          } else {
            uint64_t a2 = 0;
#pragma unroll
            for (int h = 0; h < G; h += 2) {
              const int c = qq * G + h;
              const float2 nl = *reinterpret_cast<const float2*>(nlw + c);
              float y0, y1;
              f2_split(f2_fma(f2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), c2,
                              f2(nl.x, nl.y)),
                       y0, y1);
              const uint64_t e2 = f2(fast_exp2(y0), fast_exp2(y1));
              a2 = h == 0 ? e2 : f2_add(a2, e2);
            }
            float s0, s1;
            f2_split(a2, s0, s1);
            sc[qq] = s0 + s1;
          }
        }
        // candidates at or above the floor go to this warp's sub-buffer of
        // the query, in position order; each append is counted by score bin
        // (groups of up to four queries: their tests and ballots first, one
        // warp-uniform test for a sub-buffer about to overflow, then the
        // appends as predicated stores)
        const bool chk = !all_exist || t * TILE + TILE - 1 > last_free;
        const int dpos = j + w - q_begin - q0 - qb0;  // candidate of query qb0 + qq iff dpos <= qq
        constexpr int QB = QH < 4 ? QH : 4;
#pragma unroll
        for (int q4 = 0; q4 < QH; q4 += QB) {
          bool p[QB];
          uint32_t bal[QB];
          bool full = false;
#pragma unroll
          for (int u = 0; u < QB; ++u) {
            const int qq = q4 + u;
            p[u] = __float_as_uint(sc[qq]) >= fl[qq];
            if (chk) p[u] = p[u] && dpos <= qq && qq < qvalid;
            bal[u] = __ballot_sync(0xffffffffu, p[u]);
            full = full || (bal[u] != 0 && n[qq] + 32 > uint32_t(capw));
          }
          if (full) {
#pragma unroll
            for (int u = 0; u < QB; ++u) {
              const int qq = q4 + u;
              if (bal[u] != 0 && n[qq] + 32 > uint32_t(capw)) {
                n[qq] = make_room<NB, BSHIFT>(qbuf + size_t(qq) * capw, n[qq],
                                              ms->floor_bits[qb0 + qq], k, capw, lo, ms->dig[sw],
                                              lane);
                if (lane == 0) ms->compacted[qb0 + qq] = 1;
              }
            }
          }
#pragma unroll
          for (int u = 0; u < QB; ++u) {
            const int qq = q4 + u;
            if (p[u]) {
              const uint32_t bits = __float_as_uint(sc[qq]);
              qbuf[size_t(qq) * capw + n[qq] + __popc(bal[u] & lt_mask)] =
                  make_uint2(bits, uint32_t(j));
              if (spec == 0u) atomicAdd(&ms->hist[qb0 + qq][bin_of<NB, BSHIFT>(bits, lo)], 1u);
            }
            n[qq] += __popc(bal[u]);
          }
        }
        // raise the floors this warp owns to the highest bin with at least k
        // appended entries at or above it (any snapshot of the counts gives a
        // valid floor), then take up every floor of its queries
        if (spec == 0u && (t & (kRefresh - 1)) == kRefresh - 1) {
          for (int q = half * QH + sub; q < (half + 1) * QH; q += 4) {
            uint32_t above, inbin;
            const int fb = hist_cross<NB>(ms->hist[q], uint32_t(k), lane, above, inbin);
            const uint32_t fbits = fb > 0 ? (uint32_t(fb) + lo) << BSHIFT : 0u;
            if (lane == 0 && fbits > ms->floor_bits[q]) ms->floor_bits[q] = fbits;
          }
          __syncwarp();
#pragma unroll
          for (int qq = 0; qq < QH; ++qq) fl[qq] = ms->floor_bits[qb0 + qq];
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) ms->cnt[sub][qb0 + qq] = n[qq];
      }
      scorer_sync();
      // ---- outputs of the item: one warp per query ----
      uint32_t* sp = wsort + (size_t(blockIdx.x) * SCORER_WARPS + sw) * kSortWords;  // positions
      uint2* bl = reinterpret_cast<uint2*>(sp + 2048);                               // boundary bin
      for (int q = sw; q < QT; q += SCORER_WARPS) {
        const int qrow = q0 + q;
        if (qrow >= T) continue;
        const int qpos = q_begin + qrow;  // its position
        const int ncand = max(0, qpos - w + 1);
        int32_t* out = idx + (size_t(qrow) * Hkv + g) * (k + w);
        float kv = -1.f;
        if (!score || ncand <= k) {
          for (int e = lane; e < k; e += 32) out[e] = e < ncand ? e : -1;
        } else {
          uint2* sb[4];
          uint32_t nbv[4];
          uint32_t total = 0;
          for (int v = 0; v < 4; ++v) {
            sb[v] = ws + ((size_t(blockIdx.x) * 4 + v) * QT + q) * capw;
            nbv[v] = ms->cnt[v][q];
            total += nbv[v];
          }
          // every candidate at or above the floor is buffered, so fewer than k
          // entries means the speculative floor was above the k-th best: the
          // item is recomputed without speculation
          if (total < uint32_t(k) && lane == 0) ms->item_fail = 1;
          // the bin of the k-th best: from the append histogram when every
          // appended entry is still buffered, else from one counting pass
          const uint32_t* hq = ms->hist[q];
          if (ms->compacted[q]) {
            uint32_t* hd = ms->dig[sw];
            for (int b2 = lane; b2 < NB; b2 += 32) hd[b2] = 0;
            __syncwarp();
            for_each_entry(sb, nbv, lane, [&](uint2 v, bool act, int) {
              if (act) atomicAdd(&hd[bin_of<NB, BSHIFT>(v.x, lo)], 1u);
            });
            __syncwarp();
            hq = hd;
          }
          uint32_t above = 0, inbin = 0;
          const int bstar = ok ? hist_cross<NB>(hq, uint32_t(k), lane, above, inbin) : -1;
          __syncwarp();
          uint32_t got = 0, nbl = 0, mn = 0xFFFFFFFFu;
          if (bstar >= 0) {
            const uint32_t need = uint32_t(k) - above;
            const bool all_in = inbin == need;
            // one pass: entries above the boundary bin are selected, the
            // boundary bin's entries go to a list for an exact select
            for (int v = 0; v < 4; ++v) {
              for (uint32_t base = 0; base < nbv[v]; base += 32) {
                const uint32_t e = base + lane;
                uint2 x = make_uint2(0u, 0u);
                int bx = -1;
                if (e < nbv[v]) {
                  x = sb[v][e];
                  bx = int(bin_of<NB, BSHIFT>(x.x, lo));
                }
                const bool sel = bx > bstar || (all_in && bx == bstar);
                const bool tob = !all_in && bx == bstar;
                const uint32_t bs = __ballot_sync(0xffffffffu, sel);
                const uint32_t bb = __ballot_sync(0xffffffffu, tob);
                if (sel) {
                  const uint32_t pos = got + __popc(bs & lt_mask);
                  if (pos < uint32_t(k)) sp[pos] = x.y;
                  mn = min(mn, x.x);
                }
                if (tob) {
                  const uint32_t pos = nbl + __popc(bb & lt_mask);
                  if (pos < uint32_t(kBoundaryCap)) bl[pos] = x;
                }
                got += __popc(bs);
                nbl += __popc(bb);
              }
            }
            __syncwarp();
            if (!all_in && nbl <= uint32_t(kBoundaryCap)) {
              uint2* one[4] = {bl, bl, bl, bl};
              const uint32_t nn[4] = {nbl, 0, 0, 0};
              uint64_t pf, mk;
              radix_select<NB, BSHIFT>(one, nn, need, lo, ms->dig[sw], lane, pf, mk);
              for (uint32_t base = 0; base < nbl; base += 32) {
                const uint32_t e = base + lane;
                uint2 x = make_uint2(0u, 0u);
                bool sel = false;
                if (e < nbl) {
                  x = bl[e];
                  sel = (sel_key(x) & mk) >= pf;
                }
                const uint32_t bs = __ballot_sync(0xffffffffu, sel);
                if (sel) {
                  const uint32_t pos = got + __popc(bs & lt_mask);
                  if (pos < uint32_t(k)) sp[pos] = x.y;
                  mn = min(mn, x.x);
                }
                got += __popc(bs);
              }
            }
          }
          if (bstar < 0 || (!(inbin == uint32_t(k) - above) && nbl > uint32_t(kBoundaryCap))) {
            // fall-back: an exact radix select over every buffered entry
            got = 0;
            mn = 0xFFFFFFFFu;
            uint64_t pf = 0, mk = 0;
            if (ok) radix_select<NB, BSHIFT>(sb, nbv, k, lo, ms->dig[sw], lane, pf, mk);
            for (int v = 0; v < 4; ++v) {
              for (uint32_t base = 0; base < nbv[v]; base += 32) {
                const uint32_t e = base + lane;
                uint2 x = make_uint2(0u, 0u);
                bool sel = false;
                if (e < nbv[v]) {
                  x = sb[v][e];
                  sel = (sel_key(x) & mk) >= pf;
                }
                const uint32_t bs = __ballot_sync(0xffffffffu, sel);
                if (sel) {
                  const uint32_t pos = got + __popc(bs & lt_mask);
                  if (pos < uint32_t(k)) sp[pos] = x.y;
                  mn = min(mn, x.x);
                }
                got += __popc(bs);
              }
            }
          }
          got = min(got, uint32_t(k));
          __syncwarp();
          if (k <= 1024) {
            // lane l sorts elements 32 l .. 32 l + 31 (16-byte loads), the
            // sorted run goes back through the scratch and out coalesced
            uint32_t v[32];
            uint4* spv = reinterpret_cast<uint4*>(sp) + lane * 8;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint4 x = spv[u];
              v[4 * u] = x.x;
              v[4 * u + 1] = x.y;
              v[4 * u + 2] = x.z;
              v[4 * u + 3] = x.w;
            }
#pragma unroll
            for (int r = 0; r < 32; ++r)
              if (lane * 32 + r >= int(got)) v[r] = 0xFFFFFFFFu;
            warp_sort1024_lm(v, lane);
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 8; ++u)
              spv[u] = make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
            __syncwarp();
            for (int e = lane; e < k; e += 32) out[e] = e < int(got) ? int32_t(sp[e]) : -1;
          } else {
            // k in (1024, 2048]: bitonic sort of the staging buffer
            for (int e = got + lane; e < 2048; e += 32) sp[e] = 0xFFFFFFFFu;
            __syncwarp();
            for (int size = 2; size <= 2048; size <<= 1)
              for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int i = lane; i < 1024; i += 32) {
                  const int a0 = 2 * stride * (i / stride) + (i % stride), a1 = a0 + stride;
                  const bool up = (a0 & size) == 0;
                  const uint32_t x0 = sp[a0], x1 = sp[a1];
                  if ((x0 > x1) == up) {
                    sp[a0] = x1;
                    sp[a1] = x0;
                  }
                }
                __syncwarp();
              }
            for (int e = lane; e < k; e += 32) out[e] = e < int(got) ? int32_t(sp[e]) : -1;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          kv = __uint_as_float(mn);
          if (lane == 0 && total >= uint32_t(k)) atomicMin(&ms->spec_min, mn);
          __syncwarp();
        }
        for (int t2 = lane; t2 < w; t2 += 32) {
          const int p = qpos - w + 1 + t2;
          out[k + t2] = p >= 0 ? p : -1;
        }
        if (kth != nullptr && lane == 0) kth[size_t(qrow) * Hkv + g] = kv;
      }
      scorer_sync();
      if (tid == 0 && score && speculate) {
        // only speculative items can fail; each is listed at most once
        if (ms->item_fail) {
          fail_list[atomicAdd(fail_count, 1u)] = it;
          ms->spec_bits = 0;
        } else if (ms->spec_min != 0xFFFFFFFFu) {
          ms->spec_bits = __float_as_uint(__uint_as_float(ms->spec_min) * spec_factor);
          ms->spec_g = g;
        }
      }
      scorer_sync();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NSB * 128);
  }
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int buffer_cap(int k) { return max(2 * k, 256); }

template <int G>
int stages_for() {
  // as many K stages as fit next to Q, the bookkeeping and 1 KB of alignment
  const int fixed = OFF_K + int(sizeof(Misc<G>)) + 1024;
  return min(MAX_STAGES, (227 * 1024 - fixed) / TILE_BYTES);
}

// Fraction of the previous item's smallest k-th best score that starts an
// item's floor (<= 0: no speculation).  Set through a testing hook.
float g_spec_factor = 0.9f;

template <int G>
cudaError_t launch_g(const SelectArgs& a, cudaStream_t stream) {
  constexpr int QT = TILE / G;
  CUtensorMap tmQ, tmK;
  if (!make_tmap_3d(&tmQ, a.Q, 128, a.Hq, a.T, 256, uint64_t(a.Hq) * 256, 64, G, QT))
    return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tmK, a.K, 128, a.Hkv, uint64_t(a.q_begin + a.T), 256,
                    uint64_t(a.Hkv) * 256, 64, 1, TILE))
    return cudaErrorInvalidValue;
  const int kst = stages_for<G>();
  const int smem = OFF_K + kst * TILE_BYTES + int(sizeof(Misc<G>)) + 1024;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_kernel<G>), smem);
  if (e != cudaSuccess) return e;
  const int n_items = int((a.T + QT - 1) / QT) * a.Hkv;
  const int grid = min(sm_count(), n_items);
  uint2* ws = reinterpret_cast<uint2*>(a.ws);
  uint32_t* wsort = reinterpret_cast<uint32_t*>(ws + size_t(sm_count()) * 4 * QT * buffer_cap(a.k));
  // items whose speculative floor failed: a count, then their indices
  uint32_t* fail_count = wsort + size_t(sm_count()) * SCORER_WARPS * kSortWords;
  int32_t* fail_list = reinterpret_cast<int32_t*>(fail_count + 4);
  e = cudaMemsetAsync(fail_count, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  // every item, speculating; then the failed ones again without speculation
  // (a CTA of the second launch exits at once when the list is empty)
  for (int pass = 0; pass < 2; ++pass) {
    select_kernel<G><<<grid, THREADS, smem, stream>>>(
        tmQ, tmK, a.lse, a.idx, a.kth, ws, wsort, int(a.T), a.Hkv, a.k, a.w, buffer_cap(a.k), kst,
        a.scale * kLog2e, int(a.q_begin), pass == 0 ? g_spec_factor : 0.f,
        pass == 0 ? nullptr : fail_list, fail_count, fail_list);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Variant without caller-provided workspace.  Its scratch (the per-query
// candidate sub-buffers and the sort staging of every CTA) is this file-scope
// array; the persistent kernel simply runs as many CTAs as the array can
// hold.  Nothing in it has to start at zero: every word a CTA reads was
// written earlier in the same call.  Each device has its own copy; all calls
// on one device share it, so calls whose kernels overlap on that device (for
// example on two streams) race on it.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(48) << 20;
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

// Device address of g_select_scratch in the current context.  Host code must
// not use the symbol itself as an address.  The lookup runs on every call, so
// a context that was reset and re-created never sees a stale address; the
// first call in a context also loads the module, which is why that call
// should come before any stream capture.
cudaError_t select_scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

// bytes of the file-scope scratch taken by one CTA (the documented figure:
// 4 * (128 / G) * max(2k, 256) * 8 + 262144)
size_t noalloc_cta_bytes(int QT, int k) {
  return size_t(4) * QT * buffer_cap(k) * sizeof(uint2) +
         size_t(SCORER_WARPS) * kSortWords * sizeof(uint32_t);
}
static_assert(size_t(SCORER_WARPS) * kSortWords * sizeof(uint32_t) == 262144,
              "the per-CTA sort term documented for hs2_select_topk_noalloc");

template <int G>
cudaError_t launch_noalloc_g(const SelectArgs& a, void* scratch, cudaStream_t stream) {
  constexpr int QT = TILE / G;
  const int fit = int(kNoAllocScratchBytes / noalloc_cta_bytes(QT, a.k));
  if (fit < 1) return cudaErrorNotSupported;
  CUtensorMap tmQ, tmK;
  if (!make_tmap_3d(&tmQ, a.Q, 128, a.Hq, a.T, 256, uint64_t(a.Hq) * 256, 64, G, QT))
    return cudaErrorInvalidValue;
  if (!make_tmap_3d(&tmK, a.K, 128, a.Hkv, uint64_t(a.q_begin + a.T), 256,
                    uint64_t(a.Hkv) * 256, 64, 1, TILE))
    return cudaErrorInvalidValue;
  const int kst = stages_for<G>();
  const int smem = OFF_K + kst * TILE_BYTES + int(sizeof(Misc<G>)) + 1024;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(select_kernel<G>), smem);
  if (e != cudaSuccess) return e;
  const int n_items = int((a.T + QT - 1) / QT) * a.Hkv;
  const int grid = min(min(sm_count(), n_items), fit);
  uint2* ws = reinterpret_cast<uint2*>(scratch);
  uint32_t* wsort = reinterpret_cast<uint32_t*>(ws + size_t(grid) * 4 * QT * buffer_cap(a.k));
  select_kernel<G><<<grid, THREADS, smem, stream>>>(tmQ, tmK, a.lse, a.idx, a.kth, ws, wsort,
                                                    int(a.T), a.Hkv, a.k, a.w, buffer_cap(a.k),
                                                    kst, a.scale * kLog2e, int(a.q_begin), 0.f,
                                                    nullptr, nullptr, nullptr);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

size_t select_workspace_bytes(int64_t T, int Hq, int Hkv, int k, int w) {
  (void)w;
  const int QT = TILE / (Hq / Hkv);
  const size_t n_items = size_t((T + QT - 1) / QT) * Hkv;
  return size_t(sm_count()) * (size_t(4) * QT * buffer_cap(k) * sizeof(uint2) +
                               size_t(SCORER_WARPS) * kSortWords * sizeof(uint32_t)) +
         16 + n_items * sizeof(int32_t);
}

size_t select_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

void select_set_speculation(float factor) { g_spec_factor = factor; }

cudaError_t launch_select_noalloc(const SelectArgs& a, cudaStream_t stream) {
  void* scratch = nullptr;
  cudaError_t e = select_scratch_address(&scratch);
  if (e != cudaSuccess) return e;
  switch (a.Hq / a.Hkv) {
    case 1: return launch_noalloc_g<1>(a, scratch, stream);
    case 2: return launch_noalloc_g<2>(a, scratch, stream);
    case 4: return launch_noalloc_g<4>(a, scratch, stream);
    case 8: return launch_noalloc_g<8>(a, scratch, stream);
    case 16: return launch_noalloc_g<16>(a, scratch, stream);
    default: return cudaErrorInvalidValue;
  }
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
