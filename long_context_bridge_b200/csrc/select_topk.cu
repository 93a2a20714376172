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
//              Passing candidates (score above the query's running threshold)
//              are appended to a per-query buffer in ascending position order
//              (ballot + per-warp counts).  When a buffer may overflow, one
//              warp runs a radix select over the 64-bit key
//              (score bits << 32 | ~j), keeps exactly the k best in place
//              (stable, so positions stay ascending) and raises the threshold.
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
  uint32_t thr[128];        // filter: keep scores with bits > thr
  uint32_t has_thr[128];
  uint32_t wcnt[4][128];    // per-warp pass counts of the current chunk
  uint32_t hist[4][256];    // per-warp radix histograms
};
constexpr int SMEM = OFF_MISC + int(sizeof(Misc)) + 1024;

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sdesc_sw128(tile + (ks >> 2) * CHUNK + (ks & 3) * 32, 16, 1024);
}

__device__ __forceinline__ void scorer_sync() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ uint64_t sel_key(uint2 v) {
  return (uint64_t(v.x) << 32) | uint64_t(~v.y);
}

// Keep the k best of buf[0..n) (n >= k) in place, in their original order.
// Returns the score bits of the selection threshold: every kept entry has
// score bits >= the returned value, and an entry appended later (larger j)
// can only enter the top k if its score bits are greater.
__device__ uint32_t warp_keep_topk(uint2* buf, uint32_t n, uint32_t k, uint32_t* hist,
                                   int lane) {
  uint64_t prefix = 0, mask = 0;
  uint32_t remaining = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (uint32_t e = lane; e < n; e += 32) {
      const uint64_t key = sel_key(buf[e]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l owns bins 255-8l .. 248-8l, highest first
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
    const uint32_t bal = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
    const int src = __ffs(bal) - 1;
    uint32_t bin = 0, above = 0, inbin = 0;
    if (lane == src) {
      uint32_t cum = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (cum + c8[i] >= remaining) {
          bin = 255 - 8 * lane - i;
          above = cum;
          inbin = c8[i];
          break;
        }
        cum += c8[i];
      }
    }
    bin = __shfl_sync(0xffffffffu, bin, src);
    above = __shfl_sync(0xffffffffu, above, src);
    inbin = __shfl_sync(0xffffffffu, inbin, src);
    remaining -= above;
    prefix |= uint64_t(bin) << shift;
    mask |= uint64_t(0xFF) << shift;
    __syncwarp();
    if (inbin == remaining) break;  // the whole bucket is selected
  }
  // stable in-place compaction of the selected entries
  uint32_t out = 0;
  for (uint32_t base = 0; base < n; base += 32) {
    const uint32_t e = base + lane;
    uint2 v = make_uint2(0u, 0u);
    bool sel = false;
    if (e < n) {
      v = buf[e];
      sel = (sel_key(v) & mask) >= prefix;
    }
    const uint32_t b = __ballot_sync(0xffffffffu, sel);
    if (sel) buf[out + __popc(b & ((1u << lane) - 1u))] = v;
    out += __popc(b);
  }
  __syncwarp();
  return uint32_t(prefix >> 32);
}

template <int G>
__global__ void __launch_bounds__(THREADS, 1)
    select_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const float* __restrict__ lse, int32_t* __restrict__ idx,
                  float* __restrict__ kth, uint2* __restrict__ ws, int T, int Hkv, int k, int w,
                  int cap, float scale_log2) {
  constexpr int QT = TILE / G;   // queries per item
  constexpr int QPC = 32 / G;    // queries per 32-column chunk
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
    const int sub = warp & 3;
    const int tid = threadIdx.x - 64;  // 0..127
    const uint32_t lane_addr = uint32_t(sub * 32) << 16;
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
          ms->thr[tid] = 0;
          ms->has_thr[tid] = 0;
        }
      }
      scorer_sync();
      uint2* qbuf0 = ws + size_t(blockIdx.x) * QT * cap;
      for (int t = 0; t < n_tiles; ++t, ++st) {
        const int b = st & 1, par = t & 1;
        ok = ok && mbar_wait(&ms->s_full[b], (st >> 1) & 1);
        tc_fence_after();
        const int j = t * TILE + sub * 32 + lane;  // this thread's key
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_addr + b * 128 + c * 32, r);
          tmem_wait_ld();
          if (c == 3) {
            tc_fence_before();
            mbar_arrive(&ms->s_empty[b]);
          }
          uint32_t bal[QPC];
          float sc[QPC];
#pragma unroll
          for (int qq = 0; qq < QPC; ++qq) {
            float acc = 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h)
              acc += fast_exp2(fmaf(__uint_as_float(r[qq * G + h]), scale_log2,
                                    -ms->lse2[c * 32 + qq * G + h]));
            sc[qq] = acc;
            const int q = c * QPC + qq;
            const int qpos = q0 + q;
            const bool cand = (j + w <= qpos) && qpos < T;
            const uint32_t bits = __float_as_uint(acc);
            const bool pass = cand && (!ms->has_thr[q] || bits > ms->thr[q]);
            bal[qq] = __ballot_sync(0xffffffffu, pass);
            if (lane == 0) ms->wcnt[sub][q] = __popc(bal[qq]);
          }
          scorer_sync();
#pragma unroll
          for (int qq = 0; qq < QPC; ++qq) {
            const int q = c * QPC + qq;
            uint32_t base = ms->tot[par][q];
            for (int v = 0; v < sub; ++v) base += ms->wcnt[v][q];
            if ((bal[qq] >> lane) & 1u) {
              const uint32_t pos = base + __popc(bal[qq] & ((1u << lane) - 1u));
              qbuf0[size_t(q) * cap + pos] = make_uint2(__float_as_uint(sc[qq]), uint32_t(j));
            }
            if (sub == 3 && lane == 0) ms->tot[par ^ 1][q] = base + __popc(bal[qq]);
          }
        }
        scorer_sync();
        // make room: buffers that could overflow on the next tile keep their k best
        for (int q = sub; q < QT; q += 4) {
          const uint32_t n = ms->tot[par ^ 1][q];
          if (n > uint32_t(cap - TILE)) {
            const uint32_t thr = warp_keep_topk(qbuf0 + size_t(q) * cap, n, k, ms->hist[sub], lane);
            if (lane == 0) {
              ms->tot[par ^ 1][q] = k;
              ms->thr[q] = thr;
              ms->has_thr[q] = 1;
            }
          }
        }
        scorer_sync();
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
          if (ok && n > uint32_t(k)) warp_keep_topk(qb, n, k, ms->hist[sub], lane);
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

int buffer_cap(int k) { return 2 * k + 256; }

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
