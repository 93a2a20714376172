// kernels.h -- host-side launch interface between the C ABI (hs2_api.cu) and
// the kernels.  Internal to the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hs2 {

// counts every kernel launch of the library (hs2_kernel_launches)
void count_launch(unsigned n = 1);

// sticky device status word of each kernel file: read (and clear)
unsigned status_bridge(bool clear);
unsigned status_full_attn(bool clear);
unsigned status_select(bool clear);
unsigned status_sparse(bool clear);
unsigned status_sparse_union(bool clear);
unsigned status_decode(bool clear);

// spin budget (cycles) of the bounded waits in each kernel file (testing)
cudaError_t budget_bridge(long long cycles);
cudaError_t budget_full_attn(long long cycles);
cudaError_t budget_select(long long cycles);
cudaError_t budget_sparse_union(long long cycles);
cudaError_t budget_decode(long long cycles);

// Tensor maps (bf16, 128-byte swizzle, zero fill out of bounds).
// dims/strides: x fastest; strides in bytes for dims 1.. .
bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t dim_x, uint64_t dim_y,
                  uint64_t stride_y, uint32_t box_x, uint32_t box_y);
bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t dim_x, uint64_t dim_y,
                  uint64_t dim_z, uint64_t stride_y, uint64_t stride_z, uint32_t box_x,
                  uint32_t box_y, uint32_t box_z);

// set the dynamic shared memory limit of a kernel once per device
cudaError_t ensure_smem_attr(const void* func, int bytes);

struct BridgeArgs {
  const void* H;
  const void* Wk;
  const void* Wv;
  void* K;
  void* V;
  int64_t T;
  int dm;
  int Nkv;  // n_kv_heads * 128
};
cudaError_t launch_bridge(const BridgeArgs& a, cudaStream_t stream);

struct BridgeFp8Args {
  const void* H;
  const void* Wk;
  const void* Wv;
  uint8_t* Kc;   // [T, Hkv, 128] e4m3 codes
  uint8_t* Vc;
  float* scale;  // [T, Hkv]
  int64_t T;
  int dm;
  int Nkv;       // n_kv_heads * 128
};
cudaError_t launch_bridge_fp8(const BridgeFp8Args& a, cudaStream_t stream);

struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  float* lse;
  int64_t T;        // rows of Q/O/lse
  int Hq, Hkv;
  float scale;
  int64_t q_begin;  // position of row 0 (a multiple of 128); K/V hold q_begin + T rows
};
cudaError_t launch_full_attn(const AttnArgs& a, cudaStream_t stream);

struct SelectArgs {
  const void* Q;
  const void* K;
  const float* lse;
  int32_t* idx;
  float* kth;
  int64_t T;        // rows of Q/lse/idx/kth
  int Hq, Hkv;
  float scale;
  int k, w;
  void* ws;
  size_t ws_bytes;
  int64_t q_begin;  // position of row 0 (a multiple of 128); K holds q_begin + T rows
};
size_t select_workspace_bytes(int64_t T, int Hq, int Hkv, int k, int w);
cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream);
// same kernel on the library's own file-scope scratch (no workspace argument)
size_t select_noalloc_scratch_bytes();
// fraction of the previous item's smallest k-th score that starts an item's
// floor in hs2_select_topk (<= 0: no speculation); testing hook
void select_set_speculation(float factor);
cudaError_t launch_select_noalloc(const SelectArgs& a, cudaStream_t stream);

// Decode with the context split over ranks: per sequence (row) the slice
// [lo, hi) of its cache that this rank holds.
constexpr int kMaxSpanRows = 64;
struct RowSpans {
  int lo[kMaxSpanRows];
  int hi[kMaxSpanRows];
};

struct SparseArgs {
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* idx;
  void* O;
  float* lse;
  int64_t T;  // query rows
  int Hq, Hkv;
  float scale;
  int kw;     // entries per list (k + w)
  int64_t kv_rows;  // prefill: rows of K/V (list entries must lie below it)
  // FP8 source (decode): codes + per-(token, head) scales; K/V above unused
  const uint8_t* Kc;
  const uint8_t* Vc;
  const float* ks;
  const float* vs;
  int64_t cache_T;  // decode: tokens per sequence in the cache
  RowSpans spans;   // decode: the slice of each sequence's cache to use
  float* rec;       // decode, nullable: write softmax-state records instead of O
};
cudaError_t launch_sparse(const SparseArgs& a, cudaStream_t stream);

// Sparse attention over the union of the lists of P = 256 / G consecutive
// query rows, two 128-row tiles (sparse_union.cu).  A plan covers query
// blocks qb0 .. qb0+nqb-1 (rows qb0*P ..) of every KV head; entry (g, b) =
// g * nqb + b holds uinfo[entry].x union rows at urow/umask[entry * cap ..]
// (ascending positions; bit q of a mask: the row is on the list of query row
// (qb0 + b) * P + q); bit q of uinfo[entry].y: that query's list is not empty.
constexpr int kUnionMaxEntries = 36864;  // most list entries (P * (k + w)) per item
struct UnionPlan {
  int qb0, nqb;
  int64_t cap;
  size_t bytes;
  uint2* uinfo;
  int32_t* urow;
  uint32_t* umask;
};
bool sparse_union_supported(int64_t T, int Hq, int Hkv, int kw, int64_t kv_rows);
// layout of a plan for query rows row0 .. row0 + rows - 1 (row0 a multiple of
// 128) at base (null: sizes only)
UnionPlan union_plan_layout(int64_t T, int Hq, int Hkv, int kw, int64_t row0, int64_t rows,
                            void* base);
// a.idx, a.T, a.Hq, a.Hkv, a.kw, a.kv_rows
cudaError_t launch_sparse_plan(const SparseArgs& a, const UnionPlan& pl, cudaStream_t stream);
// a.Q, a.K, a.V, a.O, a.lse, a.T, a.Hq, a.Hkv, a.scale, a.kv_rows
cudaError_t launch_sparse_union(const SparseArgs& a, const UnionPlan& pl, cudaStream_t stream);

// Fused sparse layers (bf16 K/V): the Q, O and (nullable) lse of each layer
constexpr int kMaxFusedLayers = 3;
struct SparseLayers {
  const void* Q[kMaxFusedLayers];  // bf16 [T, Hq, 128]
  void* O[kMaxFusedLayers];        // bf16 [T, Hq, 128]
  float* lse[kMaxFusedLayers];     // [T, Hq] or null
};
// most layers one fused launch takes for G query heads per KV head (1 = none)
int max_fused_layers(int G);
cudaError_t launch_sparse_fused(const SparseArgs& a, const SparseLayers& lp, int L,
                                cudaStream_t stream);

// One decode step of the block (DEC_FULL), or one part of it when each
// sequence's cache is split over ranks (the DEC_CP_* steps, in this order,
// with an all-gather of the records between consecutive steps).
enum DecodeStep {
  DEC_FULL = 0,
  DEC_CP_ATTN = 1,    // partial attention over the slice -> attn_rec
  DEC_CP_SELECT = 2,  // merge attn_recs -> o, lse; local top k of the slice -> sel_rec
  DEC_CP_SPARSE = 3,  // merge sel_recs -> idx; partial sparse layers -> sparse_rec
  DEC_CP_FINISH = 4   // merge sparse_recs -> o_sparse
};
constexpr int kDecodeRecFloats = 130;  // a softmax-state record: m, l, o[128]
constexpr int kDecodeMergeCap = 8192;  // n_ranks * k records merged per (sequence, KV head)

struct DecodeArgs {
  int step;
  const int64_t* lo_host;  // DEC_CP_*: this rank's slice [lo, hi) of each sequence
  const int64_t* hi_host;
  int n_ranks;
  float* attn_rec;           // [B][Hq][130]
  const float* attn_recs;    // [R][B][Hq][130]
  uint2* sel_rec;            // [B][Hkv][k]
  const uint2* sel_recs;     // [R][B][Hkv][k]
  float* sparse_rec;         // [n_sparse][B][Hq][130]
  const float* sparse_recs;  // [R][n_sparse][B][Hq][130]
  int B;
  const int64_t* seq_len_host;
  const void* q;
  const uint8_t* Kc;
  const uint8_t* Vc;
  const float* ks;
  const float* vs;
  void* o;
  float* lse;
  int32_t* idx;
  int n_sparse;
  const void* const* qs;
  void* const* os;
  int64_t cap;  // tokens per sequence in the cache
  int Hq, Hkv;
  float scale;
  int k, w;
  void* ws;
  size_t ws_bytes;
};
// decode limits, checked on the host before any launch
constexpr int kDecodeMaxBatch = 64;
size_t decode_workspace_bytes(int B, int64_t cap, int Hq, int Hkv, int k, int w);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// read-bandwidth probe (measurement only): `reps` passes of 16-byte loads
cudaError_t launch_read_probe(const void* buf, size_t bytes, int reps, uint32_t* sink,
                              cudaStream_t stream);

}  // namespace hs2
