// hs2_api.cu -- the C ABI declared in include/hs2.h: host-side argument
// checks, workspace sizing and kernel launches.  Every step of the block runs
// in the kernels of this library; nothing here computes results on the host.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <map>
#include <set>
#include <utility>

#include "../../include/hs2.h"
#include "common.cuh"
#include "kernels.h"

namespace hs2 {

static std::atomic<uint64_t> g_launches{0};
void count_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// ---------------------------------------------------------------------------
// tensor maps through the driver entry point (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static bool encode(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides, const uint32_t* box) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const uint32_t elem[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                  strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t dim_x, uint64_t dim_y,
                  uint64_t stride_y, uint32_t box_x, uint32_t box_y) {
  const uint64_t dims[2] = {dim_x, dim_y};
  const uint64_t strides[1] = {stride_y};
  const uint32_t box[2] = {box_x, box_y};
  return encode(map, base, 2, dims, strides, box);
}

bool make_tmap_3d(CUtensorMap* map, const void* base, uint64_t dim_x, uint64_t dim_y,
                  uint64_t dim_z, uint64_t stride_y, uint64_t stride_z, uint32_t box_x,
                  uint32_t box_y, uint32_t box_z) {
  const uint64_t dims[3] = {dim_x, dim_y, dim_z};
  const uint64_t strides[2] = {stride_y, stride_z};
  const uint32_t box[3] = {box_x, box_y, box_z};
  return encode(map, base, 3, dims, strides, box);
}

cudaError_t ensure_smem_attr(const void* func, int bytes) {
  // the largest size set so far per (kernel, device): raised when a launch
  // needs more (a kernel's dynamic size may depend on its arguments)
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  const auto it = done.find({func, dev});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[{func, dev}] = bytes;
  return e;
}

}  // namespace hs2

using namespace hs2;

// ---------------------------------------------------------------------------
// argument checks
// ---------------------------------------------------------------------------
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hs2_status check_shape(const hs2_shape* s, bool need_select) {
  if (s == nullptr) return HS2_ERR_INVALID_ARG;
  if (s->T <= 0 || s->T > INT32_MAX || s->n_q_heads <= 0 || s->n_kv_heads <= 0)
    return HS2_ERR_INVALID_ARG;
  if (!(s->scale > 0.f) || s->scale != s->scale) return HS2_ERR_INVALID_ARG;
  if (s->head_dim != 128) return HS2_ERR_UNSUPPORTED;
  if (s->n_q_heads % s->n_kv_heads != 0) return HS2_ERR_UNSUPPORTED;
  const int G = s->n_q_heads / s->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return HS2_ERR_UNSUPPORTED;
  if (double(s->T) * s->n_q_heads * 128.0 >= double(1ull << 40)) return HS2_ERR_UNSUPPORTED;
  if (need_select) {
    if (s->k_global < 0 || s->window < 1) return HS2_ERR_INVALID_ARG;
    if (s->k_global > 2048 || s->window > 2048) return HS2_ERR_UNSUPPORTED;
  }
  return HS2_OK;
}

hs2_status cuda_status(cudaError_t e) {
  return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

#define HS2_TRY(expr)                   \
  do {                                  \
    hs2_status st_ = (expr);            \
    if (st_ != HS2_OK) return st_;      \
  } while (0)

#define HS2_NEED(cond)                            \
  do {                                            \
    if (!(cond)) return HS2_ERR_INVALID_ARG;      \
  } while (0)

// The block calls build and use the union plan slab by slab, so that their
// workspace does not grow with T beyond the selection's.
constexpr int64_t kPlanSlabRows = 32768;

bool union_path(const hs2_shape* s, int64_t kv_rows) {
  return sparse_union_supported(s->T, s->n_q_heads, s->n_kv_heads, s->k_global + s->window,
                                kv_rows);
}

size_t block_prefill_bytes(const hs2_shape* s) {
  size_t need = select_workspace_bytes(s->T, s->n_q_heads, s->n_kv_heads, s->k_global, s->window);
  if (union_path(s, s->T)) {
    const UnionPlan pl = union_plan_layout(s->T, s->n_q_heads, s->n_kv_heads,
                                           s->k_global + s->window, 0,
                                           std::min<int64_t>(s->T, kPlanSlabRows), nullptr);
    need = std::max(need, pl.bytes);
  }
  return need;
}

// The sparse layers of a block: over the union plan, slab by slab, where the
// shape allows it; else one list per (row, KV head).
hs2_status block_sparse_layers(const hs2_shape* s, int64_t kv_rows, const hs2_bf16* K,
                               const hs2_bf16* V, const int32_t* idx, int32_t n_sparse,
                               const hs2_bf16* const* Q_sparse, hs2_bf16* const* O_sparse,
                               void* ws, cudaStream_t st) {
  SparseArgs a{};
  a.K = K;
  a.V = V;
  a.idx = idx;
  a.T = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.scale = s->scale;
  a.kw = s->k_global + s->window;
  a.kv_rows = kv_rows;
  if (!union_path(s, kv_rows)) {
    for (int l = 0; l < n_sparse; ++l) {
      a.Q = Q_sparse[l];
      a.O = O_sparse[l];
      HS2_TRY(cuda_status(launch_sparse(a, st)));
    }
    return HS2_OK;
  }
  for (int64_t r0 = 0; r0 < s->T; r0 += kPlanSlabRows) {
    const int64_t rows = std::min(kPlanSlabRows, s->T - r0);
    const UnionPlan pl = union_plan_layout(s->T, a.Hq, a.Hkv, a.kw, r0, rows, ws);
    HS2_TRY(cuda_status(launch_sparse_plan(a, pl, st)));
    for (int l = 0; l < n_sparse; ++l) {
      a.Q = Q_sparse[l];
      a.O = O_sparse[l];
      HS2_TRY(cuda_status(launch_sparse_union(a, pl, st)));
    }
  }
  return HS2_OK;
}


}  // namespace

extern "C" {

const char* hs2_status_string(hs2_status s) {
  switch (s) {
    case HS2_OK: return "ok";
    case HS2_ERR_INVALID_ARG: return "invalid argument";
    case HS2_ERR_UNSUPPORTED: return "unsupported shape";
    case HS2_ERR_WORKSPACE: return "workspace too small";
    case HS2_ERR_CUDA: return "CUDA error";
    case HS2_ERR_TIMEOUT: return "device-side wait timed out";
    case HS2_ERR_BAD_INDEX: return "index list entry out of range (skipped)";
  }
  return "unknown status";
}

uint64_t hs2_kernel_launches(void) { return g_launches.load(); }

hs2_status hs2_get_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return HS2_ERR_CUDA;
  unsigned v = 0;
  v |= status_bridge(true);
  v |= status_full_attn(true);
  v |= status_select(true);
  v |= status_sparse(true);
  v |= status_sparse_union(true);
  v |= status_decode(true);
  if (v == ~0u) return HS2_ERR_CUDA;
  if (v & DEV_TIMEOUT) return HS2_ERR_TIMEOUT;
  if (v & DEV_BAD_INDEX) return HS2_ERR_BAD_INDEX;
  return HS2_OK;
}

hs2_status hs2_debug_read_probe(const void* buf, size_t bytes, int32_t reps, uint32_t* sink,
                                void* stream) {
  HS2_NEED(buf && sink && aligned16(buf) && bytes >= 16 && bytes % 16 == 0 && reps >= 1);
  return cuda_status(launch_read_probe(buf, bytes, reps, sink, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_debug_set_select_speculation(float factor) {
  if (factor != factor) return HS2_ERR_INVALID_ARG;
  select_set_speculation(factor);
  return HS2_OK;
}

hs2_status hs2_debug_set_wait_budget(int64_t cycles) {
  const long long c = cycles > 0 ? static_cast<long long>(cycles) : kWaitBudgetCycles;
  cudaError_t e = budget_bridge(c);
  if (e == cudaSuccess) e = budget_full_attn(c);
  if (e == cudaSuccess) e = budget_select(c);
  if (e == cudaSuccess) e = budget_sparse_union(c);
  if (e == cudaSuccess) e = budget_decode(c);
  return cuda_status(e);
}

size_t hs2_workspace_size(int32_t op, const hs2_shape* s, int32_t batch, int32_t d_model) {
  (void)d_model;
  const bool sel = op == HS2_OP_SELECT || op == HS2_OP_BLOCK_PREFILL ||
                   op == HS2_OP_BLOCK_DECODE || op == HS2_OP_SPARSE_PLAN;
  if (check_shape(s, sel) != HS2_OK) return size_t(-1);
  switch (op) {
    case HS2_OP_BRIDGE:
    case HS2_OP_FULL_ATTN:
    case HS2_OP_SPARSE: return 0;
    case HS2_OP_SELECT:
      return select_workspace_bytes(s->T, s->n_q_heads, s->n_kv_heads, s->k_global, s->window);
    case HS2_OP_BLOCK_PREFILL: return block_prefill_bytes(s);
    case HS2_OP_SPARSE_PLAN:
      if (!union_path(s, s->T)) return size_t(-1);
      return union_plan_layout(s->T, s->n_q_heads, s->n_kv_heads, s->k_global + s->window, 0,
                               s->T, nullptr)
          .bytes;
    case HS2_OP_BLOCK_DECODE:
      if (batch <= 0 || batch > kDecodeMaxBatch || int64_t(batch) * s->T > INT32_MAX)
        return size_t(-1);
      return decode_workspace_bytes(batch, s->T, s->n_q_heads, s->n_kv_heads, s->k_global,
                                    s->window);
  }
  return size_t(-1);
}

hs2_status hs2_bridge_kv(const hs2_bf16* H, int32_t d_model, const hs2_bf16* W_k,
                         const hs2_bf16* W_v, hs2_bf16* K, hs2_bf16* V, const hs2_shape* s,
                         void* stream) {
  HS2_TRY(check_shape(s, false));
  HS2_NEED(H && W_k && W_v && K && V);
  HS2_NEED(aligned16(H) && aligned16(W_k) && aligned16(W_v) && aligned16(K) && aligned16(V));
  HS2_NEED(d_model > 0 && d_model % 64 == 0);
  BridgeArgs a{H, W_k, W_v, K, V, s->T, d_model, s->n_kv_heads * 128};
  return cuda_status(launch_bridge(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_bridge_kv_fp8(const hs2_bf16* H, int32_t d_model, const hs2_bf16* W_k,
                             const hs2_bf16* W_v, hs2_fp8e4m3* Kc, hs2_fp8e4m3* Vc, float* scale,
                             const hs2_shape* s, void* stream) {
  HS2_TRY(check_shape(s, false));
  HS2_NEED(H && W_k && W_v && Kc && Vc && scale);
  HS2_NEED(aligned16(H) && aligned16(W_k) && aligned16(W_v) && aligned16(Kc) && aligned16(Vc) &&
           aligned16(scale));
  HS2_NEED(d_model > 0 && d_model % 64 == 0);
  BridgeFp8Args a{H, W_k, W_v, Kc, Vc, scale, s->T, d_model, s->n_kv_heads * 128};
  return cuda_status(launch_bridge_fp8(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_full_attn_lse(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                             hs2_bf16* O, float* lse, const hs2_shape* s, void* stream) {
  HS2_TRY(check_shape(s, false));
  HS2_NEED(Q && K && V && O && lse);
  HS2_NEED(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O) && aligned16(lse));
  AttnArgs a{Q, K, V, O, lse, s->T, s->n_q_heads, s->n_kv_heads, s->scale};
  return cuda_status(launch_full_attn(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_select_topk(const hs2_bf16* Q, const hs2_bf16* K, const float* lse, int32_t* idx,
                           float* kth, const hs2_shape* s, void* ws, size_t ws_bytes,
                           void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(Q && K && lse && idx);
  HS2_NEED(aligned16(Q) && aligned16(K) && aligned16(lse) && aligned16(idx));
  HS2_NEED(kth == nullptr || aligned16(kth));
  const size_t need =
      select_workspace_bytes(s->T, s->n_q_heads, s->n_kv_heads, s->k_global, s->window);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return HS2_ERR_WORKSPACE;
  SelectArgs a{Q, K, lse, idx, kth, s->T, s->n_q_heads, s->n_kv_heads, s->scale,
               s->k_global, s->window, ws, ws_bytes};
  return cuda_status(launch_select(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_select_topk_noalloc(const hs2_bf16* Q, const hs2_bf16* K, const float* lse,
                                   int32_t* idx, float* kth, const hs2_shape* s, void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(Q && K && lse && idx);
  HS2_NEED(aligned16(Q) && aligned16(K) && aligned16(lse) && aligned16(idx));
  HS2_NEED(kth == nullptr || aligned16(kth));
  SelectArgs a{Q, K, lse, idx, kth, s->T, s->n_q_heads, s->n_kv_heads, s->scale,
               s->k_global, s->window, nullptr, 0};
  const cudaError_t e = launch_select_noalloc(a, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return HS2_ERR_UNSUPPORTED;
  return cuda_status(e);
}

hs2_status hs2_sparse_attn(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                           const int32_t* idx, hs2_bf16* O, float* lse, const hs2_shape* s,
                           void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(Q && K && V && idx && O);
  HS2_NEED(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(idx) && aligned16(O));
  SparseArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.idx = idx;
  a.O = O;
  a.lse = lse;
  a.T = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.scale = s->scale;
  a.kw = s->k_global + s->window;
  return cuda_status(launch_sparse(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_sparse_attn_layers(int32_t n_layers, const hs2_bf16* const* Q,
                                  const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx,
                                  hs2_bf16* const* O, float* const* lse, const hs2_shape* s,
                                  void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(n_layers >= 1 && Q && O && K && V && idx);
  HS2_NEED(aligned16(K) && aligned16(V) && aligned16(idx));
  for (int l = 0; l < n_layers; ++l) {
    HS2_NEED(Q[l] && O[l] && aligned16(Q[l]) && aligned16(O[l]));
    HS2_NEED(lse == nullptr || lse[l] == nullptr || aligned16(lse[l]));
  }
  SparseArgs a{};
  a.K = K;
  a.V = V;
  a.idx = idx;
  a.T = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.scale = s->scale;
  a.kw = s->k_global + s->window;
  const int per = max_fused_layers(s->n_q_heads / s->n_kv_heads);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int l0 = 0; l0 < n_layers;) {
    const int L = std::min(per, n_layers - l0);
    if (L == 1) {
      a.Q = Q[l0];
      a.O = O[l0];
      a.lse = lse ? lse[l0] : nullptr;
      HS2_TRY(cuda_status(launch_sparse(a, st)));
    } else {
      SparseLayers lp{};
      for (int i = 0; i < L; ++i) {
        lp.Q[i] = Q[l0 + i];
        lp.O[i] = O[l0 + i];
        lp.lse[i] = lse ? lse[l0 + i] : nullptr;
      }
      HS2_TRY(cuda_status(launch_sparse_fused(a, lp, L, st)));
    }
    l0 += L;
  }
  return HS2_OK;
}

hs2_status hs2_sparse_plan(const int32_t* idx, const hs2_shape* s, void* plan,
                           size_t plan_bytes, void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(idx && aligned16(idx));
  if (!union_path(s, s->T)) return HS2_ERR_UNSUPPORTED;
  SparseArgs a{};
  a.idx = idx;
  a.T = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.kw = s->k_global + s->window;
  a.kv_rows = s->T;
  const UnionPlan pl = union_plan_layout(s->T, a.Hq, a.Hkv, a.kw, 0, s->T, plan);
  if (plan == nullptr || plan_bytes < pl.bytes || !aligned16(plan)) return HS2_ERR_WORKSPACE;
  return cuda_status(launch_sparse_plan(a, pl, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_sparse_attn_planned(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                                   const void* plan, hs2_bf16* O, float* lse, const hs2_shape* s,
                                   void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(Q && K && V && plan && O);
  HS2_NEED(aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(plan) && aligned16(O));
  if (!union_path(s, s->T)) return HS2_ERR_UNSUPPORTED;
  SparseArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.lse = lse;
  a.T = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.scale = s->scale;
  a.kw = s->k_global + s->window;
  a.kv_rows = s->T;
  const UnionPlan pl = union_plan_layout(s->T, a.Hq, a.Hkv, a.kw, 0, s->T,
                                         const_cast<void*>(plan));
  return cuda_status(launch_sparse_union(a, pl, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_block_prefill(const hs2_bf16* H, int32_t d_model, const hs2_bf16* W_k,
                             const hs2_bf16* W_v, hs2_bf16* K, hs2_bf16* V,
                             const hs2_bf16* Q_full, hs2_bf16* O_full, float* lse, int32_t* idx,
                             int32_t n_sparse, const hs2_bf16* const* Q_sparse,
                             hs2_bf16* const* O_sparse, const hs2_shape* s, void* ws,
                             size_t ws_bytes, void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(n_sparse >= 0 && (n_sparse == 0 || (Q_sparse && O_sparse)));
  for (int l = 0; l < n_sparse; ++l) HS2_NEED(Q_sparse[l] && O_sparse[l]);
  const size_t need = block_prefill_bytes(s);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return HS2_ERR_WORKSPACE;
  for (int l = 0; l < n_sparse; ++l)
    HS2_NEED(aligned16(Q_sparse[l]) && aligned16(O_sparse[l]));
  if (H != nullptr) HS2_TRY(hs2_bridge_kv(H, d_model, W_k, W_v, K, V, s, stream));
  HS2_TRY(hs2_full_attn_lse(Q_full, K, V, O_full, lse, s, stream));
  HS2_TRY(hs2_select_topk(Q_full, K, lse, idx, nullptr, s, ws, ws_bytes, stream));
  return block_sparse_layers(s, s->T, K, V, idx, n_sparse, Q_sparse, O_sparse, ws,
                             static_cast<cudaStream_t>(stream));
}

hs2_status hs2_block_prefill_rows(int64_t q_begin, const hs2_bf16* K, const hs2_bf16* V,
                                  const hs2_bf16* Q_full, hs2_bf16* O_full, float* lse,
                                  int32_t* idx, int32_t n_sparse, const hs2_bf16* const* Q_sparse,
                                  hs2_bf16* const* O_sparse, const hs2_shape* s, void* ws,
                                  size_t ws_bytes, void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(q_begin >= 0);
  if (q_begin % 128 != 0 || q_begin + s->T > INT32_MAX) return HS2_ERR_UNSUPPORTED;
  HS2_NEED(K && V && Q_full && O_full && lse && idx);
  HS2_NEED(aligned16(K) && aligned16(V) && aligned16(Q_full) && aligned16(O_full) &&
           aligned16(lse) && aligned16(idx));
  HS2_NEED(n_sparse >= 0 && (n_sparse == 0 || (Q_sparse && O_sparse)));
  for (int l = 0; l < n_sparse; ++l)
    HS2_NEED(Q_sparse[l] && O_sparse[l] && aligned16(Q_sparse[l]) && aligned16(O_sparse[l]));
  size_t need = select_workspace_bytes(s->T, s->n_q_heads, s->n_kv_heads, s->k_global, s->window);
  if (union_path(s, q_begin + s->T))
    need = std::max(need, union_plan_layout(s->T, s->n_q_heads, s->n_kv_heads,
                                            s->k_global + s->window, 0,
                                            std::min<int64_t>(s->T, kPlanSlabRows), nullptr)
                              .bytes);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return HS2_ERR_WORKSPACE;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  AttnArgs fa{Q_full, K, V, O_full, lse, s->T, s->n_q_heads, s->n_kv_heads, s->scale, q_begin};
  HS2_TRY(cuda_status(launch_full_attn(fa, st)));
  SelectArgs sa{Q_full, K, lse, idx, nullptr, s->T, s->n_q_heads, s->n_kv_heads, s->scale,
                s->k_global, s->window, ws, ws_bytes, q_begin};
  HS2_TRY(cuda_status(launch_select(sa, st)));
  return block_sparse_layers(s, q_begin + s->T, K, V, idx, n_sparse, Q_sparse, O_sparse, ws, st);
}

hs2_status hs2_block_decode(int32_t batch, const int64_t* seq_len, const hs2_bf16* q_full,
                            const hs2_fp8e4m3* Kc, const hs2_fp8e4m3* Vc, const float* k_scale,
                            const float* v_scale, hs2_bf16* o_full, float* lse, int32_t* idx,
                            int32_t n_sparse, const hs2_bf16* const* q_sparse,
                            hs2_bf16* const* o_sparse, const hs2_shape* s, void* ws,
                            size_t ws_bytes, void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(batch > 0 && seq_len && q_full && Kc && Vc && k_scale && v_scale && o_full && lse &&
           idx);
  HS2_NEED(aligned16(q_full) && aligned16(Kc) && aligned16(Vc) && aligned16(o_full) &&
           aligned16(lse) && aligned16(idx));
  HS2_NEED((reinterpret_cast<uintptr_t>(k_scale) & 3) == 0 &&
           (reinterpret_cast<uintptr_t>(v_scale) & 3) == 0);
  if (batch > kDecodeMaxBatch || int64_t(batch) * s->T > INT32_MAX) return HS2_ERR_UNSUPPORTED;
  for (int b = 0; b < batch; ++b) HS2_NEED(seq_len[b] >= 1 && seq_len[b] <= s->T);
  HS2_NEED(n_sparse >= 0 && (n_sparse == 0 || (q_sparse && o_sparse)));
  for (int l = 0; l < n_sparse; ++l)
    HS2_NEED(q_sparse[l] && o_sparse[l] && aligned16(q_sparse[l]) && aligned16(o_sparse[l]));
  const size_t need = decode_workspace_bytes(batch, s->T, s->n_q_heads, s->n_kv_heads,
                                             s->k_global, s->window);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return HS2_ERR_WORKSPACE;
  DecodeArgs a{};
  a.B = batch;
  a.seq_len_host = seq_len;
  a.q = q_full;
  a.Kc = Kc;
  a.Vc = Vc;
  a.ks = k_scale;
  a.vs = v_scale;
  a.o = o_full;
  a.lse = lse;
  a.idx = idx;
  a.n_sparse = n_sparse;
  a.qs = reinterpret_cast<const void* const*>(q_sparse);
  a.os = reinterpret_cast<void* const*>(o_sparse);
  a.cap = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.scale = s->scale;
  a.k = s->k_global;
  a.w = s->window;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return cuda_status(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// decode with each sequence's cache split over ranks
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

// checks shared by the context-parallel decode steps: shape, batch, lengths
// and each sequence's slice [lo, hi) of its cache on this rank
hs2_status check_cp(int32_t batch, const int64_t* seq_len, const int64_t* lo, const int64_t* hi,
                    const hs2_shape* s) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(batch > 0 && seq_len);
  if (batch > kDecodeMaxBatch || int64_t(batch) * s->T > INT32_MAX) return HS2_ERR_UNSUPPORTED;
  for (int b = 0; b < batch; ++b) {
    HS2_NEED(seq_len[b] >= 1 && seq_len[b] <= INT32_MAX);
    if (lo != nullptr || hi != nullptr) {
      HS2_NEED(lo && hi && lo[b] >= 0 && lo[b] <= hi[b] && hi[b] <= seq_len[b]);
      HS2_NEED(hi[b] - lo[b] <= s->T);
    }
  }
  return HS2_OK;
}

hs2_status check_ranks(int32_t n_ranks, const hs2_shape* s) {
  HS2_NEED(n_ranks >= 1);
  if (int64_t(n_ranks) * s->k_global > kDecodeMergeCap) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

DecodeArgs cp_args(int step, int32_t batch, const int64_t* seq_len, const int64_t* lo,
                   const int64_t* hi, const hs2_shape* s) {
  DecodeArgs a{};
  a.step = step;
  a.B = batch;
  a.seq_len_host = seq_len;
  a.lo_host = lo;
  a.hi_host = hi;
  a.cap = s->T;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.scale = s->scale;
  a.k = s->k_global;
  a.w = s->window;
  return a;
}

bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

}  // namespace

extern "C" {

hs2_status hs2_decode_cp_attn(int32_t batch, const int64_t* seq_len, const int64_t* slice_lo,
                              const int64_t* slice_hi, const hs2_bf16* q_full,
                              const hs2_fp8e4m3* Kc, const hs2_fp8e4m3* Vc, const float* k_scale,
                              const float* v_scale, float* attn_rec, const hs2_shape* s,
                              void* ws, size_t ws_bytes, void* stream) {
  HS2_NEED(slice_lo && slice_hi);
  HS2_TRY(check_cp(batch, seq_len, slice_lo, slice_hi, s));
  HS2_NEED(q_full && Kc && Vc && k_scale && v_scale && attn_rec);
  HS2_NEED(aligned16(q_full) && aligned16(Kc) && aligned16(Vc) && aligned16(attn_rec));
  HS2_NEED((reinterpret_cast<uintptr_t>(k_scale) & 3) == 0 &&
           (reinterpret_cast<uintptr_t>(v_scale) & 3) == 0);
  const size_t need = decode_workspace_bytes(batch, s->T, s->n_q_heads, s->n_kv_heads,
                                             s->k_global, s->window);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return HS2_ERR_WORKSPACE;
  DecodeArgs a = cp_args(DEC_CP_ATTN, batch, seq_len, slice_lo, slice_hi, s);
  a.q = q_full;
  a.Kc = Kc;
  a.Vc = Vc;
  a.ks = k_scale;
  a.vs = v_scale;
  a.attn_rec = attn_rec;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return cuda_status(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_decode_cp_select(int32_t batch, const int64_t* seq_len, const int64_t* slice_lo,
                                const int64_t* slice_hi, int32_t n_ranks, const float* attn_recs,
                                hs2_bf16* o_full, float* lse, uint32_t* sel_rec,
                                const hs2_shape* s, void* ws, size_t ws_bytes, void* stream) {
  HS2_NEED(slice_lo && slice_hi);
  HS2_TRY(check_cp(batch, seq_len, slice_lo, slice_hi, s));
  HS2_TRY(check_ranks(n_ranks, s));
  HS2_NEED(attn_recs && o_full && lse && sel_rec);
  HS2_NEED(aligned16(attn_recs) && aligned16(o_full) && aligned16(lse) && aligned16(sel_rec));
  const size_t need = decode_workspace_bytes(batch, s->T, s->n_q_heads, s->n_kv_heads,
                                             s->k_global, s->window);
  if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return HS2_ERR_WORKSPACE;
  DecodeArgs a = cp_args(DEC_CP_SELECT, batch, seq_len, slice_lo, slice_hi, s);
  a.n_ranks = n_ranks;
  a.attn_recs = attn_recs;
  a.o = o_full;
  a.lse = lse;
  a.sel_rec = reinterpret_cast<uint2*>(sel_rec);
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return cuda_status(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_decode_cp_sparse(int32_t batch, const int64_t* seq_len, const int64_t* slice_lo,
                                const int64_t* slice_hi, int32_t n_ranks,
                                const uint32_t* sel_recs, int32_t* idx, const hs2_fp8e4m3* Kc,
                                const hs2_fp8e4m3* Vc, const float* k_scale,
                                const float* v_scale, int32_t n_sparse,
                                const hs2_bf16* const* q_sparse, float* sparse_rec,
                                const hs2_shape* s, void* stream) {
  HS2_NEED(slice_lo && slice_hi);
  HS2_TRY(check_cp(batch, seq_len, slice_lo, slice_hi, s));
  HS2_TRY(check_ranks(n_ranks, s));
  HS2_NEED(sel_recs && idx && Kc && Vc && k_scale && v_scale);
  HS2_NEED(aligned8(sel_recs) && aligned16(idx) && aligned16(Kc) && aligned16(Vc));
  HS2_NEED((reinterpret_cast<uintptr_t>(k_scale) & 3) == 0 &&
           (reinterpret_cast<uintptr_t>(v_scale) & 3) == 0);
  HS2_NEED(n_sparse >= 0 && (n_sparse == 0 || (q_sparse && sparse_rec && aligned16(sparse_rec))));
  for (int l = 0; l < n_sparse; ++l) HS2_NEED(q_sparse[l] && aligned16(q_sparse[l]));
  DecodeArgs a = cp_args(DEC_CP_SPARSE, batch, seq_len, slice_lo, slice_hi, s);
  a.n_ranks = n_ranks;
  a.sel_recs = reinterpret_cast<const uint2*>(sel_recs);
  a.idx = idx;
  a.Kc = Kc;
  a.Vc = Vc;
  a.ks = k_scale;
  a.vs = v_scale;
  a.n_sparse = n_sparse;
  a.qs = reinterpret_cast<const void* const*>(q_sparse);
  a.sparse_rec = sparse_rec;
  return cuda_status(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

hs2_status hs2_decode_cp_finish(int32_t batch, int32_t n_ranks, int32_t n_sparse,
                                const float* sparse_recs, hs2_bf16* const* o_sparse,
                                const hs2_shape* s, void* stream) {
  HS2_TRY(check_shape(s, true));
  HS2_NEED(batch > 0);
  if (batch > kDecodeMaxBatch) return HS2_ERR_UNSUPPORTED;
  HS2_TRY(check_ranks(n_ranks, s));
  HS2_NEED(n_sparse >= 1 && sparse_recs && o_sparse && aligned16(sparse_recs));
  for (int l = 0; l < n_sparse; ++l) HS2_NEED(o_sparse[l] && aligned16(o_sparse[l]));
  DecodeArgs a{};
  a.step = DEC_CP_FINISH;
  a.B = batch;
  a.Hq = s->n_q_heads;
  a.Hkv = s->n_kv_heads;
  a.k = s->k_global;
  a.cap = s->T;
  a.n_ranks = n_ranks;
  a.n_sparse = n_sparse;
  a.sparse_recs = sparse_recs;
  a.os = reinterpret_cast<void* const*>(o_sparse);
  static const int64_t one = 1;
  int64_t lens[kDecodeMaxBatch];
  for (int b = 0; b < batch; ++b) lens[b] = one;
  a.seq_len_host = lens;
  return cuda_status(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
