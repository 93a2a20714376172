/*
 * hs2.h -- C ABI of the B200 (sm_100a) HySparse2 cross-decoder block library.
 *
 * HySparse2 ("Hybrid Sparse Attention with Two-Level KV Sharing") splits a
 * model into a self-decoder and a cross-decoder.  Each cross-decoder block is
 * one full-attention layer followed by several sparse-attention layers.  The
 * block's K/V come from self-decoder hidden states (KV Bridging); the sparse
 * layers reuse that K/V cache and the full layer's token list (KV Reuse).  The
 * list holds, per query token, the 1024 earlier tokens the full layer's
 * attention scores rank highest plus a forced window of the 128 most recent.
 * Sources: javabetter.cn explainer "mimo-v3-hysparse2" (Cross-Decoder, KV Reuse,
 * KV Bridging, selection-granularity and local-window paragraphs); siami.tw
 * "小米 MiMo-V3 全新架構亮相：HySparse 2 把 1M Token 預填成本砍到 1/5",
 * sections 一 and 四; zgeo.com.cn "小米MiMo-V3架构剧透：HySparse2稀疏注意力…",
 * section 核心技术原理解析 and its comparison table; aitop.news "Xiaomi MiMo-V3
 * to Adopt New Architecture with HySparse 2".
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers are DEVICE pointers owned by the caller unless stated otherwise,
 *   16-byte aligned, dense, in these layouts (row-major, last index fastest):
 *     Q, O            [T, n_q_heads, head_dim]       bf16
 *     K, V            [T, n_kv_heads, head_dim]      bf16
 *     lse             [T, n_q_heads]                 fp32, natural log
 *     idx             [T, n_kv_heads, k_global + window]  int32
 *   Query head h uses KV head g = h / G with G = n_q_heads / n_kv_heads.
 * - bf16 and e4m3 values are passed as their raw bits (hs2_bf16, hs2_fp8e4m3).
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and never synchronises, except hs2_get_device_status.
 * - The library allocates no device memory.  Calls that need temporaries take
 *   a caller-owned workspace of at least hs2_workspace_size() bytes.
 * - Arguments are checked on the host before any launch.  A failed check
 *   returns an error and launches nothing; outputs are then untouched.
 * - Device-side waits are bounded.  A wait that runs out sets a sticky device
 *   status word, the kernel returns early, and the next
 *   hs2_get_device_status() reports HS2_ERR_TIMEOUT.
 * - Index lists passed in by the caller are checked entry by entry on the
 *   device: an entry other than -1 outside [0, T) is skipped like -1 and
 *   recorded, and the next hs2_get_device_status() reports HS2_ERR_BAD_INDEX.
 * - Supported: head_dim == 128; G in {1, 2, 4, 8, 16} (a query tile packs
 *   128 / G whole queries of one KV head, so G must divide 128);
 *   0 <= k_global <= 2048; 1 <= window <= 2048; 1 <= T <= 2^31 - 1
 *   (T * n_q_heads * 128 < 2^40).  Other shapes return HS2_ERR_UNSUPPORTED.
 * - Thread safety: calls on different streams may run concurrently; the only
 *   global state is one-time kernel attribute set-up per device.
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = 1, /* null/misaligned pointer, T <= 0, bad k/window   */
  HS2_ERR_UNSUPPORTED = 2, /* head_dim != 128, G not in {1,2,4,8,16}, ...      */
  HS2_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than required  */
  HS2_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed      */
  HS2_ERR_TIMEOUT = 5,     /* a device-side bounded wait ran out               */
  HS2_ERR_BAD_INDEX = 6    /* an index-list entry outside [-1, T) was skipped  */
} hs2_status;

typedef uint16_t hs2_bf16;    /* raw bf16 bits */
typedef uint8_t hs2_fp8e4m3;  /* raw OCP E4M3FN bits */

typedef struct {
  int64_t T;           /* tokens (prefill) or cache capacity (decode)          */
  int32_t n_q_heads;   /* Hq                                                   */
  int32_t n_kv_heads;  /* Hkv; Hq % Hkv == 0                                   */
  int32_t head_dim;    /* d; must be 128                                       */
  float scale;         /* logit scale, normally 1/sqrt(d)                      */
  int32_t k_global;    /* k: globally selected tokens per (query, KV head)     */
  int32_t window;      /* w: forced recent window, positions i-w+1 .. i        */
} hs2_shape;

/* Workspace queries (op codes for hs2_workspace_size). */
enum {
  HS2_OP_BRIDGE = 0,
  HS2_OP_FULL_ATTN = 1,
  HS2_OP_SELECT = 2,
  HS2_OP_SPARSE = 3,
  HS2_OP_BLOCK_PREFILL = 4,
  HS2_OP_BLOCK_DECODE = 5,
  HS2_OP_SPARSE_PLAN = 6  /* bytes of a plan for hs2_sparse_plan (size_t(-1): no plan path) */
};

/*
 * KV Bridging (step S1).  KV Bridging section of the javabetter.cn explainer
 * and section 一 of the siami.tw article: the cross-decoder full-attention
 * layer computes K and V from self-decoder hidden states with its own
 * projection parameters.
 *   K[t, :] = H[t, :] W_k,   V[t, :] = H[t, :] W_v
 * H [T, d_model] bf16; W_k, W_v [d_model, n_kv_heads * 128] bf16 (row-major);
 * K, V [T, n_kv_heads, 128] bf16, written with fp32 accumulation and one
 * round-to-nearest-even to bf16.  No RoPE, norm or bias (the pages name none).
 * d_model must be a positive multiple of 64.
 */
hs2_status hs2_bridge_kv(const hs2_bf16* H, int32_t d_model, const hs2_bf16* W_k,
                         const hs2_bf16* W_v, hs2_bf16* K, hs2_bf16* V,
                         const hs2_shape* shape, void* stream);

/*
 * Bridge-only prefill into the FP8 cache.  The javabetter.cn explainer's KV
 * Bridging paragraph (at prefill the cross-decoder's K/V come from the
 * self-decoder's hidden states) and the FP8 KV cache of the zgeo.com.cn
 * comparison table: step S1 fused with the cache's quantisation.
 *   K, V = bf16(H W_k), bf16(H W_v)            exactly as hs2_bridge_kv, then
 *   scale[t, g] = max(amax|K[t,g,:]|, amax|V[t,g,:]|) / 448   (fp32; 1 if 0)
 *   Kc[t, g, e] = e4m3(K[t, g, e] / scale[t, g])  (fp32 quotient, nearest,
 *                 ties to the even code, saturated at 448), likewise Vc.
 * H, W_k, W_v as in hs2_bridge_kv.  Kc, Vc [T, n_kv_heads, 128] e4m3 codes
 * and scale [T, n_kv_heads] fp32: the layout of one sequence of the decode
 * cache (hs2_block_decode reads scale as k_scale and v_scale).  Pointers
 * 16-byte aligned; d_model a positive multiple of 64.  No workspace.
 */
hs2_status hs2_bridge_kv_fp8(const hs2_bf16* H, int32_t d_model, const hs2_bf16* W_k,
                             const hs2_bf16* W_v, hs2_fp8e4m3* Kc, hs2_fp8e4m3* Vc,
                             float* scale, const hs2_shape* shape, void* stream);

/*
 * Causal GQA full attention with per-row log-sum-exp (step S2).  The block's
 * full-attention layer (Cross-Decoder paragraph of the javabetter.cn
 * explainer); its complete attention scores later rank tokens (section
 * 核心技术原理解析 of the zgeo.com.cn page).  For row i, head h, g = h / G:
 *   s_j = scale * Q[i,h] . K[j,g]  (0 <= j <= i)
 *   lse[i,h] = ln sum_j exp(s_j),  O[i,h] = sum_j exp(s_j - lse[i,h]) V[j,g]
 * O is rounded once to bf16; lse is fp32.  No workspace.
 */
hs2_status hs2_full_attn_lse(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                             hs2_bf16* O, float* lse, const hs2_shape* shape, void* stream);

/*
 * Token-level selection with forced recent window (step S3).  Selection
 * paragraphs of the javabetter.cn explainer (tokens picked one by one, e.g.
 * 1024 from the whole context, by the full layer's attention scores; the 128
 * most recent always kept), section 四 of the siami.tw article, and the
 * 1024 + 128 entry of the zgeo.com.cn comparison table.
 *   score[i,g,j] = sum over the G query heads h of g of exp(s_{h,i,j} - lse[i,h])
 *   candidates j in [0, i - w]; all of them when there are at most k,
 *   otherwise the k largest scores, equal scores going to the smaller j.
 * idx[i,g,0..k-1]: the selected positions in ascending order, then -1 padding.
 * idx[i,g,k+t] = i - w + 1 + t for t in [0, w), or -1 where that is negative.
 * kth_score (nullable) [T, n_kv_heads] fp32: score of the k-th selected token,
 * or -1 when every candidate is selected.
 * lse is the full layer's lse (as written by hs2_full_attn_lse).
 * Workspace: hs2_workspace_size(HS2_OP_SELECT, ...) bytes.
 */
hs2_status hs2_select_topk(const hs2_bf16* Q, const hs2_bf16* K, const float* lse,
                           int32_t* idx, float* kth_score, const hs2_shape* shape,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * hs2_select_topk without a workspace argument.  No counterpart on the pages:
 * this exists for callers that cannot allocate device memory themselves, for
 * example a host program whose device memory is owned and budgeted by another
 * runtime's allocator, or code on a latency-critical path that must not call
 * cudaMalloc (which may synchronise the device).  It computes exactly what
 * hs2_select_topk computes, with the same arguments minus the workspace, and
 * allocates nothing: its scratch is a 48 MiB array inside the library that
 * every GPU loading the library holds until the process exits.
 *   - The first call on a device looks up that array's device address (once
 *     per device, with the device current); make that first call before any
 *     stream capture.
 *   - The array is shared by all calls on a device and keeps the last call's
 *     contents (none of it needs to start at zero).  Calls whose kernels
 *     overlap on the same device, e.g. on two streams, race on it: serialise
 *     them.
 *   - The kernel runs as many persistent CTAs as the scratch holds; each needs
 *     4 * (128 / G) * max(2 * k_global, 256) * 8 + 262144 bytes.  A shape for
 *     which one CTA does not fit returns HS2_ERR_UNSUPPORTED.
 * Errors otherwise as hs2_select_topk (HS2_ERR_CUDA if the address lookup
 * fails).
 */
hs2_status hs2_select_topk_noalloc(const hs2_bf16* Q, const hs2_bf16* K, const float* lse,
                                   int32_t* idx, float* kth_score, const hs2_shape* shape,
                                   void* stream);

/*
 * Sparse attention over the shared K/V and index list (step S4, KV Reuse).
 * KV Reuse paragraph of the javabetter.cn explainer and the aitop.news
 * summary: each sparse layer has its own queries, reuses the full layer's K/V
 * cache and selection indices, and stores no K/V.  For row i, head h:
 *   s_j = scale * Q[i,h] . K[j,g] for j in idx[i,g,:] (entries -1 skipped)
 *   O[i,h] = sum_j softmax_j(s) V[j,g];  lse (nullable) = ln sum_j exp(s_j).
 * Entries should satisfy -1 <= idx < T and a list should hold no duplicates
 * (as written by hs2_select_topk).  Any other entry is skipped like -1 and
 * reported as HS2_ERR_BAD_INDEX by the next hs2_get_device_status(); K and V
 * are never read outside their T rows.  A row whose list is entirely -1 gets
 * O = 0, lse = -inf.  No workspace.
 */
hs2_status hs2_sparse_attn(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                           const int32_t* idx, hs2_bf16* O, float* lse,
                           const hs2_shape* shape, void* stream);

/*
 * Several sparse layers in one pass over the gathered rows (variant of
 * hs2_sparse_attn; no counterpart on the pages).  Layer l computes exactly
 * what hs2_sparse_attn(Q[l], K, V, idx, O[l], lse[l]) computes, but every
 * gathered K/V row serves all the layers' queries (up to three per pass when
 * G <= 8, one otherwise).  Valid only when every layer's queries exist before
 * the call: in a model's forward pass layer l+1's queries depend on layer l's
 * output, so the block (hs2_block_prefill) runs the layers one by one.
 * Q, O: HOST arrays of n_layers DEVICE pointers; lse: NULL or a HOST array of
 * n_layers nullable DEVICE pointers.  No workspace.
 */
hs2_status hs2_sparse_attn_layers(int32_t n_layers, const hs2_bf16* const* Q,
                                  const hs2_bf16* K, const hs2_bf16* V, const int32_t* idx,
                                  hs2_bf16* const* O, float* const* lse,
                                  const hs2_shape* shape, void* stream);

/*
 * Sparse attention in two calls, over the union of neighbouring queries'
 * lists (same operation as hs2_sparse_attn; no counterpart on the pages).
 * The lists of P = 256 / G consecutive query rows of one KV head overlap
 * heavily (their recent windows almost entirely), so each distinct listed row
 * can be gathered once for all of them (two 128-row tensor-core tiles of
 * (query, head) rows share it).
 *
 * hs2_sparse_plan: from idx [T, n_kv_heads, k_global + window] (as written by
 * hs2_select_topk, any order within a list), per (P query rows, KV head) the
 * ascending union of their lists and, per union row, which of the P queries
 * list it.  plan: a DEVICE buffer of hs2_workspace_size(HS2_OP_SPARSE_PLAN,
 * shape) bytes, 16-byte aligned, owned by the caller; it depends only on idx
 * and the shape and serves every sparse layer that shares idx.  An entry
 * outside [-1, T), or one listed twice in a row's list, is used at most once
 * and reported as HS2_ERR_BAD_INDEX by the next hs2_get_device_status().
 *
 * hs2_sparse_attn_planned: what hs2_sparse_attn(Q, K, V, idx, O, lse) writes
 * for the idx the plan was built from, up to fp32 rounding order (the union
 * rows are attended with a tcgen05 tile per 128 of them; rows a query does
 * not list get probability exactly 0).  plan must come from hs2_sparse_plan
 * with the same shape on the same stream (or a synchronised one).
 *
 * Both: HS2_ERR_UNSUPPORTED unless G = n_q_heads / n_kv_heads is 8 or 16,
 * P * (k_global + window) <= 36864 and T * n_kv_heads < 2^31;
 * HS2_ERR_WORKSPACE if plan_bytes is short.  hs2_block_prefill and
 * hs2_block_prefill_rows take this path by themselves where it applies.
 */
hs2_status hs2_sparse_plan(const int32_t* idx, const hs2_shape* shape, void* plan,
                           size_t plan_bytes, void* stream);
hs2_status hs2_sparse_attn_planned(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V,
                                   const void* plan, hs2_bf16* O, float* lse,
                                   const hs2_shape* shape, void* stream);

/*
 * The whole block at prefill: bridge (if H != NULL), full attention, selection
 * and n_sparse sparse layers sharing K/V and idx (all of the above, in order,
 * on `stream`).  Q_sparse and O_sparse are HOST arrays of n_sparse DEVICE
 * pointers.  With H == NULL, K and V are inputs and d_model, W_k, W_v are
 * ignored.  Workspace: hs2_workspace_size(HS2_OP_BLOCK_PREFILL, ...).
 */
hs2_status hs2_block_prefill(const hs2_bf16* H, int32_t d_model, const hs2_bf16* W_k,
                             const hs2_bf16* W_v, hs2_bf16* K, hs2_bf16* V,
                             const hs2_bf16* Q_full, hs2_bf16* O_full, float* lse,
                             int32_t* idx, int32_t n_sparse, const hs2_bf16* const* Q_sparse,
                             hs2_bf16* const* O_sparse, const hs2_shape* shape,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * The block at prefill for a range of query rows, given the K/V of the whole
 * causal prefix: rows of Q_full, O_full, lse, idx, Q_sparse and O_sparse are
 * positions q_begin .. q_begin + shape->T - 1; K and V [q_begin + shape->T,
 * n_kv_heads, 128] hold positions 0 .. q_begin + shape->T - 1.  Every row
 * is computed exactly as hs2_block_prefill computes it for the whole prompt
 * (full attention, selection, n_sparse sparse layers), so a prompt can be
 * split into row ranges over calls or over ranks (each rank with the
 * all-gathered K/V).  No counterpart on the pages.  q_begin must be a
 * multiple of 128 (HS2_ERR_UNSUPPORTED otherwise).  No bridge: K/V are
 * inputs.  Workspace: hs2_workspace_size(HS2_OP_BLOCK_PREFILL, shape, ...).
 */
hs2_status hs2_block_prefill_rows(int64_t q_begin, const hs2_bf16* K, const hs2_bf16* V,
                                  const hs2_bf16* Q_full, hs2_bf16* O_full, float* lse,
                                  int32_t* idx, int32_t n_sparse, const hs2_bf16* const* Q_sparse,
                                  hs2_bf16* const* O_sparse, const hs2_shape* shape,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step of the block over an FP8 KV cache (step S5).  The FP8 KV
 * cache of the zgeo.com.cn comparison table and of the javabetter.cn
 * explainer's 1M-token figures; the cross-decoder runs only while generating.
 * For each sequence b the new token is the last cache entry, i = seq_len[b]-1,
 * and the block (full attention, selection, n_sparse sparse layers) runs on
 *   K^[t,g,:] = e4m3(Kc[b,t,g,:]) * k_scale[b,t,g],  likewise V with v_scale.
 * seq_len: HOST array [batch], 1 <= seq_len[b] <= shape->T.
 * Limits: batch <= 64 and batch * shape->T <= 2^31 - 1 (HS2_ERR_UNSUPPORTED
 * otherwise, before any launch).
 * Kc, Vc [batch, shape->T, n_kv_heads, 128] e4m3; k_scale, v_scale
 * [batch, shape->T, n_kv_heads] fp32 (they may alias).
 * q_full, o_full [batch, n_q_heads, 128] bf16; lse [batch, n_q_heads] fp32;
 * idx [batch, n_kv_heads, k + w] int32; q_sparse/o_sparse: HOST arrays of
 * n_sparse DEVICE pointers to [batch, n_q_heads, 128] bf16.
 * Workspace: hs2_workspace_size(HS2_OP_BLOCK_DECODE, shape, batch, 0).
 */
hs2_status hs2_block_decode(int32_t batch, const int64_t* seq_len, const hs2_bf16* q_full,
                            const hs2_fp8e4m3* Kc, const hs2_fp8e4m3* Vc,
                            const float* k_scale, const float* v_scale, hs2_bf16* o_full,
                            float* lse, int32_t* idx, int32_t n_sparse,
                            const hs2_bf16* const* q_sparse, hs2_bf16* const* o_sparse,
                            const hs2_shape* shape, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * One decode step of the block with each sequence's context split over R
 * ranks (devices), in four calls with an all-gather of small records between
 * consecutive calls.  Not on the pages, which serve the 1M-token FP8 cache
 * from one device (zgeo.com.cn comparison table); this is the split that
 * lets that cache span several GPUs.  Every rank makes the same four calls;
 * the outputs of hs2_decode_cp_select, _sparse and _finish are identical on
 * every rank and equal to hs2_block_decode's up to fp32 rounding order (the
 * index lists are exact).
 *
 * Rank r holds, for each sequence b, the slice [slice_lo[b], slice_hi[b])
 * of its positions (HOST arrays [batch]; 0 <= lo <= hi <= seq_len[b]; the
 * ranks' slices tile [0, seq_len[b])).  Its cache stores that slice only:
 * position p at row p - slice_lo[b] of sequence b, Kc/Vc [batch, shape->T,
 * n_kv_heads, 128] e4m3 and k_scale/v_scale [batch, shape->T, n_kv_heads]
 * with shape->T >= hi - lo (the local capacity).  seq_len (HOST [batch]) is
 * the whole sequence length; the new token is position seq_len[b] - 1.
 * Records (all DEVICE memory, 16-byte aligned):
 *   attention / sparse record: 130 floats per (b, query head): the softmax
 *     state m (base-2 max logit), l (sum of 2^(x - m)), o[128] (unnormalised
 *     sum of 2^(x - m) v) over the rank's keys;
 *   selection record: 2 x uint32 per entry (score bits, position), k entries
 *     per (b, KV head): the rank's own exact top k (padded with
 *     (0, 0xFFFFFFFF) when it has fewer candidates).
 * "Gathered" inputs are the R ranks' records concatenated in rank order
 * (what an all-gather into one buffer writes).  n_ranks * k_global <= 8192.
 *
 * 1. hs2_decode_cp_attn: attention of the new token over the rank's slice ->
 *    attn_rec [batch][n_q_heads][130].  Workspace as hs2_block_decode
 *    (hs2_workspace_size(HS2_OP_BLOCK_DECODE, shape, batch, 0) with the
 *    local capacity); keep it for step 2, which reads this step's logits.
 * 2. hs2_decode_cp_select: merges the gathered attn_recs [R][batch][Hq][130]
 *    into o_full [batch, Hq, 128] bf16 and lse [batch, Hq] (natural log),
 *    scores the rank's candidates and writes its top k as sel_rec
 *    [batch][n_kv_heads][k][2].
 * 3. hs2_decode_cp_sparse: merges the gathered sel_recs [R][batch][Hkv][k][2]
 *    into idx [batch, Hkv, k + w] (the exact top k of the whole context,
 *    ascending, then the window) and runs the n_sparse sparse layers over the
 *    listed positions in the rank's slice -> sparse_rec
 *    [n_sparse][batch][Hq][130].  q_sparse: HOST array of n_sparse DEVICE
 *    pointers [batch, Hq, 128].  No workspace.
 * 4. hs2_decode_cp_finish: merges the gathered sparse_recs
 *    [R][n_sparse][batch][Hq][130] into o_sparse (HOST array of n_sparse
 *    DEVICE pointers [batch, Hq, 128] bf16).  No workspace.
 * Errors as hs2_block_decode; HS2_ERR_UNSUPPORTED if n_ranks * k > 8192.
 */
hs2_status hs2_decode_cp_attn(int32_t batch, const int64_t* seq_len, const int64_t* slice_lo,
                              const int64_t* slice_hi, const hs2_bf16* q_full,
                              const hs2_fp8e4m3* Kc, const hs2_fp8e4m3* Vc, const float* k_scale,
                              const float* v_scale, float* attn_rec, const hs2_shape* shape,
                              void* workspace, size_t workspace_bytes, void* stream);
hs2_status hs2_decode_cp_select(int32_t batch, const int64_t* seq_len, const int64_t* slice_lo,
                                const int64_t* slice_hi, int32_t n_ranks, const float* attn_recs,
                                hs2_bf16* o_full, float* lse, uint32_t* sel_rec,
                                const hs2_shape* shape, void* workspace, size_t workspace_bytes,
                                void* stream);
hs2_status hs2_decode_cp_sparse(int32_t batch, const int64_t* seq_len, const int64_t* slice_lo,
                                const int64_t* slice_hi, int32_t n_ranks,
                                const uint32_t* sel_recs, int32_t* idx, const hs2_fp8e4m3* Kc,
                                const hs2_fp8e4m3* Vc, const float* k_scale,
                                const float* v_scale, int32_t n_sparse,
                                const hs2_bf16* const* q_sparse, float* sparse_rec,
                                const hs2_shape* shape, void* stream);
hs2_status hs2_decode_cp_finish(int32_t batch, int32_t n_ranks, int32_t n_sparse,
                                const float* sparse_recs, hs2_bf16* const* o_sparse,
                                const hs2_shape* shape, void* stream);

/* Workspace bytes needed by `op` (an HS2_OP_* code) for these sizes; 0 when
 * the op needs none.  Returns (size_t)-1 for invalid arguments. */
size_t hs2_workspace_size(int32_t op, const hs2_shape* shape, int32_t batch, int32_t d_model);

/* Synchronises `stream` and reports a sticky device-side error, clearing it:
 * a bounded wait that ran out as HS2_ERR_TIMEOUT, otherwise a skipped
 * out-of-range index entry as HS2_ERR_BAD_INDEX; CUDA errors as
 * HS2_ERR_CUDA. */
hs2_status hs2_get_device_status(void* stream);

/* Testing hook, not part of the block: sets the spin budget (GPU clock
 * cycles) of every bounded wait in the library's kernels on the current
 * device, for launches that follow; cycles <= 0 restores the default of
 * 2^31.  A tiny budget makes waits run out, so a test can check that the
 * kernels unwind cleanly (they first wait, with a fixed budget, for their own
 * copies and MMAs in flight, then release tensor memory and exit) and that
 * hs2_get_device_status() reports HS2_ERR_TIMEOUT.  Synchronous; not for use
 * while library kernels run. */
hs2_status hs2_debug_set_wait_budget(int64_t cycles);

/* Testing hook, not part of the block: hs2_select_topk (and the block calls
 * that select) start each work item's score floor at `factor` times the
 * smallest k-th best score of the same CTA's previous item of that KV head
 * (default 0.9; <= 0 turns this off).  A floor above an item's true k-th best
 * is detected (a query ends with fewer than k buffered candidates) and the
 * item is recomputed without it by a second launch, so results never depend
 * on the factor; a factor of 1e30 forces every such item through that
 * recomputation.  Process-wide host state; not thread-safe. */
hs2_status hs2_debug_set_select_speculation(float factor);

/* Measurement hook, not part of the block: `reps` passes of 16-byte loads
 * through L2 over the DEVICE buffer buf (16-byte aligned, bytes a multiple
 * of 16) by a grid of 4 CTAs per SM, for the read-bandwidth denominator of a
 * roofline (a buffer that fits in L2 measures L2, a larger one HBM).  sink:
 * one DEVICE uint32, written only in the rare event that all loaded words
 * fold to one constant. */
hs2_status hs2_debug_read_probe(const void* buf, size_t bytes, int32_t reps, uint32_t* sink,
                                void* stream);

/* Static English text for a status code. */
const char* hs2_status_string(hs2_status status);

/* Launch count of the library's kernels since load (all devices). */
uint64_t hs2_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* HS2_H_ */
