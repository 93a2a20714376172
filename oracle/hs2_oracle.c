/*
 * hs2_oracle.c -- plain, slow CPU oracle of the HySparse2 cross-decoder block.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * bench's CPU-baseline leg may load this library.  It shares no code, header,
 * table or constant with the CUDA library and includes none of its files.
 *
 * Every value is widened exactly to fp64 (bf16 bits, or an e4m3 code times its
 * fp32 scale, which fp64 holds exactly) and every sum, product, exp and log is
 * taken in fp64.  Loops follow the definitions term by term; the only
 * parallelism is one host thread per (query row, KV head) pair.
 *
 * Sources (web pages on HySparse2, "Hybrid Sparse Attention with Two-Level KV
 * Sharing"), cited below by tag:
 *   [P1 s1]  siami.tw, "小米 MiMo-V3 全新架構亮相：HySparse 2 把 1M Token 預填成本砍到 1/5",
 *            section 一 (two-level KV sharing: KV Bridging, KV Reuse, token-level
 *            sparsity, forced recent window).
 *   [P1 s4]  same page, section 四 (token-level selection; forced recent window
 *            replaces the separate SWA branch).
 *   [P2 tbl] zgeo.com.cn, "小米MiMo-V3架构剧透：HySparse2稀疏注意力如何让长上下文成本暴降5倍…",
 *            section 核心技术原理解析 and its comparison table (1024 global +
 *            128 most recent tokens; FP8 KV cache).
 *   [P4]     aitop.news, "Xiaomi MiMo-V3 to Adopt New Architecture with HySparse 2"
 *            (sparse layers reuse the full-attention layer's KV cache and
 *            selection indices).
 *   [P5 ...] javabetter.cn explainer "mimo-v3-hysparse2": paragraphs on the
 *            Cross-Decoder block, KV Reuse, KV Bridging, selection granularity
 *            and the merged local window.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes): no RoPE/norm/bias on bridged K; score of key j for KV head g is the
 * sum over g's query heads of their softmax probabilities; candidates for row i
 * are j <= i-128 with the window i-127..i; ties in score go to the smaller
 * position; e4m3 is the OCP E4M3FN format.
 *
 * Parity pins live in tests/test_oracle_pins.py (special cases, invariants,
 * library routines, brute force).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* number formats                                                            */
/* ------------------------------------------------------------------------ */

static double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round an fp64 value to bf16 (8 significant bits), nearest, ties to even. */
uint16_t orc_bf16_from_f64(double x) {
  if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
  if (fabs(x) < 1.1754943508222875e-38) { /* below fp32 normal: go through fp32 */
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
  }
  uint64_t u;
  memcpy(&u, &x, 8);
  const int drop = 52 - 7; /* keep 7 stored mantissa bits */
  uint64_t lsb = (u >> drop) & 1u;
  u += ((uint64_t)1 << (drop - 1)) - 1 + lsb;
  u &= ~(((uint64_t)1 << drop) - 1);
  double r;
  memcpy(&r, &u, 8);
  float f = (float)r; /* exact: 8 significant bits, in fp32 range */
  uint32_t v;
  memcpy(&v, &f, 4);
  return (uint16_t)(v >> 16);
}

void orc_bf16_round(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_from_f64(x[i]);
}

/* OCP FP8 E4M3FN: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no
 * infinities, S.1111.111 is NaN, largest finite 448, subnormals at exponent 0.
 * [P2 tbl] and [P5] give the cache as "FP8"; the e4m3 variant is the reading. */
double orc_e4m3_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m / 8.0, -6);
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* K/V sources: bf16 rows, or e4m3 rows with one fp32 scale per (token, head) */
/* ------------------------------------------------------------------------ */

enum { ORC_BF16 = 0, ORC_E4M3 = 1 };

typedef struct {
  int kind;
  const void* data;   /* [T, Hkv, d] */
  const float* scale; /* [T, Hkv], e4m3 only */
  int Hkv, d;
} kv_src;

/* Value of every e4m3 code, filled once when the library is loaded (before
 * any parallel region reads it). */
static double e4m3_table[256];
__attribute__((constructor)) static void fill_e4m3_table(void) {
  for (int c = 0; c < 256; ++c) e4m3_table[c] = orc_e4m3_value(c);
}

static void fetch_row(const kv_src* s, int64_t t, int g, double* out) {
  int64_t base = (t * s->Hkv + g) * (int64_t)s->d;
  if (s->kind == ORC_BF16) {
    const uint16_t* p = (const uint16_t*)s->data + base;
    for (int c = 0; c < s->d; ++c) out[c] = bf16_value(p[c]);
  } else {
    const uint8_t* p = (const uint8_t*)s->data + base;
    double sc = (double)s->scale[t * s->Hkv + g];
    for (int c = 0; c < s->d; ++c) out[c] = e4m3_table[p[c]] * sc; /* exact in fp64 */
  }
}

static void fetch_q(const uint16_t* Qr, int64_t r, int h, int Hq, int d, double* out) {
  const uint16_t* p = Qr + ((int64_t)r * Hq + h) * d;
  for (int c = 0; c < d; ++c) out[c] = bf16_value(p[c]);
}

static double dot(const double* a, const double* b, int d) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

int orc_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* S1  KV Bridging: K = H W_k, V = H W_v                                      */
/* [P5 KV Bridging]: the cross-decoder's full-attention layer computes its K  */
/* and V from a self-decoder layer's hidden states with its own parameters;   */
/* [P1 s1], [P4] say the same.  out[t, n] = bf16( sum_c H[t, c] W[c, n] ).    */
/* ------------------------------------------------------------------------ */
void orc_bridge(const uint16_t* H, int64_t T, int dm, const uint16_t* W, int N, uint16_t* out) {
#pragma omp parallel
  {
    double* acc = (double*)malloc(sizeof(double) * (size_t)N);
    double* w = (double*)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t) {
      for (int n = 0; n < N; ++n) acc[n] = 0.0;
      for (int c = 0; c < dm; ++c) {
        double h = bf16_value(H[t * dm + c]);
        const uint16_t* wr = W + (int64_t)c * N;
        for (int n = 0; n < N; ++n) w[n] = bf16_value(wr[n]);
        for (int n = 0; n < N; ++n) acc[n] += h * w[n];
      }
      for (int n = 0; n < N; ++n) out[t * N + n] = orc_bf16_from_f64(acc[n]);
    }
    free(acc);
    free(w);
  }
}

/* ------------------------------------------------------------------------ */
/* f1  bridge-only prefill into the FP8 cache                                 */
/* [P5 KV Bridging] K/V of the cross-decoder come from the self-decoder's     */
/* hidden states at prefill; [P2 tbl] the cache is FP8.  K = bf16(H W_k) and  */
/* V = bf16(H W_v) exactly as in S1, then per (token t, KV head g) one fp32   */
/* scale s = max(amax|K[t,g,:]|, amax|V[t,g,:]|) / 448 (1 when that amax is   */
/* 0), and each code = e4m3(x / s): the quotient taken as an fp32 division,   */
/* rounded to the nearest e4m3 value (ties to the even code), magnitudes      */
/* above 448 saturated, the sign kept (a negative value that rounds to zero   */
/* gives the negative zero code).                                             */
/* ------------------------------------------------------------------------ */
uint8_t orc_e4m3_encode(float x) {
  const double a = fabs((double)x);
  int code;
  if (a >= 448.0) {
    code = 0x7E;
  } else {
    int lo = 0; /* largest finite positive code whose value is <= a */
    while (lo < 0x7E && orc_e4m3_value(lo + 1) <= a) ++lo;
    if (orc_e4m3_value(lo) == a) {
      code = lo;
    } else {
      const double dlo = a - orc_e4m3_value(lo), dhi = orc_e4m3_value(lo + 1) - a;
      code = dlo < dhi ? lo : dhi < dlo ? lo + 1 : (lo % 2 == 0 ? lo : lo + 1);
    }
  }
  return (uint8_t)(code | (signbit(x) ? 0x80 : 0));
}

/* rows: K and V bf16 bits [rows, d] (a row = one (token, KV head)) -> codes
 * [rows, d] and scales [rows] */
void orc_quantize_rows(const uint16_t* K, const uint16_t* V, int64_t rows, int d, uint8_t* Kc,
                       uint8_t* Vc, float* scale) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    float amax = 0.0f;
    for (int e = 0; e < d; ++e) {
      const float k = fabsf((float)bf16_value(K[r * d + e]));
      const float v = fabsf((float)bf16_value(V[r * d + e]));
      if (k > amax) amax = k;
      if (v > amax) amax = v;
    }
    const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    scale[r] = s;
    for (int e = 0; e < d; ++e) {
      const float qk = (float)bf16_value(K[r * d + e]) / s;
      const float qv = (float)bf16_value(V[r * d + e]) / s;
      Kc[r * d + e] = orc_e4m3_encode(qk);
      Vc[r * d + e] = orc_e4m3_encode(qv);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* S2  causal GQA full attention with log-sum-exp                             */
/* [P5 Cross-Decoder]: each block starts with one full-attention layer that   */
/* looks at every earlier token; [P2 原理] its complete attention scores pick */
/* the tokens for the sparse layers.  For query row i and head h (KV head     */
/* g = h / G):  s_j = scale * q_h . k_j  (j <= i),                            */
/* lse = ln sum_j exp(s_j),  o = sum_j exp(s_j - lse) v_j.                    */
/* Two passes: the max, then the sum and the weighted sum.                    */
/* ------------------------------------------------------------------------ */
void orc_full_attn(int kind, const void* K, const void* V, const float* ks, const float* vs,
                   int Hkv, int d, const uint16_t* Qr, const int64_t* rows, int64_t n, int Hq,
                   double scale, double* O, double* lse) {
  kv_src Ks = {kind, K, ks, Hkv, d}, Vs = {kind, V, vs, Hkv, d};
  const int G = Hq / Hkv;
#pragma omp parallel
  {
    double *q = (double*)malloc(sizeof(double) * d * G), *k = (double*)malloc(sizeof(double) * d);
    double* o = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1) collapse(2)
    for (int64_t r = 0; r < n; ++r) {
      for (int g = 0; g < Hkv; ++g) {
        const int64_t i = rows[r];
        double* s = (double*)malloc(sizeof(double) * (size_t)(i + 1) * G);
        for (int hh = 0; hh < G; ++hh) fetch_q(Qr, r, g * G + hh, Hq, d, q + hh * d);
        for (int64_t j = 0; j <= i; ++j) {
          fetch_row(&Ks, j, g, k);
          for (int hh = 0; hh < G; ++hh) s[hh * (i + 1) + j] = scale * dot(q + hh * d, k, d);
        }
        for (int hh = 0; hh < G; ++hh) {
          const double* sh = s + hh * (i + 1);
          double m = -INFINITY;
          for (int64_t j = 0; j <= i; ++j) m = sh[j] > m ? sh[j] : m;
          double sum = 0.0;
          for (int64_t j = 0; j <= i; ++j) sum += exp(sh[j] - m);
          double L = m + log(sum);
          lse[r * Hq + g * G + hh] = L;
          for (int c = 0; c < d; ++c) o[c] = 0.0;
          for (int64_t j = 0; j <= i; ++j) {
            double p = exp(sh[j] - L);
            fetch_row(&Vs, j, g, k);
            for (int c = 0; c < d; ++c) o[c] += p * k[c];
          }
          for (int c = 0; c < d; ++c) O[(r * Hq + g * G + hh) * (int64_t)d + c] = o[c];
        }
        free(s);
      }
    }
    free(q);
    free(k);
    free(o);
  }
}

/* ------------------------------------------------------------------------ */
/* S3  token scores and selection                                             */
/* [P5 挑选粒度]: tokens are chosen one by one (e.g. 1024 from the whole       */
/* context) by the full-attention layer's attention scores; [P5 局部窗口] and */
/* [P1 s4]: the 128 most recent tokens are always kept, replacing the SWA     */
/* branch; [P2 tbl]: 1024 global + 128 most recent.                           */
/*   score_{i,g,j} = sum_{h in g} exp(s_{h,i,j} - lse_{i,h})                 */
/*   candidates j in [0, i-128]; all of them if there are <= k, else the k   */
/*   largest scores, equal scores ordered by smaller j first;                */
/*   idx[0..k-1] = selected positions ascending, -1 padded;                  */
/*   idx[k+t] = i-w+1+t for t in [0, w), -1 where negative.                  */
/* ------------------------------------------------------------------------ */
typedef struct {
  double s;
  int64_t j;
} cand;

static int cand_cmp(const void* a, const void* b) {
  const cand *x = (const cand*)a, *y = (const cand*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int i64_cmp(const void* a, const void* b) {
  int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return (x > y) - (x < y);
}

static void score_row(const kv_src* Ks, const double* q, int G, int d, double scale,
                      const double* lse_g, int g, const int64_t* js, int64_t nj, double* out) {
  double* k = (double*)malloc(sizeof(double) * d);
  for (int64_t t = 0; t < nj; ++t) {
    fetch_row(Ks, js[t], g, k);
    double sc = 0.0;
    for (int hh = 0; hh < G; ++hh) sc += exp(scale * dot(q + hh * d, k, d) - lse_g[hh]);
    out[t] = sc;
  }
  free(k);
}

void orc_scores(int kind, const void* K, const float* ks, int Hkv, int d, const uint16_t* q_row,
                int g, int Hq, double scale, const double* lse_row, const int64_t* js, int64_t nj,
                double* out) {
  kv_src Ks = {kind, K, ks, Hkv, d};
  const int G = Hq / Hkv;
  double* q = (double*)malloc(sizeof(double) * d * G);
  for (int hh = 0; hh < G; ++hh) fetch_q(q_row, 0, g * G + hh, Hq, d, q + hh * d);
  score_row(&Ks, q, G, d, scale, lse_row + g * G, g, js, nj, out);
  free(q);
}

void orc_select(int kind, const void* K, const float* ks, int Hkv, int d, const uint16_t* Qr,
                const int64_t* rows, int64_t n, int Hq, double scale, const double* lse, int k,
                int w, int32_t* idx, double* kth) {
  kv_src Ks = {kind, K, ks, Hkv, d};
  const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
  for (int64_t r = 0; r < n; ++r) {
    for (int g = 0; g < Hkv; ++g) {
      const int64_t i = rows[r];
      int32_t* out = idx + (r * Hkv + g) * (int64_t)(k + w);
      const int64_t nc = i - w + 1 > 0 ? i - w + 1 : 0; /* candidates 0..i-w */
      int64_t nsel = nc < k ? nc : k;
      int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nsel > 0 ? nsel : 1));
      kth[r * Hkv + g] = NAN;
      if (nc <= k || k == 0) { /* all candidates, or none when k = 0 (no k-th score) */
        for (int64_t j = 0; j < nsel; ++j) sel[j] = j;
      } else {
        double* q = (double*)malloc(sizeof(double) * d * G);
        for (int hh = 0; hh < G; ++hh) fetch_q(Qr, r, g * G + hh, Hq, d, q + hh * d);
        int64_t* js = (int64_t*)malloc(sizeof(int64_t) * (size_t)nc);
        double* sc = (double*)malloc(sizeof(double) * (size_t)nc);
        cand* c = (cand*)malloc(sizeof(cand) * (size_t)nc);
        for (int64_t j = 0; j < nc; ++j) js[j] = j;
        score_row(&Ks, q, G, d, scale, lse + r * Hq + g * G, g, js, nc, sc);
        for (int64_t j = 0; j < nc; ++j) { c[j].s = sc[j]; c[j].j = j; }
        qsort(c, (size_t)nc, sizeof(cand), cand_cmp);
        for (int64_t t = 0; t < k; ++t) sel[t] = c[t].j;
        kth[r * Hkv + g] = c[k - 1].s;
        qsort(sel, (size_t)k, sizeof(int64_t), i64_cmp);
        free(q); free(js); free(sc); free(c);
      }
      for (int t = 0; t < k; ++t) out[t] = t < nsel ? (int32_t)sel[t] : -1;
      for (int t = 0; t < w; ++t) {
        int64_t p = i - w + 1 + t;
        out[k + t] = p >= 0 ? (int32_t)p : -1;
      }
      free(sel);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* S4  sparse attention over the shared K/V and index list (KV Reuse)          */
/* [P5 KV Reuse], [P4]: each sparse layer of a block attends with its own    */
/* queries to the block's full-attention K/V cache at the tokens on the full */
/* layer's list, and stores no K/V of its own.  For row i, head h:           */
/*   s_j = scale * q_h . k_j for j in idx_{i,g} (entries -1 skipped),        */
/*   lse = ln sum exp(s_j),  o = sum exp(s_j - lse) v_j.                      */
/* ------------------------------------------------------------------------ */
void orc_sparse_attn(int kind, const void* K, const void* V, const float* ks, const float* vs,
                     int Hkv, int d, const uint16_t* Qr, int64_t n, int Hq, double scale,
                     const int32_t* idx, int kw, double* O, double* lse) {
  kv_src Ks = {kind, K, ks, Hkv, d}, Vs = {kind, V, vs, Hkv, d};
  const int G = Hq / Hkv;
#pragma omp parallel
  {
    double *q = (double*)malloc(sizeof(double) * d * G), *k = (double*)malloc(sizeof(double) * d);
    double* s = (double*)malloc(sizeof(double) * (size_t)kw * G);
    double* o = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 4) collapse(2)
    for (int64_t r = 0; r < n; ++r) {
      for (int g = 0; g < Hkv; ++g) {
        const int32_t* list = idx + (r * Hkv + g) * (int64_t)kw;
        for (int hh = 0; hh < G; ++hh) fetch_q(Qr, r, g * G + hh, Hq, d, q + hh * d);
        for (int t = 0; t < kw; ++t) {
          if (list[t] < 0) continue;
          fetch_row(&Ks, list[t], g, k);
          for (int hh = 0; hh < G; ++hh) s[hh * kw + t] = scale * dot(q + hh * d, k, d);
        }
        for (int hh = 0; hh < G; ++hh) {
          const double* sh = s + hh * kw;
          double m = -INFINITY;
          for (int t = 0; t < kw; ++t)
            if (list[t] >= 0 && sh[t] > m) m = sh[t];
          double sum = 0.0;
          for (int t = 0; t < kw; ++t)
            if (list[t] >= 0) sum += exp(sh[t] - m);
          double L = m + log(sum);
          for (int c = 0; c < d; ++c) o[c] = 0.0;
          for (int t = 0; t < kw; ++t) {
            if (list[t] < 0) continue;
            double p = exp(sh[t] - L);
            fetch_row(&Vs, list[t], g, k);
            for (int c = 0; c < d; ++c) o[c] += p * k[c];
          }
          if (lse) lse[r * Hq + g * G + hh] = L;
          for (int c = 0; c < d; ++c) O[(r * Hq + g * G + hh) * (int64_t)d + c] = o[c];
        }
      }
    }
    free(q); free(k); free(s); free(o);
  }
}
