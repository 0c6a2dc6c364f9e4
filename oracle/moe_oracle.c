/*
 * moe_oracle.c -- plain, slow, CPU reference of one Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline / reference leg may load this library.  The product
 * path (the CUDA library under routing_dispatch_expert_sigmoid_b200/csrc) never
 * calls it, and the two share no code, header, table or constant.
 *
 * What the layer computes, and where the pages say so:
 *   - A router scores every expert for every token and each token keeps its
 *     top-k experts ("Paralelismo experto para el servicio MoE", section
 *     "Buceo profundo"; "Expert Parallelism: MoE 模型的并行切分", section 1).
 *   - Per-expert capacity: tokens past an expert's capacity are dropped so the
 *     expert GEMMs keep a predictable shape ("Paralelismo experto ...",
 *     "Información técnica" and the FAQ entry on keeping expert matrix
 *     multiplies uniform).
 *   - Dispatch copies each token's hidden state once per selected expert and
 *     combine sums the expert outputs weighted by the router weight
 *     ("Expert Parallelism: MoE 模型的并行切分", section 12, question 2);
 *     tokens bound for the same expert are grouped together before the send
 *     (same page, section 4, "Token sorting").
 *   - Each expert runs its own FFN on its rows ("LLM MoE Expert Parallel
 *     生产实战", section "为什么 MoE 推理会慢在'最热专家'", step 3).
 *   - Sub-experts are disjoint partitions of an expert's intermediate neurons
 *     and the routing budget k may vary per request ("MoE-Prism", summary
 *     section 2.A and 2.B).
 *   - Sigmoid scores with a per-expert selection bias, group-limited routing
 *     (8 groups, keep 4 ranked by the sum of each group's top-2 scores) and a
 *     2.5 scale on the renormalised weights come from the DeepSeek-V3-shaped
 *     workload specification; the pages only name DeepSeek-V3's node-limited
 *     routing ("Paralelismo experto ...", "Implementación en el mundo real").
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - ties in every ranking go to the lower expert (or group) index;
 *   - capacity C = ceil(cf * sum_t k_t / E), evaluated in double as written;
 *     assignments are admitted in (token, slot) order, first C per expert;
 *     dropped slots contribute 0 and the kept weights are not renormalised;
 *   - SiLU is applied to the x.W1 product: h = silu(x.W1) * (x.W3);
 *   - selection for "softmax over all experts, then top-k" is made on the
 *     logits (softmax is monotone, so the selected set is the same and no
 *     ties are created by rounding of exp);
 *   - group scores use the biased scores, weights use the unbiased ones.
 *
 * Precision: every sum and product below is accumulated in double, from the
 * stored (fp32 or bf16) values.  The one exception is the sigmoid used by the
 * biased group-limited selection: a selection is an integer decision, so it
 * is taken in fp32 by a fully specified function (oracle_spec_expf below)
 * that the GPU path implements independently with the same IEEE operations.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (see oracle/build.py).
 * -ffp-contract=off keeps the compiler from fusing a*b+c where the code does
 * not ask for fmaf explicitly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_F64 2 /* dequantised fp8 weights, exact in double */

#define OR_TOPK_SOFTMAX 0
#define OR_SOFTMAX_TOPK_RENORM 1
#define OR_SIGMOID_GROUPED 2

/* Read element i of a tensor stored as fp32 or bf16 and widen it to double.
 * bf16 is the upper half of an IEEE binary32, so widening is a shift. */
static double ld(const void *p, int dtype, size_t i) {
  if (dtype == OR_F32) return (double)((const float *)p)[i];
  if (dtype == OR_F64) return ((const double *)p)[i];
  uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float v;
  memcpy(&v, &bits, sizeof v);
  return (double)v;
}

/* ------------------------------------------------------------------------ */
/* Router: logits[t,e] = sum_i x[t,i] * Wr[i,e] (+ logit_bias[e]).            */
/* "Paralelismo experto ...", "Buceo profundo": the router scores experts.   */
/* ------------------------------------------------------------------------ */
void oracle_router_logits(int T, int d, int E, const void *x, const void *Wr, int dtype,
                          const float *logit_bias, double *logits) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i)
        acc += ld(x, dtype, (size_t)t * d + i) * ld(Wr, dtype, (size_t)i * E + e);
      if (logit_bias) acc += (double)logit_bias[e];
      logits[(size_t)t * E + e] = acc;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Specified fp32 exp and sigmoid for the biased group-limited selection.    */
/*                                                                            */
/* Method: Cody & Waite additive range reduction (Cody and Waite, "Software  */
/* Manual for the Elementary Functions", 1980) followed by the degree-7      */
/* Taylor polynomial of e^r about 0, evaluated by Horner's rule with one     */
/* fused multiply-add per step, then scaling by 2^n through the exponent     */
/* field.  Every step is a single correctly rounded IEEE binary32 operation  */
/* (mul, fma, rint, div), so any IEEE-conforming machine that performs the   */
/* same sequence gets the same bits.                                         */
/*                                                                            */
/* Constants, derived here from their definitions:                           */
/*   LOG2E  = binary32 nearest to 1/ln 2                      = 0x3FB8AA3B    */
/*   LN2_HI = ln 2 rounded to 12 significant bits = 2839/4096 = 0x3F317000    */
/*            (n*LN2_HI is exact in binary32 for |n| < 2^12)                  */
/*   LN2_LO = binary32 nearest to ln 2 - 2839/4096            = 0x3805FDF4    */
/*   C_k    = binary32 nearest to 1/k!, k = 2..7                              */
/* The argument is clamped to [-87, 87] so that 2^n stays a normal number.   */
/* ------------------------------------------------------------------------ */
static float f32_from_bits(uint32_t b) {
  float v;
  memcpy(&v, &b, sizeof v);
  return v;
}

static const float OR_LOG2E = 1.44269504088896340736f;
static const float OR_LN2_HI = 0.693115234375f;            /* 2839 / 4096 */
static const float OR_LN2_LO = 3.194618494528623e-05f;      /* ln2 - 2839/4096 */
static const float OR_INV_FACT[8] = {
    1.0f,                       /* 1/0! */
    1.0f,                       /* 1/1! */
    0.5f,                       /* 1/2! */
    0.166666666666666666667f,   /* 1/3! */
    0.0416666666666666666667f,  /* 1/4! */
    0.00833333333333333333333f, /* 1/5! */
    0.00138888888888888888889f, /* 1/6! */
    0.000198412698412698412698f /* 1/7! */
};

float oracle_spec_expf(float z) {
  if (z > 87.0f) z = 87.0f;
  if (z < -87.0f) z = -87.0f;
  float n = rintf(z * OR_LOG2E);
  float r = fmaf(-n, OR_LN2_HI, z);
  r = fmaf(-n, OR_LN2_LO, r);
  float p = OR_INV_FACT[7];
  for (int k = 6; k >= 0; --k) p = fmaf(p, r, OR_INV_FACT[k]);
  int ni = (int)n;
  float scale = f32_from_bits((uint32_t)(ni + 127) << 23);
  return p * scale;
}

float oracle_spec_sigmoidf(float z) {
  float e = oracle_spec_expf(-z);
  return 1.0f / (1.0f + e);
}

void oracle_spec_expf_n(int n, const float *z, float *out) {
  for (int i = 0; i < n; ++i) out[i] = oracle_spec_expf(z[i]);
}

void oracle_spec_sigmoidf_n(int n, const float *z, float *out) {
  for (int i = 0; i < n; ++i) out[i] = oracle_spec_sigmoidf(z[i]);
}

/* ------------------------------------------------------------------------ */
/* Gating: per token, choose k_t experts and their combine weights.          */
/* ------------------------------------------------------------------------ */
typedef struct {
  float key;
  int idx;
} keyed;

/* Descending key, ties to the lower index. */
static int cmp_keyed(const void *a, const void *b) {
  const keyed *x = (const keyed *)a, *y = (const keyed *)b;
  if (x->key > y->key) return -1;
  if (x->key < y->key) return 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/*
 * logits:   [T, E] fp32 (the values selection is decided on)
 * sel_bias: [E] fp32, only for OR_SIGMOID_GROUPED (may be NULL: zero bias)
 * k_t:      [T] per-token k in [1, k_max], or NULL for k_t = k_max
 * topk_idx: [T, k_max] out; slot j is the j-th best expert, -1 for j >= k_t
 * topk_w:   [T, k_max] out (double); 0 for j >= k_t
 */
int oracle_gating(int T, int E, int k_max, int mode, int n_groups, int topk_groups,
                  int group_score_topk, double routed_scale, const float *logits,
                  const float *sel_bias, const int *k_t, int *topk_idx, double *topk_w) {
  if (T < 0 || E <= 0 || k_max <= 0 || k_max > E) return -1;
  if (mode == OR_SIGMOID_GROUPED) {
    if (n_groups <= 0 || E % n_groups != 0 || topk_groups <= 0 || topk_groups > n_groups ||
        group_score_topk <= 0 || group_score_topk > E / n_groups)
      return -1;
    if (k_max > topk_groups * (E / n_groups)) return -1;
  }
  int bad = 0;
#pragma omp parallel
  {
    keyed *buf = (keyed *)malloc(sizeof(keyed) * (size_t)E);
    keyed *gbuf = (keyed *)malloc(sizeof(keyed) * (size_t)(n_groups > 0 ? n_groups : 1));
    float *s = (float *)malloc(sizeof(float) * (size_t)E);
    float *u = (float *)malloc(sizeof(float) * (size_t)E);
#pragma omp for schedule(static)
    for (int t = 0; t < T; ++t) {
      const float *l = logits + (size_t)t * E;
      int kt = k_t ? k_t[t] : k_max;
      if (kt < 1 || kt > k_max) {
#pragma omp atomic write
        bad = 1;
        continue;
      }
      int *oi = topk_idx + (size_t)t * k_max;
      double *ow = topk_w + (size_t)t * k_max;
      for (int j = 0; j < k_max; ++j) {
        oi[j] = -1;
        ow[j] = 0.0;
      }
      if (mode == OR_TOPK_SOFTMAX || mode == OR_SOFTMAX_TOPK_RENORM) {
        for (int e = 0; e < E; ++e) {
          buf[e].key = l[e];
          buf[e].idx = e;
        }
        qsort(buf, (size_t)E, sizeof(keyed), cmp_keyed);
        for (int j = 0; j < kt; ++j) oi[j] = buf[j].idx;
        if (mode == OR_TOPK_SOFTMAX) {
          /* Softmax over the k selected logits. */
          double m = (double)l[oi[0]], z = 0.0;
          for (int j = 0; j < kt; ++j) z += exp((double)l[oi[j]] - m);
          for (int j = 0; j < kt; ++j) ow[j] = exp((double)l[oi[j]] - m) / z;
        } else {
          /* p = softmax over all E experts; weights p_j / sum of selected p. */
          double m = (double)l[0];
          for (int e = 1; e < E; ++e)
            if ((double)l[e] > m) m = (double)l[e];
          double z = 0.0;
          for (int e = 0; e < E; ++e) z += exp((double)l[e] - m);
          double psel = 0.0;
          for (int j = 0; j < kt; ++j) psel += exp((double)l[oi[j]] - m) / z;
          for (int j = 0; j < kt; ++j) ow[j] = (exp((double)l[oi[j]] - m) / z) / psel;
        }
      } else {
        /* Sigmoid scores, biased selection keys, group-limited top-k. */
        int gsize = E / n_groups;
        for (int e = 0; e < E; ++e) {
          s[e] = oracle_spec_sigmoidf(l[e]);
          u[e] = s[e] + (sel_bias ? sel_bias[e] : 0.0f);
        }
        /* Group score: sum of the group's group_score_topk largest u, added
         * in descending order in fp32. */
        for (int g = 0; g < n_groups; ++g) {
          for (int i = 0; i < gsize; ++i) {
            buf[i].key = u[g * gsize + i];
            buf[i].idx = g * gsize + i;
          }
          qsort(buf, (size_t)gsize, sizeof(keyed), cmp_keyed);
          float sc = buf[0].key;
          for (int i = 1; i < group_score_topk; ++i) sc = sc + buf[i].key;
          gbuf[g].key = sc;
          gbuf[g].idx = g;
        }
        qsort(gbuf, (size_t)n_groups, sizeof(keyed), cmp_keyed);
        /* Candidates: every expert of the kept groups, ranked by u. */
        int nc = 0;
        for (int e = 0; e < E; ++e) {
          int g = e / gsize, keep = 0;
          for (int i = 0; i < topk_groups; ++i)
            if (gbuf[i].idx == g) keep = 1;
          if (keep) {
            buf[nc].key = u[e];
            buf[nc].idx = e;
            ++nc;
          }
        }
        qsort(buf, (size_t)nc, sizeof(keyed), cmp_keyed);
        double ssum = 0.0;
        for (int j = 0; j < kt; ++j) {
          oi[j] = buf[j].idx;
          ssum += (double)s[oi[j]];
        }
        for (int j = 0; j < kt; ++j) ow[j] = routed_scale * (double)s[oi[j]] / ssum;
      }
    }
    free(buf);
    free(gbuf);
    free(s);
    free(u);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Capacity, histogram, prefix sum and dispatch layout.                      */
/* Walk assignments in (token, slot) order; the first C assignments of each  */
/* expert are kept, the rest dropped ("Paralelismo experto ...", FAQ on      */
/* per-expert capacity).  Kept rows are laid out expert by expert, and in    */
/* (token, slot) order inside an expert: a stable sort by destination        */
/* ("Expert Parallelism: MoE 模型的并行切分", section 4, token sorting).      */
/*                                                                            */
/* counts[E]: assignments per expert before capacity; kept[E] = min(counts,C) */
/* offsets[E+1]: exclusive prefix sum of kept; slot_row[T*k_max]: the row of  */
/* a kept slot, -1 otherwise; row_src[R]: t*k_max + j of each row;            */
/* capacity_out: C (or -1 for no limit).  Returns n_dropped, or -1 on error. */
/* ------------------------------------------------------------------------ */
long long oracle_capacity_dispatch(int T, int E, int k_max, double capacity_factor,
                                   const int *topk_idx, int *counts, int *kept, int *offsets,
                                   int *slot_row, int *row_src, long long *capacity_out) {
  long long sum_k = 0;
  for (long long a = 0; a < (long long)T * k_max; ++a)
    if (topk_idx[a] >= 0) ++sum_k;
  long long C = -1;
  if (capacity_factor > 0.0) C = (long long)ceil(capacity_factor * (double)sum_k / (double)E);
  if (capacity_out) *capacity_out = C;

  for (int e = 0; e < E; ++e) counts[e] = 0;
  /* rank[a] = position of assignment a among its expert's assignments. */
  long long *rank = (long long *)malloc(sizeof(long long) * (size_t)((long long)T * k_max + 1));
  for (int t = 0; t < T; ++t)
    for (int j = 0; j < k_max; ++j) {
      long long a = (long long)t * k_max + j;
      int e = topk_idx[a];
      if (e < -1 || e >= E) {
        free(rank);
        return -1;
      }
      if (e < 0) {
        rank[a] = -1;
        continue;
      }
      rank[a] = counts[e];
      counts[e] += 1;
    }
  long long dropped = 0;
  for (int e = 0; e < E; ++e) {
    kept[e] = (C >= 0 && counts[e] > C) ? (int)C : counts[e];
    dropped += counts[e] - kept[e];
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + kept[e];
  for (long long a = 0; a < (long long)T * k_max; ++a) {
    int e = topk_idx[a];
    if (e < 0 || (C >= 0 && rank[a] >= C)) {
      slot_row[a] = -1;
      continue;
    }
    int row = offsets[e] + (int)rank[a];
    slot_row[a] = row;
    row_src[row] = (int)a;
  }
  free(rank);
  return dropped;
}

/* ------------------------------------------------------------------------ */
/* Dispatch: x_perm[r,:] = x[row_src[r] / k_max, :]  (a copy per selected     */
/* expert, "Expert Parallelism: MoE 模型的并行切分", section 12, question 2). */
/* Values are copied as stored (elem_bytes per element).                     */
/* ------------------------------------------------------------------------ */
void oracle_dispatch(int R, int k_max, int d, int elem_bytes, const int *row_src, const void *x,
                     void *x_perm) {
  for (int r = 0; r < R; ++r) {
    int t = row_src[r] / k_max;
    memcpy((char *)x_perm + (size_t)r * d * elem_bytes, (const char *)x + (size_t)t * d * elem_bytes,
           (size_t)d * elem_bytes);
  }
}

/* ------------------------------------------------------------------------ */
/* One expert's SwiGLU FFN on n rows:                                        */
/*   y = (silu(x.W1) * (x.W3)) . W2,  silu(z) = z / (1 + e^-z)               */
/* x: [n, d], W1, W3: [d, f], W2: [f, d] (row-major, stored dtype); y: [n, d] */
/* double.  "LLM MoE Expert Parallel 生产实战", step 3: each expert computes   */
/* on its own rows.                                                          */
/* ------------------------------------------------------------------------ */
static void ffn_row(int d, int f, const void *x, int x_dtype, size_t x_off, const void *W1,
                    const void *W3, const void *W2, int w_dtype, double *xr, double *g, double *u,
                    double *y) {
  for (int i = 0; i < d; ++i) xr[i] = ld(x, x_dtype, x_off + i);
  for (int c = 0; c < f; ++c) {
    g[c] = 0.0;
    u[c] = 0.0;
  }
  for (int i = 0; i < d; ++i)
    for (int c = 0; c < f; ++c) {
      g[c] += xr[i] * ld(W1, w_dtype, (size_t)i * f + c);
      u[c] += xr[i] * ld(W3, w_dtype, (size_t)i * f + c);
    }
  for (int c = 0; c < f; ++c) g[c] = (g[c] / (1.0 + exp(-g[c]))) * u[c];
  for (int o = 0; o < d; ++o) y[o] = 0.0;
  for (int c = 0; c < f; ++c)
    for (int o = 0; o < d; ++o) y[o] += g[c] * ld(W2, w_dtype, (size_t)c * d + o);
}

void oracle_expert_ffn(int n, int d, int f, const void *x, int x_dtype, const void *W1,
                       const void *W3, const void *W2, int w_dtype, double *y) {
#pragma omp parallel
  {
    double *xr = (double *)malloc(sizeof(double) * (size_t)d);
    double *g = (double *)malloc(sizeof(double) * (size_t)f);
    double *u = (double *)malloc(sizeof(double) * (size_t)f);
#pragma omp for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r)
      ffn_row(d, f, x, x_dtype, (size_t)r * d, W1, W3, W2, w_dtype, xr, g, u, y + (size_t)r * d);
    free(xr);
    free(g);
    free(u);
  }
}

/* ------------------------------------------------------------------------ */
/* Combine: out[t] = sum over kept slots j of w[t,j] * y_slot[t,j] (+ sh[t])  */
/* ("Expert Parallelism: MoE 模型的并行切分", section 12, question 2: outputs */
/* return to the token and are summed weighted by the router weight).        */
/* w: [n, k_max] double; kept: [n, k_max] 0/1; y_slot: [n, k_max, d] double;  */
/* shared: [n, d] double or NULL; out: [n, d] double.                         */
/* ------------------------------------------------------------------------ */
void oracle_combine(int n, int k_max, int d, const double *w, const int *kept,
                    const double *y_slot, const double *shared, double *out) {
  for (int t = 0; t < n; ++t) {
    double *o = out + (size_t)t * d;
    for (int c = 0; c < d; ++c) o[c] = shared ? shared[(size_t)t * d + c] : 0.0;
    for (int j = 0; j < k_max; ++j) {
      if (!kept[(size_t)t * k_max + j]) continue;
      const double *ys = y_slot + ((size_t)t * k_max + j) * d;
      for (int c = 0; c < d; ++c) o[c] += w[(size_t)t * k_max + j] * ys[c];
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Combine from expert-contiguous rows: the same sum, reading y_perm[row]     */
/* through slot_row (row of slot (t,j), -1 when dropped or padding).          */
/* y_perm: [R, d] stored dtype; shared: [T, d] stored dtype or NULL.          */
/* ------------------------------------------------------------------------ */
void oracle_combine_rows(int T, int k_max, int d, const double *w, const int *slot_row,
                         const void *y_perm, const void *shared, int dtype, double *out) {
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    double *o = out + (size_t)t * d;
    for (int c = 0; c < d; ++c) o[c] = shared ? ld(shared, dtype, (size_t)t * d + c) : 0.0;
    for (int j = 0; j < k_max; ++j) {
      int row = slot_row[(size_t)t * k_max + j];
      if (row < 0) continue;
      for (int c = 0; c < d; ++c)
        o[c] += w[(size_t)t * k_max + j] * ld(y_perm, dtype, (size_t)row * d + c);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Whole layer on a subset of tokens, for a given routing.  x is stored in   */
/* `dtype`, every weight in `w_dtype` (the same, or fp64 dequantised fp8).   */
/* For each listed token t: out[i] = sum_j w[t,j] * FFN_{idx[t,j]}(x[t])      */
/* over slots with slot_row >= 0, plus the shared expert's FFN(x[t]) when     */
/* Ws1 is given.  W1, W3: [E, d, f]; W2: [E, f, d]; Ws1, Ws3: [d, fs];        */
/* Ws2: [fs, d].  out: [n_tok, d] double.                                    */
/* ------------------------------------------------------------------------ */
void oracle_layer_tokens(int n_tok, const int *tok, int d, int E, int k_max, int f, int fs,
                         const void *x, const void *W1, const void *W3, const void *W2,
                         const void *Ws1, const void *Ws3, const void *Ws2, int dtype,
                         int w_dtype, const int *topk_idx, const double *topk_w,
                         const int *slot_row, double *out) {
  (void)E;
  size_t esz = w_dtype == OR_F64 ? 8 : (w_dtype == OR_F32 ? 4 : 2);
  int fmax = f > fs ? f : fs;
#pragma omp parallel
  {
    double *xr = (double *)malloc(sizeof(double) * (size_t)d);
    double *g = (double *)malloc(sizeof(double) * (size_t)fmax);
    double *u = (double *)malloc(sizeof(double) * (size_t)fmax);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_tok; ++i) {
      int t = tok[i];
      double *o = out + (size_t)i * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      if (Ws1 && fs > 0) {
        ffn_row(d, fs, x, dtype, (size_t)t * d, Ws1, Ws3, Ws2, w_dtype, xr, g, u, y);
        for (int c = 0; c < d; ++c) o[c] += y[c];
      }
      for (int j = 0; j < k_max; ++j) {
        size_t a = (size_t)t * k_max + j;
        if (slot_row[a] < 0) continue;
        int e = topk_idx[a];
        ffn_row(d, f, x, dtype, (size_t)t * d, (const char *)W1 + (size_t)e * d * f * esz,
                (const char *)W3 + (size_t)e * d * f * esz,
                (const char *)W2 + (size_t)e * f * d * esz, w_dtype, xr, g, u, y);
        for (int c = 0; c < d; ++c) o[c] += topk_w[a] * y[c];
      }
    }
    free(xr);
    free(g);
    free(u);
    free(y);
  }
}

/* ------------------------------------------------------------------------ */
/* FP8 expert weights.                                                       */
/* "LLM MoE Expert Parallel 生产实战", section 5 (DeepSeek-V3 served with     */
/* --quantization fp8) and section 10 (check that fp8 quantisation does not   */
/* disturb the router head): the experts' weights are stored in 8-bit        */
/* floating point while the router keeps its precision.  Reading: e4m3        */
/* codes (OCP FP8 E4M3, the finite-only variant) with one fp32 scale per      */
/* output column of each expert matrix; activations stay in the layer dtype. */
/*                                                                          */
/* e4m3: sign, 4 exponent bits (bias 7), 3 fraction bits.  Exponent field 0  */
/* holds the subnormals m * 2^-9; 1..15 hold (1 + m/8) * 2^(e-7); the code   */
/* with every exponent and fraction bit set is NaN, so the largest finite    */
/* magnitude is 1.75 * 2^8 = 448.  There is no infinity.                     */
/* ------------------------------------------------------------------------ */
double oracle_e4m3_decode(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Nearest e4m3 value, ties to the even code; finite magnitudes above 448
 * saturate to 448; NaN maps to the NaN code. */
uint8_t oracle_e4m3_encode(float v) {
  if (isnan(v)) return 0x7F;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs((double)v);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int ex;
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1): floor(log2 a) = ex - 1 */
  int E = ex - 1;
  if (E < -6) E = -6; /* below the smallest normal the grid step stays 2^-9 */
  const double step = ldexp(1.0, E - 3);
  const double q = a / step; /* exact: division by a power of two */
  double n = floor(q);
  const double rem = q - n;
  if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) == 1.0)) n += 1.0;
  const double val = n * step; /* the chosen grid point, <= 448 */
  if (val == 0.0) return sign;
  frexp(val, &ex);
  const int Ev = ex - 1;
  if (Ev < -6) return sign | (uint8_t)(val / ldexp(1.0, -9)); /* subnormal */
  const int m = (int)(val / ldexp(1.0, Ev - 3)) - 8;
  return sign | (uint8_t)((Ev + 7) << 3) | (uint8_t)m;
}

void oracle_e4m3_decode_n(long long n, const uint8_t *c, double *out) {
  for (long long i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

void oracle_e4m3_encode_n(long long n, const float *v, uint8_t *out) {
  for (long long i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* Quantise W[g][k][n] (bf16 bits) per output column (g, n):
 *   amax = max_k |W[g][k][n]|;  s = amax / 448 in fp32 (1 when amax = 0);
 *   q[g][k][n] = e4m3(W[g][k][n] / s), the quotient rounded to fp32 first.
 * The dequantised weight is e4m3_decode(q) * s. */
void oracle_quantize_fp8(int G, int K, int N, const uint16_t *W, uint8_t *q, float *scale) {
#pragma omp parallel for schedule(static)
  for (long long gn = 0; gn < (long long)G * N; ++gn) {
    const int g = (int)(gn / N), n = (int)(gn % N);
    const size_t base = (size_t)g * K * N + n;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      const double w = ld(W, OR_BF16, base + (size_t)k * N);
      const float a = (float)fabs(w);
      if (a > amax) amax = a;
    }
    const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    scale[gn] = s;
    for (int k = 0; k < K; ++k) {
      const float w = (float)ld(W, OR_BF16, base + (size_t)k * N);
      q[base + (size_t)k * N] = oracle_e4m3_encode(w / s);
    }
  }
}

/* The constants of the specified exp, for the tests that derive them
 * independently: {LOG2E, LN2_HI, LN2_LO, 1/0!, ..., 1/7!}. */
void oracle_spec_constants(float *out) {
  out[0] = OR_LOG2E;
  out[1] = OR_LN2_HI;
  out[2] = OR_LN2_LO;
  for (int k = 0; k < 8; ++k) out[3 + k] = OR_INV_FACT[k];
}
