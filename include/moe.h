/*
 * moe.h -- C ABI of a single-GPU Mixture-of-Experts layer for NVIDIA B200 (sm_100a).
 *
 * The layer (one MoE FFN block, all experts resident on one GPU):
 *
 *   1. router          logits[T,E]   = x[T,d] . Wr[d,E] (+ logit_bias[E])      fp32
 *   2. gating          per token t, k_t experts and weights (three modes below)
 *   3. capacity        per-expert histogram, capacity C, drops, prefix sum
 *   4. dispatch        x_perm[r,:] = x[t(r),:], rows grouped by expert
 *   5. expert FFN      y_perm[r,:] = (silu(x_perm[r].W1[e]) * (x_perm[r].W3[e])) . W2[e]
 *   6. combine         out[t,:] = sum_j w[t,j] * y_perm[slot_row[t,j],:] (+ shared[t,:])
 *
 * Sources for what each step computes:
 *   - router and top-k: "Paralelismo experto para el servicio MoE"
 *     (aiunderstanding.org), section "Buceo profundo", and the FAQ entry on
 *     per-token compute; "Expert Parallelism: MoE 模型的并行切分" (SGLang
 *     learning notes), section 1;
 *   - the four steps route / send to the expert / local expert compute / send
 *     back and combine: "LLM MoE Expert Parallel 生产实战" (oh-bug.com), section
 *     "为什么 MoE 推理会慢在'最热专家'";
 *   - capacity factor, token dropping: "Paralelismo experto ...", section
 *     "Información técnica" and the FAQ entry on uniform expert GEMMs;
 *   - dispatch = one copy of the token per selected expert, combine = weighted
 *     sum by the router weight: "Expert Parallelism: MoE 模型的并行切分",
 *     section 12 question 2; grouping tokens by destination: same page,
 *     section 4 ("Token sorting"), and question 4 (no padding);
 *   - per-token routing budget k_t and sub-experts: "MoE-Prism" (gist.science
 *     summary of arXiv 2510.19366), section 2.A and 2.B;
 *   - shared expert: "LLM MoE Expert Parallel 生产实战", launch checklist;
 *   - sigmoid scores + selection bias + group-limited routing + routed scale:
 *     the DeepSeek-V3-shaped workload specification (the pages only name
 *     DeepSeek-V3's node-limited routing, "Paralelismo experto ...",
 *     "Implementación en el mundo real").
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers, row-major, owned by the caller.
 *     The library never allocates, frees or synchronises in these calls;
 *     scratch memory comes from a caller workspace sized by moe_workspace_size.
 *   - Floating tensors x, Wr, W1, W3, W2, Ws1, Ws3, Ws2, x_perm and out are
 *     stored in cfg->dtype (fp32 or bf16).  The expert outputs y_perm and
 *     shared_y are always fp32, so the layer output is rounded once, after the
 *     weighted sum.  logits, topk_w, logit_bias and sel_bias are always fp32.
 *     Indices and counts are int32.
 *   - Alignment: every tensor pointer and the workspace must be 16-byte aligned,
 *     and d and f (and f_shared) must make rows a multiple of 16 bytes:
 *     d % 8 == 0 and f % 8 == 0 for bf16, d % 4 == 0 and f % 4 == 0 for fp32.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously; results are valid once the stream reaches them.
 *   - T == 0 is an empty batch: a call with a valid config returns MOE_OK and
 *     touches none of its pointers.
 *   - Host-side validation happens before any launch and returns an error code
 *     with nothing enqueued.  A failed launch returns MOE_ERR_CUDA.  Device-side
 *     checks (index bounds, pipeline wait limits) set a device error word that
 *     moe_check_errors reports.
 *   - Rows: x_perm and y_perm hold at most T*k_max rows (an upper bound known on
 *     the host); the number actually kept, R = offsets[E], stays on the device
 *     and the kernels read it there, so no call needs a device-to-host copy.
 *   - Per-device state: on its first call on a device the library looks up
 *     the device addresses of its error word and static scratch and raises
 *     its kernels' shared-memory limits, and keeps them for the life of the
 *     process (host threads may make those first calls concurrently).
 *     cudaDeviceReset destroys this state together with the device's context:
 *     make no further calls on a device after resetting it.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,  /* a null pointer, a size out of range, k_max > E, ... */
  MOE_ERR_UNSUPPORTED = -2,  /* a valid but unsupported combination (dtype, shape) */
  MOE_ERR_WORKSPACE = -3,    /* workspace missing or smaller than moe_workspace_size */
  MOE_ERR_ALIGNMENT = -4,    /* a pointer or a row size breaks the 16-byte rule */
  MOE_ERR_CUDA = -5,         /* a CUDA runtime call or a launch failed */
  MOE_ERR_DEVICE_CHECK = -6  /* moe_check_errors: a device-side check fired */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Gating modes.
 *  MOE_TOPK_SOFTMAX:        select the k_t largest logits; weights are the
 *                           softmax over the selected logits.
 *  MOE_SOFTMAX_TOPK_RENORM: p = softmax over all E logits; select the k_t
 *                           largest p; weights p_j / sum of the selected p.
 *                           (Selection is taken on the logits: softmax is
 *                           monotone, so the selected set is the same.)
 *  MOE_SIGMOID_GROUPED:     s_e = sigmoid(logit_e), u_e = s_e + sel_bias_e;
 *                           experts form n_groups contiguous groups; a group's
 *                           score is the sum of its group_score_topk largest u;
 *                           keep the topk_groups best groups; select the k_t
 *                           largest u inside kept groups; weights
 *                           routed_scale * s_j / sum of the selected s.
 * Every ranking breaks ties toward the lower expert (or group) index.  The
 * sigmoid is a fully specified fp32 function (Cody-Waite reduction, degree-7
 * Taylor polynomial, Horner with fused multiply-adds) so that selection is
 * reproducible bit for bit on any IEEE machine. */
typedef enum {
  MOE_TOPK_SOFTMAX = 0,
  MOE_SOFTMAX_TOPK_RENORM = 1,
  MOE_SIGMOID_GROUPED = 2
} moe_gating;

typedef struct {
  int32_t T;                /* tokens, >= 0 */
  int32_t d;                /* hidden size */
  int32_t E;                /* routed experts, 1..1024 */
  int32_t k_max;            /* slots per token, 1..min(E, 32) */
  int32_t f;                /* routed expert intermediate size */
  int32_t f_shared;         /* shared expert intermediate size; 0 = no shared expert */
  int32_t dtype;            /* moe_dtype: storage type of x, weights and outputs */
  int32_t gating;           /* moe_gating */
  float capacity_factor;    /* > 0: C = ceil(cf * sum_t k_t / E) in double; <= 0: no limit */
  int32_t n_groups;         /* MOE_SIGMOID_GROUPED only: E % n_groups == 0 */
  int32_t topk_groups;      /* MOE_SIGMOID_GROUPED only: 1..n_groups */
  int32_t group_score_topk; /* MOE_SIGMOID_GROUPED only: 1..E/n_groups */
  float routed_scale;       /* MOE_SIGMOID_GROUPED only: multiplies the weights */
} moe_config;

/* Routing results (all DEVICE pointers, caller-owned; sizes in elements).
 * Slots are (t, j) with 0 <= j < k_max; slot a = t*k_max + j.
 *   logits   [T*E]      fp32 router logits
 *   topk_idx [T*k_max]  j-th best expert of token t; -1 for j >= k_t
 *   topk_w   [T*k_max]  combine weight of the slot (0 for j >= k_t); weights
 *                       of dropped slots are kept as computed (the slot is
 *                       skipped by combine, not renormalised away)
 *   counts   [E]        assignments per expert before capacity
 *   kept     [E]        min(counts[e], C)
 *   offsets  [E+1]      exclusive prefix sum of kept; R = offsets[E]
 *   slot_row [T*k_max]  row of a kept slot in x_perm/y_perm, -1 when dropped or padding
 *   row_src  [T*k_max]  first R entries: slot a = t*k_max+j of each row; rows of
 *                       expert e are offsets[e]..offsets[e+1]-1, in (t, j) order;
 *                       slots are admitted per expert in (t, j) order, first C kept
 *   n_dropped [1]       sum over e of counts[e] - kept[e] */
typedef struct {
  float *logits;
  int32_t *topk_idx;
  float *topk_w;
  int32_t *counts;
  int32_t *kept;
  int32_t *offsets;
  int32_t *slot_row;
  int32_t *row_src;
  int32_t *n_dropped;
} moe_route_out;

/* Which call a workspace is sized for. */
typedef enum {
  MOE_WS_ROUTE = 0,       /* moe_route */
  MOE_WS_EXPERT_FFN = 1,  /* moe_expert_ffn */
  MOE_WS_LAYER = 2        /* moe_layer (covers the other two as well) */
} moe_ws_kind;

/* Host-only: bytes of workspace `kind` needs for cfg.  Touches no device. */
MOE_API moe_status moe_workspace_size(const moe_config *cfg, int32_t kind, size_t *bytes);

/* Steps 1-3.  x [T,d], Wr [d,E] in cfg->dtype; logit_bias [E] fp32 or NULL;
 * sel_bias [E] fp32 or NULL (MOE_SIGMOID_GROUPED); k_per_token [T] int32 in
 * [1, k_max] or NULL (k_t = k_max).  Every field of `out` must be set.
 * ws: at least moe_workspace_size(cfg, MOE_WS_ROUTE) bytes. */
MOE_API moe_status moe_route(const moe_config *cfg, const void *x, const void *Wr,
                     const float *logit_bias, const float *sel_bias,
                     const int32_t *k_per_token, const moe_route_out *out, void *ws,
                     size_t ws_bytes, void *stream);

/* moe_route without a workspace argument, for callers that cannot give this
 * library scratch memory (a plugin interface that passes only inputs and
 * outputs, a runtime whose device memory is fully planned in advance, a path
 * that must not call an allocator).  The pages have no counterpart: this is
 * an interface convenience, not a step of the method.  Results are those of
 * moe_route.  The routing step's scratch lives in a fixed 1 MiB device array
 * inside this library, held on every GPU that loads it until exit.  That
 * scratch is the capacity step's 8 * ceil(T*k_max/1024) * E bytes (rounded up
 * to a multiple of 256, plus 256), or, for bf16 layers with E % 8 == 0 and
 * T <= 128, the split-K router's partial logits (at most 768 KiB) plus 256
 * bytes.  A configuration that needs more than the array is rejected with
 * MOE_ERR_WORKSPACE before anything is enqueued.  No
 * call allocates or frees memory.  The first call on a device looks up the
 * array's device address with that device current.  All calls share the
 * array, so calls whose work overlaps on the GPU (other streams or host
 * threads on the same device) race; serialise them. */
MOE_API moe_status moe_route_static_scratch(const moe_config *cfg, const void *x,
                                            const void *Wr, const float *logit_bias,
                                            const float *sel_bias, const int32_t *k_per_token,
                                            const moe_route_out *out, void *stream);

/* Step 4.  x [T,d] -> x_perm [T*k_max, d]: x_perm[r] = x[row_src[r] / k_max]
 * for r < offsets[E]; rows past R are left untouched. */
MOE_API moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *offsets,
                        const int32_t *row_src, void *x_perm, void *stream);

/* Step 5.  Grouped SwiGLU over expert-contiguous rows: rows offsets[e] ..
 * offsets[e+1]-1 of x_perm [>= R, d] use expert e.  W1, W3 [E,d,f] and
 * W2 [E,f,d] in cfg->dtype; y_perm [T*k_max, d] fp32.  The intermediate
 * silu(x.W1)*(x.W3) is stored in the workspace (bf16 for bf16 layers, fp32 for
 * fp32 layers); accumulation is fp32.  ws: moe_workspace_size(cfg,
 * MOE_WS_EXPERT_FFN). */
MOE_API moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                          const void *W1, const void *W3, const void *W2, void *y_perm,
                          void *ws, size_t ws_bytes, void *stream);

/* Step 6.  out [T,d] = sum over j < k_max with slot_row >= 0 of
 * topk_w[t,j] * y_perm[slot_row[t,j]] (+ shared_y[t] when shared_y is not NULL;
 * y_perm [>= R, d] and shared_y [T, d] are fp32),
 * accumulated in fp32 and rounded once to cfg->dtype.  A token whose slots are
 * all dropped gets 0 (+ shared_y[t]). */
MOE_API moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *slot_row,
                       const float *topk_w, const void *shared_y, void *out, void *stream);

/* The whole layer, steps 1-6, plus the always-on shared expert when
 * cfg->f_shared > 0 (Ws1, Ws3 [d,f_shared], Ws2 [f_shared,d]; NULL otherwise),
 * whose output is added with weight 1.  route_out may be NULL (routing then
 * lives in the workspace) or name caller buffers to receive the routing.
 * ws: at least moe_workspace_size(cfg, MOE_WS_LAYER) bytes. */
MOE_API moe_status moe_layer(const moe_config *cfg, const void *x, const void *Wr,
                     const float *logit_bias, const float *sel_bias,
                     const int32_t *k_per_token, const void *W1, const void *W3,
                     const void *W2, const void *Ws1, const void *Ws3, const void *Ws2,
                     void *out, const moe_route_out *route_out, void *ws, size_t ws_bytes,
                     void *stream);

/* moe_layer, plus stage timing: events[i] (cudaEvent_t handles created by
 * the caller; NULL entries skipped, i < n_events) is recorded on `stream` at
 * stage boundary i:
 *   0 before the router           1 after routing (router, gating, capacity)
 *   2 after dispatch              3 after the up projection with SwiGLU (K5)
 *   4 after the down projection   5 after the shared expert (= 4 without one)
 *   6 after combine
 * For fp32 layers both projections run before boundary 3.  The kernels and
 * results are those of moe_layer; this call exists for profiling. */
MOE_API moe_status moe_layer_timed(const moe_config *cfg, const void *x, const void *Wr,
                                   const float *logit_bias, const float *sel_bias,
                                   const int32_t *k_per_token, const void *W1, const void *W3,
                                   const void *W2, const void *Ws1, const void *Ws3,
                                   const void *Ws2, void *out, const moe_route_out *route_out,
                                   void *ws, size_t ws_bytes, void *stream,
                                   void *const *events, int32_t n_events);

/* ---- FP8 expert weights ----------------------------------------------------
 * "LLM MoE Expert Parallel 生产实战" serves DeepSeek-V3 with fp8 quantisation
 * (section 5) and warns to check that it leaves the router head alone
 * (section 10).  Here the experts' matrices, routed and shared, are e4m3
 * codes (OCP FP8 E4M3, the finite-only variant: bias 7, 3 fraction bits,
 * largest magnitude 448) with one fp32 scale per output column: the weight
 * the layer computes with is e4m3_value(code) * scale[column].  The router
 * weights, activations and outputs stay in the layer dtype, which must be
 * MOE_BF16; d, f and f_shared must be multiples of 16.  The codes are stored
 * transposed, K contiguous (one byte each): the codes of one output column
 * of the bf16 matrix [G, K, N] are the contiguous row [g, n, :] -- the order
 * in which the GEMMs widen them.  moe_quantize_fp8 writes this layout.
 * Every pointer is a device pointer, 16-byte aligned, owned by the caller. */
typedef struct {
  const void *W1, *W3;  /* [G, f, d] e4m3 codes of the [G, d, f] matrices */
  const void *W2;       /* [G, d, f] e4m3 codes of the [G, f, d] matrix */
  const float *s1, *s3; /* [G, f] column scales of W1, W3 */
  const float *s2;      /* [G, d] column scales of W2 */
} moe_fp8_weights;

/* Weight preparation (not a hot call): W [G, K, N] bf16 -> Wq [G, N, K] e4m3
 * codes (transposed) and scale [G, N], with scale = max_k |W[g,k,n]| / 448
 * (fp32 division; 1 for an all-zero column) and Wq[g,n,k] = e4m3(W[g,k,n] /
 * scale[g,n]) of the fp32 quotient, rounded to nearest even, saturating at
 * 448.  K and N multiples of 16. */
MOE_API moe_status moe_quantize_fp8(const void *W, int32_t G, int32_t K, int32_t N, void *Wq,
                                    float *scale, void *stream);

/* moe_expert_ffn with fp8 expert weights w (G = E).  ws: moe_workspace_size(
 * cfg, MOE_WS_EXPERT_FFN). */
MOE_API moe_status moe_expert_ffn_fp8(const moe_config *cfg, const void *x_perm,
                                      const int32_t *offsets, const moe_fp8_weights *w,
                                      void *y_perm, void *ws, size_t ws_bytes, void *stream);

/* moe_layer with fp8 expert weights: `experts` (G = E) and, when
 * cfg->f_shared > 0, `shared` (G = 1, f = f_shared; NULL otherwise).  Wr
 * stays in cfg->dtype.  events / n_events as in moe_layer_timed (NULL / 0:
 * none).  ws: moe_workspace_size(cfg, MOE_WS_LAYER). */
MOE_API moe_status moe_layer_fp8(const moe_config *cfg, const void *x, const void *Wr,
                                 const float *logit_bias, const float *sel_bias,
                                 const int32_t *k_per_token, const moe_fp8_weights *experts,
                                 const moe_fp8_weights *shared, void *out,
                                 const moe_route_out *route_out, void *ws, size_t ws_bytes,
                                 void *stream, void *const *events, int32_t n_events);

/* ---- Expert parallelism ----------------------------------------------------
 * "Expert Parallelism: MoE 模型的并行切分" (SGLang learning notes), sections
 * 3 and 8, and "LLM MoE Expert Parallel 生产实战", steps 2 and 4: the E
 * experts are split over n_ranks ranks (rank r owns experts
 * [r*E/n_ranks, (r+1)*E/n_ranks)); every rank routes its own T tokens, sends
 * each kept row to the rank that owns its expert (dispatch), runs its own
 * experts on the rows it received, and sends every result back to the rank
 * and row it came from (combine), where the weighted combine runs as usual.
 *
 * The exchange is done by stores straight into the destination rank's
 * buffers (peer pointers: another GPU's memory mapped into this one over
 * NVLink, or -- when the ranks are emulated on one GPU -- plain pointers into
 * that GPU's memory); no rows are staged and the host never reads a count.
 * Every rank needs the kept-row counts of all ranks first, counts_all
 * [n_ranks][E] int32 on its device (rank s's row = its moe_route `kept`,
 * gathered by the caller, e.g. an all-gather), and the caller orders the
 * steps across ranks (the destination buffers must be free before a
 * dispatch, and a rank may read what it received only after every sender
 * finished: a barrier after each exchange).
 *
 * Receive layout on rank r: its experts' rows grouped by expert (ascending),
 * inside an expert by source rank (ascending), inside a source in the
 * source's own row order.  recv_offsets [E/n_ranks + 1] (from
 * moe_ep_plan) delimits the experts, so the received rows feed
 * moe_expert_ffn with E/n_ranks experts directly.  The returned rows land in
 * the source rank's y_back [T*k_max, d] fp32 at the rows of its own
 * dispatch layout, which moe_combine reads through slot_row.
 * n_ranks divides E; 1 <= n_ranks <= 8. */
#define MOE_EP_MAX_RANKS 8
typedef struct {
  int32_t rank;
  int32_t n_ranks;
  const int32_t *counts_all;              /* device [n_ranks][E] */
  void *recv_rows[MOE_EP_MAX_RANKS];      /* per rank: its received rows [n_ranks*T*k_max, d], cfg->dtype */
  float *y_back[MOE_EP_MAX_RANKS];        /* per rank: its returned rows [T*k_max, d] fp32 */
} moe_ep_ranks;

/* This rank's part of the exchange plan, from counts_all (device work, on
 * `stream`): recv_offsets [E/n_ranks + 1] int32 (rows received per local
 * expert, prefix summed), and send_base [E] int32 (for each expert e, the
 * row of the owner's receive buffer where this rank's rows of e start).
 * Both are device buffers owned by the caller. */
MOE_API moe_status moe_ep_plan(const moe_config *cfg, const moe_ep_ranks *ep,
                               int32_t *recv_offsets, int32_t *send_base, void *stream);

/* Dispatch: every kept row of this rank (offsets, row_src, topk_idx of its
 * moe_route) goes from the token rows x [T, d] to row
 * send_base[e] + (its index among this rank's rows of e) of the owner's
 * recv_rows. */
MOE_API moe_status moe_ep_dispatch(const moe_config *cfg, const moe_ep_ranks *ep,
                                   const void *x, const int32_t *offsets, const int32_t *row_src,
                                   const int32_t *topk_idx, const int32_t *send_base,
                                   void *stream);

/* Combine exchange: every received row's expert output (y_recv [n_ranks*T*
 * k_max, d] fp32, from moe_expert_ffn over this rank's experts) goes back to
 * its source rank's y_back, at the row the source's own dispatch layout
 * gave it. */
MOE_API moe_status moe_ep_return(const moe_config *cfg, const moe_ep_ranks *ep,
                                 const float *y_recv, const int32_t *recv_offsets, void *stream);

/* Host-only mirror of the plan (touches no device): from counts_all
 * [n_ranks][E] in host memory, rank `rank`'s recv_offsets [E/n_ranks + 1] and
 * send_base [E], and for every row p it receives (p < recv_offsets[E/n_ranks]
 * <= max_recv) the source rank recv_src[p] and the row recv_src_row[p] of the
 * source's own layout that it returns to.  For schedulers and tests that
 * check the exchange layout on the host. */
MOE_API moe_status moe_ep_plan_host(int32_t n_ranks, int32_t E, int32_t rank,
                                    const int32_t *counts_all, int32_t *recv_offsets,
                                    int32_t *send_base, int32_t *recv_src, int32_t *recv_src_row,
                                    int32_t max_recv);

/* Synchronises `stream`, then reads and clears the device error flags of the
 * current device.  *flags (may be NULL) receives them: bit 0 an index out of
 * range in a gather/scatter, bit 1 a pipeline wait that hit its time limit,
 * bit 2 an expert index or k_t out of range.  Returns MOE_ERR_DEVICE_CHECK
 * when any flag was set.
 * Time limit: every wait of the tensor-core GEMMs' pipelines (on data landing
 * in shared memory, on a free accumulator, ...) gives up after 4 s; the CTA
 * then sets bit 1, stops its other roles, lets the copies and MMAs it already
 * issued complete, frees its tensor memory and returns, so a stalled pipeline
 * ends the kernel instead of hanging the GPU.  The results of that call are
 * then undefined.  The environment variable MOE_WAIT_LIMIT_NS, read at every
 * launch, lowers the limit of the single-CTA and swap-AB engines (nanoseconds,
 * at most 4e9) -- a diagnostic that makes the waits run out on purpose; the
 * CTA-pair engine always keeps 4 s. */
MOE_API moe_status moe_check_errors(void *stream, uint32_t *flags);

/* Static description of a status code. */
MOE_API const char *moe_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
