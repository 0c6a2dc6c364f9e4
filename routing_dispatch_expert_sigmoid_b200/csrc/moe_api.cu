// The C ABI of include/moe.h: host-side validation, workspace layout and the
// order of launches.  Every call validates its arguments on the host before
// anything is enqueued; no call allocates, frees or synchronises (except
// moe_check_errors, whose job is to synchronise).
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "moe_internal.cuh"

namespace moe {

__device__ uint32_t g_moe_error_word;

// Device address of a file-scope __device__ symbol on the current device,
// looked up with that device current on its first use and cached per device.
// The slots are atomics: host threads making a device's first call at the
// same time each look the address up and store the same value, without a
// data race.
void *symbol_address_cached(std::atomic<void *> (&cache)[64], const void *symbol) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void *p = cache[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}

uint32_t *device_error_word() {
  static std::atomic<void *> addr[64];
  return static_cast<uint32_t *>(symbol_address_cached(addr, &g_moe_error_word));
}

bool pdl_enabled() {
  const char *v = getenv("MOE_PDL");  // read per launch, like the other switches
  return !(v && v[0] == '0');
}

namespace {

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

size_t esize(const moe_config &c) { return c.dtype == MOE_F32 ? 4 : 2; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status check_config(const moe_config *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d <= 0 || c->f <= 0 || c->f_shared < 0) return MOE_ERR_INVALID_ARG;
  if (c->E < 1 || c->E > 1024) return MOE_ERR_INVALID_ARG;
  if (c->k_max < 1 || c->k_max > c->E || c->k_max > 32) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c->gating < MOE_TOPK_SOFTMAX || c->gating > MOE_SIGMOID_GROUPED) return MOE_ERR_UNSUPPORTED;
  if ((long long)c->T * c->k_max > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  const int q = c->dtype == MOE_F32 ? 4 : 8;  // elements per 16 bytes
  if (c->d % q || c->f % q || c->f_shared % q) return MOE_ERR_ALIGNMENT;
  if (c->gating == MOE_SIGMOID_GROUPED) {
    if (c->n_groups < 1 || c->n_groups > 32 || c->E % c->n_groups) return MOE_ERR_INVALID_ARG;
    const int gsz = c->E / c->n_groups;
    if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return MOE_ERR_INVALID_ARG;
    if (c->group_score_topk < 1 || c->group_score_topk > gsz) return MOE_ERR_INVALID_ARG;
    if (c->group_score_topk > 8) return MOE_ERR_UNSUPPORTED;
    if (c->k_max > c->topk_groups * gsz) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// Workspace regions, each 256-byte aligned.
struct Layout {
  size_t logits, topk_idx, topk_w, counts, kept, offsets, slot_row, row_src, n_dropped;
  size_t cap_scratch, x_perm, h, y_perm, h_sh, y_sh, sh_part;
  size_t f8_xplanes, f8_hplanes, f8_scales;  // fp8 weights, decode-sized batches
  size_t total;
};

// Bytes of rows of d values in the y16 form: the fp16 values, then (256-byte
// aligned) one exponent byte per 32-column block of each row.
size_t y16_exp_offset(size_t rows, int d) { return up(rows * d * 2); }
size_t y16_bytes(size_t rows, int d) { return y16_exp_offset(rows, d) + rows * ((d + 31) / 32); }

// Decode-sized bf16 layers (at most 32 rows per expert on average) whose
// rows are whole 16-byte steps of e4m3 codes can run fp8 expert weights on
// the kind::f8f6f4 engine; their workspace holds the activation planes.
bool f8_planes_fit(const moe_config &c) {
  return c.dtype == MOE_BF16 && c.d % 16 == 0 && c.f % 16 == 0 &&
         (long long)c.T * c.k_max <= 32LL * c.E;
}

Layout layout(const moe_config &c, int kind) {
  Layout L{};
  size_t o = 0;
  const size_t slots = (size_t)c.T * c.k_max, s = esize(c);
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up(bytes);
    return at;
  };
  if (kind == MOE_WS_LAYER) {
    L.logits = take(sizeof(float) * (size_t)c.T * c.E);
    L.topk_idx = take(sizeof(int32_t) * slots);
    L.topk_w = take(sizeof(float) * slots);
    L.counts = take(sizeof(int32_t) * c.E);
    L.kept = take(sizeof(int32_t) * c.E);
    L.offsets = take(sizeof(int32_t) * (c.E + 1));
    L.slot_row = take(sizeof(int32_t) * slots);
    L.row_src = take(sizeof(int32_t) * slots);
    L.n_dropped = take(sizeof(int32_t));
  }
  if (kind == MOE_WS_LAYER || kind == MOE_WS_ROUTE) L.cap_scratch = take(route_scratch_bytes(c));
  if (kind == MOE_WS_LAYER) L.x_perm = take(slots * c.d * s);
  if (kind == MOE_WS_LAYER || kind == MOE_WS_EXPERT_FFN) L.h = take(slots * c.f * s);
  if (kind == MOE_WS_LAYER) {
    // fp32 rows (the combine rounds once), or their compact y16 form (fp16
    // values, one exponent byte per 32-column block)
    L.y_perm = take(std::max(slots * c.d * sizeof(float), y16_bytes(slots, c.d)));
    if (c.f_shared > 0) {
      L.h_sh = take((size_t)c.T * c.f_shared * s);
      L.y_sh = take((size_t)c.T * c.d * sizeof(float));
      const size_t part = shared_split_bytes(c);  // decode-sized batches only
      if (part) L.sh_part = take(part);
    }
  }
  if ((kind == MOE_WS_LAYER || kind == MOE_WS_EXPERT_FFN) && f8_planes_fit(c)) {
    // x's planes: the layer's x_perm region has exactly their size
    if (kind == MOE_WS_EXPERT_FFN) L.f8_xplanes = take(fp8_planes_bytes((int)slots, c.d));
    L.f8_hplanes = take(fp8_planes_bytes((int)slots, c.f));
    L.f8_scales = take(2 * sizeof(float) * slots);
  }
  L.total = o;
  return L;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                  \
  do {                                 \
    moe_status _st = (expr);           \
    if (_st != MOE_OK) return _st;     \
  } while (0)

#define MOE_TRY_CUDA(expr)                                  \
  do {                                                      \
    if ((expr) != cudaSuccess) return MOE_ERR_CUDA;         \
  } while (0)

moe_status need(const void *p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  return aligned16(p) ? MOE_OK : MOE_ERR_ALIGNMENT;
}
moe_status need_opt(const void *p) { return (!p || aligned16(p)) ? MOE_OK : MOE_ERR_ALIGNMENT; }
// Index / small fp32 arrays: 4-byte alignment is enough.
moe_status need4(const void *p) {
  if (!p) return MOE_ERR_INVALID_ARG;
  return (reinterpret_cast<uintptr_t>(p) & 3u) ? MOE_ERR_ALIGNMENT : MOE_OK;
}
moe_status need4_opt(const void *p) { return p ? need4(p) : MOE_OK; }

moe_status check_route_out(const moe_route_out *o) {
  if (!o) return MOE_ERR_INVALID_ARG;
  MOE_TRY(need4(o->logits));
  MOE_TRY(need4(o->topk_idx));
  MOE_TRY(need4(o->topk_w));
  MOE_TRY(need4(o->counts));
  MOE_TRY(need4(o->kept));
  MOE_TRY(need4(o->offsets));
  MOE_TRY(need4(o->slot_row));
  MOE_TRY(need4(o->row_src));
  MOE_TRY(need4(o->n_dropped));
  return MOE_OK;
}

moe_status check_ws(const moe_config &c, int kind, void *ws, size_t ws_bytes) {
  const size_t need_bytes = layout(c, kind).total;
  if (need_bytes == 0) return MOE_OK;
  if (!ws || ws_bytes < need_bytes) return MOE_ERR_WORKSPACE;
  return aligned16(ws) ? MOE_OK : MOE_ERR_ALIGNMENT;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

moe_status route_impl(const moe_config &c, const void *x, const void *Wr, const float *logit_bias,
                      const float *sel_bias, const int32_t *k_per_token, const moe_route_out &o,
                      void *cap_scratch, uint32_t *err, cudaStream_t s) {
  // Decode-sized batches: split-K router plus one fused gating/ranking kernel.
  const SmallRoutePlan plan = small_route_plan(c);
  if (plan.use) {
    MOE_TRY_CUDA(launch_route_small(c, plan, x, Wr, logit_bias, sel_bias, k_per_token, o,
                                    cap_scratch, err, s));
    return MOE_OK;
  }
  // The router is a dense contraction: bf16 layers whose logit rows are a
  // multiple of 16 bytes (E % 8 == 0, a TMA stride rule) run it on the tensor
  // cores (its epilogue writes 16-byte vectors, so the logits buffer must be
  // 16-byte aligned too); fp32 layers keep plain fp32 FMA (TF32 would miss
  // the logit tolerance).
  if (c.dtype == MOE_BF16 && c.E % 8 == 0 && aligned16(o.logits)) {
    MOE_TRY_CUDA(launch_router_tc(c.T, c.d, c.E, x, Wr, logit_bias, o.logits, err, s));
  } else {
    MOE_TRY_CUDA(launch_router(c, x, Wr, logit_bias, o.logits, s));
  }
  MOE_TRY_CUDA(launch_gating(c, o.logits, sel_bias, k_per_token, o.topk_idx, o.topk_w, err, s));
  MOE_TRY_CUDA(launch_capacity(c, o.topk_idx, o.counts, o.kept, o.offsets, o.slot_row, o.row_src,
                               o.n_dropped, cap_scratch, err, s));
  return MOE_OK;
}

// Stage events of moe_layer_timed (nullptr entries are skipped).
struct Events {
  cudaEvent_t const *ev = nullptr;
  int n = 0;
  cudaError_t mark(int i, cudaStream_t s) const {
    return (ev && i < n && ev[i]) ? cudaEventRecord(ev[i], s) : cudaSuccess;
  }
};

// One set of expert matrices: in the layer dtype, or e4m3 codes with
// per-column scales (fp8 set).
struct Weights {
  const void *W1 = nullptr, *W3 = nullptr, *W2 = nullptr;
  const float *s1 = nullptr, *s3 = nullptr, *s2 = nullptr;
  bool fp8 = false;
};
Weights plain_weights(const void *W1, const void *W3, const void *W2) {
  Weights w;
  w.W1 = W1;
  w.W3 = W3;
  w.W2 = W2;
  return w;
}
Weights fp8_weights(const moe_fp8_weights &q) {
  Weights w;
  w.W1 = q.W1;
  w.W3 = q.W3;
  w.W2 = q.W2;
  w.s1 = q.s1;
  w.s3 = q.s3;
  w.s2 = q.s2;
  w.fp8 = true;
  return w;
}
moe_status check_weights(const Weights &w) {
  MOE_TRY(need(w.W1));
  MOE_TRY(need(w.W3));
  MOE_TRY(need(w.W2));
  if (w.fp8) {  // the scales are read as float4 vectors
    MOE_TRY(need(w.s1));
    MOE_TRY(need(w.s3));
    MOE_TRY(need(w.s2));
  }
  return MOE_OK;
}
// Layers with fp8 weights: bf16 activations, rows of codes in 16-byte steps.
moe_status check_fp8_config(const moe_config &c) {
  if (c.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c.d % 16 || c.f % 16 || c.f_shared % 16) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

// Routed experts (G = E groups over rows_cap rows) or the shared expert
// (offsets == nullptr: one group of T rows).  `mid` is recorded between the
// up projection (with SwiGLU) and the down projection.  With row_src, A is
// the token rows x and the up projection gathers its rows itself.
// gate_w / gate_src (routed experts, bf16 layers): the down projection
// multiplies output row r by gate_w[gate_src[r]], its slot's gate weight.
moe_status ffn_impl(const moe_config &c, int G, const int32_t *offsets, int fixed_rows,
                    int rows_cap, int f, const void *A, const Weights &w, void *h, void *y,
                    uint32_t *err, cudaStream_t s, const Events &ev = Events(), int mid = -1,
                    const int32_t *row_src = nullptr, const float *gate_w = nullptr,
                    const int32_t *gate_src = nullptr, int8_t *yexp = nullptr) {
  if (w.fp8) {
    MOE_TRY_CUDA(launch_grouped_gemm_fp8(true, rows_cap, c.d, f, G, offsets, fixed_rows, A, w.W1,
                                         w.W3, w.s1, w.s3, h, err, s));
    MOE_TRY_CUDA(ev.mark(mid, s));
    MOE_TRY_CUDA(launch_grouped_gemm_fp8(false, rows_cap, f, c.d, G, offsets, fixed_rows, h,
                                         w.W2, nullptr, w.s2, nullptr, y, err, s, gate_w,
                                         gate_src));
    return MOE_OK;
  }
  if (c.dtype == MOE_F32) {
    MOE_TRY_CUDA(launch_ffn_simt_f32(
        rows_cap, c.d, f, G, offsets, fixed_rows, static_cast<const float *>(A),
        static_cast<const float *>(w.W1), static_cast<const float *>(w.W3),
        static_cast<const float *>(w.W2), static_cast<float *>(h), static_cast<float *>(y), s));
    MOE_TRY_CUDA(ev.mark(mid, s));
    return MOE_OK;
  }
  MOE_TRY_CUDA(launch_grouped_gemm_bf16(true, rows_cap, c.d, f, G, offsets, fixed_rows, A, w.W1,
                                        w.W3, h, err, s, row_src, c.k_max, c.T));
  MOE_TRY_CUDA(ev.mark(mid, s));
  MOE_TRY_CUDA(launch_grouped_gemm_bf16(false, rows_cap, f, c.d, G, offsets, fixed_rows, h, w.W2,
                                        nullptr, y, err, s, nullptr, 1, 0, gate_w, gate_src,
                                        yexp));
  return MOE_OK;
}

// The gate weights can be applied by the down projection's epilogue (each
// row of y_perm scaled by its slot's weight), leaving the combine a plain
// sum of the kept rows.  MOE_WEIGHTS_IN_GEMM=1 selects it for bf16 layers;
// by default the combine applies them.
bool weights_in_gemm(const moe_config &c) {
  const char *env = getenv("MOE_WEIGHTS_IN_GEMM");
  return c.dtype == MOE_BF16 && env && env[0] == '1';
}

// The routed experts' outputs of bf16 layers travel from the down projection
// to the combine in the compact y16 form (half the bytes of fp32 rows, a
// relative error of at most 2^-11 per value) when the down projection's
// engine writes it; MOE_Y16=0 keeps fp32 rows.
bool use_y16(const moe_config &c, int rows_cap, const int32_t *offsets) {
  const char *env = getenv("MOE_Y16");
  if (env && env[0] == '0') return false;
  return c.dtype == MOE_BF16 && grouped_gemm_y16_out(rows_cap, c.E, offsets, 0, c.d);
}

// The dispatch copy can be fused into the up projection (bf16 layers, engines
// that gather): the GEMM's producer fetches the token rows with TMA gather4.
// Measured on B200 it is slower for prefill-sized groups (a 128-row A tile
// needs 32 gather4 operations per k-block instead of one tiled load: Mixtral
// up projection 9.7 vs 3.7 ms) and neutral for decode, so the separate
// dispatch kernel is the default; MOE_FUSED_DISPATCH=1 selects the fusion.
bool fuse_dispatch(const moe_config &c, int rows_cap, const int32_t *offsets) {
  const char *env = getenv("MOE_FUSED_DISPATCH");
  if (!env || env[0] != '1') return false;
  return c.dtype == MOE_BF16 && grouped_gemm_can_gather(true, rows_cap, c.E, offsets, 0);
}

// fp8 weights of decode-sized layers run on the kind::f8f6f4 engine unless
// MOE_GEMM_ENGINE names one of the widening engines (single, narrow, swap).
bool use_f8_engine(const moe_config &c) {
  if (!f8_planes_fit(c)) return false;
  const char *env = getenv("MOE_GEMM_ENGINE");
  return !env || !*env || env[0] == 'f';
}

// The routed experts' FFN on fp8 weights through the kind::f8f6f4 engine:
// the rows' activation planes (gathered from the token rows A when row_src is
// given -- the dispatch step of the layer), the up projection with SwiGLU,
// the planes of h, the down projection.  Events: mark_rows after the first
// planes, mark_up after the up projection.
moe_status ffn_f8_impl(const moe_config &c, const int32_t *offsets, const void *A,
                       const int32_t *row_src, int a_rows, const Weights &w, uint8_t *xplanes,
                       uint8_t *hplanes, float *scales, void *h, void *y, uint32_t *err,
                       cudaStream_t s, const Events &ev = Events(), int mark_rows = -1,
                       int mark_up = -1, const float *gate_w = nullptr,
                       const int32_t *gate_src = nullptr) {
  const int rows_cap = c.T * c.k_max;
  float *xs = scales, *hs = scales + rows_cap;
  MOE_TRY_CUDA(launch_split_planes(A, offsets + c.E, 0, row_src, c.k_max, a_rows, rows_cap, c.d,
                                   xplanes, xs, err, s));
  MOE_TRY_CUDA(ev.mark(mark_rows, s));
  MOE_TRY_CUDA(launch_grouped_gemm_f8(true, rows_cap, c.d, c.f, c.E, offsets, xplanes, xs, w.W1,
                                      w.W3, w.s1, w.s3, h, err, s));
  MOE_TRY_CUDA(ev.mark(mark_up, s));
  MOE_TRY_CUDA(launch_split_planes(h, offsets + c.E, 0, nullptr, 1, rows_cap, rows_cap, c.f,
                                   hplanes, hs, err, s));
  MOE_TRY_CUDA(launch_grouped_gemm_f8(false, rows_cap, c.f, c.d, c.E, offsets, hplanes, hs, w.W2,
                                      nullptr, w.s2, nullptr, y, err, s, gate_w, gate_src));
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

static moe_status layer_impl(const moe_config *cfg, const void *x, const void *Wr,
                             const float *logit_bias, const float *sel_bias,
                             const int32_t *k_per_token, const Weights &we, const Weights &wsh,
                             void *out, const moe_route_out *route_out, void *ws, size_t ws_bytes,
                             void *stream, const Events &ev) {
  MOE_TRY(check_config(cfg));
  if (we.fp8) MOE_TRY(check_fp8_config(*cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  const moe_config &c = *cfg;
  MOE_TRY(need(x));
  MOE_TRY(need(Wr));
  MOE_TRY(need4_opt(logit_bias));
  MOE_TRY(need4_opt(sel_bias));
  MOE_TRY(need4_opt(k_per_token));
  MOE_TRY(check_weights(we));
  if (c.f_shared > 0) MOE_TRY(check_weights(wsh));
  MOE_TRY(need(out));
  if (route_out) MOE_TRY(check_route_out(route_out));
  MOE_TRY(check_ws(c, MOE_WS_LAYER, ws, ws_bytes));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Layout L = layout(c, MOE_WS_LAYER);
  moe_route_out r;
  if (route_out) {
    r = *route_out;
  } else {
    r.logits = at<float>(ws, L.logits);
    r.topk_idx = at<int32_t>(ws, L.topk_idx);
    r.topk_w = at<float>(ws, L.topk_w);
    r.counts = at<int32_t>(ws, L.counts);
    r.kept = at<int32_t>(ws, L.kept);
    r.offsets = at<int32_t>(ws, L.offsets);
    r.slot_row = at<int32_t>(ws, L.slot_row);
    r.row_src = at<int32_t>(ws, L.row_src);
    r.n_dropped = at<int32_t>(ws, L.n_dropped);
  }
  MOE_TRY_CUDA(ev.mark(0, s));
  MOE_TRY(route_impl(c, x, Wr, logit_bias, sel_bias, k_per_token, r, at<void>(ws, L.cap_scratch),
                     err, s));
  MOE_TRY_CUDA(ev.mark(1, s));
  const int rows_cap = c.T * c.k_max;
  void *x_perm = at<void>(ws, L.x_perm), *y_perm = at<void>(ws, L.y_perm);
  const bool wig = weights_in_gemm(c);
  int8_t *yexp = (!we.fp8 && use_y16(c, rows_cap, r.offsets))
                     ? at<int8_t>(ws, L.y_perm + y16_exp_offset((size_t)rows_cap, c.d))
                     : nullptr;
  const float *gate_w = wig ? r.topk_w : nullptr;
  const int32_t *gate_src = wig ? r.row_src : nullptr;
  if (we.fp8 && use_f8_engine(c)) {
    // dispatch = the planes of the gathered token rows (in the x_perm region)
    MOE_TRY(ffn_f8_impl(c, r.offsets, x, r.row_src, c.T, we, static_cast<uint8_t *>(x_perm),
                        at<uint8_t>(ws, L.f8_hplanes), at<float>(ws, L.f8_scales),
                        at<void>(ws, L.h), y_perm, err, s, ev, 2, 3, gate_w, gate_src));
  } else if (!we.fp8 && fuse_dispatch(c, rows_cap, r.offsets)) {
    MOE_TRY_CUDA(ev.mark(2, s));
    MOE_TRY(ffn_impl(c, c.E, r.offsets, 0, rows_cap, c.f, x, we, at<void>(ws, L.h), y_perm, err,
                     s, ev, 3, r.row_src, gate_w, gate_src, yexp));
  } else {
    // long batches: walked by token, so that each row of x leaves HBM once
    // (MOE_DISPATCH_BY_ROW=1 keeps the walk by destination row)
    const char *byrow = getenv("MOE_DISPATCH_BY_ROW");
    if (c.T >= 1024 && !(byrow && byrow[0] == '1'))
      MOE_TRY_CUDA(launch_dispatch_by_token(c, x, r.slot_row, x_perm, err, s));
    else
      MOE_TRY_CUDA(launch_dispatch(c, x, r.offsets, r.row_src, x_perm, err, s));
    MOE_TRY_CUDA(ev.mark(2, s));
    MOE_TRY(ffn_impl(c, c.E, r.offsets, 0, rows_cap, c.f, x_perm, we, at<void>(ws, L.h), y_perm,
                     err, s, ev, 3, nullptr, gate_w, gate_src, yexp));
  }
  MOE_TRY_CUDA(ev.mark(4, s));
  const void *shared_y = nullptr;
  int shared_parts = 1;
  if (c.f_shared > 0) {
    const SharedSplitPlan sp = shared_split_plan(c);
    if (sp.use) {
      const float *parts = nullptr;
      MOE_TRY_CUDA(launch_shared_split(c, sp, wsh.fp8, x, wsh.W1, wsh.W3, wsh.W2, wsh.s1, wsh.s3,
                                       wsh.s2, at<void>(ws, L.h_sh), at<float>(ws, L.y_sh),
                                       at<void>(ws, L.sh_part), &parts, &shared_parts, err, s));
      shared_y = parts;
    } else {
      MOE_TRY(ffn_impl(c, 1, nullptr, c.T, c.T, c.f_shared, x, wsh, at<void>(ws, L.h_sh),
                       at<void>(ws, L.y_sh), err, s));
      shared_y = at<void>(ws, L.y_sh);
    }
  }
  MOE_TRY_CUDA(ev.mark(5, s));
  MOE_TRY_CUDA(launch_combine(c, y_perm, r.slot_row, wig ? nullptr : r.topk_w, shared_y, out,
                               err, s, shared_parts, yexp));
  MOE_TRY_CUDA(ev.mark(6, s));
  return MOE_OK;
}

extern "C" {

moe_status moe_workspace_size(const moe_config *cfg, int32_t kind, size_t *bytes) {
  MOE_TRY(check_config(cfg));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  if (kind < MOE_WS_ROUTE || kind > MOE_WS_LAYER) return MOE_ERR_INVALID_ARG;
  *bytes = layout(*cfg, kind).total;
  return MOE_OK;
}

moe_status moe_route(const moe_config *cfg, const void *x, const void *Wr,
                     const float *logit_bias, const float *sel_bias, const int32_t *k_per_token,
                     const moe_route_out *out, void *ws, size_t ws_bytes, void *stream) {
  MOE_TRY(check_config(cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  const moe_config &c = *cfg;
  MOE_TRY(need(x));
  MOE_TRY(need(Wr));
  MOE_TRY(need4_opt(logit_bias));
  MOE_TRY(need4_opt(sel_bias));
  MOE_TRY(need4_opt(k_per_token));
  MOE_TRY(check_route_out(out));
  MOE_TRY(check_ws(c, MOE_WS_ROUTE, ws, ws_bytes));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  const Layout L = layout(c, MOE_WS_ROUTE);
  return route_impl(c, x, Wr, logit_bias, sel_bias, k_per_token, *out, at<void>(ws, L.cap_scratch),
                    err, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Routing without a caller workspace.
//
// Some callers cannot hand this library device memory for scratch: a plugin
// interface whose fixed signature carries only inputs and outputs, a runtime
// with a static memory plan in which every byte of HBM is already assigned
// (weights, caches) and a stray cudaMalloc would fail or fragment the pool, or
// a latency-critical path that must not pay for an allocator call.  For them,
// moe_route_static_scratch keeps the routing step's scratch (per-chunk
// expert histograms and their prefix sums; for decode-sized batches, the
// split-K router's partial logits, at most 768 KiB, and a ticket word) in the
// fixed device array below.
//
// The array is kStaticScratchBytes (1 MiB) on every GPU that loads this
// library, held until the process exits.  In host code its name is only a
// stand-in for the device symbol, so the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current, on the
// first call made on that device.  Every call shares the array: two calls
// whose work overlaps on the GPU (different streams, or different host
// threads on one device) race on it.  Nothing in it needs to start at zero:
// each call writes every scratch element before reading it.
static constexpr size_t kStaticScratchBytes = 1u << 20;
static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

static void *route_scratch_address() {
  static std::atomic<void *> addr[64];
  return moe::symbol_address_cached(addr, g_route_scratch);
}

moe_status moe_route_static_scratch(const moe_config *cfg, const void *x, const void *Wr,
                                    const float *logit_bias, const float *sel_bias,
                                    const int32_t *k_per_token, const moe_route_out *out,
                                    void *stream) {
  MOE_TRY(check_config(cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  const moe_config &c = *cfg;
  MOE_TRY(need(x));
  MOE_TRY(need(Wr));
  MOE_TRY(need4_opt(logit_bias));
  MOE_TRY(need4_opt(sel_bias));
  MOE_TRY(need4_opt(k_per_token));
  MOE_TRY(check_route_out(out));
  if (route_scratch_bytes(c) > kStaticScratchBytes) return MOE_ERR_WORKSPACE;
  void *scratch = route_scratch_address();
  uint32_t *err = device_error_word();
  if (!scratch || !err) return MOE_ERR_CUDA;
  return route_impl(c, x, Wr, logit_bias, sel_bias, k_per_token, *out, scratch, err,
                    static_cast<cudaStream_t>(stream));
}

moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *offsets,
                        const int32_t *row_src, void *x_perm, void *stream) {
  MOE_TRY(check_config(cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  MOE_TRY(need(x));
  MOE_TRY(need4(offsets));
  MOE_TRY(need4(row_src));
  MOE_TRY(need(x_perm));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  return cuda_status(
      launch_dispatch(*cfg, x, offsets, row_src, x_perm, err, static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                          const void *W1, const void *W3, const void *W2, void *y_perm, void *ws,
                          size_t ws_bytes, void *stream) {
  MOE_TRY(check_config(cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  const moe_config &c = *cfg;
  MOE_TRY(need(x_perm));
  MOE_TRY(need4(offsets));
  MOE_TRY(need(W1));
  MOE_TRY(need(W3));
  MOE_TRY(need(W2));
  MOE_TRY(need(y_perm));
  MOE_TRY(check_ws(c, MOE_WS_EXPERT_FFN, ws, ws_bytes));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  const Layout L = layout(c, MOE_WS_EXPERT_FFN);
  const int rows_cap = c.T * c.k_max;
  return ffn_impl(c, c.E, offsets, 0, rows_cap, c.f, x_perm, plain_weights(W1, W3, W2),
                  at<void>(ws, L.h), y_perm, err, static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_ffn_fp8(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                              const moe_fp8_weights *w, void *y_perm, void *ws, size_t ws_bytes,
                              void *stream) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_fp8_config(*cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  const moe_config &c = *cfg;
  if (!w) return MOE_ERR_INVALID_ARG;
  const Weights we = fp8_weights(*w);
  MOE_TRY(need(x_perm));
  MOE_TRY(need4(offsets));
  MOE_TRY(check_weights(we));
  MOE_TRY(need(y_perm));
  MOE_TRY(check_ws(c, MOE_WS_EXPERT_FFN, ws, ws_bytes));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  const Layout L = layout(c, MOE_WS_EXPERT_FFN);
  if (use_f8_engine(c))
    return ffn_f8_impl(c, offsets, x_perm, nullptr, c.T * c.k_max, we,
                       at<uint8_t>(ws, L.f8_xplanes), at<uint8_t>(ws, L.f8_hplanes),
                       at<float>(ws, L.f8_scales), at<void>(ws, L.h), y_perm, err,
                       static_cast<cudaStream_t>(stream));
  return ffn_impl(c, c.E, offsets, 0, c.T * c.k_max, c.f, x_perm, we, at<void>(ws, L.h), y_perm,
                  err, static_cast<cudaStream_t>(stream));
}

moe_status moe_quantize_fp8(const void *W, int32_t G, int32_t K, int32_t N, void *Wq,
                            float *scale, void *stream) {
  if (G < 0 || K < 0 || N < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)G * K * N == 0) return MOE_OK;
  if (N % 16 || K % 16) return MOE_ERR_ALIGNMENT;
  if (G > 65535) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(need(W));
  MOE_TRY(need(Wq));
  MOE_TRY(need(scale));
  return cuda_status(launch_quantize_fp8(G, K, N, W, static_cast<uint8_t *>(Wq), scale,
                                         static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *slot_row,
                       const float *topk_w, const void *shared_y, void *out, void *stream) {
  MOE_TRY(check_config(cfg));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to do, pointers unused
  MOE_TRY(need(y_perm));
  MOE_TRY(need4(slot_row));
  MOE_TRY(need4(topk_w));
  MOE_TRY(need_opt(shared_y));
  MOE_TRY(need(out));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  return cuda_status(launch_combine(*cfg, y_perm, slot_row, topk_w, shared_y, out, err,
                                    static_cast<cudaStream_t>(stream)));
}

moe_status moe_layer(const moe_config *cfg, const void *x, const void *Wr,
                     const float *logit_bias, const float *sel_bias, const int32_t *k_per_token,
                     const void *W1, const void *W3, const void *W2, const void *Ws1,
                     const void *Ws3, const void *Ws2, void *out, const moe_route_out *route_out,
                     void *ws, size_t ws_bytes, void *stream) {
  return layer_impl(cfg, x, Wr, logit_bias, sel_bias, k_per_token, plain_weights(W1, W3, W2),
                    plain_weights(Ws1, Ws3, Ws2), out, route_out, ws, ws_bytes, stream, Events());
}

moe_status moe_layer_timed(const moe_config *cfg, const void *x, const void *Wr,
                           const float *logit_bias, const float *sel_bias,
                           const int32_t *k_per_token, const void *W1, const void *W3,
                           const void *W2, const void *Ws1, const void *Ws3, const void *Ws2,
                           void *out, const moe_route_out *route_out, void *ws, size_t ws_bytes,
                           void *stream, void *const *events, int32_t n_events) {
  if (n_events < 0 || (n_events > 0 && !events)) return MOE_ERR_INVALID_ARG;
  Events ev;
  ev.ev = reinterpret_cast<cudaEvent_t const *>(events);
  ev.n = n_events;
  return layer_impl(cfg, x, Wr, logit_bias, sel_bias, k_per_token, plain_weights(W1, W3, W2),
                    plain_weights(Ws1, Ws3, Ws2), out, route_out, ws, ws_bytes, stream, ev);
}

moe_status moe_layer_fp8(const moe_config *cfg, const void *x, const void *Wr,
                         const float *logit_bias, const float *sel_bias,
                         const int32_t *k_per_token, const moe_fp8_weights *experts,
                         const moe_fp8_weights *shared, void *out,
                         const moe_route_out *route_out, void *ws, size_t ws_bytes, void *stream,
                         void *const *events, int32_t n_events) {
  if (n_events < 0 || (n_events > 0 && !events)) return MOE_ERR_INVALID_ARG;
  if (!experts || (cfg && cfg->f_shared > 0 && !shared)) return MOE_ERR_INVALID_ARG;
  Events ev;
  ev.ev = reinterpret_cast<cudaEvent_t const *>(events);
  ev.n = n_events;
  Weights wsh;
  if (shared) wsh = fp8_weights(*shared);
  wsh.fp8 = true;
  return layer_impl(cfg, x, Wr, logit_bias, sel_bias, k_per_token, fp8_weights(*experts), wsh,
                    out, route_out, ws, ws_bytes, stream, ev);
}

// ---------------------------------------------------------------------------
// Expert parallelism
static moe_status check_ep(const moe_config *cfg, const moe_ep_ranks *ep) {
  MOE_TRY(check_config(cfg));
  if (!ep) return MOE_ERR_INVALID_ARG;
  if (ep->n_ranks < 1 || ep->n_ranks > MOE_EP_MAX_RANKS || cfg->E % ep->n_ranks) return MOE_ERR_INVALID_ARG;
  if (ep->rank < 0 || ep->rank >= ep->n_ranks) return MOE_ERR_INVALID_ARG;
  if ((long long)cfg->T * cfg->k_max * ep->n_ranks > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  return need4(ep->counts_all);
}

moe_status moe_ep_plan(const moe_config *cfg, const moe_ep_ranks *ep, int32_t *recv_offsets,
                       int32_t *send_base, void *stream) {
  MOE_TRY(check_ep(cfg, ep));
  MOE_TRY(need4(recv_offsets));
  MOE_TRY(need4(send_base));
  return cuda_status(launch_ep_plan(ep->counts_all, ep->n_ranks, cfg->E, ep->rank, recv_offsets,
                                    send_base, static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_dispatch(const moe_config *cfg, const moe_ep_ranks *ep, const void *x,
                           const int32_t *offsets, const int32_t *row_src,
                           const int32_t *topk_idx, const int32_t *send_base, void *stream) {
  MOE_TRY(check_ep(cfg, ep));
  if (cfg->T == 0) return MOE_OK;  // empty batch: nothing to send
  MOE_TRY(need(x));
  MOE_TRY(need4(offsets));
  MOE_TRY(need4(row_src));
  MOE_TRY(need4(topk_idx));
  MOE_TRY(need4(send_base));
  for (int r = 0; r < ep->n_ranks; ++r) MOE_TRY(need(ep->recv_rows[r]));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  return cuda_status(launch_ep_dispatch(*cfg, ep->n_ranks, ep->recv_rows, x, offsets, row_src,
                                        topk_idx, send_base, err,
                                        static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_return(const moe_config *cfg, const moe_ep_ranks *ep, const float *y_recv,
                         const int32_t *recv_offsets, void *stream) {
  MOE_TRY(check_ep(cfg, ep));
  MOE_TRY(need(y_recv));
  MOE_TRY(need4(recv_offsets));
  for (int r = 0; r < ep->n_ranks; ++r) MOE_TRY(need(ep->y_back[r]));
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  return cuda_status(launch_ep_return(*cfg, ep->n_ranks, ep->rank, ep->counts_all, ep->y_back,
                                      y_recv, recv_offsets, err,
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_plan_host(int32_t n_ranks, int32_t E, int32_t rank, const int32_t *C,
                            int32_t *recv_offsets, int32_t *send_base, int32_t *recv_src,
                            int32_t *recv_src_row, int32_t max_recv) {
  if (n_ranks < 1 || n_ranks > MOE_EP_MAX_RANKS || E < 1 || E > 1024 || E % n_ranks)
    return MOE_ERR_INVALID_ARG;
  if (rank < 0 || rank >= n_ranks || !C || !recv_offsets || !send_base || max_recv < 0)
    return MOE_ERR_INVALID_ARG;
  const int e_loc = E / n_ranks;
  // send bases: rows of the owner's experts before e, then of e's earlier sources
  for (int r = 0; r < n_ranks; ++r) {
    long long run = 0;
    for (int j = 0; j < e_loc; ++j) {
      const int e = r * e_loc + j;
      long long before = 0;
      for (int s = 0; s < rank; ++s) before += C[(size_t)s * E + e];
      send_base[e] = (int32_t)(run + before);
      if (r == rank) recv_offsets[j] = (int32_t)run;
      for (int s = 0; s < n_ranks; ++s) run += C[(size_t)s * E + e];
    }
    if (r == rank) recv_offsets[e_loc] = (int32_t)run;
  }
  const int R = recv_offsets[e_loc];
  if (!recv_src && !recv_src_row) return MOE_OK;
  if (!recv_src || !recv_src_row || R > max_recv) return MOE_ERR_INVALID_ARG;
  // every received row: its source and the row of the source's own layout
  for (int j = 0, p = recv_offsets[0]; j < e_loc; ++j) {
    const int e = rank * e_loc + j;
    for (int s = 0; s < n_ranks; ++s) {
      long long first = 0;  // rows of s's experts before e
      for (int e2 = 0; e2 < e; ++e2) first += C[(size_t)s * E + e2];
      for (int i = 0; i < C[(size_t)s * E + e]; ++i, ++p) {
        recv_src[p] = s;
        recv_src_row[p] = (int32_t)(first + i);
      }
    }
  }
  return MOE_OK;
}

moe_status moe_check_errors(void *stream, uint32_t *flags) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t *err = device_error_word();
  if (!err) return MOE_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, err, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v && cudaMemset(err, 0, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
  if (flags) *flags = v;
  return v ? MOE_ERR_DEVICE_CHECK : MOE_OK;
}

const char *moe_status_string(int32_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null pointer or size out of range";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: valid but unsupported configuration";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT: pointer or row size not 16-byte aligned";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or launch failed";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a device-side check fired";
    default: return "unknown moe_status";
  }
}

}  // extern "C"
