// C ABI of libmoe.so: argument validation, workspace layout and kernel launches.
// Declarations and the contract of each entry point are in include/moe.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <map>
#include <mutex>
#include <utility>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {

int num_sms() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 64 && cache[dev]) return cache[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (n <= 0) n = 148;
  if (dev < 64) cache[dev] = n;
  return n;
}

namespace {

thread_local char g_err[512];

moe_status_t fail(moe_status_t code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return code;
}

moe_status_t cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_err, sizeof g_err, "%s: %s", where, cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

constexpr size_t kAlign = 1024;
inline size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Workspace regions, in order; each starts on a 1024-byte boundary.
struct Layout {
  size_t status, topk_idx, topk_w, block_base, counts, offsets, row_of, token_of_row, x_perm, h,
      y, rnorm, row_ready, split_sem, partial, end;
  size_t x_in[2], res_in[2], out_st, end_host;  // staging of the host entry points
};

Layout layout(const Shape& s) {
  Layout L;
  const size_t tk = (size_t)s.T * s.k;
  const size_t rmax = (size_t)max_padded_rows(s);
  size_t o = 0;
  L.status = o; o += up(256);
  L.topk_idx = o; o += up(tk * 4);
  L.topk_w = o; o += up(tk * 4);
  L.block_base = o; o += up((size_t)num_token_blocks(s) * s.E * 4);
  L.counts = o; o += up((size_t)s.E * 4);
  L.offsets = o; o += up((size_t)(s.E + 1) * 4);
  L.row_of = o; o += up(tk * 4);
  L.token_of_row = o; o += up(rmax * 4);
  L.x_perm = o; o += up(rmax * s.H * 2);
  L.h = o; o += up(rmax * s.I * 2);
  L.y = o; o += up(rmax * s.H * 4);
  L.rnorm = o; o += up((size_t)s.T * 4);
  L.row_ready = o; o += up((size_t)(rmax / 64) * 4);  // one-grid experts: sub-tiles of h done
  // split-K of the down GEMM (small batches only): arrival counters and partial sums
  const bool split = (int64_t)tk <= kSplitMaxRows;
  L.split_sem = o; o += split ? up((size_t)kSplitSems * 4) : 0;
  L.partial = o; o += split ? up((size_t)kMaxSplitK * tk * s.H * 4) : 0;
  L.end = o;
  for (int b = 0; b < 2; ++b) {
    L.x_in[b] = o; o += up((size_t)s.T * s.H * 2);
    L.res_in[b] = o; o += up((size_t)s.T * s.H * 2);
  }
  L.out_st = o; o += up((size_t)s.T * s.H * 2);
  L.end_host = o;
  return L;
}

moe_status_t check_shape(const moe_shape_t* sh, Shape* out) {
  if (!sh) return fail(MOE_ERR_INVALID_ARG, "shape is NULL");
  if (sh->num_tokens < 1) return fail(MOE_ERR_INVALID_ARG, "num_tokens must be >= 1 (got %lld)", (long long)sh->num_tokens);
  if (sh->num_experts < 1 || sh->num_experts > 64)
    return fail(MOE_ERR_UNSUPPORTED, "num_experts must be in [1, 64] (got %d)", sh->num_experts);
  if (sh->num_experts_per_tok < 1 || sh->num_experts_per_tok > sh->num_experts ||
      sh->num_experts_per_tok > 8)
    return fail(MOE_ERR_UNSUPPORTED, "num_experts_per_tok must be in [1, min(8, num_experts)] (got %d)",
                sh->num_experts_per_tok);
  if (sh->hidden_size <= 0 || sh->hidden_size % 128)
    return fail(MOE_ERR_UNSUPPORTED, "hidden_size must be a positive multiple of 128 (got %d)",
                sh->hidden_size);
  if (sh->intermediate_size <= 0 || sh->intermediate_size % 128)
    return fail(MOE_ERR_UNSUPPORTED, "intermediate_size must be a positive multiple of 128 (got %d)",
                sh->intermediate_size);
  if (sh->num_tokens * sh->num_experts_per_tok > (int64_t)1 << 30)
    return fail(MOE_ERR_UNSUPPORTED, "num_tokens * num_experts_per_tok must be <= 2^30 (got %lld)",
                (long long)(sh->num_tokens * sh->num_experts_per_tok));
  if (sh->weight_layout != MOE_WEIGHTS_ROW_MAJOR && sh->weight_layout != MOE_WEIGHTS_BLOCKED)
    return fail(MOE_ERR_INVALID_ARG, "weight_layout must be MOE_WEIGHTS_ROW_MAJOR or MOE_WEIGHTS_BLOCKED (got %d)",
                sh->weight_layout);
  out->T = sh->num_tokens;
  out->H = sh->hidden_size;
  out->I = sh->intermediate_size;
  out->E = sh->num_experts;
  out->k = sh->num_experts_per_tok;
  out->blocked = sh->weight_layout == MOE_WEIGHTS_BLOCKED;
  if (sh->router_bf16_logits != 0 && sh->router_bf16_logits != 1)
    return fail(MOE_ERR_INVALID_ARG, "router_bf16_logits must be 0 or 1 (got %d)",
                sh->router_bf16_logits);
  out->bf16_logits = sh->router_bf16_logits;
  const int64_t rmax = max_padded_rows(*out);
  if ((rmax / 128) * (int64_t)(out->I / 128) > INT32_MAX || (int64_t)out->E * out->I > INT32_MAX)
    return fail(MOE_ERR_UNSUPPORTED, "shape too large for 32-bit tile indices");
  return MOE_OK;
}

moe_status_t check_ptr(const void* p, const char* name, bool nullable = false) {
  if (!p) {
    if (nullable) return MOE_OK;
    return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  }
  if (reinterpret_cast<uintptr_t>(p) % 16)
    return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return MOE_OK;
}

moe_status_t check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(MOE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "workspace too small: need %zu bytes, got %zu", need, ws_bytes);
  return MOE_OK;
}

#define MOE_TRY(x)                  \
  do {                              \
    moe_status_t _s = (x);          \
    if (_s != MOE_OK) return _s;    \
  } while (0)

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s per wait

// Expert weights of one layer: bf16 (w1, w3, w2), int8 codes with per-row scales, or
// 4-bit codes with half group scales (q1 non-null; then x_perm and h are IEEE half).
struct Experts {
  const uint16_t *w1, *w3, *w2;
  const uint8_t *q1, *q3, *q2;
  const float *s1, *s3, *s2;
  const uint16_t *g1, *g3, *g2;
  int bits;
};

Experts bf16_experts(const uint16_t* w1, const uint16_t* w3, const uint16_t* w2) {
  Experts x = {};
  x.w1 = w1;
  x.w3 = w3;
  x.w2 = w2;
  return x;
}

Experts int8_experts(const uint8_t* q1, const uint8_t* q3, const uint8_t* q2, const float* s1,
                     const float* s3, const float* s2) {
  Experts x = {};
  x.q1 = q1;
  x.q3 = q3;
  x.q2 = q2;
  x.s1 = s1;
  x.s3 = s3;
  x.s2 = s2;
  x.bits = 8;
  return x;
}

Experts int4_experts(const uint8_t* q1, const uint8_t* q3, const uint8_t* q2, const uint16_t* g1,
                     const uint16_t* g3, const uint16_t* g2) {
  Experts x = {};
  x.q1 = q1;
  x.q3 = q3;
  x.q2 = q2;
  x.g1 = g1;
  x.g3 = g3;
  x.g2 = g2;
  x.bits = 4;
  return x;
}

// Workspace scratch of the expert GEMMs: the per-expert counts and the split-K regions
// of the bf16 down GEMM (null: no split), and the row-tile counters that let the
// quantised experts run both GEMMs as one grid (null: two grids).
struct SplitK {
  const int32_t* counts = nullptr;
  float* partial = nullptr;
  int32_t* sem = nullptr;
  int32_t* row_ready = nullptr;
  const int32_t* q_counts = nullptr;  // routed rows per expert (sizes one-grid row tiles)
  bool row_ready_zeroed = false;      // the gather kernel zeroed row_ready
};

moe_status_t run_experts(const Shape& s, const uint16_t* x_perm, const int32_t* offsets,
                         const Experts& w, uint16_t* h, float* y, int32_t* status,
                         cudaStream_t st, const SplitK& split = SplitK()) {
  const char* why = "";
  cudaError_t e;
  if (w.q1) {
    GemmArgsW8 g;
    g.a = x_perm;
    g.offsets = offsets;
    g.q1 = w.q1;
    g.q3 = w.q3;
    g.q2 = w.q2;
    g.s1 = w.s1;
    g.s3 = w.s3;
    g.s2 = w.s2;
    g.g1 = w.g1;
    g.g3 = w.g3;
    g.g2 = w.g2;
    g.bits = w.bits == 4 ? 4 : 8;
    g.h = h;
    g.y = y;
    g.status = status;
    g.rmax = max_padded_rows(s);
    g.timeout_ns = kTimeoutNs;
    g.row_ready = split.row_ready;
    g.row_ready_zeroed = split.row_ready_zeroed;
    g.counts = split.q_counts;
    e = launch_grouped_swiglu_w8(s, g, st, &why);
  } else {
    GemmArgs g;
    g.a = x_perm;
    g.offsets = offsets;
    g.w1 = w.w1;
    g.w3 = w.w3;
    g.w2 = w.w2;
    g.h = h;
    g.y = y;
    g.status = status;
    g.rmax = max_padded_rows(s);
    g.timeout_ns = kTimeoutNs;
    g.counts = split.counts;
    g.partial = split.partial;
    g.split_sem = split.sem;
    g.row_ready = split.row_ready;
    g.row_ready_zeroed = split.row_ready_zeroed;
    g.expert_rows = split.q_counts;
    e = launch_grouped_swiglu(s, g, st, &why);
  }
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, why);
}

moe_status_t run_forward(const Shape& s, const uint16_t* x, const uint16_t* wr, const float* bias,
                         const Experts& w, const uint16_t* res, uint16_t* out, void* ws,
                         cudaStream_t st, const uint16_t* norm_w = nullptr, float eps = 0.f) {
  const Layout L = layout(s);
  float* rnorm = norm_w ? at<float>(ws, L.rnorm) : nullptr;
  cudaError_t e = launch_router(s, x, wr, bias, at<int32_t>(ws, L.topk_idx), at<float>(ws, L.topk_w),
                                nullptr, st, norm_w, eps, rnorm);
  if (e != cudaSuccess) return cuda_fail(e, "router launch");
  e = launch_permute(s, at<int32_t>(ws, L.topk_idx), x, at<int32_t>(ws, L.counts),
                     at<int32_t>(ws, L.offsets), at<int32_t>(ws, L.row_of),
                     at<int32_t>(ws, L.token_of_row), at<uint16_t>(ws, L.x_perm),
                     at<int32_t>(ws, L.block_base), st, norm_w, rnorm, w.q1 != nullptr,
                     at<int32_t>(ws, L.row_ready), (int)(max_padded_rows(s) / 64));
  if (e != cudaSuccess) return cuda_fail(e, "permute launch");
  SplitK split;
  split.row_ready = at<int32_t>(ws, L.row_ready);
  split.row_ready_zeroed = true;
  split.q_counts = at<int32_t>(ws, L.counts);
  if (L.partial != L.end) {
    split.counts = at<int32_t>(ws, L.counts);
    split.partial = at<float>(ws, L.partial);
    split.sem = at<int32_t>(ws, L.split_sem);
  }
  MOE_TRY(run_experts(s, at<uint16_t>(ws, L.x_perm), at<int32_t>(ws, L.offsets), w,
                      at<uint16_t>(ws, L.h), at<float>(ws, L.y), at<int32_t>(ws, L.status), st,
                      split));
  e = launch_combine(s, at<float>(ws, L.y), at<int32_t>(ws, L.row_of), at<float>(ws, L.topk_w), res,
                     out, st);
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  return MOE_OK;
}

// Host-path overlap. The copies in of a host call run on a copy stream of the library's
// own, into one of two staging slots of the workspace, so they overlap the previous
// call's layer; the caller's stream waits for them (event `ready`) before the layer, and
// a slot is refilled only after the call two back has finished with the workspace: its
// layer and its copy out (event `freed`). Every region's offset depends on the shape, so
// when a call's shape differs from the previous call's on this workspace, its copies in
// may land anywhere the previous call still reads or writes: they then also wait for the
// previous call to finish.
struct HostPath {
  cudaStream_t copy = nullptr;
  cudaEvent_t ready[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
  bool freed_recorded[2] = {false, false};
  unsigned calls = 0;
  size_t prev_x_in = 0, prev_end_host = 0;  // staging layout of the previous call
};

std::mutex g_host_mutex;
std::map<std::pair<int, void*>, HostPath> g_host_paths;  // (device, workspace)

cudaError_t host_path(void* ws, HostPath** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  HostPath& h = g_host_paths[std::make_pair(dev, ws)];
  if (!h.copy) {
    e = cudaStreamCreateWithFlags(&h.copy, cudaStreamNonBlocking);
    for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
      e = cudaEventCreateWithFlags(&h.ready[b], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h.freed[b], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return e;
  }
  *out = &h;
  return cudaSuccess;
}

moe_status_t forward_host_enqueue(const moe_shape_t* shape, const moe_bf16_t* x_host,
                                  const moe_bf16_t* w_router, const float* logit_bias,
                                  const moe_bf16_t* w1, const moe_bf16_t* w3, const moe_bf16_t* w2,
                                  const moe_bf16_t* residual_host, moe_bf16_t* out_host, void* ws,
                                  size_t ws_bytes, cudaStream_t st) {
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  if (!x_host) return fail(MOE_ERR_INVALID_ARG, "x_host is NULL");
  if (!out_host) return fail(MOE_ERR_INVALID_ARG, "out_host is NULL");
  MOE_TRY(check_ptr(w_router, "w_router"));
  MOE_TRY(check_ptr(logit_bias, "logit_bias", true));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end_host));
  std::lock_guard<std::mutex> lock(g_host_mutex);
  HostPath* hp = nullptr;
  cudaError_t e = host_path(ws, &hp);
  if (e != cudaSuccess) return cuda_fail(e, "host-path stream or event creation");
  const int b = (int)(hp->calls++ & 1u);
  const size_t bytes = (size_t)s.T * s.H * 2;
  uint16_t* xd = at<uint16_t>(ws, L.x_in[b]);
  uint16_t* rd = residual_host ? at<uint16_t>(ws, L.res_in[b]) : nullptr;
  uint16_t* od = at<uint16_t>(ws, L.out_st);
  // copies in, on the copy stream, once the call two back is done with the workspace;
  // after a change of shape, also once the previous call is
  const bool moved = hp->calls > 1 && (hp->prev_x_in != L.x_in[0] || hp->prev_end_host != L.end_host);
  hp->prev_x_in = L.x_in[0];
  hp->prev_end_host = L.end_host;
  for (int j = 0; j < 2; ++j) {
    if (!hp->freed_recorded[j] || (j != b && !moved)) continue;
    e = cudaStreamWaitEvent(hp->copy, hp->freed[j], 0);
    if (e != cudaSuccess) return cuda_fail(e, "copy-stream wait");
  }
  e = cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, hp->copy);
  if (e != cudaSuccess) return cuda_fail(e, "copy of x to the device");
  if (rd) {
    e = cudaMemcpyAsync(rd, residual_host, bytes, cudaMemcpyHostToDevice, hp->copy);
    if (e != cudaSuccess) return cuda_fail(e, "copy of residual to the device");
  }
  e = cudaEventRecord(hp->ready[b], hp->copy);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, hp->ready[b], 0);
  if (e != cudaSuccess) return cuda_fail(e, "copy-in event");
  // the layer and the copy out, on the caller's stream
  MOE_TRY(run_forward(s, xd, w_router, logit_bias, bf16_experts(w1, w3, w2), rd, od, ws, st));
  e = cudaMemcpyAsync(out_host, od, bytes, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "copy of out to the host");
  e = cudaEventRecord(hp->freed[b], st);
  if (e != cudaSuccess) return cuda_fail(e, "slot event");
  hp->freed_recorded[b] = true;
  return MOE_OK;
}

}  // namespace

int validate_shape(const moe_shape_t* shape, Shape* out) { return (int)check_shape(shape, out); }

void set_error_message(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_shape_t* shape) {
  Shape s;
  if (check_shape(shape, &s) != MOE_OK) return 0;
  return layout(s).end;
}

size_t moe_workspace_size_host(const moe_shape_t* shape) {
  Shape s;
  if (check_shape(shape, &s) != MOE_OK) return 0;
  return layout(s).end_host;
}

int64_t moe_max_padded_rows(const moe_shape_t* shape) {
  Shape s;
  if (check_shape(shape, &s) != MOE_OK) return -1;
  return max_padded_rows(s);
}

const char* moe_last_error(void) { return g_err; }

moe_status_t moe_router_topk(const moe_shape_t* shape, const moe_bf16_t* x,
                             const moe_bf16_t* w_router, const float* logit_bias,
                             int32_t* topk_idx, float* topk_w, float* router_logits,
                             moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(w_router, "w_router"));
  MOE_TRY(check_ptr(logit_bias, "logit_bias", true));
  MOE_TRY(check_ptr(topk_idx, "topk_idx"));
  MOE_TRY(check_ptr(topk_w, "topk_w"));
  MOE_TRY(check_ptr(router_logits, "router_logits", true));
  cudaError_t e = launch_router(s, x, w_router, logit_bias, topk_idx, topk_w, router_logits,
                                (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "router launch");
}

moe_status_t moe_permute(const moe_shape_t* shape, const int32_t* topk_idx, const moe_bf16_t* x,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* row_of,
                         int32_t* token_of_row, moe_bf16_t* x_perm, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(topk_idx, "topk_idx"));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(expert_counts, "expert_counts"));
  MOE_TRY(check_ptr(expert_offsets, "expert_offsets"));
  MOE_TRY(check_ptr(row_of, "row_of"));
  MOE_TRY(check_ptr(token_of_row, "token_of_row"));
  MOE_TRY(check_ptr(x_perm, "x_perm"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end));
  cudaError_t e = launch_permute(s, topk_idx, x, expert_counts, expert_offsets, row_of,
                                 token_of_row, x_perm, at<int32_t>(ws, L.block_base),
                                 (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "permute launch");
}

moe_status_t moe_grouped_swiglu(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                const int32_t* expert_offsets, const moe_bf16_t* w1,
                                const moe_bf16_t* w3, const moe_bf16_t* w2, float* y_perm,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x_perm, "x_perm"));
  MOE_TRY(check_ptr(expert_offsets, "expert_offsets"));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(y_perm, "y_perm"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end));
  SplitK scratch;
  scratch.row_ready = at<int32_t>(ws, L.row_ready);
  return run_experts(s, x_perm, expert_offsets, bf16_experts(w1, w3, w2), at<uint16_t>(ws, L.h),
                     y_perm, at<int32_t>(ws, L.status), (cudaStream_t)stream, scratch);
}

moe_status_t moe_expert_gate_up(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                const int32_t* expert_offsets, const moe_bf16_t* w1,
                                const moe_bf16_t* w3, moe_bf16_t* h, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x_perm, "x_perm"));
  MOE_TRY(check_ptr(expert_offsets, "expert_offsets"));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(h, "h"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end));
  GemmArgs g = {};
  g.a = x_perm;
  g.offsets = expert_offsets;
  g.w1 = w1;
  g.w3 = w3;
  g.h = h;
  g.status = at<int32_t>(ws, 0);
  g.rmax = max_padded_rows(s);
  g.timeout_ns = kTimeoutNs;
  const char* why = "";
  cudaError_t e = launch_gate_up(s, g, (cudaStream_t)stream, &why);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, why);
}

moe_status_t moe_expert_down(const moe_shape_t* shape, const moe_bf16_t* h,
                             const int32_t* expert_offsets, const moe_bf16_t* w2, float* y_perm,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(h, "h"));
  MOE_TRY(check_ptr(expert_offsets, "expert_offsets"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(y_perm, "y_perm"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end));
  GemmArgs g = {};
  g.offsets = expert_offsets;
  g.w2 = w2;
  g.h = const_cast<uint16_t*>(h);
  g.y = y_perm;
  g.status = at<int32_t>(ws, 0);
  g.rmax = max_padded_rows(s);
  g.timeout_ns = kTimeoutNs;
  const char* why = "";
  cudaError_t e = launch_down(s, g, (cudaStream_t)stream, &why);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, why);
}

moe_status_t moe_combine(const moe_shape_t* shape, const float* y_perm, const int32_t* row_of,
                         const float* topk_w, const moe_bf16_t* residual, moe_bf16_t* out,
                         moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(y_perm, "y_perm"));
  MOE_TRY(check_ptr(row_of, "row_of"));
  MOE_TRY(check_ptr(topk_w, "topk_w"));
  MOE_TRY(check_ptr(residual, "residual", true));
  MOE_TRY(check_ptr(out, "out"));
  cudaError_t e = launch_combine(s, y_perm, row_of, topk_w, residual, out, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "combine launch");
}

moe_status_t moe_forward(const moe_shape_t* shape, const moe_bf16_t* x, const moe_bf16_t* w_router,
                         const float* logit_bias, const moe_bf16_t* w1, const moe_bf16_t* w3,
                         const moe_bf16_t* w2, const moe_bf16_t* residual, moe_bf16_t* out,
                         void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(w_router, "w_router"));
  MOE_TRY(check_ptr(logit_bias, "logit_bias", true));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(residual, "residual", true));
  MOE_TRY(check_ptr(out, "out"));
  MOE_TRY(check_ws(ws, ws_bytes, layout(s).end));
  return run_forward(s, x, w_router, logit_bias, bf16_experts(w1, w3, w2), residual, out, ws,
                     (cudaStream_t)stream);
}

moe_status_t moe_forward_rmsnorm(const moe_shape_t* shape, const moe_bf16_t* h,
                                 const moe_bf16_t* norm_weight, float eps,
                                 const moe_bf16_t* w_router, const float* logit_bias,
                                 const moe_bf16_t* w1, const moe_bf16_t* w3, const moe_bf16_t* w2,
                                 moe_bf16_t* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(h, "h"));
  MOE_TRY(check_ptr(norm_weight, "norm_weight"));
  if (!(eps >= 0.f) || eps > 1.f) return fail(MOE_ERR_INVALID_ARG, "eps must be in [0, 1]");
  MOE_TRY(check_ptr(w_router, "w_router"));
  MOE_TRY(check_ptr(logit_bias, "logit_bias", true));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(out, "out"));
  MOE_TRY(check_ws(ws, ws_bytes, layout(s).end));
  return run_forward(s, h, w_router, logit_bias, bf16_experts(w1, w3, w2), h, out, ws,
                     (cudaStream_t)stream, norm_weight, eps);
}

moe_status_t moe_forward_host(const moe_shape_t* shape, const moe_bf16_t* x_host,
                              const moe_bf16_t* w_router, const float* logit_bias,
                              const moe_bf16_t* w1, const moe_bf16_t* w3, const moe_bf16_t* w2,
                              const moe_bf16_t* residual_host, moe_bf16_t* out_host, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  cudaStream_t st = (cudaStream_t)stream;
  MOE_TRY(forward_host_enqueue(shape, x_host, w_router, logit_bias, w1, w3, w2, residual_host,
                               out_host, ws, ws_bytes, st));
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return MOE_OK;
}

moe_status_t moe_forward_host_async(const moe_shape_t* shape, const moe_bf16_t* x_host,
                                    const moe_bf16_t* w_router, const float* logit_bias,
                                    const moe_bf16_t* w1, const moe_bf16_t* w3,
                                    const moe_bf16_t* w2, const moe_bf16_t* residual_host,
                                    moe_bf16_t* out_host, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  g_err[0] = 0;
  return forward_host_enqueue(shape, x_host, w_router, logit_bias, w1, w3, w2, residual_host,
                              out_host, ws, ws_bytes, (cudaStream_t)stream);
}

moe_status_t moe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns,
                                       moe_stream_t stream) {
  g_err[0] = 0;
  MOE_TRY(check_ws(ws, ws_bytes, 256));
  if (timeout_ns == 0 || timeout_ns > 10000000000ull)
    return fail(MOE_ERR_INVALID_ARG, "timeout_ns must be in (0, 10 s]");
  cudaError_t e = launch_wait_selftest(at<int32_t>(ws, 0), timeout_ns, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "self-test launch");
}

moe_status_t moe_pack_weights(const moe_shape_t* shape, const moe_bf16_t* w1, const moe_bf16_t* w3,
                              const moe_bf16_t* w2, moe_bf16_t* w1_blocked, moe_bf16_t* w3_blocked,
                              moe_bf16_t* w2_blocked, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(w1_blocked, "w1_blocked"));
  MOE_TRY(check_ptr(w3_blocked, "w3_blocked"));
  MOE_TRY(check_ptr(w2_blocked, "w2_blocked"));
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t ei = (int64_t)s.E * s.I, eh = (int64_t)s.E * s.H;
  cudaError_t e = launch_pack_blocked(w1, w1_blocked, ei, s.H, st);
  if (e == cudaSuccess) e = launch_pack_blocked(w3, w3_blocked, ei, s.H, st);
  if (e == cudaSuccess) e = launch_pack_blocked(w2, w2_blocked, eh, s.I, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "weight packing launch");
}

moe_status_t moe_device_status(void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  if (!ws || ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace is NULL or too small");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word == 0) return MOE_OK;
  e = cudaMemsetAsync(ws, 0, sizeof word, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  if (word & kStatusTimeout)
    return fail(MOE_ERR_TIMEOUT, "a kernel gave up a bounded wait (device status 0x%x)%s",
                (unsigned)word,
                (word & kStatusUnwound) ? "; it exited with copies or MMAs possibly still in flight"
                                        : "");
  return fail(MOE_ERR_CUDA, "unknown device status 0x%x", (unsigned)word);
}

moe_status_t moe_quantize_int8(const moe_shape_t* shape, const moe_bf16_t* w1,
                               const moe_bf16_t* w3, const moe_bf16_t* w2, uint8_t* q1,
                               uint8_t* q3, uint8_t* q2, float* s1, float* s3, float* s2,
                               moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(q1, "q1"));
  MOE_TRY(check_ptr(q3, "q3"));
  MOE_TRY(check_ptr(q2, "q2"));
  MOE_TRY(check_ptr(s1, "s1"));
  MOE_TRY(check_ptr(s3, "s3"));
  MOE_TRY(check_ptr(s2, "s2"));
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t ei = (int64_t)s.E * s.I, eh = (int64_t)s.E * s.H;
  cudaError_t e = launch_quant_rows(w1, q1, s1, ei, s.H, st);
  if (e == cudaSuccess) e = launch_quant_rows(w3, q3, s3, ei, s.H, st);
  if (e == cudaSuccess) e = launch_quant_rows(w2, q2, s2, eh, s.I, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "int8 quantiser launch");
}

moe_status_t moe_grouped_swiglu_w8(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                   const int32_t* expert_offsets, const uint8_t* q1,
                                   const uint8_t* q3, const uint8_t* q2, const float* s1,
                                   const float* s3, const float* s2, float* y_perm, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x_perm, "x_perm"));
  MOE_TRY(check_ptr(expert_offsets, "expert_offsets"));
  MOE_TRY(check_ptr(q1, "q1"));
  MOE_TRY(check_ptr(q3, "q3"));
  MOE_TRY(check_ptr(q2, "q2"));
  MOE_TRY(check_ptr(s1, "s1"));
  MOE_TRY(check_ptr(s3, "s3"));
  MOE_TRY(check_ptr(s2, "s2"));
  MOE_TRY(check_ptr(y_perm, "y_perm"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end));
  // the int8 experts read half activations: convert the caller's rows into ws
  uint16_t* xh = at<uint16_t>(ws, L.x_perm);
  cudaError_t e = launch_rows_to_f16(x_perm, xh, max_padded_rows(s), s.H, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "x_perm conversion launch");
  SplitK scratch;
  scratch.row_ready = at<int32_t>(ws, L.row_ready);
  return run_experts(s, xh, expert_offsets, int8_experts(q1, q3, q2, s1, s3, s2),
                     at<uint16_t>(ws, L.h), y_perm, at<int32_t>(ws, L.status),
                     (cudaStream_t)stream, scratch);
}

moe_status_t moe_forward_w8(const moe_shape_t* shape, const moe_bf16_t* x,
                            const moe_bf16_t* w_router, const float* logit_bias,
                            const uint8_t* q1, const uint8_t* q3, const uint8_t* q2,
                            const float* s1, const float* s3,
                            const float* s2, const moe_bf16_t* residual, moe_bf16_t* out,
                            void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(w_router, "w_router"));
  MOE_TRY(check_ptr(logit_bias, "logit_bias", true));
  MOE_TRY(check_ptr(q1, "q1"));
  MOE_TRY(check_ptr(q3, "q3"));
  MOE_TRY(check_ptr(q2, "q2"));
  MOE_TRY(check_ptr(s1, "s1"));
  MOE_TRY(check_ptr(s3, "s3"));
  MOE_TRY(check_ptr(s2, "s2"));
  MOE_TRY(check_ptr(residual, "residual", true));
  MOE_TRY(check_ptr(out, "out"));
  MOE_TRY(check_ws(ws, ws_bytes, layout(s).end));
  return run_forward(s, x, w_router, logit_bias, int8_experts(q1, q3, q2, s1, s3, s2), residual,
                     out, ws, (cudaStream_t)stream);
}

moe_status_t moe_quantize_int4(const moe_shape_t* shape, const moe_bf16_t* w1,
                               const moe_bf16_t* w3, const moe_bf16_t* w2, uint8_t* q1,
                               uint8_t* q3, uint8_t* q2, uint16_t* s1, uint16_t* s3,
                               uint16_t* s2, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(w1, "w1"));
  MOE_TRY(check_ptr(w3, "w3"));
  MOE_TRY(check_ptr(w2, "w2"));
  MOE_TRY(check_ptr(q1, "q1"));
  MOE_TRY(check_ptr(q3, "q3"));
  MOE_TRY(check_ptr(q2, "q2"));
  MOE_TRY(check_ptr(s1, "s1"));
  MOE_TRY(check_ptr(s3, "s3"));
  MOE_TRY(check_ptr(s2, "s2"));
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t ei = (int64_t)s.E * s.I, eh = (int64_t)s.E * s.H;
  cudaError_t e = launch_quant_groups4(w1, q1, s1, ei, s.H, st);
  if (e == cudaSuccess) e = launch_quant_groups4(w3, q3, s3, ei, s.H, st);
  if (e == cudaSuccess) e = launch_quant_groups4(w2, q2, s2, eh, s.I, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "4-bit quantiser launch");
}

moe_status_t moe_grouped_swiglu_w4(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                   const int32_t* expert_offsets, const uint8_t* q1,
                                   const uint8_t* q3, const uint8_t* q2, const uint16_t* s1,
                                   const uint16_t* s3, const uint16_t* s2, float* y_perm,
                                   void* ws, size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x_perm, "x_perm"));
  MOE_TRY(check_ptr(expert_offsets, "expert_offsets"));
  MOE_TRY(check_ptr(q1, "q1"));
  MOE_TRY(check_ptr(q3, "q3"));
  MOE_TRY(check_ptr(q2, "q2"));
  MOE_TRY(check_ptr(s1, "s1"));
  MOE_TRY(check_ptr(s3, "s3"));
  MOE_TRY(check_ptr(s2, "s2"));
  MOE_TRY(check_ptr(y_perm, "y_perm"));
  const Layout L = layout(s);
  MOE_TRY(check_ws(ws, ws_bytes, L.end));
  // the 4-bit experts read half activations: convert the caller's rows into ws
  uint16_t* xh = at<uint16_t>(ws, L.x_perm);
  cudaError_t e = launch_rows_to_f16(x_perm, xh, max_padded_rows(s), s.H, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "x_perm conversion launch");
  SplitK scratch;
  scratch.row_ready = at<int32_t>(ws, L.row_ready);
  return run_experts(s, xh, expert_offsets, int4_experts(q1, q3, q2, s1, s3, s2),
                     at<uint16_t>(ws, L.h), y_perm, at<int32_t>(ws, L.status),
                     (cudaStream_t)stream, scratch);
}

moe_status_t moe_forward_w4(const moe_shape_t* shape, const moe_bf16_t* x,
                            const moe_bf16_t* w_router, const float* logit_bias,
                            const uint8_t* q1, const uint8_t* q3, const uint8_t* q2,
                            const uint16_t* s1, const uint16_t* s3, const uint16_t* s2,
                            const moe_bf16_t* residual, moe_bf16_t* out, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  g_err[0] = 0;
  Shape s;
  MOE_TRY(check_shape(shape, &s));
  MOE_TRY(check_ptr(x, "x"));
  MOE_TRY(check_ptr(w_router, "w_router"));
  MOE_TRY(check_ptr(logit_bias, "logit_bias", true));
  MOE_TRY(check_ptr(q1, "q1"));
  MOE_TRY(check_ptr(q3, "q3"));
  MOE_TRY(check_ptr(q2, "q2"));
  MOE_TRY(check_ptr(s1, "s1"));
  MOE_TRY(check_ptr(s3, "s3"));
  MOE_TRY(check_ptr(s2, "s2"));
  MOE_TRY(check_ptr(residual, "residual", true));
  MOE_TRY(check_ptr(out, "out"));
  MOE_TRY(check_ws(ws, ws_bytes, layout(s).end));
  return run_forward(s, x, w_router, logit_bias, int4_experts(q1, q3, q2, s1, s3, s2), residual,
                     out, ws, (cudaStream_t)stream);
}

moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int64_t* index,
                             int64_t n_rows, int64_t row_bytes, void* dst, moe_stream_t stream) {
  g_err[0] = 0;
  if (n_rows < 0 || src_rows < 0) return fail(MOE_ERR_INVALID_ARG, "row counts must be >= 0");
  if (row_bytes <= 0 || row_bytes % 16)
    return fail(MOE_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16 (got %lld)",
                (long long)row_bytes);
  if (n_rows == 0) return MOE_OK;
  MOE_TRY(check_ptr(src, "src", src_rows == 0));
  MOE_TRY(check_ptr(index, "index"));
  MOE_TRY(check_ptr(dst, "dst"));
  cudaError_t e = launch_gather_rows(src, dst, index, n_rows, src_rows, row_bytes,
                                     (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "row gather launch");
}

moe_status_t moe_ipc_alloc(size_t bytes, void** dev_ptr, void* handle) {
  g_err[0] = 0;
  if (!dev_ptr || !handle) return fail(MOE_ERR_INVALID_ARG, "dev_ptr and handle must not be NULL");
  *dev_ptr = nullptr;
  if (bytes == 0) return fail(MOE_ERR_INVALID_ARG, "bytes must be > 0");
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc of a shareable buffer");
  cudaIpcMemHandle_t h;
  e = cudaIpcGetMemHandle(&h, p);
  if (e != cudaSuccess) {
    cudaFree(p);
    return cuda_fail(e, "cudaIpcGetMemHandle");
  }
  memcpy(handle, &h, sizeof h);
  *dev_ptr = p;
  return MOE_OK;
}

moe_status_t moe_ipc_open(const void* handle, void** dev_ptr) {
  g_err[0] = 0;
  if (!dev_ptr || !handle) return fail(MOE_ERR_INVALID_ARG, "dev_ptr and handle must not be NULL");
  *dev_ptr = nullptr;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof h);
  cudaError_t e = cudaIpcOpenMemHandle(dev_ptr, h, cudaIpcMemLazyEnablePeerAccess);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cudaIpcOpenMemHandle");
}

moe_status_t moe_ipc_close(void* dev_ptr) {
  g_err[0] = 0;
  if (!dev_ptr) return MOE_OK;
  cudaError_t e = cudaIpcCloseMemHandle(dev_ptr);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cudaIpcCloseMemHandle");
}

moe_status_t moe_ipc_free(void* dev_ptr) {
  g_err[0] = 0;
  if (!dev_ptr) return MOE_OK;
  cudaError_t e = cudaFree(dev_ptr);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cudaFree of a shareable buffer");
}

moe_status_t moe_scatter_rows_peer(const void* src, int64_t src_rows, const int64_t* src_index,
                                   const int32_t* dst_rank, const int64_t* dst_row,
                                   int64_t n_rows, void* const* dst_bases, int world,
                                   int64_t dst_rows, int64_t row_bytes, int32_t* bad_rows,
                                   moe_stream_t stream) {
  g_err[0] = 0;
  if (n_rows < 0 || src_rows < 0 || dst_rows < 0)
    return fail(MOE_ERR_INVALID_ARG, "row counts must be >= 0");
  if (world < 1) return fail(MOE_ERR_INVALID_ARG, "world must be >= 1 (got %d)", world);
  if (row_bytes <= 0 || row_bytes % 16)
    return fail(MOE_ERR_INVALID_ARG, "row_bytes must be a positive multiple of 16 (got %lld)",
                (long long)row_bytes);
  if (n_rows == 0) return MOE_OK;
  MOE_TRY(check_ptr(src, "src", src_rows == 0));
  MOE_TRY(check_ptr(src_index, "src_index"));
  if (!dst_rank || !dst_row || !dst_bases)
    return fail(MOE_ERR_INVALID_ARG, "dst_rank, dst_row and dst_bases must not be NULL");
  cudaError_t e = launch_scatter_rows_peer(src, src_rows, src_index, dst_rank, dst_row, n_rows,
                                           dst_bases, world, dst_rows, row_bytes, bad_rows,
                                           (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "peer row scatter launch");
}

moe_status_t moe_combine_peer(const float* const* y_bases, int world, int64_t y_rows,
                              const int32_t* slot_rank, const int64_t* slot_row,
                              const float* topk_w, const moe_bf16_t* residual, moe_bf16_t* out,
                              int64_t num_tokens, int k, int hidden, int32_t* bad_slots,
                              moe_stream_t stream) {
  g_err[0] = 0;
  if (num_tokens < 0 || y_rows < 0) return fail(MOE_ERR_INVALID_ARG, "sizes must be >= 0");
  if (world < 1) return fail(MOE_ERR_INVALID_ARG, "world must be >= 1 (got %d)", world);
  if (k < 1 || k > 8) return fail(MOE_ERR_UNSUPPORTED, "k must be in [1, 8] (got %d)", k);
  if (hidden <= 0 || hidden % 8)
    return fail(MOE_ERR_UNSUPPORTED, "hidden must be a positive multiple of 8 (got %d)", hidden);
  if (num_tokens == 0) return MOE_OK;
  if (!y_bases || !slot_rank || !slot_row || !topk_w)
    return fail(MOE_ERR_INVALID_ARG, "y_bases, slot_rank, slot_row and topk_w must not be NULL");
  MOE_TRY(check_ptr(residual, "residual", true));
  MOE_TRY(check_ptr(out, "out"));
  cudaError_t e = launch_combine_peer(y_bases, world, y_rows, slot_rank, slot_row, topk_w,
                                      residual, out, num_tokens, hidden, k, bad_slots,
                                      (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "peer combine launch");
}

}  // extern "C"
