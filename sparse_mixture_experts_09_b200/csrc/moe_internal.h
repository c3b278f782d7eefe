// Internal declarations shared by the libmoe.so translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Routed (token, slot) pairs handled by one CTA of the histogram / scatter kernels:
// one warp's worth of tokens, so a CTA ranks its pairs with warp ballots.
constexpr int kTokensPerBlock = 32;
constexpr int kRowPad = 128;


// Device status word, first int32 of the workspace: a bounded wait ran out
// (kStatusTimeout); while unwinding after it, a wait for the kernel's own copies or
// MMAs ran out too, so they may still have been in flight when it released its tensor
// memory and exited (kStatusUnwound).
constexpr int32_t kStatusTimeout = 1;
constexpr int32_t kStatusUnwound = 2;

struct Shape {
  int64_t T;
  int H, I, E, k;
  int blocked;  // expert weights in the blocked layout
  int bf16_logits;  // router logits rounded to bf16 before scoring
};

inline int64_t max_padded_rows(const Shape& s) {
  int64_t r = s.T * s.k;
  return (r + kRowPad - 1) / kRowPad * kRowPad + (int64_t)kRowPad * s.E;
}

inline int64_t num_token_blocks(const Shape& s) {
  return (s.T + kTokensPerBlock - 1) / kTokensPerBlock;
}

// ---- launchers (each returns the launch's cudaError_t) ----

// norm_w (nullable): RMSNorm gain [H]; the router then routes the normed rows and
// writes 1/rms per token to rnorm, and the gather writes the normed rows.
cudaError_t launch_router(const Shape& s, const uint16_t* x, const uint16_t* w_router,
                          const float* logit_bias, int32_t* topk_idx, float* topk_w,
                          float* logits, cudaStream_t st, const uint16_t* norm_w = nullptr,
                          float eps = 0.f, float* rnorm = nullptr);

cudaError_t launch_permute(const Shape& s, const int32_t* topk_idx, const uint16_t* x,
                           int32_t* counts, int32_t* offsets, int32_t* row_of,
                           int32_t* token_of_row, uint16_t* x_perm, int32_t* block_base,
                           cudaStream_t st, const uint16_t* norm_w = nullptr,
                           const float* rnorm = nullptr, bool f16_out = false,
                           int32_t* zero_buf = nullptr, int zero_n = 0);

// x_perm rows [0, rows) of width H: bf16 -> IEEE half (the int8 experts' input).
cudaError_t launch_rows_to_f16(const uint16_t* src, uint16_t* dst, int64_t rows, int H,
                               cudaStream_t st);

// Split-K of the down GEMM for small batches. When its tiles would leave SMs idle, each
// tile's K range is cut into S <= kMaxSplitK parts: every part writes fp32 partial sums
// of its tile's real rows to a workspace region, and the part that finishes last sums
// the S partials in part order and writes y (the result does not depend on which part
// finishes last). Used for batches of at most kSplitMaxRows routed rows, when the
// per-expert row counts are known (they bound the rows to store).
constexpr int kMaxSplitK = 8;
constexpr int64_t kSplitMaxRows = 512;
constexpr int kSplitSems = 1024;  // arrival counters, one per (tile, epilogue warp)

struct GemmArgs {
  const uint16_t* a;        // x_perm [Rmax, K1] (GEMM1) or h [Rmax, I] (GEMM2)
  const int32_t* offsets;   // [E+1], multiples of 128
  const uint16_t* w1;
  const uint16_t* w3;
  const uint16_t* w2;
  uint16_t* h;              // [Rmax, I]
  float* y;                 // [Rmax, H]
  int32_t* status;          // device status word
  int64_t rmax;
  unsigned long long timeout_ns;
  // split-K of GEMM2 (all null: no split): per-expert routed rows [E], partial sums
  // [kMaxSplitK, T*k, H] fp32, arrival counters [kSplitSems] (GEMM1 zeroes them)
  const int32_t* counts = nullptr;
  float* partial = nullptr;
  int32_t* split_sem = nullptr;
  // [Rmax / 64] int32 scratch: given, at most 256 tokens run both GEMMs as one grid
  int32_t* row_ready = nullptr;
  // [E] routed rows per expert (nullable): they size the one-grid kernel's row tiles
  // (16-row steps); null: every row tile is sized for its full 128 rows or the batch
  const int32_t* expert_rows = nullptr;
  // row_ready was zeroed by an earlier kernel in the stream (the gather): no memset,
  // so the one-grid kernel's launch overlaps the kernels before it
  bool row_ready_zeroed = false;
};

// GEMM1 (gate/up + SwiGLU -> h) then GEMM2 (h w2^T -> y), both persistent tcgen05.
cudaError_t launch_gate_up(const Shape& s, const GemmArgs& g, cudaStream_t st, const char** why);
cudaError_t launch_down(const Shape& s, const GemmArgs& g, cudaStream_t st, const char** why);
cudaError_t launch_grouped_swiglu(const Shape& s, const GemmArgs& g, cudaStream_t st,
                                  const char** why);

// ---- weight-only int8 experts ----
// Per output row r of w [rows, K] (bf16): s[r] = max|w[r,:]| / 127 (1 for a zero row),
// q = rint(w / s) clamped to [-127, 127], both in float32; q + 128 is written in the
// tiled code layout (rows % 128 == 0, K % 64 == 0).
cudaError_t launch_quant_rows(const uint16_t* w, uint8_t* q, float* s, int64_t rows, int K,
                              cudaStream_t st);

// Per group of 64 columns of a row of w [rows, K] (bf16): s = half(max|w| / 7) (1 when
// that is zero), q = rint(w / s) clamped to [-7, 7], in float32; q + 8 is written in
// the tiled 4-bit layout and s, as IEEE half bits, in the same tile order (element
// ((row / 128) * (K / 64) + col / 64) * 128 + row % 128).
cudaError_t launch_quant_groups4(const uint16_t* w, uint8_t* q, uint16_t* s, int64_t rows, int K,
                                 cudaStream_t st);

struct GemmArgsW8 {
  const uint16_t* a = nullptr;        // x_perm [Rmax, H], IEEE half
  const int32_t* offsets = nullptr;   // [E+1], multiples of 128
  const uint8_t* q1 = nullptr;        // tiled offset-binary codes of w1 (rows E*I, K = H)
  const uint8_t* q3 = nullptr;        // same for w3
  const uint8_t* q2 = nullptr;        // tiled codes of w2 (rows E*H, K = I)
  const float* s1 = nullptr;          // int8: per-row scales [E*I]
  const float* s3 = nullptr;          // [E*I]
  const float* s2 = nullptr;          // [E*H]
  const uint16_t* g1 = nullptr;       // 4-bit: half group scales of w1, tile order
  const uint16_t* g3 = nullptr;
  const uint16_t* g2 = nullptr;
  int bits = 8;                       // 8 or 4
  uint16_t* h = nullptr;              // [Rmax, I], IEEE half
  float* y = nullptr;                 // [Rmax, H]
  int32_t* status = nullptr;
  int64_t rmax = 0;
  unsigned long long timeout_ns = 0;
  // [rmax / 64] int32 scratch: given, at most 256 tokens run both GEMMs as one grid
  // (intermediate % 256 == 0)
  int32_t* row_ready = nullptr;
  // [E] routed rows per expert (nullable): they size the one-grid kernel's sub-tiles
  // (16-row steps); null: an expert is taken to have min(T, its padded rows) rows
  const int32_t* counts = nullptr;
  // row_ready was zeroed by an earlier kernel in the stream (the gather): no memset
  bool row_ready_zeroed = false;
};

// GEMM1 (int8 or 4-bit gate/up + SwiGLU -> h) then GEMM2 (h q2^T -> y), in float16.
cudaError_t launch_grouped_swiglu_w8(const Shape& s, const GemmArgsW8& g, cudaStream_t st,
                                     const char** why);

// w [rows, cols] -> blocked layout [rows/128][cols/64][128][64] (rows % 128 == 0,
// cols % 64 == 0).
cudaError_t launch_pack_blocked(const uint16_t* w, uint16_t* wp, int64_t rows, int64_t cols,
                                cudaStream_t st);

// One thread's bounded wait on a barrier nothing arrives on (checks timeout reporting).
cudaError_t launch_wait_selftest(int32_t* status, unsigned long long timeout_ns, cudaStream_t st);

cudaError_t launch_combine(const Shape& s, const float* y, const int32_t* row_of,
                           const float* topk_w, const uint16_t* residual, uint16_t* out,
                           cudaStream_t st);

// dst[i] = src[index[i]] for i < n_rows, rows of row_bytes (a multiple of 16) bytes;
// an index outside [0, src_rows) writes a zero row.
cudaError_t launch_gather_rows(const void* src, void* dst, const int64_t* index, int64_t n_rows,
                               int64_t src_rows, int64_t row_bytes, cudaStream_t st);

// Peer-memory exchange of the expert-parallel layer (ep_peer.cu). dst_bases and y_bases
// are device arrays of `world` device pointers (this GPU's buffers or peers' mappings).
cudaError_t launch_scatter_rows_peer(const void* src, int64_t src_rows, const int64_t* src_index,
                                     const int32_t* dst_rank, const int64_t* dst_row,
                                     int64_t n_rows, void* const* dst_bases, int world,
                                     int64_t dst_rows, int64_t row_bytes, int32_t* bad,
                                     cudaStream_t st);
cudaError_t launch_combine_peer(const float* const* y_bases, int world, int64_t y_rows,
                                const int32_t* slot_rank, const int64_t* slot_row,
                                const float* topk_w, const uint16_t* residual, uint16_t* out,
                                int64_t T, int H, int k, int32_t* bad, cudaStream_t st);

int num_sms();

// Host helpers of the C ABI (moe_api.cu): shape validation returning a moe_status_t
// (message in moe_last_error), and setting the thread's moe_last_error message.
int validate_shape(const moe_shape_t* shape, Shape* out);
void set_error_message(const char* msg);

// ---- programmatic dependent launch ----
// Every kernel of the layer is launched with programmatic stream serialization: it
// may be scheduled while the previous kernel on the stream is still draining. Each
// kernel lets its own dependents launch at entry (pdl_trigger) and, before it
// touches global memory, waits until the previous grid has completed and its writes
// are visible (pdl_wait). Only launch latency and on-chip prologue work overlap.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace moe
