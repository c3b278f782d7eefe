// Weighted combine into the residual.
//
// nnterp encyclopedia, "Mixtral": each slot's expert output is scaled by its float32
// weight ("Values, by host", expert_outputs), the slots sum to routed_output
// ("expert_outputs needs the default experts implementation"), and the block adds
// it to the residual stream ("The block, in order"). Here the sum runs in fp32 in
// slot order and the result is rounded to bf16 once.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One thread per 8 consecutive outputs of a token: reads k rows of y (32 B each)
// and 16 B of residual, writes 16 B.
template <int KMAX>
__global__ void __launch_bounds__(256) k_combine(const float* __restrict__ y,
                                                 const int32_t* __restrict__ row_of,
                                                 const float* __restrict__ w,
                                                 const uint16_t* __restrict__ res,
                                                 uint16_t* __restrict__ out, int64_t T, int H,
                                                 int k) {
  pdl_trigger();
  pdl_wait();
  const int per_tok = H >> 3;
  const int64_t n = T * per_tok;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_tok;
    const int c = (int)(i - t * per_tok) * 8;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    // all rows' loads are issued before the first multiply-add; slots are then
    // accumulated in order
    int64_t r[KMAX];
    float wj[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        r[j] = row_of[t * k + j];
        wj[j] = w[t * k + j];
      }
    }
    float4 ya[KMAX], yb[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        const float4* yp = reinterpret_cast<const float4*>(y + r[j] * H + c);
        ya[j] = __ldg(yp);
        yb[j] = __ldg(yp + 1);
      }
    }
    uint4 rv = make_uint4(0, 0, 0, 0);
    if (res) rv = __ldg(reinterpret_cast<const uint4*>(res + t * H + c));
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        acc[0] = fmaf(wj[j], ya[j].x, acc[0]);
        acc[1] = fmaf(wj[j], ya[j].y, acc[1]);
        acc[2] = fmaf(wj[j], ya[j].z, acc[2]);
        acc[3] = fmaf(wj[j], ya[j].w, acc[3]);
        acc[4] = fmaf(wj[j], yb[j].x, acc[4]);
        acc[5] = fmaf(wj[j], yb[j].y, acc[5]);
        acc[6] = fmaf(wj[j], yb[j].z, acc[6]);
        acc[7] = fmaf(wj[j], yb[j].w, acc[7]);
      }
    }
    if (res) {
      const uint32_t rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = __uint_as_float(rr[q] << 16) + acc[2 * q];
        acc[2 * q + 1] = __uint_as_float(rr[q] & 0xFFFF0000u) + acc[2 * q + 1];
      }
    }
    uint4 o;
    o.x = pack_bf16x2_rn(acc[0], acc[1]);
    o.y = pack_bf16x2_rn(acc[2], acc[3]);
    o.z = pack_bf16x2_rn(acc[4], acc[5]);
    o.w = pack_bf16x2_rn(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(out + t * H + c) = o;
  }
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const float* y, const int32_t* row_of,
                           const float* topk_w, const uint16_t* residual, uint16_t* out,
                           cudaStream_t st) {
  const int64_t n = s.T * (s.H / 8);
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 32;
  if (blocks > cap) blocks = cap;
  if (s.k <= 2)
    return launch_pdl(k_combine<2>, dim3((unsigned)blocks), dim3(256), 0, st, y, row_of, topk_w,
                      residual, out, s.T, s.H, s.k);
  if (s.k <= 4)
    return launch_pdl(k_combine<4>, dim3((unsigned)blocks), dim3(256), 0, st, y, row_of, topk_w,
                      residual, out, s.T, s.H, s.k);
  return launch_pdl(k_combine<8>, dim3((unsigned)blocks), dim3(256), 0, st, y, row_of, topk_w,
                    residual, out, s.T, s.H, s.k);
}

}  // namespace moe
