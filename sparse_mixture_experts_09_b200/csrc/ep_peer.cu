// Expert parallelism over peer memory: the exchange steps of the expert-parallel layer
// as plain loads and stores into other ranks' buffers (CUDA IPC mappings over NVLink
// between GPUs), instead of an all-to-all followed by regrouping gathers.
//
// The pages say only that a config's experts may be spread over devices (Hugging Face
// "Mixtral", MixtralConfig num_local_experts); how the rows move is this library's own
// design. The arithmetic of the combine is the single-device layer's (k_combine): fp32,
// slots in order, one rounding to bf16 after the residual.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {
namespace {

// One warp per row: dst_bases[dst_rank[i]] row dst_row[i] = src row src_index[i]. Rows
// whose source, rank or destination index is out of range are skipped and counted in
// *bad (when given), so no access leaves the buffers the caller described.
__global__ void __launch_bounds__(256) k_scatter_rows_peer(
    const uint4* __restrict__ src, int64_t src_rows, const int64_t* __restrict__ src_index,
    const int32_t* __restrict__ dst_rank, const int64_t* __restrict__ dst_row, int64_t n_rows,
    uint4* const* __restrict__ dst_bases, int world, int64_t dst_rows, int64_t row_vecs,
    int32_t* bad) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t i = w0; i < n_rows; i += nw) {
    const int64_t s = src_index[i], d = dst_row[i];
    const int r = dst_rank[i];
    if (s < 0 || s >= src_rows || r < 0 || r >= world || d < 0 || d >= dst_rows) {
      if (lane == 0 && bad) atomicAdd(bad, 1);
      continue;
    }
    const uint4* p = src + s * row_vecs;
    uint4* q = dst_bases[r] + d * row_vecs;
    for (int64_t c = lane; c < row_vecs; c += 32) q[c] = __ldg(p + c);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One thread per 8 consecutive outputs of a token: slot j of token t reads row
// slot_row[t k + j] of rank slot_rank[t k + j]'s y buffer (plain loads: the buffer may
// be another GPU's), out = bf16(residual + sum_j w_j y_j) with the sum in slot order.
// A slot whose rank or row is out of range adds nothing and is counted in *bad.
template <int KMAX>
__global__ void __launch_bounds__(256) k_combine_peer(
    const float* const* __restrict__ y_bases, int world, int64_t y_rows,
    const int32_t* __restrict__ slot_rank, const int64_t* __restrict__ slot_row,
    const float* __restrict__ w, const uint16_t* __restrict__ res, uint16_t* __restrict__ out,
    int64_t T, int H, int k, int32_t* bad) {
  pdl_trigger();
  pdl_wait();
  const int per_tok = H >> 3;
  const int64_t n = T * per_tok;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_tok;
    const int c = (int)(i - t * per_tok) * 8;
    const bool first = c == 0;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    float4 ya[KMAX], yb[KMAX];
    float wj[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ya[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      yb[j] = ya[j];
      wj[j] = 0.f;
      if (j < k) {
        const int r = slot_rank[t * k + j];
        const int64_t row = slot_row[t * k + j];
        if (r >= 0 && r < world && row >= 0 && row < y_rows) {
          const float4* yp = reinterpret_cast<const float4*>(y_bases[r] + row * H + c);
          ya[j] = yp[0];
          yb[j] = yp[1];
          wj[j] = w[t * k + j];
        } else if (first && bad) {
          atomicAdd(bad, 1);
        }
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

cudaError_t launch_scatter_rows_peer(const void* src, int64_t src_rows, const int64_t* src_index,
                                     const int32_t* dst_rank, const int64_t* dst_row,
                                     int64_t n_rows, void* const* dst_bases, int world,
                                     int64_t dst_rows, int64_t row_bytes, int32_t* bad,
                                     cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  int64_t blocks = (n_rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_scatter_rows_peer, dim3((unsigned)blocks), dim3(256), 0, st,
                    static_cast<const uint4*>(src), src_rows, src_index, dst_rank, dst_row, n_rows,
                    reinterpret_cast<uint4* const*>(dst_bases), world, dst_rows, row_bytes / 16,
                    bad);
}

cudaError_t launch_combine_peer(const float* const* y_bases, int world, int64_t y_rows,
                                const int32_t* slot_rank, const int64_t* slot_row,
                                const float* topk_w, const uint16_t* residual, uint16_t* out,
                                int64_t T, int H, int k, int32_t* bad, cudaStream_t st) {
  const int64_t n = T * (H / 8);
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 32;
  if (blocks > cap) blocks = cap;
#define MOE_COMBINE_PEER(KM)                                                                 \
  launch_pdl(k_combine_peer<KM>, dim3((unsigned)blocks), dim3(256), 0, st, y_bases, world, \
             y_rows, slot_rank, slot_row, topk_w, residual, out, T, H, k, bad)
  if (k <= 2) return MOE_COMBINE_PEER(2);
  if (k <= 4) return MOE_COMBINE_PEER(4);
  return MOE_COMBINE_PEER(8);
#undef MOE_COMBINE_PEER
}

}  // namespace moe
