// Row gather: dst[i] = src[index[i]], rows of row_bytes bytes. Used by the
// expert-parallel layer to regroup the rows one rank receives from every peer
// (ordered by source rank, then expert) into expert-contiguous groups, and back.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {
namespace {

// One warp per destination row, 16-byte vectors. An index outside [0, src_rows) writes
// a zero row, so no read ever leaves the source buffer.
__global__ void __launch_bounds__(256) k_gather_rows(const uint4* __restrict__ src,
                                                     uint4* __restrict__ dst,
                                                     const int64_t* __restrict__ index,
                                                     int64_t n_rows, int64_t src_rows,
                                                     int64_t row_vecs) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = w0; r < n_rows; r += nw) {
    const int64_t s = index[r];
    uint4* d = dst + r * row_vecs;
    if (s < 0 || s >= src_rows) {
      for (int64_t c = lane; c < row_vecs; c += 32) d[c] = make_uint4(0, 0, 0, 0);
    } else {
      const uint4* p = src + s * row_vecs;
      for (int64_t c = lane; c < row_vecs; c += 32) d[c] = __ldg(p + c);
    }
  }
}

}  // namespace

cudaError_t launch_gather_rows(const void* src, void* dst, const int64_t* index, int64_t n_rows,
                               int64_t src_rows, int64_t row_bytes, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  int64_t blocks = (n_rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_gather_rows, dim3((unsigned)blocks), dim3(256), 0, st,
                    static_cast<const uint4*>(src), static_cast<uint4*>(dst), index, n_rows,
                    src_rows, row_bytes / 16);
}

}  // namespace moe
