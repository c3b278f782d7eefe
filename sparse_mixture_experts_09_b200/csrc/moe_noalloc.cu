// moe_permute_static: moe_permute for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a device workspace: code running inside a host
// whose allocator it does not own (a plug-in loaded into another framework's
// process, a real-time path that must not call into the driver's allocator), or a
// caller that has to size everything before it knows the batch. This entry point
// takes only the inputs and outputs of the permutation. The one piece of scratch the
// permutation needs for more than 32 token blocks, the per-block expert base table
// (num_token_blocks x num_experts int32), lives in the file-scope device array
// below, which every GPU that loads this library keeps until the process exits.
//
// The array is shared by every call: calls whose kernels overlap on the GPU (two
// streams, two host threads) race on it and must be serialised by the caller. Every
// entry of the table that a call reads is first written by the same call, so nothing
// has to be cleared between calls.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <mutex>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

// Capacity of the shared table: num_token_blocks * num_experts int32 entries, with
// num_token_blocks = ceil(num_tokens / 32) (256 KiB).
constexpr int64_t kStaticScratchInts = 65536;

static __device__ __align__(256) int32_t g_permute_scratch[kStaticScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {};

moe_status_t fail(moe_status_t code, const char* fmt, ...) {
  char msg[256];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof msg, fmt, ap);
  va_end(ap);
  set_error_message(msg);
  return code;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

moe_status_t moe_permute_static(const moe_shape_t* shape, const int32_t* topk_idx,
                                const moe_bf16_t* x, int32_t* expert_counts,
                                int32_t* expert_offsets, int32_t* row_of, int32_t* token_of_row,
                                moe_bf16_t* x_perm, moe_stream_t stream) {
  set_error_message("");
  Shape s;
  const int st = validate_shape(shape, &s);
  if (st != MOE_OK) return (moe_status_t)st;
  if (!topk_idx || !x || !expert_counts || !expert_offsets || !row_of || !token_of_row || !x_perm)
    return fail(MOE_ERR_INVALID_ARG, "a required pointer is NULL");
  const uintptr_t any = reinterpret_cast<uintptr_t>(topk_idx) | reinterpret_cast<uintptr_t>(x) |
                        reinterpret_cast<uintptr_t>(expert_counts) |
                        reinterpret_cast<uintptr_t>(expert_offsets) |
                        reinterpret_cast<uintptr_t>(row_of) |
                        reinterpret_cast<uintptr_t>(token_of_row) |
                        reinterpret_cast<uintptr_t>(x_perm);
  if (any % 16) return fail(MOE_ERR_INVALID_ARG, "every pointer must be 16-byte aligned");
  const int64_t need = num_token_blocks(s) * s.E;
  if (num_token_blocks(s) > 32 && need > kStaticScratchInts)
    return fail(MOE_ERR_UNSUPPORTED,
                "shape needs %lld scratch entries (ceil(num_tokens/32) * num_experts) but the "
                "static table holds %lld; use moe_permute with a workspace",
                (long long)need, (long long)kStaticScratchInts);
  // once per device, with that device current: the device address of the table, kept
  // for the life of the process (a cudaDeviceReset would make it stale; the header
  // rules that out)
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index %d too large", dev);
  int32_t* scratch;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_permute_scratch);
      if (e != cudaSuccess || !ptr)
        return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      g_scratch_ptr[dev] = static_cast<int32_t*>(ptr);
    }
    scratch = g_scratch_ptr[dev];
  }
  e = launch_permute(s, topk_idx, x, expert_counts, expert_offsets, row_of, token_of_row, x_perm,
                     scratch, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "permute launch: %s", cudaGetErrorString(e));
  return MOE_OK;
}

}  // extern "C"
