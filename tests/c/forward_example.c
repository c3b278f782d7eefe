/* The layer through the C ABI alone (include/moe.h + the CUDA runtime), as a C caller
 * uses it: allocate, size the workspace, run moe_forward on device buffers, run
 * moe_forward_host on host buffers, and check that both give the same bits; then check
 * that bad arguments come back as status codes with a message. Exit 0 on success.
 *
 *   cc forward_example.c -I include -I $CUDA/include -L $CUDA/lib64 -lcudart \
 *      <path>/libmoe.so -o forward_example && ./forward_example
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "moe.h"

#define CHECK_CUDA(x)                                                   \
  do {                                                                  \
    cudaError_t e_ = (x);                                               \
    if (e_ != cudaSuccess) {                                            \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));          \
      return 2;                                                         \
    }                                                                   \
  } while (0)
#define CHECK_MOE(x)                                                    \
  do {                                                                  \
    moe_status_t s_ = (x);                                              \
    if (s_ != MOE_OK) {                                                 \
      fprintf(stderr, "%s: status %d: %s\n", #x, (int)s_, moe_last_error()); \
      return 3;                                                         \
    }                                                                   \
  } while (0)

/* bf16 bits of a float (round to nearest even; the values here are finite) */
static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* deterministic values in [-scale, scale) */
static void fill(uint16_t* p, size_t n, uint64_t* state, float scale) {
  for (size_t i = 0; i < n; ++i) {
    *state = *state * 6364136223846793005ull + 1442695040888963407ull;
    const float u = (float)((*state >> 40) & 0xFFFFFF) / 16777216.0f;
    p[i] = to_bf16((2.0f * u - 1.0f) * scale);
  }
}

static void* upload(const void* host, size_t bytes) {
  void* d = NULL;
  if (cudaMalloc(&d, bytes) != cudaSuccess) return NULL;
  if (cudaMemcpy(d, host, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
  return d;
}

int main(void) {
  moe_shape_t shape;
  memset(&shape, 0, sizeof shape);
  shape.num_tokens = 96;
  shape.hidden_size = 256;
  shape.intermediate_size = 384;
  shape.num_experts = 8;
  shape.num_experts_per_tok = 2;
  const size_t T = 96, H = 256, I = 384, E = 8;

  uint64_t st = 12345;
  uint16_t* x = malloc(T * H * 2);
  uint16_t* res = malloc(T * H * 2);
  uint16_t* wr = malloc(E * H * 2);
  uint16_t* w1 = malloc(E * I * H * 2);
  uint16_t* w3 = malloc(E * I * H * 2);
  uint16_t* w2 = malloc(E * H * I * 2);
  fill(x, T * H, &st, 1.0f);
  fill(res, T * H, &st, 1.0f);
  fill(wr, E * H, &st, 0.1f);
  fill(w1, E * I * H, &st, 0.06f);
  fill(w3, E * I * H, &st, 0.06f);
  fill(w2, E * H * I, &st, 0.05f);

  void* dx = upload(x, T * H * 2);
  void* dres = upload(res, T * H * 2);
  void* dwr = upload(wr, E * H * 2);
  void* dw1 = upload(w1, E * I * H * 2);
  void* dw3 = upload(w3, E * I * H * 2);
  void* dw2 = upload(w2, E * H * I * 2);
  if (!dx || !dres || !dwr || !dw1 || !dw3 || !dw2) {
    fprintf(stderr, "device allocation or copy failed\n");
    return 2;
  }
  const size_t ws_bytes = moe_workspace_size_host(&shape);
  if (ws_bytes == 0) {
    fprintf(stderr, "moe_workspace_size_host rejected the shape: %s\n", moe_last_error());
    return 3;
  }
  void* ws = NULL;
  void* dout = NULL;
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMemset(ws, 0, 256));
  CHECK_CUDA(cudaMalloc(&dout, T * H * 2));

  /* device buffers */
  CHECK_MOE(moe_forward(&shape, dx, dwr, NULL, dw1, dw3, dw2, dres, dout, ws, ws_bytes, NULL));
  CHECK_CUDA(cudaDeviceSynchronize());
  CHECK_MOE(moe_device_status(ws, ws_bytes, NULL));
  uint16_t* out_dev = malloc(T * H * 2);
  CHECK_CUDA(cudaMemcpy(out_dev, dout, T * H * 2, cudaMemcpyDeviceToHost));

  /* host buffers (pinned) */
  uint16_t *hx, *hres, *hout;
  CHECK_CUDA(cudaMallocHost((void**)&hx, T * H * 2));
  CHECK_CUDA(cudaMallocHost((void**)&hres, T * H * 2));
  CHECK_CUDA(cudaMallocHost((void**)&hout, T * H * 2));
  memcpy(hx, x, T * H * 2);
  memcpy(hres, res, T * H * 2);
  CHECK_MOE(moe_forward_host(&shape, hx, dwr, NULL, dw1, dw3, dw2, hres, hout, ws, ws_bytes,
                             NULL));
  if (memcmp(hout, out_dev, T * H * 2) != 0) {
    fprintf(stderr, "moe_forward_host differs from moe_forward\n");
    return 4;
  }
  double sum = 0.0;
  for (size_t i = 0; i < T * H; ++i) {
    uint32_t u = (uint32_t)out_dev[i] << 16;
    float f;
    memcpy(&f, &u, 4);
    if (f != f) {
      fprintf(stderr, "NaN in the output\n");
      return 4;
    }
    sum += f;
  }

  /* bad arguments: a status code and a message, nothing launched */
  moe_shape_t bad = shape;
  bad.hidden_size = 100;
  if (moe_forward(&bad, dx, dwr, NULL, dw1, dw3, dw2, dres, dout, ws, ws_bytes, NULL) == MOE_OK ||
      strlen(moe_last_error()) == 0) {
    fprintf(stderr, "an invalid hidden_size was accepted\n");
    return 5;
  }
  if (moe_forward(&shape, dx, dwr, NULL, dw1, dw3, dw2, dres, dout, ws, 16, NULL) !=
      MOE_ERR_WORKSPACE) {
    fprintf(stderr, "a small workspace was accepted\n");
    return 5;
  }
  printf("ok: T=%zu H=%zu I=%zu E=%zu k=2, checksum %.6f\n", T, H, I, E, sum);
  return 0;
}
