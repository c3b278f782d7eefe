// Router + scoring, expert histogram, padded offsets, stable ranks and the gather of
// routed rows: the integer and HBM-bound steps of the sparse-MoE layer on sm_100a.
//
// Sources (nnterp encyclopedia, "Mixtral"): the router gives one logit per expert
// with no bias ("Values, by host", router_logits; "Attention has no window": no
// projection has a bias); softmax over all E in float32, keep the k largest, divide
// them by their sum, slot 0 the larger ("The router renormalizes its top 2, in
// float32"). The expert-contiguous row order is this library's own: stable on
// (expert, token, slot), groups padded to 128 rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Eight normed activations: bf16((x * r) * g), two float roundings then one bf16
// rounding; the router and the gather both use exactly this.
__device__ __forceinline__ uint4 norm8(uint4 xv, uint4 gv, float r) {
  const uint32_t xq[4] = {xv.x, xv.y, xv.z, xv.w}, gq[4] = {gv.x, gv.y, gv.z, gv.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fmul_rn(__fmul_rn(bf16_lo(xq[i]), r), bf16_lo(gq[i]));
    const float hi = __fmul_rn(__fmul_rn(bf16_hi(xq[i]), r), bf16_hi(gq[i]));
    o[i] = pack_bf16x2(lo, hi);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Router and scoring. S warps cooperate on one token (S = 1, 2, 4 or 8; S > 1 when
// there are too few tokens to keep the GPU busy): warp w of a token takes the w-th
// of S equal slices of x[t] and of every router row. Each lane accumulates its
// 8-element chunks in fp32 in a fixed order, a butterfly sum gives the warp's
// partial logits, and one thread adds the S partials in warp order, adds the bias,
// and scores: float32 softmax over all E, the k largest logits (ties to the lower
// expert index, slot 0 the largest), weights renormalised to sum to one.
//
// With NORM the router first norms its token (the block's RMSNorm before the
// mixture): r = 1 / sqrt(mean(x^2) + eps) over the whole row, then routes
// xn = bf16((x * r) * g) instead of x, and stores r for the gather, which forms the
// same xn with the same float operations.
template <int EMAX, int S, bool NORM>
__global__ void __launch_bounds__(256) k_router(const uint16_t* __restrict__ x,
                                                const uint16_t* __restrict__ wr,
                                                const float* __restrict__ bias, int64_t T,
                                                int H, int E, int k,
                                                int32_t* __restrict__ idx_out,
                                                float* __restrict__ w_out,
                                                float* __restrict__ logits_out,
                                                const uint16_t* __restrict__ norm_w, float eps,
                                                float* __restrict__ rnorm_out, int bf16_logits) {
  pdl_trigger();
  pdl_wait();
  constexpr int TOK_PER_CTA = 8 / S;
  __shared__ float part[8][EMAX];
  __shared__ float part_ss[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp / S, sub = warp % S;
  const int per = (H >> 3) / S;  // 8-element chunks per warp; H % 128 == 0 keeps it whole
  for (int64_t t0 = (int64_t)blockIdx.x * TOK_PER_CTA; t0 < T;
       t0 += (int64_t)gridDim.x * TOK_PER_CTA) {
    const int64_t t = t0 + slot;
    float acc[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[e] = 0.f;
    float rn = 1.f;
    if (NORM) {
      float ss = 0.f;
      if (t < T) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * H) + sub * per;
        for (int c = lane; c < per; c += 32) {
          const uint4 xv = __ldg(xr + c);
          const uint32_t q[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = bf16_lo(q[i]), b = bf16_hi(q[i]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (S > 1) {
        if (lane == 0) part_ss[warp] = ss;
        __syncthreads();
        ss = part_ss[slot * S];
#pragma unroll
        for (int w = 1; w < S; ++w) ss += part_ss[slot * S + w];
      }
      rn = rsqrtf(ss / (float)H + eps);
      if (sub == 0 && lane == 0 && t < T) rnorm_out[t] = rn;
    }
    if (t < T) {
      const uint4* xr = reinterpret_cast<const uint4*>(x + t * H) + sub * per;
      const uint4* wrow = reinterpret_cast<const uint4*>(wr) + sub * per;
      const uint4* grow = reinterpret_cast<const uint4*>(norm_w) + sub * per;
      const int rstride = H >> 3;
      // router rows in groups of 8: all loads of a group are issued before any use
      // (rows past E read row E-1 and are discarded), so they overlap in flight
      for (int c = lane; c < per; c += 32) {
        uint4 xv = NORM ? __ldg(xr + c) : ld_stream(xr + c);
        if (NORM) xv = norm8(xv, __ldg(grow + c), rn);
        const float x0 = bf16_lo(xv.x), x1 = bf16_hi(xv.x), x2 = bf16_lo(xv.y), x3 = bf16_hi(xv.y);
        const float x4 = bf16_lo(xv.z), x5 = bf16_hi(xv.z), x6 = bf16_lo(xv.w), x7 = bf16_hi(xv.w);
#pragma unroll
        for (int e0 = 0; e0 < EMAX; e0 += 8) {
          if (e0 < E) {
            uint4 wv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int row = e0 + q < E ? e0 + q : E - 1;
              wv[q] = __ldg(wrow + (size_t)row * rstride + c);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float a = acc[e0 + q];
              a = fmaf(x0, bf16_lo(wv[q].x), a);
              a = fmaf(x1, bf16_hi(wv[q].x), a);
              a = fmaf(x2, bf16_lo(wv[q].y), a);
              a = fmaf(x3, bf16_hi(wv[q].y), a);
              a = fmaf(x4, bf16_lo(wv[q].z), a);
              a = fmaf(x5, bf16_hi(wv[q].z), a);
              a = fmaf(x6, bf16_lo(wv[q].w), a);
              a = fmaf(x7, bf16_hi(wv[q].w), a);
              acc[e0 + q] = a;
            }
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    if (S > 1) {
      if (lane == 0) {
#pragma unroll
        for (int e = 0; e < EMAX; ++e) part[warp][e] = acc[e];
      }
      __syncthreads();
    }
    if (sub == 0 && lane == 0 && t < T) {
      float l[EMAX], p[EMAX];
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        if (e < E) {
          float v = acc[e];
          if (S > 1) {
            v = part[slot * S][e];
#pragma unroll
            for (int w = 1; w < S; ++w) v += part[slot * S + w][e];
          }
          if (bf16_logits) v = __bfloat162float(__float2bfloat16_rn(v));
          l[e] = v + (bias ? bias[e] : 0.f);
          mx = fmaxf(mx, l[e]);
          if (logits_out) logits_out[t * E + e] = l[e];
        }
      }
      // float32 softmax over all E experts
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E) { p[e] = expf(l[e] - mx); sum += p[e]; }
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E) p[e] = p[e] / sum;
      // the k largest, ranked on the float32 logit; equal logits -> lower index
      uint64_t taken = 0;
      int sel[8];
      float psel[8];
      float psum = 0.f;
      for (int j = 0; j < k; ++j) {
        int best = -1;
        float bl = 0.f, bp = 0.f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
          if (e < E && !((taken >> e) & 1ull) && (best < 0 || l[e] > bl)) {
            best = e;
            bl = l[e];
            bp = p[e];
          }
        }
        taken |= 1ull << best;
        sel[j] = best;
        psel[j] = bp;
        psum += bp;
      }
      for (int j = 0; j < k; ++j) {
        idx_out[t * k + j] = sel[j];
        w_out[t * k + j] = psel[j] / psum;
      }
    }
    if (S > 1) __syncthreads();
  }
}

// Lanes of this warp (one token each) whose routed slots include expert e.
__device__ __forceinline__ unsigned expert_lanes(const int* my, int k, bool valid, int e) {
  unsigned bits = 0;
  for (int j = 0; j < k; ++j) bits |= __ballot_sync(0xffffffffu, valid && my[j] == e);
  return bits;
}

// Per token block (32 tokens, one warp): count of routed slots per expert.
__global__ void __launch_bounds__(256) k_block_hist(const int32_t* __restrict__ idx, int64_t T,
                                                    int E, int k, int64_t nb,
                                                    int32_t* __restrict__ block_counts) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t b = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (b >= nb) return;
  const int64_t t = b * kTokensPerBlock + lane;
  const bool valid = t < T;
  int my[8];
  for (int j = 0; j < k; ++j) my[j] = valid ? idx[t * k + j] : -1;
  for (int e = 0; e < E; ++e) {
    const unsigned bits = expert_lanes(my, k, valid, e);
    if (lane == 0) block_counts[b * E + e] = __popc(bits);
  }
}

// One CTA: per-expert exclusive prefix over token blocks (in place), total counts,
// and the padded group offsets; then every block base is shifted by its group's
// offset.
__global__ void __launch_bounds__(1024) k_scan(int32_t* __restrict__ block_base, int64_t nb,
                                               int E, int32_t* __restrict__ counts,
                                               int32_t* __restrict__ offsets) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t s_count[64];
  __shared__ int32_t s_off[65];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int e = warp; e < E; e += nwarps) {
    int32_t run = 0;
    for (int64_t b0 = 0; b0 < nb; b0 += 32) {
      const int64_t b = b0 + lane;
      const int32_t v = b < nb ? block_base[b * E + e] : 0;
      int32_t incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += n;
      }
      if (b < nb) block_base[b * E + e] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_count[e] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = acc;
      acc += (s_count[e] + kRowPad - 1) / kRowPad * kRowPad;
    }
    s_off[E] = acc;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    offsets[e] = s_off[e];
    if (e < E) counts[e] = s_count[e];
  }
  for (int64_t i = threadIdx.x; i < nb * E; i += blockDim.x) block_base[i] += s_off[i % E];
}

// Per token block: the stable rank of each routed slot among its expert's slots,
// hence its row; writes row_of and token_of_row for real rows.
__global__ void __launch_bounds__(256) k_rank(const int32_t* __restrict__ idx, int64_t T, int E,
                                              int k, int64_t nb,
                                              const int32_t* __restrict__ block_base,
                                              int32_t* __restrict__ row_of,
                                              int32_t* __restrict__ token_of_row) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t b = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (b >= nb) return;
  const int64_t t = b * kTokensPerBlock + lane;
  const bool valid = t < T;
  int my[8];
  for (int j = 0; j < k; ++j) my[j] = valid ? idx[t * k + j] : -1;
  const unsigned below = (1u << lane) - 1u;
  for (int e = 0; e < E; ++e) {
    const unsigned bits = expert_lanes(my, k, valid, e);
    if (!bits) continue;
    const int32_t base = block_base[b * E + e];
    // a token's k slots name k distinct experts, so at most one slot matches e
    for (int j = 0; j < k; ++j) {
      if (valid && my[j] == e) {
        const int32_t row = base + __popc(bits & below);
        row_of[t * k + j] = row;
        token_of_row[row] = (int32_t)t;
      }
    }
  }
}

// Histogram, scan and ranks in one CTA when there are at most 32 token blocks
// (T <= 1024): warp b counts its block's slots per expert with ballots, one thread per
// expert prefixes the block counts in order, thread 0 lays out the padded groups,
// then every warp ranks its slots. Same results as k_block_hist + k_scan + k_rank.
__global__ void __launch_bounds__(1024) k_plan_small(const int32_t* __restrict__ idx, int64_t T,
                                                     int E, int k, int nb,
                                                     int32_t* __restrict__ counts,
                                                     int32_t* __restrict__ offsets,
                                                     int32_t* __restrict__ row_of,
                                                     int32_t* __restrict__ token_of_row) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t s_base[32][64];
  __shared__ int32_t s_tot[64];
  __shared__ int32_t s_off[65];
  const int b = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = (int64_t)b * kTokensPerBlock + lane;
  const bool active = b < nb;
  const bool valid = active && t < T;
  int my[8];
  for (int j = 0; j < k; ++j) my[j] = valid ? idx[t * k + j] : -1;
  if (active) {
    for (int e = 0; e < E; ++e) {
      const unsigned bits = expert_lanes(my, k, valid, e);
      if (lane == 0) s_base[b][e] = __popc(bits);
    }
  }
  __syncthreads();
  if (threadIdx.x < E) {
    const int e = threadIdx.x;
    int32_t run = 0;
    for (int bb = 0; bb < nb; ++bb) {
      const int32_t v = s_base[bb][e];
      s_base[bb][e] = run;
      run += v;
    }
    s_tot[e] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = acc;
      acc += (s_tot[e] + kRowPad - 1) / kRowPad * kRowPad;
    }
    s_off[E] = acc;
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    offsets[e] = s_off[e];
    if (e < E) counts[e] = s_tot[e];
  }
  if (active) {
    const unsigned below = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
      const unsigned bits = expert_lanes(my, k, valid, e);
      if (!bits) continue;
      const int32_t base = s_off[e] + s_base[b][e];
      for (int j = 0; j < k; ++j) {
        if (valid && my[j] == e) {
          const int32_t row = base + __popc(bits & below);
          row_of[t * k + j] = row;
          token_of_row[row] = (int32_t)t;
        }
      }
    }
  }
}

// 8 bf16 values -> 8 IEEE half values (round to nearest even; exact for magnitudes in
// [2^-14, 65504], larger ones become infinite).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint4 to_f16x8(uint4 v) {
  return make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y), bf16x2_to_f16x2(v.z),
                    bf16x2_to_f16x2(v.w));
}

// One warp per row of x_perm below R_pad: copies x[token] (as bf16, or converted to
// float16 when F16) or, on pad rows, writes zeros and token -1.
template <bool NORM, bool F16>
__global__ void __launch_bounds__(256) k_gather(const uint16_t* __restrict__ x, int H, int E,
                                                const int32_t* __restrict__ counts,
                                                const int32_t* __restrict__ offsets,
                                                int32_t* __restrict__ token_of_row,
                                                uint16_t* __restrict__ x_perm,
                                                const uint16_t* __restrict__ norm_w,
                                                const float* __restrict__ rnorm,
                                                int32_t* __restrict__ zero_buf, int zero_n) {
  pdl_trigger();
  pdl_wait();
  // the expert GEMMs' sub-tile counters start at zero (their previous users have
  // finished: every kernel before this one in the stream has)
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < zero_n; i += blockDim.x) zero_buf[i] = 0;
  __shared__ int32_t s_off[65], s_cnt[64];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    s_off[e] = offsets[e];
    if (e < E) s_cnt[e] = counts[e];
  }
  __syncthreads();
  const int64_t rows = s_off[E];
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int chunks = H >> 3;
  for (int64_t r = w0; r < rows; r += nw) {
    int e = 0;
    while (e + 1 < E && s_off[e + 1] <= r) ++e;
    const bool pad = r >= s_off[e] + s_cnt[e];
    uint4* dst = reinterpret_cast<uint4*>(x_perm + r * H);
    if (pad) {
      if (lane == 0) token_of_row[r] = -1;
      for (int c = lane; c < chunks; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
    } else if (NORM) {
      const int64_t t = token_of_row[r];
      const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
      const uint4* g = reinterpret_cast<const uint4*>(norm_w);
      const float rn = rnorm[t];
      for (int c = lane; c < chunks; c += 32) {
        const uint4 v = norm8(__ldg(src + c), __ldg(g + c), rn);
        dst[c] = F16 ? to_f16x8(v) : v;
      }
    } else if (F16) {
      const int64_t t = token_of_row[r];
      const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
      for (int c = lane; c < chunks; c += 32) dst[c] = to_f16x8(__ldg(src + c));
    } else {
      const int64_t t = token_of_row[r];
      const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
      int c = lane;
      for (; c + 96 < chunks; c += 128) {
        const uint4 a = __ldg(src + c), b2 = __ldg(src + c + 32), c2 = __ldg(src + c + 64),
                    d = __ldg(src + c + 96);
        dst[c] = a;
        dst[c + 32] = b2;
        dst[c + 64] = c2;
        dst[c + 96] = d;
      }
      for (; c < chunks; c += 32) dst[c] = __ldg(src + c);
    }
  }
}

}  // namespace

cudaError_t launch_router(const Shape& s, const uint16_t* x, const uint16_t* w_router,
                          const float* logit_bias, int32_t* topk_idx, float* topk_w,
                          float* logits, cudaStream_t st, const uint16_t* norm_w, float eps,
                          float* rnorm) {
  // enough warps to cover the GPU: split each token over S warps when T is small
  const int64_t want_warps = (int64_t)num_sms() * 32;
  int S = 1;
  while (S < 8 && s.T * S < want_warps) S *= 2;
  const int64_t tok_per_cta = 8 / S;
  int64_t blocks = (s.T + tok_per_cta - 1) / tok_per_cta;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  cudaError_t err = cudaSuccess;
#define MOE_ROUTER(EM, SS)                                                                    \
  err = norm_w ? launch_pdl(k_router<EM, SS, true>, dim3((unsigned)blocks), dim3(256), 0, st, x,  \
                            w_router, logit_bias, s.T, s.H, s.E, s.k, topk_idx, topk_w, logits, \
                            norm_w, eps, rnorm, s.bf16_logits)                                  \
               : launch_pdl(k_router<EM, SS, false>, dim3((unsigned)blocks), dim3(256), 0, st, x, \
                            w_router, logit_bias, s.T, s.H, s.E, s.k, topk_idx, topk_w, logits, \
                            norm_w, eps, rnorm, s.bf16_logits)
#define MOE_ROUTER_E(EM)           \
  switch (S) {                     \
    case 1: MOE_ROUTER(EM, 1); break; \
    case 2: MOE_ROUTER(EM, 2); break; \
    case 4: MOE_ROUTER(EM, 4); break; \
    default: MOE_ROUTER(EM, 8); break; \
  }
  if (s.E <= 8) { MOE_ROUTER_E(8) }
  else if (s.E <= 16) { MOE_ROUTER_E(16) }
  else if (s.E <= 32) { MOE_ROUTER_E(32) }
  else { MOE_ROUTER_E(64) }
#undef MOE_ROUTER_E
#undef MOE_ROUTER
  return err;
}

cudaError_t launch_permute(const Shape& s, const int32_t* topk_idx, const uint16_t* x,
                           int32_t* counts, int32_t* offsets, int32_t* row_of,
                           int32_t* token_of_row, uint16_t* x_perm, int32_t* block_base,
                           cudaStream_t st, const uint16_t* norm_w, const float* rnorm,
                           bool f16_out, int32_t* zero_buf, int zero_n) {
  const int64_t nb = num_token_blocks(s);
  cudaError_t e;
  if (nb <= 32) {
    const int threads = (int)(nb < 2 ? 2 : nb) * 32;
    e = launch_pdl(k_plan_small, dim3(1), dim3(threads), 0, st, topk_idx, s.T, s.E, s.k, (int)nb,
                   counts, offsets, row_of, token_of_row);
    if (e != cudaSuccess) return e;
  } else {
    const unsigned wblocks = (unsigned)((nb + 7) / 8);
    e = launch_pdl(k_block_hist, dim3(wblocks), dim3(256), 0, st, topk_idx, s.T, s.E, s.k, nb,
                   block_base);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_scan, dim3(1), dim3(1024), 0, st, block_base, nb, s.E, counts, offsets);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_rank, dim3(wblocks), dim3(256), 0, st, topk_idx, s.T, s.E, s.k, nb, block_base,
                   row_of, token_of_row);
    if (e != cudaSuccess) return e;
  }
  int64_t gblocks = (max_padded_rows(s) + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (gblocks > cap) gblocks = cap;
#define MOE_GATHER(NM, FH)                                                                   \
  launch_pdl(k_gather<NM, FH>, dim3((unsigned)gblocks), dim3(256), 0, st, x, s.H, s.E, counts, \
             offsets, token_of_row, x_perm, norm_w, rnorm, zero_buf, zero_n)
  if (norm_w) return f16_out ? MOE_GATHER(true, true) : MOE_GATHER(true, false);
  return f16_out ? MOE_GATHER(false, true) : MOE_GATHER(false, false);
#undef MOE_GATHER
}

}  // namespace moe
