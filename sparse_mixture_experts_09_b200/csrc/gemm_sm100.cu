// Persistent grouped GEMMs of the experts on sm_100a: TMA loads into 128-byte
// swizzled shared-memory stages, tcgen05.mma (kind::f16, bf16 in, fp32 accumulate)
// into tensor memory, a four-warp epilogue reading tensor memory with tcgen05.ld.
//
// The experts (nnterp encyclopedia, "Mixtral", "Values, by host"): mlp_neurons =
// act(gate x) * up x is what the down projection receives; act = silu (Hugging Face
// "Mixtral" doc, MixtralConfig hidden_act). The pages name a grouped matmul over
// the stacked experts as the default implementation ("expert_outputs needs the
// default experts implementation"); this is our own design of it for B200.
//
//   GEMM1 (kSwiGLU): for a 128-row tile of one expert's routed rows and 128
//     intermediate columns, B is the 128 w1 rows stacked on the 128 w3 rows, so one
//     M=128 x N=256 MMA chain yields gate (columns 0..127) and up (128..255) side by
//     side; the epilogue writes h = bf16(silu(gate) * up).
//   GEMM2 (kPlain): y = h w2^T for a 128-row tile and BN output columns, fp32 out.
//
// Roles per CTA (192 threads): warp 0 issues TMA, warp 1 owns tensor memory and
// issues MMAs, warps 2..5 drain accumulators. Two accumulators in tensor memory let
// the epilogue of one tile overlap the MMAs of the next. Tiles are visited in a
// static round-robin over a tile order that keeps an expert's rows together and
// walks its row tiles fastest, so concurrently running CTAs share weight tiles in L2.
//
// Every wait is bounded: after `timeout_ns` a role records kStatusTimeout in the
// device status word, raises a CTA-wide abort flag, and all roles unwind; the
// producer waits (bounded) for its copies in flight and the MMA warp for its MMAs
// before tensor memory is freed.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;        // bf16 elements per 128-byte swizzled row
constexpr int kThreads = 192;
#ifndef MOE_GEMM_STAGES
#define MOE_GEMM_STAGES 4
#endif
constexpr int kStages = MOE_GEMM_STAGES;
constexpr int kSwiGLU = 0;
constexpr int kPlain = 1;

template <int BN>
struct Tile {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + BAR_BYTES + 4 * 144;
  // instruction descriptor: D f32 (bit 4), A bf16 (bits 7-9 = 1), B bf16 (bits 10-12 = 1),
  // both K-major, N >> 3 at bit 17, M >> 4 at bit 24
  static constexpr uint32_t IDESC =
      (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
};

struct KParams {
  const int32_t* offsets;
  int32_t* status;
  void* out;
  int64_t out_ld;
  int E;
  int k_blocks;
  int n_tiles;
  int b_rows;  // rows of the B tensor per expert
  int blocked;  // weights in the blocked layout (MOE_WEIGHTS_BLOCKED)
  unsigned long long timeout_ns;
  // split-K (plain GEMM): counts [E] (null: no split), partial sums [kMaxSplitK, routed,
  // out_ld] fp32, arrival counters [kSplitSems]; routed = total routed rows
  const int32_t* counts;
  float* partial;
  int32_t* split_sem;
  int64_t routed;
  int32_t* zero_sem;  // gate/up: counters to zero for the down GEMM that follows (nullable)
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase. The MMA threads test the next stage's full barrier with
// it before issuing the current stage: measured on B200, a wait whose result steers the
// thread costs about 340 SM clocks between MMAs even on a completed phase, while the
// latency of a test issued ahead runs under the MMAs.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// shared-memory matrix descriptor, K-major, 128-byte swizzle: start address >> 4,
// leading byte offset 16 B (unused for swizzled K-major), stride byte offset 1024 B
// (one 8-row x 128-byte swizzle atom), version 1 (bit 46), layout SWIZZLE_128B = 2.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Bounded wait on an mbarrier phase. Returns false if the CTA aborted or the wait
// ran past timeout_ns (then it records the timeout and raises the abort flag).
__device__ __noinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        int32_t* status, unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > timeout_ns) {
        *abort_flag = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

// Bounded wait used while unwinding: ignores the abort flag; if it runs out too, it
// records kStatusUnwound.
__device__ __noinline__ void drain_phase(uint32_t bar, uint32_t parity, int32_t* status,
                                         unsigned long long timeout_ns) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > timeout_ns) {
      atomicOr(status, kStatusUnwound);
      return;
    }
  }
}

// Tensor-map coordinates (x, y) of weight row `row`, k-block `kb`. Row-major weights
// are a [rows, K] map; blocked weights ([rows/128][K/64][128][64], each 128 x 64 block
// one contiguous 16 KiB run) are a [rows * K/64, 64] map, so every TMA box of up to
// 128 rows reads contiguous memory.
__device__ __forceinline__ void wcoord(int kb, int row, int k_blocks, int blocked, int& x, int& y) {
  if (blocked) {
    x = 0;
    y = ((row >> 7) * k_blocks + kb) * 128 + (row & 127);
  } else {
    x = kb * BK;
    y = row;
  }
}

// Tile L -> (expert e, row tile m, column tile n). row_tiles[e] = offsets[e] / 128.
// Tiles of expert e occupy [row_tiles[e] * n_tiles, row_tiles[e+1] * n_tiles) and
// walk the expert's row tiles fastest.
__device__ __forceinline__ void tile_coords(int L, const int* row_tiles, int E, int n_tiles, int& e,
                                            int& m, int& n) {
  const int mrow = L / n_tiles;
  e = 0;
  while (e + 1 < E && row_tiles[e + 1] <= mrow) ++e;
  const int cnt = row_tiles[e + 1] - row_tiles[e];
  const int local = L - row_tiles[e] * n_tiles;
  n = local / cnt;
  m = row_tiles[e] + local % cnt;
}

// Work items. Whole waves of tiles run at full width (item = tile, round-robin over
// the CTAs). When the tiles left over for the last wave would fill at most half of the
// CTAs, each of them is cut into `split` (2 or 4) pieces along N, so the last wave is
// shorter by that factor and more CTAs share it. When split-K is allowed (max_ksplit >
// 1) and the tiles do not fill one wave, each tile is instead cut into `ksplit` parts
// along K (items tile * ksplit + part), ksplit chosen to minimise waves per part, at
// least kMinSplitKBlocks k-blocks per part, the fewest parts on a tie, and taken only
// when it shortens the GEMM to at most 3/4 of one wave of whole tiles (measured on
// B200: 8 parts for 128 tiles on 148 SMs, 7/8 on paper, ran 4% slower; 3 parts for 48
// tiles cut a one-token layer by 22%).
constexpr int kMinSplitKBlocks = 8;

struct Work {
  int full_items, split, items, ksplit;
  __device__ void init(int total_tiles, int grid, int max_ksplit = 1, int k_blocks = 0) {
    ksplit = 1;
    if (max_ksplit > 1 && total_tiles > 0 && total_tiles < grid) {
      int best_waves = 1;  // ksplit = 1: one wave of whole tiles
      for (int s = 2; s <= max_ksplit && k_blocks / s >= kMinSplitKBlocks; ++s) {
        const int waves = (total_tiles * s + grid - 1) / grid;
        if (waves * ksplit < best_waves * s) {  // waves / s < best_waves / ksplit
          best_waves = waves;
          ksplit = s;
        }
      }
      if (4 * best_waves > 3 * ksplit) ksplit = 1;
    }
    if (ksplit > 1) {
      full_items = 0;
      split = 1;
      items = total_tiles * ksplit;
      return;
    }
    full_items = (total_tiles / grid) * grid;
    const int rest = total_tiles - full_items;
    split = 1;
    if (rest > 0) {
      if (4 * rest <= grid) split = 4;
      else if (2 * rest <= grid) split = 2;
    }
    items = full_items + split * rest;
  }
  // item -> (tile, piece, pieces, K part)
  __device__ void get(int item, int& tile, int& piece, int& pieces, int& part) const {
    part = 0;
    if (ksplit > 1) {
      tile = item / ksplit;
      part = item - tile * ksplit;
      piece = 0;
      pieces = 1;
      return;
    }
    if (item < full_items) {
      tile = item;
      piece = 0;
      pieces = 1;
    } else {
      const int j = item - full_items;
      tile = full_items + j / split;
      piece = j % split;
      pieces = split;
    }
  }
};

template <int MODE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                   const __grid_constant__ CUtensorMap mapB1,
                   const __grid_constant__ CUtensorMap mapB0s,
                   const __grid_constant__ CUtensorMap mapB1s, const KParams p) {
  using C = Tile<BN>;
  // B rows of one weight matrix in a full tile: 128 w1 and 128 w3 rows (gate/up),
  // or BN w2 rows (down)
  constexpr int ROWS = (MODE == kSwiGLU) ? 128 : BN;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * C::STAGE_BYTES);
  // bars: full[kStages], empty[kStages], tfull[2], tempty[2], final
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* row_tiles = reinterpret_cast<int*>(tmem_holder + 2);
  int* routed_start = row_tiles + 72;  // split-K: first compact routed row of each expert

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 + a); };
  const uint32_t final_bar = bar0 + 8u * (2 * kStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    prefetch_map(&mapA);
    prefetch_map(&mapB0);
    prefetch_map(&mapB1);
    prefetch_map(&mapB0s);
    prefetch_map(&mapB1s);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // everything above is on-chip set-up; global inputs are read only after the
  // previous kernel on the stream has completed
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) row_tiles[i] = p.offsets[i] / BM;
  if (p.zero_sem && blockIdx.x == 0)
    for (int i = threadIdx.x; i < kSplitSems; i += blockDim.x) p.zero_sem[i] = 0;
  if (p.counts && threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < p.E; ++e) {
      routed_start[e] = acc;
      acc += p.counts[e];
    }
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_holder;
  Work work;
  work.init(row_tiles[p.E] * p.n_tiles, gridDim.x, (MODE == kPlain && p.counts) ? kMaxSplitK : 1,
            p.k_blocks);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < work.items && ok; w += gridDim.x) {
        int tile, piece, pieces, part, e, m, n;
        work.get(w, tile, piece, pieces, part);
        tile_coords(tile, row_tiles, p.E, p.n_tiles, e, m, n);
        const int a_row = m * BM;
        const int rp = ROWS / pieces;  // B rows per weight matrix in this item
        const int b_row = e * p.b_rows + n * ROWS + piece * rp;
        const uint32_t bytes = C::A_BYTES + (MODE == kSwiGLU ? 2 : 1) * rp * BK * 2;
        const int kb_end = (part + 1) * p.k_blocks / work.ksplit;
        for (int kb = part * p.k_blocks / work.ksplit; kb < kb_end; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!wait_phase(empty_bar(s), ph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
          mbar_expect_tx(full_bar(s), bytes);
          tma_load_2d(sa, &mapA, kb * BK, a_row, full_bar(s));
          int wx, wy;
          if (pieces == 1) {
            wcoord(kb, b_row, p.k_blocks, p.blocked, wx, wy);
            if (MODE == kSwiGLU) {
              tma_load_2d(sb, &mapB0, wx, wy, full_bar(s));
              tma_load_2d(sb + 128 * BK * 2, &mapB1, wx, wy, full_bar(s));
            } else {
              tma_load_2d(sb, &mapB0, wx, wy, full_bar(s));
              if (BN == 256) {
                wcoord(kb, b_row + 128, p.k_blocks, p.blocked, wx, wy);
                tma_load_2d(sb + 128 * BK * 2, &mapB0, wx, wy, full_bar(s));
              }
            }
          } else {
            // 32-row boxes; gate (or down) rows first, then the up rows
            for (int j = 0; j < rp; j += 32) {
              wcoord(kb, b_row + j, p.k_blocks, p.blocked, wx, wy);
              tma_load_2d(sb + j * BK * 2, &mapB0s, wx, wy, full_bar(s));
            }
            if (MODE == kSwiGLU)
              for (int j = 0; j < rp; j += 32) {
                wcoord(kb, b_row + j, p.k_blocks, p.blocked, wx, wy);
                tma_load_2d(sb + (rp + j) * BK * 2, &mapB1s, wx, wy, full_bar(s));
              }
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        const int first = it > kStages ? it - kStages : 0;
        for (int i = first; i < it; ++i)
          drain_phase(full_bar(i % kStages), (uint32_t)(i / kStages) & 1u, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int it = 0, tc = 0;
      bool ok = true, issued = false, pre = false;
      for (int w = blockIdx.x; w < work.items && ok; w += gridDim.x, ++tc) {
        int tile, piece, pieces, part;
        work.get(w, tile, piece, pieces, part);
        const uint32_t nmma = (uint32_t)((MODE == kSwiGLU ? 2 : 1) * (ROWS / pieces));
        const uint32_t idesc = (C::IDESC & ~(0x3Fu << 17)) | ((nmma >> 3) << 17);
        const int a = tc & 1;
        const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
        if (!wait_phase(tempty_bar(a), aph ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
        fence_after();
        const uint32_t d = tmem_base + (uint32_t)(a * BN);
        const int kb0 = part * p.k_blocks / work.ksplit;
        const int kb_end = (part + 1) * p.k_blocks / work.ksplit;
        for (int kb = kb0; kb < kb_end; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!pre && !wait_phase(full_bar(s), ph, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          fence_after();
          pre = mbar_test_wait(full_bar((it + 1) % kStages), (uint32_t)((it + 1) / kStages) & 1u);
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16(d, sdesc(sa + kk * 32), sdesc(sb + kk * 32), idesc,
                     (kb != kb0 || kk) ? 1u : 0u);
          }
          mma_commit(empty_bar(s));
          issued = true;
        }
        if (ok) mma_commit(tfull_bar(a));
      }
      // every MMA issued so far completes before tensor memory is released
      if (issued) {
        mma_commit(final_bar);
        drain_phase(final_bar, 0, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: warps 2..5, warp w reads TMEM lanes 32*(w%4) ..
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int tc = 0;
    for (int w = blockIdx.x; w < work.items; w += gridDim.x, ++tc) {
      int tile, piece, pieces, part, e, m, n;
      work.get(w, tile, piece, pieces, part);
      tile_coords(tile, row_tiles, p.E, p.n_tiles, e, m, n);
      const int rp = ROWS / pieces;  // output columns of this item
      const int a = tc & 1;
      const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
      int ok = 0;
      if (lane == 0) ok = wait_phase(tfull_bar(a), aph, abort_flag, p.status, p.timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * BN);
      const int64_t row = (int64_t)m * BM + row_in_tile;
      const int64_t col0 = (int64_t)n * ROWS + (int64_t)piece * rp;
      if (MODE == kSwiGLU) {
        uint16_t* h = reinterpret_cast<uint16_t*>(p.out) + row * p.out_ld + col0;
#pragma unroll 1
        for (int c = 0; c < rp; c += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(taddr + c, g);
          tmem_ld16(taddr + rp + c, u);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            const float h0 = g0 / (1.f + __expf(-g0)) * u0;
            const float h1 = g1 / (1.f + __expf(-g1)) * u1;
            pk[i] = pack_bf16x2_rn(h0, h1);
          }
          uint4* dst = reinterpret_cast<uint4*>(h + c);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      } else if (work.ksplit == 1) {
        float* y = reinterpret_cast<float*>(p.out) + row * p.out_ld + col0;
#pragma unroll 1
        for (int c = 0; c < rp; c += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + c, v);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(y + c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                 __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      } else {
        // split-K: this part's sums of the tile's real rows go to the partial buffer
        // (compact routed rows; pad rows are neither stored nor summed)
        const int local = (m - row_tiles[e]) * BM + row_in_tile;  // row within the expert
        const bool real = local < p.counts[e];
        const int64_t crow = (int64_t)routed_start[e] + local;
        const int64_t part_ld = p.routed * p.out_ld;
        float* mine = p.partial + (int64_t)part * part_ld + crow * p.out_ld + col0;
#pragma unroll 1
        for (int c = 0; c < rp; c += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + c, v);
          tmem_wait_ld();
          if (real) {
            float4* dst = reinterpret_cast<float4*>(mine + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
        // the accumulator is free once read
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(a));
        // arrival of this warp's 32 rows; the warp of the last part to arrive sums the
        // parts in part order (a fixed order, whichever part finishes last) into y
        __threadfence();
        __syncwarp();
        int last = 0;
        int32_t* sem = p.split_sem + tile * 4 + q;
        if (lane == 0) last = atomicAdd(sem, 1) == work.ksplit - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          // the warp sums its real rows one at a time, lanes across the columns
          // (coalesced), every part's load in flight before the adds
          const int local0 = local - row_in_tile + q * 32;  // the warp's first row in the expert
          const int nreal = min(32, max(0, p.counts[e] - local0));
          const float* src0 = p.partial + ((int64_t)routed_start[e] + local0) * p.out_ld + col0;
          float* y0 = reinterpret_cast<float*>(p.out) + ((int64_t)m * BM + q * 32) * p.out_ld + col0;
#pragma unroll 1
          for (int r = 0; r < nreal; ++r) {
#pragma unroll 1
            for (int c = lane * 4; c < rp; c += 128) {
              float4 v[kMaxSplitK];
#pragma unroll
              for (int s = 0; s < kMaxSplitK; ++s)
                if (s < work.ksplit)
                  v[s] = __ldcg(reinterpret_cast<const float4*>(src0 + r * p.out_ld + s * part_ld + c));
              float4 acc = v[0];
#pragma unroll
              for (int s = 1; s < kMaxSplitK; ++s)
                if (s < work.ksplit) {
                  acc.x += v[s].x;
                  acc.y += v[s].y;
                  acc.z += v[s].z;
                  acc.w += v[s].w;
                }
              *reinterpret_cast<float4*>(y0 + r * p.out_ld + c) = acc;
            }
          }
          if (lane == 0) *sem = 0;  // ready for the next launch
        }
        continue;
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(a));
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- CTA-pair variant
//
// For large batches two CTAs of a cluster compute one 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256): each CTA stages its own 128 rows of A and its
// 128 rows of B (gate/up: CTA 0 holds the w1 rows, CTA 1 the w3 rows; down: the two
// 128-row halves of the w2 tile), so a CTA moves 32 KiB per 64-wide k-block instead
// of 48 KiB. A stage holds kPairKB = 2 k-blocks (K = 128: 64 KiB per CTA, three
// stages), so every barrier handoff between the copies and the MMAs carries eight
// MMAs instead of four. Measured on B200: with K = 64 stages a k-block took about 700
// SM clocks against the tensor pipe's 512, whatever the stage count (4 to 7), the
// number of busy SMs (37 to 148) or the clock; with K = 128 stages it takes about 570.
// The pair's two row tiles are consecutive 128-row tiles of one expert; when an
// expert has an odd number, the second CTA's rows of its last pair belong to the next
// group and are computed but not stored.
//
// Synchronisation: CTA 0 (the leader) owns the full barriers (both CTAs' TMA loads
// complete transactions on them; only the leader arrives, expecting both CTAs'
// bytes) and the accumulator-empty barriers (four epilogue warps of each CTA
// arrive). The leader's MMA thread commits to the empty and accumulator-full
// barriers of both CTAs at once (multicast commit). No TMA load uses multicast.

#ifndef MOE_PAIR_STAGES
#define MOE_PAIR_STAGES 3
#endif
#ifndef MOE_PAIR_KB
#define MOE_PAIR_KB 2
#endif
constexpr int kPairStages = MOE_PAIR_STAGES;
constexpr int kPairKB = MOE_PAIR_KB;  // 64-wide k-blocks per stage

struct PairTile {
  static constexpr int A_BOX = BM * BK * 2;   // one 128-row x 64 box of A
  static constexpr int B_BOX = 128 * BK * 2;  // one 128-row x 64 box of B
  static constexpr int A_BYTES = A_BOX * kPairKB;
  static constexpr int B_BYTES = B_BOX * kPairKB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SMEM_BYTES = 1024 + kPairStages * STAGE_BYTES + 256 + 4 * 144;
  // D f32, A/B bf16 K-major, N = 256, M = 256
  static constexpr uint32_t IDESC =
      (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((256u >> 4) << 24);
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on a barrier
// that may live in the peer CTA of the pair
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive on the barrier at this shared offset in both CTAs of the pair
__device__ __forceinline__ void mma_commit_pair_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// Pair tile L -> (expert e, first row tile m0 of the pair, column tile n).
// pair_rows[e] = sum over e' < e of ceil(row tiles of e' / 2).
__device__ __forceinline__ void pair_coords(int L, const int* row_tiles, const int* pair_rows,
                                            int E, int n_tiles, int& e, int& m0, int& n) {
  const int prow = L / n_tiles;
  e = 0;
  while (e + 1 < E && pair_rows[e + 1] <= prow) ++e;
  const int cnt = pair_rows[e + 1] - pair_rows[e];
  const int local = L - pair_rows[e] * n_tiles;
  n = local / cnt;
  m0 = row_tiles[e] + 2 * (local % cnt);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm_pair(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapB0,
                        const __grid_constant__ CUtensorMap mapB1, const KParams p) {
  using C = PairTile;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairStages * C::STAGE_BYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kPairStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* row_tiles = reinterpret_cast<int*>(tmem_holder + 2);
  int* pair_rows = row_tiles + 72;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  // a role that gives up a wait also raises the other CTA's abort flag, so the pair
  // unwinds together (both CTAs stay resident until the final cluster barrier)
  const uint32_t peer_abort = mapa_shared(smem_u32((const void*)abort_flag), rank ^ 1u);
  auto abort_peer = [&]() {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
  };
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kPairStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kPairStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kPairStages + 2 + a); };
  const uint32_t final_bar = bar0 + 8u * (2 * kPairStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    prefetch_map(&mapA);
    prefetch_map(&mapB0);
    prefetch_map(&mapB1);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  // both CTAs' barriers exist before any cross-CTA arrival
  fence_before();
  __syncthreads();
  cluster_sync_all();
  fence_after();
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) row_tiles[i] = p.offsets[i] / BM;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < p.E; ++e) {
      pair_rows[e] = acc;
      acc += (row_tiles[e + 1] - row_tiles[e] + 1) / 2;
    }
    pair_rows[p.E] = acc;
  }
  __syncthreads();
  const uint32_t tmem_base = *tmem_holder;
  const int total = pair_rows[p.E] * p.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      int it = 0;
      bool ok = true;
      for (int L = pair; L < total && ok; L += npairs) {
        int e, m0, n;
        pair_coords(L, row_tiles, pair_rows, p.E, p.n_tiles, e, m0, n);
        const int a_row = (m0 + (int)rank) * BM;
        int b_row;
        const CUtensorMap* mb;
        if (MODE == kSwiGLU) {
          b_row = e * p.b_rows + n * 128;
          mb = rank == 0 ? &mapB0 : &mapB1;
        } else {
          b_row = e * p.b_rows + n * 256 + (int)rank * 128;
          mb = &mapB0;
        }
        for (int kb = 0; kb < p.k_blocks; kb += kPairKB, ++it) {
          const int s = it % kPairStages;
          const uint32_t ph = (uint32_t)(it / kPairStages) & 1u;
          if (!wait_phase(empty_bar(s), ph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            abort_peer();
            ok = false;
            break;
          }
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          if (rank == 0) mbar_expect_tx(full_bar(s), 2 * C::STAGE_BYTES);
          const uint32_t fb = mapa_shared(full_bar(s), 0);
#pragma unroll
          for (int j = 0; j < kPairKB; ++j) {
            tma_load_2d_pair(sa + j * C::A_BOX, &mapA, (kb + j) * BK, a_row, fb);
            int wx, wy;
            wcoord(kb + j, b_row, p.k_blocks, p.blocked, wx, wy);
            tma_load_2d_pair(sa + C::A_BYTES + j * C::B_BOX, mb, wx, wy, fb);
          }
        }
      }
      if (!ok && rank == 0) {
        const int first = it > kPairStages ? it - kPairStages : 0;
        for (int i = first; i < it; ++i)
          drain_phase(full_bar(i % kPairStages), (uint32_t)(i / kPairStages) & 1u, p.status,
                      p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA only)
      int it = 0, tc = 0;
      bool ok = true, issued = false, pre = false;
      for (int L = pair; L < total && ok; L += npairs, ++tc) {
        const int a = tc & 1;
        const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
        if (!wait_phase(tempty_bar(a), aph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
          abort_peer();
          break;
        }
        fence_after();
        const uint32_t d = tmem_base + (uint32_t)(a * 256);
        for (int kb = 0; kb < p.k_blocks; kb += kPairKB, ++it) {
          const int s = it % kPairStages;
          const uint32_t ph = (uint32_t)(it / kPairStages) & 1u;
          if (!pre && !wait_phase(full_bar(s), ph, abort_flag, p.status, p.timeout_ns)) {
            abort_peer();
            ok = false;
            break;
          }
          fence_after();
          pre = mbar_test_wait(full_bar((it + 1) % kPairStages),
                               (uint32_t)((it + 1) / kPairStages) & 1u);
          const uint32_t sa = smem_u32(smem + s * C::STAGE_BYTES);
          const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int j = 0; j < kPairKB; ++j)
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_bf16_pair(d, sdesc(sa + j * C::A_BOX + kk * 32),
                            sdesc(sb + j * C::B_BOX + kk * 32), C::IDESC, (kb | j | kk) ? 1u : 0u);
          mma_commit_pair_both(empty_bar(s));
          issued = true;
        }
        if (ok) mma_commit_pair_both(tfull_bar(a));
      }
      if (issued) {
        mma_commit_pair_local(final_bar);
        drain_phase(final_bar, 0, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows of the 256-row tile
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int tc = 0;
    for (int L = pair; L < total; L += npairs, ++tc) {
      int e, m0, n;
      pair_coords(L, row_tiles, pair_rows, p.E, p.n_tiles, e, m0, n);
      const int m = m0 + (int)rank;
      const bool store = m < row_tiles[e + 1];
      const int a = tc & 1;
      const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
      int ok = 0;
      if (lane == 0) {
        ok = wait_phase(tfull_bar(a), aph, abort_flag, p.status, p.timeout_ns) ? 1 : 0;
        if (!ok) abort_peer();
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * 256);
      const int64_t row = (int64_t)m * BM + row_in_tile;
      if (store) {
        if (MODE == kSwiGLU) {
          uint16_t* h = reinterpret_cast<uint16_t*>(p.out) + row * p.out_ld + (int64_t)n * 128;
#pragma unroll 1
          for (int c = 0; c < 128; c += 16) {
            uint32_t g[16], u[16];
            tmem_ld16(taddr + c, g);
            tmem_ld16(taddr + 128 + c, u);
            tmem_wait_ld();
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              const float h0 = g0 / (1.f + __expf(-g0)) * u0;
              const float h1 = g1 / (1.f + __expf(-g1)) * u1;
              pk[i] = pack_bf16x2_rn(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(h + c);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        } else {
          float* y = reinterpret_cast<float*>(p.out) + row * p.out_ld + (int64_t)n * 256;
#pragma unroll 1
          for (int c = 0; c < 256; c += 16) {
            uint32_t v[16];
            tmem_ld16(taddr + c, v);
            tmem_wait_ld();
            float4* dst = reinterpret_cast<float4*>(y + c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(tempty_bar(a));
        else mbar_arrive_cluster(mapa_shared(tempty_bar(a), 0));
      }
    }
  }

  // no CTA frees tensor memory while the pair may still use it
  fence_before();
  __syncthreads();
  cluster_sync_all();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- small batches
//
// k_decode_swap: both expert GEMMs of a batch of at most 256 tokens in one persistent
// grid, with the operands swapped: the weights are the tcgen05 M operand (128 weight
// rows per tile, loaded by TMA straight into the 128-byte swizzled K-major layout the
// MMA reads) and a sub-tile of at most NMAX of an expert's routed rows the N operand (N
// = the sub-tile's row count rounded up to 16; a token reaches an expert at most once,
// so up to NMAX tokens every expert has one sub-tile). An expert with more rows has
// several sub-tiles over the same weight tiles, consecutive tiles, so the weights cross
// HBM once. A stage holds twice KB weight boxes of 128 x 64 (gate/up: the w1 and w3
// boxes of KB k-blocks; down: twice KB k-blocks of one w2 box; KB = 2, or 1 for NMAX =
// 128 so that three stages of rows still fit) and its k-blocks of rows.
// Against the tile kernels this moves 2 KiB of routed rows per 64 KiB of weights
// instead of a 16 KiB activation tile per 32 KiB, and runs both GEMMs as one grid.
//
//   warp 0      weight boxes (TMA);
//   warp 6      routed rows (TMA, 16-row boxes); a down tile first waits until every
//               gate/up tile of its sub-tile has released its rows of h;
//   warps 1, 7  issue the MMAs (M = 128, N = rows): gate/up the first issues gate, the
//               second up; down each issues KB of the stage's 2 KB k-blocks into its
//               own partial sum;
//   warps 2-5   read the accumulators (lane = weight row, column = routed row): h =
//               bf16(silu(gate) * up) at [row, i], y = the two partial sums' sum at
//               [row, j].
// Each role tests its next stage's barriers with test_wait before starting the current
// one (measured on B200: a wait whose result steers the MMA thread costs about 340 SM
// clocks between MMAs). Every gate/up tile precedes every down tile in the order each
// CTA walks its tiles and the grid is at most one CTA per SM, so a down tile only waits
// for tiles that are running or done.
template <int NMAX>
struct DecBf16 {
  static constexpr int KB = NMAX <= 64 ? 2 : 1;                // k-blocks per matrix per stage
  static constexpr int BOXES = 2 * KB;                         // weight boxes per stage
  static constexpr int WBOX = 128 * BK * 2;                    // one 128 x 64 weight box
  static constexpr int ACT_UNIT = NMAX * 128;                  // NMAX rows of one k-block
  static constexpr int STAGE = BOXES * WBOX + BOXES * ACT_UNIT;
  static constexpr int STAGES = (220 * 1024) / STAGE;          // 3 (NMAX 16, 128), 2 (32, 64)
  static constexpr int ACC_COLS = 2 * NMAX;                    // gate, up (or two partials)
  static constexpr int TMEM_COLS = 2 * ACC_COLS <= 32    ? 32
                                   : 2 * ACC_COLS <= 64  ? 64
                                   : 2 * ACC_COLS <= 128 ? 128
                                   : 2 * ACC_COLS <= 256 ? 256
                                                         : 512;
  static constexpr int NUM_BARS = 3 * STAGES + 6;
  static constexpr int SMEM = 1024 + STAGES * STAGE + NUM_BARS * 8 + 16 + 3 * 72 * 4;
  // D f32, A and B bf16, both K-major, M = 128; N is set per tile
  static constexpr uint32_t IDESC_M128 =
      (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 4) << 24);
  static_assert(NMAX == 16 || NMAX == 32 || NMAX == 64 || NMAX == 128, "rows per tile");
  static_assert(STAGES >= 2 && STAGE % 1024 == 0, "stage plan");
  static_assert(TMEM_COLS >= 2 * ACC_COLS && TMEM_COLS <= 512, "two accumulator buffers");
  static_assert(SMEM <= 232448, "shared memory plan exceeds 227 KiB");
};

struct DecBf16Params {
  const int32_t* offsets;  // [E+1], multiples of 128
  const int32_t* counts;   // [E] routed rows per expert, or null (then NMAX rows a tile)
  uint16_t* h;             // [rows, I] bf16
  float* y;                // [rows, H] fp32
  int32_t* status;
  int32_t* row_ready;      // [rows / 64] per-sub-tile counters, zero at launch
  int E, H, I, blocked;
  int max_rows;            // most rows an expert can have: the tokens
  unsigned long long timeout_ns;
};

// Tile L -> (expert e, sub-tile m, column tile n) of a grid whose tiles are n_tiles per
// sub-tile (first_sub[e]: the expert's first sub-tile); an expert's sub-tiles of one
// column tile are consecutive, so its weight tile is read from HBM once and from L2 for
// the other sub-tiles
__device__ __forceinline__ void swap_coords(int L, const int* first_sub, int E, int n_tiles,
                                            int& e, int& m, int& n) {
  const int mrow = L / n_tiles;
  e = 0;
  while (e + 1 < E && first_sub[e + 1] <= mrow) ++e;
  const int cnt = first_sub[e + 1] - first_sub[e];
  const int local = L - first_sub[e] * n_tiles;
  n = local / cnt;
  m = first_sub[e] + local % cnt;
}

// Wait until *ready >= target (acquire: the h rows stored before the release are then
// visible), bounded like the barrier waits.
__device__ __noinline__ bool wait_count(const int32_t* ready, int target, volatile int* abort_flag,
                                        int32_t* status, unsigned long long timeout_ns) {
  const unsigned long long t0 = globaltimer();
  for (uint32_t n = 0;; ++n) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ready) : "memory");
    if (v >= target) return true;
    __nanosleep(64);
    if ((n & 63u) == 63u) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > timeout_ns) {
        *abort_flag = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}

template <int NMAX>
__global__ void __launch_bounds__(256, 1)
    k_decode_swap(const __grid_constant__ CUtensorMap mw1, const __grid_constant__ CUtensorMap mw3,
                  const __grid_constant__ CUtensorMap mw2, const __grid_constant__ CUtensorMap mx,
                  const __grid_constant__ CUtensorMap mh, const __grid_constant__ DecBf16Params p) {
  using D = DecBf16<NMAX>;
  constexpr int kS = D::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kS * D::STAGE);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + D::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* sub0 = reinterpret_cast<int*>(tmem_holder + 4);  // [E + 1]: first sub-tile of each expert
  int* nrows = sub0 + 72;                                // [E]: routed rows of each expert
  int* row_off = nrows + 72;                             // [E]: first row of each expert

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int KB = D::KB;
  // barriers: w_full (weights), a_full (rows), empty (both; the two issuers' commits) [kS];
  // t_full, t_empty [2]; final [2] (one per issuer)
  const uint32_t bar0 = smem_u32(bars);
  auto w_full = [&](int s) { return bar0 + 8u * s; };
  auto a_full = [&](int s) { return bar0 + 8u * (kS + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * kS + s); };
  auto t_full = [&](int b) { return bar0 + 8u * (3 * kS + b); };
  auto t_empty = [&](int b) { return bar0 + 8u * (3 * kS + 2 + b); };
  const uint32_t final_bar = bar0 + 8u * (3 * kS + 4);
  auto stage = [&](int s) { return smem_u32(smem + s * D::STAGE); };
  auto ph = [](int it, int n) { return (uint32_t)(it / n) & 1u; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(w_full(s), 1);
      mbar_init(a_full(s), 1);
      mbar_init(empty(s), 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(t_full(b), 2);
      mbar_init(t_empty(b), 4);
    }
    mbar_init(final_bar, 1);
    mbar_init(final_bar + 8u, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    prefetch_map(&mw1);
    prefetch_map(&mw3);
    prefetch_map(&mw2);
    prefetch_map(&mx);
    prefetch_map(&mh);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"((uint32_t)D::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < p.E; i += blockDim.x) {
    const int padded = p.offsets[i + 1] - p.offsets[i];
    nrows[i] = p.counts ? p.counts[i] : (padded < p.max_rows ? padded : p.max_rows);
    row_off[i] = p.offsets[i];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int i = 0; i < p.E; ++i) {
      sub0[i] = acc;
      acc += (nrows[i] + NMAX - 1) / NMAX;
    }
    sub0[p.E] = acc;
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // sub-tile m of expert e: its first row, and N = its rows rounded up to 16 (at most NMAX)
  auto sub_row0 = [&](int e, int m) { return row_off[e] + (m - sub0[e]) * NMAX; };
  auto tile_n = [&](int e, int m) {
    const int n = (nrows[e] - (m - sub0[e]) * NMAX + 15) & ~15;
    return n < 16 ? 16 : (n > NMAX ? NMAX : n);
  };

  const int n1 = p.I / 128, n2 = p.H / 128;          // column tiles per sub-tile
  const int kb1 = p.H / BK, kb2 = p.I / BK;          // k-blocks of w1/w3 and of w2
  const int st1 = kb1 / KB, st2 = kb2 / (2 * KB);    // stages per tile
  const int total0 = sub0[p.E] * n1;
  const int total = total0 + sub0[p.E] * n2;
  auto coords = [&](int L, bool& dn, int& e, int& m, int& n) {
    dn = L >= total0;
    swap_coords(dn ? L - total0 : L, sub0, p.E, dn ? n2 : n1, e, m, n);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- weight boxes
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        bool dn;
        int e, m, n;
        coords(L, dn, e, m, n);
        const int nst = dn ? st2 : st1;
        for (int s = 0; s < nst; ++s, ++it) {
          const int q = it % kS;
          if (!wait_phase(empty(q), ph(it, kS) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(w_full(q), D::BOXES * D::WBOX);
          const uint32_t dst = stage(q);
          int wx, wy;
          if (!dn) {
            // boxes 0 .. KB-1: w1 rows 128 n .. of expert e, k-blocks KB s ..; boxes KB ..:
            // the same of w3
#pragma unroll
            for (int j = 0; j < KB; ++j) {
              wcoord(KB * s + j, e * p.I + n * 128, kb1, p.blocked, wx, wy);
              tma_load_2d(dst + j * D::WBOX, &mw1, wx, wy, w_full(q));
              tma_load_2d(dst + (KB + j) * D::WBOX, &mw3, wx, wy, w_full(q));
            }
          } else {
            // boxes 0 .. 2KB-1: k-blocks 2KB s .. of w2 rows 128 n .. of expert e
#pragma unroll
            for (int j = 0; j < 2 * KB; ++j) {
              wcoord(2 * KB * s + j, e * p.H + n * 128, kb2, p.blocked, wx, wy);
              tma_load_2d(dst + j * D::WBOX, &mw2, wx, wy, w_full(q));
            }
          }
        }
      }
      if (!ok) {
        const int first = it > kS ? it - kS : 0;
        for (int i = first; i < it; ++i) drain_phase(w_full(i % kS), ph(i, kS), p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    if (lane == 0) {
      // ---------------- routed rows of each stage's k-blocks: KB (gate/up) or 2 KB
      // (down), N rows in 16-row boxes
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        bool dn;
        int e, m, n;
        coords(L, dn, e, m, n);
        if (dn) {
          // every gate/up tile of sub-tile m has stored its rows of h; the proxy fence
          // orders those stores before the tensor copies (async proxy) that read them
          if (!wait_count(p.row_ready + m, 4 * n1, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        const int nrow = tile_n(e, m), row0 = sub_row0(e, m);
        const CUtensorMap* map = dn ? &mh : &mx;
        const int nst = dn ? st2 : st1;
        const int nblk = dn ? 2 * KB : KB;
        for (int s = 0; s < nst; ++s, ++it) {
          const int q = it % kS;
          if (!wait_phase(empty(q), ph(it, kS) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(a_full(q), (uint32_t)(nblk * nrow * 128));
          const uint32_t dst = stage(q) + D::BOXES * D::WBOX;
          for (int b = 0; b < nblk; ++b)
            for (int j = 0; j < nrow; j += 16)
              tma_load_2d(dst + b * D::ACT_UNIT + j * 128, map, (nblk * s + b) * BK, row0 + j,
                          a_full(q));
        }
      }
      if (!ok) {
        const int first = it > kS ? it - kS : 0;
        for (int i = first; i < it; ++i) drain_phase(a_full(i % kS), ph(i, kS), p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 7) {
    if (lane == 0) {
      // ---------------- MMA issuers (mi = 0, 1): gate/up: mi 0 gate (w1 boxes), mi 1 up
      // (w3 boxes), both over the rows of the stage's KB k-blocks; down: mi's KB boxes
      // (k-blocks) into partial sum mi. The next stage's barriers are tested before this
      // stage's MMAs issue.
      const int mi = warp == 1 ? 0 : 1;
      int it = 0, tc = 0;
      bool ok = true, issued = false, pre_w = false, pre_a = false;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tc) {
        bool dn;
        int e, m, n;
        coords(L, dn, e, m, n);
        const uint32_t idesc = D::IDESC_M128 | ((uint32_t)(tile_n(e, m) >> 3) << 17);
        const int b = tc & 1;
        if (!wait_phase(t_empty(b), ph(tc, 2) ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
        fence_after();
        const uint32_t d = tmem_base + (uint32_t)(b * D::ACC_COLS + mi * NMAX);
        const int nst = dn ? st2 : st1;
        for (int s = 0; s < nst; ++s, ++it) {
          const int q = it % kS;
          if ((!pre_w && !wait_phase(w_full(q), ph(it, kS), abort_flag, p.status, p.timeout_ns)) ||
              (!pre_a && !wait_phase(a_full(q), ph(it, kS), abort_flag, p.status, p.timeout_ns))) {
            ok = false;
            break;
          }
          fence_after();
          pre_w = mbar_test_wait(w_full((it + 1) % kS), ph(it + 1, kS));
          pre_a = mbar_test_wait(a_full((it + 1) % kS), ph(it + 1, kS));
          const uint32_t sw = stage(q), sa = sw + D::BOXES * D::WBOX;
#pragma unroll
          for (int j = 0; j < KB; ++j) {
            const int box = KB * mi + j, unit = dn ? KB * mi + j : j;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_bf16(d, sdesc(sw + box * D::WBOX + kk * 32), sdesc(sa + unit * D::ACT_UNIT + kk * 32),
                       idesc, (s | j | kk) ? 1u : 0u);
          }
          mma_commit(empty(q));
          issued = true;
        }
        if (ok) mma_commit(t_full(b));
      }
      if (issued) {
        mma_commit(final_bar + 8u * mi);
        drain_phase(final_bar + 8u * mi, 0, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- epilogue: TMEM lanes 32 (warp % 4) .. = weight rows
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;
    int tc = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tc) {
      bool dn;
      int e, m, n;
      coords(L, dn, e, m, n);
      const int nrow = tile_n(e, m);
      const int b = tc & 1;
      int ok = 0;
      if (lane == 0) ok = wait_phase(t_full(b), ph(tc, 2), abort_flag, p.status, p.timeout_ns) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      fence_after();
      const uint32_t tacc =
          tmem_base + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(b * D::ACC_COLS);
      const int64_t row0 = sub_row0(e, m);
      if (!dn) {
        uint16_t* hcol = p.h + row0 * p.I + n * 128 + r;  // intermediate column n 128 + r
        for (int c0 = 0; c0 < nrow; c0 += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(tacc + c0, g);
          tmem_ld16(tacc + NMAX + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float gv = __uint_as_float(g[t]), uv = __uint_as_float(u[t]);
            hcol[(int64_t)(c0 + t) * p.I] =
                (uint16_t)(pack_bf16x2_rn(gv / (1.f + __expf(-gv)) * uv, 0.f) & 0xFFFFu);
          }
        }
        // release this warp's rows of h to the down tiles of sub-tile m
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.row_ready + m, 1);
      } else {
        float* ycol = p.y + row0 * p.H + n * 128 + r;  // hidden column n 128 + r
        for (int c0 = 0; c0 < nrow; c0 += 16) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tacc + c0, v0);
          tmem_ld16(tacc + NMAX + c0, v1);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t)
            ycol[(int64_t)(c0 + t) * p.H] = __uint_as_float(v0[t]) + __uint_as_float(v1[t]);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(t_empty(b));
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)D::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------------------- bounded-wait check
// One thread waits, with the same bounded wait the GEMMs use, on a barrier phase that
// nothing completes; after timeout_ns it records kStatusTimeout and returns.
__global__ void k_wait_selftest(int32_t* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0)
    wait_phase(smem_u32(&bar), 0, reinterpret_cast<volatile int*>(&abort_flag), status, timeout_ns);
}

// ---------------------------------------------------------------- weight packing
// w [rows, cols] row-major -> [rows/128][cols/64][128][64]; one thread per 16 bytes.
__global__ void __launch_bounds__(256) k_pack_blocked(const uint4* __restrict__ w,
                                                      uint4* __restrict__ wp, int64_t rows,
                                                      int64_t cols) {
  const int64_t kb_n = cols / BK, n = rows * cols / 8;
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < n;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = o & 7;              // 16-byte chunk within a 64-wide row
    const int64_t rr = (o >> 3) & 127;    // row within the block
    const int64_t blk = o >> 10;          // (row block, k block)
    const int64_t rb = blk / kb_n, kb = blk - rb * kb_n;
    wp[o] = w[((rb * 128 + rr) * cols + kb * BK) / 8 + c];
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 2-D bf16 tensor [rows, inner] row-major; box = 64 x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int BN>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       const CUtensorMap& b0s, const CUtensorMap& b1s, const KParams& p,
                       int64_t max_tiles, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int smem = Tile<BN>::SMEM_BYTES;
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<MODE, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int64_t grid = num_sms();
  if (grid > max_tiles) grid = max_tiles;
  return launch_pdl(k_grouped_gemm<MODE, BN>, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, st,
                    a, b0, b1, b0s, b1s, p);
}

// Clusters of two CTAs that can be resident at once for the pair kernel (cached per
// device); the pair grid never exceeds it, so every pair of a launch runs together.
template <int MODE>
int pair_capacity() {
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cache[dev]) return cache[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PairTile::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_grouped_gemm_pair<MODE>, &cfg) != cudaSuccess || n <= 0)
    n = num_sms() / 2;
  if (n > num_sms() / 2) n = num_sms() / 2;
  if (dev < 64) cache[dev] = n;
  return n;
}

template <int MODE>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const KParams& p, int64_t max_pair_tiles, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm_pair<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         PairTile::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (p.k_blocks % kPairKB) return cudaErrorInvalidValue;  // K is a multiple of 128
  int64_t pairs = pair_capacity<MODE>();
  if (pairs > max_pair_tiles) pairs = max_pair_tiles;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PairTile::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_grouped_gemm_pair<MODE>, a, b0, b1, p);
}

// Measured on B200: the pair kernel speeds up both GEMMs once an average expert has at
// least eight row tiles (1024 rows); with fewer, the half-empty pair of every expert
// with an odd tile count and the coarser waves cost more than it saves.
#ifndef MOE_PAIR_GEMM
#define MOE_PAIR_GEMM 1
#endif
bool use_pair(const Shape& s) { return MOE_PAIR_GEMM && s.T * s.k >= (int64_t)1024 * s.E; }

// Both expert GEMMs on the swap-operand kernel (row tiles of at most NMAX routed rows)
template <int NMAX>
cudaError_t launch_decode_swap(const Shape& s, const GemmArgs& g, cudaStream_t st,
                               const char** why) {
  using D = DecBf16<NMAX>;
  CUtensorMap mx, mh, mw1, mw3, mw2;
  const uint64_t EI = (uint64_t)s.E * s.I, EH = (uint64_t)s.E * s.H;
  const uint64_t wi1 = s.blocked ? BK : s.H, wr1 = s.blocked ? EI * s.H / BK : EI;
  const uint64_t wi2 = s.blocked ? BK : s.I, wr2 = s.blocked ? EH * s.I / BK : EH;
  if (!make_map(&mx, g.a, s.H, g.rmax, 16) || !make_map(&mh, g.h, s.I, g.rmax, 16) ||
      !make_map(&mw1, g.w1, wi1, wr1, 128) || !make_map(&mw3, g.w3, wi1, wr1, 128) ||
      !make_map(&mw2, g.w2, wi2, wr2, 128)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor)";
    return cudaErrorInvalidValue;
  }
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_decode_swap<NMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM);
    if (e != cudaSuccess) {
      *why = "expert GEMM shared-memory attribute";
      return e;
    }
    attr_set[dev] = true;
  }
  DecBf16Params p;
  p.offsets = g.offsets;
  p.counts = g.expert_rows ? g.expert_rows : g.counts;
  p.h = g.h;
  p.y = g.y;
  p.status = g.status;
  p.row_ready = g.row_ready;
  p.E = s.E;
  p.H = s.H;
  p.I = s.I;
  p.blocked = s.blocked;
  p.max_rows = (int)s.T;
  p.timeout_ns = g.timeout_ns;
  // the sub-tile counters start at zero (unless a kernel before this one zeroed them: a
  // memset between the two would keep this launch from overlapping that kernel's tail);
  // an expert of c rows has ceil(c / NMAX) sub-tiles, at most T k / NMAX + E in all,
  // within rmax / 64 (rmax >= T k + 128 E)
  cudaError_t e = g.row_ready_zeroed
                      ? cudaSuccess
                      : cudaMemsetAsync(g.row_ready, 0, (size_t)(g.rmax / 64) * sizeof(int32_t), st);
  if (e == cudaSuccess) {
    const int64_t tiles = ((int64_t)s.T * s.k / NMAX + s.E) * (s.I / 128 + s.H / 128);
    int64_t grid = num_sms() < tiles ? num_sms() : tiles;
    if (grid < 1) grid = 1;
    e = launch_pdl(k_decode_swap<NMAX>, dim3((unsigned)grid), dim3(256), (size_t)D::SMEM, st, mw1,
                   mw3, mw2, mx, mh, p);
  }
  if (e != cudaSuccess) *why = "expert GEMMs launch failed";
  return e;
}

#ifndef MOE_SWAP_DECODE
#define MOE_SWAP_DECODE 1
#endif

}  // namespace

cudaError_t launch_gate_up(const Shape& s, const GemmArgs& g, cudaStream_t st, const char** why) {
  CUtensorMap mx, mw1, mw3, mw1s, mw3s;
  const uint64_t EI = (uint64_t)s.E * s.I;
  const uint64_t wi = s.blocked ? BK : s.H, wr = s.blocked ? EI * s.H / BK : EI;
  if (!make_map(&mx, g.a, s.H, g.rmax, 128) || !make_map(&mw1, g.w1, wi, wr, 128) ||
      !make_map(&mw3, g.w3, wi, wr, 128) || !make_map(&mw1s, g.w1, wi, wr, 32) ||
      !make_map(&mw3s, g.w3, wi, wr, 32)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor)";
    return cudaErrorInvalidValue;
  }
  KParams p;
  p.offsets = g.offsets;
  p.status = g.status;
  p.out = g.h;
  p.out_ld = s.I;
  p.E = s.E;
  p.k_blocks = s.H / BK;
  p.n_tiles = s.I / 128;
  p.b_rows = s.I;
  p.blocked = s.blocked;
  p.timeout_ns = g.timeout_ns;
  p.counts = nullptr;
  p.partial = nullptr;
  p.split_sem = nullptr;
  p.routed = 0;
  p.zero_sem = g.counts ? g.split_sem : nullptr;
  cudaError_t e;
  if (use_pair(s))
    e = launch_pair<kSwiGLU>(mx, mw1, mw3, p, (g.rmax / BM / 2 + s.E) * p.n_tiles, st);
  else
    e = launch_one<kSwiGLU, 256>(mx, mw1, mw3, mw1s, mw3s, p, (g.rmax / BM) * p.n_tiles, st);
  if (e != cudaSuccess) *why = "gate/up GEMM launch failed";
  return e;
}

cudaError_t launch_down(const Shape& s, const GemmArgs& g, cudaStream_t st, const char** why) {
  CUtensorMap mh, mw2, mw2s;
  const uint64_t EH = (uint64_t)s.E * s.H;
  const uint64_t wi = s.blocked ? BK : s.I, wr = s.blocked ? EH * s.I / BK : EH;
  if (!make_map(&mh, g.h, s.I, g.rmax, 128) || !make_map(&mw2, g.w2, wi, wr, 128) ||
      !make_map(&mw2s, g.w2, wi, wr, 32)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor)";
    return cudaErrorInvalidValue;
  }
  KParams p;
  p.offsets = g.offsets;
  p.status = g.status;
  p.out = g.y;
  p.out_ld = s.H;
  p.E = s.E;
  p.k_blocks = s.I / BK;
  p.b_rows = s.H;
  p.blocked = s.blocked;
  p.timeout_ns = g.timeout_ns;
  // split-K needs the counts (real rows), the partial buffer and the counters, which
  // the gate/up GEMM before it has zeroed
  const bool split = g.counts && g.partial && g.split_sem && s.T * s.k <= kSplitMaxRows;
  p.counts = split ? g.counts : nullptr;
  p.partial = g.partial;
  p.split_sem = g.split_sem;
  p.routed = s.T * s.k;
  p.zero_sem = nullptr;
  cudaError_t e;
  if (s.H % 256 == 0 && use_pair(s)) {
    p.n_tiles = s.H / 256;
    e = launch_pair<kPlain>(mh, mw2, mw2, p, (g.rmax / BM / 2 + s.E) * p.n_tiles, st);
  } else if (s.H % 256 == 0) {
    p.n_tiles = s.H / 256;
    e = launch_one<kPlain, 256>(mh, mw2, mw2, mw2s, mw2s, p,
                                (g.rmax / BM) * p.n_tiles * (split ? kMaxSplitK : 1), st);
  } else {
    p.n_tiles = s.H / 128;
    e = launch_one<kPlain, 128>(mh, mw2, mw2, mw2s, mw2s, p,
                                (g.rmax / BM) * p.n_tiles * (split ? kMaxSplitK : 1), st);
  }
  if (e != cudaSuccess) *why = "down GEMM launch failed";
  return e;
}

cudaError_t launch_pack_blocked(const uint16_t* w, uint16_t* wp, int64_t rows, int64_t cols,
                                cudaStream_t st) {
  int64_t blocks = (rows * cols / 8 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  k_pack_blocked<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint4*>(w),
                                                   reinterpret_cast<uint4*>(wp), rows, cols);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int32_t* status, unsigned long long timeout_ns, cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>(status, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_grouped_swiglu(const Shape& s, const GemmArgs& g, cudaStream_t st,
                                  const char** why) {
  // the swap-operand kernel, hidden % 128 == 0: sub-tiles of 16, 32 or 64 rows (two
  // k-blocks per stage, intermediate % 256 == 0) up to 64 tokens, and up to 256 tokens
  // while the batch averages at most 56 routed rows per expert (measured: above that most
  // experts take two 64-row sub-tiles and the 128-row ones are faster); otherwise up to
  // 256 tokens 128-row sub-tiles (one k-block per stage, intermediate % 128 == 0)
  const bool rows64 = s.T <= 64 || (int64_t)s.T * s.k <= 56 * (int64_t)s.E;
  if (MOE_SWAP_DECODE && g.row_ready && s.T <= 256 && s.H % 128 == 0 && s.I % 256 == 0 && rows64)
    return s.T <= 16   ? launch_decode_swap<16>(s, g, st, why)
           : s.T <= 32 ? launch_decode_swap<32>(s, g, st, why)
                       : launch_decode_swap<64>(s, g, st, why);
  if (MOE_SWAP_DECODE && g.row_ready && s.T <= 256 && s.H % 128 == 0 && s.I % 128 == 0)
    return launch_decode_swap<128>(s, g, st, why);
  cudaError_t e = launch_gate_up(s, g, st, why);
  if (e != cudaSuccess) return e;
  return launch_down(s, g, st, why);
}

}  // namespace moe
