// Weight-only int8 experts (W8A16): the grouped GEMMs with int8 weight codes and one
// fp32 scale per output channel; and 4-bit experts (W4A16): 4-bit codes with one half
// scale per 64-column group of a row, applied while widening.
//
// Mixtral is loaded weight-only quantised to shrink it (Hugging Face "Mixtral" doc,
// "Shrinking down Mixtral using quantization"; ZeroModels "Mixtral", "Lower memory":
// int8 weights): half the weight memory of bf16, a quarter with 4-bit codes. (At
// decode the int8 kernel streams half the bytes and the 4-bit one a quarter, yet
// neither is faster than the bf16 kernel: the per-stage pipeline of copy, widening and
// MMA handoffs, not HBM, sets their pace.)
// Scheme (the pages do not fix one): per output row (channel) r, s[r] = max|w[r, :]| /
// 127 and q = rint(w / s), decided in float32; w ~ q * s. The experts compute in half
// precision, as a float16 load of the model does (Hugging Face "Mixtral" doc: the model
// in half precision, float16): the activations arrive as IEEE half, every code widens
// exactly to a half, the tensor cores accumulate in fp32, and the scale, constant along
// K, multiplies the accumulator in the epilogue: sum_k x[k] q[r,k] s[r] = s[r] sum_k
// x[k] q[r,k]. Half, not bf16, because an 8-bit code fits a half's 10-bit mantissa in
// one binade, so widening costs one byte permute and one packed subtraction per two
// codes; a bf16 has 7 mantissa bits and needs twice the integer work.
//
// Kernel k_grouped_gemm_w8: the bf16 GEMM's persistent tile loop with a widening
// stage, on 128-row tiles, or on 64-row tiles (tcgen05 M = 64) when the batch has at
// most 64 tokens. Warp roles:
//   warp 0      streams the code tiles (bulk copies: each 128-row x 64-code tile is one
//               contiguous 8 KiB run) into a code ring;
//   warp 6      loads the activation tiles (TMA, 128-byte swizzle) into their ring;
//   warps 7..   widen each code tile and store it, 128-byte swizzled, as the B operand;
//   warp 1      issues tcgen05.mma into a double-buffered TMEM accumulator;
//   warps 2-5   scale, activate and store (epilogue).
// The 4-bit kernel (BITS = 4) is the same pipeline: a code tile is 4 KiB plus its 128
// half scales, and the converters widen each code to a half and multiply it by its
// group's scale (the scale varies along K, so it cannot wait for the epilogue).
// Every wait is bounded (timeout -> status word, abort flag, drained copies).
#include <algorithm>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = 128, BK = 64;
#ifndef MOE_W8_A_STAGES
#define MOE_W8_A_STAGES 4
#endif
#ifndef MOE_W8_B_STAGES
#define MOE_W8_B_STAGES 3
#endif
#ifndef MOE_W8_CODE_STAGES
#define MOE_W8_CODE_STAGES 4
#endif
#ifndef MOE_W8_CODE_STAGES_M64
#define MOE_W8_CODE_STAGES_M64 6
#endif
#ifndef MOE_W8_A_STAGES_M64
#define MOE_W8_A_STAGES_M64 4
#endif
#ifndef MOE_W4_CODE_STAGES
#define MOE_W4_CODE_STAGES 7
#endif
#ifndef MOE_W4_CODE_STAGES_M64
#define MOE_W4_CODE_STAGES_M64 10
#endif
#ifndef MOE_W8_CONV_WARPS
#define MOE_W8_CONV_WARPS 8
#endif
constexpr int kConvWarps = MOE_W8_CONV_WARPS;
// warp 0: code copies, 1: MMA, 2-5: epilogue, 6: activation TMA, 7..: converters
constexpr int kConvWarp0 = 7;
constexpr int kThreadsW8 = 32 * (kConvWarp0 + kConvWarps);
constexpr int kSwiGLU = 0, kPlain = 1, kFused = 2;
#ifndef MOE_W8_HALF_TILES
#define MOE_W8_HALF_TILES 1
#endif
constexpr bool kUseHalfTiles = MOE_W8_HALF_TILES != 0;
#ifndef MOE_W8_DECODE_KERNEL
#define MOE_W8_DECODE_KERNEL 1
#endif
constexpr bool kUseDecodeKernel = MOE_W8_DECODE_KERNEL != 0;

// Shared-memory plan for an MT x BN tile: [A ring][B ring][code ring][barriers, TMEM
// address, row tiles]. Three rings: activation tiles (TMA -> MMA), code tiles (bulk
// copy -> converters) and widened weight tiles (converters -> MMA). MT = 128 rows, or
// 64 when every expert has at most 64 routed rows (the tile's first 64 rows hold all
// of them): the MMAs then cover only those rows, and the 8 KiB saved per activation
// stage buys deeper code prefetch.
// With BITS = 4 a code stage holds BN/128 boxes of 4 KiB codes, then BN half scales
// (stage row r's scale at element r), and more stages fit.
template <int BN, int MT, int BITS>
struct TileW8 {
  static constexpr int A_ST = MT == 64 ? MOE_W8_A_STAGES_M64 : MOE_W8_A_STAGES;
  static constexpr int B_ST = MOE_W8_B_STAGES;
  static constexpr int Q_ST = BITS == 8
                                  ? (MT == 64 ? MOE_W8_CODE_STAGES_M64 : MOE_W8_CODE_STAGES)
                                  : (MT == 64 ? MOE_W4_CODE_STAGES_M64 : MOE_W4_CODE_STAGES);
  static constexpr int A_BYTES = MT * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int BOX_CODE = 128 * BK * BITS / 8;  // code bytes of a 128-row box
  static constexpr int Q_CODE = BN * BK * BITS / 8;     // code bytes of a stage
  static constexpr int Q_BYTES = Q_CODE + (BITS == 4 ? BN * 2 : 0);
  static constexpr int B_OFF = A_ST * A_BYTES;
  static constexpr int Q_OFF = B_OFF + B_ST * B_BYTES;
  static constexpr int BAR_OFF = Q_OFF + Q_ST * Q_BYTES;
  static constexpr int NUM_BARS = 2 * (A_ST + B_ST + Q_ST) + 5;
  static constexpr int SMEM = 1024 + BAR_OFF + NUM_BARS * 8 + 8 + 65 * 4;
  static constexpr int CHUNKS = Q_CODE / 16 / (32 * kConvWarps);  // 16-byte code chunks per thread
  // D f32, A and B f16 (format 0), both K-major, M = MT, N = BN
  static constexpr uint32_t IDESC =
      (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(MT >> 4) << 24);
  static_assert(MT == 64 || MT == 128, "tile rows");
  static_assert(BITS == 8 || BITS == 4, "code width");
  static_assert(Q_BYTES % 16 == 0, "bulk copies need 16-byte stage boundaries");
  static_assert(SMEM <= 232448, "shared memory plan exceeds 227 KiB");
  static_assert(CHUNKS * 32 * kConvWarps * 16 == Q_CODE, "converter split");
};

struct W8Params {
  const uint8_t* q0;     // tiled codes of the first weight (w1 or w2)
  const uint8_t* q1;     // tiled codes of w3 (gate/up only)
  const int32_t* offsets;
  const float* scale_a;  // int8: per-row scales of the first weight (w1 or w2) [E * rows]
  const float* scale_b;  // int8: per-row scales of w3 (gate/up only)
  const uint16_t* gscale_a;  // 4-bit: half group scales of the first weight, tile order
  const uint16_t* gscale_b;  // 4-bit: of w3 (gate/up only)
  int32_t* status;
  void* out;
  int64_t out_ld;
  int E, k_blocks, n_tiles, b_rows;
  unsigned long long timeout_ns;
  // kFused: row_ready[m] counts the gate/up epilogue warps that have stored their rows
  // of h for row tile m; a down tile waits for 4 * (gate/up column tiles) of them
  int32_t* row_ready;
};

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
// Contiguous global -> shared copy of `bytes` (multiple of 16, both ends 16-byte aligned),
// completing on the mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
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

// Bounded wait on an mbarrier phase (as in the bf16 GEMM): false after the CTA aborted
// or after timeout_ns, which it records as kStatusTimeout.
__device__ __noinline__ bool wait_w8(uint32_t bar, uint32_t parity, volatile int* abort_flag,
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

// Wait until *ready >= target (an acquire load: the h rows the gate/up epilogues
// stored before their release are then visible), bounded like the barrier waits.
__device__ __noinline__ bool wait_ready(const int32_t* ready, int target, volatile int* abort_flag,
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

// The same wait executed by all 32 lanes of a warp (they stay converged): an inline
// first test, then the bounded loop.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_w8(bar, parity, abort_flag, status, timeout_ns);
}

__device__ __noinline__ void drain_w8(uint32_t bar, uint32_t parity, int32_t* status,
                                      unsigned long long timeout_ns) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > timeout_ns) {
      atomicOr(status, kStatusUnwound);
      return;
    }
  }
}

__device__ __forceinline__ void tile_coords_w8(int L, const int* row_tiles, int E, int n_tiles,
                                               int& e, int& m, int& n) {
  const int mrow = L / n_tiles;
  e = 0;
  while (e + 1 < E && row_tiles[e + 1] <= mrow) ++e;
  const int cnt = row_tiles[e + 1] - row_tiles[e];
  const int local = L - row_tiles[e] * n_tiles;
  n = local / cnt;
  m = row_tiles[e] + local % cnt;
}

// Tile number (times 128) of weight rows row .. row+127 (row a multiple of 128) and
// k-block kb in the tiled code layout; times 64 bytes it is the tile's byte offset
__device__ __forceinline__ int code_y(int row, int kb, int k_blocks) {
  return ((row >> 7) * k_blocks + kb) * 128;
}

// ---- code layout and widening ----
// Codes are stored offset-binary, u = q + 128 in [1, 255]. A 128-row x 64-column tile
// is one contiguous 8 KiB block: four 2 KiB column chunks (columns 16v .. 16v+15),
// each holding the 128 rows' 16 codes in row order, so a thread that owns a row (or
// consecutive threads that own consecutive rows) read without bank conflicts.
//
// Widening to IEEE half: the half whose high byte is 0x64 and low byte u is 1024 + u
// (exponent 2^10, 10 mantissa bits); subtracting 1152 leaves u - 128 = q exactly. One
// byte permute builds two such halves, one packed subtraction (on the FMA pipe) finishes
// them: half an integer-pipe instruction per code.
__device__ __forceinline__ uint32_t codes_to_f16x2(uint32_t w, uint32_t sel) {
  const uint32_t x = __byte_perm(w, 0x64646464u, sel);
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x64806480u));
  return r;
}

// One word (columns 4m .. 4m+3) -> half pairs (4m, 4m+1) and (4m+2, 4m+3)
__device__ __forceinline__ void widen_word(uint32_t w, uint32_t& p01, uint32_t& p23) {
  p01 = codes_to_f16x2(w, 0x4140u);
  p23 = codes_to_f16x2(w, 0x4342u);
}

// 16 codes (one chunk) -> two 16-byte runs of halves, columns 16v .. 16v+7 and +8 .. +15
__device__ __forceinline__ void widen16(const uint4 w4, uint4& lo8, uint4& hi8) {
  widen_word(w4.x, lo8.x, lo8.y);
  widen_word(w4.y, lo8.z, lo8.w);
  widen_word(w4.z, hi8.x, hi8.y);
  widen_word(w4.w, hi8.z, hi8.w);
}

// 4-bit codes, offset-binary u = q + 8, eight to a 32-bit word: column 2j of the word's
// 8 columns sits in nibble j and column 2j + 1 in nibble j + 4 (j = 0..3), so one
// shift and mask bring a column pair into the low bits of the word's two halves.
// OR-ing in 0x6400 makes the halves 1024 + u (exponent 2^10, exact), subtracting 1032
// leaves q exactly, and one packed multiply forms half(q * s), rounded once.
__device__ __forceinline__ uint32_t nibbles_to_f16x2(uint32_t w, int j, uint32_t s2) {
  const uint32_t x = ((w >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
  uint32_t d, r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(x), "r"(0x64086408u));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(d), "r"(s2));
  return r;
}

// One word (8 columns) -> one 16-byte run of 8 halves, each times the scale pair s2
__device__ __forceinline__ uint4 widen_word4(uint32_t w, uint32_t s2) {
  return make_uint4(nibbles_to_f16x2(w, 0, s2), nibbles_to_f16x2(w, 1, s2),
                    nibbles_to_f16x2(w, 2, s2), nibbles_to_f16x2(w, 3, s2));
}

// Per-channel scale of the int8 codes, applied to the fp32 accumulator; the 4-bit
// weights carry their scales already (a factor of 1, exact)
template <int BITS>
__device__ __forceinline__ float chan_scale(const float* s, int i) {
  if constexpr (BITS == 8) return __ldg(s + i);
  else return 1.f;
}

__device__ __forceinline__ uint32_t pack_f16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// MODE kSwiGLU: A = x_perm [rows, H] (half), weight tile = 128 rows of w1 then 128 rows
//   of w3 (BN = 256), h = half(silu(s1 * gate) * (s3 * up)).
// MODE kPlain:  A = h [rows, I], weight tile = BN rows of w2, y = s2 * acc (fp32).
// MODE kFused:  both in one persistent grid: the gate/up tiles (parameters p, A map
//   mapA) come first, then the down tiles (p2, mapA2, BN = 256). A down tile reads the
//   h rows of its row tile only once every gate/up tile of that row tile has stored
//   them (p.row_ready), so the down tiles fill the SMs the gate/up tail leaves idle.
//   Every gate/up tile precedes every down tile in the order each CTA walks its tiles,
//   so a down tile only ever waits for tiles that are running or done.
template <int MODE, int BN, int MT, int BITS>
__global__ void __launch_bounds__(kThreadsW8, 1)
    k_grouped_gemm_w8(const __grid_constant__ CUtensorMap mapA,
                      const __grid_constant__ CUtensorMap mapA2,
                      const __grid_constant__ W8Params p, const __grid_constant__ W8Params p2) {
  using TL = TileW8<BN, MT, BITS>;
  constexpr int kAStages = TL::A_ST, kBStages = TL::B_ST, kCodeStages = TL::Q_ST;
  constexpr int A_BYTES = TL::A_BYTES;
  static_assert(MODE == kPlain || BN == 256, "gate/up tiles hold 128 gate + 128 up columns");
  constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* bbase = smem + TL::B_OFF;
  uint8_t* qbase = smem + TL::Q_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TL::BAR_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + TL::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* row_tiles = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // barriers: a_full, a_empty [kAStages]; b_full, b_empty [kBStages]; q_full, q_empty
  // [kCodeStages]; tfull, tempty [2]; final
  const uint32_t bar0 = smem_u32(bars);
  constexpr int kB0 = 2 * kAStages, kQ0 = kB0 + 2 * kBStages, kT0 = kQ0 + 2 * kCodeStages;
  auto a_full = [&](int s) { return bar0 + 8u * s; };
  auto a_empty = [&](int s) { return bar0 + 8u * (kAStages + s); };
  auto b_full = [&](int s) { return bar0 + 8u * (kB0 + s); };
  auto b_empty = [&](int s) { return bar0 + 8u * (kB0 + kBStages + s); };
  auto q_full = [&](int q) { return bar0 + 8u * (kQ0 + q); };
  auto q_empty = [&](int q) { return bar0 + 8u * (kQ0 + kCodeStages + q); };
  auto tfull = [&](int a) { return bar0 + 8u * (kT0 + a); };
  auto tempty = [&](int a) { return bar0 + 8u * (kT0 + 2 + a); };
  const uint32_t final_bar = bar0 + 8u * (kT0 + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(a_full(s), 1);
      mbar_init(a_empty(s), 1);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(b_full(s), kConvWarps);
      mbar_init(b_empty(s), 1);
    }
    for (int q = 0; q < kCodeStages; ++q) {
      mbar_init(q_full(q), 1);
      mbar_init(q_empty(q), kConvWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 4);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) row_tiles[i] = p.offsets[i] / BM;
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // tiles L < total0 belong to the first GEMM (p), the rest (kFused) to the down GEMM (p2)
  const int total0 = row_tiles[p.E] * p.n_tiles;
  const int total = total0 + (MODE == kFused ? row_tiles[p.E] * p2.n_tiles : 0);
  auto second = [&](int L) { return MODE == kFused && L >= total0; };
  // tile L -> (expert, row tile, column tile) of its GEMM
  auto coords = [&](int L, int& e, int& m, int& n) {
    const bool d = second(L);
    tile_coords_w8(d ? L - total0 : L, row_tiles, p.E, d ? p2.n_tiles : p.n_tiles, e, m, n);
  };
  auto kblocks = [&](int L) { return second(L) ? p2.k_blocks : p.k_blocks; };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- int8 code stream: BN/128 boxes of 128 rows x 64 codes
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        int e, m, n;
        coords(L, e, m, n);
        const bool dn = second(L);
        const bool sw = MODE == kSwiGLU || (MODE == kFused && !dn);
        const W8Params& g = dn ? p2 : p;
        const int k_blocks = g.k_blocks;
        const int row0 = sw ? e * g.b_rows + n * 128 : e * g.b_rows + n * BN;
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int q = it % kCodeStages;
          const uint32_t ph = (uint32_t)(it / kCodeStages) & 1u;
          if (!wait_w8(q_empty(q), ph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t dq = smem_u32(qbase + q * TL::Q_BYTES);
          mbar_expect_tx(q_full(q), TL::Q_BYTES);
          // code_y / 128 is the tile number: its codes start at byte tile * BOX_CODE
          // and (4-bit) its 128 scales at element tile * 128 = code_y
          constexpr int kBox = TL::BOX_CODE;
          if (sw) {
            const int cy = code_y(row0, kb, k_blocks);
            const size_t off = (size_t)cy * (kBox / 128);
            bulk_load(dq, g.q0 + off, kBox, q_full(q));
            bulk_load(dq + kBox, g.q1 + off, kBox, q_full(q));
            if constexpr (BITS == 4) {
              bulk_load(dq + TL::Q_CODE, g.gscale_a + cy, 256, q_full(q));
              bulk_load(dq + TL::Q_CODE + 256, g.gscale_b + cy, 256, q_full(q));
            }
          } else {
#pragma unroll
            for (int j = 0; j < BN / 128; ++j) {
              const int cy = code_y(row0 + 128 * j, kb, k_blocks);
              bulk_load(dq + j * kBox, g.q0 + (size_t)cy * (kBox / 128), kBox, q_full(q));
              if constexpr (BITS == 4)
                bulk_load(dq + TL::Q_CODE + j * 256, g.gscale_a + cy, 256, q_full(q));
            }
          }
        }
      }
      if (!ok) {
        const int first = it > kCodeStages ? it - kCodeStages : 0;
        for (int i = first; i < it; ++i)
          drain_w8(q_full(i % kCodeStages), (uint32_t)(i / kCodeStages) & 1u, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer (the next stage's barriers are tested before this
      // stage's MMAs issue, so their latency runs under the MMAs)
      int it = 0, tc = 0;
      bool ok = true, issued = false, pre_a = false, pre_b = false;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tc) {
        const int a = tc & 1;
        const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
        if (!wait_w8(tempty(a), aph ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
        fence_after();
        const uint32_t d = tmem_base + (uint32_t)(a * BN);
        const int k_blocks = kblocks(L);
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int sa = it % kAStages, sb = it % kBStages;
          if ((!pre_a && !wait_w8(a_full(sa), (uint32_t)(it / kAStages) & 1u, abort_flag,
                                  p.status, p.timeout_ns)) ||
              (!pre_b && !wait_w8(b_full(sb), (uint32_t)(it / kBStages) & 1u, abort_flag,
                                  p.status, p.timeout_ns))) {
            ok = false;
            break;
          }
          fence_after();
          pre_a = mbar_test_wait(a_full((it + 1) % kAStages), (uint32_t)((it + 1) / kAStages) & 1u);
          pre_b = mbar_test_wait(b_full((it + 1) % kBStages), (uint32_t)((it + 1) / kBStages) & 1u);
          const uint32_t da = smem_u32(smem + sa * A_BYTES);
          const uint32_t db = smem_u32(bbase + sb * TL::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_f16(d, sdesc(da + kk * 32), sdesc(db + kk * 32), TL::IDESC, (kb | kk) ? 1u : 0u);
          mma_commit(a_empty(sa));
          mma_commit(b_empty(sb));
          issued = true;
        }
        if (ok) mma_commit(tfull(a));
      }
      if (issued) {
        mma_commit(final_bar);
        drain_w8(final_bar, 0, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    if (lane == 0) {
      // ---------------- activation tiles (half, 128-byte swizzle by the TMA)
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        int e, m, n;
        coords(L, e, m, n);
        const bool dn = second(L);
        if (dn) {
          // the h rows of this row tile, once every gate/up tile of it has stored them;
          // then a proxy fence, so the tensor copies (async proxy) see those stores
          if (!wait_ready(p.row_ready + m, 4 * p.n_tiles, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        const CUtensorMap* map = dn ? &mapA2 : &mapA;
        const int k_blocks = kblocks(L);
        for (int kb = 0; kb < k_blocks; ++kb, ++it) {
          const int sa = it % kAStages;
          const uint32_t ph = (uint32_t)(it / kAStages) & 1u;
          if (!wait_w8(a_empty(sa), ph ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(a_full(sa), A_BYTES);
          tma_load_2d(smem_u32(smem + sa * A_BYTES), map, kb * BK, m * BM, a_full(sa));
        }
      }
      if (!ok) {
        const int first = it > kAStages ? it - kAStages : 0;
        for (int i = first; i < it; ++i)
          drain_w8(a_full(i % kAStages), (uint32_t)(i / kAStages) & 1u, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp >= kConvWarp0) {
    // ---------------- converters: code tile -> half B tile in the 128-byte
    // swizzled K-major layout (row r: 128 bytes at r * 128, 16-byte chunk c stored at
    // chunk position c ^ (r & 7)). Thread ct widens the 16-byte code chunks
    // j = ct + 32 kConvWarps i of the stage (128-row tile j / 512, column chunk
    // (j / 128) % 4, row j % 128): consecutive threads read consecutive chunks, and the
    // 8 stores of a quarter-warp (8 consecutive rows) land in distinct banks.
    const int ct = threadIdx.x - kConvWarp0 * 32;
    int it = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
      const int k_blocks = kblocks(L);
      for (int kb = 0; kb < k_blocks; ++kb, ++it) {
        const int q = it % kCodeStages, sb = it % kBStages;
        if (!wait_warp(q_full(q), (uint32_t)(it / kCodeStages) & 1u, abort_flag, p.status,
                       p.timeout_ns)) {
          ok = false;
          break;
        }
        const uint4* qs = reinterpret_cast<const uint4*>(qbase + q * TL::Q_BYTES);
        uint4 v[TL::CHUNKS];
        uint32_t sc2[TL::CHUNKS];
#pragma unroll
        for (int i = 0; i < TL::CHUNKS; ++i) {
          const int j = ct + 32 * kConvWarps * i;
          v[i] = qs[j];
          if constexpr (BITS == 4) {
            // 4-bit chunk j: box j / 256, column half (j / 128) % 2, row j % 128; the
            // scale of stage row (j / 256) * 128 + j % 128, as a pair
            const uint16_t* ss =
                reinterpret_cast<const uint16_t*>(qbase + q * TL::Q_BYTES + TL::Q_CODE);
            sc2[i] = (uint32_t)ss[(j >> 8) * 128 + (j & 127)] * 0x10001u;
          } else {
            sc2[i] = 0u;
          }
        }
        if (!wait_warp(b_empty(sb), ((uint32_t)(it / kBStages) & 1u) ^ 1u, abort_flag, p.status,
                       p.timeout_ns)) {
          ok = false;
          break;
        }
        uint8_t* bs = bbase + sb * TL::B_BYTES;
#pragma unroll
        for (int i = 0; i < TL::CHUNKS; ++i) {
          const int j = ct + 32 * kConvWarps * i;
          if constexpr (BITS == 8) {
            const int r = (j >> 9) * 128 + (j & 127), c = ((j >> 7) & 3) * 2;
            uint4 lo8, hi8;
            widen16(v[i], lo8, hi8);
            uint8_t* row = bs + r * 128;
            *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = lo8;
            *reinterpret_cast<uint4*>(row + (((c + 1) ^ (r & 7)) << 4)) = hi8;
          } else {
            // 32 codes of row r, columns 32 (c / 4) .. + 31: four 16-byte runs of halves
            const int r = (j >> 8) * 128 + (j & 127), c = ((j >> 7) & 1) * 4;
            uint8_t* row = bs + r * 128;
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int mw = 0; mw < 4; ++mw)
              *reinterpret_cast<uint4*>(row + (((c + mw) ^ (r & 7)) << 4)) =
                  widen_word4(w[mw], sc2[i]);
          }
        }
        // make the generic-proxy stores visible to the tensor cores (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        // The code stage is released only now: the stores consumed every loaded chunk,
        // so no read of it is still in flight when the next TMA load overwrites it.
        if (lane == 0) {
          mbar_arrive(b_full(sb));
          mbar_arrive(q_empty(q));
        }
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lanes 32 (warp % 4) ..; with MT = 64
    // rows 16 q .. 16 q + 15 sit in the first 16 lanes of quarter q
    const int qd = warp & 3;
    const int row_in_tile = MT == 128 ? qd * 32 + lane : qd * 16 + lane;
    const bool row_valid = MT == 128 || lane < 16;
    int tc = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tc) {
      int e, m, n;
      coords(L, e, m, n);
      const bool dn = second(L);
      const bool sw = MODE == kSwiGLU || (MODE == kFused && !dn);
      const W8Params& g = dn ? p2 : p;
      const int a = tc & 1;
      const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
      if (!wait_warp(tfull(a), aph, abort_flag, p.status, p.timeout_ns)) break;
      fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(a * BN);
      const int64_t row = (int64_t)m * BM + row_in_tile;
      if (sw) {
        const float* sg = BITS == 8 ? g.scale_a + (size_t)e * g.b_rows + n * 128 : nullptr;
        const float* su = BITS == 8 ? g.scale_b + (size_t)e * g.b_rows + n * 128 : nullptr;
        uint16_t* h = reinterpret_cast<uint16_t*>(g.out) + row * g.out_ld + (int64_t)n * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(taddr + c, g);
          tmem_ld16(taddr + 128 + c, u);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g0 = __uint_as_float(g[2 * i]) * chan_scale<BITS>(sg, c + 2 * i);
            const float g1 = __uint_as_float(g[2 * i + 1]) * chan_scale<BITS>(sg, c + 2 * i + 1);
            const float u0 = __uint_as_float(u[2 * i]) * chan_scale<BITS>(su, c + 2 * i);
            const float u1 = __uint_as_float(u[2 * i + 1]) * chan_scale<BITS>(su, c + 2 * i + 1);
            pk[i] = pack_f16x2_rn(g0 / (1.f + __expf(-g0)) * u0, g1 / (1.f + __expf(-g1)) * u1);
          }
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(h + c);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if (MODE == kFused) {
          // release this warp's rows of h to the down tiles of row tile m: the stores,
          // a proxy fence (the readers copy with the async proxy) and a gpu-scope fence
          // before the count
          asm volatile("fence.proxy.async.global;" ::: "memory");
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.row_ready + m, 1);
        }
      } else {
        const float* sc = BITS == 8 ? g.scale_a + (size_t)e * g.b_rows + n * BN : nullptr;
        float* y = reinterpret_cast<float*>(g.out) + row * g.out_ld + (int64_t)n * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + c, v);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(y + c);
#pragma unroll
          for (int i = 0; i < 4 && row_valid; ++i)
            dst[i] = make_float4(__uint_as_float(v[4 * i]) * chan_scale<BITS>(sc, c + 4 * i),
                                 __uint_as_float(v[4 * i + 1]) * chan_scale<BITS>(sc, c + 4 * i + 1),
                                 __uint_as_float(v[4 * i + 2]) * chan_scale<BITS>(sc, c + 4 * i + 2),
                                 __uint_as_float(v[4 * i + 3]) * chan_scale<BITS>(sc, c + 4 * i + 3));
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(a));
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- small batches
//
// k_w8_decode: both expert GEMMs of a batch of at most 256 tokens, in one persistent
// grid, with the operands swapped. A token reaches an expert at most once, so up to 64
// tokens each expert has at most 64 routed rows, all in its one 128-row tile. The tile
// kernel above spends a full M = 64 MMA and an 8 KiB activation tile on every 64-wide
// k-block for those few rows. Here the weights are the tcgen05 M operand (128 weight
// rows per tile) and a sub-tile of at most NMAX of the expert's routed rows the N
// operand (N = the sub-tile's row count rounded up to 16), so the MMAs shrink with the
// batch. An expert with more than NMAX rows has several sub-tiles over the same weight
// tiles: consecutive tiles, so the codes of all but the first come from L2 (the widening
// is repeated). The widened weights never touch shared memory:
//
//   warp 0      streams code stages into a deep ring (bulk copies): a stage is four
//               128-row x 64-code boxes, gate/up the w1 and w3 boxes of two k-blocks,
//               down four consecutive k-blocks of one w2 box (4-bit: plus their scales);
//   warps 7-22  widen them, one thread per weight row: converter warp c takes box c / 4
//               and TMEM lanes 32 (warp % 4) .. + 31, reads its row's codes with 4
//               (int8) or 2 (4-bit) conflict-free 16-byte loads and writes 32 columns of
//               half pairs with one tcgen05.st: the tensor-memory layout of an M = 128
//               A operand (lane = row, column c = K elements 2c and 2c + 1);
//   warp 6      loads the routed rows' k-blocks (TMA, 16-row boxes, 128-byte swizzle);
//               a down tile first waits until every gate/up tile of its sub-tile has
//               released its rows of h (per-sub-tile counters);
//   warps 1, 23 issue tcgen05.mma with A in tensor memory and B (the rows) in shared
//               memory, M = 128, N = rows, each half of every stage: gate/up the first
//               issues gate and the second up, down each issues two of the four k-blocks
//               into its own partial sum (the epilogue adds the two);
//   warps 2-5   read the accumulators (lane = weight row, column = routed row): h =
//               half(silu(s1 gate) * s3 up) at [row, i], y = s2 acc at [row, j].
//
// Tiles: gate/up tile (sub-tile, n) covers intermediate columns 128 n .. + 127 over
// H / 128 stages; down tile (sub-tile, n) covers hidden columns 128 n .. + 127 over
// I / 256 stages. Every gate/up tile precedes every down tile in the order each CTA
// walks its tiles, and the grid is at most one CTA per SM, so a down tile only waits for
// tiles that are running or done.
//
// Measured on B200, and what the plan does about it. (1) An MMA of this shape (M = 128,
// N <= 64, K = 16) occupies the issuing thread for about 45 SM clocks whatever N is, so
// sixteen are about 710 clocks: below the HBM time of the 32 KiB of int8 codes they
// consume. (2) In the MMA thread, between MMAs, a commit costs about 55 clocks, a
// non-blocking test_wait about 53, and a wait whose result steers the thread about 340
// even on a phase that has long completed: barrier traffic, not the tensor pipe, set
// the pace of small stages. So a stage is 128 columns of K (sixteen MMAs), each role
// tests the barriers of its next stage with test_wait before it starts the current one
// (the latency runs under its work) and blocks only if that test failed. (3) Separate
// accumulators per MMA do not help (the pipe is not waiting on accumulation), but a
// second issuing thread does: two threads issue N = 16 MMAs at about 38 clocks each
// against 51 for one, so two threads split every stage.
template <int BITS, int NMAX>
struct DecW8 {
  static constexpr int BOX = 128 * BK * BITS / 8;                  // code bytes of a box
  static constexpr int SUBS = 4;                                   // boxes per stage
  static constexpr int Q_BYTES = SUBS * BOX + (BITS == 4 ? SUBS * 256 : 0);
  static constexpr int ACT_UNIT = NMAX * 128;                      // NMAX rows of one k-block
  static constexpr int ACC_COLS = 2 * NMAX;                        // one buffer: gate, up
  static constexpr int W_COL0 = 2 * ACC_COLS;                      // two buffers
  static constexpr int W_SLOT_COLS = SUBS * 32;                    // a widened stage
  static constexpr int W_SLOTS = (512 - W_COL0) / W_SLOT_COLS;     // widened stages in TMEM
  static constexpr int ACT_SLOT = SUBS * ACT_UNIT;                 // a slot's rows (down: 4 k-blocks)
  static constexpr int Q_FIT = (200 * 1024 - W_SLOTS * ACT_SLOT) / Q_BYTES;
  static constexpr int Q_ST = Q_FIT > 16 ? 16 : Q_FIT;
  static constexpr int CONV_WARPS = 4 * SUBS;                      // one box per warp
  static constexpr int MMA_WARP2 = 7 + CONV_WARPS;                 // the second MMA issuer
  static constexpr int THREADS = 32 * (8 + CONV_WARPS);
  static constexpr int Q_OFF = W_SLOTS * ACT_SLOT;
  static constexpr int BAR_OFF = Q_OFF + Q_ST * Q_BYTES;
  static constexpr int NUM_BARS = 2 * Q_ST + 3 * W_SLOTS + 4 + 2;
  static constexpr int SMEM = 1024 + BAR_OFF + NUM_BARS * 8 + 16 + 3 * 72 * 4;
  // D f32, A and B f16, both K-major, M = 128; N is set per tile
  static constexpr uint32_t IDESC_M128 = (1u << 4) | ((uint32_t)(128 >> 4) << 24);
  static_assert(NMAX == 16 || NMAX == 32 || NMAX == 64, "rows per sub-tile");
  static_assert(W_SLOTS >= 2 && Q_ST >= 3, "pipeline plan");
  static_assert(Q_BYTES % 16 == 0 && ACT_UNIT % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 232448, "shared memory plan exceeds 227 KiB");
};


struct DecParams {
  const uint8_t* q1;
  const uint8_t* q3;
  const uint8_t* q2;
  const float* s1;   // int8: per-row scales
  const float* s3;
  const float* s2;
  const uint16_t* g1;  // 4-bit: half group scales, tile order
  const uint16_t* g3;
  const uint16_t* g2;
  const int32_t* offsets;  // [E+1], multiples of 128
  const int32_t* counts;   // [E] routed rows per expert, or null (then min(max_rows, padded))
  uint16_t* h;             // [rows, I] half
  float* y;                // [rows, H] fp32
  int32_t* status;
  int32_t* row_ready;      // [rows / 64] per-sub-tile counters, zero at launch
  int E, H, I;
  int max_rows;            // most rows an expert can have: the tokens
  unsigned long long timeout_ns;
};

// Eight MMAs of one issuer's half of a stage in one asm block: boxes j = 0, 1 at TMEM
// columns a + 32 j, the rows of k-block j at the B descriptor + j * unit16; a K step
// moves A by 8 columns and the B descriptor by 2 (32 bytes). Only the first MMA honours
// `acc` (0 starts the tile's accumulator); the others accumulate.
template <int UNIT16>
__device__ __forceinline__ void mma_stage_half(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                               uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .b32 ak;\n\t.reg .b64 bk;\n\t"
      "setp.ne.b32 p0, %4, 0;\n\tsetp.eq.b32 p1, %4, %4;\n\t"
      "mov.b64 bk, %2;\n\tmov.b32 ak, %1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p0;\n\t"
      "add.s64 bk, bk, 2;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "add.s64 bk, bk, 2;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "add.s64 bk, bk, 2;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "add.s64 bk, bk, %5;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "add.s64 bk, bk, 2;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "add.s64 bk, bk, 2;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "add.s64 bk, bk, 2;\n\t"
      "add.u32 ak, ak, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], bk, %3, p1;\n\t"
      "}" ::"r"(d), "r"(a), "l"(b), "r"(idesc), "r"(acc), "n"(UNIT16 - 6)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint16_t half_rn(float f) {
  uint16_t v;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(v) : "f"(f));
  return v;
}

// 4-bit word (8 columns) -> four half pairs times the scale pair s2, the same values
// as widen_word4 with fewer instructions: the pairs in nibbles (1, 5) and (3, 7) are
// masked in place, giving half 1024 + 16u, and one packed fma by 1/16 minus 72 leaves
// q = u - 8 exactly (every intermediate is an integer below 2048); the pairs in
// nibbles (0, 4) and (2, 6) give 1024 + u, minus 1032. One multiply by the scale then
// rounds q * s once, as before.
__device__ __forceinline__ void widen_word4_pairs(uint32_t w, uint32_t s2, uint32_t* out) {
  const uint32_t ws = w >> 8;
  const uint32_t x0 = (w & 0x000F000Fu) | 0x64006400u;
  const uint32_t x1 = (w & 0x00F000F0u) | 0x64006400u;
  const uint32_t x2 = (ws & 0x000F000Fu) | 0x64006400u;
  const uint32_t x3 = (ws & 0x00F000F0u) | 0x64006400u;
  uint32_t q0, q1, q2, q3;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q0) : "r"(x0), "r"(0x64086408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q1) : "r"(x1), "r"(0x2C002C00u), "r"(0xD480D480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q2) : "r"(x2), "r"(0x64086408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q3) : "r"(x3), "r"(0x2C002C00u), "r"(0xD480D480u));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[0]) : "r"(q0), "r"(s2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[1]) : "r"(q1), "r"(s2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[2]) : "r"(q2), "r"(s2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[3]) : "r"(q3), "r"(s2));
}

template <int BITS, int NMAX>
__global__ void __launch_bounds__(DecW8<BITS, NMAX>::THREADS, 1)
    k_w8_decode(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapH,
                const __grid_constant__ DecParams p) {
  using D = DecW8<BITS, NMAX>;
  constexpr int kQ = D::Q_ST, kW = D::W_SLOTS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* qbase = smem + D::Q_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + D::BAR_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + D::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* sub0 = reinterpret_cast<int*>(tmem_holder + 4);  // [E + 1]: first sub-tile of each expert
  int* nrows = sub0 + 72;                                // [E]: routed rows of each expert
  int* row_off = nrows + 72;                             // [E]: first row of each expert

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // barriers: q_full, q_empty [kQ]; w_full (widened slot), a_full (the slot's rows),
  // w_empty (slot and rows free) [kW]; t_full, t_empty [2]; final
  const uint32_t bar0 = smem_u32(bars);
  constexpr int kW0 = 2 * kQ, kT0 = kW0 + 3 * kW;
  auto q_full = [&](int s) { return bar0 + 8u * s; };
  auto q_empty = [&](int s) { return bar0 + 8u * (kQ + s); };
  auto w_full = [&](int s) { return bar0 + 8u * (kW0 + s); };
  auto a_full = [&](int s) { return bar0 + 8u * (kW0 + kW + s); };
  auto w_empty = [&](int s) { return bar0 + 8u * (kW0 + 2 * kW + s); };
  auto t_full = [&](int b) { return bar0 + 8u * (kT0 + b); };
  auto t_empty = [&](int b) { return bar0 + 8u * (kT0 + 2 + b); };
  const uint32_t final_bar = bar0 + 8u * (kT0 + 4);  // and final_bar + 8: one per issuer
  auto act = [&](int ws) { return smem_u32(smem + ws * D::ACT_SLOT); };
  const int kb1 = p.H / BK, kb2 = p.I / BK;  // k-blocks of the gate/up and down weights
  // phase parity of the barrier a stage uses (ring of n), and of its previous use
  auto ph = [](int it, int n) { return (uint32_t)(it / n) & 1u; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQ; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), D::CONV_WARPS);
    }
    for (int s = 0; s < kW; ++s) {
      mbar_init(w_full(s), D::CONV_WARPS);
      mbar_init(a_full(s), 1);
      mbar_init(w_empty(s), 2);  // both issuers' commits
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
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(512u)
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
  auto sub_rows = [&](int e, int m) {
    const int n = (nrows[e] - (m - sub0[e]) * NMAX + 15) & ~15;
    return n < 16 ? 16 : (n > NMAX ? NMAX : n);
  };

  const int n1 = p.I / 128, n2 = p.H / 128;  // column tiles per sub-tile
  const int st1 = p.H / (2 * BK), st2 = p.I / (4 * BK);  // stages per tile
  const int total0 = sub0[p.E] * n1;
  const int total = total0 + sub0[p.E] * n2;
  // the sub-tiles of one expert and column tile are consecutive tiles
  auto coords = [&](int L, bool& dn, int& e, int& m, int& n) {
    dn = L >= total0;
    tile_coords_w8(dn ? L - total0 : L, sub0, p.E, dn ? n2 : n1, e, m, n);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- code stages
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        bool dn;
        int e, m, n;
        coords(L, dn, e, m, n);
        const int nst = dn ? st2 : st1;
        for (int s = 0; s < nst; ++s, ++it) {
          const int q = it % kQ;
          if (!wait_w8(q_empty(q), ph(it, kQ) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          const uint32_t dq = smem_u32(qbase + q * D::Q_BYTES);
          mbar_expect_tx(q_full(q), D::Q_BYTES);
          // boxes of one row tile and consecutive k-blocks are adjacent in memory (and
          // so are their scales)
          if (!dn) {
            // boxes 0, 1: w1 rows 128 n .. of expert e, k-blocks 2s, 2s + 1; boxes 2, 3: w3
            const int cy = code_y(e * p.I + n * 128, 2 * s, kb1);
            const size_t off = (size_t)cy * (D::BOX / 128);
            bulk_load(dq, p.q1 + off, 2 * D::BOX, q_full(q));
            bulk_load(dq + 2 * D::BOX, p.q3 + off, 2 * D::BOX, q_full(q));
            if constexpr (BITS == 4) {
              bulk_load(dq + 4 * D::BOX, p.g1 + cy, 512, q_full(q));
              bulk_load(dq + 4 * D::BOX + 512, p.g3 + cy, 512, q_full(q));
            }
          } else {
            // boxes 0..3: k-blocks 4s .. 4s + 3 of the w2 box of rows 128 n ..
            const int cy = code_y(e * p.H + n * 128, 4 * s, kb2);
            bulk_load(dq, p.q2 + (size_t)cy * (D::BOX / 128), 4 * D::BOX, q_full(q));
            if constexpr (BITS == 4) bulk_load(dq + 4 * D::BOX, p.g2 + cy, 1024, q_full(q));
          }
        }
      }
      if (!ok) {
        const int first = it > kQ ? it - kQ : 0;
        for (int i = first; i < it; ++i) drain_w8(q_full(i % kQ), ph(i, kQ), p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    if (lane == 0) {
      // ---------------- routed rows of each stage into its slot's buffer: two k-blocks
      // (gate/up) or four (down), N rows in 16-row boxes
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        bool dn;
        int e, m, n;
        coords(L, dn, e, m, n);
        if (dn) {
          // every gate/up tile of sub-tile m has stored its rows of h; the proxy fence
          // orders those stores before the tensor copies (async proxy) that read them
          if (!wait_ready(p.row_ready + m, 4 * n1, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        const int nrow = sub_rows(e, m), row0 = sub_row0(e, m);
        const CUtensorMap* map = dn ? &mapH : &mapX;
        const int nst = dn ? st2 : st1;
        const int nblk = dn ? 4 : 2;
        for (int s = 0; s < nst; ++s, ++it) {
          const int ws = it % kW;
          if (!wait_w8(w_empty(ws), ph(it, kW) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(a_full(ws), (uint32_t)(nblk * nrow * 128));
          for (int b = 0; b < nblk; ++b) {
            const int xk = (nblk * s + b) * BK;
            for (int j = 0; j < nrow; j += 16)
              tma_load_2d(act(ws) + b * D::ACT_UNIT + j * 128, map, xk, row0 + j, a_full(ws));
          }
        }
      }
      if (!ok) {
        const int first = it > kW ? it - kW : 0;
        for (int i = first; i < it; ++i) drain_w8(a_full(i % kW), ph(i, kW), p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == D::MMA_WARP2) {
    if (lane == 0) {
      // ---------------- MMA issuers (mi = 0, 1), each half of every stage. The next
      // stage's barriers are tested before this stage's MMAs issue, so their latency
      // runs under the MMAs.
      const int mi = warp == 1 ? 0 : 1;
      int it = 0, tc = 0;
      bool ok = true, issued = false, pre_w = false, pre_a = false;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tc) {
        bool dn;
        int e, m, n;
        coords(L, dn, e, m, n);
        const uint32_t idesc = D::IDESC_M128 | ((uint32_t)(sub_rows(e, m) >> 3) << 17);
        const int b = tc & 1;
        if (!wait_w8(t_empty(b), ph(tc, 2) ^ 1u, abort_flag, p.status, p.timeout_ns)) break;
        fence_after();
        const uint32_t dacc = tmem_base + (uint32_t)(b * D::ACC_COLS);
        const int nst = dn ? st2 : st1;
        for (int s = 0; s < nst; ++s, ++it) {
          const int ws = it % kW;
          if ((!pre_w && !wait_w8(w_full(ws), ph(it, kW), abort_flag, p.status, p.timeout_ns)) ||
              (!pre_a && !wait_w8(a_full(ws), ph(it, kW), abort_flag, p.status, p.timeout_ns))) {
            ok = false;
            break;
          }
          fence_after();
          pre_w = mbar_test_wait(w_full((it + 1) % kW), ph(it + 1, kW));
          pre_a = mbar_test_wait(a_full((it + 1) % kW), ph(it + 1, kW));
          // gate/up: issuer 0 gate (boxes 0, 1: w1), issuer 1 up (boxes 2, 3: w3), both
          // over the rows of k-blocks 0, 1; down: issuer mi boxes (k-blocks) 2 mi, 2 mi + 1
          // into partial sum mi
          const uint32_t wcol =
              tmem_base + (uint32_t)(D::W_COL0 + ws * D::W_SLOT_COLS + mi * 64);
          const uint64_t bd = sdesc(act(ws) + (dn ? mi * 2 * D::ACT_UNIT : 0));
          mma_stage_half<D::ACT_UNIT / 16>(dacc + mi * NMAX, wcol, bd, idesc, s ? 1u : 0u);
          mma_commit(w_empty(ws));
          issued = true;
        }
        if (ok) mma_commit(t_full(b));
      }
      if (issued) {
        mma_commit(final_bar + 8u * mi);
        drain_w8(final_bar + 8u * mi, 0, p.status, p.timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp >= 7 && warp < D::MMA_WARP2) {
    // ---------------- converters: thread = one weight row of box (warp - 7) / 4. The
    // next stage's barriers are tested before this stage's widening.
    const int sub = (warp - 7) >> 2, quarter = warp & 3;
    const int r = 32 * quarter + lane;
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    int it = 0;
    bool ok = true, pre_q = false, pre_w = false;
    for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
      const int nst = L >= total0 ? st2 : st1;
      for (int s = 0; s < nst; ++s, ++it) {
        const int q = it % kQ, ws = it % kW;
        if (!pre_q && !wait_warp(q_full(q), ph(it, kQ), abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        const int nx = it + 1;
        pre_q = mbar_test_wait(q_full(nx % kQ), ph(nx, kQ));
        const uint8_t* box = qbase + q * D::Q_BYTES + sub * D::BOX;
        uint32_t out[32];
        if constexpr (BITS == 8) {
          // chunk v: columns 16 v .. 16 v + 15 of the 128 rows, 16 bytes per row
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 c = *reinterpret_cast<const uint4*>(box + v * 2048 + r * 16);
            uint4 lo8, hi8;
            widen16(c, lo8, hi8);
            out[8 * v + 0] = lo8.x;
            out[8 * v + 1] = lo8.y;
            out[8 * v + 2] = lo8.z;
            out[8 * v + 3] = lo8.w;
            out[8 * v + 4] = hi8.x;
            out[8 * v + 5] = hi8.y;
            out[8 * v + 6] = hi8.z;
            out[8 * v + 7] = hi8.w;
          }
        } else {
          // half hf: columns 32 hf .. 32 hf + 31, one 32-bit word per 8 columns
          const uint16_t* sc =
              reinterpret_cast<const uint16_t*>(qbase + q * D::Q_BYTES + D::SUBS * D::BOX + sub * 256);
          const uint32_t s2 = (uint32_t)sc[r] * 0x10001u;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint4 c = *reinterpret_cast<const uint4*>(box + hf * 2048 + r * 16);
            widen_word4_pairs(c.x, s2, out + 16 * hf + 0);
            widen_word4_pairs(c.y, s2, out + 16 * hf + 4);
            widen_word4_pairs(c.z, s2, out + 16 * hf + 8);
            widen_word4_pairs(c.w, s2, out + 16 * hf + 12);
          }
        }
        // the codes are in registers: the stage may be refilled
        __syncwarp();
        if (lane == 0) mbar_arrive(q_empty(q));
        if (!pre_w && !wait_warp(w_empty(ws), ph(it, kW) ^ 1u, abort_flag, p.status, p.timeout_ns)) {
          ok = false;
          break;
        }
        pre_w = mbar_test_wait(w_empty(nx % kW), ph(nx, kW) ^ 1u);
        __syncwarp();
        fence_after();
        tmem_st32(tmem_base + lane_addr + (uint32_t)(D::W_COL0 + ws * D::W_SLOT_COLS + sub * 32), out);
        tmem_wait_st();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(w_full(ws));
      }
    }
  } else {
    // ---------------- epilogue: warps 2..5, TMEM lanes 32 (warp % 4) .. = weight rows
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;
    int tc = 0;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tc) {
      bool dn;
      int e, m, n;
      coords(L, dn, e, m, n);
      const int nrow = sub_rows(e, m);
      const int b = tc & 1;
      if (!wait_warp(t_full(b), ph(tc, 2), abort_flag, p.status, p.timeout_ns)) break;
      fence_after();
      const uint32_t tacc =
          tmem_base + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(b * D::ACC_COLS);
      const int64_t row0 = sub_row0(e, m);
      if (!dn) {
        const int i = n * 128 + r;  // intermediate column
        const float sg = BITS == 8 ? __ldg(p.s1 + (size_t)e * p.I + i) : 1.f;
        const float su = BITS == 8 ? __ldg(p.s3 + (size_t)e * p.I + i) : 1.f;
        uint16_t* hcol = p.h + row0 * p.I + i;
        for (int c0 = 0; c0 < nrow; c0 += 16) {
          uint32_t g[16], u[16];
          tmem_ld16(tacc + c0, g);
          tmem_ld16(tacc + NMAX + c0, u);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float gv = __uint_as_float(g[t]) * sg, uv = __uint_as_float(u[t]) * su;
            hcol[(int64_t)(c0 + t) * p.I] = half_rn(gv / (1.f + __expf(-gv)) * uv);
          }
        }
        // release this warp's rows of h to the down tiles of sub-tile m
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(p.row_ready + m, 1);
      } else {
        const int j = n * 128 + r;  // hidden column
        const float sc = BITS == 8 ? __ldg(p.s2 + (size_t)e * p.H + j) : 1.f;
        float* ycol = p.y + row0 * p.H + j;
        for (int c0 = 0; c0 < nrow; c0 += 16) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tacc + c0, v0);
          tmem_ld16(tacc + NMAX + c0, v1);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t)
            ycol[(int64_t)(c0 + t) * p.H] = (__uint_as_float(v0[t]) + __uint_as_float(v1[t])) * sc;
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512u)
                 : "memory");
  }
}

// bf16 rows -> IEEE half rows (round to nearest even), 8 values per thread-step
__global__ void __launch_bounds__(256) k_rows_to_f16(const uint4* __restrict__ src,
                                                     uint4* __restrict__ dst, int64_t n8) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(src + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      o[j] = pack_f16x2_rn(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// One warp per weight row: s = max|w| / 127, q = rint(w / s) in float32, written in
// the tiled code layout: tile (row / 128, column / 64) is the 8 KiB block number
// (row / 128) * (K / 64) + column / 64, arranged inside as described above.
__global__ void __launch_bounds__(256) k_quant_rows(const uint16_t* __restrict__ w,
                                                    uint8_t* __restrict__ q, float* __restrict__ s,
                                                    int64_t rows, int K) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int kbn = K / BK;
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const uint16_t* wr = w + r * K;
    float amax = 0.f;
    for (int c = lane; c < K; c += 32) amax = fmaxf(amax, fabsf(__uint_as_float((uint32_t)wr[c] << 16)));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float sc = amax > 0.f ? __fdiv_rn(amax, 127.f) : 1.f;
    if (lane == 0) s[r] = sc;
    const int64_t rb = r >> 7, rr = r & 127;
    for (int c = lane; c < K; c += 32) {
      const float v = __uint_as_float((uint32_t)wr[c] << 16);
      int qi = __float2int_rn(__fdiv_rn(v, sc));
      qi = qi > 127 ? 127 : (qi < -127 ? -127 : qi);
      const int64_t kb = c / BK, cc = c % BK;
      // byte of column cc in the tile: chunk cc / 16, row rr, column cc % 16
      const int64_t in_tile = (cc >> 4) * 2048 + rr * 16 + (cc & 15);
      q[(rb * kbn + kb) * (128 * BK) + in_tile] = (uint8_t)(qi + 128);
    }
  }
}

__device__ __forceinline__ uint16_t f32_to_f16_rn(float f) {
  uint16_t h;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}
__device__ __forceinline__ float f16_to_f32(uint16_t h) {
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

// One warp per weight row, four 64-column groups per step (8 lanes to a group, 8
// consecutive columns to a lane): s = half(max|w| / 7) (1 when that is zero), q =
// rint(w / s) clamped to [-7, 7], in float32. A lane packs its 8 codes (plus 8) into
// one word of the tiled 4-bit layout; the group's first lane writes the scale.
__global__ void __launch_bounds__(256) k_quant_groups4(const uint16_t* __restrict__ w,
                                                       uint8_t* __restrict__ q,
                                                       uint16_t* __restrict__ s, int64_t rows,
                                                       int K) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, grp = lane >> 3, m8 = lane & 7;
  const int kbn = K / BK;
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const uint16_t* wr = w + r * K;
    const int64_t rb = r >> 7, rr = r & 127;
    for (int kb0 = 0; kb0 < kbn; kb0 += 4) {
      const int kb = kb0 + grp;
      const bool act = kb < kbn;
      float v[8];
      if (act) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(wr + kb * BK + 8 * m8));
        const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          v[2 * t] = __uint_as_float(ww[t] << 16);
          v[2 * t + 1] = __uint_as_float(ww[t] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
      for (int off = 1; off < 8; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      uint16_t sh = f32_to_f16_rn(__fdiv_rn(amax, 7.f));
      if ((sh & 0x7FFFu) == 0) sh = 0x3C00u;  // a zero scale (in half) becomes 1
      const float sd = f16_to_f32(sh);
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        int qi = __float2int_rn(__fdiv_rn(v[i], sd));
        qi = qi > 7 ? 7 : (qi < -7 ? -7 : qi);
        const int nib = (i & 1) ? 4 + (i >> 1) : (i >> 1);
        word |= (uint32_t)(qi + 8) << (4 * nib);
      }
      if (act) {
        const int64_t tile = rb * kbn + kb;
        *reinterpret_cast<uint32_t*>(q + tile * (128 * BK / 2) + (m8 >> 2) * 2048 + rr * 16 +
                                     (m8 & 3) * 4) = word;
        if (m8 == 0) s[tile * 128 + rr] = sh;
      }
    }
  }
}

typedef CUresult (*EncodeTiledFnW8)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnW8 encode_w8() {
  static EncodeTiledFnW8 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnW8>(f);
  }
  return fn;
}

// half activations [rows, inner], box 64 x box_rows, 128-byte swizzle
bool map_act(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFnW8 fn = encode_w8();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int BN, int MT, int BITS>
cudaError_t launch_w8(const CUtensorMap& a, const W8Params& p, int64_t max_tiles, cudaStream_t st,
                      const CUtensorMap* a2 = nullptr, const W8Params* p2 = nullptr) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm_w8<MODE, BN, MT, BITS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         TileW8<BN, MT, BITS>::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int64_t grid = num_sms();
  if (grid > max_tiles) grid = max_tiles;
  if (grid < 1) grid = 1;
  return launch_pdl(k_grouped_gemm_w8<MODE, BN, MT, BITS>, dim3((unsigned)grid), dim3(kThreadsW8),
                    (size_t)TileW8<BN, MT, BITS>::SMEM, st, a, a2 ? *a2 : a, p, p2 ? *p2 : p);
}

}  // namespace

cudaError_t launch_rows_to_f16(const uint16_t* src, uint16_t* dst, int64_t rows, int H,
                               cudaStream_t st) {
  const int64_t n8 = rows * H / 8;
  int64_t blocks = (n8 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_pdl(k_rows_to_f16, dim3((unsigned)blocks), dim3(256), 0, st,
                    reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), n8);
}

cudaError_t launch_quant_rows(const uint16_t* w, uint8_t* q, float* s, int64_t rows, int K,
                              cudaStream_t st) {
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_quant_rows, dim3((unsigned)blocks), dim3(256), 0, st, w, q, s, rows, K);
}

cudaError_t launch_quant_groups4(const uint16_t* w, uint8_t* q, uint16_t* s, int64_t rows, int K,
                                 cudaStream_t st) {
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  return launch_pdl(k_quant_groups4, dim3((unsigned)blocks), dim3(256), 0, st, w, q, s, rows, K);
}

namespace {

// Both GEMMs with MT-row tiles (see TileW8), BITS-bit codes
template <int MT, int BITS>
cudaError_t launch_swiglu_w8_tiles(const Shape& s, const GemmArgsW8& g, cudaStream_t st,
                                   const char** why) {
  CUtensorMap mx, mh;
  if (!map_act(&mx, g.a, s.H, g.rmax, MT) || !map_act(&mh, g.h, s.I, g.rmax, MT)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor)";
    return cudaErrorInvalidValue;
  }
  const int64_t mt_max = g.rmax / BM;
  W8Params p1 = {};
  p1.q0 = g.q1;
  p1.q1 = g.q3;
  p1.offsets = g.offsets;
  p1.scale_a = g.s1;
  p1.scale_b = g.s3;
  p1.gscale_a = g.g1;
  p1.gscale_b = g.g3;
  p1.status = g.status;
  p1.out = g.h;
  p1.out_ld = s.I;
  p1.E = s.E;
  p1.k_blocks = s.H / BK;
  p1.n_tiles = s.I / 128;
  p1.b_rows = s.I;
  p1.timeout_ns = g.timeout_ns;
  W8Params p2 = p1;
  p2.q0 = g.q2;
  p2.q1 = nullptr;
  p2.scale_a = g.s2;
  p2.scale_b = nullptr;
  p2.gscale_a = g.g2;
  p2.gscale_b = nullptr;
  p2.out = g.y;
  p2.out_ld = s.H;
  p2.k_blocks = s.I / BK;
  p2.b_rows = s.H;
  cudaError_t e;
  if (s.H % 256 == 0 && g.row_ready) {
    // one grid for both GEMMs; the row-tile counters start at zero
    p2.n_tiles = s.H / 256;
    p1.row_ready = g.row_ready;
    e = cudaMemsetAsync(g.row_ready, 0, (size_t)mt_max * sizeof(int32_t), st);
    if (e == cudaSuccess)
      e = launch_w8<kFused, 256, MT, BITS>(mx, p1, mt_max * (p1.n_tiles + p2.n_tiles), st, &mh, &p2);
    if (e != cudaSuccess)
      *why = BITS == 8 ? "int8 expert GEMMs launch failed" : "4-bit expert GEMMs launch failed";
    return e;
  }
  e = launch_w8<kSwiGLU, 256, MT, BITS>(mx, p1, mt_max * p1.n_tiles, st);
  if (e != cudaSuccess) {
    *why = BITS == 8 ? "int8 gate/up GEMM launch failed" : "4-bit gate/up GEMM launch failed";
    return e;
  }
  if (s.H % 256 == 0) {
    p2.n_tiles = s.H / 256;
    e = launch_w8<kPlain, 256, MT, BITS>(mh, p2, mt_max * p2.n_tiles, st);
  } else {
    p2.n_tiles = s.H / 128;
    e = launch_w8<kPlain, 128, MT, BITS>(mh, p2, mt_max * p2.n_tiles, st);
  }
  if (e != cudaSuccess)
    *why = BITS == 8 ? "int8 down GEMM launch failed" : "4-bit down GEMM launch failed";
  return e;
}

// Both GEMMs on the swap-operand kernel (sub-tiles of at most NMAX routed rows)
template <int BITS, int NMAX>
cudaError_t launch_w8_decode(const Shape& s, const GemmArgsW8& g, cudaStream_t st,
                             const char** why) {
  using D = DecW8<BITS, NMAX>;
  CUtensorMap mx, mh;
  if (!map_act(&mx, g.a, s.H, g.rmax, 16) || !map_act(&mh, g.h, s.I, g.rmax, 16)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or bad tensor)";
    return cudaErrorInvalidValue;
  }
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_w8_decode<BITS, NMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM);
    if (e != cudaSuccess) {
      *why = "expert GEMM shared-memory attribute";
      return e;
    }
    attr_set[dev] = true;
  }
  DecParams p = {};
  p.q1 = g.q1;
  p.q3 = g.q3;
  p.q2 = g.q2;
  p.s1 = g.s1;
  p.s3 = g.s3;
  p.s2 = g.s2;
  p.g1 = g.g1;
  p.g3 = g.g3;
  p.g2 = g.g2;
  p.offsets = g.offsets;
  p.counts = g.counts;
  p.h = g.h;
  p.y = g.y;
  p.status = g.status;
  p.row_ready = g.row_ready;
  p.E = s.E;
  p.H = s.H;
  p.I = s.I;
  p.max_rows = (int)s.T;
  p.timeout_ns = g.timeout_ns;
  // the sub-tile counters start at zero; an expert of c rows has ceil(c / NMAX) sub-tiles,
  // so there are at most T k / NMAX + E of them, within rmax / 64 (rmax >= T k + 128 E)
  // (unless a kernel before this one zeroed them, so that this launch overlaps its tail)
  const int64_t subs = (int64_t)s.T * s.k / NMAX + s.E;
  cudaError_t e = g.row_ready_zeroed
                      ? cudaSuccess
                      : cudaMemsetAsync(g.row_ready, 0, (size_t)(g.rmax / 64) * sizeof(int32_t), st);
  if (e == cudaSuccess) {
    const int64_t tiles = subs * (s.I / 128 + s.H / 128);
    int64_t grid = std::min<int64_t>(num_sms(), tiles);
    if (grid < 1) grid = 1;
    e = launch_pdl(k_w8_decode<BITS, NMAX>, dim3((unsigned)grid), dim3(D::THREADS),
                   (size_t)D::SMEM, st, mx, mh, p);
  }
  if (e != cudaSuccess)
    *why = BITS == 8 ? "int8 expert GEMMs launch failed" : "4-bit expert GEMMs launch failed";
  return e;
}

}  // namespace

cudaError_t launch_grouped_swiglu_w8(const Shape& s, const GemmArgsW8& g, cudaStream_t st,
                                     const char** why) {
  // a token is routed to an expert at most once, so with at most 64 tokens every expert
  // has at most 64 rows, all in the first half of its 128-row tile
  const bool half_tiles = s.T <= 64 && kUseHalfTiles;
  // the swap-operand kernel: at most 64 tokens, or at most 256 tokens averaging at most
  // 48 routed rows per expert (above that most experts take two 64-row sub-tiles, each
  // widening the same weights, and the tile kernels are as fast); hidden % 128 == 0 and
  // intermediate % 256 == 0
  const bool swap_rows = s.T <= 64 || (s.T <= 256 && (int64_t)s.T * s.k <= 48 * (int64_t)s.E);
  if (swap_rows && s.H % 128 == 0 && s.I % 256 == 0 && g.row_ready && kUseDecodeKernel) {
    if (g.bits == 4)
      return s.T <= 16   ? launch_w8_decode<4, 16>(s, g, st, why)
             : s.T <= 32 ? launch_w8_decode<4, 32>(s, g, st, why)
                         : launch_w8_decode<4, 64>(s, g, st, why);
    return s.T <= 16   ? launch_w8_decode<8, 16>(s, g, st, why)
           : s.T <= 32 ? launch_w8_decode<8, 32>(s, g, st, why)
                       : launch_w8_decode<8, 64>(s, g, st, why);
  }
  if (g.bits == 4)
    return half_tiles ? launch_swiglu_w8_tiles<64, 4>(s, g, st, why)
                      : launch_swiglu_w8_tiles<128, 4>(s, g, st, why);
  return half_tiles ? launch_swiglu_w8_tiles<64, 8>(s, g, st, why)
                    : launch_swiglu_w8_tiles<128, 8>(s, g, st, why);
}

}  // namespace moe
