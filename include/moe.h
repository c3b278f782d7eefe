/*
 * moe.h - C ABI of libmoe.so, the Mixtral sparse-MoE feed-forward layer on one
 * B200 (sm_100a).
 *
 * The layer (nnterp encyclopedia, "Mixtral": "The block, in order"; "The router
 * renormalizes its top 2, in float32"; "Values, by host"; "expert_outputs needs the
 * default experts implementation"):
 *
 *   logits[t,e] = sum_h x[t,h] * w_router[e,h]                 (no bias)
 *   p[t,:]      = softmax(logits[t,:]) in float32
 *   idx[t,0..k) = the k largest, slot 0 the largest; w[t,j] = p[idx[t,j]] / sum_j p
 *   y[t,j]      = w2[e] (silu(w1[e] x[t]) * (w3[e] x[t])),  e = idx[t,j]
 *   out[t]      = residual[t] + sum_j w[t,j] * y[t,j]
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Pointers are DEVICE pointers unless the name ends in _host. The caller owns
 *   every buffer; the library allocates and frees nothing. Every entry point
 *   validates its arguments on the host, then enqueues kernels on `stream` and
 *   returns without synchronising (moe_forward_host excepted).
 * - bf16 tensors are raw IEEE bfloat16 bit patterns (moe_bf16_t), row-major,
 *   contiguous. Weights use nn.Linear [out, in] form stacked over experts:
 *   w_router [E, H]; w1 (gate) and w3 (up) [E, I, H]; w2 (down) [E, H, I]; the
 *   expert weights may instead be in the blocked layout (shape->weight_layout).
 * - Requirements (else MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED): num_tokens >= 1,
 *   1 <= num_experts_per_tok <= num_experts <= 64, num_experts_per_tok <= 8,
 *   hidden_size and intermediate_size positive multiples of 128, every pointer
 *   non-NULL (except those documented as nullable) and 16-byte aligned.
 * - Routed rows are stored expert-contiguous: a stable order on (expert, token,
 *   slot), each expert group padded to a multiple of MOE_ROW_PAD rows. Pad rows
 *   have token -1 and zero activations. moe_max_padded_rows() bounds the total.
 * - `ws` is a device workspace of at least moe_workspace_size() bytes, 256-byte
 *   aligned, whose first 256 bytes (the status word) are zero before first use;
 *   each entry point that takes it uses its own region of it. Kernels
 *   whose waits run out (a bounded spin that never completes) record
 *   MOE_ERR_TIMEOUT in the workspace; moe_device_status() reads and clears it.
 * - On failure the returned code is non-zero and moe_last_error() (thread-local)
 *   describes it. Launch failures return MOE_ERR_CUDA.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t;              /* bfloat16 bit pattern */
typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t; NULL = legacy default stream */

#define MOE_ROW_PAD 128

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_TIMEOUT = 5
} moe_status_t;

/* Layouts of the stacked expert weights w1, w3 [E, I, H] and w2 [E, H, I]:
 * ROW_MAJOR is nn.Linear's [out, in]; BLOCKED stores each [rows, K] matrix (rows =
 * E*I or E*H) as [rows/128][K/64][128][64], so every 128 x 64 tile the kernels read
 * is one contiguous 16 KiB run (moe_pack_weights converts once, at load time). */
#define MOE_WEIGHTS_ROW_MAJOR 0
#define MOE_WEIGHTS_BLOCKED 1

/* The layer's sizes, named as in MixtralConfig (Hugging Face "Mixtral" doc):
 * hidden_size, intermediate_size, num_local_experts (here num_experts) and
 * num_experts_per_tok. num_tokens = batch * sequence length. weight_layout is one of
 * the MOE_WEIGHTS_* values (a zero-initialised shape means row-major).
 * router_bf16_logits: 0 keeps the router logits in fp32; 1 rounds each logit to bf16
 * before scoring, as a bf16 load of the model does (its router's F.linear returns bf16
 * logits that are then cast to float32 for the softmax: nnterp "Mixtral", "The router
 * renormalizes its top 2, in float32"). Equal rounded logits go to the lower expert. */
typedef struct {
  int64_t num_tokens;
  int32_t hidden_size;
  int32_t intermediate_size;
  int32_t num_experts;
  int32_t num_experts_per_tok;
  int32_t weight_layout;
  int32_t router_bf16_logits;
} moe_shape_t;

/* Bytes of device workspace every workspace-taking entry point needs for `shape`;
 * 0 if the shape is invalid. */
size_t moe_workspace_size(const moe_shape_t* shape);

/* Bytes of workspace moe_forward_host needs: moe_workspace_size plus device
 * staging for x, residual and out. 0 if the shape is invalid. */
size_t moe_workspace_size_host(const moe_shape_t* shape);

/* Upper bound on the padded routed-row count R_pad = sum_e pad128(count[e]):
 * round_up(T * k, 128) + 128 * E. Size x_perm, token_of_row and y_perm with it.
 * Returns -1 if the shape is invalid. */
int64_t moe_max_padded_rows(const moe_shape_t* shape);

/* Router and scoring (nnterp "Mixtral", "The router renormalizes its top 2, in
 * float32"): one warp per token computes the E logits x . w_router[e] with fp32
 * accumulation, the float32 softmax over all E, the k largest (ranked on the
 * float32 logit, equal logits to the lower expert index, slot 0 the largest) and
 * their renormalised weights.
 *   x [T, H] bf16; w_router [E, H] bf16;
 *   logit_bias [E] fp32, nullable: added to the logits (not part of Mixtral; lets a
 *     benchmark skew the routing);
 *   topk_idx [T, k] int32 out; topk_w [T, k] fp32 out (each row sums to 1);
 *   router_logits [T, E] fp32 out, nullable (the pre-softmax logits). */
moe_status_t moe_router_topk(const moe_shape_t* shape, const moe_bf16_t* x,
                             const moe_bf16_t* w_router, const float* logit_bias,
                             int32_t* topk_idx, float* topk_w, float* router_logits,
                             moe_stream_t stream);

/* Expert-contiguous permutation (the pages hand expert indices and weights to the
 * experts module, nnterp "Mixtral", "Values, by host"; the order is this library's
 * own): a deterministic per-expert histogram, padded prefix offsets, a stable
 * rank of each (token, slot) and the gather of x rows.
 *   topk_idx [T, k] int32 in, every value in [0, E);
 *   x [T, H] bf16 in;
 *   expert_counts [E] int32 out; expert_offsets [E+1] int32 out (multiples of 128,
 *     offsets[E] = R_pad);
 *   row_of [T, k] int32 out (row of each routed slot);
 *   token_of_row [moe_max_padded_rows] int32 out (token of each row, -1 on pads;
 *     entries past R_pad untouched);
 *   x_perm [moe_max_padded_rows, H] bf16 out (pad rows zero; rows past R_pad
 *     untouched). */
moe_status_t moe_permute(const moe_shape_t* shape, const int32_t* topk_idx,
                         const moe_bf16_t* x, int32_t* expert_counts,
                         int32_t* expert_offsets, int32_t* row_of,
                         int32_t* token_of_row, moe_bf16_t* x_perm, void* ws,
                         size_t ws_bytes, moe_stream_t stream);

/* Allocation-free moe_permute. The paper has no counterpart: this entry point exists
 * for callers that cannot call cudaMalloc, and so cannot supply the workspace that
 * moe_permute takes -- for example a plug-in whose host application owns every
 * device allocation through its own pool, or a serving path that must not allocate
 * once it is running. Arguments, results and checks are those of moe_permute
 * without ws and ws_bytes.
 * Its one piece of scratch, the per-block expert base table (ceil(num_tokens / 32)
 * x num_experts int32, used only when num_tokens > 1024), lives in a 256 KiB static
 * device array inside the library, which every GPU that loads the library holds
 * until the process exits. Shapes needing more than 65536 entries return
 * MOE_ERR_UNSUPPORTED. The first call on each device, made with that device
 * current, looks up the array's device address (cudaGetSymbolAddress) and keeps it
 * for the life of the process; make that first call before any stream capture, and
 * do not call this entry point again on a device after cudaDeviceReset (the kept
 * address would be stale). Every call shares the array: calls whose
 * kernels overlap on the GPU race on it, so the caller must serialise them. A call
 * writes every table entry it reads, so nothing needs clearing between calls. */
moe_status_t moe_permute_static(const moe_shape_t* shape, const int32_t* topk_idx,
                                const moe_bf16_t* x, int32_t* expert_counts,
                                int32_t* expert_offsets, int32_t* row_of,
                                int32_t* token_of_row, moe_bf16_t* x_perm,
                                moe_stream_t stream);

/* The experts (nnterp "Mixtral", "Values, by host": mlp_neurons = act(gate)*up is
 * what the down projection receives; act = silu per MixtralConfig hidden_act):
 * two persistent tcgen05 grouped GEMMs over the ragged expert groups.
 *   GEMM1: h = bf16(silu(x_perm w1[e]^T) * (x_perm w3[e]^T)), fp32 accumulation in
 *          tensor memory, h kept in the workspace;
 *   GEMM2: y_perm = h w2[e]^T, fp32.
 *   x_perm [R_pad, H] bf16 and expert_offsets [E+1] int32 as written by moe_permute;
 *   w1, w3 [E, I, H] bf16; w2 [E, H, I] bf16;
 *   y_perm [moe_max_padded_rows, H] fp32 out for the routed rows (pad rows hold zero
 *     or are left untouched; rows past R_pad untouched). */
moe_status_t moe_grouped_swiglu(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                const int32_t* expert_offsets, const moe_bf16_t* w1,
                                const moe_bf16_t* w3, const moe_bf16_t* w2,
                                float* y_perm, void* ws, size_t ws_bytes,
                                moe_stream_t stream);

/* The two halves of moe_grouped_swiglu, for callers that keep h themselves or time
 * the GEMMs apart. `ws` as for moe_grouped_swiglu (ws_bytes >= moe_workspace_size).
 *   moe_expert_gate_up: h [moe_max_padded_rows, I] bf16 out = bf16(silu(x_perm
 *     w1[e]^T) * (x_perm w3[e]^T)) for the routed rows (pad rows zero or untouched);
 *   moe_expert_down: y_perm [moe_max_padded_rows, H] fp32 out = h w2[e]^T. */
moe_status_t moe_expert_gate_up(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                const int32_t* expert_offsets, const moe_bf16_t* w1,
                                const moe_bf16_t* w3, moe_bf16_t* h, void* ws,
                                size_t ws_bytes, moe_stream_t stream);
moe_status_t moe_expert_down(const moe_shape_t* shape, const moe_bf16_t* h,
                             const int32_t* expert_offsets, const moe_bf16_t* w2,
                             float* y_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Weighted combine into the residual (nnterp "Mixtral": expert_outputs summed over
 * the slot axis is routed_output; the block adds mlp_output to the residual):
 *   out[t] = bf16( residual[t] + sum_j topk_w[t,j] * y_perm[row_of[t,j]] ),
 * fp32 arithmetic, slots in order, a single round-to-nearest-even at the end.
 *   residual [T, H] bf16, nullable (treated as zero); out [T, H] bf16. */
moe_status_t moe_combine(const moe_shape_t* shape, const float* y_perm,
                         const int32_t* row_of, const float* topk_w,
                         const moe_bf16_t* residual, moe_bf16_t* out,
                         moe_stream_t stream);

/* The whole layer: router, permutation, experts and combine, every intermediate in
 * `ws`. residual and logit_bias are nullable. */
moe_status_t moe_forward(const moe_shape_t* shape, const moe_bf16_t* x,
                         const moe_bf16_t* w_router, const float* logit_bias,
                         const moe_bf16_t* w1, const moe_bf16_t* w3,
                         const moe_bf16_t* w2, const moe_bf16_t* residual,
                         moe_bf16_t* out, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* The mixture half of the decoder block (nnterp "Mixtral", "The block, in order":
 * out = h + mlp(post_attention_layernorm(h)); the norm is MixtralRMSNorm with
 * rms_norm_eps, 1e-5 on every checkpoint):
 *   xn[t]  = bf16( (h[t] * r[t]) * norm_weight ),  r[t] = 1 / sqrt(mean(h[t]^2) + eps),
 *   out[t] = bf16( h[t] + sum_j w[t,j] * y[t,j](xn) ).
 * The norm is fused into the router (which computes r, fp32) and the gather (which
 * writes the normed rows); h is also the residual. norm_weight [H] bf16;
 * 0 <= eps <= 1. */
moe_status_t moe_forward_rmsnorm(const moe_shape_t* shape, const moe_bf16_t* h,
                                 const moe_bf16_t* norm_weight, float eps,
                                 const moe_bf16_t* w_router, const float* logit_bias,
                                 const moe_bf16_t* w1, const moe_bf16_t* w3,
                                 const moe_bf16_t* w2, moe_bf16_t* out, void* ws,
                                 size_t ws_bytes, moe_stream_t stream);

/* moe_forward with HOST activations: copies x_host (and residual_host, nullable)
 * into the workspace, runs the layer, copies out back into out_host, and waits for
 * the stream. Host buffers should be pinned for asynchronous copies. Weights and
 * ws stay on the device; ws_bytes >= moe_workspace_size_host(shape). */
moe_status_t moe_forward_host(const moe_shape_t* shape, const moe_bf16_t* x_host,
                              const moe_bf16_t* w_router, const float* logit_bias,
                              const moe_bf16_t* w1, const moe_bf16_t* w3,
                              const moe_bf16_t* w2, const moe_bf16_t* residual_host,
                              moe_bf16_t* out_host, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/* moe_forward_host without the final wait: enqueues the copies in, the layer and the
 * copy out and returns. The copies in run on a copy stream of the library's own, into
 * one of two staging slots of `ws`, so they overlap the previous call's layer; the
 * layer and the copy out run on `stream`, which waits for them. out_host holds the
 * result, and x_host and residual_host may be reused, once the stream has reached this
 * point (for example after cudaStreamSynchronize). Calls on one stream with one ws are
 * ordered by the stream, so a serving loop can enqueue step after step and wait once;
 * the steps may change shape (a workspace sized for the largest serves them all: a
 * call whose shape differs from the previous call's copies in only after that call is
 * done with the workspace, without the overlap). Calls that may overlap on different
 * streams need separate workspaces. Host buffers must be pinned for the copies to be
 * asynchronous. */
moe_status_t moe_forward_host_async(const moe_shape_t* shape, const moe_bf16_t* x_host,
                                    const moe_bf16_t* w_router, const float* logit_bias,
                                    const moe_bf16_t* w1, const moe_bf16_t* w3,
                                    const moe_bf16_t* w2, const moe_bf16_t* residual_host,
                                    moe_bf16_t* out_host, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* Convert row-major expert weights to MOE_WEIGHTS_BLOCKED: w1, w3 [E, I, H] and w2
 * [E, H, I] in, the same-sized w1_blocked, w3_blocked, w2_blocked out (caller-owned,
 * distinct from the inputs). Asynchronous on `stream`. */
moe_status_t moe_pack_weights(const moe_shape_t* shape, const moe_bf16_t* w1,
                              const moe_bf16_t* w3, const moe_bf16_t* w2,
                              moe_bf16_t* w1_blocked, moe_bf16_t* w3_blocked,
                              moe_bf16_t* w2_blocked, moe_stream_t stream);

/* ---- Weight-only int8 experts ----
 * The pages load Mixtral weight-only quantised to shrink it (Hugging Face "Mixtral",
 * "Shrinking down Mixtral using quantization"; ZeroModels "Mixtral", "Lower memory":
 * int8 weights). They do not fix the scheme; this library uses symmetric int8 with
 * one fp32 scale per output row (channel) of each expert matrix:
 *   s[r] = max_c |w[r, c]| / 127   (1 for an all-zero row),
 *   q[r, c] = clamp(rint(w[r, c] / s[r]), -127, 127),   w[r, c] ~ q[r, c] * s[r],
 * the divisions and the rounding (to nearest, ties to even) in float32.
 * Codes are stored offset-binary, u = q + 128 (uint8, 1 .. 255), tiled: a matrix of
 * `rows` rows and K columns (w1 or w3 of all experts: rows = E*I, K = H; w2: rows =
 * E*H, K = I) is cut into 128 x 64 tiles, tile (row / 128, col / 64) being the 8 KiB
 * block number (row / 128) * (K / 64) + col / 64; inside a tile, with r = row % 128
 * and c = col % 64, the code is at byte (c / 16) * 2048 + r * 16 + c % 16.
 * Scales are [rows] fp32, row e*I + i (or e*H + j). The shape's weight_layout field
 * is ignored by these entry points.
 *
 * Precision. The int8 experts compute in IEEE half precision, as a float16 load of
 * the model does (Hugging Face "Mixtral": the model in half precision, float16): the
 * routed rows are converted bf16 -> half (exact for magnitudes in [2^-14, 65504];
 * smaller ones are rounded to half's subnormal grid, larger ones overflow to
 * infinity), each code widens exactly to a half, products accumulate in fp32, and the
 * hidden activation is stored as half:
 *   h = half(silu(s1 * (x_perm q1[e]^T)) * (s3 * (x_perm q3[e]^T))),
 *   y_perm = s2 * (h q2[e]^T)  (fp32).
 * Routing and the combine are the bf16 layer's.
 *
 * moe_quantize_int8: w1, w3 [E, I, H] and w2 [E, H, I] bf16 row-major in (device);
 * q1, q3 [E*I*H], q2 [E*H*I] codes and s1, s3 [E*I], s2 [E*H] fp32 out (device,
 * caller-owned). Asynchronous on `stream`. */
moe_status_t moe_quantize_int8(const moe_shape_t* shape, const moe_bf16_t* w1,
                               const moe_bf16_t* w3, const moe_bf16_t* w2, uint8_t* q1,
                               uint8_t* q3, uint8_t* q2, float* s1, float* s3, float* s2,
                               moe_stream_t stream);

/* moe_grouped_swiglu with int8 expert weights (codes and scales as written by
 * moe_quantize_int8), computed as described above. x_perm is bf16 as moe_permute
 * writes it (converted to half into ws); other arguments and errors as for
 * moe_grouped_swiglu. */
moe_status_t moe_grouped_swiglu_w8(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                   const int32_t* expert_offsets, const uint8_t* q1,
                                   const uint8_t* q3, const uint8_t* q2, const float* s1,
                                   const float* s3, const float* s2, float* y_perm, void* ws,
                                   size_t ws_bytes, moe_stream_t stream);

/* moe_forward with int8 expert weights: router, permutation and combine as in
 * moe_forward (the gather writes the routed rows as half), experts as in
 * moe_grouped_swiglu_w8. */
moe_status_t moe_forward_w8(const moe_shape_t* shape, const moe_bf16_t* x,
                            const moe_bf16_t* w_router, const float* logit_bias,
                            const uint8_t* q1, const uint8_t* q3, const uint8_t* q2,
                            const float* s1, const float* s3, const float* s2,
                            const moe_bf16_t* residual, moe_bf16_t* out, void* ws,
                            size_t ws_bytes, moe_stream_t stream);

/* ---- Weight-only 4-bit experts ----
 * The pages also load Mixtral in 4 bits (Hugging Face "Mixtral", "Shrinking down
 * Mixtral using quantization"; "Welcome Mixtral", "Quantizing Mixtral") and leave the
 * format to the quantisation library. This library uses symmetric 4-bit codes with one
 * IEEE-half scale per group of 64 consecutive columns of a row (one K tile):
 *   s = half(max |w| over the group / 7)   (1 when that is zero in half),
 *   q[r, c] = clamp(rint(w[r, c] / s), -7, 7),
 * the division and the rounding (to nearest, ties to even) in float32; the experts
 * multiply the weight half(q * s), one rounding of the product to half. The format
 * covers groups whose largest |w| is at most 7 * 65504 (beyond it the half scale is
 * infinite and the group's weights are not finite).
 * Codes are stored offset-binary, u = q + 8 (1 .. 15), two to a byte, tiled like the
 * int8 codes: tile (row / 128, col / 64) is the 4 KiB block number (row / 128) * (K /
 * 64) + col / 64; inside it, with r = row % 128 and c = col % 64, the code sits in the
 * 32-bit word at byte (c / 32) * 2048 + r * 16 + ((c % 32) / 8) * 4, nibble n (bits 4n
 * .. 4n+3) with n = (c % 8) / 2 for even c and 4 + (c % 8) / 2 for odd c.
 * Scales are IEEE half bit patterns in the same tile order: the scale of row `row`,
 * group g = col / 64, is element ((row / 128) * (K / 64) + g) * 128 + row % 128.
 * Buffers: q1, q3 [E*I*H/2] and q2 [E*H*I/2] bytes; s1, s3 [E*I*H/64] and s2
 * [E*H*I/64] halves. The shape's weight_layout field is ignored by these entry points.
 *
 * Precision: as the int8 experts (half activations and h, fp32 accumulation), with
 * the scales inside the weight instead of the epilogue:
 *   h = half(silu(x_perm W1q[e]^T) * (x_perm W3q[e]^T)),  y_perm = h W2q[e]^T (fp32),
 * where Wq = half(q * s).
 *
 * moe_quantize_int4: w1, w3 [E, I, H] and w2 [E, H, I] bf16 row-major in (device);
 * codes and scales out (device, caller-owned). Asynchronous on `stream`. */
moe_status_t moe_quantize_int4(const moe_shape_t* shape, const moe_bf16_t* w1,
                               const moe_bf16_t* w3, const moe_bf16_t* w2, uint8_t* q1,
                               uint8_t* q3, uint8_t* q2, uint16_t* s1, uint16_t* s3,
                               uint16_t* s2, moe_stream_t stream);

/* moe_grouped_swiglu with 4-bit expert weights (codes and scales as written by
 * moe_quantize_int4). x_perm is bf16 as moe_permute writes it (converted to half into
 * ws); other arguments and errors as for moe_grouped_swiglu. */
moe_status_t moe_grouped_swiglu_w4(const moe_shape_t* shape, const moe_bf16_t* x_perm,
                                   const int32_t* expert_offsets, const uint8_t* q1,
                                   const uint8_t* q3, const uint8_t* q2, const uint16_t* s1,
                                   const uint16_t* s3, const uint16_t* s2, float* y_perm,
                                   void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_forward with 4-bit expert weights: router, permutation and combine as in
 * moe_forward (the gather writes the routed rows as half), experts as in
 * moe_grouped_swiglu_w4. */
moe_status_t moe_forward_w4(const moe_shape_t* shape, const moe_bf16_t* x,
                            const moe_bf16_t* w_router, const float* logit_bias,
                            const uint8_t* q1, const uint8_t* q3, const uint8_t* q2,
                            const uint16_t* s1, const uint16_t* s3, const uint16_t* s2,
                            const moe_bf16_t* residual, moe_bf16_t* out, void* ws,
                            size_t ws_bytes, moe_stream_t stream);

/* Row gather for the expert-parallel layer (this library's own step; the pages say
 * only that experts may be spread over devices, Hugging Face "Mixtral", MixtralConfig
 * num_local_experts): dst[i, :] = src[index[i], :] for 0 <= i < n_rows. A rank
 * regroups the rows it received from its peers (ordered by source rank, then expert)
 * into expert-contiguous groups with it, and restores the order after the experts.
 *   src [src_rows, row_bytes] and dst [n_rows, row_bytes] device buffers, row_bytes a
 *   positive multiple of 16, 16-byte aligned; index [n_rows] int64 device array. An
 *   index outside [0, src_rows) writes a zero row (so pad rows can be produced and no
 *   read leaves src). n_rows = 0 is a no-op. src and dst must not overlap. */
moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int64_t* index,
                             int64_t n_rows, int64_t row_bytes, void* dst,
                             moe_stream_t stream);

/* ---- expert parallelism over peer memory (this library's own steps; the pages say
 * only that experts may be spread over devices, Hugging Face "Mixtral", MixtralConfig
 * num_local_experts). Rank r's receive buffers are allocated here and shared with the
 * other ranks' processes through CUDA IPC handles; a rank then stores the rows bound
 * for rank r straight into r's expert groups, and reads the experts' outputs back from
 * r's buffer in its combine. Between the steps the caller orders the ranks (a barrier
 * after each rank's stream has finished the previous step): no kernel here waits on
 * another rank. */

/* Bytes of an IPC handle (a cudaIpcMemHandle_t). */
#define MOE_IPC_HANDLE_BYTES 64

/* Allocates `bytes` (> 0) of device memory on the current device that other processes
 * may map (cudaMalloc; 256-byte aligned) and writes its handle, MOE_IPC_HANDLE_BYTES
 * bytes, to `handle` (host memory). *dev_ptr receives the buffer (NULL on failure). The
 * caller owns it: moe_ipc_free. */
moe_status_t moe_ipc_alloc(size_t bytes, void** dev_ptr, void* handle);

/* Maps a buffer that moe_ipc_alloc made in another process (on this GPU or a peer that
 * this device can access) and writes its address in this process to *dev_ptr. Opening
 * a handle in the process that made it fails (MOE_ERR_CUDA). Unmap with moe_ipc_close
 * before the owner frees it. */
moe_status_t moe_ipc_open(const void* handle, void** dev_ptr);

/* Unmaps a buffer that moe_ipc_open mapped (NULL: no-op). */
moe_status_t moe_ipc_close(void* dev_ptr);

/* Frees a buffer that moe_ipc_alloc made (NULL: no-op); every other process must have
 * unmapped it first. */
moe_status_t moe_ipc_free(void* dev_ptr);

/* Row scatter into several ranks' buffers: for 0 <= i < n_rows, row dst_row[i] of the
 * buffer dst_bases[dst_rank[i]] = row src_index[i] of src. Rows are row_bytes bytes (a
 * positive multiple of 16). src [src_rows] rows, 16-byte aligned, on this device;
 * src_index [n_rows] int64, dst_rank [n_rows] int32, dst_row [n_rows] int64 device
 * arrays; dst_bases a device array of `world` device pointers (16-byte aligned; this
 * device's buffers or peers' mappings from moe_ipc_open), each buffer dst_rows rows. A
 * row whose source index, rank or destination row is out of range is skipped and
 * counted into *bad_rows (a device int32, may be NULL). The stores are plain stores:
 * they are visible to the owner once this launch has finished on `stream`. */
moe_status_t moe_scatter_rows_peer(const void* src, int64_t src_rows, const int64_t* src_index,
                                   const int32_t* dst_rank, const int64_t* dst_row,
                                   int64_t n_rows, void* const* dst_bases, int world,
                                   int64_t dst_rows, int64_t row_bytes, int32_t* bad_rows,
                                   moe_stream_t stream);

/* Combine reading the experts' outputs from several ranks' buffers, with moe_combine's
 * arithmetic (nnterp "Mixtral": slot outputs scaled by their float32 weights, summed,
 * added to the residual; fp32 in slot order, one rounding to bf16):
 *   out[t, :] = bf16(residual[t, :] + sum_j topk_w[t, j] * y_j)
 * with y_j = row slot_row[t k + j] of the fp32 buffer y_bases[slot_rank[t k + j]].
 *   y_bases: device array of `world` device pointers, each buffer [y_rows, hidden] fp32
 *   (16-byte aligned); slot_rank [T k] int32 and slot_row [T k] int64 device arrays;
 *   topk_w [T, k] fp32; residual [T, hidden] bf16 or NULL; out [T, hidden] bf16.
 *   1 <= k <= 8, hidden a positive multiple of 8. A slot whose rank or row is out of
 *   range adds nothing and is counted into *bad_slots (device int32, may be NULL).
 *   num_tokens = 0 is a no-op. */
moe_status_t moe_combine_peer(const float* const* y_bases, int world, int64_t y_rows,
                              const int32_t* slot_rank, const int64_t* slot_row,
                              const float* topk_w, const moe_bf16_t* residual, moe_bf16_t* out,
                              int64_t num_tokens, int k, int hidden, int32_t* bad_slots,
                              moe_stream_t stream);

/* Waits for `stream`, then reads and clears the device status word in `ws`:
 * MOE_OK, or MOE_ERR_TIMEOUT if a kernel gave up a bounded wait since the last
 * call. */
moe_status_t moe_device_status(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Diagnostic of the failure path: launches one thread that waits, with the same
 * bounded wait the GEMM kernels use, on a barrier phase that nothing completes. After
 * timeout_ns (0 < timeout_ns <= 10 s) the wait gives up and records MOE_ERR_TIMEOUT
 * in the status word of `ws` (ws_bytes >= 256), which moe_device_status() then
 * reports; the context stays usable. Returns after the launch. */
moe_status_t moe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns,
                                       moe_stream_t stream);

/* Thread-local description of the last failure on this thread ("" if none). */
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
