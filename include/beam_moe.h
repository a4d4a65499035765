/*
 * beam_moe.h - C ABI of the B200 (sm_100a) Beam Mixture-of-Experts block forward pass.
 *
 * The block (Beam launch post, "Welcome Beam" page, section "Mixture of Experts"; the same text in
 * the flattened Hugging Face post on the reducer.xgoose.org digest page):
 *   - the router scores all E experts with a sigmoid of x . W_r (computed in FP32: same page,
 *     section "Residual Stream", which lists the router among the FP32 computations);
 *   - experts form n_groups contiguous groups; groups are ranked by the sum of their group_topn
 *     (2) best scores and the topk_groups (4) best groups are kept;
 *   - the topk (8) best experts inside the kept groups run; there is no shared expert;
 *   - expert outputs are combined with the router weights normalised to sum 1, then scaled by
 *     routed_scale (2.5; the Chinese digest on the reducer.xgoose.org page: "scale by 2.5");
 *   - every expert is a SwiGLU MLP, E_e(x) = W_down,e (SiLU(W_gate,e x) * (W_up,e x)), with
 *     intermediate size 2,560 at hidden size 5,120 (sections "Mixture of Experts", "Attention").
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, row-major, densely
 *     packed.  bf16 tensors are passed as raw 16-bit patterns (beam_bf16).  The caller owns every
 *     buffer, including the workspace; the library never allocates, frees or synchronises
 *     (beam_moe_device_status is the one call that synchronises).
 *   - Work is enqueued on `stream` (a cudaStream_t, NULL = legacy default stream) and returns
 *     before it completes.  Return codes report argument / launch errors only; errors found by
 *     the kernels (a bad expert id, a wait that timed out) are recorded in a per-device status
 *     word that beam_moe_device_status returns.
 *   - x, y, weights and the workspace must be 16-byte aligned; hidden and inter must be
 *     multiples of 64.  T = 0 is valid and does nothing.
 *   - Readings where the pages are silent: groups are contiguous index ranges; ties go to the
 *     lower group / expert index; slot j of a token holds its j-th best expert (descending
 *     selection value); an optional per-expert selection bias is added to the scores for group
 *     and expert selection only, never to the weights.
 *   - No C++ exception crosses this interface.  Every function is thread-safe.
 */
#ifndef BEAM_MOE_H
#define BEAM_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BEAM_MOE_API __attribute__((visibility("default")))
#else
#define BEAM_MOE_API
#endif

typedef uint16_t beam_bf16; /* raw bfloat16 bit pattern */

/* Layer shape.  Beam: {5120, 2560, 256, 8, 4, 8, 2, 2.5f}. */
typedef struct beam_moe_config {
    int32_t hidden;       /* H: model width, multiple of 64, 64..65536 */
    int32_t inter;        /* I: SwiGLU intermediate size, multiple of 64, 64..65536 */
    int32_t n_experts;    /* E: 1..256 */
    int32_t n_groups;     /* G: 1..32, divides E */
    int32_t topk_groups;  /* groups kept per token, 1..G */
    int32_t topk;         /* k: experts per token, 1..min(16, topk_groups*E/G) */
    int32_t group_topn;   /* scores summed per group for the group ranking, 1..min(8, E/G) */
    float routed_scale;   /* factor on the combined expert output (2.5); not NaN */
} beam_moe_config;

/* Return codes. */
enum {
    BEAM_MOE_OK = 0,
    BEAM_MOE_ERR_INVALID_CONFIG = 1,     /* a config field outside the ranges above */
    BEAM_MOE_ERR_NULL = 2,               /* a required pointer is NULL */
    BEAM_MOE_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
    BEAM_MOE_ERR_WORKSPACE_TOO_SMALL = 4,
    BEAM_MOE_ERR_UNSUPPORTED_DEVICE = 5, /* the current device is not compute capability 10.0 */
    BEAM_MOE_ERR_CUDA = 6,               /* a CUDA runtime / launch error */
    BEAM_MOE_ERR_DEVICE_TIMEOUT = 7,     /* status word: a bounded device-side wait expired */
    BEAM_MOE_ERR_BAD_INDEX = 8,          /* status word: an expert id outside [0, E) */
    BEAM_MOE_ERR_INVALID_ARG = 9         /* T < 0, T > 2^24 or T * k >= 2^31 */
};

/* Workspace kinds for beam_moe_workspace_size. */
enum {
    BEAM_MOE_WS_ROUTE = 0,
    BEAM_MOE_WS_PERMUTE = 1,
    BEAM_MOE_WS_EXPERTS = 2,
    BEAM_MOE_WS_FORWARD = 3,
    BEAM_MOE_WS_BLOCK = 4,
    BEAM_MOE_WS_MXFP8 = 5, /* beam_moe_experts_mxfp8 and beam_moe_forward_mxfp8 */
    BEAM_MOE_WS_W4A4 = 6,  /* beam_moe_experts_w4a4 and beam_moe_forward_w4a4 */
    BEAM_MOE_WS_ROUTE_SCREENED = 7 /* beam_moe_route_screened */
};

/*
 * The residual-stream wrapping of the block ("Welcome Beam" page, section "Residual Stream": every
 * sublayer is normalised before and after; the embedding is step 1 and step k adds the sublayer
 * output with weight 1/sqrt(k) while the stream keeps weight sqrt((k-1)/k); the norms compute in
 * FP32).  Reading: RMSNorm, x / sqrt(mean(x^2) + eps) * weight.  Beam's MoE sublayer of layer l
 * (0-based; layers 3..51 are MoE) is step k = 2l + 3.
 */
typedef struct beam_moe_sublayer {
    const float *pre_norm_weight;   /* [H] fp32, device, 16-byte aligned: scale of the norm before the block */
    const float *post_norm_weight;  /* [H] fp32, device, 16-byte aligned: scale of the norm after the block */
    float eps;                      /* RMSNorm epsilon, >= 0 */
    int32_t step;                   /* k >= 2 */
} beam_moe_sublayer;

/*
 * Bytes of workspace the call `which` needs for T tokens (0 for ROUTE).  Pure host arithmetic:
 * needs no device.  Returns 0 for an invalid config or T < 0.
 */
BEAM_MOE_API size_t beam_moe_workspace_size(const beam_moe_config *cfg, int64_t T, int which);

/*
 * Router: scores, group-limited selection and normalised weights for T tokens ("Mixture of
 * Experts" section: score with a sigmoid, 8 groups, keep 4 by top-2 sum, top 8 inside).
 *   x         [T, H]  bf16   token activations
 *   w_router  [E, H]  fp32   router projection (logit_e = x . w_router[e], accumulated in FP32)
 *   sel_bias  [E]     fp32   selection bias, or NULL for none
 *   topk_ids  [T, k]  int32  out: chosen experts, slot j = j-th best selection value
 *   topk_w    [T, k]  fp32   out: sigmoid score / sum of the chosen scores (sums to 1 per token)
 * A NaN selection value (NaN in x, w_router or sel_bias) ranks below every number: the ids stay
 * valid, distinct and inside the kept groups, and the weights of such a token may be NaN.
 */
BEAM_MOE_API int beam_moe_route(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                   const float *sel_bias, int32_t *topk_ids, float *topk_w, void *stream);

/*
 * beam_moe_route with the projection screened on the tensor cores; the same outputs, bit for bit.
 * W_r is split exactly into three bf16 planes and x . W_r is formed for every expert with tcgen05
 * (exact products, FP32 accumulation); the selection on those values reports its two decision
 * margins (last kept group vs best dropped group, last picked expert vs best one left).  A token
 * whose margins are both at least 2e-4 keeps that set, and its picks' projections are recomputed in
 * beam_moe_route's FP32 order (8 K ranges of sequential fused multiply-adds, summed in range order),
 * then ordered and normalised as there; any other token (a near-tie, NaN or infinite input) is
 * routed from its recomputed projections of every expert.  The screened values are within ~4e-5
 * of the FP32 ones (measured on Beam-shaped inputs), a fifth of the smallest margin that keeps a set.
 * The forward entry points route this way when the configuration fits (E <= 256, k <= 8, G <= 32)
 * and T >= 2048 (below that the direct router is the faster one); otherwise, and for
 * beam_moe_route, the direct FP32 router runs.
 *   Arguments as beam_moe_route, plus a workspace of beam_moe_workspace_size(cfg, T,
 *   BEAM_MOE_WS_ROUTE_SCREENED) bytes (16-byte aligned).  That size is 0 where the direct router runs
 *   (T < 2048 or a configuration outside those bounds); ws may then be NULL.
 */
BEAM_MOE_API int beam_moe_route_screened(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                         const float *w_router, const float *sel_bias, int32_t *topk_ids,
                                         float *topk_w, void *ws, size_t ws_bytes, void *stream);

/*
 * Token -> expert dispatch: stable grouping of the T*k (token, slot) pairs by expert (the pages
 * only say that each token runs on its 8 experts; the order is this library's convention).
 *   topk_ids  [T, k]   int32  in: expert of each (token, slot)
 *   counts    [E]      int32  out: pairs routed to each expert
 *   offsets   [E + 1]  int64  out: exclusive prefix sum of counts; offsets[E] = T*k
 *   row_src   [T * k]  int32  out: row r holds pair q = t*k + j; rows sorted by (expert, token)
 *   dest_row  [T * k]  int32  out: inverse of row_src
 *   ws        workspace of beam_moe_workspace_size(cfg, T, BEAM_MOE_WS_PERMUTE) bytes
 * Ids outside [0, E) set BEAM_MOE_ERR_BAD_INDEX in the status word and leave the outputs
 * undefined.
 */
BEAM_MOE_API int beam_moe_permute(const beam_moe_config *cfg, int64_t T, const int32_t *topk_ids, int32_t *counts,
                     int64_t *offsets, int32_t *row_src, int32_t *dest_row, void *ws, size_t ws_bytes,
                     void *stream);

/*
 * Expert half of the block for callers that route themselves:
 *   y[t] = routed_scale * sum_{j<k} topk_w[t,j] * E_{topk_ids[t,j]}(x[t])   (sum in slot order, FP32)
 *   x       [T, H]     bf16
 *   topk_ids, topk_w   [T, k] int32 / fp32 (ids distinct per token)
 *   w_gate  [E, I, H]  bf16   w_up [E, I, H] bf16   w_down [E, H, I] bf16
 *   y       [T, H]     bf16   out (round to nearest even)
 * The gate/up products are accumulated in FP32 on the tensor cores; SiLU(g)*u is computed in
 * FP32 and stored as bf16 for the down projection, which accumulates in FP32.
 */
BEAM_MOE_API int beam_moe_experts(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                     const float *topk_w, const beam_bf16 *w_gate, const beam_bf16 *w_up,
                     const beam_bf16 *w_down, beam_bf16 *y, void *ws, size_t ws_bytes, void *stream);

/*
 * The whole block: route, dispatch, gate/up + SwiGLU, down projection, weighted combine.
 * topk_ids_out / topk_w_out ([T, k]) receive the routing when non-NULL.
 */
BEAM_MOE_API int beam_moe_forward(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                     const float *sel_bias, const beam_bf16 *w_gate, const beam_bf16 *w_up,
                     const beam_bf16 *w_down, beam_bf16 *y, int32_t *topk_ids_out, float *topk_w_out,
                     void *ws, size_t ws_bytes, void *stream);

/*
 * One MoE sublayer on the residual stream:
 *   u          = bf16(RMSNorm(stream_in) * pre_norm_weight)        (FP32 arithmetic)
 *   y          = the block of beam_moe_forward applied to u       (FP32, not rounded)
 *   stream_out = bf16(sqrt((k-1)/k) * stream_in + RMSNorm(y) * post_norm_weight / sqrt(k))
 *   stream_in, stream_out [T, H] bf16 (may be the same buffer); u_out [T, H] bf16 or NULL (then u
 *   stays in the workspace); routing outputs as for beam_moe_forward.  Needs H <= 32768 and a
 *   workspace of beam_moe_workspace_size(cfg, T, BEAM_MOE_WS_BLOCK) bytes.
 */
BEAM_MOE_API int beam_moe_block_forward(const beam_moe_config *cfg, const beam_moe_sublayer *sub, int64_t T,
                                        const beam_bf16 *stream_in, const float *w_router, const float *sel_bias,
                                        const beam_bf16 *w_gate, const beam_bf16 *w_up, const beam_bf16 *w_down,
                                        beam_bf16 *stream_out, beam_bf16 *u_out, int32_t *topk_ids_out,
                                        float *topk_w_out, void *ws, size_t ws_bytes, void *stream);

/*
 * Dense SwiGLU MLP (Beam's first three layers: "The first 3 layers use a dense SwiGLU MLP",
 * "Welcome Beam" page, section "Mixture of Experts"):
 *   y = W_down (SiLU(W_gate x) * (W_up x))  per token, no routing and no scale
 *   x [T, hidden] bf16; w_gate, w_up [inter, hidden] bf16; w_down [hidden, inter] bf16; y [T, hidden] bf16
 * The same tensor-core engine as the experts (one expert that takes every token).  hidden and inter
 * are multiples of 64; the workspace is beam_moe_dense_workspace_size(hidden, inter, T) bytes.
 */
BEAM_MOE_API size_t beam_moe_dense_workspace_size(int32_t hidden, int32_t inter, int64_t T);
BEAM_MOE_API int beam_moe_dense_swiglu(int32_t hidden, int32_t inter, int64_t T, const beam_bf16 *x,
                                       const beam_bf16 *w_gate, const beam_bf16 *w_up, const beam_bf16 *w_down,
                                       beam_bf16 *y, void *ws, size_t ws_bytes, void *stream);

/*
 * beam_moe_forward that also records caller-created CUDA events (cudaEvent_t) on `stream` around
 * its launches, for per-kernel timing:
 *   events[0] before the router            events[4] after the gate/up + SwiGLU GEMM
 *   events[1] after the router             events[5] after the down GEMM
 *   events[2] after the dispatch kernels   events[6] after the combine
 *   events[3] after the row gather
 * Same results and launches as beam_moe_forward; `events` must hold 7 valid events.
 */
BEAM_MOE_API int beam_moe_forward_profiled(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                           const float *w_router, const float *sel_bias, const beam_bf16 *w_gate,
                                           const beam_bf16 *w_up, const beam_bf16 *w_down, beam_bf16 *y,
                                           int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                                           void *stream, void *const *events);

/*
 * FP8 expert weights.  The "Welcome Beam" page (TL;DR, "Checkpoint formats") lists BF16, FP8 and
 * NVFP4 checkpoints but gives no quantisation recipe.  This library reads FP8 as the OCP MXFP8
 * layout: E4M3 element codes (sign, 4-bit exponent with bias 7, 3-bit mantissa; exponent 0 is
 * subnormal, m * 2^-9; 0x7f / 0xff are NaN) with one UE8M0 scale code c per 32 consecutive K
 * elements of a weight row, the scale being 2^(c - 127) (c = 255 is NaN).  The dequantised weight
 *   W[e][row][k] = e4m3(w[e][row][k]) * 2^(scale[e][k / 32][row] - 127)
 * has at most 4 significant bits, so it is exactly a bf16 value whenever it lies in bf16's normal
 * range; the kernels rebuild those bf16 values in shared memory and run the same tensor-core path
 * as the bf16 weights, so results equal the bf16 entry points given the dequantised weights.
 * Codes that are NaN give undefined results.  Scales are stored K-block-major (all rows of one
 * 32-wide K block together), a layout of this library:
 *   w_gate [E, I, H] u8    w_gate_scale [E, H/32, I] u8
 *   w_up   [E, I, H] u8    w_up_scale   [E, H/32, I] u8
 *   w_down [E, H, I] u8    w_down_scale [E, I/32, H] u8
 * All six pointers are device memory, owned by the caller, 16-byte aligned.
 */
typedef struct beam_moe_fp8_experts {
    const uint8_t *w_gate;
    const uint8_t *w_gate_scale;
    const uint8_t *w_up;
    const uint8_t *w_up_scale;
    const uint8_t *w_down;
    const uint8_t *w_down_scale;
} beam_moe_fp8_experts;

/*
 * beam_moe_experts with FP8 expert weights (beam_moe_fp8_experts).  Same workspace
 * (BEAM_MOE_WS_EXPERTS), outputs and error codes; `w8` NULL -> BEAM_MOE_ERR_NULL.
 */
BEAM_MOE_API int beam_moe_experts_fp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                      const int32_t *topk_ids, const float *topk_w, const beam_moe_fp8_experts *w8,
                                      beam_bf16 *y, void *ws, size_t ws_bytes, void *stream);

/*
 * beam_moe_forward with FP8 expert weights: routing (unchanged: FP32 router weights), dispatch,
 * FP8 experts, combine.  Same workspace (BEAM_MOE_WS_FORWARD), outputs and error codes.
 * `events` is NULL, or 7 events recorded as by beam_moe_forward_profiled.
 */
BEAM_MOE_API int beam_moe_forward_fp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                      const float *w_router, const float *sel_bias, const beam_moe_fp8_experts *w8,
                                      beam_bf16 *y, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                                      size_t ws_bytes, void *stream, void *const *events);

/*
 * NVFP4 expert weights.  The "Welcome Beam" page (TL;DR, "Checkpoint formats"; section "Hardware
 * Requirements": the NVFP4 checkpoint keeps most parameters in 4 bits for Blackwell) gives no
 * quantisation recipe.  This library reads NVFP4 as NVIDIA's layout: E2M1 element codes (sign,
 * 2-bit exponent with bias 1, 1-bit mantissa; exponent 0 is subnormal, m * 0.5; magnitudes 0, 0.5,
 * 1, 1.5, 2, 3, 4, 6), two per byte with element k of a row in the low nibble of byte k/2 when k is
 * even and in the high nibble when k is odd; one E4M3 scale code per 16 consecutive K elements of
 * a weight row (non-negative, finite); one FP32 scale per weight matrix:
 *   W[e][row][k] = e2m1(code(e, row, k)) * e4m3(scale[e][k / 16][row]) * global[e]
 * The kernels rebuild e2m1 * e4m3 * 2^-9, which bf16 holds exactly, run the bf16 tensor-core path,
 * and multiply the FP32 accumulators by global[e] * 2^9.  Scale codes with the sign bit set or NaN
 * give undefined results.
 *   w_gate [E, I, H/2] u8    w_gate_scale [E, H/16, I] u8    w_gate_global [E] f32
 *   w_up   [E, I, H/2] u8    w_up_scale   [E, H/16, I] u8    w_up_global   [E] f32
 *   w_down [E, H, I/2] u8    w_down_scale [E, I/16, H] u8    w_down_global [E] f32
 * All nine pointers are device memory, owned by the caller; the code and scale arrays 16-byte
 * aligned, the scales 4-byte aligned.
 */
typedef struct beam_moe_nvfp4_experts {
    const uint8_t *w_gate;
    const uint8_t *w_gate_scale;
    const float *w_gate_global;
    const uint8_t *w_up;
    const uint8_t *w_up_scale;
    const float *w_up_global;
    const uint8_t *w_down;
    const uint8_t *w_down_scale;
    const float *w_down_global;
} beam_moe_nvfp4_experts;

/* beam_moe_experts with NVFP4 expert weights; same workspace, outputs and error codes. */
BEAM_MOE_API int beam_moe_experts_nvfp4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                        const int32_t *topk_ids, const float *topk_w,
                                        const beam_moe_nvfp4_experts *w4, beam_bf16 *y, void *ws, size_t ws_bytes,
                                        void *stream);

/* beam_moe_forward with NVFP4 expert weights; `events` is NULL or 7 events (as for the FP8 call). */
BEAM_MOE_API int beam_moe_forward_nvfp4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                        const float *w_router, const float *sel_bias,
                                        const beam_moe_nvfp4_experts *w4, beam_bf16 *y, int32_t *topk_ids_out,
                                        float *topk_w_out, void *ws, size_t ws_bytes, void *stream,
                                        void *const *events);

/*
 * Native FP8 path: the same MXFP8 expert weights (beam_moe_fp8_experts) multiplied on the tensor
 * cores with block scaling (tcgen05.mma kind::mxf8f6f4: E4M3 x E4M3, one UE8M0 scale per 32 K
 * elements on each side, FP32 accumulation).  The activations are quantised to MXFP8 as well: x per
 * token and h per dispatch row, in blocks of 32 along the reduction axis, each block scaled by the
 * smallest power of two that brings its largest magnitude to <= 448, elements rounded to the
 * nearest E4M3 value (ties to even).  This is a reading (the pages give no FP8 recipe): results
 * differ from beam_moe_forward_fp8 (bf16 activations) by the activation rounding.  The expert
 * outputs are kept in bf16 between the down projection and the combine (their 2^-9 relative rounding
 * is far below the activations' own).  Requires hidden and inter to be multiples of 128.  Workspace: beam_moe_workspace_size(cfg, T, BEAM_MOE_WS_MXFP8).
 * Other arguments, outputs and error codes as beam_moe_experts_fp8 / beam_moe_forward_fp8
 * (`events`: NULL or 7 events recorded between the stages).
 */
BEAM_MOE_API int beam_moe_experts_mxfp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                        const int32_t *topk_ids, const float *topk_w, const beam_moe_fp8_experts *w8,
                                        beam_bf16 *y, void *ws, size_t ws_bytes, void *stream);
BEAM_MOE_API int beam_moe_forward_mxfp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                        const float *w_router, const float *sel_bias, const beam_moe_fp8_experts *w8,
                                        beam_bf16 *y, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                                        size_t ws_bytes, void *stream, void *const *events);

/*
 * 4-bit path: the NVFP4 expert weights (beam_moe_nvfp4_experts) multiplied on the tensor cores with
 * block scaling (tcgen05.mma kind::mxf4nvf4, block16: E2M1 x E2M1, one E4M3 scale per 16 K elements
 * on each side, FP32 accumulation), the per-matrix FP32 scales applied to the accumulators.  The
 * activations are quantised to NVFP4 as well: x per token with a power-of-two token scale g (the
 * smallest with max|x_t| <= 6 * 448 * g), h per dispatch row with scale 1; in blocks of 16 along the
 * reduction axis, an E4M3 scale nearest to amax / (6 g) and E2M1 elements nearest to v / (s g)
 * (ties to even, saturating at 6).  This is a reading (the pages give no recipe): 4-bit activations
 * change the result by far more than the weights' rounding; beam_moe_forward_nvfp4 keeps bf16
 * activations.  Expert outputs in bf16 between the down projection and the combine, as for the
 * MXFP8 path.  Requires hidden and inter to be multiples of 256.  Workspace:
 * beam_moe_workspace_size(cfg, T, BEAM_MOE_WS_W4A4).  Other arguments, outputs and error codes as
 * beam_moe_experts_nvfp4 / beam_moe_forward_nvfp4.
 */
BEAM_MOE_API int beam_moe_experts_w4a4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                       const int32_t *topk_ids, const float *topk_w, const beam_moe_nvfp4_experts *w4,
                                       beam_bf16 *y, void *ws, size_t ws_bytes, void *stream);
BEAM_MOE_API int beam_moe_forward_w4a4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                       const float *w_router, const float *sel_bias, const beam_moe_nvfp4_experts *w4,
                                       beam_bf16 *y, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                                       size_t ws_bytes, void *stream, void *const *events);

/*
 * Expert parallelism ("Welcome Beam" page, section "Multi-GPU and multi-node": each expert lives on
 * one device while the non-expert parameters are replicated; the device count divides 256).  One
 * rank of an expert-parallel layer over N devices, rank r owning experts [r E/N, (r+1) E/N), runs:
 *   beam_moe_route, beam_moe_permute        on its own tokens, over all E experts;
 *   beam_moe_gather_rows                    its token rows in dispatch order (expert-major), so the
 *                                           rows for rank d are one contiguous block, rows
 *                                           [offsets[d E/N], offsets[(d+1) E/N]);
 *   (caller) all-to-all of those blocks     each rank receives the rows for its experts;
 *   beam_moe_expert_rows                    its local experts on the received rows (FP32 outputs in
 *                                           the received order);
 *   (caller) all-to-all back                the outputs return to the token's rank in dispatch order;
 *   beam_moe_combine                        the weighted sum in slot order, x routed_scale, bf16.
 * With the same inputs the result is bit-identical to beam_moe_forward on one device: each output
 * row sees the same GEMM tiles and K order, and the combine the same FP32 order.
 */

/*
 * x_rows[dest_row[t k + j]] = x[t] for every token t and slot j (dest_row from beam_moe_permute; a
 * negative entry, from an invalid id, writes nothing).  x [T, H], x_rows [T k, H] bf16.
 */
BEAM_MOE_API int beam_moe_gather_rows(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x,
                                      const int32_t *dest_row, beam_bf16 *x_rows, void *stream);

/* Workspace bytes of beam_moe_expert_rows for R rows (0 for an invalid shape or R < 0). */
BEAM_MOE_API size_t beam_moe_expert_rows_workspace_size(int32_t hidden, int32_t inter, int32_t n_experts,
                                                        int64_t R);

/*
 * The SwiGLU experts on rows that each name one expert: o_rows[q] = W_down,e (SiLU(W_gate,e x_q) *
 * (W_up,e x_q)) with e = row_expert[q] in [0, n_experts), in FP32 (SwiGLU product in FP32, h
 * rounded to bf16 as in the forward pass), unweighted and unscaled, in the rows' own order.
 *   x_rows [R, H] bf16; row_expert [R] int32; w_gate, w_up [n_experts, I, H], w_down [n_experts, H, I]
 *   bf16 (the caller's local experts); o_rows [R, H] fp32 out; workspace of
 *   beam_moe_expert_rows_workspace_size bytes.  An id outside [0, n_experts) sets
 *   BEAM_MOE_ERR_BAD_INDEX in the status word and leaves that row of o_rows unwritten.
 */
BEAM_MOE_API int beam_moe_expert_rows(int32_t hidden, int32_t inter, int32_t n_experts, int64_t R,
                                      const beam_bf16 *x_rows, const int32_t *row_expert, const beam_bf16 *w_gate,
                                      const beam_bf16 *w_up, const beam_bf16 *w_down, float *o_rows, void *ws,
                                      size_t ws_bytes, void *stream);

/*
 * y[t] = bf16(routed_scale * sum_{j<k} topk_w[t, j] * o_rows[dest_row[t k + j]]), FP32 fused
 * multiply-adds in slot order from zero, one multiply by routed_scale, round to nearest even.
 *   o_rows [T k, H] fp32 in dispatch order; dest_row [T k]; topk_w [T, k] fp32; y [T, H] bf16.
 */
BEAM_MOE_API int beam_moe_combine(const beam_moe_config *cfg, int64_t T, const float *o_rows,
                                  const int32_t *dest_row, const float *topk_w, beam_bf16 *y, void *stream);

/*
 * beam_moe_permute without a workspace: the same dispatch (identical outputs), with its scratch in
 * a fixed device array inside this library instead of caller memory.  The Beam pages have no
 * counterpart; this exists for callers that cannot allocate device memory when they enqueue work,
 * e.g. a plugin inside an inference server whose host framework owns all device memory, or a
 * latency-critical loop where cudaMalloc is forbidden because it can synchronise the device.
 *   - Limit: ceil(T / 256) * n_experts <= BEAM_MOE_NOALLOC_SCRATCH_INTS (65,536 ints = 256 KiB;
 *     T <= 65,536 tokens at 256 experts); larger calls return BEAM_MOE_ERR_INVALID_ARG and
 *     enqueue nothing.
 *   - The array exists once per device that loads the library and stays allocated until the
 *     process exits.  The first call on a device, with that device current, looks up the array's
 *     device address (cudaGetSymbolAddress); make that first call before any stream capture.  If
 *     the lookup fails the call returns BEAM_MOE_ERR_CUDA and enqueues nothing; only a successful
 *     lookup is kept, so the next call on that device tries again.
 *   - Allocates nothing (no cudaMalloc, cudaFree or allocating library call).  Every call shares
 *     the one array and it keeps the previous call's contents; each call overwrites every entry it
 *     reads, so nothing needs clearing.  Calls whose executions overlap on the GPU (different
 *     streams, or different host threads without ordering) race on the array: order them.
 * Arguments and outputs as for beam_moe_permute.
 */
#define BEAM_MOE_NOALLOC_SCRATCH_INTS 65536
BEAM_MOE_API int beam_moe_permute_noalloc(const beam_moe_config *cfg, int64_t T, const int32_t *topk_ids,
                                          int32_t *counts, int64_t *offsets, int32_t *row_src, int32_t *dest_row,
                                          void *stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status word
 * (BEAM_MOE_OK, BEAM_MOE_ERR_DEVICE_TIMEOUT or BEAM_MOE_ERR_BAD_INDEX), or BEAM_MOE_ERR_CUDA.
 */
BEAM_MOE_API int beam_moe_device_status(void *stream);

/*
 * Test hook for the bounded waits: launches one block that waits on a device barrier nobody
 * signals, giving up after about `timeout_us` microseconds (1..1000000), and records
 * BEAM_MOE_ERR_DEVICE_TIMEOUT in the status word.  No fault, trap or hang is involved.
 */
BEAM_MOE_API int beam_moe_selftest_timeout(int64_t timeout_us, void *stream);

/* Static description of a return code. */
BEAM_MOE_API const char *beam_moe_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_H */
