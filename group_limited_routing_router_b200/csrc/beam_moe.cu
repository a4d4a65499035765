// C ABI of the Beam MoE block forward pass on B200 (sm_100a): argument checks, workspace layout,
// TMA descriptor encoding and the launch sequence
//   router_topk -> permute_hist -> permute_scan -> permute_scatter -> [gather_rows, wide tiles]
//   -> grouped GEMM (gate/up + SwiGLU) -> grouped GEMM (down) -> combine
// all enqueued on the caller's stream with no host synchronisation.  The public contract is in
// include/beam_moe.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/beam_moe.h"

#include "common.cuh"
#include "combine.cuh"
#include "permute.cuh"
#include "gemm.cuh"
#include "gemm_2sm.cuh"
#include "gemm_fp8.cuh"
#include "gemm_mx8.cuh"
#include "norm.cuh"
#include "router.cuh"
#include "router_tc.cuh"

namespace beam {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxBlockHidden = 32768;  // the block's FP32 output row stays in shared memory
constexpr int64_t kMaxTokens = int64_t(1) << 24;

// ---- GEMM variants: <gate/up?, BN, B box rows, smem stages, TMEM slots, slot columns, gather?,
// weight-row pairs?> -----
// "wide": experts see up to ~190 tokens per tile (prefill): the dispatch also gathers x into
// dispatch order (x_perm) and both GEMMs read their token rows with tiled TMA boxes (64 rows on
// single CTAs, 32 rows on CTA pairs).
// "narrow": a few tokens per expert (decode): the gate/up GEMM gathers its rows straight from x
// with TMA gather4 (four rows per instruction; cheap when an expert has a handful of tokens).
// "pair": the down projection with two 128-row weight tiles per token tile (half the token-row bytes
// per weight byte), for the dense MLP on single CTAs: its K = 20480 makes items long, and 440 of them
// would leave a 10% wave tail on 74 CTA pairs (its gate/up runs on CTA pairs, G1_2SM_BIG).
#define G2_PAIR_ARGS false, 192, 64, 4, 2, 256, false, true
// CTA-pair variants (cta_group::2) for the MoE bf16 wide case (prefill, skew, long; the expert-rows
// entry point): <gate/up?, BN, B box rows, smem stages, TMEM slots, slot columns>; each CTA stages half
// of the token tile in 32-row boxes.  Against the single-CTA kernels (same process, alternating calls):
// prefill 4.19 vs 4.22 ms per layer, skew 12.99 vs 13.67, long 49.4 vs 54.3.
#define G1_2SM_ARGS true, 192, 32, 5, 2, 256
#define G2_2SM_ARGS false, 192, 32, 8, 2, 256
// 256-token tiles where experts span several token tiles (skew, long: tensor-bound): a third more
// products per staged byte; the down projection still keeps one TMEM slot per item.
#define G1_2SM_BIG_ARGS true, 256, 32, 4, 2, 256
#define G2_2SM_BIG_ARGS false, 256, 32, 7, 2, 256
constexpr int k2smBox = 32;
#define G1_NARROW_ARGS true, 32, 1, 6, 4, 64, true, false
#define G2_NARROW_ARGS false, 32, 32, 10, 4, 32, false, false
// FP8 variants: <gate/up?, BN, B box rows, weight stages (K = 128), B stages (K = 64), TMEM slots,
// slot columns, gather?, bf16 A ring stages in TMEM>.  The A ring takes the TMEM columns the
// accumulators leave; the prefill gate/up variant gives its accumulators 2 slots of 192 columns
// (one item of more than 96 tokens at a time) so that two A ring stages fit.
#define G1_WIDE_FP8_ARGS true, 192, 64, 3, 4, 2, 192, false, 2, false
#define G2_WIDE_FP8_ARGS false, 192, 64, 4, 5, 2, 192, false, 4, false
#define G1_NARROW_FP8_ARGS true, 32, 1, 5, 12, 2, 64, true, 6, false
#define G2_NARROW_FP8_ARGS false, 32, 32, 9, 16, 4, 32, false, 12, false
// NVFP4 variants (last argument true): the same rings; a weight stage spans K = 256 (128 bytes of
// E2M1 pairs per row) and its scale tiles are 8x larger, so they keep one stage fewer.
#define G1_WIDE_NV4_ARGS true, 192, 64, 3, 4, 2, 192, false, 2, true
#define G2_WIDE_NV4_ARGS false, 192, 64, 4, 5, 2, 192, false, 4, true
#define G1_NARROW_NV4_ARGS true, 32, 1, 4, 12, 2, 64, true, 6, true
#define G2_NARROW_NV4_ARGS false, 32, 32, 8, 16, 4, 32, false, 12, true
// Block-scaled FP8 variants (tcgen05 kind::mxf8f6f4): <gate/up?, BN, B box rows, stages (K = 128),
// TMEM slots, slot columns, gather?>; each stage also holds its scale atoms and TMEM scale columns.
#define G1_WIDE_MX8_ARGS true, 192, 64, 3, 2, 192, false, false
// 160-token gate/up tiles with a fourth stage, for batches whose experts mostly fit one such tile
// (prefill); TMEM: 2 x 160 accumulator columns + 4 x 16 scale columns.
#define G1_WIDE_MX8_160_ARGS true, 160, 32, 4, 2, 160, false, false
#define G2_WIDE_MX8_ARGS false, 192, 64, 5, 2, 192, false, false
#define G1_NARROW_MX8_ARGS true, 32, 1, 5, 4, 64, true, false
#define G2_NARROW_MX8_ARGS false, 32, 32, 10, 4, 32, false, false
// The 4-bit path (kind::mxf4nvf4): four scale-atom sets per stage, so fewer stages and a wide token
// tile of 128 (one B atom per set).  The "160" variants hold 160 tokens (two B atoms per set; TMEM:
// 2 x 160 accumulator columns + 3 (gate/up) or 4 (down) stages x 64 / 48 scale columns) for batches
// whose experts mostly fit one such tile (prefill: ~128 +- 11 tokens per expert), so that an expert
// does not spill a handful of tokens into a second tile that re-streams its weights: prefill
// 2.76 -> 2.30 ms per layer; with many tokens per expert (skew) the 128 tiles are faster.
#define G1_WIDE_NV4X_ARGS true, 128, 64, 3, 2, 128, false, true
#define G2_WIDE_NV4X_ARGS false, 128, 64, 5, 2, 128, false, true
#define G1_WIDE_NV4X_160_ARGS true, 160, 32, 3, 2, 160, false, true
#define G2_WIDE_NV4X_160_ARGS false, 160, 32, 4, 2, 160, false, true
#define G1_NARROW_NV4X_ARGS true, 32, 1, 4, 4, 64, true, true
#define G2_NARROW_NV4X_ARGS false, 32, 32, 8, 4, 32, false, true
constexpr int kWideBN = 192, kWideBox = 64, kNarrowBN = 32, kNarrowBox = 32;
constexpr int kNv4BigBN = 160, kNv4BigBox = 32;  // the 4-bit "160" variants

template <bool G, int BN, int BOXN, int ST, int NS, int SC, bool GA, bool PR>
bool set_gemm_smem() {
    return cudaFuncSetAttribute(grouped_gemm_kernel<G, BN, BOXN, ST, NS, SC, GA, PR>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                GemmCfg<G, BN, BOXN, ST, NS, SC, GA, PR>::kSmem) == cudaSuccess;
}
template <bool G, int BN, int BOXN, int W8, int BS, int NS, int SC, bool GA, int AS, bool F4>
bool set_gemm_fp8_smem() {
    return cudaFuncSetAttribute(grouped_gemm_fp8_kernel<G, BN, BOXN, W8, BS, NS, SC, GA, AS, F4>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Fp8GemmCfg<G, BN, BOXN, W8, BS, NS, SC, GA, AS, F4>::kSmem) == cudaSuccess;
}

template <bool G, int BN, int BOXN, int ST, int NS, int SC, bool GA, bool F4>
bool set_gemm_mx8_smem() {
    return cudaFuncSetAttribute(grouped_gemm_mx8_kernel<G, BN, BOXN, ST, NS, SC, GA, F4>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Mx8GemmCfg<G, BN, BOXN, ST, NS, SC, GA, F4>::kSmem) == cudaSuccess;
}
template <bool G, int BN, int BOXN, int ST, int NS, int SC, bool GA, bool F4>
void launch_gemm_mx8(int grid, cudaStream_t s, const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &s0,
                     const CUtensorMap &s1, const CUtensorMap &b, const Mx8Params &p) {
    grouped_gemm_mx8_kernel<G, BN, BOXN, ST, NS, SC, GA, F4>
        <<<grid, kMxThreads, Mx8GemmCfg<G, BN, BOXN, ST, NS, SC, GA, F4>::kSmem, s>>>(a0, a1, s0, s1, b, p);
}

// a1 is ignored by the down projection.
template <bool G, int BN, int BOXN, int ST, int NS, int SC, bool GA, bool PR>
void launch_gemm(int grid, cudaStream_t s, const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                 const GemmParams &p) {
    grouped_gemm_kernel<G, BN, BOXN, ST, NS, SC, GA, PR>
        <<<grid, kGemmThreads, GemmCfg<G, BN, BOXN, ST, NS, SC, GA, PR>::kSmem, s>>>(a0, a1, b, p);
}
template <bool G, int BN, int BOXN, int ST, int NS, int SC>
bool set_gemm2_smem() {
    return cudaFuncSetAttribute(grouped_gemm_2sm_kernel<G, BN, BOXN, ST, NS, SC>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Gemm2Cfg<G, BN, BOXN, ST, NS, SC>::kSmem) == cudaSuccess;
}
// CTA pairs of the pair GEMM that fit on the device at once (at most one CTA per SM); 0 on failure.
template <bool G, int BN, int BOXN, int ST, int NS, int SC>
int gemm2_pairs(int sms) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(static_cast<unsigned>(2 * (sms / 2)), 1, 1);
    lc.blockDim = dim3(kGemmThreads, 1, 1);
    lc.dynamicSmemBytes = Gemm2Cfg<G, BN, BOXN, ST, NS, SC>::kSmem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_2sm_kernel<G, BN, BOXN, ST, NS, SC>, &lc) != cudaSuccess)
        return 0;
    return std::min(n, sms / 2);
}
// a1 is ignored by the down projection; `pairs` clusters of 2 CTAs.
template <bool G, int BN, int BOXN, int ST, int NS, int SC>
void launch_gemm2(int pairs, cudaStream_t s, const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                  const GemmParams &p) {
    grouped_gemm_2sm_kernel<G, BN, BOXN, ST, NS, SC>
        <<<2 * pairs, kGemmThreads, Gemm2Cfg<G, BN, BOXN, ST, NS, SC>::kSmem, s>>>(a0, a1, b, p);
}
// a1 and s1 are ignored by the down projection.
template <bool G, int BN, int BOXN, int W8, int BS, int NS, int SC, bool GA, int AS, bool F4>
void launch_gemm_fp8(int grid, cudaStream_t s, const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &s0,
                     const CUtensorMap &s1, const CUtensorMap &b, const GemmParams &p, const AccScales &acc) {
    using C = Fp8GemmCfg<G, BN, BOXN, W8, BS, NS, SC, GA, AS, F4>;
    grouped_gemm_fp8_kernel<G, BN, BOXN, W8, BS, NS, SC, GA, AS, F4>
        <<<grid, C::kThreads, C::kSmem, s>>>(a0, a1, s0, s1, b, p, acc);
}

// Tile family from the mean rows per expert (T*k/E): narrow when experts see a handful of tokens.
bool narrow_tiles(const beam_moe_config *c, int64_t T) {
    return static_cast<double>(T) * c->topk / c->n_experts <= 12.0;
}

struct DeviceInfo {
    std::once_flag once;
    int status = BEAM_MOE_OK;
    int num_sms = 0;
    int clock_khz = 0;
    int pairs_g1 = 0, pairs_g2 = 0, pairs_g1b = 0, pairs_g2b = 0;  // co-resident CTA pairs (persistent grids)
};
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

template <int BN>
bool set_router_tc_smem() {
    return cudaFuncSetAttribute(router_logits_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                RsCfg<BN>::kSmem) == cudaSuccess;
}

int init_device(int *dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BEAM_MOE_ERR_UNSUPPORTED_DEVICE;
    DeviceInfo &d = g_dev[dev];
    std::call_once(d.once, [&]() {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.clock_khz, cudaDevAttrClockRate, dev) != cudaSuccess) {
            d.status = BEAM_MOE_ERR_CUDA;
            return;
        }
        if (major != 10 || minor != 0) {
            d.status = BEAM_MOE_ERR_UNSUPPORTED_DEVICE;
            return;
        }
        bool ok = cudaFuncSetAttribute(router_topk_kernel<kRtTok>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       rt_smem_bytes(kRtTok)) == cudaSuccess &&
                  cudaFuncSetAttribute(router_topk_kernel<kRtTokSmall>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       rt_smem_bytes(kRtTokSmall)) == cudaSuccess &&
                  cudaFuncSetAttribute(router_topk_kernel<kRtTokTiny>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       rt_smem_bytes(kRtTokTiny)) == cudaSuccess;
        ok = ok && set_gemm_smem<G2_PAIR_ARGS>() &&
             set_gemm_smem<G1_NARROW_ARGS>() && set_gemm_smem<G2_NARROW_ARGS>();
        ok = ok && set_gemm_fp8_smem<G1_WIDE_FP8_ARGS>() && set_gemm_fp8_smem<G2_WIDE_FP8_ARGS>() &&
             set_gemm_fp8_smem<G1_NARROW_FP8_ARGS>() && set_gemm_fp8_smem<G2_NARROW_FP8_ARGS>();
        ok = ok && set_gemm_fp8_smem<G1_WIDE_NV4_ARGS>() && set_gemm_fp8_smem<G2_WIDE_NV4_ARGS>() &&
             set_gemm_fp8_smem<G1_NARROW_NV4_ARGS>() && set_gemm_fp8_smem<G2_NARROW_NV4_ARGS>();
        ok = ok && set_gemm_mx8_smem<G1_WIDE_MX8_ARGS>() && set_gemm_mx8_smem<G2_WIDE_MX8_ARGS>() &&
             set_gemm_mx8_smem<G1_WIDE_MX8_160_ARGS>() &&
             set_gemm_mx8_smem<G1_NARROW_MX8_ARGS>() && set_gemm_mx8_smem<G2_NARROW_MX8_ARGS>();
        ok = ok && set_gemm_mx8_smem<G1_WIDE_NV4X_ARGS>() && set_gemm_mx8_smem<G2_WIDE_NV4X_ARGS>() &&
             set_gemm_mx8_smem<G1_WIDE_NV4X_160_ARGS>() && set_gemm_mx8_smem<G2_WIDE_NV4X_160_ARGS>() &&
             set_gemm_mx8_smem<G1_NARROW_NV4X_ARGS>() && set_gemm_mx8_smem<G2_NARROW_NV4X_ARGS>();
        ok = ok && cudaFuncSetAttribute(combine_norm_residual_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kMaxBlockHidden * 4) == cudaSuccess;
        ok = ok && set_router_tc_smem<32>() && set_router_tc_smem<64>() && set_router_tc_smem<128>();
        ok = ok && cudaFuncSetAttribute(router_exact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kRsPathSmem) == cudaSuccess;
        ok = ok && set_gemm2_smem<G1_2SM_ARGS>() && set_gemm2_smem<G2_2SM_ARGS>() &&
             set_gemm2_smem<G1_2SM_BIG_ARGS>() && set_gemm2_smem<G2_2SM_BIG_ARGS>();
        if (ok) {
            d.pairs_g1 = gemm2_pairs<G1_2SM_ARGS>(d.num_sms);
            d.pairs_g2 = gemm2_pairs<G2_2SM_ARGS>(d.num_sms);
            d.pairs_g1b = gemm2_pairs<G1_2SM_BIG_ARGS>(d.num_sms);
            d.pairs_g2b = gemm2_pairs<G2_2SM_BIG_ARGS>(d.num_sms);
            ok = d.pairs_g1 > 0 && d.pairs_g2 > 0 && d.pairs_g1b > 0 && d.pairs_g2b > 0;
        }
        if (!ok) d.status = BEAM_MOE_ERR_CUDA;
    });
    *dev_out = dev;
    return d.status;
}

EncodeTiledFn encode_fn() {
    std::call_once(g_encode_once, []() {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int validate(const beam_moe_config *c) {
    if (!c) return BEAM_MOE_ERR_NULL;
    if (c->hidden < 64 || c->hidden > 65536 || c->hidden % 64 || c->inter < 64 || c->inter > 65536 ||
        c->inter % 64)
        return BEAM_MOE_ERR_INVALID_CONFIG;
    if (c->n_experts < 1 || c->n_experts > 256 || c->n_groups < 1 || c->n_groups > 32 ||
        c->n_experts % c->n_groups)
        return BEAM_MOE_ERR_INVALID_CONFIG;
    const int per = c->n_experts / c->n_groups;
    if (c->topk_groups < 1 || c->topk_groups > c->n_groups) return BEAM_MOE_ERR_INVALID_CONFIG;
    if (c->topk < 1 || c->topk > 16 || c->topk > c->topk_groups * per) return BEAM_MOE_ERR_INVALID_CONFIG;
    if (c->group_topn < 1 || c->group_topn > 8 || c->group_topn > per) return BEAM_MOE_ERR_INVALID_CONFIG;
    if (!(c->routed_scale == c->routed_scale)) return BEAM_MOE_ERR_INVALID_CONFIG;  // NaN
    return BEAM_MOE_OK;
}

int check_T(const beam_moe_config *c, int64_t T) {
    if (T < 0 || T > kMaxTokens || T * c->topk >= (int64_t(1) << 31)) return BEAM_MOE_ERR_INVALID_ARG;
    return BEAM_MOE_OK;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Screened router (router_tc.cuh) scratch: the three bf16 planes of W_r, the split partial projections,
// the exact-path token list and its projections.  Pure host arithmetic: the split count aims at two
// items per SM of a 148-SM B200 whatever device runs it, so the workspace size is device independent.
struct RoutePlan {
    bool ok = false;  // false: the configuration takes the direct router
    int bn = 0, S = 0, kps = 0, n_nt = 0, n_mt = 0;
    size_t planes = 0, part = 0, list = 0, counters = 0, exact = 0, bucket = 0, xlogit = 0, listed = 0, total = 0;
};

RoutePlan route_plan(const beam_moe_config *c, int64_t T) {
    RoutePlan P;
    // below ~2k tokens the direct router is faster: the screen's exact recomputation streams 8 rows of
    // W_r per token either way, and the direct router's tiles already fill the GPU
    if (T < kRsMinTokens || c->n_experts > kRtSlots || c->topk > 8 || c->n_groups > 32 || c->hidden % kBK) return P;
    P.ok = true;
    P.bn = T >= 2048 ? 128 : (T >= 512 ? 64 : 32);
    P.n_nt = static_cast<int>((T + P.bn - 1) / P.bn);
    P.n_mt = (c->n_experts + kBM - 1) / kBM;
    const int nk = c->hidden / kBK;
    P.S = 1;
    for (int d = 1; d <= std::min(kRsMaxSplit, nk); ++d) {
        if (nk % d) continue;
        P.S = d;
        if (static_cast<int64_t>(P.n_nt) * P.n_mt * d >= 2 * 148) break;
    }
    P.kps = nk / P.S;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    const size_t E = c->n_experts, H = c->hidden;
    P.planes = take(3 * E * H * 2);
    P.part = take(static_cast<size_t>(P.S) * T * E * 4);
    P.list = take(static_cast<size_t>(T) * 4);
    P.counters = take((1 + E) * 4);  // the list's length, then the picks per expert (zeroed per call)
    P.exact = take(static_cast<size_t>(T) * E * 4);
    P.bucket = take(static_cast<size_t>(T) * E * 4);
    P.xlogit = take(static_cast<size_t>(T) * c->topk * 4);
    P.listed = take(static_cast<size_t>(T));
    P.total = off;
    return P;
}

struct Layout {
    size_t u = 0, ids = 0, w = 0, rt = 0, hist = 0, counts = 0, offsets = 0, row_src = 0, dest_row = 0, xp = 0, h = 0,
           o = 0;
    size_t total = 0;
};

int64_t n_chunks(int64_t T) { return (T + kPmTok - 1) / kPmTok; }

Layout layout(const beam_moe_config *c, int64_t T, int which) {
    Layout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    const size_t R = static_cast<size_t>(T) * c->topk;
    const size_t E = c->n_experts, H = c->hidden, I = c->inter;
    if (which == BEAM_MOE_WS_ROUTE || T == 0) return L;
    if (which == BEAM_MOE_WS_BLOCK) L.u = take(static_cast<size_t>(T) * H * 2);
    if (which == BEAM_MOE_WS_FORWARD || which == BEAM_MOE_WS_BLOCK) {
        L.ids = take(R * 4);
        L.w = take(R * 4);
        L.rt = take(route_plan(c, T).total);
    }
    L.hist = take(static_cast<size_t>(n_chunks(T)) * E * 4);
    if (which == BEAM_MOE_WS_PERMUTE) {
        L.total = off;
        return L;
    }
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 8);
    L.row_src = take(R * 4);
    L.dest_row = take(R * 4);
    if (!narrow_tiles(c, T)) L.xp = take(R * H * 2);  // x in dispatch order (wide tiles only)
    L.h = take(R * I * 2);
    L.o = take(R * H * 4);
    L.total = off;
    return L;
}

// 2D [rows][K] bf16 tensor, box {64, box_rows}, 128-byte swizzle.
bool make_map_2d(CUtensorMap *m, const void *base, uint64_t K, uint64_t rows, uint32_t box_rows) {
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D [E][M][K] bf16 weights, box {64, 128, 1}, 128-byte swizzle.
bool make_map_3d(CUtensorMap *m, const void *base, uint64_t K, uint64_t M, uint64_t E) {
    const cuuint64_t dims[3] = {K, M, E};
    const cuuint64_t strides[2] = {K * 2, K * M * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(kBM), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D [E][M][K] E4M3 weights, box {128, 128, 1}: 128-byte rows (K = 128), 128-byte swizzle.
bool make_map_3d_fp8(CUtensorMap *m, const void *base, uint64_t K, uint64_t M, uint64_t E) {
    const cuuint64_t dims[3] = {K, M, E};
    const cuuint64_t strides[2] = {K, K * M};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(2 * kBK), static_cast<cuuint32_t>(kBM), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D [E][M][K/2] E2M1 code pairs, box {128 bytes, 128, 1}: K = 256 per box, 128-byte swizzle.
bool make_map_3d_fp4(CUtensorMap *m, const void *base, uint64_t K, uint64_t M, uint64_t E) {
    return make_map_3d_fp8(m, base, K / 2, M, E);
}

// 3D [E][K/blk][M] scale codes, box {128, kb_per_stage, 1}: the K blocks of one weight stage
// (MXFP8: 4 blocks of 32 in K = 128; NVFP4: 16 blocks of 16 in K = 256).
bool make_map_scale(CUtensorMap *m, const void *base, uint64_t M, uint64_t KB, uint64_t E,
                    uint32_t kb_per_stage = 4) {
    const cuuint64_t dims[3] = {M, KB, E};
    const cuuint64_t strides[2] = {M, M * KB};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kBM), kb_per_stage, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? BEAM_MOE_OK : BEAM_MOE_ERR_CUDA; }

// Generic 2-D tensor map: [rows][inner] elements of `esize` bytes, box {box_inner, box_rows}.
bool make_map_2d_any(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t inner,
                     uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw) {
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * esize};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return encode_fn()(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int enqueue_route(const beam_moe_config *c, int64_t T, const beam_bf16 *x, const float *w_router, const float *bias,
                  int32_t *ids, float *w, cudaStream_t s) {
    RouterParams p;
    p.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    p.w = w_router;
    p.bias = bias;
    p.ids = ids;
    p.wts = w;
    p.T = T;
    p.H = c->hidden;
    p.E = c->n_experts;
    p.G = c->n_groups;
    p.topk_groups = c->topk_groups;
    p.topk = c->topk;
    p.group_topn = c->group_topn;
    // W_r tiles: 32 fp32 (one 128-byte swizzled row) x all 256 expert slots (rows >= E read as 0);
    // x tiles: 32 bf16 (64-byte swizzled row) x 64 tokens, or 16 for batches of at most 1024 tokens,
    // so that they still spread over most of the SMs (rows >= T read as 0)
    const int tok = T <= 512 ? kRtTokTiny : (T <= 1024 ? kRtTokSmall : kRtTok);
    CUtensorMap m_w, m_x;
    if (!encode_fn()) return BEAM_MOE_ERR_CUDA;
    if (!make_map_2d_any(&m_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, w_router, c->hidden, c->n_experts, kRtBK, kRtSlots,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d_any(&m_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, c->hidden, T, kRtBK, tok,
                         CU_TENSOR_MAP_SWIZZLE_64B))
        return BEAM_MOE_ERR_CUDA;
    const int64_t tiles = (T + tok - 1) / tok;
    if (tok == kRtTok)
        router_topk_kernel<kRtTok><<<static_cast<unsigned>(tiles * kRtCluster), kRtThreads, rt_smem_bytes(kRtTok), s>>>(
            m_w, m_x, p);
    else if (tok == kRtTokSmall)
        router_topk_kernel<kRtTokSmall><<<static_cast<unsigned>(tiles * kRtCluster), kRtThreads,
                                          rt_smem_bytes(kRtTokSmall), s>>>(m_w, m_x, p);
    else
        router_topk_kernel<kRtTokTiny><<<static_cast<unsigned>(tiles * kRtCluster), kRtThreads,
                                         rt_smem_bytes(kRtTokTiny), s>>>(m_w, m_x, p);
    return launch_status();
}

// The routing of enqueue_route (bit for bit) through the screened router when the configuration fits
// it and the caller's workspace holds its scratch (route_plan); the direct router otherwise.
int enqueue_route_ws(const beam_moe_config *c, int dev, int64_t T, const beam_bf16 *x, const float *w_router,
                     const float *bias, int32_t *ids, float *w, uint8_t *scratch, cudaStream_t s) {
    const RoutePlan P = route_plan(c, T);
    if (!P.ok || !scratch) return enqueue_route(c, T, x, w_router, bias, ids, w, s);
    const int E = c->n_experts, H = c->hidden;
    void *planes = scratch + P.planes;
    float *part = reinterpret_cast<float *>(scratch + P.part);
    int32_t *list = reinterpret_cast<int32_t *>(scratch + P.list);
    int32_t *list_n = reinterpret_cast<int32_t *>(scratch + P.counters);
    int32_t *bcnt = list_n + 1;
    float *exact = reinterpret_cast<float *>(scratch + P.exact);
    const int sms = g_dev[dev].num_sms;
    if (cudaMemsetAsync(list_n, 0, (1 + static_cast<size_t>(E)) * sizeof(int32_t), s) != cudaSuccess)
        return BEAM_MOE_ERR_CUDA;
    const int64_t n4 = static_cast<int64_t>(E) * H / 4;
    router_split_kernel<<<static_cast<unsigned>(std::min<int64_t>((n4 + 255) / 256, 4 * sms)), 256, 0, s>>>(
        reinterpret_cast<const float4 *>(w_router), n4, reinterpret_cast<uint2 *>(planes));
    int rc;
    if ((rc = launch_status())) return rc;
    CUtensorMap m_w, m_x;
    if (!encode_fn() || !make_map_3d(&m_w, planes, H, E, 3) || !make_map_2d(&m_x, x, H, T, P.bn))
        return BEAM_MOE_ERR_CUDA;
    const RouterTcParams q{T, H, E, P.S, P.kps, P.n_nt, P.n_mt, part, kDefaultTimeoutCycles};
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(static_cast<int64_t>(P.n_nt) * P.n_mt * P.S, sms));
    if (P.bn == 128) router_logits_kernel<128><<<grid, kRsThreads, RsCfg<128>::kSmem, s>>>(m_w, m_x, q);
    else if (P.bn == 64) router_logits_kernel<64><<<grid, kRsThreads, RsCfg<64>::kSmem, s>>>(m_w, m_x, q);
    else router_logits_kernel<32><<<grid, kRsThreads, RsCfg<32>::kSmem, s>>>(m_w, m_x, q);
    if ((rc = launch_status())) return rc;
    const RouterSelParams r{reinterpret_cast<const __nv_bfloat16 *>(x), w_router, bias, ids, w, T, H, E,
                            c->n_groups, c->topk_groups, c->topk, c->group_topn, P.S, part, list, list_n, exact,
                            bcnt, reinterpret_cast<int32_t *>(scratch + P.bucket),
                            reinterpret_cast<float *>(scratch + P.xlogit), scratch + P.listed};
    router_screen_kernel<<<static_cast<unsigned>((T + 7) / 8), 256, 0, s>>>(r);
    if ((rc = launch_status())) return rc;
    // the listed tokens' CTAs first (they start early and overlap the picks), then one persistent CTA per
    // SM for the screened picks
    const int n_chunk = (E + 31) / 32;
    const int n_exact = n_chunk * static_cast<int>(std::min<int64_t>((T + 7) / 8, 64));
    router_exact_kernel<<<static_cast<unsigned>(n_exact + sms), 256, kRsPathSmem, s>>>(r, exact, n_exact);
    if ((rc = launch_status())) return rc;
    router_finish_kernel<<<static_cast<unsigned>((T + 7) / 8), 256, 0, s>>>(r);  // list_n <= T
    return launch_status();
}

int enqueue_permute(const beam_moe_config *c, int64_t T, const int32_t *ids, int32_t *counts, int64_t *offsets,
                    int32_t *row_src, int32_t *dest_row, int32_t *hist, cudaStream_t s) {
    const int nc = static_cast<int>(n_chunks(T));
    permute_hist_kernel<<<nc, kPmThreads, 0, s>>>(ids, T, c->topk, c->n_experts, hist);
    permute_scan_kernel<<<1, 1024, 0, s>>>(hist, nc, c->n_experts, counts, offsets);
    permute_scatter_kernel<<<nc, kPmThreads, 0, s>>>(ids, T, c->topk, c->n_experts, hist, offsets, row_src,
                                                    dest_row);
    return launch_status();
}

// Records events[i] on s when profiling (events may be null).
bool record(cudaEvent_t const *events, int i, cudaStream_t s) {
    return !events || cudaEventRecord(events[i], s) == cudaSuccess;
}

// The block's last step when it runs on the residual stream: post-norm and scaled residual update.
struct BlockTail {
    const beam_bf16 *stream_in;
    const float *g_post;
    float eps, keep, add;
};

// The experts' weights: bf16 [E][rows][K], E4M3 codes with their scale codes, or E2M1 code
// pairs with their scale codes and per-matrix scales.
struct ExpertWeights {
    const void *gate, *up, *down;
    const uint8_t *s_gate, *s_up, *s_down;  // FP8: [E][K/32][rows]; FP4: [E][K/16][rows]
    const float *g_gate, *g_up, *g_down;    // FP4 only: [E]
    bool fp8, fp4;
};

ExpertWeights bf16_weights(const beam_bf16 *wg, const beam_bf16 *wu, const beam_bf16 *wd) {
    return ExpertWeights{wg, wu, wd, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, false, false};
}

int enqueue_experts(const beam_moe_config *c, int dev, int64_t T, const beam_bf16 *x, const int32_t *ids,
                    const float *w, const ExpertWeights &W, beam_bf16 *y, uint8_t *ws, const Layout &L,
                    cudaStream_t s, cudaEvent_t const *ev = nullptr, const BlockTail *tail = nullptr) {
    int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    int64_t *offsets = reinterpret_cast<int64_t *>(ws + L.offsets);
    int32_t *row_src = reinterpret_cast<int32_t *>(ws + L.row_src);
    int32_t *dest_row = reinterpret_cast<int32_t *>(ws + L.dest_row);
    int32_t *hist = reinterpret_cast<int32_t *>(ws + L.hist);
    void *h = ws + L.h;
    void *o = ws + L.o;
    const int k = c->topk, E = c->n_experts, H = c->hidden, I = c->inter;
    const uint64_t R = static_cast<uint64_t>(T) * k;
    const bool narrow = narrow_tiles(c, T);

    int rc = enqueue_permute(c, T, ids, counts, offsets, row_src, dest_row, hist, s);
    if (rc) return rc;
    if (!record(ev, 2, s)) return BEAM_MOE_ERR_CUDA;
    if (!narrow) {
        gather_rows_kernel<<<static_cast<unsigned>(T), 128, 0, s>>>(reinterpret_cast<const uint4 *>(x), T, k, H / 8,
                                                                    dest_row, reinterpret_cast<uint4 *>(ws + L.xp));
        if ((rc = launch_status())) return rc;
    }
    if (!record(ev, 3, s)) return BEAM_MOE_ERR_CUDA;

    const double mean_rows = static_cast<double>(R) / E;
    const int bn = narrow ? kNarrowBN : kWideBN;
    // bf16 weights with wide tiles run on CTA pairs, which stage their token rows in 32-row boxes
    const bool pair2 = !narrow && !W.fp8 && !W.fp4;
    const int box = narrow ? kNarrowBox : (pair2 ? k2smBox : kWideBox);
    // Weights are read once per call when (almost) every expert fits one token tile: mark them
    // evict-first so they do not push the reused activations out of L2.
    const int once = (mean_rows + 4.0 * std::sqrt(mean_rows) <= bn) ? 1 : 0;
    CUtensorMap m_wg, m_wu, m_b1, m_wd, m_h, m_sg, m_su, m_sd;
    if (!encode_fn()) return BEAM_MOE_ERR_CUDA;
    const bool b1_ok = narrow ? make_map_2d(&m_b1, x, H, static_cast<uint64_t>(T), 1)   // gather4 rows of x
                              : make_map_2d(&m_b1, ws + L.xp, H, R, box);              // tiled x_perm rows
    bool w_ok;
    if (W.fp4) {
        w_ok = make_map_3d_fp4(&m_wg, W.gate, H, I, E) && make_map_3d_fp4(&m_wu, W.up, H, I, E) &&
               make_map_3d_fp4(&m_wd, W.down, I, H, E) && make_map_scale(&m_sg, W.s_gate, I, H / 16, E, 16) &&
               make_map_scale(&m_su, W.s_up, I, H / 16, E, 16) && make_map_scale(&m_sd, W.s_down, H, I / 16, E, 16);
    } else if (W.fp8) {
        w_ok = make_map_3d_fp8(&m_wg, W.gate, H, I, E) && make_map_3d_fp8(&m_wu, W.up, H, I, E) &&
               make_map_3d_fp8(&m_wd, W.down, I, H, E) && make_map_scale(&m_sg, W.s_gate, I, H / 32, E) &&
               make_map_scale(&m_su, W.s_up, I, H / 32, E) && make_map_scale(&m_sd, W.s_down, H, I / 32, E);
    } else {
        w_ok = make_map_3d(&m_wg, W.gate, H, I, E) && make_map_3d(&m_wu, W.up, H, I, E) &&
               make_map_3d(&m_wd, W.down, I, H, E);
    }
    if (!b1_ok || !w_ok || !make_map_2d(&m_h, h, I, R, box)) return BEAM_MOE_ERR_CUDA;
    const int grid = g_dev[dev].num_sms;
    // NVFP4: the rebuilt tiles hold e2m1 x scale x 2^-9; the per-matrix scales and 2^9 multiply the
    // FP32 accumulators in the epilogue
    GemmParams p1{counts, offsets, h, E, H, I, once, kDefaultTimeoutCycles, row_src, k};
    GemmParams p2{counts, offsets, o, E, I, H, once, kDefaultTimeoutCycles, nullptr, k};
    const AccScales a1{W.g_gate, W.g_up, 512.0f}, a2{W.g_down, nullptr, 512.0f};
    if (W.fp4) {
        if (narrow) launch_gemm_fp8<G1_NARROW_NV4_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1, a1);
        else launch_gemm_fp8<G1_WIDE_NV4_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1, a1);
    } else if (W.fp8) {
        if (narrow) launch_gemm_fp8<G1_NARROW_FP8_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1, a1);
        else launch_gemm_fp8<G1_WIDE_FP8_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1, a1);
    } else {
        if (narrow) launch_gemm<G1_NARROW_ARGS>(grid, s, m_wg, m_wu, m_b1, p1);
        else if (once) launch_gemm2<G1_2SM_ARGS>(g_dev[dev].pairs_g1, s, m_wg, m_wu, m_b1, p1);
        else launch_gemm2<G1_2SM_BIG_ARGS>(g_dev[dev].pairs_g1b, s, m_wg, m_wu, m_b1, p1);
    }
    if ((rc = launch_status())) return rc;
    if (!record(ev, 4, s)) return BEAM_MOE_ERR_CUDA;
    if (W.fp4) {
        if (narrow) launch_gemm_fp8<G2_NARROW_NV4_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_h, p2, a2);
        else launch_gemm_fp8<G2_WIDE_NV4_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_h, p2, a2);
    } else if (W.fp8) {
        if (narrow) launch_gemm_fp8<G2_NARROW_FP8_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_h, p2, a2);
        else launch_gemm_fp8<G2_WIDE_FP8_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_h, p2, a2);
    } else {
        if (narrow) launch_gemm<G2_NARROW_ARGS>(grid, s, m_wd, m_wd, m_h, p2);
        else if (once) launch_gemm2<G2_2SM_ARGS>(g_dev[dev].pairs_g2, s, m_wd, m_wd, m_h, p2);
        else launch_gemm2<G2_2SM_BIG_ARGS>(g_dev[dev].pairs_g2b, s, m_wd, m_wd, m_h, p2);
    }
    if ((rc = launch_status())) return rc;
    if (!record(ev, 5, s)) return BEAM_MOE_ERR_CUDA;
    if (tail)
        combine_norm_residual_kernel<<<static_cast<unsigned>(T), kNormThreads, H * 4, s>>>(
            reinterpret_cast<const float4 *>(o), dest_row, w, k, H, c->routed_scale,
            reinterpret_cast<const uint2 *>(tail->stream_in), tail->g_post, tail->eps, tail->keep, tail->add,
            reinterpret_cast<uint2 *>(y));
    else
        combine_kernel<<<static_cast<unsigned>(T), 256, 0, s>>>(reinterpret_cast<const float4 *>(o), dest_row, w, T,
                                                                k, H / 4, c->routed_scale, reinterpret_cast<uint2 *>(y));
    if ((rc = launch_status())) return rc;
    if (!record(ev, 6, s)) return BEAM_MOE_ERR_CUDA;
    return BEAM_MOE_OK;
}

// ---- block-scaled FP8 path (MXFP8 weights and activations, tcgen05 kind::mxf8f6f4) ----------------
bool mx8_shape_ok(const beam_moe_config *c) { return c->hidden % 128 == 0 && c->inter % 128 == 0; }

struct Mx8Layout {
    size_t ids = 0, w = 0, rt = 0, hist = 0, counts = 0, offsets = 0, row_src = 0, dest_row = 0, xq = 0, xs = 0, xqp = 0,
           hq = 0, hs = 0, o = 0, total = 0;
};

Mx8Layout mx8_layout(const beam_moe_config *c, int64_t T) {
    Mx8Layout L;
    if (T == 0) return L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    const size_t R = static_cast<size_t>(T) * c->topk;
    const size_t E = c->n_experts, H = c->hidden, I = c->inter;
    L.ids = take(R * 4);
    L.w = take(R * 4);
    L.rt = take(route_plan(c, T).total);
    L.hist = take(static_cast<size_t>(n_chunks(T)) * E * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 8);
    L.row_src = take(R * 4);
    L.dest_row = take(R * 4);
    L.xq = take(static_cast<size_t>(T) * H);
    L.xs = take(static_cast<size_t>(T) * (H / 32));
    if (!narrow_tiles(c, T)) L.xqp = take(R * H);  // x codes in dispatch order (wide tiles only)
    L.hq = take(R * I);
    L.hs = take(R * (I / 32));
    L.o = take(R * H * 2);  // bf16 expert outputs
    L.total = off;
    return L;
}

int enqueue_experts_mx8(const beam_moe_config *c, int dev, int64_t T, const beam_bf16 *x, const int32_t *ids,
                        const float *w, const beam_moe_fp8_experts *W, beam_bf16 *y, uint8_t *ws, const Mx8Layout &L,
                        cudaStream_t s, cudaEvent_t const *ev) {
    int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    int64_t *offsets = reinterpret_cast<int64_t *>(ws + L.offsets);
    int32_t *row_src = reinterpret_cast<int32_t *>(ws + L.row_src);
    int32_t *dest_row = reinterpret_cast<int32_t *>(ws + L.dest_row);
    const int k = c->topk, E = c->n_experts, H = c->hidden, I = c->inter;
    const uint64_t R = static_cast<uint64_t>(T) * k;
    const bool narrow = narrow_tiles(c, T);

    int rc = enqueue_permute(c, T, ids, counts, offsets, row_src, dest_row, reinterpret_cast<int32_t *>(ws + L.hist), s);
    if (rc) return rc;
    if (!record(ev, 2, s)) return BEAM_MOE_ERR_CUDA;
    // x -> MXFP8 codes and scales (every token once), then the codes into dispatch order (wide tiles)
    const int64_t n_blocks = T * static_cast<int64_t>(H / 32);
    quant_mx8_rows_kernel<<<static_cast<unsigned>((n_blocks * 4 + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(x), n_blocks, reinterpret_cast<uint2 *>(ws + L.xq), ws + L.xs);
    if ((rc = launch_status())) return rc;
    if (!narrow) {
        gather_rows_kernel<<<static_cast<unsigned>(T), 128, 0, s>>>(reinterpret_cast<const uint4 *>(ws + L.xq), T, k,
                                                                    H / 16, dest_row, reinterpret_cast<uint4 *>(ws + L.xqp));
        if ((rc = launch_status())) return rc;
    }
    if (!record(ev, 3, s)) return BEAM_MOE_ERR_CUDA;

    const double mean_rows = static_cast<double>(R) / E;
    const bool big = !narrow && mean_rows + 2.0 * std::sqrt(mean_rows) <= 160;  // G1_WIDE_MX8_160
    const int bn = narrow ? kNarrowBN : kWideBN;
    const int box = narrow ? kNarrowBox : kWideBox;
    const int once = (mean_rows + 4.0 * std::sqrt(mean_rows) <= bn) ? 1 : 0;
    CUtensorMap m_wg, m_wu, m_wd, m_sg, m_su, m_sd, m_b1, m_b2;
    if (!encode_fn()) return BEAM_MOE_ERR_CUDA;
    const bool b1_ok = narrow ? make_map_2d_any(&m_b1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.xq, H,
                                                static_cast<uint64_t>(T), kMxBK, 1, CU_TENSOR_MAP_SWIZZLE_128B)
                              : make_map_2d_any(&m_b1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.xqp, H, R, kMxBK,
                                                big ? 32 : box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!b1_ok ||
        !make_map_2d_any(&m_b2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.hq, I, R, kMxBK, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d_fp8(&m_wg, W->w_gate, H, I, E) || !make_map_3d_fp8(&m_wu, W->w_up, H, I, E) ||
        !make_map_3d_fp8(&m_wd, W->w_down, I, H, E) || !make_map_scale(&m_sg, W->w_gate_scale, I, H / 32, E) ||
        !make_map_scale(&m_su, W->w_up_scale, I, H / 32, E) || !make_map_scale(&m_sd, W->w_down_scale, H, I / 32, E))
        return BEAM_MOE_ERR_CUDA;
    const int grid = g_dev[dev].num_sms;
    Mx8Params p1{counts, offsets, E, H, I, once, kDefaultTimeoutCycles, row_src, k, ws + L.xs, 1, ws + L.hq, ws + L.hs,
                 nullptr, nullptr, nullptr, nullptr};
    Mx8Params p2{counts, offsets, E, I, H, once, kDefaultTimeoutCycles, row_src, k, ws + L.hs, 0, nullptr, nullptr,
                 reinterpret_cast<__nv_bfloat16 *>(ws + L.o), nullptr, nullptr, nullptr};
    if (narrow) launch_gemm_mx8<G1_NARROW_MX8_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1);
    else if (big) launch_gemm_mx8<G1_WIDE_MX8_160_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1);
    else launch_gemm_mx8<G1_WIDE_MX8_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1);
    if ((rc = launch_status())) return rc;
    if (!record(ev, 4, s)) return BEAM_MOE_ERR_CUDA;
    if (narrow) launch_gemm_mx8<G2_NARROW_MX8_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_b2, p2);
    else launch_gemm_mx8<G2_WIDE_MX8_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_b2, p2);
    if ((rc = launch_status())) return rc;
    if (!record(ev, 5, s)) return BEAM_MOE_ERR_CUDA;
    combine_bf16_kernel<<<static_cast<unsigned>(T), 256, 0, s>>>(reinterpret_cast<const uint4 *>(ws + L.o), dest_row,
                                                                 w, T, k, H / 8, c->routed_scale,
                                                                 reinterpret_cast<uint4 *>(y));
    if ((rc = launch_status())) return rc;
    if (!record(ev, 6, s)) return BEAM_MOE_ERR_CUDA;
    return BEAM_MOE_OK;
}

// ---- 4-bit path (NVFP4 weights and activations, tcgen05 kind::mxf4nvf4) -------------------------
bool w4a4_shape_ok(const beam_moe_config *c) { return c->hidden % 256 == 0 && c->inter % 256 == 0; }

struct W4a4Layout {
    size_t ids = 0, w = 0, rt = 0, hist = 0, counts = 0, offsets = 0, row_src = 0, dest_row = 0, xq = 0, xs = 0, gx = 0, xqp = 0,
           hq = 0, hs = 0, o = 0, total = 0;
};

W4a4Layout w4a4_layout(const beam_moe_config *c, int64_t T) {
    W4a4Layout L;
    if (T == 0) return L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    const size_t R = static_cast<size_t>(T) * c->topk;
    const size_t E = c->n_experts, H = c->hidden, I = c->inter;
    L.ids = take(R * 4);
    L.w = take(R * 4);
    L.rt = take(route_plan(c, T).total);
    L.hist = take(static_cast<size_t>(n_chunks(T)) * E * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 8);
    L.row_src = take(R * 4);
    L.dest_row = take(R * 4);
    L.xq = take(static_cast<size_t>(T) * (H / 2));
    L.xs = take(static_cast<size_t>(T) * (H / 16));
    L.gx = take(static_cast<size_t>(T) * 4);
    if (!narrow_tiles(c, T)) L.xqp = take(R * (H / 2));
    L.hq = take(R * (I / 2));
    L.hs = take(R * (I / 16));
    L.o = take(R * H * 2);  // bf16 expert outputs
    L.total = off;
    return L;
}

int enqueue_experts_w4a4(const beam_moe_config *c, int dev, int64_t T, const beam_bf16 *x, const int32_t *ids,
                         const float *w, const beam_moe_nvfp4_experts *W, beam_bf16 *y, uint8_t *ws,
                         const W4a4Layout &L, cudaStream_t s, cudaEvent_t const *ev) {
    int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    int64_t *offsets = reinterpret_cast<int64_t *>(ws + L.offsets);
    int32_t *row_src = reinterpret_cast<int32_t *>(ws + L.row_src);
    int32_t *dest_row = reinterpret_cast<int32_t *>(ws + L.dest_row);
    const int k = c->topk, E = c->n_experts, H = c->hidden, I = c->inter;
    const uint64_t R = static_cast<uint64_t>(T) * k;
    const bool narrow = narrow_tiles(c, T);

    int rc = enqueue_permute(c, T, ids, counts, offsets, row_src, dest_row, reinterpret_cast<int32_t *>(ws + L.hist), s);
    if (rc) return rc;
    if (!record(ev, 2, s)) return BEAM_MOE_ERR_CUDA;
    quant_nv4_rows_kernel<<<static_cast<unsigned>(T), 128, 0, s>>>(reinterpret_cast<const uint4 *>(x), H,
                                                                  reinterpret_cast<uint2 *>(ws + L.xq), ws + L.xs,
                                                                  reinterpret_cast<float *>(ws + L.gx));
    if ((rc = launch_status())) return rc;
    if (!narrow) {
        gather_rows_kernel<<<static_cast<unsigned>(T), 128, 0, s>>>(reinterpret_cast<const uint4 *>(ws + L.xq), T, k,
                                                                    H / 32, dest_row, reinterpret_cast<uint4 *>(ws + L.xqp));
        if ((rc = launch_status())) return rc;
    }
    if (!record(ev, 3, s)) return BEAM_MOE_ERR_CUDA;

    const double mean_rows = static_cast<double>(R) / E;
    const bool big = !narrow && mean_rows + 2.0 * std::sqrt(mean_rows) <= kNv4BigBN;
    const int bn = narrow ? kNarrowBN : (big ? kNv4BigBN : 128);
    const int box = narrow ? kNarrowBox : (big ? kNv4BigBox : kWideBox);
    const int once = (mean_rows + 4.0 * std::sqrt(mean_rows) <= bn) ? 1 : 0;
    CUtensorMap m_wg, m_wu, m_wd, m_sg, m_su, m_sd, m_b1, m_b2;
    if (!encode_fn()) return BEAM_MOE_ERR_CUDA;
    const bool b1_ok = narrow ? make_map_2d_any(&m_b1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.xq, H / 2,
                                                static_cast<uint64_t>(T), kMxBK, 1, CU_TENSOR_MAP_SWIZZLE_128B)
                              : make_map_2d_any(&m_b1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.xqp, H / 2, R, kMxBK,
                                                box, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!b1_ok ||
        !make_map_2d_any(&m_b2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws + L.hq, I / 2, R, kMxBK, box,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_3d_fp4(&m_wg, W->w_gate, H, I, E) || !make_map_3d_fp4(&m_wu, W->w_up, H, I, E) ||
        !make_map_3d_fp4(&m_wd, W->w_down, I, H, E) || !make_map_scale(&m_sg, W->w_gate_scale, I, H / 16, E, 16) ||
        !make_map_scale(&m_su, W->w_up_scale, I, H / 16, E, 16) ||
        !make_map_scale(&m_sd, W->w_down_scale, H, I / 16, E, 16))
        return BEAM_MOE_ERR_CUDA;
    const int grid = g_dev[dev].num_sms;
    Mx8Params p1{counts, offsets, E, H, I, once, kDefaultTimeoutCycles, row_src, k, ws + L.xs, 1, ws + L.hq, ws + L.hs,
                 nullptr, W->w_gate_global, W->w_up_global, reinterpret_cast<const float *>(ws + L.gx)};
    Mx8Params p2{counts, offsets, E, I, H, once, kDefaultTimeoutCycles, row_src, k, ws + L.hs, 0, nullptr, nullptr,
                 reinterpret_cast<__nv_bfloat16 *>(ws + L.o), W->w_down_global, nullptr, nullptr};
    if (narrow) launch_gemm_mx8<G1_NARROW_NV4X_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1);
    else if (big) launch_gemm_mx8<G1_WIDE_NV4X_160_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1);
    else launch_gemm_mx8<G1_WIDE_NV4X_ARGS>(grid, s, m_wg, m_wu, m_sg, m_su, m_b1, p1);
    if ((rc = launch_status())) return rc;
    if (!record(ev, 4, s)) return BEAM_MOE_ERR_CUDA;
    if (narrow) launch_gemm_mx8<G2_NARROW_NV4X_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_b2, p2);
    else if (big) launch_gemm_mx8<G2_WIDE_NV4X_160_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_b2, p2);
    else launch_gemm_mx8<G2_WIDE_NV4X_ARGS>(grid, s, m_wd, m_wd, m_sd, m_sd, m_b2, p2);
    if ((rc = launch_status())) return rc;
    if (!record(ev, 5, s)) return BEAM_MOE_ERR_CUDA;
    combine_bf16_kernel<<<static_cast<unsigned>(T), 256, 0, s>>>(reinterpret_cast<const uint4 *>(ws + L.o), dest_row,
                                                                 w, T, k, H / 8, c->routed_scale,
                                                                 reinterpret_cast<uint4 *>(y));
    if ((rc = launch_status())) return rc;
    if (!record(ev, 6, s)) return BEAM_MOE_ERR_CUDA;
    return BEAM_MOE_OK;
}

__global__ void selftest_timeout_kernel(long long cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, cycles);  // nobody arrives: the bounded wait expires and records the status
    }
}

}  // namespace
}  // namespace beam

using namespace beam;

extern "C" {

size_t beam_moe_workspace_size(const beam_moe_config *cfg, int64_t T, int which) {
    if (validate(cfg) || check_T(cfg, T)) return 0;
    if (which < BEAM_MOE_WS_ROUTE || which > BEAM_MOE_WS_ROUTE_SCREENED) return 0;
    if (which == BEAM_MOE_WS_MXFP8) return mx8_shape_ok(cfg) ? mx8_layout(cfg, T).total : 0;
    if (which == BEAM_MOE_WS_W4A4) return w4a4_shape_ok(cfg) ? w4a4_layout(cfg, T).total : 0;
    if (which == BEAM_MOE_WS_ROUTE_SCREENED) return route_plan(cfg, T).total;
    return layout(cfg, T, which).total;
}

int beam_moe_route(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                   const float *sel_bias, int32_t *topk_ids, float *topk_w, void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !w_router || !topk_ids || !topk_w) return BEAM_MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(w_router)) return BEAM_MOE_ERR_MISALIGNED;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    return enqueue_route(cfg, T, x, w_router, sel_bias, topk_ids, topk_w, static_cast<cudaStream_t>(stream));
}

int beam_moe_route_screened(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                            const float *sel_bias, int32_t *topk_ids, float *topk_w, void *ws, size_t ws_bytes,
                            void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !w_router || !topk_ids || !topk_w) return BEAM_MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(w_router)) return BEAM_MOE_ERR_MISALIGNED;
    const RoutePlan P = route_plan(cfg, T);
    if (P.ok) {
        if (!ws) return BEAM_MOE_ERR_NULL;
        if (!aligned16(ws)) return BEAM_MOE_ERR_MISALIGNED;
        if (ws_bytes < P.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    }
    int dev;
    if ((rc = init_device(&dev))) return rc;
    return enqueue_route_ws(cfg, dev, T, x, w_router, sel_bias, topk_ids, topk_w,
                            P.ok ? static_cast<uint8_t *>(ws) : nullptr, static_cast<cudaStream_t>(stream));
}

int beam_moe_permute(const beam_moe_config *cfg, int64_t T, const int32_t *topk_ids, int32_t *counts,
                     int64_t *offsets, int32_t *row_src, int32_t *dest_row, void *ws, size_t ws_bytes,
                     void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (!counts || !offsets || (T > 0 && (!topk_ids || !row_src || !dest_row || !ws))) return BEAM_MOE_ERR_NULL;
    if (ws && !aligned16(ws)) return BEAM_MOE_ERR_MISALIGNED;
    const Layout L = layout(cfg, T, BEAM_MOE_WS_PERMUTE);
    if (ws_bytes < L.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // counts = 0, offsets = 0 keep the outputs well defined
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, s) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int64_t) * (cfg->n_experts + 1), s) != cudaSuccess)
            return BEAM_MOE_ERR_CUDA;
        return BEAM_MOE_OK;
    }
    return enqueue_permute(cfg, T, topk_ids, counts, offsets, row_src, dest_row,
                           reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + L.hist), s);
}

}  // extern "C"

namespace beam {
namespace {
// Argument checks of the experts' weights: every pointer set and 16-byte aligned.
int weights_status(const ExpertWeights &W) {
    const bool scaled = W.fp8 || W.fp4;
    if (!W.gate || !W.up || !W.down) return BEAM_MOE_ERR_NULL;
    if (scaled && (!W.s_gate || !W.s_up || !W.s_down)) return BEAM_MOE_ERR_NULL;
    if (W.fp4 && (!W.g_gate || !W.g_up || !W.g_down)) return BEAM_MOE_ERR_NULL;
    if (!aligned16(W.gate) || !aligned16(W.up) || !aligned16(W.down)) return BEAM_MOE_ERR_MISALIGNED;
    if (scaled && (!aligned16(W.s_gate) || !aligned16(W.s_up) || !aligned16(W.s_down))) return BEAM_MOE_ERR_MISALIGNED;
    if (W.fp4 && ((reinterpret_cast<uintptr_t>(W.g_gate) | reinterpret_cast<uintptr_t>(W.g_up) |
                   reinterpret_cast<uintptr_t>(W.g_down)) & 3u))
        return BEAM_MOE_ERR_MISALIGNED;
    return BEAM_MOE_OK;
}

ExpertWeights fp8_weights(const beam_moe_fp8_experts *w8) {
    return ExpertWeights{w8->w_gate, w8->w_up, w8->w_down, w8->w_gate_scale, w8->w_up_scale, w8->w_down_scale,
                         nullptr, nullptr, nullptr, true, false};
}

ExpertWeights nvfp4_weights(const beam_moe_nvfp4_experts *w4) {
    return ExpertWeights{w4->w_gate, w4->w_up, w4->w_down, w4->w_gate_scale, w4->w_up_scale, w4->w_down_scale,
                         w4->w_gate_global, w4->w_up_global, w4->w_down_global, false, true};
}

int experts_impl(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                 const float *topk_w, const ExpertWeights &W, beam_bf16 *y, void *ws, size_t ws_bytes, void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !topk_ids || !topk_w || !y || !ws) return BEAM_MOE_ERR_NULL;
    if ((rc = weights_status(W))) return rc;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return BEAM_MOE_ERR_MISALIGNED;
    const Layout L = layout(cfg, T, BEAM_MOE_WS_EXPERTS);
    if (ws_bytes < L.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    return enqueue_experts(cfg, dev, T, x, topk_ids, topk_w, W, y, static_cast<uint8_t *>(ws), L,
                           static_cast<cudaStream_t>(stream));
}

int forward_impl(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                 const float *sel_bias, const ExpertWeights &W, beam_bf16 *y, int32_t *topk_ids_out,
                 float *topk_w_out, void *ws, size_t ws_bytes, void *stream, cudaEvent_t const *ev) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !w_router || !y || !ws) return BEAM_MOE_ERR_NULL;
    if ((rc = weights_status(W))) return rc;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(y) || !aligned16(ws)) return BEAM_MOE_ERR_MISALIGNED;
    const Layout L = layout(cfg, T, BEAM_MOE_WS_FORWARD);
    if (ws_bytes < L.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    int32_t *ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t *>(wsb + L.ids);
    float *w = topk_w_out ? topk_w_out : reinterpret_cast<float *>(wsb + L.w);
    if (!record(ev, 0, s)) return BEAM_MOE_ERR_CUDA;
    if ((rc = enqueue_route_ws(cfg, dev, T, x, w_router, sel_bias, ids, w, wsb + L.rt, s))) return rc;
    if (!record(ev, 1, s)) return BEAM_MOE_ERR_CUDA;
    return enqueue_experts(cfg, dev, T, x, ids, w, W, y, wsb, L, s, ev);
}

bool events_ok(void *const *events) {
    if (!events) return false;
    for (int i = 0; i < 7; ++i)
        if (!events[i]) return false;
    return true;
}
}  // namespace
}  // namespace beam

extern "C" {

int beam_moe_experts(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                     const float *topk_w, const beam_bf16 *w_gate, const beam_bf16 *w_up, const beam_bf16 *w_down,
                     beam_bf16 *y, void *ws, size_t ws_bytes, void *stream) {
    return experts_impl(cfg, T, x, topk_ids, topk_w, bf16_weights(w_gate, w_up, w_down), y, ws, ws_bytes, stream);
}

int beam_moe_experts_fp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                         const float *topk_w, const beam_moe_fp8_experts *w8, beam_bf16 *y, void *ws, size_t ws_bytes,
                         void *stream) {
    if (!w8) return BEAM_MOE_ERR_NULL;
    return experts_impl(cfg, T, x, topk_ids, topk_w, fp8_weights(w8), y, ws, ws_bytes, stream);
}

int beam_moe_experts_nvfp4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                           const float *topk_w, const beam_moe_nvfp4_experts *w4, beam_bf16 *y, void *ws,
                           size_t ws_bytes, void *stream) {
    if (!w4) return BEAM_MOE_ERR_NULL;
    return experts_impl(cfg, T, x, topk_ids, topk_w, nvfp4_weights(w4), y, ws, ws_bytes, stream);
}

int beam_moe_forward_nvfp4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                           const float *sel_bias, const beam_moe_nvfp4_experts *w4, beam_bf16 *y,
                           int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes, void *stream,
                           void *const *events) {
    if (!w4 || (events && !events_ok(events))) return BEAM_MOE_ERR_NULL;
    return forward_impl(cfg, T, x, w_router, sel_bias, nvfp4_weights(w4), y, topk_ids_out, topk_w_out, ws, ws_bytes,
                        stream, reinterpret_cast<cudaEvent_t const *>(events));
}

int beam_moe_forward(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                     const float *sel_bias, const beam_bf16 *w_gate, const beam_bf16 *w_up, const beam_bf16 *w_down,
                     beam_bf16 *y, int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes, void *stream) {
    return forward_impl(cfg, T, x, w_router, sel_bias, bf16_weights(w_gate, w_up, w_down), y, topk_ids_out,
                        topk_w_out, ws, ws_bytes, stream, nullptr);
}

int beam_moe_forward_profiled(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                              const float *sel_bias, const beam_bf16 *w_gate, const beam_bf16 *w_up,
                              const beam_bf16 *w_down, beam_bf16 *y, int32_t *topk_ids_out, float *topk_w_out,
                              void *ws, size_t ws_bytes, void *stream, void *const *events) {
    if (!events_ok(events)) return BEAM_MOE_ERR_NULL;
    return forward_impl(cfg, T, x, w_router, sel_bias, bf16_weights(w_gate, w_up, w_down), y, topk_ids_out,
                        topk_w_out, ws, ws_bytes, stream, reinterpret_cast<cudaEvent_t const *>(events));
}

int beam_moe_forward_fp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                         const float *sel_bias, const beam_moe_fp8_experts *w8, beam_bf16 *y, int32_t *topk_ids_out,
                         float *topk_w_out, void *ws, size_t ws_bytes, void *stream, void *const *events) {
    if (!w8 || (events && !events_ok(events))) return BEAM_MOE_ERR_NULL;
    return forward_impl(cfg, T, x, w_router, sel_bias, fp8_weights(w8), y, topk_ids_out, topk_w_out, ws, ws_bytes,
                        stream, reinterpret_cast<cudaEvent_t const *>(events));
}

namespace {
int mx8_common_checks(const beam_moe_config *cfg, int64_t T, const beam_moe_fp8_experts *w8, const void *x,
                      const void *y, void *ws, size_t ws_bytes, void *const *events) {
    int rc = validate(cfg);
    if (rc) return rc;
    if (!mx8_shape_ok(cfg)) return BEAM_MOE_ERR_INVALID_CONFIG;
    if ((rc = check_T(cfg, T))) return rc;
    if (!w8 || (events && !events_ok(events))) return BEAM_MOE_ERR_NULL;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !y || !ws) return BEAM_MOE_ERR_NULL;
    if ((rc = weights_status(fp8_weights(w8)))) return rc;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return BEAM_MOE_ERR_MISALIGNED;
    if (ws_bytes < mx8_layout(cfg, T).total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    return BEAM_MOE_OK;
}
}  // namespace

int beam_moe_experts_mxfp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                           const float *topk_w, const beam_moe_fp8_experts *w8, beam_bf16 *y, void *ws,
                           size_t ws_bytes, void *stream) {
    int rc = mx8_common_checks(cfg, T, w8, x, y, ws, ws_bytes, nullptr);
    if (rc || T == 0) return rc;
    if (!topk_ids || !topk_w) return BEAM_MOE_ERR_NULL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    return enqueue_experts_mx8(cfg, dev, T, x, topk_ids, topk_w, w8, y, static_cast<uint8_t *>(ws),
                               mx8_layout(cfg, T), static_cast<cudaStream_t>(stream), nullptr);
}

int beam_moe_forward_mxfp8(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                           const float *sel_bias, const beam_moe_fp8_experts *w8, beam_bf16 *y, int32_t *topk_ids_out,
                           float *topk_w_out, void *ws, size_t ws_bytes, void *stream, void *const *events) {
    int rc = mx8_common_checks(cfg, T, w8, x, y, ws, ws_bytes, events);
    if (rc || T == 0) return rc;
    if (!w_router) return BEAM_MOE_ERR_NULL;
    if (!aligned16(w_router)) return BEAM_MOE_ERR_MISALIGNED;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    const Mx8Layout L = mx8_layout(cfg, T);
    int32_t *ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t *>(wsb + L.ids);
    float *w = topk_w_out ? topk_w_out : reinterpret_cast<float *>(wsb + L.w);
    cudaEvent_t const *ev = reinterpret_cast<cudaEvent_t const *>(events);
    if (!record(ev, 0, s)) return BEAM_MOE_ERR_CUDA;
    if ((rc = enqueue_route_ws(cfg, dev, T, x, w_router, sel_bias, ids, w, wsb + L.rt, s))) return rc;
    if (!record(ev, 1, s)) return BEAM_MOE_ERR_CUDA;
    return enqueue_experts_mx8(cfg, dev, T, x, ids, w, w8, y, wsb, L, s, ev);
}

namespace {
int w4a4_common_checks(const beam_moe_config *cfg, int64_t T, const beam_moe_nvfp4_experts *w4, const void *x,
                       const void *y, void *ws, size_t ws_bytes, void *const *events) {
    int rc = validate(cfg);
    if (rc) return rc;
    if (!w4a4_shape_ok(cfg)) return BEAM_MOE_ERR_INVALID_CONFIG;
    if ((rc = check_T(cfg, T))) return rc;
    if (!w4 || (events && !events_ok(events))) return BEAM_MOE_ERR_NULL;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !y || !ws) return BEAM_MOE_ERR_NULL;
    if ((rc = weights_status(nvfp4_weights(w4)))) return rc;
    if (!aligned16(x) || !aligned16(y) || !aligned16(ws)) return BEAM_MOE_ERR_MISALIGNED;
    if (ws_bytes < w4a4_layout(cfg, T).total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    return BEAM_MOE_OK;
}
}  // namespace

int beam_moe_experts_w4a4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *topk_ids,
                          const float *topk_w, const beam_moe_nvfp4_experts *w4, beam_bf16 *y, void *ws,
                          size_t ws_bytes, void *stream) {
    int rc = w4a4_common_checks(cfg, T, w4, x, y, ws, ws_bytes, nullptr);
    if (rc || T == 0) return rc;
    if (!topk_ids || !topk_w) return BEAM_MOE_ERR_NULL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    return enqueue_experts_w4a4(cfg, dev, T, x, topk_ids, topk_w, w4, y, static_cast<uint8_t *>(ws),
                                w4a4_layout(cfg, T), static_cast<cudaStream_t>(stream), nullptr);
}

int beam_moe_forward_w4a4(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const float *w_router,
                          const float *sel_bias, const beam_moe_nvfp4_experts *w4, beam_bf16 *y, int32_t *topk_ids_out,
                          float *topk_w_out, void *ws, size_t ws_bytes, void *stream, void *const *events) {
    int rc = w4a4_common_checks(cfg, T, w4, x, y, ws, ws_bytes, events);
    if (rc || T == 0) return rc;
    if (!w_router) return BEAM_MOE_ERR_NULL;
    if (!aligned16(w_router)) return BEAM_MOE_ERR_MISALIGNED;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    const W4a4Layout L = w4a4_layout(cfg, T);
    int32_t *ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t *>(wsb + L.ids);
    float *w = topk_w_out ? topk_w_out : reinterpret_cast<float *>(wsb + L.w);
    cudaEvent_t const *ev = reinterpret_cast<cudaEvent_t const *>(events);
    if (!record(ev, 0, s)) return BEAM_MOE_ERR_CUDA;
    if ((rc = enqueue_route_ws(cfg, dev, T, x, w_router, sel_bias, ids, w, wsb + L.rt, s))) return rc;
    if (!record(ev, 1, s)) return BEAM_MOE_ERR_CUDA;
    return enqueue_experts_w4a4(cfg, dev, T, x, ids, w, w4, y, wsb, L, s, ev);
}

int beam_moe_device_status(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v = BEAM_MOE_OK;
    const int zero = BEAM_MOE_OK;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
    return v;
}

int beam_moe_selftest_timeout(int64_t timeout_us, void *stream) {
    if (timeout_us < 1 || timeout_us > 1000000) return BEAM_MOE_ERR_INVALID_ARG;
    int dev, rc;
    if ((rc = init_device(&dev))) return rc;
    const long long cycles = static_cast<long long>(timeout_us) * g_dev[dev].clock_khz / 1000;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cycles);
    return launch_status();
}

const char *beam_moe_strerror(int code) {
    switch (code) {
        case BEAM_MOE_OK: return "ok";
        case BEAM_MOE_ERR_INVALID_CONFIG: return "invalid layer configuration";
        case BEAM_MOE_ERR_NULL: return "a required pointer is NULL";
        case BEAM_MOE_ERR_MISALIGNED: return "a pointer is not 16-byte aligned";
        case BEAM_MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case BEAM_MOE_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0, sm_100a)";
        case BEAM_MOE_ERR_CUDA: return "CUDA runtime or launch error";
        case BEAM_MOE_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
        case BEAM_MOE_ERR_BAD_INDEX: return "an expert id outside [0, n_experts)";
        case BEAM_MOE_ERR_INVALID_ARG: return "invalid argument (token count out of range)";
        default: return "unknown error code";
    }
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// beam_moe_block_forward: pre-norm -> block -> post-norm -> scaled residual update.
extern "C" int beam_moe_block_forward(const beam_moe_config *cfg, const beam_moe_sublayer *sub, int64_t T,
                                      const beam_bf16 *stream_in, const float *w_router, const float *sel_bias,
                                      const beam_bf16 *w_gate, const beam_bf16 *w_up, const beam_bf16 *w_down,
                                      beam_bf16 *stream_out, beam_bf16 *u_out, int32_t *topk_ids_out,
                                      float *topk_w_out, void *ws, size_t ws_bytes, void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if (!sub) return BEAM_MOE_ERR_NULL;
    if (cfg->hidden > kMaxBlockHidden || sub->step < 2 || !(sub->eps >= 0.0f) || !(sub->eps < INFINITY))
        return BEAM_MOE_ERR_INVALID_CONFIG;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!stream_in || !w_router || !w_gate || !w_up || !w_down || !stream_out || !ws || !sub->pre_norm_weight ||
        !sub->post_norm_weight)
        return BEAM_MOE_ERR_NULL;
    if (!aligned16(stream_in) || !aligned16(w_router) || !aligned16(w_gate) || !aligned16(w_up) ||
        !aligned16(w_down) || !aligned16(stream_out) || !aligned16(ws) || (u_out && !aligned16(u_out)) ||
        !aligned16(sub->pre_norm_weight) || !aligned16(sub->post_norm_weight))
        return BEAM_MOE_ERR_MISALIGNED;
    const Layout L = layout(cfg, T, BEAM_MOE_WS_BLOCK);
    if (ws_bytes < L.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    beam_bf16 *u = u_out ? u_out : reinterpret_cast<beam_bf16 *>(wsb + L.u);
    int32_t *ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t *>(wsb + L.ids);
    float *w = topk_w_out ? topk_w_out : reinterpret_cast<float *>(wsb + L.w);
    rmsnorm_bf16_kernel<<<static_cast<unsigned>(T), kNormThreads, 0, s>>>(
        reinterpret_cast<const uint4 *>(stream_in), sub->pre_norm_weight, sub->eps, cfg->hidden,
        reinterpret_cast<uint4 *>(u));
    if ((rc = launch_status())) return rc;
    if ((rc = enqueue_route_ws(cfg, dev, T, u, w_router, sel_bias, ids, w, wsb + L.rt, s))) return rc;
    const double k = sub->step;
    const BlockTail tail{stream_in, sub->post_norm_weight, sub->eps, static_cast<float>(std::sqrt((k - 1.0) / k)),
                         static_cast<float>(1.0 / std::sqrt(k))};
    return enqueue_experts(cfg, dev, T, u, ids, w, bf16_weights(w_gate, w_up, w_down), stream_out, wsb, L, s, nullptr,
                           &tail);
}

// ------------------------------------------------------------------------------------------------
// beam_moe_dense_swiglu: the grouped engine with one expert that takes every token in order.
namespace beam {
namespace {

__global__ void dense_schedule_kernel(int32_t *counts, int64_t *offsets, int64_t T) {
    counts[0] = static_cast<int32_t>(T);
    offsets[0] = 0;
    offsets[1] = T;
}

struct DenseLayout {
    size_t counts = 0, offsets = 0, h = 0, total = 0;
};

bool dense_shape_ok(int32_t H, int32_t I) {
    return H >= 64 && H <= 65536 && H % 64 == 0 && I >= 64 && I <= 65536 && I % 64 == 0;
}

DenseLayout dense_layout(int32_t H, int32_t I, int64_t T) {
    DenseLayout L;
    if (T == 0) return L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.counts = take(4);
    L.offsets = take(16);
    L.h = take(static_cast<size_t>(T) * I * 2);
    L.total = off;
    return L;
}

}  // namespace
}  // namespace beam

extern "C" size_t beam_moe_dense_workspace_size(int32_t hidden, int32_t inter, int64_t T) {
    if (!dense_shape_ok(hidden, inter) || T < 0 || T > kMaxTokens) return 0;
    return dense_layout(hidden, inter, T).total;
}

extern "C" int beam_moe_dense_swiglu(int32_t hidden, int32_t inter, int64_t T, const beam_bf16 *x,
                                     const beam_bf16 *w_gate, const beam_bf16 *w_up, const beam_bf16 *w_down,
                                     beam_bf16 *y, void *ws, size_t ws_bytes, void *stream) {
    if (!dense_shape_ok(hidden, inter)) return BEAM_MOE_ERR_INVALID_CONFIG;
    if (T < 0 || T > kMaxTokens) return BEAM_MOE_ERR_INVALID_ARG;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !w_gate || !w_up || !w_down || !y || !ws) return BEAM_MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(y) ||
        !aligned16(ws))
        return BEAM_MOE_ERR_MISALIGNED;
    const DenseLayout L = dense_layout(hidden, inter, T);
    if (ws_bytes < L.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev, rc;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    int32_t *counts = reinterpret_cast<int32_t *>(wsb + L.counts);
    int64_t *offsets = reinterpret_cast<int64_t *>(wsb + L.offsets);
    void *h = wsb + L.h;
    dense_schedule_kernel<<<1, 1, 0, s>>>(counts, offsets, T);
    if ((rc = launch_status())) return rc;
    // x itself is the token-ordered B operand of the gate/up GEMM (CTA pairs, 256-token tiles, 32-row boxes)
    CUtensorMap m_wg, m_wu, m_x, m_wd, m_h;
    if (!encode_fn()) return BEAM_MOE_ERR_CUDA;
    if (!make_map_3d(&m_wg, w_gate, hidden, inter, 1) || !make_map_3d(&m_wu, w_up, hidden, inter, 1) ||
        !make_map_2d(&m_x, x, hidden, static_cast<uint64_t>(T), k2smBox) ||
        !make_map_3d(&m_wd, w_down, inter, hidden, 1) ||
        !make_map_2d(&m_h, h, inter, static_cast<uint64_t>(T), kWideBox))
        return BEAM_MOE_ERR_CUDA;
    const int grid = g_dev[dev].num_sms;
    GemmParams p1{counts, offsets, h, 1, hidden, inter, 0, kDefaultTimeoutCycles, nullptr, 1};
    // the down projection's rows, rounded to bf16, are the output: one token-ordered expert needs no combine
    GemmParams p2{counts, offsets, y, 1, inter, hidden, 0, kDefaultTimeoutCycles, nullptr, 1, nullptr, 1};
    launch_gemm2<G1_2SM_BIG_ARGS>(g_dev[dev].pairs_g1b, s, m_wg, m_wu, m_x, p1);
    if ((rc = launch_status())) return rc;
    launch_gemm<G2_PAIR_ARGS>(grid, s, m_wd, m_wd, m_h, p2);
    return launch_status();
}

// ------------------------------------------------------------------------------------------------
// beam_moe_permute_noalloc: the dispatch with its scratch in a fixed device array instead of a
// caller-provided workspace, for callers that must not allocate device memory.
namespace beam {
namespace {

// Per-chunk expert counts of the dispatch: ceil(T / 256) * n_experts ints at most.  One copy per
// device that loads the library, held until the process exits.
static __device__ __align__(256) int32_t g_noalloc_scratch[BEAM_MOE_NOALLOC_SCRATCH_INTS];

struct NoallocSlot {
    std::mutex mu;
    std::atomic<int32_t *> ptr{nullptr};  // device address of g_noalloc_scratch on this device
};
NoallocSlot g_noalloc[kMaxDevices];

// Resolves the array's device address for the current device `dev` (the name g_noalloc_scratch in
// host code only stands in for the symbol; kernels get this address).  Only a successful lookup is
// kept: after a failure (for example a first call made during stream capture) the next call tries
// again.
int noalloc_scratch(int dev, int32_t **out) {
    NoallocSlot &s = g_noalloc[dev];
    int32_t *p = s.ptr.load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(s.mu);
        p = s.ptr.load(std::memory_order_relaxed);
        if (!p) {
            void *addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) {
                cudaGetLastError();  // clear this error so that a later launch check does not report it
                return BEAM_MOE_ERR_CUDA;
            }
            p = static_cast<int32_t *>(addr);
            s.ptr.store(p, std::memory_order_release);
        }
    }
    *out = p;
    return BEAM_MOE_OK;
}

}  // namespace
}  // namespace beam

extern "C" {

int beam_moe_permute_noalloc(const beam_moe_config *cfg, int64_t T, const int32_t *topk_ids, int32_t *counts,
                             int64_t *offsets, int32_t *row_src, int32_t *dest_row, void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (n_chunks(T) * cfg->n_experts > BEAM_MOE_NOALLOC_SCRATCH_INTS) return BEAM_MOE_ERR_INVALID_ARG;
    if (!counts || !offsets || (T > 0 && (!topk_ids || !row_src || !dest_row))) return BEAM_MOE_ERR_NULL;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    int32_t *scratch = nullptr;
    if ((rc = noalloc_scratch(dev, &scratch))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, s) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int64_t) * (cfg->n_experts + 1), s) != cudaSuccess)
            return BEAM_MOE_ERR_CUDA;
        return BEAM_MOE_OK;
    }
    // the histogram kernel writes every scratch entry the scan then reads: nothing to clear
    return enqueue_permute(cfg, T, topk_ids, counts, offsets, row_src, dest_row, scratch, s);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Expert-parallel building blocks: the gather of token rows into dispatch order, the experts on
// rows that arrive already dispatched (each row with one local expert id, FP32 outputs in the rows'
// own order), and the weighted combine of dispatch-ordered FP32 expert outputs.  Together with
// route and permute they are the steps of one rank of an expert-parallel layer whose exchanges
// (all-to-all of token rows and of expert outputs) the caller makes.
namespace beam {
namespace {

struct RowsLayout {
    size_t hist = 0, counts = 0, offsets = 0, row_src = 0, dest_row = 0, xp = 0, h = 0, total = 0;
};

bool rows_shape_ok(int32_t H, int32_t I, int32_t E) {
    return H >= 64 && H <= 65536 && H % 64 == 0 && I >= 64 && I <= 65536 && I % 64 == 0 && E >= 1 && E <= 256;
}

// Rows per expert decide the tile family as in the forward pass (k = 1: one row per "token").
bool rows_narrow(int32_t E, int64_t R) { return static_cast<double>(R) / E <= 12.0; }

RowsLayout rows_layout(int32_t H, int32_t I, int32_t E, int64_t R) {
    RowsLayout L;
    if (R == 0) return L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align256(off + bytes);
        return at;
    };
    L.hist = take(static_cast<size_t>(n_chunks(R)) * E * 4);
    L.counts = take(static_cast<size_t>(E) * 4);
    L.offsets = take((static_cast<size_t>(E) + 1) * 8);
    L.row_src = take(static_cast<size_t>(R) * 4);
    L.dest_row = take(static_cast<size_t>(R) * 4);
    if (!rows_narrow(E, R)) L.xp = take(static_cast<size_t>(R) * H * 2);
    L.h = take(static_cast<size_t>(R) * I * 2);
    L.total = off;
    return L;
}

}  // namespace
}  // namespace beam

extern "C" {

int beam_moe_gather_rows(const beam_moe_config *cfg, int64_t T, const beam_bf16 *x, const int32_t *dest_row,
                         beam_bf16 *x_rows, void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!x || !dest_row || !x_rows) return BEAM_MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(x_rows)) return BEAM_MOE_ERR_MISALIGNED;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    gather_rows_kernel<<<static_cast<unsigned>(T), 128, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(x), T, cfg->topk, cfg->hidden / 8, dest_row, reinterpret_cast<uint4 *>(x_rows));
    return launch_status();
}

size_t beam_moe_expert_rows_workspace_size(int32_t hidden, int32_t inter, int32_t n_experts, int64_t R) {
    if (!rows_shape_ok(hidden, inter, n_experts) || R < 0 || R > kMaxTokens) return 0;
    return rows_layout(hidden, inter, n_experts, R).total;
}

int beam_moe_expert_rows(int32_t hidden, int32_t inter, int32_t n_experts, int64_t R, const beam_bf16 *x_rows,
                         const int32_t *row_expert, const beam_bf16 *w_gate, const beam_bf16 *w_up,
                         const beam_bf16 *w_down, float *o_rows, void *ws, size_t ws_bytes, void *stream) {
    if (!rows_shape_ok(hidden, inter, n_experts)) return BEAM_MOE_ERR_INVALID_CONFIG;
    if (R < 0 || R > kMaxTokens) return BEAM_MOE_ERR_INVALID_ARG;
    if (R == 0) return BEAM_MOE_OK;
    if (!x_rows || !row_expert || !w_gate || !w_up || !w_down || !o_rows || !ws) return BEAM_MOE_ERR_NULL;
    if (!aligned16(x_rows) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(o_rows) ||
        !aligned16(ws))
        return BEAM_MOE_ERR_MISALIGNED;
    const RowsLayout L = rows_layout(hidden, inter, n_experts, R);
    if (ws_bytes < L.total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    int dev, rc;
    if ((rc = init_device(&dev))) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    int32_t *counts = reinterpret_cast<int32_t *>(wsb + L.counts);
    int64_t *offsets = reinterpret_cast<int64_t *>(wsb + L.offsets);
    int32_t *row_src = reinterpret_cast<int32_t *>(wsb + L.row_src);
    int32_t *dest_row = reinterpret_cast<int32_t *>(wsb + L.dest_row);
    // each row is a "token" with one expert: the dispatch groups rows by expert, rows in order
    beam_moe_config c1{hidden, inter, n_experts, 1, 1, 1, 1, 1.0f};
    if ((rc = enqueue_permute(&c1, R, row_expert, counts, offsets, row_src, dest_row,
                              reinterpret_cast<int32_t *>(wsb + L.hist), s)))
        return rc;
    const bool narrow = rows_narrow(n_experts, R);
    if (!narrow) {
        gather_rows_kernel<<<static_cast<unsigned>(R), 128, 0, s>>>(reinterpret_cast<const uint4 *>(x_rows), R, 1,
                                                                    hidden / 8, dest_row,
                                                                    reinterpret_cast<uint4 *>(wsb + L.xp));
        if ((rc = launch_status())) return rc;
    }
    const int box = narrow ? kNarrowBox : k2smBox;
    const int bn = narrow ? kNarrowBN : kWideBN;
    const double mean_rows = static_cast<double>(R) / n_experts;
    const int once = (mean_rows + 4.0 * std::sqrt(mean_rows) <= bn) ? 1 : 0;
    CUtensorMap m_wg, m_wu, m_b1, m_wd, m_h;
    if (!encode_fn()) return BEAM_MOE_ERR_CUDA;
    const bool b1_ok = narrow ? make_map_2d(&m_b1, x_rows, hidden, static_cast<uint64_t>(R), 1)
                              : make_map_2d(&m_b1, wsb + L.xp, hidden, static_cast<uint64_t>(R), box);
    if (!b1_ok || !make_map_3d(&m_wg, w_gate, hidden, inter, n_experts) ||
        !make_map_3d(&m_wu, w_up, hidden, inter, n_experts) || !make_map_3d(&m_wd, w_down, inter, hidden, n_experts) ||
        !make_map_2d(&m_h, wsb + L.h, inter, static_cast<uint64_t>(R), box))
        return BEAM_MOE_ERR_CUDA;
    const int grid = g_dev[dev].num_sms;
    GemmParams p1{counts, offsets, wsb + L.h, n_experts, hidden, inter, once, kDefaultTimeoutCycles, row_src, 1,
                  nullptr};
    // the down projection stores dispatch row r at the caller's row row_src[r] (k = 1)
    GemmParams p2{counts, offsets, o_rows, n_experts, inter, hidden, once, kDefaultTimeoutCycles, nullptr, 1, row_src};
    if (narrow) launch_gemm<G1_NARROW_ARGS>(grid, s, m_wg, m_wu, m_b1, p1);
    else if (once) launch_gemm2<G1_2SM_ARGS>(g_dev[dev].pairs_g1, s, m_wg, m_wu, m_b1, p1);
    else launch_gemm2<G1_2SM_BIG_ARGS>(g_dev[dev].pairs_g1b, s, m_wg, m_wu, m_b1, p1);
    if ((rc = launch_status())) return rc;
    if (narrow) launch_gemm<G2_NARROW_ARGS>(grid, s, m_wd, m_wd, m_h, p2);
    else if (once) launch_gemm2<G2_2SM_ARGS>(g_dev[dev].pairs_g2, s, m_wd, m_wd, m_h, p2);
    else launch_gemm2<G2_2SM_BIG_ARGS>(g_dev[dev].pairs_g2b, s, m_wd, m_wd, m_h, p2);
    return launch_status();
}

int beam_moe_combine(const beam_moe_config *cfg, int64_t T, const float *o_rows, const int32_t *dest_row,
                     const float *topk_w, beam_bf16 *y, void *stream) {
    int rc = validate(cfg);
    if (rc) return rc;
    if ((rc = check_T(cfg, T))) return rc;
    if (T == 0) return BEAM_MOE_OK;
    if (!o_rows || !dest_row || !topk_w || !y) return BEAM_MOE_ERR_NULL;
    if (!aligned16(o_rows) || !aligned16(y)) return BEAM_MOE_ERR_MISALIGNED;
    int dev;
    if ((rc = init_device(&dev))) return rc;
    combine_kernel<<<static_cast<unsigned>(T), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const float4 *>(o_rows), dest_row, topk_w, T, cfg->topk, cfg->hidden / 4, cfg->routed_scale,
        reinterpret_cast<uint2 *>(y));
    return launch_status();
}

}  // extern "C"
