// Router kernel R: FP32 router projection + sigmoid + group-limited top-k + weight normalisation.
//
// Beam launch post ("Welcome Beam" page, section "Mixture of Experts"): the router scores all
// experts with a sigmoid, splits them into groups, keeps the best groups ranked by the sum of
// each group's top-2 scores, then picks the top experts inside them; outputs are combined with
// normalised router weights.  Section "Residual Stream": the router computes in FP32.
//
// Layout of the work (sm_100a):
//   * one thread-block cluster of 8 CTAs per tile of 64 tokens; CTA r of the cluster computes the
//     partial logits of all 64 tokens x 256 expert slots over the r-th eighth of the hidden
//     dimension (split-K).  128 threads, 8 tokens x 16 experts of FP32 accumulators per thread,
//     32 tokens x 128 experts per warp.  W (fp32) and x (bf16) tiles arrive by TMA into a 3-stage
//     mbarrier pipeline (one thread issues two bulk copies per stage, so the compute warps issue
//     no staging instructions); x is widened from bf16 to fp32 (exact) in registers;
//   * the partial logits stay in each CTA's shared memory; after a cluster barrier, CTA r reduces
//     tokens [8r, 8r+8) over the 8 CTAs through distributed shared memory, in rank order, so the
//     FP32 sum order is fixed (deterministic);
//   * one warp per token then does the selection with warp shuffles: lane l owns experts
//     l, l+32, ...; every (value, index) comparison breaks ties toward the lower index and every
//     sum is taken in a fixed order (group score = top1 + top2; weight denominator in slot order).
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace beam {

namespace cg = cooperative_groups;

constexpr int kRtTok = 64;        // tokens per cluster tile (kRtTokSmall for small batches)
constexpr int kRtTokSmall = 16;
constexpr int kRtTokTiny = 8;
constexpr int kRtBK = 32;         // K per pipeline stage (one 128-byte row of fp32 W)
constexpr int kRtThreads = 128;   // 4 warps
constexpr int kRtCluster = 8;     // CTAs per cluster (split-K factor)
constexpr int kRtSlots = 256;     // expert slots per tile (E <= 256)
constexpr int kRtStages = 3;      // TMA pipeline depth
constexpr int kRtWBytes = kRtSlots * kRtBK * 4;  // W stage: [256 rows][32 fp32], 128-byte swizzle (32 KB)
// x stage: [TOK rows][32 bf16], 64-byte swizzle (TOK * 64 bytes)
constexpr int rt_stage_bytes(int tok) { return (kRtWBytes + tok * kRtBK * 2 + 1023) / 1024 * 1024; }
// + alignment + barriers: two CTAs per SM
constexpr int rt_smem_bytes(int tok) { return 1024 + kRtStages * rt_stage_bytes(tok) + 128; }
static_assert(kRtTok * kRtSlots * 4 <= kRtStages * rt_stage_bytes(kRtTok), "partial logits must fit in the stages");
static_assert(rt_stage_bytes(kRtTok) % 1024 == 0 && rt_stage_bytes(kRtTokTiny) % 1024 == 0,
              "stages keep the 1024-byte swizzle alignment");
static_assert(kRtTokTiny * kRtSlots * 4 <= kRtStages * rt_stage_bytes(kRtTokTiny), "partial logits fit");

struct RouterParams {
    const __nv_bfloat16 *x;  // [T, H]
    const float *w;          // [E, H]
    const float *bias;       // [E] or nullptr
    int32_t *ids;            // [T, k]
    float *wts;              // [T, k]
    int64_t T;
    int H, E, G, topk_groups, topk, group_topn;
};

struct ArgMax {
    float v;
    int i;
};

// Warp-wide argmax of (value desc, index asc); every lane gets the winner.
__device__ __forceinline__ ArgMax warp_argmax(float v, int i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
    return {v, i};
}

// An order-preserving 32-bit key of a value that is not NaN (-inf lowest; -0.0 and +0.0 share a key),
// and its inverse: warp max / min reductions (redux.sync) on keys rank values as float comparisons do.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// warp_argmax with two redux.sync reductions: the largest key, then the lowest index holding it.
__device__ __forceinline__ ArgMax warp_argmax_redux(float v, int i) {
    const uint32_t k = order_key(v);
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, k);
    const uint32_t imin = __reduce_min_sync(0xffffffffu, k == kmax ? static_cast<uint32_t>(i) : 0xffffffffu);
    return {key_value(kmax), static_cast<int>(imin)};
}

// Insert v into the descending pair (a1 >= a2).
__device__ __forceinline__ void top2_insert(float &a1, float &a2, float v) {
    a2 = fmaxf(a2, fminf(a1, v));
    a1 = fmaxf(a1, v);
}

// Group-limited selection for one token, done by one warp.  Lane l holds the scores sc[j] and selection
// values sel[j] (score + bias; -inf for masked or NaN) of experts l + 32 j.  On return lanes r < topk
// hold the r-th pick (descending selection value, lower index first on ties): my_id and its score
// my_s; den is the sum of the picked scores in pick order (every lane).  With margins != nullptr,
// margins[0] = the last kept group's score - the best dropped group's score and margins[1] = the last
// picked expert's selection value - the best one left in the kept groups (+inf where nothing is left;
// NaN where only -inf values compete); every lane gets them.
__device__ __forceinline__ void select_group_limited(const float (&sc)[8], const float (&sel)[8], int lane, int E,
                                                     int G, int topk_groups, int topk, int group_topn, int &my_id,
                                                     float &my_s, float &den, float *margins) {
    const int per = E / G;
#define EID(j) (lane + 32 * (j))
    int grp[8];  // group of expert EID(j), -1 past E
#pragma unroll
    for (int j = 0; j < 8; ++j) grp[j] = EID(j) < E ? EID(j) / per : -1;
    // ---- group scores (sum of the group's top group_topn selection values, in pick order) and the kept
    // groups (topk_groups best, lower group index first on ties)
    uint32_t kept = 0;
    float last_gs = INFINITY, next_gs = -INFINITY;
    if (group_topn == 2 && G <= 8) {
        // all groups at once: lane-local top-2 per group, then a butterfly merge of the pairs (the
        // top-2 of a union is the top-2 of the parts' top-2s; ties do not change the sum); every lane
        // ends with every group's score and ranks the groups itself
        float t1[8], t2[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            t1[g] = -INFINITY;
            t2[g] = -INFINITY;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (grp[j] == g) top2_insert(t1[g], t2[g], sel[j]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const float o1 = __shfl_xor_sync(0xffffffffu, t1[g], off);
                const float o2 = __shfl_xor_sync(0xffffffffu, t2[g], off);
                top2_insert(t1[g], t2[g], o1);
                top2_insert(t1[g], t2[g], o2);
            }
        float gs[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) gs[g] = t1[g] + t2[g];
        for (int r = 0; r <= topk_groups && r < G; ++r) {
            float bv = -INFINITY;
            int bg = -1;
#pragma unroll
            for (int g = 0; g < 8; ++g)
                if (g < G && !((kept >> g) & 1u) && (bg < 0 || gs[g] > bv)) {
                    bv = gs[g];
                    bg = g;
                }
            if (r == topk_groups) {
                next_gs = bv;  // the best dropped group
            } else {
                kept |= 1u << bg;
                last_gs = bv;
            }
        }
    } else {
        float my_gs = -INFINITY;  // lane g < G holds group g's score
        uint32_t taken = 0;
        for (int g = 0; g < G; ++g) {
            float total = 0.0f;
            for (int r = 0; r < group_topn; ++r) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const bool cand = grp[j] == g && !((taken >> j) & 1u);
                    if (cand && (sel[j] > bv || (sel[j] == bv && EID(j) < bi))) {
                        bv = sel[j];
                        bi = EID(j);
                    }
                }
                const ArgMax m = warp_argmax_redux(bv, bi);
                total = total + m.v;
                if ((m.i & 31) == lane) taken |= 1u << (m.i >> 5);
            }
            if (lane == g) my_gs = total;
        }
        for (int r = 0; r <= topk_groups && r < G; ++r) {
            const bool cand = lane < G && !((kept >> lane) & 1u);
            const ArgMax m = warp_argmax_redux(cand ? my_gs : -INFINITY, cand ? lane : 0x7fffffff);
            if (r == topk_groups) {
                next_gs = m.v;
            } else {
                kept |= 1u << m.i;
                last_gs = m.v;
            }
        }
    }
    if (margins) margins[0] = topk_groups < G ? last_gs - next_gs : INFINITY;
    // ---- topk experts inside the kept groups, in pick order (descending selection value)
    uint32_t taken = 0;
    float last_sel = -INFINITY;
    den = 0.0f;
    my_s = 0.0f;
    my_id = 0;
    for (int r = 0; r < topk; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool cand = grp[j] >= 0 && !((taken >> j) & 1u) && ((kept >> grp[j]) & 1u);
            if (cand && (sel[j] > bv || (sel[j] == bv && EID(j) < bi))) {
                bv = sel[j];
                bi = EID(j);
            }
        }
        const ArgMax m = warp_argmax_redux(bv, bi);
        float s_owner = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j == (m.i >> 5)) s_owner = sc[j];
        if ((m.i & 31) == lane) taken |= 1u << (m.i >> 5);
        const float s = __shfl_sync(0xffffffffu, s_owner, m.i & 31);
        den = den + s;
        if (lane == r) {
            my_id = m.i;
            my_s = s;
        }
        last_sel = m.v;
    }
    if (margins) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool cand = grp[j] >= 0 && !((taken >> j) & 1u) && ((kept >> grp[j]) & 1u);
            if (cand && (sel[j] > bv || (sel[j] == bv && EID(j) < bi))) {
                bv = sel[j];
                bi = EID(j);
            }
        }
        const ArgMax m = warp_argmax_redux(bv, bi);
        margins[1] = m.i == 0x7fffffff ? INFINITY : last_sel - m.v;
    }
#undef EID
}

// TOK tokens per cluster tile: 64 (8 per thread), or 16 or 8 (2 or 1 per thread) so that small batches
// still spread over most of the SMs.
template <int TOK>
__global__ void __cluster_dims__(kRtCluster, 1, 1) __launch_bounds__(kRtThreads, 2)
    router_topk_kernel(const __grid_constant__ CUtensorMap tm_w,  // W_r [E][H] fp32, box {32, 256}
                       const __grid_constant__ CUtensorMap tm_x,  // x [T][H] bf16, box {32, 64}
                       const RouterParams p) {
    extern __shared__ uint8_t rt_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rt_smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kRtStageBytes = rt_stage_bytes(TOK);  // stage stride (1024-byte aligned)
    constexpr int kTi = TOK / 8;  // tokens per thread
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRtStages * kRtStageBytes);
    uint64_t *empty = full + kRtStages;
    float *part = reinterpret_cast<float *>(smem);  // [TOK][kRtSlots] after the K loop

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int64_t t0 = static_cast<int64_t>(blockIdx.x / kRtCluster) * TOK;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    // warp tile: tokens (TOK/2)*(warp&1) + [0,TOK/2) x experts 128*(warp>>1) + [0,128).  Lane
    // (a = lane>>3, b = lane&7) owns tokens tokA + 4i (i < TOK/8) and experts expB + 8j (j < 16).
    const int a = lane >> 3, b = lane & 7;
    const int tokA = (TOK / 2) * (warp & 1) + a;
    const int expB = 128 * (warp >> 1) + b;

    // ---- split-K FP32 projection --------------------------------------------------------------
    const int nsteps = p.H / kRtBK;
    const int s_begin = rank * nsteps / kRtCluster;
    const int s_end = (rank + 1) * nsteps / kRtCluster;
    const int n_my = s_end - s_begin;

    if (tid == 0) {
        for (int i = 0; i < kRtStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kRtThreads / 32);
        }
        fence_mbar_init();
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
    }
    __syncthreads();
    auto issue = [&](int i) {  // load step s_begin + i into stage i % kRtStages
        uint8_t *st = smem + (i % kRtStages) * kRtStageBytes;
        const int k0 = (s_begin + i) * kRtBK;
        mbar_arrive_expect_tx(&full[i % kRtStages], kRtWBytes + TOK * kRtBK * 2);  // the bytes the two copies land
        tma_load_2d(st, &tm_w, &full[i % kRtStages], k0, 0, policy_evict_last());
        tma_load_2d(st + kRtWBytes, &tm_x, &full[i % kRtStages], k0, static_cast<int>(t0), policy_evict_first());
    };
    int n_issued = 0;  // meaningful in thread 0
    if (tid == 0)
        for (; n_issued < kRtStages && n_issued < n_my; ++n_issued) issue(n_issued);

    float acc[kTi][16];
#pragma unroll
    for (int i = 0; i < kTi; ++i)
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[i][j] = 0.0f;

    // Every wait below is taken by all 32 lanes of a warp and its outcome made warp-uniform, so the
    // warps stay converged; a timeout (status word set) stops the loop.
    bool ok = true;
    int i = 0;
    for (; i < n_my && ok; ++i) {
        const int st = i % kRtStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[st], (i / kRtStages) & 1u, kDefaultTimeoutCycles));
        if (!ok) break;
        const uint8_t *wsb = smem + st * kRtStageBytes;
        const uint8_t *xsb = wsb + kRtWBytes;
#pragma unroll 2
        for (int kp = 0; kp < kRtBK / 2; ++kp) {
            // W row r (r & 7 == b), fp32 k = 2kp, 2kp+1: 16-byte chunk (kp>>1) ^ b of the 128-byte row
            const int woff = ((((kp >> 1) ^ b) << 4) | ((kp & 1) << 3));
            float2 wv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                wv[j] = *reinterpret_cast<const float2 *>(wsb + (expB + 8 * j) * 128 + woff);
            // x row t, bf16 pair k = 2kp, 2kp+1: 16-byte chunk (kp>>2) ^ ((t>>1)&3) of the 64-byte row
            uint32_t xp[kTi];
#pragma unroll
            for (int i2 = 0; i2 < kTi; ++i2) {
                const int t = tokA + 4 * i2;
                xp[i2] = *reinterpret_cast<const uint32_t *>(
                    xsb + t * 64 + ((((kp >> 2) ^ ((t >> 1) & 3)) << 4) | ((kp & 3) << 2)));
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float wj = kk == 0 ? wv[j].x : wv[j].y;
#pragma unroll
                    for (int i2 = 0; i2 < kTi; ++i2) {
                        // bf16 -> fp32 is a 16-bit shift of the bit pattern (exact)
                        const float xv = __uint_as_float(kk == 0 ? (xp[i2] << 16) : (xp[i2] & 0xffff0000u));
                        acc[i2][j] = fmaf(xv, wj, acc[i2][j]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
        // warp 0 refills this stage with the step kRtStages ahead once every warp has released it
        if (warp == 0 && i + kRtStages < n_my) {
            ok = __all_sync(0xffffffffu, mbar_wait(&empty[st], (i / kRtStages) & 1u, kDefaultTimeoutCycles));
            if (ok && lane == 0) {
                issue(i + kRtStages);
                ++n_issued;
            }
            __syncwarp();
        }
    }
    // after a timeout, let this CTA's in-flight copies land before its shared memory is reused
    if (tid == 0)
        for (int q = i; q < n_issued; ++q) mbar_wait(&full[q % kRtStages], (q / kRtStages) & 1u, kDefaultTimeoutCycles);
    __syncthreads();

    // partial logits -> shared memory
#pragma unroll
    for (int i = 0; i < kTi; ++i)
#pragma unroll
        for (int j = 0; j < 16; ++j) part[(tokA + 4 * i) * kRtSlots + expB + 8 * j] = acc[i][j];
    cluster.sync();

    // ---- reduction over the cluster + selection: CTA rank takes tokens kTi*rank + [0, kTi), warp w
    // the tokens w and w + 4 among them
#define EID(j) (lane + 32 * (j))
    for (int u = 0; u < 2; ++u) {
        const int lt = warp + 4 * u;
        if (lt >= kTi) continue;
        const int tt = rank * kTi + lt;
        const int64_t t = t0 + tt;
        if (t >= p.T) continue;
        float sc[8], sel[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = EID(j);
            float logit = 0.0f;
            if (e < p.E) {
#pragma unroll
                for (int c = 0; c < kRtCluster; ++c) {
                    const float *rp = cluster.map_shared_rank(part, c);
                    logit += rp[tt * kRtSlots + e];
                }
            }
            const float s = 1.0f / (1.0f + expf(-logit));
            sc[j] = s;
            const float v = (p.bias && e < p.E) ? s + p.bias[e] : s;
            // a NaN (from NaN in x, W_r or the bias) ranks below every number, so the ids stay in [0, E)
            sel[j] = (e < p.E && v == v) ? v : -INFINITY;
        }

        float den, my_s;
        int my_id;
        select_group_limited(sc, sel, lane, p.E, p.G, p.topk_groups, p.topk, p.group_topn, my_id, my_s, den, nullptr);
        if (lane < p.topk) {
            p.ids[t * p.topk + lane] = my_id;
            p.wts[t * p.topk + lane] = my_s / den;
        }
    }
#undef EID
    // no CTA may leave while another still reads its shared memory
    cluster.sync();
}

}  // namespace beam
