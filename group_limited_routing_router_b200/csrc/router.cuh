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
//     32 tokens x 128 experts per warp; W staged by cp.async and x widened from bf16 to fp32
//     (exact) in double-buffered shared memory.  Shared memory hands each lane about one float
//     per wavefront, so the register tile is sized for 5.3 FMAs per float read;
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

constexpr int kRtTok = 64;          // tokens per cluster tile
constexpr int kRtBK = 32;           // K per shared-memory stage
constexpr int kRtWPad = kRtBK + 2;  // padded W row (floats): conflict-free 8-byte reads across experts
constexpr int kRtThreads = 128;     // 4 warps
constexpr int kRtCluster = 8;       // CTAs per cluster (split-K factor)
constexpr int kRtSlots = 256;       // expert slots per tile (E <= 256)
constexpr int kRtWFloats = 2 * kRtSlots * kRtWPad;      // W stages [2][256][34]
constexpr int kRtXFloats = 2 * kRtBK * kRtTok;          // x stages [2][32][64]
constexpr int kRtSmemFloats = kRtWFloats + kRtXFloats;  // 21504 floats = 84 KB: two CTAs per SM
static_assert(kRtTok * kRtSlots <= kRtWFloats, "partial logits must fit in the W staging area");

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

__device__ __forceinline__ void cp_async8(void *smem, const void *gmem, bool valid) {
    // 8-byte global -> shared copy that bypasses registers; zero-fills when !valid
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(valid ? 8 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Insert v into the descending pair (a1 >= a2).
__device__ __forceinline__ void top2_insert(float &a1, float &a2, float v) {
    a2 = fmaxf(a2, fminf(a1, v));
    a1 = fmaxf(a1, v);
}

__global__ void __cluster_dims__(kRtCluster, 1, 1) __launch_bounds__(kRtThreads, 2)
    router_topk_kernel(const RouterParams p) {
    extern __shared__ float4 rt_smem4[];
    float *smem = reinterpret_cast<float *>(rt_smem4);
    float *ws = smem;                 // [2][kRtSlots][kRtWPad]  (expert-major, k contiguous)
    float *xs = smem + kRtWFloats;    // [2][kRtBK][kRtTok]      (k-major, tokens contiguous)
    float *part = smem;               // [kRtTok][kRtSlots] after the K loop

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int64_t t0 = static_cast<int64_t>(blockIdx.x / kRtCluster) * kRtTok;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    // warp tile: tokens 32*(warp&1) + [0,32) x experts 128*(warp>>1) + [0,128); lane (a = lane>>3,
    // b = lane&7) owns tokens tok0 + i (i < 8) and experts exp0 + 8j (j < 16).  W reads: 8 distinct
    // rows per half-warp, 34 floats apart -> distinct banks; x reads: one address per quarter-warp.
    const int tok0 = 32 * (warp & 1) + 8 * (lane >> 3);
    const int exp0 = 128 * (warp >> 1) + (lane & 7);

    // ---- split-K FP32 projection --------------------------------------------------------------
    const int nsteps = p.H / kRtBK;
    const int s_begin = rank * nsteps / kRtCluster;
    const int s_end = (rank + 1) * nsteps / kRtCluster;

    float acc[8][16];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[i][j] = 0.0f;

    // x stage: 64 tokens x 32 k bf16 = 256 chunks of 8 bf16; chunk c = tid + 128*h (h < 2) holds
    // token c & 63, k-offset (c >> 6) * 8
    uint4 xreg[2];
    auto x_load = [&](int s) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = tid + kRtThreads * h;
            const int xt = c & 63, xc = (c >> 6) * 8;
            const bool ok = (t0 + xt) < p.T;
            xreg[h] = ok ? __ldg(reinterpret_cast<const uint4 *>(p.x + (t0 + xt) * static_cast<int64_t>(p.H) +
                                                                 s * kRtBK + xc))
                         : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto x_store = [&](int buf) {
        float *xsb = xs + buf * kRtBK * kRtTok;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = tid + kRtThreads * h;
            const int xt = c & 63, xc = (c >> 6) * 8;
            const uint32_t xw[4] = {xreg[h].x, xreg[h].y, xreg[h].z, xreg[h].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // bf16 -> fp32 is a 16-bit shift of the bit pattern (exact)
                xsb[(xc + 2 * i) * kRtTok + xt] = __uint_as_float(xw[i] << 16);
                xsb[(xc + 2 * i + 1) * kRtTok + xt] = __uint_as_float(xw[i] & 0xffff0000u);
            }
        }
    };
    // W stage: thread t copies rows t and t+128 (32 floats each) as 8-byte chunks; rows are 34 floats
    // apart in shared memory, so every destination is 8-byte aligned
    const bool w_ok0 = tid < p.E, w_ok1 = tid + kRtThreads < p.E;
    const float *wrow0 = p.w + static_cast<int64_t>(w_ok0 ? tid : 0) * p.H;
    const float *wrow1 = p.w + static_cast<int64_t>(w_ok1 ? tid + kRtThreads : 0) * p.H;
    auto w_async = [&](int s, int buf) {
        float *dst0 = ws + buf * kRtSlots * kRtWPad + tid * kRtWPad;
        float *dst1 = dst0 + kRtThreads * kRtWPad;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            cp_async8(dst0 + 2 * i, wrow0 + s * kRtBK + 2 * i, w_ok0);
            cp_async8(dst1 + 2 * i, wrow1 + s * kRtBK + 2 * i, w_ok1);
        }
        cp_async_commit();
    };

    if (s_begin < s_end) {
        w_async(s_begin, 0);
        x_load(s_begin);
        x_store(0);
        cp_async_wait_all();
        __syncthreads();
        for (int s = s_begin; s < s_end; ++s) {
            const int buf = (s - s_begin) & 1;
            if (s + 1 < s_end) {
                w_async(s + 1, buf ^ 1);
                x_load(s + 1);
            }
            const float *wsb = ws + buf * kRtSlots * kRtWPad + exp0 * kRtWPad;
            const float *xsb = xs + buf * kRtBK * kRtTok + tok0;
#pragma unroll 2
            for (int kp = 0; kp < kRtBK / 2; ++kp) {
                float2 wv[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    wv[j] = *reinterpret_cast<const float2 *>(wsb + 8 * j * kRtWPad + 2 * kp);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const float4 xa = *reinterpret_cast<const float4 *>(xsb + (2 * kp + kk) * kRtTok);
                    const float4 xb = *reinterpret_cast<const float4 *>(xsb + (2 * kp + kk) * kRtTok + 4);
                    const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float wj = kk == 0 ? wv[j].x : wv[j].y;
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i][j] = fmaf(xv[i], wj, acc[i][j]);
                    }
                }
            }
            if (s + 1 < s_end) x_store(buf ^ 1);
            cp_async_wait_all();
            __syncthreads();
        }
    }

    // partial logits -> shared memory (the staging buffers are free after the last barrier)
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 16; ++j) part[(tok0 + i) * kRtSlots + exp0 + 8 * j] = acc[i][j];
    cluster.sync();

    // ---- reduction over the cluster + selection: warp w owns tokens 8*rank + w and 8*rank + w + 4
    const int per = p.E / p.G;
#define EID(j) (lane + 32 * (j))
    for (int u = 0; u < 2; ++u) {
        const int tt = rank * 8 + warp + 4 * u;
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
            sel[j] = (e < p.E) ? (p.bias ? s + p.bias[e] : s) : -INFINITY;
        }

        // group scores: sum of the group's top group_topn selection values, in pick order
        float my_gs = -INFINITY;  // lane g < G holds group g's score
        if (p.group_topn == 2 && p.G <= 8) {
            // all groups at once: lane-local top-2 per group, then a butterfly merge of the pairs
            // (the top-2 of a union is the top-2 of the parts' top-2s; ties do not change the sum)
            float t1[8], t2[8];
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                t1[g] = -INFINITY;
                t2[g] = -INFINITY;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (EID(j) < p.E && EID(j) / per == g) top2_insert(t1[g], t2[g], sel[j]);
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
#pragma unroll
            for (int g = 0; g < 8; ++g)
                if (lane == g && g < p.G) my_gs = t1[g] + t2[g];
        } else {
            uint32_t taken = 0;
            for (int g = 0; g < p.G; ++g) {
                float total = 0.0f;
                for (int r = 0; r < p.group_topn; ++r) {
                    float bv = -INFINITY;
                    int bi = 0x7fffffff;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const bool cand = EID(j) < p.E && !((taken >> j) & 1u) && (EID(j) / per) == g;
                        if (cand && (sel[j] > bv || (sel[j] == bv && EID(j) < bi))) {
                            bv = sel[j];
                            bi = EID(j);
                        }
                    }
                    const ArgMax m = warp_argmax(bv, bi);
                    total = total + m.v;
                    if ((m.i & 31) == lane) taken |= 1u << (m.i >> 5);
                }
                if (lane == g) my_gs = total;
            }
        }
        // keep the topk_groups best groups (lower group index on ties)
        uint32_t kept = 0;
        for (int r = 0; r < p.topk_groups; ++r) {
            const bool cand = lane < p.G && !((kept >> lane) & 1u);
            const ArgMax m = warp_argmax(cand ? my_gs : -INFINITY, cand ? lane : 0x7fffffff);
            kept |= 1u << m.i;
        }
        // topk experts inside the kept groups, in pick order (descending selection value)
        uint32_t taken = 0;
        float den = 0.0f, my_s = 0.0f;
        int my_id = 0;
        for (int r = 0; r < p.topk; ++r) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const bool cand = EID(j) < p.E && !((taken >> j) & 1u) && ((kept >> (EID(j) / per)) & 1u);
                if (cand && (sel[j] > bv || (sel[j] == bv && EID(j) < bi))) {
                    bv = sel[j];
                    bi = EID(j);
                }
            }
            const ArgMax m = warp_argmax(bv, bi);
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
        }
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
