// Screened router: the same routing as router_topk_kernel (bit for bit), with the 256-way projection
// screened on the tensor cores.
//
// Beam launch post ("Welcome Beam" page, section "Mixture of Experts": sigmoid scores, 8 groups of 32,
// the 4 groups with the best top-2 sums, the top 8 experts inside them, normalised weights; section
// "Residual Stream": the router computes in FP32).  The FP32 router spends its time on the projection
// x . W_r for all 256 experts, while only the 8 chosen experts' values enter the weights and only a
// narrow band of values decides the choice.  So:
//
//   1. router_split_kernel: W_r (fp32) = W_hi + W_mid + W_lo exactly, three bf16 planes (each keeps
//      the next 8 significant bits of the residual);
//   2. router_logits_kernel: l~[t, e] = sum over the three planes of x_t . W_p,e on tcgen05 (bf16
//      products are exact, accumulation in FP32 in the tensor core), K split S ways, partial sums
//      written per split;
//   3. router_screen_kernel (one warp per token): the selection on sigmoid(l~) with its two decision
//      margins (last kept group vs best dropped group; last picked expert vs best one left).  Where
//      both margins are at least kRsMargin, the chosen set is the one exact FP32 values give (the
//      screened values are within 2e-5 of them, so a set decided by more than 4 times that cannot
//      change).  Other tokens go to a list;
//   4. router_exact_kernel, one launch: the exact FP32 projections in the direct router's order (8 K
//      ranges, each a sequential fused multiply-add chain over ascending k, summed in rank order), for
//      the screened tokens' picks (the screen appends each pick to its expert's bucket; a CTA takes
//      an expert's picks 64 at a time, so the expert's row of W_r is staged once per 64 picks and
//      only the tokens' bf16 rows stream per pick) and, for the listed tokens (eight per CTA), onto
//      every expert;
//   5. router_finish_kernel: the screened tokens' picks ordered and normalised from their exact
//      projections, and the selection on the listed tokens' projections, as router_topk_kernel does.
// Every output therefore equals router_topk_kernel's.
#pragma once

#include "router.cuh"

namespace beam {

constexpr int kRsStages = 3;
constexpr int kRsThreads = 192;      // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue (TMEM lane quarters)
constexpr float kRsMargin = 2e-4f;   // decision margin below which a token takes the exact path
constexpr int kRsMaxSplit = 16;
constexpr int kRsMinTokens = 2048;  // smaller batches take the direct router

struct RouterTcParams {
    int64_t T;
    int H, E;
    int S;          // K splits
    int kps;        // 64-wide k-steps per split
    int n_nt;       // token tiles
    int n_mt;       // expert tiles of 128
    float *part;    // [S][T][E] partial projections
    long long timeout;
};

template <int BN>
struct RsCfg {
    static constexpr int kA = kBM * kBK * 2;    // one plane's expert tile: 128 rows x 64 bf16 (16 KB)
    static constexpr int kB = BN * kBK * 2;     // token tile: BN rows x 64 bf16
    static constexpr int kStage = 3 * kA + kB;
    static constexpr int kBarOff = kRsStages * kStage;
    static constexpr int kSmem = 1024 + kBarOff + 256;
    static constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;  // two accumulator slots of BN columns
    static_assert(kStage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(kSmem <= 232448, "shared memory per CTA");
};

// W_r [E][H] fp32 -> planes [3][E][H] bf16 with hi + mid + lo == W_r (each residual is exact in FP32).
__global__ void __launch_bounds__(256) router_split_kernel(const float4 *__restrict__ w, int64_t n4,
                                                           uint2 *__restrict__ planes) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 v = __ldg(w + i);
        const float a[4] = {v.x, v.y, v.z, v.w};
        uint32_t hi[2], mid[2], lo[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float p0[2], p1[2], p2[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float x0 = a[2 * h + q];
                p0[q] = __bfloat162float(__float2bfloat16_rn(x0));
                const float r1 = x0 - p0[q];
                p1[q] = __bfloat162float(__float2bfloat16_rn(r1));
                p2[q] = __bfloat162float(__float2bfloat16_rn(r1 - p1[q]));
            }
            hi[h] = pack_bf16x2(p0[0], p0[1]);
            mid[h] = pack_bf16x2(p1[0], p1[1]);
            lo[h] = pack_bf16x2(p2[0], p2[1]);
        }
        planes[i] = make_uint2(hi[0], hi[1]);
        planes[n4 + i] = make_uint2(mid[0], mid[1]);
        planes[2 * n4 + i] = make_uint2(lo[0], lo[1]);
    }
}

// Screened projection: item = (token tile nt, expert tile mt, K split s); part[s][t][e] = sum over the
// split's K range and the three planes, FP32 accumulation in TMEM.  Persistent CTAs, two accumulator
// slots so an item's epilogue overlaps the next item's products.
template <int BN>
__global__ void __launch_bounds__(kRsThreads, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap tm_w,  // planes [3][E][H] bf16, box {64, 128, 1}
                         const __grid_constant__ CUtensorMap tm_x,  // x [T][H] bf16, box {64, BN}
                         const RouterTcParams p) {
    using C = RsCfg<BN>;
    extern __shared__ uint8_t rs_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(rs_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + kRsStages;
    uint64_t *acc_full = empty + kRsStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = p.n_nt * p.n_mt * p.S;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRsStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_w);
        prefetch_tensormap(&tm_x);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            const uint64_t pol = policy_evict_last();  // planes and x are re-read by other items
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const int s = item % p.S, mt = (item / p.S) % p.n_mt, nt = item / (p.S * p.n_mt);
                for (int kb = 0; kb < p.kps; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + stage * C::kStage;
                    const int k0 = (s * p.kps + kb) * kBK;
                    mbar_arrive_expect_tx(&full[stage], C::kStage);
#pragma unroll
                    for (int pl = 0; pl < 3; ++pl) tma_load_3d(st + pl * C::kA, &tm_w, &full[stage], k0, mt * kBM, pl, pol);
                    tma_load_2d(st + 3 * C::kA, &tm_x, &full[stage], k0, nt * BN, pol);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == kRsStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < kRsStages; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_phase >> s) & 1u, p.timeout);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = umma_idesc_bf16(kBM, BN);
            int stage = 0;
            uint32_t phase = 0, uses = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const int slot = uses & 1;
                if (!mbar_wait(&acc_empty[slot], ((uses >> 1) & 1u) ^ 1u, p.timeout)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(slot * BN);
                for (int kb = 0; kb < p.kps; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.timeout)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * C::kStage);
                    const uint64_t db = umma_desc_sw128(sa + 3 * C::kA);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
                        for (int pl = 0; pl < 3; ++pl) {
                            const uint32_t accum = (kb > 0 || kk > 0 || pl > 0) ? 1u : 0u;
                            umma_bf16(d, umma_desc_sw128(sa + pl * C::kA) + 2 * kk, db + 2 * kk, idesc, accum);
                        }
                    umma_commit(&empty[stage]);
                    if (++stage == kRsStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&acc_full[slot]);
                ++uses;
            }
            umma_commit(drain);
            mbar_wait(drain, 0, p.timeout);
        }
    } else {
        // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 ----------------
        const int q = warp & 3;
        uint32_t uses = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            const int s = item % p.S, mt = (item / p.S) % p.n_mt, nt = item / (p.S * p.n_mt);
            const int slot = uses & 1;
            if (!mbar_wait(&acc_full[slot], (uses >> 1) & 1u, p.timeout)) break;
            tc_fence_after();
            const int e = mt * kBM + q * 32 + lane;
            const uint32_t t0 = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(slot * BN);
            float *out = p.part + static_cast<int64_t>(s) * p.T * p.E;
#pragma unroll 1
            for (int c = 0; c < BN; c += 16) {
                uint32_t r[16];
                tmem_ld16(t0 + c, r);
                tmem_ld_wait();
                if (e < p.E) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t t = static_cast<int64_t>(nt) * BN + c + j;
                        if (t < p.T) out[t * p.E + e] = __uint_as_float(r[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[slot]);
            ++uses;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// The direct router's K range of cluster rank r: 32-wide steps [r n / 8, (r + 1) n / 8), n = H / 32.
__device__ __forceinline__ void rank_range(int H, int r, int &k0, int &k1) {
    const int n = H / kRtBK;
    k0 = (r * n / kRtCluster) * kRtBK;
    k1 = ((r + 1) * n / kRtCluster) * kRtBK;
}

// ---- exact projections in router_topk_kernel's order -------------------------------------------------
// The direct router forms logit_e = ((p_0 + p_1) + ...) + p_7 with p_r = fma(x_k, w_k, ...) over the
// ascending k of rank r's range, from 0.  The kernels below keep exactly those chains; their operands
// are staged through shared memory 32 k per rank at a time, with coalesced 16-byte cp.async copies
// (double buffered), so each thread's chain reads its segment without uncoalesced global loads.

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kRsSegWords = 36;  // a 32-float segment padded to 36 words: 8 consecutive segments hit distinct banks
constexpr int kRsXWords = 20;    // a 32-bf16 segment (16 words) padded to 20

// 4 fused multiply-adds in k order: w (4 fp32) against x (4 bf16 in two words, low half first)
__device__ __forceinline__ float fma4(float4 w, uint2 x, float acc) {
    acc = fmaf(__uint_as_float(x.x << 16), w.x, acc);  // bf16 -> fp32: the bits move up 16 places (exact)
    acc = fmaf(__uint_as_float(x.x & 0xffff0000u), w.y, acc);
    acc = fmaf(__uint_as_float(x.y << 16), w.z, acc);
    return fmaf(__uint_as_float(x.y & 0xffff0000u), w.w, acc);
}

__device__ __forceinline__ float4 lds_f4(const uint32_t *base, int word) {
    return *reinterpret_cast<const float4 *>(base + word);
}
__device__ __forceinline__ uint2 lds_u2(const uint32_t *base, int word) {
    return *reinterpret_cast<const uint2 *>(base + word);
}

struct RouterSelParams {
    const __nv_bfloat16 *x;  // [T, H]
    const float *w;          // [E, H]
    const float *bias;       // [E] or nullptr
    int32_t *ids;            // [T, k]
    float *wts;              // [T, k]
    int64_t T;
    int H, E, G, topk_groups, topk, group_topn;
    int S;                   // splits in part
    const float *part;       // [S][T][E]
    int32_t *list;           // [T] tokens for the exact path
    int32_t *list_n;         // their count
    const float *exact;      // [T][E] exact projections of the listed tokens (by list position)
    int32_t *bcnt;           // [E] picks in each expert's bucket (zeroed before the screen)
    int32_t *bucket;         // [E][T] the screened picks t * topk + slot, per expert, in any order
    float *xlogit;           // [T][topk] exact projection of each screened pick
    uint8_t *listed;         // [T] 1: the token takes the exact path (written by the screen for every token)
};

// sigmoid score and selection value of expert e from its projection (as router_topk_kernel)
__device__ __forceinline__ void score_of(float logit, int e, const RouterSelParams &p, float &sc, float &sel) {
    const float s = 1.0f / (1.0f + expf(-logit));
    sc = s;
    const float v = (p.bias && e < p.E) ? s + p.bias[e] : s;
    sel = (e < p.E && v == v) ? v : -INFINITY;
}

// One warp per token: the selection on the screened projections.  A token decided by both margins
// keeps its picks in ids[t] and appends each to its expert's bucket (for exact_picks and
// router_finish_kernel); any other is listed for the exact path, flagged in listed[t], and its ids are
// marked -1.
__global__ void __launch_bounds__(256) router_screen_kernel(const RouterSelParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t t = blockIdx.x * 8LL + (threadIdx.x >> 5);
    if (t >= p.T) return;
    float sc[8], sel[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        float l = 0.0f;
        if (e < p.E) {
            float v[kRsMaxSplit];
#pragma unroll
            for (int s = 0; s < kRsMaxSplit; ++s)  // issue every split's load before summing them in order
                v[s] = s < p.S ? __ldg(p.part + (static_cast<int64_t>(s) * p.T + t) * p.E + e) : 0.0f;
#pragma unroll
            for (int s = 0; s < kRsMaxSplit; ++s)
                if (s < p.S) l += v[s];
        }
        score_of(l, e, p, sc[j], sel[j]);
    }
    float den, my_s, margins[2];
    int my_id;
    select_group_limited(sc, sel, lane, p.E, p.G, p.topk_groups, p.topk, p.group_topn, my_id, my_s, den, margins);
    const bool certain = margins[0] >= kRsMargin && margins[1] >= kRsMargin;  // NaN margins are not
    if (!certain && lane == 0) p.list[atomicAdd(p.list_n, 1)] = static_cast<int32_t>(t);
    if (lane == 0) p.listed[t] = certain ? 0 : 1;
    if (lane < p.topk) {
        p.ids[t * p.topk + lane] = certain ? my_id : -1;
        if (certain) {
            const int pos = atomicAdd(p.bcnt + my_id, 1);  // < T: a token picks an expert at most once
            p.bucket[static_cast<int64_t>(my_id) * p.T + pos] = static_cast<int32_t>(t * p.topk + lane);
        }
    }
}

// ---- exact path: one launch, two kinds of CTAs ------------------------------------------------------
// The first n_exact CTAs project the listed tokens onto every expert, eight tokens at a time
// (exact_batch); the rest (one per SM, persistent) take the screened picks expert by expert, 64 at a
// time (exact_picks).  Both stage their operands with a cp.async ring.

constexpr int kRsExactStages = 4;
constexpr int kRsExactW = 256 * kRsSegWords, kRsExactX = 8 * 8 * kRsXWords, kRsExactBuf = kRsExactW + kRsExactX;
constexpr int kRsExactWords = kRsExactStages * kRsExactBuf + 8 * 256;

constexpr int kRxPicks = 64;                      // picks per item
constexpr int kRxStages = 4;
constexpr int kRxX = 8 * kRxPicks * kRsXWords;    // x segments [rank][pick][20 words]: 16-byte reads of 8 lanes hit distinct banks
constexpr int kRxW = 8 * 32;                      // the expert's W_r segments [rank][32 fp32]
constexpr int kRxBuf = kRxX + kRxW;
constexpr int kRxWords = kRxStages * kRxBuf + 8 * kRxPicks + 2 * kRxPicks + kRtSlots + 1;

constexpr int kRsPathSmem = (kRxWords > kRsExactWords ? kRxWords : kRsExactWords) * 4;
static_assert(kRsPathSmem <= 232448, "shared memory per CTA");
static_assert(kRxBuf % 4 == 0 && kRxX % 4 == 0, "16-byte aligned staging");

__device__ __forceinline__ uint4 lds_u4(const uint32_t *base, int word) {
    return *reinterpret_cast<const uint4 *>(base + word);
}

// Persistent CTA `cta` of `n_ctas`: items (expert e, chunk c) = picks 64 c .. 64 c + 63 of e's bucket.
// Warp r runs rank r's chains; lane q the picks q and q + 32.  Per 32-k step the CTA stages the
// expert's eight W_r segments and the picks' eight x segments each; the rank sums go to xlogit in
// rank order, exactly as the direct router forms them.
__device__ __forceinline__ void exact_picks(const RouterSelParams &p, uint32_t *smem, int cta, int n_ctas) {
    float *partial = reinterpret_cast<float *>(smem + kRxStages * kRxBuf);  // [pick][rank]
    int32_t *rows = reinterpret_cast<int32_t *>(partial + 8 * kRxPicks);    // token of each pick
    int32_t *ent = rows + kRxPicks;                                         // pick entry t * topk + slot
    int *tile_start = ent + kRxPicks;                                       // item prefix [E + 1]
    const int tid = threadIdx.x, r = tid >> 5, q = tid & 31;
    item_prefix(p.bcnt, p.E, 1, kRxPicks, tile_start);
    __syncthreads();
    const int total = tile_start[p.E];
    const int n_steps = (p.H / kRtBK + kRtCluster - 1) / kRtCluster;
    int ck0, clen;
    rank_range(p.H, r, ck0, clen);
    clen -= ck0;
    // copies: x part tid % 4 of pick tid / 4 for every rank; W: rank tid / 8, part tid % 8 (tid < 64)
    const int xp = tid >> 2, xpart = tid & 3;
    int xk0[kRtCluster], xlen[kRtCluster];
#pragma unroll
    for (int rr = 0; rr < kRtCluster; ++rr) {
        rank_range(p.H, rr, xk0[rr], xlen[rr]);
        xlen[rr] -= xk0[rr];
    }
    int wk0 = 0, wlen = 0;
    if (tid < 64) {
        rank_range(p.H, tid >> 3, wk0, wlen);
        wlen -= wk0;
    }
    const uint32_t ring = smem_u32(smem);
    for (int item = cta; item < total; item += n_ctas) {
        int lo = 0, hi = p.E - 1;  // largest e with tile_start[e] <= item
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_start[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo, c = item - tile_start[e];
        const int n = min(kRxPicks, p.bcnt[e] - c * kRxPicks);
        if (tid < kRxPicks) {
            const int32_t en = tid < n ? p.bucket[static_cast<int64_t>(e) * p.T + c * kRxPicks + tid] : -1;
            ent[tid] = en;
            rows[tid] = en >= 0 ? en / p.topk : 0;
        }
        __syncthreads();
        const bool xon = xp < n;
        const __nv_bfloat16 *xsrc = p.x + static_cast<int64_t>(rows[xp]) * p.H + 8 * xpart;
        const float *wsrc = p.w + static_cast<int64_t>(e) * p.H + wk0 + 4 * (tid & 7);
        auto issue = [&](int st) {  // stage st into ring slot st % kRxStages; always one commit group
            if (st < n_steps) {
                const uint32_t buf = ring + static_cast<uint32_t>((st % kRxStages) * kRxBuf * 4);
                const int k = 32 * st;
                if (xon) {
#pragma unroll
                    for (int rr = 0; rr < kRtCluster; ++rr)
                        if (k < xlen[rr])
                            cp_async16(buf + static_cast<uint32_t>(((rr * kRxPicks + xp) * kRsXWords + 4 * xpart) * 4),
                                       xsrc + xk0[rr] + k);
                }
                if (tid < 64 && k < wlen)
                    cp_async16(buf + static_cast<uint32_t>((kRxX + (tid >> 3) * 32 + 4 * (tid & 7)) * 4), wsrc + k);
            }
            cp_async_commit();
        };
        float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int st = 0; st < kRxStages - 1; ++st) issue(st);
        for (int st = 0; st < n_steps; ++st) {
            // stage st has landed for every thread, and every thread is done with stage st - 1, whose
            // slot the refill below takes: one barrier per step
            cp_async_wait<kRxStages - 2>();
            __syncthreads();
            issue(st + kRxStages - 1);
            if (32 * st < clen) {
                const uint32_t *cur = smem + (st % kRxStages) * kRxBuf;
                const uint32_t *wr = cur + kRxX + r * 32;
                const uint32_t *x0 = cur + (r * kRxPicks + q) * kRsXWords, *x1 = x0 + 32 * kRsXWords;
#pragma unroll
                for (int kk = 0; kk < 32; kk += 8) {
                    const float4 wlo = lds_f4(wr, kk), whi = lds_f4(wr, kk + 4);
                    const uint4 v0 = lds_u4(x0, kk / 2), v1 = lds_u4(x1, kk / 2);
                    a0 = fma4(wlo, make_uint2(v0.x, v0.y), a0);
                    a0 = fma4(whi, make_uint2(v0.z, v0.w), a0);
                    a1 = fma4(wlo, make_uint2(v1.x, v1.y), a1);
                    a1 = fma4(whi, make_uint2(v1.z, v1.w), a1);
                }
            }
        }
        cp_async_wait<0>();
        partial[q * 8 + r] = a0;
        partial[(q + 32) * 8 + r] = a1;
        __syncthreads();
        if (tid < n) {  // the ranks in order
            float l = 0.0f;
#pragma unroll
            for (int rr = 0; rr < kRtCluster; ++rr) l += partial[tid * 8 + rr];
            p.xlogit[ent[tid]] = l;
        }
        __syncthreads();
    }
}

// One CTA: the exact projections of listed tokens 8 bt .. 8 bt + 7 onto experts e0 .. e0 + 31.  Thread
// (e, r) runs rank r's chain of expert e for the eight tokens; per 32-k step the CTA stages the 256 W_r
// segments ([e][r][36 words]) and the tokens' x segments ([token][r][20 words]).
__device__ __forceinline__ void exact_batch(const RouterSelParams &p, float *exact, int n, int bt, int e0,
                                            uint32_t *smem) {
    float *partial = reinterpret_cast<float *>(smem + kRsExactStages * kRsExactBuf);  // [token][e][r]
    const int tid = threadIdx.x, el = tid >> 3, r = tid & 7;
    // rank ranges this thread touches: its W copies (rank (tid / 8) % 8), its x copy (rank (tid / 4) % 8)
    // and its chain (rank tid % 8)
    const int n_steps = (p.H / kRtBK + kRtCluster - 1) / kRtCluster;
    int wk0, wlen, xk0, xlen, clen;
    {
        int a, b;
        rank_range(p.H, (tid >> 3) & 7, a, b);
        wk0 = a;
        wlen = b - a;
        rank_range(p.H, (tid >> 2) & 7, a, b);
        xk0 = a;
        xlen = b - a;
        rank_range(p.H, r, a, b);
        clen = b - a;
    }
    const int nt = min(8, n - 8 * bt);
    // this thread's copy addresses, fixed over the steps: W chunk q = tid + 256 i -> segment q / 8 (expert
    // q / 64, rank (tid / 8) % 8), part tid % 8; x: token tid / 32, rank (tid / 4) % 8, part tid % 4
    const int wpart = tid & 7, xtok = tid >> 5;
    const uint32_t ring = smem_u32(smem);
    const int64_t xrow = xtok < nt ? static_cast<int64_t>(p.list[8 * bt + xtok]) : 0;
    const __nv_bfloat16 *xsrc = p.x + xrow * p.H + xk0 + 8 * (tid & 3);
    const uint32_t xdst =
        static_cast<uint32_t>((kRsExactW + (xtok * 8 + ((tid >> 2) & 7)) * kRsXWords + 4 * (tid & 3)) * 4);
    auto issue = [&](int st) {
        if (st < n_steps) {
            const uint32_t buf = ring + static_cast<uint32_t>((st % kRsExactStages) * kRsExactBuf * 4);
            const int k = 32 * st;
            if (k < wlen) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {  // W: chunk q = tid + 256 i -> segment q / 8 = (e, r), part q % 8
                    const int seg = (tid >> 3) + 32 * i, e = seg >> 3;
                    if (e0 + e < p.E)
                        cp_async16(buf + static_cast<uint32_t>((seg * kRsSegWords + 4 * wpart) * 4),
                                   p.w + static_cast<int64_t>(e0 + e) * p.H + wk0 + k + 4 * wpart);
                }
            }
            if (xtok < nt && k < xlen) cp_async16(buf + xdst, xsrc + k);
        }
        cp_async_commit();
    };
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int st = 0; st < kRsExactStages - 1; ++st) issue(st);
    for (int st = 0; st < n_steps; ++st) {
        issue(st + kRsExactStages - 1);
        cp_async_wait<kRsExactStages - 1>();
        __syncthreads();
        if (32 * st < clen) {
            const uint32_t *cur = smem + (st % kRsExactStages) * kRsExactBuf;
            const uint32_t *wseg = cur + tid * kRsSegWords;
#pragma unroll
            for (int kk = 0; kk < 32; kk += 4) {
                const float4 w4 = lds_f4(wseg, kk);
#pragma unroll
                for (int tk = 0; tk < 8; ++tk)
                    acc[tk] = fma4(w4, lds_u2(cur + kRsExactW + (tk * 8 + r) * kRsXWords, kk / 2), acc[tk]);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int tk = 0; tk < 8; ++tk) partial[(tk * 32 + el) * 8 + r] = acc[tk];
    __syncthreads();
    {  // thread (token tid / 32, expert tid % 32): the ranks in order
        const int tk = tid >> 5, e = tid & 31;
        if (tk < nt && e0 + e < p.E) {
            float l = 0.0f;
#pragma unroll
            for (int q = 0; q < kRtCluster; ++q) l += partial[(tk * 32 + e) * 8 + q];
            exact[static_cast<int64_t>(8 * bt + tk) * p.E + e0 + e] = l;
        }
    }
    __syncthreads();
}

// blockIdx.x < n_exact: exact_batch over (expert chunk blockIdx.x % n_chunk, batches blockIdx.x / n_chunk
// + k n_exact / n_chunk); the rest: exact_picks, persistent.
__global__ void __launch_bounds__(256, 1) router_exact_kernel(const RouterSelParams p, float *exact, int n_exact) {
    extern __shared__ __align__(16) uint32_t rs_path_smem[];
    if (static_cast<int>(blockIdx.x) < n_exact) {
        const int n = *p.list_n;
        const int n_chunk = (p.E + 31) / 32, slots = n_exact / n_chunk;
        const int chunk = blockIdx.x % n_chunk;
        for (int bt = blockIdx.x / n_chunk; bt < (n + 7) / 8; bt += slots) exact_batch(p, exact, n, bt, 32 * chunk, rs_path_smem);
        return;
    }
    exact_picks(p, rs_path_smem, static_cast<int>(blockIdx.x) - n_exact, static_cast<int>(gridDim.x) - n_exact);
}

// One warp: the selection of router_topk_kernel for listed token list[i] on its exact projections.
__device__ __noinline__ void list_select(const RouterSelParams &p, int64_t i, int lane) {
    const int64_t t = p.list[i];
    float sc[8], sel[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        score_of(e < p.E ? p.exact[i * p.E + e] : 0.0f, e, p, sc[j], sel[j]);
    }
    float den, my_s;
    int my_id;
    select_group_limited(sc, sel, lane, p.E, p.G, p.topk_groups, p.topk, p.group_topn, my_id, my_s, den, nullptr);
    if (lane < p.topk) {
        p.ids[t * p.topk + lane] = my_id;
        p.wts[t * p.topk + lane] = my_s / den;
    }
}

// The selection of router_topk_kernel from exact projections, one warp per global warp index g:
//   (a) screened token g (lane j holds pick j): the picks ordered by (selection value desc, expert asc)
//       from their exact projections and normalised in that order;
//   (b) listed token list[g]: the full selection on its projections onto every expert.
// (a) skips the listed tokens by their flag, not by their ids: (b) of another warp may be writing
// those ids meanwhile.
__global__ void __launch_bounds__(256) router_finish_kernel(const RouterSelParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t g = blockIdx.x * 8LL + (threadIdx.x >> 5);
    if (g < p.T && !p.listed[g]) {
        const int64_t t = g;
        const int my_id = lane < p.topk ? p.ids[t * p.topk + lane] : 0;
        {
            float s_p = 0.0f, sel_p = -INFINITY;
            if (lane < p.topk) score_of(p.xlogit[t * p.topk + lane], my_id, p, s_p, sel_p);
            // this pick's slot: the picks ahead of it (the order is total: the experts differ)
            int ahead = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float sv = __shfl_sync(0xffffffffu, sel_p, i);
                const int ev = __shfl_sync(0xffffffffu, my_id, i);
                if (i < p.topk && (sv > sel_p || (sv == sel_p && ev < my_id))) ++ahead;
            }
            // lane r takes the pick of slot r; the denominator sums the slots in order
            float s_slot = 0.0f;
            int e_slot = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int a = __shfl_sync(0xffffffffu, ahead, i);
                const float sv = __shfl_sync(0xffffffffu, s_p, i);
                const int ev = __shfl_sync(0xffffffffu, my_id, i);
                if (i < p.topk && a == lane) {
                    s_slot = sv;
                    e_slot = ev;
                }
            }
            float den = 0.0f;
            for (int r = 0; r < p.topk; ++r) den = den + __shfl_sync(0xffffffffu, s_slot, r);
            if (lane < p.topk) {
                p.ids[t * p.topk + lane] = e_slot;
                p.wts[t * p.topk + lane] = s_slot / den;
            }
        }
    }
    if (g < *p.list_n) list_select(p, g, lane);
}

}  // namespace beam
