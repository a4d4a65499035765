// Dispatch kernels P: stable grouping of the T*k routed (token, slot) pairs by expert, and the row
// gather of x into that order for the wide-tile gate/up GEMM.
//
// The pages only say that each token runs on its 8 experts; this is the library's deterministic
// convention: rows sorted by (expert ascending, token ascending).  Three launches:
//   permute_hist    one CTA per chunk of 256 tokens counts its pairs per expert (shared-memory
//                   integer atomics: the counts do not depend on their order);
//   permute_scan    one CTA turns the per-chunk counts into per-chunk bases, the per-expert counts
//                   and the exclusive offsets;
//   permute_scatter one CTA per chunk again; each warp owns 32 tokens, gets its per-expert base
//                   from the warp-order prefix, and ranks its pairs 32 at a time in (token, slot)
//                   order with __match_any_sync, so the result is bit-identical on every run.
// The per-chunk counts live in caller-provided scratch (the workspace).
#pragma once

#include "common.cuh"

namespace beam {

constexpr int kPmTok = 256;      // tokens per chunk (one CTA)
constexpr int kPmThreads = 256;  // 8 warps x 32 tokens
constexpr int kPmMaxE = 256;

__global__ void __launch_bounds__(kPmThreads) permute_hist_kernel(const int32_t *__restrict__ ids, int64_t T, int k,
                                                                    int E, int32_t *__restrict__ hist) {
    __shared__ int cnt[kPmMaxE];
    for (int e = threadIdx.x; e < E; e += kPmThreads) cnt[e] = 0;
    __syncthreads();
    const int64_t tb = static_cast<int64_t>(blockIdx.x) * kPmTok;
    const int64_t te = min(T, tb + kPmTok);
    bool bad = false;
    for (int64_t q = tb * k + threadIdx.x; q < te * k; q += kPmThreads) {
        const int e = ids[q];
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&cnt[e], 1);
        else bad = true;
    }
    if (bad) set_status(BEAM_MOE_ERR_BAD_INDEX);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kPmThreads) hist[static_cast<int64_t>(blockIdx.x) * E + e] = cnt[e];
}

// One CTA of 1024 threads: thread (e = tid % 256, part = tid / 256) walks a quarter of the chunks.
__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t *__restrict__ hist, int nchunks, int E,
                                                              int32_t *__restrict__ counts,
                                                              int64_t *__restrict__ offsets) {
    __shared__ int partsum[4][kPmMaxE];
    __shared__ int cnt_s[kPmMaxE];
    const int e = threadIdx.x & 255, part = threadIdx.x >> 8;
    const int c0 = part * nchunks / 4, c1 = (part + 1) * nchunks / 4;
    int run = 0;
    if (e < E) {
        for (int c = c0; c < c1; ++c) {
            const int v = hist[static_cast<int64_t>(c) * E + e];
            hist[static_cast<int64_t>(c) * E + e] = run;
            run += v;
        }
    }
    partsum[part][e] = run;
    __syncthreads();
    if (e < E) {
        int base = 0;
        for (int q = 0; q < part; ++q) base += partsum[q][e];
        if (base)
            for (int c = c0; c < c1; ++c) hist[static_cast<int64_t>(c) * E + e] += base;
        if (part == 0) {
            const int tot = partsum[0][e] + partsum[1][e] + partsum[2][e] + partsum[3][e];
            counts[e] = tot;
            cnt_s[e] = tot;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int q = 0; q < E; ++q) {
            offsets[q] = acc;
            acc += cnt_s[q];
        }
        offsets[E] = acc;
    }
}

__global__ void __launch_bounds__(kPmThreads) permute_scatter_kernel(const int32_t *__restrict__ ids, int64_t T,
                                                                       int k, int E,
                                                                       const int32_t *__restrict__ hist,
                                                                       const int64_t *__restrict__ offsets,
                                                                       int32_t *__restrict__ row_src,
                                                                       int32_t *__restrict__ dest_row) {
    __shared__ int cnt[kPmThreads / 32][kPmMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < (kPmThreads / 32) * kPmMaxE; i += kPmThreads) (&cnt[0][0])[i] = 0;
    __syncthreads();
    const int64_t tw0 = static_cast<int64_t>(blockIdx.x) * kPmTok + warp * 32;
    const int64_t tw1 = min(T, tw0 + 32);
    const int64_t q0 = tw0 * k, q1 = tw1 > tw0 ? tw1 * k : q0;
    for (int64_t q = q0 + lane; q < q1; q += 32) {
        const int e = ids[q];
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&cnt[warp][e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kPmThreads) {
        int run = static_cast<int>(offsets[e]) + hist[static_cast<int64_t>(blockIdx.x) * E + e];
        for (int w = 0; w < kPmThreads / 32; ++w) {
            const int c = cnt[w][e];
            cnt[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int64_t qb = q0; qb < q1; qb += 32) {
        const int64_t q = qb + lane;
        const int e = q < q1 ? ids[q] : -1;
        const bool valid = static_cast<unsigned>(e) < static_cast<unsigned>(E);
        const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
        int base = 0, rank = 0;
        uint32_t peers = 0;
        if (!valid && q < q1) dest_row[q] = -1;  // a bad id: no row (gather and combine skip it)
        if (valid) {
            peers = __match_any_sync(vmask, e);
            rank = __popc(peers & lt_mask);
            base = cnt[warp][e];
            const int r = base + rank;
            dest_row[q] = r;
            row_src[r] = static_cast<int32_t>(q);
        }
        __syncwarp();
        if (valid && rank == 0) cnt[warp][e] = base + __popc(peers);
        __syncwarp();
    }
}

// x_perm[dest_row[t*k + j]] = x[t] for every slot j: each token row is read once and written k times
// (the wide-tile gate/up GEMM reads its token rows from x_perm with tiled TMA boxes).
__global__ void __launch_bounds__(128) gather_rows_kernel(const uint4 *__restrict__ x, int64_t T, int k, int nvec,
                                                            const int32_t *__restrict__ dest_row,
                                                            uint4 *__restrict__ xp) {
    __shared__ int64_t rows[16];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < k) rows[threadIdx.x] = dest_row[t * k + threadIdx.x];
    __syncthreads();
    const uint4 *src = x + t * nvec;
    constexpr int U = 4;  // loads in flight per thread before its stores
    for (int c0 = threadIdx.x; c0 < nvec; c0 += U * blockDim.x) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * blockDim.x;
            if (c < nvec) v[u] = __ldg(src + c);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * blockDim.x;
            if (c < nvec)
                for (int j = 0; j < k; ++j)
                    if (rows[j] >= 0) xp[rows[j] * nvec + c] = v[u];
        }
    }
}

}  // namespace beam
