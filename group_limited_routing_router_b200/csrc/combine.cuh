// Combine kernel C: y[t] = routed_scale * sum_{j<k} w[t, j] * o[dest_row[t*k + j]]
// ("Expert outputs are combined with normalized router weights and scaled by 2.5": "Welcome Beam"
// page, section "Mixture of Experts").  FP32 fused multiply-adds in slot order j = 0..k-1 starting
// from zero, one multiply by routed_scale, round-to-nearest-even to bf16.  16-byte loads of the
// expert outputs, one CTA per token.  combine_kernel takes FP32 expert outputs (the paths with bf16
// activations); combine_bf16_kernel takes bf16 ones (the block-scaled paths, whose activations are
// quantised to 8 or 4 bits, so the 2^-9 relative rounding of o is far below their own error).
#pragma once

#include "common.cuh"

namespace beam {

__global__ void __launch_bounds__(256) combine_kernel(const float4 *__restrict__ o, const int32_t *__restrict__ dest_row,
                                                        const float *__restrict__ w, int64_t T, int k, int H4,
                                                        float scale, uint2 *__restrict__ y) {
    __shared__ int64_t rows[16];
    __shared__ float wt[16];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = dest_row[t * k + threadIdx.x];
        wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < H4; c += blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        // up to 8 slots: every row's load is issued before the sums, which stay in slot order
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = (j < k && rows[j] >= 0) ? __ldg(o + rows[j] * H4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (j >= k || rows[j] < 0) continue;  // a bad expert id (reported through the status word)
            const float wj = wt[j];
            acc.x = fmaf(wj, v[j].x, acc.x);
            acc.y = fmaf(wj, v[j].y, acc.y);
            acc.z = fmaf(wj, v[j].z, acc.z);
            acc.w = fmaf(wj, v[j].w, acc.w);
        }
        for (int j = 8; j < k; ++j) {  // more than 8 slots
            if (rows[j] < 0) continue;
            const float4 u = __ldg(o + rows[j] * H4 + c);
            const float wj = wt[j];
            acc.x = fmaf(wj, u.x, acc.x);
            acc.y = fmaf(wj, u.y, acc.y);
            acc.z = fmaf(wj, u.z, acc.z);
            acc.w = fmaf(wj, u.w, acc.w);
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(scale * acc.x, scale * acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(scale * acc.z, scale * acc.w);
        uint2 out;
        out.x = *reinterpret_cast<uint32_t *>(&lo);
        out.y = *reinterpret_cast<uint32_t *>(&hi);
        y[t * H4 + c] = out;
    }
}

__global__ void __launch_bounds__(256) combine_bf16_kernel(const uint4 *__restrict__ o,
                                                             const int32_t *__restrict__ dest_row,
                                                             const float *__restrict__ w, int64_t T, int k, int H8,
                                                             float scale, uint4 *__restrict__ y) {
    __shared__ int64_t rows[16];
    __shared__ float wt[16];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = dest_row[t * k + threadIdx.x];
        wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < H8; c += blockDim.x) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < k; ++j) {
            if (rows[j] < 0) continue;  // a bad expert id (reported through the status word)
            const uint4 v = __ldg(o + rows[j] * H8 + c);
            const float wj = wt[j];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // bf16 -> fp32 is exact: the bits move up 16 places
                acc[2 * i] = fmaf(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = fmaf(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
        }
        uint32_t r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(scale * acc[2 * i], scale * acc[2 * i + 1]);
            r[i] = *reinterpret_cast<const uint32_t *>(&pr);
        }
        y[t * H8 + c] = make_uint4(r[0], r[1], r[2], r[3]);
    }
}

}  // namespace beam
