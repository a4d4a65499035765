// Combine kernel C: y[t] = routed_scale * sum_{j<k} w[t, j] * o[dest_row[t*k + j]]
// ("Expert outputs are combined with normalized router weights and scaled by 2.5": "Welcome Beam"
// page, section "Mixture of Experts").  FP32 fused multiply-adds in slot order j = 0..k-1 starting
// from zero, one multiply by routed_scale, round-to-nearest-even to bf16.  16-byte loads of the
// expert outputs, 8-byte stores of 4 bf16; one CTA per token.
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
        for (int j = 0; j < k; ++j) {
            if (rows[j] < 0) continue;  // a bad expert id (reported through the status word)
            const float4 v = __ldg(o + rows[j] * H4 + c);
            const float wj = wt[j];
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(scale * acc.x, scale * acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(scale * acc.z, scale * acc.w);
        uint2 out;
        out.x = *reinterpret_cast<uint32_t *>(&lo);
        out.y = *reinterpret_cast<uint32_t *>(&hi);
        y[t * H4 + c] = out;
    }
}

}  // namespace beam
