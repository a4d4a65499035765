// Sublayer norms and the scaled residual update around the MoE block.
//
// "Welcome Beam" page, section "Residual Stream": every sublayer is normalised before and after;
// the input embedding is step 1, and at step k the sublayer output is added with weight 1/sqrt(k)
// while the stream keeps weight sqrt((k-1)/k); the norms compute in FP32.  Reading: RMSNorm with a
// learned per-channel scale, x / sqrt(mean(x^2) + eps) * g.
//
//   rmsnorm_bf16_kernel           u[t]  = bf16(x[t] / sqrt(mean(x[t]^2) + eps) * g_pre)
//   combine_norm_residual_kernel  y[t]  = routed_scale * sum_j w[t,j] * o[dest_row(t,j)]   (FP32)
//                                 out[t] = bf16(sqrt((k-1)/k) * s[t] + RMSNorm(y[t]) * g_post / sqrt(k))
// One CTA per token; every FP32 reduction is taken in a fixed order (deterministic).  The combine
// keeps its FP32 row in shared memory, so the post-norm and the residual update cost no extra HBM
// pass over the block output.
#pragma once

#include "common.cuh"

namespace beam {

constexpr int kNormThreads = 256;

// Sum of v over the block's 256 threads: butterfly within each warp, then the 8 warp sums in order.
__device__ __forceinline__ float block_sum_fixed(float v, float *red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) s += red[w];
    __syncthreads();
    return s;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&b);
}

// One CTA per token: FP32 sum of squares in a fixed order, IEEE sqrt and division, bf16 RNE output.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_bf16_kernel(const uint4 *__restrict__ x,
                                                                     const float *__restrict__ g, float eps, int H,
                                                                     uint4 *__restrict__ u) {
    __shared__ float red[kNormThreads / 32];
    const int64_t t = blockIdx.x;
    const int nvec = H / 8;
    const uint4 *row = x + t * nvec;
    float ss = 0.0f;
    for (int c = threadIdx.x; c < nvec; c += kNormThreads) {
        float f[8];
        bf16x8_to_f32(__ldg(row + c), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
    }
    ss = block_sum_fixed(ss, red);
    const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
    for (int c = threadIdx.x; c < nvec; c += kNormThreads) {
        float f[8];
        bf16x8_to_f32(__ldg(row + c), f);
        const float4 g0 = __ldg(reinterpret_cast<const float4 *>(g) + 2 * c);
        const float4 g1 = __ldg(reinterpret_cast<const float4 *>(g) + 2 * c + 1);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        uint4 o;
        o.x = pack_bf16x2(f[0] * inv * gg[0], f[1] * inv * gg[1]);
        o.y = pack_bf16x2(f[2] * inv * gg[2], f[3] * inv * gg[3]);
        o.z = pack_bf16x2(f[4] * inv * gg[4], f[5] * inv * gg[5]);
        o.w = pack_bf16x2(f[6] * inv * gg[6], f[7] * inv * gg[7]);
        u[t * nvec + c] = o;
    }
}

// One CTA per token: weighted combine of the k expert rows (FP32, slot order), post-norm of the
// FP32 row, scaled residual update with the incoming stream, bf16 RNE output.  `out` may equal
// `stream_in` (each element is read before it is written, by the same thread).
__global__ void __launch_bounds__(kNormThreads)
    combine_norm_residual_kernel(const float4 *__restrict__ o, const int32_t *__restrict__ dest_row,
                                 const float *__restrict__ w, int k, int H, float scale, const uint2 *stream_in,
                                 const float *__restrict__ g, float eps, float keep, float add, uint2 *out) {
    extern __shared__ float4 ysm[];  // [H/4] FP32 block output of this token
    __shared__ int64_t rows[16];
    __shared__ float wt[16];
    __shared__ float red[kNormThreads / 32];
    const int64_t t = blockIdx.x;
    const int H4 = H / 4;
    if (threadIdx.x < k) {
        rows[threadIdx.x] = dest_row[t * k + threadIdx.x];
        wt[threadIdx.x] = w[t * k + threadIdx.x];
    }
    __syncthreads();
    float ss = 0.0f;
    for (int c = threadIdx.x; c < H4; c += kNormThreads) {
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
        const float4 y = make_float4(scale * acc.x, scale * acc.y, scale * acc.z, scale * acc.w);
        ysm[c] = y;
        ss = fmaf(y.x, y.x, ss);
        ss = fmaf(y.y, y.y, ss);
        ss = fmaf(y.z, y.z, ss);
        ss = fmaf(y.w, y.w, ss);
    }
    ss = block_sum_fixed(ss, red);
    const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
    for (int c = threadIdx.x; c < H4; c += kNormThreads) {
        const float4 y = ysm[c];
        const float4 gg = __ldg(reinterpret_cast<const float4 *>(g) + c);
        const uint2 sv = stream_in[t * H4 + c];
        const float s0 = __uint_as_float(sv.x << 16), s1 = __uint_as_float(sv.x & 0xffff0000u);
        const float s2 = __uint_as_float(sv.y << 16), s3 = __uint_as_float(sv.y & 0xffff0000u);
        uint2 r;
        r.x = pack_bf16x2(fmaf(add, y.x * inv * gg.x, keep * s0), fmaf(add, y.y * inv * gg.y, keep * s1));
        r.y = pack_bf16x2(fmaf(add, y.z * inv * gg.z, keep * s2), fmaf(add, y.w * inv * gg.w, keep * s3));
        out[t * H4 + c] = r;
    }
}

}  // namespace beam
