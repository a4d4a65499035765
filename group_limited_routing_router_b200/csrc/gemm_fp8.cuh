// Grouped expert GEMMs with block-scaled low-precision expert weights.  Same work items, orientation
// (swap-AB: weight rows on the MMA's M side, the expert's tokens on N), accumulator slots and
// epilogue as the bf16 kernel in gemm.cuh; the tensor cores still multiply bf16 x bf16 into FP32.
//   FP8 (MXFP8): E4M3 codes, one power-of-two UE8M0 scale per 32 consecutive K elements.
//   FP4 (NVFP4): E2M1 codes, two per byte (even k in the low nibble), one E4M3 scale per 16
//     consecutive K elements, one FP32 scale per weight matrix.
// "Checkpoint formats: BF16, FP8, and NVFP4" ("Welcome Beam" page, TL;DR; section "Hardware
// Requirements": most parameters in 4 bits on Blackwell); the pages give no quantisation recipe,
// so the layouts are the OCP microscaling and NVIDIA NVFP4 ones, scales stored K-block-major.
// Both rebuild exact bf16 values: E4M3 x 2^k has at most 4 significant bits, E2M1 x E4M3 x 2^-9 at
// most 6.  The NVFP4 per-matrix scale (times the 2^9) multiplies the FP32 accumulators in the
// epilogue.
//
// Rings and roles (threads = 256 + 32 * converter warps):
//   weight ring (W8STAGES): per stage the A tile(s) as 128 rows x 128 bytes (K = 128 of E4M3 or
//     K = 256 of E2M1; 128-byte swizzle: a weight row contributes 128 contiguous bytes, the piece
//     size at which DRAM streams best) and their scale tiles [K-blocks of the stage][128 rows].
//     Warp 0 lane 0 loads it (TMA); the converters release it as soon as they have read it, so the
//     weight stream never waits on the tensor core.
//   B ring (BSTAGES): one 64-wide k-step of the expert's token rows (tiled TMA boxes, or TMA
//     gather4 straight from x).  Warp 2 loads it; the MMA releases it.
//   A ring (ASTAGES, in TMEM after the accumulator slots): the bf16 A tile(s) of one 64-wide
//     k-step.  Converter warps (from warp 8 on) rebuild them from the codes with tcgen05.st; the
//     MMA reads its A operand from TMEM and frees the stage with tcgen05.commit.
//   Warp 1 lane 0 issues tcgen05.mma; warps 4..7 run the epilogue.
// Every wait is bounded (status word BEAM_MOE_ERR_DEVICE_TIMEOUT on expiry).
#pragma once

#include "gemm.cuh"

namespace beam {

// Converter warps per A tile: each (A tile, 64-wide k-step) splits into 8 warp units (4 TMEM lane
// quadrants x 2 quarters of 32 K elements); a converter warp takes 8 / kConvPerTile of them.
constexpr int kConvPerTile = 8;

constexpr int round1024(int v) { return (v + 1023) / 1024 * 1024; }

constexpr int fp8_gemm_threads(bool gate_up) { return 256 + 32 * kConvPerTile * (gate_up ? 2 : 1); }

template <bool GATE_UP, int BN, int BOXN, int W8STAGES, int BSTAGES, int NSLOT, int SLOT_COLS, bool GATHER,
          int ASTAGES, bool FP4 = false>
struct Fp8GemmCfg {
    static constexpr int kNumA = GATE_UP ? 2 : 1;
    static constexpr int kConvWarps = kConvPerTile * kNumA;
    static constexpr int kConvUnits = 8 / kConvPerTile;  // warp units per converter warp
    static constexpr int kThreads = fp8_gemm_threads(GATE_UP);
    static constexpr int kK8 = (FP4 ? 4 : 2) * kBK;       // K per weight ring stage
    static constexpr int kSteps = kK8 / kBK;              // 64-wide k-steps per weight stage
    static constexpr int kBlk = FP4 ? 16 : 32;            // K elements per scale code
    static constexpr int kA8 = kBM * 128;                 // one A tile of the stage, bytes
    static constexpr int kSc = (kK8 / kBlk) * kBM;        // one scale tile, bytes
    static constexpr int kScOff = kNumA * kA8;            // scale tiles after the A tiles
    static constexpr int kW8Stage = round1024(kNumA * (kA8 + kSc));
    static constexpr int kB = BN * kBK * 2;               // B tile of one 64-wide k-step
    static constexpr int kBox = BOXN * kBK * 2;
    static constexpr int kBOff = W8STAGES * kW8Stage;
    static constexpr int kACol = NSLOT * SLOT_COLS;       // TMEM column of the A ring
    static constexpr int kTmemCols = pow2_cols(NSLOT * SLOT_COLS + ASTAGES * kNumA * 32);
    static constexpr int kBarOff = kBOff + BSTAGES * kB;
    static constexpr int kBarBytes = 1024;
    static constexpr int kTokOff = kBarOff + kBarBytes + 4 * (kPmMaxE + 1);
    static constexpr int kSmem = 1024 + kTokOff + (GATHER ? 4 * BN : 0) + 64;
    static_assert(kB % 1024 == 0 && (GATHER || kBox % 1024 == 0), "tiles must keep 1024-byte alignment");
    static_assert(BN % BOXN == 0 && BN % 16 == 0 && BN <= 256, "token tile");
    static_assert(!GATHER || BOXN == 1, "gathered B rows come one row per box, four per instruction");
    static_assert(NSLOT * SLOT_COLS + ASTAGES * kNumA * 32 <= 512, "TMEM has 512 columns");
    static_assert(GATE_UP ? (BN <= SLOT_COLS && (NSLOT >= 2 || BN <= SLOT_COLS / 2)) : BN <= SLOT_COLS,
                  "an item must fit in its TMEM slots");
    static_assert((2 * W8STAGES + 2 * BSTAGES + 2 * NSLOT + 1 + 2 * ASTAGES) * 8 + 4 <= kBarBytes, "barriers");
    static_assert(kThreads <= 1024 && kSmem <= 232448, "block resources");
};

// E4M3 -> bf16 by integer rebuild.  For a code b = s eeee mmm, the 16-bit pattern
// s | (b & 0x7f) << 4 read as bf16 has exponent field e and mantissa mmm0000: the value
// e4m3(b) * 2^-120, for normal codes (e >= 1: (1 + m/8) 2^(e-127)) and subnormal ones (e = 0:
// m/8 * 2^-126, a bf16 subnormal) alike.  prmt places each byte in the low half of a 16-bit lane
// with its sign replicated into the byte above, so one shift and one mask put sign, exponent and
// mantissa in place.  A bf16 multiply by 2^(c-7) restores the value times the block scale 2^(c-127);
// when c - 7 exceeds bf16's largest exponent (c > 134) a second factor follows.  The product has
// at most 4 significant bits, so it is exact whenever it is a normal bf16 number.
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// bf16x2 factors for scale code c: 2^(c-7) (or 2^127 when c > 134), then 2^(c-134) (or 1).
__device__ __forceinline__ uint32_t fp8_factor1(uint32_t c) { return ((c > 134u ? 254u : c + 120u) << 7) * 0x10001u; }
__device__ __forceinline__ uint32_t fp8_factor2(uint32_t c) { return ((c > 134u ? c - 7u : 127u) << 7) * 0x10001u; }

// Four codes (one 32-bit word, lowest byte first) -> bf16 pairs (codes 0,1) and (codes 2,3).
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t f1, uint32_t &lo, uint32_t &hi) {
    uint32_t a, b;
    asm("prmt.b32 %0, %1, 0, 0x9180;" : "=r"(a) : "r"(w));  // [sign(b1) b1 sign(b0) b0]
    asm("prmt.b32 %0, %1, 0, 0xB3A2;" : "=r"(b) : "r"(w));  // [sign(b3) b3 sign(b2) b2]
    lo = bf16x2_mul((a << 4) & 0x87F087F0u, f1);
    hi = bf16x2_mul((b << 4) & 0x87F087F0u, f1);
}

// E2M1 -> bf16 by the same kind of integer rebuild.  For a code n = s ee m, the 16-bit pattern
// s << 15 | (n & 7) << 6 read as bf16 has exponent field e and mantissa m000000: the value
// e2m1(n) * 2^-126 (e = 0: m/2 * 2^-126, a bf16 subnormal).  For a byte holding codes n0 (low
// nibble) and n1, lo * 0x1040 puts n0's magnitude at bits 6..8 and its sign at bit 15, and
// hi * 0x01040000 puts n1's at bits 22..24 and 31; the two products use disjoint bits, and the
// mask keeps those.  A bf16 multiply by the block scale s x 2^117 gives e2m1 x s x 2^-9, exact.
__device__ __forceinline__ uint32_t e2m1x2_to_bf16x2(uint32_t byte, uint32_t f) {
    const uint32_t pat = ((byte & 0x0Fu) * 0x1040u | (byte & 0xF0u) * 0x01040000u) & 0x81C081C0u;
    return bf16x2_mul(pat, f);
}
// bf16x2 factor for an E4M3 block-scale code c (sign bit ignored): e4m3(c) x 2^117, exact (the
// E4M3 value has at most 4 significant bits; 448 x 2^117 < 2^126).  (c & 0x7f) << 4 read as bf16 is
// e4m3(c) x 2^-120, subnormal codes included; FP32 then multiplies by 2^118 and 2^119.
__device__ __forceinline__ uint32_t e4m3_scale_factor(uint32_t c) {
    float v = __uint_as_float(((c & 0x7Fu) << 4) << 16);
    v *= 0x1p118f;
    v *= 0x1p119f;
    const uint32_t b = __float_as_uint(v) >> 16;
    return b | (b << 16);
}

// Per-expert FP32 factors for the accumulators (NVFP4: the per-matrix scales times 2^9): A0 (gate or
// down) and A1 (up), each multiplied by mul.
struct AccScales {
    const float *s0, *s1;
    float mul;
};

// gemm_epilogue (gemm.cuh) with the accumulators first multiplied by the item's expert factors.
template <bool GATE_UP, int BN, int NSLOT, int SLOT_COLS>
__device__ __forceinline__ void gemm_epilogue_scaled(int q, const int *tile_start, int total, const GemmParams &p,
                                                     const AccScales &acc, uint32_t tmem_base, uint64_t *acc_full,
                                                     uint64_t *acc_empty) {
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    uint32_t uses = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
        const int u = slots_of<GATE_UP, SLOT_COLS>(it.n_mma);
        bool ok = true;
        for (int i = 0; i < u && ok; ++i) {
            const uint32_t c = uses + i;
            ok = mbar_wait(&acc_full[c % NSLOT], (c / NSLOT) & 1u, p.timeout);
        }
        if (!ok) break;
        tc_fence_after();
        const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
        const int m = it.mt * kBM + q * 32 + lane;  // weight row of this thread
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(s0 * SLOT_COLS);
        const uint32_t t1 = tmem_base + lane_off +
                            static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
        const float f0 = acc.s0[it.e] * acc.mul;
        const float f1 = GATE_UP ? acc.s1[it.e] * acc.mul : 1.0f;
        for (int c = 0; c < it.n_valid; c += 16) {
            uint32_t r0[16];
            tmem_ld16(t0 + c, r0);
            if (GATE_UP) {
                uint32_t r1[16];
                tmem_ld16(t1 + c, r1);
                tmem_ld_wait();
                if (m < p.M) {
                    __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(p.out);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c + j < it.n_valid)
                            h[(it.row0 + c + j) * p.M + m] =
                                __float2bfloat16_rn(silu_mul(f0 * __uint_as_float(r0[j]), f1 * __uint_as_float(r1[j])));
                }
            } else {
                tmem_ld_wait();
                if (m < p.M) {
                    float *o = reinterpret_cast<float *>(p.out);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c + j < it.n_valid)
                            o[(it.row0 + c + j) * p.M + m] = f0 * __uint_as_float(r0[j]);
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int i = 0; i < u; ++i) mbar_arrive(&acc_empty[(uses + i) % NSLOT]);
        uses += u;
    }
}

template <bool GATE_UP, int BN, int BOXN, int W8STAGES, int BSTAGES, int NSLOT, int SLOT_COLS, bool GATHER,
          int ASTAGES, bool FP4 = false>
__global__ void __launch_bounds__(fp8_gemm_threads(GATE_UP), 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tm_a0,  // codes of W_gate (G1) / W_down (G2):
                                                                        // [E][M][K] E4M3, or [E][M][K/2] E2M1 pairs
                            const __grid_constant__ CUtensorMap tm_a1,  // codes of W_up (G1); unused for G2
                            const __grid_constant__ CUtensorMap tm_s0,  // scale codes of A0 [E][K/kBlk][M]
                            const __grid_constant__ CUtensorMap tm_s1,  // scale codes of A1
                            const __grid_constant__ CUtensorMap tm_b,   // B rows [rows][K] (GATHER: x [T][K])
                            const GemmParams p,
                            const AccScales acc) {  // FP4: per-expert accumulator factors
    using C = Fp8GemmCfg<GATE_UP, BN, BOXN, W8STAGES, BSTAGES, NSLOT, SLOT_COLS, GATHER, ASTAGES, FP4>;
    extern __shared__ uint8_t gemm_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *w8_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *w8_empty = w8_full + W8STAGES;
    uint64_t *b_full = w8_empty + W8STAGES;
    uint64_t *b_empty = b_full + BSTAGES;
    uint64_t *acc_full = b_empty + BSTAGES;
    uint64_t *acc_empty = acc_full + NSLOT;
    uint64_t *drain = acc_empty + NSLOT;
    uint64_t *a_ready = drain + 1;
    uint64_t *a_free = a_ready + ASTAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(a_free + ASTAGES);
    int *tile_start = reinterpret_cast<int *>(smem + C::kBarOff + C::kBarBytes);
    int *tok = reinterpret_cast<int *>(smem + C::kTokOff);  // GATHER: token of each row of the item

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int n_mt = (p.M + kBM - 1) / kBM;
    const int n_kb = p.K / kBK;          // 64-wide k-steps per item
    const int n_w8 = (n_kb + C::kSteps - 1) / C::kSteps;  // weight ring stages per item (the last may be partial)

    if (threadIdx.x == 0) {
        for (int s = 0; s < W8STAGES; ++s) {
            mbar_init(&w8_full[s], 1);
            mbar_init(&w8_empty[s], C::kConvWarps);
        }
        for (int s = 0; s < BSTAGES; ++s) {
            mbar_init(&b_full[s], 1);
            mbar_init(&b_empty[s], 1);
        }
        for (int a = 0; a < NSLOT; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(drain, 1);
        for (int j = 0; j < ASTAGES; ++j) {
            mbar_init(&a_ready[j], C::kConvWarps);
            mbar_init(&a_free[j], 1);
        }
        fence_mbar_init();
        prefetch_tensormap(&tm_a0);
        prefetch_tensormap(&tm_s0);
        if (GATE_UP) {
            prefetch_tensormap(&tm_a1);
            prefetch_tensormap(&tm_s1);
        }
        prefetch_tensormap(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    item_prefix(p.counts, E, n_mt, BN, tile_start);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[E];

    if (warp == 0) {
        // ---------------- weight producer: code tiles + scales, 128 bytes of each row per stage ----------------
        if (lane == 0) {
            const uint64_t pol_w = p.weights_once ? policy_evict_first() : policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
                for (int kb = 0; kb < n_w8; ++kb) {
                    if (!mbar_wait(&w8_empty[stage], phase ^ 1u, p.timeout)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * C::kW8Stage;
                    mbar_arrive_expect_tx(&w8_full[stage], C::kNumA * (C::kA8 + C::kSc));
                    // the code maps are byte-typed: 128 bytes of each row per stage
                    tma_load_3d(sa, &tm_a0, &w8_full[stage], kb * 128, it.mt * kBM, it.e, pol_w);
                    tma_load_3d(sa + C::kScOff, &tm_s0, &w8_full[stage], it.mt * kBM, kb * (C::kK8 / C::kBlk),
                                it.e, pol_w);
                    if (GATE_UP) {
                        tma_load_3d(sa + C::kA8, &tm_a1, &w8_full[stage], kb * 128, it.mt * kBM, it.e, pol_w);
                        tma_load_3d(sa + C::kScOff + C::kSc, &tm_s1, &w8_full[stage], it.mt * kBM,
                                    kb * (C::kK8 / C::kBlk), it.e, pol_w);
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == W8STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < W8STAGES; ++s)  // every load issued has landed before the CTA may exit
                if ((issued >> s) & 1u) mbar_wait(&w8_full[s], (issued_phase >> s) & 1u, p.timeout);
        }
    } else if (warp == 2) {
        // ---------------- B producer: the expert's token rows, one 64-wide k-step per stage ----------------
        const uint64_t pol_x = policy_evict_last();  // activations: re-read by the other weight-row tiles
        int stage = 0;
        uint32_t phase = 0, issued = 0, issued_phase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
            if (GATHER) {
                // rows past the expert's tokens (up to the MMA's N) repeat its first token: valid, ignored
                for (int r = lane; r < it.n_mma; r += 32) {
                    const int rr = r < it.n_valid ? r : 0;
                    tok[r] = p.row_src[it.row0 + rr] / p.topk;
                }
                __syncwarp();
            }
            if (lane == 0) {
                const int nbox = GATHER ? (it.n_mma + 3) / 4 : (it.n_mma + BOXN - 1) / BOXN;
                const uint32_t bytes = nbox * (GATHER ? 4 * kBK * 2 : C::kBox);
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(&b_empty[stage], phase ^ 1u, p.timeout)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sb = smem + C::kBOff + stage * C::kB;
                    mbar_arrive_expect_tx(&b_full[stage], bytes);
                    if (GATHER) {
                        for (int g = 0; g < nbox; ++g)  // rows 4g..4g+3 land 128 B apart, as a tiled box would
                            tma_gather4(sb + g * 4 * kBK * 2, &tm_b, &b_full[stage], kb * kBK, tok[4 * g],
                                        tok[4 * g + 1], tok[4 * g + 2], tok[4 * g + 3], pol_x);
                    } else {
                        for (int b = 0; b < nbox; ++b)
                            tma_load_2d(sb + b * C::kBox, &tm_b, &b_full[stage], kb * kBK,
                                        static_cast<int>(it.row0) + b * BOXN, pol_x);
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == BSTAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            stage = __shfl_sync(0xffffffffu, stage, 0);
            phase = __shfl_sync(0xffffffffu, phase, 0);
            __syncwarp();  // tok[] is rewritten for the next item only after lane 0 issued this one
        }
        if (lane == 0)
            for (int s = 0; s < BSTAGES; ++s)
                if ((issued >> s) & 1u) mbar_wait(&b_full[s], (issued_phase >> s) & 1u, p.timeout);
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer: A from the TMEM ring, B from the smem ring ----------------
            int bstage = 0;
            uint32_t bphase = 0, kstep = 0, uses = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
                const uint32_t idesc = umma_idesc_bf16(kBM, it.n_mma);
                const int u = slots_of<GATE_UP, SLOT_COLS>(it.n_mma);
                const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
                for (int i = 0; i < u && ok; ++i) {
                    const uint32_t c = uses + i;
                    ok = mbar_wait(&acc_empty[c % NSLOT], ((c / NSLOT) & 1u) ^ 1u, p.timeout);
                }
                if (!ok) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + static_cast<uint32_t>(s0 * SLOT_COLS);
                const uint32_t d1 =
                    tmem_base + static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
                for (int kb = 0; kb < n_kb; ++kb, ++kstep) {
                    const uint32_t j = kstep % ASTAGES;
                    if (!mbar_wait(&a_ready[j], (kstep / ASTAGES) & 1u, p.timeout) ||
                        !mbar_wait(&b_full[bstage], bphase, p.timeout)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t db = umma_desc_sw128(smem_u32(smem + C::kBOff + bstage * C::kB));
                    const uint32_t a0 = tmem_base + static_cast<uint32_t>(C::kACol + j * C::kNumA * 32);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        // 16 bf16 K elements = 8 TMEM columns of A; +32 bytes in the B swizzle row = +2
                        umma_bf16_ta(d0, a0 + 8 * kk, db + 2 * kk, idesc, accum);
                        if (GATE_UP) umma_bf16_ta(d1, a0 + 32 + 8 * kk, db + 2 * kk, idesc, accum);
                    }
                    umma_commit(&a_free[j]);        // A ring stage and B stage are free once these MMAs
                    umma_commit(&b_empty[bstage]);  // have completed
                    if (++bstage == BSTAGES) {
                        bstage = 0;
                        bphase ^= 1u;
                    }
                }
                if (!ok) break;
                for (int i = 0; i < u; ++i) umma_commit(&acc_full[(uses + i) % NSLOT]);
                uses += u;
            }
            umma_commit(drain);  // all issued MMAs complete before TMEM is released
            mbar_wait(drain, 0, p.timeout);
        }
    } else if (warp >= 4 && warp < 8) {
        if constexpr (FP4)
            gemm_epilogue_scaled<GATE_UP, BN, NSLOT, SLOT_COLS>(warp - 4, tile_start, total, p, acc, tmem_base,
                                                                acc_full, acc_empty);
        else
            gemm_epilogue<GATE_UP, BN, NSLOT, SLOT_COLS, false, 1>(warp - 4, 0, tile_start, total, p, tmem_base,
                                                                   acc_full, acc_empty);
    } else if (warp >= 8) {
        // ---------------- converters: codes (smem) -> bf16 A ring (TMEM) ----------------
        // Converter warp wc = w - 8 owns TMEM lane quadrant wc % 4 (weight rows r = 32 (wc % 4) + lane)
        // and units u = wc / 4 + i * kConvWarps / 4 (i < kConvUnits) = (A tile u / 2, quarter u % 2) of
        // each 64-wide k-step: per unit a thread reads 32 codes (E4M3: two 16-byte chunks of the
        // 128-byte-swizzled row r, one scale code; E2M1: one chunk, two scale codes), releases the
        // weight stage after its last k-step, and writes the 32 bf16 values to 16 TMEM columns of
        // lane r.
        const int wc = warp - 8;
        const int r = 32 * (wc & 3) + lane;
        const uint32_t lane_base = static_cast<uint32_t>(32 * (wc & 3)) << 16;
        int stage = 0;
        uint32_t phase = 0, kstep = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            for (int kb = 0; kb < n_kb; ++kb, ++kstep) {
                const uint32_t j = kstep % ASTAGES;
                const int h = kb % C::kSteps;  // 64-wide k-step within the weight stage
                const bool last = h == C::kSteps - 1 || kb == n_kb - 1;
                ok = __all_sync(0xffffffffu, (h != 0 || mbar_wait(&w8_full[stage], phase, p.timeout)) &&
                                                 mbar_wait(&a_free[j], ((kstep / ASTAGES) & 1u) ^ 1u, p.timeout));
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + stage * C::kW8Stage);
                uint4 q[C::kConvUnits][2];
                uint32_t c[C::kConvUnits][2];
                bool big = false;
#pragma unroll
                for (int i = 0; i < C::kConvUnits; ++i) {
                    const int u = (wc >> 2) + i * (C::kConvWarps / 4);
                    const int a = u >> 1, hf = u & 1;
                    const uint32_t src = st + a * C::kA8 + r * 128;
                    const uint32_t sc = st + C::kScOff + a * C::kSc + r;
                    if (FP4) {
                        // 16 bytes = 32 codes at K 64h + 32hf of the stage: chunk 2h + hf; blocks of 16
                        q[i][0] = lds128(src + (((2 * h + hf) ^ (r & 7)) << 4));
                        c[i][0] = lds_u8(sc + (4 * h + 2 * hf) * kBM);
                        c[i][1] = lds_u8(sc + (4 * h + 2 * hf + 1) * kBM);
                    } else {
                        const int ch = 4 * h + 2 * hf;  // first 16-byte chunk of this thread's 32 codes
                        q[i][0] = lds128(src + ((ch ^ (r & 7)) << 4));
                        q[i][1] = lds128(src + (((ch + 1) ^ (r & 7)) << 4));
                        c[i][0] = lds_u8(sc + (2 * h + hf) * kBM);
                        big |= c[i][0] > 134u;
                    }
                }
                if (!FP4) big = __any_sync(0xffffffffu, big);  // a scale code that needs the second factor
                uint32_t o[C::kConvUnits][16];
#pragma unroll
                for (int i = 0; i < C::kConvUnits; ++i) {
                    if (FP4) {
                        const uint32_t qw[4] = {q[i][0].x, q[i][0].y, q[i][0].z, q[i][0].w};
                        const uint32_t f[2] = {e4m3_scale_factor(c[i][0]), e4m3_scale_factor(c[i][1])};
#pragma unroll
                        for (int b = 0; b < 16; ++b)  // byte b holds K 2b, 2b+1: TMEM column b of the unit
                            o[i][b] = e2m1x2_to_bf16x2((qw[b >> 2] >> (8 * (b & 3))) & 0xFFu, f[b >> 3]);
                    } else {
                        const uint32_t qw[8] = {q[i][0].x, q[i][0].y, q[i][0].z, q[i][0].w,
                                                q[i][1].x, q[i][1].y, q[i][1].z, q[i][1].w};
                        const uint32_t f1 = fp8_factor1(c[i][0]);
#pragma unroll
                        for (int w = 0; w < 8; ++w) e4m3x4_to_bf16x4(qw[w], f1, o[i][2 * w], o[i][2 * w + 1]);
                        if (big) {
                            const uint32_t f2 = fp8_factor2(c[i][0]);
#pragma unroll
                            for (int e = 0; e < 16; ++e) o[i][e] = bf16x2_mul(o[i][e], f2);
                        }
                    }
                }
                if (last) {
                    // the codes are consumed (the values above depend on them): hand the stage back
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&w8_empty[stage]);
                    if (++stage == W8STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
#pragma unroll
                for (int i = 0; i < C::kConvUnits; ++i) {
                    const int u = (wc >> 2) + i * (C::kConvWarps / 4);
                    const int a = u >> 1, hf = u & 1;
                    const uint32_t col = static_cast<uint32_t>(C::kACol + (j * C::kNumA + a) * 32 + hf * 16);
                    tmem_st16(tmem_base + lane_base + col, o[i]);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_ready[j]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace beam
