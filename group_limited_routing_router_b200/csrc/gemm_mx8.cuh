// Grouped expert GEMMs on the block-scaled FP8 tensor-core path: tcgen05.mma kind::mxf8f6f4 with
// E4M3 weights and E4M3 activations, one UE8M0 scale per 32 K elements on each side, FP32
// accumulation in TMEM.  The weights are an MXFP8 checkpoint ("Checkpoint formats: BF16, FP8, and
// NVFP4": "Welcome Beam" page, TL;DR); the activations (x for the gate/up projection, h for the
// down projection) are quantised to MXFP8 per row in blocks of 32 along K, the reading this path
// takes (the pages give no FP8 recipe).
//
//   G1 (gate/up + SwiGLU): h[r, i] = SiLU(x~[r] . W_gate[e, i]) * (x~[r] . W_up[e, i]) in FP32,
//        then h~ = MXFP8(h) per row: blocks of 32 consecutive i are the 32 lanes of one epilogue
//        warp, so the block maximum is a warp reduction; codes h_q [R][I], scales h_s [R][I/32].
//   G2 (down): o[r, j] = h~[r] . W_down[e, j]  (FP32, stored bf16)
//
// Same work items, swap-AB orientation (weight rows on the MMA's M side, the expert's tokens on N),
// accumulator slots and persistent grid as gemm.cuh.  Per stage K = 128 (one 128-byte row of E4M3
// per operand row, 128-byte swizzle), i.e. four MMAs of K = 32, one per scale block.
//
// Scale factors.  The MMA reads them from TMEM: for an operand of up to 128 rows and one stage,
// a 512-byte atom byte[16 (r % 32) + 4 (r / 32) + kb] (row r, K-block kb of the stage) copied by
// tcgen05.cp .32x128b.warpx4 into four TMEM columns (row r at lane r % 32 of every lane quarter,
// column r / 32, byte kb); a B operand of up to 256 rows takes two atoms (eight columns).  The MMA
// of K-block kb selects byte kb (scale-factor id in the instruction descriptor and in the top two
// bits of the TMEM address).  Each smem stage has its own TMEM scale columns.
//
// Warp roles (384 threads):
//   warp 0 lane 0  TMA: A tile(s) [128 rows x 128 B], their raw scale tiles [4 K-blocks][128 rows]
//                  (the checkpoint's K-block-major layout), B rows (tiled boxes of dispatch-ordered
//                  rows, or gather4 of token rows);
//   warp 1         TMEM owner; lane 0 issues tcgen05.cp (scales) and tcgen05.mma;
//   warp 2         scale-factor builder: per stage, B's scales straight from global memory (one
//                  32-bit word = the stage's 4 K-blocks of one row) and A's from the raw tiles
//                  (a 4x4 byte transpose per lane), written as atoms; then fence.proxy.async and
//                  the stage's sf_ready barrier;
//   warps 4..11    epilogue: two warps per TMEM lane quarter (warp w reads lanes 32 (w % 4)..+31),
//                  taking alternate 16-column chunks of the item's tokens.
// 4-bit variant (FP4 = true): tcgen05.mma kind::mxf4nvf4 .block16 with NVFP4 weights (E2M1 code
// pairs, one E4M3 scale per 16 K elements, an FP32 scale per weight matrix) and NVFP4 activations
// (x with a power-of-two scale per token, h with scale 1; E4M3 scale per 16, E2M1 elements).  A
// 128-byte operand row then holds K = 256, one MMA takes K = 64 and reads one 32-bit word of four
// scales per row, so each MMA of the stage has its own set of atoms (four per operand and stage).
// The FP32 scales multiply the accumulators in the epilogues (G1: weight matrix x token; G2: weight
// matrix).
// Every wait is bounded (status word BEAM_MOE_ERR_DEVICE_TIMEOUT on expiry).
#pragma once

#include "gemm.cuh"

namespace beam {

constexpr int kMxBK = 128;        // K per stage (bytes of an E4M3 row)
constexpr int kMxThreads = 384;   // warps 0..3 producer / MMA / scale factors / idle, 4..11 epilogue
constexpr int kMxEpiWarps = 8;
constexpr int kMxAtom = 512;      // scale atom: 128 rows x 4 K-blocks

template <bool GATE_UP, int BN, int BOXN, int STAGES, int NSLOT, int SLOT_COLS, bool GATHER, bool FP4 = false>
struct Mx8GemmCfg {
    static constexpr int kNumA = GATE_UP ? 2 : 1;
    static constexpr int kA = kBM * kMxBK;                 // 16 KB
    static constexpr int kB = BN * kMxBK;
    static constexpr int kBox = BOXN * kMxBK;
    static constexpr int kSfbAtoms = (BN + 127) / 128;
    static constexpr int kSets = FP4 ? 4 : 1;              // atom sets per stage (one per MMA for FP4)
    static constexpr int kKbStage = FP4 ? 16 : 4;          // scale blocks per row per stage
    static constexpr int kRawA = kKbStage * kBM;           // raw scale tile [K-blocks][128 rows]
    static constexpr int kSetAtoms = kNumA + kSfbAtoms;    // atoms of one set: A tile(s), then B
    // stage: [A tiles][B][raw SFA x kNumA][atom sets]
    static constexpr int kBOff = kNumA * kA;
    static constexpr int kRawOff = kBOff + kB;
    static constexpr int kAtomOff = kRawOff + kNumA * kRawA;
    static constexpr int kStage = (kAtomOff + kSets * kSetAtoms * kMxAtom + 1023) / 1024 * 1024;
    static constexpr int kSfColsPerSet = 4 * kSetAtoms;
    static constexpr int kSfColsPerStage = kSets * kSfColsPerSet;
    static constexpr int kSfCol = NSLOT * SLOT_COLS;       // first TMEM scale column
    static constexpr int kTmemCols = 512;
    static constexpr int kBarOff = STAGES * kStage;
    // full / sf_ready / empty per stage, acc_full / acc_empty per slot, drain, then the TMEM address
    static constexpr int kBarBytes = ((3 * STAGES + 2 * NSLOT + 1) * 8 + 4 + 15) / 16 * 16;
    static constexpr int kTileOff = kBarOff + kBarBytes;                 // item prefix [E + 1]
    static constexpr int kTokOff = kTileOff + 4 * (kPmMaxE + 1);         // GATHER: token of each row [BN]
    static constexpr int kEpiOff = (kTokOff + (GATHER ? 4 * BN : 0) + 15) / 16 * 16;  // gate/up epilogue: per-warp staging of h~
    static constexpr int kEpiWarp = GATE_UP ? 16 * 32 + 16 * 2 : 0;     // 16 columns x (32 code bytes + 2 scale bytes)
    static constexpr int kSmem = 1024 + kEpiOff + kMxEpiWarps * kEpiWarp + 64;
    static_assert(kA % 1024 == 0 && kB % 1024 == 0 && (GATHER || kBox % 1024 == 0), "swizzled tiles");
    static_assert(BN % BOXN == 0 && BN % 16 == 0 && BN <= 256, "token tile");
    static_assert(!GATHER || BOXN == 1, "gathered B rows: one-row boxes, four per instruction");
    static_assert(kSfCol + STAGES * kSfColsPerStage <= 512, "TMEM has 512 columns");
    static_assert(GATE_UP ? (BN <= SLOT_COLS && (NSLOT >= 2 || BN <= SLOT_COLS / 2)) : BN <= SLOT_COLS,
                  "an item must fit in its TMEM slots");
    static_assert(kSmem + 256 <= 232448, "shared memory per CTA (dynamic + the kernel's static bytes)");
};

struct Mx8Params {
    const int32_t *counts;     // [E]
    const int64_t *offsets;    // [E + 1]
    int E;
    int K;                     // reduction length in elements (G1: H, G2: I); a multiple of 128 (FP4: 256)
    int M;                     // weight rows (G1: I, G2: H)
    int weights_once;
    long long timeout;
    const int32_t *row_src;    // dispatch row -> (token, slot) pair q
    int topk;
    // activation scales: B row n of an item is dispatch row r = row0 + n; its scale row is
    // s_rows[sf_token ? row_src[r] / topk : r] with K/32 bytes per row
    const uint8_t *b_scale;
    int sf_token;
    // G1 outputs: h codes [R][M] (FP4: [R][M/2], two codes per byte) and scales [R][M/32] (FP4:
    // [R][M/16]); G2 output: o [R][M] bf16
    uint8_t *h_q;
    uint8_t *h_s;
    __nv_bfloat16 *o;
    // FP4: FP32 scale per weight matrix [E] (g_a0: gate or down; g_a1: up) and per token [T]
    const float *g_a0;
    const float *g_a1;
    const float *g_tok;
};

// Instruction descriptor, kind::mxf8f6f4 with block scaling: A and B E4M3 (format 0), K-major,
// N >> 3 at [17,23), UE8M0 scales (bit 23), M >> 4 at [24,29); scale-factor ids at [4,6) (B) and
// [29,31) (A) select the K-block's byte.
__device__ __forceinline__ uint32_t umma_idesc_mx8(int M, int N, uint32_t sf_id) {
    return (sf_id << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24) |
           (sf_id << 29);
}

__device__ __forceinline__ void umma_mx8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), UE4M3 scales (bit 23 = 0),
// K = 64 per MMA, one scale word (four blocks of 16) per row.
__device__ __forceinline__ uint32_t umma_idesc_nv4(int M, int N) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_nv4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Shared-memory descriptor of a 512-byte scale atom for tcgen05.cp .32x128b: 32 rows of 16 bytes,
// no swizzle, 8-row core matrices 128 bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128u >> 4) << 16;
    d |= static_cast<uint64_t>(128u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    return d;
}

__device__ __forceinline__ void tmem_cp_sf_atom(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Atom byte offset of (row r, word of the stage's 4 K-blocks) for rows < 256 (two atoms).
__device__ __forceinline__ int sf_atom_off(int r) { return (r >> 7) * kMxAtom + 16 * (r & 31) + 4 * ((r >> 5) & 3); }

// UE8M0 code of a block whose largest magnitude is amax (finite): 127 + the smallest e with
// amax <= 448 * 2^e; 0 for amax = 0.  448 = 1.75 * 2^8, so e = E - 8, plus one when the mantissa
// of amax exceeds 1.75.  Returns the code and the FP32 factor 2^-e that scales the block into E4M3.
__device__ __forceinline__ uint32_t mx_scale_code(float amax, float &inv) {
    const uint32_t u = __float_as_uint(amax);
    if (amax == 0.0f) {
        inv = 0.0f;
        return 0u;
    }
    const int E = static_cast<int>((u >> 23) & 0xFFu) - 127;
    const int e = E - 8 + ((u & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
    return static_cast<uint32_t>(e + 127);
}

// Two FP32 values (already scaled into E4M3 range) -> two E4M3 codes (nearest, ties to even).
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two FP32 values -> two E2M1 codes (nearest, ties to even, saturating at 6): lo in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi),
        "f"(lo));
    return r;
}

// An E4M3 code -> its value (exact in FP32).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    const uint16_t c = static_cast<uint16_t>(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// The E2M1 code (sign in bit 3) of the value nearest to v / s, ties to even, saturating at 6, for an
// E4M3 scale s > 0, without dividing: the rounding boundaries between the E2M1 magnitudes (0.25,
// 0.75, 1.25, 1.75, 2.5, 3.5, 5) times s are exact in FP32 (at most 3 + 4 significant bits), so
// comparing |v| with them decides the rounding of the exact quotient.  A value on a boundary goes
// to the even code: above the boundaries with an odd index only when equal.
__device__ __forceinline__ uint32_t e2m1_code_of_quotient(float v, float s) {
    const float m = fabsf(v);
    uint32_t k = (m > 0.25f * s) + (m >= 0.75f * s) + (m > 1.25f * s) + (m >= 1.75f * s) + (m > 2.5f * s) +
                 (m >= 3.5f * s) + (m > 5.0f * s);
    return k | (v < 0.0f ? 8u : 0u);
}

// The NVFP4 block of 16 (row scale 1) of the value v held by each of 16 lanes (lanes 0..15 or 16..31):
// returns this lane's E2M1 code and sets the block's E4M3 scale code.  The block scale is the E4M3
// value nearest to amax / 6, formed as amax times a rounded 1/6 (within two FP32 ulp of the quotient,
// which moves the decision only for values that close to an E4M3 rounding boundary).
__device__ __forceinline__ uint32_t nv4_quant16(float v, uint32_t half_mask, uint32_t &scale_code) {
    const float amax = __uint_as_float(__reduce_max_sync(half_mask, __float_as_uint(fabsf(v))));
    scale_code = e4m3x2_from_f32(fminf(amax * (1.0f / 6.0f), 448.0f), 0.0f) & 0xFFu;
    const float s = e4m3_to_f32(scale_code);
    return s > 0.0f ? e2m1_code_of_quotient(v, s) : 0u;
}

// G1 epilogue with MXFP8 h: the 32 lanes of warp q hold weight rows (i) 32q..32q+31 of the tile,
// one block of 32 along i per token column.
template <int BN, int NSLOT, int SLOT_COLS>
__device__ __forceinline__ void mx8_epilogue_g1(int q, int half, const int *tile_start, int total, const Mx8Params &p,
                                                uint32_t tmem_base, uint64_t *acc_full, uint64_t *acc_empty,
                                                uint8_t *stg) {
    constexpr int kCh = (BN + 31) / 32;  // 16-column chunks of this warp (the quarter's two warps alternate)
    const int lane = threadIdx.x & 31;
    uint32_t uses = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Item it = decode_item(item, tile_start, p.E, BN, p.counts, p.offsets);
        const int u = slots_of<true, SLOT_COLS>(it.n_mma);
        bool ok = true;
        for (int i = 0; i < u && ok; ++i) {
            const uint32_t c = uses + i;
            ok = mbar_wait(&acc_full[c % NSLOT], (c / NSLOT) & 1u, p.timeout);
        }
        if (!ok) break;
        tc_fence_after();
        const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
        const int m = it.mt * kBM + q * 32 + lane;
        const bool row_ok = m < p.M;
        const int blk = (it.mt * kBM + q * 32) >> 5;  // this warp's block of 32 along i
        const bool blk_ok = blk * 32 < p.M;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(s0 * SLOT_COLS);
        const uint32_t t1 = tmem_base + lane_off +
                            static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
        // SwiGLU of this warp's columns into registers; the accumulator slots go back to the MMA before
        // the quantisation, so the next item's products overlap it
        float hv[kCh][16];
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int c = 16 * half + 32 * cc;
            if (c < it.n_valid) {
                uint32_t rg[16], ru[16];
                tmem_ld16(t0 + c, rg);
                tmem_ld16(t1 + c, ru);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    hv[cc][j] = row_ok ? silu_mul(__uint_as_float(rg[j]), __uint_as_float(ru[j])) : 0.0f;
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int i = 0; i < u; ++i) mbar_arrive(&acc_empty[(uses + i) % NSLOT]);
        uses += u;
        // the warp's 32 rows of a token column are 32 code bytes and one scale byte: staged in shared
        // memory per 16 columns, then lane j writes column j's pieces (two 16-byte and one 1-byte store)
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int c = 16 * half + 32 * cc;
            if (c < it.n_valid) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    // the block maximum: |h| >= 0, so its bit pattern orders like the value
                    const float amax =
                        __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hv[cc][j]))));
                    float inv;
                    const uint32_t code = mx_scale_code(amax, inv);
                    stg[32 * j + lane] = static_cast<uint8_t>(e4m3x2_from_f32(hv[cc][j] * inv, 0.0f) & 0xFFu);
                    if (lane == 0) stg[512 + j] = static_cast<uint8_t>(code);
                }
                __syncwarp();
                if (lane < 16 && c + lane < it.n_valid && blk_ok) {
                    const int64_t r = it.row0 + c + lane;
                    const int m0 = it.mt * kBM + q * 32;  // this warp's first row (a multiple of 32)
                    if (m0 + 32 <= p.M) {
                        uint4 *dst = reinterpret_cast<uint4 *>(p.h_q + r * p.M + m0);
                        dst[0] = *reinterpret_cast<const uint4 *>(stg + 32 * lane);
                        dst[1] = *reinterpret_cast<const uint4 *>(stg + 32 * lane + 16);
                    }
                    p.h_s[r * (p.M >> 5) + blk] = stg[512 + lane];
                }
                __syncwarp();
            }
        }
    }
}

// G1 epilogue of the 4-bit path: accumulators times the FP32 scales (weight matrix x token), SwiGLU,
// then h~ = NVFP4(h) with row scale 1: lanes 0..15 and 16..31 of warp q are two blocks of 16 along i.
// Codes are packed two per byte (even i in the low nibble) by the even lanes.
template <int BN, int NSLOT, int SLOT_COLS>
__device__ __forceinline__ void nv4_epilogue_g1(int q, int half, const int *tile_start, int total, const Mx8Params &p,
                                                uint32_t tmem_base, uint64_t *acc_full, uint64_t *acc_empty,
                                                uint8_t *stg) {
    constexpr int kCh = (BN + 31) / 32;  // 16-column chunks of this warp (the quarter's two warps alternate)
    const int lane = threadIdx.x & 31;
    const uint32_t half_mask = lane < 16 ? 0x0000FFFFu : 0xFFFF0000u;
    uint32_t uses = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Item it = decode_item(item, tile_start, p.E, BN, p.counts, p.offsets);
        const int u = slots_of<true, SLOT_COLS>(it.n_mma);
        // token scales of this warp's columns (lanes j and j + 16 hold column c + j), loaded before the
        // accumulators are ready
        float gtl[kCh];
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int jl = 16 * half + 32 * cc + (lane & 15);
            gtl[cc] = jl < it.n_valid ? __ldg(p.g_tok + p.row_src[it.row0 + jl] / p.topk) : 0.0f;
        }
        const float gg = __ldg(p.g_a0 + it.e), gu = __ldg(p.g_a1 + it.e);
        bool ok = true;
        for (int i = 0; i < u && ok; ++i) {
            const uint32_t c = uses + i;
            ok = mbar_wait(&acc_full[c % NSLOT], (c / NSLOT) & 1u, p.timeout);
        }
        if (!ok) break;
        tc_fence_after();
        const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
        const int m = it.mt * kBM + q * 32 + lane;
        const bool row_ok = m < p.M;
        const int blk = m >> 4;  // this lane's block of 16 along i
        const bool blk_ok = (blk << 4) < p.M;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(s0 * SLOT_COLS);
        const uint32_t t1 = tmem_base + lane_off +
                            static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
        // SwiGLU of this warp's columns into registers; the accumulator slots go back to the MMA before
        // the quantisation, so the next item's products overlap it
        float hv[kCh][16];
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int c = 16 * half + 32 * cc;
            if (c < it.n_valid) {
                uint32_t rg[16], ru[16];
                tmem_ld16(t0 + c, rg);
                tmem_ld16(t1 + c, ru);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float gt = __shfl_sync(0xffffffffu, gtl[cc], j);
                    hv[cc][j] = row_ok && c + j < it.n_valid
                                    ? silu_mul(__uint_as_float(rg[j]) * (gg * gt), __uint_as_float(ru[j]) * (gu * gt))
                                    : 0.0f;
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int i = 0; i < u; ++i) mbar_arrive(&acc_empty[(uses + i) % NSLOT]);
        uses += u;
        // the warp's 32 rows of a token column are 16 code bytes and 2 scale bytes: staged in shared
        // memory per 16 columns, then lane j writes column j's pieces (one 16-byte and one 2-byte store)
#pragma unroll
        for (int cc = 0; cc < kCh; ++cc) {
            const int c = 16 * half + 32 * cc;
            if (c < it.n_valid) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    uint32_t sc;
                    const uint32_t code = nv4_quant16(hv[cc][j], half_mask, sc);
                    const uint32_t odd = __shfl_down_sync(0xffffffffu, code, 1);
                    if ((lane & 1) == 0) stg[16 * j + (lane >> 1)] = static_cast<uint8_t>(code | (odd << 4));
                    if ((lane & 15) == 0) stg[256 + 2 * j + (lane >> 4)] = static_cast<uint8_t>(sc);
                }
                __syncwarp();
                if (lane < 16 && c + lane < it.n_valid && row_ok && blk_ok) {
                    const int64_t r = it.row0 + c + lane;
                    const int m0 = it.mt * kBM + q * 32;  // this warp's first row (a multiple of 32)
                    *reinterpret_cast<uint4 *>(p.h_q + r * (p.M >> 1) + (m0 >> 1)) =
                        *reinterpret_cast<const uint4 *>(stg + 16 * lane);
                    *reinterpret_cast<uint16_t *>(p.h_s + r * (p.M >> 4) + (m0 >> 4)) =
                        *reinterpret_cast<const uint16_t *>(stg + 256 + 2 * lane);
                }
                __syncwarp();
            }
        }
    }
}

// G2 epilogue: o rows in dispatch order, FP32 accumulators (FP4: times the weight matrix's FP32 scale)
// rounded to bf16.
template <int BN, int NSLOT, int SLOT_COLS, bool FP4>
__device__ __forceinline__ void mx8_epilogue_g2(int q, int half, const int *tile_start, int total, const Mx8Params &p,
                                                uint32_t tmem_base, uint64_t *acc_full, uint64_t *acc_empty) {
    const int lane = threadIdx.x & 31;
    uint32_t uses = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Item it = decode_item(item, tile_start, p.E, BN, p.counts, p.offsets);
        if (!mbar_wait(&acc_full[uses % NSLOT], (uses / NSLOT) & 1u, p.timeout)) break;
        tc_fence_after();
        const int m = it.mt * kBM + q * 32 + lane;
        const float gd = FP4 ? __ldg(p.g_a0 + it.e) : 1.0f;
        const uint32_t t0 =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>((uses % NSLOT) * SLOT_COLS);
        for (int c = 16 * half; c < it.n_valid; c += 32) {
            uint32_t r0[16];
            tmem_ld16(t0 + c, r0);
            tmem_ld_wait();
            if (m < p.M) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c + j < it.n_valid)
                        p.o[(it.row0 + c + j) * p.M + m] = __float2bfloat16_rn(__uint_as_float(r0[j]) * gd);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[uses % NSLOT]);
        uses += 1;
    }
}

template <bool GATE_UP, int BN, int BOXN, int STAGES, int NSLOT, int SLOT_COLS, bool GATHER, bool FP4>
__global__ void __launch_bounds__(kMxThreads, 1)
    grouped_gemm_mx8_kernel(const __grid_constant__ CUtensorMap tm_a0,  // W_gate (G1) / W_down (G2): E4M3 [E][M][K]
                            const __grid_constant__ CUtensorMap tm_a1,  // W_up (G1); unused for G2
                            const __grid_constant__ CUtensorMap tm_s0,  // scale codes [E][K/32][M] of a0
                            const __grid_constant__ CUtensorMap tm_s1,  // of a1
                            const __grid_constant__ CUtensorMap tm_b,   // B rows E4M3 [rows][K]
                            const Mx8Params p) {
    using C = Mx8GemmCfg<GATE_UP, BN, BOXN, STAGES, NSLOT, SLOT_COLS, GATHER, FP4>;
    extern __shared__ uint8_t mx8_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(mx8_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *sf_ready = full + STAGES;
    uint64_t *empty = sf_ready + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint64_t *acc_empty = acc_full + NSLOT;
    uint64_t *drain = acc_empty + NSLOT;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *tile_start = reinterpret_cast<int *>(smem + C::kTileOff);
    int *tok = reinterpret_cast<int *>(smem + C::kTokOff);  // GATHER: token of each row of the item

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int n_mt = (p.M + kBM - 1) / kBM;
    const int n_kb = p.K / (FP4 ? 2 * kMxBK : kMxBK);  // stages: one 128-byte row of codes each

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sf_ready[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < NSLOT; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kMxEpiWarps);
        }
        mbar_init(drain, 1);
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
        // ---------------- TMA producer ----------------
        const uint64_t pol_w = p.weights_once ? policy_evict_first() : policy_evict_normal();
        const uint64_t pol_x = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued = 0, issued_phase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
            if (GATHER) {
                for (int r = lane; r < it.n_mma; r += 32) {
                    const int rr = r < it.n_valid ? r : 0;
                    tok[r] = p.row_src[it.row0 + rr] / p.topk;
                }
                __syncwarp();
            }
            if (lane == 0) {
                const int nbox = GATHER ? (it.n_mma + 3) / 4 : (it.n_mma + BOXN - 1) / BOXN;
                const uint32_t bytes = C::kNumA * (C::kA + C::kRawA) + nbox * (GATHER ? 4 * kMxBK : C::kBox);
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + stage * C::kStage;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_3d(st, &tm_a0, &full[stage], kb * kMxBK, it.mt * kBM, it.e, pol_w);
                    tma_load_3d(st + C::kRawOff, &tm_s0, &full[stage], it.mt * kBM, C::kKbStage * kb, it.e, pol_w);
                    if (GATE_UP) {
                        tma_load_3d(st + C::kA, &tm_a1, &full[stage], kb * kMxBK, it.mt * kBM, it.e, pol_w);
                        tma_load_3d(st + C::kRawOff + C::kRawA, &tm_s1, &full[stage], it.mt * kBM, C::kKbStage * kb,
                                    it.e, pol_w);
                    }
                    uint8_t *sb = st + C::kBOff;
                    if (GATHER) {
                        for (int g = 0; g < nbox; ++g)
                            tma_gather4(sb + g * 4 * kMxBK, &tm_b, &full[stage], kb * kMxBK, tok[4 * g], tok[4 * g + 1],
                                        tok[4 * g + 2], tok[4 * g + 3], pol_x);
                    } else {
                        for (int bx = 0; bx < nbox; ++bx)
                            tma_load_2d(sb + bx * C::kBox, &tm_b, &full[stage], kb * kMxBK,
                                        static_cast<int>(it.row0) + bx * BOXN, pol_x);
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            stage = __shfl_sync(0xffffffffu, stage, 0);
            phase = __shfl_sync(0xffffffffu, phase, 0);
        }
        if (lane == 0)
            for (int s = 0; s < STAGES; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_phase >> s) & 1u, p.timeout);
    } else if (warp == 2) {
        // ---------------- scale-factor builder ----------------
        const int kbs = p.K / (FP4 ? 16 : 32);  // scale bytes per activation row
        constexpr int kRowIt = (BN + 31) / 32;
        // B's scale words are loaded two stages ahead of the stage they belong to (a load cursor that
        // runs over the same (item, kb) sequence), so their global-memory latency overlaps the
        // building of the two stages before; each item's scale rows are looked up once.
        int l_item = blockIdx.x, l_kb = 0;
        int64_t l_srow[kRowIt];
        auto l_rows = [&]() {
            if (l_item >= total) return;
            const Item li = decode_item(l_item, tile_start, E, BN, p.counts, p.offsets);
#pragma unroll
            for (int i = 0; i < kRowIt; ++i) {
                const int n = lane + 32 * i;
                const int64_t r = li.row0 + n;
                l_srow[i] = n < li.n_valid ? (p.sf_token ? static_cast<int64_t>(p.row_src[r] / p.topk) : r) : -1;
            }
        };
        // the stage's scale words of every row (FP8: one word = 4 K-blocks; FP4: four words, one per MMA)
        auto l_next = [&](uint4 (&wb)[kRowIt]) {
#pragma unroll
            for (int i = 0; i < kRowIt; ++i) {
                wb[i] = make_uint4(0u, 0u, 0u, 0u);
                if (l_item < total && l_srow[i] >= 0) {
                    if (FP4) wb[i] = __ldg(reinterpret_cast<const uint4 *>(p.b_scale + l_srow[i] * kbs + 16 * l_kb));
                    else wb[i].x = __ldg(reinterpret_cast<const uint32_t *>(p.b_scale + l_srow[i] * kbs + 4 * l_kb));
                }
            }
            if (++l_kb == n_kb) {
                l_kb = 0;
                l_item += gridDim.x;
                l_rows();
            }
        };
        l_rows();
        uint4 wb[kRowIt], wb1[kRowIt];
        l_next(wb);
        l_next(wb1);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            for (int kb = 0; kb < n_kb && ok; ++kb) {
                uint4 wb2[kRowIt];
                l_next(wb2);
                ok = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase, p.timeout));
                if (!ok) break;
                uint8_t *st = smem + stage * C::kStage;
                uint8_t *atoms = st + C::kAtomOff;
#pragma unroll
                for (int i = 0; i < kRowIt; ++i) {
                    const int n = lane + 32 * i;
                    if (n < BN) {
                        const uint32_t w4[4] = {wb[i].x, wb[i].y, wb[i].z, wb[i].w};
#pragma unroll
                        for (int set = 0; set < C::kSets; ++set)
                            *reinterpret_cast<uint32_t *>(atoms + (set * C::kSetAtoms + C::kNumA) * kMxAtom +
                                                          sf_atom_off(n)) = w4[set];
                    }
                }
                // A: raw [K-blocks][128 rows] -> atoms; lane l takes rows 4l..4l+3, set by set
#pragma unroll
                for (int a = 0; a < C::kNumA; ++a) {
                    const uint8_t *raw = st + C::kRawOff + a * C::kRawA;
#pragma unroll
                    for (int set = 0; set < C::kSets; ++set) {
                        uint32_t w[4];
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            w[k4] = *reinterpret_cast<const uint32_t *>(raw + (4 * set + k4) * kBM + 4 * lane);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t sel = static_cast<uint32_t>(i | ((4 + i) << 4));
                            const uint32_t lo = __byte_perm(w[0], w[1], sel);
                            const uint32_t hi = __byte_perm(w[2], w[3], sel);
                            *reinterpret_cast<uint32_t *>(atoms + (set * C::kSetAtoms + a) * kMxAtom +
                                                          sf_atom_off(4 * lane + i)) = __byte_perm(lo, hi, 0x5410);
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[stage]);
#pragma unroll
                for (int i = 0; i < kRowIt; ++i) {
                    wb[i] = wb1[i];
                    wb1[i] = wb2[i];
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            int stage = 0;
            uint32_t phase = 0;
            uint32_t uses = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
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
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(&sf_ready[stage], phase, p.timeout)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * C::kStage);
                    const uint32_t atoms = sa + C::kAtomOff;
                    const uint32_t sf_col = tmem_base + static_cast<uint32_t>(C::kSfCol + stage * C::kSfColsPerStage);
#pragma unroll
                    for (int a = 0; a < C::kSets * C::kSetAtoms; ++a)
                        tmem_cp_sf_atom(sf_col + 4 * a, sf_atom_desc(atoms + a * kMxAtom));
                    const uint64_t da0 = umma_desc_sw128(sa);
                    const uint64_t da1 = umma_desc_sw128(sa + C::kA);
                    const uint64_t db = umma_desc_sw128(sa + C::kBOff);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint32_t accum = (kb > 0 || k4 > 0) ? 1u : 0u;
                        // +32 bytes along K inside the swizzle row = +2 in the 16-byte address field
                        if (FP4) {
                            // MMA k4 reads its own atom set (a whole scale word per row)
                            const uint32_t set_col = sf_col + static_cast<uint32_t>(k4 * C::kSfColsPerSet);
                            const uint32_t idesc = umma_idesc_nv4(kBM, it.n_mma);
                            umma_nv4(d0, da0 + 2 * k4, db + 2 * k4, idesc, set_col, set_col + 4 * C::kNumA, accum);
                            if (GATE_UP) umma_nv4(d1, da1 + 2 * k4, db + 2 * k4, idesc, set_col + 4, set_col + 4 * C::kNumA,
                                                  accum);
                        } else {
                            // MMA k4 reads byte k4 of the stage's scale words
                            const uint32_t idesc = umma_idesc_mx8(kBM, it.n_mma, static_cast<uint32_t>(k4));
                            const uint32_t byte = static_cast<uint32_t>(k4) << 30;
                            const uint32_t sfb = sf_col + 4 * C::kNumA;
                            umma_mx8(d0, da0 + 2 * k4, db + 2 * k4, idesc, sf_col | byte, sfb | byte, accum);
                            if (GATE_UP)
                                umma_mx8(d1, da1 + 2 * k4, db + 2 * k4, idesc, (sf_col + 4) | byte, sfb | byte, accum);
                        }
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                for (int i = 0; i < u; ++i) umma_commit(&acc_full[(uses + i) % NSLOT]);
                uses += u;
            }
            umma_commit(drain);
            mbar_wait(drain, 0, p.timeout);
        }
    } else if (warp >= 4) {
        const int q = warp & 3, half = (warp - 4) >> 2;
        uint8_t *stg = smem + C::kEpiOff + (warp - 4) * C::kEpiWarp;
        if (GATE_UP && FP4)
            nv4_epilogue_g1<BN, NSLOT, SLOT_COLS>(q, half, tile_start, total, p, tmem_base, acc_full, acc_empty, stg);
        else if (GATE_UP)
            mx8_epilogue_g1<BN, NSLOT, SLOT_COLS>(q, half, tile_start, total, p, tmem_base, acc_full, acc_empty, stg);
        else mx8_epilogue_g2<BN, NSLOT, SLOT_COLS, FP4>(q, half, tile_start, total, p, tmem_base, acc_full, acc_empty);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// x [T][H] bf16 -> MXFP8 codes x_q [T][H] and scale codes x_s [T][H/32]: 4 threads per block of 32,
// 8 elements each (one 16-byte load, one 8-byte store).
__global__ void __launch_bounds__(256) quant_mx8_rows_kernel(const uint4 *__restrict__ x, int64_t n_blocks,
                                                             uint2 *__restrict__ q, uint8_t *__restrict__ s) {
    const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;  // 8-element group
    const int64_t blk = t >> 2;
    const bool live = blk < n_blocks;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (live) v = __ldg(x + t);
    float f[8];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    float inv;
    const uint32_t code = mx_scale_code(amax, inv);
    uint2 out;
    out.x = e4m3x2_from_f32(f[0] * inv, f[1] * inv) | (e4m3x2_from_f32(f[2] * inv, f[3] * inv) << 16);
    out.y = e4m3x2_from_f32(f[4] * inv, f[5] * inv) | (e4m3x2_from_f32(f[6] * inv, f[7] * inv) << 16);
    if (live) {
        q[t] = out;
        if ((t & 3) == 0) s[blk] = static_cast<uint8_t>(code);
    }
}

}  // namespace beam

namespace beam {

// x [T][H] bf16 -> NVFP4 codes x_q [T][H/2] (two per byte, even k low), E4M3 scale codes x_s [T][H/16]
// and the token's power-of-two scale g[T] (the smallest g with amax_row <= 6 * 448 * g).  One CTA per
// token; each thread takes blocks of 16.
__global__ void __launch_bounds__(128) quant_nv4_rows_kernel(const uint4 *__restrict__ x, int H,
                                                             uint2 *__restrict__ q, uint8_t *__restrict__ s,
                                                             float *__restrict__ g_out) {
    __shared__ uint32_t warp_max[4];
    const int64_t t = blockIdx.x;
    const uint4 *row = x + t * (H / 8);
    const int nb = H / 16;
    uint32_t amax_bits = 0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
        const uint4 v0 = __ldg(row + 2 * b), v1 = __ldg(row + 2 * b + 1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
            amax_bits = max(amax_bits, max((w[i] << 16) & 0x7FFFFFFFu, w[i] & 0x7FFF0000u));
    }
    amax_bits = __reduce_max_sync(0xffffffffu, amax_bits);
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax_bits;
    __syncthreads();
    amax_bits = max(max(warp_max[0], warp_max[1]), max(warp_max[2], warp_max[3]));
    // 6 * 448 = 2688 = 1.3125 * 2^11: e = E - 11, plus one when the mantissa exceeds 1.3125
    float g = 1.0f;
    if (amax_bits != 0u) {
        const int E = static_cast<int>(amax_bits >> 23) - 127;
        const int e = E - 11 + ((amax_bits & 0x7FFFFFu) > 0x280000u ? 1 : 0);
        g = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
    }
    if (threadIdx.x == 0) g_out[t] = g;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
        const uint4 v0 = __ldg(row + 2 * b), v1 = __ldg(row + 2 * b + 1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float f[16];
        float bmax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            bmax = fmaxf(bmax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
        }
        const uint32_t sc = e4m3x2_from_f32(fminf(__fdiv_rn(bmax, 6.0f * g), 448.0f), 0.0f) & 0xFFu;
        const float sg = e4m3_to_f32(sc) * g;
        uint32_t packed[2] = {0u, 0u};
        if (sg > 0.0f) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                packed[i >> 2] |= e2m1x2_from_f32(__fdiv_rn(f[2 * i], sg), __fdiv_rn(f[2 * i + 1], sg)) << (8 * (i & 3));
        }
        q[t * nb + b] = make_uint2(packed[0], packed[1]);
        s[t * nb + b] = static_cast<uint8_t>(sc);
    }
}

}  // namespace beam
