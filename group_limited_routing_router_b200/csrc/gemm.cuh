// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM, TMA-fed).
//
//   G1 (gate/up + SwiGLU): for expert e and its rows r (tokens routed to e, in dispatch order)
//        h[r, i] = SiLU(x[r] . W_gate[e, i]) * (x[r] . W_up[e, i])          (FP32, stored bf16)
//   G2 (down):  o[r, j] = h[r] . W_down[e, j]                                 (FP32)
// "each a SwiGLU MLP with an intermediate size of 2,560" ("Welcome Beam" page, section "Mixture of
// Experts"); the SwiGLU product is computed in FP32 (section "Residual Stream").
//
// Orientation (swap-AB): the MMA's M side (128) walks the expert's weight rows, its N side the
// expert's tokens (N = tokens rounded up to 16, at most BN).  At the Beam shapes an expert sees
// ~8 tokens in a decode batch and 128 +- 11 in a 4096-token prefill, so one token tile covers all of
// an expert's tokens and every weight byte crosses HBM once per call.
//
// Work item = (expert e, weight-row tile mt, token tile nt of BN); a weight-row tile is 128 rows, or
// with PAIR (down projection) two adjacent 128-row tiles that share the item's token tile, so that
// each token-row byte staged from L2 feeds twice the weight bytes (as W_gate and W_up share it in G1).  Items are numbered
// expert-major, then mt, then nt, from the per-expert counts (read on the device; no host sync);
// a persistent grid of one CTA per SM takes items round-robin.
//
// Warp roles (320 threads): warp 0 lane 0 = TMA producer; warp 1 = TMEM owner, lane 0 issues
// tcgen05.mma; warps 2..9 = epilogue, two per TMEM lane quadrant (warp w reads lanes 32(w%4)..+31 and
// takes every other 16-token chunk of the item, so that an item's slots drain in half the time:
// while they drain the next item's MMAs wait whenever it needs both slots).  Shared memory is a
// STAGES-deep ring of {A tile(s) 128x64 bf16, B tile of up to BN x 64 bf16}, 128-byte swizzled by
// TMA; the B tile is loaded in boxes of BOXN rows, only as many as the item's tokens need.
//
// TMEM holds NSLOT accumulator slots of SLOT_COLS fp32 columns, used round-robin.  G2 and small G1
// items take one slot (G1: gate in its first half, up in its second half); a G1 item with more
// than SLOT_COLS/2 tokens takes two consecutive slots (gate in one, up in the other), so large
// experts stay in one token tile while small ones keep the epilogue overlapped with the next MMAs.
// Every wait is bounded (status word BEAM_MOE_ERR_DEVICE_TIMEOUT on expiry).
#pragma once

#include "common.cuh"

namespace beam {

constexpr int kBM = 128;  // weight rows per tile (UMMA M)
constexpr int kBK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int kGemmThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kGemmEpiWarps = 8;

constexpr int pow2_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }

template <bool GATE_UP, int BN, int BOXN, int STAGES, int NSLOT, int SLOT_COLS, bool GATHER = false,
          bool PAIR = false>
struct GemmCfg {
    static constexpr int kA = kBM * kBK * 2;                 // one A tile, bytes
    static constexpr int kB = BN * kBK * 2;                  // B tile, bytes (room for BN rows)
    static constexpr int kBox = BOXN * kBK * 2;              // one B box, bytes
    static constexpr int kNumA = (GATE_UP || PAIR) ? 2 : 1;   // A tiles per stage
    static constexpr int kRows = PAIR ? 2 * kBM : kBM;        // weight rows per item
    static constexpr int kStage = kNumA * kA + kB;
    static constexpr int kTmemCols = pow2_cols(NSLOT * SLOT_COLS);
    static constexpr int kBarOff = STAGES * kStage;
    static constexpr int kTokOff = kBarOff + 256 + 4 * (kPmMaxE + 1);     // gathered token ids [BN]
    static constexpr int kSmem = 1024 + kTokOff + (GATHER ? 4 * BN : 0) + 64;
    static_assert(kStage % 1024 == 0 && (GATHER || kBox % 1024 == 0), "tiles must keep 1024-byte alignment");
    static_assert(BN % BOXN == 0 && BN % 16 == 0 && BN <= 256, "token tile");
    static_assert(!GATHER || BOXN == 1, "gathered B rows come one row per box, four per instruction");
    static_assert(NSLOT * SLOT_COLS <= 512, "TMEM has 512 columns");
    static_assert((GATE_UP || PAIR) ? (BN <= SLOT_COLS && (NSLOT >= 2 || BN <= SLOT_COLS / 2)) : BN <= SLOT_COLS,
                  "an item must fit in its TMEM slots");
    static_assert(!(GATE_UP && PAIR), "PAIR is a down-projection layout");
    static_assert(kSmem <= 232448, "shared memory per CTA");
};

struct GemmParams {
    const int32_t *counts;    // [E]
    const int64_t *offsets;   // [E + 1]
    void *out;                // G1: h [R, I] bf16; G2: o [R, H] fp32 (bf16 when out_bf16)
    int E;
    int K;                    // reduction length (G1: H, G2: I)
    int M;                    // weight rows (G1: I, G2: H)
    int weights_once;         // 1: each weight tile is read once per call -> L2 evict-first
    long long timeout;
    const int32_t *row_src;   // GATHER: dispatch row -> (token, slot) pair q; token = q / topk
    int topk;
    const int32_t *out_row;   // G2 only, nullable: dispatch row r is stored at output row out_row[r]
    int out_bf16;             // G2 only: 1 stores the accumulators rounded to bf16 (RNE) instead of fp32
};

// Work-item decode from the per-CTA prefix table.
struct Item {
    int e, mt, nt, n_valid, n_mma;
    int64_t row0;
};

__device__ __forceinline__ Item decode_item(int item, const int *tile_start, int E, int BN, const int32_t *counts,
                                            const int64_t *offsets) {
    int lo = 0, hi = E - 1;  // largest e with tile_start[e] <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tile_start[mid] <= item) lo = mid;
        else hi = mid - 1;
    }
    Item it;
    it.e = lo;
    const int cnt = counts[lo];
    const int n_nt = (cnt + BN - 1) / BN;
    const int local = item - tile_start[lo];
    it.mt = local / n_nt;
    it.nt = local - it.mt * n_nt;
    it.n_valid = min(BN, cnt - it.nt * BN);
    it.n_mma = (it.n_valid + 15) & ~15;
    it.row0 = offsets[lo] + static_cast<int64_t>(it.nt) * BN;
    return it;
}

// Per-expert item counts -> exclusive prefix in tile_start[0..E] (E <= 256 <= blockDim.x, which is a
// multiple of 32 and at most 1024).  Contains __syncthreads: every thread of the block calls it.
__device__ __forceinline__ void item_prefix(const int32_t *counts, int E, int n_mt, int BN, int *tile_start) {
    __shared__ int warp_tot[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = threadIdx.x;
    const int v = e < E ? n_mt * ((counts[e] + BN - 1) / BN) : 0;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    if (e < E) tile_start[e] = base + incl - v;
    if (e == E - 1) tile_start[E] = base + incl;
}

// TMEM slots an item occupies.
// TWO: the item has two accumulators (G1: gate and up; PAIR: its two weight-row halves).
template <bool TWO, int SLOT_COLS>
__device__ __forceinline__ int slots_of(int n_mma) {
    return (TWO && n_mma > SLOT_COLS / 2) ? 2 : 1;
}

// G2: the accumulators of weight row m for the item's tokens c..c+15 go to o (fp32, or bf16 when
// out_bf16), row out_row[r] when that map is given.
__device__ __forceinline__ void store_down_row(const GemmParams &p, const Item &it, int c, int m, const uint32_t (&r)[16]) {
    if (m >= p.M) return;
    if (p.out_bf16) {
        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.out);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (c + j < it.n_valid) o[(it.row0 + c + j) * p.M + m] = __float2bfloat16_rn(__uint_as_float(r[j]));
    } else {
        float *o = reinterpret_cast<float *>(p.out);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (c + j < it.n_valid) {
                const int64_t row = it.row0 + c + j;
                const int64_t dst = p.out_row ? static_cast<int64_t>(__ldg(p.out_row + row)) : row;
                o[dst * p.M + m] = __uint_as_float(r[j]);
            }
    }
}

// G1 with two epilogue warps per lane quadrant (warp `sub` takes the 16-column chunks 16 sub + 32 i):
// SiLU(gate) * up of the thread's weight row, rounded to bf16 and kept in registers as pairs (token
// columns 2j, 2j + 1 of chunk i in hv[i][j]), so that the TMEM slots can be released before any h
// store is issued: an item with more than SLOT_COLS / 2 tokens holds both slots, the next item's
// products wait for them, and stores issued while the weight stream saturates the memory system
// would hold that release back.
template <int BN>
__device__ __forceinline__ void swiglu_to_regs(uint32_t t0, uint32_t t1, int sub, int n_valid,
                                               uint32_t (&hv)[(BN + 31) / 32][8]) {
#pragma unroll
    for (int i = 0; i < (BN + 31) / 32; ++i) {
        const int c = 16 * sub + 32 * i;
        if (c < n_valid) {  // warp-uniform
            uint32_t r0[16], r1[16];
            tmem_ld16(t0 + c, r0);
            tmem_ld16(t1 + c, r1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const __nv_bfloat162 v =
                    __floats2bfloat162_rn(silu_mul(__uint_as_float(r0[2 * j]), __uint_as_float(r1[2 * j])),
                                          silu_mul(__uint_as_float(r0[2 * j + 1]), __uint_as_float(r1[2 * j + 1])));
                hv[i][j] = *reinterpret_cast<const uint32_t *>(&v);
            }
        }
    }
}
__device__ __forceinline__ void st_b16_hint(uint16_t *addr, uint16_t v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.b16 [%0], %1, %2;" ::"l"(addr), "h"(v), "l"(policy) : "memory");
}
// The h values of swiglu_to_regs: weight row m (< M) of the item's tokens.  Stored L2-evict-last: the
// down projection reads h right after this launch, and lines that stay in L2 are neither re-read from
// DRAM there nor written back in the middle of this launch's weight stream (evict-first).
template <int BN>
__device__ __forceinline__ void store_h_regs(const GemmParams &p, const Item &it, int sub, int m,
                                             const uint32_t (&hv)[(BN + 31) / 32][8]) {
    const int64_t ld = p.M;
    uint16_t *h = reinterpret_cast<uint16_t *>(p.out) + (it.row0 + 16 * sub) * ld + m;
    const uint64_t pol = policy_evict_last();
#pragma unroll
    for (int i = 0; i < (BN + 31) / 32; ++i) {
        const int left = it.n_valid - (16 * sub + 32 * i);  // valid columns from this chunk on
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (j < left) st_b16_hint(h + (32 * i + j) * ld, static_cast<uint16_t>(hv[i][j >> 1] >> (16 * (j & 1))), pol);
    }
}

// Epilogue (q reads TMEM lanes 32q..32q+31; NSUB warps share a lane quadrant, warp sub taking the
// 16-column chunks sub, sub + NSUB, ...): per item, wait for its accumulator slot(s), then write G1:
// h = bf16(SiLU(gate) * up) (with NSUB = 2 through registers, stored after the release) or G2: o =
// the accumulators (both halves of the weight-row pair with PAIR), and release the slot(s) (acc_empty
// counts 4 * NSUB arrivals).
template <bool GATE_UP, int BN, int NSLOT, int SLOT_COLS, bool PAIR, int NSUB>
__device__ __forceinline__ void gemm_epilogue(int q, int sub, const int *tile_start, int total, const GemmParams &p,
                                              uint32_t tmem_base, uint64_t *acc_full, uint64_t *acc_empty) {
    constexpr int kRows = PAIR ? 2 * kBM : kBM;
    constexpr bool kDefer = GATE_UP && NSUB == 2;
    const int lane = threadIdx.x & 31;
    const int E = p.E;
    uint32_t uses = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
        const int u = slots_of<GATE_UP || PAIR, SLOT_COLS>(it.n_mma);
        bool ok = true;
        for (int i = 0; i < u && ok; ++i) {
            const uint32_t c = uses + i;
            ok = mbar_wait(&acc_full[c % NSLOT], (c / NSLOT) & 1u, p.timeout);
        }
        if (!ok) break;
        tc_fence_after();
        const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
        const int m = it.mt * kRows + q * 32 + lane;  // weight row of this thread (PAIR: and m + 128)
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(s0 * SLOT_COLS);
        const uint32_t t1 = tmem_base + lane_off +
                            static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
        uint32_t hv[kDefer ? (BN + 31) / 32 : 1][8];
        if constexpr (kDefer) swiglu_to_regs<BN>(t0, t1, sub, it.n_valid, hv);
        for (int c = 16 * sub; c < (kDefer ? 0 : it.n_valid); c += 16 * NSUB) {
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
                                __float2bfloat16_rn(silu_mul(__uint_as_float(r0[j]), __uint_as_float(r1[j])));
                }
            } else if (PAIR) {
                uint32_t r1[16];
                tmem_ld16(t1 + c, r1);
                tmem_ld_wait();
                store_down_row(p, it, c, m, r0);
                store_down_row(p, it, c, m + kBM, r1);
            } else {
                tmem_ld_wait();
                store_down_row(p, it, c, m, r0);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int i = 0; i < u; ++i) mbar_arrive(&acc_empty[(uses + i) % NSLOT]);
        uses += u;
        if constexpr (kDefer)
            if (m < p.M) store_h_regs<BN>(p, it, sub, m, hv);
    }
}

template <bool GATE_UP, int BN, int BOXN, int STAGES, int NSLOT, int SLOT_COLS, bool GATHER = false,
          bool PAIR = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a0,  // W_gate (G1) / W_down (G2): [E][M][K]
                        const __grid_constant__ CUtensorMap tm_a1,  // W_up (G1); unused for G2
                        const __grid_constant__ CUtensorMap tm_b,   // B rows [rows][K]: box BOXN rows, or
                                                                    // GATHER: x [T][K] with a one-row box
                        const GemmParams p) {
    using C = GemmCfg<GATE_UP, BN, BOXN, STAGES, NSLOT, SLOT_COLS, GATHER, PAIR>;
    extern __shared__ uint8_t gemm_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint64_t *acc_empty = acc_full + NSLOT;
    uint64_t *drain = acc_empty + NSLOT;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *tile_start = reinterpret_cast<int *>(smem + C::kBarOff + 256);
    int *tok = reinterpret_cast<int *>(smem + C::kTokOff);  // GATHER: token of each row of the item

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int n_mt = (p.M + C::kRows - 1) / C::kRows;
    const int n_kb = p.K / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < NSLOT; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], kGemmEpiWarps);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_a0);
        if (GATE_UP) prefetch_tensormap(&tm_a1);
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
        // ---------------- TMA producer (lane 0 issues; with GATHER the warp first loads the item's token ids)
        const uint64_t pol_w = p.weights_once ? policy_evict_first() : policy_evict_normal();
        const uint64_t pol_x = policy_evict_last();  // activations: re-read by the other weight-row tiles
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued = 0, issued_phase = 0;  // per stage: ever issued / phase of the last issue
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
                const uint32_t bytes = C::kNumA * C::kA + nbox * (GATHER ? 4 * kBK * 2 : C::kBox);
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * C::kStage;
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_3d(sa, &tm_a0, &full[stage], kb * kBK, it.mt * C::kRows, it.e, pol_w);
                    if (GATE_UP) tma_load_3d(sa + C::kA, &tm_a1, &full[stage], kb * kBK, it.mt * kBM, it.e, pol_w);
                    // PAIR: the second half may start past M (zero-filled by the TMA unit; never stored)
                    if (PAIR) tma_load_3d(sa + C::kA, &tm_a0, &full[stage], kb * kBK, it.mt * C::kRows + kBM, it.e, pol_w);
                    uint8_t *sb = sa + C::kNumA * C::kA;
                    if (GATHER) {
                        for (int g = 0; g < nbox; ++g)  // rows 4g..4g+3 land 128 B apart, as a tiled box would
                            tma_gather4(sb + g * 4 * kBK * 2, &tm_b, &full[stage], kb * kBK, tok[4 * g],
                                        tok[4 * g + 1], tok[4 * g + 2], tok[4 * g + 3], pol_x);
                    } else {
                        for (int b = 0; b < nbox; ++b)
                            tma_load_2d(sb + b * C::kBox, &tm_b, &full[stage], kb * kBK,
                                        static_cast<int>(it.row0) + b * BOXN, pol_x);
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
        // every load this thread issued has landed before the CTA may exit
        if (lane == 0)
            for (int s = 0; s < STAGES; ++s)
                if ((issued >> s) & 1u) mbar_wait(&full[s], (issued_phase >> s) & 1u, p.timeout);
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            int stage = 0;
            uint32_t phase = 0;
            uint32_t uses = 0;  // TMEM slot uses so far
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
                const uint32_t idesc = umma_idesc_bf16(kBM, it.n_mma);
                const int u = slots_of<GATE_UP || PAIR, SLOT_COLS>(it.n_mma);
                const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
                for (int i = 0; i < u && ok; ++i) {
                    const uint32_t c = uses + i;
                    ok = mbar_wait(&acc_empty[c % NSLOT], ((c / NSLOT) & 1u) ^ 1u, p.timeout);
                }
                if (!ok) break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + static_cast<uint32_t>(s0 * SLOT_COLS);
                const uint32_t d1 = tmem_base + static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, p.timeout)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * C::kStage);
                    const uint64_t da0 = umma_desc_sw128(sa);
                    const uint64_t da1 = umma_desc_sw128(sa + C::kA);
                    const uint64_t db = umma_desc_sw128(sa + C::kNumA * C::kA);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                        // +32 bytes along K inside the swizzle row = +2 in the 16-byte address field
                        umma_bf16(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
                        if (GATE_UP || PAIR) umma_bf16(d1, da1 + 2 * kk, db + 2 * kk, idesc, accum);
                    }
                    umma_commit(&empty[stage]);  // frees the smem stage once these MMAs completed
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                for (int i = 0; i < u; ++i) umma_commit(&acc_full[(uses + i) % NSLOT]);
                uses += u;
            }
            // all issued MMAs complete before TMEM is released
            umma_commit(drain);
            mbar_wait(drain, 0, p.timeout);
        }
    } else {
        // warps 2..9: two per TMEM lane quadrant (a warp reads the quadrant warp % 4)
        gemm_epilogue<GATE_UP, BN, NSLOT, SLOT_COLS, PAIR, 2>(warp & 3, (warp - 2) / 4, tile_start, total, p,
                                                              tmem_base, acc_full, acc_empty);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace beam
