// Grouped expert GEMMs on CTA pairs: tcgen05.mma.cta_group::2 (one M = 256 product spread over the
// two SMs of a cluster of 2).  Same work as gemm.cuh's wide kernels (G1: gate/up + SwiGLU, G2: down
// projection, swap-AB, persistent, expert-major items), for experts with tens to hundreds of tokens.
//
// Why pairs.  An item streams its weight tile once from HBM while its token tile is re-read from L2
// by every weight-row tile of the expert.  On one SM both share the shared-memory ring, and at ~130
// tokens per expert the token rows take 30-40% of each stage, which caps the weight bytes an SM keeps
// in flight (and so the HBM rate each SM sustains).  With cta_group::2 the pair computes a 256-row
// weight tile against the whole token tile while each CTA stages only HALF of the token rows: CTA r
// holds weight rows 128 r..128 r + 127 of the tile and token rows [r N/2, (r+1) N/2) of the MMA's N.
// The saved space becomes deeper weight rings (G1: 5 stages instead of 4, G2: 8 instead of 5), and a
// down-projection item keeps one accumulator per CTA, so its epilogue always overlaps the next item.
//
// Roles per CTA (320 threads, as gemm.cuh): warp 0 lane 0 = TMA producer for this CTA's halves; warp 1
// = TMEM (allocated for the pair with cta_group::2), and in the leader CTA (cluster rank 0) lane 0
// issues every MMA of the pair; warps 2..9 = epilogue on this CTA's 128 accumulator lanes.
// Synchronisation:
//   full[s]      leader only: the leader's producer arms it with both CTAs' bytes; both producers'
//                TMA loads (cta_group::2 form) complete their bytes on it;
//   empty[s]     each CTA: the leader's commit of stage s arrives on both (multicast to ranks 0, 1);
//   acc_full[a]  each CTA: the leader's commit of an item's last MMA arrives on both;
//   acc_empty[a] leader only: all 16 epilogue warps of the pair arrive (the peer's remotely).
// Before the pair's TMEM is released, a cluster barrier follows (a) the leader's wait for its last
// MMA, (b) both epilogues and (c) each producer's wait for the consumption of every stage it loaded,
// so no MMA, TMEM read or TMA write of either CTA is still in flight.  Every mbarrier wait is bounded
// (status word BEAM_MOE_ERR_DEVICE_TIMEOUT on expiry); no load uses multicast.
#pragma once

#include "gemm.cuh"

namespace beam {

// ---- cluster and cta_group::2 primitives ---------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address in CTA `rank`'s shared memory of the variable at this CTA's shared address `addr`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
    return d;
}
// Every thread of both CTAs: release this CTA's prior writes to the pair, wait for the peer's.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier given by its cluster address (this CTA's or the peer's).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// TMA tile load into this CTA's shared memory whose bytes complete on an mbarrier of either CTA of the
// pair (cta_group::2 form; no multicast).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int c0,
                                                 int c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(bar_cluster), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar_cluster), "l"(policy)
        : "memory");
}
// Leader CTA only: D[256 x N] (+)= A . B^T over both CTAs' tiles at the same shared offsets.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives once on the mbarrier at this shared offset in both CTAs of the pair when the pair's MMAs
// issued so far have completed (tcgen05.commit with a CTA mask; this is not a TMA load).
__device__ __forceinline__ void umma_commit_pair_both(uint64_t *bar) {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(mask)
        : "memory");
}
__device__ __forceinline__ void umma_commit_pair_self(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- configuration -------------------------------------------------------------------------------
constexpr int kPairRows = 2 * kBM;  // weight rows per pair item

template <bool GATE_UP, int BN, int BOXN, int STAGES, int NSLOT, int SLOT_COLS>
struct Gemm2Cfg {
    static constexpr int kA = kBM * kBK * 2;                     // this CTA's A tile (128 rows), bytes
    static constexpr int kNumA = GATE_UP ? 2 : 1;
    static constexpr int kHalfRows = ((BN / 2 + BOXN - 1) / BOXN) * BOXN;  // token rows staged per CTA
    static constexpr int kB = kHalfRows * kBK * 2;
    static constexpr int kBox = BOXN * kBK * 2;
    static constexpr int kStage = kNumA * kA + kB;
    static constexpr int kTmemCols = pow2_cols(NSLOT * SLOT_COLS);
    static constexpr int kBarOff = STAGES * kStage;
    static constexpr int kTileOff = kBarOff + 256;
    static constexpr int kSmem = 1024 + kTileOff + 4 * (kPmMaxE + 1) + 64;
    static_assert(kStage % 1024 == 0 && kBox % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(BN % 16 == 0 && BN <= 256, "token tile: the pair's MMA takes N = 16..256 in steps of 16");
    static_assert(8 * (2 * STAGES + 2 * NSLOT + 1) + 4 <= 256, "barrier area");
    static_assert(NSLOT * SLOT_COLS <= 512, "TMEM has 512 columns");
    static_assert(GATE_UP ? (BN <= SLOT_COLS && (NSLOT >= 2 || BN <= SLOT_COLS / 2)) : BN <= SLOT_COLS,
                  "an item must fit in its TMEM slots");
    static_assert(kSmem + 128 <= 232448, "shared memory per CTA (dynamic + the 128 static bytes)");
};

// Epilogue of one CTA of the pair: its 128 accumulator lanes are weight rows 128 rank + lane of the
// item's 256-row tile; the slots are released on the leader's acc_empty.  Two warps share each lane
// quadrant (warp `sub` takes the 16-column chunks 16 sub + 32 i).
//   G1: h goes through registers and is stored after the slots are released (swiglu_to_regs);
//   G2: all of the thread's fp32 chunks are loaded from TMEM with one wait (up to 96 registers), the
//       slot is released, and then the o rows are stored (measured: 3-4% off the down projection at
//       prefill, skew and long against storing chunk by chunk from TMEM).
template <bool GATE_UP, int BN, int NSLOT, int SLOT_COLS>
__device__ __forceinline__ void gemm2_epilogue(int q, int sub, uint32_t rank, int pair, int n_pairs,
                                               const int *tile_start, int total, const GemmParams &p,
                                               uint32_t tmem_base, uint64_t *acc_full, uint64_t *acc_empty) {
    constexpr int kChunks = (BN + 31) / 32;  // chunks per thread
    const int lane = threadIdx.x & 31;
    const uint32_t acc_empty_lead = mapa_shared(smem_u32(acc_empty), 0);
    uint32_t uses = 0;
    for (int item = pair; item < total; item += n_pairs) {
        const Item it = decode_item(item, tile_start, p.E, BN, p.counts, p.offsets);
        const int u = slots_of<GATE_UP, SLOT_COLS>(it.n_mma);
        bool ok = true;
        for (int i = 0; i < u && ok; ++i) {
            const uint32_t c = uses + i;
            ok = mbar_wait(&acc_full[c % NSLOT], (c / NSLOT) & 1u, p.timeout);
        }
        if (!ok) break;
        tc_fence_after();
        const int s0 = uses % NSLOT, s1 = (uses + 1) % NSLOT;
        const int m = it.mt * kPairRows + static_cast<int>(rank) * kBM + q * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
        const uint32_t t0 = tmem_base + lane_off + static_cast<uint32_t>(s0 * SLOT_COLS);
        const uint32_t t1 = tmem_base + lane_off +
                            static_cast<uint32_t>(u == 2 ? s1 * SLOT_COLS : s0 * SLOT_COLS + SLOT_COLS / 2);
        uint32_t hv[GATE_UP ? kChunks : 1][8];   // G1: bf16 pairs of h (swiglu_to_regs)
        uint32_t ov[GATE_UP ? 1 : kChunks][16];  // G2: fp32 accumulators, chunk i = columns 16 sub + 32 i
        if constexpr (GATE_UP) {
            swiglu_to_regs<BN>(t0, t1, sub, it.n_valid, hv);
        } else {
#pragma unroll
            for (int i = 0; i < kChunks; ++i)
                if (16 * sub + 32 * i < it.n_valid) tmem_ld16(t0 + 16 * sub + 32 * i, ov[i]);  // warp-uniform
            tmem_ld_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int i = 0; i < u; ++i)
                mbar_arrive_cluster(acc_empty_lead + 8u * static_cast<uint32_t>((uses + i) % NSLOT));
        uses += u;
        if constexpr (GATE_UP) {
            if (m < p.M) store_h_regs<BN>(p, it, sub, m, hv);
        } else {
#pragma unroll
            for (int i = 0; i < kChunks; ++i)
                if (16 * sub + 32 * i < it.n_valid) store_down_row(p, it, 16 * sub + 32 * i, m, ov[i]);
        }
    }
}

template <bool GATE_UP, int BN, int BOXN, int STAGES, int NSLOT, int SLOT_COLS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tm_a0,  // W_gate (G1) / W_down (G2): [E][M][K]
                            const __grid_constant__ CUtensorMap tm_a1,  // W_up (G1); unused for G2
                            const __grid_constant__ CUtensorMap tm_b,   // dispatch-ordered rows [R][K], BOXN-row box
                            const GemmParams p) {
    using C = Gemm2Cfg<GATE_UP, BN, BOXN, STAGES, NSLOT, SLOT_COLS>;
    extern __shared__ uint8_t gemm_smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;
    uint64_t *acc_empty = acc_full + NSLOT;
    uint64_t *drain = acc_empty + NSLOT;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *tile_start = reinterpret_cast<int *>(smem + C::kTileOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader (issues the pair's MMAs), 1: peer
    const int pair = static_cast<int>(cluster_id_x()), n_pairs = static_cast<int>(cluster_count_x());
    const int E = p.E;
    const int n_mt = (p.M + kPairRows - 1) / kPairRows;
    const int n_kb = p.K / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < NSLOT; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 2 * kGemmEpiWarps);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
        prefetch_tensormap(&tm_a0);
        if (GATE_UP) prefetch_tensormap(&tm_a1);
        prefetch_tensormap(&tm_b);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    item_prefix(p.counts, E, n_mt, BN, tile_start);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers are initialised before either signals the other's
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tile_start[E];

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer: this CTA's weight rows and half of the token rows
            const uint64_t pol_w = p.weights_once ? policy_evict_first() : policy_evict_normal();
            const uint64_t pol_x = policy_evict_last();  // activations: re-read by the other weight-row tiles
            const uint32_t full_lead = mapa_shared(smem_u32(full), 0);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_phase = 0;  // per stage: ever issued / ring phase of the last issue
            bool ok = true;
            for (int item = pair; item < total && ok; item += n_pairs) {
                const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
                const int half = it.n_mma / 2;  // token rows per CTA (n_mma is a multiple of 16)
                const int nbox = (half + BOXN - 1) / BOXN;
                const int b_row = static_cast<int>(it.row0) + static_cast<int>(rank) * half;
                const int a_row = it.mt * kPairRows + static_cast<int>(rank) * kBM;
                const uint32_t pair_bytes = 2u * static_cast<uint32_t>(C::kNumA * C::kA + nbox * C::kBox);
                for (int kb = 0; kb < n_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.timeout)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + stage * C::kStage;
                    const uint32_t bar = full_lead + 8u * static_cast<uint32_t>(stage);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], pair_bytes);
                    tma_load_3d_pair(sa, &tm_a0, bar, kb * kBK, a_row, it.e, pol_w);
                    if (GATE_UP) tma_load_3d_pair(sa + C::kA, &tm_a1, bar, kb * kBK, a_row, it.e, pol_w);
                    uint8_t *sb = sa + C::kNumA * C::kA;
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d_pair(sb + b * C::kBox, &tm_b, bar, kb * kBK, b_row + b * BOXN, pol_x);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every stage this CTA loaded has been consumed by the pair's MMAs (so its bytes landed)
            for (int s = 0; s < STAGES; ++s)
                if ((issued >> s) & 1u) mbar_wait(&empty[s], (issued_phase >> s) & 1u, p.timeout);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer for the pair (leader CTA) ----------------
            int stage = 0;
            uint32_t phase = 0;
            uint32_t uses = 0;
            bool ok = true;
            for (int item = pair; item < total && ok; item += n_pairs) {
                const Item it = decode_item(item, tile_start, E, BN, p.counts, p.offsets);
                const uint32_t idesc = umma_idesc_bf16(kPairRows, it.n_mma);
                const int u = slots_of<GATE_UP, SLOT_COLS>(it.n_mma);
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
                        umma_bf16_pair(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
                        if (GATE_UP) umma_bf16_pair(d1, da1 + 2 * kk, db + 2 * kk, idesc, accum);
                    }
                    umma_commit_pair_both(&empty[stage]);  // frees stage `stage` in both CTAs
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                for (int i = 0; i < u; ++i) umma_commit_pair_both(&acc_full[(uses + i) % NSLOT]);
                uses += u;
            }
            // every MMA of the pair has completed before either CTA releases its TMEM
            umma_commit_pair_self(drain);
            mbar_wait(drain, 0, p.timeout);
        }
    } else {
        gemm2_epilogue<GATE_UP, BN, NSLOT, SLOT_COLS>(warp & 3, (warp - 2) / 4, rank, pair, n_pairs, tile_start,
                                                      total, p, tmem_base, acc_full, acc_empty);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, C::kTmemCols);
}

}  // namespace beam
