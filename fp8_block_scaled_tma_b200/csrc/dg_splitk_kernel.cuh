// dg_splitk_kernel.cuh -- split-K variant of the FP8 block-scaled GEMM kernel for sm_100a, for
// dense problems with too few output tiles to fill the GPU (small M, the memory-bound regime).
//
// Same method as dg_kernel.cuh (DeepSeek開源第三彈 -- the DeepGEMM release write-up --
// "深入了解DeepGEMM": fine-grained scales, two-level accumulation).  The K blocks of one
// 128 x BN output tile are split over the S CTAs of a thread-block cluster (S <= 8):
//   - CTA r of the cluster runs the usual TMA -> tcgen05.mma -> TMEM -> promotion pipeline over
//     its K blocks [r * Kb / S, (r + 1) * Kb / S), with TMA boxes spanning two K blocks;
//   - each CTA then writes its fp32 partial tile into its own shared memory (the drained
//     pipeline buffers), the cluster synchronises, and CTA r sums the rows of slice r over all
//     S partials through distributed shared memory in the fixed order s = 0 .. S-1 (the result
//     does not depend on timing) and stores them as bf16;
//   - no global workspace and no atomics; a second cluster barrier keeps every CTA's shared
//     memory alive until its peers have read it.
#pragma once

#include "dg_kernel.cuh"

namespace dg {

constexpr int kSplitKbPerStage = 2;
constexpr int kMaxSplits = 8;

template <int BN>
struct SplitCfg {
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN must be a multiple of 32 in [64, 256]");
    static constexpr int kCols = BN / 2;
    static constexpr int kPart1 = (kCols <= 96) ? kCols : ((kCols / 2 + 15) / 16 * 16);
    static constexpr int kTmemBufs = (kTmemCols / BN) >= 4 ? 4 : (kTmemCols / BN);
    static constexpr int kAKbBytes = kBlockM * kBlockK;
    static constexpr int kBKbBytes = BN * kBlockK;
    static constexpr int kABytes = kSplitKbPerStage * kAKbBytes;
    static constexpr int kStageBytes = kSplitKbPerStage * (kAKbBytes + kBKbBytes);
    static constexpr uint32_t kTxBytes = kStageBytes;
    static constexpr uint32_t kTxBytesFp4B = kSplitKbPerStage * (kAKbBytes + kBKbBytes / 2);  // packed E2M1 B
    static constexpr uint32_t kIdesc = ptx::idesc_e4m3_f32(kBlockM, BN);
    static constexpr int kPartLd = BN + 4;  // fp32 row stride of the partial tile (bank spread)
    static constexpr int kPartBytes = kBlockM * kPartLd * 4;
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d)
{
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// Load from a peer's shared memory.  No "memory" clobber, so that a thread can keep many of
// these in flight and sum later; volatile keeps them after the cluster barrier (also volatile)
// that publishes the peers' partials.
__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t cluster_addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(cluster_addr));
    return v;
}

__device__ __forceinline__ void st_global_v2(void *p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// Params conventions: p.m_tiles / p.n_tiles count 128 x BN tiles; p.raster_m holds S (the
// splits per tile = the cluster size); the grid is tiles * S CTAs.
template <int BN>
__global__ void __launch_bounds__(kNumThreads, 1)
    dg_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_b, const Params p)
{
    using C = SplitCfg<BN>;
    constexpr int KS = kSplitKbPerStage;
    __shared__ SmemCtl ctl;
    extern __shared__ uint8_t smem_raw[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int S = p.raster_m;
    const int r = static_cast<int>(ptx::cluster_ctarank());
    const int tile = static_cast<int>(ptx::cluster_id_x());
    const int m0 = (tile % p.m_tiles) * kBlockM;
    const int n0 = (tile / p.m_tiles) * BN;
    const int kb_begin = static_cast<int>(static_cast<long long>(r) * p.num_kb / S);
    const int kb_end = static_cast<int>(static_cast<long long>(r + 1) * p.num_kb / S);
    const int nkb = kb_end - kb_begin;

    const uint32_t smem_base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    auto stage_a = [&](int s) { return smem_base + s * C::kStageBytes; };
    auto stage_b = [&](int s) { return smem_base + s * C::kStageBytes + C::kABytes; };
    const uint32_t bar_full = ptx::smem_addr(&ctl.full[0]);
    const uint32_t bar_empty = ptx::smem_addr(&ctl.empty[0]);
    const uint32_t bar_tfull = ptx::smem_addr(&ctl.tmem_full[0]);
    const uint32_t bar_tempty = ptx::smem_addr(&ctl.tmem_empty[0]);
    const uint32_t bar_drain = ptx::smem_addr(&ctl.drain);
    volatile int *abort_flag = &ctl.abort_flag;
    ptx::griddep_launch_dependents();  // the next grid may start its set-up as SMs free up

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1);
            ptx::mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < C::kTmemBufs; ++b) {
            ptx::mbar_init(bar_tfull + 8 * b, 1);
            ptx::mbar_init(bar_tempty + 8 * b, kNumMathWarps);
        }
        ptx::mbar_init(bar_drain, 1);
        ptx::mbar_init(ptx::smem_addr(&ctl.stall), 1);
        ctl.abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(&ctl.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    // no global memory is touched before the grids this one depends on are complete
    ptx::griddep_wait();
    // The producer issues its first stages at once: they need only this CTA's barriers, which
    // its own lane 0 has just initialised, so the DRAM latency of the first loads overlaps the
    // TMEM allocation and the block barrier.  The stage ring then continues from there.
    uint32_t n_op = 0;  // producer: operand loads issued
    int ps = 0;         // producer: next stage
    uint32_t pph = 0;   // producer: its phase
    if (warp == 0) {
        __syncwarp();
        const int pre = min(p.stages, (nkb + KS - 1) / KS);
        if (ptx::elect_one()) {
            for (int i = 0; i < pre; ++i) {
                const uint32_t fb = bar_full + 8 * i;
                ptx::mbar_arrive_expect_tx(fb, p.idesc_b ? C::kTxBytesFp4B : C::kTxBytes);
                ptx::tma_load_4d(stage_a(i), &tmap_a, fb, 0, m0, kb_begin + i * KS, 0);
                ptx::tma_load_4d(stage_b(i), &tmap_b, fb, 0, n0, kb_begin + i * KS, 0);
            }
        }
        __syncwarp();
        n_op = static_cast<uint32_t>(pre);
        ps = pre == p.stages ? 0 : pre;
        pph = pre == p.stages ? 1u : 0u;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl.tmem_base;

    // rows [m0, m0 + rows_valid) of this tile are real
    const int rows_valid = min(kBlockM, p.M - m0);

    if (warp < kFirstMathWarp) {
        ptx::setmaxnreg_dec<40>();
        if (warp == 0) {
            // ---------------- TMA producer (after the stages issued during set-up) ----------------
            int s = ps;
            uint32_t ph = pph;
            for (int kb0 = kb_begin + static_cast<int>(n_op) * KS; kb0 < kb_end; kb0 += KS) {
                if (!__all_sync(0xffffffffu, wait_one(bar_empty + 8 * s, ph ^ 1, p, abort_flag)))
                    break;
                if (ptx::elect_one()) {
                    const uint32_t fb = bar_full + 8 * s;
                    ptx::mbar_arrive_expect_tx(fb, p.idesc_b ? C::kTxBytesFp4B : C::kTxBytes);
                    ptx::tma_load_4d(stage_a(s), &tmap_a, fb, 0, m0, kb0, 0);
                    ptx::tma_load_4d(stage_b(s), &tmap_b, fb, 0, n0, kb0, 0);
                }
                __syncwarp();
                ++n_op;
                if (++s == p.stages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            int pending = n_op < static_cast<uint32_t>(p.stages) ? static_cast<int>(n_op) : p.stages;
            int ds = s;
            uint32_t dph = ph;
            for (int i = 0; i < pending; ++i) {
                if (--ds < 0) {
                    ds = p.stages - 1;
                    dph ^= 1;
                }
                wait_drain(bar_full + 8 * ds, dph);
            }
            __syncwarp();
        } else if (warp == 1) {
            // ---------------- MMA issuer ----------------
            int s = 0;
            uint32_t ph = 0;
            int buf = 0;
            uint32_t bph = 0;
            bool ok = !p.inject_stall ||
                      __all_sync(0xffffffffu, wait_one(ptx::smem_addr(&ctl.stall), 0, p, abort_flag));
            for (int kb0 = kb_begin; kb0 < kb_end && ok; kb0 += KS) {
                if (!__all_sync(0xffffffffu, wait_one(bar_full + 8 * s, ph, p, abort_flag)))
                    break;
                const int nk = (kb_end - kb0) < KS ? (kb_end - kb0) : KS;
                for (int kk = 0; kk < nk; ++kk) {
                    if (!__all_sync(0xffffffffu, wait_one(bar_tempty + 8 * buf, bph ^ 1, p, abort_flag))) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    if (ptx::elect_one()) {
                        const uint64_t adesc = ptx::sdesc_kmajor_sw128(stage_a(s) + kk * C::kAKbBytes);
                        const uint64_t bdesc = ptx::sdesc_kmajor_sw128(stage_b(s) + kk * C::kBKbBytes);
                        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
                        for (int k = 0; k < kBlockK / kUmmaK; ++k)
                            ptx::mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::kIdesc | p.idesc_b,
                                            k > 0 ? 1u : 0u);
                        ptx::mma_commit(bar_tfull + 8 * buf);
                    }
                    __syncwarp();
                    if (++buf == C::kTmemBufs) {
                        buf = 0;
                        bph ^= 1;
                    }
                }
                if (!ok)
                    break;
                if (ptx::elect_one())
                    ptx::mma_commit(bar_empty + 8 * s);
                __syncwarp();
                if (++s == p.stages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (ptx::elect_one())
                ptx::mma_commit(bar_drain);
            __syncwarp();
            wait_drain(bar_drain, 0);
            __syncwarp();
        }
        // producer and MMA warpgroup: wait for the partials, then help nothing (the promotion
        // warps do the reduction); they only take part in the cluster barriers below
        ptx::tc_fence_before();
        ptx::cluster_sync();
        ptx::cluster_sync();
    } else {
        ptx::setmaxnreg_inc<232>();
        // ---------------- promotion over this CTA's K blocks ----------------
        const int mw = warp - kFirstMathWarp;
        const int half = mw / 4;
        const int q = warp % 4;
        const int row = q * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(half * C::kCols);
        constexpr int P1 = C::kPart1;
        constexpr int P2 = C::kCols - P1;
        const int col0 = n0 + half * C::kCols;
        const int nb_lo = min(col0 / kBlockK, p.num_nb - 1);
        const int nb_hi = min((col0 + C::kCols - 1) / kBlockK, p.num_nb - 1);
        const int split = min(C::kCols, max(0, (nb_lo + 1) * kBlockK - col0));
        // this CTA's K range, viewed as a K loop of nkb blocks starting at kb_begin
        const float *sfb_lo = p.sfb + static_cast<size_t>(nb_lo) * p.num_kb + kb_begin;
        const float *sfb_hi = p.sfb + static_cast<size_t>(nb_hi) * p.num_kb + kb_begin;
        const float *sa_ptr = p.sfa + static_cast<size_t>(kb_begin) * p.sfa_ld +
                              min(m0 + row, p.sfa_ld - 1);
        float acc[C::kCols];
#pragma unroll
        for (int c = 0; c < C::kCols; ++c)
            acc[c] = 0.0f;
        int buf = 0;
        uint32_t bph = 0;
        Params pk = p;
        pk.num_kb = nkb;  // the promotion loop walks this CTA's K blocks only
        KbScales s0, s1;
        load_kb_scales(s0, sa_ptr, sfb_lo, sfb_hi, p.sfa_ld, 0, nkb);
        load_kb_scales(s1, sa_ptr, sfb_lo, sfb_hi, p.sfa_ld, 1, nkb);
        promote_tile<BN, P1, P2, C::kCols, C::kTmemBufs>(
            acc, s0, s1, sa_ptr, sfb_lo, sfb_hi, lane_base, bar_tfull, buf, bph,
            [&](int b, uint32_t &rel, bool &remote) {
                rel = bar_tempty + 8 * b;
                remote = false;
            },
            split, lane, pk, abort_flag);

        // ---- the partial tile into this CTA's shared memory (pipeline buffers are drained:
        // every MMA of this CTA completed before its last partial was read) ----
        if (row < rows_valid) {
            const uint32_t dst = smem_base + static_cast<uint32_t>((row * C::kPartLd + half * C::kCols) * 4);
#pragma unroll
            for (int c = 0; c < C::kCols; c += 4)
                st_shared_v4(dst + c * 4, acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
        }
        ptx::tc_fence_before();
        ptx::cluster_sync();  // every CTA's partial is in place

        // ---- reduction of row slice r over the S partials, fixed order ----
        // Each thread loads the S partials of kBatch 4-column chunks before summing any, so
        // that up to kBatch * S remote loads are in flight (one at a time is latency-bound).
        const int rows_per = (rows_valid + S - 1) / S;
        const int r_begin = r * rows_per;
        const int r_end = min(rows_valid, r_begin + rows_per);
        constexpr int kChunksPerRow = BN / 4;
        constexpr int kThreads = kNumMathWarps * 32;
        constexpr int kBatch = 4;
        const int n_chunks = (r_end > r_begin ? r_end - r_begin : 0) * kChunksPerRow;
        const int t = threadIdx.x - kFirstMathWarp * 32;  // 0 .. 255
        for (int c0 = t; c0 < n_chunks; c0 += kBatch * kThreads) {
            float4 v[kBatch][kMaxSplits];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int ci = c0 + j * kThreads;
                if (ci < n_chunks) {
                    const int rr = r_begin + ci / kChunksPerRow;
                    const int cc = (ci % kChunksPerRow) * 4;
                    const uint32_t local = smem_base + static_cast<uint32_t>((rr * C::kPartLd + cc) * 4);
#pragma unroll
                    for (int s2 = 0; s2 < kMaxSplits; ++s2)
                        if (s2 < S)
                            v[j][s2] = ld_shared_cluster_v4(ptx::map_to_rank(local, static_cast<uint32_t>(s2)));
                }
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int ci = c0 + j * kThreads;
                if (ci < n_chunks) {
                    const int rr = r_begin + ci / kChunksPerRow;
                    const int col = n0 + (ci % kChunksPerRow) * 4;
                    float4 sum = v[j][0];
#pragma unroll
                    for (int s2 = 1; s2 < kMaxSplits; ++s2) {
                        if (s2 < S) {
                            sum.x += v[j][s2].x;
                            sum.y += v[j][s2].y;
                            sum.z += v[j][s2].z;
                            sum.w += v[j][s2].w;
                        }
                    }
                    if (col < p.N) {
                        __nv_bfloat16 *dst = p.d + static_cast<size_t>(m0 + rr) * p.N + col;
                        st_global_v2(dst, ptx::pack_bf16x2(sum.x, sum.y), ptx::pack_bf16x2(sum.z, sum.w));
                    }
                }
            }
        }
        ptx::cluster_sync();  // peers are done reading this CTA's partial
    }

    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace dg
