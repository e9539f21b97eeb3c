// dg_pair_kernel.cuh -- the CTA-pair variant of the FP8 block-scaled GEMM kernel for sm_100a
// (dense and masked-grouped layouts).
//
// Same method as dg_kernel.cuh (DeepSeek開源第三彈 -- the DeepGEMM release write-up --
// "深入了解DeepGEMM": fine-grained scales, two-level accumulation), mapped onto a 2-CTA cluster:
//   - the pair owns a 256 x BN output tile; CTA r of the pair owns rows [128 r, 128 r + 128);
//   - each CTA loads ITS OWN 128 rows of A and ITS HALF (BN/2 rows) of B -- no multicast -- so a
//     CTA moves 128 x 128 + BN/2 x 128 bytes per K block instead of 128 x 128 + BN x 128;
//   - one TMA box spans kKbPerStage K blocks (fewer, larger copies: the TMA engine's per-copy
//     cost, not L2, bounds small boxes); the A scales of a stage arrive in one small box in a
//     ring of their own, so a stage is freed by the MMA alone;
//   - the even CTA issues tcgen05.mma.cta_group::2 (M = 256) per 32-wide K step; the partial of
//     each 128-wide K block lands in both CTAs' tensor memory, and commits are multicast to both
//     CTAs' barriers;
//   - each CTA's promotion warps scale and accumulate their own rows exactly as in the 1-CTA
//     kernel, release the TMEM buffer to the even CTA's MMA warp with a cluster arrive, and
//     write the tile through the same TMA-store epilogue.
// Barriers that collect work of both CTAs (stage full, TMEM buffer empty) live in the even CTA.
#pragma once

#include "dg_kernel.cuh"

namespace dg {

constexpr int kKbPerStage = 2;  // K blocks per TMA box / pipeline stage

template <int BN>
struct PairCfg {
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN must be a multiple of 32 in [64, 256]");
    static constexpr int kHalfN = BN / 2;                          // B rows per CTA
    static constexpr int kCols = BN / 2;                           // columns per promotion thread
    static constexpr int kPart1 = (kCols <= 96) ? kCols : ((kCols / 2 + 15) / 16 * 16);
    static constexpr int kTmemBufs = (kTmemCols / BN) >= 4 ? 4 : (kTmemCols / BN);
    static constexpr int kAKbBytes = kBlockM * kBlockK;            // A bytes per K block per CTA
    static constexpr int kBKbBytes = kHalfN * kBlockK;             // B bytes per K block per CTA
    static constexpr int kABytes = kKbPerStage * kAKbBytes;
    static constexpr int kBBytes = kKbPerStage * kBKbBytes;
    static constexpr int kStageBytes = kABytes + kBBytes;          // multiple of 1024
    static constexpr uint32_t kTxBytesPerCta = kABytes + kBBytes;
    static constexpr uint32_t kTxBytesPerCtaFp4B = kABytes + kBBytes / 2;  // packed E2M1 B
    static constexpr uint32_t kIdesc = ptx::idesc_e4m3_f32(2 * kBlockM, BN);
    static constexpr int kSfaSlotBytes = kKbPerStage * kBlockM * 4;  // A scales of one stage
};

// Waits in the pair kernel use the default (CTA-scope acquire) form, like the one-CTA kernel:
// the cross-CTA arrivals they observe hand over tensor memory or TMA bytes, ordered by the
// tcgen05 fences and transaction counts rather than by memory release/acquire.
__device__ __forceinline__ bool wait_one_c(uint32_t bar, uint32_t parity, const Params &p,
                                           volatile int *abort_flag)
{
    if (ptx::mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity))
            return true;
        if (*abort_flag)
            return false;
        if (ptx::global_timer_ns() - t0 > p.timeout_ns) {
            *abort_flag = 1;
            record_error(p.err, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_drain_c(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = ptx::global_timer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::global_timer_ns() - t0 > kDrainTimeoutNs)
            return false;
    }
    return true;
}

// Pair tile t -> coordinates.  m0 is the first row of the 256-row pair tile within its group.
template <int L>
__device__ __forceinline__ void resolve_pair_tile(const Params &p, const SmemCtl &ctl, int t, Tile &ti)
{
    if (L == kMasked) {
        int lo = 0, hi = p.G - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (ctl.tile_prefix[mid] <= t)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int g = lo;
        int mm = __ldg(p.masked_m + g);
        mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
        const int mt = (mm + 2 * kBlockM - 1) / (2 * kBlockM);
        const int local = t - ctl.tile_prefix[g];
        ti.g = g;
        ti.m0 = (local % mt) * 2 * kBlockM;
        ti.n0 = local / mt;
        ti.a_z = g;
    } else {
        const int band = p.raster_m * p.n_tiles;
        const int b = t / band;
        const int r = t - b * band;
        const int m_base = b * p.raster_m;
        int h = p.m_tiles - m_base;
        h = h < p.raster_m ? h : p.raster_m;
        ti.m0 = (m_base + r % h) * 2 * kBlockM;
        ti.n0 = r / h;
        ti.a_z = 0;
        ti.g = 0;
    }
}

// Params conventions for this kernel: p.m_tiles counts 256-row pair tiles; tiles are walked by
// clusters (cluster id, cluster count) instead of CTAs.
template <int L, int BN>
__global__ void __launch_bounds__(kNumThreads, 1)
    dg_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                        const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_sfa,
                        const __grid_constant__ CUtensorMap tmap_d, const Params p)
{
    using C = PairCfg<BN>;
    constexpr int KS = kKbPerStage;
    __shared__ SmemCtl ctl;
    extern __shared__ uint8_t smem_raw[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const uint32_t rank = ptx::cluster_ctarank();     // 0: even CTA (issues the MMAs), 1: odd
    const int pair = static_cast<int>(ptx::cluster_id_x());
    const int num_pairs = static_cast<int>(ptx::num_clusters_x());
    const uint32_t smem_base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t *smem_gen = smem_raw + (smem_base - ptx::smem_addr(smem_raw));

    auto stage_a = [&](int s) { return smem_base + s * C::kStageBytes; };
    auto stage_b = [&](int s) { return smem_base + s * C::kStageBytes + C::kABytes; };
    const int sfa_off = p.stages * C::kStageBytes;  // A-scale ring after the operand stages
    auto sfa_slot = [&](int j) { return smem_base + sfa_off + j * C::kSfaSlotBytes; };
    auto sfa_ptr = [&](int j) {
        return reinterpret_cast<const float *>(smem_gen + sfa_off + j * C::kSfaSlotBytes);
    };
    const uint32_t bar_full = ptx::smem_addr(&ctl.full[0]);
    const uint32_t bar_empty = ptx::smem_addr(&ctl.empty[0]);
    const uint32_t bar_tfull = ptx::smem_addr(&ctl.tmem_full[0]);
    const uint32_t bar_tempty = ptx::smem_addr(&ctl.tmem_empty[0]);
    const uint32_t bar_drain = ptx::smem_addr(&ctl.drain);
    const uint32_t bar_sfull = ptx::smem_addr(&ctl.sfa_full[0]);
    const uint32_t bar_sempty = ptx::smem_addr(&ctl.sfa_empty[0]);
    volatile int *abort_flag = &ctl.abort_flag;
    ptx::griddep_launch_dependents();  // the next grid may start its set-up as SMs free up

    // ---- set-up ------------------------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 2);   // one expect_tx arrival from each CTA (even CTA's copy)
            ptx::mbar_init(bar_empty + 8 * s, 1);  // the pair MMA commit (both CTAs' copies)
        }
        for (int j = 0; j < kSfaSlots; ++j) {
            ptx::mbar_init(bar_sfull + 8 * j, 1);              // this CTA's scale box
            ptx::mbar_init(bar_sempty + 8 * j, kNumMathWarps); // this CTA's promotion warps
        }
        for (int b = 0; b < C::kTmemBufs; ++b) {
            ptx::mbar_init(bar_tfull + 8 * b, 1);                  // pair MMA commit
            ptx::mbar_init(bar_tempty + 8 * b, 2 * kNumMathWarps); // both CTAs' promotion warps
        }
        ptx::mbar_init(bar_drain, 1);
        ptx::mbar_init(ptx::smem_addr(&ctl.stall), 1);
        ctl.abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
        ptx::prefetch_tmap(&tmap_sfa);
        ptx::prefetch_tmap(&tmap_d);
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_addr(&ctl.tmem_base), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    // no global memory is touched before the grids this one depends on are complete
    ptx::griddep_wait();
    if (L == kMasked) {
        if (warp == 2 && lane == 0) {
            int acc = 0;
            for (int g = 0; g < p.G; ++g) {
                ctl.tile_prefix[g] = acc;
                int mm = __ldg(p.masked_m + g);
                if (mm < 0 || mm > p.M) {
                    if (blockIdx.x == 0)
                        record_error(p.err, kErrLayout);
                    mm = mm < 0 ? 0 : p.M;
                }
                acc += (mm + 2 * kBlockM - 1) / (2 * kBlockM) * p.n_tiles;
            }
            ctl.tile_prefix[p.G] = acc;
            ctl.total_tiles = acc;
        }
    } else if (threadIdx.x == 0) {
        ctl.total_tiles = p.num_tiles;
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA traffic
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl.tmem_base;
    const int num_tiles = ctl.total_tiles;

    if (warp < kFirstMathWarp) {
        ptx::setmaxnreg_dec<40>();
        if (warp == 0) {
            // ---------------- TMA producer (each CTA loads its own A rows and B half) ----------
            const uint32_t full0 = ptx::map_to_rank(bar_full, 0);  // stage barriers of the even CTA
            uint32_t n_op = 0, n_sfa = 0;
            int s = 0, j = 0;
            uint32_t ph = 0, jph = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                Tile ti;
                resolve_pair_tile<L>(p, ctl, t, ti);
                const int a_row = ti.m0 + static_cast<int>(rank) * kBlockM;
                const int b_row = ti.n0 * BN + static_cast<int>(rank) * C::kHalfN;
                for (int kb0 = 0; kb0 < p.num_kb; kb0 += KS) {
                    // A scales of the stage's K blocks (one box: 128 rows x KS K blocks)
                    if (!__all_sync(0xffffffffu, wait_one_c(bar_sempty + 8 * j, jph ^ 1, p, abort_flag))) {
                        ok = false;
                        break;
                    }
                    if (ptx::elect_one()) {
                        ptx::mbar_arrive_expect_tx(bar_sfull + 8 * j, C::kSfaSlotBytes);
                        ptx::tma_load_3d(sfa_slot(j), &tmap_sfa, bar_sfull + 8 * j, a_row, kb0, ti.a_z);
                    }
                    __syncwarp();
                    ++n_sfa;
                    if (++j == kSfaSlots) {
                        j = 0;
                        jph ^= 1;
                    }
                    if (!__all_sync(0xffffffffu, wait_one_c(bar_empty + 8 * s, ph ^ 1, p, abort_flag))) {
                        ok = false;
                        break;
                    }
                    if (ptx::elect_one()) {
                        const uint32_t fb = full0 + 8 * s;
                        ptx::mbar_arrive_expect_tx_cluster(fb, p.idesc_b ? C::kTxBytesPerCtaFp4B : C::kTxBytesPerCta);
                        ptx::tma_load_4d_pair(stage_a(s), &tmap_a, fb, 0, a_row, kb0, ti.a_z);
                        ptx::tma_load_4d_pair(stage_b(s), &tmap_b, fb, 0, b_row, kb0, ti.g);
                    }
                    __syncwarp();
                    ++n_op;
                    if (++s == p.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // Wind down.  Operand loads signal the even CTA's stage barriers, so the even CTA
            // drains them for both CTAs (a final cluster barrier keeps the odd CTA alive until
            // then).
            {
                int pending = n_sfa < static_cast<uint32_t>(kSfaSlots) ? static_cast<int>(n_sfa) : kSfaSlots;
                int dj = j;
                uint32_t dph = jph;
                for (int i = 0; i < pending; ++i) {
                    if (--dj < 0) {
                        dj = kSfaSlots - 1;
                        dph ^= 1;
                    }
                    wait_drain_c(bar_sfull + 8 * dj, dph);
                }
            }
            if (rank == 0) {
                int pending = n_op < static_cast<uint32_t>(p.stages) ? static_cast<int>(n_op) : p.stages;
                int ds = s;
                uint32_t dph = ph;
                for (int i = 0; i < pending; ++i) {
                    if (--ds < 0) {
                        ds = p.stages - 1;
                        dph ^= 1;
                    }
                    wait_drain_c(bar_full + 8 * ds, dph);
                }
            }
            __syncwarp();
        } else if (warp == 1 && rank == 0) {
            // ---------------- pair MMA issuer (even CTA; whole warp, one lane issues) ----------
            int s = 0;
            uint32_t ph = 0;
            int buf = 0;
            uint32_t bph = 0;
            bool ok = !p.inject_stall ||
                      __all_sync(0xffffffffu, wait_one_c(ptx::smem_addr(&ctl.stall), 0, p, abort_flag));
            for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                for (int kb0 = 0; kb0 < p.num_kb && ok; kb0 += KS) {
                    if (!__all_sync(0xffffffffu, wait_one_c(bar_full + 8 * s, ph, p, abort_flag))) {
                        ok = false;
                        break;
                    }
                    const int nk = (p.num_kb - kb0) < KS ? (p.num_kb - kb0) : KS;
                    for (int kk = 0; kk < nk; ++kk) {
                        if (!__all_sync(0xffffffffu, wait_one_c(bar_tempty + 8 * buf, bph ^ 1, p, abort_flag))) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        if (ptx::elect_one()) {
                            const uint64_t adesc =
                                ptx::sdesc_kmajor_sw128(stage_a(s) + kk * C::kAKbBytes);
                            const uint64_t bdesc =
                                ptx::sdesc_kmajor_sw128(stage_b(s) + kk * C::kBKbBytes);
                            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
                            for (int k = 0; k < kBlockK / kUmmaK; ++k)
                                ptx::mma_f8f6f4_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::kIdesc | p.idesc_b,
                                                     k > 0 ? 1u : 0u);
                            ptx::mma_commit_pair_multicast(bar_tfull + 8 * buf, 0x3);
                        }
                        __syncwarp();
                        if (++buf == C::kTmemBufs) {
                            buf = 0;
                            bph ^= 1;
                        }
                    }
                    if (!ok)
                        break;
                    // the stage is free in both CTAs once these MMAs complete
                    if (ptx::elect_one())
                        ptx::mma_commit_pair_multicast(bar_empty + 8 * s, 0x3);
                    __syncwarp();
                    if (++s == p.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            if (ptx::elect_one())
                ptx::mma_commit_pair_local(bar_drain);
            __syncwarp();
            wait_drain_c(bar_drain, 0);
            __syncwarp();
        }
    } else {
        ptx::setmaxnreg_inc<232>();
        // ---------------- promotion + epilogue (each CTA, its own 128 rows) ----------------
        const int mw = warp - kFirstMathWarp;
        const int half = mw / 4;
        const int q = warp % 4;
        const int row = q * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(half * C::kCols);
        const uint32_t tempty0 = ptx::map_to_rank(bar_tempty, 0);  // even CTA's buffer barriers
        constexpr int P1 = C::kPart1;
        constexpr int P2 = C::kCols - P1;
        // this warp's ring of output staging boxes, after the operand stages and the A-scale ring
        const uint32_t epi_ring = smem_base + static_cast<uint32_t>(sfa_off + kSfaSlots * C::kSfaSlotBytes) +
                                  static_cast<uint32_t>(mw * kEpiWarpBytes);
        int ebuf = 0;
        int sj = 0;
        uint32_t sjph = 0;
        int buf = 0;
        uint32_t bph = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += num_pairs) {
            Tile ti;
            resolve_pair_tile<L>(p, ctl, t, ti);
            const int m0c = ti.m0 + static_cast<int>(rank) * kBlockM;  // this CTA's first row
            const int n0 = ti.n0 * BN;
            const int col0 = n0 + half * C::kCols;
            const int nb_lo = min(col0 / kBlockK, p.num_nb - 1);
            const int nb_hi = min((col0 + C::kCols - 1) / kBlockK, p.num_nb - 1);
            const int split = min(C::kCols, max(0, (nb_lo + 1) * kBlockK - col0));
            const float *sfb_lo = p.sfb + (static_cast<size_t>(ti.g) * p.num_nb + nb_lo) * p.num_kb;
            const float *sfb_hi = p.sfb + (static_cast<size_t>(ti.g) * p.num_nb + nb_hi) * p.num_kb;
            float acc[C::kCols];
#pragma unroll
            for (int c = 0; c < C::kCols; ++c)
                acc[c] = 0.0f;

            // B scales of the stage's two K blocks, loaded one stage ahead
            float lo0 = __ldg(sfb_lo), hi0 = __ldg(sfb_hi);
            const int k1 = p.num_kb > 1 ? 1 : 0;
            float lo1 = __ldg(sfb_lo + k1), hi1 = __ldg(sfb_hi + k1);
            auto release_of = [&](int b, uint32_t &rel, bool &remote) {
                // the even CTA's own promotion warps arrive locally, the odd CTA's remotely
                remote = rank != 0;
                rel = remote ? tempty0 + 8 * b : bar_tempty + 8 * b;
            };
            for (int kb0 = 0; kb0 < p.num_kb && ok; kb0 += KS) {
                if (!__all_sync(0xffffffffu, wait_one_c(bar_sfull + 8 * sj, sjph, p, abort_flag))) {
                    ok = false;
                    break;
                }
                const float *ring = sfa_ptr(sj);
                uint32_t rel;
                bool remote;
                // first K block of the stage
                release_of(buf, rel, remote);
                ok = promote_kb<P1, P2>(acc, ring[row], lo0, hi0, lane_base + static_cast<uint32_t>(buf * BN),
                                        bar_tfull + 8 * buf, bph, rel, remote, split, lane, p, abort_flag);
                if (++buf == C::kTmemBufs) {
                    buf = 0;
                    bph ^= 1;
                }
                {
                    const int kn = kb0 + 2 < p.num_kb ? kb0 + 2 : p.num_kb - 1;
                    lo0 = __ldg(sfb_lo + kn);
                    hi0 = __ldg(sfb_hi + kn);
                }
                // second K block of the stage (absent in a final odd stage)
                if (ok && kb0 + 1 < p.num_kb) {
                    release_of(buf, rel, remote);
                    ok = promote_kb<P1, P2>(acc, ring[kBlockM + row], lo1, hi1,
                                            lane_base + static_cast<uint32_t>(buf * BN), bar_tfull + 8 * buf,
                                            bph, rel, remote, split, lane, p, abort_flag);
                    if (++buf == C::kTmemBufs) {
                        buf = 0;
                        bph ^= 1;
                    }
                    const int kn = kb0 + 3 < p.num_kb ? kb0 + 3 : p.num_kb - 1;
                    lo1 = __ldg(sfb_lo + kn);
                    hi1 = __ldg(sfb_hi + kn);
                }
                // the stage's scales have been read: free the slot
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(bar_sempty + 8 * sj);
                if (++sj == kSfaSlots) {
                    sj = 0;
                    sjph ^= 1;
                }
            }
            if (!ok)
                break;

            // ---- epilogue ----
            const int grow = m0c + row;
            bool valid;
            size_t out_row;
            if (L == kMasked) {
                int mm = __ldg(p.masked_m + ti.g);
                mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
                valid = grow < mm;
                out_row = static_cast<size_t>(ti.g) * p.M + grow;
            } else {
                valid = grow < p.M;
                out_row = static_cast<size_t>(grow);
            }
            store_tile_rows<L, C::kCols>(acc, p, &tmap_d, epi_ring, ebuf, valid, out_row, col0, lane);
        }
        // every staged output box is written (and its shared memory read) before exit
        if (lane == 0)
            ptx::bulk_wait_group_all();
        __syncwarp();
    }

    // ---- tear-down: both CTAs past their last tcgen05 operation and cross-CTA arrival ----
    __syncwarp();
    ptx::tc_fence_before();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace dg
