// dg_swap_kernel.cuh -- small-M variant of the FP8 block-scaled NT GEMM for sm_100a, with the
// operand roles of the tensor-core instruction swapped.
//
// Same method as dg_kernel.cuh (DeepSeek開源第三彈 -- the DeepGEMM release write-up --
// "深入了解DeepGEMM": fine-grained scales, two-level accumulation), for dense problems with at
// most 128 rows of A (decode-sized token counts, the memory-bound regime).  The MMA computes the
// transposed tile D^T = B . A^T:
//   - its M side (128 TMEM lanes) holds 128 rows of B, one 128 x 128 scale block of B per K
//     block, so the B scale is one number per tile and K block;
//   - its N side holds the TN <= 128 token rows of A (TN = 32, 64 or 128), so a TMEM buffer is
//     only R * TN columns wide and 4 to 8 buffers fit in tensor memory.  With that many
//     partials in flight, the round trip that recycles a buffer (MMA commit -> promotion ->
//     release) overlaps itself and no longer sets the pace; the kernel streams B.
//   - a tile covers R = 1 or 2 blocks of 128 B rows (two MMAs per K step into adjacent column
//     ranges) so that very wide N still fits in one wave.
// Promotion: each thread owns one B row (its TMEM lane) and R * TN / 2 columns (tokens); per K
// block it adds partial * (sa[token] * sb[block]) into fp32 registers.  The products
// sa * sb of the CTA's whole K range are formed once in shared memory (A's scales arrive by one
// TMA box), so the K loop costs one FFMA and a quarter broadcast load per element.
// K is split over the S CTAs of a cluster exactly as in dg_splitk_kernel.cuh: each CTA writes
// its fp32 partial (token-major) into its own shared memory, and CTA r sums its slice of the
// tile over all S partials in the fixed order s = 0 .. S-1 through distributed shared memory
// and stores bf16 rows of D.  No global workspace, no atomics; the output does not depend on
// timing.
#pragma once

#include "dg_splitk_kernel.cuh"

namespace dg {

constexpr int kSwapKbPerStage = 2;
constexpr int kSwapMaxBufs = 8;
constexpr int kSwapMaxScaleBytes = 48 * 1024;

struct SwapCtl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tmem_full[kSwapMaxBufs];
    uint64_t tmem_empty[kSwapMaxBufs];
    uint64_t scales;
    uint64_t drain;
    uint64_t stall;  // never signalled: the target of the fault-injection test hook
    uint32_t tmem_base;
    int abort_flag;
};

template <int TN, int R>
struct SwapCfg {
    static_assert(TN == 32 || TN == 64 || TN == 128, "token tile of 32, 64 or 128 rows");
    static_assert(R == 1 || R == 2, "one or two 128-row blocks of B per tile");
    static constexpr int kRows = kBlockM * R;             // B rows per tile
    static constexpr int kBufCols = R * TN;               // TMEM columns per buffer
    static constexpr int kBufs = (kTmemCols / kBufCols) < kSwapMaxBufs ? (kTmemCols / kBufCols)
                                                                      : kSwapMaxBufs;
    static constexpr int kCols = kBufCols / 2;            // columns per promotion thread
    static constexpr int kPart1 = kCols <= 64 ? kCols : 64;
    static constexpr int kPart2 = kCols - kPart1;
    static constexpr int kBKbBytes = kRows * kBlockK;     // B per K block in shared memory
    static constexpr int kAKbBytes = TN * kBlockK;        // A per K block
    static constexpr int kBBytes = kSwapKbPerStage * kBKbBytes;
    static constexpr int kStageBytes = kSwapKbPerStage * (kBKbBytes + kAKbBytes);  // multiple of 1024
    static constexpr uint32_t kTxBytes = kStageBytes;
    // TMA counts a packed E2M1 B at 4 bits per element (it lands at 8 bits per element)
    static constexpr uint32_t kTxBytesFp4B = kSwapKbPerStage * (kBKbBytes / 2 + kAKbBytes);
    static constexpr uint32_t kIdesc = ptx::idesc_e4m3_f32(kBlockM, TN);
    static constexpr int kPartBytes = TN * kRows * 4;     // fp32 partial, [token][B row]
};

__device__ __forceinline__ float ld_shared_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 ld_shared_v4f(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v)
{
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Barrier of the eight promotion warps only (named barrier 1).
__device__ __forceinline__ void promotion_bar_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kNumMathWarps * 32) : "memory");
}

// Params conventions: p.n_tiles counts tiles of R * 128 B rows; p.raster_m holds S (the K
// splits per tile = the cluster size); p.m_tiles holds the height of A's scale box, the K blocks
// of the longest split; the grid is n_tiles * S CTAs.  B-format bits in p.idesc_b (E2M1) are
// moved to the A-format field: B is the instruction's A operand here.
template <int TN, int R>
__global__ void __launch_bounds__(kNumThreads, 1)
    dg_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmap_a,
                        const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_sa, const Params p)
{
    using C = SwapCfg<TN, R>;
    constexpr int KS = kSwapKbPerStage;
    __shared__ SwapCtl ctl;
    extern __shared__ uint8_t smem_raw[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int S = p.raster_m;
    const int kb_box = p.m_tiles;
    const int r = static_cast<int>(ptx::cluster_ctarank());
    const int tile = static_cast<int>(ptx::cluster_id_x());
    const int n0 = tile * C::kRows;
    const int kb_begin = static_cast<int>(static_cast<long long>(r) * p.num_kb / S);
    const int kb_end = static_cast<int>(static_cast<long long>(r + 1) * p.num_kb / S);
    const int nkb = kb_end - kb_begin;
    const bool fp4 = p.idesc_b != 0;
    const uint32_t idesc = C::kIdesc | (((p.idesc_b >> 10) & 7u) << 7);

    const uint32_t smem_base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    auto stage_b = [&](int s) { return smem_base + s * C::kStageBytes; };
    auto stage_a = [&](int s) { return smem_base + s * C::kStageBytes + C::kBBytes; };
    // A's scales [kb_box][TN] (the TMA box), then, for R = 2, the products [kb_box][R][TN];
    // for R = 1 the products overwrite the scales in place
    const uint32_t sa_raw = smem_base + static_cast<uint32_t>(p.stages * C::kStageBytes);
    const uint32_t sc_tab = R == 1 ? sa_raw : sa_raw + static_cast<uint32_t>(kb_box * TN * 4);
    const uint32_t bar_full = ptx::smem_addr(&ctl.full[0]);
    const uint32_t bar_empty = ptx::smem_addr(&ctl.empty[0]);
    const uint32_t bar_tfull = ptx::smem_addr(&ctl.tmem_full[0]);
    const uint32_t bar_tempty = ptx::smem_addr(&ctl.tmem_empty[0]);
    const uint32_t bar_scales = ptx::smem_addr(&ctl.scales);
    const uint32_t bar_drain = ptx::smem_addr(&ctl.drain);
    volatile int *abort_flag = &ctl.abort_flag;
    ptx::griddep_launch_dependents();  // the next grid may start its set-up as SMs free up

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1);
            ptx::mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < C::kBufs; ++b) {
            ptx::mbar_init(bar_tfull + 8 * b, 1);
            ptx::mbar_init(bar_tempty + 8 * b, kNumMathWarps);
        }
        ptx::mbar_init(bar_scales, 1);
        ptx::mbar_init(bar_drain, 1);
        ptx::mbar_init(ptx::smem_addr(&ctl.stall), 1);
        ctl.abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
        ptx::prefetch_tmap(&tmap_sa);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(&ctl.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    // no global memory is touched before the grids this one depends on are complete
    ptx::griddep_wait();
    // The producer issues A's scales and its first stages at once (they need only this CTA's
    // barriers, initialised by its own lane 0), so their DRAM latency overlaps the set-up.
    const uint32_t tx = fp4 ? C::kTxBytesFp4B : C::kTxBytes;
    uint32_t n_op = 0;  // producer: operand loads issued
    int ps = 0;         // producer: next stage
    uint32_t pph = 0;   // producer: its phase
    if (warp == 0) {
        __syncwarp();
        const int pre = min(p.stages, (nkb + KS - 1) / KS);
        if (ptx::elect_one()) {
            ptx::mbar_arrive_expect_tx(bar_scales, static_cast<uint32_t>(kb_box * TN * 4));
            ptx::tma_load_3d(sa_raw, &tmap_sa, bar_scales, 0, kb_begin, 0);
            for (int i = 0; i < pre; ++i) {
                const uint32_t fb = bar_full + 8 * i;
                ptx::mbar_arrive_expect_tx(fb, tx);
                ptx::tma_load_4d(stage_b(i), &tmap_b, fb, 0, n0, kb_begin + i * KS, 0);
                ptx::tma_load_4d(stage_a(i), &tmap_a, fb, 0, 0, kb_begin + i * KS, 0);
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
                    ptx::mbar_arrive_expect_tx(fb, tx);
                    ptx::tma_load_4d(stage_b(s), &tmap_b, fb, 0, n0, kb0, 0);
                    ptx::tma_load_4d(stage_a(s), &tmap_a, fb, 0, 0, kb0, 0);
                }
                __syncwarp();
                ++n_op;
                if (++s == p.stages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            // wind-down: every copy issued has landed before shared memory is reused or freed
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
            wait_drain(bar_scales, 0);
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
                        const uint64_t bdesc = ptx::sdesc_kmajor_sw128(stage_a(s) + kk * C::kAKbBytes);
#pragma unroll
                        for (int rb = 0; rb < R; ++rb) {
                            const uint64_t adesc = ptx::sdesc_kmajor_sw128(
                                stage_b(s) + kk * C::kBKbBytes + rb * kBlockM * kBlockK);
                            const uint32_t d_tmem =
                                tmem_base + static_cast<uint32_t>(buf * C::kBufCols + rb * TN);
#pragma unroll
                            for (int k = 0; k < kBlockK / kUmmaK; ++k)
                                ptx::mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc,
                                                k > 0 ? 1u : 0u);
                        }
                        ptx::mma_commit(bar_tfull + 8 * buf);
                    }
                    __syncwarp();
                    if (++buf == C::kBufs) {
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
        // producer and MMA warps take part only in the cluster barriers below
        ptx::tc_fence_before();
        ptx::cluster_sync();
        ptx::cluster_sync();
    } else {
        ptx::setmaxnreg_inc<232>();
        const int mw = warp - kFirstMathWarp;
        const int half = mw / 4;
        const int q = warp % 4;                            // TMEM lane quarter of this warp
        const int col_off = half * C::kCols;               // first buffer column of this thread
        const int rb = col_off / TN;                       // its 128-row block of B
        const int tok0 = col_off % TN;                     // its first token
        const int n_local = rb * kBlockM + q * 32 + lane;  // its B row within the tile
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(col_off);
        const int t = threadIdx.x - kFirstMathWarp * 32;   // 0 .. 255

        // ---- the scale products sa[token] * sb[block] of this CTA's K range, once ----
        bool ok = __all_sync(0xffffffffu, wait_one(bar_scales, 0, p, abort_flag));
        if (ok) {
            const int nb0 = n0 / kBlockK;
            for (int e = t; e < nkb * R * TN; e += kNumMathWarps * 32) {
                const int kbl = e / (R * TN);
                const int rbe = (e / TN) % R;
                const int j = e % TN;
                const int nb = min(nb0 + rbe, p.num_nb - 1);
                const float sb = __ldg(p.sfb + static_cast<size_t>(nb) * p.num_kb + kb_begin + kbl);
                const float sa = ld_shared_f32(sa_raw + static_cast<uint32_t>((kbl * TN + j) * 4));
                st_shared_f32(sc_tab + static_cast<uint32_t>(e * 4), sa * sb);
            }
        }
        promotion_bar_sync();

        // ---- promotion over this CTA's K blocks ----
        float acc[C::kCols];
#pragma unroll
        for (int c = 0; c < C::kCols; ++c)
            acc[c] = 0.0f;
        int buf = 0;
        uint32_t bph = 0;
        for (int kbl = 0; kbl < nkb && ok; ++kbl) {
            if (!__all_sync(0xffffffffu, wait_one(bar_tfull + 8 * buf, bph, p, abort_flag))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t taddr = lane_base + static_cast<uint32_t>(buf * C::kBufCols);
            const uint32_t cbase = sc_tab + static_cast<uint32_t>(((kbl * R + rb) * TN + tok0) * 4);
            const uint32_t rel = bar_tempty + 8 * buf;
            auto release = [&]() {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(rel);
            };
            uint32_t pr[C::kPart1];
            ptx::tmem_ld_cols<C::kPart1>(taddr, pr);
            ptx::tmem_wait_cols<C::kPart1>(pr);
            if (C::kPart2 == 0)
                release();  // the whole partial is in registers: free the buffer first
#pragma unroll
            for (int c = 0; c < C::kPart1; c += 4) {
                const float4 f = ld_shared_v4f(cbase + static_cast<uint32_t>(c * 4));
                acc[c + 0] = fmaf(__uint_as_float(pr[c + 0]), f.x, acc[c + 0]);
                acc[c + 1] = fmaf(__uint_as_float(pr[c + 1]), f.y, acc[c + 1]);
                acc[c + 2] = fmaf(__uint_as_float(pr[c + 2]), f.z, acc[c + 2]);
                acc[c + 3] = fmaf(__uint_as_float(pr[c + 3]), f.w, acc[c + 3]);
            }
            if (C::kPart2 > 0) {
                constexpr int P2 = C::kPart2 > 0 ? C::kPart2 : 16;
                ptx::tmem_ld_cols<P2>(taddr + C::kPart1, pr);
                ptx::tmem_wait_cols<P2>(pr);
                release();
#pragma unroll
                for (int c = 0; c < C::kPart2; c += 4) {
                    const float4 f = ld_shared_v4f(cbase + static_cast<uint32_t>((C::kPart1 + c) * 4));
                    const int a0 = C::kPart1 + c;
                    acc[a0 + 0] = fmaf(__uint_as_float(pr[c + 0]), f.x, acc[a0 + 0]);
                    acc[a0 + 1] = fmaf(__uint_as_float(pr[c + 1]), f.y, acc[a0 + 1]);
                    acc[a0 + 2] = fmaf(__uint_as_float(pr[c + 2]), f.z, acc[a0 + 2]);
                    acc[a0 + 3] = fmaf(__uint_as_float(pr[c + 3]), f.w, acc[a0 + 3]);
                }
            }
            if (++buf == C::kBufs) {
                buf = 0;
                bph ^= 1;
            }
        }

        // ---- the partial, token-major, into this CTA's shared memory (the operand stages are
        // drained: every MMA of this CTA completed before its last partial was read) ----
        const int m_valid = min(p.M, TN);
#pragma unroll
        for (int c = 0; c < C::kCols; ++c) {
            if (tok0 + c < m_valid)
                st_shared_f32(smem_base + static_cast<uint32_t>(((tok0 + c) * C::kRows + n_local) * 4),
                              acc[c]);
        }
        ptx::tc_fence_before();
        ptx::cluster_sync();  // every CTA's partial is in place

        // ---- reduction of this CTA's slice over the S partials, fixed order ----
        // A chunk is 4 consecutive B rows of one token; CTA r takes chunks [r C / S, (r+1) C / S).
        constexpr int kChunksPerTok = C::kRows / 4;
        constexpr int kThreads = kNumMathWarps * 32;
        constexpr int kBatch = 4;
        const int n_chunks = m_valid * kChunksPerTok;
        const int c_begin = static_cast<int>(static_cast<long long>(r) * n_chunks / S);
        const int c_end = static_cast<int>(static_cast<long long>(r + 1) * n_chunks / S);
        for (int c0 = c_begin + t; c0 < c_end; c0 += kBatch * kThreads) {
            float4 v[kBatch][kMaxSplits];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int ci = c0 + j * kThreads;
                if (ci < c_end) {
                    const int tok = ci / kChunksPerTok;
                    const int nl = (ci % kChunksPerTok) * 4;
                    const uint32_t local = smem_base + static_cast<uint32_t>((tok * C::kRows + nl) * 4);
#pragma unroll
                    for (int s2 = 0; s2 < kMaxSplits; ++s2)
                        if (s2 < S)
                            v[j][s2] = ld_shared_cluster_v4(ptx::map_to_rank(local, static_cast<uint32_t>(s2)));
                }
            }
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                const int ci = c0 + j * kThreads;
                if (ci < c_end) {
                    const int tok = ci / kChunksPerTok;
                    const int col = n0 + (ci % kChunksPerTok) * 4;
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
                        __nv_bfloat16 *dst = p.d + static_cast<size_t>(tok) * p.N + col;
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
