// dg_swap_sk_kernel.cuh -- stream-K variant of the swapped-operand kernel: every SM takes an
// equal share of the K blocks of a small-M dense problem, and the partial sums of a tile are
// added through a global workspace.
//
// Same method and tile as dg_swap_kernel.cuh (DeepSeek開源第三彈 -- the DeepGEMM release
// write-up -- "深入了解DeepGEMM": fine-grained scales, two-level accumulation; the MMA computes
// D^T = B . A^T with 128 rows of B on its 128-lane side and the TN tokens on its N side).  What
// differs is how the work is cut.  The cluster kernel splits each tile's K range evenly over the
// S CTAs of a cluster, so its grid is (tiles x S) CTAs, often well under the SM count (56 tiles
// of 7168 rows of B fill 112 SMs at S = 2 and cannot use 3).  Here the problem is a line of
// U = tiles x K/128 units (one K block of one tile); CTA i of P takes units
// [i U / P, (i + 1) U / P), so all P = #SMs CTAs stream the same number of K blocks of B.  A
// CTA's range covers the end of one tile and the start of the next at most (P >= tiles keeps it
// under one tile's K blocks), i.e. one or two segments.  For each segment it promotes the
// partial exactly as the cluster kernel does and stores it (fp32, token-major) in its own slot
// of the workspace; the last contributor of a tile -- found with an atomic counter per tile --
// adds the tile's partials in K order (the same fixed order whoever arrives last, so the result
// does not depend on timing), rounds to bf16, writes D, and returns the counter to zero.
#pragma once

#include "dg_swap_kernel.cuh"

namespace dg {

// First unit of CTA i when U units are split over P CTAs.
__host__ __device__ __forceinline__ long long sk_unit_begin(long long i, long long U, int P)
{
    return i * U / P;
}

// The contributors of tile t: CTAs j_lo .. j_lo + n - 1 (consecutive).
__device__ __forceinline__ void sk_contributors(int t, int num_kb, long long U, int P, int &j_lo, int &n)
{
    const long long x0 = static_cast<long long>(t) * num_kb;   // first unit of the tile
    const long long x1 = x0 + num_kb;                           // one past its last
    long long j = x0 * P / U;                                   // estimate, then exact
    if (j > 0)
        --j;
    while (j + 1 < P && sk_unit_begin(j + 1, U, P) <= x0)
        ++j;
    j_lo = static_cast<int>(j);
    n = 0;
    while (j < P && sk_unit_begin(j, U, P) < x1) {
        ++n;
        ++j;
    }
}

// Params conventions: p.n_tiles counts tiles of 128 B rows; p.m_tiles holds H, the most units
// a CTA takes (the height of each A-scale box); p.ws / p.ws_count are the workspace's partial
// slots (2 per CTA, TN x 128 floats each) and its per-tile counters.  The grid is P CTAs, no
// clusters.  B-format bits in p.idesc_b (E2M1) move to the A-format field as in the cluster
// kernel.
template <int TN>
__global__ void __launch_bounds__(kNumThreads, 1)
    dg_gemm_swap_sk_kernel(const __grid_constant__ CUtensorMap tmap_a,
                           const __grid_constant__ CUtensorMap tmap_b,
                           const __grid_constant__ CUtensorMap tmap_sa, const Params p)
{
    using C = SwapCfg<TN, 1>;
    constexpr int KS = kSwapKbPerStage;
    __shared__ SwapCtl ctl;
    __shared__ int s_last;
    extern __shared__ uint8_t smem_raw[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int P = static_cast<int>(gridDim.x);
    const int H = p.m_tiles;
    const long long U = static_cast<long long>(p.n_tiles) * p.num_kb;
    const long long u0 = sk_unit_begin(blockIdx.x, U, P);
    const long long u1 = sk_unit_begin(blockIdx.x + 1, U, P);
    // the CTA's segments s = 0, 1: (tile t0 + s, first K block, K blocks)
    const int t0 = static_cast<int>(u0 / p.num_kb);
    const int kb00 = static_cast<int>(u0 - static_cast<long long>(t0) * p.num_kb);
    const int nkb0 = static_cast<int>(min(u1, static_cast<long long>(t0 + 1) * p.num_kb) - u0);
    const int nseg = (u1 > static_cast<long long>(t0 + 1) * p.num_kb) ? 2 : 1;
    const int nkb1 = nseg == 2 ? static_cast<int>(u1 - static_cast<long long>(t0 + 1) * p.num_kb) : 0;
    auto seg_tile = [&](int sg) { return t0 + sg; };
    auto seg_kb0 = [&](int sg) { return sg == 0 ? kb00 : 0; };
    auto seg_nkb = [&](int sg) { return sg == 0 ? nkb0 : nkb1; };
    const bool fp4 = p.idesc_b != 0;
    const uint32_t idesc = C::kIdesc | (((p.idesc_b >> 10) & 7u) << 7);

    const uint32_t smem_base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    auto stage_b = [&](int s) { return smem_base + s * C::kStageBytes; };
    auto stage_a = [&](int s) { return smem_base + s * C::kStageBytes + C::kBBytes; };
    // A's scales of segment s [H][TN] at sa_raw + s H TN, replaced in place by the products
    // sa[token] * sb[block of the segment's tile]
    const uint32_t sa_raw = smem_base + static_cast<uint32_t>(p.stages * C::kStageBytes);
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
    const uint32_t tx = fp4 ? C::kTxBytesFp4B : C::kTxBytes;
    // The stages of the CTA in order: segment s, K blocks [kb, kb + KS) within it.  The
    // producer issues A's scales and its first stages during set-up (they need only this CTA's
    // barriers), so their DRAM latency overlaps the set-up.
    int pseg = 0, pkb = 0;  // producer: next stage to load
    uint32_t n_op = 0;
    int ps = 0;
    uint32_t pph = 0;
    if (warp == 0) {
        __syncwarp();
        if (ptx::elect_one()) {
            ptx::mbar_arrive_expect_tx(bar_scales, static_cast<uint32_t>(nseg * H * TN * 4));
            for (int s = 0; s < nseg; ++s)
                ptx::tma_load_3d(sa_raw + static_cast<uint32_t>(s * H * TN * 4), &tmap_sa, bar_scales, 0,
                                 seg_kb0(s), 0);
        }
        __syncwarp();
        while (pseg < nseg && static_cast<int>(n_op) < p.stages) {
            if (ptx::elect_one()) {
                const uint32_t fb = bar_full + 8 * ps;
                ptx::mbar_arrive_expect_tx(fb, tx);
                ptx::tma_load_4d(stage_b(ps), &tmap_b, fb, 0, seg_tile(pseg) * kBlockM, seg_kb0(pseg) + pkb, 0);
                ptx::tma_load_4d(stage_a(ps), &tmap_a, fb, 0, 0, seg_kb0(pseg) + pkb, 0);
            }
            __syncwarp();
            ++n_op;
            if (++ps == p.stages) {
                ps = 0;
                pph ^= 1;
            }
            pkb += KS;
            if (pkb >= seg_nkb(pseg)) {
                pkb = 0;
                ++pseg;
            }
        }
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
            while (pseg < nseg) {
                if (!__all_sync(0xffffffffu, wait_one(bar_empty + 8 * s, ph ^ 1, p, abort_flag)))
                    break;
                if (ptx::elect_one()) {
                    const uint32_t fb = bar_full + 8 * s;
                    ptx::mbar_arrive_expect_tx(fb, tx);
                    ptx::tma_load_4d(stage_b(s), &tmap_b, fb, 0, seg_tile(pseg) * kBlockM, seg_kb0(pseg) + pkb, 0);
                    ptx::tma_load_4d(stage_a(s), &tmap_a, fb, 0, 0, seg_kb0(pseg) + pkb, 0);
                }
                __syncwarp();
                ++n_op;
                if (++s == p.stages) {
                    s = 0;
                    ph ^= 1;
                }
                pkb += KS;
                if (pkb >= seg_nkb(pseg)) {
                    pkb = 0;
                    ++pseg;
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
            for (int sg = 0; sg < nseg && ok; ++sg) {
                for (int kb = 0; kb < seg_nkb(sg) && ok; kb += KS) {
                    if (!__all_sync(0xffffffffu, wait_one(bar_full + 8 * s, ph, p, abort_flag))) {
                        ok = false;
                        break;
                    }
                    const int nk = (seg_nkb(sg) - kb) < KS ? (seg_nkb(sg) - kb) : KS;
                    for (int kk = 0; kk < nk; ++kk) {
                        if (!__all_sync(0xffffffffu, wait_one(bar_tempty + 8 * buf, bph ^ 1, p, abort_flag))) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        if (ptx::elect_one()) {
                            const uint64_t bdesc = ptx::sdesc_kmajor_sw128(stage_a(s) + kk * C::kAKbBytes);
                            const uint64_t adesc = ptx::sdesc_kmajor_sw128(stage_b(s) + kk * C::kBKbBytes);
                            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * C::kBufCols);
#pragma unroll
                            for (int k = 0; k < kBlockK / kUmmaK; ++k)
                                ptx::mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0 ? 1u : 0u);
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
            }
            if (ptx::elect_one())
                ptx::mma_commit(bar_drain);
            __syncwarp();
            wait_drain(bar_drain, 0);
            __syncwarp();
        }
    } else {
        ptx::setmaxnreg_inc<232>();
        const int mw = warp - kFirstMathWarp;
        const int half = mw / 4;
        const int q = warp % 4;                            // TMEM lane quarter of this warp
        const int tok0 = half * C::kCols;                  // first token of this thread
        const int n_local = q * 32 + lane;                 // its B row within the tile
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(tok0);
        const int t = threadIdx.x - kFirstMathWarp * 32;   // 0 .. 255
        const int m_valid = min(p.M, TN);

        // ---- the scale products of both segments, once ----
        bool ok = __all_sync(0xffffffffu, wait_one(bar_scales, 0, p, abort_flag));
        if (ok) {
            for (int sg = 0; sg < nseg; ++sg) {
                const int nb = min(seg_tile(sg), p.num_nb - 1);
                const uint32_t tab = sa_raw + static_cast<uint32_t>(sg * H * TN * 4);
                for (int e = t; e < seg_nkb(sg) * TN; e += kNumMathWarps * 32) {
                    const int kbl = e / TN;
                    const float sb = __ldg(p.sfb + static_cast<size_t>(nb) * p.num_kb + seg_kb0(sg) + kbl);
                    st_shared_f32(tab + static_cast<uint32_t>(e * 4),
                                  ld_shared_f32(tab + static_cast<uint32_t>(e * 4)) * sb);
                }
            }
        }
        promotion_bar_sync();

        int buf = 0;
        uint32_t bph = 0;
        for (int sg = 0; sg < nseg; ++sg) {
            // ---- promotion over the segment's K blocks ----
            float acc[C::kCols];
#pragma unroll
            for (int c = 0; c < C::kCols; ++c)
                acc[c] = 0.0f;
            const uint32_t tab = sa_raw + static_cast<uint32_t>(sg * H * TN * 4);
            for (int kbl = 0; kbl < seg_nkb(sg) && ok; ++kbl) {
                if (!__all_sync(0xffffffffu, wait_one(bar_tfull + 8 * buf, bph, p, abort_flag))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t taddr = lane_base + static_cast<uint32_t>(buf * C::kBufCols);
                const uint32_t cbase = tab + static_cast<uint32_t>((kbl * TN + tok0) * 4);
                uint32_t pr[C::kCols];
                ptx::tmem_ld_cols<C::kCols>(taddr, pr);
                ptx::tmem_wait_cols<C::kCols>(pr);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    ptx::mbar_arrive(bar_tempty + 8 * buf);
#pragma unroll
                for (int c = 0; c < C::kCols; c += 4) {
                    const float4 f = ld_shared_v4f(cbase + static_cast<uint32_t>(c * 4));
                    acc[c + 0] = fmaf(__uint_as_float(pr[c + 0]), f.x, acc[c + 0]);
                    acc[c + 1] = fmaf(__uint_as_float(pr[c + 1]), f.y, acc[c + 1]);
                    acc[c + 2] = fmaf(__uint_as_float(pr[c + 2]), f.z, acc[c + 2]);
                    acc[c + 3] = fmaf(__uint_as_float(pr[c + 3]), f.w, acc[c + 3]);
                }
                if (++buf == C::kBufs) {
                    buf = 0;
                    bph ^= 1;
                }
            }
            ok = __all_sync(0xffffffffu, ok);

            // ---- the partial, token-major, into this segment's workspace slot ----
            const int tile = seg_tile(sg);
            float *slot = p.ws + (static_cast<size_t>(blockIdx.x) * 2 + sg) * (TN * kBlockM);
            if (ok) {
#pragma unroll
                for (int c = 0; c < C::kCols; ++c)
                    if (tok0 + c < m_valid)
                        slot[(tok0 + c) * kBlockM + n_local] = acc[c];
            }
            __threadfence();
            promotion_bar_sync();  // every thread's partial is stored and fenced
            int j_lo, n_contrib;
            sk_contributors(tile, p.num_kb, U, P, j_lo, n_contrib);
            if (t == 0) {
                // a wait that gave up anywhere in the CTA (the abort flag is set before the
                // waiting thread reaches the barrier above) leaves the tile to the error path
                int last = 0;
                if (ok && !*abort_flag) {
                    const int old = atomicAdd(p.ws_count + tile, 1);
                    last = old == n_contrib - 1;
                    if (last)
                        p.ws_count[tile] = 0;  // back to zero for the next call
                }
                s_last = last;
            }
            promotion_bar_sync();
            if (s_last) {
                // ---- the tile's sum over its contributors in K order, rounded to bf16 ----
                // A chunk is 4 consecutive B rows of one token; a thread owns up to kMaxChunks of
                // them and, for up to kGroup contributors at a time, issues every load before any
                // add (one L2 round trip per group, not per load); the adds keep the K order.
                __threadfence();
                constexpr int kChunksPerTok = kBlockM / 4;
                constexpr int kThreads = kNumMathWarps * 32;
                constexpr int kMaxChunks = (TN * kChunksPerTok + kThreads - 1) / kThreads;
                constexpr int kGroup = kMaxChunks <= 4 ? 4 : 2;
                const int n_chunks = m_valid * kChunksPerTok;
                const int n0 = tile * kBlockM;
                float4 sum[kMaxChunks];
                for (int g0 = 0; g0 < n_contrib; g0 += kGroup) {
                    float4 v[kGroup][kMaxChunks];
#pragma unroll
                    for (int jj = 0; jj < kGroup; ++jj) {
                        if (g0 + jj < n_contrib) {
                            const int j = j_lo + g0 + jj;
                            // the tile is CTA j's first segment unless j starts in the tile before
                            const int sj = (sk_unit_begin(j, U, P) / p.num_kb == tile) ? 0 : 1;
                            const float *src = p.ws + (static_cast<size_t>(j) * 2 + sj) * (TN * kBlockM);
#pragma unroll
                            for (int c = 0; c < kMaxChunks; ++c) {
                                const int ci = t + c * kThreads;
                                if (ci < n_chunks)
                                    v[jj][c] = __ldcg(reinterpret_cast<const float4 *>(
                                        src + (ci / kChunksPerTok) * kBlockM + (ci % kChunksPerTok) * 4));
                            }
                        }
                    }
#pragma unroll
                    for (int jj = 0; jj < kGroup; ++jj) {
                        if (g0 + jj < n_contrib) {
#pragma unroll
                            for (int c = 0; c < kMaxChunks; ++c) {
                                if (g0 + jj == 0) {
                                    sum[c] = v[jj][c];
                                } else {
                                    sum[c].x += v[jj][c].x;
                                    sum[c].y += v[jj][c].y;
                                    sum[c].z += v[jj][c].z;
                                    sum[c].w += v[jj][c].w;
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (int c = 0; c < kMaxChunks; ++c) {
                    const int ci = t + c * kThreads;
                    const int col = n0 + (ci % kChunksPerTok) * 4;
                    if (ci < n_chunks && col < p.N) {
                        __nv_bfloat16 *dst = p.d + static_cast<size_t>(ci / kChunksPerTok) * p.N + col;
                        st_global_v2(dst, ptx::pack_bf16x2(sum[c].x, sum[c].y), ptx::pack_bf16x2(sum[c].z, sum[c].w));
                    }
                }
            }
        }
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
