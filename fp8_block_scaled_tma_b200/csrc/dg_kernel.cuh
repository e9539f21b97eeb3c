// dg_kernel.cuh -- the sm_100a FP8 block-scaled NT GEMM kernel (dense, contiguous-grouped and
// masked-grouped layouts share it; only the tile scheduler differs).
//
// Method (DeepSeek開源第三彈 -- the DeepGEMM release write-up -- "深入了解DeepGEMM"): FP8 inputs
// with DeepSeek-V3 fine-grained scales (fp32 per 1x128 tile of A, per 128x128 block of B), and
// two-level accumulation: the tensor cores form the product of one 128-wide K slice, the CUDA
// cores multiply it by sa*sb and add it to an fp32 accumulator.  The layouts are those of
// "如何使用" (NT dense, MoE contiguous, MoE masked).
//
// Blackwell design (one CTA of 384 threads per SM, persistent over output tiles):
//   warp 0          TMA producer: per K block loads A [128 x 128 B] and B [BN x 128 B] (both with
//                   the 128-byte swizzle) into one operand stage.  Each TMA copy costs the copy
//                   engine a fixed amount of time besides its bytes, so the small fp32 scales
//                   are not copied by TMA: the promotion threads read them from global memory.
//   warp 1          allocates tensor memory, then issues 4 x tcgen05.mma kind::f8f6f4 (K = 32
//                   each) per K block into one of NB TMEM buffers of BN fp32 columns, and
//                   commits the stage (free) and the buffer (full) to mbarriers.
//   warps 4..11     promotion: each thread owns one output row (its TMEM lane) and BN/2
//                   columns; per K block it loads the fresh partial from TMEM, frees the
//                   buffer, and adds partial * sa[row] * sb[block] into fp32 registers (sa and
//                   sb are read with plain loads two K blocks ahead).  After the last K
//                   block it rounds to bf16, stages its 32-row slice of the tile in shared
//                   memory and writes it with one to three TMA stores.
// Every wait is bounded by a %globaltimer limit; on expiry the kernel records DG_ERR_TIMEOUT,
// drains its outstanding copies and MMAs, frees tensor memory and returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

constexpr int kBlockM = 128;           // rows per tile (one TMEM lane each)
constexpr int kBlockK = 128;           // K per scale block = K per promotion
constexpr int kUmmaK = 32;             // K of one tcgen05.mma kind::f8f6f4
constexpr int kNumThreads = 384;
constexpr int kNumMathWarps = 8;
constexpr int kFirstMathWarp = 4;
constexpr int kMaxStages = 8;
constexpr int kTmemCols = 512;
constexpr int kMaxMaskedGroups = 1024;
constexpr uint64_t kDrainTimeoutNs = 1000000000ull;  // fixed bound for the wind-down waits

constexpr int kErrTimeout = -4;
constexpr int kErrLayout = -6;

enum Layout : int { kDense = 0, kContiguous = 1, kMasked = 2 };

struct Params {
    int M;          // dense: M, contiguous: M_total, masked: M_max
    int N;
    int K;
    int G;
    int num_kb;     // K / 128
    int num_nb;     // ceil(N / 128): scale blocks of B along N
    int m_tiles;    // ceil(M / 128)
    int n_tiles;    // ceil(N / BN)
    int num_tiles;  // dense / contiguous: m_tiles * n_tiles; masked: computed on the device
    int stages;
    int raster_m;   // m-tiles per raster band (dense / contiguous)
    const float *sfa;   // A scales, MN-major: sfa[(a_z * num_kb + kb) * sfa_ld + row]
    int sfa_ld;         // align4(rows of a group)
    const float *sfb;
    __nv_bfloat16 *d;
    const int *m_indices;
    const int *masked_m;
    int *err;
    unsigned long long timeout_ns;
    int inject_stall;   // test hook: the MMA issuer first waits on a barrier nothing signals
    uint32_t idesc_b;   // B-format bits of the MMA instruction descriptor: 0 e4m3, or e2m1
                        // (FP4 B, staged by TMA in the padded 8-bit layout of kind::f8f6f4)
    float *ws;          // stream-K kernel: the workspace's fp32 partial slots
    int *ws_count;      // stream-K kernel: its per-tile arrival counters (zero between calls)
};

template <int BN>
struct Cfg {
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32, 256]");
    static constexpr int kCols = BN / 2;                      // columns per promotion thread
    // The partial of one K block is read from TMEM in one burst when the accumulator and the
    // partial fit in registers together (kCols <= 96), else in two halves.
    static constexpr int kPart1 = (kCols <= 96) ? kCols : ((kCols / 2 + 15) / 16 * 16);
    static constexpr int kTmemBufs = (kTmemCols / BN) >= 4 ? 4 : (kTmemCols / BN);
    static constexpr int kABytes = kBlockM * kBlockK;         // 16 KB
    static constexpr int kBBytes = BN * kBlockK;
    static constexpr int kStageBytes = kABytes + kBBytes;     // multiple of 1024
    static constexpr uint32_t kTxBytes = kABytes + kBBytes;
    // TMA counts a packed E2M1 operand at 4 bits per element, though it lands in shared memory
    // at 8 bits per element (16 values, then 8 bytes of gap)
    static constexpr uint32_t kTxBytesFp4B = kABytes + kBBytes / 2;
    static constexpr uint32_t kIdesc = ptx::idesc_e4m3_f32(kBlockM, BN);
};

// Static shared memory: barriers and the bookkeeping words.
constexpr int kSfaSlots = 8;  // A-scale ring of the CTA-pair kernel (one slot per stage)

struct SmemCtl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t sfa_full[kSfaSlots];
    uint64_t sfa_empty[kSfaSlots];
    uint64_t tmem_full[4];
    uint64_t tmem_empty[4];
    uint64_t drain;
    uint64_t stall;      // never signalled: the target of the fault-injection test hook
    uint32_t tmem_base;
    int abort_flag;
    int total_tiles;
    int tile_prefix[kMaxMaskedGroups + 1];
};

struct Tile {
    int g;       // group (expert) of the tile; 0 for dense
    int m0;      // first row of the tile within its group
    int n0;      // first column
    int a_z;     // TMA z coordinate of A / SFA (group for masked, else 0)
};

__device__ __forceinline__ void record_error(int *err, int code)
{
    atomicCAS(err, 0, code);
}

// Resolves tile t to its coordinates.  Returns false when the tile has no valid row and must
// be skipped (contiguous layout only).  All roles call it with the same t and read the same
// (read-only) index arrays, so they agree.
template <int L>
__device__ __forceinline__ bool resolve_tile(const Params &p, const SmemCtl &ctl, int t, Tile &ti)
{
    if (L == kMasked) {
        // find g with prefix[g] <= t < prefix[g + 1]
        int lo = 0, hi = p.G - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (ctl.tile_prefix[mid] <= t)
                lo = mid;
            else
                hi = mid - 1;
        }
        int g = lo;
        int mm = __ldg(p.masked_m + g);
        mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
        int mt = (mm + kBlockM - 1) / kBlockM;
        int local = t - ctl.tile_prefix[g];
        ti.g = g;
        ti.m0 = (local % mt) * kBlockM;
        ti.n0 = (local / mt);  // scaled by BN by the caller
        ti.a_z = g;
        return true;
    } else {
        int band = p.raster_m * p.n_tiles;
        int b = t / band;
        int r = t - b * band;
        int m_base = b * p.raster_m;
        int h = p.m_tiles - m_base;
        h = h < p.raster_m ? h : p.raster_m;
        ti.m0 = (m_base + r % h) * kBlockM;
        ti.n0 = r / h;
        ti.a_z = 0;
        ti.g = 0;
        if (L == kContiguous) {
            // the tile's expert is that of its first non-padding row; an index below -1 breaks
            // the layout contract (reported, and the row is treated as padding: not written)
            int g = __ldg(p.m_indices + ti.m0);
            if (g < -1)
                record_error(p.err, kErrLayout);
            if (g < 0) {
                int end = ti.m0 + kBlockM < p.M ? ti.m0 + kBlockM : p.M;
                for (int r2 = ti.m0 + 1; r2 < end && g < 0; ++r2) {
                    g = __ldg(p.m_indices + r2);
                    if (g < -1)
                        record_error(p.err, kErrLayout);
                }
            }
            if (g < 0)
                return false;          // an all-padding tile: nothing to write
            if (g >= p.G) {
                record_error(p.err, kErrLayout);
                return false;
            }
            ti.g = g;
        }
        return true;
    }
}

// Bounded wait by one thread.  Returns false on timeout or when another role aborted.
__device__ __forceinline__ bool wait_one(uint32_t bar, uint32_t parity, const Params &p,
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

// Wait used while winding down: a fixed bound independent of the configurable limit.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = ptx::global_timer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::global_timer_ns() - t0 > kDrainTimeoutNs)
            return false;
    }
    return true;
}

// Scales a promotion thread needs for one K block: sa of its row and sb of the (at most two)
// 128-column blocks of B its columns touch.
struct KbScales {
    float sa, lo, hi;
};

__device__ __forceinline__ void load_kb_scales(KbScales &s, const float *sa_ptr, const float *sb_lo,
                                               const float *sb_hi, int ld, int kb, int nkb)
{
    kb = kb < nkb ? kb : nkb - 1;
    s.sa = __ldg(sa_ptr + static_cast<size_t>(kb) * ld);
    s.lo = __ldg(sb_lo + kb);
    s.hi = __ldg(sb_hi + kb);
}

// Promotion of one K block by one thread: waits for the partial in TMEM buffer `buf`, reads the
// thread's kCols columns (in one burst when P2 == 0, else in two), frees the buffer by arriving
// on `release_bar` (a cluster address when `remote`), and adds partial * sa * sb into acc.
// Columns >= split use the higher B scale block.  Returns false when the wait gave up.
// The scale products are formed after the TMEM wait so that a late scale never delays the
// release of the buffer.
template <int P1, int P2, int NCOLS>
__device__ __forceinline__ bool promote_kb(float (&acc)[NCOLS], float sa, float sb_lo, float sb_hi,
                                           uint32_t taddr, uint32_t full_bar, uint32_t parity,
                                           uint32_t release_bar, bool remote, int split,
                                           int lane, const Params &p, volatile int *abort_flag)
{
    if (!__all_sync(0xffffffffu, wait_one(full_bar, parity, p, abort_flag)))
        return false;
    ptx::tc_fence_after();
    uint32_t pr[P1];
    ptx::tmem_ld_cols<P1>(taddr, pr);
    ptx::tmem_wait_cols<P1>(pr);
    auto release = [&]() {
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if (remote)
                ptx::mbar_arrive_cluster(release_bar);
            else
                ptx::mbar_arrive(release_bar);
        }
    };
    if (P2 == 0)
        release();  // the whole partial is in registers: free the buffer before the arithmetic
    const float scale_lo = sa * sb_lo;
    const float scale_hi = sa * sb_hi;
    // two columns per packed FMA (the promotion's FMAs sit between the two TMEM reads of a
    // wide tile, on the path that recycles the buffer: half the instructions shortens it)
#pragma unroll
    for (int g16 = 0; g16 < P1 / 16; ++g16) {
        const uint64_t ff = ptx::pack_f32x2((16 * g16 >= split) ? scale_hi : scale_lo);
#pragma unroll
        for (int e = 0; e < 16; e += 2)
            ptx::ffma2(acc[16 * g16 + e], acc[16 * g16 + e + 1], pr[16 * g16 + e], pr[16 * g16 + e + 1], ff);
    }
    if (P2 > 0) {
        // second part reuses the same registers
        ptx::tmem_ld_cols<(P2 > 0 ? P2 : 16)>(taddr + P1, pr);
        ptx::tmem_wait_cols<(P2 > 0 ? P2 : 16)>(pr);
        release();
#pragma unroll
        for (int g16 = 0; g16 < P2 / 16; ++g16) {
            const uint64_t ff = ptx::pack_f32x2((P1 + 16 * g16 >= split) ? scale_hi : scale_lo);
#pragma unroll
            for (int e = 0; e < 16; e += 2)
                ptx::ffma2(acc[P1 + 16 * g16 + e], acc[P1 + 16 * g16 + e + 1], pr[16 * g16 + e],
                           pr[16 * g16 + e + 1], ff);
        }
    }
    return true;
}

// The K loop of a promotion thread for one tile.  It is unrolled by two with two named scale
// sets, each reloaded right after its use, so a scale load has a whole K block to land and no
// register move waits on it.  s0 / s1 arrive holding the scales of K blocks 0 and 1 (loaded by
// the caller, early enough to have landed).  `tbuf_release(buf)` gives the barrier address that
// frees buffer `buf` (and whether it is remote).
template <int BN, int P1, int P2, int NCOLS, int NBUF, class Release>
__device__ __forceinline__ bool promote_tile(float (&acc)[NCOLS], KbScales s0, KbScales s1,
                                             const float *sa_ptr, const float *sb_lo,
                                             const float *sb_hi, uint32_t lane_base,
                                             uint32_t bar_tfull, int &buf, uint32_t &bph,
                                             Release tbuf_release, int split, int lane,
                                             const Params &p, volatile int *abort_flag)
{
    auto step = [&](const KbScales &sc) -> bool {
        uint32_t rel;
        bool remote;
        tbuf_release(buf, rel, remote);
        const bool ok = promote_kb<P1, P2>(acc, sc.sa, sc.lo, sc.hi,
                                           lane_base + static_cast<uint32_t>(buf * BN),
                                           bar_tfull + 8 * buf, bph, rel, remote, split, lane, p,
                                           abort_flag);
        if (++buf == NBUF) {
            buf = 0;
            bph ^= 1;
        }
        return ok;
    };
    for (int kb = 0; kb < p.num_kb; kb += 2) {
        if (!step(s0))
            return false;
        load_kb_scales(s0, sa_ptr, sb_lo, sb_hi, p.sfa_ld, kb + 2, p.num_kb);
        if (kb + 1 < p.num_kb) {
            if (!step(s1))
                return false;
            load_kb_scales(s1, sa_ptr, sb_lo, sb_hi, p.sfa_ld, kb + 3, p.num_kb);
        }
    }
    return true;
}

// ---- epilogue -------------------------------------------------------------------------------
// A promotion warp owns 32 output rows x kCols columns of a tile.  It rounds them to bf16 into a
// ring of kEpiBufs staging boxes in shared memory (32 rows x 16 columns each) and hands every
// box to the TMA engine as an asynchronous store, so the warp goes back to promoting the next
// tile while the copy engine writes whole 32-byte sectors of D.  (Direct per-row stores from
// the promotion threads touch 32 rows per instruction and cost more time than the promotion of
// a short-K tile.)  A box row is 32 bytes; with the 32-byte swizzle the 16-byte chunk index is
// XORed with address bit 7 (bit 2 of the row), which puts the warp's 16-byte shared stores on
// distinct banks.  Row-masked warps (a partial masked or contiguous tile) store directly.
constexpr int kEpiCols = 16;
constexpr int kEpiRows = 32;
constexpr int kEpiBoxBytes = kEpiRows * kEpiCols * 2;                    // 1 KB
constexpr int kEpiBufs = 2;
constexpr int kEpiWarpBytes = kEpiBufs * kEpiBoxBytes;
constexpr int kEpiBytes = kNumMathWarps * kEpiWarpBytes;                 // 16 KB per CTA

// Stores this warp's rows [y0, y0 + 32) x columns [x0, x0 + NCOLS) of D (a 2-D view of
// bf16 rows, N wide) through the warp's staging ring `ring`; `ebuf` is the ring position,
// carried across tiles.  The TMA store clips at the view's bounds.
template <int NCOLS>
__device__ __forceinline__ void store_rows_tma(const float (&acc)[NCOLS], const CUtensorMap *tmap_d,
                                               uint32_t ring, int &ebuf, int x0, int y0, int N,
                                               int lane)
{
    static_assert(NCOLS % kEpiCols == 0, "columns per thread must be a multiple of 16");
    const uint32_t sw = static_cast<uint32_t>((lane >> 2) & 1);
#pragma unroll
    for (int c = 0; c < NCOLS / kEpiCols; ++c) {
        if (x0 + c * kEpiCols < N) {
            const uint32_t box = ring + static_cast<uint32_t>(ebuf * kEpiBoxBytes);
            // the store that last read this box must be done reading it
            if (lane == 0)
                ptx::bulk_wait_group_read<kEpiBufs - 1>();
            __syncwarp();
            const uint32_t r = box + static_cast<uint32_t>(lane * kEpiCols * 2);
            const float *v = acc + c * kEpiCols;
            ptx::st_shared_v4(r + (sw << 4), ptx::pack_bf16x2(v[0], v[1]), ptx::pack_bf16x2(v[2], v[3]),
                              ptx::pack_bf16x2(v[4], v[5]), ptx::pack_bf16x2(v[6], v[7]));
            ptx::st_shared_v4(r + ((sw ^ 1u) << 4), ptx::pack_bf16x2(v[8], v[9]),
                              ptx::pack_bf16x2(v[10], v[11]), ptx::pack_bf16x2(v[12], v[13]),
                              ptx::pack_bf16x2(v[14], v[15]));
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_store_2d(tmap_d, box, x0 + c * kEpiCols, y0);
                ptx::bulk_commit_group();
            }
            ebuf = ebuf + 1 == kEpiBufs ? 0 : ebuf + 1;
        }
    }
}

// ---- whole-tile staging (one-CTA kernel) ----
// Each TMA store costs its issuing thread ~190 cycles and each staging round a proxy fence, so
// the one-CTA kernel, whose shared memory allows it, stages a warp's whole 32-row slice of the
// tile at once and writes it with at most three stores: the NCOLS columns split into pieces of
// 64, 32 and 16 columns (box rows of 128, 64 and 32 bytes, each with the swizzle of its row
// width, so the warp's 16-byte shared stores hit distinct banks).  The pieces of all warps are
// grouped by width (all 64-column pieces first), which keeps every piece aligned to its swizzle
// pattern.  The store reading a warp's slice has a whole tile to finish before the warp
// stages its next slice.
template <int NCOLS>
struct EpiPieces {
    static_assert(NCOLS % 16 == 0, "columns per thread must be a multiple of 16");
    static constexpr int kN64 = NCOLS / 64;
    static constexpr int kN32 = (NCOLS % 64) / 32;
    static constexpr int kN16 = (NCOLS % 32) / 16;
    static constexpr int kWarp64 = kN64 * kEpiRows * 64 * 2;  // bytes per warp, 64-column pieces
    static constexpr int kWarp32 = kN32 * kEpiRows * 32 * 2;
    static constexpr int kWarp16 = kN16 * kEpiRows * 16 * 2;
    static constexpr int kCtaBytes = kNumMathWarps * (kWarp64 + kWarp32 + kWarp16);
};

// Host-side twin of EpiPieces<BN / 2>::kCtaBytes.
constexpr int whole_tile_epi_bytes(int bn)
{
    return kNumMathWarps * kEpiRows * (bn / 2) * 2;
}

// One thread's row (`lane` of the box) of a W-column piece at shared address `piece`, from
// v[0 .. W).  The 16-byte chunk j of row r lands at chunk j XOR (the row's swizzle phase).
template <int W>
__device__ __forceinline__ void stage_piece_row(const float *v, uint32_t piece, int lane)
{
    constexpr int kRowBytes = W * 2;
    const uint32_t row = piece + static_cast<uint32_t>(lane * kRowBytes);
    const uint32_t sw = static_cast<uint32_t>((lane * kRowBytes) >> 7) & (kRowBytes / 16 - 1);
#pragma unroll
    for (int j = 0; j < W / 8; ++j)
        ptx::st_shared_v4(row + ((static_cast<uint32_t>(j) ^ sw) << 4),
                          ptx::pack_bf16x2(v[8 * j], v[8 * j + 1]), ptx::pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                          ptx::pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), ptx::pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}

// Stores this warp's rows [y0, y0 + 32) x columns [x0, x0 + NCOLS) of D through the warp's
// whole-tile staging: `s64`, `s32`, `s16` are the warp's first piece of each width.
template <int NCOLS>
__device__ __forceinline__ void store_rows_whole(const float (&acc)[NCOLS], const CUtensorMap *map64,
                                                 const CUtensorMap *map32, const CUtensorMap *map16,
                                                 uint32_t s64, uint32_t s32, uint32_t s16, int x0,
                                                 int y0, int N, int lane)
{
    using E = EpiPieces<NCOLS>;
    // the stores of this warp's previous tile must be done reading the staging
    if (lane == 0)
        ptx::bulk_wait_group_read<0>();
    __syncwarp();
#pragma unroll
    for (int i = 0; i < E::kN64; ++i)
        stage_piece_row<64>(acc + 64 * i, s64 + static_cast<uint32_t>(i * kEpiRows * 128), lane);
    if constexpr (E::kN32 > 0)
        stage_piece_row<32>(acc + 64 * E::kN64, s32, lane);
    if constexpr (E::kN16 > 0)
        stage_piece_row<16>(acc + 64 * E::kN64 + 32 * E::kN32, s16, lane);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < E::kN64; ++i)
            if (x0 + 64 * i < N)
                ptx::tma_store_2d(map64, s64 + static_cast<uint32_t>(i * kEpiRows * 128), x0 + 64 * i, y0);
        if constexpr (E::kN32 > 0)
            if (x0 + 64 * E::kN64 < N)
                ptx::tma_store_2d(map32, s32, x0 + 64 * E::kN64, y0);
        if constexpr (E::kN16 > 0)
            if (x0 + 64 * E::kN64 + 32 * E::kN32 < N)
                ptx::tma_store_2d(map16, s16, x0 + 64 * E::kN64 + 32 * E::kN32, y0);
        ptx::bulk_commit_group();
    }
}

// Direct stores of one thread's row segment (columns [col0, col0 + NCOLS) of row `drow`).
template <int NCOLS>
__device__ __forceinline__ void store_row_direct(const float (&acc)[NCOLS], __nv_bfloat16 *drow,
                                                 int col0, int N)
{
#pragma unroll
    for (int j = 0; j < NCOLS / 8; ++j) {
        const int col = col0 + 8 * j;
        if (col < N) {
            ptx::st_global_v4(drow + col, ptx::pack_bf16x2(acc[8 * j], acc[8 * j + 1]),
                              ptx::pack_bf16x2(acc[8 * j + 2], acc[8 * j + 3]),
                              ptx::pack_bf16x2(acc[8 * j + 4], acc[8 * j + 5]),
                              ptx::pack_bf16x2(acc[8 * j + 6], acc[8 * j + 7]));
        }
    }
}

// Output of one tile by one promotion warp.  `valid` says whether this lane's row may be
// written and `out_row` is its row in the 2-D view of D.  The TMA path needs all 32 rows
// writable, except in the dense layout where the store clips rows >= M by itself.
template <int L, int NCOLS>
__device__ __forceinline__ void store_tile_rows(const float (&acc)[NCOLS], const Params &p,
                                                const CUtensorMap *tmap_d, uint32_t ring,
                                                int &ebuf, bool valid, size_t out_row, int col0,
                                                int lane)
{
    if (!__any_sync(0xffffffffu, valid))
        return;
    const bool whole = (L == kDense) || __all_sync(0xffffffffu, valid);
    if (whole) {
        const int y0 = __shfl_sync(0xffffffffu, static_cast<int>(out_row), 0);
        store_rows_tma<NCOLS>(acc, tmap_d, ring, ebuf, col0, y0, p.N, lane);
    } else if (valid) {
        store_row_direct<NCOLS>(acc, p.d + out_row * p.N, col0, p.N);
    }
}

// store_tile_rows with the whole-tile staging of the one-CTA kernel.
template <int L, int NCOLS>
__device__ __forceinline__ void store_tile_rows_whole(const float (&acc)[NCOLS], const Params &p,
                                                      const CUtensorMap *map64, const CUtensorMap *map32,
                                                      const CUtensorMap *map16, uint32_t s64,
                                                      uint32_t s32, uint32_t s16, bool valid,
                                                      size_t out_row, int col0, int lane)
{
    if (!__any_sync(0xffffffffu, valid))
        return;
    const bool whole = (L == kDense) || __all_sync(0xffffffffu, valid);
    if (whole) {
        const int y0 = __shfl_sync(0xffffffffu, static_cast<int>(out_row), 0);
        store_rows_whole<NCOLS>(acc, map64, map32, map16, s64, s32, s16, col0, y0, p.N, lane);
    } else if (valid) {
        store_row_direct<NCOLS>(acc, p.d + out_row * p.N, col0, p.N);
    }
}

template <int L, int BN>
__global__ void __launch_bounds__(kNumThreads, 1)
    dg_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_d64,
                   const __grid_constant__ CUtensorMap tmap_d32,
                   const __grid_constant__ CUtensorMap tmap_d16, const Params p)
{
    using C = Cfg<BN>;
    __shared__ SmemCtl ctl;
    extern __shared__ uint8_t smem_raw[];

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    // stage buffers start on a 1024-byte boundary (the 128-byte swizzle atom)
    const uint32_t smem_base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t *smem_gen = smem_raw + (smem_base - ptx::smem_addr(smem_raw));

    auto stage_a = [&](int s) { return smem_base + s * C::kStageBytes; };
    auto stage_b = [&](int s) { return smem_base + s * C::kStageBytes + C::kABytes; };
    const uint32_t bar_full = ptx::smem_addr(&ctl.full[0]);
    const uint32_t bar_empty = ptx::smem_addr(&ctl.empty[0]);
    const uint32_t bar_tfull = ptx::smem_addr(&ctl.tmem_full[0]);
    const uint32_t bar_tempty = ptx::smem_addr(&ctl.tmem_empty[0]);
    const uint32_t bar_drain = ptx::smem_addr(&ctl.drain);
    volatile int *abort_flag = &ctl.abort_flag;
    ptx::griddep_launch_dependents();  // the next grid may start its set-up as SMs free up

    // ---- set-up ------------------------------------------------------------------------
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
        ptx::prefetch_tmap(&tmap_d64);
        ptx::prefetch_tmap(&tmap_d32);
        ptx::prefetch_tmap(&tmap_d16);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(&ctl.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    // no global memory is touched before the grids this one depends on are complete
    ptx::griddep_wait();
    if (L == kMasked) {
        if (warp == 2 && lane == 0) {
            // prefix over groups of (m-tiles of the group) * n_tiles
            int acc = 0;
            for (int g = 0; g < p.G; ++g) {
                ctl.tile_prefix[g] = acc;
                int mm = __ldg(p.masked_m + g);
                if (mm < 0 || mm > p.M) {
                    if (blockIdx.x == 0)
                        record_error(p.err, kErrLayout);
                    mm = mm < 0 ? 0 : p.M;
                }
                acc += (mm + kBlockM - 1) / kBlockM * p.n_tiles;
            }
            ctl.tile_prefix[p.G] = acc;
            ctl.total_tiles = acc;
        }
    } else if (threadIdx.x == 0) {
        ctl.total_tiles = p.num_tiles;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl.tmem_base;
    const int num_tiles = ctl.total_tiles;

    if (warp < kFirstMathWarp) {
        ptx::setmaxnreg_dec<40>();
        if (warp == 0) {
            // ---------------- TMA producer (whole warp; one elected lane issues) ----------------
            uint32_t n_op = 0;  // operand loads issued
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                Tile ti;
                if (!resolve_tile<L>(p, ctl, t, ti))
                    continue;
                const int n0 = ti.n0 * BN;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!__all_sync(0xffffffffu, wait_one(bar_empty + 8 * s, ph ^ 1, p, abort_flag))) {
                        ok = false;
                        break;
                    }
                    if (ptx::elect_one()) {
                        const uint32_t fb = bar_full + 8 * s;
                        ptx::mbar_arrive_expect_tx(fb, p.idesc_b ? C::kTxBytesFp4B : C::kTxBytes);
                        ptx::tma_load_3d(stage_a(s), &tmap_a, fb, kb * kBlockK, ti.m0, ti.a_z);
                        ptx::tma_load_3d(stage_b(s), &tmap_b, fb, kb * kBlockK, n0, ti.g);
                    }
                    __syncwarp();
                    ++n_op;
                    if (++s == p.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // Wind down: every issued load must have landed before the CTA may exit.  Only the
            // last (ring size) loads can still be in flight; waiting on a slot's most recent
            // phase returns at once if it was already consumed.
            {
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
            }
            __syncwarp();
        } else if (warp == 1) {
            // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
            int s = 0;
            uint32_t ph = 0;
            int buf = 0;
            uint32_t bph = 0;
            bool ok = !p.inject_stall ||
                      __all_sync(0xffffffffu, wait_one(ptx::smem_addr(&ctl.stall), 0, p, abort_flag));
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                Tile ti;
                if (!resolve_tile<L>(p, ctl, t, ti))
                    continue;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    bool w = wait_one(bar_tempty + 8 * buf, bph ^ 1, p, abort_flag) &&
                             wait_one(bar_full + 8 * s, ph, p, abort_flag);
                    if (!__all_sync(0xffffffffu, w)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    if (ptx::elect_one()) {
                        const uint64_t adesc = ptx::sdesc_kmajor_sw128(stage_a(s));
                        const uint64_t bdesc = ptx::sdesc_kmajor_sw128(stage_b(s));
                        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
                        for (int k = 0; k < kBlockK / kUmmaK; ++k) {
                            // advance the start address by 32 bytes (2 x 16 B) per K step
                            ptx::mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::kIdesc | p.idesc_b,
                                            k > 0 ? 1u : 0u);
                        }
                        ptx::mma_commit(bar_empty + 8 * s);
                        ptx::mma_commit(bar_tfull + 8 * buf);
                    }
                    __syncwarp();
                    if (++s == p.stages) {
                        s = 0;
                        ph ^= 1;
                    }
                    if (++buf == C::kTmemBufs) {
                        buf = 0;
                        bph ^= 1;
                    }
                }
            }
            // Wind down: all issued MMAs complete before tensor memory is released.
            if (ptx::elect_one())
                ptx::mma_commit(bar_drain);
            __syncwarp();
            wait_drain(bar_drain, 0);
            __syncwarp();
        }
    } else {
        ptx::setmaxnreg_inc<232>();
        // ---------------- promotion + epilogue ----------------
        const int mw = warp - kFirstMathWarp;     // 0..7
        const int half = mw / 4;                  // which half of the BN columns
        const int q = warp % 4;                   // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;            // row within the tile
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(half * C::kCols);
        constexpr int P1 = C::kPart1;             // columns loaded before the first wait
        constexpr int P2 = C::kCols - P1;         // columns loaded after it (0 if all at once)
        // this warp's output staging pieces (64-, 32- and 16-column), after the operand stages
        using EP = EpiPieces<C::kCols>;
        const uint32_t epi0 = smem_base + static_cast<uint32_t>(p.stages * C::kStageBytes);
        const uint32_t s64 = epi0 + static_cast<uint32_t>(mw * EP::kWarp64);
        const uint32_t s32 = epi0 + static_cast<uint32_t>(kNumMathWarps * EP::kWarp64 + mw * EP::kWarp32);
        const uint32_t s16 = epi0 + static_cast<uint32_t>(kNumMathWarps * (EP::kWarp64 + EP::kWarp32) +
                                                          mw * EP::kWarp16);
        int buf = 0;
        uint32_t bph = 0;
        bool ok = true;
        // Everything a thread needs to start a tile, including the scales of its first two K
        // blocks: prepared for the next tile before the current tile's epilogue, so that those
        // global loads land while the epilogue runs instead of stalling the first promotion.
        struct TileCtx {
            Tile ti;
            int col0, split;
            const float *sfb_lo, *sfb_hi, *sa_ptr;
            KbScales s0, s1;
        };
        auto prepare = [&](int t, TileCtx &c) -> bool {
            if (!resolve_tile<L>(p, ctl, t, c.ti))
                return false;
            c.col0 = c.ti.n0 * BN + half * C::kCols;  // first global column of this thread
            // the (at most two) 128-column scale blocks of B this thread's columns touch; the
            // boundary (if any) lies on a 16-column group edge
            const int nb_lo = min(c.col0 / kBlockK, p.num_nb - 1);
            const int nb_hi = min((c.col0 + C::kCols - 1) / kBlockK, p.num_nb - 1);
            c.split = min(C::kCols, max(0, (nb_lo + 1) * kBlockK - c.col0));  // first hi column
            c.sfb_lo = p.sfb + (static_cast<size_t>(c.ti.g) * p.num_nb + nb_lo) * p.num_kb;
            c.sfb_hi = p.sfb + (static_cast<size_t>(c.ti.g) * p.num_nb + nb_hi) * p.num_kb;
            // this thread's A scales: one per K block, num_kb rows of sfa_ld apart (rows past
            // the scale matrix read its last row; they are not stored)
            c.sa_ptr = p.sfa + static_cast<size_t>(c.ti.a_z) * p.num_kb * p.sfa_ld +
                       min(c.ti.m0 + row, p.sfa_ld - 1);
            load_kb_scales(c.s0, c.sa_ptr, c.sfb_lo, c.sfb_hi, p.sfa_ld, 0, p.num_kb);
            load_kb_scales(c.s1, c.sa_ptr, c.sfb_lo, c.sfb_hi, p.sfa_ld, 1, p.num_kb);
            return true;
        };
        int t = blockIdx.x;
        TileCtx cur;
        while (t < num_tiles && !prepare(t, cur))
            t += gridDim.x;
        while (t < num_tiles && ok) {
            const Tile ti = cur.ti;
            const int col0 = cur.col0;
            float acc[C::kCols];
#pragma unroll
            for (int c = 0; c < C::kCols; ++c)
                acc[c] = 0.0f;

            ok = promote_tile<BN, P1, P2, C::kCols, C::kTmemBufs>(
                acc, cur.s0, cur.s1, cur.sa_ptr, cur.sfb_lo, cur.sfb_hi, lane_base, bar_tfull, buf,
                bph,
                [&](int b, uint32_t &rel, bool &remote) {
                    rel = bar_tempty + 8 * b;
                    remote = false;
                },
                cur.split, lane, p, abort_flag);
            if (!ok)
                break;
            // the next tile of this CTA, its scales in flight during this epilogue
            int tn = t + static_cast<int>(gridDim.x);
            while (tn < num_tiles && !prepare(tn, cur))
                tn += gridDim.x;
            t = tn;

            // ---- epilogue: bf16 rounding, TMA stores of whole warps, direct stores otherwise ----
            const int grow = ti.m0 + row;  // row within the group
            bool valid;
            size_t out_row;
            if (L == kDense) {
                valid = grow < p.M;
                out_row = static_cast<size_t>(grow);
            } else if (L == kContiguous) {
                valid = false;
                if (grow < p.M) {
                    const int gi = __ldg(p.m_indices + grow);
                    valid = gi == ti.g;
                    if ((gi >= 0 && gi != ti.g) || gi < -1)
                        record_error(p.err, kErrLayout);
                }
                out_row = static_cast<size_t>(grow);
            } else {
                int mm = __ldg(p.masked_m + ti.g);
                mm = mm < 0 ? 0 : (mm > p.M ? p.M : mm);
                valid = grow < mm;
                out_row = static_cast<size_t>(ti.g) * p.M + grow;
            }
            store_tile_rows_whole<L, C::kCols>(acc, p, &tmap_d64, &tmap_d32, &tmap_d16, s64, s32, s16,
                                               valid, out_row, col0, lane);
        }
        // every staged output box is written (and its shared memory read) before exit
        if (lane == 0)
            ptx::bulk_wait_group_all();
        __syncwarp();
    }

    // ---- tear-down: everyone is past its last tcgen05 operation ----------------------------
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace dg
