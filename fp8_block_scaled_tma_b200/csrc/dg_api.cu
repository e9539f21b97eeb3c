// dg_api.cu -- host side of the C ABI declared in include/dg.h: argument checks, tile choice,
// TMA tensor maps, and the launch of the sm_100a kernel on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/dg.h"
#include "dg_kernel.cuh"
#include "dg_map_cache.h"
#include "dg_pair_kernel.cuh"
#include "dg_quant_kernel.cuh"
#include "dg_splitk_kernel.cuh"
#include "dg_swap_kernel.cuh"
#include "dg_swap_sk_kernel.cuh"

namespace {

using dg::Params;

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;
constexpr int kMinDynSmem = 120 * 1024;  // keeps one CTA per SM (each takes all 512 TMEM columns)

__device__ int g_device_error;  // the device error word read by dg_poll_device_error
__device__ int g_polled_error;  // the value dg_poll_device_error last took from it

// Takes the error word and resets it in one atomic step, so that no error recorded by a
// kernel running on another stream can fall between the read and the reset.
__global__ void dg_take_error_kernel()
{
    g_polled_error = atomicExch(&g_device_error, 0);
}

struct DeviceInfo {
    bool init = false;
    int status = DG_OK;
    int num_sms = 0;
    int smem_optin = 0;
    int *err_ptr = nullptr;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
struct KernelSmem {
    int static_bytes = -1;  // static shared memory of the kernel
    int limit_set = 0;      // dynamic shared-memory limit already set on this device
};
KernelSmem g_smem[kMaxDevices][3][8];       // 1-CTA kernels, per device / layout / BN
KernelSmem g_smem_pair[kMaxDevices][3][8];  // CTA-pair kernels
KernelSmem g_smem_split[kMaxDevices][8];    // split-K kernels, per BN
KernelSmem g_smem_swap[kMaxDevices][6];     // swapped-operand kernels, per (TN, R)
KernelSmem g_smem_swap_sk[kMaxDevices][2];  // stream-K swapped-operand kernels, per TN (32, 64)
// 0 auto, 1 one-CTA kernels, 2 CTA pairs where possible, 3 split-K (dense), 4 swapped operands
// (dense, M <= 128), 5 stream-K swapped operands (dense, M <= 64, needs the caller's workspace)
int g_family = 0;
int g_num_sms_cap = 0;
unsigned long long g_timeout_ns = kDefaultTimeoutNs;
int g_override_bn = 0;
int g_override_stages = 0;
int g_override_splits = 0;
int g_inject_stall = 0;
int g_pdl = 1;  // launch with programmatic stream serialisation (dg_set_pdl)
// clusters of each size (index = cluster size, 1..8) that can be resident at once, per device
// and kernel family; 0 = not queried yet
int g_max_clusters[kMaxDevices][9][9];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
dg::TensorMapCache g_map_cache;  // encoded tensor maps, keyed on every encode argument

struct LastLaunch {
    bool valid = false;
    int block_n = 0, stages = 0, grid = 0, tiles = 0, pair = 0, splits = 1, family = 1;
};
thread_local LastLaunch t_last;

bool debug_enabled()
{
    static int v = -1;
    if (v < 0) {
        const char *e = std::getenv("DG_DEBUG");
        v = (e && e[0] && e[0] != '0') ? 1 : 0;
    }
    return v == 1;
}

// Appends the programmatic-dependent-launch attribute when it is enabled: the kernel may then
// be scheduled while the previous kernel of the stream finishes; every kernel waits for it
// (griddepcontrol.wait) before touching global memory, so stream order is kept.
int add_pdl_attr(cudaLaunchAttribute *attr, int n)
{
    int on;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        on = g_pdl;
    }
    if (!on)
        return n;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    return n + 1;
}

// Per-device set-up: checks for sm_100, reads SM count and shared-memory limit, and resolves
// the address of the device error word.  Called with the device current.
int device_setup(int &dev_out, DeviceInfo *&info)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return DG_ERR_UNSUPPORTED;
    }
    if (dev < 0 || dev >= kMaxDevices)
        return DG_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_dev[dev];
    if (!d.init) {
        d.init = true;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            d.status = DG_ERR_UNSUPPORTED;
        } else if (major != 10 || minor != 0) {
            d.status = DG_ERR_UNSUPPORTED;
        } else {
            cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) {
                cudaGetLastError();
                d.status = DG_ERR_CUDA;
            } else {
                d.err_ptr = static_cast<int *>(p);
                d.status = DG_OK;
            }
        }
        if (d.status == DG_OK && g_encode == nullptr) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr) {
                cudaGetLastError();
                d.status = DG_ERR_CUDA;
            } else {
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
        }
    }
    dev_out = dev;
    info = &d;
    return d.status;
}

int inject_stall_flag()
{
    std::lock_guard<std::mutex> lock(g_mutex);
    return g_inject_stall;
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

int align4(int x)
{
    return (x + 3) / 4 * 4;
}

// cuTensorMapEncodeTiled through the cache of encoded maps (a hit is byte-identical to what the
// driver would encode for the same arguments).
CUresult encode_tiled(CUtensorMap *map, CUtensorMapDataType dt, cuuint32_t rank, void *base,
                      const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                      const cuuint32_t *estr, CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                      CUtensorMapL2promotion l2, CUtensorMapFloatOOBfill oob)
{
    dg::TensorMapKey key;
    dg::make_map_key(key, dt, rank, base, dims, strides, box, estr, il, sw, l2, oob);
    return g_map_cache.get(key, map, [&](CUtensorMap *out) {
        return g_encode(out, dt, rank, base, dims, strides, box, estr, il, sw, l2, oob);
    });
}

// 3-D tiled tensor map: dims/strides innermost first (strides in bytes for dims 1, 2).
int make_map(CUtensorMap *map, CUtensorMapDataType dt, void *base, uint64_t d0, uint64_t d1,
             uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1,
             CUtensorMapSwizzle swz)
{
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode_tiled(map, dt, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// 2-D view [rows][N] of the bf16 output for the TMA-store epilogues: one box is 32 rows x
// `box_cols` columns (16, 32 or 64), swizzled with the box's row width (32, 64 or 128 bytes) as
// the kernels' staging boxes are.
int make_map_d(CUtensorMap *map, void *base, uint64_t N, uint64_t rows, int box_cols = dg::kEpiCols)
{
    cuuint64_t dims[2] = {N, rows};
    cuuint64_t strides[1] = {N * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(dg::kEpiRows)};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = box_cols == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : box_cols == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

int stage_bytes_rt(int bn)
{
    return dg::kBlockM * dg::kBlockK + bn * dg::kBlockK;  // A tile + B tile (multiple of 1024)
}



// 4-D view [groups][K/128][rows][128 elements] of a K-major operand: one box holds `kbs`
// consecutive 128-wide K blocks of `box_rows` rows, laid out K block by K block in shared memory,
// 128 bytes per row and K block.  fp4: the operand is packed E2M1 (K/2 bytes per row), which
// TMA expands into the padded layout tcgen05 kind::f8f6f4 reads (16 values in 8 bytes, then
// 8 bytes of gap), so shared memory holds the same 128 bytes per row and K block as e4m3.
int make_map_kblocks(CUtensorMap *map, void *base, uint64_t K, uint64_t rows, uint64_t groups,
                     uint32_t box_rows, uint32_t kbs, bool fp4 = false)
{
    const uint64_t row_bytes = fp4 ? K / 2 : K;
    cuuint64_t dims[4] = {128, rows, K / 128, groups};
    cuuint64_t strides[3] = {row_bytes, fp4 ? 64u : 128u, row_bytes * rows};
    cuuint32_t box[4] = {128, box_rows, kbs, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode_tiled(map, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                          4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

template <int L, int BN>
void *pair_kernel_ptr()
{
    return reinterpret_cast<void *>(&dg::dg_gemm_pair_kernel<L, BN>);
}

void *pick_pair_kernel(int layout, int bn)
{
#define DG_PCASE(BNV)                                                                          \
    case BNV:                                                                                  \
        return layout == dg::kDense ? pair_kernel_ptr<dg::kDense, BNV>()                        \
                                    : pair_kernel_ptr<dg::kMasked, BNV>();
    if (layout == dg::kContiguous)
        return nullptr;
    switch (bn) {
        DG_PCASE(128)
        DG_PCASE(160)
        DG_PCASE(192)
        DG_PCASE(224)
        DG_PCASE(256)
    default:
        return nullptr;
    }
#undef DG_PCASE
}

int pair_stage_bytes(int bn)
{
    return dg::kKbPerStage * (dg::kBlockM * dg::kBlockK + bn / 2 * dg::kBlockK);
}

constexpr int kPairSfaRingBytes = dg::kSfaSlots * dg::kKbPerStage * dg::kBlockM * 4;

// Tile heuristic of the pair kernel: 256-row pair tiles, waves over SM pairs.
// Time model shared by the tile choosers.  A persistent CTA (or CTA pair) walks its tiles one
// after another, so the time is (tiles per CTA, rounded up) x (time of one tile).  Measured on
// B200 (dense 4096-row shapes, BN from 160 to 256, both kernel families), one K block of one
// tile costs about kTileFixed + BN column-units: a fixed part (the MMA-commit -> promotion ->
// buffer-release round trip, ~600-750 cycles) plus ~1.5-2 cycles per column (MMA, tensor-memory
// reads and FFMA promotion); the CTA-pair kernel is nearly flat in BN.  So whole waves decide,
// and among equal wave counts the narrower tile wins.  Columns computed past N are wasted work.
// (An earlier fit with a fixed part of 190 units picked BN = 224 for 8192 x 7168 x 18432, 14
// waves of pair tiles, where BN = 256 runs 13 waves and measured 3 % faster.)
constexpr double kTileFixed = 400.0;
// Dense problems use CTA pairs only for long K: measured on B200, the pair kernel is ahead by a
// few percent at K = 16384 and level with or behind the one-CTA kernel at K <= 7168, where its
// longer per-tile start-up weighs more.
constexpr int kPairMinKBlocks = 96;

double tile_time(long long row_tiles, int N, int bn, int slots)
{
    const long long n_tiles = (N + bn - 1) / bn;
    const long long tiles = n_tiles * row_tiles;
    const long long waves = (tiles + slots - 1) / slots;
    return static_cast<double>(waves) * (kTileFixed + bn);
}

int choose_pair_block_n(long long pair_row_tiles, int N, int num_pairs)
{
    int best_bn = 256;
    double best = 1e300;
    for (int bn = 128; bn <= 256; bn += 32) {
        const double t = tile_time(pair_row_tiles, N, bn, num_pairs);
        if (t < best - 1e-9 || (std::abs(t - best) <= 1e-9 && bn > best_bn)) {
            best = t;
            best_bn = bn;
        }
    }
    return best_bn;
}

template <int BN>
void *splitk_kernel_ptr()
{
    return reinterpret_cast<void *>(&dg::dg_gemm_splitk_kernel<BN>);
}

void *pick_splitk_kernel(int bn)
{
    switch (bn) {
    case 64: return splitk_kernel_ptr<64>();
    case 96: return splitk_kernel_ptr<96>();
    case 128: return splitk_kernel_ptr<128>();
    case 160: return splitk_kernel_ptr<160>();
    case 192: return splitk_kernel_ptr<192>();
    case 224: return splitk_kernel_ptr<224>();
    case 256: return splitk_kernel_ptr<256>();
    default: return nullptr;
    }
}

// Largest number of clusters of `csize` CTAs (one CTA per SM, `dyn_smem` bytes each) that can be
// resident at once: clusters live inside one GPC, so this can be below sms / csize.
int max_active_clusters(void *fn, int csize, int dyn_smem, int dev, int family_slot)
{
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        int v = g_max_clusters[dev][family_slot][csize];
        if (v > 0)
            return v;
    }
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(csize, 1, 1);
    cfg.blockDim = dim3(dg::kNumThreads, 1, 1);
    cfg.dynamicSmemBytes = dyn_smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    g_max_clusters[dev][family_slot][csize] = n;
    return n;
}

// Split-K choice for dense problems with few output tiles: BN and the number of K splits S
// (cluster size) minimising a simple time model -- the larger of the per-CTA TMA time (bytes
// the CTA copies at ~100 GB/s), the whole problem's HBM time and the per-CTA MMA issue time --
// plus a fixed launch/prologue cost and the cross-CTA reduction.  Returns false if no
// configuration fits in one wave of CTAs.
template <class Capacity>
bool choose_splitk(int M, int N, int K, int sms, int bn_fixed, int s_fixed, Capacity capacity,
                   int &bn_out, int &s_out)
{
    const int num_kb = K / dg::kBlockK;
    const int m_tiles = (M + dg::kBlockM - 1) / dg::kBlockM;
    double best = 1e300;
    bool found = false;
    // BN below 128 is searched only when forced: the fitted model below covers 128..256
    for (int bn = 256; bn >= (bn_fixed != 0 ? 64 : 128); bn -= 32) {
        if (bn_fixed != 0 && bn != bn_fixed)
            continue;
        const long long tiles = static_cast<long long>(m_tiles) * ((N + bn - 1) / bn);
        if (tiles > sms)
            continue;
        const int s_max = static_cast<int>(std::min<long long>(std::min(dg::kMaxSplits, num_kb), sms / tiles));
        for (int S = 1; S <= s_max; ++S) {
            if (s_fixed != 0 && S != s_fixed)
                continue;
            // every cluster of the grid must be resident at once (one wave)
            if (tiles > capacity(bn, S))
                continue;
            // Time model (ns), least-squares fitted to B200 timings of every (BN, S) on ten
            // memory-bound shapes (M = 64 / 128): a CTA walks its K blocks at ~(537 + 2.85 BN)
            // cycles each (the TMEM buffer round trip of the two-level accumulation), all CTAs
            // together cannot beat HBM, and with S > 1 the cluster barriers and the reduction
            // through distributed shared memory cost ~0.26 us per split plus ~0.14 ns per
            // partial element of a slice.  (A fixed per-launch cost does not change the choice.)
            const int kb_per = (num_kb + S - 1) / S;
            const double t_kb = kb_per * (537.0 + 2.85 * bn) / 1.9;
            const double t_hbm = (static_cast<double>(N) * K + static_cast<double>(M) * K) / 6500.0;
            const double t_red = S > 1 ? 263.0 * S + 0.139 * bn * std::min(M, dg::kBlockM) : 0.0;
            const double t = std::max(t_kb, t_hbm) + t_red;
            if (t < best - 1e-9) {
                best = t;
                bn_out = bn;
                s_out = S;
                found = true;
            }
        }
    }
    return found;
}

template <int L, int BN>
void *kernel_ptr()
{
    return reinterpret_cast<void *>(&dg::dg_gemm_kernel<L, BN>);
}

void *pick_kernel(int layout, int bn)
{
#define DG_CASE(BNV)                                                                           \
    case BNV:                                                                                  \
        return layout == dg::kDense        ? kernel_ptr<dg::kDense, BNV>()                       \
               : layout == dg::kContiguous ? kernel_ptr<dg::kContiguous, BNV>()                  \
                                           : kernel_ptr<dg::kMasked, BNV>();
    switch (bn) {
        DG_CASE(32)
        DG_CASE(64)
        DG_CASE(96)
        DG_CASE(128)
        DG_CASE(160)
        DG_CASE(192)
        DG_CASE(224)
        DG_CASE(256)
    default:
        return nullptr;
    }
#undef DG_CASE
}

// Tile heuristic: among BN in {32..256} pick the one with the smallest estimated time, where a
// tile of BN columns costs max(MMA time ~ BN, load time ~ 128 + BN) and tiles run in waves over
// the SMs (non-power-of-two BN exists to even out the last wave).
int choose_block_n(int rows_tiles, int N, int num_sms)
{
    int best_bn = 256;
    double best = 1e300;
    for (int bn = 32; bn <= 256; bn += 32) {
        const double t = tile_time(rows_tiles, N, bn, num_sms);
        if (t < best - 1e-9 || (std::abs(t - best) <= 1e-9 && bn > best_bn)) {
            best = t;
            best_bn = bn;
        }
    }
    return best_bn;
}

struct LaunchArgs {
    int layout;
    const void *a;
    const float *sfa;
    const void *b;
    const float *sfb;
    void *d;
    const int *m_indices;
    const int *masked_m;
    int M;  // dense M / M_total / M_max
    int N, K, G;
    int expected_m;
    void *stream;
    int b_fp4 = 0;  // B holds packed E2M1 (two per byte) instead of E4M3 codes
    void *ws = nullptr;      // caller's workspace (dense calls; may be null)
    size_t ws_bytes = 0;
};

int launch_splitk(const LaunchArgs &args, int dev, DeviceInfo *info, int bn, int S,
                  int stages_override, unsigned long long timeout)
{
    const int M = args.M, N = args.N, K = args.K;
    const int num_kb = K / dg::kBlockK;
    const int num_nb = (N + dg::kBlockK - 1) / dg::kBlockK;
    const int m_tiles = (M + dg::kBlockM - 1) / dg::kBlockM;
    const int n_tiles = (N + bn - 1) / bn;
    void *fn = pick_splitk_kernel(bn);
    if (fn == nullptr)
        return DG_ERR_INVALID_ARG;
    const int sbytes = dg::kSplitKbPerStage * (dg::kBlockM * dg::kBlockK + bn * dg::kBlockK);
    const int part_bytes = dg::kBlockM * (bn + 4) * 4;
    int stages = 0, dyn_smem = 0;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        KernelSmem &ks = g_smem_split[dev][bn / 32 - 1];
        if (ks.static_bytes < 0) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, fn);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.static_bytes = static_cast<int>(fa.sharedSizeBytes);
        }
        const int dyn_cap = info->smem_optin - ks.static_bytes;
        stages = std::min(dg::kMaxStages, (dyn_cap - 1024) / sbytes);
        if (stages_override > 0)
            stages = std::min(stages, stages_override);
        if (stages < 2 || part_bytes + 1024 > dyn_cap)
            return DG_ERR_UNSUPPORTED;
        // the pipeline buffers, reused for the fp32 partial tile after the K loop
        dyn_smem = std::max(stages * sbytes, part_bytes) + 1024;
        dyn_smem = std::min(std::max(dyn_smem, kMinDynSmem), dyn_cap);
        if (ks.limit_set < dyn_smem) {
            cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.limit_set = dyn_smem;
        }
    }
    CUtensorMap map_a, map_b;
    if (make_map_kblocks(&map_a, const_cast<void *>(args.a), K, M, 1, dg::kBlockM,
                         dg::kSplitKbPerStage) != DG_OK ||
        make_map_kblocks(&map_b, const_cast<void *>(args.b), K, N, 1, bn, dg::kSplitKbPerStage,
                         args.b_fp4 != 0) != DG_OK) {
        if (debug_enabled())
            std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled failed (split-K)\n");
        return DG_ERR_CUDA;
    }
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.num_kb = num_kb;
    p.num_nb = num_nb;
    p.m_tiles = m_tiles;
    p.n_tiles = n_tiles;
    p.stages = stages;
    p.raster_m = S;
    p.sfa = args.sfa;
    p.sfa_ld = align4(M);
    p.sfb = args.sfb;
    p.d = static_cast<__nv_bfloat16 *>(args.d);
    p.err = info->err_ptr;
    p.timeout_ns = timeout;
    p.inject_stall = inject_stall_flag();
    p.idesc_b = args.b_fp4 ? dg::ptx::kIdescBFormatE2M1 : 0u;
    p.num_tiles = m_tiles * n_tiles;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(p.num_tiles * S, 1, 1);
    cfg.blockDim = dim3(dg::kNumThreads, 1, 1);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = static_cast<cudaStream_t>(args.stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 1);
    void *kargs[] = {&map_a, &map_b, &p};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, kargs);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] split-K launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    t_last.valid = true;
    t_last.block_n = bn;
    t_last.stages = stages;
    t_last.grid = p.num_tiles * S;
    t_last.tiles = p.num_tiles;
    t_last.pair = 0;
    t_last.splits = S;
    t_last.family = 3;
    if (debug_enabled())
        std::fprintf(stderr, "[dg] split-K M=%d N=%d K=%d BN=%d S=%d stages=%d grid=%d smem=%d\n", M, N,
                     K, bn, S, stages, p.num_tiles * S, dyn_smem);
    return DG_OK;
}

int launch_pair(const LaunchArgs &args, int dev, DeviceInfo *info, int sms, int bn,
                int stages_override, unsigned long long timeout)
{
    const int M = args.M, N = args.N, K = args.K, G = args.G;
    const int num_kb = K / dg::kBlockK;
    const int num_nb = (N + dg::kBlockK - 1) / dg::kBlockK;
    const int pair_m_tiles = (M + 2 * dg::kBlockM - 1) / (2 * dg::kBlockM);
    const int num_pairs = sms / 2;
    if (bn == 0) {
        long long row_tiles = pair_m_tiles;
        if (args.layout == dg::kMasked) {
            int em = args.expected_m > 0 ? std::min(args.expected_m, M) : M;
            row_tiles = static_cast<long long>(G) * ((em + 2 * dg::kBlockM - 1) / (2 * dg::kBlockM));
        }
        bn = choose_pair_block_n(std::max<long long>(1, row_tiles), N, num_pairs);
    }
    void *fn = pick_pair_kernel(args.layout, bn);
    if (fn == nullptr)
        return DG_ERR_INVALID_ARG;
    const int n_tiles = (N + bn - 1) / bn;
    const int sbytes = pair_stage_bytes(bn);
    int stages = 0, dyn_smem = 0;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        KernelSmem &ks = g_smem_pair[dev][args.layout][bn / 32 - 1];
        if (ks.static_bytes < 0) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, fn);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.static_bytes = static_cast<int>(fa.sharedSizeBytes);
        }
        const int dyn_cap = info->smem_optin - ks.static_bytes;
        stages = std::min(dg::kMaxStages, (dyn_cap - 1024 - kPairSfaRingBytes - dg::kEpiBytes) / sbytes);
        if (stages_override > 0)
            stages = std::min(stages, stages_override);
        if (stages < 2)
            return DG_ERR_UNSUPPORTED;
        // operand stages, the A-scale ring, the output staging boxes, and slack to align the
        // stages to 1024 bytes
        dyn_smem = stages * sbytes + kPairSfaRingBytes + dg::kEpiBytes + 1024;
        dyn_smem = std::min(std::max(dyn_smem, kMinDynSmem), dyn_cap);
        if (ks.limit_set < dyn_smem) {
            cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.limit_set = dyn_smem;
        }
    }

    const int a_groups = (args.layout == dg::kMasked) ? G : 1;
    const int b_groups = (args.layout == dg::kDense) ? 1 : G;
    const int m4 = align4(M);
    CUtensorMap map_a, map_b, map_sfa, map_d;
    if (make_map_d(&map_d, args.d, N, static_cast<uint64_t>(M) * a_groups) != DG_OK ||
        make_map_kblocks(&map_a, const_cast<void *>(args.a), K, M, a_groups, dg::kBlockM,
                         dg::kKbPerStage) != DG_OK ||
        make_map_kblocks(&map_b, const_cast<void *>(args.b), K, N, b_groups, bn / 2,
                         dg::kKbPerStage, args.b_fp4 != 0) != DG_OK ||
        // A scales [groups][K/128][align4(rows)]: one box = 128 rows x kKbPerStage K blocks
        make_map(&map_sfa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float *>(args.sfa), m4,
                 num_kb, a_groups, static_cast<uint64_t>(m4) * 4,
                 static_cast<uint64_t>(m4) * 4 * num_kb, dg::kBlockM, dg::kKbPerStage,
                 CU_TENSOR_MAP_SWIZZLE_NONE) != DG_OK) {
        if (debug_enabled())
            std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled failed (pair)\n");
        return DG_ERR_CUDA;
    }

    Params p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = (args.layout == dg::kDense) ? 1 : G;
    p.num_kb = num_kb;
    p.num_nb = num_nb;
    p.m_tiles = pair_m_tiles;
    p.n_tiles = n_tiles;
    p.stages = stages;
    p.raster_m = 8;
    p.sfa = args.sfa;
    p.sfa_ld = m4;
    p.sfb = args.sfb;
    p.d = static_cast<__nv_bfloat16 *>(args.d);
    p.m_indices = nullptr;
    p.masked_m = args.masked_m;
    p.err = info->err_ptr;
    p.timeout_ns = timeout;
    p.inject_stall = inject_stall_flag();
    p.idesc_b = args.b_fp4 ? dg::ptx::kIdescBFormatE2M1 : 0u;
    long long tiles = (args.layout == dg::kMasked)
                          ? static_cast<long long>(G) * pair_m_tiles * n_tiles
                          : static_cast<long long>(pair_m_tiles) * n_tiles;
    if (tiles > 0x7FFFFFFFLL)
        return DG_ERR_INVALID_ARG;
    p.num_tiles = static_cast<int>(tiles);
    int resident = max_active_clusters(fn, 2, dyn_smem, dev, args.layout == dg::kDense ? 0 : 1);
    if (resident <= 0 || resident > num_pairs)
        resident = num_pairs;
    const int pairs = static_cast<int>(std::min<long long>(resident, tiles));
    if (pairs <= 0)
        return DG_OK;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(dg::kNumThreads, 1, 1);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = static_cast<cudaStream_t>(args.stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 1);
    void *kargs[] = {&map_a, &map_b, &map_sfa, &map_d, &p};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, kargs);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] pair launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    t_last.valid = true;
    t_last.block_n = bn;
    t_last.stages = stages;
    t_last.grid = 2 * pairs;
    t_last.tiles = p.num_tiles;
    t_last.pair = 1;
    t_last.splits = 1;
    t_last.family = 2;
    if (debug_enabled())
        std::fprintf(stderr, "[dg] pair layout=%d M=%d N=%d K=%d G=%d BN=%d stages=%d grid=%d tiles=%d smem=%d\n",
                     args.layout, M, N, K, G, bn, stages, 2 * pairs, p.num_tiles, dyn_smem);
    return DG_OK;
}

// ---- swapped-operand kernel (dense, M <= 128) ------------------------------------------------

int swap_index(int tn, int R)
{
    const int t = tn == 32 ? 0 : tn == 64 ? 1 : tn == 128 ? 2 : -1;
    return (t < 0 || (R != 1 && R != 2)) ? -1 : t * 2 + (R - 1);
}

template <int TN, int R>
void *swap_kernel_ptr()
{
    return reinterpret_cast<void *>(&dg::dg_gemm_swap_kernel<TN, R>);
}

void *pick_swap_kernel(int tn, int R)
{
    switch (swap_index(tn, R)) {
    case 0: return swap_kernel_ptr<32, 1>();
    case 1: return swap_kernel_ptr<32, 2>();
    case 2: return swap_kernel_ptr<64, 1>();
    case 3: return swap_kernel_ptr<64, 2>();
    case 4: return swap_kernel_ptr<128, 1>();
    case 5: return swap_kernel_ptr<128, 2>();
    default: return nullptr;
    }
}

int swap_token_tile(int M)
{
    return M <= 32 ? 32 : M <= 64 ? 64 : 128;
}

int swap_stage_bytes(int tn, int R)
{
    return dg::kSwapKbPerStage * (R * dg::kBlockM * dg::kBlockK + tn * dg::kBlockK);
}

int swap_scale_bytes(int tn, int R, int kb_box)
{
    return kb_box * tn * 4 * (R == 1 ? 1 : 3);
}

// Choice of R (128-row blocks of B per tile) and S (K splits = cluster size) for the
// swapped-operand kernel.  Time model: the problem cannot beat HBM, a CTA cannot pull more
// than ~80 GB/s through its TMA pipeline, and with S > 1 the cluster barriers and the
// reduction through distributed shared memory cost ~0.26 us per split plus ~0.14 ns per partial
// element (the split-K kernel's fitted constants).  Returns false if nothing fits in one wave.
template <class Capacity>
bool choose_swap(int M, int N, int K, bool fp4, int sms, int dyn_cap, int r_fixed, int s_fixed,
                 Capacity capacity, int &r_out, int &s_out)
{
    const int num_kb = K / dg::kBlockK;
    const int nblocks = (N + dg::kBlockM - 1) / dg::kBlockM;
    const int tn = swap_token_tile(M);
    const double b_bytes = static_cast<double>(N) * K * (fp4 ? 0.5 : 1.0);
    const double t_hbm = (b_bytes + static_cast<double>(M) * K) / 6500.0;  // ns
    double best = 1e300;
    bool found = false;
    for (int R = 1; R <= 2; ++R) {
        if (r_fixed != 0 && R != r_fixed)
            continue;
        const long long tiles = (nblocks + R - 1) / R;
        for (int S = 1; S <= dg::kMaxSplits; ++S) {
            if (s_fixed != 0 && S != s_fixed)
                continue;
            if (S > num_kb)
                continue;
            const int kb_box = (num_kb + S - 1) / S;
            if (kb_box > 256 || swap_scale_bytes(tn, R, kb_box) > dg::kSwapMaxScaleBytes)
                continue;
            // at least two operand stages, which also hold the fp32 partial after the K loop
            const int sbytes = swap_stage_bytes(tn, R);
            const int stages = std::min(dg::kMaxStages, (dyn_cap - 1024 - swap_scale_bytes(tn, R, kb_box)) / sbytes);
            if (stages < 2 || stages * sbytes < tn * R * dg::kBlockM * 4)
                continue;
            if (tiles * S > sms || tiles > capacity(tn, R, S))
                continue;
            const double kb_bytes = R * dg::kBlockM * dg::kBlockK * (fp4 ? 0.5 : 1.0) +
                                    static_cast<double>(tn) * dg::kBlockK;
            const double t_cta = kb_box * kb_bytes / 80.0;
            const double t_red = S > 1 ? 263.0 * S + 0.139 * std::min(M, tn) * R * dg::kBlockM : 0.0;
            const double t = std::max(t_hbm, t_cta) + t_red;
            if (t < best - 1e-9) {
                best = t;
                r_out = R;
                s_out = S;
                found = true;
            }
        }
    }
    return found;
}

int launch_swap(const LaunchArgs &args, int dev, DeviceInfo *info, int R, int S,
                int stages_override, unsigned long long timeout)
{
    const int M = args.M, N = args.N, K = args.K;
    const int num_kb = K / dg::kBlockK;
    const int num_nb = (N + dg::kBlockK - 1) / dg::kBlockK;
    const int tn = swap_token_tile(M);
    const int idx = swap_index(tn, R);
    void *fn = pick_swap_kernel(tn, R);
    if (fn == nullptr || M > 128 || S < 1 || S > dg::kMaxSplits || S > num_kb)
        return DG_ERR_INVALID_ARG;
    const int n_tiles = (N + R * dg::kBlockM - 1) / (R * dg::kBlockM);
    const int kb_box = (num_kb + S - 1) / S;
    const int sbytes = swap_stage_bytes(tn, R);
    const int scale_bytes = swap_scale_bytes(tn, R, kb_box);
    const int part_bytes = tn * R * dg::kBlockM * 4;
    if (kb_box > 256 || scale_bytes > dg::kSwapMaxScaleBytes)
        return DG_ERR_UNSUPPORTED;
    int stages = 0, dyn_smem = 0;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        KernelSmem &ks = g_smem_swap[dev][idx];
        if (ks.static_bytes < 0) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, fn);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.static_bytes = static_cast<int>(fa.sharedSizeBytes);
        }
        const int dyn_cap = info->smem_optin - ks.static_bytes;
        stages = std::min(dg::kMaxStages, (dyn_cap - 1024 - scale_bytes) / sbytes);
        if (stages_override > 0)
            stages = std::min(stages, stages_override);
        // the operand stages are reused for the fp32 partial after the K loop
        if (stages < 2 || stages * sbytes < part_bytes)
            return DG_ERR_UNSUPPORTED;
        dyn_smem = stages * sbytes + scale_bytes + 1024;
        dyn_smem = std::min(std::max(dyn_smem, kMinDynSmem), dyn_cap);
        if (ks.limit_set < dyn_smem) {
            cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.limit_set = dyn_smem;
        }
    }
    const int sfa_ld = align4(M);
    CUtensorMap map_a, map_b, map_sa;
    if (make_map_kblocks(&map_a, const_cast<void *>(args.a), K, M, 1, tn, dg::kSwapKbPerStage) != DG_OK ||
        make_map_kblocks(&map_b, const_cast<void *>(args.b), K, N, 1, R * dg::kBlockM,
                         dg::kSwapKbPerStage, args.b_fp4 != 0) != DG_OK ||
        make_map(&map_sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float *>(args.sfa), sfa_ld,
                 num_kb, 1, static_cast<uint64_t>(sfa_ld) * 4, static_cast<uint64_t>(sfa_ld) * 4 * num_kb,
                 tn, kb_box, CU_TENSOR_MAP_SWIZZLE_NONE) != DG_OK) {
        if (debug_enabled())
            std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled failed (swapped operands)\n");
        return DG_ERR_CUDA;
    }
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.num_kb = num_kb;
    p.num_nb = num_nb;
    p.m_tiles = kb_box;
    p.n_tiles = n_tiles;
    p.stages = stages;
    p.raster_m = S;
    p.sfa = args.sfa;
    p.sfa_ld = sfa_ld;
    p.sfb = args.sfb;
    p.d = static_cast<__nv_bfloat16 *>(args.d);
    p.err = info->err_ptr;
    p.timeout_ns = timeout;
    p.inject_stall = inject_stall_flag();
    p.idesc_b = args.b_fp4 ? dg::ptx::kIdescBFormatE2M1 : 0u;
    p.num_tiles = n_tiles;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(n_tiles * S, 1, 1);
    cfg.blockDim = dim3(dg::kNumThreads, 1, 1);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = static_cast<cudaStream_t>(args.stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 1);
    void *kargs[] = {&map_a, &map_b, &map_sa, &p};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, kargs);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] swapped-operand launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    t_last.valid = true;
    t_last.block_n = R * dg::kBlockM;
    t_last.stages = stages;
    t_last.grid = n_tiles * S;
    t_last.tiles = n_tiles;
    t_last.pair = 0;
    t_last.splits = S;
    t_last.family = 4;
    if (debug_enabled())
        std::fprintf(stderr, "[dg] swap M=%d N=%d K=%d TN=%d R=%d S=%d stages=%d grid=%d smem=%d\n", M,
                     N, K, tn, R, S, stages, n_tiles * S, dyn_smem);
    return DG_OK;
}

// ---- stream-K swapped-operand kernel (dense, M <= 64, caller's workspace) --------------------

template <int TN>
void *swap_sk_kernel_ptr()
{
    return reinterpret_cast<void *>(&dg::dg_gemm_swap_sk_kernel<TN>);
}

void *pick_swap_sk_kernel(int tn)
{
    return tn == 32 ? swap_sk_kernel_ptr<32>() : tn == 64 ? swap_sk_kernel_ptr<64>() : nullptr;
}

// The stream-K plan of a dense call: P CTAs (one per SM), U = tiles x K/128 units, at most H
// units per CTA.  Returns false where the kernel does not apply: more than 64 tokens, fewer
// units than SMs, more tiles than SMs (a CTA's range would span three tiles), or an A-scale box
// taller than TMA allows.
struct SkPlan {
    int tn = 0, P = 0, n_tiles = 0, H = 0;
    size_t part_bytes = 0, count_bytes = 0;
    size_t total() const { return part_bytes + count_bytes; }
};

bool plan_swap_sk(int M, int N, int K, int sms, SkPlan &pl)
{
    if (M < 1 || M > 64 || sms < 1)
        return false;
    const int num_kb = K / dg::kBlockK;
    pl.tn = swap_token_tile(M);
    pl.n_tiles = (N + dg::kBlockM - 1) / dg::kBlockM;
    pl.P = sms;
    const long long U = static_cast<long long>(pl.n_tiles) * num_kb;
    if (pl.n_tiles > pl.P || U < pl.P)
        return false;
    pl.H = static_cast<int>((U + pl.P - 1) / pl.P);
    if (pl.H > 256 || pl.H > num_kb)
        return false;
    pl.part_bytes = static_cast<size_t>(pl.P) * 2 * pl.tn * dg::kBlockM * 4;
    pl.count_bytes = (static_cast<size_t>(pl.n_tiles) * 4 + 255) / 256 * 256;
    return true;
}

int launch_swap_sk(const LaunchArgs &args, int dev, DeviceInfo *info, const SkPlan &pl, float *ws,
                   int *ws_count, int stages_override, unsigned long long timeout)
{
    const int M = args.M, N = args.N, K = args.K;
    const int num_kb = K / dg::kBlockK;
    const int num_nb = (N + dg::kBlockK - 1) / dg::kBlockK;
    void *fn = pick_swap_sk_kernel(pl.tn);
    if (fn == nullptr)
        return DG_ERR_INVALID_ARG;
    const int idx = pl.tn == 32 ? 0 : 1;
    const int sbytes = swap_stage_bytes(pl.tn, 1);
    const int scale_bytes = 2 * pl.H * pl.tn * 4;
    int stages = 0, dyn_smem = 0;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        KernelSmem &ks = g_smem_swap_sk[dev][idx];
        if (ks.static_bytes < 0) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, fn);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.static_bytes = static_cast<int>(fa.sharedSizeBytes);
        }
        const int dyn_cap = info->smem_optin - ks.static_bytes;
        stages = std::min(dg::kMaxStages, (dyn_cap - 1024 - scale_bytes) / sbytes);
        if (stages_override > 0)
            stages = std::min(stages, stages_override);
        if (stages < 2)
            return DG_ERR_UNSUPPORTED;
        dyn_smem = stages * sbytes + scale_bytes + 1024;
        dyn_smem = std::min(std::max(dyn_smem, kMinDynSmem), dyn_cap);
        if (ks.limit_set < dyn_smem) {
            cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                return DG_ERR_CUDA;
            }
            ks.limit_set = dyn_smem;
        }
    }
    const int sfa_ld = align4(M);
    CUtensorMap map_a, map_b, map_sa;
    if (make_map_kblocks(&map_a, const_cast<void *>(args.a), K, M, 1, pl.tn, dg::kSwapKbPerStage) != DG_OK ||
        make_map_kblocks(&map_b, const_cast<void *>(args.b), K, N, 1, dg::kBlockM, dg::kSwapKbPerStage,
                         args.b_fp4 != 0) != DG_OK ||
        make_map(&map_sa, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float *>(args.sfa), sfa_ld, num_kb, 1,
                 static_cast<uint64_t>(sfa_ld) * 4, static_cast<uint64_t>(sfa_ld) * 4 * num_kb, pl.tn, pl.H,
                 CU_TENSOR_MAP_SWIZZLE_NONE) != DG_OK) {
        if (debug_enabled())
            std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled failed (stream-K)\n");
        return DG_ERR_CUDA;
    }
    Params p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = 1;
    p.num_kb = num_kb;
    p.num_nb = num_nb;
    p.m_tiles = pl.H;
    p.n_tiles = pl.n_tiles;
    p.num_tiles = pl.n_tiles;
    p.stages = stages;
    p.raster_m = pl.P;
    p.sfa = args.sfa;
    p.sfa_ld = sfa_ld;
    p.sfb = args.sfb;
    p.d = static_cast<__nv_bfloat16 *>(args.d);
    p.err = info->err_ptr;
    p.timeout_ns = timeout;
    p.inject_stall = inject_stall_flag();
    p.idesc_b = args.b_fp4 ? dg::ptx::kIdescBFormatE2M1 : 0u;
    p.ws = ws;
    p.ws_count = ws_count;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(pl.P, 1, 1);
    cfg.blockDim = dim3(dg::kNumThreads, 1, 1);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = static_cast<cudaStream_t>(args.stream);
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 0);
    void *kargs[] = {&map_a, &map_b, &map_sa, &p};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, kargs);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] stream-K launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    t_last.valid = true;
    t_last.block_n = dg::kBlockM;
    t_last.stages = stages;
    t_last.grid = pl.P;
    t_last.tiles = pl.n_tiles;
    t_last.pair = 0;
    t_last.splits = pl.H;
    t_last.family = 5;
    if (debug_enabled())
        std::fprintf(stderr, "[dg] stream-K M=%d N=%d K=%d TN=%d P=%d H=%d stages=%d smem=%d\n", M, N, K,
                     pl.tn, pl.P, pl.H, stages, dyn_smem);
    return DG_OK;
}

int launch(const LaunchArgs &args)
{
    int dev = 0;
    DeviceInfo *info = nullptr;
    int st = device_setup(dev, info);
    if (st != DG_OK)
        return st;

    const int M = args.M, N = args.N, K = args.K, G = args.G;
    const int num_kb = K / dg::kBlockK;
    const int num_nb = (N + dg::kBlockK - 1) / dg::kBlockK;
    const int m_tiles = (M + dg::kBlockM - 1) / dg::kBlockM;
    int sms = info->num_sms;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_num_sms_cap > 0 && g_num_sms_cap < sms)
            sms = g_num_sms_cap;
    }

    // tile choice
    int bn;
    int stages_override;
    unsigned long long timeout;
    int pair_mode;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        bn = g_override_bn;
        stages_override = g_override_stages;
        timeout = g_timeout_ns;
        pair_mode = g_family;
    }
    // Swapped operands for dense problems with few rows (decode-sized token counts): B rows on
    // the MMA's 128-lane side, the tokens on its N side.  Family 4 forces it for M <= 128.  Auto
    // mode takes it for M <= 64 with one 128-row block of B per tile, where it measured ahead of
    // split-K on B200 (1-2 us on the 2112 / 4096 / 7168-wide decode shapes); with 65-128 tokens,
    // or when the tiles need two row blocks to fit in one wave, split-K and the one-CTA kernel
    // were level or faster.  (In auto mode a block_n override keeps the families it names.)
    // Stream-K over every SM (dense M <= 64, family 5, the caller's workspace).  Automatic mode
    // does not take it: on B200 it measured slower than the cluster kernels on every decode
    // shape tried (64 x 7168 x 16384: 43.0 vs 36.9 us; 64 x 4096 x 7168: 26.1 vs 18.5 us), the
    // partial round trip through L2 and the fix-up costing more than the SMs it adds.
    if (args.layout == dg::kDense && pair_mode == 5) {
        SkPlan pl;
        if (!plan_swap_sk(M, N, K, sms, pl))
            return DG_ERR_UNSUPPORTED;
        if (args.ws == nullptr || args.ws_bytes < pl.total())
            return DG_ERR_WORKSPACE;
        float *ws = static_cast<float *>(args.ws);
        int *cnt = reinterpret_cast<int *>(static_cast<char *>(args.ws) + pl.part_bytes);
        return launch_swap_sk(args, dev, info, pl, ws, cnt, stages_override, timeout);
    }
    const bool swap_auto = pair_mode == 0 && bn == 0 && M <= 64;
    if (args.layout == dg::kDense && M <= 128 && (pair_mode == 4 || swap_auto)) {
        int splits_override;
        {
            std::lock_guard<std::mutex> lock(g_mutex);
            splits_override = g_override_splits;
        }
        const int r_fixed = bn == 128 ? 1 : bn == 256 ? 2 : (pair_mode == 0 ? 1 : 0);
        auto capacity = [&](int ctn, int cR, int cs) -> long long {
            void *fn = pick_swap_kernel(ctn, cR);
            const int smem = std::max(std::min(2 * swap_stage_bytes(ctn, cR) + 16 * 1024, 200 * 1024),
                                      kMinDynSmem);
            int n = max_active_clusters(fn, cs, smem, dev, 3 + swap_index(ctn, cR));
            if (n <= 0)
                n = sms / cs;
            return std::min<long long>(n, sms / cs);
        };
        int R = 0, S = 0;
        // static shared memory of the swapped kernel is a few hundred bytes: leave 1 KB for it
        const int dyn_cap = info->smem_optin - 1024;
        if (choose_swap(M, N, K, args.b_fp4 != 0, sms, dyn_cap, r_fixed, splits_override, capacity,
                        R, S)) {
            const int st_swap = launch_swap(args, dev, info, R, S, stages_override, timeout);
            if (st_swap != DG_ERR_UNSUPPORTED || pair_mode == 4)
                return st_swap;
        } else if (pair_mode == 4) {
            return DG_ERR_UNSUPPORTED;
        }
    }
    if (pair_mode == 4)
        pair_mode = 0;  // layouts and sizes the swapped kernel does not take run as in auto mode
    // Split-K clusters for dense problems with few output tiles (the memory-bound small-M
    // regime): auto mode uses them for M <= 256.
    if (args.layout == dg::kDense && (pair_mode == 3 || (pair_mode == 0 && M <= 256)) &&
        (bn == 0 || pick_splitk_kernel(bn) != nullptr)) {
        int sbn = 0, S = 0;
        int splits_override;
        {
            std::lock_guard<std::mutex> lock(g_mutex);
            splits_override = g_override_splits;
        }
        auto capacity = [&](int cbn, int cs) -> long long {
            void *fn = pick_splitk_kernel(cbn);
            const int sb = dg::kSplitKbPerStage * (dg::kBlockM * dg::kBlockK + cbn * dg::kBlockK);
            const int smem = std::max(std::min(2 * sb, 200 * 1024), kMinDynSmem);
            int n = max_active_clusters(fn, cs, smem, dev, 2);
            if (n <= 0)
                n = sms / cs;
            return std::min<long long>(n, sms / cs);
        };
        if (choose_splitk(M, N, K, sms, bn, splits_override, capacity, sbn, S)) {
            if (S > 1 || pair_mode == 3)
                return launch_splitk(args, dev, info, sbn, S, stages_override, timeout);
            // one split: the one-CTA kernel does the same work without the reduction round
            // trip through shared memory
            if (bn == 0)
                bn = sbn;
        }
    }
    // CTA pairs (cta_group::2) for the dense and masked layouts: 256-row tiles whose B half is
    // loaded by each CTA.  Auto mode uses them for dense problems with more than 192 rows and
    // long K (kPairMinKBlocks).  Masked problems stay on the one-CTA kernel: they are bound by
    // streaming each expert's B once, and a one-CTA tile takes in all BN rows of B per K block
    // where a pair tile splits them over two SMs (measured on B200, G=32, M_max=256, N=4096,
    // K=7168: 236 us one-CTA vs 258 us pair, interleaved runs).  Family 2 still forces pairs.
    bool use_pair = false;
    if (args.layout != dg::kContiguous && sms >= 2 && pair_mode != 1 && pair_mode != 3) {
        if (pair_mode == 2)
            use_pair = true;
        else if (args.layout == dg::kDense)
            use_pair = M > 192 && num_kb >= kPairMinKBlocks;
        else
            use_pair = false;  // masked: the one-CTA kernel measured ahead (see below)
        if (bn != 0 && pick_pair_kernel(args.layout, bn) == nullptr)
            use_pair = false;  // the block_n override names a tile the pair kernel lacks
    }
    if (use_pair)
        return launch_pair(args, dev, info, sms, bn, stages_override, timeout);
    if (bn == 0) {
        long long row_tiles = m_tiles;
        if (args.layout == dg::kMasked) {
            int em = args.expected_m > 0 ? std::min(args.expected_m, M) : M;
            row_tiles = static_cast<long long>(G) * ((em + dg::kBlockM - 1) / dg::kBlockM);
        }
        bn = choose_block_n(static_cast<int>(std::max<long long>(1, row_tiles)), N, sms);
    }
    const int n_tiles = (N + bn - 1) / bn;
    const int sbytes = stage_bytes_rt(bn);
    void *fn = pick_kernel(args.layout, bn);
    if (fn == nullptr)
        return DG_ERR_INVALID_ARG;
    int dyn_smem = 0;
    int stages = 0;
    {
        // The dynamic shared-memory limit of each kernel is raised once per device and only
        // when a launch needs more, so launches can be captured into CUDA graphs.
        std::lock_guard<std::mutex> lock(g_mutex);
        KernelSmem &ks = g_smem[dev][args.layout][bn / 32 - 1];
        if (ks.static_bytes < 0) {
            cudaFuncAttributes fa;
            cudaError_t e = cudaFuncGetAttributes(&fa, fn);
            if (e != cudaSuccess) {
                cudaGetLastError();
                if (debug_enabled())
                    std::fprintf(stderr, "[dg] cudaFuncGetAttributes: %s\n", cudaGetErrorString(e));
                return DG_ERR_CUDA;
            }
            ks.static_bytes = static_cast<int>(fa.sharedSizeBytes);
        }
        const int dyn_cap = info->smem_optin - ks.static_bytes;  // dynamic bytes allowed
        const int epi = dg::whole_tile_epi_bytes(bn);
        stages = std::min(dg::kMaxStages, (dyn_cap - 1024 - epi) / sbytes);
        if (stages_override > 0)
            stages = std::min(stages, stages_override);
        if (stages < 2)
            return DG_ERR_UNSUPPORTED;
        // operand stages, the output staging of a whole tile, and slack to align the stages to
        // 1024 bytes
        dyn_smem = stages * sbytes + epi + 1024;
        dyn_smem = std::min(std::max(dyn_smem, kMinDynSmem), dyn_cap);
        if (ks.limit_set < dyn_smem) {
            cudaError_t e =
                cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_smem);
            if (e != cudaSuccess) {
                cudaGetLastError();
                if (debug_enabled())
                    std::fprintf(stderr, "[dg] cudaFuncSetAttribute(%d): %s\n", dyn_smem,
                                 cudaGetErrorString(e));
                return DG_ERR_CUDA;
            }
            ks.limit_set = dyn_smem;
        }
    }

    // tensor maps
    const int a_rows = (args.layout == dg::kMasked) ? M : M;
    const int a_groups = (args.layout == dg::kMasked) ? G : 1;
    const int b_groups = (args.layout == dg::kDense) ? 1 : G;
    const int m4 = align4(M);
    CUtensorMap map_a, map_b, map_d64, map_d32, map_d16;
    const uint64_t d_rows = static_cast<uint64_t>(a_rows) * a_groups;
    if (make_map_d(&map_d64, args.d, N, d_rows, 64) != DG_OK ||
        make_map_d(&map_d32, args.d, N, d_rows, 32) != DG_OK ||
        make_map_d(&map_d16, args.d, N, d_rows, 16) != DG_OK ||
        make_map(&map_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<void *>(args.a), K, a_rows,
                 a_groups, static_cast<uint64_t>(K), static_cast<uint64_t>(K) * a_rows, dg::kBlockK,
                 dg::kBlockM, CU_TENSOR_MAP_SWIZZLE_128B) != DG_OK ||
        (args.b_fp4
             ? make_map(&map_b, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, const_cast<void *>(args.b), K, N,
                        b_groups, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(K) / 2 * N,
                        dg::kBlockK, bn, CU_TENSOR_MAP_SWIZZLE_128B)
             : make_map(&map_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<void *>(args.b), K, N,
                        b_groups, static_cast<uint64_t>(K), static_cast<uint64_t>(K) * N, dg::kBlockK,
                        bn, CU_TENSOR_MAP_SWIZZLE_128B)) != DG_OK) {
        if (debug_enabled())
            std::fprintf(stderr, "[dg] cuTensorMapEncodeTiled failed\n");
        return DG_ERR_CUDA;
    }

    Params p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = K;
    p.G = (args.layout == dg::kDense) ? 1 : G;
    p.num_kb = num_kb;
    p.num_nb = num_nb;
    p.m_tiles = m_tiles;
    p.n_tiles = n_tiles;
    p.stages = stages;
    p.raster_m = 16;
    p.sfa = args.sfa;
    p.sfa_ld = m4;
    p.sfb = args.sfb;
    p.d = static_cast<__nv_bfloat16 *>(args.d);
    p.m_indices = args.m_indices;
    p.masked_m = args.masked_m;
    p.err = info->err_ptr;
    p.timeout_ns = timeout;
    p.inject_stall = inject_stall_flag();
    p.idesc_b = args.b_fp4 ? dg::ptx::kIdescBFormatE2M1 : 0u;
    long long tiles;
    if (args.layout == dg::kMasked)
        tiles = static_cast<long long>(G) * m_tiles * n_tiles;  // upper bound; exact on device
    else
        tiles = static_cast<long long>(m_tiles) * n_tiles;
    if (tiles > 0x7FFFFFFFLL)
        return DG_ERR_INVALID_ARG;
    p.num_tiles = static_cast<int>(tiles);
    int grid = static_cast<int>(std::min<long long>(sms, tiles));
    if (grid <= 0)
        return DG_OK;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(dg::kNumThreads, 1, 1);
    cfg.dynamicSmemBytes = dyn_smem;
    cfg.stream = static_cast<cudaStream_t>(args.stream);
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 0);
    void *kargs[] = {&map_a, &map_b, &map_d64, &map_d32, &map_d16, &p};
    cudaError_t e = cudaLaunchKernelExC(&cfg, fn, kargs);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    t_last.valid = true;
    t_last.block_n = bn;
    t_last.stages = stages;
    t_last.grid = grid;
    t_last.tiles = p.num_tiles;
    t_last.pair = 0;
    t_last.splits = 1;
    t_last.family = 1;
    if (debug_enabled())
        std::fprintf(stderr, "[dg] layout=%d M=%d N=%d K=%d G=%d BN=%d stages=%d grid=%d tiles=%d smem=%d\n",
                     args.layout, M, N, K, G, bn, stages, grid, p.num_tiles, dyn_smem);
    return DG_OK;
}

int check_common(const void *a, const float *sfa, const void *b, const float *sfb, void *d, int N,
                 int K)
{
    if (!a || !sfa || !b || !sfb || !d)
        return DG_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(sfa) || !aligned16(b) || !aligned16(sfb) || !aligned16(d))
        return DG_ERR_INVALID_ARG;
    if (K <= 0 || K % dg::kBlockK != 0 || N <= 0 || N % 8 != 0)
        return DG_ERR_INVALID_ARG;
    return DG_OK;
}

int launch_swiglu_quantize(const void *h, void *q, float *sfa, int M, int I, const int *masked_m,
                           int rows_per_group, void *stream)
{
    int dev = 0;
    DeviceInfo *info = nullptr;
    int st = device_setup(dev, info);
    if (st != DG_OK)
        return st;
    const long long blocks_x = (static_cast<long long>(M) + dg::kQuantRowsPerBlock - 1) / dg::kQuantRowsPerBlock;
    if (blocks_x > 0x7FFFFFFFLL || I / dg::kBlockK > 65535)
        return DG_ERR_INVALID_ARG;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(blocks_x), static_cast<unsigned>(I / dg::kBlockK), 1);
    cfg.blockDim = dim3(dg::kQuantThreads, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 0);
    const __nv_bfloat16 *hp = static_cast<const __nv_bfloat16 *>(h);
    uint8_t *qp = static_cast<uint8_t *>(q);
    cudaError_t e = cudaLaunchKernelEx(&cfg, dg::dg_swiglu_quantize_1x128_kernel, hp, qp, sfa, M, I,
                                       masked_m, rows_per_group);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] swiglu-quantize launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    return DG_OK;
}

int launch_quantize(const void *x, void *q, float *sfa, int M, int K, void *stream)
{
    int dev = 0;
    DeviceInfo *info = nullptr;
    int st = device_setup(dev, info);
    if (st != DG_OK)
        return st;
    const long long blocks_x = (static_cast<long long>(M) + dg::kQuantRowsPerBlock - 1) / dg::kQuantRowsPerBlock;
    if (blocks_x > 0x7FFFFFFFLL || K / dg::kBlockK > 65535)
        return DG_ERR_INVALID_ARG;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(blocks_x), static_cast<unsigned>(K / dg::kBlockK), 1);
    cfg.blockDim = dim3(dg::kQuantThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    cfg.attrs = attr;
    cfg.numAttrs = add_pdl_attr(attr, 0);
    const __nv_bfloat16 *xp = static_cast<const __nv_bfloat16 *>(x);
    uint8_t *qp = static_cast<uint8_t *>(q);
    int m4 = align4(M);
    cudaError_t e = cudaLaunchKernelEx(&cfg, dg::dg_quantize_1x128_kernel, xp, qp, sfa, M, K, m4);
    if (e != cudaSuccess) {
        cudaGetLastError();
        if (debug_enabled())
            std::fprintf(stderr, "[dg] quantize launch failed: %s\n", cudaGetErrorString(e));
        return DG_ERR_CUDA;
    }
    return DG_OK;
}

}  // namespace

extern "C" {

int dg_swiglu_quantize_fp8_1x128(const void *h, void *q, float *sfa, int M, int I,
                                 const int *masked_m, int rows_per_group, void *stream)
{
    if (M < 0 || I <= 0 || I % dg::kBlockK != 0)
        return DG_ERR_INVALID_ARG;
    if (masked_m != nullptr && (rows_per_group <= 0 || M % rows_per_group != 0))
        return DG_ERR_INVALID_ARG;
    if (M == 0)
        return DG_OK;
    if (!h || !q || !sfa || !aligned16(h) || !aligned16(q) || !aligned16(sfa))
        return DG_ERR_INVALID_ARG;
    return launch_swiglu_quantize(h, q, sfa, M, I, masked_m, masked_m ? rows_per_group : 0, stream);
}

int dg_quantize_fp8_1x128(const void *x, void *q, float *sfa, int M, int K, void *stream)
{
    if (M < 0 || K <= 0 || K % dg::kBlockK != 0)
        return DG_ERR_INVALID_ARG;
    if (M == 0)
        return DG_OK;
    if (!x || !q || !sfa || !aligned16(x) || !aligned16(q) || !aligned16(sfa))
        return DG_ERR_INVALID_ARG;
    return launch_quantize(x, q, sfa, M, K, stream);
}

}  // extern "C"

namespace {

// B of the FP8 x FP4 entries is packed E2M1; the tensor map for that layout wants a 32-byte
// aligned base.
bool b_aligned(const void *b, int b_fp4)
{
    return (reinterpret_cast<uintptr_t>(b) & (b_fp4 ? 31u : 15u)) == 0;
}

int gemm_dense(const void *a, const float *sfa, const void *b, const float *sfb, void *d, int M,
               int N, int K, void *stream, int b_fp4, void *ws = nullptr, size_t ws_bytes = 0)
{
    if (M < 0)
        return DG_ERR_INVALID_ARG;
    if (M == 0)
        return (N > 0 && N % 8 == 0 && K > 0 && K % dg::kBlockK == 0) ? DG_OK : DG_ERR_INVALID_ARG;
    int st = check_common(a, sfa, b, sfb, d, N, K);
    if (st != DG_OK)
        return st;
    if (!b_aligned(b, b_fp4))
        return DG_ERR_INVALID_ARG;
    if (ws != nullptr && (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return DG_ERR_INVALID_ARG;
    LaunchArgs la{dg::kDense, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0, stream, b_fp4, ws, ws_bytes};
    return launch(la);
}

int gemm_contiguous(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                    const int *m_indices, int M_total, int N, int K, int G, void *stream, int b_fp4)
{
    if (M_total < 0 || M_total % dg::kBlockM != 0 || G <= 0)
        return DG_ERR_INVALID_ARG;
    if (M_total == 0)
        return (N > 0 && N % 8 == 0 && K > 0 && K % dg::kBlockK == 0) ? DG_OK : DG_ERR_INVALID_ARG;
    int st = check_common(a, sfa, b, sfb, d, N, K);
    if (st != DG_OK)
        return st;
    if (!b_aligned(b, b_fp4))
        return DG_ERR_INVALID_ARG;
    if (!m_indices || (reinterpret_cast<uintptr_t>(m_indices) & 3u))
        return DG_ERR_INVALID_ARG;
    LaunchArgs la{dg::kContiguous, a, sfa, b, sfb, d, m_indices, nullptr, M_total, N, K, G, 0,
                  stream, b_fp4};
    return launch(la);
}

int gemm_masked(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                const int *masked_m, int G, int M_max, int N, int K, int expected_m, void *stream,
                int b_fp4)
{
    if (G <= 0 || G > dg::kMaxMaskedGroups || M_max < 0 || expected_m < 0)
        return DG_ERR_INVALID_ARG;
    if (M_max == 0)
        return (N > 0 && N % 8 == 0 && K > 0 && K % dg::kBlockK == 0) ? DG_OK : DG_ERR_INVALID_ARG;
    int st = check_common(a, sfa, b, sfb, d, N, K);
    if (st != DG_OK)
        return st;
    if (!b_aligned(b, b_fp4))
        return DG_ERR_INVALID_ARG;
    if (!masked_m || (reinterpret_cast<uintptr_t>(masked_m) & 3u))
        return DG_ERR_INVALID_ARG;
    LaunchArgs la{dg::kMasked, a, sfa, b, sfb, d, nullptr, masked_m, M_max, N, K, G, expected_m,
                  stream, b_fp4};
    return launch(la);
}

// ---- the dense GEMM without any allocation: the stream-K kernel with built-in scratch ----------

// Scratch of dg_gemm_fp8_fp8_bf16_nt_noalloc: the stream-K kernel's partial slots and, after
// them, its per-tile arrival counters.  A file-scope device array, so every GPU that loads the
// library holds it until the process exits.  Host code may not use its name as an address: the
// device address is looked up once per device (noalloc_scratch) and passed to the kernel.
constexpr size_t kNoAllocScratchBytes = size_t(12) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void *g_noalloc_ptr[kMaxDevices];  // device address of the array, per device (null: not looked up)

// The array's device address on the current device `dev`, looked up on the first call there.
int noalloc_scratch(int dev, unsigned char *&ptr)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return DG_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    ptr = static_cast<unsigned char *>(g_noalloc_ptr[dev]);
    return DG_OK;
}

}  // namespace

extern "C" {

int dg_gemm_fp8_fp8_bf16_nt(const void *a, const float *sfa, const void *b, const float *sfb,
                            void *d, int M, int N, int K, void *workspace, size_t workspace_bytes,
                            void *stream)
{
    return gemm_dense(a, sfa, b, sfb, d, M, N, K, stream, 0, workspace, workspace_bytes);
}

int dg_gemm_fp8_fp8_bf16_nt_noalloc(const void *a, const float *sfa, const void *b, const float *sfb,
                                    void *d, int M, int N, int K, void *stream)
{
    if (M < 0)
        return DG_ERR_INVALID_ARG;
    if (M == 0)
        return (N > 0 && N % 8 == 0 && K > 0 && K % dg::kBlockK == 0) ? DG_OK : DG_ERR_INVALID_ARG;
    int st = check_common(a, sfa, b, sfb, d, N, K);
    if (st != DG_OK)
        return st;
    if (!b_aligned(b, 0))
        return DG_ERR_INVALID_ARG;
    int dev = 0;
    DeviceInfo *info = nullptr;
    st = device_setup(dev, info);
    if (st != DG_OK)
        return st;
    int sms = info->num_sms;
    int stages_override;
    unsigned long long timeout;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_num_sms_cap > 0 && g_num_sms_cap < sms)
            sms = g_num_sms_cap;
        stages_override = g_override_stages;
        timeout = g_timeout_ns;
    }
    SkPlan pl;
    if (!plan_swap_sk(M, N, K, sms, pl))
        return DG_ERR_UNSUPPORTED;
    if (pl.total() > kNoAllocScratchBytes)
        return DG_ERR_WORKSPACE;  // more scratch than the built-in array holds
    unsigned char *scratch = nullptr;
    st = noalloc_scratch(dev, scratch);
    if (st != DG_OK)
        return st;
    // the tile counters start at zero whatever an earlier call left there
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch + pl.part_bytes, 0, pl.count_bytes, s) != cudaSuccess) {
        cudaGetLastError();
        return DG_ERR_CUDA;
    }
    LaunchArgs la{dg::kDense, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0, stream, 0};
    return launch_swap_sk(la, dev, info, pl, reinterpret_cast<float *>(scratch),
                          reinterpret_cast<int *>(scratch + pl.part_bytes), stages_override, timeout);
}

int dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(const void *a, const float *sfa, const void *b,
                                                 const float *sfb, void *d, const int *m_indices,
                                                 int M_total, int N, int K, int G, void *workspace,
                                                 size_t workspace_bytes, void *stream)
{
    (void)workspace;
    (void)workspace_bytes;
    return gemm_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G, stream, 0);
}

int dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(const void *a, const float *sfa, const void *b,
                                             const float *sfb, void *d, const int *masked_m, int G,
                                             int M_max, int N, int K, int expected_m,
                                             void *workspace, size_t workspace_bytes, void *stream)
{
    (void)workspace;
    (void)workspace_bytes;
    return gemm_masked(a, sfa, b, sfb, d, masked_m, G, M_max, N, K, expected_m, stream, 0);
}

int dg_gemm_fp8_fp4_bf16_nt(const void *a, const float *sfa, const void *b, const float *sfb,
                            void *d, int M, int N, int K, void *stream)
{
    return gemm_dense(a, sfa, b, sfb, d, M, N, K, stream, 1);
}

int dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(const void *a, const float *sfa, const void *b,
                                                 const float *sfb, void *d, const int *m_indices,
                                                 int M_total, int N, int K, int G, void *stream)
{
    return gemm_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G, stream, 1);
}

int dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(const void *a, const float *sfa, const void *b,
                                             const float *sfb, void *d, const int *masked_m, int G,
                                             int M_max, int N, int K, int expected_m, void *stream)
{
    return gemm_masked(a, sfa, b, sfb, d, masked_m, G, M_max, N, K, expected_m, stream, 1);
}

int dg_set_num_sms(int n)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    int prev = g_num_sms_cap;
    g_num_sms_cap = n > 0 ? n : 0;
    return prev;
}

int dg_get_num_sms(void)
{
    int dev = 0;
    DeviceInfo *info = nullptr;
    int st = device_setup(dev, info);
    if (st != DG_OK)
        return st;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_num_sms_cap > 0 && g_num_sms_cap < info->num_sms)
        return g_num_sms_cap;
    return info->num_sms;
}

int dg_get_tma_aligned_size(int x, int elem_bytes)
{
    if (x < 0 || elem_bytes <= 0)
        return DG_ERR_INVALID_ARG;
    // smallest x' >= x with x' * elem_bytes % 16 == 0
    long long step = 16;
    long long g = elem_bytes;
    long long a = step, b2 = g;
    while (b2) {
        long long tmp = a % b2;
        a = b2;
        b2 = tmp;
    }
    long long unit = step / a;  // elements per alignment unit
    long long r = (static_cast<long long>(x) + unit - 1) / unit * unit;
    return r > 0x7FFFFFFFLL ? DG_ERR_INVALID_ARG : static_cast<int>(r);
}

size_t dg_get_workspace_size(int kind, int M, int N, int K, int G)
{
    (void)G;
    if (kind != 0 || N <= 0 || K <= 0 || K % dg::kBlockK != 0)
        return 0;
    int dev = 0;
    DeviceInfo *info = nullptr;
    if (device_setup(dev, info) != DG_OK)
        return 0;
    int sms = info->num_sms;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_num_sms_cap > 0 && g_num_sms_cap < sms)
            sms = g_num_sms_cap;
    }
    SkPlan pl;
    return plan_swap_sk(M, N, K, sms, pl) ? pl.total() : 0;
}

const char *dg_status_string(int status)
{
    switch (status) {
    case DG_OK:
        return "DG_OK";
    case DG_ERR_INVALID_ARG:
        return "DG_ERR_INVALID_ARG: invalid argument";
    case DG_ERR_UNSUPPORTED:
        return "DG_ERR_UNSUPPORTED: no sm_100 device or unsupported configuration";
    case DG_ERR_CUDA:
        return "DG_ERR_CUDA: a CUDA call failed";
    case DG_ERR_TIMEOUT:
        return "DG_ERR_TIMEOUT: a device pipeline wait timed out";
    case DG_ERR_WORKSPACE:
        return "DG_ERR_WORKSPACE: workspace missing or too small";
    case DG_ERR_LAYOUT:
        return "DG_ERR_LAYOUT: an index array broke its layout contract";
    default:
        return "unknown dg_status";
    }
}

int dg_poll_device_error(void *stream)
{
    int dev = 0;
    DeviceInfo *info = nullptr;
    int st = device_setup(dev, info);
    if (st != DG_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int value = 0;
    dg_take_error_kernel<<<1, 1, 0, s>>>();
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&value, g_polled_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return DG_ERR_CUDA;
    }
    return value;
}

unsigned long long dg_set_wait_timeout_ns(unsigned long long ns)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    unsigned long long prev = g_timeout_ns;
    g_timeout_ns = ns ? ns : kDefaultTimeoutNs;
    return prev;
}

int dg_set_config_override(int block_n, int num_stages, int splits)
{
    if (block_n != 0 && (block_n < 32 || block_n > 256 || block_n % 32 != 0))
        return DG_ERR_INVALID_ARG;
    if (num_stages != 0 && (num_stages < 2 || num_stages > dg::kMaxStages))
        return DG_ERR_INVALID_ARG;
    if (splits < 0 || splits > dg::kMaxSplits)
        return DG_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    g_override_bn = block_n;
    g_override_stages = num_stages;
    g_override_splits = splits;
    return DG_OK;
}

int dg_set_fault_injection(int mode)
{
    if (mode < 0 || mode > 1)
        return DG_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    int prev = g_inject_stall;
    g_inject_stall = mode;
    return prev;
}

int dg_set_pdl(int enable)
{
    if (enable != 0 && enable != 1)
        return DG_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    int prev = g_pdl;
    g_pdl = enable;
    return prev;
}

int dg_set_tensor_map_cache(int enable)
{
    if (enable != 0 && enable != 1)
        return DG_ERR_INVALID_ARG;
    return g_map_cache.set_enabled(enable == 1) ? 1 : 0;
}

int dg_get_tensor_map_cache_stats(unsigned long long *hits, unsigned long long *misses)
{
    unsigned long long h = 0, m = 0;
    g_map_cache.stats(h, m);
    if (hits)
        *hits = h;
    if (misses)
        *misses = m;
    return DG_OK;
}

int dg_set_kernel_family(int family)
{
    if (family < 0 || family > 5)
        return DG_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    int prev = g_family;
    g_family = family;
    return prev;
}

int dg_get_last_launch(int *block_n, int *num_stages, int *grid, int *num_tiles, int *family,
                       int *splits)
{
    if (!t_last.valid)
        return DG_ERR_INVALID_ARG;
    if (family)
        *family = t_last.family;
    if (splits)
        *splits = t_last.splits;
    if (block_n)
        *block_n = t_last.block_n;
    if (num_stages)
        *num_stages = t_last.stages;
    if (grid)
        *grid = t_last.grid;
    if (num_tiles)
        *num_tiles = t_last.tiles;
    return DG_OK;
}

}  // extern "C"
