// dg_quant_kernel.cuh -- per-token (1 x 128) FP8 quantisation of bf16 activations for sm_100a:
// the step just before the GEMM, writing the e4m3 codes and the fp32 scales directly in the
// MN-major, TMA-aligned layout the GEMM reads.
//
// Method (DeepSeek開源第三彈 -- the DeepGEMM release write-up -- "深入了解DeepGEMM": activations
// carry one fp32 scale per 1 x 128 tile; "如何使用": the TMA-aligned scale layout).  For each row
// m and K block kb, in fp32 (every operation rounded to nearest even):
//     amax   = max(max |x| over the 128 elements, 1e-4)
//     factor = 448 / amax,  scale = amax / 448   (two divisions per tile)
//     q      = e4m3(x * factor)                  (round to nearest even, saturating at 448)
// The work is a stream through HBM (2 bytes in, 1 byte + 4/128 bytes out per element), so the
// kernel is built to spend few instructions per byte: a half-warp per tile (8 elements, one
// 16-byte load per lane), shuffle amax within the half-warp, one multiply and half a
// conversion per element, and 8 rows per warp with all their loads issued first, so that every
// SM keeps enough bytes in flight to cover DRAM latency.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;                         // row pairs per warp, loads in flight
constexpr int kQuantRowsPerWarp = 2 * kQuantUnroll;     // a half-warp per 128-element tile
constexpr int kQuantRowsPerBlock = (kQuantThreads / 32) * kQuantRowsPerWarp;

__device__ __forceinline__ uint4 ld_nc_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Two fp32 values to two e4m3 codes (round to nearest even, saturating to +-448); `lo` lands
// in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// x: bf16 [M][K]; q: e4m3 [M][K]; sfa: fp32 [K/128][sfa_ld], sfa_ld = align4(M).  Grid:
// (ceil(M / kQuantRowsPerBlock), K / 128); warp w of block (bx, kb) handles the 8 consecutive
// rows bx * 64 + 8 w + [0, 8) of K block kb, two rows at a time: lanes 0-15 the even row,
// lanes 16-31 the odd one, 8 elements (one 16-byte load) per lane.
__global__ void __launch_bounds__(kQuantThreads)
    dg_quantize_1x128_kernel(const __nv_bfloat16 *__restrict__ x, uint8_t *__restrict__ q,
                             float *__restrict__ sfa, int M, int K, int sfa_ld)
{
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4;
    const int hl = lane & 15;
    const int kb = blockIdx.y;
    const int row0 = blockIdx.x * kQuantRowsPerBlock + (threadIdx.x >> 5) * kQuantRowsPerWarp;
    const size_t col = static_cast<size_t>(kb) * 128 + hl * 8;
    uint4 raw[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
        const int row = row0 + 2 * u + half;
        raw[u] = row < M ? ld_nc_v4(x + static_cast<size_t>(row) * K + col) : make_uint4(0, 0, 0, 0);
    }
    float scales[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
        const int row = row0 + 2 * u + half;
        // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
        float f[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
        float amax = fabsf(f[0]);
#pragma unroll
        for (int i = 1; i < 8; ++i)
            amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)  // within the half-warp of this row
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        amax = fmaxf(amax, 1e-4f);
        const float factor = 448.0f / amax;
        const float scale = amax / 448.0f;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = f[i] * factor;
        if (row < M) {
            const uint32_t c01 = cvt_e4m3x2(v[0], v[1]), c23 = cvt_e4m3x2(v[2], v[3]);
            const uint32_t c45 = cvt_e4m3x2(v[4], v[5]), c67 = cvt_e4m3x2(v[6], v[7]);
            uint2 out;
            out.x = c01 | (c23 << 16);
            out.y = c45 | (c67 << 16);
            *reinterpret_cast<uint2 *>(q + static_cast<size_t>(row) * K + col) = out;
        }
        scales[u] = scale;
    }
    // the warp's 8 scales (rows row0 .. row0 + 7) are consecutive in the MN-major layout:
    // lanes 0 and 16 hold the even and odd rows; lane 0 gathers and stores them
    float odd[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u)
        odd[u] = __shfl_sync(0xffffffffu, scales[u], 16);
    if (lane == 0) {
        float *dst = sfa + static_cast<size_t>(kb) * sfa_ld + row0;
        if (row0 + kQuantRowsPerWarp <= M) {
            // row0 is a multiple of 8 and sfa_ld of 4: 16-byte aligned vector stores
            reinterpret_cast<float4 *>(dst)[0] = make_float4(scales[0], odd[0], scales[1], odd[1]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(scales[2], odd[2], scales[3], odd[3]);
        } else {
#pragma unroll
            for (int u = 0; u < kQuantUnroll; ++u) {
                if (row0 + 2 * u < M)
                    dst[2 * u] = scales[u];
                if (row0 + 2 * u + 1 < M)
                    dst[2 * u + 1] = odd[u];
            }
        }
    }
}

// ---- SwiGLU followed by the same quantisation --------------------------------------------------
// Between the two grouped GEMMs of an MoE layer: each row of the first GEMM's bf16 output h
// [M][2I] holds the gate half h[:, 0:I] and the up half h[:, I:2I]; the second GEMM's A operand
// is y = silu(gate) * up, silu(g) = g / (1 + exp(-g)) in fp32 with the GPU's fast exponential
// and division (y within a few fp32 ulps of exact), quantised per 1 x 128 tile as above.  With masked_m (the masked MoE layout, M = G * rows_per_group), row r of group g is
// processed only when r < masked_m[g], and the scales use that layout's per-group form
// [G][I/128][align4(rows_per_group)]; otherwise all rows, scales [I/128][align4(M)].
__global__ void __launch_bounds__(kQuantThreads)
    dg_swiglu_quantize_1x128_kernel(const __nv_bfloat16 *__restrict__ h, uint8_t *__restrict__ q,
                                    float *__restrict__ sfa, int M, int I, const int *masked_m,
                                    int rows_per_group)
{
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4;
    const int hl = lane & 15;
    const int kb = blockIdx.y;
    const int kbs = I / 128;
    const int row0 = blockIdx.x * kQuantRowsPerBlock + (threadIdx.x >> 5) * kQuantRowsPerWarp;
    const size_t col = static_cast<size_t>(kb) * 128 + hl * 8;
    bool valid[kQuantUnroll];
    uint4 gr[kQuantUnroll], ur[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
        const int row = row0 + 2 * u + half;
        bool v = row < M;
        if (v && masked_m != nullptr) {
            const int g = row / rows_per_group;
            v = row - g * rows_per_group < __ldg(masked_m + g);
        }
        valid[u] = v;
        if (v) {
            const __nv_bfloat16 *hr = h + static_cast<size_t>(row) * 2 * I + col;
            gr[u] = ld_nc_v4(hr);
            ur[u] = ld_nc_v4(hr + I);
        } else {
            gr[u] = make_uint4(0, 0, 0, 0);
            ur[u] = make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
        const int row = row0 + 2 * u + half;
        const uint32_t gw[4] = {gr[u].x, gr[u].y, gr[u].z, gr[u].w};
        const uint32_t uw[4] = {ur[u].x, ur[u].y, ur[u].z, ur[u].w};
        float y[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float g = __uint_as_float(j == 0 ? gw[i] << 16 : gw[i] & 0xFFFF0000u);
                const float up = __uint_as_float(j == 0 ? uw[i] << 16 : uw[i] & 0xFFFF0000u);
                // fast exponential and division (a few ulps; 0 for 1 + e^-g beyond 2^126,
                // the limit of silu there)
                y[2 * i + j] = __fdividef(g, 1.0f + __expf(-g)) * up;
            }
        }
        float amax = fabsf(y[0]);
#pragma unroll
        for (int i = 1; i < 8; ++i)
            amax = fmaxf(amax, fabsf(y[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)  // within the half-warp of this row
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        amax = fmaxf(amax, 1e-4f);
        const float factor = 448.0f / amax;
        const float scale = amax / 448.0f;
        if (valid[u]) {
            const uint32_t c01 = cvt_e4m3x2(y[0] * factor, y[1] * factor);
            const uint32_t c23 = cvt_e4m3x2(y[2] * factor, y[3] * factor);
            const uint32_t c45 = cvt_e4m3x2(y[4] * factor, y[5] * factor);
            const uint32_t c67 = cvt_e4m3x2(y[6] * factor, y[7] * factor);
            uint2 out;
            out.x = c01 | (c23 << 16);
            out.y = c45 | (c67 << 16);
            *reinterpret_cast<uint2 *>(q + static_cast<size_t>(row) * I + col) = out;
            if (hl == 0) {
                size_t idx;
                if (masked_m != nullptr) {
                    const int g = row / rows_per_group;
                    const int r = row - g * rows_per_group;
                    const int ld = (rows_per_group + 3) / 4 * 4;
                    idx = (static_cast<size_t>(g) * kbs + kb) * ld + r;
                } else {
                    idx = static_cast<size_t>(kb) * ((M + 3) / 4 * 4) + row;
                }
                sfa[idx] = scale;
            }
        }
    }
}

}  // namespace dg
