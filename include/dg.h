/*
 * dg.h -- C ABI of the B200 (sm_100a) FP8 block-scaled NT GEMM library.
 *
 * The operation (DeepSeek開源第三彈 -- the DeepGEMM release write-up -- sections
 * "深入了解DeepGEMM" and "如何使用"): an FP8 GEMM with fine-grained scaling taken from DeepSeek-V3,
 * in the NT layout (non-transposed left operand, transposed right operand), with bf16 output:
 *
 *     D[m][n] = sum_kb  sfa(m, kb) * sfb(n / 128, kb) * sum_{k in K-block kb} a[m][k] * b[n][k]
 *
 * a and b hold e4m3 codes (OCP FP8 E4M3, no infinities, max 448).  sfa is the fp32 scale of
 * each 1x128 tile of a (one per row and 128-wide K block), sfb the fp32 scale of each 128x128
 * block of b.  The product of each 128-wide K slice is formed on the tensor cores and then
 * scaled and added into an fp32 accumulator on the CUDA cores (the "two-level accumulation"
 * of "深入了解DeepGEMM"), then rounded to bf16 (round to nearest even).
 *
 * Conventions for every call below:
 *   - Every pointer is a DEVICE pointer owned by the caller.  The library never allocates,
 *     frees or synchronises on these calls; all work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL means the legacy default stream).
 *   - Base pointers must be 16-byte aligned.  K must be a positive multiple of 128 and N a
 *     positive multiple of 8 (16-byte output rows).
 *   - Return value: DG_OK (0) when the work was enqueued, otherwise a negative dg_status.
 *     Errors found before the launch (DG_ERR_INVALID_ARG, DG_ERR_UNSUPPORTED) launch
 *     nothing and leave d untouched.  DG_ERR_CUDA reports a failed launch.
 *   - Scales of a are stored MN-major ("TMA-aligned", see dg_get_tma_aligned_size): for each
 *     K block kb, the scales of all rows are contiguous, padded to a multiple of 4 rows:
 *       sfa[kb * align4(M) + m].
 *     Scales of b are row-major per 128-row block: sfb[nb * (K/128) + kb].
 *   - Device-side contract checks and the pipeline watchdog record an error word that
 *     dg_poll_device_error() reads (see there); they never trap.
 */
#ifndef DG_B200_DG_H
#define DG_B200_DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dg_status {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = -1, /* null/misaligned pointer, bad size, K % 128 != 0, N % 8 != 0 */
    DG_ERR_UNSUPPORTED = -2, /* no CUDA device, or the current device is not sm_100 */
    DG_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed (launch, tensor map) */
    DG_ERR_TIMEOUT = -4,     /* device: a pipeline wait exceeded its time limit */
    DG_ERR_WORKSPACE = -5,   /* workspace missing or smaller than dg_get_workspace_size() */
    DG_ERR_LAYOUT = -6       /* device: an index array broke its contract (see each call) */
} dg_status;

/* Dense GEMM, "gemm_fp8_fp8_bf16_nt" of "如何使用".
 *   a   e4m3 [M][K] row-major          sfa fp32 [K/128][align4(M)]  (MN-major)
 *   b   e4m3 [N][K] row-major          sfb fp32 [ceil(N/128)][K/128]
 *   d   bf16 [M][N] row-major (written: all M x N elements)
 * M >= 0 (M == 0 is a no-op).  workspace / workspace_bytes: used only by the stream-K kernel
 * (kernel family 5, M <= 64; see dg_get_workspace_size), which needs at least
 * dg_get_workspace_size(0, M, N, K, 1) bytes, 256-byte aligned and zero-filled before first use
 * (DG_ERR_WORKSPACE otherwise); other calls accept NULL / 0.  A workspace that is not 256-byte
 * aligned is DG_ERR_INVALID_ARG. */
int dg_gemm_fp8_fp8_bf16_nt(const void *a, const float *sfa, const void *b, const float *sfb,
                            void *d, int M, int N, int K, void *workspace,
                            size_t workspace_bytes, void *stream);

/* The dense GEMM of dg_gemm_fp8_fp8_bf16_nt for callers that cannot allocate device memory,
 * allocating nothing itself.  (The DeepGEMM pages have no counterpart: this is a calling
 * convention of this library.)  Some callers may not call cudaMalloc or any allocating routine
 * during their work: a serving loop whose device memory is planned and reserved up front, an
 * operator running inside another runtime that receives only its inputs and outputs, or code on
 * a latency-critical thread, where cudaMalloc can synchronise the device.  They cannot provide
 * the workspace the stream-K kernel needs (dg_get_workspace_size), so this entry runs that
 * kernel -- every SM streams an equal share of the K blocks -- with its scratch in an array
 * built into the library: a file-scope device array of 12 MiB that every GPU loading the
 * library holds until the process exits.
 *   Same arguments, layouts and results as dg_gemm_fp8_fp8_bf16_nt (without the workspace);
 *   takes dense calls with 1 <= M <= 64 whose tiles of 128 rows of B x K/128 number at least the
 *   SMs, and no more tiles than SMs (DG_ERR_UNSUPPORTED otherwise); DG_ERR_WORKSPACE when the
 *   partial sums would not fit the 12 MiB (with the 148 SMs of a B200: 9.25 MiB at M <= 64).
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress, once
 *   per device, with that device current); make that first call before any stream capture.
 *   Each call clears the array's tile counters on `stream` before its kernel.  Every call on a
 *   device shares the one array, which keeps the last call's contents: calls that overlap on the
 *   GPU (other streams, other host threads) race and must be serialised by the caller.
 *   M == 0 is a no-op. */
int dg_gemm_fp8_fp8_bf16_nt_noalloc(const void *a, const float *sfa, const void *b, const float *sfb,
                                    void *d, int M, int N, int K, void *stream);

/* Contiguous-layout grouped GEMM for MoE, "m_grouped_gemm_fp8_fp8_bf16_nt_contiguous" of
 * "如何使用" (the token rows of several experts are concatenated along M).
 *   a          e4m3 [M_total][K]          sfa fp32 [K/128][M_total]
 *   b          e4m3 [G][N][K]             sfb fp32 [G][ceil(N/128)][K/128]
 *   d          bf16 [M_total][N]
 *   m_indices  int32 [M_total] on the device: the expert of each row, in [0, G), or -1 for a
 *              padding row.  Rows with -1 are NOT written.
 * M_total must be a multiple of 128 and every aligned 128-row tile may hold rows of one
 * expert only (plus -1 rows): the segments of each expert are padded to 128 rows.  A tile
 * that breaks this, or an index outside [-1, G), sets DG_ERR_LAYOUT on the device and the
 * offending rows are not written.  G >= 1; M_total == 0 is a no-op. */
int dg_m_grouped_gemm_fp8_fp8_bf16_nt_contiguous(const void *a, const float *sfa, const void *b,
                                                 const float *sfb, void *d, const int *m_indices,
                                                 int M_total, int N, int K, int G,
                                                 void *workspace, size_t workspace_bytes,
                                                 void *stream);

/* Masked-layout grouped GEMM for MoE decoding, "m_grouped_gemm_fp8_fp8_bf16_nt_masked" of
 * "如何使用" (a fixed-size batch per expert of which only the first masked_m[g] rows hold
 * tokens).
 *   a          e4m3 [G][M_max][K]         sfa fp32 [G][K/128][align4(M_max)]
 *   b          e4m3 [G][N][K]             sfb fp32 [G][ceil(N/128)][K/128]
 *   d          bf16 [G][M_max][N]
 *   masked_m   int32 [G] on the device, 0 <= masked_m[g] <= M_max.  Rows r >= masked_m[g] of
 *              group g are NOT written.  A value outside [0, M_max] sets DG_ERR_LAYOUT and is
 *              clamped.
 *   expected_m host-side hint of the typical masked_m (used only to choose tiles; never
 *              changes results).  masked_m is read on the device only, so the call needs no
 *              host synchronisation.
 * 1 <= G <= 1024 (the device-side tile scheduler keeps a prefix sum per group), M_max >= 0
 * (M_max == 0 is a no-op), expected_m >= 0; DG_ERR_INVALID_ARG otherwise. */
int dg_m_grouped_gemm_fp8_fp8_bf16_nt_masked(const void *a, const float *sfa, const void *b,
                                             const float *sfb, void *d, const int *masked_m,
                                             int G, int M_max, int N, int K, int expected_m,
                                             void *workspace, size_t workspace_bytes,
                                             void *stream);

/* FP8 x FP4 variants: the mixed-precision "FP8 x FP4" matrix multiplication that the DeepGEMM
 * update news item ("Perpustakaan operator GPU sumber terbuka DeepSeek DeepGEMM memperbarui
 * versi besar ...") lists among the additions.  The item fixes neither the FP4 format, its
 * layout nor its scales; these calls take the plainest reading:
 *   - b holds OCP FP4 E2M1 values (sign, 2 exponent bits with bias 1, 1 mantissa bit; values
 *     +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}), packed two per byte along K: element k of a row is the
 *     low nibble of byte k/2 when k is even, the high nibble when k is odd.  A row of b is
 *     K/2 bytes; groups follow each other ([G][N][K/2] for the grouped calls).
 *   - sfb is unchanged: one fp32 scale per 128 x 128 block of b, [G][N/128][K/128].
 *   - a, sfa, d, m_indices, masked_m and every other rule are those of the FP8 x FP8 call of
 *     the same name, and the result is the same formula with b's E2M1 values in place of e4m3.
 * The tensor cores take e4m3 x e2m1 directly; nothing is converted in memory.  b must be 32-byte
 * aligned (DG_ERR_INVALID_ARG otherwise).  No workspace is used. */
int dg_gemm_fp8_fp4_bf16_nt(const void *a, const float *sfa, const void *b, const float *sfb,
                            void *d, int M, int N, int K, void *stream);

int dg_m_grouped_gemm_fp8_fp4_bf16_nt_contiguous(const void *a, const float *sfa, const void *b,
                                                 const float *sfb, void *d, const int *m_indices,
                                                 int M_total, int N, int K, int G, void *stream);

int dg_m_grouped_gemm_fp8_fp4_bf16_nt_masked(const void *a, const float *sfa, const void *b,
                                             const float *sfb, void *d, const int *masked_m, int G,
                                             int M_max, int N, int K, int expected_m, void *stream);

/* Per-token FP8 quantisation of activations: the step that produces the GEMMs' A operand and
 * its scales (the fine-grained 1 x 128 activation scaling of "深入了解DeepGEMM", written in the
 * TMA-aligned scale layout that the utility functions of "如何使用" serve).  For each row m and
 * K block kb, in fp32 with IEEE round-to-nearest-even operations:
 *     amax    = max(max |x[m][128 kb .. 128 kb + 127]|, 1e-4)
 *     scale   = amax / 448                     (written to sfa)
 *     q[m][k] = e4m3(x[m][k] * (448 / amax)), round to nearest even, saturating at +-448
 *   x    bf16 [M][K] row-major (device); finite values (NaN / inf give unspecified codes)
 *   q    e4m3 codes [M][K] row-major (device, written)
 *   sfa  fp32 [K/128][align4(M)], MN-major: the layout every GEMM here reads (device, written;
 *        the padding entries of rows M .. align4(M)-1 are not written)
 *   M >= 0 (0 launches nothing), K > 0 and K % 128 == 0, pointers 16-byte aligned, K/128 <=
 *   65535.  The caller owns all buffers; nothing is allocated; asynchronous on `stream`.
 * Returns DG_OK, DG_ERR_INVALID_ARG (nothing launched), DG_ERR_UNSUPPORTED or DG_ERR_CUDA. */
int dg_quantize_fp8_1x128(const void *x, void *q, float *sfa, int M, int K, void *stream);

/* SwiGLU followed by the same per-token FP8 quantisation: the step between the two grouped
 * GEMMs of an MoE layer ("如何使用": grouped GEMMs for MoE; the fused gate/up projection's bf16
 * output feeds the down projection's FP8 A operand).  Row m of h holds the gate half h[m][0:I]
 * and the up half h[m][I:2I]; in fp32
 *     y[m][i] = silu(g) * u,  silu(g) = g / (1 + exp(-g)),  g = h[m][i], u = h[m][I + i]
 * and y is quantised per 1 x 128 tile exactly as dg_quantize_fp8_1x128 does.
 *   h         bf16 [M][2I] row-major (device)
 *   q         e4m3 codes [M][I] row-major (device, written for processed rows)
 *   sfa       fp32 scales: without masked_m [I/128][align4(M)] (the dense / contiguous
 *             layout); with masked_m [G][I/128][align4(rows_per_group)] (the masked layout),
 *             G = M / rows_per_group
 *   masked_m  NULL (every row) or int32 [G] on the device: row r of group g (r = m mod
 *             rows_per_group) is processed only when r < masked_m[g]; other rows' q and sfa
 *             entries are not written
 *   M >= 0, I > 0 and I % 128 == 0, I/128 <= 65535, pointers 16-byte aligned; with masked_m,
 *   rows_per_group > 0 and M % rows_per_group == 0.  exp is the GPU's fast exponential, so y
 * can differ from an exact evaluation by a few fp32 ulps (codes can then differ by one step
 *   next to an e4m3 rounding midpoint).  Returns DG_OK, DG_ERR_INVALID_ARG (nothing
 *   launched), DG_ERR_UNSUPPORTED or DG_ERR_CUDA. */
int dg_swiglu_quantize_fp8_1x128(const void *h, void *q, float *sfa, int M, int I,
                                 const int *masked_m, int rows_per_group, void *stream);

/* The SM-count utility of "如何使用": caps the number of SMs the persistent kernels occupy so
 * that other work (for example communication kernels) can run beside them.  n <= 0 restores
 * "all SMs".  Returns the previous cap (0 = all). */
int dg_set_num_sms(int n);

/* Number of SMs the kernels will use on the current device (the cap, or all SMs).  Returns
 * DG_ERR_UNSUPPORTED when no device is present. */
int dg_get_num_sms(void);

/* The TMA-alignment utility of "如何使用": the smallest x' >= x such that x' * elem_bytes is a
 * multiple of 16 bytes (the tensor-memory-accelerator stride rule).  For the fp32 scales of
 * a this is align4(M).  Returns DG_ERR_INVALID_ARG for x < 0 or elem_bytes <= 0. */
int dg_get_tma_aligned_size(int x, int elem_bytes);

/* Bytes of workspace a call of `kind` (0 dense, 1 contiguous, 2 masked) with these sizes can
 * use on the current device; 0 means the call uses none.  Only the stream-K kernel (kernel
 * family 5 of dg_set_kernel_family, dense calls with M <= 64) uses one: every SM takes an equal
 * share of the K blocks, each writes its fp32 partial sums into the workspace, and the last
 * contributor of an output tile adds them in K order (deterministic) and writes D.  Automatic
 * mode never needs a workspace (it measured slower than the cluster kernels on B200, so it is
 * opt-in), and a call outside family 5 ignores one.  Layout, owned by the caller:
 * [SMs][2][TN][128] fp32 partial slots, then one int32 arrival counter per 128-row tile of B.
 * Zero-fill it before its first use; every call leaves the counters at zero again, except one
 * that reports DG_ERR_TIMEOUT (zero-fill it again then).  Calls that share a workspace must not
 * overlap on the GPU (use one per stream).  The size depends on the SM budget
 * (dg_set_num_sms). */
size_t dg_get_workspace_size(int kind, int M, int N, int K, int G);

/* Static, human-readable text for a dg_status value. */
const char *dg_status_string(int status);

/* Reads the device error word that contract checks and the pipeline watchdog set, resets it
 * to 0, and returns it (DG_OK, DG_ERR_TIMEOUT or DG_ERR_LAYOUT).  The read and the reset are
 * one atomic exchange on the device, enqueued on `stream`.  There is ONE word per device,
 * shared by the kernels of every stream and thread: an error is seen by the first poll that
 * runs after the kernel recorded it, whichever stream that poll is on, and a kernel still
 * running on another stream may record its error after this poll (synchronise the device, or
 * every stream that ran this library's kernels, before polling to see them all).  This call
 * SYNCHRONISES `stream`; it is meant for tests and debugging, not for the hot path. */
int dg_poll_device_error(void *stream);

/* Time limit, in nanoseconds, of every pipeline wait inside the kernels (default 2e9).
 * A wait that exceeds it sets DG_ERR_TIMEOUT on the device and the kernel winds down
 * (outstanding copies and tensor-core work are drained, tensor memory is freed) instead of
 * hanging.  0 restores the default.  Returns the previous value. */
unsigned long long dg_set_wait_timeout_ns(unsigned long long ns);

/* Test hook for the watchdog: mode 1 makes every following launch's MMA issuer first wait on a
 * barrier that nothing signals, so the wait runs out after the dg_set_wait_timeout_ns limit and
 * the kernel reports DG_ERR_TIMEOUT and winds down (no fault, no hang).  0 (default) turns it
 * off.  Returns the previous mode, or DG_ERR_INVALID_ARG. */
int dg_set_fault_injection(int mode);

/* Tuning/testing override of the tile choice: block_n in {32, 64, ..., 256} (the N extent of a
 * tile; 0 = heuristic), the number of shared-memory pipeline stages (0 = as many as fit) and the
 * number of K splits of the split-K kernel (1..8; 0 = heuristic).  Returns DG_ERR_INVALID_ARG
 * for unsupported values. */
int dg_set_config_override(int block_n, int num_stages, int splits);

/* Tuning/testing switch between the kernel families: 0 = automatic (default); 1 = the one-CTA
 * persistent kernels; 2 = the CTA-pair kernels (tcgen05 cta_group::2, 256-row tiles) wherever the
 * layout allows them (dense and masked; the contiguous layout always uses one-CTA tiles because
 * its expert segments are only 128-row aligned); 3 = the split-K cluster kernel for dense calls
 * whose output tiles fit in one wave (the K blocks of a tile are split over up to 8 CTAs that
 * reduce their fp32 partials through distributed shared memory, in a fixed order); 4 = the
 * swapped-operand kernel for dense calls with M <= 128 (B rows on the MMA's 128-row side, the
 * tokens on its N side, K split over a cluster as in 3; block_n 128 or 256 of
 * dg_set_config_override selects one or two 128-row blocks of B per tile), other calls run as
 * in automatic mode; 5 = the stream-K swapped-operand kernel for dense calls with M <= 64 (see
 * dg_get_workspace_size; DG_ERR_WORKSPACE when the call's workspace is missing or too small,
 * DG_ERR_UNSUPPORTED for shapes it does not take: fewer K blocks x tiles than SMs, more tiles
 * than SMs).  Automatic mode uses the swapped-operand kernel for dense M <= 64 with one
 * 128-row block of B per tile (when no block_n override is set), split-K for dense M <= 256 when
 * more than one split pays (else the one-CTA kernel), pairs for dense M > 256 with
 * K >= 96 * 128, and the one-CTA kernels otherwise (contiguous and masked included).  Results agree within the parity tolerance whichever
 * family runs.  Returns the previous value, or DG_ERR_INVALID_ARG. */
int dg_set_kernel_family(int family);

/* Programmatic dependent launch (a Hopper/Blackwell launch feature, not on the pages; on by
 * default).  When enabled, every GEMM is launched with programmatic stream serialisation: its
 * CTAs may be scheduled, and run their on-chip set-up (barrier initialisation, tensor-memory
 * allocation, tensor-map prefetch), while the previous kernel of the stream finishes; each kernel
 * signals its dependents at entry and executes griddepcontrol.wait before its first access to
 * global memory, so results and stream ordering are the same with the switch on or off.  The
 * overlap only happens between back-to-back kernels (an event or memcpy in between is a full
 * dependency).  enable: 0 or 1.  Returns the previous value, or DG_ERR_INVALID_ARG. */
int dg_set_pdl(int enable);

/* The cache of encoded TMA tensor maps (on by default).  Every GEMM call describes its operands
 * with two to four tensor maps; an entry is keyed on every argument of the encoding (element
 * type, base address, sizes, strides, box, swizzle, ...), so a hit is exactly the map that would
 * be encoded and repeated calls on the same buffers skip the encoding.  enable 0 turns it off
 * and drops every entry, 1 turns it on.  Returns the previous setting (0 or 1), or
 * DG_ERR_INVALID_ARG.  Host-side only; thread-safe. */
int dg_set_tensor_map_cache(int enable);

/* Hits and misses of the tensor-map cache since the library was loaded (NULL pointers are
 * skipped).  Returns DG_OK. */
int dg_get_tensor_map_cache_stats(unsigned long long *hits, unsigned long long *misses);

/* Describes the most recent launch on this host thread: fills any non-NULL pointer with the
 * chosen block_n, pipeline stages, grid size (CTAs), output tile count, kernel family (1 to 5
 * as in dg_set_kernel_family) and K splits per tile (for the stream-K kernel: the most K blocks
 * one CTA takes).  Returns DG_OK, or DG_ERR_INVALID_ARG
 * when nothing was launched yet. */
int dg_get_last_launch(int *block_n, int *num_stages, int *grid, int *num_tiles, int *family,
                       int *splits);

#ifdef __cplusplus
}
#endif

#endif /* DG_B200_DG_H */
