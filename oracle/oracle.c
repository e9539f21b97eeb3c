/*
 * oracle.c -- plain, slow, obviously correct CPU oracle for the FP8 block-scaled NT GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or execute this
 * file.  Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.  It
 * shares no code, header, table or constant generator with the CUDA library.
 *
 * What it computes (DeepGEMM release write-up, "深入了解DeepGEMM": an FP8 GEMM with
 * fine-grained scaling from DeepSeek-V3, in the NT layout of "如何使用", with the grouped
 * contiguous and masked layouts for MoE):
 *
 *   D[m][n] = bf16_rne( sum_{kb} sa[m][kb] * sb[n/128][kb] * S[m][n][kb] )
 *   S[m][n][kb] = sum_{k = 128 kb}^{128 kb + 127} e4m3(a[m][k]) * e4m3(b[n][k])
 *
 * a is M x K row-major (codes), b is N x K row-major (codes, "transposed RHS"),
 * sa is the fp32 scale of each 1x128 tile of a (logical [M][K/128]), sb the fp32 scale of
 * each 128x128 block of b (logical [ceil(N/128)][K/128]).  The real value of an element is
 * code * scale.  The outer sum runs in fp64 and is rounded ONCE to bf16, round-to-nearest-
 * even.  The inner slice sum S is exact in fp64: every e4m3 product has at most 8
 * significant bits and is a multiple of 2^-18, and 128 such terms stay below 2^25, so the
 * sum needs fewer than 53 bits and its value does not depend on the order of summation.
 *
 * The oracle also returns, per element, the fp64 value before rounding and the magnitude
 * sum  sum_k |sa a| |sb b|  that the parity tolerance is defined on.
 *
 * Grouped forms:
 *   contiguous: rows of several experts concatenated; m_indices[r] names the expert of row r,
 *               -1 marks a padding row, whose output is not written.
 *   masked:     a is [G][M_max][K]; only rows r < masked_m[g] of group g are written.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORC_BLOCK 128

/* ---- element formats --------------------------------------------------------------- */

/* OCP 8-bit floating point, E4M3 ("fn": no infinities).  Bit 7 is the sign, bits 6..3 the
 * exponent with bias 7, bits 2..0 the mantissa.  Exponent field 0 holds subnormals
 * (m/8) * 2^-6; exponent field 15 with mantissa 7 is NaN; every other code is normal,
 * (1 + m/8) * 2^(e-7), so the largest finite magnitude is 1.75 * 2^8 = 448. */
double orc_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* IEEE-754 round-to-nearest-even of a double to bfloat16 (1 sign, 8 exponent bits with
 * bias 127, 7 stored mantissa bits), returned as its bit pattern.  One rounding step:
 * the quantum at |x| is 2^(e-7) for a normal binade 2^e <= |x| < 2^(e+1), and 2^-133
 * below the smallest normal 2^-126.  Dividing by a power of two is exact, so the
 * rounding happens in rint() alone, which rounds half to even in the default mode. */
uint16_t orc_bf16_rne(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    if (isnan(x))
        return 0x7FC0;
    if (ax == 0.0)
        return sign;
    if (isinf(x))
        return sign | 0x7F80;
    int fe;
    frexp(ax, &fe);       /* ax = f * 2^fe, f in [0.5, 1) */
    int e = fe - 1;       /* 2^e <= ax < 2^(e+1) */
    double q = (e < -126) ? ldexp(1.0, -133) : ldexp(1.0, e - 7);
    double n = rint(ax / q);  /* integer number of quanta, ties to even */
    if (e < -126) {
        /* subnormal (or rounds up to the smallest normal when n == 128) */
        return sign | (uint16_t)n;
    }
    /* normal: n in [128, 256]; n == 256 carries into the next binade */
    int64_t bits = ((int64_t)(e + 127) << 7) + ((int64_t)n - 128);
    if (bits >= 0x7F80)
        return sign | 0x7F80; /* overflow to infinity */
    return sign | (uint16_t)bits;
}

/* IEEE-754 round-to-nearest-even of a float to E4M3 with saturation to the largest finite
 * magnitude (448): the conversion of the per-token quantisation below.  Written from the
 * format's definition: normal codes (1 + m/8) 2^(e-7) for e = 1..15 (e = 15 only m <= 6),
 * subnormal codes (m/8) 2^-6; the quantum is 2^-9 below 2^-6 and 2^(E-3) in binade E.  NaN in,
 * NaN code out; -0 keeps its sign. */
uint8_t orc_e4m3_encode(float v)
{
    if (v != v)
        return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0)
        return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: multiples of 2^-9; q = 8 is the smallest normal, code 0x08 */
        const double q = rint(ldexp(a, 9));
        return sign | (uint8_t)q;
    }
    int e;
    frexp(a, &e);             /* a = f 2^e, f in [0.5, 1): binade E = e - 1 */
    int E = e - 1;
    double q = rint(ldexp(a, 3 - E));   /* in [8, 16] */
    if (q >= 16.0) {
        q = 8.0;
        E += 1;
    }
    const int code = ((E + 7) << 3) | ((int)q - 8);
    return sign | (uint8_t)(code > 0x7E ? 0x7E : code);
}

/* OCP 4-bit floating point E2M1 (the FP4 of the FP8 x FP4 GEMM that the DeepGEMM update news
 * item, "Perpustakaan operator GPU sumber terbuka DeepSeek DeepGEMM memperbarui versi besar",
 * lists among the additions): bit 3 the sign, bits 2..1 the exponent (bias 1), bit 0 the mantissa; exponent 0 is
 * subnormal (m / 2).  Values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}; no infinities or NaN. */
double orc_e2m1_decode(uint8_t nibble)
{
    const int s = (nibble >> 3) & 1, e = (nibble >> 1) & 3, m = nibble & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Expands packed E2M1 rows (two elements per byte, element 2j in the low nibble of byte j)
 * into E4M3 codes of the same values -- every E2M1 value is an E4M3 value -- so the FP8 x FP4
 * GEMM is the FP8 GEMM of the expanded operand.  packed [rows][K/2] -> codes [rows][K]. */
void orc_e2m1_to_e4m3(const uint8_t *packed, int64_t rows, int64_t K, uint8_t *codes)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            const uint8_t byte = packed[r * (K / 2) + k / 2];
            const uint8_t nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
            codes[r * K + k] = orc_e4m3_encode((float)orc_e2m1_decode(nib));
        }
}

/* ---- per-token (1 x 128) FP8 quantisation of bf16 activations ------------------------- */

/* The step before the GEMM (DeepGEMM release write-up, "深入了解DeepGEMM": activations carry
 * one scale per 1 x 128 tile).  For each row m and K block kb, in fp32:
 *     amax   = max(max |x| over the tile, 1e-4)
 *     factor = 448 / amax                 (one division per tile)
 *     scale  = amax / 448                 (the dequantisation scale the GEMM reads)
 *     q[k]   = e4m3_rne(x[k] * factor)    (saturating at 448)
 * x is bf16 bits [M][K]; q codes [M][K]; sa the logical scales [M][K/128].  Every step is a
 * single fp32 operation rounded to nearest even, as the GPU kernel computes it, so the integer
 * codes and the scales can be compared bit for bit. */
int orc_quantize_1x128(const uint16_t *x, int64_t M, int64_t K, uint8_t *q, float *sa)
{
    if (K % ORC_BLOCK != 0 || M < 0)
        return -1;
    const int64_t kbs = K / ORC_BLOCK;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t kb = 0; kb < kbs; ++kb) {
            const uint16_t *xt = x + m * K + kb * ORC_BLOCK;
            float vals[ORC_BLOCK];
            float amax = 0.0f;
            for (int i = 0; i < ORC_BLOCK; ++i) {
                uint32_t w = (uint32_t)xt[i] << 16;  /* bf16 -> fp32 is exact */
                float f;
                memcpy(&f, &w, 4);
                vals[i] = f;
                const float a = fabsf(f);
                if (a > amax)
                    amax = a;
            }
            const float amax_c = amax > 1e-4f ? amax : 1e-4f;
            const float factor = 448.0f / amax_c;
            sa[m * kbs + kb] = amax_c / 448.0f;
            for (int i = 0; i < ORC_BLOCK; ++i)
                q[m * K + kb * ORC_BLOCK + i] = orc_e4m3_encode(vals[i] * factor);
        }
    }
    return 0;
}

/* ---- SwiGLU followed by the per-token FP8 quantisation --------------------------------- */

/* Between the two grouped GEMMs of an MoE layer (the fused gate/up projection, then the down
 * projection; DeepGEMM release write-up, "如何使用": grouped GEMMs for MoE), each token row of
 * the first GEMM's bf16 output h [M][2I] holds the gate half h[:, 0:I] and the up half
 * h[:, I:2I].  The activation is
 *     y[m][i] = silu(g) * u,  silu(g) = g / (1 + exp(-g)),  g = h[m][i], u = h[m][I + i]
 * computed here in fp64 and rounded once to fp32 (y32, returned for the tests), then
 * quantised exactly as orc_quantize_1x128 does (fp32 amax, factor 448 / amax, scale amax / 448,
 * e4m3 round to nearest even).  Rows with row_valid[m] == 0 (NULL: all valid) are skipped and
 * their outputs left untouched.  q [M][I], sa [M][I/128], y32 [M][I] (may be NULL). */
int orc_swiglu_quantize(const uint16_t *h, int64_t M, int64_t I, const uint8_t *row_valid,
                        uint8_t *q, float *sa, float *y32)
{
    if (I % ORC_BLOCK != 0 || M < 0)
        return -1;
    const int64_t kbs = I / ORC_BLOCK;
    for (int64_t m = 0; m < M; ++m) {
        if (row_valid && !row_valid[m])
            continue;
        for (int64_t kb = 0; kb < kbs; ++kb) {
            float vals[ORC_BLOCK];
            float amax = 0.0f;
            for (int i = 0; i < ORC_BLOCK; ++i) {
                const int64_t col = kb * ORC_BLOCK + i;
                uint32_t wg = (uint32_t)h[m * 2 * I + col] << 16;
                uint32_t wu = (uint32_t)h[m * 2 * I + I + col] << 16;
                float g, u;
                memcpy(&g, &wg, 4);
                memcpy(&u, &wu, 4);
                const double y = (double)g / (1.0 + exp(-(double)g)) * (double)u;
                const float yf = (float)y;
                vals[i] = yf;
                if (y32)
                    y32[m * I + col] = yf;
                const float a = fabsf(yf);
                if (a > amax)
                    amax = a;
            }
            const float amax_c = amax > 1e-4f ? amax : 1e-4f;
            const float factor = 448.0f / amax_c;
            sa[m * kbs + kb] = amax_c / 448.0f;
            for (int i = 0; i < ORC_BLOCK; ++i)
                q[m * I + kb * ORC_BLOCK + i] = orc_e4m3_encode(vals[i] * factor);
        }
    }
    return 0;
}

/* ---- one output row ------------------------------------------------------------------ */

typedef struct {
    const double *lut;   /* e4m3 code -> value */
    const uint8_t *b;    /* [N][K] codes of the B matrix this row multiplies */
    const float *sb;     /* [ceil(N/128)][K/128] */
    int64_t N, K;
} orc_bmat;

/* Computes one row of D from one row of A (codes a_row[K], scales sa_row[K/128]).
 * Writes n in [0, N) of out_bits / out_acc / out_abs (the latter two may be NULL). */
static void orc_row(const orc_bmat *bm, const uint8_t *a_row, const float *sa_row,
                    double *a_dec, uint16_t *out_bits, double *out_acc, double *out_abs)
{
    const int64_t K = bm->K, N = bm->N, Kb = K / ORC_BLOCK;
    for (int64_t k = 0; k < K; ++k)
        a_dec[k] = bm->lut[a_row[k]];
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *b_row = bm->b + n * K;
        const float *sb_row = bm->sb + (n / ORC_BLOCK) * Kb;
        double acc = 0.0, mag = 0.0;
        for (int64_t kb = 0; kb < Kb; ++kb) {
            double s = 0.0, s_abs = 0.0;
            for (int64_t k = kb * ORC_BLOCK; k < (kb + 1) * ORC_BLOCK; ++k) {
                double p = a_dec[k] * bm->lut[b_row[k]];
                s += p;
                s_abs += fabs(p);
            }
            double scale = (double)sa_row[kb] * (double)sb_row[kb];
            acc += scale * s;
            mag += fabs(scale) * s_abs;
        }
        out_bits[n] = orc_bf16_rne(acc);
        if (out_acc)
            out_acc[n] = acc;
        if (out_abs)
            out_abs[n] = mag;
    }
}

/* ---- row jobs and threads -------------------------------------------------------------- */

/* A job is a list of "tasks": (A row pointer, scale row pointer, B matrix, output slot). */
typedef struct {
    const uint8_t *a_row;
    const float *sa_row;
    int64_t group;    /* which B matrix */
    int64_t out_row;  /* row index in the output arrays */
} orc_task;

typedef struct {
    const orc_task *tasks;
    int64_t begin, end;
    const orc_bmat *bmats;
    uint16_t *out_bits;
    double *out_acc, *out_abs;
    int64_t N, K;
} orc_slice;

static void *orc_worker(void *arg)
{
    orc_slice *sl = (orc_slice *)arg;
    double *a_dec = (double *)malloc(sizeof(double) * (size_t)sl->K);
    if (!a_dec)
        return (void *)1;
    for (int64_t t = sl->begin; t < sl->end; ++t) {
        const orc_task *tk = &sl->tasks[t];
        int64_t o = tk->out_row * sl->N;
        orc_row(&sl->bmats[tk->group], tk->a_row, tk->sa_row, a_dec, sl->out_bits + o,
                sl->out_acc ? sl->out_acc + o : NULL, sl->out_abs ? sl->out_abs + o : NULL);
    }
    free(a_dec);
    return NULL;
}

static int orc_run(const orc_task *tasks, int64_t n_tasks, const orc_bmat *bmats, int64_t N,
                   int64_t K, uint16_t *out_bits, double *out_acc, double *out_abs, int n_threads)
{
    if (n_threads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = c > 0 ? (int)c : 1;
    }
    if (n_threads > n_tasks)
        n_threads = n_tasks > 0 ? (int)n_tasks : 1;
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    orc_slice *sl = (orc_slice *)calloc((size_t)n_threads, sizeof(orc_slice));
    if (!th || !sl) {
        free(th);
        free(sl);
        return -1;
    }
    int rc = 0;
    for (int i = 0; i < n_threads; ++i) {
        sl[i].tasks = tasks;
        sl[i].begin = n_tasks * i / n_threads;
        sl[i].end = n_tasks * (i + 1) / n_threads;
        sl[i].bmats = bmats;
        sl[i].out_bits = out_bits;
        sl[i].out_acc = out_acc;
        sl[i].out_abs = out_abs;
        sl[i].N = N;
        sl[i].K = K;
        if (pthread_create(&th[i], NULL, orc_worker, &sl[i]) != 0) {
            n_threads = i;
            rc = -1;
            break;
        }
    }
    for (int i = 0; i < n_threads; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret)
            rc = -1;
    }
    free(th);
    free(sl);
    return rc;
}

static void orc_lut(double lut[256])
{
    for (int c = 0; c < 256; ++c)
        lut[c] = orc_e4m3_decode((uint8_t)c);
}

/* ---- public entry points ---------------------------------------------------------------- */

/* Dense GEMM on a chosen list of rows of A.
 * a [M][K] codes, sa [M][K/128], b [N][K] codes, sb [ceil(N/128)][K/128].
 * rows[i] (0 <= rows[i] < M) is computed into output row i: out_bits [n_rows][N] (bf16 bits),
 * out_acc / out_abs [n_rows][N] fp64 (may be NULL).  Returns 0, or -1 on bad arguments. */
int orc_gemm_dense_rows(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                        int64_t M, int64_t N, int64_t K, const int64_t *rows, int64_t n_rows,
                        uint16_t *out_bits, double *out_acc, double *out_abs, int n_threads)
{
    if (K <= 0 || K % ORC_BLOCK != 0 || N <= 0 || M < 0 || n_rows < 0)
        return -1;
    double lut[256];
    orc_lut(lut);
    const int64_t Kb = K / ORC_BLOCK;
    orc_bmat bm = {lut, b, sb, N, K};
    orc_task *tasks = (orc_task *)calloc((size_t)(n_rows > 0 ? n_rows : 1), sizeof(orc_task));
    if (!tasks)
        return -1;
    for (int64_t i = 0; i < n_rows; ++i) {
        if (rows[i] < 0 || rows[i] >= M) {
            free(tasks);
            return -1;
        }
        tasks[i].a_row = a + rows[i] * K;
        tasks[i].sa_row = sa + rows[i] * Kb;
        tasks[i].group = 0;
        tasks[i].out_row = i;
    }
    int rc = orc_run(tasks, n_rows, &bm, N, K, out_bits, out_acc, out_abs, n_threads);
    free(tasks);
    return rc;
}

/* Dense GEMM over all rows: out_bits [M][N]. */
int orc_gemm_dense(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                   int64_t M, int64_t N, int64_t K, uint16_t *out_bits, double *out_acc,
                   double *out_abs, int n_threads)
{
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)(M > 0 ? M : 1));
    if (!rows)
        return -1;
    for (int64_t m = 0; m < M; ++m)
        rows[m] = m;
    int rc = orc_gemm_dense_rows(a, sa, b, sb, M, N, K, rows, M, out_bits, out_acc, out_abs,
                                 n_threads);
    free(rows);
    return rc;
}

/* Contiguous grouped GEMM.  a [M_total][K], sa [M_total][K/128], b [G][N][K],
 * sb [G][ceil(N/128)][K/128], m_indices [M_total] in [0, G) or -1.
 * Row r with m_indices[r] = g >= 0 is written to out row r (out_* are [M_total][N]);
 * rows with -1 are left as the caller filled them.  If rows != NULL only the listed rows are
 * considered.  Returns -1 on bad arguments (including an index >= G or < -1). */
int orc_gemm_contiguous(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                        const int32_t *m_indices, int64_t M_total, int64_t N, int64_t K,
                        int64_t G, const int64_t *rows, int64_t n_rows, uint16_t *out_bits,
                        double *out_acc, double *out_abs, int n_threads)
{
    if (K <= 0 || K % ORC_BLOCK != 0 || N <= 0 || M_total < 0 || G <= 0)
        return -1;
    double lut[256];
    orc_lut(lut);
    const int64_t Kb = K / ORC_BLOCK, Nb = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    orc_bmat *bm = (orc_bmat *)calloc((size_t)G, sizeof(orc_bmat));
    int64_t cnt = rows ? n_rows : M_total;
    orc_task *tasks = (orc_task *)calloc((size_t)(cnt > 0 ? cnt : 1), sizeof(orc_task));
    if (!bm || !tasks) {
        free(bm);
        free(tasks);
        return -1;
    }
    for (int64_t g = 0; g < G; ++g) {
        bm[g].lut = lut;
        bm[g].b = b + g * N * K;
        bm[g].sb = sb + g * Nb * Kb;
        bm[g].N = N;
        bm[g].K = K;
    }
    int64_t n_tasks = 0;
    for (int64_t i = 0; i < cnt; ++i) {
        int64_t r = rows ? rows[i] : i;
        if (r < 0 || r >= M_total)
            goto bad;
        int32_t g = m_indices[r];
        if (g < -1 || g >= G)
            goto bad;
        if (g < 0)
            continue; /* padding row: not written */
        tasks[n_tasks].a_row = a + r * K;
        tasks[n_tasks].sa_row = sa + r * Kb;
        tasks[n_tasks].group = g;
        tasks[n_tasks].out_row = r;
        ++n_tasks;
    }
    int rc = orc_run(tasks, n_tasks, bm, N, K, out_bits, out_acc, out_abs, n_threads);
    free(bm);
    free(tasks);
    return rc;
bad:
    free(bm);
    free(tasks);
    return -1;
}

/* Masked grouped GEMM.  a [G][M_max][K], sa [G][M_max][K/128], b [G][N][K],
 * sb [G][ceil(N/128)][K/128], masked_m [G] with 0 <= masked_m[g] <= M_max.
 * Row r < masked_m[g] of group g goes to out row g*M_max + r (out_* are [G][M_max][N]);
 * other rows are left as the caller filled them.  If rows != NULL, rows[i] are flattened
 * indices g*M_max + r and only those are considered. */
int orc_gemm_masked(const uint8_t *a, const float *sa, const uint8_t *b, const float *sb,
                    const int32_t *masked_m, int64_t G, int64_t M_max, int64_t N, int64_t K,
                    const int64_t *rows, int64_t n_rows, uint16_t *out_bits, double *out_acc,
                    double *out_abs, int n_threads)
{
    if (K <= 0 || K % ORC_BLOCK != 0 || N <= 0 || M_max < 0 || G <= 0)
        return -1;
    for (int64_t g = 0; g < G; ++g)
        if (masked_m[g] < 0 || masked_m[g] > M_max)
            return -1;
    double lut[256];
    orc_lut(lut);
    const int64_t Kb = K / ORC_BLOCK, Nb = (N + ORC_BLOCK - 1) / ORC_BLOCK;
    orc_bmat *bm = (orc_bmat *)calloc((size_t)G, sizeof(orc_bmat));
    int64_t cnt = rows ? n_rows : G * M_max;
    orc_task *tasks = (orc_task *)calloc((size_t)(cnt > 0 ? cnt : 1), sizeof(orc_task));
    if (!bm || !tasks) {
        free(bm);
        free(tasks);
        return -1;
    }
    for (int64_t g = 0; g < G; ++g) {
        bm[g].lut = lut;
        bm[g].b = b + g * N * K;
        bm[g].sb = sb + g * Nb * Kb;
        bm[g].N = N;
        bm[g].K = K;
    }
    int64_t n_tasks = 0;
    for (int64_t i = 0; i < cnt; ++i) {
        int64_t flat = rows ? rows[i] : i;
        if (flat < 0 || flat >= G * M_max) {
            free(bm);
            free(tasks);
            return -1;
        }
        int64_t g = flat / M_max, r = flat % M_max;
        if (r >= masked_m[g])
            continue; /* beyond the valid count: not written */
        tasks[n_tasks].a_row = a + flat * K;
        tasks[n_tasks].sa_row = sa + flat * Kb;
        tasks[n_tasks].group = g;
        tasks[n_tasks].out_row = flat;
        ++n_tasks;
    }
    int rc = orc_run(tasks, n_tasks, bm, N, K, out_bits, out_acc, out_abs, n_threads);
    free(bm);
    free(tasks);
    return rc;
}
