/*
 * Plain CPU oracle for the nested r-bit GEMM (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg call
 * this code.  It shares nothing with the CUDA library: no header, no table,
 * no helper.  It is written for obviousness, not speed: every loop follows
 * the definition directly.
 *
 * Definitions followed (MatGPTQ, "Efficient and Accurate Inference over
 * Nested Quantized Models", abstract: lower-precision models are read from
 * the higher-precision parent by reading fewer bits, and an r-bit model reads
 * exactly r bits; MatGPTQ author page abstract: the most significant bits
 * are sliced at inference time):
 *
 *   slice:   q_r = q >> (8 - r)                         (top r bits of q)
 *   level:   v_r = 2^(8-r) * q_r + 2^(7-r) - 128
 *   weight:  w[n,k] = s16[n, k/128] * v_r[n,k]
 *   output:  Y[m,n] = sum_k X[m,k] * w[n,k]   (fp64, ascending k)
 *
 * Bit-plane layout (the exact-r-bit storage, the library's own format: the
 * pages fix no layout).  Rows are padded with zero rows to N128, a multiple
 * of 128; G = K / 128.  The buffer is 8 planes of N128*K/32 uint32 words,
 * plane p holding bit (7 - p) of the parent code (most significant plane
 * first), so an r-bit model is the first r planes.  Inside a plane the
 * 128-row x 128-column block (t, g) occupies the 512 words starting at
 * (t*G + g)*512; row i of the block is words 4i .. 4i+3, and bit j of word w
 * of that row holds the code at column 128g + 32w + j.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>

static int64_t rows128(int64_t N) { return (N + 127) / 128 * 128; }

/* Word index of (plane p, row n, column k) in the tiled layout. */
static int64_t word_at(int p, int64_t n, int64_t k, int64_t N, int64_t K)
{
    int64_t G = K / 128;
    int64_t plane = rows128(N) * (K / 32);
    return p * plane + ((n / 128) * G + k / 128) * 512 + (n % 128) * 4 + (k % 128) / 32;
}

/* Build the 8 planes bit by bit from the parent codes (padding rows zero). */
void oracle_pack(const uint8_t *codes, int64_t N, int64_t K, uint32_t *planes)
{
    memset(planes, 0, (size_t)8 * rows128(N) * (K / 32) * sizeof(uint32_t));
    for (int p = 0; p < 8; ++p) {
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k) {
                uint8_t q = codes[n * K + k];
                uint32_t bit = (q >> (7 - p)) & 1u;
                planes[word_at(p, n, k, N, K)] |= bit << (k % 32);
            }
        }
    }
}

/* Read back the r-bit codes q_r from the first r planes. */
void oracle_unpack(const uint32_t *planes, int64_t N, int64_t K, int r,
                   uint8_t *codes_r)
{
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            unsigned q = 0;
            for (int p = 0; p < r; ++p) {
                uint32_t word = planes[word_at(p, n, k, N, K)];
                unsigned bit = (word >> (k % 32)) & 1u;
                q = (q << 1) | bit;      /* plane 0 is the most significant */
            }
            codes_r[n * K + k] = (uint8_t)q;
        }
    }
}

/* The dequantized level of an r-bit code, exactly, in fp64. */
static double level(unsigned q_r, int r)
{
    double a = (double)(1u << (8 - r));                 /* 2^(8-r) */
    double b = (r == 8) ? 0.5 : (double)(1u << (7 - r)); /* 2^(7-r) */
    return a * (double)q_r + b - 128.0;
}

/*
 * Y[m, n] for every (m, n): X is M x K (bf16 values widened to fp64),
 * codes N x K (parent, 8-bit), s16 N x (K/128) (the fp16-stored scales
 * widened to fp64).  The r-bit slice is taken inside.
 */
void oracle_gemm_f64(const double *X, const uint8_t *codes, const double *s16,
                     int64_t M, int64_t N, int64_t K, int r, double *Y)
{
    int64_t G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                unsigned q_r = (unsigned)codes[n * K + k] >> (8 - r);
                double w = s16[n * G + k / 128] * level(q_r, r);
                acc += X[m * K + k] * w;
            }
            Y[m * N + n] = acc;
        }
    }
}

/* The same definition for a list of (m, n) output positions only. */
void oracle_gemm_f64_at(const double *X, const uint8_t *codes,
                        const double *s16, int64_t K, int r,
                        int64_t count, const int64_t *ms, const int64_t *ns,
                        double *out)
{
    int64_t G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            unsigned q_r = (unsigned)codes[n * K + k] >> (8 - r);
            double w = s16[n * G + k / 128] * level(q_r, r);
            acc += X[m * K + k] * w;
        }
        out[i] = acc;
    }
}

/*
 * Asymmetric variant (MatGPTQ paper page, captions of Tables 4-7:
 * "asymmetric MatGPTQ"; the pages give no formula, the reading taken: each
 * 128-column group also has a zero point z, real-valued in units of the
 * 8-bit code and stored as fp16, shared by every r like the scale):
 *
 *   level:   u_r = 2^(8-r) * q_r + 2^(7-r) - z16[n, k/128]
 *   weight:  w[n,k] = s16[n, k/128] * u_r[n,k]
 *
 * z = 128 gives the symmetric level v_r above.
 */
static double level_asym(unsigned q_r, int r, double z)
{
    double a = (double)(1u << (8 - r));                 /* 2^(8-r) */
    double b = (r == 8) ? 0.5 : (double)(1u << (7 - r)); /* 2^(7-r) */
    return a * (double)q_r + b - z;
}

void oracle_gemm_asym_f64(const double *X, const uint8_t *codes, const double *s16,
                          const double *z16, int64_t M, int64_t N, int64_t K, int r,
                          double *Y)
{
    int64_t G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                unsigned q_r = (unsigned)codes[n * K + k] >> (8 - r);
                double w = s16[n * G + k / 128] * level_asym(q_r, r, z16[n * G + k / 128]);
                acc += X[m * K + k] * w;
            }
            Y[m * N + n] = acc;
        }
    }
}

void oracle_gemm_asym_f64_at(const double *X, const uint8_t *codes, const double *s16,
                             const double *z16, int64_t K, int r, int64_t count,
                             const int64_t *ms, const int64_t *ns, double *out)
{
    int64_t G = K / 128;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            unsigned q_r = (unsigned)codes[n * K + k] >> (8 - r);
            double w = s16[n * G + k / 128] * level_asym(q_r, r, z16[n * G + k / 128]);
            acc += X[m * K + k] * w;
        }
        out[i] = acc;
    }
}

/* Number of OpenMP threads the gemm loops use (1 without OpenMP). */
int oracle_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
