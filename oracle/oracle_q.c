/*
 * Oracle: GGUF block dequantisation and quantised GEMV in f64.
 *
 * TEST INFRASTRUCTURE ONLY.  This file belongs to the plain CPU oracle that the
 * CUDA path is checked against.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or constant with the CUDA library.
 *
 * What it computes, and where the pages fix it:
 *  - Weights are GGUF Q4_0 blocks (4-bit values with an f16 scale, SwarmLLM
 *    README on "Peer-to-peer LLM inference in browser tabs, Qwen 3.8 27B",
 *    paragraph after the peer diagram; model table "GGUF Q4_0") or GGUF Q8_0
 *    blocks (same README, model table "GGUF Q8_0 / Q4_0"; ChatTorrent README,
 *    "What it can run": f32, f16 and q8 weights are supported).
 *  - Q4_0 block: binary16 scale d (little endian) then 16 bytes; element j
 *    (j < 16) is the low nibble of byte j, element j+16 its high nibble;
 *    weight = (nibble - 8) * d.  Q8_0 block: binary16 d then 32 signed bytes;
 *    weight = q * d.  Block b of a row covers input columns 32b .. 32b+31.
 *  - A projection is y = x W^T, so one token streams the whole weight set a
 *    single time (same README, paragraph after the peer diagram).
 *
 * Everything is done in double precision, in the plain order of the
 * definitions: each output is one sequential dot product over the input
 * columns.  Output rows are independent, so OpenMP spreads rows over threads;
 * that changes no sum.  Compiled without fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <omp.h>

enum { ORC_Q4_0 = 2, ORC_Q8_0 = 8 };

/* IEEE 754 binary16 -> double, from the format's definition: sign bit,
 * 5-bit exponent with bias 15, 10-bit fraction; exponent 0 is subnormal
 * (fraction * 2^-24), exponent 31 is inf/nan. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* Element-wise binary16 -> double over an array (for checking the decoder). */
void orc_f16_array(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_f16_to_f64(h[i]);
}

static int block_bytes(int qtype)
{
    return qtype == ORC_Q4_0 ? 18 : qtype == ORC_Q8_0 ? 34 : 0;
}

/* Dequantise one 32-weight block into w[0..31]. */
static void dequant_block(int qtype, const uint8_t *blk, double *w)
{
    double d = orc_f16_to_f64((uint16_t)(blk[0] | (blk[1] << 8)));
    const uint8_t *qs = blk + 2;
    if (qtype == ORC_Q4_0) {
        for (int j = 0; j < 16; ++j) {
            w[j] = (double)((int)(qs[j] & 0x0f) - 8) * d;
            w[j + 16] = (double)((int)(qs[j] >> 4) - 8) * d;
        }
    } else {
        for (int j = 0; j < 32; ++j)
            w[j] = (double)(int8_t)qs[j] * d;
    }
}

/* Dequantise a whole [rows, cols] matrix of blocks into out[rows*cols].
 * Returns 0, or -1 on a bad argument. */
int orc_dequant(int qtype, const uint8_t *blocks, int64_t rows, int64_t cols, double *out)
{
    int bb = block_bytes(qtype);
    if (!bb || cols % 32 || rows < 0)
        return -1;
    int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b)
            dequant_block(qtype, blocks + (r * nb + b) * bb, out + r * cols + b * 32);
    return 0;
}

/* y[t][r] = sum_c W[r][c] * x[t][c] for t < n, r < rows; x is [n][cols],
 * y is [n][rows].  Each sum runs over c = 0 .. cols-1 in order. */
int orc_qgemv(int qtype, const uint8_t *blocks, int64_t rows, int64_t cols,
              const double *x, int n, double *y)
{
    int bb = block_bytes(qtype);
    if (!bb || cols % 32 || rows < 0 || n < 0)
        return -1;
    int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double w[32];
        double acc[64];
        for (int t0 = 0; t0 < n; t0 += 64) {
            int tn = n - t0 < 64 ? n - t0 : 64;
            for (int t = 0; t < tn; ++t)
                acc[t] = 0.0;
            for (int64_t b = 0; b < nb; ++b) {
                dequant_block(qtype, blocks + (r * nb + b) * bb, w);
                for (int t = 0; t < tn; ++t) {
                    const double *xt = x + (int64_t)(t0 + t) * cols + b * 32;
                    double a = acc[t];
                    for (int j = 0; j < 32; ++j)
                        a += w[j] * xt[j];
                    acc[t] = a;
                }
            }
            for (int t = 0; t < tn; ++t)
                y[(int64_t)(t0 + t) * rows + r] = acc[t];
        }
    }
    return 0;
}

int orc_threads(void)
{
    return omp_get_max_threads();
}
