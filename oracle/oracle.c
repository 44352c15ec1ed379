/*
 * oracle.c -- CPU oracle for the emulated RCCLX collectives.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg, never by the library.  It is deliberately
 * plain: one thread, no blocking, no vectorisation, no reassociation.  Build
 * with `-O2 -ffp-contract=off` and without fast-math so that every `a op b`
 * on floats below is one correctly rounded IEEE binary32 operation.
 *
 * What is computed, and where it comes from
 * -----------------------------------------
 * Sources (web pages about Meta's RCCLX, quoted by title and section):
 *   [DDA-es]  RCCLX post, Spanish copy (athrundataintelligence.com),
 *             "Ataque directo a datos (DDA): colectivos ligeros adentro del nodo"
 *   [LP-es]   same post, "Colectivos de mengua precisión"
 *   [DDA-pt]  "Meta open-sources RCCLX" summary (dev.infolabhq.com/pt),
 *             "Direct Data Access (DDA) — De O(N) para O(1) de Latência"
 *   [LP-pt]   same summary, "Coletivos de Baixa Precisão — Compressão FP8 com
 *             Precisão FP32"
 *   [API-pt]  same summary, "Primeiros Passos com Torchcomms"
 *
 * - DDA-flat [DDA-pt, DDA-es]: every rank reads the buffers of all ranks and
 *   reduces them itself, so every rank ends with the full SUM.
 * - DDA-tree [DDA-pt, DDA-es]: the allreduce is split into a reduce-scatter
 *   phase (rank c reduces chunk c of every rank's buffer) followed by an
 *   all-gather phase (every rank fetches every reduced chunk).
 * - Low-precision collectives [LP-es, LP-pt]: AllReduce, AllGather, AlltoAll
 *   and ReduceScatter on FP32 or BF16 data; what travels is FP8 (up to 4:1
 *   smaller than FP32), every arithmetic step is FP32, and precision is lost
 *   only at the quantisations (one or two per collective).
 *
 * Readings fixed by this library where the pages say only "FP8":
 *   - format OCP E4M3 "fn" (max finite 448, no infinities);
 *   - one fp32 scale per block of 128 consecutive elements, blocks anchored at
 *     the first element of the segment a sender quantises;
 *   - scale s = fl32(amax / 448), amax = max |x| over the block;
 *   - code = e4m3 round-to-nearest-even of fl32(x / s), saturating at +-448;
 *     the sign is kept, so -0 and tiny negatives give code 0x80;
 *   - s == 0 (all-zero block or underflow) stores scale 0 and codes +-0;
 *   - dequantised value = fl32(e4m3_value(code) * s);
 *   - every emulated wire hop quantises, including a rank's own contribution
 *     (so all ranks end bit-identical): flat FP8 quantises once, tree FP8 twice
 *     (the reduced chunk is quantised again before the all-gather);
 *   - SUM order is rank 0, 1, ..., N-1 from the first term: acc = w(x_0),
 *     acc = fl32(acc + w(x_s));
 *   - bf16 inputs widen exactly to fp32; bf16 outputs are one round-to-nearest-
 *     even of the fp32 result;
 *   - tree chunks hold C = 128 * ceil(ceil(count / 128) / N) elements, so FP8
 *     blocks never straddle a chunk;
 *   - with one rank nothing crosses a wire: every collective is a copy.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 128
#define ORC_E4M3_MAX 448.0f

/* ------------------------------------------------------------------ bits */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static size_t elem_size(int dtype) { return dtype == ORC_BF16 ? 2 : 4; }

/* ------------------------------------------------------------ e4m3 codec */

/* Value of an E4M3 code: sign bit 7, exponent bits 6..3 (bias 7), mantissa
 * bits 2..0.  Exponent 0 is subnormal: m * 2^-9; otherwise (8 + m) * 2^(e-10).
 * Codes 0x7F and 0xFF are NaN. */
float orc_e4m3_value(uint8_t code)
{
    int sign = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if ((code & 0x7F) == 0x7F)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10);
    return (float)(sign ? -v : v);
}

/* Round the non-negative integer sig * 2^-shift to the nearest integer, ties to
 * even.  shift >= 1. */
static uint32_t round_shift_rne(uint32_t sig, int shift)
{
    if (shift >= 32)
        return 0; /* sig < 2^24, so the value is below one half */
    uint32_t q = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u)))
        q += 1;
    return q;
}

/* Nearest E4M3 code of a finite fp32 value, ties to even, saturating: every
 * |v| >= 448 gives the largest finite magnitude 0x7E. */
uint8_t orc_e4m3_encode(float v)
{
    uint32_t u = bits_from_f32(v);
    uint8_t sign = (uint8_t)((u >> 31) << 7);
    uint32_t a = u & 0x7FFFFFFFu;           /* bits of |v| */
    uint32_t exp_field = a >> 23;
    uint32_t mant = a & 0x7FFFFFu;

    if (a >= 0x43E00000u)                   /* |v| >= 448 */
        return sign | 0x7E;

    if (a < 0x3C800000u) {                  /* |v| < 2^-6: subnormal grid k * 2^-9 */
        /* |v| = sig * 2^(pow2); k = RNE(|v| * 2^9) in [0, 8]; k = 8 is the
         * smallest normal (code 0x08), so the code is k itself. */
        uint32_t sig;
        int pow2;
        if (exp_field == 0) { sig = mant; pow2 = -149; }
        else { sig = mant | 0x800000u; pow2 = (int)exp_field - 150; }
        if (sig == 0)
            return sign;
        /* |v| < 2^-6 means pow2 + 9 <= -21, so the shift is at least 21. */
        return sign | (uint8_t)round_shift_rne(sig, -(pow2 + 9));
    }

    /* 2^-6 <= |v| < 448: keep 3 of the 23 mantissa bits, ties to even; a carry
     * out of the mantissa moves into the exponent by plain addition. */
    {
        int e_unb = (int)exp_field - 127;            /* in [-6, 8] */
        uint32_t q = round_shift_rne(mant, 20);      /* in [0, 8]  */
        uint32_t mag = ((uint32_t)(e_unb + 7) << 3) + q;
        return sign | (uint8_t)mag;                  /* <= 0x7E since |v| < 448 */
    }
}

void orc_e4m3_encode_bits_range(uint32_t first, size_t n, uint8_t *out)
{
    for (size_t i = 0; i < n; ++i)
        out[i] = orc_e4m3_encode(f32_from_bits(first + (uint32_t)i));
}

/* ------------------------------------------------------------------- bf16 */

float orc_bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* Round-to-nearest-even of a finite fp32 to bf16 (overflow rounds to inf). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u = bits_from_f32(f);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------- row load / store */

/* Read len elements of row `row` starting at element `off` into fp32. */
static void load_f32(int dtype, const void *base, size_t stride, size_t row,
                     size_t off, size_t len, float *dst)
{
    if (dtype == ORC_F32) {
        const float *p = (const float *)base + row * stride + off;
        for (size_t i = 0; i < len; ++i)
            dst[i] = p[i];
    } else {
        const uint16_t *p = (const uint16_t *)base + row * stride + off;
        for (size_t i = 0; i < len; ++i)
            dst[i] = orc_bf16_to_f32(p[i]);
    }
}

/* Write len fp32 values as `dtype` (bf16: one RNE each). */
static void store_f32(int dtype, void *base, size_t stride, size_t row,
                      size_t off, size_t len, const float *src)
{
    if (dtype == ORC_F32) {
        float *p = (float *)base + row * stride + off;
        for (size_t i = 0; i < len; ++i)
            p[i] = src[i];
    } else {
        uint16_t *p = (uint16_t *)base + row * stride + off;
        for (size_t i = 0; i < len; ++i)
            p[i] = orc_f32_to_bf16(src[i]);
    }
}

static void copy_elems(int dtype, const void *sbase, size_t sstride, size_t srow, size_t soff,
                       void *dbase, size_t dstride, size_t drow, size_t doff, size_t len)
{
    size_t es = elem_size(dtype);
    const char *s = (const char *)sbase + (srow * sstride + soff) * es;
    char *d = (char *)dbase + (drow * dstride + doff) * es;
    memmove(d, s, len * es);
}

static int all_finite(const float *x, size_t len)
{
    for (size_t i = 0; i < len; ++i)
        if (!isfinite(x[i]))
            return 0;
    return 1;
}

/* ------------------------------------------------- one block, one segment */

/* Quantise one block of len (<= 128) fp32 values. */
static void quant_block(const float *x, size_t len, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (size_t i = 0; i < len; ++i) {
        float ax = fabsf(x[i]);
        if (ax > amax)
            amax = ax;
    }
    float s = amax / ORC_E4M3_MAX;
    *scale = s;
    for (size_t i = 0; i < len; ++i) {
        if (s == 0.0f)
            codes[i] = signbit(x[i]) ? 0x80 : 0x00;
        else
            codes[i] = orc_e4m3_encode(x[i] / s);
    }
}

static void dequant_block(const uint8_t *codes, size_t len, float s, float *y)
{
    for (size_t i = 0; i < len; ++i)
        y[i] = orc_e4m3_value(codes[i]) * s;
}

/* Quantise a segment of len values in 128-blocks anchored at x[0]. */
static void quant_segment(const float *x, size_t len, uint8_t *codes, float *scales)
{
    for (size_t b = 0; b * ORC_BLOCK < len; ++b) {
        size_t lo = b * ORC_BLOCK;
        size_t n = len - lo < ORC_BLOCK ? len - lo : ORC_BLOCK;
        quant_block(x + lo, n, codes + lo, &scales[b]);
    }
}

static void dequant_segment(const uint8_t *codes, const float *scales, size_t len, float *y)
{
    for (size_t b = 0; b * ORC_BLOCK < len; ++b) {
        size_t lo = b * ORC_BLOCK;
        size_t n = len - lo < ORC_BLOCK ? len - lo : ORC_BLOCK;
        dequant_block(codes + lo, n, scales[b], y + lo);
    }
}

static size_t nblocks(size_t len) { return (len + ORC_BLOCK - 1) / ORC_BLOCK; }

/* What a receiver holds after one segment crossed the wire: the segment itself
 * on a native wire; on the FP8 wire, the dequantised sender-side quantisation
 * of it.  In place on x.  Returns 0, or -1 on a non-finite FP8 input. */
static int wire_segment(int wire, float *x, size_t len)
{
    if (wire == ORC_NATIVE || len == 0)
        return 0;
    if (!all_finite(x, len))
        return -1;
    uint8_t *codes = (uint8_t *)malloc(len);
    float *scales = (float *)malloc(nblocks(len) * sizeof(float));
    if (!codes || !scales) { free(codes); free(scales); return -2; }
    quant_segment(x, len, codes, scales);
    dequant_segment(codes, scales, len, x);
    free(codes);
    free(scales);
    return 0;
}

/* --------------------------------------------------------- quantise APIs */

int orc_quantize(int dtype, const void *x, size_t rows, size_t n, size_t stride,
                 uint8_t *codes, float *scales)
{
    if ((dtype != ORC_F32 && dtype != ORC_BF16) || stride < n)
        return -1;
    float *row = (float *)malloc((n ? n : 1) * sizeof(float));
    if (!row)
        return -2;
    for (size_t r = 0; r < rows; ++r) {
        load_f32(dtype, x, stride, r, 0, n, row);
        if (!all_finite(row, n)) { free(row); return -1; }
        quant_segment(row, n, codes + r * stride, scales + r * nblocks(n));
    }
    free(row);
    return 0;
}

int orc_dequantize(const uint8_t *codes, const float *scales, size_t rows, size_t n,
                   size_t stride, int dtype, void *y)
{
    if ((dtype != ORC_F32 && dtype != ORC_BF16) || stride < n)
        return -1;
    float *row = (float *)malloc((n ? n : 1) * sizeof(float));
    if (!row)
        return -2;
    for (size_t r = 0; r < rows; ++r) {
        dequant_segment(codes + r * stride, scales + r * nblocks(n), n, row);
        store_f32(dtype, y, stride, r, 0, n, row);
    }
    free(row);
    return 0;
}

/* ------------------------------------------------------------ collectives */

static int check_common(int dtype, int wire, int nranks)
{
    if (dtype != ORC_F32 && dtype != ORC_BF16)
        return -1;
    if (wire != ORC_NATIVE && wire != ORC_FP8)
        return -1;
    if (nranks < 1)
        return -1;
    return 0;
}

/* sum[i] = w(X[0][off+i]) + w(X[1][off+i]) + ... + w(X[N-1][off+i]), rank
 * order, each term being what arrives from that rank over the wire (the wire
 * quantises each rank's segment with blocks anchored at `off`). */
static int reduce_segment(int dtype, int wire, const void *send, size_t stride,
                          size_t off, size_t len, int nranks, float *sum)
{
    float *term = (float *)malloc((len ? len : 1) * sizeof(float));
    if (!term)
        return -2;
    for (int s = 0; s < nranks; ++s) {
        load_f32(dtype, send, stride, (size_t)s, off, len, term);
        if (wire_segment(wire, term, len) != 0) { free(term); return -1; }
        if (s == 0) {
            for (size_t i = 0; i < len; ++i)
                sum[i] = term[i];
        } else {
            for (size_t i = 0; i < len; ++i)
                sum[i] = sum[i] + term[i];
        }
    }
    free(term);
    return 0;
}

/* DDA-flat [DDA-pt, DDA-es]: each rank reads every rank's buffer and reduces
 * locally; the N local reductions are identical, so it is computed once per
 * element index and written to all N output rows. */
int orc_allreduce_flat(int dtype, int wire, const void *send, void *recv,
                       size_t count, size_t stride, int nranks)
{
    if (check_common(dtype, wire, nranks) || stride < count)
        return -1;
    if (nranks == 1) {
        copy_elems(dtype, send, stride, 0, 0, recv, stride, 0, 0, count);
        return 0;
    }
    float *sum = (float *)malloc((count ? count : 1) * sizeof(float));
    if (!sum)
        return -2;
    int rc = reduce_segment(dtype, wire, send, stride, 0, count, nranks, sum);
    if (rc == 0)
        for (int r = 0; r < nranks; ++r)
            store_f32(dtype, recv, stride, (size_t)r, 0, count, sum);
    free(sum);
    return rc;
}

size_t orc_tree_chunk(size_t count, int nranks)
{
    size_t blocks = nblocks(count);
    size_t per_rank = (blocks + (size_t)nranks - 1) / (size_t)nranks;
    return per_rank * ORC_BLOCK;
}

/* DDA-tree [DDA-pt, DDA-es]: phase 1 is a reduce-scatter -- rank c reduces
 * chunk c of all ranks' buffers -- and phase 2 an all-gather -- every rank
 * fetches every reduced chunk.  On the FP8 wire the reduced chunk is quantised
 * by its owner before phase 2 (the second quantisation [LP-es]). */
int orc_allreduce_tree(int dtype, int wire, const void *send, void *recv,
                       size_t count, size_t stride, int nranks)
{
    if (check_common(dtype, wire, nranks) || stride < count)
        return -1;
    if (nranks == 1) {
        copy_elems(dtype, send, stride, 0, 0, recv, stride, 0, 0, count);
        return 0;
    }
    size_t C = orc_tree_chunk(count, nranks);
    float *chunk = (float *)malloc((C ? C : 1) * sizeof(float));
    /* the payload each chunk owner publishes between the two phases */
    uint8_t *pay_codes = (uint8_t *)malloc(count ? count : 1);
    float *pay_scales = (float *)malloc((nblocks(count) ? nblocks(count) : 1) * sizeof(float));
    int rc = 0;
    if (!chunk || !pay_codes || !pay_scales) { rc = -2; goto done; }

    /* Phase 1: reduce-scatter. */
    for (int c = 0; c < nranks && rc == 0; ++c) {
        size_t lo = (size_t)c * C;
        if (lo >= count)
            break;
        size_t len = count - lo < C ? count - lo : C;
        rc = reduce_segment(dtype, wire, send, stride, lo, len, nranks, chunk);
        if (rc)
            break;
        if (wire == ORC_NATIVE)
            store_f32(dtype, recv, stride, (size_t)c, lo, len, chunk);
        else
            quant_segment(chunk, len, pay_codes + lo, pay_scales + lo / ORC_BLOCK);
    }

    /* Phase 2: all-gather. */
    for (int c = 0; c < nranks && rc == 0; ++c) {
        size_t lo = (size_t)c * C;
        if (lo >= count)
            break;
        size_t len = count - lo < C ? count - lo : C;
        if (wire == ORC_NATIVE) {
            for (int r = 0; r < nranks; ++r)
                if (r != c)
                    copy_elems(dtype, recv, stride, (size_t)c, lo, recv, stride, (size_t)r, lo, len);
        } else {
            dequant_segment(pay_codes + lo, pay_scales + lo / ORC_BLOCK, len, chunk);
            for (int r = 0; r < nranks; ++r)
                store_f32(dtype, recv, stride, (size_t)r, lo, len, chunk);
        }
    }
done:
    free(chunk);
    free(pay_codes);
    free(pay_scales);
    return rc;
}

/* ReduceScatter [LP-es]: out[r][j] = SUM_s w(X[s][r*m + j]), j < m. */
int orc_reduce_scatter(int dtype, int wire, const void *send, size_t send_stride,
                       void *recv, size_t recv_stride, size_t m, int nranks)
{
    if (check_common(dtype, wire, nranks) || recv_stride < m ||
        send_stride < (size_t)nranks * m)
        return -1;
    if (nranks == 1) {
        copy_elems(dtype, send, send_stride, 0, 0, recv, recv_stride, 0, 0, m);
        return 0;
    }
    float *sum = (float *)malloc((m ? m : 1) * sizeof(float));
    if (!sum)
        return -2;
    int rc = 0;
    for (int r = 0; r < nranks && rc == 0; ++r) {
        rc = reduce_segment(dtype, wire, send, send_stride, (size_t)r * m, m, nranks, sum);
        if (rc == 0)
            store_f32(dtype, recv, recv_stride, (size_t)r, 0, m, sum);
    }
    free(sum);
    return rc;
}

/* AllGather [LP-es]: out[r][s*m + j] = w(Y[s][j]). */
int orc_all_gather(int dtype, int wire, const void *send, size_t send_stride,
                   void *recv, size_t recv_stride, size_t m, int nranks)
{
    if (check_common(dtype, wire, nranks) || send_stride < m ||
        recv_stride < (size_t)nranks * m)
        return -1;
    if (nranks == 1) {
        copy_elems(dtype, send, send_stride, 0, 0, recv, recv_stride, 0, 0, m);
        return 0;
    }
    float *seg = (float *)malloc((m ? m : 1) * sizeof(float));
    if (!seg)
        return -2;
    int rc = 0;
    for (int s = 0; s < nranks && rc == 0; ++s) {
        if (wire == ORC_NATIVE) {
            for (int r = 0; r < nranks; ++r)
                copy_elems(dtype, send, send_stride, (size_t)s, 0,
                           recv, recv_stride, (size_t)r, (size_t)s * m, m);
        } else {
            load_f32(dtype, send, send_stride, (size_t)s, 0, m, seg);
            rc = wire_segment(wire, seg, m);
            if (rc == 0)
                for (int r = 0; r < nranks; ++r)
                    store_f32(dtype, recv, recv_stride, (size_t)r, (size_t)s * m, m, seg);
        }
    }
    free(seg);
    return rc;
}

/* AlltoAll [LP-es]: out[r][s*m + j] = w(X[s][r*m + j]) -- chunk r of rank s
 * goes to rank r, landing at position s. */
int orc_alltoall(int dtype, int wire, const void *send, size_t send_stride,
                 void *recv, size_t recv_stride, size_t m, int nranks)
{
    if (check_common(dtype, wire, nranks) || send_stride < (size_t)nranks * m ||
        recv_stride < (size_t)nranks * m)
        return -1;
    if (nranks == 1) {
        copy_elems(dtype, send, send_stride, 0, 0, recv, recv_stride, 0, 0, m);
        return 0;
    }
    float *seg = (float *)malloc((m ? m : 1) * sizeof(float));
    if (!seg)
        return -2;
    int rc = 0;
    for (int s = 0; s < nranks && rc == 0; ++s) {
        for (int r = 0; r < nranks && rc == 0; ++r) {
            if (wire == ORC_NATIVE) {
                copy_elems(dtype, send, send_stride, (size_t)s, (size_t)r * m,
                           recv, recv_stride, (size_t)r, (size_t)s * m, m);
            } else {
                load_f32(dtype, send, send_stride, (size_t)s, (size_t)r * m, m, seg);
                rc = wire_segment(wire, seg, m);
                if (rc == 0)
                    store_f32(dtype, recv, recv_stride, (size_t)r, (size_t)s * m, m, seg);
            }
        }
    }
    free(seg);
    return rc;
}
