/*
 * tcf4_oracle.c -- the CPU oracle for trellis-coded FP4 decoding and its products.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU-baseline leg of the
 * bench load this library. The CUDA library shares no code, header, table or helper with it,
 * and neither side calls the other.
 *
 * Plain C99, single-threaded, no intrinsics, fp64 arithmetic. Each function restates one step
 * of the method from the pages it cites, in their order and notation:
 *
 *   [XT]   "XOR-Trellis: Hadamard-free FP4 LLM quantization" news page (aimodeling.com, English
 *          and Chinese editions), bullet "XOR-Trellis FP4 decoder": four palettes P0..P3, a
 *          16-bit sliding state, four masked parities 0x1089/0x2112/0x0A24/0x2441 giving
 *          p0, p1, q0, q1; (p0, p1) pick the palette, (q0, q1) permute branch -> entry.
 *          Bullet "Curvature-aware Viterbi objective": additive distortion weighted by the
 *          diagonal D of H = L D L^T, searched offline by Viterbi.
 *   [HEPH] "HEPH: 3-Bit Grid-Aligned Trellis Quantization of MXFP4 Mixture-of-Experts for
 *          Accurate, Hadamard-Free Serving", abstract: each block reuses its UE8M0 exponent as
 *          the exact scale, the codebook is the 15 distinct E2M1 values, so every decoded
 *          weight is an MXFP4 element; mode 1 decodes in-kernel, mode 2 expands to MXFP4.
 *   [TTP]  "Tied Trit-Planes: Constraining PTQTP to a Uniform Nine-Level Quantizer ...",
 *          section 2.1 (MXFP4 = fp4-e2m1 codes with one e8m0 scale per 32 elements, exactly
 *          dequantizable) and its OCP MX v1.0 reference (E2M1 and E8M0 encodings).
 *
 * Where the pages leave a step open, the reading taken is written beside the step:
 *   - the new 2-bit branch symbol enters the state at bits 14-15 and the window slides down by
 *     one symbol (the four masks together cover exactly bits 0-13, so the branch bits never
 *     reach a parity and all four branches of a state share one palette);
 *   - the value is read from the state after the new symbol entered;
 *   - palette index p = p0 + 2*p1, permutation q = q0 + 2*q1, entry e = b XOR q  [unpinned:
 *     the pages fix no bit order and XOR is the reading of "XOR + palette lookup"];
 *   - branch symbol b = lo + 2*hi, stream packed planar per 32-weight block (word 0 holds the
 *     low bits of symbols 0..31, bit i = symbol i; word 1 the high bits)  [unpinned];
 *   - the state is 0 at the start of every segment of seg_len weights along a row;
 *   - P3's zero is -0 (code 0x8), so the 16 palette slots are the 16 E2M1 codes;
 *   - an MXFP4 byte holds element 2u in its low nibble and 2u+1 in its high nibble;
 *   - the second, interleaved packing (below) stores each row as one bit string, two bits per
 *     symbol, low bit first, LSB-first in 32-bit words  [unpinned, like the planar packing].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* [XT] decoder bullet: the four local reconstruction palettes, as printed. */
static const double XT_PALETTE[4][4] = {
    {-6.0, -1.5, 0.0, 2.0}, /* P0 */
    {-4.0, -1.0, 0.5, 3.0}, /* P1 */
    {-3.0, -0.5, 1.0, 4.0}, /* P2 */
    {-2.0, -0.0, 1.5, 6.0}, /* P3 (its zero read as -0) */
};
/* [XT] decoder bullet: the masks whose parities give p0, p1, q0, q1, in that order. */
static const uint32_t XT_MASK[4] = {0x1089u, 0x2112u, 0x0A24u, 0x2441u};

/* Exported copies so tests can compare the tables with the printed values. */
void oracle_tables(double palette_out[16], uint32_t masks_out[4]) {
    for (int p = 0; p < 4; p++)
        for (int e = 0; e < 4; e++) palette_out[4 * p + e] = XT_PALETTE[p][e];
    for (int i = 0; i < 4; i++) masks_out[i] = XT_MASK[i];
}

/* [TTP]/OCP MX: E2M1 = 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent field 0
 * is subnormal (0 or 0.5). */
double oracle_e2m1_value(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return s ? -mag : mag;
}

/* The E2M1 code of an exactly representable value, matching the sign of zero. */
int oracle_e2m1_code(double v, uint8_t *code) {
    for (int c = 0; c < 16; c++) {
        double d = oracle_e2m1_value((uint8_t)c);
        if (d == v && (signbit(d) != 0) == (signbit(v) != 0)) {
            *code = (uint8_t)c;
            return ORACLE_OK;
        }
    }
    return ORACLE_EINVAL;
}

/* [TTP]/OCP MX: an E8M0 (UE8M0) scale byte E means 2^(E-127); E = 0xFF is NaN. */
double oracle_ue8m0_value(uint8_t E) { return E == 0xFF ? NAN : ldexp(1.0, (int)E - 127); }

/* The XOR-Trellis news page's paragraph on the grouping format pairs E2M1 elements with E5M3 block
 * scales and gives no encoding for the scale. Reading: 8 bits, no sign bit (block scales are positive), exponent
 * in bits 7..3 with bias 15, mantissa in bits 2..0; exponent 0 is subnormal (2^-14 * m/8), exponent
 * 31 is NaN; one scale per 32-weight block, as for UE8M0. */
double oracle_e5m3_value(uint8_t b) {
    int e = b >> 3, m = b & 7;
    if (e == 31) return NAN;
    if (e == 0) return ldexp((double)m / 8.0, -14);
    return ldexp(1.0 + (double)m / 8.0, e - 15);
}

#define SCALE_UE8M0 0
#define SCALE_E5M3 1

static double scale_value(uint8_t b, int fmt) {
    return fmt == SCALE_E5M3 ? oracle_e5m3_value(b) : oracle_ue8m0_value(b);
}

static int parity16(uint32_t v) {
    int p = 0;
    for (int i = 0; i < 16; i++) p ^= (int)((v >> i) & 1u);
    return p;
}

/* [XT] 16-bit sliding state: the new branch symbol enters at bits 14-15. */
uint32_t oracle_state_push(uint32_t s, uint32_t b) { return ((s >> 2) | ((b & 3u) << 14)) & 0xFFFFu; }

/* [XT] masked parities -> palette index p and palette entry e for the state s (after push). */
void oracle_state_decode(uint32_t s, int *p_out, int *e_out) {
    int p0 = parity16(s & XT_MASK[0]);
    int p1 = parity16(s & XT_MASK[1]);
    int q0 = parity16(s & XT_MASK[2]);
    int q1 = parity16(s & XT_MASK[3]);
    int p = p0 | (p1 << 1);       /* the first pair selects the palette */
    int q = q0 | (q1 << 1);       /* the second pair permutes branch -> entry */
    int b = (int)((s >> 14) & 3u); /* the branch symbol that just entered */
    *p_out = p;
    *e_out = b ^ q;
}

double oracle_state_value(uint32_t s) {
    int p, e;
    oracle_state_decode(s, &p, &e);
    return XT_PALETTE[p][e];
}

/* The MXFP4 element code of the value a state decodes to ([HEPH]: every decoded weight is a
 * valid E2M1 element). Returns 0xFF if the palette value were not an E2M1 value. */
uint8_t oracle_state_code(uint32_t s) {
    uint8_t c;
    if (oracle_e2m1_code(oracle_state_value(s), &c) != ORACLE_OK) return 0xFF;
    return c;
}

/* Branch symbol of weight k of row n under the planar packing. */
static uint32_t symbol_at(const uint32_t *stream, int64_t cols, int64_t n, int64_t k) {
    int64_t j = k / 32, i = k % 32;
    const uint32_t *blk = stream + 2 * (n * (cols / 32) + j);
    return ((blk[0] >> i) & 1u) | (((blk[1] >> i) & 1u) << 1);
}

static int check_shape(int64_t rows, int64_t cols, int64_t seg_len) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return ORACLE_EINVAL;
    if (cols > 0 && (seg_len <= 0 || seg_len % 32 != 0 || cols % seg_len != 0)) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/* Decoded E2M1 codes, one byte per weight, [rows][cols]. */
int oracle_decode_codes(const uint32_t *stream, int64_t rows, int64_t cols, int64_t seg_len, uint8_t *codes) {
    if (check_shape(rows, cols, seg_len)) return ORACLE_EINVAL;
    for (int64_t n = 0; n < rows; n++) {
        uint32_t s = 0;
        for (int64_t k = 0; k < cols; k++) {
            if (k % seg_len == 0) s = 0;
            s = oracle_state_push(s, symbol_at(stream, cols, n, k));
            codes[n * cols + k] = oracle_state_code(s);
        }
    }
    return ORACLE_OK;
}

/* One decoded row in fp64: palette value times its block's scale ([HEPH] grid-aligned; or the
 * E5M3 block scale of the XOR-Trellis page's grouping format when fmt is SCALE_E5M3). */
static void decode_row(const uint32_t *stream, const uint8_t *scales, int64_t cols, int64_t seg_len,
                       int64_t n, double *w, int fmt) {
    uint32_t s = 0;
    for (int64_t k = 0; k < cols; k++) {
        if (k % seg_len == 0) s = 0;
        s = oracle_state_push(s, symbol_at(stream, cols, n, k));
        w[k] = oracle_state_value(s) * scale_value(scales[n * (cols / 32) + k / 32], fmt);
    }
}

static int decode_values_fmt(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols,
                             int64_t seg_len, double *w, int fmt) {
    if (check_shape(rows, cols, seg_len)) return ORACLE_EINVAL;
    for (int64_t n = 0; n < rows; n++) decode_row(stream, scales, cols, seg_len, n, w + n * cols, fmt);
    return ORACLE_OK;
}

int oracle_decode_values(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols,
                         int64_t seg_len, double *w) {
    return decode_values_fmt(stream, scales, rows, cols, seg_len, w, SCALE_UE8M0);
}

int oracle_decode_values_e5m3(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols,
                              int64_t seg_len, double *w) {
    return decode_values_fmt(stream, scales, rows, cols, seg_len, w, SCALE_E5M3);
}

/* [HEPH] mode 2: packed MXFP4, [rows][cols/2] bytes (even element in the low nibble) plus the
 * scale bytes copied unchanged. */
int oracle_expand_mxfp4(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols,
                        int64_t seg_len, uint8_t *nibbles, uint8_t *out_scales) {
    if (check_shape(rows, cols, seg_len)) return ORACLE_EINVAL;
    for (int64_t n = 0; n < rows; n++) {
        uint32_t s = 0;
        for (int64_t k = 0; k < cols; k++) {
            if (k % seg_len == 0) s = 0;
            s = oracle_state_push(s, symbol_at(stream, cols, n, k));
            uint8_t c = oracle_state_code(s);
            uint8_t *byte = nibbles + n * (cols / 2) + k / 2;
            if (k % 2 == 0)
                *byte = c;
            else
                *byte = (uint8_t)(*byte | (c << 4));
        }
    }
    memcpy(out_scales, scales, (size_t)(rows * (cols / 32)));
    return ORACLE_OK;
}

/* ---------------------------------------------------------------- interleaved packing
 * A second packing of the same stream (a reading; the pages fix none): each row is one bit string
 * in which symbol k takes bits 2k (its low bit) and 2k+1 (its high bit), stored LSB-first in 32-bit
 * words, so block j of a row owns words 2j (its symbols 0..15) and 2j+1 (symbols 16..31).
 * Under this packing the [XT] "16-bit sliding state" is literally a window of the bit string. */

/* Bit p of row n's bit string. */
static uint32_t il_bit(const uint32_t *il, int64_t cols, int64_t n, int64_t p) {
    return (il[n * (cols / 16) + p / 32] >> (p % 32)) & 1u;
}

/* [XT] decoder bullet, read on the interleaved bit string: the state of weight k is the 16 bits of
 * the row's string that end with symbol k's high bit (bit m of the state = string bit 2k - 14 + m),
 * with every bit before the start of k's segment read as 0. No symbol recurrence is used here. */
int oracle_decode_codes_interleaved(const uint32_t *il, int64_t rows, int64_t cols, int64_t seg_len,
                                    uint8_t *codes) {
    if (check_shape(rows, cols, seg_len)) return ORACLE_EINVAL;
    for (int64_t n = 0; n < rows; n++)
        for (int64_t k = 0; k < cols; k++) {
            int64_t start = 2 * (k - k % seg_len);
            uint32_t s = 0;
            for (int m = 0; m < 16; m++) {
                int64_t p = 2 * k - 14 + m;
                if (p >= start) s |= il_bit(il, cols, n, p) << m;
            }
            codes[n * cols + k] = oracle_state_code(s);
        }
    return ORACLE_OK;
}

/* Interleaved -> planar: symbol k of a row (bits 2k, 2k+1 of its string) becomes bit k % 32 of the
 * low and high words of its block. */
int oracle_repack_interleaved(const uint32_t *il, int64_t rows, int64_t cols, uint32_t *planar) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return ORACLE_EINVAL;
    for (int64_t n = 0; n < rows; n++)
        for (int64_t j = 0; j < cols / 32; j++) {
            uint32_t lo = 0, hi = 0;
            for (int64_t i = 0; i < 32; i++) {
                int64_t k = 32 * j + i;
                lo |= il_bit(il, cols, n, 2 * k) << i;
                hi |= il_bit(il, cols, n, 2 * k + 1) << i;
            }
            planar[2 * (n * (cols / 32) + j)] = lo;
            planar[2 * (n * (cols / 32) + j) + 1] = hi;
        }
    return ORACLE_OK;
}

/* bf16 bit pattern -> value (bf16 is the top half of an IEEE binary32). */
double oracle_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even (8 significant bits, binary32 exponent
 * range, subnormals with quantum 2^-133, overflow to infinity). */
double oracle_bf16_round(double v) {
    if (v == 0.0 || isnan(v) || isinf(v)) return v;
    int ex;
    double m = frexp(fabs(v), &ex); /* |v| = m * 2^ex, m in [0.5, 1) */
    double r;
    if (ex - 1 >= -126) {
        r = ldexp(nearbyint(ldexp(m, 8)), ex - 8); /* 8 significant bits */
    } else {
        r = ldexp(nearbyint(ldexp(fabs(v), 133)), -133); /* subnormal quantum */
    }
    if (r > 3.3895313892515355e38) r = INFINITY; /* beyond the largest finite bf16 */
    return copysign(r, v);
}

uint16_t oracle_bf16_bits(double v) {
    float f = (float)oracle_bf16_round(v); /* exact: a bf16 value is a binary32 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* Products y[t][i] = sum_k w[row_i][k] * x[t][k] in fp64, summed in k order, for the rows
 * listed in row_ids (all rows in order when row_ids is NULL, nr = rows). Also returns the
 * Euclidean norm of each listed decoded row in wnorm (may be NULL). x holds bf16 bits [T][cols].
 * The sum's rounding error is at most cols * 2^-53 * sum |w x|. */
static int gemv_fmt(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols, int64_t seg_len,
                    const uint16_t *x, int64_t T, const int64_t *row_ids, int64_t nr, double *y, double *wnorm,
                    int fmt) {
    if (check_shape(rows, cols, seg_len) || T < 0 || nr < 0) return ORACLE_EINVAL;
    if (row_ids == NULL && nr != rows) return ORACLE_EINVAL;
    double *w = (double *)malloc(sizeof(double) * (size_t)(cols > 0 ? cols : 1));
    double *xv = (double *)malloc(sizeof(double) * (size_t)(T * cols > 0 ? T * cols : 1));
    if (!w || !xv) {
        free(w);
        free(xv);
        return ORACLE_ENOMEM;
    }
    for (int64_t i = 0; i < T * cols; i++) xv[i] = oracle_bf16_value(x[i]);
    for (int64_t i = 0; i < nr; i++) {
        int64_t n = row_ids ? row_ids[i] : i;
        if (n < 0 || n >= rows) {
            free(w);
            free(xv);
            return ORACLE_EINVAL;
        }
        decode_row(stream, scales, cols, seg_len, n, w, fmt);
        if (wnorm) {
            double ss = 0.0;
            for (int64_t k = 0; k < cols; k++) ss += w[k] * w[k];
            wnorm[i] = sqrt(ss);
        }
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0;
            for (int64_t k = 0; k < cols; k++) acc += w[k] * xv[t * cols + k];
            y[t * nr + i] = acc;
        }
    }
    free(w);
    free(xv);
    return ORACLE_OK;
}

int oracle_gemv(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols, int64_t seg_len,
                const uint16_t *x, int64_t T, const int64_t *row_ids, int64_t nr, double *y, double *wnorm) {
    return gemv_fmt(stream, scales, rows, cols, seg_len, x, T, row_ids, nr, y, wnorm, SCALE_UE8M0);
}

/* The same products with E5M3 block scales (reading above oracle_e5m3_value). */
int oracle_gemv_e5m3(const uint32_t *stream, const uint8_t *scales, int64_t rows, int64_t cols, int64_t seg_len,
                     const uint16_t *x, int64_t T, const int64_t *row_ids, int64_t nr, double *y, double *wnorm) {
    return gemv_fmt(stream, scales, rows, cols, seg_len, x, T, row_ids, nr, y, wnorm, SCALE_E5M3);
}

/* [HEPH] mode 2, consumer side: the same products from a resident MXFP4 tensor. By the OCP MX
 * definition ([TTP] section 2.1) element k of row n is E2M1(code) * 2^(E-127), code = nibble k of
 * the row (low nibble of byte k/2 for even k), E = scales[n][k/32]. y[t][i] = sum_k w x in fp64, in
 * k order, for the rows in row_ids (all rows when NULL, nr = rows); wnorm as in oracle_gemv. */
int oracle_mxfp4_gemv(const uint8_t *nibbles, const uint8_t *scales, int64_t rows, int64_t cols, const uint16_t *x,
                      int64_t T, const int64_t *row_ids, int64_t nr, double *y, double *wnorm) {
    if (rows < 0 || cols < 0 || cols % 32 != 0 || T < 0 || nr < 0) return ORACLE_EINVAL;
    if (row_ids == NULL && nr != rows) return ORACLE_EINVAL;
    double *w = (double *)malloc(sizeof(double) * (size_t)(cols > 0 ? cols : 1));
    double *xv = (double *)malloc(sizeof(double) * (size_t)(T * cols > 0 ? T * cols : 1));
    if (!w || !xv) {
        free(w);
        free(xv);
        return ORACLE_ENOMEM;
    }
    for (int64_t i = 0; i < T * cols; i++) xv[i] = oracle_bf16_value(x[i]);
    for (int64_t i = 0; i < nr; i++) {
        int64_t n = row_ids ? row_ids[i] : i;
        if (n < 0 || n >= rows) {
            free(w);
            free(xv);
            return ORACLE_EINVAL;
        }
        for (int64_t k = 0; k < cols; k++) {
            uint8_t byte = nibbles[n * (cols / 2) + k / 2];
            uint8_t code = (k % 2 == 0) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4);
            w[k] = oracle_e2m1_value(code) * oracle_ue8m0_value(scales[n * (cols / 32) + k / 32]);
        }
        if (wnorm) {
            double ss = 0.0;
            for (int64_t k = 0; k < cols; k++) ss += w[k] * w[k];
            wnorm[i] = sqrt(ss);
        }
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0;
            for (int64_t k = 0; k < cols; k++) acc += w[k] * xv[t * cols + k];
            y[t * nr + i] = acc;
        }
    }
    free(w);
    free(xv);
    return ORACLE_OK;
}

/* [XT] Viterbi bullet: the D-weighted additive distortion of one segment,
 *   cost = sum_k D[k] * (target[k] - P(s_k) * scale[k])^2,
 * minimised over the 4^L branch sequences of a segment that starts in state 0 and may end in
 * any state. The search keeps, for every 14-bit predecessor window (the previous 7 symbols),
 * the cheapest path reaching it; a window has 4 predecessors (the 2 bits that slide out).
 * Ties go to the lower predecessor window, and at the end to the lower final window.
 * Returns the minimum cost (or -1 on a bad argument / allocation failure) and the branch
 * symbols in sym_out[L]. */
double oracle_viterbi_encode(const double *target, const double *D, const double *scale, int64_t L,
                             uint8_t *sym_out) {
    enum { NW = 1 << 14 };
    if (L <= 0) return L == 0 ? 0.0 : -1.0;
    double *cost = (double *)malloc(sizeof(double) * NW);
    double *next = (double *)malloc(sizeof(double) * NW);
    uint8_t *back = (uint8_t *)malloc((size_t)L * NW);
    if (!cost || !next || !back) {
        free(cost);
        free(next);
        free(back);
        return -1.0;
    }
    for (int w = 0; w < NW; w++) cost[w] = INFINITY;
    cost[0] = 0.0;
    for (int64_t k = 0; k < L; k++) {
        for (uint32_t wn = 0; wn < NW; wn++) {
            uint32_t b = wn >> 12;             /* the symbol pushed at step k */
            double best = INFINITY;
            int best_r = 0;
            for (uint32_t r = 0; r < 4; r++) { /* predecessor windows in increasing order */
                uint32_t wp = ((wn & 0xFFFu) << 2) | r;
                if (isinf(cost[wp])) continue;
                uint32_t s = wp | (b << 14); /* the full 16-bit state after the push */
                double d = target[k] - oracle_state_value(s) * scale[k];
                double c = cost[wp] + D[k] * d * d;
                if (c < best) {
                    best = c;
                    best_r = (int)r;
                }
            }
            next[wn] = best;
            back[(size_t)k * NW + wn] = (uint8_t)best_r;
        }
        double *tmp = cost;
        cost = next;
        next = tmp;
    }
    uint32_t wn = 0;
    for (uint32_t w = 1; w < NW; w++)
        if (cost[w] < cost[wn]) wn = w;
    double best = cost[wn];
    for (int64_t k = L - 1; k >= 0; k--) {
        sym_out[k] = (uint8_t)(wn >> 12);
        wn = ((wn & 0xFFFu) << 2) | back[(size_t)k * NW + wn];
    }
    free(cost);
    free(next);
    free(back);
    return best;
}

/* Exhaustive search over all 4^L sequences (L <= 8) of the same cost, for checking Viterbi.
 * Ties keep the first sequence in increasing base-4 order (symbol 0 most significant). */
double oracle_bruteforce_encode(const double *target, const double *D, const double *scale, int64_t L,
                                uint8_t *sym_out) {
    if (L < 0 || L > 8) return -1.0;
    uint64_t total = 1ull << (2 * L);
    double best = INFINITY;
    uint64_t best_seq = 0;
    for (uint64_t q = 0; q < total; q++) {
        uint32_t s = 0;
        double c = 0.0;
        for (int64_t k = 0; k < L; k++) {
            uint32_t b = (uint32_t)((q >> (2 * (L - 1 - k))) & 3u);
            s = oracle_state_push(s, b);
            double d = target[k] - oracle_state_value(s) * scale[k];
            c += D[k] * d * d;
        }
        if (c < best) {
            best = c;
            best_seq = q;
        }
    }
    for (int64_t k = 0; k < L; k++) sym_out[k] = (uint8_t)((best_seq >> (2 * (L - 1 - k))) & 3u);
    return best;
}
