/*
 * lores_oracle.c -- plain, slow CPU oracle for one LoReS decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file.  It is used by the test-suite, by the smoke check and by
 * the CPU-baseline leg of the benchmark.  It shares no source with the CUDA
 * library: every definition below is written out again from the method's
 * description and from the arithmetic definition of the state format.
 *
 * Sources (page titles; "Quantizing Recurrent Language Models Is Easier Than
 * You Think", summary page):
 *   - General recurrence form, Introduction:  S_t = S_{t-1} diag(a_t)
 *     (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t.
 *   - Key properties, Intra-State Quantization: the state is dequantized,
 *     updated and requantized on every decode step.
 *   - Proposition 1: symmetric absmax scale s_G = max|S_G| / r with
 *     r = 2^(b-1) - 1; value-axis grouping (one scale per value row, here
 *     optionally split into key blocks of G entries).
 *   - Proposition 3 / Table 6: stochastic rounding of the requantization.
 *   - Table 5 text and the abstract: decay-based mixed precision per head.
 *
 * Readings where the pages are silent (each is a choice, not a page fact):
 *   - Scales are recomputed from the updated state on every step.
 *   - The readout o_t = S_t q_t uses S_t = S' + w k^T (S' = S_{t-1} diag(alpha)
 *     in fp32, w in fp32) evaluated exactly, i.e. before requantization and before
 *     the fp32 rounding of the stored entries.
 *   - Products and sums are fp32 with the association written below.  The
 *     projection u = S'k is exact up to one rounding where the state is integer
 *     codes with one scale per value row (codes one byte or one nibble each,
 *     value-axis groups of G = d_k): alpha_j k_j is put on a fixed-point grid
 *     (Y_j = rint(alpha_j k_j 2^E), |Y_j| <= 2^30), the integer sum
 *     U_i = sum_j c_ij Y_j is exact, and u_i = fl32(fl64(s_i U_i) 2^-E).
 *     Elsewhere (fp32 state, several scales per row, bit planes, per-channel
 *     widths, key-axis scales) S'k uses a fixed fp32 order (16-column blocks,
 *     four interleaved sequential chains per block by half and column parity,
 *     then a pairwise combine of the block sums, nearest partners first) so
 *     that two implementations that follow it agree bit for bit.  The readout
 *     is summed in double.
 *   - Scale and its inverse: s = m * fl(1/r); inv = r * y, where y ~ 1/m comes
 *     from three Newton-Raphson steps y <- y + y(1 - m y) (fma form) started
 *     from the exponent-reflected seed bits(y0) = 0x7F000000 - bits(m).  The
 *     relative error of inv is below 1e-6, far inside what the quantizer's
 *     range argument needs (2^-16).  Group maxima outside [2^-100, 2^100] are
 *     not scaled: below, the group is stored as zero; above, the row is
 *     treated as overflow (stored as zero and flagged).
 *   - Stochastic rounding adds an 8-bit dither on a grid of 1/256 of a code
 *     step: t = fma(x, inv, 49152 + d/256); code = floor(t - 49152).  49152 is
 *     1.5 * 2^15, whose float spacing is exactly 1/256, so the fma rounds
 *     x*inv to the nearest 1/256 and adds d/256 exactly.  With d uniform in
 *     0..255 the code is unbiased up to that 1/512-step rounding.
 *   - The dither bytes come from a counter hash keyed on seed, step, sequence,
 *     head, row and column: SplitMix64 (Steele, Lea, Flood 2014) and the
 *     MurmurHash3 32-bit finalizer (Appleby) make the per-tile key; each
 *     16-column block of a row folds its counter once, and each of its four
 *     words folds that again with a multiplier of its own.  The
 *     pages fix no random source; what the method needs (Proposition 3) is a
 *     dither byte uniform on 0..255 and independent of x and of the other
 *     entries' bytes, which the tests check statistically.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -frounding-math -fPIC -shared
 * (no fast-math; fmaf is used only where the definition says fma).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Counter-based random bits                                                */
/* ------------------------------------------------------------------------ */

/* SplitMix64 output for generator state z (state advanced by the golden
 * gamma, then the variant-13 mixer).  Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; constants as published by
 * Vigna for splitmix64. */
uint64_t lo_splitmix64(uint64_t z)
{
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* MurmurHash3 32-bit finalizer (Appleby). */
uint32_t lo_fmix32(uint32_t h)
{
    h ^= h >> 16;
    h *= 0x85EBCA6Bu;
    h ^= h >> 13;
    h *= 0xC2B2AE35u;
    h ^= h >> 16;
    return h;
}

/* 32-bit key of one decode step of one handle. */
uint32_t lo_step_key(uint64_t seed, uint64_t step)
{
    uint64_t k = lo_splitmix64(seed ^ lo_splitmix64(step));
    return (uint32_t)(k ^ (k >> 32));
}

/* 32-bit key of one (sequence, head) tile: tile_index = b * H + h. */
uint32_t lo_tile_key(uint32_t step_key, uint32_t tile_index)
{
    return lo_fmix32(step_key + 0x85EBCA77u * (tile_index + 1u));
}

/* Multiply-fold: the low and high 32-bit halves of the 64-bit product a * b,
 * XORed. */
uint32_t lo_mulfold(uint32_t a, uint32_t b)
{
    uint64_t p = (uint64_t)a * (uint64_t)b;
    return (uint32_t)p ^ (uint32_t)(p >> 32);
}

/* Multipliers of the four words of a 16-column block. */
static const uint32_t kDitherMul[4] = {0x846CA68Bu, 0xCC9E2D51u, 0x1B873593u, 0xE6546B65u};

/* Dither word q (0..3) of the 16-column block whose counter is c: one multiply-fold of
 * c, then one with the word's own multiplier. */
uint32_t lo_dither_word(uint32_t c, int q)
{
    return lo_mulfold(lo_mulfold(c, 0x7FEB352Du), kDitherMul[q & 3]);
}

/* Dither byte d in 0..255 for state element (i, j) of a tile.  Row i is cut into
 * 16-column blocks; block n4 = i d_k/16 + j/16 has counter c = tile_key + golden *
 * (4 n4 + 1) (golden = 0x9E3779B9, mod 2^32), and four words, word q for columns
 * 16 n4 + 4q .. 16 n4 + 4q + 3; column j takes byte j mod 4 of word (j mod 16) / 4. */
uint32_t lo_dither(uint32_t tile_key, int d_k, int i, int j)
{
    uint32_t n4 = (uint32_t)i * (uint32_t)(d_k / 16) + (uint32_t)(j / 16);
    uint32_t h = lo_dither_word(tile_key + 0x9E3779B9u * (4u * n4 + 1u), (j % 16) / 4);
    return (h >> (8 * (j % 4))) & 0xFFu;
}

/* Dither words of count consecutive 4-column quads of a tile, quads n0, n0 + 1, ...
 * (quad n = word n mod 4 of block n / 4; for statistical tests of the stream). */
void lo_dither_words(uint32_t tile_key, uint32_t n0, int count, uint32_t *out)
{
    for (int k = 0; k < count; ++k) {
        uint32_t n = n0 + (uint32_t)k;
        out[k] = lo_dither_word(tile_key + 0x9E3779B9u * (4u * (n / 4u) + 1u), (int)(n % 4u));
    }
}

/* ------------------------------------------------------------------------ */
/* State layout                                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
    int d_k, d_v;      /* state is d_v x d_k (value rows, key columns)       */
    int group;         /* key entries per scale, divides d_k                 */
    int bits;          /* 4..8 (b-bit codes) or 32 (unquantized fp32 state)  */
    int delta;         /* 0 or 1: delta correction on/off                     */
    int diag;          /* 0: scalar decay; 1: decay per key column           */
    int stochastic;    /* 1: stochastic rounding; 0: round to nearest        */
    int axis;          /* 0: value-axis groups (scales [d_v][d_k/G]);
                        * 1: key-axis (one scale per key column, scales [d_k]) */
    const int *group_bits; /* NULL, or bits (4..8) of each of the d_k/G key groups:
                            * per-channel precision (value axis only; bits unused) */
    int dense;         /* 1: 5- to 7-bit codes in bit planes (see dense_*); 0: one
                        * byte per code.  Per-head bits only (group_bits NULL). */
} lo_cfg;

static int code_max(int bits) { return (1 << (bits - 1)) - 1; }

/* Bits of key group g, and its storage: 4-bit codes as nibbles, 5 to 8 bits in bytes. */
static int group_bits_of(const lo_cfg *c, int g) { return c->group_bits ? c->group_bits[g] : c->bits; }
static int storage_of(int bits) { return bits == 4 ? 4 : 8; }

/* A quantized row stores its key groups back to back, group g in
 * G * storage(bits_g) / 8 bytes (with equal bits: the plain row-major layout). */
static size_t group_offset(const lo_cfg *c, int g)
{
    size_t off = 0;
    for (int h = 0; h < g; h++)
        off += (size_t)c->group * storage_of(group_bits_of(c, h)) / 8;
    return off;
}
static size_t quant_row_bytes(const lo_cfg *c) { return group_offset(c, c->d_k / c->group); }

/* Dense b-bit codes, b = 5, 6, 7 (cfg.dense = 1).  A code c is stored in offset binary,
 * u = c + 2^(b-1) in [1, 2^b - 1], split into bit planes laid out one row after another:
 *   row = [4-bit plane: d_k/2 bytes][2-bit plane: d_k/4 bytes if b >= 6]
 *         [1-bit plane: d_k/8 bytes if b is odd], padded to a multiple of 8 bytes.
 * 4-bit plane: u & 15 of column j in byte j/2, low nibble for even j (the int4 layout).
 * 2-bit plane: (u >> 4) & 3; the 16-column block l owns the 4 bytes at 4l; inside the
 *   block, byte p (p = 0..3) holds column 8+2p in bits 0-1, column 9+2p in bits 2-3,
 *   column 2p in bits 4-5 and column 2p+1 in bits 6-7.
 * 1-bit plane: the top bit of u (bit 4 for b = 5, bit 6 for b = 7); block l owns the 2
 *   bytes at 2l; byte 0 holds columns 0, 2, 4, 6 in bits 0-3 and columns 1, 3, 5, 7 in
 *   bits 4-7, byte 1 likewise columns 8..15.
 * (These positions let a lane that holds 16 columns rebuild each code's byte with a few
 * shifts and masks per 4 codes.) */
static int is_dense(const lo_cfg *c) { return c->dense && !c->group_bits && c->bits >= 5 && c->bits <= 7; }
static size_t dense_row_bytes(const lo_cfg *c)
{
    size_t b = (size_t)c->d_k * c->bits / 8;
    return (b + 7) / 8 * 8;
}
static size_t plane2_offset(const lo_cfg *c) { return (size_t)c->d_k / 2; }
static size_t plane1_offset(const lo_cfg *c) { return (size_t)c->d_k / 2 + (c->bits >= 6 ? (size_t)c->d_k / 4 : 0); }
/* byte and bit of column j's field in the 2-bit / 1-bit plane of a row */
static void plane2_pos(int j, size_t *byte, int *bit)
{
    int l = j / 16, cc = j % 16, p = (cc % 8) / 2;
    *byte = (size_t)4 * l + p;
    *bit = cc < 8 ? (cc % 2 == 0 ? 4 : 6) : (cc % 2 == 0 ? 0 : 2);
}
static void plane1_pos(int j, size_t *byte, int *bit)
{
    int l = j / 16, cc = j % 16, half = cc / 8, k = cc % 8;
    *byte = (size_t)2 * l + half;
    *bit = (k % 2 == 0) ? k / 2 : 4 + k / 2;
}
static int dense_get(const lo_cfg *c, const uint8_t *codes, int i, int j)
{
    const uint8_t *row = codes + (size_t)i * dense_row_bytes(c);
    uint8_t nb = row[j / 2];
    int u = (j % 2 == 0) ? (nb & 0xF) : (nb >> 4);
    size_t at;
    int bit;
    if (c->bits >= 6) {
        plane2_pos(j, &at, &bit);
        u |= ((row[plane2_offset(c) + at] >> bit) & 3) << 4;
    }
    if (c->bits % 2 == 1) {
        plane1_pos(j, &at, &bit);
        u |= ((row[plane1_offset(c) + at] >> bit) & 1) << (c->bits - 1);
    }
    return u - (1 << (c->bits - 1));
}
static void dense_put(const lo_cfg *c, uint8_t *codes, int i, int j, int code)
{
    uint8_t *row = codes + (size_t)i * dense_row_bytes(c);
    int u = code + (1 << (c->bits - 1));
    uint8_t *nb = &row[j / 2];
    if (j % 2 == 0)
        *nb = (uint8_t)((*nb & 0xF0) | (u & 0xF));
    else
        *nb = (uint8_t)((*nb & 0x0F) | ((u & 0xF) << 4));
    size_t at;
    int bit;
    if (c->bits >= 6) {
        plane2_pos(j, &at, &bit);
        uint8_t *q = &row[plane2_offset(c) + at];
        *q = (uint8_t)((*q & ~(3 << bit)) | (((u >> 4) & 3) << bit));
    }
    if (c->bits % 2 == 1) {
        plane1_pos(j, &at, &bit);
        uint8_t *q = &row[plane1_offset(c) + at];
        *q = (uint8_t)((*q & ~(1 << bit)) | (((u >> (c->bits - 1)) & 1) << bit));
    }
}

/* Read code (i, j) from a packed tile.  5 to 8 bits: one byte per code, two's
 * complement (or the dense planes above).  4 bits: two codes per byte, even column in
 * the low nibble, odd column in the high nibble, two's complement nibbles. */
static int get_code(const lo_cfg *c, const uint8_t *codes, int i, int j)
{
    if (is_dense(c))
        return dense_get(c, codes, i, j);
    int g = j / c->group, jj = j - g * c->group;
    const uint8_t *grp = codes + (size_t)i * quant_row_bytes(c) + group_offset(c, g);
    if (group_bits_of(c, g) != 4)
        return (int)(int8_t)grp[jj];
    uint8_t byte = grp[jj / 2];
    int nib = (jj % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return nib >= 8 ? nib - 16 : nib;
}

static void put_code(const lo_cfg *c, uint8_t *codes, int i, int j, int code)
{
    if (is_dense(c)) {
        dense_put(c, codes, i, j, code);
        return;
    }
    int g = j / c->group, jj = j - g * c->group;
    uint8_t *grp = codes + (size_t)i * quant_row_bytes(c) + group_offset(c, g);
    if (group_bits_of(c, g) != 4) {
        grp[jj] = (uint8_t)(int8_t)code;
        return;
    }
    size_t at = (size_t)jj / 2;
    uint8_t nib = (uint8_t)(code & 0xF);
    if (jj % 2 == 0)
        grp[at] = (uint8_t)((grp[at] & 0xF0) | nib);
    else
        grp[at] = (uint8_t)((grp[at] & 0x0F) | (nib << 4));
}

int lo_get_code(const lo_cfg *c, const uint8_t *codes, int i, int j) { return get_code(c, codes, i, j); }
void lo_put_code(const lo_cfg *c, uint8_t *codes, int i, int j, int code) { put_code(c, codes, i, j, code); }

/* ------------------------------------------------------------------------ */
/* Fixed-order dot product                                                  */
/* ------------------------------------------------------------------------ */

/* sum_j a_j b_j for n = 16*L, L a power of two <= 16.  The row is cut into L
 * blocks of 16 consecutive columns.  In block l, chain (h, p) (h = 0, 1 the
 * half of the block, p = 0, 1 the column parity) is a sequential fma chain from
 * zero over columns 16l + 8h + p + 2m, m = 0..3 ascending; the block sum is
 * (chain(0,0) + chain(1,0)) + (chain(0,1) + chain(1,1)).  The L block sums are
 * then combined pairwise, partner at distance 1, then 2, 4, ..., L/2. */
float lo_dot_b16(const float *a, const float *b, int n)
{
    float p[16], nxt[16];
    int L = n / 16;
    for (int l = 0; l < L; l++) {
        float ch[2][2];
        for (int h = 0; h < 2; h++)
            for (int par = 0; par < 2; par++) {
                float acc = 0.0f;
                for (int m = 0; m < 4; m++) {
                    int j = 16 * l + 8 * h + par + 2 * m;
                    acc = fmaf(a[j], b[j], acc);
                }
                ch[h][par] = acc;
            }
        p[l] = (ch[0][0] + ch[1][0]) + (ch[0][1] + ch[1][1]);
    }
    for (int stride = 1; stride < L; stride *= 2) {
        for (int l = 0; l < L; l++)
            nxt[l] = p[l] + p[l ^ stride];
        memcpy(p, nxt, sizeof(float) * L);
    }
    return p[0];
}

/* Approximate 1/m for m in [2^-100, 2^100]: seed from reflecting the exponent
 * field (exact for powers of two, within 12.5% otherwise), then three
 * Newton-Raphson steps for f(y) = 1/y - m, written y <- y + y (1 - m y) with
 * fmas.  Each step squares the relative error: 1.3e-1 -> 1.6e-2 -> 2.4e-4 -> ~1e-7. */
float lo_recip_nr(float m)
{
    uint32_t bm, by;
    float y;
    memcpy(&bm, &m, 4);
    by = 0x7F000000u - bm;
    memcpy(&y, &by, 4);
    for (int it = 0; it < 3; it++) {
        float e = fmaf(-m, y, 1.0f);
        y = fmaf(y, e, y);
    }
    return y;
}

/* ------------------------------------------------------------------------ */
/* Exact projection for rows of integer codes with one scale                */
/* ------------------------------------------------------------------------ */

/* The heads whose projection u = S'k is the exact integer contraction: codes one
 * byte or one nibble each, one scale per value row. */
static int exact_projection(const lo_cfg *c)
{
    return c->bits != 32 && !is_dense(c) && !c->group_bits && !c->axis && c->group == c->d_k;
}

/* Fixed-point copy of p_j = alpha_j y_j (exact in double): E = 29 - floor(log2 max|p|)
 * so that max|p| 2^E lies in [2^29, 2^30), and Y_j = rint(p_j 2^E) (ties to even),
 * |Y_j| <= 2^30.  All p zero: E = 0, Y = 0.  Returns 0 if some p_j is not finite. */
int lo_fixed_point(const float *alpha, int diag, const float *y, int n, int32_t *Y, int *E)
{
    double m = 0.0;
    for (int j = 0; j < n; j++) {
        double p = (double)(diag ? alpha[j] : alpha[0]) * (double)y[j];
        if (!isfinite(p))
            return 0;
        if (fabs(p) > m)
            m = fabs(p);
    }
    int e = 0;
    *E = 0;
    if (m > 0.0) {
        frexp(m, &e);          /* m = f 2^e, f in [1/2, 1): floor(log2 m) = e - 1 */
        *E = 30 - e;
    }
    for (int j = 0; j < n; j++) {
        double p = (double)(diag ? alpha[j] : alpha[0]) * (double)y[j];
        Y[j] = (int32_t)nearbyint(ldexp(p, *E));
    }
    return 1;
}

/* u_i = fl32(fl64(s_i U_i) 2^-E) with U_i = sum_j c_ij Y_j, the integer sum exact. */
float lo_exact_projection(const lo_cfg *c, const uint8_t *codes, float s, int i,
                          const int32_t *Y, int E)
{
    int64_t U = 0;
    for (int j = 0; j < c->d_k; j++)
        U += (int64_t)get_code(c, codes, i, j) * (int64_t)Y[j];
    return (float)ldexp((double)s * (double)U, -E);
}

/* ------------------------------------------------------------------------ */
/* Requantization of one value row (Proposition 1 scale, SR or RTN)         */
/* ------------------------------------------------------------------------ */

/* x: the updated fp32 row (d_k entries).  Writes the row's codes and its
 * d_k/G scales; group g uses r = 2^(b_g - 1) - 1 of its own bit width.  A row
 * that holds a non-finite entry (or one above 2^100) is stored as zero (scales
 * 0, codes 0) and reported with return value 1. */
static int requantize_row(const lo_cfg *c, const float *x, int i, uint32_t tile_key,
                          uint8_t *codes, float *scales)
{
    const float m_lo = 0x1p-100f, m_hi = 0x1p100f;
    const int ng = c->d_k / c->group;
    int bad = 0;
    for (int j = 0; j < c->d_k; j++)
        if (!isfinite(x[j]))
            bad = 1;
    for (int g = 0; g < ng && !bad; g++)
        for (int j = g * c->group; j < (g + 1) * c->group; j++)
            if (fabsf(x[j]) > m_hi)
                bad = 1;                  /* overflow: treated like a non-finite row */
    for (int g = 0; g < ng; g++) {
        const int r = code_max(group_bits_of(c, g));
        const float inv_r = 1.0f / (float)r;              /* fl(1/r), round to nearest */
        float m = 0.0f;
        for (int j = g * c->group; j < (g + 1) * c->group; j++)
            if (fabsf(x[j]) > m)
                m = fabsf(x[j]);
        float inv = 0.0f, s = 0.0f;
        if (!bad && m >= m_lo) {
            inv = (float)r * lo_recip_nr(m);
            s = m * inv_r;
        }
        scales[(size_t)i * ng + g] = s;
        for (int j = g * c->group; j < (g + 1) * c->group; j++) {
            int code = 0;
            if (inv != 0.0f) {
                float d = c->stochastic ? (float)lo_dither(tile_key, c->d_k, i, j) : 128.0f;
                float t = fmaf(x[j], inv, 49152.0f + d / 256.0f);
                code = (int)floorf(t - 49152.0f);
            }
            put_code(c, codes, i, j, code);
        }
    }
    return bad;
}

/* Key-axis requantization of a whole tile X (d_v x d_k): one scale per key column,
 * s_j = m_j * fl(1/r) with m_j = max_i |X_ij| (Proposition 1's column range C_j).  A
 * column with an entry that is inf, NaN or above 2^100 is stored as zero (scale 0,
 * codes 0) and reported with return value 1; a column whose maximum is below 2^-100 is
 * stored as zero. */
static int requantize_tile_key(const lo_cfg *c, const float *X, uint32_t tile_key,
                               uint8_t *codes, float *scales)
{
    const int r = code_max(c->bits);
    const float inv_r = 1.0f / (float)r;
    int flag = 0;
    for (int j = 0; j < c->d_k; j++) {
        int bad = 0;
        float m = 0.0f;
        for (int i = 0; i < c->d_v; i++) {
            float a = X[(size_t)i * c->d_k + j];
            if (!isfinite(a) || fabsf(a) > 0x1p100f)
                bad = 1;
            else if (fabsf(a) > m)
                m = fabsf(a);
        }
        float inv = 0.0f, s = 0.0f;
        if (!bad && m >= 0x1p-100f) {
            inv = (float)r * lo_recip_nr(m);
            s = m * inv_r;
        }
        flag |= bad;
        scales[j] = s;
        for (int i = 0; i < c->d_v; i++) {
            int code = 0;
            if (inv != 0.0f) {
                float d = c->stochastic ? (float)lo_dither(tile_key, c->d_k, i, j) : 128.0f;
                float t = fmaf(X[(size_t)i * c->d_k + j], inv, 49152.0f + d / 256.0f);
                code = (int)floorf(t - 49152.0f);
            }
            put_code(c, codes, i, j, code);
        }
    }
    return flag;
}

/* ------------------------------------------------------------------------ */
/* One decode step of one (sequence, head) tile                             */
/* ------------------------------------------------------------------------ */

/* state: packed codes (bits 8/4) or float[d_v*d_k] (bits 32), updated in place.
 * scales: float[d_v * d_k/G] (ignored for bits 32), updated in place.
 * q, k: d_k floats; v: d_v floats; alpha: 1 float (scalar decay) or d_k
 * floats (diag); beta: scalar.  o_out: d_v doubles.  x_out (optional, may be
 * NULL): the updated fp32 state before requantization, d_v*d_k floats.
 * Returns 1 if any row held a non-finite value, else 0. */
int lo_tile_step(const lo_cfg *c, void *state, float *scales,
                 const float *q, const float *k, const float *v,
                 const float *alpha, float beta, uint32_t tile_key,
                 double *o_out, float *x_out)
{
    const int dk = c->d_k, ng = dk / c->group;
    float *Sp = malloc(sizeof(float) * dk);   /* S_{t-1} diag(alpha), one row */
    float *x = malloc(sizeof(float) * dk);    /* S_t, one row                 */
    float *X = (c->axis && c->bits != 32) ? malloc(sizeof(float) * dk * (size_t)c->d_v) : NULL;
    int flag = 0;
    /* exact projection: the fixed-point alpha k, once per tile */
    const int exact = c->delta && exact_projection(c);
    int32_t *Y = exact ? malloc(sizeof(int32_t) * dk) : NULL;
    int E = 0, kfinite = 1;
    if (exact)
        kfinite = lo_fixed_point(alpha, c->diag, k, dk, Y, &E);
    for (int i = 0; i < c->d_v; i++) {
        /* dequantize and decay: entry (i, j) is c_ij * (s_ig * alpha_j) */
        for (int j = 0; j < dk; j++) {
            float aj = c->diag ? alpha[j] : alpha[0];
            if (c->bits == 32) {
                Sp[j] = ((float *)state)[(size_t)i * dk + j] * aj;
            } else {
                float s = c->axis ? scales[j] : scales[(size_t)i * ng + j / c->group];
                Sp[j] = (float)get_code(c, (uint8_t *)state, i, j) * (s * aj);
            }
        }
        /* write: w_i = beta (v_i - delta u_i), u_i = (S' k)_i */
        float w;
        if (exact) {
            float u = kfinite ? lo_exact_projection(c, (const uint8_t *)state, scales[i], i, Y, E) : NAN;
            w = beta * (v[i] - u);
        } else if (c->delta) {
            float u = lo_dot_b16(Sp, k, dk);
            w = beta * (v[i] - u);
        } else {
            w = beta * v[i];
        }
        for (int j = 0; j < dk; j++)
            x[j] = fmaf(w, k[j], Sp[j]);
        /* readout o_i = (S_t q)_i with S_t = S' + w k^T evaluated exactly (in double)
         * from the fp32 S' and w, before any rounding of the stored state */
        double o = 0.0;
        for (int j = 0; j < dk; j++)
            o += ((double)Sp[j] + (double)w * (double)k[j]) * (double)q[j];
        o_out[i] = o;
        if (x_out)
            memcpy(x_out + (size_t)i * dk, x, sizeof(float) * dk);
        /* requantize (or store the fp32 state) */
        if (c->bits == 32) {
            for (int j = 0; j < dk; j++) {
                if (!isfinite(x[j]))
                    flag = 1;
                ((float *)state)[(size_t)i * dk + j] = x[j];
            }
        } else if (c->axis) {
            memcpy(X + (size_t)i * dk, x, sizeof(float) * dk);   /* quantized after all rows */
        } else {
            flag |= requantize_row(c, x, i, tile_key, (uint8_t *)state, scales);
        }
    }
    if (X) {
        flag |= requantize_tile_key(c, X, tile_key, (uint8_t *)state, scales);
        free(X);
    }
    free(Sp);
    free(x);
    free(Y);
    return flag;
}

/* ------------------------------------------------------------------------ */
/* The plain definition of the same step                                    */
/* ------------------------------------------------------------------------ */

/* One decode step written as the pages state it, with none of the evaluation
 * choices above: every product and sum in double precision in plain order,
 *   S'_ij = c_ij s_ig alpha_j,  u_i = sum_j S'_ij k_j,  w_i = beta (v_i - delta u_i),
 *   x_ij = S'_ij + w_i k_j,     o_i = sum_j x_ij q_j,
 * and the requantization of Proposition 1 and Proposition 3 with plain division:
 * per group m = max |x|, the stored scale s = m / r rounded once to fp32, y = x r / m,
 * code = floor(y + (d + 1/2) / 256) with the same dither byte d as the step above (an
 * 8-bit uniform offset in (0, 1)), or floor(y + 1/2) for round to nearest, clamped to
 * [-r, r].  The non-finite, overflow (above 2^100) and tiny (below 2^-100) rules are the
 * step's.  Key-axis groups: m and the scale per key column over the tile.
 * The evaluated step (lo_tile_step) must agree with this one within the parity bounds:
 * its fixed fp32 dot order, Newton reciprocal and 1/256-grid quantizer are evaluation
 * choices, not a different method.  Same arguments and results as lo_tile_step
 * (x_out: x rounded to fp32). */
static int quantize_group_plain(const lo_cfg *c, const double *x, int n, int stride, int bits,
                                const uint32_t *dither, int *codes_out, float *s_out)
{
    const int r = code_max(bits);
    double m = 0.0;
    int bad = 0;
    for (int a = 0; a < n; a++) {
        double v = x[(size_t)a * stride];
        if (!isfinite(v) || fabs(v) > 0x1p100)
            bad = 1;
        else if (fabs(v) > m)
            m = fabs(v);
    }
    if (bad || m < 0x1p-100) {
        for (int a = 0; a < n; a++)
            codes_out[a] = 0;
        *s_out = 0.0f;
        return bad;
    }
    *s_out = (float)(m / (double)r);
    for (int a = 0; a < n; a++) {
        double y = x[(size_t)a * stride] * (double)r / m;
        double u = c->stochastic ? ((double)dither[a] + 0.5) / 256.0 : 0.5;
        int code = (int)floor(y + u);
        if (code > r) code = r;
        if (code < -r) code = -r;
        codes_out[a] = code;
    }
    return 0;
}

int lo_tile_step_plain(const lo_cfg *c, void *state, float *scales,
                       const float *q, const float *k, const float *v,
                       const float *alpha, float beta, uint32_t tile_key,
                       double *o_out, float *x_out)
{
    const int dk = c->d_k, dv = c->d_v, ng = dk / c->group;
    double *X = malloc(sizeof(double) * (size_t)dk * dv);
    double *Sp = malloc(sizeof(double) * dk);
    uint32_t *dith = malloc(sizeof(uint32_t) * (dk > dv ? dk : dv));
    int *cod = malloc(sizeof(int) * (dk > dv ? dk : dv));
    int flag = 0;
    for (int i = 0; i < dv; i++) {
        for (int j = 0; j < dk; j++) {
            double aj = c->diag ? alpha[j] : alpha[0];
            if (c->bits == 32)
                Sp[j] = (double)((float *)state)[(size_t)i * dk + j] * aj;
            else {
                double s = c->axis ? scales[j] : scales[(size_t)i * ng + j / c->group];
                Sp[j] = (double)get_code(c, (uint8_t *)state, i, j) * s * aj;
            }
        }
        double u = 0.0;
        for (int j = 0; j < dk; j++)
            u += Sp[j] * (double)k[j];
        double w = (double)beta * ((double)v[i] - (c->delta ? u : 0.0));
        double o = 0.0;
        for (int j = 0; j < dk; j++) {
            double xv = Sp[j] + w * (double)k[j];
            X[(size_t)i * dk + j] = xv;
            o += xv * (double)q[j];
        }
        o_out[i] = o;
    }
    if (x_out)
        for (size_t e = 0; e < (size_t)dk * dv; e++)
            x_out[e] = (float)X[e];
    if (c->bits == 32) {
        for (size_t e = 0; e < (size_t)dk * dv; e++) {
            float f = (float)X[e];
            if (!isfinite(f))
                flag = 1;
            ((float *)state)[e] = f;
        }
    } else if (c->axis) {
        for (int j = 0; j < dk; j++) {
            for (int i = 0; i < dv; i++)
                dith[i] = lo_dither(tile_key, dk, i, j);
            flag |= quantize_group_plain(c, X + j, dv, dk, c->bits, dith, cod, &scales[j]);
            for (int i = 0; i < dv; i++)
                put_code(c, (uint8_t *)state, i, j, cod[i]);
        }
    } else {
        for (int i = 0; i < dv; i++) {
            /* a row with any non-finite (or overflowing) entry is stored as zero */
            int rowbad = 0;
            for (int j = 0; j < dk; j++) {
                double xv = X[(size_t)i * dk + j];
                if (!isfinite(xv) || fabs(xv) > 0x1p100)
                    rowbad = 1;
            }
            for (int g = 0; g < ng; g++) {
                const int j0 = g * c->group;
                for (int j = 0; j < c->group; j++)
                    dith[j] = lo_dither(tile_key, dk, i, j0 + j);
                float s;
                quantize_group_plain(c, X + (size_t)i * dk + j0, c->group, 1,
                                     group_bits_of(c, g), dith, cod, &s);
                if (rowbad) {
                    s = 0.0f;
                    for (int j = 0; j < c->group; j++)
                        cod[j] = 0;
                }
                scales[(size_t)i * ng + g] = s;
                for (int j = 0; j < c->group; j++)
                    put_code(c, (uint8_t *)state, i, j0 + j, cod[j]);
            }
            flag |= rowbad;
        }
    }
    free(X);
    free(Sp);
    free(dith);
    free(cod);
    return flag;
}

/* Quantize an fp32 tile S (d_v x d_k) into codes and scales with the same
 * quantizer as the decode step.  Returns 1 if a row was non-finite. */
int lo_tile_quantize(const lo_cfg *c, const float *S, uint8_t *codes, float *scales,
                     uint32_t tile_key)
{
    if (c->axis)
        return requantize_tile_key(c, S, tile_key, codes, scales);
    int flag = 0;
    for (int i = 0; i < c->d_v; i++)
        flag |= requantize_row(c, S + (size_t)i * c->d_k, i, tile_key, codes, scales);
    return flag;
}

/* Dequantize a tile: S_ij = c_ij * s_ig. */
void lo_tile_dequant(const lo_cfg *c, const uint8_t *codes, const float *scales, float *S)
{
    const int ng = c->d_k / c->group;
    for (int i = 0; i < c->d_v; i++)
        for (int j = 0; j < c->d_k; j++)
            S[(size_t)i * c->d_k + j] =
                (float)get_code(c, codes, i, j) *
                (c->axis ? scales[j] : scales[(size_t)i * ng + j / c->group]);
}

/* ------------------------------------------------------------------------ */
/* Decay-based mixed precision (create time)                                */
/* ------------------------------------------------------------------------ */

/* The round(frac_high * H) heads with the largest mean decay (slowest to
 * forget) get bits_high, the rest bits_low.  Equal decays: lower head index
 * first.  Plain selection, one head at a time. */
void lo_assign_bits_by_decay(const float *mean_decay, int H, float frac_high,
                             int bits_high, int bits_low, int *out_bits)
{
    int n_high = (int)floor((double)frac_high * (double)H + 0.5);
    if (n_high < 0) n_high = 0;
    if (n_high > H) n_high = H;
    char *taken = calloc((size_t)H, 1);
    for (int h = 0; h < H; h++)
        out_bits[h] = bits_low;
    for (int n = 0; n < n_high; n++) {
        int best = -1;
        for (int h = 0; h < H; h++)
            if (!taken[h] && (best < 0 || mean_decay[h] > mean_decay[best]))
                best = h;
        taken[best] = 1;
        out_bits[best] = bits_high;
    }
    free(taken);
}
