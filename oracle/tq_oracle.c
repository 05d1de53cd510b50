/*
 * tq_oracle.c -- plain, slow CPU oracle for the ternary weight-only grouped
 * linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant generator with the CUDA library; it is written from the
 * definitions on the pages it cites, one step at a time, with no blocking,
 * fusion or reordering beyond what those definitions state.
 *
 * Sources (page title, section):
 *   [codec]  precisit/pack-unpack-run, the codec.py description: the group
 *            scale is the mean of |w| kept as fp16; trits round w / scale
 *            half to even; base-3 digits, five to a byte; each group starts
 *            on a byte boundary, its unused digit slots holding the zero
 *            trit; byte values 243..255 are invalid; the decoder gives bf16.
 *   [rules]  precisit/pack-unpack-run, the paragraph after it: no calibration;
 *            a scale stored as zero decodes to an all-zero group; G divides
 *            the number of columns.
 *   [rate]   precisit/pack-unpack-run, payload-rate paragraph:
 *            8*(ceil(G/5)+2)/G bits per weight.
 *   [two]    "Autoregressive Language Model on the 6502 Processor", summary:
 *            BitNet ternary weights (-1, 0, 1) packed four parameters per
 *            byte (the 2-bit alternative to the base-3 codec).
 *   [w4]     tiny-llm "Week 2 Day 3: Quantize the Model", "Group-Wise Affine
 *            Quantization", "Reconstruct a Stored Group" and "Packed Storage
 *            Layout": unsigned 4-bit codes, eight per 32-bit word with the
 *            first code in the low nibble; per group of G columns a bf16
 *            scale (signed) and a bf16 bias; weight = q * scale + bias.
 *   [mm]     tiny-llm "Week 2 Day 3: Quantize the Model", "Mathematical
 *            Formulation" and "Computation Flow": C[i,k] = sum_j A[i,j]*B[k,j]
 *            with B reconstructed per group of G input columns, accumulated in
 *            float.
 *
 * Readings where the pages leave a step open (each one is a documented
 * choice, listed with its reason in the design notes):
 *   - the mean is the exact rational (sum |w|)/G, rounded once to binary16
 *     with ties to even (order-free, so any correct implementation agrees);
 *   - trit -> base-3 digit is d = t + 1 (-1 -> 0, 0 -> 1, +1 -> 2);
 *   - the first weight of a byte is its least-significant digit (x 3^0);
 *   - padding digits are the zero trit, d = 1; a decoder rejects a group
 *     whose padding digits are anything else;
 *   - a group whose mean rounds to +0 stores scale +0 and all-zero trits;
 *   - a group holding a NaN/Inf weight, or whose mean overflows binary16,
 *     is flagged and stored as a zero group;
 *   - decoded weight = +0 for a zero trit or zero scale, else
 *     sign(t) * RNE_bf16(scale); a group that fails validation decodes to
 *     bf16 NaN so that any product with it is NaN;
 *   - matmul reference: fp64 sum of exact products of bf16 activations and
 *     decoded bf16 weights.
 *   - 2-bit format [two]: the same groups, scales and trits as the base-3
 *     codec; code c = t + 1 in two bits, four per byte, the first weight in
 *     the least-significant bits; ceil(G/4) bytes per group, byte-aligned,
 *     padding codes 1 (zero trit); code 3 is invalid (error bit 1, like a
 *     byte >= 243), a padding code other than 1 sets error bit 2.
 *
 * Error bits returned (same meaning as the library's asynchronous flags):
 *   1  a code byte >= 243          2  non-canonical padding digit
 *   4  non-finite weight           8  stored scale NaN/Inf/negative
 *   16 group mean overflows binary16
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ERR_BYTE     1u
#define ERR_PADDING  2u
#define ERR_WEIGHT   4u
#define ERR_SCALE    8u
#define ERR_OVERFLOW 16u

/* ------------------------------------------------------------------ */
/* Number formats, written from the IEEE 754 binary16 definition and   */
/* the bfloat16 definition (binary32 with the low 16 bits dropped).    */
/* ------------------------------------------------------------------ */

/* Exact value of a bfloat16 bit pattern. */
double oracle_bf16_value(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 7) & 0xFF;
    int f = h & 0x7F;
    double v;
    if (e == 0xFF)
        return f ? NAN : (sign ? -INFINITY : INFINITY);
    if (e == 0)
        v = ldexp((double)f, -133);            /* subnormal: f * 2^-126 / 2^7 */
    else
        v = ldexp((double)(f | 0x80), e - 134); /* (1.f) * 2^(e-127)         */
    return sign ? -v : v;
}

/* Exact value of a binary16 bit pattern. */
double oracle_fp16_value(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0x1F)
        return f ? NAN : (sign ? -INFINITY : INFINITY);
    if (e == 0)
        v = ldexp((double)f, -24);
    else
        v = ldexp((double)(f | 0x400), e - 25);
    return sign ? -v : v;
}

/* Round a double to the nearest bfloat16, ties to even. */
uint16_t oracle_bf16_round(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return sign | 0x7F80;
    int ex;
    frexp(a, &ex);               /* a = fr * 2^ex, fr in [0.5, 1) */
    int E = ex - 1;              /* floor(log2 a)                 */
    int qexp = (E < -126) ? -133 : E - 7;   /* quantum of the target binade */
    double q = ldexp(a, -qexp);  /* exact: scaling by a power of two */
    double n = floor(q);
    double rem = q - n;          /* exact */
    if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0))
        n += 1.0;
    uint32_t bits;
    if (E < -126)
        bits = (uint32_t)n;      /* subnormal; n == 128 encodes 2^-126 */
    else
        bits = ((uint32_t)(E + 127) << 7) + ((uint32_t)n - 128u);
    if (bits >= 0x7F80)
        return sign | 0x7F80;
    return sign | (uint16_t)bits;
}

/* ------------------------------------------------------------------ */
/* Exact group sum: a little-endian big integer of 32-bit limbs in     */
/* units of 2^-133, the smallest bfloat16 subnormal.  Every finite     */
/* bfloat16 magnitude is an integer number of these units below 2^262. */
/* ------------------------------------------------------------------ */

#define NLIMB 12 /* 384 bits: 262 bits per value + up to 2^32 addends */

typedef struct {
    uint32_t l[NLIMB];
} bigsum;

static void big_add_shifted(bigsum *s, uint32_t m, int shift)
{
    /* s += m * 2^shift, m < 2^32 */
    int limb = shift / 32, bit = shift % 32;
    uint64_t add = (uint64_t)m << bit;  /* at most 64 bits wide */
    uint64_t carry = 0;
    for (int i = limb; i < NLIMB; i++) {
        uint64_t t = (uint64_t)s->l[i] + (add & 0xFFFFFFFFu) + carry;
        s->l[i] = (uint32_t)t;
        carry = t >> 32;
        add >>= 32;
        if (add == 0 && carry == 0)
            break;
    }
}

/* q = s / d, returns the remainder; d > 0. */
static uint32_t big_divmod(const bigsum *s, uint32_t d, bigsum *q)
{
    uint64_t r = 0;
    for (int i = NLIMB - 1; i >= 0; i--) {
        uint64_t cur = (r << 32) | s->l[i];
        q->l[i] = (uint32_t)(cur / d);
        r = cur % d;
    }
    return (uint32_t)r;
}

static int big_msb(const bigsum *s) /* -1 if zero */
{
    for (int i = NLIMB - 1; i >= 0; i--)
        if (s->l[i])
            return i * 32 + 31 - __builtin_clz(s->l[i]);
    return -1;
}

static int big_bit(const bigsum *s, int k)
{
    if (k < 0 || k >= NLIMB * 32)
        return 0;
    return (s->l[k / 32] >> (k % 32)) & 1;
}

/* Is any bit of s below position k set? */
static int big_any_below(const bigsum *s, int k)
{
    for (int i = 0; i < k && i < NLIMB * 32; i++)
        if (big_bit(s, i))
            return 1;
    return 0;
}

/*
 * [codec] the group scale: mean of |w|, kept as fp16.
 * Computes S = sum |w_j| exactly, then s = RNE_binary16(S / G) by exact
 * comparison with the binary16 grid.  Returns error bits; *s_out is the
 * stored scale (+0 for an all-zero, tiny, non-finite or overflowing group).
 */
uint32_t oracle_group_scale(const uint16_t *w, int64_t G, uint16_t *s_out)
{
    bigsum S;
    memset(&S, 0, sizeof S);
    *s_out = 0;
    for (int64_t j = 0; j < G; j++) {
        uint16_t a = w[j] & 0x7FFF;              /* |w_j| */
        int e = a >> 7, f = a & 0x7F;
        if (e == 0xFF)
            return ERR_WEIGHT;                   /* NaN or Inf weight */
        if (e == 0)
            big_add_shifted(&S, (uint32_t)f, 0);               /* f * 2^-133 */
        else
            big_add_shifted(&S, (uint32_t)(f | 0x80), e - 1);  /* (1.f)*2^(e-127) */
    }
    /* mean = S / G in units of 2^-133: integer part Q, remainder r */
    bigsum Q;
    uint32_t r = big_divmod(&S, (uint32_t)G, &Q);
    int P = big_msb(&Q);
    if (P < 0)
        return 0;                 /* mean < 2^-133: rounds to +0 */
    int E = P - 133;              /* floor(log2(mean)) */
    if (E > 15)
        return ERR_OVERFLOW;      /* mean >= 2^16 > largest finite binary16 */
    int Eeff = E < -14 ? -14 : E; /* binary16 subnormals share the 2^-14 binade */
    int k = (Eeff - 10) + 133;    /* one binary16 ulp = 2^k units */
    /* significand: floor(mean / ulp), at most 11 bits */
    uint32_t mant = 0;
    for (int i = 0; i < 12; i++)
        mant |= (uint32_t)big_bit(&Q, k + i) << i;
    /* round half to even on the discarded part (Q mod 2^k) + r/G */
    int half_bit = big_bit(&Q, k - 1);
    int below_half_nonzero = big_any_below(&Q, k - 1) || r != 0;
    int up = half_bit && (below_half_nonzero || (mant & 1));
    mant += up;
    uint32_t bits = ((uint32_t)(Eeff + 14) << 10) + mant;
    if (bits >= 0x7C00)
        return ERR_OVERFLOW;      /* rounded up to infinity */
    *s_out = (uint16_t)bits;
    return 0;
}

/*
 * [codec] trits by rounding half to even, [rules] zero scale => zero group.
 * t = clamp(round_half_even(w / s), -1, +1); the quotient of a bf16 by a
 * binary16 is computed in binary64, where it is exact enough that no false
 * tie can appear (a true quotient near 1/2 differs from it by far more than
 * one binary64 ulp), and nearbyint rounds half to even.
 */
int oracle_trit(uint16_t w, uint16_t s)
{
    if (s == 0)
        return 0;
    double q = oracle_bf16_value(w) / oracle_fp16_value(s);
    double t = nearbyint(q); /* default rounding mode: nearest, ties to even */
    if (t > 1.0)
        t = 1.0;
    if (t < -1.0)
        t = -1.0;
    return (int)t;
}

/* [codec] bytes per group: ceil(G/5) */
int64_t oracle_bytes_per_group(int64_t G)
{
    return (G + 4) / 5;
}

/*
 * Quantize and pack one row-major [N x K] bf16 matrix.
 * codes:  [N][K/G][ceil(G/5)] bytes, scales: [N][K/G] binary16.
 * Returns the OR of every group's error bits.
 */
uint32_t oracle_quantize_pack(const uint16_t *W, int64_t N, int64_t K, int64_t G,
                              uint8_t *codes, uint16_t *scales)
{
    uint32_t err = 0;
    int64_t ng = K / G, B = oracle_bytes_per_group(G);
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < ng; g++) {
            const uint16_t *w = W + n * K + g * G;
            uint16_t s;
            uint32_t e = oracle_group_scale(w, G, &s);
            err |= e;
            scales[n * ng + g] = s;
            uint8_t *out = codes + (n * ng + g) * B;
            for (int64_t q = 0; q < B; q++) {
                int byte = 0, p3 = 1;
                for (int i = 0; i < 5; i++) {
                    int64_t j = 5 * q + i;
                    int t = (j < G && e == 0) ? oracle_trit(w[j], s) : 0; /* pad = zero trit */
                    byte += (t + 1) * p3;                                  /* digit d = t + 1 */
                    p3 *= 3;
                }
                out[q] = (uint8_t)byte;
            }
        }
    }
    return err;
}

/*
 * [codec] decoding: bytes 243..255 are invalid; digits are read least
 * significant first; a group's weights are restored as bf16.
 * W_out: [N x K] bf16.  Returns the OR of every group's error bits.
 */
uint32_t oracle_unpack_bf16(const uint8_t *codes, const uint16_t *scales, int64_t N,
                            int64_t K, int64_t G, uint16_t *W_out)
{
    uint32_t err = 0;
    int64_t ng = K / G, B = oracle_bytes_per_group(G);
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < ng; g++) {
            uint16_t s = scales[n * ng + g];
            const uint8_t *in = codes + (n * ng + g) * B;
            uint16_t *w = W_out + n * K + g * G;
            uint32_t e = 0;
            if ((s & 0x8000) || ((s >> 10) & 0x1F) == 0x1F)
                e |= ERR_SCALE;                     /* negative, NaN or Inf scale */
            for (int64_t q = 0; q < B; q++) {
                int byte = in[q];
                if (byte >= 243) {
                    e |= ERR_BYTE;
                    continue;
                }
                for (int i = 0; i < 5; i++) {
                    int d = byte % 3;
                    byte /= 3;
                    int64_t j = 5 * q + i;
                    if (j >= G) {
                        if (d != 1)
                            e |= ERR_PADDING;
                        continue;
                    }
                    int t = d - 1;
                    if (t == 0 || s == 0)
                        w[j] = 0x0000;
                    else {
                        uint16_t mag = oracle_bf16_round(oracle_fp16_value(s));
                        w[j] = (uint16_t)(mag | (t < 0 ? 0x8000 : 0));
                    }
                }
            }
            if (e) {
                for (int64_t j = 0; j < G; j++)
                    w[j] = 0x7FC0;                  /* rejected group: NaN */
            }
            err |= e;
        }
    }
    return err;
}

/* Value of every bf16 bit pattern, filled once from oracle_bf16_value. */
static double bf16_table[65536];
static int bf16_table_ready = 0;

static const double *bf16_values(void)
{
    if (!bf16_table_ready) {
        for (uint32_t h = 0; h < 65536; h++)
            bf16_table[h] = oracle_bf16_value((uint16_t)h);
        bf16_table_ready = 1;
    }
    return bf16_table;
}

/*
 * [mm] Y[m][n] = sum_k X[m][k] * What[n][k] for the requested rows m in
 * rows[0..nrows) (all rows if rows == NULL), accumulated in binary64 in
 * increasing k.  Each product of two bf16 values is exact in binary64.
 * Y: [nrows x N] binary64.
 */
void oracle_matmul(const uint16_t *X, int64_t M, const int64_t *rows, int64_t nrows,
                   const uint16_t *What, int64_t N, int64_t K, double *Y)
{
    (void)M;
    const double *v = bf16_values();
    for (int64_t ri = 0; ri < nrows; ri++) {
        int64_t m = rows ? rows[ri] : ri;
        const uint16_t *x = X + m * K;
        for (int64_t n = 0; n < N; n++) {
            const uint16_t *w = What + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += v[x[k]] * v[w[k]];
            Y[ri * N + n] = acc;
        }
    }
}

/* Same, for a list of (m, n) output coordinates: Y[i] = row m_i . column n_i */
void oracle_matmul_points(const uint16_t *X, const uint16_t *What, int64_t K,
                          const int64_t *m_idx, const int64_t *n_idx, int64_t npts,
                          double *Y)
{
    const double *v = bf16_values();
    for (int64_t i = 0; i < npts; i++) {
        const uint16_t *x = X + m_idx[i] * K;
        const uint16_t *w = What + n_idx[i] * K;
        double acc = 0.0;
        for (int64_t k = 0; k < K; k++)
            acc += v[x[k]] * v[w[k]];
        Y[i] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* [two] The 2-bit ternary format: four codes per byte.                */
/* ------------------------------------------------------------------ */

/* [two] bytes per group: ceil(G/4) */
int64_t oracle_bytes_per_group2(int64_t G)
{
    return (G + 3) / 4;
}

/*
 * Quantize and pack into the 2-bit format.  Scale and trits are those of
 * oracle_group_scale and oracle_trit ([codec], [rules]); weight j of a
 * group is code (t + 1) at bits 2 (j % 4) of byte j / 4 ([two]).
 * codes: [N][K/G][ceil(G/4)] bytes, scales: [N][K/G] binary16.
 */
uint32_t oracle_quantize_pack2(const uint16_t *W, int64_t N, int64_t K, int64_t G,
                               uint8_t *codes, uint16_t *scales)
{
    uint32_t err = 0;
    int64_t ng = K / G, B = oracle_bytes_per_group2(G);
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < ng; g++) {
            const uint16_t *w = W + n * K + g * G;
            uint16_t s;
            uint32_t e = oracle_group_scale(w, G, &s);
            err |= e;
            scales[n * ng + g] = s;
            uint8_t *out = codes + (n * ng + g) * B;
            for (int64_t q = 0; q < B; q++) {
                int byte = 0;
                for (int i = 0; i < 4; i++) {
                    int64_t j = 4 * q + i;
                    int t = (j < G && e == 0) ? oracle_trit(w[j], s) : 0; /* pad = zero trit */
                    byte |= (t + 1) << (2 * i);                            /* code c = t + 1 */
                }
                out[q] = (uint8_t)byte;
            }
        }
    }
    return err;
}

/*
 * [two] decoding: code 3 is invalid; padding codes must be 1; decoded
 * weights as for the base-3 codec (+0 for a zero trit or zero scale, else
 * sign(t) * RNE_bf16(scale); a rejected group decodes to NaN).
 */
uint32_t oracle_unpack2_bf16(const uint8_t *codes, const uint16_t *scales, int64_t N,
                             int64_t K, int64_t G, uint16_t *W_out)
{
    uint32_t err = 0;
    int64_t ng = K / G, B = oracle_bytes_per_group2(G);
    for (int64_t n = 0; n < N; n++) {
        for (int64_t g = 0; g < ng; g++) {
            uint16_t s = scales[n * ng + g];
            const uint8_t *in = codes + (n * ng + g) * B;
            uint16_t *w = W_out + n * K + g * G;
            uint32_t e = 0;
            if ((s & 0x8000) || ((s >> 10) & 0x1F) == 0x1F)
                e |= ERR_SCALE;                     /* negative, NaN or Inf scale */
            for (int64_t q = 0; q < B; q++) {
                for (int i = 0; i < 4; i++) {
                    int c = (in[q] >> (2 * i)) & 3;
                    int64_t j = 4 * q + i;
                    if (c == 3) {
                        e |= ERR_BYTE;
                        continue;
                    }
                    if (j >= G) {
                        if (c != 1)
                            e |= ERR_PADDING;
                        continue;
                    }
                    int t = c - 1;
                    if (t == 0 || s == 0)
                        w[j] = 0x0000;
                    else {
                        uint16_t mag = oracle_bf16_round(oracle_fp16_value(s));
                        w[j] = (uint16_t)(mag | (t < 0 ? 0x8000 : 0));
                    }
                }
            }
            if (e) {
                for (int64_t j = 0; j < G; j++)
                    w[j] = 0x7FC0;                  /* rejected group: NaN */
            }
            err |= e;
        }
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* [w4] The W4A16 affine format: decoding only (the page's checkpoint   */
/* supplies codes, scales and biases; it gives no quantizer).           */
/* ------------------------------------------------------------------ */

/*
 * Reconstruct every weight of a row-major [N x K] W4 matrix in binary64:
 * code q of column k is nibble k % 8 (bits 4 (k % 8) .. 4 (k % 8) + 3) of
 * word k / 8 of its row; w = q * s + b with the group's bf16 scale s and bias
 * b (group k / G).  q * s is exact (a 4-bit integer times an 8-bit
 * significand); the sum with b is exact unless the two differ by more than
 * about 40 binades.  codes: [N][K/8] uint32; scales, biases: [N][K/G] bf16.
 */
void oracle_w4_dequant(const uint32_t *codes, const uint16_t *scales, const uint16_t *biases,
                       int64_t N, int64_t K, int64_t G, double *W_out)
{
    int64_t ng = K / G, words = K / 8;
    for (int64_t n = 0; n < N; n++) {
        for (int64_t k = 0; k < K; k++) {
            uint32_t word = codes[n * words + k / 8];
            int q = (int)((word >> (4 * (k % 8))) & 0xFu);
            double sc = oracle_bf16_value(scales[n * ng + k / G]);
            double bi = oracle_bf16_value(biases[n * ng + k / G]);
            W_out[n * K + k] = (double)q * sc + bi;
        }
    }
}
