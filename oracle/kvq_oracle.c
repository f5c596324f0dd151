/*
 * kvq_oracle.c -- plain, slow CPU oracle for norm-separated, per-channel
 * low-bit KV-cache quantization and softmax decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this code.  It shares nothing
 * with the CUDA library: no headers, helpers, tables or constants.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (see oracle/build.py).  -ffp-contract=off matters: every multiply and add
 * below is a separately rounded IEEE-754 binary32 operation.
 *
 * Sources (page title, section):
 *  [P1] "KV cache INT4 quantization ... nsep+pchan" post, section "Fix
 *       (nsep+pchan)": split every K/V vector into an FP16 norm and a unit
 *       direction, then quantize the direction with per-channel scales;
 *       symmetric codes clamped to +-7 with round-to-nearest.
 *  [P2] "Rotated Runtime Smooth" analysis, master equation and symbol list:
 *       R = (1/sqrt(K)) [s_ij], s_ij in {-1,+1}, R R^T = I; the runtime
 *       smoothing scale s_j is the max |.| of channel j over the tokens;
 *       alpha = max|X| / (2^(N-1) - 1) for symmetric N-bit quantization;
 *       section "Experiments": KV cache with group size 128 and RTN.
 *  [P3] "NSNQuant" explainer, section "Method: 1. Normalize-Shift-Normalize":
 *       normalize every token to norm sqrt(d), subtract the per-channel mean,
 *       renormalize to sqrt(d), keeping s1, o, s2 to rebuild the tensor;
 *       section "2. Hadamard Transform"; section "4. Implementation details":
 *       residual tokens are kept in full precision until a block is full.
 *  [P4] "Activation-guided compensation and orthogonal residuals" abstract:
 *       randomized Hadamard rotation with random sign patterns.
 *
 * Readings taken where the pages are silent:
 *  - block = 128 tokens; pchan scale = max over the block's tokens, per channel;
 *  - sums (norms, NSN means) are fp32 pairwise (recursive halving) sums;
 *  - codes = round-half-even of the exact product u * (1/sigma16), clamped;
 *  - the rotation's 1/sqrt(d) is folded into the per-token normalization;
 *  - NSN subtracts the stored fp16 mean so that encoder and decoder agree;
 *  - packed layouts: offset-binary codes (code 0 never stored); INT4 two per
 *    byte low nibble first; INT2 four per byte; INT3 as a 2-bit plane
 *    followed by a 1-bit plane; bits 5..8 (oracle only) one code per byte;
 *  - random signs: SplitMix64 (Steele, Lea, Flood 2014) seeded with `seed`,
 *    sign_c = -1 when bit 63 of the c-th output is set.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KO_T 128 /* tokens per scale block */

enum { KO_NORM_SEP = 1, KO_PER_CHANNEL = 2, KO_NSN = 4, KO_HADAMARD = 8, KO_DQ = 16 };

typedef struct {
    int d;               /* head dim: power of two, 2..1024 */
    int bits;            /* 2..8 */
    unsigned flags;      /* KO_* */
    const int8_t* signs; /* [d] of +-1, or NULL = all +1 (plain Hadamard) */
} ko_cfg;

/* ------------------------------------------------------------------ */
/* IEEE 754 binary16 conversions, written from the format definition. */
/* ------------------------------------------------------------------ */

/* binary32 -> binary16, round to nearest, ties to even. */
uint16_t ko_f32_to_f16(float f)
{
    uint32_t bits;
    memcpy(&bits, &f, 4);
    uint16_t sign = (uint16_t)((bits >> 16) & 0x8000u);
    if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
    double a = fabs((double)f);
    if (isinf(f)) return (uint16_t)(sign | 0x7C00u);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; a rounded value of 1024 quanta is
           the smallest normal number and has the matching encoding. */
        double q = nearbyint(a / ldexp(1.0, -24));
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e;
    frexp(a, &e);       /* a = m * 2^e with m in [0.5, 1) */
    int E = e - 1;      /* a in [2^E, 2^(E+1)) */
    double q = nearbyint(a / ldexp(1.0, E - 10)); /* in [1024, 2048] */
    if (q == 2048.0) { q = 1024.0; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(q - 1024.0));
}

float ko_f16_to_f32(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return (float)(s ? -v : v);
}

/* ------------------------------------------------------------------ */
/* Random signs for the randomized Hadamard transform [P4], [P2].      */
/* ------------------------------------------------------------------ */

uint64_t ko_splitmix64_next(uint64_t* state)
{
    uint64_t z = (*state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

void ko_make_signs(uint64_t seed, int d, int8_t* out)
{
    uint64_t st = seed;
    for (int c = 0; c < d; c++)
        out[c] = (ko_splitmix64_next(&st) >> 63) ? (int8_t)-1 : (int8_t)1;
}

/* ------------------------------------------------------------------ */
/* Building blocks                                                     */
/* ------------------------------------------------------------------ */

/* Unnormalized Walsh-Hadamard butterflies in Sylvester order: for stride
   h = 1, 2, 4, ..., d/2 every pair (i, i+h) with (i & h) == 0 becomes
   (v_i + v_{i+h}, v_i - v_{i+h}).  H_d H_d^T = d I, so R = H_d / sqrt(d)
   is the orthogonal rotation of [P2] with entries +-1/sqrt(d). */
void ko_fwht(float* v, int d)
{
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int j = i; j < i + h; j++) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
}

/* fp32 pairwise sum of n (a power of two) values v[0], v[s], v[2s], ...:
   sum(first half) + sum(second half), recursively. */
float ko_pairwise_sum(const float* v, long n, long s)
{
    if (n == 1) return v[0];
    long h = n / 2;
    return ko_pairwise_sum(v, h, s) + ko_pairwise_sum(v + h * s, h, s);
}

/* Euclidean norm: fp32 square of every entry, pairwise fp32 sum, IEEE sqrt. */
static float ko_l2(const float* v, int d)
{
    float sq[1024];
    for (int c = 0; c < d; c++) sq[c] = v[c] * v[c];
    return sqrtf(ko_pairwise_sum(sq, d, 1));
}

int ko_qmax(int bits) { return (1 << (bits - 1)) - 1; } /* [P2]: 2^(N-1)-1 */

int ko_row_bytes(int d, int bits) { return bits <= 4 ? d * bits / 8 : d; }

/* Per-token fp16 parameters stored for a flag set. */
int ko_ntok(unsigned flags)
{
    int n;
    if (flags & KO_NSN) n = (flags & KO_DQ) ? 1 : 2; /* s1, s2 (under DQ s1 is in the block record) */
    else n = (flags & KO_NORM_SEP) ? 1 : 0;         /* norm */
    if (!(flags & KO_PER_CHANNEL)) n += 1;          /* token scale, last */
    return n;
}

void ko_pack_row(const int8_t* q, int d, int bits, uint8_t* out)
{
    int off = 1 << (bits - 1);
    int rb = ko_row_bytes(d, bits);
    memset(out, 0, (size_t)rb);
    for (int c = 0; c < d; c++) {
        unsigned e = (unsigned)(q[c] + off);
        if (bits == 4) out[c / 2] |= (uint8_t)(e << (4 * (c % 2)));
        else if (bits == 2) out[c / 4] |= (uint8_t)(e << (2 * (c % 4)));
        else if (bits == 3) {
            out[c / 4] |= (uint8_t)((e & 3u) << (2 * (c % 4)));
            out[d / 4 + c / 8] |= (uint8_t)(((e >> 2) & 1u) << (c % 8));
        } else out[c] = (uint8_t)e;
    }
}

/* Returns the number of illegal (zero) offset-binary codes found. */
int ko_unpack_row(const uint8_t* in, int d, int bits, int8_t* q)
{
    int off = 1 << (bits - 1), bad = 0;
    for (int c = 0; c < d; c++) {
        unsigned e;
        if (bits == 4) e = (in[c / 2] >> (4 * (c % 2))) & 15u;
        else if (bits == 2) e = (in[c / 4] >> (2 * (c % 4))) & 3u;
        else if (bits == 3)
            e = ((in[c / 4] >> (2 * (c % 4))) & 3u) | (((in[d / 4 + c / 8] >> (c % 8)) & 1u) << 2);
        else e = in[c];
        if (e == 0) bad++;
        q[c] = (int8_t)((int)e - off);
    }
    return bad;
}

/* ------------------------------------------------------------------ */
/* Double quantization of the NSN side parameters [P3 "Double          */
/* Quantization (DQ)": the mean o and the scale s1 are themselves      */
/* quantized to 4 bits].  Per block of T tokens, one byte record:      */
/*   [0, d/2)            o codes: e = q + 8, channel 2j in the low      */
/*                       nibble of byte j (the INT4 layout)             */
/*   [d/2, d/2 + T/2)    s1 codes: q in 0..15, token 2j in the low      */
/*                       nibble of byte j                               */
/*   then fp16 sigma_o, lo, step; zero padding to a multiple of 16.     */
/* o: symmetric, sigma_o = fp16(max|o| / 7), q = clamp(rne(o / sigma_o),*/
/*    -7, 7), o_hat = q * sigma_o.                                      */
/* s1 (positive): over [lo, lo + 15 step] with lo = fp16(min s1),       */
/*    step = fp16(max(max s1 - lo, 0) / 15), q = clamp(rne((s1 - lo) /  */
/*    step), 0, 15), s1_hat = lo + q * step.                            */
/* ------------------------------------------------------------------ */
int ko_dq_record_bytes(int d) { return (d / 2 + KO_T / 2 + 6 + 15) / 16 * 16; }

/* fp16 words per block of the NSN offsets array: d means, or the record. */
int ko_off_words(unsigned flags, int d) { return (flags & KO_DQ) ? ko_dq_record_bytes(d) / 2 : d; }

static int ko_code_range(double y, int lo, int hi)
{
    double r = nearbyint(y);
    if (r > hi) r = hi;
    if (r < lo) r = lo;
    return (int)r;
}

static void ko_dq_encode(const float* o, const float* s1, int d, uint8_t* rec, float* ohat)
{
    const int T = KO_T, rb = ko_dq_record_bytes(d);
    memset(rec, 0, (size_t)rb);
    float m = 0.0f;
    for (int c = 0; c < d; c++) if (fabsf(o[c]) > m) m = fabsf(o[c]);
    uint16_t so = ko_f32_to_f16(m / 7.0f);
    float sof = ko_f16_to_f32(so);
    float invo = sof > 0.0f ? 1.0f / sof : 0.0f;
    for (int c = 0; c < d; c++) {
        int q = ko_code_range((double)o[c] * (double)invo, -7, 7);
        rec[c / 2] |= (uint8_t)((unsigned)(q + 8) << (4 * (c % 2)));
        ohat[c] = (float)q * sof;
    }
    float mn = s1[0], mx = s1[0];
    for (int t = 1; t < T; t++) { if (s1[t] < mn) mn = s1[t]; if (s1[t] > mx) mx = s1[t]; }
    uint16_t lo16 = ko_f32_to_f16(mn);
    float lo = ko_f16_to_f32(lo16);
    float span = mx - lo;
    if (span < 0.0f) span = 0.0f;
    uint16_t st16 = ko_f32_to_f16(span / 15.0f);
    float st = ko_f16_to_f32(st16);
    float invs = st > 0.0f ? 1.0f / st : 0.0f;
    for (int t = 0; t < T; t++) {
        int q = ko_code_range((double)(s1[t] - lo) * (double)invs, 0, 15);
        rec[d / 2 + t / 2] |= (uint8_t)((unsigned)q << (4 * (t % 2)));
    }
    memcpy(rec + d / 2 + T / 2, &so, 2);
    memcpy(rec + d / 2 + T / 2 + 2, &lo16, 2);
    memcpy(rec + d / 2 + T / 2 + 4, &st16, 2);
}

/* o_hat [d] and s1_hat [T] from a record. */
void ko_dq_decode(const uint8_t* rec, int d, float* ohat, float* s1hat)
{
    const int T = KO_T;
    uint16_t so, lo16, st16;
    memcpy(&so, rec + d / 2 + T / 2, 2);
    memcpy(&lo16, rec + d / 2 + T / 2 + 2, 2);
    memcpy(&st16, rec + d / 2 + T / 2 + 4, 2);
    float sof = ko_f16_to_f32(so), lo = ko_f16_to_f32(lo16), st = ko_f16_to_f32(st16);
    for (int c = 0; c < d; c++) {
        int q = (int)((rec[c / 2] >> (4 * (c % 2))) & 15u) - 8;
        ohat[c] = (float)q * sof;
    }
    for (int t = 0; t < T; t++) {
        int q = (int)((rec[d / 2 + t / 2] >> (4 * (t % 2))) & 15u);
        s1hat[t] = lo + (float)q * st;
    }
}

/* nearest integer to the exact product u * inv (both fp32, so the product is
   exact in binary64), ties to even, clamped to [-qmax, qmax]. */
static int ko_code(float u, float inv, int qmax)
{
    double r = nearbyint((double)u * (double)inv);
    if (r > qmax) r = qmax;
    if (r < -qmax) r = -qmax;
    return (int)r;
}

/* ------------------------------------------------------------------ */
/* Quantize one block of KO_T tokens of one (batch, head).             */
/*   x     [T][d]  fp16 bits                                           */
/*   codes [T][row_bytes]                                              */
/*   tok   [T][ntok] fp16 bits: NSN (s1, s2); nsep (norm); naive       */
/*         (token scale); nsep without pchan (norm, token scale)       */
/*   chan  [d] fp16 bits per-channel scale (PER_CHANNEL)               */
/*   off   [d] fp16 bits per-channel mean (NSN)                        */
/* ------------------------------------------------------------------ */
/* y (optional, [T][d] doubles): the exact product u * inv that each code
   rounds; it exposes the value the codes are taken from and changes nothing
   else. */
static void ko_quantize_block_impl(const ko_cfg* cfg, const uint16_t* x, uint8_t* codes,
                                   uint16_t* tok, uint16_t* chan, uint16_t* off, double* y)
{
    const int d = cfg->d, T = KO_T, qmax = ko_qmax(cfg->bits);
    const unsigned fl = cfg->flags;
    const int ntok = ko_ntok(fl);
    const float RSQD = (float)(1.0 / sqrt((double)d));
    const float SQD = (float)sqrt((double)d);
    const float c0 = (fl & KO_HADAMARD) ? RSQD : 1.0f;

    float* w = (float*)malloc(sizeof(float) * (size_t)T * d); /* working rows */
    float* ks = (float*)malloc(sizeof(float) * T);            /* per-token factor */
    int8_t* q = (int8_t*)malloc((size_t)T * d);

    for (int t = 0; t < T; t++)
        for (int c = 0; c < d; c++) w[t * d + c] = ko_f16_to_f32(x[t * d + c]);

    if (fl & KO_NSN) {
        const int dq = (fl & KO_DQ) != 0;
        float s1v[KO_T], of[1024], oh[1024];
        /* [P3] Normalize: token norm -> sqrt(d); s1 = ||x|| / sqrt(d). */
        for (int t = 0; t < T; t++) {
            float* r = w + t * d;
            float n1 = ko_l2(r, d);
            s1v[t] = n1 * RSQD;
            if (!dq) tok[t * ntok + 0] = ko_f32_to_f16(s1v[t]);
            float r1 = n1 > 0.0f ? SQD / n1 : 0.0f;
            for (int c = 0; c < d; c++) r[c] = r[c] * r1;
        }
        /* [P3] Shift: subtract the per-channel mean over the block.  The
           encoder subtracts the mean the decoder will add back: the stored
           fp16 one, or under DQ its 4-bit reconstruction. */
        for (int c = 0; c < d; c++) of[c] = ko_pairwise_sum(w + c, T, d) * (1.0f / (float)T);
        if (dq) {
            ko_dq_encode(of, s1v, d, (uint8_t*)off, oh);
        } else {
            for (int c = 0; c < d; c++) {
                off[c] = ko_f32_to_f16(of[c]);
                oh[c] = ko_f16_to_f32(off[c]);
            }
        }
        /* [P3] Normalize again: s2 = ||b|| / sqrt(d). */
        for (int t = 0; t < T; t++) {
            float* r = w + t * d;
            for (int c = 0; c < d; c++) r[c] = r[c] - oh[c];
            float n2 = ko_l2(r, d);
            tok[t * ntok + (dq ? 0 : 1)] = ko_f32_to_f16(n2 * RSQD);
            ks[t] = n2 > 0.0f ? c0 / n2 : 0.0f;
        }
    } else if (fl & KO_NORM_SEP) {
        /* [P1] norm separation: FP16 norm + unit direction. */
        for (int t = 0; t < T; t++) {
            float n = ko_l2(w + t * d, d);
            tok[t * ntok + 0] = ko_f32_to_f16(n);
            ks[t] = n > 0.0f ? c0 / n : 0.0f;
        }
    } else {
        for (int t = 0; t < T; t++) ks[t] = c0;
    }

    /* Rotation [P2]/[P4]: direction = H (s (.) w) * (1/sqrt(d)) * (1/norm). */
    for (int t = 0; t < T; t++) {
        float* r = w + t * d;
        if (fl & KO_HADAMARD) {
            if (cfg->signs)
                for (int c = 0; c < d; c++) if (cfg->signs[c] < 0) r[c] = -r[c];
            ko_fwht(r, d);
        }
        for (int c = 0; c < d; c++) r[c] = r[c] * ks[t];
    }

    /* Scales [P2]: alpha = max|.| / qmax, per channel over the block's tokens
       (pchan) or per token over the channels. */
    if (fl & KO_PER_CHANNEL) {
        for (int c = 0; c < d; c++) {
            float m = 0.0f;
            for (int t = 0; t < T; t++) { float a = fabsf(w[t * d + c]); if (a > m) m = a; }
            chan[c] = ko_f32_to_f16(m / (float)qmax);
            float sf = ko_f16_to_f32(chan[c]);
            float inv = sf > 0.0f ? 1.0f / sf : 0.0f;
            for (int t = 0; t < T; t++) {
                q[t * d + c] = (int8_t)ko_code(w[t * d + c], inv, qmax);
                if (y) y[t * d + c] = (double)w[t * d + c] * (double)inv;
            }
        }
    } else {
        for (int t = 0; t < T; t++) {
            float m = 0.0f;
            for (int c = 0; c < d; c++) { float a = fabsf(w[t * d + c]); if (a > m) m = a; }
            uint16_t s16 = ko_f32_to_f16(m / (float)qmax);
            tok[t * ntok + ntok - 1] = s16;
            float sf = ko_f16_to_f32(s16);
            float inv = sf > 0.0f ? 1.0f / sf : 0.0f;
            for (int c = 0; c < d; c++) {
                q[t * d + c] = (int8_t)ko_code(w[t * d + c], inv, qmax);
                if (y) y[t * d + c] = (double)w[t * d + c] * (double)inv;
            }
        }
    }

    const int rb = ko_row_bytes(d, cfg->bits);
    for (int t = 0; t < T; t++) ko_pack_row(q + t * d, d, cfg->bits, codes + (size_t)t * rb);
    free(w); free(ks); free(q);
}

void ko_quantize_block(const ko_cfg* cfg, const uint16_t* x, uint8_t* codes,
                       uint16_t* tok, uint16_t* chan, uint16_t* off)
{
    ko_quantize_block_impl(cfg, x, codes, tok, chan, off, NULL);
}

/* ------------------------------------------------------------------ */
/* Dequantize one block back to fp32 (the inverse of the steps above). */
/* Returns the number of illegal zero codes met.                       */
/* ------------------------------------------------------------------ */
int ko_dequantize_block(const ko_cfg* cfg, const uint8_t* codes, const uint16_t* tok,
                        const uint16_t* chan, const uint16_t* off, float* out)
{
    const int d = cfg->d, T = KO_T;
    const unsigned fl = cfg->flags;
    const int ntok = ko_ntok(fl), rb = ko_row_bytes(d, cfg->bits);
    const float RSQD = (float)(1.0 / sqrt((double)d));
    const float SQD = (float)sqrt((double)d);
    int8_t q[1024];
    float w[1024], ohat[1024], s1hat[KO_T];
    int bad = 0;
    const int dq = (fl & KO_NSN) && (fl & KO_DQ);
    if (dq) ko_dq_decode((const uint8_t*)off, d, ohat, s1hat);
    else if (fl & KO_NSN)
        for (int c = 0; c < d; c++) ohat[c] = ko_f16_to_f32(off[c]);
    for (int t = 0; t < T; t++) {
        bad += ko_unpack_row(codes + (size_t)t * rb, d, cfg->bits, q);
        for (int c = 0; c < d; c++) {
            float sf = (fl & KO_PER_CHANNEL) ? ko_f16_to_f32(chan[c])
                                             : ko_f16_to_f32(tok[t * ntok + ntok - 1]);
            w[c] = (float)q[c] * sf;
        }
        float* o = out + (size_t)t * d;
        int had = (fl & KO_HADAMARD) != 0;
        if (had) ko_fwht(w, d);
        if (fl & KO_NSN) {
            float s1 = dq ? s1hat[t] : ko_f16_to_f32(tok[t * ntok + 0]);
            float s2 = ko_f16_to_f32(tok[t * ntok + (dq ? 0 : 1)]);
            float kb = had ? s2 : s2 * SQD;
            for (int c = 0; c < d; c++) {
                float b = w[c] * kb;
                if (had && cfg->signs && cfg->signs[c] < 0) b = -b;
                o[c] = s1 * (b + ohat[c]);
            }
        } else if (fl & KO_NORM_SEP) {
            float n = ko_f16_to_f32(tok[t * ntok + 0]);
            if (had) {
                float kd = n * RSQD;
                for (int c = 0; c < d; c++) {
                    float v = w[c] * kd;
                    o[c] = (cfg->signs && cfg->signs[c] < 0) ? -v : v;
                }
            } else {
                for (int c = 0; c < d; c++) o[c] = n * w[c];
            }
        } else {
            for (int c = 0; c < d; c++) {
                float v = had ? w[c] * RSQD : w[c];
                o[c] = (had && cfg->signs && cfg->signs[c] < 0) ? -v : v;
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------ */
/* Cache-level loops for one (batch, kv-head) slice.                   */
/* Layouts per slice: x [ntok][d]; codes [S_max][row_bytes];           */
/* tok [S_max][ntok]; chan, off [S_max/T][d].                          */
/* ------------------------------------------------------------------ */
/* y: NULL, or [ntok][d] doubles that receive the exact pre-rounding
   product of every code (see ko_quantize_block_impl). */
void ko_quantize_slice_y(const ko_cfg* cfg, const uint16_t* x, long t0, long ntok,
                         uint8_t* codes, uint16_t* tok, uint16_t* chan, uint16_t* off, double* y)
{
    const int d = cfg->d, rb = ko_row_bytes(d, cfg->bits), nt = ko_ntok(cfg->flags);
    for (long t = 0; t < ntok; t += KO_T) {
        long tb = t0 + t, blk = tb / KO_T;
        ko_quantize_block_impl(cfg, x + (size_t)t * d, codes + (size_t)tb * rb,
                               tok ? tok + (size_t)tb * nt : NULL,
                               chan ? chan + (size_t)blk * d : NULL,
                               off ? off + (size_t)blk * ko_off_words(cfg->flags, d) : NULL,
                               y ? y + (size_t)t * d : NULL);
    }
}

void ko_quantize_slice(const ko_cfg* cfg, const uint16_t* x, long t0, long ntok,
                       uint8_t* codes, uint16_t* tok, uint16_t* chan, uint16_t* off)
{
    ko_quantize_slice_y(cfg, x, t0, ntok, codes, tok, chan, off, NULL);
}

int ko_dequantize_slice(const ko_cfg* cfg, const uint8_t* codes, const uint16_t* tok,
                        const uint16_t* chan, const uint16_t* off, long t0, long ntok, float* out)
{
    const int d = cfg->d, rb = ko_row_bytes(d, cfg->bits), nt = ko_ntok(cfg->flags);
    int bad = 0;
    for (long t = 0; t < ntok; t += KO_T) {
        long tb = t0 + t, blk = tb / KO_T;
        bad += ko_dequantize_block(cfg, codes + (size_t)tb * rb,
                                   tok ? tok + (size_t)tb * nt : NULL,
                                   chan ? chan + (size_t)blk * d : NULL,
                                   off ? off + (size_t)blk * ko_off_words(cfg->flags, d) : NULL, out + (size_t)t * d);
    }
    return bad;
}

/* ------------------------------------------------------------------ */
/* Sign-pattern selection for the randomized Hadamard rotation [P4]:   */
/* quantize a sample with each candidate sign vector and keep the one  */
/* whose reconstruction error is smallest.                             */
/*   x      [n_blocks][T][d] fp16 bits: the sample, whole blocks       */
/*   signs  [n_cand][d] of +-1: the candidate sign vectors             */
/*   err    [n_cand] out: sum over the sample of (x_hat - x)^2 in fp64  */
/* The error of a block is the pairwise (recursive halving) sum over   */
/* its tokens of the pairwise sum over channels of the squared         */
/* differences; the blocks are added in order.  Returns the index of   */
/* the smallest error (the lowest index among equal ones).             */
/* ------------------------------------------------------------------ */
static double ko_pairwise_sum_f64(const double* v, long n)
{
    if (n == 1) return v[0];
    long h = n / 2;
    return ko_pairwise_sum_f64(v, h) + ko_pairwise_sum_f64(v + h, h);
}

int ko_select_signs(const ko_cfg* cfg, const uint16_t* x, long n_blocks, const int8_t* signs, int n_cand,
                    double* err)
{
    const int d = cfg->d, T = KO_T, rb = ko_row_bytes(d, cfg->bits), nt = ko_ntok(cfg->flags);
    uint8_t* codes = (uint8_t*)malloc((size_t)T * rb);
    uint16_t* tok = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * (nt > 0 ? nt : 1));
    uint16_t chan[1024], off[1024];
    float* xh = (float*)malloc(sizeof(float) * (size_t)T * d);
    double sq[1024], rowe[KO_T];
    int best = 0;
    for (int k = 0; k < n_cand; k++) {
        ko_cfg c = *cfg;
        c.signs = signs + (size_t)k * d;
        double e = 0.0;
        for (long b = 0; b < n_blocks; b++) {
            const uint16_t* xb = x + (size_t)b * T * d;
            ko_quantize_block(&c, xb, codes, tok, chan, off);
            ko_dequantize_block(&c, codes, tok, chan, off, xh);
            for (int t = 0; t < T; t++) {
                for (int ch = 0; ch < d; ch++) {
                    double df = (double)xh[t * d + ch] - (double)ko_f16_to_f32(xb[t * d + ch]);
                    sq[ch] = df * df;
                }
                rowe[t] = ko_pairwise_sum_f64(sq, d);
            }
            e = e + ko_pairwise_sum_f64(rowe, T);
        }
        err[k] = e;
        if (e < err[best]) best = k;
    }
    free(codes); free(tok); free(xh);
    return best;
}

/* ------------------------------------------------------------------ */
/* Softmax attention of g query heads over L cached tokens, in fp64,   */
/* brute force: out_j = sum_t softmax_t(scale * q_j . k_t) v_t.        */
/*   q [g][d] fp16 bits; k, v [L][d] fp32; out [g][d] fp64.            */
/* L == 0 gives a zero output.                                          */
/* ------------------------------------------------------------------ */
void ko_attention_f64(int g, int d, long L, const uint16_t* q, const float* k,
                      const float* v, double scale, double* out)
{
    double* lg = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int j = 0; j < g; j++) {
        double* o = out + (size_t)j * d;
        for (int c = 0; c < d; c++) o[c] = 0.0;
        if (L == 0) continue;
        double m = -INFINITY;
        for (long t = 0; t < L; t++) {
            double s = 0.0;
            for (int c = 0; c < d; c++)
                s += (double)ko_f16_to_f32(q[j * d + c]) * (double)k[(size_t)t * d + c];
            lg[t] = scale * s;
            if (lg[t] > m) m = lg[t];
        }
        double z = 0.0;
        for (long t = 0; t < L; t++) { lg[t] = exp(lg[t] - m); z += lg[t]; }
        for (long t = 0; t < L; t++) {
            double p = lg[t] / z;
            for (int c = 0; c < d; c++) o[c] += p * (double)v[(size_t)t * d + c];
        }
    }
    free(lg);
}

/* Array helpers for the test harness (elementwise, no arithmetic of their own). */
void ko_f32_to_f16_array(const float* in, long n, uint16_t* out)
{
    for (long i = 0; i < n; i++) out[i] = ko_f32_to_f16(in[i]);
}

void ko_f16_to_f32_array(const uint16_t* in, long n, float* out)
{
    for (long i = 0; i < n; i++) out[i] = ko_f16_to_f32(in[i]);
}
