/*
 * fp8_oracle.c -- plain CPU oracle for the FP8 W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library.  The GPU library
 * never links, includes or calls it, and it shares no code with the GPU
 * path (no common headers, tables or helpers).
 *
 * What it computes, and where the pages say so:
 *
 *   [P1] "Llama 3 精读实录：FP8 量化与长上下文实测的完整记录", section 2.1
 *        (两种 FP8 格式的本质区别): E4M3 = 4 exponent bits and 3 mantissa
 *        bits, largest value 448; E5M2 = 5 and 2, largest 57344; inference
 *        uses E4M3 for weights and activations.
 *   [P2] "Llama-3.1-8B-Instruct-FP8-Dynamic" explainer, section "FP8 动态量化"
 *        table: weights 8-bit float, one scale per output channel from a
 *        minmax observer; input activations 8-bit float, dynamic, one scale
 *        per token; lm_head not quantized.
 *   [P4] "Llama-3.1-70B-FP8-Dynamic" explainer, section 1.2 (名字里的
 *        "Dynamic"): the same scheme; FAQ Q2: activations quantized per token
 *        at inference time.
 *   [P5] "Llama-3.2-3B-Instruct-FP8-Block" explainer, quantization_config
 *        table: weight block_structure [128, 128]; input activations in
 *        dynamic groups of 128; lm_head ignored.
 *
 * Readings taken where the pages leave a step open (each listed in the
 * design notes):
 *   - E4M3 is the "FN" variant: no infinities, codes 0x7F/0xFF are NaN.  It is
 *     the variant whose largest finite value is the 448 that [P1] prints.
 *   - A symmetric minmax observer gives amax = max|x| over the unit and
 *     scale s = amax / 448, one IEEE fp32 division.  amax == 0 gives s = 1.
 *   - The code of x is E4M3(fl32(x / s)): an IEEE fp32 quotient, then the
 *     nearest E4M3 value, ties to the even mantissa, saturating at +-448,
 *     sign kept (a negative value that rounds to zero is -0, code 0x80).
 *   - The layer output is y[m,n] = sum_k deq(xq[m,k]) * deq(wq[n,k]) with
 *     deq(q) = E4M3value(q) * scale; block mode sums per 128-wide K slice
 *     with that slice's two scales.  It is computed here EXACTLY: every finite
 *     E4M3 value is an integer multiple of 2^-9, so the dot product of codes is
 *     an exact int64 sum, scaled once in double and rounded to fp32.
 *
 * The E4M3 encoder is a nearest-value search over the table of the 127
 * non-negative finite E4M3 values (built from the decoder), not bit
 * manipulation: it is written to be independent of how a GPU converts.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

/* ---------------------------------------------------------------- formats */

/* E4M3FN decode from the bit fields: s.eeee.mmm, exponent bias 7. */
ORC_EXPORT double orc_e4m3_decode(uint8_t code) {
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 15 && m == 7) return NAN;                 /* the only NaN pattern   */
    if (e == 0) mag = ldexp((double)m, -9);            /* subnormal: m * 2^-9    */
    else mag = ldexp(1.0 + m / 8.0, e - 7);            /* (1 + m/8) * 2^(e-7)    */
    return s ? -mag : mag;
}

/* E5M2 decode (IEEE-like: exponent bias 15, inf and NaN at exponent 31).
 * Used only to check the format facts [P1] prints. */
ORC_EXPORT double orc_e5m2_decode(uint8_t code) {
    int s = (code >> 7) & 1;
    int e = (code >> 2) & 0x1F;
    int m = code & 0x3;
    double mag;
    if (e == 31) mag = (m == 0) ? INFINITY : NAN;
    else if (e == 0) mag = ldexp((double)m, -16);
    else mag = ldexp(1.0 + m / 4.0, e - 15);
    return s ? -mag : mag;
}

static double g_mag[127];     /* value of code c, c = 0x00 .. 0x7E, ascending */
static int g_mag_ready = 0;

static void build_mag_table(void) {
    if (g_mag_ready) return;
    for (int c = 0; c < 127; ++c) g_mag[c] = orc_e4m3_decode((uint8_t)c);
    g_mag_ready = 1;
}

/* Nearest E4M3 code to a finite float: bisection for the two neighbouring
 * table values, then the closer one; an exact tie goes to the code whose
 * mantissa LSB (= code LSB) is 0.  Values beyond 448 have only one neighbour
 * (448), which is saturation.  The sign bit is copied from v. */
ORC_EXPORT uint8_t orc_e4m3_encode(float v) {
    build_mag_table();
    double a = fabs((double)v);
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    uint8_t c;
    if (a >= g_mag[126]) {
        c = 126;
    } else {
        int lo = 0, hi = 126;                 /* g_mag[lo] <= a < g_mag[hi] */
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (g_mag[mid] <= a) lo = mid; else hi = mid;
        }
        double dl = a - g_mag[lo], dh = g_mag[hi] - a;
        if (dl < dh) c = (uint8_t)lo;
        else if (dh < dl) c = (uint8_t)hi;
        else c = (uint8_t)((lo & 1) ? hi : lo);
    }
    return (uint8_t)(c | sign);
}

/* Encode n floats (scale 1), for sweeps over many values. */
ORC_EXPORT void orc_e4m3_encode_n(const float* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

static inline float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ----------------------------------------------------------- quantization */

/* Scale of one unit from its amax: s = fl32(amax / 448), or 1 when amax = 0. */
static float scale_from_amax(float amax) {
    volatile float num = amax;            /* keep it an IEEE single division */
    if (amax == 0.0f) return 1.0f;
    return num / 448.0f;
}

/* Round to the nearest bf16, ties to even (finite inputs). */
static uint16_t float_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t upper = u >> 16, lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* The scale rounded to bf16, the dtype the FP8 checkpoints store scales in
 * (reading: the 72.67 GB of [P4] section 二 matches bf16 scales), before the
 * codes are computed, so that the codes are those a bf16-scale checkpoint
 * holds.  A scale that rounds to zero (amax below 448 * 2^-134) becomes 1,
 * like amax = 0: every code of such a unit is zero either way. */
static float scale_to_bf16(float s) {
    float r = bf16_to_float(float_to_bf16(s));
    return r == 0.0f ? 1.0f : r;
}

static inline uint8_t code_of(float x, float s) {
    volatile float q = x / s;             /* fp32 quotient, RNE */
    return orc_e4m3_encode(q);
}

/* One scale per row: per-token activations [P2, P4] and per-output-channel
 * weights [P2] are the same operation on X[M,K] and on W[N,K].
 * x: bf16 bits [rows, ld], q: [rows, ldq], s: [rows]. */
static void quant_rows_impl(const uint16_t* x, int64_t rows, int64_t K, int64_t ld,
                            uint8_t* q, int64_t ldq, float* s, int scale_bf16) {
    build_mag_table();                    /* before the rows run in parallel (they are independent) */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(x[r * ld + k]));
            if (a > amax) amax = a;
        }
        float sr = scale_from_amax(amax);
        if (scale_bf16) sr = scale_to_bf16(sr);
        s[r] = sr;
        for (int64_t k = 0; k < K; ++k) q[r * ldq + k] = code_of(bf16_to_float(x[r * ld + k]), sr);
    }
}

/* One scale per 128 consecutive input features of each token [P5].
 * K must be a multiple of 128.  s: [M, K/128] row-major. */
static void quant_groups128_impl(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                                 uint8_t* q, int64_t ldq, float* s, int scale_bf16) {
    int64_t G = K / 128;
    build_mag_table();
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            float amax = 0.0f;
            for (int64_t k = g * 128; k < g * 128 + 128; ++k) {
                float a = fabsf(bf16_to_float(x[m * ld + k]));
                if (a > amax) amax = a;
            }
            float sg = scale_from_amax(amax);
            if (scale_bf16) sg = scale_to_bf16(sg);
            s[m * G + g] = sg;
            for (int64_t k = g * 128; k < g * 128 + 128; ++k)
                q[m * ldq + k] = code_of(bf16_to_float(x[m * ld + k]), sg);
        }
    }
}

/* One scale per 128 x 128 tile of W[N,K] [P5, block_structure [128, 128]].
 * K must be a multiple of 128; the last row-tile may be shorter than 128
 * (amax over the rows that exist).  s: [ceil(N/128), K/128] row-major. */
static void quant_blocks128_impl(const uint16_t* w, int64_t N, int64_t K, int64_t ld,
                                 uint8_t* q, int64_t ldq, float* s, int scale_bf16) {
    int64_t NB = (N + 127) / 128, KB = K / 128;
    build_mag_table();
#pragma omp parallel for schedule(static)
    for (int64_t nb = 0; nb < NB; ++nb) {
        int64_t n1 = (nb + 1) * 128 < N ? (nb + 1) * 128 : N;
        for (int64_t kb = 0; kb < KB; ++kb) {
            float amax = 0.0f;
            for (int64_t n = nb * 128; n < n1; ++n)
                for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) {
                    float a = fabsf(bf16_to_float(w[n * ld + k]));
                    if (a > amax) amax = a;
                }
            float sb = scale_from_amax(amax);
            if (scale_bf16) sb = scale_to_bf16(sb);
            s[nb * KB + kb] = sb;
            for (int64_t n = nb * 128; n < n1; ++n)
                for (int64_t k = kb * 128; k < kb * 128 + 128; ++k)
                    q[n * ldq + k] = code_of(bf16_to_float(w[n * ld + k]), sb);
        }
    }
}

/* Static scale: [P1] section 2 (FP8 量化实操) calibrates each tensor offline
 * from percentiles of a calibration set (the 99.9% and 0.1% quantiles as its
 * range, not min/max) instead of the runtime amax; at run time every element
 * is coded with that fixed scale, saturating beyond it.  x: bf16 [rows, ld];
 * q: [rows, ldq]. */
ORC_EXPORT void orc_quant_static(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, float s,
                                 uint8_t* q, int64_t ldq) {
    build_mag_table();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) q[r * ldq + k] = code_of(bf16_to_float(x[r * ld + k]), s);
}

/* Exported forms: fp32 scales, and scales rounded to bf16 first ("_s16"). */
ORC_EXPORT void orc_quant_rows(const uint16_t* x, int64_t rows, int64_t K, int64_t ld,
                               uint8_t* q, int64_t ldq, float* s) {
    quant_rows_impl(x, rows, K, ld, q, ldq, s, 0);
}
ORC_EXPORT void orc_quant_groups128(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                                    uint8_t* q, int64_t ldq, float* s) {
    quant_groups128_impl(x, M, K, ld, q, ldq, s, 0);
}
ORC_EXPORT void orc_quant_blocks128(const uint16_t* w, int64_t N, int64_t K, int64_t ld,
                                    uint8_t* q, int64_t ldq, float* s) {
    quant_blocks128_impl(w, N, K, ld, q, ldq, s, 0);
}
ORC_EXPORT void orc_quant_rows_s16(const uint16_t* x, int64_t rows, int64_t K, int64_t ld,
                                   uint8_t* q, int64_t ldq, float* s) {
    quant_rows_impl(x, rows, K, ld, q, ldq, s, 1);
}
ORC_EXPORT void orc_quant_groups128_s16(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                                        uint8_t* q, int64_t ldq, float* s) {
    quant_groups128_impl(x, M, K, ld, q, ldq, s, 1);
}
ORC_EXPORT void orc_quant_blocks128_s16(const uint16_t* w, int64_t N, int64_t K, int64_t ld,
                                        uint8_t* q, int64_t ldq, float* s) {
    quant_blocks128_impl(w, N, K, ld, q, ldq, s, 1);
}

/* ------------------------------------------------- RMSNorm, then per token */
/*
 * [P1] section 1.3 (编码器细节：RMSNorm 与 SwiGLU 的实现差异): Llama 3 normalises
 * with RMSNorm before attention and before the MLP, eps = 1e-5; section 5
 * (the fine-tuning notes) keeps RMSNorm in BF16.  So the input of the q/k/v and
 * gate/up projections is y = RMSNorm(x) in bf16, and its per-token
 * quantization is the activation quantization above applied to y.
 * Readings (the pages print no formula): with x in bf16 and gamma the bf16
 * weight,
 *   ms   = the exact mean over the row of x^2, rounded once to fp32
 *   d    = fl32(ms + eps)
 *   rstd = 1 / sqrt(d), rounded once to fp32
 *   h    = bf16(fl32(x * rstd)),  y = bf16(fl32(gamma * h))
 * (normalise in fp32, return to bf16, then scale by the bf16 weight).
 * Every rounding above is one IEEE round-to-nearest-even of an exact value,
 * so the oracle computes each one from the exact value, in integers where a
 * double would round first.
 */

/* The exact sum of squares of a row.  A bf16 value is an integer multiple of
 * 2^-133 (its subnormal step), so its square is an integer multiple of
 * 2^-266, below 2^256.  The sum is kept as a non-negative integer in units of
 * 2^-266, in little-endian 64-bit limbs: up to 2^31 squares need 553 bits,
 * nine limbs hold 576. */
#define SQ_LIMBS 9

__extension__ typedef unsigned __int128 u128;   /* GCC's 128-bit integer */

static void sq_add(uint64_t* acc, uint16_t b) {
    int e = (b >> 7) & 0xFF;                 /* |x| = m * 2^(p - 133):                   */
    uint64_t m = b & 0x7F;                   /*   subnormal (e == 0): m = mantissa, p = 0 */
    int p = 0;                               /*   normal: m = 128 + mantissa, p = e - 1  */
    if (e != 0) { m += 128; p = e - 1; }
    uint64_t sq = m * m;                     /* x^2 = sq * 2^(2p - 266), sq < 2^16      */
    int bit = 2 * p, li = bit / 64, bo = bit % 64;
    uint64_t lo = sq << bo, hi = bo ? sq >> (64 - bo) : 0;
    uint64_t old = acc[li];
    acc[li] += lo;
    uint64_t carry = (acc[li] < old) ? 1 : 0;
    for (int i = li + 1; i < SQ_LIMBS && (hi || carry); ++i) {
        old = acc[i];
        acc[i] += hi + carry;                /* hi < 2^16: no double wrap */
        carry = (acc[i] < old) ? 1 : 0;
        hi = 0;
    }
}

static int sq_bit(const uint64_t* a, int i) { return (int)((a[i / 64] >> (i % 64)) & 1u); }

/* fl32(S * 2^-266 / K) for the integer S in acc: long division by K, then
 * round to nearest even at 24 significant bits, or at the fixed subnormal
 * step 2^-149 (bit 117 of the quotient), whichever is coarser. */
static float sq_mean_f32(const uint64_t* acc, int64_t K) {
    uint64_t q[SQ_LIMBS];
    u128 rem = 0;
    for (int i = SQ_LIMBS - 1; i >= 0; --i) {
        u128 cur = (rem << 64) | acc[i];
        q[i] = (uint64_t)(cur / (uint64_t)K);
        rem = cur % (uint64_t)K;
    }
    int top = -1;
    for (int i = 64 * SQ_LIMBS - 1; i >= 0; --i)
        if (sq_bit(q, i)) { top = i; break; }
    if (top < 0) return 0.0f;                /* below 2^-266: rounds to zero */
    int lsb = top - 23 > 117 ? top - 23 : 117;   /* no bits kept when top < 117 (below 2^-149) */
    uint32_t mant = 0;
    for (int i = top; i >= lsb; --i) mant = (mant << 1) | (uint32_t)sq_bit(q, i);
    int round = sq_bit(q, lsb - 1);
    int sticky = rem != 0;
    for (int i = lsb - 2; i >= 0 && !sticky; --i) sticky = sq_bit(q, i);
    if (round && (sticky || (mant & 1u))) mant += 1u;
    return ldexpf((float)mant, lsb - 266);
}

/* x = X * 2^ex with X an integer of at most 24 bits, for a positive finite fp32. */
static void f32_int_exp(float x, uint64_t* X, int* ex) {
    int e;
    float fr = frexpf(x, &e);                /* x = fr * 2^e, fr in [0.5, 1) */
    *X = (uint64_t)ldexpf(fr, 24);
    *ex = e - 24;
}

/* Sign of mid^2 * d - 1, exactly, where mid = (a + b) / 2 for positive fp32
 * a < b and positive fp32 d. */
static int mid_sq_d_vs_one(float a, float b, float d) {
    uint64_t A, B, D;
    int ea, eb, ed;
    f32_int_exp(a, &A, &ea);
    f32_int_exp(b, &B, &eb);
    f32_int_exp(d, &D, &ed);
    int e0 = ea < eb ? ea : eb;              /* both on the scale of the smaller exponent */
    A <<= (ea - e0);
    B <<= (eb - e0);
    uint64_t Mid = A + B;                    /* mid = Mid * 2^(e0 - 1), Mid < 2^26 */
    u128 P = (u128)Mid * Mid * D;   /* < 2^76 */
    int E = 2 * (e0 - 1) + ed;               /* mid^2 d = P * 2^E */
    if (E >= 0) return (P == 1 && E == 0) ? 0 : 1;
    if (-E >= 100) return -1;                /* P < 2^76 < 2^-E */
    u128 one = (u128)1 << (-E);
    return P < one ? -1 : (P > one ? 1 : 0);
}

static int f32_odd(float r) {
    uint32_t u;
    memcpy(&u, &r, 4);
    return (int)(u & 1u);
}

/* 1 / sqrt(d) rounded to the nearest fp32 (ties to even), for positive finite
 * d.  A double estimate gives a candidate r; 1/sqrt(d) lies above the
 * midpoint of r and its upper neighbour exactly when that midpoint squared
 * times d is below 1, which is decided in integers; r moves until both
 * midpoints around it bracket 1/sqrt(d). */
static float rsqrt_f32_rn(float d) {
    float r = (float)(1.0 / sqrt((double)d));
    for (;;) {
        float up = nextafterf(r, INFINITY);
        int c = mid_sq_d_vs_one(r, up, d);
        if (c < 0 || (c == 0 && f32_odd(r))) { r = up; continue; }
        float dn = nextafterf(r, 0.0f);
        c = mid_sq_d_vs_one(dn, r, d);
        if (c > 0 || (c == 0 && f32_odd(r))) { r = dn; continue; }
        return r;
    }
}

/* Reciprocal RMS of every row: rstd = RN(1 / sqrt(fl32(ms + eps))) with ms the
 * exact mean of squares rounded once to fp32.  Rows whose mean of squares
 * overflows fp32 are outside the definition (rstd 0 is returned for them). */
ORC_EXPORT void orc_rmsnorm_rstd(const uint16_t* x, int64_t rows, int64_t K, int64_t ld, float eps, float* rstd) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        uint64_t acc[SQ_LIMBS] = {0};
        for (int64_t k = 0; k < K; ++k) sq_add(acc, x[r * ld + k]);
        float ms = sq_mean_f32(acc, K);
        volatile float d = ms + eps;                   /* fp32 addition */
        if (!(d > 0.0f) || isinf(d)) { rstd[r] = d > 0.0f ? 0.0f : INFINITY; continue; }
        rstd[r] = rsqrt_f32_rn(d);
    }
}

/* The fp32 number `ulps` steps away from the positive r (test knob: 0 is r). */
static float step_ulps(float r, int ulps) {
    for (; ulps > 0; --ulps) r = nextafterf(r, INFINITY);
    for (; ulps < 0; ++ulps) r = nextafterf(r, 0.0f);
    return r;
}

/* RMSNorm of each row with the oracle's own rstd (moved by `rstd_ulps` fp32
 * steps: 0 is the definition; the parity tests also take +-1 to accept a
 * kernel whose rstd is one ulp off), then per-token quantization.
 * gamma: bf16 bits [K].  q/s as orc_quant_rows; y (bf16 bits [rows, K])
 * receives the normalised rows and rstd_out [rows] the rstd used. */
ORC_EXPORT void orc_rmsnorm_quant_rows(const uint16_t* x, const uint16_t* gamma, int64_t rows, int64_t K,
                                       int64_t ld, float eps, int rstd_ulps, uint8_t* q, int64_t ldq, float* s,
                                       uint16_t* y, float* rstd_out) {
    orc_rmsnorm_rstd(x, rows, K, ld, eps, rstd_out);
    build_mag_table();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float rs = step_ulps(rstd_out[r], rstd_ulps);
        rstd_out[r] = rs;
        uint16_t* yr = y + r * K;
        for (int64_t k = 0; k < K; ++k) {
            volatile float t = bf16_to_float(x[r * ld + k]) * rs;
            uint16_t h = float_to_bf16(t);
            volatile float g = bf16_to_float(gamma[k]) * bf16_to_float(h);
            yr[k] = float_to_bf16(g);
        }
        orc_quant_rows(yr, 1, K, K, q + r * ldq, ldq, s + r);
    }
}

/* ----------------------------------------------------------------- linear */

/* Integer mantissa of a code: E4M3value(c) = ik(c) * 2^-9 exactly. */
static int32_t g_ik[256];
static int g_ik_ready = 0;

static void build_ik_table(void) {
    if (g_ik_ready) return;
    for (int c = 0; c < 256; ++c) {
        double v = orc_e4m3_decode((uint8_t)c);
        g_ik[c] = isnan(v) ? 0 : (int32_t)ldexp(v, 9);
    }
    g_ik_ready = 1;
}

/* Exact sum over k in [k0, k1) of E4M3value(a[k]) * E4M3value(b[k]), times 2^18. */
static int64_t code_dot(const uint8_t* a, const uint8_t* b, int64_t k0, int64_t k1) {
    int64_t acc = 0;
    for (int64_t k = k0; k < k1; ++k) acc += (int64_t)g_ik[a[k]] * (int64_t)g_ik[b[k]];
    return acc;
}

/* Channel/token mode: y[m,n] = xs[m] * ws[n] * sum_k x(m,k) w(n,k), the
 * x_scale[m] * w_scale[n] product applied to the FP8 dot product [P2, P4]. */
static float linear_channel_one(const uint8_t* xq, const float* xs, const uint8_t* wq,
                                const float* ws, int64_t K, int64_t ldx, int64_t ldw,
                                int64_t m, int64_t n) {
    int64_t S = code_dot(xq + m * ldx, wq + n * ldw, 0, K);
    return (float)((double)xs[m] * (double)ws[n] * ldexp((double)S, -18));
}

/* Block mode: sum over 128-wide K slices of the slice's exact dot product
 * times x_scale[m, kb] * w_scale[n / 128, kb] [P5]. */
static float linear_block_one(const uint8_t* xq, const float* xs, const uint8_t* wq,
                              const float* ws, int64_t K, int64_t ldx, int64_t ldw,
                              int64_t m, int64_t n) {
    int64_t KB = K / 128;
    double y = 0.0;
    for (int64_t kb = 0; kb < KB; ++kb) {
        int64_t S = code_dot(xq + m * ldx, wq + n * ldw, kb * 128, kb * 128 + 128);
        y += (double)xs[m * KB + kb] * (double)ws[(n / 128) * KB + kb] * ldexp((double)S, -18);
    }
    return (float)y;
}

/* Full output Y[M,N] (fp32), mode 0 = channel/token, 1 = block-128. */
ORC_EXPORT void orc_linear(const uint8_t* xq, const float* xs, const uint8_t* wq,
                           const float* ws, int64_t M, int64_t N, int64_t K,
                           int64_t ldx, int64_t ldw, int mode, float* y) {
    build_ik_table();
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            y[m * N + n] = mode == 0
                ? linear_channel_one(xq, xs, wq, ws, K, ldx, ldw, m, n)
                : linear_block_one(xq, xs, wq, ws, K, ldx, ldw, m, n);
}

/* --------------------------------------------- weight-only FP8 (W8A16) */
/*
 * [P4] hardware section and FAQ Q1: without FP8 tensor cores (A100) the FP8
 * weights are dequantized when the layer runs and multiplied with bf16
 * activations.  y[m,n] = ws[n] * sum_k x[m,k] * E4M3value(wq[n,k]), x the
 * bf16 activations (not quantized); the sum is taken in double (each product
 * is exact in double) and the result rounded once to fp32.  y: [M, N].
 */
ORC_EXPORT void orc_linear_w8a16(const uint16_t* x, const uint8_t* wq, const float* ws,
                                 int64_t M, int64_t N, int64_t K, float* y) {
    build_mag_table();
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)bf16_to_float(x[m * K + k]) * orc_e4m3_decode(wq[n * K + k]);
            y[m * N + n] = (float)(acc * (double)ws[n]);
        }
}

/* ------------------------------------------------- gate/up with SiLU * up */
/*
 * [P1] section 1.3 (编码器细节：RMSNorm 与 SwiGLU 的实现差异): the Llama MLP
 * computes gate and up separately and multiplies SiLU(gate) by up (SwiGLU);
 * the product is down_proj's input.  Reading (the pages print no formula):
 * with g and u the bf16 outputs of the gate and up linears,
 *   act = bf16( bf16(silu(g)) * u ),  silu(v) = v / (1 + e^-v),
 * silu evaluated exactly (double) and rounded once to bf16, the product of
 * two bf16 values exact in fp32 and rounded once to bf16.
 * act: bf16 bits [M, N] (row-major, stride N).  Channel/token scales. */
ORC_EXPORT void orc_linear_swiglu(const uint8_t* xq, const float* xs, const uint8_t* wq_gate,
                                  const float* ws_gate, const uint8_t* wq_up, const float* ws_up,
                                  int64_t M, int64_t N, int64_t K, uint16_t* act) {
    build_ik_table();
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float g = linear_channel_one(xq, xs, wq_gate, ws_gate, K, K, K, m, n);
            float u = linear_channel_one(xq, xs, wq_up, ws_up, K, K, K, m, n);
            double gb = (double)bf16_to_float(float_to_bf16(g));
            double ub = (double)bf16_to_float(float_to_bf16(u));
            uint16_t sb = float_to_bf16((float)(gb / (1.0 + exp(-gb))));
            volatile float p = bf16_to_float(sb) * (float)ub;
            act[m * N + n] = float_to_bf16(p);
        }
}

/* Selected outputs y[i] = Y[ms[i], ns[i]], for spot checks at full size. */
ORC_EXPORT void orc_linear_at(const uint8_t* xq, const float* xs, const uint8_t* wq,
                              const float* ws, int64_t K, int64_t ldx, int64_t ldw, int mode,
                              const int64_t* ms, const int64_t* ns, int64_t count, float* y) {
    build_ik_table();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i)
        y[i] = mode == 0
            ? linear_channel_one(xq, xs, wq, ws, K, ldx, ldw, ms[i], ns[i])
            : linear_block_one(xq, xs, wq, ws, K, ldx, ldw, ms[i], ns[i]);
}
