/*
 * kvq_oracle.c - TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, fp64 CPU restatement of the rotated-angle KV-cache codec and
 * of attention over its codes.  It exists only to check the CUDA library:
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * load it.  It shares no code, header or table with the CUDA path.
 *
 * Method followed: "TurboAngle: Near-Lossless KV Cache Compression via
 * Uniform Angle Quantization", Abstract:
 *   - a random diagonal rotation followed by the Fast Walsh-Hadamard
 *     transform makes consecutive element pairs roughly uniform on the
 *     circle;
 *   - each pair's angle is quantized uniformly with a codebook of size L
 *     (set per layer, separately for K and V: "per-layer early-boost");
 *   - pair norms are quantized asymmetrically: 8-bit for keys, 4-bit in log
 *     space for values; no calibration data.
 * The abstract gives these steps in words.  The exact formulas below are the
 * plainest reading of them (they match the definitions stated in
 * include/kvq.h, which this file does not include):
 *   z      = H D x / sqrt(d), H[j][k] = (-1)^popcount(j&k) (Sylvester order)
 *   a_i    = floor((atan2(z[2i+1], z[2i]) + pi) L / (2 pi)) mod L,
 *            a_i = 0 for an exactly zero pair
 *   LIN8   M = fp16(max r), c = min(255, floor(255 r / M + 1/2))
 *   LOG4   l = log2(max(r, 2^-24)), LO/HI = fp16(min/max l),
 *          c = clamp(floor(15 (l - LO) / (HI - LO) + 1/2), 0, 15)
 *   theta^ = -pi + (a + 1/2) 2 pi / L (bin centre)
 * Attention is the textbook definition on the materialised dequantized
 * vectors (kvq_oracle_attend); kvq_oracle_attend_rotated is a second,
 * streaming form in the rotated domain used only to pin the first.
 *
 * Exactness: an fp16 value is an integer multiple of 2^-24 below 2^16, so
 * every partial sum of H D x over d <= 256 terms is an integer multiple of
 * 2^-24 below 2^24, i.e. exact in fp64.  The unscaled rotation is therefore
 * exact and the angle is taken from it.
 *
 * Flags: per pair, bit 0 marks an angle within 1e-6 rad of a bin edge, bit 1
 * a norm code within 1e-6 (relative) of its rounding edge, bit 2 a vector
 * whose fp16 parameter lies within 1e-6 (relative) of an fp16 rounding
 * midpoint.  Codes carrying a flag may legitimately differ between two
 * correct implementations.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_MODE_LIN8 0
#define ORACLE_MODE_LOG4 1
#define ORACLE_MODE_EXACT 2 /* oracle only: norms kept as fp64, for pins */

#define FLAG_ANGLE 1
#define FLAG_NORM 2
#define FLAG_PARAM 4

static const double EDGE_TOL = 1e-6;
static const double PI = 3.14159265358979323846264338327950288;

/* ---------------------------------------------------------------- fp16 -- */

static double half_to_double(uint16_t h) {
    _Float16 f;
    memcpy(&f, &h, 2);
    return (double)f;
}

/* Round to nearest even, straight from double (no detour through float). */
static uint16_t double_to_half(double x) {
    _Float16 f = (_Float16)x;
    uint16_t h;
    memcpy(&h, &f, 2);
    return h;
}

uint16_t kvq_oracle_double_to_half(double x) { return double_to_half(x); }
double kvq_oracle_half_to_double(uint16_t h) { return half_to_double(h); }

/* 1 if |v| lies within rel*|v| of a midpoint between two adjacent finite
 * fp16 values, i.e. where round-to-nearest could go either way. */
static int near_half_midpoint(double v, double rel) {
    double a = fabs(v);
    uint16_t h = double_to_half(a);
    if (h >= 0x7C00) h = 0x7BFF; /* saturated range: compare with top value */
    double hv = half_to_double(h);
    double tol = rel * a;
    if (h < 0x7BFF) {
        double up = half_to_double((uint16_t)(h + 1));
        if (fabs(a - 0.5 * (hv + up)) <= tol) return 1;
    }
    if (h > 0) {
        double dn = half_to_double((uint16_t)(h - 1));
        if (fabs(a - 0.5 * (hv + dn)) <= tol) return 1;
    }
    return 0;
}

/* ------------------------------------------------------------ layout --- */

int kvq_oracle_angle_bits(int L) {
    if (L < 2 || L > 65536) return -1;
    int b = 1;
    while ((1L << b) < (long)L) b++;
    return b;
}

/* Bytes per token: which 0 = angle words, 1 = norms, 2 = params. */
long kvq_oracle_row_bytes(int d, int L, int mode, int which) {
    int P = d / 2;
    int b = kvq_oracle_angle_bits(L);
    if (b < 0 || d < 4 || (d & (d - 1)) != 0) return -1;
    if (which == 0) return 4L * (((long)P * b + 31) / 32);
    if (which == 1) {
        if (mode == ORACLE_MODE_LIN8) return P;
        if (mode == ORACLE_MODE_LOG4) return P / 2;
        if (mode == ORACLE_MODE_EXACT) return 8L * P;
        return -1;
    }
    if (which == 2) {
        if (mode == ORACLE_MODE_LIN8) return 2;
        if (mode == ORACLE_MODE_LOG4) return 4;
        if (mode == ORACLE_MODE_EXACT) return 0;
        return -1;
    }
    return -1;
}

/* --------------------------------------------------------- rotation ---- */

static int hadamard(int j, int k) {
    return (__builtin_popcount((unsigned)(j & k)) & 1) ? -1 : 1;
}

/* zt = H y, plain O(d^2) sum (unscaled). */
static void hadamard_transform(const double* y, int d, double* zt) {
    for (int j = 0; j < d; j++) {
        double acc = 0.0;
        for (int k = 0; k < d; k++) acc += hadamard(j, k) * y[k];
        zt[j] = acc;
    }
}

/* z = H D x, optionally divided by sqrt(d). */
void kvq_oracle_rotate(const double* x, const int8_t* s, int d, int scaled,
                       double* z) {
    double y[256];
    for (int k = 0; k < d; k++) y[k] = s[k] * x[k];
    hadamard_transform(y, d, z);
    if (scaled)
        for (int j = 0; j < d; j++) z[j] = z[j] / sqrt((double)d);
}

/* x = D H z / sqrt(d): the inverse of the scaled rotation (H symmetric,
 * H H = d I, D D = I). */
void kvq_oracle_unrotate(const double* z, const int8_t* s, int d, double* x) {
    double w[256];
    hadamard_transform(z, d, w);
    for (int k = 0; k < d; k++) x[k] = s[k] * w[k] / sqrt((double)d);
}

/* --------------------------------------------------------- bit pack ---- */

static void put_bits(uint32_t* words, long bitpos, int nbits, uint32_t value) {
    for (int t = 0; t < nbits; t++)
        if ((value >> t) & 1u) words[(bitpos + t) / 32] |= 1u << ((bitpos + t) % 32);
}

static uint32_t get_bits(const uint32_t* words, long bitpos, int nbits) {
    uint32_t v = 0;
    for (int t = 0; t < nbits; t++)
        if ((words[(bitpos + t) / 32] >> ((bitpos + t) % 32)) & 1u) v |= 1u << t;
    return v;
}

static void words_to_bytes(const uint32_t* words, long nwords, uint8_t* out) {
    for (long w = 0; w < nwords; w++)
        for (int k = 0; k < 4; k++) out[4 * w + k] = (uint8_t)(words[w] >> (8 * k));
}

static void bytes_to_words(const uint8_t* in, long nwords, uint32_t* words) {
    for (long w = 0; w < nwords; w++) {
        words[w] = 0;
        for (int k = 0; k < 4; k++) words[w] |= (uint32_t)in[4 * w + k] << (8 * k);
    }
}

/* fp16 parameter: round to nearest even, saturate to the largest finite
 * value, and store a zero as +0 (reading: the sign of a zero parameter
 * carries no value, and for an exactly zero log-norm it would only echo the
 * rounding of the fp64 logarithm). */
static void put_half(uint8_t* dst, double v) {
    uint16_t h = double_to_half(v);
    if ((h & 0x7FFF) >= 0x7C00) h = (uint16_t)((h & 0x8000) | 0x7BFF); /* saturate */
    if (h == 0x8000) h = 0; /* -0 -> +0 */
    dst[0] = (uint8_t)(h & 0xFF);
    dst[1] = (uint8_t)(h >> 8);
}

static double get_half(const uint8_t* src) {
    return half_to_double((uint16_t)(src[0] | (src[1] << 8)));
}

/* ----------------------------------------------------------- encode ---- */

/* Encode one head vector.
 *   x_half     d fp16 bit patterns          s   d signs (+1 / -1)
 *   angle_row  row_bytes(which=0) bytes     norm_row / param_row likewise
 *   flags      P bytes (FLAG_* bits), may be NULL
 * Returns 0, or -1 for unsupported arguments. */
int kvq_oracle_encode(const uint16_t* x_half, const int8_t* s, int d, int L,
                      int mode, uint8_t* angle_row, uint8_t* norm_row,
                      uint8_t* param_row, uint8_t* flags) {
    enum { DMAX = 256 };
    int P = d / 2;
    int b = kvq_oracle_angle_bits(L);
    if (b < 0 || d < 4 || d > DMAX || (d & (d - 1)) != 0) return -1;
    if (mode < 0 || mode > 2) return -1;

    /* Step 1: the random diagonal, y = D x. */
    double y[DMAX];
    for (int k = 0; k < d; k++) y[k] = s[k] * half_to_double(x_half[k]);

    /* Step 2: the Walsh-Hadamard transform; zt unscaled (exact), z scaled. */
    double zt[DMAX], z[DMAX];
    hadamard_transform(y, d, zt);
    for (int j = 0; j < d; j++) z[j] = zt[j] / sqrt((double)d);

    /* Step 3: consecutive pairs in polar form. */
    double r[DMAX / 2];
    int a[DMAX / 2];
    uint8_t fl[DMAX / 2];
    for (int i = 0; i < P; i++) {
        fl[i] = 0;
        r[i] = hypot(z[2 * i], z[2 * i + 1]);
        /* Step 4: uniform angle quantization, L bins over (-pi, pi]. */
        double u = zt[2 * i], v = zt[2 * i + 1];
        if (u == 0.0 && v == 0.0) {
            a[i] = 0;
            continue;
        }
        double theta = atan2(v, u);
        double t = (theta + PI) * (double)L / (2.0 * PI);
        double ft = floor(t);
        a[i] = (int)ft % L;
        double f = t - ft, width = 2.0 * PI / (double)L;
        if (f * width < EDGE_TOL || (1.0 - f) * width < EDGE_TOL) fl[i] |= FLAG_ANGLE;
    }

    /* Step 5: norm quantization. */
    long nb = kvq_oracle_row_bytes(d, L, mode, 1);
    memset(norm_row, 0, (size_t)nb);
    if (mode == ORACLE_MODE_LIN8) {
        double mx = 0.0;
        for (int i = 0; i < P; i++) mx = r[i] > mx ? r[i] : mx;
        put_half(param_row, mx);
        double M = get_half(param_row);
        int pflag = near_half_midpoint(mx, EDGE_TOL);
        for (int i = 0; i < P; i++) {
            int c = 0;
            if (M > 0.0) {
                double vq = 255.0 * r[i] / M;
                double q = floor(vq + 0.5);
                c = q > 255.0 ? 255 : (int)q;
                if (fabs((vq - floor(vq)) - 0.5) < EDGE_TOL * fmax(vq, 1.0)) fl[i] |= FLAG_NORM;
            }
            norm_row[i] = (uint8_t)c;
            if (pflag) fl[i] |= FLAG_PARAM;
        }
    } else if (mode == ORACLE_MODE_LOG4) {
        double l[DMAX / 2];
        double lmin = INFINITY, lmax = -INFINITY;
        for (int i = 0; i < P; i++) {
            l[i] = log2(fmax(r[i], ldexp(1.0, -24)));
            lmin = fmin(lmin, l[i]);
            lmax = fmax(lmax, l[i]);
        }
        put_half(param_row, lmin);
        put_half(param_row + 2, lmax);
        double LO = get_half(param_row), HI = get_half(param_row + 2);
        int pflag = near_half_midpoint(lmin, EDGE_TOL) || near_half_midpoint(lmax, EDGE_TOL);
        for (int i = 0; i < P; i++) {
            int c = 0;
            if (HI != LO) {
                double vq = 15.0 * (l[i] - LO) / (HI - LO);
                double q = floor(vq + 0.5);
                c = q < 0.0 ? 0 : (q > 15.0 ? 15 : (int)q);
                if (fabs((vq - floor(vq)) - 0.5) < EDGE_TOL * fmax(fabs(vq), 1.0)) fl[i] |= FLAG_NORM;
            }
            norm_row[i / 2] |= (uint8_t)(c << (4 * (i % 2)));
            if (pflag) fl[i] |= FLAG_PARAM;
        }
    } else { /* ORACLE_MODE_EXACT: norms kept as fp64 */
        memcpy(norm_row, r, sizeof(double) * (size_t)P);
    }

    /* Step 6: pack the angle codes, LSB first, into 32-bit words. */
    long nw = kvq_oracle_row_bytes(d, L, mode, 0) / 4;
    uint32_t words[DMAX / 2 * 16 / 32 + 1];
    memset(words, 0, sizeof(words));
    for (int i = 0; i < P; i++) put_bits(words, (long)i * b, b, (uint32_t)a[i]);
    words_to_bytes(words, nw, angle_row);

    if (flags) memcpy(flags, fl, (size_t)P);
    return 0;
}

/* Batched encode over n vectors with contiguous rows. */
int kvq_oracle_encode_batch(const uint16_t* x_half, long n, const int8_t* s,
                            int d, int L, int mode, uint8_t* angles,
                            uint8_t* norms, uint8_t* params, uint8_t* flags) {
    long ab = kvq_oracle_row_bytes(d, L, mode, 0);
    long nb = kvq_oracle_row_bytes(d, L, mode, 1);
    long pb = kvq_oracle_row_bytes(d, L, mode, 2);
    if (ab < 0 || nb < 0 || pb < 0) return -1;
    for (long v = 0; v < n; v++) {
        int rc = kvq_oracle_encode(x_half + v * d, s, d, L, mode, angles + v * ab,
                                   norms + v * nb, params + v * pb,
                                   flags ? flags + v * (d / 2) : NULL);
        if (rc) return rc;
    }
    return 0;
}

/* ----------------------------------------------------------- decode ---- */

/* Read one token's codes back: angle codes a[P], norm codes c[P] (LIN8/LOG4)
 * and the reconstructed norms rhat[P].  Returns 0 or -1. */
int kvq_oracle_unpack(const uint8_t* angle_row, const uint8_t* norm_row,
                      const uint8_t* param_row, int d, int L, int mode,
                      int32_t* a, int32_t* c, double* rhat) {
    int P = d / 2;
    int b = kvq_oracle_angle_bits(L);
    if (b < 0) return -1;
    long nw = kvq_oracle_row_bytes(d, L, mode, 0) / 4;
    uint32_t words[256 / 2 * 16 / 32 + 1];
    bytes_to_words(angle_row, nw, words);
    for (int i = 0; i < P; i++) a[i] = (int32_t)get_bits(words, (long)i * b, b);
    if (mode == ORACLE_MODE_LIN8) {
        double M = get_half(param_row);
        for (int i = 0; i < P; i++) {
            c[i] = norm_row[i];
            rhat[i] = c[i] * M / 255.0;
        }
    } else if (mode == ORACLE_MODE_LOG4) {
        double LO = get_half(param_row), HI = get_half(param_row + 2);
        for (int i = 0; i < P; i++) {
            c[i] = (norm_row[i / 2] >> (4 * (i % 2))) & 0xF;
            rhat[i] = exp2(LO + c[i] * (HI - LO) / 15.0);
        }
    } else if (mode == ORACLE_MODE_EXACT) {
        memcpy(rhat, norm_row, sizeof(double) * (size_t)P);
        for (int i = 0; i < P; i++) c[i] = 0;
    } else {
        return -1;
    }
    return 0;
}

/* Reconstruction angle of code a: the centre of bin a. */
double kvq_oracle_theta_hat(int a, int L) {
    return -PI + (a + 0.5) * 2.0 * PI / (double)L;
}

/* Rotated-domain reconstruction zhat[d] of one token. */
int kvq_oracle_dequant_rotated(const uint8_t* angle_row, const uint8_t* norm_row,
                               const uint8_t* param_row, int d, int L, int mode,
                               double* zhat) {
    int32_t a[128], c[128];
    double rh[128];
    if (d > 256 || kvq_oracle_unpack(angle_row, norm_row, param_row, d, L, mode, a, c, rh))
        return -1;
    for (int i = 0; i < d / 2; i++) {
        double th = kvq_oracle_theta_hat(a[i], L);
        zhat[2 * i] = rh[i] * cos(th);
        zhat[2 * i + 1] = rh[i] * sin(th);
    }
    return 0;
}

/* Original-domain dequantized vector xhat = D H zhat / sqrt(d). */
int kvq_oracle_dequant(const uint8_t* angle_row, const uint8_t* norm_row,
                       const uint8_t* param_row, const int8_t* s, int d, int L,
                       int mode, double* xhat) {
    double zh[256];
    if (kvq_oracle_dequant_rotated(angle_row, norm_row, param_row, d, L, mode, zh)) return -1;
    kvq_oracle_unrotate(zh, s, d, xhat);
    return 0;
}

int kvq_oracle_dequant_batch(const uint8_t* angles, const uint8_t* norms,
                             const uint8_t* params, long n, const int8_t* s,
                             int d, int L, int mode, double* xhat) {
    long ab = kvq_oracle_row_bytes(d, L, mode, 0);
    long nb = kvq_oracle_row_bytes(d, L, mode, 1);
    long pb = kvq_oracle_row_bytes(d, L, mode, 2);
    if (ab < 0 || nb < 0 || pb < 0) return -1;
    for (long v = 0; v < n; v++) {
        int rc = kvq_oracle_dequant(angles + v * ab, norms + v * nb, params + v * pb,
                                    s, d, L, mode, xhat + v * d);
        if (rc) return rc;
    }
    return 0;
}

/* -------------------------------------------------------- attention ---- */

/* Textbook attention of G queries over T materialised keys/values:
 *   s_t = tau q.k_t,  p = softmax(s) (max subtracted),  out = sum_t p_t v_t.
 * T == 0 gives zeros. */
void kvq_oracle_attend(const double* q, const double* khat, const double* vhat,
                       int G, long T, int d, double tau, double* scores_tmp,
                       double* out) {
    for (int h = 0; h < G; h++) {
        double* o = out + (long)h * d;
        for (int j = 0; j < d; j++) o[j] = 0.0;
        if (T == 0) continue;
        double mx = -INFINITY;
        for (long t = 0; t < T; t++) {
            double dot = 0.0;
            for (int j = 0; j < d; j++) dot += q[(long)h * d + j] * khat[t * d + j];
            scores_tmp[t] = tau * dot;
            if (scores_tmp[t] > mx) mx = scores_tmp[t];
        }
        double den = 0.0;
        for (long t = 0; t < T; t++) {
            scores_tmp[t] = exp(scores_tmp[t] - mx);
            den += scores_tmp[t];
        }
        for (long t = 0; t < T; t++)
            for (int j = 0; j < d; j++) o[j] += scores_tmp[t] / den * vhat[t * d + j];
    }
}

/* Second form, used only to pin the first: rotate q once, score every token
 * straight from its codes, keep a running softmax, accumulate p * zhat_V in
 * the rotated domain and apply the inverse rotation once per head. */
int kvq_oracle_attend_rotated(const double* q, int G, int d, double tau,
                              const int8_t* sk, const int8_t* sv, int LK, int mk,
                              const uint8_t* ka, const uint8_t* kn, const uint8_t* kp,
                              int LV, int mv, const uint8_t* va, const uint8_t* vn,
                              const uint8_t* vp, long T, double* out) {
    long kab = kvq_oracle_row_bytes(d, LK, mk, 0), knb = kvq_oracle_row_bytes(d, LK, mk, 1);
    long kpb = kvq_oracle_row_bytes(d, LK, mk, 2);
    long vab = kvq_oracle_row_bytes(d, LV, mv, 0), vnb = kvq_oracle_row_bytes(d, LV, mv, 1);
    long vpb = kvq_oracle_row_bytes(d, LV, mv, 2);
    if (kab < 0 || vab < 0 || d > 256) return -1;
    int P = d / 2;
    for (int h = 0; h < G; h++) {
        double qr[256], acc[256], zv[256];
        int32_t a[128], c[128];
        double rh[128];
        kvq_oracle_rotate(q + (long)h * d, sk, d, 1, qr);
        for (int j = 0; j < d; j++) acc[j] = 0.0;
        double m = -INFINITY, den = 0.0;
        for (long t = 0; t < T; t++) {
            kvq_oracle_unpack(ka + t * kab, kn + t * knb, kp + t * kpb, d, LK, mk, a, c, rh);
            double sc = 0.0;
            for (int i = 0; i < P; i++) {
                double th = kvq_oracle_theta_hat(a[i], LK);
                sc += rh[i] * (qr[2 * i] * cos(th) + qr[2 * i + 1] * sin(th));
            }
            sc *= tau;
            double mnew = sc > m ? sc : m;
            double scale = exp(m - mnew); /* exp(-inf) = 0 on the first token */
            double p = exp(sc - mnew);
            den = den * scale + p;
            kvq_oracle_dequant_rotated(va + t * vab, vn + t * vnb, vp + t * vpb, d, LV, mv, zv);
            for (int j = 0; j < d; j++) acc[j] = acc[j] * scale + p * zv[j];
            m = mnew;
        }
        if (T == 0 || den == 0.0) {
            for (int j = 0; j < d; j++) out[(long)h * d + j] = 0.0;
            continue;
        }
        for (int j = 0; j < d; j++) acc[j] /= den;
        kvq_oracle_unrotate(acc, sv, d, out + (long)h * d);
    }
    return 0;
}
