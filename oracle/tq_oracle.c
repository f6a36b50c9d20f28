/*
 * tq_oracle.c -- plain fp64 CPU oracle for imatrix-weighted group-scale search,
 * round-to-nearest, low-bit packing and weighted reconstruction error.
 *
 * TEST INFRASTRUCTURE.  This file is the checker the CUDA library is compared
 * against.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load it.  It shares no code, header, table or constant
 * generator with the CUDA path: every table below is computed here from its
 * definition.
 *
 * Sources (web pages; cited by title and section):
 *  [NeUQI]  "NeUQI Accuracy Validation" (intel/auto-round docs/neuqi_acc.md),
 *           opening paragraph: asymmetric layers run a joint (scale, integer
 *           zero-point) search, symmetric layers a two-stage signed-scale search,
 *           both weighted by the activation imatrix; results bullet 2: the
 *           "64/32" grid.
 *  [TT]     "Quantize on TT cards: CUDA-free GPTQ/LDLQ bfp4 pipeline" (tt-stack
 *           issue #67), pipeline table step 1 (H = sum X^T X), step 3 (the
 *           GPTQ/LDLQ column sweep) and "Risks to measure: Precision" (proxy
 *           error tr(E H E^T)/tr(W H W^T); fp32 host propagation).
 *  [NVFP4]  "Nemotron-Cascade-2-30B-A3B-NVFP4" model card, Quantization Recipe
 *           table (NVFP4 group 16, MSE-calibrated static block scales) and the
 *           Calibration line (weight-MSE calibration).
 *  [INT3]   "int3-g64 (fmt=5)" (colibri PR #168), Design: Layout bullet
 *           (24 bytes per 64 weights: 16 B low plane of 2-bit values, 8 B high
 *           plane of 1-bit values, v in [-4,3] stored as v+4, one f32 scale per
 *           group) and Tests (outlier-row RMS vs per-row int4).
 *
 * Readings where the pages are silent are listed beside each function.  All
 * code decisions (round-to-nearest of w/s) are taken on the IEEE fp32
 * quotient, the precision the weights and scales are stored in; losses and
 * sums are accumulated in fp64 in natural element order.
 *
 * Build: gcc -O2 -fPIC -shared -fopenmp -ffp-contract=off (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* imatrix                                                             */
/* ------------------------------------------------------------------ */

/* m_j = (1/T) * sum_t x_{t,j}^2 for one [T, I] activation matrix with row
 * stride ld.  [NeUQI] opening paragraph ("weighted by the activation
 * imatrix"); [TT] step 1: H = sum_t x_t^T x_t, whose diagonal is T * m. */
ORC_API void orc_imatrix(const float* X, int64_t T, int64_t I, int64_t ld, double* m)
{
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < I; ++j) {
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            double x = (double)X[t * ld + j];
            s += x * x;
        }
        m[j] = T > 0 ? s / (double)T : 0.0;
    }
}

/* ------------------------------------------------------------------ */
/* Hessian H = sum_t x_t^T x_t                                         */
/* ------------------------------------------------------------------ */

/* H[i][j] = sum_t x_{t,i} x_{t,j} in fp64 for one [T, I] activation matrix
 * with row stride ld ([TT] pipeline table, step 1: the per-linear-input
 * Hessian accumulated over the calibration tokens).  Products of fp32 (and
 * bf16) values are exact in fp64; the sum is taken in token order.  H is
 * written in full (both triangles), row stride I. */
ORC_API void orc_hessian(const float* X, int64_t T, int64_t I, int64_t ld, double* H)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < I; ++i) {
        for (int64_t j = i; j < I; ++j) {
            double s = 0.0;
            for (int64_t t = 0; t < T; ++t) s += (double)X[t * ld + i] * (double)X[t * ld + j];
            H[i * I + j] = s;
            H[j * I + i] = s;
        }
    }
}

/* One entry H[i][j] (for sampled checks of large H). */
ORC_API double orc_hessian_entry(const float* X, int64_t T, int64_t ld, int64_t i, int64_t j)
{
    double s = 0.0;
    for (int64_t t = 0; t < T; ++t) s += (double)X[t * ld + i] * (double)X[t * ld + j];
    return s;
}

/* Proxy error with a full Hessian ([TT] "Risks to measure: Precision"):
 * num = tr(E H E^T) = sum_o sum_{i,j} e_{o,i} H_{i,j} e_{o,j}, E = W - What,
 * den = tr(W H W^T), for one O x I matrix; fp64 throughout. */
ORC_API void orc_proxy_error_full(const float* W, const float* What, int64_t O, int64_t I,
                                  const double* H, double* num, double* den)
{
    double n = 0.0, d = 0.0;
    #pragma omp parallel for reduction(+:n, d) schedule(static)
    for (int64_t o = 0; o < O; ++o) {
        const float* w = W + o * I;
        const float* wh = What + o * I;
        for (int64_t i = 0; i < I; ++i) {
            double hn = 0.0, hd = 0.0;
            for (int64_t j = 0; j < I; ++j) {
                hn += H[i * I + j] * ((double)w[j] - (double)wh[j]);
                hd += H[i * I + j] * (double)w[j];
            }
            n += ((double)w[i] - (double)wh[i]) * hn;
            d += (double)w[i] * hd;
        }
    }
    *num = n;
    *den = d;
}

/* ------------------------------------------------------------------ */
/* Round-to-nearest helpers                                            */
/* ------------------------------------------------------------------ */

/* Integer code of w under scale s: round half to even of the fp32 quotient
 * w/s, clamped to [lo, hi].  A zero scale gives code 0 (the group or block
 * holds no magnitude to represent). */
static double rtn_code(float w, float s, double lo, double hi)
{
    if (s == 0.0f) return 0.0;
    float y = w / s;                 /* IEEE single division */
    double q = nearbyint((double)y); /* current rounding mode: to nearest, ties to even */
    if (q < lo) q = lo;
    if (q > hi) q = hi;
    return q;
}

/* ------------------------------------------------------------------ */
/* Symmetric int3-g64 two-stage signed-scale search                    */
/* ------------------------------------------------------------------ */

/* Stage-1 magnitude ratios r_k = fl32(lo + ((hi - lo) * k) / (n1 - 1)),
 * k = 0..n1-1, i.e. n1 points of linspace(lo, hi) rounded once to fp32.
 * Scale of candidate c = 2k + sigma: s = (1 - 2 sigma) * fl32(r_k * M) * 0.25,
 * with M = max|w| over the group and 0.25 = 1/4 (the int3 grid's positive
 * reach).  [NeUQI] opening paragraph: "two-stage signed scale search". */
ORC_API float orc_sym_stage1_ratio(int n1, double lo, double hi, int k)
{
    return (float)(lo + ((hi - lo) * (double)k) / (double)(n1 - 1));
}

/* Stage-2 ratio i around stage-1 magnitude k*: n2 points of linspace over
 * [r_{k*} - delta, r_{k*} + delta] in fp64, rounded once to fp32, where
 * delta = (hi - lo)/(n1 - 1) is the stage-1 spacing (reading: "refinements
 * around the best" span the neighbouring stage-1 points). */
ORC_API float orc_sym_stage2_ratio(int n1, int n2, double lo, double hi, int kstar, int i)
{
    double delta = (hi - lo) / (double)(n1 - 1);
    double center = lo + ((hi - lo) * (double)kstar) / (double)(n1 - 1);
    return (float)((center - delta) + (2.0 * delta * (double)i) / (double)(n2 - 1));
}

static float sym_scale(float r, float M, int negative)
{
    float a = (float)((double)r * (double)M); /* exact product, rounded once */
    a = a * 0.25f;
    return negative ? -a : a;
}

/* Weighted squared error of one group under scale s, codes v in [-4, 3]:
 * L = sum_j m_j (w_j - s v_j)^2 in fp64. */
ORC_API double orc_sym_loss(const float* w, const float* m, int n, float s, int8_t* v_out)
{
    double L = 0.0;
    for (int j = 0; j < n; ++j) {
        double v = rtn_code(w[j], s, -4.0, 3.0);
        double e = (double)w[j] - (double)s * v;
        L += (double)m[j] * (e * e);
        if (v_out) v_out[j] = (int8_t)v;
    }
    return L;
}

/* One group of n <= 64 weights.  Returns the candidate index: 2k+sigma for a
 * stage-1 winner, 2*n1 + i for a stage-2 winner, -1 for an all-zero group.
 * Ties keep the lower index (a candidate replaces the incumbent only when its
 * loss is strictly smaller).  Stage 2 keeps the stage-1 sign and replaces the
 * stage-1 winner only on a strict improvement. */
ORC_API int orc_search_sym_group(const float* w, const float* m, int n, int n1, int n2,
                                 double lo, double hi, float* scale_out, double* loss_out,
                                 int8_t* codes_out)
{
    float M = 0.0f;
    for (int j = 0; j < n; ++j) { float a = fabsf(w[j]); if (a > M) M = a; }
    if (M == 0.0f) {
        *scale_out = 0.0f; *loss_out = 0.0;
        if (codes_out) memset(codes_out, 0, (size_t)n);
        return -1;
    }
    int best = -1; double bestL = INFINITY; float bestS = 0.0f;
    for (int k = 0; k < n1; ++k) {
        float r = orc_sym_stage1_ratio(n1, lo, hi, k);
        for (int sg = 0; sg < 2; ++sg) {
            float s = sym_scale(r, M, sg);
            double L = orc_sym_loss(w, m, n, s, NULL);
            if (L < bestL) { bestL = L; best = 2 * k + sg; bestS = s; }
        }
    }
    int kstar = best / 2, sgstar = best % 2;
    int best2 = best; double bestL2 = bestL; float bestS2 = bestS;
    for (int i = 0; i < n2; ++i) {
        float r = orc_sym_stage2_ratio(n1, n2, lo, hi, kstar, i);
        float s = sym_scale(r, M, sgstar);
        double L = orc_sym_loss(w, m, n, s, NULL);
        if (L < bestL2) { bestL2 = L; best2 = 2 * n1 + i; bestS2 = s; }
    }
    *scale_out = bestS2; *loss_out = bestL2;
    if (codes_out) orc_sym_loss(w, m, n, bestS2, codes_out);
    return best2;
}

/* ------------------------------------------------------------------ */
/* Asymmetric int4-g128 joint (scale, integer zero-point) search       */
/* ------------------------------------------------------------------ */

/* Scale factor table c_k = fl32(f_k / 15), f_k = lo + ((hi - lo) * k)/(ns - 1):
 * candidate scale s_k = fl32(c_k * R), R = fl32(wmax - wmin).  Reading: the
 * pages give the "64/32" grid size but not its range; the range is taken
 * equal to the symmetric stage-1 window [0.5, 1.2]. */
ORC_API float orc_asym_scale_factor(int ns, double lo, double hi, int k)
{
    double f = lo + ((hi - lo) * (double)k) / (double)(ns - 1);
    return (float)(f / 15.0);
}

/* Zero-point i of nz: z_i = rint(15 i / (nz - 1)) (ties to even).  Reading:
 * "32 integer zero-points in [0,15]" names more points than integers in the
 * range; the nz points are spread evenly over [0,15] and rounded, so every
 * integer 0..15 occurs and duplicates never win under the strict-improvement
 * rule. */
ORC_API int orc_asym_zero(int nz, int i)
{
    return (int)nearbyint((15.0 * (double)i) / (double)(nz - 1));
}

ORC_API double orc_asym_loss(const float* w, const float* m, int n, float s, int z, uint8_t* q_out)
{
    double L = 0.0;
    for (int j = 0; j < n; ++j) {
        double q;
        if (s == 0.0f) q = (double)z;
        else {
            float y = w[j] / s;
            q = nearbyint((double)y) + (double)z;
            if (q < 0.0) q = 0.0;
            if (q > 15.0) q = 15.0;
        }
        double e = (double)w[j] - (double)s * (q - (double)z);
        L += (double)m[j] * (e * e);
        if (q_out) q_out[j] = (uint8_t)q;
    }
    return L;
}

/* One group of n <= 128 weights.  Candidate index ns_idx = nz * k + i.
 * Degenerate groups: wmax == wmin == 0 gives s = 0, z = 0 and index -1;
 * wmax == wmin != 0 uses R = |wmax|. */
ORC_API int orc_search_asym_group(const float* w, const float* m, int n, int ns, int nz,
                                  double lo, double hi, float* scale_out, uint8_t* zero_out,
                                  double* loss_out, uint8_t* q_out)
{
    float wmin = w[0], wmax = w[0];
    for (int j = 1; j < n; ++j) { if (w[j] < wmin) wmin = w[j]; if (w[j] > wmax) wmax = w[j]; }
    float R = (float)((double)wmax - (double)wmin);
    if (R == 0.0f) {
        if (wmax == 0.0f) {
            *scale_out = 0.0f; *zero_out = 0; *loss_out = 0.0;
            if (q_out) memset(q_out, 0, (size_t)n);
            return -1;
        }
        R = fabsf(wmax);
    }
    int best = -1; double bestL = INFINITY; float bestS = 0.0f; int bestZ = 0;
    for (int k = 0; k < ns; ++k) {
        float c = orc_asym_scale_factor(ns, lo, hi, k);
        float s = (float)((double)c * (double)R);
        for (int i = 0; i < nz; ++i) {
            int z = orc_asym_zero(nz, i);
            double L = orc_asym_loss(w, m, n, s, z, NULL);
            if (L < bestL) { bestL = L; best = nz * k + i; bestS = s; bestZ = z; }
        }
    }
    *scale_out = bestS; *zero_out = (uint8_t)bestZ; *loss_out = bestL;
    if (q_out) orc_asym_loss(w, m, n, bestS, bestZ, q_out);
    return best;
}

/* ------------------------------------------------------------------ */
/* NVFP4-g16: E2M1 elements, E4M3 block scales, fp32 global scale      */
/* ------------------------------------------------------------------ */

/* E4M3 (e4m3fn) decode: s eeee mmm, bias 7; exponent 0 is subnormal
 * (m * 2^-9); 0x7F / 0xFF are NaN; 0x7E = 448 is the largest finite value. */
ORC_API double orc_e4m3_decode(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, mt = code & 7;
    if (e == 15 && mt == 7) return NAN;
    double v = (e == 0) ? ldexp((double)mt, -9) : ldexp(1.0 + (double)mt / 8.0, e - 7);
    return s ? -v : v;
}

static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Magnitude code (0..7) of y >= 0 under E2M1 round-to-nearest-even with
 * saturation: the nearest of {0,.5,1,1.5,2,3,4,6}; a tie goes to the even
 * code; values above 6 (and +inf) give 6; NaN gives 0. */
ORC_API int orc_e2m1_rne_mag(float y)
{
    if (isnan(y)) return 0;
    if (y > 6.0f) return 7;   /* saturate: also keeps huge y from tying 4 and 6 */
    double best_d = INFINITY; int best = 0;
    for (int i = 0; i < 8; ++i) {
        double d = fabs((double)y - E2M1_MAG[i]);
        if (d < best_d || (d == best_d && (i % 2) == 0)) { best_d = d; best = i; }
    }
    return best;
}

/* Per-tensor global scale g = fl32(amax / (6 * 448)). */
ORC_API float orc_nvfp4_global(const float* W, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) { float a = fabsf(W[i]); if (a > amax) amax = a; }
    return (float)((double)amax / 2688.0);
}

/* The `window` positive finite E4M3 codes (1..126) whose values lie nearest
 * t = a / (6 g), ties to the lower code, listed in ascending code order.
 * Reading of "the 16 E4M3 codes nearest amax/6": t is the block amax over 6
 * in units of the global scale.  Distances are compared as
 * |6 g dec(c) - a| (the distance to t scaled by 6g > 0, which orders codes
 * the same way); every term is exact in fp64 (6 g dec(c) has at most 31
 * significant bits), so no rounding can reorder two codes.  Done as the plain
 * definition: rank all 126 codes by (distance, code), keep the first
 * `window`. */
ORC_API void orc_nvfp4_window(float a, float g, int window, int* codes_out)
{
    int chosen[127]; memset(chosen, 0, sizeof chosen);
    double g6 = 6.0 * (double)g;
    for (int r = 0; r < window; ++r) {
        int best = -1; double bd = INFINITY;
        for (int c = 1; c <= 126; ++c) {
            if (chosen[c]) continue;
            double d = fabs(g6 * orc_e4m3_decode(c) - (double)a);
            if (d < bd) { bd = d; best = c; }   /* strict: ties keep the lower code */
        }
        chosen[best] = 1;
    }
    int k = 0;
    for (int c = 1; c <= 126; ++c) if (chosen[c]) codes_out[k++] = c;
}

ORC_API double orc_nvfp4_loss(const float* w, const float* m, int n, float S, uint8_t* c_out)
{
    double L = 0.0;
    for (int j = 0; j < n; ++j) {
        int mag;
        if (S == 0.0f) mag = 0;
        else mag = orc_e2m1_rne_mag(fabsf(w[j]) / S);
        double e = fabs((double)w[j]) - (double)S * E2M1_MAG[mag];
        L += (double)m[j] * (e * e);
        if (c_out) c_out[j] = (uint8_t)((mag != 0 && w[j] < 0.0f) ? (mag | 8) : mag);
    }
    return L;
}

/* One block of n <= 16 weights under global scale g.  Returns the chosen
 * E4M3 scale code (1..126), or -1 (scale byte 0, codes 0) for an all-zero
 * block or g == 0.  Candidates are the window codes in ascending order with
 * block scale S = fl32(g * dec(e)); ties keep the lower code. */
ORC_API int orc_search_nvfp4_block(const float* w, const float* m, int n, float g, int window,
                                   double* loss_out, uint8_t* c_out)
{
    float a = 0.0f;
    for (int j = 0; j < n; ++j) { float v = fabsf(w[j]); if (v > a) a = v; }
    if (a == 0.0f || g == 0.0f) {
        double L = 0.0;
        for (int j = 0; j < n; ++j) L += (double)m[j] * ((double)w[j] * (double)w[j]);
        *loss_out = L;
        if (c_out) memset(c_out, 0, (size_t)n);
        return -1;
    }
    int codes[126];
    orc_nvfp4_window(a, g, window, codes);
    int best = -1; double bestL = INFINITY;
    for (int r = 0; r < window; ++r) {
        float S = (float)((double)g * orc_e4m3_decode(codes[r]));
        double L = orc_nvfp4_loss(w, m, n, S, NULL);
        if (L < bestL) { bestL = L; best = codes[r]; }
    }
    *loss_out = bestL;
    if (c_out) orc_nvfp4_loss(w, m, n, (float)((double)g * orc_e4m3_decode(best)), c_out);
    return best;
}

/* ------------------------------------------------------------------ */
/* Batched searches over [n_mat, O, I] (OpenMP over independent groups) */
/* ------------------------------------------------------------------ */

/* W: n_mat matrices, row stride ld, matrix stride ms.  m: imatrix of matrix e
 * at m + e * m_stride (m_stride 0 = shared).  Outputs per group [n_mat, O, G]
 * and codes [n_mat, O, I] (int8 v for int3; uint8 q for int4; uint8 E2M1 code
 * for NVFP4).  Any output pointer may be NULL. */
ORC_API void orc_search_sym_int3(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld,
                                 int64_t ms, const float* m, int64_t m_stride, int n1, int n2,
                                 double lo, double hi, float* scales, int32_t* idx, double* loss,
                                 int8_t* codes)
{
    const int64_t G = (I + 63) / 64;
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t gi = 0; gi < n_mat * O * G; ++gi) {
        int64_t e = gi / (O * G), o = (gi / G) % O, k = gi % G;
        int64_t j0 = k * 64; int n = (int)((I - j0) < 64 ? (I - j0) : 64);
        const float* w = W + e * ms + o * ld + j0;
        const float* mm = m + e * m_stride + j0;
        float s; double L;
        int c = orc_search_sym_group(w, mm, n, n1, n2, lo, hi, &s, &L,
                                     codes ? codes + (e * O + o) * I + j0 : NULL);
        if (scales) scales[gi] = s;
        if (idx) idx[gi] = c;
        if (loss) loss[gi] = L;
    }
}

/* g: weights per group, 128 (int4-g128) or 64 (int4-g64: the per-projection
 * ablation's int4-g64 scheme on the int3-g64 page, read as the same joint
 * search on 64-weight groups). */
ORC_API void orc_search_asym_int4(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld,
                                  int64_t ms, const float* m, int64_t m_stride, int ns, int nz,
                                  double lo, double hi, float* scales, uint8_t* zeros, int32_t* idx,
                                  double* loss, uint8_t* codes, int g)
{
    const int64_t G = (I + g - 1) / g;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t gi = 0; gi < n_mat * O * G; ++gi) {
        int64_t e = gi / (O * G), o = (gi / G) % O, k = gi % G;
        int64_t j0 = k * g; int n = (int)((I - j0) < g ? (I - j0) : g);
        const float* w = W + e * ms + o * ld + j0;
        const float* mm = m + e * m_stride + j0;
        float s; uint8_t z; double L;
        int c = orc_search_asym_group(w, mm, n, ns, nz, lo, hi, &s, &z, &L,
                                      codes ? codes + (e * O + o) * I + j0 : NULL);
        if (scales) scales[gi] = s;
        if (zeros) zeros[gi] = z;
        if (idx) idx[gi] = c;
        if (loss) loss[gi] = L;
    }
}

/* gscale: per-matrix global scale g (computed by the caller with
 * orc_nvfp4_global, or any given value).  scale_codes: E4M3 byte per block. */
ORC_API void orc_search_nvfp4(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld,
                              int64_t ms, const float* m, int64_t m_stride, const float* gscale,
                              int window, uint8_t* scale_codes, int32_t* idx, double* loss,
                              uint8_t* codes)
{
    const int64_t G = (I + 15) / 16;
    #pragma omp parallel for schedule(dynamic, 256)
    for (int64_t gi = 0; gi < n_mat * O * G; ++gi) {
        int64_t e = gi / (O * G), o = (gi / G) % O, k = gi % G;
        int64_t j0 = k * 16; int n = (int)((I - j0) < 16 ? (I - j0) : 16);
        const float* w = W + e * ms + o * ld + j0;
        const float* mm = m + e * m_stride + j0;
        double L;
        int c = orc_search_nvfp4_block(w, mm, n, gscale[e], window, &L,
                                       codes ? codes + (e * O + o) * I + j0 : NULL);
        if (scale_codes) scale_codes[gi] = (uint8_t)(c < 0 ? 0 : c);
        if (idx) idx[gi] = c;
        if (loss) loss[gi] = L;
    }
}

/* Loss of GIVEN per-group parameters (for re-evaluating another
 * implementation's choices): the same per-group losses as above, over every
 * group of [n_mat, O, I]. */
ORC_API void orc_loss_given_int3(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld,
                                 int64_t ms, const float* m, int64_t m_stride, const float* scales,
                                 double* loss)
{
    const int64_t G = (I + 63) / 64;
    #pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < n_mat * O * G; ++gi) {
        int64_t e = gi / (O * G), o = (gi / G) % O, k = gi % G;
        int64_t j0 = k * 64; int n = (int)((I - j0) < 64 ? (I - j0) : 64);
        loss[gi] = orc_sym_loss(W + e * ms + o * ld + j0, m + e * m_stride + j0, n, scales[gi], NULL);
    }
}

ORC_API void orc_loss_given_int4(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld,
                                 int64_t ms, const float* m, int64_t m_stride, const float* scales,
                                 const uint8_t* zeros, double* loss, int g)
{
    const int64_t G = (I + g - 1) / g;
    #pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < n_mat * O * G; ++gi) {
        int64_t e = gi / (O * G), o = (gi / G) % O, k = gi % G;
        int64_t j0 = k * g; int n = (int)((I - j0) < g ? (I - j0) : g);
        loss[gi] = orc_asym_loss(W + e * ms + o * ld + j0, m + e * m_stride + j0, n, scales[gi],
                                 zeros[gi], NULL);
    }
}

ORC_API void orc_loss_given_nvfp4(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld,
                                  int64_t ms, const float* m, int64_t m_stride,
                                  const uint8_t* scale_codes, const float* gscale, double* loss)
{
    const int64_t G = (I + 15) / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t gi = 0; gi < n_mat * O * G; ++gi) {
        int64_t e = gi / (O * G), o = (gi / G) % O, k = gi % G;
        int64_t j0 = k * 16; int n = (int)((I - j0) < 16 ? (I - j0) : 16);
        float S = (float)((double)gscale[e] * orc_e4m3_decode(scale_codes[gi]));
        loss[gi] = orc_nvfp4_loss(W + e * ms + o * ld + j0, m + e * m_stride + j0, n, S, NULL);
    }
}

/* ------------------------------------------------------------------ */
/* FP8 (E4M3) with one scale per tensor                                */
/* ------------------------------------------------------------------ */

/* Code of a non-negative E4M3 value v (exactly representable). */
static int e4m3_code_of_value(double v)
{
    if (v == 0.0) return 0;
    if (v < ldexp(1.0, -6)) return (int)(v * 512.0);          /* subnormal: m 2^-9 */
    int e;
    double f = frexp(v, &e);                                  /* v = f 2^e, f in [0.5, 1) */
    return ((e - 1 + 7) << 3) | (int)((2.0 * f - 1.0) * 8.0);  /* (1 + m/8) 2^(E-7) */
}

/* E4M3 code of y: round to nearest, ties to the even code, saturating at
 * +-448 (the largest finite e4m3fn value); a value that rounds to zero is
 * code 0 (+0); NaN gives 0.  [NVFP4] recipe table: FP8 per-tensor for the
 * shared experts and the Mamba linears.  The rounding step is 2^-9 below
 * 2^-6 (subnormals) and 2^(floor(log2 y) - 3) above (3 mantissa bits). */
ORC_API int orc_e4m3_rne(float y)
{
    double a = fabs((double)y);
    if (!(a == a)) return 0;
    double v;
    if (a >= 448.0) v = 448.0;
    else {
        double step = a < ldexp(1.0, -6) ? ldexp(1.0, -9) : ldexp(1.0, ilogb(a) - 3);
        v = nearbyint(a / step) * step;                       /* a / step is exact */
        if (v > 448.0) v = 448.0;
    }
    int c = e4m3_code_of_value(v);
    return (y < 0.0f && c != 0) ? (c | 0x80) : c;
}

/* Candidate k of the per-tensor grid: ratio r_k = fl32(lo + ((hi - lo) k) /
 * (n - 1)) of amax / 448, scale s_k = fl32(r_k amax / 448) (one rounding).
 * Reading: the NeUQI search window [0.5, 1.2], as the asymmetric grid's. */
ORC_API float orc_fp8_scale(int n, double lo, double hi, int k, float amax)
{
    float r = (float)(lo + ((hi - lo) * (double)k) / (double)(n - 1));
    return (float)((double)r * (double)amax / 448.0);
}

/* Per matrix: amax = max |w|; for each of the n candidate scales the loss
 * L_k = sum_{o,j} m_j (w - fl32(s_k dec(c)))^2 with c = orc_e4m3_rne(fl32(w / s_k))
 * (fp64); the chosen k is the lowest of the minimum loss.  amax = 0 gives
 * scale 0, index -1, loss 0 and codes 0.  codes: [n_mat][O][I] u8 (optional);
 * losses: [n_mat][n] (optional). */
ORC_API void orc_search_fp8(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms,
                            const float* m, int64_t m_stride, int n, double lo, double hi,
                            float* scales, int32_t* idx, double* loss, double* losses, uint8_t* codes)
{
    for (int64_t e = 0; e < n_mat; ++e) {
        const float* We = W + e * ms;
        const float* me = m + e * m_stride;
        double amax = 0.0;
        for (int64_t o = 0; o < O; ++o)
            for (int64_t j = 0; j < I; ++j) {
                double a = fabs((double)We[o * ld + j]);
                if (a > amax) amax = a;
            }
        int best = -1;
        double bestL = INFINITY;
        float bestS = 0.0f;
        for (int k = 0; k < n; ++k) {
            float sk = orc_fp8_scale(n, lo, hi, k, (float)amax);
            double L = 0.0;
            if (amax > 0.0) {
                #pragma omp parallel for reduction(+:L) schedule(static)
                for (int64_t o = 0; o < O; ++o)
                    for (int64_t j = 0; j < I; ++j) {
                        float w = We[o * ld + j];
                        int c = orc_e4m3_rne(w / sk);
                        double wh = (double)(float)((double)sk * orc_e4m3_decode(c));
                        double d = (double)w - wh;
                        L += (double)me[j] * (d * d);
                    }
            }
            if (losses) losses[e * n + k] = L;
            if (amax > 0.0 && L < bestL) { bestL = L; best = k; bestS = sk; }
        }
        if (amax == 0.0) { bestL = 0.0; bestS = 0.0f; best = -1; }
        scales[e] = bestS;
        if (idx) idx[e] = best;
        if (loss) loss[e] = bestL;
        if (codes)
            for (int64_t o = 0; o < O; ++o)
                for (int64_t j = 0; j < I; ++j)
                    codes[(e * O + o) * I + j] = bestS == 0.0f ? 0 : (uint8_t)orc_e4m3_rne(We[o * ld + j] / bestS);
    }
}

/* What = fl32(s dec(c)) for codes [n_mat][O][I] and one scale per matrix. */
ORC_API void orc_dequant_fp8(const uint8_t* c, int64_t n_mat, int64_t OI, const float* scales, float* out)
{
    for (int64_t e = 0; e < n_mat; ++e)
        for (int64_t i = 0; i < OI; ++i)
            out[e * OI + i] = (float)((double)scales[e] * orc_e4m3_decode(c[e * OI + i]));
}

/* ------------------------------------------------------------------ */
/* Imatrix-weighted Lloyd-Max 2-bit codebook                           */
/* ------------------------------------------------------------------ */
/* "Phase 2: math-accuracy regression on tq3a-tq2e g32" (turboquant-mlx issue
 * #2), Phase-2 candidate 1: a Lloyd-Max codebook for the 2-bit experts fit to
 * calibration data instead of the data-free one, fixed and shared.  Reading:
 * 32-weight groups with an absmax scale s = max |w|; normalised values
 * u = fl32(w / s) (0 when s = 0); one 4-level codebook c_0 < ... < c_3 (fp32)
 * shared by every matrix of the call, fit by Lloyd iterations that minimise
 * sum m_j (w - s c_a)^2 = sum omega (u - c_a)^2, omega = m_j s^2: each
 * element goes to the nearest level (ties to the lower one: u above the exact
 * midpoint (c_i + c_{i+1}) / 2 moves up), each level becomes the
 * omega-weighted mean of its elements (fp64, rounded once to fp32; an empty
 * level keeps its value); start from the data-free Lloyd-Max levels of a
 * uniform source on [-1, 1], {-3/4, -1/4, 1/4, 3/4}. */

static double lm_u(float w, float s) { return s == 0.0f ? 0.0 : (double)(w / s); }

static int lm_assign(double u, const float* c)
{
    int a = 0;
    for (int i = 0; i < 3; ++i)
        if (u > ((double)c[i] + (double)c[i + 1]) / 2.0) a = i + 1;
    return a;
}

/* Group absmax scales [rows][G32] of W. */
static void lm_scales(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms, float* scales)
{
    const int64_t G = (I + 31) / 32;
    for (int64_t e = 0; e < n_mat; ++e)
        for (int64_t o = 0; o < O; ++o)
            for (int64_t k = 0; k < G; ++k) {
                float a = 0.0f;
                for (int64_t j = 32 * k; j < I && j < 32 * k + 32; ++j) {
                    float v = fabsf(W[e * ms + o * ld + j]);
                    if (v > a) a = v;
                }
                scales[(e * O + o) * G + k] = a;
            }
}

/* n_iter Lloyd iterations.  codebook: in/out [4] (the start, then the fit);
 * scales: out [n_mat][O][G32]; codes: out [n_mat][O][I] (0..3, optional);
 * loss: out, sum m (w - s c_a)^2 over every matrix for the final codebook;
 * history: optional [n_iter + 1] losses before each update and after the last. */
ORC_API void orc_lloyd_max_g32(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms,
                               const float* m, int64_t m_stride, int n_iter, float* codebook, float* scales,
                               uint8_t* codes, double* loss, double* history)
{
    const int64_t G = (I + 31) / 32;
    lm_scales(W, n_mat, O, I, ld, ms, scales);
    for (int it = 0; it <= n_iter; ++it) {
        double num[4] = {0, 0, 0, 0}, den[4] = {0, 0, 0, 0}, L = 0.0;
        for (int64_t e = 0; e < n_mat; ++e)
            for (int64_t o = 0; o < O; ++o)
                for (int64_t j = 0; j < I; ++j) {
                    float s = scales[(e * O + o) * G + j / 32];
                    double u = lm_u(W[e * ms + o * ld + j], s);
                    int a = lm_assign(u, codebook);
                    double om = (double)m[e * m_stride + j] * (double)s * (double)s;
                    num[a] += om * u;
                    den[a] += om;
                    double d = u - (double)codebook[a];
                    L += om * d * d;
                }
        if (history) history[it] = L;
        if (it == n_iter) { *loss = L; break; }
        for (int i = 0; i < 4; ++i)
            if (den[i] > 0.0) codebook[i] = (float)(num[i] / den[i]);
    }
    if (codes)
        for (int64_t e = 0; e < n_mat; ++e)
            for (int64_t o = 0; o < O; ++o)
                for (int64_t j = 0; j < I; ++j)
                    codes[(e * O + o) * I + j] = (uint8_t)lm_assign(
                        lm_u(W[e * ms + o * ld + j], scales[(e * O + o) * G + j / 32]), codebook);
}

/* Codes for a given codebook and the group absmax scales. */
ORC_API void orc_lloyd_max_assign(const float* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms,
                                  const float* codebook, float* scales, uint8_t* codes)
{
    const int64_t G = (I + 31) / 32;
    lm_scales(W, n_mat, O, I, ld, ms, scales);
    for (int64_t e = 0; e < n_mat; ++e)
        for (int64_t o = 0; o < O; ++o)
            for (int64_t j = 0; j < I; ++j)
                codes[(e * O + o) * I + j] = (uint8_t)lm_assign(
                    lm_u(W[e * ms + o * ld + j], scales[(e * O + o) * G + j / 32]), codebook);
}

/* 2-bit codes (0..3) [rows][I] -> 8-byte records per 32-weight group:
 * element k of a group at bits 2 (k % 4) of byte k / 4; padding code 0. */
ORC_API void orc_pack_lm2(const uint8_t* codes, int64_t rows, int64_t I, uint8_t* out)
{
    const int64_t G = (I + 31) / 32;
    memset(out, 0, (size_t)(rows * G * 8));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            int64_t k = j % 32, gi = r * G + j / 32;
            out[gi * 8 + k / 4] |= (uint8_t)((codes[r * I + j] & 3) << (2 * (k % 4)));
        }
}

/* What = fl32(s c_a) for codes [rows][I], group scales [rows][G32]. */
ORC_API void orc_dequant_lm2(const uint8_t* codes, int64_t rows, int64_t I, const float* scales,
                             const float* codebook, float* out)
{
    const int64_t G = (I + 31) / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j)
            out[r * I + j] = (float)((double)scales[r * G + j / 32] * (double)codebook[codes[r * I + j] & 3]);
}

/* ------------------------------------------------------------------ */
/* Round-to-nearest with given scales (pack path)                      */
/* ------------------------------------------------------------------ */

/* rows = n_mat * O contiguous rows of I weights (row stride I). */
ORC_API void orc_rtn_int3(const float* W, int64_t rows, int64_t I, const float* scales, int8_t* v)
{
    const int64_t G = (I + 63) / 64;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j)
            v[r * I + j] = (int8_t)rtn_code(W[r * I + j], scales[r * G + j / 64], -4.0, 3.0);
}

ORC_API void orc_rtn_int4(const float* W, int64_t rows, int64_t I, const float* scales,
                          const uint8_t* zeros, uint8_t* q, int g)
{
    const int64_t G = (I + g - 1) / g;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            float s = scales[r * G + j / g]; int z = zeros[r * G + j / g];
            double qq;
            if (s == 0.0f) qq = (double)z;
            else {
                qq = nearbyint((double)(W[r * I + j] / s)) + (double)z;
                if (qq < 0.0) qq = 0.0;
                if (qq > 15.0) qq = 15.0;
            }
            q[r * I + j] = (uint8_t)qq;
        }
}

/* rows of one matrix share g; mat_rows = O (rows per matrix). */
ORC_API void orc_rtn_nvfp4(const float* W, int64_t rows, int64_t mat_rows, int64_t I,
                           const uint8_t* scale_codes, const float* gscale, uint8_t* c)
{
    const int64_t G = (I + 15) / 16;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float g = gscale[r / mat_rows];
        for (int64_t j = 0; j < I; ++j) {
            int sc = scale_codes[r * G + j / 16];
            float S = (float)((double)g * orc_e4m3_decode(sc));
            float w = W[r * I + j];
            int mag = (S == 0.0f) ? 0 : orc_e2m1_rne_mag(fabsf(w) / S);
            c[r * I + j] = (uint8_t)((mag != 0 && w < 0.0f) ? (mag | 8) : mag);
        }
    }
}

/* NVFP4 activations for a W4A4 product ([NVFP4] recipe table: the routed
 * experts run W4A4 with 16-element groups; the card gives no activation
 * recipe, so the reading is the weights' one without the search): per
 * tensor g = fl32(amax / 2688); per 16-element block of a row (amax b) the
 * positive finite E4M3 code nearest b / (6 g), ties to the lower code (the
 * first code of orc_nvfp4_window; 0 when b or g is 0); the elements' E2M1
 * codes by orc_rtn_nvfp4's rule.  scale_codes: [rows][ceil(I/16)], codes:
 * [rows][I] (sign in bit 3). */
ORC_API void orc_nvfp4_quant_act(const float* X, int64_t rows, int64_t I, float* g_out, uint8_t* scale_codes,
                                 uint8_t* codes)
{
    const int64_t G = (I + 15) / 16;
    const float g = orc_nvfp4_global(X, rows * I);
    *g_out = g;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < G; ++k) {
            float b = 0.0f;
            for (int64_t j = 16 * k; j < I && j < 16 * k + 16; ++j) {
                float a = fabsf(X[r * I + j]);
                if (a > b) b = a;
            }
            int code = 0;
            if (g > 0.0f && b > 0.0f) orc_nvfp4_window(b, g, 1, &code);
            scale_codes[r * G + k] = (uint8_t)code;
        }
    orc_rtn_nvfp4(X, rows, rows, I, scale_codes, &g, codes);
}

/* W4A4 product of NVFP4 weights and NVFP4 activations (the consumer of the
 * packed experts on a block-scaled tensor core):
 *   y[b][o] = gw gx sum_k dec(ew[o][k]) dec(ex[b][k]) sum_{j in block k} dec(cw[o][j]) dec(cx[b][j]),
 * the exact value of the block-scaled representation (reading: the global
 * scales multiply once, the E4M3 block scales per block, no rounding of the
 * dequantized elements); fp64, each block's sum of E2M1 products exact. */
ORC_API void orc_gemm_nvfp4(const uint8_t* cw, const uint8_t* ew, float gw, int64_t O, const uint8_t* cx,
                            const uint8_t* ex, float gx, int64_t B, int64_t I, double* y)
{
    const int64_t G = (I + 15) / 16;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t o = 0; o < O; ++o) {
            double acc = 0.0;
            for (int64_t k = 0; k < G; ++k) {
                double p = 0.0;
                for (int64_t j = 16 * k; j < I && j < 16 * k + 16; ++j) {
                    const int u = cw[o * I + j], v = cx[b * I + j];
                    const double dw = (u & 8) ? -E2M1_MAG[u & 7] : E2M1_MAG[u & 7];
                    const double dx = (v & 8) ? -E2M1_MAG[v & 7] : E2M1_MAG[v & 7];
                    p += dw * dx;
                }
                acc += orc_e4m3_decode(ew[o * G + k]) * orc_e4m3_decode(ex[b * G + k]) * p;
            }
            y[b * O + o] = (double)gw * (double)gx * acc;
        }
}

/* ------------------------------------------------------------------ */
/* Packing ([INT3] Design: Layout; nibble order for int4 / NVFP4)      */
/* ------------------------------------------------------------------ */

/* int3-g64: per group a 24-byte record.  u_i = v_i + 4.  Bytes 0..15: low
 * plane, element i in byte i/4 at bits 2(i%4).  Bytes 16..23: high plane,
 * element i at bit i%8 of byte 16 + i/8.  Records in [row][group] order; tail
 * positions past I hold v = 0 (u = 4). */
ORC_API void orc_pack_int3(const int8_t* v, int64_t rows, int64_t I, uint8_t* out)
{
    const int64_t G = (I + 63) / 64;
    memset(out, 0, (size_t)(rows * G * 24));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < G; ++k) {
            uint8_t* rec = out + (r * G + k) * 24;
            for (int i = 0; i < 64; ++i) {
                int64_t j = k * 64 + i;
                int u = (j < I ? v[r * I + j] : 0) + 4;
                rec[i / 4] |= (uint8_t)((u & 3) << (2 * (i % 4)));
                rec[16 + i / 8] |= (uint8_t)(((u >> 2) & 1) << (i % 8));
            }
        }
}

ORC_API void orc_unpack_int3(const uint8_t* in, int64_t rows, int64_t I, int8_t* v)
{
    const int64_t G = (I + 63) / 64;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            const uint8_t* rec = in + (r * G + j / 64) * 24;
            int i = (int)(j % 64);
            int lo = (rec[i / 4] >> (2 * (i % 4))) & 3;
            int hi = (rec[16 + i / 8] >> (i % 8)) & 1;
            v[r * I + j] = (int8_t)((lo | (hi << 2)) - 4);
        }
}

/* Nibble pack: group of `g` codes in g/2 bytes, element 2k in the low
 * nibble of byte k, element 2k+1 in the high nibble.  Tail positions hold
 * `pad` (per group: the zero-point for int4 so they dequantize to 0; 0 for
 * NVFP4). */
ORC_API void orc_pack_nibbles(const uint8_t* c, int64_t rows, int64_t I, int g,
                              const uint8_t* pad_per_group, uint8_t* out)
{
    const int64_t G = (I + g - 1) / g;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < G; ++k) {
            uint8_t pad = pad_per_group ? pad_per_group[r * G + k] : 0;
            uint8_t* rec = out + (r * G + k) * (g / 2);
            for (int i = 0; i < g / 2; ++i) {
                int64_t j0 = k * g + 2 * i, j1 = j0 + 1;
                int lo = (j0 < I ? c[r * I + j0] : pad) & 15;
                int hi = (j1 < I ? c[r * I + j1] : pad) & 15;
                rec[i] = (uint8_t)(lo | (hi << 4));
            }
        }
}

ORC_API void orc_unpack_nibbles(const uint8_t* in, int64_t rows, int64_t I, int g, uint8_t* c)
{
    const int64_t G = (I + g - 1) / g;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            uint8_t b = in[(r * G + j / g) * (g / 2) + (j % g) / 2];
            c[r * I + j] = (uint8_t)((j % 2) ? (b >> 4) : (b & 15));
        }
}

/* ------------------------------------------------------------------ */
/* Dequantization (fp32 semantics, rounded once)                       */
/* ------------------------------------------------------------------ */

ORC_API void orc_dequant_int3(const int8_t* v, int64_t rows, int64_t I, const float* scales, float* out)
{
    const int64_t G = (I + 63) / 64;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j)
            out[r * I + j] = (float)((double)scales[r * G + j / 64] * (double)v[r * I + j]);
}

ORC_API void orc_dequant_int4(const uint8_t* q, int64_t rows, int64_t I, const float* scales,
                              const uint8_t* zeros, float* out, int g)
{
    const int64_t G = (I + g - 1) / g;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            int64_t gi = r * G + j / g;
            out[r * I + j] = (float)((double)scales[gi] * ((double)q[r * I + j] - (double)zeros[gi]));
        }
}

/* GPTQ/LDLQ column sweep ([TT] pipeline table, step 3: the columns are
 * rounded one after another and each one's rounding error is carried to the
 * later columns through the inverse Hessian's triangular factor), with the group scales
 * (and zero-points) fixed by the search.  U: upper triangular, H^-1 = U^T U
 * (fp32, I x I rows of ldu; only the upper triangle is read; U_ii > 0).  Per
 * row, for each column i in order:
 *   code of the current w_i under its group's scale (the format's RTN:
 *   rtn_code, or the int4 zero-point form of orc_rtn_int4), dequantized
 *   value what_i = fl32(s v) / fl32(s (q - z)),
 *   e_i = (w_i - what_i) / U_ii in fp32,
 *   w_j <- w_j - e_i U_ij for every later column j, one fused multiply-add
 *   (fmaf) each.
 * Precision (reading): fp32, the page's host propagator ("cpu-float32").
 * The page's 128-column blocks and its propagation matmul
 * W[:, rest] -= E U[blk, rest] reorder nothing when every weight's updates
 * are applied in column order, as here.  loss[r] = sum_i e_i^2 in fp64,
 * which in exact arithmetic is (w - What) H (w - What)^T for the row.
 * fmt: 3 = int3 (codes v in [-4, 3], g = 64), 4 = int4 (codes q in [0, 15],
 * zeros per group, g = 128 or 64).  codes: int8 [rows][I]. */
ORC_API void orc_gptq_sweep(const float* W, int64_t rows, int64_t I, int fmt, int g, const float* scales,
                            const uint8_t* zeros, const float* U, int64_t ldu, int8_t* codes, double* loss)
{
    const int64_t G = (I + g - 1) / g;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        float* w = (float*)malloc((size_t)I * sizeof(float));
        memcpy(w, W + r * I, (size_t)I * sizeof(float));
        double L = 0.0;
        for (int64_t i = 0; i < I; ++i) {
            const float s = scales[r * G + i / g];
            double code;
            float what;
            if (fmt == 3) {
                code = rtn_code(w[i], s, -4.0, 3.0);
                what = (float)((double)s * code);
            } else {
                const int z = zeros[r * G + i / g];
                if (s == 0.0f) code = (double)z;
                else {
                    code = nearbyint((double)(w[i] / s)) + (double)z;
                    if (code < 0.0) code = 0.0;
                    if (code > 15.0) code = 15.0;
                }
                what = (float)((double)s * (code - (double)z));
            }
            codes[r * I + i] = (int8_t)code;
            const float e = (w[i] - what) / U[i * ldu + i];
            L += (double)e * (double)e;
            for (int64_t j = i + 1; j < I; ++j) w[j] = fmaf(-e, U[i * ldu + j], w[j]);
        }
        loss[r] = L;
        free(w);
    }
}

ORC_API void orc_dequant_nvfp4(const uint8_t* c, int64_t rows, int64_t mat_rows, int64_t I,
                               const uint8_t* scale_codes, const float* gscale, float* out)
{
    const int64_t G = (I + 15) / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < I; ++j) {
            float S = (float)((double)gscale[r / mat_rows] * orc_e4m3_decode(scale_codes[r * G + j / 16]));
            int code = c[r * I + j];
            double v = E2M1_MAG[code & 7] * ((code & 8) ? -1.0 : 1.0);
            out[r * I + j] = (float)((double)S * v);
        }
}

/* ------------------------------------------------------------------ */
/* Weighted reconstruction error ([TT] Risks to measure: Precision)    */
/* ------------------------------------------------------------------ */

/* num = sum_{o,j} m_j (W - What)^2 = tr(E H E^T), den = sum m_j W^2 =
 * tr(W H W^T) with H = diag(m), over one O x I matrix (row stride I). */
ORC_API void orc_proxy_error(const float* W, const float* What, int64_t O, int64_t I,
                             const float* m, double* num, double* den)
{
    double a = 0.0, b = 0.0;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t j = 0; j < I; ++j) {
            double w = (double)W[o * I + j];
            double e = w - (double)What[o * I + j];
            a += (double)m[j] * (e * e);
            b += (double)m[j] * (w * w);
        }
    *num = a; *den = b;
}

/* Per-row int4 absmax baseline of [INT3] Tests (the shipped per-row format
 * the outlier-row RMS test compares against): s = max|w_row| / 7,
 * q = clamp(rint(w/s), -8, 7), What = fl32(s q). */
ORC_API void orc_rowwise_int4(const float* W, int64_t rows, int64_t I, float* What)
{
    for (int64_t r = 0; r < rows; ++r) {
        float M = 0.0f;
        for (int64_t j = 0; j < I; ++j) { float a = fabsf(W[r * I + j]); if (a > M) M = a; }
        float s = (float)((double)M / 7.0);
        for (int64_t j = 0; j < I; ++j) {
            double q = rtn_code(W[r * I + j], s, -8.0, 7.0);
            What[r * I + j] = (float)((double)s * q);
        }
    }
}

ORC_API int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
