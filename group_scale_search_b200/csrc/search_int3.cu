// Symmetric int3-g64 two-stage signed-scale search with fused RTN + pack.
//
// Method ("NeUQI Accuracy Validation", opening paragraph: symmetric layers run
// a two-stage signed scale search weighted by the activation imatrix):
//   stage 1: candidates s = +-fl32(r_k M)/4, r_k on an n1-point grid of
//            [lo, hi], M = max|w| of the group;
//   stage 2: n2 ratios spread over [r_k* - d, r_k* + d] with the stage-1 sign;
//   codes v = clamp(rint(w/s), -4, 3); loss L = sum_j m_j (w_j - s v_j)^2;
//   ties keep the lowest candidate index.
// Layout of the packed record: "int3-g64 (fmt=5)", Design: Layout.
//
// B200 mapping: one warp per 64-weight group, lane k = stage-1 magnitude k
// (both signs) and then stage-2 ratio k.  The group's (w, m) pairs sit in
// shared memory and are read with broadcast 16-byte loads, so every candidate
// reuses one HBM read of the group.  Elements are split once per group into
// "small" ones (|w| < 3.49 s_min: no candidate can clamp them) and the rest:
// for small elements the +s and -s candidates have identical errors (round
// half to even is odd-symmetric), so stage 1 evaluates them once per
// magnitude and only the few large elements per sign.  Candidates are ranked
// in fp32 with the multiply-by-reciprocal rounding; all candidates within a
// relative 2^-16 of the best are re-evaluated in fp64 with codes from the IEEE
// quotient, which decides the winner exactly as the definition does.
#include "group_pack.cuh"

#include <climits>

namespace tq {

constexpr int SYM_WARPS = 32;
// Ranking window.  A candidate's fp32 loss is within eps of its exact loss,
// relative: the reciprocal (one Newton step on rcp.approx) is within 2^-24 of
// 1/s, so a code differs from the IEEE quotient's only where y = w/s lies
// within |y| 2^-23 <= 4.5 2^-23 of a half-integer, which moves that element's
// term by at most 8 x 4.5 2^-23 = 2^-17.8 of itself; the fp32 sums (chains of
// at most 35 additions, 3 roundings per term) add at most 38 2^-24 = 2^-18.75.
// eps <= 2^-17.2, and a candidate the fp32 order could misplace is within
// (1 + eps) / (1 - eps) - 1 <= 2^-16.2 of the fp32 best: WIN = 2^-16 covers it.
constexpr float WIN = 1.52587890625e-05f;   // 2^-16

// 1/s to within 2^-24 (relative): rcp.approx refined by one Newton step.
__device__ __forceinline__ float rcp_refined(float s) {
    const float r = rcp_approx(s);
    return __fmaf_rn(r, __fmaf_rn(-s, r, 1.f), r);
}

struct SymArgs {
    const void* W;
    int64_t n_mat, O, I, ld, ms;
    const float* m;
    int64_t m_stride;
    float* scales;
    int32_t* idx;
    double* loss;
    uint8_t* packed;
    GroupIndex gi;
    int n1, n2;
    float r_lo;          // smallest ratio of either stage
    float r1[32];
    float r2[32 * 32];   // [k*][i]
};

// Two elements (w2, m2) under magnitude s, no clamp possible: the rounded
// quotient, the residual and the weighted square as packed fp32x2 ops.
__device__ __forceinline__ float2 err_free2(float2 w2, float2 m2, float2 ns2, float2 inv2, float2 acc) {
    const float2 t = __ffma2_rn(w2, inv2, make_float2(MAGIC, MAGIC));
    const float2 q = __fadd2_rn(t, make_float2(-MAGIC, -MAGIC));
    const float2 e = __ffma2_rn(ns2, q, w2);
    return __ffma2_rn(__fmul2_rn(m2, e), e, acc);
}

// Two elements under +s and -s: the rounded quotient is shared, only the
// clamp differs ([-4, 3] for +s, which is [-3, 4] in units of -s).
__device__ __forceinline__ void err_both2(float2 w2, float2 m2, float2 ns2, float2 inv2, float2& accP, float2& accN) {
    const float2 t = __ffma2_rn(w2, inv2, make_float2(MAGIC, MAGIC));
    float2 tp, tn;
    tp.x = fminf(fmaxf(t.x, MAGIC - 4.f), MAGIC + 3.f);
    tp.y = fminf(fmaxf(t.y, MAGIC - 4.f), MAGIC + 3.f);
    tn.x = fminf(fmaxf(t.x, MAGIC - 3.f), MAGIC + 4.f);
    tn.y = fminf(fmaxf(t.y, MAGIC - 3.f), MAGIC + 4.f);
    const float2 qp = __fadd2_rn(tp, make_float2(-MAGIC, -MAGIC));
    const float2 qn = __fadd2_rn(tn, make_float2(-MAGIC, -MAGIC));
    const float2 ep = __ffma2_rn(ns2, qp, w2);
    const float2 en = __ffma2_rn(ns2, qn, w2);
    accP = __ffma2_rn(__fmul2_rn(m2, ep), ep, accP);
    accN = __ffma2_rn(__fmul2_rn(m2, en), en, accN);
}

__device__ __forceinline__ float2 err_clamped2(float2 w2, float2 m2, float2 ns2, float2 inv2, float lo, float hi, float2 acc) {
    float2 t = __ffma2_rn(w2, inv2, make_float2(MAGIC, MAGIC));
    t.x = fminf(fmaxf(t.x, lo), hi);
    t.y = fminf(fmaxf(t.y, lo), hi);
    const float2 q = __fadd2_rn(t, make_float2(-MAGIC, -MAGIC));
    const float2 e = __ffma2_rn(ns2, q, w2);
    return __ffma2_rn(__fmul2_rn(m2, e), e, acc);
}

// fp64 loss of signed scale s over the warp's 64 elements (lane: l, l + 32),
// codes those of the IEEE quotient (rtn_fast: the reciprocal's rounding is
// redone with the IEEE division wherever it could differ).  Identical in
// every lane.
__device__ __forceinline__ double loss64_int3(float w0, float m0, float w1, float m1, float s) {
    const float inv = rcp_approx(s);
    const double v0 = rtn_fast(w0, s, inv, -4.f, 3.f), v1 = rtn_fast(w1, s, inv, -4.f, 3.f);
    const double e0 = __dsub_rn(static_cast<double>(w0), __dmul_rn(static_cast<double>(s), v0));
    const double e1 = __dsub_rn(static_cast<double>(w1), __dmul_rn(static_cast<double>(s), v1));
    const double t = __dadd_rn(__dmul_rn(static_cast<double>(m0), __dmul_rn(e0, e0)),
                               __dmul_rn(static_cast<double>(m1), __dmul_rn(e1, e1)));
    return group_sum_d(t, FULL, 32);
}

// Warp argmin of non-negative losses (NaN ranks as +inf) whose candidate
// indices grow with the lane: one min-reduction of the loss bits (non-negative
// floats order like their bit patterns) and a ballot for the lowest lane that
// holds it -- the lowest index on ties, as warp_argmin gives.
__device__ __forceinline__ void warp_argmin_by_lane(float& L, int& idx) {
    const unsigned key = L >= 0.f ? (__float_as_uint(L) & 0x7fffffffu) : 0x7f800000u;
    const unsigned kmin = __reduce_min_sync(FULL, key);
    const int src = __ffs(__ballot_sync(FULL, key == kmin)) - 1;
    L = __uint_as_float(kmin);
    idx = __shfl_sync(FULL, idx, src);
}

// The group's 64 weights (and imatrix weights) as lane l holds them:
// elements l and l + 32, zero past the group's n real elements.
template <typename T>
struct SymLoad {
    float w0, w1, m0, m1;
    int n;
    __device__ __forceinline__ void load(const SymArgs& a, const T* W, int64_t gid, int lane) {
        uint32_t e32, o32, k32;
        a.gi.split(static_cast<uint32_t>(gid), e32, o32, k32);
        const int64_t j0 = static_cast<int64_t>(k32) << 6;
        n = static_cast<int>(min(static_cast<int64_t>(64), a.I - j0));
        const T* wp = W + static_cast<int64_t>(e32) * a.ms + static_cast<int64_t>(o32) * a.ld + j0;
        const float* mp = a.m + static_cast<int64_t>(e32) * a.m_stride + j0;
        w0 = lane < n ? Elem<T>::load(wp + lane) : 0.f;
        w1 = lane + 32 < n ? Elem<T>::load(wp + lane + 32) : 0.f;
        m0 = lane < n ? __ldg(mp + lane) : 0.f;
        m1 = lane + 32 < n ? __ldg(mp + lane + 32) : 0.f;
    }
};

template <typename T>
__global__ void __launch_bounds__(SYM_WARPS * 32)
k_search_int3(const __grid_constant__ SymArgs a) {
    __shared__ float r2s[32 * 32];
    __shared__ __align__(16) float lists[SYM_WARPS][2][2][64];   // [warp][small|large][w|m][element]

    for (int i = threadIdx.x; i < 32 * 32; i += blockDim.x) r2s[i] = a.r2[i];
    __syncthreads();

    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t G = (a.I + 63) >> 6;
    const int64_t OG = a.O * G;
    const int64_t total = a.n_mat * OG;
    const bool act1 = lane < a.n1, act2 = lane < a.n2;
    const float r1v = a.r1[act1 ? lane : 0];
    float* smw = lists[wid][0][0];
    float* smm = lists[wid][0][1];
    float* lgw = lists[wid][1][0];
    float* lgm = lists[wid][1][1];
    const T* W = static_cast<const T*>(a.W);
    const unsigned lt = (1u << lane) - 1u;

    const int64_t gstride = static_cast<int64_t>(gridDim.x) * SYM_WARPS;
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * SYM_WARPS + wid; gid < total; gid += gstride) {
        SymLoad<T> cur;
        cur.load(a, W, gid, lane);
        const int n = cur.n;
        const bool v0 = lane < n, v1 = lane + 32 < n;
        const float w0 = cur.w0, w1 = cur.w1, m0 = cur.m0, m1 = cur.m1;
        const float M = warp_max_abs(w0, w1);
        uint8_t* rec = a.packed ? a.packed + gid * 24 : nullptr;

        if (M == 0.f) {   // nothing to fit: scale 0, codes 0
            if (lane == 0) {
                a.scales[gid] = 0.f;
                if (a.idx) a.idx[gid] = -1;
                if (a.loss) a.loss[gid] = 0.0;
            }
            if (rec) pack_int3_record(4u, 4u, lane, rec);
            continue;
        }

        // ---- fp32 ranking works on w, m scaled by exact powers of two
        const float pw = pow2_inv_binade(M);
        const float mmax = warp_max_abs(m0, m1);
        const float pm = mmax > 0.f ? pow2_inv_binade(mmax) : 1.f;
        const float Ms = __fmul_rn(M, pw);
        const float x0 = __fmul_rn(w0, pw), x1 = __fmul_rn(w1, pw);
        const float n0 = __fmul_rn(m0, pm), n1v = __fmul_rn(m1, pm);

        // ---- split elements: small ones cannot be clamped by any candidate
        const float s_lo = __fmul_rn(__fmul_rn(a.r_lo, Ms), 0.25f);
        const float thr = __fmul_rn(3.49f, s_lo);
        const bool sm0 = v0 && fabsf(x0) < thr, sm1 = v1 && fabsf(x1) < thr;
        const bool lg0 = v0 && !sm0, lg1 = v1 && !sm1;
        const unsigned bs0 = __ballot_sync(FULL, sm0), bs1 = __ballot_sync(FULL, sm1);
        const unsigned bl0 = __ballot_sync(FULL, lg0), bl1 = __ballot_sync(FULL, lg1);
        const int ns0 = __popc(bs0), ns = ns0 + __popc(bs1);
        const int nl0 = __popc(bl0), nl = nl0 + __popc(bl1);
        const int ns_pad = (ns + 3) & ~3, nl_pad = (nl + 1) & ~1;
        __syncwarp();   // previous group's readers are done with the lists
        if (sm0) { const int p = __popc(bs0 & lt); smw[p] = x0; smm[p] = n0; }
        if (sm1) { const int p = ns0 + __popc(bs1 & lt); smw[p] = x1; smm[p] = n1v; }
        if (lg0) { const int p = __popc(bl0 & lt); lgw[p] = x0; lgm[p] = n0; }
        if (lg1) { const int p = nl0 + __popc(bl1 & lt); lgw[p] = x1; lgm[p] = n1v; }
        if (lane < ns_pad - ns) { smw[ns + lane] = 0.f; smm[ns + lane] = 0.f; }   // zero pairs add exactly 0
        if (lane < nl_pad - nl) { lgw[nl + lane] = 0.f; lgm[nl + lane] = 0.f; }
        __syncwarp();
        const float4* spw = reinterpret_cast<const float4*>(smw);
        const float4* spm = reinterpret_cast<const float4*>(smm);

        // ---- stage 1: lane = magnitude, both signs
        const float s1 = __fmul_rn(__fmul_rn(r1v, Ms), 0.25f);    // scaled candidate
        const float s1o = __fmul_rn(__fmul_rn(r1v, M), 0.25f);    // the candidate itself
        const float i1 = rcp_refined(s1);
        const float2 ns1 = make_float2(-s1, -s1), inv1 = make_float2(i1, i1);
        float2 accC = make_float2(0.f, 0.f), accD = make_float2(0.f, 0.f);
        float2 accP = make_float2(0.f, 0.f), accN = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int j = 0; j < (ns_pad >> 2); ++j) {   // two independent accumulator chains
            const float4 w4 = spw[j], m4 = spm[j];
            accC = err_free2(make_float2(w4.x, w4.y), make_float2(m4.x, m4.y), ns1, inv1, accC);
            accD = err_free2(make_float2(w4.z, w4.w), make_float2(m4.z, m4.w), ns1, inv1, accD);
        }
        accC = __fadd2_rn(accC, accD);
        for (int j = 0; j < (nl_pad >> 1); ++j) {
            const float2 w2 = reinterpret_cast<const float2*>(lgw)[j], m2 = reinterpret_cast<const float2*>(lgm)[j];
            err_both2(w2, m2, ns1, inv1, accP, accN);
        }
        const float cC = __fadd_rn(accC.x, accC.y);
        const float LP = __fadd_rn(cC, __fadd_rn(accP.x, accP.y)), LN = __fadd_rn(cC, __fadd_rn(accN.x, accN.y));

        float L = __int_as_float(0x7f800000);
        int bi = INT_MAX;
        if (act1) {
            if (LN < LP) { L = LN; bi = 2 * lane + 1; } else { L = LP; bi = 2 * lane; }
        }
        warp_argmin_by_lane(L, bi);
        if (bi < 0 || bi >= 2 * a.n1) bi = 0;   // every loss non-finite: keep index 0
        int b1 = bi;
        bool have64 = false;
        double L1d = 0.0;
        {
            const float thr1 = __fmaf_rn(L, WIN, L);
            unsigned mpos = __ballot_sync(FULL, act1 && LP <= thr1);
            unsigned mneg = __ballot_sync(FULL, act1 && LN <= thr1);
            if (__popc(mpos) + __popc(mneg) > 1) {   // near tie: decide in fp64
                double best = __longlong_as_double(0x7ff0000000000000ll);
                int bidx = bi;
                while (mpos | mneg) {
                    const int kp = mpos ? __ffs(mpos) - 1 : 64, kn = mneg ? __ffs(mneg) - 1 : 64;
                    int kk, sg;
                    if (kp <= kn) { kk = kp; sg = 0; mpos &= mpos - 1; } else { kk = kn; sg = 1; mneg &= mneg - 1; }
                    const float sk = __shfl_sync(FULL, s1o, kk);
                    const double Ld = loss64_int3(w0, m0, w1, m1, sg ? -sk : sk);
                    if (Ld < best) { best = Ld; bidx = 2 * kk + sg; }
                }
                b1 = bidx; have64 = true; L1d = best;
            }
        }

        // ---- stage 2: lane = refinement i around magnitude k*, sign of the winner
        const int ks = b1 >> 1, sg = b1 & 1;
        const float r2v = r2s[ks * 32 + (act2 ? lane : 0)];
        const float s2 = __fmul_rn(__fmul_rn(r2v, Ms), 0.25f);
        const float s2o = __fmul_rn(__fmul_rn(r2v, M), 0.25f);
        const float i2 = rcp_refined(s2);
        const float clo = sg ? MAGIC - 3.f : MAGIC - 4.f, chi = sg ? MAGIC + 4.f : MAGIC + 3.f;
        const float2 ns2 = make_float2(-s2, -s2), inv2 = make_float2(i2, i2);
        float2 a2 = make_float2(0.f, 0.f), a2b = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int j = 0; j < (ns_pad >> 2); ++j) {
            const float4 w4 = spw[j], m4 = spm[j];
            a2 = err_free2(make_float2(w4.x, w4.y), make_float2(m4.x, m4.y), ns2, inv2, a2);
            a2b = err_free2(make_float2(w4.z, w4.w), make_float2(m4.z, m4.w), ns2, inv2, a2b);
        }
        a2 = __fadd2_rn(a2, a2b);
        for (int j = 0; j < (nl_pad >> 1); ++j) {
            const float2 w2 = reinterpret_cast<const float2*>(lgw)[j], m2 = reinterpret_cast<const float2*>(lgm)[j];
            a2 = err_clamped2(w2, m2, ns2, inv2, clo, chi, a2);
        }
        const float acc2 = __fadd_rn(a2.x, a2.y);
        const float L1f = __shfl_sync(FULL, sg ? LN : LP, ks);   // incumbent's fp32 loss
        const float L2 = act2 ? acc2 : __int_as_float(0x7f800000);
        float L2m = L2;
        int b2 = act2 ? 2 * a.n1 + lane : INT_MAX;
        warp_argmin_by_lane(L2m, b2);

        const float Lmin = fminf(L1f, L2m);
        const float thr2 = __fmaf_rn(Lmin, WIN, Lmin);
        const bool inc_in = L1f <= thr2;
        unsigned c2 = __ballot_sync(FULL, act2 && L2 <= thr2);
        int bf;
        double lossd;
        if (static_cast<int>(inc_in) + __popc(c2) > 1) {   // near tie: decide in fp64
            double best = __longlong_as_double(0x7ff0000000000000ll);
            int bidx = b2;
            if (inc_in) {
                if (!have64) {
                    const float sk = __shfl_sync(FULL, s1o, ks);
                    L1d = loss64_int3(w0, m0, w1, m1, sg ? -sk : sk);
                }
                best = L1d; bidx = b1;
            }
            while (c2) {
                const int i = __ffs(c2) - 1;
                c2 &= c2 - 1;
                const float si = __shfl_sync(FULL, s2o, i);
                const double Ld = loss64_int3(w0, m0, w1, m1, sg ? -si : si);
                if (Ld < best) { best = Ld; bidx = 2 * a.n1 + i; }
            }
            bf = bidx;
            lossd = best;
        } else if (L2m < L1f) {
            bf = b2; lossd = static_cast<double>(L2m) * inv_pow2_sq(pw, pm);
        } else {
            bf = b1; lossd = have64 ? L1d : static_cast<double>(L1f) * inv_pow2_sq(pw, pm);
        }

        if (bf < 0 || bf >= 2 * a.n1 + a.n2) bf = b1;
        float sfin;
        if (bf < 2 * a.n1) {
            const float sk = __shfl_sync(FULL, s1o, bf >> 1);
            sfin = (bf & 1) ? -sk : sk;
        } else {
            const float si = __shfl_sync(FULL, s2o, bf - 2 * a.n1);
            sfin = sg ? -si : si;
        }
        if (lane == 0) {
            a.scales[gid] = sfin;
            if (a.idx) a.idx[gid] = bf;
            if (a.loss) a.loss[gid] = lossd;
        }
        if (rec) {
            const float invf = rcp_approx(sfin);
            const unsigned u0 = static_cast<unsigned>(static_cast<int>(rtn_fast(w0, sfin, invf, -4.f, 3.f)) + 4);
            const unsigned u1 = static_cast<unsigned>(static_cast<int>(rtn_fast(w1, sfin, invf, -4.f, 3.f)) + 4);
            pack_int3_record(u0, u1, lane, rec);
        }
    }
}

// Host side: candidate ratio tables from their definitions (fp64, rounded
// once to fp32), then one persistent launch.
tq_status launch_search_int3(const tq_mat* W, const float* m, int64_t m_stride,
                             const tq_search_params* p, float* scales, int32_t* idx, double* loss,
                             uint8_t* packed, cudaStream_t st) {
    if (p->sym_n1 < 2 || p->sym_n1 > 32 || p->sym_n2 < 2 || p->sym_n2 > 32)
        return set_error(TQ_ERR_UNSUPPORTED, "int3 search: sym_n1 and sym_n2 must be in [2, 32]");
    if (!(p->sym_lo > 0.0) || !(p->sym_hi >= p->sym_lo))
        return set_error(TQ_ERR_INVALID_ARG, "int3 search: need 0 < sym_lo <= sym_hi");
    static thread_local SymArgs a;
    a.W = W->ptr; a.n_mat = W->n_mat; a.O = W->rows; a.I = W->cols; a.ld = W->ld;
    a.ms = W->n_mat > 1 ? W->mat_stride : 0;
    a.m = m; a.m_stride = m_stride;
    a.scales = scales; a.idx = idx; a.loss = loss; a.packed = packed;
    a.n1 = p->sym_n1; a.n2 = p->sym_n2;
    const double lo = p->sym_lo, hi = p->sym_hi;
    const double delta = (hi - lo) / static_cast<double>(a.n1 - 1);
    float rmin = 1e30f;
    for (int k = 0; k < 32; ++k) {
        a.r1[k] = k < a.n1 ? static_cast<float>(lo + ((hi - lo) * static_cast<double>(k)) / static_cast<double>(a.n1 - 1)) : 1.0f;
        if (k < a.n1) rmin = fminf(rmin, a.r1[k]);
    }
    for (int k = 0; k < 32; ++k) {
        const double center = lo + ((hi - lo) * static_cast<double>(k)) / static_cast<double>(a.n1 - 1);
        for (int i = 0; i < 32; ++i) {
            float r = 1.0f;
            if (k < a.n1 && i < a.n2)
                r = static_cast<float>((center - delta) + (2.0 * delta * static_cast<double>(i)) / static_cast<double>(a.n2 - 1));
            a.r2[k * 32 + i] = r;
            if (k < a.n1 && i < a.n2) rmin = fminf(rmin, r);
        }
    }
    if (!(rmin > 0.0f)) return set_error(TQ_ERR_INVALID_ARG, "int3 search: candidate ratios must be positive");
    a.r_lo = rmin;

    const int64_t G = (W->cols + 63) / 64;
    const int64_t total = W->n_mat * W->rows * G;
    if (total >= (int64_t(1) << 32)) return set_error(TQ_ERR_UNSUPPORTED, "int3 search: more than 2^32 groups");
    a.gi = GroupIndex(W->rows, G);
    int bpsm = 0;
    const bool bf16 = W->dtype == TQ_BF16;
    if (bf16) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, k_search_int3<uint16_t>, SYM_WARPS * 32, 0);
    else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, k_search_int3<float>, SYM_WARPS * 32, 0);
    if (bpsm < 1) bpsm = 1;
    const int64_t need = (total + SYM_WARPS - 1) / SYM_WARPS;
    const int grid = static_cast<int>(min(need, static_cast<int64_t>(num_sms()) * bpsm));
    if (bf16) k_search_int3<uint16_t><<<grid, SYM_WARPS * 32, 0, st>>>(a);
    else k_search_int3<float><<<grid, SYM_WARPS * 32, 0, st>>>(a);
    return check_launch("int3 search");
}

}  // namespace tq
