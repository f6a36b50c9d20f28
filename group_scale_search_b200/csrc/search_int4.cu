// Asymmetric int4-g128 joint (scale, integer zero-point) search with fused
// RTN + nibble pack.
//
// Method ("NeUQI Accuracy Validation", opening paragraph and results bullet 2:
// asymmetric layers run a joint (scale, integer zero-point) search weighted by
// the activation imatrix, on a "64/32" grid):
//   s_k = fl32(c_k R), c_k = fl32(f_k / 15), f_k evenly over [lo, hi], R = wmax - wmin;
//   z_i = rint(15 i / (nz - 1)); q = clamp(rint(w/s) + z, 0, 15);
//   L = sum_j m_j (w_j - s (q_j - z))^2; ties keep the lowest index nz k + i.
//
// The same search runs on 64-weight groups (int4-g64: the page "int3-g64
// (fmt=5)"'s per-projection ablation table lists an int4-g64 scheme, and its
// thread the grouped int4 format fmt=4): lanes then hold 2 weights each; and
// on 32-weight groups ("Phase 2: math-accuracy regression on tq3a-tq2e g32",
// Summary: group_size=32), one weight per lane.
//
// B200 mapping: one warp per 128-weight group; lane l owns scales l and l+32
// (and 64 p + l, 64 p + 32 + l in pass p of a grid of more than 64 scales:
// the "256/64" end of the page's quality ladder, results bullet 2) and all 16
// distinct zero-points.  The group's weights (and sqrt of their
// imatrix weights) are staged in shared memory and broadcast to all lanes, so
// the 1024 candidates reuse one HBM read.  Zero-points repeated in the
// 32-point list never win under the lowest-index rule, so only the first
// occurrence of each is evaluated.
//
// Per candidate-element the clamp is one min or max: with s > 0 the code
// r = rint(w/s) has the sign of w, so a negative weight can only be clamped
// at the low end (code -z) and a non-negative one only at the high end (code
// 15 - z).  With u = w - s r the unclamped error the clamped error is
// u + s d(z), d(z) = min(r + z, 0) for w < 0 and max(r - 15 + z, 0) for
// w >= 0.  Elements are split by sign once per group (uniform branches), every
// error carries a factor sqrt(m) so the weighted square is one FMA, and
// Blackwell's packed fp32x2 add/FMA evaluate two zero-points per instruction:
// per pair of candidate-elements FADD2 (excess), two FMNMX, FFMA2 (error),
// FFMA2 (accumulate).  Each error is formed by one FMA from exact products,
// so every term keeps a few ulp of relative accuracy.  Near ties (relative
// 2^-15) are re-ranked in fp64 with codes from the IEEE quotient, exactly as
// the definition ranks them.
#include "group_pack.cuh"

#include <climits>

namespace tq {

// Warps per block: one block per SM, as many warps as the registers allow
// (g128: 96 registers, g64: 80, g32: 72 per thread).  Measured on the dense
// int4-g128 workloads: one 640-thread block per SM beat five 128-thread
// blocks (2.12 against 2.22 ms on 4096 x 4096, 3.29 against 3.45 ms on the
// dense model's first linear).
template <int GS>
__host__ __device__ constexpr int asym_warps() { return GS == 128 ? 20 : (GS == 64 ? 24 : 28); }
constexpr float AWIN = 3.0517578125e-05f;   // 2^-15: bound on fp32 ranking error x 2 (with margin)

struct AsymArgs {
    const void* W;
    int64_t n_mat, O, I, ld, ms;
    const float* m;
    int64_t m_stride;
    float* scales;
    uint8_t* zeros;
    int32_t* idx;
    double* loss;
    uint8_t* packed;
    GroupIndex gi;
    int ns, nz;
    int zfirst[16];      // lowest i with z_i = z
    int8_t zval[64];     // z_i for i < nz (nz <= 64)
    float c[256];        // fl32(f_k / 15), k < ns <= 256
};

// Lane l holds elements 4l..4l+3 of the group.
template <typename T> struct Load4;
template <> struct Load4<uint16_t> {
    static __device__ __forceinline__ void go(const uint16_t* p, float w[4]) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
        w[0] = __uint_as_float(v.x << 16); w[1] = __uint_as_float(v.x & 0xffff0000u);
        w[2] = __uint_as_float(v.y << 16); w[3] = __uint_as_float(v.y & 0xffff0000u);
    }
};
template <> struct Load4<float> {
    static __device__ __forceinline__ void go(const float* p, float w[4]) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(p));
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    }
};

// Lane l holds elements 2l, 2l+1 of a 64-weight group.
template <typename T> struct Load2;
template <> struct Load2<uint16_t> {
    static __device__ __forceinline__ void go(const uint16_t* p, float w[2]) {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(p));
        w[0] = __uint_as_float(v << 16); w[1] = __uint_as_float(v & 0xffff0000u);
    }
};
template <> struct Load2<float> {
    static __device__ __forceinline__ void go(const float* p, float w[2]) {
        const float2 v = __ldg(reinterpret_cast<const float2*>(p));
        w[0] = v.x; w[1] = v.y;
    }
};

// Lane l holds element l of a 32-weight group.
template <typename T> struct Load1;
template <> struct Load1<uint16_t> {
    static __device__ __forceinline__ void go(const uint16_t* p, float w[1]) { w[0] = bf16_bits_to_f32(__ldg(p)); }
};
template <> struct Load1<float> {
    static __device__ __forceinline__ void go(const float* p, float w[1]) { w[0] = __ldg(p); }
};

__device__ __forceinline__ unsigned ord_key(float x) {   // order-preserving float -> uint
    const unsigned b = __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_val(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <int EPL>
__device__ __forceinline__ double loss64_int4(const float w[EPL], const float m[EPL], float s, int z) {
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const float q = (s == 0.f) ? static_cast<float>(z)
                                   : fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w[i], s)), static_cast<float>(z)), 0.f), 15.f);
        const double e = __dsub_rn(static_cast<double>(w[i]),
                                   __dmul_rn(static_cast<double>(s), static_cast<double>(q) - static_cast<double>(z)));
        t = __dadd_rn(t, __dmul_rn(static_cast<double>(m[i]), __dmul_rn(e, e)));
    }
    return group_sum_d(t, FULL, 32);
}

// Accumulates, for the 16 zero-points of one scale, m e(z)^2 of one element
// (pairs z = 2p, 2p + 1 packed in float2).  With u = w - s r the unclamped
// error and d(z) the integer clamp excess -- max(r - 15 + z, 0) for w >= 0,
// min(r + z, 0) for w < 0 -- the error is e = u + s d.  Every quantity carries
// sqrt(m): u' = sqrt(m) u, q = sqrt(m) s, e' = fma(q, d, u') (exact product,
// one rounding, no cancellation), and the weighted square is fma(e', e', acc).
template <bool POS>
__device__ __forceinline__ void acc_scale(float w, float sm, float s, float inv, float2 (&acc)[8]) {
    const float r = __fsub_rn(__fmaf_rn(w, inv, MAGIC), MAGIC);         // rint(w/s)
    const float u = __fmul_rn(sm, __fmaf_rn(-s, r, w));                  // sqrt(m) (w - s r)
    const float q = __fmul_rn(sm, s);                                   // sqrt(m) s
    const float rb = POS ? __fsub_rn(r, 15.f) : r;                      // d(z) = clamp excess of rb + z
    const float2 qq = make_float2(q, q), uu = make_float2(u, u), rr = make_float2(rb, rb);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        const float2 t = __fadd2_rn(rr, make_float2(static_cast<float>(2 * p), static_cast<float>(2 * p + 1)));
        float2 d;
        if (POS) { d.x = fmaxf(t.x, 0.f); d.y = fmaxf(t.y, 0.f); }
        else     { d.x = fminf(t.x, 0.f); d.y = fminf(t.y, 0.f); }
        const float2 e = __ffma2_rn(qq, d, uu);
        acc[p] = __ffma2_rn(e, e, acc[p]);
    }
}

template <typename T, int NP, int GS>
__global__ void __launch_bounds__(asym_warps<GS>() * 32)
k_search_int4(const __grid_constant__ AsymArgs a) {
    constexpr int EPL = GS / 32;   // elements per lane: 4 (g128), 2 (g64) or 1 (g32)
    constexpr int ASYM_WARPS = asym_warps<GS>();
    __shared__ __align__(16) float2 lists[ASYM_WARPS][GS + 4];   // two sign lists, each padded to even length
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t G = (a.I + GS - 1) / GS;
    const int64_t OG = a.O * G;
    const int64_t total = a.n_mat * OG;
    const T* W = static_cast<const T*>(a.W);
    float2* list = lists[wid];
    const float4* list4 = reinterpret_cast<const float4*>(list);

    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * ASYM_WARPS + wid; gid < total;
         gid += static_cast<int64_t>(gridDim.x) * ASYM_WARPS) {
        uint32_t e32, o32, k32;
        a.gi.split(static_cast<uint32_t>(gid), e32, o32, k32);
        const int64_t e = e32, o = o32, k = k32;
        const int64_t j0 = k * GS;
        const int n = static_cast<int>(min(static_cast<int64_t>(GS), a.I - j0));
        const T* wp = W + e * a.ms + o * a.ld + j0;
        const float* mp = a.m + e * a.m_stride + j0;
        float w[EPL], mv[EPL];
        bool val[EPL];
        if (n == GS) {
            if constexpr (EPL == 4) {
                Load4<T>::go(wp + 4 * lane, w);
                const float4 mm = __ldg(reinterpret_cast<const float4*>(mp + 4 * lane));
                mv[0] = mm.x; mv[1] = mm.y; mv[2] = mm.z; mv[3] = mm.w;
            } else if constexpr (EPL == 2) {
                Load2<T>::go(wp + 2 * lane, w);
                const float2 mm = __ldg(reinterpret_cast<const float2*>(mp + 2 * lane));
                mv[0] = mm.x; mv[1] = mm.y;
            } else {
                Load1<T>::go(wp + lane, w);
                mv[0] = __ldg(mp + lane);
            }
#pragma unroll
            for (int i = 0; i < EPL; ++i) val[i] = true;
        } else {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int j = EPL * lane + i;
                val[i] = j < n;
                w[i] = val[i] ? Elem<T>::load(wp + j) : 0.f;
                mv[i] = val[i] ? __ldg(mp + j) : 0.f;
            }
        }
        unsigned kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (val[i]) { kmin = min(kmin, ord_key(w[i])); kmax = max(kmax, ord_key(w[i])); }
        const float wmin = ord_val(__reduce_min_sync(FULL, kmin));
        const float wmax = ord_val(__reduce_max_sync(FULL, kmax));
        float R = __fsub_rn(wmax, wmin);
        uint8_t* rec = a.packed ? a.packed + gid * (GS / 2) : nullptr;
        if (R == 0.f) {
            if (wmax == 0.f) {   // all-zero group: s = 0, z = 0, q = 0
                if (lane == 0) {
                    a.scales[gid] = 0.f; a.zeros[gid] = 0;
                    if (a.idx) a.idx[gid] = -1;
                    if (a.loss) a.loss[gid] = 0.0;
                }
                if (rec) { const unsigned q0[EPL] = {}; pack_int4_lane<EPL>(q0, lane, rec); }
                continue;
            }
            R = fabsf(wmax);
        }

        // fp32 ranking works on w, m scaled by exact powers of two
        const float pw = pow2_inv_binade(fmaxf(fabsf(wmin), fabsf(wmax)));
        float mloc = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) mloc = fmaxf(mloc, fabsf(mv[i]));
        const float mmax = __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(mloc)));
        const float pm = mmax > 0.f ? pow2_inv_binade(mmax) : 1.f;
        const double back = inv_pow2_sq(pw, pm);
        const float Rs = __fmul_rn(R, pw);
        // split by sign: negative weights first, non-negative after (tail: (0, 0))
        float x[EPL], sq[EPL];
        bool neg[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            x[i] = __fmul_rn(w[i], pw);
            sq[i] = sqrtf(__fmul_rn(mv[i], pm));
            neg[i] = val[i] && x[i] < 0.f;
        }
        unsigned bn[EPL];
        int nneg = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) { bn[i] = __ballot_sync(FULL, neg[i]); nneg += __popc(bn[i]); }
        const int npos_real = n - nneg;
        const int nneg_pad = (nneg + 1) & ~1;
        const int npos_pad = (npos_real + 1) & ~1;
        __syncwarp();
        {
            int before_n = 0, before_p = 0;
            const unsigned lt = (1u << lane) - 1u;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const unsigned bp = __ballot_sync(FULL, val[i] && !neg[i]);
                if (neg[i]) list[before_n + __popc(bn[i] & lt)] = make_float2(x[i], sq[i]);
                else if (val[i]) list[nneg_pad + before_p + __popc(bp & lt)] = make_float2(x[i], sq[i]);
                before_n += __popc(bn[i]);
                before_p += __popc(bp);
            }
            if (lane == 0 && nneg_pad > nneg) list[nneg] = make_float2(0.f, 0.f);
            if (lane == 0 && npos_pad > npos_real) list[nneg_pad + npos_real] = make_float2(0.f, 0.f);
        }
        __syncwarp();

        // NP passes of 64 scales: lane l takes scales 64 p + l (A) and 64 p + 32 + l (B).
        // A pass flags its candidates within the window of the running minimum; the
        // minimum only falls, so the flags are a superset of the final window.
        float L = __int_as_float(0x7f800000);
        int bi = INT_MAX;
        unsigned wm[NP];
#pragma unroll
        for (int ps = 0; ps < NP; ++ps) {
            const int kA = 64 * ps + lane, kB = kA + 32;
            const bool actA = kA < a.ns, actB = kB < a.ns;
            if (NP > 1 && !__any_sync(FULL, actA)) {   // passes past ns
                wm[ps] = 0u;
                continue;
            }
            const float cA = a.c[actA ? kA : 0], cB = a.c[actB ? kB : 0];
            const float sA = __fmul_rn(cA, Rs), sB = __fmul_rn(cB, Rs);
            const float iA = rcp_approx(sA), iB = rcp_approx(sB);
            float2 a2[8], b2[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) { a2[p] = make_float2(0.f, 0.f); b2[p] = make_float2(0.f, 0.f); }
            for (int j = 0; j < (nneg_pad >> 1); ++j) {
                const float4 p = list4[j];
                acc_scale<false>(p.x, p.y, sA, iA, a2);
                acc_scale<false>(p.x, p.y, sB, iB, b2);
                acc_scale<false>(p.z, p.w, sA, iA, a2);
                acc_scale<false>(p.z, p.w, sB, iB, b2);
            }
            for (int j = nneg_pad >> 1; j < ((nneg_pad + npos_pad) >> 1); ++j) {
                const float4 p = list4[j];
                acc_scale<true>(p.x, p.y, sA, iA, a2);
                acc_scale<true>(p.x, p.y, sB, iB, b2);
                acc_scale<true>(p.z, p.w, sA, iA, a2);
                acc_scale<true>(p.z, p.w, sB, iB, b2);
            }
            float accA[16], accB[16];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                accA[2 * p] = a2[p].x; accA[2 * p + 1] = a2[p].y;
                accB[2 * p] = b2[p].x; accB[2 * p + 1] = b2[p].y;
            }

            // lane-local argmin in index order (all of scale A precede scale B)
            float Lp = __int_as_float(0x7f800000);
            int bp = INT_MAX;
            if (actA) {
#pragma unroll
                for (int z = 0; z < 16; ++z)
                    if (accA[z] < Lp) { Lp = accA[z]; bp = a.nz * kA + a.zfirst[z]; }
            }
            if (actB) {
#pragma unroll
                for (int z = 0; z < 16; ++z)
                    if (accB[z] < Lp) { Lp = accB[z]; bp = a.nz * kB + a.zfirst[z]; }
            }
            warp_argmin(Lp, bp);
            if (Lp < L) { L = Lp; bi = bp; }   // earlier passes hold lower indices: ties keep them
            const float thr = __fmaf_rn(L, AWIN, L);
            unsigned f = 0u;
#pragma unroll
            for (int z = 0; z < 16; ++z) {
                if (actA && accA[z] <= thr) f |= 1u << z;
                if (actB && accB[z] <= thr) f |= 1u << (16 + z);
            }
            wm[ps] = f;
        }
        int cnt = 0;
#pragma unroll
        for (int ps = 0; ps < NP; ++ps) cnt += __popc(wm[ps]);
        cnt = static_cast<int>(__reduce_add_sync(FULL, static_cast<unsigned>(cnt)));
        double lossd = static_cast<double>(L) * back;
        if (cnt > 1) {   // near tie: decide in fp64, candidates in index order
            double best = __longlong_as_double(0x7ff0000000000000ll);
            int bidx = bi;
#pragma unroll
            for (int ps = 0; ps < NP; ++ps) {
                for (int part = 0; part < 2; ++part) {
                    unsigned ls = __ballot_sync(FULL, part ? (wm[ps] >> 16) != 0u : (wm[ps] & 0xffffu) != 0u);
                    while (ls) {
                        const int l2 = __ffs(ls) - 1;
                        ls &= ls - 1;
                        unsigned zm = __shfl_sync(FULL, wm[ps], l2);
                        zm = part ? (zm >> 16) : (zm & 0xffffu);
                        const int k = 64 * ps + 32 * part + l2;
                        const float sc = __fmul_rn(a.c[k], R);
                        while (zm) {
                            const int z = __ffs(zm) - 1;
                            zm &= zm - 1;
                            const double Ld = loss64_int4<EPL>(w, mv, sc, z);
                            if (Ld < best) { best = Ld; bidx = a.nz * k + a.zfirst[z]; }
                        }
                    }
                }
            }
            bi = bidx;
            lossd = best;
        }

        if (bi < 0 || bi >= a.nz * a.ns) bi = a.zfirst[0];   // every loss non-finite
        const int kb = bi / a.nz;
        const int zb = a.zval[bi - kb * a.nz];
        const float sfin = __fmul_rn(a.c[kb], R);
        if (lane == 0) {
            a.scales[gid] = sfin;
            a.zeros[gid] = static_cast<uint8_t>(zb);
            if (a.idx) a.idx[gid] = bi;
            if (a.loss) a.loss[gid] = lossd;
        }
        if (rec) {
            unsigned q[EPL];
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const float qq = (sfin == 0.f || !val[i]) ? static_cast<float>(zb)
                    : fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w[i], sfin)), static_cast<float>(zb)), 0.f), 15.f);
                q[i] = static_cast<unsigned>(qq);
            }
            pack_int4_lane<EPL>(q, lane, rec);
        }
    }
}

template <int NP, int GS>
void launch_int4(const AsymArgs& a, bool bf16, int64_t total, cudaStream_t st) {
    int bpsm = 0;
    constexpr int ASYM_WARPS = asym_warps<GS>();
    if (bf16) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, k_search_int4<uint16_t, NP, GS>, ASYM_WARPS * 32, 0);
    else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, k_search_int4<float, NP, GS>, ASYM_WARPS * 32, 0);
    if (bpsm < 1) bpsm = 1;
    const int64_t need = (total + ASYM_WARPS - 1) / ASYM_WARPS;
    const int grid = static_cast<int>(min(need, static_cast<int64_t>(num_sms()) * bpsm));
    if (bf16) k_search_int4<uint16_t, NP, GS><<<grid, ASYM_WARPS * 32, 0, st>>>(a);
    else k_search_int4<float, NP, GS><<<grid, ASYM_WARPS * 32, 0, st>>>(a);
}

tq_status launch_search_int4(const tq_mat* W, int gsize, const float* m, int64_t m_stride,
                             const tq_search_params* p, float* scales, uint8_t* zeros, int32_t* idx,
                             double* loss, uint8_t* packed, cudaStream_t st) {
    if (p->asym_n_scale < 2 || p->asym_n_scale > 256)
        return set_error(TQ_ERR_UNSUPPORTED, "int4 search: asym_n_scale must be in [2, 256]");
    if (p->asym_n_zero < 16 || p->asym_n_zero > 64)
        return set_error(TQ_ERR_UNSUPPORTED, "int4 search: asym_n_zero must be in [16, 64]");
    if (!(p->asym_lo > 0.0) || !(p->asym_hi >= p->asym_lo))
        return set_error(TQ_ERR_INVALID_ARG, "int4 search: need 0 < asym_lo <= asym_hi");
    AsymArgs a;
    a.W = W->ptr; a.n_mat = W->n_mat; a.O = W->rows; a.I = W->cols; a.ld = W->ld;
    a.ms = W->n_mat > 1 ? W->mat_stride : 0;
    a.m = m; a.m_stride = m_stride;
    a.scales = scales; a.zeros = zeros; a.idx = idx; a.loss = loss; a.packed = packed;
    a.ns = p->asym_n_scale; a.nz = p->asym_n_zero;
    const double lo = p->asym_lo, hi = p->asym_hi;
    for (int k = 0; k < 256; ++k) {
        const double f = lo + ((hi - lo) * static_cast<double>(k)) / static_cast<double>(a.ns - 1);
        a.c[k] = k < a.ns ? static_cast<float>(f / 15.0) : 1.0f;
    }
    for (int z = 0; z < 16; ++z) a.zfirst[z] = -1;
    for (int i = 0; i < 64; ++i) {
        int z = 0;
        if (i < a.nz) {
            z = static_cast<int>(nearbyint((15.0 * static_cast<double>(i)) / static_cast<double>(a.nz - 1)));
            if (a.zfirst[z] < 0) a.zfirst[z] = i;
        }
        a.zval[i] = static_cast<int8_t>(z);
    }
    for (int z = 0; z < 16; ++z)
        if (a.zfirst[z] < 0) return set_error(TQ_ERR_UNSUPPORTED, "int4 search: zero-point %d not on the grid", z);

    const int64_t G = (W->cols + gsize - 1) / gsize;
    const int64_t total = W->n_mat * W->rows * G;
    if (total >= (int64_t(1) << 32)) return set_error(TQ_ERR_UNSUPPORTED, "int4 search: more than 2^32 groups");
    a.gi = GroupIndex(W->rows, G);
    const bool bf16 = W->dtype == TQ_BF16;
    if (gsize == 128) {
        if (a.ns <= 64) launch_int4<1, 128>(a, bf16, total, st);
        else launch_int4<4, 128>(a, bf16, total, st);
    } else if (gsize == 64) {
        if (a.ns <= 64) launch_int4<1, 64>(a, bf16, total, st);
        else launch_int4<4, 64>(a, bf16, total, st);
    } else {
        if (a.ns <= 64) launch_int4<1, 32>(a, bf16, total, st);
        else launch_int4<4, 32>(a, bf16, total, st);
    }
    return check_launch("int4 search");
}

}  // namespace tq
