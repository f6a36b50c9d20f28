// NVFP4-g16 block-scale search (E2M1 elements, E4M3 block scale, fp32
// per-tensor global scale) with fused RTN + pack.
//
// Method ("Nemotron-Cascade-2-30B-A3B-NVFP4" model card, Quantization Recipe
// table: NVFP4, group size 16, MSE-calibrated static block scales; weight-MSE
// calibration), weighted by the imatrix like the integer formats:
//   g = fl32(amax / (6 * 448)) per tensor;
//   per 16-block with a = max|w|: the `window` E4M3 codes whose values are
//   nearest a / (6 g) (ties to the lower code), ranked by exact distance
//   |6 g dec(c) - a|; block scale S = fl32(g dec(e));
//   codes c = E2M1 round-to-nearest-even (saturating) of |w| / S, sign apart;
//   L = sum_j m_j (|w_j| - S dec(c_j))^2; ties keep the lower code.
//
// B200 mapping: one lane per 16-weight block.  A lane loads its block's
// weights (two 16-byte loads) and imatrix (four) into registers, finds the
// window start by a binary search of exact fp64 predicates, and loops over the
// window codes with the block in registers: per pair of candidate-elements one
// packed fp32x2 multiply, the hardware E2M1 conversion (round to nearest even,
// saturating) and back, and packed FMA/multiply/FMA for the weighted square.  Candidates whose fp32 loss is within a relative 2^-15 of the
// lane's best are queued; half-warps then re-rank each queued block in fp64
// with codes from the IEEE quotient (one lane per element), which decides the
// winner exactly as the definition does.  The winner's codes (E2M1 rounding
// of the IEEE quotient, nvfp4_rtn) are packed into the block's 8 bytes by
// the lane.
#include "group_pack.cuh"

#include <cuda_fp16.h>

#include <climits>

namespace tq {

// One block per SM with as many warps as the registers allow (80 per
// thread): measured 3.21 ms against 3.58 ms for six 128-thread blocks on the
// 128-expert NVFP4 stack.
constexpr int FP4_THREADS = 768;
constexpr int FP4_WARPS = FP4_THREADS / 32;
constexpr float FWIN = 3.0517578125e-05f;   // 2^-15
constexpr int FP4_DYN_SMEM = FP4_WARPS * 32 * (8 + 17 * 8 + 4);
// E4M3 values from a shared-memory table (true) or built from the code's
// bit fields in registers (false).
constexpr bool FP4_DEC_SMEM = true;

struct Fp4Args {
    const void* W;
    int64_t n_mat, O, I, ld, ms;
    const float* m;
    int64_t m_stride;
    const float* g;        // per-matrix global scale
    uint8_t* scales;
    int32_t* idx;
    double* loss;
    uint8_t* packed;
    GroupIndex gi;
    int window;
};

// Largest E4M3 code whose value does not exceed t (clamped to [1, 126]); only
// an estimate is needed (the exact window search brackets it).
__device__ __forceinline__ int e4m3_floor_code(float t) {
    if (!(t > 0.f)) return 1;
    if (t < 0.015625f) return max(1, static_cast<int>(t * 512.f));
    const unsigned b = __float_as_uint(t);
    const int E = static_cast<int>((b >> 23) & 255u) - 127;
    const int c = ((E + 7) << 3) | static_cast<int>((b >> 20) & 7u);
    return min(max(c, 1), 126);
}

__device__ __forceinline__ double half_sum_d(double v) {
#pragma unroll
    for (int off = 8; off; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(FULL, v, off));
    return v;
}

// E2M1 rounding of a pair with the hardware conversions (round to nearest
// even, saturating at 6): fp32x2 -> packed e2m1x2 -> f16x2 (exact) -> fp32x2.
// Ranking only; the exact codes come from e2m1_round on the IEEE quotient.
__device__ __forceinline__ float2 e2m1_round2_hw(float2 x) {
    unsigned h2;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %2, %1; cvt.rn.f16x2.e2m1x2 %0, t; }"
        : "=r"(h2) : "f"(x.x), "f"(x.y));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

template <typename T> struct Load16;
template <> struct Load16<uint16_t> {
    static __device__ __forceinline__ void go(const uint16_t* p, int n, float w[16]) {
        if (n == 16) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
            const unsigned u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                w[2 * i] = __uint_as_float(u[i] << 16);
                w[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = i < n ? bf16_bits_to_f32(__ldg(p + i)) : 0.f;
        }
    }
};
template <> struct Load16<float> {
    static __device__ __forceinline__ void go(const float* p, int n, float w[16]) {
        if (n == 16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(p) + i);
                w[4 * i] = a.x; w[4 * i + 1] = a.y; w[4 * i + 2] = a.z; w[4 * i + 3] = a.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = i < n ? __ldg(p + i) : 0.f;
        }
    }
};

template <typename T>
__global__ void __launch_bounds__(FP4_THREADS)
k_search_nvfp4(const __grid_constant__ Fp4Args a) {
    __shared__ float dec[128];   // E4M3 values (a table beats building them per lane)
    // dynamic: qres_l[FP4_WARPS][32] (re-ranked losses), qdat[FP4_WARPS][32][17]
    // (each lane's block (w, m), padded against bank conflicts), qres_c[FP4_WARPS][32]
    extern __shared__ double fp4_dyn[];
    double (*qres_l)[32] = reinterpret_cast<double (*)[32]>(fp4_dyn);
    float2 (*qdat)[32][17] = reinterpret_cast<float2 (*)[32][17]>(fp4_dyn + FP4_WARPS * 32);
    int (*qres_c)[32] = reinterpret_cast<int (*)[32]>(fp4_dyn + FP4_WARPS * 32 + FP4_WARPS * 32 * 17);
    for (int i = threadIdx.x; i < 128; i += blockDim.x) dec[i] = e4m3_value(i);
    __syncthreads();
    auto decv = [&](int c) { return FP4_DEC_SMEM ? dec[c] : e4m3_value(static_cast<unsigned>(c)); };
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int half = lane >> 4, hl = lane & 15;
    const int64_t G = (a.I + 15) >> 4;
    const int64_t total = a.n_mat * a.O * G;
    const int Wn = a.window;
    const int lo_max = 127 - Wn;   // window [lo, lo + Wn - 1] inside codes 1..126
    const T* W = static_cast<const T*>(a.W);

    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * FP4_WARPS + wid) * 32; base < total;
         base += static_cast<int64_t>(gridDim.x) * FP4_THREADS) {
        const int64_t bid = base + lane;
        const bool vb = bid < total;
        int64_t e = 0, j0 = 0;
        int n = 0;
        float w[16], mv[16];
        if (vb) {
            uint32_t e32, o32, k32;
            a.gi.split(static_cast<uint32_t>(bid), e32, o32, k32);
            e = e32;
            j0 = static_cast<int64_t>(k32) << 4;
            n = static_cast<int>(min(static_cast<int64_t>(16), a.I - j0));
            Load16<T>::go(W + e * a.ms + static_cast<int64_t>(o32) * a.ld + j0, n, w);
            const float* mp = a.m + e * a.m_stride + j0;
            if (n == 16) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 q = __ldg(reinterpret_cast<const float4*>(mp) + i);
                    mv[4 * i] = q.x; mv[4 * i + 1] = q.y; mv[4 * i + 2] = q.z; mv[4 * i + 3] = q.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) mv[i] = i < n ? __ldg(mp + i) : 0.f;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) { w[i] = 0.f; mv[i] = 0.f; }
        }
        float amax = 0.f, mmax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) { amax = fmaxf(amax, fabsf(w[i])); mmax = fmaxf(mmax, fabsf(mv[i])); }
        const float g = vb ? __ldg(a.g + e) : 0.f;
        const bool degen = (amax == 0.f) || (g == 0.f);
        __syncwarp();   // the previous iteration's readers are done with qdat
#pragma unroll
        for (int i = 0; i < 16; ++i) qdat[wid][lane][i] = make_float2(w[i], mv[i]);

        int lo = 1, cbest = 0;
        unsigned winmask = 0u;
        float Lbest = 0.f;
        double back = 1.0;
        if (!degen) {
            // ---- window start: first lo with d(lo) <= d(lo + Wn), d(c) = |6 g dec(c) - a| (exact in fp64)
            const double g6 = 6.0 * static_cast<double>(g), ad = static_cast<double>(amax);
            const int cdn = e4m3_floor_code(amax / fmaxf(6.f * g, 1e-30f));
            int lo_a = max(1, cdn - 17), hi_a = min(lo_max, cdn + 2);
            while (lo_a < hi_a) {
                const int mid = (lo_a + hi_a) >> 1;
                const bool p = fabs(__dsub_rn(__dmul_rn(g6, static_cast<double>(decv(mid))), ad)) >
                               fabs(__dsub_rn(__dmul_rn(g6, static_cast<double>(decv(mid + Wn))), ad));
                if (p) lo_a = mid + 1; else hi_a = mid;
            }
            lo = lo_a;
            // ---- fp32 ranking on |w|, m scaled by exact powers of two
            const float pw = pow2_inv_binade(amax);
            const float pm = mmax > 0.f ? pow2_inv_binade(mmax) : 1.f;
            back = inv_pow2_sq(pw, pm);
            float2 aw2[8], mm2[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                aw2[i] = make_float2(__fmul_rn(fabsf(w[2 * i]), pw), __fmul_rn(fabsf(w[2 * i + 1]), pw));
                mm2[i] = make_float2(__fmul_rn(mv[2 * i], pm), __fmul_rn(mv[2 * i + 1], pm));
            }
            float L[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int code = lo + (c < Wn ? c : 0);
                const float S = __fmul_rn(__fmul_rn(g, decv(code)), pw);
                const float inv = rcp_approx(S);
                const float2 S2 = make_float2(-S, -S), inv2 = make_float2(inv, inv);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 y = e2m1_round2_hw(__fmul2_rn(aw2[i], inv2));
                    const float2 er = __ffma2_rn(S2, y, aw2[i]);
                    acc = __ffma2_rn(__fmul2_rn(mm2[i], er), er, acc);
                }
                L[c] = c < Wn ? __fadd_rn(acc.x, acc.y) : __int_as_float(0x7f800000);
            }
            Lbest = L[0];
#pragma unroll
            for (int c = 1; c < 16; ++c)
                if (L[c] < Lbest) { Lbest = L[c]; cbest = c; }
            const float thr = __fmaf_rn(Lbest, FWIN, Lbest);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                if (L[c] <= thr) winmask |= 1u << c;
        }

        // ---- near ties: half-warps re-rank queued blocks in fp64, candidates in code order
        const bool need = __popc(winmask) > 1;
        unsigned queue = __ballot_sync(FULL, need);
        if (queue) {
            __syncwarp();
            while (queue) {
                const int own0 = __ffs(queue) - 1;
                queue &= queue - 1;
                const int own1 = queue ? __ffs(queue) - 1 : -1;
                if (own1 >= 0) queue &= queue - 1;
                const int own = half ? own1 : own0;
                const int src = own >= 0 ? own : own0;
                const unsigned omask = __shfl_sync(FULL, winmask, src);
                const int olo = __shfl_sync(FULL, lo, src);
                const float og = __shfl_sync(FULL, g, src);
                float2 d = qdat[wid][src][hl];
                d.x = fabsf(d.x);
                unsigned todo = own >= 0 ? omask : 0u;
                double best = __longlong_as_double(0x7ff0000000000000ll);
                int bc = 0;
                while (__any_sync(FULL, todo != 0u)) {
                    const int c = todo ? __ffs(todo) - 1 : 0;
                    const float Sc = __fmul_rn(og, e4m3_value(olo + c));
                    const float y = e2m1_round(__fdiv_rn(d.x, Sc));
                    const double er = __dsub_rn(static_cast<double>(d.x),
                                                __dmul_rn(static_cast<double>(Sc), static_cast<double>(y)));
                    const double Ld = half_sum_d(__dmul_rn(static_cast<double>(d.y), __dmul_rn(er, er)));
                    if (todo) {
                        if (Ld < best) { best = Ld; bc = c; }
                        todo &= todo - 1;
                    }
                }
                if (own >= 0 && hl == 0) { qres_c[wid][own] = bc; qres_l[wid][own] = best; }
            }
            __syncwarp();
        }

        double lossd;
        if (need) { cbest = qres_c[wid][lane]; lossd = qres_l[wid][lane]; }
        else lossd = static_cast<double>(Lbest) * back;

        // ---- outputs and exact RTN + pack of the lane's block
        if (vb) {
            const int code = lo + cbest;
            uint32_t wd0 = 0u, wd1 = 0u;
            if (!degen) {
                float wv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) wv[i] = qdat[wid][lane][i].x;
                uint32_t pk[2];
                nvfp4_rtn<16>(wv, __fmul_rn(g, e4m3_value(code)), pk);
                wd0 = pk[0];
                wd1 = pk[1];
            } else {
                lossd = 0.0;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 d = qdat[wid][lane][i];
                    const double wdv = static_cast<double>(d.x);
                    lossd = __dadd_rn(lossd, __dmul_rn(static_cast<double>(d.y), __dmul_rn(wdv, wdv)));
                }
            }
            a.scales[bid] = degen ? 0 : static_cast<uint8_t>(code);
            if (a.idx) a.idx[bid] = degen ? -1 : code;
            if (a.loss) a.loss[bid] = lossd;
            if (a.packed) *reinterpret_cast<uint2*>(a.packed + bid * 8) = make_uint2(wd0, wd1);
        }
    }
}

// amax -> g = fl32(amax / 2688), in place.
__global__ void k_global_from_amax(float* g, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) g[i] = __fdiv_rn(g[i], 2688.0f);
}

tq_status launch_amax(const tq_mat* W, float* amax, cudaStream_t st);   // imatrix.cu

tq_status launch_search_nvfp4(const tq_mat* W, const float* m, int64_t m_stride,
                              const tq_search_params* p, uint8_t* scales, float* gscale, int32_t* idx,
                              double* loss, uint8_t* packed, cudaStream_t st) {
    if (p->fp4_window < 1 || p->fp4_window > 16)
        return set_error(TQ_ERR_UNSUPPORTED, "nvfp4 search: fp4_window must be in [1, 16]");
    tq_status s = launch_amax(W, gscale, st);
    if (s != TQ_OK) return s;
    k_global_from_amax<<<static_cast<unsigned>((W->n_mat + 255) / 256), 256, 0, st>>>(gscale, W->n_mat);
    if ((s = check_launch("nvfp4 global scale")) != TQ_OK) return s;

    Fp4Args a;
    a.W = W->ptr; a.n_mat = W->n_mat; a.O = W->rows; a.I = W->cols; a.ld = W->ld;
    a.ms = W->n_mat > 1 ? W->mat_stride : 0;
    a.m = m; a.m_stride = m_stride; a.g = gscale;
    a.scales = scales; a.idx = idx; a.loss = loss; a.packed = packed;
    a.window = p->fp4_window;
    const int64_t G = (W->cols + 15) / 16;
    const int64_t total = W->n_mat * W->rows * G;
    if (total >= (int64_t(1) << 32)) return set_error(TQ_ERR_UNSUPPORTED, "nvfp4 search: more than 2^32 blocks");
    a.gi = GroupIndex(W->rows, G);
    int bpsm = 0;
    const bool bf16 = W->dtype == TQ_BF16;
    auto kern = bf16 ? reinterpret_cast<const void*>(k_search_nvfp4<uint16_t>)
                     : reinterpret_cast<const void*>(k_search_nvfp4<float>);
    if (FP4_DYN_SMEM > 48 * 1024) {   // above the default limit: opt in once per device
        static int opted[64][2] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= 64 || !opted[dev][bf16]) {
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, FP4_DYN_SMEM);
            if (dev >= 0 && dev < 64) opted[dev][bf16] = 1;
        }
    }
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, kern, FP4_THREADS, FP4_DYN_SMEM);
    if (bpsm < 1) bpsm = 1;
    const int64_t need = (total + FP4_THREADS - 1) / FP4_THREADS;
    const int grid = static_cast<int>(min(need, static_cast<int64_t>(num_sms()) * bpsm));
    if (bf16) k_search_nvfp4<uint16_t><<<grid, FP4_THREADS, FP4_DYN_SMEM, st>>>(a);
    else k_search_nvfp4<float><<<grid, FP4_THREADS, FP4_DYN_SMEM, st>>>(a);
    return check_launch("nvfp4 search");
}

}  // namespace tq
