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
// B200 mapping: a half-warp per block, lane = one window code; each warp
// works on two blocks at a time.  E2M1 rounding is done in the FMA pipe by
// adding and subtracting a binade-dependent power of two.  Near ties are
// re-ranked in fp64 with codes from the IEEE quotient.
#include "group_pack.cuh"

#include <climits>

namespace tq {

constexpr int FP4_WARPS = 8;
constexpr float FWIN = 3.0517578125e-05f;   // 2^-15

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
    int window;
};

// Largest E4M3 code whose value does not exceed t (clamped to [1, 126]); only
// an estimate is needed (the window search tests 32 positions around it).
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

// fp64 loss of block scale S for this lane's element (|w| = aw), summed over
// the half-warp; codes from the IEEE quotient.
__device__ __forceinline__ double loss64_fp4(float aw, float mv, float S) {
    const float y = (S == 0.f) ? 0.f : e2m1_round(__fdiv_rn(aw, S));
    const double e = __dsub_rn(static_cast<double>(aw), __dmul_rn(static_cast<double>(S), static_cast<double>(y)));
    return half_sum_d(__dmul_rn(static_cast<double>(mv), __dmul_rn(e, e)));
}

template <typename T>
__global__ void __launch_bounds__(FP4_WARPS * 32)
k_search_nvfp4(const __grid_constant__ Fp4Args a) {
    __shared__ float dec[128];
    __shared__ __align__(16) float2 blk[FP4_WARPS][2][16];
    for (int i = threadIdx.x; i < 128; i += blockDim.x) dec[i] = e4m3_value(i);
    __syncthreads();

    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int half = lane >> 4, hl = lane & 15;
    const unsigned hbits = half ? 0xffff0000u : 0x0000ffffu;
    const int64_t G = (a.I + 15) >> 4;
    const int64_t OG = a.O * G;
    const int64_t total = a.n_mat * OG;
    const int Wn = a.window;
    const int lo_max = 127 - Wn;   // window [lo, lo + Wn - 1] inside codes 1..126
    const T* W = static_cast<const T*>(a.W);
    const float4* mine4 = reinterpret_cast<const float4*>(blk[wid][half]);

    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * FP4_WARPS + wid) * 2; base < total;
         base += static_cast<int64_t>(gridDim.x) * FP4_WARPS * 2) {
        const int64_t bid = base + half;
        const bool vb = bid < total;
        int64_t e = 0, o = 0, kb = 0;
        if (vb) { e = bid / OG; const int64_t rem = bid - e * OG; o = rem / G; kb = rem - o * G; }
        const int64_t j0 = kb << 4;
        const int n = vb ? static_cast<int>(min(static_cast<int64_t>(16), a.I - j0)) : 0;
        const bool ve = hl < n;
        const float w = ve ? Elem<T>::load(W + e * a.ms + o * a.ld + j0 + hl) : 0.f;
        const float mv = ve ? __ldg(a.m + e * a.m_stride + j0 + hl) : 0.f;
        const float aw = fabsf(w);
        float amax = aw;
#pragma unroll
        for (int off = 8; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
        const float g = vb ? __ldg(a.g + e) : 0.f;
        const bool degen = (amax == 0.f) || (g == 0.f);

        // fp32 ranking works on |w|, m scaled by exact powers of two
        const float pw = amax > 0.f ? pow2_inv_binade(amax) : 1.f;
        float mmax = fabsf(mv);
#pragma unroll
        for (int off = 8; off; off >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(FULL, mmax, off));
        const float pm = mmax > 0.f ? pow2_inv_binade(mmax) : 1.f;
        const double back = 1.0 / (static_cast<double>(pw) * static_cast<double>(pw) * static_cast<double>(pm));
        __syncwarp();
        blk[wid][half][hl] = make_float2(__fmul_rn(aw, pw), __fmul_rn(mv, pm));
        __syncwarp();

        // ---- window: first lo with d(lo) <= d(lo + Wn), d(c) = |6 g dec(c) - a| (exact in fp64)
        const double g6 = 6.0 * static_cast<double>(g), ad = static_cast<double>(amax);
        const int cdn = e4m3_floor_code(amax / fmaxf(6.f * g, 1e-30f));
        const int la = min(max(cdn - 16 + hl, 1), lo_max - 1);
        const int lb = min(max(cdn + hl, 1), lo_max - 1);
        const bool pa = fabs(__dsub_rn(__dmul_rn(g6, dec[la]), ad)) > fabs(__dsub_rn(__dmul_rn(g6, dec[la + Wn]), ad));
        const bool pb = fabs(__dsub_rn(__dmul_rn(g6, dec[lb]), ad)) > fabs(__dsub_rn(__dmul_rn(g6, dec[lb + Wn]), ad));
        const unsigned ba = (__ballot_sync(FULL, pa) & hbits) >> (16 * half);
        const unsigned bb = (__ballot_sync(FULL, pb) & hbits) >> (16 * half);
        int lo;
        if (ba != 0xffffu) lo = min(max(cdn - 16 + (__ffs(~ba) - 1), 1), lo_max - 1);
        else if (bb != 0xffffu) lo = min(max(cdn + (__ffs(~bb) - 1), 1), lo_max - 1);
        else lo = min(max(cdn + 16, 1), lo_max);   // every tested start moves right

        // ---- candidate loop: lane hl = code lo + hl
        const bool act = hl < Wn;
        const int code = lo + (act ? hl : 0);
        const float S = __fmul_rn(g, dec[code]);       // the candidate block scale
        const float Ss = __fmul_rn(S, pw);               // scaled like the block
        const float invS = __frcp_rn(Ss);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 p = mine4[j];
            {
                const float y = e2m1_round(__fmul_rn(p.x, invS));
                const float er = __fmaf_rn(-Ss, y, p.x);
                acc = __fmaf_rn(__fmul_rn(p.y, er), er, acc);
            }
            {
                const float y = e2m1_round(__fmul_rn(p.z, invS));
                const float er = __fmaf_rn(-Ss, y, p.z);
                acc = __fmaf_rn(__fmul_rn(p.w, er), er, acc);
            }
        }
        float L = (act && !degen) ? acc : __int_as_float(0x7f800000);
        int ci = (act && !degen) ? code : INT_MAX;
        const float Lmine = L;
        group_argmin(L, ci, FULL, 16);
        const float thr = __fmaf_rn(L, FWIN, L);
        unsigned win = (__ballot_sync(FULL, act && !degen && Lmine <= thr) & hbits) >> (16 * half);
        double lossd = static_cast<double>(L) * back;
        // near ties: both halves walk their in-window candidates in code order
        int nwin = __popc(win);
        const bool need = nwin > 1;
        double best = __longlong_as_double(0x7ff0000000000000ll);
        int bcode = ci;
        unsigned todo = need ? win : 0u;
        while (__any_sync(FULL, todo != 0u)) {
            const int pos = todo ? __ffs(todo) - 1 : 0;
            const float Sc = __shfl_sync(FULL, S, (half << 4) + pos);
            const double Ld = loss64_fp4(aw, mv, Sc);
            if (todo) {
                if (Ld < best) { best = Ld; bcode = lo + pos; }
                todo &= todo - 1;
            }
        }
        if (need) { ci = bcode; lossd = best; }
        if (!degen && (ci < lo || ci >= lo + Wn)) ci = lo;   // every loss non-finite

        // ---- outputs and exact RTN + pack
        const int src = (half << 4) + (degen ? 0 : (ci - lo));
        const float Sf = __shfl_sync(FULL, S, src);
        double dl = 0.0;
        if (__any_sync(FULL, degen)) {
            const double wd = static_cast<double>(w);
            dl = half_sum_d(__dmul_rn(static_cast<double>(mv), __dmul_rn(wd, wd)));
        }
        unsigned c4 = 0u;
        if (!degen && aw != 0.f) {
            const int mag = e2m1_mag_code(e2m1_round(__fdiv_rn(aw, Sf)));
            c4 = static_cast<unsigned>(mag) | ((mag != 0 && w < 0.f) ? 8u : 0u);
        }
        if (vb && hl == 0) {
            a.scales[bid] = degen ? 0 : static_cast<uint8_t>(ci);
            if (a.idx) a.idx[bid] = degen ? -1 : ci;
            if (a.loss) a.loss[bid] = degen ? dl : lossd;
        }
        if (a.packed) {
            unsigned v = (c4 & 15u) << (4u * static_cast<unsigned>(hl & 7));
            v |= __shfl_xor_sync(FULL, v, 1);
            v |= __shfl_xor_sync(FULL, v, 2);
            v |= __shfl_xor_sync(FULL, v, 4);
            if (vb && (hl & 7) == 0) reinterpret_cast<uint32_t*>(a.packed + bid * 8)[hl >> 3] = v;
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
    int bpsm = 0;
    const bool bf16 = W->dtype == TQ_BF16;
    if (bf16) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, k_search_nvfp4<uint16_t>, FP4_WARPS * 32, 0);
    else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bpsm, k_search_nvfp4<float>, FP4_WARPS * 32, 0);
    if (bpsm < 1) bpsm = 1;
    const int64_t need = (total + 2 * FP4_WARPS - 1) / (2 * FP4_WARPS);
    const int grid = static_cast<int>(min(need, static_cast<int64_t>(num_sms()) * bpsm));
    if (bf16) k_search_nvfp4<uint16_t><<<grid, FP4_WARPS * 32, 0, st>>>(a);
    else k_search_nvfp4<float><<<grid, FP4_WARPS * 32, 0, st>>>(a);
    return check_launch("nvfp4 search");
}

}  // namespace tq
