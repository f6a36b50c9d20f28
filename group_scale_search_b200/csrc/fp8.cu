// FP8 (E4M3) weights with one scale per tensor, the scale chosen by an
// imatrix-weighted search.
//
// Source: "Nemotron-Cascade-2-30B-A3B-NVFP4" model card, Quantization Recipe
// table: the shared experts and the Mamba mixer linears are stored as FP8 with
// one scale per tensor (MSE-calibrated recipe).  Reading: the scale is chosen
// the way the other formats choose theirs, by the imatrix-weighted squared
// error, over candidates s_k = fl32(r_k amax / 448) with r_k = fl32(lo + (hi -
// lo) k / (n - 1)) on the NeUQI window [0.5, 1.2]; codes are E4M3
// round-to-nearest-even of the IEEE quotient fl32(w / s), saturating at 448,
// +0 for a zero result; What = fl32(s dec(c)).
//
// B200 mapping:
//  * k_fp8_loss: a block stages 1024 weights (and their imatrix weights) of
//    one matrix in shared memory; thread (k, p) evaluates candidate k on the
//    elements p, p + 4, ... (the 32 lanes of a warp read the same element:
//    broadcast; 4 consecutive elements per shared-memory load).  The code
//    comes from the hardware E4M3 conversion of the two products
//    w inv (1 -+ 2^-20), which bracket the IEEE quotient (E4M3 rounding is
//    monotone), and from an IEEE division where the two disagree; elements
//    go in pairs through packed fp32x2 products, one conversion per bracket
//    end and one decode; w - What is exact in fp32 for ratios >= 0.5 and the
//    weighted square is accumulated in fp64.  Blocks write per-candidate
//    partial sums; k_fp8_pick adds them in block order (deterministic) and
//    takes the lowest candidate of the minimum.
//  * k_fp8_pack / k_fp8_dequant: octet walkers (8 weights per thread, one
//    16-byte bf16 load / one 8-byte code store) with the same conversions.
#include "walk.cuh"

namespace tq {

tq_status launch_amax(const tq_mat* W, float* amax, cudaStream_t st);   // imatrix.cu

constexpr int F8_MAXC = 64;
constexpr int F8_THREADS = 1024;      // 64 candidates x 16 element lanes (one block per SM measured 6 % faster than four of 256)
constexpr int F8_CHUNK = 1024;        // elements staged per block iteration
constexpr int64_t F8_TARGET_BLOCKS = 2048;

// E4M3 codes of two fp32 values (nearest, ties to even, saturating at +-448),
// `lo` in the low byte.
__device__ __forceinline__ unsigned e4m3x2_from_f32(float lo, float hi) {
    unsigned short h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(h) : "f"(lo), "f"(hi));
    return h;
}

// The two E4M3 values of a 16-bit pair of codes (low byte first), exactly.
__device__ __forceinline__ float2 f8x2_to_f32(unsigned two) {
    unsigned h2;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "r"(two));
    __half2_raw raw;
    raw.x = static_cast<unsigned short>(h2 & 0xffffu);
    raw.y = static_cast<unsigned short>(h2 >> 16);
    return __half22float2(__half2(raw));
}

__device__ __forceinline__ unsigned e4m3_canon(unsigned c) { return (c & 0x7fu) ? c : 0u; }   // -0 -> +0

// E4M3 code of fl32(w / s): bracketed products, IEEE division where they disagree.
// `fast` is false for a zero, subnormal or extreme scale.
__device__ __forceinline__ unsigned fp8_code(float w, float s, float ilo, float ihi, bool fast) {
    if (fast) {
        const unsigned two = e4m3x2_from_f32(__fmul_rn(w, ilo), __fmul_rn(w, ihi));
        const unsigned a = e4m3_canon(two & 0xffu), b = e4m3_canon(two >> 8);
        if (a == b) return a;
    }
    if (s == 0.f) return 0u;
    return e4m3_canon(e4m3x2_from_f32(__fdiv_rn(w, s), 0.f) & 0xffu);
}

struct Fp8Scale {
    float s, ilo, ihi;
    bool fast;
    __device__ __forceinline__ explicit Fp8Scale(float s_) : s(s_) {
        const unsigned se = (__float_as_uint(s) >> 23) & 255u;
        fast = se >= 3u && se <= 251u;
        const float inv = fast ? rcp_approx(s) : 0.f;
        ilo = __fmul_rn(inv, 0.99999904632568359375f);   // 1 - 2^-20
        ihi = __fmul_rn(inv, 1.00000095367431640625f);   // 1 + 2^-20
    }
    __device__ __forceinline__ unsigned code(float w) const { return fp8_code(w, s, ilo, ihi, fast); }
};

// s_k = fl32(r_k amax / 448), computed as the oracle defines it (fp64, one rounding).
__device__ __forceinline__ float fp8_cand(float r, float amax) {
    return __double2float_rn(__ddiv_rn(__dmul_rn(static_cast<double>(r), static_cast<double>(amax)), 448.0));
}

struct F8Args {
    const void* W;
    int64_t O, I, ld, ms;
    const float* m;
    int64_t m_stride;
    int n;
    float r[F8_MAXC];
    const float* amax;   // [n_mat]
    double* part;        // [n_mat][bpm][n]
    int64_t bpm;         // blocks per matrix
};

// E4M3 codes of fl32(w0 / s), fl32(w1 / s) as a pair (w0's in the low
// byte), for the loss loop: one packed multiply per bracket end, one
// conversion per end for both elements; an IEEE division only for an element
// whose two ends disagree.  The sign of a zero result is kept (it does not
// change the error).
__device__ __forceinline__ unsigned fp8_code_pair(float w0, float w1, const Fp8Scale& sc) {
    const float2 ww = make_float2(w0, w1);
    const float2 lo = __fmul2_rn(ww, make_float2(sc.ilo, sc.ilo)), hi = __fmul2_rn(ww, make_float2(sc.ihi, sc.ihi));
    const unsigned clo = e4m3x2_from_f32(lo.x, lo.y), chi = e4m3x2_from_f32(hi.x, hi.y);
    if (sc.fast && clo == chi) return clo;
    if (sc.s == 0.f) return 0u;
    unsigned c = clo;
    if (!sc.fast || ((clo ^ chi) & 0xffu)) c = (c & 0xff00u) | (e4m3x2_from_f32(__fdiv_rn(w0, sc.s), 0.f) & 0xffu);
    if (!sc.fast || ((clo ^ chi) & 0xff00u)) c = (c & 0xffu) | ((e4m3x2_from_f32(__fdiv_rn(w1, sc.s), 0.f) & 0xffu) << 8);
    return c;
}

// EXACT_F32: every candidate ratio is >= 0.5, so |w / s| <= 896 and w - What
// is exact in fp32 (Sterbenz: What is 0 or within a factor 2 of w).
template <typename T, bool EXACT_F32>
__global__ void __launch_bounds__(F8_THREADS)
k_fp8_loss(const __grid_constant__ F8Args a) {
    __shared__ __align__(16) float sw[F8_CHUNK];
    __shared__ __align__(16) double smv[F8_CHUNK];
    __shared__ double red[F8_THREADS / F8_MAXC][F8_MAXC];
    constexpr int P = F8_THREADS / F8_MAXC;   // element lanes
    const int k = threadIdx.x & (F8_MAXC - 1), p = threadIdx.x / F8_MAXC;
    const int64_t e = blockIdx.y, b = blockIdx.x;
    const float amax = a.amax[e];
    const bool active = k < a.n && amax > 0.f;
    const Fp8Scale sc(active ? fp8_cand(a.r[k], amax) : 1.f);
    const T* W = static_cast<const T*>(a.W) + e * a.ms;
    const float* m = a.m + e * a.m_stride;
    const int64_t r0 = a.O * b / a.bpm, r1 = a.O * (b + 1) / a.bpm;   // this block's rows
    const int64_t n_el = (r1 - r0) * a.I;
    double acc = 0.0;
    if (amax > 0.f) {
        for (int64_t c0 = 0; c0 < n_el; c0 += F8_CHUNK) {
            const int nc = static_cast<int>(min(static_cast<int64_t>(F8_CHUNK), n_el - c0));
            __syncthreads();
            // element c0 + i of the block's rows: one division per chunk, then
            // the column steps on by the thread stride (wrapping into the next row)
            int64_t rq = (c0 + threadIdx.x) / a.I;
            int64_t jq = c0 + threadIdx.x - rq * a.I;
            for (int i = threadIdx.x; i < F8_CHUNK; i += F8_THREADS) {   // zeros past the chunk's end
                float w = 0.f, mm = 0.f;
                if (i < nc) {
                    w = Elem<T>::load(W + (r0 + rq) * a.ld + jq);
                    mm = __ldg(m + jq);
                }
                sw[i] = w;
                smv[i] = static_cast<double>(mm);
                jq += F8_THREADS;
                while (jq >= a.I) { jq -= a.I; ++rq; }
            }
            __syncthreads();
            if (active) {
                const float4* sw4 = reinterpret_cast<const float4*>(sw);
                const double2* sm2 = reinterpret_cast<const double2*>(smv);
                for (int i4 = p; 4 * i4 < nc; i4 += P) {   // 4 consecutive elements per step
                    const float4 w4 = sw4[i4];
                    const double2 ma = sm2[2 * i4], mb = sm2[2 * i4 + 1];
                    const float w[4] = {w4.x, w4.y, w4.z, w4.w};
                    const double mv[4] = {ma.x, ma.y, mb.x, mb.y};
                    const float2 s2 = make_float2(sc.s, sc.s);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {   // elements 2h, 2h + 1 as a pair
                        const float2 ww = make_float2(w[2 * h], w[2 * h + 1]);
                        const float2 wh = __fmul2_rn(s2, f8x2_to_f32(fp8_code_pair(ww.x, ww.y, sc)));
                        double d0, d1;
                        if constexpr (EXACT_F32) {
                            const float2 d = __fadd2_rn(ww, make_float2(-wh.x, -wh.y));
                            d0 = static_cast<double>(d.x);
                            d1 = static_cast<double>(d.y);
                        } else {
                            d0 = __dsub_rn(static_cast<double>(ww.x), static_cast<double>(wh.x));
                            d1 = __dsub_rn(static_cast<double>(ww.y), static_cast<double>(wh.y));
                        }
                        acc = __fma_rn(mv[2 * h], __dmul_rn(d0, d0), acc);   // padding: m = 0
                        acc = __fma_rn(mv[2 * h + 1], __dmul_rn(d1, d1), acc);
                    }
                }
            }
        }
    }
    red[p][k] = acc;
    __syncthreads();
    if (p == 0 && k < a.n) {
        double t = red[0][k];
#pragma unroll
        for (int q = 1; q < P; ++q) t = __dadd_rn(t, red[q][k]);
        a.part[(e * a.bpm + b) * a.n + k] = t;
    }
}

// One block of 64 threads per matrix: L_k = sum over blocks in order; the
// lowest k of the minimum.
struct F8Ratios {
    float r[F8_MAXC];
};

__global__ void k_fp8_pick(const double* __restrict__ part, int64_t bpm, int n, const __grid_constant__ F8Ratios rr,
                           const float* __restrict__ amax, float* __restrict__ scales, int32_t* __restrict__ idx,
                           double* __restrict__ loss, double* __restrict__ losses) {
    const float* r = rr.r;
    __shared__ double L[F8_MAXC];
    const int64_t e = blockIdx.x;
    const int k = threadIdx.x;
    double t = 0.0;
    if (k < n)
        for (int64_t b = 0; b < bpm; ++b) t = __dadd_rn(t, part[(e * bpm + b) * n + k]);
    if (k < n) {
        L[k] = t;
        if (losses) losses[e * n + k] = t;
    }
    __syncthreads();
    if (k == 0) {
        const float am = amax[e];
        int best = -1;
        double bl = __longlong_as_double(0x7ff0000000000000ll);
        if (am > 0.f)
            for (int q = 0; q < n; ++q)
                if (L[q] < bl) { bl = L[q]; best = q; }
        if (best < 0) bl = 0.0;
        scales[e] = best < 0 ? 0.f : fp8_cand(r[best], am);
        if (idx) idx[e] = best;
        if (loss) loss[e] = bl;
    }
}

// E4M3 codes of W with one scale per matrix: 8 weights per thread.
template <typename T>
__global__ void k_fp8_pack(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms,
                           const float* __restrict__ scales, int64_t n_mat, uint8_t* __restrict__ out) {
    const int64_t C = (I + 7) >> 3, total = n_mat * O * C;
    const bool vec = (I & 7) == 0;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = t / C, c = t - row * C, e = row / O, o = row - e * O;
        const int64_t j = c << 3;
        const int n = static_cast<int>(min(static_cast<int64_t>(8), I - j));
        Oct<T> oc;
        oc.load(W + e * ms + o * ld + j, n);
        float w[8];
        oc.get(w);
        const Fp8Scale sc(__ldg(scales + e));
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) lo |= sc.code(w[i]) << (8 * i);
#pragma unroll
        for (int i = 0; i < 4; ++i) hi |= sc.code(w[4 + i]) << (8 * i);
        uint8_t* dst = out + row * I + j;
        if (vec) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < n) dst[i] = static_cast<uint8_t>(((i < 4 ? lo : hi) >> (8 * (i & 3))) & 0xffu);
        }
    }
}

template <typename O>
__global__ void k_fp8_dequant(const uint8_t* __restrict__ codes, const float* __restrict__ scales, int64_t n_mat,
                              int64_t Orows, int64_t I, O* __restrict__ out) {
    const int64_t C = (I + 7) >> 3, total = n_mat * Orows * C;
    const bool vec = (I & 7) == 0;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = t / C, c = t - row * C, e = row / Orows;
        const int64_t j = c << 3;
        const int n = static_cast<int>(min(static_cast<int64_t>(8), I - j));
        const uint8_t* src = codes + row * I + j;
        uint32_t lo = 0u, hi = 0u;
        if (vec) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
            lo = v.x; hi = v.y;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < n) (i < 4 ? lo : hi) |= static_cast<uint32_t>(__ldg(src + i)) << (8 * (i & 3));
        }
        const float s = __ldg(scales + e);
        float v[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t wd = h ? hi : lo;
            const float2 a = f8x2_to_f32(wd & 0xffffu), b = f8x2_to_f32(wd >> 16);
            v[4 * h] = __fmul_rn(s, a.x); v[4 * h + 1] = __fmul_rn(s, a.y);
            v[4 * h + 2] = __fmul_rn(s, b.x); v[4 * h + 3] = __fmul_rn(s, b.y);
        }
        O* dst = out + row * I + j;
        if (vec) {   // rows of a multiple of 8 elements: 32-byte (fp32) / 16-byte (bf16) aligned octets
            if constexpr (sizeof(O) == 4) {
                float4* d = reinterpret_cast<float4*>(dst);
                d[0] = make_float4(v[0], v[1], v[2], v[3]);
                d[1] = make_float4(v[4], v[5], v[6], v[7]);
            } else {
                uint32_t u[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                    u[i] = *reinterpret_cast<uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(dst) = make_uint4(u[0], u[1], u[2], u[3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < n) {
                    if constexpr (sizeof(O) == 4) dst[i] = v[i];
                    else dst[i] = __float2bfloat16_rn(v[i]);
                }
            }
        }
    }
}

static int64_t fp8_bpm(const tq_mat* W) {
    int64_t b = F8_TARGET_BLOCKS / W->n_mat;
    b = b < 1 ? 1 : b;
    return b > W->rows ? W->rows : b;
}

static int64_t fp8_grid(int64_t work_items) {
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    const int64_t need = (work_items + 255) / 256;
    return need < 1 ? 1 : (need < cap ? need : cap);
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_fp8_workspace_bytes(const tq_mat* W) {
    if (!W || W->n_mat < 1 || W->rows < 1) return 0;
    const int64_t amax_bytes = (W->n_mat * 4 + 15) / 16 * 16;
    return static_cast<size_t>(amax_bytes + W->n_mat * fp8_bpm(W) * F8_MAXC * 8);
}

TQ_API tq_status tq_search_fp8(const tq_mat* W, const float* m, int64_t m_stride, int32_t n_cand, double lo,
                               double hi, float* scales, int32_t* cand_idx, double* loss, double* losses,
                               uint8_t* packed, void* workspace, size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_search_fp8 W");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(m != nullptr && scales != nullptr && workspace != nullptr, "tq_search_fp8: null pointer");
    TQ_REQUIRE(aligned16(workspace), "tq_search_fp8: workspace not 16-byte aligned");
    TQ_REQUIRE(W->n_mat == 1 || m_stride == 0 || m_stride >= W->cols, "tq_search_fp8: m_stride must be 0 or >= cols");
    TQ_REQUIRE(packed == nullptr || aligned16(packed), "tq_search_fp8: packed not 16-byte aligned");
    if (n_cand < 2 || n_cand > F8_MAXC) return set_error(TQ_ERR_UNSUPPORTED, "tq_search_fp8: n_cand must be in [2, 64]");
    TQ_REQUIRE(lo > 0.0 && hi >= lo, "tq_search_fp8: need 0 < lo <= hi");
    TQ_REQUIRE(W->n_mat <= 65535, "tq_search_fp8: more than 65535 matrices");
    TQ_REQUIRE(workspace_bytes >= tq_fp8_workspace_bytes(W), "tq_search_fp8: workspace too small");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float* amax = static_cast<float*>(workspace);
    const int64_t amax_bytes = (W->n_mat * 4 + 15) / 16 * 16;
    double* part = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + amax_bytes);
    if ((s = launch_amax(W, amax, st)) != TQ_OK) return s;
    F8Args a;
    a.W = W->ptr; a.O = W->rows; a.I = W->cols; a.ld = W->ld; a.ms = W->n_mat > 1 ? W->mat_stride : 0;
    a.m = m; a.m_stride = W->n_mat > 1 ? m_stride : 0;
    a.n = n_cand;
    for (int k = 0; k < F8_MAXC; ++k)
        a.r[k] = k < n_cand ? static_cast<float>(lo + ((hi - lo) * static_cast<double>(k)) / static_cast<double>(n_cand - 1))
                            : 1.0f;
    a.amax = amax; a.part = part; a.bpm = fp8_bpm(W);
    const dim3 grid(static_cast<unsigned>(a.bpm), static_cast<unsigned>(W->n_mat));
    const bool exact32 = lo >= 0.5;   // every ratio >= 0.5 (the ratios rise from lo)
    if (W->dtype == TQ_BF16) exact32 ? k_fp8_loss<uint16_t, true><<<grid, F8_THREADS, 0, st>>>(a)
                                     : k_fp8_loss<uint16_t, false><<<grid, F8_THREADS, 0, st>>>(a);
    else exact32 ? k_fp8_loss<float, true><<<grid, F8_THREADS, 0, st>>>(a)
                 : k_fp8_loss<float, false><<<grid, F8_THREADS, 0, st>>>(a);
    F8Ratios rr;
    for (int k = 0; k < F8_MAXC; ++k) rr.r[k] = a.r[k];
    k_fp8_pick<<<static_cast<unsigned>(W->n_mat), F8_MAXC, 0, st>>>(part, a.bpm, n_cand, rr, amax, scales, cand_idx,
                                                                   loss, losses);
    if (packed) {
        const int64_t work = W->n_mat * W->rows * ((W->cols + 7) / 8);
        if (W->dtype == TQ_BF16)
            k_fp8_pack<uint16_t><<<static_cast<unsigned>(fp8_grid(work)), 256, 0, st>>>(
                static_cast<const uint16_t*>(W->ptr), W->rows, W->cols, W->ld, a.ms, scales, W->n_mat, packed);
        else
            k_fp8_pack<float><<<static_cast<unsigned>(fp8_grid(work)), 256, 0, st>>>(
                static_cast<const float*>(W->ptr), W->rows, W->cols, W->ld, a.ms, scales, W->n_mat, packed);
    }
    return check_launch("tq_search_fp8");
}

TQ_API tq_status tq_pack_fp8(const tq_mat* W, const float* scales, uint8_t* packed, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_pack_fp8 W");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(scales != nullptr && packed != nullptr, "tq_pack_fp8: null pointer");
    TQ_REQUIRE(aligned16(packed), "tq_pack_fp8: packed not 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0;
    const int64_t work = W->n_mat * W->rows * ((W->cols + 7) / 8);
    if (W->dtype == TQ_BF16)
        k_fp8_pack<uint16_t><<<static_cast<unsigned>(fp8_grid(work)), 256, 0, st>>>(
            static_cast<const uint16_t*>(W->ptr), W->rows, W->cols, W->ld, ms, scales, W->n_mat, packed);
    else
        k_fp8_pack<float><<<static_cast<unsigned>(fp8_grid(work)), 256, 0, st>>>(
            static_cast<const float*>(W->ptr), W->rows, W->cols, W->ld, ms, scales, W->n_mat, packed);
    return check_launch("tq_pack_fp8");
}

TQ_API tq_status tq_dequant_fp8(const uint8_t* packed, const float* scales, int64_t n_mat, int64_t O, int64_t I,
                                void* out, int32_t out_dtype, tq_stream_t stream) {
    clear_error();
    TQ_REQUIRE(packed && scales && out, "tq_dequant_fp8: null pointer");
    TQ_REQUIRE(n_mat >= 1 && O >= 1 && I >= 1, "tq_dequant_fp8: empty shape");
    TQ_REQUIRE(aligned16(packed) && aligned16(out), "tq_dequant_fp8: packed/out not 16-byte aligned");
    if (elem_bytes(out_dtype) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant_fp8: out dtype %d", out_dtype);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t work = n_mat * O * ((I + 7) / 8);
    if (out_dtype == TQ_BF16)
        k_fp8_dequant<__nv_bfloat16><<<static_cast<unsigned>(fp8_grid(work)), 256, 0, st>>>(
            packed, scales, n_mat, O, I, static_cast<__nv_bfloat16*>(out));
    else
        k_fp8_dequant<float><<<static_cast<unsigned>(fp8_grid(work)), 256, 0, st>>>(packed, scales, n_mat, O, I,
                                                                                     static_cast<float*>(out));
    return check_launch("tq_dequant_fp8");
}
