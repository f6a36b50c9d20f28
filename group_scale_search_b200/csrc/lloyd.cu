// Imatrix-weighted Lloyd-Max 2-bit codebook on absmax-normalised 32-weight
// groups, and its 2-bit codes.
//
// Source: "Phase 2: math-accuracy regression on tq3a-tq2e g32"
// (turboquant-mlx issue #2), Phase-2 candidate 1: fit the 2-bit experts'
// Lloyd-Max codebook to calibration data instead of the data-free one, and
// keep it fixed and shared.  Reading (the page gives the idea only): groups of
// 32 weights with s = max |w|; u = fl32(w / s) (0 when s = 0); one 4-level
// codebook c_0 < c_1 < c_2 < c_3 (fp32) shared by every matrix of the call,
// minimising sum m_j (w - s c_a)^2 = sum omega (u - c_a)^2 with
// omega = m_j s^2 by Lloyd iterations: every element goes to the nearest level
// (u above the exact midpoint (c_i + c_{i+1}) / 2 moves up, so ties go to the
// lower level), every level becomes the omega-weighted mean of its elements
// (fp64, rounded once to fp32; an empty level keeps its value).  The start is
// supplied by the caller (the data-free Lloyd-Max levels of a uniform source,
// {-3/4, -1/4, 1/4, 3/4}, by default in the binding).  Codes: 2 bits per
// weight, a 32-weight group in 8 bytes (element k of the group at bits
// 2 (k % 4) of byte k / 4; padding past I is code 0); What = fl32(s c_a).
//
// B200 mapping: one HBM pass per iteration (k_lm_pass: 8 weights per thread,
// one 16-byte bf16 load; u from a per-group reciprocal with a Markstein
// correction; per-level fp64 sums of omega u and omega by predicated adds and
// the sum of omega u^2 in registers, added over the block in a fixed tree),
// then one block (k_lm_update) adds the block partials in block order
// (deterministic), takes the loss sum omega (u - c_a)^2 from the sums and
// writes the new codebook.  The group scales
// come from one pass before (k_lm_scales: 4 threads per group, shuffle max).
#include "walk.cuh"

namespace tq {

constexpr int LM_THREADS = 256;
constexpr int LM_SUMS = 9;   // num[4] = sum omega u, den[4] = sum omega per level; sum omega u^2

// Flat thread index -> (row, octet) with each row's octets padded to whole
// groups (4 octets per group), so a group is 4 consecutive threads.
struct LmGeom {
    int64_t rows, I, G, per_row;   // per_row = 4 G octets
    GroupIndex gi;                 // octet t -> (matrix, row, octet of the row), 32-bit (< 2^32 octets)
    FastDiv pr;                    // octet t -> row of the flattened batch
};

template <typename T>
__global__ void k_lm_scales(const T* __restrict__ W, int64_t O, int64_t ld, int64_t ms, LmGeom g,
                            float* __restrict__ scales) {
    const int64_t total = g.rows * g.per_row;
    for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x; t0 < total; t0 += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = t0 + threadIdx.x;
        float a = 0.f;
        if (t < total) {
            uint32_t e, o, c;
            g.gi.split(static_cast<uint32_t>(t), e, o, c);
            const int64_t j = static_cast<int64_t>(c) << 3;
            if (j < g.I) {
                Oct<T> oc;
                oc.load(W + static_cast<int64_t>(e) * ms + static_cast<int64_t>(o) * ld + j,
                        static_cast<int>(min(static_cast<int64_t>(8), g.I - j)));
                float w[8];
                oc.get(w);
#pragma unroll
                for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(w[i]));
            }
        }
        a = fmaxf(a, __shfl_xor_sync(FULL, a, 1));
        a = fmaxf(a, __shfl_xor_sync(FULL, a, 2));
        if (t < total && (t & 3) == 0) scales[t >> 2] = a;
    }
}

// fl32(w / s) for the elements of one group: with r = fl32(1/s), the
// correction q1 = fma(fma(-s, q0, w), r, q0) of q0 = w r is the correctly
// rounded quotient when s, w, r, q0, the residual and the quotient are all
// normal (Markstein): with s in [2^-60, 2^60] and |w| >= 2^-60, |u| lies in
// [2^-120, 1] (|w| <= s: s is the group's max |w|).  Elsewhere (tiny w,
// extreme or zero s) the IEEE division.
struct LmDiv {
    float s, r;
    bool fast;
    __device__ __forceinline__ explicit LmDiv(float s_) : s(s_) {
        fast = s >= 8.673617379884035e-19f && s <= 1.152921504606847e18f;   // [2^-60, 2^60]
        r = fast ? __frcp_rn(s) : 0.f;
    }
    __device__ __forceinline__ float u(float w) const {
        if (fast && fabsf(w) >= 8.673617379884035e-19f) {
            const float q0 = __fmul_rn(w, r);
            return __fmaf_rn(__fmaf_rn(-s, q0, w), r, q0);
        }
        return s == 0.f ? 0.f : __fdiv_rn(w, s);
    }
};

template <typename T>
__global__ void __launch_bounds__(LM_THREADS)
k_lm_pass(const T* __restrict__ W, int64_t O, int64_t ld, int64_t ms, const float* __restrict__ m, int64_t m_stride,
          LmGeom g, const float* __restrict__ scales, const float* __restrict__ codebook, double* __restrict__ part) {
    __shared__ double red[LM_THREADS / 32][LM_SUMS];
    const double c0 = codebook[0], c1 = codebook[1], c2 = codebook[2], c3 = codebook[3];
    const double m01 = (c0 + c1) * 0.5, m12 = (c1 + c2) * 0.5, m23 = (c2 + c3) * 0.5;   // exact
    double acc[LM_SUMS];
#pragma unroll
    for (int i = 0; i < LM_SUMS; ++i) acc[i] = 0.0;
    const int64_t total = g.rows * g.per_row;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint32_t e, o, c;
        g.gi.split(static_cast<uint32_t>(t), e, o, c);
        const int64_t j = static_cast<int64_t>(c) << 3;
        if (j >= g.I) continue;
        const int n = static_cast<int>(min(static_cast<int64_t>(8), g.I - j));
        Oct<T> oc;
        oc.load(W + static_cast<int64_t>(e) * ms + static_cast<int64_t>(o) * ld + j, n);
        float w[8];
        oc.get(w);
        Oct<float> mo;
        mo.load(m + static_cast<int64_t>(e) * m_stride + j, n);
        float mv[8];
        mo.get(mv);
        const float s = __ldg(scales + (t >> 2));
        const double s2 = static_cast<double>(s) * static_cast<double>(s);
        const LmDiv dv(s);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double u = static_cast<double>(dv.u(w[i]));
            const double om = static_cast<double>(mv[i]) * s2;   // padding: m = 0
            const double ou = om * u;
            acc[8] = __fma_rn(ou, u, acc[8]);
            // one predicated add per sum: the level's accumulators only
            if (u > m12) {
                if (u > m23) { acc[3] += ou; acc[7] += om; } else { acc[2] += ou; acc[6] += om; }
            } else {
                if (u > m01) { acc[1] += ou; acc[5] += om; } else { acc[0] += ou; acc[4] += om; }
            }
        }
    }
    // block sum in a fixed order: warp butterfly, then warps in order
#pragma unroll
    for (int i = 0; i < LM_SUMS; ++i) {
        double v = acc[i];
#pragma unroll
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(FULL, v, off);
        acc[i] = v;
    }
    if ((threadIdx.x & 31) == 0)
#pragma unroll
        for (int i = 0; i < LM_SUMS; ++i) red[threadIdx.x >> 5][i] = acc[i];
    __syncthreads();
    if (threadIdx.x < LM_SUMS) {
        double v = red[0][threadIdx.x];
        for (int wv = 1; wv < LM_THREADS / 32; ++wv) v += red[wv][threadIdx.x];
        part[static_cast<int64_t>(blockIdx.x) * LM_SUMS + threadIdx.x] = v;
    }
}

// Adds the block partials in order; writes history[it] and, unless this was
// the last pass, the new codebook (an empty level keeps its value).
__global__ void k_lm_update(const double* __restrict__ part, int blocks, float* __restrict__ codebook, int it,
                            int last, double* __restrict__ loss, double* __restrict__ history) {
    __shared__ double sum[LM_SUMS];
    if (threadIdx.x < LM_SUMS) {
        double v = 0.0;
        for (int b = 0; b < blocks; ++b) v += part[static_cast<int64_t>(b) * LM_SUMS + threadIdx.x];
        sum[threadIdx.x] = v;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // sum omega (u - c_a)^2 = sum omega u^2 - 2 sum_a c_a N_a + sum_a c_a^2 D_a
        double L = sum[8];
        for (int i = 0; i < 4; ++i) {
            const double c = codebook[i];
            L = L - 2.0 * c * sum[i] + c * c * sum[4 + i];
        }
        L = L > 0.0 ? L : 0.0;
        if (history) history[it] = L;
        if (last) {
            if (loss) *loss = L;
        } else {
            for (int i = 0; i < 4; ++i)
                if (sum[4 + i] > 0.0) codebook[i] = __double2float_rn(sum[i] / sum[4 + i]);
        }
    }
}

// 2-bit codes: a group's 4 threads write 2 bytes each (8 weights).
template <typename T>
__global__ void k_lm_pack(const T* __restrict__ W, int64_t O, int64_t ld, int64_t ms, LmGeom g,
                          const float* __restrict__ scales, const float* __restrict__ codebook,
                          uint8_t* __restrict__ packed) {
    const double c0 = codebook[0], c1 = codebook[1], c2 = codebook[2], c3 = codebook[3];
    const double m01 = (c0 + c1) * 0.5, m12 = (c1 + c2) * 0.5, m23 = (c2 + c3) * 0.5;
    const int64_t total = g.rows * g.per_row;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint32_t e, o, c;
        g.gi.split(static_cast<uint32_t>(t), e, o, c);
        const int64_t j = static_cast<int64_t>(c) << 3;
        unsigned bits = 0u;
        if (j < g.I) {
            const int n = static_cast<int>(min(static_cast<int64_t>(8), g.I - j));
            Oct<T> oc;
            oc.load(W + static_cast<int64_t>(e) * ms + static_cast<int64_t>(o) * ld + j, n);
            float w[8];
            oc.get(w);
            const LmDiv dv(__ldg(scales + (t >> 2)));
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double u = static_cast<double>(dv.u(w[i]));
                const unsigned a = (u > m01 ? 1u : 0u) + (u > m12 ? 1u : 0u) + (u > m23 ? 1u : 0u);
                bits |= (i < n ? a : 0u) << (2 * i);
            }
        }
        reinterpret_cast<uint16_t*>(packed)[t] = static_cast<uint16_t>(bits);
    }
}

template <typename OT>
__global__ void k_lm_dequant(const uint8_t* __restrict__ packed, const float* __restrict__ scales,
                             const float* __restrict__ codebook, LmGeom g, OT* __restrict__ out) {
    const float cb[4] = {codebook[0], codebook[1], codebook[2], codebook[3]};
    const int64_t total = g.rows * g.per_row;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = g.pr.div(static_cast<uint32_t>(t)), c = t - row * g.per_row;
        const int64_t j = c << 3;
        if (j >= g.I) continue;
        const int n = static_cast<int>(min(static_cast<int64_t>(8), g.I - j));
        const unsigned bits = __ldg(reinterpret_cast<const uint16_t*>(packed) + t);
        const float s = __ldg(scales + (t >> 2));
        OT* dst = out + row * g.I + j;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < n) {
                const unsigned a = (bits >> (2 * i)) & 3u;
                const float ca = a == 0 ? cb[0] : (a == 1 ? cb[1] : (a == 2 ? cb[2] : cb[3]));
                const float v = __fmul_rn(s, ca);
                if constexpr (sizeof(OT) == 4) dst[i] = v;
                else dst[i] = __float2bfloat16_rn(v);
            }
        }
    }
}

// O: rows per matrix (the flattened rows are n_mat * O).
static LmGeom lm_geom(int64_t rows, int64_t O, int64_t I) {
    LmGeom g;
    g.rows = rows; g.I = I; g.G = (I + 31) / 32; g.per_row = 4 * g.G;
    g.gi = GroupIndex(O, g.per_row);
    g.pr = FastDiv(static_cast<uint32_t>(g.per_row));
    return g;
}

static int64_t lm_blocks(int64_t threads_needed) {
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    const int64_t need = (threads_needed + LM_THREADS - 1) / LM_THREADS;
    return need < 1 ? 1 : (need < cap ? need : cap);
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_lloyd_workspace_bytes(const tq_mat* W) {
    if (!W || W->n_mat < 1 || W->rows < 1 || W->cols < 1) return 0;
    const LmGeom g = lm_geom(W->n_mat * W->rows, W->rows, W->cols);
    return static_cast<size_t>(lm_blocks(g.rows * g.per_row) * LM_SUMS * 8);
}

TQ_API tq_status tq_lloyd_max_g32(const tq_mat* W, const float* m, int64_t m_stride, int32_t n_iter, float* codebook,
                                  float* scales, uint8_t* packed, double* loss, double* history, void* workspace,
                                  size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_lloyd_max_g32 W");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(m && codebook && scales && workspace, "tq_lloyd_max_g32: null pointer");
    TQ_REQUIRE(aligned16(m) && aligned16(workspace), "tq_lloyd_max_g32: m/workspace not 16-byte aligned");
    TQ_REQUIRE(W->n_mat == 1 || m_stride == 0 || (m_stride >= W->cols && m_stride % 4 == 0),
               "tq_lloyd_max_g32: m_stride must be 0 or a multiple of 4 >= cols");
    TQ_REQUIRE(packed == nullptr || aligned16(packed), "tq_lloyd_max_g32: packed not 16-byte aligned");
    TQ_REQUIRE(n_iter >= 0 && n_iter <= 1000, "tq_lloyd_max_g32: n_iter in [0, 1000]");
    TQ_REQUIRE(workspace_bytes >= tq_lloyd_workspace_bytes(W), "tq_lloyd_max_g32: workspace too small");
    TQ_REQUIRE(W->n_mat * W->rows * 4 * ((W->cols + 31) / 32) < (int64_t(1) << 32),
               "tq_lloyd_max_g32: more than 2^32 octets of weights in one call");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const LmGeom g = lm_geom(W->n_mat * W->rows, W->rows, W->cols);
    const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0, mst = W->n_mat > 1 ? m_stride : 0;
    const int64_t threads = g.rows * g.per_row;
    const unsigned blocks = static_cast<unsigned>(lm_blocks(threads));
    double* part = static_cast<double*>(workspace);
    const bool bf = W->dtype == TQ_BF16;
    if (bf) k_lm_scales<uint16_t><<<blocks, LM_THREADS, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->rows, W->ld, ms, g, scales);
    else k_lm_scales<float><<<blocks, LM_THREADS, 0, st>>>(static_cast<const float*>(W->ptr), W->rows, W->ld, ms, g, scales);
    for (int it = 0; it <= n_iter; ++it) {
        if (bf) k_lm_pass<uint16_t><<<blocks, LM_THREADS, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->rows, W->ld, ms,
                                                                      m, mst, g, scales, codebook, part);
        else k_lm_pass<float><<<blocks, LM_THREADS, 0, st>>>(static_cast<const float*>(W->ptr), W->rows, W->ld, ms,
                                                                m, mst, g, scales, codebook, part);
        k_lm_update<<<1, 32, 0, st>>>(part, static_cast<int>(blocks), codebook, it, it == n_iter ? 1 : 0, loss, history);
    }
    if (packed) {
        if (bf) k_lm_pack<uint16_t><<<blocks, LM_THREADS, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->rows, W->ld, ms, g,
                                                                      scales, codebook, packed);
        else k_lm_pack<float><<<blocks, LM_THREADS, 0, st>>>(static_cast<const float*>(W->ptr), W->rows, W->ld, ms, g,
                                                                scales, codebook, packed);
    }
    return check_launch("tq_lloyd_max_g32");
}

TQ_API tq_status tq_dequant_lm2(const uint8_t* packed, const float* codebook, const float* scales, int64_t n_mat,
                                int64_t O, int64_t I, void* out, int32_t out_dtype, tq_stream_t stream) {
    clear_error();
    TQ_REQUIRE(packed && codebook && scales && out, "tq_dequant_lm2: null pointer");
    TQ_REQUIRE(n_mat >= 1 && O >= 1 && I >= 1, "tq_dequant_lm2: empty shape");
    TQ_REQUIRE(aligned16(packed), "tq_dequant_lm2: packed not 16-byte aligned");
    TQ_REQUIRE(n_mat * O * 4 * ((I + 31) / 32) < (int64_t(1) << 32), "tq_dequant_lm2: more than 2^32 octets");
    if (elem_bytes(out_dtype) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant_lm2: out dtype %d", out_dtype);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const LmGeom g = lm_geom(n_mat * O, O, I);
    const unsigned blocks = static_cast<unsigned>(lm_blocks(g.rows * g.per_row));
    if (out_dtype == TQ_BF16)
        k_lm_dequant<__nv_bfloat16><<<blocks, LM_THREADS, 0, st>>>(packed, scales, codebook, g, static_cast<__nv_bfloat16*>(out));
    else
        k_lm_dequant<float><<<blocks, LM_THREADS, 0, st>>>(packed, scales, codebook, g, static_cast<float*>(out));
    return check_launch("tq_dequant_lm2");
}
