// imatrix-weighted reconstruction error per matrix ("Quantize on TT cards:
// CUDA-free GPTQ/LDLQ bfp4 pipeline", tt-stack issue #67, "Risks to measure:
// Precision": proxy error tr(E H E^T) / tr(W H W^T)); with H = diag(m):
//   num = sum_{o,j} m_j (W - What)^2,  den = sum_{o,j} m_j W^2.
//
// B200 mapping (HBM-bound): one thread per 16 consecutive weights of a group;
// it dequantizes its packed codes in registers (no What round trip through
// memory), reads W with 16-byte loads and m (L2-resident, shared by every
// row), sums the 16 terms in fp32 and folds them into fp64.  Each block
// writes an fp64 partial to the workspace; the last block of a matrix (atomic
// ticket) adds the partials in block order, so the result is deterministic.
#include "group_pack.cuh"

namespace tq {


constexpr int PX_THREADS = 256;

// Grid: x = 256-chunk column tiles (a chunk = 16 weights of one group),
// y = row slices, z = matrices.  Each thread loads its chunk's 16 imatrix
// weights once and walks the rows of its slice.
struct PxGeom { int64_t cblocks, slices, rps; };

inline PxGeom px_geometry(int64_t n_mat, int64_t O, int64_t I) {
    PxGeom g;
    const int64_t C = (I + 15) / 16;
    g.cblocks = (C + PX_THREADS - 1) / PX_THREADS;
    int64_t s = (16 * 148 + g.cblocks * n_mat - 1) / (g.cblocks * n_mat);
    s = s < 1 ? 1 : (s > O ? O : s);
    g.rps = (O + s - 1) / s;
    g.slices = (O + g.rps - 1) / g.rps;
    return g;
}

template <typename T>
__device__ __forceinline__ void load16(const T* p, bool full, int n, float w[16]);
template <>
__device__ __forceinline__ void load16<uint16_t>(const uint16_t* p, bool full, int n, float w[16]) {
    if (full) {
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
template <>
__device__ __forceinline__ void load16<float>(const float* p, bool full, int n, float w[16]) {
    if (full) {
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

template <typename T>
__global__ void __launch_bounds__(PX_THREADS)
k_proxy(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms, const uint8_t* __restrict__ packed,
        int fmt, const void* scales, const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
        const float* __restrict__ m, int64_t m_stride, int64_t rps, double* __restrict__ part_out,
        unsigned* __restrict__ tickets, double* __restrict__ num, double* __restrict__ den) {
    const int lg = fmt == TQ_INT3_G64_SYM ? 2 : (fmt == TQ_INT4_G128_ASYM ? 3 : 0);   // log2(chunks per group)
    const int64_t G = (I + (16 << lg) - 1) >> (4 + lg);
    const int64_t C = (I + 15) >> 4;
    const int64_t e = blockIdx.z;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * PX_THREADS + threadIdx.x;
    const int64_t nblk = static_cast<int64_t>(gridDim.x) * gridDim.y;
    const int64_t bid = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
    double an = 0.0, ad = 0.0;
    if (c < C) {
        const int64_t k = c >> lg;
        const int part = static_cast<int>(c & ((1 << lg) - 1));
        const int64_t j = c << 4;
        const int n = static_cast<int>(min(static_cast<int64_t>(16), I - j));
        const bool full = n == 16;
        float mm[16];
        const float* mp = m + e * m_stride + j;
        if (full) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 a4 = __ldg(reinterpret_cast<const float4*>(mp) + i);
                mm[4 * i] = a4.x; mm[4 * i + 1] = a4.y; mm[4 * i + 2] = a4.z; mm[4 * i + 3] = a4.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) mm[i] = i < n ? __ldg(mp + i) : 0.f;
        }
        const int64_t o0 = static_cast<int64_t>(blockIdx.y) * rps;
        const int64_t o1 = min(O, o0 + rps);
        for (int64_t o = o0; o < o1; ++o) {
            float v[16], w[16];
            dq_unit(fmt, packed, scales, zeros, gs, O * G, (e * O + o) * G + k, part, v);
            load16<T>(W + e * ms + o * ld + j, full, n, w);
            float sn = 0.f, sd = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float d = __fsub_rn(w[i], v[i]);
                sn = __fmaf_rn(__fmul_rn(mm[i], d), d, sn);
                sd = __fmaf_rn(__fmul_rn(mm[i], w[i]), w[i], sd);
            }
            an += static_cast<double>(sn);
            ad += static_cast<double>(sd);
        }
    }
    // block reduction in fp64, fixed order
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        an += __shfl_xor_sync(FULL, an, off);
        ad += __shfl_xor_sync(FULL, ad, off);
    }
    __shared__ double sw[2][PX_THREADS / 32];
    __shared__ bool last;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) { sw[0][wid] = an; sw[1][wid] = ad; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double bn = 0.0, bd = 0.0;
        for (int i = 0; i < PX_THREADS / 32; ++i) { bn += sw[0][i]; bd += sw[1][i]; }
        part_out[(e * nblk + bid) * 2] = bn;
        part_out[(e * nblk + bid) * 2 + 1] = bd;
        __threadfence();
        last = atomicAdd(tickets + e, 1u) == static_cast<unsigned>(nblk - 1);
    }
    __syncthreads();
    if (last) {   // the matrix's last block adds the partials: fixed strides, fixed tree
        __threadfence();
        double tn = 0.0, td = 0.0;
        for (int64_t b = threadIdx.x; b < nblk; b += PX_THREADS) {
            tn += __ldcg(part_out + (e * nblk + b) * 2);
            td += __ldcg(part_out + (e * nblk + b) * 2 + 1);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            tn += __shfl_xor_sync(FULL, tn, off);
            td += __shfl_xor_sync(FULL, td, off);
        }
        __syncthreads();
        if (lane == 0) { sw[0][wid] = tn; sw[1][wid] = td; }
        __syncthreads();
        if (threadIdx.x == 0) {
            double bn = 0.0, bd = 0.0;
            for (int i = 0; i < PX_THREADS / 32; ++i) { bn += sw[0][i]; bd += sw[1][i]; }
            num[e] = bn;
            den[e] = bd;
        }
    }
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_proxy_workspace_bytes(const tq_mat* W, int32_t fmt) {
    const int64_t g = group_of(fmt);
    if (!W || g == 0 || W->n_mat < 1 || W->rows < 1 || W->cols < 1) return 0;
    const PxGeom pg = px_geometry(W->n_mat, W->rows, W->cols);
    const int64_t tick = ((W->n_mat * 4 + 15) / 16) * 16;
    return static_cast<size_t>(tick + W->n_mat * pg.cblocks * pg.slices * 16);
}

TQ_API tq_status tq_proxy_error(const tq_mat* W, const uint8_t* packed, int32_t fmt, const void* scales,
                                const uint8_t* zeros, const float* global_scale, const float* m,
                                int64_t m_stride, double* num, double* den, void* workspace,
                                size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_proxy_error W");
    if (s != TQ_OK) return s;
    const int64_t g = group_of(fmt);
    if (g == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_proxy_error: unknown format %d", fmt);
    TQ_REQUIRE(packed && scales && m && num && den, "tq_proxy_error: null pointer");
    TQ_REQUIRE(aligned16(packed) && aligned16(m), "tq_proxy_error: packed/m not 16-byte aligned");
    TQ_REQUIRE(W->n_mat == 1 || m_stride == 0 || (m_stride >= W->cols && m_stride % 4 == 0),
               "tq_proxy_error: m_stride must be 0 or a multiple of 4 >= cols");
    TQ_REQUIRE(fmt != TQ_INT4_G128_ASYM || zeros != nullptr, "tq_proxy_error: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_proxy_error: NVFP4 needs global_scale");
    TQ_REQUIRE(workspace && aligned16(workspace), "tq_proxy_error: workspace null or not 16-byte aligned");
    const size_t need = tq_proxy_workspace_bytes(W, fmt);
    TQ_REQUIRE(workspace_bytes >= need, "tq_proxy_error: workspace too small (%zu < %zu)", workspace_bytes, need);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const PxGeom pg = px_geometry(W->n_mat, W->rows, W->cols);
    const int64_t tick = ((W->n_mat * 4 + 15) / 16) * 16;
    unsigned* tickets = static_cast<unsigned*>(workspace);
    double* parts = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + tick);
    cudaError_t ce = cudaMemsetAsync(tickets, 0, static_cast<size_t>(W->n_mat) * 4, st);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_proxy_error: %s", cudaGetErrorString(ce));
    const dim3 grid(static_cast<unsigned>(pg.cblocks), static_cast<unsigned>(pg.slices), static_cast<unsigned>(W->n_mat));
    const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0;
    const int64_t mst = W->n_mat > 1 ? m_stride : 0;
    if (W->dtype == TQ_BF16)
        k_proxy<uint16_t><<<grid, PX_THREADS, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->rows, W->cols, W->ld, ms,
                                                      packed, fmt, scales, zeros, global_scale, m, mst, pg.rps, parts,
                                                      tickets, num, den);
    else
        k_proxy<float><<<grid, PX_THREADS, 0, st>>>(static_cast<const float*>(W->ptr), W->rows, W->cols, W->ld, ms,
                                                   packed, fmt, scales, zeros, global_scale, m, mst, pg.rps, parts,
                                                   tickets, num, den);
    return check_launch("tq_proxy_error");
}
