// Activation imatrix m_j = alpha * sum_t x_{t,j}^2 ("NeUQI Accuracy
// Validation", opening paragraph: the search is weighted by the activation
// imatrix; tt-stack issue #67, pipeline step 1: H = sum X^T X, whose diagonal
// over T is this) and the per-matrix amax for the NVFP4 global scale.
//
// B200 mapping (HBM-bound column reduction): a block covers 32 x VEC
// consecutive columns (16-byte loads, VEC = 8 bf16 / 4 fp32 per lane) and a
// slice of tokens; its 8 warps walk interleaved tokens with 4 loads in
// flight each.  Squares are summed in fp32 over runs of 32 tokens and folded
// into fp64; the 8 warps are combined in shared memory.  With one token
// slice per column tile the block writes m itself; with several, each
// (slice, column) partial goes to the caller's workspace and the last slice
// block of the tile to finish (atomic ticket) adds the slices in slice order,
// so results do not depend on scheduling.
#include "tq_internal.cuh"

#include <mutex>

namespace tq {

constexpr int IM_THREADS = 256;
constexpr int IM_WARPS = IM_THREADS / 32;

template <typename T> struct VecOf { static constexpr int n = 16 / sizeof(T); };

template <typename T>
__device__ __forceinline__ void load_vec(const T* p, float* out);
template <>
__device__ __forceinline__ void load_vec<uint16_t>(const uint16_t* p, float* out) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    const unsigned u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(u[i] << 16);
        out[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void load_vec<float>(const float* p, float* out) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}

// A 16-byte load as VEC floats.
template <typename T>
__device__ __forceinline__ void unpack_vec(uint4 v, float* out);
template <>
__device__ __forceinline__ void unpack_vec<uint16_t>(uint4 v, float* out) {
    const unsigned u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(u[i] << 16);
        out[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void unpack_vec<float>(uint4 v, float* out) {
    out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
    out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
}

// Token rows in flight per warp in the main loop (loads kept as loaded, 4
// registers each, so many can be in flight).
constexpr int IM_U = 16;

// Adds the squares of U token rows (t, t + IM_WARPS, ...) of this lane's
// VEC columns to acc, all U loads issued before any is used.
template <typename T, int U>
__device__ __forceinline__ void im_rows(const T* base, int64_t t, int64_t ld, float* acc) {
    constexpr int VEC = 16 / sizeof(T);
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) raw[u] = __ldg(reinterpret_cast<const uint4*>(base + (t + u * IM_WARPS) * ld));
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float x[VEC];
        unpack_vec<T>(raw[u], x);
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = __fmaf_rn(x[i], x[i], acc[i]);
    }
}

struct ImGeom {
    int64_t col_tiles, slices, tokens_per_slice;
};

// Token slices per (column tile, matrix): the count that minimises the
// modelled time, waves x (tokens per slice + IM_BLOCK_COST), where a wave is
// IM_RESIDENT blocks per SM (what this kernel's registers allow on sm_100a)
// and a slice holds at least 64 tokens.  Whole waves matter: a last wave
// with few blocks costs as much as a full one.
constexpr int64_t IM_RESIDENT = 4;
constexpr int64_t IM_BLOCK_COST = 16;

inline ImGeom im_geometry(const tq_mat* X) {
    const int vec = X->dtype == TQ_BF16 ? 8 : 4;
    ImGeom g;
    g.col_tiles = (X->cols + 32 * vec - 1) / (32 * vec);
    const int64_t base = g.col_tiles * X->n_mat;
    const int64_t resident = IM_RESIDENT * num_sms();
    const int64_t max_s = max(static_cast<int64_t>(1), (X->rows + 63) / 64);
    int64_t best_s = 1, best_cost = -1;
    for (int64_t s = 1; s <= min(max_s, static_cast<int64_t>(4096)); ++s) {
        const int64_t tps = (X->rows + s - 1) / s;
        const int64_t slices = (X->rows + tps - 1) / tps;
        const int64_t waves = (base * slices + resident - 1) / resident;
        const int64_t cost = waves * (tps + IM_BLOCK_COST);
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_s = s; }
    }
    g.tokens_per_slice = (X->rows + best_s - 1) / best_s;
    g.slices = (X->rows + g.tokens_per_slice - 1) / g.tokens_per_slice;
    return g;
}

inline int64_t im_ticket_bytes(const ImGeom& g, int64_t n_mat) { return ((g.col_tiles * n_mat * 4 + 15) / 16) * 16; }

// Writes one (matrix, column) result: alpha * s rounded once to fp32, added
// to the existing m when accumulating.
__device__ __forceinline__ void im_store(float* __restrict__ m, int64_t idx, double s, double alpha, int accumulate) {
    float v = static_cast<float>(alpha * s);
    if (accumulate) v = __fadd_rn(m[idx], v);
    m[idx] = v;
}

// Each block sums its token slice of one column tile; with one slice it
// writes m itself, otherwise it writes its fp64 partial and the last slice
// block of the (tile, matrix) to finish (atomic ticket) adds the slices'
// partials in slice order and writes m.
template <typename T>
__global__ void __launch_bounds__(IM_THREADS, IM_RESIDENT)
k_imatrix_partial(const T* __restrict__ X, int64_t Tn, int64_t I, int64_t ld, int64_t ms,
                  int64_t tps, double* __restrict__ partial, int64_t n_mat, int64_t slices,
                  unsigned* __restrict__ tickets, float* __restrict__ m, int64_t m_stride, double alpha,
                  int accumulate) {
    constexpr int VEC = VecOf<T>::n;
    __shared__ double red[IM_WARPS][32 * VEC];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t tile = blockIdx.x, slice = blockIdx.y, e = blockIdx.z;
    const int64_t col = tile * 32 * VEC + lane * VEC;
    const int64_t t0 = slice * tps, t1 = min(Tn, t0 + tps);
    const T* base = X + e * ms + col;
    const bool full = col + VEC <= I;

    double accd[VEC];
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) { accd[i] = 0.0; acc[i] = 0.f; }
    int run = 0;
    int64_t t = t0 + wid;
    if (full) {
        // IM_U token rows in flight per warp, then 8 and 4 (short slices keep
        // their loads in flight too), then one at a time.
        for (; t + (IM_U - 1) * IM_WARPS < t1; t += IM_U * IM_WARPS) {
            im_rows<T, IM_U>(base, t, ld, acc);
            run += IM_U;
            if (run >= 32) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) { accd[i] += static_cast<double>(acc[i]); acc[i] = 0.f; }
                run = 0;
            }
        }
        for (; t + 7 * IM_WARPS < t1; t += 8 * IM_WARPS) {
            im_rows<T, 8>(base, t, ld, acc);
            if ((run += 8) >= 32) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) { accd[i] += static_cast<double>(acc[i]); acc[i] = 0.f; }
                run = 0;
            }
        }
        for (; t + 3 * IM_WARPS < t1; t += 4 * IM_WARPS) {
            im_rows<T, 4>(base, t, ld, acc);
            if ((run += 4) >= 32) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) { accd[i] += static_cast<double>(acc[i]); acc[i] = 0.f; }
                run = 0;
            }
        }
        for (; t < t1; t += IM_WARPS) {
            float x[VEC];
            load_vec<T>(base + t * ld, x);
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc[i] = __fmaf_rn(x[i], x[i], acc[i]);
        }
    } else if (col < I) {   // the row's last columns (lanes past its end have nothing to add)
        for (; t < t1; t += IM_WARPS) {
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
                if (col + i < I) {
                    const float v = Elem<T>::load(base + t * ld + i);
                    acc[i] = __fmaf_rn(v, v, acc[i]);
                }
            }
            if (++run >= 32) {
#pragma unroll
                for (int i = 0; i < VEC; ++i) { accd[i] += static_cast<double>(acc[i]); acc[i] = 0.f; }
                run = 0;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[wid][lane * VEC + i] = accd[i] + static_cast<double>(acc[i]);
    __syncthreads();
    for (int c = threadIdx.x; c < 32 * VEC; c += IM_THREADS) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < IM_WARPS; ++w) s += red[w][c];
        const int64_t j = tile * 32 * VEC + c;
        if (j < I) {
            if (slices == 1) im_store(m, e * m_stride + j, 0.0 + s, alpha, accumulate);
            else partial[(slice * n_mat + e) * I + j] = s;
        }
    }
    if (slices == 1) return;   // block-uniform
    __shared__ bool last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        last = atomicAdd(tickets + e * gridDim.x + tile, 1u) == static_cast<unsigned>(slices - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int c = threadIdx.x; c < 32 * VEC; c += IM_THREADS) {   // slices added in order, as one pass would
        const int64_t j = tile * 32 * VEC + c;
        if (j >= I) continue;
        const double* p = partial + e * I + j;
        const int64_t step = n_mat * I;
        double s = 0.0;
        for (int64_t k = 0; k < slices; ++k) s += __ldcg(p + k * step);
        im_store(m, e * m_stride + j, s, alpha, accumulate);
    }
}


// ------------------------------------------------------------------ amax

// One warp per row at a time (warps of all blocks interleaved over the
// matrix's rows), each lane with 4 16-byte loads in flight; the blocks of
// one matrix are sized to fill one wave of resident blocks.
constexpr int AM_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(AM_THREADS)
k_amax(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms, unsigned* __restrict__ amax) {
    constexpr int VEC = VecOf<T>::n;
    const int64_t e = blockIdx.y;
    const T* base = W + e * ms;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (AM_THREADS / 32);
    const int64_t nvec = I / VEC;   // whole 16-byte vectors per row (rows start 16-byte aligned)
    float mx = 0.f;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (AM_THREADS / 32) + (threadIdx.x >> 5); r < O; r += nwarps) {
        const T* row = base + r * ld;
        int64_t c = lane;
        for (; c + 96 < nvec; c += 128) {
            uint4 v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = __ldg(reinterpret_cast<const uint4*>(row + (c + 32 * q) * VEC));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float x[VEC];
                unpack_vec<T>(v[q], x);
#pragma unroll
                for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(x[i]));
            }
        }
        for (; c < nvec; c += 32) {
            float x[VEC];
            load_vec<T>(row + c * VEC, x);
#pragma unroll
            for (int i = 0; i < VEC; ++i) mx = fmaxf(mx, fabsf(x[i]));
        }
        for (int64_t i = nvec * VEC + lane; i < I; i += 32) mx = fmaxf(mx, fabsf(Elem<T>::load(row + i)));
    }
    unsigned u = __reduce_max_sync(FULL, __float_as_uint(mx));
    __shared__ unsigned wmax[AM_THREADS / 32];
    if (lane == 0) wmax[threadIdx.x >> 5] = u;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned v = threadIdx.x < AM_THREADS / 32 ? wmax[threadIdx.x] : 0u;
        v = __reduce_max_sync(FULL, v);
        if (threadIdx.x == 0) atomicMax(amax + e, v);   // non-negative floats order like their bits
    }
}

tq_status launch_amax(const tq_mat* W, float* amax, cudaStream_t st) {
    TQ_REQUIRE(W->n_mat <= 65535, "amax: more than 65535 matrices in one call");
    cudaError_t ce = cudaMemsetAsync(amax, 0, static_cast<size_t>(W->n_mat) * sizeof(float), st);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "amax: %s", cudaGetErrorString(ce));
    int per_sm = 0;
    const bool bf = W->dtype == TQ_BF16;
    if ((bf ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_amax<uint16_t>, AM_THREADS, 0)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_amax<float>, AM_THREADS, 0)) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t slots = static_cast<int64_t>(num_sms()) * per_sm;
    const int64_t per = max(static_cast<int64_t>(1), slots / W->n_mat);   // blocks per matrix
    const int64_t need = (W->rows + AM_THREADS / 32 - 1) / (AM_THREADS / 32);   // one row per warp at most
    const dim3 grid(static_cast<unsigned>(min(per, need)), static_cast<unsigned>(W->n_mat));
    const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0;
    if (bf)
        k_amax<uint16_t><<<grid, AM_THREADS, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->rows, W->cols, W->ld,
                                                      ms, reinterpret_cast<unsigned*>(amax));
    else
        k_amax<float><<<grid, AM_THREADS, 0, st>>>(static_cast<const float*>(W->ptr), W->rows, W->cols, W->ld, ms,
                                                   reinterpret_cast<unsigned*>(amax));
    return check_launch("amax");
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_imatrix_workspace_bytes(const tq_mat* X) {
    if (!X || X->n_mat < 1 || X->rows < 1 || X->cols < 1 || elem_bytes(X->dtype) == 0) return 0;
    const ImGeom g = im_geometry(X);
    if (g.slices == 1) return 16;   // one slice: m is written directly, nothing is kept between blocks
    return static_cast<size_t>(im_ticket_bytes(g, X->n_mat) + g.slices * X->n_mat * X->cols * sizeof(double));
}

TQ_API tq_status tq_imatrix(const tq_mat* X, float* m, int64_t m_stride, float alpha, int32_t accumulate,
                            void* workspace, size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(X, "tq_imatrix X");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(m != nullptr, "tq_imatrix: null m");
    TQ_REQUIRE(m_stride >= X->cols || X->n_mat == 1, "tq_imatrix: m_stride < cols");
    TQ_REQUIRE(workspace != nullptr && aligned16(workspace), "tq_imatrix: workspace null or not 16-byte aligned");
    const size_t need = tq_imatrix_workspace_bytes(X);
    TQ_REQUIRE(workspace_bytes >= need, "tq_imatrix: workspace too small (%zu < %zu bytes)", workspace_bytes, need);
    const ImGeom g = im_geometry(X);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // workspace: the tickets (one per column tile and matrix), then the partials
    const int64_t tick = im_ticket_bytes(g, X->n_mat);
    unsigned* tickets = static_cast<unsigned*>(workspace);
    double* partial = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + tick);
    if (g.slices > 1) {
        const cudaError_t ce = cudaMemsetAsync(tickets, 0, static_cast<size_t>(g.col_tiles * X->n_mat) * 4, st);
        if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_imatrix: %s", cudaGetErrorString(ce));
    }
    const dim3 grid(static_cast<unsigned>(g.col_tiles), static_cast<unsigned>(g.slices), static_cast<unsigned>(X->n_mat));
    const int64_t ms = X->n_mat > 1 ? X->mat_stride : 0;
    const int64_t mst = X->n_mat > 1 ? m_stride : 0;
    if (X->dtype == TQ_BF16)
        k_imatrix_partial<uint16_t><<<grid, IM_THREADS, 0, st>>>(
            static_cast<const uint16_t*>(X->ptr), X->rows, X->cols, X->ld, ms, g.tokens_per_slice, partial, X->n_mat,
            g.slices, tickets, m, mst, static_cast<double>(alpha), accumulate);
    else
        k_imatrix_partial<float><<<grid, IM_THREADS, 0, st>>>(
            static_cast<const float*>(X->ptr), X->rows, X->cols, X->ld, ms, g.tokens_per_slice, partial, X->n_mat,
            g.slices, tickets, m, mst, static_cast<double>(alpha), accumulate);
    return check_launch("imatrix");
}

// ------------------------------------------------------------------ allocation-free variant
//
// Scratch for tq_imatrix_static: a fixed 4 MiB of device memory that every
// GPU loading this library keeps until the process exits.  In host code the
// symbol only names a host-side shadow, so its device address is looked up
// once per device (with that device current) and cached.

constexpr size_t IM_STATIC_BYTES = size_t(4) << 20;
static __device__ __align__(256) double g_im_scratch[IM_STATIC_BYTES / sizeof(double)];

static std::mutex g_im_mu;
static void* g_im_ptr[64];

static tq_status im_static_ptr(void** out) {
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_imatrix_static: %s", cudaGetErrorString(ce));
    if (dev < 0 || dev >= 64) return set_error(TQ_ERR_UNSUPPORTED, "tq_imatrix_static: device %d", dev);
    std::lock_guard<std::mutex> lk(g_im_mu);
    if (!g_im_ptr[dev]) {
        void* p = nullptr;
        ce = cudaGetSymbolAddress(&p, g_im_scratch);
        if (ce != cudaSuccess || !p)
            return set_error(TQ_ERR_CUDA, "tq_imatrix_static: scratch lookup: %s", cudaGetErrorString(ce));
        g_im_ptr[dev] = p;
    }
    *out = g_im_ptr[dev];
    return TQ_OK;
}

TQ_API size_t tq_imatrix_static_capacity(void) { return IM_STATIC_BYTES; }

TQ_API tq_status tq_imatrix_static(const tq_mat* X, float* m, int64_t m_stride, float alpha, int32_t accumulate,
                                   tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(X, "tq_imatrix_static X");
    if (s != TQ_OK) return s;
    const size_t need = tq_imatrix_workspace_bytes(X);
    if (need > IM_STATIC_BYTES)
        return set_error(TQ_ERR_INVALID_ARG,
                         "tq_imatrix_static: this shape needs %zu bytes of scratch, above the fixed %zu; "
                         "use tq_imatrix with a caller-provided workspace",
                         need, IM_STATIC_BYTES);
    void* ws = nullptr;
    if ((s = im_static_ptr(&ws)) != TQ_OK) return s;
    return tq_imatrix(X, m, m_stride, alpha, accumulate, ws, IM_STATIC_BYTES, stream);
}

TQ_API tq_status tq_amax(const tq_mat* W, float* amax, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_amax W");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(amax != nullptr, "tq_amax: null output");
    return launch_amax(W, amax, reinterpret_cast<cudaStream_t>(stream));
}
