// imatrix-weighted reconstruction error per matrix ("Quantize on TT cards:
// CUDA-free GPTQ/LDLQ bfp4 pipeline", tt-stack issue #67, "Risks to measure:
// Precision": proxy error tr(E H E^T) / tr(W H W^T)); with H = diag(m):
//   num = sum_{o,j} m_j (W - What)^2,  den = sum_{o,j} m_j W^2.
//
// B200 mapping (HBM-bound): one thread per octet (8 consecutive weights of a
// group) walking the rows of its slice.  The block's weight tile streams into
// shared memory by bulk copies (TMA, issued by one thread, completed on
// mbarriers) PX_STAGES tiles of PX_RB rows ahead, so about 48 KB per block
// are in flight without costing registers; each thread keeps its 8 imatrix
// weights in registers, dequantizes in registers (no What round trip through
// memory), sums the 8 terms in fp32 and folds them into fp64 per row.  Each block writes an fp64 partial to
// the workspace; the last block of a matrix (atomic ticket) adds the
// partials in block order, so the result is deterministic for a given
// device.
#include "walk.cuh"

namespace tq {

// Fixed block budget, so the workspace size (one fp64 pair per block) does
// not depend on the device.
constexpr int64_t PX_TARGET_BLOCKS = 148 * 8;

inline Walk px_geometry(int64_t n_mat, int64_t O, int64_t I) {
    return walk_geometry(n_mat, O, (I + 7) / 8, PX_TARGET_BLOCKS);
}

// Adds the 8 terms of one octet in fp32 (two interleaved partial sums of
// fp32x2 pairs): m (W - What)^2 and m W^2.
__device__ __forceinline__ void px_terms(const float w[8], const float v[8], const float mm[8], float& sn,
                                         float& sd) {
    float2 an = make_float2(0.f, 0.f), ad = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float2 m2 = make_float2(mm[i], mm[i + 1]);
        const float2 ww = make_float2(w[i], w[i + 1]);
        const float2 d = __fadd2_rn(ww, make_float2(-v[i], -v[i + 1]));
        an = __ffma2_rn(__fmul2_rn(m2, d), d, an);
        ad = __ffma2_rn(__fmul2_rn(m2, ww), ww, ad);
    }
    sn = __fadd_rn(an.x, an.y);
    sd = __fadd_rn(ad.x, ad.y);
}

// Row data in flight: PX_STAGES stages of PX_RB rows of the block's weight
// tile (its full octets: `width` x 16 bytes of bf16 per row), filled by bulk
// copies that one thread issues; the packed bits and scales (a quarter to an
// eighth of the bytes) are loaded by each thread one tile ahead.
constexpr int PX_RB = 4;
constexpr int PX_STAGES = 3;

template <typename T>
inline size_t px_smem_bytes(int width) {
    return 64 + static_cast<size_t>(PX_STAGES) * PX_RB * width * sizeof(T) * 8;
}

// Set when a wait for a bulk copy gave up (the results are then invalid);
// read and cleared by tq_sync.
static __device__ unsigned g_px_fault;

template <int FMT, typename T>
__global__ void __launch_bounds__(256)
k_proxy(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms, const uint8_t* __restrict__ packed,
        const void* scales, const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
        const float* __restrict__ m, int64_t m_stride, int64_t rps, double* __restrict__ part_out,
        unsigned* __restrict__ tickets, double* __restrict__ num, double* __restrict__ den) {
    using F = FmtTraits<FMT>;
    constexpr int OB = static_cast<int>(sizeof(T)) * 8;   // bytes of one octet of W
    extern __shared__ __align__(128) uint8_t px_smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(px_smem);
    uint8_t* tiles = px_smem + 64;
    const int width = static_cast<int>(blockDim.x), t = static_cast<int>(threadIdx.x);
    const size_t row_bytes = static_cast<size_t>(width) * OB, stage_bytes = PX_RB * row_bytes;

    const int64_t G = (I + F::group - 1) / F::group;
    const int64_t e = blockIdx.z;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * width;
    const int64_t c = c0 + t;
    const int64_t nblk = static_cast<int64_t>(gridDim.x) * gridDim.y;
    const int64_t bid = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
    const int nwarps = static_cast<int>(blockDim.x >> 5);
    const int64_t C = (I + 7) >> 3, CF = I >> 3;   // octets per row, full octets per row
    const uint32_t seg = static_cast<uint32_t>(max(static_cast<int64_t>(0), min(CF - c0, static_cast<int64_t>(width))) * OB);
    const int64_t o0 = static_cast<int64_t>(blockIdx.y) * rps, o1 = min(O, o0 + rps);
    const int64_t ntiles = (o1 - o0 + PX_RB - 1) / PX_RB;
    const T* wtile = W + e * ms + c0 * 8;   // row o of the tile at wtile + o * ld

    if (t == 0) {
#pragma unroll
        for (int st = 0; st < PX_STAGES; ++st) mbar_init(&bars[st], 1);
        mbar_init_fence();
    }
    __syncthreads();
    auto issue = [&](int64_t tile) {
        const int st = static_cast<int>(tile % PX_STAGES);
        const int64_t r0 = o0 + tile * PX_RB;
        const int rows = static_cast<int>(min(static_cast<int64_t>(PX_RB), o1 - r0));
        mbar_expect_tx(&bars[st], static_cast<uint32_t>(rows) * seg);
        if (seg)
            for (int r = 0; r < rows; ++r)
                bulk_g2s(tiles + st * stage_bytes + r * row_bytes, wtile + (r0 + r) * ld, seg, &bars[st]);
    };
    if (t == 0)
        for (int64_t tile = 0; tile < min(static_cast<int64_t>(PX_STAGES), ntiles); ++tile) issue(tile);

    const bool active = c < C;
    const int64_t k = c >> F::lg;
    const int oct = static_cast<int>(c & ((1 << F::lg) - 1));
    const int64_t j = c << 3;
    const int n = active ? static_cast<int>(min(static_cast<int64_t>(8), I - j)) : 0;
    float mm[8];
    {
        Oct<float> mo;
        mo.load(m + e * m_stride + j, n);
        mo.get(mm);
    }
    const float g = (FMT == TQ_NVFP4_G16 && active) ? __ldg(gs + e) : 0.f;
    const int64_t gbase = e * O * G + k;
    OctQ qn[PX_RB];
#pragma unroll
    for (int r = 0; r < PX_RB; ++r)
        if (active && o0 + r < o1) qn[r] = load_q<FMT>(packed, scales, zeros, gbase + (o0 + r) * G, oct);
    double an = 0.0, ad = 0.0;
    int64_t tile = 0;
    for (; tile < ntiles; ++tile) {
        const int st = static_cast<int>(tile % PX_STAGES);
        const int64_t r0 = o0 + tile * PX_RB;
        OctQ qc[PX_RB];
#pragma unroll
        for (int r = 0; r < PX_RB; ++r) qc[r] = qn[r];
#pragma unroll
        for (int r = 0; r < PX_RB; ++r)   // next tile's codes and scales, while this one is worked on
            if (active && r0 + PX_RB + r < o1) qn[r] = load_q<FMT>(packed, scales, zeros, gbase + (r0 + PX_RB + r) * G, oct);
        const bool got = mbar_wait(&bars[st], static_cast<uint32_t>((tile / PX_STAGES) & 1));
        if (active && got) {
#pragma unroll
            for (int r = 0; r < PX_RB; ++r) {
                if (r0 + r >= o1) break;
                Oct<T> ow;
                if (n == 8) {
                    const uint4* src = reinterpret_cast<const uint4*>(tiles + st * stage_bytes + r * row_bytes + t * OB);
                    if constexpr (sizeof(T) == 2) {
                        ow.v = src[0];
                    } else {
                        const uint4 a = src[0], b = src[1];
                        ow.a = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w));
                        ow.b = make_float4(__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w));
                    }
                } else {
                    ow.load(W + e * ms + (r0 + r) * ld + j, n);   // the row's last, partial octet
                }
                float w[8], v[8], sn, sd;
                ow.get(w);
                dec_oct<FMT>(qc[r], g, v);
                px_terms(w, v, mm, sn, sd);
                an += static_cast<double>(sn);
                ad += static_cast<double>(sd);
            }
        }
        if (__syncthreads_or(!got)) break;   // every thread has read the stage (or a wait gave up)
        if (t == 0 && tile + PX_STAGES < ntiles) {
            fence_proxy_async_smem();
            issue(tile + PX_STAGES);
        }
    }
    if (tile < ntiles) {   // a wait gave up: flag it and let the copies in flight land before exiting
        if (t == 0) {
            atomicOr(&g_px_fault, 1u);
            for (int64_t u = tile; u < min(ntiles, tile + PX_STAGES); ++u)
                mbar_wait(&bars[u % PX_STAGES], static_cast<uint32_t>((u / PX_STAGES) & 1));
        }
        an = ad = 0.0;
    }
    // block reduction in fp64, fixed order
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        an += __shfl_xor_sync(FULL, an, off);
        ad += __shfl_xor_sync(FULL, ad, off);
    }
    __shared__ double sw[2][8];
    __shared__ bool last;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) { sw[0][wid] = an; sw[1][wid] = ad; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double bn = 0.0, bd = 0.0;
        for (int i = 0; i < nwarps; ++i) { bn += sw[0][i]; bd += sw[1][i]; }
        part_out[(e * nblk + bid) * 2] = bn;
        part_out[(e * nblk + bid) * 2 + 1] = bd;
        __threadfence();
        last = atomicAdd(tickets + e, 1u) == static_cast<unsigned>(nblk - 1);
    }
    __syncthreads();
    if (last) {   // the matrix's last block adds the partials: fixed strides, fixed tree
        __threadfence();
        double tn = 0.0, td = 0.0;
        for (int64_t b = threadIdx.x; b < nblk; b += blockDim.x) {
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
            for (int i = 0; i < nwarps; ++i) { bn += sw[0][i]; bd += sw[1][i]; }
            num[e] = bn;
            den[e] = bd;
        }
    }
}

// At most one wave of resident blocks (slices per matrix rounded down, so no
// second partial wave) and at most the block count the workspace is sized
// for (PX_TARGET_BLOCKS, rounded up: never fewer slots than blocks).
template <int FMT, typename T>
void launch_proxy(const tq_mat* W, int64_t ms, const uint8_t* packed, const void* scales, const uint8_t* zeros,
                  const float* gs, const float* m, int64_t mst, double* parts, unsigned* tickets, double* num,
                  double* den, cudaStream_t st) {
    const int64_t cols = (W->cols + 7) / 8;
    Walk pg = walk_geometry(W->n_mat, W->rows, cols, 1);
    const size_t smem = px_smem_bytes<T>(static_cast<int>(pg.width));
    cudaFuncSetAttribute(k_proxy<FMT, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_proxy<FMT, T>, static_cast<int>(pg.width), smem) !=
            cudaSuccess || per_sm < 1)
        per_sm = 1;
    pg = walk_geometry(W->n_mat, W->rows, cols, min(PX_TARGET_BLOCKS, static_cast<int64_t>(num_sms()) * per_sm),
                       false);
    const dim3 grid(static_cast<unsigned>(pg.cblocks), static_cast<unsigned>(pg.slices), static_cast<unsigned>(W->n_mat));
    k_proxy<FMT, T><<<grid, static_cast<unsigned>(pg.width), smem, st>>>(static_cast<const T*>(W->ptr), W->rows,
                                                                         W->cols, W->ld, ms, packed, scales, zeros, gs,
                                                                         m, mst, pg.rps, parts, tickets, num, den);
}

// Reads and clears the bulk-copy wait flag of the proxy kernels (tq_sync).
bool take_proxy_fault() {
    unsigned f = 0;
    const unsigned zero = 0;
    if (cudaMemcpyFromSymbol(&f, g_px_fault, sizeof f) != cudaSuccess) return false;
    if (f) cudaMemcpyToSymbol(g_px_fault, &zero, sizeof zero);
    return f != 0;
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_proxy_workspace_bytes(const tq_mat* W, int32_t fmt) {
    const int64_t g = group_of(fmt);
    if (!W || g == 0 || W->n_mat < 1 || W->rows < 1 || W->cols < 1) return 0;
    const Walk pg = px_geometry(W->n_mat, W->rows, W->cols);
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
    TQ_REQUIRE(W->n_mat <= 65535, "tq_proxy_error: more than 65535 matrices in one call");
    const int64_t tick = ((W->n_mat * 4 + 15) / 16) * 16;
    unsigned* tickets = static_cast<unsigned*>(workspace);
    double* parts = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + tick);
    cudaError_t ce = cudaMemsetAsync(tickets, 0, static_cast<size_t>(W->n_mat) * 4, st);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_proxy_error: %s", cudaGetErrorString(ce));
    const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0;
    const int64_t mst = W->n_mat > 1 ? m_stride : 0;
    const bool bf = W->dtype == TQ_BF16;
    if (fmt == TQ_INT3_G64_SYM)
        bf ? launch_proxy<TQ_INT3_G64_SYM, uint16_t>(W, ms, packed, scales, zeros, global_scale, m, mst, parts, tickets, num, den, st)
           : launch_proxy<TQ_INT3_G64_SYM, float>(W, ms, packed, scales, zeros, global_scale, m, mst, parts, tickets, num, den, st);
    else if (fmt == TQ_INT4_G128_ASYM)
        bf ? launch_proxy<TQ_INT4_G128_ASYM, uint16_t>(W, ms, packed, scales, zeros, global_scale, m, mst, parts, tickets, num, den, st)
           : launch_proxy<TQ_INT4_G128_ASYM, float>(W, ms, packed, scales, zeros, global_scale, m, mst, parts, tickets, num, den, st);
    else
        bf ? launch_proxy<TQ_NVFP4_G16, uint16_t>(W, ms, packed, scales, zeros, global_scale, m, mst, parts, tickets, num, den, st)
           : launch_proxy<TQ_NVFP4_G16, float>(W, ms, packed, scales, zeros, global_scale, m, mst, parts, tickets, num, den, st);
    return check_launch("tq_proxy_error");
}
