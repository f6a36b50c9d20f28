// Proxy error with the full Hessian H = X^T X of the calibration activations
// ("Quantize on TT cards: CUDA-free GPTQ/LDLQ bfp4 pipeline", tt-stack issue
// #67, "Risks to measure: Precision": the gate compares tr(E H E^T) /
// tr(W H W^T), E = W - What), on the tensor cores and without forming H:
//   tr(E H E^T) = sum_t sum_o (E x_t)_o^2 = ||X E^T||_F^2,  tr(W H W^T) = ||X W^T||_F^2.
//
// Both products are GEMMs with M = T tokens, N = O rows, K = I, all operands
// K-major (rows of X, E and W are contiguous in I), computed in one pass over
// X: every 64-column chunk of X is loaded once and multiplied by the chunk of
// E and the chunk of W, into two fp32 accumulators.  E = W - What (fp64, then
// rounded once to fp32) enters as two bf16 pieces E1 = bf16(E), E2 =
// bf16(E - E1), laid side by side along K ([E1 | E2], each padded to a
// multiple of 64 columns): E1 + E2 carries 16 significant bits of E (relative
// error at most 2^-16, within the fp32 accumulation's own bound once K >= 512;
// a third piece would make it exact and cost a third more MMAs).  W
// (bf16) is an exact operand as it is.  The epilogue squares and sums both
// accumulator tiles in fp64; nothing of the products is stored.
//
// B200 mapping (one CTA per 128 x 256 tile of the products, 4 warps, 1 CTA
// per SM): TMA (128-byte swizzle, 64-column K boxes) fills a 3-slot ring of X
// chunks (16 KB) and a 5-slot ring of E1 / E2 / W chunks (32 KB); one thread
// issues tcgen05.mma.cta_group::1.kind::f16 (bf16 in, fp32 accumulate, both
// operands K-major) into TMEM columns 0-255 (X E^T) and 256-511 (X W^T); the 4
// warps read TMEM (tcgen05.ld), add the squares of their rows in fp64, and
// the CTA writes one partial per product; a last kernel adds the partials of
// each matrix in order (deterministic).  Waits on mbarriers are bounded: one
// that runs out makes the CTA write NaN partials and count the timeout.
#include <cuda.h>

#include <mutex>

#include "walk.cuh"

namespace tq {

constexpr int PF_M = 128, PF_N = 256, PF_BK = 64, PF_THREADS = 128;
constexpr int PF_PIECES = 2;                               // bf16 pieces of E
constexpr int PF_OPS = PF_PIECES + 1;                      // B operands per X chunk: E1, E2, W
constexpr int PF_XS = 3, PF_BS = 5;                        // ring slots
constexpr int PF_X_BYTES = PF_M * PF_BK * 2;               // 16 KB
constexpr int PF_B_BYTES = PF_N * PF_BK * 2;               // 32 KB
constexpr int PF_RING_BYTES = PF_XS * PF_X_BYTES + PF_BS * PF_B_BYTES;
constexpr int PF_NBAR = 2 * PF_XS + 2 * PF_BS + 1;
constexpr int PF_SMEM_BYTES = PF_RING_BYTES + 1024 + 256;
constexpr unsigned PF_WAIT_LIMIT = DEFAULT_WAIT_LIMIT;
static_assert(PF_NBAR * 8 + 4 + 6 * 4 <= 192 && PF_RING_BYTES + 1023 + 256 <= PF_SMEM_BYTES, "shared layout");

__device__ unsigned g_pf_timeouts = 0;

__device__ __forceinline__ uint32_t pf_smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool pf_wait(uint32_t bar, unsigned parity, unsigned limit = PF_WAIT_LIMIT) {
    for (unsigned it = 0; it < limit; ++it) {
        unsigned ok;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    atomicAdd(&g_pf_timeouts, 1u);
    return false;
}

__device__ __forceinline__ void pf_tma_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void pf_arm(uint32_t bar, int bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void pf_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// K-major operand, 128-byte swizzle: rows of 64 K-elements (128 B), groups of
// 8 rows 1024 B apart (SBO); LBO unused (1).
__device__ __forceinline__ uint64_t pf_desc(uint32_t addr) {
    return (static_cast<uint64_t>((addr >> 4) & 0x3fffu)) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16, fp32 accumulate, bf16 A and B, both K-major, M = 128, N = 256.
constexpr uint32_t PF_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(PF_N >> 3) << 17) |
                              (static_cast<uint32_t>(PF_M >> 4) << 24);

struct PfArgs {
    int kx;              // 64-column chunks of X (Ip / 64); E piece p of chunk c at E column p Ip + 64 c
    int tiles_m, tiles_n;
    double* pn;          // [n_mat][tiles_m * tiles_n] partials of ||X E^T||^2
    double* pd;          // the same for ||X W^T||^2
    unsigned wait_limit; // try_wait rounds of the ring waits
};

__device__ __forceinline__ double pf_tile_sq(uint32_t taddr) {
    double sq = 0.0;
#pragma unroll 1
    for (int c0 = 0; c0 < PF_N; c0 += 32) {
        uint32_t r[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
            "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
              "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
              "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(taddr + static_cast<uint32_t>(c0)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const double v = static_cast<double>(__uint_as_float(r[i]));
            sq = __fma_rn(v, v, sq);
        }
    }
    return sq;
}

__global__ void __launch_bounds__(PF_THREADS, 1)
k_pf_gemm(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap emap,
          const __grid_constant__ CUtensorMap wmap, const __grid_constant__ PfArgs a) {
    const int tm = static_cast<int>(blockIdx.x) % a.tiles_m, tn = static_cast<int>(blockIdx.x) / a.tiles_m;
    const int e = static_cast<int>(blockIdx.y);
    extern __shared__ uint8_t pf_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pf_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PF_RING_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + PF_NBAR);
    // progress: [0] X chunks armed, [1] X chunks consumed, [2] B chunks armed, [3] B chunks consumed,
    //           [4] every wait succeeded, [5] all MMAs complete
    int* progress = reinterpret_cast<int*>(tmem_slot + 1);
    double* red = reinterpret_cast<double*>(smem + PF_RING_BYTES + 192);
    const uint32_t xs0 = pf_smem_u32(smem), bs0 = xs0 + PF_XS * PF_X_BYTES;
    const uint32_t xfull = pf_smem_u32(bars), xempty = xfull + 8 * PF_XS;
    const uint32_t bfull = xempty + 8 * PF_XS, bempty = bfull + 8 * PF_BS, done = bempty + 8 * PF_BS;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nc = a.kx, nb = PF_OPS * nc;

    if (threadIdx.x == 0) {
        for (int i = 0; i < PF_NBAR; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(xfull + 8 * i) : "memory");
        for (int i = 0; i < 6; ++i) progress[i] = 0;
        progress[4] = 1;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(pf_smem_u32(tmem_slot)),
                     "r"(2 * PF_N));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {   // TMA producer: chunk c brings X_c, then E1_c, E2_c, W_c
        bool ok = true;
        for (int j = 0; j < nb && ok; ++j) {
            const int c = j / PF_OPS, p = j - c * PF_OPS;
            if (p == 0) {
                const int xs = c % PF_XS;
                if (!(ok = pf_wait(xempty + 8 * xs, ((c / PF_XS) & 1) ^ 1, a.wait_limit))) break;
                pf_arm(xfull + 8 * xs, PF_X_BYTES);
                pf_tma_3d(xs0 + xs * PF_X_BYTES, &xmap, xfull + 8 * xs, c * PF_BK, tm * PF_M, e);
                progress[0] = c + 1;
            }
            const int bs = j % PF_BS;
            if (!(ok = pf_wait(bempty + 8 * bs, ((j / PF_BS) & 1) ^ 1, a.wait_limit))) break;
            pf_arm(bfull + 8 * bs, PF_B_BYTES);
            if (p < PF_PIECES)
                pf_tma_3d(bs0 + bs * PF_B_BYTES, &emap, bfull + 8 * bs, (p * nc + c) * PF_BK, tn * PF_N, e);
            else
                pf_tma_3d(bs0 + bs * PF_B_BYTES, &wmap, bfull + 8 * bs, c * PF_BK, tn * PF_N, e);
            progress[2] = j + 1;
        }
        if (!ok) progress[4] = 0;
    } else if (warp == 1 && lane == 0) {   // MMA issuer
        bool ok = true;
        for (int j = 0; j < nb && ok; ++j) {
            const int c = j / PF_OPS, p = j - c * PF_OPS, xs = c % PF_XS, bs = j % PF_BS;
            if (p == 0 && !(ok = pf_wait(xfull + 8 * xs, (c / PF_XS) & 1, a.wait_limit))) break;
            if (!(ok = pf_wait(bfull + 8 * bs, (j / PF_BS) & 1, a.wait_limit))) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sa = xs0 + xs * PF_X_BYTES, sb = bs0 + bs * PF_B_BYTES;
            const uint32_t d = tmem + (p < PF_PIECES ? 0u : static_cast<uint32_t>(PF_N));
            const bool first = c == 0 && (p == 0 || p == PF_PIECES);   // the first product into each accumulator
#pragma unroll
            for (int kk = 0; kk < PF_BK / 16; ++kk) {   // 16 K-elements = 32 bytes of each row
                const uint32_t acc = (!first || kk != 0) ? 1u : 0u;
                asm volatile(
                    "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d),
                    "l"(pf_desc(sa + 32 * kk)), "l"(pf_desc(sb + 32 * kk)), "r"(PF_IDESC), "r"(acc)
                    : "memory");
            }
            pf_commit(bempty + 8 * bs);
            progress[3] = j + 1;
            if (p == PF_OPS - 1) {
                pf_commit(xempty + 8 * xs);
                progress[1] = c + 1;
            }
        }
        if (!ok) progress[4] = 0;
        pf_commit(done);
    }

    if (warp == 1 && lane == 0) progress[5] = pf_wait(done, 0) ? 1 : 0;
    __syncthreads();
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // epilogue: this thread's row of the tile (token tm * 128 + 32 warp + lane), squares in fp64
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    double sn = pf_tile_sq(trow), sd = pf_tile_sq(trow + PF_N);
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        sn += __shfl_xor_sync(FULL, sn, off);
        sd += __shfl_xor_sync(FULL, sd, off);
    }
    if (lane == 0) { red[warp] = sn; red[4 + warp] = sd; }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = progress[4] != 0 && progress[5] != 0;
        const double nan = __longlong_as_double(0x7ff8000000000000ll);
        const int64_t slot = static_cast<int64_t>(e) * a.tiles_m * a.tiles_n + blockIdx.x;
        a.pn[slot] = ok ? ((red[0] + red[1]) + red[2]) + red[3] : nan;
        a.pd[slot] = ok ? ((red[4] + red[5]) + red[6]) + red[7] : nan;
        // after a timeout: wait (bounded) for the copies armed but never consumed
        for (int c = progress[1]; c < progress[0]; ++c)
            if (!pf_wait(xfull + 8 * (c % PF_XS), (c / PF_XS) & 1)) break;
        for (int j = progress[3]; j < progress[2]; ++j)
            if (!pf_wait(bfull + 8 * (j % PF_BS), (j / PF_BS) & 1)) break;
        if (progress[5] == 0) pf_wait(done, 0);   // the committed MMAs, before TMEM is freed
    }
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * PF_N));
}

// E = W - What in PF_PIECES bf16 pieces, rows of [E1 | E2], each Ip columns (zeros past I).
template <int FMT, typename T>
__global__ void k_pf_prep(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms,
                          const uint8_t* __restrict__ packed, const void* __restrict__ scales,
                          const uint8_t* __restrict__ zeros, const float* __restrict__ gs, int64_t n_mat, int64_t Ip,
                          __nv_bfloat16* __restrict__ ep) {
    using F = FmtTraits<FMT>;
    const int64_t G = (I + F::group - 1) / F::group, Cp = Ip >> 3, total = n_mat * O * Cp;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = t / Cp, c = t - row * Cp, e = row / O, o = row - e * O;
        const int64_t j = c << 3;
        float w[8], v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) { w[i] = 0.f; v[i] = 0.f; }
        if (j < I) {
            const int n = static_cast<int>(min(static_cast<int64_t>(8), I - j));
            Oct<T> oc;
            oc.load(W + e * ms + o * ld + j, n);
            oc.get(w);
            const int64_t k = j / F::group;
            const int oct = static_cast<int>((j % F::group) >> 3);
            const QPtr<FMT> qp(packed, scales, zeros, row * G + k, G);
            dec_oct<FMT>(load_q<FMT>(qp, oct), FMT == TQ_NVFP4_G16 ? __ldg(gs + e) : 0.f, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) if (i >= n) { w[i] = 0.f; v[i] = 0.f; }
        }
        uint32_t pc[PF_PIECES][4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
#pragma unroll
            for (int q = 0; q < PF_PIECES; ++q) pc[q][h] = 0;
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int i = 2 * h + b;
                float r = __double2float_rn(static_cast<double>(w[i]) - static_cast<double>(v[i]));
#pragma unroll
                for (int q = 0; q < PF_PIECES; ++q) {   // piece q = bf16 of what the earlier pieces left (exact)
                    const __nv_bfloat16 a = __float2bfloat16_rn(r);
                    r = __fsub_rn(r, __bfloat162float(a));
                    pc[q][h] |= static_cast<uint32_t>(__bfloat16_as_ushort(a)) << (16 * b);
                }
            }
        }
        __nv_bfloat16* dst = ep + row * PF_PIECES * Ip + j;
#pragma unroll
        for (int q = 0; q < PF_PIECES; ++q)
            *reinterpret_cast<uint4*>(dst + q * Ip) = make_uint4(pc[q][0], pc[q][1], pc[q][2], pc[q][3]);
    }
}

__global__ void k_pf_reduce(const double* __restrict__ pn, const double* __restrict__ pd, int64_t tiles,
                            double* __restrict__ num, double* __restrict__ den) {
    const int64_t e = blockIdx.x;
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int64_t t = 0; t < tiles; ++t) { a += pn[e * tiles + t]; b += pd[e * tiles + t]; }
        num[e] = a;
        den[e] = b;
    }
}

using PfEncode = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PfEncode pf_encode() {
    static std::once_flag once;
    static PfEncode fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PfEncode>(p);
    });
    return fn;
}

// 3D bf16 tensor map {cols, rows, n_mat}, box {64, box_rows, 1}, 128-byte swizzle.
static bool pf_map(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int64_t n_mat, int64_t ld,
                   int64_t ms, int box_rows) {
    PfEncode enc = pf_encode();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(n_mat)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2), static_cast<cuuint64_t>(ms * 2)};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1}, es[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool proxy_full_take_timeouts() {
    unsigned n = 0;
    if (cudaMemcpyFromSymbol(&n, g_pf_timeouts, sizeof(n)) != cudaSuccess || n == 0) return false;
    const unsigned zero = 0;
    cudaMemcpyToSymbol(g_pf_timeouts, &zero, sizeof(zero));
    return true;
}

static int64_t pf_ip(int64_t I) { return (I + 63) / 64 * 64; }
static int64_t pf_tiles(const tq_mat* X, const tq_mat* W) {
    return ((X->rows + PF_M - 1) / PF_M) * ((W->rows + PF_N - 1) / PF_N);
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_proxy_full_workspace_bytes(const tq_mat* X, const tq_mat* W) {
    if (!X || !W || W->n_mat < 1 || W->rows < 1 || W->cols < 1) return 0;
    const int64_t ep = W->n_mat * W->rows * PF_PIECES * pf_ip(W->cols) * 2;
    const int64_t parts = 2 * W->n_mat * pf_tiles(X, W) * 8;
    return static_cast<size_t>((ep + 255) / 256 * 256 + parts);
}

TQ_API tq_status tq_proxy_error_full(const tq_mat* X, const tq_mat* W, const uint8_t* packed, int32_t fmt,
                                     const void* scales, const uint8_t* zeros, const float* global_scale,
                                     double* num, double* den, void* workspace, size_t workspace_bytes,
                                     tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_proxy_error_full W");
    if (s != TQ_OK) return s;
    if ((s = check_mat(X, "tq_proxy_error_full X")) != TQ_OK) return s;
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_proxy_error_full: unknown format %d", fmt);
    if (X->dtype != TQ_BF16 || W->dtype != TQ_BF16)
        return set_error(TQ_ERR_UNSUPPORTED, "tq_proxy_error_full: X and W must be bf16");
    TQ_REQUIRE(packed && scales && num && den && workspace, "tq_proxy_error_full: null pointer");
    TQ_REQUIRE(X->cols == W->cols && X->n_mat == W->n_mat, "tq_proxy_error_full: X and W must share I and n_mat");
    TQ_REQUIRE(aligned16(packed) && aligned16(workspace), "tq_proxy_error_full: packed/workspace not 16-byte aligned");
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "tq_proxy_error_full: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_proxy_error_full: NVFP4 needs global_scale");
    TQ_REQUIRE(W->n_mat <= 65535 && X->rows < (int64_t(1) << 31) && W->rows < (int64_t(1) << 31) &&
                   W->cols < (int64_t(1) << 24),
               "tq_proxy_error_full: sizes out of range");
    TQ_REQUIRE(workspace_bytes >= tq_proxy_full_workspace_bytes(X, W), "tq_proxy_error_full: workspace too small");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t Ip = pf_ip(W->cols), O = W->rows, E = W->n_mat;
    __nv_bfloat16* ep = static_cast<__nv_bfloat16*>(workspace);
    const int64_t ep_bytes = (E * O * PF_PIECES * Ip * 2 + 255) / 256 * 256;
    const int64_t tiles = pf_tiles(X, W);
    double* pn = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + ep_bytes);
    double* pd = pn + E * tiles;
    // tensor maps first (host only), so a failure launches nothing
    CUtensorMap xm, em, wm;
    const int64_t xms = E > 1 ? X->mat_stride : X->rows * X->ld;
    const int64_t wms = E > 1 ? W->mat_stride : W->rows * W->ld;
    if (!pf_map(&xm, X->ptr, X->cols, X->rows, E, X->ld, xms, PF_M) ||
        !pf_map(&em, ep, PF_PIECES * Ip, O, E, PF_PIECES * Ip, O * PF_PIECES * Ip, PF_N) ||
        !pf_map(&wm, W->ptr, W->cols, O, E, W->ld, wms, PF_N))
        return set_error(TQ_ERR_CUDA, "tq_proxy_error_full: tensor map encoding failed");
    // E = W - What in bf16 pieces
    {
        const int64_t ms = E > 1 ? W->mat_stride : 0;
        const int64_t work = E * O * (Ip / 8);
        const unsigned grid = static_cast<unsigned>(min((work + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
        const uint16_t* Wp = static_cast<const uint16_t*>(W->ptr);
        if (fmt == TQ_INT3_G64_SYM)
            k_pf_prep<TQ_INT3_G64_SYM, uint16_t><<<grid, 256, 0, st>>>(Wp, O, W->cols, W->ld, ms, packed, scales, zeros, global_scale, E, Ip, ep);
        else if (fmt == TQ_INT4_G128_ASYM)
            k_pf_prep<TQ_INT4_G128_ASYM, uint16_t><<<grid, 256, 0, st>>>(Wp, O, W->cols, W->ld, ms, packed, scales, zeros, global_scale, E, Ip, ep);
        else if (fmt == TQ_INT4_G64_ASYM)
            k_pf_prep<TQ_INT4_G64_ASYM, uint16_t><<<grid, 256, 0, st>>>(Wp, O, W->cols, W->ld, ms, packed, scales, zeros, global_scale, E, Ip, ep);
        else if (fmt == TQ_INT4_G32_ASYM)
            k_pf_prep<TQ_INT4_G32_ASYM, uint16_t><<<grid, 256, 0, st>>>(Wp, O, W->cols, W->ld, ms, packed, scales, zeros, global_scale, E, Ip, ep);
        else
            k_pf_prep<TQ_NVFP4_G16, uint16_t><<<grid, 256, 0, st>>>(Wp, O, W->cols, W->ld, ms, packed, scales, zeros, global_scale, E, Ip, ep);
    }
    static std::once_flag attr;
    std::call_once(attr, [] { cudaFuncSetAttribute(k_pf_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM_BYTES); });
    PfArgs a;
    a.tiles_m = static_cast<int>((X->rows + PF_M - 1) / PF_M);
    a.tiles_n = static_cast<int>((O + PF_N - 1) / PF_N);
    a.kx = static_cast<int>(Ip / 64);
    a.pn = pn;
    a.pd = pd;
    a.wait_limit = pipeline_wait_limit();
    k_pf_gemm<<<dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(E)), PF_THREADS, PF_SMEM_BYTES, st>>>(xm, em, wm, a);
    k_pf_reduce<<<static_cast<unsigned>(E), 32, 0, st>>>(pn, pd, tiles, num, den);
    return check_launch("tq_proxy_error_full");
}
