// Hessian of a linear's inputs, H = sum_t x_t^T x_t (fp32), from bf16
// activations X [T][I] on the 5th-generation tensor cores.
//
// Source: "Quantize on TT cards: CUDA-free GPTQ/LDLQ bfp4 pipeline" (tt-stack
// issue #67), pipeline table step 1: the per-linear-input Hessian accumulated
// in fp32 over the calibration tokens, a pure rank-k accumulation (its
// diagonal is T times the activation imatrix).  The page measures the bf16
// X^T X on its own accelerator at 5.9e-5 relative error (stage-1 precision
// results); here the products of bf16 values are exact and only the fp32
// accumulation rounds.
//
// As a GEMM: H[i][j] = sum_t X[t][i] X[t][j], M = N = I, K = T; both operands
// are columns of row-major X, i.e. MN-major in memory, which the tensor core
// reads directly (no transpose pass).  H is symmetric, so only tiles that
// reach the upper triangle are computed, and each upper entry is written to
// both triangles (exactly symmetric output).
//
// B200 mapping (one CTA per 128 x 256 tile of H, 4 warps, 2 CTAs per SM, all
// 512 TMEM columns in use):
//  * TMA (cp.async.bulk.tensor, 128-byte swizzle) brings 32-token slices of the
//    128-column A panel and the 256-column B panel into a 4-stage shared-memory
//    ring (24 KB per stage); when the A panel is half of the B panel (tiles on
//    the diagonal) only B is loaded and A is read from it.
//  * One thread issues tcgen05.mma (kind::f16, bf16 in, fp32 accumulate,
//    M = 128, N = 256, K = 16, both operands MN-major from shared memory); the
//    accumulator lives in 256 TMEM columns.  tcgen05.commit frees a stage when
//    its MMAs have read it.  A 128 x 256 tile keeps the shared-memory traffic
//    (TMA writes plus operand reads) under the bandwidth a 128 x 128 tile
//    exceeds at the tensor cores' rate.
//  * The 4 warps read the accumulator with tcgen05.ld (warp w: rows 32w..32w+31)
//    into the (then free) ring, 128 columns at a time, padded so that row and
//    column walks are conflict-free, and store the upper entries and their
//    mirror images with coalesced rows.
//  * Tiles are grouped in 1024 x 1024 super-blocks so that the CTAs in flight
//    share their panels in L2.
// Every wait on an mbarrier has an iteration limit; when a wait of the
// copy/MMA ring runs out the kernel records it (tq_sync reports it), skips
// the stores, waits (with the default limit) for the MMAs it committed and
// the copies it issued, frees TMEM and returns.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "tq_internal.cuh"

namespace tq {

constexpr int HS_M = 128;         // tile rows (A panel: 128 columns of X)
constexpr int HS_BK = 32;         // tokens per stage
constexpr int HS_STAGES = 4;
constexpr int HS_THREADS = 128;
constexpr int HS_SUPER_M = 8;                          // a super-block: 1024 x 1024 of H
constexpr int HS_BOX_BYTES = 64 * HS_BK * 2;           // one TMA box: 64 columns x 32 tokens, bf16
constexpr int HS_A_BYTES = (HS_M / 64) * HS_BOX_BYTES;

// Tile columns N (B panel: N columns of X): 256, or 128 where the tiles of
// the upper triangle fill whole waves better (chosen per shape at launch).
template <int N>
struct HsCfg {
    static_assert(N == 256 || N == 128, "tile width");
    static constexpr int SUPER_N = 1024 / N;
    static constexpr int B_BYTES = (N / 64) * HS_BOX_BYTES;
    static constexpr int STAGE_BYTES = HS_A_BYTES + B_BYTES;
    static constexpr int SMEM_BYTES = HS_STAGES * STAGE_BYTES + 1024 /* alignment */ + 256 /* barriers */;
    // Instruction descriptor: kind::f16, fp32 accumulator, bf16 A and B, both
    // MN-major, M = 128, N.
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                      (static_cast<uint32_t>(N >> 3) << 17) |
                                      (static_cast<uint32_t>(HS_M >> 4) << 24);
};
constexpr unsigned HS_WAIT_LIMIT = DEFAULT_WAIT_LIMIT;  // try_wait rounds before a wait is declared hung

__device__ unsigned g_hs_timeouts = 0;

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Waits for the phase of parity `parity` to complete; false after `limit` rounds.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, unsigned parity, unsigned limit = HS_WAIT_LIMIT) {
    for (unsigned it = 0; it < limit; ++it) {
        unsigned ok;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    atomicAdd(&g_hs_timeouts, 1u);
    return false;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Shared-memory matrix descriptor: MN-major operand, 128-byte swizzle, 64
// elements (128 B) per row along M/N, rows = tokens.  LBO = bytes between
// consecutive 64-column boxes, SBO = bytes between groups of 8 token rows.
// A box of the 3-D map from shared memory to global memory (bulk group).
__device__ __forceinline__ void hs_tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

__device__ __forceinline__ uint64_t umma_desc(uint32_t addr) {
    constexpr uint64_t lbo = HS_BOX_BYTES >> 4, sbo = (8 * 128) >> 4;
    return (static_cast<uint64_t>((addr >> 4) & 0x3fffu)) | (lbo << 16) | (sbo << 32) | (1ull << 46) |
           (2ull << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------------ kernel

struct HsArgs {
    int64_t T, I, ldh, hms;   // tokens, columns, H row stride, H matrix stride (elements)
    float* H;
    float alpha;
    int accumulate;
    int h_tma;                // H leaves by TMA stores where a quarter is wholly above the diagonal
    int nbm, nbn;             // 128-row and N-column blocks
    int nsb;                  // super-blocks per side
    unsigned wait_limit;      // try_wait rounds of the ring waits
};

template <int N>
__global__ void __launch_bounds__(HS_THREADS, 1)
k_hessian(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap hmap,
          const __grid_constant__ HsArgs a) {
    using C = HsCfg<N>;
    constexpr int HS_N = N, HS_SUPER_N = C::SUPER_N, HS_B_BYTES = C::B_BYTES, HS_STAGE_BYTES = C::STAGE_BYTES;
    constexpr int R = N / HS_M;   // row tiles per column tile (2 or 1)
    // the tile: super-block pair (BI <= BJ), then a 128 x N tile inside it
    int p = static_cast<int>(blockIdx.x) / (HS_SUPER_M * HS_SUPER_N);
    const int local = static_cast<int>(blockIdx.x) % (HS_SUPER_M * HS_SUPER_N);
    int BI = 0;
    while (p >= a.nsb - BI) { p -= a.nsb - BI; ++BI; }
    const int BJ = BI + p;
    const int bi = BI * HS_SUPER_M + local / HS_SUPER_N, bj = BJ * HS_SUPER_N + local % HS_SUPER_N;
    if (bi >= a.nbm || bj >= a.nbn || R * bj + R - 1 < bi) return;   // past the edge or below the diagonal
    const int e = static_cast<int>(blockIdx.y);
    const bool a_in_b = bi / R == bj;   // the A panel is part of the B panel: load B only

    extern __shared__ uint8_t hs_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(hs_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + HS_STAGES * HS_STAGE_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * HS_STAGES + 1);
    int* progress = reinterpret_cast<int*>(tmem_slot + 1);   // [0] armed, [1] consumed, [2] loops ok, [3] MMAs done
    const uint32_t s_base = smem_u32(smem);
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + HS_STAGES), done = smem_u32(bars + 2 * HS_STAGES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = static_cast<int>((a.T + HS_BK - 1) / HS_BK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < HS_STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(done, 1);
        progress[0] = 0;
        progress[1] = 0;
        progress[2] = 1;
        progress[3] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {   // the whole warp allocates N TMEM columns (128 lanes x N fp32)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(HS_N));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {   // TMA producer
        const uint32_t bytes = a_in_b ? HS_B_BYTES : HS_STAGE_BYTES;
        int k = 0;
        for (; k < nk; ++k) {
            const int s = k % HS_STAGES;
            if (!mbar_wait(empty0 + 8 * s, ((k / HS_STAGES) & 1) ^ 1, a.wait_limit)) break;
            const uint32_t st = s_base + s * HS_STAGE_BYTES, bar = full0 + 8 * s;
            mbar_expect_tx(bar, bytes);
            const int t0 = k * HS_BK;
            if (!a_in_b) {
#pragma unroll
                for (int q = 0; q < HS_M / 64; ++q)
                    tma_load_3d(st + q * HS_BOX_BYTES, &xmap, bar, bi * HS_M + 64 * q, t0, e);
            }
#pragma unroll
            for (int q = 0; q < HS_N / 64; ++q)
                tma_load_3d(st + HS_A_BYTES + q * HS_BOX_BYTES, &xmap, bar, bj * HS_N + 64 * q, t0, e);
            progress[0] = k + 1;
        }
        if (k < nk) progress[2] = 0;
    } else if (warp == 1 && lane == 0) {   // MMA issuer
        int k = 0;
        for (; k < nk; ++k) {
            const int s = k % HS_STAGES;
            if (!mbar_wait(full0 + 8 * s, (k / HS_STAGES) & 1, a.wait_limit)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sb = s_base + s * HS_STAGE_BYTES + HS_A_BYTES;
            const uint32_t sa = a_in_b ? sb + (bi % R) * (HS_M / 64) * HS_BOX_BYTES : s_base + s * HS_STAGE_BYTES;
#pragma unroll
            for (int kk = 0; kk < HS_BK / 16; ++kk)   // 16 tokens = 16 rows of 128 B per MMA
                umma_bf16(tmem, umma_desc(sa + kk * 2048), umma_desc(sb + kk * 2048), C::IDESC, (k | kk) != 0);
            umma_commit(empty0 + 8 * s);   // the stage is free once these MMAs have read it
            progress[1] = k + 1;
        }
        if (k < nk) progress[2] = 0;
        umma_commit(done);                 // every MMA issued so far is complete
    }

    // epilogue.  One thread waits for the MMAs; the others wait at the block
    // barrier (no spinning).  The accumulator leaves through shared memory
    // (the ring is free once every MMA is complete), 64 columns at a time.
    // A quarter wholly above the diagonal is written, with its mirror image,
    // by TMA stores: the rows as 32-column chunks of 128 rows x 128 B in the
    // 128-byte swizzled layout (thread r writes 16-byte unit u of its row at
    // u ^ (r % 8)), the mirror as 32-row chunks of the transposed quarter
    // (64 rows of 128 B; a warp writes one 128-byte row per column).  A
    // quarter that crosses the diagonal stores its upper-triangle entries and
    // their mirror images from a padded tile with coalesced rows; entries
    // below the diagonal are left to their mirror, so H is exactly symmetric.
    if (warp == 1 && lane == 0) progress[3] = mbar_wait(done, 0) ? 1 : 0;
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const bool ok = progress[3] != 0 && progress[2] != 0;
    float* He = a.H + static_cast<int64_t>(e) * a.hms;
    const int64_t r0 = static_cast<int64_t>(bi) * HS_M;
    const int rr = warp * 32 + lane;   // this thread's accumulator row
    bool stored = false;               // TMA stores issued (thread 0)
#pragma unroll 1
    for (int qh = 0; qh < HS_N / 64; ++qh) {
        const int64_t ca = static_cast<int64_t>(bj) * HS_N + 64 * qh;   // the quarter's first column
        if (!ok || ca >= a.I || ca + 63 < r0) continue;                  // past the edge or below the diagonal
        const bool tma = a.h_tma && ca >= r0 + HS_M;   // wholly above the diagonal
        constexpr int LDT = 64 + 1;                     // padded tile: row and column walks are conflict-free
        float* tile = reinterpret_cast<float*>(smem);
        // the quarter's two 32-column halves, one at a time (32 registers of values)
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            float v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(64 * qh + 32 * h), v);
            if (a.alpha != 1.0f) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(a.alpha, v[i]);
            }
            if (tma) {
                float4* row = reinterpret_cast<float4*>(smem + h * (HS_M * 128) + rr * 128);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    row[u ^ (rr & 7)] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                uint8_t* mch = smem + 2 * (HS_M * 128) + warp * (64 * 128);   // mirror chunk of rows 32 warp ..
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int cc = 32 * h + c;
                    *reinterpret_cast<float*>(mch + cc * 128 + (((lane >> 2) ^ (cc & 7)) << 4) + ((lane & 3) << 2)) =
                        v[c];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) tile[rr * LDT + 32 * h + i] = v[i];
            }
        }
        if (tma) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            if (threadIdx.x == 0) {
#pragma unroll 1
                for (int h = 0; h < 2; ++h)
                    for (int half = 0; half < 2; ++half)
                        if (ca + 32 * h < a.I && r0 + 64 * half < a.I)
                            hs_tma_store_3d(&hmap, s_base + h * (HS_M * 128) + half * (64 * 128),
                                            static_cast<int>(ca + 32 * h), static_cast<int>(r0 + 64 * half), e);
#pragma unroll 1
                for (int k = 0; k < HS_M / 32; ++k)
                    if (r0 + 32 * k < a.I)
                        hs_tma_store_3d(&hmap, s_base + 2 * (HS_M * 128) + k * (64 * 128), static_cast<int>(r0 + 32 * k),
                                        static_cast<int>(ca), e);
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");   // the chunks may be rewritten
                stored = true;
            }
            __syncthreads();
        } else {
            __syncthreads();
#pragma unroll 4
            for (int idx = threadIdx.x; idx < HS_M * 64; idx += HS_THREADS) {   // H[r0 + r][ca + c]
                const int r = idx >> 6, c = idx & 63;
                const int64_t gr = r0 + r, gc = ca + c;
                if (gr < a.I && gc < a.I && gc >= gr) {
                    float* q = He + gr * a.ldh + gc;
                    const float x = tile[r * LDT + c];
                    *q = a.accumulate ? __fadd_rn(*q, x) : x;
                }
            }
#pragma unroll 4
            for (int idx = threadIdx.x; idx < HS_M * 64; idx += HS_THREADS) {   // mirror: H[ca + c][r0 + r]
                const int c = idx >> 7, r = idx & 127;
                const int64_t gr = r0 + r, gc = ca + c;
                if (gr < a.I && gc < a.I && gc > gr) {
                    float* q = He + gc * a.ldh + gr;
                    const float x = tile[r * LDT + c];
                    *q = a.accumulate ? __fadd_rn(*q, x) : x;
                }
            }
            __syncthreads();
        }
    }
    if (stored) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // the stores are complete

    // teardown: drain copies armed but not consumed and (if the epilogue's
    // wait gave up) the committed MMAs, then free TMEM
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = progress[1]; k < progress[0]; ++k)
            if (!mbar_wait(full0 + 8 * (k % HS_STAGES), (k / HS_STAGES) & 1)) break;
        if (progress[3] == 0) mbar_wait(done, 0);
    }
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(HS_N));
    }
}

// ------------------------------------------------------------------ host

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiled encode_tiled() {
    static std::once_flag once;
    static EncodeTiled fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

bool hessian_take_timeouts() {
    unsigned n = 0;
    if (cudaMemcpyFromSymbol(&n, g_hs_timeouts, sizeof(n)) != cudaSuccess || n == 0) return false;
    const unsigned zero = 0;
    cudaMemcpyToSymbol(g_hs_timeouts, &zero, sizeof(zero));
    return true;
}

}  // namespace tq

using namespace tq;

TQ_API tq_status tq_hessian(const tq_mat* X, float* H, int64_t ldh, int64_t h_mat_stride, float alpha,
                            int32_t accumulate, tq_stream_t stream) {
    clear_error();
    TQ_REQUIRE(X && X->ptr && H, "tq_hessian: null pointer");
    if (X->dtype != TQ_BF16) return set_error(TQ_ERR_UNSUPPORTED, "tq_hessian: activations must be bf16");
    TQ_REQUIRE(X->n_mat >= 1 && X->rows >= 1 && X->cols >= 1, "tq_hessian: empty shape");
    TQ_REQUIRE(X->ld >= X->cols && (X->ld * 2) % 16 == 0, "tq_hessian: X row stride must be >= I and a multiple of 16 bytes");
    TQ_REQUIRE(X->n_mat == 1 || (X->mat_stride >= X->rows * X->ld && (X->mat_stride * 2) % 16 == 0),
               "tq_hessian: X matrix stride must be >= T*ld and a multiple of 16 bytes");
    TQ_REQUIRE(aligned16(X->ptr), "tq_hessian: X not 16-byte aligned");
    TQ_REQUIRE(ldh >= X->cols, "tq_hessian: ldh < I");
    TQ_REQUIRE(X->n_mat == 1 || h_mat_stride >= X->cols * ldh, "tq_hessian: H matrix stride < I*ldh");
    TQ_REQUIRE(X->rows < (int64_t(1) << 31) && X->cols < (int64_t(1) << 31) && X->n_mat <= 65535,
               "tq_hessian: T, I < 2^31 and n_mat <= 65535");
    EncodeTiled enc = encode_tiled();
    if (!enc) return set_error(TQ_ERR_CUDA, "tq_hessian: cuTensorMapEncodeTiled unavailable");

    CUtensorMap map;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(X->cols), static_cast<cuuint64_t>(X->rows),
                                static_cast<cuuint64_t>(X->n_mat)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(X->ld * 2),
                                   static_cast<cuuint64_t>((X->n_mat > 1 ? X->mat_stride : X->rows * X->ld) * 2)};
    const cuuint32_t box[3] = {64, HS_BK, 1}, estr[3] = {1, 1, 1};
    CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(X->ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(TQ_ERR_CUDA, "tq_hessian: tensor map encoding failed (%d)", static_cast<int>(r));

    HsArgs a;
    a.T = X->rows; a.I = X->cols; a.ldh = ldh; a.hms = X->n_mat > 1 ? h_mat_stride : 0;
    a.H = H; a.alpha = alpha; a.accumulate = accumulate ? 1 : 0;
    // H by TMA stores: written (not accumulated), 16-byte aligned rows and matrices
    CUtensorMap hmap;
    memset(&hmap, 0, sizeof hmap);
    a.h_tma = !accumulate && aligned16(H) && ldh % 4 == 0 && (X->n_mat == 1 || h_mat_stride % 4 == 0) &&
              X->cols >= 64;
    if (a.h_tma) {
        const cuuint64_t hd[3] = {static_cast<cuuint64_t>(X->cols), static_cast<cuuint64_t>(X->cols),
                                  static_cast<cuuint64_t>(X->n_mat)};
        const cuuint64_t hs[2] = {static_cast<cuuint64_t>(ldh * 4),
                                  static_cast<cuuint64_t>((X->n_mat > 1 ? h_mat_stride : X->cols * ldh) * 4)};
        const cuuint32_t hbox[3] = {32, 64, 1};
        CUresult hr = enc(&hmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, H, hd, hs, hbox, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (hr != CUDA_SUCCESS) a.h_tma = 0;
    }
    a.nbm = static_cast<int>((X->cols + HS_M - 1) / HS_M);
    a.nsb = static_cast<int>((X->cols + 1023) / 1024);
    a.wait_limit = pipeline_wait_limit();
    static std::once_flag attr;
    std::call_once(attr, [] {
        cudaFuncSetAttribute(k_hessian<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, HsCfg<256>::SMEM_BYTES);
        cudaFuncSetAttribute(k_hessian<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, HsCfg<128>::SMEM_BYTES);
    });
    // The tile width: the SMs' time is about waves x resident tiles per SM x
    // columns per tile; 128-column tiles where that is less (more, narrower
    // tiles that fill the last wave better), else 256.
    // Resident CTAs per SM, counted from the three limits: shared memory
    // (with the per-block reserve), registers and TMEM columns (512 per SM).
    auto resident = [&](int n, const void* kern, int smem) {
        int dev = 0, smem_sm = 0, reserve = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&reserve, cudaDevAttrReservedSharedMemoryPerBlock, dev);
        cudaFuncAttributes fa;
        int by_regs = 1;
        if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess && fa.numRegs > 0) {
            const int per_warp = (fa.numRegs * 32 + 255) / 256 * 256;   // allocated per warp in units of 256
            by_regs = 65536 / (per_warp * (HS_THREADS / 32));
        }
        const int by_smem = smem_sm > 0 ? smem_sm / (smem + reserve) : 1;
        const int by_tmem = 512 / n;
        return max(1, min(by_smem, min(by_regs, by_tmem)));
    };
    auto cost = [&](int n, const void* kern, int smem) {
        const int64_t nbn = (X->cols + n - 1) / n, r = n / HS_M;
        int64_t tiles = 0;
        for (int64_t bi = 0; bi < a.nbm; ++bi) tiles += nbn - min(nbn, bi / r);   // tiles with r bj + r - 1 >= bi
        const int per_sm = resident(n, kern, smem);
        const int64_t slots = static_cast<int64_t>(num_sms()) * per_sm;
        return ((tiles * X->n_mat + slots - 1) / slots) * per_sm * n;
    };
    const bool narrow = cost(128, reinterpret_cast<const void*>(k_hessian<128>), HsCfg<128>::SMEM_BYTES) <
                        cost(256, reinterpret_cast<const void*>(k_hessian<256>), HsCfg<256>::SMEM_BYTES);
    const int n = narrow ? 128 : 256;
    a.nbn = static_cast<int>((X->cols + n - 1) / n);
    const int64_t pairs = static_cast<int64_t>(a.nsb) * (a.nsb + 1) / 2;
    const int64_t gx = pairs * HS_SUPER_M * (1024 / n);
    TQ_REQUIRE(gx < (int64_t(1) << 31), "tq_hessian: I too large");
    dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(X->n_mat));
    if (narrow)
        k_hessian<128><<<grid, HS_THREADS, HsCfg<128>::SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream)>>>(map, hmap, a);
    else
        k_hessian<256><<<grid, HS_THREADS, HsCfg<256>::SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream)>>>(map, hmap, a);
    return check_launch("tq_hessian");
}
