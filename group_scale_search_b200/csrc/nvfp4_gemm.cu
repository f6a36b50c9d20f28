// NVFP4 W4A4 product on the block-scaled tensor cores: the consumer of the
// NVFP4-g16 expert records.
//
// Source: "Nemotron-Cascade-2-30B-A3B-NVFP4" model card, Quantization Recipe
// table (the routed experts run W4A4 with group size 16: E2M1 elements, one
// E4M3 scale per 16 elements, an fp32 scale per tensor) and Serving
// Instructions (the FP4 MoE GEMM on Blackwell).  The card says nothing of how
// activations are quantized; the reading taken is the weights' recipe without
// the search: per tensor g = fl32(amax / 2688), per 16-element block the
// positive finite E4M3 code nearest b / (6 g) (b the block amax, distance
// |6 g dec(c) - b| exact in fp64, ties to the lower code), elements by E2M1
// round-to-nearest-even of the IEEE quotient with sign (zero always +0).  The
// product is the value of the block-scaled representation:
//   y[t][o] = g_x g_w sum_k dec(ex[t][k]) dec(ew[o][k]) sum_{j in block k} dec(cx[t][j]) dec(cw[o][j]).
//
// Three calls:
//  * tq_quant_nvfp4_act: the activation quantizer (amax per matrix, then one
//    thread per 16-element block: nearest E4M3 code by a binary search of
//    exact fp64 predicates, E2M1 codes by the shared NVFP4 RTN), writing
//    records in the weights' NVFP4 layout (8 bytes per block, element 2k in
//    the low nibble of byte k) and [row][block] E4M3 scale codes.
//  * tq_nvfp4_scales_to_mma: the [row][block] scale codes of a matrix batch
//    re-laid out as the tensor core's scale-factor tiles (below), rows padded
//    to a multiple of 256 and blocks to a multiple of 16 with zeros.  Weights
//    are re-laid out once; activations once per call.
//  * tq_gemm_nvfp4: the GEMM, M = tokens, N = weight rows, K = I, both
//    operands K-major (rows of packed codes are contiguous in I).
//
// Scale-factor tile: for 128 rows x 4 blocks (one K = 64 step of the MMA) a
// 512-byte chunk, byte (r % 32) * 16 + (r / 32) * 4 + k for row r (0..127)
// and block k (0..3): the source layout of tcgen05.cp.32x128b.warpx4, which
// puts the chunk in TMEM lanes r % 32 of every 32-lane quarter, column r / 32,
// byte k -- where the block-scaled MMA reads the scale of row r.  Chunks are
// ordered [matrix][row tile][k chunk].
//
// B200 mapping of the GEMM (one CTA per 128 x 256 output tile, 4 warps, 1
// CTA per SM):
//  * TMA (128-byte swizzle) brings 256-element K slices (128 bytes of packed
//    codes per row) of the 128-token A tile and the 256-row B tile into a
//    4-stage shared-memory ring; three 1-D bulk copies bring the stage's
//    scale chunks (A: 4 chunks, B: 2 x 4 chunks), all on one mbarrier.
//  * One thread copies the stage's scale chunks into TMEM (tcgen05.cp,
//    double-buffered by stage parity) and issues four
//    tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M = 128, N = 256, K = 64,
//    E4M3 scales every 16 elements, fp32 accumulate in TMEM columns 0-255);
//    tcgen05.commit frees the stage once they have read it.
//  * The 4 warps read the accumulator (tcgen05.ld, warp w: tokens 32w..32w+31),
//    scale it by g_x g_w and store fp32 rows of y.
// Every mbarrier wait is bounded (see tq_debug_set_wait_limit); a CTA whose
// ring wait gives up stores nothing, waits with the default limit for the
// copies it issued and the MMAs it committed, frees TMEM and returns, and the
// next tq_sync reports it.
#include <cuda.h>

#include <mutex>

#include "walk.cuh"

namespace tq {

// ------------------------------------------------------------------ activation quantizer

// Largest E4M3 code (1..126) whose value does not exceed the fp32 value t
// (1 below the smallest subnormal); exact for t itself, so within one code
// of the floor code of the exact quotient b / (6 g) that t rounds.
__device__ __forceinline__ int e4m3_floor(float t) {
    if (!(t > 0.f)) return 1;
    if (t < 0.015625f) return max(1, static_cast<int>(t * 512.f));
    const unsigned u = __float_as_uint(t);
    const int E = static_cast<int>((u >> 23) & 255u) - 127;
    return min(max(((E + 7) << 3) | static_cast<int>((u >> 20) & 7u), 1), 126);
}

// The positive finite E4M3 code (1..126) nearest t = b / (6 g) by the exact
// distance d(c) = |6 g dec(c) - b| (fp64: 6 g dec(c) has at most 31
// significant bits), ties to the lower code.  The nearest code is the floor
// code of the exact t or the next one; an fp32 estimate of t within a few
// ulps (b times the approximate reciprocal inv6g of 6 g) is within one code
// of that floor (E4M3 codes are at least 2^-3 apart relatively), so the four
// codes around it hold the answer, compared in ascending order with strict
// improvement.  inv6g = 0 (6 g outside the range where the approximate
// reciprocal is accurate) takes the IEEE quotient instead.
__device__ __forceinline__ int nearest_e4m3_code(float b, float g, float inv6g) {
    const double g6 = 6.0 * static_cast<double>(g), bd = static_cast<double>(b);
    const float t = inv6g != 0.f ? __fmul_rn(b, inv6g) : __fdiv_rn(b, __fmul_rn(6.f, g));
    const int c0 = max(1, min(123, e4m3_floor(t) - 1));
    int best = c0;
    double bdist = fabs(__dsub_rn(__dmul_rn(g6, static_cast<double>(e4m3_value(c0))), bd));
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        const double d = fabs(__dsub_rn(__dmul_rn(g6, static_cast<double>(e4m3_value(c0 + i))), bd));
        if (d < bdist) { bdist = d; best = c0 + i; }
    }
    return best;
}

// amax -> g = fl32(amax / 2688), in place.
__global__ void k_act_global(float* g, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) g[i] = __fdiv_rn(g[i], 2688.0f);
}

template <typename T>
__global__ void __launch_bounds__(256)
k_quant_act_nvfp4(const T* __restrict__ X, int64_t I, int64_t ld, int64_t ms, const float* __restrict__ gs,
                  GroupIndex gi, int64_t total, uint8_t* __restrict__ scales, uint8_t* __restrict__ packed) {
    for (int64_t bid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; bid < total;
         bid += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        uint32_t e, r, k;
        gi.split(static_cast<uint32_t>(bid), e, r, k);
        const int64_t j0 = static_cast<int64_t>(k) << 4;
        const int n = static_cast<int>(min(static_cast<int64_t>(16), I - j0));
        const T* p = X + e * ms + static_cast<int64_t>(r) * ld + j0;
        Oct<T> o0, o1;
        o0.load(p, min(n, 8));
        o1.load(p + 8, max(n - 8, 0));
        float w[16];
        o0.get(w);
        o1.get(w + 8);
        float b = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) b = fmaxf(b, fabsf(w[i]));
        const float g = __ldg(gs + e);
        const float g6f = __fmul_rn(6.f, g);
        const float inv6g = (g6f > 1e-30f && g6f < 1e30f) ? rcp_approx(g6f) : 0.f;
        const int code = (g > 0.f && b > 0.f) ? nearest_e4m3_code(b, g, inv6g) : 0;
        const float S = code ? __fmul_rn(g, e4m3_value(static_cast<unsigned>(code))) : 0.f;
        uint32_t pk[2];
        nvfp4_rtn<16>(w, S, pk);
        scales[bid] = static_cast<uint8_t>(code);
        *reinterpret_cast<uint2*>(packed + bid * 8) = make_uint2(pk[0], pk[1]);
    }
}

// ------------------------------------------------------------------ scale-factor tiles

__host__ __device__ inline int64_t sf_row_tiles(int64_t rows) { return 2 * ((rows + 255) / 256); }
__host__ __device__ inline int64_t sf_k_chunks(int64_t G) { return 4 * ((G + 15) / 16); }

// One thread per output word (4 blocks of one row): coalesced writes.
__global__ void k_sf_to_mma(const uint8_t* __restrict__ sc, int64_t rows, int64_t G, int64_t RT, int64_t KC,
                            int64_t total_words, uint32_t* __restrict__ out) {
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < total_words;
         w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t chunk = w >> 7;
        const int within = static_cast<int>(w & 127);
        const int64_t kc = chunk % KC, rt = (chunk / KC) % RT, e = chunk / (KC * RT);
        const int64_t r = rt * 128 + (within >> 2) + 32 * (within & 3);
        uint32_t v = 0u;
        if (r < rows) {
            const uint8_t* src = sc + (e * rows + r) * G;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t k = 4 * kc + q;
                if (k < G) v |= static_cast<uint32_t>(__ldg(src + k)) << (8 * q);
            }
        }
        out[w] = v;
    }
}

// ------------------------------------------------------------------ GEMM

constexpr int NG_M = 128;
constexpr int NG_BKB = 128;                                 // K bytes per stage (256 E2M1 codes)
constexpr int NG_THREADS = 128;
constexpr int NG_A_BYTES = NG_M * NG_BKB;                   // 16 KB
constexpr int NG_SFA_BYTES = 4 * 512;                       // 4 MMAs x one 128-row chunk

// Tile shapes: 128 tokens x BN weight rows.  BN = 256: 4 stages, 216 KB of
// shared memory and all 512 TMEM columns, one CTA per SM.  BN = 128: 3
// stages, 2 CTAs per SM (each 256 TMEM columns), so one CTA's epilogue runs
// while the other's MMAs do.
template <int BN>
struct NgCfg {
    static constexpr int N = BN;
    static constexpr int HALVES = BN / 128;                          // 128-row scale tiles per B tile
    static constexpr int STAGES = BN == 256 ? 4 : 3;
    static constexpr int B_BYTES = BN * NG_BKB;
    static constexpr int SFB_BYTES = 4 * 512 * HALVES;               // 4 MMAs x HALVES chunks
    static constexpr int STAGE_BYTES = NG_A_BYTES + B_BYTES + NG_SFA_BYTES + SFB_BYTES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
    static constexpr uint32_t SF_COL = BN;                           // first scale column
    static constexpr uint32_t SF_COLS = 16 + 16 * HALVES;             // per stage parity: A 4 x 4, B 4 x 4 x HALVES
    static constexpr uint32_t TMEM_COLS = BN == 256 ? 512 : 256;      // accumulator + 2 x SF_COLS, a power of 2
    static constexpr int MIN_BLOCKS = BN == 256 ? 1 : 2;
    // kind::mxf4nvf4 block-scaled descriptor: E2M1 A and B (format 1), both
    // K-major, UE4M3 scales, dense K = 64, N = BN, M = 128.
    static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                      (static_cast<uint32_t>(NG_M >> 4) << 24);
    static_assert(STAGE_BYTES % 1024 == 0, "stage bases stay 1024-byte aligned");
    static_assert(SF_COL + 2 * SF_COLS <= TMEM_COLS, "TMEM columns");
    static_assert(SMEM_BYTES * MIN_BLOCKS <= 232448, "shared memory");
};

__device__ unsigned g_ng_timeouts = 0;

__device__ __forceinline__ uint32_t ng_smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool ng_wait(uint32_t bar, unsigned parity, unsigned limit = DEFAULT_WAIT_LIMIT) {
    for (unsigned it = 0; it < limit; ++it) {
        unsigned ok;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    atomicAdd(&g_ng_timeouts, 1u);
    return false;
}

__device__ __forceinline__ void ng_tma_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void ng_bulk(uint32_t dst, const void* src, unsigned bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// K-major operand, 128-byte swizzle: rows of 128 bytes (256 E2M1 codes),
// groups of 8 rows 1024 B apart (SBO); LBO unused (1).
__device__ __forceinline__ uint64_t ng_desc_sw128(uint32_t addr) {
    return (static_cast<uint64_t>((addr >> 4) & 0x3fffu)) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Source of tcgen05.cp.32x128b: 32 rows of 16 bytes, no swizzle, core
// matrices of 8 rows 128 B apart (SBO).
__device__ __forceinline__ uint64_t ng_desc_sf(uint32_t addr) {
    return (static_cast<uint64_t>((addr >> 4) & 0x3fffu)) | (1ull << 16) | (8ull << 32) | (1ull << 46);
}

__device__ __forceinline__ void ng_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void ng_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t tsfa,
                                       uint32_t tsfb, uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
        : "memory");
}

__device__ __forceinline__ void ng_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void ng_ld32(uint32_t taddr, float (&v)[32]) {
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

struct NgArgs {
    int64_t T, O;
    int tiles_m, nk;
    int64_t kc;                 // scale chunks per row tile (a multiple of 4: whole stages)
    int64_t rt_a, rt_b;         // row tiles per matrix of the A and B scale tiles
    const uint8_t* sfa;         // scale tiles of A (activations)
    const uint8_t* sfb;         // scale tiles of B (weights)
    const float* gx;
    const float* gw;
    float* y;                   // [n_mat][T][O]
    int y_tma;                  // O % 4 == 0: the tile leaves through shared memory by TMA stores
    unsigned wait_limit;
};

__device__ __forceinline__ void ng_tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

template <int BN>
__global__ void __launch_bounds__(NG_THREADS, NgCfg<BN>::MIN_BLOCKS)
k_gemm_nvfp4(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
             const __grid_constant__ CUtensorMap ymap, const __grid_constant__ NgArgs a) {
    using C = NgCfg<BN>;
    constexpr int NG_N = C::N, NG_STAGES = C::STAGES, NG_STAGE_BYTES = C::STAGE_BYTES, NG_B_BYTES = C::B_BYTES;
    const int tm = static_cast<int>(blockIdx.x) % a.tiles_m, tn = static_cast<int>(blockIdx.x) / a.tiles_m;
    const int e = static_cast<int>(blockIdx.y);
    extern __shared__ uint8_t ng_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ng_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NG_STAGES * NG_STAGE_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NG_STAGES + 1);
    int* progress = reinterpret_cast<int*>(tmem_slot + 1);   // [0] armed, [1] consumed, [2] ring ok, [3] MMAs done
    const uint32_t s_base = ng_smem_u32(smem);
    const uint32_t full0 = ng_smem_u32(bars), empty0 = full0 + 8 * NG_STAGES, done = empty0 + 8 * NG_STAGES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = a.nk;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * NG_STAGES + 1; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * i) : "memory");
        progress[0] = 0;
        progress[1] = 0;
        progress[2] = 1;
        progress[3] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(ng_smem_u32(tmem_slot)),
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {   // producer: TMA for the codes, bulk copies for the scale chunks
        const uint8_t* sfa = a.sfa + (static_cast<int64_t>(e) * a.rt_a + tm) * a.kc * 512;
        const uint8_t* sfb0 = a.sfb + (static_cast<int64_t>(e) * a.rt_b + C::HALVES * tn) * a.kc * 512;
        const uint8_t* sfb1 = sfb0 + a.kc * 512;
        int kt = 0;
        for (; kt < nk; ++kt) {
            const int s = kt % NG_STAGES;
            if (!ng_wait(empty0 + 8 * s, ((kt / NG_STAGES) & 1) ^ 1, a.wait_limit)) break;
            const uint32_t st = s_base + s * NG_STAGE_BYTES, bar = full0 + 8 * s;
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(NG_STAGE_BYTES)
                         : "memory");
            ng_tma_3d(st, &amap, bar, kt * NG_BKB, tm * NG_M, e);
            ng_tma_3d(st + NG_A_BYTES, &bmap, bar, kt * NG_BKB, tn * NG_N, e);
            const int64_t off = static_cast<int64_t>(4 * kt) * 512;
            ng_bulk(st + NG_A_BYTES + NG_B_BYTES, sfa + off, NG_SFA_BYTES, bar);
            ng_bulk(st + NG_A_BYTES + NG_B_BYTES + NG_SFA_BYTES, sfb0 + off, 2048, bar);
            if (C::HALVES == 2) ng_bulk(st + NG_A_BYTES + NG_B_BYTES + NG_SFA_BYTES + 2048, sfb1 + off, 2048, bar);
            progress[0] = kt + 1;
        }
        if (kt < nk) progress[2] = 0;
    } else if (warp == 1 && lane == 0) {   // scale copies and MMAs
        int kt = 0;
        for (; kt < nk; ++kt) {
            const int s = kt % NG_STAGES;
            if (!ng_wait(full0 + 8 * s, (kt / NG_STAGES) & 1, a.wait_limit)) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sa = s_base + s * NG_STAGE_BYTES, sb = sa + NG_A_BYTES;
            const uint32_t ssfa = sb + NG_B_BYTES, ssfb = ssfa + NG_SFA_BYTES;
            const uint32_t tsf = tmem + C::SF_COL + C::SF_COLS * static_cast<uint32_t>(kt & 1);
            constexpr uint32_t BC = 4 * C::HALVES;   // TMEM columns of B's scales per MMA
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                ng_cp_sf(tsf + 4 * j, ng_desc_sf(ssfa + 512 * j));
                ng_cp_sf(tsf + 16 + BC * j, ng_desc_sf(ssfb + 512 * j));
                if (C::HALVES == 2) ng_cp_sf(tsf + 16 + BC * j + 4, ng_desc_sf(ssfb + 2048 + 512 * j));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)   // K = 64 codes = 32 bytes of each row per MMA
                ng_mma(tmem, ng_desc_sw128(sa + 32 * j), ng_desc_sw128(sb + 32 * j), C::IDESC, tsf + 4 * j,
                       tsf + 16 + BC * j, (kt | j) != 0);
            ng_commit(empty0 + 8 * s);   // the stage is free once these have read it
            progress[1] = kt + 1;
        }
        if (kt < nk) progress[2] = 0;
        ng_commit(done);
    }

    if (warp == 1 && lane == 0) progress[3] = ng_wait(done, 0) ? 1 : 0;
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const bool ok = progress[3] != 0 && progress[2] != 0;
    const int64_t m = static_cast<int64_t>(tm) * NG_M + warp * 32 + lane;
    const float gg = __fmul_rn(__ldg(a.gx + e), __ldg(a.gw + e));
    float* yr = a.y + (static_cast<int64_t>(e) * a.T + m) * a.O;
    if (ok && a.y_tma) {
        // The tile goes through the (now idle) ring as 32-column chunks of
        // 128 rows x 128 B in the 128-byte swizzled layout, and leaves by TMA
        // stores (rows and columns past the matrix are clipped).  Thread r
        // writes its row's 16-byte unit u at u ^ (r % 8): conflict-free.
        const int r = warp * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < NG_N; c0 += 32) {
            float v[32];
            ng_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), v);
            float4* row = reinterpret_cast<float4*>(smem + (c0 / 32) * (NG_M * 128) + r * 128);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                row[u ^ (r & 7)] = make_float4(__fmul_rn(v[4 * u], gg), __fmul_rn(v[4 * u + 1], gg),
                                               __fmul_rn(v[4 * u + 2], gg), __fmul_rn(v[4 * u + 3], gg));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int q = 0; q < NG_N / 32; ++q)
                if (static_cast<int64_t>(tn) * NG_N + 32 * q < a.O)
                    ng_tma_store_3d(&ymap, s_base + q * (NG_M * 128), tn * NG_N + 32 * q, tm * NG_M, e);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
    } else {
        const bool vec = (a.O & 3) == 0;
#pragma unroll 1
        for (int c0 = 0; c0 < NG_N; c0 += 32) {
            float v[32];
            ng_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), v);
            const int64_t o0 = static_cast<int64_t>(tn) * NG_N + c0;
            if (!ok || m >= a.T || o0 >= a.O) continue;
            if (vec && o0 + 32 <= a.O) {
                float4* d = reinterpret_cast<float4*>(yr + o0);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    d[i] = make_float4(__fmul_rn(v[4 * i], gg), __fmul_rn(v[4 * i + 1], gg),
                                       __fmul_rn(v[4 * i + 2], gg), __fmul_rn(v[4 * i + 3], gg));
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (o0 + i < a.O) yr[o0 + i] = __fmul_rn(v[i], gg);
            }
        }
    }

    // teardown: the copies armed but not consumed and (if the wait above gave
    // up) the committed MMAs, with the default limit; then free TMEM
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = progress[1]; k < progress[0]; ++k)
            if (!ng_wait(full0 + 8 * (k % NG_STAGES), (k / NG_STAGES) & 1)) break;
        if (progress[3] == 0) ng_wait(done, 0);
    }
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
}

// ------------------------------------------------------------------ persistent GEMM

// Persistent form: one CTA per SM walks the output tiles (128 tokens x 128
// weight rows) in order, with warp roles: warp 0 lane 0 feeds a 4-stage ring
// (TMA + bulk copies, as above) across tile boundaries; warp 1 lane 0 issues
// the scale copies and MMAs into one of two TMEM accumulators (columns 0-127
// and 128-255); warps 2-5 drain the other accumulator -- tcgen05.ld, scale,
// swizzled shared-memory tile, TMA store -- while the next tile's MMAs run.
// mbarriers: full/empty per stage (copies / MMA reads), acc_full per
// accumulator (MMAs complete, tcgen05.commit) and acc_empty per accumulator
// (the 128 epilogue threads have read it).
// The persistent form (true) or one CTA per tile (false).
constexpr bool NG_PERSISTENT = false;
constexpr int NP_STAGES = 4;
constexpr int NP_THREADS = 192;
constexpr int NP_B_BYTES = 128 * NG_BKB;
constexpr int NP_STAGE_BYTES = NG_A_BYTES + NP_B_BYTES + NG_SFA_BYTES + 2048;
// The output tile leaves through a shared-memory staging tile by TMA stores
// (true) or straight from registers (false: more ring stages fit).
constexpr bool NP_STAGED = true;
constexpr int NP_OUT_BYTES = NP_STAGED ? 128 * 128 * 4 : 0;      // one fp32 output tile
constexpr int NP_SMEM_BYTES = NP_STAGES * NP_STAGE_BYTES + NP_OUT_BYTES + 1024 + 256;
constexpr uint32_t NP_SF_COL = 256, NP_SF_COLS = 32;           // per k-step parity: A 4 x 4, B 4 x 4
constexpr uint32_t NP_IDESC = NgCfg<128>::IDESC;
static_assert(NP_STAGE_BYTES % 1024 == 0 && NP_SMEM_BYTES <= 232448, "persistent GEMM shared memory");

__device__ __forceinline__ void ng_named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__global__ void __launch_bounds__(NP_THREADS, 1)
k_gemm_nvfp4_persistent(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                        const __grid_constant__ CUtensorMap ymap, const __grid_constant__ NgArgs a,
                        int tiles_n, int64_t n_tiles) {
    extern __shared__ uint8_t np_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(np_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* outbuf = smem + NP_STAGES * NP_STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(outbuf + NP_OUT_BYTES);
    // bars: full[S], empty[S], acc_full[2], acc_empty[2], done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NP_STAGES + 5);
    volatile int* st = reinterpret_cast<volatile int*>(tmem_slot + 1);   // [0] armed, [1] consumed, [2] abort
    const uint32_t s_base = ng_smem_u32(smem), o_base = ng_smem_u32(outbuf);
    const uint32_t full0 = ng_smem_u32(bars), empty0 = full0 + 8 * NP_STAGES;
    const uint32_t accf0 = empty0 + 8 * NP_STAGES, acce0 = accf0 + 16, done = acce0 + 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = a.nk;
    const int tiles_per_mat = a.tiles_m * tiles_n;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2 * NP_STAGES + 2; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * i) : "memory");
        for (int i = 0; i < 2; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 128;" ::"r"(acce0 + 8 * i) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(done) : "memory");
        st[0] = 0;
        st[1] = 0;
        st[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(ng_smem_u32(tmem_slot)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    auto tile_of = [&](int64_t t, int& e, int& tm, int& tn) {
        e = static_cast<int>(t / tiles_per_mat);
        const int r = static_cast<int>(t - static_cast<int64_t>(e) * tiles_per_mat);
        tn = r / a.tiles_m;
        tm = r - tn * a.tiles_m;
    };

    if (warp == 0 && lane == 0) {   // producer, across tile boundaries
        int q = 0;   // stage uses so far
        bool ok = true;
        for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            int e, tm, tn;
            tile_of(t, e, tm, tn);
            const uint8_t* sfa = a.sfa + (static_cast<int64_t>(e) * a.rt_a + tm) * a.kc * 512;
            const uint8_t* sfb = a.sfb + (static_cast<int64_t>(e) * a.rt_b + tn) * a.kc * 512;
            for (int kt = 0; kt < nk; ++kt, ++q) {
                const int s = q % NP_STAGES;
                if (st[2] || !ng_wait(empty0 + 8 * s, ((q / NP_STAGES) & 1) ^ 1, a.wait_limit)) { ok = false; break; }
                const uint32_t sb = s_base + s * NP_STAGE_BYTES, bar = full0 + 8 * s;
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(NP_STAGE_BYTES)
                             : "memory");
                ng_tma_3d(sb, &amap, bar, kt * NG_BKB, tm * NG_M, e);
                ng_tma_3d(sb + NG_A_BYTES, &bmap, bar, kt * NG_BKB, tn * 128, e);
                const int64_t off = static_cast<int64_t>(4 * kt) * 512;
                ng_bulk(sb + NG_A_BYTES + NP_B_BYTES, sfa + off, NG_SFA_BYTES, bar);
                ng_bulk(sb + NG_A_BYTES + NP_B_BYTES + NG_SFA_BYTES, sfb + off, 2048, bar);
                st[0] = q + 1;
            }
        }
        if (!ok) st[2] = 1;
    } else if (warp == 1 && lane == 0) {   // scale copies and MMAs
        int q = 0, i = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
            const int b = i & 1, u = i >> 1;
            if (st[2] || !ng_wait(acce0 + 8 * b, (u & 1) ^ 1, a.wait_limit)) { ok = false; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t acc = tmem + 128u * static_cast<uint32_t>(b);
            for (int kt = 0; kt < nk; ++kt, ++q) {
                const int s = q % NP_STAGES;
                if (st[2] || !ng_wait(full0 + 8 * s, (q / NP_STAGES) & 1, a.wait_limit)) { ok = false; break; }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t sa = s_base + s * NP_STAGE_BYTES, sb = sa + NG_A_BYTES;
                const uint32_t ssfa = sb + NP_B_BYTES, ssfb = ssfa + NG_SFA_BYTES;
                const uint32_t tsf = tmem + NP_SF_COL + NP_SF_COLS * static_cast<uint32_t>(q & 1);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    ng_cp_sf(tsf + 4 * j, ng_desc_sf(ssfa + 512 * j));
                    ng_cp_sf(tsf + 16 + 4 * j, ng_desc_sf(ssfb + 512 * j));
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    ng_mma(acc, ng_desc_sw128(sa + 32 * j), ng_desc_sw128(sb + 32 * j), NP_IDESC, tsf + 4 * j,
                           tsf + 16 + 4 * j, (kt | j) != 0);
                ng_commit(empty0 + 8 * s);
                st[1] = q + 1;
            }
            if (!ok) break;
            ng_commit(accf0 + 8 * b);   // this tile's accumulator is complete once its MMAs are
        }
        if (!ok) st[2] = 1;
        ng_commit(done);
    } else if (warp >= 2) {   // epilogue: 4 warps, warp w reads TMEM lanes 32 (w % 4) ..
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;   // row of the tile
        int i = 0;
        for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
            const int b = i & 1, u = i >> 1;
            if (!ng_wait(accf0 + 8 * b, u & 1, a.wait_limit) || st[2]) { st[2] = 1; break; }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            int e, tm, tn;
            tile_of(t, e, tm, tn);
            const float gg = __fmul_rn(__ldg(a.gx + e), __ldg(a.gw + e));
            const uint32_t acc = tmem + 128u * static_cast<uint32_t>(b) + (static_cast<uint32_t>(quarter * 32) << 16);
            if (NP_STAGED && a.y_tma) {
                if (threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                ng_named_sync(1, 128);   // the previous tile's stores have read the staging tile
#pragma unroll 1
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    float v[32];
                    ng_ld32(acc + static_cast<uint32_t>(c0), v);
                    float4* row = reinterpret_cast<float4*>(outbuf + (c0 / 32) * (NG_M * 128) + r * 128);
#pragma unroll
                    for (int w = 0; w < 8; ++w)
                        row[w ^ (r & 7)] = make_float4(__fmul_rn(v[4 * w], gg), __fmul_rn(v[4 * w + 1], gg),
                                                       __fmul_rn(v[4 * w + 2], gg), __fmul_rn(v[4 * w + 3], gg));
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acce0 + 8 * b) : "memory");
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                ng_named_sync(1, 128);
                if (threadIdx.x == 64) {
                    for (int qq = 0; qq < 4; ++qq)
                        if (static_cast<int64_t>(tn) * 128 + 32 * qq < a.O)
                            ng_tma_store_3d(&ymap, o_base + qq * (NG_M * 128), tn * 128 + 32 * qq, tm * NG_M, e);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            } else {
                const int64_t m = static_cast<int64_t>(tm) * NG_M + r;
                float* yr = a.y + (static_cast<int64_t>(e) * a.T + m) * a.O;
#pragma unroll 1
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    float v[32];
                    ng_ld32(acc + static_cast<uint32_t>(c0), v);
                    const int64_t o0 = static_cast<int64_t>(tn) * 128 + c0;
                    if (m < a.T && o0 < a.O) {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            if (o0 + k < a.O) yr[o0 + k] = __fmul_rn(v[k], gg);
                    }
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acce0 + 8 * b) : "memory");
            }
        }
        if (threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }

    // teardown: the copies armed but not consumed and the MMAs committed,
    // with the default limit; then free TMEM
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = st[1]; k < st[0]; ++k)
            if (!ng_wait(full0 + 8 * (k % NP_STAGES), (k / NP_STAGES) & 1)) break;
        ng_wait(done, 0);
    }
    __syncthreads();
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
}

// ------------------------------------------------------------------ host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn ng_encode() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool nvfp4_gemm_take_timeouts() {
    unsigned n = 0;
    if (cudaMemcpyFromSymbol(&n, g_ng_timeouts, sizeof(n)) != cudaSuccess || n == 0) return false;
    const unsigned zero = 0;
    cudaMemcpyToSymbol(g_ng_timeouts, &zero, sizeof(zero));
    return true;
}

tq_status launch_amax(const tq_mat* W, float* amax, cudaStream_t st);   // imatrix.cu

}  // namespace tq

using namespace tq;

TQ_API tq_status tq_quant_nvfp4_act(const tq_mat* X, uint8_t* packed, uint8_t* scales, float* global_scale,
                                    tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(X, "tq_quant_nvfp4_act X");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(packed && scales && global_scale, "tq_quant_nvfp4_act: null output");
    TQ_REQUIRE(aligned16(packed), "tq_quant_nvfp4_act: packed not 16-byte aligned");
    const int64_t G = (X->cols + 15) / 16;
    const int64_t total = X->n_mat * X->rows * G;
    TQ_REQUIRE(total < (int64_t(1) << 32), "tq_quant_nvfp4_act: more than 2^32 blocks");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if ((s = launch_amax(X, global_scale, st)) != TQ_OK) return s;
    k_act_global<<<static_cast<unsigned>((X->n_mat + 255) / 256), 256, 0, st>>>(global_scale, X->n_mat);
    const GroupIndex gi(X->rows, G);
    const int64_t ms = X->n_mat > 1 ? X->mat_stride : 0;
    // one wave of resident blocks (a second, partial wave would leave most
    // SMs idle for its duration)
    int per_sm = 0;
    if ((X->dtype == TQ_BF16
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_act_nvfp4<uint16_t>, 256, 0)
             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_quant_act_nvfp4<float>, 256, 0)) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const unsigned grid =
        static_cast<unsigned>(min((total + 255) / 256, static_cast<int64_t>(num_sms()) * per_sm));
    if (X->dtype == TQ_BF16)
        k_quant_act_nvfp4<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(X->ptr), X->cols, X->ld, ms,
                                                          global_scale, gi, total, scales, packed);
    else
        k_quant_act_nvfp4<float><<<grid, 256, 0, st>>>(static_cast<const float*>(X->ptr), X->cols, X->ld, ms,
                                                       global_scale, gi, total, scales, packed);
    return check_launch("tq_quant_nvfp4_act");
}

TQ_API size_t tq_nvfp4_scales_mma_bytes(int64_t n_mat, int64_t rows, int64_t cols) {
    if (n_mat < 1 || rows < 1 || cols < 1) return 0;
    return static_cast<size_t>(n_mat * sf_row_tiles(rows) * sf_k_chunks((cols + 15) / 16) * 512);
}

TQ_API tq_status tq_nvfp4_scales_to_mma(const uint8_t* scales, int64_t n_mat, int64_t rows, int64_t cols,
                                        uint8_t* out, tq_stream_t stream) {
    clear_error();
    TQ_REQUIRE(scales && out, "tq_nvfp4_scales_to_mma: null pointer");
    TQ_REQUIRE(n_mat >= 1 && rows >= 1 && cols >= 1, "tq_nvfp4_scales_to_mma: empty shape");
    TQ_REQUIRE(aligned16(out), "tq_nvfp4_scales_to_mma: out not 16-byte aligned");
    const int64_t G = (cols + 15) / 16, RT = sf_row_tiles(rows), KC = sf_k_chunks(G);
    const int64_t words = n_mat * RT * KC * 128;
    const unsigned grid = static_cast<unsigned>(min((words + 255) / 256, static_cast<int64_t>(num_sms()) * 8));
    k_sf_to_mma<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(scales, rows, G, RT, KC, words,
                                                                           reinterpret_cast<uint32_t*>(out));
    return check_launch("tq_nvfp4_scales_to_mma");
}

TQ_API tq_status tq_gemm_nvfp4(const uint8_t* x_packed, const uint8_t* x_scales_mma, const float* x_global,
                               const uint8_t* w_packed, const uint8_t* w_scales_mma, const float* w_global,
                               int64_t n_mat, int64_t T, int64_t O, int64_t I, float* y, tq_stream_t stream) {
    clear_error();
    TQ_REQUIRE(x_packed && x_scales_mma && x_global && w_packed && w_scales_mma && w_global && y,
               "tq_gemm_nvfp4: null pointer");
    TQ_REQUIRE(n_mat >= 1 && T >= 1 && O >= 1 && I >= 1, "tq_gemm_nvfp4: empty shape");
    TQ_REQUIRE(I % 32 == 0, "tq_gemm_nvfp4: I must be a multiple of 32 (rows of packed codes 16-byte aligned)");
    TQ_REQUIRE(aligned16(x_packed) && aligned16(w_packed) && aligned16(x_scales_mma) && aligned16(w_scales_mma) &&
               aligned16(y), "tq_gemm_nvfp4: pointers must be 16-byte aligned");
    TQ_REQUIRE(n_mat <= 65535 && T < (int64_t(1) << 31) && O < (int64_t(1) << 31) && I < (int64_t(1) << 31),
               "tq_gemm_nvfp4: sizes out of range");
    EncodeTiledFn enc = ng_encode();
    if (!enc) return set_error(TQ_ERR_CUDA, "tq_gemm_nvfp4: cuTensorMapEncodeTiled unavailable");
    const int64_t rowb = I / 2;
#ifndef TQ_NG_N
#define TQ_NG_N 128
#endif
    constexpr int BN = TQ_NG_N;
    using C = NgCfg<BN>;
    CUtensorMap amap, bmap, ymap;
    const cuuint32_t estr[3] = {1, 1, 1};
    memset(&ymap, 0, sizeof ymap);
    const int y_tma = (O % 4) == 0;
    if (y_tma) {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(O), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(n_mat)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(O * 4), static_cast<cuuint64_t>(T * O * 4)};
        const cuuint32_t box[3] = {32, NG_M, 1};
        CUresult r = enc(&ymap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, y, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return set_error(TQ_ERR_CUDA, "tq_gemm_nvfp4: y tensor map (%d)", static_cast<int>(r));
    }
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(rowb), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(n_mat)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(rowb), static_cast<cuuint64_t>(T * rowb)};
        const cuuint32_t box[3] = {NG_BKB, NG_M, 1};
        CUresult r = enc(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(x_packed), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return set_error(TQ_ERR_CUDA, "tq_gemm_nvfp4: A tensor map (%d)", static_cast<int>(r));
    }
    {
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(rowb), static_cast<cuuint64_t>(O), static_cast<cuuint64_t>(n_mat)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(rowb), static_cast<cuuint64_t>(O * rowb)};
        const cuuint32_t box[3] = {NG_BKB, static_cast<cuuint32_t>(BN), 1};
        CUresult r = enc(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(w_packed), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return set_error(TQ_ERR_CUDA, "tq_gemm_nvfp4: B tensor map (%d)", static_cast<int>(r));
    }
    NgArgs a;
    a.T = T;
    a.O = O;
    a.tiles_m = static_cast<int>((T + NG_M - 1) / NG_M);
    const int64_t tiles_n = (O + BN - 1) / BN;
    a.nk = static_cast<int>((rowb + NG_BKB - 1) / NG_BKB);
    a.kc = sf_k_chunks((I + 15) / 16);
    a.rt_a = sf_row_tiles(T);
    a.rt_b = sf_row_tiles(O);
    a.sfa = x_scales_mma;
    a.sfb = w_scales_mma;
    a.gx = x_global;
    a.gw = w_global;
    a.y = y;
    a.y_tma = y_tma;
    a.wait_limit = pipeline_wait_limit();
    TQ_REQUIRE(a.kc == 4 * a.nk, "tq_gemm_nvfp4: internal tiling mismatch");
    const int64_t tiles = static_cast<int64_t>(a.tiles_m) * tiles_n;
    TQ_REQUIRE(tiles < (int64_t(1) << 31), "tq_gemm_nvfp4: too many tiles");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (NG_PERSISTENT && BN == 128) {
        static std::once_flag pattr;
        std::call_once(pattr, [] {
            cudaFuncSetAttribute(k_gemm_nvfp4_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize, NP_SMEM_BYTES);
        });
        const int64_t n_tiles = tiles * n_mat;
        const unsigned grid = static_cast<unsigned>(min(n_tiles, static_cast<int64_t>(num_sms())));
        k_gemm_nvfp4_persistent<<<grid, NP_THREADS, NP_SMEM_BYTES, st>>>(amap, bmap, ymap, a,
                                                                         static_cast<int>(tiles_n), n_tiles);
        return check_launch("tq_gemm_nvfp4");
    }
    static std::once_flag attr;
    std::call_once(attr, [] {
        cudaFuncSetAttribute(k_gemm_nvfp4<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    });
    k_gemm_nvfp4<BN><<<dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(n_mat)), NG_THREADS, C::SMEM_BYTES,
                   st>>>(amap, bmap, ymap, a);
    return check_launch("tq_gemm_nvfp4");
}
