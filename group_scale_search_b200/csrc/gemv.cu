// Decode-time consumer of the packed formats: y = What x for a few token
// vectors (B <= 8), What as tq_dequant defines it (int3 s v, int4 s (q - z),
// NVFP4 fl32(fl32(g dec(e)) dec(c))), read straight from the records.  This is
// the step after packing: the int3-g64 format page ("int3-g64 (fmt=5)",
// colibri PR #168) multiplies over the packed records in exact fp32 with the
// scale applied once per group (Design, Kernel bullet), has no CUDA path for
// the format (Design, GPU bullet) and calls the decode regime fetch-bound
// (Why this format, item 2).  At a few tokens the product is bound by the HBM
// read of the records, so it runs on the CUDA cores, not the tensor cores.
//
// Arithmetic: per group (NVFP4: per block) the integer (or E2M1) values d are
// multiplied with x in fp32 FMAs (d x is exact inside the FMA), and the
// group's sum is scaled once: y += s * sum(d x).  In exact arithmetic that is
// sum(What x); the rounding differs from multiplying the rounded What by x by
// at most one unit roundoff per term plus the summation's own roundings.
//
// B200 mapping.  A block of 8 warps stages x (converted to fp32) in shared
// memory, swizzled so that lane l's 32 x values of its current quad lie in 8
// float4 slots at a stride of 32 float4 (conflict-free LDS.128).  Each warp
// takes R consecutive rows of one matrix; lane l takes the quads (32 weights)
// l, l + 32, ... of those rows: one 16-byte load of codes per row per quad
// (int4: a quarter record; NVFP4: two block records; int3: half a record, as
// 8 + 4 bytes), so consecutive lanes read consecutive bytes of a row.  The R
// rows share every x load.  Integers become floats as 2^23 + k (byte_perm)
// and (2^23 + k) - (2^23 + z) is exact, paired in fp32x2 adds; products go
// into fp32x2 FMAs.  Lane sums are added by a fixed butterfly, so the result
// does not depend on scheduling.  Blocks take contiguous runs of row chunks,
// so x is staged again only when the matrix (per-matrix x) or the column tile
// (I beyond one tile) changes.
#include <atomic>
#include <mutex>

#include "walk.cuh"

namespace tq {

constexpr int GV_WARPS = 8;
constexpr int GV_THREADS = GV_WARPS * 32;
constexpr int64_t GV_XS_BYTES = 96 * 1024;   // x tile budget: two blocks per SM (their register share)

template <int B> __host__ __device__ constexpr int gv_rows() { return B <= 2 ? 4 : 2; }   // rows per warp

// Columns of x per staged tile: a multiple of 1024 (32 lanes x 32 weights),
// no more than the row needs.
inline int64_t gv_tile(int64_t B, int64_t I) {
    int64_t k = GV_XS_BYTES / (B * 4 * 1024);
    k = k < 1 ? 1 : k;
    const int64_t need = (I + 1023) / 1024;
    return 1024 * (need < k ? need : k);
}

// x[b][j0 .. j0 + TI) of matrix e as fp32 into the swizzled tile (zeros past I).
__device__ __forceinline__ void gv_stage(float4* xs, const void* x, bool x_bf16, int64_t xoff, int64_t I,
                                         int64_t j0, int64_t TI, int B, bool vec) {
    const int64_t slots = TI >> 2;   // float4 slots per vector, a multiple of GV_THREADS
    for (int b = 0; b < B; ++b) {
        for (int64_t s = threadIdx.x; s < slots; s += GV_THREADS) {
            const int64_t l = s & 31, ti = s >> 5;
            const int64_t j = j0 + (((ti >> 3) * 32 + l) * 32) + 4 * (ti & 7);
            const int64_t base = xoff + b * I + j;
            float f[4];
            if (x_bf16) {
                const uint16_t* p = static_cast<const uint16_t*>(x) + base;
                if (vec && j + 3 < I) {
                    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
                    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
                    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c) f[c] = j + c < I ? bf16_bits_to_f32(__ldg(p + c)) : 0.f;
                }
            } else {
                const float* p = static_cast<const float*>(x) + base;
                if (vec && j + 3 < I) {
                    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
                    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c) f[c] = j + c < I ? __ldg(p + c) : 0.f;
                }
            }
            xs[b * slots + s] = make_float4(f[0], f[1], f[2], f[3]);
        }
    }
}

// One quad (32 weights) of one row: codes and per-group factors.
struct Quad {
    uint32_t w[4];   // int: 8 nibbles per word (word k = weights 8k..8k+7); NVFP4: 2 E2M1 codes per byte
    float s0, s1;    // int: group scale (s1 unused); NVFP4: the two blocks' fl32(g dec(e))
    int z;           // int: zero-point (int3: 4)
};

// A16: NVFP4 rows start on 16-byte boundaries (an even number of blocks per row).
template <int FMT, bool A16>
__device__ __forceinline__ Quad gv_load(const uint8_t* rec_row, const void* sc_row, const uint8_t* zp_row, float g,
                                        int64_t q, int64_t G) {
    Quad u;
    if constexpr (FMT == TQ_INT4_G128_ASYM) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(rec_row) + q);
        u.w[0] = v.x; u.w[1] = v.y; u.w[2] = v.z; u.w[3] = v.w;
        u.s0 = __ldg(static_cast<const float*>(sc_row) + (q >> 2));
        u.z = __ldg(zp_row + (q >> 2));
    } else if constexpr (FMT == TQ_INT3_G64_SYM) {
        const uint8_t* rec = rec_row + (q >> 1) * 24;
        const int h = static_cast<int>(q & 1);
        const uint2 lo = __ldg(reinterpret_cast<const uint2*>(rec + 8 * h));
        const uint32_t hi = __ldg(reinterpret_cast<const uint32_t*>(rec + 16 + 4 * h));
        u.w[0] = int3_nibbles(lo.x & 0xffffu, hi & 0xffu);
        u.w[1] = int3_nibbles(lo.x >> 16, (hi >> 8) & 0xffu);
        u.w[2] = int3_nibbles(lo.y & 0xffffu, (hi >> 16) & 0xffu);
        u.w[3] = int3_nibbles(lo.y >> 16, hi >> 24);
        u.s0 = __ldg(static_cast<const float*>(sc_row) + (q >> 1));
        u.z = 4;
    } else {
        const uint8_t* sc = static_cast<const uint8_t*>(sc_row) + 2 * q;
        if constexpr (A16) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(rec_row) + q);
            u.w[0] = v.x; u.w[1] = v.y; u.w[2] = v.z; u.w[3] = v.w;
            const unsigned e2 = __ldg(reinterpret_cast<const uint16_t*>(sc));
            u.s0 = __fmul_rn(g, e4m3_value(e2 & 0xffu));
            u.s1 = __fmul_rn(g, e4m3_value(e2 >> 8));
        } else {   // the second block may lie past the row (odd block count): it then counts as zero
            const uint2 a = __ldg(reinterpret_cast<const uint2*>(rec_row) + 2 * q);
            const bool two = 2 * q + 1 < G;
            const uint2 b = two ? __ldg(reinterpret_cast<const uint2*>(rec_row) + 2 * q + 1) : make_uint2(0u, 0u);
            u.w[0] = a.x; u.w[1] = a.y; u.w[2] = b.x; u.w[3] = b.y;
            u.s0 = __fmul_rn(g, e4m3_value(__ldg(sc)));
            u.s1 = two ? __fmul_rn(g, e4m3_value(__ldg(sc + 1))) : 0.f;
        }
        u.z = 0;
    }
    return u;
}

// d values of word k of an integer quad, as 4 pairs (elements 2i, 2i+1):
// (2^23 + code) - (2^23 + z), exact.
__device__ __forceinline__ void gv_int_pairs(uint32_t bits, float2 noff, float2 d[4]) {
    const uint32_t ev = bits & 0x0f0f0f0fu, od = (bits >> 4) & 0x0f0f0f0fu;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const unsigned sel = 0x5640u | static_cast<unsigned>(i);   // bytes: (byte i, 0, 0, 0x4b)
        d[i] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(ev, 0x4b00u, sel)),
                                      __uint_as_float(__byte_perm(od, 0x4b00u, sel))), noff);
    }
}

// acc[r][b] += s * sum over the quad's weights of d x (NVFP4: per block),
// for the R rows' quads u and lane's x slots at xq (vector b at b * slots).
template <int FMT, int B, int R>
__device__ __forceinline__ void gv_quad(const Quad (&u)[R], const float4* xq, int64_t slots, float (&acc)[R][B]) {
    float2 p[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) p[r][b] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {        // word k: weights 8k .. 8k + 7 of the quad
        float4 xv[B][2];                 // float4 slots 2k, 2k + 1: shared by the R rows
#pragma unroll
        for (int b = 0; b < B; ++b) {
            xv[b][0] = xq[b * slots + (2 * k) * 32];
            xv[b][1] = xq[b * slots + (2 * k + 1) * 32];
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            float2 d[4];                 // pairs (8k + 2i, 8k + 2i + 1)
            if constexpr (FMT == TQ_NVFP4_G16) {
#pragma unroll
                for (int i = 0; i < 4; ++i) d[i] = e2m1x2_to_f32((u[r].w[k] >> (8 * i)) & 0xffu);
            } else {
                const float o = f23(static_cast<unsigned>(u[r].z) & 0xffu);
                gv_int_pairs(u[r].w[k], make_float2(-o, -o), d);
            }
#pragma unroll
            for (int b = 0; b < B; ++b) {
                p[r][b] = __ffma2_rn(d[0], make_float2(xv[b][0].x, xv[b][0].y), p[r][b]);
                p[r][b] = __ffma2_rn(d[1], make_float2(xv[b][0].z, xv[b][0].w), p[r][b]);
                p[r][b] = __ffma2_rn(d[2], make_float2(xv[b][1].x, xv[b][1].y), p[r][b]);
                p[r][b] = __ffma2_rn(d[3], make_float2(xv[b][1].z, xv[b][1].w), p[r][b]);
            }
        }
        if constexpr (FMT == TQ_NVFP4_G16) {
            if (k == 1) {   // end of the first block: scale it, restart the partial sums
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int b = 0; b < B; ++b) {
                        acc[r][b] = __fmaf_rn(u[r].s0, __fadd_rn(p[r][b].x, p[r][b].y), acc[r][b]);
                        p[r][b] = make_float2(0.f, 0.f);
                    }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b)
            acc[r][b] = __fmaf_rn(FMT == TQ_NVFP4_G16 ? u[r].s1 : u[r].s0, __fadd_rn(p[r][b].x, p[r][b].y),
                                  acc[r][b]);
}

// y[e][b][o] = sum_j What[e, o, j] x[e][b][j]; x [n_mat or 1][B][I] (x_ms
// elements between matrices, 0 when shared), y [n_mat][B][O] fp32.
// The block's warps form 8 >> wl row groups of 1 << wl warps; a row group
// takes R rows of a chunk and its warps split the row's quads (warp slice s
// takes quads (32 i + s) * 32 + lane ... in steps of 32 << wl), their sums
// added in slice order.  Chunks of (8 >> wl) * R rows of one matrix, cpm
// per matrix.  Each lane's next quads are loaded before the current ones
// are used.
template <int FMT, int B, bool A16>
__global__ void __launch_bounds__(GV_THREADS)
k_dequant_gemv(const uint8_t* __restrict__ packed, const void* __restrict__ scales,
               const uint8_t* __restrict__ zeros, const float* __restrict__ gs, int64_t n_mat, int64_t O,
               int64_t I, const void* __restrict__ x, int x_bf16, int64_t x_ms, int64_t TI, int64_t cpm, int wl,
               float* __restrict__ y) {
    constexpr int R = gv_rows<B>();
    using F = FmtTraits<FMT>;
    extern __shared__ float4 xs[];
    __shared__ float red[GV_WARPS][R * B];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = warp & ((1 << wl) - 1), rgi = warp >> wl;
    const int64_t rows_per_chunk = static_cast<int64_t>(GV_WARPS >> wl) * R;
    const int64_t G = (I + F::group - 1) / F::group;
    const int64_t nq = (I + 31) >> 5;                 // quads per row
    const int64_t nT = (I + TI - 1) / TI;             // column tiles
    const int64_t slots = TI >> 2;
    const int64_t rec_bytes = G * F::rec;             // record bytes per row
    const int64_t qstep = static_cast<int64_t>(32) << wl;
    const bool vec = (I % 4) == 0 && (x_ms % 4) == 0;
    const int64_t nchunks = n_mat * cpm;
    const int64_t c0 = nchunks * blockIdx.x / gridDim.x, c1 = nchunks * (blockIdx.x + 1) / gridDim.x;
    int64_t staged_e = -1, staged_t = -1;
    for (int64_t c = c0; c < c1; ++c) {
        const int64_t e = c / cpm;
        const int64_t ob = (c - e * cpm) * rows_per_chunk + rgi * R;
        const float g = FMT == TQ_NVFP4_G16 ? __ldg(gs + e) : 0.f;
        const int64_t row0 = e * O;   // this matrix's first row
        const uint8_t* rec_m = packed + row0 * rec_bytes;
        const void* sc_m = FMT == TQ_NVFP4_G16 ? static_cast<const void*>(static_cast<const uint8_t*>(scales) + row0 * G)
                                               : static_cast<const void*>(static_cast<const float*>(scales) + row0 * G);
        const uint8_t* zp_m = FMT == TQ_INT4_G128_ASYM ? zeros + row0 * G : nullptr;
        int rr[R];   // rows within the matrix; rows past O repeat the last one and are not stored
#pragma unroll
        for (int r = 0; r < R; ++r) rr[r] = static_cast<int>(min(ob + r, O - 1));
        auto load = [&](Quad (&u)[R], int64_t q) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int64_t ro = rr[r];
                u[r] = gv_load<FMT, A16>(rec_m + ro * rec_bytes,
                                         FMT == TQ_NVFP4_G16
                                             ? static_cast<const void*>(static_cast<const uint8_t*>(sc_m) + ro * G)
                                             : static_cast<const void*>(static_cast<const float*>(sc_m) + ro * G),
                                         FMT == TQ_INT4_G128_ASYM ? zp_m + ro * G : nullptr, g, q, G);
            }
        };
        float acc[R][B];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int b = 0; b < B; ++b) acc[r][b] = 0.f;
        for (int64_t t = 0; t < nT; ++t) {
            if (staged_t != t || (staged_e != e && x_ms != 0)) {   // block-uniform
                __syncthreads();
                gv_stage(xs, x, x_bf16 != 0, e * x_ms, I, t * TI, TI, B, vec);
                __syncthreads();
                staged_t = t;
                staged_e = e;
            }
            const int64_t qb = t * (TI >> 5);
            const int64_t nqt = min(TI >> 5, nq - qb);
            int64_t qt = static_cast<int64_t>(slice) * 32 + lane;   // quad within the tile
            bool have = qt < nqt;
            Quad cur[R];
            if (have) load(cur, qb + qt);
            while (have) {
                const int64_t qn = qt + qstep;
                const bool hn = qn < nqt;
                Quad nxt[R];
                if (hn) load(nxt, qb + qn);
                gv_quad<FMT, B, R>(cur, xs + (qt >> 5) * 256 + lane, slots, acc);
#pragma unroll
                for (int r = 0; r < R; ++r) cur[r] = nxt[r];
                qt = qn;
                have = hn;
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int b = 0; b < B; ++b) {
                float s = acc[r][b];
#pragma unroll
                for (int off = 16; off; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(FULL, s, off));
                if (wl == 0) {
                    if (lane == 0 && ob + r < O) y[(e * B + b) * O + ob + r] = s;
                } else if (lane == 0) {
                    red[warp][r * B + b] = s;
                }
            }
        }
        if (wl != 0) {   // block-uniform: add the slices' sums in slice order
            __syncthreads();
            if (slice == 0 && lane < R * B) {
                float s = red[warp][lane];
                for (int k = 1; k < (1 << wl); ++k) s = __fadd_rn(s, red[warp + k][lane]);
                const int r = lane / B, b = lane - (lane / B) * B;
                if (ob + r < O) y[(e * B + b) * O + ob + r] = s;
            }
            __syncthreads();
        }
    }
}

// Resident blocks per SM of k_dequant_gemv<FMT, B, A16> for each tile width
// (1024 .. 24576 columns), found once; the dynamic shared memory limit is
// raised once per instantiation.
template <int FMT, int B, bool A16>
int gv_blocks_per_sm(int64_t TI, size_t smem) {
    static std::atomic<int> cache[25];
    static std::once_flag raised;
    auto kern = k_dequant_gemv<FMT, B, A16>;
    std::call_once(raised, [&] {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(GV_XS_BYTES));
    });
    const int64_t i = TI / 1024;
    int n = i < 25 ? cache[i].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, GV_THREADS, smem) != cudaSuccess || n < 1) n = 1;
        if (i < 25) cache[i].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int FMT, int B, bool A16>
void launch_gemv(const uint8_t* packed, const void* scales, const uint8_t* zeros, const float* gs, int64_t n_mat,
                 int64_t O, int64_t I, const void* x, bool x_bf16, int64_t x_ms, float* y, cudaStream_t st) {
    constexpr int R = gv_rows<B>();
    const int64_t TI = gv_tile(B, I);
    const size_t smem = static_cast<size_t>(B * TI * 4);
    const int per_sm = gv_blocks_per_sm<FMT, B, A16>(TI, smem);
    const int64_t slots = static_cast<int64_t>(num_sms()) * per_sm;
    // Split rows' quads over more warps while the chunks do not fill the
    // resident blocks and every warp keeps at least one quad per lane.
    const int64_t nq = (I + 31) / 32;
    int wl = 0;
    auto chunks = [&](int l) { return n_mat * ((O + (GV_WARPS >> l) * R - 1) / ((GV_WARPS >> l) * R)); };
    while (wl < 3 && chunks(wl) < slots && nq >= (static_cast<int64_t>(32) << (wl + 1))) ++wl;
    const int64_t cpm = (O + (GV_WARPS >> wl) * R - 1) / ((GV_WARPS >> wl) * R);
    const int64_t grid = min(n_mat * cpm, slots);
    k_dequant_gemv<FMT, B, A16><<<static_cast<unsigned>(grid), GV_THREADS, smem, st>>>(
        packed, scales, zeros, gs, n_mat, O, I, x, x_bf16 ? 1 : 0, x_ms, TI, cpm, wl, y);
}

template <int FMT, bool A16>
void launch_gemv_b(int64_t B, const uint8_t* packed, const void* scales, const uint8_t* zeros, const float* gs,
                   int64_t n_mat, int64_t O, int64_t I, const void* x, bool x_bf16, int64_t x_ms, float* y,
                   cudaStream_t st) {
    switch (B) {
        case 1: launch_gemv<FMT, 1, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        case 2: launch_gemv<FMT, 2, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        case 3: launch_gemv<FMT, 3, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        case 4: launch_gemv<FMT, 4, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        case 5: launch_gemv<FMT, 5, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        case 6: launch_gemv<FMT, 6, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        case 7: launch_gemv<FMT, 7, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
        default: launch_gemv<FMT, 8, A16>(packed, scales, zeros, gs, n_mat, O, I, x, x_bf16, x_ms, y, st); break;
    }
}

}  // namespace tq

using namespace tq;

TQ_API tq_status tq_dequant_gemv(const uint8_t* packed, int32_t fmt, const void* scales, const uint8_t* zeros,
                                 const float* global_scale, int64_t n_mat, int64_t O, int64_t I, const void* x,
                                 int32_t x_dtype, int64_t B, int64_t x_mat_stride, float* y, tq_stream_t stream) {
    clear_error();
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant_gemv: unknown format %d", fmt);
    if (elem_bytes(x_dtype) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant_gemv: x dtype %d", x_dtype);
    TQ_REQUIRE(packed && scales && x && y, "tq_dequant_gemv: null pointer");
    TQ_REQUIRE(n_mat >= 1 && O >= 1 && I >= 1, "tq_dequant_gemv: empty shape");
    TQ_REQUIRE(B >= 1 && B <= 8, "tq_dequant_gemv: B must be in [1, 8]");
    TQ_REQUIRE(x_mat_stride == 0 || x_mat_stride >= B * I, "tq_dequant_gemv: x_mat_stride must be 0 or >= B*I");
    TQ_REQUIRE(aligned16(packed) && aligned16(x), "tq_dequant_gemv: packed/x not 16-byte aligned");
    TQ_REQUIRE(fmt != TQ_INT4_G128_ASYM || zeros != nullptr, "tq_dequant_gemv: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_dequant_gemv: NVFP4 needs global_scale");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t xms = n_mat > 1 ? x_mat_stride : 0;
    const bool xb = x_dtype == TQ_BF16;
    if (fmt == TQ_INT3_G64_SYM) {
        launch_gemv_b<TQ_INT3_G64_SYM, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else if (fmt == TQ_INT4_G128_ASYM) {
        launch_gemv_b<TQ_INT4_G128_ASYM, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else if (((I + 15) / 16) % 2 == 0 && (reinterpret_cast<uintptr_t>(scales) & 1u) == 0) {
        launch_gemv_b<TQ_NVFP4_G16, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else {
        launch_gemv_b<TQ_NVFP4_G16, false>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    }
    return check_launch("tq_dequant_gemv");
}
