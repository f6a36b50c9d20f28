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
// into fp32x2 FMAs.  int3 codes are decoded by position across the quad's 4
// octets (the low-plane bytes gathered with one byte_perm, the high-plane bit
// shifted into place), so x is staged in that order for int3.  E2M1 and E4M3
// codes go through the hardware f16x2 conversions.  Lane sums are added by a
// fixed butterfly, so the result does not depend on scheduling.  Blocks take
// contiguous runs of row chunks, so x is staged again only when the matrix
// (per-matrix x) or the column tile (I beyond one tile) changes; a chunk's
// first code loads are issued before x is staged.  Rows of few quads are
// split over 2, 4 or 8 warps so that small matrices still fill the GPU.
//
// What bounds it (ncu, one B200): the decode instructions.  At B = 1 the
// kernel issues about 4.5 (NVFP4) to 5 (int3) instructions per weight, and
// the ALU pipe, not DRAM, is the busiest unit; small matrices (a few MB of
// records) are bound by latency (x staging, one HBM round trip, the launch).

#include <atomic>
#include <mutex>

#include "walk.cuh"

namespace tq {

// Warps per block and x tile budget (bytes of shared memory per block):
// B = 1 runs GV_WARPS1 warps per block, more vectors 8 warps at up to 128
// registers (two blocks per SM).
constexpr int GV_WARPS1 = 8;
template <int B> __host__ __device__ constexpr int gv_warps() { return B == 1 ? GV_WARPS1 : 8; }
template <int B> __host__ __device__ constexpr int gv_threads() { return gv_warps<B>() * 32; }
template <int B> __host__ __device__ constexpr int64_t gv_xs_bytes() { return B == 1 ? 216 * 1024 * GV_WARPS1 / 24 : 72 * 1024; }

template <int B> __host__ __device__ constexpr int gv_rows() { return B <= 2 ? 4 : 2; }   // rows per warp
template <int B> __host__ __device__ constexpr int gv_min_blocks() { return B == 1 ? 24 / GV_WARPS1 : 2; }   // per SM
constexpr bool GV_DB = false;   // double-buffered code loads (measured slower)

// Columns of x per staged tile: a multiple of 1024 (32 lanes x 32 weights),
// no more than the row needs.
template <int B>
inline int64_t gv_tile(int64_t I) {
    int64_t k = gv_xs_bytes<B>() / (B * 4 * 1024);
    k = k < 1 ? 1 : k;
    const int64_t need = (I + 1023) / 1024;
    return 1024 * (need < k ? need : k);
}

// x[b][j0 .. j0 + TI) of matrix e as fp32 into the swizzled tile (zeros past
// I).  Slot i (0..7) of a lane's quad holds 4 of the quad's 32 columns:
// 4i .. 4i + 3 (int4, NVFP4), or i, 8 + i, 16 + i, 24 + i (int3: the
// columns at position i of the quad's 4 octets, in the order its decoding
// produces them).  A thread stages one quad (32 columns) at a time: four
// 16-byte loads of bf16 x (eight of fp32) where the quad lies inside the row
// and vec (16-byte aligned rows) holds, then its 8 slots.
template <bool OCT_MAJOR>
__device__ __forceinline__ void gv_stage(float4* xs, const void* x, bool x_bf16, int64_t xoff, int64_t I,
                                         int64_t j0, int64_t TI, int B, bool vec) {
    const int64_t slots = TI >> 2;   // float4 slots per vector
    const int64_t nqt = TI >> 5;     // quads of the tile
    for (int b = 0; b < B; ++b) {
        const int64_t base = xoff + b * I;
        for (int64_t qd = threadIdx.x; qd < nqt; qd += blockDim.x) {
            const int64_t jq = j0 + qd * 32;   // the quad's first column
            float4* dst = xs + b * slots + (qd >> 5) * 256 + (qd & 31);   // slot i of the quad at dst[32 i]
            if (vec && x_bf16 && jq + 31 < I) {   // raw bf16 words, widened as the slots are written
                const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + base + jq);
                uint32_t w[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 u = __ldg(p + v);
                    w[4 * v] = u.x; w[4 * v + 1] = u.y; w[4 * v + 2] = u.z; w[4 * v + 3] = u.w;
                }
                auto col = [&](int c) {   // column c of the quad: word c / 2, low half for even c
                    return __uint_as_float((c & 1) ? (w[c >> 1] & 0xffff0000u) : (w[c >> 1] << 16));
                };
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[32 * i] = OCT_MAJOR ? make_float4(col(i), col(8 + i), col(16 + i), col(24 + i))
                                            : make_float4(col(4 * i), col(4 * i + 1), col(4 * i + 2), col(4 * i + 3));
                continue;
            }
            // fp32 x, or a quad at the row's end / rows not 16-byte aligned: slot by slot
#pragma unroll 1
            for (int i = 0; i < 8; ++i) {
                float f[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int64_t j = jq + (OCT_MAJOR ? 8 * c + i : 4 * i + c);
                    f[c] = j < I ? (x_bf16 ? bf16_bits_to_f32(__ldg(static_cast<const uint16_t*>(x) + base + j))
                                           : __ldg(static_cast<const float*>(x) + base + j))
                                 : 0.f;
                }
                dst[32 * i] = make_float4(f[0], f[1], f[2], f[3]);
            }
        }
    }
}

// The two E4M3 values of a 16-bit pair of codes (low byte first) as fp32,
// exactly (every E4M3 value is an f16 value).
__device__ __forceinline__ float2 e4m3x2_to_f32(unsigned two_codes) {
    unsigned h2;
    asm("{ .reg .b16 t; cvt.u16.u32 t, %1; cvt.rn.f16x2.e4m3x2 %0, t; }" : "=r"(h2) : "r"(two_codes));
    __half2_raw raw;
    raw.x = static_cast<unsigned short>(h2 & 0xffffu);
    raw.y = static_cast<unsigned short>(h2 >> 16);
    return __half22float2(__half2(raw));
}

// One quad (32 weights) of one row: codes and per-group factors.
struct Quad {
    uint32_t w[4];   // int4: 8 nibbles per word (word k = weights 8k..8k+7); NVFP4: 2 E2M1 codes per byte;
                     // int3: low-plane bytes gathered by position (w0: positions 0-3, w1: 4-7; byte o =
                     // octet o), w2 = high plane (byte o = octet o)
    float s0, s1;    // int: group scale (s1 unused); NVFP4: the two blocks' fl32(g dec(e))
    int z;           // int4: zero-point
};

// Where the current quads of a warp's R rows sit in the records, scales and
// zero-points: one base pointer per array for the first row and 32-bit row
// offsets (the rows are consecutive; rows past the matrix repeat its last
// row), moved on by dq quads (a multiple of 32) without multiplications.
// A16: NVFP4 rows start on 16-byte boundaries (an even number of blocks per row).
template <int FMT, bool A16, int R>
struct GvRows {
    const uint8_t* c;    // codes of the first row's quad (int3: its low-plane half)
    const uint8_t* s;    // scales of the first row's group (bytes)
    const uint8_t* z;    // int4: zero-points
    int cof[R], gof[R];  // row offsets: record bytes, groups
    int ho;              // int3: high-plane half minus low-plane half
    int q, G;            // NVFP4 rows with an odd block count: the last quad may hold one block
    __device__ __forceinline__ void init(const uint8_t* packed, const void* scales, const uint8_t* zeros, int G_,
                                         int64_t row0, const int (&rr)[R], int q_) {
        constexpr int rec = FmtTraits<FMT>::rec, group = FmtTraits<FMT>::group;
        G = G_;
        q = q_;
        const int64_t g0 = row0 * G;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            cof[r] = rr[r] * G * rec;
            gof[r] = rr[r] * G;
        }
        const int qg = q * 32 / group;   // the quad's group (NVFP4: its first block)
        if constexpr (FMT == TQ_INT3_G64_SYM) {
            const int h = q & 1;
            c = packed + g0 * rec + static_cast<int64_t>(qg) * rec + 8 * h;
            ho = 16 - 4 * h;
        } else {
            c = packed + g0 * rec + static_cast<int64_t>(q) * 16;
        }
        s = static_cast<const uint8_t*>(scales) + (g0 + qg) * (FMT == TQ_NVFP4_G16 ? 1 : 4);
        z = is_int4(FMT) ? zeros + g0 + qg : nullptr;
    }
    __device__ __forceinline__ Quad load(int r, float g) const {
        Quad u;
        const uint8_t* cr = c + cof[r];
        if constexpr (is_int4(FMT)) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(cr));
            u.w[0] = v.x; u.w[1] = v.y; u.w[2] = v.z; u.w[3] = v.w;
            u.s0 = __ldg(reinterpret_cast<const float*>(s) + gof[r]);
            u.z = __ldg(z + gof[r]);
        } else if constexpr (FMT == TQ_INT3_G64_SYM) {
            const uint2 lo = __ldg(reinterpret_cast<const uint2*>(cr));
            u.w[0] = __byte_perm(lo.x, lo.y, 0x6420u);   // byte o: octet o's low-plane byte for positions 0-3
            u.w[1] = __byte_perm(lo.x, lo.y, 0x7531u);   // ... for positions 4-7
            u.w[2] = __ldg(reinterpret_cast<const uint32_t*>(cr + ho));
            u.s0 = __ldg(reinterpret_cast<const float*>(s) + gof[r]);
        } else {
            unsigned e2;   // the two blocks' E4M3 codes, first in the low byte
            const uint8_t* sr = s + gof[r];
            if constexpr (A16) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(cr));
                u.w[0] = v.x; u.w[1] = v.y; u.w[2] = v.z; u.w[3] = v.w;
                e2 = __ldg(reinterpret_cast<const uint16_t*>(sr));
            } else {   // the second block may lie past the row: it then counts as zero (code 0)
                const uint2 a = __ldg(reinterpret_cast<const uint2*>(cr));
                const bool two = 2 * q + 1 < G;
                const uint2 b = two ? __ldg(reinterpret_cast<const uint2*>(cr) + 1) : make_uint2(0u, 0u);
                u.w[0] = a.x; u.w[1] = a.y; u.w[2] = b.x; u.w[3] = b.y;
                e2 = __ldg(sr) | (two ? static_cast<unsigned>(__ldg(sr + 1)) << 8 : 0u);
            }
            const float2 d = e4m3x2_to_f32(e2 & 0x7f7fu);   // magnitudes, as tq_dequant reads the codes
            u.s0 = __fmul_rn(g, d.x);
            u.s1 = __fmul_rn(g, d.y);
        }
        return u;
    }
    __device__ __forceinline__ void next(int dq) {
        if constexpr (is_int4(FMT)) {   // dq quads = dq * 32 / group groups
            constexpr int qpg = FmtTraits<FMT>::group / 32;
            c += 16 * dq; s += 4 * (dq / qpg); z += dq / qpg;
        } else if constexpr (FMT == TQ_INT3_G64_SYM) {
            c += 12 * dq; s += 2 * dq;
        } else {
            c += 16 * dq; s += 2 * dq; q += dq;
        }
    }
};

// d values of word k of an int4 quad, as 4 pairs (elements 2i, 2i+1):
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

// v = u - 4 of position a (0..7) of the quad's 4 octets (octets 0, 1 in d0,
// octets 2, 3 in d1): u = low-plane bits 2(a & 3).. of the gathered byte,
// plus 4 x the high-plane bit a of the octet's byte; (2^23 + u) - (2^23 + 4).
__device__ __forceinline__ void gv_int3_pos(const Quad& q, int a, float2& d0, float2& d1) {
    const uint32_t lo = (q.w[a >> 2] >> (2 * (a & 3))) & 0x03030303u;
    const uint32_t hs = a >= 2 ? (q.w[2] >> (a - 2)) : (q.w[2] << (2 - a));
    const uint32_t u = (hs & 0x04040404u) | lo;
    const float o = f23(4u);
    const float2 noff = make_float2(-o, -o);
    d0 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4b00u, 0x5640u)),
                                __uint_as_float(__byte_perm(u, 0x4b00u, 0x5641u))), noff);
    d1 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(u, 0x4b00u, 0x5642u)),
                                __uint_as_float(__byte_perm(u, 0x4b00u, 0x5643u))), noff);
}

// The 8 E2M1 values of a word (low nibble of byte 0 first) as fp32 pairs.
__device__ __forceinline__ void gv_e2m1x8(uint32_t w, float2 d[4]) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2_raw raw;
        raw.x = static_cast<unsigned short>(h[i] & 0xffffu);
        raw.y = static_cast<unsigned short>(h[i] >> 16);
        d[i] = __half22float2(__half2(raw));
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
            float2 d[4];                 // d[0], d[1] pair with slot 2k; d[2], d[3] with slot 2k + 1
            if constexpr (FMT == TQ_NVFP4_G16) {
                gv_e2m1x8(u[r].w[k], d);
            } else if constexpr (FMT == TQ_INT3_G64_SYM) {
                gv_int3_pos(u[r], 2 * k, d[0], d[1]);
                gv_int3_pos(u[r], 2 * k + 1, d[2], d[3]);
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
__global__ void __launch_bounds__(gv_threads<B>(), gv_min_blocks<B>())
k_dequant_gemv(const uint8_t* __restrict__ packed, const void* __restrict__ scales,
               const uint8_t* __restrict__ zeros, const float* __restrict__ gs, int64_t n_mat, int64_t O,
               int64_t I, const void* __restrict__ x, int x_bf16, int64_t x_ms, int64_t TI, int64_t cpm, int wl,
               float* __restrict__ y) {
    constexpr int R = gv_rows<B>();
    using F = FmtTraits<FMT>;
    extern __shared__ float4 xs[];
    constexpr int GV_WARPS = gv_warps<B>();
    __shared__ float red[GV_WARPS][R * B];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = warp & ((1 << wl) - 1), rgi = warp >> wl;
    const int64_t rows_per_chunk = static_cast<int64_t>(GV_WARPS >> wl) * R;
    const int64_t G = (I + F::group - 1) / F::group;
    const int64_t nq = (I + 31) >> 5;                 // quads per row
    const int64_t nT = (I + TI - 1) / TI;             // column tiles
    const int64_t slots = TI >> 2;
    const int qstep = 32 << wl;
    // 16-byte x loads: rows (and matrices) of x start on 16-byte boundaries
    const int64_t xa = x_bf16 ? 8 : 4;
    const bool vec = (I % xa) == 0 && (x_ms % xa) == 0;
    const int64_t nchunks = n_mat * cpm;
    const int64_t c0 = nchunks * blockIdx.x / gridDim.x, c1 = nchunks * (blockIdx.x + 1) / gridDim.x;
    int64_t staged_e = -1, staged_t = -1;
    // Column tiles outermost: x is staged once per tile (and matrix, where x
    // is per matrix) for all of the block's chunks, and each row's y adds the
    // tiles' partial sums in tile order (the block owns its rows).
    for (int64_t t = 0; t < nT; ++t) {
        const int64_t qb = t * (TI >> 5);
        const int nqt = static_cast<int>(min(TI >> 5, nq - qb));
        for (int64_t c = c0; c < c1; ++c) {
            const int64_t e = c / cpm;
            const int64_t ob = (c - e * cpm) * rows_per_chunk + rgi * R;
            const float g = FMT == TQ_NVFP4_G16 ? __ldg(gs + e) : 0.f;
            const int64_t ofirst = min(ob, O - 1);
            int rr[R];   // rows relative to the first; rows past O repeat the last one and are not stored
#pragma unroll
            for (int r = 0; r < R; ++r) rr[r] = static_cast<int>(min(ob + r, O - 1) - ofirst);
            float acc[R][B];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int b = 0; b < B; ++b) acc[r][b] = 0.f;
            int qt = slice * 32 + lane;   // quad within the tile
            bool have = qt < nqt;
            GvRows<FMT, A16, R> rw;
            rw.init(packed, scales, zeros, static_cast<int>(G), e * O + ofirst, rr, static_cast<int>(qb) + qt);
            Quad cur[R];
            if (have) {                   // the first loads are in flight while x is staged
#pragma unroll
                for (int r = 0; r < R; ++r) cur[r] = rw.load(r, g);
            }
            if (staged_t != t || (staged_e != e && x_ms != 0)) {   // block-uniform
                __syncthreads();
                gv_stage<FMT == TQ_INT3_G64_SYM>(xs, x, x_bf16 != 0, e * x_ms, I, t * TI, TI, B, vec);
                __syncthreads();
                staged_t = t;
                staged_e = e;
            }
            while (have) {
                const int qn = qt + qstep;
                const bool hn = qn < nqt;
                if constexpr (GV_DB) {    // the next quads' loads are issued before these are used
                    Quad nxt[R];
                    if (hn) {
                        rw.next(qstep);
#pragma unroll
                        for (int r = 0; r < R; ++r) nxt[r] = rw.load(r, g);
                    }
                    gv_quad<FMT, B, R>(cur, xs + (qt >> 5) * 256 + lane, slots, acc);
#pragma unroll
                    for (int r = 0; r < R; ++r) cur[r] = nxt[r];
                } else {
                    gv_quad<FMT, B, R>(cur, xs + (qt >> 5) * 256 + lane, slots, acc);
                    if (hn) {
                        rw.next(qstep);
#pragma unroll
                        for (int r = 0; r < R; ++r) cur[r] = rw.load(r, g);
                    }
                }
                qt = qn;
                have = hn;
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    float s = acc[r][b];
#pragma unroll
                    for (int off = 16; off; off >>= 1) s = __fadd_rn(s, __shfl_xor_sync(FULL, s, off));
                    if (wl == 0) {
                        if (lane == 0 && ob + r < O) {
                            float* yp = y + (e * B + b) * O + ob + r;
                            *yp = t == 0 ? s : __fadd_rn(*yp, s);
                        }
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
                    if (ob + r < O) {
                        float* yp = y + (e * B + b) * O + ob + r;
                        *yp = t == 0 ? s : __fadd_rn(*yp, s);
                    }
                }
                __syncthreads();
            }
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
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(gv_xs_bytes<B>()));
    });
    const int64_t i = TI / 1024;
    int n = i < 25 ? cache[i].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, gv_threads<B>(), smem) != cudaSuccess || n < 1)
            n = 1;
        if (i < 25) cache[i].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int FMT, int B, bool A16>
void launch_gemv(const uint8_t* packed, const void* scales, const uint8_t* zeros, const float* gs, int64_t n_mat,
                 int64_t O, int64_t I, const void* x, bool x_bf16, int64_t x_ms, float* y, cudaStream_t st) {
    constexpr int R = gv_rows<B>();
    constexpr int GV_WARPS = gv_warps<B>();
    const int64_t TI = gv_tile<B>(I);
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
    k_dequant_gemv<FMT, B, A16><<<static_cast<unsigned>(grid), gv_threads<B>(), smem, st>>>(
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
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "tq_dequant_gemv: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_dequant_gemv: NVFP4 needs global_scale");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t xms = n_mat > 1 ? x_mat_stride : 0;
    const bool xb = x_dtype == TQ_BF16;
    if (gemv_mma_ok(fmt, I, B, xms, xb)) {   // several bf16 vectors: the tensor-core form (gemv_mma.cu)
        launch_gemv_mma(fmt, packed, scales, zeros, global_scale, n_mat, O, I, x, B, xms, y, st);
        return check_launch("tq_dequant_gemv");
    }
    if (fmt == TQ_INT3_G64_SYM) {
        launch_gemv_b<TQ_INT3_G64_SYM, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else if (fmt == TQ_INT4_G128_ASYM) {
        launch_gemv_b<TQ_INT4_G128_ASYM, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else if (fmt == TQ_INT4_G64_ASYM) {
        launch_gemv_b<TQ_INT4_G64_ASYM, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else if (fmt == TQ_INT4_G32_ASYM) {
        launch_gemv_b<TQ_INT4_G32_ASYM, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else if (((I + 15) / 16) % 2 == 0 && (reinterpret_cast<uintptr_t>(scales) & 1u) == 0) {
        launch_gemv_b<TQ_NVFP4_G16, true>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    } else {
        launch_gemv_b<TQ_NVFP4_G16, false>(B, packed, scales, zeros, global_scale, n_mat, O, I, x, xb, xms, y, st);
    }
    return check_launch("tq_dequant_gemv");
}
