// Dequant-GEMV on the tensor cores for bf16 token vectors (2 <= B <= 8):
// y[e][b][o] = sum over groups of s * sum_{j in group} d_j x[e][b][j], the
// same product as the CUDA-core kernel of gemv.cu, with the per-group sums
// sum d_j x_j taken by bf16 m16n8k16 MMAs.  The decoded values d (int3 v,
// int4 q - z, NVFP4 dec(c)) are small integers or E2M1 values, exact in
// bf16, and bf16 x is exact too, so every product is exact; each group gets
// an accumulator of its own, scaled once by its fp32 factor in the epilogue,
// so no group scale is ever rounded into a bf16 operand.
//
// B200 mapping.  A block is 4 warps on the same 16 RT rows of one matrix;
// warp w takes groups w, w + 4, ... of every row, and the warps' partial sums
// are added in warp order at the end.  Per warp and group, each m16 tile of
// rows is one A operand per k16 step, decoded in registers from the records
// (no shared-memory round trip), and x (8 vectors, zero past B) is the B
// operand, loaded once per group and shared by the RT tiles.  The k index of
// the MMA is a permutation of the group's columns chosen so that lane
// (gid, tig) of the fragment layouts reads 4 consecutive codes and 4
// consecutive x values per step: in a run of C = min(g, 64) columns (S = C/16
// steps), lane tig owns columns [4 S tig, 4 S tig + 4 S), step s its columns
// 4 S tig + 4 s .. + 3, which the MMA sees as k = 2 tig, 2 tig + 1, 2 tig + 8,
// 2 tig + 9.  A and B use the same permutation, so the sum is unchanged.
//
// Decoding: an int4 code n becomes the bf16 bits 0x4300 | n = 128 + n by
// one byte permute per pair, and a bf16x2 subtraction of 128 + z leaves q - z
// exactly.  An int3 code u = v + 4 (its planes spread into nibbles first) and
// an E2M1 magnitude select the high and the low byte of their bf16 value from
// two 8-byte tables by byte permutes (the code is the permute's selector);
// the E2M1 sign bit is moved into place.
//
// Rounding: products are exact; a k16 MMA step accumulates its 16 products
// into the group's fp32 accumulator (the bound below takes 2^-22 of the
// magnitudes per step); the epilogue's fma(s, D, y) rounds once per group,
// in group order per warp; the 4 warps' sums are added in order.
//   |y - sum What x| <= (4 g/16 + ceil(G/4) + 4) 2^-24 sum |What x|
// (G = groups per row), plus underflow.
#include "walk.cuh"

namespace tq {

constexpr int GM_WARPS = 4;

__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// 4 integer codes n0..n3 (nibbles of c, code i at bits 4i) minus the offset
// zz = bf16x2(128 + z, 128 + z): bf16x2 (n0 - z, n1 - z) and (n2 - z, n3 - z).
__device__ __forceinline__ void int_codes4_bf16(uint32_t c, uint32_t zz, uint32_t& p0, uint32_t& p1) {
    const uint32_t sp = (c & 0x0f0fu) | ((c << 12) & 0x0f0f0000u);   // bytes n0, n2, n1, n3
    p0 = bf16x2_sub(__byte_perm(sp, 0x43434343u, 0x4240), zz);         // 0x4300 | n0, 0x4300 | n1
    p1 = bf16x2_sub(__byte_perm(sp, 0x43434343u, 0x4341), zz);
}

// 4 E2M1 codes (code i at bits 4i of c) as bf16x2 (c0, c1) and (c2, c3),
// exactly: magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} from two byte tables, the
// sign bit (code bit 3) to bit 15 of its half.
__device__ __forceinline__ void e2m1_codes4_bf16(uint32_t c, uint32_t& p0, uint32_t& p1) {
    const uint32_t sel = c & 0x7777u;
    const uint32_t hi = __byte_perm(0x3f3f3f00u, 0x40404040u, sel);
    const uint32_t lo = __byte_perm(0xc0800000u, 0xc0804000u, sel);
    p0 = __byte_perm(lo, hi, 0x5140) | ((c << 12) & 0x8000u) | ((c << 24) & 0x80000000u);
    p1 = __byte_perm(lo, hi, 0x7362) | ((c << 4) & 0x8000u) | ((c << 16) & 0x80000000u);
}

// 4 int3 codes u = v + 4 (nibbles of c, code i at bits 4i, each < 8) as
// bf16x2 (v0, v1) and (v2, v3), exactly: the code itself selects the high
// and the low byte of bf16(u - 4) from two 8-byte tables.
__device__ __forceinline__ void int3_codes4_bf16(uint32_t c, uint32_t& p0, uint32_t& p1) {
    // bf16 of -4 .. 3: c080 c040 c000 bf80 0000 3f80 4000 4040
    const uint32_t hi = __byte_perm(0xbfc0c0c0u, 0x40403f00u, c);
    const uint32_t lo = __byte_perm(0x80004080u, 0x40008000u, c);
    p0 = __byte_perm(lo, hi, 0x5140);
    p1 = __byte_perm(lo, hi, 0x7362);
}

template <int FMT> struct GmFmt;
template <> struct GmFmt<TQ_INT3_G64_SYM> { static constexpr int g = 64, rec = 24; };
template <> struct GmFmt<TQ_INT4_G128_ASYM> { static constexpr int g = 128, rec = 64; };
template <> struct GmFmt<TQ_INT4_G64_ASYM> { static constexpr int g = 64, rec = 32; };
template <> struct GmFmt<TQ_INT4_G32_ASYM> { static constexpr int g = 32, rec = 16; };
template <> struct GmFmt<TQ_NVFP4_G16> { static constexpr int g = 16, rec = 8; };

// The record bytes lane tig needs from one row for run h of its group (C =
// min(g, 64) columns, lane part = 4 S codes: int3 the low-plane word and the
// high-plane half-word, int4 and NVFP4 the nibbles) as nibble words (code i
// of the lane part at bits 4 (i % 8) of word i / 8): int3 planes spread into
// u = v + 4.
template <int FMT>
__device__ __forceinline__ void gm_nibbles(const uint32_t (&raw)[2], uint32_t (&w)[2]) {
    if constexpr (FMT == TQ_INT3_G64_SYM) {
        w[0] = int3_nibbles(raw[0] & 0xffffu, raw[1] & 0xffu);
        w[1] = int3_nibbles(raw[0] >> 16, raw[1] >> 8);
    } else {
        w[0] = raw[0];
        w[1] = raw[1];
    }
}

struct GmArgs {
    const uint8_t* packed;
    const void* scales;
    const uint8_t* zeros;
    const float* gs;
    int64_t n_mat, O, I, x_ms, B;
    const uint16_t* x;
    float* y;
    int64_t row_blocks;   // blocks per matrix
};

// The record bytes lane tig needs from one row for run h of its group (C =
// min(g, 64) columns, lane part = 4 S codes), loaded raw: int3 the low-plane
// word and the high-plane half-word, int4 and NVFP4 the nibbles.
template <int FMT>
__device__ __forceinline__ void gm_load(const uint8_t* rec, int h, int tig, uint32_t (&w)[2]) {
    if constexpr (FMT == TQ_INT3_G64_SYM) {   // 16 codes: low plane bits 32 tig.., high plane bits 16 tig..
        w[0] = __ldg(reinterpret_cast<const uint32_t*>(rec) + tig);
        w[1] = __ldg(reinterpret_cast<const uint16_t*>(rec + 16) + tig);
    } else if constexpr (FMT == TQ_INT4_G128_ASYM || FMT == TQ_INT4_G64_ASYM) {   // 16 codes, 8 bytes
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(rec + 32 * h) + tig);
        w[0] = v.x;
        w[1] = v.y;
    } else if constexpr (FMT == TQ_INT4_G32_ASYM) {   // 8 codes, 4 bytes
        w[0] = __ldg(reinterpret_cast<const uint32_t*>(rec) + tig);
        w[1] = 0u;
    } else {   // NVFP4: 4 codes, 2 bytes
        w[0] = __ldg(reinterpret_cast<const uint16_t*>(rec) + tig);
        w[1] = 0u;
    }
}

template <int FMT, int RT>
__global__ void __launch_bounds__(GM_WARPS * 32)
k_gemv_mma(const __grid_constant__ GmArgs a) {
    using F = GmFmt<FMT>;
    constexpr int g = F::g, C = g < 64 ? g : 64, S = C / 16, H = g / C;
    __shared__ float red[GM_WARPS][RT][4][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int64_t e = blockIdx.x / a.row_blocks;
    const int64_t o0 = (blockIdx.x - e * a.row_blocks) * (16 * RT);
    const int64_t I = a.I, O = a.O;
    const int64_t G = (I + g - 1) / g;
    const uint16_t* xr = a.x + e * a.x_ms + static_cast<int64_t>(gid) * I;   // this lane's x vector (b = gid)
    const bool xb = gid < a.B;
    const float ge = FMT == TQ_NVFP4_G16 ? __ldg(a.gs + e) : 0.f;
    // this lane's rows: o0 + 16 t + gid (A rows 0-7 of tile t) and + 8 (rows 8-15)
    int64_t row[RT][2];
    bool ok[RT][2];
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            row[t][h] = e * O + o0 + 16 * t + gid + 8 * h;
            ok[t][h] = o0 + 16 * t + gid + 8 * h < O;
        }
    float y[RT][4];
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) y[t][i] = 0.f;

    // Group k's loads (codes, zero-points, factors and x of every run) are
    // issued while group k - 4 is computed, raw: nothing waits for them
    // before their group's turn.
    uint32_t cw[H][RT][2][2], zr[RT][2], sr[RT][2], xw[H][2 * S];
    auto load = [&](int64_t k) {
#pragma unroll
        for (int h = 0; h < H; ++h) {
            // x: this lane's 4 S columns of run h (whole 16-byte chunks: I is a multiple of 8)
            const int64_t c0 = k * g + h * C + 4 * S * tig;
#pragma unroll
            for (int q = 0; q < (S + 1) / 2; ++q) {
                const int64_t cq = c0 + 8 * q;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if constexpr (S == 1) {
                    if (xb && cq < I) {
                        const uint2 u = __ldg(reinterpret_cast<const uint2*>(xr + cq));
                        v.x = u.x;
                        v.y = u.y;
                    }
                } else {
                    if (xb && cq < I) v = __ldg(reinterpret_cast<const uint4*>(xr + cq));
                }
                xw[h][4 * q] = v.x;
                xw[h][4 * q + 1] = v.y;
                if (2 * S > 4 * q + 2) {
                    xw[h][4 * q + 2] = v.z;
                    xw[h][4 * q + 3] = v.w;
                }
            }
        }
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int h = 0; h < H; ++h) cw[h][t][r][0] = cw[h][t][r][1] = 0u;
                zr[t][r] = 0u;
                sr[t][r] = 0u;
                if (ok[t][r]) {
                    const int64_t gi = row[t][r] * G + k;
#pragma unroll
                    for (int h = 0; h < H; ++h) gm_load<FMT>(a.packed + gi * F::rec, h, tig, cw[h][t][r]);
                    if constexpr (is_int4(FMT)) zr[t][r] = __ldg(a.zeros + gi);
                    if constexpr (FMT == TQ_NVFP4_G16) sr[t][r] = __ldg(static_cast<const uint8_t*>(a.scales) + gi);
                    else sr[t][r] = __float_as_uint(__ldg(static_cast<const float*>(a.scales) + gi));
                }
            }
    };
    if (warp < G) load(warp);
#pragma unroll 1
    for (int64_t k = warp; k < G; k += GM_WARPS) {
        // this group's data, then the next group's loads
        uint32_t ccw[H][RT][2][2], czr[RT][2], csr[RT][2], cxw[H][2 * S];
#pragma unroll
        for (int h = 0; h < H; ++h) {
#pragma unroll
            for (int i = 0; i < 2 * S; ++i) cxw[h][i] = xw[h][i];
#pragma unroll
            for (int t = 0; t < RT; ++t)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    ccw[h][t][r][0] = cw[h][t][r][0];
                    ccw[h][t][r][1] = cw[h][t][r][1];
                }
        }
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                czr[t][r] = zr[t][r];
                csr[t][r] = sr[t][r];
            }
        if (k + GM_WARPS < G) load(k + GM_WARPS);
        float D[RT][4];
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
            for (int i = 0; i < 4; ++i) D[t][i] = 0.f;
#pragma unroll
        for (int h = 0; h < H; ++h) {
            uint32_t nib[RT][2][2];
#pragma unroll
            for (int t = 0; t < RT; ++t)
#pragma unroll
                for (int r = 0; r < 2; ++r) gm_nibbles<FMT>(ccw[h][t][r], nib[t][r]);
#pragma unroll
            for (int s = 0; s < S; ++s) {
                const uint32_t b0 = cxw[h][2 * s], b1 = cxw[h][2 * s + 1];
#pragma unroll
                for (int t = 0; t < RT; ++t) {
                    uint32_t A[4];
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const uint32_t c16 = (s & 1) ? nib[t][r][s >> 1] >> 16 : (nib[t][r][s >> 1] & 0xffffu);
                        uint32_t p0, p1;
                        if constexpr (FMT == TQ_NVFP4_G16) {
                            e2m1_codes4_bf16(c16, p0, p1);
                        } else if constexpr (FMT == TQ_INT3_G64_SYM) {
                            int3_codes4_bf16(c16, p0, p1);
                        } else {
                            const uint32_t z = czr[t][r];
                            int_codes4_bf16(c16, 0x43004300u | z | (z << 16), p0, p1);
                        }
                        A[r] = p0;       // a0 (rows 0-7) / a1 (rows 8-15): k = 2 tig, 2 tig + 1
                        A[2 + r] = p1;   // a2 / a3: k = 2 tig + 8, 2 tig + 9
                    }
                    mma_16816_bf16(D[t], A, b0, b1);
                }
            }
        }
        // the group's factor, once: rows gid (D 0, 1) and gid + 8 (D 2, 3)
#pragma unroll
        for (int t = 0; t < RT; ++t) {
            float sc[2];
#pragma unroll
            for (int r = 0; r < 2; ++r)
                sc[r] = FMT == TQ_NVFP4_G16 ? __fmul_rn(ge, e4m3_value(csr[t][r])) : __uint_as_float(csr[t][r]);
            y[t][0] = __fmaf_rn(sc[0], D[t][0], y[t][0]);
            y[t][1] = __fmaf_rn(sc[0], D[t][1], y[t][1]);
            y[t][2] = __fmaf_rn(sc[1], D[t][2], y[t][2]);
            y[t][3] = __fmaf_rn(sc[1], D[t][3], y[t][3]);
        }
    }
    // the warps' sums in warp order; lane (gid, tig) holds y[b = 2 tig + (i & 1)][o = gid + 8 (i >> 1)]
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][t][i][lane] = y[t][i];
    __syncthreads();
    for (int idx = threadIdx.x; idx < RT * 4 * 32; idx += blockDim.x) {
        const int t = idx / 128, i = (idx / 32) & 3, l = idx & 31;
        float v = red[0][t][i][l];
#pragma unroll
        for (int w = 1; w < GM_WARPS; ++w) v = __fadd_rn(v, red[w][t][i][l]);
        const int64_t b = 2 * (l & 3) + (i & 1);
        const int64_t o = o0 + 16 * t + (l >> 2) + 8 * (i >> 1);
        if (b < a.B && o < O) a.y[(e * a.B + b) * O + o] = v;
    }
}

// The tensor-core form applies to bf16 x whose rows are whole 16-byte chunks.
bool gemv_mma_ok(int32_t fmt, int64_t I, int64_t B, int64_t x_ms, bool x_bf16) {
    (void)fmt;
    return x_bf16 && B >= 2 && I % 8 == 0 && x_ms % 8 == 0;
}

template <int FMT, int RT>
void launch_gm(const GmArgs& a0, cudaStream_t st) {
    GmArgs a = a0;
    a.row_blocks = (a.O + 16 * RT - 1) / (16 * RT);
    k_gemv_mma<FMT, RT><<<static_cast<unsigned>(a.n_mat * a.row_blocks), GM_WARPS * 32, 0, st>>>(a);
}

// 32 rows per block where that still gives two blocks per SM, else 16.
template <int FMT>
void launch_gm_fmt(const GmArgs& a, cudaStream_t st) {
    const int64_t sms = num_sms();
    auto blocks = [&](int rt) { return a.n_mat * ((a.O + 16 * rt - 1) / (16 * rt)); };
    if (blocks(2) >= 2 * sms) launch_gm<FMT, 2>(a, st);
    else launch_gm<FMT, 1>(a, st);
}

void launch_gemv_mma(int32_t fmt, const uint8_t* packed, const void* scales, const uint8_t* zeros, const float* gs,
                     int64_t n_mat, int64_t O, int64_t I, const void* x, int64_t B, int64_t x_ms, float* y,
                     cudaStream_t st) {
    GmArgs a;
    a.packed = packed; a.scales = scales; a.zeros = zeros; a.gs = gs;
    a.n_mat = n_mat; a.O = O; a.I = I; a.x_ms = x_ms; a.B = B;
    a.x = static_cast<const uint16_t*>(x);
    a.y = y;
    a.row_blocks = 1;
    switch (fmt) {
        case TQ_INT3_G64_SYM: launch_gm_fmt<TQ_INT3_G64_SYM>(a, st); break;
        case TQ_INT4_G128_ASYM: launch_gm_fmt<TQ_INT4_G128_ASYM>(a, st); break;
        case TQ_INT4_G64_ASYM: launch_gm_fmt<TQ_INT4_G64_ASYM>(a, st); break;
        case TQ_INT4_G32_ASYM: launch_gm_fmt<TQ_INT4_G32_ASYM>(a, st); break;
        default: launch_gm_fmt<TQ_NVFP4_G16>(a, st); break;
    }
}

}  // namespace tq
