// Building blocks of the stand-alone streaming kernels (RTN + pack with given
// scales, dequantization, proxy error).  All three walk a matrix batch in
// octets: 8 consecutive weights of one group (an int3-g64 group holds 8
// octets, an int4-g128 group 16, an NVFP4-g16 block 2).  One thread per octet
// column: a bf16 octet is one 16-byte load (and a bf16 dequantized octet one
// 16-byte store), so the 32 lanes of a warp touch 512 contiguous bytes of a
// row per instruction, every 32-byte sector whole.
//
// A thread keeps its octet column (and what depends only on the column: its
// imatrix weights, its place in the record) and walks rows two at a time,
// both rows' loads issued before either is used.  No integer division is
// needed in the walk.
#pragma once
#include "group_pack.cuh"

namespace tq {

// lg = log2(octets per group), rec = record bytes per group.
template <int FMT> struct FmtTraits;
template <> struct FmtTraits<TQ_INT3_G64_SYM> { static constexpr int lg = 3, group = 64, rec = 24; };
template <> struct FmtTraits<TQ_INT4_G128_ASYM> { static constexpr int lg = 4, group = 128, rec = 64; };
template <> struct FmtTraits<TQ_INT4_G64_ASYM> { static constexpr int lg = 3, group = 64, rec = 32; };
template <> struct FmtTraits<TQ_INT4_G32_ASYM> { static constexpr int lg = 2, group = 32, rec = 16; };
template <> struct FmtTraits<TQ_NVFP4_G16> { static constexpr int lg = 1, group = 16, rec = 8; };

// ------------------------------------------------------------------ host geometry

struct Walk {
    int64_t width;     // threads per block = octet columns per block (a multiple of 32, <= 256)
    int64_t cblocks;   // column tiles per row
    int64_t slices;    // row slices per matrix
    int64_t rps;       // rows per slice
};

// `cols` octet columns per row, `rows` rows per matrix, about `target_blocks`
// blocks in all (at least that many when round_up, at most that many
// otherwise unless every matrix already needs more).  Column tiles are
// balanced so a ragged row idles fewer than 32 threads per tile.
inline Walk walk_geometry(int64_t n_mat, int64_t rows, int64_t cols, int64_t target_blocks, bool round_up = true) {
    Walk w;
    w.cblocks = (cols + 255) / 256;
    const int64_t per = (cols + w.cblocks - 1) / w.cblocks;
    w.width = (per + 31) / 32 * 32;
    int64_t s = round_up ? (target_blocks + w.cblocks * n_mat - 1) / (w.cblocks * n_mat)
                         : target_blocks / (w.cblocks * n_mat);
    s = s < 1 ? 1 : (s > rows ? rows : s);
    w.rps = (rows + s - 1) / s;
    w.slices = (rows + w.rps - 1) / w.rps;
    return w;
}

// ------------------------------------------------------------------ device: rows

// Position of one thread's octet in row r of a matrix batch whose rows run
// over all matrices in order: matrix e, row o, and the octet's address.
template <typename T>
struct RowCursor {
    const T* base;
    int64_t O, ld, ms, j, e, o;
    const T* ptr;
    __device__ __forceinline__ RowCursor(const T* W, int64_t O_, int64_t ld_, int64_t ms_, int64_t j_, int64_t r)
        : base(W), O(O_), ld(ld_), ms(ms_), j(j_) {
        e = r / O;
        o = r - e * O;
        ptr = base + e * ms + o * ld + j;
    }
    __device__ __forceinline__ void next() {
        if (++o == O) {
            o = 0;
            ++e;
            ptr = base + e * ms + j;
        } else {
            ptr += ld;
        }
    }
    // n rows on (a division only where the step crosses into another matrix)
    __device__ __forceinline__ void advance(int64_t n) {
        o += n;
        if (o >= O) {
            e += o / O;
            o %= O;
            ptr = base + e * ms + o * ld + j;
        } else {
            ptr += n * ld;
        }
    }
};

// ------------------------------------------------------------------ device: weights

// The 8 weights of an octet as loaded (n of them valid, the rest 0): one
// 16-byte load for bf16, two for fp32, when all 8 are valid (row strides are
// multiples of 16 bytes and octets start at multiples of 8 elements).
template <typename T> struct Oct;
template <> struct Oct<uint16_t> {
    uint4 v;
    __device__ __forceinline__ void load(const uint16_t* p, int n) {
        if (n == 8) {
            v = __ldg(reinterpret_cast<const uint4*>(p));
        } else {
            uint32_t u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const unsigned lo = 2 * i < n ? __ldg(p + 2 * i) : 0u;
                const unsigned hi = 2 * i + 1 < n ? __ldg(p + 2 * i + 1) : 0u;
                u[i] = lo | (hi << 16);
            }
            v = make_uint4(u[0], u[1], u[2], u[3]);
        }
    }
    __device__ __forceinline__ void get(float w[8]) const {
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            w[2 * i] = __uint_as_float(u[i] << 16);
            w[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        }
    }
};
template <> struct Oct<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p, int n) {
        if (n == 8) {
            a = __ldg(reinterpret_cast<const float4*>(p));
            b = __ldg(reinterpret_cast<const float4*>(p) + 1);
        } else {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = i < n ? __ldg(p + i) : 0.f;
            a = make_float4(f[0], f[1], f[2], f[3]);
            b = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
    __device__ __forceinline__ void get(float w[8]) const {
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
};

// ------------------------------------------------------------------ device: codes of one octet

// Where one thread's octet sits in the per-group outputs of a row: its
// group's record, scale and zero-point.  Advancing to the next row adds the
// row strides (G records / scales / zero-points), no index arithmetic.
template <int FMT>
struct QPtr {
    const uint8_t* rec;
    const void* sc;
    const uint8_t* zp;
    int64_t G;
    __device__ __forceinline__ QPtr(const uint8_t* packed, const void* scales, const uint8_t* zeros, int64_t gid,
                                    int64_t G_)
        : G(G_) {
        rec = packed + gid * FmtTraits<FMT>::rec;
        sc = FMT == TQ_NVFP4_G16 ? static_cast<const void*>(static_cast<const uint8_t*>(scales) + gid)
                                 : static_cast<const void*>(static_cast<const float*>(scales) + gid);
        zp = zeros ? zeros + gid : nullptr;
    }
    __device__ __forceinline__ void skip(int64_t rows) {   // `rows` rows on
        rec += rows * G * FmtTraits<FMT>::rec;
        sc = FMT == TQ_NVFP4_G16 ? static_cast<const void*>(static_cast<const uint8_t*>(sc) + rows * G)
                                 : static_cast<const void*>(static_cast<const float*>(sc) + rows * G);
        if (is_int4(FMT)) zp += rows * G;
    }
    __device__ __forceinline__ void next() {
        rec += G * FmtTraits<FMT>::rec;
        sc = FMT == TQ_NVFP4_G16 ? static_cast<const void*>(static_cast<const uint8_t*>(sc) + G)
                                 : static_cast<const void*>(static_cast<const float*>(sc) + G);
        if (is_int4(FMT)) zp += G;
    }
};

// The packed bits, scale and zero-point of octet `oct` of the group at q.
// bits: int3 = its 8 codes u as nibbles (built from its 2 low-plane bytes and
// its high-plane byte); int4 = its 4 record bytes (8 nibbles); NVFP4 = its
// half of the 8-byte record.  For NVFP4, s is the decoded E4M3 block scale
// (the caller multiplies by the global scale).
struct OctQ {
    uint32_t bits;
    float s;
    int z;
};

// 8 int3 codes from their planes: lo = 8 x 2 bits (element k at bits 2k,
// 2k+1), hi = 8 x 1 bit (element k at bit k) -> 8 nibbles, by shift-and-mask
// spreading of both planes.
__device__ __forceinline__ uint32_t int3_nibbles(uint32_t lo, uint32_t hi) {
    uint32_t x = lo;
    x = (x | (x << 8)) & 0x00ff00ffu;
    x = (x | (x << 4)) & 0x0f0f0f0fu;
    x = (x | (x << 2)) & 0x33333333u;
    uint32_t y = hi;
    y = (y | (y << 12)) & 0x000f000fu;
    y = (y | (y << 6)) & 0x03030303u;
    y = (y | (y << 3)) & 0x11111111u;
    return x | (y << 2);
}

template <int FMT>
__device__ __forceinline__ OctQ load_q(const QPtr<FMT>& q, int oct) {
    OctQ o;
    if constexpr (FMT == TQ_INT3_G64_SYM) {
        o.bits = int3_nibbles(__ldg(reinterpret_cast<const uint16_t*>(q.rec) + oct), __ldg(q.rec + 16 + oct));
        o.s = __ldg(static_cast<const float*>(q.sc));
        o.z = 4;
    } else if constexpr (is_int4(FMT)) {
        o.bits = __ldg(reinterpret_cast<const uint32_t*>(q.rec) + oct);
        o.s = __ldg(static_cast<const float*>(q.sc));
        o.z = __ldg(q.zp);
    } else {
        o.bits = __ldg(reinterpret_cast<const uint32_t*>(q.rec) + (oct & 1));
        o.s = e4m3_value(__ldg(static_cast<const uint8_t*>(q.sc)));
        o.z = 0;
    }
    return o;
}

// The codes and scale of NO consecutive octets starting at octet `oct` (a
// multiple of NO, so all of them lie in the group at q): bits[i] for octet
// oct + i, in the form load_q gives.
template <int NO>
struct UnitQ {
    uint32_t bits[NO];
    float s;
    int z;
};

template <int FMT, int NO>
__device__ __forceinline__ UnitQ<NO> load_unit_q(const QPtr<FMT>& q, int oct) {
    static_assert(NO == 1 || NO == 2, "units of one or two octets");
    UnitQ<NO> u;
    if constexpr (NO == 1) {
        const OctQ o = load_q<FMT>(q, oct);
        u.bits[0] = o.bits; u.s = o.s; u.z = o.z;
    } else if constexpr (FMT == TQ_INT3_G64_SYM) {
        const uint32_t lo = __ldg(reinterpret_cast<const uint32_t*>(q.rec + 2 * oct));
        const uint32_t hi = __ldg(reinterpret_cast<const uint16_t*>(q.rec + 16 + oct));
        u.bits[0] = int3_nibbles(lo & 0xffffu, hi & 0xffu);
        u.bits[1] = int3_nibbles(lo >> 16, hi >> 8);
        u.s = __ldg(static_cast<const float*>(q.sc));
        u.z = 4;
    } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(q.rec + (FMT == TQ_NVFP4_G16 ? 0 : 4 * oct)));
        u.bits[0] = v.x; u.bits[1] = v.y;
        if constexpr (is_int4(FMT)) {
            u.s = __ldg(static_cast<const float*>(q.sc));
            u.z = __ldg(q.zp);
        } else {
            u.s = e4m3_value(__ldg(static_cast<const uint8_t*>(q.sc)));
            u.z = 0;
        }
    }
    return u;
}

// 2^23 + k for a small non-negative integer k, as a float; subtracting 2^23
// (exactly) gives k without an integer-to-float conversion.
__device__ __forceinline__ float f23(unsigned k) { return __uint_as_float(0x4b000000u | k); }

// Dequantized values of an octet, rounded once to fp32 exactly as the pages'
// formulas: int3 s v, int4 s (q - z), NVFP4 fl32(fl32(g dec(e)) dec(c)).
// Integers become floats as 2^23 + k (exact) and the offset 2^23 + z comes
// off in the same fp32 addition, pairs of elements per fp32x2 instruction;
// NVFP4 bytes are decoded by the hardware E2M1 conversion (exact).
template <int FMT>
__device__ __forceinline__ void dec_oct(const OctQ& q, float g, float v[8]) {
    if constexpr (FMT == TQ_NVFP4_G16) {
        const float S = __fmul_rn(g, q.s);
        const float2 S2 = make_float2(S, S);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const float2 r = __fmul2_rn(S2, e2m1x2_to_f32((q.bits >> (8 * b)) & 0xffu));
            v[2 * b] = r.x; v[2 * b + 1] = r.y;
        }
    } else {   // int3 (u = v + 4, z = 4) and int4: s (q - z) from 8 nibbles
        const float o = f23(static_cast<unsigned>(q.z) & 0xffu);   // 2^23 + z
        const float2 noff = make_float2(-o, -o), s2 = make_float2(q.s, q.s);
        const uint32_t ev = q.bits & 0x0f0f0f0fu, od = (q.bits >> 4) & 0x0f0f0f0fu;   // elements 2k, 2k+1 in byte k
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const unsigned sel = 0x5640u | static_cast<unsigned>(k);    // bytes: (byte k, 0, 0, 0x4b)
            const float2 x = make_float2(__uint_as_float(__byte_perm(ev, 0x4b00u, sel)),
                                         __uint_as_float(__byte_perm(od, 0x4b00u, sel)));
            const float2 r = __fmul2_rn(s2, __fadd2_rn(x, noff));
            v[2 * k] = r.x; v[2 * k + 1] = r.y;
        }
    }
}

// ------------------------------------------------------------------ device: RTN codes of one octet

// Integer codes q_i = clamp(rint(w_i / s) + z, 0, HI) of an octet, as 8
// nibbles (element i in bits 4i..4i+3), where rint rounds the IEEE fp32
// quotient half to even (int3: z = 4, HI = 7 gives the stored
// u = clamp(rint(w/s), -4, 3) + 4; int4: HI = 15).  Elements at or past n and
// a zero scale give z.
//
// Fast path (s normal and not extreme): with inv = rcp(s) (within 2^-21
// relative of 1/s), the exact products w inv (1 -+ 2^-20) bracket the IEEE
// quotient; one FMA per end adds 1.5 2^23, which rounds the product to an
// integer, half to even, in the low mantissa bits.  Rounding is monotone, so
// when both ends give the same integer it is the quotient's.  Both ends are
// finite or both are the same infinity (a quotient beyond +-2^127 clamps
// either way); where they differ (a quotient within about 2^-20 of a
// half-integer, or of magnitude 2^22 or more) that element (int4) or the
// whole octet (int3, measured faster there) is redone with IEEE divisions.
// For NaN weights the codes are unspecified.
template <int HI>
__device__ __forceinline__ uint32_t rtn_int_oct(const float w[8], int n, float s, int z) {
    const unsigned se = (__float_as_uint(s) >> 23) & 255u;
    bool exact = se < 3u || se > 251u;   // zero, subnormal or extreme scales
    uint32_t nib = 0u;
    if (!exact) {
        const float inv = rcp_approx(s);
        const float lo = __fmul_rn(inv, 0.99999904632568359375f), hi = __fmul_rn(inv, 1.00000095367431640625f);
        const float2 ilo = make_float2(lo, lo), ihi = make_float2(hi, hi), M2 = make_float2(MAGIC, MAGIC);
        const int zo = z - static_cast<int>(0x4b400000u);   // code = bits(t) - bits(1.5 2^23) + z
        uint32_t diff = 0u, bytes[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 ww = make_float2(w[2 * p], w[2 * p + 1]);
            const float2 tl = __ffma2_rn(ww, ilo, M2), th = __ffma2_rn(ww, ihi, M2);
            diff |= (__float_as_uint(tl.x) ^ __float_as_uint(th.x)) | (__float_as_uint(tl.y) ^ __float_as_uint(th.y));
            const int c0 = __vimin_s32_relu(static_cast<int>(__float_as_uint(tl.x)) + zo, HI);
            const int c1 = __vimin_s32_relu(static_cast<int>(__float_as_uint(tl.y)) + zo, HI);
            bytes[p] = static_cast<uint32_t>(c0 + 16 * c1);
        }
        nib = __byte_perm(__byte_perm(bytes[0], bytes[1], 0x0040u), __byte_perm(bytes[2], bytes[3], 0x0040u), 0x5410u);
        if (HI == 7) {
            exact = diff != 0u;   // int3: the whole octet with IEEE divisions (measured faster for int3)
        } else if (diff) {   // int4: elements whose bracket ends disagree take an IEEE division, one at a time
            const float zf = static_cast<float>(z);
            uint32_t todo = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                todo |= (__float_as_uint(__fmaf_rn(w[i], lo, MAGIC)) != __float_as_uint(__fmaf_rn(w[i], hi, MAGIC)) ? 1u : 0u) << i;
            while (todo) {
                const int i = __ffs(todo) - 1;
                todo &= todo - 1u;
                float wi = w[0];
#pragma unroll
                for (int k = 1; k < 8; ++k) wi = i == k ? w[k] : wi;
                const float qf = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(wi, s)), zf), 0.f), static_cast<float>(HI));
                nib = (nib & ~(15u << (4 * i))) | ((static_cast<uint32_t>(qf) & 15u) << (4 * i));
            }
        }
    }
    if (exact) {   // zero, subnormal or extreme scale (or an int3 disagreement): IEEE divisions throughout
        nib = 0u;
        const float zf = static_cast<float>(z);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float qf = zf;
            if (s != 0.f) qf = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w[i], s)), zf), 0.f), static_cast<float>(HI));
            nib |= (static_cast<uint32_t>(qf) & 15u) << (4 * i);
        }
    }
    if (n < 8) {   // padding: code z
        const uint32_t keep = n <= 0 ? 0u : (0xffffffffu >> (32 - 4 * n));
        nib = (nib & keep) | ((static_cast<uint32_t>(z) & 15u) * 0x11111111u & ~keep);
    }
    return nib;
}

// Stores an octet's integer codes (8 nibbles) into its share of the record
// at rec: int3 = 2 low-plane bytes (bits 0-1 of each code) + 1 high-plane
// byte (bit 2), gathered with shift-and-mask compression; int4 = the 4 bytes
// as they are.
template <int FMT>
__device__ __forceinline__ void store_oct(uint8_t* rec, int oct, uint32_t nib) {
    if constexpr (FMT == TQ_INT3_G64_SYM) {
        uint32_t x = nib & 0x33333333u;
        x = (x | (x >> 2)) & 0x0f0f0f0fu;
        x = (x | (x >> 4)) & 0x00ff00ffu;
        x = (x | (x >> 8)) & 0x0000ffffu;
        uint32_t y = (nib >> 2) & 0x11111111u;
        y = (y | (y >> 3)) & 0x03030303u;
        y = (y | (y >> 6)) & 0x000f000fu;
        y = (y | (y >> 12)) & 0x000000ffu;
        reinterpret_cast<uint16_t*>(rec)[oct] = static_cast<uint16_t>(x);
        rec[16 + oct] = static_cast<uint8_t>(y);
    } else {
        reinterpret_cast<uint32_t*>(rec)[oct] = nib;
    }
}

// Stores NO octets' integer codes (nibble words) into the record at rec,
// starting at octet `oct` (a multiple of NO).
template <int FMT, int NO>
__device__ __forceinline__ void store_unit(uint8_t* rec, int oct, const uint32_t nib[NO]) {
    if constexpr (NO == 1) {
        store_oct<FMT>(rec, oct, nib[0]);
    } else if constexpr (FMT == TQ_INT3_G64_SYM) {
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t x = nib[i] & 0x33333333u;
            x = (x | (x >> 2)) & 0x0f0f0f0fu;
            x = (x | (x >> 4)) & 0x00ff00ffu;
            x = (x | (x >> 8)) & 0x0000ffffu;
            uint32_t y = (nib[i] >> 2) & 0x11111111u;
            y = (y | (y >> 3)) & 0x03030303u;
            y = (y | (y >> 6)) & 0x000f000fu;
            y = (y | (y >> 12)) & 0x000000ffu;
            lo |= x << (16 * i);
            hi |= y << (8 * i);
        }
        *reinterpret_cast<uint32_t*>(rec + 2 * oct) = lo;
        *reinterpret_cast<uint16_t*>(rec + 16 + oct) = static_cast<uint16_t>(hi);
    } else {
        *reinterpret_cast<uint2*>(rec + 4 * oct) = make_uint2(nib[0], nib[1]);
    }
}

}  // namespace tq
