// Private helpers of the tq CUDA library (host validation + device building
// blocks).  Not part of the C ABI; see include/tq.h for the interface.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stdio.h>
#include <stdarg.h>
#include <string.h>

#include "../../include/tq.h"

#define TQ_API extern "C" __attribute__((visibility("default")))

namespace tq {

// ------------------------------------------------------------------ host: errors

tq_status set_error(tq_status st, const char* fmt, ...);
void clear_error();
tq_status check_launch(const char* what);

#define TQ_REQUIRE(cond, ...)                                          \
    do {                                                               \
        if (!(cond)) return ::tq::set_error(TQ_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// True (and the count cleared) if a tq_hessian launch since the last call
// gave up on a pipeline wait.
bool hessian_take_timeouts();
// The same for tq_proxy_error_full's GEMM pipeline.
bool proxy_full_take_timeouts();
// The same for tq_gemm_nvfp4.
bool nvfp4_gemm_take_timeouts();

inline int elem_bytes(int32_t dt) { return dt == TQ_BF16 ? 2 : (dt == TQ_F32 ? 4 : 0); }

__host__ __device__ inline int64_t group_of(int32_t fmt) {
    return fmt == TQ_INT3_G64_SYM ? 64 : fmt == TQ_INT4_G128_ASYM ? 128 : fmt == TQ_INT4_G64_ASYM ? 64
         : fmt == TQ_INT4_G32_ASYM ? 32 : fmt == TQ_NVFP4_G16 ? 16 : 0;
}
__host__ __device__ inline int64_t record_bytes(int32_t fmt) {
    return fmt == TQ_INT3_G64_SYM ? 24 : fmt == TQ_INT4_G128_ASYM ? 64 : fmt == TQ_INT4_G64_ASYM ? 32
         : fmt == TQ_INT4_G32_ASYM ? 16 : fmt == TQ_NVFP4_G16 ? 8 : 0;
}
// The asymmetric int4 formats (nibble codes with a zero-point), any group size.
__host__ __device__ constexpr bool is_int4(int fmt) {
    return fmt == TQ_INT4_G128_ASYM || fmt == TQ_INT4_G64_ASYM || fmt == TQ_INT4_G32_ASYM;
}

// The tensor-core form of tq_dequant_gemv (bf16 x, 2 <= B <= 8, I and the
// x matrix stride multiples of 8) and its launch.
bool gemv_mma_ok(int32_t fmt, int64_t I, int64_t B, int64_t x_ms, bool x_bf16);
void launch_gemv_mma(int32_t fmt, const uint8_t* packed, const void* scales, const uint8_t* zeros, const float* gs,
                     int64_t n_mat, int64_t O, int64_t I, const void* x, int64_t B, int64_t x_ms, float* y,
                     cudaStream_t st);

// Try-wait rounds of the tensor-core pipelines' ring waits for the next
// launch (tq_debug_set_wait_limit; default 2^22).
unsigned pipeline_wait_limit();
constexpr unsigned DEFAULT_WAIT_LIMIT = 1u << 22;

// Validates a matrix batch descriptor; returns TQ_OK or an error (set).
tq_status check_mat(const tq_mat* X, const char* name);

int num_sms();

// ------------------------------------------------------------------ index arithmetic

// Division of 32-bit unsigned integers by a fixed divisor d >= 1 with a
// multiply-high and a shift (the round-up method of Granlund and Montgomery,
// "Division by invariant integers using multiplication", 1994): with
// s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (umulhi(n, m) + n) >> s for every 32-bit n.
struct FastDiv {
    uint32_t d, m;
    int s;
    FastDiv() : d(1), m(1), s(0) {}
    explicit FastDiv(uint32_t dv) : d(dv ? dv : 1), s(0) {
        while ((uint64_t(1) << s) < d) ++s;
        m = static_cast<uint32_t>(((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1);
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        return static_cast<uint32_t>((static_cast<uint64_t>(__umulhi(n, m)) + n) >> s);
    }
};

// Group gid of [n_mat][O][G] -> (matrix, row, group) with 32-bit arithmetic.
struct GroupIndex {
    FastDiv og, g;
    uint32_t OG, G;
    GroupIndex() : OG(1), G(1) {}
    GroupIndex(int64_t O, int64_t Gn) : og(static_cast<uint32_t>(O * Gn)), g(static_cast<uint32_t>(Gn)),
                                         OG(static_cast<uint32_t>(O * Gn)), G(static_cast<uint32_t>(Gn)) {}
    __device__ __forceinline__ void split(uint32_t gid, uint32_t& e, uint32_t& o, uint32_t& k) const {
        e = og.div(gid);
        const uint32_t rem = gid - e * OG;
        o = g.div(rem);
        k = rem - o * G;
    }
};

// ------------------------------------------------------------------ device helpers

constexpr unsigned FULL = 0xffffffffu;
// Adding then subtracting 1.5 * 2^23 rounds an fp32 value of magnitude below
// 2^22 to an integer, half to even (the sum's ulp is 1 under round-to-nearest).
constexpr float MAGIC = 12582912.0f;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return __ldg(p); }
};
template <> struct Elem<uint16_t> {   // bf16 stored as raw bits
    static __device__ __forceinline__ float load(const uint16_t* p) { return bf16_bits_to_f32(__ldg(p)); }
};

// Warp-wide lexicographic (loss, index) minimum; every lane ends with it.
// NaN losses rank as +inf so every lane agrees on the result.
__device__ __forceinline__ void warp_argmin(float& L, int& idx) {
    if (L != L) L = __int_as_float(0x7f800000);
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        float Lo = __shfl_xor_sync(FULL, L, off);
        int io = __shfl_xor_sync(FULL, idx, off);
        if (Lo < L || (Lo == L && io < idx)) { L = Lo; idx = io; }
    }
}

// Butterfly sum: every lane of the group ends with the bit-identical total
// (each step adds the same pair of operands on both partner lanes).
__device__ __forceinline__ double group_sum_d(double v, unsigned mask, int width) {
    for (int off = width >> 1; off; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(mask, v, off));
    return v;
}

// 2^-e for the binade e of x > 0 (x * pow2_inv_binade(x) lies in [1, 2) for
// normal x; subnormal x are scaled by 2^126).  Multiplying by it is exact for
// normal results, so codes and candidate scales are unchanged and losses
// scale by exact powers of two: the fp32 ranking works on values of order one
// whatever the group's magnitude (it cannot underflow or overflow).
__device__ __forceinline__ float pow2_inv_binade(float x) {
    int E = static_cast<int>((__float_as_uint(x) >> 23) & 255u);
    E = min(max(E, 1), 253);
    return __uint_as_float(static_cast<unsigned>(254 - E) << 23);
}

__device__ __forceinline__ float warp_max_abs(float a, float b) {
    unsigned u = max(__float_as_uint(fabsf(a)), __float_as_uint(fabsf(b)));
    return __uint_as_float(__reduce_max_sync(FULL, u));
}

// Approximate reciprocal (hardware, within 1 ulp).  Used only where a value
// ranks candidates in fp32; every decision it could flip is re-taken in fp64.
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// 1 / (pw^2 pm) for powers of two pw, pm (exact in fp64, no division).
__device__ __forceinline__ double inv_pow2_sq(float pw, float pm) {
    const int ew = static_cast<int>((__float_as_uint(pw) >> 23) & 255u) - 127;
    const int em = static_cast<int>((__float_as_uint(pm) >> 23) & 255u) - 127;
    return __longlong_as_double(static_cast<long long>(1023 - 2 * ew - em) << 52);
}

// Integer code of w under scale s: round half to even of the IEEE fp32
// quotient w/s, clamped to [lo, hi]; scale 0 gives code 0.
__device__ __forceinline__ float rtn_exact(float w, float s, float lo, float hi) {
    if (s == 0.0f) return 0.0f;
    float y = rintf(__fdiv_rn(w, s));
    return fminf(fmaxf(y, lo), hi);
}

// Same code as rtn_exact(w, s, lo, hi) given inv = rcp_approx(s): the
// approximate quotient w * inv lies within 2^-21 |q| of the IEEE quotient q,
// so their rounded codes agree unless it is within 2^-20 |q| of a
// half-integer; only then is the IEEE quotient formed.
__device__ __forceinline__ float rtn_fast(float w, float s, float inv, float lo, float hi) {
    if (s == 0.0f) return 0.0f;
    const float y = __fmul_rn(w, inv);
    float r = rintf(y);
    if (fabsf(__fsub_rn(y, r)) >= 0.5f - fabsf(y) * 9.5367431640625e-07f) r = rintf(__fdiv_rn(w, s));
    return fminf(fmaxf(r, lo), hi);
}

// E2M1 round-to-nearest-even with saturation of y >= 0, returned as its value
// in {0, .5, 1, 1.5, 2, 3, 4, 6}.  The spacing of E2M1 values at y is half
// the power of two at or below max(y, 1); adding and subtracting 1.5 * 2^22
// times that power of two rounds y to a multiple of the spacing, half to even
// (even multiples are exactly the even E2M1 codes), and min(., 6) saturates.
__device__ __forceinline__ float e2m1_round(float y) {
    unsigned e = __float_as_uint(y) & 0x7f800000u;
    e = max(e, 0x3f800000u);
    float C = __uint_as_float(e + 0x0b400000u);
    float r = __fsub_rn(__fadd_rn(y, C), C);
    return fminf(r, 6.0f);
}

// Hardware E2M1 conversions of sm_100a.  e2m1x2_from_f32: a pair of fp32
// values rounded to E2M1 (nearest, ties to even, saturating at +-6) and packed
// into one byte, `lo` in the low nibble.  For every non-NaN input y the
// nibble is the magnitude code e2m1_mag_code(e2m1_round(|y|)), with bit 3 set
// when y has its sign bit set (-0 included); tq_selftest_e2m1 checks that on
// every such fp32 value.
__device__ __forceinline__ unsigned e2m1x2_from_f32(float lo, float hi) {
    unsigned short r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %2, %1; cvt.u16.u8 %0, t; }" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}

// Eight values at once: the four e2m1x2 bytes of (x0, x1) .. (x6, x7) packed
// into one word, element i in bits 4i..4i+3.
__device__ __forceinline__ uint32_t e2m1x8_from_f32(float x0, float x1, float x2, float x3, float x4, float x5,
                                                    float x6, float x7) {
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b16 h0, h1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b16 h0, {b0, b1};\n\t"
        "mov.b16 h1, {b2, b3};\n\t"
        "mov.b32 %0, {h0, h1};\n\t}"
        : "=r"(w)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
    return w;
}

// The two E2M1 values of an e2m1x2 byte (low nibble first) as fp32, exactly
// (every E2M1 value is an f16 value; code 8 is -0).
__device__ __forceinline__ float2 e2m1x2_to_f32(unsigned byte) {
    unsigned h2;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(byte));
    __half2_raw raw;
    raw.x = static_cast<unsigned short>(h2 & 0xffffu);
    raw.y = static_cast<unsigned short>(h2 >> 16);
    return __half22float2(__half2(raw));
}

// E2M1 magnitude code (0..7) of a value produced by e2m1_round.
__device__ __forceinline__ int e2m1_mag_code(float v) {
    return v < 2.0f ? static_cast<int>(v * 2.0f) : (v < 4.0f ? static_cast<int>(v) + 2 : (v < 5.0f ? 6 : 7));
}

// E2M1 magnitude of code 0..7: {0, .5, 1, 1.5, 2, 3, 4, 6}.
__device__ __forceinline__ float e2m1_value(unsigned c) {
    return c < 4u ? 0.5f * static_cast<float>(c) : (c < 6u ? static_cast<float>(c - 2u) : (c == 6u ? 4.0f : 6.0f));
}

// E4M3 (e4m3fn) value of code bits c, sign bit ignored (codes 1..126 are the
// positive finite values, 0 is zero), built from the bit fields without an
// integer-to-float conversion: normal codes (exponent field e >= 1, mantissa
// m) are 2^(e-7) (1 + m/8), i.e. the fp32 pattern (c << 20) + (120 << 23);
// subnormal codes are m 2^-9, taken as ((2^23 + m) - 2^23) 2^-9.
__host__ __device__ __forceinline__ float e4m3_value(unsigned c) {
    c &= 0x7fu;
    const uint32_t b = c < 8u ? (0x4b000000u | c) : (c << 20) + 0x3c000000u;
    float v;
    memcpy(&v, &b, sizeof v);
    return c < 8u ? (v - 8388608.0f) * 0.001953125f : v;
}

}  // namespace tq
