// Warp-level packing of one group's codes into its record (shared by the
// fused search kernels and the stand-alone pack kernels).
#pragma once
#include "tq_internal.cuh"

namespace tq {

// int3-g64 record ("int3-g64 (fmt=5)", Design: Layout): lane l holds the
// stored values u = v + 4 of elements l and l + 32.  Low plane (bytes 0..15):
// element i at byte i/4, bits 2(i%4), i.e. bit 2i of the little-endian plane,
// so word w (4 bytes) holds elements 16w..16w+15.  High plane (bytes 16..23):
// element i at bit i of the 64-bit little-endian plane.  Lane 0 stores the 24
// bytes as three 8-byte words (records are 8-byte aligned).
__device__ __forceinline__ void pack_int3_record(unsigned u0, unsigned u1, int lane, uint8_t* rec) {
    const unsigned sh = 2u * static_cast<unsigned>(lane & 15);
    const unsigned a = (u0 & 3u) << sh, b = (u1 & 3u) << sh;
    const bool lo16 = lane < 16;
    const unsigned w0 = __reduce_or_sync(FULL, lo16 ? a : 0u);
    const unsigned w1 = __reduce_or_sync(FULL, lo16 ? 0u : a);
    const unsigned w2 = __reduce_or_sync(FULL, lo16 ? b : 0u);
    const unsigned w3 = __reduce_or_sync(FULL, lo16 ? 0u : b);
    const unsigned h0 = __ballot_sync(FULL, (u0 >> 2) & 1u);
    const unsigned h1 = __ballot_sync(FULL, (u1 >> 2) & 1u);
    if (lane == 0) {
        uint2* r = reinterpret_cast<uint2*>(rec);
        r[0] = make_uint2(w0, w1);
        r[1] = make_uint2(w2, w3);
        r[2] = make_uint2(h0, h1);
    }
}

// int4 records: g/2 bytes, element 2k in the low nibble of byte k.  Lane l
// holds elements EPL l .. EPL l + EPL - 1: with 4 (g128) it stores bytes 2l,
// 2l+1, with 2 (g64) byte l; with 1 (g32) the even lane stores byte l/2 with
// its odd neighbour's code (from a shuffle) in the high nibble.  Every lane
// of the warp must call it.
template <int EPL>
__device__ __forceinline__ void pack_int4_lane(const unsigned q[EPL], int lane, uint8_t* rec) {
    if constexpr (EPL == 4) {
        const unsigned v = (q[0] & 15u) | ((q[1] & 15u) << 4) | ((q[2] & 15u) << 8) | ((q[3] & 15u) << 12);
        reinterpret_cast<uint16_t*>(rec)[lane] = static_cast<uint16_t>(v);
    } else if constexpr (EPL == 2) {
        rec[lane] = static_cast<uint8_t>((q[0] & 15u) | ((q[1] & 15u) << 4));
    } else {
        const unsigned hi = __shfl_down_sync(FULL, q[0] & 15u, 1);
        if ((lane & 1) == 0) rec[lane >> 1] = static_cast<uint8_t>((q[0] & 15u) | (hi << 4));
    }
}

// NVFP4 codes of N (8 or 16) weights under block scale S = fl32(g dec(e)):
// magnitude = E2M1 round-half-to-even, saturating at 6, of the IEEE fp32
// quotient |w| / S; sign in bit 3 when w < 0 and the magnitude is not 0
// (every zero is +0); code 0 when S == 0.  Written as N/8 words of 8
// nibbles, element i of a word in bits 4i..4i+3.
//
// Fast path (S positive, normal and not extreme): with inv = rcp(S), w inv
// approximates the IEEE quotient w / S within 2^-21 relative, so the
// products w inv (1 -+ 2^-20) bracket it.  The hardware conversion rounds
// signed values (ties to even, saturating, sign kept, -0 for a negative value
// that rounds to zero; tq_selftest_e2m1 checks it against the definition on
// every non-NaN fp32 value); E2M1 rounding is monotone, so when both ends
// give the same code that is the quotient's.  A -0 is then made +0 with a
// word-wide test for zero magnitudes.  Otherwise -- a quotient within about
// 2^-20 of a rounding midpoint -- that element's code is redone with an IEEE
// division.  For NaN weights the codes are unspecified.
// The NVFP4 code of one weight from the IEEE quotient (the definition,
// spelled out): magnitude by arithmetic E2M1 rounding, sign when w < 0 and
// the magnitude is not 0.
__device__ __forceinline__ uint32_t nvfp4_code_exact(float w, float S) {
    const float aw = fabsf(w);
    unsigned mag = 0u;
    if (S != 0.f && aw != 0.f) mag = static_cast<unsigned>(e2m1_mag_code(e2m1_round(__fdiv_rn(aw, S)))) & 7u;
    return mag | ((mag != 0u && w < 0.f) ? 8u : 0u);
}

template <int N>
__device__ __forceinline__ void nvfp4_rtn(const float w[N], float S, uint32_t m[N / 8]) {
    const unsigned se = __float_as_uint(S) >> 23;   // sign bit included: positive S gives se < 256
    if (!(S > 0.f) || se < 3u || se > 251u) {       // zero, negative, subnormal or extreme block scale
#pragma unroll
        for (int h = 0; h < N / 8; ++h) {
            m[h] = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) m[h] |= nvfp4_code_exact(w[8 * h + i], S) << (4 * i);
        }
        return;
    }
    const float inv = rcp_approx(S);
    const float lo = __fmul_rn(inv, 0.99999904632568359375f), hi = __fmul_rn(inv, 1.00000095367431640625f);
    const float2 lo2 = make_float2(lo, lo), hi2 = make_float2(hi, hi);
#pragma unroll
    for (int h = 0; h < N / 8; ++h) {
        float yl[8], yh[8];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float2 ww = make_float2(w[8 * h + 2 * p], w[8 * h + 2 * p + 1]);
            const float2 a = __fmul2_rn(ww, lo2), b = __fmul2_rn(ww, hi2);
            yl[2 * p] = a.x; yl[2 * p + 1] = a.y; yh[2 * p] = b.x; yh[2 * p + 1] = b.y;
        }
        uint32_t x = e2m1x8_from_f32(yl[0], yl[1], yl[2], yl[3], yl[4], yl[5], yl[6], yl[7]);
        const uint32_t d = x ^ e2m1x8_from_f32(yh[0], yh[1], yh[2], yh[3], yh[4], yh[5], yh[6], yh[7]);
        if (d) {
            // Elements whose bracket ends disagree take an IEEE division, one
            // at a time: the element is picked with a chain of selects (no
            // per-element branch, no indexed registers).
            uint32_t todo = ((d | (d >> 1) | (d >> 2) | (d >> 3)) & 0x11111111u);
            while (todo) {
                const int b = __ffs(todo) - 1;   // bit 4i of element i
                todo &= todo - 1u;
                float wi = w[8 * h];
#pragma unroll
                for (int i = 1; i < 8; ++i) wi = b == 4 * i ? w[8 * h + i] : wi;
                x = (x & ~(15u << b)) | (nvfp4_code_exact(wi, S) << b);
            }
        }
        // a -0 (sign with magnitude 0) becomes +0: magnitude + 7 carries into
        // bit 3 of its nibble exactly when the magnitude is not 0
        const uint32_t mag = x & 0x77777777u;
        m[h] = mag | (x & (mag + 0x77777777u) & 0x88888888u);
    }
}

}  // namespace tq
