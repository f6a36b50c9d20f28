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

// int4-g128 record: 64 bytes, element 2k in the low nibble of byte k.  Lane l
// holds elements 4l..4l+3 and stores bytes 2l, 2l+1.
__device__ __forceinline__ void pack_int4_lane(const unsigned q[4], int lane, uint8_t* rec) {
    const unsigned v = (q[0] & 15u) | ((q[1] & 15u) << 4) | ((q[2] & 15u) << 8) | ((q[3] & 15u) << 12);
    reinterpret_cast<uint16_t*>(rec)[lane] = static_cast<uint16_t>(v);
}

// NVFP4-g16 record: 8 bytes, element 2k in the low nibble of byte k.  The 16
// lanes of a half-warp hold one block's codes (lane hl = element hl); lanes
// hl = 0 and 8 store the two 4-byte words.
__device__ __forceinline__ void pack_nvfp4_half(unsigned code, int hl, unsigned mask, uint8_t* rec) {
    unsigned v = (code & 15u) << (4u * static_cast<unsigned>(hl & 7));
    v |= __shfl_xor_sync(mask, v, 1);
    v |= __shfl_xor_sync(mask, v, 2);
    v |= __shfl_xor_sync(mask, v, 4);
    if ((hl & 7) == 0) reinterpret_cast<uint32_t*>(rec)[hl >> 3] = v;
}

// Dequantizes the 16 weights of unit (group gid, part) into v[], rounding
// once to fp32: int3 s v, int4 s (q - z), NVFP4 fl32(fl32(g dec(e)) dec(c)).
// blocks_per_mat (O * G) maps an NVFP4 block to its matrix's global scale.
__device__ __forceinline__ void dq_unit(int fmt, const uint8_t* __restrict__ packed, const void* scales,
                                        const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
                                        int64_t blocks_per_mat, int64_t gid, int part, float v[16]) {
    if (fmt == TQ_INT3_G64_SYM) {
        const uint8_t* rec = packed + gid * 24;
        const uint32_t lo = __ldg(reinterpret_cast<const uint32_t*>(rec) + part);
        const uint32_t hi = __ldg(reinterpret_cast<const uint16_t*>(rec + 16) + part);
        const float s = __ldg(static_cast<const float*>(scales) + gid);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int u = static_cast<int>(((lo >> (2 * i)) & 3u) | (((hi >> i) & 1u) << 2));
            v[i] = __fmul_rn(s, static_cast<float>(u - 4));
        }
    } else if (fmt == TQ_INT4_G128_ASYM) {
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(packed + gid * 64) + part);
        const float s = __ldg(static_cast<const float*>(scales) + gid);
        const int z = __ldg(zeros + gid);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t wd = i < 8 ? b.x : b.y;
            const int q = static_cast<int>((wd >> (4 * (i & 7))) & 15u);
            v[i] = __fmul_rn(s, static_cast<float>(q - z));
        }
    } else {
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(packed + gid * 8));
        const int64_t e = gid / blocks_per_mat;
        const float S = __fmul_rn(__ldg(gs + e), e4m3_value(__ldg(static_cast<const uint8_t*>(scales) + gid)));
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t wd = i < 8 ? b.x : b.y;
            const unsigned c = (wd >> (4 * (i & 7))) & 15u;
            const float mg = e2m1_value(c & 7u);
            v[i] = __fmul_rn(S, (c & 8u) ? -mg : mg);
        }
    }
}

}  // namespace tq
