// Self-test of the hardware E2M1 conversions that the NVFP4 path relies on
// (round-to-nearest of a block's elements in the RTN, packing and search, and
// decoding in dequantization and the proxy error), against the arithmetic
// definition: round half to even on the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6},
// saturating at 6 ("NVFP4" element format: E2M1 with an E4M3 block scale).
//
// Rounding: every fp32 value but NaN (both signs, zeros and infinities
// included; a negative value keeps its sign bit in bit 3 of the nibble, -0
// too), once in the low nibble (paired with 6.0) and once in the high nibble
// (paired with 0.0), so both the values and the nibble order are checked,
// and once through the eight-value form used for whole octets.
// Decoding: all 256 bytes, bit for bit (code 8 is -0).
#include "tq_internal.cuh"

namespace tq {

static __device__ unsigned long long g_st_count;
static __device__ unsigned g_st_first;

__global__ void k_selftest_e2m1_round() {
    const uint64_t half = 0x7f800001ull;   // fp32 bit patterns +0 .. +inf, then -0 .. -inf
    unsigned long long bad = 0;
    unsigned first = 0xffffffffu;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < 2 * half;
         i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const unsigned u = i < half ? static_cast<unsigned>(i) : (static_cast<unsigned>(i - half) | 0x80000000u);
        const float y = __uint_as_float(u);
        const unsigned r = static_cast<unsigned>(e2m1_mag_code(e2m1_round(fabsf(y)))) | ((u >> 28) & 8u);
        const unsigned a = e2m1x2_from_f32(y, 6.0f);
        const unsigned b = e2m1x2_from_f32(0.0f, y);
        // eight at once: (y, 6, 0, y, -y, 1, y, .5) -> nibbles (r, 7, 0, r, r ^ 8, 2, r, 1)
        const uint32_t w8 = e2m1x8_from_f32(y, 6.0f, 0.0f, y, -y, 1.0f, y, 0.5f);
        const uint32_t e8 = r | (7u << 4) | (r << 12) | ((r ^ 8u) << 16) | (2u << 20) | (r << 24) | (1u << 28);
        if (a != (r | 0x70u) || b != (r << 4) || w8 != e8) {
            ++bad;
            first = min(first, u);
        }
    }
    if (bad) {
        atomicAdd(&g_st_count, bad);
        atomicMin(&g_st_first, first);
    }
}

__global__ void k_selftest_e2m1_decode() {
    const unsigned b = threadIdx.x;   // one byte per thread, 256 threads
    const float2 v = e2m1x2_to_f32(b);
    const unsigned lo = b & 15u, hi = b >> 4;
    const float elo = (lo & 8u) ? -e2m1_value(lo & 7u) : e2m1_value(lo & 7u);
    const float ehi = (hi & 8u) ? -e2m1_value(hi & 7u) : e2m1_value(hi & 7u);
    if (__float_as_uint(v.x) != __float_as_uint(elo) || __float_as_uint(v.y) != __float_as_uint(ehi)) {
        atomicAdd(&g_st_count, 1ull);
        atomicMin(&g_st_first, 0x80000000u | b);
    }
}

}  // namespace tq

using namespace tq;

TQ_API tq_status tq_selftest_e2m1(uint64_t* mismatches, uint32_t* first_bad, tq_stream_t stream) {
    clear_error();
    TQ_REQUIRE(mismatches != nullptr, "tq_selftest_e2m1: null mismatches");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const unsigned long long zero = 0;
    const unsigned none = 0xffffffffu;
    cudaError_t ce = cudaMemcpyToSymbolAsync(g_st_count, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st);
    if (ce == cudaSuccess) ce = cudaMemcpyToSymbolAsync(g_st_first, &none, sizeof none, 0, cudaMemcpyHostToDevice, st);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_selftest_e2m1: %s", cudaGetErrorString(ce));
    k_selftest_e2m1_round<<<num_sms() * 8, 256, 0, st>>>();
    tq_status s = check_launch("tq_selftest_e2m1 round");
    if (s != TQ_OK) return s;
    k_selftest_e2m1_decode<<<1, 256, 0, st>>>();
    if ((s = check_launch("tq_selftest_e2m1 decode")) != TQ_OK) return s;
    unsigned long long cnt = 0;
    unsigned first = 0;
    ce = cudaMemcpyFromSymbolAsync(&cnt, g_st_count, sizeof cnt, 0, cudaMemcpyDeviceToHost, st);
    if (ce == cudaSuccess) ce = cudaMemcpyFromSymbolAsync(&first, g_st_first, sizeof first, 0, cudaMemcpyDeviceToHost, st);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_selftest_e2m1: %s", cudaGetErrorString(ce));
    *mismatches = cnt;
    if (first_bad) *first_bad = first;
    return TQ_OK;
}
