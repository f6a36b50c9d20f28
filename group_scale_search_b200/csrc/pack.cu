// Round-to-nearest with given scales + packing, code packing/unpacking and
// dequantization for int3-g64, int4-g128 and NVFP4-g16.
//
// Layouts: "int3-g64 (fmt=5)" (colibri PR #168), Design: Layout bullet (24-byte
// records of a 2-bit low plane and a 1-bit high plane, v + 4); int4 and NVFP4
// records hold one code per nibble, element 2k in the low nibble of byte k.
// Dequantization rounds once to fp32: s v, s (q - z), fl32(fl32(g dec(e)) dec(c)).
#include "group_pack.cuh"

namespace tq {

constexpr int PK_WARPS = 8;

inline int pk_grid(int64_t units, int per_block) {
    const int64_t need = (units + per_block - 1) / per_block;
    return static_cast<int>(min(need, static_cast<int64_t>(num_sms()) * 16));
}

// ------------------------------------------------------------------ RTN + pack with given scales

template <typename T>
__global__ void __launch_bounds__(PK_WARPS * 32)
k_pack_int3(const T* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms,
            const float* __restrict__ scales, uint8_t* __restrict__ packed) {
    const int lane = threadIdx.x & 31;
    const int64_t G = (I + 63) >> 6, OG = O * G, total = n_mat * OG;
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * PK_WARPS + (threadIdx.x >> 5); gid < total;
         gid += static_cast<int64_t>(gridDim.x) * PK_WARPS) {
        const int64_t e = gid / OG, rem = gid - e * OG, o = rem / G, k = rem - o * G;
        const int64_t j0 = k << 6;
        const int n = static_cast<int>(min(static_cast<int64_t>(64), I - j0));
        const T* wp = W + e * ms + o * ld + j0;
        const float s = __ldg(scales + gid);
        const float w0 = lane < n ? Elem<T>::load(wp + lane) : 0.f;
        const float w1 = lane + 32 < n ? Elem<T>::load(wp + lane + 32) : 0.f;
        const unsigned u0 = static_cast<unsigned>(static_cast<int>(rtn_exact(w0, s, -4.f, 3.f)) + 4);
        const unsigned u1 = static_cast<unsigned>(static_cast<int>(rtn_exact(w1, s, -4.f, 3.f)) + 4);
        pack_int3_record(u0, u1, lane, packed + gid * 24);
    }
}

template <typename T>
__global__ void __launch_bounds__(PK_WARPS * 32)
k_pack_int4(const T* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms,
            const float* __restrict__ scales, const uint8_t* __restrict__ zeros, uint8_t* __restrict__ packed) {
    const int lane = threadIdx.x & 31;
    const int64_t G = (I + 127) >> 7, OG = O * G, total = n_mat * OG;
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * PK_WARPS + (threadIdx.x >> 5); gid < total;
         gid += static_cast<int64_t>(gridDim.x) * PK_WARPS) {
        const int64_t e = gid / OG, rem = gid - e * OG, o = rem / G, k = rem - o * G;
        const int64_t j0 = k << 7;
        const int n = static_cast<int>(min(static_cast<int64_t>(128), I - j0));
        const T* wp = W + e * ms + o * ld + j0;
        const float s = __ldg(scales + gid);
        const float z = static_cast<float>(__ldg(zeros + gid));
        unsigned q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * lane + i;
            float qq = z;
            if (j < n && s != 0.f)
                qq = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(Elem<T>::load(wp + j), s)), z), 0.f), 15.f);
            q[i] = static_cast<unsigned>(qq);
        }
        pack_int4_lane(q, lane, packed + gid * 64);
    }
}

template <typename T>
__global__ void __launch_bounds__(PK_WARPS * 32)
k_pack_nvfp4(const T* W, int64_t n_mat, int64_t O, int64_t I, int64_t ld, int64_t ms,
             const uint8_t* __restrict__ scales, const float* __restrict__ gs, uint8_t* __restrict__ packed) {
    const int lane = threadIdx.x & 31, half = lane >> 4, hl = lane & 15;
    const int64_t G = (I + 15) >> 4, OG = O * G, total = n_mat * OG;
    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * PK_WARPS + (threadIdx.x >> 5)) * 2; base < total;
         base += static_cast<int64_t>(gridDim.x) * PK_WARPS * 2) {
        const int64_t bid = base + half;
        const bool vb = bid < total;
        unsigned c4 = 0u;
        if (vb) {
            const int64_t e = bid / OG, rem = bid - e * OG, o = rem / G, kb = rem - o * G;
            const int64_t j = (kb << 4) + hl;
            if (j < I) {
                const float w = Elem<T>::load(W + e * ms + o * ld + j);
                const float S = __fmul_rn(__ldg(gs + e), e4m3_value(__ldg(scales + bid)));
                const float aw = fabsf(w);
                if (S != 0.f && aw != 0.f) {
                    const int mag = e2m1_mag_code(e2m1_round(__fdiv_rn(aw, S)));
                    c4 = static_cast<unsigned>(mag) | ((mag != 0 && w < 0.f) ? 8u : 0u);
                }
            }
        }
        unsigned v = (c4 & 15u) << (4u * static_cast<unsigned>(hl & 7));
        v |= __shfl_xor_sync(FULL, v, 1);
        v |= __shfl_xor_sync(FULL, v, 2);
        v |= __shfl_xor_sync(FULL, v, 4);
        if (vb && (hl & 7) == 0) reinterpret_cast<uint32_t*>(packed + bid * 8)[hl >> 3] = v;
    }
}

// ------------------------------------------------------------------ pack / unpack integer codes

// One thread per group record; codes are dense [rows][cols] bytes.
__global__ void k_pack_codes(const uint8_t* __restrict__ codes, int fmt, int64_t rows, int64_t cols,
                             const uint8_t* __restrict__ zeros, uint8_t* __restrict__ packed) {
    const int g = fmt == TQ_INT3_G64_SYM ? 64 : (fmt == TQ_INT4_G128_ASYM ? 128 : 16);
    const int64_t G = (cols + g - 1) / g;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gid >= rows * G) return;
    const int64_t r = gid / G, k = gid - r * G;
    const uint8_t* c = codes + r * cols + k * g;
    const int n = static_cast<int>(min(static_cast<int64_t>(g), cols - k * g));
    if (fmt == TQ_INT3_G64_SYM) {
        uint32_t lo[4] = {0u, 0u, 0u, 0u};
        uint32_t hi[2] = {0u, 0u};
        for (int i = 0; i < 64; ++i) {
            const unsigned u = (i < n ? static_cast<unsigned>(static_cast<int>(static_cast<int8_t>(c[i])) + 4) : 4u) & 7u;
            lo[i >> 4] |= (u & 3u) << (2 * (i & 15));
            hi[i >> 5] |= (u >> 2) << (i & 31);
        }
        uint32_t* rec = reinterpret_cast<uint32_t*>(packed + gid * 24);
        rec[0] = lo[0]; rec[1] = lo[1]; rec[2] = lo[2]; rec[3] = lo[3]; rec[4] = hi[0]; rec[5] = hi[1];
    } else {
        const unsigned pad = (fmt == TQ_INT4_G128_ASYM && zeros) ? (zeros[gid] & 15u) : 0u;
        uint32_t* rec = reinterpret_cast<uint32_t*>(packed + gid * (g / 2));
        for (int wd = 0; wd < g / 8; ++wd) {
            uint32_t v = 0u;
            for (int i = 0; i < 8; ++i) {
                const int j = wd * 8 + i;
                const unsigned q = (j < n ? c[j] : pad) & 15u;
                v |= q << (4 * i);
            }
            rec[wd] = v;
        }
    }
}

__global__ void k_unpack_codes(const uint8_t* __restrict__ packed, int fmt, int64_t rows, int64_t cols,
                               uint8_t* __restrict__ codes) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= rows * cols) return;
    const int64_t r = idx / cols, j = idx - r * cols;
    if (fmt == TQ_INT3_G64_SYM) {
        const int64_t G = (cols + 63) >> 6;
        const uint8_t* rec = packed + (r * G + (j >> 6)) * 24;
        const int i = static_cast<int>(j & 63);
        const unsigned u = ((rec[i >> 2] >> (2 * (i & 3))) & 3u) | (((rec[16 + (i >> 3)] >> (i & 7)) & 1u) << 2);
        codes[idx] = static_cast<uint8_t>(static_cast<int8_t>(static_cast<int>(u) - 4));
    } else {
        const int g = fmt == TQ_INT4_G128_ASYM ? 128 : 16;
        const int64_t G = (cols + g - 1) / g;
        const uint8_t b = packed[(r * G + j / g) * (g / 2) + (j % g) / 2];
        codes[idx] = (j & 1) ? static_cast<uint8_t>(b >> 4) : static_cast<uint8_t>(b & 15u);
    }
}

// ------------------------------------------------------------------ dequant
// One thread per 16 consecutive outputs of one group: int3 = a quarter
// record (4 low-plane bytes + 2 high-plane bytes), int4 = an eighth (8 bytes),
// NVFP4 = a whole block (8 bytes).

template <typename O> __device__ __forceinline__ O to_out(float v);
template <> __device__ __forceinline__ float to_out<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename O>
__device__ __forceinline__ void store16(O* dst, const float v[16], bool vec_ok, int nvalid) {
    if (vec_ok && nvalid == 16) {
        if constexpr (sizeof(O) == 4) {
            float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int i = 0; i < 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
            uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                uint32_t u[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * k], v[8 * i + 2 * k + 1]);
                    u[k] = *reinterpret_cast<const uint32_t*>(&h);
                }
                d[i] = make_uint4(u[0], u[1], u[2], u[3]);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
            if (i < nvalid) dst[i] = to_out<O>(v[i]);
    }
}

// Grid: x = 256-chunk column tiles of a row (a chunk = 16 weights of one
// group), y = row slices, z = matrices; each thread keeps its chunk column and
// walks the rows of its slice (no integer division in the loop).
template <typename O>
__global__ void __launch_bounds__(256)
k_dequant(const uint8_t* __restrict__ packed, int fmt, const void* scales, const uint8_t* __restrict__ zeros,
          const float* __restrict__ gs, int64_t Orows, int64_t I, int64_t rows_per_slice, O* __restrict__ out) {
    const int lg = fmt == TQ_INT3_G64_SYM ? 2 : (fmt == TQ_INT4_G128_ASYM ? 3 : 0);   // log2(chunks per group)
    const int64_t G = (I + (16 << lg) - 1) >> (4 + lg);
    const int64_t c = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    const int64_t C = (I + 15) >> 4;
    if (c >= C) return;
    const int64_t k = c >> lg;
    const int part = static_cast<int>(c & ((1 << lg) - 1));
    const int64_t e = blockIdx.z;
    const int64_t j = c << 4;
    const int nvalid = static_cast<int>(min(static_cast<int64_t>(16), I - j));
    const bool vec_ok = ((I * static_cast<int64_t>(sizeof(O))) % 16) == 0;
    const int64_t o0 = static_cast<int64_t>(blockIdx.y) * rows_per_slice;
    const int64_t o1 = min(Orows, o0 + rows_per_slice);
    for (int64_t o = o0; o < o1; ++o) {
        const int64_t row = e * Orows + o;
        float v[16];
        dq_unit(fmt, packed, scales, zeros, gs, Orows * G, row * G + k, part, v);
        store16<O>(out + row * I + j, v, vec_ok, nvalid);
    }
}

}  // namespace tq

using namespace tq;

static tq_status check_fmt(int32_t fmt, const char* who) {
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "%s: unknown format %d", who, fmt);
    return TQ_OK;
}

TQ_API tq_status tq_pack(const tq_mat* W, int32_t fmt, const void* scales, const uint8_t* zeros,
                         const float* global_scale, uint8_t* packed, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_pack W");
    if (s != TQ_OK) return s;
    if ((s = check_fmt(fmt, "tq_pack")) != TQ_OK) return s;
    TQ_REQUIRE(scales != nullptr && packed != nullptr, "tq_pack: null scales or packed");
    TQ_REQUIRE(aligned16(packed), "tq_pack: packed not 16-byte aligned");
    TQ_REQUIRE(fmt != TQ_INT4_G128_ASYM || zeros != nullptr, "tq_pack: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_pack: NVFP4 needs global_scale");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0;
    const int64_t G = tq_num_groups(fmt, W->n_mat * W->rows, W->cols);
    const bool bf = W->dtype == TQ_BF16;
    if (fmt == TQ_INT3_G64_SYM) {
        const int grid = pk_grid(G, PK_WARPS);
        if (bf) k_pack_int3<uint16_t><<<grid, PK_WARPS * 32, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->n_mat, W->rows, W->cols, W->ld, ms, static_cast<const float*>(scales), packed);
        else k_pack_int3<float><<<grid, PK_WARPS * 32, 0, st>>>(static_cast<const float*>(W->ptr), W->n_mat, W->rows, W->cols, W->ld, ms, static_cast<const float*>(scales), packed);
    } else if (fmt == TQ_INT4_G128_ASYM) {
        const int grid = pk_grid(G, PK_WARPS);
        if (bf) k_pack_int4<uint16_t><<<grid, PK_WARPS * 32, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->n_mat, W->rows, W->cols, W->ld, ms, static_cast<const float*>(scales), zeros, packed);
        else k_pack_int4<float><<<grid, PK_WARPS * 32, 0, st>>>(static_cast<const float*>(W->ptr), W->n_mat, W->rows, W->cols, W->ld, ms, static_cast<const float*>(scales), zeros, packed);
    } else {
        const int grid = pk_grid(G, 2 * PK_WARPS);
        if (bf) k_pack_nvfp4<uint16_t><<<grid, PK_WARPS * 32, 0, st>>>(static_cast<const uint16_t*>(W->ptr), W->n_mat, W->rows, W->cols, W->ld, ms, static_cast<const uint8_t*>(scales), global_scale, packed);
        else k_pack_nvfp4<float><<<grid, PK_WARPS * 32, 0, st>>>(static_cast<const float*>(W->ptr), W->n_mat, W->rows, W->cols, W->ld, ms, static_cast<const uint8_t*>(scales), global_scale, packed);
    }
    return check_launch("tq_pack");
}

TQ_API tq_status tq_pack_codes(const uint8_t* codes, int32_t fmt, int64_t rows, int64_t cols,
                               const uint8_t* zeros, uint8_t* packed, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_pack_codes");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(codes && packed, "tq_pack_codes: null pointer");
    TQ_REQUIRE(rows >= 1 && cols >= 1, "tq_pack_codes: empty shape");
    TQ_REQUIRE(aligned16(packed), "tq_pack_codes: packed not 16-byte aligned");
    const int64_t n = tq_num_groups(fmt, rows, cols);
    k_pack_codes<<<static_cast<unsigned>((n + 127) / 128), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        codes, fmt, rows, cols, zeros, packed);
    return check_launch("tq_pack_codes");
}

TQ_API tq_status tq_unpack_codes(const uint8_t* packed, int32_t fmt, int64_t rows, int64_t cols,
                                 uint8_t* codes, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_unpack_codes");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(codes && packed, "tq_unpack_codes: null pointer");
    TQ_REQUIRE(rows >= 1 && cols >= 1, "tq_unpack_codes: empty shape");
    const int64_t n = rows * cols;
    k_unpack_codes<<<static_cast<unsigned>((n + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        packed, fmt, rows, cols, codes);
    return check_launch("tq_unpack_codes");
}

TQ_API tq_status tq_dequant(const uint8_t* packed, int32_t fmt, const void* scales, const uint8_t* zeros,
                            const float* global_scale, int64_t n_mat, int64_t O, int64_t I, void* out,
                            int32_t out_dtype, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_dequant");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(packed && scales && out, "tq_dequant: null pointer");
    TQ_REQUIRE(n_mat >= 1 && O >= 1 && I >= 1, "tq_dequant: empty shape");
    TQ_REQUIRE(aligned16(packed) && aligned16(out), "tq_dequant: packed/out not 16-byte aligned");
    TQ_REQUIRE(fmt != TQ_INT4_G128_ASYM || zeros != nullptr, "tq_dequant: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_dequant: NVFP4 needs global_scale");
    if (elem_bytes(out_dtype) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant: out dtype %d", out_dtype);
    const int64_t C = (I + 15) / 16;
    const int64_t cblocks = (C + 255) / 256;
    int64_t slices = (16 * static_cast<int64_t>(num_sms()) + cblocks * n_mat - 1) / (cblocks * n_mat);
    slices = max(static_cast<int64_t>(1), min(slices, O));
    const int64_t rps = (O + slices - 1) / slices;
    slices = (O + rps - 1) / rps;
    const dim3 grid(static_cast<unsigned>(cblocks), static_cast<unsigned>(slices), static_cast<unsigned>(n_mat));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (out_dtype == TQ_BF16)
        k_dequant<__nv_bfloat16><<<grid, 256, 0, st>>>(packed, fmt, scales, zeros, global_scale, O, I, rps,
                                                       static_cast<__nv_bfloat16*>(out));
    else
        k_dequant<float><<<grid, 256, 0, st>>>(packed, fmt, scales, zeros, global_scale, O, I, rps,
                                               static_cast<float*>(out));
    return check_launch("tq_dequant");
}
