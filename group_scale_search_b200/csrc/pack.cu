// Round-to-nearest with given scales + packing, code packing/unpacking and
// dequantization for int3-g64, int4-g128 and NVFP4-g16.
//
// Layouts: "int3-g64 (fmt=5)" (colibri PR #168), Design: Layout bullet (24-byte
// records of a 2-bit low plane and a 1-bit high plane, v + 4); int4 and NVFP4
// records hold one code per nibble, element 2k in the low nibble of byte k.
// Dequantization rounds once to fp32: s v, s (q - z), fl32(fl32(g dec(e)) dec(c)).
#include "batch.cuh"

namespace tq {

// Blocks of `kernel` (at `threads` per block) resident on one SM.
template <typename K>
int64_t resident_blocks(K kernel, int threads) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

// ------------------------------------------------------------------ RTN + pack with given scales
// One thread per octet column (8 weights of one group, the last group's
// padding included); it writes its share of the record: int3 = 2 low-plane
// bytes + 1 high-plane byte, int4 = 4 bytes, NVFP4 = half the record.

// Octets per thread of tq_pack (one or two consecutive octets of one group:
// two halve the per-row loads of scales and the loop work per weight; for
// NVFP4 two octets are one whole block).
template <int FMT> __host__ __device__ constexpr int pk_no() { return 2; }
// Rows per iteration of tq_pack for int3 and NVFP4 and of tq_dequant (all
// their loads issued before any is used); NVFP4 pack, with the more
// instructions per weight, prefers one row (more resident warps).  int4 pack
// keeps PK_AHEAD rows of loads in flight ahead of the row it packs.
template <int FMT> __host__ __device__ constexpr int pk_rows() { return FMT == TQ_NVFP4_G16 ? 1 : 2; }
constexpr int PK_AHEAD = 1;
constexpr int DQ_ROWS = 2;

// RTN codes of NO consecutive octets (starting at octet `oct` of the group
// whose record is at rec) into their share of the record.  sc: the group's
// scale (NVFP4: the block scale S = fl32(g dec(e))); z: int4 zero-point.
template <int FMT, typename T, int NO>
__device__ __forceinline__ void pack_unit(const Oct<T> o[NO], const int n[NO], float sc, int z, uint8_t* rec,
                                          int oct) {
    if constexpr (FMT == TQ_NVFP4_G16) {   // padding has w = 0: code 0
        float w[8 * NO];
#pragma unroll
        for (int i = 0; i < NO; ++i) o[i].get(w + 8 * i);
        uint32_t m[NO];
        nvfp4_rtn<8 * NO>(w, sc, m);
        if constexpr (NO == 1) reinterpret_cast<uint32_t*>(rec)[oct & 1] = m[0];
        else *reinterpret_cast<uint2*>(rec) = make_uint2(m[0], m[1]);
    } else {
        uint32_t nib[NO];
#pragma unroll
        for (int i = 0; i < NO; ++i) {
            float w[8];
            o[i].get(w);
            nib[i] = FMT == TQ_INT3_G64_SYM ? rtn_int_oct<7>(w, n[i], sc, 4) : rtn_int_oct<15>(w, n[i], sc, z);
        }
        store_unit<FMT, NO>(rec, oct, nib);
    }
}

// One unit of a grouped tq_pack launch.
struct PkUnit {
    const void* W;
    int64_t O, I, ld, ms, n_rows;
    const void* scales;
    const uint8_t* zeros;
    const float* gs;
    uint8_t* packed;
    BatchSlot s;
};
struct PkArgs {
    int n;
    PkUnit u[BATCH_MAX];
};

// Blocks: the units' ranges of the 1-D grid; within a unit, column tiles
// (a unit column = NO octets) times blocks of consecutive rows of its whole
// batch (rows of all matrices in order, so every block gets the same
// number of rows whatever the matrix count).  Pointers to the weights,
// records, scales and zero-points advance by their row strides.
// Row walkers per block (blockDim.y): they share the block's unit columns
// and take interleaved rows of its range.  Measured on the full-size
// workloads: four walkers per block for int3 (0.523 -> 0.479 ms on the MoE
// stack), one for int4 and NVFP4 (four: 0.411 -> 0.550 ms on the NVFP4 MoE
// stack, where the 1024-thread bound leaves one block of 24 warps per SM
// instead of six of 6).
template <int FMT> __host__ __device__ constexpr int pk_py() { return FMT == TQ_INT3_G64_SYM ? 4 : 1; }

// The body of both kernels below: column tile cx (cw unit columns wide) and
// row block ry of one unit.
template <int FMT, typename T, int NO>
__device__ __forceinline__ void pack_rows(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms,
                                          int64_t n_rows, int64_t rpb, const void* scales,
                                          const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
                                          uint8_t* __restrict__ packed, int64_t cx, int64_t ry, int64_t cw) {
    using F = FmtTraits<FMT>;
    const int64_t G = (I + F::group - 1) / F::group;
    const int64_t u = cx * cw + threadIdx.x;
    if (threadIdx.x >= cw || u >= (G << F::lg) / NO) return;   // no barrier in these kernels
    const int64_t c = u * NO;   // first octet of the unit
    const int64_t k = c >> F::lg;
    const int oct = static_cast<int>(c & ((1 << F::lg) - 1));
    const int64_t j = c << 3;
    int n[NO];
#pragma unroll
    for (int i = 0; i < NO; ++i)
        n[i] = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(8), I - j - 8 * i)));
    const int64_t py = blockDim.y;
    const int64_t r0 = ry * rpb + threadIdx.y, r1 = min(n_rows, r0 - threadIdx.y + rpb);
    RowCursor<T> cur(W, O, ld, ms, j, r0);
    const int64_t rstride = py * G * F::rec;   // this walker's rows: r0, r0 + py, ...
    uint8_t* rec = packed + (r0 * G + k) * F::rec;
    const float* sp = static_cast<const float*>(scales) + (r0 * G + k);          // int3, int4
    const uint8_t* bp = static_cast<const uint8_t*>(scales) + (r0 * G + k);      // NVFP4 block scales
    const uint8_t* zp = zeros ? zeros + (r0 * G + k) : nullptr;
    int64_t ecur = cur.e;
    float g = (FMT == TQ_NVFP4_G16 && r0 < r1) ? __ldg(gs + ecur) : 0.f;
    if constexpr (is_int4(FMT)) {
        // int4: a ring of PK_AHEAD rows.  A row's loads (weights, scale,
        // zero-point) are issued PK_AHEAD rows before it is packed and used
        // only then, so the walker keeps rows in flight while it computes
        // (0.637 -> 0.685 of the HBM peak on the grouped 27B-layer
        // projections; int3 and NVFP4, whose walkers hold more registers,
        // measured slower this way and load two rows, or one, then pack them).
        constexpr int L = PK_AHEAD;
        Oct<T> rw[L][NO];
        float sr[L];
        int zc[L];
        int64_t rl = r0;
        auto load = [&](int h) {
            sr[h] = 0.f;
            zc[h] = 0;
            if (rl < r1) {
#pragma unroll
                for (int i = 0; i < NO; ++i) rw[h][i].load(cur.ptr + 8 * i, n[i]);
                sr[h] = __ldg(sp);
                zc[h] = __ldg(zp);
            }
            cur.advance(py);
            rl += py;
            sp += py * G;
            zp += py * G;
        };
#pragma unroll
        for (int h = 0; h < L; ++h) load(h);
        for (int64_t r = r0; r < r1; r += L * py) {
#pragma unroll
            for (int h = 0; h < L; ++h) {
                if (r + h * py >= r1) break;
                Oct<T> w[NO];
#pragma unroll
                for (int i = 0; i < NO; ++i) w[i] = rw[h][i];
                const float s0 = sr[h];
                const int z0 = zc[h];
                load(h);   // the row L rows on
                pack_unit<FMT, T, NO>(w, n, s0, z0, rec + h * rstride, oct);
            }
            rec += L * rstride;
        }
    } else {
        constexpr int ROWS = pk_rows<FMT>();
        for (int64_t r = r0; r < r1; r += ROWS * py) {
            Oct<T> rw[ROWS][NO];
            float sc[ROWS];
#pragma unroll
            for (int h = 0; h < ROWS; ++h) {
                sc[h] = 0.f;
                if (r + h * py < r1) {
#pragma unroll
                    for (int i = 0; i < NO; ++i) rw[h][i].load(cur.ptr + 8 * i, n[i]);
                    if constexpr (FMT == TQ_NVFP4_G16) {
                        if (cur.e != ecur) { ecur = cur.e; g = __ldg(gs + ecur); }
                        sc[h] = __fmul_rn(g, e4m3_value(__ldg(bp + h * py * G)));
                    } else {
                        sc[h] = __ldg(sp + h * py * G);
                    }
                }
                cur.advance(py);
            }
#pragma unroll
            for (int h = 0; h < ROWS; ++h) {
                if (r + h * py >= r1) break;
                pack_unit<FMT, T, NO>(rw[h], n, sc[h], 0, rec + h * rstride, oct);
            }
            rec += ROWS * rstride;
            sp += ROWS * py * G;
            bp += ROWS * py * G;
        }
    }
}

// Resident blocks the one-unit int4 pack is compiled for: 64 registers, so
// a dense matrix's 256-wide tiles fit four blocks per SM (0.43 -> 0.47 of the
// HBM peak on 4096 x 4096; the grouped kernel measured slower so bounded and
// keeps the compiler's choice).  0 leaves the other formats to the compiler.
template <int FMT> __host__ __device__ constexpr int pk_min_blocks() { return is_int4(FMT) ? 4 : 0; }

// One unit: grid x = column tiles, y = row blocks.
template <int FMT, typename T, int NO>
__global__ void __launch_bounds__(256 * pk_py<FMT>(), pk_min_blocks<FMT>())
k_pack(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms, int64_t n_rows, int64_t rpb,
       const void* scales, const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
       uint8_t* __restrict__ packed) {
    pack_rows<FMT, T, NO>(W, O, I, ld, ms, n_rows, rpb, scales, zeros, gs, packed, blockIdx.x, blockIdx.y,
                          blockDim.x);
}

// Several units: each block looks up its unit's range of the 1-D grid.
template <int FMT, typename T, int NO>
__global__ void __launch_bounds__(256 * pk_py<FMT>())
k_pack_batch(const __grid_constant__ PkArgs a) {
    const PkUnit& p = a.u[batch_unit(a.u, a.n, blockIdx.x)];
    const int64_t lb = static_cast<int64_t>(blockIdx.x) - p.s.block0;
    pack_rows<FMT, T, NO>(static_cast<const T*>(p.W), p.O, p.I, p.ld, p.ms, p.n_rows, p.s.rpb, p.scales, p.zeros,
                          p.gs, p.packed, lb % p.s.cblocks, lb / p.s.cblocks, p.s.cw);
}

// ------------------------------------------------------------------ pack / unpack integer codes

// One thread per group record; codes are dense [rows][cols] bytes.
__global__ void k_pack_codes(const uint8_t* __restrict__ codes, int fmt, int64_t rows, int64_t cols,
                             const uint8_t* __restrict__ zeros, uint8_t* __restrict__ packed) {
    const int g = static_cast<int>(group_of(fmt));
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
        const unsigned pad = (is_int4(fmt) && zeros) ? (zeros[gid] & 15u) : 0u;
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
        const int g = static_cast<int>(group_of(fmt));
        const int64_t G = (cols + g - 1) / g;
        const uint8_t b = packed[(r * G + j / g) * (g / 2) + (j % g) / 2];
        codes[idx] = (j & 1) ? static_cast<uint8_t>(b >> 4) : static_cast<uint8_t>(b & 15u);
    }
}

// ------------------------------------------------------------------ dequant
// One thread per octet column (8 consecutive outputs of one group).

template <typename O>
__device__ __forceinline__ void store8(O* dst, const float v[8], bool vec_ok, int nvalid) {
    if (vec_ok && nvalid == 8) {
        if constexpr (sizeof(O) == 4) {
            float4* d = reinterpret_cast<float4*>(dst);
            d[0] = make_float4(v[0], v[1], v[2], v[3]);
            d[1] = make_float4(v[4], v[5], v[6], v[7]);
        } else {
            uint32_t u[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
                u[k] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(dst) = make_uint4(u[0], u[1], u[2], u[3]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < nvalid) {
                if constexpr (sizeof(O) == 4) dst[i] = v[i];
                else dst[i] = __float2bfloat16_rn(v[i]);
            }
        }
    }
}

// One unit of a grouped tq_dequant launch.
struct DqUnit {
    const uint8_t* packed;
    const void* scales;
    const uint8_t* zeros;
    const float* gs;
    int64_t Orows, I, n_rows;
    void* out;
    BatchSlot s;
};
struct DqArgs {
    int n;
    DqUnit u[BATCH_MAX];
};

// Within a unit: octet-column tiles times blocks of consecutive rows of its
// whole batch (the output is dense, so a row's place does not depend on its
// matrix).  A thread loads DQ_ROWS rows' codes and scales before decoding
// any of them.  The body of both kernels below: column tile cx (cw octet
// columns wide) and row block ry of one unit.
template <int FMT, typename O>
__device__ __forceinline__ void dequant_rows(const uint8_t* __restrict__ packed, const void* scales,
                                             const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
                                             int64_t Orows, int64_t I, int64_t n_rows, int64_t rpb,
                                             O* __restrict__ out, int64_t cx, int64_t ry, int64_t cw) {
    using F = FmtTraits<FMT>;
    const int64_t G = (I + F::group - 1) / F::group;
    const int64_t c = cx * cw + threadIdx.x;
    if (threadIdx.x >= cw || c >= ((I + 7) >> 3)) return;
    const int64_t k = c >> F::lg;
    const int oct = static_cast<int>(c & ((1 << F::lg) - 1));
    const int64_t j = c << 3;
    const int nvalid = static_cast<int>(min(static_cast<int64_t>(8), I - j));
    const bool vec_ok = ((I * static_cast<int64_t>(sizeof(O))) % 16) == 0;
    const int64_t r0 = ry * rpb, r1 = min(n_rows, r0 + rpb);
    int64_t e = 0, next_e = n_rows;   // NVFP4: matrix of row r and the first row of the next matrix
    float g = 0.f;
    if (FMT == TQ_NVFP4_G16) {
        e = r0 / Orows;
        next_e = (e + 1) * Orows;
        g = __ldg(gs + e);
    }
    QPtr<FMT> qp(packed, scales, zeros, r0 * G + k, G);
    O* dst = out + r0 * I + j;
    for (int64_t r = r0; r < r1; r += DQ_ROWS, dst += DQ_ROWS * I) {
        OctQ q[DQ_ROWS];
#pragma unroll
        for (int h = 0; h < DQ_ROWS; ++h) {
            if (r + h < r1) q[h] = load_q<FMT>(qp, oct);
            qp.next();
        }
#pragma unroll
        for (int h = 0; h < DQ_ROWS; ++h) {
            if (r + h >= r1) break;
            if (FMT == TQ_NVFP4_G16 && r + h == next_e) { ++e; next_e += Orows; g = __ldg(gs + e); }
            float v[8];
            dec_oct<FMT>(q[h], g, v);
            store8<O>(dst + h * I, v, vec_ok, nvalid);
        }
    }
}

// One unit: grid x = octet-column tiles, y = row blocks.  At most 32
// registers (8 blocks of 256 threads per SM): the loads in flight come from
// resident warps.
template <int FMT, typename O>
__global__ void __launch_bounds__(256, 8)
k_dequant(const uint8_t* __restrict__ packed, const void* scales, const uint8_t* __restrict__ zeros,
          const float* __restrict__ gs, int64_t Orows, int64_t I, int64_t n_rows, int64_t rpb, O* __restrict__ out) {
    dequant_rows<FMT, O>(packed, scales, zeros, gs, Orows, I, n_rows, rpb, out, blockIdx.x, blockIdx.y, blockDim.x);
}

// Several units: each block looks up its unit's range of the 1-D grid.
template <int FMT, typename O>
__global__ void __launch_bounds__(256, 8)
k_dequant_batch(const __grid_constant__ DqArgs a) {
    const DqUnit& p = a.u[batch_unit(a.u, a.n, blockIdx.x)];
    const int64_t lb = static_cast<int64_t>(blockIdx.x) - p.s.block0;
    dequant_rows<FMT, O>(p.packed, p.scales, p.zeros, p.gs, p.Orows, p.I, p.n_rows, p.s.rpb, static_cast<O*>(p.out),
                         lb % p.s.cblocks, lb / p.s.cblocks, p.s.cw);
}

// ------------------------------------------------------------------ host launchers
// The grid holds at most as many blocks as the SMs keep resident (one wave),
// split over the units by size; within a unit, rows split evenly over its
// row blocks.

template <int FMT, typename T>
void launch_pack(int n, const tq_mat* W, const void* const* scales, const uint8_t* const* zeros,
                 const float* const* gs, uint8_t* const* packed, cudaStream_t st) {
    const int64_t g = FmtTraits<FMT>::group;
    constexpr int NO = pk_no<FMT>();
    constexpr int PY = pk_py<FMT>();
    int64_t cols[BATCH_MAX], rows[BATCH_MAX];
    for (int i = 0; i < n; ++i) {
        cols[i] = (W[i].cols + g - 1) / g * (g / 8) / NO;
        rows[i] = W[i].n_mat * W[i].rows;
    }
    int64_t width = 32;
    BatchSlot sl[BATCH_MAX];
    batch_split(n, cols, rows, 1, sl, &width);   // the widest tile sets the block shape
    const dim3 block(static_cast<unsigned>(width), static_cast<unsigned>(PY));
    if (n == 1) {
        const int64_t slots = static_cast<int64_t>(num_sms()) * resident_blocks(k_pack<FMT, T, NO>, static_cast<int>(width) * PY);
        batch_split(1, cols, rows, slots, sl, &width);
        const int64_t ms = W->n_mat > 1 ? W->mat_stride : 0;
        const dim3 grid(static_cast<unsigned>(sl[0].cblocks), static_cast<unsigned>(sl[0].rblocks));
        k_pack<FMT, T, NO><<<grid, block, 0, st>>>(static_cast<const T*>(W->ptr), W->rows, W->cols, W->ld, ms,
                                                   rows[0], sl[0].rpb, scales[0], zeros ? zeros[0] : nullptr,
                                                   gs ? gs[0] : nullptr, packed[0]);
        return;
    }
    static thread_local PkArgs a;
    const int64_t slots = static_cast<int64_t>(num_sms()) * resident_blocks(k_pack_batch<FMT, T, NO>, static_cast<int>(width) * PY);
    const int64_t blocks = batch_split(n, cols, rows, slots, sl, &width);
    a.n = n;
    for (int i = 0; i < n; ++i) {
        PkUnit& u = a.u[i];
        u.W = W[i].ptr; u.O = W[i].rows; u.I = W[i].cols; u.ld = W[i].ld;
        u.ms = W[i].n_mat > 1 ? W[i].mat_stride : 0;
        u.n_rows = rows[i];
        u.scales = scales[i]; u.zeros = zeros ? zeros[i] : nullptr; u.gs = gs ? gs[i] : nullptr;
        u.packed = packed[i];
        u.s = sl[i];
    }
    k_pack_batch<FMT, T, NO><<<static_cast<unsigned>(blocks), block, 0, st>>>(a);
}

template <int FMT, typename O>
void launch_dequant(int n, const uint8_t* const* packed, const void* const* scales, const uint8_t* const* zeros,
                    const float* const* gs, const int64_t* n_mat, const int64_t* Orows, const int64_t* I,
                    void* const* out, cudaStream_t st) {
    int64_t cols[BATCH_MAX], rows[BATCH_MAX];
    for (int i = 0; i < n; ++i) {
        cols[i] = (I[i] + 7) / 8;
        rows[i] = n_mat[i] * Orows[i];
    }
    int64_t width = 32;
    BatchSlot sl[BATCH_MAX];
    batch_split(n, cols, rows, 1, sl, &width);
    if (n == 1) {
        const int64_t slots = static_cast<int64_t>(num_sms()) * resident_blocks(k_dequant<FMT, O>, static_cast<int>(width));
        batch_split(1, cols, rows, slots, sl, &width);
        const dim3 grid(static_cast<unsigned>(sl[0].cblocks), static_cast<unsigned>(sl[0].rblocks));
        k_dequant<FMT, O><<<grid, static_cast<unsigned>(width), 0, st>>>(
            packed[0], scales[0], zeros ? zeros[0] : nullptr, gs ? gs[0] : nullptr, Orows[0], I[0], rows[0],
            sl[0].rpb, static_cast<O*>(out[0]));
        return;
    }
    static thread_local DqArgs a;
    const int64_t slots = static_cast<int64_t>(num_sms()) * resident_blocks(k_dequant_batch<FMT, O>, static_cast<int>(width));
    const int64_t blocks = batch_split(n, cols, rows, slots, sl, &width);
    a.n = n;
    for (int i = 0; i < n; ++i) {
        DqUnit& u = a.u[i];
        u.packed = packed[i]; u.scales = scales[i]; u.zeros = zeros ? zeros[i] : nullptr; u.gs = gs ? gs[i] : nullptr;
        u.Orows = Orows[i]; u.I = I[i]; u.n_rows = rows[i]; u.out = out[i];
        u.s = sl[i];
    }
    k_dequant_batch<FMT, O><<<static_cast<unsigned>(blocks), static_cast<unsigned>(width), 0, st>>>(a);
}

}  // namespace tq

using namespace tq;

static tq_status check_fmt(int32_t fmt, const char* who) {
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "%s: unknown format %d", who, fmt);
    return TQ_OK;
}

// Checks of one unit of tq_pack / tq_pack_batch.
static tq_status check_pack_unit(const tq_mat* W, int32_t fmt, const void* scales, const uint8_t* zeros,
                                 const float* global_scale, const uint8_t* packed, const char* who) {
    tq_status s = check_mat(W, who);
    if (s != TQ_OK) return s;
    TQ_REQUIRE(scales != nullptr && packed != nullptr, "%s: null scales or packed", who);
    TQ_REQUIRE(aligned16(packed), "%s: packed not 16-byte aligned", who);
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "%s: int4 needs zeros", who);
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "%s: NVFP4 needs global_scale", who);
    return TQ_OK;
}

static void dispatch_pack(int n, const tq_mat* W, int32_t fmt, const void* const* scales,
                          const uint8_t* const* zeros, const float* const* gs, uint8_t* const* packed,
                          cudaStream_t st) {
    const bool bf = W[0].dtype == TQ_BF16;
    if (fmt == TQ_INT3_G64_SYM) bf ? launch_pack<TQ_INT3_G64_SYM, uint16_t>(n, W, scales, zeros, gs, packed, st)
                                   : launch_pack<TQ_INT3_G64_SYM, float>(n, W, scales, zeros, gs, packed, st);
    else if (fmt == TQ_INT4_G128_ASYM) bf ? launch_pack<TQ_INT4_G128_ASYM, uint16_t>(n, W, scales, zeros, gs, packed, st)
                                          : launch_pack<TQ_INT4_G128_ASYM, float>(n, W, scales, zeros, gs, packed, st);
    else if (fmt == TQ_INT4_G64_ASYM) bf ? launch_pack<TQ_INT4_G64_ASYM, uint16_t>(n, W, scales, zeros, gs, packed, st)
                                         : launch_pack<TQ_INT4_G64_ASYM, float>(n, W, scales, zeros, gs, packed, st);
    else if (fmt == TQ_INT4_G32_ASYM) bf ? launch_pack<TQ_INT4_G32_ASYM, uint16_t>(n, W, scales, zeros, gs, packed, st)
                                         : launch_pack<TQ_INT4_G32_ASYM, float>(n, W, scales, zeros, gs, packed, st);
    else bf ? launch_pack<TQ_NVFP4_G16, uint16_t>(n, W, scales, zeros, gs, packed, st)
            : launch_pack<TQ_NVFP4_G16, float>(n, W, scales, zeros, gs, packed, st);
}

TQ_API tq_status tq_pack(const tq_mat* W, int32_t fmt, const void* scales, const uint8_t* zeros,
                         const float* global_scale, uint8_t* packed, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_pack");
    if (s != TQ_OK) return s;
    if ((s = check_pack_unit(W, fmt, scales, zeros, global_scale, packed, "tq_pack")) != TQ_OK) return s;
    dispatch_pack(1, W, fmt, &scales, &zeros, &global_scale, &packed, reinterpret_cast<cudaStream_t>(stream));
    return check_launch("tq_pack");
}

TQ_API tq_status tq_pack_batch(int32_t n, const tq_mat* W, int32_t fmt, const void* const* scales,
                               const uint8_t* const* zeros, const float* const* global_scale,
                               uint8_t* const* packed, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_pack_batch");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(n >= 1 && n <= TQ_MAX_BATCH, "tq_pack_batch: n = %d outside [1, %d]", n, TQ_MAX_BATCH);
    TQ_REQUIRE(W && scales && packed, "tq_pack_batch: null array");
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "tq_pack_batch: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_pack_batch: NVFP4 needs global_scale");
    for (int i = 0; i < n; ++i) {
        if ((s = check_pack_unit(&W[i], fmt, scales[i], zeros ? zeros[i] : nullptr,
                                 global_scale ? global_scale[i] : nullptr, packed[i], "tq_pack_batch")) != TQ_OK)
            return s;
        TQ_REQUIRE(W[i].dtype == W[0].dtype, "tq_pack_batch: units of different dtypes");
    }
    dispatch_pack(n, W, fmt, scales, zeros, global_scale, packed, reinterpret_cast<cudaStream_t>(stream));
    return check_launch("tq_pack_batch");
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

static tq_status check_dequant_unit(const uint8_t* packed, int32_t fmt, const void* scales, const uint8_t* zeros,
                                    const float* global_scale, int64_t n_mat, int64_t O, int64_t I, const void* out,
                                    const char* who) {
    TQ_REQUIRE(packed && scales && out, "%s: null pointer", who);
    TQ_REQUIRE(n_mat >= 1 && O >= 1 && I >= 1, "%s: empty shape", who);
    TQ_REQUIRE(aligned16(packed) && aligned16(out), "%s: packed/out not 16-byte aligned", who);
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "%s: int4 needs zeros", who);
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "%s: NVFP4 needs global_scale", who);
    return TQ_OK;
}

static void dispatch_dequant(int n, const uint8_t* const* packed, int32_t fmt, const void* const* scales,
                             const uint8_t* const* zeros, const float* const* gs, const int64_t* n_mat,
                             const int64_t* O, const int64_t* I, void* const* out, bool bf, cudaStream_t st) {
    if (fmt == TQ_INT3_G64_SYM)
        bf ? launch_dequant<TQ_INT3_G64_SYM, __nv_bfloat16>(n, packed, scales, zeros, gs, n_mat, O, I, out, st)
           : launch_dequant<TQ_INT3_G64_SYM, float>(n, packed, scales, zeros, gs, n_mat, O, I, out, st);
    else if (fmt == TQ_INT4_G128_ASYM)
        bf ? launch_dequant<TQ_INT4_G128_ASYM, __nv_bfloat16>(n, packed, scales, zeros, gs, n_mat, O, I, out, st)
           : launch_dequant<TQ_INT4_G128_ASYM, float>(n, packed, scales, zeros, gs, n_mat, O, I, out, st);
    else if (fmt == TQ_INT4_G64_ASYM)
        bf ? launch_dequant<TQ_INT4_G64_ASYM, __nv_bfloat16>(n, packed, scales, zeros, gs, n_mat, O, I, out, st)
           : launch_dequant<TQ_INT4_G64_ASYM, float>(n, packed, scales, zeros, gs, n_mat, O, I, out, st);
    else if (fmt == TQ_INT4_G32_ASYM)
        bf ? launch_dequant<TQ_INT4_G32_ASYM, __nv_bfloat16>(n, packed, scales, zeros, gs, n_mat, O, I, out, st)
           : launch_dequant<TQ_INT4_G32_ASYM, float>(n, packed, scales, zeros, gs, n_mat, O, I, out, st);
    else
        bf ? launch_dequant<TQ_NVFP4_G16, __nv_bfloat16>(n, packed, scales, zeros, gs, n_mat, O, I, out, st)
           : launch_dequant<TQ_NVFP4_G16, float>(n, packed, scales, zeros, gs, n_mat, O, I, out, st);
}

TQ_API tq_status tq_dequant(const uint8_t* packed, int32_t fmt, const void* scales, const uint8_t* zeros,
                            const float* global_scale, int64_t n_mat, int64_t O, int64_t I, void* out,
                            int32_t out_dtype, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_dequant");
    if (s != TQ_OK) return s;
    if ((s = check_dequant_unit(packed, fmt, scales, zeros, global_scale, n_mat, O, I, out, "tq_dequant")) != TQ_OK)
        return s;
    if (elem_bytes(out_dtype) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant: out dtype %d", out_dtype);
    dispatch_dequant(1, &packed, fmt, &scales, &zeros, &global_scale, &n_mat, &O, &I, &out, out_dtype == TQ_BF16,
                     reinterpret_cast<cudaStream_t>(stream));
    return check_launch("tq_dequant");
}

TQ_API tq_status tq_dequant_batch(int32_t n, const uint8_t* const* packed, int32_t fmt, const void* const* scales,
                                  const uint8_t* const* zeros, const float* const* global_scale,
                                  const int64_t* n_mat, const int64_t* O, const int64_t* I, void* const* out,
                                  int32_t out_dtype, tq_stream_t stream) {
    clear_error();
    tq_status s = check_fmt(fmt, "tq_dequant_batch");
    if (s != TQ_OK) return s;
    TQ_REQUIRE(n >= 1 && n <= TQ_MAX_BATCH, "tq_dequant_batch: n = %d outside [1, %d]", n, TQ_MAX_BATCH);
    TQ_REQUIRE(packed && scales && n_mat && O && I && out, "tq_dequant_batch: null array");
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "tq_dequant_batch: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_dequant_batch: NVFP4 needs global_scale");
    if (elem_bytes(out_dtype) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_dequant_batch: out dtype %d", out_dtype);
    for (int i = 0; i < n; ++i)
        if ((s = check_dequant_unit(packed[i], fmt, scales[i], zeros ? zeros[i] : nullptr,
                                    global_scale ? global_scale[i] : nullptr, n_mat[i], O[i], I[i], out[i],
                                    "tq_dequant_batch")) != TQ_OK)
            return s;
    dispatch_dequant(n, packed, fmt, scales, zeros, global_scale, n_mat, O, I, out, out_dtype == TQ_BF16,
                     reinterpret_cast<cudaStream_t>(stream));
    return check_launch("tq_dequant_batch");
}
