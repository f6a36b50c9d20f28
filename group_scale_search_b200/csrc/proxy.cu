// imatrix-weighted reconstruction error per matrix ("Quantize on TT cards:
// CUDA-free GPTQ/LDLQ bfp4 pipeline", tt-stack issue #67, "Risks to measure:
// Precision": proxy error tr(E H E^T) / tr(W H W^T)); with H = diag(m):
//   num = sum_{o,j} m_j (W - What)^2,  den = sum_{o,j} m_j W^2.
//
// B200 mapping (HBM-bound): one thread per two octets (16 consecutive
// weights of a group, two 16-byte loads of bf16) walking the rows of its
// block; its 16 imatrix weights sit in shared memory (read only by it), it
// dequantizes in registers (no What round trip through memory), sums the
// terms in fp32 and folds them into fp64 per row.  The blocks split the rows
// of the whole batch (all matrices' rows in order) evenly, one wave of
// resident blocks, so every SM is kept busy whatever the matrix count; where
// a block's rows cross from one matrix to the next it writes the fp64
// partial of the finished matrix to the workspace, and the last block to
// finish a matrix (atomic ticket) adds that matrix's partials in block
// order, so the result is deterministic for a given device.
#include "batch.cuh"

namespace tq {

// Bound on the blocks of one launch (one wave of resident blocks at most),
// so the workspace size does not depend on the device.
constexpr int64_t PX_MAX_BLOCKS = 148 * 8;

// Octets per thread: two consecutive octets of one group (one 16-weight
// NVFP4 block; half the per-row code and scale loads of one octet).
// Measured on the MoE and dense workloads: two octets, one row per
// iteration, imatrix weights in shared memory (60-64 registers, 4 blocks of
// up to 256 threads per SM) beat two rows in flight per thread at 3 blocks
// per SM, and beat a private ring of 2-4 rows per thread filled by
// asynchronous 16-byte copies (0.65 against 0.57 ms on the int3 MoE stack).
constexpr int PX_NO = 2;
// Row walkers per block (blockDim.y): they share the block's columns (and
// its imatrix weights in shared memory) and take interleaved rows.
// Measured on the full-size workloads: one block of four walkers per SM
// beat four one-walker blocks (0.550 -> 0.486 ms on the int3 MoE stack,
// 0.027 -> 0.026 ms on the dense q projection, even on the NVFP4 stack).
// At launch the walkers fill a block of up to 1024 threads (tiles narrower
// than 256 columns get more walkers: 5 for the NVFP4 stack's 192-wide tiles,
// 0.378 -> 0.343 ms); PX_PY sets the register bound.
constexpr int PX_PY = 4;
constexpr bool PX_FILL = true;

inline int64_t px_cols(int64_t I) { return ((I + 7) / 8 + PX_NO - 1) / PX_NO; }

// Workspace of a grouped launch: every unit's tickets (one per matrix), all
// together at the front (one memset), then per unit an fp64 (num, den) pair
// per (block row y + matrix e, column tile): the blocks whose rows reach into
// matrix e are a contiguous run of y, and a later y never reaches an earlier
// matrix, so (e + y) never repeats between two (block, matrix) pairs of one
// column tile.  A unit gets at most PX_MAX_BLOCKS / (its column tiles) block
// rows (the launch holds at most PX_MAX_BLOCKS blocks), so its slots are
// sized for that many.
struct PxLayout {
    int64_t ticket_off[BATCH_MAX];   // in tickets
    int64_t part_off[BATCH_MAX];     // in bytes from the workspace start
    int64_t bytes;
};

inline PxLayout px_layout(int n, const tq_mat* W) {
    PxLayout L;
    int64_t cols[BATCH_MAX], rows[BATCH_MAX], width = 32;
    BatchSlot sl[BATCH_MAX];
    for (int i = 0; i < n; ++i) {
        cols[i] = px_cols(W[i].cols);
        rows[i] = W[i].n_mat * W[i].rows;
    }
    batch_split(n, cols, rows, 1, sl, &width);   // the launch's column tiles (they do not depend on the device)
    int64_t t = 0;
    for (int i = 0; i < n; ++i) { L.ticket_off[i] = t; t += W[i].n_mat; }
    int64_t off = ((t * 4 + 15) / 16) * 16;
    for (int i = 0; i < n; ++i) {
        const int64_t cb = sl[i].cblocks;
        int64_t rb = PX_MAX_BLOCKS / cb;
        rb = rb < 1 ? 1 : (rb > rows[i] ? rows[i] : rb);
        L.part_off[i] = off;
        off += (W[i].n_mat + rb) * cb * 16;
    }
    L.bytes = off;
    return L;
}

// One unit of a grouped proxy launch.
struct PxUnit {
    const void* W;
    int64_t O, I, ld, ms, n_rows;
    const uint8_t* packed;
    const void* scales;
    const uint8_t* zeros;
    const float* gs;
    const float* m;
    int64_t m_stride;
    double* part;
    unsigned* tickets;
    double* num;
    double* den;
    BatchSlot s;
};
struct PxArgs {
    int n;
    PxUnit u[BATCH_MAX];
};

// Adds the 8 terms of one octet in fp32 (two interleaved partial sums of
// fp32x2 pairs): m (W - What)^2 and m W^2.
__device__ __forceinline__ void px_terms(const float w[8], const float v[8], const float mm[8], float& sn,
                                         float& sd) {
    float2 an = make_float2(0.f, 0.f), ad = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float2 m2 = make_float2(mm[i], mm[i + 1]);
        const float2 ww = make_float2(w[i], w[i + 1]);
        const float2 d = __fadd2_rn(ww, make_float2(-v[i], -v[i + 1]));
        an = __ffma2_rn(__fmul2_rn(m2, d), d, an);
        ad = __ffma2_rn(__fmul2_rn(m2, ww), ww, ad);
    }
    sn = __fadd_rn(an.x, an.y);
    sd = __fadd_rn(ad.x, ad.y);
}

// The body of both kernels below: column tile x (cw unit columns wide, cb
// tiles) and row block y (rpb rows) of one unit.
template <int FMT, typename T, int NO>
__device__ __forceinline__ void proxy_rows(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms,
                                           int64_t n_rows, const uint8_t* __restrict__ packed, const void* scales,
                                           const uint8_t* __restrict__ zeros, const float* __restrict__ gs,
                                           const float* __restrict__ m, int64_t m_stride, double* __restrict__ part,
                                           unsigned* __restrict__ tickets, double* __restrict__ num,
                                           double* __restrict__ den, int64_t x, int64_t y, int64_t cb, int64_t rpb,
                                           int64_t cw) {
    using F = FmtTraits<FMT>;
    const int64_t G = (I + F::group - 1) / F::group;
    const int64_t C = (I + 7) >> 3;
    const int64_t u = x * cw + threadIdx.x;
    const bool active = threadIdx.x < cw && u < (C + NO - 1) / NO;
    const int nthreads = static_cast<int>(blockDim.x * blockDim.y);
    const int tid = static_cast<int>(threadIdx.y * blockDim.x + threadIdx.x);
    const int nwarps = nthreads >> 5;   // blockDim.x is a multiple of 32
    const int lane = tid & 31, wid = tid >> 5;
    const int64_t py = blockDim.y, ty = threadIdx.y;
    __shared__ float4 msm[2 * NO][256];
    __shared__ double sw[2][32];
    __shared__ bool last;
    const int64_t c = u * NO;
    const int64_t k = c >> F::lg;
    const int oct = static_cast<int>(c & ((1 << F::lg) - 1));
    const int64_t j = c << 3;
    int n[NO];
#pragma unroll
    for (int i = 0; i < NO; ++i)
        n[i] = static_cast<int>(max(static_cast<int64_t>(0), min(static_cast<int64_t>(8), I - j - 8 * i)));
    int64_t r = y * rpb;
    const int64_t r1 = min(n_rows, r + rpb);
    int64_t e = r / O;
    bool first = true;
    while (r < r1) {   // the block's rows of matrix e: [r, seg_end); the same for every thread
        const int64_t seg_end = min(r1, (e + 1) * O);
        if (active && ty == 0 && (first || m_stride != 0)) {
#pragma unroll
            for (int i = 0; i < NO; ++i) {
                Oct<float> mo;
                mo.load(m + e * m_stride + j + 8 * i, n[i]);
                msm[2 * i][threadIdx.x] = mo.a;   // read by the column's walkers
                msm[2 * i + 1][threadIdx.x] = mo.b;
            }
        }
        __syncthreads();
        double an = 0.0, ad = 0.0;
        if (active) {
            const float g = FMT == TQ_NVFP4_G16 ? __ldg(gs + e) : 0.f;
            // this walker's rows: r + ty, r + ty + py, ...
            const T* wp = W + e * ms + (r + ty - e * O) * ld + j;
            QPtr<FMT> qp(packed, scales, zeros, (r + ty) * G + k, G);
            for (int64_t o = r + ty; o < seg_end; o += py, wp += py * ld) {
                Oct<T> rw[NO];
#pragma unroll
                for (int i = 0; i < NO; ++i) rw[i].load(wp + 8 * i, n[i]);
                const UnitQ<NO> q = load_unit_q<FMT, NO>(qp, oct);
                qp.skip(py);
                float sn = 0.f, sd = 0.f;
#pragma unroll
                for (int i = 0; i < NO; ++i) {
                    float w[8], v[8], mm[8], tn, td;
                    rw[i].get(w);
                    dec_oct<FMT>(OctQ{q.bits[i], q.s, q.z}, g, v);
                    const float4 a = msm[2 * i][threadIdx.x], b = msm[2 * i + 1][threadIdx.x];
                    mm[0] = a.x; mm[1] = a.y; mm[2] = a.z; mm[3] = a.w;
                    mm[4] = b.x; mm[5] = b.y; mm[6] = b.z; mm[7] = b.w;
                    px_terms(w, v, mm, tn, td);
                    sn = __fadd_rn(sn, tn);
                    sd = __fadd_rn(sd, td);
                }
                an += static_cast<double>(sn);
                ad += static_cast<double>(sd);
            }
        }
        // the block's partial of matrix e, in fp64, fixed order
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            an += __shfl_xor_sync(FULL, an, off);
            ad += __shfl_xor_sync(FULL, ad, off);
        }
        if (lane == 0) { sw[0][wid] = an; sw[1][wid] = ad; }
        __syncthreads();
        // blocks (all column tiles) whose rows reach into matrix e
        const int64_t ylo = (e * O) / rpb, yhi = ((e + 1) * O - 1) / rpb;
        if (tid == 0) {
            double bn = 0.0, bd = 0.0;
            for (int i = 0; i < nwarps; ++i) { bn += sw[0][i]; bd += sw[1][i]; }
            part[((e + y) * cb + x) * 2] = bn;
            part[((e + y) * cb + x) * 2 + 1] = bd;
            __threadfence();
            last = atomicAdd(tickets + e, 1u) == static_cast<unsigned>((yhi - ylo + 1) * cb - 1);
        }
        __syncthreads();
        if (last) {   // the matrix's last block adds its partials: y ascending, then column tiles
            __threadfence();
            const int64_t np = (yhi - ylo + 1) * cb;
            double tn = 0.0, td = 0.0;
            for (int64_t t = tid; t < np; t += nthreads) {
                const int64_t idx = (e + ylo) * cb + t;   // (e + yy) * cb + x with yy = ylo + t / cb, x = t % cb
                tn += __ldcg(part + idx * 2);
                td += __ldcg(part + idx * 2 + 1);
            }
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                tn += __shfl_xor_sync(FULL, tn, off);
                td += __shfl_xor_sync(FULL, td, off);
            }
            __syncthreads();
            if (lane == 0) { sw[0][wid] = tn; sw[1][wid] = td; }
            __syncthreads();
            if (tid == 0) {
                double bn = 0.0, bd = 0.0;
                for (int i = 0; i < nwarps; ++i) { bn += sw[0][i]; bd += sw[1][i]; }
                num[e] = bn;
                den[e] = bd;
            }
        }
        __syncthreads();   // sw, msm and `last` are reused by the next matrix
        r = seg_end;
        ++e;
        first = false;
    }
}

// One unit: grid x = column tiles, y = row blocks.
template <int FMT, typename T, int NO>
__global__ void __launch_bounds__(256 * PX_PY, 4 / PX_PY)
k_proxy(const T* __restrict__ W, int64_t O, int64_t I, int64_t ld, int64_t ms, int64_t n_rows,
        const uint8_t* __restrict__ packed, const void* scales, const uint8_t* __restrict__ zeros,
        const float* __restrict__ gs, const float* __restrict__ m, int64_t m_stride, int64_t rpb,
        double* __restrict__ part, unsigned* __restrict__ tickets, double* __restrict__ num,
        double* __restrict__ den) {
    proxy_rows<FMT, T, NO>(W, O, I, ld, ms, n_rows, packed, scales, zeros, gs, m, m_stride, part, tickets, num, den,
                           blockIdx.x, blockIdx.y, gridDim.x, rpb, blockDim.x);
}

// Several units: each block looks up its unit's range of the 1-D grid.
template <int FMT, typename T, int NO>
__global__ void __launch_bounds__(256 * PX_PY, 4 / PX_PY)
k_proxy_batch(const __grid_constant__ PxArgs args) {
    const PxUnit& p = args.u[batch_unit(args.u, args.n, blockIdx.x)];
    const int64_t lb = static_cast<int64_t>(blockIdx.x) - p.s.block0;
    proxy_rows<FMT, T, NO>(static_cast<const T*>(p.W), p.O, p.I, p.ld, p.ms, p.n_rows, p.packed, p.scales, p.zeros,
                           p.gs, p.m, p.m_stride, p.part, p.tickets, p.num, p.den, lb % p.s.cblocks,
                           lb / p.s.cblocks, p.s.cblocks, p.s.rpb, p.s.cw);
}

// One wave of resident blocks at most (and at most PX_MAX_BLOCKS, the count
// the workspace is sized for), split over the units by size.
template <int FMT, typename T>
void launch_proxy(int n, const tq_mat* W, const uint8_t* const* packed, const void* const* scales,
                  const uint8_t* const* zeros, const float* const* gs, const float* const* m,
                  const int64_t* m_stride, double* const* num, double* const* den, uint8_t* ws, const PxLayout& L,
                  cudaStream_t st) {
    int64_t cols[BATCH_MAX], rows[BATCH_MAX];
    for (int i = 0; i < n; ++i) {
        cols[i] = px_cols(W[i].cols);
        rows[i] = W[i].n_mat * W[i].rows;
    }
    int64_t width = 32;
    BatchSlot sl[BATCH_MAX];
    batch_split(n, cols, rows, 1, sl, &width);
    // One unit: the direct-argument kernel, except for int3, where the
    // grouped kernel measured faster on one unit too (0.476 against 0.502 ms
    // on the int3 MoE stack; 0.380 against 0.377 ms on the NVFP4 stack).
    const bool direct = n == 1 && FMT != TQ_INT3_G64_SYM;
    auto kern = direct ? reinterpret_cast<const void*>(k_proxy<FMT, T, PX_NO>)
                       : reinterpret_cast<const void*>(k_proxy_batch<FMT, T, PX_NO>);
    int per_sm = 0;
    // as many walkers as fill a block of up to 1024 threads (narrow tiles: more walkers)
    const int py = PX_FILL ? static_cast<int>(min(static_cast<int64_t>(8), 1024 / width)) : PX_PY;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, static_cast<int>(width) * py, 0) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t slots = min(static_cast<int64_t>(num_sms()) * per_sm, PX_MAX_BLOCKS);
    const int64_t blocks = batch_split(n, cols, rows, slots, sl, &width);
    const dim3 block(static_cast<unsigned>(width), static_cast<unsigned>(py));
    if (direct) {
        const dim3 grid(static_cast<unsigned>(sl[0].cblocks), static_cast<unsigned>(sl[0].rblocks));
        k_proxy<FMT, T, PX_NO><<<grid, block, 0, st>>>(
            static_cast<const T*>(W->ptr), W->rows, W->cols, W->ld, W->n_mat > 1 ? W->mat_stride : 0, rows[0],
            packed[0], scales[0], zeros ? zeros[0] : nullptr, gs ? gs[0] : nullptr, m[0],
            W->n_mat > 1 ? m_stride[0] : 0, sl[0].rpb, reinterpret_cast<double*>(ws + L.part_off[0]),
            reinterpret_cast<unsigned*>(ws) + L.ticket_off[0], num[0], den[0]);
        return;
    }
    static thread_local PxArgs a;
    a.n = n;
    for (int i = 0; i < n; ++i) {
        PxUnit& u = a.u[i];
        u.W = W[i].ptr; u.O = W[i].rows; u.I = W[i].cols; u.ld = W[i].ld;
        u.ms = W[i].n_mat > 1 ? W[i].mat_stride : 0;
        u.n_rows = rows[i];
        u.packed = packed[i]; u.scales = scales[i]; u.zeros = zeros ? zeros[i] : nullptr; u.gs = gs ? gs[i] : nullptr;
        u.m = m[i];
        u.m_stride = W[i].n_mat > 1 ? m_stride[i] : 0;
        u.part = reinterpret_cast<double*>(ws + L.part_off[i]);
        u.tickets = reinterpret_cast<unsigned*>(ws) + L.ticket_off[i];
        u.num = num[i]; u.den = den[i];
        u.s = sl[i];
    }
    k_proxy_batch<FMT, T, PX_NO><<<static_cast<unsigned>(blocks), block, 0, st>>>(a);
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_proxy_batch_workspace_bytes(int32_t n, const tq_mat* W, int32_t fmt) {
    if (!W || n < 1 || n > TQ_MAX_BATCH || group_of(fmt) == 0) return 0;
    for (int i = 0; i < n; ++i)
        if (W[i].n_mat < 1 || W[i].rows < 1 || W[i].cols < 1) return 0;
    return static_cast<size_t>(px_layout(n, W).bytes);
}

TQ_API size_t tq_proxy_workspace_bytes(const tq_mat* W, int32_t fmt) {
    return tq_proxy_batch_workspace_bytes(1, W, fmt);
}

static tq_status check_proxy_unit(const tq_mat* W, const uint8_t* packed, int32_t fmt, const void* scales,
                                  const uint8_t* zeros, const float* global_scale, const float* m, int64_t m_stride,
                                  const double* num, const double* den, const char* who) {
    tq_status s = check_mat(W, who);
    if (s != TQ_OK) return s;
    TQ_REQUIRE(packed && scales && m && num && den, "%s: null pointer", who);
    TQ_REQUIRE(aligned16(packed) && aligned16(m), "%s: packed/m not 16-byte aligned", who);
    TQ_REQUIRE(W->n_mat == 1 || m_stride == 0 || (m_stride >= W->cols && m_stride % 4 == 0),
               "%s: m_stride must be 0 or a multiple of 4 >= cols", who);
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "%s: int4 needs zeros", who);
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "%s: NVFP4 needs global_scale", who);
    return TQ_OK;
}

static tq_status run_proxy(int n, const tq_mat* W, const uint8_t* const* packed, int32_t fmt,
                           const void* const* scales, const uint8_t* const* zeros, const float* const* gs,
                           const float* const* m, const int64_t* m_stride, double* const* num, double* const* den,
                           void* workspace, size_t workspace_bytes, cudaStream_t st, const char* who) {
    TQ_REQUIRE(workspace && aligned16(workspace), "%s: workspace null or not 16-byte aligned", who);
    const PxLayout L = px_layout(n, W);
    TQ_REQUIRE(workspace_bytes >= static_cast<size_t>(L.bytes), "%s: workspace too small (%zu < %zu)", who,
               workspace_bytes, static_cast<size_t>(L.bytes));
    int64_t nt = 0;
    for (int i = 0; i < n; ++i) nt += W[i].n_mat;
    cudaError_t ce = cudaMemsetAsync(workspace, 0, static_cast<size_t>(nt) * 4, st);
    if (ce != cudaSuccess) return set_error(TQ_ERR_CUDA, "%s: %s", who, cudaGetErrorString(ce));
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const bool bf = W[0].dtype == TQ_BF16;
#define TQ_PX_ARGS n, W, packed, scales, zeros, gs, m, m_stride, num, den, ws, L, st
    if (fmt == TQ_INT3_G64_SYM)
        bf ? launch_proxy<TQ_INT3_G64_SYM, uint16_t>(TQ_PX_ARGS) : launch_proxy<TQ_INT3_G64_SYM, float>(TQ_PX_ARGS);
    else if (fmt == TQ_INT4_G128_ASYM)
        bf ? launch_proxy<TQ_INT4_G128_ASYM, uint16_t>(TQ_PX_ARGS) : launch_proxy<TQ_INT4_G128_ASYM, float>(TQ_PX_ARGS);
    else if (fmt == TQ_INT4_G64_ASYM)
        bf ? launch_proxy<TQ_INT4_G64_ASYM, uint16_t>(TQ_PX_ARGS) : launch_proxy<TQ_INT4_G64_ASYM, float>(TQ_PX_ARGS);
    else if (fmt == TQ_INT4_G32_ASYM)
        bf ? launch_proxy<TQ_INT4_G32_ASYM, uint16_t>(TQ_PX_ARGS) : launch_proxy<TQ_INT4_G32_ASYM, float>(TQ_PX_ARGS);
    else
        bf ? launch_proxy<TQ_NVFP4_G16, uint16_t>(TQ_PX_ARGS) : launch_proxy<TQ_NVFP4_G16, float>(TQ_PX_ARGS);
#undef TQ_PX_ARGS
    return check_launch(who);
}

TQ_API tq_status tq_proxy_error(const tq_mat* W, const uint8_t* packed, int32_t fmt, const void* scales,
                                const uint8_t* zeros, const float* global_scale, const float* m,
                                int64_t m_stride, double* num, double* den, void* workspace,
                                size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_proxy_error: unknown format %d", fmt);
    tq_status s = check_proxy_unit(W, packed, fmt, scales, zeros, global_scale, m, m_stride, num, den,
                                   "tq_proxy_error");
    if (s != TQ_OK) return s;
    return run_proxy(1, W, &packed, fmt, &scales, &zeros, &global_scale, &m, &m_stride, &num, &den, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream), "tq_proxy_error");
}

TQ_API tq_status tq_proxy_error_batch(int32_t n, const tq_mat* W, const uint8_t* const* packed, int32_t fmt,
                                      const void* const* scales, const uint8_t* const* zeros,
                                      const float* const* global_scale, const float* const* m,
                                      const int64_t* m_stride, double* const* num, double* const* den,
                                      void* workspace, size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_proxy_error_batch: unknown format %d", fmt);
    TQ_REQUIRE(n >= 1 && n <= TQ_MAX_BATCH, "tq_proxy_error_batch: n = %d outside [1, %d]", n, TQ_MAX_BATCH);
    TQ_REQUIRE(W && packed && scales && m && m_stride && num && den, "tq_proxy_error_batch: null array");
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "tq_proxy_error_batch: int4 needs zeros");
    TQ_REQUIRE(fmt != TQ_NVFP4_G16 || global_scale != nullptr, "tq_proxy_error_batch: NVFP4 needs global_scale");
    for (int i = 0; i < n; ++i) {
        tq_status s = check_proxy_unit(&W[i], packed[i], fmt, scales[i], zeros ? zeros[i] : nullptr,
                                       global_scale ? global_scale[i] : nullptr, m[i], m_stride[i], num[i], den[i],
                                       "tq_proxy_error_batch");
        if (s != TQ_OK) return s;
        TQ_REQUIRE(W[i].dtype == W[0].dtype, "tq_proxy_error_batch: units of different dtypes");
    }
    return run_proxy(n, W, packed, fmt, scales, zeros, global_scale, m, m_stride, num, den, workspace,
                     workspace_bytes, reinterpret_cast<cudaStream_t>(stream), "tq_proxy_error_batch");
}
