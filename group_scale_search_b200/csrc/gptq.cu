// GPTQ/LDLQ column sweep ("Quantize on TT cards: CUDA-free GPTQ/LDLQ bfp4
// pipeline", tt-stack issue #67, pipeline table step 3: columns are rounded
// one at a time within 128-wide blocks, and each block's rounding errors E
// reach the columns after it through W[:, rest] -= E U[blk, rest], U the
// inverse Hessian's triangular factor), with the group scales and
// zero-points the search chose.
//
// Per row, column i in order: the code of the current w_i under its group's
// parameters (the format's round-to-nearest on the IEEE fp32 quotient), its
// dequantized value What_i, e_i = (w_i - What_i) / U_ii, and
// w_j <- w_j - e_i U_ij for every later column j, one fp32 fused
// multiply-add each (fp32 is the page's host propagator).  Every weight
// receives its updates in column order, whichever block they come from, so
// the result is bitwise that of the unblocked sweep and does not depend on
// the tiling below.
//
// B200 mapping: rows are independent given U, so a CTA takes 16 rows of one
// matrix and carries them through every 128-column block:
//  * serial part: the block's 128 x 128 triangle of U sits in shared memory;
//    a warp keeps 2 rows' 128 block weights in registers (4 per lane); the
//    owner lane's w_i is broadcast by a shuffle and every lane rounds it (the
//    same arithmetic, so no second broadcast), then updates its later
//    columns; lane 0 records the code and e_i.
//  * propagation (nearly all the flops): each thread owns later columns j
//    and keeps the 16 rows' w_j in registers; for i = 0..127 in order it
//    loads U_ij once (coalesced, from L2; the next four in flight) and applies
//    16 FMAs, e_i read as float4 broadcasts from shared memory.
// The rows' fp32 working copy lives in the workspace: one read and one write
// of the remaining columns per block.
#include "walk.cuh"

namespace tq {

constexpr int GQ_B = 128;                         // block width (columns)
constexpr int GQ_R = 16;                          // rows per CTA
constexpr int GQ_THREADS = 256;
constexpr int GQ_RPW = GQ_R / (GQ_THREADS / 32);  // rows per warp in the serial part
constexpr int GQ_SMEM_BYTES = (GQ_B * GQ_B + GQ_R * GQ_B) * 4;
static_assert(GQ_RPW * (GQ_THREADS / 32) == GQ_R, "rows split evenly over the warps");
static_assert(GQ_B % 8 == 0, "the propagation takes the block in steps of 8 columns");

struct GqArgs {
    const void* W;           // [n_mat][O][I] rows of ld, matrices ms apart (bf16 or fp32)
    int64_t O, I, ld, ms;
    const float* scales;     // [n_mat][O][G]
    const uint8_t* zeros;    // [n_mat][O][G] (int4)
    const float* U;          // [n_mat or 1][I][ldu], ums apart
    int64_t ldu, ums;
    float* wk;               // [n_mat][O][I] fp32 working copy
    int8_t* codes;           // [n_mat][O][I]
    double* loss;            // [n_mat][O] or null
};

__device__ __forceinline__ float gq_load(const uint16_t* p) { return bf16_bits_to_f32(*p); }
__device__ __forceinline__ float gq_load(const float* p) { return *p; }

// Round-to-nearest of w under a fixed scale: rint of the IEEE quotient w / s,
// clamped to the code range; a zero scale gives code 0 (int3) or z (int4).
// Returns the dequantized value fl32(s v) or fl32(s (q - z)).
template <int FMT>
__device__ __forceinline__ float gq_round(float w, float s, int z, int& code) {
    if constexpr (FMT == TQ_INT3_G64_SYM) {
        float v = 0.f;
        if (s != 0.f) v = fminf(fmaxf(rintf(__fdiv_rn(w, s)), -4.f), 3.f);
        code = static_cast<int>(v);
        return __fmul_rn(s, v);
    } else {
        const float zf = static_cast<float>(z);
        float q = zf;
        if (s != 0.f) q = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(w, s)), zf), 0.f), 15.f);
        code = static_cast<int>(q);
        return __fmul_rn(s, __fsub_rn(q, zf));
    }
}

// Four consecutive columns i..i+3 of the block applied to the GQ_R rows'
// accumulators in column order: acc_r <- fma(-e_{r,i}, U_ij, acc_r).
__device__ __forceinline__ void gq_step(float (&acc)[GQ_R], const float* Eb_i, const float (&u)[4]) {
#pragma unroll
    for (int r = 0; r < GQ_R; ++r) {
        const float4 ev = *reinterpret_cast<const float4*>(Eb_i + r * GQ_B);
        acc[r] = __fmaf_rn(-ev.x, u[0], acc[r]);
        acc[r] = __fmaf_rn(-ev.y, u[1], acc[r]);
        acc[r] = __fmaf_rn(-ev.z, u[2], acc[r]);
        acc[r] = __fmaf_rn(-ev.w, u[3], acc[r]);
    }
}

template <int FMT, typename T>
__global__ void __launch_bounds__(GQ_THREADS, 2) k_gptq(const GqArgs a) {
    using F = FmtTraits<FMT>;
    extern __shared__ float4 gq_smem4[];
    float* Ut = reinterpret_cast<float*>(gq_smem4);   // [GQ_B][GQ_B]: the block's triangle of U
    float* Eb = Ut + GQ_B * GQ_B;                      // [GQ_R][GQ_B]: the block's e_i per row
    const int64_t e = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * GQ_R;
    const int nr = static_cast<int>(min(static_cast<int64_t>(GQ_R), a.O - r0));
    const int64_t I = a.I, G = (I + F::group - 1) / F::group;
    const int64_t grow0 = e * a.O + r0;               // global row index of the CTA's first row
    const float* U = a.U + e * a.ums;
    float* wk = a.wk + grow0 * I;
    const T* W = static_cast<const T*>(a.W) + e * a.ms + r0 * a.ld;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int r = 0; r < nr; ++r)
        for (int64_t j = tid; j < I; j += GQ_THREADS) wk[r * I + j] = gq_load(W + r * a.ld + j);

    double lossr[GQ_RPW];
#pragma unroll
    for (int k = 0; k < GQ_RPW; ++k) lossr[k] = 0.0;

    for (int64_t b0 = 0; b0 < I; b0 += GQ_B) {
        const int nb = static_cast<int>(min(static_cast<int64_t>(GQ_B), I - b0));
        for (int idx = tid; idx < GQ_B * GQ_B; idx += GQ_THREADS) {
            const int i = idx / GQ_B, j = idx % GQ_B;
            Ut[idx] = (i < nb && j < nb && j >= i) ? __ldg(U + (b0 + i) * a.ldu + b0 + j) : 0.f;
        }
        __syncthreads();   // the tile, and the working copy written before this block

        // ---- serial part: the block's columns in order
        float w[GQ_RPW][4];
#pragma unroll
        for (int k = 0; k < GQ_RPW; ++k) {
            const int row = warp * GQ_RPW + k;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int j = lane + 32 * t;
                w[k][t] = (row < nr && j < nb) ? wk[row * I + b0 + j] : 0.f;
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
#pragma unroll 1
            for (int il = 0; il < 32; ++il) {
                const int i = 32 * t + il;
                if (i >= nb) break;
                const float uii = Ut[i * GQ_B + i];
                const int64_t col = b0 + i;
#pragma unroll
                for (int k = 0; k < GQ_RPW; ++k) {
                    const int row = warp * GQ_RPW + k;
                    const float wi = __shfl_sync(FULL, w[k][t], il);
                    float s = 0.f;
                    int z = 0;
                    if (row < nr) {
                        const int64_t gi = (grow0 + row) * G + col / F::group;
                        s = __ldg(a.scales + gi);
                        if constexpr (is_int4(FMT)) z = __ldg(a.zeros + gi);
                    }
                    int code;
                    const float what = gq_round<FMT>(wi, s, z, code);
                    const float ei = __fdiv_rn(__fsub_rn(wi, what), uii);
                    lossr[k] += static_cast<double>(ei) * static_cast<double>(ei);
                    if (lane == 0 && row < nr) {
                        a.codes[(grow0 + row) * I + col] = static_cast<int8_t>(code);
                        Eb[row * GQ_B + i] = ei;
                    }
#pragma unroll
                    for (int t2 = t; t2 < 4; ++t2) {
                        const int j = lane + 32 * t2;
                        if (j > i) w[k][t2] = __fmaf_rn(-ei, Ut[i * GQ_B + j], w[k][t2]);
                    }
                }
            }
        }
        __syncthreads();   // every row's e_i of the block

        // ---- propagation to the later columns (a later column exists only when the block is full)
        for (int64_t j = b0 + GQ_B + tid; j < I; j += GQ_THREADS) {
            // two sets of four U_ij: one set is in flight (L2 latency) while the other is used
            const float* up = U + b0 * a.ldu + j;
            float ua[4], ub[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                ua[q] = __ldg(up + q * a.ldu);
                ub[q] = __ldg(up + (4 + q) * a.ldu);
            }
            float acc[GQ_R];
#pragma unroll
            for (int r = 0; r < GQ_R; ++r) acc[r] = r < nr ? wk[r * I + j] : 0.f;
#pragma unroll 1
            for (int i = 0; i < GQ_B; i += 8) {
                gq_step(acc, Eb + i, ua);
                if (i + 8 < GQ_B) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) ua[q] = __ldg(up + (i + 8 + q) * a.ldu);
                }
                gq_step(acc, Eb + i + 4, ub);
                if (i + 12 < GQ_B) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) ub[q] = __ldg(up + (i + 12 + q) * a.ldu);
                }
            }
#pragma unroll
            for (int r = 0; r < GQ_R; ++r)
                if (r < nr) wk[r * I + j] = acc[r];
        }
        __syncthreads();   // before the next block reads the working copy and reuses the tiles
    }
    if (a.loss && lane == 0) {
#pragma unroll
        for (int k = 0; k < GQ_RPW; ++k) {
            const int row = warp * GQ_RPW + k;
            if (row < nr) a.loss[grow0 + row] = lossr[k];
        }
    }
}

template <int FMT, typename T>
static void launch_gptq(const GqArgs& a, int64_t n_mat, cudaStream_t st) {
    static bool attr = [] {
        return cudaFuncSetAttribute(k_gptq<FMT, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, GQ_SMEM_BYTES) ==
               cudaSuccess;
    }();
    (void)attr;
    const dim3 grid(static_cast<unsigned>((a.O + GQ_R - 1) / GQ_R), static_cast<unsigned>(n_mat));
    k_gptq<FMT, T><<<grid, GQ_THREADS, GQ_SMEM_BYTES, st>>>(a);
}

}  // namespace tq

using namespace tq;

TQ_API size_t tq_gptq_workspace_bytes(const tq_mat* W) {
    if (!W || W->n_mat < 1 || W->rows < 1 || W->cols < 1) return 0;
    return static_cast<size_t>(W->n_mat * W->rows * W->cols * 4);
}

TQ_API tq_status tq_gptq_sweep(const tq_mat* W, int32_t fmt, const void* scales, const uint8_t* zeros,
                               const float* U, int64_t ldu, int64_t u_mat_stride, int8_t* codes, double* loss,
                               void* workspace, size_t workspace_bytes, tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_gptq_sweep W");
    if (s != TQ_OK) return s;
    if (fmt != TQ_INT3_G64_SYM && !is_int4(fmt))
        return set_error(TQ_ERR_UNSUPPORTED, "tq_gptq_sweep: format %d (int3-g64 and int4 only)", fmt);
    TQ_REQUIRE(scales && U && codes && workspace, "tq_gptq_sweep: null pointer");
    TQ_REQUIRE(!is_int4(fmt) || zeros != nullptr, "tq_gptq_sweep: int4 needs zeros");
    TQ_REQUIRE(ldu >= W->cols, "tq_gptq_sweep: ldu (%lld) < I", (long long)ldu);
    TQ_REQUIRE(u_mat_stride == 0 || u_mat_stride >= W->cols * ldu, "tq_gptq_sweep: u_mat_stride < I * ldu");
    TQ_REQUIRE(aligned16(workspace) && (reinterpret_cast<uintptr_t>(U) & 3u) == 0,
               "tq_gptq_sweep: workspace not 16-byte aligned or U not 4-byte aligned");
    TQ_REQUIRE(W->n_mat <= 65535 && W->rows < (int64_t(1) << 31) && W->cols < (int64_t(1) << 31),
               "tq_gptq_sweep: sizes out of range");
    TQ_REQUIRE(workspace_bytes >= tq_gptq_workspace_bytes(W), "tq_gptq_sweep: workspace too small");
    GqArgs a;
    a.W = W->ptr;
    a.O = W->rows;
    a.I = W->cols;
    a.ld = W->ld;
    a.ms = W->n_mat > 1 ? W->mat_stride : 0;
    a.scales = static_cast<const float*>(scales);
    a.zeros = zeros;
    a.U = U;
    a.ldu = ldu;
    a.ums = u_mat_stride;
    a.wk = static_cast<float*>(workspace);
    a.codes = codes;
    a.loss = loss;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = W->dtype == TQ_BF16;
    if (fmt == TQ_INT3_G64_SYM)
        bf ? launch_gptq<TQ_INT3_G64_SYM, uint16_t>(a, W->n_mat, st) : launch_gptq<TQ_INT3_G64_SYM, float>(a, W->n_mat, st);
    else if (fmt == TQ_INT4_G128_ASYM)
        bf ? launch_gptq<TQ_INT4_G128_ASYM, uint16_t>(a, W->n_mat, st) : launch_gptq<TQ_INT4_G128_ASYM, float>(a, W->n_mat, st);
    else if (fmt == TQ_INT4_G64_ASYM)
        bf ? launch_gptq<TQ_INT4_G64_ASYM, uint16_t>(a, W->n_mat, st) : launch_gptq<TQ_INT4_G64_ASYM, float>(a, W->n_mat, st);
    else
        bf ? launch_gptq<TQ_INT4_G32_ASYM, uint16_t>(a, W->n_mat, st) : launch_gptq<TQ_INT4_G32_ASYM, float>(a, W->n_mat, st);
    return check_launch("tq_gptq_sweep");
}
