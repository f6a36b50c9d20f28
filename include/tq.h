/*
 * tq.h -- C ABI of the group-scale search library: imatrix-weighted search of
 * per-group quantization scales (and integer zero-points), round-to-nearest,
 * packing into int3-g64 / int4-g128 / NVFP4-g16, dequantization and the
 * imatrix-weighted reconstruction error.  Every call runs hand-written CUDA
 * kernels for NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *  [NeUQI]  "NeUQI Accuracy Validation" (intel/auto-round docs/neuqi_acc.md):
 *           opening paragraph (asymmetric layers: joint (scale, integer
 *           zero-point) search; symmetric layers: two-stage signed-scale search;
 *           both weighted by the activation imatrix) and results bullet 2
 *           ("64/32" grid).
 *  [TT]     "Quantize on TT cards: CUDA-free GPTQ/LDLQ bfp4 pipeline" (tt-stack
 *           issue #67): pipeline table step 1 (H = sum X^T X) and "Risks to
 *           measure: Precision" (proxy error tr(E H E^T) / tr(W H W^T)).
 *  [NVFP4]  "Nemotron-Cascade-2-30B-A3B-NVFP4" model card: Quantization Recipe
 *           table (NVFP4, group size 16, MSE-calibrated static block scales).
 *  [INT3]   "int3-g64 (fmt=5)" (colibri PR #168): Design, Layout bullet.
 *  [G32]    "Phase 2: math-accuracy regression on tq3a-tq2e g32"
 *           (turboquant-mlx issue #2): Summary (group_size=32).
 *
 * Conventions shared by every call
 *  - Memory: every tensor pointer is a DEVICE pointer owned by the caller.
 *    The library never allocates device memory; calls that need scratch take
 *    a caller-provided workspace sized by the matching *_workspace_bytes().
 *  - Streams: every call enqueues work on `stream` (NULL = legacy default
 *    stream) and returns without synchronising.  Errors raised by kernels
 *    after launch surface at the caller's next synchronisation.
 *  - Errors: arguments are validated on the host before anything is
 *    enqueued; a call that returns an error has enqueued nothing (except
 *    TQ_ERR_CUDA, raised when a launch itself fails).  tq_last_error_string()
 *    describes the last error of the calling thread.
 *  - Layout: weights W are batches of n_mat row-major O x I matrices; groups
 *    run along I (the input dimension), G = ceil(I / g) groups per row.  A
 *    last group shorter than g is a tail group: only its real elements enter
 *    maxima and losses, and its packed record is padded (see tq_pack_codes).
 *    Per-group outputs (scales, zero-points, indices, losses) are dense
 *    [n_mat][O][G]; packed records are dense in the same order.
 *  - Alignment: tensor base pointers must be 16-byte aligned and row strides
 *    (ld * element size) multiples of 16 bytes.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* tq_stream_t;

typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad sizes or strides */
    TQ_ERR_UNSUPPORTED = 2,  /* a dtype/format/grid this build does not run   */
    TQ_ERR_CUDA = 3          /* a kernel launch or CUDA runtime call failed   */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* Most units one grouped call (tq_pack_batch, tq_dequant_batch,
 * tq_proxy_error_batch) takes. */
#define TQ_MAX_BATCH 16

typedef enum {
    TQ_INT4_G128_ASYM = 4,   /* nibble codes q in [0,15], f32 scale, u8 zero per 128 weights */
    TQ_INT3_G64_SYM = 5,     /* two bit-planes, v in [-4,3] as v+4, f32 scale per 64 weights  */
    TQ_INT4_G64_ASYM = 6,    /* as TQ_INT4_G128_ASYM with 64 weights per group (32-byte records) */
    TQ_INT4_G32_ASYM = 7,    /* as TQ_INT4_G128_ASYM with 32 weights per group (16-byte records) [G32] */
    TQ_NVFP4_G16 = 16        /* E2M1 codes, E4M3 scale byte per 16 weights, f32 global scale   */
} tq_format;

/* A batch of n_mat matrices of rows x cols elements of `dtype`.
 * Element (e, o, j) lives at ptr + (e * mat_stride + o * ld + j) elements. */
typedef struct tq_mat {
    const void* ptr;
    int32_t dtype;       /* tq_dtype */
    int32_t reserved;
    int64_t n_mat;
    int64_t rows;        /* O (or T tokens for activations) */
    int64_t cols;        /* I */
    int64_t ld;          /* >= cols */
    int64_t mat_stride;  /* >= rows * ld, or 0 when n_mat == 1 */
} tq_mat;

/* Candidate grids ([NeUQI]; readings of the unspecified parts in brackets).
 *  Symmetric int3: stage 1 = sym_n1 magnitude ratios r_k = fl32(lo + ((hi-lo)k)/(n1-1))
 *    of max|w|/4, each with both signs: candidate 2k+sigma has scale
 *    (1-2 sigma) fl32(r_k max|w|) / 4.  Stage 2 = sym_n2 ratios spread evenly over
 *    [r_k* - d, r_k* + d], d = (hi-lo)/(n1-1), with the stage-1 winner's sign,
 *    candidate index 2 n1 + i [reading: "refinements around the best"].
 *  Asymmetric int4: scale s_k = fl32(fl32(f_k / 15) (wmax - wmin)),
 *    f_k = lo + ((hi-lo)k)/(ns-1) [reading: range equal to the symmetric window];
 *    zero-point z_i = rint(15 i / (nz - 1)) [reading of "32 integer zero-points
 *    in [0,15]"]; candidate index nz k + i.
 *  NVFP4: the fp4_window E4M3 codes nearest a/(6 g) (a = block max|w|,
 *    g = global scale); candidate index = the E4M3 code. */
typedef struct tq_search_params {
    int32_t sym_n1;        /* 32 */
    int32_t sym_n2;        /* 32 */
    double  sym_lo;        /* 0.5 */
    double  sym_hi;        /* 1.2 */
    int32_t asym_n_scale;  /* 64 */
    int32_t asym_n_zero;   /* 32 */
    double  asym_lo;       /* 0.5 */
    double  asym_hi;       /* 1.2 */
    int32_t fp4_window;    /* 16 */
    int32_t reserved;
} tq_search_params;

/* Fills the defaults above. */
void tq_default_params(tq_search_params* p);

/* Message of the calling thread's last error ("" if none). Never NULL. */
const char* tq_last_error_string(void);

/* Library version string, e.g. "tq 1.0 sm_100a". */
const char* tq_version(void);

/* Weights per group: 64, 128 or 16; 0 for an unknown format. */
int64_t tq_group_size(int32_t fmt);

/* Groups (= scales) of `rows` rows of `cols` weights: rows * ceil(cols / g). */
int64_t tq_num_groups(int32_t fmt, int64_t rows, int64_t cols);

/* Packed code bytes of `rows` rows of `cols` weights: int3 rows*G*24 ([INT3]
 * Layout: 3.5 bits/weight with the f32 scale), int4 rows*G*64, NVFP4 rows*G*8.
 * 0 for an unknown format. */
size_t tq_packed_bytes(int32_t fmt, int64_t rows, int64_t cols);

/* ------------------------------------------------------------------ imatrix
 * m[e*m_stride + j] = alpha * sum_t X[e, t, j]^2 (+ m[...] if accumulate).
 * With alpha = 1/T this is the activation imatrix of [NeUQI], the diagonal of
 * H = sum X^T X over T ([TT] step 1).  X: bf16 or f32, [n_mat, T, I].
 * m: f32 device array, m_stride >= I.  Sums are fp32 over short token runs
 * folded into fp64, reduced across blocks in a fixed order (deterministic).
 * workspace: device scratch of at least tq_imatrix_workspace_bytes() bytes
 * (no alignment beyond 16 bytes; contents need no initialisation).
 * accumulate != 0 adds to the existing m (token-sharded calibration). */
size_t tq_imatrix_workspace_bytes(const tq_mat* X);
tq_status tq_imatrix(const tq_mat* X, float* m, int64_t m_stride, float alpha, int32_t accumulate,
                     void* workspace, size_t workspace_bytes, tq_stream_t stream);

/* ------------------------------------------------------------------ imatrix without allocation
 * No counterpart in the source pages: this is a packaging variant of
 * tq_imatrix for callers that cannot allocate device memory on the path that
 * calls it -- for example code running inside another engine's enqueue hook
 * that is handed only its input and output buffers, or a process whose
 * device memory is fully pre-planned by an arena that does not grant
 * scratch.  Same arguments and results as tq_imatrix, but the scratch is a
 * fixed tq_imatrix_static_capacity() bytes (4 MiB) of device memory inside
 * the library, held by every GPU that loads it until the process exits.
 *  - Shapes whose tq_imatrix_workspace_bytes() exceed the capacity are
 *    rejected with TQ_ERR_INVALID_ARG (use tq_imatrix with a workspace).
 *  - The first call on each device looks up the scratch address on that
 *    device (it must be the current device); make that first call before
 *    any stream capture.
 *  - All calls share the one scratch array: calls whose kernels may overlap
 *    on the GPU (other streams, other host threads) race and give wrong
 *    results; serialise them.  Nothing in the scratch needs to start at
 *    zero, so the previous call's leftovers are harmless.
 *  - Calls no allocating routine (no cudaMalloc/cudaFree). */
size_t tq_imatrix_static_capacity(void);
tq_status tq_imatrix_static(const tq_mat* X, float* m, int64_t m_stride, float alpha, int32_t accumulate,
                            tq_stream_t stream);

/* ------------------------------------------------------------------ amax
 * amax[e] = max |W[e]| over matrix e (f32).  Used for the NVFP4 per-tensor
 * global scale g = fl32(amax / (6 * 448)). */
tq_status tq_amax(const tq_mat* W, float* amax, tq_stream_t stream);

/* ------------------------------------------------------------------ search
 * For every group (block) of every row of every matrix: pick the candidate of
 * the format's grid (tq_search_params) with the smallest imatrix-weighted
 * squared error L = sum_j m_j (w_j - what_j)^2, where the codes of each
 * candidate are round-to-nearest (half to even) of the fp32 quotient w/s,
 * clamped to the format's range ([NeUQI] opening paragraph; [NVFP4] recipe
 * table for the E2M1 / E4M3 search).  Ties keep the lowest candidate index.
 * Candidates are ranked in fp32 on the group's weights and imatrix scaled by
 * exact powers of two (so magnitudes never under- or overflow); candidates
 * within a relative 2^-15 of the best are re-ranked in fp64 with codes from
 * the IEEE quotient, which reproduces the definition's choice.
 *
 *  W:      bf16/f32 weights.  m: f32 imatrix of matrix e at m + e * m_stride
 *          (m_stride = 0: one imatrix for every matrix), >= cols entries.
 *  fmt:    tq_format.  params: NULL = tq_default_params.
 *  scales: int3/int4: f32 [n_mat][O][G] (int3 scales carry the sign);
 *          NVFP4: u8 E4M3 codes [n_mat][O][G].  Required.
 *  zeros:  int4: u8 [n_mat][O][G], required; others must be NULL.
 *  global_scale: NVFP4: f32 [n_mat], written with g = fl32(amax / 2688)
 *          (computed by this call); others must be NULL.
 *  cand_idx: optional int32 [n_mat][O][G]: chosen candidate index (int3:
 *          2k+sigma or 2 n1 + i; int4: nz k + i; NVFP4: the E4M3 code), -1 for
 *          a group with nothing to fit (all zero).
 *  loss:   optional f64 [n_mat][O][G]: the chosen candidate's loss (from the
 *          fp32 ranking, or its fp64 value when a near tie was re-ranked).
 *  packed: optional u8 [n_mat * O * G * record bytes]: the chosen codes packed
 *          as tq_pack would (round-to-nearest and packing fused into the
 *          search).
 * Grid limits of this build: sym_n1, sym_n2 in [2, 32]; asym_n_scale in
 * [2, 256] (more than 64 scales run in passes of 64: the "256/64" end of
 * [NeUQI]'s ladder, results bullet 2), asym_n_zero in [16, 64] (every
 * integer zero-point 0..15 occurs);
 * fp4_window in [1, 16].  Others return TQ_ERR_UNSUPPORTED. */
tq_status tq_search_groups(const tq_mat* W, const float* m, int64_t m_stride, int32_t fmt,
                           const tq_search_params* params, void* scales, uint8_t* zeros,
                           float* global_scale, int32_t* cand_idx, double* loss, uint8_t* packed,
                           tq_stream_t stream);

/* ------------------------------------------------------------------ pack
 * Round-to-nearest of W with the given scales (and zero-points / global
 * scale) and pack: bit-identical to the packed output of tq_search_groups for
 * the same scales.  Arguments as tq_search_groups; global_scale is an INPUT
 * here (f32 [n_mat]). */
tq_status tq_pack(const tq_mat* W, int32_t fmt, const void* scales, const uint8_t* zeros,
                  const float* global_scale, uint8_t* packed, tq_stream_t stream);

/* tq_pack of n units in one launch (1 <= n <= TQ_MAX_BATCH; one format and
 * one weight dtype; shapes free): unit i is W[i] with scales[i], zeros[i],
 * global_scale[i], packed[i] as tq_pack takes them.  W and the pointer arrays
 * are host arrays of n entries (zeros may be NULL when fmt is not int4,
 * global_scale when it is not NVFP4).  The units share one wave of resident
 * blocks, split by their sizes, so small matrices do not each pay a launch's
 * ramp-up and tail.  Results are those of n tq_pack calls.  Errors as tq_pack,
 * TQ_ERR_INVALID_ARG for n out of range or mixed dtypes. */
tq_status tq_pack_batch(int32_t n, const tq_mat* W, int32_t fmt, const void* const* scales,
                        const uint8_t* const* zeros, const float* const* global_scale,
                        uint8_t* const* packed, tq_stream_t stream);

/* Pack integer codes: `codes` is dense [rows][cols] bytes (int3: int8 v in
 * [-4,3]; int4: q in [0,15]; NVFP4: 4-bit E2M1 code, sign in bit 3).
 * Records ([INT3] Layout): int3 = 24 bytes per 64 weights, u = v + 4, low
 * plane bytes 0..15 with element i at byte i/4 bits 2(i%4), high plane bytes
 * 16..23 with element i at bit i%8 of byte 16 + i/8.  int4 / NVFP4 = one byte
 * per two weights, element 2k in the low nibble of byte k.  Tail positions:
 * int3 v = 0, int4 q = zeros[group] (dequantizes to 0; zeros may be NULL for
 * q = 0), NVFP4 code 0.  Codes outside the format's range are masked to its
 * bit width. */
tq_status tq_pack_codes(const uint8_t* codes, int32_t fmt, int64_t rows, int64_t cols,
                        const uint8_t* zeros, uint8_t* packed, tq_stream_t stream);

/* Inverse of tq_pack_codes for the real (non-tail) positions. */
tq_status tq_unpack_codes(const uint8_t* packed, int32_t fmt, int64_t rows, int64_t cols,
                          uint8_t* codes, tq_stream_t stream);

/* ------------------------------------------------------------------ dequant
 * What = s v (int3), s (q - z) (int4), fl32(fl32(g dec(e)) dec(c)) (NVFP4),
 * each rounded once to fp32 (then to bf16, round-to-nearest-even, when
 * out_dtype is TQ_BF16).  out: dense [n_mat][O][I] of out_dtype. */
tq_status tq_dequant(const uint8_t* packed, int32_t fmt, const void* scales, const uint8_t* zeros,
                     const float* global_scale, int64_t n_mat, int64_t O, int64_t I, void* out,
                     int32_t out_dtype, tq_stream_t stream);

/* tq_dequant of n units in one launch (1 <= n <= TQ_MAX_BATCH; one format
 * and one out_dtype): unit i is packed[i], scales[i], zeros[i],
 * global_scale[i], n_mat[i] x O[i] x I[i], out[i].  All arguments but fmt,
 * out_dtype and stream are host arrays of n entries (zeros / global_scale
 * may be NULL as in tq_pack_batch).  Results are those of n tq_dequant calls;
 * errors as tq_dequant. */
tq_status tq_dequant_batch(int32_t n, const uint8_t* const* packed, int32_t fmt, const void* const* scales,
                           const uint8_t* const* zeros, const float* const* global_scale,
                           const int64_t* n_mat, const int64_t* O, const int64_t* I, void* const* out,
                           int32_t out_dtype, tq_stream_t stream);

/* ------------------------------------------------------------------ dequant-GEMV
 * The decode-time consumer of the packed formats ([INT3] Design: Kernel
 * bullet, exact-fp32 product with the scale applied per group; GPU bullet;
 * the step after packing): for b < B,
 *   y[e][b][o] = sum_j What[e][o][j] * x[e][b][j],
 * What the dequantized weights as tq_dequant defines them.  Computed as
 * sum over groups (NVFP4: blocks) of s * sum_j d_j x_j in fp32 (d = v,
 * q - z or dec(c); s = the group scale or fl32(g dec(e))), in an order fixed
 * by the shape alone.  bf16 x with B >= 2, I and x_mat_stride multiples of 8:
 * each group's sum on the tensor cores (bf16 MMA, every product d_j x_j
 * exact, fp32 accumulation per group), scaled once per group in group order
 * by each of 4 warps (groups w, w + 4, ...), the warps' sums added in order;
 * |y - sum What x| <= (g/4 + ceil(G/4) + 4) u sum |What x| (g = group size,
 * G = groups per row, u = 2^-24).  Otherwise on the CUDA cores: for each
 * column tile (the columns whose x fits the kernel's shared memory at once),
 * per lane over its 32-weight quads, a butterfly over 32 lanes, then (rows
 * split over up to 8 warps) the warps' sums in order; the tiles' sums are
 * added in tile order; |y - sum What x| <= (4 ceil(I/1024) + 30) u
 * sum |What x|.  Both deterministic, plus underflow.
 * packed / scales / zeros / global_scale: as tq_dequant; packed 16-byte
 * aligned.  x: x_dtype (TQ_F32 / TQ_BF16) dense [n_mat][B][I] with
 * x_mat_stride elements between matrices (0: one x shared by all
 * matrices), 16-byte aligned.  y: fp32 dense [n_mat][B][O], written once
 * per element.  B in [1, 8] (larger batches are a GEMM, not this call).
 * Errors: TQ_ERR_INVALID for null pointers, empty shapes, B outside [1, 8],
 * 0 < x_mat_stride < B*I, misaligned packed/x, int4 without zeros or NVFP4
 * without global_scale; TQ_ERR_UNSUPPORTED for an unknown fmt or x_dtype;
 * nothing is enqueued then. */
tq_status tq_dequant_gemv(const uint8_t* packed, int32_t fmt, const void* scales, const uint8_t* zeros,
                          const float* global_scale, int64_t n_mat, int64_t O, int64_t I, const void* x,
                          int32_t x_dtype, int64_t B, int64_t x_mat_stride, float* y, tq_stream_t stream);

/* ------------------------------------------------------------------ NVFP4 W4A4 product
 * [NVFP4] Quantization Recipe table (routed experts W4A4, group size 16) and
 * Serving Instructions (FP4 MoE GEMM on Blackwell): y = x W^T with both
 * operands NVFP4, on the block-scaled tensor cores.
 *
 * tq_quant_nvfp4_act: activations X (bf16 or fp32 tq_mat, n_mat matrices of
 * T tokens x I) to NVFP4 with the weights' recipe minus the search: per
 * matrix g = fl32(amax / 2688) (global_scale[n_mat], fp32); per 16-element
 * block the positive finite E4M3 code nearest b / (6 g), b the block amax,
 * by the exact distance |6 g dec(c) - b| with ties to the lower code (0 for
 * an all-zero block or g = 0); elements E2M1 round-to-nearest-even of the
 * IEEE quotient x / fl32(g dec(code)), saturating, sign in bit 3, zero +0.
 * packed: NVFP4 records as tq_pack writes them (8 bytes per block, element
 * 2k in the low nibble of byte k), dense [n_mat][T][ceil(I/16)]; scales:
 * E4M3 codes [n_mat][T][ceil(I/16)].  Errors as tq_pack.
 *
 * tq_nvfp4_scales_to_mma: E4M3 block-scale codes [n_mat][rows][ceil(cols/16)]
 * re-laid out as the tensor core's scale tiles (out: tq_nvfp4_scales_mma_bytes
 * bytes, 16-byte aligned): per matrix, row tiles of 128 rows (their count
 * rounded up to an even number) by chunks of 4 blocks (rounded up to a
 * multiple of 4), each chunk 512 bytes with the scale of row r, block k at
 * byte (r % 32) * 16 + ((r % 128) / 32) * 4 + k % 4; order [matrix][row
 * tile][chunk]; padding is zero.  Weights need it once; activations per call.
 *
 * tq_gemm_nvfp4: y[e][t][o] = x_global[e] w_global[e] sum_k dec(ex[e][t][k])
 * dec(ew[e][o][k]) sum_{j in block k} dec(cx[e][t][j]) dec(cw[e][o][j]),
 * fp32 [n_mat][T][O] (row stride O), for records x_packed [n_mat][T][I/16]
 * and w_packed [n_mat][O][I/16] (8 bytes per block, as tq_search_groups /
 * tq_pack / tq_quant_nvfp4_act write them) and scales in the tiles of
 * tq_nvfp4_scales_to_mma (T and O rows).  I must be a multiple of 32 and
 * every pointer 16-byte aligned.  Accumulation is fp32 on the tensor cores:
 * |y - y_exact| <= (I/16 + 32) 2^-22 sum_j |x_j w_j| (dequantized values),
 * plus one rounding of the global-scale product.  Errors: TQ_ERR_INVALID_ARG
 * for null/misaligned pointers or bad sizes.  A pipeline wait that exceeds
 * its limit makes the CTA store nothing and the next tq_sync return
 * TQ_ERR_CUDA. */
tq_status tq_quant_nvfp4_act(const tq_mat* X, uint8_t* packed, uint8_t* scales, float* global_scale,
                             tq_stream_t stream);
size_t tq_nvfp4_scales_mma_bytes(int64_t n_mat, int64_t rows, int64_t cols);
tq_status tq_nvfp4_scales_to_mma(const uint8_t* scales, int64_t n_mat, int64_t rows, int64_t cols, uint8_t* out,
                                 tq_stream_t stream);
tq_status tq_gemm_nvfp4(const uint8_t* x_packed, const uint8_t* x_scales_mma, const float* x_global,
                        const uint8_t* w_packed, const uint8_t* w_scales_mma, const float* w_global,
                        int64_t n_mat, int64_t T, int64_t O, int64_t I, float* y, tq_stream_t stream);

/* ------------------------------------------------------------------ FP8 per tensor
 * E4M3 weights with one fp32 scale per matrix ([NVFP4] Quantization Recipe
 * table: FP8 per-tensor for the shared experts and the Mamba linears).  The
 * scale is searched like the other formats' (imatrix-weighted squared error):
 * candidates s_k = fl32(r_k amax / 448), r_k = fl32(lo + (hi - lo) k /
 * (n_cand - 1)), amax = max |w| of the matrix; loss L_k = sum_{o,j} m_j
 * (w - fl32(s_k dec(c)))^2 in fp64 with c the E4M3 code of fl32(w / s_k)
 * (round to nearest, ties to even, saturating at 448, +0 for a zero
 * result); the lowest k of the minimum wins (deterministic: fixed partition,
 * fixed reduction order).  amax = 0 gives scale 0, index -1, loss 0, codes 0.
 * scales: f32 [n_mat] (required); cand_idx: i32 [n_mat], loss: f64 [n_mat],
 * losses: f64 [n_mat][n_cand] (optional); packed: u8 [n_mat][O][I] E4M3 codes
 * of the chosen scale (optional, 16-byte aligned).  n_cand in [2, 64]
 * (TQ_ERR_UNSUPPORTED otherwise); 0 < lo <= hi.  workspace: >=
 * tq_fp8_workspace_bytes(W), 16-byte aligned, no initialisation needed.
 * tq_pack_fp8 writes the codes for given scales; tq_dequant_fp8 writes
 * What = fl32(s dec(c)) (fp32, or its RNE to bf16) as dense [n_mat][O][I]
 * (scale codes are read as e4m3fn; 0x7F/0xFF are outside the domain). */
size_t tq_fp8_workspace_bytes(const tq_mat* W);
tq_status tq_search_fp8(const tq_mat* W, const float* m, int64_t m_stride, int32_t n_cand, double lo, double hi,
                        float* scales, int32_t* cand_idx, double* loss, double* losses, uint8_t* packed,
                        void* workspace, size_t workspace_bytes, tq_stream_t stream);
tq_status tq_pack_fp8(const tq_mat* W, const float* scales, uint8_t* packed, tq_stream_t stream);
tq_status tq_dequant_fp8(const uint8_t* packed, const float* scales, int64_t n_mat, int64_t O, int64_t I,
                         void* out, int32_t out_dtype, tq_stream_t stream);

/* ------------------------------------------------------------------ Lloyd-Max 2-bit codebook
 * A 4-level codebook for 2-bit weights fit to the data ("Phase 2:
 * math-accuracy regression on tq3a-tq2e g32", Phase-2 candidate 1), read as:
 * 32-weight groups with the absmax scale s; u = fl32(w / s) (0 for s = 0);
 * one fp32 codebook c_0 < ... < c_3 shared by every matrix of the call,
 * fit by n_iter Lloyd iterations that minimise sum m_j (w - s c_a)^2: each
 * element to the nearest level (ties to the lower: u above the exact fp64
 * midpoint moves up), each level to the (m s^2)-weighted mean of its elements
 * (fp64 sums, rounded once to fp32; an empty level keeps its value).
 * codebook: device f32 [4], the start on entry (sorted), the fit on return;
 * scales: f32 [n_mat][O][ceil(I/32)] (out); packed: optional 2-bit codes, 8
 * bytes per group (element k at bits 2 (k % 4) of byte k / 4; padding 0);
 * loss: optional f64 [1], the weighted error of the final codebook; history:
 * optional f64 [n_iter + 1], the error before each update and after the last.
 * Deterministic (fixed partition and reduction order).  m: f32 [I] or
 * [n_mat][I] (m_stride), 16-byte aligned.  workspace: >=
 * tq_lloyd_workspace_bytes(W), 16-byte aligned.  n_iter in [0, 1000].
 * tq_dequant_lm2: What = fl32(s c_a), dense [n_mat][O][I] fp32 or bf16. */
size_t tq_lloyd_workspace_bytes(const tq_mat* W);
tq_status tq_lloyd_max_g32(const tq_mat* W, const float* m, int64_t m_stride, int32_t n_iter, float* codebook,
                           float* scales, uint8_t* packed, double* loss, double* history, void* workspace,
                           size_t workspace_bytes, tq_stream_t stream);
tq_status tq_dequant_lm2(const uint8_t* packed, const float* codebook, const float* scales, int64_t n_mat,
                         int64_t O, int64_t I, void* out, int32_t out_dtype, tq_stream_t stream);

/* ------------------------------------------------------------------ Hessian
 * H[e] = alpha * sum_t X[e][t]^T X[e][t] (+ H[e] when accumulate): the
 * per-linear-input Hessian ([TT] pipeline table, step 1), fp32, from bf16
 * activations X (tq_mat: n_mat sites of T tokens x I columns, ld and
 * mat_stride multiples of 8 elements, 16-byte aligned), on the tensor cores
 * (bf16 products exact, fp32 accumulation; alpha applied once, after).
 * Its diagonal is T * the imatrix of tq_imatrix.  H: fp32 dense [n_mat][I]
 * rows of ldh >= I elements, h_mat_stride >= I * ldh between sites; both
 * triangles are written, exactly symmetric.  Error bound against the exact
 * sum: |H - X^T X| <= (T/16 + 32) 2^-22 (|X|^T |X|) elementwise (every
 * 16-token step of the accumulation rounds once).  Errors: TQ_ERR_INVALID_ARG
 * for null/misaligned pointers, bad sizes or strides; TQ_ERR_UNSUPPORTED for
 * fp32 X.  A pipeline wait that exceeds its limit makes the kernel give up
 * (results undefined) and the next tq_sync return TQ_ERR_CUDA. */
tq_status tq_hessian(const tq_mat* X, float* H, int64_t ldh, int64_t h_mat_stride, float alpha,
                     int32_t accumulate, tq_stream_t stream);

/* ------------------------------------------------------------------ proxy error
 * Per matrix e ([TT] "Risks to measure: Precision", H = diag(m)):
 *   num[e] = sum_{o,j} m_j (W - What)^2 = tr(E H E^T),
 *   den[e] = sum_{o,j} m_j W^2          = tr(W H W^T),
 * with What the fp32 dequantized weights of `packed`.  fp64 outputs, fixed
 * reduction order.  workspace: >= tq_proxy_workspace_bytes(); its contents
 * need no initialisation. */
size_t tq_proxy_workspace_bytes(const tq_mat* W, int32_t fmt);
tq_status tq_proxy_error(const tq_mat* W, const uint8_t* packed, int32_t fmt, const void* scales,
                         const uint8_t* zeros, const float* global_scale, const float* m,
                         int64_t m_stride, double* num, double* den, void* workspace,
                         size_t workspace_bytes, tq_stream_t stream);

/* tq_proxy_error of n units in one launch (1 <= n <= TQ_MAX_BATCH; one
 * format, one weight dtype): unit i is W[i], packed[i], scales[i], zeros[i],
 * global_scale[i], m[i] (m_stride[i]) -> num[i][e], den[i][e].  W, m_stride
 * and the pointer arrays are host arrays of n entries.  workspace: >=
 * tq_proxy_batch_workspace_bytes(n, W, fmt), no initialisation needed.  The
 * values are those of n tq_proxy_error calls up to the order of their fp64
 * additions (fixed for a given device and batch); errors as tq_proxy_error. */
size_t tq_proxy_batch_workspace_bytes(int32_t n, const tq_mat* W, int32_t fmt);
tq_status tq_proxy_error_batch(int32_t n, const tq_mat* W, const uint8_t* const* packed, int32_t fmt,
                               const void* const* scales, const uint8_t* const* zeros,
                               const float* const* global_scale, const float* const* m,
                               const int64_t* m_stride, double* const* num, double* const* den,
                               void* workspace, size_t workspace_bytes, tq_stream_t stream);

/* ------------------------------------------------------------------ proxy error, full Hessian
 * Per matrix e ([TT] "Risks to measure: Precision", H = X^T X of the
 * calibration activations, never formed):
 *   num[e] = tr(E H E^T) = ||X E^T||_F^2,  E = W - What,
 *   den[e] = tr(W H W^T) = ||X W^T||_F^2,
 * on the tensor cores, one pass over X for both products.  X: bf16 tq_mat of
 * n_mat sites of T tokens x I columns; W: bf16 tq_mat [n_mat][O][I] (same I
 * and n_mat); What: the fp32 dequantized weights of `packed` (fmt, scales,
 * zeros, global_scale as in tq_dequant).  E is rounded once to fp32 and
 * carried as two bf16 pieces E1 + E2 (16 significant bits, relative error at
 * most 2^-16); the products are exact, Y = X E^T accumulates in fp32 and its
 * squares add in fp64 in a fixed order (deterministic).  Error bound:
 * |Y - X E^T| <= Delta = ((K/16 + 32) 2^-22 + 2^-15) (|X| |E|^T) elementwise,
 * K = 2 ceil(I/64) 64 for num (ceil(I/64) 64 and no 2^-15 term for den), and
 * |num - ||X E^T||^2| <= sum_{t,o} (2 |Y| + Delta) Delta.
 * workspace: >= tq_proxy_full_workspace_bytes(X, W) (E's pieces, 4 bytes per
 * weight with I padded to a multiple of 64, plus two fp64 per 128 x 256 tile
 * of Y), 16-byte aligned, needs no initialisation.  Errors:
 * TQ_ERR_INVALID_ARG for null/misaligned pointers, bad sizes or strides, a
 * small workspace; TQ_ERR_UNSUPPORTED for fp32 X or W or an unknown format.
 * A pipeline wait that exceeds its limit makes the kernel give up (the
 * matrix's num/den become NaN) and the next tq_sync return TQ_ERR_CUDA. */
size_t tq_proxy_full_workspace_bytes(const tq_mat* X, const tq_mat* W);
tq_status tq_proxy_error_full(const tq_mat* X, const tq_mat* W, const uint8_t* packed, int32_t fmt,
                              const void* scales, const uint8_t* zeros, const float* global_scale,
                              double* num, double* den, void* workspace, size_t workspace_bytes,
                              tq_stream_t stream);

/* ------------------------------------------------------------------ GPTQ/LDLQ column sweep
 * [TT] pipeline table, step 3: the columns are rounded one after another and
 * each one's rounding error is carried to the later columns through the
 * inverse Hessian's triangular factor, with the group scales (and
 * zero-points) of a search held fixed.  U: fp32 upper triangular factor with H^-1 = U^T U, rows of ldu >= I
 * elements, u_mat_stride elements between matrices (0: one factor for every
 * matrix); only its upper triangle is read; U_ii > 0 (the caller's Cholesky
 * of the damped, inverted H).  Per row, for each column i in order:
 *   code of the current w_i under its group's scale (round half to even of
 *   the IEEE fp32 quotient, clamped; int3 v in [-4, 3], int4 q in [0, 15]
 *   with the group's zero-point; a zero scale gives v = 0 / q = z),
 *   What_i = fl32(s v) or fl32(s (q - z)),
 *   e_i = (w_i - What_i) / U_ii (fp32),
 *   w_j <- fma(-e_i, U_ij, w_j) for every j > i (fp32, in column order).
 * Deterministic and independent of the tiling: results are bitwise those of
 * the unblocked sweep.  W: bf16 or fp32 tq_mat [n_mat][O][I]; fmt:
 * TQ_INT3_G64_SYM or an int4 format (g128, g64, g32); scales f32 and
 * zeros u8 [n_mat][O][ceil(I/g)] as tq_search_groups writes them.  codes:
 * int8 [n_mat][O][I] (int3: v; int4: q), the input of tq_pack_codes.  loss:
 * optional fp64 [n_mat][O], sum_i e_i^2 per row in column order (equal to
 * (w - What) H (w - What)^T in exact arithmetic).  workspace: >=
 * tq_gptq_workspace_bytes(W) (an fp32 working copy of W), 16-byte aligned.
 * Errors: TQ_ERR_INVALID_ARG for null/misaligned pointers, ldu < I, a short
 * u_mat_stride or workspace; TQ_ERR_UNSUPPORTED for NVFP4. */
size_t tq_gptq_workspace_bytes(const tq_mat* W);
tq_status tq_gptq_sweep(const tq_mat* W, int32_t fmt, const void* scales, const uint8_t* zeros, const float* U,
                        int64_t ldu, int64_t u_mat_stride, int8_t* codes, double* loss, void* workspace,
                        size_t workspace_bytes, tq_stream_t stream);

/* ------------------------------------------------------------------ testing aid
 * Synchronises `stream` and returns TQ_ERR_CUDA if it or an earlier kernel
 * failed (including a tq_hessian, tq_proxy_error_full or tq_gemm_nvfp4 launch
 * that gave up on a pipeline wait). */
tq_status tq_sync(tq_stream_t stream);

/* Testing aid for the give-up path of the tensor-core pipelines: the number
 * of try-wait rounds after which a pipeline wait of a later tq_hessian,
 * tq_proxy_error_full or tq_gemm_nvfp4 launch (in this process) gives up; rounds < 0 restores
 * the default (2^22 rounds, seconds of waiting).  Only the waits of the
 * copy/MMA ring use it: a launch that gives up still waits, with the default
 * limit, for every copy it issued and every MMA it committed before it frees
 * its shared memory and tensor memory, so a small limit (0 gives up at the
 * first wait, before any copy is issued) leaves nothing in flight.  Not for
 * production use; returns TQ_OK. */
tq_status tq_debug_set_wait_limit(int64_t rounds);

/* Self-test of the GPU's E2M1 conversion instructions, on which the NVFP4
 * round-to-nearest (search, tq_pack) and decoding (tq_dequant,
 * tq_proxy_error) rely.  The pages define the element format only (E2M1:
 * values 0, .5, 1, 1.5, 2, 3, 4, 6 with a sign; [NVFP4] Quantization Recipe);
 * this call has no counterpart there.  Checks every fp32 value but NaN
 * (rounded half to even, saturating at 6, sign in bit 3 even for -0) in both
 * nibbles of a byte, and all 256 bytes decoded bit for bit.  *mismatches (host) gets the
 * number of failing cases, 0 on a conforming GPU; *first_bad (host, may be
 * NULL) the first failing fp32 pattern (0x80000000 | byte for a decode
 * failure, 0xffffffff when none).  Uses two words of static device memory
 * (concurrent calls race on them) and synchronises `stream`. */
tq_status tq_selftest_e2m1(uint64_t* mismatches, uint32_t* first_bad, tq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
