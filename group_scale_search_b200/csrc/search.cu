// tq_search_groups: argument validation and dispatch to the per-format
// search kernels (search_int3.cu, search_int4.cu, search_nvfp4.cu).
#include "tq_internal.cuh"

namespace tq {
tq_status launch_search_int3(const tq_mat* W, const float* m, int64_t m_stride, const tq_search_params* p,
                             float* scales, int32_t* idx, double* loss, uint8_t* packed, cudaStream_t st);
tq_status launch_search_int4(const tq_mat* W, int gsize, const float* m, int64_t m_stride, const tq_search_params* p,
                             float* scales, uint8_t* zeros, int32_t* idx, double* loss, uint8_t* packed,
                             cudaStream_t st);
tq_status launch_search_nvfp4(const tq_mat* W, const float* m, int64_t m_stride, const tq_search_params* p,
                              uint8_t* scales, float* gscale, int32_t* idx, double* loss, uint8_t* packed,
                              cudaStream_t st);
}  // namespace tq

using namespace tq;

TQ_API tq_status tq_search_groups(const tq_mat* W, const float* m, int64_t m_stride, int32_t fmt,
                                  const tq_search_params* params, void* scales, uint8_t* zeros,
                                  float* global_scale, int32_t* cand_idx, double* loss, uint8_t* packed,
                                  tq_stream_t stream) {
    clear_error();
    tq_status s = check_mat(W, "tq_search_groups W");
    if (s != TQ_OK) return s;
    if (group_of(fmt) == 0) return set_error(TQ_ERR_UNSUPPORTED, "tq_search_groups: unknown format %d", fmt);
    TQ_REQUIRE(m != nullptr && aligned16(m), "tq_search_groups: m null or not 16-byte aligned");
    TQ_REQUIRE(W->n_mat == 1 || m_stride == 0 || (m_stride >= W->cols && m_stride % 4 == 0),
               "tq_search_groups: m_stride must be 0 or a multiple of 4 >= cols");
    TQ_REQUIRE(scales != nullptr, "tq_search_groups: null scales");
    TQ_REQUIRE(packed == nullptr || aligned16(packed), "tq_search_groups: packed not 16-byte aligned");
    TQ_REQUIRE(is_int4(fmt) == (zeros != nullptr),
               "tq_search_groups: zeros required for int4 and only for int4");
    TQ_REQUIRE((fmt == TQ_NVFP4_G16) == (global_scale != nullptr),
               "tq_search_groups: global_scale required for NVFP4 and only for NVFP4");
    tq_search_params def;
    if (!params) { tq_default_params(&def); params = &def; }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t mst = W->n_mat > 1 ? m_stride : 0;
    if (fmt == TQ_INT3_G64_SYM)
        return launch_search_int3(W, m, mst, params, static_cast<float*>(scales), cand_idx, loss, packed, st);
    if (is_int4(fmt))
        return launch_search_int4(W, static_cast<int>(group_of(fmt)), m, mst, params, static_cast<float*>(scales),
                                  zeros, cand_idx, loss, packed, st);
    return launch_search_nvfp4(W, m, mst, params, static_cast<uint8_t*>(scales), global_scale, cand_idx, loss,
                               packed, st);
}
