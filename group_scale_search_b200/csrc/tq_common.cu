// Host-side plumbing of the tq library: error state, sizes, defaults.
#include "tq_internal.cuh"

#include <string.h>

#include <atomic>

namespace tq {

static std::atomic<int64_t> g_wait_limit{-1};

unsigned pipeline_wait_limit() {
    const int64_t v = g_wait_limit.load(std::memory_order_relaxed);
    return v < 0 ? DEFAULT_WAIT_LIMIT : static_cast<unsigned>(v > 0xffffffffll ? 0xffffffffll : v);
}

static thread_local char g_err[512];

tq_status set_error(tq_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

void clear_error() { g_err[0] = 0; }

tq_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return TQ_OK;
}

tq_status check_mat(const tq_mat* X, const char* name) {
    TQ_REQUIRE(X != nullptr, "%s: null descriptor", name);
    TQ_REQUIRE(X->ptr != nullptr, "%s: null data pointer", name);
    const int eb = elem_bytes(X->dtype);
    if (eb == 0) return set_error(TQ_ERR_UNSUPPORTED, "%s: dtype %d not supported", name, X->dtype);
    TQ_REQUIRE(X->n_mat >= 1 && X->rows >= 1 && X->cols >= 1, "%s: empty or negative shape", name);
    TQ_REQUIRE(X->ld >= X->cols, "%s: ld (%lld) < cols (%lld)", name, (long long)X->ld, (long long)X->cols);
    TQ_REQUIRE(X->n_mat == 1 || X->mat_stride >= X->rows * X->ld,
               "%s: mat_stride (%lld) < rows*ld", name, (long long)X->mat_stride);
    TQ_REQUIRE(aligned16(X->ptr), "%s: data pointer not 16-byte aligned", name);
    TQ_REQUIRE((X->ld * eb) % 16 == 0, "%s: row stride not a multiple of 16 bytes", name);
    TQ_REQUIRE(X->n_mat == 1 || (X->mat_stride * eb) % 16 == 0,
               "%s: matrix stride not a multiple of 16 bytes", name);
    return TQ_OK;
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

}  // namespace tq

using namespace tq;

TQ_API void tq_default_params(tq_search_params* p) {
    if (!p) return;
    memset(p, 0, sizeof *p);
    p->sym_n1 = 32; p->sym_n2 = 32; p->sym_lo = 0.5; p->sym_hi = 1.2;
    p->asym_n_scale = 64; p->asym_n_zero = 32; p->asym_lo = 0.5; p->asym_hi = 1.2;
    p->fp4_window = 16;
}

TQ_API const char* tq_last_error_string(void) { return g_err; }

TQ_API const char* tq_version(void) { return "tq 1.0 sm_100a"; }

TQ_API int64_t tq_group_size(int32_t fmt) { return group_of(fmt); }

TQ_API int64_t tq_num_groups(int32_t fmt, int64_t rows, int64_t cols) {
    const int64_t g = group_of(fmt);
    if (g == 0 || rows < 0 || cols < 0) return 0;
    return rows * ((cols + g - 1) / g);
}

TQ_API size_t tq_packed_bytes(int32_t fmt, int64_t rows, int64_t cols) {
    return static_cast<size_t>(tq_num_groups(fmt, rows, cols) * record_bytes(fmt));
}

TQ_API tq_status tq_debug_set_wait_limit(int64_t rounds) {
    clear_error();
    g_wait_limit.store(rounds < 0 ? -1 : rounds, std::memory_order_relaxed);
    return TQ_OK;
}

TQ_API tq_status tq_sync(tq_stream_t stream) {
    clear_error();
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(TQ_ERR_CUDA, "tq_sync: %s", cudaGetErrorString(e));
    if (hessian_take_timeouts()) return set_error(TQ_ERR_CUDA, "tq_sync: a tq_hessian pipeline wait timed out");
    if (proxy_full_take_timeouts())
        return set_error(TQ_ERR_CUDA, "tq_sync: a tq_proxy_error_full pipeline wait timed out");
    if (nvfp4_gemm_take_timeouts())
        return set_error(TQ_ERR_CUDA, "tq_sync: a tq_gemm_nvfp4 pipeline wait timed out");
    return TQ_OK;
}
