// capi.cu -- the extern "C" entry points of libmxq (declared in include/mxq.h).
//
// Each call checks its arguments on the host, launches nothing on an argument error,
// and otherwise enqueues its kernel(s) on the caller's stream and returns without
// synchronizing.  No call allocates memory.

#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "mxq.h"
#include "mxq_launch.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MXQ_OK;
    std::strncpy(g_last_cuda_error, cudaGetErrorString(e), sizeof(g_last_cuda_error) - 1);
    g_last_cuda_error[sizeof(g_last_cuda_error) - 1] = '\0';
    return MXQ_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// a * b * c without int64 overflow (all non-negative)
bool mul_ok(int64_t a, int64_t b, int64_t c, int64_t* out) {
    const int64_t lim = INT64_MAX / 4;  // keep byte offsets of 2-byte elements in range
    if (a != 0 && b > lim / a) return false;
    const int64_t ab = a * b;
    if (ab != 0 && c > lim / ab) return false;
    *out = ab * c;
    return true;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace

namespace mxq {

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace mxq

extern "C" {

int mx_quantize(const void* x_bf16, int64_t batch, int64_t rows, int64_t cols, int axes,
                uint8_t* q_row, uint8_t* s_row, uint8_t* q_col, uint8_t* s_col, void* stream) {
    if (axes < 1 || axes > 3) return MXQ_ERR_ARG;
    if (batch < 0 || rows < 0 || cols < 0) return MXQ_ERR_SHAPE;
    const bool do_row = (axes & MXQ_AXIS_ROW) != 0, do_col = (axes & MXQ_AXIS_COL) != 0;
    if (cols % 32 != 0 || (do_col && rows % 32 != 0)) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(batch, rows, cols, &n)) return MXQ_ERR_SHAPE;
    if (n == 0) return MXQ_OK;  // empty tensors may carry NULL data pointers
    if (!x_bf16) return MXQ_ERR_NULL;
    if (do_row && (!q_row || !s_row)) return MXQ_ERR_NULL;
    if (do_col && (!q_col || !s_col)) return MXQ_ERR_NULL;
    if (!aligned(x_bf16, 16)) return MXQ_ERR_ALIGN;
    if (do_row && !aligned(q_row, 16)) return MXQ_ERR_ALIGN;
    if (do_col && !aligned(q_col, 16)) return MXQ_ERR_ALIGN;
    const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
    cudaError_t e;
    if (do_row && !do_col)
        e = mxq::launch_quant_rows(x, q_row, s_row, n / 32, as_stream(stream));
    else
        e = mxq::launch_quant_tile(x, batch, rows, cols, do_row, do_col, q_row, s_row, q_col, s_col,
                                   as_stream(stream));
    return cuda_status(e);
}

int mx_dequantize(const uint8_t* q, const uint8_t* s, int64_t batch, int64_t rows, int64_t cols,
                  int axis, void* y_bf16, void* stream) {
    if (axis != MXQ_AXIS_ROW && axis != MXQ_AXIS_COL) return MXQ_ERR_ARG;
    if (batch < 0 || rows < 0 || cols < 0) return MXQ_ERR_SHAPE;
    if (cols % 32 != 0 || (axis == MXQ_AXIS_COL && rows % 32 != 0)) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(batch, rows, cols, &n)) return MXQ_ERR_SHAPE;
    if (n == 0) return MXQ_OK;  // empty tensors may carry NULL data pointers
    if (!q || !s || !y_bf16) return MXQ_ERR_NULL;
    if (!aligned(q, 16) || !aligned(y_bf16, 16)) return MXQ_ERR_ALIGN;
    uint16_t* y = static_cast<uint16_t*>(y_bf16);
    cudaError_t e = axis == MXQ_AXIS_ROW
                        ? mxq::launch_dequant_rows(q, s, y, n, as_stream(stream))
                        : mxq::launch_dequant_tile(q, s, batch, rows, cols, y, as_stream(stream));
    return cuda_status(e);
}

int fp8_per_group_rowwise_quant(const void* x_bf16, int64_t M, int64_t K, const int32_t* offs,
                                int32_t G, int out_layout, uint8_t* q, float* scales,
                                void* stream) {
    if (out_layout != MXQ_LAYOUT_ROW_MAJOR && out_layout != MXQ_LAYOUT_COL_MAJOR) return MXQ_ERR_ARG;
    if (M < 0 || K < 0 || G < 0) return MXQ_ERR_SHAPE;
    if (K % 8 != 0 || G > 65535) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(M, K, 1, &n)) return MXQ_ERR_SHAPE;
    if (K == 0 || G == 0) return MXQ_OK;
    if (!offs || !scales) return MXQ_ERR_NULL;
    if (M > 0 && (!x_bf16 || !q)) return MXQ_ERR_NULL;
    if (!aligned(offs, 4) || !aligned(scales, 4)) return MXQ_ERR_ALIGN;
    if (M > 0 && (!aligned(x_bf16, 16) || !aligned(q, 16))) return MXQ_ERR_ALIGN;
    cudaError_t e = mxq::launch_per_group(static_cast<const uint16_t*>(x_bf16), M, K, offs, G,
                                          out_layout == MXQ_LAYOUT_COL_MAJOR, q, scales,
                                          as_stream(stream));
    return cuda_status(e);
}

int fp8_per_group_rowwise_quant_batched(const void* x_bf16, int64_t E, int64_t M, int64_t K, int out_layout,
                                        uint8_t* q, float* scales, void* stream) {
    if (out_layout != MXQ_LAYOUT_ROW_MAJOR && out_layout != MXQ_LAYOUT_COL_MAJOR) return MXQ_ERR_ARG;
    if (E < 0 || M < 0 || K < 0) return MXQ_ERR_SHAPE;
    if (K % 8 != 0 || E > 65535) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(E, M, K, &n) || E * M > 0x7FFFFFFFLL) return MXQ_ERR_SHAPE;
    if (K == 0 || E == 0) return MXQ_OK;
    if (!scales) return MXQ_ERR_NULL;
    if (M > 0 && (!x_bf16 || !q)) return MXQ_ERR_NULL;
    if (!aligned(scales, 4)) return MXQ_ERR_ALIGN;
    if (M > 0 && (!aligned(x_bf16, 16) || !aligned(q, 16))) return MXQ_ERR_ALIGN;
    if (M == 0) {  // every matrix empty: only the scales, 448 / fp32(1e-12)
        cudaError_t e = mxq::launch_per_group(nullptr, 0, K, nullptr, (int32_t)E, false, nullptr, scales,
                                              as_stream(stream), 1);
        return cuda_status(e);
    }
    cudaError_t e = mxq::launch_per_group(static_cast<const uint16_t*>(x_bf16), E * M, K, nullptr, (int32_t)E,
                                          out_layout == MXQ_LAYOUT_COL_MAJOR, q, scales, as_stream(stream),
                                          (int)M);
    return cuda_status(e);
}

int fp8_per_group_rowwise_plan(int64_t M, int64_t K, int32_t G, int out_layout, int n_sm, int* kernel,
                               int* slab_cols, int* cluster, int* tile_rows, int* threads) {
    if (!kernel || !slab_cols || !cluster || !tile_rows || !threads) return MXQ_ERR_NULL;
    if (out_layout != MXQ_LAYOUT_ROW_MAJOR && out_layout != MXQ_LAYOUT_COL_MAJOR) return MXQ_ERR_ARG;
    if (M < 0 || K < 0 || G < 0 || n_sm < 0) return MXQ_ERR_SHAPE;
    if (K % 8 != 0 || G > 65535) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(M, K, 1, &n)) return MXQ_ERR_SHAPE;
    if (n_sm == 0) {
        n_sm = mxq::sm_count();
        if (n_sm <= 0) return MXQ_ERR_CUDA;
    }
    const mxq::PerGroupPlan p = mxq::plan_per_group(M, K, G, out_layout == MXQ_LAYOUT_COL_MAJOR, n_sm);
    *kernel = p.kind;
    *slab_cols = p.w;
    *cluster = p.cl;
    *tile_rows = p.r_cap;
    *threads = p.threads;
    return MXQ_OK;
}

int mxq_transpose_u8(const uint8_t* src, int64_t batch, int64_t rows, int64_t cols, uint8_t* dst, void* stream) {
    if (batch < 0 || rows < 0 || cols < 0) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(batch, rows, cols, &n)) return MXQ_ERR_SHAPE;
    if (n == 0) return MXQ_OK;
    if (!src || !dst) return MXQ_ERR_NULL;
    return cuda_status(mxq::launch_transpose_u8(src, batch, rows, cols, dst, as_stream(stream)));
}

int64_t mx_scales_blocked_bytes(int64_t batch, int64_t rows, int64_t n_k, int32_t G) {
    if (batch < 0 || rows < 0 || n_k < 0 || G < 0 || (G > 0 && batch != 1)) return -1;
    int64_t n = 0;
    if (!mul_ok(batch, rows + 128 * (int64_t)G + 128, n_k + 4, &n)) return -1;
    return mxq::scales_blocked_bytes(batch, rows, n_k, G);
}

int mx_scales_to_blocked(const uint8_t* s, int64_t batch, int64_t rows, int64_t n_k, const int32_t* offs,
                         int32_t G, uint8_t* out, void* stream) {
    if (batch < 0 || rows < 0 || n_k < 0 || G < 0) return MXQ_ERR_SHAPE;
    if (G > 0 && batch != 1) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(batch, rows + 128 * (int64_t)G + 128, n_k + 4, &n)) return MXQ_ERR_SHAPE;
    if (n_k == 0 || batch == 0 || (G == 0 && rows == 0)) return MXQ_OK;
    if (G > 0 && !offs) return MXQ_ERR_NULL;
    if (!out || (rows > 0 && !s)) return MXQ_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(out) & 15) != 0) return MXQ_ERR_ALIGN;
    if (G > 0 && (reinterpret_cast<uintptr_t>(offs) & 3) != 0) return MXQ_ERR_ALIGN;
    return cuda_status(mxq::launch_scales_to_blocked(s, batch, rows, n_k, offs, G, out, as_stream(stream)));
}

int mx_grouped_gemm(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb, const uint8_t* sfb,
                    const int32_t* offs, int32_t G, int64_t M, int64_t N, int64_t K, void* out_bf16, void* stream) {
    if (M < 0 || N < 0 || K < 0 || G < 0) return MXQ_ERR_SHAPE;
    if (K % 128 != 0 || N % 256 != 0 || G > 65535) return MXQ_ERR_SHAPE;
    int64_t n = 0;
    if (!mul_ok(M + 128 * (int64_t)G, N + K, 1, &n) || !mul_ok(G, N, K, &n)) return MXQ_ERR_SHAPE;
    if (M == 0 || N == 0 || K == 0 || G == 0) return MXQ_OK;
    if (!qa || !sfa || !qb || !sfb || !offs || !out_bf16) return MXQ_ERR_NULL;
    if (!aligned(qa, 16) || !aligned(qb, 16) || !aligned(sfa, 16) || !aligned(sfb, 16) || !aligned(out_bf16, 16) ||
        !aligned(offs, 4))
        return MXQ_ERR_ALIGN;
    return cuda_status(mxq::launch_mx_grouped_gemm(qa, sfa, qb, sfb, offs, G, M, N, K,
                                                   static_cast<uint16_t*>(out_bf16), as_stream(stream)));
}

int mx_e4m3_encode_f32(const float* x, int64_t n, uint8_t* q, void* stream) {
    if (n < 0) return MXQ_ERR_SHAPE;
    if (n == 0) return MXQ_OK;
    if (!x || !q) return MXQ_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16)) return MXQ_ERR_ALIGN;
    return cuda_status(mxq::launch_encode_f32(x, q, n, as_stream(stream)));
}

const char* mxq_status_string(int status) {
    switch (status) {
        case MXQ_OK: return "MXQ_OK";
        case MXQ_ERR_NULL: return "MXQ_ERR_NULL: a required pointer is NULL";
        case MXQ_ERR_SHAPE: return "MXQ_ERR_SHAPE: invalid sizes for this layout";
        case MXQ_ERR_ALIGN: return "MXQ_ERR_ALIGN: pointer alignment rule violated";
        case MXQ_ERR_ARG: return "MXQ_ERR_ARG: enum argument out of range";
        case MXQ_ERR_CUDA: return "MXQ_ERR_CUDA: the CUDA runtime rejected a launch";
        case MXQ_ERR_NOT_IMPLEMENTED: return "MXQ_ERR_NOT_IMPLEMENTED";
        default: return "unknown mxq status";
    }
}

const char* mxq_last_cuda_error(void) { return g_last_cuda_error; }

int mxq_wait_timeouts(unsigned int* count) {
    if (!count) return MXQ_ERR_NULL;
    const unsigned int n = mxq::read_wait_timeouts(), m = mxq::read_gemm_timeouts();
    if (n == 0xFFFFFFFFu || m == 0xFFFFFFFFu) return MXQ_ERR_CUDA;
    *count = n + m;
    return MXQ_OK;
}

int mxq_wait_abandoned(unsigned int* count) {
    if (!count) return MXQ_ERR_NULL;
    const unsigned int n = mxq::read_wait_abandoned();
    if (n == 0xFFFFFFFFu) return MXQ_ERR_CUDA;
    *count = n;
    return MXQ_OK;
}

int mxq_set_wait_limit_ns(uint64_t ns) {
    mxq::set_wait_limit_ns(ns);
    return MXQ_OK;
}

}  // extern "C"
