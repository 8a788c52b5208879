// api.cu -- the extern "C" boundary of libqmm (declared in include/qmm.h).
//
// Every entry point validates its arguments completely before enqueueing
// anything, reports failures as qmm_status values (mlx-rs
// ops/quantization.rs returns Result with an Exception; Emily checks its
// arguments and raises before any MLX call), and never lets a C++ exception
// cross the ABI.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "qmm_internal.cuh"

namespace qmm {

__device__ DeviceState g_qmm_state = {0, 0, kDefaultWaitNs};

namespace {

thread_local std::string t_last_error;
// Activation rows up to which the SIMT decode kernels are used (AUTO path).
constexpr int64_t kGemvMaxRows = 4;
qmm_path g_path = QMM_PATH_AUTO;
std::atomic<int> g_fault{QMM_FAULT_NONE};

qmm_status fail(qmm_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
qmm_status fail(qmm_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

qmm_status cuda_fail(cudaError_t e, const char *what) {
    return fail(QMM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Mode strings: "affine" (default), and the microscaled modes, which carry a
// fixed group size and bits and no biases (Emily.QuantizedWeight, section
// Microscaled modes).
qmm_status parse_mode(const char *mode, int *out) {
    *out = QMM_MODE_AFFINE;
    if (mode == nullptr || std::strcmp(mode, "affine") == 0) return QMM_OK;
    if (!std::strcmp(mode, "mxfp4")) *out = QMM_MODE_MXFP4;
    else if (!std::strcmp(mode, "mxfp8")) *out = QMM_MODE_MXFP8;
    else if (!std::strcmp(mode, "nvfp4")) *out = QMM_MODE_NVFP4;
    else return fail(QMM_ERR_INVALID_ARG, "unknown quantization mode \"%s\"", mode);
    return QMM_OK;
}

qmm_status check_common(qmm_dtype dt, int group_size, int bits, const char *mode,
                        int *mode_out = nullptr) {
    int m = QMM_MODE_AFFINE;
    qmm_status st = parse_mode(mode, &m);
    if (st != QMM_OK) return st;
    if (mode_out) *mode_out = m;
    if (dt != QMM_F32 && dt != QMM_BF16 && dt != QMM_F16)
        return fail(QMM_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    if (m != QMM_MODE_AFFINE) {
        const int gs = m == QMM_MODE_NVFP4 ? 16 : 32, b = m == QMM_MODE_MXFP8 ? 8 : 4;
        if (group_size != gs || bits != b)
            return fail(QMM_ERR_INVALID_ARG, "mode \"%s\" needs group_size=%d and bits=%d (got %d, %d)",
                        mode, gs, b, group_size, bits);
        return QMM_OK;
    }
    if (bits != 2 && bits != 3 && bits != 4 && bits != 6 && bits != 8)
        return fail(QMM_ERR_INVALID_ARG, "bits must be 2, 3, 4, 6 or 8 (got %d)", bits);
    if (group_size != 32 && group_size != 64 && group_size != 128)
        return fail(QMM_ERR_INVALID_ARG, "group_size must be 32, 64 or 128 (got %d)", group_size);
    return QMM_OK;
}

#define QMM_CHECK_PTR(p, name)                                                        \
    do {                                                                              \
        if ((p) == nullptr) return fail(QMM_ERR_INVALID_ARG, "%s is NULL", name);     \
        if (!aligned16(p)) return fail(QMM_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
    } while (0)

qmm_status check_matmul(const void *x, int64_t M, int64_t K, const uint32_t *wq,
                        const void *scales, const void *biases, int64_t N, int transpose,
                        int group_size, void *y, int mode = QMM_MODE_AFFINE) {
    if (M < 0 || N < 0 || K <= 0)
        return fail(QMM_ERR_INVALID_ARG, "sizes must satisfy M >= 0, N >= 0, K > 0");
    const int64_t packed_axis = transpose ? K : N;
    if (packed_axis % group_size != 0)
        return fail(QMM_ERR_INVALID_ARG,
                    "the packed axis (%s = %lld) must be a multiple of group_size %d",
                    transpose ? "K" : "N", (long long)packed_axis, group_size);
    if (M == 0 || N == 0) return QMM_OK;
    QMM_CHECK_PTR(x, "x");
    QMM_CHECK_PTR(wq, "wq");
    QMM_CHECK_PTR(scales, "scales");
    if (mode != QMM_MODE_AFFINE) {
        if (biases != nullptr)
            return fail(QMM_ERR_INVALID_ARG, "biases must be NULL in a microscaled mode");
    } else {
        if (biases == nullptr)
            return fail(QMM_ERR_INVALID_ARG, "biases is NULL (required for mode \"affine\")");
        QMM_CHECK_PTR(biases, "biases");
    }
    QMM_CHECK_PTR(y, "y");
    return QMM_OK;
}

// Whether gather_qmm can take the grouped tensor-core path (which needs the
// workspace) for these sizes.
bool gather_tc_supported(qmm_dtype dtype, int64_t x_batch, int64_t M, int64_t K, int64_t N,
                         int64_t n_experts, int64_t batch, int bits, int transpose) {
    GroupedArgs probe{};
    probe.transpose = transpose != 0;
    probe.K = K;
    probe.N = N;
    probe.bits = bits;
    probe.rows = batch * M;
    probe.x_rows = x_batch * M;
    probe.n_experts = n_experts;
    return gemm_grouped_supported(dtype, probe) && gather_prep_fits(n_experts);
}

qmm_status finish_launch(cudaError_t e, const char *what) {
    if (e != cudaSuccess) return cuda_fail(e, what);
    return QMM_OK;
}

}  // namespace

// Products with microscaled weights: the tensor-core GEMM for more than a few
// activation rows ([N, K] layout), else the SIMT kernels (any shape, either
// layout; the gather entry takes affine weights only).
cudaError_t launch_mx_matmul(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    // more than a few activation rows: the tensor-core GEMM where it applies;
    // a few rows of E2M1 codes: the streaming decode kernel; a few rows of
    // E4M3 codes: the GEMM too (the SIMT kernel is ~3x slower there)
    if (a.M > kGemvMaxRows && gemm_supported(dt, a)) return launch_gemm(dt, a, s);
    if (gemv_fast_supported(dt, a)) return launch_gemv_fast(dt, a, s);
    if (gemm_supported(dt, a)) return launch_gemm(dt, a, s);
    return launch_gemv(dt, a, s);
}

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int *device_error_word() {
    static int *cached[64] = {nullptr};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return nullptr;
    if (cached[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_qmm_state) != cudaSuccess) return nullptr;
        cached[dev] = &static_cast<DeviceState *>(p)->error;
    }
    return cached[dev];
}

int injected_fault() { return g_fault.load(std::memory_order_relaxed); }

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace qmm

using namespace qmm;

extern "C" {

qmm_status qmm_quantize(const void *w, qmm_dtype dtype, int64_t rows, int64_t cols,
                        int group_size, int bits, const char *mode, uint32_t *wq, void *scales,
                        void *biases, void *stream) {
    try {
        int md = QMM_MODE_AFFINE;
        qmm_status st = check_common(dtype, group_size, bits, mode, &md);
        if (st != QMM_OK) return st;
        if (rows < 0 || cols <= 0 || cols % group_size != 0)
            return fail(QMM_ERR_INVALID_ARG,
                        "need rows >= 0 and cols a positive multiple of group_size");
        if (rows == 0) return QMM_OK;
        QMM_CHECK_PTR(w, "w");
        QMM_CHECK_PTR(wq, "wq");
        QMM_CHECK_PTR(scales, "scales");
        if (md != QMM_MODE_AFFINE) {
            if (biases != nullptr)
                return fail(QMM_ERR_INVALID_ARG, "biases must be NULL in a microscaled mode");
            QuantArgs a{w, rows, cols, group_size, bits, wq, scales, nullptr, md};
            return finish_launch(launch_quantize_mx(dtype, a, (cudaStream_t)stream), "quantize launch");
        }
        QMM_CHECK_PTR(biases, "biases");
        QuantArgs a{w, rows, cols, group_size, bits, wq, scales, biases};
        return finish_launch(launch_quantize(dtype, a, (cudaStream_t)stream), "quantize launch");
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_quantize");
    }
}

qmm_status qmm_dequantize(const uint32_t *wq, const void *scales, const void *biases,
                          qmm_dtype dtype, int64_t rows, int64_t cols, int group_size, int bits,
                          const char *mode, void *out, void *stream) {
    try {
        int md = QMM_MODE_AFFINE;
        qmm_status st = check_common(dtype, group_size, bits, mode, &md);
        if (st != QMM_OK) return st;
        if (rows < 0 || cols <= 0 || cols % group_size != 0)
            return fail(QMM_ERR_INVALID_ARG,
                        "need rows >= 0 and cols a positive multiple of group_size");
        if (rows == 0) return QMM_OK;
        QMM_CHECK_PTR(wq, "wq");
        QMM_CHECK_PTR(scales, "scales");
        if (md != QMM_MODE_AFFINE) {
            if (biases != nullptr)
                return fail(QMM_ERR_INVALID_ARG, "biases must be NULL in a microscaled mode");
            QMM_CHECK_PTR(out, "out");
            DequantArgs a{wq, scales, nullptr, rows, cols, group_size, bits, out, md};
            return finish_launch(launch_dequantize_mx(dtype, a, (cudaStream_t)stream),
                                 "dequantize launch");
        }
        if (biases == nullptr)
            return fail(QMM_ERR_INVALID_ARG, "biases is NULL (required for mode \"affine\")");
        QMM_CHECK_PTR(biases, "biases");
        QMM_CHECK_PTR(out, "out");
        DequantArgs a{wq, scales, biases, rows, cols, group_size, bits, out};
        return finish_launch(launch_dequantize(dtype, a, (cudaStream_t)stream),
                             "dequantize launch");
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_dequantize");
    }
}

}  // extern "C"

namespace {

// quantized_matmul with an optional layer bias (quantized_dense) and an
// optional stream-K workspace: the implementation of the three entry points.
qmm_status route_matmul(qmm_dtype dtype, const QmmArgs &a, cudaStream_t s);

// x_host / y_host (qmm_quantized_matmul_host): when given, the copy of x_host
// into x is enqueued once every argument has been checked, and the copy of y
// into y_host once the product has been launched (unless the product kernel
// wrote y_host itself).  mapped: x_host / y_host are already the device
// mappings of page-locked host memory (qmm_quantized_matmul_mapped).
qmm_status matmul_impl(const void *x, int64_t M, int64_t K, const uint32_t *wq, const void *scales,
                       const void *biases, qmm_dtype dtype, int64_t N, int transpose, int group_size,
                       int bits, const char *mode, const void *bias, double bias_value, void *y,
                       void *workspace, size_t workspace_bytes, void *stream,
                       const void *x_host = nullptr, void *y_host = nullptr, bool mapped = false) {
    try {
        int md = QMM_MODE_AFFINE;
        qmm_status st = check_common(dtype, group_size, bits, mode, &md);
        if (st != QMM_OK) return st;
        st = check_matmul(x, M, K, wq, scales, biases, N, transpose, group_size, y, md);
        if (st != QMM_OK) return st;
        if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
            return fail(QMM_ERR_WORKSPACE, "workspace must be 256-byte aligned");
        if (M == 0 || N == 0) return QMM_OK;
        if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & (dtype == QMM_F32 ? 3u : 1u)))
            return fail(QMM_ERR_INVALID_ARG, "bias is not aligned to its element size");
        if (!std::isfinite(bias_value))
            return fail(QMM_ERR_INVALID_ARG, "bias_value must be finite");
        QmmArgs a{x, wq, scales, biases, y, M, N, K, group_size, bits, transpose != 0};
        a.mode = md;
        a.bias = bias;
        a.bias_value = (float)bias_value;
        a.ws = workspace;
        a.ws_bytes = workspace ? workspace_bytes : 0;
        cudaStream_t s = (cudaStream_t)stream;
        const size_t es = dtype == QMM_F32 ? 4 : 2;
        // Page-locked host buffers are copied by kernels that read or write
        // their device mapping (chained with the product by programmatic
        // dependent launch), or written by the product kernel itself; other
        // host memory goes through the copy engines.
        if (x_host != nullptr) {
            const size_t bytes = (size_t)(M * K) * es;
            const void *xm = mapped ? x_host : mapped_host_pointer(x_host);
            cudaError_t e = xm ? launch_mapped_copy(xm, const_cast<void *>(x), bytes, s)
                               : cudaMemcpyAsync(const_cast<void *>(x), x_host, bytes, cudaMemcpyHostToDevice, s);
            if (e != cudaSuccess) return cuda_fail(e, "copy of x_host");
        }
        void *ym = nullptr;
        if (y_host != nullptr) ym = mapped ? y_host : const_cast<void *>(mapped_host_pointer(y_host));
        a.y2 = ym;
        const qmm_status launched = route_matmul(dtype, a, s);
        if (launched != QMM_OK || y_host == nullptr || a.y2_written) return launched;
        const size_t bytes = (size_t)(M * N) * es;
        cudaError_t e = ym ? launch_mapped_copy(y, ym, bytes, s)
                           : cudaMemcpyAsync(y_host, y, bytes, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return cuda_fail(e, "copy into y_host");
        return QMM_OK;
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_quantized_matmul");
    }
}

// Kernel choice and launch of one checked product (see qmm_set_path).
qmm_status route_matmul(qmm_dtype dtype, const QmmArgs &a, cudaStream_t s) {
    try {
        const int md = a.mode;
        if (md != QMM_MODE_AFFINE) {
            if (g_path == QMM_PATH_DECODE_TC)
                return fail(QMM_ERR_UNSUPPORTED, "the decode tensor-core path takes affine weights");
            if (g_path == QMM_PATH_GEMM) {
                if (!gemm_supported(dtype, a))
                    return fail(QMM_ERR_UNSUPPORTED,
                                "the tensor-core path takes microscaled weights as bf16/f16, "
                                "transpose, (K / group_size) %% 16 == 0");
                return finish_launch(launch_gemm(dtype, a, s), "tensor-core gemm launch");
            }
            if (g_path == QMM_PATH_GEMV)
                return finish_launch(gemv_fast_supported(dtype, a) ? launch_gemv_fast(dtype, a, s)
                                                                    : launch_gemv(dtype, a, s),
                                     "gemv launch");
            return finish_launch(launch_mx_matmul(dtype, a, s), "microscaled matmul launch");
        }
        const bool tc_ok = gemm_supported(dtype, a);
        if (g_path == QMM_PATH_GEMM) {
            if (!tc_ok)
                return fail(QMM_ERR_UNSUPPORTED,
                            "the tensor-core path needs bf16/f16, K %% 64 == 0 and whole 16-byte "
                            "packed rows");
            return finish_launch(launch_gemm(dtype, a, s), "tensor-core gemm launch");
        }
        // Decode shapes of the [N, K] layout (1..4 rows) stream the weight
        // through the SIMT decode kernel where it takes the codes (2/4/8
        // bits), else through the tensor-core GEMM (3/6 bits: ~3x faster than
        // the general SIMT kernel); larger activation counts, and the [K, N]
        // layout at any count, use the GEMM.  The decode tensor-core kernel
        // runs when forced, and for the 2-bit case below.
        if (g_path == QMM_PATH_DECODE_TC) {
            if (!gemv_tc_supported(dtype, a))
                return fail(QMM_ERR_UNSUPPORTED,
                            "the decode tensor-core path needs bf16/f16, transpose, 1..16 rows, 2- or "
                            "4-bit codes, group size 32..128, K %% 512 == 0, (K / group_size) %% 8 == 0, "
                            "16-byte aligned operands");
            if (a.ws == nullptr || a.ws_bytes < gemv_tc_workspace_bytes(a.K))
                return fail(QMM_ERR_WORKSPACE,
                            "the decode tensor-core path needs a workspace of "
                            "qmm_quantized_matmul_workspace_size bytes");
            return finish_launch(launch_gemv_tc(dtype, a, s), "decode tensor-core launch");
        }
        // 2-bit codes, 3..8 rows: the decode tensor-core kernel when the
        // caller gave its workspace (14336 x 4096, 4 rows: 18.0 against
        // 30.9 us on the SIMT decode kernel; 8 rows: 21.6 against 23.6 us on
        // the GEMM).  Elsewhere it is not faster.
        if (g_path == QMM_PATH_AUTO && a.bits == 2 && a.M >= 3 && a.M <= 8 && gemv_tc_supported(dtype, a) &&
            a.ws != nullptr && a.ws_bytes >= gemv_tc_workspace_bytes(a.K))
            return finish_launch(launch_gemv_tc(dtype, a, s), "decode tensor-core launch");
        const bool few_rows = a.M <= kGemvMaxRows && a.transpose;
        if (g_path == QMM_PATH_GEMV || few_rows || !tc_ok) {
            if (gemv_fast_supported(dtype, a))
                return finish_launch(launch_gemv_fast(dtype, a, s), "gemv launch");
            if (g_path == QMM_PATH_GEMV || !tc_ok)
                return finish_launch(launch_gemv(dtype, a, s), "gemv launch");
        }
        return finish_launch(launch_gemm(dtype, a, s), "tensor-core gemm launch");
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_quantized_matmul");
    }
}

}  // namespace

extern "C" {

qmm_status qmm_quantized_matmul_ws(const void *x, int64_t M, int64_t K, const uint32_t *wq,
                                   const void *scales, const void *biases, qmm_dtype dtype,
                                   int64_t N, int transpose, int group_size, int bits,
                                   const char *mode, void *y, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    return matmul_impl(x, M, K, wq, scales, biases, dtype, N, transpose, group_size, bits, mode,
                       nullptr, 0.0, y, workspace, workspace_bytes, stream);
}

qmm_status qmm_quantized_matmul_host(const void *x_host, void *x_dev, int64_t M, int64_t K,
                                     const uint32_t *wq, const void *scales, const void *biases,
                                     qmm_dtype dtype, int64_t N, int transpose, int group_size,
                                     int bits, const char *mode, void *y_dev, void *y_host,
                                     void *workspace, size_t workspace_bytes, void *stream) {
    if ((x_host == nullptr && M > 0 && K > 0) || (y_host == nullptr && M > 0 && N > 0))
        return fail(QMM_ERR_INVALID_ARG, "x_host and y_host must not be NULL");
    return matmul_impl(x_dev, M, K, wq, scales, biases, dtype, N, transpose, group_size, bits, mode,
                       nullptr, 0.0, y_dev, workspace, workspace_bytes, stream,
                       M > 0 && K > 0 ? x_host : nullptr, M > 0 && N > 0 ? y_host : nullptr);
}

qmm_status qmm_quantized_matmul_mapped(const void *x_map, void *x_dev, int64_t M, int64_t K,
                                       const uint32_t *wq, const void *scales, const void *biases,
                                       qmm_dtype dtype, int64_t N, int transpose, int group_size,
                                       int bits, const char *mode, void *y_dev, void *y_map,
                                       void *workspace, size_t workspace_bytes, void *stream) {
    if ((x_map == nullptr && M > 0 && K > 0) || (y_map == nullptr && M > 0 && N > 0))
        return fail(QMM_ERR_INVALID_ARG, "x_map and y_map must not be NULL");
    return matmul_impl(x_dev, M, K, wq, scales, biases, dtype, N, transpose, group_size, bits, mode,
                       nullptr, 0.0, y_dev, workspace, workspace_bytes, stream,
                       M > 0 && K > 0 ? x_map : nullptr, M > 0 && N > 0 ? y_map : nullptr, true);
}

void *qmm_mapped_pointer(const void *host) {
    if (host == nullptr) return nullptr;
    try {
        return const_cast<void *>(mapped_host_pointer(host));
    } catch (...) {
        return nullptr;
    }
}

qmm_status qmm_quantized_dense(const void *x, int64_t M, int64_t K, const uint32_t *wq,
                               const void *scales, const void *biases, qmm_dtype dtype, int64_t N,
                               int transpose, int group_size, int bits, const char *mode,
                               const void *bias, double bias_value, void *y, void *workspace,
                               size_t workspace_bytes, void *stream) {
    return matmul_impl(x, M, K, wq, scales, biases, dtype, N, transpose, group_size, bits, mode,
                       bias, bias_value, y, workspace, workspace_bytes, stream);
}

qmm_status qmm_quantized_matmul(const void *x, int64_t M, int64_t K, const uint32_t *wq,
                                const void *scales, const void *biases, qmm_dtype dtype,
                                int64_t N, int transpose, int group_size, int bits,
                                const char *mode, void *y, void *stream) {
    return qmm_quantized_matmul_ws(x, M, K, wq, scales, biases, dtype, N, transpose, group_size,
                                   bits, mode, y, nullptr, 0, stream);
}

size_t qmm_quantized_matmul_workspace_size(int64_t M, int64_t K, int64_t N, int transpose,
                                           int bits, qmm_dtype dtype) {
    try {
        // The forced decode tensor-core kernel keeps its prepared activations
        // in the workspace; under the automatic path decode shapes go to the
        // SIMT decode kernel, which takes none.
        if (g_path == QMM_PATH_DECODE_TC) {
            if (M < 1 || M > 16 || !transpose || (bits != 2 && bits != 4) ||
                (dtype != QMM_BF16 && dtype != QMM_F16) || K <= 0)
                return 0;
            return gemv_tc_workspace_bytes(K);
        }
        if (g_path == QMM_PATH_AUTO && bits == 2 && M >= 3 && M <= 8 && transpose &&
            (dtype == QMM_BF16 || dtype == QMM_F16) && K > 0 && K % 512 == 0)
            return std::max(gemv_tc_workspace_bytes(K), gemm_workspace_size(dtype, M, K, N, true, bits));
        // 1..4 rows of [N, K]: the streaming decode kernel (no workspace)
        // takes 2-, 4- and 8-bit codes; 3- and 6-bit codes go to the GEMM.
        if (g_path != QMM_PATH_GEMM && M <= kGemvMaxRows && transpose && bits != 3 && bits != 6)
            return 0;
        return gemm_workspace_size(dtype, M, K, N, transpose != 0, bits);
    } catch (...) {
        return 0;
    }
}

size_t qmm_gather_qmm_workspace_size(int64_t batch, int64_t M, int64_t K, int64_t n_experts,
                                     qmm_dtype dtype) {
    // Only the tensor-core path (bf16/f16) uses the workspace.
    if (dtype != QMM_BF16 && dtype != QMM_F16) return 0;
    if (batch <= 0 || M <= 0 || K <= 0 || n_experts <= 0) return 0;
    if (batch > INT32_MAX || M > INT32_MAX || batch * M > INT32_MAX / 2) return 0;
    return gather_ws_layout(batch, M, K, n_experts, 2).total;
}

qmm_status qmm_gather_qmm(const void *x, int64_t x_batch, int64_t M, int64_t K,
                          const uint32_t *wq, const void *scales, const void *biases,
                          qmm_dtype dtype, int64_t n_experts, int64_t N,
                          const int32_t *lhs_indices, const int32_t *rhs_indices, int64_t batch,
                          int transpose, int group_size, int bits, const char *mode,
                          int sorted_indices, void *y, void *workspace, size_t workspace_bytes,
                          void *stream) {
    // sorted_indices is accepted for parity with the upstream signature.  The
    // preparation kernel checks the order of rhs_indices itself and skips the
    // reorder whenever it is already sorted, so the hint is neither needed nor
    // trusted: a wrong hint cannot produce wrong results.
    (void)sorted_indices;
    try {
        int md = QMM_MODE_AFFINE;
        qmm_status st = check_common(dtype, group_size, bits, mode, &md);
        if (st != QMM_OK) return st;
        if (md != QMM_MODE_AFFINE)
            return fail(QMM_ERR_UNSUPPORTED,
                        "gather_qmm takes affine weights (its callers pass mode \"affine\")");
        if (batch < 0 || x_batch < 1 || n_experts < 1 || M < 0 || N < 0 || K <= 0)
            return fail(QMM_ERR_INVALID_ARG,
                        "need batch >= 0, x_batch >= 1, n_experts >= 1, M >= 0, N >= 0, K > 0");
        // (An empty batch has nothing to index: its index arrays may be NULL.)
        if (batch > 0 && lhs_indices == nullptr && x_batch != 1 && x_batch != batch)
            return fail(QMM_ERR_INVALID_ARG,
                        "without lhs_indices, x_batch (%lld) must be 1 or batch (%lld)",
                        (long long)x_batch, (long long)batch);
        if (batch > 0 && rhs_indices == nullptr && n_experts != 1 && n_experts != batch)
            return fail(QMM_ERR_INVALID_ARG,
                        "without rhs_indices, n_experts (%lld) must be 1 or batch (%lld)",
                        (long long)n_experts, (long long)batch);
        if (batch > INT32_MAX || M > INT32_MAX || batch * M > INT32_MAX / 2)
            return fail(QMM_ERR_UNSUPPORTED, "batch * M must stay below 2^30 rows");
        // Sizes always; pointers only when there is work (empty tensors may be NULL).
        st = check_matmul(x, batch == 0 ? 0 : M, K, wq, scales, biases, N, transpose, group_size, y);
        if (st != QMM_OK) return st;
        if (batch == 0 || M == 0 || N == 0) return QMM_OK;
        if (lhs_indices != nullptr && (reinterpret_cast<uintptr_t>(lhs_indices) & 3u))
            return fail(QMM_ERR_INVALID_ARG, "lhs_indices is not 4-byte aligned");
        if (rhs_indices != nullptr && (reinterpret_cast<uintptr_t>(rhs_indices) & 3u))
            return fail(QMM_ERR_INVALID_ARG, "rhs_indices is not 4-byte aligned");
        cudaStream_t s = (cudaStream_t)stream;
        const GatherIndex gi{lhs_indices, rhs_indices, batch, x_batch, n_experts};

        const bool tc_ok = gather_tc_supported(dtype, x_batch, M, K, N, n_experts, batch, bits,
                                               transpose);
        if (g_path == QMM_PATH_GEMM && !tc_ok)
            return fail(QMM_ERR_UNSUPPORTED,
                        "the tensor-core gather path needs bf16/f16, transpose, K %% 64 == 0");
        if (tc_ok && g_path != QMM_PATH_GEMV) {
            const size_t need = qmm_gather_qmm_workspace_size(batch, M, K, n_experts, dtype);
            if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u))
                return fail(QMM_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
            if (workspace_bytes < need)
                return fail(QMM_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu",
                            workspace_bytes, need);
            GatherCall c{};
            c.x = x;
            c.M = M;
            c.K = K;
            c.N = N;
            c.wq = wq;
            c.scales = scales;
            c.biases = biases;
            c.gi = gi;
            c.transpose = transpose != 0;
            c.group_size = group_size;
            c.bits = bits;
            c.y = y;
            c.workspace = workspace;
            return finish_launch(launch_gather_tc(dtype, c, s), "gather_qmm tensor-core launch");
        }
        QmmArgs a{x, wq, scales, biases, y, M, N, K, group_size, bits, transpose != 0};
        return finish_launch(launch_gemv_gather(dtype, a, gi, s), "gather_qmm launch");
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_gather_qmm");
    }
}

// qqmm workspace: the quantized activations (codes, scale bytes) and their
// exact dequantized copy, each piece 256-byte aligned.
struct QqmmWorkspace {
    size_t xq, xs, xd, total;
};
static QqmmWorkspace qqmm_layout(int64_t M, int64_t K, int group_size, int bits, qmm_dtype dt) {
    auto up = [](size_t v) { return (v + 255) & ~(size_t)255; };
    QqmmWorkspace w{};
    w.xq = 0;
    w.xs = up((size_t)M * (size_t)(K * bits / 32) * 4);
    w.xd = w.xs + up((size_t)M * (size_t)(K / group_size));
    w.total = w.xd + up((size_t)M * (size_t)K * (dt == QMM_F32 ? 4 : 2));
    return w;
}

size_t qmm_qqmm_workspace_size(int64_t M, int64_t K, int group_size, int bits, qmm_dtype dtype) {
    if (M <= 0 || K <= 0 || (group_size != 16 && group_size != 32) || K % group_size) return 0;
    if (dtype != QMM_F32 && dtype != QMM_BF16 && dtype != QMM_F16) return 0;
    return qqmm_layout(M, K, group_size, bits, dtype).total;
}

qmm_status qmm_qqmm(const void *x, int64_t M, int64_t K, qmm_dtype dtype, const uint32_t *wq,
                    const void *w_scales, int64_t N, int group_size, int bits, const char *mode,
                    void *y, void *workspace, size_t workspace_bytes, void *stream) {
    try {
        int md = QMM_MODE_AFFINE;
        qmm_status st = check_common(dtype, group_size, bits, mode, &md);
        if (st != QMM_OK) return st;
        if (md != QMM_MODE_NVFP4 && md != QMM_MODE_MXFP8)
            return fail(QMM_ERR_UNSUPPORTED, "qqmm supports modes \"nvfp4\" and \"mxfp8\"");
        st = check_matmul(x, M, K, wq, w_scales, nullptr, N, 1, group_size, y, md);
        if (st != QMM_OK) return st;
        if (M == 0 || N == 0) return QMM_OK;
        const QqmmWorkspace L = qqmm_layout(M, K, group_size, bits, dtype);
        if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return fail(QMM_ERR_WORKSPACE, "workspace must be a 256-byte aligned device buffer");
        if (workspace_bytes < L.total)
            return fail(QMM_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
        cudaStream_t s = (cudaStream_t)stream;
        char *ws = static_cast<char *>(workspace);
        uint32_t *xq = reinterpret_cast<uint32_t *>(ws + L.xq);
        void *xs = ws + L.xs, *xd = ws + L.xd;
        // 1. the activations quantized in the weight's mode (rows of x, groups
        //    along K), 2. their exact dequantized values, 3. the product with
        //    the quantized weight.
        QuantArgs qa{x, M, K, group_size, bits, xq, xs, nullptr, md};
        cudaError_t e = launch_quantize_mx(dtype, qa, s);
        if (e != cudaSuccess) return cuda_fail(e, "qqmm: quantize the activations");
        DequantArgs da{xq, xs, nullptr, M, K, group_size, bits, xd, md};
        e = launch_dequantize_mx(dtype, da, s);
        if (e != cudaSuccess) return cuda_fail(e, "qqmm: dequantize the activations");
        QmmArgs a{xd, wq, w_scales, nullptr, y, M, N, K, group_size, bits, true};
        a.mode = md;
        return finish_launch(launch_mx_matmul(dtype, a, s), "qqmm product launch");
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_qqmm");
    }
}

qmm_status qmm_gather_qmm_static(const void *x, int64_t x_batch, int64_t M, int64_t K,
                                 const uint32_t *wq, const void *scales, const void *biases,
                                 qmm_dtype dtype, int64_t n_experts, int64_t N,
                                 const int32_t *lhs_indices, const int32_t *rhs_indices,
                                 int64_t batch, int transpose, int group_size, int bits,
                                 const char *mode, int sorted_indices, void *y, void *stream) {
    try {
        // Only the tensor-core path uses the scratch; the size limit applies
        // to calls that take it.  (Invalid sizes are left to qmm_gather_qmm.)
        const bool sizes_ok = batch >= 0 && x_batch >= 1 && n_experts >= 1 && M >= 0 && N >= 0 &&
                              K > 0 && batch <= INT32_MAX && M <= INT32_MAX &&
                              batch * M <= INT32_MAX / 2;
        if (sizes_ok && g_path != QMM_PATH_GEMV &&
            gather_tc_supported(dtype, x_batch, M, K, N, n_experts, batch, bits, transpose)) {
            const size_t need = qmm_gather_qmm_workspace_size(batch, M, K, n_experts, dtype);
            if (need > QMM_GATHER_STATIC_SCRATCH_BYTES)
                return fail(QMM_ERR_WORKSPACE,
                            "this call needs %zu bytes of scratch; the built-in scratch holds %u "
                            "(call qmm_gather_qmm with a workspace instead)",
                            need, (unsigned)QMM_GATHER_STATIC_SCRATCH_BYTES);
        }
        void *scratch = nullptr;
        const cudaError_t e = gather_static_scratch(&scratch);
        if (e != cudaSuccess) return cuda_fail(e, "look up the built-in gather scratch");
        return qmm_gather_qmm(x, x_batch, M, K, wq, scales, biases, dtype, n_experts, N,
                              lhs_indices, rhs_indices, batch, transpose, group_size, bits, mode,
                              sorted_indices, y, scratch, QMM_GATHER_STATIC_SCRATCH_BYTES, stream);
    } catch (...) {
        return fail(QMM_ERR_CUDA, "unexpected exception in qmm_gather_qmm_static");
    }
}

qmm_status qmm_device_status(void *stream, int reset) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int word = 0;
    e = cudaMemcpyFromSymbol(&word, g_qmm_state, sizeof(int), offsetof(DeviceState, error));
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (reset && word != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_qmm_state, &zero, sizeof(int), offsetof(DeviceState, error));
        if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    }
    if (word == QMM_ERR_TIMEOUT) return fail(QMM_ERR_TIMEOUT, "a kernel's bounded wait timed out");
    if (word == QMM_ERR_INDEX) return fail(QMM_ERR_INDEX, "an index was out of range");
    if (word != 0) return fail((qmm_status)word, "device error word %d", word);
    return QMM_OK;
}

qmm_status qmm_set_wait_limit_ns(uint64_t ns) {
    if (ns == 0) ns = kDefaultWaitNs;
    const unsigned long long v = ns;
    const cudaError_t e = cudaMemcpyToSymbol(g_qmm_state, &v, sizeof(v), offsetof(DeviceState, wait_ns));
    if (e != cudaSuccess) return cuda_fail(e, "set the wait limit");
    return QMM_OK;
}

qmm_status qmm_inject_fault(qmm_fault fault) {
    if (fault != QMM_FAULT_NONE && fault != QMM_FAULT_STREAMK_NO_PUBLISH)
        return fail(QMM_ERR_INVALID_ARG, "unknown fault %d", (int)fault);
    g_fault.store((int)fault, std::memory_order_relaxed);
    return QMM_OK;
}

qmm_status qmm_set_path(qmm_path path) {
    if (path != QMM_PATH_AUTO && path != QMM_PATH_GEMV && path != QMM_PATH_GEMM &&
        path != QMM_PATH_DECODE_TC)
        return fail(QMM_ERR_INVALID_ARG, "unknown path %d", (int)path);
    g_path = path;
    return QMM_OK;
}

const char *qmm_status_string(qmm_status s) {
    switch (s) {
    case QMM_OK: return "QMM_OK";
    case QMM_ERR_INVALID_ARG: return "QMM_ERR_INVALID_ARG";
    case QMM_ERR_UNSUPPORTED: return "QMM_ERR_UNSUPPORTED";
    case QMM_ERR_CUDA: return "QMM_ERR_CUDA";
    case QMM_ERR_TIMEOUT: return "QMM_ERR_TIMEOUT";
    case QMM_ERR_INDEX: return "QMM_ERR_INDEX";
    case QMM_ERR_WORKSPACE: return "QMM_ERR_WORKSPACE";
    }
    return "QMM_ERR_UNKNOWN";
}

uint64_t qmm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *qmm_last_error(void) { return t_last_error.c_str(); }

int qmm_version(void) { return 100; }

}  // extern "C"
