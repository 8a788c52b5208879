// qmm_internal.cuh -- shared device helpers and launcher declarations for the
// libqmm CUDA sources (sm_100a).  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qmm.h"

namespace qmm {

// Quantization modes (the `mode` string of the C ABI).
enum QmmMode { QMM_MODE_AFFINE = 0, QMM_MODE_MXFP4 = 1, QMM_MODE_MXFP8 = 2, QMM_MODE_NVFP4 = 3 };

// ---------------------------------------------------------------------------
// Storage dtypes: fp32 <-> T conversions, round-to-nearest-even on the way in.
// ---------------------------------------------------------------------------
template <typename T> struct Dt;
template <> struct Dt<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Dt<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};
template <> struct Dt<__half> {
    static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
    static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
};

// Device-side state of the library, one per device, defined in api.cu:
// the error word (QMM_OK when clear) and the limit of the bounded waits.
// Kernels that can fail receive the address of the error word
// (device_error_word()), set it with atomicCAS so that the first error
// recorded wins, and find the wait limit beside it.
struct DeviceState {
    int error;
    int pad;
    unsigned long long wait_ns;  // limit of a bounded wait on another party
};
__device__ __forceinline__ void record_device_error(int *word, int code) {
    atomicCAS(word, 0, code);
}
// Limit of a bounded wait, read only once a wait has not completed at once.
__device__ __forceinline__ unsigned long long wait_limit_ns(const int *word) {
    return *reinterpret_cast<const volatile unsigned long long *>(
        reinterpret_cast<const char *>(word) + offsetof(DeviceState, wait_ns));
}
int *device_error_word();  // host: device address of the error word (current device)
// Leading bytes of a matmul workspace that every call leaves zero (the
// stream-K ready flags); other users of the workspace start past them.
constexpr size_t kWsFlagBytes = 4096;
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;  // 2 s

// Host-side test injection (qmm_inject_fault); read when a launch is built.
int injected_fault();

// Host: the current device (-1 if the runtime cannot say).
int current_device();

// Host: apply a kernel's launch attributes once per device and per requested
// dynamic shared-memory size, instead of on every call.  `apply` performs the
// cudaFuncSetAttribute calls (and any check) for `smem` bytes; its result is
// remembered only on success.
template <typename Tag, typename Fn>
cudaError_t configure_once(size_t smem, Fn &&apply) {
    static std::mutex mu;
    static size_t done[64] = {0};
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return apply();
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev] >= smem && done[dev] != 0) return cudaSuccess;
    const cudaError_t e = apply();
    if (e == cudaSuccess) done[dev] = std::max(done[dev], smem);
    return e;
}

// ---------------------------------------------------------------------------
// Launchers (host).  Each returns cudaSuccess or the launch error.  Arguments
// have been validated by the ABI layer.
// ---------------------------------------------------------------------------
struct QuantArgs {
    const void *w;
    int64_t rows, cols;
    int group_size, bits;
    uint32_t *wq;
    void *scales, *biases;
    int mode = QMM_MODE_AFFINE;  // microscaled: scales are bytes, no biases
};
cudaError_t launch_quantize(qmm_dtype dt, const QuantArgs &a, cudaStream_t s);
cudaError_t launch_quantize_mx(qmm_dtype dt, const QuantArgs &a, cudaStream_t s);

struct DequantArgs {
    const uint32_t *wq;
    const void *scales, *biases;
    int64_t rows, cols;
    int group_size, bits;
    void *out;
    int mode = QMM_MODE_AFFINE;
};
cudaError_t launch_dequantize(qmm_dtype dt, const DequantArgs &a, cudaStream_t s);
cudaError_t launch_dequantize_mx(qmm_dtype dt, const DequantArgs &a, cudaStream_t s);

// One quantized product y[M, N] = x[M, K] (*) W.
struct QmmArgs {
    const void *x;       // [*, K]
    const uint32_t *wq;  // packed weight of this problem
    const void *scales, *biases;
    void *y;             // [*, N]
    int64_t M, N, K;
    int group_size, bits;
    bool transpose;
    void *ws = nullptr;  // stream-K workspace (zeroed flags first), or null
    size_t ws_bytes = 0;
    // Layer bias added before the output is rounded (quantized_dense):
    // y[m, n] += bias[n] (if bias) + bias_value.
    const void *bias = nullptr;
    float bias_value = 0.f;
    int mode = QMM_MODE_AFFINE;  // microscaled: scales are bytes, biases null
    // A second destination for the result (the device mapping of page-locked
    // host memory, [*, N]), or null.  Kernels that can write it in their
    // epilogue set y2_written; otherwise the caller copies y there.
    void *y2 = nullptr;
    mutable bool y2_written = false;
};

// Bias term of output feature n: bias[n] (if any) plus the scalar.
template <typename T>
__device__ __forceinline__ float layer_bias(const void *bias, float value, int64_t n) {
    return bias ? Dt<T>::to_f(static_cast<const T *>(bias)[n]) + value : value;
}
cudaError_t launch_gemv(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
bool gemv_supported(qmm_dtype dt, const QmmArgs &a);
cudaError_t launch_gemv_fast(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
bool gemv_fast_supported(qmm_dtype dt, const QmmArgs &a);
cudaError_t launch_gemv_tc(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
bool gemv_tc_supported(qmm_dtype dt, const QmmArgs &a);
size_t gemv_tc_workspace_bytes(int64_t K);
// Copies for qmm_quantized_matmul_host (copy.cu): the device address of a
// page-locked host pointer (nullptr if it is not page-locked), and a copy
// kernel chained by programmatic dependent launch.
const void *mapped_host_pointer(const void *p);
cudaError_t launch_mapped_copy(const void *src, void *dst, size_t bytes, cudaStream_t s);
cudaError_t launch_gemm(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
cudaError_t launch_mx_matmul(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);  // microscaled weights
// Bytes of stream-K workspace the tensor-core path can use for these sizes
// (0 when it would keep whole tiles).
size_t gemm_workspace_size(qmm_dtype dt, int64_t M, int64_t K, int64_t N, bool transpose, int bits);
bool gemm_supported(qmm_dtype dt, const QmmArgs &a);

// ---------------------------------------------------------------------------
// gather_qmm
// ---------------------------------------------------------------------------
// Batch entry b uses activations x[xi(b)] and expert ei(b):
//   xi = lhs ? lhs[b] : (x_batch == 1 ? 0 : b),  ei = rhs ? rhs[b] : (n_experts == 1 ? 0 : b).
// An entry whose xi or ei is out of range is "invalid": its output rows are
// zero and the device error word gets QMM_ERR_INDEX.
struct GatherIndex {
    const int32_t *lhs, *rhs;  // nullable
    int64_t batch, x_batch, n_experts;
};

__device__ __forceinline__ bool gather_entry(const GatherIndex &gi, int64_t b, int64_t &xi,
                                             int64_t &ei) {
    xi = gi.lhs ? (int64_t)__ldg(gi.lhs + b) : (gi.x_batch == 1 ? 0 : b);
    ei = gi.rhs ? (int64_t)__ldg(gi.rhs + b) : (gi.n_experts == 1 ? 0 : b);
    return xi >= 0 && xi < gi.x_batch && ei >= 0 && ei < gi.n_experts;
}

// Header the preparation kernel writes at the start of the workspace.
struct GatherHeader {
    int num_chunks;     // entries of the chunk table
    int use_x;          // 1: the sorted row order is x's own, read x directly
    int valid_entries;  // batch entries with in-range indices (sorted first)
    int pad;
};

// SIMT batched path (any dtype, either layout): one product per entry.
cudaError_t launch_gemv_gather(qmm_dtype dt, const QmmArgs &a, const GatherIndex &gi, cudaStream_t s);

// Grouped tensor-core product over rows sorted by expert.
struct GroupedArgs {
    const void *x;           // [x_rows = x_batch * M, K]
    const void *x_sorted;    // [rows, K] (workspace)
    const uint32_t *wq;      // [n_experts * N, K * bits / 32]
    const void *scales, *biases;
    void *y;                 // [batch * M, N]
    int64_t x_rows, rows, N, K, n_experts, max_chunks;
    int group_size, bits;
    bool transpose;
    int chunk_rows;          // 64, 128 or 256: rows per chunk at most
    const GatherHeader *hdr;
    const int4 *chunks;
    const int32_t *dst_rows;
};
bool gemm_grouped_supported(qmm_dtype dt, const GroupedArgs &g);
cudaError_t launch_gemm_grouped(qmm_dtype dt, const GroupedArgs &g, cudaStream_t s);

// Byte offsets of the tensor-core path's pieces in the caller's workspace
// (each 256-byte aligned), and the total size.
struct GatherWorkspace {
    size_t hdr, chunks, perm, dst_rows, x_sorted, total;
    int64_t max_chunks;
};
GatherWorkspace gather_ws_layout(int64_t batch, int64_t M, int64_t K, int64_t n_experts,
                                 int elt_bytes);
int gather_chunk_rows(int64_t rows);       // tile width (64/128/256) for `rows` sorted rows
bool gather_prep_fits(int64_t n_experts);  // the sort's histograms fit shared memory

struct GatherCall {
    const void *x;  // [x_batch, M, K]
    int64_t M, K, N;
    const uint32_t *wq;
    const void *scales, *biases;
    GatherIndex gi;
    bool transpose;
    int group_size, bits;
    void *y;  // [batch, M, N]
    void *workspace;
};
cudaError_t launch_gather_tc(qmm_dtype dt, const GatherCall &c, cudaStream_t s);
// Device address of the built-in scratch (QMM_GATHER_STATIC_SCRATCH_BYTES) on
// the current device; looked up on the first call per device.
cudaError_t gather_static_scratch(void **ptr);

int num_sms();
void count_launches(int n);  // bump the process-wide launch counter

}  // namespace qmm
