// qmm_internal.cuh -- shared device helpers and launcher declarations for the
// libqmm CUDA sources (sm_100a).  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qmm.h"

namespace qmm {

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

// Device-side error word (QMM_OK when clear), defined in api.cu.  Kernels
// that can fail receive its device address (device_error_word()) and set it
// with atomicCAS so that the first error recorded wins.
__device__ __forceinline__ void record_device_error(int *word, int code) {
    atomicCAS(word, 0, code);
}
int *device_error_word();  // host: device address of the word (current device)

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
};
cudaError_t launch_quantize(qmm_dtype dt, const QuantArgs &a, cudaStream_t s);

struct DequantArgs {
    const uint32_t *wq;
    const void *scales, *biases;
    int64_t rows, cols;
    int group_size, bits;
    void *out;
};
cudaError_t launch_dequantize(qmm_dtype dt, const DequantArgs &a, cudaStream_t s);

// One (possibly batched) quantized product.  Rows of x and y are addressed
// through optional row maps so that gather_qmm can reuse the same kernels:
//   activation row i of problem p reads  x + x_row(p, i) * K
//   and writes                           y + y_row(p, i) * N
struct QmmArgs {
    const void *x;       // [*, K]
    const uint32_t *wq;  // packed weight of this problem
    const void *scales, *biases;
    void *y;             // [*, N]
    int64_t M, N, K;
    int group_size, bits;
    bool transpose;
};
cudaError_t launch_gemv(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
bool gemv_supported(qmm_dtype dt, const QmmArgs &a);
cudaError_t launch_gemv_fast(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
bool gemv_fast_supported(qmm_dtype dt, const QmmArgs &a);
cudaError_t launch_gemm(qmm_dtype dt, const QmmArgs &a, cudaStream_t s);
bool gemm_supported(qmm_dtype dt, const QmmArgs &a);

int num_sms();
void count_launches(int n);  // bump the process-wide launch counter

}  // namespace qmm
