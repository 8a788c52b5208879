// mx.cu -- quantize and dequantize in the microscaled modes (Emily.QuantizedWeight,
// section Microscaled modes; EMLX.Quantization, sections quantize and dequantize,
// which accept every mode): per group of 32 (mxfp4, mxfp8) or 16 (nvfp4)
// consecutive elements along the last axis, one scale byte and 32/bits codes
// per uint32 word, least significant first; no biases.
//
// Scale rule (OCP Microscaling Formats v1.0, conversion to MX; NVIDIA NVFP4):
//   mx    X = 2^(floor(log2 max|v|) - emax), emax = 2 (E2M1) or 8 (E4M3),
//         clamped to E8M0's range, stored as the byte floor(log2 X) + 127;
//         elements v * 2^-(floor(log2 X)) in E2M1 / E4M3;
//   nvfp4 X = max|v| / 6 rounded to E4M3 (the byte), elements v / X in E2M1;
// element conversions round to nearest-even and saturate (hardware cvt);
// an all-zero group stores zeros.  HBM-bound: one thread per group.
#include "mx.cuh"
#include "qmm_internal.cuh"

namespace qmm {
namespace {

template <int MODE> struct MxGeom;
template <> struct MxGeom<QMM_MODE_MXFP4> { static constexpr int GS = 32, BITS = 4, EMAX = 2; };
template <> struct MxGeom<QMM_MODE_MXFP8> { static constexpr int GS = 32, BITS = 8, EMAX = 8; };
template <> struct MxGeom<QMM_MODE_NVFP4> { static constexpr int GS = 16, BITS = 4; };  // scale from amax / 6

// floor(log2 a) of a finite a > 0 from its bits (subnormals included).
__device__ __forceinline__ int ilog2f(float a) {
    const uint32_t u = __float_as_uint(a);
    const int e = (int)((u >> 23) & 0xFFu);
    return e != 0 ? e - 127 : (31 - __clz((int)u)) - 149;
}

template <typename T, int N>
__device__ __forceinline__ void load_group(const T *src, float (&v)[N]) {
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 f = *reinterpret_cast<const float4 *>(src + i);
            v[i] = f.x;
            v[i + 1] = f.y;
            v[i + 2] = f.z;
            v[i + 3] = f.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            const uint4 u = *reinterpret_cast<const uint4 *>(src + i);
            const T *h = reinterpret_cast<const T *>(&u);
#pragma unroll
            for (int j = 0; j < 8; ++j) v[i + j] = Dt<T>::to_f(h[j]);
        }
    }
}

template <typename T, int MODE>
__global__ void __launch_bounds__(256)
quantize_mx_kernel(const T *__restrict__ w, int64_t groups, uint32_t *__restrict__ wq,
                   uint8_t *__restrict__ scales) {
    using G = MxGeom<MODE>;
    constexpr int GS = G::GS, WPG = GS * G::BITS / 32;  // words per group
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= groups) return;
    float v[GS];
    load_group<T, GS>(w + gid * GS, v);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < GS; ++i) amax = fmaxf(amax, fabsf(v[i]));
    uint32_t scode = 0;
    bool zero = true;
    if constexpr (MODE == QMM_MODE_NVFP4) {
        const float s32 = __fdiv_rn(amax, 6.0f);
        const float four[4] = {s32, s32, s32, s32};
        scode = mxf::e4m3x4(four) & 0xFFu;  // (the first of the four codes)
        const float sdq = mxf::scale_value<MODE>(scode);
        zero = !(sdq != 0.f);
#pragma unroll
        for (int i = 0; i < GS; ++i) v[i] = zero ? 0.f : __fdiv_rn(v[i], sdq);
    } else {
        zero = !(amax > 0.f);
        if (!zero) {
            const int shared = min(127, max(-127, ilog2f(amax) - G::EMAX));
            scode = (uint32_t)(shared + 127);
            const float mult = __uint_as_float((uint32_t)(127 - shared) << 23);  // 2^-shared
#pragma unroll
            for (int i = 0; i < GS; ++i) v[i] = __fmul_rn(v[i], mult);
        }
    }
    uint32_t out[WPG];
#pragma unroll
    for (int k = 0; k < WPG; ++k) {
        if constexpr (G::BITS == 8) out[k] = zero ? 0u : mxf::e4m3x4(v + 4 * k);
        else out[k] = zero ? 0u : mxf::e2m1x8(v + 8 * k);
    }
    uint32_t *dst = wq + gid * WPG;
    if constexpr (WPG == 2) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(out[0], out[1]);
    } else {
#pragma unroll
        for (int k = 0; k < WPG; k += 4)
            *reinterpret_cast<uint4 *>(dst + k) = make_uint4(out[k], out[k + 1], out[k + 2], out[k + 3]);
    }
    scales[gid] = (uint8_t)scode;
}

// One thread per packed word: its 32/bits elements times the group's scale
// value (exact in fp32), rounded to the output dtype.
template <typename T, int MODE>
__global__ void __launch_bounds__(256)
dequantize_mx_kernel(const uint32_t *__restrict__ wq, const uint8_t *__restrict__ scales,
                     int64_t words, T *__restrict__ out) {
    using G = MxGeom<MODE>;
    constexpr int EPW = 32 / G::BITS;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= words) return;
    const float x = mxf::scale_value<MODE>(scales[i * EPW / G::GS]);
    float e[EPW];
    mxf::elements<MODE>(wq[i], e);
    T r[EPW];
#pragma unroll
    for (int j = 0; j < EPW; ++j) r[j] = Dt<T>::from_f(__fmul_rn(x, e[j]));
    T *dst = out + i * EPW;
#pragma unroll
    for (int j = 0; j < EPW; ++j) dst[j] = r[j];
}

template <typename T, int MODE>
cudaError_t quantize_mx_t(const QuantArgs &a, cudaStream_t s) {
    const int64_t groups = a.rows * (a.cols / MxGeom<MODE>::GS);
    const int64_t blocks = (groups + 255) / 256;
    quantize_mx_kernel<T, MODE><<<(unsigned)blocks, 256, 0, s>>>(
        static_cast<const T *>(a.w), groups, a.wq, static_cast<uint8_t *>(a.scales));
    count_launches(1);
    return cudaGetLastError();
}

template <typename T, int MODE>
cudaError_t dequantize_mx_t(const DequantArgs &a, cudaStream_t s) {
    const int64_t words = a.rows * a.cols * MxGeom<MODE>::BITS / 32;
    const int64_t blocks = (words + 255) / 256;
    dequantize_mx_kernel<T, MODE><<<(unsigned)blocks, 256, 0, s>>>(
        a.wq, static_cast<const uint8_t *>(a.scales), words, static_cast<T *>(a.out));
    count_launches(1);
    return cudaGetLastError();
}

template <typename T>
cudaError_t quantize_mx_dtype(const QuantArgs &a, cudaStream_t s) {
    switch (a.mode) {
    case QMM_MODE_MXFP4: return quantize_mx_t<T, QMM_MODE_MXFP4>(a, s);
    case QMM_MODE_MXFP8: return quantize_mx_t<T, QMM_MODE_MXFP8>(a, s);
    default: return quantize_mx_t<T, QMM_MODE_NVFP4>(a, s);
    }
}

template <typename T>
cudaError_t dequantize_mx_dtype(const DequantArgs &a, cudaStream_t s) {
    switch (a.mode) {
    case QMM_MODE_MXFP4: return dequantize_mx_t<T, QMM_MODE_MXFP4>(a, s);
    case QMM_MODE_MXFP8: return dequantize_mx_t<T, QMM_MODE_MXFP8>(a, s);
    default: return dequantize_mx_t<T, QMM_MODE_NVFP4>(a, s);
    }
}

}  // namespace

cudaError_t launch_quantize_mx(qmm_dtype dt, const QuantArgs &a, cudaStream_t s) {
    if (a.rows * (a.cols / 16) > (int64_t)UINT32_MAX * 256) return cudaErrorInvalidValue;
    switch (dt) {
    case QMM_F32: return quantize_mx_dtype<float>(a, s);
    case QMM_BF16: return quantize_mx_dtype<__nv_bfloat16>(a, s);
    default: return quantize_mx_dtype<__half>(a, s);
    }
}

cudaError_t launch_dequantize_mx(qmm_dtype dt, const DequantArgs &a, cudaStream_t s) {
    if (a.rows * a.cols / 4 > (int64_t)UINT32_MAX * 256) return cudaErrorInvalidValue;
    switch (dt) {
    case QMM_F32: return dequantize_mx_dtype<float>(a, s);
    case QMM_BF16: return dequantize_mx_dtype<__nv_bfloat16>(a, s);
    default: return dequantize_mx_dtype<__half>(a, s);
    }
}

}  // namespace qmm
