// quantize.cu -- group-wise affine quantize and dequantize (sm_100a).
//
// Quantization runs along the last axis, one scale and one bias per
// `group_size` consecutive elements, `bits`-bit codes packed 32/bits per
// uint32 least-significant first (3- and 6-bit codes: back to back in the
// row's bit stream, see quantize_chunk_kernel) (EMLX.Quantization, section quantize;
// Emily.QuantizedWeight, section Layout; mlx-rs ops/quantization.rs,
// quantize / dequantize).
//
// Both kernels are HBM-bound streams with 16-byte vector loads and stores
// (quantize: a thread per 16 bytes of codes; dequantize: a thread per packed
// word), and the group min/max reduced across the lanes that share a group
// with warp shuffles.  Every floating-point step uses an explicitly rounded
// intrinsic so the result is bit-identical to a sequential IEEE fp32
// evaluation of the same rule.
#include <algorithm>
#include <type_traits>

#include "ptx_sm100.cuh"
#include "qmm_internal.cuh"

namespace qmm {

namespace {

template <typename T, int N>
__device__ __forceinline__ void load_elems(const T *__restrict__ p, float (&v)[N]) {
    constexpr int BYTES = N * (int)sizeof(T);
    if constexpr (BYTES % 16 == 0) {
        constexpr int NV = BYTES / 16;
        uint4 raw[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) raw[i] = __ldg(reinterpret_cast<const uint4 *>(p) + i);
        const T *t = reinterpret_cast<const T *>(raw);
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = Dt<T>::to_f(t[i]);
    } else {
        static_assert(BYTES == 8, "unexpected vector width");
        uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p));
        const T *t = reinterpret_cast<const T *>(&raw);
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = Dt<T>::to_f(t[i]);
    }
}

template <typename T, int N>
__device__ __forceinline__ void store_elems(T *__restrict__ p, const T (&t)[N]) {
    constexpr int BYTES = N * (int)sizeof(T);
    if constexpr (BYTES % 16 == 0) {
        constexpr int NV = BYTES / 16;
#pragma unroll
        for (int i = 0; i < NV; ++i)
            reinterpret_cast<uint4 *>(p)[i] = reinterpret_cast<const uint4 *>(t)[i];
    } else {
        static_assert(BYTES == 8, "unexpected vector width");
        *reinterpret_cast<uint2 *>(p) = *reinterpret_cast<const uint2 *>(t);
    }
}

// The codes of two elements: rint((v - b) / s) clamped to [0, QMAX], with
// the quotient correctly rounded (IEEE division) as the rule states.  A
// product with the rounded reciprocal differs from that quotient by at most a
// couple of units in the last place, which can change rint only next to a
// half integer; the exact division runs there, so the result is the
// division's in every case.  Clamping before rounding gives the same code
// (outside [0, QMAX] both quotients end on the boundary code) and keeps the
// value in the range where adding and subtracting 1.5 * 2^23 rounds it to an
// integer (ties to even) and the sum's low bits hold that integer: full-rate
// arithmetic, no conversion instructions, and the subtractions, products and
// adds two lanes per instruction.  A NaN quotient gives code 0.
__device__ __forceinline__ void code_pair(float v0, float v1, float b, float s, float r, float qmax,
                                          uint32_t &c0, uint32_t &c1) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    using namespace ptx;
    const unsigned long long mm = f2pack(kMagic, kMagic);
    const unsigned long long t = f2sub(f2pack(v0, v1), f2pack(b, b));
    float y0, y1;
    f2unpack(f2mul(t, f2pack(r, r)), y0, y1);
    const unsigned long long y = f2pack(fminf(fmaxf(y0, 0.f), qmax), fminf(fmaxf(y1, 0.f), qmax));
    const unsigned long long a = f2add(y, mm);
    float d0, d1, a0, a1;
    f2unpack(f2sub(y, f2sub(a, mm)), d0, d1);
    f2unpack(a, a0, a1);
    if (fabsf(d0) > 0.499f || fabsf(d1) > 0.499f) {  // next to a half integer: divide
        float t0, t1;
        f2unpack(t, t0, t1);
        if (fabsf(d0) > 0.499f) a0 = __fadd_rn(fminf(fmaxf(__fdiv_rn(t0, s), 0.f), qmax), kMagic);
        if (fabsf(d1) > 0.499f) a1 = __fadd_rn(fminf(fmaxf(__fdiv_rn(t1, s), 0.f), qmax), kMagic);
    }
    c0 = __float_as_uint(a0) - 0x4B400000u;
    c1 = __float_as_uint(a1) - 0x4B400000u;
}

// One thread per WPT packed words (16 bytes of codes when a group holds that
// many); `tpg` = threads per group (a power of two <= 32), so the lanes of one
// group are contiguous and aligned within the warp.
// 16-bit elements with 4- or 8-bit codes fit 40 registers: six CTAs per SM.
template <typename T, int BITS, int WPT>
__global__ void __launch_bounds__(256, (sizeof(T) == 2 && BITS >= 4) ? 6 : 1)
quantize_kernel(const T *__restrict__ w, int64_t n_threads, int tpg,
                uint32_t *__restrict__ wq, T *__restrict__ scales, T *__restrict__ biases) {
    constexpr int EPW = 32 / BITS;
    constexpr int NE = EPW * WPT;  // elements per thread
    constexpr int QMAX = (1 << BITS) - 1;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool valid = tid < n_threads;

    // 16-bit elements stay packed two per register (half the registers of
    // fp32 copies: more threads per SM) and the group's min and max are taken
    // on the pairs with packed 16-bit min/max (exact selections, NaN-ignoring
    // like fminf/fmaxf); each pair is widened to fp32 only to form its codes.
    constexpr bool kPacked = sizeof(T) == 2;
    constexpr int NV = kPacked ? 1 : NE;
    constexpr int NR = kPacked ? NE / 2 : 1;
    float v[NV];
    uint32_t raw[NR];
    float lo, hi;
    if constexpr (kPacked) {
        using V2 = typename std::conditional<std::is_same<T, __half>::value, __half2, __nv_bfloat162>::type;
#pragma unroll
        for (int i = 0; i < NR; i += 4) {
            const uint4 u = valid ? __ldg(reinterpret_cast<const uint4 *>(w + tid * NE) + i / 4) : make_uint4(0, 0, 0, 0);
            raw[i] = u.x; raw[i + 1] = u.y; raw[i + 2] = u.z; raw[i + 3] = u.w;
        }
        V2 mn = *reinterpret_cast<const V2 *>(&raw[0]), mx = mn;
#pragma unroll
        for (int i = 1; i < NR; ++i) {
            const V2 t = *reinterpret_cast<const V2 *>(&raw[i]);
            mn = __hmin2(mn, t);
            mx = __hmax2(mx, t);
        }
        lo = fminf(Dt<T>::to_f(mn.x), Dt<T>::to_f(mn.y));
        hi = fmaxf(Dt<T>::to_f(mx.x), Dt<T>::to_f(mx.y));
    } else {
        if (valid) {
            load_elems<T, NE>(w + tid * NE, v);
        } else {
#pragma unroll
            for (int j = 0; j < NV; ++j) v[j] = 0.f;
        }
        lo = v[0];
        hi = v[0];
#pragma unroll
        for (int j = 1; j < NV; ++j) {
            lo = fminf(lo, v[j]);
            hi = fmaxf(hi, v[j]);
        }
    }
    // Invalid lanes form whole groups (n_threads is a multiple of tpg), and
    // the xor partners of a lane stay inside its own group.
    for (int off = tpg >> 1; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (!valid) return;

    const float scale32 = __fdiv_rn(__fsub_rn(hi, lo), (float)QMAX);
    const T s_t = Dt<T>::from_f(scale32);
    const T b_t = Dt<T>::from_f(lo);
    const float s = Dt<T>::to_f(s_t);
    const float b = Dt<T>::to_f(b_t);
    const float r = __frcp_rn(s);

    uint32_t packed[WPT];
#pragma unroll
    for (int k = 0; k < WPT; ++k) packed[k] = 0u;
    if (s != 0.f) {
#pragma unroll
        for (int k = 0; k < WPT; ++k) {
#pragma unroll
            for (int j = 0; j < EPW; j += 2) {
                float v0, v1;
                if constexpr (kPacked) {
                    const uint32_t pr = raw[(k * EPW + j) / 2];
                    v0 = Dt<T>::to_f(*reinterpret_cast<const T *>(&pr));
                    v1 = Dt<T>::to_f(*(reinterpret_cast<const T *>(&pr) + 1));
                } else {
                    v0 = v[k * EPW + j];
                    v1 = v[k * EPW + j + 1];
                }
                uint32_t c0, c1;
                code_pair(v0, v1, b, s, r, (float)QMAX, c0, c1);
                packed[k] |= (c0 << (j * BITS)) | (c1 << ((j + 1) * BITS));
            }
        }
    }
    uint32_t *dst = wq + tid * WPT;
    if constexpr (WPT == 4) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    } else if constexpr (WPT == 2) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[1]);
    } else {
        dst[0] = packed[0];
    }
    if ((threadIdx.x & (tpg - 1)) == 0) {
        const int64_t g = tid / tpg;
        scales[g] = s_t;
        biases[g] = b_t;
    }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(256)
dequantize_kernel(const uint32_t *__restrict__ wq, const T *__restrict__ scales,
                  const T *__restrict__ biases, int64_t n_words, int tpg, T *__restrict__ out) {
    constexpr int EPW = 32 / BITS;
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    const int64_t word = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (word >= n_words) return;
    const int64_t g = word / tpg;
    const float s = Dt<T>::to_f(scales[g]);
    const float b = Dt<T>::to_f(biases[g]);
    const uint32_t packed = __ldg(wq + word);
    T o[EPW];
#pragma unroll
    for (int j = 0; j < EPW; ++j)
        o[j] = Dt<T>::from_f(__fmaf_rn(s, (float)((packed >> (j * BITS)) & MASK), b));
    store_elems<T, EPW>(out + word * EPW, o);
}

// 3- and 6-bit codes do not divide a word: element j of a row occupies bits
// [j*bits, (j+1)*bits) of the row's bit stream, least significant first, so
// 32 consecutive codes fill exactly `bits` words ("a chunk") and a chunk
// never leaves its group (group_size >= 32).  One thread per chunk; the
// group's min/max are reduced over its group_size/32 lanes.
template <typename T, int BITS>
__global__ void __launch_bounds__(256)
quantize_chunk_kernel(const T *__restrict__ w, int64_t n_chunks, int tpg,
                      uint32_t *__restrict__ wq, T *__restrict__ scales, T *__restrict__ biases) {
    constexpr int QMAX = (1 << BITS) - 1;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool valid = c < n_chunks;
    float v[32];
    if (valid) {
        load_elems<T, 32>(w + c * 32, v);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int j = 1; j < 32; ++j) {
        lo = fminf(lo, v[j]);
        hi = fmaxf(hi, v[j]);
    }
    for (int off = tpg >> 1; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (!valid) return;
    const float scale32 = __fdiv_rn(__fsub_rn(hi, lo), (float)QMAX);
    const T s_t = Dt<T>::from_f(scale32);
    const T b_t = Dt<T>::from_f(lo);
    const float s = Dt<T>::to_f(s_t);
    const float b = Dt<T>::to_f(b_t);
    uint32_t out[BITS];
#pragma unroll
    for (int i = 0; i < BITS; ++i) out[i] = 0u;
    if (s != 0.f) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            int q = __float2int_rn(__fdiv_rn(__fsub_rn(v[j], b), s));
            q = min(max(q, 0), QMAX);
            const int bit = j * BITS, wi = bit >> 5, off = bit & 31;
            out[wi] |= (uint32_t)q << off;
            if (off + BITS > 32) out[wi + 1] |= (uint32_t)q >> (32 - off);
        }
    }
    uint32_t *dst = wq + c * BITS;
#pragma unroll
    for (int i = 0; i < BITS; ++i) dst[i] = out[i];
    if ((threadIdx.x & (tpg - 1)) == 0) {
        const int64_t g = c / tpg;
        scales[g] = s_t;
        biases[g] = b_t;
    }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(256)
dequantize_chunk_kernel(const uint32_t *__restrict__ wq, const T *__restrict__ scales,
                        const T *__restrict__ biases, int64_t n_chunks, int tpg,
                        T *__restrict__ out) {
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= n_chunks) return;
    const int64_t g = c / tpg;
    const float s = Dt<T>::to_f(scales[g]);
    const float b = Dt<T>::to_f(biases[g]);
    uint32_t in[BITS];
#pragma unroll
    for (int i = 0; i < BITS; ++i) in[i] = __ldg(wq + c * BITS + i);
    T o[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int bit = j * BITS, wi = bit >> 5, off = bit & 31;
        uint32_t q = in[wi] >> off;
        if (off + BITS > 32) q |= in[wi + 1] << (32 - off);
        o[j] = Dt<T>::from_f(__fmaf_rn(s, (float)(q & MASK), b));
    }
    store_elems<T, 32>(out + c * 32, o);
}

template <typename T>
cudaError_t quantize_t(const QuantArgs &a, cudaStream_t s) {
    if (a.bits == 3 || a.bits == 6) {
        const int64_t n_chunks = a.rows * (a.cols / 32);
        const int tpg = a.group_size / 32;
        const int64_t blocks = (n_chunks + 255) / 256;
        auto w = static_cast<const T *>(a.w);
        auto sc = static_cast<T *>(a.scales);
        auto bi = static_cast<T *>(a.biases);
        if (a.bits == 3) quantize_chunk_kernel<T, 3><<<blocks, 256, 0, s>>>(w, n_chunks, tpg, a.wq, sc, bi);
        else quantize_chunk_kernel<T, 6><<<blocks, 256, 0, s>>>(w, n_chunks, tpg, a.wq, sc, bi);
        count_launches(1);
        return cudaGetLastError();
    }
    const int epw = 32 / a.bits;
    const int words_per_group = a.group_size / epw;
    // 4 words (16 bytes of codes) per thread, fewer when a group is smaller
    // (2-bit codes, group size 32: 2 words).
    const int wpt = std::min(4, words_per_group);
    const int64_t n_threads = a.rows * (a.cols / epw) / wpt;
    const int tpg = words_per_group / wpt;
    const int64_t blocks = (n_threads + 255) / 256;
    auto w = static_cast<const T *>(a.w);
    auto sc = static_cast<T *>(a.scales);
    auto bi = static_cast<T *>(a.biases);
    if (a.bits == 2 && wpt == 2)
        quantize_kernel<T, 2, 2><<<blocks, 256, 0, s>>>(w, n_threads, tpg, a.wq, sc, bi);
    else if (a.bits == 2)
        quantize_kernel<T, 2, 4><<<blocks, 256, 0, s>>>(w, n_threads, tpg, a.wq, sc, bi);
    else if (a.bits == 4)
        quantize_kernel<T, 4, 4><<<blocks, 256, 0, s>>>(w, n_threads, tpg, a.wq, sc, bi);
    else
        quantize_kernel<T, 8, 4><<<blocks, 256, 0, s>>>(w, n_threads, tpg, a.wq, sc, bi);
    count_launches(1);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dequantize_t(const DequantArgs &a, cudaStream_t s) {
    if (a.bits == 3 || a.bits == 6) {
        const int64_t n_chunks = a.rows * (a.cols / 32);
        const int tpg = a.group_size / 32;
        const int64_t blocks = (n_chunks + 255) / 256;
        auto sc = static_cast<const T *>(a.scales);
        auto bi = static_cast<const T *>(a.biases);
        auto out = static_cast<T *>(a.out);
        if (a.bits == 3) dequantize_chunk_kernel<T, 3><<<blocks, 256, 0, s>>>(a.wq, sc, bi, n_chunks, tpg, out);
        else dequantize_chunk_kernel<T, 6><<<blocks, 256, 0, s>>>(a.wq, sc, bi, n_chunks, tpg, out);
        count_launches(1);
        return cudaGetLastError();
    }
    const int epw = 32 / a.bits;
    const int64_t n_words = a.rows * (a.cols / epw);
    const int tpg = a.group_size / epw;
    const int64_t blocks = (n_words + 255) / 256;
    auto sc = static_cast<const T *>(a.scales);
    auto bi = static_cast<const T *>(a.biases);
    auto out = static_cast<T *>(a.out);
    switch (a.bits) {
    case 2: dequantize_kernel<T, 2><<<blocks, 256, 0, s>>>(a.wq, sc, bi, n_words, tpg, out); break;
    case 4: dequantize_kernel<T, 4><<<blocks, 256, 0, s>>>(a.wq, sc, bi, n_words, tpg, out); break;
    default: dequantize_kernel<T, 8><<<blocks, 256, 0, s>>>(a.wq, sc, bi, n_words, tpg, out); break;
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(qmm_dtype dt, const QuantArgs &a, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    switch (dt) {
    case QMM_F32: return quantize_t<float>(a, s);
    case QMM_BF16: return quantize_t<__nv_bfloat16>(a, s);
    default: return quantize_t<__half>(a, s);
    }
}

cudaError_t launch_dequantize(qmm_dtype dt, const DequantArgs &a, cudaStream_t s) {
    if (a.rows == 0) return cudaSuccess;
    switch (dt) {
    case QMM_F32: return dequantize_t<float>(a, s);
    case QMM_BF16: return dequantize_t<__nv_bfloat16>(a, s);
    default: return dequantize_t<__half>(a, s);
    }
}

}  // namespace qmm
