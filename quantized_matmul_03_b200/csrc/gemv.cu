// gemv.cu -- SIMT quantized matmul for few activation rows (decode shapes).
//
// y = x @ W^T (transpose, W stored [N, K]) or y = x @ W (W stored [K, N]),
// W = scale * q + bias group-wise along W's last stored axis (mlx-rs
// ops/quantization.rs, quantized_matmul; Emily.Quantization.Layers,
// quantized_dense for the two layouts).  The packed weight is streamed once;
// nothing dense is written back.
//
// gemv_t (transpose):  a warp owns RW weight rows; its lanes stride the row's
//   packed words (128-byte coalesced warp loads) against activations staged in
//   shared memory chunk by chunk along K, accumulate in fp32 registers and
//   finish with a warp-shuffle reduction.
// gemv_n (no transpose): a lane owns one packed word column (32/bits output
//   features); the K range is split across the CTA's warps and across the
//   CTAs of a thread-block cluster, and the partial sums are reduced through
//   shared memory and then distributed shared memory.
#include <algorithm>

#include <cooperative_groups.h>

#include "mx.cuh"
#include "qmm_internal.cuh"

namespace cg = cooperative_groups;

namespace qmm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Which product a CTA computes: blockIdx.z + b0 is the batch entry; a plain
// matmul is the one-entry batch with zero strides.  gather_qmm entries
// resolve their activation and expert through GatherIndex; an entry with an
// out-of-range index computes nothing and writes zeros.
struct BatchView {
    GatherIndex gi;
    int64_t b0;
    int64_t x_stride, w_stride, sb_stride, y_stride;  // elements / words per entry
    const void *bias;  // layer bias (plain matmul only), added before rounding
    float bias_value;
    int *err;
};

// Offsets (in elements / words) of this CTA's entry; false for an invalid one.
struct EntryOffsets {
    int64_t x, w, sb, y;
};
__device__ __forceinline__ bool select_entry(const BatchView &bv, EntryOffsets &o) {
    const int64_t b = bv.b0 + blockIdx.z;
    int64_t xi, ei;
    const bool valid = gather_entry(bv.gi, b, xi, ei);
    if (!valid) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
            record_device_error(bv.err, QMM_ERR_INDEX);
        xi = ei = 0;
    }
    o.x = xi * bv.x_stride;
    o.w = ei * bv.w_stride;
    o.sb = ei * bv.sb_stride;
    o.y = b * bv.y_stride;
    return valid;
}

// The kernels walk packed rows in chunks: one word (32/bits codes) for 2-,
// 4- and 8-bit codes; for 3- and 6-bit codes, which run back to back in the
// row's bit stream, the `bits` words that hold 32 codes exactly.  A chunk
// never leaves its group (group_size >= 32).
template <int BITS> struct Chunk {
    static constexpr int W = (BITS == 3 || BITS == 6) ? BITS : 1;  // words per chunk
    static constexpr int E = W * 32 / BITS;                        // codes per chunk
};

// The E weights of one chunk: affine s*q + b (fmaf, as dequantize), or, in a
// microscaled mode, X * element (exact).  `sb` indexes the chunk's group in
// scales (and biases).
template <typename T, int BITS, int MODE>
__device__ __forceinline__ void chunk_weights(const uint32_t *pk, const void *scales,
                                              const void *biases, int64_t sb, float *wv) {
    constexpr int E = Chunk<BITS>::E;
    if constexpr (MODE == QMM_MODE_AFFINE) {
        constexpr uint32_t MASK = (1u << BITS) - 1u;
        const float s = Dt<T>::to_f(static_cast<const T *>(scales)[sb]);
        const float b = Dt<T>::to_f(static_cast<const T *>(biases)[sb]);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int bit = e * BITS, wi = bit >> 5, off = bit & 31;
            uint32_t q = pk[wi] >> off;
            if (off + BITS > 32) q |= pk[wi + 1] << (32 - off);
            wv[e] = __fmaf_rn(s, (float)(q & MASK), b);
        }
    } else {
        const float x = mxf::scale_value<MODE>(static_cast<const uint8_t *>(scales)[sb]);
        mxf::elements<MODE>(pk[0], wv);
#pragma unroll
        for (int e = 0; e < E; ++e) wv[e] = __fmul_rn(x, wv[e]);
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// ---------------------------------------------------------------------------
// transpose = true
// ---------------------------------------------------------------------------
template <typename T, int BITS, int MT, int RW, int MODE>
__global__ void __launch_bounds__(kThreads)
gemv_t_kernel(const T *__restrict__ x, const uint32_t *__restrict__ wq,
              const void *__restrict__ scales, const void *__restrict__ biases,
              T *__restrict__ y, int M, int64_t N, int64_t K, int group_size, int kc,
              const BatchView bv) {
    constexpr int CW = Chunk<BITS>::W, CE = Chunk<BITS>::E;
    extern __shared__ float xs[];  // [MT][kc]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row0 = (int64_t)blockIdx.x * (kWarps * RW) + (int64_t)warp * RW;
    const int64_t wpr = K * BITS / 32;    // packed words per weight row
    const int64_t gpr = K / group_size;   // groups per weight row

    EntryOffsets eo;
    const bool valid = select_entry(bv, eo);
    x += eo.x;
    wq += eo.w;
    const int64_t sb0 = eo.sb;
    y += eo.y;

    float acc[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

    for (int64_t k0 = 0; valid && k0 < K; k0 += kc) {  // (CTA-uniform condition)
        const int klen = (int)min((int64_t)kc, K - k0);
        __syncthreads();
        for (int i = threadIdx.x; i < MT * klen; i += kThreads) {
            const int m = i / klen, kk = i - m * klen;
            xs[m * kc + kk] = (m < M) ? Dt<T>::to_f(x[(int64_t)m * K + k0 + kk]) : 0.f;
        }
        __syncthreads();
        const int clen = klen / CE;   // chunks of this activation chunk (kc % 128 == 0)
#pragma unroll
        for (int r = 0; r < RW; ++r) {
            const int64_t row = row0 + r;
            if (row >= N) break;  // warp-uniform
            const uint32_t *wr = wq + row * wpr + k0 * BITS / 32;
            for (int j = lane; j < clen; j += 32) {
                uint32_t pk[CW];
#pragma unroll
                for (int i = 0; i < CW; ++i) pk[i] = __ldg(wr + j * CW + i);
                const int64_t g = (k0 + (int64_t)j * CE) / group_size;
                float wv[CE];
                chunk_weights<T, BITS, MODE>(pk, scales, biases, sb0 + row * gpr + g, wv);
#pragma unroll
                for (int e = 0; e < CE; ++e) {
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        acc[r][m] = __fmaf_rn(xs[m * kc + j * CE + e], wv[e], acc[r][m]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        const int64_t row = row0 + r;
        if (row >= N) break;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float v = warp_sum(acc[r][m]);
            if (lane == 0 && m < M)
                y[(int64_t)m * N + row] = Dt<T>::from_f(v + layer_bias<T>(bv.bias, bv.bias_value, row));
        }
    }
}

// ---------------------------------------------------------------------------
// transpose = false: W stored [K, N], groups run along N.
// ---------------------------------------------------------------------------
template <typename T, int BITS, int MT, int MODE>
__global__ void __launch_bounds__(kThreads)
gemv_n_kernel(const T *__restrict__ x, const uint32_t *__restrict__ wq,
              const void *__restrict__ scales, const void *__restrict__ biases,
              T *__restrict__ y, int M, int64_t N, int64_t K, int group_size, int64_t k_split,
              const BatchView bv) {
    constexpr int CW = Chunk<BITS>::W, EPW = Chunk<BITS>::E;  // (EPW: codes per chunk)
    constexpr int NE = EPW * MT;           // partial sums per lane
    __shared__ float red[kWarps][NE][32];  // per-warp partials
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    EntryOffsets eo;
    const bool valid = select_entry(bv, eo);
    x += eo.x;
    wq += eo.w;
    const int64_t sb0 = eo.sb;
    y += eo.y;
    const int64_t wpr = N * BITS / 32;      // packed words per weight row
    const int64_t cpr = N / EPW;            // chunks per weight row
    const int64_t gpr = N / group_size;
    const int64_t col = (int64_t)blockIdx.x * 32 + lane;  // chunk column
    const bool col_ok = col < cpr;
    const int64_t kbeg = (int64_t)blockIdx.y * k_split;
    const int64_t kend = min(K, kbeg + k_split);

    float acc[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) acc[i] = 0.f;

    if (col_ok && valid) {
        const int64_t g = col * EPW / group_size;
        for (int64_t k = kbeg + warp; k < kend; k += kWarps) {
            uint32_t pk[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) pk[i] = __ldg(wq + k * wpr + col * CW + i);
            float wv[EPW];
            chunk_weights<T, BITS, MODE>(pk, scales, biases, sb0 + k * gpr + g, wv);
            float xv[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) xv[m] = (m < M) ? Dt<T>::to_f(x[(int64_t)m * K + k]) : 0.f;
#pragma unroll
            for (int e = 0; e < EPW; ++e) {
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[e * MT + m] = __fmaf_rn(xv[m], wv[e], acc[e * MT + m]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NE; ++i) red[warp][i][lane] = acc[i];
    __syncthreads();
    // Sum the warps' partials into warp 0's slot.
    for (int i = threadIdx.x; i < NE * 32; i += kThreads) {
        const int e = i >> 5, l = i & 31;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][e][l];
        red[0][e][l] = v;
    }
    // Sum across the cluster's CTAs (the K splits) via distributed shared memory.
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int nrank = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    for (int i = rank * kThreads + threadIdx.x; i < NE * 32; i += nrank * kThreads) {
        const int e = i >> 5, l = i & 31;
        float v = 0.f;
        for (int q = 0; q < nrank; ++q) v += cluster.map_shared_rank(&red[0][0][0], q)[e * 32 + l];
        const int64_t c = (int64_t)blockIdx.x * 32 + l;
        const int ei = e / MT, m = e - ei * MT;
        if (c < cpr && m < M)
            y[(int64_t)m * N + c * EPW + ei] =
                Dt<T>::from_f(v + layer_bias<T>(bv.bias, bv.bias_value, c * EPW + ei));
    }
    cluster.sync();
}

template <typename T, int BITS, int MT, int MODE>
cudaError_t run_gemv_t(const QmmArgs &a, int M, const T *x, T *y, const BatchView &bv, int nb,
                       cudaStream_t s) {
    constexpr int RW = 2;
    const int64_t rows_per_cta = kWarps * RW;
    const int64_t gx = (a.N + rows_per_cta - 1) / rows_per_cta;
    // Activation chunk: at most 48 KB of fp32, a multiple of 128 elements.
    int kc = (int)std::min<int64_t>(a.K, (48 * 1024 / 4) / MT);
    kc = (kc / 128) * 128;
    if (kc <= 0) kc = 128;
    if (kc > a.K) kc = (int)a.K;
    const size_t smem = (size_t)MT * kc * sizeof(float);
    gemv_t_kernel<T, BITS, MT, RW, MODE><<<dim3((unsigned)gx, 1, nb), kThreads, smem, s>>>(
        x, a.wq, a.scales, a.biases, y, M, a.N, a.K, a.group_size, kc, bv);
    count_launches(1);
    return cudaGetLastError();
}

template <typename T, int BITS, int MT, int MODE>
cudaError_t run_gemv_n(const QmmArgs &a, int M, const T *x, T *y, const BatchView &bv, int nb,
                       cudaStream_t s) {
    const int64_t cpr = a.N / Chunk<BITS>::E;
    const int gx = (int)((cpr + 31) / 32);
    // Split K over a cluster of up to 8 CTAs so that small-N problems still
    // fill the GPU; each split is at least 64 rows of W.
    int ks = 8;
    while (ks > 1 && (int64_t)gx * ks * nb > 4LL * num_sms()) ks >>= 1;
    while (ks > 1 && a.K / ks < 64) ks >>= 1;
    const int64_t k_split = (a.K + ks - 1) / ks;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gx, ks, nb);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = ks;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launches(1);
    return cudaLaunchKernelEx(&cfg, gemv_n_kernel<T, BITS, MT, MODE>, x, a.wq, a.scales, a.biases,
                              y, M, a.N, a.K, a.group_size, k_split, bv);
}

// Largest activation tile per launch: gemv_t keeps RW*MT accumulators per
// lane; gemv_n keeps (32/bits)*MT, capped at 32 (so MT <= bits).  Entries of
// a batch go to gridDim.z, at most 65535 per launch.
template <typename T, int BITS, int MODE = QMM_MODE_AFFINE>
cudaError_t gemv_bits(const QmmArgs &a, const BatchView &bv0, int64_t batch, cudaStream_t s) {
    const T *x = static_cast<const T *>(a.x);
    T *y = static_cast<T *>(a.y);
    // (3-/6-bit chunks hold 32 codes per lane: one activation row at a time)
    const int tile = a.transpose ? 16 : (BITS == 3 || BITS == 6 ? 1 : BITS);
    for (int64_t b0 = 0; b0 < batch; b0 += 65535) {
        const int nb = (int)std::min<int64_t>(65535, batch - b0);
        BatchView bv = bv0;
        bv.b0 = b0;
        for (int64_t m0 = 0; m0 < a.M; m0 += tile) {
            const int mt = (int)std::min<int64_t>(tile, a.M - m0);
            const T *xm = x + m0 * a.K;
            T *ym = y + m0 * a.N;
            cudaError_t e;
            if (a.transpose) {
                if (mt == 1) e = run_gemv_t<T, BITS, 1, MODE>(a, mt, xm, ym, bv, nb, s);
                else if (mt == 2) e = run_gemv_t<T, BITS, 2, MODE>(a, mt, xm, ym, bv, nb, s);
                else if (mt <= 4) e = run_gemv_t<T, BITS, 4, MODE>(a, mt, xm, ym, bv, nb, s);
                else if (mt <= 8) e = run_gemv_t<T, BITS, 8, MODE>(a, mt, xm, ym, bv, nb, s);
                else e = run_gemv_t<T, BITS, 16, MODE>(a, mt, xm, ym, bv, nb, s);
            } else {
                if (mt == 1) e = run_gemv_n<T, BITS, 1, MODE>(a, mt, xm, ym, bv, nb, s);
                else if constexpr (BITS == 3 || BITS == 6) e = cudaErrorInvalidValue;
                else if (mt == 2) e = run_gemv_n<T, BITS, 2, MODE>(a, mt, xm, ym, bv, nb, s);
                else if constexpr (BITS == 4 || BITS == 8) {
                    if (mt <= 4) e = run_gemv_n<T, BITS, 4, MODE>(a, mt, xm, ym, bv, nb, s);
                    else if constexpr (BITS >= 8) e = run_gemv_n<T, BITS, 8, MODE>(a, mt, xm, ym, bv, nb, s);
                    else e = cudaErrorInvalidValue;
                } else {
                    e = cudaErrorInvalidValue;
                }
            }
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t gemv_t_dtype(const QmmArgs &a, const BatchView &bv, int64_t batch, cudaStream_t s) {
    switch (a.mode) {
    case QMM_MODE_MXFP4: return gemv_bits<T, 4, QMM_MODE_MXFP4>(a, bv, batch, s);
    case QMM_MODE_NVFP4: return gemv_bits<T, 4, QMM_MODE_NVFP4>(a, bv, batch, s);
    case QMM_MODE_MXFP8: return gemv_bits<T, 8, QMM_MODE_MXFP8>(a, bv, batch, s);
    default: break;
    }
    switch (a.bits) {
    case 2: return gemv_bits<T, 2>(a, bv, batch, s);
    case 3: return gemv_bits<T, 3>(a, bv, batch, s);
    case 4: return gemv_bits<T, 4>(a, bv, batch, s);
    case 6: return gemv_bits<T, 6>(a, bv, batch, s);
    default: return gemv_bits<T, 8>(a, bv, batch, s);
    }
}

cudaError_t gemv_dispatch(qmm_dtype dt, const QmmArgs &a, const BatchView &bv, int64_t batch,
                          cudaStream_t s) {
    switch (dt) {
    case QMM_F32: return gemv_t_dtype<float>(a, bv, batch, s);
    case QMM_BF16: return gemv_t_dtype<__nv_bfloat16>(a, bv, batch, s);
    default: return gemv_t_dtype<__half>(a, bv, batch, s);
    }
}

}  // namespace

bool gemv_supported(qmm_dtype, const QmmArgs &) { return true; }

cudaError_t launch_gemv(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    if (a.M == 0 || a.N == 0) return cudaSuccess;
    BatchView bv{};
    bv.gi = GatherIndex{nullptr, nullptr, 1, 1, 1};
    bv.bias = a.bias;
    bv.bias_value = a.bias_value;
    bv.err = device_error_word();
    return gemv_dispatch(dt, a, bv, 1, s);
}

// a describes one entry: x points at x[0] ([M, K]), wq/scales/biases at
// expert 0, y at y[0] ([M, N]).
cudaError_t launch_gemv_gather(qmm_dtype dt, const QmmArgs &a, const GatherIndex &gi, cudaStream_t s) {
    if (a.M == 0 || a.N == 0 || gi.batch == 0) return cudaSuccess;
    const int64_t wrows = a.transpose ? a.N : a.K, wcols = a.transpose ? a.K : a.N;
    BatchView bv{};
    bv.gi = gi;
    bv.x_stride = a.M * a.K;
    bv.w_stride = wrows * (wcols * a.bits / 32);
    bv.sb_stride = wrows * (wcols / a.group_size);
    bv.y_stride = a.M * a.N;
    bv.err = device_error_word();
    return gemv_dispatch(dt, a, bv, gi.batch, s);
}

}  // namespace qmm
