// gemv_fast.cu -- HBM-streaming quantized GEMV for one activation row
// (decode), transpose layout: y[n] = sum_k x[k] * (s[n,g] * q[n,k] + b[n,g]),
// W stored [N, K] (mlx-rs ops/quantization.rs, quantized_matmul;
// Emily.Quantization.Layers, quantized_dense with transpose: true).
//
// The weight is read exactly once, in 16-byte slices.  A "team" of TW warps
// covers one weight row: lane l of team-warp w owns the same UPL consecutive
// slices of every row it visits, so the activation values it multiplies are
// loaded once into registers and never re-read.  Per group the product is
// factored as  s * sum(x*q) + b * sum(x):  codes become bf16/f16 values with
// one LOP3 per pair (magic-exponent trick: OR-ing a code into the mantissa of
// 128.0 (bf16) / 1024.0 (f16) gives OFF + q exactly), multiplied into fp32
// accumulators, and the OFF * sum(x) term is folded into the bias.  Each lane
// keeps one partial per row for a batch of RB rows and the warp reduces them
// all at once with a butterfly reduce-scatter; the team's warps then combine
// through shared memory.  Rows are split evenly over a persistent grid of
// teams and loads run P rows ahead of the arithmetic.
#include <algorithm>
#include <cstdlib>
#include <type_traits>

#include "qmm_internal.cuh"

namespace qmm {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint16_t ldg_u16(const void *p) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// 16-bit storage type traits for the fast path.
template <typename T> struct Half16;
template <> struct Half16<__nv_bfloat16> {
    static constexpr uint32_t MAGIC = 0x43004300u;  // bf16 128.0 | 128.0
    static constexpr float OFF = 128.f;
    static __device__ __forceinline__ float to_f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }
    // acc_lo += lo(x) * lo(t); acc_hi += hi(x) * hi(t), products exact in fp32.
    static __device__ __forceinline__ void fma2(float &lo, float &hi, uint32_t xp, uint32_t t) {
        asm("{.reg .b16 xl, xh, tl, th;\n\t"
            "mov.b32 {xl, xh}, %2;\n\t"
            "mov.b32 {tl, th}, %3;\n\t"
            "fma.rn.f32.bf16 %0, xl, tl, %0;\n\t"
            "fma.rn.f32.bf16 %1, xh, th, %1;\n\t}"
            : "+f"(lo), "+f"(hi)
            : "r"(xp), "r"(t));
    }
};
template <> struct Half16<__half> {
    static constexpr uint32_t MAGIC = 0x64006400u;  // f16 1024.0 | 1024.0
    static constexpr float OFF = 1024.f;
    static __device__ __forceinline__ float to_f(uint16_t h) {
        return __half2float(__ushort_as_half(h));
    }
    static __device__ __forceinline__ void fma2(float &lo, float &hi, uint32_t xp, uint32_t t) {
        asm("{.reg .b16 xl, xh, tl, th;\n\t"
            "mov.b32 {xl, xh}, %2;\n\t"
            "mov.b32 {tl, th}, %3;\n\t"
            "fma.rn.f32.f16 %0, xl, tl, %0;\n\t"
            "fma.rn.f32.f16 %1, xh, th, %1;\n\t}"
            : "+f"(lo), "+f"(hi)
            : "r"(xp), "r"(t));
    }
};

// Alternative inner step: unpack both halves to fp32 and use the packed
// fp32x2 FMA.  Selected by VAR == 1.
template <typename T>
__device__ __forceinline__ void fma2_f32x2(float &lo, float &hi, float2 xf, uint32_t t);
template <>
__device__ __forceinline__ void fma2_f32x2<__nv_bfloat16>(float &lo, float &hi, float2 xf, uint32_t t) {
    float2 q = make_float2(__uint_as_float(t << 16), __uint_as_float(t & 0xffff0000u));
    float2 a = __ffma2_rn(xf, q, make_float2(lo, hi));
    lo = a.x;
    hi = a.y;
}

// Codes per 16-byte slice, and the pairing of codes produced by one LOP3:
//   bits 4: word w, step e (0..3) -> codes (8w+e, 8w+e+4)
//   bits 2: word w, step e (0..7) -> codes (16w+e, 16w+e+8)
//   bits 8: word w, step e (0..1) -> codes (4w+e, 4w+e+2)   (f16 only)
template <int BITS> struct Pack {
    static constexpr int EPW = 32 / BITS;           // codes per word
    static constexpr int EPU = 4 * EPW;             // codes per slice
    static constexpr int STEPS = EPW / 2;           // LOP3 steps per word
    static constexpr uint32_t MASK = BITS == 8 ? 0x00FF00FFu : (BITS == 4 ? 0x000F000Fu : 0x00030003u);
};

// Reduce v[0..RB) across the warp; afterwards lane l (l < RB) holds the warp
// sum of everyone's v[l] in v[0].  Butterfly reduce-scatter: log2(32) rounds,
// each halving the live slots.
template <int RB>
__device__ __forceinline__ float reduce_scatter(float (&v)[RB], int lane) {
    static_assert(RB == 32 || RB == 16, "batch of 16 or 32 rows");
    if constexpr (RB == 16) {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], 16);
    }
#pragma unroll
    for (int s = RB / 2; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int j = 0; j < s; ++j) {
            const float send = upper ? v[j] : v[j + s];
            const float keep = upper ? v[j + s] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return v[0];
}

template <typename T, int BITS, int UPL, int P, int RB, int VAR>
__global__ void __launch_bounds__(kThreads, 2)
qgemv_t_fast_kernel(const T *__restrict__ x, const uint32_t *__restrict__ wq,
                    const T *__restrict__ scales, const T *__restrict__ biases,
                    T *__restrict__ y, int N, int K, int group_size, int TW, int rows_per_team) {
    using H = Half16<T>;
    using PK = Pack<BITS>;
    constexpr int EPU = PK::EPU;
    constexpr int NX = 4 * PK::STEPS;  // packed x pairs per slice (= EPU / 2)
    static_assert(BITS != 8 || VAR == 0, "8-bit codes use the f16 magic only");
    static_assert(P == 1 || P == 2 || P == 4, "prefetch depth must divide the row batch");

    __shared__ float red[kWarps][RB];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // The block holds whole teams only (blockDim.x = teams * TW * 32); a warp
    // outside every team would wait at a team barrier nobody else reaches.
    const int teams_per_cta = (int)(blockDim.x >> 5) / TW;
    if (warp >= teams_per_cta * TW) return;
    const int team = warp / TW, wt = warp - team * TW;
    const int gteam = blockIdx.x * teams_per_cta + team;
    const int row0 = gteam * rows_per_team;
    const int nrows = max(0, min(rows_per_team, N - row0));
    const int spr = K / EPU;                 // slices per row
    const int gpr = K / group_size;          // groups per row
    const int64_t row_words = (int64_t)K / PK::EPW;

    // ---- this lane's slices and their activations ------------------------
    int sl[UPL];
    bool sv[UPL];
    uint32_t xp[UPL][NX];     // x pairs matching the LOP3 code pairing
    float2 xf[UPL][VAR == 1 ? NX : 1];
    float xs[UPL];            // sum of x over the slice
    int gi[UPL];              // group of the slice
#pragma unroll
    for (int u = 0; u < UPL; ++u) {
        sl[u] = (wt * 32 + lane) * UPL + u;
        sv[u] = sl[u] < spr;
        gi[u] = sv[u] ? (sl[u] * EPU) / group_size : 0;
        xs[u] = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            // EPW x values of word w: EPW*2 bytes = (EPW/8) uint4
            uint32_t raw[PK::EPW / 2];
            const T *xw = x + (int64_t)sl[u] * EPU + w * PK::EPW;
            if constexpr (PK::EPW == 4) {
                uint2 v = sv[u] ? *reinterpret_cast<const uint2 *>(xw) : make_uint2(0, 0);
                raw[0] = v.x; raw[1] = v.y;
            } else {
#pragma unroll
                for (int c = 0; c < PK::EPW / 8; ++c) {
                    uint4 v = sv[u] ? *reinterpret_cast<const uint4 *>(xw + c * 8) : make_uint4(0, 0, 0, 0);
                    raw[4 * c + 0] = v.x; raw[4 * c + 1] = v.y; raw[4 * c + 2] = v.z; raw[4 * c + 3] = v.w;
                }
            }
            // pair e: codes (e, e + EPW/2) of this word
#pragma unroll
            for (int e = 0; e < PK::STEPS; ++e) {
                const int a = e, b = e + PK::EPW / 2;  // element indices within the word
                const uint32_t ra = raw[a >> 1], rb = raw[b >> 1];
                const uint32_t lo = (a & 1) ? (ra >> 16) : (ra & 0xffffu);
                const uint32_t hi = (b & 1) ? (rb & 0xffff0000u) : (rb << 16);
                xp[u][w * PK::STEPS + e] = lo | hi;
                const float fa = H::to_f((uint16_t)lo), fb = H::to_f((uint16_t)(hi >> 16));
                if constexpr (VAR == 1) xf[u][w * PK::STEPS + e] = make_float2(fa, fb);
                xs[u] += fa + fb;
            }
        }
    }

    // ---- software pipeline over this team's rows ------------------------
    uint4 wb[P][UPL];
    uint16_t sb[P][UPL], bb[P][UPL];
    auto load_row = [&](int p, int r) {
        const int64_t row = row0 + r;
        const uint32_t *wr = wq + row * row_words;
#pragma unroll
        for (int u = 0; u < UPL; ++u) {
            if (sv[u]) {
                wb[p][u] = ldg_stream(wr + (int64_t)sl[u] * 4);
                sb[p][u] = ldg_u16(scales + row * gpr + gi[u]);
                bb[p][u] = ldg_u16(biases + row * gpr + gi[u]);
            } else {
                wb[p][u] = make_uint4(0, 0, 0, 0);
                sb[p][u] = 0;
                bb[p][u] = 0;
            }
        }
    };
#pragma unroll
    for (int p = 0; p < P; ++p)
        if (p < nrows) load_row(p, p);

    const int nbatch = (nrows + RB - 1) / RB;
    for (int bt = 0; bt < nbatch; ++bt) {
        float part[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            const int r = bt * RB + j;
            float acc = 0.f;
            if (r < nrows) {
                const int p = j % P;
#pragma unroll
                for (int u = 0; u < UPL; ++u) {
                    float lo = 0.f, hi = 0.f;
                    const uint32_t wv[4] = {wb[p][u].x, wb[p][u].y, wb[p][u].z, wb[p][u].w};
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
#pragma unroll
                        for (int e = 0; e < PK::STEPS; ++e) {
                            const uint32_t t = ((wv[w] >> (BITS * e)) & PK::MASK) | H::MAGIC;
                            if constexpr (VAR == 1)
                                fma2_f32x2<T>(lo, hi, xf[u][w * PK::STEPS + e], t);
                            else
                                H::fma2(lo, hi, xp[u][w * PK::STEPS + e], t);
                        }
                    }
                    const float s = H::to_f(sb[p][u]);
                    const float b = H::to_f(bb[p][u]);
                    // s * sum(x*(OFF+q)) + (b - OFF*s) * sum(x)
                    acc = __fmaf_rn(s, lo + hi, acc);
                    acc = __fmaf_rn(__fmaf_rn(-H::OFF, s, b), xs[u], acc);
                }
                if (r + P < nrows) load_row(p, r + P);
            }
            part[j] = acc;
        }
        const float v = reduce_scatter<RB>(part, lane);
        // Combine the team's warps: lane l holds this warp's sum for row bt*RB + l.
        if (lane < RB) red[warp][lane] = v;
        if (TW > 1) {
            asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(TW * 32) : "memory");
        } else {
            __syncwarp();
        }
        if (wt == 0 && lane < RB) {
            float tot = 0.f;
            for (int q = 0; q < TW; ++q) tot += red[team * TW + q][lane];
            const int r = bt * RB + lane;
            if (r < nrows) y[row0 + r] = Dt<T>::from_f(tot);
        }
        if (TW > 1) {
            asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(TW * 32) : "memory");
        } else {
            __syncwarp();
        }
    }
}

// Inner-loop variant and slices per lane.  Defaults are the measured best;
// QMM_GEMV_VAR / QMM_GEMV_UPL override them for experiments.
int env_int(const char *name, int dflt) {
    const char *v = getenv(name);
    return v ? atoi(v) : dflt;
}
int g_var = env_int("QMM_GEMV_VAR", 0);
int g_upl = env_int("QMM_GEMV_UPL", 0);  // 0 = auto

template <typename T, int BITS, int UPL, int VAR>
cudaError_t launch_fast(const QmmArgs &a, cudaStream_t s) {
    using PK = Pack<BITS>;
    constexpr int P = 4;
    constexpr int RB = 32;
    const int spr = (int)(a.K / PK::EPU);
    const int TW = (spr + 32 * UPL - 1) / (32 * UPL);
    auto kern = qgemv_t_fast_kernel<T, BITS, UPL, P, RB, VAR>;
    const int teams_per_cta = kWarps / TW;          // TW <= kWarps (checked by the caller)
    const int threads = teams_per_cta * TW * 32;    // whole teams only
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
    if (e != cudaSuccess) return e;
    per_sm = std::max(per_sm, 1);
    const int64_t teams = (int64_t)num_sms() * per_sm * teams_per_cta;
    const int rows_per_team = (int)((a.N + teams - 1) / teams);
    const int64_t need_teams = (a.N + rows_per_team - 1) / rows_per_team;
    const int grid = (int)((need_teams + teams_per_cta - 1) / teams_per_cta);
    kern<<<grid, threads, 0, s>>>(static_cast<const T *>(a.x), a.wq, static_cast<const T *>(a.scales),
                                    static_cast<const T *>(a.biases), static_cast<T *>(a.y),
                                    (int)a.N, (int)a.K, a.group_size, TW, rows_per_team);
    count_launches(1);
    return cudaGetLastError();
}

template <typename T, int BITS>
cudaError_t fast_bits(const QmmArgs &a, cudaStream_t s) {
    using PK = Pack<BITS>;
    const int spr = (int)(a.K / PK::EPU);
    const bool two = g_upl == 2 || spr > 32 * 8;  // keep TW <= 8
    if constexpr (BITS == 4 && std::is_same<T, __nv_bfloat16>::value) {
        if (g_var == 1) return two ? launch_fast<T, BITS, 2, 1>(a, s) : launch_fast<T, BITS, 1, 1>(a, s);
    }
    return two ? launch_fast<T, BITS, 2, 0>(a, s) : launch_fast<T, BITS, 1, 0>(a, s);
}

}  // namespace

// The fast path takes one activation row of a bf16/f16 problem in the
// transpose layout, whole 16-byte slices per row, one group per slice at
// least (group_size >= codes per slice), and a team of at most 8 warps.
bool gemv_fast_supported(qmm_dtype dt, const QmmArgs &a) {
    if (!a.transpose || a.M != 1) return false;
    if (dt == QMM_F32) return false;
    if (dt == QMM_BF16 && a.bits == 8) return false;  // no exact bf16 magic for 8-bit codes
    const int epu = 128 / a.bits;
    if (a.K % epu != 0 || a.group_size < epu) return false;
    if (a.K > (int64_t)epu * 32 * 2 * kWarps) return false;
    if (a.N > INT32_MAX || a.K > INT32_MAX) return false;
    return true;
}

cudaError_t launch_gemv_fast(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    if (dt == QMM_BF16) {
        switch (a.bits) {
        case 2: return fast_bits<__nv_bfloat16, 2>(a, s);
        default: return fast_bits<__nv_bfloat16, 4>(a, s);
        }
    }
    switch (a.bits) {
    case 2: return fast_bits<__half, 2>(a, s);
    case 4: return fast_bits<__half, 4>(a, s);
    default: return fast_bits<__half, 8>(a, s);
    }
}

}  // namespace qmm
