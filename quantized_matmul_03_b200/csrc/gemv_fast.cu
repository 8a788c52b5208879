// gemv_fast.cu -- HBM-streaming quantized GEMV for 1..4 activation rows
// (decode), transpose layout:  y[m, n] = sum_k x[m, k] * (s[n,g] q[n,k] + b[n,g])
// with W stored [N, K] (mlx-rs ops/quantization.rs, quantized_matmul;
// Emily.Quantization.Layers, quantized_dense with transpose: true).
//
// Memory side.  The weight's rows are cut into stages of SR rows, each one
// contiguous byte range of the packed weight (and of the scales and biases),
// dealt round-robin over the CTAs so that the copies in flight at any moment
// cover one contiguous stretch of memory.  A producer warp streams a CTA's
// stages through a ring of shared-memory slots with 1-D bulk copies
// (cp.async.bulk) completing on mbarriers, so ~100 KB per SM are in flight
// regardless of register pressure.  The weight is read exactly once.
//
// Arithmetic side.  A team of TW consumer warps covers one weight row; lane l
// owns the same 16-byte slice(s) of every row, so its activations live in
// registers for the whole kernel.  Per group the product is factored as
//   s * sum(x q) + b * sum(x).
// For sum(x q) the codes stay integers: one AND spreads a word's codes into
// byte lanes ("planes": for 4-bit codes, bytes of w & 0x0F0F0F0F are codes
// 0,2,4,6 and bytes of (w >> 4) & 0x0F0F0F0F are codes 1,3,5,7), and DP2A
// multiplies two bytes by two signed 16-bit activations and accumulates in
// int32.  The activations of each 16-byte slice are held in 16-bit block
// fixed point, x_int = rint(x * 2^sh) with sh chosen from the slice's largest
// |x| so that |x_int| < 2^14: the representation error is at most 2^-15 of
// the slice maximum, and every product and sum after it is exact.  A slice's
// integer sum is multiplied by s * 2^-sh in fp32, and sum(x) is the sum of the
// same fixed-point values, so the result is the exact product of the
// dequantized weight with the rounded activations, rounded once per slice.
// Per word of 4-bit codes this is 3 ALU + 4 DP2A instructions (8-bit codes:
// 2 DP2A, no ALU), which keeps the ALU pipe, the limiter of an fp32
// formulation, below the memory time.  Lane partials for a stage's rows are
// combined by a butterfly reduce-scatter into one shared-memory slot per
// warp, summed in a fixed warp order at the end (results repeat bit for bit)
// and written out in one pass per CTA.
//
// Microscaled E2M1 weights (mxfp4, nvfp4; Emily.QuantizedWeight, Microscaled
// modes): twice an E2M1 value is an integer in [-12, 12].  Four codes become
// the bytes 128 + 2e with two PRMT table lookups and one IADD3 (see
// e2m1_word_to_u8), and DP2A takes them as it takes affine codes; the 128
// offset is taken out by starting each group's accumulator at -128 sum(x_int).
// Per group the integer sum is scaled by X/2 (X the group's scale value),
// with no bias term.  The stages then carry the codes and the scale bytes.
#include <algorithm>
#include <cstdlib>
#include <type_traits>

#include "mx.cuh"
#include "ptx_sm100.cuh"
#include "qmm_internal.cuh"

namespace qmm {
namespace {

constexpr int kCW = 12;                   // consumer warps
constexpr int kThreads = 32 * (kCW + 1);  // plus one producer warp

// Per-SM hand-off between consecutive CTAs of this kernel.  Under
// programmatic dependent launch the next call's CTA sits beside the current
// one on the SM from the current call's start; if it streams its first stages
// at once, those copies compete with the current call's own stage copies,
// which are on the critical path.  So a CTA takes a ticket per SM and issues
// its first copy only once the CTA before it on the same SM has at most one
// stage left to issue (or after a short bound; waiting for all of them, or
// for two or three stages left, was measured slower).  This orders memory
// traffic only: results do not depend on it.
constexpr int kMaxSm = 1024;
constexpr uint64_t kHandoffWaitNs = 8000;
__device__ unsigned long long g_sm_ticket[kMaxSm];  // CTAs that entered, per SM
__device__ unsigned long long g_sm_issued[kMaxSm];  // highest ticket + 1 with <= 1 stage to issue
__device__ unsigned long long g_sm_grid[kMaxSm];    // %gridid of the latest ticket's CTA

// Code planes of a packed word: plane p = (w >> p*BITS) & byte-mask, whose
// byte j is code j*NP + p (NP = 8/BITS planes).  DP2A.lo takes bytes 0,1 and
// DP2A.hi bytes 2,3, so the activation pairs of plane p are
//   lo: (x[p], x[NP + p])     hi: (x[2NP + p], x[3NP + p]).
template <int BITS> struct Planes {
    static constexpr int NP = 8 / BITS;        // planes per word
    static constexpr uint32_t BYTE_MASK = ((1u << BITS) - 1u) * 0x01010101u;
    // element (within the word) of half h (0/1) of pair k (k = 2p + {0: lo, 1: hi})
    static __host__ __device__ constexpr int elem(int k, int h) {
        return (k & 1) * 2 * NP + h * NP + (k >> 1);
    }
};

__device__ __forceinline__ int dp2a_lo(int xa, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(xa), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi(int xa, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(xa), "r"(b), "r"(c));
    return d;
}

// acc0/acc1 += sum over the word's codes of x_int * q.
template <int BITS, int P = 0>
__device__ __forceinline__ void dot_word(uint32_t w, const int *xp, int &acc0, int &acc1) {
    using PL = Planes<BITS>;
    if constexpr (P < PL::NP) {
        const uint32_t plane = (P == 0 ? w : (w >> (P * BITS))) & PL::BYTE_MASK;
        acc0 = dp2a_lo(xp[2 * P], plane, acc0);
        acc1 = dp2a_hi(xp[2 * P + 1], plane, acc1);
        dot_word<BITS, P + 1>(w, xp, acc0, acc1);
    }
}

// Sum v[0..V) over the 32 lanes; afterwards lane l holds the total of index
// (l mod V).  Butterfly halving over lane bits below V, then xor-reduction
// over the remaining lane bits.
template <int V>
__device__ __forceinline__ float reduce_scatter(float (&v)[V], int lane) {
#pragma unroll
    for (int s = V / 2; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int j = 0; j < s; ++j) {
            const float send = upper ? v[j] : v[j + s];
            const float keep = upper ? v[j + s] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    float r = v[0];
#pragma unroll
    for (int s = V; s < 32; s <<= 1) r += __shfl_xor_sync(0xffffffffu, r, s);
    return r;
}

__device__ __forceinline__ float h16_to_f(uint16_t h, bool is_bf16) {
    return is_bf16 ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
}

// Element e of 16-bit elements packed two per word (element 2k in the low half).
template <bool BF16, int N>
__device__ __forceinline__ float elem_to_f(const uint32_t (&w)[N], int e) {
    const uint32_t v = w[e >> 1];
    if constexpr (BF16) return __uint_as_float((e & 1) ? (v & 0xFFFF0000u) : (v << 16));
    return __half2float(__ushort_as_half((unsigned short)((e & 1) ? (v >> 16) : (v & 0xFFFFu))));
}

// 2 * E2M1 magnitude of codes 0..7, as a PRMT table of 8 bytes.
constexpr uint32_t kE2m1Lo = 0x03020100u, kE2m1Hi = 0x0C080604u;

// PRMT in its generic form: byte n of the result is byte (c >> 4n) & 7 of
// {b:a}, or, when bit 3 of that nibble is set, that byte's sign replicated.
// (__byte_perm is defined on the three low selector bits only, so the sign
// form is written out.)
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// The eight E2M1 codes of w (code j at bits 4j..4j+3, its sign in bit 3 of
// the nibble) as unsigned bytes 128 + 2 e_j: v[0] holds codes 0..3, v[1]
// codes 4..7.  A PRMT on the raw nibbles gives the table magnitude of every
// non-negative code and 0 for a negative one (the code's sign bit asks for
// the sign of a table byte, and every table byte is positive); on the
// nibbles with their sign bits flipped it gives the converse.  Per byte the
// sum 128 + pos - neg lies in [116, 140], so no byte borrows from another.
__device__ __forceinline__ void e2m1_word_to_u8(uint32_t w, uint32_t *v) {
    const uint32_t wn = w ^ 0x88888888u;
    v[0] = prmt(kE2m1Lo, kE2m1Hi, w) + 0x80808080u - prmt(kE2m1Lo, kE2m1Hi, wn);
    v[1] = prmt(kE2m1Lo, kE2m1Hi, w >> 16) + 0x80808080u - prmt(kE2m1Lo, kE2m1Hi, wn >> 16);
}

// One-row variants with one slice per lane are held to 72 registers, so that
// two CTAs (this call's and the next one's) fit the SM's register file (416
// threads x 72 x 2 <= 65536).  A minimum-blocks launch bound gave 64 registers
// and a slower loop.
template <int BITS, int MR, int UPL>
constexpr int stream_max_regs() { return (MR == 1 && UPL == 1 && BITS != 2) ? 72 : 168; }

template <typename T, int BITS, int MR, int UPL, int RPT, int MODE = QMM_MODE_AFFINE>
__global__ void __launch_bounds__(kThreads, 1) __maxnreg__((stream_max_regs<BITS, MR, UPL>()))
qgemv_stream_kernel(const T *__restrict__ x, const uint32_t *__restrict__ wq,
                    const T *__restrict__ scales, const T *__restrict__ biases,
                    T *__restrict__ y, int M, int N, int K, int group_size, int rpc, int R,
                    int q, int S, int TW, const T *__restrict__ bias, float bias_value, int *err,
                    T *__restrict__ y2) {
    constexpr int EPW = 32 / BITS;       // codes per word
    constexpr int EPU = 4 * EPW;         // codes per 16-byte slice
    constexpr int STEPS = EPW / 2;       // code pairs per word
    constexpr int V = MR * RPT;          // partials per lane per stage
    constexpr bool kBF16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr bool MX = MODE != QMM_MODE_AFFINE;   // E2M1 elements, scale bytes, no biases
    constexpr bool NV = MODE == QMM_MODE_NVFP4;    // two groups of 16 per 32-code slice
    static_assert(!MX || BITS == 4, "microscaled codes here are E2M1");
    static_assert((V & (V - 1)) == 0 && V <= 32, "V must be a power of two <= 32");

    extern __shared__ __align__(128) uint8_t smem[];
    const int NT = kCW / TW;                 // teams; warps past NT*TW only pace the ring
    const int SR = NT * RPT;                 // rows per stage
    const int row_bytes = K / 8 * BITS;
    const int gpr = K / group_size;
    constexpr int NSB = MX ? 1 : 2;          // per-group arrays per row: scales (+ biases)
    const int sb_bytes = MX ? gpr : gpr * 2;  // bytes of one array per row
    const int stage_bytes = SR * (row_bytes + NSB * sb_bytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)S * stage_bytes);
    float *ysm = reinterpret_cast<float *>(bars + 2 * S);
    // Rows: R rounds of SR-row stages dealt across the grid (stage i of CTA b
    // holds rows (i * grid + b) * SR ...), so that the copies in flight at
    // any moment cover one contiguous stretch of the weight; then one final
    // stage of at most q rows per CTA.  Local row r of stage i = r / SR.
    const int grid = (int)gridDim.x, b = (int)blockIdx.x;
    const int tr0 = R * grid * SR + b * q;           // first row of the final stage
    const int nq = max(0, min(q, N - tr0));
    const int nrows = R * SR + nq;                   // rows of this CTA (<= rpc)
    const int nst = R + (nq > 0 ? 1 : 0);
    auto stage_row0 = [&](int i) { return i < R ? (i * grid + b) * SR : tr0; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = ptx::smem_addr(bars), empty0 = ptx::smem_addr(bars + S);

    for (int i = threadIdx.x; i < TW * MR * rpc; i += kThreads) ysm[i] = 0.f;
    // Thread 0 is the producer (warp 0, lane 0); it takes the SM's hand-off
    // ticket before this grid lets the next one launch, so that on every SM
    // the tickets follow the order of the calls (a CTA of a later call that
    // took an earlier ticket would hold this one back until the hand-off's
    // time bound).
    // A CTA that finds a CTA of its own grid ahead of it on the SM (the grid
    // did not fit one CTA per SM beside the previous call) does not wait.
    uint32_t smid = 0;
    unsigned long long ticket = 0;
    bool same_grid = false;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(full0 + 8 * s, 1);
            ptx::mbar_init(empty0 + 8 * s, kCW);
        }
        ptx::fence_mbar_init();
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        if (smid < (uint32_t)kMaxSm) {
            unsigned long long gid;
            asm volatile("mov.u64 %0, %%gridid;" : "=l"(gid));
            ticket = atomicAdd(&g_sm_ticket[smid], 1ull);
            same_grid = atomicExch(&g_sm_grid[smid], gid) == gid;
        }
    }
    __syncthreads();
    // Let the next launch in the stream begin its own prologue (barrier set-up
    // and weight streaming) as this grid's CTAs retire.  Everything this grid
    // reads before grid_dependency_wait() is the packed weight, its scales and
    // biases.  Only a preceding kernel that itself allows an early start
    // (griddepcontrol.launch_dependents) can still be running then: in this
    // library that is this kernel or a copy kernel of the host-buffer calls,
    // which write none of them; qmm_quantize,
    // which does write them, never allows it, so a call after it starts only
    // once it has completed.  The header states the rule for other writers.
    ptx::grid_launch_dependents();

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0) {
            const uint8_t *wsrc = reinterpret_cast<const uint8_t *>(wq);
            const uint8_t *ssrc = reinterpret_cast<const uint8_t *>(scales);
            const uint8_t *bsrc = reinterpret_cast<const uint8_t *>(biases);
            const bool handoff = smid < (uint32_t)kMaxSm;
            if (handoff && !same_grid) {
                const uint64_t t0 = ptx::globaltimer_ns();
                for (;;) {
                    unsigned long long done;
                    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(done) : "l"(&g_sm_issued[smid]));
                    if (done >= ticket || ptx::globaltimer_ns() - t0 > kHandoffWaitNs) break;
                    __nanosleep(128);
                }
            }
            // Ring slot and phase advance without integer division.
            for (int i = 0, s = 0, ph = 0; i < nst; ++i) {
                if (i >= S) ptx::mbar_wait(empty0 + 8 * s, ph ^ 1, err);
                const int nr = min(SR, nrows - i * SR);
                const uint32_t wb = (uint32_t)(nr * row_bytes), sb = (uint32_t)(nr * sb_bytes);
                const uint32_t st = ptx::smem_addr(smem + (size_t)s * stage_bytes);
                const uint32_t bar = full0 + 8 * s;
                ptx::mbar_arrive_expect_tx(bar, wb + NSB * sb);
                const int64_t roff = stage_row0(i);
                ptx::bulk_g2s(st, wsrc + roff * row_bytes, wb, bar);
                ptx::bulk_g2s(st + SR * row_bytes, ssrc + roff * sb_bytes, sb, bar);
                if constexpr (!MX)
                    ptx::bulk_g2s(st + SR * row_bytes + SR * sb_bytes, bsrc + roff * sb_bytes, sb, bar);
                if (handoff && i == max(0, nst - 2)) atomicMax(&g_sm_issued[smid], ticket + 1);
                if (++s == S) {
                    s = 0;
                    ph ^= 1;
                }
            }
            if (handoff) atomicMax(&g_sm_issued[smid], ticket + 1);
            // The CTA must not exit while a copy into its ring can still land
            // (the consumers may have given up on a stage after a timeout).
            for (int i = max(0, nst - S); i < nst; ++i)
                ptx::mbar_drain(full0 + 8 * (i % S), (i / S) & 1, err);
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - 1;
        const int team = cw / TW, wt = cw - team * TW;
        const bool active = team < NT;
        const int spr = K / EPU;

        int sl[UPL];
        bool sv[UPL];
        int gi[UPL], soff[UPL];   // group index and byte offset of the slice (0 if unused)
#pragma unroll
        for (int u = 0; u < UPL; ++u) {
            sl[u] = (wt * 32 + lane) * UPL + u;
            sv[u] = active && sl[u] < spr;
            gi[u] = sv[u] ? (sl[u] * EPU) / group_size : 0;
            soff[u] = sv[u] ? sl[u] * 16 : 0;
        }

        // The activations may be the output of the preceding kernel in the
        // stream: wait for it (and for every earlier grid) to complete and
        // its writes to become visible to this grid.
        ptx::grid_dependency_wait();
        // Activations in 16-bit block fixed point per slice (see the header):
        // packed (lo, hi) int16 pairs in DP2A order, the slice's scale-back
        // 2^-sh, and the slice sum of the fixed-point values for the bias term.
        int xp[MR][UPL][4 * STEPS];
        float fsc[MR][UPL];
        float xsum[MR][UPL];
        // E2M1: -128 times the sum of x_int over each group of the slice (the
        // codes enter DP2A as 128 + 2e); nvfp4 has two groups per slice
        int xoff[MR][UPL][2];
#pragma unroll
        for (int m = 0; m < MR; ++m) {
#pragma unroll
            for (int u = 0; u < UPL; ++u) {
                const bool ok = sv[u] && m < M;
                uint32_t raw[EPU / 2];  // the slice's 16-bit elements, two per word
#pragma unroll
                for (int c = 0; c < EPU / 8; ++c) {
                    const uint4 r = ok ? *reinterpret_cast<const uint4 *>(
                                             x + (int64_t)m * K + (int64_t)sl[u] * EPU + 8 * c)
                                       : make_uint4(0, 0, 0, 0);
                    raw[4 * c] = r.x;
                    raw[4 * c + 1] = r.y;
                    raw[4 * c + 2] = r.z;
                    raw[4 * c + 3] = r.w;
                }
                // Largest |x|: the bit patterns of non-negative IEEE values
                // order as the values, so a packed unsigned 16-bit max of the
                // words with their sign bits cleared finds it.
                uint32_t mx2 = 0;
#pragma unroll
                for (int q = 0; q < EPU / 2; ++q) mx2 = ptx::max_u16x2(mx2, raw[q] & 0x7FFF7FFFu);
                const uint32_t mbits = max(mx2 & 0xFFFFu, mx2 >> 16);
                const float amax = kBF16 ? __uint_as_float(mbits << 16)
                                         : __half2float(__ushort_as_half((unsigned short)mbits));
                // amax < 2^ex (ex = biased exponent - 126); x * 2^sh < 2^14 with
                // sh = 14 - ex, clamped so that 2^sh and 2^-sh are normal floats
                // (the lower clamp is reached by no finite 16-bit value: bf16
                // stays below 2^128, so sh >= -114).
                const int ex = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126;
                const int sh = min(126, max(-126, 14 - ex));
                const float up = __uint_as_float((uint32_t)(127 + sh) << 23);
                fsc[m][u] = __uint_as_float((uint32_t)(127 - sh) << 23);
                // x_int = rint(x 2^sh) by adding 1.5 * 2^23: x 2^sh is exact and
                // |x 2^sh| < 2^14, so the sum rounds (to nearest, ties to even)
                // at the units place and its low 16 bits are x_int's two's
                // complement; the sum of the words, less the offsets, is the
                // exact sum of the x_int.
                uint32_t isum[2] = {0u, 0u};
#pragma unroll
                for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
                    for (int k = 0; k < STEPS; ++k) {
                        // affine: plane order; E2M1: consecutive pairs
                        const int e0 = MX ? 2 * k : Planes<BITS>::elem(k, 0);
                        const int e1 = MX ? 2 * k + 1 : Planes<BITS>::elem(k, 1);
                        const uint32_t lo = __float_as_uint(
                            __fmaf_rn(elem_to_f<kBF16>(raw, wd * EPW + e0), up, 12582912.0f));
                        const uint32_t hi = __float_as_uint(
                            __fmaf_rn(elem_to_f<kBF16>(raw, wd * EPW + e1), up, 12582912.0f));
                        xp[m][u][wd * STEPS + k] = (int)__byte_perm(lo, hi, 0x5410);
                        isum[NV && wd >= 2] += lo + hi;
                    }
                }
                constexpr uint32_t kOff = 0x4B400000u;  // the bits of 1.5 * 2^23
                if constexpr (MX) {
                    const int g0 = (int)(isum[0] - (NV ? EPU / 2 : EPU) * kOff);
                    const int g1 = NV ? (int)(isum[1] - (EPU / 2) * kOff) : 0;
                    xoff[m][u][0] = -128 * g0;
                    xoff[m][u][1] = -128 * g1;
                    xsum[m][u] = 0.f;
                } else {
                    xsum[m][u] = fsc[m][u] * (float)(int)(isum[0] - EPU * kOff);
                    xoff[m][u][0] = xoff[m][u][1] = 0;
                }
            }
        }

        for (int i = 0, s = 0, ph = 0; i < nst; ++i) {
            ptx::mbar_wait(full0 + 8 * s, ph, err);
            const uint8_t *st = smem + (size_t)s * stage_bytes;
            float part[V];
#pragma unroll
            for (int q = 0; q < V; ++q) part[q] = 0.f;
            // Rows of this stage: SR, except in the block's last stage.
            const int rows_here = nrows - i * SR;
            // A full stage computes all RPT rows without branches so their DP2A
            // chains interleave (rows past the block's end read stale but
            // in-bounds stage bytes and are dropped by the selects); the
            // block's last, partial stage skips a team's rows past its end,
            // which shortens the tail that every call waits for.
            auto rows = [&](auto full) {
                constexpr bool FULL = decltype(full)::value;
#pragma unroll
                for (int j = 0; j < RPT; ++j) {
                    const int jr = team + j * NT;           // row within the stage (< SR)
                    if constexpr (!FULL) {
                        if (jr >= rows_here) continue;
                    }
                    const bool rv = i * SR + jr < nrows;
                    const uint8_t *wrow = st + jr * row_bytes;
                    const uint8_t *srow = st + SR * row_bytes + jr * sb_bytes;
#pragma unroll
                    for (int u = 0; u < UPL; ++u) {
                        const uint4 wv = *reinterpret_cast<const uint4 *>(wrow + soff[u]);
                        const bool use = rv && sv[u];
                        if constexpr (MX) {
                            // X/2 of the slice's group (groups 2 slice and 2 slice + 1
                            // for nvfp4), exact in fp32
                            const float x0 = 0.5f * mxf::scale_value<MODE>(srow[gi[u]]);
                            [[maybe_unused]] const float x1 =
                                NV ? 0.5f * mxf::scale_value<MODE>(srow[gi[u] + 1]) : 0.f;
                            uint32_t v[8];
                            e2m1_word_to_u8(wv.x, v + 0);
                            e2m1_word_to_u8(wv.y, v + 2);
                            e2m1_word_to_u8(wv.z, v + 4);
                            e2m1_word_to_u8(wv.w, v + 6);
#pragma unroll
                            for (int m = 0; m < MR; ++m) {
                                // a: codes 0..15 (nvfp4: the first group), b: codes 16..31
                                int a0 = xoff[m][u][0], a1 = 0, b0 = xoff[m][u][1], b1 = 0;
#pragma unroll
                                for (int q = 0; q < 8; ++q) {
                                    int &c0 = (NV && q >= 4) ? b0 : a0;
                                    int &c1 = (NV && q >= 4) ? b1 : a1;
                                    // word q / 2, codes 4 (q % 2) .. +3: pairs (0,1) and (2,3)
                                    c0 = dp2a_lo(xp[m][u][(q >> 1) * STEPS + 2 * (q & 1)], v[q], c0);
                                    c1 = dp2a_hi(xp[m][u][(q >> 1) * STEPS + 2 * (q & 1) + 1], v[q], c1);
                                }
                                // (X/2 * 2^-sh) first, as for the affine scale below
                                float c = (x0 * fsc[m][u]) * (float)(a0 + a1);
                                if constexpr (NV) c = __fmaf_rn(x1 * fsc[m][u], (float)(b0 + b1), c);
                                part[m * RPT + j] += use ? c : 0.f;
                            }
                            continue;
                        }
                        const float sc = h16_to_f(*reinterpret_cast<const uint16_t *>(srow + gi[u] * 2), kBF16);
                        const float bi = h16_to_f(
                            *reinterpret_cast<const uint16_t *>(srow + SR * sb_bytes + gi[u] * 2), kBF16);
#pragma unroll
                        for (int m = 0; m < MR; ++m) {
                            int a0 = 0, a1 = 0;
                            dot_word<BITS>(wv.x, &xp[m][u][0 * STEPS], a0, a1);
                            dot_word<BITS>(wv.y, &xp[m][u][1 * STEPS], a0, a1);
                            dot_word<BITS>(wv.z, &xp[m][u][2 * STEPS], a0, a1);
                            dot_word<BITS>(wv.w, &xp[m][u][3 * STEPS], a0, a1);
                            // (s * 2^-sh) first: the integer sum times 2^-sh alone
                            // can exceed the fp32 range for activations near the
                            // top of bf16's range, while the product with s cannot
                            // unless the result itself does.
                            const float c = __fmaf_rn(sc * fsc[m][u], (float)(a0 + a1), bi * xsum[m][u]);
                            part[m * RPT + j] += use ? c : 0.f;
                        }
                    }
                }
            };
            if (active) {
                if (rows_here >= SR) rows(std::true_type{});
                else rows(std::false_type{});
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(empty0 + 8 * s);
            const float v = reduce_scatter<V>(part, lane);
            if (active && lane < V) {
                const int m = lane / RPT, j = lane - m * RPT;
                const int r = i * SR + team + j * NT;
                if (m < M && r < nrows) ysm[(wt * MR + m) * rpc + r] = v;
            }
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
        }
    }
    __syncthreads();
    // A row's team warps in a fixed order, so that results repeat bit for bit.
    for (int idx = threadIdx.x; idx < M * nrows; idx += kThreads) {
        const int m = idx / nrows, r = idx - m * nrows;
        float acc = 0.f;
        for (int t = 0; t < TW; ++t) acc += ysm[(t * MR + m) * rpc + r];
        const int i = min(r / SR, R);
        const int gr = stage_row0(i) + (r - i * SR);
        const T v = Dt<T>::from_f(acc + layer_bias<T>(bias, bias_value, gr));
        y[(int64_t)m * N + gr] = v;
        if (y2) y2[(int64_t)m * N + gr] = v;  // (host memory through its mapping)
    }
}

struct StreamPlan {
    int upl, tw, rpt, sr, stages, rpc, rounds, q, grid;
    size_t smem;
};

// Shared memory per CTA: one CTA per SM with a ring of at most 110 KB, so that
// the next call's CTA (launched early by programmatic dependent launch) fits
// beside it and fills its own ring while this one finishes.
constexpr size_t kSmemPerSm = 110 * 1024;

int rows_per_team_stage(int mr) { return mr == 4 ? 2 : 4; }

bool plan_stream(const QmmArgs &a, int mr, int ctas_per_sm, StreamPlan &p) {
    const int bits = a.bits;
    const int epu = 128 / bits;
    const int64_t spr = a.K / epu;
    p.upl = spr > 32 * kCW ? 2 : 1;
    p.tw = (int)((spr + 32 * p.upl - 1) / (32 * p.upl));
    if (p.tw > kCW) return false;
    const int nt = kCW / p.tw;
    p.rpt = rows_per_team_stage(mr);
    p.sr = nt * p.rpt;
    const int64_t row_bytes = a.K / 8 * bits;
    // per row: scales and biases (affine, 16-bit) or scale bytes (E2M1)
    const bool mx = a.mode != QMM_MODE_AFFINE;
    const int64_t sb_bytes = a.K / a.group_size * (mx ? 1 : 2);
    const int64_t stage = (int64_t)p.sr * (row_bytes + (mx ? 1 : 2) * sb_bytes);
    // One CTA per SM (more, in waves, when a CTA's rows would pass 2048 / mr
    // or its partial slots -- one per team warp, activation row and row --
    // 24 KB); fewer for small N.
    const int64_t ctas = (int64_t)num_sms() * ctas_per_sm;
    const int64_t cap = std::max<int64_t>(1, std::min<int64_t>(2048 / mr, 6144 / (p.tw * mr)));
    int64_t grid = std::min<int64_t>(ctas, a.N);
    if ((a.N + grid - 1) / grid > cap) grid = (a.N + cap - 1) / cap;
    if (grid > (1 << 30) / p.sr) return false;
    // R full rounds of sr-row stages over the grid, then q rows per CTA
    p.rounds = (int)(a.N / (grid * p.sr));
    const int64_t rem = a.N - (int64_t)p.rounds * grid * p.sr;
    p.q = (int)((rem + grid - 1) / grid);
    p.rpc = p.rounds * p.sr + p.q;
    p.grid = (int)grid;
    const size_t budget = kSmemPerSm / ctas_per_sm;
    const size_t slots = (size_t)p.tw * mr * p.rpc * 4;
    const size_t fixed = 16 * 8 + slots + 128;
    if ((size_t)stage * 2 + fixed > budget) return false;
    p.stages = (int)std::min<int64_t>(8, (int64_t)((budget - fixed) / stage));
    p.smem = (size_t)p.stages * stage + (size_t)2 * p.stages * 8 + slots;
    return p.stages >= 2;
}

// Variants whose activations and partials fit the register file without
// spilling (checked with ptxas -v): rows x slices per lane is bounded by the
// codes per slice (32 for 4-bit, 16 for 8-bit, 64 for 2-bit).
// The 4-row variant of 4-bit codes uses ~123 registers: one CTA per SM, so
// it gives up the overlap with the next call but reads the weight once for
// 3-4 rows (4 rows: 20.9 -> 17.5 us against two 2-row launches).
bool stream_variant_fits(int bits, int mr, int upl) {
    if (mr == 1) return bits != 2 || upl == 1;
    if (bits == 4) return (mr == 2 || mr == 4) && upl == 1;
    if (bits == 8) return mr == 2 || upl == 1;
    return false;
}

template <typename T, int BITS, int MR, int UPL, int MODE>
cudaError_t launch_stream(const QmmArgs &a, cudaStream_t s) {
    constexpr int RPT = MR == 4 ? 2 : 4;
    auto kern = qgemv_stream_kernel<T, BITS, MR, UPL, RPT, MODE>;
    // One CTA per SM (the next call's CTAs take the other half of the SM).
    StreamPlan p{};
    if (!plan_stream(a, MR, 1, p)) return cudaErrorInvalidValue;
    struct Tag;
    cudaError_t e = configure_once<Tag>(p.smem, [&]() {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
        if (r != cudaSuccess) return r;
        // All of the SM's unified L1/shared storage as shared memory, so that a
        // second CTA (of the next call) fits beside this one.
        r = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (r != cudaSuccess) return r;
        int got = 0;
        r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&got, kern, kThreads, p.smem);
        if (r != cudaSuccess) return r;
        return got < 1 ? cudaErrorInvalidConfiguration : cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    // Programmatic stream serialization: this grid may start while the
    // preceding kernel of the stream finishes (see grid_dependency_wait()).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T *>(a.x), a.wq,
                           static_cast<const T *>(a.scales), static_cast<const T *>(a.biases),
                           static_cast<T *>(a.y), (int)a.M, (int)a.N, (int)a.K, a.group_size,
                           p.rpc, p.rounds, p.q, p.stages, p.tw, static_cast<const T *>(a.bias), a.bias_value,
                           device_error_word(), static_cast<T *>(a.y2));
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

// One launch for rows [0, mr) of a (mr in {1, 2, 4}, a variant that fits).
template <typename T, int BITS, int MODE>
cudaError_t stream_rows(const QmmArgs &a, int mr, cudaStream_t s) {
    StreamPlan p{};
    if (!plan_stream(a, mr, 1, p)) return cudaErrorInvalidValue;
    if (mr == 1) {
        if (p.upl == 1) return launch_stream<T, BITS, 1, 1, MODE>(a, s);
        if constexpr (BITS != 2) return launch_stream<T, BITS, 1, 2, MODE>(a, s);
    }
    if constexpr (BITS != 2) {
        if (mr == 2 && p.upl == 1) return launch_stream<T, BITS, 2, 1, MODE>(a, s);
    }
    if constexpr (BITS == 8) {
        if (mr == 2) return launch_stream<T, BITS, 2, 2, MODE>(a, s);
    }
    if constexpr (BITS != 2) {
        if (mr == 4 && p.upl == 1) return launch_stream<T, BITS, 4, 1, MODE>(a, s);
    }
    return cudaErrorInvalidValue;
}

// Widest variant (4, 2 or 1 rows) that fits the registers for `rows`
// remaining activation rows (3 rows take the 4-row variant with one row
// unused: one pass over the weight instead of two); 0 if none does.
int pick_rows(const QmmArgs &a, int64_t rows) {
    for (int mr : {4, 2, 1}) {
        if (mr > rows && !(mr == 4 && rows == 3)) continue;
        QmmArgs t = a;
        t.M = mr;
        StreamPlan p{};
        if (plan_stream(t, mr, 1, p) && stream_variant_fits(a.bits, mr, p.upl)) return mr;
    }
    return 0;
}

// Rows go through the widest variant that fits, a launch per row block (for
// example 4-bit codes: 3 or 4 rows in one 4-row launch; 2-bit codes: 3 rows =
// 2 + 1).
template <typename T, int BITS, int MODE = QMM_MODE_AFFINE>
cudaError_t stream_bits(const QmmArgs &a, cudaStream_t s) {
    for (int64_t m0 = 0; m0 < a.M;) {
        const int mr = pick_rows(a, a.M - m0);
        if (mr == 0) return cudaErrorInvalidValue;
        QmmArgs t = a;
        t.M = std::min<int64_t>(mr, a.M - m0);
        t.x = static_cast<const T *>(a.x) + m0 * a.K;
        t.y = static_cast<T *>(a.y) + m0 * a.N;
        if (a.y2) t.y2 = static_cast<T *>(a.y2) + m0 * a.N;
        const cudaError_t e = stream_rows<T, BITS, MODE>(t, mr, s);
        if (e != cudaSuccess) return e;
        m0 += t.M;
    }
    return cudaSuccess;
}

}  // namespace

// Fast path: bf16/f16, transpose layout, 1..4 rows, whole 16-byte slices per
// row, scales/biases rows of whole 16-byte units, no group boundary inside a
// slice (group_size >= codes per slice; nvfp4: exactly two groups per slice),
// rows at most 12 warps wide.  Affine 2-, 4- and 8-bit codes, mxfp4, nvfp4.
bool gemv_fast_supported(qmm_dtype dt, const QmmArgs &a) {
    if (!a.transpose || a.M < 1 || a.M > 4) return false;
    if (dt != QMM_BF16 && dt != QMM_F16) return false;
    const int epu = 128 / a.bits;
    if (a.mode == QMM_MODE_AFFINE) {
        if (a.bits != 2 && a.bits != 4 && a.bits != 8) return false;
        if (a.K % epu != 0 || a.group_size < epu) return false;
        if ((a.K / a.group_size) % 8 != 0) return false;
    } else {
        if (a.mode != QMM_MODE_MXFP4 && a.mode != QMM_MODE_NVFP4) return false;
        if (a.bits != 4 || a.K % epu != 0) return false;
        if ((a.K / a.group_size) % 16 != 0) return false;  // scale rows of whole 16-byte units
    }
    if (a.N > (1 << 30) || a.K > (1 << 24)) return false;
    if ((reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases) |
         reinterpret_cast<uintptr_t>(a.wq)) & 15)
        return false;
    // Every row block must find a variant; one-row launches always can when
    // the single-row plan fits.
    return pick_rows(a, 1) == 1;
}

cudaError_t launch_gemv_fast(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    a.y2_written = a.y2 != nullptr;
    if (a.mode == QMM_MODE_MXFP4)
        return dt == QMM_BF16 ? stream_bits<__nv_bfloat16, 4, QMM_MODE_MXFP4>(a, s)
                              : stream_bits<__half, 4, QMM_MODE_MXFP4>(a, s);
    if (a.mode == QMM_MODE_NVFP4)
        return dt == QMM_BF16 ? stream_bits<__nv_bfloat16, 4, QMM_MODE_NVFP4>(a, s)
                              : stream_bits<__half, 4, QMM_MODE_NVFP4>(a, s);
    if (dt == QMM_BF16) {
        switch (a.bits) {
        case 2: return stream_bits<__nv_bfloat16, 2>(a, s);
        case 4: return stream_bits<__nv_bfloat16, 4>(a, s);
        default: return stream_bits<__nv_bfloat16, 8>(a, s);
        }
    }
    switch (a.bits) {
    case 2: return stream_bits<__half, 2>(a, s);
    case 4: return stream_bits<__half, 4>(a, s);
    default: return stream_bits<__half, 8>(a, s);
    }
}

}  // namespace qmm
