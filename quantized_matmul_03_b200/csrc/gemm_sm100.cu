// gemm_sm100.cu -- tensor-core quantized matmul for many activation rows
// (prefill):  y[m, n] = sum_k x[m, k] * (s[n,g] q[n,k] + b[n,g])  with W stored
// [N, K] (mlx-rs ops/quantization.rs, quantized_matmul; Emily
// Quantization.Layers, quantized_dense with transpose: true), and x @ W with W
// stored [K, N].  The dense weight never exists in global memory: each 128 x 64
// tile is dequantized on chip right before the tensor cores consume it.
//
// Orientation ("swap AB"): the UMMA M dimension (128) runs over weight rows n
// and the UMMA N dimension (BN = 16..256) over activation rows m, so the
// dequantized tile is the A operand and the activations are the B operand:
//     D[n, m] (TMEM, fp32) += W~[n, k] * x[m, k]   for k-blocks of 64.
// The activations are K-major bf16/f16 in the canonical 128-byte-swizzle
// layout (8-row x 128-byte atoms, row r's 16-byte chunk c at chunk c ^ (r mod 8)).
//
// Where the dequantized tile lives:
//   [N, K] layout  tensor memory (tcgen05.st by the dequantize threads, MMA in
//                  its TMEM-A form).  Shared memory then carries only the
//                  activation, packed-code and scale/bias tiles, which keeps
//                  the per-SM shared-memory traffic (TMA writes + tensor-core
//                  reads + the dequantize threads' reads) below its ceiling
//                  and frees room for ring stages and an output staging slab;
//   [K, N] layout  and the grouped (gather) product: a swizzled shared-memory
//                  tile (MN-major for [K, N], K-major for grouped).
//
// Roles (one CTA per SM, persistent over output tiles):
//   warps 0-7   dequantize, as two groups of four warps taking alternate
//               k-blocks; thread r of a group owns weight row r, reads the
//               packed codes and scale/bias windows the producers staged,
//               forms s*q + b two codes at a time (bf16x2/f16x2 FMA, one
//               rounding) and writes its row of the A tile;
//   warps 8-11  epilogue: tcgen05.ld of the accumulator quadrant the warp may
//               address (lanes 32*(warp%4)..), convert, then either stage the
//               values in shared memory for one tensor store per slab or
//               store y directly (grouped rows, wide [K, N] tiles, unaligned
//               y); under stream-K a CTA that stops inside a tile leaves an
//               fp32 partial in the caller's workspace, and the CTA holding
//               the tile's last k-block adds it before storing;
//   warps 12,14,15  producers: TMA loads of the packed weight tile, the
//               activation tile and the scale/bias windows of each k-block
//               into a ring of stages;
//   warp 13     MMA issuer (one thread) and TMEM owner.
// Every wait is a bounded mbarrier wait (device error word on timeout); no
// cluster multicast is used.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mx.cuh"
#include "ptx_sm100.cuh"
#include "qmm_internal.cuh"
#include "tcgen05.cuh"

namespace qmm {
namespace {

constexpr int kDqWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kWarpTma = kDqWarps + kEpiWarps;  // 12: packed-tile loads
constexpr int kWarpMma = kWarpTma + 1;          // 13
constexpr int kWarpTmaB = kWarpMma + 1;         // 14: activation loads
constexpr int kWarpTmaS = kWarpMma + 2;         // 15: scale/bias window loads
constexpr int kThreads = 32 * (kWarpTmaS + 1);  // 512
constexpr int kBM = 128;                        // weight rows per tile (UMMA M)
constexpr int kBK = 64;                         // k per stage: one 128-byte swizzle row
constexpr int kSkMaxBN = 64;                    // widest tile that stream-K splits
// Packed tile of one k-block, [N, K] layout: 128 rows of kBK*bits/8 bytes
// (3-bit codes: 24 bytes, which no tensor copy can start on for odd k-blocks,
// so a 32-byte box from the 16-byte boundary below is staged instead).
// [K, N] layout: 64 k-rows of 128*bits/8 bytes.
constexpr int packed_pitch(int bits) { return bits == 3 ? 32 : kBK * bits / 8; }
constexpr int packed_stage_bytes(int bits, bool kmajor) {
    return kmajor ? kBM * packed_pitch(bits) : kBK * kBM * bits / 8;
}

// ---------------------------------------------------------------------------
// Dequantization of a half k-block of one weight row (32 codes) into four
// 16-byte chunks of 16-bit values, two codes per FMA.
// ---------------------------------------------------------------------------
template <typename T> struct Pair;
template <> struct Pair<__nv_bfloat16> {
    using V2 = __nv_bfloat162;
    static constexpr uint32_t MAGIC = 0x43004300u;  // 128.0 | 128.0
    static __device__ __forceinline__ V2 bits(uint32_t u) { return *reinterpret_cast<V2 *>(&u); }
    static __device__ __forceinline__ uint32_t ubits(V2 v) { return *reinterpret_cast<uint32_t *>(&v); }
    static __device__ __forceinline__ V2 off() { return __float2bfloat162_rn(128.f); }
    static __device__ __forceinline__ V2 splat(uint16_t h) {
        __nv_bfloat16 b = *reinterpret_cast<__nv_bfloat16 *>(&h);
        return __bfloat162bfloat162(b);
    }
};
template <> struct Pair<__half> {
    using V2 = __half2;
    static constexpr uint32_t MAGIC = 0x64006400u;  // 1024.0 | 1024.0
    static __device__ __forceinline__ V2 bits(uint32_t u) { return *reinterpret_cast<V2 *>(&u); }
    static __device__ __forceinline__ uint32_t ubits(V2 v) { return *reinterpret_cast<uint32_t *>(&v); }
    static __device__ __forceinline__ V2 off() { return __float2half2_rn(1024.f); }
    static __device__ __forceinline__ V2 splat(uint16_t h) {
        __half b = *reinterpret_cast<__half *>(&h);
        return __half2half2(b);
    }
};

// 3- and 6-bit codes: the 32 codes fill BITS words as one bit stream, code j
// at bits [j*BITS, (j+1)*BITS), so a pair of codes (2i, 2i+1) is the 2*BITS
// bits from bit 2i*BITS, which may straddle two words (one funnel shift).
// The pair goes to the two 16-bit halves, then the magic-number conversion.
template <typename T, int BITS>
__device__ __forceinline__ void dequant_half_stream(const uint32_t *w, uint16_t s16, uint16_t b16,
                                                    uint4 (&out)[4]) {
    using P = Pair<T>;
    using V2 = typename P::V2;
    constexpr uint32_t M = (1u << BITS) - 1u;
    const V2 s2 = P::splat(s16), b2 = P::splat(b16), off = P::off();
    uint32_t vals[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int pos = 2 * i * BITS, wi = pos >> 5, sh = pos & 31;
        const uint32_t u = sh + 2 * BITS <= 32 ? (w[wi] >> sh) : __funnelshift_r(w[wi], w[wi + 1], sh);
        const uint32_t t = (u & M) | ((u << (16 - BITS)) & (M << 16)) | P::MAGIC;
        vals[i] = P::ubits(__hfma2(__hsub2(P::bits(t), off), s2, b2));
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
        out[c] = make_uint4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
}

// Magic-number path (4- and 2-bit codes; 8-bit codes with f16): OR a code
// into the mantissa of OFF (exact), subtract OFF (exact), then s*q + b.
// Produces 16-bit values in k order, 8 per output uint4.  (3- and 6-bit
// codes: dequant_half_stream.)
template <typename T, int BITS>
__device__ __forceinline__ void dequant_half(const uint32_t *w, uint16_t s16, uint16_t b16,
                                             uint4 (&out)[4]) {
    if constexpr (BITS == 3 || BITS == 6) {
        dequant_half_stream<T, BITS>(w, s16, b16, out);
        return;
    } else {
    using P = Pair<T>;
    using V2 = typename P::V2;
    constexpr int EPW = 32 / BITS;                 // codes per word
    constexpr int NW = 32 / EPW;                   // words per 32 codes
    constexpr uint32_t MASK = BITS == 8 ? 0x00FF00FFu : (BITS == 4 ? 0x000F000Fu : 0x00030003u);
    const V2 s2 = P::splat(s16), b2 = P::splat(b16), off = P::off();
    uint32_t vals[16];  // 32 values as 16 pairs (2i, 2i+1)
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) {
        // step e yields codes (e, e + EPW/2) of the word
        uint32_t pe[EPW / 2];
#pragma unroll
        for (int e = 0; e < EPW / 2; ++e) {
            const uint32_t t = ((w[wi] >> (BITS * e)) & MASK) | P::MAGIC;
            const V2 q = __hsub2(P::bits(t), off);
            pe[e] = P::ubits(__hfma2(q, s2, b2));
        }
        // re-pair (e, e+H) into consecutive pairs (2i, 2i+1)
        constexpr int H = EPW / 2;
#pragma unroll
        for (int i = 0; i < EPW / 2; ++i) {
            const int a = 2 * i, b = 2 * i + 1;  // element indices within the word
            const uint32_t ra = pe[a % H], rb = pe[b % H];
            const uint32_t sel = (a < H ? 0x0010u : 0x0032u) | (b < H ? 0x5400u : 0x7600u);
            vals[wi * (EPW / 2) + i] = __byte_perm(ra, rb, sel);
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
        out[c] = make_uint4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
    }
}

// 8-bit codes with bf16 (no exact bf16 magic for 0..255): fp32 magic.
template <>
__device__ __forceinline__ void dequant_half<__nv_bfloat16, 8>(const uint32_t *w, uint16_t s16,
                                                               uint16_t b16, uint4 (&out)[4]) {
    const float s = __uint_as_float((uint32_t)s16 << 16), b = __uint_as_float((uint32_t)b16 << 16);
    uint32_t vals[16];
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) {
        float f[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float q = __uint_as_float(__byte_perm(w[wi], 0x4B000000u, 0x7650u + e)) - 8388608.f;
            f[e] = __fmaf_rn(s, q, b);
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]), hi = __floats2bfloat162_rn(f[2], f[3]);
        vals[2 * wi] = *reinterpret_cast<uint32_t *>(&lo);
        vals[2 * wi + 1] = *reinterpret_cast<uint32_t *>(&hi);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
        out[c] = make_uint4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
}

// Microscaled weights (mxfp4/nvfp4: E2M1 codes, mxfp8: E4M3 codes): 32
// elements of one row as 16-bit values X * element, exact (both factors are
// exact in 16 bits and so is their product); x0 scales elements 0..15, x1
// elements 16..31 (equal unless the group size is 16).
template <typename T, int MODE>
__device__ __forceinline__ void dequant_half_mx(const uint32_t *w, float x0, float x1, uint4 (&out)[4]) {
    constexpr int NW = MODE == QMM_MODE_MXFP8 ? 8 : 4;  // words per 32 elements
    uint32_t vals[16];
#pragma unroll
    for (int wi = 0; wi < NW; ++wi) {
        float e[32 / NW];  // elements of one word
        mxf::elements<MODE>(w[wi], e);
        const float x = wi < NW / 2 ? x0 : x1;
#pragma unroll
        for (int i = 0; i < 16 / NW; ++i) {
            const float a = __fmul_rn(x, e[2 * i]), b = __fmul_rn(x, e[2 * i + 1]);
            uint32_t pr;
            if constexpr (std::is_same<T, __half>::value) {
                const __half2 h = __floats2half2_rn(a, b);
                pr = *reinterpret_cast<const uint32_t *>(&h);
            } else {
                const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                pr = *reinterpret_cast<const uint32_t *>(&h);
            }
            vals[wi * (16 / NW) + i] = pr;
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
        out[c] = make_uint4(vals[4 * c], vals[4 * c + 1], vals[4 * c + 2], vals[4 * c + 3]);
}

// Position of k-block c in a ring of n stages -- slot c mod n, phase parity
// (c div n) mod 2, and whether c >= n -- advanced one k-block at a time
// without integer division.
struct RingPos {
    int slot = 0, phase = 0;
    bool wrapped = false;
    __device__ __forceinline__ void next(int n) {
        if (++slot == n) {
            slot = 0;
            phase ^= 1;
            wrapped = true;
        }
    }
};


struct GemmParams {
    const void *scales, *biases;
    void *y;
    int M, N, K, group_size;
    int m_tiles, n_tiles, num_tiles, stages;
    int sb_tma;  // [N, K] layout: scale/bias windows arrive by TMA with each stage
    int stg_rows;  // output rows staged per tensor store (0: direct stores)
    // Stream-K (narrow tiles with the staged epilogue): CTA b works through
    // k-blocks [b*sk_len, (b+1)*sk_len) of the (tile, k-block) space.
    // sk_len = 0: whole tiles blockIdx.x, + gridDim.x, ...
    int sk_len;
    float *sk_ws;    // per CTA: one fp32 partial tile, [quadrant][chunk][lane][CW]
    int *sk_flags;   // per CTA and quadrant: 1 while its partial awaits the tile's owner
    int sk_no_publish;  // test injection: parts are written but their flags never raised
    const void *bias;   // layer bias [N] or null, plus bias_value (not in grouped mode)
    float bias_value;
    int *err;
    // Grouped (gather_qmm) mode only: the chunk table and row map the
    // preparation kernel wrote.  Tile t covers chunk t / n_tiles and weight
    // rows (t % n_tiles) * 128 of that chunk's expert.
    const GatherHeader *hdr;
    const int4 *chunks;     // {expert, first sorted row, rows, 0}
    const int32_t *dst_rows;  // sorted activation row -> output row
};

// What one CTA needs to know about an output tile.
struct Tile {
    int n0;     // first output feature (weight row within the expert)
    int wrow0;  // first row of the stacked weight (expert * N + n0)
    int m0;     // first activation row (of x, or of the sorted rows)
    int rows;   // activation rows in the tile
};

template <int BN, bool GROUPED>
__device__ __forceinline__ Tile decode_tile(const GemmParams &p, int tile) {
    Tile t;
    if constexpr (GROUPED) {
        const int4 c = __ldg(p.chunks + tile / p.n_tiles);
        t.n0 = (tile % p.n_tiles) * kBM;
        t.wrow0 = c.x * p.N + t.n0;
        t.m0 = c.y;
        t.rows = c.z;
    } else {
        t.n0 = (tile / p.m_tiles) * kBM;
        t.wrow0 = t.n0;
        t.m0 = (tile % p.m_tiles) * BN;
        t.rows = min(BN, p.M - t.m0);
    }
    return t;
}

template <bool GROUPED>
__device__ __forceinline__ int tile_count(const GemmParams &p) {
    if constexpr (GROUPED) return __ldg(&p.hdr->num_chunks) * p.n_tiles;
    else return p.num_tiles;
}

// One unit of a CTA's work: k-blocks [kb0, kb1) of output tile `tile`.
struct Unit {
    int tile, kb0, kb1;
};

// The units of one CTA, identical for every role: whole tiles blockIdx.x,
// + gridDim.x, ...; or, under stream-K, the CTA's run of the (tile, k-block)
// space walked from its end, so a tile split between CTAs b and b+1 is
// finished last by b+1 (which combines the parts) after b wrote its part
// first -- a waiting CTA only ever waits for lower-numbered ones.
struct Work {
    int next, stride, count, KB;  // whole tiles
    int cur, begin;               // stream-K
    __device__ Work(const GemmParams &p, int num_tiles, int KB_) {
        KB = KB_;
        next = blockIdx.x;
        stride = gridDim.x;
        const bool sk = p.sk_len > 0;
        count = sk ? 0 : num_tiles;
        begin = sk ? (int)blockIdx.x * p.sk_len : 0;
        cur = sk ? min(num_tiles * KB, begin + p.sk_len) : 0;
    }
    __device__ bool get(Unit &u) {
        if (next < count) {
            u.tile = next;
            u.kb0 = 0;
            u.kb1 = KB;
            next += stride;
            return true;
        }
        if (cur <= begin) return false;
        const int tile = (cur - 1) / KB;  // once per unit, not per k-block
        const int ts = tile * KB;
        u.tile = tile;
        u.kb0 = max(ts, begin) - ts;
        u.kb1 = cur - ts;
        cur = ts + u.kb0;
        return true;
    }
};

// GROUPED: gather_qmm's grouped product.  Activation tiles then arrive as
// 64-row boxes (only as many as the chunk has rows), from tmap_xs (the sorted
// copy) or tmap_x (x itself, when the sorted order is x's own); the MMA N is
// the chunk's row count rounded up to 16; outputs go through the row map.
//
// KMAJOR = false: the weight is stored [K, N] (transpose = false), packed and
// grouped along N.  Each 64 x 128 packed tile (64 k-rows of 128 features)
// arrives by TMA; dequantize thread (k, h) expands the 64 features of half h
// of row k and writes them as 16-byte chunks of an MN-major, 128-byte-swizzled
// A tile (atoms of 64 features x 8 k-rows), which the MMA reads with the
// A-major bit set.  Everything else is shared with the K-major path.
// MODE: affine (scale and bias windows, 16-bit) or a microscaled mode
// (scale bytes only: windows of 16 groups; [N, K] layout, not grouped).
template <typename T, int BITS, int BN, bool GROUPED, bool KMAJOR = true, int MODE = QMM_MODE_AFFINE>
__global__ void __launch_bounds__(kThreads, 1)
qgemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_xs,
                const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_s,
                const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_y,
                const GemmParams p) {
    static_assert(KMAJOR || !GROUPED, "the grouped product is built for the [N, K] layout");
    constexpr bool MX = MODE != QMM_MODE_AFFINE;
    static_assert(!MX || (KMAJOR && !GROUPED), "microscaled weights: [N, K] layout, not grouped");
    constexpr bool kF16 = std::is_same<T, __half>::value;
    constexpr int A_BYTES = kBM * kBK * 2;         // 16 KB dequantized tile
    constexpr int B_BYTES = BN * kBK * 2;          // activation tile
    constexpr int P_ROW = packed_pitch(BITS);      // staged packed bytes per row per k-block
    constexpr int P_BYTES = packed_stage_bytes(BITS, KMAJOR);
    constexpr int W_WORDS = kBK * BITS / 32;       // packed words per row per k-block
    // [N, K] layout: the dequantized tile goes to tensor memory (A operand of
    // the MMA) instead of shared memory.  512 columns: accumulators (two
    // buffers, or one of 256 columns) then a ring of 32-column A slots.
    // (Shared-memory A measured slower at every tile width, narrow tiles
    // included: 16 activation rows, 14336 x 4096 int4: 26.8 against 24.4 us.)
    constexpr bool TS = KMAJOR && !GROUPED;
    constexpr int NACC = (TS && 2 * BN > 256) ? 1 : 2;
    constexpr uint32_t A_COL0 = NACC * BN < 32 ? 32 : NACC * BN;
    constexpr uint32_t TMEM_COLS = TS ? 512 : (2 * BN < 32 ? 32 : 2 * BN);
    // Split stage barriers (below) for the wide TMEM-A tiles, where the TMA
    // latency of the packed tile is on the critical chain; elsewhere one
    // barrier per stage (measured faster for narrow tiles and [K, N]).
    constexpr bool SPLIT = TS && BN >= 128;
    constexpr uint32_t IDESC = make_idesc(kF16, kBM, BN, !KMAJOR);
    // MN-major A tile: feature atoms (64 features) 1 KB apart, 8-k-row groups 2 KB apart.
    constexpr uint32_t MN_LBO = 1024, MN_SBO = 2048;

    extern __shared__ uint8_t smem_raw[];
    const int S = p.stages;
    // 1024-byte aligned carve-up: A[S] (shared-memory A only) | B[S] | P[S] |
    // scale/bias windows[S] | output slabs | barriers | tmem slot
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const uint32_t a0 = base, b0 = a0 + (TS ? 0 : S * A_BYTES), p0 = b0 + S * B_BYTES;
    // Scale/bias windows ([N, K] layout with sb_tma): per stage 8 groups x 128
    // rows of scales (2 KB) then of biases (2 KB), row r at byte 16 r.
    constexpr int SB_BYTES = 2 * kBM * 16;
    const uint32_t sb0 = p0 + S * P_BYTES;
    // Output staging: one slab of stg_rows x 32 values per epilogue warp.
    const uint32_t out0 = sb0 + (p.sb_tma ? S * SB_BYTES : 0);
    const uint32_t bar0 = out0 + (uint32_t)kEpiWarps * 64u * (uint32_t)p.stg_rows;
    // Per stage: full_p (packed tile + scale/bias windows landed; without
    // SPLIT also the activation tile), full_b (activation tile landed, SPLIT
    // only), full_a (A tile written), p_empty (SPLIT only: the dequantize
    // group has read the packed tile and windows, which can be refilled
    // before the MMA runs), b_empty (the MMAs of the stage are done:
    // activation tile and A slot free; without SPLIT the whole stage).
    const uint32_t full_p = bar0, full_b = bar0 + 8 * S, full_a = bar0 + 16 * S;
    const uint32_t p_empty = bar0 + 24 * S, b_empty = bar0 + 32 * S;
    // done: the MMA issuer's last tcgen05.mma has completed (tensor memory
    // may be freed).
    const uint32_t acc_full = bar0 + 40 * S, acc_empty = acc_full + 16, done = acc_empty + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + (done + 8 - base));
    const uint8_t *pg = gbase + (p0 - base);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // one arrival per producer warp that signals the barrier
            ptx::mbar_init(full_p + 8 * s, (p.sb_tma ? 2 : 1) + (SPLIT ? 0 : 1));
            ptx::mbar_init(full_b + 8 * s, 1);
            ptx::mbar_init(full_a + 8 * s, kDqWarps / 2);  // one dequant group per k-block
            ptx::mbar_init(p_empty + 8 * s, kDqWarps / 2);
            ptx::mbar_init(b_empty + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(acc_full + 8 * a, 1);
            ptx::mbar_init(acc_empty + 8 * a, kEpiWarps);
        }
        ptx::mbar_init(done, 1);
        ptx::fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(ptx::smem_addr(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int KB = (p.K + kBK - 1) / kBK;
    const int gpr = p.K / p.group_size;
    const int num_tiles = tile_count<GROUPED>(p);

    if (!KMAJOR && warp < kDqWarps) {
        // --------------- dequantize, weight stored [K, N] ---------------
        // Thread t of a group: k-row kl = (t mod 8) + 8 (t div 16), feature
        // half h = (t div 8) mod 2, so the 8 threads of a store phase cover 8
        // different k-rows of one half (conflict-free 16-byte stores).
        const int grp = warp >> 2, t = threadIdx.x & (kBM - 1);
        const int kl = (t & 7) + 8 * (t >> 4), h = (t >> 3) & 1;
        const uint16_t *sc = static_cast<const uint16_t *>(p.scales);
        const uint16_t *bi = static_cast<const uint16_t *>(p.biases);
        const int gs_log = __ffs(p.group_size) - 1;  // group_size is a power of two
        const int gpn = p.N >> gs_log;                 // groups per stored row
        int c = 0;
        RingPos rp;
        Work wk(p, num_tiles, KB);
        for (Unit u; wk.get(u);) {
            const Tile tl = decode_tile<BN, GROUPED>(p, u.tile);
            const int f0 = tl.n0 + 64 * h;  // first feature of this thread's half
            const bool v0 = f0 < p.N, v1 = f0 + 32 < p.N;
            const int g0 = f0 >> gs_log, g1 = (f0 + 32) >> gs_log;
            for (int kb = u.kb0; kb < u.kb1; ++kb, ++c, rp.next(S)) {
                if ((c & 1) != grp) continue;
                const int s = rp.slot;
                const int64_t srow = (int64_t)(kb * kBK + kl) * gpn;
                const uint16_t s0 = v0 ? __ldg(sc + srow + g0) : (uint16_t)0;
                const uint16_t b0v = v0 ? __ldg(bi + srow + g0) : (uint16_t)0;
                const uint16_t s1 = v1 ? __ldg(sc + srow + g1) : (uint16_t)0;
                const uint16_t b1v = v1 ? __ldg(bi + srow + g1) : (uint16_t)0;
                ptx::mbar_wait(full_p + 8 * s, rp.phase, p.err);
                // Packed row kl (16*BITS bytes, unswizzled), half h.
                const uint8_t *prow = pg + s * P_BYTES + kl * (16 * BITS) + h * (8 * BITS);
                uint32_t w[2 * BITS];
                if constexpr (BITS == 3) {  // 24 bytes, 8-byte aligned
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        const uint2 u = *reinterpret_cast<const uint2 *>(prow + 8 * q);
                        w[2 * q] = u.x; w[2 * q + 1] = u.y;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < BITS / 2; ++q) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(prow + 16 * q);
                        w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
                    }
                }
                // A stage s is free: its refill (full_p above) waited for the
                // MMAs of k-block c - S.
                uint8_t *arow = gbase + (a0 - base) + s * A_BYTES + (kl >> 3) * MN_SBO + h * MN_LBO +
                                (kl & 7) * 128;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint4 out[4];
                    dequant_half<T, BITS>(w + hh * BITS, hh ? s1 : s0, hh ? b1v : b0v, out);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int chunk = 4 * hh + j;
                        *reinterpret_cast<uint4 *>(arow + ((chunk ^ (kl & 7)) << 4)) = out[j];
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(full_a + 8 * s);
            }
        }
    } else if (warp < kDqWarps) {
        // ------------------------- dequantize -------------------------
        // Two groups of four warps take alternate k-blocks, so two k-blocks
        // are dequantized at once; thread r of a group owns weight row r.
        const int grp = warp >> 2, r = threadIdx.x & (kBM - 1);
        const uint16_t *sc = static_cast<const uint16_t *>(p.scales);
        const uint16_t *bi = static_cast<const uint16_t *>(p.biases);
        // Scales/biases are read 8 groups (16 bytes) at a time, one window
        // ahead of use, when rows are whole 16-byte units; else one by one.
        const bool vec = (gpr % 8) == 0;
        const int gs_log = __ffs(p.group_size) - 1;  // group_size is a power of two
        int c = 0;
        RingPos rp;
        Work wk(p, num_tiles, KB);
        for (Unit u; wk.get(u);) {
            const Tile t = decode_tile<BN, GROUPED>(p, u.tile);
            const bool rv = t.n0 + r < p.N;
            const int64_t wrow = (int64_t)t.wrow0 + r;
            const uint16_t *srow = sc + wrow * gpr, *brow = bi + wrow * gpr;
            uint4 s_cur = make_uint4(0, 0, 0, 0), b_cur = s_cur, s_nxt = s_cur, b_nxt = s_cur;
            int wbase = 0;  // first group of the current window
            if (vec && rv && !p.sb_tma) {
                s_cur = __ldg(reinterpret_cast<const uint4 *>(srow));
                b_cur = __ldg(reinterpret_cast<const uint4 *>(brow));
                if (gpr > 8) {
                    s_nxt = __ldg(reinterpret_cast<const uint4 *>(srow + 8));
                    b_nxt = __ldg(reinterpret_cast<const uint4 *>(brow + 8));
                }
            }
            auto scale_bias = [&](int g, uint16_t &s16, uint16_t &b16) {
                if (vec) {
                    while (g >= wbase + 8) {  // advance the window, fetch the one after
                        s_cur = s_nxt;
                        b_cur = b_nxt;
                        wbase += 8;
                        if (rv && wbase + 8 < gpr) {
                            s_nxt = __ldg(reinterpret_cast<const uint4 *>(srow + wbase + 8));
                            b_nxt = __ldg(reinterpret_cast<const uint4 *>(brow + wbase + 8));
                        }
                    }
                    const int o = g - wbase;
                    const uint32_t sw = pick_word(s_cur, o >> 1), bw = pick_word(b_cur, o >> 1);
                    s16 = (uint16_t)((o & 1) ? (sw >> 16) : (sw & 0xffffu));
                    b16 = (uint16_t)((o & 1) ? (bw >> 16) : (bw & 0xffffu));
                } else {
                    s16 = rv ? __ldg(srow + g) : (uint16_t)0;
                    b16 = rv ? __ldg(brow + g) : (uint16_t)0;
                }
            };
            for (int kb = u.kb0; kb < u.kb1; ++kb, ++c, rp.next(S)) {
                if ((c & 1) != grp) continue;
                const int s = rp.slot;
                uint16_t s0, b0v, s1, b1v;
                const int g0 = (kb * kBK) >> gs_log, g1 = (kb * kBK + 32) >> gs_log;
                if (!p.sb_tma) {
                    scale_bias(g0, s0, b0v);
                    scale_bias(g1, s1, b1v);
                }
                ptx::mbar_wait(full_p + 8 * s, rp.phase, p.err);
                float mx[4] = {0.f, 0.f, 0.f, 0.f};  // microscaled: scales of elements 16i..16i+15
                if constexpr (MX) {
                    // Row r's window of 16 scale bytes starts at group (g & ~15).
                    const uint8_t *sw = gbase + (sb0 - base) + s * SB_BYTES + r * 16;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        mx[i] = mxf::scale_value<MODE>(sw[((kb * kBK + 16 * i) >> gs_log) & 15]);
                } else if (p.sb_tma) {
                    // Row r's window of 8 groups starts at group (g0 & ~7).
                    const uint8_t *sw = gbase + (sb0 - base) + s * SB_BYTES + r * 16;
                    const int o0 = (g0 & 7) * 2, o1 = (g1 - (g0 & ~7)) * 2;
                    s0 = *reinterpret_cast<const uint16_t *>(sw + o0);
                    b0v = *reinterpret_cast<const uint16_t *>(sw + SB_BYTES / 2 + o0);
                    s1 = *reinterpret_cast<const uint16_t *>(sw + o1);
                    b1v = *reinterpret_cast<const uint16_t *>(sw + SB_BYTES / 2 + o1);
                }
                // The packed tile was staged with the swizzle matching its row
                // width (none / 32B / 64B): 16-byte chunk q of row r sits at
                // chunk q ^ ((r >> 2) & 1) (32-byte rows) or q ^ ((r >> 1) & 3)
                // (64-byte rows); 48-byte rows (6-bit codes) are unswizzled.
                const uint8_t *prow = pg + s * P_BYTES + r * P_ROW;
                uint32_t w[2 * BITS];  // 64 codes
                if constexpr (BITS == 2) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(prow);
                    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
                } else if constexpr (BITS == 3) {
                    // 32-byte row staged from word (6 kb) & ~3: the k-block's six
                    // words start at word 0 (even kb) or 2 (odd kb).
                    const int x = (r >> 2) & 1;
                    uint32_t a8[8];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(prow + ((q ^ x) << 4));
                        a8[4 * q] = u.x; a8[4 * q + 1] = u.y; a8[4 * q + 2] = u.z; a8[4 * q + 3] = u.w;
                    }
                    const bool odd = (kb & 1) != 0;
#pragma unroll
                    for (int i = 0; i < 6; ++i) w[i] = odd ? a8[i + 2] : a8[i];
                } else if constexpr (BITS == 6) {
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(prow + 16 * q);
                        w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
                    }
                } else if constexpr (BITS == 4) {
                    const int x = (r >> 2) & 1;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(prow + ((q ^ x) << 4));
                        w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
                    }
                } else {
                    const int x = (r >> 1) & 3;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(prow + ((q ^ x) << 4));
                        w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
                    }
                }
                if constexpr (TS) {
                    uint32_t v[32];  // row r's 64 values of the k-block, two per column
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint4 out[4];
                        if constexpr (MX) dequant_half_mx<T, MODE>(w + hh * BITS, mx[2 * hh], mx[2 * hh + 1], out);
                        else dequant_half<T, BITS>(w + hh * BITS, hh ? s1 : s0, hh ? b1v : b0v, out);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[16 * hh + 4 * j] = out[j].x;
                            v[16 * hh + 4 * j + 1] = out[j].y;
                            v[16 * hh + 4 * j + 2] = out[j].z;
                            v[16 * hh + 4 * j + 3] = out[j].w;
                        }
                    }
                    // SPLIT: the codes and windows have been consumed, so stage
                    // s's packed tile can be refilled; A slot s was last read by
                    // the MMAs of k-block c - S.  Otherwise the refill of stage
                    // s (full_p above) already waited for those MMAs.
                    if constexpr (SPLIT) {
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(p_empty + 8 * s);
                        if (rp.wrapped) ptx::mbar_wait(b_empty + 8 * s, rp.phase ^ 1, p.err);
                    }
                    tc_fence_after();
                    tmem_st32(tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + A_COL0 + 32u * s, v);
                    tmem_st_wait();
                    tc_fence_before();
                } else {
                    uint8_t *arow = gbase + (a0 - base) + s * A_BYTES + r * 128;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        uint4 out[4];
                        dequant_half<T, BITS>(w + hh * BITS, hh ? s1 : s0, hh ? b1v : b0v, out);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int chunk = 4 * hh + j;
                            *reinterpret_cast<uint4 *>(arow + ((chunk ^ (r & 7)) << 4)) = out[j];
                        }
                    }
                    ptx::fence_proxy_async_smem();  // generic writes -> tensor-core reads
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(full_a + 8 * s);
            }
        }
    } else if (warp < kWarpTma) {
        // ------------------------- epilogue -------------------------
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        T *y = static_cast<T *>(p.y);
        int i = 0;
        Work wk(p, num_tiles, KB);
        for (Unit u; wk.get(u); ++i) {
            const int acc = NACC == 2 ? (i & 1) : 0, use = NACC == 2 ? (i >> 1) : i;
            const Tile t = decode_tile<BN, GROUPED>(p, u.tile);
            ptx::mbar_wait(acc_full + 8 * acc, use & 1, p.err);
            tc_fence_after();
            if (!GROUPED && p.stg_rows > 0) {
                // Staged: TMEM -> registers -> this warp's slab ([m][32 n],
                // n contiguous) -> one tensor store per slab; rows past M and
                // columns past N are clipped by the store.  The accumulator is
                // handed back as soon as its last columns are in registers.
                constexpr int CW = BN < 32 ? BN : 32;
                const int nj = (t.rows + CW - 1) / CW, cpp = p.stg_rows / CW;
                const uint32_t stg = out0 + (uint32_t)q * 64u * (uint32_t)p.stg_rows;
                // Stream-K: a unit that ends before the tile's last k-block
                // leaves its fp32 part in this CTA's workspace slot; the unit
                // holding the last k-block (the tile's owner) adds the parts of
                // the lower-numbered CTAs that hold its first k-blocks, in CTA
                // order after its own, so the sum is the same on every run.
                const size_t slot = (size_t)kBM * BN;  // floats per CTA
                const size_t qoff = (size_t)q * 32 * BN + (size_t)lane * CW;
                constexpr bool kSk = BN <= kSkMaxBN && !GROUPED;  // compiled only where used
                if (kSk && p.sk_len > 0 && u.kb1 < KB) {
                    float *dst = p.sk_ws + blockIdx.x * slot + qoff;
#pragma unroll 1
                    for (int jw = 0; jw < nj; ++jw) {
                        uint32_t v[32];
                        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + acc * BN + CW * jw;
                        if constexpr (CW == 32) tmem_ld32(taddr, v);
                        else tmem_ld16(taddr, v);
                        tmem_ld_wait();
                        if (jw == nj - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(acc_empty + 8 * acc);
                        }
                        uint4 *d4 = reinterpret_cast<uint4 *>(dst + (size_t)jw * 32 * CW);
#pragma unroll
                        for (int c4 = 0; c4 < CW / 4; ++c4)
                            d4[c4] = make_uint4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
                    }
                    __threadfence();
                    __syncwarp();
                    if (lane == 0 && !p.sk_no_publish) atomicExch(p.sk_flags + 4 * blockIdx.x + q, 1);
                    continue;
                }
                int src0 = 0, nsrc = 0;
                if (kSk && p.sk_len > 0 && u.kb0 > 0) {
                    src0 = (u.tile * KB) / p.sk_len;
                    nsrc = (int)blockIdx.x - src0;
                    if (lane == 0) {
                        const uint64_t limit = wait_limit_ns(p.err);
                        for (int sI = 0; sI < nsrc; ++sI) {
                            int *f = p.sk_flags + 4 * (src0 + sI) + q;
                            const uint64_t t0 = ptx::globaltimer_ns();
                            for (;;) {
                                int fv;
                                asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(fv) : "l"(f));
                                if (fv != 0) break;
                                if (ptx::globaltimer_ns() - t0 > limit) {
                                    record_device_error(p.err, QMM_ERR_TIMEOUT);
                                    break;
                                }
                                __nanosleep(64);
                            }
                        }
                    }
                    __syncwarp();
                }
                const float lb = layer_bias<T>(p.bias, p.bias_value, min(t.n0 + 32 * q + lane, p.N - 1));
                int j = 0;
                for (int m_off = 0; m_off < t.rows; m_off += p.stg_rows) {
                    if (lane == 0) bulk_wait_read0();  // the slab's last store has read it
                    __syncwarp();
#pragma unroll 1
                    for (int jj = 0; jj < cpp && j < nj; ++jj, ++j) {
                        uint32_t v[32];
                        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + acc * BN + CW * j;
                        if constexpr (CW == 32) tmem_ld32(taddr, v);
                        else tmem_ld16(taddr, v);
                        tmem_ld_wait();
                        if (j == nj - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(acc_empty + 8 * acc);
                        }
#pragma unroll 1
                        for (int sI = 0; sI < nsrc; ++sI) {
                            const float4 *src = reinterpret_cast<const float4 *>(
                                p.sk_ws + (size_t)(src0 + sI) * slot + qoff + (size_t)j * 32 * CW);
#pragma unroll
                            for (int c4 = 0; c4 < CW / 4; ++c4) {
                                const float4 f = __ldcg(src + c4);
                                v[4 * c4] = __float_as_uint(__uint_as_float(v[4 * c4]) + f.x);
                                v[4 * c4 + 1] = __float_as_uint(__uint_as_float(v[4 * c4 + 1]) + f.y);
                                v[4 * c4 + 2] = __float_as_uint(__uint_as_float(v[4 * c4 + 2]) + f.z);
                                v[4 * c4 + 3] = __float_as_uint(__uint_as_float(v[4 * c4 + 3]) + f.w);
                            }
                        }
                        const uint32_t row0 = stg + (uint32_t)(jj * CW) * 64u + 2u * lane;
#pragma unroll
                        for (int cc = 0; cc < CW; ++cc) sts16(row0 + 64u * cc, out_bits<T>(__uint_as_float(v[cc]) + lb));
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmap_y, stg, t.n0 + 32 * q, t.m0 + m_off);
                        bulk_commit();
                    }
                }
                // The parts are consumed: clear their flags for the next call.
                if (lane == 0)
                    for (int sI = 0; sI < nsrc; ++sI) atomicExch(p.sk_flags + 4 * (src0 + sI) + q, 0);
                continue;
            }
            const int n = t.n0 + 32 * q + lane;
            const float lb = GROUPED ? 0.f : layer_bias<T>(p.bias, p.bias_value, min(n, p.N - 1));
            // Columns acc*BN .. acc*BN+BN-1 of this warp's 32 lanes, 32 (or, for
            // BN = 16, 16) columns per load so no load leaves the allocation;
            // column chunks past the tile's rows are skipped.
            constexpr int CW = BN < 32 ? BN : 32;
            const int nj = (t.rows + CW - 1) / CW;
#pragma unroll 1
            for (int j = 0; j < nj; ++j) {
                uint32_t v[32];
                const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + acc * BN + CW * j;
                if constexpr (CW == 32) tmem_ld32(taddr, v);
                else tmem_ld16(taddr, v);
                tmem_ld_wait();
                // Output row of column CW*j + cc: lane cc holds it, shuffled out.
                int my_dst = 0;
                if constexpr (GROUPED) {
                    const int mm = CW * j + (lane & (CW - 1));
                    if (mm < t.rows) my_dst = __ldg(p.dst_rows + t.m0 + mm);
                }
#pragma unroll
                for (int cc = 0; cc < CW; ++cc) {
                    const int mm = CW * j + cc;
                    int64_t dst;
                    if constexpr (GROUPED) dst = __shfl_sync(0xffffffffu, my_dst, cc);
                    else dst = t.m0 + mm;
                    if (n < p.N && mm < t.rows)
                        y[dst * p.N + n] = Dt<T>::from_f(__uint_as_float(v[cc]) + lb);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(acc_empty + 8 * acc);
        }
        if (lane == 0) bulk_wait0();
    } else if (warp == kWarpTma || warp == kWarpTmaB || warp == kWarpTmaS) {
        // ------------------------- producers -------------------------
        // Issuing a TMA load takes one thread several hundred cycles, so the
        // stage's loads come from three warps in parallel: the packed tile
        // (warp 12), the activation boxes (warp 14), the scale and bias
        // windows (warp 15).  Each arrives with its own byte count on full_p
        // (SPLIT: the activation tile on full_b).
        const int role = warp == kWarpTma ? 0 : (warp == kWarpTmaB ? 1 : 2);
        if (lane == 0 && (role < 2 || (KMAJOR && p.sb_tma))) {
            const int gs_log = __ffs(p.group_size) - 1;
            int c = 0;
            RingPos rp;
            const CUtensorMap *xmap = &tmap_x;
            if constexpr (GROUPED) {
                if (__ldg(&p.hdr->use_x) == 0) xmap = &tmap_xs;
            }
            Work wk(p, num_tiles, KB);
            for (Unit u; wk.get(u);) {
                const Tile t = decode_tile<BN, GROUPED>(p, u.tile);
                // Grouped tiles load only the 64-row boxes that hold their rows.
                const int nbox = GROUPED ? (t.rows + 63) / 64 : 1;
                const uint32_t bbytes = GROUPED ? (uint32_t)nbox * 64u * kBK * 2u : (uint32_t)B_BYTES;
                for (int kb = u.kb0; kb < u.kb1; ++kb, ++c, rp.next(S)) {
                    const int s = rp.slot;
                    // SPLIT: the packed tile and windows are free once the
                    // dequantize group has read them, the activation tile once
                    // the MMAs ran; otherwise the whole stage once the MMAs ran.
                    const bool own = SPLIT && role != 1;
                    if (rp.wrapped) ptx::mbar_wait((own ? p_empty : b_empty) + 8 * s, rp.phase ^ 1, p.err);
                    const uint32_t fb = ((SPLIT && role == 1) ? full_b : full_p) + 8 * s;
                    if (role == 0) {
                        ptx::mbar_arrive_expect_tx(fb, P_BYTES);
                        if constexpr (KMAJOR)
                            tma_load_2d(p0 + s * P_BYTES, &tmap_w, BITS == 3 ? (kb * W_WORDS) & ~3 : kb * W_WORDS,
                                        t.wrow0, fb);
                        else  // 64 k-rows x 128 features of the [K, N] packed weight
                            tma_load_2d(p0 + s * P_BYTES, &tmap_w, t.n0 * BITS / 32, kb * kBK, fb);
                    } else if (role == 1) {
                        ptx::mbar_arrive_expect_tx(fb, bbytes);
                        for (int j = 0; j < nbox; ++j)
                            tma_load_2d(b0 + s * B_BYTES + j * 64 * kBK * 2, xmap, kb * kBK, t.m0 + 64 * j, fb);
                    } else if constexpr (MX) {
                        // the 16 scale bytes (8 two-byte units of the map) holding
                        // this k-block's groups; no biases
                        ptx::mbar_arrive_expect_tx(fb, SB_BYTES / 2);
                        const int wx = (((kb * kBK) >> gs_log) >> 4) << 3;
                        tma_load_2d(sb0 + s * SB_BYTES, &tmap_s, wx, t.wrow0, fb);
                    } else {
                        // the window of 8 groups holding this k-block's groups
                        ptx::mbar_arrive_expect_tx(fb, SB_BYTES);
                        const int wx = ((kb * kBK) >> gs_log) & ~7;
                        tma_load_2d(sb0 + s * SB_BYTES, &tmap_s, wx, t.wrow0, fb);
                        tma_load_2d(sb0 + s * SB_BYTES + SB_BYTES / 2, &tmap_b, wx, t.wrow0, fb);
                    }
                }
            }
            // Drain: wait (bounded by the fixed limit) for the last copies to
            // land before exit.
            for (int d = max(0, c - S); d < c; ++d)
                ptx::mbar_drain(((SPLIT && role == 1) ? full_b : full_p) + 8 * (d % S), (d / S) & 1, p.err);
        }
    } else if (warp == kWarpMma) {
        // ------------------------- MMA issuer -------------------------
        // The warp walks the loop converged; one elected lane waits for the
        // stage's A tile (and, SPLIT, its activation tile: otherwise a complete
        // full_a implies a complete full_p), issues the four MMAs and commits
        // them to b_empty, which frees the activation tile and the A slot.
        const bool leader = elect_one();
        int c = 0, i = 0;
        RingPos rp;
        Work wk(p, num_tiles, KB);
        for (Unit u; wk.get(u); ++i) {
            const int acc = NACC == 2 ? (i & 1) : 0, use = NACC == 2 ? (i >> 1) : i;
            uint32_t idesc = IDESC;
            {
                const Tile t = decode_tile<BN, GROUPED>(p, u.tile);
                if (GROUPED || t.rows < BN) idesc = make_idesc(kF16, kBM, (t.rows + 15) & ~15, !KMAJOR);
            }
            if (leader && i >= NACC) ptx::mbar_wait(acc_empty + 8 * acc, (use + 1) & 1, p.err);
            __syncwarp();
            tc_fence_after();
            const uint32_t d = tmem_base + acc * BN;
            for (int kb = u.kb0; kb < u.kb1; ++kb, ++c, rp.next(S)) {
                const int s = rp.slot;
                if (leader) {
                    ptx::mbar_wait<false>(full_a + 8 * s, rp.phase, p.err);
                    if constexpr (SPLIT) ptx::mbar_wait<false>(full_b + 8 * s, rp.phase, p.err);
                    tc_fence_after();
                    const uint64_t db = sw128_desc(b0 + s * B_BYTES);
                    if constexpr (TS) {
                        // UMMA K = 16: 8 columns of the A slot, 32 bytes of B rows.
                        const uint32_t ta = tmem_base + A_COL0 + 32u * s;
                        tc_mma_ts(d, ta, db, idesc, kb != u.kb0);
                        tc_mma_ts(d, ta + 8, db + 2, idesc, 1);
                        tc_mma_ts(d, ta + 16, db + 4, idesc, 1);
                        tc_mma_ts(d, ta + 24, db + 6, idesc, 1);
                    } else {
                        // UMMA K = 16: 32 bytes along a K-major 128-byte row, or two
                        // 8-k-row groups (2 * SBO bytes) of the MN-major tile.
                        const uint64_t da = KMAJOR ? sw128_desc(a0 + s * A_BYTES)
                                                   : sw128_mn_desc(a0 + s * A_BYTES, MN_LBO, MN_SBO);
                        constexpr uint64_t DA = KMAJOR ? 2 : (2 * MN_SBO) >> 4;
                        tc_mma(d, da, db, idesc, kb != u.kb0);
                        tc_mma(d, da + DA, db + 2, idesc, 1);
                        tc_mma(d, da + 2 * DA, db + 4, idesc, 1);
                        tc_mma(d, da + 3 * DA, db + 6, idesc, 1);
                    }
                    tc_commit(b_empty + 8 * s);
                }
                __syncwarp();
            }
            if (leader) tc_commit(acc_full + 8 * acc);
            __syncwarp();
        }
        // Every MMA issued must have completed before tensor memory is freed,
        // also when a wait above gave up early.
        if (leader) {
            tc_commit(done);
            ptx::mbar_drain(done, 0, p.err);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
int pick_bn(int64_t M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

// Shared-memory budget of one CTA: S stages of (A + B + P [+ scale/bias
// windows]) plus barriers.
template <int BITS, int BN, bool KMAJOR = true>
bool gemm_smem_plan(bool sb_tma, int &stages, size_t &smem, bool a_smem, size_t extra = 0) {
    constexpr int A_BYTES = kBM * kBK * 2, B_BYTES = BN * kBK * 2;
    constexpr int P_BYTES = packed_stage_bytes(BITS, KMAJOR);
    const int STAGE = (a_smem ? A_BYTES : 0) + B_BYTES + P_BYTES + (sb_tma ? 2 * kBM * 16 : 0);
    constexpr size_t kSmemMax = 227 * 1024;
    const size_t fixed = 1024 /*alignment*/ + 64 /*acc bars + slot*/ + extra;
    stages = (int)std::min<size_t>(8, (kSmemMax - fixed) / (STAGE + 40));
    smem = fixed + (size_t)stages * (STAGE + 40);
    return stages >= 2;
}

// Staging the scale/bias windows costs 4 KB per stage; use it only when the
// ring keeps its depth (it was measured faster at equal depth, slower with one
// stage fewer).
template <int BITS, int BN>
bool sb_windows_fit() {
    int s0, s1;
    size_t m0, m1;
    gemm_smem_plan<BITS, BN>(false, s0, m0, true);
    gemm_smem_plan<BITS, BN>(true, s1, m1, true);
    return s1 >= s0;
}

// Scale or bias window map over [rows, gpr] 16-bit values: 8 groups (16
// bytes) x 128 rows per box, unswizzled.  Needs gpr % 8 == 0 (rows of whole
// 16-byte units).
bool make_sb_map(CUtensorMap *map, const void *ptr, uint64_t rows, int64_t gpr) {
    return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, ptr, (uint64_t)gpr, rows, (uint64_t)gpr * 2, 8,
                       kBM, CU_TENSOR_MAP_SWIZZLE_NONE);
}

CUtensorMapDataType act_type(bool f16) {
    return f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// Packed-weight map over `rows` stacked weight rows: one 128-row tile of one
// k-block per box (3-bit codes: 32 of the row's bytes, see packed_pitch),
// swizzled to match its row width (16 / 32 / 64 bytes; 48 unswizzled).
template <int BITS>
bool make_weight_map(CUtensorMap *map, const uint32_t *wq, uint64_t rows, int64_t K) {
    const uint64_t words = (uint64_t)K * BITS / 32;
    const CUtensorMapSwizzle sw = (BITS == 2 || BITS == 6) ? CU_TENSOR_MAP_SWIZZLE_NONE
                                  : BITS == 8              ? CU_TENSOR_MAP_SWIZZLE_64B
                                                           : CU_TENSOR_MAP_SWIZZLE_32B;
    return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, words, rows, words * 4,
                       packed_pitch(BITS) / 4, kBM, sw);
}

// Packed weight stored [K, N]: one 64 k-row x 128-feature tile per box
// (128*BITS/32 words per row, unswizzled).
template <int BITS>
bool make_weight_map_kn(CUtensorMap *map, const uint32_t *wq, int64_t K, int64_t N) {
    const uint64_t words = (uint64_t)N * BITS / 32;
    return make_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, wq, words, (uint64_t)K, words * 4,
                       kBM * BITS / 32, kBK, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Stream-K workspace layout (caller-owned, zeroed before first use): the
// flags first, 4 per SM (a fixed place, so that calls of any shape find them
// zero), then one fp32 partial tile slot per SM of 128 x 64 values (stream-K
// runs only tiles of at most 64 activation rows).
constexpr size_t kSkFlagBytes = kWsFlagBytes;
size_t sk_workspace_bytes() { return kSkFlagBytes + (size_t)num_sms() * kBM * kSkMaxBN * sizeof(float); }

template <typename T, int BITS, int BN, bool KMAJOR, int MODE = QMM_MODE_AFFINE>
cudaError_t run_gemm_layout(const QmmArgs &a, cudaStream_t s) {
    constexpr bool MX = MODE != QMM_MODE_AFFINE;
    constexpr bool a_smem = !KMAJOR;  // [K, N]: MN-major A tile in shared memory
    const int64_t gpr = a.K / a.group_size;
    // [N, K] layout: scale/bias windows come by TMA, and the output is staged
    // for tensor stores when the ring keeps at least 4 stages (whole tile,
    // else half of it per store).  Microscaled weights: windows of 16 scale
    // bytes (rows of whole 16-byte units).
    const bool sb_tma = KMAJOR && (MX ? gpr % 16 == 0 : gpr % 8 == 0);
    if (MX && !sb_tma) return cudaErrorInvalidValue;
    int stages = 0, stg_rows = 0;
    size_t smem = 0;
    // (The [K, N] layout stages only narrow tiles, which stream-K may split;
    // its wide tiles keep direct stores and the deeper ring.)
    const bool y_ok = (KMAJOR || BN <= kSkMaxBN) && (a.N * 2) % 16 == 0 &&
                      (reinterpret_cast<uintptr_t>(a.y) & 15) == 0;
    if (y_ok) {
        for (int rows = BN; rows >= 16 && stg_rows == 0; rows /= 2)
            if (gemm_smem_plan<BITS, BN, KMAJOR>(sb_tma, stages, smem, a_smem, (size_t)kEpiWarps * 64 * rows) &&
                stages >= 4)
                stg_rows = rows;
    }
    if (stg_rows == 0 && !gemm_smem_plan<BITS, BN, KMAJOR>(sb_tma, stages, smem, a_smem))
        return cudaErrorInvalidConfiguration;
    constexpr bool kF16 = std::is_same<T, __half>::value;
    CUtensorMap tx, tw, ts, tb, ty;
    if (!make_map_2d(&tx, act_type(kF16), a.x, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.K * 2, kBK, BN,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (KMAJOR ? !make_weight_map<BITS>(&tw, a.wq, (uint64_t)a.N, a.K)
               : !make_weight_map_kn<BITS>(&tw, a.wq, a.K, a.N))
        return cudaErrorInvalidValue;
    if (MX) {
        // the scale bytes read as two-byte units: [N, gpr / 2], 8 units per box
        if (!make_sb_map(&ts, a.scales, (uint64_t)a.N, gpr / 2)) return cudaErrorInvalidValue;
        tb = ts;  // unused
    } else if (sb_tma) {
        if (!make_sb_map(&ts, a.scales, (uint64_t)a.N, gpr) || !make_sb_map(&tb, a.biases, (uint64_t)a.N, gpr))
            return cudaErrorInvalidValue;
    } else {
        ts = tx;  // unused
        tb = tx;
    }
    if (stg_rows > 0) {
        if (!make_map_2d(&ty, act_type(kF16), a.y, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.N * 2, 32,
                         (uint32_t)stg_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    } else {
        ty = tx;  // unused
    }

    GemmParams p{};
    p.sb_tma = sb_tma ? 1 : 0;
    p.stg_rows = stg_rows;
    p.scales = a.scales;
    p.biases = a.biases;
    p.y = a.y;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.group_size = a.group_size;
    p.m_tiles = (int)((a.M + BN - 1) / BN);
    p.n_tiles = (int)((a.N + kBM - 1) / kBM);
    p.num_tiles = p.m_tiles * p.n_tiles;
    p.stages = stages;
    p.bias = a.bias;
    p.bias_value = a.bias_value;
    p.err = device_error_word();
    int grid = std::min(p.num_tiles, num_sms());
    // Stream-K when there are fewer tiles than SMs and tiles are narrow
    // (decode batches, small weights): every SM takes an equal run of at
    // least 8 k-blocks if that shortens the busiest CTA's run by 10 % or more
    // (M=16, 4096 x 4096: 24.6 -> 13.3 us; M=64: 24.8 -> 19.7 us).  The
    // owner of a split tile reads the other parts' fp32 partials one round
    // trip per 32 columns, which for tiles of 128 or more activation rows
    // costs more than the split gains (M=128, 14336 x 4096: 28.1 -> 36.2 us),
    // and with one or more full waves the last, partial wave runs on lightly
    // loaded SMs (prefill M=2048 with its tail split: unchanged), so both keep
    // whole tiles.
    if (BN <= kSkMaxBN && stg_rows > 0 && p.num_tiles < num_sms() && a.ws != nullptr &&
        a.ws_bytes >= sk_workspace_bytes() && (size_t)num_sms() * 4 * sizeof(int) <= kSkFlagBytes) {
        const int64_t KB = a.K / kBK, sms = num_sms();
        const int64_t total = (int64_t)p.num_tiles * KB;
        const int64_t len = std::max<int64_t>(8, (total + sms - 1) / sms);
        if (total < (1LL << 30) && len * 10 <= KB * 9) {
            p.sk_len = (int)len;
            p.sk_no_publish = injected_fault() == QMM_FAULT_STREAMK_NO_PUBLISH;
            p.sk_flags = static_cast<int *>(a.ws);
            p.sk_ws = reinterpret_cast<float *>(static_cast<char *>(a.ws) + kSkFlagBytes);
            grid = (int)((total + len - 1) / len);
        }
    }
    auto kern = qgemm_tc_kernel<T, BITS, BN, false, KMAJOR, MODE>;
    struct Tag;
    cudaError_t e = configure_once<Tag>(smem, [&]() {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(tx, tx, tw, ts, tb, ty, p);
    count_launches(1);
    return cudaGetLastError();
}

template <typename T, int BITS, int BN>
cudaError_t run_gemm(const QmmArgs &a, cudaStream_t s) {
    return a.transpose ? run_gemm_layout<T, BITS, BN, true>(a, s) : run_gemm_layout<T, BITS, BN, false>(a, s);
}

template <typename T, int BITS, int BN>
cudaError_t run_gemm_grouped(const GroupedArgs &g, cudaStream_t s) {
    const int64_t gpr = g.K / g.group_size;
    const bool sb_tma = gpr % 8 == 0 && sb_windows_fit<BITS, BN>();
    int stages;
    size_t smem;
    if (!gemm_smem_plan<BITS, BN>(sb_tma, stages, smem, true)) return cudaErrorInvalidConfiguration;
    constexpr bool kF16 = std::is_same<T, __half>::value;
    // Activation maps: 64-row boxes over x viewed as [x_batch * M, K] and over
    // the sorted copy [rows, K].
    CUtensorMap tx, txs, tw, ts, tb;
    if (!make_map_2d(&tx, act_type(kF16), g.x, (uint64_t)g.K, (uint64_t)g.x_rows, (uint64_t)g.K * 2,
                     kBK, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&txs, act_type(kF16), g.x_sorted, (uint64_t)g.K, (uint64_t)g.rows,
                     (uint64_t)g.K * 2, kBK, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_weight_map<BITS>(&tw, g.wq, (uint64_t)g.n_experts * (uint64_t)g.N, g.K))
        return cudaErrorInvalidValue;
    const uint64_t wrows = (uint64_t)g.n_experts * (uint64_t)g.N;
    if (sb_tma) {
        if (!make_sb_map(&ts, g.scales, wrows, gpr) || !make_sb_map(&tb, g.biases, wrows, gpr))
            return cudaErrorInvalidValue;
    } else {
        ts = tx;  // unused
        tb = tx;
    }

    GemmParams p{};
    p.scales = g.scales;
    p.biases = g.biases;
    p.y = g.y;
    p.M = (int)g.rows;
    p.N = (int)g.N;
    p.K = (int)g.K;
    p.group_size = g.group_size;
    p.n_tiles = (int)((g.N + kBM - 1) / kBM);
    p.m_tiles = 0;
    p.num_tiles = 0;  // read from the header on the device
    p.stages = stages;
    p.err = device_error_word();
    p.hdr = g.hdr;
    p.chunks = g.chunks;
    p.dst_rows = g.dst_rows;
    p.sb_tma = sb_tma ? 1 : 0;
    auto kern = qgemm_tc_kernel<T, BITS, BN, true>;
    struct Tag;
    cudaError_t e = configure_once<Tag>(smem, [&]() {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = g.max_chunks * (int64_t)p.n_tiles;
    const int grid = (int)std::min<int64_t>(max_tiles, num_sms());
    kern<<<grid, kThreads, smem, s>>>(tx, txs, tw, ts, tb, tx, p);
    count_launches(1);
    return cudaGetLastError();
}

// Microscaled weights, [N, K] layout.
template <typename T, int MODE>
cudaError_t gemm_mx(const QmmArgs &a, cudaStream_t s) {
    constexpr int BITS = MODE == QMM_MODE_MXFP8 ? 8 : 4;
    switch (pick_bn(a.M)) {
    case 16: return run_gemm_layout<T, BITS, 16, true, MODE>(a, s);
    case 32: return run_gemm_layout<T, BITS, 32, true, MODE>(a, s);
    case 64: return run_gemm_layout<T, BITS, 64, true, MODE>(a, s);
    case 128: return run_gemm_layout<T, BITS, 128, true, MODE>(a, s);
    default: return run_gemm_layout<T, BITS, 256, true, MODE>(a, s);
    }
}

template <typename T>
cudaError_t gemm_mx_dtype(const QmmArgs &a, cudaStream_t s) {
    switch (a.mode) {
    case QMM_MODE_MXFP4: return gemm_mx<T, QMM_MODE_MXFP4>(a, s);
    case QMM_MODE_MXFP8: return gemm_mx<T, QMM_MODE_MXFP8>(a, s);
    default: return gemm_mx<T, QMM_MODE_NVFP4>(a, s);
    }
}

template <typename T, int BITS>
cudaError_t gemm_bits(const QmmArgs &a, cudaStream_t s) {
    switch (pick_bn(a.M)) {
    case 16: return run_gemm<T, BITS, 16>(a, s);
    case 32: return run_gemm<T, BITS, 32>(a, s);
    case 64: return run_gemm<T, BITS, 64>(a, s);
    case 128: return run_gemm<T, BITS, 128>(a, s);
    default: return run_gemm<T, BITS, 256>(a, s);
    }
}

template <typename T, int BITS>
cudaError_t grouped_bits(const GroupedArgs &g, cudaStream_t s) {
    switch (g.chunk_rows) {
    case 64: return run_gemm_grouped<T, BITS, 64>(g, s);
    case 128: return run_gemm_grouped<T, BITS, 128>(g, s);
    default: return run_gemm_grouped<T, BITS, 256>(g, s);
    }
}

}  // namespace

// The tensor-core path: bf16/f16, K a multiple of the 64-wide k-block, packed
// rows of whole 16-byte units (K*bits/8 for [N, K] storage, N*bits/8 for
// [K, N] storage), sizes in int range.
bool gemm_supported(qmm_dtype dt, const QmmArgs &a) {
    if (dt != QMM_BF16 && dt != QMM_F16) return false;
    if (a.mode != QMM_MODE_AFFINE) {
        // microscaled weights: [N, K] layout, scale rows of whole 16-byte units
        if (!a.transpose || (a.K / a.group_size) % 16 != 0 || a.K % kBK != 0) return false;
        if (a.M > INT32_MAX / 2 || a.N > INT32_MAX / 2 || a.K > INT32_MAX / 2) return false;
        return encode_fn() != nullptr;
    }
    if (a.bits < 2 || a.bits > 8 || a.bits == 5 || a.bits == 7) return false;
    if (a.K % kBK != 0) return false;
    if (((a.transpose ? a.K : a.N) * a.bits / 8) % 16 != 0) return false;
    if (a.M > INT32_MAX / 2 || a.N > INT32_MAX / 2 || a.K > INT32_MAX / 2) return false;
    return encode_fn() != nullptr;
}

size_t gemm_workspace_size(qmm_dtype dt, int64_t M, int64_t K, int64_t N, bool transpose, int bits) {
    if ((dt != QMM_BF16 && dt != QMM_F16) || M <= 0 || N <= 0 || K % kBK != 0) return 0;
    if (pick_bn(M) > kSkMaxBN) return 0;
    const int64_t tiles = ((M + pick_bn(M) - 1) / pick_bn(M)) * ((N + kBM - 1) / kBM);
    if (tiles >= num_sms()) return 0;
    (void)bits;
    return sk_workspace_bytes();
}

cudaError_t launch_gemm(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    if (a.mode != QMM_MODE_AFFINE)
        return dt == QMM_BF16 ? gemm_mx_dtype<__nv_bfloat16>(a, s) : gemm_mx_dtype<__half>(a, s);
    if (dt == QMM_BF16) {
        switch (a.bits) {
        case 2: return gemm_bits<__nv_bfloat16, 2>(a, s);
        case 3: return gemm_bits<__nv_bfloat16, 3>(a, s);
        case 4: return gemm_bits<__nv_bfloat16, 4>(a, s);
        case 6: return gemm_bits<__nv_bfloat16, 6>(a, s);
        default: return gemm_bits<__nv_bfloat16, 8>(a, s);
        }
    }
    switch (a.bits) {
    case 2: return gemm_bits<__half, 2>(a, s);
    case 3: return gemm_bits<__half, 3>(a, s);
    case 4: return gemm_bits<__half, 4>(a, s);
    case 6: return gemm_bits<__half, 6>(a, s);
    default: return gemm_bits<__half, 8>(a, s);
    }
}

bool gemm_grouped_supported(qmm_dtype dt, const GroupedArgs &g) {
    if (!g.transpose) return false;
    if (g.bits < 2 || g.bits > 8 || g.bits == 5 || g.bits == 7) return false;
    if (dt != QMM_BF16 && dt != QMM_F16) return false;
    if (g.K % kBK != 0) return false;
    if ((g.K * g.bits / 8) % 16 != 0) return false;
    if (g.N > INT32_MAX / 2 || g.K > INT32_MAX / 2) return false;
    if (g.rows > INT32_MAX / 2 || g.x_rows > INT32_MAX / 2) return false;
    if (g.n_experts * g.N > INT32_MAX / 2) return false;  // TMA row coordinates
    return encode_fn() != nullptr;
}

cudaError_t launch_gemm_grouped(qmm_dtype dt, const GroupedArgs &g, cudaStream_t s) {
    if (dt == QMM_BF16) {
        switch (g.bits) {
        case 2: return grouped_bits<__nv_bfloat16, 2>(g, s);
        case 3: return grouped_bits<__nv_bfloat16, 3>(g, s);
        case 4: return grouped_bits<__nv_bfloat16, 4>(g, s);
        case 6: return grouped_bits<__nv_bfloat16, 6>(g, s);
        default: return grouped_bits<__nv_bfloat16, 8>(g, s);
        }
    }
    switch (g.bits) {
    case 2: return grouped_bits<__half, 2>(g, s);
    case 3: return grouped_bits<__half, 3>(g, s);
    case 4: return grouped_bits<__half, 4>(g, s);
    case 6: return grouped_bits<__half, 6>(g, s);
    default: return grouped_bits<__half, 8>(g, s);
    }
}

}  // namespace qmm
