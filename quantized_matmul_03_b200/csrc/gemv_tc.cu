// gemv_tc.cu -- decode-shaped quantized matmul on the integer tensor cores
// for 1..16 activation rows, W stored [N, K] (transpose), 2- and 4-bit codes,
// bf16/f16 activations:
//     y[m, n] = sum_g s[n,g] sum_{k in g} q[n,k] x[m,k] + b[n,g] sum_{k in g} x[m,k]
// (mlx-rs ops/quantization.rs, quantized_matmul; Emily.Quantization.Layers,
// quantized_dense: the packed weight is streamed once per call and never
// expanded into a dense weight in memory).
//
// Formulation.  The codes enter the MMA as exact unsigned bytes and the
// activations as exact block fixed point, so every multiply-add of a group is
// an exact int32 sum on the tensor cores (tcgen05.mma kind::i8):
//   activations: per row m and group g, x ~ x_int 2^-e with e chosen from the
//     group's largest |x| so that x_int is a 16-bit integer (representation
//     error below 2^-15 of that largest |x|; 2^-14 for a value that rounds
//     up to 2^15 and is held at 2^15 - 1), split as x_int = 256 h + l with
//     h in [-128, 127] and l in [0, 255];  X_g[m] = sum of x (fp32);
//   codes: a 4-bit word w gives the bytes (w & 0x0F0F0F0F) = codes 0,2,4,6
//     and ((w >> 4) & 0x0F0F0F0F) = codes 1,3,5,7 (2-bit: four planes, codes
//     p, 4+p, 8+p, 12+p), so the A operand holds each word's codes in that
//     order, and h and l are stored in the same order;
//   per group one unsigned MMA per K = 32 against B rows (h + 128, l, 1):
//     D_h' = sum q (h + 128), D_l = sum q l and D_1 = sum q, so
//     D_h = D_h' - 128 D_1 exactly (all below 2^22 in magnitude for codes of
//     at most 4 bits and groups of at most 128), then
//     y[m, n] += s 2^-e (256 D_h + D_l) + b X_g[m]  in fp32.
// A prep kernel writes h, l, 2^-e and X_g once per call into the workspace;
// the product kernel reads them with tensor copies.
//
// Orientation: UMMA M = 128 over weight rows (each CTA owns R <= 128
// contiguous rows; A rows past R are never read back), UMMA N = 16 over
// activation rows (48 B rows: 16 of h + 128, 16 of l, the row of ones and
// padding), K = 32 per instruction; per group one accumulator of 48 columns,
// a ring of 10.
//
// Roles (640 threads, one CTA per SM with deep rings: every code stage, A
// slot and accumulator in flight hides part of the MMA round trip, which a
// shallow ring exposed once per slot):
//   warps 0, 1   tensor copies of the packed codes, 128 bytes of every owned
//                row per stage (alternate stages), 128-byte swizzled;
//   warp 2       waits for the prep kernel (griddepcontrol.wait), copies the
//                call's whole (2^-e, X) table once (its own area: were it
//                carried with the B tiles, a B stage could be refilled only
//                after the epilogue had finished its groups, which paced the
//                whole pipeline), then per four A slots their B tiles (one
//                3-D tensor copy of 4 x 48 rows x 128 bytes: a tensor copy
//                costs its issuing thread several hundred cycles, whatever
//                its size);
//   warps 3, 20  MMA issuers (one elected lane each) for the even and the
//                odd A slots: a tcgen05 instruction occupies its issuing
//                thread for ~100+ cycles, so one thread issuing 4 MMAs and
//                3 commits per slot set the pace; warp 3 also owns tensor
//                memory;
//   warps 4-11   code expansion: two groups of four warps take alternate A
//                slots (128 codes of every row, 128-byte swizzled K-major u8);
//   warps 12-19  epilogue, two halves of four (one warp per lane quadrant)
//                taking alternate groups, two of them per round (one wait
//                for six tensor-memory loads): the step above in fp32
//                registers, two activation rows per packed f32x2
//                instruction; at the end the halves' sums are added through
//                shared memory and y stored per row.
// Every wait is bounded (device error word on timeout); before exiting or
// freeing tensor memory a CTA waits, with the fixed limit, for its own copies
// and MMAs.  No cluster multicast is used.
#include <algorithm>
#include <type_traits>

#include "ptx_sm100.cuh"
#include "qmm_internal.cuh"
#include "tcgen05.cuh"

namespace qmm {
namespace {

constexpr int kThreads = 672;
constexpr int kWarpB = 2, kWarpMma = 3, kWarpUnp = 4, kWarpEpi = 12;
constexpr int kEpiWarps = 8;
constexpr int kWarpMma2 = kWarpEpi + kEpiWarps;  // 20: the second MMA issuer
constexpr int kASlots = 6;          // A slots: 128 codes x R rows, u8
constexpr int kSlotsPerB = 4;       // A slots per activation stage
constexpr int kBStages = 2;         // activation ring
constexpr int kBRows = 48;          // h + 128 (16), l (16), ones (1), padding
constexpr int kBTile = kBRows * 128;  // B tile of one A slot
constexpr int kBStage = kSlotsPerB * kBTile;
constexpr int kMaxGroups = 128;     // groups per row whose table fits (16 KB)
constexpr int kDCols = kBRows;      // accumulator columns per group
constexpr int kDSlots = 10;         // group accumulators (10 x 48 of 512 columns)
constexpr int kDPerIssuer = kDSlots / 2;  // each MMA issuer has its own five

// Accumulator slot and use of group g: the issuer of its A slot (128 codes,
// gpa groups) takes the slots par*5 .. par*5+4 in turn, so each slot's uses
// come from one thread in order (two issuers sharing slots could get two
// phases ahead of a slot's barrier, where a parity wait cannot tell them
// apart).
__device__ __forceinline__ void group_slot(int g, int gpa, int &d, int &use) {
    const int a = g / gpa, par = a & 1;
    const int k = (a >> 1) * gpa + (g - a * gpa);  // ordinal among the issuer's groups
    d = par * kDPerIssuer + k % kDPerIssuer;
    use = k / kDPerIssuer;
}
constexpr uint32_t kTmemCols = 512;
constexpr int kTmemThreads = 32 * (kThreads / 32 - kWarpMma);  // warps that use tensor memory
constexpr int kMaxRows = 128;
constexpr size_t kSmemBudget = 220 * 1024;

// Instruction descriptor of kind::i8: s32 accumulator, A and B u8, both
// K-major, M = 128, N = kBRows.
constexpr uint32_t idesc_u8() {
    return (2u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(kBRows >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void tc_mma_i8(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(desc_a), "l"(desc_b), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Byte order of the A operand (and of h and l) within a packed word: output
// position j of a 16-element chunk holds element perm(j) of the chunk.
template <int BITS> __host__ __device__ constexpr int perm_elem(int j) {
    if constexpr (BITS == 4) {
        // two words of 8 codes: 0,2,4,6,1,3,5,7 each
        const int w = j >> 3, t = j & 7;
        return 8 * w + (t < 4 ? 2 * t : 2 * (t - 4) + 1);
    } else {
        // one word of 16 codes: plane p = j / 4 holds codes p, 4+p, 8+p, 12+p
        return 4 * (j & 3) + (j >> 2);
    }
}

struct I8Params {
    const uint16_t *scales, *biases;
    void *y;
    const void *bias;  // layer bias [N] or null, plus bias_value, added before rounding
    float bias_value;
    int M, N, K, gpr, gs_log;
    int R;             // rows per CTA (at most)
    int S;             // code-ring stages
    int stage_bytes;   // per code stage (1024-aligned)
    int a_bytes;       // per A slot: whole 8-row atoms of R rows
    int *err;
};

// ---------------------------------------------------------------------------
// Prep: activations -> h + 128, l (permuted byte order), (2^-e, X) per
// (group, row).  Workspace: [48][K] bytes (rows 0..15 h + 128, 16..31 l, 32
// ones; rows past M and rows 33..47 unused) then [K / group_size][16] float2.  One thread per (row, 16-element chunk); the
// gs/16 threads of a group are adjacent lanes.
// ---------------------------------------------------------------------------
template <typename T, int BITS>
__global__ void __launch_bounds__(256)
qdecode_prep_kernel(const T *__restrict__ x, int M, int K, int gs_log, uint8_t *__restrict__ ws) {
    // The next grid (the product) may start its weight stream now.
    ptx::grid_launch_dependents();
    // x may be the output of the preceding kernel, and the workspace may
    // still be read by the product kernel of the previous call: wait for
    // both (every earlier grid) to complete.
    ptx::grid_dependency_wait();
    const int cpr = K >> 4;  // chunks per row
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    const bool ok = idx < M * cpr;
    const int m = ok ? idx / cpr : 0, c = ok ? idx - m * cpr : 0;
    float v[16];
    if (ok) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (int64_t)m * K + 16 * c);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 u = __ldcg(src + h);
            const T *t = reinterpret_cast<const T *>(&u);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[8 * h + i] = Dt<T>::to_f(t[i]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
    }
    float amax = 0.f, sum = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        amax = fmaxf(amax, fabsf(v[i]));
        sum += v[i];
    }
    // Group of gs/16 adjacent lanes (2, 4 or 8): out-of-range threads form
    // whole groups (M * cpr is a multiple of gs/16).
    const int tpg = 1 << (gs_log - 4);
    for (int o = 1; o < tpg; o <<= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    if (!ok) return;
    // amax < 2^ex; e = 15 - ex puts every |x 2^e| below 2^15, clamped so that
    // 2^e and 2^-e are normal floats.
    const int ex = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126;
    const int e = min(126, max(-126, 15 - ex));
    const float up = __uint_as_float((uint32_t)(127 + e) << 23);
    uint32_t hw[4] = {0, 0, 0, 0}, lw[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int xi = min(32767, __float2int_rn(v[perm_elem<BITS>(j)] * up));
        const uint32_t hb = (uint32_t)((xi >> 8) + 128) & 0xffu, lb = (uint32_t)xi & 0xffu;
        hw[j >> 2] |= hb << (8 * (j & 3));
        lw[j >> 2] |= lb << (8 * (j & 3));
    }
    uint8_t *row_h = ws + (int64_t)m * K + 16 * c;
    *reinterpret_cast<uint4 *>(row_h) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(row_h + (int64_t)16 * K) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    if (m == 0) *reinterpret_cast<uint4 *>(ws + (int64_t)32 * K + 16 * c) = make_uint4(0x01010101u, 0x01010101u,
                                                                                        0x01010101u, 0x01010101u);
    if ((c & (tpg - 1)) == 0) {
        float2 *tab = reinterpret_cast<float2 *>(ws + (int64_t)48 * K);
        tab[(int64_t)(c >> (gs_log - 4)) * 16 + m] = make_float2(__uint_as_float((uint32_t)(127 - e) << 23), sum);
    }
}

// Codes of one row for one A slot (128 codes) -> 8 chunks of 16 u8 bytes in
// the permuted order; w holds BITS * 4 words.
template <int BITS>
__device__ __forceinline__ void expand_codes(const uint32_t (&w)[BITS * 4], uint32_t (&o)[32]) {
    if constexpr (BITS == 4) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            o[2 * i] = w[i] & 0x0F0F0F0Fu;
            o[2 * i + 1] = (w[i] >> 4) & 0x0F0F0F0Fu;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int p = 0; p < 4; ++p) o[4 * i + p] = (w[i] >> (2 * p)) & 0x03030303u;
        }
    }
}

template <int N> __device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]);
template <> __device__ __forceinline__ void tmem_ld_cols<1>(uint32_t taddr, uint32_t (&v)[1]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v[0]) : "r"(taddr) : "memory");
}
template <> __device__ __forceinline__ void tmem_ld_cols<2>(uint32_t taddr, uint32_t (&v)[2]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                 : "=r"(v[0]), "=r"(v[1])
                 : "r"(taddr)
                 : "memory");
}
template <> __device__ __forceinline__ void tmem_ld_cols<4>(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(taddr)
                 : "memory");
}
template <> __device__ __forceinline__ void tmem_ld_cols<8>(uint32_t taddr, uint32_t (&v)[8]) {
    tmem_ld8(taddr, v);
}
template <> __device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// MR: activation rows the kernel is built for (1, 2, 4, 8, 16; the call has
// M <= MR).  The MMAs always use N = 16 (h and l tiles of 16 rows each).
template <typename T, int BITS, int MR>
__global__ void __launch_bounds__(kThreads, 1)
qgemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_b,
                const float2 *__restrict__ tab, const I8Params p) {
    constexpr bool kF16 = std::is_same<T, __half>::value;
    constexpr int SPC = 512 / (BITS * 64);         // A slots per 128-byte code chunk (4-bit 2, 2-bit 4)
    constexpr uint32_t IDESC = idesc_u8();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const int S = p.S;
    const uint32_t c0 = base;                                          // code ring
    const uint32_t a0 = c0 + (uint32_t)S * (uint32_t)p.stage_bytes;    // A ring
    // (the MMA reads 128 rows of an A slot; rows past R of the last slot fall
    // into the B ring that follows, inside the allocation)
    const uint32_t b0 = a0 + (uint32_t)kASlots * (uint32_t)p.a_bytes;  // B ring
    const uint32_t red0 = b0 + kBStages * kBStage;  // epilogue halves: MR x 128 floats
    const uint32_t tab0 = red0 + (uint32_t)MR * 128u * 4u;  // (2^-e, X) per (group, row)
    const uint32_t bar0 = tab0 + (uint32_t)kMaxGroups * 128u;
    const uint32_t fullC = bar0, emptyC = fullC + 8 * S;
    const uint32_t fullA = emptyC + 8 * S, emptyA = fullA + 8 * kASlots;
    const uint32_t fullB = emptyA + 8 * kASlots, emptyB = fullB + 8 * kBStages;
    const uint32_t fullD = emptyB + 8 * kBStages, emptyD = fullD + 8 * kDSlots;
    const uint32_t done = emptyD + 8 * kDSlots, fullT = done + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + (fullT + 8 - base));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * p.R;
    const int R = max(0, min(p.R, p.N - r0));
    const int NA = p.K >> 7;                       // A slots (128 codes each)
    const int NST = NA / SPC;                      // code stages
    const int G = p.K >> p.gs_log;                 // groups per row
    const int gpa = 128 >> p.gs_log;               // groups per A slot
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(fullC + 8 * s, 1);
            ptx::mbar_init(emptyC + 8 * s, 8);     // every expansion warp, once per stage
        }
        for (int a = 0; a < kASlots; ++a) {
            ptx::mbar_init(fullA + 8 * a, 4);      // the four warps of one expansion group
            ptx::mbar_init(emptyA + 8 * a, 1);
        }
        for (int b = 0; b < kBStages; ++b) {
            ptx::mbar_init(fullB + 8 * b, 1);
            ptx::mbar_init(emptyB + 8 * b, 2);     // one commit from each MMA issuer
        }
        for (int d = 0; d < kDSlots; ++d) {
            ptx::mbar_init(fullD + 8 * d, 1);
            ptx::mbar_init(emptyD + 8 * d, 4);     // the four epilogue warps of the group's half
        }
        ptx::mbar_init(done, 2);               // both MMA issuers
        ptx::mbar_init(fullT, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();  // barriers initialised
    // Let the next kernel of the stream launch (the next call's prep kernel,
    // which waits for this grid before it writes the workspace).  Before
    // griddepcontrol.wait this grid reads only the packed weight, its scales
    // and biases (the rule for their writers is in qmm.h).
    ptx::grid_launch_dependents();
    // The producers start at once; the warps that use tensor memory wait for
    // the allocation (which waits for the CTA of the previous call on this SM
    // to free its columns) and learn its address through a named barrier.
    uint32_t tmem = 0;
    if (warp >= kWarpMma) {
        if (warp == kWarpMma) {
            tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
        asm volatile("bar.sync 1, %0;" ::"r"(kTmemThreads) : "memory");
        tc_fence_after();
        tmem = *tmem_slot;
    }

    if (warp < kWarpB) {
        // ---------------- packed-code producers ----------------
        if (lane == 0) {
            for (int st = warp; st < NST; st += 2) {
                const int slot = st % S;
                if (st >= S) ptx::mbar_wait(emptyC + 8 * slot, ((st / S) - 1) & 1, p.err);
                ptx::mbar_arrive_expect_tx(fullC + 8 * slot, (uint32_t)p.R * 128u);
                tma_load_2d(c0 + (uint32_t)slot * (uint32_t)p.stage_bytes, &tmap_w, st * 32, r0, fullC + 8 * slot);
            }
            // The CTA must not exit while a copy into its ring can still land.
            for (int st = max(0, NST - S); st < NST; ++st)
                if ((st & 1) == warp) ptx::mbar_drain(fullC + 8 * (st % S), (st / S) & 1, p.err);
        }
    } else if (warp == kWarpB) {
        // ---------------- h/l tiles and tables ----------------
        if (lane == 0) {
            // The workspace is written by this call's prep kernel: wait for it.
            ptx::grid_dependency_wait();
            ptx::mbar_arrive_expect_tx(fullT, (uint32_t)G * 128u);
            ptx::bulk_g2s(tab0, tab, (uint32_t)G * 128u, fullT);
            const int NB = NA / kSlotsPerB;
            for (int bt = 0; bt < NB; ++bt) {
                const int bs = bt % kBStages;
                if (bt >= kBStages) ptx::mbar_wait(emptyB + 8 * bs, ((bt / kBStages) - 1) & 1, p.err);
                const uint32_t dst = b0 + (uint32_t)bs * kBStage;
                ptx::mbar_arrive_expect_tx(fullB + 8 * bs, (uint32_t)(kSlotsPerB * kBTile));
                tma_load_3d(dst, &tmap_b, 0, 0, bt * kSlotsPerB, fullB + 8 * bs);
            }
            for (int bt = max(0, NB - kBStages); bt < NB; ++bt)
                ptx::mbar_drain(fullB + 8 * (bt % kBStages), (bt / kBStages) & 1, p.err);
            ptx::mbar_drain(fullT, 0, p.err);
        }
    } else if (warp == kWarpMma || warp == kWarpMma2) {
        // ---------------- MMA issuers ----------------
        // Issuer par takes the A slots a = par mod 2.  A group lies inside one
        // slot, so each accumulator is written by one issuer per use; an A
        // slot index recurs kASlots (even) slots later, with the same issuer;
        // each activation stage is released by one commit from each.
        const int par = warp == kWarpMma2 ? 1 : 0;
        const bool leader = elect_one();
        const int gs_mask = (1 << p.gs_log) - 1;
        for (int a = par; a < NA; a += 2) {
            const int as = a % kASlots, bt = a / kSlotsPerB, bs = bt % kBStages, sub = a - bt * kSlotsPerB;
            if (leader) {
                ptx::mbar_wait<false>(fullA + 8 * as, (a / kASlots) & 1, p.err);
                if (sub == par) ptx::mbar_wait<false>(fullB + 8 * bs, (bt / kBStages) & 1, p.err);
                tc_fence_after();
                const uint32_t btile = b0 + (uint32_t)bs * kBStage + (uint32_t)sub * kBTile;
                const uint64_t da = sw128_desc(a0 + (uint32_t)as * (uint32_t)p.a_bytes);
                const uint64_t db = sw128_desc(btile);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int e0 = a * 128 + 32 * j;
                    const int g = e0 >> p.gs_log;
                    int d, use;
                    group_slot(g, gpa, d, use);
                    const bool first = (e0 & gs_mask) == 0, last = ((e0 + 32) & gs_mask) == 0;
                    if (first && use > 0) {
                        ptx::mbar_wait<false>(emptyD + 8 * d, (use - 1) & 1, p.err);
                        tc_fence_after();
                    }
                    // K = 32 bytes per instruction: 2 units of 16 bytes along the rows.
                    tc_mma_i8(tmem + (uint32_t)(kDCols * d), da + 2u * j, db + 2u * j, IDESC, first ? 0u : 1u);
                    if (last) tc_commit(fullD + 8 * d);
                }
                tc_commit(emptyA + 8 * as);
                if (sub >= kSlotsPerB - 2) tc_commit(emptyB + 8 * bs);
            }
            __syncwarp();
        }
        // Every MMA must have completed before tensor memory is freed, also
        // when a wait above gave up early.
        if (leader) {
            tc_commit(done);
            ptx::mbar_drain(done, 0, p.err);
        }
        __syncwarp();
    } else if (warp < kWarpEpi) {
        // ---------------- code expansion ----------------
        const int h = (warp - kWarpUnp) >> 2, q = warp & 3;
        const int j = 32 * q + lane;                  // row of this lane within the CTA
        const bool valid = j < R;
        const uint32_t arow = (uint32_t)(j >> 3) * 1024u + (uint32_t)(j & 7) * 128u;
        for (int a = h; a < NA; a += 2) {
            const int st = a / SPC, sp = a - st * SPC;
            const int slot = st % S;
            if (sp < 2) ptx::mbar_wait(fullC + 8 * slot, (st / S) & 1, p.err);
            const int as = a % kASlots;
            if (a >= kASlots) ptx::mbar_wait<false>(emptyA + 8 * as, ((a / kASlots) - 1) & 1, p.err);
            uint32_t w[BITS * 4];
            if (valid) {
                const uint8_t *row = gbase + (c0 - base) + slot * p.stage_bytes + j * 128;
#pragma unroll
                for (int c = 0; c < BITS; ++c) {     // BITS chunks of 16 bytes = 128 codes
                    const int chunk = (sp * BITS + c) ^ (j & 7);
                    const uint4 u = *reinterpret_cast<const uint4 *>(row + (chunk << 4));
                    w[4 * c] = u.x;
                    w[4 * c + 1] = u.y;
                    w[4 * c + 2] = u.z;
                    w[4 * c + 3] = u.w;
                }
            }
            __syncwarp();
            // This group's reads of the stage are done after its last slot there.
            if (lane == 0 && sp >= SPC - 2) ptx::mbar_arrive(emptyC + 8 * slot);
            if (valid) {
                uint32_t o[32];
                expand_codes<BITS>(w, o);
                uint8_t *dst = gbase + (a0 - base) + as * p.a_bytes + arow;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(dst + ((c ^ (j & 7)) << 4)) =
                        make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
            }
            ptx::fence_proxy_async_smem();  // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(fullA + 8 * as);
        }
    } else {
        // ---------------- epilogue ----------------
        // Half h of the eight warps takes the groups g = h mod 2; warp (q, h)
        // reads tensor-memory lane quadrant q (rows 32q..32q+31).
        using namespace ptx;
        constexpr int P = (MR + 1) / 2;             // pairs of activation rows
        const int q = warp & 3, half = (warp - kWarpEpi) >> 2;
        const int j = 32 * q + lane;
        const int64_t rowg = (int64_t)r0 + j;
        const bool valid = j < R;
        const uint16_t *srow = p.scales + (valid ? rowg : 0) * p.gpr;
        const uint16_t *brow = p.biases + (valid ? rowg : 0) * p.gpr;
        const unsigned long long mm = f2pack(12582912.0f, 12582912.0f), k256 = f2pack(256.f, 256.f);
        unsigned long long acc[P];
#pragma unroll
        for (int i = 0; i < P; ++i) acc[i] = 0ull;  // (+0.0, +0.0)
        // Scales and biases of the row in 16-byte windows of 8 groups, the
        // next window loaded while the current one is used (with most of
        // the SM's on-chip memory given to shared memory, a 2-byte load per
        // group would wait on L2 every time).
        uint4 s_cur = make_uint4(0, 0, 0, 0), b_cur = s_cur, s_nxt = s_cur, b_nxt = s_cur;
        if (valid) {
            s_cur = __ldg(reinterpret_cast<const uint4 *>(srow));
            b_cur = __ldg(reinterpret_cast<const uint4 *>(brow));
            if (G > 8) {
                s_nxt = __ldg(reinterpret_cast<const uint4 *>(srow + 8));
                b_nxt = __ldg(reinterpret_cast<const uint4 *>(brow + 8));
            }
        }
        int wbase = 0;
        ptx::mbar_wait(fullT, 0, p.err);  // the call's (2^-e, X) table
        for (int g = half; g < G; g += 2) {
            int d, use;
            group_slot(g, gpa, d, use);
            if (g >= wbase + 8) {
                s_cur = s_nxt;
                b_cur = b_nxt;
                wbase += 8;
                if (valid && wbase + 8 < G) {
                    s_nxt = __ldg(reinterpret_cast<const uint4 *>(srow + wbase + 8));
                    b_nxt = __ldg(reinterpret_cast<const uint4 *>(brow + wbase + 8));
                }
            }
            const int o = g - wbase;
            const uint32_t sw = pick_word(s_cur, o >> 1), bw = pick_word(b_cur, o >> 1);
            const uint16_t s16 = (uint16_t)((o & 1) ? (sw >> 16) : (sw & 0xffffu));
            const uint16_t b16 = (uint16_t)((o & 1) ? (bw >> 16) : (bw & 0xffffu));
            const float sv = kF16 ? __half2float(__ushort_as_half(s16)) : __uint_as_float((uint32_t)s16 << 16);
            const float bv = kF16 ? __half2float(__ushort_as_half(b16)) : __uint_as_float((uint32_t)b16 << 16);
            ptx::mbar_wait<false>(fullD + 8 * d, use & 1, p.err);
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kDCols * d);
            uint32_t vh[MR], vl[MR], v1[1];
            tmem_ld_cols<MR>(taddr, vh);
            tmem_ld_cols<MR>(taddr + 16u, vl);
            tmem_ld_cols<1>(taddr + 32u, v1);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(emptyD + 8 * d);
            const float *tb = reinterpret_cast<const float *>(gbase + (tab0 - base)) + g * 32;
            const unsigned long long s2 = f2pack(sv, sv), b2 = f2pack(bv, bv);
            // D_h = D_h' - 128 D_1, moved into the mantissa of 1.5 * 2^23
            const uint32_t ch = 0x4B400000u - (v1[0] << 7);
#pragma unroll
            for (int i = 0; i < P; ++i) {
                // rows 2i and 2i+1 (MR = 1: lane 1 repeats row 0 and is dropped)
                const int m0 = 2 * i, m1 = MR > 1 ? 2 * i + 1 : 0;
                // D_h and D_l are below 2^22 in magnitude: exact as floats by
                // the 1.5 * 2^23 bias; then 256 D_h + D_l, and the group's step
                // s 2^-e (256 D_h + D_l) + b X with (2^-e, X) from the table
                const unsigned long long fh = f2sub(u2pack(vh[m0] + ch, vh[m1] + ch), mm);
                const unsigned long long fl = f2sub(u2pack(vl[m0] + 0x4B400000u, vl[m1] + 0x4B400000u), mm);
                const float4 t = *reinterpret_cast<const float4 *>(tb + 2 * m0);  // p0, X0, p1, X1
                const unsigned long long sp = f2mul(s2, f2pack(t.x, t.z));
                acc[i] = f2fma(sp, f2fma(k256, fh, fl), f2fma(b2, f2pack(t.y, t.w), acc[i]));
            }
        }
        float accf[2 * P];
#pragma unroll
        for (int i = 0; i < P; ++i) f2unpack(acc[i], accf[2 * i], accf[2 * i + 1]);
        // The odd-group half hands its sums to the even-group half.
        float *red = reinterpret_cast<float *>(gbase + (red0 - base));
        if (half == 1) {
#pragma unroll
            for (int m = 0; m < MR; ++m) red[m * 128 + j] = accf[m];
        }
        asm volatile("bar.sync 2, %0;" ::"r"(32 * kEpiWarps) : "memory");
        if (half == 0 && valid) {
            T *y = static_cast<T *>(p.y);
            const float lb = layer_bias<T>(p.bias, p.bias_value, rowg);
#pragma unroll
            for (int m = 0; m < MR; ++m)
                if (m < p.M) y[(int64_t)m * p.N + rowg] = Dt<T>::from_f(accf[m] + red[m * 128 + j] + lb);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

struct TcPlan {
    int grid, R, S, stage_bytes, a_bytes;
    size_t smem;
};

bool plan_tc(const QmmArgs &a, TcPlan &p) {
    const int64_t sms = num_sms();
    int64_t G = std::min<int64_t>(sms, (a.N + 7) / 8);
    int64_t R = std::min<int64_t>((a.N + G - 1) / G, kMaxRows);
    G = (a.N + R - 1) / R;  // every CTA owns at least one row
    p.grid = (int)G;
    p.R = (int)R;
    p.stage_bytes = (int)(((R * 128) + 1023) / 1024 * 1024);
    p.a_bytes = (int)(((R + 7) / 8) * 1024);
    const size_t ring_b = (size_t)kBStages * kBStage;
    const size_t bars = 512;
    const size_t red = (size_t)16 * 128 * 4;  // epilogue halves' sums (at most 16 rows)
    const size_t table = (size_t)kMaxGroups * 128;
    const size_t fixed = 1024 /*alignment*/ + (size_t)kASlots * p.a_bytes + ring_b + red + table + bars;
    if (fixed + 2 * (size_t)p.stage_bytes > kSmemBudget) return false;
    p.S = (int)std::min<size_t>(8, (kSmemBudget - fixed) / p.stage_bytes);
    p.smem = fixed + (size_t)p.S * p.stage_bytes;
    return p.S >= 2;
}

template <typename T, int BITS, int MR>
cudaError_t launch_tc(const QmmArgs &a, cudaStream_t s) {
    auto kern = qgemv_tc_kernel<T, BITS, MR>;
    TcPlan p{};
    if (!plan_tc(a, p)) return cudaErrorInvalidValue;
    struct Tag;
    cudaError_t e = configure_once<Tag>(p.smem, [&]() {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    cudaSharedmemCarveoutMaxShared);
    });
    if (e != cudaSuccess) return e;
    uint8_t *ws = static_cast<uint8_t *>(a.ws) + kWsFlagBytes;
    const int gs_log = __builtin_ctz((unsigned)a.group_size);
    // Packed codes as [N rows, K*BITS/32 words]: a box is 32 words (128 bytes)
    // of R rows, 128-byte swizzled; rows past N read as zero.  B rows, [48, K]
    // bytes, viewed as [K/128 slots][48 rows][128 bytes]: a box is the 48 x 128
    // tiles of kSlotsPerB consecutive slots, 128-byte swizzled, tile after tile.
    CUtensorMap tw, tb;
    const uint64_t words = (uint64_t)a.K * BITS / 32;
    if (!make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.wq, words, (uint64_t)a.N, words * 4, 32,
                     (uint32_t)p.R, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    {
        const uint64_t dims[3] = {128, (uint64_t)kBRows, (uint64_t)a.K / 128};
        const uint64_t strides[2] = {(uint64_t)a.K, 128};
        const uint32_t box[3] = {128, (uint32_t)kBRows, (uint32_t)kSlotsPerB};
        if (!make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, ws, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    {
        const int64_t threads = a.M * (a.K / 16);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((threads + 255) / 256), 1, 1);
        cfg.blockDim = dim3(256, 1, 1);
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, qdecode_prep_kernel<T, BITS>, static_cast<const T *>(a.x), (int)a.M,
                               (int)a.K, gs_log, ws);
        if (e != cudaSuccess) return e;
        count_launches(1);
    }
    I8Params dp{};
    dp.y = a.y;
    dp.scales = static_cast<const uint16_t *>(a.scales);
    dp.biases = static_cast<const uint16_t *>(a.biases);
    dp.M = (int)a.M;
    dp.N = (int)a.N;
    dp.K = (int)a.K;
    dp.gpr = (int)(a.K / a.group_size);
    dp.gs_log = gs_log;
    dp.R = p.R;
    dp.S = p.S;
    dp.stage_bytes = p.stage_bytes;
    dp.a_bytes = p.a_bytes;
    dp.bias = a.bias;
    dp.bias_value = a.bias_value;
    dp.err = device_error_word();
    const float2 *tab = reinterpret_cast<const float2 *>(ws + (size_t)kBRows * a.K);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tw, tb, tab, dp);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

template <typename T, int BITS>
cudaError_t tc_rows(const QmmArgs &a, cudaStream_t s) {
    if (a.M <= 1) return launch_tc<T, BITS, 1>(a, s);
    if (a.M <= 2) return launch_tc<T, BITS, 2>(a, s);
    if (a.M <= 4) return launch_tc<T, BITS, 4>(a, s);
    if (a.M <= 8) return launch_tc<T, BITS, 8>(a, s);
    return launch_tc<T, BITS, 16>(a, s);
}

}  // namespace

// Workspace of the decode tensor-core path: past the leading flag bytes
// (left untouched), the B rows as [48, K] bytes and the (2^-e, X) table,
// K / group_size x 16 float2, at most K / 32 groups.
size_t gemv_tc_workspace_bytes(int64_t K) {
    return kWsFlagBytes + (size_t)kBRows * (size_t)K + (size_t)(K / 32) * 16 * sizeof(float2);
}

// bf16/f16, transpose, 1..16 rows, 2- or 4-bit codes, K a multiple of 512
// (whole code chunks), group size 32/64/128 with groups per row a multiple of
// 8 (16-byte scale/bias windows), 16-byte aligned operands.  (The
// call also needs a workspace of gemv_tc_workspace_bytes(K), checked apart.)
bool gemv_tc_supported(qmm_dtype dt, const QmmArgs &a) {
    if (!a.transpose || a.M < 1 || a.M > 16) return false;
    if (dt != QMM_BF16 && dt != QMM_F16) return false;
    if (a.mode != QMM_MODE_AFFINE) return false;
    if (a.bits != 2 && a.bits != 4) return false;
    if (a.group_size < 32 || a.group_size > 128) return false;
    if (a.K % 512 != 0 || (a.K / a.group_size) % 8 != 0 || a.K / a.group_size > kMaxGroups) return false;
    if (a.N < 1 || a.N > (1 << 30) || a.K > (1 << 20)) return false;
    if ((reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.wq) |
         reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases) |
         reinterpret_cast<uintptr_t>(a.ws)) & 15)
        return false;
    TcPlan p{};
    if (!plan_tc(a, p)) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_gemv_tc(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    if (dt == QMM_BF16) return a.bits == 4 ? tc_rows<__nv_bfloat16, 4>(a, s) : tc_rows<__nv_bfloat16, 2>(a, s);
    return a.bits == 4 ? tc_rows<__half, 4>(a, s) : tc_rows<__half, 2>(a, s);
}

}  // namespace qmm
