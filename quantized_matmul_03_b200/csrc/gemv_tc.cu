// gemv_tc.cu -- decode-shaped quantized matmul on the tensor cores for 1..16
// activation rows, W stored [N, K] (transpose), 2- and 4-bit codes, bf16/f16:
//     y[m, n] = sum_k x[m, k] * (s[n,g] q[n,k] + b[n,g])
// (mlx-rs ops/quantization.rs, quantized_matmul; Emily.Quantization.Layers,
// quantized_dense: the packed weight is streamed once per call, never
// expanded into a dense weight in memory).
//
// The product is bound by reading the packed weight, but the work of turning
// codes into something a multiplier can use is not: done on the CUDA cores
// it sets the pace (and grows with the number of activation rows).  Here the
// CUDA cores only place codes into 16-bit operands and the tensor cores do
// every multiply-add, so one kernel serves 1..16 rows at the same cost, and
// the code placement -- which does not depend on x -- runs while the previous
// kernel of the stream is still finishing (programmatic dependent launch).
//
// Formulation.  A code q enters the MMA as the exact 16-bit value
// a = 1 + q/QS (the code ORed into the mantissa of 1.0 at the highest field
// position a byte move reaches; QS = 16 for 4-bit and 4 for 2-bit codes with
// bf16, 64 and 16 with f16).  Per group g of group_size elements the MMA
// leaves, in fp32 tensor memory,
//     D_g[n, m] = sum_{k in g} a[n,k] x[m,k] = X_g[m] + (1/QS) sum_{k in g} q[n,k] x[m,k]
// with X_g[m] = sum_{k in g} x[m,k], so
//     y[m, n] = sum_g (QS s[n,g]) (D_g[n, m] - X_g[m]) + b[n,g] X_g[m].
// X_g comes from the MMA as well: lane 31 of every 32-lane quadrant of the A
// operand holds code 0 everywhere (a = 1), so D_g[lane 31] = X_g.
//
// Orientation: UMMA M = 128 tensor-memory lanes over weight rows (each CTA
// owns R <= 124 contiguous rows, RQ = ceil(R/4) per lane quadrant), UMMA N =
// 16 over activation rows, K = 16 per instruction, one accumulator of 16
// columns per group (a ring of 8).
//
// Roles (512 threads, two CTAs per SM: the next call's CTA fits beside this
// one and fills its own ring while this one finishes):
//   warps 0, 1   TMA loads of the packed codes, 128 bytes of every owned row
//                per stage (alternate stages), into a ring of shared-memory
//                stages (128-byte swizzle: conflict-free row reads);
//   warp 2       waits for the preceding grids (griddepcontrol.wait), then
//                copies the activation rows into shared memory in the
//                canonical 128-byte-swizzled K-major layout of the B operand;
//   warp 3       tensor-memory owner and MMA issuer (one elected lane);
//   warps 4-11   code placement: two groups of four warps take alternate
//                k-blocks of 64; thread l of quadrant q places row q*RQ + l
//                (32 columns of bf16x2 / f16x2 per k-block) with one
//                tcgen05.st;
//   warps 12-15  epilogue: per group, tcgen05.ld of its quadrant's
//                accumulator, the scale/bias step above in fp32 registers,
//                and at the end one store of y per row.
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

constexpr int kThreads = 512;
constexpr int kWarpX = 2, kWarpMma = 3, kWarpUnp = 4, kWarpEpi = 12;
// Tensor memory: all 512 columns.  A k-block's A operand goes from code
// placement through the MMA and back to an empty slot in a round trip of a
// few thousand cycles, so the ring must hold many k-blocks to keep both
// sides busy.  (The next call's CTA, beside this one, streams codes into its
// shared-memory ring while its tcgen05.alloc waits for these columns.)
constexpr int kASlots = 12;         // A operand slots (32 columns each)
constexpr int kDSlots = 8;          // group accumulators (16 columns each)
constexpr int kPlaceBatch = 3;      // k-blocks a placement warp stores per wait
constexpr int kBStageKb = 8;        // k-blocks per activation stage
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol0 = kASlots * 32;
constexpr int kTmemThreads = 32 * (16 - kWarpMma);  // warps that use tensor memory
constexpr int kMaxRows = 124;       // rows per CTA: 31 per quadrant + lane 31
constexpr size_t kSmemBudget = 110 * 1024;

// Per-SM hand-off between consecutive CTAs of this kernel (see the decode
// kernel in gemv_fast.cu): a CTA issues its first copy once the CTA before it
// on the same SM has at most one stage left to issue, or after a short bound.
// It orders memory traffic only; results do not depend on it.
constexpr int kMaxSm = 1024;
constexpr uint64_t kHandoffWaitNs = 20000;
__device__ unsigned long long g_tc_ticket[kMaxSm];
__device__ unsigned long long g_tc_issued[kMaxSm];

struct DecParams {
    const void *x;
    void *y;
    const uint16_t *scales, *biases;
    int M, N, K, gpr, gs_log;
    int R, RQ;        // rows of this CTA (at most), rows per lane quadrant
    int S;            // code-ring stages
    int stage_bytes;  // per code stage (1024-aligned)
    int KB;           // k-blocks of 64
    const void *bias; // layer bias [N] or null, plus bias_value, added before rounding
    float bias_value;
    int *err;
};

// The code field sits at mantissa bit P of each 16-bit half of 1.0 (the
// highest position a byte move can reach), so a = 1 + q/QS with QS =
// 2^(mantissa bits - P): the offset 1 is at most QS times the code step,
// which keeps the accumulator's rounding small next to the code term.
template <typename T, int BITS> struct Field;
template <> struct Field<__nv_bfloat16, 4> { static constexpr int P = 3; };  // QS = 16
template <> struct Field<__nv_bfloat16, 2> { static constexpr int P = 5; };  // QS = 4
template <> struct Field<__half, 4> { static constexpr int P = 4; };         // QS = 64
template <> struct Field<__half, 2> { static constexpr int P = 6; };         // QS = 16
template <typename T> struct One2;
template <> struct One2<__nv_bfloat16> {
    static constexpr uint32_t V = 0x3F803F80u;  // bf16 1.0 | 1.0 (7 mantissa bits)
    static constexpr int MB = 7;
};
template <> struct One2<__half> {
    static constexpr uint32_t V = 0x3C003C00u;  // f16 1.0 | 1.0 (10 mantissa bits)
    static constexpr int MB = 10;
};
template <typename T, int BITS> struct Magic {
    static constexpr int P = Field<T, BITS>::P;
    static constexpr uint32_t ONE2 = One2<T>::V;
    static constexpr uint32_t MASK = (((1u << BITS) - 1u) << P) * 0x00010001u;
    static constexpr float QS = (float)(1 << (One2<T>::MB - P));
};

// Word w shifted so that the code at bit `from` lands at bit `to`.
template <int FROM, int TO>
__device__ __forceinline__ uint32_t align_field(uint32_t w) {
    if constexpr (TO >= FROM) return w << (TO - FROM);
    else return w >> (FROM - TO);
}

// Codes of one k-block of one row (64 codes) -> 32 columns of 16-bit pairs
// (element 2i in the low half of column i), a = 1 + q/QS, in k order.
// Byte i of a word holds codes 2i, 2i+1 (4-bit) or 4i..4i+3 (2-bit); PRMT
// puts byte i of one shifted copy of the word in the low half and byte i of
// another in the high half, so one AND/OR (LOP3) leaves the two codes of a
// pair at bit P of the two mantissas.
template <typename T, int BITS>
__device__ __forceinline__ void place_codes(const uint32_t (&w)[BITS * 2], uint32_t (&v)[32]) {
    using MG = Magic<T, BITS>;
    constexpr int P = MG::P;
    if constexpr (BITS == 4) {
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
            const uint32_t lo = align_field<0, P>(w[wi]), hi = align_field<4, P>(w[wi]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t t = __byte_perm(lo, hi, (uint32_t)(i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12)));
                v[4 * wi + i] = (t & MG::MASK) | MG::ONE2;
            }
        }
    } else {
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const uint32_t a0 = align_field<0, P>(w[wi]), a1 = align_field<2, P>(w[wi]);
            const uint32_t a2 = align_field<4, P>(w[wi]), a3 = align_field<6, P>(w[wi]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t sel = (uint32_t)(i | (i << 4) | ((4 + i) << 8) | ((4 + i) << 12));
                v[8 * wi + 2 * i] = (__byte_perm(a0, a1, sel) & MG::MASK) | MG::ONE2;
                v[8 * wi + 2 * i + 1] = (__byte_perm(a2, a3, sel) & MG::MASK) | MG::ONE2;
            }
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
// M <= MR).  The B operand holds NB = 8 (MR <= 8) or 16 rows; the MMA is
// always N = 16 (with NB = 8 its rows 8..15 are other shared-memory bytes,
// and their accumulator columns are never read).
template <typename T, int BITS, int MR>
__global__ void __launch_bounds__(kThreads, 2)
qgemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const DecParams p) {
    constexpr bool kF16 = std::is_same<T, __half>::value;
    constexpr int NB = MR <= 8 ? 8 : 16;
    constexpr int B_KB = NB * 128;                 // bytes of one k-block of B
    constexpr int B_STAGE = kBStageKb * B_KB;
    constexpr int KBS = BITS == 4 ? 4 : 8;         // k-blocks per 128-byte code chunk
    constexpr uint32_t IDESC = make_idesc(kF16, 128, 16);
    constexpr float QS = Magic<T, BITS>::QS;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - raw);
    const int S = p.S;
    const uint32_t c0 = base;                                   // code ring
    const uint32_t b0 = c0 + (uint32_t)S * (uint32_t)p.stage_bytes;  // activation ring
    // (NB = 8: the MMA's rows 8..15 of the last k-block read up to 1 KB past
    // the ring; that padding keeps them inside the allocation.)
    const uint32_t bar0 = b0 + 2 * B_STAGE + (NB == 8 ? 1024 : 0);
    const uint32_t fullC = bar0, emptyC = fullC + 8 * S;
    const uint32_t fullA = emptyC + 8 * S, emptyA = fullA + 8 * kASlots;
    const uint32_t fullB = emptyA + 8 * kASlots, emptyB = fullB + 16;
    const uint32_t fullD = emptyB + 16, emptyD = fullD + 8 * kDSlots;
    const uint32_t done = emptyD + 8 * kDSlots, go = done + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + (go + 8 - base));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * p.R;
    const int R = max(0, min(p.R, p.N - r0));
    const int KB = p.KB;
    const int NST = KB / KBS;                      // code stages
    const int G = p.K >> p.gs_log;                 // groups per row
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(fullC + 8 * s, 1);
            ptx::mbar_init(emptyC + 8 * s, 8);     // every placement warp, once per stage
        }
        for (int a = 0; a < kASlots; ++a) {
            ptx::mbar_init(fullA + 8 * a, 4);      // the four warps of one placement group
            ptx::mbar_init(emptyA + 8 * a, 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(fullB + 8 * b, 1);
            ptx::mbar_init(emptyB + 8 * b, 1);
        }
        for (int d = 0; d < kDSlots; ++d) {
            ptx::mbar_init(fullD + 8 * d, 1);
            ptx::mbar_init(emptyD + 8 * d, 4);     // the four epilogue warps
        }
        ptx::mbar_init(done, 1);
        ptx::mbar_init(go, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();  // barriers initialised
    // Let the next call in the stream start its prologue and its own code
    // stream now.  Before griddepcontrol.wait this grid reads only the packed
    // weight, its scales and biases (the rule for their writers is in qmm.h).
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

    if (warp < kWarpX) {
        // ---------------- packed-code producers ----------------
        if (lane == 0) {
            uint32_t smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            const bool handoff = smid < (uint32_t)kMaxSm;
            unsigned long long ticket = 0;
            if (warp == 0) {
                if (handoff) {
                    ticket = atomicAdd(&g_tc_ticket[smid], 1ull);
                    const uint64_t t0 = ptx::globaltimer_ns();
                    for (;;) {
                        unsigned long long dn;
                        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(dn) : "l"(&g_tc_issued[smid]));
                        if (dn >= ticket || ptx::globaltimer_ns() - t0 > kHandoffWaitNs) break;
                        __nanosleep(128);
                    }
                }
                ptx::mbar_arrive(go);
            } else {
                ptx::mbar_wait(go, 0, p.err);
            }
            for (int st = warp; st < NST; st += 2) {
                const int slot = st % S;
                if (st >= S) ptx::mbar_wait(emptyC + 8 * slot, ((st / S) - 1) & 1, p.err);
                ptx::mbar_arrive_expect_tx(fullC + 8 * slot, (uint32_t)p.R * 128u);
                tma_load_2d(c0 + (uint32_t)slot * (uint32_t)p.stage_bytes, &tmap_w, st * 32, r0, fullC + 8 * slot);
                if (warp == 0 && handoff && st >= NST - 2) atomicMax(&g_tc_issued[smid], ticket + 1);
            }
            if (warp == 0 && handoff) atomicMax(&g_tc_issued[smid], ticket + 1);
            // The CTA must not exit while a copy into its ring can still land.
            for (int st = max(0, NST - S); st < NST; ++st)
                if ((st & 1) == warp) ptx::mbar_drain(fullC + 8 * (st % S), (st / S) & 1, p.err);
        }
    } else if (warp == kWarpX) {
        // ---------------- activations (B operand) ----------------
        // x may be the output of the preceding kernel: wait for it.  The rows
        // are read through L2 only (ld.global.cg), never from a stale L1 line.
        ptx::grid_dependency_wait();
        const T *x = static_cast<const T *>(p.x);
        const int units = p.M * 64;  // (row, k-block of the stage, 16-byte chunk)
        for (int bs = 0; bs < KB / kBStageKb; ++bs) {
            const int slot = bs & 1;
            if (bs >= 2) ptx::mbar_wait(emptyB + 8 * slot, ((bs >> 1) - 1) & 1, p.err);
            uint8_t *dst = gbase + (b0 - base) + slot * B_STAGE;
            for (int u0 = 0; u0 < units; u0 += 32 * 4) {
                uint4 v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int u = u0 + 32 * i + lane;
                    if (u < units) {
                        const int r = u >> 6, b = (u >> 3) & 7, c = u & 7;
                        v[i] = __ldcg(reinterpret_cast<const uint4 *>(x + (int64_t)r * p.K +
                                                                      (bs * kBStageKb + b) * 64 + c * 8));
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int u = u0 + 32 * i + lane;
                    if (u < units) {
                        const int r = u >> 6, b = (u >> 3) & 7, c = u & 7;
                        *reinterpret_cast<uint4 *>(dst + b * B_KB + r * 128 + ((c ^ (r & 7)) << 4)) = v[i];
                    }
                }
            }
            ptx::fence_proxy_async_smem();  // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(fullB + 8 * slot);
        }
    } else if (warp == kWarpMma) {
        // ---------------- MMA issuer ----------------
        const bool leader = elect_one();
        const int gs_mask = (1 << p.gs_log) - 1;
        for (int kb = 0; kb < KB; ++kb) {
            const int a = kb % kASlots;
            const int bslot = (kb / kBStageKb) & 1;
            if (leader) {
                ptx::mbar_wait<false>(fullA + 8 * a, (kb / kASlots) & 1, p.err);
                if (kb % kBStageKb == 0) ptx::mbar_wait<false>(fullB + 8 * bslot, (kb / (2 * kBStageKb)) & 1, p.err);
                const uint64_t db = sw128_desc(b0 + bslot * B_STAGE + (kb % kBStageKb) * B_KB);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int e0 = kb * 64 + 16 * j;
                    const int g = e0 >> p.gs_log, d = g & (kDSlots - 1);
                    const bool first = (e0 & gs_mask) == 0, last = ((e0 + 16) & gs_mask) == 0;
                    if (first && g >= kDSlots) ptx::mbar_wait<false>(emptyD + 8 * d, ((g / kDSlots) - 1) & 1, p.err);
                    tc_fence_after();
                    tc_mma_ts(tmem + kDCol0 + 16u * d, tmem + 32u * a + 8u * j, db + 2u * j, IDESC, first ? 0u : 1u);
                    if (last) tc_commit(fullD + 8 * d);
                }
                tc_commit(emptyA + 8 * a);
                if (kb % kBStageKb == kBStageKb - 1 || kb == KB - 1) tc_commit(emptyB + 8 * bslot);
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
        // ---------------- code placement ----------------
        const int h = (warp - kWarpUnp) >> 2, q = warp & 3;
        const int j = q * p.RQ + lane;                 // row of this lane within the CTA
        const bool valid = lane < p.RQ && j < R;       // (lane 31 never holds a row)
        // Batches of kPlaceBatch own k-blocks: each is stored as soon as it is
        // placed, and one tcgen05.wait::st covers the batch before its A
        // slots are published.
        for (int kb0 = h; kb0 < KB; kb0 += 2 * kPlaceBatch) {
#pragma unroll
            for (int t = 0; t < kPlaceBatch; ++t) {
                const int kb = kb0 + 2 * t;
                if (kb >= KB) break;
                const int st = kb / KBS, kbs = kb % KBS;
                const int slot = st % S;
                if (kbs < 2) ptx::mbar_wait(fullC + 8 * slot, (st / S) & 1, p.err);
                const int a = kb % kASlots;
                if (kb >= kASlots) ptx::mbar_wait<false>(emptyA + 8 * a, ((kb / kASlots) - 1) & 1, p.err);
                uint32_t w[BITS * 2];
#pragma unroll
                for (int i = 0; i < BITS * 2; ++i) w[i] = 0;  // code 0 (a = 1) for lanes without a row
                if (valid) {
                    const uint8_t *row = gbase + (c0 - base) + slot * p.stage_bytes + j * 128;
#pragma unroll
                    for (int c = 0; c < BITS / 2; ++c) {
                        const int chunk = (kbs * (BITS / 2) + c) ^ (j & 7);
                        const uint4 u = *reinterpret_cast<const uint4 *>(row + (chunk << 4));
                        w[4 * c] = u.x;
                        w[4 * c + 1] = u.y;
                        w[4 * c + 2] = u.z;
                        w[4 * c + 3] = u.w;
                    }
                }
                __syncwarp();
                // This group's reads of the stage are done after its last k-block there.
                if (lane == 0 && kbs >= KBS - 2) ptx::mbar_arrive(emptyC + 8 * slot);
                uint32_t v[32];
                place_codes<T, BITS>(w, v);
                tc_fence_after();
                tmem_st32(tmem + ((uint32_t)(32 * q) << 16) + 32u * a, v);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < kPlaceBatch; ++t) {
                    const int kb = kb0 + 2 * t;
                    if (kb < KB) ptx::mbar_arrive(fullA + 8 * (kb % kASlots));
                }
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;
        const int j = q * p.RQ + lane;
        const bool valid = lane < p.RQ && j < R;
        const int64_t rowg = (int64_t)r0 + j;
        const uint16_t *srow = p.scales + (valid ? rowg : 0) * p.gpr;
        const uint16_t *brow = p.biases + (valid ? rowg : 0) * p.gpr;
        // Scale/bias windows of 8 groups (16 bytes), one window ahead.
        uint4 s_cur = make_uint4(0, 0, 0, 0), b_cur = s_cur, s_nxt = s_cur, b_nxt = s_cur;
        if (valid) {
            s_cur = __ldg(reinterpret_cast<const uint4 *>(srow));
            b_cur = __ldg(reinterpret_cast<const uint4 *>(brow));
            if (G > 8) {
                s_nxt = __ldg(reinterpret_cast<const uint4 *>(srow + 8));
                b_nxt = __ldg(reinterpret_cast<const uint4 *>(brow + 8));
            }
        }
        float acc[MR];
#pragma unroll
        for (int m = 0; m < MR; ++m) acc[m] = 0.f;
        int wbase = 0;
        for (int g = 0; g < G; ++g) {
            const int d = g & (kDSlots - 1);
            if (g >= wbase + 8) {
                s_cur = s_nxt;
                b_cur = b_nxt;
                wbase += 8;
                if (valid && wbase + 8 < G) {
                    s_nxt = __ldg(reinterpret_cast<const uint4 *>(srow + wbase + 8));
                    b_nxt = __ldg(reinterpret_cast<const uint4 *>(brow + wbase + 8));
                }
            }
            ptx::mbar_wait<false>(fullD + 8 * d, (g / kDSlots) & 1, p.err);
            tc_fence_after();
            uint32_t v[MR];
            tmem_ld_cols<MR>(tmem + ((uint32_t)(32 * q) << 16) + kDCol0 + 16u * d, v);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(emptyD + 8 * d);
            const int o = g - wbase;
            const uint32_t sw = pick_word(s_cur, o >> 1), bw = pick_word(b_cur, o >> 1);
            const uint16_t s16 = (uint16_t)((o & 1) ? (sw >> 16) : (sw & 0xffffu));
            const uint16_t b16 = (uint16_t)((o & 1) ? (bw >> 16) : (bw & 0xffffu));
            const float s = kF16 ? __half2float(__ushort_as_half(s16)) : __uint_as_float((uint32_t)s16 << 16);
            const float bv = kF16 ? __half2float(__ushort_as_half(b16)) : __uint_as_float((uint32_t)b16 << 16);
            const float sp = s * QS;                   // exact
#pragma unroll
            for (int m = 0; m < MR; ++m) {
                const float dm = __uint_as_float(v[m]);
                const float xs = __shfl_sync(0xffffffffu, dm, 31);  // X_g[m] from the all-ones lane
                // (QS s)(D - X) + b X: the difference first, so that no term is
                // larger than the result's own scale.
                acc[m] = __fmaf_rn(sp, dm - xs, __fmaf_rn(bv, xs, acc[m]));
            }
        }
        if (valid) {
            T *y = static_cast<T *>(p.y);
            const float lb = layer_bias<T>(p.bias, p.bias_value, rowg);
#pragma unroll
            for (int m = 0; m < MR; ++m)
                if (m < p.M) y[(int64_t)m * p.N + rowg] = Dt<T>::from_f(acc[m] + lb);
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
    int grid, R, RQ, S, stage_bytes;
    size_t smem;
};

bool plan_tc(const QmmArgs &a, int mr, TcPlan &p) {
    const int64_t sms = num_sms();
    int64_t G = std::min<int64_t>(sms, (a.N + 7) / 8);
    int64_t R = std::min<int64_t>((a.N + G - 1) / G, kMaxRows);
    G = (a.N + R - 1) / R;  // every CTA owns at least one row
    p.grid = (int)G;
    p.R = (int)R;
    p.RQ = (int)((R + 3) / 4);
    p.stage_bytes = (int)(((R * 128) + 1023) / 1024 * 1024);
    const int nb = mr <= 8 ? 8 : 16;
    const size_t bring = (size_t)2 * kBStageKb * nb * 128 + (nb == 8 ? 1024 : 0);
    const size_t bars = 512;
    const size_t fixed = 1024 /*alignment*/ + bring + bars;
    if (fixed + 2 * (size_t)p.stage_bytes > kSmemBudget) return false;
    p.S = (int)std::min<size_t>(8, (kSmemBudget - fixed) / p.stage_bytes);
    p.smem = fixed + (size_t)p.S * p.stage_bytes;
    return p.S >= 2;
}

template <typename T, int BITS, int MR>
cudaError_t launch_tc(const QmmArgs &a, cudaStream_t s) {
    auto kern = qgemv_tc_kernel<T, BITS, MR>;
    TcPlan p{};
    if (!plan_tc(a, MR, p)) return cudaErrorInvalidValue;
    struct Tag;
    cudaError_t e = configure_once<Tag>(p.smem, [&]() {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
        if (r != cudaSuccess) return r;
        return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    cudaSharedmemCarveoutMaxShared);
    });
    if (e != cudaSuccess) return e;
    // Packed codes as [N rows, K*BITS/32 words]: a box is 32 words (128 bytes)
    // of R rows, 128-byte swizzled; rows past N read as zero.
    CUtensorMap tw;
    const uint64_t words = (uint64_t)a.K * BITS / 32;
    if (!make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.wq, words, (uint64_t)a.N, words * 4, 32,
                     (uint32_t)p.R, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    DecParams dp{};
    dp.x = a.x;
    dp.y = a.y;
    dp.scales = static_cast<const uint16_t *>(a.scales);
    dp.biases = static_cast<const uint16_t *>(a.biases);
    dp.M = (int)a.M;
    dp.N = (int)a.N;
    dp.K = (int)a.K;
    dp.gpr = (int)(a.K / a.group_size);
    dp.gs_log = __builtin_ctz((unsigned)a.group_size);
    dp.R = p.R;
    dp.RQ = p.RQ;
    dp.S = p.S;
    dp.stage_bytes = p.stage_bytes;
    dp.KB = (int)(a.K / 64);
    dp.bias = a.bias;
    dp.bias_value = a.bias_value;
    dp.err = device_error_word();
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
    e = cudaLaunchKernelEx(&cfg, kern, tw, dp);
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

// bf16/f16, transpose, 1..16 rows, 2- or 4-bit codes, K a multiple of 512
// (whole activation stages and code chunks), groups per row a multiple of 8
// (16-byte scale/bias windows), 16-byte aligned operands.
bool gemv_tc_supported(qmm_dtype dt, const QmmArgs &a) {
    if (!a.transpose || a.M < 1 || a.M > 16) return false;
    if (dt != QMM_BF16 && dt != QMM_F16) return false;
    if (a.mode != QMM_MODE_AFFINE) return false;
    if (a.bits != 2 && a.bits != 4) return false;
    if (a.K % 512 != 0 || (a.K / a.group_size) % 8 != 0) return false;
    if (a.N < 1 || a.N > (1 << 30) || a.K > (1 << 20)) return false;
    if ((reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.wq) |
         reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases)) & 15)
        return false;
    TcPlan p{};
    if (!plan_tc(a, a.M <= 8 ? 8 : 16, p)) return false;
    return encode_fn() != nullptr;
}

cudaError_t launch_gemv_tc(qmm_dtype dt, const QmmArgs &a, cudaStream_t s) {
    if (dt == QMM_BF16) return a.bits == 4 ? tc_rows<__nv_bfloat16, 4>(a, s) : tc_rows<__nv_bfloat16, 2>(a, s);
    return a.bits == 4 ? tc_rows<__half, 4>(a, s) : tc_rows<__half, 2>(a, s);
}

}  // namespace qmm
