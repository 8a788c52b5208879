// gather.cu -- gather_qmm: y[b] = x[xi(b)] (*) W[ei(b)] for a batch of
// (activation, expert) pairs (EMLX.Quantization, section
// gather_quantized_matmul; mlx-rs ops/quantization.rs, gather_qmm).  No
// expert weight is ever copied: the grouped product reads each expert's
// packed rows where they lie in the stacked [E, N, K*bits/32] array.
//
// Tensor-core path (bf16/f16, transpose):
//   1. gather_prep_kernel (one CTA): validates every entry's indices, checks
//      whether the expert keys are already non-decreasing, and if not sorts
//      the entries by expert (stable counting sort: per-warp histograms, one
//      scan, warp-ranked scatter).  It then cuts each expert's rows into
//      chunks of at most `cap` rows (the tile width of the product) and writes
//      the chunk table, the sorted-row -> output-row map and a header.
//   2. gather_rows_kernel: copies the activation rows into sorted order (skipped
//      when that order is x's own) and writes zeros to the output rows of
//      entries with out-of-range indices.
//   3. the grouped tensor-core kernel (gemm_sm100.cu) walks chunk x 128-row
//      output tiles, reading the weight tiles of each chunk's expert.
// Everything the kernels need is in the caller's workspace; nothing is
// allocated.  The layout of that workspace is gather_ws_layout below.
#include <algorithm>
#include <mutex>

#include "qmm_internal.cuh"

namespace qmm {

namespace {

constexpr int kPrepThreads = 1024;
constexpr int kPrepSmemInts = 200 * 1024 / 4;

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

// Expert key of entry b: its expert, or n_experts for an invalid entry (so
// invalid entries sort last).
__device__ __forceinline__ int entry_key(const GatherIndex &gi, int64_t b) {
    int64_t xi, ei;
    return gather_entry(gi, b, xi, ei) ? (int)ei : (int)gi.n_experts;
}

// Exclusive prefix sum of a[0..L) in place (shared memory), by the whole
// block; a[L] receives the total.  tmp: 32 ints of shared memory.
__device__ void block_exclusive_scan(int *a, int L, int *tmp) {
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = (nthr + 31) >> 5;
    const int per = (L + nthr - 1) / nthr;
    const int lo = min(L, tid * per), hi = min(L, lo + per);
    int s = 0;
    for (int i = lo; i < hi; ++i) s += a[i];
    int x = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int v = lane < nwarps ? tmp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += y;
        }
        tmp[lane] = v;
    }
    __syncthreads();
    int run = x - s + (warp > 0 ? tmp[warp - 1] : 0);
    for (int i = lo; i < hi; ++i) {
        const int t = a[i];
        a[i] = run;
        run += t;
    }
    if (tid == 0) a[L] = tmp[nwarps - 1];
    __syncthreads();
}

// Rows per chunk for an expert with `rows` rows: as even as possible, a
// multiple of 16 (the MMA N step), at most cap.
__device__ __forceinline__ int chunk_size(int rows, int cap) {
    const int n0 = (rows + cap - 1) / cap;
    const int even = (rows + n0 - 1) / n0;
    return min(cap, (even + 15) & ~15);
}

struct PrepArgs {
    GatherIndex gi;
    int64_t M;
    int cap;            // rows per chunk at most (the product's tile width)
    int W;              // warps that count (segments of the batch)
    int x_identity_ok;  // lhs absent and x_batch == batch
    GatherHeader *hdr;
    int4 *chunks;
    int32_t *perm;      // sorted position -> batch entry
    int32_t *dst_rows;  // sorted activation row -> output row
    int *err;
};

__global__ void __launch_bounds__(kPrepThreads, 1) gather_prep_kernel(const PrepArgs a) {
    extern __shared__ int sm[];
    __shared__ int tmp[32];
    __shared__ int unsorted;
    const GatherIndex &gi = a.gi;
    const int E = (int)gi.n_experts, E1 = E + 1, W = a.W;
    const int64_t batch = gi.batch;
    int *cnt = sm;                  // [W][E1] per-warp counts, then bases
    int *koff = sm + W * E1;        // [E1 + 1] first sorted position of each key
    int *nch = koff + (E1 + 1);     // [E1 + 1] chunks per expert, then first chunk
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;

    for (int i = tid; i < W * E1; i += nthr) cnt[i] = 0;
    if (tid == 0) unsorted = 0;
    __syncthreads();
    for (int64_t b = tid + 1; b < batch; b += nthr)
        if (entry_key(gi, b - 1) > entry_key(gi, b)) unsorted = 1;

    // Per-warp histograms over contiguous segments of the batch.
    const int64_t seg = (batch + W - 1) / W;
    const int64_t lo = (int64_t)warp * seg, hi = min(batch, lo + seg);
    if (warp < W) {
        for (int64_t base = lo; base < hi; base += 32) {
            const int64_t b = base + lane;
            const bool act = b < hi;
            const int key = act ? entry_key(gi, b) : -1 - lane;
            const unsigned same = __match_any_sync(0xffffffffu, key);
            if (act && lane == __ffs(same) - 1) cnt[warp * E1 + key] += __popc(same);
        }
    }
    __syncthreads();
    for (int k = tid; k < E1; k += nthr) {
        int run = 0;
        for (int w = 0; w < W; ++w) {
            const int t = cnt[w * E1 + k];
            cnt[w * E1 + k] = run;
            run += t;
        }
        koff[k] = run;
    }
    __syncthreads();
    block_exclusive_scan(koff, E1, tmp);
    for (int i = tid; i < W * E1; i += nthr) cnt[i] += koff[i % E1];
    __syncthreads();

    const bool identity = unsorted == 0;
    if (identity) {
        for (int64_t i = tid; i < batch; i += nthr) a.perm[i] = (int32_t)i;
    } else if (warp < W) {
        // Stable scatter: lanes with the same key take consecutive slots in
        // lane order, and each warp's segment follows the earlier warps'.
        const unsigned lt = (1u << lane) - 1u;
        for (int64_t base = lo; base < hi; base += 32) {
            const int64_t b = base + lane;
            const bool act = b < hi;
            const int key = act ? entry_key(gi, b) : -1 - lane;
            const unsigned same = __match_any_sync(0xffffffffu, key);
            int pos = 0;
            if (act) pos = cnt[warp * E1 + key] + __popc(same & lt);
            __syncwarp();
            if (act) {
                a.perm[pos] = (int32_t)b;
                if (lane == __ffs(same) - 1) cnt[warp * E1 + key] += __popc(same);
            }
            __syncwarp();
        }
    }

    // Chunks of each expert's rows.
    const int M = (int)a.M;
    for (int k = tid; k < E1; k += nthr) {
        const int rows = k < E ? (koff[k + 1] - koff[k]) * M : 0;
        nch[k] = rows ? (rows + chunk_size(rows, a.cap) - 1) / chunk_size(rows, a.cap) : 0;
    }
    __syncthreads();
    block_exclusive_scan(nch, E1, tmp);
    for (int k = tid; k < E; k += nthr) {
        const int rows = (koff[k + 1] - koff[k]) * M;
        if (rows == 0) continue;
        const int size = chunk_size(rows, a.cap);
        const int first = koff[k] * M;
        for (int j = 0, c = nch[k]; j * size < rows; ++j, ++c)
            a.chunks[c] = make_int4(k, first + j * size, min(size, rows - j * size), 0);
    }
    __syncthreads();  // perm complete (global writes of this block)

    const int valid = koff[E];
    for (int64_t r = tid; r < (int64_t)valid * M; r += nthr) {
        const int64_t i = r / M, m = r - i * M;
        a.dst_rows[r] = (int32_t)((int64_t)a.perm[i] * M + m);
    }
    if (tid == 0) {
        a.hdr->num_chunks = nch[E1];
        a.hdr->use_x = (identity && a.x_identity_ok) ? 1 : 0;
        a.hdr->valid_entries = valid;
        a.hdr->pad = 0;
        if (valid < batch) record_device_error(a.err, QMM_ERR_INDEX);
    }
}

// Sorted activation rows (unless x is already in that order) and zeroed
// output rows of invalid entries.  One row per CTA iteration, 16-byte moves.
template <typename T>
__global__ void __launch_bounds__(128) gather_rows_kernel(const GatherIndex gi, int64_t M, int64_t K,
                                                          int64_t N, const T *__restrict__ x,
                                                          T *__restrict__ xs, T *__restrict__ y,
                                                          const int32_t *__restrict__ perm,
                                                          const GatherHeader *__restrict__ hdr) {
    const int64_t R = gi.batch * M;
    const int valid = __ldg(&hdr->valid_entries);
    const bool copy = __ldg(&hdr->use_x) == 0;
    const int64_t vec = K * (int64_t)sizeof(T) / 16;  // K * sizeof(T) is a multiple of 16
    for (int64_t r = blockIdx.x; r < R; r += gridDim.x) {
        const int64_t i = r / M, m = r - i * M;
        const int64_t b = __ldg(perm + i);
        if (i < valid) {
            if (!copy) continue;
            int64_t xi, ei;
            gather_entry(gi, b, xi, ei);
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (xi * M + m) * K);
            uint4 *dst = reinterpret_cast<uint4 *>(xs + r * K);
            for (int64_t v = threadIdx.x; v < vec; v += blockDim.x) dst[v] = __ldg(src + v);
        } else {
            T *row = y + (b * M + m) * N;
            for (int64_t n = threadIdx.x; n < N; n += blockDim.x) row[n] = Dt<T>::from_f(0.f);
        }
    }
}

}  // namespace

GatherWorkspace gather_ws_layout(int64_t batch, int64_t M, int64_t K, int64_t n_experts,
                                 int elt_bytes) {
    GatherWorkspace w{};
    const int64_t R = batch * M;
    w.max_chunks = n_experts + (R + 63) / 64 + 1;
    size_t off = 0;
    w.hdr = off;
    off += round256(sizeof(GatherHeader));
    w.chunks = off;
    off += round256((size_t)w.max_chunks * sizeof(int4));
    w.perm = off;
    off += round256((size_t)batch * sizeof(int32_t));
    w.dst_rows = off;
    off += round256((size_t)R * sizeof(int32_t));
    w.x_sorted = off;
    off += round256((size_t)R * (size_t)K * (size_t)elt_bytes);
    w.total = off;
    return w;
}

int gather_chunk_rows(int64_t rows) { return rows <= 64 ? 64 : (rows <= 128 ? 128 : 256); }

bool gather_prep_fits(int64_t n_experts) {
    const int64_t E1 = n_experts + 1;
    return (kPrepSmemInts - 2 * (E1 + 1)) / E1 >= 1;
}

cudaError_t launch_gather_tc(qmm_dtype dt, const GatherCall &c, cudaStream_t s) {
    const int64_t R = c.gi.batch * c.M;
    const GatherWorkspace w = gather_ws_layout(c.gi.batch, c.M, c.K, c.gi.n_experts, 2);
    uint8_t *ws = static_cast<uint8_t *>(c.workspace);
    GatherHeader *hdr = reinterpret_cast<GatherHeader *>(ws + w.hdr);
    int4 *chunks = reinterpret_cast<int4 *>(ws + w.chunks);
    int32_t *perm = reinterpret_cast<int32_t *>(ws + w.perm);
    int32_t *dst_rows = reinterpret_cast<int32_t *>(ws + w.dst_rows);
    void *x_sorted = ws + w.x_sorted;
    const int cap = gather_chunk_rows(R);

    // 1. prep
    PrepArgs p{};
    p.gi = c.gi;
    p.M = c.M;
    p.cap = cap;
    const int64_t E1 = c.gi.n_experts + 1;
    p.W = (int)std::min<int64_t>(32, (kPrepSmemInts - 2 * (E1 + 1)) / E1);
    if (p.W < 1) return cudaErrorInvalidValue;
    p.x_identity_ok = (c.gi.lhs == nullptr && c.gi.x_batch == c.gi.batch) ? 1 : 0;
    p.hdr = hdr;
    p.chunks = chunks;
    p.perm = perm;
    p.dst_rows = dst_rows;
    p.err = device_error_word();
    const size_t smem = (size_t)(p.W * E1 + 2 * (E1 + 1)) * sizeof(int);
    struct Tag;
    cudaError_t e = configure_once<Tag>(smem, [&]() {
        return cudaFuncSetAttribute(gather_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
    if (e != cudaSuccess) return e;
    gather_prep_kernel<<<1, kPrepThreads, smem, s>>>(p);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // 2. rows
    const int grid = (int)std::min<int64_t>(R, (int64_t)num_sms() * 8);
    if (dt == QMM_BF16)
        gather_rows_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
            c.gi, c.M, c.K, c.N, static_cast<const __nv_bfloat16 *>(c.x),
            static_cast<__nv_bfloat16 *>(x_sorted), static_cast<__nv_bfloat16 *>(c.y), perm, hdr);
    else
        gather_rows_kernel<__half><<<grid, 128, 0, s>>>(
            c.gi, c.M, c.K, c.N, static_cast<const __half *>(c.x), static_cast<__half *>(x_sorted),
            static_cast<__half *>(c.y), perm, hdr);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // 3. grouped product
    GroupedArgs g{};
    g.x = c.x;
    g.x_sorted = x_sorted;
    g.wq = c.wq;
    g.scales = c.scales;
    g.biases = c.biases;
    g.y = c.y;
    g.x_rows = c.gi.x_batch * c.M;
    g.rows = R;
    g.N = c.N;
    g.K = c.K;
    g.n_experts = c.gi.n_experts;
    g.max_chunks = w.max_chunks;
    g.group_size = c.group_size;
    g.bits = c.bits;
    g.transpose = c.transpose;
    g.chunk_rows = cap;
    g.hdr = hdr;
    g.chunks = chunks;
    g.dst_rows = dst_rows;
    return launch_gemm_grouped(dt, g, s);
}

// ---------------------------------------------------------------------------
// Built-in scratch for qmm_gather_qmm_static: a fixed device array in this
// module, so that callers without a device allocator get the tensor-core path
// without passing a workspace.  Its address is looked up once per device.
// Nothing in it needs to start at zero: the preparation kernel writes every
// byte the later kernels read.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_gather_scratch[QMM_GATHER_STATIC_SCRATCH_BYTES];

cudaError_t gather_static_scratch(void **ptr) {
    static void *cached[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gather_scratch);
        if (e != cudaSuccess) return e;
        cached[dev] = p;
    }
    *ptr = cached[dev];
    return cudaSuccess;
}

}  // namespace qmm
