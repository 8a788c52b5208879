// copy.cu -- copies between page-locked host memory and device memory done by
// kernels instead of the copy engines, for qmm_quantized_matmul_host.  A
// page-locked allocation is mapped into the device's address space, so a
// kernel can read or write it directly; launched with programmatic dependent
// launch, such a copy sits in the same chain as the products around it: the
// next product's launch, and its weight stream, start while the copy runs,
// where a copy-engine transfer between two kernels would make every product
// start cold.  Each copy kernel waits (griddepcontrol.wait) for the preceding
// grid before it touches memory, so it never overwrites data a previous
// kernel still reads, nor reads a result not yet written.  It reads with
// ld.global.cg (L2 only): every byte is used once.
#include "ptx_sm100.cuh"
#include "qmm_internal.cuh"

namespace qmm {
namespace {

// Small CTAs: a copy kernel launched early sits in griddepcontrol.wait beside
// the two decode-kernel CTAs of an SM (this call's and the next one's), which
// leave it only ~5,600 registers; a larger CTA there would keep the next
// call's CTA from starting early on that SM.
constexpr int kCopyThreads = 64;
constexpr int kCopyUnroll = 8;  // 16-byte loads in flight per thread

__global__ void __launch_bounds__(kCopyThreads)
mapped_copy_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst, int64_t bytes, int vec16) {
    // Wait for the preceding grid (the previous product), then let the next
    // kernel of the stream launch: it is placed once the previous call's CTAs
    // have left the SMs (one per SM), and fills its ring while this copy runs.
    ptx::grid_dependency_wait();
    ptx::grid_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (vec16) {
        // all of a thread's loads first (one round trip over the bus), then
        // the stores
        const uint4 *s = reinterpret_cast<const uint4 *>(src);
        uint4 *d = reinterpret_cast<uint4 *>(dst);
        const int64_t n = bytes / 16;
        for (int64_t i0 = t0; i0 < n; i0 += stride * kCopyUnroll) {
            uint4 v[kCopyUnroll];
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) {
                const int64_t i = i0 + u * stride;
                if (i < n) v[u] = __ldcg(s + i);
            }
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) {
                const int64_t i = i0 + u * stride;
                if (i < n) d[i] = v[u];
            }
        }
    } else {
        for (int64_t i = t0; i < bytes; i += stride) dst[i] = __ldcg(src + i);
    }
}

}  // namespace

// The address through which a kernel on the current device reaches the
// page-locked host memory at p, or nullptr when p is not page-locked or not
// mapped (then the caller uses a copy engine).
const void *mapped_host_pointer(const void *p) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        (void)cudaGetLastError();  // (a failed query leaves a non-sticky error)
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) return nullptr;
    return at.devicePointer;
}

cudaError_t launch_mapped_copy(const void *src, void *dst, size_t bytes, cudaStream_t s) {
    if (bytes == 0) return cudaSuccess;
    const bool vec16 = bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                       (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
    const int64_t units = vec16 ? (int64_t)(bytes / 16) : (int64_t)bytes;
    const int64_t per_cta = (int64_t)kCopyThreads * (vec16 ? kCopyUnroll : 1);
    const unsigned grid = (unsigned)std::min<int64_t>((units + per_cta - 1) / per_cta, 4 * (int64_t)num_sms());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kCopyThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, mapped_copy_kernel, static_cast<const uint8_t *>(src),
                                       static_cast<uint8_t *>(dst), (int64_t)bytes, vec16 ? 1 : 0);
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace qmm
