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

__global__ void __launch_bounds__(256)
mapped_copy_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst, int64_t bytes, int vec16) {
    // Let the next kernel of the stream (the product, or the next step's
    // copy) launch now; it waits for this grid where it depends on it.
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (vec16) {
        const uint4 *s = reinterpret_cast<const uint4 *>(src);
        uint4 *d = reinterpret_cast<uint4 *>(dst);
        for (int64_t i = t0; i < bytes / 16; i += stride) d[i] = __ldcg(s + i);
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
    const unsigned grid = (unsigned)std::min<int64_t>((units + 255) / 256, 4 * (int64_t)num_sms());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
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
