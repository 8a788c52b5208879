/*
 * qmm.h -- C ABI of libqmm, group-wise affine quantized matmul for NVIDIA
 * B200 (sm_100a).
 *
 * The operations follow the MLX quantization API as these documents describe it:
 *   EMLX.Quantization (emlx 0.4.2): quantize, dequantize, quantized_matmul,
 *     gather_quantized_matmul;
 *   Emily.QuantizedWeight (emily 0.7.2), section Layout: the packed value /
 *     scales / biases layout;
 *   Emily.Quantization.Layers (emily 1.0.0), quantized_dense: the two weight
 *     layouts selected by `transpose`;
 *   mlx-rs src/mlx_rs/ops/quantization.rs: quantize, quantized_matmul,
 *     dequantize, gather_qmm and their defaults (mode "affine", group size 64,
 *     4 bits).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  Every array argument is a DEVICE pointer owned by the caller,
 *   row-major and contiguous, and 16-byte aligned (misaligned pointers are
 *   rejected with QMM_ERR_INVALID_ARG).  The library allocates no device
 *   memory; gather_qmm and qmm_quantized_matmul_ws take caller-provided
 *   workspaces.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream).  Calls only enqueue work and return; results are ready
 *   when the stream is synchronised.
 * Errors.  Arguments are validated before anything is launched; on any error
 *   nothing is enqueued.  Exceptions never cross the ABI.  A thread-local
 *   message for the last failure is available from qmm_last_error().
 * Packing.  bits in {2, 3, 4, 6, 8} (Emily.QuantizedWeight, from_dense); a
 *   row of cols codes takes cols*bits/32 uint32 words; code j of a row
 *   occupies bits [j*bits, (j+1)*bits) of the row's bit stream, bit i of the
 *   stream being bit (i mod 32) of word i/32 (least significant first).  For
 *   2, 4 and 8 bits that is bit (j mod 32/bits)*bits of word j/(32/bits);
 *   3- and 6-bit codes may straddle two words.
 * Groups.  group_size in {32, 64, 128}; one scale and one bias per group of
 *   consecutive elements along the LAST STORED axis of the weight (the packed
 *   axis), for both matmul layouts.
 * Dtypes.  "affine": scales and biases share the dense weight's dtype;
 *   outputs take the scales dtype (EMLX.Quantization, section
 *   quantized_matmul); activations must have that dtype too.
 * Mode.  `mode` NULL means "affine" (the default in every document above).
 *   The microscaled modes of Emily.QuantizedWeight, section Microscaled modes,
 *   fix group_size and bits and have no biases (pass NULL):
 *     "mxfp4"  group_size 32, bits 4: E2M1 elements, one E8M0 scale byte per group
 *     "mxfp8"  group_size 32, bits 8: E4M3 elements, one E8M0 scale byte per group
 *     "nvfp4"  group_size 16, bits 4: E2M1 elements, one E4M3 scale byte per group
 *   scales is then a uint8 array [rows, cols/group_size]; the `dtype`
 *   argument names the dense weight's dtype for qmm_quantize, the output's
 *   for qmm_dequantize, and the activations' (= output's) for the matmuls
 *   (EMLX.Quantization, section gather_quantized_matmul: with u8 scales the
 *   output follows the activations).  Quantize rule: mx modes X =
 *   2^(floor(log2 max|v|) - emax), emax 2 (E2M1) or 8 (E4M3), clamped to
 *   E8M0's range (OCP Microscaling Formats v1.0); nvfp4 X = max|v|/6 rounded
 *   to E4M3; elements v/X rounded to nearest-even and saturated; an
 *   all-zero group stores zeros; dequantized w = X * element.  A group size or
 *   bits other than the mode's, or non-NULL biases, is QMM_ERR_INVALID_ARG.
 *   gather_qmm takes "affine" weights only (QMM_ERR_UNSUPPORTED otherwise).
 *   Any other mode string returns QMM_ERR_INVALID_ARG.
 */
#ifndef QMM_H
#define QMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QMM_OK = 0,
    QMM_ERR_INVALID_ARG = 1, /* bad size, pointer, group size, bits, ... */
    QMM_ERR_UNSUPPORTED = 2, /* valid, but not for this entry or forced path */
    QMM_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    QMM_ERR_TIMEOUT = 4,     /* a kernel's bounded wait ran out (device word) */
    QMM_ERR_INDEX = 5,       /* an expert / row index was out of range */
    QMM_ERR_WORKSPACE = 6    /* workspace missing or smaller than required */
} qmm_status;

typedef enum { QMM_F32 = 0, QMM_BF16 = 1, QMM_F16 = 2 } qmm_dtype;

/*
 * qmm_quantize -- EMLX.Quantization, section quantize; mlx-rs quantize.
 * Quantizes w[rows, cols] (dtype `dtype`) group by group along its last axis.
 *   w       in : [rows, cols] dense weight (leading axes flattened into rows)
 *   wq      out: [rows, cols*bits/32] uint32 packed codes
 *   scales  out: [rows, cols/group_size], dtype `dtype`
 *   biases  out: [rows, cols/group_size], dtype `dtype`
 * Rule ("affine"): bias = group min, scale = (max - min)/(2^bits - 1) in
 * fp32, both rounded to `dtype` (nearest-even); q = clamp(rint((w - bias) /
 * scale), 0, 2^bits - 1) against the stored scale and bias, 0 when the scale
 * is 0.  Microscaled modes: see the header's Mode paragraph (scales uint8,
 * biases NULL).  cols must be a positive multiple of group_size; rows may be
 * 0 (no-op).
 */
qmm_status qmm_quantize(const void *w, qmm_dtype dtype, int64_t rows, int64_t cols,
                        int group_size, int bits, const char *mode,
                        uint32_t *wq, void *scales, void *biases, void *stream);

/*
 * qmm_dequantize -- EMLX.Quantization, section dequantize (every mode);
 * mlx-rs dequantize.
 *   "affine": out[r, c] = round_to_dtype(fmaf(scale[r, c/gs], q[r, c], bias[r, c/gs]))
 *   wq [rows, cols*bits/32], scales/biases [rows, cols/gs], out [rows, cols],
 *   all in `dtype` except wq.  Microscaled modes: out = round_to_dtype(X *
 *   element), scales uint8, biases NULL, `dtype` the output's.
 */
qmm_status qmm_dequantize(const uint32_t *wq, const void *scales, const void *biases,
                          qmm_dtype dtype, int64_t rows, int64_t cols, int group_size,
                          int bits, const char *mode, void *out, void *stream);

/*
 * qmm_quantized_matmul -- mlx-rs quantized_matmul; EMLX.Quantization, section
 * quantized_matmul; Emily.Quantization.Layers, quantized_dense.
 *   x [M, K] (dtype), y [M, N] (dtype).
 *   transpose != 0: W is [N, K] ("[out, in]"), y = x @ W^T;
 *                   wq [N, K*bits/32], scales/biases [N, K/gs]; K % gs == 0.
 *   transpose == 0: W is [K, N] ("[in, out]"), y = x @ W;
 *                   wq [K, N*bits/32], scales/biases [K, N/gs]; N % gs == 0.
 * The packed weight is streamed and dequantized inside the product; no dense
 * weight is written to memory.  M == 0 or N == 0 is a no-op.
 * Early start: the decode kernel (bf16/f16, transpose, M <= 4) is launched
 *   with programmatic dependent launch.  If the kernel queued just before it
 *   on the stream allows dependents to start early (PTX
 *   griddepcontrol.launch_dependents), the decode kernel may begin reading
 *   wq, scales and biases -- never x -- before that kernel has finished.  So
 *   wq, scales and biases must not be written by such a kernel right before
 *   the call.  Kernels that do not allow an early start (the usual case, and
 *   every kernel of this library that writes a packed weight, such as
 *   qmm_quantize) complete before the call reads anything.
 */
qmm_status qmm_quantized_matmul(const void *x, int64_t M, int64_t K,
                                const uint32_t *wq, const void *scales, const void *biases,
                                qmm_dtype dtype, int64_t N, int transpose,
                                int group_size, int bits, const char *mode,
                                void *y, void *stream);

/*
 * qmm_quantized_matmul_ws -- qmm_quantized_matmul with a caller workspace.
 * Nothing in the documents this library follows has a counterpart: the
 * workspace only lets the tensor-core path split the k-blocks of each output
 * tile over several CTAs ("stream-K") when a problem has fewer 128-feature
 * weight tiles than the GPU has SMs and at most 64 activation rows per tile
 * (decode batches of 5..64 rows with W [N, K] -- 1..64 rows for 3- and 6-bit
 * codes, which the streaming decode kernel does not take -- 1..64 rows with
 * W [K, N], small weights), so that every SM works.
 *   workspace: NULL (whole tiles, exactly qmm_quantized_matmul), or device
 *     memory of at least qmm_quantized_matmul_workspace_size(...) bytes,
 *     256-byte aligned, ZEROED before its first use; every call that returns
 *     QMM_OK leaves it zeroed again (after a QMM_ERR_TIMEOUT from
 *     qmm_device_status, zero it again).  Calls in flight at once must not
 *     share a workspace.  A workspace smaller than needed for a call's split
 *     is not used (whole tiles).  Misaligned: QMM_ERR_WORKSPACE.  (The
 *     decode tensor-core path, QMM_PATH_DECODE_TC, writes its prepared
 *     activations past the first 4096 bytes and leaves those bytes zero.)
 * Results: the parts of a split tile are added in a fixed order, so repeated
 *   calls return identical bits; they can differ from the whole-tile result
 *   in fp32 rounding.
 * qmm_quantized_matmul_workspace_size returns the bytes a call of these sizes
 * can use (0 when it would not split).
 */
size_t qmm_quantized_matmul_workspace_size(int64_t M, int64_t K, int64_t N, int transpose,
                                           int bits, qmm_dtype dtype);
qmm_status qmm_quantized_matmul_ws(const void *x, int64_t M, int64_t K,
                                   const uint32_t *wq, const void *scales, const void *biases,
                                   qmm_dtype dtype, int64_t N, int transpose,
                                   int group_size, int bits, const char *mode,
                                   void *y, void *workspace, size_t workspace_bytes,
                                   void *stream);

/*
 * qmm_quantized_matmul_host -- qmm_quantized_matmul_ws for activations and a
 * result that live in host memory.  Nothing in the documents this library
 * follows has a counterpart (their arrays live wherever the framework keeps
 * them); it is the one call a host program makes per product.  On `stream`
 * it enqueues, in order: the copy of M*K elements from x_host into x_dev,
 * the product of x_dev into y_dev (exactly qmm_quantized_matmul_ws), and the
 * copy of M*N elements from y_dev into y_host.  Page-locked host buffers are
 * copied by kernels that read or write their device mapping (each waits for
 * the preceding kernel of the stream, then lets the next one start, so the
 * product fills its weight ring while x is copied); when the product runs on
 * the streaming decode kernel (W [N, K], 1..4 rows), that kernel also writes
 * the result into a page-locked y_host itself and no copy follows.  Other
 * host memory goes through the copy engines.
 *   x_host, y_host: host memory; page-locked memory makes both copies
 *     asynchronous (with pageable memory they behave as cudaMemcpyAsync
 *     does).  y_host holds the result once the stream has completed the
 *     call's work (cudaStreamSynchronize, or an event recorded after it).
 *   x_dev, y_dev: caller-owned device buffers of M*K and M*N elements of the
 *     activation dtype (x_dev as x of qmm_quantized_matmul_ws).
 *   Element size: 4 bytes for QMM_F32, 2 for QMM_BF16/QMM_F16 (the microscaled
 *     modes: the activation dtype given as `dtype`).
 * Errors: those of qmm_quantized_matmul_ws (argument errors are found
 * before anything is enqueued; when a call returns an error, the copy into
 * y_host has not been enqueued); a NULL host buffer with a nonzero size:
 * QMM_ERR_INVALID_ARG; a failed copy: QMM_ERR_CUDA.
 */
qmm_status qmm_quantized_matmul_host(const void *x_host, void *x_dev, int64_t M, int64_t K,
                                     const uint32_t *wq, const void *scales, const void *biases,
                                     qmm_dtype dtype, int64_t N, int transpose,
                                     int group_size, int bits, const char *mode,
                                     void *y_dev, void *y_host, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * qmm_mapped_pointer -- the address through which kernels on the current
 * device reach the page-locked host memory at `host` (cudaHostAlloc, or
 * cudaHostRegister'ed with mapping), or NULL when `host` is NULL, not
 * page-locked or not mapped.  One runtime query per call.
 *
 * qmm_quantized_matmul_mapped -- qmm_quantized_matmul_host for page-locked
 * buffers whose mappings the caller looked up once with qmm_mapped_pointer,
 * for the repeated per-step call of a serving loop: nothing is queried per
 * call, x is copied in by a kernel and the result reaches y_map as in
 * qmm_quantized_matmul_host.
 *   x_map, y_map: mappings returned by qmm_mapped_pointer for host buffers of
 *     M*K and M*N elements; the memory must stay page-locked (and mapped)
 *     while calls that use it are in flight.  NULL with a nonzero size:
 *     QMM_ERR_INVALID_ARG.
 *   Every other argument, the results and the errors: as
 *     qmm_quantized_matmul_host.
 */
void *qmm_mapped_pointer(const void *host);
qmm_status qmm_quantized_matmul_mapped(const void *x_map, void *x_dev, int64_t M, int64_t K,
                                       const uint32_t *wq, const void *scales, const void *biases,
                                       qmm_dtype dtype, int64_t N, int transpose, int group_size,
                                       int bits, const char *mode, void *y_dev, void *y_map,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * qmm_quantized_dense -- Emily.Quantization.Layers, quantized_dense: the
 * dense-layer form x @ W (+ bias) on a quantized weight, in either layout.
 * The page lets the bias be a tensor or a number; here both are taken and
 * added together:
 *   y[m, n] = round_to_dtype( sum_k x[m, k] W~[k, n] + bias[n] + bias_value )
 * with the product exactly as qmm_quantized_matmul computes it (same paths,
 * layouts, sizes and errors) and the bias added in fp32 in the product's
 * epilogue, before the single rounding of the output (no second pass over y).
 *   bias        NULL, or a device array of N values in `dtype` (one per output
 *               feature, broadcast over the rows of x), aligned to its element
 *               size;
 *   bias_value  a number added to every output (0 for none); must be finite.
 *   workspace, workspace_bytes  as for qmm_quantized_matmul_ws (may be NULL/0).
 * With bias == NULL and bias_value == 0 the result is qmm_quantized_matmul's.
 */
qmm_status qmm_quantized_dense(const void *x, int64_t M, int64_t K,
                               const uint32_t *wq, const void *scales, const void *biases,
                               qmm_dtype dtype, int64_t N, int transpose,
                               int group_size, int bits, const char *mode,
                               const void *bias, double bias_value,
                               void *y, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * qmm_qqmm -- mlx-rs ops/quantization.rs, qqmm: the product with BOTH operands
 * quantized, y = Q(x) @ Q(W)^T, in mode "nvfp4" (group_size 16, bits 4) or
 * "mxfp8" (32, 8).  The activations are quantized on the fly along K by the
 * same rule as a weight (see Mode above); the weight is already quantized:
 *   x [M, K] in `dtype`; wq [N, K*bits/32], w_scales [N, K/gs] uint8 (as
 *   qmm_quantize writes them in that mode); y [M, N] in `dtype`.
 * The call has no transpose argument: W is stored [N, K].  No per-tensor
 * global scales (the mlx-rs call passes none).  The product of the two
 * dequantized operands is formed in fp32 (every element value and scale is
 * exact in 16 bits, so the operands are exact).
 *   workspace: device memory of qmm_qqmm_workspace_size(M, K, group_size,
 *     bits, dtype) bytes, 256-byte aligned, for the quantized activations (its
 *     contents need not be initialised); two calls in flight must not share
 *     one.  Too small or misaligned: QMM_ERR_WORKSPACE.
 * Other modes: QMM_ERR_UNSUPPORTED.  Three kernels per call (quantize x,
 * dequantize x, product).
 */
size_t qmm_qqmm_workspace_size(int64_t M, int64_t K, int group_size, int bits, qmm_dtype dtype);
qmm_status qmm_qqmm(const void *x, int64_t M, int64_t K, qmm_dtype dtype,
                    const uint32_t *wq, const void *w_scales, int64_t N,
                    int group_size, int bits, const char *mode,
                    void *y, void *workspace, size_t workspace_bytes, void *stream);

/*
 * qmm_gather_qmm -- EMLX.Quantization, section gather_quantized_matmul;
 * mlx-rs gather_qmm.  Experts are stacked on the weight's leading axis:
 *   transpose != 0: wq [n_experts, N, K*bits/32], scales/biases [n_experts, N, K/gs]
 *   transpose == 0: wq [n_experts, K, N*bits/32], scales/biases [n_experts, K, N/gs]
 *   x [x_batch, M, K]; y [batch, M, N].
 * For b in [0, batch):
 *   y[b] = x[xi] @ W[ei]^T (or x[xi] @ W[ei] when transpose == 0), with
 *   xi = lhs_indices[b] if lhs_indices else (x_batch == 1 ? 0 : b),
 *   ei = rhs_indices[b] if rhs_indices else (n_experts == 1 ? 0 : b).
 * Without lhs_indices, x_batch must be 1 or batch; without rhs_indices,
 * n_experts must be 1 or batch.  Indices are int32 device arrays of length
 * `batch` (4-byte aligned); with batch == 0 the call does nothing and the
 * index pointers may be NULL.  No expert weight is copied.
 * sorted_indices: the caller's promise (EMLX.Quantization, section
 *   gather_quantized_matmul) that rhs_indices is non-decreasing.  The
 *   library checks the order itself on the device and skips its reorder
 *   whenever the keys are already sorted, so the hint is accepted but never
 *   trusted: a wrong hint cannot give wrong results.
 * Paths: bf16/f16 with transpose != 0 and K % 64 == 0 sort the rows by expert
 *   and run the grouped tensor-core product (three kernels: prepare, gather
 *   rows, product).  Other cases (f32, transpose == 0) run the SIMT kernels
 *   with one grid slice per batch entry.  qmm_set_path() forces either.
 * Out-of-range indices: the affected output rows are written as zeros and a
 *   later qmm_device_status() reports QMM_ERR_INDEX; nothing is read or
 *   written out of bounds.
 * workspace: device scratch of at least qmm_gather_qmm_workspace_size(...)
 *   bytes, 256-byte aligned, used by the tensor-core path only (the size is 0
 *   for f32); its contents need not be initialised and are not preserved.
 *   Two calls in flight at once must not share a workspace.  Too small or
 *   misaligned: QMM_ERR_WORKSPACE.
 * Errors: QMM_ERR_INVALID_ARG for sizes that do not broadcast or misaligned
 *   pointers, QMM_ERR_UNSUPPORTED for batch * M >= 2^30 rows.
 */
size_t qmm_gather_qmm_workspace_size(int64_t batch, int64_t M, int64_t K,
                                     int64_t n_experts, qmm_dtype dtype);

qmm_status qmm_gather_qmm(const void *x, int64_t x_batch, int64_t M, int64_t K,
                          const uint32_t *wq, const void *scales, const void *biases,
                          qmm_dtype dtype, int64_t n_experts, int64_t N,
                          const int32_t *lhs_indices, const int32_t *rhs_indices,
                          int64_t batch, int transpose, int group_size, int bits,
                          const char *mode, int sorted_indices,
                          void *y, void *workspace, size_t workspace_bytes,
                          void *stream);

/*
 * qmm_gather_qmm_static -- gather_qmm without a caller workspace.  Nothing in
 * the documents this library follows has a counterpart: it is a convenience
 * of this library for callers that cannot hand over device memory, such as a
 * plain C host that links no device allocator, or a step that must not
 * allocate (cudaMalloc can synchronise the device).  It allocates nothing:
 * the tensor-core path uses a fixed scratch array of
 * QMM_GATHER_STATIC_SCRATCH_BYTES built into the library (one per device).
 *
 * Arguments, layouts, results and errors are those of qmm_gather_qmm.  In
 * addition, a call that takes the tensor-core path (bf16/f16, transpose != 0,
 * K % 64 == 0, not forced onto the SIMT path by qmm_set_path) and whose
 * qmm_gather_qmm_workspace_size(batch, M, K, n_experts, dtype) exceeds
 * QMM_GATHER_STATIC_SCRATCH_BYTES returns QMM_ERR_WORKSPACE before launching
 * anything (use qmm_gather_qmm with a workspace for such sizes); calls on the
 * SIMT path use no scratch and have no such limit.  Example: x [512, 1, 4096]
 * bf16 needs about 4.2 MB.
 *
 * The scratch needs no initialisation (nothing in it must start at zero).
 * The first call on a device looks up the scratch's address, so make it
 * before any stream capture.  All calls on one device share the one scratch:
 * two calls whose work overlaps in time (on different streams, or from
 * different host threads) race on it and may return wrong results.  Calls
 * queued one after another on the same stream are safe.
 */
#define QMM_GATHER_STATIC_SCRATCH_BYTES (8u << 20)
qmm_status qmm_gather_qmm_static(const void *x, int64_t x_batch, int64_t M, int64_t K,
                                 const uint32_t *wq, const void *scales, const void *biases,
                                 qmm_dtype dtype, int64_t n_experts, int64_t N,
                                 const int32_t *lhs_indices, const int32_t *rhs_indices,
                                 int64_t batch, int transpose, int group_size, int bits,
                                 const char *mode, int sorted_indices, void *y, void *stream);

/*
 * qmm_device_status -- synchronise `stream`, then read (and, if `reset` is
 * non-zero, clear) the library's device-side error word, set by kernels whose
 * bounded waits time out (QMM_ERR_TIMEOUT) or that meet an out-of-range index
 * (QMM_ERR_INDEX).  Returns QMM_OK when the word is clear.
 */
qmm_status qmm_device_status(void *stream, int reset);

/*
 * qmm_set_wait_limit_ns -- limit of the bounded waits with which kernels
 * wait on another party (a tile part another CTA leaves, a ring stage another
 * warp fills), on the CURRENT device.  0 restores the default of 2 s.  When a
 * wait runs out, the kernel records QMM_ERR_TIMEOUT in the device error word,
 * carries on without the data (its results are then wrong but every access
 * stays in bounds), and still waits, with the fixed 2 s limit, for its own
 * copies and tensor-core work in flight before it exits.  For tests of the
 * failure path; synchronous with the host.
 */
qmm_status qmm_set_wait_limit_ns(uint64_t ns);

/*
 * qmm_inject_fault -- host-side fault injection for tests of the failure
 * path (process-wide; read when a kernel launch is prepared).
 *   QMM_FAULT_NONE                 no injection (the default);
 *   QMM_FAULT_STREAMK_NO_PUBLISH   in the stream-K split of the tensor-core
 *     product (qmm_quantized_matmul_ws with a workspace), the CTAs that leave
 *     a tile part write it but never raise its ready flag, so the tile's
 *     owner waits on a flag that nothing sets until the wait limit runs out
 *     (QMM_ERR_TIMEOUT).  Such a call leaves the workspace flags as they were
 *     and its output is wrong; zero the workspace before the next call.
 * Nothing is injected on the device: no kernel faults, traps or hangs.
 */
typedef enum { QMM_FAULT_NONE = 0, QMM_FAULT_STREAMK_NO_PUBLISH = 1 } qmm_fault;
qmm_status qmm_inject_fault(qmm_fault fault);

/*
 * Kernel-path selection for qmm_quantized_matmul (process-wide; the default
 * is QMM_PATH_AUTO: 1..4 rows of a W [N, K] product run on the streaming
 * decode kernel when it takes the codes -- affine 2/4/8 bits, mxfp4, nvfp4 --
 * and on the tensor-core GEMM otherwise (bf16/f16); more rows, and W [K, N],
 * on the GEMM).  QMM_PATH_GEMV forces the SIMT decode kernels (M <= 16
 * rows at a time), QMM_PATH_GEMM the tensor-core (tcgen05) GEMM, and
 * QMM_PATH_DECODE_TC the decode tensor-core kernel (bf16/f16, transpose,
 * 1..16 rows, 2- or 4-bit codes, group size 32..128, K % 512 == 0,
 * (K / group_size) % 8 == 0; two
 * launches per call: a prep kernel turns x into per-group block fixed point
 * (16-bit integers split into a signed and an unsigned byte, error below
 * 2^-15 of the group's largest |x|) in the workspace, then an integer MMA
 * product; it needs the workspace that qmm_quantized_matmul_workspace_size
 * reports under this path, else QMM_ERR_WORKSPACE; QMM_PATH_AUTO takes it
 * for 2-bit codes with 3..8 rows when the workspace is given, where it is
 * the fastest kernel).  A forced path that cannot run a given call returns
 * QMM_ERR_UNSUPPORTED.
 */
typedef enum {
    QMM_PATH_AUTO = 0,
    QMM_PATH_GEMV = 1,
    QMM_PATH_GEMM = 2,
    QMM_PATH_DECODE_TC = 3
} qmm_path;
qmm_status qmm_set_path(qmm_path path);

/*
 * Number of CUDA kernels this process has launched through libqmm so far
 * (all devices, all entry points).  For accounting in benchmarks and tests.
 */
uint64_t qmm_launch_count(void);

const char *qmm_status_string(qmm_status status);
const char *qmm_last_error(void);
int qmm_version(void); /* major*10000 + minor*100 + patch */

#ifdef __cplusplus
}
#endif

#endif /* QMM_H */
