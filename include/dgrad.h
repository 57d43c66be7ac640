/*
 * dgrad.h -- C ABI of libdgrad, a B200 (sm_100a) engine for convolution
 * backward-data ("dgrad"): dX = dgrad(dY, W) on NHWC activations.
 *
 * Operation.  For a forward convolution with dilation 1, stride S, per-axis
 * padding (pad_h, pad_w) and output extents
 *     Ho = floor((H + 2*pad_h - KH) / S) + 1,   Wo = floor((W + 2*pad_w - KW) / S) + 1
 * ("channel-packed and large-filter depthwise dgrad", Technical Details,
 * per-axis padding: Wo uses PAD_W), dgrad is the adjoint of the forward map in
 * its input:
 *     dX[n,h,w,c] = sum over (ho,wo,k,r,s) with h = ho*S - pad_h + r and
 *                   w = wo*S - pad_w + s of dY[n,ho,wo,k] * Wt(k,r,s,c).
 * Two shape classes are served:
 *   - pointwise: 1x1 filter, stride 1, no padding, one group.  dX[M,C] =
 *     dY[M,K] . W[K,C] with M = N*H*W, dY offset m*K + k, W offset k*C + c and
 *     dX offset m*C + c ("add the pointwise fast path dgrad was missing",
 *     Technical Details and the fast-path commit message);
 *   - depthwise: groups = C = K (depth multiplier 1), W[KH][KW][C].  Stride 1
 *     runs as a correlation of dY with the 180-degree rotated filter at padding
 *     KH-1-pad_h rows and KW-1-pad_w columns, filters up to 64 a side, square or
 *     not; stride > 1 runs as a row-streaming kernel whose accumulator rows sit
 *     in circular slots (registers, or a shared-memory ring) ("channel-packed and large-filter
 *     depthwise dgrad", Technical Details: rotated-filter dgrad and the
 *     channel-packed row-streaming dgrad).
 *
 * Layouts (all dense, channels innermost, no padding between rows):
 *     dY  [N][Ho][Wo][K]      dX [N][H][W][C]
 *     W   pointwise [K][C];   depthwise [KH][KW][C]
 * Element type: DGRAD_F32 (float in, float out), DGRAD_BF16 (bf16 in, bf16 out)
 * or DGRAD_F16 (f16 in, f16 out).  Accumulation is always fp32; a 16-bit dX is
 * rounded once, to nearest even.
 *
 * Memory and streams.  Every pointer is device memory the caller owns (for
 * example a PyTorch CUDA tensor's data pointer) on the current device.  Calls
 * enqueue work on `stream` (a cudaStream_t; NULL is the legacy default stream)
 * and return without synchronising; the library allocates no device memory per
 * call.  dX is written in full (never accumulated into), so it needs no zeroing.
 * Alignment: every base pointer 16-byte aligned, and K and C multiples of 8
 * (bf16, f16) or 4 (f32), so that every channel row starts on 16 bytes.
 *
 * Errors.  Arguments are validated on the host before anything is launched; a
 * rejected call launches nothing and leaves dX untouched.  A launch failure is
 * reported as DGRAD_ERR_CUDA (the CUDA error is kept for dgrad_last_cuda_error).
 * Kernels never trap: a device-side wait that runs past its limit sets a status
 * word and the kernel returns; dgrad_check_status reports it.
 */
#ifndef DGRAD_H
#define DGRAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Problem geometry (the pages' DirectConvProblem: extents, filter, stride and
 * per-axis padding; "channel-packed and large-filter depthwise dgrad",
 * Technical Details, per-axis padding).  H, W are dX's spatial extents; C is
 * dX's channel count and K dY's.  Dilation is 1.  pad_w == -1 means "same as
 * pad_h" (the pages' sentinel); any other negative value is invalid. */
typedef struct {
    int64_t N, H, W, C, K;
    int32_t KH, KW, stride;
    int32_t pad_h, pad_w;
} dgrad_problem_t;

/* Element type of dY, W and dX (one type for all three).  DGRAD_F16 is served by
 * every entry point: dgrad_pointwise, its split-K variants, dgrad_dense,
 * dgrad_grouped and dgrad_depthwise_tc run tcgen05 MMAs on f16 operands with
 * fp32 accumulation; dgrad_depthwise widens f16 to fp32 on load and uses fp32
 * FMAs.  DGRAD_F32 is served by dgrad_pointwise and dgrad_depthwise only. */
typedef enum { DGRAD_F32 = 0, DGRAD_BF16 = 1, DGRAD_F16 = 2 } dgrad_dtype_t;

/* Depthwise kernel choice.  AUTO: rotated-filter for stride 1, row-streaming
 * otherwise.  ROTATED requires stride 1.  ROWSTREAM serves any stride (at
 * stride 1 it is a cross-check of the rotated-filter kernel). */
typedef enum { DGRAD_DW_AUTO = 0, DGRAD_DW_ROTATED = 1, DGRAD_DW_ROWSTREAM = 2 } dgrad_dw_mode_t;

typedef enum {
    DGRAD_OK = 0,
    DGRAD_ERR_INVALID = 1,      /* null pointer, non-positive extent, pad_w < -1, Ho or Wo < 1 ... */
    DGRAD_ERR_UNSUPPORTED = 2,  /* valid geometry this entry point does not serve */
    DGRAD_ERR_ALIGNMENT = 3,    /* base pointer or channel row not 16-byte aligned */
    DGRAD_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
    DGRAD_ERR_TIMEOUT = 5,      /* a kernel gave up waiting (reported by dgrad_check_status) */
    DGRAD_ERR_BOUNDS = 6        /* libdgrad_debug.so only: a store index check failed (dgrad_check_status) */
} dgrad_status_t;

/* Pointwise dgrad, dX[M,C] = dY[M,K] . W[K,C] with M = N*H*W.
 * Requires KH = KW = 1, stride 1, pad_h = pad_w = 0 (else DGRAD_ERR_UNSUPPORTED;
 * the pointwise page's shape class).  DGRAD_BF16 runs on the tcgen05 tensor
 * cores (TMA-fed shared-memory tiles, fp32 accumulators in tensor memory);
 * DGRAD_F16 runs on them through the tap kernel of dgrad_grouped (one 1x1 tap);
 * DGRAD_F32 runs as an fp32 FMA kernel (no reduced-precision inputs). */
dgrad_status_t dgrad_pointwise(const dgrad_problem_t* prob, dgrad_dtype_t dtype,
                               const void* dY, const void* W, void* dX, void* stream);

/* Split-K pointwise dgrad for problems with few output tiles (small M = N*H*W,
 * long K): each 128 x 128 tile's K-loop is split into `splits` ranges that run
 * on different SMs; partial tiles are written as fp32 to `workspace` and then
 * summed in split order (deterministic: no atomics, nothing to zero) and
 * rounded once to bf16 (or f16) into dX.  Same shape class and layouts as
 * dgrad_pointwise; DGRAD_BF16 or DGRAD_F16 (else DGRAD_ERR_UNSUPPORTED).  The pages'
 * implicit-GEMM dgrad has a split-K mode ("add the pointwise fast path dgrad
 * was missing", review-fix commit: split-K sub-GEMMs, dX accumulated
 * atomically).
 * splits: 1 .. 64, or 0 to let the library choose one that fills the GPU.
 * workspace: caller-owned device memory, 16-byte aligned, at least the size
 * dgrad_pointwise_splitk_workspace reports for the same problem and splits;
 * its contents on entry do not matter and are clobbered.  Too small or null:
 * DGRAD_ERR_INVALID. */
dgrad_status_t dgrad_pointwise_splitk(const dgrad_problem_t* prob, dgrad_dtype_t dtype, int splits,
                                      const void* dY, const void* W, void* dX,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes dgrad_pointwise_splitk needs for `splits` (0: the automatic
 * choice, which is returned in *splits_used when that pointer is non-null).
 * Queries the current device's SM count for the automatic choice. */
dgrad_status_t dgrad_pointwise_splitk_workspace(const dgrad_problem_t* prob, int splits, size_t* bytes,
                                                int* splits_used);

/* ---- A variant for callers that cannot allocate (no counterpart on the
 * pages: their kernels take whatever workspace their host framework gives). ---- */

/* Size of the fixed split-K scratch buffer built into the library: 8 MiB, one
 * buffer per device. */
#define DGRAD_SPLITK_SCRATCH_BYTES ((size_t)8 << 20)

/* dgrad_pointwise_splitk with no workspace argument: the fp32 partial tiles go
 * to a fixed buffer of DGRAD_SPLITK_SCRATCH_BYTES that is part of the
 * library's device image (CUDA reserves it when it loads the library's code on
 * a device), so the call allocates nothing: no cudaMalloc, no framework
 * allocator.  It serves callers that have no workspace to pass and must not
 * allocate at call time, for example a plugin or callback running inside a
 * framework that owns all device memory, or code that runs while a caching
 * allocator is reclaiming memory and so cannot call back into it.
 * Same shape class, dtype, layouts, kernels and results as
 * dgrad_pointwise_splitk with the same split count.
 * splits: 1 .. 64, or 0 for the automatic count, lowered as far as needed for
 * the partial tiles to fit the buffer.  When the partial tiles still need more
 * than DGRAD_SPLITK_SCRATCH_BYTES (splits * M * C * 4 bytes, M = N*H*W; with
 * splits 0, even one split's M * C * 4), the call returns
 * DGRAD_ERR_UNSUPPORTED and launches nothing.
 * Nothing in the buffer has to start at zero and nothing clears it: each split
 * writes its whole partial tile before the reduction reads it.
 * Set-up: the first call on each device (with that device current) looks up
 * the buffer's device address and keeps it for the life of the process; make
 * that first call before any stream capture begins.  The kept address belongs
 * to the device's primary context: resetting the device (cudaDeviceReset) or
 * calling from another context is not supported.
 * Races: there is ONE buffer per device.  Calls whose work may overlap on the
 * same device (issued to different streams, or from several host threads
 * without ordering between their streams) write the same buffer and corrupt
 * each other's results.  Calls ordered on one stream are safe. */
dgrad_status_t dgrad_pointwise_splitk_noalloc(const dgrad_problem_t* prob, dgrad_dtype_t dtype, int splits,
                                              const void* dY, const void* W, void* dX, void* stream);

/* Grouped dgrad: `groups` groups, each of K/groups dY and C/groups dX channels,
 * any KH x KW filter and stride, on the tcgen05 tensor cores; W is
 * [KH][KW][K][C/groups] (tap-major; each tap holds, for every dY channel k, the
 * C/groups filter values of k's group).  A 1x1 filter is the pages' grouped
 * pointwise dgrad (per-group output channel base and a C/groups W stride; "add
 * the pointwise fast path dgrad was missing", Technical Details).  Each group
 * runs as its own set of phase GEMMs, as in dgrad_dense.  groups must divide K
 * and C (else DGRAD_ERR_INVALID); K/groups and C/groups multiples of 8 (else
 * DGRAD_ERR_ALIGNMENT); DGRAD_BF16 or DGRAD_F16; other limits as dgrad_dense. */
dgrad_status_t dgrad_grouped(const dgrad_problem_t* prob, int64_t groups, dgrad_dtype_t dtype, const void* dY,
                             const void* W, void* dX, void* stream);

/* Dense (ungrouped, groups = 1) dgrad with a KH x KW filter and any stride, on
 * the tcgen05 tensor cores; W is [KH][KW][K][C] (tap-major: each tap is a
 * pointwise [K][C] matrix).  The pages' main dgrad engine decomposes a strided
 * dgrad by output phase into stride*stride sub-GEMMs ("add the pointwise fast
 * path dgrad was missing", Technical Details); here each phase's GEMM sums, over
 * the phase's taps, products of a shifted window of dY (K deep) with that tap's
 * [K][C] matrix, so no im2col buffer is built.  DGRAD_BF16 or DGRAD_F16 (else
 * DGRAD_ERR_UNSUPPORTED); KH, KW, stride <= 64; K and C multiples of 8; padding
 * any value >= 0 that leaves Ho, Wo >= 1. */
dgrad_status_t dgrad_dense(const dgrad_problem_t* prob, dgrad_dtype_t dtype, const void* dY, const void* W, void* dX,
                           void* stream);

/* Depthwise dgrad (groups = C; requires K == C, else DGRAD_ERR_UNSUPPORTED).
 * Rotated-filter mode requires stride 1, KH and KW <= 64 and
 * 0 <= pad_h <= KH-1, 0 <= pad_w <= KW-1 (the rotated padding KH-1-pad_h and
 * KW-1-pad_w is then non-negative).  Row-streaming requires KH, KW <= 64,
 * stride <= 8, 0 <= pad_h <= KH-1 and 0 <= pad_w <= KW-1.  Any element type:
 * 16-bit inputs are widened to fp32 on load and dX is rounded once. */
dgrad_status_t dgrad_depthwise(const dgrad_problem_t* prob, dgrad_dtype_t dtype,
                               dgrad_dw_mode_t mode,
                               const void* dY, const void* W, void* dX, void* stream);

/* Stride-1 depthwise dgrad on the tensor cores, for large filters.  Each
 * channel's plane is a sum of GEMMs, one per filter line along the shorter
 * filter side, whose other operand is the banded (Toeplitz) matrix of that
 * filter line along the longer side: the implicit-GEMM formulation of the
 * rotated-filter correlation ("channel-packed and large-filter depthwise
 * dgrad", Technical Details: rotated-filter dgrad; the pages sent large filters
 * through an implicit-GEMM path before the FP32 rotated-filter kernel).  The
 * MMAs run in bf16 (or f16) with fp32 accumulation (tcgen05), so results equal
 * those of dgrad_depthwise up to fp32 summation order.
 * Requirements: DGRAD_BF16 or DGRAD_F16, stride 1, K == C, KH and KW <= 64,
 * 0 <= pad_h <= KH-1, 0 <= pad_w <= KW-1, N, H, W <= 65535; else
 * DGRAD_ERR_UNSUPPORTED (also when the filter is too large for the tile plan).
 * workspace: caller-owned device memory, 16-byte aligned, at least the size
 * dgrad_depthwise_tc_workspace reports; it holds dY and dX as per-channel planes
 * (channel-outermost copies of both); its contents on entry do not matter.
 * Three kernels run in order on `stream`: dY to planes, the tensor-core kernel,
 * planes to dX. */
dgrad_status_t dgrad_depthwise_tc(const dgrad_problem_t* prob, dgrad_dtype_t dtype, const void* dY, const void* W,
                                  void* dX, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes dgrad_depthwise_tc needs (0 for an empty batch); returns the
 * same refusals as dgrad_depthwise_tc for the problem (host only). */
dgrad_status_t dgrad_depthwise_tc_workspace(const dgrad_problem_t* prob, size_t* bytes);

/* Output extents of the forward convolution the problem describes (host only,
 * no CUDA call).  Returns DGRAD_ERR_INVALID for an invalid problem. */
dgrad_status_t dgrad_out_dims(const dgrad_problem_t* prob, int64_t* Ho, int64_t* Wo);

/* Synchronise `stream`, then report (and clear) the device status word of the
 * current device: DGRAD_ERR_TIMEOUT if any kernel gave up waiting since the
 * last check, DGRAD_ERR_BOUNDS if (in the debug build, libdgrad_debug.so, built
 * from the same sources with -DDGRAD_DEBUG) a hand-indexed store fell outside
 * its output buffer and was skipped, DGRAD_ERR_CUDA if the stream reported an
 * error, else DGRAD_OK. */
dgrad_status_t dgrad_check_status(void* stream);

/* Static, human-readable text for a status code. */
const char* dgrad_status_string(dgrad_status_t status);

/* The last CUDA error code the library saw on this thread (0 if none). */
int dgrad_last_cuda_error(void);

/* ---- Diagnostics (no counterpart on the pages; they support testing and
 * measurement of the entry points above). ---- */

/* Enqueue one small kernel whose bounded wait is made to run out: it waits on a
 * barrier nothing completes for `limit_cycles` SM cycles (0 .. 2e9), then
 * records a timeout in the status word exactly as the dgrad kernels do and
 * returns.  dgrad_check_status then reports DGRAD_ERR_TIMEOUT and clears it.
 * Used to test the failure path without faulting or hanging the GPU. */
dgrad_status_t dgrad_selftest_timeout(long long limit_cycles, void* stream);

/* Enqueue an fp32 FMA-rate probe: `blocks` CTAs of 256 threads, each thread
 * running `iters` rounds of 16 independent FMAs (packed != 0: as 8 fma.rn.f32x2).
 * Work = blocks * 256 * iters * 16 FMAs.  `sink` is a device buffer of at least
 * `blocks` floats that keeps the work live (normally left untouched). */
dgrad_status_t dgrad_fma_probe(int blocks, int iters, int packed, float* sink, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DGRAD_H */
