// launchers.h -- host-side entry points of the individual kernels, called by
// the C ABI layer (dgrad_abi.cu) after it has validated the problem.  Each
// launcher only enqueues work on `stream`; none synchronises or allocates.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dgrad {

// Pointwise dgrad as a GEMM: dX[M][C] = dY[M][K] * W[K][C], all row-major.
struct PwArgs {
    int64_t M, K, C;
    const void* dY;
    const void* W;
    void* dX;
    int* status;  // device status word
    bool f16;     // 16-bit operands are f16 (split-K path; bf16 otherwise)
};

// fp32 in / fp32 out, fp32 FMA (no reduced-precision tensor-core path).
cudaError_t launch_pointwise_f32(const PwArgs& a, cudaStream_t stream);

// bf16 in / bf16 out on tcgen05 with TMEM accumulators.  map_a covers dY as a
// 2-D [M][K] bf16 tensor with a 64 x 128 box (K innermost) and map_b covers W as
// a 2-D [K][C] bf16 tensor with a 64 x 64 box (C innermost), both with the
// 128-byte swizzle.  bn is the tile width along C (64, 128 or 256).
cudaError_t launch_pointwise_tc(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                int bn, int num_sms, cudaStream_t stream);

// Resident-W tcgen05 variant: each CTA keeps its 128-column slice of W in
// shared memory (needs K <= 512 and ceil(C/128) <= num_sms/2) and writes dX
// through map_d, a 2-D [M][C] bf16 map with a 64 x 128 box and the 128-byte
// swizzle.  map_b must have a 64 x 64 box as above.
bool pointwise_tc_resident_ok(const PwArgs& a, int num_sms);
cudaError_t launch_pointwise_tc_resident(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                         const CUtensorMap& map_d, int num_sms, cudaStream_t stream);

// SM-pair tcgen05 variant (cta_group::2, clusters of two CTAs): 256 x bn tiles
// (bn = 256 or 128), each CTA holding 128 dY rows and bn/2 W columns per
// k-block.  Maps as for the resident variant.
cudaError_t launch_pointwise_tc_pair(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                     const CUtensorMap& map_d, int bn, int num_sms, cudaStream_t stream);

// Split-K tcgen05 variant for small M: partial tiles go to ws (fp32,
// [splits][M][C]), then a reduction kernel sums them in split order and writes
// bf16 dX.  pointwise_splitk_auto picks a split count that fills the SMs.
int pointwise_splitk_auto(const PwArgs& a, int num_sms);
size_t pointwise_splitk_workspace_bytes(const PwArgs& a, int splits);
cudaError_t launch_pointwise_tc_splitk(const PwArgs& a, const CUtensorMap& map_a, const CUtensorMap& map_b,
                                       int splits, float* ws, int num_sms, cudaStream_t stream);

// Dense or grouped KH x KW dgrad on tcgen05, by output phase (S*S sub-GEMMs),
// bf16 or f16 (f16 = true).  G groups of Kg dY and Cg dX channels; W is
// [KH][KW][K][Cg].  map_a covers dY as a 5-D tensor (Kg, G, Wo, Ho, N) with a
// 64 x 1 x 16 x 8 x 1 box and the 128-byte swizzle; map_b covers W as a 4-D
// tensor (Cg, Kg, G, KH*KW) with a 64 x 64 x 1 x 1 box and the 128-byte swizzle.
// plan_dense fills the phase-grid fields (hq_min, wq_min, nth, ntw) from the
// geometry; bn is the channel tile (64, 128 or 256).
struct DenseArgs {
    void* dX;
    int* status;
    int N, H, W, C, K, Ho, Wo, KH, KW, S, ph, pw;
    int G, Kg, Cg;
    bool f16;
    int hq_min, wq_min, nth, ntw, nc, num_tiles;
};
void plan_dense(DenseArgs* d);
cudaError_t launch_dense_tc(const DenseArgs& d, const CUtensorMap& map_a, const CUtensorMap& map_b, int bn,
                            int num_sms, cudaStream_t stream);

// Keep a CUDA error code for dgrad_last_cuda_error (entry points defined
// outside the ABI file report their failures through this).
void record_cuda_error(cudaError_t e);

// Depthwise problem (groups = C = K), NHWC, dense.
struct DwArgs {
    int N, H, W, C, Ho, Wo, KH, KW, S, ph, pw;
    bool bf16;  // element type of dY, W and dX: bf16 (true), or f32 / f16 (false)
    bool f16;   // element type f16 (bf16 is false then)
    int elem_kind() const { return f16 ? 2 : bf16 ? 1 : 0; }   // ElemKind of the device code
    const void* dY;
    const void* filt;  // W[KH][KW][C]
    void* dX;
    int* status;
};

// Stride-1 rotated-filter correlation.  Requires S == 1, KH, KW <= 64.
cudaError_t launch_dw_rotated(const DwArgs& a, cudaStream_t stream);

// Stride-1 depthwise for small filters (3x3, 5x5, 7x7; bf16 or f16): one TMA halo
// tile per CTA.  dy_map covers dY as a 4-D 16-bit tensor (C, Wo, Ho, N innermost first)
// with the box dw_tile_box returns; dx_map (or null) covers dX the same way (C, W, H, N)
// with box_dx, and the kernel then stores each output tile through it.
// cudaErrorNotSupported when not compiled.
bool dw_tile_box(const DwArgs& a, unsigned box[4], unsigned box_dx[4]);
cudaError_t launch_dw_tile(const DwArgs& a, const CUtensorMap& dy_map, const CUtensorMap* dx_map, cudaStream_t stream);

// Stride-1 depthwise on the tcgen05 tensor cores (bf16): each channel plane as
// a sum of banded-Toeplitz GEMMs, one per filter line.  plan_dw_toeplitz picks
// the plane orientation and tile and returns false when the problem does not
// fit; the launch needs a workspace of ws_in + ws_out + ws_f bytes (planar dY,
// planar dX, packed filter lines and the split partials) and map_b, a 4-D bf16 map of the planar dY
// [C][Yi][N][Xsi] with dims (Xi, N, Yi, C), box (64, 8, b_rows, 1), 128-byte
// swizzle, zero fill.
struct ToepPlan {
    int orient, KY, KX, py, px, Yi, Xi, Xsi, Yo, Xo, Xso;
    int P, TW, XT, NH, Ks, NR, NI, NB, nfb, npanels, half_l, f_words, a_col0, a_cols, na;
    int clip;   // one tile spans the row: K clipped to the input columns inside the image
    int a_smem, a_slots, nacc;   // A_i as shared-memory tables of a_slots core matrices; accumulator sets
    uint32_t a_off, a_bytes;     // offset of the first A table and the stride between them
    int tma_epi;          // the MMA epilogue stores staged boxes by TMA (needs ToepMaps::d_store)
    uint32_t stg_off;     // its staging boxes in shared memory
    int nstg;             // staging boxes per epilogue half (1 or 2)
    uint32_t panel_bytes, b_bytes, f_off, bar_off;
    // B blocks b_stride bytes apart; the TMA box brings b_rows rows starting b_zt rows into a
    // block (b_rows = NR, b_zt = 0 unless the blocks share their zero rows, which the kernel
    // writes once at z_off / z_len)
    int b_zt, b_rows;
    uint32_t b_stride, z_off[3], z_len[3];
    // split: CTAs take equal ranges of shift steps; part_slots fp32 partial tiles at part_off
    // and as many flags at flag_off, both offsets into the ws_f region
    int split, part_slots;
    size_t part_off, flag_off;
    size_t smem, ws_in, ws_out, ws_f;
};
// Tensor maps of one call: b as above; for the transposes (when tma_transpose),
// the NHWC maps of dY and dX (dims C, W, H, N; box 64 channels by 64 positions
// along the plane's x axis: W in orientation 0, H in orientation 1) and the
// planar maps of the workspace planes (dims X, N, Y, C; box 64 x by 64 c), all
// with the 128-byte swizzle.  Without them the transposes run on CUDA cores.
struct ToepMaps {
    CUtensorMap b;
    CUtensorMap pack_src, pack_dst, unpack_src, unpack_dst;
    bool tma_transpose;
    // the planar dX [C][Yo][N][Xso] (dims Xo, N, Yo, C), box (64, 8, 8, 1), no swizzle:
    // the MMA epilogue's stores when the plan has tma_epi
    CUtensorMap d_store;
    bool tma_epi;
};
bool plan_dw_toeplitz(const DwArgs& a, ToepPlan* p, bool nhwc = false);
// The same formulation reading NHWC dY and writing NHWC dX directly, with clusters
// of 8 CTAs (8 channels) and no workspace; p from plan_dw_toeplitz(a, &p, true).
cudaError_t launch_dw_toeplitz_nhwc(const DwArgs& a, const ToepPlan& p, cudaStream_t stream);
cudaError_t launch_dw_toeplitz(const DwArgs& a, const ToepPlan& p, const ToepMaps& maps, void* ws, int num_sms,
                               cudaStream_t stream);

// Row-streaming kernel with a circular shared-memory accumulator ring (any S <= 8).
cudaError_t launch_dw_rowstream(const DwArgs& a, cudaStream_t stream);

// Register-blocked row-streaming kernel for the compiled (KH, KW, S) set, bf16
// or f16.  dy_map covers dY as a 4-D 16-bit tensor (C, Wo, Ho, N innermost first)
// with no swizzle; dx_map and dx_map8 (or null) cover dX the same way (C, W, H, N),
// with boxes of one row and of rows_dx8 rows, and the register-ring kernel then
// stores its final rows through them.  Returns cudaErrorNotSupported when no
// instantiation fits.
cudaError_t launch_dw_rowstream_fast(const DwArgs& a, const CUtensorMap& dy_map, const CUtensorMap* dx_map,
                                     const CUtensorMap* dx_map8, int G, cudaStream_t stream);

// Boxes (inner first) the fast row-streaming kernel loads from dY and stores into
// dX (box_dx one row high; rows_dx8 the rows of the taller box), or false when the
// problem has no fast instantiation.
bool dw_rowstream_fast_box(const DwArgs& a, unsigned box[4], unsigned box_dx[4], unsigned* rows_dx8);

// Number of SMs of the current device (cached per device).
int device_sm_count();

}  // namespace dgrad
