// dw_toeplitz_nhwc.cu -- stride-1 depthwise dgrad on the tcgen05 tensor cores,
// reading NHWC dY and writing NHWC dX directly (no planar copies, no workspace).
//
// The arithmetic is the banded-Toeplitz formulation of the rotated-filter
// correlation ("channel-packed and large-filter depthwise dgrad", Technical
// Details: rotated-filter dgrad; the implicit-GEMM form large filters took on
// the pages before the FP32 kernel): for one channel, 8 images, 2*NH output rows
// and 64 output columns, D[(p, xl)][(h', img)] = sum_i A_i * B_i with A_i the
// Toeplitz band of filter line i - p (built in tensor memory) and B_i the input
// rows P*h' + i - py (a shared-memory block seen through a descriptor that moves
// one 1024-byte swizzle atom per shift step).  toeplitz_core.cuh holds the A
// builder and the MMA sequence of a step.
//
// What is new here is where B comes from and where D goes.
//   * Channels are interleaved in NHWC: one 16-byte chunk holds 8 channels of a
//     position.  A cluster of 8 CTAs works on 8 consecutive channels (CTA rank k
//     on channel 8*cb + k) of the same tile.  Each CTA loads its share of the
//     tile's input window as whole chunks (8 positions along x at a time),
//     transposes each 8 x 8 block of 16-bit values in registers, and stores row
//     k -- channel k's 8 consecutive columns -- straight into CTA k's B block
//     (shared memory of the cluster, 128-byte swizzled layout).  Every dY byte
//     is read once from memory and used.
//   * The accumulator of CTA k holds channel k only.  Its epilogue writes dX in
//     a permuted order: for each group of 8 output columns, the chunk at column
//     8*xg + k receives channel k's 8 values.  Once all 8 CTAs have written a
//     tile, each transposes its share of the tile's 8 x 8 blocks in place,
//     which leaves the final NHWC layout.  dX is written twice, both times into
//     L2, and reaches memory once.  A ragged last column group (width not a
//     multiple of 8) is written in the final layout directly.
//
// Roles (448 threads, one CTA per SM, clusters of 8):
//   warp 0      packs the filter lines of the CTA's channel (two buffers)
//   warp 1      TMEM allocation (512 columns) and the MMA issuer (one lane)
//   warps 2-5   A builders: each thread writes its row of A_i with tcgen05.st
//   warps 6-13  epilogue and data movement: drain the accumulator, fill the next
//               B blocks of the cluster, write and then transpose dX
// Every wait is bounded; a timeout is recorded in the status word, raises the
// CTA's abort flag and lets the CTA wind down.  No role leaves before the final
// cluster barrier, so no CTA exits while a peer may still write to it.
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "host_util.h"
#include "launchers.h"
#include "toeplitz_core.cuh"

namespace dgrad {
namespace {
using namespace toep;

constexpr int kThreadsN = 448;
constexpr int kCluster = 8;           // CTAs per cluster = channels per 16-byte chunk
constexpr uint32_t kTmemColsN = 512;
constexpr int kMaxAN = 4;             // A buffers in tensor memory
constexpr int kEcThreads = 256;       // epilogue / data-movement threads (warps 6-13)
constexpr int kEcWarp0 = 6;
constexpr int kNumBarsN = kNumBarsNhwc;
static_assert(kNumBarsN == 2 * kMaxAN + 10, "barrier count of the NHWC kernel");
constexpr int kBarEc = 1;             // named barrier id of the epilogue warps

struct ToepNArgs {
    const uint16_t* dY;       // NHWC dY (16-bit patterns)
    const uint16_t* filt;     // W[KH][KW][C]
    uint16_t* dX;             // NHWC dX
    int* status;
    int N, C, KH, KW, orient;
    int KY, KX, py, px;
    int Yi, Xi, Yo, Xo;        // plane extents of dY (input) and dX (output)
    long long sNi, sYi, sXi;   // dY element strides of (image, plane y, plane x)
    long long sNo, sYo, sXo;   // dX element strides
    int P, TW, XT, NH, Ks, NR, NI, half_l, npanels;
    int num_xt, num_yt, num_g, num_su;
    int a_col0, a_cols, na;
    int f16, full_plane;
    int clip;                  // one tile spans the row: the window starts at input column 0
    int nfb;                   // filter-line buffers: 2, or 1 when two do not fit
    uint32_t panel_bytes, b_bytes, f_words, f_off, bar_off;
    long long dx_bytes;        // size of dX (index checks of the debug build)
};

struct Tile {
    int cb, g, Y0, x0, xb;
};

__device__ __forceinline__ Tile decode_tile(const ToepNArgs& a, int su)
{
    Tile t;
    const int xt = su % a.num_xt;
    int r = su / a.num_xt;
    const int yt = r % a.num_yt;
    r /= a.num_yt;
    t.g = r % a.num_g;
    t.cb = r / a.num_g;
    t.Y0 = yt * a.P * a.NH;
    t.x0 = xt * a.XT * a.TW;
    t.xb = a.clip ? 0 : floor8(t.x0 - a.px);
    return t;
}

// Super-units [*b, *e) of this cluster: a contiguous range, so that the tiles of
// one channel block follow each other and clusters running at the same time work
// on neighbouring channel blocks (whose chunks share memory sectors).
__device__ __forceinline__ void cluster_range(const ToepNArgs& a, int* b, int* e)
{
    const int ncl = static_cast<int>(gridDim.x) / kCluster;
    const int cl = static_cast<int>(blockIdx.x) / kCluster;
    *b = static_cast<int>((static_cast<long long>(cl) * a.num_su) / ncl);
    *e = static_cast<int>((static_cast<long long>(cl + 1) * a.num_su) / ncl);
}

__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_nc_v4(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// The part of a tile's input window that has to be written into the B blocks:
// rows r (input row Y0 - py + r), images and 8-column groups xg (input columns
// xb + 8*xg .. + 7).  With one tile per plane the parts of the window outside
// the image are zeroed once at start and never written again; otherwise every
// position is written (zero outside the image).
struct Win {
    int r_lo, r_hi, nimg, xg_lo, xg_hi;
};

__device__ __forceinline__ Win window_of(const ToepNArgs& a, const Tile& t)
{
    Win w;
    const int nxg = 8 * a.npanels;
    if (a.full_plane) {
        w.r_lo = max(0, a.py - t.Y0);
        w.r_hi = min(a.NR, a.py - t.Y0 + a.Yi);
        w.nimg = min(8, a.N - 8 * t.g);
        w.xg_lo = max(0, -t.xb / 8);
        w.xg_hi = min(nxg, (a.Xi - t.xb + 7) / 8);
    } else {
        w.r_lo = 0;
        w.r_hi = a.NR;
        w.nimg = 8;
        w.xg_lo = 0;
        w.xg_hi = nxg;
    }
    if (w.r_hi < w.r_lo) w.r_hi = w.r_lo;
    if (w.xg_hi < w.xg_lo) w.xg_hi = w.xg_lo;
    return w;
}

// Element offset in dY of channel block cb at (image, plane row y, plane column x).
__device__ __forceinline__ long long in_off(const ToepNArgs& a, int img, int y, int x, int cb)
{
    return img * a.sNi + y * a.sYi + x * a.sXi + 8LL * cb;
}

__device__ __forceinline__ long long out_off(const ToepNArgs& a, int img, int y, int x, int cb)
{
    return img * a.sNo + y * a.sYo + x * a.sXo + 8LL * cb;
}

// Item i of the window: (r, img, xg) and whether its row and image lie in the input.
__device__ __forceinline__ void win_item(const ToepNArgs& a, const Tile& t, const Win& w, int i, int* r, int* img,
                                         int* xg, int* yin, bool* row_ok)
{
    const int nxg = w.xg_hi - w.xg_lo;
    *xg = w.xg_lo + i % nxg;
    const int q = i / nxg;
    *img = q % w.nimg;
    *r = w.r_lo + q / w.nimg;
    *yin = t.Y0 - a.py + *r;
    *row_ok = *yin >= 0 && *yin < a.Yi && 8 * t.g + *img < a.N;
}

// Write this thread's share of a tile's window into the B blocks of the 8 CTAs
// of the cluster.  b_local is this CTA's shared-memory address of its B block;
// every CTA has its block at the same address.
__device__ void fill_window(const ToepNArgs& a, const Tile& t, int rank, int e, uint32_t b_local)
{
    const Win w = window_of(a, t);
    const int n = (w.r_hi - w.r_lo) * w.nimg * (w.xg_hi - w.xg_lo);
    for (int i = rank * kEcThreads + e; i < n; i += kCluster * kEcThreads) {
        int r, img, xg, y;
        bool ok;
        win_item(a, t, w, i, &r, &img, &xg, &y, &ok);
        const int x = t.xb + 8 * xg;
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            v[u] = (ok && x + u >= 0 && x + u < a.Xi) ? ld_nc_v4(a.dY + in_off(a, 8 * t.g + img, y, x + u, t.cb))
                                                      : make_uint4(0, 0, 0, 0);
        const int R = r * 8 + img;
        const uint32_t off = static_cast<uint32_t>(xg >> 3) * a.panel_bytes + static_cast<uint32_t>(R) * 128u +
                             (static_cast<uint32_t>((xg & 7) ^ (R & 7)) << 4);
        // channel k of the 8 columns, stored to CTA k as soon as it is formed
#pragma unroll
        if (!store_ok(nullptr, a.b_bytes, reinterpret_cast<const void*>(static_cast<uintptr_t>(off)), 16, a.status))
            continue;   // debug build: outside the B block (recorded)
        for (int k = 0; k < kCluster; ++k)
            st_cluster_v4(mapa_shared(b_local + off, static_cast<uint32_t>(k)), transpose8x8_col(v, k));
    }
}

// Transpose this thread's share of a finished tile's complete 8-column groups
// from the permuted order the epilogues wrote (chunk 8*xg + k holds channel k's
// columns 8*xg .. 8*xg + 7) to NHWC.
__device__ void transpose_tile_out(const ToepNArgs& a, const Tile& t, int rank, int e)
{
    const int nimg = min(8, a.N - 8 * t.g);
    const int y_hi = min(t.Y0 + a.P * a.NH, a.Yo);
    const int x_hi = min(t.x0 + a.XT * a.TW, a.Xo);
    const int g_lo = t.x0 / 8;
    const int ng = x_hi / 8 - g_lo;
    const int nrow = y_hi - t.Y0;
    if (ng <= 0 || nrow <= 0 || nimg <= 0) return;
    const int n = nimg * nrow * ng;
    for (int i = rank * kEcThreads + e; i < n; i += kCluster * kEcThreads) {
        const int xg = g_lo + i % ng;
        const int q = i / ng;
        const int y = t.Y0 + q % nrow;
        const int img = 8 * t.g + q / nrow;
        uint16_t* base = a.dX + out_off(a, img, y, 8 * xg, t.cb);
        if (!store_ok(a.dX, a.dx_bytes, base, 16, a.status) ||
            !store_ok(a.dX, a.dx_bytes, base + 7 * a.sXo, 16, a.status))
            continue;   // debug build: outside dX (recorded)
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = ld_cg_v4(base + u * a.sXo);
#pragma unroll
        for (int u = 0; u < 8; ++u) st_v4(base + u * a.sXo, transpose8x8_col(v, u));
    }
}

// Pack the rotated filter lines of channel c into a padded-line buffer (warp 0):
// line ry holds F[ry][rx] at tap index rx + kOff, two taps per word, with
// F[ry][rx] = W[KH-1-ry][KW-1-rx] (orientation 0) or W[KH-1-rx][KW-1-ry]
// (orientation 1).  Only the words that hold taps are written; the rest of the
// buffer was zeroed at start.  Lane l writes word kOff/2 + l of every line,
// eight lines per batch of loads.
__device__ void pack_filter(const ToepNArgs& a, int c, uint32_t* buf, int lane)
{
    const int nw = (a.KX + 1) / 2;
    if (lane >= nw) return;
    const int rx0 = 2 * lane;
    uint32_t* dst = buf + kOff / 2 + lane;
    for (int ry0 = 0; ry0 < a.KY; ry0 += 8) {
        uint32_t lo[8], hi[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int ry = ry0 + u;
            lo[u] = hi[u] = 0;
            if (ry < a.KY) {
                const int r0 = a.orient ? (a.KH - 1 - rx0) : (a.KH - 1 - ry);
                const int s0 = a.orient ? (a.KW - 1 - ry) : (a.KW - 1 - rx0);
                lo[u] = a.filt[(static_cast<long long>(r0) * a.KW + s0) * a.C + c];
                if (rx0 + 1 < a.KX) {
                    const int r1 = a.orient ? (a.KH - 2 - rx0) : r0;
                    const int s1 = a.orient ? s0 : (a.KW - 2 - rx0);
                    hi[u] = a.filt[(static_cast<long long>(r1) * a.KW + s1) * a.C + c];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (ry0 + u < a.KY) dst[(ry0 + u) * a.half_l] = lo[u] | (hi[u] << 16);
    }
}

struct MmaCtxN {
    uint64_t* b_full;    // 8 arrivals: every CTA of the cluster has written its share of this CTA's B block
    uint64_t* bfree;     // 8 arrivals: every CTA's MMAs have finished reading its B block
    uint64_t* a_full;
    uint64_t* a_empty;
    uint64_t* d_full;
    uint64_t* d_empty;
    const volatile int* abort_flag;
    uint32_t tmem_base;
    uint32_t bblk_addr;
};

// The MMA issuer's loop over the cluster's tiles, compiled per (16-deep steps,
// sub-tiles).  Per tile: wait until the cluster has filled the B block and the
// epilogue has drained the accumulator, run the shift steps, then signal the
// accumulator full (this CTA) and the B block free (every CTA of the cluster).
template <int KQ, int XT>
__device__ __noinline__ bool mma_role_n(const ToepNArgs& a, const MmaCtxN& c, int ntiles)
{
    const int ncol_sub = 8 * a.NH;
    const uint32_t idesc =
        a.f16 ? idesc_f16_f32(128, ncol_sub, /*b_mn_major=*/false) : idesc_bf16_f32(128, ncol_sub, false);
    const uint32_t sbo = static_cast<uint32_t>(a.P) * 1024u;
    const uint32_t pb16 = a.panel_bytes >> 4;
    uint32_t d_tmem[4];
#pragma unroll
    for (int sx = 0; sx < 4; ++sx) d_tmem[sx] = c.tmem_base + static_cast<uint32_t>(sx * ncol_sub);
    const uint32_t a_first = c.tmem_base + static_cast<uint32_t>(a.a_col0);
    const uint32_t a_last = a_first + static_cast<uint32_t>((a.na - 1) * a.a_cols);
    // The loop reads registers only: the MMA and commit statements clobber memory, so
    // fields read through `a` or `c` would be loaded again after each of them, and this
    // single thread's issue rate bounds the tensor pipe's.
    const int NI = a.NI;
    const uint32_t a_cols = static_cast<uint32_t>(a.a_cols), bblk_addr = c.bblk_addr;
    uint64_t* const b_full = c.b_full;
    uint64_t* const d_empty = c.d_empty;
    uint64_t* const d_full = c.d_full;
    uint64_t* const a_full = c.a_full;
    uint64_t* const a_empty = c.a_empty;
    uint64_t* const bfree = c.bfree;
    const volatile int* const abort_flag = c.abort_flag;
    uint32_t ab = 0, aph = 0;
    uint32_t a_tmem = a_first;
    for (int t = 0; t < ntiles; ++t) {
        const uint32_t ph = static_cast<uint32_t>(t) & 1u;
        if (!mbar_wait_remote(b_full, ph, abort_flag) || !mbar_wait(d_empty, ph ^ 1u, abort_flag)) return false;
        fence_proxy_async_smem();
        tc_fence_after();
        uint64_t desc = sw128_desc(bblk_addr, 16, sbo);
        for (int i = 0; i < NI; ++i) {
            if (!mbar_wait(&a_full[ab], aph, abort_flag)) return false;
            tc_fence_after();
            issue_step<KQ, XT>(d_tmem, a_tmem, desc, pb16, idesc, i == 0);
            umma_commit(&a_empty[ab]);
            desc += 64;   // next shift step: one 1024-byte atom
            if (a_tmem == a_last) {
                a_tmem = a_first;
                ab = 0;
                aph ^= 1u;
            } else {
                a_tmem += a_cols;
                ++ab;
            }
        }
        umma_commit(d_full);
        umma_commit_mc(bfree, static_cast<uint16_t>((1u << kCluster) - 1u));
    }
    return true;
}

template <int XT>
__device__ __forceinline__ bool mma_role_nx(int kq, const ToepNArgs& a, const MmaCtxN& c, int ntiles)
{
    switch (kq) {
    case 1: return mma_role_n<1, XT>(a, c, ntiles);
    case 2: return mma_role_n<2, XT>(a, c, ntiles);
    case 3: return mma_role_n<3, XT>(a, c, ntiles);
    case 4: return mma_role_n<4, XT>(a, c, ntiles);
    case 5: return mma_role_n<5, XT>(a, c, ntiles);
    case 6: return mma_role_n<6, XT>(a, c, ntiles);
    case 7: return mma_role_n<7, XT>(a, c, ntiles);
    case 8: return mma_role_n<8, XT>(a, c, ntiles);
    default: return mma_role_n<9, XT>(a, c, ntiles);
    }
}

// Shared-memory objects and per-CTA values the roles work with.
struct KCtx {
    uint8_t* bblk;
    uint32_t* fwords;
    uint64_t *a_full, *a_empty, *d_full, *d_empty, *b_full, *bfree, *dx_ready, *f_full, *f_empty;
    volatile int* abort_flag;
    uint32_t tmem_base, rank;
    int su_begin, ntiles;
};

// A builders (warps 2-5): each thread writes its row of A_i for every shift step.
__device__ __forceinline__ void abuild_role(const ToepNArgs& a, const KCtx& k, int warp, int lane)
{
    uint32_t* fwords = k.fwords;
    uint64_t* a_full = k.a_full;
    uint64_t* a_empty = k.a_empty;
    uint64_t* d_full = k.d_full;
    uint64_t* d_empty = k.d_empty;
    uint64_t* b_full = k.b_full;
    uint64_t* bfree = k.bfree;
    uint64_t* dx_ready = k.dx_ready;
    uint64_t* f_full = k.f_full;
    uint64_t* f_empty = k.f_empty;
    volatile int* abort_flag = k.abort_flag;
    const uint32_t tmem_base = k.tmem_base;
    const uint32_t rank = k.rank;
    const int su_begin = k.su_begin;
    const int ntiles = k.ntiles;
    const uint32_t na = static_cast<uint32_t>(a.na);
    const int ncol_sub = 8 * a.NH;
    uint8_t* bblk = k.bblk;
    (void)fwords; (void)a_full; (void)a_empty; (void)d_full; (void)d_empty; (void)b_full; (void)bfree;
    (void)dx_ready; (void)f_full; (void)f_empty; (void)tmem_base; (void)rank; (void)na; (void)ncol_sub; (void)bblk;
    // ----------------------------------------------------------- A builders
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    const int p = m / a.TW;
    const int xl = m % a.TW;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t ab = 0, aph = 0, fcount = 0;
    int prev_cb = -1;
    const uint32_t* fbuf = fwords;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
        const Tile tl = decode_tile(a, su_begin + t);
        if (tl.cb != prev_cb) {
            const uint32_t fb = fcount % static_cast<uint32_t>(a.nfb);
            const uint32_t n = fcount / static_cast<uint32_t>(a.nfb);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&f_full[fb], n & 1u, abort_flag))) {
                ok = false;
                break;
            }
            fbuf = fwords + fb * a.f_words;
            ++fcount;
            prev_cb = tl.cb;
        }
        // A_i[m][j] = F[i-p][j + e], e = xb - x0 + px - xl; padded tap index t0 = e + kOff >= 0.
        const int t0 = tl.xb - tl.x0 + a.px - xl + kOff;
        const uint32_t* rowbase = fbuf + (t0 >> 1);
        const bool odd = (t0 & 1) != 0;
        // registers for the loop (its statements clobber memory)
        const int NI = a.NI, KY = a.KY, kq = a.Ks >> 4, half_l = a.half_l;
        const uint32_t a_base = tmem_base + lane_addr + static_cast<uint32_t>(a.a_col0);
        const uint32_t a_cols = static_cast<uint32_t>(a.a_cols);
        for (int i = 0; i < NI; ++i) {
            const uint32_t b = ab;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&a_empty[b], aph ^ 1u, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int ry = i - p;
            const uint32_t taddr = a_base + b * a_cols;
            const bool nonzero = ry >= 0 && ry < KY;
            store_a(kq, taddr, rowbase + (nonzero ? ry : 0) * half_l, odd, nonzero);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&a_full[b]);
            if (++ab == na) {
                ab = 0;
                aph ^= 1u;
            }
        }
        // done with this channel's filter lines: the packer may reuse the buffer
        const bool last = t + 1 >= ntiles || decode_tile(a, su_begin + t + 1).cb != tl.cb;
        if (ok && last) mbar_arrive(&f_empty[(fcount - 1u) % static_cast<uint32_t>(a.nfb)]);
    }
    if (!ok) {
        report_timeout(a.status);
        *abort_flag = 1;
    }
}

// Epilogue and data movement (warps 6-13).
__device__ __forceinline__ void ec_role(const ToepNArgs& a, const KCtx& k, int warp, int lane)
{
    uint32_t* fwords = k.fwords;
    uint64_t* a_full = k.a_full;
    uint64_t* a_empty = k.a_empty;
    uint64_t* d_full = k.d_full;
    uint64_t* d_empty = k.d_empty;
    uint64_t* b_full = k.b_full;
    uint64_t* bfree = k.bfree;
    uint64_t* dx_ready = k.dx_ready;
    uint64_t* f_full = k.f_full;
    uint64_t* f_empty = k.f_empty;
    volatile int* abort_flag = k.abort_flag;
    const uint32_t tmem_base = k.tmem_base;
    const uint32_t rank = k.rank;
    const int su_begin = k.su_begin;
    const int ntiles = k.ntiles;
    const uint32_t na = static_cast<uint32_t>(a.na);
    const int ncol_sub = 8 * a.NH;
    uint8_t* bblk = k.bblk;
    (void)fwords; (void)a_full; (void)a_empty; (void)d_full; (void)d_empty; (void)b_full; (void)bfree;
    (void)dx_ready; (void)f_full; (void)f_empty; (void)tmem_base; (void)rank; (void)na; (void)ncol_sub; (void)bblk;
    // ----------------------------------------- epilogue and data movement
    const int e = static_cast<int>(threadIdx.x) - kEcWarp0 * 32;
    const int quarter = warp & 3;
    const int half = (warp - kEcWarp0) >> 2;
    const int m = quarter * 32 + lane;
    const int p = m / a.TW;
    const int xl = m % a.TW;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int hcols = (a.XT * ncol_sub) >> 1;   // accumulator columns per half: at most 128
    const int nch = hcols >> 5;
    const uint32_t b_local = smem_u32(bblk);
    const uint32_t b_full_local = smem_u32(b_full);
    const uint32_t dx_ready_local = smem_u32(dx_ready);
    // tell every CTA of the cluster that this CTA's share of a B block (or of a
    // tile's dX) has been written
    auto signal_all = [&](uint32_t bar_local) {
        if (e == 0)
            for (uint32_t k = 0; k < kCluster; ++k) mbar_arrive_cluster(mapa_shared(bar_local, k));
    };
    bool ok = true;
    if (ntiles > 0) {
        const Tile t0 = decode_tile(a, su_begin);
        fill_window(a, t0, static_cast<int>(rank), e, b_local);
        fence_proxy_async_cluster();
        fence_acq_rel_cluster();
        named_barrier_sync(kBarEc, kEcThreads);
        signal_all(b_full_local);
    }
    for (int t = 0; t < ntiles; ++t) {
        const Tile tl = decode_tile(a, su_begin + t);
        const uint32_t ph = static_cast<uint32_t>(t) & 1u;
        // 1. drain the accumulator into registers (bf16 or f16 pairs) and release it
        ok = named_barrier_and(kBarEc, kEcThreads, ok && mbar_wait(d_full, ph, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t pk[64];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            if (cc < nch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(half * hcols + cc * 32), v);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    pk[cc * 16 + k] = a.f16 ? float2_to_f16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]))
                                            : float2_to_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
            }
        }
        tc_fence_before();
        mbar_arrive(d_empty);
        // 2. once every CTA's MMAs are done with their B blocks, write the next tile's
        //    window into them (the last tile only waits, so that every CTA's final
        //    B-free arrivals have landed before the cluster exits)
        ok = named_barrier_and(kBarEc, kEcThreads, mbar_wait_remote(bfree, ph, abort_flag));
        if (!ok) break;
        if (t + 1 < ntiles) {
            fill_window(a, decode_tile(a, su_begin + t + 1), static_cast<int>(rank), e, b_local);
            fence_proxy_async_cluster();
            fence_acq_rel_cluster();
            named_barrier_sync(kBarEc, kEcThreads);
            signal_all(b_full_local);
        }
        // 3. write this tile's dX in the permuted order (ragged column groups final)
        const bool img_full = 8 * tl.g + 8 <= a.N;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            if (cc < nch) {
                const int col0 = half * hcols + cc * 32;
                const int sx = col0 / ncol_sub;
                const int n0 = col0 - sx * ncol_sub;
                const int x = tl.x0 + sx * a.TW + xl;
                if (x < a.Xo) {
                    const bool grp = (x | 7) < a.Xo;   // the 8-column group of x is complete
                    const long long xterm =
                        grp ? (static_cast<long long>((x & ~7) + static_cast<int>(rank)) * a.sXo + (x & 7))
                            : (static_cast<long long>(x) * a.sXo + static_cast<int>(rank));
                    uint16_t* colbase = a.dX + xterm + 8LL * tl.cb + static_cast<long long>(8 * tl.g) * a.sNo;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int n = n0 + 2 * k;
                        const int y = tl.Y0 + a.P * (n >> 3) + p;
                        const int img = n & 7;
                        const uint32_t v = pk[cc * 16 + k];
                        if (y < a.Yo) {
                            uint16_t* d = colbase + img * a.sNo + y * a.sYo;
                            if ((img_full || 8 * tl.g + img < a.N) && store_ok(a.dX, a.dx_bytes, d, 2, a.status))
                                d[0] = static_cast<uint16_t>(v & 0xFFFFu);
                            if ((img_full || 8 * tl.g + img + 1 < a.N) &&
                                store_ok(a.dX, a.dx_bytes, d + a.sNo, 2, a.status))
                                d[a.sNo] = static_cast<uint16_t>(v >> 16);
                        }
                    }
                }
            }
        }
        fence_acq_rel_cluster();
        named_barrier_sync(kBarEc, kEcThreads);
        signal_all(dx_ready_local + 8u * ph);
        // 4. once all 8 CTAs have written the tile, transpose this CTA's share in place
        ok = named_barrier_and(kBarEc, kEcThreads,
                               mbar_wait_remote(&dx_ready[ph], (static_cast<uint32_t>(t) >> 1) & 1u, abort_flag));
        if (!ok) break;
        transpose_tile_out(a, tl, static_cast<int>(rank), e);
    }
    if (!ok && e == 0) {
        report_timeout(a.status);
        *abort_flag = 1;
    }
}

__global__ void __launch_bounds__(kThreadsN, 1)
    dw_toeplitz_nhwc_kernel(const __grid_constant__ ToepNArgs a)
{
    pdl_wait();      // the previous kernel on the stream has finished
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint8_t* bblk = smem;                                             // this CTA's B block
    uint32_t* fwords = reinterpret_cast<uint32_t*>(smem + a.f_off);   // padded-filter buffers (nfb of them)
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* a_full = bars;                 // [kMaxAN]
    uint64_t* a_empty = bars + kMaxAN;       // [kMaxAN]
    uint64_t* d_full = bars + 2 * kMaxAN;
    uint64_t* d_empty = d_full + 1;
    uint64_t* b_full = d_full + 2;
    uint64_t* bfree = d_full + 3;
    uint64_t* dx_ready = d_full + 4;         // [2]
    uint64_t* f_full = d_full + 6;           // [2]
    uint64_t* f_empty = d_full + 8;          // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBarsN);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    int su_begin, su_end;
    cluster_range(a, &su_begin, &su_end);
    const int ntiles = su_end - su_begin;
    const uint32_t na = static_cast<uint32_t>(a.na);
    const int ncol_sub = 8 * a.NH;

    if (threadIdx.x == 0) {
        for (int b = 0; b < kMaxAN; ++b) {
            mbar_init(&a_full[b], 128);
            mbar_init(&a_empty[b], 1);
        }
        mbar_init(d_full, 1);
        mbar_init(d_empty, kEcThreads);
        mbar_init(b_full, kCluster);
        mbar_init(bfree, kCluster);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&dx_ready[b], kCluster);
            mbar_init(&f_full[b], 1);
            mbar_init(&f_empty[b], 128);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemColsN);
        tmem_relinquish();
    }
    // Zero both filter buffers (only tap words are written later) and, with one
    // tile per plane, the B block (the window outside the image stays zero).
    {
        uint4* f4 = reinterpret_cast<uint4*>(fwords);
        const int nf = static_cast<int>(a.nfb * a.f_words / 4);
        for (int i = threadIdx.x; i < nf; i += kThreadsN) f4[i] = make_uint4(0, 0, 0, 0);
        if (a.full_plane) {
            uint4* b4 = reinterpret_cast<uint4*>(bblk);
            const int nb = static_cast<int>(a.b_bytes / 16);
            for (int i = threadIdx.x; i < nb; i += kThreadsN) b4[i] = make_uint4(0, 0, 0, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();   // every CTA's barriers are initialised and its B block zeroed
    const uint32_t tmem_base = *tmem_slot;
    const KCtx kc{bblk, fwords, a_full, a_empty, d_full, d_empty, b_full, bfree, dx_ready, f_full, f_empty,
                  abort_flag, tmem_base, rank, su_begin, ntiles};

    if (warp == 0) {
        // ------------------------------------------------------ filter packer
        uint32_t fcount = 0;
        int prev_cb = -1;
        for (int t = 0; t < ntiles; ++t) {
            const Tile tl = decode_tile(a, su_begin + t);
            if (tl.cb == prev_cb) continue;
            prev_cb = tl.cb;
            const uint32_t nfb = static_cast<uint32_t>(a.nfb);
            const uint32_t fb = fcount % nfb, n = fcount / nfb;
            if (!__all_sync(0xFFFFFFFFu, n < 1 || mbar_wait(&f_empty[fb], (n - 1u) & 1u, abort_flag))) {
                if (lane == 0) {
                    report_timeout(a.status);
                    *abort_flag = 1;
                }
                break;
            }
            pack_filter(a, 8 * tl.cb + static_cast<int>(rank), fwords + fb * a.f_words, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&f_full[fb]);
            ++fcount;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            MmaCtxN ctx{b_full, bfree, a_full, a_empty, d_full, d_empty, abort_flag, tmem_base, smem_u32(bblk)};
            const int kq = a.Ks >> 4;
            const bool ok = a.XT == 1   ? mma_role_nx<1>(kq, a, ctx, ntiles)
                            : a.XT == 2 ? mma_role_nx<2>(kq, a, ctx, ntiles)
                                        : mma_role_nx<4>(kq, a, ctx, ntiles);
            if (!ok) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
        }
    } else if (warp < kEcWarp0) {
        abuild_role(a, kc, warp, lane);
    } else {
        ec_role(a, kc, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, kTmemColsN);
    }
    cluster_sync();   // no CTA leaves while a peer may still write to its shared memory
}

// Clusters of 8 that can be resident at once for this kernel at `smem` bytes
// (cached per device and size; 0 when none fits).
int max_active_clusters(size_t smem)
{
    struct Entry {
        int dev;
        size_t smem;
        int n;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (const Entry& x : cache)
            if (x.dev == dev && x.smem == smem) return x.n;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCluster * 64);
    cfg.blockDim = dim3(kThreadsN);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kCluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, dw_toeplitz_nhwc_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> lk(mu);
    cache.push_back({dev, smem, n});
    return n;
}

}  // namespace

cudaError_t launch_dw_toeplitz_nhwc(const DwArgs& a, const ToepPlan& p, cudaStream_t stream)
{
    if (a.N <= 0) return cudaSuccess;
    if (a.C % kCluster != 0) return cudaErrorInvalidValue;
    ToepNArgs t{};
    t.dY = static_cast<const uint16_t*>(a.dY);
    t.filt = static_cast<const uint16_t*>(a.filt);
    t.dX = static_cast<uint16_t*>(a.dX);
    t.status = a.status;
    t.N = a.N;
    t.C = a.C;
    t.KH = a.KH;
    t.KW = a.KW;
    t.orient = p.orient;
    t.KY = p.KY;
    t.KX = p.KX;
    t.py = p.py;
    t.px = p.px;
    t.Yi = p.Yi;
    t.Xi = p.Xi;
    t.Yo = p.Yo;
    t.Xo = p.Xo;
    const long long C = a.C;
    t.sNi = static_cast<long long>(a.Ho) * a.Wo * C;
    t.sYi = p.orient ? C : static_cast<long long>(a.Wo) * C;
    t.sXi = p.orient ? static_cast<long long>(a.Wo) * C : C;
    t.sNo = static_cast<long long>(a.H) * a.W * C;
    t.sYo = p.orient ? C : static_cast<long long>(a.W) * C;
    t.sXo = p.orient ? static_cast<long long>(a.W) * C : C;
    t.P = p.P;
    t.TW = p.TW;
    t.XT = p.XT;
    t.NH = p.NH;
    t.Ks = p.Ks;
    t.NR = p.NR;
    t.NI = p.NI;
    t.half_l = p.half_l;
    t.npanels = p.npanels;
    t.clip = p.clip;
    t.num_xt = (p.Xo + p.XT * p.TW - 1) / (p.XT * p.TW);
    t.num_yt = (p.Yo + p.P * p.NH - 1) / (p.P * p.NH);
    t.num_g = (a.N + 7) / 8;
    const long long nsu = static_cast<long long>(a.C / kCluster) * t.num_g * t.num_yt * t.num_xt;
    if (nsu > 0x3FFFFFFFLL) return cudaErrorInvalidValue;
    t.num_su = static_cast<int>(nsu);
    t.a_col0 = p.a_col0;
    t.a_cols = p.a_cols;
    t.na = p.na;
    t.f16 = a.f16 ? 1 : 0;
    t.full_plane = (t.num_xt == 1 && t.num_yt == 1) ? 1 : 0;
    t.nfb = p.nfb;
    t.dx_bytes = static_cast<long long>(a.N) * a.H * a.W * a.C * 2;
    t.panel_bytes = p.panel_bytes;
    t.b_bytes = p.b_bytes;
    t.f_words = static_cast<uint32_t>(p.f_words);
    t.f_off = p.f_off;
    t.bar_off = p.bar_off;
    if (p.NB != 1 || (p.nfb != 1 && p.nfb != 2) || (p.f_words % 4) != 0) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(dw_toeplitz_nhwc_kernel), static_cast<int>(p.smem));
    if (e != cudaSuccess) return e;
    const int ncl_max = max_active_clusters(p.smem);
    if (ncl_max < 1) return cudaErrorNotSupported;
    const int ncl = static_cast<int>(nsu < ncl_max ? nsu : ncl_max);
    e = launch_kernel(dw_toeplitz_nhwc_kernel, dim3(static_cast<unsigned>(ncl * kCluster)), dim3(kThreadsN), p.smem,
                      stream, kCluster, t);
    return e;
}

}  // namespace dgrad
