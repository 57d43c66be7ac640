// dw_toeplitz.cu -- stride-1 depthwise dgrad on the tcgen05 tensor cores.
//
// At stride 1, depthwise dgrad is a per-channel correlation of dY with the
// 180-degree rotated filter at padding KH-1-pad_h, KW-1-pad_w ("channel-packed
// and large-filter depthwise dgrad", Technical Details: rotated-filter dgrad).
// Along one spatial axis (the "x" axis below) that correlation is a product
// with a banded Toeplitz matrix built from one filter line, so each channel's
// plane becomes a sum of GEMMs, one per filter line -- the formulation the
// pages' implicit-GEMM fallback stands for when large filters went through it
// (same page, Summary).  On the pages' own hardware large filters move to the
// FP32 rotated-filter kernel; on B200 the tensor cores have 20x the FP32 rate,
// so the banded product wins even though most of each Toeplitz tile is zero.
//
// Plane orientation.  out[y][x] = sum_{ry<KY, rx<KX} in[y+ry-py][x+rx-px] *
// F[ry][rx] with F the rotated filter.  Either (y, x) = (h, w) with F[ry][rx] =
// W[KH-1-ry][KW-1-rx] (orientation 0), or (y, x) = (w, h) with F[ry][rx] =
// W[KH-1-rx][KW-1-ry] (orientation 1); the host picks the one with less MMA
// work, i.e. the Toeplitz band along the filter's long side.
//
// GEMM tile (one channel c, 8 images, 2*NH output rows, 64 output columns):
//   M = 128 rows m = (p, xl): output row y = Y0 + 2*h' + p, column x = x0 + xl;
//   N = 8*NH columns n = (h', img);
//   shift step i = 0 .. KY (output-row phase p plus filter line ry = i - p):
//     A_i[m][j] = F[i-p][xb + j - x0 - xl + px]   (zero outside the filter)
//     B_i[j][n] = in[img][Y0 + 2*h' + i - py][xb + j]
//   D[m][n] = sum_i A_i * B_i, K = j in [0, K) with xb = x0 - px rounded down
//   to a multiple of 8.
// B_i for every i lives in one shared-memory block: K-major panels of 64
// columns j with the 128-byte swizzle, one 128-byte row per (yrow, img) in
// (yrow*8 + img) order, so each input row yrow is exactly one 1024-byte swizzle
// atom.  Row (h', img) of B_i is row (2*h' + i, img), so B_i is that block seen
// through a descriptor whose start moves by one atom per shift step and whose
// row-group stride is two atoms: one TMA load of the planar input per 64
// columns serves every shift.  When one tile spans the whole plane height, every
// block has the same rows of zero padding above and below the image; the two
// blocks then share the zero rows between them, which the kernel writes once, and
// each TMA load brings only the image rows (31x31 on 64-row planes: 173 KB for
// both blocks instead of 188 KB, which leaves room for six A tables instead of
// three; 110.4 -> 106.4 us on B200).  A_i is Toeplitz along both of its axes at the
// granularity of 8 x 8 core matrices when each 8-row group holds 4 columns of
// both row phases, so for P = 2 it is stored as a table of a_slots distinct
// 128-byte core matrices (3.75 KB at K = 64) that the MMA's no-swizzle
// descriptor walks with overlapping strides (build_a_tables); four warps write
// the tables into a ring of shared-memory buffers and tensor memory holds two
// accumulator sets, so one tile's epilogue overlaps the next tile's MMAs.
// Other tiles (P = 4, 8), or tables that do not fit, keep A_i as a 128 x K tile
// written by the four warps straight into tensor memory (up to four buffers)
// after one accumulator set.  bf16 or f16 operands: the transposes, the filter packing
// and the TMA copies move 16-bit patterns, only the MMA's operand format and the
// output rounding depend on the type.  The A builders read the channel's filter lines, padded
// with zeros and packed two taps per word, from shared memory; the producer
// brings them in with one bulk copy whenever the channel changes.
//
// Two transposes run around the MMA kernel, all through the caller's workspace:
// the first writes NHWC dY as planes [C][Yi][N][Xs] (channels outermost, images
// between rows and columns), and extra CTAs of the same launch write the padded
// filter lines of every channel; the second writes the planar output of the MMA
// epilogue back to NHWC dX.  Both are dw_transpose_tma_kernel (TMA on both
// sides); when a tensor map cannot be encoded, dw_transpose_kernel (CUDA cores)
// and a separate dw_filter_pack_kernel launch do the same.
//
// Launch order.  Like every kernel here, these wait for the kernel before them
// (griddepcontrol.wait) before touching global memory.  Unlike the others, they
// do not let the next kernel start early: the MMA kernel and a transpose fit on
// one SM together, and a transpose CTA waiting next to the MMA kernel slowed
// the 51x5 problem by 6% (measured), while the early start saved nothing here.
//
// Roles (448 threads, one CTA per SM, a contiguous range of tiles per CTA so
// that the image groups of one channel follow each other):
//   warp 0      producer: filter lines (bulk copy) and B panels (TMA)
//   warp 1      TMEM allocation (512 columns) and the MMA issuer (one lane)
//   warps 2-5   A builders: A_i tables in shared memory, or each thread's row of
//               A_i in tensor memory with tcgen05.st
//   warps 6-13  epilogue: two warps per TMEM lane quarter drain an accumulator
//               set into registers, release it, then round to bf16 and store planes
// Every wait is bounded; a timeout is recorded in the status word, raises the
// CTA's abort flag, lets issued copies and MMAs finish and frees TMEM.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "toeplitz_core.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {
using namespace toep;

constexpr int kThreadsT = 448;   // 14 warps: producer, MMA, 4 A builders, 8 epilogue
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxA = 6;         // A buffers: tensor-memory tiles (at most 4) or shared-memory tables
constexpr int kMaxB = 2;         // B blocks in shared memory
constexpr int kNumBars = 2 * kMaxB + 2 * kMaxA + 10;   // + d_full[2], d_empty[2], drain, f_full[2], f_empty[2], d_init


struct ToepArgs {
    const uint32_t* fpack;       // padded filter lines, f_words per channel
    __nv_bfloat16* dXp;          // planar output [C][Yo][N][Xso]
    int* status;
    int N, C, Yo, Xo, Xso;
    int KY, py, px;
    int P, TW, XT, NH, Ks, NR, NI, half_l, NB;
    int num_xt, num_yt, num_g, num_units;
    int a_col0, a_cols, na;      // TMEM column of A buffer 0, columns per buffer, buffer count
    int a_smem;                  // A_i lives in shared memory as a table of 8 x 8 core matrices (below)
    int a_slots;                 // 128-byte core matrices per table: 16 + P*(Ks/8 - 1)
    uint32_t a_off, a_bytes;     // offset of table 0 and the stride between tables
    int nacc;                    // accumulator sets in tensor memory: 2 when A is in shared memory
    int f16;                     // operands and output are f16 (else bf16)
    int clip;                    // one tile spans the row: B starts at input column 0 (xb = 0)
    int nfb;                     // filter-line buffers: 2 when they fit, so the next channel's lines load early
    int tma_epi;                 // the epilogue stages 8 x 8 x 64 boxes in shared memory and stores them by TMA
    uint32_t stg_off;            // 8 KB staging boxes: one or two per epilogue half
    int nstg;                    // staging boxes per half (two: a box is staged while the last one is read)
    uint32_t panel_bytes, b_bytes, npanels, f_bytes, f_words, f_off, bar_off;
    // B blocks: b_stride bytes apart.  When a tile spans the whole plane height, the rows of
    // zero padding above and below the image are written once, and neighbouring blocks share
    // the zero rows between them; the TMA box then carries only the image rows: it starts
    // b_zt rows into the block (b_ld_off bytes) and brings b_ld_bytes.
    uint32_t b_stride, b_ld_off, b_ld_bytes;
    int b_zt;
    uint32_t z_off[3], z_len[3];  // the zero rows, written at the start
    // split: the CTAs take equal ranges of shift steps instead of whole tiles.  A tile whose
    // steps two CTAs share is started by the higher CTA, which writes its fp32 partial sum
    // to part[its block] ([set_cols][128], column-major) and sets part_flag[its block]; the
    // lower CTA ends with the tile's first steps, adds that partial and stores the result.
    int split;
    float* part;
    int* part_flag;
    long long dxp_bytes;         // size of the planar output (index checks of the debug build)
};

struct Unit {
    int c, g, Y0, x0, xb;
};

__device__ __forceinline__ Unit decode_unit(const ToepArgs& a, int u)
{
    Unit t;
    const int xt = u % a.num_xt;
    int r = u / a.num_xt;
    const int yt = r % a.num_yt;
    r /= a.num_yt;
    t.g = r % a.num_g;
    t.c = r / a.num_g;
    t.Y0 = yt * a.P * a.NH;
    t.x0 = xt * a.XT * a.TW;
    t.xb = a.clip ? 0 : floor8(t.x0 - a.px);
    return t;
}

// Shared-memory barriers and addresses the MMA issuer works with.
struct MmaCtx {
    uint64_t* b_full;
    uint64_t* b_empty;
    uint64_t* a_full;
    uint64_t* a_empty;
    uint64_t* d_full;            // [nacc]
    uint64_t* d_empty;           // [nacc]
    const volatile int* abort_flag;
    uint32_t tmem_base;
    uint32_t bblk_addr;
    uint32_t a_addr;             // A table 0 (A in shared memory)
    uint64_t* d_init;            // split: the partial is in the last unit's accumulator set
};

// The MMAs of one shift step with A_i in shared memory: as issue_step, with the
// A descriptor advancing by two core matrices along K (2 * LBO = 256*P bytes)
// per 16-deep step.
template <int KQ, int XT>
__device__ __forceinline__ void issue_step_ss(const uint32_t (&d_tmem)[4], uint64_t a_desc_i, uint64_t desc_i,
                                              uint32_t pb16, uint32_t a_q16, uint32_t idesc, bool first)
{
    constexpr int TW = 64 / XT;
#pragma unroll
    for (int q = 0; q < KQ; ++q) {
#pragma unroll
        for (int sx = 0; sx < XT; ++sx) {
            const int col = sx * TW + 16 * q;
            const uint64_t bd = desc_i + static_cast<uint64_t>((col >> 6) * pb16 + ((col & 63) >> 4) * 2);
            umma_f16(d_tmem[sx], a_desc_i + static_cast<uint64_t>(q) * a_q16, bd, idesc,
                     (first && q == 0) ? 0u : 1u);
        }
    }
}

// The MMA issuer's loop over its units, compiled per (16-deep steps per tile,
// sub-tiles) so that each shift step is a short straight run of MMAs: buffer
// indices and phases advance incrementally and the B descriptor moves by one
// swizzle atom per step.  Returns false when a wait gave up.
template <int KQ, int XT, bool AS>
__device__ __noinline__ bool mma_role(const ToepArgs& a, const MmaCtx& c, int u_begin, int u_end, int i_first,
                                      int i_last)
{
    const int ncol_sub = 8 * a.NH;
    const uint32_t idesc =
        a.f16 ? idesc_f16_f32(128, ncol_sub, /*b_mn_major=*/false) : idesc_bf16_f32(128, ncol_sub, false);
    const uint32_t sbo = static_cast<uint32_t>(a.P) * 1024u;
    const uint32_t pb16 = a.panel_bytes >> 4;
    // accumulator set s of sub-tile sx at column s*XT*ncol_sub + sx*ncol_sub
    const uint32_t set_cols = static_cast<uint32_t>(a.XT * ncol_sub);
    uint32_t d_tmem[4];
#pragma unroll
    for (int sx = 0; sx < 4; ++sx) d_tmem[sx] = c.tmem_base + static_cast<uint32_t>(sx * ncol_sub);
    const uint32_t a_first = c.tmem_base + static_cast<uint32_t>(a.a_col0);
    // A tables: no swizzle, K-major; core matrix (g, kc) at slot g + P*kc, i.e. SBO = 128
    // bytes between 8-row groups and LBO = 128*P bytes between 8-column steps of K
    const uint64_t a_desc0 = noswz_desc(c.a_addr, 128u * static_cast<uint32_t>(a.P), 128u);
    const uint32_t a_q16 = 16u * static_cast<uint32_t>(a.P);
    const uint32_t a_buf16 = a.a_bytes >> 4;
    // Everything the loop reads lives in registers: the MMA and commit statements clobber
    // memory, so fields read through `a` or `c` would be loaded again after each of them,
    // and this single thread's issue rate bounds the tensor pipe's.
    const int NI = a.NI;
    const bool split = a.split != 0;
    const uint32_t na = static_cast<uint32_t>(a.na), nb = static_cast<uint32_t>(a.NB);
    const uint32_t a_cols = static_cast<uint32_t>(a.a_cols), b_stride = a.b_stride, bblk_addr = c.bblk_addr;
    const bool two_acc = a.nacc == 2;
    uint64_t* const b_full = c.b_full;
    uint64_t* const b_empty = c.b_empty;
    uint64_t* const a_full = c.a_full;
    uint64_t* const a_empty = c.a_empty;
    uint64_t* const d_full = c.d_full;
    uint64_t* const d_empty = c.d_empty;
    const volatile int* const abort_flag = c.abort_flag;
    uint32_t bb = 0, bph = 0, ab = 0, aph = 0;
    uint32_t a_tmem = a_first;
    for (int u = u_begin; u < u_end; ++u) {
        const uint32_t k = static_cast<uint32_t>(u - u_begin);
        const uint32_t acc = two_acc ? (k & 1u) : 0u;
        const uint32_t use = two_acc ? (k >> 1) : k;
        if (!mbar_wait(&b_full[bb], bph, abort_flag) || !mbar_wait(&d_empty[acc], (use & 1u) ^ 1u, abort_flag))
            return false;
        tc_fence_after();
        uint32_t d_set[4];
#pragma unroll
        for (int sx = 0; sx < 4; ++sx) d_set[sx] = d_tmem[sx] + acc * set_cols;
        // shift steps [ib, ie) of this unit (all of them unless the CTAs split it); when this
        // CTA ends inside its last unit, that unit's accumulator starts from the partial of
        // the unit's last steps (written by the epilogue warps), so its MMAs all accumulate
        const int ib = u == u_begin ? i_first : 0;
        const int ie = u == u_end - 1 ? i_last : NI;
        const bool from_partial = split && ie < NI;
        if (from_partial) {
            if (!mbar_wait(c.d_init, 0, abort_flag)) return false;
            tc_fence_after();
        }
        uint64_t desc = sw128_desc(bblk_addr + bb * b_stride, 16, sbo) + 64u * static_cast<uint32_t>(ib);
        uint64_t a_desc = a_desc0 + static_cast<uint64_t>(ab * a_buf16);
        for (int i = ib; i < ie; ++i) {
            if (!mbar_wait(&a_full[ab], aph, abort_flag)) return false;
            tc_fence_after();
            if (AS)
                issue_step_ss<KQ, XT>(d_set, a_desc, desc, pb16, a_q16, idesc, i == ib && !from_partial);
            else
                issue_step<KQ, XT>(d_set, a_tmem, desc, pb16, idesc, i == ib && !from_partial);
            umma_commit(&a_empty[ab]);   // A buffer free once these MMAs have read it
            desc += 64;                   // next shift step: one 1024-byte atom
            if (++ab == na) {
                a_tmem = a_first;
                a_desc = a_desc0;
                ab = 0;
                aph ^= 1u;
            } else {
                a_tmem += a_cols;
                a_desc += a_buf16;
            }
        }
        umma_commit(&d_full[acc]);
        umma_commit(&b_empty[bb]);
        if (++bb == nb) {
            bb = 0;
            bph ^= 1u;
        }
    }
    return true;
}

template <int XT, bool AS>
__device__ __forceinline__ bool mma_role_x(int kq, const ToepArgs& a, const MmaCtx& c, int u_begin, int u_end,
                                           int i_first, int i_last)
{
    switch (kq) {
    case 1: return mma_role<1, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 2: return mma_role<2, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 3: return mma_role<3, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 4: return mma_role<4, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 5: return mma_role<5, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 6: return mma_role<6, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 7: return mma_role<7, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    case 8: return mma_role<8, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    default: return mma_role<9, XT, AS>(a, c, u_begin, u_end, i_first, i_last);
    }
}

// A_i in shared memory (P = 2).  Row m of the MMA tile is m = 8g + r with r = 4p
// + xr: output row phase p, output column xl = 4*(15 - g) + xr.  Core matrix (g,
// kc) of A_i (rows 8g.., K columns 8kc..) then holds, in row r and column e,
// F[i-p][c0 + 8kc + e - xl] with c0 = xb - x0 + px, which depends on g and kc only
// through 4*(g + 2kc): every core matrix is one of a_slots = 16 + 2*(K/8 - 1)
// distinct 128-byte blocks, and block s = g + 2kc holds in row r taps w(s, xr) =
// c0 - 60 + 4s - xr .. +7 of line i-p.  The MMA's descriptor walks the blocks with
// SBO = 128 bytes (8-row groups) and LBO = 256 bytes (8-column steps of K), so A_i
// takes a_slots*128 bytes (3.75 KB at K = 64) instead of a 16 KB tile.  A builder
// thread owns pairs (s, xr), q = tb and tb + 128: row xr of block s takes line i's
// window, row 4 + xr line i-1's, which is the window the thread loaded for row xr
// at the step before, so each step reads one window per pair.  A line outside the
// filter reads as zeros.  Returns false when a wait gave up.
constexpr int kMaxAPairs = 2;   // (block, column) pairs per builder thread: a_slots <= 64
__device__ __forceinline__ uint4 load_window(const uint32_t* src, bool odd)
{
    const uint32_t w0 = src[0], w1 = src[1], w2 = src[2], w3 = src[3];
    const uint32_t w4 = odd ? src[4] : 0u;
    const uint32_t sh = odd ? 16u : 0u;
    return make_uint4(__funnelshift_r(w0, w1, sh), __funnelshift_r(w1, w2, sh), __funnelshift_r(w2, w3, sh),
                      __funnelshift_r(w3, w4, sh));
}

__device__ __forceinline__ bool build_a_tables(const ToepArgs& a, const Unit& t, const uint32_t* lines,
                                               uint8_t* tables, uint64_t* a_full, uint64_t* a_empty,
                                               const volatile int* abort_flag, int tb, uint32_t& ab, uint32_t& aph,
                                               int ib, int ie)
{
    const int c0 = t.xb - t.x0 + a.px;
    const int npairs = 4 * a.a_slots;
    const int NI = a.NI, KY = a.KY, half_l = a.half_l;   // registers (the loop's statements clobber memory)
    const uint32_t na = static_cast<uint32_t>(a.na), a_bytes = a.a_bytes;
    int wo[kMaxAPairs], off[kMaxAPairs];
    bool odd[kMaxAPairs];
    uint4 prev[kMaxAPairs];
#pragma unroll
    for (int k = 0; k < kMaxAPairs; ++k) {
        const int q = tb + 128 * k;
        const int sl = q >> 2;
        const int xr = q & 3;
        const int t0 = c0 - 60 + 4 * sl - xr + kOff;   // >= 2: c0 >= -7, kOff = 72
        wo[k] = t0 >> 1;
        odd[k] = (t0 & 1) != 0;
        off[k] = 128 * sl + 16 * xr;
        prev[k] = make_uint4(0u, 0u, 0u, 0u);          // line ib - 1 (none when ib = 0)
        if (ib > 0 && ib - 1 < KY && q < npairs) prev[k] = load_window(lines + (ib - 1) * half_l + wo[k], odd[k]);
    }
    (void)NI;
    for (int i = ib; i < ie; ++i) {
        uint4 cur[kMaxAPairs];
#pragma unroll
        for (int k = 0; k < kMaxAPairs; ++k) {
            cur[k] = make_uint4(0u, 0u, 0u, 0u);
            if (tb + 128 * k < npairs && i < KY) cur[k] = load_window(lines + i * half_l + wo[k], odd[k]);
        }
        if (!mbar_wait(&a_empty[ab], aph ^ 1u, abort_flag)) return false;
        uint8_t* tab = tables + ab * a_bytes;
#pragma unroll
        for (int k = 0; k < kMaxAPairs; ++k) {
            if (tb + 128 * k < npairs) {
                *reinterpret_cast<uint4*>(tab + off[k]) = cur[k];        // phase 0: line i
                *reinterpret_cast<uint4*>(tab + off[k] + 64) = prev[k];  // phase 1: line i-1
            }
            prev[k] = cur[k];
        }
        fence_proxy_async_smem();   // the tensor core reads the table through the async proxy
        mbar_arrive(&a_full[ab]);
        if (++ab == na) {
            ab = 0;
            aph ^= 1u;
        }
    }
    return true;
}

// Units [u_begin, u_end) of this CTA: a contiguous range, so that the tiles of
// one channel follow each other and share one filter load.
__device__ __forceinline__ void unit_range(const ToepArgs& a, int* u_begin, int* u_end)
{
    *u_begin = static_cast<int>((static_cast<long long>(blockIdx.x) * a.num_units) / gridDim.x);
    *u_end = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * a.num_units) / gridDim.x);
}

// Split tiles (ToepArgs::split), one epilogue thread: its accumulator row (TMEM lane)
// in the nch 32-column chunks from taddr, against a partial laid out [column][128 rows]
// from `out` / `in` (this thread's row and first column already applied).  Eight
// columns at a time, so that these rare paths need few registers beside the drain's.
__device__ __forceinline__ void partial_out(uint32_t taddr, int nch, float* out)
{
#pragma unroll 1
    for (int c8 = 0; c8 < 4 * nch; ++c8) {
        uint32_t v[8];
        tmem_ld_32x32b_x8(taddr + 8u * static_cast<uint32_t>(c8), v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k) __stcg(out + (8 * c8 + k) * 128, __uint_as_float(v[k]));
    }
}

__device__ __forceinline__ void partial_init(uint32_t taddr, int nch, const float* in)
{
#pragma unroll 1
    for (int h = 0; h < 2 * nch; ++h) {
        // 16 loads issued together (16 KB in flight per SM), then two 8-column stores
        uint32_t q[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) q[k] = __float_as_uint(__ldcg(in + (16 * h + k) * 128));
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            uint32_t v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = q[8 * g + k];
            tmem_st_32x32b_x8(taddr + 16u * static_cast<uint32_t>(h) + 8u * static_cast<uint32_t>(g), v);
        }
    }
    tmem_wait_st();
}

// With split: the steps [sb, se) of this CTA in the sequence of all units' shift
// steps; units [u_begin, u_end), the first from step i_first, the last up to step
// i_last (exclusive).  Without split: whole units, i_first = 0, i_last = NI.
__device__ __forceinline__ void step_range(const ToepArgs& a, int* u_begin, int* u_end, int* i_first, int* i_last)
{
    if (!a.split) {
        unit_range(a, u_begin, u_end);
        *i_first = 0;
        *i_last = a.NI;
        return;
    }
    const long long total = static_cast<long long>(a.num_units) * a.NI;
    const long long sb = (static_cast<long long>(blockIdx.x) * total) / gridDim.x;
    const long long se = (static_cast<long long>(blockIdx.x + 1) * total) / gridDim.x;
    *u_begin = static_cast<int>(sb / a.NI);
    *i_first = static_cast<int>(sb - static_cast<long long>(*u_begin) * a.NI);
    *u_end = static_cast<int>((se + a.NI - 1) / a.NI);
    *i_last = static_cast<int>(se - static_cast<long long>(*u_end - 1) * a.NI);
}

__global__ void __launch_bounds__(kThreadsT, 1)
    dw_toeplitz_kernel(const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_d,
                       const __grid_constant__ ToepArgs a)
{
    pdl_wait();      // the previous kernel on the stream has finished
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint8_t* bblk = smem;                                               // NB blocks of B panels (128-byte swizzle)
    uint32_t* fwords = reinterpret_cast<uint32_t*>(smem + a.f_off);     // nfb buffers of padded filter lines
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* b_full = bars;                          // [kMaxB]
    uint64_t* b_empty = bars + kMaxB;                 // [kMaxB]
    uint64_t* a_full = bars + 2 * kMaxB;              // [kMaxA]
    uint64_t* a_empty = a_full + kMaxA;               // [kMaxA]
    uint64_t* d_full = a_empty + kMaxA;               // [2]
    uint64_t* d_empty = d_full + 2;                   // [2]
    uint64_t* drain = d_full + 4;
    uint64_t* f_full = d_full + 5;                    // [2]
    uint64_t* f_empty = d_full + 7;                   // [2]
    uint64_t* d_init = d_full + 9;                    // split: the last unit's accumulator holds the partial
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t na = static_cast<uint32_t>(a.na);
    const uint32_t nb = static_cast<uint32_t>(a.NB);
    const int ncol_sub = 8 * a.NH;                    // accumulator columns per sub-tile
    int u_begin, u_end, i_first, i_last;
    step_range(a, &u_begin, &u_end, &i_first, &i_last);

    if (threadIdx.x == 0) {
        for (int b = 0; b < kMaxB; ++b) {
            mbar_init(&b_full[b], 1);
            mbar_init(&b_empty[b], 1);
        }
        for (int b = 0; b < kMaxA; ++b) {
            mbar_init(&a_full[b], 128);
            mbar_init(&a_empty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&d_full[b], 1);
            mbar_init(&d_empty[b], 256);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&f_full[b], 1);
            mbar_init(&f_empty[b], 128);
        }
        mbar_init(drain, 1);
        mbar_init(d_init, 256);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&map_b);
    // the shared zero rows of the B blocks, once; the tensor core reads them through the
    // async proxy (the barrier below orders them before the first MMA)
#pragma unroll
    for (int z = 0; z < 3; ++z)
        for (uint32_t o = 16u * threadIdx.x; o < a.z_len[z]; o += 16u * kThreadsT)
            *reinterpret_cast<uint4*>(bblk + a.z_off[z] + o) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // Per unit: the filter lines when the channel changes (one bulk copy into
        // the next of nfb buffers, so with two the next channel's lines load while
        // the builders still use the current ones), then the B panels (one TMA box
        // per 64 columns) into the next B block.
        if (lane == 0) {
            const uint32_t nfb = static_cast<uint32_t>(a.nfb);
            uint32_t ub = 0, fe = 0;
            int prev_c = -1;
            bool ok = true;
            for (int u = u_begin; u < u_end; ++u) {
                const Unit t = decode_unit(a, u);
                if (t.c != prev_c) {
                    const uint32_t fb = fe % nfb;
                    if (!mbar_wait(&f_empty[fb], ((fe / nfb) & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&f_full[fb], a.f_bytes);
                    bulk_load(fwords + fb * a.f_words, a.fpack + static_cast<int64_t>(t.c) * a.f_words, a.f_bytes,
                              &f_full[fb]);
                    ++fe;
                    prev_c = t.c;
                }
                const uint32_t bb = ub % nb;
                if (!mbar_wait(&b_empty[bb], ((ub / nb) & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&b_full[bb], a.b_ld_bytes);
                uint8_t* blk = bblk + bb * a.b_stride + a.b_ld_off;
                for (uint32_t pn = 0; pn < a.npanels; ++pn)
                    tma_load_4d(blk + pn * a.panel_bytes, &map_b, &b_full[bb], t.xb + 64 * static_cast<int>(pn),
                                8 * t.g, t.Y0 - a.py + a.b_zt, t.c);
                ++ub;
            }
            if (!ok) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
            // the last copies have landed before the CTA may exit
            for (uint32_t k = (ub > nb ? ub - nb : 0); k < ub; ++k)
                if (!mbar_wait(&b_full[k % nb], (k / nb) & 1u)) {
                    report_timeout(a.status);
                    *abort_flag = 1;
                }
            if (fe > 0 && !mbar_wait(&f_full[(fe - 1u) % nfb], ((fe - 1u) / nfb) & 1u)) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            MmaCtx ctx{b_full,    b_empty,        a_full,   a_empty, d_full, d_empty, abort_flag, tmem_base,
                       smem_u32(bblk), smem_u32(smem + a.a_off), d_init};
            const int kq = a.Ks >> 4;
            bool ok;
            if (a.a_smem)
                ok = a.XT == 1   ? mma_role_x<1, true>(kq, a, ctx, u_begin, u_end, i_first, i_last)
                     : a.XT == 2 ? mma_role_x<2, true>(kq, a, ctx, u_begin, u_end, i_first, i_last)
                                 : mma_role_x<4, true>(kq, a, ctx, u_begin, u_end, i_first, i_last);
            else
                ok = a.XT == 1   ? mma_role_x<1, false>(kq, a, ctx, u_begin, u_end, i_first, i_last)
                     : a.XT == 2 ? mma_role_x<2, false>(kq, a, ctx, u_begin, u_end, i_first, i_last)
                                 : mma_role_x<4, false>(kq, a, ctx, u_begin, u_end, i_first, i_last);
            if (!ok) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
            umma_commit(drain);
            if (!mbar_wait(drain, 0)) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
        }
    } else if (warp < 6) {
        // ----------------------------------------------------------- A builders
        const int quarter = warp & 3;
        const int m = quarter * 32 + lane;
        const int p = m / a.TW;
        const int xl = m % a.TW;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t nfb = static_cast<uint32_t>(a.nfb);
        uint32_t ab = 0, aph = 0, fe = 0, fb = 0;
        int prev_c = -1;
        bool ok = true;
        for (int u = u_begin; u < u_end && ok; ++u) {
            const Unit t = decode_unit(a, u);
            if (t.c != prev_c) {
                fb = fe % nfb;
                if (!mbar_wait(&f_full[fb], (fe / nfb) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                ++fe;
                prev_c = t.c;
            }
            const int ib = u == u_begin ? i_first : 0;
            const int ie = u == u_end - 1 ? i_last : a.NI;
            if (a.a_smem) {
                ok = build_a_tables(a, t, fwords + fb * a.f_words, smem + a.a_off, a_full, a_empty, abort_flag,
                                    threadIdx.x - 64, ab, aph, ib, ie);
                const bool last = u + 1 >= u_end || decode_unit(a, u + 1).c != t.c;
                if (ok && last) mbar_arrive(&f_empty[fb]);
                continue;
            }
            // A_i[m][j] = F[i-p][j + e], e = xb - x0 + px - xl (the same for every sub-tile);
            // padded tap index t0 = e + kOff >= 0.
            const int t0 = t.xb - t.x0 + a.px - xl + kOff;
            const uint32_t* rowbase = fwords + fb * a.f_words + (t0 >> 1);
            const bool odd = (t0 & 1) != 0;
            // registers for the loop (its statements clobber memory)
            const int KY = a.KY, kq = a.Ks >> 4, half_l = a.half_l;
            const uint32_t a_base = tmem_base + lane_addr + static_cast<uint32_t>(a.a_col0);
            const uint32_t a_cols = static_cast<uint32_t>(a.a_cols);
            for (int i = ib; i < ie; ++i) {
                const uint32_t b = ab;
                if (!mbar_wait(&a_empty[b], aph ^ 1u, abort_flag)) {
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
            // Done with this channel's filter lines: let the producer replace them.
            const bool last = u + 1 >= u_end || decode_unit(a, u + 1).c != t.c;
            if (ok && last) mbar_arrive(&f_empty[fb]);
        }
        if (!ok) {
            report_timeout(a.status);
            *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------- epilogue
        // Two warps per TMEM lane quarter, each draining half of the accumulator
        // columns into registers (as bf16 pairs) before releasing the accumulator.
        const int quarter = warp & 3;
        const int half = (warp - 6) >> 2;
        const int m = quarter * 32 + lane;
        // row m of the accumulator: output row phase p and column xl (see build_a_tables
        // for the order of the rows when A is in shared memory)
        const int R = 8 / a.P;
        const int p = a.a_smem ? (m & 7) / R : m / a.TW;
        const int xl = a.a_smem ? R * (15 - (m >> 3)) + (m & 7) % R : m % a.TW;
        const uint32_t set_cols = static_cast<uint32_t>(a.XT * ncol_sub);
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const int hcols = (a.XT * ncol_sub) >> 1;   // columns per half: at most 128
        const int nch = hcols >> 5;                  // 32-column chunks per half: 1 .. 4
        const int64_t img_stride = a.Xso;
        // a 16-bit store into the planar output (checked against its size in the debug build)
        auto put16 = [&](uint16_t* d, uint32_t v) {
            if (store_ok(a.dXp, a.dxp_bytes, d, 2, a.status)) d[0] = static_cast<uint16_t>(v);
        };
        const int64_t hrow_stride = static_cast<int64_t>(a.P) * a.N * a.Xso;
        uint32_t ub = 0;
        bool ok = true;
        const int part_row_i = m + half * hcols * 128;
        uint32_t stg_seq = 0;   // staged boxes of this half so far
        // split, CTA ending inside its last unit: that unit's accumulator set is freed by the
        // drain of the unit two before it (or is unused); the partial of the last unit's
        // remaining steps (the next CTA's first unit, ready long before) is written into it
        // right after that drain (after the first unit's, when the CTA has only two), while
        // the next unit's MMAs run, and the issuer waits for it.  A CTA sets its own flag
        // before it waits for the next CTA's, so the waits never form a chain.
        const bool init_last = a.split && i_last < a.NI;
        const int init_after = max(u_end - 3, u_begin);
        auto write_last_partial = [&]() -> bool {
            bool fw = true;
            if (warp == 6 && lane == 0) fw = flag_wait_gpu(a.part_flag + blockIdx.x + 1, abort_flag);
            if (!named_barrier_and(3, 256, fw)) return false;
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            const uint32_t acc_last = static_cast<uint32_t>(u_end - 1 - u_begin) & 1u;
            partial_init(tmem_base + lane_addr + acc_last * set_cols + static_cast<uint32_t>(half * hcols), nch,
                         a.part + static_cast<size_t>(blockIdx.x + 1) * 128 * set_cols + part_row_i);
            tc_fence_before();
            mbar_arrive(d_init);
            return true;
        };
        for (int u = u_begin; u < u_end; ++u) {
            const Unit t = decode_unit(a, u);
            const uint32_t acc = a.nacc == 2 ? (ub & 1u) : 0u;
            const uint32_t use = a.nacc == 2 ? (ub >> 1) : ub;
            const bool w = mbar_wait(&d_full[acc], use & 1u, abort_flag);
            // with staging boxes the half's 128 threads meet at named barriers, and with split
            // all 256 epilogue threads meet at barrier 3, so they agree on whether to go on
            const bool go = a.split      ? named_barrier_and(3, 256, w)
                            : a.tma_epi ? named_barrier_and(1 + half, 128, w)
                                        : w;
            if (!go) {
                ok = false;
                break;
            }
            uint16_t* stg0 = reinterpret_cast<uint16_t*>(smem + a.stg_off + half * a.nstg * 8192);
            const bool issuer = lane == 0 && (warp & 3) == 2;   // warps 6 and 10
            // P = 2, one sub-tile, staging boxes: the 128 threads of this half hold every row
            // m = (p, xl) of their 32-column chunk cc, i.e. 8 output rows (4 h' x 2 phases) x 8
            // images x 64 columns of one channel's planes; they stage that box in shared memory
            // and one thread stores it with TMA, which clips the ragged edges.
            auto stage_chunk = [&](int cc, const uint32_t* q) {
                (void)cc;
                uint16_t* stg = stg0 + (a.nstg == 2 ? (stg_seq & 1u) * 4096u : 0u);
                ++stg_seq;   // boxes alternate between the buffers in the order they are staged
                // the box staged in this buffer before has been read (with two buffers the
                // last box may still be in flight)
                if (issuer) {
                    if (a.nstg == 2)
                        bulk_wait_group_read<1>();
                    else
                        bulk_wait_group_read<0>();
                }
                named_barrier_sync(1 + half, 128);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int hp = (2 * k) >> 3;            // h' offset inside the chunk
                    const int img = (2 * k) & 7;
                    const uint32_t v = q[k];
                    stg[((2 * hp + p) * 8 + img) * 64 + xl] = static_cast<uint16_t>(v & 0xFFFFu);
                    stg[((2 * hp + p) * 8 + img + 1) * 64 + xl] = static_cast<uint16_t>(v >> 16);
                }
                fence_proxy_async_smem();
                named_barrier_sync(1 + half, 128);
                if (issuer) {
                    const int hp0 = (half * hcols + cc * 32) >> 3;
                    tma_store_4d(&map_d, stg, t.x0, 8 * t.g, t.Y0 + 2 * hp0, t.c);
                    bulk_commit_group();
                }
            };
            // split: the first unit of a CTA that starts inside it holds the unit's last steps,
            // whose fp32 partial goes to part[blockIdx.x] ([column][row m]); the last unit of a
            // CTA that ends inside it started from part[blockIdx.x + 1] (below) and is drained
            // and stored as usual.
            const uint32_t tacc = tmem_base + lane_addr + acc * set_cols + static_cast<uint32_t>(half * hcols);
            const size_t part_stride = static_cast<size_t>(128) * set_cols;
            const size_t part_row = static_cast<size_t>(m) + static_cast<size_t>(half * hcols) * 128;
            if (a.split && u == u_begin && i_first > 0) {
                tc_fence_after();
                partial_out(tacc, nch, a.part + static_cast<size_t>(blockIdx.x) * part_stride + part_row);
                tc_fence_before();
                mbar_arrive(&d_empty[acc]);
                __threadfence();                 // every epilogue thread's partial is written ...
                named_barrier_sync(3, 256);
                if (warp == 6 && lane == 0) flag_set_gpu(a.part_flag + blockIdx.x);   // ... before the flag
                if (init_last && u == init_after && !write_last_partial()) {
                    ok = false;
                    break;
                }
                ++ub;
                continue;
            }
            tc_fence_after();
            uint32_t pk[64];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                if (cc < nch) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(
                        tmem_base + lane_addr + acc * set_cols + static_cast<uint32_t>(half * hcols + cc * 32), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        pk[cc * 16 + k] = a.f16 ? float2_to_f16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]))
                                                : float2_to_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                }
            }
            tc_fence_before();
            mbar_arrive(&d_empty[acc]);   // the accumulator may be overwritten now
            if (init_last && u == init_after && !write_last_partial()) {
                ok = false;
                break;
            }
            if (a.tma_epi) {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    if (cc < nch) stage_chunk(cc, pk + cc * 16);
                ++ub;
                continue;
            }
            const bool full = t.Y0 + a.P * a.NH <= a.Yo && 8 * t.g + 8 <= a.N;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                if (cc < nch) {
                    // a 32-column chunk lies inside one sub-tile (ncol_sub is a multiple of 32)
                    const int col0 = half * hcols + cc * 32;
                    const int sx = col0 / ncol_sub;
                    const int n0 = col0 - sx * ncol_sub;          // column within the sub-tile
                    const int x = t.x0 + sx * a.TW + xl;
                    if (x < a.Xo) {
                        const int hp0 = n0 >> 3;
                        uint16_t* base = reinterpret_cast<uint16_t*>(a.dXp) +
                                         ((static_cast<int64_t>(t.c) * a.Yo + t.Y0 + a.P * hp0 + p) * a.N + 8 * t.g) *
                                             a.Xso + x;
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int hp = (2 * k) >> 3;              // h' offset inside the chunk
                            const int img = (2 * k) & 7;
                            uint16_t* dst = base + hp * hrow_stride + img * img_stride;
                            const uint32_t v = pk[cc * 16 + k];
                            if (full) {
                                put16(dst, v & 0xFFFFu);
                                put16(dst + img_stride, v >> 16);
                            } else if (t.Y0 + a.P * (hp0 + hp) + p < a.Yo) {
                                if (8 * t.g + img < a.N) put16(dst, v & 0xFFFFu);
                                if (8 * t.g + img + 1 < a.N) put16(dst + img_stride, v >> 16);
                            }
                        }
                    }
                }
            }
            ++ub;
        }
        if (!ok) {
            report_timeout(a.status);
            *abort_flag = 1;
        }
        if (a.tma_epi && lane == 0 && (warp & 3) == 2) bulk_wait_group<0>();   // the boxes have been written
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Padded filter lines of every channel, in the plane orientation: line ry of
// channel c is F[ry][rx] = W[KH-1-ry][KW-1-rx] (orientation 0) or
// W[KH-1-rx][KW-1-ry] (orientation 1) at tap index rx + kOff, zero elsewhere;
// word w of a line holds taps (2w - kOff, 2w + 1 - kOff).  f_words words per
// channel.  One CTA handles one line ry of 32 channels: the taps are read
// channel-contiguous (coalesced) into shared memory, then each warp writes whole
// lines.  A line has at most 64 taps, so each thread issues all of its (at most
// eight) tap loads before the first store: the CTA waits on one memory latency.
constexpr int kPackThreads = 256;
constexpr int kPackPer = 64 * 32 / kPackThreads;   // tap loads per thread

__device__ __forceinline__ void pack_filter_block(const __nv_bfloat16* __restrict__ filt, uint32_t* __restrict__ dst,
                                                  int C, int KH, int KW, int KY, int KX, int orient, int half_l,
                                                  int f_words, int bx, int ry)
{
    __shared__ uint16_t taps[64][34];   // [rx][channel]
    const int c0 = bx * 32;
    const unsigned short* w16 = reinterpret_cast<const unsigned short*>(filt);
    unsigned short v[kPackPer];
#pragma unroll
    for (int k = 0; k < kPackPer; ++k) {
        const int idx = threadIdx.x + k * kPackThreads;
        const int rx = idx >> 5;
        const int cl = idx & 31;
        const int r = orient ? (KH - 1 - rx) : (KH - 1 - ry);
        const int s = orient ? (KW - 1 - ry) : (KW - 1 - rx);
        v[k] = (rx < KX && c0 + cl < C) ? w16[(static_cast<int64_t>(r) * KW + s) * C + c0 + cl] : 0;
    }
#pragma unroll
    for (int k = 0; k < kPackPer; ++k) {
        const int idx = threadIdx.x + k * kPackThreads;
        if ((idx >> 5) < KX) taps[idx >> 5][idx & 31] = v[k];
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    for (int cl = warp; cl < 32; cl += blockDim.x >> 5) {
        const int c = c0 + cl;
        if (c >= C) break;
        uint32_t* line = dst + static_cast<int64_t>(c) * f_words + static_cast<int64_t>(ry) * half_l;
        for (int w = lane; w < half_l; w += 32) {
            const int rx0 = 2 * w - kOff;
            const uint32_t lo = (rx0 >= 0 && rx0 < KX) ? taps[rx0][cl] : 0u;
            const uint32_t hi = (rx0 + 1 >= 0 && rx0 + 1 < KX) ? taps[rx0 + 1][cl] : 0u;
            line[w] = lo | (hi << 16);
        }
        if (ry == KY - 1)   // zero the words that round the channel's block up to f_words
            for (int w = KY * half_l + lane; w < f_words; w += 32) dst[static_cast<int64_t>(c) * f_words + w] = 0u;
    }
}

__global__ void __launch_bounds__(kPackThreads)
    dw_filter_pack_kernel(const __nv_bfloat16* __restrict__ filt, uint32_t* __restrict__ dst, int C, int KH, int KW,
                          int KY, int KX, int orient, int half_l, int f_words, int* part_flag, int nflags)
{
    pdl_wait();      // the previous kernel on the stream has finished
    if (blockIdx.x == 0 && blockIdx.y == 0)   // the split flags of the MMA kernel that follows
        for (int i = threadIdx.x; i < nflags; i += blockDim.x) part_flag[i] = 0;
    pack_filter_block(filt, dst, C, KH, KW, KY, KX, orient, half_l, f_words, blockIdx.x, blockIdx.y);
}

// NHWC <-> planar [C][Y][N][Xs] for bf16.  The NHWC side addresses element
// (n, y, x, c) at n*sN + y*sY + x*sX + c; the planar side at ((c*Y + y)*N + n)*Xs
// + x.  A tile is 64 x-positions by 64 channels of one (n, y), moved as 16-byte
// chunks through a shared-memory transpose.  Each CTA takes kRowsPerCta
// consecutive y of one (n, x block, channel block): it loads all of their tiles
// into registers first (eight 16-byte loads per thread in flight), then
// transposes and stores them one after the other.
constexpr int kRowsPerCta = 4;

template <bool TO_PLANAR>
__global__ void __launch_bounds__(256)
    dw_transpose_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int N, int Y, int X,
                        int Xs, int C, int64_t sN, int64_t sY, int64_t sX, long long dst_bytes, int* status)
{
    pdl_wait();      // the previous kernel on the stream has finished
    __shared__ uint32_t tile[64][33];   // [row][pair]: rows are x (to planar) or c (from planar)
    const int nct = (C + 63) >> 6;
    const int ct = blockIdx.x % nct;
    const int x0 = (blockIdx.x / nct) * 64;
    const int c0 = ct * 64;
    const int y0 = blockIdx.y * kRowsPerCta;
    const int n = blockIdx.z;
    uint4 v[kRowsPerCta][2];
#pragma unroll
    for (int r = 0; r < kRowsPerCta; ++r) {
        const int y = y0 + r;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int idx = threadIdx.x + 256 * k;
            const int row = idx >> 3;          // x (to planar) or c (from planar)
            const int col = (idx & 7) * 8;     // c chunk (to planar) or x chunk (from planar)
            v[r][k] = make_uint4(0, 0, 0, 0);
            if (y < Y) {
                if (TO_PLANAR) {
                    if (x0 + row < X && c0 + col < C)
                        v[r][k] = *reinterpret_cast<const uint4*>(src + n * sN + y * sY +
                                                                  static_cast<int64_t>(x0 + row) * sX + c0 + col);
                } else {
                    if (c0 + row < C && x0 + col < X)
                        v[r][k] = *reinterpret_cast<const uint4*>(
                            src + ((static_cast<int64_t>(c0 + row) * Y + y) * N + n) * Xs + x0 + col);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerCta; ++r) {
        const int y = y0 + r;
        if (y >= Y) break;   // uniform across the CTA
        if (r > 0) __syncthreads();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int idx = threadIdx.x + 256 * k;
            const int row = idx >> 3;
            const int col = (idx & 7) * 8;
            tile[row][col / 2 + 0] = v[r][k].x;
            tile[row][col / 2 + 1] = v[r][k].y;
            tile[row][col / 2 + 2] = v[r][k].z;
            tile[row][col / 2 + 3] = v[r][k].w;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int idx = threadIdx.x + 256 * k;
            const int orow = idx >> 3;         // c (to planar) or x (from planar)
            const int ocol = (idx & 7) * 8;    // x chunk (to planar) or c chunk (from planar)
            const int sh = (orow & 1) * 16;
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t lo = (tile[ocol + 2 * j][orow >> 1] >> sh) & 0xFFFFu;
                const uint32_t hi = (tile[ocol + 2 * j + 1][orow >> 1] >> sh) & 0xFFFFu;
                w[j] = lo | (hi << 16);
            }
            if (TO_PLANAR) {
                __nv_bfloat16* d = dst + ((static_cast<int64_t>(c0 + orow) * Y + y) * N + n) * Xs + x0 + ocol;
                if (c0 + orow < C && x0 + ocol < X && store_ok(dst, dst_bytes, d, 16, status))
                    *reinterpret_cast<uint4*>(d) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                __nv_bfloat16* d = dst + n * sN + y * sY + static_cast<int64_t>(x0 + orow) * sX + c0 + ocol;
                if (x0 + orow < X && c0 + ocol < C && store_ok(dst, dst_bytes, d, 16, status))
                    *reinterpret_cast<uint4*>(d) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
}

// The same NHWC <-> planar move with TMA on both sides: a persistent kernel
// walks 64 x 64 tiles with a four-deep ring of loaded tiles (128-byte swizzle,
// rows of 64 elements), transposes each in-warp with ldmatrix.trans and
// stmatrix (conflict-free on swizzled rows), and writes it back with a TMA
// store, which clips the ragged edges.  Tile t = ((n*Y + y)*nxb + xb)*ncb + cb.
// src_map and dst_map are the NHWC map (dims C, W, H, N; box 64 channels by 64
// positions along x) and the planar map (dims X, N, Y, C; box 64 x by 64 c), in
// the order of the move.
constexpr int kTrStages = 4;

struct TrArgs {
    int to_planar, orient, N, Y, nxb, ncb, ntiles;
    int* status;
    int grid_tr;   // CTAs that transpose; CTAs past them pack filter lines (dY launch only)
    const __nv_bfloat16* filt;
    uint32_t* fpk;
    int C, KH, KW, KY, KX, half_l, f_words, pack_ncb;
    int* part_flag;   // split flags of the MMA kernel that follows, cleared by the first packing CTA
    int nflags;
};

__device__ __forceinline__ void tr_coords(const TrArgs& a, int t, bool nhwc_side, int (&c)[4])
{
    const int cb = t % a.ncb;
    int q = t / a.ncb;
    const int xb = q % a.nxb;
    q /= a.nxb;
    const int y = q % a.Y;
    const int n = q / a.Y;
    if (nhwc_side) {   // (C, W, H, N): x is W in orientation 0, H in orientation 1
        c[0] = cb * 64;
        c[1] = a.orient ? y : xb * 64;
        c[2] = a.orient ? xb * 64 : y;
        c[3] = n;
    } else {           // (X, N, Y, C)
        c[0] = xb * 64;
        c[1] = n;
        c[2] = y;
        c[3] = cb * 64;
    }
}

__global__ void __launch_bounds__(256)
    dw_transpose_tma_kernel(const __grid_constant__ CUtensorMap src_map, const __grid_constant__ CUtensorMap dst_map,
                            const __grid_constant__ TrArgs a)
{
    pdl_wait();      // the previous kernel on the stream has finished
    if (static_cast<int>(blockIdx.x) >= a.grid_tr) {   // the filter-packing CTAs of the dY launch
        const int b = static_cast<int>(blockIdx.x) - a.grid_tr;
        if (b == 0)
            for (int i = threadIdx.x; i < a.nflags; i += blockDim.x) a.part_flag[i] = 0;
        pack_filter_block(a.filt, a.fpk, a.C, a.KH, a.KW, a.KY, a.KX, a.orient, a.half_l, a.f_words, b % a.pack_ncb,
                          b / a.pack_ncb);
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* in_t = smem;                                  // kTrStages tiles of 8 KB
    uint8_t* out_t = smem + kTrStages * 8192;              // 2 tiles of 8 KB
    uint64_t* full = reinterpret_cast<uint64_t*>(out_t + 2 * 8192);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const bool src_nhwc = a.to_planar != 0;
    if (tid == 0) {
        for (int s = 0; s < kTrStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    int issued[kTrStages] = {0, 0, 0, 0};   // loads thread 0 has issued into each stage
    if (tid == 0) {
        tma_prefetch_desc(&src_map);
        tma_prefetch_desc(&dst_map);
        for (int s = 0; s < kTrStages; ++s) {
            const int t = static_cast<int>(blockIdx.x) + s * a.grid_tr;
            if (t >= a.ntiles) break;
            int c[4];
            tr_coords(a, t, src_nhwc, c);
            mbar_arrive_expect_tx(&full[s], 8192);
            tma_load_4d(in_t + s * 8192, &src_map, &full[s], c[0], c[1], c[2], c[3]);
            ++issued[s];
        }
    }
    bool aborted = false;
    int k = 0;
    for (int t = blockIdx.x; t < a.ntiles; t += a.grid_tr, ++k) {
        const int s = k % kTrStages;
        const int o = k & 1;
        const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((k / kTrStages) & 1));
        if (tid == 0 && k >= 2) bulk_wait_group_read<1>();   // the store of tile k-2 has read out[o]
        if (__syncthreads_or(!ok)) {
            if (tid == 0) report_timeout(a.status);
            aborted = true;
            break;
        }
        // warp w transposes the eight 8x8 blocks of rows 8w .. 8w+7: block (w, j) of the
        // input becomes block (j, w) of the output
        const uint32_t in_base = smem_u32(in_t + s * 8192);
        const uint32_t out_base = smem_u32(out_t + o * 8192);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int m = lane >> 3;                 // matrix of this lane's address
            const int j = 4 * h + m;                 // input chunk (column block)
            const int rin = 8 * warp + (lane & 7);   // input row
            uint32_t r[4];
            ldmatrix_x4_trans(in_base + rin * 128 + ((j ^ (rin & 7)) << 4), r);
            const int rout = 8 * j + (lane & 7);     // output row
            stmatrix_x4(out_base + rout * 128 + ((warp ^ (rout & 7)) << 4), r);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            int c[4];
            tr_coords(a, t, !src_nhwc, c);
            tma_store_4d(&dst_map, out_t + o * 8192, c[0], c[1], c[2], c[3]);
            bulk_commit_group();
            const int tn = t + kTrStages * a.grid_tr;
            if (tn < a.ntiles) {
                tr_coords(a, tn, src_nhwc, c);
                mbar_arrive_expect_tx(&full[s], 8192);
                tma_load_4d(in_t + s * 8192, &src_map, &full[s], c[0], c[1], c[2], c[3]);
                ++issued[s];
            }
        }
    }
    if (tid == 0) {
        if (aborted)   // let the loads still in flight land (bounded) before the CTA exits
            for (int s = 0; s < kTrStages; ++s)
                if (issued[s] > 0) mbar_wait(&full[s], static_cast<uint32_t>((issued[s] - 1) & 1));
        bulk_wait_group<0>();   // every store has completed before the CTA exits
    }
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool plan_dw_toeplitz(const DwArgs& a, ToepPlan* out, bool nhwc)
{
    if (!(a.bf16 || a.f16) || a.S != 1) return false;
    // Tile shapes (P row phases, NH row groups, XT sub-tiles of 128/P columns), in the
    // order measured fastest on B200: N = 256 tiles (two row phases) first.  Smaller
    // tiles issue more MMAs per output at a lower rate per MMA, so they serve only
    // filters whose B block would not fit otherwise.  Among the two orientations the
    // first fitting shape with fewer MMAs (rounds of tiles x shift steps x depth)
    // wins.  The plan does not depend on the device, so the workspace size can be
    // queried on the host.
    constexpr int kPlanSms = 148;
    static const int cand[][3] = {{2, 32, 1}, {2, 16, 1}, {4, 16, 2}, {4, 8, 2}, {8, 8, 4}, {8, 4, 4}};
    // DGRAD_TC_TILE="orient,P,NH,XT" restricts the plan to that shape (testing and tuning).
    int force[4] = {-1, -1, -1, -1};
    // DGRAD_TC_CLIP=0 keeps the full Toeplitz band for single-tile rows (testing and tuning).
    const char* clp = dgrad::tuning_env("DGRAD_TC_CLIP");
    const bool no_clip = clp && strcmp(clp, "0") == 0;
    // DGRAD_TC_EPI=store keeps the epilogue's direct 16-bit stores (testing and tuning).
    const char* epi = dgrad::tuning_env("DGRAD_TC_EPI");
    const bool no_tma_epi = epi && strcmp(epi, "store") == 0;
    // DGRAD_TC_A=tmem keeps A_i in tensor memory, written by the builders; DGRAD_TC_A=smem takes
    // the shared-memory tables whenever they fit (testing and tuning).
    const char* amode = dgrad::tuning_env("DGRAD_TC_A");
    const bool no_a_smem = amode && strcmp(amode, "tmem") == 0;
    const bool force_a_smem = amode && strcmp(amode, "smem") == 0;
    // DGRAD_TC_SHZ=0 gives every B block its own zero rows, loaded with the image rows (testing
    // and tuning).
    const char* shz = dgrad::tuning_env("DGRAD_TC_SHZ");
    const bool no_shz = shz && strcmp(shz, "0") == 0;
    // DGRAD_TC_SPLIT=0 keeps whole tiles per CTA (testing and tuning).
    const char* spl = dgrad::tuning_env("DGRAD_TC_SPLIT");
    const bool no_split = spl && strcmp(spl, "0") == 0;
    // DGRAD_TC_STG=1 keeps one epilogue staging box per half (testing and tuning).
    const char* stgs = dgrad::tuning_env("DGRAD_TC_STG");
    const bool one_stg = stgs && strcmp(stgs, "1") == 0;
    // DGRAD_TC_NA=n takes at most n shared-memory tables; DGRAD_TC_NFB=1 one filter-line buffer
    // (testing and tuning).
    const char* nas = dgrad::tuning_env("DGRAD_TC_NA");
    const int max_na = nas ? atoi(nas) : kMaxA;
    const char* nfs = dgrad::tuning_env("DGRAD_TC_NFB");
    const bool one_fb = nfs && strcmp(nfs, "1") == 0;
    if (const char* ft = dgrad::tuning_env("DGRAD_TC_TILE"))
        if (sscanf(ft, "%d,%d,%d,%d", &force[0], &force[1], &force[2], &force[3]) != 4) force[0] = -1;
    bool have = false;
    ToepPlan best{};
    double best_cost = 0;
    for (int orient = 0; orient < 2; ++orient) {
        ToepPlan g{};
        g.orient = orient;
        g.KY = orient ? a.KW : a.KH;
        g.KX = orient ? a.KH : a.KW;
        g.py = orient ? (a.KW - 1 - a.pw) : (a.KH - 1 - a.ph);
        g.px = orient ? (a.KH - 1 - a.ph) : (a.KW - 1 - a.pw);
        g.Yi = orient ? a.Wo : a.Ho;
        g.Xi = orient ? a.Ho : a.Wo;
        g.Yo = orient ? a.W : a.H;
        g.Xo = orient ? a.H : a.W;
        g.Xsi = (g.Xi + 7) & ~7;
        g.Xso = (g.Xo + 7) & ~7;
        const int mis = (-g.px) - floor8(-g.px);   // the same for every tile (x0 is a multiple of 8)
        for (const auto& cd : cand) {
            if (force[0] >= 0 && (force[0] != orient || force[1] != cd[0] || force[2] != cd[1] || force[3] != cd[2]))
                continue;
            ToepPlan p = g;
            p.P = cd[0];
            p.NH = cd[1];
            p.XT = cd[2];
            p.TW = 128 / p.P;
            // When one tile of one sub-tile spans the whole output row, the K range (input
            // columns j) is clipped to the columns inside the image, starting at j = 0: the
            // columns outside are the zero padding, whose B rows are zero and add nothing.  For
            // 64-wide planes this takes K from 96 to 64 at 31x31 and from 128 to 64 at 51x5, and
            // one 64-column panel then fits twice in shared memory.
            p.clip = p.XT == 1 && p.Xo <= p.TW && !no_clip ? 1 : 0;
            if (p.clip)
                p.Ks = (std::max(std::min(p.Xi, p.TW + p.KX - 1 - p.px), 16) + 15) & ~15;
            else
                p.Ks = (p.TW + p.KX - 1 + mis + 15) & ~15;
            if (p.Ks > 144) continue;
            const int span = (p.XT - 1) * p.TW + p.Ks;
            p.npanels = (span + 63) / 64;
            p.NR = p.P * p.NH + p.KY - 1;
            if (p.NR > 256) continue;
            p.NI = p.KY + p.P - 1;
            // a line holds every tap a row reads: from word t0/2, Ks/2 + 1 words, t0 at most
            // px + kOff when clipped (xb = x0 = 0, xl = 0), kOff - mis otherwise
            p.half_l = p.clip ? ((p.px + kOff) >> 1) + (p.Ks >> 1) + 1 : (p.Ks + kOff + 8) / 2;
            p.f_words = static_cast<int>(round_up(static_cast<size_t>(p.KY) * p.half_l, 4));
            p.a_cols = ((p.Ks / 2) + 31) & ~31;
            const int ncols_d = p.XT * 8 * p.NH;
            if (ncols_d > 256 || (ncols_d / 2) % 32 != 0) continue;
            // The planar kernel keeps A_i in shared memory (tables of core matrices, see
            // build_a_tables) for P = 2 when a table has at most 32*kMaxAPairs blocks, a
            // layout with two or more tables fits and a tile runs at least 16 shift steps;
            // tensor memory then holds two accumulator sets.  Otherwise A_i goes to tensor
            // memory after one accumulator set.  Measured on B200 (bench suite): 31x31 (32
            // steps) 109.6 us with tables against 113.4 us in tensor memory, 51x5 and 5x51 (6
            // steps) 60.9 us against 59.6 us.
            p.a_slots = 16 + p.P * (p.Ks / 8 - 1);
            p.a_bytes = static_cast<uint32_t>(p.a_slots) * 128u;
            p.a_col0 = ncols_d;
            const int na_tmem = std::min((static_cast<int>(kTmemCols) - p.a_col0) / p.a_cols, 4);
            p.panel_bytes = static_cast<uint32_t>(p.NR) * 1024u;
            p.b_bytes = static_cast<uint32_t>(p.npanels) * p.panel_bytes;
            // When a tile spans the whole plane height, every B block holds the same zt = py
            // rows of zero padding above the image rows and zb below them.  With two blocks
            // those rows are written once, and the zero rows between the blocks serve both:
            // [zt zeros][image rows][max(zt, zb) zeros][image rows][zb zeros].  For 31x31 on
            // 64-row planes that is 173 KB instead of 188 KB, which leaves room for more A
            // tables, and each TMA box carries 64 rows instead of 94.
            const int zt = p.py, zb = p.NR - p.py - p.Yi;
            const bool shz_ok = !nhwc && !no_shz && p.npanels == 1 && p.Yo <= p.P * p.NH && zt > 0 && zb > 0;
            bool fits = false;
            // The NHWC kernel keeps one B block (the cluster refills it) and two filter
            // buffers, or one when two do not fit.  The planar kernel takes two B blocks when
            // they fit and, for P = 2 with one sub-tile, 16 KB of epilogue staging boxes when
            // they fit as well; then, with A in shared memory, 6 down to 2 tables; then two
            // filter-line buffers when they fit as well.
            const bool stg_ok = !nhwc && p.P == 2 && p.XT == 1 && !no_tma_epi;
            const bool smem_a_ok = !nhwc && !no_a_smem && p.P == 2 && p.a_slots * 4 <= 128 * kMaxAPairs &&
                                   (p.NI >= 16 || force_a_smem);
            for (int amode = smem_a_ok ? 0 : 1; amode < 2 && !fits; ++amode) {
                p.a_smem = amode == 0 ? 1 : 0;
                p.nacc = p.a_smem ? 2 : 1;
                p.na = na_tmem;
                if (!p.a_smem && p.na < 2) break;
                const int n_na = p.a_smem ? kMaxA - 1 : 1;
                for (int opt = 0; opt < 8 * n_na && !fits; ++opt) {
                    // o: B blocks (o / 4), staging (o / 2 % 2), filter buffers (o % 2); with tables,
                    // their count runs between the (B blocks, staging) groups and the filter
                    // buffers: more tables before a second filter buffer (31x31 on B200: 6 tables
                    // with one buffer 106.4 us, 4 tables with two 107.0 us, 4 with one 108.3 us)
                    const int rem = opt % (2 * n_na);
                    const int o = (opt / (2 * n_na)) * 2 + rem % 2;
                    if (nhwc) {
                        if (o >= 2) break;
                        p.NB = 1;
                        p.nfb = 2 - o;
                        p.tma_epi = 0;
                    } else {
                        p.NB = kMaxB - o / 4;                   // B blocks: 2, then 1
                        p.tma_epi = stg_ok && (o / 2) % 2 == 0 ? 1 : 0;   // staging, then none
                        p.nfb = o % 2 == 0 ? 2 : 1;             // filter buffers: 2, then 1
                        if (!stg_ok && (o / 2) % 2 == 1) continue;   // the same layouts as the options before
                        if (p.a_smem) p.na = kMaxA - rem / 2;
                        if ((p.a_smem && p.na > max_na) || (one_fb && p.nfb == 2)) continue;
                    }
                    p.b_zt = 0;
                    p.b_rows = p.NR;
                    p.b_stride = p.b_bytes;
                    for (int z = 0; z < 3; ++z) p.z_off[z] = p.z_len[z] = 0;
                    p.f_off = static_cast<uint32_t>(p.NB) * p.b_bytes;
                    if (shz_ok && p.NB == 2) {
                        const uint32_t D = static_cast<uint32_t>(p.Yi), ut = static_cast<uint32_t>(zt),
                                       ub = static_cast<uint32_t>(zb), um = std::max(ut, ub);
                        p.b_zt = zt;
                        p.b_rows = p.Yi;
                        p.b_stride = (D + um) * 1024u;
                        p.z_off[0] = 0;
                        p.z_len[0] = ut * 1024u;
                        p.z_off[1] = (ut + D) * 1024u;
                        p.z_len[1] = um * 1024u;
                        p.z_off[2] = (ut + 2u * D + um) * 1024u;
                        p.z_len[2] = ub * 1024u;
                        p.f_off = (ut + 2u * D + um + ub) * 1024u;
                    }
                    p.bar_off = static_cast<uint32_t>(round_up(p.f_off + 4ull * p.nfb * p.f_words, 16));
                    size_t end = p.bar_off + (nhwc ? kNumBarsNhwc : kNumBars) * 8 + 16;
                    p.a_off = 0;
                    if (p.a_smem) {
                        // plus slack, so that the descriptor's addresses would stay inside the
                        // allocation even with its two strides exchanged
                        p.a_off = static_cast<uint32_t>(round_up(end, 128));
                        end = p.a_off + static_cast<size_t>(p.na) * p.a_bytes +
                              128u * (p.P - 1) * static_cast<size_t>(std::max(0, 16 - p.Ks / 8));
                    }
                    p.stg_off = 0;
                    p.nstg = 1;
                    if (p.tma_epi) {
                        p.stg_off = static_cast<uint32_t>(round_up(end, 1024));
                        end = p.stg_off + 2 * 8192;
                        // a second staging box per half when it fits beside everything else
                        if (end + 2 * 8192 + 1024 <= 227 * 1024 && !one_stg) {
                            p.nstg = 2;
                            end += 2 * 8192;
                        }
                    }
                    // At least 120 KB, so that one CTA runs per SM (each allocates all 512 TMEM columns).
                    p.smem = end + 1024;
                    if (p.smem < 120 * 1024) p.smem = 120 * 1024;
                    fits = p.smem <= 227 * 1024;
                }
            }
            if (!fits) continue;
            const long long num_yt = (p.Yo + p.P * p.NH - 1) / (p.P * p.NH);
            const long long num_xt = (p.Xo + p.XT * p.TW - 1) / (p.XT * p.TW);
            const long long units = num_xt * num_yt * ((a.N + 7) / 8) * a.C;
            const double rounds = static_cast<double>((units + kPlanSms - 1) / kPlanSms);
            const double cost = rounds * p.NI * p.XT * (p.Ks / 16) * (8.0 * p.NH);
            if (!have || cost < best_cost) {
                best = p;
                best_cost = cost;
                have = true;
            }
            break;   // first fitting shape of this orientation
        }
    }
    if (!have) return false;
    best.ws_in = round_up(static_cast<size_t>(a.C) * best.Yi * a.N * best.Xsi * 2, 256);
    best.ws_out = round_up(static_cast<size_t>(a.C) * best.Yo * a.N * best.Xso * 2, 256);
    best.ws_f = round_up(static_cast<size_t>(a.C) * best.f_words * 4, 256);
    // Split: with A tables (two accumulator sets, so a partial's write overlaps the next
    // tile's MMAs) the CTAs take equal ranges of shift steps, and the tiles two CTAs share
    // pass an fp32 partial through the workspace: one [set_cols][128] slot and one flag
    // per CTA, after the filter lines.
    const long long units = static_cast<long long>((best.Xo + best.XT * best.TW - 1) / (best.XT * best.TW)) *
                            ((best.Yo + best.P * best.NH - 1) / (best.P * best.NH)) * ((a.N + 7) / 8) * a.C;
    best.split = best.a_smem && best.tma_epi && !no_split ? 1 : 0;   // the split path stores staged boxes
    best.part_slots = best.split ? static_cast<int>(std::min<long long>(units, kPlanSms)) : 0;
    best.part_off = best.ws_f;
    if (best.split) {
        const size_t set_cols = static_cast<size_t>(best.XT) * 8 * best.NH;
        best.flag_off = best.part_off + round_up(static_cast<size_t>(best.part_slots) * 128 * set_cols * 4, 256);
        best.ws_f = best.flag_off + round_up(static_cast<size_t>(best.part_slots) * 4, 256);
    } else {
        best.flag_off = best.ws_f;
    }
    *out = best;
    return true;
}

cudaError_t launch_dw_toeplitz(const DwArgs& a, const ToepPlan& p, const ToepMaps& maps, void* ws, int num_sms,
                               cudaStream_t stream)
{
    const CUtensorMap& map_b = maps.b;
    // The MMA kernel's grid (one CTA per SM at most) and whether its CTAs split tiles:
    // only with more tiles than CTAs, so that no tile is shared by more than two CTAs.
    // DGRAD_TC_GRID=n caps the grid (testing: it makes small problems split).
    const long long units = static_cast<long long>((p.Xo + p.XT * p.TW - 1) / (p.XT * p.TW)) *
                            ((p.Yo + p.P * p.NH - 1) / (p.P * p.NH)) * ((a.N + 7) / 8) * a.C;
    if (units > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    int mma_grid = static_cast<int>(units < num_sms ? units : num_sms);
    if (const char* g = dgrad::tuning_env("DGRAD_TC_GRID")) {
        const int v = atoi(g);
        if (v > 0 && v < mma_grid) mma_grid = v;
    }
    const bool split = p.split && maps.tma_epi && units > mma_grid && mma_grid <= p.part_slots;
    float* part = split ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + p.ws_in + p.ws_out + p.part_off)
                        : nullptr;
    int* part_flag = split ? reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + p.ws_in + p.ws_out + p.flag_off)
                           : nullptr;
    const int nflags = split ? mma_grid : 0;
    const int tr_smem = (kTrStages + 2) * 8192 + kTrStages * 8 + 1024;
    if (maps.tma_transpose) {
        cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(dw_transpose_tma_kernel), tr_smem);
        if (e != cudaSuccess) return e;
    }
    static_assert(kPackThreads == 256, "the filter-packing CTAs share the transpose launch's block size");
    // with pack_to set, CTAs past the transposing ones pack the filter lines into it
    auto tma_transpose = [&](const CUtensorMap& src, const CUtensorMap& dst, bool to_planar, int Y, int X,
                             uint32_t* pack_to) {
        TrArgs t{};
        t.to_planar = to_planar ? 1 : 0;
        t.orient = p.orient;
        t.N = a.N;
        t.Y = Y;
        t.nxb = (X + 63) / 64;
        t.ncb = (a.C + 63) / 64;
        t.ntiles = a.N * Y * t.nxb * t.ncb;
        t.status = a.status;
        const int grid = t.ntiles < 4 * num_sms ? t.ntiles : 4 * num_sms;   // four CTAs per SM
        t.grid_tr = grid;
        int pack_blocks = 0;
        if (pack_to) {
            t.filt = static_cast<const __nv_bfloat16*>(a.filt);
            t.fpk = pack_to;
            t.C = a.C;
            t.KH = a.KH;
            t.KW = a.KW;
            t.KY = p.KY;
            t.KX = p.KX;
            t.half_l = p.half_l;
            t.f_words = p.f_words;
            t.pack_ncb = (a.C + 31) / 32;
            pack_blocks = t.pack_ncb * p.KY;
            t.part_flag = part_flag;
            t.nflags = nflags;
        }
        {
            const cudaError_t le_ = launch_kernel(dw_transpose_tma_kernel, dim3(grid + pack_blocks), dim3(256), tr_smem, stream, 1,
                                                 src, dst, t);
            if (le_ != cudaSuccess) return le_;
        }
        return cudaGetLastError();
    };
    if (a.N <= 0) return cudaSuccess;
    auto* dYp = static_cast<__nv_bfloat16*>(ws);
    auto* dXp = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + p.ws_in);
    auto* fpk = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + p.ws_in + p.ws_out);
    const int nct = (a.C + 63) / 64;
    const int64_t C = a.C;
    {
        // dY [N][Ho][Wo][C] -> [C][Yi][N][Xsi]
        const int64_t sN = static_cast<int64_t>(a.Ho) * a.Wo * C;
        const int64_t sY = p.orient ? C : static_cast<int64_t>(a.Wo) * C;
        const int64_t sX = p.orient ? static_cast<int64_t>(a.Wo) * C : C;
        cudaError_t e;
        if (maps.tma_transpose) {
            e = tma_transpose(maps.pack_src, maps.pack_dst, true, p.Yi, p.Xi, fpk);   // packs the filters too
        } else {
            dim3 grid(static_cast<unsigned>(((p.Xi + 63) / 64) * nct),
                      static_cast<unsigned>((p.Yi + kRowsPerCta - 1) / kRowsPerCta), static_cast<unsigned>(a.N));
            {
                const cudaError_t le_ = launch_kernel(dw_transpose_kernel<true>, dim3(grid), dim3(256), 0, stream, 1,
                                                     static_cast<const __nv_bfloat16*>(a.dY), dYp, a.N,
                                                                p.Yi, p.Xi, p.Xsi, a.C, sN, sY, sX,
                                                                static_cast<long long>(p.ws_in), a.status);
                if (le_ != cudaSuccess) return le_;
            }
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            dim3 fgrid(static_cast<unsigned>((a.C + 31) / 32), static_cast<unsigned>(p.KY));
            {
                const cudaError_t le_ = launch_kernel(dw_filter_pack_kernel, dim3(fgrid), dim3(kPackThreads), 0, stream, 1,
                                                     static_cast<const __nv_bfloat16*>(a.filt), fpk,
                                                                    a.C, a.KH, a.KW, p.KY, p.KX, p.orient, p.half_l,
                                                                    p.f_words, part_flag, nflags);
                if (le_ != cudaSuccess) return le_;
            }
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) return e;
    }
    {
        ToepArgs t{};
        t.fpack = fpk;
        t.dXp = dXp;
        t.status = a.status;
        t.N = a.N;
        t.C = a.C;
        t.Yo = p.Yo;
        t.Xo = p.Xo;
        t.Xso = p.Xso;
        t.KY = p.KY;
        t.py = p.py;
        t.px = p.px;
        t.P = p.P;
        t.TW = p.TW;
        t.XT = p.XT;
        t.NH = p.NH;
        t.Ks = p.Ks;
        t.NR = p.NR;
        t.NI = p.NI;
        t.half_l = p.half_l;
        t.NB = p.NB;
        t.num_xt = (p.Xo + p.XT * p.TW - 1) / (p.XT * p.TW);
        t.num_yt = (p.Yo + p.P * p.NH - 1) / (p.P * p.NH);
        t.num_g = (a.N + 7) / 8;
        t.num_units = static_cast<int>(units);
        t.split = split ? 1 : 0;
        t.part = part;
        t.part_flag = part_flag;
        t.a_col0 = p.a_col0;
        t.a_cols = p.a_cols;
        t.na = p.na;
        t.a_smem = p.a_smem;
        t.a_slots = p.a_slots;
        t.a_off = p.a_off;
        t.a_bytes = p.a_bytes;
        t.nacc = p.nacc;
        t.f16 = a.f16 ? 1 : 0;
        t.panel_bytes = p.panel_bytes;
        t.b_bytes = p.b_bytes;
        t.b_stride = p.b_stride;
        t.b_zt = p.b_zt;
        t.b_ld_off = static_cast<uint32_t>(p.b_zt) * 1024u;
        t.b_ld_bytes = static_cast<uint32_t>(p.b_rows) * 1024u * static_cast<uint32_t>(p.npanels);
        for (int z = 0; z < 3; ++z) {
            t.z_off[z] = p.z_off[z];
            t.z_len[z] = p.z_len[z];
        }
        t.npanels = static_cast<uint32_t>(p.npanels);
        t.f_words = static_cast<uint32_t>(p.f_words);
        t.f_bytes = static_cast<uint32_t>(p.f_words) * 4u;
        t.f_off = p.f_off;
        t.nfb = p.nfb;
        t.clip = p.clip;
        t.tma_epi = p.tma_epi && maps.tma_epi ? 1 : 0;
        t.stg_off = p.stg_off;
        t.nstg = p.nstg;
        t.bar_off = p.bar_off;
        t.dxp_bytes = static_cast<long long>(p.ws_out);
        cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(dw_toeplitz_kernel), static_cast<int>(p.smem));
        if (e != cudaSuccess) return e;
        e = launch_kernel(dw_toeplitz_kernel, dim3(mma_grid), dim3(kThreadsT), p.smem, stream, 1, map_b,
                          maps.tma_epi ? maps.d_store : map_b, t);
        if (e != cudaSuccess) return e;
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    {
        // [C][Yo][N][Xso] -> dX [N][H][W][C]
        const int64_t sN = static_cast<int64_t>(a.H) * a.W * C;
        const int64_t sY = p.orient ? C : static_cast<int64_t>(a.W) * C;
        const int64_t sX = p.orient ? static_cast<int64_t>(a.W) * C : C;
        if (maps.tma_transpose) {
            cudaError_t e = tma_transpose(maps.unpack_src, maps.unpack_dst, false, p.Yo, p.Xo, nullptr);
            if (e != cudaSuccess) return e;
        } else {
            dim3 grid(static_cast<unsigned>(((p.Xo + 63) / 64) * nct),
                      static_cast<unsigned>((p.Yo + kRowsPerCta - 1) / kRowsPerCta), static_cast<unsigned>(a.N));
            {
                const cudaError_t le_ = launch_kernel(dw_transpose_kernel<false>, dim3(grid), dim3(256), 0, stream, 1,
                                                     dXp, static_cast<__nv_bfloat16*>(a.dX), a.N, p.Yo,
                                                                 p.Xo, p.Xso, a.C, sN, sY, sX,
                                                                 static_cast<long long>(a.N) * a.H * a.W * a.C * 2,
                                                                 a.status);
                if (le_ != cudaSuccess) return le_;
            }
        }
    }
    return cudaGetLastError();
}

}  // namespace dgrad
