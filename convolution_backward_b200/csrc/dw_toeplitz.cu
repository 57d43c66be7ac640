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
// columns serves every shift.  A_i is a 128 x K bf16 tile written by four warps
// straight into tensor memory (up to four buffers), so the MMA reads only B
// from shared memory.  The A builders read the channel's filter lines, padded
// with zeros and packed two taps per word, from shared memory; the producer
// brings them in with one bulk copy whenever the channel changes.
//
// Three helper kernels run around the MMA kernel, all through the caller's
// workspace: dw_pack_kernel writes NHWC dY as planes [C][Yi][N][Xs] (channels
// outermost, images between rows and columns), dw_filter_pack_kernel writes the
// padded filter lines of every channel, and dw_unpack_kernel writes the planar
// output of the MMA epilogue back to NHWC dX.
//
// Roles (448 threads, one CTA per SM, a contiguous range of tiles per CTA so
// that the image groups of one channel follow each other):
//   warp 0      producer: filter lines (bulk copy) and B panels (TMA)
//   warp 1      TMEM allocation (512 columns) and the MMA issuer (one lane)
//   warps 2-5   A builders: each thread writes its row of A_i with tcgen05.st
//   warps 6-13  epilogue: two warps per TMEM lane quarter drain the accumulator
//               into registers, release it, then round to bf16 and store planes
// Every wait is bounded; a timeout is recorded in the status word, raises the
// CTA's abort flag, lets issued copies and MMAs finish and frees TMEM.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kTW = 64;          // output columns per tile
constexpr int kP = 2;            // output-row phases stacked in M
constexpr int kThreadsT = 448;   // 14 warps: producer, MMA, 4 A builders, 8 epilogue
constexpr int kOff = kTW + 8;    // offset of filter tap 0 in a padded filter line
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxA = 4;         // A buffers in tensor memory
constexpr int kNumBars = 2 + 2 * kMaxA + 5;

__host__ __device__ inline int floor8(int v) { return v >= 0 ? (v & ~7) : -((-v + 7) & ~7); }

struct ToepArgs {
    const uint32_t* fpack;       // padded filter lines, f_words per channel
    __nv_bfloat16* dXp;          // planar output [C][Yo][N][Xso]
    int* status;
    int N, C, Yo, Xo, Xso;
    int KY, py, px;
    int NH, K, NR, NI, half_l;
    int num_xt, num_yt, num_g, num_units;
    int a_col0, a_cols, na;      // TMEM column of A buffer 0, columns per buffer, buffer count
    uint32_t panel_bytes, b_bytes, f_bytes, f_words, f_off, bar_off;
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
    t.Y0 = yt * kP * a.NH;
    t.x0 = xt * kTW;
    t.xb = floor8(t.x0 - a.px);
    return t;
}

// One thread's row of A_i: taps t0 .. t0 + 2*KQ*8 - 1 of a padded filter line
// (word w holds taps 2w, 2w+1), i.e. KQ*8 words starting at word t0/2, shifted by
// one tap when t0 is odd; then written to tensor memory 8 columns at a time.
template <int KQ>
__device__ __forceinline__ void store_a_row(uint32_t taddr, const uint32_t* src, bool odd, bool nonzero)
{
    uint32_t v[KQ * 8 + 1];
#pragma unroll
    for (int k = 0; k < KQ * 8 + 1; ++k) v[k] = nonzero ? src[k] : 0u;
#pragma unroll
    for (int q = 0; q < KQ; ++q) {
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = odd ? __funnelshift_r(v[q * 8 + k], v[q * 8 + k + 1], 16) : v[q * 8 + k];
        tmem_st_32x32b_x8(taddr + 8u * q, w);
    }
}

__device__ __forceinline__ void store_a(int kq, uint32_t taddr, const uint32_t* src, bool odd, bool nonzero)
{
    switch (kq) {
    case 4: store_a_row<4>(taddr, src, odd, nonzero); break;
    case 5: store_a_row<5>(taddr, src, odd, nonzero); break;
    case 6: store_a_row<6>(taddr, src, odd, nonzero); break;
    case 7: store_a_row<7>(taddr, src, odd, nonzero); break;
    case 8: store_a_row<8>(taddr, src, odd, nonzero); break;
    default: store_a_row<9>(taddr, src, odd, nonzero); break;
    }
}

// Units [u_begin, u_end) of this CTA: a contiguous range, so that the image
// groups of one channel follow each other and share one filter load.
__device__ __forceinline__ void unit_range(const ToepArgs& a, int* u_begin, int* u_end)
{
    *u_begin = static_cast<int>((static_cast<long long>(blockIdx.x) * a.num_units) / gridDim.x);
    *u_end = static_cast<int>((static_cast<long long>(blockIdx.x + 1) * a.num_units) / gridDim.x);
}

__global__ void __launch_bounds__(kThreadsT, 1)
    dw_toeplitz_kernel(const __grid_constant__ CUtensorMap map_b, const __grid_constant__ ToepArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint8_t* bblk = smem;                                               // B panels (128-byte swizzle)
    uint32_t* fwords = reinterpret_cast<uint32_t*>(smem + a.f_off);     // padded filter lines
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* b_full = bars + 0;
    uint64_t* b_empty = bars + 1;
    uint64_t* a_full = bars + 2;              // [kMaxA]
    uint64_t* a_empty = bars + 2 + kMaxA;     // [kMaxA]
    uint64_t* d_full = bars + 2 + 2 * kMaxA;
    uint64_t* d_empty = d_full + 1;
    uint64_t* f_full = d_full + 2;
    uint64_t* f_empty = d_full + 3;
    uint64_t* drain = d_full + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t na = static_cast<uint32_t>(a.na);
    int u_begin, u_end;
    unit_range(a, &u_begin, &u_end);

    if (threadIdx.x == 0) {
        mbar_init(b_full, 1);
        mbar_init(b_empty, 1);
        for (int b = 0; b < kMaxA; ++b) {
            mbar_init(&a_full[b], 128);
            mbar_init(&a_empty[b], 1);
        }
        mbar_init(d_full, 1);
        mbar_init(d_empty, 256);
        mbar_init(f_full, 1);
        mbar_init(f_empty, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&map_b);
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
        // Per unit: the filter lines when the channel changes (one bulk copy),
        // then the B panels (one TMA box per 64 columns).
        if (lane == 0) {
            uint32_t ub = 0, fe = 0;
            int prev_c = -1;
            bool ok = true;
            for (int u = u_begin; u < u_end; ++u) {
                const Unit t = decode_unit(a, u);
                if (t.c != prev_c) {
                    if (!mbar_wait(f_empty, (fe & 1u) ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(f_full, a.f_bytes);
                    bulk_load(fwords, a.fpack + static_cast<int64_t>(t.c) * a.f_words, a.f_bytes, f_full);
                    ++fe;
                    prev_c = t.c;
                }
                if (!mbar_wait(b_empty, (ub & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(b_full, a.b_bytes);
                for (int pn = 0; pn * 64 < a.K; ++pn)
                    tma_load_4d(bblk + pn * a.panel_bytes, &map_b, b_full, t.xb + 64 * pn, 8 * t.g, t.Y0 - a.py, t.c);
                ++ub;
            }
            if (!ok) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
            // the last copies have landed before the CTA may exit
            if (ub > 0 && !mbar_wait(b_full, (ub - 1u) & 1u)) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
            if (fe > 0 && !mbar_wait(f_full, (fe - 1u) & 1u)) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, 8 * a.NH, /*b_mn_major=*/false);
            const uint32_t b_addr = smem_u32(bblk);
            uint32_t ub = 0, step = 0;
            bool ok = true;
            for (int u = u_begin; u < u_end && ok; ++u) {
                if (!mbar_wait(b_full, ub & 1u, abort_flag) || !mbar_wait(d_empty, (ub & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int i = 0; i < a.NI; ++i) {
                    const uint32_t b = step % na;
                    if (!mbar_wait(&a_full[b], (step / na) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_tmem =
                        tmem_base + static_cast<uint32_t>(a.a_col0) + b * static_cast<uint32_t>(a.a_cols);
                    // B_i: rows (h', img) are panel rows (2h' + i, img); one shift step is one
                    // 1024-byte swizzle atom, the row-group stride two atoms.
                    for (int q = 0; q < (a.K >> 4); ++q) {
                        const uint32_t start = b_addr + static_cast<uint32_t>(q >> 2) * a.panel_bytes +
                                               static_cast<uint32_t>(i) * 1024u + static_cast<uint32_t>(q & 3) * 32u;
                        const uint64_t bdesc = sw128_desc(start, 16, kP * 1024u);
                        umma_f16_ts(tmem_base, a_tmem + 8u * q, bdesc, idesc, (i | q) != 0 ? 1u : 0u);
                    }
                    umma_commit(&a_empty[b]);   // A buffer free once these MMAs have read it
                    ++step;
                }
                if (!ok) break;
                umma_commit(d_full);
                umma_commit(b_empty);
                ++ub;
            }
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
        const int p = m / kTW;
        const int xl = m % kTW;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint32_t step = 0, fe = 0;
        int prev_c = -1;
        bool ok = true;
        for (int u = u_begin; u < u_end && ok; ++u) {
            const Unit t = decode_unit(a, u);
            if (t.c != prev_c) {
                if (!mbar_wait(f_full, fe & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                ++fe;
                prev_c = t.c;
            }
            // A_i[m][j] = F[i-p][j + e], e = xb - x0 + px - xl; padded tap index t0 = e + kOff >= 0.
            const int t0 = t.xb - t.x0 + a.px - xl + kOff;
            const uint32_t* rowbase = fwords + (t0 >> 1);
            const bool odd = (t0 & 1) != 0;
            for (int i = 0; i < a.NI; ++i) {
                const uint32_t b = step % na;
                if (!mbar_wait(&a_empty[b], ((step / na) & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int ry = i - p;
                const uint32_t taddr =
                    tmem_base + lane_addr + static_cast<uint32_t>(a.a_col0) + b * static_cast<uint32_t>(a.a_cols);
                const bool nonzero = ry >= 0 && ry < a.KY;
                store_a(a.K >> 4, taddr, rowbase + (nonzero ? ry : 0) * a.half_l, odd, nonzero);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&a_full[b]);
                ++step;
            }
            // Done with this channel's filter lines: let the producer replace them.
            const bool last = u + 1 >= u_end || decode_unit(a, u + 1).c != t.c;
            if (ok && last) mbar_arrive(f_empty);
        }
        if (!ok) {
            report_timeout(a.status);
            *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------- epilogue
        // Two warps per TMEM lane quarter, each draining half of the columns into
        // registers (as bf16 pairs) before releasing the accumulator.
        const int quarter = warp & 3;
        const int half = (warp - 6) >> 2;
        const int m = quarter * 32 + lane;
        const int p = m / kTW;
        const int xl = m % kTW;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const int ncol = 4 * a.NH;          // columns per half: 128 or 64
        const int nch = ncol >> 5;          // 32-column chunks per half: 4 or 2
        const int64_t img_stride = a.Xso;
        const int64_t hrow_stride = static_cast<int64_t>(kP) * a.N * a.Xso;
        uint32_t ub = 0;
        bool ok = true;
        for (int u = u_begin; u < u_end; ++u) {
            const Unit t = decode_unit(a, u);
            if (!mbar_wait(d_full, ub & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t pk[64];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                if (cc < nch) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(half * ncol + cc * 32), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        pk[cc * 16 + k] = float2_to_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                }
            }
            tc_fence_before();
            mbar_arrive(d_empty);   // the accumulator may be overwritten now
            const int x = t.x0 + xl;
            if (x < a.Xo) {
                // column n = half*ncol + k: h' = n >> 3, image 8g + (n & 7), row Y0 + 2h' + p
                const int hp0 = (half * ncol) >> 3;
                uint16_t* base = reinterpret_cast<uint16_t*>(a.dXp) +
                                 ((static_cast<int64_t>(t.c) * a.Yo + t.Y0 + kP * hp0 + p) * a.N + 8 * t.g) * a.Xso + x;
                const bool full = t.Y0 + kP * a.NH <= a.Yo && 8 * t.g + 8 <= a.N;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    if (cc < nch) {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const int kk = cc * 32 + 2 * k;        // column within the half (even)
                            const int hp = kk >> 3;
                            const int img = kk & 7;
                            uint16_t* dst = base + hp * hrow_stride + img * img_stride;
                            const uint32_t v = pk[cc * 16 + k];
                            if (full) {
                                dst[0] = static_cast<uint16_t>(v & 0xFFFFu);
                                dst[img_stride] = static_cast<uint16_t>(v >> 16);
                            } else if (t.Y0 + kP * (hp0 + hp) + p < a.Yo) {
                                if (8 * t.g + img < a.N) dst[0] = static_cast<uint16_t>(v & 0xFFFFu);
                                if (8 * t.g + img + 1 < a.N) dst[img_stride] = static_cast<uint16_t>(v >> 16);
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
// word w of a line holds taps (2w - kOff, 2w + 1 - kOff).  f_words words per channel.
__global__ void __launch_bounds__(128)
    dw_filter_pack_kernel(const __nv_bfloat16* __restrict__ filt, uint32_t* __restrict__ dst, int C, int KH, int KW,
                          int KY, int KX, int orient, int half_l, int f_words)
{
    const int c = blockIdx.x;
    const unsigned short* w16 = reinterpret_cast<const unsigned short*>(filt);
    for (int idx = threadIdx.x; idx < f_words; idx += blockDim.x) {
        uint32_t packed = 0;
        const int ry = idx / half_l;
        const int w = idx - ry * half_l;
        if (ry < KY) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int rx = 2 * w + h - kOff;
                if (rx >= 0 && rx < KX) {
                    const int r = orient ? (KH - 1 - rx) : (KH - 1 - ry);
                    const int s = orient ? (KW - 1 - ry) : (KW - 1 - rx);
                    packed |= static_cast<uint32_t>(w16[(static_cast<int64_t>(r) * KW + s) * C + c]) << (16 * h);
                }
            }
        }
        dst[static_cast<int64_t>(c) * f_words + idx] = packed;
    }
}

// NHWC -> planar [C][Y][N][Xs]: element (n, y, x, c) of the source sits at
// n*sN + y*sY + x*sX + c.  One CTA moves a 64 (x) x 64 (c) tile of one (n, y).
__global__ void __launch_bounds__(256)
    dw_pack_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int N, int Y, int X,
                   int Xs, int C, int64_t sN, int64_t sY, int64_t sX)
{
    __shared__ uint32_t tile[64][33];   // [x][c pair]
    const int nct = (C + 63) >> 6;
    const int ct = blockIdx.x % nct;
    const int xt = blockIdx.x / nct;
    const int y = blockIdx.y;
    const int n = blockIdx.z;
    const int c0 = ct * 64;
    const int x0 = xt * 64;
    for (int idx = threadIdx.x; idx < 512; idx += 256) {
        const int xr = idx >> 3;
        const int cc = (idx & 7) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (x0 + xr < X && c0 + cc < C)
            v = *reinterpret_cast<const uint4*>(src + n * sN + y * sY + static_cast<int64_t>(x0 + xr) * sX + c0 + cc);
        tile[xr][cc / 2 + 0] = v.x;
        tile[xr][cc / 2 + 1] = v.y;
        tile[xr][cc / 2 + 2] = v.z;
        tile[xr][cc / 2 + 3] = v.w;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 512; idx += 256) {
        const int cr = idx >> 3;
        const int xc = (idx & 7) * 8;
        const int c = c0 + cr;
        const int x = x0 + xc;
        if (c >= C || x >= X) continue;
        const int sh = (cr & 1) * 16;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t lo = (tile[xc + 2 * k][cr >> 1] >> sh) & 0xFFFFu;
            const uint32_t hi = (tile[xc + 2 * k + 1][cr >> 1] >> sh) & 0xFFFFu;
            w[k] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4*>(dst + ((static_cast<int64_t>(c) * Y + y) * N + n) * Xs + x) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// planar [C][Y][N][Xs] -> NHWC (inverse of dw_pack_kernel).
__global__ void __launch_bounds__(256)
    dw_unpack_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int N, int Y, int X,
                     int Xs, int C, int64_t sN, int64_t sY, int64_t sX)
{
    __shared__ uint32_t tile[64][33];   // [c][x pair]
    const int nct = (C + 63) >> 6;
    const int ct = blockIdx.x % nct;
    const int xt = blockIdx.x / nct;
    const int y = blockIdx.y;
    const int n = blockIdx.z;
    const int c0 = ct * 64;
    const int x0 = xt * 64;
    for (int idx = threadIdx.x; idx < 512; idx += 256) {
        const int cr = idx >> 3;
        const int xc = (idx & 7) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (c0 + cr < C && x0 + xc < X)
            v = *reinterpret_cast<const uint4*>(src + ((static_cast<int64_t>(c0 + cr) * Y + y) * N + n) * Xs + x0 + xc);
        tile[cr][xc / 2 + 0] = v.x;
        tile[cr][xc / 2 + 1] = v.y;
        tile[cr][xc / 2 + 2] = v.z;
        tile[cr][xc / 2 + 3] = v.w;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 512; idx += 256) {
        const int xr = idx >> 3;
        const int cc = (idx & 7) * 8;
        const int x = x0 + xr;
        const int c = c0 + cc;
        if (x >= X || c >= C) continue;
        const int sh = (xr & 1) * 16;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t lo = (tile[cc + 2 * k][xr >> 1] >> sh) & 0xFFFFu;
            const uint32_t hi = (tile[cc + 2 * k + 1][xr >> 1] >> sh) & 0xFFFFu;
            w[k] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4*>(dst + n * sN + y * sY + static_cast<int64_t>(x) * sX + c) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool plan_dw_toeplitz(const DwArgs& a, ToepPlan* out)
{
    if (!a.bf16 || a.S != 1) return false;
    bool have = false;
    ToepPlan best{};
    long long best_cost = 0;
    for (int orient = 0; orient < 2; ++orient) {
        ToepPlan p{};
        p.orient = orient;
        p.KY = orient ? a.KW : a.KH;
        p.KX = orient ? a.KH : a.KW;
        p.py = orient ? (a.KW - 1 - a.pw) : (a.KH - 1 - a.ph);
        p.px = orient ? (a.KH - 1 - a.ph) : (a.KW - 1 - a.pw);
        p.Yi = orient ? a.Wo : a.Ho;
        p.Xi = orient ? a.Ho : a.Wo;
        p.Yo = orient ? a.W : a.H;
        p.Xo = orient ? a.H : a.W;
        p.Xsi = (p.Xi + 7) & ~7;
        p.Xso = (p.Xo + 7) & ~7;
        const int mis = (-p.px) - floor8(-p.px);
        p.K = (kTW + p.KX - 1 + mis + 15) & ~15;
        if (p.K > 144) continue;
        p.NI = p.KY + kP - 1;
        p.half_l = (p.K + kOff + 8) / 2;     // words per padded filter line
        p.f_words = static_cast<int>(round_up(static_cast<size_t>(p.KY) * p.half_l, 4));
        p.a_cols = ((p.K / 2) + 31) & ~31;
        const int panels = (p.K + 63) / 64;
        bool fits = false;
        for (int nh : {32, 16}) {
            p.NH = nh;
            p.NR = kP * nh - 1 + p.KY;
            if (p.NR > 256) continue;
            p.a_col0 = 8 * nh;                               // the accumulator takes columns [0, 8*NH)
            p.na = (static_cast<int>(kTmemCols) - p.a_col0) / p.a_cols;
            if (p.na < 2) continue;
            if (p.na > kMaxA) p.na = kMaxA;
            p.panel_bytes = static_cast<uint32_t>(p.NR) * 1024u;
            p.b_bytes = static_cast<uint32_t>(panels) * p.panel_bytes;
            p.f_off = p.b_bytes;
            p.bar_off = static_cast<uint32_t>(round_up(p.f_off + 4ull * p.f_words, 16));
            // At least 120 KB, so that one CTA runs per SM (each allocates all 512 TMEM columns).
            p.smem = p.bar_off + kNumBars * 8 + 16 + 1024;
            if (p.smem < 120 * 1024) p.smem = 120 * 1024;
            if (p.smem <= 227 * 1024) {
                fits = true;
                break;
            }
        }
        if (!fits) continue;
        const int num_yt = (p.Yo + kP * p.NH - 1) / (kP * p.NH);
        const int num_xt = (p.Xo + kTW - 1) / kTW;
        // MMA work per channel-image: tiles x shift steps x K x N
        const long long cost = static_cast<long long>(num_yt) * num_xt * p.NI * p.K * p.NH;
        if (!have || cost < best_cost) {
            best = p;
            best_cost = cost;
            have = true;
        }
    }
    if (!have) return false;
    best.ws_in = round_up(static_cast<size_t>(a.C) * best.Yi * a.N * best.Xsi * 2, 256);
    best.ws_out = round_up(static_cast<size_t>(a.C) * best.Yo * a.N * best.Xso * 2, 256);
    best.ws_f = round_up(static_cast<size_t>(a.C) * best.f_words * 4, 256);
    *out = best;
    return true;
}

cudaError_t launch_dw_toeplitz(const DwArgs& a, const ToepPlan& p, const CUtensorMap& map_b, void* ws,
                               int num_sms, cudaStream_t stream)
{
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
        dim3 grid(static_cast<unsigned>(((p.Xi + 63) / 64) * nct), static_cast<unsigned>(p.Yi),
                  static_cast<unsigned>(a.N));
        dw_pack_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(a.dY), dYp, a.N, p.Yi, p.Xi,
                                                 p.Xsi, a.C, sN, sY, sX);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        dw_filter_pack_kernel<<<a.C, 128, 0, stream>>>(static_cast<const __nv_bfloat16*>(a.filt), fpk, a.C, a.KH,
                                                       a.KW, p.KY, p.KX, p.orient, p.half_l, p.f_words);
        e = cudaGetLastError();
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
        t.NH = p.NH;
        t.K = p.K;
        t.NR = p.NR;
        t.NI = p.NI;
        t.half_l = p.half_l;
        t.num_xt = (p.Xo + kTW - 1) / kTW;
        t.num_yt = (p.Yo + kP * p.NH - 1) / (kP * p.NH);
        t.num_g = (a.N + 7) / 8;
        const long long units = static_cast<long long>(t.num_xt) * t.num_yt * t.num_g * a.C;
        if (units > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
        t.num_units = static_cast<int>(units);
        t.a_col0 = p.a_col0;
        t.a_cols = p.a_cols;
        t.na = p.na;
        t.panel_bytes = p.panel_bytes;
        t.b_bytes = p.b_bytes;
        t.f_words = static_cast<uint32_t>(p.f_words);
        t.f_bytes = static_cast<uint32_t>(p.f_words) * 4u;
        t.f_off = p.f_off;
        t.bar_off = p.bar_off;
        cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(dw_toeplitz_kernel), static_cast<int>(p.smem));
        if (e != cudaSuccess) return e;
        const int grid = static_cast<int>(units < num_sms ? units : num_sms);
        dw_toeplitz_kernel<<<grid, kThreadsT, p.smem, stream>>>(map_b, t);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    {
        // [C][Yo][N][Xso] -> dX [N][H][W][C]
        const int64_t sN = static_cast<int64_t>(a.H) * a.W * C;
        const int64_t sY = p.orient ? C : static_cast<int64_t>(a.W) * C;
        const int64_t sX = p.orient ? static_cast<int64_t>(a.W) * C : C;
        dim3 grid(static_cast<unsigned>(((p.Xo + 63) / 64) * nct), static_cast<unsigned>(p.Yo),
                  static_cast<unsigned>(a.N));
        dw_unpack_kernel<<<grid, 256, 0, stream>>>(dXp, static_cast<__nv_bfloat16*>(a.dX), a.N, p.Yo, p.Xo, p.Xso,
                                                   a.C, sN, sY, sX);
    }
    return cudaGetLastError();
}

}  // namespace dgrad
