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
// B_i for every i lives in one shared-memory block: K-major core matrices of 8
// rows (yrow, img) x 8 columns j, rows in (yrow*8 + img) order, one block of NR
// rows per 8 columns.  Row (h', img) of B_i is row (2*h' + i, img), so B_i is
// that block seen through a descriptor whose start moves by 128 bytes per step
// and whose row-group stride is 256 bytes: one TMA load of the planar input per
// 8 columns serves every shift.  A_i is a 128 x K bf16 tile written by four warps
// straight into tensor memory (two buffers), so the MMA reads only B from
// shared memory.
//
// The planar input [C][Yi][N][Xs] (channels outermost, images between rows and
// columns) is written by dw_pack_kernel from NHWC dY, and the planar output by
// the MMA epilogue; dw_unpack_kernel writes it back to NHWC dX.  Both live in a
// caller workspace.
//
// Roles (320 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer of the B block (single buffer)
//   warp 1     TMEM allocation (512 columns) and the MMA issuer (one lane)
//   warps 2-5  A builders: filter lines staged in shared memory, each thread
//              writes its row of A_i with tcgen05.st
//   warps 6-9  epilogue: tcgen05.ld, round to bf16, planar stores
// Every wait is bounded; a timeout is recorded in the status word, raises the
// CTA's abort flag, lets issued copies and MMAs finish and frees TMEM.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kTW = 64;          // output columns per tile
constexpr int kP = 2;            // output-row phases stacked in M
constexpr int kThreadsT = 320;
constexpr int kOff = kTW + 8;    // offset of filter tap 0 in a padded filter line
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACol0 = 256; // first TMEM column of the A buffers

__host__ __device__ inline int floor8(int v) { return v >= 0 ? (v & ~7) : -((-v + 7) & ~7); }

struct ToepArgs {
    const __nv_bfloat16* filt;   // W [KH][KW][C]
    __nv_bfloat16* dXp;          // planar output [C][Yo][N][Xso]
    int* status;
    int N, C, Yo, Xo, Xso;
    int KH, KW, KY, KX, py, px, orient;
    int NH, K, NR, NI, L;
    int num_xt, num_yt, num_g, num_units;
    int a_cols;
    uint32_t b_bytes, f_off, bar_off;
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

__global__ void __launch_bounds__(kThreadsT, 1)
    dw_toeplitz_kernel(const __grid_constant__ CUtensorMap map_b, const __grid_constant__ ToepArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint8_t* bblk = smem;
    uint16_t* fpad = reinterpret_cast<uint16_t*>(smem + a.f_off);   // [2][KY][L]
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
    uint64_t* b_full = bars + 0;
    uint64_t* b_empty = bars + 1;
    uint64_t* a_full = bars + 2;    // [2]
    uint64_t* a_empty = bars + 4;   // [2]
    uint64_t* d_full = bars + 6;
    uint64_t* d_empty = bars + 7;
    uint64_t* drain = bars + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int kcols = a.K >> 3;
    const uint32_t nr_bytes = static_cast<uint32_t>(a.NR) * 128u;

    if (threadIdx.x == 0) {
        mbar_init(b_full, 1);
        mbar_init(b_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&a_full[b], 128);
            mbar_init(&a_empty[b], 1);
        }
        mbar_init(d_full, 1);
        mbar_init(d_empty, 128);
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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t ub = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < a.num_units; u += gridDim.x) {
                const Unit t = decode_unit(a, u);
                if (!mbar_wait(b_empty, (ub & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(b_full, a.b_bytes);
                for (int kk = 0; kk < kcols; ++kk)
                    tma_load_4d(bblk + kk * nr_bytes, &map_b, b_full, t.xb + 8 * kk, 8 * t.g, t.Y0 - a.py, t.c);
                ++ub;
            }
            if (!ok) {
                report_timeout(a.status);
                *abort_flag = 1;
            }
            if (ub > 0 && !mbar_wait(b_full, (ub - 1u) & 1u)) {   // the last copies have landed
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
            for (int u = blockIdx.x; u < a.num_units && ok; u += gridDim.x) {
                if (!mbar_wait(b_full, ub & 1u, abort_flag) || !mbar_wait(d_empty, (ub & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int i = 0; i < a.NI; ++i) {
                    const uint32_t b = step & 1u;
                    if (!mbar_wait(&a_full[b], (step >> 1) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem_base + kACol0 + b * static_cast<uint32_t>(a.a_cols);
                    for (int q = 0; q < (a.K >> 4); ++q) {
                        const uint64_t bdesc =
                            noswz_desc(b_addr + static_cast<uint32_t>(2 * q) * nr_bytes + static_cast<uint32_t>(i) * 128u,
                                       nr_bytes, kP * 128u);
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
        const int tid = threadIdx.x - 64;   // 0 .. 127
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        uint16_t* fp0 = fpad;
        uint16_t* fp1 = fpad + a.KY * a.L;
        uint32_t step = 0;
        int prev_c = -1;
        bool ok = true;
        // Every builder walks every unit, even after a failed wait, so that all
        // 128 threads meet the same sequence of named barriers.
        for (int u = blockIdx.x; u < a.num_units; u += gridDim.x) {
            const Unit t = decode_unit(a, u);
            if (t.c != prev_c) {
                named_barrier_sync(1, 128);   // every builder is done with the previous filter
                const int total = 2 * a.KY * a.L;
                for (int idx = tid; idx < total; idx += 128) {
                    const int copy = idx >= a.KY * a.L ? 1 : 0;
                    const int rem = idx - copy * a.KY * a.L;
                    const int ry = rem / a.L;
                    const int rx = rem - ry * a.L + copy - kOff;
                    uint16_t v = 0;
                    if (rx >= 0 && rx < a.KX) {
                        const int r = a.orient ? (a.KH - 1 - rx) : (a.KH - 1 - ry);
                        const int s = a.orient ? (a.KW - 1 - ry) : (a.KW - 1 - rx);
                        v = __ldg(reinterpret_cast<const unsigned short*>(a.filt) +
                                  (static_cast<int64_t>(r) * a.KW + s) * a.C + t.c);
                    }
                    fpad[idx] = v;
                }
                named_barrier_sync(1, 128);
                prev_c = t.c;
            }
            // A_i[m][j] = F[i-p][j + e], e = xb - x0 + px - xl; padded index t0 = e + kOff >= 0.
            const int t0 = t.xb - t.x0 + a.px - xl + kOff;
            const uint16_t* rowbase = (t0 & 1) ? (fp1 + t0 - 1) : (fp0 + t0);
            for (int i = 0; i < a.NI && ok; ++i) {
                const uint32_t b = step & 1u;
                if (!mbar_wait(&a_empty[b], ((step >> 1) & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int ry = i - p;
                const uint32_t taddr = tmem_base + lane_addr + kACol0 + b * static_cast<uint32_t>(a.a_cols);
                if (ry >= 0 && ry < a.KY) {
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(rowbase + ry * a.L);
                    for (int q = 0; q < (a.K >> 4); ++q) {
                        uint32_t v[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) v[k] = src[q * 8 + k];
                        tmem_st_32x32b_x8(taddr + 8u * q, v);
                    }
                } else {
                    uint32_t z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                    for (int q = 0; q < (a.K >> 4); ++q) tmem_st_32x32b_x8(taddr + 8u * q, z);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&a_full[b]);
                ++step;
            }
        }
        if (!ok) {
            report_timeout(a.status);
            *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int m = quarter * 32 + lane;
        const int p = m / kTW;
        const int xl = m % kTW;
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        const int nchunks = (8 * a.NH) / 32;
        uint32_t ub = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < a.num_units; u += gridDim.x) {
            const Unit t = decode_unit(a, u);
            if (!mbar_wait(d_full, ub & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int x = t.x0 + xl;
            const bool xok = x < a.Xo;
            for (int cc = 0; cc < nchunks; ++cc) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(cc * 32), v);
                tmem_wait_ld();
                if (cc == nchunks - 1) {
                    tc_fence_before();
                    mbar_arrive(d_empty);   // accumulator may be overwritten now
                }
                if (xok) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int n = cc * 32 + k;
                        const int y = t.Y0 + kP * (n >> 3) + p;
                        const int img = 8 * t.g + (n & 7);
                        if (y < a.Yo && img < a.N) {
                            const __nv_bfloat16 o = __float2bfloat16_rn(__uint_as_float(v[k]));
                            a.dXp[((static_cast<int64_t>(t.c) * a.Yo + y) * a.N + img) * a.Xso + x] = o;
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
        p.NI = p.KY + kP - 1;
        p.L = p.K + kOff + 8;
        p.a_cols = ((p.K / 2) + 31) & ~31;
        if (kACol0 + 2 * p.a_cols > kTmemCols) continue;
        bool fits = false;
        for (int nh : {32, 16}) {
            p.NH = nh;
            p.NR = kP * nh - 1 + p.KY;
            if (p.NR > 256) continue;
            p.b_bytes = static_cast<uint32_t>((p.K / 8) * p.NR * 128);
            p.f_off = static_cast<uint32_t>(round_up(p.b_bytes, 128));
            p.bar_off = static_cast<uint32_t>(round_up(p.f_off + 2ull * p.KY * p.L * 2, 16));
            // At least 120 KB, so that one CTA runs per SM (each allocates all 512 TMEM columns).
            p.smem = p.bar_off + 9 * 8 + 16 + 1024;
            if (p.smem < 120 * 1024) p.smem = 120 * 1024;
            if (p.smem <= 227 * 1024) {
                fits = true;
                break;
            }
        }
        if (!fits) continue;
        const int num_yt = (p.Yo + kP * p.NH - 1) / (kP * p.NH);
        const int num_xt = (p.Xo + kTW - 1) / kTW;
        // MMA work per channel-image: tiles x shift steps x K x N x M
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
    *out = best;
    return true;
}

cudaError_t launch_dw_toeplitz(const DwArgs& a, const ToepPlan& p, const CUtensorMap& map_b, void* ws,
                               int num_sms, cudaStream_t stream)
{
    if (a.N <= 0) return cudaSuccess;
    auto* dYp = static_cast<__nv_bfloat16*>(ws);
    auto* dXp = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + p.ws_in);
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
    }
    {
        ToepArgs t{};
        t.filt = static_cast<const __nv_bfloat16*>(a.filt);
        t.dXp = dXp;
        t.status = a.status;
        t.N = a.N;
        t.C = a.C;
        t.Yo = p.Yo;
        t.Xo = p.Xo;
        t.Xso = p.Xso;
        t.KH = a.KH;
        t.KW = a.KW;
        t.KY = p.KY;
        t.KX = p.KX;
        t.py = p.py;
        t.px = p.px;
        t.orient = p.orient;
        t.NH = p.NH;
        t.K = p.K;
        t.NR = p.NR;
        t.NI = p.NI;
        t.L = p.L;
        t.num_xt = (p.Xo + kTW - 1) / kTW;
        t.num_yt = (p.Yo + kP * p.NH - 1) / (kP * p.NH);
        t.num_g = (a.N + 7) / 8;
        const long long units = static_cast<long long>(t.num_xt) * t.num_yt * t.num_g * a.C;
        if (units > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
        t.num_units = static_cast<int>(units);
        t.a_cols = p.a_cols;
        t.b_bytes = p.b_bytes;
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
