// dense_tc.cu -- dense and grouped KH x KW dgrad on the Blackwell tensor cores.
//
// dX[n,h,w,c] = sum over (ho,wo,k,r,s) with h = ho*S - pad_h + r, w = wo*S -
// pad_w + s and k in c's group of dY[n,ho,wo,k] * W[r][s][k][c - group base]
// (G groups of Kg dY and Cg dX channels; W is [KH][KW][K][Cg], G = 1 dense).
// Each group is its own GEMM: dY is seen as a 5-D tensor (Kg, G, Wo, Ho, N) and
// W as (Cg, Kg, G, KH*KW), so the zero fill of the TMA boxes stops every k-block
// and channel tile at its group's edge.  Split by output phase (the
// pages' sub-pixel decomposition of strided dgrad into S*S sub-GEMMs, "add the
// pointwise fast path dgrad was missing", Technical Details): for a = (h +
// pad_h) mod S and b = (w + pad_w) mod S, the rows h = S*hq + a - pad_h and
// columns w = S*wq + b - pad_w receive exactly the taps r = a + S*t, s = b + S*u,
// from dY[n, hq - t, wq - u, :].  So each phase is a sum over its taps of GEMMs
//     D[(hq,wq)][c] += dY[n, hq - t, wq - u][k] * W[a + S*t][b + S*u][k][c],
// whose A operand is dY shifted by (t, u): a 4-D TMA box at an offset
// coordinate, with the tensor's zero fill supplying the padding.  Stride 1 is
// the single phase (0, 0).  No im2col buffer, no gather.
//
// Tile: 128 positions = 8 rows hq x 16 columns wq of one phase of one image
// (M), BN channels of one group (N); K-loop over the phase's taps x 64-deep
// k-blocks of the group.  bf16 or f16 operands (same type for A and B), fp32
// accumulation, output in the input type.
// Kernel structure as the streaming pointwise kernel (persistent, one CTA per
// SM, 192 threads): warp 0 TMA producer (A box 64 k x 16 wq x 8 hq, W box BN c x
// 64 k, 128-byte swizzle), warp 1 TMEM allocation and MMA issue (M = 128, N =
// BN, K = 16) into two accumulators, warps 2-5 epilogue (tcgen05.ld, round to
// bf16, 16-byte stores to the positions the phase owns).  Every wait is
// bounded; a timeout is recorded in the status word and the kernel winds down.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr int kTH = 8;    // tile rows (hq)
constexpr int kTW = 16;   // tile columns (wq)

template <int BN, int STAGES>
struct DenseLayout {
    static constexpr int kABytes = kBM * kBK * 2;   // 16 KB
    static constexpr int kBBytes = kBK * BN * 2;    // 8 KB per 64 columns
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kTileBytes = STAGES * kStageBytes;
    static constexpr int kNumBars = 2 * STAGES + 5;
    static constexpr int kBytes = kTileBytes + kNumBars * 8 + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr uint32_t kTmemCols = 2 * BN;
};

// One tile: image n, phase (a, b), first hq / wq, group g, first channel of the group.
struct DTile {
    int n, a, b, hq0, wq0, g, c0, nt, nu;
};

__device__ __forceinline__ DTile decode_tile(const DenseArgs& d, int t, int bn)
{
    DTile r;
    const int ct = t % d.nc;
    int q = t / d.nc;
    r.g = q % d.G;
    q /= d.G;
    const int wt = q % d.ntw;
    q /= d.ntw;
    const int ht = q % d.nth;
    q /= d.nth;
    const int ph = q % (d.S * d.S);
    r.n = q / (d.S * d.S);
    r.a = ph / d.S;
    r.b = ph % d.S;
    r.hq0 = d.hq_min + ht * kTH;
    r.wq0 = d.wq_min + wt * kTW;
    r.c0 = ct * bn;
    r.nt = (d.KH - r.a + d.S - 1) / d.S;   // taps r = a + S*t, t < nt
    r.nu = (d.KW - r.b + d.S - 1) / d.S;
    return r;
}

template <int BN, int STAGES, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    dense_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ DenseArgs d)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using L = DenseLayout<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kTileBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_kb = (d.Kg + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < d.num_tiles && ok; t += gridDim.x) {
                const DTile tl = decode_tile(d, t, BN);
                for (int ti = 0; ti < tl.nt && ok; ++ti) {
                    for (int ui = 0; ui < tl.nu && ok; ++ui) {
                        const int tap = (tl.a + d.S * ti) * d.KW + (tl.b + d.S * ui);
                        for (int kb = 0; kb < num_kb; ++kb) {
                            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
                            uint8_t* a_tile = smem + stage * L::kStageBytes;
                            uint8_t* b_tile = a_tile + L::kABytes;
                            // A: dY[n, hq0 - t .. +8, wq0 - u .. +16, group g, kb*64 .. +64] (zero outside)
                            tma_load_5d(a_tile, &map_a, &full[stage], kb * kBK, tl.g, tl.wq0 - ui, tl.hq0 - ti,
                                        tl.n);
                            // B: W[tap][group g][kb*64 .. +64][c0 .. c0 + BN] (zero outside)
#pragma unroll
                            for (int j = 0; j < BN / 64; ++j)
                                tma_load_4d(b_tile + j * 8192, &map_b, &full[stage], tl.c0 + j * 64, kb * kBK, tl.g,
                                            tap);
                            ++issued;
                            if (++stage == STAGES) {
                                stage = 0;
                                phase ^= 1u;
                            }
                        }
                    }
                }
            }
            if (!ok) {
                report_timeout(d.status);
                *abort_flag = 1;
            }
            for (long long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
                const int s = static_cast<int>(i % STAGES);
                const uint32_t par = static_cast<uint32_t>((i / STAGES) & 1);
                if (!mbar_wait(&full[s], par)) {
                    report_timeout(d.status);
                    *abort_flag = 1;
                }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc =
                F16 ? idesc_f16_f32(kBM, BN, /*b_mn_major=*/true) : idesc_bf16_f32(kBM, BN, /*b_mn_major=*/true);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < d.num_tiles && ok; t += gridDim.x) {
                const DTile tl = decode_tile(d, t, BN);
                const int nsteps = tl.nt * tl.nu * num_kb;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int st = 0; st < nsteps; ++st) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + stage * L::kStageBytes);
                    const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t a_desc = sw128_desc(a_addr + kk * 32, 16, 1024);
                        const uint64_t b_desc = sw128_desc(b_addr + kk * 2048, 8192, 1024);
                        umma_f16(d_tmem, a_desc, b_desc, idesc, (st | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                report_timeout(d.status);
                *abort_flag = 1;
            }
            umma_commit(drain);
            if (!mbar_wait(drain, 0)) {
                report_timeout(d.status);
                *abort_flag = 1;
            }
        }
    } else {
        // ----------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;           // tile position: hq0 + row/16, wq0 + row%16
        const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < d.num_tiles; t += gridDim.x) {
            const DTile tl = decode_tile(d, t, BN);
            if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int h = d.S * (tl.hq0 + row / kTW) + tl.a - d.ph;
            const int w = d.S * (tl.wq0 + row % kTW) + tl.b - d.pw;
            const bool pos_ok = h >= 0 && h < d.H && w >= 0 && w < d.W;
            uint16_t* out_row = reinterpret_cast<uint16_t*>(d.dX) +
                                ((static_cast<int64_t>(tl.n) * d.H + (pos_ok ? h : 0)) * d.W + (pos_ok ? w : 0)) * d.C +
                                static_cast<int64_t>(tl.g) * d.Cg;
            // A phase with no taps (filter extent below the stride) receives nothing: its
            // positions are written as zeros and the accumulator is not read.
            const bool no_taps = tl.nt == 0 || tl.nu == 0;
#pragma unroll 1
            for (int chunk = 0; chunk < BN / 32; ++chunk) {
                uint32_t v[32];
                if (no_taps) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = 0u;
                } else {
                    tmem_ld_32x32b_x32(tmem_base + lane_addr + static_cast<uint32_t>(acc * BN + chunk * 32), v);
                    tmem_wait_ld();
                }
                const int col0 = tl.c0 + chunk * 32;
                if (pos_ok) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int col = col0 + g * 8;
                        if (col < d.Cg) {
                            auto cvt = [](uint32_t lo, uint32_t hi) {
                                return F16 ? float2_to_f16x2(__uint_as_float(lo), __uint_as_float(hi))
                                           : float2_to_bf16x2(__uint_as_float(lo), __uint_as_float(hi));
                            };
                            uint4 o;
                            o.x = cvt(v[g * 8 + 0], v[g * 8 + 1]);
                            o.y = cvt(v[g * 8 + 2], v[g * 8 + 3]);
                            o.z = cvt(v[g * 8 + 4], v[g * 8 + 5]);
                            o.w = cvt(v[g * 8 + 6], v[g * 8 + 7]);
                            *reinterpret_cast<uint4*>(out_row + col) = o;
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            report_timeout(d.status);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem_base, L::kTmemCols);
    }
}

template <int BN, int STAGES>
cudaError_t launch_dense_bn(DenseArgs d, const CUtensorMap& map_a, const CUtensorMap& map_b, int num_sms,
                            cudaStream_t stream)
{
    using L = DenseLayout<BN, STAGES>;
    auto kern = d.f16 ? dense_tc_kernel<BN, STAGES, true> : dense_tc_kernel<BN, STAGES, false>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), L::kAlloc);
    if (e != cudaSuccess) return e;
    d.nc = (d.Cg + BN - 1) / BN;
    const long long tiles = static_cast<long long>(d.N) * d.S * d.S * d.nth * d.ntw * d.G * d.nc;
    if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    d.num_tiles = static_cast<int>(tiles);
    if (d.num_tiles == 0) return cudaSuccess;
    const int grid = d.num_tiles < num_sms ? d.num_tiles : num_sms;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(grid), dim3(kThreads), L::kAlloc, stream, 1,
                                             map_a, map_b, d);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

}  // namespace

void plan_dense(DenseArgs* d)
{
    // hq covers the union of every phase's rows: h = S*hq + a - ph in [0, H) for some a
    // in [0, S), i.e. hq in [ceil((ph - S + 1) / S), floor((H - 1 + ph) / S)]
    auto ceil_div = [](int v, int s) { return v >= 0 ? (v + s - 1) / s : -((-v) / s); };
    d->hq_min = ceil_div(d->ph - d->S + 1, d->S);
    d->wq_min = ceil_div(d->pw - d->S + 1, d->S);
    const int hq_max = (d->H - 1 + d->ph) / d->S;
    const int wq_max = (d->W - 1 + d->pw) / d->S;
    d->nth = (hq_max - d->hq_min + 1 + kTH - 1) / kTH;
    d->ntw = (wq_max - d->wq_min + 1 + kTW - 1) / kTW;
}

cudaError_t launch_dense_tc(const DenseArgs& d, const CUtensorMap& map_a, const CUtensorMap& map_b, int bn,
                            int num_sms, cudaStream_t stream)
{
    if (d.N <= 0) return cudaSuccess;
    switch (bn) {
    case 64: return launch_dense_bn<64, 8>(d, map_a, map_b, num_sms, stream);
    case 256: return launch_dense_bn<256, 4>(d, map_a, map_b, num_sms, stream);
    default: return launch_dense_bn<128, 6>(d, map_a, map_b, num_sms, stream);
    }
}

}  // namespace dgrad
