// dw_tile.cu -- stride-1 depthwise dgrad for small filters (up to 7 x 7), bf16 or f16.
//
// The rotated-filter correlation of "channel-packed and large-filter depthwise
// dgrad" (Technical Details, rotated-filter dgrad):
//     dX[n,h,w,c] = sum_{r'<KH, s'<KW} dY[n, h-P'h+r', w-P'w+s', c] * W[KH-1-r'][KW-1-s'][c],
// P'h = KH-1-pad_h, P'w = KW-1-pad_w, dY zero off the image.
//
// Small filters make this HBM-bound (a few FMAs per byte), so the kernel is
// built for one memory round trip per CTA and many CTAs in flight:
//   * a CTA owns an output tile of TH rows x TW columns x 32 channels; one TMA
//     load brings its whole halo tile [TH+KH-1][TW+KW-1][32] of dY into shared
//     memory, the out-of-image part zero-filled by the TMA (that is the padding);
//   * thread (channel pair, row slot, column slot) computes R rows x TAT columns;
//     it walks the R+KH-1 input rows it needs once, converting each 16-bit pair
//     to fp32 once, and applies every filter row that input row reaches
//     (packed fma.rn.f32x2, the rotated filter held in registers);
//   * results are rounded to the I/O format into an output tile [TH][TW][32] that
//     replaces the halo tile in shared memory, and one TMA box stores it, clipping
//     the ragged edges (3x3 on 8 x 56 x 56 x 128: 5.68 -> 5.16 us on B200 against
//     direct 4-byte stores, which DGRAD_TILE_STORE=direct keeps for testing).
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

#include <cstring>

namespace dgrad {
namespace {

struct TileParams {
    uint16_t* dX;         // 16-bit elements (bf16 or f16)
    const uint16_t* filt;
    int* status;
    int N, H, W, C, ph, pw;
    int CS, RS;       // column and row slots per CTA (threads = 16 * CS * RS)
    int TH, TW;       // output tile
    int nX, nY, nC;
    int tma_out;          // the output tile is staged in shared memory and stored with one TMA box
    long long dx_bytes;   // size of dX (index checks of the debug build)
};

template <int KH, int KW, int R, int TAT, int EK>
__global__ void __launch_bounds__(256)
    dw_tile_kernel(const __grid_constant__ CUtensorMap dy_map, const __grid_constant__ CUtensorMap dx_map,
                   const TileParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 127u) & ~127u) - raw);
    const int LWt = p.TW + KW - 1;                        // staged columns
    const int LHt = p.TH + KH - 1;                        // staged rows
    const uint32_t tile_bytes = static_cast<uint32_t>(LWt * LHt * 64);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + ((tile_bytes + 15u) & ~15u));
    const uint32_t* tile = reinterpret_cast<const uint32_t*>(smem);   // [LHt][LWt][16] 16-bit pairs

    int u = blockIdx.x;
    const int xblk = u % p.nX;
    u /= p.nX;
    const int yblk = u % p.nY;
    u /= p.nY;
    const int cblk = u % p.nC;
    const int n = u / p.nC;
    const int tid = threadIdx.x;
    const int cp = tid & 15;
    const int slot = tid >> 4;
    const int cs = slot % p.CS;
    const int rs = slot / p.CS;
    const int c0 = cblk * 32;
    const int c = c0 + 2 * cp;
    const int h0 = yblk * p.TH;
    const int w0 = xblk * p.TW;

    if (tid == 0) {
        // While the previous kernel may still run, only an L2 prefetch of this CTA's halo
        // tile: L2 is the point of coherence, so the load below still sees that kernel's
        // writes; the DRAM reads overlap its tail.
        tma_prefetch_desc(&dy_map);
        tma_prefetch_l2_4d(&dy_map, c0, w0 - (KW - 1 - p.pw), h0 - (KH - 1 - p.ph), n);
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, tile_bytes);
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem)),
            "l"(reinterpret_cast<uint64_t>(&dy_map)), "r"(smem_u32(bar)), "r"(c0),
            "r"(w0 - (KW - 1 - p.pw)), "r"(h0 - (KH - 1 - p.ph)), "r"(n)
            : "memory");
    }
    // rotated filter taps of this channel pair: wr[r'][s'] = W[KH-1-r'][KW-1-s']
    float2 wr[KH][KW];
    const bool c_ok = c < p.C;
#pragma unroll
    for (int r = 0; r < KH; ++r)
#pragma unroll
        for (int s = 0; s < KW; ++s)
            wr[r][s] = c_ok ? h16x2_to_float2<EK>(__ldg(reinterpret_cast<const uint32_t*>(
                                  p.filt + ((KH - 1 - r) * KW + (KW - 1 - s)) * p.C + c)))
                            : make_float2(0.f, 0.f);

    const bool ok = mbar_wait(bar, 0);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            report_timeout(p.status);
            mbar_wait(bar, 0);   // let the copy land before the shared memory is released
        }
        return;
    }

    float2 acc[R][TAT];
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < TAT; ++j) acc[i][j] = make_float2(0.f, 0.f);

    const int row0 = rs * R;          // first output row of this thread inside the tile
    const int col0 = cs * TAT;
#pragma unroll
    for (int i = 0; i < R + KH - 1; ++i) {
        // staged input row row0 + i feeds output rows row0 + ro with filter row r' = i - ro
        float2 x[TAT + KW - 1];
        const uint32_t* src = tile + ((row0 + i) * LWt + col0) * 16 + cp;
#pragma unroll
        for (int m = 0; m < TAT + KW - 1; ++m) x[m] = h16x2_to_float2<EK>(src[m * 16]);
        // taps outermost: consecutive FMAs update different accumulators
#pragma unroll
        for (int s = 0; s < KW; ++s)
#pragma unroll
            for (int ro = 0; ro < R; ++ro) {
                const int rr = i - ro;
                if (rr < 0 || rr >= KH) continue;
#pragma unroll
                for (int j = 0; j < TAT; ++j) acc[ro][j] = ffma2(x[j + s], wr[rr][s], acc[ro][j]);
            }
    }

    if (p.tma_out) {
        // The output tile [TH][TW][32 channels] replaces the halo tile in shared memory and
        // one TMA box stores it; the box clips rows, columns and channels past dX.
        __syncthreads();   // every thread has read the halo tile
        uint32_t* out_t = reinterpret_cast<uint32_t*>(smem);
#pragma unroll
        for (int ro = 0; ro < R; ++ro)
#pragma unroll
            for (int j = 0; j < TAT; ++j)
                out_t[((row0 + ro) * p.TW + col0 + j) * 16 + cp] = float2_to_h16x2<EK>(acc[ro][j].x, acc[ro][j].y);
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&dx_map, smem, c0, w0, h0, n);
            bulk_commit_group();
            bulk_wait_group<0>();   // the tile has been read and written before the CTA ends
        }
        return;
    }
    if (!c_ok) return;
    const long long row_elems = static_cast<long long>(p.W) * p.C;
    uint16_t* obase = p.dX + static_cast<long long>(n) * p.H * row_elems + c;
#pragma unroll
    for (int ro = 0; ro < R; ++ro) {
        const int h = h0 + row0 + ro;
        if (h >= p.H || row0 + ro >= p.TH) continue;
        uint16_t* orow = obase + static_cast<long long>(h) * row_elems;
#pragma unroll
        for (int j = 0; j < TAT; ++j) {
            const int w = w0 + col0 + j;
            if (w < p.W && col0 + j < p.TW &&
                store_ok(p.dX, p.dx_bytes, orow + static_cast<long long>(w) * p.C, 4, p.status))
                *reinterpret_cast<uint32_t*>(orow + static_cast<long long>(w) * p.C) =
                    float2_to_h16x2<EK>(acc[ro][j].x, acc[ro][j].y);
        }
    }
}

template <int KH, int KW, int R, int TAT>
TileParams plan_tile(const DwArgs& a)
{
    TileParams p{};
    p.dX = static_cast<uint16_t*>(a.dX);
    p.filt = static_cast<const uint16_t*>(a.filt);
    p.status = a.status;
    p.N = a.N; p.H = a.H; p.W = a.W; p.C = a.C; p.ph = a.ph; p.pw = a.pw;
    p.dx_bytes = static_cast<long long>(a.N) * a.H * a.W * a.C * 2;
    // columns: as few column slots as cover the row (at most 16), balanced
    int cs = (a.W + TAT - 1) / TAT;
    if (cs > 16) {
        const int strips = (cs + 15) / 16;
        cs = (cs + strips - 1) / strips;
    }
    p.CS = cs;
    p.TW = cs * TAT;
    // rows: fill up to 256 threads, but keep enough CTAs in flight
    int rs = 16 / cs;
    if (rs < 1) rs = 1;
    p.RS = rs;
    p.TH = rs * R;
    p.nX = (a.W + p.TW - 1) / p.TW;
    p.nY = (a.H + p.TH - 1) / p.TH;
    p.nC = (a.C + 31) / 32;
    return p;
}

template <int KH, int KW, int R, int TAT>
cudaError_t launch_tile(const DwArgs& a, const CUtensorMap& map, const CUtensorMap* dx_map, cudaStream_t stream)
{
    TileParams p = plan_tile<KH, KW, R, TAT>(a);
    // DGRAD_TILE_STORE=direct keeps the direct 4-byte stores of dX (testing and tuning)
    const char* ts = dgrad::tuning_env("DGRAD_TILE_STORE");
    p.tma_out = dx_map != nullptr && !(ts && strcmp(ts, "direct") == 0) ? 1 : 0;
    const long long blocks = static_cast<long long>(a.N) * p.nC * p.nY * p.nX;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    const size_t tile = static_cast<size_t>(p.TW + KW - 1) * (p.TH + KH - 1) * 64;
    const size_t smem = ((tile + 15) & ~static_cast<size_t>(15)) + 16 + 128;
    auto kern = a.f16 ? dw_tile_kernel<KH, KW, R, TAT, kF16> : dw_tile_kernel<KH, KW, R, TAT, kBF16>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(static_cast<unsigned>(blocks)), dim3(16 * p.CS * p.RS), smem, stream, 1,
                                             map, p.tma_out ? *dx_map : map, p);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

#define DGRAD_TILE_SET(X) \
    X(3, 3, 2, 8)         \
    X(5, 5, 2, 8)         \
    X(7, 7, 2, 8)

}  // namespace

bool dw_tile_box(const DwArgs& a, unsigned box[4], unsigned box_dx[4])
{
    if (!(a.bf16 || a.f16) || a.S != 1) return false;
#define DGRAD_TILE_BOX(kh, kw, r, tat)                                                              \
    if (a.KH == kh && a.KW == kw) {                                                                 \
        const TileParams p = plan_tile<kh, kw, r, tat>(a);                                          \
        box[0] = 32; box[1] = static_cast<unsigned>(p.TW + kw - 1);                                  \
        box[2] = static_cast<unsigned>(p.TH + kh - 1); box[3] = 1;                                   \
        box_dx[0] = 32; box_dx[1] = static_cast<unsigned>(p.TW);                                    \
        box_dx[2] = static_cast<unsigned>(p.TH); box_dx[3] = 1;                                     \
        return true;                                                                                \
    }
    DGRAD_TILE_SET(DGRAD_TILE_BOX)
#undef DGRAD_TILE_BOX
    return false;
}

cudaError_t launch_dw_tile(const DwArgs& a, const CUtensorMap& dy_map, const CUtensorMap* dx_map, cudaStream_t stream)
{
    if (!(a.bf16 || a.f16) || a.S != 1) return cudaErrorNotSupported;
#define DGRAD_TILE_LAUNCH(kh, kw, r, tat) \
    if (a.KH == kh && a.KW == kw) return launch_tile<kh, kw, r, tat>(a, dy_map, dx_map, stream);
    DGRAD_TILE_SET(DGRAD_TILE_LAUNCH)
#undef DGRAD_TILE_LAUNCH
    return cudaErrorNotSupported;
}

}  // namespace dgrad
