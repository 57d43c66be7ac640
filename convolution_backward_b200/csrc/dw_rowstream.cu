// dw_rowstream.cu -- depthwise dgrad by row streaming (any stride).
//
// The row-streaming schedule of "channel-packed and large-filter depthwise
// dgrad" (Technical Details, channel-packed row-streaming dgrad): dY rows are
// streamed in order, each row adds its contributions into accumulator rows held
// in a circular buffer, and once no later dY row can reach a dX row that row is
// final and is written out; a tail flushes the rows past the last dY row.
// With h = ho*S - pad_h + r and x = wo*S - pad_w + s:
//     acc[h mod R][x][c] += dY[n,ho,wo,c] * W[r][s][c]
// and after dY row ho every dX row h < (ho+1)*S - pad_h is final.  R = max(KH, S)
// slots suffice: row ho touches KH consecutive rows, and the rows flushed after
// it span at most S.  Rows no dY row reaches come out as zeros.
//
// B200 design.  The accumulator ring lives in shared memory as fp32 channel
// pairs.  A CTA (256 threads) owns one image, 32 channels and a strip of 16 to
// 64 dX columns; thread (pair cp, column slot xs) owns columns x0+xs+16q, so
// every ring entry is private to one thread and the ring needs no barriers.
// Each dY row segment the strip needs is staged once in shared memory (fp32
// pairs, 128-bit loads, the next row prefetched into registers while the
// current one is applied).  For a dX column x only the taps s = s0, s0+S, ...
// with s0 = (x + pad_w) mod S reach it, each from dY column (x + pad_w - s)/S;
// the thread walks them with a stride and no divisions in the tap loop.  The
// filter, converted to fp32 pairs, sits in shared memory when it fits and is
// read through the read-only cache otherwise.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kCB = 32;
constexpr int kPairs = 16;
constexpr int kThreads = 256;
constexpr int kMaxTX = 64;       // dX columns per CTA, at most
constexpr int kMaxQ = kMaxTX / 16;
constexpr int kMaxSmemTaps = 512;
constexpr size_t kSmemBudget = 200 * 1024;
constexpr int kMaxPF = 4;        // 16-byte prefetch registers per thread for one dY row segment

struct RsParams {
    const void* dY;
    const void* filt;
    void* dX;
    int N, H, W, C, Ho, Wo, KH, KW, S, ph, pw;
    int R;        // ring slots
    int TX, Q;    // dX columns per CTA (multiple of 16) and per thread (TX / 16)
    int nX, nC;   // column strips, channel blocks
    int LW;       // dY columns staged per row
    bool w_in_smem;
    long long dx_bytes;   // size of dX (index checks of the debug build)
    int* status;
};

__device__ __forceinline__ int floor_div(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

template <int EK>
struct RsChunk {
    static constexpr int kElems = EK == kF32 ? 4 : 8;
    static constexpr int kPerPos = kCB / kElems;
    static constexpr int kPairs = kElems / 2;
};

template <int EK>
__device__ __forceinline__ void rs_chunk_to_pairs(const uint4& v, float2* dst)
{
    if constexpr (EK != kF32) {
        dst[0] = h16x2_to_float2<EK>(v.x);
        dst[1] = h16x2_to_float2<EK>(v.y);
        dst[2] = h16x2_to_float2<EK>(v.z);
        dst[3] = h16x2_to_float2<EK>(v.w);
    } else {
        dst[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
        dst[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
    }
}

template <int EK>
__global__ void __launch_bounds__(kThreads)
    dw_rowstream_kernel(const RsParams p)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using Ch = RsChunk<EK>;
    using T = typename std::conditional<EK == kF32, float, uint16_t>::type;
    extern __shared__ float2 sm2[];
    float2* ring = sm2;                                   // [R][TX][16]
    float2* dyrow = ring + p.R * p.TX * kPairs;           // [LW][16]
    float2* wsm = dyrow + p.LW * kPairs;                  // [KH*KW][16] when staged

    int u = blockIdx.x;
    const int xblk = u % p.nX;
    u /= p.nX;
    const int cblk = u % p.nC;
    const int n = u / p.nC;

    const int tid = threadIdx.x;
    const int cp = tid & 15;
    const int xs = tid >> 4;
    const int c0 = cblk * kCB;
    const int x0 = xblk * p.TX;
    const int c = c0 + 2 * cp;
    const bool c_ok = c < p.C;
    // first dY column any column of the strip reads
    const int wo_base = floor_div(x0 + p.pw - (p.KW - 1), p.S);

    const long long C = p.C;
    const T* __restrict__ dy = static_cast<const T*>(p.dY) + static_cast<long long>(n) * p.Ho * p.Wo * C;
    const T* __restrict__ wg = static_cast<const T*>(p.filt);
    T* __restrict__ dx = static_cast<T*>(p.dX) + static_cast<long long>(n) * p.H * p.W * C;

    // Clear this thread's ring entries.
    for (int sl = 0; sl < p.R; ++sl)
        for (int q = 0; q < p.Q; ++q) ring[(sl * p.TX + xs + 16 * q) * kPairs + cp] = make_float2(0.f, 0.f);

    if (p.w_in_smem) {
        const int items = p.KH * p.KW * Ch::kPerPos;
        for (int it = tid; it < items; it += kThreads) {
            const int tap = it / Ch::kPerPos;
            const int ch = it - tap * Ch::kPerPos;
            const int cc = c0 + ch * Ch::kElems;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (cc < p.C) v = __ldg(reinterpret_cast<const uint4*>(wg + tap * C + cc));
            rs_chunk_to_pairs<EK>(v, wsm + tap * kPairs + ch * Ch::kPairs);
        }
    }

    const int row_items = p.LW * Ch::kPerPos;
    auto fetch_row = [&](int ho, uint4 (&pf)[kMaxPF]) {
#pragma unroll
        for (int k = 0; k < kMaxPF; ++k) {
            const int it = tid + k * kThreads;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (it < row_items) {
                const int j = it / Ch::kPerPos;
                const int ch = it - j * Ch::kPerPos;
                const int wo = wo_base + j;
                const int cc = c0 + ch * Ch::kElems;
                if (wo >= 0 && wo < p.Wo && cc < p.C)
                    v = __ldg(reinterpret_cast<const uint4*>(dy + (static_cast<long long>(ho) * p.Wo + wo) * C + cc));
            }
            pf[k] = v;
        }
    };
    auto store_row = [&](const uint4 (&pf)[kMaxPF]) {
#pragma unroll
        for (int k = 0; k < kMaxPF; ++k) {
            const int it = tid + k * kThreads;
            if (it < row_items) {
                const int j = it / Ch::kPerPos;
                const int ch = it - j * Ch::kPerPos;
                rs_chunk_to_pairs<EK>(pf[k], dyrow + j * kPairs + ch * Ch::kPairs);
            }
        }
    };
    auto weight = [&](int tap) -> float2 {
        if (p.w_in_smem) return wsm[tap * kPairs + cp];
        if (!c_ok) return make_float2(0.f, 0.f);
        if constexpr (EK != kF32)
            return h16x2_to_float2<EK>(__ldg(reinterpret_cast<const uint32_t*>(wg + tap * C + c)));
        else
            return __ldg(reinterpret_cast<const float2*>(wg + tap * C + c));
    };
    auto flush_row = [&](int h) {
        const int sl = h % p.R;
#pragma unroll
        for (int q = 0; q < kMaxQ; ++q) {
            if (q >= p.Q) break;
            const int xl = xs + 16 * q;
            const int x = x0 + xl;
            float2* e = ring + (sl * p.TX + xl) * kPairs + cp;
            const float2 v = *e;
            *e = make_float2(0.f, 0.f);
            T* o = dx + (static_cast<long long>(h) * p.W + x) * C + c;
            if (x < p.W && c_ok && store_ok(p.dX, p.dx_bytes, o, EK != kF32 ? 4 : 8, p.status)) {
                if constexpr (EK != kF32)
                    *reinterpret_cast<uint32_t*>(o) = float2_to_h16x2<EK>(v.x, v.y);
                else
                    *reinterpret_cast<float2*>(o) = v;
            }
        }
    };

    uint4 pf[kMaxPF];
    fetch_row(0, pf);
    int next_flush = 0;
    for (int ho = 0; ho < p.Ho; ++ho) {
        __syncthreads();                 // previous row's readers are done
        store_row(pf);
        __syncthreads();
        if (ho + 1 < p.Ho) fetch_row(ho + 1, pf);
#pragma unroll
        for (int q = 0; q < kMaxQ; ++q) {
            if (q >= p.Q) break;
            const int xl = xs + 16 * q;
            const int x = x0 + xl;
            if (x >= p.W) continue;
            const int s0 = (x + p.pw) % p.S;
            const int j0 = (x + p.pw - s0) / p.S - wo_base;   // staged index of tap s0
            for (int r = 0; r < p.KH; ++r) {
                const int h = ho * p.S - p.ph + r;
                if (h < 0 || h >= p.H) continue;
                float2 sum = make_float2(0.f, 0.f);
                int j = j0;
                for (int s = s0; s < p.KW; s += p.S, --j)
                    sum = ffma2(dyrow[j * kPairs + cp], weight(r * p.KW + s), sum);
                float2* e = ring + ((h % p.R) * p.TX + xl) * kPairs + cp;
                float2 v = *e;
                v.x += sum.x;
                v.y += sum.y;
                *e = v;
            }
        }
        int done = (ho + 1) * p.S - p.ph;
        if (done > p.H) done = p.H;
        for (; next_flush < done; ++next_flush) flush_row(next_flush);
    }
    for (; next_flush < p.H; ++next_flush) flush_row(next_flush);   // tail
}

template <int EK>
cudaError_t launch_t(const RsParams& p, long long blocks, size_t smem, cudaStream_t stream)
{
    auto kern = dw_rowstream_kernel<EK>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), smem, stream, 1,
                                             p);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dw_rowstream(const DwArgs& a, cudaStream_t stream)
{
    RsParams p{};
    p.dY = a.dY;
    p.filt = a.filt;
    p.dX = a.dX;
    p.N = a.N; p.H = a.H; p.W = a.W; p.C = a.C; p.Ho = a.Ho; p.Wo = a.Wo;
    p.KH = a.KH; p.KW = a.KW; p.S = a.S; p.ph = a.ph; p.pw = a.pw;
    p.dx_bytes = static_cast<long long>(a.N) * a.H * a.W * a.C * (a.elem_kind() == kF32 ? 4 : 2);
    p.status = a.status;
    p.R = a.KH > a.S ? a.KH : a.S;
    p.nC = (a.C + kCB - 1) / kCB;
    // Widest strip (64, 48, 32 or 16 columns) whose ring and staged row fit the
    // budget; the filter is staged too when it still fits.
    auto smem_for = [&](int tx, bool wsm) {
        const int lw = (tx - 1 + a.KW - 1) / a.S + 2;   // dY columns a strip of tx dX columns reads
        return (static_cast<size_t>(p.R) * tx + lw + (wsm ? a.KH * a.KW : 0)) * kPairs * sizeof(float2);
    };
    p.TX = kMaxTX;
    while (p.TX > 16 && smem_for(p.TX, false) > kSmemBudget) p.TX -= 16;
    p.Q = p.TX / 16;
    p.w_in_smem = a.KH * a.KW <= kMaxSmemTaps && smem_for(p.TX, true) <= kSmemBudget;
    p.nX = (a.W + p.TX - 1) / p.TX;
    p.LW = (p.TX - 1 + a.KW - 1) / a.S + 2;
    const size_t smem = smem_for(p.TX, p.w_in_smem);
    if (smem > kSmemBudget) return cudaErrorInvalidConfiguration;
    const int per_pos = a.elem_kind() == kF32 ? RsChunk<kF32>::kPerPos : RsChunk<kBF16>::kPerPos;
    if (p.LW * per_pos > kMaxPF * kThreads) return cudaErrorInvalidConfiguration;
    const long long blocks = static_cast<long long>(a.N) * p.nC * p.nX;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    if (a.f16) return launch_t<kF16>(p, blocks, smem, stream);
    if (a.bf16) return launch_t<kBF16>(p, blocks, smem, stream);
    return launch_t<kF32>(p, blocks, smem, stream);
}

}  // namespace dgrad
