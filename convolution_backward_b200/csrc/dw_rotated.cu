// dw_rotated.cu -- stride-1 depthwise dgrad as a rotated-filter correlation.
//
// A stride-1 depthwise dgrad equals the forward correlation of dY with the
// filter turned by 180 degrees, at padding KH-1-pad_h rows and KW-1-pad_w
// columns: weight row r is read from row KH-1-r, back to front ("channel-packed
// and large-filter depthwise dgrad", Technical Details, rotated-filter dgrad):
//     dX[n,h,w,c] = sum_{r'<KH, s'<KW} dY[n, h-P'h+r', w-P'w+s', c] * W[KH-1-r'][KW-1-s'][c]
// with P'h = KH-1-pad_h, P'w = KW-1-pad_w and dY read as zero off the image.
//
// B200 design.  The correlation is FMA-bound for large filters, so the inner
// loop is built to be nearly all packed fp32 FMAs (fma.rn.f32x2 on channel
// pairs):
//   - "A" is the filter's longer axis (w for square filters), "B" the other.
//     A thread owns one channel pair, one output line along A and TAT
//     consecutive outputs on it; their accumulators stay in registers.
//   - The CTA (256 threads = 16 channel pairs x 16 line/strip slots) covers 32
//     channels, TB output lines and NS*TAT outputs along A.  The loop runs over
//     the filter's B index jb: step jb needs rotated filter line jb (KA taps)
//     and dY lines b0-P'B+jb .. +TB-1, a window that slides by one line per
//     step.  dY lines sit in a shared-memory ring of TB+1 lines, converted once
//     to fp32 pairs on arrival; the next line and next filter line are fetched
//     into registers with 128-bit loads while the current step computes.
//   - Per step a thread loads the KA taps of its filter line into registers
//     (the pages' "one filter row register-resident") and streams the
//     TAT+KA-1 dY values of its strip through them: TAT*KA packed FMAs for
//     TAT+KA-1 shared-memory loads.
// KA is a compile-time parameter; a filter whose A extent has no exact
// instantiation runs in the next larger one with zero taps appended.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

#include <cstdlib>

namespace dgrad {
namespace {

constexpr int kCB = 32;       // channels per CTA
constexpr int kPairs = 16;    // channel pairs per CTA
constexpr int kThreads = 256;
constexpr int kMaxPF = 4;     // 16-byte prefetch registers per thread for one dY line

struct RotParams {
    const void* dY;
    const void* filt;
    void* dX;
    int C;
    int OA, OB;               // dX extents along A and B
    int IA, IB;               // dY extents along A and B
    int KA, KB;               // filter extents along A and B
    int PA, PB;               // rotated paddings along A and B
    long long in_sA, in_sB, in_sN;
    long long out_sA, out_sB, out_sN;
    int w_sA, w_sB;           // filter strides along A and B (W is [KH][KW][C])
    int NS, TB, TAC, LA, RING;
    long long dx_bytes;       // size of dX (index checks of the debug build)
    int* status;
    int nA, nB, nC;
};

template <int EK>
struct Chunk {
    // A 16-byte chunk holds 8 16-bit or 4 f32 channels.
    static constexpr int kElems = EK == kF32 ? 4 : 8;
    static constexpr int kPerPos = kCB / kElems;   // chunks per position (32 channels)
    static constexpr int kPairs = kElems / 2;      // channel pairs per chunk
};

template <int EK>
__device__ __forceinline__ void chunk_to_pairs(const uint4& v, float2* dst)
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

template <int KAI, int TAT, int EK>
__global__ void __launch_bounds__(kThreads, 2)
    dw_rot_kernel(const RotParams p)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using Ch = Chunk<EK>;
    using T = typename std::conditional<EK == kF32, float, uint16_t>::type;
    extern __shared__ float2 sm2[];
    float2* ring = sm2;                                  // [RING][LA][16]
    float2* wbuf = sm2 + p.RING * p.LA * kPairs;         // [2][KAI][16]

    int u = blockIdx.x;
    const int ablk = u % p.nA;
    u /= p.nA;
    const int bblk = u % p.nB;
    u /= p.nB;
    const int cblk = u % p.nC;
    const int n = u / p.nC;

    const int tid = threadIdx.x;
    const int cp = tid & 15;
    const int slot = tid >> 4;
    const int line = slot / p.NS;
    const int strip = slot - line * p.NS;
    const int c0 = cblk * kCB;
    const int b0 = bblk * p.TB;
    const int a0 = ablk * p.TAC;
    const int ib0 = b0 - p.PB;    // dY line held by ring index 0
    const int ia0 = a0 - p.PA;    // dY position of ring column 0

    const T* __restrict__ dy = static_cast<const T*>(p.dY) + static_cast<long long>(n) * p.in_sN;
    const T* __restrict__ wg = static_cast<const T*>(p.filt);
    T* __restrict__ dx = static_cast<T*>(p.dX) + static_cast<long long>(n) * p.out_sN;

    // Fill plan, fixed for the whole CTA: item k of this thread is dY position
    // pos = it / kPerPos of a line, channel chunk ch = it % kPerPos (it = tid + k*256).
    // Only the line index changes from step to step.
    const int line_items = p.LA * Ch::kPerPos;
    int goff[kMaxPF];        // element offset inside a dY line (position and channel)
    int soff[kMaxPF];        // float2 offset inside a ring line
    uint32_t vmask = 0;      // bit k: item k lies inside the image along A and inside C
    uint32_t imask = 0;      // bit k: item k exists
#pragma unroll
    for (int k = 0; k < kMaxPF; ++k) {
        const int it = tid + k * kThreads;
        const int pos = it / Ch::kPerPos;
        const int ch = it - pos * Ch::kPerPos;
        const int ia = ia0 + pos;
        const int c = c0 + ch * Ch::kElems;
        goff[k] = static_cast<int>(ia * p.in_sA) + c;
        soff[k] = pos * kPairs + ch * Ch::kPairs;
        if (it < line_items) {
            imask |= 1u << k;
            if (ia >= 0 && ia < p.IA && c < p.C) vmask |= 1u << k;
        }
    }
    constexpr int kWItems = KAI * Ch::kPerPos;
    constexpr int kWPF = (kWItems + kThreads - 1) / kThreads;
    int wgoff[kWPF];
    int wsoff[kWPF];
    uint32_t wvmask = 0, wimask = 0;
#pragma unroll
    for (int k = 0; k < kWPF; ++k) {
        const int it = tid + k * kThreads;
        const int ia = it / Ch::kPerPos;
        const int ch = it - ia * Ch::kPerPos;
        const int c = c0 + ch * Ch::kElems;
        // tap ia of a rotated filter line is W[B index KB-1-jb][A index KA-1-ia]
        wgoff[k] = (p.KA - 1 - ia) * p.w_sA + c;
        wsoff[k] = ia * kPairs + ch * Ch::kPairs;
        if (it < kWItems) {
            wimask |= 1u << k;
            if (ia < p.KA && c < p.C) wvmask |= 1u << k;
        }
    }

    auto fetch_line = [&](int i, uint4 (&pf)[kMaxPF]) {
        const int ib = ib0 + i;
        const uint32_t m = (ib >= 0 && ib < p.IB) ? vmask : 0u;
        const T* base = dy + static_cast<long long>(ib) * p.in_sB;
#pragma unroll
        for (int k = 0; k < kMaxPF; ++k)
            pf[k] = (m >> k) & 1u ? __ldg(reinterpret_cast<const uint4*>(base + goff[k])) : make_uint4(0u, 0u, 0u, 0u);
    };
    auto store_line = [&](int slot_idx, const uint4 (&pf)[kMaxPF]) {
        float2* dst = ring + slot_idx * p.LA * kPairs;
#pragma unroll
        for (int k = 0; k < kMaxPF; ++k)
            if ((imask >> k) & 1u) chunk_to_pairs<EK>(pf[k], dst + soff[k]);
    };
    auto fetch_wline = [&](int jb, uint4 (&pw)[kWPF]) {
        const T* base = wg + (p.KB - 1 - jb) * p.w_sB;
#pragma unroll
        for (int k = 0; k < kWPF; ++k)
            pw[k] = (wvmask >> k) & 1u ? __ldg(reinterpret_cast<const uint4*>(base + wgoff[k]))
                                       : make_uint4(0u, 0u, 0u, 0u);
    };
    auto store_wline = [&](int jb, const uint4 (&pw)[kWPF]) {
        float2* dst = wbuf + (jb & 1) * KAI * kPairs;
#pragma unroll
        for (int k = 0; k < kWPF; ++k)
            if ((wimask >> k) & 1u) chunk_to_pairs<EK>(pw[k], dst + wsoff[k]);
    };

    // Prologue: the first TB dY lines and filter line 0.
    {
        uint4 pf[kMaxPF];
        for (int i = 0; i < p.TB; ++i) {
            fetch_line(i, pf);
            store_line(i, pf);
        }
        uint4 pw[kWPF];
        fetch_wline(0, pw);
        store_wline(0, pw);
    }
    __syncthreads();

    float2 acc[TAT];
#pragma unroll
    for (int j = 0; j < TAT; ++j) acc[j] = make_float2(0.f, 0.f);

    int read_slot = line;              // ring slot of dY line (line + jb)
    int fill_slot = p.TB;              // ring slot of dY line (TB + jb), the one fetched during step jb
    for (int jb = 0; jb < p.KB; ++jb) {
        const bool more = jb + 1 < p.KB;
        uint4 pf[kMaxPF];
        uint4 pw[kWPF];
        if (more) {
            fetch_line(p.TB + jb, pf);
            fetch_wline(jb + 1, pw);
        }
        float2 wr[KAI];
        const float2* wsrc = wbuf + (jb & 1) * KAI * kPairs + cp;
#pragma unroll
        for (int ia = 0; ia < KAI; ++ia) wr[ia] = wsrc[ia * kPairs];
        const float2* src = ring + (read_slot * p.LA + strip * TAT) * kPairs + cp;
#pragma unroll
        for (int q = 0; q < TAT + KAI - 1; ++q) {
            const float2 x = src[q * kPairs];
#pragma unroll
            for (int j = 0; j < TAT; ++j) {
                const int ia = q - j;
                if (ia >= 0 && ia < KAI) acc[j] = ffma2(x, wr[ia], acc[j]);
            }
        }
        if (more) {
            store_line(fill_slot, pf);
            store_wline(jb + 1, pw);
        }
        if (++read_slot == p.RING) read_slot = 0;
        if (++fill_slot == p.RING) fill_slot = 0;
        __syncthreads();
    }

    const int b = b0 + line;
    const int c = c0 + 2 * cp;
    if (b >= p.OB || c >= p.C) return;
    T* out = dx + b * p.out_sB + c;
#pragma unroll
    for (int j = 0; j < TAT; ++j) {
        const int a = a0 + strip * TAT + j;
        if (a < p.OA && store_ok(p.dX, p.dx_bytes, out + a * p.out_sA, EK != kF32 ? 4 : 8, p.status)) {
            if constexpr (EK != kF32)
                *reinterpret_cast<uint32_t*>(out + a * p.out_sA) = float2_to_h16x2<EK>(acc[j].x, acc[j].y);
            else
                *reinterpret_cast<float2*>(out + a * p.out_sA) = acc[j];
        }
    }
}

constexpr int kInstKA[] = {1, 3, 5, 7, 9, 11, 13, 15, 17, 21, 25, 31, 33, 41, 51, 64};

template <int KAI>
constexpr int tat_for() { return KAI <= 7 ? 8 : 16; }
// The alternative (tuning) width: 16 for short lines, 8 for long ones.  32 outputs
// per thread were measured slower for long lines and spilled registers at KA >= 13,
// so they are not built.
template <int KAI>
constexpr int tat_alt() { return KAI <= 7 ? 16 : 8; }

template <int KAI, int TAT, int EK>
cudaError_t launch_one(RotParams& p, long long blocks, cudaStream_t stream)
{
    const size_t smem = static_cast<size_t>(p.RING * p.LA + 2 * KAI) * kPairs * sizeof(float2);
    auto kern = dw_rot_kernel<KAI, TAT, EK>;
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), smem, stream, 1,
                                             p);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

template <int TAT, int KAI>
void plan_tiles(RotParams& p)
{
    int need = (p.OA + TAT - 1) / TAT;
    int ns = 1;
    while (ns < need && ns < 16) ns *= 2;
    // DGRAD_ROT_NS caps the strips per CTA (fewer strips, more lines: less fill per output)
    const char* e = dgrad::tuning_env("DGRAD_ROT_NS");
    if (e && atoi(e) >= 1 && atoi(e) < ns) ns = atoi(e);
    p.NS = ns;
    p.TB = 16 / ns;
    p.TAC = ns * TAT;
    p.LA = p.TAC + KAI - 1;
    p.RING = p.TB + 1;
    p.nA = (p.OA + p.TAC - 1) / p.TAC;
    p.nB = (p.OB + p.TB - 1) / p.TB;
    p.nC = (p.C + kCB - 1) / kCB;
}

template <int KAI, int TAT>
cudaError_t dispatch_t(RotParams& p, int N, int ek, cudaStream_t stream)
{
    plan_tiles<TAT, KAI>(p);
    const long long blocks = static_cast<long long>(N) * p.nC * p.nB * p.nA;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    const int per_pos = ek == kF32 ? Chunk<kF32>::kPerPos : Chunk<kBF16>::kPerPos;
    if (p.LA * per_pos > kMaxPF * kThreads) return cudaErrorInvalidConfiguration;
    if (ek == kF16) return launch_one<KAI, TAT, kF16>(p, blocks, stream);
    if (ek == kBF16) return launch_one<KAI, TAT, kBF16>(p, blocks, stream);
    return launch_one<KAI, TAT, kF32>(p, blocks, stream);
}

// Outputs per thread along A: tat_for<KAI>() by default; DGRAD_ROT_TAT may select tat_alt<KAI>().
template <int KAI>
cudaError_t dispatch(RotParams& p, int N, int ek, cudaStream_t stream)
{
    const char* e = dgrad::tuning_env("DGRAD_ROT_TAT");
    if (e && atoi(e) == tat_alt<KAI>()) return dispatch_t<KAI, tat_alt<KAI>()>(p, N, ek, stream);
    return dispatch_t<KAI, tat_for<KAI>()>(p, N, ek, stream);
}

}  // namespace

cudaError_t launch_dw_rotated(const DwArgs& a, cudaStream_t stream)
{
    RotParams p{};
    p.dY = a.dY;
    p.filt = a.filt;
    p.dX = a.dX;
    p.C = a.C;
    const long long C = a.C;
    const bool slide_w = a.KW >= a.KH;   // slide along the longer filter axis
    if (slide_w) {
        p.OA = a.W; p.OB = a.H; p.IA = a.Wo; p.IB = a.Ho;
        p.KA = a.KW; p.KB = a.KH; p.PA = a.KW - 1 - a.pw; p.PB = a.KH - 1 - a.ph;
        p.in_sA = C; p.in_sB = a.Wo * C; p.out_sA = C; p.out_sB = a.W * C;
        p.w_sA = a.C; p.w_sB = a.KW * a.C;
    } else {
        p.OA = a.H; p.OB = a.W; p.IA = a.Ho; p.IB = a.Wo;
        p.KA = a.KH; p.KB = a.KW; p.PA = a.KH - 1 - a.ph; p.PB = a.KW - 1 - a.pw;
        p.in_sA = a.Wo * C; p.in_sB = C; p.out_sA = a.W * C; p.out_sB = C;
        p.w_sA = a.KW * a.C; p.w_sB = a.C;
    }
    p.in_sN = static_cast<long long>(a.Ho) * a.Wo * C;
    p.out_sN = static_cast<long long>(a.H) * a.W * C;
    p.dx_bytes = p.out_sN * a.N * (a.elem_kind() == kF32 ? 4 : 2);
    p.status = a.status;

    int kai = 0;
    for (int v : kInstKA)
        if (v >= p.KA) { kai = v; break; }
    switch (kai) {
    case 1: return dispatch<1>(p, a.N, a.elem_kind(), stream);
    case 3: return dispatch<3>(p, a.N, a.elem_kind(), stream);
    case 5: return dispatch<5>(p, a.N, a.elem_kind(), stream);
    case 7: return dispatch<7>(p, a.N, a.elem_kind(), stream);
    case 9: return dispatch<9>(p, a.N, a.elem_kind(), stream);
    case 11: return dispatch<11>(p, a.N, a.elem_kind(), stream);
    case 13: return dispatch<13>(p, a.N, a.elem_kind(), stream);
    case 15: return dispatch<15>(p, a.N, a.elem_kind(), stream);
    case 17: return dispatch<17>(p, a.N, a.elem_kind(), stream);
    case 21: return dispatch<21>(p, a.N, a.elem_kind(), stream);
    case 25: return dispatch<25>(p, a.N, a.elem_kind(), stream);
    case 31: return dispatch<31>(p, a.N, a.elem_kind(), stream);
    case 33: return dispatch<33>(p, a.N, a.elem_kind(), stream);
    case 41: return dispatch<41>(p, a.N, a.elem_kind(), stream);
    case 51: return dispatch<51>(p, a.N, a.elem_kind(), stream);
    case 64: return dispatch<64>(p, a.N, a.elem_kind(), stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dgrad
