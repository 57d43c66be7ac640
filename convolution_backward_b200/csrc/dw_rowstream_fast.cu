// dw_rowstream_fast.cu -- row-streaming depthwise dgrad, register-blocked (bf16 or f16).
//
// The row-streaming schedule of "channel-packed and large-filter depthwise
// dgrad" (Technical Details, channel-packed row-streaming dgrad) for strided
// filters with compile-time KH, KW, S (KH >= S, KW >= S):
//   - dY rows stream through the kernel in order; dY row ho adds
//     dY[ho][wo] * W[r][s] into dX row h = ho*S - pad_h + r, column
//     x = wo*S - pad_w + s;
//   - once no later dY row can reach a dX row it is final and is written out;
//     the rows still open are carried in a circular accumulator buffer in
//     shared memory;
//   - after the last dY row the open rows are flushed (rows no dY row reaches
//     come out as zeros).
//
// B200 design.
//   * Work unit (one CTA): image n, 32 channels (16 pairs), a strip of TX dX
//     columns and a band of BH dX rows.  The band's dY rows (plus the
//     (KH-S)/S rows of halo above it) stream through a 6-deep TMA ring: each
//     stage is a 4-D tile [G dY rows][LW dY columns][32 channels] whose
//     out-of-image part the TMA fills with zeros, which is exactly the padding.
//   * Thread (pair cp, slot): a slot owns Q dX columns of one column phase
//     (x + pad_w) mod S, spaced S apart.  All taps reaching that phase have
//     the same parity s = s0, s0+S, ..., so the thread keeps just those
//     KH * ceil((KW-s0)/S) filter taps in registers, and Q + NT - 1 dY values
//     per row feed Q * KH * NT packed FMAs (fma.rn.f32x2 on channel pairs).
//   * G dY rows are applied per step, all in registers: they touch
//     (G-1)*S + KH dX rows, of which the first KH-S come in from the shared
//     accumulator ring (the rows left open by the previous step), the first
//     G*S are final afterwards and are rounded to 16 bits and stored, and the last
//     KH-S go back to the ring.  Ring entries are private to their thread, so
//     the ring needs no barriers; one __syncthreads per step recycles the TMA
//     stage.
//   * Waits on the TMA barriers are bounded and report a timeout instead of
//     hanging.
//   * The register-ring kernel (below) writes each step's final rows, rounded to
//     16 bits, into one of two staging buffers in shared memory ([TX columns][32
//     channels] per row); after the step's barrier lane 0 of every warp stores some
//     of the rows that lie in the CTA's band, one TMA box each, which clips the
//     ragged columns and channels.  The compute threads then spend one shared-memory
//     store per output instead of an address computation, a bounds test and a
//     global store (7x7 stride 2, 32 x 112 x 112 x 96 on B200: 43.0 us with direct
//     stores, 41.0 us with one thread issuing every box, 37.4 us with the boxes
//     spread over the warps, 35.8 us with one box of all of a step's rows when they
//     all lie in the band).
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

#include <algorithm>
#include <cstdlib>
#include <cstring>

namespace dgrad {
namespace {

constexpr int kStages = 6;
constexpr int kMaxThreads = 256;

struct FastParams {
    uint16_t* dX;         // 16-bit elements (bf16 or f16)
    const uint16_t* filt;
    int* status;
    int N, H, W, C, Ho, Wo, ph, pw;
    int nslot;    // slots per CTA (threads = 16 * nslot), a multiple of 2*S
    int TX;       // dX columns per strip = nslot * Q
    int LW;       // dY columns per staged row
    int BH;       // dX rows per band (multiple of G*S)
    int nX, nC, nB;
    int tma_out;          // register ring: final rows are staged in shared memory and stored by TMA
    long long dx_bytes;   // size of dX (index checks of the debug build)
};

template <int KH, int KW, int S, int Q, int G>
struct RsGeom {
    static constexpr int RB = (G - 1) * S + KH;   // dX rows one step touches
    static constexpr int NF = G * S;              // rows final after a step
    static constexpr int NC = KH - S;             // rows carried to the next step
    static constexpr int NTMAX = (KW + S - 1) / S;
    static_assert(KH >= S && KW >= S, "filter must be at least the stride");
    static_assert(Q % 2 == 0, "carried rows are stored as column pairs");
};

// One step with a fixed tap count NT (the thread's column phase has NT taps).
template <int KH, int KW, int S, int Q, int G, int NT, int EK>
__device__ __forceinline__ void rs_step(float2 (&acc)[RsGeom<KH, KW, S, Q, G>::RB][Q],
                                        const float2 (&wr)[KH][RsGeom<KH, KW, S, Q, G>::NTMAX],
                                        const uint32_t* stage, int LW, int cp, int col0)
{
    // stage: [G][LW][32 channels] 16-bit -> as uint32 pairs: [G][LW][16]
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float2 dv[Q + NT - 1];
        const uint32_t* row = stage + (g * LW + col0) * 16 + cp;
#pragma unroll
        for (int m = 0; m < Q + NT - 1; ++m) dv[m] = h16x2_to_float2<EK>(row[m * 16]);
        // taps outermost: consecutive FMAs update different accumulators
#pragma unroll
        for (int i = 0; i < NT; ++i)
#pragma unroll
            for (int r = 0; r < KH; ++r)
#pragma unroll
                for (int q = 0; q < Q; ++q)
                    acc[g * S + r][q] = ffma2(dv[q - i + NT - 1], wr[r][i], acc[g * S + r][q]);
    }
}

template <int KH, int KW, int S, int Q, int G, int EK>
__global__ void __launch_bounds__(kMaxThreads, 1)
    dw_rs_fast_kernel(const __grid_constant__ CUtensorMap dy_map, const FastParams p)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    using Geo = RsGeom<KH, KW, S, Q, G>;
    constexpr int RB = Geo::RB, NF = Geo::NF, NC = Geo::NC, NTMAX = Geo::NTMAX;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 127u) & ~127u) - raw);   // TMA destinations 128-byte aligned
    const int nthreads = 16 * p.nslot;
    const int stage_bytes = G * p.LW * 64;                       // 32 16-bit channels = 64 bytes
    const int stage_stride = (stage_bytes + 127) & ~127;         // TMA destinations are 128-byte aligned
    uint32_t* stages = reinterpret_cast<uint32_t*>(smem);
    float4* carry = reinterpret_cast<float4*>(smem + kStages * stage_stride);  // [NC][Q/2][nthreads]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * stage_stride +
                                                 NC * (Q / 2) * nthreads * sizeof(float4));

    int u = blockIdx.x;
    const int xblk = u % p.nX;
    u /= p.nX;
    const int band = u % p.nB;
    u /= p.nB;
    const int cblk = u % p.nC;
    const int n = u / p.nC;

    const int tid = threadIdx.x;
    const int cp = tid & 15;
    const int slot = tid >> 4;
    const int warp = slot >> 1;
    const int t = warp % S;                          // column offset of this slot's phase
    const int j = (warp / S) * 2 + (slot & 1);       // column group within the phase
    const int x0 = xblk * p.TX;
    const int c0 = cblk * 32;
    const int c = c0 + 2 * cp;
    const bool c_ok = c < p.C;
    const int s0 = ((x0 + t + p.pw) % S + S) % S;    // first tap reaching this phase
    const int nt = (KW - s0 + S - 1) / S;            // taps reaching it
    // dY column of tap (q = 0, i = 0) for this slot, and the strip's first staged column
    const int e = (x0 + t + p.pw - s0) / S + j * Q;
    const int wo_start = (x0 + p.pw - (KW - 1)) >= 0 ? (x0 + p.pw - (KW - 1)) / S
                                                       : -((-(x0 + p.pw - (KW - 1)) + S - 1) / S);
    const int col0 = e - (nt - 1) - wo_start;        // staged column of dv[0]
    // store addressing: dX row h of this thread's columns is obase + h*row_elems + xoff[q]
    const long long row_elems = static_cast<long long>(p.W) * p.C;
    uint16_t* obase = p.dX + static_cast<long long>(n) * p.H * row_elems + c;
    int xoff[Q];
    uint32_t xmask = 0;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        const int x = x0 + t + S * (j * Q + q);
        xoff[q] = x * p.C;
        if (x < p.W && c_ok) xmask |= 1u << q;
    }

    const int h0 = band * p.BH;
    const int h1 = min(h0 + p.BH, p.H);
    // first dY row reaching the band (halo rows above it contribute only to discarded rows)
    int ho_lo = h0 + p.ph - KH + 1;
    ho_lo = ho_lo <= 0 ? 0 : (ho_lo + S - 1) / S;
    const int hb0 = ho_lo * S - p.ph;                // first dX row of the first step
    const int nsteps = (h1 - hb0 + NF - 1) / NF;

    // filter taps of this phase, in registers: wr[r][i] = W[r][s0 + S*i]
    float2 wr[KH][NTMAX];
#pragma unroll
    for (int r = 0; r < KH; ++r)
#pragma unroll
        for (int i = 0; i < NTMAX; ++i) {
            const int s = s0 + S * i;
            float2 v = make_float2(0.f, 0.f);
            if (s < KW && c_ok)
                v = h16x2_to_float2<EK>(__ldg(reinterpret_cast<const uint32_t*>(p.filt + (r * KW + s) * p.C + c)));
            wr[r][i] = v;
        }
    // clear this thread's carried rows
#pragma unroll
    for (int r = 0; r < NC; ++r)
#pragma unroll
        for (int qh = 0; qh < Q / 2; ++qh) carry[(r * (Q / 2) + qh) * nthreads + tid] = make_float4(0.f, 0.f, 0.f, 0.f);

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int step) {
        const int sidx = step % kStages;
        mbar_arrive_expect_tx(&full[sidx], stage_bytes);
        // coordinates (channel, wo, ho, n); out-of-range parts are zero-filled
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(reinterpret_cast<uint8_t*>(stages) +
                                                                   sidx * stage_stride)),
            "l"(reinterpret_cast<uint64_t>(&dy_map)), "r"(smem_u32(&full[sidx])), "r"(c0), "r"(wo_start),
            "r"(ho_lo + step * G), "r"(n)
            : "memory");
    };
    int issued = 0;   // steps whose tile has been requested (thread 0's count)
    if (tid == 0) {
        tma_prefetch_desc(&dy_map);
        for (; issued < kStages - 1 && issued < nsteps; ++issued) issue(issued);
    }

    for (int step = 0; step < nsteps; ++step) {
        if (tid == 0 && issued < nsteps) issue(issued++);
        float2 acc[RB][Q];
#pragma unroll
        for (int r = 0; r < NC; ++r)
#pragma unroll
            for (int qh = 0; qh < Q / 2; ++qh) {
                const float4 v = carry[(r * (Q / 2) + qh) * nthreads + tid];
                acc[r][2 * qh] = make_float2(v.x, v.y);
                acc[r][2 * qh + 1] = make_float2(v.z, v.w);
            }
#pragma unroll
        for (int r = NC; r < RB; ++r)
#pragma unroll
            for (int q = 0; q < Q; ++q) acc[r][q] = make_float2(0.f, 0.f);

        const int sidx = step % kStages;
        const bool ok = mbar_wait(&full[sidx], static_cast<uint32_t>((step / kStages) & 1));
        // every thread leaves together if any of them gave up waiting
        if (__syncthreads_or(!ok)) {
            if (tid == 0) report_timeout(p.status);
            break;
        }
        const uint32_t* stage = reinterpret_cast<const uint32_t*>(reinterpret_cast<uint8_t*>(stages) +
                                                                  sidx * stage_stride);
        if (nt == NTMAX)
            rs_step<KH, KW, S, Q, G, NTMAX, EK>(acc, wr, stage, p.LW, cp, col0);
        else
            rs_step<KH, KW, S, Q, G, NTMAX - 1, EK>(acc, wr, stage, p.LW, cp, col0);

        // rows hb .. hb+NF-1 are final
        const int hb = hb0 + step * NF;
#pragma unroll
        for (int i = 0; i < NF; ++i) {
            const int h = hb + i;
            if (h >= h0 && h < h1) {
                uint16_t* orow = obase + static_cast<long long>(h) * row_elems;
#pragma unroll
                for (int q = 0; q < Q; ++q)
                    if (((xmask >> q) & 1u) && store_ok(p.dX, p.dx_bytes, orow + xoff[q], 4, p.status))
                        *reinterpret_cast<uint32_t*>(orow + xoff[q]) = float2_to_h16x2<EK>(acc[i][q].x, acc[i][q].y);
            }
        }
        // rows hb+NF .. hb+RB-1 stay open: back to the ring
#pragma unroll
        for (int r = 0; r < NC; ++r)
#pragma unroll
            for (int qh = 0; qh < Q / 2; ++qh)
                carry[(r * (Q / 2) + qh) * nthreads + tid] =
                    make_float4(acc[NF + r][2 * qh].x, acc[NF + r][2 * qh].y, acc[NF + r][2 * qh + 1].x,
                                acc[NF + r][2 * qh + 1].y);
        __syncthreads();   // every thread is done with this stage before it is refilled
    }
    // Let every requested tile land before the CTA's shared memory can be reused.
    if (tid == 0)
        for (int s = (issued > kStages ? issued - kStages : 0); s < issued; ++s)
            if (!mbar_wait(&full[s % kStages], static_cast<uint32_t>((s / kStages) & 1))) report_timeout(p.status);
}

// ---------------------------------------------------------------------------
// Register-ring variant.  The circular accumulator slots live in registers, as
// in the pages' design (their accumulator-slot budget is a register budget):
// acc[RS][Q] with RS >= KH slots, dX row h in slot (h - hb0) mod RS.  Each TMA
// stage carries GT dY rows and S*GT is a multiple of RS, so inside a stage every
// slot index is a compile-time constant and the ring "rotates" by renaming;
// nothing is carried through shared memory and there is one barrier per stage.
// After dY row t of the band the S rows in slots (S*t .. S*t+S-1) mod RS are
// final: they are stored (if inside the band) and cleared.
template <int KH, int KW, int S, int Q, int RS, int GT, int NT, int EK, bool TMA_OUT>
__device__ __forceinline__ void rs_reg_stage(float2 (&acc)[RS][Q], const float2 (&wr)[KH][(KW + S - 1) / S],
                                             const uint32_t* stage, int LW, int cp, int col0, int hb, int h0,
                                             int h1, uint16_t* obase, long long row_elems,
                                             const int (&xoff)[Q], uint32_t xmask, const void* dx_base,
                                             long long dx_bytes, int* status, uint32_t* stg,
                                             const int (&soff)[Q], int row_words)
{
    static_assert((S * GT) % RS == 0 && RS >= KH && KH >= S, "ring geometry");
    // dY row k of the stage, converted to fp32 pairs; row k+1 is loaded while row k computes
    float2 dv[Q + NT - 1];
    auto load_row = [&](int k, float2 (&d)[Q + NT - 1]) {
        const uint32_t* row = stage + (k * LW + col0) * 16 + cp;
#pragma unroll
        for (int m = 0; m < Q + NT - 1; ++m) d[m] = h16x2_to_float2<EK>(row[m * 16]);
    };
    load_row(0, dv);
#pragma unroll
    for (int k = 0; k < GT; ++k) {
        float2 nx[Q + NT - 1];
        if (k + 1 < GT) load_row(k + 1, nx);
        // Taps outermost: consecutive FMAs go to the KH * Q different accumulators,
        // so no FMA waits on the one just before it.  Rows r >= KH-S are touched
        // for the first time (their slot was flushed earlier), so their first tap
        // is a multiply, not an add onto a cleared slot.
#pragma unroll
        for (int i = 0; i < NT; ++i)
#pragma unroll
            for (int r = 0; r < KH; ++r)
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    float2& a = acc[(S * k + r) % RS][q];
                    const float2 x = dv[q - i + NT - 1];
                    if (r >= KH - S && i == 0)
                        a = make_float2(x.x * wr[r][0].x, x.y * wr[r][0].y);
                    else
                        a = ffma2(x, wr[r][i], a);
                }
#pragma unroll
        for (int i = 0; i < S; ++i) {
            const int slot = (S * k + i) % RS;
            if (TMA_OUT) {
                // staged row S*k + i of this stage: [TX columns][32 channels]; rows outside the
                // band, columns past the image and channels past C are never stored
                uint32_t* srow = stg + (S * k + i) * row_words;
#pragma unroll
                for (int q = 0; q < Q; ++q) srow[soff[q]] = float2_to_h16x2<EK>(acc[slot][q].x, acc[slot][q].y);
                continue;
            }
            const int h = hb + S * k + i;
            if (h >= h0 && h < h1) {
                uint16_t* orow = obase + static_cast<long long>(h) * row_elems;
#pragma unroll
                for (int q = 0; q < Q; ++q)
                    if (((xmask >> q) & 1u) && store_ok(dx_base, dx_bytes, orow + xoff[q], 4, status))
                        *reinterpret_cast<uint32_t*>(orow + xoff[q]) =
                            float2_to_h16x2<EK>(acc[slot][q].x, acc[slot][q].y);
            }
        }
        if (k + 1 < GT)
#pragma unroll
            for (int m = 0; m < Q + NT - 1; ++m) dv[m] = nx[m];
    }
}

template <int KH, int KW, int S, int Q, int RS, int GT, int EK>
__global__ void __launch_bounds__(kMaxThreads, 1)
    dw_rs_reg_kernel(const __grid_constant__ CUtensorMap dy_map, const __grid_constant__ CUtensorMap dx_map,
                     const __grid_constant__ CUtensorMap dx_map8, const FastParams p)
{
    constexpr int NTMAX = (KW + S - 1) / S;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 127u) & ~127u) - raw);
    const int stage_bytes = GT * p.LW * 64;
    const int stage_stride = (stage_bytes + 127) & ~127;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * stage_stride);

    int u = blockIdx.x;
    const int xblk = u % p.nX;
    u /= p.nX;
    const int band = u % p.nB;
    u /= p.nB;
    const int cblk = u % p.nC;
    const int n = u / p.nC;
    const int tid = threadIdx.x;
    const int cp = tid & 15;
    const int slot = tid >> 4;
    const int warp = slot >> 1;
    const int t = warp % S;
    const int j = (warp / S) * 2 + (slot & 1);
    const int x0 = xblk * p.TX;
    const int c0 = cblk * 32;
    const int c = c0 + 2 * cp;
    const bool c_ok = c < p.C;
    const int s0 = (x0 + t + p.pw) % S;
    const int nt = (KW - s0 + S - 1) / S;
    const int e = (x0 + t + p.pw - s0) / S + j * Q;
    const int wo_start = (x0 + p.pw - (KW - 1)) >= 0 ? (x0 + p.pw - (KW - 1)) / S
                                                       : -((-(x0 + p.pw - (KW - 1)) + S - 1) / S);
    const int col0 = e - (nt - 1) - wo_start;
    const long long row_elems = static_cast<long long>(p.W) * p.C;
    uint16_t* obase = p.dX + static_cast<long long>(n) * p.H * row_elems + c;
    int xoff[Q], soff[Q];
    uint32_t xmask = 0;
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        const int x = x0 + t + S * (j * Q + q);
        xoff[q] = x * p.C;
        soff[q] = (x - x0) * 16 + cp;   // word of the staged row: [TX columns][16 channel pairs]
        if (x < p.W && c_ok) xmask |= 1u << q;
    }
    // staged output rows (tma_out): two buffers of GT*S rows of TX columns x 32 channels
    const int row_words = p.TX * 16;
    uint32_t* stg0 = reinterpret_cast<uint32_t*>(
        smem + ((kStages * stage_stride + kStages * 8 + 127) & ~127));
    const int h0 = band * p.BH;
    const int h1 = min(h0 + p.BH, p.H);
    int ho_lo = h0 + p.ph - KH + 1;
    ho_lo = ho_lo <= 0 ? 0 : (ho_lo + S - 1) / S;
    const int hb0 = ho_lo * S - p.ph;
    const int nrows = (h1 - hb0 + S - 1) / S;          // dY rows until every band row is final
    const int nstages = (nrows + GT - 1) / GT;
    if (tid == 0) {
        // While the previous kernel may still run, only L2 prefetches of the first stages'
        // tiles (L2 is the point of coherence, so the loads still see that kernel's writes).
        tma_prefetch_desc(&dy_map);
        for (int st = 0; st < kStages - 1 && st < nstages; ++st)
            tma_prefetch_l2_4d(&dy_map, c0, wo_start, ho_lo + st * GT, n);
    }
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up

    float2 wr[KH][NTMAX];
#pragma unroll
    for (int r = 0; r < KH; ++r)
#pragma unroll
        for (int i = 0; i < NTMAX; ++i) {
            const int sx = s0 + S * i;
            wr[r][i] = (sx < KW && c_ok)
                           ? h16x2_to_float2<EK>(__ldg(reinterpret_cast<const uint32_t*>(p.filt + (r * KW + sx) * p.C + c)))
                           : make_float2(0.f, 0.f);
        }
    if (tid == 0) {
        for (int sidx = 0; sidx < kStages; ++sidx) mbar_init(&full[sidx], 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int st) {
        const int sidx = st % kStages;
        mbar_arrive_expect_tx(&full[sidx], stage_bytes);
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem + sidx * stage_stride)),
            "l"(reinterpret_cast<uint64_t>(&dy_map)), "r"(smem_u32(&full[sidx])), "r"(c0), "r"(wo_start),
            "r"(ho_lo + st * GT), "r"(n)
            : "memory");
    };
    int issued = 0;
    if (tid == 0)
        for (; issued < kStages - 1 && issued < nstages; ++issued) issue(issued);

    float2 acc[RS][Q];
#pragma unroll
    for (int i = 0; i < RS; ++i)
#pragma unroll
        for (int q = 0; q < Q; ++q) acc[i][q] = make_float2(0.f, 0.f);

    // tma_out: lane 0 of every warp stores some of each stage's rows (rows warp, warp + nwarps,
    // ...), so the issue is spread and no one thread holds the next barrier up
    const bool storer = p.tma_out && (tid & 31) == 0;
    const int nwarps = static_cast<int>(blockDim.x) >> 5;
    for (int st = 0; st < nstages; ++st) {
        if (tid == 0 && issued < nstages) issue(issued++);
        // the staging buffer of this stage was last stored two stages ago: its reads are done
        if (storer) bulk_wait_group_read<1>();
        const int sidx = st % kStages;
        const bool ok = mbar_wait(&full[sidx], static_cast<uint32_t>((st / kStages) & 1));
        if (__syncthreads_or(!ok)) {
            if (tid == 0) report_timeout(p.status);
            break;
        }
        const uint32_t* stage = reinterpret_cast<const uint32_t*>(smem + sidx * stage_stride);
        const int hb = hb0 + st * GT * S;
        uint32_t* stg = stg0 + (st & 1) * (GT * S) * row_words;
        if (p.tma_out) {
            if (nt == NTMAX)
                rs_reg_stage<KH, KW, S, Q, RS, GT, NTMAX, EK, true>(acc, wr, stage, p.LW, cp, col0, hb, h0, h1, obase,
                                                                row_elems, xoff, xmask, p.dX, p.dx_bytes, p.status,
                                                                stg, soff, row_words);
            else
                rs_reg_stage<KH, KW, S, Q, RS, GT, NTMAX - 1, EK, true>(acc, wr, stage, p.LW, cp, col0, hb, h0, h1,
                                                                    obase, row_elems, xoff, xmask, p.dX,
                                                                    p.dx_bytes, p.status, stg, soff, row_words);
            fence_proxy_async_smem();   // the TMA store reads the staged rows through the async proxy
        } else if (nt == NTMAX) {
            rs_reg_stage<KH, KW, S, Q, RS, GT, NTMAX, EK, false>(acc, wr, stage, p.LW, cp, col0, hb, h0, h1, obase,
                                                             row_elems, xoff, xmask, p.dX, p.dx_bytes, p.status, stg,
                                                             soff, row_words);
        } else {
            rs_reg_stage<KH, KW, S, Q, RS, GT, NTMAX - 1, EK, false>(acc, wr, stage, p.LW, cp, col0, hb, h0, h1,
                                                                 obase, row_elems, xoff, xmask, p.dX, p.dx_bytes,
                                                                 p.status, stg, soff, row_words);
        }
        __syncthreads();
        if (storer) {
            // the stage's final rows hb .. hb + GT*S - 1 that lie in this band: one box of all
            // of them when they all do (thread 0), else one row box each (TMA clips columns
            // past W and channels past C)
            if (hb >= h0 && hb + GT * S <= h1) {
                if (warp == 0) tma_store_4d(&dx_map8, stg, c0, x0, hb, n);
            } else {
#pragma unroll 1
                for (int r = warp; r < GT * S; r += nwarps) {
                    const int h = hb + r;
                    if (h >= h0 && h < h1) tma_store_4d(&dx_map, stg + r * row_words, c0, x0, h, n);
                }
            }
            bulk_commit_group();
        }
    }
    if (tid == 0)
        for (int sx = (issued > kStages ? issued - kStages : 0); sx < issued; ++sx)
            if (!mbar_wait(&full[sx % kStages], static_cast<uint32_t>((sx / kStages) & 1))) report_timeout(p.status);
    if (storer) bulk_wait_group<0>();   // the staged rows have been written
}

// Shared memory of one CTA: the TMA stages (G dY rows of LW columns each), their
// barriers and, for the shared-ring kernel, the carried accumulator rows.
inline size_t stage_smem(int G, int LW) { return static_cast<size_t>(kStages) * ((G * LW * 64 + 127) & ~127); }
inline size_t fast_smem(int G, int LW, int NC, int Q, int nthreads)
{
    return stage_smem(G, LW) + static_cast<size_t>(NC) * (Q / 2) * nthreads * sizeof(float4) + kStages * 8 + 128;
}
inline size_t reg_smem(int GT, int LW, int S = 1, int TX = 0)
{
    // stages, barriers, then (staged output) two buffers of GT*S rows of TX columns x 64 bytes
    return ((stage_smem(GT, LW) + kStages * 8 + 127) & ~static_cast<size_t>(127)) +
           2 * static_cast<size_t>(GT) * S * TX * 64 + 128;
}

// Strip and band plan.  kern / smem (the kernel that will run and its dynamic
// shared memory per CTA) size the bands; without them one band covers dX.
template <int KH, int KW, int S, int Q, int G>
FastParams plan_fast(const DwArgs& a, const void* kern = nullptr, size_t (*smem_of)(int LW, int nthreads) = nullptr)
{
    static_assert(KH >= S && KW >= S, "filter must be at least the stride");
    FastParams p{};
    p.dX = static_cast<uint16_t*>(a.dX);
    p.filt = static_cast<const uint16_t*>(a.filt);
    p.status = a.status;
    p.N = a.N; p.H = a.H; p.W = a.W; p.C = a.C; p.Ho = a.Ho; p.Wo = a.Wo; p.ph = a.ph; p.pw = a.pw;
    p.dx_bytes = static_cast<long long>(a.N) * a.H * a.W * a.C * 2;
    // strip width: pick the slot count (multiple of 2*S, at most 16) that wastes the fewest columns
    int best = -1, best_waste = 1 << 30;
    for (int ns = 16; ns >= 2 * S; ns -= 2 * S) {
        const int tx = ns * Q;
        const int strips = (a.W + tx - 1) / tx;
        const int waste = strips * tx - a.W;
        if (waste < best_waste) {
            best_waste = waste;
            best = ns;
        }
    }
    p.nslot = best;
    p.TX = best * Q;
    p.LW = (p.TX - 1 + KW - 1) / S + 2;
    p.nX = (a.W + p.TX - 1) / p.TX;
    p.nC = (a.C + 31) / 32;
    // Bands: band rows are a multiple of G*S.  Each band streams its BH/S dY rows
    // plus (KH-S)/S rows of halo above it and pays a fixed start (filter taps,
    // pipeline fill), so a CTA costs about BH/S + (KH-S)/S + 2 dY rows; the CTAs
    // run in ceil(CTAs / resident slots) waves.  The band count minimises waves
    // times CTA cost, which avoids a nearly empty last wave.
    const int nf = G * S;
    const long long base = static_cast<long long>(a.N) * p.nC * p.nX;
    const int nthreads = 16 * p.nslot;
    int per_sm = 1;
    if (kern && smem_of) {
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nthreads, smem_of(p.LW, nthreads)) ==
                cudaSuccess &&
            occ >= 1)
            per_sm = occ;
    }
    const long long slots = static_cast<long long>(device_sm_count()) * per_sm;
    const int max_nb = kern ? std::min(16, (a.H + nf - 1) / nf) : 1;
    int nb_best = 1;
    double cost_best = 0.0;
    for (int nb = 1; nb <= max_nb; ++nb) {
        int bh = (a.H + nb - 1) / nb;
        bh = ((bh + nf - 1) / nf) * nf;
        const int bands = (a.H + bh - 1) / bh;
        const long long waves = (base * bands + slots - 1) / slots;
        const double cost = static_cast<double>(waves) * (static_cast<double>(bh + KH - S) / S + 2.0);
        if (nb == 1 || cost < cost_best - 1e-9) {
            cost_best = cost;
            nb_best = nb;
        }
    }
    // DGRAD_RS_BANDS=n forces the band count (testing and tuning)
    if (const char* eb = dgrad::tuning_env("DGRAD_RS_BANDS"))
        if (atoi(eb) >= 1 && kern) nb_best = std::min(atoi(eb), max_nb);
    int bh = (a.H + nb_best - 1) / nb_best;
    bh = ((bh + nf - 1) / nf) * nf;
    p.BH = bh;
    p.nB = (a.H + bh - 1) / bh;
    return p;
}

template <int KH, int KW, int S, int Q, int G>
cudaError_t launch_fast(const DwArgs& a, const CUtensorMap& map, cudaStream_t stream)
{
    using Geo = RsGeom<KH, KW, S, Q, G>;
    auto kern = a.f16 ? dw_rs_fast_kernel<KH, KW, S, Q, G, kF16> : dw_rs_fast_kernel<KH, KW, S, Q, G, kBF16>;
    auto smem_of = [](int lw, int nthreads) { return fast_smem(G, lw, Geo::NC, Q, nthreads); };
    const FastParams p = plan_fast<KH, KW, S, Q, G>(a, reinterpret_cast<const void*>(kern), smem_of);
    const long long blocks = static_cast<long long>(a.N) * p.nC * p.nX * p.nB;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    const int nthreads = 16 * p.nslot;
    const size_t smem = fast_smem(G, p.LW, Geo::NC, Q, nthreads);
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(static_cast<unsigned>(blocks)), dim3(nthreads), smem, stream, 1,
                                             map, p);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

// DGRAD_RS_STORE=direct keeps the register-ring kernel's direct 4-byte stores of dX
// (testing and tuning); by default its final rows are staged and stored by TMA.
static bool rs_direct_store()
{
    const char* e = dgrad::tuning_env("DGRAD_RS_STORE");
    return e && strcmp(e, "direct") == 0;
}

template <int KH, int KW, int S, int Q, int RS, int GT>
cudaError_t launch_reg(const DwArgs& a, const CUtensorMap& map, const CUtensorMap* dx_map,
                       const CUtensorMap* dx_map8, cudaStream_t stream)
{
    // plan as the shared-ring kernel with G = GT (band rows a multiple of S*GT)
    auto kern = a.f16 ? dw_rs_reg_kernel<KH, KW, S, Q, RS, GT, kF16> : dw_rs_reg_kernel<KH, KW, S, Q, RS, GT, kBF16>;
    const bool tma_out = dx_map != nullptr && dx_map8 != nullptr && !rs_direct_store();
    auto smem_tma = [](int lw, int nthreads) { return reg_smem(GT, lw, S, (nthreads / 16) * Q); };
    auto smem_direct = [](int lw, int) { return reg_smem(GT, lw); };
    FastParams p = plan_fast<KH, KW, S, Q, GT>(a, reinterpret_cast<const void*>(kern),
                                               tma_out ? +smem_tma : +smem_direct);
    p.tma_out = tma_out ? 1 : 0;
    const long long blocks = static_cast<long long>(a.N) * p.nC * p.nX * p.nB;
    if (blocks <= 0) return cudaSuccess;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    const int nthreads = 16 * p.nslot;
    const size_t smem = tma_out ? reg_smem(GT, p.LW, S, p.TX) : reg_smem(GT, p.LW);
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    {
        const cudaError_t le_ = launch_kernel(kern, dim3(static_cast<unsigned>(blocks)), dim3(nthreads), smem, stream, 1,
                                             map, tma_out ? *dx_map : map, tma_out ? *dx_map8 : map, p);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

}  // namespace

// Register-ring set: (KH, KW, S) -> (Q, ring slots RS, dY rows per stage GT).
// Two output columns per thread: twice the threads of four columns at two thirds
// of the registers, which measured 7% faster on the 7x7 stride-2 workload.
#define DGRAD_RS_REG_SET(X) \
    X(7, 7, 2, 2, 8, 4)     \
    X(5, 5, 2, 2, 8, 4)     \
    X(3, 3, 2, 2, 4, 4)

// Four output columns per thread, selected with DGRAD_RS_Q=4.
#define DGRAD_RS_REG_Q4_SET(X) \
    X(7, 7, 2, 4, 8, 4)        \
    X(5, 5, 2, 4, 8, 4)        \
    X(3, 3, 2, 4, 4, 4)

static bool reg_q4()
{
    const char* e = dgrad::tuning_env("DGRAD_RS_Q");
    return e && atoi(e) == 4;
}

static bool use_reg_ring()
{
    const char* e = dgrad::tuning_env("DGRAD_RS_KERNEL");
    return !(e && strcmp(e, "smem") == 0);
}

// The compiled set: (KH, KW, S) -> (Q, G).
#define DGRAD_RS_FAST_SET(X) \
    X(7, 7, 2, 4, 2)         \
    X(5, 5, 2, 4, 2)         \
    X(3, 3, 2, 4, 4)

// Alternative step depths (G), selected with DGRAD_RS_G for tuning.
#define DGRAD_RS_ALT_SET(X) \
    X(7, 7, 2, 4, 1)         \
    X(5, 5, 2, 4, 1)         \
    X(3, 3, 2, 4, 2)

static int alt_g()
{
    const char* e = dgrad::tuning_env("DGRAD_RS_G");
    return e && *e ? atoi(e) : 0;
}

bool dw_rowstream_fast_box(const DwArgs& a, unsigned box[4], unsigned box_dx[4], unsigned* rows_dx8)
{
    if (!(a.bf16 || a.f16)) return false;
    box_dx[0] = 32; box_dx[1] = 1; box_dx[2] = 1; box_dx[3] = 1;
    *rows_dx8 = 1;
    if (use_reg_ring()) {
#define DGRAD_RS_REG_BOX(kh, kw, s, q, rs, gt)                                                     \
        if (a.KH == kh && a.KW == kw && a.S == s) {                                                 \
            const FastParams p = plan_fast<kh, kw, s, q, gt>(a);                                    \
            box[0] = 32; box[1] = static_cast<unsigned>(p.LW); box[2] = gt; box[3] = 1;            \
            box_dx[1] = static_cast<unsigned>(p.TX);                                                \
            *rows_dx8 = static_cast<unsigned>(gt * s);                                              \
            return true;                                                                            \
        }
        if (reg_q4()) { DGRAD_RS_REG_Q4_SET(DGRAD_RS_REG_BOX) }
        DGRAD_RS_REG_SET(DGRAD_RS_REG_BOX)
#undef DGRAD_RS_REG_BOX
        return false;
    }
    const int ga = alt_g();
#define DGRAD_RS_BOX(kh, kw, s, q, g)                                  \
    if (a.KH == kh && a.KW == kw && a.S == s && (ga == 0 || ga == g)) { \
        const FastParams p = plan_fast<kh, kw, s, q, g>(a);            \
        box[0] = 32; box[1] = static_cast<unsigned>(p.LW); box[2] = g; box[3] = 1; \
        return true;                                                   \
    }
    if (ga != 0) { DGRAD_RS_ALT_SET(DGRAD_RS_BOX) }
    DGRAD_RS_FAST_SET(DGRAD_RS_BOX)
#undef DGRAD_RS_BOX
    return false;
}

// Returns cudaErrorNotSupported when no specialised instantiation serves the problem.
cudaError_t launch_dw_rowstream_fast(const DwArgs& a, const CUtensorMap& dy_map, const CUtensorMap* dx_map,
                                     const CUtensorMap* dx_map8, int G, cudaStream_t stream)
{
    (void)G;
    if (!(a.bf16 || a.f16)) return cudaErrorNotSupported;
    if (use_reg_ring()) {
#define DGRAD_RS_REG_LAUNCH(kh, kw, s, q, rs, gt) \
        if (a.KH == kh && a.KW == kw && a.S == s) return launch_reg<kh, kw, s, q, rs, gt>(a, dy_map, dx_map, dx_map8, stream);
        if (reg_q4()) { DGRAD_RS_REG_Q4_SET(DGRAD_RS_REG_LAUNCH) }
        DGRAD_RS_REG_SET(DGRAD_RS_REG_LAUNCH)
#undef DGRAD_RS_REG_LAUNCH
        return cudaErrorNotSupported;
    }
    const int ga = alt_g();
#define DGRAD_RS_LAUNCH(kh, kw, s, q, g) \
    if (a.KH == kh && a.KW == kw && a.S == s && (ga == 0 || ga == g)) return launch_fast<kh, kw, s, q, g>(a, dy_map, stream);
    if (ga != 0) { DGRAD_RS_ALT_SET(DGRAD_RS_LAUNCH) }
    DGRAD_RS_FAST_SET(DGRAD_RS_LAUNCH)
#undef DGRAD_RS_LAUNCH
    return cudaErrorNotSupported;
}

}  // namespace dgrad
