// toeplitz_core.cuh -- device pieces of the banded-Toeplitz depthwise MMA
// kernels: the padded filter-line format, the A-row builder (filter line ->
// tensor memory) and the MMA sequence of one shift step.
#pragma once

#include "common.cuh"

namespace dgrad {
namespace toep {

constexpr int kNumBarsNhwc = 18;   // mbarriers of the NHWC kernel (dw_toeplitz_nhwc.cu)
constexpr int kOff = 72;   // offset of filter tap 0 in a padded filter line (>= 64 + 8)

__host__ __device__ inline int floor8(int v) { return v >= 0 ? (v & ~7) : -((-v + 7) & ~7); }

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
    case 1: store_a_row<1>(taddr, src, odd, nonzero); break;
    case 2: store_a_row<2>(taddr, src, odd, nonzero); break;
    case 3: store_a_row<3>(taddr, src, odd, nonzero); break;
    case 4: store_a_row<4>(taddr, src, odd, nonzero); break;
    case 5: store_a_row<5>(taddr, src, odd, nonzero); break;
    case 6: store_a_row<6>(taddr, src, odd, nonzero); break;
    case 7: store_a_row<7>(taddr, src, odd, nonzero); break;
    case 8: store_a_row<8>(taddr, src, odd, nonzero); break;
    default: store_a_row<9>(taddr, src, odd, nonzero); break;
    }
}

// The MMAs of one shift step: for each 16-deep step q and sub-tile sx (sub-tiles
// innermost, so consecutive MMAs go to different accumulators), D_sx += A[:, 16q..]
// * B columns sx*TW + 16q ... (TW = 64 / XT).  The B descriptor of the step is
// precomputed; each MMA only adds a constant to it (start address field, units of
// 16 bytes: one 64-column panel is pb16, 16 columns are 2).
template <int KQ, int XT>
__device__ __forceinline__ void issue_step(const uint32_t (&d_tmem)[4], uint32_t a_tmem, uint64_t desc_i,
                                           uint32_t pb16, uint32_t idesc, bool first)
{
    constexpr int TW = 64 / XT;
#pragma unroll
    for (int q = 0; q < KQ; ++q) {
#pragma unroll
        for (int sx = 0; sx < XT; ++sx) {
            const int col = sx * TW + 16 * q;
            const uint64_t bd = desc_i + static_cast<uint64_t>((col >> 6) * pb16 + ((col & 63) >> 4) * 2);
            umma_f16_ts(d_tmem[sx], a_tmem + 8u * q, bd, idesc, (first && q == 0) ? 0u : 1u);
        }
    }
}

}  // namespace toep
}  // namespace dgrad
