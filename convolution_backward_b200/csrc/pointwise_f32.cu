// pointwise_f32.cu -- pointwise (1x1) dgrad in fp32: dX[M][C] = dY[M][K] * W[K][C].
//
// The pointwise shape class ("add the pointwise fast path dgrad was missing",
// Technical Details) as an fp32 GEMM on the FMA pipes.  fp32 inputs keep full
// precision: tensor-core tf32 would round the operands to 10 mantissa bits,
// far outside a 1e-5 relative tolerance.  Addressing is affine (m*K + k,
// k*C + c, m*C + c); the K-loop stages a 64 x 64 slice of dY and a 64 x 64
// slice of W in shared memory and each thread accumulates a 4 x 4 block.  The
// next slice is loaded into registers while the current one is consumed, so a
// short K (the small problems this kernel serves) costs one memory latency.
// When 64-row tiles would leave most SMs idle (a few hundred rows), the tiles
// are 16 rows high and each thread accumulates 1 x 4: four times the CTAs, a
// quarter of the serial FMA chain per thread.
// Requires K % 4 == 0 and C % 4 == 0 (16-byte rows), checked by the caller.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kTC = 64, kTK = 64;
constexpr int kThreads = 256;

// TM output rows per CTA (64 or 16); each thread accumulates RT = TM / 16 rows x 4 columns.
template <int TM>
__global__ void __launch_bounds__(kThreads)
    pw_f32_kernel(const float* __restrict__ dY, const float* __restrict__ W, float* __restrict__ dX, int M,
                  int K, int C, int* status)
{
    constexpr int RT = TM / 16;
    constexpr int kLdA = TM * kTK / 4 / kThreads;    // float4 loads per thread of a dY slice
    constexpr int kLdB = kTK * kTC / 4 / kThreads;   // of a W slice
    {
        // While the previous kernel may still run, only L2 prefetches of the first slice this
        // thread loads (L2 is the point of coherence, so the loads still see its writes).
        const int m = blockIdx.x * TM + (threadIdx.x >> 4);
        const int k = (threadIdx.x & 15) * 4;
        if (m < M && k < K) asm volatile("prefetch.global.L2 [%0];" ::"l"(dY + static_cast<int64_t>(m) * K + k));
        const int c = blockIdx.y * kTC + (threadIdx.x & 15) * 4;
        if ((threadIdx.x >> 4) < K && c < C)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(W + static_cast<int64_t>(threadIdx.x >> 4) * C + c));
    }
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    __shared__ __align__(16) float As[kTK][TM + 4];    // dY slice, stored k-major
    __shared__ __align__(16) float Bs[kTK][kTC];       // W slice
    const int tid = threadIdx.x;
    const int tx = tid & 15;             // 4 output columns each
    const int ty = tid >> 4;             // RT output rows each
    const int m0 = blockIdx.x * TM;
    const int c0 = blockIdx.y * kTC;

    float4 ra[kLdA], rb[kLdB];
    // load j of a slice: dY row (tid + 256 j) / 16, k chunk (tid % 16);
    // W row (tid + 256 j) / 16, c chunk (tid % 16)
    auto load = [&](int k0) {
#pragma unroll
        for (int j = 0; j < kLdA; ++j) {
            const int it = tid + j * kThreads;
            const int m = m0 + (it >> 4);
            const int k = k0 + (it & 15) * 4;
            ra[j] = (m < M && k < K) ? *reinterpret_cast<const float4*>(dY + static_cast<int64_t>(m) * K + k)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < kLdB; ++j) {
            const int it = tid + j * kThreads;
            const int kb = k0 + (it >> 4);
            const int c = c0 + (it & 15) * 4;
            rb[j] = (kb < K && c < C) ? *reinterpret_cast<const float4*>(W + static_cast<int64_t>(kb) * C + c)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    float acc[RT][4] = {};
    load(0);
    for (int k0 = 0; k0 < K; k0 += kTK) {
#pragma unroll
        for (int j = 0; j < kLdA; ++j) {
            const int it = tid + j * kThreads;
            const int ml = it >> 4, kl = (it & 15) * 4;
            As[kl + 0][ml] = ra[j].x;
            As[kl + 1][ml] = ra[j].y;
            As[kl + 2][ml] = ra[j].z;
            As[kl + 3][ml] = ra[j].w;
        }
#pragma unroll
        for (int j = 0; j < kLdB; ++j) {
            const int it = tid + j * kThreads;
            *reinterpret_cast<float4*>(&Bs[it >> 4][(it & 15) * 4]) = rb[j];
        }
        __syncthreads();
        if (k0 + kTK < K) load(k0 + kTK);   // in flight while this slice is consumed
#pragma unroll 16
        for (int kk = 0; kk < kTK; ++kk) {
            float av[RT];
            if constexpr (RT == 4) {
                const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
                av[0] = a.x;
                av[1] = a.y;
                av[2] = a.z;
                av[3] = a.w;
            } else {
#pragma unroll
                for (int i = 0; i < RT; ++i) av[i] = As[kk][ty * RT + i];
            }
            const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const int c = c0 + tx * 4;
    if (c >= C) return;
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int m = m0 + ty * RT + i;
        if (m < M && store_ok(dX, static_cast<long long>(M) * C * 4, dX + static_cast<int64_t>(m) * C + c, 16, status))
            *reinterpret_cast<float4*>(dX + static_cast<int64_t>(m) * C + c) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

}  // namespace

cudaError_t launch_pointwise_f32(const PwArgs& a, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    // 64-row tiles when they give at least 64 CTAs, 16-row tiles otherwise
    const long long nc = (a.C + kTC - 1) / kTC;
    const bool small = ((a.M + 63) / 64) * nc < 64;
    const int tm = small ? 16 : 64;
    dim3 grid(static_cast<unsigned>((a.M + tm - 1) / tm), static_cast<unsigned>(nc));
    {
        const cudaError_t le_ = launch_kernel(small ? pw_f32_kernel<16> : pw_f32_kernel<64>, dim3(grid),
                                             dim3(kThreads), 0, stream, 1,
                                             static_cast<const float*>(a.dY), static_cast<const float*>(a.W),
                                            static_cast<float*>(a.dX), static_cast<int>(a.M),
                                            static_cast<int>(a.K), static_cast<int>(a.C), a.status);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

}  // namespace dgrad
