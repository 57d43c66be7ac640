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
// Requires K % 4 == 0 and C % 4 == 0 (16-byte rows), checked by the caller.
#include "common.cuh"
#include "host_util.h"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kTM = 64, kTC = 64, kTK = 64;
constexpr int kThreads = 256;
constexpr int kLd = kTM * kTK / 4 / kThreads;   // float4 loads per thread per operand slice

__global__ void __launch_bounds__(kThreads)
    pw_f32_kernel(const float* __restrict__ dY, const float* __restrict__ W, float* __restrict__ dX, int M,
                  int K, int C, int* status)
{
    pdl_wait();      // the previous kernel on the stream has finished
    pdl_trigger();   // the next one may start its set-up
    __shared__ __align__(16) float As[kTK][kTM + 4];   // dY slice, stored k-major (rows of 272 bytes)
    __shared__ __align__(16) float Bs[kTK][kTC];       // W slice
    const int tid = threadIdx.x;
    const int tx = tid & 15;             // 4 output columns each
    const int ty = tid >> 4;             // 4 output rows each
    const int m0 = blockIdx.x * kTM;
    const int c0 = blockIdx.y * kTC;

    float4 ra[kLd], rb[kLd];
    // load j of a slice: dY row (tid + 256 j) / 16, k chunk (tid % 16);
    // W row (tid + 256 j) / 16, c chunk (tid % 16)
    auto load = [&](int k0) {
#pragma unroll
        for (int j = 0; j < kLd; ++j) {
            const int it = tid + j * kThreads;
            const int m = m0 + (it >> 4);
            const int k = k0 + (it & 15) * 4;
            ra[j] = (m < M && k < K) ? *reinterpret_cast<const float4*>(dY + static_cast<int64_t>(m) * K + k)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            const int kb = k0 + (it >> 4);
            const int c = c0 + (it & 15) * 4;
            rb[j] = (kb < K && c < C) ? *reinterpret_cast<const float4*>(W + static_cast<int64_t>(kb) * C + c)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    float acc[4][4] = {};
    load(0);
    for (int k0 = 0; k0 < K; k0 += kTK) {
#pragma unroll
        for (int j = 0; j < kLd; ++j) {
            const int it = tid + j * kThreads;
            const int ml = it >> 4, kl = (it & 15) * 4;
            As[kl + 0][ml] = ra[j].x;
            As[kl + 1][ml] = ra[j].y;
            As[kl + 2][ml] = ra[j].z;
            As[kl + 3][ml] = ra[j].w;
            *reinterpret_cast<float4*>(&Bs[it >> 4][(it & 15) * 4]) = rb[j];
        }
        __syncthreads();
        if (k0 + kTK < K) load(k0 + kTK);   // in flight while this slice is consumed
#pragma unroll 16
        for (int kk = 0; kk < kTK; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const int c = c0 + tx * 4;
    if (c >= C) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m < M && store_ok(dX, static_cast<long long>(M) * C * 4, dX + static_cast<int64_t>(m) * C + c, 16, status))
            *reinterpret_cast<float4*>(dX + static_cast<int64_t>(m) * C + c) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

}  // namespace

cudaError_t launch_pointwise_f32(const PwArgs& a, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>((a.M + kTM - 1) / kTM), static_cast<unsigned>((a.C + kTC - 1) / kTC));
    {
        const cudaError_t le_ = launch_kernel(pw_f32_kernel, dim3(grid), dim3(kThreads), 0, stream, 1,
                                             static_cast<const float*>(a.dY), static_cast<const float*>(a.W),
                                            static_cast<float*>(a.dX), static_cast<int>(a.M),
                                            static_cast<int>(a.K), static_cast<int>(a.C), a.status);
        if (le_ != cudaSuccess) return le_;
    }
    return cudaGetLastError();
}

}  // namespace dgrad
