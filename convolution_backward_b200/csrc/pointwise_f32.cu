// pointwise_f32.cu -- pointwise (1x1) dgrad in fp32: dX[M][C] = dY[M][K] * W[K][C].
//
// The pointwise shape class ("add the pointwise fast path dgrad was missing",
// Technical Details) as an fp32 GEMM on the FMA pipes.  fp32 inputs keep full
// precision: tensor-core tf32 would round the operands to 10 mantissa bits,
// far outside a 1e-5 relative tolerance.  Addressing is affine (m*K + k,
// k*C + c, m*C + c); the K-loop stages a 64 x 16 slice of dY and a 16 x 64
// slice of W in shared memory and each thread accumulates a 4 x 4 block.
// Requires K % 4 == 0 and C % 4 == 0 (16-byte rows), checked by the caller.
#include "common.cuh"
#include "launchers.h"

namespace dgrad {
namespace {

constexpr int kTM = 64, kTC = 64, kTK = 16;

__global__ void __launch_bounds__(256)
    pw_f32_kernel(const float* __restrict__ dY, const float* __restrict__ W, float* __restrict__ dX, int M,
                  int K, int C)
{
    __shared__ float As[kTK][kTM + 4];   // dY slice, stored k-major
    __shared__ float Bs[kTK][kTC];       // W slice
    const int tid = threadIdx.x;
    const int tx = tid & 15;             // 4 output columns each
    const int ty = tid >> 4;             // 4 output rows each
    const int m0 = blockIdx.x * kTM;
    const int c0 = blockIdx.y * kTC;

    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += kTK) {
        {   // dY[m0 + tid/4][k0 + 4*(tid%4) .. +3]
            const int m = m0 + (tid >> 2);
            const int k = k0 + (tid & 3) * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < M && k < K) v = *reinterpret_cast<const float4*>(dY + static_cast<int64_t>(m) * K + k);
            As[(tid & 3) * 4 + 0][tid >> 2] = v.x;
            As[(tid & 3) * 4 + 1][tid >> 2] = v.y;
            As[(tid & 3) * 4 + 2][tid >> 2] = v.z;
            As[(tid & 3) * 4 + 3][tid >> 2] = v.w;
        }
        {   // W[k0 + tid/16][c0 + 4*(tid%16) .. +3]
            const int k = k0 + (tid >> 4);
            const int c = c0 + (tid & 15) * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k < K && c < C) v = *reinterpret_cast<const float4*>(W + static_cast<int64_t>(k) * C + c);
            *reinterpret_cast<float4*>(&Bs[tid >> 4][(tid & 15) * 4]) = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kTK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    const int c = c0 + tx * 4;
    if (c >= C) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m < M)
            *reinterpret_cast<float4*>(dX + static_cast<int64_t>(m) * C + c) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

}  // namespace

cudaError_t launch_pointwise_f32(const PwArgs& a, cudaStream_t stream)
{
    if (a.M <= 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>((a.M + kTM - 1) / kTM), static_cast<unsigned>((a.C + kTC - 1) / kTC));
    pw_f32_kernel<<<grid, 256, 0, stream>>>(static_cast<const float*>(a.dY), static_cast<const float*>(a.W),
                                            static_cast<float*>(a.dX), static_cast<int>(a.M),
                                            static_cast<int>(a.K), static_cast<int>(a.C));
    return cudaGetLastError();
}

}  // namespace dgrad
