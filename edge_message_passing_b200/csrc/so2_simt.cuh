// Plain FP32 SIMT form of the per-m SO(2) block products, used to validate the
// tensor-core path: for each block b of a cohort,
//   Y[:, cols_b] = X[:, cols_b] @ B_b^T,  B_b the stacked (K_b x K_b) weight in [n][k] order.
#pragma once
#include "emp_common.cuh"

namespace emp {

__global__ void __launch_bounds__(256) k_so2_simt(int M, int C, const float* __restrict__ A,
                                                 const float* __restrict__ Bl, float* __restrict__ Cm) {
  const int b = blockIdx.z;
  const int K = blk_width(b) * C, N = K;
  const int n0 = blockIdx.y * 128, m0 = blockIdx.x * 128;
  if (n0 >= N) return;
  const float* Ab = A + blk_off(b) * C;
  const float* Bb = Bl + (size_t)wblk_off(b) * C * C;
  float* Cb = Cm + blk_off(b) * C;
  const size_t ld = (size_t)16 * C;
  __shared__ float As[16][132];
  __shared__ float Bs[16][132];
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int idx = t + q * 256, r = idx >> 4, kk = idx & 15;
      const int m = m0 + r, nn = n0 + r;
      As[kk][r] = (m < M) ? Ab[(size_t)m * ld + k0 + kk] : 0.f;
      Bs[kk][r] = (nn < N) ? Bb[(size_t)nn * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[8], bb[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) bb[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int nn = n0 + tx + 16 * j;
      if (nn < N) Cb[(size_t)m * ld + nn] = acc[i][j];
    }
  }
}

inline void so2_simt(int M, int C, const float* A, const float* B, float* Y, cudaStream_t s) {
  dim3 grid((M + 127) / 128, (6 * C + 127) / 128, 4);
  k_so2_simt<<<grid, 256, 0, s>>>(M, C, A, B, Y);
}

}  // namespace emp
