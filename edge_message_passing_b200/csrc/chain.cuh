// Radial projection chain with the algebraic fold (page "deepmd-kit PR #6108:
// radial head fold", section "What"): W_eff = vstack_l(U_l M_l) (128 x 25) is
// formed once; per call kc = x_flat W_eff and y0 = x[:,0,:] U_0, and the input
// gradient g_x = g_kc W_eff^T (+ g_y0 U_0^T on degree 0).
#pragma once
#include "emp_common.cuh"

namespace emp {

struct Chain {
  float* Weff;   // [128][25]
  float* U0;     // [32][64]
  float* bfwd;   // tensor-core operand images (weights split into hi and lo) of the forward
  float* bbwd;   // and of the backward
  void* base;
};

// W_eff[k][j] = sum_h U_l[kk][h] M[64 l + h][j] with l = k / 32, kk = k % 32 (double accumulation)
__global__ void k_chain_fold(const float* __restrict__ U, const float* __restrict__ M, float* __restrict__ Weff,
                             float* __restrict__ U0) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx < 128 * 25) {
    const int k = idx / 25, j = idx % 25, l = k / 32, kk = k % 32;
    double s = 0.0;
    for (int h = 0; h < 64; ++h) s += (double)U[(l * 32 + kk) * 64 + h] * (double)M[(64 * l + h) * 25 + j];
    Weff[idx] = (float)s;
  }
  if (idx < 32 * 64) U0[idx] = U[idx];
}

}  // namespace emp
