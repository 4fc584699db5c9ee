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

constexpr int CH_ROWS = 128;

struct ChainFwdSmem {
  float sx[CH_ROWS][129];
  float sw[128][32];          // W_eff padded to 32 columns
  float su[32][64];
};
struct ChainBwdSmem {
  float sg[CH_ROWS][26];
  float sh[CH_ROWS][65];
  float sw[25][128];          // W_eff^T
  float su[64][32];           // U0^T
};

// forward: 128 rows per block, 256 threads; thread = (row group of 8, output group)
__global__ void __launch_bounds__(256) k_chain_fwd(long long E, const float* __restrict__ x,
                                                  const float* __restrict__ Weff, const float* __restrict__ U0,
                                                  float* __restrict__ kc, float* __restrict__ y0) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChainFwdSmem& S = *reinterpret_cast<ChainFwdSmem*>(smem_raw);
  auto& sx = S.sx;
  auto& sw = S.sw;
  auto& su = S.su;
  const int t = threadIdx.x;
  const long long r0 = (long long)blockIdx.x * CH_ROWS;
  for (int idx = t; idx < 128 * 32; idx += 256) {
    const int k = idx >> 5, j = idx & 31;
    sw[k][j] = j < 25 ? Weff[k * 25 + j] : 0.f;
  }
  for (int idx = t; idx < 32 * 64; idx += 256) su[idx >> 6][idx & 63] = U0[idx];
  for (int idx = t; idx < CH_ROWS * 128; idx += 256) {
    const int r = idx >> 7, k = idx & 127;
    const long long e = r0 + r;
    sx[r][k] = e < E ? x[(size_t)e * 128 + k] : 0.f;
  }
  __syncthreads();
  // kc: 128 rows x 32 cols -> thread: 8 rows (rg + 16 i) x 2 cols (cg, cg + 16)
  {
    const int rg = t >> 4, cg = t & 15;
    float acc[8][2];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = 0.f;
    for (int k = 0; k < 128; ++k) {
      const float w0 = sw[k][cg], w1 = sw[k][cg + 16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = sx[rg + 16 * i][k];
        acc[i][0] = fmaf(a, w0, acc[i][0]);
        acc[i][1] = fmaf(a, w1, acc[i][1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long e = r0 + rg + 16 * i;
      if (e < E) {
        kc[(size_t)e * 25 + cg] = acc[i][0];
        if (cg + 16 < 25) kc[(size_t)e * 25 + cg + 16] = acc[i][1];
      }
    }
  }
  // y0: 128 rows x 64 cols over k < 32 -> thread: 8 rows x 4 cols
  {
    const int rg = t >> 4, cg = t & 15;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k = 0; k < 32; ++k) {
      float w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j] = su[k][cg + 16 * j];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = sx[rg + 16 * i][k];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a, w[j], acc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long e = r0 + rg + 16 * i;
      if (e < E)
#pragma unroll
        for (int j = 0; j < 4; ++j) y0[(size_t)e * 64 + cg + 16 * j] = acc[i][j];
    }
  }
}

// input gradient: g_x [E][128]
__global__ void __launch_bounds__(256) k_chain_bwd(long long E, const float* __restrict__ g_kc,
                                                  const float* __restrict__ g_y0, const float* __restrict__ Weff,
                                                  const float* __restrict__ U0, float* __restrict__ g_x) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChainBwdSmem& S = *reinterpret_cast<ChainBwdSmem*>(smem_raw);
  auto& sg = S.sg;
  auto& sh = S.sh;
  auto& sw = S.sw;
  auto& su = S.su;
  const int t = threadIdx.x;
  const long long r0 = (long long)blockIdx.x * CH_ROWS;
  for (int idx = t; idx < 128 * 25; idx += 256) sw[idx % 25][idx / 25] = Weff[idx];
  for (int idx = t; idx < 32 * 64; idx += 256) su[idx & 63][idx >> 6] = U0[idx];
  for (int idx = t; idx < CH_ROWS * 25; idx += 256) {
    const long long e = r0 + idx / 25;
    sg[idx / 25][idx % 25] = e < E ? g_kc[(size_t)r0 * 25 + idx] : 0.f;
  }
  for (int idx = t; idx < CH_ROWS * 64; idx += 256) {
    const long long e = r0 + (idx >> 6);
    sh[idx >> 6][idx & 63] = e < E ? g_y0[(size_t)r0 * 64 + idx] : 0.f;
  }
  __syncthreads();
  const int rg = t >> 4, cg = t & 15;   // 8 rows x 8 cols (cg + 16 j)
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int q = 0; q < 25; ++q) {
    float w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = sw[q][cg + 16 * j];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = sg[rg + 16 * i][q];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a, w[j], acc[i][j]);
    }
  }
  // degree-0 block (columns < 32): j = 0, 1 -> columns cg and cg + 16
  for (int h = 0; h < 64; ++h) {
    const float w0 = su[h][cg], w1 = su[h][cg + 16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = sh[rg + 16 * i][h];
      acc[i][0] = fmaf(a, w0, acc[i][0]);
      acc[i][1] = fmaf(a, w1, acc[i][1]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long e = r0 + rg + 16 * i;
    if (e < E)
#pragma unroll
      for (int j = 0; j < 8; ++j) g_x[(size_t)e * 128 + cg + 16 * j] = acc[i][j];
  }
}

}  // namespace emp
