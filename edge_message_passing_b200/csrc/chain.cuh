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

constexpr int CH_ROWS = 64;          // rows per tile
constexpr int CH_BUF = 2;            // tiles in flight per block (bulk-copy ring)

// The staged rows are padded (one bulk copy per row) so that the 4 rows a warp reads at
// one k fall into different banks.
constexpr int CH_XP = 132;           // pitch (floats) of the staged x rows
constexpr int CH_HP = 68;            // pitch (floats) of the staged g_y0 rows
struct ChainFwdSmem {
  float sx[CH_BUF][CH_ROWS][CH_XP];  // x tiles
  float sw[128][32];                 // W_eff padded to 32 columns
  float su[32][64];                  // U_0
  uint64_t full[CH_BUF];
};
struct ChainBwdSmem {
  float sg[CH_BUF][CH_ROWS * 25 + 28];   // g_kc tiles (rows of 25, contiguous; padded to 16 bytes)
  float sh[CH_BUF][CH_ROWS][CH_HP];      // g_y0 tiles
  float sw[25][128];                     // W_eff^T
  float su[64][32];                      // U_0^T
  uint64_t full[CH_BUF];
};

__device__ __forceinline__ float4 f4fma(float a, float4 b, float4 c) {
  return make_float4(fmaf(a, b.x, c.x), fmaf(a, b.y, c.y), fmaf(a, b.z, c.z), fmaf(a, b.w, c.w));
}

// bulk copy of n bytes (a multiple of 16; both addresses 16-byte aligned) into this CTA's
// shared memory, completing on bar
__device__ __forceinline__ void chain_g2s(void* dst, const void* src, uint32_t n, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(tc::smem_u32(dst)), "l"(src), "r"(n), "r"(tc::smem_u32(bar))
               : "memory");
}

// forward: persistent blocks of 256 threads (weights staged once) over 64-row tiles of x,
// which arrive by bulk copy one tile ahead.  kc: thread = 2 rows x 4 columns (of 32, 25
// kept), each sum split over even and odd groups of 4 k (four independent chains); y0:
// thread = 2 rows x 8 columns.
constexpr int CH_FWD_THREADS = 256;
__global__ void __launch_bounds__(CH_FWD_THREADS) k_chain_fwd(long long E, const float* __restrict__ x,
                                                             const float* __restrict__ Weff,
                                                             const float* __restrict__ U0, float* __restrict__ kc,
                                                             float* __restrict__ y0) {
  extern __shared__ __align__(128) unsigned char chain_smem[];
  ChainFwdSmem& S = *reinterpret_cast<ChainFwdSmem*>(chain_smem);
  const int t = threadIdx.x;
  const long long ntiles = (E + CH_ROWS - 1) / CH_ROWS;
  const long long nmine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (nmine == 0) return;
  if (t == 0) {
    for (int b = 0; b < CH_BUF; ++b) tc::mbar_init(&S.full[b], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int idx = t; idx < 128 * 32; idx += CH_FWD_THREADS) {
    const int k = idx >> 5, j = idx & 31;
    S.sw[k][j] = j < 25 ? Weff[k * 25 + j] : 0.f;
  }
  for (int idx = t; idx < 32 * 64; idx += CH_FWD_THREADS) S.su[idx >> 6][idx & 63] = U0[idx];
  __syncthreads();
  auto issue = [&](long long i) {
    const int b = (int)(i % CH_BUF);
    const long long r0 = (blockIdx.x + i * gridDim.x) * CH_ROWS;
    const int nr = (int)min((long long)CH_ROWS, E - r0);
    tc::mbar_expect_tx(&S.full[b], (uint32_t)nr * 512);
    for (int r = 0; r < nr; ++r) chain_g2s(&S.sx[b][r][0], x + (size_t)(r0 + r) * 128, 512, &S.full[b]);
  };
  if (t == 0)
    for (long long i = 0; i < min((long long)CH_BUF, nmine); ++i) issue(i);
  const int rg = t >> 3, cg = t & 7;   // rows 2 rg, 2 rg + 1
  const int ra = 2 * rg, rb = ra + 1;
  for (long long i = 0; i < nmine; ++i) {
    const int b = (int)(i % CH_BUF);
    const long long r0 = (blockIdx.x + i * gridDim.x) * CH_ROWS;
    const long long nr = min((long long)CH_ROWS, E - r0);
    tc::mbar_wait(&S.full[b], (uint32_t)((i / CH_BUF) & 1));   // bounded; a timeout sets the device error
    const float* xa_row = &S.sx[b][ra][0];
    const float* xb_row = &S.sx[b][rb][0];
    {
      float4 a0[2], a1[2];
      a0[0] = a0[1] = a1[0] = a1[1] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int k = 0; k < 128; k += 4) {
        const int h = (k >> 2) & 1;
        const float4 xa = *reinterpret_cast<const float4*>(xa_row + k);
        const float4 xb = *reinterpret_cast<const float4*>(xb_row + k);
        const float xav[4] = {xa.x, xa.y, xa.z, xa.w}, xbv[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 w = *reinterpret_cast<const float4*>(&S.sw[k + q][4 * cg]);
          a0[h] = f4fma(xav[q], w, a0[h]);
          a1[h] = f4fma(xbv[q], w, a1[h]);
        }
      }
      const float o0[4] = {a0[0].x + a0[1].x, a0[0].y + a0[1].y, a0[0].z + a0[1].z, a0[0].w + a0[1].w};
      const float o1[4] = {a1[0].x + a1[1].x, a1[0].y + a1[1].y, a1[0].z + a1[1].z, a1[0].w + a1[1].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = 4 * cg + j;
        if (col < 25) {
          if (ra < nr) kc[(size_t)(r0 + ra) * 25 + col] = o0[j];
          if (rb < nr) kc[(size_t)(r0 + rb) * 25 + col] = o1[j];
        }
      }
    }
    {
      // y0 columns 4 cg .. +3 and 32 + 4 cg .. +3
      float4 a00 = make_float4(0.f, 0.f, 0.f, 0.f), a01 = a00, a10 = a00, a11 = a00;
#pragma unroll 4
      for (int k = 0; k < 32; k += 4) {
        const float4 xa = *reinterpret_cast<const float4*>(xa_row + k);
        const float4 xb = *reinterpret_cast<const float4*>(xb_row + k);
        const float xav[4] = {xa.x, xa.y, xa.z, xa.w}, xbv[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 u0 = *reinterpret_cast<const float4*>(&S.su[k + q][4 * cg]);
          const float4 u1 = *reinterpret_cast<const float4*>(&S.su[k + q][32 + 4 * cg]);
          a00 = f4fma(xav[q], u0, a00);
          a01 = f4fma(xav[q], u1, a01);
          a10 = f4fma(xbv[q], u0, a10);
          a11 = f4fma(xbv[q], u1, a11);
        }
      }
      float4* y4 = reinterpret_cast<float4*>(y0);
      if (ra < nr) {
        y4[(size_t)(r0 + ra) * 16 + cg] = a00;
        y4[(size_t)(r0 + ra) * 16 + 8 + cg] = a01;
      }
      if (rb < nr) {
        y4[(size_t)(r0 + rb) * 16 + cg] = a10;
        y4[(size_t)(r0 + rb) * 16 + 8 + cg] = a11;
      }
    }
    __syncthreads();                   // tile b read by every thread: free for the next copy
    if (t == 0 && i + CH_BUF < nmine) issue(i + CH_BUF);
  }
}

// input gradient g_x [E][128], persistent blocks over 64-row tiles of g_kc and g_y0 (bulk
// copies one tile ahead): thread = 2 rows x 16 columns (4 cg + 32 j .. +3, j = 0..3), so that
// every thread holds 4 columns of the degree-0 block (columns < 32, which also get g_y0 U_0^T)
__global__ void __launch_bounds__(256) k_chain_bwd(long long E, const float* __restrict__ g_kc,
                                                  const float* __restrict__ g_y0, const float* __restrict__ Weff,
                                                  const float* __restrict__ U0, float* __restrict__ g_x) {
  extern __shared__ __align__(128) unsigned char chain_smem[];
  ChainBwdSmem& S = *reinterpret_cast<ChainBwdSmem*>(chain_smem);
  const int t = threadIdx.x;
  const long long ntiles = (E + CH_ROWS - 1) / CH_ROWS;
  const long long nmine = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (nmine == 0) return;
  if (t == 0) {
    for (int b = 0; b < CH_BUF; ++b) tc::mbar_init(&S.full[b], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int idx = t; idx < 128 * 25; idx += 256) S.sw[idx % 25][idx / 25] = Weff[idx];
  for (int idx = t; idx < 32 * 64; idx += 256) S.su[idx & 63][idx >> 6] = U0[idx];
  __syncthreads();
  // g_kc rows are 100 bytes: a tile of 64 rows starts 16-byte aligned (64 x 100 = 6400 bytes);
  // a short last tile copies its rows rounded up to 16 bytes within the tile's own extent
  // only when that stays inside the array, else it is read with plain loads.
  auto issue = [&](long long i) {
    const int b = (int)(i % CH_BUF);
    const long long r0 = (blockIdx.x + i * gridDim.x) * CH_ROWS;
    const long long nr = min((long long)CH_ROWS, E - r0);
    const uint32_t bh = (uint32_t)(nr * 256);
    const uint32_t bg = (uint32_t)(nr * 100) & ~15u;      // whole 16-byte units of the g_kc rows
    tc::mbar_expect_tx(&S.full[b], bh + bg);
    if (bg) chain_g2s(&S.sg[b][0], g_kc + (size_t)r0 * 25, bg, &S.full[b]);
    for (int r = 0; r < (int)nr; ++r) chain_g2s(&S.sh[b][r][0], g_y0 + (size_t)(r0 + r) * 64, 256, &S.full[b]);
  };
  if (t == 0)
    for (long long i = 0; i < min((long long)CH_BUF, nmine); ++i) issue(i);
  const int rg = t >> 3, cg = t & 7;
  const int ra = 2 * rg, rb = ra + 1;
  for (long long i = 0; i < nmine; ++i) {
    const int b = (int)(i % CH_BUF);
    const long long r0 = (blockIdx.x + i * gridDim.x) * CH_ROWS;
    const long long nr = min((long long)CH_ROWS, E - r0);
    tc::mbar_wait(&S.full[b], (uint32_t)((i / CH_BUF) & 1));   // bounded; a timeout sets the device error
    // the g_kc floats past the copied 16-byte units (at most 3, only in a short last tile)
    const int ncopied = (int)(((nr * 100) & ~15ll) / 4);
    for (int q = ncopied + t; q < nr * 25; q += 256) S.sg[b][q] = g_kc[(size_t)r0 * 25 + q];
    __syncthreads();
    const float* ga_row = &S.sg[b][ra * 25];
    const float* gb_row = &S.sg[b][rb * 25];
    float4 a[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int j = 0; j < 4; ++j) a[r][j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 5
    for (int q = 0; q < 25; ++q) {
      const float ga = ga_row[q], gb = gb_row[q];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 w = *reinterpret_cast<const float4*>(&S.sw[q][32 * j + 4 * cg]);
        a[0][j] = f4fma(ga, w, a[0][j]);
        a[1][j] = f4fma(gb, w, a[1][j]);
      }
    }
    // degree-0 block: columns 4 cg .. +3 (j = 0)
    const float* ha_row = &S.sh[b][ra][0];
    const float* hb_row = &S.sh[b][rb][0];
#pragma unroll 8
    for (int h = 0; h < 64; ++h) {
      const float4 u = *reinterpret_cast<const float4*>(&S.su[h][4 * cg]);
      a[0][0] = f4fma(ha_row[h], u, a[0][0]);
      a[1][0] = f4fma(hb_row[h], u, a[1][0]);
    }
    float4* gx4 = reinterpret_cast<float4*>(g_x);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (ra < nr) gx4[(size_t)(r0 + ra) * 32 + 8 * j + cg] = a[0][j];
      if (rb < nr) gx4[(size_t)(r0 + rb) * 32 + 8 * j + cg] = a[1][j];
    }
    __syncthreads();                   // tile b read by every thread: free for the next copy
    if (t == 0 && i + CH_BUF < nmine) issue(i + CH_BUF);
  }
}

}  // namespace emp
