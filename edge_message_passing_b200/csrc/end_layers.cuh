// The first and the last interaction layer of the energy + force step, where the
// SO(2) convolution touches degree 0 on one side only.
//
// First layer: its input is the species embedding, degree 0 only (the initial
// features of the seeded workloads), so the rotated input has the single column
// x~[l=0, m=0] = R[0] (.) x_send[0] and only the m = 0 mixing block sees it.
// The message of edge e is then m_e[l, m'] = D^l_e[0, m'] (W0 x~_e)[l], which is
// linear in x~_e, so the receiver sum can be taken before the mixing:
//   Z_i[l, m', c] = sum_{e: recv(e) = i} D^l_e[0, m'] R_e[0, c] x_send(e)[0, c]
//   S_i[l, m', c'] = sum_c W0[(l, c'), (0, c)] Z_i[l, m', c]
// (one product per node instead of one per edge).  The backward needs, per edge,
// only the degree-0 radial scale gradient and the edge torque; both follow from
// the per-node H_i[l, m', c] = sum_c' W0[(l, c'), (0, c)] gS_i[l, m', c'].
//
// Last layer: the energy reads the last features through their degree-0
// channels only (the readout acts on x[l=0], and the gate's degree-0 output
// SiLU(a0) depends on a0 alone), so only the degree-0 part of the last layer's
// receiver sums is needed: S_i[0, c'] = sum_e (W0 x~_e)[0, c'] with
// x~_e[l, 0, c] = R_e[l, c] sum_m' D^l_e[0, m'] x_send(e)[l, m', c] (only the
// m = 0 block can reach degree 0).  Again the sum over edges comes first:
//   X_i[l, c] = sum_{e: recv(e) = i} x~_e[l, 0, c],  S_i[0, c'] = sum W0[(0, c'), (l, c)] X_i[l, c].
// Its output gradient is degree 0 only, so dE/dx~_e = G_recv(e) with the per-node
// G_i[l, c] = sum_c' W0[(0, c'), (l, c)] gS_i[0, c'] (m = 0 entries; the others vanish),
// and the y^T J g_y part of the torque vanishes (g_y lives in degree 0, where the
// generators are zero).
//
// These are exact rearrangements of the same sums (the model of the page
// "first-order SO(2) input-gradient path": radial scales, Wigner-D rotation,
// per-m mixing, rotation back, normalised receiver sum); they change only the
// order of floating-point additions.  All sums have a fixed order: receiver i's
// edges ascending, one block per receiver.
#pragma once
#include "emp_common.cuh"
#include "model.cuh"

namespace emp {

// index, inside the 84 Wigner-D floats of an edge, of D^l[m][n]
__host__ __device__ constexpr int dix(int l, int m, int n) { return dblk_off(l) + (m + l) * (2 * l + 1) + (n + l); }

// the structural generator pair (a < b) of degree l joining m = a_m and m = b_m
__host__ __device__ constexpr int jpair_of(int l, int am, int bm, int p = 0) {
  return p >= NJPAIR ? -1
       : (jpair_a(p) == lm_index(l, am) && jpair_b(p) == lm_index(l, bm)) ? p
       : jpair_of(l, am, bm, p + 1);
}

constexpr int EL_CH = 16;   // edges staged per chunk

// ------------------------------------------------------------------ first layer, forward
// Z[i][k][c] for the receiver i = blockIdx.x; one thread per channel (blockDim.x = C).  R holds the
// first layer's degree-0 scales only: rows of C floats.
__global__ void __launch_bounds__(256) k_first_fwd(int C, const int* __restrict__ recv_off,
                                                   const int* __restrict__ send, const int* __restrict__ rrow,
                                                   const float* __restrict__ D, const float* __restrict__ R,
                                                   const float* __restrict__ x, float* __restrict__ Z) {
  __shared__ float sd[EL_CH][16];      // the m = 0 row of each degree block, per edge
  __shared__ int ss[EL_CH], sr[EL_CH];
  const int i = blockIdx.x, c = threadIdx.x;
  const int e0 = recv_off[i], e1 = recv_off[i + 1];
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  for (int eb = e0; eb < e1; eb += EL_CH) {
    const int n = min(EL_CH, e1 - eb);
    __syncthreads();
    for (int q = c; q < n * 16; q += blockDim.x) {
      const int k = q & 15, l = k == 0 ? 0 : k < 4 ? 1 : k < 9 ? 2 : 3;
      sd[q >> 4][k] = D[(size_t)(eb + (q >> 4)) * NDBLK + dix(l, 0, k - l * l - l)];
    }
    for (int q = c; q < n; q += blockDim.x) {
      ss[q] = send[eb + q];
      sr[q] = rrow ? rrow[eb + q] : eb + q;
    }
    __syncthreads();
#pragma unroll 4
    for (int q = 0; q < n; ++q) {
      const float v = R[(size_t)sr[q] * C + c] * x[(size_t)ss[q] * 16 * C + c];
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k] = fmaf(sd[q][k], v, acc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) Z[((size_t)i * 16 + k) * C + c] = acc[k];
}

// ------------------------------------------------------------------ last layer, forward
// X[i][l][c] for the receiver i = blockIdx.x; one thread per channel.
__global__ void __launch_bounds__(256) k_last_fwd(int C, const int* __restrict__ recv_off,
                                                  const int* __restrict__ send, const int* __restrict__ rrow,
                                                  const float* __restrict__ D, const float* __restrict__ R,
                                                  const float* __restrict__ x, float* __restrict__ X) {
  __shared__ float sd[EL_CH][16];
  __shared__ int ss[EL_CH], sr[EL_CH];
  const int i = blockIdx.x, c = threadIdx.x;
  const int e0 = recv_off[i], e1 = recv_off[i + 1];
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int eb = e0; eb < e1; eb += EL_CH) {
    const int n = min(EL_CH, e1 - eb);
    __syncthreads();
    for (int q = c; q < n * 16; q += blockDim.x) {
      const int k = q & 15, l = k == 0 ? 0 : k < 4 ? 1 : k < 9 ? 2 : 3;
      sd[q >> 4][k] = D[(size_t)(eb + (q >> 4)) * NDBLK + dix(l, 0, k - l * l - l)];
    }
    for (int q = c; q < n; q += blockDim.x) {
      ss[q] = send[eb + q];
      sr[q] = rrow ? rrow[eb + q] : eb + q;
    }
    __syncthreads();
#pragma unroll 2
    for (int q = 0; q < n; ++q) {
      const float* xs = x + (size_t)ss[q] * 16 * C + c;
      const float* Rr = R + (size_t)sr[q] * 4 * C + c;
      float xv[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) xv[k] = xs[k * C];
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        float u = 0.f;
#pragma unroll
        for (int k = l * l; k < (l + 1) * (l + 1); ++k) u = fmaf(sd[q][k], xv[k], u);
        acc[l] = fmaf(Rr[l * C], u, acc[l]);
      }
    }
  }
#pragma unroll
  for (int l = 0; l < 4; ++l) X[((size_t)i * 4 + l) * C + c] = acc[l];
}

// ------------------------------------------------------------------ torque of a staged chunk
// red[q][w][j]: warp w's channel sums of the edge-frame torque components; the sums over the
// warps (in order), the frame and the cross product with r, added to g_r (one thread per edge).
__device__ __forceinline__ void finish_torque(int n, int nw, int eb, const float* red, const float* svec,
                                              float* __restrict__ g_r) {
  const int q = threadIdx.x;
  if (q >= n) return;
  float sx = 0.f, sy = 0.f;
  for (int w = 0; w < nw; ++w) {
    sx += red[(q * nw + w) * 2 + 0];
    sy += red[(q * nw + w) * 2 + 1];
  }
  const float vx = svec[3 * q], vy = svec[3 * q + 1], vz = svec[3 * q + 2];
  const float d2 = vx * vx + vy * vy + vz * vz;
  const float inv = rsqrtf(d2);
  float Rf[3][3];
  edge_frame<float>(vx * inv, vy * inv, vz * inv, Rf);
  const float ax = -(Rf[0][0] * sx + Rf[1][0] * sy);
  const float ay = -(Rf[0][1] * sx + Rf[1][1] * sy);
  const float az = -(Rf[0][2] * sx + Rf[1][2] * sy);
  const float id2 = 1.f / d2;
  const size_t e = (size_t)(eb + q);
  g_r[3 * e + 0] += (ay * vz - az * vy) * id2;
  g_r[3 * e + 1] += (az * vx - ax * vz) * id2;
  g_r[3 * e + 2] += (ax * vy - ay * vx) * id2;
}

// stage the chunk's Wigner-D rows (84 floats per edge), edge vectors, senders and radial rows
__device__ __forceinline__ void stage_chunk(int eb, int n, const float* __restrict__ D, const float* __restrict__ vec,
                                            const int* __restrict__ send, const int* __restrict__ rrow, float* sD,
                                            float* svec, int* ss, int* sr) {
  const int t = threadIdx.x;
  for (int q = t; q < n * (NDBLK / 4); q += blockDim.x)
    reinterpret_cast<float4*>(sD)[q] = reinterpret_cast<const float4*>(D + (size_t)eb * NDBLK)[q];
  for (int q = t; q < n * 3; q += blockDim.x) svec[q] = vec[(size_t)eb * 3 + q];
  for (int q = t; q < n; q += blockDim.x) {
    ss[q] = send[eb + q];
    sr[q] = rrow ? rrow[eb + q] : eb + q;
  }
}

// ------------------------------------------------------------------ first layer, backward
// Per edge of receiver i = blockIdx.x (one thread per channel; R rows of C floats, the degree-0
// scales; dE/dR rows of 4C floats, of which the first C are written): with H_i (per-node, see the
// top of this file), K[l][m] = sum_m' D^l[m][m'] H_i[l][m'] for m = -1, 0, 1:
//   dE/dx~[0,0] = sum_l K[l][0];  dE/dR[0] = dE/dx~[0,0] x_send[0]  (split hi/lo, row rr)
//   torque: the y^T J g_y term with y = W0 x~ (m = 0 only): per degree l, the channel sums
//   P[l][m] = sum_c x~[0,0,c] K[l][m][c] enter as -P[l][-1] on the pair (-1, 0) and
//   +P[l][+1] on the pair (0, +1).
// With gx (weight gradients: dE/demb needs dE/dx_0), also the layer's gradient with respect to
// the degree-0 input of the senders, gathered at the receiver through the mirror edges as in
// the last layer: gx[i][0] += sum_{e in recv(i)} R_e[0] sum_l (-1)^l sum_m' D^l_e[0][m'] H_send(e)[l][m'].
__global__ void __launch_bounds__(256) k_first_bwd(int C, const int* __restrict__ recv_off,
                                                   const int* __restrict__ send, const int* __restrict__ rrow,
                                                   const float* __restrict__ vec, const float* __restrict__ D,
                                                   const float* __restrict__ R, const float* __restrict__ x,
                                                   const float* __restrict__ H, float* __restrict__ gR_hi,
                                                   float* __restrict__ gR_lo, float* __restrict__ g_r,
                                                   float* __restrict__ gx) {
  __shared__ __align__(16) float sD[EL_CH * NDBLK];
  __shared__ float svec[EL_CH * 3];
  __shared__ int ss[EL_CH], sr[EL_CH];
  __shared__ float red[EL_CH * 8 * 2];
  const int i = blockIdx.x, c = threadIdx.x, warp = c >> 5, lane = c & 31, nw = blockDim.x >> 5;
  const int e0 = recv_off[i], e1 = recv_off[i + 1];
  float h[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) h[k] = H[((size_t)i * 16 + k) * C + c];
  constexpr int P1m = jpair_of(1, -1, 0), P1p = jpair_of(1, 0, 1);
  constexpr int P2m = jpair_of(2, -1, 0), P2p = jpair_of(2, 0, 1);
  constexpr int P3m = jpair_of(3, -1, 0), P3p = jpair_of(3, 0, 1);
  static_assert(P1m >= 0 && P1p >= 0 && P2m >= 0 && P2p >= 0 && P3m >= 0 && P3p >= 0, "generator pairs");
  float gsend = 0.f;
  for (int eb = e0; eb < e1; eb += EL_CH) {
    const int n = min(EL_CH, e1 - eb);
    __syncthreads();
    stage_chunk(eb, n, D, vec, send, rrow, sD, svec, ss, sr);
    __syncthreads();
#pragma unroll 1
    for (int q = 0; q < n; ++q) {
      const float* Dq = sD + q * NDBLK;
      const float x0 = x[(size_t)ss[q] * 16 * C + c];
      const float r0 = R[(size_t)sr[q] * C + c];
      const float xt = r0 * x0;
      if (gx) {
        const float* hs = H + (size_t)ss[q] * 16 * C + c;
        float v = hs[0];
#pragma unroll
        for (int l = 1; l <= 3; ++l) {
          float u = 0.f;
#pragma unroll
          for (int nn = -l; nn <= l; ++nn) u = fmaf(Dq[dix(l, 0, nn)], hs[(l * l + l + nn) * C], u);
          v = (l & 1) ? v - u : v + u;
        }
        gsend = fmaf(r0, v, gsend);
      }
      float g0 = h[0];
      float bx = 0.f, by = 0.f;
#define EMP_FIRST_DEG(L, PM, PP)                                                       \
      {                                                                                \
        float km = 0.f, k0 = 0.f, kp = 0.f;                                            \
        _Pragma("unroll") for (int nn = -L; nn <= L; ++nn) {                           \
          const float hv = h[L * L + L + nn];                                          \
          km = fmaf(Dq[dix(L, -1, nn)], hv, km);                                       \
          k0 = fmaf(Dq[dix(L, 0, nn)], hv, k0);                                        \
          kp = fmaf(Dq[dix(L, 1, nn)], hv, kp);                                        \
        }                                                                              \
        g0 += k0;                                                                      \
        const float pm = xt * km, pp = xt * kp;                                        \
        bx = fmaf(c_jx[PP], pp, fmaf(-c_jx[PM], pm, bx));                              \
        by = fmaf(c_jy[PP], pp, fmaf(-c_jy[PM], pm, by));                              \
      }
      EMP_FIRST_DEG(1, P1m, P1p)
      EMP_FIRST_DEG(2, P2m, P2p)
      EMP_FIRST_DEG(3, P3m, P3p)
#undef EMP_FIRST_DEG
      const float gr = g0 * x0;
      const float ghi = tf32_rna(gr);
      gR_hi[(size_t)sr[q] * 4 * C + c] = ghi;
      gR_lo[(size_t)sr[q] * 4 * C + c] = tf32_rna(gr - ghi);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        bx += __shfl_xor_sync(0xffffffffu, bx, o);
        by += __shfl_xor_sync(0xffffffffu, by, o);
      }
      if (lane == 0) {
        red[(q * nw + warp) * 2 + 0] = bx;
        red[(q * nw + warp) * 2 + 1] = by;
      }
    }
    __syncthreads();
    finish_torque(n, nw, eb, red, svec, g_r);
  }
  if (gx) gx[(size_t)i * 16 * C + c] += gsend;
}

// ------------------------------------------------------------------ last layer, backward
// Per edge e of receiver i = blockIdx.x (one thread per channel), with G_i (per node):
//   u[l][m] = sum_m' D^l[m][m'] x_send[l][m'] (m = -1, 0, 1);  gu[l] = R[l] G_i[l]
//   dE/dR[l] = G_i[l] u[l][0]  (split hi/lo, row rr)
//   torque: the gu^T J u term with gu at m = 0 only: -gu u[l][-1] on the pair (-1, 0),
//   +gu u[l][+1] on the pair (0, +1)
// and the sender sums dE/dx_send of the layer, gathered at the receiver: for the edges e'
// whose sender is i (the mirrors (j, i, -S) of i's own edges (i, j, S)),
//   dE/dx[i][l][m'] += sum_{e in recv(i)} (-1)^l D^l_e[0][m'] R_e[l] G_send(e)[l]
// because the m = 0 row of D^l is a multiple of the real spherical harmonics of the edge
// direction (Y_l(-r) = (-1)^l Y_l(r)) and the radial scale of an edge and its mirror are equal
// (same length, unordered species pair).  One writer per node: gx[i] += that sum.
__global__ void __launch_bounds__(256) k_last_bwd(int C, const int* __restrict__ recv_off,
                                                  const int* __restrict__ send, const int* __restrict__ rrow,
                                                  const float* __restrict__ vec, const float* __restrict__ D,
                                                  const float* __restrict__ R, const float* __restrict__ x,
                                                  const float* __restrict__ G, float* __restrict__ gR_hi,
                                                  float* __restrict__ gR_lo, float* __restrict__ g_r,
                                                  float* __restrict__ gx) {
  __shared__ __align__(16) float sD[EL_CH * NDBLK];
  __shared__ float svec[EL_CH * 3];
  __shared__ int ss[EL_CH], sr[EL_CH];
  __shared__ float red[EL_CH * 8 * 2];
  const int i = blockIdx.x, c = threadIdx.x, warp = c >> 5, lane = c & 31, nw = blockDim.x >> 5;
  const int e0 = recv_off[i], e1 = recv_off[i + 1];
  float gi[4];
#pragma unroll
  for (int l = 0; l < 4; ++l) gi[l] = G[((size_t)i * 4 + l) * C + c];
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  constexpr int P1m = jpair_of(1, -1, 0), P1p = jpair_of(1, 0, 1);
  constexpr int P2m = jpair_of(2, -1, 0), P2p = jpair_of(2, 0, 1);
  constexpr int P3m = jpair_of(3, -1, 0), P3p = jpair_of(3, 0, 1);
  static_assert(P1m >= 0 && P1p >= 0 && P2m >= 0 && P2p >= 0 && P3m >= 0 && P3p >= 0, "generator pairs");
  for (int eb = e0; eb < e1; eb += EL_CH) {
    const int n = min(EL_CH, e1 - eb);
    __syncthreads();
    stage_chunk(eb, n, D, vec, send, rrow, sD, svec, ss, sr);
    __syncthreads();
#pragma unroll 1
    for (int q = 0; q < n; ++q) {
      const float* Dq = sD + q * NDBLK;
      const float* xs = x + (size_t)ss[q] * 16 * C + c;
      const float* Rr = R + (size_t)sr[q] * 4 * C + c;
      const float* Gs = G + (size_t)ss[q] * 4 * C + c;
      float xv[16], rl[4], gs[4];
#pragma unroll
      for (int k = 0; k < 16; ++k) xv[k] = xs[k * C];
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        rl[l] = Rr[l * C];
        gs[l] = Gs[l * C];
      }
      float gr[4];
      float bx = 0.f, by = 0.f;
      // degree 0: u = x[0], no torque
      gr[0] = gi[0] * xv[0];
      acc[0] = fmaf(rl[0], gs[0], acc[0]);
#define EMP_LAST_DEG(L, PM, PP)                                                        \
      {                                                                                \
        float um = 0.f, u0 = 0.f, up = 0.f;                                            \
        _Pragma("unroll") for (int nn = -L; nn <= L; ++nn) {                           \
          const float xvv = xv[L * L + L + nn];                                        \
          um = fmaf(Dq[dix(L, -1, nn)], xvv, um);                                      \
          u0 = fmaf(Dq[dix(L, 0, nn)], xvv, u0);                                       \
          up = fmaf(Dq[dix(L, 1, nn)], xvv, up);                                       \
        }                                                                              \
        gr[L] = gi[L] * u0;                                                            \
        const float gu = rl[L] * gi[L];                                                \
        bx = fmaf(c_jx[PP], gu * up, fmaf(-c_jx[PM], gu * um, bx));                    \
        by = fmaf(c_jy[PP], gu * up, fmaf(-c_jy[PM], gu * um, by));                    \
        const float ms = (L & 1 ? -1.f : 1.f) * rl[L] * gs[L];                         \
        _Pragma("unroll") for (int nn = -L; nn <= L; ++nn)                             \
          acc[L * L + L + nn] = fmaf(Dq[dix(L, 0, nn)], ms, acc[L * L + L + nn]);      \
      }
      EMP_LAST_DEG(1, P1m, P1p)
      EMP_LAST_DEG(2, P2m, P2p)
      EMP_LAST_DEG(3, P3m, P3p)
#undef EMP_LAST_DEG
      const size_t go = (size_t)sr[q] * 4 * C + c;
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const float hi = tf32_rna(gr[l]);
        gR_hi[go + l * C] = hi;
        gR_lo[go + l * C] = tf32_rna(gr[l] - hi);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        bx += __shfl_xor_sync(0xffffffffu, bx, o);
        by += __shfl_xor_sync(0xffffffffu, by, o);
      }
      if (lane == 0) {
        red[(q * nw + warp) * 2 + 0] = bx;
        red[(q * nw + warp) * 2 + 1] = by;
      }
    }
    __syncthreads();
    finish_torque(n, nw, eb, red, svec, g_r);
  }
  float* g = gx + (size_t)i * 16 * C + c;
#pragma unroll
  for (int k = 0; k < 16; ++k) g[k * C] += acc[k];
}

// ------------------------------------------------------------------ per-node products (FP32)
// Up to four products per launch (blockIdx.z): out[r][n] = sum_k A(r)[k] B[n * ldb + k] for
// k < K, n < Nn, r < rows, where row r is component r % w of node r / w:
// A(r) = A + (r / w) a_node + (r % w) a_comp, and likewise out(r) = out + (r / w) o_node + (r % w) o_comp.
// 64 x 64 output tiles, 256 threads, a 4 x 4 register tile each, K in steps of 32 staged in
// shared memory.  Plain FP32 fused multiply-adds in ascending k.
constexpr int NG_T = 64, NG_K = 32, NG_MAX = 4;
struct NodeGemm {
  int n, K, Nn;
  int rows[NG_MAX], w[NG_MAX];
  const float* A[NG_MAX];
  long long a_node[NG_MAX];
  int a_comp[NG_MAX];
  const float* B[NG_MAX];
  int ldb[NG_MAX];
  float* out[NG_MAX];
  long long o_node[NG_MAX];
  int o_comp[NG_MAX];
};
__global__ void __launch_bounds__(256) k_node_gemm(const __grid_constant__ NodeGemm p) {
  __shared__ __align__(16) float As[NG_K][NG_T + 4];
  __shared__ __align__(16) float Bs[NG_K][NG_T + 4];
  const int z = blockIdx.z;
  const int rows = p.rows[z], w = p.w[z], K = p.K, Nn = p.Nn;
  const int r0 = blockIdx.x * NG_T, n0 = blockIdx.y * NG_T;
  if (r0 >= rows) return;
  const float* __restrict__ A = p.A[z];
  const float* __restrict__ B = p.B[z];
  const int t = threadIdx.x;
  const int tr = (t >> 4) * 4, tn = (t & 15) * 4;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  for (int k0 = 0; k0 < K; k0 += NG_K) {
    __syncthreads();
    for (int q = t; q < NG_T * NG_K; q += 256) {
      const int rr = q / NG_K, kk = q % NG_K;
      const int r = r0 + rr, n = n0 + rr, k = k0 + kk;
      As[kk][rr] = (r < rows && k < K) ? A[(long long)(r / w) * p.a_node[z] + (long long)(r % w) * p.a_comp[z] + k] : 0.f;
      Bs[kk][rr] = (n < Nn && k < K) ? B[(long long)n * p.ldb[z] + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < NG_K; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][tr]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tn]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + tr + i;
    if (r >= rows) continue;
    float* o = p.out[z] + (long long)(r / w) * p.o_node[z] + (long long)(r % w) * p.o_comp[z];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (n0 + tn + j < Nn) o[n0 + tn + j] = acc[i][j];
  }
}

// ------------------------------------------------------------------ readout activation
// Given z[i][t] = (W_ro h_i[0])_t (a per-node product): e_i = sum_t w_o[t] SiLU(z_it) (one warp per
// atom, lanes over t in order, then a fixed xor tree) and, in place, z_it <- w_o[t] SiLU'(z_it) =
// dE/dz (the next per-node product turns it into dE/dh_i[0] = (dE/dz) W_ro).
// With silu_out (weight gradients), also SiLU(z_it) there (dE/dw_o = sum_i SiLU(z_i)).
__global__ void k_readout_act(int N, int H, const float* __restrict__ w_o, float* __restrict__ z,
                              float* __restrict__ e_atom, float* __restrict__ silu_out) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (i >= N) return;
  float* zi = z + (size_t)i * H;
  float e = 0.f;
  for (int t = lane; t < H; t += 32) {
    const float v = zi[t], wt = w_o[t], sv = silu_f(v);
    e = fmaf(wt, sv, e);
    zi[t] = wt * dsilu_f(v);
    if (silu_out) silu_out[(size_t)i * H + t] = sv;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
  if (lane == 0) e_atom[i] = e;
}

// ------------------------------------------------------------------ edge geometry
// D(R_e) (84 floats) and d = |r_e| from the float32 edge vector; GEO_EPB edges per block of as
// many threads, the Wigner-D rows staged in shared memory so that the block stores them as
// contiguous float4 runs.
constexpr int GEO_EPB = 64;
__global__ void __launch_bounds__(GEO_EPB) k_geometry_staged(long long E, const float* __restrict__ vec,
                                                             float* __restrict__ D, float* __restrict__ dist) {
  __shared__ __align__(16) float sD[GEO_EPB * NDBLK];
  const long long e0 = (long long)blockIdx.x * GEO_EPB;
  const long long e = e0 + threadIdx.x;
  if (e < E) {
    const float vx = vec[3 * e], vy = vec[3 * e + 1], vz = vec[3 * e + 2];
    const float d = sqrtf(vx * vx + vy * vy + vz * vz);
    const float inv = 1.0f / d;
    float R[3][3];
    edge_frame<float>(vx * inv, vy * inv, vz * inv, R);
    float Dl[NDBLK];
    wigner_blocks<float>(R, Dl);
#pragma unroll
    for (int k = 0; k < NDBLK; ++k) sD[threadIdx.x * NDBLK + k] = Dl[k];
    dist[e] = d;
  }
  __syncthreads();
  const int n = (int)min((long long)GEO_EPB, E - e0);
  float4* dst = reinterpret_cast<float4*>(D + e0 * NDBLK);
  const float4* src = reinterpret_cast<const float4*>(sD);
  for (int q = threadIdx.x; q < n * (NDBLK / 4); q += GEO_EPB) dst[q] = src[q];
}

// ------------------------------------------------------------------ weight gradients
// Sums over rows of outer products (the reduction of a weight gradient over edges or nodes):
// part[z][a][b] = sum over rows r of split z of A(r)[a] B(r)[b], a < Na, b < Nb, with
// A(r) = A + (r / w) a_node + (r % w) a_comp (and A2 at the same offset added when not null:
// the two halves of a 3xTF32 split give back the value), likewise B(r).  128 x 128 output tiles
// (blockIdx.x over a, blockIdx.y over b; an 8 x 8 register tile per thread), rows in steps of 16
// staged in shared memory, splits of rows_per_split rows over blockIdx.z; k_tn_reduce adds the
// splits in order.  FP32, every sum in a fixed order.
struct TnArgs {
  int rows, w, Na, Nb, rows_per_split;
  const float* A;
  const float* A2;
  long long a_node;
  int a_comp;
  const float* B;
  const float* B2;
  long long b_node;
  int b_comp;
  float* part;
};
constexpr int TN_T = 128, TN_K = 32;       // output tile edge, rows per staged step
constexpr int TN_PER = TN_K * TN_T / 256;  // staged elements of each operand per thread and step
__global__ void __launch_bounds__(256) k_tn(const __grid_constant__ TnArgs p) {
  __shared__ __align__(16) float As[TN_K][TN_T + 4];
  __shared__ __align__(16) float Bs[TN_K][TN_T + 4];
  const int a0 = blockIdx.x * TN_T, b0 = blockIdx.y * TN_T;
  const int r_begin = blockIdx.z * p.rows_per_split, r_end = min(p.rows, r_begin + p.rows_per_split);
  const int t = threadIdx.x;
  // thread (ty, tx) owns a 8 x 8 register tile: rows a0 + 4 ty + {0..3, 64..67}, columns b0 + 4 tx + {0..3, 64..67}
  const int ty = t >> 4, tx = t & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  // thread t stages column t % 128 of rows t / 128 + 2 i of a step; the next step's values are
  // loaded into registers while this step is computed
  const int cc = t & (TN_T - 1), r_lane = t >> 7;
  float pa[TN_PER], pb[TN_PER];
  auto load = [&](int rb) {
#pragma unroll
    for (int i = 0; i < TN_PER; ++i) {
      const int r = rb + r_lane + 2 * i;
      float av = 0.f, bv = 0.f;
      if (r < r_end) {
        const int rn = p.w == 1 ? r : r / p.w, rc = p.w == 1 ? 0 : r % p.w;
        const long long ao = (long long)rn * p.a_node + (long long)rc * p.a_comp;
        const long long bo = (long long)rn * p.b_node + (long long)rc * p.b_comp;
        if (a0 + cc < p.Na) av = p.A[ao + a0 + cc] + (p.A2 ? p.A2[ao + a0 + cc] : 0.f);
        if (b0 + cc < p.Nb) bv = p.B[bo + b0 + cc] + (p.B2 ? p.B2[bo + b0 + cc] : 0.f);
      }
      pa[i] = av;
      pb[i] = bv;
    }
  };
  if (r_begin < r_end) load(r_begin);
  for (int rb = r_begin; rb < r_end; rb += TN_K) {
    __syncthreads();
#pragma unroll
    for (int i = 0; i < TN_PER; ++i) {
      As[r_lane + 2 * i][cc] = pa[i];
      Bs[r_lane + 2 * i][cc] = pb[i];
    }
    __syncthreads();
    if (rb + TN_K < r_end) load(rb + TN_K);
#pragma unroll 8
    for (int kk = 0; kk < TN_K; ++kk) {
      const float4 a_lo = *reinterpret_cast<const float4*>(&As[kk][4 * ty]);
      const float4 a_hi = *reinterpret_cast<const float4*>(&As[kk][64 + 4 * ty]);
      const float4 b_lo = *reinterpret_cast<const float4*>(&Bs[kk][4 * tx]);
      const float4 b_hi = *reinterpret_cast<const float4*>(&Bs[kk][64 + 4 * tx]);
      const float av[8] = {a_lo.x, a_lo.y, a_lo.z, a_lo.w, a_hi.x, a_hi.y, a_hi.z, a_hi.w};
      const float bv[8] = {b_lo.x, b_lo.y, b_lo.z, b_lo.w, b_hi.x, b_hi.y, b_hi.z, b_hi.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  float* out = p.part + (size_t)blockIdx.z * p.Na * p.Nb;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int a = a0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
    if (a >= p.Na) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int b = b0 + (j < 4 ? 4 * tx + j : 64 + 4 * tx + j - 4);
      if (b < p.Nb) out[(size_t)a * p.Nb + b] = acc[i][j];
    }
  }
}

// out[a * ldo + b] = (accumulate ? out : 0) + sum over z in order of part[z][a][b]
__global__ void k_tn_reduce(int splits, int Na, int Nb, const float* __restrict__ part, float* __restrict__ out,
                            int ldo, int accumulate) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= Na * Nb) return;
  const int a = idx / Nb, b = idx % Nb;
  float s = accumulate ? out[(size_t)a * ldo + b] : 0.f;
  for (int z = 0; z < splits; ++z) s += part[(size_t)z * Na * Nb + idx];
  out[(size_t)a * ldo + b] = s;
}

// From the gradient dB of a layer's stacked blocks (72 C^2 floats, [n][k] per block, as the
// forward stacks them) to the weights in the blob's order: W0 [4C][4C], then for m = 1, 2, 3
// Wr_m, Wi_m [(4-m)C][(4-m)C].  With block b = [[Wr, -Wi], [Wi, Wr]] (rows +, -; columns +, -):
// dWr = dB[+][+] + dB[-][-], dWi = dB[-][+] - dB[+][-].
__global__ void k_unstack_so2(int C, const float* __restrict__ dB, float* __restrict__ out) {
  const size_t total = (size_t)(16 + 2 * (9 + 4 + 1)) * C * C;   // W0 and the three (Wr, Wi) pairs
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    if (idx < (size_t)16 * C * C) {
      out[idx] = dB[idx];
      continue;
    }
    size_t o = (size_t)16 * C * C;
    for (int m = 1; m <= 3; ++m) {
      const size_t h = (size_t)(4 - m) * C, hh = h * h;
      if (idx < o + 2 * hh) {
        const size_t q = idx - o;
        const bool imag = q >= hh;
        const size_t i = (q % hh) / h, j = q % h;
        const float* B = dB + (size_t)wblk_off(m) * C * C;
        const size_t K = 2 * h;
        out[idx] = imag ? B[(h + i) * K + j] - B[i * K + h + j] : B[i * K + j] + B[(h + i) * K + h + j];
        break;
      }
      o += 2 * hh;
    }
  }
}

// out[c] = sum_i v[i][c] (i ascending), c < n, rows of ld floats
__global__ void k_colsum(int N, int n, const float* __restrict__ v, int ld, float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n) return;
  float s = 0.f;
  for (int i = 0; i < N; ++i) s += v[(size_t)i * ld + c];
  out[c] = s;
}

// dE/demb[s][c] = sum over atoms i of species s (ascending) of g[i][0][c]
__global__ void k_species_sum(int N, int C, int S, const int* __restrict__ species, const float* __restrict__ g,
                              float* __restrict__ demb) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= S * C) return;
  const int s = idx / C, c = idx % C;
  float acc = 0.f;
  for (int i = 0; i < N; ++i)
    if ((species ? species[i] : 0) == s) acc += g[(size_t)i * 16 * C + c];
  demb[idx] = acc;
}

}  // namespace emp
