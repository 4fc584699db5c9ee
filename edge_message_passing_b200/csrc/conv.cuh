// Per-edge kernels of the SO(2) message-passing layer and its cohort-wise
// backward (page "first-order SO(2) input-gradient path": the reverse mixing
// chain is finished one receiver-sorted 8192-edge cohort at a time; page
// "deepmd-kit PR #6108": radial basis -> radial network; the model's steps are
// the convolution of the spec workloads: Bessel basis with polynomial
// envelope, radial MLP giving per-(l, channel) scales, Wigner-D rotation of the
// sender's irreps into the edge frame, per-m SO(2) mixing, rotation back and a
// normalised sum onto the receiver).
//
// Thread mapping of the edge kernels: blockDim = (C, EPB); thread x owns channel
// c = x and its 16 components; row y owns one edge at a time.  Every edge's 84
// Wigner-D values are staged in shared memory.  All sums over edges have a fixed
// order (edges ascending within a receiver or sender segment, cohorts in order),
// so results are bitwise reproducible.
#pragma once
#include "emp_common.cuh"
#include "model.cuh"

namespace emp {

constexpr float PI_F = 3.14159265358979323846f;

// ------------------------------------------------------------------ rotations

__device__ __forceinline__ int deg_of(int k) { return k == 0 ? 0 : k < 4 ? 1 : k < 9 ? 2 : 3; }

// V adjacent channels per thread: float, float2 or float4 arithmetic, loads and stores
template <int V> struct VecT;
template <> struct VecT<1> { typedef float type; };
template <> struct VecT<2> { typedef float2 type; };
template <> struct VecT<4> { typedef float4 type; };

__device__ __forceinline__ float vfma(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ float2 vfma(float a, float2 b, float2 c) { return make_float2(fmaf(a, b.x, c.x), fmaf(a, b.y, c.y)); }
__device__ __forceinline__ float4 vfma(float a, float4 b, float4 c) {
  return make_float4(fmaf(a, b.x, c.x), fmaf(a, b.y, c.y), fmaf(a, b.z, c.z), fmaf(a, b.w, c.w));
}
__device__ __forceinline__ float vmul(float a, float b) { return a * b; }
__device__ __forceinline__ float2 vmul(float2 a, float2 b) { return make_float2(a.x * b.x, a.y * b.y); }
__device__ __forceinline__ float4 vmul(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
template <typename T> __device__ __forceinline__ T vset(float v);
template <> __device__ __forceinline__ float vset<float>(float v) { return v; }
template <> __device__ __forceinline__ float2 vset<float2>(float v) { return make_float2(v, v); }
template <> __device__ __forceinline__ float4 vset<float4>(float v) { return make_float4(v, v, v, v); }
__device__ __forceinline__ void vsplit(float v, float& h, float& l) {
  h = tf32_rna(v);
  l = tf32_rna(v - h);
}
__device__ __forceinline__ void vsplit(float2 v, float2& h, float2& l) {
  vsplit(v.x, h.x, l.x);
  vsplit(v.y, h.y, l.y);
}
__device__ __forceinline__ void vsplit(float4 v, float4& h, float4& l) {
  vsplit(v.x, h.x, l.x);
  vsplit(v.y, h.y, l.y);
  vsplit(v.z, h.z, l.z);
  vsplit(v.w, h.w, l.w);
}

__device__ __forceinline__ float vsub(float a, float b) { return a - b; }
__device__ __forceinline__ float2 vsub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float vadd(float a, float b) { return a + b; }
__device__ __forceinline__ float2 vadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float vscale(float a, float b) { return a * b; }
__device__ __forceinline__ float2 vscale(float a, float2 b) { return make_float2(a * b.x, a * b.y); }
__device__ __forceinline__ float hsum(float a) { return a; }
__device__ __forceinline__ float hsum(float2 a) { return a.x + a.y; }
__device__ __forceinline__ float vdot(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ float2 vdot(float2 a, float2 b, float2 c) { return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y)); }

// ------------------------------------------------------------------ radial part
// e_n(d) = u(d/rc) sin(n pi d / rc) / d, u(x) = 1 - 28 x^6 + 48 x^7 - 21 x^8 for x < 1,
// and its derivative in d (one basis function: every (row, n) pair is its own work item).
__device__ __forceinline__ void bessel_n(float d, float rc, int n, float& e, float& de) {
  const float x = d / rc;
  const float x2 = x * x, x5 = x2 * x2 * x, x6 = x5 * x;
  float u = 1.f + x6 * (-28.f + x * (48.f - 21.f * x));
  float du = x5 * (-168.f + x * (336.f - 168.f * x)) / rc;
  if (x >= 1.f) { u = 0.f; du = 0.f; }
  const float inv = 1.f / d;
  const float k = PI_F * (float)(n + 1) / rc;
  float s, c;
  sincosf(k * d, &s, &c);
  e = u * s * inv;
  de = du * s * inv + u * (k * c * inv - s * inv * inv);
}

__device__ __forceinline__ int pair_of(int a, int b, int S) {
  const int lo = a < b ? a : b, hi = a < b ? b : a;
  return lo * S - lo * (lo - 1) / 2 + (hi - lo);
}

struct RadialArgs {
  const float* rad;        // model radial weights (per layer, per pair): W1 [64][8], W2 [64][64], W3 [4C][64]
  size_t layer_off;        // float offset of layer t's first pair
  size_t pair_stride;      // floats per pair
  int C, n_species, pair_radial;
  float rc;
};

constexpr int RT = 64;      // rows per radial tile
constexpr int RAD_THREADS = 256;
constexpr int RP = 68;      // padded pitch of the transposed [64][RT] tiles (16-byte rows)

// Shared memory of a radial tile.  Thread t owns the 4 x 4 register tile of rows
// 4 (t >> 4) .. +3 and hidden units 4 (t & 15) .. +3 in every layer, so layer 1's
// outputs, layer 2's outputs and the backward's dE/dh1 of a thread share positions.
struct RadialSmem {
  float e[RT][8];
  float de[RT][8];
  float W1[64 * 8];        // [j][n]
  float W2T[64][RP];       // [i][o] = W2[o][i]
  float W2[64][RP];        // backward: [o][i]
  float h1T[64][RP];       // [i][r]
  float gT[64][RP];        // backward: dE/dz2 as [o][r]
  int pair[RT];
  int edge[RT];
  float dist[RT];
  unsigned mask;
};

// rows r0 .. r0+63 of the (pair-sorted, or edge-ordered when perm is null) row list:
// edge, pair, distance and the basis (with its derivative when want_de)
__device__ void radial_tile_setup(RadialSmem& s, long long r0, long long E, const int* __restrict__ perm,
                                  const float* __restrict__ dist, const int* __restrict__ recv,
                                  const int* __restrict__ send, const int* __restrict__ species, const RadialArgs& a,
                                  bool want_de) {
  const int t = threadIdx.x;
  if (t == 0) s.mask = 0u;
  __syncthreads();
  if (t < RT) {
    const long long r = r0 + t;
    int p = 0, e = -1;
    float d = 1.f;
    if (r < E) {
      e = perm ? perm[r] : (int)r;
      d = dist[e];
      if (a.pair_radial) p = pair_of(species[recv[e]], species[send[e]], a.n_species);
      atomicOr(&s.mask, 1u << p);
    }
    s.pair[t] = r < E ? p : -1;
    s.edge[t] = e;
    s.dist[t] = d;
  }
  __syncthreads();
  for (int idx = t; idx < RT * 8; idx += RAD_THREADS) {
    const int r = idx >> 3, n = idx & 7;
    float ev, dv;
    bessel_n(s.dist[r], a.rc, n, ev, dv);
    s.e[r][n] = ev;
    if (want_de) s.de[r][n] = dv;
  }
}

// pair p's weights into shared memory (W2 also untransposed for the backward)
__device__ void radial_stage_weights(RadialSmem& s, const float* __restrict__ W1, const float* __restrict__ W2,
                                     bool want_w2) {
  const int t = threadIdx.x;
  for (int idx = t; idx < 64 * 8; idx += RAD_THREADS) s.W1[idx] = __ldg(&W1[idx]);
  for (int idx = t; idx < 64 * 64; idx += RAD_THREADS) {
    const int o = idx >> 6, i = idx & 63;
    const float w = __ldg(&W2[idx]);
    s.W2T[i][o] = w;
    if (want_w2) s.W2[o][i] = w;
  }
}

// layer 1 of the thread's tile: z1[r][j] = sum_n W1[j][n] e[r][n]; h1 = SiLU(z1) stored as h1T
__device__ __forceinline__ void radial_layer1(RadialSmem& s, int r0, int j0, float (&z1)[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float acc = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) acc = fmaf(s.W1[(j0 + b) * 8 + n], s.e[r0 + a][n], acc);
      z1[a][b] = acc;
    }
#pragma unroll
  for (int b = 0; b < 4; ++b)
    *reinterpret_cast<float4*>(&s.h1T[j0 + b][r0]) =
        make_float4(silu_fast(z1[0][b]), silu_fast(z1[1][b]), silu_fast(z1[2][b]), silu_fast(z1[3][b]));
}

// layer 2 of the thread's tile: z2[r][o] = sum_i W2[o][i] h1[r][i]
__device__ __forceinline__ void radial_layer2(const RadialSmem& s, int r0, int j0, float (&z2)[4][4]) {
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) z2[a][b] = 0.f;
#pragma unroll 8
  for (int i = 0; i < 64; ++i) {
    const float4 h = *reinterpret_cast<const float4*>(&s.h1T[i][r0]);
    const float4 w = *reinterpret_cast<const float4*>(&s.W2T[i][j0]);
    const float hv[4] = {h.x, h.y, h.z, h.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) z2[a][b] = fmaf(hv[a], wv[b], z2[a][b]);
  }
}

// h2 rows (3xTF32 split) of the radial network for every row: the input of the
// tensor-core head R = h2 W3^T
__global__ void __launch_bounds__(RAD_THREADS) k_radial_h2(long long E, const int* __restrict__ perm,
                                                          const float* __restrict__ dist, const int* __restrict__ recv,
                                                          const int* __restrict__ send, const int* __restrict__ species,
                                                          RadialArgs a, float* __restrict__ h2_hi,
                                                          float* __restrict__ h2_lo) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RadialSmem& s = *reinterpret_cast<RadialSmem*>(smem_raw);
  const int t = threadIdx.x;
  const int r0 = (t >> 4) * 4, j0 = (t & 15) * 4;
  int staged = -1;                     // pair whose weights are in shared memory
  for (long long r0g = (long long)blockIdx.x * RT; r0g < E; r0g += (long long)gridDim.x * RT) {
  radial_tile_setup(s, r0g, E, perm, dist, recv, send, species, a, false);
  unsigned mask = s.mask;
  while (mask) {
    const int p = __ffs(mask) - 1;
    mask &= mask - 1;
    if (p != staged) {
      const float* W1 = a.rad + a.layer_off + (size_t)p * a.pair_stride;
      radial_stage_weights(s, W1, W1 + 64 * 8, false);
      staged = p;
    }
    __syncthreads();
    float z[4][4];
    radial_layer1(s, r0, j0, z);
    __syncthreads();
    radial_layer2(s, r0, j0, z);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const long long r = r0g + r0 + q;
      if (s.pair[r0 + q] != p) continue;
      float hi[4], lo[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float v = silu_fast(z[q][b]);
        hi[b] = tf32_rna(v);
        lo[b] = tf32_rna(v - hi[b]);
      }
      *reinterpret_cast<float4*>(h2_hi + (size_t)r * 64 + j0) = make_float4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<float4*>(h2_lo + (size_t)r * 64 + j0) = make_float4(lo[0], lo[1], lo[2], lo[3]);
    }
    __syncthreads();
  }
  }
}

// dE/dd from dE/dh2 (rows gh2 [E][64], the tensor-core product dE/dR W3); adds (dE/dd) rhat to g_r
// (when g_r is not null).
// With rows_out (weight gradients), also each row's basis e [8], h1 [64], dE/dz1 [64] and
// dE/dz2 [64] into rows_out[row][200], for the sums dE/dW2 = sum dE/dz2 (x) h1 and
// dE/dW1 = sum dE/dz1 (x) e.
constexpr int RAD_ROW_FLOATS = 8 + 3 * 64;
__global__ void __launch_bounds__(RAD_THREADS) k_radial_bwd(long long E, const int* __restrict__ perm,
                                                           const float* __restrict__ dist,
                                                           const float* __restrict__ vec, const int* __restrict__ recv,
                                                           const int* __restrict__ send, const int* __restrict__ species,
                                                           RadialArgs a, const float* __restrict__ gh2,
                                                           float* __restrict__ g_r, float* __restrict__ rows_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RadialSmem& s = *reinterpret_cast<RadialSmem*>(smem_raw);
  const int t = threadIdx.x;
  const int r0 = (t >> 4) * 4, j0 = (t & 15) * 4;
  int staged = -1;                     // pair whose weights are in shared memory
  for (long long r0g = (long long)blockIdx.x * RT; r0g < E; r0g += (long long)gridDim.x * RT) {
  radial_tile_setup(s, r0g, E, perm, dist, recv, send, species, a, true);
  float g[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const long long r = r0g + r0 + q;
    const float4 v = r < E ? *reinterpret_cast<const float4*>(gh2 + (size_t)r * 64 + j0) : make_float4(0.f, 0.f, 0.f, 0.f);
    g[q][0] = v.x; g[q][1] = v.y; g[q][2] = v.z; g[q][3] = v.w;
  }
  unsigned mask = s.mask;
  while (mask) {
    const int p = __ffs(mask) - 1;
    mask &= mask - 1;
    const float* W1 = a.rad + a.layer_off + (size_t)p * a.pair_stride;
    if (p != staged) {
      radial_stage_weights(s, W1, W1 + 64 * 8, true);
      staged = p;
    }
    __syncthreads();
    float z1[4][4], z2[4][4];
    radial_layer1(s, r0, j0, z1);
    __syncthreads();
    radial_layer2(s, r0, j0, z2);
    // dE/dz2 = dE/dh2 SiLU'(z2), stored transposed
#pragma unroll
    for (int b = 0; b < 4; ++b)
      *reinterpret_cast<float4*>(&s.gT[j0 + b][r0]) =
          make_float4(g[0][b] * dsilu_fast(z2[0][b]), g[1][b] * dsilu_fast(z2[1][b]), g[2][b] * dsilu_fast(z2[2][b]),
                      g[3][b] * dsilu_fast(z2[3][b]));
    __syncthreads();
    // dE/dh1[r][i] = sum_o dE/dz2[r][o] W2[o][i]; dE/dz1 = dE/dh1 SiLU'(z1)
    float gh[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int b = 0; b < 4; ++b) gh[q][b] = 0.f;
#pragma unroll 8
    for (int o = 0; o < 64; ++o) {
      const float4 gz = *reinterpret_cast<const float4*>(&s.gT[o][r0]);
      const float4 w = *reinterpret_cast<const float4*>(&s.W2[o][j0]);
      const float gv[4] = {gz.x, gz.y, gz.z, gz.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int b = 0; b < 4; ++b) gh[q][b] = fmaf(gv[q], wv[b], gh[q][b]);
    }
    if (rows_out) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const long long r = r0g + r0 + q;
        if (s.pair[r0 + q] != p) continue;
        float* ro = rows_out + (size_t)r * RAD_ROW_FLOATS;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          ro[8 + j0 + b] = s.h1T[j0 + b][r0 + q];
          ro[72 + j0 + b] = gh[q][b] * dsilu_fast(z1[q][b]);
          ro[136 + j0 + b] = s.gT[j0 + b][r0 + q];
        }
        if (j0 == 0)
#pragma unroll
          for (int n = 0; n < 8; ++n) ro[n] = s.e[r0 + q][n];
      }
    }
    // dE/dd[r] = sum_j dE/dz1[r][j] sum_n W1[j][n] de_n[r]: this thread's 4 units, then
    // summed over the 16 threads of the half-warp that share the rows
    float part[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float acc = 0.f;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float w = 0.f;
#pragma unroll
        for (int n = 0; n < 8; ++n) w = fmaf(s.W1[(j0 + b) * 8 + n], s.de[r0 + q][n], w);
        acc = fmaf(gh[q][b] * dsilu_fast(z1[q][b]), w, acc);
      }
      part[q] = acc;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) part[q] += __shfl_xor_sync(0xffffffffu, part[q], off);
    if ((t & 15) == 0 && g_r) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (s.pair[r0 + q] != p) continue;
        const int e = s.edge[r0 + q];
        const float inv = 1.f / s.dist[r0 + q];
        g_r[3 * e + 0] += part[q] * vec[3 * e + 0] * inv;
        g_r[3 * e + 1] += part[q] * vec[3 * e + 1] * inv;
        g_r[3 * e + 2] += part[q] * vec[3 * e + 2] * inv;
      }
    }
    __syncthreads();
  }
  }
}

// Stable, deterministic counting sort of the edges by species pair (one block of
// 1024 threads; thread t owns a contiguous run of edges).  perm[k] = edge at row k,
// inv[e] = row of edge e, off[p] = first row of pair p (off[n_pairs] = E).
constexpr int PS_THREADS = 1024;
__global__ void __launch_bounds__(PS_THREADS) k_pair_sort(long long E, int n_species, int n_pairs,
                                                         const int* __restrict__ recv, const int* __restrict__ send,
                                                         const int* __restrict__ species, int* __restrict__ perm,
                                                         int* __restrict__ inv, int* __restrict__ off) {
  extern __shared__ int cnt[];          // [n_pairs][PS_THREADS]
  __shared__ int wsum[32];
  __shared__ int ptot[33];
  const int t = threadIdx.x;
  const long long per = (E + PS_THREADS - 1) / PS_THREADS;
  const long long b = t * per, en = min(E, b + per);
  for (int p = 0; p < n_pairs; ++p) cnt[p * PS_THREADS + t] = 0;
  for (long long e = b; e < en; ++e) ++cnt[pair_of(species[recv[e]], species[send[e]], n_species) * PS_THREADS + t];
  __syncthreads();
  const int lane = t & 31, w = t >> 5;
  for (int p = 0; p < n_pairs; ++p) {
    const int c = cnt[p * PS_THREADS + t];
    int v = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) wsum[w] = v;
    __syncthreads();
    if (t == 0) {
      int acc = 0;
      for (int q = 0; q < 32; ++q) { const int y = wsum[q]; wsum[q] = acc; acc += y; }
      ptot[p] = acc;
    }
    __syncthreads();
    cnt[p * PS_THREADS + t] = wsum[w] + v - c;     // exclusive prefix within pair p
    __syncthreads();
  }
  if (t == 0) {
    int acc = 0;
    for (int p = 0; p < n_pairs; ++p) { const int y = ptot[p]; ptot[p] = acc; off[p] = acc; acc += y; }
    off[n_pairs] = acc;
  }
  __syncthreads();
  for (long long e = b; e < en; ++e) {
    const int p = pair_of(species[recv[e]], species[send[e]], n_species);
    const int pos = ptot[p] + cnt[p * PS_THREADS + t]++;
    perm[pos] = (int)e;
    inv[e] = pos;
  }
}

// degree-L block of one edge and channel: rotate v (global frame, stride C) by D^L into the
// edge frame; optionally scale by Rl; write fp32 and/or the 3xTF32 split into m-major columns
template <int L>
__device__ __forceinline__ void rotate_write_degree(const float* __restrict__ Dr, const float* __restrict__ v, int C,
                                                    float Rl, float* __restrict__ f32, float* __restrict__ hi,
                                                    float* __restrict__ lo) {
  constexpr int W = 2 * L + 1, O = L * L;
  const float* B = Dr + dblk_off(L);
  float a[W];
#pragma unroll
  for (int n = 0; n < W; ++n) a[n] = v[(O + n) * C];
#pragma unroll
  for (int m = 0; m < W; ++m) {
    float u = 0.f;
#pragma unroll
    for (int n = 0; n < W; ++n) u = fmaf(B[m * W + n], a[n], u);
    u *= Rl;
    const int col = col_of_k(O + m) * C;
    if (f32) f32[col] = u;
    if (hi) {
      const float h = tf32_rna(u);
      hi[col] = h;
      lo[col] = tf32_rna(u - h);
    }
  }
}


// ------------------------------------------------------------------ rotate back + receiver sums
// S[i] (+)= sum over the cohort's edges of receiver i of D_e^T y_e.
// The cohort's rows (receiver-sorted) are cut into chunks of RB_CHUNK consecutive
// edges, one block of C threads (one per channel) per chunk.  A thread sums its
// chunk's messages in edge order, one running sum per receiver run.  A receiver
// whose edges (within the cohort) all lie in the chunk is finished at once: its
// sum is written to S, added to the running sum that S carries when the receiver's
// edges began in an earlier cohort.  A receiver that crosses a chunk boundary
// leaves its chunk sum in a partial slot (slot 0: the chunk's first receiver, slot
// 1: its last), and k_rb_combine adds the partials in chunk order.  The order of
// every sum is fixed, so results are reproducible.
constexpr int RB_CHUNK = 8;

template <typename T>
__device__ __forceinline__ void rb_flush(int i, int c0, int c1, long long e0, long long e1, int chunk, int first_recv,
                                         const int* __restrict__ recv_off, int CV, int t, const T (&acc)[16],
                                         T* __restrict__ S, T* __restrict__ P) {
  const long long lo = max((long long)recv_off[i], e0) - e0, hi = min((long long)recv_off[i + 1], e1) - e0;
  if (lo >= c0 && hi <= c1) {
    T* Si = S + (size_t)i * 16 * CV + t;
    const bool carry = recv_off[i] < e0;
#pragma unroll
    for (int k = 0; k < 16; ++k) Si[k * CV] = carry ? vadd(Si[k * CV], acc[k]) : acc[k];
  } else {
    T* Pc = P + ((size_t)chunk * 2 + (i == first_recv ? 0 : 1)) * 16 * CV + t;
#pragma unroll
    for (int k = 0; k < 16; ++k) Pc[k * CV] = acc[k];
  }
}

// u = D^T x per degree block for V channels (D in shared memory)
template <typename T>
__device__ __forceinline__ void rotate16t_v(const float* __restrict__ D, const T (&x)[16], T (&u)[16]) {
  u[0] = x[0];
#pragma unroll
  for (int l = 1; l <= 3; ++l) {
    const int w = 2 * l + 1, o = l * l;
    const float* B = D + dblk_off(l);
#pragma unroll
    for (int m = 0; m < w; ++m) {
      T acc = vset<T>(0.f);
#pragma unroll
      for (int n = 0; n < w; ++n) acc = vfma(B[n * w + m], x[o + n], acc);
      u[o + m] = acc;
    }
  }
}

// One block of C / RB_V threads (RB_V adjacent channels each) per 8-edge chunk; y rows of 16C.
constexpr int RB_V = 2;
template <int V>
__global__ void __launch_bounds__(128) k_rb_chunks(long long e0, long long e1, int C,
                                                 const int* __restrict__ recv, const int* __restrict__ recv_off,
                                                 const float* __restrict__ D, const float* __restrict__ Y,
                                                 float* __restrict__ S, float* __restrict__ P) {
  typedef typename VecT<V>::type T;
  __shared__ __align__(16) float sD[RB_CHUNK * NDBLK];
  __shared__ int srv[RB_CHUNK];
  const int t = threadIdx.x, CV = C / V;
  const int n = (int)(e1 - e0);
  const T* Yv = reinterpret_cast<const T*>(Y);
  T* Sv = reinterpret_cast<T*>(S);
  T* Pv = reinterpret_cast<T*>(P);
  const int nchunks = (n + RB_CHUNK - 1) / RB_CHUNK;
  for (int chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int c0 = chunk * RB_CHUNK, nch = min(RB_CHUNK, n - c0), c1 = c0 + nch;
    __syncthreads();
    for (int q = t; q < nch * (NDBLK / 4); q += CV)
      reinterpret_cast<float4*>(sD)[q] = reinterpret_cast<const float4*>(D + (size_t)(e0 + c0) * NDBLK)[q];
    if (t < nch) srv[t] = recv[e0 + c0 + t];
    __syncthreads();
    const int first = srv[0];
    int cur = first;
    T acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = vset<T>(0.f);
#pragma unroll 1
    for (int k = 0; k < nch; ++k) {
      const T* y = Yv + (size_t)(c0 + k) * 16 * CV + t;
      T yv[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) yv[q] = y[col_of_k(q) * CV];
      if (srv[k] != cur) {
        rb_flush(cur, c0, c1, e0, e1, chunk, first, recv_off, CV, t, acc, Sv, Pv);
#pragma unroll
        for (int q = 0; q < 16; ++q) acc[q] = vset<T>(0.f);
        cur = srv[k];
      }
      const float* Dk = sD + k * NDBLK;
      T m[16];
      rotate16t_v(Dk, yv, m);
#pragma unroll
      for (int q = 0; q < 16; ++q) acc[q] = vadd(acc[q], m[q]);
    }
    rb_flush(cur, c0, c1, e0, e1, chunk, first, recv_off, CV, t, acc, Sv, Pv);
  }
}

// receivers of the cohort that cross a chunk boundary: S[i] = carried sum + chunk partials in
// order.  Block (x, k): receivers first + x, first + x + gridDim.x, ..., component k.  A
// chunk's partial of receiver i is in slot 0 when i is the chunk's first receiver, which
// holds for every chunk after the first one the receiver touches, and for that first one
// when the receiver's edges start at the chunk's start.
__global__ void k_rb_combine(long long e0, long long e1, int C, const int* __restrict__ recv,
                             const int* __restrict__ recv_off, const float* __restrict__ P, float* __restrict__ S) {
  constexpr int B = 16;
  const int c = threadIdx.x, k = blockIdx.y;
  const int first = recv[e0], last = recv[e1 - 1];
  for (int i = first + blockIdx.x; i <= last; i += gridDim.x) {
    const long long lo = max((long long)recv_off[i], e0) - e0, hi = min((long long)recv_off[i + 1], e1) - e0;
    if (hi <= lo) continue;
    const int cf = (int)(lo / RB_CHUNK), cl = (int)((hi - 1) / RB_CHUNK);
    if (cf == cl) continue;
    float* Si = S + ((size_t)i * 16 + k) * C + c;
    float acc = recv_off[i] < e0 ? *Si : 0.f;
    for (int ch0 = cf; ch0 <= cl; ch0 += B) {
      float v[B];
#pragma unroll
      for (int u = 0; u < B; ++u) {
        const int ch = ch0 + u;
        const int slot = (ch > cf || lo == (long long)ch * RB_CHUNK) ? 0 : 1;
        v[u] = ch <= cl ? P[(((size_t)ch * 2 + slot) * 16 + k) * C + c] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < B; ++u)
        if (ch0 + u <= cl) acc += v[u];
    }
    *Si = acc;
  }
}

// ------------------------------------------------------------------ node update, readout
// a = S / avg; gated: x_next = x + G(a) with G(a)[0] = SiLU(a0), G(a)[l>0] = a SiLU(a0); else x_next = a
__global__ void k_update(int N, int C, float inv_avg, int gated, float* __restrict__ S_to_a,
                         const float* __restrict__ x, float* __restrict__ x_next) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * C) return;
  const int i = idx / C, c = idx % C;
  float a[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    a[k] = S_to_a[((size_t)i * 16 + k) * C + c] * inv_avg;
    S_to_a[((size_t)i * 16 + k) * C + c] = a[k];
  }
  if (gated) {
    const float s = silu_f(a[0]);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float gk = k == 0 ? s : a[k] * s;
      x_next[((size_t)i * 16 + k) * C + c] = x[((size_t)i * 16 + k) * C + c] + gk;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x_next[((size_t)i * 16 + k) * C + c] = a[k];
  }
}

// energy = sum_i e_i in double, fixed order (one block)
__global__ void k_energy_sum(int N, const float* __restrict__ e_atom, double* __restrict__ energy) {
  __shared__ double part[1024];
  const int t = threadIdx.x;
  double s = 0.0;
  for (int i = t; i < N; i += blockDim.x) s += (double)e_atom[i];
  part[t] = s;
  __syncthreads();
  for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
    if (t < w) part[t] += part[t + w];
    __syncthreads();
  }
  if (t == 0) energy[0] = part[0];
}

// ------------------------------------------------------------------ backward
// gS = dE/dS (S = raw receiver sums) from g = dE/dx_next; gx = residual part of dE/dx
__global__ void k_gate_bwd(int N, int C, float inv_avg, int gated, const float* __restrict__ a,
                           const float* __restrict__ g, float* __restrict__ gS, float* __restrict__ gx) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * C) return;
  const int i = idx / C, c = idx % C;
  float gv[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) gv[k] = g[((size_t)i * 16 + k) * C + c];
  if (gated) {
    const float a0 = a[(size_t)i * 16 * C + c];
    const float s = silu_f(a0), ds = dsilu_f(a0);
    float acc = gv[0];
#pragma unroll
    for (int k = 1; k < 16; ++k) acc = fmaf(gv[k], a[((size_t)i * 16 + k) * C + c], acc);
    gS[(size_t)i * 16 * C + c] = acc * ds * inv_avg;
#pragma unroll
    for (int k = 1; k < 16; ++k) gS[((size_t)i * 16 + k) * C + c] = gv[k] * s * inv_avg;
#pragma unroll
    for (int k = 0; k < 16; ++k) gx[((size_t)i * 16 + k) * C + c] = gv[k];
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      gS[((size_t)i * 16 + k) * C + c] = gv[k] * inv_avg;
      gx[((size_t)i * 16 + k) * C + c] = 0.f;
    }
  }
}

// per edge, from y (kept from the forward, or recomputed), g_y and g_x~ = W^T g_y:
//   gR[e][l][c] = sum_m g_x~ u;  g_u = R (.) g_x~;  g_xs = D^T g_u (-> GXS, [16][C] rows)
//   b_j = sum_c (y^T J_j g_y + g_u^T J_j u), j = x, y (edge frame); a = -R_e^T (b_x, b_y, 0);
//   g_r[e] += (a x r) / |r|^2  (direction part of dE/dr; the radial part is added by k_radial_bwd)
// J_x, J_y are antisymmetric and couple components of one degree whose |m| differ by
// one, so v^T J w = sum over the structural pairs (a < b) of J_ab (v_a w_b - v_b w_a).
template <int L, typename T>
__device__ __forceinline__ void torque_pairs_l(const T* v, const T* w, T& bx, T& by) {
  // v, w: the 2L+1 components of degree L (local index m + L)
  constexpr int p0 = L == 1 ? 0 : L == 2 ? 2 : 8;
  constexpr int p1 = L == 1 ? 2 : L == 2 ? 8 : NJPAIR;
#pragma unroll
  for (int p = p0; p < p1; ++p) {
    const int A = jpair_a(p) - L * L, B = jpair_b(p) - L * L;
    const T q = vsub(vmul(v[A], w[B]), vmul(v[B], w[A]));
    bx = vfma(c_jx[p], q, bx);
    by = vfma(c_jy[p], q, by);
  }
}

// degree-L part of the per-edge backward for V = sizeof(T) / 4 adjacent channels; the row
// pointers are offset to the thread's first channel and have a stride of CV vectors
template <int L, typename T>
__device__ __forceinline__ void bwd_edge_degree(const float* __restrict__ Dr, const T* __restrict__ xs,
                                                const T* __restrict__ yrow, const T* __restrict__ gsrow,
                                                const T* __restrict__ gxtrow, T Rl, int CV,
                                                T (&gxs)[16], T& grl, T& bx, T& by) {
  constexpr int W = 2 * L + 1, O = L * L;
  const float* B = Dr + dblk_off(L);
  T v[W], u[W], gu[W];
#pragma unroll
  for (int n = 0; n < W; ++n) v[n] = xs[(O + n) * CV];
#pragma unroll
  for (int m = 0; m < W; ++m) {
    T a = vset<T>(0.f);
#pragma unroll
    for (int n = 0; n < W; ++n) a = vfma(B[m * W + n], v[n], a);
    u[m] = a;
  }
  grl = vset<T>(0.f);
#pragma unroll
  for (int m = 0; m < W; ++m) {
    const T g = gxtrow[col_of_k(O + m) * CV];
    grl = vdot(g, u[m], grl);
    gu[m] = vmul(Rl, g);
  }
  if (L > 0) {
    torque_pairs_l<L>(gu, u, bx, by);
    // g_y = D gS[recv] (edge frame), recomputed from the receiver's row
#pragma unroll
    for (int n = 0; n < W; ++n) v[n] = gsrow[(O + n) * CV];
#pragma unroll
    for (int m = 0; m < W; ++m) {
      T a = vset<T>(0.f);
#pragma unroll
      for (int n = 0; n < W; ++n) a = vfma(B[m * W + n], v[n], a);
      u[m] = a;
    }
#pragma unroll
    for (int m = 0; m < W; ++m) v[m] = yrow[col_of_k(O + m) * CV];
    torque_pairs_l<L>(v, u, bx, by);
  }
#pragma unroll
  for (int m = 0; m < W; ++m) {
    T a = vset<T>(0.f);
#pragma unroll
    for (int n = 0; n < W; ++n) a = vfma(B[n * W + m], gu[n], a);
    gxs[O + m] = vadd(gxs[O + m], a);
  }
}

// Per-edge backward over the cohort, one block of C threads (one per channel) per
// contiguous range of `per` positions.  The positions follow the cohort's sender sort
// (perm), so each sender's edges are consecutive: the block sums g_xs over each sender
// run in registers and stores the sum of each run piece (a run, or the part of one that
// lies in the range) as row Pg[first position of the piece]; k_gx_combine then adds every
// run's pieces to g_x[sender] in order.
// The rows an edge reads (y, g_x~, gS of the receiver, x of the sender, R and its
// Wigner-D blocks, all contiguous) are brought into a BE_STAGES-deep shared-memory ring by bulk copies
// (cp.async.bulk, completing on one mbarrier per stage) issued by thread 0 ahead of
// use, so the loads of later edges overlap the arithmetic of the current one.  The
// per-edge torque sums are kept per position and finished for the whole range at
// the end, by one thread per edge.
constexpr int BE_STAGES = 2;
constexpr int BE_MAXP = 64;           // positions per block at most

struct BeMeta {
  int el, rr, j, i;                   // cohort-local row, radial row, sender, receiver
};

// Whether the sender's node row goes through the ring too (else it is read from global
// memory: the node array stays in L2, and consecutive positions of a sender run share it).
// Staged measured faster, although the smaller ring would allow four blocks per SM.
constexpr bool BE_STAGE_X = true;
// stage layout (floats): Y [16C] | gS[recv] [16C] | GXT [16C] | (X [16C]) | R [4C] | D [84]
__host__ __device__ inline size_t be_stage_floats(int C) { return (size_t)(BE_STAGE_X ? 68 : 52) * C + NDBLK; }
constexpr int BE_MAXP_EDGE = 32;      // positions per block at most (backward edge kernel)
constexpr int BE_BLOCKS_PER_SM = 3;   // resident blocks the ring's shared memory allows
__host__ __device__ inline size_t be_smem_bytes(int C) {
  return BE_STAGES * be_stage_floats(C) * 4 + BE_STAGES * 8 + (size_t)BE_MAXP_EDGE * 2 * ((C + 31) / 32) * 4 +
         BE_MAXP_EDGE * sizeof(BeMeta) + BE_MAXP_EDGE * 4 * 4;
}
// positions per block for a cohort of n edges on `sms` SMs
inline int be_per(long long n, int sms) {
  const long long want = (n + BE_BLOCKS_PER_SM * sms - 1) / (BE_BLOCKS_PER_SM * sms);
  return (int)std::max<long long>(1, std::min<long long>(BE_MAXP_EDGE, want));
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

template <int V>
__global__ void __launch_bounds__(256, 2)
    k_bwd_edge(long long e0, long long e1, int C, int per,
               const int* __restrict__ send, const int* __restrict__ rrow, const float* __restrict__ vec,
               const float* __restrict__ D, const float* __restrict__ R, const float* __restrict__ x,
               const float* __restrict__ Y, const float* __restrict__ gS, const float* __restrict__ GXT,
               const int* __restrict__ recv, const int* __restrict__ perm,
               float* __restrict__ gR_hi,
               float* __restrict__ gR_lo, float* __restrict__ g_r, float* __restrict__ Pg) {
  typedef typename VecT<V>::type T;
  extern __shared__ __align__(128) unsigned char be_smem[];
  const size_t SF = be_stage_floats(C);
  float* stage0 = reinterpret_cast<float*>(be_smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(be_smem + BE_STAGES * SF * 4);
  const int CV = C / V;
  const int nw = (CV + 31) / 32;
  float* red = reinterpret_cast<float*>(full + BE_STAGES);               // [BE_MAXP_EDGE][2][nw]
  BeMeta* meta = reinterpret_cast<BeMeta*>(red + BE_MAXP_EDGE * 2 * nw);
  float* svec = reinterpret_cast<float*>(meta + BE_MAXP_EDGE);           // [BE_MAXP_EDGE][4]
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int n = (int)(e1 - e0);
  const int p0 = blockIdx.x * per, p1 = min(n, p0 + per);
  if (p0 >= p1) return;
  const int np = p1 - p0;
  if (t == 0) {
    for (int s = 0; s < BE_STAGES; ++s) tc::mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int q = t; q < np; q += CV) {
    const int el = perm[e0 + p0 + q];
    const long long e = e0 + el;
    meta[q] = BeMeta{el, rrow ? rrow[e] : (int)e, send[e], recv[e]};
    svec[4 * q + 0] = vec[3 * e];
    svec[4 * q + 1] = vec[3 * e + 1];
    svec[4 * q + 2] = vec[3 * e + 2];
  }
  __syncthreads();
  // bytes of each section that the edge's arithmetic reads
  const uint32_t bY = 64u * C, bG = 64u * C, bX = 64u * C, bR = 16u * C;
  auto issue = [&](int q) {
    const int s = q % BE_STAGES;
    float* st = stage0 + s * SF;
    const BeMeta m = meta[q];
    const int oR = BE_STAGE_X ? 64 * C : 48 * C;
    tc::mbar_expect_tx(&full[s], bY + bG + bX + (BE_STAGE_X ? bX : 0u) + bR + NDBLK * 4);
    bulk_g2s(st, Y + (size_t)m.el * 16 * C, bY, &full[s]);
    bulk_g2s(st + 16 * C, gS + (size_t)m.i * 16 * C, bG, &full[s]);
    bulk_g2s(st + 32 * C, GXT + (size_t)m.el * 16 * C, bX, &full[s]);
    if (BE_STAGE_X) bulk_g2s(st + 48 * C, x + (size_t)m.j * 16 * C, bX, &full[s]);
    bulk_g2s(st + oR, R + (size_t)m.rr * 4 * C, bR, &full[s]);
    bulk_g2s(st + oR + 4 * C, D + (size_t)(e0 + m.el) * NDBLK, NDBLK * 4, &full[s]);
  };
  int nissued = 0;                     // positions whose copies thread 0 has issued
  if (t == 0)
    for (; nissued < min(BE_STAGES, np); ++nissued) issue(nissued);
  T gxs[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) gxs[k] = vset<T>(0.f);
  int qs = 0;                          // first position of the current sender run piece
  T* gHv = reinterpret_cast<T*>(gR_hi);
  T* gLv = reinterpret_cast<T*>(gR_lo);
  T* Pgv = reinterpret_cast<T*>(Pg);
  int qdone = np;                      // positions waited for by every thread
#pragma unroll 1
  for (int q = 0; q < np; ++q) {
    const int s = q % BE_STAGES;
    // bounded; a timeout sets the device error, and the block leaves the loop (all threads at once)
    const bool arrived = tc::mbar_wait(&full[s], (uint32_t)((q / BE_STAGES) & 1));
    const float* st = stage0 + s * SF;
    const BeMeta m = meta[q];
    const T* sY = reinterpret_cast<const T*>(st) + t;
    const T* sGS = reinterpret_cast<const T*>(st + 16 * C) + t;
    const T* sGX = reinterpret_cast<const T*>(st + 32 * C) + t;
    const T* sX = BE_STAGE_X ? reinterpret_cast<const T*>(st + 48 * C) + t
                             : reinterpret_cast<const T*>(x + (size_t)m.j * 16 * C) + t;
    const int oR = BE_STAGE_X ? 64 * C : 48 * C;
    const T* sR = reinterpret_cast<const T*>(st + oR) + t;
    const float* Dr = st + oR + 4 * C;
    const size_t go = (size_t)m.rr * 4 * CV + t;
    T bx = vset<T>(0.f), by = vset<T>(0.f), gr, h, l;
    const T zero = vset<T>(0.f);
    bwd_edge_degree<0>(Dr, sX, sY, sGS, sGX, sR[0], CV, gxs, gr, bx, by);
    vsplit(gr, h, l);
    gHv[go] = h;
    gLv[go] = l;
    bwd_edge_degree<1>(Dr, sX, sY, sGS, sGX, sR[CV], CV, gxs, gr, bx, by);
    vsplit(gr, h, l);
    gHv[go + CV] = h;
    gLv[go + CV] = l;
    bwd_edge_degree<2>(Dr, sX, sY, sGS, sGX, sR[2 * CV], CV, gxs, gr, bx, by);
    vsplit(gr, h, l);
    gHv[go + 2 * CV] = h;
    gLv[go + 2 * CV] = l;
    bwd_edge_degree<3>(Dr, sX, sY, sGS, sGX, sR[3 * CV], CV, gxs, gr, bx, by);
    vsplit(gr, h, l);
    gHv[go + 3 * CV] = h;
    gLv[go + 3 * CV] = l;
    // fixed-order sums of (b_x, b_y) over this thread's channels, the warp, then (at the end) the warps
    float sx = hsum(bx), sy = hsum(by);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sx += __shfl_xor_sync(0xffffffffu, sx, o);
      sy += __shfl_xor_sync(0xffffffffu, sy, o);
    }
    if (lane == 0) {
      red[(q * 2 + 0) * nw + warp] = sx;
      red[(q * 2 + 1) * nw + warp] = sy;
    }
    if (q == np - 1 || meta[q + 1].j != m.j) {
      // end of a sender run piece: its sum becomes row Pg[first position of the piece]
      T* dst = Pgv + (size_t)(p0 + qs) * 16 * CV + t;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        dst[k * CV] = gxs[k];
        gxs[k] = zero;
      }
      qs = q + 1;
    }
    // stage s read by every thread: free for reuse (unless a wait ran out: then stop)
    if (__syncthreads_or(!arrived)) {
      qdone = q;
      break;
    }
    if (t == 0 && q + BE_STAGES < np) issue(nissued++);
  }
  // torque of every edge of the range: a = -R_e^T (b_x, b_y, 0), g_r += (a x r) / |r|^2
  for (int q = t; q < np; q += CV) {
    const long long e = e0 + meta[q].el;
    float sx = 0.f, sy = 0.f;
    for (int w = 0; w < nw; ++w) {
      sx += red[(q * 2 + 0) * nw + w];
      sy += red[(q * 2 + 1) * nw + w];
    }
    const float vx = svec[4 * q], vy = svec[4 * q + 1], vz = svec[4 * q + 2];
    const float d2 = vx * vx + vy * vy + vz * vz;
    const float inv = rsqrtf(d2);
    float Rf[3][3];
    edge_frame<float>(vx * inv, vy * inv, vz * inv, Rf);
    const float ax = -(Rf[0][0] * sx + Rf[1][0] * sy);
    const float ay = -(Rf[0][1] * sx + Rf[1][1] * sy);
    const float az = -(Rf[0][2] * sx + Rf[1][2] * sy);
    const float id2 = 1.f / d2;
    g_r[3 * e + 0] += (ay * vz - az * vy) * id2;
    g_r[3 * e + 1] += (az * vx - ax * vz) * id2;
    g_r[3 * e + 2] += (ax * vy - ay * vx) * id2;
  }
  // after a wait that ran out, wait (bounded) for the copies still in flight so that none is
  // landing in shared memory when the block exits
  if (t == 0)
    for (int q = qdone; q < nissued; ++q) tc::mbar_wait(&full[q % BE_STAGES], (uint32_t)((q / BE_STAGES) & 1));
}

// channels per thread of the backward edge kernel.  One: with the ring's shared memory
// allowing three blocks per SM, C threads per block keep the most warps resident (the
// kernel is bound by resident warps; two channels per thread measured 10 % slower), and
// C threads always fill whole warps, which the torque sums reduce over.
constexpr int BE_V = 1;

// g_x[sender] += the cohort's sender runs, each the sum of its pieces in position order: a run
// [b, en) has pieces starting at b and at every multiple of `per` inside it (rows of Pg).
// One block of C threads per run (runs x, x + gridDim.x, ...), all 16 components at once.
__global__ void k_gx_combine(long long e0, long long e1, int C, int cohort_idx, int per, const int* __restrict__ send,
                             const int* __restrict__ perm, const int* __restrict__ seg, const int* __restrict__ nseg,
                             const float* __restrict__ Pg, float* __restrict__ gx) {
  const int c = threadIdx.x;
  const int ns = nseg[cohort_idx];
  const int n = (int)(e1 - e0);
  for (int r = blockIdx.x; r < ns; r += gridDim.x) {
    const int b = seg[e0 + r], en = r + 1 < ns ? seg[e0 + r + 1] : n;
    float* g = gx + (size_t)send[e0 + perm[e0 + b]] * 16 * C + c;
    float acc[16], old[16];
    const float* P0 = Pg + (size_t)b * 16 * C + c;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      acc[k] = P0[k * C];
      old[k] = g[k * C];
    }
    for (int p = (b / per + 1) * per; p < en; p += per) {
      const float* Pp = Pg + (size_t)p * 16 * C + c;
#pragma unroll
      for (int k = 0; k < 16; ++k) acc[k] += Pp[k * C];
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) g[k * C] = old[k] + acc[k];
  }
}

// ------------------------------------------------------------------ staged rotate-in / backward prep
// Rotate-in (BWD = false): XT[e - e0][col(k) C + c] = R_e[l(k)][c] (D_e x_send)[k][c] in
// the edge frame, m-major columns, split hi/lo for the products.  Backward prep (BWD =
// true): also GY = D_e gS[recv] (edge-frame output gradient), split.  Rotate-in with R null
// rotates the rows unscaled: called with the receivers as `send` and gS as `x`, it writes g_y
// alone (the backward prep when y is kept from the forward).  x~ and g_y rows are 16C
// floats.  One block of C / V threads (V adjacent channels each, vector loads and stores) per
// contiguous range of `per` edges.  The rows
// an edge reads (x of the sender, gS of the receiver, R and its Wigner-D blocks) are
// brought into an RS_STAGES-deep shared-memory ring by bulk copies issued by thread 0
// ahead of use.
constexpr int RS_STAGES = 3;         // at most 4: the barriers take 32 bytes before the metadata

// Whether the backward prep stages the receiver's gS row per edge (else it reads it from global
// memory: in edge order consecutive edges share the receiver, so L1 serves the repeats).  Both
// measured the same: with twice the resident warps the kernel is no faster, its 32 KB of
// writes per edge bound it.
constexpr bool RS_STAGE_G = true;
__host__ __device__ inline size_t rs_stage_floats(int C, bool bwd) {
  return (size_t)(bwd && RS_STAGE_G ? 36 : 20) * C + NDBLK;
}
__host__ __device__ inline size_t rs_smem_bytes(int C, bool bwd) {
  return RS_STAGES * rs_stage_floats(C, bwd) * 4 + 32 + (size_t)BE_MAXP * 4 * 4;
}
inline int rs_per(long long n, int sms, int blocks_per_sm) {
  const long long want = (n + (long long)blocks_per_sm * sms - 1) / ((long long)blocks_per_sm * sms);
  return (int)std::max<long long>(1, std::min<long long>(BE_MAXP, want));
}

// degree-L block for V channels: rotate v (node layout, stride CV vectors) by D^L into the
// edge frame, scale by Rl and store the 3xTF32 split into m-major columns
template <int L, typename T>
__device__ __forceinline__ void rotate_write_degree_v(const float* __restrict__ Dr, const T* __restrict__ v, int CV,
                                                      T Rl, T* __restrict__ hi, T* __restrict__ lo) {
  constexpr int W = 2 * L + 1, O = L * L;
  const float* B = Dr + dblk_off(L);
  T a[W];
#pragma unroll
  for (int n = 0; n < W; ++n) a[n] = v[(O + n) * CV];
#pragma unroll
  for (int m = 0; m < W; ++m) {
    T u = vset<T>(0.f);
#pragma unroll
    for (int n = 0; n < W; ++n) u = vfma(B[m * W + n], a[n], u);
    u = vmul(u, Rl);
    T h, l;
    vsplit(u, h, l);
    const int col = col_of_k(O + m) * CV;
    hi[col] = h;
    lo[col] = l;
  }
}

template <bool BWD, int V>
__global__ void __launch_bounds__(256)
    k_rotate_staged(long long e0, long long e1, int C, int per, const int* __restrict__ recv,
                    const int* __restrict__ send, const int* __restrict__ rrow, const float* __restrict__ D,
                    const float* __restrict__ R, const float* __restrict__ x, const float* __restrict__ gS,
                    float* __restrict__ XT, float* __restrict__ XTlo, float* __restrict__ GYhi,
                    float* __restrict__ GYlo) {
  typedef typename VecT<V>::type T;
  extern __shared__ __align__(128) unsigned char rs_smem[];
  const size_t SF = rs_stage_floats(C, BWD);
  float* stage0 = reinterpret_cast<float*>(rs_smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(rs_smem + RS_STAGES * SF * 4);
  int4* meta = reinterpret_cast<int4*>(full + 4);                         // [BE_MAXP] (j, i, rr, -), 16-byte aligned
  const int t = threadIdx.x, CV = C / V;
  const int n = (int)(e1 - e0);
  const int p0 = blockIdx.x * per, p1 = min(n, p0 + per);
  if (p0 >= p1) return;
  const int np = p1 - p0;
  if (t == 0) {
    for (int s = 0; s < RS_STAGES; ++s) tc::mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int q = t; q < np; q += CV) {
    const long long e = e0 + p0 + q;
    meta[q] = make_int4(send[e], BWD ? recv[e] : 0, rrow ? rrow[e] : (int)e, 0);
  }
  __syncthreads();
  constexpr bool SG = BWD && RS_STAGE_G;
  const bool hasR = R != nullptr;      // forward form without R: the rows are rotated unscaled
  const uint32_t bX = 64u * C, bG = SG ? 64u * C : 0u, bR = hasR ? 16u * C : 0u;
  const int offG = 16 * C, offR = (SG ? 32 : 16) * C, offD = offR + 4 * C;
  auto issue = [&](int q) {
    const int s = q % RS_STAGES;
    float* st = stage0 + s * SF;
    const int4 m = meta[q];
    tc::mbar_expect_tx(&full[s], bX + bG + bR + NDBLK * 4);
    bulk_g2s(st, x + (size_t)m.x * 16 * C, bX, &full[s]);
    if (SG) bulk_g2s(st + offG, gS + (size_t)m.y * 16 * C, bG, &full[s]);
    if (hasR) bulk_g2s(st + offR, R + (size_t)m.z * 4 * C, bR, &full[s]);
    bulk_g2s(st + offD, D + (size_t)(e0 + p0 + q) * NDBLK, NDBLK * 4, &full[s]);
  };
  int nissued = 0;                     // positions whose copies thread 0 has issued
  if (t == 0)
    for (; nissued < min(RS_STAGES, np); ++nissued) issue(nissued);
  T* XTv = reinterpret_cast<T*>(XT);
  T* XLv = reinterpret_cast<T*>(XTlo);
  T* GHv = reinterpret_cast<T*>(GYhi);
  T* GLv = reinterpret_cast<T*>(GYlo);
  int qdone = np;                      // positions waited for by every thread
#pragma unroll 1
  for (int q = 0; q < np; ++q) {
    const int s = q % RS_STAGES;
    // bounded; a timeout sets the device error, and the block leaves the loop (all threads at once)
    const bool arrived = tc::mbar_wait(&full[s], (uint32_t)((q / RS_STAGES) & 1));
    const float* st = stage0 + s * SF;
    const T* sX = reinterpret_cast<const T*>(st) + t;
    const T* sR = reinterpret_cast<const T*>(st + offR) + t;
    const float* Dr = st + offD;
    const size_t ro = (size_t)(p0 + q) * 16 * CV + t;
    const T one = vset<T>(1.f);
    rotate_write_degree_v<0>(Dr, sX, CV, hasR ? sR[0] : one, XTv + ro, XLv + ro);
    rotate_write_degree_v<1>(Dr, sX, CV, hasR ? sR[CV] : one, XTv + ro, XLv + ro);
    rotate_write_degree_v<2>(Dr, sX, CV, hasR ? sR[2 * CV] : one, XTv + ro, XLv + ro);
    rotate_write_degree_v<3>(Dr, sX, CV, hasR ? sR[3 * CV] : one, XTv + ro, XLv + ro);
    if (BWD) {
      const T* sG = SG ? reinterpret_cast<const T*>(st + offG) + t
                       : reinterpret_cast<const T*>(gS + (size_t)meta[q].y * 16 * C) + t;
      rotate_write_degree_v<0>(Dr, sG, CV, one, GHv + ro, GLv + ro);
      rotate_write_degree_v<1>(Dr, sG, CV, one, GHv + ro, GLv + ro);
      rotate_write_degree_v<2>(Dr, sG, CV, one, GHv + ro, GLv + ro);
      rotate_write_degree_v<3>(Dr, sG, CV, one, GHv + ro, GLv + ro);
    }
    // stage s read by every thread: free for reuse (unless a wait ran out: then stop)
    if (__syncthreads_or(!arrived)) {
      qdone = q;
      break;
    }
    if (t == 0 && q + RS_STAGES < np) issue(nissued++);
  }
  // after a wait that ran out, wait (bounded) for the copies still in flight
  if (t == 0)
    for (int q = qdone; q < nissued; ++q) tc::mbar_wait(&full[q % RS_STAGES], (uint32_t)((q / RS_STAGES) & 1));
}

// vector widths (channels per thread) of the staged rotate kernels
constexpr int RS_V_FWD = 4;
constexpr int RS_V_BWD = 1;

// ------------------------------------------------------------------ cohort sender order
// For each cohort: its edges sorted by (sender, edge), the start of each sender
// segment, and the number of segments.  One block per cohort.
__global__ void k_cohort_sort(long long E, int cohort, const int* __restrict__ send, int* __restrict__ perm,
                              int* __restrict__ seg, int* __restrict__ nseg) {
  extern __shared__ unsigned long long keys[];     // [P]
  __shared__ int wsum[32];
  const long long e0 = (long long)blockIdx.x * cohort;
  const int n = (int)min((long long)cohort, E - e0);
  int P = 1;
  while (P < n) P <<= 1;
  for (int k = threadIdx.x; k < P; k += blockDim.x)
    keys[k] = k < n ? (((unsigned long long)(unsigned)send[e0 + k]) << 21) | (unsigned long long)k : ~0ull;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < P; t += blockDim.x) {
        const int partner = t ^ stride;
        if (partner > t) {
          const bool up = (t & size) == 0;
          const unsigned long long a = keys[t], b = keys[partner];
          if ((a > b) == up) { keys[t] = b; keys[partner] = a; }
        }
      }
      __syncthreads();
    }
  }
  // segment starts: serial over chunks, each thread a contiguous chunk
  const int T = blockDim.x;
  const int per = (n + T - 1) / T;
  const int b = threadIdx.x * per, en = min(n, b + per);
  int cnt = 0;
  for (int k = b; k < en; ++k)
    if (k == 0 || (keys[k] >> 21) != (keys[k - 1] >> 21)) ++cnt;
  // block exclusive scan of cnt (T <= 1024)
  int v = cnt;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) wsum[w] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int q = 0; q < (T + 31) / 32; ++q) { const int y = wsum[q]; wsum[q] = acc; acc += y; }
    nseg[blockIdx.x] = acc;
  }
  __syncthreads();
  int pos = wsum[w] + v - cnt;
  for (int k = b; k < en; ++k) {
    if (k == 0 || (keys[k] >> 21) != (keys[k - 1] >> 21)) seg[e0 + pos++] = k;
    perm[e0 + k] = (int)(keys[k] & ((1ull << 21) - 1));
  }
}

// ------------------------------------------------------------------ forces and virial
// F_i = sum over receiver i's edges of (g_e - g_mirror(e)), edge order
__global__ void k_forces(int N, const int* __restrict__ recv_off, const int* __restrict__ mirror,
                         const float* __restrict__ g_r, float* __restrict__ F) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  float fx = 0.f, fy = 0.f, fz = 0.f;
  for (int e = recv_off[i]; e < recv_off[i + 1]; ++e) {
    const int m = mirror[e];
    fx += g_r[3 * e + 0] - g_r[3 * m + 0];
    fy += g_r[3 * e + 1] - g_r[3 * m + 1];
    fz += g_r[3 * e + 2] - g_r[3 * m + 2];
  }
  F[3 * i + 0] = fx;
  F[3 * i + 1] = fy;
  F[3 * i + 2] = fz;
}

constexpr int VIR_BLOCKS = 256;
// virial partials: block b sums edges b, b + VIR_BLOCKS*T, ... in double
__global__ void k_virial_partial(long long E, const float* __restrict__ vec, const float* __restrict__ g_r,
                                 double* __restrict__ part) {
  __shared__ double s[9][256];
  const int t = threadIdx.x;
  double acc[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  for (long long e = (long long)blockIdx.x * blockDim.x + t; e < E; e += (long long)gridDim.x * blockDim.x)
    for (int a = 0; a < 3; ++a)
      for (int b = 0; b < 3; ++b) acc[a * 3 + b] -= (double)vec[3 * e + a] * (double)g_r[3 * e + b];
  for (int q = 0; q < 9; ++q) s[q][t] = acc[q];
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (t < w)
      for (int q = 0; q < 9; ++q) s[q][t] += s[q][t + w];
    __syncthreads();
  }
  if (t == 0)
    for (int q = 0; q < 9; ++q) part[blockIdx.x * 9 + q] = s[q][0];
}

__global__ void k_virial_final(int nb, const double* __restrict__ part, float* __restrict__ vir) {
  const int q = threadIdx.x;
  if (q >= 9) return;
  double s = 0.0;
  for (int b = 0; b < nb; ++b) s += part[b * 9 + q];
  vir[q] = (float)s;
}

// x_0: degree 0 = emb[species], higher degrees zero
__global__ void k_embed(int N, int C, const int* __restrict__ species, int n_species, const float* __restrict__ emb,
                        float* __restrict__ x) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * 16 * C) return;
  const int i = idx / (16 * C), r = idx % (16 * C), k = r / C, c = r % C;
  int s = species ? species[i] : 0;
  if (s < 0 || s >= n_species) { set_device_error(DEV_ERR_INDEX); s = 0; }
  x[idx] = k == 0 ? emb[(size_t)s * C + c] : 0.f;
}

__global__ void k_scale(size_t n, float a, float* __restrict__ v) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] *= a;
}

}  // namespace emp
