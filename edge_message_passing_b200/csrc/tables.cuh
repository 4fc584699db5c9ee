// Certified radial tables: an opt-in replacement of the radial network's hidden layers
// (page FastMACE, "Rewrite screens: adopted and rejected", OPT6-T04 / OPT6-T05 radial
// tables: per species pair and interaction, the radial chain up to the hidden layers'
// output as float64-fitted piecewise Chebyshev tables of degree 10 on dyadic pieces,
// values and length derivatives within 1e-7 of their local scale; float32 on the device).
//
// The tabulated function is h2(d) in R^64 (Bessel basis with the polynomial envelope, W1,
// SiLU, W2, SiLU) of one layer's radial network; the head R = W3 h2 stays the tensor-core
// product.  The tables are built on the host in double precision when the caller enables
// them: [0, rc] is bisected into dyadic pieces [i rc / 2^L, (i+1) rc / 2^L] until, at 48
// Chebyshev extrema of a piece (its ends included), every output of the degree-10
// interpolant through the 11 Chebyshev points of the first kind, and of its derivative,
// is within tol of that output's local scale (its largest magnitude on the piece, at least
// 1e-3 of its largest magnitude on the whole range).  On the device a row's length d
// selects its piece through a map of the finest level's bins, t = (2 d - a - b) / (b - a),
// and Clenshaw's recurrence sums the series (forward: h2; backward: the derivative series
// dotted with dE/dh2, giving dE/dd).
#pragma once
#include <vector>
#include <cmath>
#include "emp_common.cuh"
#include "model.cuh"
#include "conv.cuh"

namespace emp {
namespace tab {

constexpr int DEG = 10;                      // polynomial degree
constexpr int NC = DEG + 1;                  // coefficients per output
constexpr int H = 64;                        // tabulated outputs (the hidden width)
constexpr int MAX_LEVEL = 14;
constexpr int N_CHECK = 48;
constexpr double FLOOR = 1e-3;
// one piece on the device: [a, 2/(b-a), 0, 0], c[NC][H], dc[DEG][H] (d-derivative series)
constexpr int PIECE_FLOATS = 4 + NC * H + DEG * H;

struct HostPiece {
  double a, b;
  int level;
  std::vector<double> c, dc;                 // [NC][H], [DEG][H]
};

// ------------------------------------------------------------------ the function, in double
// sin(k d) / d = k j0(k d) and its d-derivative -k^2 j1(k d), by series for small arguments
inline void sinc_terms(double k, double d, double& f, double& df) {
  const double x = k * d;
  if (x < 0.5) {
    const double x2 = x * x;
    f = k * (1.0 - x2 / 6.0 * (1.0 - x2 / 20.0 * (1.0 - x2 / 42.0 * (1.0 - x2 / 72.0 * (1.0 - x2 / 110.0)))));
    const double j1 = x / 3.0 * (1.0 - x2 / 10.0 * (1.0 - x2 / 28.0 * (1.0 - x2 / 54.0 * (1.0 - x2 / 88.0 * (1.0 - x2 / 130.0)))));
    df = -k * k * j1;
  } else {
    const double s = std::sin(x), c = std::cos(x);
    f = s / d;
    df = -k * k * (s / (x * x) - c / x);
  }
}

inline double silu_d(double z) { return z / (1.0 + std::exp(-z)); }
inline double dsilu_d(double z) {
  const double s = 1.0 / (1.0 + std::exp(-z));
  return s * (1.0 + z * (1.0 - s));
}

// h2(d) and dh2/dd of one radial network (W1 [64][8], W2 [64][64], float weights)
inline void hidden(const float* W1, const float* W2, double rc, double d, double* h2, double* dh2) {
  double e[8], de[8];
  const double x = d / rc;
  double u = 0.0, du = 0.0;
  if (x < 1.0) {
    const double x2 = x * x, x5 = x2 * x2 * x, x6 = x5 * x;
    u = 1.0 + x6 * (-28.0 + x * (48.0 - 21.0 * x));
    du = x5 * (-168.0 + x * (336.0 - 168.0 * x)) / rc;
  }
  for (int n = 0; n < 8; ++n) {
    const double k = M_PI * (n + 1) / rc;
    double f, df;
    sinc_terms(k, d, f, df);
    e[n] = u * f;
    de[n] = du * f + u * df;
  }
  double h1[H], dh1[H];
  for (int j = 0; j < H; ++j) {
    double z = 0.0, dz = 0.0;
    for (int n = 0; n < 8; ++n) {
      z += (double)W1[j * 8 + n] * e[n];
      dz += (double)W1[j * 8 + n] * de[n];
    }
    h1[j] = silu_d(z);
    dh1[j] = dsilu_d(z) * dz;
  }
  for (int o = 0; o < H; ++o) {
    double z = 0.0, dz = 0.0;
    for (int i = 0; i < H; ++i) {
      z += (double)W2[o * H + i] * h1[i];
      dz += (double)W2[o * H + i] * dh1[i];
    }
    h2[o] = silu_d(z);
    dh2[o] = dsilu_d(z) * dz;
  }
}

// ------------------------------------------------------------------ building a table
// interpolant through the Chebyshev points of the first kind on [a, b]: coefficients c[NC][H]
// and those of its d-derivative dc[DEG][H]
inline void fit_piece(const float* W1, const float* W2, double rc, double a, double b, std::vector<double>& c,
                      std::vector<double>& dc) {
  std::vector<double> f(NC * H);
  double h2[H], dh2[H];
  for (int j = 0; j < NC; ++j) {
    const double t = std::cos(M_PI * (2 * j + 1) / (2.0 * NC));
    hidden(W1, W2, rc, 0.5 * (a + b) + 0.5 * (b - a) * t, h2, dh2);
    for (int o = 0; o < H; ++o) f[j * H + o] = h2[o];
  }
  c.assign(NC * H, 0.0);
  for (int k = 0; k < NC; ++k)
    for (int j = 0; j < NC; ++j) {
      const double T = std::cos(k * M_PI * (2 * j + 1) / (2.0 * NC));
      for (int o = 0; o < H; ++o) c[k * H + o] += (2.0 / NC) * T * f[j * H + o];
    }
  for (int o = 0; o < H; ++o) c[o] *= 0.5;
  // derivative series: d_{k-1} = d_{k+1} + 2 k c_k, d_0 halved, then times 2 / (b - a)
  std::vector<double> d((NC + 1) * H, 0.0);
  for (int k = NC - 1; k >= 1; --k)
    for (int o = 0; o < H; ++o) d[(k - 1) * H + o] = d[(k + 1) * H + o] + 2.0 * k * c[k * H + o];
  for (int o = 0; o < H; ++o) d[o] *= 0.5;
  dc.assign(DEG * H, 0.0);
  for (int k = 0; k < DEG; ++k)
    for (int o = 0; o < H; ++o) dc[k * H + o] = d[k * H + o] * (2.0 / (b - a));
}

inline double clenshaw(const std::vector<double>& c, int n, int o, double t) {
  double b1 = 0.0, b2 = 0.0;
  for (int k = n - 1; k >= 1; --k) {
    const double b0 = 2.0 * t * b1 - b2 + c[k * H + o];
    b2 = b1;
    b1 = b0;
  }
  return t * b1 - b2 + c[o];
}

// the table of one radial network on [0, rc]; pieces ordered by their start
inline std::vector<HostPiece> build(const float* W1, const float* W2, double rc, double tol) {
  double gs[H] = {0}, gds[H] = {0};
  double h2[H], dh2[H];
  for (int q = 0; q < 4096; ++q) {
    hidden(W1, W2, rc, rc * (q + 0.5) / 4096.0, h2, dh2);
    for (int o = 0; o < H; ++o) {
      gs[o] = std::max(gs[o], std::fabs(h2[o]));
      gds[o] = std::max(gds[o], std::fabs(dh2[o]));
    }
  }
  std::vector<HostPiece> out;
  struct Todo { double a, b; int level; };
  std::vector<Todo> stack{{0.0, rc, 0}};
  while (!stack.empty()) {
    const Todo td = stack.back();
    stack.pop_back();
    HostPiece p{td.a, td.b, td.level, {}, {}};
    fit_piece(W1, W2, rc, td.a, td.b, p.c, p.dc);
    double s[H] = {0}, sd[H] = {0};
    static thread_local std::vector<double> fv, fd, tt;
    fv.assign(N_CHECK * H, 0.0);
    fd.assign(N_CHECK * H, 0.0);
    tt.assign(N_CHECK, 0.0);
    for (int q = 0; q < N_CHECK; ++q) {
      const double x = td.a + 0.5 * (td.b - td.a) * (1.0 - std::cos(M_PI * q / (N_CHECK - 1)));
      hidden(W1, W2, rc, x, &fv[q * H], &fd[q * H]);
      tt[q] = (2.0 * x - td.a - td.b) / (td.b - td.a);
      for (int o = 0; o < H; ++o) {
        s[o] = std::max(s[o], std::fabs(fv[q * H + o]));
        sd[o] = std::max(sd[o], std::fabs(fd[q * H + o]));
      }
    }
    bool ok = true;
    for (int q = 0; q < N_CHECK && ok; ++q)
      for (int o = 0; o < H && ok; ++o) {
        const double so = std::max(s[o], FLOOR * gs[o]), sdo = std::max(sd[o], FLOOR * gds[o]);
        if (std::fabs(clenshaw(p.c, NC, o, tt[q]) - fv[q * H + o]) > tol * so) ok = false;
        if (std::fabs(clenshaw(p.dc, DEG, o, tt[q]) - fd[q * H + o]) > tol * sdo) ok = false;
      }
    if (ok || td.level >= MAX_LEVEL) {
      out.push_back(std::move(p));
    } else {
      const double m = 0.5 * (td.a + td.b);
      stack.push_back({m, td.b, td.level + 1});
      stack.push_back({td.a, m, td.level + 1});
    }
  }
  std::sort(out.begin(), out.end(), [](const HostPiece& x, const HostPiece& y) { return x.a < y.a; });
  return out;
}

// ------------------------------------------------------------------ device side
// hdr[4 q]: finest level L, first piece, first map entry, pieces (q = layer * n_pairs + pair);
// map[first map entry + bin] for the 2^L bins of [0, rc): the piece holding the bin
struct Args {
  const int* hdr;
  const int* map;
  const float* pieces;
  int layer, n_pairs, n_species, pair_radial;
  int fixed_pair;                            // >= 0: every row uses this network
  float rc;
};

__device__ __forceinline__ int row_pair(const Args& a, const int* recv, const int* send, const int* species, int e) {
  if (a.fixed_pair >= 0) return a.fixed_pair;
  return a.pair_radial ? pair_of(species[recv[e]], species[send[e]], a.n_species) : 0;
}

__device__ __forceinline__ const float* piece_of(const Args& a, int p, float d) {
  const int* h = a.hdr + 4 * (a.layer * a.n_pairs + p);
  const int L = h[0], nbin = 1 << L;
  int bin = (int)(d * (float)nbin / a.rc);
  bin = bin < 0 ? 0 : bin >= nbin ? nbin - 1 : bin;
  return a.pieces + (size_t)(h[1] + a.map[h[2] + bin]) * PIECE_FLOATS;
}

constexpr int TAB_THREADS = 256;
constexpr int TAB_LANES = 16;                // threads per row, 4 outputs each

// h2 rows (3xTF32 split) of the radial network from the table: the input of the head R = h2 W3^T
__global__ void __launch_bounds__(TAB_THREADS) k_radial_h2_table(long long E, const int* __restrict__ perm,
                                                                 const float* __restrict__ dist,
                                                                 const int* __restrict__ recv,
                                                                 const int* __restrict__ send,
                                                                 const int* __restrict__ species, Args a,
                                                                 float* __restrict__ h2_hi, float* __restrict__ h2_lo) {
  const int lane = threadIdx.x % TAB_LANES, o = 4 * lane;
  for (long long r = ((long long)blockIdx.x * TAB_THREADS + threadIdx.x) / TAB_LANES; r < E;
       r += (long long)gridDim.x * (TAB_THREADS / TAB_LANES)) {
    const int e = perm ? perm[r] : (int)r;
    const float d = dist[e];
    const float* pc = piece_of(a, row_pair(a, recv, send, species, e), d);
    const float t = (d - pc[0]) * pc[1] - 1.0f;
    const float* c = pc + 4;
    float4 b1 = make_float4(0.f, 0.f, 0.f, 0.f), b2 = b1;
    const float t2 = 2.0f * t;
#pragma unroll
    for (int k = NC - 1; k >= 1; --k) {
      const float4 ck = *reinterpret_cast<const float4*>(c + k * H + o);
      const float4 b0 = make_float4(fmaf(t2, b1.x, ck.x - b2.x), fmaf(t2, b1.y, ck.y - b2.y), fmaf(t2, b1.z, ck.z - b2.z),
                                    fmaf(t2, b1.w, ck.w - b2.w));
      b2 = b1;
      b1 = b0;
    }
    const float4 c0 = *reinterpret_cast<const float4*>(c + o);
    const float v[4] = {fmaf(t, b1.x, c0.x - b2.x), fmaf(t, b1.y, c0.y - b2.y), fmaf(t, b1.z, c0.z - b2.z),
                        fmaf(t, b1.w, c0.w - b2.w)};
    float hi[4], lo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      hi[q] = tf32_rna(v[q]);
      lo[q] = tf32_rna(v[q] - hi[q]);
    }
    *reinterpret_cast<float4*>(h2_hi + (size_t)r * H + o) = make_float4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<float4*>(h2_lo + (size_t)r * H + o) = make_float4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// dE/dd = sum_j dE/dh2_j dh2_j/dd from the table's derivative series; adds (dE/dd) rhat to g_r
__global__ void __launch_bounds__(TAB_THREADS) k_radial_bwd_table(long long E, const int* __restrict__ perm,
                                                                  const float* __restrict__ dist,
                                                                  const float* __restrict__ vec,
                                                                  const int* __restrict__ recv,
                                                                  const int* __restrict__ send,
                                                                  const int* __restrict__ species, Args a,
                                                                  const float* __restrict__ gh2,
                                                                  float* __restrict__ g_r) {
  // a warp holds two rows (16 lanes each) and loops while its first row exists, so that every
  // lane takes part in the shuffles below
  const int lane = threadIdx.x % TAB_LANES, o = 4 * lane, half = (threadIdx.x & 31) / TAB_LANES;
  const long long warp = ((long long)blockIdx.x * TAB_THREADS + threadIdx.x) >> 5;
  const long long stride = (long long)gridDim.x * (TAB_THREADS / TAB_LANES);
  for (long long base = 2 * warp; base < E; base += stride) {
    const long long r = base + half;
    const bool live = r < E;
    float s = 0.f;
    int e = 0;
    if (live) {
      e = perm ? perm[r] : (int)r;
      const float d = dist[e];
      const float* pc = piece_of(a, row_pair(a, recv, send, species, e), d);
      const float t = (d - pc[0]) * pc[1] - 1.0f;
      const float* c = pc + 4 + NC * H;        // the derivative series
      float4 b1 = make_float4(0.f, 0.f, 0.f, 0.f), b2 = b1;
      const float t2 = 2.0f * t;
#pragma unroll
      for (int k = DEG - 1; k >= 1; --k) {
        const float4 ck = *reinterpret_cast<const float4*>(c + k * H + o);
        const float4 b0 = make_float4(fmaf(t2, b1.x, ck.x - b2.x), fmaf(t2, b1.y, ck.y - b2.y),
                                      fmaf(t2, b1.z, ck.z - b2.z), fmaf(t2, b1.w, ck.w - b2.w));
        b2 = b1;
        b1 = b0;
      }
      const float4 c0 = *reinterpret_cast<const float4*>(c + o);
      const float4 g = *reinterpret_cast<const float4*>(gh2 + (size_t)r * H + o);
      s = g.x * fmaf(t, b1.x, c0.x - b2.x);
      s = fmaf(g.y, fmaf(t, b1.y, c0.y - b2.y), s);
      s = fmaf(g.z, fmaf(t, b1.z, c0.z - b2.z), s);
      s = fmaf(g.w, fmaf(t, b1.w, c0.w - b2.w), s);
    }
    // fixed-order sum over the 16 lanes of the row
#pragma unroll
    for (int off = TAB_LANES / 2; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (live && lane == 0) {
      const float inv = 1.f / dist[e];
      g_r[3 * (size_t)e + 0] += s * vec[3 * (size_t)e + 0] * inv;
      g_r[3 * (size_t)e + 1] += s * vec[3 * (size_t)e + 1] * inv;
      g_r[3 * (size_t)e + 2] += s * vec[3 * (size_t)e + 2] * inv;
    }
  }
}

}  // namespace tab
}  // namespace emp
