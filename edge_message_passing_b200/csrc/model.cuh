// Model object: device copies of the weights, the stacked SO(2) blocks (and
// their transposes for the input gradient), their 3xTF32 split, and the
// rotation-generator values used by the edge-direction gradient.
#pragma once
#include <vector>
#include <cstring>
#include "emp_common.cuh"
#include "so2_tc.cuh"

namespace emp {

// generator values on the 18 structural pairs (a < b): J[a][b] for J_x and J_y
__constant__ float c_jx[NJPAIR];
__constant__ float c_jy[NJPAIR];

struct Model {
  emp_model_spec spec;
  int H, Hro, n_pairs;
  // device pointers (all inside one allocation)
  float* emb;                   // [S][C]
  float* rad;                   // per layer per pair: W1 [H][8], W2 [H][H], W3 [4C][H]
  float* so2_fwd;               // per layer: 72 C^2 stacked blocks, [n][k]
  float* so2_bwd;               // per layer: transposed blocks
  float* so2_fwd_hi;            // 3xTF32 split of so2_fwd / so2_bwd
  float* so2_fwd_lo;
  float* so2_bwd_hi;
  float* so2_bwd_lo;
  float* ro_W;                  // [Hro][C]
  float* ro_w;                  // [Hro]
  float* ro_WT;                 // [C][Hro]
  void* base;
  int device;
  std::vector<So2BMaps> bmaps_fwd, bmaps_bwd;   // tensor maps of each layer's stacked blocks
  // radial head W3 [4C][64] of each (layer, pair) split for 3xTF32, and its transpose [64][4C]
  float *w3_hi, *w3_lo, *w3t_hi, *w3t_lo;
  std::vector<MapPair> w3_maps, w3t_maps;      // index t * n_pairs + p
  std::vector<MapPair> w3n_maps;                // the first C rows of W3 (degree-0 scales only)
  std::vector<MapPair> w3f_maps, w3fn_maps;     // the same for the fused radial kernel (its MMA N)
  std::vector<MapPair> w3t128_maps;             // W3^T for the grouped products (w3t_maps: the fused backward's)
  size_t w3_stride() const { return (size_t)4 * spec.C * 64; }
  // host copy of the radial weights (W1, W2, W3 per layer and pair), for building radial tables
  std::vector<float> rad_host;
  // certified radial tables (tables.cuh), when enabled: one device allocation
  void* tab_base = nullptr;
  int* tab_hdr = nullptr;
  int* tab_map = nullptr;
  float* tab_pieces = nullptr;
  bool tab_on = false;

  size_t rad_stride() const { return (size_t)H * 8 + (size_t)H * H + (size_t)4 * spec.C * H; }
  const float* W1(int t, int p) const { return rad + ((size_t)t * n_pairs + p) * rad_stride(); }
  const float* W2(int t, int p) const { return W1(t, p) + (size_t)H * 8; }
  const float* W3(int t, int p) const { return W2(t, p) + (size_t)H * H; }
  size_t so2_stride() const { return (size_t)WLAYER_CC * spec.C * spec.C; }
};

// ------------------------------------------------------------- host helpers
inline size_t weight_count(const emp_model_spec& s) {
  const size_t C = s.C, H = s.radial_hidden, Hro = s.readout_hidden > 0 ? s.readout_hidden : s.C;
  const size_t npair = s.pair_radial ? (size_t)s.n_species * (s.n_species + 1) / 2 : 1;
  size_t n = (size_t)s.n_species * C;
  for (int t = 0; t < s.n_layers; ++t) {
    n += npair * (H * s.n_basis + H * H + 4 * C * H);
    n += 16 * C * C;
    for (int m = 1; m <= 3; ++m) n += 2 * (size_t)(4 - m) * C * (4 - m) * C;
  }
  n += Hro * C + Hro;
  return n;
}

inline bool spec_ok(const emp_model_spec& s) {
  const int Hro = s.readout_hidden > 0 ? s.readout_hidden : s.C;
  return s.C >= 32 && s.C <= 256 && s.C % 32 == 0 && s.n_layers >= 1 && s.n_layers <= 16 &&
         s.n_species >= 1 && s.n_species <= 16 && s.n_basis == 8 && s.radial_hidden == 64 &&
         Hro >= 1 && Hro <= 256 && s.cohort_edges >= 128 && s.cohort_edges % 128 == 0 &&
         s.cohort_edges <= (1 << 14) && s.cutoff > 0.f && s.env_p == 6 && s.avg_degree > 0.f &&
         (!s.pair_radial || s.n_species * (s.n_species + 1) / 2 <= 32);
}

// forward-mode dual numbers for the exact generator J_k = d/de D(exp(e [e_k]x)) at e = 0
struct Dual {
  double v, d;
  __host__ __device__ Dual(double a = 0.0, double b = 0.0) : v(a), d(b) {}
};
__host__ __device__ inline Dual operator+(Dual a, Dual b) { return Dual(a.v + b.v, a.d + b.d); }
__host__ __device__ inline Dual operator-(Dual a, Dual b) { return Dual(a.v - b.v, a.d - b.d); }
__host__ __device__ inline Dual operator-(Dual a) { return Dual(-a.v, -a.d); }
__host__ __device__ inline Dual operator*(Dual a, Dual b) { return Dual(a.v * b.v, a.v * b.d + a.d * b.v); }
__host__ __device__ inline bool operator<(Dual a, Dual b) { return a.v < b.v; }

// J[k][84]: derivative of the 84 D values along rotation generator k
inline void generator_blocks(double J[3][NDBLK]) {
  for (int k = 0; k < 3; ++k) {
    Dual R[3][3];
    for (int a = 0; a < 3; ++a)
      for (int b = 0; b < 3; ++b) R[a][b] = Dual(a == b ? 1.0 : 0.0, 0.0);
    // [e_k]x : (e_k x v)
    const int p = (k + 1) % 3, q = (k + 2) % 3;
    R[q][p].d = 1.0;
    R[p][q].d = -1.0;
    Dual D[NDBLK];
    wigner_blocks<Dual>(R, D);
    for (int i = 0; i < NDBLK; ++i) J[k][i] = D[i].d;
  }
}

// value of block-diagonal generator J (84 layout) at component pair (a, b)
inline double gen_at(const double* J84, int a, int b) {
  int la = 0;
  while ((la + 1) * (la + 1) <= a) ++la;
  int lb = 0;
  while ((lb + 1) * (lb + 1) <= b) ++lb;
  if (la != lb) return 0.0;
  const int w = 2 * la + 1, ma = a - la * la, mb = b - la * la;
  return J84[dblk_off(la) + ma * w + mb];
}

// stacked SO(2) blocks of one layer from its raw W0, Wr_m, Wi_m (device kernel)
__global__ void k_stack_so2(const float* __restrict__ W0, const float* __restrict__ Wr1, const float* __restrict__ Wi1,
                            const float* __restrict__ Wr2, const float* __restrict__ Wi2, const float* __restrict__ Wr3,
                            const float* __restrict__ Wi3, int C, float* __restrict__ fwd, float* __restrict__ bwd) {
  const size_t total = (size_t)WLAYER_CC * C * C;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += (size_t)gridDim.x * blockDim.x) {
    int b = 3;
    while (b > 0 && idx < (size_t)wblk_off(b) * C * C) --b;
    const size_t local = idx - (size_t)wblk_off(b) * C * C;
    const int K = blk_width(b) * C;
    const int n = (int)(local / K), k = (int)(local % K);
    float v;
    if (b == 0) {
      v = W0[(size_t)n * K + k];
    } else {
      const int h = (4 - b) * C;
      const int sn = n / h, sk = k / h, i = n % h, j = k % h;
      const float* Wr = b == 1 ? Wr1 : b == 2 ? Wr2 : Wr3;
      const float* Wi = b == 1 ? Wi1 : b == 2 ? Wi2 : Wi3;
      // y+ = Wr x+ - Wi x- ; y- = Wi x+ + Wr x-
      if (sn == sk) v = Wr[(size_t)i * h + j];
      else v = (sn == 0 ? -1.f : 1.f) * Wi[(size_t)i * h + j];
    }
    fwd[idx] = v;
    bwd[(size_t)wblk_off(b) * C * C + (size_t)k * K + n] = v;
  }
}

// dst [cols][rows] = src [rows][cols]^T
__global__ void k_transpose(const float* __restrict__ src, float* __restrict__ dst, int rows, int cols) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * cols) return;
  const int r = idx / cols, c = idx % cols;
  dst[(size_t)c * rows + r] = src[idx];
}

// 3xTF32 split: hi = TF32(a), lo = TF32(a - hi), TF32 being round to nearest, ties away from zero,
// at the 10th explicit mantissa bit.  Done on the bits: add half of the 13 dropped bits' range to
// the magnitude and clear them (a carry out of the mantissa steps the exponent, which is the
// correct rounding up to the next binade; subnormals, zeros and infinities come out right too).
// Two full-rate integer operations, where the conversion instruction issues at a lower rate; the
// kernels that split whole tiles run it millions of times per launch.  emp_tf32_split_selftest
// checks it against cvt.rna.tf32.f32 on every non-NaN 32-bit pattern.
__device__ __forceinline__ float tf32_rna(float a) {
  return __uint_as_float((__float_as_uint(a) + 0x1000u) & 0xFFFFE000u);
}
// the same rounding by the conversion instruction (the self-test's reference)
__device__ __forceinline__ float tf32_rna_cvt(float a) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(a));
  return __uint_as_float(r);
}

__global__ void k_split_tf32(const float* __restrict__ a, float* __restrict__ hi, float* __restrict__ lo, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float h = tf32_rna(a[i]);
    hi[i] = h;
    lo[i] = tf32_rna(a[i] - h);
  }
}

}  // namespace emp
