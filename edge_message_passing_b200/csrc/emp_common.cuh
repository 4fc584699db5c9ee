// Internal definitions shared by the library's CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>

#include "emp.h"

namespace emp {

constexpr int NCOMP = 16;   // (lmax + 1)^2 irrep components for lmax = 3
constexpr int NDBLK = 84;   // floats of the block-diagonal Wigner-D per edge: 1 + 9 + 25 + 49

__host__ __device__ constexpr int lm_index(int l, int m) { return l * l + l + m; }
// start of degree l's (2l+1)^2 block inside the 84 floats
__host__ __device__ constexpr int dblk_off(int l) { return l == 0 ? 0 : l == 1 ? 1 : l == 2 ? 10 : 35; }

// SO(2) m-blocks (b = |m|): the rotated features of one edge are laid out as
// [ m=0: (l=0..3) | m=+1: (l=1..3) | m=-1: (l=1..3) | m=+2 | m=-2 | m=+3 | m=-3 ],
// each (l) entry a run of C channels.  Block b occupies columns
// [blk_off(b) C, (blk_off(b) + blk_width(b)) C) of the 16C-wide row.
__host__ __device__ constexpr int blk_width(int b) { return b == 0 ? 4 : b == 1 ? 6 : b == 2 ? 4 : 2; }
__host__ __device__ constexpr int blk_off(int b) { return b == 0 ? 0 : b == 1 ? 4 : b == 2 ? 10 : 14; }
// column (in units of C) of component (l, m)
__host__ __device__ constexpr int col_of(int l, int m) {
  return blk_off(m < 0 ? -m : m) + (m < 0 ? (4 - (-m)) : 0) + (l - (m < 0 ? -m : m));
}
// column (units of C) of component index k = lm
__host__ __device__ constexpr int col_of_k(int k) {
  return k == 0 ? col_of(0, 0)
       : k < 4 ? col_of(1, k - 2)
       : k < 9 ? col_of(2, k - 6)
       : col_of(3, k - 12);
}
// offset (units of C*C) of block b's stacked (K x K) weight in a layer's 72 C^2 floats
__host__ __device__ constexpr int wblk_off(int b) { return b == 0 ? 0 : b == 1 ? 16 : b == 2 ? 52 : 68; }
constexpr int WLAYER_CC = 72;   // sum over blocks of blk_width^2

// ------------------------------------------------------------- device errors
// Error codes recorded by kernels (first one wins); read by emp_last_device_error.
enum DeviceError : int {
  DEV_OK = 0,
  DEV_ERR_INDEX = 1,       // an index read from a buffer was out of range
  DEV_ERR_DEGREE = 2,      // a receiver had more candidates than the sort buffer holds
  DEV_ERR_TIMEOUT = 3,     // a bounded mbarrier wait ran out
  DEV_ERR_MIRROR = 4,      // mirror edge not found
};

__device__ int g_device_error = 0;   // the library is one translation unit

__device__ __forceinline__ void set_device_error(int code) { atomicCAS(&g_device_error, 0, code); }

// ------------------------------------------------------------- edge frame
// Two-chart rotation R with R rhat = z.  For rhat_z >= 0 it is the rotation
// about rhat x z taking rhat to z (Rodrigues form, stable since 1 + z >= 1):
//   R = [[1 - x^2/(1+z), -x y/(1+z), -x], [-x y/(1+z), 1 - y^2/(1+z), -y], [x, y, z]].
// For rhat_z < 0 a half turn about x is applied first: R = R'(x, -y, -z) diag(1, -1, -1).
template <typename T>
__host__ __device__ inline void edge_frame(T x, T y, T z, T R[3][3]) {
  const bool flip = z < T(0);
  if (flip) { y = -y; z = -z; }
  const T k = T(1) / (T(1) + z);
  R[0][0] = T(1) - x * x * k; R[0][1] = -x * y * k;        R[0][2] = -x;
  R[1][0] = -x * y * k;       R[1][1] = T(1) - y * y * k;  R[1][2] = -y;
  R[2][0] = x;                R[2][1] = y;                 R[2][2] = z;
  if (flip) {
    for (int i = 0; i < 3; ++i) { R[i][1] = -R[i][1]; R[i][2] = -R[i][2]; }
  }
}

// ------------------------------------------------------------- Wigner-D
// Real-basis rotation matrices by the Ivanic-Ruedenberg recursion (J. Phys.
// Chem. 100, 6342 (1996); erratum 102, 9099 (1998)): block l is built from
// block 1 (the Cartesian rotation in the (y, z, x) order) and block l-1.
// D[(m+l)(2l+1) + (n+l)] holds D^l_{m n}; the block maps global-frame
// components to frame components: u = D(R) x.
namespace ir {

template <typename T, int L>
__host__ __device__ __forceinline__ T r1(const T* R1, int i, int j) { return R1[(i + 1) * 3 + (j + 1)]; }

template <typename T, int L>
__host__ __device__ __forceinline__ T dprev(const T* Dp, int a, int b) {
  return Dp[(a + (L - 1)) * (2 * L - 1) + (b + (L - 1))];
}

// the recursion's P function for degree L (a in -(L-1)..L-1, b in -L..L)
template <typename T, int L>
__host__ __device__ __forceinline__ T Pf(const T* R1, const T* Dp, int i, int a, int b) {
  if (b == L) return r1<T, L>(R1, i, 1) * dprev<T, L>(Dp, a, L - 1) - r1<T, L>(R1, i, -1) * dprev<T, L>(Dp, a, -(L - 1));
  if (b == -L) return r1<T, L>(R1, i, 1) * dprev<T, L>(Dp, a, -(L - 1)) + r1<T, L>(R1, i, -1) * dprev<T, L>(Dp, a, L - 1);
  return r1<T, L>(R1, i, 0) * dprev<T, L>(Dp, a, b);
}

template <typename T, int L>
__host__ __device__ __forceinline__ void block(const T* R1, const T* Dp, T* Dl) {
#pragma unroll
  for (int m = -L; m <= L; ++m) {
#pragma unroll
    for (int n = -L; n <= L; ++n) {
      const int am = m < 0 ? -m : m;
      const double denom = (n == L || n == -L) ? double(2 * L * (2 * L - 1)) : double((L + n) * (L - n));
      const double cu = sqrt(double((L + m) * (L - m)) / denom);
      const double cv = 0.5 * sqrt((m == 0 ? 2.0 : 1.0) * double((L + am - 1) * (L + am)) / denom) * (m == 0 ? -1.0 : 1.0);
      const double cw = (m == 0) ? 0.0 : -0.5 * sqrt(double((L - am - 1) * (L - am)) / denom);
      T val = T(0);
      if (cu != 0.0) val = val + T(cu) * Pf<T, L>(R1, Dp, 0, m, n);
      if (cv != 0.0) {
        T V;
        if (m == 0) {
          V = Pf<T, L>(R1, Dp, 1, 1, n) + Pf<T, L>(R1, Dp, -1, -1, n);
        } else if (m > 0) {
          V = (m == 1) ? T(sqrt(2.0)) * Pf<T, L>(R1, Dp, 1, m - 1, n)
                       : Pf<T, L>(R1, Dp, 1, m - 1, n) - Pf<T, L>(R1, Dp, -1, -m + 1, n);
        } else {
          V = (m == -1) ? T(sqrt(2.0)) * Pf<T, L>(R1, Dp, -1, -m - 1, n)
                        : Pf<T, L>(R1, Dp, 1, m + 1, n) + Pf<T, L>(R1, Dp, -1, -m - 1, n);
        }
        val = val + T(cv) * V;
      }
      if (cw != 0.0) {
        T W = (m > 0) ? Pf<T, L>(R1, Dp, 1, m + 1, n) + Pf<T, L>(R1, Dp, -1, -m - 1, n)
                      : Pf<T, L>(R1, Dp, 1, m - 1, n) - Pf<T, L>(R1, Dp, -1, -m + 1, n);
        val = val + T(cw) * W;
      }
      Dl[(m + L) * (2 * L + 1) + (n + L)] = val;
    }
  }
}

}  // namespace ir

// All four blocks (84 values) from a 3x3 rotation R (u = D x maps global to frame).
template <typename T>
__host__ __device__ inline void wigner_blocks(const T R[3][3], T* D) {
  // degree 1 in the (y, z, x) order: D1[a][b] = R[s(a)][s(b)], s = (1, 2, 0)
  const int s[3] = {1, 2, 0};
  D[0] = T(1);
  T* D1 = D + dblk_off(1);
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b) D1[a * 3 + b] = R[s[a]][s[b]];
  ir::block<T, 2>(D1, D1, D + dblk_off(2));
  ir::block<T, 3>(D1, D + dblk_off(2), D + dblk_off(3));
}

// The 18 component pairs (a < b) on which the rotation generators J_x and J_y
// can be non-zero: same degree, |m| differing by one.
constexpr int NJPAIR = 18;
__host__ __device__ constexpr int jpair_a(int p) {
  // l = 1: (-1,0) (0,1) ; l = 2: (-2,-1) (-2,1) (-1,0) (0,1) (-1,2) (1,2)
  // l = 3: (-3,-2) (-3,2) (-2,-1) (-2,1) (-1,0) (0,1) (-2,3) (2,3) (-1,2) (1,2)
  return p == 0 ? lm_index(1, -1) : p == 1 ? lm_index(1, 0)
       : p == 2 ? lm_index(2, -2) : p == 3 ? lm_index(2, -2) : p == 4 ? lm_index(2, -1) : p == 5 ? lm_index(2, 0)
       : p == 6 ? lm_index(2, -1) : p == 7 ? lm_index(2, 1)
       : p == 8 ? lm_index(3, -3) : p == 9 ? lm_index(3, -3) : p == 10 ? lm_index(3, -2) : p == 11 ? lm_index(3, -2)
       : p == 12 ? lm_index(3, -1) : p == 13 ? lm_index(3, 0) : p == 14 ? lm_index(3, -2) : p == 15 ? lm_index(3, 2)
       : p == 16 ? lm_index(3, -1) : lm_index(3, 1);
}
__host__ __device__ constexpr int jpair_b(int p) {
  return p == 0 ? lm_index(1, 0) : p == 1 ? lm_index(1, 1)
       : p == 2 ? lm_index(2, -1) : p == 3 ? lm_index(2, 1) : p == 4 ? lm_index(2, 0) : p == 5 ? lm_index(2, 1)
       : p == 6 ? lm_index(2, 2) : p == 7 ? lm_index(2, 2)
       : p == 8 ? lm_index(3, -2) : p == 9 ? lm_index(3, 2) : p == 10 ? lm_index(3, -1) : p == 11 ? lm_index(3, 1)
       : p == 12 ? lm_index(3, 0) : p == 13 ? lm_index(3, 1) : p == 14 ? lm_index(3, 3) : p == 15 ? lm_index(3, 3)
       : p == 16 ? lm_index(3, 2) : lm_index(3, 2);
}

// ------------------------------------------------------------- misc math
// SiLU and its derivative with the fast exponential and division intrinsics (a few ulp):
// the radial network evaluates them 128-192 times per edge and layer
__device__ __forceinline__ float sigmoid_fast(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }
__device__ __forceinline__ float silu_fast(float z) { return z * sigmoid_fast(z); }
__device__ __forceinline__ float dsilu_fast(float z) {
  const float s = sigmoid_fast(z);
  return s * (1.0f + z * (1.0f - s));
}
__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }
__device__ __forceinline__ float dsilu_f(float z) {
  const float s = 1.0f / (1.0f + expf(-z));
  return s * (1.0f + z * (1.0f - s));
}

}  // namespace emp

#define EMP_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t _e = (expr);                                 \
    if (_e != cudaSuccess) return EMP_ERR_CUDA;              \
  } while (0)
