// Bit-exact cell-list neighbour list.
//
// An edge (i, j, S) exists iff r = (x_j - x_i) + S*L (per component, IEEE double,
// separate roundings) has d2 = (rx*rx + ry*ry) + rz*rz < rc*rc, (i, i, 0) excluded
// ("first-order SO(2) input-gradient path" page, workload section: the
// neighbour list of the perturbed diamond cells).  Atoms are binned by their
// wrapped coordinate into cells no smaller than rc (times 1 + 1e-9), so the
// stencil enumerates a superset of the edges in exact arithmetic; every
// candidate is then tested with the definition above, so the set is exact.
// Each receiver's edges are sorted by (sender, S) in shared memory, which makes
// the order independent of the (atomic) binning order.
#pragma once
#include "emp_common.cuh"

namespace emp {
namespace nl {

constexpr int MAX_CAND = 4096;       // sort buffer per receiver
constexpr int MAX_SHIFT = 127;       // |S| per component that the sort key holds (and its mirror -S)
constexpr int EMIT_THREADS = 512;

struct Grid {
  int nc[3];      // cells per dimension
  int s[3];       // stencil half-width per dimension
  double L[3];
  double rc2;
  int n_cells;
};

struct Ws {
  int* cell_of;       // [N]
  int* wrap;          // [N][3]
  int* cell_count;    // [N]  (n_cells <= N)
  int* cell_start;    // [N+1]
  int* cell_cursor;   // [N]
  int* cell_atoms;    // [N]
  int* deg;           // [N]
  int* flags;         // [4]: non-finite position, degree above MAX_CAND, shift beyond MAX_SHIFT
  long long* total;   // [1]
};

__device__ __forceinline__ bool within(const double* __restrict__ pos, int i, int j,
                                       int Sx, int Sy, int Sz, const Grid& G,
                                       double& rx, double& ry, double& rz) {
  rx = __dadd_rn(__dsub_rn(pos[3 * j + 0], pos[3 * i + 0]), __dmul_rn((double)Sx, G.L[0]));
  ry = __dadd_rn(__dsub_rn(pos[3 * j + 1], pos[3 * i + 1]), __dmul_rn((double)Sy, G.L[1]));
  rz = __dadd_rn(__dsub_rn(pos[3 * j + 2], pos[3 * i + 2]), __dmul_rn((double)Sz, G.L[2]));
  const double d2 = __dadd_rn(__dadd_rn(__dmul_rn(rx, rx), __dmul_rn(ry, ry)), __dmul_rn(rz, rz));
  return d2 < G.rc2 && !(i == j && Sx == 0 && Sy == 0 && Sz == 0);
}

__global__ void k_bin(const double* __restrict__ pos, int n, Grid G, Ws w) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int c[3];
  for (int d = 0; d < 3; ++d) {
    const double x = pos[3 * i + d];
    if (!isfinite(x)) { atomicExch(&w.flags[0], 1); c[d] = 0; w.wrap[3 * i + d] = 0; continue; }
    const double q = x / G.L[d];
    const double f = floor(q);
    w.wrap[3 * i + d] = (int)f;
    int ci = (int)((q - f) * G.nc[d]);
    ci = ci < 0 ? 0 : (ci >= G.nc[d] ? G.nc[d] - 1 : ci);
    c[d] = ci;
  }
  const int cell = (c[0] * G.nc[1] + c[1]) * G.nc[2] + c[2];
  w.cell_of[i] = cell;
  atomicAdd(&w.cell_count[cell], 1);
}

// exclusive scan of `in[n]` into `out[n+1]` by one block (sizes here are <= N)
__global__ void k_scan(const int* __restrict__ in, int* __restrict__ out, int n, long long* total) {
  __shared__ int partial[1024];
  const int t = threadIdx.x, T = blockDim.x;
  const int per = (n + T - 1) / T;
  const int b = t * per, e = min(n, b + per);
  int s = 0;
  for (int k = b; k < e; ++k) s += in[k];
  partial[t] = s;
  __syncthreads();
  if (t == 0) {
    int acc = 0;
    for (int k = 0; k < T; ++k) { int v = partial[k]; partial[k] = acc; acc += v; }
    out[n] = acc;
    if (total) *total = acc;
  }
  __syncthreads();
  int acc = partial[t];
  for (int k = b; k < e; ++k) { out[k] = acc; acc += in[k]; }
}

__global__ void k_fill_cells(int n, Ws w) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int c = w.cell_of[i];
  const int k = atomicAdd(&w.cell_cursor[c], 1);
  w.cell_atoms[w.cell_start[c] + k] = i;
}

__device__ __forceinline__ void cell_coords(int cell, const Grid& G, int c[3]) {
  c[2] = cell % G.nc[2];
  c[1] = (cell / G.nc[2]) % G.nc[1];
  c[0] = cell / (G.nc[1] * G.nc[2]);
}

// visit every candidate (j, S) of receiver i; `f(j, Sx, Sy, Sz)` is called by
// the thread that owns the candidate (threads stride over each cell's atoms).
template <typename F>
__device__ __forceinline__ void for_candidates(int i, const Grid& G, const Ws& w, int lane, int nlanes, F&& f) {
  int ci[3];
  cell_coords(w.cell_of[i], G, ci);
  const int wi0 = w.wrap[3 * i + 0], wi1 = w.wrap[3 * i + 1], wi2 = w.wrap[3 * i + 2];
  for (int dx = -G.s[0]; dx <= G.s[0]; ++dx) {
    const int ux = ci[0] + dx;
    const int Tx = (int)floor((double)ux / G.nc[0]);
    const int cx = ux - Tx * G.nc[0];
    for (int dy = -G.s[1]; dy <= G.s[1]; ++dy) {
      const int uy = ci[1] + dy;
      const int Ty = (int)floor((double)uy / G.nc[1]);
      const int cy = uy - Ty * G.nc[1];
      for (int dz = -G.s[2]; dz <= G.s[2]; ++dz) {
        const int uz = ci[2] + dz;
        const int Tz = (int)floor((double)uz / G.nc[2]);
        const int cz = uz - Tz * G.nc[2];
        const int cell = (cx * G.nc[1] + cy) * G.nc[2] + cz;
        const int b = w.cell_start[cell], e = w.cell_start[cell + 1];
        for (int k = b + lane; k < e; k += nlanes) {
          const int j = w.cell_atoms[k];
          // shift in the frame of the raw (unwrapped) positions
          f(j, Tx - w.wrap[3 * j + 0] + wi0, Ty - w.wrap[3 * j + 1] + wi1, Tz - w.wrap[3 * j + 2] + wi2);
        }
      }
    }
  }
}

__global__ void k_count(const double* __restrict__ pos, int n, Grid G, Ws w) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n) return;
  const int i = warp;
  int cnt = 0;
  bool far = false;
  for_candidates(i, G, w, lane, 32, [&](int j, int Sx, int Sy, int Sz) {
    double rx, ry, rz;
    if (within(pos, i, j, Sx, Sy, Sz, G, rx, ry, rz)) {
      ++cnt;
      far |= Sx < -MAX_SHIFT || Sx > MAX_SHIFT || Sy < -MAX_SHIFT || Sy > MAX_SHIFT || Sz < -MAX_SHIFT || Sz > MAX_SHIFT;
    }
  });
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  far = __any_sync(0xffffffffu, far);
  if (lane == 0) {
    w.deg[i] = cnt;
    if (cnt > MAX_CAND) atomicExch(&w.flags[1], 1);   // more edges than the per-receiver sort holds
    if (far) atomicExch(&w.flags[2], 1);              // an image shift the edge key cannot hold
  }
}

__device__ __forceinline__ unsigned long long edge_key(int j, int Sx, int Sy, int Sz) {
  return ((unsigned long long)(unsigned)j << 24) | ((unsigned long long)((Sx + 128) & 255) << 16) |
         ((unsigned long long)((Sy + 128) & 255) << 8) | (unsigned long long)((Sz + 128) & 255);
}

__global__ void __launch_bounds__(EMIT_THREADS) k_emit(const double* __restrict__ pos, int n, Grid G, Ws w,
                                                      const int* __restrict__ off, emp_graph g) {
  __shared__ unsigned long long keys[MAX_CAND];
  __shared__ int cnt;
  const int i = blockIdx.x;
  const int deg = w.deg[i];
  if (deg > MAX_CAND) {
    if (threadIdx.x == 0) set_device_error(DEV_ERR_DEGREE);
    return;
  }
  if (threadIdx.x == 0) cnt = 0;
  __syncthreads();
  for_candidates(i, G, w, threadIdx.x, blockDim.x, [&](int j, int Sx, int Sy, int Sz) {
    double rx, ry, rz;
    if (within(pos, i, j, Sx, Sy, Sz, G, rx, ry, rz)) {
      const int k = atomicAdd(&cnt, 1);
      if (k < MAX_CAND) keys[k] = edge_key(j, Sx, Sy, Sz);
    }
  });
  __syncthreads();
  if (cnt != deg) {
    if (threadIdx.x == 0) set_device_error(DEV_ERR_INDEX);
    return;
  }
  // bitonic sort of the (unique) keys, padded to a power of two
  int P = 1;
  while (P < deg) P <<= 1;
  for (int k = deg + threadIdx.x; k < P; k += blockDim.x) keys[k] = ~0ull;
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
  const int base = off[i];
  for (int k = threadIdx.x; k < deg; k += blockDim.x) {
    const unsigned long long key = keys[k];
    const int j = (int)(key >> 24);
    const int Sx = (int)((key >> 16) & 255) - 128;
    const int Sy = (int)((key >> 8) & 255) - 128;
    const int Sz = (int)(key & 255) - 128;
    double rx, ry, rz;
    within(pos, i, j, Sx, Sy, Sz, G, rx, ry, rz);
    const int e = base + k;
    g.recv[e] = i;
    g.send[e] = j;
    g.shift[3 * e + 0] = Sx;
    g.shift[3 * e + 1] = Sy;
    g.shift[3 * e + 2] = Sz;
    g.vec[3 * e + 0] = __double2float_rn(rx);
    g.vec[3 * e + 1] = __double2float_rn(ry);
    g.vec[3 * e + 2] = __double2float_rn(rz);
  }
  if (threadIdx.x == 0) g.recv_off[i] = base;
  if (i == n - 1 && threadIdx.x == 0) g.recv_off[n] = base + deg;
}

// mirror[e] = index of (j, i, -S): binary search in receiver j's sorted segment
__global__ void k_mirror(long long E, int n, emp_graph g) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int i = g.recv[e], j = g.send[e];
  if (j < 0 || j >= n) { set_device_error(DEV_ERR_INDEX); return; }
  const unsigned long long want = edge_key(i, -g.shift[3 * e], -g.shift[3 * e + 1], -g.shift[3 * e + 2]);
  int lo = g.recv_off[j], hi = g.recv_off[j + 1] - 1;
  int found = -1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const unsigned long long k = edge_key(g.send[mid], g.shift[3 * mid], g.shift[3 * mid + 1], g.shift[3 * mid + 2]);
    if (k == want) { found = mid; break; }
    if (k < want) lo = mid + 1; else hi = mid - 1;
  }
  if (found < 0) set_device_error(DEV_ERR_MIRROR);
  g.mirror[e] = found < 0 ? (int)e : found;
}

// ------------------------------------------------------------------ skin reuse
// Edge vectors of an existing graph at new positions (same (i, j, S) topology, the same
// operations as the build: r = (x_j - x_i) + S L per component in double, rounded to float)
__global__ void k_refresh(long long E, const double* __restrict__ pos, const double* __restrict__ L, emp_graph g) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const int i = g.recv[e], j = g.send[e];
#pragma unroll
  for (int d = 0; d < 3; ++d) {
    const double r = __dadd_rn(__dsub_rn(pos[3 * j + d], pos[3 * i + d]), __dmul_rn((double)g.shift[3 * e + d], L[d]));
    g.vec[3 * e + d] = __double2float_rn(r);
  }
}

// largest squared displacement |x_i - x_ref_i|^2 over the atoms (one block; fixed tree)
__global__ void k_max_disp2(int n, const double* __restrict__ pos, const double* __restrict__ ref, double* __restrict__ out) {
  __shared__ double m[256];
  double v = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    double s = 0.0;
    for (int d = 0; d < 3; ++d) {
      const double q = pos[3 * i + d] - ref[3 * i + d];
      s += q * q;
    }
    v = fmax(v, s);
  }
  m[threadIdx.x] = v;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) m[threadIdx.x] = fmax(m[threadIdx.x], m[threadIdx.x + w]);
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = m[0];
}

}  // namespace nl
}  // namespace emp
