// C-ABI entry points of the equivariant edge message-passing library.
// One translation unit: the kernel headers are included here.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>
#include <algorithm>

#include "emp_common.cuh"

#include "nl.cuh"
#include "model.cuh"
#include "conv.cuh"
#include "so2_tc.cuh"
#include "chain.cuh"
#include "chain_tc.cuh"
#include "end_layers.cuh"
#include "tables.cuh"
#include "radial_tc.cuh"

using namespace emp;

#include <map>
#include <string>
#include <mutex>

namespace {

// ------------------------------------------------------------------ launch counting and event timing
// Every kernel launch is counted.  When profiling is on, a pair of CUDA events
// is recorded on the launching stream around each launch of a named kernel
// family, so a benchmark can read the device time of each family.
struct Prof {
  std::mutex mu;
  bool on = false;
  long long launches = 0;
  std::map<std::string, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>> ev;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void clear() {
    for (auto& kv : ev)
      for (auto& pr : kv.second) { pool.push_back(pr.first); pool.push_back(pr.second); }
    ev.clear();
  }
} g_prof;

struct Scope {
  const char* name;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  Scope(const char* n, cudaStream_t st, int count = 1) : name(n), s(st) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    g_prof.launches += count;
    if (g_prof.on) {
      a = g_prof.get();
      cudaEventRecord(a, s);
    }
  }
  ~Scope() {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    cudaEvent_t b = g_prof.get();
    cudaEventRecord(b, s);
    g_prof.ev[name].push_back({a, b});
  }
};

inline size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------------ workspace layout
struct WsLayout {
  size_t gxP2, D, dist, R, rbP, nodeZ, nodeX, zro, dB, tnp, silu, radrows, trT, trTmp, trPad, gxP, XT2, XTlo2, Y2, gRhi, gRlo, h2hi, h2lo, gh2, pperm, pinv, poff, g_r, xs, aggs, gx0, gx1, gS, e_atom, XT, Y, GXT, XTlo, GYhi, GYlo, perm, seg, nseg, vir, counter;
  size_t Ykeep = 0;          // y of every per-edge layer, kept from the forward (keep_y)
  bool keep_y = false;
  size_t total;
};

// partial sums of the weight-gradient reductions (k_tn): room for the largest splits used
constexpr int TN_SPLITS = 296;     // row splits of a reduction: up to two blocks per SM when it has few output tiles
inline size_t tn_part_floats(int C) { return std::max((size_t)16 * 36 * C * C, (size_t)TN_SPLITS * 4 * C * 64); }

// keep_y: the layers between the first and the last keep their per-edge mixing outputs y
// [E][16C] from the forward for the backward (one product fewer per cohort there, and no x~ in
// the backward prep); without it the backward recomputes y from x~ cohort by cohort.
WsLayout ws_layout(const Model& m, long long E, int N, bool grad = false, bool keep_y = false) {
  WsLayout L{};
  L.keep_y = keep_y;
  const size_t C = m.spec.C, T = m.spec.n_layers;
  const size_t coh = std::min<long long>(m.spec.cohort_edges, std::max<long long>(E, 1));
  const size_t ncoh = E > 0 ? (E + m.spec.cohort_edges - 1) / m.spec.cohort_edges : 0;
  const size_t feat = (size_t)N * 16 * C * 4;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t r = o; o = align_up(o + bytes); return r; };
  L.D = take((size_t)E * NDBLK * 4);
  L.dist = take((size_t)E * 4);
  // radial scales kept for the backward: the first layer's degree-0 columns (rows of C), then
  // rows of 4C for every later layer (a single layer of mp_forward takes rows of 4C at the start)
  L.R = take(std::max((size_t)E * C + (T - 1) * (size_t)E * 4 * C, (size_t)E * 4 * C) * 4);
  L.rbP = take(((2 * coh + RB_CHUNK - 1) / RB_CHUNK) * 2 * 16 * C * 4);   // chunk partials of two cohorts
  L.gRhi = take((size_t)E * 4 * C * 4);
  L.gRlo = take((size_t)E * 4 * C * 4);
  if (grad || m.tab_on) {   // per-row radial hidden values: only the tables' path and the weight gradients
    L.h2hi = take((size_t)E * 64 * 4);
    L.h2lo = take((size_t)E * 64 * 4);
    L.gh2 = take((size_t)E * 64 * 4);
  }
  L.pperm = take((size_t)E * 4);
  L.pinv = take((size_t)E * 4);
  L.poff = take(64 * 4);
  L.g_r = take((size_t)E * 3 * 4);
  L.xs = take((T + 1) * feat);
  L.aggs = take(T * feat);
  L.gx0 = take(feat);
  L.gx1 = take(feat);
  L.gS = take(feat);
  L.nodeZ = take(feat);
  L.nodeX = take((size_t)N * 4 * C * 4);
  L.zro = take((size_t)N * std::max(m.Hro, 1) * 4);
  L.e_atom = take((size_t)N * 4);
  const size_t cb = coh * 16 * C * 4;
  L.gxP = take(cb);
  L.gxP2 = take(cb);        // run pieces of every other cohort (the backward's sender sums)
  // the per-edge product operands and results hold two cohorts (one product launch per pair of
  // cohorts); the second cohort's rows start one cohort in (XT2, XTlo2, Y2)
  L.XT = take(2 * cb);
  L.XT2 = L.XT + cb;
  L.XTlo = take(2 * cb);
  L.XTlo2 = L.XTlo + cb;
  if (!keep_y) {
    L.Y = take(2 * cb);
    L.Y2 = L.Y + cb;
  }
  L.GXT = take(2 * cb);
  L.GYhi = take(2 * cb);
  L.GYlo = take(2 * cb);
  L.perm = take((size_t)E * 4);
  L.seg = take((size_t)E * 4);
  L.nseg = take(ncoh * 4 + 4);
  L.vir = take(VIR_BLOCKS * 9 * 8);
  L.counter = take(64);
  if (grad) {               // weight gradients: stacked SO(2) block sums, reduction partials, SiLU of the
    L.dB = take((size_t)WLAYER_CC * C * C * 4);          // readout, per-row radial values
    L.tnp = take(tn_part_floats((int)C) * 4);
    L.silu = take((size_t)N * std::max(m.Hro, 1) * 4);
    L.radrows = take((size_t)E * RAD_ROW_FLOATS * 4);
    // the SO(2) block sums on the tensor cores: a cohort pair's g_y and x~ (hi, lo) transposed to
    // [16C][rows padded to 32], and one block's product before it is added to dB
    L.trPad = (2 * coh + 31) / 32 * 32;
    L.trT = take(4 * (size_t)16 * C * L.trPad * 4);
    L.trTmp = take((size_t)tc::MAXSUB * 6 * C * 6 * C * 4);
  }
  if (keep_y && T > 2) L.Ykeep = take((T - 2) * (size_t)E * 16 * C * 4);
  L.total = o;
  return L;
}

// The layout an energy call runs with: y kept from the forward when the workspace (less `extra`
// bytes the call places after the layout) holds it, else recomputed in the backward.
WsLayout call_layout(const Model& m, long long E, int N, bool grad, size_t ws_bytes, size_t extra) {
  WsLayout L = ws_layout(m, E, N, grad, true);
  if (ws_bytes >= L.total + extra) return L;
  return ws_layout(m, E, N, grad, false);
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

// the edge arrays may be null when there are no edges (an empty tensor has no storage)
bool graph_ok(const emp_graph* g) {
  return g && g->recv_off && g->n_edges >= 0 && g->n_edges < (1ll << 31) &&
         (g->n_edges == 0 || (g->recv && g->send && g->mirror && g->vec));
}

tab::Args table_args(const Model& m, int t, int fixed_pair = -1) {
  tab::Args a;
  a.hdr = m.tab_hdr;
  a.map = m.tab_map;
  a.pieces = m.tab_pieces;
  a.layer = t;
  a.n_pairs = m.n_pairs;
  a.n_species = m.spec.n_species;
  a.pair_radial = m.spec.pair_radial;
  a.fixed_pair = fixed_pair;
  a.rc = m.spec.cutoff;
  return a;
}

RadialArgs radial_args(const Model& m, int t) {
  RadialArgs a;
  a.rad = m.rad;
  a.pair_stride = m.rad_stride();
  a.layer_off = (size_t)t * m.n_pairs * a.pair_stride;
  a.C = m.spec.C;
  a.n_species = m.spec.n_species;
  a.pair_radial = m.spec.pair_radial;
  a.rc = m.spec.cutoff;
  return a;
}


int grid_for(long long n, int per, int cap = 148 * 32) {
  long long g = (n + per - 1) / per;
  return (int)std::max<long long>(1, std::min<long long>(g, cap));
}

// SO(2) block products of a cohort on the tensor cores (3xTF32, operands pre-split):
// one operand set (forward; backward transpose) or two sharing the rows (backward: recompute + transpose)
int so2_product(const Model& m, long long M, const So2Part* parts, int nparts, int* counter, cudaStream_t s) {
  Scope sc_("so2_tc", s);
  return so2_tc(M, m.spec.C, parts, nparts, counter, s);
}

// per-node FP32 products (end_layers.cuh: k_node_gemm), up to NG_MAX in one launch
struct NodeProducts {
  NodeGemm p{};
  int max_rows = 0;
  NodeProducts(int K, int Nn) { p.K = K; p.Nn = Nn; }
  void add(int rows, int w, const float* A, long long a_node, int a_comp, const float* B, int ldb, float* out,
           long long o_node, int o_comp) {
    const int z = p.n++;
    p.rows[z] = rows; p.w[z] = w; p.A[z] = A; p.a_node[z] = a_node; p.a_comp[z] = a_comp;
    p.B[z] = B; p.ldb[z] = ldb; p.out[z] = out; p.o_node[z] = o_node; p.o_comp[z] = o_comp;
    max_rows = std::max(max_rows, rows);
  }
  void launch(cudaStream_t s, const char* name = "node_gemm") {
    if (p.n == 0 || max_rows <= 0) return;
    const dim3 grid((unsigned)((max_rows + NG_T - 1) / NG_T), (unsigned)((p.Nn + NG_T - 1) / NG_T), (unsigned)p.n);
    Scope sc_(name, s);
    k_node_gemm<<<grid, 256, 0, s>>>(p);
  }
};

// weight-gradient reduction over rows (end_layers.cuh: k_tn, k_tn_reduce): out (+)= sum_r A(r) (x) B(r)
void tn_sum(int Na, int Nb, int rows, int w, const float* A, const float* A2, long long a_node, int a_comp,
            const float* B, const float* B2, long long b_node, int b_comp, float* out, int ldo, bool accumulate,
            float* part, size_t part_floats, cudaStream_t s) {
  int splits = 0, rps = NG_K;
  if (rows > 0) {
    // enough blocks for two per SM, each split at least 256 rows, within the partials' room
    const int tiles = ((Na + TN_T - 1) / TN_T) * ((Nb + TN_T - 1) / TN_T);
    splits = std::min(TN_SPLITS, std::max(1, (2 * tc::num_sms() + tiles - 1) / tiles));
    splits = std::min(splits, std::max(1, rows / 256));
    while (splits > 1 && (size_t)splits * Na * Nb > part_floats) --splits;
    rps = (rows + splits - 1) / splits;
    rps = (rps + TN_K - 1) / TN_K * TN_K;
    splits = (rows + rps - 1) / rps;
    TnArgs a{rows, w, Na, Nb, rps, A, A2, a_node, a_comp, B, B2, b_node, b_comp, part};
    Scope sc_("weight_grad", s);
    k_tn<<<dim3((unsigned)((Na + TN_T - 1) / TN_T), (unsigned)((Nb + TN_T - 1) / TN_T), (unsigned)splits), 256, 0, s>>>(a);
  }
  Scope sc_("weight_grad", s);
  k_tn_reduce<<<(unsigned)((Na * Nb + 255) / 256), 256, 0, s>>>(splits, Na, Nb, part, out, ldo, accumulate ? 1 : 0);
}

// dst[c][r] = src[r][c] for r < rows (dst rows ld_dst floats apart), 0 for rows <= r < ld_dst:
// 32 x 32 tiles through shared memory
__global__ void k_transpose_pad(const float* __restrict__ src, int rows, int cols, long long ld_src,
                                float* __restrict__ dst, int ld_dst) {
  __shared__ float tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int r = r0 + k, c = c0 + threadIdx.x;
    tile[k][threadIdx.x] = (r < rows && c < cols) ? src[(size_t)r * ld_src + c] : 0.f;
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int c = c0 + k, r = r0 + threadIdx.x;
    if (c < cols && r < ld_dst) dst[(size_t)c * ld_dst + r] = tile[threadIdx.x][k];
  }
}

// dB_b += sum over the rows of a cohort pair of g_y (x) x~ for the four SO(2) blocks, as 3xTF32
// products on the tensor cores: the hi and lo rows transposed (the row index becomes K, padded with
// zero rows to a multiple of 32).  Per block the rows are cut into up to eight K-chunks, one
// product each (a sub-problem of one launch: eight times the output tiles, and each accumulator
// sums at most a few thousand rows in tensor memory); the chunks' products are then added to dB
// in FP32, in chunk order.
int so2_block_sums(int C, long long M, const float* GYhi, const float* GYlo, const float* XThi, const float* XTlo,
                   float* dB, void* ws, const WsLayout& L, int* counter, cudaStream_t s) {
  const int pad = (int)((M + 31) / 32 * 32);
  if (pad > (int)L.trPad) return EMP_ERR_ARG;
  float* T = at<float>(ws, L.trT);
  const size_t plane = (size_t)16 * C * L.trPad;
  const float* src[4] = {GYhi, GYlo, XThi, XTlo};
  {
    Scope sc_("wgrad_blocks", s);
    const dim3 grid((unsigned)((16 * C + 31) / 32), (unsigned)(pad / 32));
    for (int q = 0; q < 4; ++q)
      k_transpose_pad<<<grid, dim3(32, 8), 0, s>>>(src[q], (int)M, 16 * C, 16ll * C, T + q * plane, (int)L.trPad);
  }
  const int csz = ((pad + tc::MAXSUB - 1) / tc::MAXSUB + 31) / 32 * 32;   // rows per K-chunk
  const int nch = (pad + csz - 1) / csz;
  float* tmp = at<float>(ws, L.trTmp);
  for (int b = 0; b < 4; ++b) {
    const int K = blk_width(b) * C, o = blk_off(b) * C;
    MapPair a, bm[tc::MAXSUB];
    int st = make_pair128(&a, T + (size_t)o * L.trPad, T + plane + (size_t)o * L.trPad, K, pad, (int)L.trPad, tc::BM);
    if (st != EMP_OK) return st;
    GemmSub subs[tc::MAXSUB];
    for (int c = 0; c < nch; ++c) {
      const int k0 = c * csz, kn = std::min(csz, pad - k0);
      st = make_pair128(&bm[c], T + 2 * plane + (size_t)o * L.trPad + k0, T + 3 * plane + (size_t)o * L.trPad + k0, K,
                        kn, (int)L.trPad, tc::b_box_rows(K));
      if (st != EMP_OK) return st;
      subs[c] = GemmSub{&a.hi, &a.lo, &bm[c].hi, &bm[c].lo, k0, kn, K, 0, tmp + (size_t)c * K * K};
    }
    {
      Scope sc_("wgrad_blocks", s);
      st = tc_group(K, K, subs, nch, counter, s);
    }
    if (st != EMP_OK) return st;
    Scope sc_("wgrad_blocks", s);
    k_tn_reduce<<<(unsigned)((K * K + 255) / 256), 256, 0, s>>>(nch, K, K, tmp, dB + (size_t)wblk_off(b) * C * C, K, 1);
  }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

// float offsets of each weight in the blob order (include/emp.h: mp_weight_count)
struct BlobOffsets {
  std::vector<size_t> rad, so2;     // rad[t * n_pairs + p] (W1, then W2, then W3), so2[t] (W0, Wr1, Wi1, ...)
  size_t ro_W = 0, ro_w = 0;
};
BlobOffsets blob_offsets(const Model& m) {
  BlobOffsets b;
  const size_t C = m.spec.C;
  size_t o = (size_t)m.spec.n_species * C;
  for (int t = 0; t < m.spec.n_layers; ++t) {
    for (int p = 0; p < m.n_pairs; ++p) {
      b.rad.push_back(o);
      o += m.rad_stride();
    }
    b.so2.push_back(o);
    o += (size_t)(16 + 2 * (9 + 4 + 1)) * C * C;
  }
  b.ro_W = o;
  b.ro_w = o + (size_t)m.Hro * C;
  return b;
}

// tensor maps of a cohort buffer pair (rows of 16C) for the full cohort size and for the last (short) cohort
struct CohortMaps {
  So2AMaps full, tail;
  long long coh = 0, tail_rows = 0;
  int build(int C, long long E, long long cohort, const float* hi, const float* lo) {
    coh = std::min(E, cohort);
    tail_rows = E % cohort;
    if (coh > 0) {
      const int st = make_pair128(&full, hi, lo, coh, 16 * C, 16 * C, tc::BM);
      if (st != EMP_OK) return st;
    }
    if (tail_rows > 0 && tail_rows != coh) return make_pair128(&tail, hi, lo, tail_rows, 16 * C, 16 * C, tc::BM);
    return EMP_OK;
  }
  const So2AMaps* get(long long rows) const { return rows == coh ? &full : &tail; }
};

void split(const float* a, float* hi, float* lo, size_t n, cudaStream_t s) {
  { Scope sc_("split", s); k_split_tf32<<<grid_for((long long)n, 256, 148 * 16), 256, 0, s>>>(a, hi, lo, n); }
}

// A second stream per device and host thread for the short, latency-bound combine
// kernels: each runs beside the next cohort's leading kernels and is joined back
// before the first kernel that reads what it writes (or rewrites what it reads).  The
// stream and its two events are created on the first call of the thread that is not
// being captured; until then (and if creation fails) the combines run on the caller's
// stream.  They are per thread so that calls from different host threads never share
// an event; calls of one thread on different streams share the second stream, which
// orders their combines but adds no other dependency.
struct Side {
  cudaStream_t aux = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr, join2 = nullptr;
  bool pending = false;       // a combine was issued on aux and not yet joined
  int issued = 0;             // combines issued through this Side
  cudaStream_t s = nullptr;
  // run the launch f on aux after everything issued on s so far
  template <typename F>
  void run(F f) {
    if (!aux) { f(s); return; }
    cudaEventRecord(fork, s);
    cudaStreamWaitEvent(aux, fork, 0);
    f(aux);
    cudaEventRecord(issued & 1 ? join2 : join, aux);
    ++issued;
    pending = true;
  }
  // make s wait for the last combine
  void wait() {
    if (aux && pending) cudaStreamWaitEvent(s, (issued - 1) & 1 ? join2 : join, 0);
    pending = false;
  }
  // make s wait for the combine before the last (for buffers used every other combine)
  void wait_second_last() {
    if (aux && issued >= 2) cudaStreamWaitEvent(s, issued & 1 ? join2 : join, 0);
  }
};
thread_local Side g_side[64];

Side side_for(cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  Side out;
  out.s = s;
  if (dev < 0 || dev >= 64) return out;
  Side& d = g_side[dev];
  if (!d.aux) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return out;
    cudaStream_t a = nullptr;
    cudaEvent_t f = nullptr, j = nullptr, j2 = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) { cudaGetLastError(); return out; }
    if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j2, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return out;
    }
    d.aux = a;
    d.fork = f;
    d.join = j;
    d.join2 = j2;
  }
  out.aux = d.aux;
  out.fork = d.fork;
  out.join = d.join;
  out.join2 = d.join2;
  return out;
}

// [per-edge product launches: begin] (bench.py ties the mixing's DRAM traffic figure to this text)
// forward of layer t over all cohorts: S (raw receiver sums) from x (all degrees)
// Ykeep: where y of all E edges goes (rows in edge order, kept for the backward), or null (the
// cohort buffers)
int layer_forward(const Model& m, const emp_graph* g, int t, const float* x, const float* D, const float* R, const int* rrow,
                  float* S, void* ws, const WsLayout& L, cudaStream_t s, float* Ykeep = nullptr) {
  const int C = m.spec.C;
  const long long E = g->n_edges, coh = m.spec.cohort_edges;
  float* XT[2] = {at<float>(ws, L.XT), at<float>(ws, L.XT2)};
  float* XTlo[2] = {at<float>(ws, L.XTlo), at<float>(ws, L.XTlo2)};
  float* Y[2] = {at<float>(ws, L.Y), at<float>(ws, L.Y2)};
  float* P = at<float>(ws, L.rbP);
  Side side = side_for(s);
  CohortMaps am[2];
  for (int b = 0; b < 2; ++b) {
    const int st0 = am[b].build(C, E, coh, XT[b], XTlo[b]);
    if (st0 != EMP_OK) return st0;
  }
  int* counter = at<int>(ws, L.counter);
  // Full cohorts are taken two at a time (a shorter last cohort alone): both are rotated in
  // by one launch, one grouped launch computes both cohorts' products (twice the tiles, so the
  // CTA pairs stay evenly loaded), and one launch takes the receiver sums of both.
  for (long long e0 = 0; e0 < E;) {
    const long long e1 = std::min(E, e0 + coh);
    const bool two = e1 < E && std::min(E, e1 + coh) - e1 == e1 - e0;
    const long long ee[3] = {e0, e1, two ? e1 + (e1 - e0) : e1};
    const int nc = two ? 2 : 1;
    const long long M = e1 - e0;
    if (Ykeep)
      for (int b = 0; b < nc; ++b) Y[b] = Ykeep + (size_t)ee[b] * 16 * C;
    {
      // rotate-in of the group's cohorts in one launch: the second cohort's x~ rows follow the
      // first's (a pair is two full cohorts, and its buffers are contiguous)
      const long long Mt = ee[nc] - ee[0];
      const int per = rs_per(Mt, tc::num_sms(), 6);
      Scope sc_("rotate_in", s);
      k_rotate_staged<false, RS_V_FWD><<<(unsigned)((Mt + per - 1) / per), C / RS_V_FWD, rs_smem_bytes(C, false), s>>>(
          ee[0], ee[nc], C, per, g->recv, g->send, rrow, D, R, x, nullptr, XT[0], XTlo[0], nullptr, nullptr);
    }
    So2Part parts[2] = {{am[0].get(M), &m.bmaps_fwd[t], Y[0]}, {am[1].get(M), &m.bmaps_fwd[t], Y[1]}};
    const int st = so2_product(m, M, parts, nc, counter, s);
    if (st != EMP_OK) return st;
    {
      // the receiver sums of the group's cohorts in one launch: their y rows are contiguous (a
      // pair is two full cohorts), and chunk partials fold in chunk order across the cohort
      // boundary as they would cohort by cohort
      const long long c0 = ee[0], c1 = ee[nc];
      const int nchunks = (int)((c1 - c0 + RB_CHUNK - 1) / RB_CHUNK);
      side.wait();        // the previous group's combine: S of its last receiver, and P
      { Scope sc_("rotate_back_scatter", s); k_rb_chunks<RB_V><<<nchunks, C / RB_V, 0, s>>>(c0, c1, C, g->recv, g->recv_off, D, Y[0], S, P); }
      side.run([&](cudaStream_t q) {
        Scope sc_("rb_combine", q);
        k_rb_combine<<<dim3((unsigned)std::min<long long>(c1 - c0, 128), 16), C, 0, q>>>(c0, c1, C, g->recv, g->recv_off, P, S);
      });
    }
    e0 = ee[2];
  }
  side.wait();
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}
// [per-edge product launches: end]

// Rows of the radial network: edge order for one radial network, pair-sorted for
// per-pair networks (stable counting sort on the device; the pair offsets stay there, and the
// radial products take their row ranges from them).  host_offsets: also read the offsets back
// (the weight-gradient sums need them on the host; this synchronises).
struct RadialRows {
  const int* perm = nullptr;   // row -> edge (null: identity)
  const int* inv = nullptr;    // edge -> row
  const int* off_dev = nullptr;// [n_pairs + 1] first row of each pair (device; null for one network)
  std::vector<int> off;        // the same on the host, when asked for (one network: {0, E})
};

int radial_rows(const Model& m, const emp_graph* g, const int* species, void* ws, const WsLayout& L,
                RadialRows& rr, cudaStream_t s, bool host_offsets = false) {
  const long long E = g->n_edges;
  rr.off.assign(m.n_pairs + 1, 0);
  if (!m.spec.pair_radial) {
    rr.off[1] = (int)E;
    return EMP_OK;
  }
  int* perm = at<int>(ws, L.pperm);
  int* inv = at<int>(ws, L.pinv);
  int* off = at<int>(ws, L.poff);
  { Scope sc_("pair_sort", s); k_pair_sort<<<1, PS_THREADS, (size_t)m.n_pairs * PS_THREADS * 4, s>>>(
        E, m.spec.n_species, m.n_pairs, g->recv, g->send, species, perm, inv, off); }
  if (host_offsets) {
    EMP_CUDA_TRY(cudaMemcpyAsync(rr.off.data(), off, (m.n_pairs + 1) * sizeof(int), cudaMemcpyDeviceToHost, s));
    EMP_CUDA_TRY(cudaStreamSynchronize(s));
  }
  rr.perm = perm;
  rr.inv = inv;
  rr.off_dev = off;
  return EMP_OK;
}

// R rows [E][4C] of layer t: hidden layers on SIMT, head R = h2 W3^T on the tensor cores
// ncols: 4C, or C when only the degree-0 scales are used (the first layer: degree-0 input);
// R rows are ncols floats apart
// use_tables: the radial hidden layers from the certified tables (when the model has them);
// h2_only: stop after the hidden layers (h2 hi/lo in the workspace), no head product
int radial_forward(const Model& m, const emp_graph* g, int t, const int* species, const float* dist, float* R,
                   const RadialRows& rr, void* ws, const WsLayout& L, cudaStream_t s, int ncols, bool use_tables = true,
                   bool h2_only = false) {
  const long long E = g->n_edges;
  const int C = m.spec.C;
  float* h2hi = at<float>(ws, L.h2hi);
  float* h2lo = at<float>(ws, L.h2lo);
  if (!(m.tab_on && use_tables) && !h2_only) {
    // the network itself: basis, hidden layers and head in one kernel (h2 stays on chip)
    const MapPair* bm[tc::MAXSUB];
    for (int p = 0; p < m.n_pairs; ++p) bm[p] = &(ncols == C ? m.w3fn_maps : m.w3f_maps)[(size_t)t * m.n_pairs + p];
    const RadialArgs ra = radial_args(m, t);
    Scope sc_("radial_fwd", s);
    return rtc::radial_fwd(E, ncols, rr.off_dev, m.n_pairs, rr.perm, dist, ra.rad, ra.layer_off, ra.pair_stride, ra.rc,
                           bm, R, at<int>(ws, L.counter), s);
  }
  if (m.tab_on && use_tables) {
    Scope sc_("radial_h2", s);
    tab::k_radial_h2_table<<<(unsigned)std::min<long long>((E + 15) / 16, 16 * tc::num_sms()), tab::TAB_THREADS, 0, s>>>(
        E, rr.perm, dist, g->recv, g->send, species, table_args(m, t), h2hi, h2lo);
  } else {
    Scope sc_("radial_h2", s);
    k_radial_h2<<<(unsigned)std::min<long long>((E + RT - 1) / RT, 3 * tc::num_sms()), RAD_THREADS, sizeof(RadialSmem), s>>>(
        E, rr.perm, dist, g->recv, g->send, species, radial_args(m, t), h2hi, h2lo);
  }
  if (h2_only) return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
  // one launch: a sub-problem per radial network over its (device) row range
  MapPair a;
  int st = make_pair128(&a, h2hi, h2lo, E, 64, 64, tc::BM);
  if (st != EMP_OK) return st;
  GemmSub subs[tc::MAXSUB];
  for (int p = 0; p < m.n_pairs; ++p) {
    const MapPair& b = (ncols == C ? m.w3n_maps : m.w3_maps)[(size_t)t * m.n_pairs + p];
    subs[p] = GemmSub{&a.hi, &a.lo, &b.hi, &b.lo, 0, 64, ncols, 0, R};
  }
  Scope sc_("radial_head", s);
  return tc_group(E, ncols, subs, m.n_pairs, at<int>(ws, L.counter), s, rr.off_dev);
}

// dE/dd of layer t from dE/dR (rows split hi/lo), added as (dE/dd) rhat to g_r: with the network, one
// kernel (head transpose, recomputed hidden layers and their backward; radial_tc.cuh); with the
// tables, dE/dh2 = dE/dR W3 on the tensor cores, then the tables' derivative
// kcols: 4C, or C when only the degree-0 scales carry a gradient (the first layer)
// rows_out (weight gradients; network only): also each row's e, h1, dE/dz1, dE/dz2 (dE/dh2 on the
// tensor cores, then k_radial_bwd without the g_r update)
int radial_backward(const Model& m, const emp_graph* g, int t, const int* species, const float* dist,
                    const RadialRows& rr, float* g_r, void* ws, const WsLayout& L, cudaStream_t s, int kcols,
                    bool use_tables = true, float* rows_out = nullptr) {
  const long long E = g->n_edges;
  const int C = m.spec.C;
  float* gRhi = at<float>(ws, L.gRhi);
  float* gRlo = at<float>(ws, L.gRlo);
  float* gh2 = at<float>(ws, L.gh2);
  if (!(m.tab_on && use_tables)) {
    // the network itself: head transpose, recomputed hidden layers and their backward in one kernel
    MapPair a;
    int st = make_pair(&a, gRhi, gRlo, E, 4 * C, 4 * C, tc::BM);
    if (st != EMP_OK) return st;
    const MapPair* bm[tc::MAXSUB];
    for (int p = 0; p < m.n_pairs; ++p) bm[p] = &m.w3t_maps[(size_t)t * m.n_pairs + p];
    const RadialArgs ra = radial_args(m, t);
    {
      Scope sc_("radial_bwd", s);
      st = rtc::radial_bwd(E, kcols, rr.off_dev, m.n_pairs, rr.perm, dist, g->vec, g_r, ra.rad, ra.layer_off,
                           ra.pair_stride, ra.rc, a, bm, at<int>(ws, L.counter), s);
    }
    if (st != EMP_OK || !rows_out) return st;
    g_r = nullptr;          // weight gradients: the per-row values below, g_r already done
  }
  {
    MapPair a;
    int st = make_pair128(&a, gRhi, gRlo, E, 4 * C, 4 * C, tc::BM);
    if (st != EMP_OK) return st;
    GemmSub subs[tc::MAXSUB];
    for (int p = 0; p < m.n_pairs; ++p) {
      const MapPair& b = m.w3t128_maps[(size_t)t * m.n_pairs + p];
      subs[p] = GemmSub{&a.hi, &a.lo, &b.hi, &b.lo, 0, kcols, 64, 0, gh2};
    }
    Scope sc_("radial_head_bwd", s);
    st = tc_group(E, 64, subs, m.n_pairs, at<int>(ws, L.counter), s, rr.off_dev);
    if (st != EMP_OK) return st;
  }
  if (m.tab_on && use_tables) {
    Scope sc_("radial_bwd", s);
    tab::k_radial_bwd_table<<<(unsigned)std::min<long long>((E + 15) / 16, 16 * tc::num_sms()), tab::TAB_THREADS, 0, s>>>(
        E, rr.perm, dist, g->vec, g->recv, g->send, species, table_args(m, t), gh2, g_r);
  } else {
    Scope sc_("radial_rows", s);
    k_radial_bwd<<<(unsigned)std::min<long long>((E + RT - 1) / RT, 2 * tc::num_sms()), RAD_THREADS, sizeof(RadialSmem), s>>>(
        E, rr.perm, dist, g->vec, g->recv, g->send, species, radial_args(m, t), gh2, g_r, rows_out);
  }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

bool g_attrs_set = false;
int ensure_attrs() {
  if (g_attrs_set) return EMP_OK;
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_radial_h2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(RadialSmem)));
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_pair_sort, cudaFuncAttributeMaxDynamicSharedMemorySize, 32 * PS_THREADS * 4));
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_radial_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(RadialSmem)));
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_cohort_sort, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 << 14));
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_bwd_edge<BE_V>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)be_smem_bytes(256)));
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_rotate_staged<false, RS_V_FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)rs_smem_bytes(256, false)));
  EMP_CUDA_TRY(cudaFuncSetAttribute(k_rotate_staged<true, RS_V_BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)rs_smem_bytes(256, true)));
  EMP_CUDA_TRY(cudaFuncSetAttribute(ctc::k_chain_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, ctc::smem_bytes(true)));
  EMP_CUDA_TRY(cudaFuncSetAttribute(ctc::k_chain_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, ctc::smem_bytes(false)));
  int st = so2_tc_init();
  if (st != EMP_OK) return st;
  st = rtc::init();
  if (st != EMP_OK) return st;
  g_attrs_set = true;
  return EMP_OK;
}

// tf32_rna against the conversion instruction over every 32-bit pattern (NaNs skipped): the count of
// patterns where they differ
__global__ void k_tf32_selftest(unsigned long long* mismatches) {
  unsigned long long bad = 0;
  for (uint64_t b = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; b < (1ull << 32);
       b += (uint64_t)gridDim.x * blockDim.x) {
    const float a = __uint_as_float((uint32_t)b);
    if (a != a) continue;
    if (__float_as_uint(tf32_rna(a)) != __float_as_uint(tf32_rna_cvt(a))) ++bad;
  }
  if (bad) atomicAdd(mismatches, bad);
}

// One bounded wait on an mbarrier that nothing arrives on: it runs out after the limit in
// force (emp_set_wait_limit), records EMP_ERR_TIMEOUT in the device error word and returns.
__global__ void k_wait_selftest() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) tc::mbar_wait(&bar, 0);
}

// (d, 0, 0): an edge vector of length d along x, and the x component of g_r back
__global__ void k_length_vec(long long n, const float* __restrict__ d, float* __restrict__ vec) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  vec[3 * i] = d[i];
  vec[3 * i + 1] = 0.f;
  vec[3 * i + 2] = 0.f;
}
__global__ void k_take_x(long long n, const float* __restrict__ g_r, float* __restrict__ out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = g_r[3 * i];
}

// recv_off of a rank's local view: its edges [eb, eb + El) re-based to 0, every other receiver's range empty
__global__ void k_local_offsets(int N, const int* __restrict__ recv_off, int eb, int El, int* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i > N) return;
  const int v = recv_off[i] - eb;
  out[i] = v < 0 ? 0 : v > El ? El : v;
}

int check_device() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EMP_ERR_UNSUPPORTED;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return EMP_ERR_UNSUPPORTED;
  return major == 10 ? EMP_OK : EMP_ERR_UNSUPPORTED;
}

}  // namespace

// ------------------------------------------------------------------ fixed scratch of nl_build_noalloc
// Held by every device that loads the library, until the process exits.  Every
// nl_build_noalloc call on a device shares it: calls whose work overlaps on the
// GPU (different streams, no ordering between them) race on it.  nl_build clears
// everything that must start at zero (cell counters, cursors, flags) at the start
// of each call, and writes every other entry before reading it.
static __device__ __align__(256) unsigned char g_nl_noalloc_scratch[EMP_NL_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, on every call: the lookup is
// cheap once the module is loaded, and an address kept from before a device reset
// would point into a context that no longer exists.
int nl_noalloc_scratch_address(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_nl_noalloc_scratch) != cudaSuccess || !ptr) return EMP_ERR_CUDA;
  *out = ptr;
  return EMP_OK;
}
}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* emp_status_string(int status) {
  switch (status) {
    case EMP_OK: return "ok";
    case EMP_ERR_ARG: return "invalid argument";
    case EMP_ERR_CAPACITY: return "graph capacity smaller than the edge count";
    case EMP_ERR_CUDA: return "CUDA runtime error";
    case EMP_ERR_TIMEOUT: return "bounded device wait timed out";
    case EMP_ERR_NONFINITE: return "non-finite positions";
    case EMP_ERR_WORKSPACE: return "workspace too small";
    case EMP_ERR_DEVICE: return "device-side check failed";
    case EMP_ERR_UNSUPPORTED: return "unsupported device or size";
    default: return "unknown status";
  }
}

int emp_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.clear();
  g_prof.on = enable != 0;
  return EMP_OK;
}

int emp_profile_read(const char* name, double* total_ms, int64_t* launches) {
  if (!name || !total_ms || !launches) return EMP_ERR_ARG;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  double ms = 0.0;
  int64_t n = 0;
  for (auto& kv : g_prof.ev) {
    if (std::strcmp(name, "*") != 0 && kv.first != name) continue;
    for (auto& pr : kv.second) {
      if (cudaEventSynchronize(pr.second) != cudaSuccess) return EMP_ERR_CUDA;
      float t = 0.f;
      if (cudaEventElapsedTime(&t, pr.first, pr.second) != cudaSuccess) return EMP_ERR_CUDA;
      ms += t;
      ++n;
    }
  }
  *total_ms = ms;
  *launches = n;
  return EMP_OK;
}

int emp_profile_names(char* buf, size_t n) {
  if (!buf || n == 0) return EMP_ERR_ARG;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  std::string all;
  for (auto& kv : g_prof.ev) { all += kv.first; all += ','; }
  std::strncpy(buf, all.c_str(), n - 1);
  buf[n - 1] = 0;
  return EMP_OK;
}

int64_t emp_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  return g_prof.launches;
}

int emp_tf32_mma_rate(int32_t iters, cudaStream_t stream, double* tflops) {
  if (!tflops || iters < 1) return EMP_ERR_ARG;
  int st = check_device();
  if (st != EMP_OK) return st;
  st = ensure_attrs();
  if (st != EMP_OK) return st;
  const int pairs = tc::num_sms() / 2;
  cudaEvent_t a = nullptr, b = nullptr;
  EMP_CUDA_TRY(cudaEventCreate(&a));
  EMP_CUDA_TRY(cudaEventCreate(&b));
  static unsigned seed = 1;
  cudaEventRecord(a, stream);
  { Scope sc_("tf32_rate", stream); tc::k_tf32_rate<<<2 * pairs, 128, tc::RATE_SMEM, stream>>>(iters, seed++); }
  cudaEventRecord(b, stream);
  const cudaError_t e1 = cudaEventSynchronize(b);
  float ms = 0.f;
  const cudaError_t e2 = cudaEventElapsedTime(&ms, a, b);
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (e1 != cudaSuccess || e2 != cudaSuccess || cudaGetLastError() != cudaSuccess) return EMP_ERR_CUDA;
  // per round: the k-steps of one 32-wide stage (four), each three M = 256, N = 256, K = 8 products per pair
  const double flops = (double)pairs * iters * (tc::BK2 / 8) * 3 * 2.0 * 256 * 256 * 8;
  *tflops = flops / (ms * 1e-3) / 1e12;
  return EMP_OK;
}

int emp_set_wait_limit(int64_t cycles) {
  const long long v = cycles > 0 ? (long long)cycles : tc::TIMEOUT_CYCLES;
  EMP_CUDA_TRY(cudaMemcpyToSymbol(tc::g_wait_cycles, &v, sizeof(v)));
  return EMP_OK;
}

int emp_wait_selftest(cudaStream_t stream) {
  int st = check_device();
  if (st != EMP_OK) return st;
  k_wait_selftest<<<1, 32, 0, stream>>>();
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

int emp_tf32_split_selftest(uint64_t* mismatches) {
  if (!mismatches) return EMP_ERR_ARG;
  int st = check_device();
  if (st != EMP_OK) return st;
  unsigned long long* d = nullptr;
  EMP_CUDA_TRY(cudaMalloc(&d, sizeof(unsigned long long)));
  cudaMemset(d, 0, sizeof(unsigned long long));
  k_tf32_selftest<<<148 * 8, 256>>>(d);
  unsigned long long h = 0;
  const cudaError_t e = cudaMemcpy(&h, d, sizeof(h), cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess) return EMP_ERR_CUDA;
  *mismatches = h;
  return EMP_OK;
}

int emp_last_device_error(void) {
  int h = 0, z = 0;
  if (cudaMemcpyFromSymbol(&h, g_device_error, sizeof(int)) != cudaSuccess) return EMP_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_error, &z, sizeof(int)) != cudaSuccess) return EMP_ERR_CUDA;
  if (h == 0) return EMP_OK;
  return h == DEV_ERR_TIMEOUT ? EMP_ERR_TIMEOUT : EMP_ERR_DEVICE;
}

// ------------------------------------------------------------------ neighbour list
size_t nl_workspace_bytes(int32_t n_atoms) {
  const size_t n = std::max(n_atoms, 1);
  return align_up(n * 4) * 7 + align_up(n * 12) + align_up(16) + align_up(8) + 4096;
}

static int nl_build_impl(const emp_nl_params* p, const double* pos, emp_graph* g, int64_t* n_edges, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  if (!p || !pos || !g || !n_edges || !ws) return EMP_ERR_ARG;
  const int N = p->n_atoms;
  if (N < 1 || !(p->cutoff > 0) || !g->recv_off) return EMP_ERR_ARG;
  for (int d = 0; d < 3; ++d)
    if (!(p->box[d] > 0) || !std::isfinite(p->box[d])) return EMP_ERR_ARG;
  if (ws_bytes < nl_workspace_bytes(N)) return EMP_ERR_WORKSPACE;
  if (p->capacity > 0 && !(g->recv && g->send && g->mirror && g->shift && g->vec)) return EMP_ERR_ARG;
  int st = check_device();
  if (st != EMP_OK) return st;
  // cell grid: cells no smaller than rc (1 + 1e-9), at most N cells
  nl::Grid G;
  const double rcp = p->cutoff * (1.0 + 1e-9);
  long long ncell = 1;
  for (int d = 0; d < 3; ++d) {
    G.L[d] = p->box[d];
    G.nc[d] = std::max(1, (int)std::floor(p->box[d] / rcp));
  }
  while ((ncell = (long long)G.nc[0] * G.nc[1] * G.nc[2]) > N) {
    int d = 0;
    for (int q = 1; q < 3; ++q)
      if (G.nc[q] > G.nc[d]) d = q;
    G.nc[d] = std::max(1, G.nc[d] / 2);
  }
  for (int d = 0; d < 3; ++d) G.s[d] = (int)std::ceil(rcp / (p->box[d] / G.nc[d]));
  G.rc2 = p->cutoff * p->cutoff;
  G.n_cells = (int)ncell;
  // workspace carve
  char* w = static_cast<char*>(ws);
  size_t o = 0;
  auto take = [&](size_t b) { char* r = w + o; o += align_up(b); return r; };
  nl::Ws W;
  W.cell_of = (int*)take(N * 4);
  W.wrap = (int*)take((size_t)N * 12);
  W.cell_count = (int*)take(N * 4);
  W.cell_start = (int*)take((size_t)(N + 1) * 4);
  W.cell_cursor = (int*)take(N * 4);
  W.cell_atoms = (int*)take(N * 4);
  W.deg = (int*)take(N * 4);
  W.flags = (int*)take(16);
  W.total = (long long*)take(8);
  EMP_CUDA_TRY(cudaMemsetAsync(W.cell_count, 0, (size_t)G.n_cells * 4, stream));
  EMP_CUDA_TRY(cudaMemsetAsync(W.cell_cursor, 0, (size_t)G.n_cells * 4, stream));
  EMP_CUDA_TRY(cudaMemsetAsync(W.flags, 0, 16, stream));
  { Scope sc_("nl", stream); nl::k_bin<<<(N + 255) / 256, 256, 0, stream>>>(pos, N, G, W); }
  { Scope sc_("nl", stream); nl::k_scan<<<1, 1024, 0, stream>>>(W.cell_count, W.cell_start, G.n_cells, nullptr); }
  { Scope sc_("nl", stream); nl::k_fill_cells<<<(N + 255) / 256, 256, 0, stream>>>(N, W); }
  { Scope sc_("nl", stream); nl::k_count<<<(N * 32 + 255) / 256, 256, 0, stream>>>(pos, N, G, W); }
  { Scope sc_("nl", stream); nl::k_scan<<<1, 1024, 0, stream>>>(W.deg, g->recv_off, N, W.total); }
  long long total = 0;
  int flags[4] = {0, 0, 0, 0};
  EMP_CUDA_TRY(cudaMemcpyAsync(&total, W.total, 8, cudaMemcpyDeviceToHost, stream));
  EMP_CUDA_TRY(cudaMemcpyAsync(flags, W.flags, 16, cudaMemcpyDeviceToHost, stream));
  EMP_CUDA_TRY(cudaStreamSynchronize(stream));
  if (flags[0]) return EMP_ERR_NONFINITE;
  *n_edges = total;
  g->n_edges = total;
  g->n_atoms = N;
  if (flags[1]) return EMP_ERR_DEVICE;         // a receiver with more than nl::MAX_CAND edges
  if (flags[2]) return EMP_ERR_UNSUPPORTED;    // an image shift beyond +-nl::MAX_SHIFT box lengths
  if (total > p->capacity) return EMP_ERR_CAPACITY;
  if (total >= (1ll << 31)) return EMP_ERR_CAPACITY;
  { Scope sc_("nl", stream); nl::k_emit<<<N, nl::EMIT_THREADS, 0, stream>>>(pos, N, G, W, g->recv_off, *g); }
  if (total > 0) { Scope sc_("nl", stream); nl::k_mirror<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(total, N, *g); }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

int nl_build(const emp_nl_params* p, const double* pos, emp_graph* g, int64_t* n_edges, void* ws,
             size_t ws_bytes, cudaStream_t stream) {
  return nl_build_impl(p, pos, g, n_edges, ws, ws_bytes, stream);
}

// Neighbour list with the library's own fixed scratch (no allocation anywhere).
// For callers that cannot allocate device memory themselves -- for example a
// plug-in inside a host program whose device memory all comes from that
// program's own pool, or a code path that must not trigger the device-wide
// synchronisation cudaMalloc/cudaFree can cause.  The scratch is the file-scope
// array g_nl_noalloc_scratch above; its device address is looked up on each call,
// with the caller's device current.
int nl_build_noalloc(const emp_nl_params* p, const double* pos, emp_graph* g, int64_t* n_edges,
                     cudaStream_t stream) {
  if (!p || !pos || !g || !n_edges) return EMP_ERR_ARG;
  if (p->n_atoms > EMP_NL_NOALLOC_MAX_ATOMS) return EMP_ERR_WORKSPACE;
  if (nl_workspace_bytes(std::max(p->n_atoms, 1)) > sizeof(g_nl_noalloc_scratch)) return EMP_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = nl_noalloc_scratch_address(&scratch);
  if (st != EMP_OK) return st;
  return nl_build_impl(p, pos, g, n_edges, scratch, sizeof(g_nl_noalloc_scratch), stream);
}

int nl_refresh(const emp_nl_params* p, const double* pos, const double* pos_ref, double skin, emp_graph* g,
               int32_t* rebuild, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!p || !pos || !pos_ref || !g || !rebuild || !ws || !(skin >= 0.0) || !graph_ok(g)) return EMP_ERR_ARG;
  if (p->n_atoms < 1 || g->n_atoms != p->n_atoms || g->n_edges > 0 && !g->shift) return EMP_ERR_ARG;
  for (int d = 0; d < 3; ++d)
    if (!(p->box[d] > 0) || !std::isfinite(p->box[d])) return EMP_ERR_ARG;
  if (ws_bytes < 64) return EMP_ERR_WORKSPACE;
  int st = check_device();
  if (st != EMP_OK) return st;
  double* L = static_cast<double*>(ws);
  double* disp2 = L + 4;
  EMP_CUDA_TRY(cudaMemcpyAsync(L, p->box, 3 * sizeof(double), cudaMemcpyHostToDevice, stream));
  if (g->n_edges > 0) {
    Scope sc_("nl", stream);
    nl::k_refresh<<<(unsigned)((g->n_edges + 255) / 256), 256, 0, stream>>>(g->n_edges, pos, L, *g);
  }
  { Scope sc_("nl", stream); nl::k_max_disp2<<<1, 256, 0, stream>>>(p->n_atoms, pos, pos_ref, disp2); }
  double h = 0.0;
  EMP_CUDA_TRY(cudaMemcpyAsync(&h, disp2, sizeof(double), cudaMemcpyDeviceToHost, stream));
  EMP_CUDA_TRY(cudaStreamSynchronize(stream));
  if (!std::isfinite(h)) return EMP_ERR_NONFINITE;
  // a pair within rc now was within rc + skin at pos_ref while no atom moved more than skin / 2
  *rebuild = 4.0 * h > skin * skin ? 1 : 0;
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

// ------------------------------------------------------------------ model
size_t mp_weight_count(const emp_model_spec* spec) { return spec ? weight_count(*spec) : 0; }

int mp_model_create(const emp_model_spec* spec, const float* weights, size_t n_floats, void** model) {
  if (!spec || !weights || !model) return EMP_ERR_ARG;
  if (!spec_ok(*spec)) return EMP_ERR_ARG;
  if (n_floats != weight_count(*spec)) return EMP_ERR_ARG;
  int st = check_device();
  if (st != EMP_OK) return st;
  st = ensure_attrs();
  if (st != EMP_OK) return st;
  Model* m = new Model();
  m->spec = *spec;
  m->H = spec->radial_hidden;
  m->Hro = spec->readout_hidden > 0 ? spec->readout_hidden : spec->C;
  m->n_pairs = spec->pair_radial ? spec->n_species * (spec->n_species + 1) / 2 : 1;
  cudaGetDevice(&m->device);
  const size_t C = spec->C, T = spec->n_layers, S = spec->n_species;
  const size_t n_emb = S * C, n_rad = T * m->n_pairs * m->rad_stride(), n_so2 = T * m->so2_stride();
  const size_t n_ro = (size_t)m->Hro * C + m->Hro;
  const size_t n_w3 = T * m->n_pairs * (size_t)4 * C * 64;
  const size_t total = n_emb + n_rad + 6 * n_so2 + 4 * n_w3 + n_ro + (size_t)m->Hro * C + n_floats;   // + raw staging
  float* base = nullptr;
  if (cudaMalloc(&base, total * 4) != cudaSuccess) { delete m; return EMP_ERR_CUDA; }
  m->base = base;
  m->emb = base;
  m->rad = m->emb + n_emb;
  m->so2_fwd = m->rad + n_rad;
  m->so2_bwd = m->so2_fwd + n_so2;
  m->so2_fwd_hi = m->so2_bwd + n_so2;
  m->so2_fwd_lo = m->so2_fwd_hi + n_so2;
  m->so2_bwd_hi = m->so2_fwd_lo + n_so2;
  m->so2_bwd_lo = m->so2_bwd_hi + n_so2;
  m->w3_hi = m->so2_bwd_lo + n_so2;
  m->w3_lo = m->w3_hi + n_w3;
  m->w3t_hi = m->w3_lo + n_w3;
  m->w3t_lo = m->w3t_hi + n_w3;
  m->ro_W = m->w3t_lo + n_w3;
  m->ro_w = m->ro_W + (size_t)m->Hro * C;
  m->ro_WT = m->ro_w + m->Hro;
  float* raw = m->ro_WT + (size_t)m->Hro * C;
  auto fail = [&](int code) { cudaFree(base); delete m; return code; };
  if (cudaMemcpy(raw, weights, n_floats * 4, cudaMemcpyHostToDevice) != cudaSuccess) return fail(EMP_ERR_CUDA);
  // walk the blob in declaration order
  size_t o = 0;
  if (cudaMemcpy(m->emb, raw + o, n_emb * 4, cudaMemcpyDeviceToDevice) != cudaSuccess) return fail(EMP_ERR_CUDA);
  o += n_emb;
  const size_t H = m->H;
  for (size_t t = 0; t < T; ++t) {
    const size_t rad_t = m->n_pairs * m->rad_stride();
    if (cudaMemcpy(m->rad + t * rad_t, raw + o, rad_t * 4, cudaMemcpyDeviceToDevice) != cudaSuccess)
      return fail(EMP_ERR_CUDA);
    m->rad_host.insert(m->rad_host.end(), weights + o, weights + o + rad_t);
    o += rad_t;
    const float* W0 = raw + o;
    o += 16 * C * C;
    const float* Wr[3];
    const float* Wi[3];
    for (int mm = 1; mm <= 3; ++mm) {
      const size_t h = (4 - mm) * C;
      Wr[mm - 1] = raw + o;
      o += h * h;
      Wi[mm - 1] = raw + o;
      o += h * h;
    }
    k_stack_so2<<<256, 256>>>(W0, Wr[0], Wi[0], Wr[1], Wi[1], Wr[2], Wi[2], (int)C, m->so2_fwd + t * m->so2_stride(),
                              m->so2_bwd + t * m->so2_stride());
  }
  (void)H;
  if (cudaMemcpy(m->ro_W, raw + o, n_ro * 4, cudaMemcpyDeviceToDevice) != cudaSuccess) return fail(EMP_ERR_CUDA);
  o += n_ro;
  if (o != n_floats) return fail(EMP_ERR_ARG);
  k_transpose<<<(int)((m->Hro * C + 255) / 256), 256>>>(m->ro_W, m->ro_WT, m->Hro, (int)C);
  k_split_tf32<<<256, 256>>>(m->so2_fwd, m->so2_fwd_hi, m->so2_fwd_lo, n_so2);
  k_split_tf32<<<256, 256>>>(m->so2_bwd, m->so2_bwd_hi, m->so2_bwd_lo, n_so2);
  // radial heads: W3 split, and W3^T split (input gradient dE/dh2 = dE/dR W3)
  for (size_t t = 0; t < T; ++t)
    for (int p = 0; p < m->n_pairs; ++p) {
      const size_t wo = (t * m->n_pairs + p) * m->w3_stride();
      const float* W3 = m->W3((int)t, p);
      float* tmpT = m->w3t_hi + wo;   // transpose lands in the hi slot, then is split in place
      k_transpose<<<(int)((m->w3_stride() + 255) / 256), 256>>>(W3, tmpT, 4 * (int)C, 64);
      k_split_tf32<<<64, 256>>>(W3, m->w3_hi + wo, m->w3_lo + wo, m->w3_stride());
      k_split_tf32<<<64, 256>>>(tmpT, m->w3t_hi + wo, m->w3t_lo + wo, m->w3_stride());
    }
  m->w3_maps.resize(T * m->n_pairs);
  m->w3n_maps.resize(T * m->n_pairs);
  m->w3f_maps.resize(T * m->n_pairs);
  m->w3fn_maps.resize(T * m->n_pairs);
  m->w3t_maps.resize(T * m->n_pairs);
  m->w3t128_maps.resize(T * m->n_pairs);
  for (size_t q = 0; q < T * m->n_pairs; ++q) {
    const size_t wo = q * m->w3_stride();
    if (make_pair128(&m->w3_maps[q], m->w3_hi + wo, m->w3_lo + wo, 4 * C, 64, 64, tc::b_box_rows(4 * (int)C)) != EMP_OK ||
        make_pair128(&m->w3n_maps[q], m->w3_hi + wo, m->w3_lo + wo, C, 64, 64, tc::b_box_rows((int)C)) != EMP_OK ||
        make_pair128(&m->w3t128_maps[q], m->w3t_hi + wo, m->w3t_lo + wo, 64, 4 * (int)C, 4 * (int)C, tc::b_box_rows(64)) !=
            EMP_OK ||
        make_pair(&m->w3f_maps[q], m->w3_hi + wo, m->w3_lo + wo, 4 * C, 64, 64, rtc::fwd_bn(4 * (int)C) / 2) != EMP_OK ||
        make_pair(&m->w3fn_maps[q], m->w3_hi + wo, m->w3_lo + wo, C, 64, 64, rtc::fwd_bn((int)C) / 2) != EMP_OK ||
        make_pair(&m->w3t_maps[q], m->w3t_hi + wo, m->w3t_lo + wo, 64, 4 * (int)C, 4 * (int)C, tc::b_box_rows(64)) !=
            EMP_OK)
      return fail(EMP_ERR_CUDA);
  }
  m->bmaps_fwd.resize(T);
  m->bmaps_bwd.resize(T);
  for (size_t t = 0; t < T; ++t) {
    const size_t off = t * m->so2_stride();
    if (so2_make_bmaps(&m->bmaps_fwd[t], (int)C, m->so2_fwd_hi + off, m->so2_fwd_lo + off) != EMP_OK ||
        so2_make_bmaps(&m->bmaps_bwd[t], (int)C, m->so2_bwd_hi + off, m->so2_bwd_lo + off) != EMP_OK)
      return fail(EMP_ERR_CUDA);
  }
  // rotation generators on the structural pairs; every other entry must vanish
  double J[3][NDBLK];
  generator_blocks(J);
  float jx[NJPAIR], jy[NJPAIR];
  double outside = 0.0;
  for (int a = 0; a < 16; ++a)
    for (int b = 0; b < 16; ++b) {
      bool listed = false;
      for (int q = 0; q < NJPAIR; ++q)
        if ((jpair_a(q) == a && jpair_b(q) == b) || (jpair_a(q) == b && jpair_b(q) == a)) listed = true;
      if (!listed) outside += std::fabs(gen_at(J[0], a, b)) + std::fabs(gen_at(J[1], a, b));
    }
  if (outside > 1e-12) return fail(EMP_ERR_DEVICE);
  for (int q = 0; q < NJPAIR; ++q) {
    jx[q] = (float)gen_at(J[0], jpair_a(q), jpair_b(q));
    jy[q] = (float)gen_at(J[1], jpair_a(q), jpair_b(q));
  }
  if (cudaMemcpyToSymbol(c_jx, jx, sizeof(jx)) != cudaSuccess) return fail(EMP_ERR_CUDA);
  if (cudaMemcpyToSymbol(c_jy, jy, sizeof(jy)) != cudaSuccess) return fail(EMP_ERR_CUDA);
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(EMP_ERR_CUDA);
  *model = m;
  return EMP_OK;
}

void mp_model_destroy(void* model) {
  if (!model) return;
  Model* m = static_cast<Model*>(model);
  if (m->tab_base) cudaFree(m->tab_base);
  cudaFree(m->base);
  delete m;
}

int mp_model_radial_tables(void* model, double tol, int32_t* n_pieces) {
  if (!model) return EMP_ERR_ARG;
  Model* m = static_cast<Model*>(model);
  if (m->tab_base) {
    cudaFree(m->tab_base);
    m->tab_base = nullptr;
  }
  m->tab_on = false;
  m->tab_hdr = m->tab_map = nullptr;
  m->tab_pieces = nullptr;
  if (n_pieces) *n_pieces = 0;
  if (!(tol > 0.0)) return EMP_OK;                  // tables off: the radial network itself
  if (!(tol >= 1e-12) || m->spec.radial_hidden != tab::H) return EMP_ERR_ARG;
  int st = check_device();
  if (st != EMP_OK) return st;
  const int T = m->spec.n_layers, P = m->n_pairs;
  std::vector<int> hdr(4 * (size_t)T * P), map;
  std::vector<float> pieces;
  for (int t = 0; t < T; ++t)
    for (int p = 0; p < P; ++p) {
      const float* W1 = m->rad_host.data() + ((size_t)t * P + p) * m->rad_stride();
      const std::vector<tab::HostPiece> tb = tab::build(W1, W1 + 64 * 8, (double)m->spec.cutoff, tol);
      int L = 0;
      for (const auto& q : tb) L = std::max(L, q.level);
      const int q = t * P + p;
      hdr[4 * q + 0] = L;
      hdr[4 * q + 1] = (int)(pieces.size() / tab::PIECE_FLOATS);
      hdr[4 * q + 2] = (int)map.size();
      hdr[4 * q + 3] = (int)tb.size();
      // every bin of the finest level lies inside exactly one (dyadic) piece
      const int nbin = 1 << L;
      size_t k = 0;
      for (int b = 0; b < nbin; ++b) {
        const double c = ((double)b + 0.5) * m->spec.cutoff / nbin;
        while (k + 1 < tb.size() && c >= tb[k].b) ++k;
        map.push_back((int)k);
      }
      for (const auto& pc : tb) {
        pieces.push_back((float)pc.a);
        pieces.push_back((float)(2.0 / (pc.b - pc.a)));
        pieces.push_back(0.f);
        pieces.push_back(0.f);
        for (double v : pc.c) pieces.push_back((float)v);
        for (double v : pc.dc) pieces.push_back((float)v);
      }
    }
  const size_t bh = align_up(hdr.size() * 4), bm = align_up(map.size() * 4), bp = pieces.size() * 4;
  char* base = nullptr;
  if (cudaMalloc(&base, bh + bm + bp) != cudaSuccess) return EMP_ERR_CUDA;
  if (cudaMemcpy(base, hdr.data(), hdr.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(base + bh, map.data(), map.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(base + bh + bm, pieces.data(), bp, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(base);
    return EMP_ERR_CUDA;
  }
  m->tab_base = base;
  m->tab_hdr = reinterpret_cast<int*>(base);
  m->tab_map = reinterpret_cast<int*>(base + bh);
  m->tab_pieces = reinterpret_cast<float*>(base + bh + bm);
  m->tab_on = true;
  if (n_pieces) *n_pieces = (int32_t)(pieces.size() / tab::PIECE_FLOATS);
  return EMP_OK;
}

int mp_radial_hidden(const void* model, int32_t layer, int32_t pair, int64_t n, const float* d, float* h2_hi,
                     float* h2_lo, const float* g_h2, float* dE_dd, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!model || n < 0 || (n > 0 && (!d || !h2_hi || !h2_lo))) return EMP_ERR_ARG;
  const Model& m = *static_cast<const Model*>(model);
  if (layer < 0 || layer >= m.spec.n_layers || pair < 0 || pair >= m.n_pairs) return EMP_ERR_ARG;
  if (g_h2 && (!dE_dd || !ws)) return EMP_ERR_ARG;
  if (n >= (1ll << 31)) return EMP_ERR_ARG;
  if (g_h2 && ws_bytes < (size_t)n * 24 + 256) return EMP_ERR_WORKSPACE;
  if (n == 0) return EMP_OK;
  int st = check_device();
  if (st != EMP_OK) return st;
  RadialArgs ra = radial_args(m, layer);
  ra.pair_radial = 0;
  ra.layer_off += (size_t)pair * ra.pair_stride;
  if (m.tab_on) {
    Scope sc_("radial_h2", stream);
    tab::k_radial_h2_table<<<(unsigned)std::min<long long>((n + 15) / 16, 16 * tc::num_sms()), tab::TAB_THREADS, 0, stream>>>(
        n, nullptr, d, nullptr, nullptr, nullptr, table_args(m, layer, pair), h2_hi, h2_lo);
  } else {
    Scope sc_("radial_h2", stream);
    k_radial_h2<<<(unsigned)std::min<long long>((n + RT - 1) / RT, 3 * tc::num_sms()), RAD_THREADS, sizeof(RadialSmem), stream>>>(
        n, nullptr, d, nullptr, nullptr, nullptr, ra, h2_hi, h2_lo);
  }
  if (g_h2) {
    float* vec = static_cast<float*>(ws);
    float* g_r = vec + 3 * n;
    { Scope sc_("radial_aux", stream); k_length_vec<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(n, d, vec); }
    EMP_CUDA_TRY(cudaMemsetAsync(g_r, 0, (size_t)n * 12, stream));
    if (m.tab_on) {
      Scope sc_("radial_bwd", stream);
      tab::k_radial_bwd_table<<<(unsigned)std::min<long long>((n + 15) / 16, 16 * tc::num_sms()), tab::TAB_THREADS, 0, stream>>>(
          n, nullptr, d, vec, nullptr, nullptr, nullptr, table_args(m, layer, pair), g_h2, g_r);
    } else {
      Scope sc_("radial_bwd", stream);
      k_radial_bwd<<<(unsigned)std::min<long long>((n + RT - 1) / RT, 2 * tc::num_sms()), RAD_THREADS, sizeof(RadialSmem), stream>>>(
          n, nullptr, d, vec, nullptr, nullptr, nullptr, ra, g_h2, g_r, nullptr);
    }
    { Scope sc_("radial_aux", stream); k_take_x<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(n, g_r, dE_dd); }
  }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

size_t mp_workspace_bytes(const void* model, int64_t n_edges, int32_t n_atoms) {
  if (!model || n_edges < 0 || n_atoms < 1) return 0;
  return ws_layout(*static_cast<const Model*>(model), n_edges, n_atoms, false, true).total;
}

size_t mp_workspace_bytes_min(const void* model, int64_t n_edges, int32_t n_atoms) {
  if (!model || n_edges < 0 || n_atoms < 1) return 0;
  return ws_layout(*static_cast<const Model*>(model), n_edges, n_atoms).total;
}


int mp_forward(const void* model, const emp_graph* g, int32_t layer, const int32_t* species, const float* x_in,
               float* agg_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!model || !graph_ok(g) || !x_in || !agg_out || !ws || g->n_atoms < 1) return EMP_ERR_ARG;
  const Model& m = *static_cast<const Model*>(model);
  if (layer < 0 || layer >= m.spec.n_layers) return EMP_ERR_ARG;
  if (m.spec.pair_radial && !species) return EMP_ERR_ARG;
  const long long E = g->n_edges;
  const int N = g->n_atoms, C = m.spec.C;
  const WsLayout L = ws_layout(m, E, N);
  if (ws_bytes < L.total) return EMP_ERR_WORKSPACE;
  int st = check_device();
  if (st != EMP_OK) return st;
  EMP_CUDA_TRY(cudaMemsetAsync(agg_out, 0, (size_t)N * 16 * C * 4, stream));
  if (E == 0) return EMP_OK;
  float* D = at<float>(ws, L.D);
  float* dist = at<float>(ws, L.dist);
  float* R = at<float>(ws, L.R);
  { Scope sc_("geometry", stream); k_geometry_staged<<<(unsigned)((E + GEO_EPB - 1) / GEO_EPB), GEO_EPB, 0, stream>>>(E, g->vec, D, dist); }
  RadialRows rr;
  st = radial_rows(m, g, species, ws, L, rr, stream);
  if (st != EMP_OK) return st;
  st = radial_forward(m, g, layer, species, dist, R, rr, ws, L, stream, 4 * C);
  if (st != EMP_OK) return st;
  st = layer_forward(m, g, layer, x_in, D, R, rr.inv, agg_out, ws, L, stream);
  if (st != EMP_OK) return st;
  const size_t n = (size_t)N * 16 * C;
  { Scope sc_("scale", stream); k_scale<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(n, 1.0f / m.spec.avg_degree, agg_out); }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

// Receiver-range sharding: this rank takes the edges of receivers [a, b); `g` is then the rank's
// local view (its edges, recv_off re-based, empty ranges outside [a, b)), `global` the whole graph.
struct Shard {
  const emp_graph* global = nullptr;
  long long e_begin = 0;
  int rank = 0;
  emp_allreduce_fn allreduce = nullptr;
  void* ctx = nullptr;
};

// Energy and forces (mp_energy_forces); with grad (mp_energy_weight_grad) also dE/dW in the blob order;
// with sh (mp_energy_forces_sharded) the part of the step of one rank.
static int energy_forces_impl(const Model& m, const emp_graph* g, const int32_t* species, double* energy, float* forces,
                              float* virial, float* atom_energy, float* grad, void* ws, size_t ws_bytes,
                              cudaStream_t stream, const Shard* sh = nullptr) {
  if ((m.spec.pair_radial || m.spec.n_species > 1) && !species) return EMP_ERR_ARG;
  const long long E = g->n_edges, coh = m.spec.cohort_edges;
  const int N = g->n_atoms, C = m.spec.C, T = m.spec.n_layers;
  const bool wgrad = grad != nullptr;
  const bool tables = !wgrad;           // weight gradients need the radial network itself
  const long long E_all = sh ? sh->global->n_edges : E;
  // sharded: the whole graph's g_r, then the rank's receiver offsets, after the layout
  const size_t shard_extra = sh ? align_up((size_t)E_all * 12 + 4) + align_up((size_t)(N + 1) * 4) : 0;
  const WsLayout L = call_layout(m, E, N, wgrad, ws_bytes, shard_extra);
  if (ws_bytes < L.total + shard_extra) return EMP_ERR_WORKSPACE;
  int st = check_device();
  if (st != EMP_OK) return st;
  const size_t feat = (size_t)N * 16 * C;
  // the caller's sum over the ranks, in place, ordered on the stream
  auto allreduce = [&](float* buf, size_t n) -> int {
    if (!sh) return EMP_OK;
    return sh->allreduce(buf, n, stream, sh->ctx) == 0 ? EMP_OK : EMP_ERR_CUDA;
  };
  float* D = at<float>(ws, L.D);
  float* dist = at<float>(ws, L.dist);
  float* Rall = at<float>(ws, L.R);
  float* gRhi = at<float>(ws, L.gRhi);
  float* gRlo = at<float>(ws, L.gRlo);
  float* g_r = at<float>(ws, L.g_r);
  float* xs = at<float>(ws, L.xs);
  float* aggs = at<float>(ws, L.aggs);
  float* gxa = at<float>(ws, L.gx0);
  float* gxb = at<float>(ws, L.gx1);
  float* gS = at<float>(ws, L.gS);
  float* e_atom = atom_energy ? atom_energy : at<float>(ws, L.e_atom);
  float* XT = at<float>(ws, L.XT);
  float* XTlo = at<float>(ws, L.XTlo);
  float* Y = L.keep_y ? nullptr : at<float>(ws, L.Y);
  float* GYhi = at<float>(ws, L.GYhi);
  float* GYlo = at<float>(ws, L.GYlo);
  float* GXT = at<float>(ws, L.GXT);
  int* perm = at<int>(ws, L.perm);
  int* seg = at<int>(ws, L.seg);
  int* nseg = at<int>(ws, L.nseg);
  const float inv_avg = 1.0f / m.spec.avg_degree;
  int* counter = at<int>(ws, L.counter);
  Side side = side_for(stream);
  CohortMaps am_xt, am_gy;                 // pairs of cohorts (the backward's product launches)
  st = am_xt.build(C, E, 2 * coh, XT, XTlo);
  if (st != EMP_OK) return st;
  st = am_gy.build(C, E, 2 * coh, GYhi, GYlo);
  if (st != EMP_OK) return st;

  EMP_CUDA_TRY(cudaMemsetAsync(g_r, 0, (size_t)E * 12 + 4, stream));
  EMP_CUDA_TRY(cudaMemsetAsync(aggs, 0, (size_t)T * feat * 4, stream));
  { Scope sc_("embed", stream); k_embed<<<(unsigned)((feat + 255) / 256), 256, 0, stream>>>(N, C, species, m.spec.n_species, m.emb, xs); }
  if (E > 0) {
    { Scope sc_("geometry", stream); k_geometry_staged<<<(unsigned)((E + GEO_EPB - 1) / GEO_EPB), GEO_EPB, 0, stream>>>(E, g->vec, D, dist); }
    if (T > 2) {      // sender order of the cohorts, for the backward of the layers between the first and the last
      const int ncoh = (int)((E + coh - 1) / coh);
      int P = 1;
      while (P < coh) P <<= 1;
      { Scope sc_("cohort_sort", stream); k_cohort_sort<<<ncoh, 1024, (size_t)P * 8, stream>>>(E, (int)coh, g->send, perm, seg, nseg); }
    }
  }
  RadialRows rr;
  if (E > 0) {
    st = radial_rows(m, g, species, ws, L, rr, stream, wgrad);
    if (st != EMP_OK) return st;
  }
  // The first layer (its input, the species embedding, is degree 0 only) and the last layer
  // (read through degree 0 only) sum over each receiver's edges first and mix once per node
  // (end_layers.cuh); the layers between them run the per-edge products over cohorts.
  float* nodeZ = at<float>(ws, L.nodeZ);   // Z (first layer forward), H (first layer backward)
  float* nodeX = at<float>(ws, L.nodeX);   // X (last layer forward), G (last layer backward)
  const BlobOffsets bo = blob_offsets(m);
  float* dB = wgrad ? at<float>(ws, L.dB) : nullptr;       // dE/d(stacked SO(2) blocks) of one layer
  float* tnp = wgrad ? at<float>(ws, L.tnp) : nullptr;
  float* radrows = wgrad ? at<float>(ws, L.radrows) : nullptr;
  const unsigned nb_node = (unsigned)N;
  // ---------------- forward
  for (int t = 0; t < T; ++t) {
    float* R = Rall + (t == 0 ? 0 : (size_t)E * C + (size_t)(t - 1) * E * 4 * C);
    float* S = aggs + (size_t)t * feat;
    const float* W0 = m.so2_fwd + (size_t)t * m.so2_stride();
    const bool first = t == 0, last = t == T - 1;
    if (E > 0) {
      st = radial_forward(m, g, t, species, dist, R, rr, ws, L, stream, first ? C : 4 * C, tables);
      if (st != EMP_OK) return st;
      if (first) {
        { Scope sc_("first_fwd", stream); k_first_fwd<<<nb_node, C, 0, stream>>>(C, g->recv_off, g->send, rr.inv, D, R, xs, nodeZ); }
        // S_i[l, m', c'] = sum_c W0[(l, c'), (0, c)] Z_i[l, m', c], one product per degree
        NodeProducts np(C, C);
        for (int l = 0; l < 4; ++l)
          np.add(N * (2 * l + 1), 2 * l + 1, nodeZ + l * l * C, 16ll * C, C, W0 + (size_t)l * C * 4 * C, 4 * C,
                 S + l * l * C, 16ll * C, C);
        np.launch(stream);
      } else if (last) {
        { Scope sc_("last_fwd", stream); k_last_fwd<<<nb_node, C, 0, stream>>>(C, g->recv_off, g->send, rr.inv, D, R, xs + (size_t)t * feat, nodeX); }
        // S_i[0, c'] = sum_(l, c) W0[(0, c'), (l, c)] X_i[l, c]; the other components are not needed
        NodeProducts np(4 * C, C);
        np.add(N, 1, nodeX, 4ll * C, 0, W0, 4 * C, S, 16ll * C, 0);
        np.launch(stream);
      } else {
        st = layer_forward(m, g, t, xs + (size_t)t * feat, D, R, rr.inv, S, ws, L, stream,
                           L.keep_y ? at<float>(ws, L.Ykeep) + (size_t)(t - 1) * E * 16 * C : nullptr);
        if (st != EMP_OK) return st;
      }
    }
    // sharded: every receiver's sums come from the one rank that owns it; the sum over ranks gathers them
    st = allreduce(S, feat);
    if (st != EMP_OK) return st;
    { Scope sc_("update", stream); k_update<<<(unsigned)((N * C + 255) / 256), 256, 0, stream>>>(N, C, inv_avg, m.spec.gated, S,
                                                                   xs + (size_t)t * feat, xs + (size_t)(t + 1) * feat); }
  }
  {
    // e_i = w_o . SiLU(W_ro h_i[0]) and dE/dh_i (degree 0 only): two per-node products around
    // the activation
    float* zro = at<float>(ws, L.zro);
    NodeProducts z(C, m.Hro);
    z.add(N, 1, xs + (size_t)T * feat, 16ll * C, 0, m.ro_W, C, zro, m.Hro, 0);
    z.launch(stream, "readout");
    float* silu = wgrad ? at<float>(ws, L.silu) : nullptr;
    { Scope sc_("readout", stream); k_readout_act<<<(unsigned)((N * 32 + 255) / 256), 256, 0, stream>>>(N, m.Hro, m.ro_w, zro, e_atom, silu); }
    if (wgrad) {
      // dE/dw_o = sum_i SiLU(z_i); dE/dW_ro = sum_i (dE/dz_i) (x) h_i[0]
      EMP_CUDA_TRY(cudaMemsetAsync(grad, 0, weight_count(m.spec) * 4, stream));
      { Scope sc_("weight_grad", stream); k_colsum<<<(unsigned)((m.Hro + 127) / 128), 128, 0, stream>>>(N, m.Hro, silu, m.Hro, grad + bo.ro_w); }
      tn_sum(m.Hro, C, N, 1, zro, nullptr, m.Hro, 0, xs + (size_t)T * feat, nullptr, 16ll * C, 0, grad + bo.ro_W, C, false,
             tnp, tn_part_floats(C), stream);
    }
    EMP_CUDA_TRY(cudaMemsetAsync(gxa, 0, feat * 4, stream));
    NodeProducts gh(m.Hro, C);
    gh.add(N, 1, zro, m.Hro, 0, m.ro_WT, m.Hro, gxa, 16ll * C, 0);
    gh.launch(stream, "readout");
  }
  { Scope sc_("energy_sum", stream); k_energy_sum<<<1, 1024, 0, stream>>>(N, e_atom, energy); }
  // ---------------- backward, one layer at a time in reverse
  for (int t = T - 1; t >= 0; --t) {
    const float* R = Rall + (t == 0 ? 0 : (size_t)E * C + (size_t)(t - 1) * E * 4 * C);
    const float* xt = xs + (size_t)t * feat;
    const float* Wb = m.so2_bwd + (size_t)t * m.so2_stride();
    const bool first = t == 0, last = t == T - 1;
    { Scope sc_("gate_bwd", stream); k_gate_bwd<<<(unsigned)((N * C + 255) / 256), 256, 0, stream>>>(N, C, inv_avg, m.spec.gated,
                                                                     aggs + (size_t)t * feat, gxa, gS, gxb); }
    // sharded: the residual part of dE/dx_t enters the sum over ranks once (rank 0)
    if (sh && sh->rank != 0 && t > 0) EMP_CUDA_TRY(cudaMemsetAsync(gxb, 0, feat * 4, stream));
    if (wgrad) {
      EMP_CUDA_TRY(cudaMemsetAsync(dB, 0, (size_t)WLAYER_CC * C * C * 4, stream));
      if (E > 0 && first) {
        // dW0[(l, c'), (0, c)] = sum over (i, m') of gS_i[l, m', c'] Z_i[l, m', c]  (Z: the forward's sums)
        for (int l = 0; l < 4; ++l)
          tn_sum(C, C, N * (2 * l + 1), 2 * l + 1, gS + l * l * C, nullptr, 16ll * C, C, nodeZ + l * l * C, nullptr,
                 16ll * C, C, dB + (size_t)l * C * 4 * C, 4 * C, false, tnp, tn_part_floats(C), stream);
      } else if (E > 0 && last) {
        // dW0[(0, c'), (l, c)] = sum_i gS_i[0, c'] X_i[l, c]
        tn_sum(C, 4 * C, N, 1, gS, nullptr, 16ll * C, 0, nodeX, nullptr, 4ll * C, 0, dB, 4 * C, false, tnp,
               tn_part_floats(C), stream);
      }
    }
    if (E > 0 && first) {
      // H_i[l, m', c] = sum_c' W0[(l, c'), (0, c)] gS_i[l, m', c']
      NodeProducts np(C, C);
      for (int l = 0; l < 4; ++l)
        np.add(N * (2 * l + 1), 2 * l + 1, gS + l * l * C, 16ll * C, C, Wb + (size_t)l * C, 4 * C, nodeZ + l * l * C,
               16ll * C, C);
      np.launch(stream);
      // with weight gradients also dE/dx_0 (degree 0 of the senders) for dE/demb
      { Scope sc_("first_bwd", stream); k_first_bwd<<<nb_node, C, 0, stream>>>(C, g->recv_off, g->send, rr.inv, g->vec, D, R, xt, nodeZ, gRhi, gRlo, g_r, wgrad ? gxb : nullptr); }
    } else if (E > 0 && last) {
      // the output gradient is degree 0 only: G_i[l, c] = sum_c' W0[(0, c'), (l, c)] gS_i[0, c']
      NodeProducts np(C, 4 * C);
      np.add(N, 1, gS, 16ll * C, 0, Wb, 4 * C, nodeX, 4ll * C, 0);
      np.launch(stream);
      { Scope sc_("last_bwd", stream); k_last_bwd<<<nb_node, C, 0, stream>>>(C, g->recv_off, g->send, rr.inv, g->vec, D, R, xt, nodeX, gRhi, gRlo, g_r, gxb); }
    } else if (E > 0) {
      // [per-edge product launches: begin]
      // Cohorts are taken two at a time: one backward prep and one grouped product launch (the
      // transposed blocks, and the recomputed forward blocks unless y was kept) over both, then
      // the per-edge backward and the sender sums cohort by cohort, in order.
      const float* Ykept = L.keep_y ? at<float>(ws, L.Ykeep) + (size_t)(t - 1) * E * 16 * C : nullptr;
      int ci = 0;
      for (long long g0 = 0; g0 < E; g0 += 2 * coh) {
        const long long g1 = std::min(E, g0 + 2 * coh), M = g1 - g0;
        if (Ykept && !wgrad) {
          // g_y alone: the receivers' gS rows rotated into the edge frame
          const int per = rs_per(M, tc::num_sms(), 6);
          Scope sc_("bwd_prep", stream);
          k_rotate_staged<false, RS_V_FWD><<<(unsigned)((M + per - 1) / per), C / RS_V_FWD, rs_smem_bytes(C, false), stream>>>(
              g0, g1, C, per, nullptr, g->recv, nullptr, D, nullptr, gS, nullptr, GYhi, GYlo, nullptr, nullptr);
        } else {
          const int per = rs_per(M, tc::num_sms(), 3);
          Scope sc_("bwd_prep", stream);
          k_rotate_staged<true, RS_V_BWD><<<(unsigned)((M + per - 1) / per), C / RS_V_BWD, rs_smem_bytes(C, true), stream>>>(
              g0, g1, C, per, g->recv, g->send, rr.inv, D, R, xt, gS, XT, XTlo, GYhi, GYlo);
        }
        const So2Part xt_part{am_xt.get(M), &m.bmaps_fwd[t], Y}, gy_part{am_gy.get(M), &m.bmaps_bwd[t], GXT};
        So2Part parts[2] = {xt_part, gy_part};
        st = Ykept ? so2_product(m, M, &gy_part, 1, counter, stream) : so2_product(m, M, parts, 2, counter, stream);
        if (st != EMP_OK) return st;
        const float* Yg = Ykept ? Ykept + (size_t)g0 * 16 * C : Y;   // the pair's y rows
        if (wgrad) {   // dB_b += sum over the cohorts' edges of g_y (x) x~ per block (both as their hi + lo)
          st = so2_block_sums(C, M, GYhi, GYlo, XT, XTlo, dB, ws, L, counter, stream);
          if (st != EMP_OK) return st;
        }
        for (long long e0 = g0; e0 < g1; e0 += coh, ++ci) {
          const long long e1 = std::min(g1, e0 + coh), n = e1 - e0;
          const size_t ro = (size_t)(e0 - g0) * 16 * C;     // the cohort's rows in the pair's buffers
          // per-edge backward and the sender sums of dE/dx_send into gxb
          const int per = be_per(n, tc::num_sms());
          const int nb = (int)((n + per - 1) / per);
          // run pieces in two buffers, cohort by cohort in turn: the combine of the cohort before
          // last has read this one (the last combine may still run beside this kernel)
          float* Pg = at<float>(ws, ci & 1 ? L.gxP2 : L.gxP);
          side.wait_second_last();
          {
            Scope sc_("bwd_edge", stream);
            k_bwd_edge<BE_V><<<nb, C / BE_V, be_smem_bytes(C), stream>>>(e0, e1, C, per, g->send, rr.inv, g->vec, D, R,
                                                               xt, Yg + ro, gS, GXT + ro, g->recv, perm, gRhi, gRlo, g_r, Pg);
          }
          side.run([&](cudaStream_t q) {
            Scope sc_("gx_combine", q);
            k_gx_combine<<<(unsigned)std::min<long long>(n, 2048), C, 0, q>>>(e0, e1, C, ci, per, g->send, perm, seg,
                                                                            nseg, Pg, gxb);
          });
        }
      }
      side.wait();        // g_x of this layer complete
      // [per-edge product launches: end]
    }
    if (wgrad) {
      Scope sc_("weight_grad", stream);
      k_unstack_so2<<<256, 256, 0, stream>>>(C, dB, grad + bo.so2[t]);
    }
    if (E > 0) {
      if (wgrad) {
        // dW3 = sum over a network's rows of dE/dR (x) h2 (h2 of this layer recomputed)
        st = radial_forward(m, g, t, species, dist, nullptr, rr, ws, L, stream, first ? C : 4 * C, false, true);
        if (st != EMP_OK) return st;
        const float* h2hi = at<float>(ws, L.h2hi);
        const float* h2lo = at<float>(ws, L.h2lo);
        for (int p = 0; p < m.n_pairs; ++p) {
          const int r0 = rr.off[p], n = rr.off[p + 1] - r0;
          tn_sum(first ? C : 4 * C, 64, n, 1, gRhi + (size_t)r0 * 4 * C, gRlo + (size_t)r0 * 4 * C, 4ll * C, 0,
                 h2hi + (size_t)r0 * 64, h2lo + (size_t)r0 * 64, 64, 0, grad + bo.rad[(size_t)t * m.n_pairs + p] + 64 * 8 + 64 * 64,
                 64, false, tnp, tn_part_floats(C), stream);
        }
      }
      st = radial_backward(m, g, t, species, dist, rr, g_r, ws, L, stream, first ? C : 4 * C, tables, radrows);
      if (st != EMP_OK) return st;
      if (wgrad)
        for (int p = 0; p < m.n_pairs; ++p) {
          // dW2 = sum dE/dz2 (x) h1, dW1 = sum dE/dz1 (x) e over the network's rows
          const int r0 = rr.off[p], n = rr.off[p + 1] - r0;
          const float* rows = radrows + (size_t)r0 * RAD_ROW_FLOATS;
          float* gw = grad + bo.rad[(size_t)t * m.n_pairs + p];
          tn_sum(64, 64, n, 1, rows + 136, nullptr, RAD_ROW_FLOATS, 0, rows + 8, nullptr, RAD_ROW_FLOATS, 0, gw + 64 * 8, 64,
                 false, tnp, tn_part_floats(C), stream);
          tn_sum(64, 8, n, 1, rows + 72, nullptr, RAD_ROW_FLOATS, 0, rows, nullptr, RAD_ROW_FLOATS, 0, gw, 8, false, tnp,
                 tn_part_floats(C), stream);
        }
    }
    if (t > 0) {     // sharded: the senders' gradients from every rank's edges
      st = allreduce(gxb, feat);
      if (st != EMP_OK) return st;
    }
    std::swap(gxa, gxb);
  }
  if (wgrad) {
    Scope sc_("weight_grad", stream);
    k_species_sum<<<(unsigned)((m.spec.n_species * C + 127) / 128), 128, 0, stream>>>(N, C, m.spec.n_species, species, gxa, grad);
  }
  const emp_graph* gf = g;                  // the graph the forces and the virial are summed over
  float* gr_all = g_r;
  if (sh) {
    // the edge gradients of every rank, placed at their edges of the whole graph and summed over ranks
    gf = sh->global;
    gr_all = reinterpret_cast<float*>(static_cast<char*>(ws) + L.total);
    EMP_CUDA_TRY(cudaMemsetAsync(gr_all, 0, (size_t)E_all * 12, stream));
    if (E > 0) EMP_CUDA_TRY(cudaMemcpyAsync(gr_all + 3 * sh->e_begin, g_r, (size_t)E * 12, cudaMemcpyDeviceToDevice, stream));
    st = allreduce(gr_all, (size_t)E_all * 3);
    if (st != EMP_OK) return st;
  }
  { Scope sc_("forces", stream); k_forces<<<(N + 127) / 128, 128, 0, stream>>>(N, gf->recv_off, gf->mirror, gr_all, forces); }
  if (virial) {
    double* part = at<double>(ws, L.vir);
    { Scope sc_("virial", stream); k_virial_partial<<<VIR_BLOCKS, 256, 0, stream>>>(gf->n_edges, gf->vec, gr_all, part); }
    { Scope sc_("virial", stream); k_virial_final<<<1, 32, 0, stream>>>(VIR_BLOCKS, part, virial); }
  }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

int mp_energy_forces(const void* model, const emp_graph* g, const int32_t* species, double* energy, float* forces,
                     float* virial, float* atom_energy, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!model || !graph_ok(g) || !energy || !forces || !ws || g->n_atoms < 1) return EMP_ERR_ARG;
  return energy_forces_impl(*static_cast<const Model*>(model), g, species, energy, forces, virial, atom_energy, nullptr, ws,
                            ws_bytes, stream);
}

size_t mp_sharded_workspace_bytes(const void* model, int64_t n_edges_local, int64_t n_edges, int32_t n_atoms) {
  if (!model || n_edges_local < 0 || n_edges < n_edges_local || n_atoms < 1) return 0;
  return ws_layout(*static_cast<const Model*>(model), n_edges_local, n_atoms, false, true).total +
         align_up((size_t)n_edges * 12 + 4) + align_up((size_t)(n_atoms + 1) * 4);
}

int mp_energy_forces_sharded(const void* model, const emp_graph* g, int32_t atom_begin, int32_t atom_end, int32_t rank,
                             const int32_t* species, double* energy, float* forces, float* virial, float* atom_energy,
                             emp_allreduce_fn allreduce, void* ctx, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!model || !graph_ok(g) || !energy || !forces || !ws || !allreduce || g->n_atoms < 1) return EMP_ERR_ARG;
  if (atom_begin < 0 || atom_end < atom_begin || atom_end > g->n_atoms || rank < 0) return EMP_ERR_ARG;
  const Model& m = *static_cast<const Model*>(model);
  const int N = g->n_atoms;
  int st = check_device();
  if (st != EMP_OK) return st;
  // this rank's edges: those of receivers [atom_begin, atom_end) (read back: the local view needs them)
  int off[2] = {0, 0};
  EMP_CUDA_TRY(cudaMemcpyAsync(&off[0], g->recv_off + atom_begin, 4, cudaMemcpyDeviceToHost, stream));
  EMP_CUDA_TRY(cudaMemcpyAsync(&off[1], g->recv_off + atom_end, 4, cudaMemcpyDeviceToHost, stream));
  EMP_CUDA_TRY(cudaStreamSynchronize(stream));
  const long long eb = off[0], El = (long long)off[1] - off[0];
  if (El < 0) return EMP_ERR_ARG;
  // the layout energy_forces_impl takes (y kept if the workspace holds it), then the extras
  const size_t extra = align_up((size_t)g->n_edges * 12 + 4) + align_up((size_t)(N + 1) * 4);
  const size_t need = call_layout(m, El, N, false, ws_bytes, extra).total + extra;
  if (ws_bytes < need) return EMP_ERR_WORKSPACE;
  const size_t ro_at = need - align_up((size_t)(N + 1) * 4);
  int* recv_off_local = reinterpret_cast<int*>(static_cast<char*>(ws) + ro_at);
  { Scope sc_("shard", stream); k_local_offsets<<<(unsigned)((N + 1 + 255) / 256), 256, 0, stream>>>(N, g->recv_off, (int)eb, (int)El, recv_off_local); }
  emp_graph gl = *g;
  gl.recv = g->recv + eb;
  gl.send = g->send + eb;
  gl.mirror = nullptr;           // global edge indices: only the whole graph's forces use them
  gl.shift = g->shift ? g->shift + 3 * eb : nullptr;
  gl.vec = g->vec + 3 * eb;
  gl.recv_off = recv_off_local;
  gl.n_edges = El;
  Shard sh;
  sh.global = g;
  sh.e_begin = eb;
  sh.rank = rank;
  sh.allreduce = allreduce;
  sh.ctx = ctx;
  return energy_forces_impl(m, &gl, species, energy, forces, virial, atom_energy, nullptr, ws, ws_bytes, stream, &sh);
}

size_t mp_weight_grad_workspace_bytes(const void* model, int64_t n_edges, int32_t n_atoms) {
  if (!model || n_edges < 0 || n_atoms < 1) return 0;
  return ws_layout(*static_cast<const Model*>(model), n_edges, n_atoms, true, true).total;
}

int mp_energy_weight_grad(const void* model, const emp_graph* g, const int32_t* species, double* energy, float* forces,
                          float* grad, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!model || !graph_ok(g) || !energy || !forces || !grad || !ws || g->n_atoms < 1) return EMP_ERR_ARG;
  return energy_forces_impl(*static_cast<const Model*>(model), g, species, energy, forces, nullptr, nullptr, grad, ws,
                            ws_bytes, stream);
}

// One SO(2) mixing of a batch of edge-frame rows (the per-m block products
// alone): Y = X B_b^T per block (transpose = 0) or Y = X B_b (transpose = 1),
// X and Y [M][16C] in the m-major column layout.  Workspace: 2 M 16C floats.
int mp_so2_mix(const void* model, int32_t layer, int32_t transpose, int64_t M, const float* X, float* Y, void* ws,
               size_t ws_bytes, cudaStream_t stream) {
  if (!model || !X || !Y || M < 0 || (M > 0 && !ws)) return EMP_ERR_ARG;
  const Model& m = *static_cast<const Model*>(model);
  if (layer < 0 || layer >= m.spec.n_layers) return EMP_ERR_ARG;
  const size_t n = (size_t)M * 16 * m.spec.C;
  if (ws_bytes < 2 * n * 4 + 256) return EMP_ERR_WORKSPACE;
  if (M == 0) return EMP_OK;
  int st = check_device();
  if (st != EMP_OK) return st;
  float* hi = static_cast<float*>(ws);
  float* lo = hi + n;
  int* counter = reinterpret_cast<int*>(lo + n);
  split(X, hi, lo, n, stream);
  So2AMaps am;
  st = so2_make_amaps(&am, m.spec.C, M, hi, lo);
  if (st != EMP_OK) return st;
  So2Part part{&am, transpose ? &m.bmaps_bwd[layer] : &m.bmaps_fwd[layer], Y};
  return so2_product(m, M, &part, 1, counter, stream);
}

// ------------------------------------------------------------------ radial chain
int mp_chain_create(const float* U, const float* M, void** chain) {
  if (!U || !M || !chain) return EMP_ERR_ARG;
  int st = check_device();
  if (st != EMP_OK) return st;
  st = ensure_attrs();
  if (st != EMP_OK) return st;
  Chain* c = new Chain();
  float* base = nullptr;
  const size_t n = 128 * 25 + 32 * 64 + 2 * ctc::B_FLOATS + 4 * 32 * 64 + 256 * 25;
  if (cudaMalloc(&base, n * 4) != cudaSuccess) { delete c; return EMP_ERR_CUDA; }
  c->base = base;
  c->Weff = base;
  c->U0 = base + 128 * 25;
  c->bfwd = c->U0 + 32 * 64;
  c->bbwd = c->bfwd + ctc::B_FLOATS;
  float* dU = c->bbwd + ctc::B_FLOATS;
  float* dM = dU + 4 * 32 * 64;
  if (cudaMemcpy(dU, U, 4 * 32 * 64 * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(dM, M, 256 * 25 * 4, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(base);
    delete c;
    return EMP_ERR_CUDA;
  }
  k_chain_fold<<<(128 * 25 + 255) / 256, 256>>>(dU, dM, c->Weff, c->U0);
  ctc::k_chain_bmats<<<(ctc::B_FLOATS + 255) / 256, 256>>>(c->Weff, c->U0, c->bfwd, c->bbwd);
  if (cudaDeviceSynchronize() != cudaSuccess) { cudaFree(base); delete c; return EMP_ERR_CUDA; }
  *chain = c;
  return EMP_OK;
}

void mp_chain_destroy(void* chain) {
  if (!chain) return;
  Chain* c = static_cast<Chain*>(chain);
  cudaFree(c->base);
  delete c;
}

int mp_radial_chain(const void* chain, int64_t E, const float* x, float* kc, float* y0, const float* g_kc,
                    const float* g_y0, float* g_x, cudaStream_t stream) {
  if (!chain || E < 0 || (E > 0 && (!x || !kc || !y0))) return EMP_ERR_ARG;
  if (g_x && E > 0 && (!g_kc || !g_y0)) return EMP_ERR_ARG;
  auto a16 = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  if (!a16(x) || !a16(kc) || !a16(y0) || (g_x && (!a16(g_x) || !a16(g_y0) || !a16(g_kc)))) return EMP_ERR_ARG;
  if (E == 0) return EMP_OK;
  const Chain& c = *static_cast<const Chain*>(chain);
  if (E > INT32_MAX - ctc::BM) return EMP_ERR_ARG;             // tensor-map row coordinates are 32-bit
  // persistent: one CTA per SM (its shared memory and all of TMEM), 128-row tiles round-robin
  const long long nt = (E + ctc::BM - 1) / ctc::BM;
  const unsigned g = (unsigned)std::min<long long>(nt, tc::num_sms());
  CUtensorMap mx;
  if (!tc::make_map(&mx, x, 128, (uint64_t)E, 128, ctc::BM)) return EMP_ERR_CUDA;
  { Scope sc_("chain_fwd", stream); ctc::k_chain_tc<true><<<g, ctc::THREADS, ctc::smem_bytes(true), stream>>>(E, mx, nullptr, c.bfwd, kc, y0); }
  if (g_x) {
    CUtensorMap mg;
    if (!tc::make_map(&mg, g_y0, 64, (uint64_t)E, 64, ctc::BM)) return EMP_ERR_CUDA;
    Scope sc_("chain_bwd", stream);
    ctc::k_chain_tc<false><<<g, ctc::THREADS, ctc::smem_bytes(false), stream>>>(E, mg, g_kc, c.bbwd, g_x, nullptr);
  }
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

}  // extern "C"
