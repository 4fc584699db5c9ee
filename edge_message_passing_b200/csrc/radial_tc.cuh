// The radial network of a layer in one kernel (page "deepmd-kit PR #6108": edge
// length -> radial basis -> radial network -> per-(l, channel) scales; the model's
// network is 8 Bessel functions with the polynomial envelope, 8 -> 64 -> 64 with
// SiLU, then the head 64 -> 4C):
//   R[row] = W3 SiLU(W2 SiLU(W1 e(d_row)))
// for the rows of one or several radial networks (species pairs), each over its own
// device row range of the pair-sorted row list.
//
// Persistent kernel on CTA pairs (clusters of 2, cta_group::2); a tile is 256 rows
// (128 per CTA) of one network; every product is 3xTF32 (a = hi + lo, hi = RN_tf32(a),
// lo = RN_tf32(a - hi); lo.hi + hi.lo + hi.hi accumulated in FP32 in tensor memory).
// In each CTA:
//  - eight hidden warps evaluate the basis and z1 = W1 e on SIMT (8 x 4 register tiles)
//    and write h1 = SiLU(z1), split, into the shared-memory A operand (64-byte-swizzled
//    K-major, the layout the MMA descriptors read); the leader's hidden thread issues
//    z2 = h1 W2^T (N = 64, W2 split into shared memory when the network changes); the
//    hidden warps read z2 back from tensor memory (a row and 32 units per thread) and
//    write h2 = SiLU(z2), split, over h1: the A operand of the head.  Two A buffers, so
//    the next tile's hidden layers run while the head of this one does;
//  - the leader's hidden thread also takes the tiles from the counter and publishes
//    them, one tile ahead, to every role of both CTAs;
//  - warp 0 streams the head weights W3 (hi, lo; this CTA's half of each n-tile's rows
//    per k-block) into a TMA ring deep enough to cover the L2 latency;
//  - the leader's warp 1 issues the head products R = h2 W3^T in n-tiles of up to 128
//    columns into a ring of three TMEM accumulators;
//  - eight epilogue warps (two per TMEM lane quarter) store the R rows: TMEM -> registers -> a 128-byte-swizzled
//    staging tile per warp -> one TMA bulk store per 32 x 32 block (plain masked stores
//    for a block whose rows run past the network's range).
// h1 and h2 never reach global memory.  Every wait is bounded: on timeout the CTA records
// a device error, stops, waits (bounded) for its own copies and MMAs and frees TMEM.
#pragma once
#include "so2_tc.cuh"
#include "conv.cuh"

namespace emp {
namespace rtc {

constexpr int BM = 128;                          // rows per CTA (256 per pair)
constexpr int HID_WARPS = 8;
constexpr int HID_THREADS = 32 * HID_WARPS;
constexpr int EPI_WARPS = 8;                     // two per TMEM lane quarter, alternate 32-column chunks
constexpr int HID_W0 = 2 + EPI_WARPS;            // first hidden warp
constexpr int THREADS = 32 * (HID_W0 + HID_WARPS);
constexpr int KB = 4;                            // 16-wide k-blocks of h2 (K = 64)
constexpr int AK_BYTES = BM * 64;                // one k-block of hi (or lo): 128 rows x 64 bytes
constexpr int ABUF_BYTES = 2 * KB * AK_BYTES;    // hi k-blocks, then lo k-blocks: 64 KB
constexpr int BST = 5;                           // W3 ring stages
constexpr int BHALF = 64 * 64;                   // hi (or lo) half of a stage: up to 64 rows x 64 bytes
constexpr int BSTAGE_BYTES = 2 * BHALF;
constexpr int NACC = 3;                          // head accumulators (ring of n-tiles)
constexpr int ACC_COLS = 128;                    // one head accumulator (MMA N <= 128)
constexpr int ZCOL = NACC * ACC_COLS;            // z2, 64 columns
constexpr int TMEM_FWD = 512;
constexpr int EPI_TILE = 32 * 128;               // a 32 x 32 fp32 staging tile (128-byte swizzle)
constexpr int OFF_A = 0;                         // two A buffers: h1, then h2 (hi k-blocks, then lo)
constexpr int OFF_B = OFF_A + 2 * ABUF_BYTES;
constexpr int OFF_EPI = OFF_B + BST * BSTAGE_BYTES;   // a staging tile per epilogue warp
constexpr int OFF_W2 = OFF_EPI + EPI_WARPS * EPI_TILE;   // W2 (B of z2): this CTA's 32 rows, hi then lo
constexpr int OFF_W1 = OFF_W2 + 2 * KB * 32 * 64;
constexpr int OFF_E = OFF_W1 + 64 * 8 * 4;
constexpr int OFF_D = OFF_E + BM * 8 * 4;
constexpr int OFF_BAR = OFF_D + BM * 4;
constexpr int BAR_BYTES = 512;
constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;
static_assert(SMEM <= 232448, "shared memory per CTA");
static_assert(OFF_EPI % 1024 == 0 && OFF_W2 % 1024 == 0 && OFF_B % 1024 == 0, "operand and staging alignment");
static_assert(ZCOL + 64 <= TMEM_FWD, "tensor memory columns");

// MMA N of the head for ncols output columns: ncols up to 128, else the widest of 128, 96, 64, 32 dividing it
__host__ __device__ constexpr int fwd_bn(int n) {
  return n <= 128 ? n : n % 128 == 0 ? 128 : n % 96 == 0 ? 96 : n % 64 == 0 ? 64 : 32;
}

struct Args {
  int nsub;              // radial networks, each over rows [row_off[s], row_off[s + 1])
  int mtiles;            // 256-row tiles per network (an upper bound when row_off is set)
  int M;                 // rows (upper bound of every range)
  int ncols, bn, ntiles; // output columns, MMA N, n-tiles per row tile
  const int* row_off;    // device [nsub + 1], or null (one network over [0, M))
  int* counter;          // tile counter (zeroed by the host)
  float* out;            // R [M][ncols]
  const int* perm;       // row -> edge, or null (identity)
  const float* dist;     // edge lengths by edge
  const float* rad;      // radial weights: per network W1 [64][8], W2 [64][64], ...
  size_t layer_off, pair_stride;
  float rc;
};
struct Maps {
  CUtensorMap b_hi[tc::MAXSUB], b_lo[tc::MAXSUB];   // W3 rows [ncols][64], boxes of bn / 2 rows
  CUtensorMap out;                                  // R [M][ncols], 32 x 32 boxes, 128-byte swizzle (stores)
};

__device__ __forceinline__ int row_base(const Args& a, int s) { return a.row_off ? a.row_off[s] : 0; }
__device__ __forceinline__ int row_end(const Args& a, int s) { return a.row_off ? a.row_off[s + 1] : a.M; }

// next row tile; tiles past a network's range are skipped along with the rest of that network
__device__ __forceinline__ int next_tile(const Args& a, int total) {
  int t = atomicAdd(a.counter, 1);
  while (a.row_off && t < total) {
    const int s = t / a.mtiles;
    if ((t % a.mtiles) * 2 * BM < row_end(a, s) - row_base(a, s)) break;
    atomicMax(a.counter, (s + 1) * a.mtiles);
    t = atomicAdd(a.counter, 1);
  }
  return t;
}

__device__ __forceinline__ void hid_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ void tma_store(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(src)), "r"(x), "r"(y)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the bulk stores this thread issued have read their shared-memory source
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// byte offset of element (row r, k) (k < 16) in a k-block of 64-byte rows, 64-byte swizzle
__device__ __forceinline__ uint32_t swz(int r, int k) {
  return (uint32_t)(r * 64 + ((((k >> 2) ^ (r >> 1)) & 3) << 4) + (k & 3) * 4);
}

// the 3xTF32 products of a 64-deep contraction (4 k-blocks of A and B) into TMEM column block d
__device__ __forceinline__ void mma_k64(uint32_t d, uint32_t a_hi, uint32_t a_lo, uint32_t b_hi, uint32_t b_lo,
                                        uint32_t b_kstride, uint32_t idesc) {
#pragma unroll
  for (int kb = 0; kb < KB; ++kb)
#pragma unroll
    for (int kk = 0; kk < tc::BK / 8; ++kk) {
      const uint32_t ao = kb * AK_BYTES + kk * 32, bo = kb * b_kstride + kk * 32;
      tc::mma_tf32_pair(d, tc::sdesc(a_lo + ao), tc::sdesc(b_hi + bo), idesc, (kb | kk) ? 1u : 0u);
      tc::mma_tf32_pair(d, tc::sdesc(a_hi + ao), tc::sdesc(b_lo + bo), idesc, 1u);
      tc::mma_tf32_pair(d, tc::sdesc(a_hi + ao), tc::sdesc(b_hi + bo), idesc, 1u);
    }
}

// W2 of network `sub` for the hidden products, split and swizzled as this CTA's 32 rows of a
// 64-row K-major B operand: rows n of W2 (W2 itself, z2 = h1 W2^T) or of W2^T (the backward's
// dE/dh1 = dE/dz2 W2), hi k-blocks at dst, lo k-blocks at dst + 4 * 2048
__device__ __forceinline__ void stage_w2(unsigned char* dst, const float* w2, uint32_t rank, bool transposed, int h) {
  for (int idx = h; idx < 32 * 64; idx += HID_THREADS) {
    const int nl = idx >> 6, k = idx & 63, n = (int)rank * 32 + nl;
    const float a = __ldg(&w2[transposed ? k * 64 + n : n * 64 + k]);
    const uint32_t o = (uint32_t)((k >> 4) * 2048) + swz(nl, k & 15);
    const float ah = tf32_rna(a);
    *reinterpret_cast<float*>(dst + o) = ah;
    *reinterpret_cast<float*>(dst + KB * 2048 + o) = tf32_rna(a - ah);
  }
}

// layer 1 of a 128-row tile (rows r0..r0+7, units j0..j0+3 of thread h): h1 = SiLU(W1 e) split into
// hi/lo and written as the A operand of z2 (abuf: hi k-blocks, then lo k-blocks)
__device__ __forceinline__ void layer1_to_a(const float* W1T, const float* sE, unsigned char* abuf, int r0, int j0) {
  float w1v[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const float4 w = *reinterpret_cast<const float4*>(W1T + n * 64 + j0);
    w1v[n][0] = w.x; w1v[n][1] = w.y; w1v[n][2] = w.z; w1v[n][3] = w.w;
  }
  unsigned char* ab = abuf + (j0 >> 4) * AK_BYTES;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const float4 ea = *reinterpret_cast<const float4*>(sE + (r0 + a) * 8);
    const float4 eb = *reinterpret_cast<const float4*>(sE + (r0 + a) * 8 + 4);
    const float ev[8] = {ea.x, ea.y, ea.z, ea.w, eb.x, eb.y, eb.z, eb.w};
    float hi[4], lo[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float acc = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) acc = fmaf(w1v[n][b], ev[n], acc);
      const float v = silu_fast(acc);
      hi[b] = tf32_rna(v);
      lo[b] = tf32_rna(v - hi[b]);
    }
    const uint32_t o = swz(r0 + a, j0 & 15);
    *reinterpret_cast<float4*>(ab + o) = make_float4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<float4*>(ab + KB * AK_BYTES + o) = make_float4(lo[0], lo[1], lo[2], lo[3]);
  }
}

__device__ __forceinline__ int next_tile_of(const Args& a, int total) { return next_tile(a, total); }

// The leader's hidden thread h == 0 as the tile scheduler: keeps the published tiles one ahead of
// its own loop (so that the other roles start the next tile early) and returns tile j.
template <class A>
__device__ __forceinline__ int publish_ahead(int j, int& published, bool& ended, uint64_t* tq_full, uint64_t* tq_empty,
                                             int* tq, volatile int* vabort, int total, const A& args) {
  using namespace tc;
  while (published <= j + 1 && !ended) {
    const int ps = published % TQ;
    int tn;
    if (published >= TQ && !mbar_wait_cluster(&tq_empty[ps], ((published / TQ) - 1) & 1)) {
      *vabort = 1;
      tn = total;
    } else {
      tn = *vabort ? total : next_tile_of(args, total);
    }
    tq[ps] = tn;
    remote_store(map_to_rank(smem_u32(&tq[ps]), 1), tn);
    mbar_arrive(&tq_full[ps]);
    remote_arrive(map_to_rank(smem_u32(&tq_full[ps]), 1));
    ended = tn >= total;
    ++published;
  }
  return tq[j % TQ];
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_radial_fwd_tc(const __grid_constant__ Args g, const __grid_constant__ Maps maps, int total_tiles) {
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);    // [BST] (the leader's are used)
  uint64_t* empty = full + BST;                                    // [BST]
  uint64_t* acc_full = empty + BST;                                // [NACC]
  uint64_t* acc_empty = acc_full + NACC;                           // [NACC] (the leader's are used)
  uint64_t* a_full = acc_empty + NACC;                             // [2] (the leader's are used)
  uint64_t* a_empty = a_full + 2;                                  // [2]
  uint64_t* a1_full = a_empty + 2;                                 // (the leader's is used)
  uint64_t* z2_full = a1_full + 1;
  uint64_t* drain = z2_full + 1;
  uint64_t* drain2 = drain + 1;
  uint64_t* tq_full = drain2 + 1;                                  // [TQ]
  uint64_t* tq_empty = tq_full + TQ;                               // [TQ] (the leader's are used)
  int* tq = reinterpret_cast<int*>(tq_empty + TQ);                 // [TQ]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq + TQ);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* issued = abort_flag + 1;
  int* consumed = issued + 1;
  int* hid_word = consumed + 1;                                    // broadcast to the hidden warps

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < BST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI_WARPS);   // the epilogue warps of both CTAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a_full[b], 2);           // the hidden warps of each CTA, once
      mbar_init(&a_empty[b], 1);
    }
    mbar_init(a1_full, 2);
    mbar_init(z2_full, 1);
    mbar_init(drain, 1);
    mbar_init(drain2, 1);
    for (int j = 0; j < TQ; ++j) {
      mbar_init(&tq_full[j], 1);
      mbar_init(&tq_empty[j], 2 * (2 + EPI_WARPS));   // leader: producer, MMA, epilogue; peer: producer, epilogue, hidden
    }
    *abort_flag = 0;
    *issued = 0;
    *consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)TMEM_FWD));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* vabort = abort_flag;
  const uint32_t full_l = map_to_rank(smem_u32(full), 0);
  const uint32_t acc_empty_l = map_to_rank(smem_u32(acc_empty), 0);
  const uint32_t a_full_l = map_to_rank(smem_u32(a_full), 0);
  const uint32_t a1_full_l = map_to_rank(smem_u32(a1_full), 0);
  const uint32_t tq_empty_l = map_to_rank(smem_u32(tq_empty), 0);
  const int bh = g.bn / 2;                 // this CTA's W3 rows per n-tile

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- W3 producer (both CTAs)
    int it = 0;
    for (int j = 0;; ++j) {
      const int slot = j % TQ;
      if (!mbar_wait_cluster(&tq_full[slot], (j / TQ) & 1)) { *vabort = 1; break; }
      const int t = tq[slot];
      if (leader) mbar_arrive(&tq_empty[slot]);
      else remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
      if (t >= total_tiles) break;
      const int sub = t / g.mtiles;
      bool stop = false;
      for (int n = 0; n < g.ntiles && !stop; ++n)
        for (int kc = 0; kc < KB; ++kc, ++it) {
          const int s = it % BST;
          if (it >= BST && !mbar_wait(&empty[s], ((it / BST) - 1) & 1)) { *vabort = 1; stop = true; break; }
          if (*vabort) { stop = true; break; }   // the scheduler then publishes the end to every role
          unsigned char* st = smem + OFF_B + s * BSTAGE_BYTES;
          if (leader) mbar_expect_tx(&full[s], 2 * 2 * bh * 64);
          const uint32_t fb = full_l + (uint32_t)(s * 8);
          tma_load_pair(st, &maps.b_hi[sub], fb, kc * BK, n * g.bn + (int)rank * bh);
          tma_load_pair(st + BHALF, &maps.b_lo[sub], fb, kc * BK, n * g.bn + (int)rank * bh);
          *issued = it + 1;
        }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- head MMA issuer (leader only)
    int it = 0, i = 0;
    bool ok = true;
    const uint32_t idesc = idesc_pair(g.bn);
    for (int j = 0; ok; ++j) {
      const int slot = j % TQ;
      if (!mbar_wait(&tq_full[slot], (j / TQ) & 1)) { ok = false; break; }
      const int t = tq[slot];
      mbar_arrive(&tq_empty[slot]);
      if (t >= total_tiles) break;
      const int ab = j & 1;
      if (!mbar_wait_cluster(&a_full[ab], (j >> 1) & 1)) { ok = false; break; }
      fence_after();
      const uint32_t a_base = smem_u32(smem + OFF_A + ab * ABUF_BYTES);
      for (int n = 0; n < g.ntiles; ++n, ++i) {
        const int buf = i % NACC;
        if (i >= NACC && !mbar_wait_cluster(&acc_empty[buf], ((i / NACC) - 1) & 1)) { ok = false; break; }
        fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * ACC_COLS);
        for (int kc = 0; kc < KB; ++kc, ++it) {
          const int s = it % BST;
          if (!mbar_wait(&full[s], (it / BST) & 1)) { ok = false; break; }
          *consumed = it + 1;
          fence_after();
          const uint32_t a_hi = a_base + kc * AK_BYTES;
          const uint32_t a_lo = a_hi + KB * AK_BYTES;
          const uint32_t b_hi = smem_u32(smem + OFF_B + s * BSTAGE_BYTES);
          const uint32_t b_lo = b_hi + BHALF;
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            const uint32_t off = kk * 32;
            mma_tf32_pair(d, sdesc(a_lo + off), sdesc(b_hi + off), idesc, (kc | kk) ? 1u : 0u);
            mma_tf32_pair(d, sdesc(a_hi + off), sdesc(b_lo + off), idesc, 1u);
            mma_tf32_pair(d, sdesc(a_hi + off), sdesc(b_hi + off), idesc, 1u);
          }
          mma_commit_pair(&empty[s]);
        }
        if (!ok) break;
        mma_commit_pair(&acc_full[buf]);
      }
      if (!ok) break;
      mma_commit_pair(&a_empty[ab]);     // both CTAs may overwrite this A buffer once these MMAs are done
    }
    if (!ok) *vabort = 1;
    mma_commit_pair(drain);
    mbar_wait(drain, 0);
  } else if (warp >= 2 && warp < HID_W0) {
    // ---------------------------------------------------------------- epilogue (both CTAs: own 128 rows)
    const int q = warp & 3, ehalf = (warp - 2) >> 2;    // lane quarter; which 32-column chunks
    int i = 0;
    for (int j = 0;; ++j) {
      const int slot = j % TQ;
      if (!mbar_wait_cluster(&tq_full[slot], (j / TQ) & 1)) { *vabort = 1; break; }
      const int t = tq[slot];
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tq_empty[slot]);
        else remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
      }
      if (t >= total_tiles) break;
      const int sub = t / g.mtiles;
      const int mw = row_base(g, sub) + (t % g.mtiles) * 2 * BM + (int)rank * BM + q * 32;
      const int mend = row_end(g, sub);
      const bool whole = mw + 32 <= mend;          // else the rows past the range are masked
      bool ok = true;
      for (int n = 0; n < g.ntiles; ++n, ++i) {
        const int buf = i % NACC;
        if (!mbar_wait(&acc_full[buf], (i / NACC) & 1)) { ok = false; break; }
        fence_after();
        float* obase = g.out + (size_t)n * g.bn;
#pragma unroll 1
        for (int cc = 32 * ehalf; cc < g.bn; cc += 64) {
          float v[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * ACC_COLS + cc), v);
          unsigned char* stg = smem + OFF_EPI + (warp - 2) * EPI_TILE;
          if (lane == 0) bulk_wait_read0();        // this warp's previous store has read the staging tile
          __syncwarp();
          // row `lane` as eight 16-byte chunks, chunk c at position c ^ (row & 7)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          if (whole) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // staged by threads, read by the copy engine
            __syncwarp();
            if (lane == 0) tma_store(&maps.out, stg, n * g.bn + cc, mw);
          } else {
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int rr = k * 4 + (lane >> 3), c = lane & 7;
              const int m = mw + rr;
              const float4 w = *reinterpret_cast<const float4*>(stg + rr * 128 + ((c ^ (rr & 7)) << 4));
              if (m < mend && cc + 4 * c < g.bn) *reinterpret_cast<float4*>(obase + (size_t)m * g.ncols + cc + 4 * c) = w;
            }
            __syncwarp();
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive(&acc_empty[buf]);
          else remote_arrive(acc_empty_l + (uint32_t)(buf * 8));
        }
      }
      if (!ok) { *vabort = 1; break; }
    }
    if (lane == 0) bulk_wait_all();
  } else if (warp >= HID_W0) {
    // ---------------------------------------------------------------- hidden layers -> h2 hi/lo in the A buffer
    const int h = threadIdx.x - 32 * HID_W0;
    const int r0 = (h >> 4) * 8, j0 = (h & 15) * 4;     // layer-1 register tile
    const int qz = warp & 3, half = (warp - HID_W0) >> 2;
    const int row = qz * 32 + lane, u0 = half * 32;     // z2 read-back: a row, 32 units
    float* W1T = reinterpret_cast<float*>(smem + OFF_W1);     // [n][j] = W1[j][n]
    float* sE = reinterpret_cast<float*>(smem + OFF_E);       // [r][n]
    float* sD = reinterpret_cast<float*>(smem + OFF_D);
    unsigned char* w2s = smem + OFF_W2;
    int staged = -1, published = 0;
    bool ended = false, issued_any = false;
    for (int j = 0;; ++j) {
      const int slot = j % TQ;
      const int ab = j & 1;
      unsigned char* abuf = smem + OFF_A + ab * ABUF_BYTES;
      if (h == 0) {
        int t;
        if (leader) {
          t = publish_ahead(j, published, ended, tq_full, tq_empty, tq, vabort, total_tiles, g);
        } else if (mbar_wait_cluster(&tq_full[slot], (j / TQ) & 1)) {
          t = tq[slot];
          remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
        } else {
          t = -1;
        }
        if (t >= 0 && t < total_tiles && j >= 2 && !mbar_wait(&a_empty[ab], ((j >> 1) - 1) & 1)) t = -1;
        if (t < 0) { *vabort = 1; t = total_tiles; }
        *hid_word = t;
      }
      hid_sync();
      const int t = *hid_word;
      if (t >= total_tiles) break;
      const int sub = t / g.mtiles;
      const int base = row_base(g, sub) + (t % g.mtiles) * 2 * BM + (int)rank * BM;
      const int rend = row_end(g, sub);
      if (h < BM) {
        const int r = base + h;
        float d = 1.f;
        if (r < rend) d = g.dist[g.perm ? g.perm[r] : r];
        sD[h] = d;
      }
      if (sub != staged) {
        const float* w1 = g.rad + g.layer_off + (size_t)sub * g.pair_stride;
        for (int idx = h; idx < 64 * 8; idx += HID_THREADS) W1T[(idx & 7) * 64 + (idx >> 3)] = __ldg(&w1[idx]);
        stage_w2(w2s, w1 + 64 * 8, rank, false, h);
        staged = sub;
      }
      hid_sync();
      for (int idx = h; idx < BM * 8; idx += HID_THREADS) {
        float ev, dv;
        bessel_n(sD[idx >> 3], g.rc, idx & 7, ev, dv);
        sE[idx] = ev;
      }
      hid_sync();
      layer1_to_a(W1T, sE, abuf, r0, j0);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // h1 and W2 written by threads, read by the MMAs
      hid_sync();
      if (h == 0) {
        if (leader) {
          mbar_arrive(a1_full);
          // z2 = h1 W2^T once both CTAs' h1 rows are in place
          if (mbar_wait_cluster(a1_full, j & 1)) {
            fence_after();
            const uint32_t au = smem_u32(abuf);
            mma_k64(tmem + ZCOL, au, au + KB * AK_BYTES, smem_u32(w2s), smem_u32(w2s + KB * 2048), 2048, idesc_pair(64));
            mma_commit_pair(z2_full);
            issued_any = true;
          } else {
            *vabort = 1;
          }
        } else {
          remote_arrive(a1_full_l);
        }
        const bool ok = !*vabort && mbar_wait(z2_full, j & 1);
        if (!ok) *vabort = 1;
        *hid_word = ok ? 1 : 0;
      }
      hid_sync();
      if (!*hid_word) break;
      fence_after();
      // h2 = SiLU(z2): a row and 32 units per thread, over h1 in the A buffer (z2 has read it)
      {
        float z2[32];
        tmem_ld32(tmem + ((uint32_t)(qz * 32) << 16) + (uint32_t)(ZCOL + u0), z2);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float hi[4], lo[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float v = silu_fast(z2[4 * c + b]);
            hi[b] = tf32_rna(v);
            lo[b] = tf32_rna(v - hi[b]);
          }
          const int k = u0 + 4 * c;
          const uint32_t o = (uint32_t)((k >> 4) * AK_BYTES) + swz(row, k & 15);
          *reinterpret_cast<float4*>(abuf + o) = make_float4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<float4*>(abuf + KB * AK_BYTES + o) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_before();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // h2 written by threads, read by the MMAs
      hid_sync();
      if (h == 0) {
        if (leader) mbar_arrive(&a_full[ab]);
        else remote_arrive(a_full_l + (uint32_t)(ab * 8));
      }
    }
    if (h == 0 && leader && issued_any) {
      mma_commit_pair(drain2);           // every product this thread issued has completed
      mbar_wait(drain2, 0);
    }
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  if (threadIdx.x == 0 && leader && *vabort) {
    // let W3 loads of either CTA still in flight land (they complete on the leader's barriers)
    const int peer_issued = remote_load(map_to_rank(smem_u32(issued), 1));
    const int last = max(*issued, peer_issued);
    for (int it = *consumed; it < last; ++it) mbar_wait(&full[it % BST], (it / BST) & 1);
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)TMEM_FWD));
  }
}

// R rows [M][ncols] of nsub radial networks over their row ranges (row_off, device; or one network
// over [0, M) when null); b_maps[s]: network s's W3 (hi, lo) maps with boxes of fwd_bn(ncols) / 2 rows.
inline int radial_fwd(long long M, int ncols, const int* row_off, int nsub, const int* perm, const float* dist,
                      const float* rad, size_t layer_off, size_t pair_stride, float rc, const MapPair* const* b_maps,
                      float* out, int* counter, cudaStream_t s) {
  if (M <= 0) return EMP_OK;
  if (nsub < 1 || nsub > tc::MAXSUB || M >= (1ll << 31) || ncols < 32 || ncols % 32 != 0) return EMP_ERR_ARG;
  Args g{};
  Maps maps;
  g.nsub = nsub;
  g.M = (int)M;
  g.mtiles = (int)((M + 2 * BM - 1) / (2 * BM));
  g.ncols = ncols;
  g.bn = fwd_bn(ncols);
  g.ntiles = ncols / g.bn;
  g.row_off = row_off;
  g.counter = counter;
  g.out = out;
  g.perm = perm;
  g.dist = dist;
  g.rad = rad;
  g.layer_off = layer_off;
  g.pair_stride = pair_stride;
  g.rc = rc;
  for (int q = 0; q < nsub; ++q) {
    maps.b_hi[q] = b_maps[q]->hi;
    maps.b_lo[q] = b_maps[q]->lo;
  }
  {
    auto fn = tc::encode_fn();
    if (!fn) return EMP_ERR_UNSUPPORTED;
    cuuint64_t dims[2] = {(cuuint64_t)ncols, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)ncols * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&maps.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return EMP_ERR_CUDA;
  }
  const long long total = (long long)nsub * g.mtiles;
  if (total >= (1ll << 31)) return EMP_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(counter, 0, sizeof(int), s) != cudaSuccess) return EMP_ERR_CUDA;
  const int pairs = (int)std::min<long long>(total, tc::num_sms() / 2);
  k_radial_fwd_tc<<<2 * pairs, THREADS, SMEM, s>>>(g, maps, (int)total);
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

// ------------------------------------------------------------------ backward
// dE/dd of every row from dE/dR (rows split hi/lo), adding (dE/dd) rhat to g_r:
//   dE/dh2 = dE/dR W3          (K = kcols, N = 64; the head's transpose)
//   z2 = W2 h1 (recomputed),   dE/dz2 = dE/dh2 SiLU'(z2)
//   dE/dh1 = W2^T dE/dz2,      dE/dz1 = dE/dh1 SiLU'(z1)
//   dE/dd = sum_j dE/dz1[j] sum_n W1[j][n] de_n/dd
// the three 64-wide contractions in 3xTF32 on the tensor cores, the rest on SIMT.
// Persistent kernel on CTA pairs, 256-row tiles (128 per CTA):
//  - warp 0 streams the tile's dE/dR k-blocks (hi, lo) and W3^T (this CTA's 32 of the
//    64 rows) into a 5-stage TMA ring; the leader's warp 1 issues the head products into
//    one of two 64-column TMEM accumulators (the next tile's head runs while the hidden
//    warps finish this one);
//  - eight hidden warps evaluate the basis and its derivative, z1 and h1 = SiLU(z1) (8 x 4
//    register tiles) and write h1 hi/lo as the A operand of z2; the leader's hidden thread
//    issues z2 = h1 W2^T, then, once the hidden warps have formed dE/dz2 (a row and 32
//    units per thread, read back from TMEM) in the same buffer, dE/dh1 = dE/dz2 W2; the
//    hidden warps read dE/dh1 back and finish dE/dd per row.
// The leader's hidden warps also take the tiles from the counter.
constexpr int B_THREADS = 32 * 10;
constexpr int B_HID_W0 = 2;                      // hidden warps 2..9
constexpr int B_ST = 5;
constexpr int B_AK = BM * 64;                    // one k-block of dE/dR hi (or lo): 8 KB
constexpr int B_BK = 32 * 64;                    // one k-block of W3^T hi (or lo): 32 rows, 2 KB
constexpr int B_STAGE = 2 * B_AK + 2 * B_BK;     // 20 KB
constexpr int B_OFF_H = 0;                       // h1, then dE/dz2 (hi k-blocks, then lo): 64 KB
constexpr int B_OFF_W2 = B_OFF_H + ABUF_BYTES;   // W2 (B of z2): this CTA's 32 rows, hi then lo
constexpr int B_OFF_W2T = B_OFF_W2 + 2 * 4 * B_BK;   // W2^T (B of dE/dh1)
constexpr int B_OFF_RING = B_OFF_W2T + 2 * 4 * B_BK;
constexpr int B_OFF_W1 = B_OFF_RING + B_ST * B_STAGE;
constexpr int B_OFF_E = B_OFF_W1 + 64 * 8 * 4;
constexpr int B_OFF_DE = B_OFF_E + BM * 8 * 4;
constexpr int B_OFF_D = B_OFF_DE + BM * 8 * 4;
constexpr int B_OFF_EDGE = B_OFF_D + BM * 4;
constexpr int B_OFF_GD = B_OFF_EDGE + BM * 4;
constexpr int B_OFF_BAR = B_OFF_GD + 2 * BM * 4;
constexpr int B_SMEM = B_OFF_BAR + BAR_BYTES + 1024;
constexpr int B_TMEM_COLS = 256;                 // dE/dh2 x 2, then z2 / dE/dh1
constexpr int B_ZCOL = 128;
static_assert(B_SMEM <= 232448, "shared memory per CTA");
static_assert(B_OFF_RING % 1024 == 0 && B_OFF_W2 % 1024 == 0 && B_OFF_W2T % 1024 == 0, "operand alignment");

struct BwdArgs {
  int nsub, mtiles, M;
  int kcols;             // columns of dE/dR that carry a gradient (4C, or C in the first layer)
  const int* row_off;
  int* counter;
  const int* perm;       // row -> edge, or null
  const float* dist;     // by edge
  const float* vec;      // by edge, [E][3]
  float* g_r;            // by edge, [E][3]: += (dE/dd) rhat
  const float* rad;
  size_t layer_off, pair_stride;
  float rc;
};
struct BwdMaps {
  CUtensorMap a_hi, a_lo;                         // dE/dR [M][4C], boxes of 128 rows x 16
  CUtensorMap b_hi[tc::MAXSUB], b_lo[tc::MAXSUB]; // W3^T [64][4C], boxes of 32 rows x 16
};

__device__ __forceinline__ int row_base_b(const BwdArgs& a, int s) { return a.row_off ? a.row_off[s] : 0; }
__device__ __forceinline__ int row_end_b(const BwdArgs& a, int s) { return a.row_off ? a.row_off[s + 1] : a.M; }
__device__ __forceinline__ int next_tile_b(const BwdArgs& a, int total) {
  int t = atomicAdd(a.counter, 1);
  while (a.row_off && t < total) {
    const int s = t / a.mtiles;
    if ((t % a.mtiles) * 2 * BM < row_end_b(a, s) - row_base_b(a, s)) break;
    atomicMax(a.counter, (s + 1) * a.mtiles);
    t = atomicAdd(a.counter, 1);
  }
  return t;
}

__device__ __forceinline__ int next_tile_of(const BwdArgs& a, int total) { return next_tile_b(a, total); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(B_THREADS, 1)
    k_radial_bwd_tc(const __grid_constant__ BwdArgs g, const __grid_constant__ BwdMaps maps, int total_tiles) {
  using namespace tc;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + B_OFF_BAR);  // [B_ST] (the leader's are used)
  uint64_t* empty = full + B_ST;                                   // [B_ST]
  uint64_t* gh2_full = empty + B_ST;                               // [2]
  uint64_t* gh2_empty = gh2_full + 2;                              // [2] (the leader's are used)
  uint64_t* a1_full = gh2_empty + 2;                               // (the leader's is used)
  uint64_t* a2_full = a1_full + 1;                                 // (the leader's is used)
  uint64_t* z2_full = a2_full + 1;
  uint64_t* gh1_full = z2_full + 1;
  uint64_t* drain = gh1_full + 1;
  uint64_t* drain2 = drain + 1;
  uint64_t* tq_full = drain2 + 1;                                  // [TQ]
  uint64_t* tq_empty = tq_full + TQ;                               // [TQ] (the leader's are used)
  int* tq = reinterpret_cast<int*>(tq_empty + TQ);                 // [TQ]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq + TQ);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* issued = abort_flag + 1;
  int* consumed = issued + 1;
  int* hid_word = consumed + 1;                                    // broadcast to the hidden warps

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < B_ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&gh2_full[b], 1);
      mbar_init(&gh2_empty[b], 2);        // the hidden warps of each CTA, once
    }
    mbar_init(a1_full, 2);
    mbar_init(a2_full, 2);
    mbar_init(z2_full, 1);
    mbar_init(gh1_full, 1);
    mbar_init(drain, 1);
    mbar_init(drain2, 1);
    for (int j = 0; j < TQ; ++j) {
      mbar_init(&tq_full[j], 1);
      mbar_init(&tq_empty[j], 4);         // leader: producer, MMA; peer: producer, hidden
    }
    *abort_flag = 0;
    *issued = 0;
    *consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)B_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* vabort = abort_flag;
  const uint32_t full_l = map_to_rank(smem_u32(full), 0);
  const uint32_t gh2_empty_l = map_to_rank(smem_u32(gh2_empty), 0);
  const uint32_t a1_full_l = map_to_rank(smem_u32(a1_full), 0);
  const uint32_t a2_full_l = map_to_rank(smem_u32(a2_full), 0);
  const uint32_t tq_empty_l = map_to_rank(smem_u32(tq_empty), 0);
  const int KC = g.kcols / BK;
  const uint32_t idesc64 = idesc_pair(64);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- dE/dR and W3^T producer (both CTAs)
    int it = 0;
    for (int j = 0;; ++j) {
      const int slot = j % TQ;
      if (!mbar_wait_cluster(&tq_full[slot], (j / TQ) & 1)) { *vabort = 1; break; }
      const int t = tq[slot];
      if (leader) mbar_arrive(&tq_empty[slot]);
      else remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
      if (t >= total_tiles) break;
      const int sub = t / g.mtiles;
      const int arow = row_base_b(g, sub) + (t % g.mtiles) * 2 * BM + (int)rank * BM;
      for (int kc = 0; kc < KC; ++kc, ++it) {
        const int s = it % B_ST;
        if (it >= B_ST && !mbar_wait(&empty[s], ((it / B_ST) - 1) & 1)) { *vabort = 1; break; }
        if (*vabort) break;
        unsigned char* st = smem + B_OFF_RING + s * B_STAGE;
        if (leader) mbar_expect_tx(&full[s], 2 * B_STAGE);
        const uint32_t fb = full_l + (uint32_t)(s * 8);
        tma_load_pair(st, &maps.a_hi, fb, kc * BK, arow);
        tma_load_pair(st + B_AK, &maps.a_lo, fb, kc * BK, arow);
        tma_load_pair(st + 2 * B_AK, &maps.b_hi[sub], fb, kc * BK, (int)rank * 32);
        tma_load_pair(st + 2 * B_AK + B_BK, &maps.b_lo[sub], fb, kc * BK, (int)rank * 32);
        *issued = it + 1;
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- head-transpose MMA issuer (leader only)
    int it = 0;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      const int slot = j % TQ;
      if (!mbar_wait(&tq_full[slot], (j / TQ) & 1)) { ok = false; break; }
      const int t = tq[slot];
      mbar_arrive(&tq_empty[slot]);
      if (t >= total_tiles) break;
      const int gb = j & 1;
      if (j >= 2 && !mbar_wait_cluster(&gh2_empty[gb], ((j >> 1) - 1) & 1)) { ok = false; break; }
      fence_after();
      const uint32_t d = tmem + (uint32_t)(gb * 64);
      for (int kc = 0; kc < KC; ++kc, ++it) {
        const int s = it % B_ST;
        if (!mbar_wait(&full[s], (it / B_ST) & 1)) { ok = false; break; }
        *consumed = it + 1;
        fence_after();
        const uint32_t a_hi = smem_u32(smem + B_OFF_RING + s * B_STAGE);
        const uint32_t a_lo = a_hi + B_AK, b_hi = a_hi + 2 * B_AK, b_lo = b_hi + B_BK;
#pragma unroll
        for (int kk = 0; kk < BK / 8; ++kk) {
          const uint32_t off = kk * 32;
          mma_tf32_pair(d, sdesc(a_lo + off), sdesc(b_hi + off), idesc64, (kc | kk) ? 1u : 0u);
          mma_tf32_pair(d, sdesc(a_hi + off), sdesc(b_lo + off), idesc64, 1u);
          mma_tf32_pair(d, sdesc(a_hi + off), sdesc(b_hi + off), idesc64, 1u);
        }
        mma_commit_pair(&empty[s]);
      }
      if (!ok) break;
      mma_commit_pair(&gh2_full[gb]);
    }
    if (!ok) *vabort = 1;
    mma_commit_pair(drain);
    mbar_wait(drain, 0);
  } else if (warp >= B_HID_W0) {
    // ---------------------------------------------------------------- hidden warps
    const int h = threadIdx.x - 32 * B_HID_W0;
    const int r0 = (h >> 4) * 8, j0 = (h & 15) * 4;     // layer-1 register tile
    const int q = warp & 3, half = (warp - B_HID_W0) >> 2;
    const int row = q * 32 + lane, u0 = half * 32;      // TMEM read-back: a row, 32 units
    float* W1T = reinterpret_cast<float*>(smem + B_OFF_W1);   // [n][j]
    float* sE = reinterpret_cast<float*>(smem + B_OFF_E);
    float* sDE = reinterpret_cast<float*>(smem + B_OFF_DE);
    float* sD = reinterpret_cast<float*>(smem + B_OFF_D);
    int* sEdge = reinterpret_cast<int*>(smem + B_OFF_EDGE);
    float* sGD = reinterpret_cast<float*>(smem + B_OFF_GD);
    unsigned char* hbuf = smem + B_OFF_H;
    const uint32_t hbuf_u = smem_u32(hbuf);
    int staged = -1;
    bool issued_any = false;                            // the leader's h == 0 issued MMAs (drained at exit)
    int published = 0;                                  // the leader's h == 0: tiles published so far
    bool ended = false;
    for (int j = 0;; ++j) {
      const int slot = j % TQ;
      const int gb = j & 1;
      if (h == 0) {
        int t;
        if (leader) {
          // the scheduler, one tile ahead: the head of tile j + 1 streams while these warps finish tile j
          t = publish_ahead(j, published, ended, tq_full, tq_empty, tq, vabort, total_tiles, g);
        } else if (mbar_wait_cluster(&tq_full[slot], (j / TQ) & 1)) {
          t = tq[slot];
          remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
        } else {
          *vabort = 1;
          t = total_tiles;
        }
        *hid_word = t;
      }
      hid_sync();
      const int t = *hid_word;
      if (t >= total_tiles) break;
      const int sub = t / g.mtiles;
      const int base = row_base_b(g, sub) + (t % g.mtiles) * 2 * BM + (int)rank * BM;
      const int rend = row_end_b(g, sub);
      if (h < BM) {
        const int r = base + h;
        int e = -1;
        float d = 1.f;
        if (r < rend) {
          e = g.perm ? g.perm[r] : r;
          d = g.dist[e];
        }
        sD[h] = d;
        sEdge[h] = e;
      }
      if (sub != staged) {
        // W1 transposed; this CTA's 32 rows of W2 (B of z2) and of W2^T (B of dE/dh1), split and swizzled
        const float* w1 = g.rad + g.layer_off + (size_t)sub * g.pair_stride;
        for (int idx = h; idx < 64 * 8; idx += HID_THREADS) W1T[(idx & 7) * 64 + (idx >> 3)] = __ldg(&w1[idx]);
        stage_w2(smem + B_OFF_W2, w1 + 64 * 8, rank, false, h);
        stage_w2(smem + B_OFF_W2T, w1 + 64 * 8, rank, true, h);
        staged = sub;
      }
      hid_sync();
      for (int idx = h; idx < BM * 8; idx += HID_THREADS) {
        float ev, dv;
        bessel_n(sD[idx >> 3], g.rc, idx & 7, ev, dv);
        sE[idx] = ev;
        sDE[idx] = dv;
      }
      hid_sync();
      // ---- z1, h1 = SiLU(z1) as the A operand of z2
      layer1_to_a(W1T, sE, hbuf, r0, j0);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // h1 and W2 written by threads, read by the MMAs
      hid_sync();
      if (h == 0) {
        if (leader) {
          mbar_arrive(a1_full);
          // z2 = h1 W2^T once both CTAs' h1 rows are in place
          if (mbar_wait_cluster(a1_full, j & 1)) {
            fence_after();
            mma_k64(tmem + B_ZCOL, hbuf_u, hbuf_u + KB * AK_BYTES, smem_u32(smem + B_OFF_W2),
                    smem_u32(smem + B_OFF_W2 + 4 * B_BK), B_BK, idesc64);
            mma_commit_pair(z2_full);
            issued_any = true;
          } else {
            *vabort = 1;
          }
        } else {
          remote_arrive(a1_full_l);
        }
        // z2 of this tile and dE/dh2 of its head
        const bool ok = !*vabort && mbar_wait(z2_full, j & 1) && mbar_wait(&gh2_full[gb], (j >> 1) & 1);
        if (!ok) *vabort = 1;
        *hid_word = ok ? 1 : 0;
      }
      hid_sync();
      if (!*hid_word) break;
      fence_after();
      // ---- dE/dz2 = dE/dh2 SiLU'(z2): a row and 32 units per thread, into the A buffer (h1 is consumed)
      {
        float z2[32], gh2[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(B_ZCOL + u0), z2);
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(gb * 64 + u0), gh2);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float hi[4], lo[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float v = gh2[4 * c + b] * dsilu_fast(z2[4 * c + b]);
            hi[b] = tf32_rna(v);
            lo[b] = tf32_rna(v - hi[b]);
          }
          const int k = u0 + 4 * c;
          const uint32_t o = (uint32_t)((k >> 4) * AK_BYTES) + swz(row, k & 15);
          *reinterpret_cast<float4*>(hbuf + o) = make_float4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<float4*>(hbuf + KB * AK_BYTES + o) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_before();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      hid_sync();
      if (h == 0) {
        // this CTA's dE/dh2 buffer is read: the head of tile j + 2 may use it
        if (leader) mbar_arrive(&gh2_empty[gb]);
        else remote_arrive(gh2_empty_l + (uint32_t)(gb * 8));
        if (leader) {
          mbar_arrive(a2_full);
          // dE/dh1 = dE/dz2 W2 into the z2 columns (z2 is read in both CTAs)
          if (mbar_wait_cluster(a2_full, j & 1)) {
            fence_after();
            mma_k64(tmem + B_ZCOL, hbuf_u, hbuf_u + KB * AK_BYTES, smem_u32(smem + B_OFF_W2T),
                    smem_u32(smem + B_OFF_W2T + 4 * B_BK), B_BK, idesc64);
            mma_commit_pair(gh1_full);
          } else {
            *vabort = 1;
          }
        } else {
          remote_arrive(a2_full_l);
        }
        const bool ok = !*vabort && mbar_wait(gh1_full, j & 1);
        if (!ok) *vabort = 1;
        *hid_word = ok ? 1 : 0;
      }
      hid_sync();
      if (!*hid_word) break;
      fence_after();
      // ---- dE/dz1 = dE/dh1 SiLU'(z1) (z1 recomputed for this thread's row and units), dE/dd
      {
        float gh1[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(B_ZCOL + u0), gh1);
        const float4 ea = *reinterpret_cast<const float4*>(sE + row * 8);
        const float4 eb = *reinterpret_cast<const float4*>(sE + row * 8 + 4);
        const float4 da = *reinterpret_cast<const float4*>(sDE + row * 8);
        const float4 db = *reinterpret_cast<const float4*>(sDE + row * 8 + 4);
        const float ev[8] = {ea.x, ea.y, ea.z, ea.w, eb.x, eb.y, eb.z, eb.w};
        const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
        float part = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          float z = 0.f, w = 0.f;
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            const float wn = W1T[n * 64 + u0 + k];
            z = fmaf(wn, ev[n], z);
            w = fmaf(wn, dv[n], w);
          }
          part = fmaf(gh1[k] * dsilu_fast(z), w, part);
        }
        sGD[half * BM + row] = part;
      }
      fence_before();
      hid_sync();
      if (h < BM) {
        const int e = sEdge[h];
        if (e >= 0) {
          const float gd = sGD[h] + sGD[BM + h];
          const float inv = 1.f / sD[h];
          g.g_r[3 * e + 0] += gd * g.vec[3 * e + 0] * inv;
          g.g_r[3 * e + 1] += gd * g.vec[3 * e + 1] * inv;
          g.g_r[3 * e + 2] += gd * g.vec[3 * e + 2] * inv;
        }
      }
    }
    if (h == 0 && leader && issued_any) {
      mma_commit_pair(drain2);           // every product this thread issued has completed
      mbar_wait(drain2, 0);
    }
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  if (threadIdx.x == 0 && leader && *vabort) {
    const int peer_issued = remote_load(map_to_rank(smem_u32(issued), 1));
    const int last = max(*issued, peer_issued);
    for (int it = *consumed; it < last; ++it) mbar_wait(&full[it % B_ST], (it / B_ST) & 1);
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)B_TMEM_COLS));
  }
}

// dE/dd of the rows of nsub radial networks (row ranges as in radial_fwd) from dE/dR (hi/lo
// rows [M][4C], kcols of them carrying a gradient); adds (dE/dd) rhat to g_r (by edge).
// a: the dE/dR (hi, lo) maps (boxes of 128 rows); b_maps[s]: network s's W3^T (hi, lo) maps
// (boxes of 32 rows).
inline int radial_bwd(long long M, int kcols, const int* row_off, int nsub, const int* perm, const float* dist,
                      const float* vec, float* g_r, const float* rad, size_t layer_off, size_t pair_stride, float rc,
                      const MapPair& a, const MapPair* const* b_maps, int* counter, cudaStream_t s) {
  if (M <= 0) return EMP_OK;
  if (nsub < 1 || nsub > tc::MAXSUB || M >= (1ll << 31) || kcols < 16 || kcols % 16 != 0) return EMP_ERR_ARG;
  BwdArgs g{};
  BwdMaps maps;
  g.nsub = nsub;
  g.M = (int)M;
  g.mtiles = (int)((M + 2 * BM - 1) / (2 * BM));
  g.kcols = kcols;
  g.row_off = row_off;
  g.counter = counter;
  g.perm = perm;
  g.dist = dist;
  g.vec = vec;
  g.g_r = g_r;
  g.rad = rad;
  g.layer_off = layer_off;
  g.pair_stride = pair_stride;
  g.rc = rc;
  maps.a_hi = a.hi;
  maps.a_lo = a.lo;
  for (int q = 0; q < nsub; ++q) {
    maps.b_hi[q] = b_maps[q]->hi;
    maps.b_lo[q] = b_maps[q]->lo;
  }
  const long long total = (long long)nsub * g.mtiles;
  if (total >= (1ll << 31)) return EMP_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(counter, 0, sizeof(int), s) != cudaSuccess) return EMP_ERR_CUDA;
  const int pairs = (int)std::min<long long>(total, tc::num_sms() / 2);
  k_radial_bwd_tc<<<2 * pairs, B_THREADS, B_SMEM, s>>>(g, maps, (int)total);
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

inline int init() {
  if (cudaFuncSetAttribute(k_radial_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess ||
      cudaFuncSetAttribute(k_radial_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, B_SMEM) != cudaSuccess)
    return EMP_ERR_CUDA;
  return EMP_OK;
}

}  // namespace rtc
}  // namespace emp
