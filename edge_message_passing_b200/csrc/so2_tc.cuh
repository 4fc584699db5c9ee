// Per-m SO(2) channel mixing on the 5th-generation tensor cores (tcgen05, sm_100a)
// in 3xTF32 so that the products keep FP32 accuracy: the pages run the mixing
// in strict FP32 with TF32 off ("first-order SO(2) input-gradient path",
// "Primary capacity": strict level2 mixing FP32, TF32/AMP off), so each operand
// is split a = hi + lo with hi = RN_tf32(a), lo = RN_tf32(a - hi), and
//   Y = A_lo B_hi^T + A_hi B_lo^T + A_hi B_hi^T   (FP32 accumulation in TMEM).
//
// A launch is a group of sub-problems that share the row count M (one cohort):
//   out_s[:, col_s : col_s + K_s] = A_{a(s)}[:, col_s : col_s + K_s] @ B_s^T,
// B_s a (K_s x K_s) matrix stored [n][k] (K-major).  The forward of a layer is
// the 4 m-blocks of the cohort, the backward the 4 transposed blocks; when the
// backward recomputes y (smallest workspace) it groups the 4 forward blocks with
// the 4 transposed blocks (8 sub-problems, two A operands).
//
// Persistent kernel on CTA pairs (clusters of 2, cta_group::2): each pair computes
// 256 x 256 output tiles taken from a shared atomic counter (tiles ordered by
// decreasing K).  In each CTA warp 0 issues TMA loads (128-byte swizzle, 32 fp32 of
// K per row) of its 128 A rows and its half of the B rows, hi and lo, into a 3-stage
// ring of 64 KB stages; the
// even CTA's warp 1 issues tcgen05.mma (one thread) into one of two TMEM
// accumulators (2 x 256 columns) in both CTAs; warps 2..5 of each CTA drain its
// other accumulator with tcgen05.ld and store FP32 rows, so the epilogue of a tile
// overlaps the next tile's MMAs.  Every mbarrier wait is bounded: on timeout the
// CTA records a device error, stops, waits (bounded) for its own copies and MMAs
// and frees TMEM.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <algorithm>
#include "emp_common.cuh"

namespace emp {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 16;                 // fp32 elements per 64-byte swizzled row (the radial kernels' operands)
constexpr int BK2 = 32;                // fp32 elements per 128-byte swizzled row (the grouped products' operands)
constexpr int THREADS = 192;
constexpr int MAXSUB = 8;
constexpr int TMEM_COLS = 512;         // two 128 x 256 fp32 accumulators
constexpr long long TIMEOUT_CYCLES = 4000000000ll;   // default bound of every mbarrier wait: ~2 s at 1.9 GHz
// The bound in force (clock64 cycles); set by emp_set_wait_limit, read by every bounded wait.
__device__ long long g_wait_cycles = TIMEOUT_CYCLES;

constexpr int A_BYTES = BM * BK2 * 4;  // 16 KB: 128 rows of one 32-wide k-block

struct Group {
  int M, nsub, mtiles;
  int a_idx[MAXSUB];    // which A operand pair (0 or 1)
  int b_idx[MAXSUB];    // which B map pair
  int acol[MAXSUB];     // first A column of the sub-problem
  int K[MAXSUB];
  int N[MAXSUB];        // output columns
  int bn[MAXSUB];       // tile width (MMA N): tile_n(N), a multiple of 16 up to 256
  int ccol[MAXSUB];     // first output column
  int ntiles[MAXSUB];   // n-tiles per m-tile
  int first[MAXSUB + 1];// first tile index of each sub-problem (sub-problems ordered by decreasing K)
  int ldc;              // row pitch (elements) of the outputs
  float* out[MAXSUB];
  int* counter;         // dynamic tile counter (zeroed by the host before the launch)
  // null, or device row ranges: sub-problem s covers rows [row_off[s], row_off[s + 1]) of its A
  // operand and output (M and mtiles are then upper bounds; tiles past a range are skipped)
  const int* row_off;
};

struct Maps {
  CUtensorMap a_hi[2], a_lo[2];             // [M rows][ld cols]
  CUtensorMap b_hi[MAXSUB], b_lo[MAXSUB];   // [K rows][K cols]
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait; false (and a device error) if the phase did not complete in time
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > g_wait_cycles) {
      set_device_error(DEV_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tma_load(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// shared-memory matrix descriptor: K-major, 64-byte swizzle, 8-row groups 512 B apart
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(512 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)4 << 61);
}
// the same for 128-byte rows: 128-byte swizzle, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t sdesc128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct TileInfo {
  int m0, sub, n0;
};

constexpr int TQ = 4;    // depth of the tile-index ring from the scheduler to the MMA and epilogue warps

// Tile width (MMA N) of a product with N output columns: N itself up to 256; beyond that
// the widest of 256, 192, 128 that divides N (no padded columns), else 256.
__host__ __device__ constexpr int tile_n(int n) {
  return n <= BN ? n : n % BN == 0 ? BN : n % 192 == 0 ? 192 : n % 128 == 0 ? 128 : BN;
}
// The products run on CTA pairs (cta_group::2); B tensor maps hold half-height tiles.
__host__ __device__ constexpr int b_box_rows(int n) { return tile_n(n) / 2; }

// ------------------------------------------------------------------ 2-SM form (cta_group::2)
// A pair of CTAs (a cluster of 2 on neighbouring SMs) computes a 256 x bn tile with
// one tcgen05.mma.cta_group::2 stream issued by the even CTA (the leader): each CTA
// stages its own 128 rows of A and its own half (bn/2 rows) of B, so each SM reads
// half the B bytes per flop that the 1-SM form does.  Both CTAs' TMA loads complete
// on the leader's full barrier; the MMA completion is multicast to both CTAs' stage
// and accumulator barriers; the leader takes tiles from the counter and publishes
// each index to both CTAs (distributed shared memory + remote mbarrier arrive).
constexpr int ST2 = 3;
constexpr int B2_BYTES = (BN / 2) * BK2 * 4;           // 16 KB: half of a 256-row B tile
constexpr int STAGE2 = 2 * A_BYTES + 2 * B2_BYTES;     // 64 KB per CTA
constexpr int EPI_PITCH = 36;                          // floats per staged row (16-byte aligned, conflict-free)
constexpr int EPI_BYTES = 4 * 32 * EPI_PITCH * 4;      // one 32 x 32 staging tile per epilogue warp
constexpr int SMEM2 = ST2 * STAGE2 + 1024 + 512 + EPI_BYTES;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local_addr), "r"(rank));
  return a;
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void remote_store(uint32_t cluster_addr, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ int remote_load(uint32_t cluster_addr) {
  int v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (clock64() - t0 > g_wait_cycles) {
      set_device_error(DEV_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* map, uint32_t leader_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma_tf32_pair(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
// arrive (once) on the barrier at this address in both CTAs of the pair when the issued MMAs are done
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(smem_u32(bar)), "h"((uint16_t)3)
      : "memory");
}
__host__ __device__ constexpr uint32_t idesc_pair(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ TileInfo tile_info2(const Group& g, int t) {
  TileInfo ti;
  int s = 0;
  while (s < g.nsub - 1 && t >= g.first[s + 1]) ++s;
  const int r = t - g.first[s];
  ti.sub = s;
  ti.m0 = (r / g.ntiles[s]) * (2 * BM);
  ti.n0 = (r % g.ntiles[s]) * g.bn[s];
  return ti;
}

__device__ __forceinline__ int row_base(const Group& g, int sub) { return g.row_off ? g.row_off[sub] : 0; }
__device__ __forceinline__ int row_end(const Group& g, int sub) { return g.row_off ? g.row_off[sub + 1] : g.M; }

// next tile index for the pair: with device row ranges, a tile past its sub-problem's rows is
// dead, and so is every later tile of that sub-problem (m-tiles in order), so the counter jumps
// to the next sub-problem
__device__ __forceinline__ int next_tile(const Group& g, int total) {
  int t = atomicAdd(g.counter, 1);
  while (g.row_off && t < total) {
    const TileInfo ti = tile_info2(g, t);
    if (ti.m0 < row_end(g, ti.sub) - row_base(g, ti.sub)) break;
    atomicMax(g.counter, g.first[ti.sub + 1]);
    t = atomicAdd(g.counter, 1);
  }
  return t;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_so2_tc2(const __grid_constant__ Group g, const __grid_constant__ Maps maps, int total_tiles) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST2 * STAGE2);   // [ST2] (the leader's are used)
  uint64_t* empty = full + ST2;                                        // [ST2]
  uint64_t* acc_full = empty + ST2;                                    // [2]
  uint64_t* acc_empty = acc_full + 2;                                  // [2] (the leader's are used)
  uint64_t* drain = acc_empty + 2;
  uint64_t* tq_full = drain + 1;                                       // [TQ]
  uint64_t* tq_empty = tq_full + TQ;                                   // [TQ] (the leader's are used)
  int* tq = reinterpret_cast<int*>(tq_empty + TQ);                     // [TQ]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq + TQ);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* issued = abort_flag + 1;
  int* consumed = issued + 1;
  float* epi = reinterpret_cast<float*>(smem + ST2 * STAGE2 + 512);   // epilogue staging tiles

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);        // 4 epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    for (int j = 0; j < TQ; ++j) {
      mbar_init(&tq_full[j], 1);
      mbar_init(&tq_empty[j], 10);        // leader MMA + 4 leader epilogue warps + peer producer + 4 peer warps
    }
    *abort_flag = 0;
    *issued = 0;
    *consumed = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* vabort = abort_flag;
  // addresses in the leader CTA (barriers the peer arrives on)
  const uint32_t full_l = map_to_rank(smem_u32(full), 0);
  const uint32_t acc_empty_l = map_to_rank(smem_u32(acc_empty), 0);
  const uint32_t tq_empty_l = map_to_rank(smem_u32(tq_empty), 0);

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- scheduler + TMA producer
    int it = 0;
    for (int j = 0;; ++j) {
      const int slot = j % TQ;
      int t;
      if (leader) {
        if (j >= TQ && !mbar_wait_cluster(&tq_empty[slot], ((j / TQ) - 1) & 1)) { *vabort = 1; t = total_tiles; }
        else t = *vabort ? total_tiles : next_tile(g, total_tiles);
        tq[slot] = t;
        remote_store(map_to_rank(smem_u32(&tq[slot]), 1), t);
        mbar_arrive(&tq_full[slot]);
        remote_arrive(map_to_rank(smem_u32(&tq_full[slot]), 1));
      } else {
        if (!mbar_wait_cluster(&tq_full[slot], (j / TQ) & 1)) { *vabort = 1; break; }
        t = tq[slot];
        remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
      }
      if (t >= total_tiles) break;
      const TileInfo ti = tile_info2(g, t);
      const int a = g.a_idx[ti.sub], b = g.b_idx[ti.sub];
      const int nk = g.K[ti.sub] / BK2;
      const int bh = g.bn[ti.sub] / 2;                       // this CTA's B rows
      for (int kc = 0; kc < nk; ++kc, ++it) {
        const int s = it % ST2;
        if (it >= ST2 && !mbar_wait(&empty[s], ((it / ST2) - 1) & 1)) { *vabort = 1; break; }
        if (*vabort) break;
        unsigned char* st = smem + s * STAGE2;
        if (leader) mbar_expect_tx(&full[s], 2 * (2 * A_BYTES + 2 * bh * BK2 * 4));
        const uint32_t fb = full_l + (uint32_t)(s * 8);
        const int arow = row_base(g, ti.sub) + ti.m0 + (int)rank * BM;
        tma_load_pair(st, &maps.a_hi[a], fb, g.acol[ti.sub] + kc * BK2, arow);
        tma_load_pair(st + A_BYTES, &maps.a_lo[a], fb, g.acol[ti.sub] + kc * BK2, arow);
        tma_load_pair(st + 2 * A_BYTES, &maps.b_hi[b], fb, kc * BK2, ti.n0 + (int)rank * bh);
        tma_load_pair(st + 2 * A_BYTES + B2_BYTES, &maps.b_lo[b], fb, kc * BK2, ti.n0 + (int)rank * bh);
        *issued = it + 1;
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    int it = 0;
    bool ok = true;
    for (int i = 0;; ++i) {
      const int slot = i % TQ;
      if (!mbar_wait(&tq_full[slot], (i / TQ) & 1)) { ok = false; break; }
      const int t = tq[slot];
      mbar_arrive(&tq_empty[slot]);
      if (t >= total_tiles) break;
      const TileInfo ti = tile_info2(g, t);
      const int nk = g.K[ti.sub] / BK2;
      const int buf = i & 1;
      if (i >= 2 && !mbar_wait_cluster(&acc_empty[buf], ((i >> 1) - 1) & 1)) { ok = false; break; }
      fence_after();
      const uint32_t d = tmem + (uint32_t)(buf * BN);
      const uint32_t idesc = idesc_pair(g.bn[ti.sub]);
      for (int kc = 0; kc < nk; ++kc, ++it) {
        const int s = it % ST2;
        if (!mbar_wait(&full[s], (it / ST2) & 1)) { ok = false; break; }
        *consumed = it + 1;
        fence_after();
        const uint32_t a_hi = smem_u32(smem + s * STAGE2);
        const uint32_t a_lo = a_hi + A_BYTES;
        const uint32_t b_hi = a_hi + 2 * A_BYTES;
        const uint32_t b_lo = b_hi + B2_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK2 / 8; ++kk) {
          const uint32_t off = kk * 32;
          mma_tf32_pair(d, sdesc128(a_lo + off), sdesc128(b_hi + off), idesc, (kc | kk) ? 1u : 0u);
          mma_tf32_pair(d, sdesc128(a_hi + off), sdesc128(b_lo + off), idesc, 1u);
          mma_tf32_pair(d, sdesc128(a_hi + off), sdesc128(b_hi + off), idesc, 1u);
        }
        mma_commit_pair(&empty[s]);
      }
      if (!ok) break;
      mma_commit_pair(&acc_full[buf]);
    }
    if (!ok) *vabort = 1;
    mma_commit_pair(drain);
    mbar_wait(drain, 0);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue (both CTAs: own 128 rows)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    for (int i = 0;; ++i) {
      const int slot = i % TQ;
      if (!mbar_wait_cluster(&tq_full[slot], (i / TQ) & 1)) { *vabort = 1; break; }
      const int t = tq[slot];
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(&tq_empty[slot]);
        else remote_arrive(tq_empty_l + (uint32_t)(slot * 8));
      }
      if (t >= total_tiles) break;
      const TileInfo ti = tile_info2(g, t);
      const int buf = i & 1;
      if (!mbar_wait(&acc_full[buf], (i >> 1) & 1)) { *vabort = 1; break; }
      fence_after();
      // 32 x 32 chunks: TMEM -> registers (a row per thread) -> this warp's staging tile ->
      // rows stored 8 threads x 16 bytes at a time, so every store writes whole 128-byte segments
      const int mw = row_base(g, ti.sub) + ti.m0 + (int)rank * BM + q * 32;
      const int mend = row_end(g, ti.sub);
      const int N = g.N[ti.sub], bn = g.bn[ti.sub];
      float* obase = g.out[ti.sub] + (size_t)g.ccol[ti.sub] + ti.n0;
      float* stg = epi + q * 32 * EPI_PITCH;
      (void)row;
#pragma unroll 1
      for (int cc = 0; cc < bn; cc += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + cc), v);
        if (ti.n0 + cc < N) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(stg + lane * EPI_PITCH + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int rr = k * 4 + (lane >> 3), c4 = (lane & 7) * 4;
            const int m = mw + rr;
            const float4 w = *reinterpret_cast<const float4*>(stg + rr * EPI_PITCH + c4);
            if (m < mend) *reinterpret_cast<float4*>(obase + (size_t)m * g.ldc + cc + c4) = w;
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
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  if (threadIdx.x == 0 && leader && *vabort) {
    // let loads of either CTA still in flight land (they complete on the leader's barriers)
    const int peer_issued = remote_load(map_to_rank(smem_u32(issued), 1));
    const int last = max(*issued, peer_issued);
    for (int it = *consumed; it < last; ++it) mbar_wait(&full[it % ST2], (it / ST2) & 1);
  }
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)TMEM_COLS));
  }
}

// ------------------------------------------------------------------ tensor-pipe rate
// The ceiling the SO(2) products are measured against: each CTA pair issues `iters` rounds of
// the product kernel's k-stage (for each of the four 8-wide k-steps of a 32-column stage, the
// three 3xTF32 products tcgen05.mma.cta_group::2.kind::tf32 of M = 256, N = 256, K = 8) on
// operands resident in shared memory, into one TMEM accumulator, then commits once and waits
// (bounded).  The operands are pseudo-random values of ordinary magnitude so that the pipe
// switches as it does on real data.
constexpr int RATE_COLS = 256;
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1) k_tf32_rate(int iters, unsigned seed) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + STAGE2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = cluster_rank();
  float* f = reinterpret_cast<float*>(smem);
  for (int i = threadIdx.x; i < STAGE2 / 4; i += blockDim.x) {
    uint32_t h = (uint32_t)i * 2654435761u ^ (seed + 97u * rank + 7919u * blockIdx.x);
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    f[i] = (float)(h & 0xffffu) * (1.0f / 32768.0f) - 1.0f;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // operands written by threads, read by the MMAs
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)RATE_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  cluster_sync();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  if (rank == 0 && threadIdx.x == 0) {
    const uint32_t a_hi = smem_u32(smem), a_lo = a_hi + A_BYTES, b_hi = a_hi + 2 * A_BYTES, b_lo = b_hi + B2_BYTES;
    const uint32_t idesc = idesc_pair(BN);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < BK2 / 8; ++kk) {
        const uint32_t off = kk * 32;
        mma_tf32_pair(tmem, sdesc128(a_lo + off), sdesc128(b_hi + off), idesc, (it | kk) ? 1u : 0u);
        mma_tf32_pair(tmem, sdesc128(a_hi + off), sdesc128(b_lo + off), idesc, 1u);
        mma_tf32_pair(tmem, sdesc128(a_hi + off), sdesc128(b_hi + off), idesc, 1u);
      }
    }
    mma_commit_pair(done);              // arrives on `done` in both CTAs when every MMA has completed
  }
  if (threadIdx.x == 0) mbar_wait(done, 0);
  fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)RATE_COLS));
  }
}
constexpr int RATE_SMEM = STAGE2 + 1024 + 64;

// ------------------------------------------------------------------ host side
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// box_cols 16 with the 64-byte swizzle (the radial kernels' operands) or 32 with the 128-byte
// swizzle (the grouped products' operands)
inline bool make_map(CUtensorMap* m, const float* base, uint64_t cols, uint64_t rows, uint64_t row_pitch_elems,
                     uint32_t box_rows, uint32_t box_cols = BK) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_pitch_elems * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == BK2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace tc

inline int so2_tc_init() {
  if (!tc::encode_fn()) return EMP_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(tc::k_so2_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM2) != cudaSuccess ||
      cudaFuncSetAttribute(tc::k_tf32_rate, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::RATE_SMEM) != cudaSuccess)
    return EMP_ERR_CUDA;
  return EMP_OK;
}

// One plain product on the tensor cores (3xTF32): out[:, ccol + n] = sum_k A[:, acol + k] B[n][k].
struct GemmSub {
  const CUtensorMap* a_hi;
  const CUtensorMap* a_lo;
  const CUtensorMap* b_hi;
  const CUtensorMap* b_lo;
  int acol, K, N, ccol;
  float* out;
};

// Launch a group of products sharing the row count M (at most two distinct A operands).
// Sub-problems are reordered by decreasing K; counter: one device int, zeroed here.  With
// row_off (device, nsub + 1 entries in the subs' given order), sub-problem s covers rows
// [row_off[s], row_off[s + 1]) only, M being an upper bound of every range.
inline int tc_group(long long M, int ldc, const GemmSub* subs, int nsub, int* counter, cudaStream_t s,
                    const int* row_off = nullptr) {
  if (M <= 0) return EMP_OK;
  if (nsub < 1 || nsub > tc::MAXSUB || M >= (1ll << 31)) return EMP_ERR_ARG;
  tc::Group g{};
  tc::Maps maps;
  g.M = (int)M;
  g.row_off = row_off;
  g.ldc = ldc;
  g.nsub = nsub;
  g.mtiles = (int)((M + 2 * tc::BM - 1) / (2 * tc::BM));
  g.counter = counter;
  int ord[tc::MAXSUB];
  for (int i = 0; i < nsub; ++i) ord[i] = i;
  if (!row_off)        // with device row ranges the subs keep their order (row_off is indexed by it)
    std::stable_sort(ord, ord + nsub, [&](int a, int b) { return subs[a].K > subs[b].K; });
  const CUtensorMap* a_seen[2] = {nullptr, nullptr};
  int na = 0;
  long long first = 0;
  for (int q = 0; q < nsub; ++q) {
    const GemmSub& u = subs[ord[q]];
    if (u.K % tc::BK2 != 0 || u.N < 32 || u.N % 32 != 0) return EMP_ERR_ARG;
    int a = 0;
    while (a < na && a_seen[a] != u.a_hi) ++a;
    if (a == na) {
      if (na == 2) return EMP_ERR_ARG;
      a_seen[na] = u.a_hi;
      maps.a_hi[na] = *u.a_hi;
      maps.a_lo[na] = *u.a_lo;
      ++na;
    }
    maps.b_hi[q] = *u.b_hi;
    maps.b_lo[q] = *u.b_lo;
    g.a_idx[q] = a;
    g.b_idx[q] = q;
    g.acol[q] = u.acol;
    g.K[q] = u.K;
    g.N[q] = u.N;
    g.bn[q] = tc::tile_n(u.N);
    g.ccol[q] = u.ccol;
    g.ntiles[q] = (u.N + g.bn[q] - 1) / g.bn[q];
    g.out[q] = u.out;
    g.first[q] = (int)first;
    first += (long long)g.ntiles[q] * g.mtiles;
  }
  if (first >= (1ll << 31)) return EMP_ERR_UNSUPPORTED;
  g.first[nsub] = (int)first;
  if (cudaMemsetAsync(counter, 0, sizeof(int), s) != cudaSuccess) return EMP_ERR_CUDA;
  const int pairs = (int)std::min<long long>(first, tc::num_sms() / 2);
  tc::k_so2_tc2<<<2 * pairs, tc::THREADS, tc::SMEM2, s>>>(g, maps, (int)first);
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

// Tensor maps (hi, lo) of a row-major fp32 matrix [rows][cols] with row pitch ld,
// tiles of box_rows rows (BM for A operands, min(N, 256) / 2 for B operands): make_pair for the
// radial kernels (16-column boxes), make_pair128 for the grouped products (32-column boxes).
struct MapPair {
  CUtensorMap hi, lo;
};
inline int make_pair(MapPair* m, const float* hi, const float* lo, long long rows, int cols, int ld, int box_rows,
                     int box_cols = tc::BK) {
  if (!tc::make_map(&m->hi, hi, cols, rows, ld, box_rows, box_cols)) return EMP_ERR_CUDA;
  if (!tc::make_map(&m->lo, lo, cols, rows, ld, box_rows, box_cols)) return EMP_ERR_CUDA;
  return EMP_OK;
}
inline int make_pair128(MapPair* m, const float* hi, const float* lo, long long rows, int cols, int ld, int box_rows) {
  return make_pair(m, hi, lo, rows, cols, ld, box_rows, tc::BK2);
}

// Tensor maps of one operand set of the SO(2) mixing: A (hi, lo) rows [M][16C] and a
// layer's stacked 4-block weights (hi, lo).  Built once (weights: at model
// creation; activations: once per call and cohort size) and reused by every launch.
struct So2BMaps {
  MapPair blk[4];
};
typedef MapPair So2AMaps;

inline int so2_make_bmaps(So2BMaps* m, int C, const float* b_hi, const float* b_lo) {
  for (int b = 0; b < 4; ++b) {
    const int K = blk_width(b) * C;
    const size_t off = (size_t)wblk_off(b) * C * C;
    int st = make_pair128(&m->blk[b], b_hi + off, b_lo + off, K, K, K, tc::b_box_rows(K));
    if (st != EMP_OK) return st;
  }
  return EMP_OK;
}

inline int so2_make_amaps(So2AMaps* m, int C, long long M, const float* a_hi, const float* a_lo) {
  return make_pair128(m, a_hi, a_lo, M, 16 * C, 16 * C, tc::BM);
}

struct So2Part {
  const So2AMaps* a;
  const So2BMaps* b;
  float* out;
};

// SO(2) mixing of a cohort: one operand set (forward) or two sharing the rows (backward).
inline int so2_tc(long long M, int C, const So2Part* parts, int nparts, int* counter, cudaStream_t s) {
  if (nparts < 1 || nparts > 2) return EMP_ERR_ARG;
  GemmSub subs[tc::MAXSUB];
  int n = 0;
  for (int p = 0; p < nparts; ++p)
    for (int b = 0; b < 4; ++b, ++n) {
      const int K = blk_width(b) * C;
      subs[n] = GemmSub{&parts[p].a->hi, &parts[p].a->lo, &parts[p].b->blk[b].hi, &parts[p].b->blk[b].lo,
                        blk_off(b) * C, K, K, blk_off(b) * C, parts[p].out};
    }
  return tc_group(M, 16 * C, subs, n, counter, s);
}

}  // namespace emp
