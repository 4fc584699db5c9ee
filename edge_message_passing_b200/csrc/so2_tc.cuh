// Per-m SO(2) channel mixing on the 5th-generation tensor cores (tcgen05, sm_100a)
// in 3xTF32 so that the products keep FP32 accuracy: the pages run the mixing
// in strict FP32 with TF32 off ("first-order SO(2) input-gradient path",
// "Primary capacity": strict level2 mixing FP32, TF32/AMP off), so each operand
// is split a = hi + lo with hi = RN_tf32(a), lo = RN_tf32(a - hi), and
//   Y = A_hi B_hi^T + A_hi B_lo^T + A_lo B_hi^T   (FP32 accumulation in TMEM).
//
// For block b (= |m|) of a cohort:  Y[:, cols_b] = X[:, cols_b] @ B_b^T with
// B_b the (K_b x K_b) stacked weight stored [n][k] (K-major), K_b = blk_width(b) C.
//
// One CTA computes a 128 x BN output tile of one block.  Warp 0 issues TMA
// loads (128B-swizzled, 32 fp32 of K per row) into an ST-stage ring guarded by
// mbarriers; warp 1 allocates TMEM and issues tcgen05.mma (one thread);
// warps 2..5 read the accumulator back with tcgen05.ld and store FP32 rows.
// Every mbarrier wait is bounded: on timeout the CTA records a device error,
// drains what it issued and frees its TMEM.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include "emp_common.cuh"

namespace emp {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 32;                 // fp32 elements per 128-byte swizzled row
constexpr int BN = 128;
constexpr int ST = 3;
constexpr int THREADS = 192;
constexpr long long TIMEOUT_CYCLES = 4000000000ll;   // ~2 s at 1.9 GHz

constexpr int A_BYTES = BM * BK * 4;   // 16 KB
constexpr int B_BYTES = BN * BK * 4;   // 16 KB
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
constexpr int SMEM_BYTES = ST * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct Maps {
  CUtensorMap a_hi, a_lo;       // [M rows][16C cols]
  CUtensorMap b_hi[4], b_lo[4]; // block b: [K_b rows][K_b cols]
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
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
    if (clock64() - t0 > TIMEOUT_CYCLES) {
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

// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// instruction descriptor: D f32, A/B tf32, both K-major, M = 128, N = BN
constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(IDESC), "r"(accum));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
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

// n-tile index -> (block b, first output column of the tile within the block)
__device__ __forceinline__ void tile_of(int C, int y, int& b, int& n0) {
  for (b = 0; b < 4; ++b) {
    const int nt = (blk_width(b) * C + BN - 1) / BN;
    if (y < nt) { n0 = y * BN; return; }
    y -= nt;
  }
  b = -1;
  n0 = 0;
}

__global__ void __launch_bounds__(THREADS, 1) k_so2_tc(int M, int C, const __grid_constant__ Maps maps,
                                                       float* __restrict__ Y) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * STAGE_BYTES);
  uint64_t* empty = full + ST;
  uint64_t* acc_bar = empty + ST;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, n0;
  tile_of(C, blockIdx.y, b, n0);
  if (b < 0) return;
  const int K = blk_width(b) * C, N = K;
  const int m0 = blockIdx.x * BM;
  const int col0 = blk_off(b) * C;      // column offset of the block in the 16C-wide rows
  const int nk = K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)BN));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % ST;
      if (kc >= ST && !mbar_wait(&empty[s], ((kc / ST) - 1) & 1)) { atomicExch(abort_flag, 1); break; }
      if (*(volatile int*)abort_flag) break;
      unsigned char* st = smem + s * STAGE_BYTES;
      mbar_expect_tx(&full[s], STAGE_BYTES);
      tma_load(st, &maps.a_hi, &full[s], col0 + kc * BK, m0);
      tma_load(st + A_BYTES, &maps.a_lo, &full[s], col0 + kc * BK, m0);
      tma_load(st + 2 * A_BYTES, &maps.b_hi[b], &full[s], kc * BK, n0);
      tma_load(st + 2 * A_BYTES + B_BYTES, &maps.b_lo[b], &full[s], kc * BK, n0);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    bool ok = true;
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % ST;
      if (!mbar_wait(&full[s], (kc / ST) & 1)) { ok = false; atomicExch(abort_flag, 1); break; }
      fence_after();
      const uint32_t a_hi = smem_u32(smem + s * STAGE_BYTES);
      const uint32_t a_lo = a_hi + A_BYTES;
      const uint32_t b_hi = a_hi + 2 * A_BYTES;
      const uint32_t b_lo = b_hi + B_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 8; ++kk) {
        const uint32_t off = kk * 32;   // 8 fp32 of K = 32 bytes inside the swizzled row
        const uint32_t acc = (kc | kk) ? 1u : 0u;
        mma_tf32(tmem, sdesc(a_lo + off), sdesc(b_hi + off), acc);
        mma_tf32(tmem, sdesc(a_hi + off), sdesc(b_lo + off), 1u);
        mma_tf32(tmem, sdesc(a_hi + off), sdesc(b_hi + off), 1u);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(ok ? acc_bar : drain_bar);
    if (!ok) mbar_wait(drain_bar, 0);     // let issued MMAs finish before TMEM is freed
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;               // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const bool ok = mbar_wait(acc_bar, 0);
    fence_after();
    if (ok) {
      const int m = m0 + row;
      float* yrow = Y + (size_t)m * 16 * C + col0 + n0;
#pragma unroll 1
      for (int cc = 0; cc < BN; cc += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)cc, v);
        if (m < M && n0 + cc < N) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(yrow + cc + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // wait (bounded) for loads that may still be landing in shared memory
    for (int s = 0; s < ST; ++s) mbar_try_wait(&full[s], 0);
  }
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)BN));
  }
}

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

inline bool make_map(CUtensorMap* m, const float* base, uint64_t cols, uint64_t rows, uint64_t row_pitch_elems,
                     uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_pitch_elems * 4};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

inline int so2_tc_init() {
  if (!tc::encode_fn()) return EMP_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(tc::k_so2_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES) != cudaSuccess)
    return EMP_ERR_CUDA;
  return EMP_OK;
}

inline int so2_tc_tiles(int C) {
  int n = 0;
  for (int b = 0; b < 4; ++b) n += (blk_width(b) * C + tc::BN - 1) / tc::BN;
  return n;
}

// Y (M x 16C) = per-block products of A (M x 16C) with the layer's stacked weights (split hi/lo)
inline int so2_tc(long long M, int C, const float* A_hi, const float* A_lo, const float* B_hi, const float* B_lo,
                  float* Y, cudaStream_t s) {
  if (M <= 0) return EMP_OK;
  tc::Maps maps;
  if (!tc::make_map(&maps.a_hi, A_hi, 16 * C, M, 16 * C, tc::BM)) return EMP_ERR_CUDA;
  if (!tc::make_map(&maps.a_lo, A_lo, 16 * C, M, 16 * C, tc::BM)) return EMP_ERR_CUDA;
  for (int b = 0; b < 4; ++b) {
    const uint64_t K = (uint64_t)blk_width(b) * C;
    const size_t off = (size_t)wblk_off(b) * C * C;
    if (!tc::make_map(&maps.b_hi[b], B_hi + off, K, K, K, tc::BN)) return EMP_ERR_CUDA;
    if (!tc::make_map(&maps.b_lo[b], B_lo + off, K, K, K, tc::BN)) return EMP_ERR_CUDA;
  }
  dim3 grid((unsigned)((M + tc::BM - 1) / tc::BM), so2_tc_tiles(C));
  tc::k_so2_tc<<<grid, tc::THREADS, tc::SMEM_BYTES, s>>>((int)M, C, maps, Y);
  return cudaGetLastError() == cudaSuccess ? EMP_OK : EMP_ERR_CUDA;
}

}  // namespace emp
