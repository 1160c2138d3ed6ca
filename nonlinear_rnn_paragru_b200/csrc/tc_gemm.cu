// tc_gemm.cu -- batched fp32 matrix products on the 5th-generation tensor
// cores: C[z] = A[z] B[z]^T, A[z] M x K and B[z] N x K row-major (both
// K-major), fp32 in memory, tf32 multiplies (tcgen05.mma kind::tf32) with
// fp32 accumulation in tensor memory.
//
// These are the contractions of the dense-Jacobian Newton solve: the
// recurrent pre-activations (states times the stacked recurrent matrices) and
// the products of D x D Jacobian blocks that compose the scan's chunk maps
// ("Параллельность RNN?", §1.3: a general cell's Jacobian blocks are full
// D x D matrices, and composing two steps of the linear recurrence multiplies
// them).
//
// One CTA of 4 warps per 128 x 128 output tile of one z:
//   thread 0   issues the TMA loads of 32-wide K slices of A and B (128-byte
//              swizzle: one slice row is one 128-byte swizzle row) into a
//              3-stage ring, each stage completing on its mbarrier;
//   thread 32  issues 4 tcgen05.mma per slice (K = 8 each), accumulating in a
//              128-lane x 128-column tensor-memory tile, and commits each
//              stage back to the producer and, at the end, to the epilogue;
//   all warps  read the accumulator (warp w owns lanes 32w..32w+31, i.e.
//              output rows) with tcgen05.ld and store it to C, row-major or
//              transposed per z (store_mode).
// Every wait is bounded: a wait that runs out sets *err, the CTA skips its
// stores, and it frees its tensor memory before returning.  Loads past the
// matrices' edges read zeros (TMA out-of-bounds fill); stores are masked.
//
// Large launches (at least one 128 x 256 output tile per SM) take the
// persistent form instead, one CTA per SM working off tiles in a fixed
// order: 128 x 256 tiles (a third less operand traffic per product than
// 128 x 128), a 4-stage ring of 48 KB stages, and two 128 x 256 accumulators
// in tensor memory (all 512 columns), so the epilogue of one tile overlaps
// the products of the next.  Warp 0 loads, warp 1 issues the products,
// warps 2-5 (tensor-memory lane quarters 2, 3, 0, 1) read the accumulators
// and store.
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"

namespace pararnn {

namespace {

constexpr int kTcBM = 128, kTcBN = 128;
constexpr int kTcBK = 32;  // fp32 elements per K slice: one 128-byte swizzle row
constexpr int kTcStages = 3;
constexpr int kTcABytes = kTcBM * kTcBK * 4;
constexpr int kTcBBytes = kTcBN * kTcBK * 4;
constexpr int kTcStageBytes = kTcABytes + kTcBBytes;
constexpr int kTcSmem = kTcStages * kTcStageBytes + 1024;  // + alignment slack
constexpr int kTcThreads = 128;
constexpr uint32_t kTcCols = 128;  // tensor-memory columns (fp32 accumulator, N = 128)
constexpr uint64_t kTcTimeoutNs = 2000000000ull;

// instruction descriptor: fp32 accumulator, tf32 A and B, both K-major,
// N = 128, M = 128
constexpr uint32_t kTcIdesc = (1u << 4) | (2u << 7) | (2u << 10) |
                              ((uint32_t)(kTcBN >> 3) << 17) | ((uint32_t)(kTcBM >> 4) << 24);

struct TcParams {
  float* C;
  int M, N, K, Z;
  int store_mode;  // 0: C[z] row-major M x N; 1: C[z] transposed (N x M);
                   // 2: row-major for odd z, transposed for even z;
                   // 3: C[z] row-major, the product added to what C holds
  int* err;        // set to 1 by a CTA whose wait ran out
};

// shared-memory matrix descriptor of a K-major operand tile with 128-byte
// swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)1u << 16;                           // leading byte offset (16 B units)
  d |= (uint64_t)(1024u >> 4) << 32;                 // stride byte offset: 8-row groups
  d |= (uint64_t)1u << 46;                           // descriptor version
  d |= (uint64_t)2u << 61;                           // 128-byte swizzle
  return d;
}

__device__ __forceinline__ void tc_mma(uint32_t tmem, uint64_t da, uint64_t db, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
      "l"(da), "l"(db), "r"(kTcIdesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 32 consecutive accumulator columns of this warp's 32 lanes
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TcShared {
  uint64_t full[kTcStages], empty[kTcStages], done;
  uint32_t tmem;
  int fail;
};

__global__ void __launch_bounds__(kTcThreads, 2)
    tc_gemm_tf32(const __grid_constant__ CUtensorMap ma, const __grid_constant__ CUtensorMap mb,
                 const TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ TcShared sh;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 1-D grid: z outermost, then the n tile, then the m tile
  const int tm = (p.M + kTcBM - 1) / kTcBM, tn = (p.N + kTcBN - 1) / kTcBN;
  const int z = blockIdx.x / (tm * tn), rem = blockIdx.x - z * (tm * tn);
  const int m0 = (rem % tm) * kTcBM, n0 = (rem / tm) * kTcBN;
  const int nk = (p.K + kTcBK - 1) / kTcBK;

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    mbar_init(&sh.done, 1);
    sh.fail = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sh.tmem)),
                 "r"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;

  if (tid == 0) {
    // producer: the K slices of A (rows m0..) and B (rows n0..) into the ring
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kTcStages;
      if (kb >= kTcStages &&
          !mbar_wait_bounded(&sh.empty[s], ((kb / kTcStages) - 1) & 1, kTcTimeoutNs)) {
        sh.fail = 1;
        break;
      }
      unsigned char* st = smem + s * kTcStageBytes;
      mbar_arrive_expect_tx(&sh.full[s], (unsigned)kTcStageBytes);
      tma_load_3d(st, &ma, &sh.full[s], kb * kTcBK, m0, z);
      tma_load_3d(st + kTcABytes, &mb, &sh.full[s], kb * kTcBK, n0, z);
    }
  } else if (tid == 32) {
    // MMA issuer
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kTcStages;
      if (!mbar_wait_bounded(&sh.full[s], (kb / kTcStages) & 1, kTcTimeoutNs)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * kTcStageBytes), b0 = a0 + kTcABytes;
#pragma unroll
      for (int k = 0; k < kTcBK / 8; ++k)  // K = 8 tf32 (32 bytes) per instruction
        tc_mma(tmem, tc_sdesc(a0 + k * 32), tc_sdesc(b0 + k * 32), (kb | k) != 0);
      tc_commit(&sh.empty[s]);  // the stage is free once these products are done
    }
    if (!ok) sh.fail = 1;
    tc_commit(&sh.done);  // every product issued so far is done
  }
  // epilogue
  __syncwarp();
  bool ok = mbar_wait_bounded(&sh.done, 0, kTcTimeoutNs);
  tc_fence_after();
  __syncthreads();
  ok = ok && sh.fail == 0;
  if (!ok) {
    if (tid == 0) atomicExch(p.err, 1);
  } else {
    const int row = m0 + warp * 32 + lane;
    const bool trans = p.store_mode == 1 || (p.store_mode == 2 && (z & 1) == 0);
    float* Cz = p.C + (size_t)z * p.M * p.N;
#pragma unroll 1
    for (int c0 = 0; c0 < kTcBN; c0 += 32) {
      if (n0 + c0 >= p.N) break;
      uint32_t r[32];
      tc_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, r);
      if (row < p.M) {
        if (trans) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = n0 + c0 + j;
            if (col < p.N) Cz[(size_t)col * p.M + row] = __uint_as_float(r[j]);
          }
        } else if (p.store_mode == 3) {
          float* dst = Cz + (size_t)row * p.N + n0 + c0;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (n0 + c0 + j < p.N) dst[j] += __uint_as_float(r[j]);
        } else {
          float* dst = Cz + (size_t)row * p.N + n0 + c0;
          if (n0 + c0 + 32 <= p.N && (p.N & 3) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + j) =
                  make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                              __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + c0 + j < p.N) dst[j] = __uint_as_float(r[j]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols)
                 : "memory");
}

// ------------------------------------------------------ persistent form --
constexpr int kPgBM = 128, kPgBN = 256;
constexpr int kPgStages = 4;
constexpr int kPgABytes = kPgBM * kTcBK * 4;                  // 16384
constexpr int kPgBBytes = kPgBN * kTcBK * 4;                  // 32768: two 128-row boxes
constexpr int kPgStageBytes = kPgABytes + kPgBBytes;
constexpr int kPgSmem = kPgStages * kPgStageBytes + 1024;     // + alignment slack
constexpr int kPgThreads = 192;
constexpr uint32_t kPgCols = 512;                              // two fp32 accumulators, N = 256
constexpr uint32_t kPgIdesc = (1u << 4) | (2u << 7) | (2u << 10) |
                              ((uint32_t)(kPgBN >> 3) << 17) | ((uint32_t)(kPgBM >> 4) << 24);
static_assert(kPgBN % kTcBM == 0, "the B tile is whole boxes of the operand map");

struct PgShared {
  uint64_t full[kPgStages], empty[kPgStages];
  uint64_t acc_full[2], acc_empty[2], done;
  uint32_t tmem;
  int fail;
};

__device__ __forceinline__ void pg_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool pg_failed(const PgShared& sh) {
  return *reinterpret_cast<const volatile int*>(&sh.fail) != 0;
}
__device__ __forceinline__ void pg_fail(PgShared& sh) {
  *reinterpret_cast<volatile int*>(&sh.fail) = 1;
}
__device__ __forceinline__ void pg_mma(uint32_t tmem, uint64_t da, uint64_t db, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
      "l"(da), "l"(db), "r"(kPgIdesc), "r"(acc)
      : "memory");
}

__global__ void __launch_bounds__(kPgThreads, 1)
    tc_gemm_tf32_persistent(const __grid_constant__ CUtensorMap ma,
                            const __grid_constant__ CUtensorMap mb, const TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ PgShared sh;
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tm = (p.M + kPgBM - 1) / kPgBM, tn = (p.N + kPgBN - 1) / kPgBN;
  const int ntiles = tm * tn * p.Z;
  const int nk = (p.K + kTcBK - 1) / kTcBK;

  if (tid == 0) {
    for (int s = 0; s < kPgStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh.acc_full[a], 1);
      mbar_init(&sh.acc_empty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(&sh.done, 1);
    sh.fail = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&sh.tmem)),
                 "r"(kPgCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;

  if (warp == 0) {
    if (lane == 0) {
      // producer: every tile's K slices into the ring
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !pg_failed(sh); tile += gridDim.x) {
        const int z = tile / (tm * tn), rem = tile - z * (tm * tn);
        const int m0 = (rem % tm) * kPgBM, n0 = (rem / tm) * kPgBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPgStages;
          if (it >= kPgStages &&
              !mbar_wait_bounded(&sh.empty[s], ((it / kPgStages) - 1) & 1, kTcTimeoutNs)) {
            pg_fail(sh);
            break;
          }
          unsigned char* st = smem + s * kPgStageBytes;
          mbar_arrive_expect_tx(&sh.full[s], (unsigned)kPgStageBytes);
          tma_load_3d(st, &ma, &sh.full[s], kb * kTcBK, m0, z);
#pragma unroll
          for (int h = 0; h < kPgBN / kTcBM; ++h)
            tma_load_3d(st + kPgABytes + h * kTcBM * kTcBK * 4, &mb, &sh.full[s], kb * kTcBK,
                        n0 + h * kTcBM, z);
        }
      }
      // loads still in flight (a failed run): wait for them, bounded
      if (pg_failed(sh))
        for (int back = 1; back <= kPgStages && it - back >= 0; ++back) {
          const int j = it - back;
          mbar_wait_bounded(&sh.full[j % kPgStages], (j / kPgStages) & 1, kTcTimeoutNs);
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // products: a tile into accumulator j & 1, once the epilogue has read
      // what that accumulator held two tiles before
      int it = 0, j = 0;
      for (int tile = blockIdx.x; tile < ntiles && !pg_failed(sh); tile += gridDim.x, ++j) {
        const int ab = j & 1;
        if (j >= 2 && !mbar_wait_bounded(&sh.acc_empty[ab], ((j >> 1) - 1) & 1, kTcTimeoutNs)) {
          pg_fail(sh);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * kPgBN);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPgStages;
          if (!mbar_wait_bounded(&sh.full[s], (it / kPgStages) & 1, kTcTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kPgStageBytes), b0 = a0 + kPgABytes;
#pragma unroll
          for (int k = 0; k < kTcBK / 8; ++k)  // K = 8 tf32 (32 bytes) per instruction
            pg_mma(d, tc_sdesc(a0 + k * 32), tc_sdesc(b0 + k * 32), (kb | k) != 0);
          tc_commit(&sh.empty[s]);  // the stage is free once these products are done
        }
        if (!ok) {
          pg_fail(sh);
          break;
        }
        tc_commit(&sh.acc_full[ab]);
      }
      tc_commit(&sh.done);  // every product issued is done
    }
  } else {
    // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (rows)
    const int eq = warp & 3;
    const bool trans_all = p.store_mode == 1;
    int j = 0;
    for (int tile = blockIdx.x; tile < ntiles && !pg_failed(sh); tile += gridDim.x, ++j) {
      const int ab = j & 1;
      if (!mbar_wait_bounded(&sh.acc_full[ab], (j >> 1) & 1, kTcTimeoutNs)) {
        pg_fail(sh);
        break;
      }
      tc_fence_after();
      const int z = tile / (tm * tn), rem = tile - z * (tm * tn);
      const int m0 = (rem % tm) * kPgBM, n0 = (rem / tm) * kPgBN;
      const int row = m0 + eq * 32 + lane;
      const bool trans = trans_all || (p.store_mode == 2 && (z & 1) == 0);
      float* Cz = p.C + (size_t)z * p.M * p.N;
#pragma unroll 1
      for (int c0 = 0; c0 < kPgBN; c0 += 32) {
        if (n0 + c0 >= p.N) break;
        uint32_t r[32];
        tc_ld32(tmem + ((uint32_t)(eq * 32) << 16) + (uint32_t)(ab * kPgBN + c0), r);
        if (row < p.M) {
          if (trans) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int col = n0 + c0 + jj;
              if (col < p.N) Cz[(size_t)col * p.M + row] = __uint_as_float(r[jj]);
            }
          } else if (p.store_mode == 3) {
            float* dst = Cz + (size_t)row * p.N + n0 + c0;
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (n0 + c0 + jj < p.N) dst[jj] += __uint_as_float(r[jj]);
          } else {
            float* dst = Cz + (size_t)row * p.N + n0 + c0;
            if (n0 + c0 + 32 <= p.N && (p.N & 3) == 0) {
#pragma unroll
              for (int jj = 0; jj < 32; jj += 4)
                *reinterpret_cast<float4*>(dst + jj) =
                    make_float4(__uint_as_float(r[jj]), __uint_as_float(r[jj + 1]),
                                __uint_as_float(r[jj + 2]), __uint_as_float(r[jj + 3]));
            } else {
#pragma unroll
              for (int jj = 0; jj < 32; ++jj)
                if (n0 + c0 + jj < p.N) dst[jj] = __uint_as_float(r[jj]);
            }
          }
        }
      }
      // this warp has read its quarter of the accumulator: the products may
      // reuse it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pg_arrive(&sh.acc_empty[ab]);
    }
  }
  // every product done before the tensor memory goes back (bounded)
  if (tid == 0 && !mbar_wait_bounded(&sh.done, 0, kTcTimeoutNs)) pg_fail(sh);
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && sh.fail) atomicExch(p.err, 1);
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPgCols)
                 : "memory");
}

PFN_cuTensorMapEncodeTiled_v12000 tc_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

// Tensor map over `rows` x K fp32 matrices, Z of them `zstride` floats apart,
// with 32 x 128 boxes and 128-byte swizzle (the operand layout of tc_gemm).
// base and zstride * 4 must be 16-byte multiples, K a multiple of 4.
int tc_operand_map(CUtensorMap* map, const float* base, int K, int rows, int Z, long long zstride) {
  auto fn = tc_encode();
  if (fn == nullptr) return 1;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)Z};
  cuuint64_t strides[2] = {(cuuint64_t)K * 4, (cuuint64_t)zstride * 4};
  cuuint32_t box[3] = {(cuuint32_t)kTcBK, (cuuint32_t)kTcBM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : 1;
}

// C[z] = A[z] B[z]^T for z < Z through the operand maps of tc_operand_map
// (A: M rows, B: N rows, both K wide).  Returns 0 or a CUDA error.
int launch_tc_gemm(const CUtensorMap& ma, const CUtensorMap& mb, float* C, int M, int N, int K,
                   int Z, int store_mode, int* err, cudaStream_t stream) {
  static_assert(kTcBM == kTcBN, "one box shape serves both operands");
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_tf32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kTcSmem);
  if (e != cudaSuccess) return (int)e;
  TcParams p;
  p.C = C;
  p.M = M;
  p.N = N;
  p.K = K;
  p.Z = Z;
  p.store_mode = store_mode;
  p.err = err;
  const long long tiles = (long long)((M + kTcBM - 1) / kTcBM) * ((N + kTcBN - 1) / kTcBN) * Z;
  if (tiles >= (1LL << 31)) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long ptiles = (long long)((M + kPgBM - 1) / kPgBM) * ((N + kPgBN - 1) / kPgBN) * Z;
  if (ptiles >= sms) {  // the persistent form: one CTA per SM
    e = cudaFuncSetAttribute(tc_gemm_tf32_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPgSmem);
    if (e != cudaSuccess) return (int)e;
    tc_gemm_tf32_persistent<<<(unsigned)sms, kPgThreads, kPgSmem, stream>>>(ma, mb, p);
    return (int)cudaGetLastError();
  }
  tc_gemm_tf32<<<(unsigned)tiles, kTcThreads, kTcSmem, stream>>>(ma, mb, p);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
