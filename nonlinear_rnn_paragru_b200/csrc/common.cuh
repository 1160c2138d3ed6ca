// common.cuh -- device helpers shared by the solver kernels (sm_100a only).
//
// PTX wrappers for the special-function unit, NaN-propagating max, the
// acquire/release flag protocol of the cross-block look-back, mbarriers and
// TMA bulk-tensor loads, plus the workspace layout the host and the kernels
// agree on.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pararnn.h"

namespace pararnn {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kChan = 32;  // channels per tile (one warp width)

// ------------------------------------------------------------ arithmetic --
// 2^x on the MUFU pipe (ftz).  Saturates to +inf / 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 1/x on the MUFU pipe (ftz); rcp(inf) = 0.
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// max that returns NaN if either operand is NaN (so a NaN residual can never
// look converged).
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float y;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
  return y;
}
// tanh by the one-instruction hardware approximation (relative error about
// 2^-11): only for the inexact early Newton evaluations, never for one that
// decides convergence
__device__ __forceinline__ float tanh_apx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// the same over three operands, in one instruction
__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float y;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}
// min that returns NaN if either operand is NaN: the clamps of exponent
// arguments, so that a NaN input stays NaN (fminf would return the bound and
// turn it into a saturated gate) and the solve reports it as non-finite.
__device__ __forceinline__ float fmin_nan(float a, float b) {
  float y;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
  return y;
}

// ------------------------------------------------------- memory ordering --
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ float2 ld_relaxed_f2(const float2* p) {
  float2 v;
  asm volatile("ld.relaxed.gpu.global.v2.f32 {%0, %1}, [%2];"
               : "=f"(v.x), "=f"(v.y) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_relaxed_f4(const float4* p) {
  float4 v;
  asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------ mbarrier and TMA --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on an mbarrier phase; false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity,
                                                  uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}
// 4-D tiled bulk-tensor load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// 3-D tiled bulk-tensor load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 3-D tiled bulk-tensor store from shared memory (its bulk group committed
// by the caller); coordinates past the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x,
                                             int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// this thread's committed bulk stores have read their shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// this thread's committed bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------- division by invariants --
// n / d for 0 <= n < 2^31 by one multiply-high, the method of Granlund and
// Montgomery ("Division by invariant integers using multiplication", 1994,
// Fig. 4.1), with the (N+1)-bit sum kept in 32 bits because n < 2^31.
struct FastDiv {
  unsigned m;
  int l;
};
inline FastDiv fast_div(unsigned d) {
  int l = 0;
  while ((1ull << l) < d) ++l;
  const unsigned long long m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
  return FastDiv{(unsigned)m, l};
}
__device__ __forceinline__ int fast_quot(int n, FastDiv v) {
  return (int)((__umulhi(v.m, (unsigned)n) + (unsigned)n) >> v.l);
}

// ------------------------------------------------------------ workspace --
// Forward-solve workspace:
//   [0, 256)           header: epoch, ticket counter
//   flags  u32 [nrec]  look-back record flags, nrec = cluster chunks * (max_iters+1)
//   vals   f32 [nrec][kChan][RW]  record payload (RW floats per channel)
//   chan_k int [B*D]   per-channel convergence iterate (histogram input)
//   seg    u32 [B*D/8] segments stored per 8-channel tile (segment-queue solve)
// A record flag is (epoch << 3) | (kind << 1) | ok.  The look-back paths
// clear their flag slice at the start of every call (the epoch alone cannot
// tell a stale flag from another path's leftovers in a shared workspace); the
// paths without look-back keep their scratch after the header.
constexpr size_t kWsHeaderBytes = 256;
struct WsHeader {
  unsigned epoch;
  unsigned ticket;
  unsigned ticket_odd;  // tile counter of the odd-numbered segments of a row solve
  unsigned pad[61];
};
enum : unsigned { kRecAgg = 1, kRecIncl = 2 };

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct FwdWsLayout {
  size_t flags, vals, chan_k, seg, total;
};
__host__ __device__ inline FwdWsLayout fwd_ws_layout(size_t nchunks, int max_iters, int rec_floats,
                                                     size_t BD) {
  FwdWsLayout L;
  size_t nrec = nchunks * (size_t)(max_iters + 1);
  L.flags = kWsHeaderBytes;
  L.vals = L.flags + align256(nrec * 4);
  L.chan_k = L.vals + align256(nrec * kChan * rec_floats * 4);
  L.seg = L.chan_k + align256(BD * 4);
  L.total = L.seg + align256((BD + 7) / 8 * 4);
  return L;
}

// Everything a forward-solve kernel needs besides the tensor map.
// The inexact early Newton evaluations (the one-instruction tanh) run while a
// tile's or item's max |r| is above this; exact ones decide convergence.  On
// configuration-2 inputs an item takes three inexact evaluations, and the
// exact ones then converge in as many evaluations as from exact steps
// throughout (fp64 model of the iteration with 2^-11 gate errors; measured
// thresholds of 0.03, 0.3 and 1.0 were slower)
constexpr float kApxTau = 0.1f;

struct FwdParams {
  const float* a;     // [G][D]
  const float* bias;  // [G][D] or null
  const float* h0;    // [B][D] or null
  const float* c0;    // [B][D] or null (LSTM)
  float* h;           // [B][T][D]
  float* c;           // [B][T][D] (LSTM)
  int B, T, D;
  int nDT;            // channel tiles per batch row: ceil(D / 32)
  int nC;             // sequence chunks (CTAs) per tile
  int CL;             // CTAs per cluster (consecutive chunks of one tile)
  int nCC;            // cluster chunks per tile: ceil(nC / CL)
  int max_iters;
  float tol;
  float apx_tau;      // ParaGRU row kernel: inexact evaluations above this residual (0: none)
  float spec_tau;     // row kernels: a residual-only check follows an exact step from at most this
  float chk_tol;      // and certifies the iterate below this
  unsigned flags;
  int inject_chunk;
  uint64_t timeout_ns;
  WsHeader* hdr;
  unsigned* rec_flags;
  float* rec_vals;
  int* chan_k;        // [B*D] or null
  pararnn_stats* stats;
  // whole-sequence (row) kernel only: the projections (fp32 read directly),
  // the first step, the length and the index of the segment this launch
  // solves, and the batch stride of h0 in floats (a segment starts from the
  // state the one before it ended with)
  const void* u;
  int t_base, t_len, seg;
  long long ld_h0;
  // segment-queue solves: per-tile segment counts (zero at launch), the
  // number of (tile, segment) items, and the item that withholds its
  // publication for testing (-1: none); the item counter is hdr->ticket
  unsigned* seg_done;
  int nitems;
  int withhold_item;
};

}  // namespace pararnn
