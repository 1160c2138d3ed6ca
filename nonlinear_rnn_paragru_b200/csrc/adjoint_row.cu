// adjoint_row.cu -- reverse (adjoint) scan of a solved ParaGRU trajectory for
// sequences of up to 4096 steps with bf16 input projections: 8 channels per
// CTA, a cluster of CLS = ceil(T / 512) CTAs per tile, two CTAs per SM.
//
// With the converged states the loss gradient flows back through the
// transposed block-bidiagonal system ("Параллельность RNN?", §1.3):
//   lambda_t = g_t + carry_{t+1},  carry_t = A_t lambda_t  (A_t = df_t/dh),
//   du_t = (df_t/du_t) lambda_t,  da = sum_t (df_t/da) lambda_t,
//   dbias = sum_t du_t,  dL/dh0 = carry_1,
// a linear recurrence run backwards in time, i.e. a reverse scan of affine
// maps carry_in -> carry_out.
//
// A tile is 8 consecutive channels of one batch row over the whole sequence.
// CTA rank r of the cluster owns steps [512 r, 512 (r+1)): 8 warps x 32
// lanes, lane = (k, c) with the channel c = lane % 8 fastest and k = lane / 8
// one of four 16-step chunks; a thread takes its chunk as 8 step pairs
// (i, i + 8), every add, multiply and fma one packed fp32x2 instruction.
//   pass 1 (backwards over the chunk): re-evaluate the cell and compose each
//     half-chunk's map carry_in -> carry_out, from which the chunk's map;
//   scan: a suffix scan over the warp's four chunks by shuffles; each thread
//     composes the maps of the warps after its own from shared memory (one
//     CTA barrier); the CTA's map goes to the CTAs before it in the cluster
//     by remote asynchronous stores that complete on the receiver's mbarrier;
//   pass 2 (backwards): re-evaluate the cell, run the exact recurrence from
//     the true incoming carry, write du and accumulate da / dbias partials.
// Per-CTA partials are summed by a second kernel in a fixed order, so the
// result is bitwise reproducible.
//
// Data: per chunk three TMA boxes into a 2304-byte slot: u (bf16 rows
// [t][gate][8 ch], 19 steps), the states h_{t-1} (fp32, 20 steps) and dL/dh
// (fp32, 19 steps).  Chunk k of a warp is loaded k steps early and read at a
// k-row offset, so the four chunks a warp reads at one step fall in disjoint
// bank windows.  The other CTA on the SM covers a tile's load (an L2
// prefetch of the next tile's boxes measured slower).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "adjoint_cell.cuh"
#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cga = cooperative_groups;

constexpr int kArThreads = 256;
constexpr int kArWarps = 8;
constexpr int kArSteps = kArWarps * kArK * kArL;  // 512 steps per CTA
constexpr int kArChunks = kArSteps / kArL;        // 32
constexpr int kArSmem = kArChunks * kArS;     // 73728
constexpr int kArMaxCluster = 8;
constexpr int kArTmax = kArSteps * kArMaxCluster;  // 4096
constexpr unsigned kArTileBytes =
    kArChunks * (kArUBox * kArUStep + kArHBox * kArSStep + kArGBox * kArSStep);
static_assert(kArWarps == kArC, "one scan row per channel");
// mailbox ring: slots used round robin by tile, a cluster barrier every
// kArSyncEvery tiles (see the tile loop)
constexpr int kArSlots = 8, kArSyncEvery = 4;
static_assert(kArSlots >= 2 * kArSyncEvery, "a slot is rewritten only after a barrier past its use");

struct ArShared {
  float2 wagg[2][kArWarps][kArC];        // per (warp, channel) suffix map of the warp
  __align__(16) float2 mbox[kArSlots][kArMaxCluster][kArC];  // CTA maps of the later ranks
  float red[kArWarps][6][kArC];          // partial sums per warp
  __align__(16) float par[7][kArC];      // a (3 rows), bias (3 rows), h0
  uint64_t bar;                          // the tile's loads
  uint64_t mbar[kArSlots];               // mailbox barriers, by slot
};


__device__ __forceinline__ uint32_t ar_mapa(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void ar_st_async_v2(uint32_t raddr, float2 v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];"
      ::"r"(raddr), "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void ar_st_async_v4(uint32_t raddr, float4 v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(raddr), "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)),
      "r"(__float_as_uint(v.z)), "r"(__float_as_uint(v.w)), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void ar_bulk_load(void* dst, const void* src, unsigned bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
struct ArParams {
  const float *a, *bias, *h0;
  float *du, *dh0, *part;
  int B, T, D;
  uint64_t timeout_ns;
  int* status;
  int withhold_rank;  // testing: this cluster rank withholds its map in its
                      // cluster's last tile (-1: none)
};

// Warp 0: the tile's boxes (u, h_{t-1}, dL/dh per chunk; lane q issues
// chunk q's three) and its a, bias, h0 rows, all on `bar`.
__device__ __forceinline__ void ar_issue(unsigned char* smem, ArShared& sh,
                                         const CUtensorMap* mu, const CUtensorMap* mh,
                                         const CUtensorMap* mg, const ArParams& p, int b,
                                         int d0, int t0, int lane) {
  static_assert(kArChunks == 32, "one chunk per lane");
  const unsigned pb = kArC * 4;
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(&sh.bar, kArTileBytes + 3 * pb + (p.bias ? 3 * pb : 0) +
                                       (p.h0 ? pb : 0));
    for (int g = 0; g < 3; ++g) {
      ar_bulk_load(&sh.par[g][0], p.a + (size_t)g * p.D + d0, pb, &sh.bar);
      if (p.bias) ar_bulk_load(&sh.par[3 + g][0], p.bias + (size_t)g * p.D + d0, pb, &sh.bar);
    }
    if (p.h0) ar_bulk_load(&sh.par[6][0], p.h0 + (size_t)b * p.D + d0, pb, &sh.bar);
  }
  __syncwarp();
  const int q = lane, k = q % kArK, ts = t0 + q * kArL - k;
  unsigned char* slot = smem + q * kArS;
  tma_load_4d(slot + kArUOff, mu, &sh.bar, d0, 0, ts, b);
  tma_load_3d(slot + kArHOff, mh, &sh.bar, d0, ts - 1, b);
  tma_load_3d(slot + kArGOff, mg, &sh.bar, d0, ts, b);
}

template <int CLS>
__global__ void __launch_bounds__(kArThreads, 2)
    adjoint_row(const __grid_constant__ CUtensorMap mu, const __grid_constant__ CUtensorMap mh,
                const __grid_constant__ CUtensorMap mg, const ArParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ ArShared sh;
  cga::cluster_group cluster = cga::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (CLS > 1) ? (int)cluster.block_rank() : 0;
  const int c = lane % kArC, kk = lane / kArC;
  const int q = warp * kArK + kk;
  const int nDTc = (p.D + kArC - 1) / kArC;
  const int ntiles = p.B * nDTc;
  const int nclus = gridDim.x / CLS, clus = blockIdx.x / CLS;
  const int t0 = rank * kArSteps;
  const unsigned rx = (unsigned)((CLS - 1 - rank) * kArC * 8);

  if (tid < 7 * kArC) (&sh.par[0][0])[tid] = 0.f;
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    if (CLS > 1)
      for (int j = 0; j < kArSlots; ++j) {
        mbar_init(&sh.mbar[j], 1);
        mbar_arrive_expect_tx(&sh.mbar[j], rx);
      }
  }
  __syncthreads();
  if (CLS > 1) cluster.sync();
  if (warp == 0 && clus < ntiles) {
    const int b = clus / nDTc;
    ar_issue(smem, sh, &mu, &mh, &mg, p, b, (clus - b * nDTc) * kArC, t0, lane);
  }
  const unsigned char* slot = smem + q * kArS;
  const unsigned char* ubase = slot + kArUOff + kk * kArUStep + c * 2;
  const float* hbase = reinterpret_cast<const float*>(slot + kArHOff + kk * kArSStep) + c;
  const float* gbase = reinterpret_cast<const float*>(slot + kArGOff + kk * kArSStep) + c;
  const bool first = (rank == 0 && q == 0);
  int status = 0, n = 0;
  for (int tile = clus; tile < ntiles; tile += nclus, ++n) {
    const int par = n & 1;
    const int b = tile / nDTc, d0 = (tile - b * nDTc) * kArC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int next = tile + nclus;
    // the exchange runs from later ranks to earlier ones only: this barrier,
    // every kArSyncEvery tiles, keeps the CTAs of a cluster within that many
    // tiles of each other, so a mailbox slot (reused every kArSlots tiles) is
    // not written again before its reader is done with it
    const int ms = n % kArSlots;  // mailbox slot of this tile
    if (CLS > 1 && n % kArSyncEvery == 0) cluster.sync();
    if (!mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;
    ArCell k;
    float2 S, BZ, BR, BC;
    float h0v;
    {
      const float az = sh.par[0][c], ar = sh.par[1][c], ac = sh.par[2][c];
      k.AZ = af2(az, az);
      k.AR = af2(ar, ar);
      k.AC = af2(ac, ac);
      const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
      k.AZ2 = af2(az2, az2);
      k.AR2 = af2(ar2, ar2);
      k.AC2 = af2(ac2, ac2);
      S = af2(-kLog2e, -kLog2e);
      const float bz = -kLog2e * sh.par[3][c], br = -kLog2e * sh.par[4][c],
                  bc = 2.f * kLog2e * sh.par[5][c];
      BZ = af2(bz, bz);
      BR = af2(br, br);
      BC = af2(bc, bc);
      h0v = sh.par[6][c];
    }

    // ---- pass 1: the two half-chunk maps, backwards
    float2 PM = af2(1.f, 1.f), DM = af2(0.f, 0.f);
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UZ, UR, UC, A, GZ, GR, GC, RH;
      ar_args(ubase + i * kArUStep, ubase + (i + kArH) * kArUStep, S, BZ, BR, BC, UZ, UR, UC);
      float2 HP = af2(hbase[i * kArC], hbase[(i + kArH) * kArC]);  // h_{t-1}
      if (i == 0 && first) HP.x = h0v;
      const float2 G = af2(gbase[i * kArC], gbase[(i + kArH) * kArC]);
      ar_cell(k, HP, UZ, UR, UC, A, GZ, GR, GC, RH);
      DM = amul(A, aadd(G, DM));
      PM = amul(A, PM);
    }
    // the chunk's map: the first half after the second
    float2 inc = ar_after(af2(PM.x, DM.x), af2(PM.y, DM.y));
    // suffix scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
    for (int o = kArC; o < 32; o <<= 1) {
      const float2 nx = af2(__shfl_down_sync(kFull, inc.x, o), __shfl_down_sync(kFull, inc.y, o));
      if (lane + o < 32) inc = ar_after(inc, nx);
    }
    // the carry entering the warp -> the carry entering this chunk
    float2 xm = af2(__shfl_down_sync(kFull, inc.x, kArC), __shfl_down_sync(kFull, inc.y, kArC));
    if (kk == kArK - 1) xm = af2(1.f, 0.f);
    if (kk == 0) sh.wagg[par][warp][c] = inc;
    __syncthreads();
    // the warps after this one: the CTA's incoming carry -> this warp's
    float2 cw = af2(1.f, 0.f);
#pragma unroll
    for (int w = kArWarps - 1; w > 0; --w)
      if (w > warp) cw = ar_after(sh.wagg[par][w][c], cw);
    float cin_cta = 0.f;  // carry entering this CTA from the steps after it
    if (CLS > 1) {
      // testing: a withheld map in the cluster's last tile (no later
      // exchange reuses a barrier whose phase did not complete)
      const bool withhold = rank == p.withhold_rank && next >= ntiles;
      if (warp == 0 && kk == 0 && rank > 0 && !withhold) {
        const float2 m = ar_after(inc, cw);  // the CTA's map of channel c
        for (int r = 0; r < rank; ++r)
          ar_st_async_v2(ar_mapa(smem_u32(&sh.mbox[ms][rank][c]), r), m,
                         ar_mapa(smem_u32(&sh.mbar[ms]), r));
      }
      // The last rank receives nothing, so it neither waits nor re-arms: a
      // zero-byte re-arm completes the next phase at once, and a warp yet to
      // wait would then wait for the phase after that one.
      const bool got =
          rank == CLS - 1 || mbar_wait_bounded(&sh.mbar[ms], (n / kArSlots) & 1, p.timeout_ns);
      if (!got && status == 0) status = PARARNN_STATUS_TIMEOUT;
#pragma unroll
      for (int r = CLS - 1; r > 0; --r) {
        if (r > rank) {
          const float2 m = sh.mbox[ms][r][c];
          cin_cta = fmaf(m.x, cin_cta, m.y);
        }
      }
      __syncwarp();
      // a phase that did not complete is not re-armed: a second arrival on
      // it would be one more than the barrier counts
      if (tid == 0 && rank < CLS - 1 && got) mbar_arrive_expect_tx(&sh.mbar[ms], rx);
    }
    const float cwarp = fmaf(cw.x, cin_cta, cw.y);
    const float cchunk = fmaf(xm.x, cwarp, xm.y);

    // ---- pass 2: the exact recurrence, du and the partial sums
    float2 CARRY = af2(fmaf(PM.y, cchunk, DM.y), cchunk);  // entering steps 7 and 15
    float2 SAZ = af2(0.f, 0.f), SAR = SAZ, SAC = SAZ, SBZ = SAZ, SBR = SAZ, SBC = SAZ;
    const int tq = t0 + q * kArL;
    float* dub = p.du + (((size_t)b * p.T + tq) * 3) * p.D + d;
    bool bad = false;
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UZ, UR, UC, A, GZ, GR, GC, RH;
      ar_args(ubase + i * kArUStep, ubase + (i + kArH) * kArUStep, S, BZ, BR, BC, UZ, UR, UC);
      float2 HP = af2(hbase[i * kArC], hbase[(i + kArH) * kArC]);
      if (i == 0 && first) HP.x = h0v;
      const float2 G = af2(gbase[i * kArC], gbase[(i + kArH) * kArC]);
      ar_cell(k, HP, UZ, UR, UC, A, GZ, GR, GC, RH);
      const float2 LAM = aadd(G, CARRY);
      const float2 DZ = amul(GZ, LAM), DR = amul(GR, LAM), DC = amul(GC, LAM);
      SAZ = afma(DZ, HP, SAZ);
      SAR = afma(DR, HP, SAR);
      SAC = afma(DC, RH, SAC);
      SBZ = aadd(SBZ, DZ);
      SBR = aadd(SBR, DR);
      SBC = aadd(SBC, DC);
      CARRY = amul(A, LAM);
      if (dval) {
        if (tq + i < p.T) {
          float* o = dub + (size_t)i * 3 * p.D;
          o[0] = DZ.x;
          o[p.D] = DR.x;
          o[2 * (size_t)p.D] = DC.x;
          bad |= !isfinite(DZ.x) || !isfinite(DR.x) || !isfinite(DC.x);
        }
        if (tq + kArH + i < p.T) {
          float* o = dub + (size_t)(kArH + i) * 3 * p.D;
          o[0] = DZ.y;
          o[p.D] = DR.y;
          o[2 * (size_t)p.D] = DC.y;
          bad |= !isfinite(DZ.y) || !isfinite(DR.y) || !isfinite(DC.y);
        }
      }
    }
    if (first && dval && p.dh0) p.dh0[(size_t)b * p.D + d] = CARRY.x;
    // partial sums of the CTA: over the two halves, the warp's chunks, then
    // the warps in order
    float v[6] = {SAZ.x + SAZ.y, SAR.x + SAR.y, SAC.x + SAC.y,
                  SBZ.x + SBZ.y, SBR.x + SBR.y, SBC.x + SBC.y};
#pragma unroll
    for (int j = 0; j < 6; ++j) {
      v[j] = dval ? v[j] : 0.f;
      v[j] += __shfl_xor_sync(kFull, v[j], 8);
      v[j] += __shfl_xor_sync(kFull, v[j], 16);
    }
    if (kk == 0)
#pragma unroll
      for (int j = 0; j < 6; ++j) sh.red[warp][j][c] = v[j];
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    __syncthreads();
    // every pass of this tile is done: the slots take the next tile
    if (warp == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      ar_issue(smem, sh, &mu, &mh, &mg, p, b2, (next - b2 * nDTc) * kArC, t0, lane);
    }
    if (tid < 6 * kArC) {
      const int j = tid / kArC, cc = tid % kArC;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kArWarps; ++w) s += sh.red[w][j][cc];
      p.part[((size_t)tile * CLS + rank) * (6 * kArC) + tid] = s;
    }
  }
  const int st = __reduce_max_sync(kFull, status);
  if (lane == 0 && st) atomicMax(p.status, st);
  if (CLS > 1) cluster.sync();
}


// ---------------------------------------------------------------- ParaLSTM --
// The same structure for the 2x2 Jacobian: lambda = (lambda_c, lambda_h), the
// loss gradient enters through lambda_h, carry_t = A_t^T lambda_t.  Per chunk
// four boxes (u, c_{t-1}, h_{t-1}, dL/dh) in the slot of adjoint_cell.cuh.
constexpr int kAlSmem = kArChunks * kAlS;     // 102400
constexpr unsigned kAlTileBytes =
    kArChunks * (kArUBox * kAlUStep + 2 * kArHBox * kArSStep + kArGBox * kArSStep);
static_assert(kArUBox * kAlUStep <= kAlCOff && kAlCOff + kArHBox * kArSStep <= kAlHOff &&
                  kAlHOff + kArHBox * kArSStep <= kAlGOff &&
                  kAlGOff + kArGBox * kArSStep <= kAlS && kAlS % 128 == 0 &&
                  kAlCOff % 128 == 0 && kAlHOff % 128 == 0 && kAlGOff % 128 == 0,
              "ParaLSTM chunk slot layout");

// a smaller mailbox ring than ParaGRU's (its entries are four times larger),
// so that two CTAs still share an SM: 4 slots, a cluster barrier every 2 tiles
constexpr int kAlSlots = 4, kAlSyncEvery = 2;
static_assert(kAlSlots >= 2 * kAlSyncEvery, "a slot is rewritten only after a barrier past its use");

struct AlShared {
  // per (warp, channel) suffix map: (m), (d, -, -); a CTA barrier separates a
  // tile's reads from the next tile's writes, so one buffer suffices
  float4 wagg[kArWarps][kArC][2];
  __align__(16) float4 mbox[kAlSlots][kArMaxCluster][kArC][2];  // CTA maps of the later ranks
  float red[kArWarps][8][kArC];          // partial sums per warp
  __align__(16) float par[10][kArC];     // a (4 rows), bias (4 rows), c0, h0
  uint64_t bar;
  uint64_t mbar[kAlSlots];
};

struct AlParams {
  const float *a, *bias, *c0, *h0;
  float *du, *dc0, *dh0, *part;
  int B, T, D;
  uint64_t timeout_ns;
  int* status;
  int withhold_rank;  // as for ArParams
};

// Warp 0: the tile's boxes (lane q issues chunk q's four) and its a, bias,
// c0, h0 rows, all on `bar`.
__device__ __forceinline__ void al_issue(unsigned char* smem, AlShared& sh, const CUtensorMap* mu,
                                         const CUtensorMap* mc, const CUtensorMap* mh,
                                         const CUtensorMap* mg, const AlParams& p, int b,
                                         int d0, int t0, int lane) {
  const unsigned pb = kArC * 4;
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(&sh.bar, kAlTileBytes + 4 * pb + (p.bias ? 4 * pb : 0) +
                                       (p.c0 ? pb : 0) + (p.h0 ? pb : 0));
    for (int g = 0; g < 4; ++g) {
      ar_bulk_load(&sh.par[g][0], p.a + (size_t)g * p.D + d0, pb, &sh.bar);
      if (p.bias) ar_bulk_load(&sh.par[4 + g][0], p.bias + (size_t)g * p.D + d0, pb, &sh.bar);
    }
    if (p.c0) ar_bulk_load(&sh.par[8][0], p.c0 + (size_t)b * p.D + d0, pb, &sh.bar);
    if (p.h0) ar_bulk_load(&sh.par[9][0], p.h0 + (size_t)b * p.D + d0, pb, &sh.bar);
  }
  __syncwarp();
  const int q = lane, k = q % kArK, ts = t0 + q * kArL - k;
  unsigned char* slot = smem + q * kAlS;
  tma_load_4d(slot + kAlUOff, mu, &sh.bar, d0, 0, ts, b);
  tma_load_3d(slot + kAlCOff, mc, &sh.bar, d0, ts - 1, b);
  tma_load_3d(slot + kAlHOff, mh, &sh.bar, d0, ts - 1, b);
  tma_load_3d(slot + kAlGOff, mg, &sh.bar, d0, ts, b);
}

__device__ __forceinline__ Aff2 al_shfl_down(const Aff2& a, int o) {
  return Aff2{__shfl_down_sync(kFull, a.m00, o), __shfl_down_sync(kFull, a.m01, o),
              __shfl_down_sync(kFull, a.m10, o), __shfl_down_sync(kFull, a.m11, o),
              __shfl_down_sync(kFull, a.d0, o),  __shfl_down_sync(kFull, a.d1, o)};
}

template <int CLS>
__global__ void __launch_bounds__(kArThreads, 2)
    adjoint_row_lstm(const __grid_constant__ CUtensorMap mu, const __grid_constant__ CUtensorMap mc,
                     const __grid_constant__ CUtensorMap mh, const __grid_constant__ CUtensorMap mg,
                     const AlParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ AlShared sh;
  cga::cluster_group cluster = cga::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (CLS > 1) ? (int)cluster.block_rank() : 0;
  const int c = lane % kArC, kk = lane / kArC;
  const int q = warp * kArK + kk;
  const int nDTc = (p.D + kArC - 1) / kArC;
  const int ntiles = p.B * nDTc;
  const int nclus = gridDim.x / CLS, clus = blockIdx.x / CLS;
  const int t0 = rank * kArSteps;
  const unsigned rx = (unsigned)((CLS - 1 - rank) * kArC * 32);

  if (tid < 10 * kArC) (&sh.par[0][0])[tid] = 0.f;
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    if (CLS > 1)
      for (int j = 0; j < kAlSlots; ++j) {
        mbar_init(&sh.mbar[j], 1);
        mbar_arrive_expect_tx(&sh.mbar[j], rx);
      }
  }
  __syncthreads();
  if (CLS > 1) cluster.sync();
  if (warp == 0 && clus < ntiles) {
    const int b = clus / nDTc;
    al_issue(smem, sh, &mu, &mc, &mh, &mg, p, b, (clus - b * nDTc) * kArC, t0, lane);
  }
  const unsigned char* slot = smem + q * kAlS;
  const unsigned char* ubase = slot + kAlUOff + kk * kAlUStep + c * 2;
  const float* cbase = reinterpret_cast<const float*>(slot + kAlCOff + kk * kArSStep) + c;
  const float* hbase = reinterpret_cast<const float*>(slot + kAlHOff + kk * kArSStep) + c;
  const float* gbase = reinterpret_cast<const float*>(slot + kAlGOff + kk * kArSStep) + c;
  const bool first = (rank == 0 && q == 0);
  int status = 0, n = 0;
  for (int tile = clus; tile < ntiles; tile += nclus, ++n) {
    const int b = tile / nDTc, d0 = (tile - b * nDTc) * kArC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int next = tile + nclus;
    const int ms = n % kAlSlots;
    if (CLS > 1 && n % kAlSyncEvery == 0) cluster.sync();
    if (!mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;
    AlCell k;
    float2 BS[4];
    float c0v, h0v;
    {
      const float ai = sh.par[0][c], af = sh.par[1][c], ag = sh.par[2][c], ao = sh.par[3][c];
      k.AI = af2(ai, ai);
      k.AF = af2(af, af);
      k.AG = af2(ag, ag);
      k.AO = af2(ao, ao);
      k.AI2 = af2(-kLog2e * ai, -kLog2e * ai);
      k.AF2 = af2(-kLog2e * af, -kLog2e * af);
      k.AG2 = af2(2.f * kLog2e * ag, 2.f * kLog2e * ag);
      k.AO2 = af2(-kLog2e * ao, -kLog2e * ao);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float bs = (g == 2 ? 2.f * kLog2e : -kLog2e) * sh.par[4 + g][c];
        BS[g] = af2(bs, bs);
      }
      c0v = sh.par[8][c];
      h0v = sh.par[9][c];
    }
    auto state = [&](int i, float2& CP, float2& HP, float2& G) {
      CP = af2(cbase[i * kArC], cbase[(i + kArH) * kArC]);  // (c, h)_{t-1}
      HP = af2(hbase[i * kArC], hbase[(i + kArH) * kArC]);
      if (i == 0 && first) {
        CP.x = c0v;
        HP.x = h0v;
      }
      G = af2(gbase[i * kArC], gbase[(i + kArH) * kArC]);
    };

    // ---- pass 1: the two half-chunk maps (carry_in -> carry_out), backwards
    float2 M00 = af2(1.f, 1.f), M01 = af2(0.f, 0.f), M10 = M01, M11 = M00, D0 = M01, D1 = M01;
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UI, UF, UG, UO, CP, HP, G, F, X, KK, A11, GCI, GCF, GCG, DOT;
      al_args(ubase + i * kAlUStep, ubase + (i + kArH) * kAlUStep, BS, UI, UF, UG, UO);
      state(i, CP, HP, G);
      al_cell(k, CP, HP, UI, UF, UG, UO, F, X, KK, A11, GCI, GCF, GCG, DOT);
      const float2 A10 = amul(KK, F);
      // carry_out = A^T (carry_in + (0, g)); compose after the map so far
      const float2 E1 = aadd(D1, G);
      const float2 n00 = afma(F, M00, amul(A10, M10)), n01 = afma(F, M01, amul(A10, M11));
      const float2 n10 = afma(X, M00, amul(A11, M10)), n11 = afma(X, M01, amul(A11, M11));
      const float2 nd0 = afma(F, D0, amul(A10, E1)), nd1 = afma(X, D0, amul(A11, E1));
      M00 = n00;
      M01 = n01;
      M10 = n10;
      M11 = n11;
      D0 = nd0;
      D1 = nd1;
    }
    const Aff2 Mx{M00.x, M01.x, M10.x, M11.x, D0.x, D1.x};
    const Aff2 My{M00.y, M01.y, M10.y, M11.y, D0.y, D1.y};
    // the chunk's map: the first half after the second
    Aff2 inc = Mx.after(My);
    // suffix scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
    for (int o = kArC; o < 32; o <<= 1) {
      const Aff2 nx = al_shfl_down(inc, o);
      if (lane + o < 32) inc = inc.after(nx);
    }
    Aff2 xm = al_shfl_down(inc, kArC);
    if (kk == kArK - 1) xm = Aff2::id();
    if (kk == 0) {
      sh.wagg[warp][c][0] = make_float4(inc.m00, inc.m01, inc.m10, inc.m11);
      sh.wagg[warp][c][1] = make_float4(inc.d0, inc.d1, 0.f, 0.f);
    }
    __syncthreads();
    Aff2 cw = Aff2::id();
#pragma unroll
    for (int w = kArWarps - 1; w > 0; --w)
      if (w > warp) {
        const float4 m4 = sh.wagg[w][c][0], v4 = sh.wagg[w][c][1];
        cw = Aff2{m4.x, m4.y, m4.z, m4.w, v4.x, v4.y}.after(cw);
      }
    float2 cin_cta = af2(0.f, 0.f);
    if (CLS > 1) {
      const bool withhold = rank == p.withhold_rank && next >= ntiles;  // testing
      if (warp == 0 && kk == 0 && rank > 0 && !withhold) {
        const Aff2 m = inc.after(cw);  // the CTA's map of channel c
        const float4 m0 = make_float4(m.m00, m.m01, m.m10, m.m11);
        const float4 m1 = make_float4(m.d0, m.d1, 0.f, 0.f);
        for (int r = 0; r < rank; ++r) {
          const uint32_t rb = ar_mapa(smem_u32(&sh.mbar[ms]), r);
          ar_st_async_v4(ar_mapa(smem_u32(&sh.mbox[ms][rank][c][0]), r), m0, rb);
          ar_st_async_v4(ar_mapa(smem_u32(&sh.mbox[ms][rank][c][1]), r), m1, rb);
        }
      }
      // the last rank receives nothing: no wait, no re-arm (as for ParaGRU)
      const bool got =
          rank == CLS - 1 || mbar_wait_bounded(&sh.mbar[ms], (n / kAlSlots) & 1, p.timeout_ns);
      if (!got && status == 0) status = PARARNN_STATUS_TIMEOUT;
#pragma unroll
      for (int r = CLS - 1; r > 0; --r) {
        if (r > rank) {
          const float4 m0 = sh.mbox[ms][r][c][0], m1 = sh.mbox[ms][r][c][1];
          cin_cta = Aff2{m0.x, m0.y, m0.z, m0.w, m1.x, m1.y}.apply(cin_cta);
        }
      }
      __syncwarp();
      if (tid == 0 && rank < CLS - 1 && got) mbar_arrive_expect_tx(&sh.mbar[ms], rx);
    }
    const float2 cchunk = xm.apply(cw.apply(cin_cta));
    const float2 cx = My.apply(cchunk);  // entering step 7 from step 8

    // ---- pass 2: the exact recurrence, du and the partial sums
    float2 LC = af2(cx.x, cchunk.x), LH = af2(cx.y, cchunk.y);
    float2 SA[4], SB[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) SA[g] = SB[g] = af2(0.f, 0.f);
    const int tq = t0 + q * kArL;
    float* dub = p.du + (((size_t)b * p.T + tq) * 4) * p.D + d;
    bool bad = false;
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UI, UF, UG, UO, CP, HP, G, F, X, KK, A11, GCI, GCF, GCG, DOT;
      al_args(ubase + i * kAlUStep, ubase + (i + kArH) * kAlUStep, BS, UI, UF, UG, UO);
      state(i, CP, HP, G);
      al_cell(k, CP, HP, UI, UF, UG, UO, F, X, KK, A11, GCI, GCF, GCG, DOT);
      const float2 LHE = aadd(LH, G);                      // lambda_h
      const float2 LCH = afma(KK, LHE, LC);                // lambda_c + kk lambda_h
      const float2 DU[4] = {amul(GCI, LCH), amul(GCF, LCH), amul(GCG, LCH), amul(DOT, LHE)};
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        SA[g] = afma(DU[g], HP, SA[g]);
        SB[g] = aadd(SB[g], DU[g]);
      }
      // carry = A^T lambda = (f (lambda_c + kk lambda_h), X (...) + a_o du_o)
      LC = amul(F, LCH);
      LH = afma(X, LCH, amul(k.AO, DU[3]));
      if (dval) {
        if (tq + i < p.T) {
          float* o = dub + (size_t)i * 4 * p.D;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            o[(size_t)g * p.D] = DU[g].x;
            bad |= !isfinite(DU[g].x);
          }
        }
        if (tq + kArH + i < p.T) {
          float* o = dub + (size_t)(kArH + i) * 4 * p.D;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            o[(size_t)g * p.D] = DU[g].y;
            bad |= !isfinite(DU[g].y);
          }
        }
      }
    }
    if (first && dval) {
      if (p.dc0) p.dc0[(size_t)b * p.D + d] = LC.x;
      if (p.dh0) p.dh0[(size_t)b * p.D + d] = LH.x;
    }
    float v[8];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      v[g] = SA[g].x + SA[g].y;
      v[4 + g] = SB[g].x + SB[g].y;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = dval ? v[j] : 0.f;
      v[j] += __shfl_xor_sync(kFull, v[j], 8);
      v[j] += __shfl_xor_sync(kFull, v[j], 16);
    }
    if (kk == 0)
#pragma unroll
      for (int j = 0; j < 8; ++j) sh.red[warp][j][c] = v[j];
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    __syncthreads();
    if (warp == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      al_issue(smem, sh, &mu, &mc, &mh, &mg, p, b2, (next - b2 * nDTc) * kArC, t0, lane);
    }
    if (tid < 8 * kArC) {
      const int j = tid / kArC, cc = tid % kArC;
      float sacc = 0.f;
#pragma unroll
      for (int w = 0; w < kArWarps; ++w) sacc += sh.red[w][j][cc];
      p.part[((size_t)tile * CLS + rank) * (8 * kArC) + tid] = sacc;
    }
  }
  const int st = __reduce_max_sync(kFull, status);
  if (lane == 0 && st) atomicMax(p.status, st);
  if (CLS > 1) cluster.sync();
}

// da[g][d] and dbias[g][d]: per-CTA partials summed over batch rows and
// cluster ranks in a fixed order (bitwise reproducible).  One warp per
// output: lane j sums the terms j, j + 32, ... in order, then the 32 lane
// sums are added by a fixed shuffle tree.
__global__ void adjoint_row_reduce(const float* __restrict__ part, float* da, float* dbias, int B,
                                   int D, int cls, int G) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // over G * D
  const int lane = threadIdx.x & 31;
  if (i >= G * D) return;
  const int g = i / D, d = i - g * D;
  const int nDTc = (D + kArC - 1) / kArC, dt = d / kArC, cc = d % kArC;
  const int nterm = B * cls;
  float sa = 0.f, sb = 0.f;
  for (int j = lane; j < nterm; j += 32) {
    const int b = j / cls, r = j - b * cls;
    const float* pp = part + ((size_t)(b * nDTc + dt) * cls + r) * (2 * G * kArC);
    sa += pp[g * kArC + cc];
    sb += pp[(G + g) * kArC + cc];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sa += __shfl_xor_sync(kFull, sa, o);
    sb += __shfl_xor_sync(kFull, sb, o);
  }
  if (lane == 0) {
    da[i] = sa;
    if (dbias) dbias[i] = sb;
  }
}

__global__ void adjoint_row_init(int* status) { *status = 0; }

// da, dbias from per-(tile, part) partial sums (parts: cluster ranks, or the
// segments of the queue adjoint), in a fixed order
void adjoint_row_reduce_launch(const float* part, float* da, float* dbias, int B, int D, int cls,
                               int G, cudaStream_t stream) {
  adjoint_row_reduce<<<(G * D * 32 + 255) / 256, 256, 0, stream>>>(part, da, dbias, B, D, cls, G);
}

int adjoint_row_cluster(int T) {
  if (T > kArTmax) return 0;
  int cls = 1;
  while (cls * kArSteps < T) cls *= 2;
  return cls;
}
int adjoint_row_channels() { return kArC; }
int adjoint_row_box_steps(int which) { return which == 0 ? kArUBox : (which == 1 ? kArHBox : kArGBox); }
size_t adjoint_row_part_bytes(int G, int B, int T, int D) {
  return (size_t)B * ((D + kArC - 1) / kArC) * adjoint_row_cluster(T) * 2 * G * kArC * 4;
}

template <int CLS>
static int launch_ar_t(const CUtensorMap* maps, const ArParams& p, cudaStream_t stream) {
  const long long ntiles = (long long)p.B * ((p.D + kArC - 1) / kArC);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = adjoint_row<CLS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kArSmem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kArThreads);
  cfg.dynamicSmemBytes = kArSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CLS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclus = 2 * sms / CLS;
  cfg.gridDim = dim3(nclus * CLS);
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) == cudaSuccess && active > 0)
    nclus = std::min(nclus, active);
  cudaGetLastError();
  nclus = (int)std::min<long long>(nclus, ntiles);
  if (nclus < 1) nclus = 1;
  cfg.gridDim = dim3(nclus * CLS);
  return (int)cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], p);
}

// maps: u (box 8 x 3 x 19), h (box 8 x 20), dL/dh (box 8 x 19)
int launch_adjoint_row(const CUtensorMap* maps, const float* a, const float* bias,
                       const float* h0, float* du, float* da, float* dbias, float* dh0, int B,
                       int T, int D, int* status, void* ws, uint64_t timeout_ns,
                       int withhold_rank, cudaStream_t stream) {
  ArParams p;
  p.a = a;
  p.bias = bias;
  p.h0 = h0;
  p.du = du;
  p.dh0 = dh0;
  p.part = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kWsHeaderBytes);
  p.B = B;
  p.T = T;
  p.D = D;
  p.timeout_ns = timeout_ns;
  p.status = status;
  p.withhold_rank = withhold_rank;
  const int cls = adjoint_row_cluster(T);
  adjoint_row_init<<<1, 1, 0, stream>>>(status);
  if (cudaGetLastError() != cudaSuccess) return 1;
  int e;
  switch (cls) {
    case 1: e = launch_ar_t<1>(maps, p, stream); break;
    case 2: e = launch_ar_t<2>(maps, p, stream); break;
    case 4: e = launch_ar_t<4>(maps, p, stream); break;
    case 8: e = launch_ar_t<8>(maps, p, stream); break;
    default: return 1;
  }
  if (e) return e;
  adjoint_row_reduce<<<(3 * D * 32 + 255) / 256, 256, 0, stream>>>(p.part, da, dbias, B, D, cls, 3);
  return (int)cudaGetLastError();
}

template <int CLS>
static int launch_al_t(const CUtensorMap* maps, const AlParams& p, cudaStream_t stream) {
  const long long ntiles = (long long)p.B * ((p.D + kArC - 1) / kArC);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = adjoint_row_lstm<CLS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kAlSmem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kArThreads);
  cfg.dynamicSmemBytes = kAlSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CLS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclus = 2 * sms / CLS;
  cfg.gridDim = dim3(nclus * CLS);
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) == cudaSuccess && active > 0)
    nclus = std::min(nclus, active);
  cudaGetLastError();
  nclus = (int)std::min<long long>(nclus, ntiles);
  if (nclus < 1) nclus = 1;
  cfg.gridDim = dim3(nclus * CLS);
  return (int)cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], p);
}

// maps: u (box 8 x 4 x 19), c and h (box 8 x 20), dL/dh (box 8 x 19)
int launch_adjoint_row_lstm(const CUtensorMap* maps, const float* a, const float* bias,
                            const float* c0, const float* h0, float* du, float* da,
                            float* dbias, float* dc0, float* dh0, int B, int T, int D,
                            int* status, void* ws, uint64_t timeout_ns, int withhold_rank,
                            cudaStream_t stream) {
  AlParams p;
  p.a = a;
  p.bias = bias;
  p.c0 = c0;
  p.h0 = h0;
  p.du = du;
  p.dc0 = dc0;
  p.dh0 = dh0;
  p.part = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + kWsHeaderBytes);
  p.B = B;
  p.T = T;
  p.D = D;
  p.timeout_ns = timeout_ns;
  p.status = status;
  p.withhold_rank = withhold_rank;
  const int cls = adjoint_row_cluster(T);
  adjoint_row_init<<<1, 1, 0, stream>>>(status);
  if (cudaGetLastError() != cudaSuccess) return 1;
  int e;
  switch (cls) {
    case 1: e = launch_al_t<1>(maps, p, stream); break;
    case 2: e = launch_al_t<2>(maps, p, stream); break;
    case 4: e = launch_al_t<4>(maps, p, stream); break;
    case 8: e = launch_al_t<8>(maps, p, stream); break;
    default: return 1;
  }
  if (e) return e;
  adjoint_row_reduce<<<(4 * D * 32 + 255) / 256, 256, 0, stream>>>(p.part, da, dbias, B, D, cls, 4);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
