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

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cga = cooperative_groups;

constexpr int kArThreads = 256;
constexpr int kArWarps = 8;
constexpr int kArC = 8;                       // channels per tile
constexpr int kArK = 32 / kArC;               // chunks per warp
constexpr int kArL = 16;                      // steps per chunk
constexpr int kArH = kArL / 2;                // step pairs per chunk
constexpr int kArSteps = kArWarps * kArK * kArL;  // 512 steps per CTA
constexpr int kArChunks = kArSteps / kArL;        // 32
constexpr int kArUStep = 3 * kArC * 2;        // 48 bytes per step of u
constexpr int kArSStep = kArC * 4;            // 32 bytes per step of h or dL/dh
constexpr int kArUBox = kArL + kArK - 1;      // 19 steps
constexpr int kArHBox = kArL + kArK;          // 20 steps (one more: h_{t-1})
constexpr int kArGBox = kArL + kArK - 1;      // 19 steps
constexpr int kArUOff = 0, kArHOff = 1024, kArGOff = 1664;
constexpr int kArS = 2304;                    // chunk slot
constexpr int kArSmem = kArChunks * kArS;     // 73728
constexpr int kArMaxCluster = 8;
constexpr int kArTmax = kArSteps * kArMaxCluster;  // 4096
constexpr unsigned kArTileBytes =
    kArChunks * (kArUBox * kArUStep + kArHBox * kArSStep + kArGBox * kArSStep);
static_assert(kArUBox * kArUStep <= kArHOff && kArHOff + kArHBox * kArSStep <= kArGOff &&
                  kArGOff + kArGBox * kArSStep <= kArS && kArS % 128 == 0 &&
                  kArHOff % 128 == 0 && kArGOff % 128 == 0,
              "chunk slot layout");
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

__device__ __forceinline__ float2 af2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 afma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 amul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 aadd(float2 a, float2 b) { return __fadd2_rn(a, b); }

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
};

// affine map x -> P x + d, as float2 (P, d); (f o g)(x) = f(g(x))
__device__ __forceinline__ float2 ar_after(float2 f, float2 g) {
  return af2(f.x * g.x, fmaf(f.x, g.y, f.y));
}

struct ArCell {
  float2 AZ2, AR2, AC2, AZ, AR, AC;  // scaled (argument) and raw weights, both lanes
};

// The cell at a step pair: from the previous state HP and the pre-scaled
// arguments UZ, UR, UC, the Jacobian A = df/dh and the pieces
// GZ = df/du_z, GR = df/du_r, GC = df/du_c, RH = r h.
__device__ __forceinline__ void ar_cell(const ArCell& k, float2 HP, float2 UZ, float2 UR,
                                        float2 UC, float2& A, float2& GZ, float2& GR,
                                        float2& GC, float2& RH) {
  const float2 ONE = af2(1.f, 1.f), M1 = af2(-1.f, -1.f), M2 = af2(-2.f, -2.f);
  const float2 F4 = af2(4.f, 4.f), M4 = af2(-4.f, -4.f);
  const float2 TZ = afma(k.AZ2, HP, UZ), TR = afma(k.AR2, HP, UR);
  const float2 EZ = af2(ex2(fminf(TZ.x, 31.f)), ex2(fminf(TZ.y, 31.f)));
  const float2 ER = af2(ex2(fminf(TR.x, 31.f)), ex2(fminf(TR.y, 31.f)));
  const float2 PZ = aadd(ONE, EZ), PR = aadd(ONE, ER);
  const float2 PP = amul(PZ, PR);
  const float inv = rcp(PP.x * PP.y);
  const float2 INV = af2(PP.y * inv, PP.x * inv);
  const float2 Z = amul(PR, INV), R = amul(PZ, INV);
  RH = amul(R, HP);
  const float2 TC = afma(k.AC2, RH, UC);
  const float2 EC = af2(ex2(fminf(TC.x, 31.f)), ex2(fminf(TC.y, 31.f)));
  const float2 PC = aadd(ONE, EC);
  const float ic = rcp(PC.x * PC.y);
  const float2 TT = af2(PC.y * ic, PC.x * ic);
  const float2 C = afma(M2, TT, ONE);                 // tanh
  const float2 CMH = afma(HP, M1, C);
  const float2 OMZ = afma(Z, M1, ONE);
  const float2 ZZ = amul(Z, OMZ);                     // z(1-z)
  const float2 RR = amul(R, afma(R, M1, ONE));        // r(1-r)
  GZ = amul(CMH, ZZ);                                 // (c-h) z(1-z)
  GC = amul(Z, amul(TT, afma(TT, M4, F4)));           // z (1-c^2)
  const float2 GCA = amul(GC, k.AC);
  GR = amul(GCA, amul(HP, RR));                       // z(1-c^2) a_c h r(1-r)
  const float2 Q = afma(amul(k.AR, HP), RR, R);       // r + a_r h r(1-r)
  A = afma(GCA, Q, afma(amul(k.AZ, ZZ), CMH, OMZ));
}

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

// pre-scaled arguments of a step pair: -log2e u_z + b'_z, ... from bf16 rows
__device__ __forceinline__ void ar_args(const unsigned char* ux, const unsigned char* uy, float2 S,
                                        float2 BZ, float2 BR, float2 BC, float2& UZ, float2& UR,
                                        float2& UC) {
  const unsigned short* rx = reinterpret_cast<const unsigned short*>(ux);
  const unsigned short* ry = reinterpret_cast<const unsigned short*>(uy);
  const float2 SC = af2(2.f * kLog2e, 2.f * kLog2e);
  UZ = afma(S, af2(__uint_as_float((unsigned)rx[0] << 16), __uint_as_float((unsigned)ry[0] << 16)), BZ);
  UR = afma(S, af2(__uint_as_float((unsigned)rx[kArC] << 16),
                   __uint_as_float((unsigned)ry[kArC] << 16)), BR);
  UC = afma(SC, af2(__uint_as_float((unsigned)rx[2 * kArC] << 16),
                    __uint_as_float((unsigned)ry[2 * kArC] << 16)), BC);
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
      if (warp == 0 && kk == 0 && rank > 0) {
        const float2 m = ar_after(inc, cw);  // the CTA's map of channel c
        for (int r = 0; r < rank; ++r)
          ar_st_async_v2(ar_mapa(smem_u32(&sh.mbox[ms][rank][c]), r), m,
                         ar_mapa(smem_u32(&sh.mbar[ms]), r));
      }
      if (!mbar_wait_bounded(&sh.mbar[ms], (n / kArSlots) & 1, p.timeout_ns) && status == 0)
        status = PARARNN_STATUS_TIMEOUT;
#pragma unroll
      for (int r = CLS - 1; r > 0; --r) {
        if (r > rank) {
          const float2 m = sh.mbox[ms][r][c];
          cin_cta = fmaf(m.x, cin_cta, m.y);
        }
      }
      __syncwarp();
      if (tid == 0) mbar_arrive_expect_tx(&sh.mbar[ms], rx);
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

// da[g][d] and dbias[g][d]: per-CTA partials summed over batch rows and
// cluster ranks in a fixed order (bitwise reproducible).  One warp per
// output: lane j sums the terms j, j + 32, ... in order, then the 32 lane
// sums are added by a fixed shuffle tree.
__global__ void adjoint_row_reduce(const float* __restrict__ part, float* da, float* dbias, int B,
                                   int D, int cls) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // over 3 * D
  const int lane = threadIdx.x & 31;
  if (i >= 3 * D) return;
  const int g = i / D, d = i - g * D;
  const int nDTc = (D + kArC - 1) / kArC, dt = d / kArC, cc = d % kArC;
  const int nterm = B * cls;
  float sa = 0.f, sb = 0.f;
  for (int j = lane; j < nterm; j += 32) {
    const int b = j / cls, r = j - b * cls;
    const float* pp = part + ((size_t)(b * nDTc + dt) * cls + r) * (6 * kArC);
    sa += pp[g * kArC + cc];
    sb += pp[(3 + g) * kArC + cc];
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

int adjoint_row_cluster(int T) {
  if (T > kArTmax) return 0;
  int cls = 1;
  while (cls * kArSteps < T) cls *= 2;
  return cls;
}
int adjoint_row_channels() { return kArC; }
int adjoint_row_box_steps(int which) { return which == 0 ? kArUBox : (which == 1 ? kArHBox : kArGBox); }
size_t adjoint_row_part_bytes(int B, int T, int D) {
  return (size_t)B * ((D + kArC - 1) / kArC) * adjoint_row_cluster(T) * 6 * kArC * 4;
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
                       int T, int D, int* status, void* ws, cudaStream_t stream) {
  ArParams p;
  p.a = a;
  p.bias = bias;
  p.h0 = h0;
  p.du = du;
  p.dh0 = dh0;
  p.part = static_cast<float*>(ws);
  p.B = B;
  p.T = T;
  p.D = D;
  p.timeout_ns = 2000000000ull;
  p.status = status;
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
  adjoint_row_reduce<<<(3 * D * 32 + 255) / 256, 256, 0, stream>>>(p.part, da, dbias, B, D, cls);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
