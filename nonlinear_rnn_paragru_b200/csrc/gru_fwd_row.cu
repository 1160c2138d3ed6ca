// gru_fwd_row.cu -- fused Newton-scan ParaGRU solve for sequences (or
// segments of sequences) of up to 4096 steps with bf16 or fp32 input
// projections: 8 channels per CTA, a cluster of CLS = ceil(T / 1024) CTAs per
// tile, two CTAs per SM, the cell evaluated on packed fp32 pairs.
//
// A tile is 8 consecutive channels of one batch row over the steps this launch
// solves: the whole sequence, or one segment of it that starts from the state
// the segment before ended with (the host launches the segments in order).  CTA
// rank r of the cluster owns steps [1024 r, 1024 (r+1)) of them: 8 warps x 32
// lanes, lane = (k, c) with the channel c = lane % 8 fastest and k = lane / 8
// one of four 32-step chunks; warp w covers steps [128 w, 128 w + 128) of the
// CTA's range.  A thread keeps its chunk's iterate h and running Jacobian
// product P in registers (64 of its 128), and two CTAs share an SM so that one
// CTA's barriers and scans hide behind the other's cell evaluations.
//
// Per iteration ("Параллельность RNN?", §1.2-§1.3): each thread evaluates the
// cell, residual and diagonal Jacobian on its 32 steps and scans them serially
// (h'_t = f_t + A_t ds_{t-1}, running product P_t).  The 32 steps are taken
// as 16 pairs (i, i + 16): both halves of the chunk are scanned side by side
// from a zero incoming delta, so every add, multiply and fma of the cell and
// of the local scan is one packed fp32x2 instruction (each lane rounded as
// its scalar form); the second half is composed after the first when the
// chunk's map is formed and in the fix-up.  The chunk maps (P, ds) are
// scanned: over the four chunks of a warp by shuffles; over the 8 warps of the
// CTA after one CTA barrier, each thread composing the maps of the warps
// before its own from shared memory; over the CTAs of the cluster by remote
// asynchronous stores into the peers' mailboxes (the CTA's map and last state
// to the CTAs after it, its residual maximum to all), each completing on the
// receiver's mbarrier, so a CTA waits only for the bytes it needs and no
// cluster-wide barrier is taken per iteration.  The fix-up adds P_t ds_in.
// Mailboxes and per-warp data are double-buffered by the parity of a phase
// counter that runs on across tiles.  The cluster stops at the first exact
// evaluation whose residual over the tile is below tol: after its update
// when the evaluation formed the step, or on the iterate itself when it was
// a residual-only check (the evaluation after an exact step from a residual
// at most sqrt(tol)); at the cap it ends with a residual-only evaluation.
// The state before each chunk is re-anchored every iteration to its
// predecessor's pre-update last state plus the incoming delta.
//
// Data: bf16 u arrives by four TMA boxes of 256 steps into the top of the
// CTA's 98 KB buffer, fp32 u by four boxes that fill it from its start (the
// expansion then takes its second block first, so that it stays in place);
// the next tile's boxes are prefetched into L2 meanwhile; a, bias and
// h0 of the next tile's channels are read with plain loads a tile ahead into
// a double-buffered block.  Once per tile u is expanded in place into the
// fp32 arguments -log2e u_z + b'_z, -log2e u_r + b'_r, 2 log2e u_c + b'_c
// (b' the bias scaled alike), stored per chunk as [gate][pair i][channel]
// {step i, step i + 16}: one 8-byte load per gate and pair, channel c at slot
// c ^ ((i >> 1) & 7) of its pair row so that the expansion's stores are free
// of bank conflicts.  Chunk slots are 3136 bytes, so the four chunks a warp
// reads fall in alternate 64-byte bank halves.  Steps past T get a z argument
// of 3e30 (clamped to 31), so z < 5e-10 and f(h) = h.
// Clusters are persistent over tiles; the next tile's boxes are issued as
// soon as the last pass of the current tile is done.  States are stored
// straight from registers (the 8 lanes of a chunk write a 32-byte run).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "gru_row_pass.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cgs = cooperative_groups;

constexpr int kRowThreads = 256;
constexpr int kRowWarps = 8;
constexpr int kRowSteps = kRowWarps * kRowK * kRowL;  // 1024 steps per CTA
constexpr int kRowChunks = kRowSteps / kRowL;         // 32 chunks per CTA
constexpr int kRowU = kRowChunks * kRowS;             // 100352: the tile's fp32 arguments
constexpr int kRowNBox = kRowSteps / kRowBox;         // 4
constexpr int kRowStage = kRowU - kRowNBox * kRowBoxBytes;  // bf16 staging at the top
constexpr int kRowSmem = kRowU;
constexpr int kRowMaxCluster = 4;
constexpr int kRowTmax = kRowSteps * kRowMaxCluster;  // 4096
static_assert(kRowStage % 128 == 0 && kRowBoxBytes % 128 == 0, "TMA destinations");
static_assert(kRowThreads == (kRowChunks / 2) * kRowH, "the expansion: one (chunk, pair) per thread");
// expansion block 0 (chunks below kRowChunks / 2) writes below every staged byte
static_assert((kRowChunks / 2) * kRowS <= kRowStage, "in-place expansion order");
// fp32 u: the four 256-step boxes fill the buffer from its start (96 bytes a
// step); the expansion takes block 1 first, whose slots lie above every row
// of block 0, then block 0, whose slots reach into block 1's rows only
constexpr int kRowBoxBytesF32 = kRowBox * 3 * kRowC * 4;    // 24576
static_assert(kRowNBox * kRowBoxBytesF32 <= kRowU &&
                  (kRowChunks / 2) * kRowS >= (kRowChunks / 2) * kRowL * 3 * kRowC * 4,
              "in-place fp32 expansion order");

struct RowMailbox {  // written by the cluster peers with remote async stores
  float4 map[kRowMaxCluster][kRowC];   // (P, ds, last state before the update, -) by rank
  float cmax[kRowMaxCluster];          // CTA max|r| by rank
};

struct RowShared {
  float2 wagg[2][kRowWarps][kRowC];  // per (warp, channel) inclusive map of the warp
  float wlast[2][kRowWarps][kRowC];  // per (warp, channel): last state before the update
  float wmax[2][kRowWarps];
  float wcm[2][kRowWarps][kRowC];    // per (warp, channel) max|r| (histogram)
  __align__(16) RowMailbox mbox[2];
  // a (3 rows), bias (3 rows), h0 of a tile's channels, by tile parity
  __align__(16) float par[2][7][kRowC];
  uint64_t bar;                      // the staging buffer's mbarrier
  uint64_t mbar[2];                  // mailbox mbarriers, by parity
  int ntile[4];                      // tile indices published by cluster rank 0
};

// shared::cluster address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_u32(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// remote asynchronous stores that complete on the receiver's mbarrier
__device__ __forceinline__ void st_async_v4(uint32_t raddr, float4 v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(raddr), "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)),
      "r"(__float_as_uint(v.z)), "r"(__float_as_uint(v.w)), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void st_async_b32(uint32_t raddr, unsigned v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
               ::"r"(raddr), "r"(v), "r"(rbar)
               : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Thread 0: load the tile's four 256-step boxes for CTA `rank` into the
// staging area, on `bar`.
// The tile's boxes that hold steps of this CTA's range (nbox of them, 0 to
// 4; the expansion takes steps past the range as zeros).
template <bool kF32>
__device__ __forceinline__ void row_issue(unsigned char* smem, RowShared& sh,
                                          const CUtensorMap* map, int b, int d0, int t0,
                                          int nbox) {
  constexpr int kStage = kF32 ? 0 : kRowStage, kBox = kF32 ? kRowBoxBytesF32 : kRowBoxBytes;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(&sh.bar, (unsigned)(nbox * kBox));
  for (int j = 0; j < nbox; ++j)
    tma_load_4d(smem + kStage + j * kBox, map, &sh.bar, d0, 0, t0 + j * kRowBox, b);
}
// Parameter j (0..55) of the tile at (b, d0): a[g][c] (j < 24), bias[g][c]
// (j < 48, 0 when absent), h0[c] (0 when absent).
__device__ __forceinline__ float row_param(const FwdParams& p, int j, int b, int d0) {
  const int row = j / kRowC, c = j % kRowC;
  if (row < 3) return p.a[(size_t)row * p.D + d0 + c];
  if (row < 6) return p.bias ? p.bias[(size_t)(row - 3) * p.D + d0 + c] : 0.f;
  return p.h0 ? p.h0[(size_t)b * p.ld_h0 + d0 + c] : 0.f;
}
// L2 prefetch of a tile's boxes (no shared memory touched).
__device__ __forceinline__ void row_prefetch(const CUtensorMap* map, int b, int d0, int t0,
                                             int nbox) {
  for (int j = 0; j < nbox; ++j)
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(d0), "r"(0), "r"(t0 + j * kRowBox), "r"(b)
                 : "memory");
}
// Bytes a CTA of rank `rank` receives per exchange phase: the maps of the CTAs
// before it and the residual maximum of every other CTA.
__host__ __device__ constexpr unsigned row_rx_bytes(int rank, int cls) {
  return (unsigned)(rank * kRowC * 16 + (cls - 1) * 4);
}

template <int CLS, bool kF32>
__global__ void __launch_bounds__(kRowThreads, 2)
    gru_newton_row(const __grid_constant__ CUtensorMap map, const FwdParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ RowShared sh;
  cgs::cluster_group cluster = cgs::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (CLS > 1) ? (int)cluster.block_rank() : 0;
  const int c = lane % kRowC, kk = lane / kRowC;
  const int q = warp * kRowK + kk;           // chunk index within the CTA
  const int nDTc = (p.D + kRowC - 1) / kRowC;
  const int ntiles = p.B * nDTc;
  const int nclus = gridDim.x / CLS, clus = blockIdx.x / CLS;
  const int t0 = rank * kRowSteps;           // first step of this CTA in the segment
  const int tg0 = p.t_base + t0;             // ... in the sequence
  // boxes of this CTA's range that hold steps of the segment
  const int nbox = min(kRowNBox, max(0, (p.t_len - t0 + kRowBox - 1) / kRowBox));
  const unsigned rx = row_rx_bytes(rank, CLS);

  // the first tile's parameters; later tiles' are loaded a tile ahead
  if (tid < 7 * kRowC && clus < ntiles) {
    const int b = clus / nDTc;
    (&sh.par[0][0][0])[tid] = row_param(p, tid, b, (clus - b * nDTc) * kRowC);
  }
  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    if (CLS > 1) {
      mbar_init(&sh.mbar[0], 1);
      mbar_init(&sh.mbar[1], 1);
      mbar_arrive_expect_tx(&sh.mbar[0], rx);
      mbar_arrive_expect_tx(&sh.mbar[1], rx);
    }
  }
  __syncthreads();
  // the peers' mailbox barriers are armed before anyone sends
  if (CLS > 1) cluster.sync();
  if (tid == 0 && clus < ntiles) {
    const int b = clus / nDTc;
    row_issue<kF32>(smem, sh, &map, b, (clus - b * nDTc) * kRowC, tg0, nbox);
  }
  const unsigned char* base = smem + q * kRowS;
  int status = 0;
  int n = 0;
  unsigned phase = 0;  // exchange phases so far, over all tiles
  // Tiles: the first two of a cluster are clus and clus + nclus; after that
  // each cluster takes the next ticket of a counter (zero at launch), so
  // clusters that meet slowly converging tiles take fewer.  Cluster rank 0
  // draws the ticket for tile n + 2 at the start of tile n and publishes it
  // into every CTA's ring at the end of tile n; the barrier opening each tile
  // makes it visible.  Tickets rise monotonically, so no tile is skipped.
  const bool drawer = rank == 0 && tid == kRowThreads - 32;
  // even and odd segments draw from two counters; each launch zeroes the one
  // the next segment's launch will draw from (the solve's first counter is
  // zeroed before the first launch)
  if (blockIdx.x == 0 && tid == 0) *((p.seg & 1) ? &p.hdr->ticket : &p.hdr->ticket_odd) = 0u;
  unsigned ticket = 0;
  int tile = clus, next = clus + nclus;
  for (; tile < ntiles; tile = next, ++n) {
    if (CLS > 1)
      cluster.sync();
    else
      __syncthreads();
    if (n >= 1) next = sh.ntile[(n + 1) & 3];
    if (drawer) ticket = atomicAdd((p.seg & 1) ? &p.hdr->ticket_odd : &p.hdr->ticket, 1u);
    // the next tile's parameters: loaded now, stored at the end of this tile
    const int pj = tid - 32;
    float pnext = 0.f;
    if (pj >= 0 && pj < 7 * kRowC && next < ntiles) {
      const int b2 = next / nDTc;
      pnext = row_param(p, pj, b2, (next - b2 * nDTc) * kRowC);
    }
    const int pb = n & 1;
    const int b = tile / nDTc, d0 = (tile - b * nDTc) * kRowC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    if (tid == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      row_prefetch(&map, b2, (next - b2 * nDTc) * kRowC, tg0, nbox);
    }
    if (!mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;
    // ---- expand the staged bf16 rows [t][gate][8 ch] into the fp32 arguments
    // in two blocks of 512 steps (each block's rows are read before any of
    // its slots is written; block 0 writes below all staging bytes).  Thread
    // (qb, i) takes steps i and i + 16 of chunk qb of the block.
    {
      const int qb = tid / kRowH, i = tid % kRowH;
      const int sw = row_swizzle(i);
#pragma unroll 1
      for (int bi = 0; bi < 2; ++bi) {
        const int blk = kF32 ? 1 - bi : bi;  // fp32: block 1 first (in place)
        const int qq = blk * (kRowChunks / 2) + qb;
        const int ta = qq * kRowL + i, tb = ta + kRowH;  // steps within the CTA
        const bool pa = t0 + ta >= p.t_len, pbd = t0 + tb >= p.t_len;
        // the 8 channels of gate g at steps ta (xa) and tb (xb) from the
        // staged rows (bf16 at the top of the buffer, fp32 from its start)
        float xa[3][kRowC], xb[3][kRowC];
        if (kF32) {
#pragma unroll
          for (int g = 0; g < 3; ++g) {
            const float4* ra = reinterpret_cast<const float4*>(smem + (ta * 3 + g) * kRowC * 4);
            const float4* rb = reinterpret_cast<const float4*>(smem + (tb * 3 + g) * kRowC * 4);
            const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 a0 = pa ? z4 : ra[0], a1 = pa ? z4 : ra[1];
            const float4 b0 = pbd ? z4 : rb[0], b1 = pbd ? z4 : rb[1];
            const float fa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float fb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int cc = 0; cc < kRowC; ++cc) {
              xa[g][cc] = fa[cc];
              xb[g][cc] = fb[cc];
            }
          }
        } else {
#pragma unroll
          for (int g = 0; g < 3; ++g) {
            const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
            const uint4 va = pa ? z4 : *reinterpret_cast<const uint4*>(
                smem + kRowStage + (ta / kRowBox) * kRowBoxBytes + ((ta % kRowBox) * 3 + g) * 16);
            const uint4 vb = pbd ? z4 : *reinterpret_cast<const uint4*>(
                smem + kRowStage + (tb / kRowBox) * kRowBoxBytes + ((tb % kRowBox) * 3 + g) * 16);
            const unsigned wa[4] = {va.x, va.y, va.z, va.w};
            const unsigned wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
            for (int cc = 0; cc < kRowC; ++cc) {
              const int sh16 = (cc & 1) ? 0 : 16;
              const unsigned mk = (cc & 1) ? 0xffff0000u : 0xffffffffu;
              xa[g][cc] = __uint_as_float((wa[cc >> 1] << sh16) & mk);
              xb[g][cc] = __uint_as_float((wb[cc >> 1] << sh16) & mk);
            }
          }
        }
        __syncthreads();
        unsigned char* dst = smem + qq * kRowS + i * kRowC * 8;
#pragma unroll
        for (int g = 0; g < 3; ++g) {
          const float sc = (g == 2) ? 2.f * kLog2e : -kLog2e;
#pragma unroll
          for (int cc = 0; cc < kRowC; ++cc) {
            const float bs = sc * sh.par[pb][3 + g][cc];
            float2 o = ffma2(f2(sc, sc), f2(xa[g][cc], xb[g][cc]), f2(bs, bs));
            if (g == 0) {  // steps past T: z < 5e-10 whatever a_z h is
              if (pa) o.x = 3e30f;
              if (pbd) o.y = 3e30f;
            }
            *reinterpret_cast<float2*>(dst + g * kRowH * kRowC * 8 + (cc ^ sw) * 8) = o;
          }
        }
        __syncthreads();
      }
    }
    const float az = sh.par[pb][0][c], ar = sh.par[pb][1][c], ac = sh.par[pb][2][c];
    const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
    const float2 AZ2 = f2(az2, az2), AR2 = f2(ar2, ar2), AC2 = f2(ac2, ac2), AZ = f2(az, az);
    const float h0v = sh.par[pb][6][c];
    const bool first = (rank == 0 && q == 0);  // chunk holding step 0

    float2 H[kRowH], P[kRowH];
#pragma unroll
    for (int i = 0; i < kRowH; ++i) {
      H[i] = f2(0.f, 0.f);
      P[i] = f2(1.f, 1.f);
    }
    float hb = first ? h0v : 0.f;  // state before this chunk
    // last_bad: updates applied before the last evaluation that left the
    // channel at or above tol (histogram); nupd: updates applied so far
    int last_bad = -1, updates = 0, k = 0, nupd = 0;
    float final_m = 0.f;
    bool apx = p.apx_tau > 0.f;  // cluster-uniform: set from the tile's residual maximum
    // one Newton iteration of the tile (kMode 0: exact evaluation and update,
    // 1: inexact evaluation and update, 2: exact residual only, at the cap or
    // as a check that certifies the iterate); true when the tile is done
    auto iterate = [&](auto mode) -> bool {
      constexpr int kMode = decltype(mode)::value;
      constexpr bool resid_only = kMode == 2, apx_eval = kMode == 1;
      const bool cap = resid_only && k >= p.max_iters;
      const int par = phase & 1;
      const unsigned mpar = (phase >> 1) & 1;  // phase parity of mbar[par]
      ++phase;
      const float last_pre = H[kRowH - 1].y;
      float2 DL, PA;
      float m;
      if constexpr (resid_only)
        m = row_pass<kRowH, false>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
      else if constexpr (apx_eval)
        m = row_pass_apx<kRowH>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
      else
        m = row_pass<kRowH, true>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
      if (!dval) m = 0.f;
      // the chunk's map: second half after the first
      float IP = PA.y * PA.x, Id = fmaf(PA.y, DL.x, DL.y);
      // inclusive scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
      for (int o = kRowC; o < 32; o <<= 1) {
        const float oP = __shfl_up_sync(kFull, IP, o), od = __shfl_up_sync(kFull, Id, o);
        if (lane >= o) {
          Id = fmaf(IP, od, Id);
          IP *= oP;
        }
      }
      // exclusive: the delta entering the warp -> the delta entering this chunk
      float xP = __shfl_up_sync(kFull, IP, kRowC), xd = __shfl_up_sync(kFull, Id, kRowC);
      if (kk == 0) {
        xP = 1.f;
        xd = 0.f;
      }
      // residuals are >= 0 (or NaN with the sign cleared): their bit patterns
      // order like unsigned integers, NaN above +inf
      const unsigned wm = __reduce_max_sync(kFull, __float_as_uint(m));
      // the channel's maximum over the warp's four chunks (lanes c + 8k)
      unsigned cmu = __float_as_uint(m);
      cmu = max(cmu, __shfl_xor_sync(kFull, cmu, 8));
      cmu = max(cmu, __shfl_xor_sync(kFull, cmu, 16));
      if (kk == kRowK - 1) {
        sh.wagg[par][warp][c] = make_float2(IP, Id);
        sh.wlast[par][warp][c] = last_pre;
      }
      if (kk == 0) sh.wcm[par][warp][c] = __uint_as_float(cmu);
      if (lane == 0) sh.wmax[par][warp] = __uint_as_float(wm);
      __syncthreads();
      // the histogram input: the channel's own maximum over this CTA's steps
      // (warp 0, lanes 0..7 track it; the other CTAs of the cluster track
      // theirs and the per-channel index is the maximum over them)
      if (q == 0) {
        float chm = 0.f;
#pragma unroll
        for (int w = 0; w < kRowWarps; ++w) chm = fmax_nan(chm, sh.wcm[par][w][c]);
        if (apx_eval || !(chm < p.tol)) last_bad = nupd;
      }
      // maps of the warps before this one: CTA incoming delta -> delta
      // entering this warp; and the CTA's residual maximum
      float cP = 1.f, cd = 0.f;
#pragma unroll
      for (int w = 0; w < kRowWarps - 1; ++w) {
        if (w < warp) {
          const float2 a2 = sh.wagg[par][w][c];
          cd = fmaf(a2.x, cd, a2.y);
          cP *= a2.x;
        }
      }
      const float4 wm0 = *reinterpret_cast<const float4*>(&sh.wmax[par][0]);
      const float4 wm1 = *reinterpret_cast<const float4*>(&sh.wmax[par][4]);
      float tmax = fmax_nan(fmax_nan(fmax_nan(wm0.x, wm0.y), fmax_nan(wm0.z, wm0.w)),
                            fmax_nan(fmax_nan(wm1.x, wm1.y), fmax_nan(wm1.z, wm1.w)));
      float din_cta = 0.f;          // delta entering this CTA
      float prev_cta_last = h0v;    // state before this CTA's first step
      if (CLS > 1) {
        // testing: the CTA of rank inject_chunk withholds its last exchange
        // (the residual-only evaluation at the cap), so its peers' bounded
        // waits run out
        const bool withhold =
            cap && (p.flags & PARARNN_FLAG_INJECT_WITHHOLD) && rank == p.inject_chunk;
        if (warp == kRowWarps - 1 && !withhold) {
          // the CTA map of channel c: last warp's inclusive map after the
          // warps before it; to every CTA after this one.  Lanes r < CLS
          // send the residual maximum to CTA r.
          const float cmax = tmax;
          if (kk == kRowK - 1) {
            const float4 v = make_float4(IP * cP, fmaf(IP, cd, Id), last_pre, 0.f);
            for (int r = rank + 1; r < CLS; ++r)
              st_async_v4(mapa_u32(smem_u32(&sh.mbox[par].map[rank][c]), r), v,
                          mapa_u32(smem_u32(&sh.mbar[par]), r));
          }
          if (lane < CLS && lane != rank)
            st_async_b32(mapa_u32(smem_u32(&sh.mbox[par].cmax[rank]), lane),
                         __float_as_uint(cmax), mapa_u32(smem_u32(&sh.mbar[par]), lane));
        }
        const bool got = mbar_wait_bounded(&sh.mbar[par], mpar, p.timeout_ns);
        if (!got && status == 0) status = PARARNN_STATUS_TIMEOUT;
#pragma unroll
        for (int r = 0; r < CLS; ++r) {
          if (r != rank) tmax = fmax_nan(tmax, sh.mbox[par].cmax[r]);
          if (r < rank) {
            const float4 a4 = sh.mbox[par].map[r][c];
            din_cta = fmaf(a4.x, din_cta, a4.y);
            if (r == rank - 1) prev_cta_last = a4.z;
          }
        }
        // re-arm this mailbox for its next phase; every thread of the CTA
        // has passed the wait before any peer can send that phase's bytes.
        // A phase that did not complete is not re-armed (a second arrival on
        // it would be one more than the barrier counts): later waits on it
        // run out too and the solve reports TIMEOUT.
        __syncwarp();
        if (tid == 0 && got) mbar_arrive_expect_tx(&sh.mbar[par], rx);
      }
      final_m = tmax;
      // an inexact evaluation never decides convergence; the first one whose
      // residual is at most apx_tau hands over to exact evaluations
      const bool own_ok = !apx_eval && tmax < p.tol;
      if (apx_eval && tmax <= p.apx_tau) apx = false;
      if constexpr (resid_only) {
        updates = nupd;
        if (cap && !own_ok && status == 0) status = PARARNN_STATUS_NOT_CONVERGED;
        return cap || own_ok;
      }
      const float cin = fmaf(cP, din_cta, cd);  // delta entering this warp
      const float din = first ? 0.f : fmaf(xP, cin, xd);
      float prev_last = __shfl_up_sync(kFull, last_pre, kRowC);
      if (kk == 0) prev_last = (warp == 0) ? prev_cta_last : sh.wlast[par][warp - 1][c];
      hb = first ? h0v : prev_last + din;
      // deltas entering the two halves of the chunk
      const float2 DIN = f2(din, fmaf(PA.x, din, DL.x));
#pragma unroll
      for (int i = 0; i < kRowH; ++i) H[i] = ffma2(P[i], DIN, H[i]);
      updates = ++nupd;
      return own_ok;
    };
    // inexact iterations while the residual is large, then exact ones to
    // convergence or the cap (k: the evaluation's index).  An exact step
    // from a residual at most spec_tau (sqrt(tol)) lands below tol with
    // quadratic convergence, so the evaluation after it is a residual-only
    // check: if it certifies, the tile ends on that iterate without forming
    // the step; if not, the next evaluation forms the step at the same
    // iterate.
    for (; apx && k < p.max_iters; ++k) iterate(std::integral_constant<int, 1>{});
    bool spec = false;
    for (;; ++k) {
      if (k >= p.max_iters) {
        iterate(std::integral_constant<int, 2>{});
        break;
      }
      if (spec) {
        spec = false;
        if (iterate(std::integral_constant<int, 2>{})) break;
        continue;
      }
      if (iterate(std::integral_constant<int, 0>{})) break;
      spec = final_m <= p.spec_tau;
    }
    // every thread of the CTA is past its last pass of this tile (the
    // barrier of the last exchange): the staging area takes the next tile
    if (tid == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      row_issue<kF32>(smem, sh, &map, b2, (next - b2 * nDTc) * kRowC, tg0, nbox);
    }
    if (pj >= 0 && pj < 7 * kRowC) (&sh.par[pb ^ 1][0][0])[pj] = pnext;

    if (drawer) {
      const int nt = 2 * nclus + (int)ticket;
      for (int r = 0; r < CLS; ++r) {
        int* dst = (r == rank) ? &sh.ntile[(n + 2) & 3] : cluster.map_shared_rank(&sh.ntile[(n + 2) & 3], r);
        *dst = nt;
      }
    }
    // ---- states straight from registers
    bool bad = false;
    if (dval) {
      const int tq = t0 + q * kRowL;
      float* out = p.h + ((size_t)b * p.T + p.t_base + tq) * p.D + d;
#pragma unroll
      for (int i = 0; i < kRowH; ++i) {
        if (tq + i < p.t_len) {
          out[(size_t)i * p.D] = H[i].x;
          bad |= !isfinite(H[i].x);
        }
        if (tq + kRowH + i < p.t_len) {
          out[(size_t)(kRowH + i) * p.D] = H[i].y;
          bad |= !isfinite(H[i].y);
        }
      }
    }
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    if (p.chan_k != nullptr && q == 0 && dval)
      atomicMax(&p.chan_k[(size_t)b * p.D + d], last_bad + 1);
    if (tid == 0) {
      atomicMax(&p.stats->iters, updates);
      atomicMax(&p.stats->evals, k + 1);
      atomicMax(reinterpret_cast<int*>(&p.stats->max_residual), __float_as_int(final_m));
    }
  }
  const int st = __reduce_max_sync(kFull, status);
  if (lane == 0 && st) atomicMax(&p.stats->status, st);
  // no CTA leaves while a peer may still store into its mailboxes
  if (CLS > 1) cluster.sync();
}

// ------------------------------------------------------------- launcher --
// CTAs per cluster for sequences of length T; 0 when this solve does not apply
int gru_row_cluster(int T) {
  return T <= 1024 ? 1 : (T <= 2048 ? 2 : (T <= kRowTmax ? 4 : 0));
}
int gru_row_box_steps() { return kRowBox; }
int gru_row_channels() { return kRowC; }

template <int CLS, bool kF32>
static int launch_row_t(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream) {
  const long long ntiles = (long long)p.B * ((p.D + kRowC - 1) / kRowC);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = gru_newton_row<CLS, kF32>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRowSmem);
  if (e != cudaSuccess) return (int)e;
  // persistent clusters: as many as can be resident (two CTAs per SM), at
  // most one per tile
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kRowThreads);
  cfg.dynamicSmemBytes = kRowSmem;
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
  return (int)cudaLaunchKernelEx(&cfg, kern, map, p);
}

// One launch solves steps [p.t_base, p.t_base + p.t_len) (t_len <= 4096) of
// every tile; u is bf16 through `map` or, with f32, read from p.u.
int launch_gru_row(const CUtensorMap& map, const FwdParams& p, bool f32, cudaStream_t stream) {
  switch (gru_row_cluster(p.t_len)) {
    case 1: return f32 ? launch_row_t<1, true>(map, p, stream) : launch_row_t<1, false>(map, p, stream);
    case 2: return f32 ? launch_row_t<2, true>(map, p, stream) : launch_row_t<2, false>(map, p, stream);
    case 4: return f32 ? launch_row_t<4, true>(map, p, stream) : launch_row_t<4, false>(map, p, stream);
    default: return 1;
  }
}
int gru_row_max_steps() { return kRowTmax; }
// steps one CTA holds: a cluster of k CTAs solves up to k times this many
int gru_row_cta_steps() { return kRowSteps; }

}  // namespace pararnn
