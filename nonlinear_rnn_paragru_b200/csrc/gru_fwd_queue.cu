// gru_fwd_queue.cu -- fused Newton-scan ParaGRU solve of many 8-channel
// tiles with bf16 input projections: every sequence is cut into segments of
// NW * 128 steps, and all (tile, segment) items of the solve are worked off
// by one persistent launch from a queue.
//
// An item is 8 consecutive channels of one batch row over one segment.  Its
// Newton solve ("Параллельность RNN?", §1.2-§1.3) starts from the state the
// tile's previous segment converged to, exactly as a solve of the whole
// sequence would see it at convergence: the fixed point of the segment given
// its true initial state is the true trajectory over the segment.  A CTA of
// NW warps holds a segment: lane = (chunk k = lane / 8, channel c = lane % 8),
// a thread keeps its 32-step chunk's iterate and running Jacobian product in
// registers, and each iteration runs the cell pass of gru_row_pass.cuh, a
// shuffle scan over the warp's four chunks, one CTA barrier and a scan over
// the warps from shared memory, and the fix-up.  The item stops at the first
// exact evaluation whose residual over the item is below tol: after its
// update when the evaluation formed the step, or on the iterate itself when
// it was a residual-only check (the evaluation after an exact step from a
// residual at most sqrt(tol)).  At the cap it ends with a residual-only
// evaluation.
//
// Queue.  Items are numbered segment-major (item = s * ntiles + tile) and
// CTAs draw them from a counter one item ahead, so a CTA's items increase.
// Segment s of a tile may start only once segment s - 1 has stored its
// states: that CTA publishes the segment count of the tile with a release
// store after its stores, and the first chunk's threads of the successor
// wait for it with a bounded acquire poll before reading their initial state.
// The item with the lowest number that is not done is always being worked on
// and never waits (its predecessor has a lower number), so the queue cannot
// deadlock while all CTAs are resident; a wait that runs out sets TIMEOUT.
// With at least as many tiles as resident CTAs the predecessor of an item was
// drawn about a wave earlier and has normally finished.
//
// Data.  u arrives by NW / 2 TMA boxes of 256 steps into the top of the
// CTA's argument buffer and is expanded in place into fp32 gate arguments
// (the layout of gru_row_pass.cuh); the next item's boxes are issued as soon
// as the last pass of the current item is done, and prefetched into L2 when
// the item is drawn.  a and bias of the next item's channels are loaded
// while the current item runs.  Compared with one launch per segment, the
// queue leaves no SM idle at a segment boundary, and with four CTAs of four
// warps per SM the CTAs' barrier and load phases overlap other CTAs' passes.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "gru_row_pass.cuh"

namespace pararnn {

namespace {

constexpr unsigned kFull = 0xffffffffu;

struct QParams {
  const float* a;       // [3][D]
  const float* bias;    // [3][D] or null
  const float* h0;      // [B][D] or null
  float* h;             // [B][T][D]
  int B, T, D;
  int nDTc;             // 8-channel tiles per batch row
  int ntiles;           // B * nDTc
  int nseg;             // segments per sequence
  int nitems;           // ntiles * nseg (below 2^31: B*T*D <= 2^40)
  FastDiv dv_tiles, dv_ndtc;  // division by ntiles and by nDTc
  int max_iters;
  float tol;
  float apx_tau;
  float spec_tau;       // a residual-only check follows an exact step from at most this        // inexact evaluations while the item's residual is above this (0: none)
  uint64_t timeout_ns;
  unsigned* counter;    // item tickets (zero at launch)
  unsigned* seg_done;   // [ntiles] segments of each tile stored (zero at launch)
  int* chan_k;          // [B * D] or null
  pararnn_stats* stats;
  int withhold_item;    // testing: this item never publishes its segment (-1: none)
};

// NW warps per CTA, L steps per thread (chunk)
template <int NW, int L>
struct QCfg {
  static constexpr int kThreads = NW * 32;
  static constexpr int kH = L / 2;                          // step pairs per chunk
  static constexpr int kSteps = NW * kRowK * L;             // steps per item
  static constexpr int kChunks = kSteps / L;
  static constexpr int kS = 3 * L * kRowC * 4 + 64;         // chunk slot
  static constexpr int kU = kChunks * kS;                   // fp32 argument bytes
  static constexpr int kNBox = kSteps / kRowBox;
  static constexpr int kStage = kU - kNBox * kRowBoxBytes;  // bf16 staging at the top
  static constexpr int kBlocks = kChunks * kH / kThreads;   // expansion blocks
  static_assert(kNBox >= 1 && kSteps % kRowBox == 0, "whole TMA boxes per item");
  static_assert(kStage % 128 == 0 && kRowBoxBytes % 128 == 0, "TMA destinations");
  static_assert(kBlocks * kThreads == kChunks * kH, "the expansion: one (chunk, pair) per thread");
  // two blocks: block 0 (the first half of the chunks) writes below every
  // staged byte; one block reads everything before it writes anything
  static_assert(kBlocks == 1 || (kBlocks == 2 && (kChunks / 2) * kS <= kStage),
                "in-place expansion order");
  static_assert(kS % 128 == 64, "a warp's four chunks in alternate 64-byte bank halves");
  static_assert(kSteps * kRowC * 4 <= kStage, "the states' store buffer below the staging area");
  static_assert(NW == 4 || NW == 8, "the CTA's residual maximum is read as float4s");
};

template <int NW>
struct QShared {
  float2 wagg[2][NW][kRowC];   // per (warp, channel) inclusive map of the warp
  float wlast[2][NW][kRowC];   // per (warp, channel) last state before the update
  float wcm[2][NW][kRowC];     // per (warp, channel) max|r| (histogram)
  __align__(16) float wmax[2][NW];
  __align__(16) float par[2][6][kRowC];  // a (3 rows), bias (3 rows), by item parity
  uint64_t bar;                // the staging area's mbarrier
  int nx[2];                   // this and the next item, by item parity
};

// An item's segment, tile, batch row and first channel (item = segment *
// ntiles + tile, tile = row * nDTc + channel block), by multiply-high division
__device__ __forceinline__ int q_seg(const QParams& p, int item) {
  return fast_quot(item, p.dv_tiles);
}
__device__ __forceinline__ int q_tile(const QParams& p, int item) {
  return item - q_seg(p, item) * p.ntiles;
}
__device__ __forceinline__ int q_row(const QParams& p, int tile) {
  return fast_quot(tile, p.dv_ndtc);
}
__device__ __forceinline__ int q_d0(const QParams& p, int tile) {
  return (tile - q_row(p, tile) * p.nDTc) * kRowC;
}
__device__ __forceinline__ void q_issue(unsigned char* smem, int stage, int nbox, uint64_t* bar,
                                        const CUtensorMap* map, int b, int d0, int t0) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(bar, (unsigned)(nbox * kRowBoxBytes));
  for (int j = 0; j < nbox; ++j)
    tma_load_4d(smem + stage + j * kRowBoxBytes, map, bar, d0, 0, t0 + j * kRowBox, b);
}
__device__ __forceinline__ void q_prefetch(const CUtensorMap* map, int nbox, int b, int d0,
                                           int t0) {
  for (int j = 0; j < nbox; ++j)
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(d0), "r"(0), "r"(t0 + j * kRowBox), "r"(b)
                 : "memory");
}
// a[g][c] (j < 24) or bias[g][c] (j < 48, 0 when absent) of the tile at d0
__device__ __forceinline__ float q_param(const QParams& p, int j, int d0) {
  const int row = j / kRowC, c = j % kRowC;
  if (row < 3) return p.a[(size_t)row * p.D + d0 + c];
  return p.bias ? p.bias[(size_t)(row - 3) * p.D + d0 + c] : 0.f;
}
__device__ __forceinline__ int q_draw(unsigned* counter) {
  return (int)min(atomicAdd(counter, 1u), 0x7fffffffu);
}

template <int NW, int L, int MINB>
__global__ void __launch_bounds__(NW * 32, MINB)
    gru_newton_queue(const __grid_constant__ CUtensorMap map,
                     const __grid_constant__ CUtensorMap hmap, const QParams p) {
  using Cfg = QCfg<NW, L>;
  constexpr int kH = Cfg::kH;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ QShared<NW> sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane % kRowC, kk = lane / kRowC;
  const int q = warp * kRowK + kk;  // chunk index within the item
  const unsigned char* base = smem + q * Cfg::kS;

  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    sh.nx[0] = q_draw(p.counter);
  }
  __syncthreads();
  int item = sh.nx[0];
  if (item < p.nitems) {
    const int tile = q_tile(p, item);
    const int d0 = q_d0(p, tile);
    if (tid < 6 * kRowC) (&sh.par[0][0][0])[tid] = q_param(p, tid, d0);
    if (tid == 0)
      q_issue(smem, Cfg::kStage, Cfg::kNBox, &sh.bar, &map, q_row(p, tile), d0,
              q_seg(p, item) * Cfg::kSteps);
  }
  int status = 0;
  unsigned phase = 0;  // exchange phases so far, over all items
  int prev_item = -1;
  // CTA-uniform: 0 while the staged boxes arrive, else 1 + the phase parity of
  // the wait that ran out (no box is issued after that)
  int dead = 0;
  for (int n = 0; item < p.nitems; ++n) {
    __syncthreads();
    // publish the previous item: its states' bulk stores (issued by thread 0)
    // complete, then the proxy fence, the fence and the release order them
    // before the count.  The wait also frees the stores' shared memory before
    // this item's expansion writes there.  Warp 1 draws the next ticket
    // meanwhile: both wait on memory.
    if (tid == 0 && prev_item >= 0) {
      bulk_wait_all();
      if (prev_item != p.withhold_item) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        st_release(&p.seg_done[q_tile(p, prev_item)], (unsigned)q_seg(p, prev_item) + 1u);
      }
    }
    if (tid == 32) sh.nx[(n + 1) & 1] = q_draw(p.counter);
    const int pb = n & 1;
    const int tile = q_tile(p, item), seg = q_seg(p, item);
    const int b = q_row(p, tile), d0 = q_d0(p, tile);
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int t_base = seg * Cfg::kSteps;
    const int t_len = min(Cfg::kSteps, p.T - t_base);
    bool got = true;
    if (!dead) {
      got = mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns);
      if (!got) status = PARARNN_STATUS_TIMEOUT;
    }
    // a phase that did not complete is never re-armed: no more boxes then
    if (!dead && !__syncthreads_and(got)) dead = 1 + (n & 1);
    // ---- expand the staged bf16 rows [t][gate][8 ch] into fp32 arguments in
    // two blocks (each block's rows are read before any of its slots is
    // written; block 0 writes below all staging bytes)
    {
      const int qb = tid / kH, i = tid % kH;
      const int sw = row_swizzle(i);
#pragma unroll 1
      for (int blk = 0; blk < Cfg::kBlocks; ++blk) {
        const int qq = blk * (Cfg::kChunks / Cfg::kBlocks) + qb;
        const int ta = qq * L + i, tb = ta + kH;
        const bool pa = ta >= t_len, pbd = tb >= t_len;
        float xa[3][kRowC], xb[3][kRowC];
#pragma unroll
        for (int g = 0; g < 3; ++g) {
          const uint4 va = *reinterpret_cast<const uint4*>(
              smem + Cfg::kStage + (ta / kRowBox) * kRowBoxBytes + ((ta % kRowBox) * 3 + g) * 16);
          const uint4 vb = *reinterpret_cast<const uint4*>(
              smem + Cfg::kStage + (tb / kRowBox) * kRowBoxBytes + ((tb % kRowBox) * 3 + g) * 16);
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
        __syncthreads();
        unsigned char* dst = smem + qq * Cfg::kS + i * kRowC * 8;
#pragma unroll
        for (int g = 0; g < 3; ++g) {
          const float sc = (g == 2) ? 2.f * kLog2e : -kLog2e;
#pragma unroll
          for (int cc = 0; cc < kRowC; ++cc) {
            const float bs = sc * sh.par[pb][3 + g][cc];
            float2 o = ffma2(f2(sc, sc), f2(xa[g][cc], xb[g][cc]), f2(bs, bs));
            if (g == 0) {  // steps past the segment: z < 5e-10 whatever a_z h is
              if (pa) o.x = 3e30f;
              if (pbd) o.y = 3e30f;
            }
            *reinterpret_cast<float2*>(dst + g * kH * kRowC * 8 + (cc ^ sw) * 8) = o;
          }
        }
        __syncthreads();
      }
    }
    // the next item: its boxes prefetched into L2 and its parameters loaded
    // now, the parameters stored after the last pass
    const int pj = tid - 32;
    float pnext = 0.f;
    {
      const int next = sh.nx[(n + 1) & 1];
      if (next < p.nitems) {
        const int ntile = q_tile(p, next);
        const int nd0 = q_d0(p, ntile);
        if (tid == 0)
          q_prefetch(&map, Cfg::kNBox, q_row(p, ntile), nd0, q_seg(p, next) * Cfg::kSteps);
        if (pj >= 0 && pj < 6 * kRowC) pnext = q_param(p, pj, nd0);
      }
    }

    const float az = sh.par[pb][0][c], ar = sh.par[pb][1][c], ac = sh.par[pb][2][c];
    const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
    const float2 AZ2 = f2(az2, az2), AR2 = f2(ar2, ar2), AC2 = f2(ac2, ac2), AZ = f2(az, az);
    const bool first = (q == 0);  // the chunk holding the segment's first step
    // the segment's initial state: h0, or the last state of the previous
    // segment once that segment's CTA has published it
    float h0v = 0.f;
    if (first) {
      if (seg == 0) {
        h0v = (p.h0 && dval) ? p.h0[(size_t)b * p.D + d] : 0.f;
      } else {
        const unsigned* f = &p.seg_done[tile];
        if (ld_acquire(f) < (unsigned)seg) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire(f) < (unsigned)seg) {
            if (globaltimer_ns() - t0 > p.timeout_ns) {
              status = PARARNN_STATUS_TIMEOUT;
              break;
            }
          }
        }
        if (dval) h0v = __ldcg(p.h + ((size_t)b * p.T + t_base - 1) * p.D + d);
      }
    }

    float2 H[kH], P[kH];
#pragma unroll
    for (int i = 0; i < kH; ++i) {
      H[i] = f2(0.f, 0.f);
      P[i] = f2(1.f, 1.f);
    }
    float hb = first ? h0v : 0.f;  // state before this chunk
    // last_bad: updates applied before the last evaluation that left the
    // channel at or above tol (histogram); nupd: updates applied so far
    int last_bad = -1, updates = 0, k = 0, nupd = 0;
    float final_m = 0.f;
    bool apx = p.apx_tau > 0.f;  // CTA-uniform: set from the item's residual maximum
    // one Newton iteration of the item (kMode 0: exact evaluation and update,
    // 1: inexact evaluation and update, 2: exact residual only, at the cap or
    // as a check that certifies the iterate); true when the item is done
    auto iterate = [&](auto mode) -> bool {
      constexpr int kMode = decltype(mode)::value;
      constexpr bool resid_only = kMode == 2, apx_eval = kMode == 1;
      const int par = phase & 1;
      ++phase;
      const float last_pre = H[kH - 1].y;
      float2 DL, PA;
      float m;
      if constexpr (resid_only)
        m = row_pass<kH, false>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
      else if constexpr (apx_eval)
        m = row_pass_apx<kH>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
      else
        m = row_pass<kH, true>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
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
      float xP = __shfl_up_sync(kFull, IP, kRowC), xd = __shfl_up_sync(kFull, Id, kRowC);
      if (kk == 0) {
        xP = 1.f;
        xd = 0.f;
      }
      // residuals are >= 0 (or NaN with the sign cleared): their bit patterns
      // order like unsigned integers, NaN above +inf
      const unsigned wm = __reduce_max_sync(kFull, __float_as_uint(m));
      unsigned cmu = __float_as_uint(m);
      cmu = max(cmu, __shfl_xor_sync(kFull, cmu, 8));
      cmu = max(cmu, __shfl_xor_sync(kFull, cmu, 16));
      if (!resid_only && kk == kRowK - 1) {
        sh.wagg[par][warp][c] = make_float2(IP, Id);
        sh.wlast[par][warp][c] = last_pre;
      }
      if (kk == 0) sh.wcm[par][warp][c] = __uint_as_float(cmu);
      if (lane == 0) sh.wmax[par][warp] = __uint_as_float(wm);
      __syncthreads();
      if (q == 0) {  // the channel's own maximum over the item (histogram)
        float chm = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) chm = fmax_nan(chm, sh.wcm[par][w][c]);
        if (apx_eval || !(chm < p.tol)) last_bad = nupd;
      }
      // the delta entering this warp: the maps of the warps before it applied
      // to the zero delta entering the item; and the item's residual maximum
      float cd = 0.f;
#pragma unroll
      for (int w = 0; w < NW - 1; ++w) {
        if (w < warp) {
          const float2 a2 = sh.wagg[par][w][c];
          cd = fmaf(a2.x, cd, a2.y);
        }
      }
      float tmax = 0.f;
#pragma unroll
      for (int w4 = 0; w4 < NW; w4 += 4) {
        const float4 v = *reinterpret_cast<const float4*>(&sh.wmax[par][w4]);
        tmax = fmax_nan(tmax, fmax_nan(fmax_nan(v.x, v.y), fmax_nan(v.z, v.w)));
      }
      final_m = tmax;
      // an inexact evaluation never decides convergence; the first one whose
      // residual is at most apx_tau hands over to exact evaluations
      const bool own_ok = !apx_eval && tmax < p.tol;
      if (apx_eval && tmax <= p.apx_tau) apx = false;
      if constexpr (resid_only) {
        updates = nupd;
        const bool cap = k >= p.max_iters;
        if (cap && !own_ok && status == 0) status = PARARNN_STATUS_NOT_CONVERGED;
        // a check certifies below tol, as an exact evaluation that forms the
        // step does: a ParaGRU state stays inside (-1, 1), where the fp32
        // rounding of the states and of this evaluation is about 1e-7
        return cap || own_ok;
      }
      const float din = first ? 0.f : fmaf(xP, cd, xd);  // delta entering this chunk
      float prev_last = __shfl_up_sync(kFull, last_pre, kRowC);
      if (kk == 0) prev_last = (warp == 0) ? h0v : sh.wlast[par][warp - 1][c];
      hb = first ? h0v : prev_last + din;
      const float2 DIN = f2(din, fmaf(PA.x, din, DL.x));
#pragma unroll
      for (int i = 0; i < kH; ++i) H[i] = ffma2(P[i], DIN, H[i]);
      updates = ++nupd;
      return own_ok;
    };
    // inexact iterations while the residual is large, then exact ones to
    // convergence or the cap (k: the evaluation's index).  An exact step
    // from a residual at most spec_tau (sqrt(tol)) lands below tol with
    // quadratic convergence, so the evaluation after it is a residual-only
    // check: if it certifies, the item ends on that iterate without forming
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
    // every thread is past its last pass of this item (the barrier of the last
    // exchange): the staging area takes the next item
    const int next = sh.nx[(n + 1) & 1];
    if (tid == 0 && !dead && next < p.nitems) {
      const int ntile = q_tile(p, next);
      q_issue(smem, Cfg::kStage, Cfg::kNBox, &sh.bar, &map, q_row(p, ntile),
              q_d0(p, ntile), q_seg(p, next) * Cfg::kSteps);
    }
    if (pj >= 0 && pj < 6 * kRowC) (&sh.par[pb ^ 1][0][0])[pj] = pnext;
    // ---- states: from registers into the buffer below the staging area
    // ([step][8 ch], 16 KB; every pass is done and the next item's boxes
    // land above it), then two 256-step bulk-tensor stores (steps past T are
    // not written).  Indices re-derived from the item.
    item = sh.nx[n & 1];
    const int itile = q_tile(p, item), it_base = q_seg(p, item) * Cfg::kSteps;
    const int ib = q_row(p, itile), id = q_d0(p, itile) + c;
    const int it_len = min(Cfg::kSteps, p.T - it_base);
    bool bad = false;
    {
      float* sts = reinterpret_cast<float*>(smem);
      const int tq = q * L;
#pragma unroll
      for (int i = 0; i < kH; ++i) {
        sts[(tq + i) * kRowC + c] = H[i].x;
        sts[(tq + kH + i) * kRowC + c] = H[i].y;
        if (id < p.D) {
          bad |= tq + i < it_len && !isfinite(H[i].x);
          bad |= tq + kH + i < it_len && !isfinite(H[i].y);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (tid == 0) {
        const int d0i = q_d0(p, itile);
#pragma unroll
        for (int j = 0; j < Cfg::kNBox; ++j)
          tma_store_3d(&hmap, smem + j * kRowBox * kRowC * 4, d0i, it_base + j * kRowBox, ib);
        bulk_commit();
      }
    }
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    if (p.chan_k != nullptr && q == 0 && id < p.D)
      atomicMax(&p.chan_k[(size_t)ib * p.D + id], last_bad + 1);
    if (tid == 0) {
      atomicMax(&p.stats->iters, updates);
      atomicMax(&p.stats->evals, k + 1);
      atomicMax(reinterpret_cast<int*>(&p.stats->max_residual), __float_as_int(final_m));
    }
    prev_item = item;
    item = next;
  }
  __syncthreads();
  if (tid == 0 && prev_item >= 0) {
    bulk_wait_all();
    if (prev_item != p.withhold_item) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __threadfence();
      st_release(&p.seg_done[q_tile(p, prev_item)], (unsigned)q_seg(p, prev_item) + 1u);
    }
  }
  // boxes still in flight into the staging area: wait for them (bounded)
  if (dead && tid == 0) mbar_wait_bounded(&sh.bar, (unsigned)(dead - 1), p.timeout_ns);
  const int st = __reduce_max_sync(kFull, status);
  if (lane == 0 && st) atomicMax(&p.stats->status, st);
}

// the configuration the library runs: 4 warps per CTA, 32-step chunks
// (512-step segments), 4 CTAs per SM.  Measured on configuration 2 (B200,
// CUDA events): 345 us, against 354 us for 16-step chunks at 5 CTAs per SM
// (96 registers) and 366 us at 6 (80 registers, a few spills): more resident
// warps did not pay for the doubled per-step scan work.  8 warps per CTA
// (1024-step segments, 2 CTAs per SM) measured 6% slower: the per-item work
// halves per step, but every iteration's barrier spans twice the warps.
constexpr int kQW = 4, kQL = 32, kQMinB = 4;
using QRun = QCfg<kQW, kQL>;

int launch_queue(const CUtensorMap& map, const CUtensorMap& hmap, const QParams& p,
                 cudaStream_t stream) {
  auto kern = gru_newton_queue<kQW, kQL, kQMinB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, QRun::kU);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, sms = 148, per_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, QRun::kThreads, QRun::kU) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  cudaGetLastError();
  // persistent: every CTA resident at once (the queue's progress argument)
  const long long grid = std::min<long long>((long long)sms * per_sm, p.nitems);
  kern<<<(unsigned)std::max<long long>(grid, 1), QRun::kThreads, QRun::kU, stream>>>(map, hmap, p);
  return (int)cudaGetLastError();
}

}  // namespace

int gru_queue_steps() { return QRun::kSteps; }
int gru_queue_channels() { return kRowC; }
int gru_queue_box_steps() { return kRowBox; }

// Resident CTAs of the segment-queue solve on the current device (0 if it
// cannot run).
int gru_queue_resident() {
  int dev = 0, sms = 148, per_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = gru_newton_queue<kQW, kQL, kQMinB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, QRun::kU) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, QRun::kThreads, QRun::kU) !=
          cudaSuccess)
    per_sm = 0;
  cudaGetLastError();
  return sms * per_sm;
}

// One launch solves every segment of every tile; u is bf16 through `map`
// (boxes of 8 channels x 3 gates x 256 steps).  counter and seg_done must be
// zero at launch (ntiles entries of seg_done).
// hmap: the states h [B][T][D], box 8 channels x 256 steps
int launch_gru_queue(const CUtensorMap& map, const CUtensorMap& hmap, const FwdParams& f,
                     unsigned* counter, unsigned* seg_done, cudaStream_t stream) {
  QParams p;
  p.a = f.a;
  p.bias = f.bias;
  p.h0 = f.h0;
  p.h = f.h;
  p.B = f.B;
  p.T = f.T;
  p.D = f.D;
  p.nDTc = (f.D + kRowC - 1) / kRowC;
  p.ntiles = f.B * p.nDTc;
  p.dv_tiles = fast_div((unsigned)p.ntiles);
  p.dv_ndtc = fast_div((unsigned)p.nDTc);
  p.nseg = (f.T + QRun::kSteps - 1) / QRun::kSteps;
  if ((long long)p.ntiles * p.nseg >= (1LL << 31)) return 1;
  p.nitems = p.ntiles * p.nseg;
  p.max_iters = f.max_iters;
  p.tol = f.tol;
  p.apx_tau = (f.flags & PARARNN_FLAG_EXACT_STEPS) ? 0.f : kApxTau;
  p.spec_tau = f.tol > 0.f ? std::sqrt(f.tol) : -1.f;
  p.timeout_ns = f.timeout_ns;
  p.counter = counter;
  p.seg_done = seg_done;
  p.chan_k = f.chan_k;
  p.stats = f.stats;
  p.withhold_item = (f.flags & PARARNN_FLAG_INJECT_WITHHOLD) ? f.inject_chunk : -1;
  return launch_queue(map, hmap, p, stream);
}

}  // namespace pararnn
