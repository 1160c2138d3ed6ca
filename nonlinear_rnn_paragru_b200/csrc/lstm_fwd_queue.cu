// lstm_fwd_queue.cu -- fused Newton-scan ParaLSTM solve of many 8-channel
// tiles with bf16 input projections: every sequence is cut into 128-step
// segments, and all (tile, segment) items of the solve are worked off by one
// persistent launch from a queue.
//
// An item is 8 consecutive channels of one batch row over one segment; its
// Newton solve ("Параллельность RNN?", §1.2-§1.3) starts from the state
// (c, h) the tile's previous segment converged to.  A CTA of 4 warps holds a
// segment: lane = (chunk k = lane / 8, channel c = lane % 8), a thread keeps
// its 8-step chunk's iterate (c, h) and the running products P of the 2x2
// Jacobians in registers, taken as 4 packed step pairs (i, i + 4) so that
// every add, multiply and fma is one fp32x2 instruction (each lane rounded
// as its scalar form).  Each iteration: the cell pass, a shuffle scan of the
// chunk maps (2x2 matrix, 2-vector) over the warp's four chunks, one CTA
// barrier and a composition over the warps from shared memory, and the
// fix-up.  The item stops at the first exact evaluation whose residual over
// the item is below tol: after its update when the evaluation formed the
// step, or on the iterate itself when it was a residual-only check below
// tol / 2 (the evaluation after an exact step from a residual at most
// sqrt(tol / 2)).  At the cap it ends with a residual-only evaluation.
//
// Inexact early evaluations.  While the item's max |r| is above 0.1 the cell
// is evaluated with the one-instruction tanh (sigma(x) = 1/2 + 1/2 tanh(x/2);
// gates within about 2^-11 relative), then exactly: an ex2 and a reciprocal
// per gate and per tanh(c'), sigma(x) = 1 / (1 + 2^(-x log2 e)) and
// tanh(y) = 1 - 2 / (1 + 2^(2y log2 e)).  Unclamped, a saturating argument
// gives 2^x = inf and a reciprocal of 0, the gate's limit, and a NaN stays
// NaN.  (Sharing one reciprocal between the six sigmoids of a step pair
// needed a clamp per argument and a longer dependency chain: 1% slower.)
// Only exact evaluations decide convergence.  PARARNN_FLAG_EXACT_STEPS makes
// every evaluation exact.
//
// Queue.  Items are numbered segment-major (item = s * ntiles + tile) and
// drawn from a counter one ahead, so a CTA's items increase.  Segment s of a
// tile starts once segment s - 1 has stored its states: that CTA publishes the
// tile's segment count with a release store after its stores, and the first
// chunk's threads of the successor wait for it with a bounded acquire poll.
// The item with the lowest number that is not done is always being worked on
// and never waits, so the queue cannot deadlock while all CTAs are resident;
// a wait that runs out sets TIMEOUT.
//
// Registers and occupancy.  Eight steps per thread keep a thread's state at
// 48 registers, so four CTAs of 4 warps share an SM (16 warps), against one
// CTA of 8 warps with 16 steps per thread in the whole-sequence kernel.
//
// Data.  u arrives by one TMA box of 128 steps into a staging area, is
// expanded into fp32 arguments (-log2e u + b' for i, f, o; 2 log2e u + b' for
// g) laid out per chunk q as [gate][pair i][channel] {step i, step i + 4},
// channel c at slot c ^ ((q + 2 (i >> 1)) & 7): the expansion's lanes, which
// cover 8 chunks x 4 pairs of one channel, then write each 256-byte row
// with every bank pair twice, and a warp's reads in the pass stay one
// 64-byte window per chunk.  The next item's box is issued as soon
// as the expansion is done.  a, bias (and c0, h0 for a first segment) of the
// next item's channels are loaded during the current item.  Steps past T get
// i and o shut and f open.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <type_traits>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace {

constexpr unsigned kLqFull = 0xffffffffu;
constexpr int kLqC = 8;                             // channels per tile
constexpr int kLqK = 32 / kLqC;                     // chunks per warp
constexpr int kLqW = 4;                             // warps per CTA
constexpr int kLqThreads = kLqW * 32;
constexpr int kLqL = 8;                             // steps per chunk (per thread)
constexpr int kLqH = kLqL / 2;                      // step pairs per chunk
constexpr int kLqG = 4;                             // gates i, f, g, o
constexpr int kLqSteps = kLqW * kLqK * kLqL;        // 128 steps per item
constexpr int kLqChunks = kLqSteps / kLqL;          // 16
constexpr int kLqRowB = kLqH * kLqC * 8;            // one gate of a chunk: 256 bytes
constexpr int kLqS = kLqG * kLqRowB + 64;           // chunk slot: 1088 bytes
constexpr int kLqU = kLqChunks * kLqS;              // 17408: the item's fp32 arguments
constexpr int kLqBoxBytes = kLqSteps * kLqG * kLqC * 2;  // 8192: one box of 128 steps
constexpr int kLqStage = kLqU;                      // bf16 staging after the arguments
// the item's final (c, h), [128 steps][8 ch] each, for the bulk-tensor stores
constexpr int kLqStates = kLqStage + kLqBoxBytes;
constexpr int kLqSmem = kLqStates + 2 * kLqSteps * kLqC * 4;
constexpr int kLqMinB = 4;                          // CTAs per SM
static_assert(kLqS % 128 == 64, "a warp's four chunks in alternate 64-byte bank halves");
static_assert(kLqW % 4 == 0, "the item's residual maximum is read as float4s");
static_assert(kLqStage % 128 == 0, "TMA destination");
static_assert(2 * kLqThreads == kLqChunks * kLqH * kLqG, "the expansion: two gates per thread");

struct LqParams {
  const float* a;       // [4][D]
  const float* bias;    // [4][D] or null
  const float* c0;      // [B][D] or null
  const float* h0;      // [B][D] or null
  float* c;             // [B][T][D]
  float* h;             // [B][T][D]
  int B, T, D;
  int nDTc;             // 8-channel tiles per batch row
  int ntiles;           // B * nDTc
  int nitems;           // ntiles * segments (below 2^31)
  FastDiv dv_tiles, dv_ndtc;  // division by ntiles and by nDTc
  int max_iters;
  float tol;
  float apx_tau;        // inexact evaluations while the item's residual is above this (0: none)
  float spec_tau;       // a residual-only check follows an exact step from at most this
  float chk_tol;        // and certifies the iterate below this (tol / 2)
  uint64_t timeout_ns;
  unsigned* counter;    // item tickets (zero at launch)
  unsigned* seg_done;   // [ntiles] segments of each tile stored (zero at launch)
  int* chan_k;          // [B * D] or null
  pararnn_stats* stats;
  int withhold_item;    // testing: this item never publishes its segment (-1: none)
};

struct LqShared {
  // per (warp, channel): the warp's inclusive map (m00 m01 m10 m11 | d0 d1)
  // and its last state (c, h) before the update, by exchange parity
  float4 wagg[2][kLqW][kLqC][2];
  float wcm[2][kLqW][kLqC];              // per (warp, channel) max|r| (histogram)
  __align__(16) float wmax[2][kLqW];
  // a (4 rows), bias (4 rows), c0, h0 of an item's channels, by item parity
  float par[2][10][kLqC];
  uint64_t bar;                          // the staging area's mbarrier
  int nx[2];                             // the item after this one, by parity
};

__device__ __forceinline__ float2 qf2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 qfma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 qmul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 qadd(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 qtanh(float2 a) { return qf2(tanh_apx(a.x), tanh_apx(a.y)); }
__device__ __forceinline__ float2 qex2(float2 a) { return qf2(ex2(a.x), ex2(a.y)); }
__device__ __forceinline__ float2 qrcp(float2 a) { return qf2(rcp(a.x), rcp(a.y)); }

struct LqPar {
  float2 ai2, af2, ag2, ao2;  // h coefficients of the stored arguments
  float2 ai, af, ag, ao;      // the raw diagonal weights (Jacobian)
};

// One pass over a chunk (kMode 0: exact evaluation and local scan, 1: the
// same with the one-instruction tanh, 2: exact residual only).  (C[i], H[i])
// is the iterate at steps (i, i + 4), (cb, hb) the state before the chunk.
// Unless kMode is 2 the two half-chunks are scanned from a zero incoming
// delta: C, H become the local solution, P the running products, Mx / My
// the halves' maps.  Returns max over steps of max(|c_t - c'_t|, |h_t - h'_t|).
template <int kMode>
__device__ __forceinline__ float lq_pass(const unsigned char* __restrict__ base, int so0, int so1,
                                         float cb,
                                         float hb, float2 (&C)[kLqH], float2 (&H)[kLqH],
                                         float2 (&P00)[kLqH], float2 (&P01)[kLqH],
                                         float2 (&P10)[kLqH], float2 (&P11)[kLqH],
                                         const LqPar& k, Aff2& Mx, Aff2& My) {
  const float2 ONE = qf2(1.f, 1.f), M1 = qf2(-1.f, -1.f), M2 = qf2(-2.f, -2.f);
  const float2 F4 = qf2(4.f, 4.f), M4 = qf2(-4.f, -4.f), HALF = qf2(0.5f, 0.5f);
  const float2 TL = qf2(2.f * kLog2e, 2.f * kLog2e);
  const float2 KG = qf2(-0.5f / kLog2e, -0.5f / kLog2e), KC = qf2(0.5f / kLog2e, 0.5f / kLog2e);
  float m = 0.f;
  float2 dc = qf2(0.f, 0.f), dh = qf2(0.f, 0.f);
  float2 p00 = ONE, p01 = qf2(0.f, 0.f), p10 = qf2(0.f, 0.f), p11 = ONE;
  float2 CP = qf2(cb, C[kLqH - 1].x), HP = qf2(hb, H[kLqH - 1].x);  // before steps 0 and 4
#pragma unroll
  for (int i = 0; i < kLqH; ++i) {
    const unsigned char* bi = base + ((i >> 1) ? so1 : so0) + i * kLqC * 8;
    const float2 UI = *reinterpret_cast<const float2*>(bi);
    const float2 UF = *reinterpret_cast<const float2*>(bi + 1 * kLqRowB);
    const float2 UG = *reinterpret_cast<const float2*>(bi + 2 * kLqRowB);
    const float2 UO = *reinterpret_cast<const float2*>(bi + 3 * kLqRowB);
    const float2 CT = C[i], HT = H[i];
    float2 I, F, O, G, TC;  // gates, tanh(g argument), tanh(c')
    float2 DI, DF, DO, DG, DT;  // i(1-i), f(1-f), o(1-o), 1-g^2, 1-tanh^2(c')
    float2 CN;
    if constexpr (kMode == 1) {
      I = qfma(HALF, qtanh(qmul(qfma(k.ai2, HP, UI), KG)), HALF);
      F = qfma(HALF, qtanh(qmul(qfma(k.af2, HP, UF), KG)), HALF);
      O = qfma(HALF, qtanh(qmul(qfma(k.ao2, HP, UO), KG)), HALF);
      G = qtanh(qmul(qfma(k.ag2, HP, UG), KC));
      CN = qfma(F, CP, qmul(I, G));                          // c' = f c + i g
      TC = qtanh(CN);
      if constexpr (kMode != 2) {
        DG = qfma(qmul(G, M1), G, ONE);
        DT = qfma(qmul(TC, M1), TC, ONE);
      }
    } else {
      const float2 PI = qadd(ONE, qex2(qfma(k.ai2, HP, UI)));
      const float2 PF = qadd(ONE, qex2(qfma(k.af2, HP, UF)));
      const float2 PO = qadd(ONE, qex2(qfma(k.ao2, HP, UO)));
      const float2 PG = qadd(ONE, qex2(qfma(k.ag2, HP, UG)));
      I = qrcp(PI);
      F = qrcp(PF);
      O = qrcp(PO);
      const float2 TG = qrcp(PG);                           // 1/(1+e^{2y})
      G = qfma(M2, TG, ONE);                                // tanh(y_g)
      CN = qfma(F, CP, qmul(I, G));
      const float2 TC1 = qrcp(qadd(ONE, qex2(qmul(TL, CN))));
      TC = qfma(M2, TC1, ONE);                              // tanh(c')
      if constexpr (kMode != 2) {
        DG = qmul(TG, qfma(TG, M4, F4));                    // 1 - g^2 = 4t(1-t)
        DT = qmul(TC1, qfma(TC1, M4, F4));
      }
    }
    const float2 HN = qmul(O, TC);                          // h' = o tanh(c')
    const float2 RC = qfma(CN, M1, CT), RH = qfma(HN, M1, HT);
    m = fmax3_nan(fmax3_nan(m, fabsf(RC.x), fabsf(RC.y)), fabsf(RH.x), fabsf(RH.y));
    if constexpr (kMode != 2) {
      DI = qmul(I, qfma(I, M1, ONE));
      DF = qmul(F, qfma(F, M1, ONE));
      DO = qmul(O, qfma(O, M1, ONE));
      // dc'/dh through the arguments of i, f, g
      const float2 X = qfma(qmul(CP, DF), k.af, qfma(qmul(G, DI), k.ai, qmul(qmul(I, DG), k.ag)));
      const float2 KK = qmul(O, DT);                        // dh'/dc'
      const float2 A00 = F, A01 = X, A10 = qmul(KK, F);
      const float2 A11 = qfma(qmul(DO, TC), k.ao, qmul(KK, X));
      const float2 CNEW = qfma(A00, dc, qfma(A01, dh, CN));
      const float2 HNEW = qfma(A10, dc, qfma(A11, dh, HN));
      dc = qfma(CT, M1, CNEW);
      dh = qfma(HT, M1, HNEW);
      const float2 n00 = qfma(A00, p00, qmul(A01, p10)), n01 = qfma(A00, p01, qmul(A01, p11));
      const float2 n10 = qfma(A10, p00, qmul(A11, p10)), n11 = qfma(A10, p01, qmul(A11, p11));
      p00 = n00;
      p01 = n01;
      p10 = n10;
      p11 = n11;
      C[i] = CNEW;
      H[i] = HNEW;
      P00[i] = p00;
      P01[i] = p01;
      P10[i] = p10;
      P11[i] = p11;
    }
    CP = CT;
    HP = HT;
  }
  Mx = Aff2{p00.x, p01.x, p10.x, p11.x, dc.x, dh.x};
  My = Aff2{p00.y, p01.y, p10.y, p11.y, dc.y, dh.y};
  return m;
}

__device__ __forceinline__ Aff2 lq_shfl_up(const Aff2& a, int o) {
  return Aff2{__shfl_up_sync(kLqFull, a.m00, o), __shfl_up_sync(kLqFull, a.m01, o),
              __shfl_up_sync(kLqFull, a.m10, o), __shfl_up_sync(kLqFull, a.m11, o),
              __shfl_up_sync(kLqFull, a.d0, o),  __shfl_up_sync(kLqFull, a.d1, o)};
}

// Parameter j (0..79) of the item's tile at (b, d0): a[g][c] (j < 32),
// bias[g][c] (j < 64, 0 when absent), c0[c], h0[c] (0 when absent).
__device__ __forceinline__ float lq_param(const LqParams& p, int j, int b, int d0) {
  const int row = j / kLqC, c = j % kLqC;
  if (row < kLqG) return p.a[(size_t)row * p.D + d0 + c];
  if (row < 2 * kLqG) return p.bias ? p.bias[(size_t)(row - kLqG) * p.D + d0 + c] : 0.f;
  if (row == 8) return p.c0 ? p.c0[(size_t)b * p.D + d0 + c] : 0.f;
  return p.h0 ? p.h0[(size_t)b * p.D + d0 + c] : 0.f;
}
// An item's segment, tile, batch row and first channel (item = segment *
// ntiles + tile, tile = row * nDTc + channel block), by multiply-high division
__device__ __forceinline__ int lq_seg(const LqParams& p, int item) {
  return fast_quot(item, p.dv_tiles);
}
__device__ __forceinline__ int lq_tile(const LqParams& p, int item) {
  return item - lq_seg(p, item) * p.ntiles;
}
__device__ __forceinline__ int lq_row(const LqParams& p, int tile) {
  return fast_quot(tile, p.dv_ndtc);
}
__device__ __forceinline__ int lq_d0(const LqParams& p, int tile) {
  return (tile - lq_row(p, tile) * p.nDTc) * kLqC;
}
__device__ __forceinline__ void lq_issue(unsigned char* smem, uint64_t* bar, const CUtensorMap* map,
                                         int b, int d0, int t0) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(bar, (unsigned)kLqBoxBytes);
  tma_load_4d(smem + kLqStage, map, bar, d0, 0, t0, b);
}
__device__ __forceinline__ int lq_draw(unsigned* counter) {
  return (int)min(atomicAdd(counter, 1u), 0x7fffffffu);
}

__global__ void __launch_bounds__(kLqThreads, kLqMinB)
    lstm_newton_queue(const __grid_constant__ CUtensorMap map,
                      const __grid_constant__ CUtensorMap cmap,
                      const __grid_constant__ CUtensorMap hmap, const LqParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ LqShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane % kLqC, kk = lane / kLqC;
  const int q = warp * kLqK + kk;  // chunk index within the item
  const unsigned char* base = smem + q * kLqS;
  // this thread's channel slot in its chunk for pairs 0, 1 and for pairs 2, 3
  const int so0 = (c ^ (q & 7)) * 8, so1 = (c ^ ((q + 2) & 7)) * 8;

  if (tid == 0) {
    mbar_init(&sh.bar, 1);
    sh.nx[0] = lq_draw(p.counter);
  }
  __syncthreads();
  int item = sh.nx[0];
  if (item < p.nitems) {
    const int tile = lq_tile(p, item), b = lq_row(p, tile), d0 = lq_d0(p, tile);
    if (tid < 10 * kLqC) (&sh.par[0][0][0])[tid] = lq_param(p, tid, b, d0);
    if (tid == 0) lq_issue(smem, &sh.bar, &map, b, d0, lq_seg(p, item) * kLqSteps);
  }
  int status = 0;
  unsigned phase = 0;  // exchange phases so far, over all items
  int prev_item = -1;
  // CTA-uniform: 0 while the staged boxes arrive, else 1 + the phase parity of
  // the wait that ran out (no box is issued after that)
  int dead = 0;
  for (int n = 0; item < p.nitems; ++n) {
    __syncthreads();
    // publish the previous item: its states' bulk stores (issued by thread
    // 32) complete, then the proxy fence, the fence and the release order
    // them before the count.  Warp 0 draws the next ticket meanwhile: both
    // wait on memory.  The completed stores have also read the states buffer,
    // which this item fills again at its end.
    if (tid == 32 && prev_item >= 0) {
      bulk_wait_all();
      if (prev_item != p.withhold_item) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        st_release(&p.seg_done[lq_tile(p, prev_item)], (unsigned)lq_seg(p, prev_item) + 1u);
      }
    }
    // the item after this one: drawn now, stored before the item's first
    // barrier (the atomic's latency overlaps the wait for the boxes)
    int ticket = 0;
    if (tid == 0) ticket = lq_draw(p.counter);
    const int pb = n & 1;
    const int tile = lq_tile(p, item), seg = lq_seg(p, item);
    const int b = lq_row(p, tile), d0 = lq_d0(p, tile);
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int t_base = seg * kLqSteps;
    const int t_len = min(kLqSteps, p.T - t_base);
    const bool first = (q == 0);  // the chunk holding the segment's first step
    // the segment's initial state: (c0, h0), or the last states of the
    // previous segment once that segment's CTA has published them (waited
    // for and loaded here, so that the loads overlap the wait for the box)
    float pc0 = 0.f, ph0 = 0.f;
    if (first && seg > 0) {
      const unsigned* f = &p.seg_done[tile];
      if (ld_acquire(f) < (unsigned)seg) {
        const uint64_t w0 = globaltimer_ns();
        while (ld_acquire(f) < (unsigned)seg) {
          if (globaltimer_ns() - w0 > p.timeout_ns) {
            status = PARARNN_STATUS_TIMEOUT;
            break;
          }
        }
      }
      const size_t ip = ((size_t)b * p.T + t_base - 1) * p.D + d;
      pc0 = dval ? __ldcg(p.c + ip) : 0.f;
      ph0 = dval ? __ldcg(p.h + ip) : 0.f;
    }
    bool got = true;
    if (!dead) {
      got = mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns);
      if (!got) status = PARARNN_STATUS_TIMEOUT;
    }
    // ---- expand the staged bf16 rows [t][gate][8 ch] into fp32 arguments:
    // thread (unit, half) takes steps i and i + 4 of chunk qq, gates 2 half
    // and 2 half + 1
    {
      const int unit = tid % (kLqChunks * kLqH), half = tid / (kLqChunks * kLqH);
      const int qq = unit / kLqH, i = unit % kLqH;
      const int sw = (qq + 2 * (i >> 1)) & 7;
      const int ta = qq * kLqL + i, tb = ta + kLqH;  // steps within the item
      const bool pa = ta >= t_len, pbd = tb >= t_len;
      unsigned char* dst = smem + qq * kLqS + i * kLqC * 8;
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = 2 * half + gg;
        const uint4 va =
            *reinterpret_cast<const uint4*>(smem + kLqStage + (ta * kLqG + g) * 16);
        const uint4 vb =
            *reinterpret_cast<const uint4*>(smem + kLqStage + (tb * kLqG + g) * 16);
        const float sc = (g == 2) ? 2.f * kLog2e : -kLog2e;
        // steps past T: i, o shut, f open, g 0
        const float padv = (g == 1) ? -3e30f : ((g == 2) ? 0.f : 3e30f);
        const unsigned wa[4] = {va.x, va.y, va.z, va.w};
        const unsigned wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int cc = 0; cc < kLqC; ++cc) {
          const int s16 = (cc & 1) ? 0 : 16;
          const unsigned mk = (cc & 1) ? 0xffff0000u : 0xffffffffu;
          const float xa = __uint_as_float((wa[cc >> 1] << s16) & mk);
          const float xb = __uint_as_float((wb[cc >> 1] << s16) & mk);
          const float bs = sc * sh.par[pb][kLqG + g][cc];
          float2 o = qfma(qf2(sc, sc), qf2(xa, xb), qf2(bs, bs));
          if (pa) o.x = padv;
          if (pbd) o.y = padv;
          *reinterpret_cast<float2*>(dst + g * kLqRowB + (cc ^ sw) * 8) = o;
        }
      }
    }
    LqPar k;
    {
      const float ai = sh.par[pb][0][c], af = sh.par[pb][1][c], ag = sh.par[pb][2][c],
                  ao = sh.par[pb][3][c];
      k.ai = qf2(ai, ai);
      k.af = qf2(af, af);
      k.ag = qf2(ag, ag);
      k.ao = qf2(ao, ao);
      const float ai2 = -kLog2e * ai, af2 = -kLog2e * af, ag2 = 2.f * kLog2e * ag,
                  ao2 = -kLog2e * ao;
      k.ai2 = qf2(ai2, ai2);
      k.af2 = qf2(af2, af2);
      k.ag2 = qf2(ag2, ag2);
      k.ao2 = qf2(ao2, ao2);
    }
    float c0v = sh.par[pb][8][c], h0v = sh.par[pb][9][c];
    if (tid == 0) sh.nx[(n + 1) & 1] = ticket;  // read after the barrier below
    // a phase that did not complete is never re-armed: no more boxes then
    if (dead) {
      __syncthreads();
    } else if (!__syncthreads_and(got)) {
      dead = 1 + (n & 1);
    }
    // the staging area is free: the next item's box; its parameters now
    const int next = sh.nx[(n + 1) & 1];
    const int pj = tid - 32;
    float pnext = 0.f;
    if (next < p.nitems) {
      const int ntile = lq_tile(p, next), nb = lq_row(p, ntile), nd0 = lq_d0(p, ntile);
      if (tid == 0 && !dead) lq_issue(smem, &sh.bar, &map, nb, nd0, lq_seg(p, next) * kLqSteps);
      if (pj >= 0 && pj < 10 * kLqC) pnext = lq_param(p, pj, nb, nd0);
    }
    if (first && seg > 0) {
      c0v = pc0;
      h0v = ph0;
    }

    float2 C[kLqH], H[kLqH], P00[kLqH], P01[kLqH], P10[kLqH], P11[kLqH];
#pragma unroll
    for (int i = 0; i < kLqH; ++i) {
      C[i] = qf2(0.f, 0.f);
      H[i] = qf2(0.f, 0.f);
      P00[i] = P01[i] = P10[i] = P11[i] = qf2(0.f, 0.f);
    }
    float cb = first ? c0v : 0.f, hb = first ? h0v : 0.f;  // state before this chunk
    // last_bad: updates applied before the last evaluation that left the
    // channel at or above tol (histogram); nupd: updates applied so far
    int last_bad = -1, updates = 0, kit = 0, nupd = 0;
    float final_m = 0.f;
    bool apx = p.apx_tau > 0.f;  // CTA-uniform: set from the item's residual maximum
    // one Newton iteration of the item (kMode as in lq_pass; 2 at the cap or
    // as a check that certifies the iterate); true when the item is done
    auto iterate = [&](auto mode) -> bool {
      constexpr int kMode = decltype(mode)::value;
      constexpr bool resid_only = kMode == 2, apx_eval = kMode == 1;
      const int par = phase & 1;
      ++phase;
      const float lastc = C[kLqH - 1].y, lasth = H[kLqH - 1].y;
      Aff2 Mx, My;
      float m = lq_pass<kMode>(base, so0, so1, cb, hb, C, H, P00, P01, P10, P11, k, Mx, My);
      if (!dval) m = 0.f;
      // the chunk's map: second half after the first
      Aff2 inc = My.after(Mx), xm = Aff2::id();
      if constexpr (!resid_only) {
        // inclusive scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
        for (int o = kLqC; o < 32; o <<= 1) {
          const Aff2 prev = lq_shfl_up(inc, o);
          if (lane >= o) inc = inc.after(prev);
        }
        // exclusive: the delta entering the warp -> the delta entering this chunk
        xm = lq_shfl_up(inc, kLqC);
        if (kk == 0) xm = Aff2::id();
      }
      const unsigned wm = __reduce_max_sync(kLqFull, __float_as_uint(m));
      unsigned cmu = __float_as_uint(m);
      cmu = max(cmu, __shfl_xor_sync(kLqFull, cmu, 8));
      cmu = max(cmu, __shfl_xor_sync(kLqFull, cmu, 16));
      if (!resid_only && kk == kLqK - 1) {
        sh.wagg[par][warp][c][0] = make_float4(inc.m00, inc.m01, inc.m10, inc.m11);
        sh.wagg[par][warp][c][1] = make_float4(inc.d0, inc.d1, lastc, lasth);
      }
      if (kk == 0) sh.wcm[par][warp][c] = __uint_as_float(cmu);
      if (lane == 0) sh.wmax[par][warp] = __uint_as_float(wm);
      __syncthreads();
      if (q == 0) {  // the channel's own maximum over the item (histogram)
        float chm = 0.f;
#pragma unroll
        for (int w = 0; w < kLqW; ++w) chm = fmax_nan(chm, sh.wcm[par][w][c]);
        if (apx_eval || !(chm < p.tol)) last_bad = nupd;
      }
      // the delta entering this warp: the maps of the warps before it applied
      // to the zero delta entering the item; and the item's residual maximum
      float2 cin = qf2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kLqW - 1; ++w) {
        if (!resid_only && w < warp) {
          const float4 m0 = sh.wagg[par][w][c][0], m1 = sh.wagg[par][w][c][1];
          cin = qf2(fmaf(m0.x, cin.x, fmaf(m0.y, cin.y, m1.x)),
                    fmaf(m0.z, cin.x, fmaf(m0.w, cin.y, m1.y)));
        }
      }
      float tmax = 0.f;
#pragma unroll
      for (int w4 = 0; w4 < kLqW; w4 += 4) {
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
        const bool cap = kit >= p.max_iters;
        if (cap && !own_ok && status == 0) status = PARARNN_STATUS_NOT_CONVERGED;
        // a check certifies below tol / 2: the margin covers the fp32
        // rounding of the states and of this evaluation, so that the exact
        // residual of the returned states stays below tol
        return cap || tmax < p.chk_tol;
      }
      const float2 din = first ? qf2(0.f, 0.f) : xm.apply(cin);  // delta entering this chunk
      float2 prev_last = qf2(__shfl_up_sync(kLqFull, lastc, kLqC),
                             __shfl_up_sync(kLqFull, lasth, kLqC));
      if (kk == 0) {
        if (warp == 0) {
          prev_last = qf2(c0v, h0v);
        } else {
          const float4 l1 = sh.wagg[par][warp - 1][c][1];
          prev_last = qf2(l1.z, l1.w);
        }
      }
      cb = first ? c0v : prev_last.x + din.x;
      hb = first ? h0v : prev_last.y + din.y;
      // deltas entering the two halves of the chunk
      const float2 dy = Mx.apply(din);
      const float2 DINC = qf2(din.x, dy.x), DINH = qf2(din.y, dy.y);
#pragma unroll
      for (int i = 0; i < kLqH; ++i) {
        C[i] = qfma(P00[i], DINC, qfma(P01[i], DINH, C[i]));
        H[i] = qfma(P10[i], DINC, qfma(P11[i], DINH, H[i]));
      }
      updates = ++nupd;
      return own_ok;
    };
    // inexact iterations while the residual is large, then exact ones to
    // convergence or the cap (kit: the evaluation's index).  An exact step
    // from a residual at most spec_tau (sqrt(tol / 2)) lands below tol / 2
    // with quadratic convergence, so the evaluation after it is a
    // residual-only check: if it certifies, the item ends on that iterate
    // without forming the step; if not, the next evaluation forms the step at
    // the same iterate.
    for (; apx && kit < p.max_iters; ++kit) iterate(std::integral_constant<int, 1>{});
    bool spec = false;
    for (;; ++kit) {
      if (kit >= p.max_iters) {
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
    if (pj >= 0 && pj < 10 * kLqC) (&sh.par[pb ^ 1][0][0])[pj] = pnext;

    // ---- states: from registers into the states buffer ([step][8 ch] for c
    // and for h), then one bulk-tensor store each (steps past T are not
    // written)
    bool bad = false;
    {
      float* cs = reinterpret_cast<float*>(smem + kLqStates);
      float* hs = cs + kLqSteps * kLqC;
      const int tq = q * kLqL;
#pragma unroll
      for (int i = 0; i < kLqH; ++i) {
        cs[(tq + i) * kLqC + c] = C[i].x;
        hs[(tq + i) * kLqC + c] = H[i].x;
        cs[(tq + kLqH + i) * kLqC + c] = C[i].y;
        hs[(tq + kLqH + i) * kLqC + c] = H[i].y;
        if (dval) {
          bad |= tq + i < t_len && (!isfinite(C[i].x) || !isfinite(H[i].x));
          bad |= tq + kLqH + i < t_len && (!isfinite(C[i].y) || !isfinite(H[i].y));
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (tid == 32) {
        tma_store_3d(&cmap, cs, d0, t_base, b);
        tma_store_3d(&hmap, hs, d0, t_base, b);
        bulk_commit();
      }
    }
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    if (p.chan_k != nullptr && q == 0 && dval)
      atomicMax(&p.chan_k[(size_t)b * p.D + d], last_bad + 1);
    if (tid == 0) {
      atomicMax(&p.stats->iters, updates);
      atomicMax(&p.stats->evals, kit + 1);
      atomicMax(reinterpret_cast<int*>(&p.stats->max_residual), __float_as_int(final_m));
    }
    prev_item = item;
    item = next;
  }
  __syncthreads();
  if (tid == 32 && prev_item >= 0) {
    bulk_wait_all();
    if (prev_item != p.withhold_item) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __threadfence();
      st_release(&p.seg_done[lq_tile(p, prev_item)], (unsigned)lq_seg(p, prev_item) + 1u);
    }
  }
  // a box still in flight into the staging area: wait for it (bounded)
  if (dead && tid == 0) mbar_wait_bounded(&sh.bar, (unsigned)(dead - 1), p.timeout_ns);
  const int st = __reduce_max_sync(kLqFull, status);
  if (lane == 0 && st) atomicMax(&p.stats->status, st);
}

int lq_per_sm() {
  int per_sm = 0;
  if (cudaFuncSetAttribute(lstm_newton_queue, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kLqSmem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lstm_newton_queue, kLqThreads,
                                                    kLqSmem) != cudaSuccess)
    per_sm = 0;
  cudaGetLastError();
  return per_sm;
}

}  // namespace

int lstm_queue_steps() { return kLqSteps; }
int lstm_queue_box_steps() { return kLqSteps; }

// Resident CTAs of the segment-queue solve on the current device (0 if it
// cannot run).
int lstm_queue_resident() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * lq_per_sm();
}

// One launch solves every 128-step segment of every tile; u is bf16 through
// `map` (boxes of 8 channels x 4 gates x 128 steps).  counter and seg_done
// (ntiles entries) must be zero at launch.
// cmap, hmap: the states c, h [B][T][D], box 8 channels x 128 steps
int launch_lstm_queue(const CUtensorMap& map, const CUtensorMap& cmap, const CUtensorMap& hmap,
                      const FwdParams& f, unsigned* counter,
                      unsigned* seg_done, cudaStream_t stream) {
  LqParams p;
  p.a = f.a;
  p.bias = f.bias;
  p.c0 = f.c0;
  p.h0 = f.h0;
  p.c = f.c;
  p.h = f.h;
  p.B = f.B;
  p.T = f.T;
  p.D = f.D;
  p.nDTc = (f.D + kLqC - 1) / kLqC;
  p.ntiles = f.B * p.nDTc;
  p.dv_tiles = fast_div((unsigned)p.ntiles);
  p.dv_ndtc = fast_div((unsigned)p.nDTc);
  const long long nitems = (long long)p.ntiles * ((f.T + kLqSteps - 1) / kLqSteps);
  if (nitems >= (1LL << 31)) return 1;
  p.nitems = (int)nitems;
  p.max_iters = f.max_iters;
  p.tol = f.tol;
  p.apx_tau = (f.flags & PARARNN_FLAG_EXACT_STEPS) ? 0.f : kApxTau;
  p.chk_tol = 0.5f * f.tol;
  p.spec_tau = f.tol > 0.f ? std::sqrt(p.chk_tol) : -1.f;
  p.timeout_ns = f.timeout_ns;
  p.counter = counter;
  p.seg_done = seg_done;
  p.chan_k = f.chan_k;
  p.stats = f.stats;
  p.withhold_item = (f.flags & PARARNN_FLAG_INJECT_WITHHOLD) ? f.inject_chunk : -1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_sm = std::max(1, lq_per_sm());
  // persistent: every CTA resident at once (the queue's progress argument)
  const long long grid = std::min<long long>((long long)sms * per_sm, p.nitems);
  lstm_newton_queue<<<(unsigned)std::max<long long>(grid, 1), kLqThreads, kLqSmem, stream>>>(
      map, cmap, hmap, p);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
