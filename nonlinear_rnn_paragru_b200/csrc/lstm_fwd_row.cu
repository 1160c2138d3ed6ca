// lstm_fwd_row.cu -- fused Newton-scan ParaLSTM solve for sequences (or
// segments of sequences) of up to 4096 steps with bf16 input projections: 8
// channels per CTA, a cluster of CLS = ceil(T / 512) CTAs per tile, the cell
// evaluated on packed fp32 pairs.
//
// A tile is 8 consecutive channels of one batch row over the steps this launch
// solves: the whole sequence, or one segment of it that starts from the (c, h)
// the segment before ended with (the host launches the segments in order).  CTA
// rank r of the cluster owns steps [512 r, 512 (r+1)) of them: 8 warps x 32
// lanes, lane = (k, c) with the channel c = lane % 8 fastest and k = lane / 8
// one of four 16-step chunks; warp w covers steps [64 w, 64 w + 64) of the
// CTA's range.  A thread keeps its chunk's iterate (c, h) and the running
// product P of the 2x2 Jacobians in registers (96 of them), one CTA per SM.
//
// Per iteration ("Параллельность RNN?", §1.2-§1.3): each thread evaluates the
// cell, the residual over c and h and the 2x2 Jacobian on its 16 steps and
// scans them serially (s'_t = f_t + A_t ds_{t-1}, running product P_t).  The
// 16 steps are taken as 8 pairs (i, i + 8): both halves of the chunk are
// scanned side by side from a zero incoming delta, so every add, multiply and
// fma is one packed fp32x2 instruction (each lane rounded as its scalar
// form); the second half is composed after the first when the chunk's map is
// formed and in the fix-up.  One reciprocal serves the six sigmoids i, f, o
// of a pair, one the pair's two tanh(g) and one its two tanh(c'); every
// exponent argument is clamped at 21, so a product of six (1 + 2^x) stays
// below 2^127 (the clamp moves a gate by under 5e-7).
// The chunk maps (2x2 matrix, 2-vector) are scanned: over the four chunks of
// a warp by shuffles; over the 8 warps after one CTA barrier, each thread
// composing the maps of the warps before its own from shared memory; over
// the CTAs of the cluster by remote asynchronous stores into the peers'
// mailboxes (the CTA's map and last state to the CTAs after it, its residual
// maximum to all), each completing on the receiver's mbarrier.  The fix-up
// adds P_t ds_in.  Mailboxes and per-warp data are double-buffered by the
// parity of a phase counter that runs on across tiles.  The cluster stops at
// the first exact evaluation whose residual over the tile is below tol: after
// its update when the evaluation formed the step, or on the iterate itself
// when it was a residual-only check below tol / 2 (the evaluation after a
// step from a residual at most sqrt(tol / 2)); at the cap it ends with a
// residual-only evaluation.  The state before each chunk is re-anchored
// every iteration to its predecessor's pre-update last state plus the
// incoming delta.
//
// Data: the tile's u arrives bf16 by two TMA boxes of 256 steps into a
// staging area (a, bias, c0 and h0 of the next tile's channels are read with
// plain loads a tile ahead into a double-buffered block) and is expanded,
// once per tile, into the fp32
// arguments -log2e u + b' (i, f, o) and 2 log2e u + b' (g), stored per chunk
// as [gate][pair i][channel] {step i, step i + 8}, channel c at slot
// c ^ (i >> 1): one 8-byte load per gate and pair.  The next tile's boxes are
// issued as soon as the expansion is done.  Steps past T get i and o shut and
// f open.  States are stored straight from registers.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cgl = cooperative_groups;

constexpr int kLrThreads = 256;
constexpr int kLrWarps = 8;
constexpr int kLrC = 8;                      // channels per tile
constexpr int kLrK = 32 / kLrC;              // chunks per warp
constexpr int kLrL = 16;                     // steps per chunk (per thread)
constexpr int kLrH = kLrL / 2;               // step pairs per chunk
constexpr int kLrG = 4;                      // gates i, f, g, o
constexpr int kLrSteps = kLrWarps * kLrK * kLrL;  // 512 steps per CTA
constexpr int kLrChunks = kLrSteps / kLrL;        // 32 chunks per CTA
constexpr int kLrRowB = kLrH * kLrC * 8;          // one gate of a chunk: 512 bytes
constexpr int kLrS = kLrG * kLrRowB + 64;         // chunk slot: 2048 + 64 bytes
constexpr int kLrU = kLrChunks * kLrS;            // 67584: the tile's fp32 arguments
constexpr int kLrBox = 256;                       // steps per TMA box
constexpr int kLrBoxBytes = kLrBox * kLrG * kLrC * 2;  // 16384
constexpr int kLrNBox = kLrSteps / kLrBox;        // 2
constexpr int kLrStage = kLrU;                    // bf16 staging after the arguments
constexpr int kLrSmem = kLrStage + kLrNBox * kLrBoxBytes;
constexpr int kLrMaxCluster = 8;
constexpr int kLrTmax = kLrSteps * kLrMaxCluster;  // 4096
static_assert(kLrStage % 128 == 0 && kLrBoxBytes % 128 == 0, "TMA destinations");
static_assert(kLrThreads == kLrChunks * kLrH, "the expansion: one (chunk, pair) per thread");
static_assert(kLrWarps == kLrC, "one row of warp maps per channel");

struct LrMailbox {  // written by the cluster peers with remote async stores
  // by rank and channel: (m00, m01, m10, m11), (d_c, d_h, last c, last h)
  float4 map[kLrMaxCluster][kLrC][2];
  float cmax[kLrMaxCluster];
};

struct LrShared {
  // per (warp, channel): the warp's inclusive map and its last state before
  // the update, laid out like a mailbox entry
  float4 wagg[2][kLrWarps][kLrC][2];
  float wmax[2][kLrWarps];
  float wcm[2][kLrWarps][kLrC];       // per (warp, channel) max|r| (histogram)
  __align__(16) LrMailbox mbox[2];
  // a (4 rows), bias (4 rows), c0, h0 of a tile's channels, by tile parity
  __align__(16) float par[2][10][kLrC];
  uint64_t bar;                       // the staging area's mbarrier
  uint64_t mbar[2];                   // mailbox mbarriers, by parity
};

__device__ __forceinline__ float2 lf2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 lfma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 lmul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 ladd(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 lclamp(float2 a, float hi) {
  return lf2(fmin_nan(a.x, hi), fmin_nan(a.y, hi));
}
__device__ __forceinline__ float2 lex2(float2 a) { return lf2(ex2(a.x), ex2(a.y)); }
__device__ __forceinline__ int lr_swizzle(int i) { return i >> 1; }

__device__ __forceinline__ uint32_t lr_mapa(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void lr_st_async_v4(uint32_t raddr, float4 v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(raddr), "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)),
      "r"(__float_as_uint(v.z)), "r"(__float_as_uint(v.w)), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void lr_st_async_b32(uint32_t raddr, unsigned v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
               ::"r"(raddr), "r"(v), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void lr_bulk_load(void* dst, const void* src, unsigned bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// an Aff2 map <-> two float4 (matrix; vector and two spare lanes)
__device__ __forceinline__ Aff2 lr_map(const float4& m, const float4& v) {
  return Aff2{m.x, m.y, m.z, m.w, v.x, v.y};
}
__device__ __forceinline__ Aff2 lr_shfl_up(const Aff2& a, int o) {
  return Aff2{__shfl_up_sync(kFull, a.m00, o), __shfl_up_sync(kFull, a.m01, o),
              __shfl_up_sync(kFull, a.m10, o), __shfl_up_sync(kFull, a.m11, o),
              __shfl_up_sync(kFull, a.d0, o),  __shfl_up_sync(kFull, a.d1, o)};
}

struct LrPar {
  float2 ai2, af2, ag2, ao2;  // h coefficients of the arguments (-log2e a; 2 log2e a for g)
  float2 ai, af, ag, ao;      // the raw diagonal weights (Jacobian)
};

// One pass over a chunk: (C[i], H[i]) = the iterate at steps (i, i + 8),
// (cb, hb) the state before the chunk.  With kFull the two half-chunks are
// scanned from a zero incoming delta: C, H become the local solution, P the
// running products, and DC, DH / Q* the halves' delta out and product.
// Returns max over steps of max(|c_t - c'_t|, |h_t - h'_t|).
template <bool kFull>
__device__ __forceinline__ float lr_pass(const unsigned char* __restrict__ base, int c8, float cb,
                                         float hb, float2 (&C)[kLrH], float2 (&H)[kLrH],
                                         float2 (&P00)[kLrH], float2 (&P01)[kLrH],
                                         float2 (&P10)[kLrH], float2 (&P11)[kLrH],
                                         const LrPar& k, float2& DCo, float2& DHo, Aff2& Mx,
                                         Aff2& My) {
  const float2 ONE = lf2(1.f, 1.f), M1 = lf2(-1.f, -1.f), M2 = lf2(-2.f, -2.f);
  const float2 F4 = lf2(4.f, 4.f), M4 = lf2(-4.f, -4.f);
  const float2 TL = lf2(2.f * kLog2e, 2.f * kLog2e);
  float m = 0.f;
  float2 dc = lf2(0.f, 0.f), dh = lf2(0.f, 0.f);
  float2 p00 = ONE, p01 = lf2(0.f, 0.f), p10 = lf2(0.f, 0.f), p11 = ONE;
  float2 CP = lf2(cb, C[kLrH - 1].x), HP = lf2(hb, H[kLrH - 1].x);  // before steps 0 and 8
#pragma unroll
  for (int i = 0; i < kLrH; ++i) {
    const unsigned char* bi = base + ((c8 ^ (lr_swizzle(i) * 8)) + i * kLrC * 8);
    const float2 UI = *reinterpret_cast<const float2*>(bi);
    const float2 UF = *reinterpret_cast<const float2*>(bi + 1 * kLrRowB);
    const float2 UG = *reinterpret_cast<const float2*>(bi + 2 * kLrRowB);
    const float2 UO = *reinterpret_cast<const float2*>(bi + 3 * kLrRowB);
    const float2 CT = C[i], HT = H[i];
    const float2 EI = lex2(lclamp(lfma(k.ai2, HP, UI), 21.f));
    const float2 EF = lex2(lclamp(lfma(k.af2, HP, UF), 21.f));
    const float2 EO = lex2(lclamp(lfma(k.ao2, HP, UO), 21.f));
    const float2 EG = lex2(lclamp(lfma(k.ag2, HP, UG), 21.f));
    const float2 PI = ladd(ONE, EI), PF = ladd(ONE, EF), PO = ladd(ONE, EO);
    const float2 PFO = lmul(PF, PO), PIO = lmul(PI, PO), PIF = lmul(PI, PF);
    const float2 Q = lmul(PI, PFO);
    const float iq = rcp(Q.x * Q.y);
    const float2 IQ = lf2(Q.y * iq, Q.x * iq);            // 1/(pi pf po) per step
    const float2 I = lmul(PFO, IQ), F = lmul(PIO, IQ), O = lmul(PIF, IQ);
    const float2 PG = ladd(ONE, EG);
    const float ig = rcp(PG.x * PG.y);
    const float2 TG = lf2(PG.y * ig, PG.x * ig);          // 1/(1+e^{2y})
    const float2 G = lfma(M2, TG, ONE);                   // tanh(y_g)
    const float2 CN = lfma(F, CP, lmul(I, G));            // c' = f c + i g
    const float2 EC = lex2(lclamp(lmul(TL, CN), 21.f));
    const float2 PC = ladd(ONE, EC);
    const float icn = rcp(PC.x * PC.y);
    const float2 TC1 = lf2(PC.y * icn, PC.x * icn);
    const float2 TC = lfma(M2, TC1, ONE);                 // tanh(c')
    const float2 HN = lmul(O, TC);                        // h' = o tanh(c')
    const float2 RC = lfma(CN, M1, CT), RH = lfma(HN, M1, HT);
    m = fmax3_nan(fmax3_nan(m, fabsf(RC.x), fabsf(RC.y)), fabsf(RH.x), fabsf(RH.y));
    if (kFull) {
      const float2 DI = lmul(I, lfma(I, M1, ONE));        // i(1-i)
      const float2 DF = lmul(F, lfma(F, M1, ONE));
      const float2 DO = lmul(O, lfma(O, M1, ONE));
      const float2 DG = lmul(TG, lfma(TG, M4, F4));       // 1 - g^2 = 4t(1-t)
      const float2 DT = lmul(TC1, lfma(TC1, M4, F4));     // 1 - tanh^2(c')
      // dc'/dh through the pre-activations of i, f, g
      const float2 X = lfma(lmul(CP, DF), k.af, lfma(lmul(G, DI), k.ai, lmul(lmul(I, DG), k.ag)));
      const float2 KK = lmul(O, DT);                      // dh'/dc'
      const float2 A00 = F, A01 = X, A10 = lmul(KK, F);
      const float2 A11 = lfma(lmul(DO, TC), k.ao, lmul(KK, X));
      const float2 CNEW = lfma(A00, dc, lfma(A01, dh, CN));
      const float2 HNEW = lfma(A10, dc, lfma(A11, dh, HN));
      dc = lfma(CT, M1, CNEW);
      dh = lfma(HT, M1, HNEW);
      const float2 n00 = lfma(A00, p00, lmul(A01, p10)), n01 = lfma(A00, p01, lmul(A01, p11));
      const float2 n10 = lfma(A10, p00, lmul(A11, p10)), n11 = lfma(A10, p01, lmul(A11, p11));
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
  DCo = dc;
  DHo = dh;
  Mx = Aff2{p00.x, p01.x, p10.x, p11.x, dc.x, dh.x};
  My = Aff2{p00.y, p01.y, p10.y, p11.y, dc.y, dh.y};
  return m;
}

// Thread 0: the tile's two 256-step boxes, on `bar`.
__device__ __forceinline__ void lr_issue(unsigned char* smem, LrShared& sh, const CUtensorMap* map,
                                         int b, int d0, int t0) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(&sh.bar, (unsigned)(kLrNBox * kLrBoxBytes));
  for (int j = 0; j < kLrNBox; ++j)
    tma_load_4d(smem + kLrStage + j * kLrBoxBytes, map, &sh.bar, d0, 0, t0 + j * kLrBox, b);
}
// Parameter j (0..79) of the tile at (b, d0): a[g][c] (j < 32), bias[g][c]
// (j < 64, 0 when absent), c0[c], h0[c] (0 when absent).
__device__ __forceinline__ float lr_param(const FwdParams& p, int j, int b, int d0) {
  const int row = j / kLrC, c = j % kLrC;
  if (row < kLrG) return p.a[(size_t)row * p.D + d0 + c];
  if (row < 2 * kLrG) return p.bias ? p.bias[(size_t)(row - kLrG) * p.D + d0 + c] : 0.f;
  if (row == 8) return p.c0 ? p.c0[(size_t)b * p.ld_h0 + d0 + c] : 0.f;
  return p.h0 ? p.h0[(size_t)b * p.ld_h0 + d0 + c] : 0.f;
}

// Bytes a CTA of rank `rank` receives per exchange phase.
__host__ __device__ constexpr unsigned lr_rx_bytes(int rank, int cls) {
  return (unsigned)(rank * kLrC * 32 + (cls - 1) * 4);
}

template <int CLS>
__global__ void __launch_bounds__(kLrThreads, 1)
    lstm_newton_row(const __grid_constant__ CUtensorMap map, const FwdParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ LrShared sh;
  cgl::cluster_group cluster = cgl::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (CLS > 1) ? (int)cluster.block_rank() : 0;
  const int c = lane % kLrC, kk = lane / kLrC;
  const int q = warp * kLrK + kk;            // chunk index within the CTA
  const int nDTc = (p.D + kLrC - 1) / kLrC;
  const int ntiles = p.B * nDTc;
  const int nclus = gridDim.x / CLS, clus = blockIdx.x / CLS;
  const int t0 = rank * kLrSteps;            // first step of this CTA
  const unsigned rx = lr_rx_bytes(rank, CLS);

  int cur = clus;  // the current tile
  // the first tile's parameters; later tiles' are loaded a tile ahead
  if (tid < 10 * kLrC && cur < ntiles) {
    const int b = cur / nDTc;
    (&sh.par[0][0][0])[tid] = lr_param(p, tid, b, (cur - b * nDTc) * kLrC);
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
  if (CLS > 1) cluster.sync();  // the peers' mailbox barriers are armed before anyone sends
  if (tid == 0 && cur < ntiles) {
    const int b = cur / nDTc;
    lr_issue(smem, sh, &map, b, (cur - b * nDTc) * kLrC, p.t_base + t0);
  }
  const unsigned char* base = smem + q * kLrS;
  int status = 0;
  int n = 0;
  unsigned phase = 0;  // exchange phases so far, over all tiles
  for (; cur < ntiles; ++n) {
    const int tile = cur;
    const int t_base = p.t_base;   // the launch's first step
    const int t_len = p.t_len;
    const int b = tile / nDTc, d0 = (tile - b * nDTc) * kLrC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int next = tile + nclus;
    // the next tile's parameters: loaded now, stored at the end of this tile
    const int pj = tid - 32;
    float pnext = 0.f;
    if (pj >= 0 && pj < 10 * kLrC && next < ntiles) {
      const int b2 = next / nDTc;
      pnext = lr_param(p, pj, b2, (next - b2 * nDTc) * kLrC);
    }
    const int pb = n & 1;
    if (!mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;
    // ---- expand the staged bf16 rows [t][gate][8 ch] into the fp32
    // arguments.  Thread (qq, i) takes steps i and i + 8 of chunk qq.
    {
      const int qq = tid / kLrH, i = tid % kLrH;
      const int sw = lr_swizzle(i);
      const int ta = qq * kLrL + i, tb = ta + kLrH;  // steps within the CTA
      const bool pa = t0 + ta >= t_len, pbd = t0 + tb >= t_len;
      unsigned char* dst = smem + qq * kLrS + i * kLrC * 8;
#pragma unroll
      for (int g = 0; g < kLrG; ++g) {
        const uint4 va = *reinterpret_cast<const uint4*>(
            smem + kLrStage + (ta / kLrBox) * kLrBoxBytes + ((ta % kLrBox) * kLrG + g) * 16);
        const uint4 vb = *reinterpret_cast<const uint4*>(
            smem + kLrStage + (tb / kLrBox) * kLrBoxBytes + ((tb % kLrBox) * kLrG + g) * 16);
        const float sc = (g == 2) ? 2.f * kLog2e : -kLog2e;
        // steps past T: i, o shut (argument -> clamp), f open (e = 0), g 0
        const float padv = (g == 1) ? -3e30f : ((g == 2) ? 0.f : 3e30f);
        const unsigned wa[4] = {va.x, va.y, va.z, va.w};
        const unsigned wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int cc = 0; cc < kLrC; ++cc) {
          const int sh16 = (cc & 1) ? 0 : 16;
          const unsigned mk = (cc & 1) ? 0xffff0000u : 0xffffffffu;
          const float xa = __uint_as_float((wa[cc >> 1] << sh16) & mk);
          const float xb = __uint_as_float((wb[cc >> 1] << sh16) & mk);
          const float bs = sc * sh.par[pb][kLrG + g][cc];
          float2 o = lfma(lf2(sc, sc), lf2(xa, xb), lf2(bs, bs));
          if (pa) o.x = padv;
          if (pbd) o.y = padv;
          *reinterpret_cast<float2*>(dst + g * kLrRowB + (cc ^ sw) * 8) = o;
        }
      }
    }
    LrPar k;
    {
      const float ai = sh.par[pb][0][c], af = sh.par[pb][1][c], ag = sh.par[pb][2][c],
                  ao = sh.par[pb][3][c];
      k.ai = lf2(ai, ai);
      k.af = lf2(af, af);
      k.ag = lf2(ag, ag);
      k.ao = lf2(ao, ao);
      const float ai2 = -kLog2e * ai, af2 = -kLog2e * af, ag2 = 2.f * kLog2e * ag,
                  ao2 = -kLog2e * ao;
      k.ai2 = lf2(ai2, ai2);
      k.af2 = lf2(af2, af2);
      k.ag2 = lf2(ag2, ag2);
      k.ao2 = lf2(ao2, ao2);
    }
    float c0v = sh.par[pb][8][c], h0v = sh.par[pb][9][c];
    __syncthreads();
    // the staging area and the parameter rows are free: the next tile's
    if (tid == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      lr_issue(smem, sh, &map, b2, (next - b2 * nDTc) * kLrC, p.t_base + t0);
    }
    const bool first = (rank == 0 && q == 0);  // chunk holding step 0

    float2 C[kLrH], H[kLrH], P00[kLrH], P01[kLrH], P10[kLrH], P11[kLrH];
#pragma unroll
    for (int i = 0; i < kLrH; ++i) {
      C[i] = lf2(0.f, 0.f);
      H[i] = lf2(0.f, 0.f);
      P00[i] = P01[i] = P10[i] = P11[i] = lf2(0.f, 0.f);
    }
    float cb = first ? c0v : 0.f, hb = first ? h0v : 0.f;  // state before this chunk
    // last_bad: updates applied before the last evaluation that left the
    // channel at or above tol (histogram); nupd: updates applied so far.
    // spec: the last step started from a residual at most spec_tau, so this
    // evaluation is a residual-only check that may certify the iterate.
    int last_bad = -1, updates = 0, kit = 0, nupd = 0;
    float final_m = 0.f;
    bool spec = false;
    for (;; ++kit) {
      const bool cap = (kit >= p.max_iters);
      const bool ronly = cap || spec;
      const int par = phase & 1;
      const unsigned mpar = (phase >> 1) & 1;  // phase parity of mbar[par]
      ++phase;
      const float lastc = C[kLrH - 1].y, lasth = H[kLrH - 1].y;
      float2 DC, DH;
      Aff2 Mx, My;
      float m;
      if (ronly)
        m = lr_pass<false>(base, c * 8, cb, hb, C, H, P00, P01, P10, P11, k, DC, DH, Mx, My);
      else
        m = lr_pass<true>(base, c * 8, cb, hb, C, H, P00, P01, P10, P11, k, DC, DH, Mx, My);
      if (!dval) m = 0.f;
      // the chunk's map: second half after the first
      Aff2 inc = My.after(Mx);
      // inclusive scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
      for (int o = kLrC; o < 32; o <<= 1) {
        const Aff2 prev = lr_shfl_up(inc, o);
        if (lane >= o) inc = inc.after(prev);
      }
      // exclusive: the delta entering the warp -> the delta entering this chunk
      Aff2 xm = lr_shfl_up(inc, kLrC);
      if (kk == 0) xm = Aff2::id();
      const unsigned wm = __reduce_max_sync(kFull, __float_as_uint(m));
      // the channel's maximum over the warp's four chunks (lanes c + 8k)
      unsigned cmu = __float_as_uint(m);
      cmu = max(cmu, __shfl_xor_sync(kFull, cmu, 8));
      cmu = max(cmu, __shfl_xor_sync(kFull, cmu, 16));
      if (kk == kLrK - 1) {
        sh.wagg[par][warp][c][0] = make_float4(inc.m00, inc.m01, inc.m10, inc.m11);
        sh.wagg[par][warp][c][1] = make_float4(inc.d0, inc.d1, lastc, lasth);
      }
      if (kk == 0) sh.wcm[par][warp][c] = __uint_as_float(cmu);
      if (lane == 0) sh.wmax[par][warp] = __uint_as_float(wm);
      __syncthreads();
      // the histogram input: the channel's own maximum over this CTA's steps
      // (warp 0, lanes 0..7; every CTA of the cluster records its own)
      if (q == 0) {
        float chm = 0.f;
#pragma unroll
        for (int w = 0; w < kLrWarps; ++w) chm = fmax_nan(chm, sh.wcm[par][w][c]);
        if (!(chm < p.tol)) last_bad = nupd;
      }
      // maps of the warps before this one: CTA incoming delta -> delta
      // entering this warp; and the CTA's residual maximum
      Aff2 cw = Aff2::id();
#pragma unroll
      for (int w = 0; w < kLrWarps - 1; ++w) {
        if (w < warp) cw = lr_map(sh.wagg[par][w][c][0], sh.wagg[par][w][c][1]).after(cw);
      }
      const float4 wm0 = *reinterpret_cast<const float4*>(&sh.wmax[par][0]);
      const float4 wm1 = *reinterpret_cast<const float4*>(&sh.wmax[par][4]);
      float tmax = fmax_nan(fmax_nan(fmax_nan(wm0.x, wm0.y), fmax_nan(wm0.z, wm0.w)),
                            fmax_nan(fmax_nan(wm1.x, wm1.y), fmax_nan(wm1.z, wm1.w)));
      float2 din_cta = lf2(0.f, 0.f);            // delta entering this CTA
      float2 prev_cta_last = lf2(c0v, h0v);      // state before this CTA's first step
      if (CLS > 1) {
        // testing: the CTA of rank inject_chunk withholds its last exchange
        // (the residual-only evaluation at the cap)
        const bool withhold =
            cap && (p.flags & PARARNN_FLAG_INJECT_WITHHOLD) && rank == p.inject_chunk;
        if (warp == kLrWarps - 1 && !withhold) {
          const float cmax = tmax;
          if (kk == kLrK - 1) {
            const Aff2 cm = inc.after(cw);  // the CTA's map of channel c
            const float4 v0 = make_float4(cm.m00, cm.m01, cm.m10, cm.m11);
            const float4 v1 = make_float4(cm.d0, cm.d1, lastc, lasth);
            for (int r = rank + 1; r < CLS; ++r) {
              const uint32_t rb = lr_mapa(smem_u32(&sh.mbar[par]), r);
              lr_st_async_v4(lr_mapa(smem_u32(&sh.mbox[par].map[rank][c][0]), r), v0, rb);
              lr_st_async_v4(lr_mapa(smem_u32(&sh.mbox[par].map[rank][c][1]), r), v1, rb);
            }
          }
          if (lane < CLS && lane != rank)
            lr_st_async_b32(lr_mapa(smem_u32(&sh.mbox[par].cmax[rank]), lane),
                            __float_as_uint(cmax), lr_mapa(smem_u32(&sh.mbar[par]), lane));
        }
        const bool got = mbar_wait_bounded(&sh.mbar[par], mpar, p.timeout_ns);
        if (!got && status == 0) status = PARARNN_STATUS_TIMEOUT;
#pragma unroll
        for (int r = 0; r < CLS; ++r) {
          if (r != rank) tmax = fmax_nan(tmax, sh.mbox[par].cmax[r]);
          if (r < rank) {
            const float4 m0 = sh.mbox[par].map[r][c][0], m1 = sh.mbox[par].map[r][c][1];
            din_cta = lf2(fmaf(m0.x, din_cta.x, fmaf(m0.y, din_cta.y, m1.x)),
                          fmaf(m0.z, din_cta.x, fmaf(m0.w, din_cta.y, m1.y)));
            if (r == rank - 1) prev_cta_last = lf2(m1.z, m1.w);
          }
        }
        // a phase that did not complete is not re-armed (see the ParaGRU
        // row kernel)
        __syncwarp();
        if (tid == 0 && got) mbar_arrive_expect_tx(&sh.mbar[par], rx);
      }
      final_m = tmax;
      const bool own_ok = tmax < p.tol;
      if (ronly) {
        updates = nupd;
        if (cap) {
          if (!own_ok && status == 0) status = PARARNN_STATUS_NOT_CONVERGED;
          break;
        }
        // the check: certified below chk_tol, else the next evaluation forms
        // the step at the same iterate
        spec = false;
        if (tmax < p.chk_tol) break;
        continue;
      }
      const float2 cin = cw.apply(din_cta);             // delta entering this warp
      const float2 din = first ? lf2(0.f, 0.f) : xm.apply(cin);
      float2 prev_last = lf2(__shfl_up_sync(kFull, lastc, kLrC), __shfl_up_sync(kFull, lasth, kLrC));
      if (kk == 0) {
        if (warp == 0) {
          prev_last = prev_cta_last;
        } else {
          const float4 l1 = sh.wagg[par][warp - 1][c][1];
          prev_last = lf2(l1.z, l1.w);
        }
      }
      cb = first ? c0v : prev_last.x + din.x;
      hb = first ? h0v : prev_last.y + din.y;
      // deltas entering the two halves of the chunk
      const float2 dy = Mx.apply(din);
      const float2 DINC = lf2(din.x, dy.x), DINH = lf2(din.y, dy.y);
#pragma unroll
      for (int i = 0; i < kLrH; ++i) {
        C[i] = lfma(P00[i], DINC, lfma(P01[i], DINH, C[i]));
        H[i] = lfma(P10[i], DINC, lfma(P11[i], DINH, H[i]));
      }
      updates = ++nupd;
      if (own_ok) break;
      spec = tmax <= p.spec_tau;
    }

    if (pj >= 0 && pj < 10 * kLrC) (&sh.par[pb ^ 1][0][0])[pj] = pnext;
    __syncthreads();  // the next tile reads them

    // ---- states straight from registers
    bool bad = false;
    if (dval) {
      const int tq = t0 + q * kLrL;
      const size_t o0 = ((size_t)b * p.T + t_base + tq) * p.D + d;
#pragma unroll
      for (int i = 0; i < kLrH; ++i) {
        if (tq + i < t_len) {
          p.c[o0 + (size_t)i * p.D] = C[i].x;
          p.h[o0 + (size_t)i * p.D] = H[i].x;
          bad |= !isfinite(C[i].x) || !isfinite(H[i].x);
        }
        if (tq + kLrH + i < t_len) {
          p.c[o0 + (size_t)(kLrH + i) * p.D] = C[i].y;
          p.h[o0 + (size_t)(kLrH + i) * p.D] = H[i].y;
          bad |= !isfinite(C[i].y) || !isfinite(H[i].y);
        }
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
    cur = next;
  }
  const int st = __reduce_max_sync(kFull, status);
  if (lane == 0 && st) atomicMax(&p.stats->status, st);
  // no CTA leaves while a peer may still store into its mailboxes
  if (CLS > 1) cluster.sync();
}

// ------------------------------------------------------------- launcher --
int lstm_row_cluster(int T) {
  if (T > kLrTmax) return 0;
  int cls = 1;
  while (cls * kLrSteps < T) cls *= 2;
  return cls;
}
int lstm_row_box_steps() { return kLrBox; }
// steps one CTA holds: a cluster of k CTAs solves up to k times this many
int lstm_row_cta_steps() { return kLrSteps; }
int lstm_row_channels() { return kLrC; }

template <int CLS>
static int launch_lr_t(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream) {
  const long long ntiles = (long long)p.B * ((p.D + kLrC - 1) / kLrC);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = lstm_newton_row<CLS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLrSmem);
  if (e != cudaSuccess) return (int)e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kLrThreads);
  cfg.dynamicSmemBytes = kLrSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CLS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclus = sms / CLS;
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

int launch_lstm_row(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream) {
  switch (lstm_row_cluster(p.t_len)) {
    case 1: return launch_lr_t<1>(map, p, stream);
    case 2: return launch_lr_t<2>(map, p, stream);
    case 4: return launch_lr_t<4>(map, p, stream);
    case 8: return launch_lr_t<8>(map, p, stream);
    default: return 1;
  }
}

}  // namespace pararnn
