// gru_fwd_seq.cu -- fused Newton-scan ParaGRU solve for sequences of up to
// 4096 steps with bf16 input projections: 8 channels per CTA, a cluster of
// CLS = ceil(T / 1024) CTAs per tile, two CTAs per SM, the cell evaluated on
// packed fp32 pairs.
//
// A tile is 8 consecutive channels of one batch row over the whole sequence.
// CTA rank r of the cluster owns steps [1024 r, 1024 (r+1)): 8 warps x 32
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
// CTA by one scan warp per channel, after one CTA barrier; over the CTAs of
// the cluster through distributed shared memory (the scan warp pushes the
// CTA's map and last state into the mailboxes of the CTAs after it, one
// cluster barrier).  The fix-up adds P_t ds_in.  Mailboxes and per-warp data
// are double-buffered by the parity of a phase counter that runs on across
// tiles.  The cluster stops after the update of the first iteration whose
// residual over the tile is below tol, or after a residual-only evaluation at
// the cap; the state before each chunk is re-anchored every iteration to its
// predecessor's pre-update last state plus the incoming delta.
//
// Data: the tile's u arrives bf16 by four TMA boxes of 256 steps into the top
// of the CTA's 98 KB buffer and is expanded in place, once per tile, into the
// fp32 arguments -log2e u_z + b'_z, -log2e u_r + b'_r, 2 log2e u_c + b'_c
// (b' the bias scaled alike), stored per chunk as [gate][pair i][channel]
// {step i, step i + 16}: one 8-byte load per gate and pair, channel c at slot
// c ^ ((i >> 1) & 7) of its pair row so that the expansion's stores are free
// of bank conflicts.  Chunk slots are 3136 bytes, so the four chunks a warp
// reads fall in alternate 64-byte bank halves.  Steps past T get a z argument of 3e30 (clamped to 63), so z -> 0 and f(h) = h.
// Clusters are persistent over tiles; the next tile's boxes are issued as
// soon as the last pass of the current tile is done.  States are stored
// straight from registers (the 8 lanes of a chunk write a 32-byte run).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cgs = cooperative_groups;

constexpr int kRowThreads = 256;
constexpr int kRowWarps = 8;
constexpr int kRowC = 8;                     // channels per tile
constexpr int kRowK = 32 / kRowC;            // chunks per warp
constexpr int kRowL = 32;                    // steps per chunk (per thread)
constexpr int kRowH = kRowL / 2;             // step pairs per chunk
constexpr int kRowSteps = kRowWarps * kRowK * kRowL;  // 1024 steps per CTA
constexpr int kRowChunks = kRowSteps / kRowL;         // 32 chunks per CTA
constexpr int kRowS = 3 * kRowL * kRowC * 4 + 64;     // chunk slot: 3072 bytes + 64
constexpr int kRowU = kRowChunks * kRowS;             // 100352: the tile's fp32 arguments
constexpr int kRowBox = 256;                          // steps per TMA box
constexpr int kRowBoxBytes = kRowBox * 3 * kRowC * 2;  // 12288
constexpr int kRowNBox = kRowSteps / kRowBox;         // 4
constexpr int kRowStage = kRowU - kRowNBox * kRowBoxBytes;  // bf16 staging at the top
constexpr int kRowSmem = kRowU;
constexpr int kRowMaxCluster = 4;
constexpr float kRowLn2 = 0.693147180559945309f;
constexpr int kRowTmax = kRowSteps * kRowMaxCluster;  // 4096
static_assert(kRowStage % 128 == 0 && kRowBoxBytes % 128 == 0, "TMA destinations");
// expansion block j writes chunk slots below the staging bytes of blocks > j
static_assert((kRowBox / kRowL) * kRowS * (kRowNBox - 1) <=
                  kRowStage + kRowBoxBytes * (kRowNBox - 1), "in-place expansion order");
static_assert(kRowThreads == kRowBox, "the expansion takes one step of a box per thread");

struct RowMailbox {  // written by the cluster peers (push model)
  float2 agg[kRowMaxCluster][kRowC];   // CTA map (P, ds) per channel, by rank
  float last[kRowMaxCluster][kRowC];   // CTA's last state before the update
  float cmax[kRowMaxCluster];          // CTA's max|r|
};

struct RowShared {
  float2 wagg[2][kRowWarps][kRowC];  // per (warp, channel) map, then its exclusive prefix
  float wlast[2][kRowWarps][kRowC];  // per (warp, channel): last state before the update
  float wmax[2][kRowWarps];
  RowMailbox mbox[2];
  float bias[3][kRowC];              // scaled bias of the tile's channels
  uint64_t bar;                      // the staging buffer's mbarrier
};

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// channel slot of channel c in pair row i is c ^ row_swizzle(i)
__host__ __device__ constexpr int row_swizzle(int i) { return (i >> 1) & 7; }

// One pass over a chunk: H[i] = (h_i, h_{i+16}) is the iterate, hb the state
// before the chunk.  With kFull the two half-chunks are scanned from a zero
// incoming delta: H becomes the local solution, P the running products, and
// DL / PA the halves' (delta out, product).  Returns max |h_t - f_t|.
// AZ2, AR2, AC2: the h coefficients of the three arguments (-log2e a_z,
// -log2e a_r, 2 log2e a_c); AZ = a_z.
template <bool kFull>
__device__ __forceinline__ float row_pass(const unsigned char* __restrict__ base, int c8, float hb,
                                          float2 (&H)[kRowH], float2 (&P)[kRowH], float2 AZ2,
                                          float2 AR2, float2 AC2, float2 AZ, float2& DLo,
                                          float2& PAo) {
  const float2 ONE = f2(1.f, 1.f), M1 = f2(-1.f, -1.f), M2 = f2(-2.f, -2.f);
  // a_r = -ln2 AR2 and 4 a_c = 2 ln2 AC2: the constants ride on r(1-r), t(1-t)
  const float2 NL = f2(-kRowLn2, -kRowLn2), PL = f2(kRowLn2, kRowLn2);
  const float2 TL = f2(2.f * kRowLn2, 2.f * kRowLn2), MTL = f2(-2.f * kRowLn2, -2.f * kRowLn2);
  float m = 0.f;
  float2 DL = f2(0.f, 0.f), PA = ONE;
  float2 HP = f2(hb, H[kRowH - 1].x);  // states before steps 0 and 16
#pragma unroll
  for (int i = 0; i < kRowH; ++i) {
    const unsigned char* bi = base + ((c8 ^ (row_swizzle(i) * 8)) + i * kRowC * 8);
    const float2 UZ = *reinterpret_cast<const float2*>(bi);
    const float2 UR = *reinterpret_cast<const float2*>(bi + 1 * kRowH * kRowC * 8);
    const float2 UC = *reinterpret_cast<const float2*>(bi + 2 * kRowH * kRowC * 8);
    const float2 HT = H[i];
    // z, r = 1/(1+e) with e = 2^(argument); one shared reciprocal per step
    const float2 TZ = ffma2(AZ2, HP, UZ), TR = ffma2(AR2, HP, UR);
    const float2 EZ = f2(ex2(fminf(TZ.x, 63.f)), ex2(fminf(TZ.y, 63.f)));
    const float2 ER = f2(ex2(fminf(TR.x, 63.f)), ex2(fminf(TR.y, 63.f)));
    const float2 PZ = fadd2(ONE, EZ), PR = fadd2(ONE, ER);
    const float2 PP = fmul2(PZ, PR);
    const float2 INV = f2(rcp(PP.x), rcp(PP.y));
    const float2 Z = fmul2(PR, INV), R = fmul2(PZ, INV);
    const float2 RH = fmul2(R, HP);
    const float2 TC = ffma2(AC2, RH, UC);
    const float2 EC = f2(ex2(TC.x), ex2(TC.y));             // e^{2y}
    const float2 PC = fadd2(ONE, EC);
    const float2 TT = f2(rcp(PC.x), rcp(PC.y));             // t = 1/(1+e^{2y})
    const float2 C = ffma2(M2, TT, ONE);                    // tanh(y) = 1 - 2t
    const float2 CMH = ffma2(HP, M1, C);
    const float2 F = ffma2(Z, CMH, HP);
    const float2 DF = ffma2(F, M1, HT);
    m = fmax_nan(m, fabsf(DF.x));
    m = fmax_nan(m, fabsf(DF.y));
    if (kFull) {
      // A = (1-z) + a_z z(1-z)(c-h) + (1-c^2) z a_c (r + a_r h r(1-r)),
      // with 1-c^2 = 4t(1-t)
      const float2 OMZ = ffma2(Z, M1, ONE);
      const float2 A1 = ffma2(fmul2(AZ, fmul2(Z, OMZ)), CMH, OMZ);
      const float2 T1 = fmul2(TT, ffma2(TT, MTL, TL));   // 2 ln2 t(1-t)
      const float2 S = fmul2(fmul2(Z, T1), AC2);
      const float2 RR = fmul2(R, ffma2(R, PL, NL));      // -ln2 r(1-r)
      const float2 Q = ffma2(fmul2(AR2, HP), RR, R);
      const float2 A = ffma2(S, Q, A1);
      const float2 HN = ffma2(A, DL, F);
      DL = ffma2(HT, M1, HN);
      PA = fmul2(PA, A);
      H[i] = HN;
      P[i] = PA;
    }
    HP = HT;
  }
  DLo = DL;
  PAo = PA;
  return m;
}

// Thread 0: load the tile's four 256-step boxes for CTA `rank` into the
// staging area.
__device__ __forceinline__ void row_issue(unsigned char* smem, uint64_t* bar,
                                          const CUtensorMap* map, int b, int d0, int t0) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(bar, (unsigned)(kRowNBox * kRowBoxBytes));
  for (int j = 0; j < kRowNBox; ++j)
    tma_load_4d(smem + kRowStage + j * kRowBoxBytes, map, bar, d0, 0, t0 + j * kRowBox, b);
}

template <int CLS>
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
  const int t0 = rank * kRowSteps;           // first step of this CTA

  if (tid == 0) mbar_init(&sh.bar, 1);
  __syncthreads();
  if (tid == 0 && clus < ntiles) {
    const int b = clus / nDTc;
    row_issue(smem, &sh.bar, &map, b, (clus - b * nDTc) * kRowC, t0);
  }
  const unsigned char* base = smem + q * kRowS;
  int status = 0;
  int n = 0;
  unsigned phase = 0;  // exchange phases so far, over all tiles
  for (int tile = clus; tile < ntiles; tile += nclus, ++n) {
    const int b = tile / nDTc, d0 = (tile - b * nDTc) * kRowC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    if (tid < 3 * kRowC) {
      const int g = tid / kRowC, cc = tid - g * kRowC;
      const float v = (p.bias && d0 + cc < p.D) ? p.bias[g * p.D + d0 + cc] : 0.f;
      sh.bias[g][cc] = (g == 2 ? 2.f * kLog2e : -kLog2e) * v;
    }
    if (!mbar_wait_bounded(&sh.bar, n & 1, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;
    __syncthreads();
    // ---- expand the staged bf16 rows [t][gate][8 ch] into the fp32 arguments,
    // box by box (each box's rows are read before any of its slots is
    // written).  Thread j takes step j of the box: a warp writes one chunk,
    // and the swizzle spreads its 32 stores over the 32 banks.
#pragma unroll 1
    for (int j = 0; j < kRowNBox; ++j) {
      uint4 v[3];
#pragma unroll
      for (int g = 0; g < 3; ++g)
        v[g] = *reinterpret_cast<const uint4*>(smem + kRowStage + j * kRowBoxBytes +
                                               (tid * 3 + g) * 16);
      __syncthreads();
      const int t = j * kRowBox + tid;  // step within the CTA
      const int qq = t / kRowL, s = t % kRowL, i = s % kRowH;
      float* dst = reinterpret_cast<float*>(smem + qq * kRowS + i * kRowC * 8 + (s / kRowH) * 4);
      const int sw = row_swizzle(i);
      const bool pad = (t0 + t >= p.T);
#pragma unroll
      for (int g = 0; g < 3; ++g) {
        const float sc = (g == 2) ? 2.f * kLog2e : -kLog2e;
        const unsigned w[4] = {v[g].x, v[g].y, v[g].z, v[g].w};
#pragma unroll
        for (int cc = 0; cc < kRowC; ++cc) {
          const unsigned bits = (cc & 1) ? (w[cc >> 1] & 0xffff0000u) : (w[cc >> 1] << 16);
          float o = fmaf(sc, __uint_as_float(bits), sh.bias[g][cc]);
          if (g == 0 && pad) o = 3e30f;  // clamps to 2^63 whatever a_z h is
          dst[g * kRowH * kRowC * 2 + (cc ^ sw) * 2] = o;
        }
      }
      __syncthreads();
    }
    float az = 0.f, ar = 0.f, ac = 0.f;
    if (dval) {
      az = p.a[d];
      ar = p.a[p.D + d];
      ac = p.a[2 * p.D + d];
    }
    const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
    const float2 AZ2 = f2(az2, az2), AR2 = f2(ar2, ar2), AC2 = f2(ac2, ac2), AZ = f2(az, az);
    const float h0v = (dval && p.h0) ? p.h0[(size_t)b * p.D + d] : 0.f;
    const bool first = (rank == 0 && q == 0);  // chunk holding step 0

    float2 H[kRowH], P[kRowH];
#pragma unroll
    for (int i = 0; i < kRowH; ++i) {
      H[i] = f2(0.f, 0.f);
      P[i] = f2(1.f, 1.f);
    }
    float hb = first ? h0v : 0.f;  // state before this chunk
    int last_bad = -1, updates = 0, k = 0;
    float final_m = 0.f;
    for (;; ++k) {
      const bool cap = (k >= p.max_iters);
      const int par = phase & 1;
      ++phase;
      const float last_pre = H[kRowH - 1].y;
      float2 DL, PA;
      float m;
      if (cap)
        m = row_pass<false>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
      else
        m = row_pass<true>(base, c * 8, hb, H, P, AZ2, AR2, AC2, AZ, DL, PA);
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
      if (kk == kRowK - 1) {
        sh.wagg[par][warp][c] = make_float2(IP, Id);
        sh.wlast[par][warp][c] = last_pre;
      }
      if (lane == 0) sh.wmax[par][warp] = __uint_as_float(wm);
      __syncthreads();
      {
        // scan warp for channel `warp` (one per channel): lane l < 8 holds
        // warp l's map; inclusive scan by shuffles, written back in place as
        // the exclusive prefix (CTA incoming delta -> delta entering warp l)
        static_assert(kRowWarps == kRowC, "one scan warp per channel");
        const int cs = warp;
        float2 e = make_float2(1.f, 0.f);
        if (lane < kRowWarps) e = sh.wagg[par][lane][cs];
#pragma unroll
        for (int o = 1; o < kRowWarps; o <<= 1) {
          const float pP = __shfl_up_sync(kFull, e.x, o), pd = __shfl_up_sync(kFull, e.y, o);
          if (lane >= o) {
            e.y = fmaf(e.x, pd, e.y);
            e.x *= pP;
          }
        }
        float sP = __shfl_up_sync(kFull, e.x, 1), sd = __shfl_up_sync(kFull, e.y, 1);
        if (lane == 0) {
          sP = 1.f;
          sd = 0.f;
        }
        // the CTA's residual maximum (warp 0 publishes it)
        const float wv = (lane < kRowWarps) ? sh.wmax[par][lane] : 0.f;
        const unsigned cm = __reduce_max_sync(kFull, __float_as_uint(wv));
        if (lane < kRowWarps) sh.wagg[par][lane][cs] = make_float2(sP, sd);
        if (CLS > 1 && lane == kRowWarps - 1) {
          // this CTA's map and last state, to every CTA from this one on
          const float lastc = sh.wlast[par][kRowWarps - 1][cs];
          for (int r = rank; r < CLS; ++r) {
            RowMailbox* mb = (r == rank) ? &sh.mbox[par] : cluster.map_shared_rank(&sh.mbox[par], r);
            mb->agg[rank][cs] = e;
            mb->last[rank][cs] = lastc;
          }
        }
        if (warp == 0 && lane < CLS) {
          RowMailbox* mb =
              (lane == rank) ? &sh.mbox[par] : cluster.map_shared_rank(&sh.mbox[par], lane);
          mb->cmax[rank] = __uint_as_float(cm);
        }
      }
      if (CLS > 1)
        cluster.sync();
      else
        __syncthreads();
      const float2 pre = sh.wagg[par][warp][c];
      float tmax = 0.f;
      float din_cta = 0.f;          // delta entering this CTA
      float prev_cta_last = h0v;    // state before this CTA's first step
#pragma unroll
      for (int r = 0; r < CLS; ++r) {
        tmax = fmax_nan(tmax, sh.mbox[par].cmax[r]);
        if (r < rank) {
          const float2 a2 = sh.mbox[par].agg[r][c];
          din_cta = fmaf(a2.x, din_cta, a2.y);
        }
      }
      if (CLS > 1 && rank > 0) prev_cta_last = sh.mbox[par].last[rank - 1][c];
      // the histogram input uses the tile's maximum, an upper bound of the
      // channel's own residual
      if (!(tmax < p.tol)) last_bad = k;
      final_m = tmax;
      const bool own_ok = tmax < p.tol;
      if (cap) {
        updates = k;
        if (!own_ok && status == 0) status = PARARNN_STATUS_NOT_CONVERGED;
        break;
      }
      const float cin = fmaf(pre.x, din_cta, pre.y);  // delta entering this warp
      const float din = first ? 0.f : fmaf(xP, cin, xd);
      float prev_last = __shfl_up_sync(kFull, last_pre, kRowC);
      if (kk == 0) prev_last = (warp == 0) ? prev_cta_last : sh.wlast[par][warp - 1][c];
      hb = first ? h0v : prev_last + din;
      // deltas entering the two halves of the chunk
      const float2 DIN = f2(din, fmaf(PA.x, din, DL.x));
#pragma unroll
      for (int i = 0; i < kRowH; ++i) H[i] = ffma2(P[i], DIN, H[i]);
      updates = k + 1;
      if (own_ok) break;
    }
    // every thread of the CTA is past its last pass of this tile (the
    // barrier of the last exchange): the staging area takes the next tile
    const int next = tile + nclus;
    if (tid == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      row_issue(smem, &sh.bar, &map, b2, (next - b2 * nDTc) * kRowC, t0);
    }

    // ---- states straight from registers
    bool bad = false;
    if (dval) {
      const int tq = t0 + q * kRowL;
      float* out = p.h + ((size_t)b * p.T + tq) * p.D + d;
#pragma unroll
      for (int i = 0; i < kRowH; ++i) {
        if (tq + i < p.T) {
          out[(size_t)i * p.D] = H[i].x;
          bad |= !isfinite(H[i].x);
        }
        if (tq + kRowH + i < p.T) {
          out[(size_t)(kRowH + i) * p.D] = H[i].y;
          bad |= !isfinite(H[i].y);
        }
      }
    }
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    if (p.chan_k != nullptr && q == 0 && rank == 0 && dval)
      atomicMax(&p.chan_k[(size_t)b * p.D + d], last_bad + 1);
    if (tid == 0) {
      atomicMax(&p.stats->iters, updates);
      atomicMax(&p.stats->evals, k + 1);
      atomicMax(reinterpret_cast<int*>(&p.stats->max_residual), __float_as_int(final_m));
    }
  }
  const int st = __reduce_max_sync(kFull, status);
  if (lane == 0 && st) atomicMax(&p.stats->status, st);
}

// ------------------------------------------------------------- launcher --
int gru_row_cluster(int T) {
  return T <= 1024 ? 1 : (T <= 2048 ? 2 : (T <= kRowTmax ? 4 : 0));
}
// non-zero when this solve applies to sequences of length T
int gru_seq_wpc(int T) { return gru_row_cluster(T); }
int gru_row_box_steps() { return kRowBox; }
int gru_row_channels() { return kRowC; }

template <int CLS>
static int launch_row_t(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream) {
  const long long ntiles = (long long)p.B * ((p.D + kRowC - 1) / kRowC);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto kern = gru_newton_row<CLS>;
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

int launch_gru_seq(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream) {
  switch (gru_row_cluster(p.T)) {
    case 1: return launch_row_t<1>(map, p, stream);
    case 2: return launch_row_t<2>(map, p, stream);
    case 4: return launch_row_t<4>(map, p, stream);
    default: return 1;
  }
}

}  // namespace pararnn
