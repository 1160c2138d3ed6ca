// gru_fwd_seq.cu -- fused Newton-scan ParaGRU solve for sequences of up to
// 4096 steps with bf16 input projections: 16 channels per CTA, a cluster of
// CLS = ceil(T / 1024) CTAs per tile, the scan mostly inside the CTA.
//
// A tile is 16 consecutive channels of one batch row over the whole
// sequence.  CTA rank r of the cluster owns steps [1024 r, 1024 (r+1)):
// 32 warps x 32 lanes, lane = (k, c) with the channel c = lane % 16 fastest
// and k = lane / 16 one of two 16-step chunks; warp w covers steps
// [32 w, 32 w + 32) of the CTA's range (16K elements per CTA, one CTA per SM,
// 64 registers per thread so 32 warps hide the special-function latency).
//
// Per iteration ("Параллельность RNN?", §1.2-§1.3): each thread evaluates the
// cell, residual and diagonal Jacobian on its 16 steps and scans them serially
// (h'_t = f_t + A_t ds_{t-1}, running product P_t).  The affine chunk
// aggregates (P, ds) are scanned: over the two chunks of a warp by a shuffle,
// over the warps of the CTA through shared memory (every thread composes the
// maps of the warps before it), and over the CTAs of the cluster through
// distributed shared memory (each CTA pushes its map, last state and residual
// into its peers' mailboxes; one cluster barrier).  The fix-up adds
// P_t ds_in.  Two barriers per iteration (the CTA's and the cluster's);
// mailboxes and per-warp data are double-buffered by iteration parity.  The
// cluster stops after the update of the first iteration whose residual over
// the tile is below tol, or after a residual-only evaluation at the cap; the
// state before each chunk is re-anchored every iteration to its
// predecessor's pre-update last state plus the incoming delta.
//
// Data: u stays bf16 in shared memory in the global row order [t][gate][16]
// (96 bytes per step), one TMA box per 16-step chunk in a 128-byte-aligned
// slot of 1664 bytes.  A warp reads chunks 2w and 2w+1 at the same step; so
// that the two land in different banks, odd chunks are loaded from one step
// earlier (17-step boxes) and read at a 96-byte offset: the 32 lanes then read
// 16 distinct words.
// Clusters are persistent over tiles and the next tile's boxes are loaded
// into the second of two buffers while the current tile iterates.  States are
// stored straight from registers: the 16 lanes of a chunk write a 64-byte run
// of a row.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cgs = cooperative_groups;

constexpr int kRowThreads = 1024;
constexpr int kRowWarps = 32;
constexpr int kRowC = 16;                    // channels per tile
constexpr int kRowK = 32 / kRowC;            // chunks per warp
constexpr int kRowL = 16;                    // steps per chunk (per thread)
constexpr int kRowSteps = kRowWarps * kRowK * kRowL;  // 1024 steps per CTA
constexpr int kRowChunks = kRowSteps / kRowL;         // 64 chunks per CTA
constexpr int kRowRowB = 2 * kRowC;          // bytes of one (t, gate) row
constexpr int kRowStepB = 3 * kRowRowB;      // 96 bytes per step
constexpr int kRowBoxSteps = kRowL + 1;      // 17: odd chunks start one step early
constexpr int kRowBoxBytes = kRowBoxSteps * kRowStepB;  // 1632 per TMA box
constexpr int kRowS = 1664;                  // chunk slot, a multiple of 128 bytes
constexpr int kRowBuf = kRowChunks * kRowS;  // 106496 bytes per buffer
constexpr int kRowSmem = 2 * kRowBuf;
constexpr int kRowMaxCluster = 4;
constexpr int kRowTmax = kRowSteps * kRowMaxCluster;  // 4096

struct RowMailbox {  // written by the cluster peers (push model)
  float2 agg[kRowMaxCluster][kRowC];   // CTA map (P, ds) per channel, by rank
  float last[kRowMaxCluster][kRowC];   // CTA's last state before the update
  float cmax[kRowMaxCluster];          // CTA's max|r|
};

struct RowShared {
  float2 wagg[2][kRowWarps][kRowC];  // per (warp, channel) map (P, ds), by parity
  float wlast[2][kRowWarps][kRowC];  // per (warp, channel): last state before the update
  float wmax[2][kRowWarps];
  RowMailbox mbox[2];
  uint64_t bar[2];                   // one mbarrier per u buffer
};

template <bool kFull>
__device__ __forceinline__ float row_pass(const unsigned char* __restrict__ base, float hp,
                                          float (&h)[kRowL], float (&P)[kRowL], float az, float ar,
                                          float ac, float az2, float ar2, float ac2, float bz2,
                                          float br2, float bc2, float& dl_out, float& P_out) {
  float m = 0.f, dl = 0.f, Pacc = 1.f;
#pragma unroll
  for (int i = 0; i < kRowL; ++i) {
    const unsigned short* row = reinterpret_cast<const unsigned short*>(base + i * kRowStepB);
    const float uz = __uint_as_float((unsigned)row[0] << 16);
    const float ur = __uint_as_float((unsigned)row[kRowC] << 16);
    const float uc = __uint_as_float((unsigned)row[2 * kRowC] << 16);
    const float ht = h[i];
    // z, r = 1/(1+e) with e = 2^(-log2e (a h + u + b)); one shared reciprocal
    const float ez = ex2(fminf(fmaf(az2, hp, fmaf(-kLog2e, uz, bz2)), 63.f));
    const float er = ex2(fminf(fmaf(ar2, hp, fmaf(-kLog2e, ur, br2)), 63.f));
    const float pz = 1.f + ez, pr = 1.f + er;
    const float inv = rcp(pz * pr);
    const float z = pr * inv;
    const float r = pz * inv;
    const float rh = r * hp;
    const float ec = ex2(fmaf(ac2, rh, fmaf(2.f * kLog2e, uc, bc2)));  // e^{2y}
    const float c = fmaf(-2.f, rcp(1.f + ec), 1.f);                    // tanh(y)
    const float cmh = c - hp;
    const float f = fmaf(z, cmh, hp);
    m = fmax_nan(m, fabsf(ht - f));
    if (kFull) {
      const float omz = 1.f - z;
      const float zz = z * omz;
      const float omc2 = fmaf(-c, c, 1.f);
      const float rr = fmaf(-r, r, r);
      const float q = fmaf(ar * hp, rr, r);
      const float s = (z * omc2) * ac;
      float A = fmaf(az * zz, cmh, omz);
      A = fmaf(s, q, A);
      const float hn = fmaf(A, dl, f);
      dl = hn - ht;
      Pacc *= A;
      h[i] = hn;
      P[i] = Pacc;
    }
    hp = ht;
  }
  dl_out = dl;
  P_out = Pacc;
  return m;
}

// Thread 0: load the 64 chunk boxes of one tile for CTA `rank` into `buf`.
__device__ __forceinline__ void row_issue(unsigned char* buf, uint64_t* bar, const CUtensorMap* map,
                                          int b, int d0, int t0) {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  mbar_arrive_expect_tx(bar, (unsigned)(kRowChunks * kRowBoxBytes));
  for (int ch = 0; ch < kRowChunks; ++ch)
    tma_load_4d(buf + ch * kRowS, map, bar, d0, 0, t0 + ch * kRowL - (ch & 1), b);
}

template <int CLS>
__global__ void __launch_bounds__(kRowThreads, 1)
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

  if (tid == 0) {
    mbar_init(&sh.bar[0], 1);
    mbar_init(&sh.bar[1], 1);
  }
  __syncthreads();
  if (tid == 0 && clus < ntiles) {
    const int b = clus / nDTc;
    row_issue(smem, &sh.bar[0], &map, b, (clus - b * nDTc) * kRowC, t0);
  }
  int status = 0;
  int n = 0;
  for (int tile = clus; tile < ntiles; tile += nclus, ++n) {
    const int bi = n & 1;
    unsigned char* buf = smem + bi * kRowBuf;
    const int next = tile + nclus;
    if (tid == 0 && next < ntiles) {
      const int b2 = next / nDTc;
      row_issue(smem + (bi ^ 1) * kRowBuf, &sh.bar[bi ^ 1], &map, b2, (next - b2 * nDTc) * kRowC,
                t0);
    }
    if (!mbar_wait_bounded(&sh.bar[bi], (n >> 1) & 1, p.timeout_ns))
      status = PARARNN_STATUS_TIMEOUT;
    const int b = tile / nDTc, d0 = (tile - b * nDTc) * kRowC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    // steps past the end of the sequence: u_z = -2e30 so that z -> 0, f(h) = h
    const int tend = min(kRowSteps, p.T - t0);  // valid steps of this CTA (may be <= 0)
    if (tend < kRowSteps) {
      for (int e = max(tend, 0) * kRowC + tid; e < kRowSteps * kRowC; e += kRowThreads) {
        const int t = e / kRowC, cc = e - t * kRowC;
        const int qq = t >> 4;
        *reinterpret_cast<unsigned short*>(buf + qq * kRowS + ((t & 15) + (qq & 1)) * kRowStepB +
                                           cc * 2) = (unsigned short)0xf1c9u;
      }
      __syncthreads();
    }
    float az = 0.f, ar = 0.f, ac = 0.f, bz = 0.f, br = 0.f, bc = 0.f;
    if (dval) {
      az = p.a[d];
      ar = p.a[p.D + d];
      ac = p.a[2 * p.D + d];
      if (p.bias) {
        bz = p.bias[d];
        br = p.bias[p.D + d];
        bc = p.bias[2 * p.D + d];
      }
    }
    const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
    const float bz2 = -kLog2e * bz, br2 = -kLog2e * br, bc2 = 2.f * kLog2e * bc;
    const float h0v = (dval && p.h0) ? p.h0[(size_t)b * p.D + d] : 0.f;
    const bool first = (rank == 0 && q == 0);  // chunk holding step 0
    const unsigned char* base = buf + q * kRowS + (q & 1) * kRowStepB + c * 2;

    float h[kRowL], P[kRowL];
#pragma unroll
    for (int i = 0; i < kRowL; ++i) {
      h[i] = 0.f;
      P[i] = 1.f;
    }
    float hb = first ? h0v : 0.f;  // state before this chunk
    int last_bad = -1, updates = 0, k = 0;
    float final_m = 0.f;
    for (;; ++k) {
      const bool cap = (k >= p.max_iters);
      const int par = k & 1;
      const float last_pre = h[kRowL - 1];
      float dl, Pw, m;
      if (cap)
        m = row_pass<false>(base, hb, h, P, az, ar, ac, az2, ar2, ac2, bz2, br2, bc2, dl, Pw);
      else
        m = row_pass<true>(base, hb, h, P, az, ar, ac, az2, ar2, ac2, bz2, br2, bc2, dl, Pw);
      if (!dval) m = 0.f;
      // the warp's two chunks of channel c (lanes c and c + 16)
      const float oP = __shfl_up_sync(kFull, Pw, kRowC), od = __shfl_up_sync(kFull, dl, kRowC);
      float IP = Pw, Id = dl;
      if (kk == 1) {
        Id = fmaf(Pw, od, dl);
        IP = Pw * oP;
      }
      float wm = m;
#pragma unroll
      for (int o = 16; o; o >>= 1) wm = fmax_nan(wm, __shfl_xor_sync(kFull, wm, o));
      if (kk == kRowK - 1) {
        sh.wagg[par][warp][c] = make_float2(IP, Id);
        sh.wlast[par][warp][c] = last_pre;
      }
      if (lane == 0) sh.wmax[par][warp] = wm;
      __syncthreads();
      // map of the warps before this one (this CTA's incoming delta -> delta
      // entering the warp), and the CTA's map and residual
      float cP = 1.f, cd = 0.f;
      for (int w = 0; w < warp; ++w) {
        const float2 a2 = sh.wagg[par][w][c];
        cd = fmaf(a2.x, cd, a2.y);
        cP *= a2.x;
      }
      float cmax = 0.f;
#pragma unroll
      for (int w = 0; w < kRowWarps; ++w) cmax = fmax_nan(cmax, sh.wmax[par][w]);
      float tmax = cmax;
      float din_cta = 0.f;          // delta entering this CTA
      float prev_cta_last = h0v;    // state before this CTA's first step
      if (CLS > 1) {
        if (warp == kRowWarps - 1 && kk == kRowK - 1) {
          // this CTA's map = last warp's inclusive map o maps of the warps before
          const float2 mapc = make_float2(IP * cP, fmaf(IP, cd, Id));
          for (int r = rank; r < CLS; ++r) {
            RowMailbox* mb = (r == rank) ? &sh.mbox[par] : cluster.map_shared_rank(&sh.mbox[par], r);
            mb->agg[rank][c] = mapc;
            mb->last[rank][c] = last_pre;
          }
        }
        if (tid < CLS && tid != rank) cluster.map_shared_rank(&sh.mbox[par], tid)->cmax[rank] = cmax;
        if (tid == 0) sh.mbox[par].cmax[rank] = cmax;
        cluster.sync();
#pragma unroll
        for (int r = 0; r < CLS; ++r) {
          tmax = fmax_nan(tmax, sh.mbox[par].cmax[r]);
          if (r < rank) {
            const float2 a2 = sh.mbox[par].agg[r][c];
            din_cta = fmaf(a2.x, din_cta, a2.y);
          }
        }
        if (rank > 0) prev_cta_last = sh.mbox[par].last[rank - 1][c];
      }
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
      const float cin = fmaf(cP, din_cta, cd);  // delta entering this warp
      const float din = first ? 0.f : (kk == 0 ? cin : fmaf(oP, cin, od));
      float prev_last = __shfl_up_sync(kFull, last_pre, kRowC);
      if (kk == 0) prev_last = (warp == 0) ? prev_cta_last : sh.wlast[par][warp - 1][c];
      hb = first ? h0v : prev_last + din;
#pragma unroll
      for (int i = 0; i < kRowL; ++i) h[i] = fmaf(P[i], din, h[i]);
      updates = k + 1;
      if (own_ok) break;
    }

    // ---- states straight from registers
    bool bad = false;
    if (dval) {
      const int tq = t0 + q * kRowL;
      float* out = p.h + ((size_t)b * p.T + tq) * p.D + d;
#pragma unroll
      for (int i = 0; i < kRowL; ++i) {
        if (tq + i < p.T) {
          out[(size_t)i * p.D] = h[i];
          bad |= !isfinite(h[i]);
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
    // buffer bi is refilled two tiles on; peers may still read this CTA's
    // mailbox of the last iteration until they pass their next barrier
    __syncthreads();
    if (CLS > 1) cluster.sync();
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
int gru_row_box_steps() { return kRowBoxSteps; }
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
  // persistent clusters: as many as can be resident, at most one per tile
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

int launch_gru_seq(const CUtensorMap& map, const FwdParams& p, cudaStream_t stream) {
  switch (gru_row_cluster(p.T)) {
    case 1: return launch_row_t<1>(map, p, stream);
    case 2: return launch_row_t<2>(map, p, stream);
    case 4: return launch_row_t<4>(map, p, stream);
    default: return 1;
  }
}

}  // namespace pararnn
