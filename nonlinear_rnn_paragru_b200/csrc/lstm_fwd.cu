// lstm_fwd.cu -- fused Newton-scan forward solve of the ParaLSTM recurrence.
//
// Same organisation as the ParaGRU solve (gru_fwd.cu), with a 2-state
// channel s = (c, h) and a 2x2 Jacobian block per channel and step
// ("Apple научила классические RNN масштабироваться до 7B параметров...",
// "Что именно сделали технически", item 3: ParaLSTM gives 2x2
// block-diagonal Jacobians).  One CTA owns 32 channels x kTC = 96 steps:
//   * u (i, f, g, o projections) arrives once by TMA and is rewritten as
//     pre-scaled fp32 rows [t][channel][gate] (bias folded in),
//   * each thread (warp w, lane l) keeps (c, h) of channel l for steps
//     [24w, 24w + 24) in registers, plus the running product P_t of the 2x2
//     Jacobians since the start of its sub-chunk (fp32: six registers per
//     step, hence 4 warps per CTA and two CTAs per SM).
// Newton iteration k ("Параллельность RNN?", §1.2-§1.3): evaluate the cell,
// the residual r_t = s_t - f(s_{t-1}) and A_t = df/ds (s_{t-1}); solve
// ds_t = A_t ds_{t-1} - r_t by scanning the affine pairs (A, -r) thread-
// serially, across warps, across the CTAs of a cluster (DSMEM mailboxes) and
// across cluster chunks (decoupled look-back); update s <- s + ds.  Stopping
// and the iteration cap follow the ParaGRU solve.
#include <cuda_bf16.h>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace cg = cooperative_groups;

constexpr int kLstmNW = 4;                  // warps per CTA
constexpr int kLstmL = 24;                  // steps per thread
constexpr int kLstmTC = kLstmNW * kLstmL;   // steps per chunk
constexpr int kLstmRow = kChan * 16;        // bytes per step row: float4 [32]
constexpr int kLstmSmemU = kLstmTC * kLstmRow;  // 48 KB
constexpr int kLstmThreads = kLstmNW * 32;
constexpr int kLstmMaxCluster = 16;
// Padded steps past the end of the sequence: forget gate 1, input and output
// gates 2^-40, so f(c, h) ~= (c, 0) -- they converge after one update, never
// hold up the stopping test and never influence a real step.
constexpr float kLstmPadOpen = -1e30f;  // pre-scaled arg -> e = 0  -> gate 1
constexpr float kLstmPadShut = 1e30f;   // pre-scaled arg -> e = 2^40 -> gate ~0

struct LstmSlot {
  Aff2 agg[kLstmMaxCluster][kChan];
  float cmax[kLstmMaxCluster];
  float2 dinc[kChan];
  float2 plast[kChan];  // last (c, h) before the update of CTA rank-1
  float2 clast[kChan];  // last (c, h) before the update of the previous cluster chunk
  int upok;
  int timeout;
  int haveclast;
};

struct LstmShared {
  Aff2 agg[kLstmNW][kChan];    // warp aggregates, then exclusive warp prefixes
  float2 din[kLstmNW][kChan];  // incoming delta of each warp's sub-chunk
  float2 slo[kLstmNW][kChan];  // each warp's last (c, h) before the update
  float2 bnd[kLstmNW][kChan];  // each warp's boundary for the next iteration
  float chmax[kLstmNW][kChan];
  float wmax[kLstmNW];
  LstmSlot slot[2];
  int ctl[4];
  uint64_t bar;
};

struct LstmConsts {
  float ai, af, ag, ao;      // raw diagonal weights (Jacobian)
  float ai2, af2, ag2, ao2;  // pre-scaled: -log2e a (i, f, o), 2 log2e a (g)
};

// One pass over the thread's 24 steps: evaluate the cell (and, when kFull, its
// Jacobian and the local scan).  Returns the lane's max |r| over c and h.
template <bool kFull>
__device__ __forceinline__ float lstm_pass(const unsigned char* __restrict__ rows, int lane,
                                           float cp, float hp, float (&c)[kLstmL],
                                           float (&h)[kLstmL], float (&P00)[kLstmL],
                                           float (&P01)[kLstmL], float (&P10)[kLstmL],
                                           float (&P11)[kLstmL], const LstmConsts& k,
                                           Aff2& agg) {
  float m = 0.f, dc = 0.f, dh = 0.f;
  float p00 = 1.f, p01 = 0.f, p10 = 0.f, p11 = 1.f;
#pragma unroll
  for (int s = 0; s < kLstmL; ++s) {
    const float4 uu = reinterpret_cast<const float4*>(rows + s * kLstmRow)[lane];
    const float ct = c[s], ht = h[s];
    // sigmoids of i, f, o share one reciprocal (arguments clamped so the
    // product of the three denominators stays finite)
    const float ei = ex2(fmin_nan(fmaf(k.ai2, hp, uu.x), 40.f));
    const float ef = ex2(fmin_nan(fmaf(k.af2, hp, uu.y), 40.f));
    const float eo = ex2(fmin_nan(fmaf(k.ao2, hp, uu.w), 40.f));
    const float eg = ex2(fmaf(k.ag2, hp, uu.z));
    const float pi = 1.f + ei, pf = 1.f + ef, po = 1.f + eo;
    const float pfo = pf * po;
    const float inv = rcp(pi * pfo);
    const float gi = pfo * inv;
    const float gf = (pi * po) * inv;
    const float go = (pi * pf) * inv;
    const float gg = fmaf(-2.f, rcp(1.f + eg), 1.f);
    const float cn = fmaf(gf, cp, gi * gg);  // c' = f c + i g
    const float ecn = ex2((2.f * kLog2e) * cn);
    const float tc = fmaf(-2.f, rcp(1.f + ecn), 1.f);  // tanh(c')
    const float hn = go * tc;                           // h' = o tanh(c')
    m = fmax_nan(m, fmax_nan(fabsf(ct - cn), fabsf(ht - hn)));
    if (kFull) {
      const float di = fmaf(-gi, gi, gi), df = fmaf(-gf, gf, gf), dg = fmaf(-gg, gg, 1.f);
      const float dox = fmaf(-go, go, go), dtc = fmaf(-tc, tc, 1.f);
      // dc'/dh through the pre-activations of i, f, g
      const float X = fmaf(cp * df, k.af, fmaf(gg * di, k.ai, (gi * dg) * k.ag));
      const float kk = go * dtc;
      const float a00 = gf, a01 = X, a10 = kk * gf, a11 = fmaf(dox * tc, k.ao, kk * X);
      // local scan: s'_t = f_t + A_t ds_{t-1}
      const float cnew = fmaf(a00, dc, fmaf(a01, dh, cn));
      const float hnew = fmaf(a10, dc, fmaf(a11, dh, hn));
      dc = cnew - ct;
      dh = hnew - ht;
      const float q00 = fmaf(a00, p00, a01 * p10), q01 = fmaf(a00, p01, a01 * p11);
      const float q10 = fmaf(a10, p00, a11 * p10), q11 = fmaf(a10, p01, a11 * p11);
      p00 = q00;
      p01 = q01;
      p10 = q10;
      p11 = q11;
      c[s] = cnew;
      h[s] = hnew;
      P00[s] = p00;
      P01[s] = p01;
      P10[s] = p10;
      P11[s] = p11;
    }
    cp = ct;
    hp = ht;
  }
  agg = Aff2{p00, p01, p10, p11, dc, dh};
  return m;
}

template <bool kBF16>
__global__ void __launch_bounds__(kLstmThreads, 2)
    lstm_newton_fused(const __grid_constant__ CUtensorMap tmap, const FwdParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  __shared__ LstmShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CL = p.CL;
  const int rank = (CL > 1) ? (int)cluster.block_rank() : 0;
  const bool multi = p.nCC > 1;

  if (tid == 0) {
    sh.ctl[0] = multi ? (rank == 0 ? (int)atomicAdd(&p.hdr->ticket, 1u) : -1)
                      : (int)(blockIdx.x / CL);
    sh.ctl[1] = multi ? (int)(*(volatile unsigned*)&p.hdr->epoch) : 0;
    sh.ctl[2] = 0;
    mbar_init(&sh.bar, 1);
  }
  if (CL > 1) cluster.sync();
  else __syncthreads();
  if (multi && rank != 0 && tid == 0) {
    const int* r0 = cluster.map_shared_rank(&sh.ctl[0], 0);
    sh.ctl[0] = r0[0];
  }
  __syncthreads();
  const int ticket = sh.ctl[0];
  const unsigned epoch = (unsigned)sh.ctl[1];
  const int tile = ticket / p.nCC, jc = ticket - tile * p.nCC;
  const int j = jc * CL + rank;
  const int b = tile / p.nDT, d0 = (tile - b * p.nDT) * kChan;
  const int t0 = j * kLstmTC;
  const int d = d0 + lane;
  const bool dval = d < p.D;
  constexpr unsigned kBytes = kLstmTC * 4 * kChan * (kBF16 ? 2 : 4);
  unsigned char* raw = dyn + (kBF16 ? kLstmSmemU / 2 : 0);

  if (tid == 0) {
    mbar_arrive_expect_tx(&sh.bar, kBytes);
    tma_load_4d(raw, &tmap, &sh.bar, d0, 0, t0, b);
  }
  LstmConsts K = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float bb[4] = {0.f, 0.f, 0.f, 0.f};
  if (dval) {
    K.ai = p.a[d];
    K.af = p.a[p.D + d];
    K.ag = p.a[2 * p.D + d];
    K.ao = p.a[3 * p.D + d];
    if (p.bias) {
#pragma unroll
      for (int q = 0; q < 4; ++q) bb[q] = p.bias[q * p.D + d];
    }
  }
  K.ai2 = -kLog2e * K.ai;
  K.af2 = -kLog2e * K.af;
  K.ag2 = 2.f * kLog2e * K.ag;
  K.ao2 = -kLog2e * K.ao;
  const float sc[4] = {-kLog2e, -kLog2e, 2.f * kLog2e, -kLog2e};
  float cb = 0.f, hbv = 0.f;  // boundary (c, h) of warp 0
  if (j == 0 && dval) {
    if (p.c0) cb = p.c0[(size_t)b * p.D + d];
    if (p.h0) hbv = p.h0[(size_t)b * p.D + d];
  }

  int status = 0;
  if (!mbar_wait_bounded(&sh.bar, 0, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;

  // ---- rewrite u as pre-scaled fp32 rows [t][channel][gate]
  auto prep = [&](int t, const float (&v)[4]) {
    float4 o;
    if (t0 + t < p.T) {
      o = make_float4(sc[0] * (v[0] + bb[0]), sc[1] * (v[1] + bb[1]), sc[2] * (v[2] + bb[2]),
                      sc[3] * (v[3] + bb[3]));
    } else {
      o = make_float4(kLstmPadShut, kLstmPadOpen, 0.f, kLstmPadShut);
    }
    reinterpret_cast<float4*>(dyn + t * kLstmRow)[lane] = o;
  };
  if constexpr (kBF16) {
    // raw [t][g][32] bf16 (256 B per step) sits in the upper half; expand
    // 16-step blocks in increasing t so no write lands on an unread row.
    const __nv_bfloat16* rb = reinterpret_cast<const __nv_bfloat16*>(raw);
    constexpr int kRowsPerWarp = 16 / kLstmNW;
#pragma unroll 1
    for (int blk = 0; blk < kLstmTC / 16; ++blk) {
      float v[kRowsPerWarp][4];
#pragma unroll
      for (int q = 0; q < kRowsPerWarp; ++q) {
        const int t = blk * 16 + warp * kRowsPerWarp + q;
#pragma unroll
        for (int g = 0; g < 4; ++g) v[q][g] = __bfloat162float(rb[(t * 4 + g) * kChan + lane]);
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < kRowsPerWarp; ++q) prep(blk * 16 + warp * kRowsPerWarp + q, v[q]);
      __syncthreads();
    }
  } else {
    // raw [t][g][32] fp32 is the same 512 B per step: transpose in place,
    // each warp its own rows.
#pragma unroll 2
    for (int q = 0; q < kLstmL; ++q) {
      const int t = warp * kLstmL + q;
      const float* rf = reinterpret_cast<const float*>(dyn + t * kLstmRow);
      float v[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) v[g] = rf[g * kChan + lane];
      __syncwarp();
      prep(t, v);
      __syncwarp();
    }
    __syncthreads();
  }

  float c[kLstmL], h[kLstmL], P00[kLstmL], P01[kLstmL], P10[kLstmL], P11[kLstmL];
#pragma unroll
  for (int s = 0; s < kLstmL; ++s) {
    c[s] = h[s] = 0.f;
    P00[s] = P11[s] = 1.f;
    P01[s] = P10[s] = 0.f;
  }
  const int tw0 = warp * kLstmL;
  const int nvalid = min(kLstmL, p.T - (t0 + tw0));
  const unsigned char* rows = dyn + tw0 * kLstmRow;
  const int rec_stride = p.max_iters + 1;
  const int ticket0 = ticket - jc;
  const bool publisher = multi && rank == CL - 1 && jc < p.nCC - 1 &&
                         !((p.flags & PARARNN_FLAG_INJECT_WITHHOLD) && ticket == p.inject_chunk);

  bool frozen = (jc == 0);
  int last_bad = -1;
  float final_m = 0.f;
  int updates = 0, k = 0;
  float bc = (warp == 0) ? cb : 0.f, bh = (warp == 0) ? hbv : 0.f;  // s_{t-1} of this warp

  for (;; ++k) {
    const bool cap = (k >= p.max_iters);
    const int par = k & 1;
    sh.slo[warp][lane] = make_float2(c[kLstmL - 1], h[kLstmL - 1]);
    Aff2 wagg;
    float m = cap ? lstm_pass<false>(rows, lane, bc, bh, c, h, P00, P01, P10, P11, K, wagg)
                  : lstm_pass<true>(rows, lane, bc, bh, c, h, P00, P01, P10, P11, K, wagg);
    if (!dval) m = 0.f;
    sh.agg[warp][lane] = wagg;
    sh.chmax[warp][lane] = m;
    float wm = m;
#pragma unroll
    for (int o = 16; o; o >>= 1) wm = fmax_nan(wm, __shfl_xor_sync(kFull, wm, o));
    if (lane == 0) sh.wmax[warp] = wm;
    __syncthreads();

    if (warp == 0) {
      Aff2 cta = Aff2::id();
      float cm = 0.f, chm = 0.f;
#pragma unroll
      for (int w = 0; w < kLstmNW; ++w) {
        const Aff2 ag = sh.agg[w][lane];
        sh.agg[w][lane] = cta;
        cta = ag.after(cta);
        cm = fmax_nan(cm, sh.wmax[w]);
        chm = fmax_nan(chm, sh.chmax[w][lane]);
      }
      if (dval && !(chm < p.tol)) last_bad = k;
      sh.slot[par].agg[rank][lane] = cta;
      if (lane == 0) sh.slot[par].cmax[rank] = cm;
      for (int r = 0; r < CL; ++r) {
        if (r == rank) continue;
        LstmSlot* peer = cluster.map_shared_rank(&sh.slot[par], r);
        if (r > rank) peer->agg[rank][lane] = cta;
        if (r == rank + 1) peer->plast[lane] = sh.slo[kLstmNW - 1][lane];
        if (lane == 0) peer->cmax[rank] = cm;
      }
    }
    if (CL > 1) cluster.sync();
    else __syncthreads();
    Aff2 ex = Aff2::id();
    float clmax = 0.f;
    if (warp == 0) {
      const LstmSlot& sl = sh.slot[par];
#pragma unroll
      for (int r = 0; r < kLstmMaxCluster; ++r) {
        if (r < rank) ex = sl.agg[r][lane].after(ex);
        if (r < CL) clmax = fmax_nan(clmax, sl.cmax[r]);
      }
      final_m = clmax;
      if (multi && rank == CL - 1 && !cap) {
        const bool own_ok = clmax < p.tol;
        const Aff2 clus = sl.agg[rank][lane].after(ex);
        const size_t rec = (size_t)ticket * rec_stride + k;
        float* rv = p.rec_vals + rec * (size_t)(kChan * rec_floats<Aff2>());
        float2 dinc = make_float2(0.f, 0.f), clast = make_float2(0.f, 0.f);
        bool up_ok = true, to = false, have = false;
        if (publisher) rec_put_last(rv, lane, sh.slo[kLstmNW - 1][lane]);
        if (!frozen) {
          if (publisher) {
            rec_put_agg(rv, lane, clus);
            publish_flag(&p.rec_flags[rec], make_flag(epoch, kRecAgg, own_ok));
          }
          if (lookback<Aff2, float2>(p.rec_flags, p.rec_vals, ticket0, jc, k, rec_stride, epoch,
                                     p.timeout_ns, dinc, up_ok, &clast)) {
            have = true;
          } else {
            dinc = make_float2(0.f, 0.f);
            up_ok = true;
            to = true;
          }
        }
        if (publisher) {
          rec_put_incl(rv, lane, clus.apply(dinc));
          publish_flag(&p.rec_flags[rec], make_flag(epoch, kRecIncl, up_ok && own_ok));
        }
        for (int r = 0; r < CL; ++r) {
          LstmSlot* peer = (r == rank) ? &sh.slot[par] : cluster.map_shared_rank(&sh.slot[par], r);
          peer->dinc[lane] = dinc;
          peer->clast[lane] = clast;
          if (lane == 0) {
            peer->upok = up_ok ? 1 : 0;
            peer->timeout = to ? 1 : 0;
            peer->haveclast = have ? 1 : 0;
          }
        }
      }
    }
    if (multi && !cap) cluster.sync();
    if (warp == 0) {
      const bool own_ok = clmax < p.tol;
      int stop = 0;
      if (cap) {
        stop = 1;
        updates = k;
        if (!own_ok && status == 0) status = PARARNN_STATUS_NOT_CONVERGED;
      } else {
        float2 dinc = make_float2(0.f, 0.f);
        bool up_ok = true;
        float2 base = make_float2(bc, bh);  // this CTA's boundary before the update
        if (multi) {
          dinc = sh.slot[par].dinc[lane];
          up_ok = sh.slot[par].upok != 0;
          if (sh.slot[par].timeout) status = PARARNN_STATUS_TIMEOUT;
          if (rank == 0 && sh.slot[par].haveclast) base = sh.slot[par].clast[lane];
        }
        if (rank > 0) base = sh.slot[par].plast[lane];
        if (up_ok) frozen = true;
        const float2 din = ex.apply(dinc);
        stop = (up_ok && own_ok) ? 1 : 0;
        updates = k + 1;
#pragma unroll
        for (int w = 0; w < kLstmNW; ++w) {
          const float2 dw = sh.agg[w][lane].apply(din);
          const float2 b0 = (w == 0) ? base : sh.slo[w - 1][lane];
          sh.din[w][lane] = dw;
          sh.bnd[w][lane] = make_float2(b0.x + dw.x, b0.y + dw.y);
        }
      }
      if (lane == 0) sh.ctl[2] = stop;
    }
    __syncthreads();
    if (!cap) {
      const float2 din = sh.din[warp][lane];
      const float2 nb = sh.bnd[warp][lane];
      bc = nb.x;
      bh = nb.y;
#pragma unroll
      for (int s = 0; s < kLstmL; ++s) {
        c[s] = fmaf(P00[s], din.x, fmaf(P01[s], din.y, c[s]));
        h[s] = fmaf(P10[s], din.x, fmaf(P11[s], din.y, h[s]));
      }
    }
    if (sh.ctl[2]) break;
  }
  if (CL > 1) cluster.sync();

  bool bad = false;
  if (dval) {
    const size_t o = ((size_t)b * p.T + t0 + tw0) * p.D + d;
#pragma unroll
    for (int s = 0; s < kLstmL; ++s) {
      if (s < nvalid) {
        p.c[o + (size_t)s * p.D] = c[s];
        p.h[o + (size_t)s * p.D] = h[s];
        bad |= !isfinite(c[s]) || !isfinite(h[s]);
      }
    }
  }
  if (__syncthreads_or(bad) && tid == 0 && status < PARARNN_STATUS_NONFINITE)
    status = PARARNN_STATUS_NONFINITE;
  if (warp == 0) {
    if (p.chan_k != nullptr && dval) atomicMax(&p.chan_k[(size_t)b * p.D + d], last_bad + 1);
    const int st = __reduce_max_sync(kFull, status);
    if (lane == 0) {
      atomicMax(&p.stats->iters, updates);
      atomicMax(&p.stats->evals, k + 1);
      atomicMax(reinterpret_cast<int*>(&p.stats->max_residual), __float_as_int(final_m));
      atomicMax(&p.stats->status, st);
    }
  } else if (tid == 32 && status != 0) {
    atomicMax(&p.stats->status, status);
  }
}

// ------------------------------------------------------------- launcher --
template <bool kBF16>
static int launch_lstm_t(const CUtensorMap& tmap, const FwdParams& p, int nctas,
                         cudaStream_t stream) {
  auto kern = lstm_newton_fused<kBF16>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLstmSmemU);
  if (e != cudaSuccess) return (int)e;
  if (p.CL > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return (int)e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kLstmThreads);
  cfg.dynamicSmemBytes = kLstmSmemU;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return (int)cudaLaunchKernelEx(&cfg, kern, tmap, p);
}

int launch_lstm_fwd(const CUtensorMap& tmap, bool bf16, const FwdParams& p, int nctas,
                    cudaStream_t stream) {
  return bf16 ? launch_lstm_t<true>(tmap, p, nctas, stream)
              : launch_lstm_t<false>(tmap, p, nctas, stream);
}

int lstm_max_cluster(bool bf16) {
  auto kern = bf16 ? lstm_newton_fused<true> : lstm_newton_fused<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLstmSmemU) !=
      cudaSuccess)
    return 0;
  for (int cl : {16, 8, 4, 2, 1}) {
    if (cl > 8 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl * 64);
    cfg.blockDim = dim3(kLstmThreads);
    cfg.dynamicSmemBytes = kLstmSmemU;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) return cl;
    cudaGetLastError();
  }
  return 0;
}

int lstm_chunk_steps() { return kLstmTC; }

}  // namespace pararnn
