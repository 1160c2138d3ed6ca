// gru_fwd.cu -- fused Newton-scan forward solve of the ParaGRU recurrence.
//
// One CTA owns a tile of 32 consecutive channels (one per lane) of one batch
// row over a chunk of kTC = 256 time steps, and keeps it on chip for every
// Newton iteration:
//   * the gate projections u arrive once by a TMA bulk-tensor load and are
//     rewritten in shared memory as pre-scaled fp32 (bias folded in),
//   * the iterate h and the running Jacobian products P live in registers
//     (warp w, lane l owns channel l for steps [32w, 32w + 32) of the chunk).
// Newton iteration k ("Параллельность RNN?", §1.2-§1.3):
//   1. evaluate the cell at the iterate: f_t = f(h_{t-1}, u_t), the residual
//      r_t = h_t - f_t and the diagonal Jacobian A_t = df/dh (h_{t-1}),
//   2. solve ds_t = A_t ds_{t-1} - r_t by an associative scan of the affine
//      pairs (A, -r): thread-serial over its 32 steps, across the 8 warps
//      through shared memory, across the CTAs of a thread-block cluster (up to
//      16 chunks = 4096 steps) through distributed shared memory, and across
//      cluster chunks of longer sequences by decoupled look-back,
//   3. update h <- h + ds.
// Written per element as h'_t = f_t + A_t ds_{t-1}: the local pass produces
// h'_t with a zero incoming delta and P_t = prod A; the fix-up adds P_t ds_in.
//
// Stopping (per cluster chunk, decided identically by all its CTAs and in a
// way every downstream cluster chunk agrees with): after the update of
// iteration k a cluster chunk stops when its own max|r| at iteration k and
// that of every upstream cluster chunk are below tol; its successors then
// treat the boundary as fixed.  At most max_iters updates are applied; a
// residual-only evaluation closes a run that hits the cap.
#include <cuda_bf16.h>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

constexpr int kGruNW = 8;               // warps per CTA
constexpr int kGruL = 32;               // steps per thread
constexpr int kGruTC = kGruNW * kGruL;  // steps per chunk
constexpr int kGruRow = kChan * 12;     // bytes per step row: float2 zr[32], float c[32]
constexpr int kGruSmemU = kGruTC * kGruRow;  // 96 KB
constexpr int kGruThreads = kGruNW * 32;
// Steps past the end of the sequence (the ragged last chunk) get an update
// gate of 2^-63, so f(h) = h there: they cost nothing to converge, never hold
// up the stopping test and never influence a real step (they come after it).
constexpr float kPadZ = 1e30f;

// Per-CTA mailbox written by the other CTAs of the cluster (push model:
// every CTA stores its aggregate into the mailboxes of its successors, so
// after one cluster barrier each CTA composes from its own shared memory).
// Double-buffered by iteration parity, so one barrier per iteration suffices.
constexpr int kMaxCluster = 16;
struct GruSlot {
  Aff1 agg[kMaxCluster][kChan];  // aggregate of cluster rank r (r < own rank)
  float cmax[kMaxCluster];       // max|r| of every rank
  float dinc[kChan];             // incoming delta of the cluster chunk
  float plast[kChan];            // last state (pre-update) of CTA rank-1
  float clast[kChan];            // last state (pre-update) of the previous cluster chunk
  int upok;                      // upstream cluster chunks all below tol
  int timeout;                   // the look-back gave up
  int haveclast;                 // clast is valid this iteration
};

struct GruShared {
  float2 agg[kGruNW][kChan];   // warp aggregates, then exclusive warp prefixes
  float din[kGruNW][kChan];    // incoming delta of each warp's sub-chunk
  float hlo[kGruNW][kChan];    // each warp's last state before the update
  float bnd[kGruNW][kChan];    // each warp's boundary state for the next iteration
  float chmax[kGruNW][kChan];  // per (warp, channel) max|r|
  float wmax[kGruNW];
  GruSlot slot[2];
  int ctl[4];
  uint64_t bar;
};

// One pass of cell evaluation (+ Jacobian and local scan when kFull) over the
// thread's 32 steps.  Returns the lane's max|r|.
template <bool kFull>
__device__ __forceinline__ float gru_pass(const unsigned char* __restrict__ rows, int lane,
                                          float hp, float (&h)[kGruL], float (&P)[kGruL],
                                          float az, float ar, float ac, float az2, float ar2,
                                          float ac2, float& dl_out, float& P_out) {
  float m = 0.f, dl = 0.f, Pacc = 1.f;
#pragma unroll
  for (int i = 0; i < kGruL; ++i) {
    const float2 zr = reinterpret_cast<const float2*>(rows + i * kGruRow)[lane];
    const float uc = reinterpret_cast<const float*>(rows + i * kGruRow + 256)[lane];
    const float ht = h[i];
    // z = 1/(1+ez), r = 1/(1+er) share one reciprocal; arguments are clamped
    // so that (1+ez)(1+er) stays finite (sigmoid below 2^-63 reads as 2^-63).
    const float ez = ex2(fmin_nan(fmaf(az2, hp, zr.x), 63.f));
    const float er = ex2(fmin_nan(fmaf(ar2, hp, zr.y), 63.f));
    const float pz = 1.f + ez, pr = 1.f + er;
    const float inv = rcp(pz * pr);
    const float z = pr * inv;
    const float r = pz * inv;
    const float rh = r * hp;
    const float ec = ex2(fmaf(ac2, rh, uc));        // e^{2 y}
    const float c = fmaf(-2.f, rcp(1.f + ec), 1.f);  // tanh(y)
    const float cmh = c - hp;
    const float f = fmaf(z, cmh, hp);                // (1-z) h + z c
    const float res = ht - f;
    m = fmax_nan(m, fabsf(res));
    if (kFull) {
      // A = (1-z) + a_z z(1-z)(c-h) + a_c z(1-c^2)(r + a_r h r(1-r))
      const float omz = 1.f - z;
      const float zz = z * omz;
      const float omc2 = fmaf(-c, c, 1.f);
      const float rr = fmaf(-r, r, r);
      const float q = fmaf(ar * hp, rr, r);
      const float s = (z * omc2) * ac;
      float A = fmaf(az * zz, cmh, omz);
      A = fmaf(s, q, A);
      const float hn = fmaf(A, dl, f);  // h'_t = f_t + A_t ds_{t-1}
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

namespace cg = cooperative_groups;

template <bool kBF16>
__global__ void __launch_bounds__(kGruThreads, 2)
    gru_newton_fused(const __grid_constant__ CUtensorMap tmap, const FwdParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  __shared__ GruShared sh;
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CL = p.CL;
  const int rank = (CL > 1) ? (int)cluster.block_rank() : 0;
  const bool multi = p.nCC > 1;  // cross-cluster look-back needed

  if (tid == 0) {
    // cluster chunks take tickets in order (only rank 0 draws; only needed
    // when a tile spans several cluster chunks)
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
  const int ticket = sh.ctl[0];  // cluster-chunk ticket: tile * nCC + jc
  const unsigned epoch = (unsigned)sh.ctl[1];
  const int tile = ticket / p.nCC, jc = ticket - tile * p.nCC;
  const int j = jc * CL + rank;  // chunk index in the tile
  const int b = tile / p.nDT, d0 = (tile - b * p.nDT) * kChan;
  const int t0 = j * kGruTC;
  const int d = d0 + lane;
  const bool dval = d < p.D;
  constexpr unsigned kBytes = kGruTC * 3 * kChan * (kBF16 ? 2 : 4);
  unsigned char* raw = dyn + (kBF16 ? kGruSmemU / 2 : 0);

  if (tid == 0) {
    mbar_arrive_expect_tx(&sh.bar, kBytes);
    tma_load_4d(raw, &tmap, &sh.bar, d0, 0, t0, b);
  }
  // per-channel constants (overlap the load)
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
  float hbnd = (j == 0 && p.h0 != nullptr && dval) ? p.h0[(size_t)b * p.D + d] : 0.f;

  int status = 0;
  if (!mbar_wait_bounded(&sh.bar, 0, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;

  // ---- rewrite u as pre-scaled fp32 rows: zr = -log2e (u_{z,r} + b), c = 2 log2e (u_c + b)
  if constexpr (kBF16) {
    // raw [t][g][32] bf16 sits in the upper half; convert 32-step blocks in
    // increasing t so no write lands on a row not yet read.
    const __nv_bfloat16* rb = reinterpret_cast<const __nv_bfloat16*>(raw);
#pragma unroll 1
    for (int blk = 0; blk < kGruTC / 32; ++blk) {
      float v[4][3];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = blk * 32 + warp * 4 + q;
#pragma unroll
        for (int g = 0; g < 3; ++g) v[q][g] = __bfloat162float(rb[(t * 3 + g) * kChan + lane]);
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = blk * 32 + warp * 4 + q;
        reinterpret_cast<float2*>(dyn + t * kGruRow)[lane] =
            make_float2(t0 + t < p.T ? -kLog2e * (v[q][0] + bz) : kPadZ, -kLog2e * (v[q][1] + br));
        reinterpret_cast<float*>(dyn + t * kGruRow + 256)[lane] = 2.f * kLog2e * (v[q][2] + bc);
      }
      __syncthreads();
    }
  } else {
    // raw [t][g][32] fp32 occupies exactly the rows it becomes; each warp
    // converts its own 32 rows in place.
#pragma unroll 4
    for (int q = 0; q < kGruL; ++q) {
      const int t = warp * kGruL + q;
      const float* rf = reinterpret_cast<const float*>(dyn + t * kGruRow);
      const float vz = rf[lane], vr = rf[kChan + lane], vc = rf[2 * kChan + lane];
      __syncwarp();
      reinterpret_cast<float2*>(dyn + t * kGruRow)[lane] =
          make_float2(t0 + t < p.T ? -kLog2e * (vz + bz) : kPadZ, -kLog2e * (vr + br));
      reinterpret_cast<float*>(dyn + t * kGruRow + 256)[lane] = 2.f * kLog2e * (vc + bc);
      __syncwarp();
    }
    __syncthreads();
  }

  float h[kGruL], P[kGruL];
#pragma unroll
  for (int i = 0; i < kGruL; ++i) {
    h[i] = 0.f;
    P[i] = 1.f;
  }
  const int tw0 = warp * kGruL;
  const int nvalid = min(kGruL, p.T - (t0 + tw0));
  const unsigned char* rows = dyn + tw0 * kGruRow;
  const int rec_stride = p.max_iters + 1;
  const int ticket0 = ticket - jc;  // ticket of cluster chunk 0 of this tile
  const bool publisher = multi && rank == CL - 1 && jc < p.nCC - 1 &&
                         !((p.flags & PARARNN_FLAG_INJECT_WITHHOLD) && ticket == p.inject_chunk);

  bool frozen = (jc == 0);  // upstream cluster chunks fixed
  int last_bad = -1;        // warp 0: last evaluation whose channel max|r| >= tol
  float final_m = 0.f;
  int updates = 0, k = 0;
  // h_{t-1} before this warp's first step (warp 0: the CTA boundary).  Each
  // iteration it is re-anchored to the owner's last state before the update
  // plus this iteration's incoming delta, so it tracks the stored state to
  // within one update's rounding; the previous warp's / CTA's / cluster
  // chunk's pre-update last state travels with the aggregates.
  float hb = (warp == 0) ? hbnd : 0.f;

  for (;; ++k) {
    const bool cap = (k >= p.max_iters);
    const int par = k & 1;
    sh.hlo[warp][lane] = h[kGruL - 1];
    float dl, Pw, m;
    if (cap)
      m = gru_pass<false>(rows, lane, hb, h, P, az, ar, ac, az2, ar2, ac2, dl, Pw);
    else
      m = gru_pass<true>(rows, lane, hb, h, P, az, ar, ac, az2, ar2, ac2, dl, Pw);
    if (!dval) m = 0.f;
    sh.agg[warp][lane] = make_float2(Pw, dl);
    sh.chmax[warp][lane] = m;
    float wm = m;
#pragma unroll
    for (int o = 16; o; o >>= 1) wm = fmax_nan(wm, __shfl_xor_sync(kFull, wm, o));
    if (lane == 0) sh.wmax[warp] = wm;
    __syncthreads();

    // ---- CTA level: compose the warps' aggregates in order; agg[w] becomes
    // the exclusive prefix of warp w inside the CTA.  Then push the CTA
    // aggregate to the successors in the cluster and the residual to all.
    if (warp == 0) {
      Aff1 cta = Aff1::id();
      float cm = 0.f, chm = 0.f;
#pragma unroll
      for (int w = 0; w < kGruNW; ++w) {
        const float2 ag = sh.agg[w][lane];
        sh.agg[w][lane] = make_float2(cta.P, cta.d);
        cta = Aff1{ag.x, ag.y}.after(cta);
        cm = fmax_nan(cm, sh.wmax[w]);
        chm = fmax_nan(chm, sh.chmax[w][lane]);
      }
      if (dval && !(chm < p.tol)) last_bad = k;
      sh.slot[par].agg[rank][lane] = cta;
      if (lane == 0) sh.slot[par].cmax[rank] = cm;
      for (int r = 0; r < CL; ++r) {
        if (r == rank) continue;
        GruSlot* peer = cluster.map_shared_rank(&sh.slot[par], r);
        if (r > rank) peer->agg[rank][lane] = cta;
        if (r == rank + 1) peer->plast[lane] = sh.hlo[kGruNW - 1][lane];
        if (lane == 0) peer->cmax[rank] = cm;
      }
    }
    if (CL > 1) cluster.sync();
    else __syncthreads();
    Aff1 ex = Aff1::id();
    float clmax = 0.f;
    if (warp == 0) {
      const GruSlot& sl = sh.slot[par];
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        if (r < rank) ex = sl.agg[r][lane].after(ex);
        if (r < CL) clmax = fmax_nan(clmax, sl.cmax[r]);
      }
      final_m = clmax;
      // ---- across cluster chunks: the last CTA of the cluster publishes,
      // looks back and pushes the result to every CTA of the cluster
      if (multi && rank == CL - 1 && !cap) {
        const bool own_ok = clmax < p.tol;
        const Aff1 clus = sl.agg[rank][lane].after(ex);
        const size_t rec = (size_t)ticket * rec_stride + k;
        float* rv = p.rec_vals + rec * (size_t)(kChan * 4);
        float dinc = 0.f, clast = 0.f;
        bool up_ok = true, to = false, have = false;
        if (publisher) rec_put_last(rv, lane, sh.hlo[kGruNW - 1][lane]);
        if (!frozen) {
          if (publisher) {
            rec_put_agg(rv, lane, clus);
            publish_flag(&p.rec_flags[rec], make_flag(epoch, kRecAgg, own_ok));
          }
          if (lookback<Aff1, float>(p.rec_flags, p.rec_vals, ticket0, jc, k, rec_stride, epoch,
                                    p.timeout_ns, dinc, up_ok, &clast)) {
            have = true;
          } else {
            dinc = 0.f;
            up_ok = true;
            to = true;
          }
        }
        if (publisher) {
          rec_put_incl(rv, lane, clus.apply(dinc));
          publish_flag(&p.rec_flags[rec], make_flag(epoch, kRecIncl, up_ok && own_ok));
        }
        for (int r = 0; r < CL; ++r) {
          GruSlot* peer = (r == rank) ? &sh.slot[par] : cluster.map_shared_rank(&sh.slot[par], r);
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
        float dinc = 0.f;
        bool up_ok = true;
        float base = hb;  // this CTA's boundary before the update
        if (multi) {
          dinc = sh.slot[par].dinc[lane];
          up_ok = sh.slot[par].upok != 0;
          if (sh.slot[par].timeout) status = PARARNN_STATUS_TIMEOUT;
          if (rank == 0 && sh.slot[par].haveclast) base = sh.slot[par].clast[lane];
        }
        if (rank > 0) base = sh.slot[par].plast[lane];
        if (up_ok) frozen = true;
        const float din = ex.apply(dinc);  // incoming delta of this CTA
        stop = (up_ok && own_ok) ? 1 : 0;
        updates = k + 1;
#pragma unroll
        for (int w = 0; w < kGruNW; ++w) {
          const float2 e = sh.agg[w][lane];
          const float dw = fmaf(e.x, din, e.y);
          sh.din[w][lane] = dw;
          sh.bnd[w][lane] = (w == 0 ? base : sh.hlo[w - 1][lane]) + dw;
        }
      }
      if (lane == 0) sh.ctl[2] = stop;
    }
    __syncthreads();
    if (!cap) {
      const float din = sh.din[warp][lane];
      hb = sh.bnd[warp][lane];
#pragma unroll
      for (int i = 0; i < kGruL; ++i) h[i] = fmaf(P[i], din, h[i]);
    }
    if (sh.ctl[2]) break;
  }
  // no CTA may leave while a cluster peer can still read its slots
  if (CL > 1) cluster.sync();

  // ---- write the states once
  bool bad = false;
  if (dval) {
    float* out = p.h + ((size_t)b * p.T + t0 + tw0) * p.D + d;
#pragma unroll
    for (int i = 0; i < kGruL; ++i) {
      if (i < nvalid) {
        out[(size_t)i * p.D] = h[i];
        bad |= !isfinite(h[i]);
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
static int launch_gru_t(const CUtensorMap& tmap, const FwdParams& p, int nctas,
                        cudaStream_t stream) {
  const size_t smem = kGruSmemU;
  auto kern = gru_newton_fused<kBF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  if (p.CL > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return (int)e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kGruThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmap, p);
  return (int)e;
}

int launch_gru_fwd(const CUtensorMap& tmap, bool bf16, const FwdParams& p, int nctas,
                   cudaStream_t stream) {
  return bf16 ? launch_gru_t<true>(tmap, p, nctas, stream)
              : launch_gru_t<false>(tmap, p, nctas, stream);
}

// Largest cluster size (16 or 8, or smaller) that can be resident for this
// kernel; 0 if the query fails.
int gru_max_cluster(bool bf16) {
  int best = 0;
  for (int cl : {16, 8, 4, 2, 1}) {
    auto kern = bf16 ? gru_newton_fused<true> : gru_newton_fused<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGruSmemU) !=
        cudaSuccess)
      return 0;
    if (cl > 8 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl * 64);
    cfg.blockDim = dim3(kGruThreads);
    cfg.dynamicSmemBytes = kGruSmemU;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) {
      best = cl;
      break;
    }
    cudaGetLastError();
  }
  return best;
}

int gru_chunk_steps() { return kGruTC; }

}  // namespace pararnn
