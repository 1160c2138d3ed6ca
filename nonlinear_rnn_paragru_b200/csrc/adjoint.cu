// adjoint.cu -- reverse (adjoint) scan of a solved ParaGRU / ParaLSTM
// trajectory.
//
// With the converged states the loss gradient flows back through the same
// block-bidiagonal structure ("Параллельность RNN?", §1.3), transposed:
//   lambda_{T} = g_T,  lambda_t = g_t + A_{t+1}^T lambda_{t+1},
// a linear recurrence run backwards in time, i.e. a reverse scan of affine
// maps.  From lambda: du_t = (df_t/du_t)^T lambda_t, da = sum (df_t/da)^T
// lambda_t, dbias = sum du_t, d(s_0) = A_1^T lambda_1.
//
// One CTA handles 32 channels x kTC steps; thread (warp w, lane l) handles
// channel l over a contiguous range of L steps.
//   pass 1 (reverse over the range): evaluate the Jacobians and compose the
//     range's affine map carry_in -> carry_out, where carry = A_s^T lambda_s
//     is what step s hands to step s-1;
//   scan: compose the maps across the 8 warps (shared memory) and across the
//     CTAs of the sequence by decoupled look-back from its end (one record
//     per chunk; chunks take tickets from the last one backwards);
//   pass 2 (reverse): re-evaluate the cell, run the exact recurrence from the
//     true incoming carry, write du and accumulate da / dbias partials.
// u, the states and dL/dh of the chunk arrive by TMA bulk-tensor loads into
// shared memory (one mbarrier), so both passes read on-chip data.  Per-CTA
// partial sums of da and dbias are reduced by a second kernel in a fixed
// order (reproducible).
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

constexpr int kAdjNW = 8;
constexpr int kAdjThreads = kAdjNW * 32;

// -------------------------------------------------------------- cells --
__device__ __forceinline__ float sigm(float x) { return rcp(1.f + ex2(-kLog2e * x)); }
__device__ __forceinline__ float tanhx(float x) {
  return fmaf(-2.f, rcp(1.f + ex2(2.f * kLog2e * x)), 1.f);
}

struct GruCell {
  static constexpr int G = 3;
  static constexpr int L = 16;
  static constexpr int kMinBlocks = 3;
  using E = Aff1;
  using V = float;
  struct S {  // state s_{t-1}
    float h;
  };
  struct K {
    float a[3], b[3];
  };
  __device__ static V zero() { return 0.f; }
  // Jacobian df/ds at (s_prev, u); optionally the gradient pieces.
  template <bool kGrad>
  __device__ static void eval(const S& s, const float (&u)[4], const K& k, float& A, float* du_c,
                              float* da_c) {
    const float hp = s.h;
    const float z = sigm(fmaf(k.a[0], hp, u[0] + k.b[0]));
    const float r = sigm(fmaf(k.a[1], hp, u[1] + k.b[1]));
    const float rh = r * hp;
    const float c = tanhx(fmaf(k.a[2], rh, u[2] + k.b[2]));
    const float zz = fmaf(-z, z, z), rr = fmaf(-r, r, r), cc = fmaf(-c, c, 1.f);
    const float gz = (c - hp) * zz;    // df/dpre_z
    const float gc = z * cc;           // df/dpre_c
    const float gr = gc * k.a[2] * hp * rr;  // df/dpre_r
    A = (1.f - z) + gz * k.a[0] + gc * k.a[2] * fmaf(hp * rr, k.a[1], r);
    if (kGrad) {
      du_c[0] = gz;
      du_c[1] = gr;
      du_c[2] = gc;
      da_c[0] = hp;
      da_c[1] = hp;
      da_c[2] = rh;
    }
  }
};

struct LstmCell {
  static constexpr int G = 4;
  static constexpr int L = 8;
  static constexpr int kMinBlocks = 2;
  using E = Aff2;
  using V = float2;  // (lambda_c, lambda_h)
  struct S {
    float c, h;
  };
  struct K {
    float a[4], b[4];
  };
  __device__ static V zero() { return make_float2(0.f, 0.f); }
  // A = d(c', h')/d(c, h) at (s_prev, u) stored as A[0..3] = a00 a01 a10 a11.
  // du_c[q]: the adjoint contribution per gate is du_q = du_c[q] . (lc, lh),
  // stored as pairs; da_c = pre-activation derivative w.r.t. a_q (= h_prev).
  template <bool kGrad>
  __device__ static void eval(const S& s, const float (&u)[4], const K& k, float (&A)[4],
                              float* du_c, float* da_c) {
    const float cp = s.c, hp = s.h;
    const float i = sigm(fmaf(k.a[0], hp, u[0] + k.b[0]));
    const float f = sigm(fmaf(k.a[1], hp, u[1] + k.b[1]));
    const float g = tanhx(fmaf(k.a[2], hp, u[2] + k.b[2]));
    const float o = sigm(fmaf(k.a[3], hp, u[3] + k.b[3]));
    const float cn = fmaf(f, cp, i * g);
    const float tc = tanhx(cn);
    const float di = fmaf(-i, i, i), df = fmaf(-f, f, f), dg = fmaf(-g, g, 1.f),
                dox = fmaf(-o, o, o), dtc = fmaf(-tc, tc, 1.f);
    const float gci = g * di, gcf = cp * df, gcg = i * dg;  // dc'/dpre_{i,f,g}
    const float kk = o * dtc;                               // dh'/dc'
    const float X = fmaf(gcf, k.a[1], fmaf(gci, k.a[0], gcg * k.a[2]));
    A[0] = f;
    A[1] = X;
    A[2] = kk * f;
    A[3] = fmaf(dox * tc, k.a[3], kk * X);
    if (kGrad) {
      // du_q = dc'/dpre_q * lc + dh'/dpre_q * lh
      du_c[0] = gci; du_c[1] = kk * gci;
      du_c[2] = gcf; du_c[3] = kk * gcf;
      du_c[4] = gcg; du_c[5] = kk * gcg;
      du_c[6] = 0.f; du_c[7] = dox * tc;
      da_c[0] = hp;
    }
  }
};

// the carry map of one step, transposed: x -> A^T x
__device__ __forceinline__ Aff1 mat_only(float A) { return Aff1{A, 0.f}; }
__device__ __forceinline__ Aff2 mat_only(const float (&A)[4]) {
  return Aff2{A[0], A[2], A[1], A[3], 0.f, 0.f};
}

struct AdjParams {
  const void* u;
  const float *a, *bias, *c0, *h0, *c, *h, *dLdh;
  float *du, *da, *dbias, *dc0, *dh0;
  int B, T, D, nDT, nC;
  uint64_t timeout_ns;
  int inject_chunk;  // testing: the chunk with this ticket publishes no records (-1: none)
  WsHeader* hdr;
  unsigned* rec_flags;
  float* rec_vals;
  float* part;  // [nchunks][2G][32]
  int* status;
};

// State before the chunk (global), and states inside it (shared memory).
template <class Cell>
__device__ __forceinline__ typename Cell::S boundary_state(const AdjParams& p, int b, int t0,
                                                           int d, bool dval);
template <>
__device__ __forceinline__ GruCell::S boundary_state<GruCell>(const AdjParams& p, int b, int t0,
                                                              int d, bool dval) {
  if (!dval) return {0.f};
  if (t0 == 0) return {p.h0 ? p.h0[(size_t)b * p.D + d] : 0.f};
  return {p.h[((size_t)b * p.T + t0 - 1) * p.D + d]};
}
template <>
__device__ __forceinline__ LstmCell::S boundary_state<LstmCell>(const AdjParams& p, int b, int t0,
                                                                int d, bool dval) {
  if (!dval) return {0.f, 0.f};
  if (t0 == 0)
    return {p.c0 ? p.c0[(size_t)b * p.D + d] : 0.f, p.h0 ? p.h0[(size_t)b * p.D + d] : 0.f};
  const size_t i = ((size_t)b * p.T + t0 - 1) * p.D + d;
  return {p.c[i], p.h[i]};
}
template <class Cell>
__device__ __forceinline__ typename Cell::S tile_state(const float* hs, const float* cs, int s,
                                                       int lane);
template <>
__device__ __forceinline__ GruCell::S tile_state<GruCell>(const float* hs, const float*, int s,
                                                          int lane) {
  return {hs[s * kChan + lane]};
}
template <>
__device__ __forceinline__ LstmCell::S tile_state<LstmCell>(const float* hs, const float* cs,
                                                            int s, int lane) {
  return {cs[s * kChan + lane], hs[s * kChan + lane]};
}

template <class Cell, bool kBF16>
__device__ __forceinline__ void load_u(const unsigned char* tile, int s, int lane, float (&u)[4]) {
#pragma unroll
  for (int q = 0; q < Cell::G; ++q) {
    if constexpr (kBF16)
      u[q] = __bfloat162float(
          reinterpret_cast<const __nv_bfloat16*>(tile)[(s * Cell::G + q) * kChan + lane]);
    else
      u[q] = reinterpret_cast<const float*>(tile)[(s * Cell::G + q) * kChan + lane];
  }
  if (Cell::G == 3) u[3] = 0.f;
}

// Shared-memory tiles of one chunk: u [TC][G][32] (bf16 or fp32), then the
// fp32 tiles h [TC][32], c [TC][32] (ParaLSTM) and dL/dh [TC][32].
template <class Cell, bool kBF16>
struct AdjTiles {
  static constexpr int TC = kAdjNW * Cell::L;
  static constexpr int kU = TC * Cell::G * kChan * (kBF16 ? 2 : 4);
  static constexpr int kS = TC * kChan * 4;
  static constexpr int kNS = (Cell::G == 4) ? 3 : 2;  // state/grad tiles
  static constexpr int kBytes = kU + kNS * kS;
};

template <class Cell, bool kBF16>
__global__ void __launch_bounds__(kAdjThreads, Cell::kMinBlocks)
    adjoint_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmh,
                   const __grid_constant__ CUtensorMap tmc, const __grid_constant__ CUtensorMap tmg,
                   const AdjParams p) {
  using E = typename Cell::E;
  using V = typename Cell::V;
  using S = typename Cell::S;
  using Tiles = AdjTiles<Cell, kBF16>;
  constexpr int L = Cell::L, G = Cell::G, TC = kAdjNW * L;
  extern __shared__ __align__(1024) unsigned char tile[];
  const float* h_t = reinterpret_cast<const float*>(tile + Tiles::kU);
  const float* g_t = reinterpret_cast<const float*>(tile + Tiles::kU + Tiles::kS);
  const float* c_t = reinterpret_cast<const float*>(tile + Tiles::kU + 2 * Tiles::kS);
  __shared__ E agg[kAdjNW][kChan];
  __shared__ float red[kAdjNW][2 * G][kChan];
  __shared__ int ctl[4];
  __shared__ uint64_t bar;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    ctl[0] = (int)atomicAdd(&p.hdr->ticket, 1u);
    ctl[1] = (int)(*(volatile unsigned*)&p.hdr->epoch);
    ctl[3] = 0;  // CTA status
    mbar_init(&bar, 1);
  }
  __syncthreads();
  const int ticket = ctl[0];
  const unsigned epoch = (unsigned)ctl[1];
  const int tl = ticket / p.nC, v = ticket - tl * p.nC;  // v-th chunk from the end
  const int j = p.nC - 1 - v;
  const int b = tl / p.nDT, d0 = (tl - b * p.nDT) * kChan;
  const int t0 = j * TC;
  const int d = d0 + lane;
  const bool dval = d < p.D;
  if (tid == 0) {
    mbar_arrive_expect_tx(&bar, (unsigned)Tiles::kBytes);
    tma_load_4d(tile, &tmap, &bar, d0, 0, t0, b);
    tma_load_3d(tile + Tiles::kU, &tmh, &bar, d0, t0, b);
    tma_load_3d(tile + Tiles::kU + Tiles::kS, &tmg, &bar, d0, t0, b);
    if (G == 4) tma_load_3d(tile + Tiles::kU + 2 * Tiles::kS, &tmc, &bar, d0, t0, b);
  }
  // the state before this thread's first step
  const S s_before_chunk = boundary_state<Cell>(p, b, t0, d, dval);
  typename Cell::K K;
#pragma unroll
  for (int q = 0; q < G; ++q) {
    K.a[q] = dval ? p.a[q * p.D + d] : 0.f;
    K.b[q] = (dval && p.bias) ? p.bias[q * p.D + d] : 0.f;
  }
  int status = 0;
  if (!mbar_wait_bounded(&bar, 0, p.timeout_ns)) status = PARARNN_STATUS_TIMEOUT;

  const int a0 = warp * L;             // first local step of this thread
  const int nvalid = min(L, p.T - (t0 + a0));
  // dL/dh and states past the end of the sequence arrive as zeros (TMA fill)
  auto gval = [&](int s) -> float { return g_t[(a0 + s) * kChan + lane]; };
  auto state_at = [&](int s) -> S {   // state after local step s of this thread
    return (a0 + s < 0) ? s_before_chunk : tile_state<Cell>(h_t, c_t, a0 + s, lane);
  };

  // ---- pass 1: compose this range's carry map (reverse).  accm maps the
  // incoming carry (A^T lambda handed down by the step after the range) to
  // the carry leaving the current step.
  E accm = E::id();
  {
#pragma unroll 4
    for (int s = L - 1; s >= 0; --s) {
      float u[4];
      load_u<Cell, kBF16>(tile, a0 + s, lane, u);
      const S sp = state_at(s - 1);
      if constexpr (G == 3) {
        float A;
        Cell::template eval<false>(sp, u, K, A, nullptr, nullptr);
        accm = Aff1{1.f, gval(s)}.after(accm);  // lambda_s = g_s + carry
        accm = mat_only(A).after(accm);         // carry out = A_s^T lambda_s
      } else {
        float A[4];
        Cell::template eval<false>(sp, u, K, A, nullptr, nullptr);
        accm = Aff2{1.f, 0.f, 0.f, 1.f, 0.f, gval(s)}.after(accm);
        accm = mat_only(A).after(accm);
      }
    }
  }
  agg[warp][lane] = accm;  // carry into this range -> carry out of its first step
  __syncthreads();

  // ---- CTA: exclusive (reverse) prefixes per warp, then the chunk's map
  if (warp == 0) {
    E cur = E::id();  // maps CTA incoming carry -> carry into warp w
    for (int w = kAdjNW - 1; w >= 0; --w) {
      const E e = agg[w][lane];
      agg[w][lane] = cur;
      cur = e.after(cur);
    }
    // cross-chunk: records indexed by (tile, v); v increases in processing order
    V kin = Cell::zero();
    const int stride = 1;
    const size_t rec = (size_t)ticket;
    float* rv = p.rec_vals + rec * (size_t)(kChan * rec_floats<E>());
    const bool publish = ticket != p.inject_chunk;
    if (v > 0) {
      rec_put_agg(rv, lane, cur);
      if (publish) publish_flag(&p.rec_flags[rec], make_flag(epoch, kRecAgg, true));
      bool ok;
      if (!lookback<E, V>(p.rec_flags, p.rec_vals, ticket - v, v, 0, stride, epoch, p.timeout_ns,
                          kin, ok)) {
        kin = Cell::zero();
        status = PARARNN_STATUS_TIMEOUT;
      }
    }
    rec_put_incl(rv, lane, cur.apply(kin));
    if (publish) publish_flag(&p.rec_flags[rec], make_flag(epoch, kRecIncl, true));
    if (status) atomicMax(&ctl[3], status);
    // the incoming carry of every warp, as a constant map
    for (int w = 0; w < kAdjNW; ++w) {
      const V kw = agg[w][lane].apply(kin);
      if constexpr (G == 3)
        agg[w][lane] = Aff1{0.f, kw};
      else
        agg[w][lane] = Aff2{0.f, 0.f, 0.f, 0.f, kw.x, kw.y};
    }
  }
  __syncthreads();
  V carry = agg[warp][lane].apply(Cell::zero());

  // ---- pass 2: exact reverse recurrence, du and da / dbias partials
  float sa[G], sb[G];
#pragma unroll
  for (int q = 0; q < G; ++q) sa[q] = sb[q] = 0.f;
  bool bad = false;
  {
#pragma unroll 2
    for (int s = L - 1; s >= 0; --s) {
      float u[4];
      load_u<Cell, kBF16>(tile, a0 + s, lane, u);
      const S sp = state_at(s - 1);
      const float gs = gval(s);
      float du_c[8], da_c[3];
      float out[4];
      if constexpr (G == 3) {
        float A;
        Cell::template eval<true>(sp, u, K, A, du_c, da_c);
        const float lam = gs + carry;
#pragma unroll
        for (int q = 0; q < 3; ++q) {
          out[q] = du_c[q] * lam;
          sa[q] = fmaf(out[q], da_c[q], sa[q]);
          sb[q] += out[q];
        }
        carry = A * lam;
      } else {
        float A[4];
        Cell::template eval<true>(sp, u, K, A, du_c, da_c);
        const float lc = carry.x, lh = gs + carry.y;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          out[q] = fmaf(du_c[2 * q], lc, du_c[2 * q + 1] * lh);
          sa[q] = fmaf(out[q], da_c[0], sa[q]);
          sb[q] += out[q];
        }
        carry = make_float2(fmaf(A[0], lc, A[2] * lh), fmaf(A[1], lc, A[3] * lh));
      }
      if (dval && s < nvalid) {
        float* o = p.du + (((size_t)b * p.T + t0 + a0 + s) * G) * p.D + d;
#pragma unroll
        for (int q = 0; q < G; ++q) {
          o[(size_t)q * p.D] = out[q];
          bad |= !isfinite(out[q]);
        }
      }
    }
  }
  // d L / d s_0: the carry out of the first step of the sequence
  if (j == 0 && warp == 0 && dval) {
    if constexpr (G == 3) {
      if (p.dh0) p.dh0[(size_t)b * p.D + d] = carry;
    } else {
      if (p.dc0) p.dc0[(size_t)b * p.D + d] = carry.x;
      if (p.dh0) p.dh0[(size_t)b * p.D + d] = carry.y;
    }
  }
  // ---- partial sums: fixed-order reduction over the warps
#pragma unroll
  for (int q = 0; q < G; ++q) {
    red[warp][q][lane] = dval ? sa[q] : 0.f;
    red[warp][G + q][lane] = dval ? sb[q] : 0.f;
  }
  __syncthreads();
  for (int q = warp; q < 2 * G; q += kAdjNW) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kAdjNW; ++w) acc += red[w][q][lane];
    p.part[((size_t)ticket * 2 * G + q) * kChan + lane] = acc;
  }
  if (bad) atomicMax(&ctl[3], PARARNN_STATUS_NONFINITE);
  if (status) atomicMax(&ctl[3], status);
  __syncthreads();
  if (tid == 0 && ctl[3]) atomicMax(p.status, ctl[3]);
}

// da[q][d] = sum over (b, chunk) of the per-CTA partials, in a fixed order:
// block (q, channel tile), warp w sums chunks w, w + 8, ... of every batch
// row in order, then the 8 warp sums are added in warp order.
__global__ void adjoint_reduce(const float* __restrict__ part, float* da, float* dbias, int B,
                               int D, int nDT, int nC, int G) {
  __shared__ float ws[kAdjNW][kChan];
  const int q = blockIdx.x / nDT, dt = blockIdx.x - q * nDT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc = 0.f;
  for (int b = 0; b < B; ++b) {
    const size_t tl = (size_t)b * nDT + dt;
    for (int v = warp; v < nC; v += kAdjNW)
      acc += part[(((tl * nC + v) * 2 * G) + q) * kChan + lane];
  }
  ws[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kAdjNW; ++w) t += ws[w][lane];
    const int d = dt * kChan + lane;
    if (d < D) {
      if (q < G)
        da[q * D + d] = t;
      else if (dbias)
        dbias[(q - G) * D + d] = t;
    }
  }
}

// New epoch, ticket counter and status; and the look-back flags cleared, so
// no flag another call left in the workspace can pass for one of this call.
__global__ void adjoint_init(WsHeader* hdr, int* status, unsigned* flags, size_t nflags) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    unsigned e = (hdr->epoch + 1u) & 0x1fffffffu;
    if (e == 0u) e = 1u;
    hdr->epoch = e;
    hdr->ticket = 0u;
    *status = 0;
  }
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nflags;
       i += (size_t)gridDim.x * blockDim.x)
    flags[i] = 0u;
}

// ---------------------------------------------------------------- host --
int adjoint_chunk_steps(int cell) {
  return kAdjNW * (cell == PARARNN_GRU ? GruCell::L : LstmCell::L);
}

struct AdjLayout {
  size_t flags, vals, part, total;
};
static AdjLayout adj_layout(int cell, int B, int T, int D) {
  const int tc = adjoint_chunk_steps(cell);
  const int G = cell == PARARNN_GRU ? 3 : 4, RF = cell == PARARNN_GRU ? 4 : 12;
  const size_t nch = (size_t)B * ((D + kChan - 1) / kChan) * ((T + tc - 1) / tc);
  AdjLayout L;
  L.flags = kWsHeaderBytes;
  L.vals = L.flags + align256(nch * 4);
  L.part = L.vals + align256(nch * kChan * RF * 4);
  L.total = L.part + align256(nch * 2 * G * kChan * 4);
  return L;
}

size_t adjoint_ws_bytes(int cell, int B, int T, int D) { return adj_layout(cell, B, T, D).total; }

template <class Cell, bool kBF16>
static int launch_adj_t(const CUtensorMap* maps, const AdjParams& p, int nch,
                        cudaStream_t stream) {
  const int smem = AdjTiles<Cell, kBF16>::kBytes;
  auto kern = adjoint_kernel<Cell, kBF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return (int)e;
  kern<<<nch, kAdjThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], p);
  return (int)cudaGetLastError();
}

int launch_adjoint(int cell, bool bf16, const CUtensorMap* maps, const void* u, const float* a,
                   const float* bias, const float* c0, const float* h0, const float* c,
                   const float* h, const float* dLdh, float* du, float* da, float* dbias,
                   float* dc0, float* dh0, int B, int T, int D, int* status, void* ws,
                   uint64_t timeout_ns, int inject_chunk, cudaStream_t stream) {
  const int tc = adjoint_chunk_steps(cell);
  const int G = cell == PARARNN_GRU ? 3 : 4;
  const AdjLayout Lw = adj_layout(cell, B, T, D);
  unsigned char* w = static_cast<unsigned char*>(ws);
  AdjParams p;
  p.u = u;
  p.a = a;
  p.bias = bias;
  p.c0 = c0;
  p.h0 = h0;
  p.c = c;
  p.h = h;
  p.dLdh = dLdh;
  p.du = du;
  p.da = da;
  p.dbias = dbias;
  p.dc0 = dc0;
  p.dh0 = dh0;
  p.B = B;
  p.T = T;
  p.D = D;
  p.nDT = (D + kChan - 1) / kChan;
  p.nC = (T + tc - 1) / tc;
  p.timeout_ns = timeout_ns;
  p.inject_chunk = inject_chunk;
  p.hdr = reinterpret_cast<WsHeader*>(w);
  p.rec_flags = reinterpret_cast<unsigned*>(w + Lw.flags);
  p.rec_vals = reinterpret_cast<float*>(w + Lw.vals);
  p.part = reinterpret_cast<float*>(w + Lw.part);
  p.status = status;
  const long long nch = (long long)B * p.nDT * p.nC;
  if (nch >= (1LL << 31)) return 1;
  adjoint_init<<<(unsigned)std::min<long long>((nch + 255) / 256, 256), 256, 0, stream>>>(
      p.hdr, status, p.rec_flags, (size_t)nch);
  if (cudaGetLastError() != cudaSuccess) return 1;
  int e;
  if (cell == PARARNN_GRU)
    e = bf16 ? launch_adj_t<GruCell, true>(maps, p, (int)nch, stream)
             : launch_adj_t<GruCell, false>(maps, p, (int)nch, stream);
  else
    e = bf16 ? launch_adj_t<LstmCell, true>(maps, p, (int)nch, stream)
             : launch_adj_t<LstmCell, false>(maps, p, (int)nch, stream);
  if (e) return e;
  adjoint_reduce<<<2 * G * p.nDT, kAdjThreads, 0, stream>>>(p.part, da, dbias, B, D, p.nDT, p.nC,
                                                             G);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
