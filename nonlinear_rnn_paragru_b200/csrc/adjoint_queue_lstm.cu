// adjoint_queue_lstm.cu -- reverse (adjoint) scan of a solved ParaLSTM
// trajectory with bf16 input projections for many 8-channel tiles: every
// 256-step segment of every tile in one persistent launch, last segments
// first.
//
// The ParaGRU queue adjoint (adjoint_queue.cu) with the 2x2 Jacobian
// ("Параллельность RNN?", §1.3, transposed): lambda = (lambda_c, lambda_h),
// the loss gradient enters through lambda_h, carry_t = A_t^T lambda_t;
// du_{i,f,g} = (gci, gcf, gcg) (lambda_c + kk lambda_h), du_o = dot lambda_h
// (the cell of adjoint_cell.cuh), da = sum_t du_t h_{t-1}, dbias = sum_t du_t,
// and dL/dc0, dL/dh0 the carry out of the first step.
//
// Items (8 channels of one batch row over one segment) are numbered so that
// every tile's last segment comes first (item = r * ntiles + tile for the
// segment r from the end) and drawn from a counter one ahead.  A CTA of 4
// warps holds a segment (lane = (chunk k = lane / 8, channel c = lane % 8),
// 16 steps per thread as 8 packed step pairs); every warp stages its own four
// chunks and its own copy of the tile's parameter rows on its own mbarrier
// and loads the next item's as soon as its pass 2 is done:
//   pass 1: each chunk's map carry_in -> carry_out (2x2 matrix, 2-vector),
//     backwards;
//   scan: a suffix scan over the warp's four chunks by shuffles, and over the
//     warps from shared memory after one CTA barrier (the only one per item);
//   carry: a segment publishes the carry it passes to the segment before it
//     as two 64-bit words per channel, (lambda_c bits, count) and (lambda_h
//     bits, count), the count being the segments published from the tile's
//     end; each word is single-copy atomic and names its writer, so relaxed
//     loads (issued when the item starts, checked after pass 1, polled with a
//     bound if not there yet) need no fence; the words are written before
//     pass 2, so the chain of segments advances one map application per
//     segment;
//   pass 2: the exact recurrence from the true carry, du written and the
//     da / dbias partial sums kept per warp, summed over the warps in a fixed
//     order after the next item's barrier (reduced over the items afterwards
//     in a fixed order: bitwise reproducible).
// The lowest-numbered item that has not published is always being worked on
// and never waits, so the queue cannot deadlock while all CTAs are resident;
// a wait that runs out sets TIMEOUT.  Four CTAs share an SM (51.2 KB of
// staged chunks each).
#include <cuda_bf16.h>

#include <algorithm>

#include "adjoint_cell.cuh"
#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace {

constexpr unsigned kAlqFull = 0xffffffffu;
constexpr int kAlqWarps = 4;
constexpr int kAlqThreads = kAlqWarps * 32;
constexpr int kAlqChunks = kAlqWarps * kArK;       // 16
constexpr int kAlqSteps = kAlqChunks * kArL;       // 256 steps per item
constexpr int kAlqSmem = kAlqChunks * kAlS;        // 51200
constexpr unsigned kAlqWarpBytes =
    kArK * (kArUBox * kAlUStep + 2 * kArHBox * kArSStep + kArGBox * kArSStep);

struct AlqParams {
  const float *a, *bias, *c0, *h0;
  float *du, *dc0, *dh0, *part;
  // [ntiles][8][2]: the carry (lambda_c, lambda_h) a segment passes to the
  // one before it, each as (float bits) | (segments published from the end) << 32
  unsigned long long* carry;
  unsigned* counter;   // item tickets (zero at launch)
  int B, T, D, nDTc, ntiles, nseg, nitems;
  uint64_t timeout_ns;
  int* status;
  int withhold_item;   // testing: this item never publishes its carry (-1: none)
};

struct AlqShared {
  uint64_t bar[kAlqWarps];            // per warp: its chunks' boxes and parameters
  float par[kAlqWarps][10][kArC];     // per warp: a (4 rows), bias (4 rows), c0, h0
  float4 wagg[2][kAlqWarps][kArC][2]; // by item parity: per (warp, channel) suffix map
  float red[2][kAlqWarps][8][kArC];   // by item parity: partial sums per warp
  float2 cin[2][kArC];                // by item parity: carry entering the last step
  int nx[2];                          // the item after this one, by parity
};

__device__ __forceinline__ void alq_bulk(void* dst, const void* src, unsigned bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ unsigned long long alq_ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void alq_st_word(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long alq_word(float v, int count) {
  return (unsigned long long)__float_as_uint(v) | ((unsigned long long)count << 32);
}
__device__ __forceinline__ Aff2 alq_shfl_down(const Aff2& a, int o) {
  return Aff2{__shfl_down_sync(kAlqFull, a.m00, o), __shfl_down_sync(kAlqFull, a.m01, o),
              __shfl_down_sync(kAlqFull, a.m10, o), __shfl_down_sync(kAlqFull, a.m11, o),
              __shfl_down_sync(kAlqFull, a.d0, o),  __shfl_down_sync(kAlqFull, a.d1, o)};
}

// Warp `warp`: its four chunks' boxes (u, c_{t-1}, h_{t-1}, dL/dh; lane k
// issues chunk k's four), its copy of the a and bias rows and, for a first
// segment, the c0 and h0 rows of the item at (b, d0, t0), all on the warp's
// mbarrier.  The rows are 16-byte aligned (the caller checks the pointers;
// d0 is a multiple of 8 and D of 8).
__device__ __forceinline__ void alq_issue(unsigned char* smem, AlqShared& sh,
                                          const CUtensorMap* mu, const CUtensorMap* mc,
                                          const CUtensorMap* mh, const CUtensorMap* mg,
                                          const AlqParams& p, int warp, int b, int d0, int t0,
                                          int lane) {
  const unsigned pb = kArC * 4;
  const bool first_seg = t0 == 0;
  uint64_t* bar = &sh.bar[warp];
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, kAlqWarpBytes + 4 * pb + (p.bias ? 4 * pb : 0) +
                                   ((first_seg && p.c0) ? pb : 0) +
                                   ((first_seg && p.h0) ? pb : 0));
  }
  __syncwarp();
  if (lane < kArK) {
    const int q = warp * kArK + lane, ts = t0 + q * kArL - lane;
    unsigned char* slot = smem + q * kAlS;
    tma_load_4d(slot + kAlUOff, mu, bar, d0, 0, ts, b);
    tma_load_3d(slot + kAlCOff, mc, bar, d0, ts - 1, b);
    tma_load_3d(slot + kAlHOff, mh, bar, d0, ts - 1, b);
    tma_load_3d(slot + kAlGOff, mg, bar, d0, ts, b);
  } else if (lane < kArK + 4) {
    const int g = lane - kArK;
    alq_bulk(&sh.par[warp][g][0], p.a + (size_t)g * p.D + d0, pb, bar);
    if (p.bias) alq_bulk(&sh.par[warp][4 + g][0], p.bias + (size_t)g * p.D + d0, pb, bar);
  } else if (lane == kArK + 4 && first_seg && p.c0) {
    alq_bulk(&sh.par[warp][8][0], p.c0 + (size_t)b * p.D + d0, pb, bar);
  } else if (lane == kArK + 5 && first_seg && p.h0) {
    alq_bulk(&sh.par[warp][9][0], p.h0 + (size_t)b * p.D + d0, pb, bar);
  }
}

__device__ __forceinline__ int alq_draw(unsigned* counter) {
  return (int)min(atomicAdd(counter, 1u), 0x7fffffffu);
}

__global__ void __launch_bounds__(kAlqThreads, 4)
    adjoint_queue_lstm(const __grid_constant__ CUtensorMap mu,
                       const __grid_constant__ CUtensorMap mc,
                       const __grid_constant__ CUtensorMap mh,
                       const __grid_constant__ CUtensorMap mg, const AlqParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ AlqShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane % kArC, kk = lane / kArC;
  const int q = warp * kArK + kk;

  for (int i = tid; i < kAlqWarps * 10 * kArC; i += kAlqThreads) (&sh.par[0][0][0])[i] = 0.f;
  if (tid < kAlqWarps) mbar_init(&sh.bar[tid], 1);
  if (tid == 0) sh.nx[0] = alq_draw(p.counter);
  __syncthreads();
  int item = sh.nx[0];
  if (item < p.nitems) {
    const int tile = item % p.ntiles, seg = p.nseg - 1 - item / p.ntiles;
    alq_issue(smem, sh, &mu, &mc, &mh, &mg, p, warp, tile / p.nDTc, (tile % p.nDTc) * kArC,
              seg * kAlqSteps, lane);
  }
  const unsigned char* slot = smem + q * kAlS;
  const unsigned char* ubase = slot + kAlUOff + kk * kAlUStep + c * 2;
  const float* cbase = reinterpret_cast<const float*>(slot + kAlCOff + kk * kArSStep) + c;
  const float* hbase = reinterpret_cast<const float*>(slot + kAlHOff + kk * kArSStep) + c;
  const float* gbase = reinterpret_cast<const float*>(slot + kAlGOff + kk * kArSStep) + c;
  const float* pw = &sh.par[warp][0][0] + c;
  int status = 0;
  int n = 0, prev_part = -1;  // prev_part: the partial-sum row of the item before
  // 0 while this warp's boxes arrive, else 1 + the phase parity of the wait
  // that ran out (the warp issues no more loads)
  int dead = 0;
  for (; item < p.nitems; ++n) {
    const int par = n & 1;
    if (tid == 0) sh.nx[par ^ 1] = alq_draw(p.counter);
    const int tile = item % p.ntiles, r = item / p.ntiles, seg = p.nseg - 1 - r;
    const int b = tile / p.nDTc, d0 = (tile % p.nDTc) * kArC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int t0 = seg * kAlqSteps;
    const bool first = (seg == 0 && q == 0);  // the chunk holding step 0
    // the carry words of the segment after this one, fetched now, read after pass 1
    unsigned long long wc = 0ull, wh = 0ull;
    unsigned long long* cwp = &p.carry[((size_t)tile * kArC + c) * 2];
    if (tid < kArC && r > 0) {
      wc = alq_ld_word(cwp);
      wh = alq_ld_word(cwp + 1);
    }
    if (!dead) {
      // a phase that did not complete is never re-armed: the warp stops loading
      if (!__all_sync(kAlqFull, mbar_wait_bounded(&sh.bar[warp], (unsigned)par, p.timeout_ns))) {
        dead = 1 + par;
        status = PARARNN_STATUS_TIMEOUT;
      }
    }
    AlCell k;
    float2 BS[4];
    float c0v, h0v;
    {
      const float ai = pw[0 * kArC], af = pw[1 * kArC], ag = pw[2 * kArC], ao = pw[3 * kArC];
      k.AI = af2(ai, ai);
      k.AF = af2(af, af);
      k.AG = af2(ag, ag);
      k.AO = af2(ao, ao);
      k.AI2 = af2(-kLog2e * ai, -kLog2e * ai);
      k.AF2 = af2(-kLog2e * af, -kLog2e * af);
      k.AG2 = af2(2.f * kLog2e * ag, 2.f * kLog2e * ag);
      k.AO2 = af2(-kLog2e * ao, -kLog2e * ao);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float bs = (g == 2 ? 2.f * kLog2e : -kLog2e) * pw[(4 + g) * kArC];
        BS[g] = af2(bs, bs);
      }
      c0v = (seg == 0) ? pw[8 * kArC] : 0.f;
      h0v = (seg == 0) ? pw[9 * kArC] : 0.f;
    }
    auto state = [&](int i, float2& CP, float2& HP, float2& G) {
      CP = af2(cbase[i * kArC], cbase[(i + kArH) * kArC]);  // (c, h)_{t-1}
      HP = af2(hbase[i * kArC], hbase[(i + kArH) * kArC]);
      if (i == 0 && first) {
        CP.x = c0v;
        HP.x = h0v;
      }
      G = af2(gbase[i * kArC], gbase[(i + kArH) * kArC]);
    };

    // ---- pass 1: the two half-chunk maps (carry_in -> carry_out), backwards
    float2 M00 = af2(1.f, 1.f), M01 = af2(0.f, 0.f), M10 = M01, M11 = M00, D0 = M01, D1 = M01;
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UI, UF, UG, UO, CP, HP, G, F, X, KK, A11, GCI, GCF, GCG, DOT;
      al_args(ubase + i * kAlUStep, ubase + (i + kArH) * kAlUStep, BS, UI, UF, UG, UO);
      state(i, CP, HP, G);
      al_cell(k, CP, HP, UI, UF, UG, UO, F, X, KK, A11, GCI, GCF, GCG, DOT);
      const float2 A10 = amul(KK, F);
      // carry_out = A^T (carry_in + (0, g)); compose after the map so far
      const float2 E1 = aadd(D1, G);
      const float2 n00 = afma(F, M00, amul(A10, M10)), n01 = afma(F, M01, amul(A10, M11));
      const float2 n10 = afma(X, M00, amul(A11, M10)), n11 = afma(X, M01, amul(A11, M11));
      const float2 nd0 = afma(F, D0, amul(A10, E1)), nd1 = afma(X, D0, amul(A11, E1));
      M00 = n00;
      M01 = n01;
      M10 = n10;
      M11 = n11;
      D0 = nd0;
      D1 = nd1;
    }
    const Aff2 Mx{M00.x, M01.x, M10.x, M11.x, D0.x, D1.x};
    const Aff2 My{M00.y, M01.y, M10.y, M11.y, D0.y, D1.y};
    // the chunk's map: the first half after the second
    Aff2 inc = Mx.after(My);
    // suffix scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
    for (int o = kArC; o < 32; o <<= 1) {
      const Aff2 nx = alq_shfl_down(inc, o);
      if (lane + o < 32) inc = inc.after(nx);
    }
    // the carry entering the warp -> the carry entering this chunk
    Aff2 xm = alq_shfl_down(inc, kArC);
    if (kk == kArK - 1) xm = Aff2::id();
    if (kk == 0) {
      sh.wagg[par][warp][c][0] = make_float4(inc.m00, inc.m01, inc.m10, inc.m11);
      sh.wagg[par][warp][c][1] = make_float4(inc.d0, inc.d1, 0.f, 0.f);
    }
    // the carry entering this segment's last step: zero for the last segment,
    // else the words the segment after it published (count r)
    if (tid < kArC) {
      float2 cin = af2(0.f, 0.f);
      if (r > 0) {
        if ((unsigned)(wc >> 32) < (unsigned)r || (unsigned)(wh >> 32) < (unsigned)r) {
          const uint64_t w0 = globaltimer_ns();
          do {
            wc = alq_ld_word(cwp);
            wh = alq_ld_word(cwp + 1);
            if ((unsigned)(wc >> 32) >= (unsigned)r && (unsigned)(wh >> 32) >= (unsigned)r) break;
            if (globaltimer_ns() - w0 > p.timeout_ns) {
              status = PARARNN_STATUS_TIMEOUT;
              break;
            }
          } while (true);
        }
        cin = af2(__uint_as_float((unsigned)wc), __uint_as_float((unsigned)wh));
      }
      sh.cin[par][c] = cin;
    }
    __syncthreads();
    // every warp is done with the item before: its partial sums, in warp order
    if (prev_part >= 0 && tid < 8 * kArC) {
      const int j = tid / kArC, cc = tid % kArC;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kAlqWarps; ++w) s += sh.red[par ^ 1][w][j][cc];
      p.part[(size_t)prev_part * (8 * kArC) + tid] = s;
    }
    // the warps after this one: the segment's incoming carry -> this warp's
    Aff2 cw = Aff2::id();
#pragma unroll
    for (int w = kAlqWarps - 1; w > 0; --w)
      if (w > warp) {
        const float4 m4 = sh.wagg[par][w][c][0], v4 = sh.wagg[par][w][c][1];
        cw = Aff2{m4.x, m4.y, m4.z, m4.w, v4.x, v4.y}.after(cw);
      }
    const float2 cin_seg = sh.cin[par][c];
    // publish the carry this segment passes to the one before it: its map
    // (the warp-0 chunk-0 suffix after the other warps) applied to cin_seg
    if (warp == 0 && kk == 0 && item != p.withhold_item) {
      const float2 out = inc.after(cw).apply(cin_seg);
      alq_st_word(cwp, alq_word(out.x, r + 1));
      alq_st_word(cwp + 1, alq_word(out.y, r + 1));
    }
    const float2 cchunk = xm.apply(cw.apply(cin_seg));
    const float2 cx = My.apply(cchunk);  // entering step 7 from step 8

    // ---- pass 2: the exact recurrence, du and the partial sums
    float2 LC = af2(cx.x, cchunk.x), LH = af2(cx.y, cchunk.y);
    float2 SA[4], SB[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) SA[g] = SB[g] = af2(0.f, 0.f);
    const int tq = t0 + q * kArL;
    float* dub = p.du + (((size_t)b * p.T + tq) * 4) * p.D + d;
    bool bad = false;
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UI, UF, UG, UO, CP, HP, G, F, X, KK, A11, GCI, GCF, GCG, DOT;
      al_args(ubase + i * kAlUStep, ubase + (i + kArH) * kAlUStep, BS, UI, UF, UG, UO);
      state(i, CP, HP, G);
      al_cell(k, CP, HP, UI, UF, UG, UO, F, X, KK, A11, GCI, GCF, GCG, DOT);
      const float2 LHE = aadd(LH, G);                      // lambda_h
      const float2 LCH = afma(KK, LHE, LC);                // lambda_c + kk lambda_h
      const float2 DU[4] = {amul(GCI, LCH), amul(GCF, LCH), amul(GCG, LCH), amul(DOT, LHE)};
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        SA[g] = afma(DU[g], HP, SA[g]);
        SB[g] = aadd(SB[g], DU[g]);
      }
      // carry = A^T lambda = (f (lambda_c + kk lambda_h), X (...) + a_o du_o)
      LC = amul(F, LCH);
      LH = afma(X, LCH, amul(k.AO, DU[3]));
      if (dval) {
        if (tq + i < p.T) {
          float* o = dub + (size_t)i * 4 * p.D;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            o[(size_t)g * p.D] = DU[g].x;
            bad |= !isfinite(DU[g].x);
          }
        }
        if (tq + kArH + i < p.T) {
          float* o = dub + (size_t)(kArH + i) * 4 * p.D;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            o[(size_t)g * p.D] = DU[g].y;
            bad |= !isfinite(DU[g].y);
          }
        }
      }
    }
    if (first && dval) {
      if (p.dc0) p.dc0[(size_t)b * p.D + d] = LC.x;
      if (p.dh0) p.dh0[(size_t)b * p.D + d] = LH.x;
    }
    // this warp's slots and parameters are free: the next item's
    const int next = sh.nx[par ^ 1];
    __syncwarp();
    if (!dead && next < p.nitems) {
      const int nt = next % p.ntiles, ns = p.nseg - 1 - next / p.ntiles;
      alq_issue(smem, sh, &mu, &mc, &mh, &mg, p, warp, nt / p.nDTc, (nt % p.nDTc) * kArC,
                ns * kAlqSteps, lane);
    }
    // the warp's partial sums: over the two halves, then the warp's chunks
    float v[8];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      v[g] = SA[g].x + SA[g].y;
      v[4 + g] = SB[g].x + SB[g].y;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = dval ? v[j] : 0.f;
      v[j] += __shfl_xor_sync(kAlqFull, v[j], 8);
      v[j] += __shfl_xor_sync(kAlqFull, v[j], 16);
    }
    if (kk == 0)
#pragma unroll
      for (int j = 0; j < 8; ++j) sh.red[par][warp][j][c] = v[j];
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    prev_part = tile * p.nseg + seg;
    item = next;
  }
  // the last item's partial sums
  __syncthreads();
  if (prev_part >= 0 && tid < 8 * kArC) {
    const int j = tid / kArC, cc = tid % kArC;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kAlqWarps; ++w) s += sh.red[(n - 1) & 1][w][j][cc];
    p.part[(size_t)prev_part * (8 * kArC) + tid] = s;
  }
  // copies still in flight into this warp's slots: wait for them (bounded)
  if (dead) mbar_wait_bounded(&sh.bar[warp], (unsigned)(dead - 1), p.timeout_ns);
  const int st = __reduce_max_sync(kAlqFull, status);
  if (lane == 0 && st) atomicMax(p.status, st);
}

__global__ void adjoint_queue_lstm_init(int* status, unsigned* counter,
                                        unsigned long long* carry, int nwords) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    *status = 0;
    *counter = 0u;
  }
  for (int j = i; j < nwords; j += gridDim.x * blockDim.x) carry[j] = 0ull;
}

int alq_per_sm() {
  int per_sm = 0;
  if (cudaFuncSetAttribute(adjoint_queue_lstm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kAlqSmem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adjoint_queue_lstm, kAlqThreads,
                                                    kAlqSmem) != cudaSuccess)
    per_sm = 0;
  cudaGetLastError();
  return per_sm;
}

}  // namespace

void adjoint_row_reduce_launch(const float* part, float* da, float* dbias, int B, int D, int cls,
                               int G, cudaStream_t stream);

// Workspace bytes past the 256-byte header: partial sums, carry words, count.
size_t adjoint_queue_lstm_bytes(int B, int T, int D) {
  const size_t ntiles = (size_t)B * ((D + kArC - 1) / kArC);
  const size_t nseg = (size_t)(T + kAlqSteps - 1) / kAlqSteps;
  return align256(ntiles * nseg * 8 * kArC * 4) + align256(ntiles * kArC * 2 * 8) + 256;
}

// Resident CTAs of the ParaLSTM queue adjoint on the current device.
int adjoint_queue_lstm_resident() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * alq_per_sm();
}

// maps: u (box 8 x 4 x 19), c and h (box 8 x 20), dL/dh (box 8 x 19); ws: the
// workspace past its header, adjoint_queue_lstm_bytes(B, T, D) bytes
int launch_adjoint_queue_lstm(const CUtensorMap* maps, const float* a, const float* bias,
                              const float* c0, const float* h0, float* du, float* da,
                              float* dbias, float* dc0, float* dh0, int B, int T, int D,
                              int* status, void* ws, uint64_t timeout_ns, int withhold_item,
                              cudaStream_t stream) {
  AlqParams p;
  p.a = a;
  p.bias = bias;
  p.c0 = c0;
  p.h0 = h0;
  p.du = du;
  p.dc0 = dc0;
  p.dh0 = dh0;
  p.B = B;
  p.T = T;
  p.D = D;
  p.nDTc = (D + kArC - 1) / kArC;
  p.ntiles = B * p.nDTc;
  p.nseg = (T + kAlqSteps - 1) / kAlqSteps;
  if ((long long)p.ntiles * p.nseg >= (1LL << 31)) return 1;
  p.nitems = p.ntiles * p.nseg;
  p.timeout_ns = timeout_ns;
  p.status = status;
  p.withhold_item = withhold_item;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.part = reinterpret_cast<float*>(w);
  w += align256((size_t)p.nitems * 8 * kArC * 4);
  p.carry = reinterpret_cast<unsigned long long*>(w);
  w += align256((size_t)p.ntiles * kArC * 2 * 8);
  p.counter = reinterpret_cast<unsigned*>(w);
  const int nwords = p.ntiles * kArC * 2;
  adjoint_queue_lstm_init<<<(unsigned)std::min(1024, (nwords + 255) / 256 + 1), 256, 0,
                            stream>>>(status, p.counter, p.carry, nwords);
  const int per_sm = std::max(1, alq_per_sm());
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = std::min<long long>((long long)sms * per_sm, p.nitems);
  adjoint_queue_lstm<<<(unsigned)std::max<long long>(grid, 1), kAlqThreads, kAlqSmem, stream>>>(
      maps[0], maps[1], maps[2], maps[3], p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  adjoint_row_reduce_launch(p.part, da, dbias, B, D, p.nseg, 4, stream);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
