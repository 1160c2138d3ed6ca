// adjoint_queue_lstm.cu -- reverse (adjoint) scan of a solved ParaLSTM
// trajectory with bf16 input projections: every 128-step segment of every
// 32-channel tile in one persistent launch, last segments first.
//
// The ParaGRU queue adjoint (adjoint_queue.cu) with the 2x2 Jacobian
// ("Параллельность RNN?", §1.3, transposed): lambda = (lambda_c, lambda_h),
// the loss gradient enters through lambda_h, carry_t = A_t^T lambda_t;
// du_{i,f,g} = (gci, gcf, gcg) (lambda_c + kk lambda_h), du_o = dot lambda_h
// (the cell of adjoint_cell.cuh), da = sum_t du_t h_{t-1}, dbias = sum_t du_t,
// and dL/dc0, dL/dh0 the carry out of the first step.
//
// Items (32 channels of one batch row over one segment) are numbered so that
// every tile's last segment comes first (item = r * ntiles + tile for the
// segment r from the end) and drawn from a counter two ahead.  A CTA of 16
// warps holds a segment: warp w the 8-step chunk w, lane c channel c, the 8
// steps as 4 packed step pairs (i, i + 4).  Every warp stages its own chunk
// (u as 64-byte rows, c_{t-1}, h_{t-1} and dL/dh as 128-byte rows) on its own
// mbarriers, and warp 0 the tile's parameter rows for the whole CTA, in two
// stages: the next item's boxes are in flight while the CTA works on this one.
//   pass 1: each chunk's map carry_in -> carry_out (2x2 matrix, 2-vector),
//     backwards;
//   scan: the carry entering a chunk is the segment's incoming carry taken
//     through the maps of the chunks after it, read from shared memory after
//     one CTA barrier (the only one per item);
//   carry: a segment publishes the carry it passes to the segment before it
//     as two 64-bit words per channel, (lambda_c bits, count) and (lambda_h
//     bits, count), the count being the segments published from the tile's
//     end; each word is single-copy atomic and names its writer, so relaxed
//     loads (issued when the item starts, checked after pass 1, polled with a
//     bound if not there yet) need no fence; the words are written before
//     pass 2, so the chain of segments advances one map application per
//     segment;
//   pass 2: the exact recurrence from the true carry (the cell evaluated
//     again), du written (a warp stores whole 128-byte lines) and the da /
//     dbias partial sums kept per warp, summed over the warps in a fixed order
//     after the next item's barrier and over the items afterwards in a fixed
//     order: bitwise reproducible.
// The lowest-numbered item that has not published is always some CTA's
// current item and never waits (the items a CTA holds but has not started
// are numbered above its current one), so the queue cannot deadlock while all
// CTAs are resident; a wait that runs out sets TIMEOUT.
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include "adjoint_cell.cuh"
#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

namespace {

constexpr unsigned kAlqFull = 0xffffffffu;
constexpr int kAlqC = 32;                          // channels per tile (lanes)
constexpr int kAlqW = 16;                          // warps per CTA = chunks per item
constexpr int kAlqThreads = kAlqW * 32;
constexpr int kAlqL = 8;                           // steps per chunk (per thread)
constexpr int kAlqH = kAlqL / 2;                   // step pairs per chunk
constexpr int kAlqSteps = kAlqW * kAlqL;           // 128 steps per item
// a warp's stage: u [8 steps][i f g o][32 ch] bf16, then c_{t-1}, h_{t-1} and
// dL/dh [8][32] fp32
constexpr int kAlqUStep = 4 * kAlqC * 2;           // 256 bytes per step of u
constexpr int kAlqSStep = kAlqC * 4;               // 128 bytes per step of a state
constexpr int kAlqUOff = 0, kAlqCOff = kAlqL * kAlqUStep;
constexpr int kAlqHOff = kAlqCOff + kAlqL * kAlqSStep, kAlqGOff = kAlqHOff + kAlqL * kAlqSStep;
constexpr int kAlqS = kAlqGOff + kAlqL * kAlqSStep;  // 5120 bytes per warp and stage
constexpr unsigned kAlqBoxBytes = kAlqS;
// the CTA's parameter rows per stage: a (4 rows), bias (4), c0, h0
constexpr int kAlqPar = 10 * kAlqC * 4;            // 1280 bytes
// dynamic shared memory: the warps' stages, the parameter stages, then the
// scan maps, partial sums, carries, mbarriers and tickets
constexpr int kAlqParOff = 2 * kAlqW * kAlqS;                       // 163840
constexpr int kAlqMapOff = kAlqParOff + 2 * kAlqPar;                // [2][16][3][32] float2
constexpr int kAlqRedOff = kAlqMapOff + 2 * kAlqW * 3 * kAlqC * 8;  // [2][16][8][32] float
constexpr int kAlqCinOff = kAlqRedOff + 2 * kAlqW * 8 * kAlqC * 4;  // [2][32] float2
constexpr int kAlqBarOff = kAlqCinOff + 2 * kAlqC * 8;              // [2][16 + 1] u64
constexpr int kAlqNxOff = kAlqBarOff + 2 * (kAlqW + 1) * 8;         // [2] int
constexpr int kAlqSmem = kAlqNxOff + 16;
static_assert(kAlqCOff % 128 == 0 && kAlqHOff % 128 == 0 && kAlqGOff % 128 == 0 &&
                  kAlqS % 128 == 0 && kAlqParOff % 128 == 0 && kAlqPar % 128 == 0 &&
                  kAlqBarOff % 8 == 0,
              "stage layout");
static_assert(kAlqSmem <= 227 * 1024, "one CTA per SM");

struct AlqParams {
  const float *a, *bias, *c0, *h0;
  float *du, *dc0, *dh0, *part;
  // [ntiles][32][2]: the carry (lambda_c, lambda_h) a segment passes to the
  // one before it, each as (float bits) | (segments published from the end) << 32
  unsigned long long* carry;
  unsigned* counter;   // item tickets (zero at launch)
  int B, T, D, nDT, ntiles, nseg, nitems;
  FastDiv div_tiles, div_nDT;
  uint64_t timeout_ns;
  int* status;
  int withhold_item;   // testing: this item never publishes its carry (-1: none)
};

struct AlqItem {
  int tile, r, b, d0, t0;
};
__device__ __forceinline__ AlqItem alq_decode(const AlqParams& p, int item) {
  AlqItem it;
  it.r = fast_quot(item, p.div_tiles);
  it.tile = item - it.r * p.ntiles;
  it.b = fast_quot(it.tile, p.div_nDT);
  it.d0 = (it.tile - it.b * p.nDT) * kAlqC;
  it.t0 = (p.nseg - 1 - it.r) * kAlqSteps;
  return it;
}

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

// Warp `warp`: its chunk's four boxes of item `it` (u, c_{t-1}, h_{t-1},
// dL/dh; lanes 0-3) into stage buffer `st` on mbarrier `bar`; warp 0 also
// the tile's parameter rows (lanes 4-13: the channels below D, a and bias
// rows, and c0, h0 for a first segment) into `par` on mbarrier `pbar`.  The
// rows are 16-byte aligned (the caller checks the pointers; d0 and D are
// multiples of 8).
__device__ __forceinline__ void alq_issue(unsigned char* st, uint64_t* bar, float* par,
                                          uint64_t* pbar, const CUtensorMap* mu,
                                          const CUtensorMap* mc, const CUtensorMap* mh,
                                          const CUtensorMap* mg, const AlqParams& p,
                                          const AlqItem& it, int warp, int lane) {
  const unsigned pb = (unsigned)min(kAlqC, p.D - it.d0) * 4;
  const bool first_seg = it.t0 == 0;
  if (lane == 0) {
    // this warp's reads of the stage (generic proxy) before the copies into it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, kAlqBoxBytes);
    if (warp == 0)
      mbar_arrive_expect_tx(pbar, 4 * pb + (p.bias ? 4 * pb : 0) +
                                      ((first_seg && p.c0) ? pb : 0) +
                                      ((first_seg && p.h0) ? pb : 0));
  }
  __syncwarp();
  const int ts = it.t0 + warp * kAlqL;
  if (lane == 0) {
    tma_load_4d(st + kAlqUOff, mu, bar, it.d0, 0, ts, it.b);
  } else if (lane == 1) {
    tma_load_3d(st + kAlqCOff, mc, bar, it.d0, ts - 1, it.b);
  } else if (lane == 2) {
    tma_load_3d(st + kAlqHOff, mh, bar, it.d0, ts - 1, it.b);
  } else if (lane == 3) {
    tma_load_3d(st + kAlqGOff, mg, bar, it.d0, ts, it.b);
  } else if (warp == 0) {
    if (lane < 8) {
      const int g = lane - 4;
      alq_bulk(par + g * kAlqC, p.a + (size_t)g * p.D + it.d0, pb, pbar);
    } else if (lane < 12) {
      const int g = lane - 8;
      if (p.bias) alq_bulk(par + (4 + g) * kAlqC, p.bias + (size_t)g * p.D + it.d0, pb, pbar);
    } else if (lane == 12) {
      if (first_seg && p.c0) alq_bulk(par + 8 * kAlqC, p.c0 + (size_t)it.b * p.D + it.d0, pb, pbar);
    } else if (lane == 13) {
      if (first_seg && p.h0) alq_bulk(par + 9 * kAlqC, p.h0 + (size_t)it.b * p.D + it.d0, pb, pbar);
    }
  }
}

__device__ __forceinline__ int alq_draw(unsigned* counter) {
  return (int)min(atomicAdd(counter, 1u), 0x7fffffffu);
}

// pre-scaled arguments of a step pair from bf16 rows [i f g o][32 channels]
__device__ __forceinline__ void alq_args(const unsigned short* rx, const unsigned short* ry,
                                         const float2 (&BS)[4], float2& UI, float2& UF,
                                         float2& UG, float2& UO) {
  const float2 S = af2(-kLog2e, -kLog2e), SG = af2(2.f * kLog2e, 2.f * kLog2e);
  auto ld = [&](int g) {
    return af2(__uint_as_float((unsigned)rx[g * kAlqC] << 16),
               __uint_as_float((unsigned)ry[g * kAlqC] << 16));
  };
  UI = afma(S, ld(0), BS[0]);
  UF = afma(S, ld(1), BS[1]);
  UG = afma(SG, ld(2), BS[2]);
  UO = afma(S, ld(3), BS[3]);
}

__global__ void __launch_bounds__(kAlqThreads, 1)
    adjoint_queue_lstm(const __grid_constant__ CUtensorMap mu,
                       const __grid_constant__ CUtensorMap mc,
                       const __grid_constant__ CUtensorMap mh,
                       const __grid_constant__ CUtensorMap mg, const AlqParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* st0 = smem + warp * kAlqS;             // this warp's stage 0
  unsigned char* st1 = smem + (kAlqW + warp) * kAlqS;   // and stage 1
  float* par0 = reinterpret_cast<float*>(smem + kAlqParOff);
  float* par1 = reinterpret_cast<float*>(smem + kAlqParOff + kAlqPar);
  float2* wmap = reinterpret_cast<float2*>(smem + kAlqMapOff);   // [2][16][3][32]
  float* red = reinterpret_cast<float*>(smem + kAlqRedOff);      // [2][16][8][32]
  float2* cinb = reinterpret_cast<float2*>(smem + kAlqCinOff);   // [2][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAlqBarOff);  // [2][17]: warps, params
  int* nx = reinterpret_cast<int*>(smem + kAlqNxOff);

  // parameter rows start at zero (bias, c0 and h0 stay so when absent, c0
  // and h0 outside first segments); rows of channels at or above D are never
  // copied: their lanes compute on whatever the stage holds and store nothing
  for (int i = tid; i < 2 * 10 * kAlqC; i += kAlqThreads) par0[i] = 0.f;
  if (tid < 2 * (kAlqW + 1)) mbar_init(&bars[tid], 1);
  if (tid == 0) {
    nx[0] = alq_draw(p.counter);
    nx[1] = alq_draw(p.counter);
  }
  __syncthreads();
  int item = nx[0], nxt = nx[1];
  __syncthreads();
  // pend: per stage, 1 + the parity of a phase armed and not yet waited for
  // (this warp's boxes; warp 0 also the parameters)
  int pend0 = 0, pend1 = 0;
  AlqItem cur = alq_decode(p, item < p.nitems ? item : 0);
  if (item < p.nitems) {
    alq_issue(st0, &bars[warp], par0, &bars[kAlqW], &mu, &mc, &mh, &mg, p, cur, warp, lane);
    pend0 = 1;
  }
  int status = 0;
  bool live = true;    // false once a wait for this warp's boxes ran out
  int prev_part = -1;  // the partial-sum row of the item before
  int n = 0;
  for (; item < p.nitems; ++n) {
    const int s = n & 1;
    uint64_t* sbar = bars + s * (kAlqW + 1);
    // the ticket of the item after the next one: stored just before the barrier
    int ticket = 0;
    if (tid == 0) ticket = alq_draw(p.counter);
    // the next item's boxes into the other stage (the CTA is done with it:
    // every parameter read of the item before precedes its barrier)
    AlqItem nit = alq_decode(p, nxt < p.nitems ? nxt : 0);
    if (live && nxt < p.nitems) {
      alq_issue(s ? st0 : st1, bars + (s ^ 1) * (kAlqW + 1) + warp, s ? par0 : par1,
                bars + (s ^ 1) * (kAlqW + 1) + kAlqW, &mu, &mc, &mh, &mg, p, nit, warp, lane);
      if (s) pend0 = 1 + (((n + 1) >> 1) & 1);
      else pend1 = 1 + (((n + 1) >> 1) & 1);
    }
    const int d = cur.d0 + lane;
    const bool dval = d < p.D;
    const bool first = (cur.t0 == 0 && warp == 0);  // the chunk holding step 0
    // the carry words of the segment after this one, fetched now, read after pass 1
    unsigned long long* cwp = &p.carry[((size_t)cur.tile * kAlqC + lane) * 2];
    unsigned long long wc = 0ull, wh = 0ull;
    if (warp == 0 && cur.r > 0) {
      wc = alq_ld_word(cwp);
      wh = alq_ld_word(cwp + 1);
    }
    if (live) {
      // a phase that did not complete is never re-armed: the warp stops loading
      const unsigned ph = (unsigned)((n >> 1) & 1);
      bool ok = mbar_wait_bounded(&sbar[warp], ph, p.timeout_ns);
      if (ok) ok = mbar_wait_bounded(&sbar[kAlqW], ph, p.timeout_ns);
      if (__all_sync(kAlqFull, ok)) {
        if (s) pend1 = 0;
        else pend0 = 0;
      } else {
        live = false;
        status = PARARNN_STATUS_TIMEOUT;
      }
    }
    const unsigned char* stg = s ? st1 : st0;
    const unsigned short* ubase = reinterpret_cast<const unsigned short*>(stg + kAlqUOff) + lane;
    const float* cbase = reinterpret_cast<const float*>(stg + kAlqCOff) + lane;
    const float* hbase = reinterpret_cast<const float*>(stg + kAlqHOff) + lane;
    const float* gbase = reinterpret_cast<const float*>(stg + kAlqGOff) + lane;
    const float* pw = (s ? par1 : par0) + lane;
    AlCell k;
    float2 BS[4];
    float c0v, h0v;
    {
      const float ai = pw[0 * kAlqC], af = pw[1 * kAlqC], ag = pw[2 * kAlqC], ao = pw[3 * kAlqC];
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
        const float bs = (g == 2 ? 2.f * kLog2e : -kLog2e) * pw[(4 + g) * kAlqC];
        BS[g] = af2(bs, bs);
      }
      c0v = first ? pw[8 * kAlqC] : 0.f;
      h0v = first ? pw[9 * kAlqC] : 0.f;
    }
    auto state = [&](int i, float2& CP, float2& HP, float2& G) {
      CP = af2(cbase[i * kAlqC], cbase[(i + kAlqH) * kAlqC]);  // (c, h)_{t-1}
      HP = af2(hbase[i * kAlqC], hbase[(i + kAlqH) * kAlqC]);
      if (i == 0 && first) {
        CP.x = c0v;
        HP.x = h0v;
      }
      G = af2(gbase[i * kAlqC], gbase[(i + kAlqH) * kAlqC]);
    };

    // ---- pass 1: the two half-chunk maps (carry_in -> carry_out), backwards
    float2 M00 = af2(1.f, 1.f), M01 = af2(0.f, 0.f), M10 = M01, M11 = M00, D0 = M01, D1 = M01;
#pragma unroll
    for (int i = kAlqH - 1; i >= 0; --i) {
      float2 UI, UF, UG, UO, CP, HP, G, F, X, KK, A11, GCI, GCF, GCG, DOT;
      alq_args(ubase + i * (kAlqUStep / 2), ubase + (i + kAlqH) * (kAlqUStep / 2), BS, UI, UF,
               UG, UO);
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
    const Aff2 inc = Mx.after(My);
    {
      float2* mw = wmap + ((s * kAlqW + warp) * 3) * kAlqC + lane;
      mw[0] = af2(inc.m00, inc.m01);
      mw[kAlqC] = af2(inc.m10, inc.m11);
      mw[2 * kAlqC] = af2(inc.d0, inc.d1);
    }
    // the carry entering this segment's last step: zero for the last segment,
    // else the words the segment after it published (count r)
    if (warp == 0) {
      float2 cin = af2(0.f, 0.f);
      const int r = cur.r;
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
      cinb[s * kAlqC + lane] = cin;
    }
    if (tid == 0) nx[s] = ticket;
    __syncthreads();
    const int nn = nx[s];  // the item after the next one
    // every warp is done with the item before: its partial sums, in warp order
    if (prev_part >= 0 && tid < 8 * kAlqC) {
      const float* rp = red + (s ^ 1) * kAlqW * 8 * kAlqC + tid;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kAlqW; ++w) sum += rp[w * 8 * kAlqC];
      p.part[(size_t)prev_part * (8 * kAlqC) + tid] = sum;
    }
    // the carry entering this chunk: the segment's incoming carry through the
    // maps of the chunks after this one, last first
    float2 cchunk = cinb[s * kAlqC + lane];
#pragma unroll 2
    for (int w = kAlqW - 1; w > warp; --w) {
      const float2* mw = wmap + ((s * kAlqW + w) * 3) * kAlqC + lane;
      const float2 m0 = mw[0], m1 = mw[kAlqC], dv = mw[2 * kAlqC];
      cchunk = Aff2{m0.x, m0.y, m1.x, m1.y, dv.x, dv.y}.apply(cchunk);
    }
    // publish the carry this segment passes to the one before it: chunk 0's
    // map applied to the carry entering chunk 0
    if (warp == 0 && item != p.withhold_item) {
      const float2 out = inc.apply(cchunk);
      alq_st_word(cwp, alq_word(out.x, cur.r + 1));
      alq_st_word(cwp + 1, alq_word(out.y, cur.r + 1));
    }
    const float2 cx = My.apply(cchunk);  // entering step 3 from step 4

    // ---- pass 2: the exact recurrence, du and the partial sums; a chunk
    // inside T with its channel below D (warp-uniform but for a partial last
    // tile) takes the copy of the loop without per-step tests
    float2 LC = af2(cx.x, cchunk.x), LH = af2(cx.y, cchunk.y);
    float2 SA[4], SB[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) SA[g] = SB[g] = af2(0.f, 0.f);
    const int tq = cur.t0 + warp * kAlqL;
    float* dub = p.du + (((size_t)cur.b * p.T + tq) * 4) * p.D + d;
    auto pass2 = [&](auto full) {
      constexpr bool kFull = decltype(full)::value;
#pragma unroll
      for (int i = kAlqH - 1; i >= 0; --i) {
        float2 UI, UF, UG, UO, CP, HP, G, F, X, KK, A11, GCI, GCF, GCG, DOT;
        alq_args(ubase + i * (kAlqUStep / 2), ubase + (i + kAlqH) * (kAlqUStep / 2), BS, UI, UF,
                 UG, UO);
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
        float* ox = dub + (size_t)i * 4 * p.D;
        float* oy = dub + (size_t)(kAlqH + i) * 4 * p.D;
        if (kFull || (dval && tq + i < p.T)) {
#pragma unroll
          for (int g = 0; g < 4; ++g) ox[(size_t)g * p.D] = DU[g].x;
        }
        if (kFull || (dval && tq + kAlqH + i < p.T)) {
#pragma unroll
          for (int g = 0; g < 4; ++g) oy[(size_t)g * p.D] = DU[g].y;
        }
      }
    };
    if (dval && tq + kAlqL <= p.T)
      pass2(std::true_type{});
    else
      pass2(std::false_type{});
    if (first && dval) {
      if (p.dc0) p.dc0[(size_t)cur.b * p.D + d] = LC.x;
      if (p.dh0) p.dh0[(size_t)cur.b * p.D + d] = LH.x;
    }
    // the warp's partial sums per channel.  Every du of the chunk enters one
    // of the dbias sums, so a non-finite du (or an overflowing sum) leaves one
    // of them non-finite.
    float v[8];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      v[g] = SA[g].x + SA[g].y;
      v[4 + g] = SB[g].x + SB[g].y;
    }
    bool bad = false;
    float* rw = red + (s * kAlqW + warp) * 8 * kAlqC + lane;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rw[j * kAlqC] = v[j];
      bad |= !isfinite(v[j]);
    }
    if (dval && bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    prev_part = cur.tile * p.nseg + (p.nseg - 1 - cur.r);
    item = nxt;
    nxt = nn;
    cur = nit;
  }
  // the last item's partial sums
  __syncthreads();
  if (prev_part >= 0 && tid < 8 * kAlqC) {
    const float* rp = red + ((n - 1) & 1) * kAlqW * 8 * kAlqC + tid;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kAlqW; ++w) sum += rp[w * 8 * kAlqC];
    p.part[(size_t)prev_part * (8 * kAlqC) + tid] = sum;
  }
  // copies still in flight into this warp's stages (warp 0: and the
  // parameter stages): wait for them (bounded)
  if (pend0) {
    mbar_wait_bounded(&bars[warp], (unsigned)(pend0 - 1), p.timeout_ns);
    if (warp == 0) mbar_wait_bounded(&bars[kAlqW], (unsigned)(pend0 - 1), p.timeout_ns);
  }
  if (pend1) {
    mbar_wait_bounded(&bars[kAlqW + 1 + warp], (unsigned)(pend1 - 1), p.timeout_ns);
    if (warp == 0) mbar_wait_bounded(&bars[2 * kAlqW + 1], (unsigned)(pend1 - 1), p.timeout_ns);
  }
  const int sts = __reduce_max_sync(kAlqFull, status);
  if (lane == 0 && sts) atomicMax(p.status, sts);
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

// da[g][d], dbias[g][d] = the items' partial sums of channel d, over the
// batch rows and segments in a fixed order (a warp per output pair)
__global__ void adjoint_queue_lstm_reduce(const float* __restrict__ part, float* da,
                                          float* dbias, int B, int D, int nDT, int nseg) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // over 4 * D
  const int lane = threadIdx.x & 31;
  if (i >= 4 * D) return;
  const int g = i / D, d = i - g * D;
  const int dt = d / kAlqC, cc = d % kAlqC;
  const int nterm = B * nseg;
  float sa = 0.f, sb = 0.f;
#pragma unroll 8
  for (int j = lane; j < nterm; j += 32) {
    const int b = j / nseg, r = j - b * nseg;
    const float* pp = part + ((size_t)(b * nDT + dt) * nseg + r) * (8 * kAlqC);
    sa += pp[g * kAlqC + cc];
    sb += pp[(4 + g) * kAlqC + cc];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    sa += __shfl_xor_sync(kAlqFull, sa, o);
    sb += __shfl_xor_sync(kAlqFull, sb, o);
  }
  if (lane == 0) {
    da[i] = sa;
    if (dbias) dbias[i] = sb;
  }
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

int adjoint_queue_lstm_channels() { return kAlqC; }

// Workspace bytes past the 256-byte header: partial sums, carry words, count.
size_t adjoint_queue_lstm_bytes(int B, int T, int D) {
  const size_t ntiles = (size_t)B * ((D + kAlqC - 1) / kAlqC);
  const size_t nseg = (size_t)(T + kAlqSteps - 1) / kAlqSteps;
  return align256(ntiles * nseg * 8 * kAlqC * 4) + align256(ntiles * kAlqC * 2 * 8) + 256;
}

// Resident CTAs of the ParaLSTM queue adjoint on the current device.
int adjoint_queue_lstm_resident() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * alq_per_sm();
}

// maps: u (box 32 x 4 x 8), c, h and dL/dh (box 32 x 8); ws: the workspace
// past its header, adjoint_queue_lstm_bytes(B, T, D) bytes
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
  p.nDT = (D + kAlqC - 1) / kAlqC;
  p.ntiles = B * p.nDT;
  p.nseg = (T + kAlqSteps - 1) / kAlqSteps;
  if ((long long)p.ntiles * p.nseg >= (1LL << 31) - 4) return 1;
  p.nitems = p.ntiles * p.nseg;
  p.div_tiles = fast_div((unsigned)p.ntiles);
  p.div_nDT = fast_div((unsigned)p.nDT);
  p.timeout_ns = timeout_ns;
  p.status = status;
  p.withhold_item = withhold_item;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.part = reinterpret_cast<float*>(w);
  w += align256((size_t)p.nitems * 8 * kAlqC * 4);
  p.carry = reinterpret_cast<unsigned long long*>(w);
  w += align256((size_t)p.ntiles * kAlqC * 2 * 8);
  p.counter = reinterpret_cast<unsigned*>(w);
  const int nwords = p.ntiles * kAlqC * 2;
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
  adjoint_queue_lstm_reduce<<<(4 * D * 32 + 255) / 256, 256, 0, stream>>>(p.part, da, dbias, B, D,
                                                                          p.nDT, p.nseg);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
