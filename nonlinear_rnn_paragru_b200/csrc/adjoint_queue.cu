// adjoint_queue.cu -- reverse (adjoint) scan of a solved ParaGRU trajectory
// with bf16 input projections: every 128-step segment of every 32-channel
// tile in one persistent launch, last segments first.
//
// The gradient flows back through the transposed block-bidiagonal system
// ("Параллельность RNN?", §1.3):
//   lambda_t = g_t + carry_{t+1},  carry_t = A_t lambda_t  (A_t = df_t/dh),
//   du_t = (df_t/du_t) lambda_t,  da = sum_t (df_t/da) lambda_t,
//   dbias = sum_t du_t,  dL/dh0 = carry_1.
// A segment needs from the steps after it only the carry entering its last
// step.  An item is 32 channels of one batch row over one segment; items are
// numbered so that every tile's last segment comes first (item = r * ntiles +
// tile for the segment r from the end) and drawn from a counter two ahead.
// A CTA of 16 warps holds a segment: warp w the 8-step chunk w, lane c channel
// c, the 8 steps as 4 packed step pairs (i, i + 4) through the cell of
// adjoint_cell.cuh.  Every warp stages its own chunk (u as 64-byte rows, h_{t-1}
// and dL/dh as 128-byte rows: few, full-width copy rows) and its own copy of
// the tile's parameters on its own mbarriers, in two stages: the next item's
// boxes are in flight while the warp works on this one.
//   pass 1: each chunk's map carry_in -> carry_out, backwards, keeping the
//     cell's results (A, the three df/du, r h) of every step in registers;
//   scan: the carry entering a chunk is the segment's incoming carry taken
//     through the chunk maps of the warps after it, read from shared memory
//     after one CTA barrier (the only one per item);
//   carry: a segment publishes the carry it passes to the segment before it
//     as one 64-bit word per channel (the value's bits and the count of
//     segments published from the end), so that a single relaxed load, issued
//     when the item starts and checked after pass 1 (a bounded poll if it is
//     not there yet), brings both; the word is written before pass 2, so the
//     chain of segments advances one map application per segment;
//   pass 2: the exact recurrence from the true carry on the kept results: du
//     written (a warp stores whole 128-byte lines) and da / dbias partial sums
//     kept per warp, summed over the warps in a fixed order after the next
//     item's barrier and over the items afterwards in a fixed order: bitwise
//     reproducible.
// The lowest-numbered item that has not published is always some CTA's
// current item and never waits (the items a CTA holds but has not started
// are numbered above its current one), so the queue cannot deadlock while all
// CTAs are resident; a wait that runs out sets TIMEOUT.
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include "adjoint_cell.cuh"
#include "common.cuh"

namespace pararnn {

namespace {

constexpr unsigned kAqFull = 0xffffffffu;
constexpr int kAqC = 32;                           // channels per tile (lanes)
constexpr int kAqW = 16;                           // warps per CTA = chunks per item
constexpr int kAqThreads = kAqW * 32;
constexpr int kAqL = 8;                            // steps per chunk (per thread)
constexpr int kAqH = kAqL / 2;                     // step pairs per chunk
constexpr int kAqSteps = kAqW * kAqL;              // 128 steps per item
// a warp's stage: u [8 steps][3 gates][32 ch] bf16, h_{t-1} [8][32] fp32,
// dL/dh [8][32] fp32, then a, bias (3 rows each) and h0 (1 row) of the tile
constexpr int kAqUStep = 3 * kAqC * 2;             // 192 bytes per step of u
constexpr int kAqSStep = kAqC * 4;                 // 128 bytes per step of h, dL/dh
constexpr int kAqUOff = 0, kAqHOff = kAqL * kAqUStep, kAqGOff = kAqHOff + kAqL * kAqSStep;
constexpr int kAqPOff = kAqGOff + kAqL * kAqSStep;
constexpr int kAqS = kAqPOff + 7 * kAqC * 4;       // 4480 bytes per warp and stage
static_assert(kAqHOff % 128 == 0 && kAqGOff % 128 == 0 && kAqPOff % 128 == 0 &&
                  kAqS % 128 == 0,
              "stage layout");
constexpr int kAqSmem = 2 * kAqW * kAqS;           // 143360
constexpr unsigned kAqBoxBytes = kAqL * (kAqUStep + 2 * kAqSStep);  // 3584

struct AqParams {
  const float *a, *bias, *h0;
  // part: [6][nDT * 32][B * nseg] per-item partial sums of da (rows 0-2) and
  // dbias (rows 3-5), the item's term (b * nseg + segment) innermost
  float *du, *dh0, *part;
  // [ntiles][32]: the carry a segment passes to the one before it, as
  // (float bits) | (segments published from the end of the tile) << 32
  unsigned long long* carry;
  unsigned* counter;   // item tickets (zero at launch)
  int B, T, D, nDT, ntiles, nseg, nitems, nterm;
  FastDiv div_tiles, div_nDT;
  uint64_t timeout_ns;
  int* status;
  int withhold_item;   // testing: this item never publishes its carry (-1: none)
};

struct AqShared {
  uint64_t bar[2][kAqW];              // [stage][warp]: the warp's boxes and parameters
  float2 wagg[2][kAqW][kAqC];         // by item parity: per (warp, channel) chunk map
  float red[2][kAqW][6][kAqC];        // by item parity: partial sums per warp
  float cin[2][kAqC];                 // by item parity: carry entering the last step
  int nx[2];                          // the item two after the current one, by parity
};

// An item's place: batch row, first channel, first step, segment from the end.
struct AqItem {
  int tile, r, b, d0, t0;
};
__device__ __forceinline__ AqItem aq_decode(const AqParams& p, int item) {
  AqItem it;
  it.r = fast_quot(item, p.div_tiles);
  it.tile = item - it.r * p.ntiles;
  it.b = fast_quot(it.tile, p.div_nDT);
  it.d0 = (it.tile - it.b * p.nDT) * kAqC;
  it.t0 = (p.nseg - 1 - it.r) * kAqSteps;
  return it;
}

__device__ __forceinline__ void aq_bulk(void* dst, const void* src, unsigned bytes,
                                        uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ unsigned long long aq_ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void aq_st_word(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Warp `warp`, stage buffer `st` (mbarrier `bar`): its chunk's boxes of item
// `it` (u, h_{t-1}, dL/dh; lanes 0-2) and its copy of the tile's a, bias, h0
// rows (lanes 3-9: the channels below D, 16-byte aligned rows: the caller
// checks the pointers, d0 and D are multiples of 8).
__device__ __forceinline__ void aq_issue(unsigned char* st, uint64_t* bar, const CUtensorMap* mu,
                                         const CUtensorMap* mh, const CUtensorMap* mg,
                                         const AqParams& p, const AqItem& it, int warp,
                                         int lane) {
  const unsigned pb = (unsigned)min(kAqC, p.D - it.d0) * 4;
  if (lane == 0) {
    // this warp's reads of the stage (generic proxy) before the copies into it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, kAqBoxBytes + 3 * pb + (p.bias ? 3 * pb : 0) + (p.h0 ? pb : 0));
  }
  __syncwarp();
  const int ts = it.t0 + warp * kAqL;
  float* par = reinterpret_cast<float*>(st + kAqPOff);
  if (lane == 0) {
    tma_load_4d(st + kAqUOff, mu, bar, it.d0, 0, ts, it.b);
  } else if (lane == 1) {
    tma_load_3d(st + kAqHOff, mh, bar, it.d0, ts - 1, it.b);
  } else if (lane == 2) {
    tma_load_3d(st + kAqGOff, mg, bar, it.d0, ts, it.b);
  } else if (lane < 6) {
    const int g = lane - 3;
    aq_bulk(par + g * kAqC, p.a + (size_t)g * p.D + it.d0, pb, bar);
  } else if (lane < 9) {
    const int g = lane - 6;
    if (p.bias) aq_bulk(par + (3 + g) * kAqC, p.bias + (size_t)g * p.D + it.d0, pb, bar);
  } else if (lane == 9) {
    if (p.h0) aq_bulk(par + 6 * kAqC, p.h0 + (size_t)it.b * p.D + it.d0, pb, bar);
  }
}

__device__ __forceinline__ int aq_draw(unsigned* counter) {
  return (int)min(atomicAdd(counter, 1u), 0x7fffffffu);
}

// pre-scaled arguments of a step pair from bf16 rows [gate][32 channels]
__device__ __forceinline__ void aq_args(const unsigned short* rx, const unsigned short* ry,
                                        float2 S, float2 BZ, float2 BR, float2 BC, float2& UZ,
                                        float2& UR, float2& UC) {
  const float2 SC = af2(2.f * kLog2e, 2.f * kLog2e);
  UZ = afma(S, af2(__uint_as_float((unsigned)rx[0] << 16), __uint_as_float((unsigned)ry[0] << 16)),
            BZ);
  UR = afma(S, af2(__uint_as_float((unsigned)rx[kAqC] << 16),
                   __uint_as_float((unsigned)ry[kAqC] << 16)), BR);
  UC = afma(SC, af2(__uint_as_float((unsigned)rx[2 * kAqC] << 16),
                    __uint_as_float((unsigned)ry[2 * kAqC] << 16)), BC);
}

__global__ void __launch_bounds__(kAqThreads, 1)
    adjoint_queue(const __grid_constant__ CUtensorMap mu, const __grid_constant__ CUtensorMap mh,
                  const __grid_constant__ CUtensorMap mg, const AqParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ AqShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* st0 = smem + warp * kAqS;              // this warp's stage 0
  unsigned char* st1 = smem + (kAqW + warp) * kAqS;     // and stage 1

  // parameter rows start at zero (bias and h0 stay so when absent); rows of
  // channels at or above D are never copied: their lanes compute on whatever
  // the stage holds and store nothing
  for (int i = lane; i < 7 * kAqC; i += 32) {
    reinterpret_cast<float*>(st0 + kAqPOff)[i] = 0.f;
    reinterpret_cast<float*>(st1 + kAqPOff)[i] = 0.f;
  }
  if (tid < 2 * kAqW) mbar_init(&sh.bar[tid / kAqW][tid % kAqW], 1);
  if (tid == 0) {
    sh.nx[0] = aq_draw(p.counter);
    sh.nx[1] = aq_draw(p.counter);
  }
  __syncthreads();
  int item = sh.nx[0], nxt = sh.nx[1];
  __syncthreads();
  // pend: per stage, 1 + the parity of a phase armed and not yet waited for
  int pend0 = 0, pend1 = 0;
  AqItem cur = aq_decode(p, item < p.nitems ? item : 0);
  if (item < p.nitems) {
    aq_issue(st0, &sh.bar[0][warp], &mu, &mh, &mg, p, cur, warp, lane);
    pend0 = 1;
  }
  int status = 0;
  bool live = true;    // false once a wait for this warp's boxes ran out
  long long prev_part = -1;  // the partial-sum offset of the item before
  int n = 0;
  for (; item < p.nitems; ++n) {
    const int s = n & 1;
    // the ticket of the item after the next one: stored just before the barrier
    int ticket = 0;
    if (tid == 0) ticket = aq_draw(p.counter);
    // the next item's boxes into the other stage (this warp is done with it)
    AqItem nit = aq_decode(p, nxt < p.nitems ? nxt : 0);
    if (live && nxt < p.nitems) {
      aq_issue(s ? st0 : st1, &sh.bar[s ^ 1][warp], &mu, &mh, &mg, p, nit, warp, lane);
      if (s) pend0 = 1 + (((n + 1) >> 1) & 1);
      else pend1 = 1 + (((n + 1) >> 1) & 1);
    }
    const int d = cur.d0 + lane;
    const bool dval = d < p.D;
    const bool first = (cur.t0 == 0 && warp == 0);  // the chunk holding step 0
    // the carry word of the segment after this one, fetched now, read after pass 1
    unsigned long long cword = 0ull;
    if (warp == 0 && cur.r > 0) cword = aq_ld_word(&p.carry[(size_t)cur.tile * kAqC + lane]);
    if (live) {
      // a phase that did not complete is never re-armed: the warp stops loading
      if (__all_sync(kAqFull, mbar_wait_bounded(&sh.bar[s][warp], (unsigned)((n >> 1) & 1),
                                                p.timeout_ns))) {
        if (s) pend1 = 0;
        else pend0 = 0;
      } else {
        live = false;
        status = PARARNN_STATUS_TIMEOUT;
      }
    }
    const unsigned char* stg = s ? st1 : st0;
    const unsigned short* ubase = reinterpret_cast<const unsigned short*>(stg + kAqUOff) + lane;
    const float* hbase = reinterpret_cast<const float*>(stg + kAqHOff) + lane;
    const float* gbase = reinterpret_cast<const float*>(stg + kAqGOff) + lane;
    const float* pw = reinterpret_cast<const float*>(stg + kAqPOff) + lane;
    ArCell k;
    float2 S, BZ, BR, BC;
    float h0v;
    {
      const float az = pw[0 * kAqC], ar = pw[1 * kAqC], ac = pw[2 * kAqC];
      k.AZ = af2(az, az);
      k.AR = af2(ar, ar);
      k.AC = af2(ac, ac);
      const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
      k.AZ2 = af2(az2, az2);
      k.AR2 = af2(ar2, ar2);
      k.AC2 = af2(ac2, ac2);
      S = af2(-kLog2e, -kLog2e);
      const float bz = -kLog2e * pw[3 * kAqC], br = -kLog2e * pw[4 * kAqC],
                  bc = 2.f * kLog2e * pw[5 * kAqC];
      BZ = af2(bz, bz);
      BR = af2(br, br);
      BC = af2(bc, bc);
      h0v = pw[6 * kAqC];
    }

    // ---- pass 1: the two half-chunk maps, backwards; the cell kept per pair
    float2 KA[kAqH], KZ[kAqH], KR[kAqH], KC[kAqH], KH[kAqH];
    float2 PM = af2(1.f, 1.f), DM = af2(0.f, 0.f);
#pragma unroll
    for (int i = kAqH - 1; i >= 0; --i) {
      float2 UZ, UR, UC;
      aq_args(ubase + i * (kAqUStep / 2), ubase + (i + kAqH) * (kAqUStep / 2), S, BZ, BR, BC,
              UZ, UR, UC);
      float2 HP = af2(hbase[i * kAqC], hbase[(i + kAqH) * kAqC]);  // h_{t-1}
      if (i == 0 && first) HP.x = h0v;
      const float2 G = af2(gbase[i * kAqC], gbase[(i + kAqH) * kAqC]);
      ar_cell(k, HP, UZ, UR, UC, KA[i], KZ[i], KR[i], KC[i], KH[i]);
      DM = amul(KA[i], aadd(G, DM));
      PM = amul(KA[i], PM);
    }
    // the chunk's map: the first half after the second
    const float2 inc = ar_after(af2(PM.x, DM.x), af2(PM.y, DM.y));
    sh.wagg[s][warp][lane] = inc;
    // the carry entering this segment's last step: zero for the last segment,
    // else the word the segment after it published (count r)
    if (warp == 0) {
      float cin = 0.f;
      if (cur.r > 0) {
        if ((unsigned)(cword >> 32) < (unsigned)cur.r) {
          const uint64_t w0 = globaltimer_ns();
          do {
            cword = aq_ld_word(&p.carry[(size_t)cur.tile * kAqC + lane]);
            if ((unsigned)(cword >> 32) >= (unsigned)cur.r) break;
            if (globaltimer_ns() - w0 > p.timeout_ns) {
              status = PARARNN_STATUS_TIMEOUT;
              break;
            }
          } while (true);
        }
        cin = __uint_as_float((unsigned)cword);
      }
      sh.cin[s][lane] = cin;
    }
    if (tid == 0) sh.nx[s] = ticket;
    __syncthreads();
    const int nn = sh.nx[s];  // the item after the next one
    // every warp is done with the item before: its partial sums, in warp order
    if (prev_part >= 0 && tid < 6 * kAqC) {
      const int j = tid / kAqC, cc = tid % kAqC;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kAqW; ++w) sum += sh.red[s ^ 1][w][j][cc];
      p.part[prev_part + ((size_t)j * p.nDT * kAqC + cc) * p.nterm] = sum;
    }
    // the carry entering this chunk: the segment's incoming carry through the
    // maps of the chunks after this one, last first
    float cchunk = sh.cin[s][lane];
#pragma unroll 3
    for (int w = kAqW - 1; w > warp; --w) {
      const float2 m = sh.wagg[s][w][lane];
      cchunk = fmaf(m.x, cchunk, m.y);
    }
    // publish the carry this segment passes to the one before it: chunk 0's
    // map applied to the carry entering chunk 0
    if (warp == 0 && item != p.withhold_item)
      aq_st_word(&p.carry[(size_t)cur.tile * kAqC + lane],
                 (unsigned long long)__float_as_uint(fmaf(inc.x, cchunk, inc.y)) |
                     ((unsigned long long)(cur.r + 1) << 32));

    // ---- pass 2: the exact recurrence from the true carry, du and the sums;
    // a chunk inside T with its channel below D (warp-uniform but for a
    // partial last tile) takes the copy of the loop without per-step tests
    float2 CARRY = af2(fmaf(PM.y, cchunk, DM.y), cchunk);  // entering steps 3 and 7
    float2 SAZ = af2(0.f, 0.f), SAR = SAZ, SAC = SAZ, SBZ = SAZ, SBR = SAZ, SBC = SAZ;
    const int tq = cur.t0 + warp * kAqL;
    float* dub = p.du + (((size_t)cur.b * p.T + tq) * 3) * p.D + d;
    auto pass2 = [&](auto full) {
      constexpr bool kFull = decltype(full)::value;
#pragma unroll
      for (int i = kAqH - 1; i >= 0; --i) {
        float2 HP = af2(hbase[i * kAqC], hbase[(i + kAqH) * kAqC]);
        if (i == 0 && first) HP.x = h0v;
        const float2 G = af2(gbase[i * kAqC], gbase[(i + kAqH) * kAqC]);
        const float2 LAM = aadd(G, CARRY);
        const float2 DZ = amul(KZ[i], LAM), DR = amul(KR[i], LAM), DC = amul(KC[i], LAM);
        SAZ = afma(DZ, HP, SAZ);
        SAR = afma(DR, HP, SAR);
        SAC = afma(DC, KH[i], SAC);
        SBZ = aadd(SBZ, DZ);
        SBR = aadd(SBR, DR);
        SBC = aadd(SBC, DC);
        CARRY = amul(KA[i], LAM);
        float* ox = dub + (size_t)i * 3 * p.D;
        float* oy = dub + (size_t)(kAqH + i) * 3 * p.D;
        if (kFull || (dval && tq + i < p.T)) {
          ox[0] = DZ.x;
          ox[p.D] = DR.x;
          ox[2 * (size_t)p.D] = DC.x;
        }
        if (kFull || (dval && tq + kAqH + i < p.T)) {
          oy[0] = DZ.y;
          oy[p.D] = DR.y;
          oy[2 * (size_t)p.D] = DC.y;
        }
      }
    };
    if (dval && tq + kAqL <= p.T)
      pass2(std::true_type{});
    else
      pass2(std::false_type{});
    if (first && dval && p.dh0) p.dh0[(size_t)cur.b * p.D + d] = CARRY.x;
    // the warp's partial sums per channel.  Every du of the chunk enters one
    // of the dbias sums, so a non-finite du (or an overflowing sum) leaves one
    // of them non-finite.
    const float v[6] = {SAZ.x + SAZ.y, SAR.x + SAR.y, SAC.x + SAC.y,
                        SBZ.x + SBZ.y, SBR.x + SBR.y, SBC.x + SBC.y};
#pragma unroll
    for (int j = 0; j < 6; ++j) sh.red[s][warp][j][lane] = v[j];
    const bool bad = !isfinite(v[0]) || !isfinite(v[1]) || !isfinite(v[2]) ||
                     !isfinite(v[3]) || !isfinite(v[4]) || !isfinite(v[5]);
    if (dval && bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    prev_part = (long long)cur.d0 * p.nterm + (long long)cur.b * p.nseg + (p.nseg - 1 - cur.r);
    item = nxt;
    nxt = nn;
    cur = nit;
  }
  // the last item's partial sums
  __syncthreads();
  if (prev_part >= 0 && tid < 6 * kAqC) {
    const int j = tid / kAqC, cc = tid % kAqC;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kAqW; ++w) sum += sh.red[(n - 1) & 1][w][j][cc];
    p.part[prev_part + ((size_t)j * p.nDT * kAqC + cc) * p.nterm] = sum;
  }
  // copies still in flight into this warp's stages: wait for them (bounded)
  if (pend0) mbar_wait_bounded(&sh.bar[0][warp], (unsigned)(pend0 - 1), p.timeout_ns);
  if (pend1) mbar_wait_bounded(&sh.bar[1][warp], (unsigned)(pend1 - 1), p.timeout_ns);
  const int sts = __reduce_max_sync(kAqFull, status);
  if (lane == 0 && sts) atomicMax(p.status, sts);
}

__global__ void adjoint_queue_init(int* status, unsigned* counter, unsigned long long* carry,
                                   int nwords) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    *status = 0;
    *counter = 0u;
  }
  for (int j = i; j < nwords; j += gridDim.x * blockDim.x) carry[j] = 0ull;
}

// da[g][d], dbias[g][d] = the items' partial sums of channel d, over the
// batch rows and segments in a fixed order: a warp per output, its lanes
// reading the output's terms as whole lines
__global__ void adjoint_queue_reduce(const float* __restrict__ part, float* da, float* dbias,
                                     int D, int Dp, int nterm) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // over 6 * D
  const int lane = threadIdx.x & 31;
  if (i >= 6 * D) return;
  const int j = i / D, d = i - j * D;
  const float* pp = part + ((size_t)j * Dp + d) * nterm;
  float s = 0.f;
#pragma unroll 8
  for (int t = lane; t < nterm; t += 32) s += pp[t];
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(kAqFull, s, o);
  if (lane == 0) {
    if (j < 3) da[i] = s;
    else if (dbias) dbias[i - 3 * D] = s;
  }
}

}  // namespace

int adjoint_queue_steps() { return kAqSteps; }
int adjoint_queue_channels() { return kAqC; }
// steps per TMA box: u, h (from the state before the chunk's first step), dL/dh
int adjoint_queue_box_steps(int) { return kAqL; }

// Workspace bytes past the 256-byte header: partial sums, carries, counts.
size_t adjoint_queue_bytes(int B, int T, int D) {
  const size_t ntiles = (size_t)B * ((D + kAqC - 1) / kAqC);
  const size_t nseg = (size_t)(T + kAqSteps - 1) / kAqSteps;
  return align256(ntiles * nseg * 6 * kAqC * 4) + align256(ntiles * kAqC * 8) + 256;
}

// Resident CTAs of the queue adjoint on the current device.
int adjoint_queue_resident() {
  int dev = 0, sms = 148, per_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaFuncSetAttribute(adjoint_queue, cudaFuncAttributeMaxDynamicSharedMemorySize, kAqSmem) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adjoint_queue, kAqThreads,
                                                    kAqSmem) != cudaSuccess)
    per_sm = 0;
  cudaGetLastError();
  return sms * per_sm;
}

// maps: u (box 32 x 3 x 8), h (box 32 x 8), dL/dh (box 32 x 8); ws: the
// workspace past its header, adjoint_queue_bytes(B, T, D) bytes
int launch_adjoint_queue(const CUtensorMap* maps, const float* a, const float* bias,
                         const float* h0, float* du, float* da, float* dbias, float* dh0, int B,
                         int T, int D, int* status, void* ws, uint64_t timeout_ns,
                         int withhold_item, cudaStream_t stream) {
  AqParams p;
  p.a = a;
  p.bias = bias;
  p.h0 = h0;
  p.du = du;
  p.dh0 = dh0;
  p.B = B;
  p.T = T;
  p.D = D;
  p.nDT = (D + kAqC - 1) / kAqC;
  p.ntiles = B * p.nDT;
  p.nseg = (T + kAqSteps - 1) / kAqSteps;
  if ((long long)p.ntiles * p.nseg >= (1LL << 31) - 4) return 1;
  p.nitems = p.ntiles * p.nseg;
  p.nterm = B * p.nseg;
  p.div_tiles = fast_div((unsigned)p.ntiles);
  p.div_nDT = fast_div((unsigned)p.nDT);
  p.timeout_ns = timeout_ns;
  p.status = status;
  p.withhold_item = withhold_item;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.part = reinterpret_cast<float*>(w);
  w += align256((size_t)p.nitems * 6 * kAqC * 4);
  p.carry = reinterpret_cast<unsigned long long*>(w);
  w += align256((size_t)p.ntiles * kAqC * 8);
  p.counter = reinterpret_cast<unsigned*>(w);
  const int nwords = p.ntiles * kAqC;
  adjoint_queue_init<<<(unsigned)std::min(1024, (nwords + 255) / 256 + 1), 256, 0, stream>>>(
      status, p.counter, p.carry, nwords);
  cudaError_t e = cudaFuncSetAttribute(adjoint_queue, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kAqSmem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, sms = 148, per_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adjoint_queue, kAqThreads, kAqSmem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  cudaGetLastError();
  const long long grid = std::min<long long>((long long)sms * per_sm, p.nitems);
  adjoint_queue<<<(unsigned)std::max<long long>(grid, 1), kAqThreads, kAqSmem, stream>>>(
      maps[0], maps[1], maps[2], p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  adjoint_queue_reduce<<<(6 * D * 32 + 255) / 256, 256, 0, stream>>>(p.part, da, dbias, D,
                                                                      p.nDT * kAqC, p.nterm);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
