// adjoint_queue.cu -- reverse (adjoint) scan of a solved ParaGRU trajectory
// with bf16 input projections for many 8-channel tiles: every 256-step
// segment of every tile in one persistent launch, last segments first.
//
// The gradient flows back through the transposed block-bidiagonal system
// ("Параллельность RNN?", §1.3):
//   lambda_t = g_t + carry_{t+1},  carry_t = A_t lambda_t  (A_t = df_t/dh),
//   du_t = (df_t/du_t) lambda_t,  da = sum_t (df_t/da) lambda_t,
//   dbias = sum_t du_t,  dL/dh0 = carry_1.
// A segment needs from the steps after it only the carry entering its last
// step.  An item is 8 channels of one batch row over one segment; items are
// numbered so that every tile's last segment comes first (item = r * ntiles +
// tile for the segment r from the end) and drawn from a counter one ahead.
// A CTA of 4 warps holds a segment (lane = (chunk k = lane / 8, channel c =
// lane % 8), 16 steps per thread, the cell of adjoint_cell.cuh); every warp
// stages its own four chunks and its own copy of the tile's parameters on its
// own mbarrier, and loads the next item's as soon as its pass 2 is done:
//   pass 1: each chunk's map carry_in -> carry_out, backwards;
//   scan: a suffix scan over the warp's four chunks by shuffles, and over the
//     warps from shared memory after one CTA barrier (the only one per item);
//   carry: a segment publishes the carry it passes to the segment before it
//     as one 64-bit word per channel (the value's bits and the count of
//     segments published from the end), so that a single relaxed load, issued
//     when the item starts and checked after pass 1 (a bounded poll if it is
//     not there yet), brings both; the word is written before pass 2, so the
//     chain of segments advances one map application per segment;
//   pass 2: the exact recurrence from the true carry, du written and da /
//     dbias partial sums kept per warp, summed over the warps in a fixed order
//     after the next item's barrier (reduced over the items afterwards in a
//     fixed order: bitwise reproducible).
// The lowest-numbered item that has not published is always being worked on
// and never waits, so the queue cannot deadlock while all CTAs are resident;
// a wait that runs out sets TIMEOUT.  Five CTAs share an SM (92 registers a
// thread, 40 KB of shared memory a CTA; 251 us against 274 us with four for
// B=8 T=4096 D=1024), against two CTAs of 8 warps in clusters exchanging maps
// every tile for the whole-sequence kernel.
#include <cuda_bf16.h>

#include <algorithm>

#include "adjoint_cell.cuh"
#include "common.cuh"

namespace pararnn {

namespace {

constexpr unsigned kAqFull = 0xffffffffu;
constexpr int kAqWarps = 4;
constexpr int kAqThreads = kAqWarps * 32;
constexpr int kAqChunks = kAqWarps * kArK;        // 16
constexpr int kAqSteps = kAqChunks * kArL;        // 256 steps per item
constexpr int kAqSmem = kAqChunks * kArS;         // 36864
constexpr unsigned kAqWarpBytes =
    kArK * (kArUBox * kArUStep + kArHBox * kArSStep + kArGBox * kArSStep);

struct AqParams {
  const float *a, *bias, *h0;
  float *du, *dh0, *part;
  // [ntiles][8]: the carry a segment passes to the one before it, as
  // (float bits) | (segments published from the end of the tile) << 32
  unsigned long long* carry;
  unsigned* counter;   // item tickets (zero at launch)
  int B, T, D, nDTc, ntiles, nseg, nitems;
  uint64_t timeout_ns;
  int* status;
  int withhold_item;   // testing: this item never publishes its carry (-1: none)
};

struct AqShared {
  uint64_t bar[kAqWarps];           // per warp: its chunks' boxes and parameters
  float par[kAqWarps][7][kArC];     // per warp: a (3 rows), bias (3 rows), h0
  float2 wagg[2][kAqWarps][kArC];   // by item parity: per (warp, channel) suffix map
  float red[2][kAqWarps][6][kArC];  // by item parity: partial sums per warp
  float cin[2][kArC];               // by item parity: carry entering the last step
  int nx[2];                        // the item after this one, by parity
};

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

// Warp `warp`: its four chunks' boxes (u, h_{t-1}, dL/dh; lane k issues chunk
// k's three) and its copy of the a, bias, h0 rows of the item at (b, d0, t0),
// all on the warp's mbarrier.  The rows are 16-byte aligned (the caller
// checks the pointers; d0 is a multiple of 8 and D of 8).
__device__ __forceinline__ void aq_issue(unsigned char* smem, AqShared& sh,
                                         const CUtensorMap* mu, const CUtensorMap* mh,
                                         const CUtensorMap* mg, const AqParams& p, int warp,
                                         int b, int d0, int t0, int lane) {
  const unsigned pb = kArC * 4;
  uint64_t* bar = &sh.bar[warp];
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, kAqWarpBytes + 3 * pb + (p.bias ? 3 * pb : 0) + (p.h0 ? pb : 0));
  }
  __syncwarp();
  if (lane < kArK) {
    const int q = warp * kArK + lane, ts = t0 + q * kArL - lane;
    unsigned char* slot = smem + q * kArS;
    tma_load_4d(slot + kArUOff, mu, bar, d0, 0, ts, b);
    tma_load_3d(slot + kArHOff, mh, bar, d0, ts - 1, b);
    tma_load_3d(slot + kArGOff, mg, bar, d0, ts, b);
  } else if (lane < kArK + 3) {
    const int g = lane - kArK;
    aq_bulk(&sh.par[warp][g][0], p.a + (size_t)g * p.D + d0, pb, bar);
    if (p.bias) aq_bulk(&sh.par[warp][3 + g][0], p.bias + (size_t)g * p.D + d0, pb, bar);
  } else if (lane == kArK + 3 && p.h0) {
    aq_bulk(&sh.par[warp][6][0], p.h0 + (size_t)b * p.D + d0, pb, bar);
  }
}

__device__ __forceinline__ int aq_draw(unsigned* counter) {
  return (int)min(atomicAdd(counter, 1u), 0x7fffffffu);
}

__global__ void __launch_bounds__(kAqThreads, 5)
    adjoint_queue(const __grid_constant__ CUtensorMap mu, const __grid_constant__ CUtensorMap mh,
                  const __grid_constant__ CUtensorMap mg, const AqParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ AqShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane % kArC, kk = lane / kArC;
  const int q = warp * kArK + kk;

  for (int i = tid; i < kAqWarps * 7 * kArC; i += kAqThreads) (&sh.par[0][0][0])[i] = 0.f;
  if (tid < kAqWarps) mbar_init(&sh.bar[tid], 1);
  if (tid == 0) sh.nx[0] = aq_draw(p.counter);
  __syncthreads();
  int item = sh.nx[0];
  if (item < p.nitems) {
    const int tile = item % p.ntiles, seg = p.nseg - 1 - item / p.ntiles;
    aq_issue(smem, sh, &mu, &mh, &mg, p, warp, tile / p.nDTc, (tile % p.nDTc) * kArC,
             seg * kAqSteps, lane);
  }
  const unsigned char* slot = smem + q * kArS;
  const unsigned char* ubase = slot + kArUOff + kk * kArUStep + c * 2;
  const float* hbase = reinterpret_cast<const float*>(slot + kArHOff + kk * kArSStep) + c;
  const float* gbase = reinterpret_cast<const float*>(slot + kArGOff + kk * kArSStep) + c;
  const float* pw = &sh.par[warp][0][0] + c;
  int status = 0;
  int n = 0, prev_part = -1;  // prev_part: the partial-sum row of the item before
  bool live = true;           // false once a wait for this warp's boxes ran out
  int fail_par = 0;
  for (; item < p.nitems; ++n) {
    const int par = n & 1;
    if (tid == 0) sh.nx[par ^ 1] = aq_draw(p.counter);
    const int tile = item % p.ntiles, r = item / p.ntiles, seg = p.nseg - 1 - r;
    const int b = tile / p.nDTc, d0 = (tile % p.nDTc) * kArC;
    const int d = d0 + c;
    const bool dval = d < p.D;
    const int t0 = seg * kAqSteps;
    const bool first = (seg == 0 && q == 0);  // the chunk holding step 0
    // the carry word of the segment after this one, fetched now, read after pass 1
    unsigned long long cword = 0ull;
    if (tid < kArC && r > 0) cword = aq_ld_word(&p.carry[(size_t)tile * kArC + c]);
    if (live) {
      // a phase that did not complete is never re-armed: the warp stops loading
      if (!__all_sync(kAqFull, mbar_wait_bounded(&sh.bar[warp], (unsigned)par, p.timeout_ns))) {
        live = false;
        fail_par = par;
        status = PARARNN_STATUS_TIMEOUT;
      }
    }
    ArCell k;
    float2 S, BZ, BR, BC;
    float h0v;
    {
      const float az = pw[0 * kArC], ar = pw[1 * kArC], ac = pw[2 * kArC];
      k.AZ = af2(az, az);
      k.AR = af2(ar, ar);
      k.AC = af2(ac, ac);
      const float az2 = -kLog2e * az, ar2 = -kLog2e * ar, ac2 = 2.f * kLog2e * ac;
      k.AZ2 = af2(az2, az2);
      k.AR2 = af2(ar2, ar2);
      k.AC2 = af2(ac2, ac2);
      S = af2(-kLog2e, -kLog2e);
      const float bz = -kLog2e * pw[3 * kArC], br = -kLog2e * pw[4 * kArC],
                  bc = 2.f * kLog2e * pw[5 * kArC];
      BZ = af2(bz, bz);
      BR = af2(br, br);
      BC = af2(bc, bc);
      h0v = pw[6 * kArC];
    }

    // ---- pass 1: the two half-chunk maps, backwards
    float2 PM = af2(1.f, 1.f), DM = af2(0.f, 0.f);
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UZ, UR, UC, A, GZ, GR, GC, RH;
      ar_args(ubase + i * kArUStep, ubase + (i + kArH) * kArUStep, S, BZ, BR, BC, UZ, UR, UC);
      float2 HP = af2(hbase[i * kArC], hbase[(i + kArH) * kArC]);  // h_{t-1}
      if (i == 0 && first) HP.x = h0v;
      const float2 G = af2(gbase[i * kArC], gbase[(i + kArH) * kArC]);
      ar_cell(k, HP, UZ, UR, UC, A, GZ, GR, GC, RH);
      DM = amul(A, aadd(G, DM));
      PM = amul(A, PM);
    }
    // the chunk's map: the first half after the second
    float2 inc = ar_after(af2(PM.x, DM.x), af2(PM.y, DM.y));
    // suffix scan over the warp's four chunks of channel c (lanes c + 8k)
#pragma unroll
    for (int o = kArC; o < 32; o <<= 1) {
      const float2 nx = af2(__shfl_down_sync(kAqFull, inc.x, o), __shfl_down_sync(kAqFull, inc.y, o));
      if (lane + o < 32) inc = ar_after(inc, nx);
    }
    // the carry entering the warp -> the carry entering this chunk
    float2 xm = af2(__shfl_down_sync(kAqFull, inc.x, kArC), __shfl_down_sync(kAqFull, inc.y, kArC));
    if (kk == kArK - 1) xm = af2(1.f, 0.f);
    if (kk == 0) sh.wagg[par][warp][c] = inc;
    // the carry entering this segment's last step: zero for the last segment,
    // else the word the segment after it published (count r)
    if (tid < kArC) {
      float cin = 0.f;
      if (r > 0) {
        if ((unsigned)(cword >> 32) < (unsigned)r) {
          const uint64_t w0 = globaltimer_ns();
          do {
            cword = aq_ld_word(&p.carry[(size_t)tile * kArC + c]);
            if ((unsigned)(cword >> 32) >= (unsigned)r) break;
            if (globaltimer_ns() - w0 > p.timeout_ns) {
              status = PARARNN_STATUS_TIMEOUT;
              break;
            }
          } while (true);
        }
        cin = __uint_as_float((unsigned)cword);
      }
      sh.cin[par][c] = cin;
    }
    __syncthreads();
    // every warp is done with the item before: its partial sums, in warp order
    if (prev_part >= 0 && tid < 6 * kArC) {
      const int j = tid / kArC, cc = tid % kArC;
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kAqWarps; ++w) s += sh.red[par ^ 1][w][j][cc];
      p.part[(size_t)prev_part * (6 * kArC) + tid] = s;
    }
    // the warps after this one: the segment's incoming carry -> this warp's
    float2 cw = af2(1.f, 0.f);
#pragma unroll
    for (int w = kAqWarps - 1; w > 0; --w)
      if (w > warp) cw = ar_after(sh.wagg[par][w][c], cw);
    const float cin_seg = sh.cin[par][c];
    // publish the carry this segment passes to the one before it: its map
    // (the warp-0 chunk-0 suffix after the other warps) applied to cin_seg
    if (warp == 0 && kk == 0 && item != p.withhold_item) {
      const float2 m = ar_after(inc, cw);
      aq_st_word(&p.carry[(size_t)tile * kArC + c],
                 (unsigned long long)__float_as_uint(fmaf(m.x, cin_seg, m.y)) |
                     ((unsigned long long)(r + 1) << 32));
    }
    const float cwarp = fmaf(cw.x, cin_seg, cw.y);
    const float cchunk = fmaf(xm.x, cwarp, xm.y);

    // ---- pass 2: the exact recurrence, du and the partial sums
    float2 CARRY = af2(fmaf(PM.y, cchunk, DM.y), cchunk);  // entering steps 7 and 15
    float2 SAZ = af2(0.f, 0.f), SAR = SAZ, SAC = SAZ, SBZ = SAZ, SBR = SAZ, SBC = SAZ;
    const int tq = t0 + q * kArL;
    float* dub = p.du + (((size_t)b * p.T + tq) * 3) * p.D + d;
    bool bad = false;
#pragma unroll
    for (int i = kArH - 1; i >= 0; --i) {
      float2 UZ, UR, UC, A, GZ, GR, GC, RH;
      ar_args(ubase + i * kArUStep, ubase + (i + kArH) * kArUStep, S, BZ, BR, BC, UZ, UR, UC);
      float2 HP = af2(hbase[i * kArC], hbase[(i + kArH) * kArC]);
      if (i == 0 && first) HP.x = h0v;
      const float2 G = af2(gbase[i * kArC], gbase[(i + kArH) * kArC]);
      ar_cell(k, HP, UZ, UR, UC, A, GZ, GR, GC, RH);
      const float2 LAM = aadd(G, CARRY);
      const float2 DZ = amul(GZ, LAM), DR = amul(GR, LAM), DC = amul(GC, LAM);
      SAZ = afma(DZ, HP, SAZ);
      SAR = afma(DR, HP, SAR);
      SAC = afma(DC, RH, SAC);
      SBZ = aadd(SBZ, DZ);
      SBR = aadd(SBR, DR);
      SBC = aadd(SBC, DC);
      CARRY = amul(A, LAM);
      if (dval) {
        if (tq + i < p.T) {
          float* o = dub + (size_t)i * 3 * p.D;
          o[0] = DZ.x;
          o[p.D] = DR.x;
          o[2 * (size_t)p.D] = DC.x;
          bad |= !isfinite(DZ.x) || !isfinite(DR.x) || !isfinite(DC.x);
        }
        if (tq + kArH + i < p.T) {
          float* o = dub + (size_t)(kArH + i) * 3 * p.D;
          o[0] = DZ.y;
          o[p.D] = DR.y;
          o[2 * (size_t)p.D] = DC.y;
          bad |= !isfinite(DZ.y) || !isfinite(DR.y) || !isfinite(DC.y);
        }
      }
    }
    if (first && dval && p.dh0) p.dh0[(size_t)b * p.D + d] = CARRY.x;
    // this warp's slots and parameters are free: the next item's
    const int next = sh.nx[par ^ 1];
    __syncwarp();
    if (live && next < p.nitems) {
      const int nt = next % p.ntiles, ns = p.nseg - 1 - next / p.ntiles;
      aq_issue(smem, sh, &mu, &mh, &mg, p, warp, nt / p.nDTc, (nt % p.nDTc) * kArC,
               ns * kAqSteps, lane);
    }
    // the warp's partial sums: over the two halves, then the warp's chunks
    float v[6] = {SAZ.x + SAZ.y, SAR.x + SAR.y, SAC.x + SAC.y,
                  SBZ.x + SBZ.y, SBR.x + SBR.y, SBC.x + SBC.y};
#pragma unroll
    for (int j = 0; j < 6; ++j) {
      v[j] = dval ? v[j] : 0.f;
      v[j] += __shfl_xor_sync(kAqFull, v[j], 8);
      v[j] += __shfl_xor_sync(kAqFull, v[j], 16);
    }
    if (kk == 0)
#pragma unroll
      for (int j = 0; j < 6; ++j) sh.red[par][warp][j][c] = v[j];
    if (bad && status < PARARNN_STATUS_NONFINITE) status = PARARNN_STATUS_NONFINITE;
    prev_part = tile * p.nseg + seg;
    item = next;
  }
  // the last item's partial sums
  __syncthreads();
  if (prev_part >= 0 && tid < 6 * kArC) {
    const int j = tid / kArC, cc = tid % kArC;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kAqWarps; ++w) s += sh.red[(n - 1) & 1][w][j][cc];
    p.part[(size_t)prev_part * (6 * kArC) + tid] = s;
  }
  // copies still in flight into this warp's slots: wait for them (bounded)
  if (!live) mbar_wait_bounded(&sh.bar[warp], (unsigned)fail_par, p.timeout_ns);
  const int st = __reduce_max_sync(kAqFull, status);
  if (lane == 0 && st) atomicMax(p.status, st);
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

}  // namespace

void adjoint_row_reduce_launch(const float* part, float* da, float* dbias, int B, int D, int cls,
                               int G, cudaStream_t stream);

int adjoint_queue_steps() { return kAqSteps; }

// Workspace bytes past the 256-byte header: partial sums, carries, counts.
size_t adjoint_queue_bytes(int B, int T, int D) {
  const size_t ntiles = (size_t)B * ((D + kArC - 1) / kArC);
  const size_t nseg = (size_t)(T + kAqSteps - 1) / kAqSteps;
  return align256(ntiles * nseg * 6 * kArC * 4) + align256(ntiles * kArC * 8) + 256;
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

// maps: u (box 8 x 3 x 19), h (box 8 x 20), dL/dh (box 8 x 19); ws: the
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
  p.nDTc = (D + kArC - 1) / kArC;
  p.ntiles = B * p.nDTc;
  p.nseg = (T + kAqSteps - 1) / kAqSteps;
  if ((long long)p.ntiles * p.nseg >= (1LL << 31)) return 1;
  p.nitems = p.ntiles * p.nseg;
  p.timeout_ns = timeout_ns;
  p.status = status;
  p.withhold_item = withhold_item;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.part = reinterpret_cast<float*>(w);
  w += align256((size_t)p.nitems * 6 * kArC * 4);
  p.carry = reinterpret_cast<unsigned long long*>(w);
  w += align256((size_t)p.ntiles * kArC * 8);
  p.counter = reinterpret_cast<unsigned*>(w);
  const int nwords = p.ntiles * kArC;
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
  adjoint_row_reduce_launch(p.part, da, dbias, B, D, p.nseg, 3, stream);
  return (int)cudaGetLastError();
}

}  // namespace pararnn
