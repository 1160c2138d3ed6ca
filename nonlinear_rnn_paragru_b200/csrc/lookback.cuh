// lookback.cuh -- cross-CTA scan machinery shared by the Newton solves.
//
// The linear system of one Newton iteration is the recurrence
// ds_t = A_t ds_{t-1} + b_t, whose steps are affine maps x -> A x + b; they
// compose associatively, (A2, b2) o (A1, b1) = (A2 A1, A2 b1 + b2), which is
// what lets the recurrence be scanned in parallel ("Параллельность RNN?",
// §1.3, "Уровень 2").  The solvers scan at three levels: thread-serial, across
// the warps of a CTA, and across CTAs.  Across CTAs:
//
//  * inside a thread-block cluster (up to 16 CTAs = one "cluster chunk" of the
//    sequence) every CTA publishes its aggregate in shared memory; after one
//    cluster barrier each CTA composes its predecessors' aggregates read
//    through distributed shared memory;
//  * across cluster chunks of a long sequence, by decoupled look-back: in
//    iteration k a cluster chunk publishes its aggregate (AGG) as soon as its
//    own scan is done, and its inclusive end delta (INCL) once it knows its
//    incoming delta; a successor composes predecessors' aggregates back to the
//    first inclusive record.  Lanes poll up to 32 predecessors at once.
//
// Cluster chunks take tickets in sequence order, so every wait is on a
// cluster that is running or done.  Every global wait is bounded by a
// wall-clock timeout; on expiry the caller reports PARARNN_STATUS_TIMEOUT.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace pararnn {

constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------ affine elements --
// Scalar map x -> P x + d (ParaGRU: diagonal Jacobian, one channel per lane).
struct Aff1 {
  float P, d;
  __device__ static Aff1 id() { return {1.f, 0.f}; }
  // (*this) o e : apply e first
  __device__ Aff1 after(const Aff1& e) const { return {P * e.P, fmaf(P, e.d, d)}; }
  __device__ float apply(float x) const { return fmaf(P, x, d); }
};

// 2x2 map x -> M x + d on (c, h) (ParaLSTM: 2x2 block Jacobian per channel).
struct Aff2 {
  float m00, m01, m10, m11, d0, d1;
  __device__ static Aff2 id() { return {1.f, 0.f, 0.f, 1.f, 0.f, 0.f}; }
  __device__ Aff2 after(const Aff2& e) const {
    Aff2 r;
    r.m00 = fmaf(m00, e.m00, m01 * e.m10);
    r.m01 = fmaf(m00, e.m01, m01 * e.m11);
    r.m10 = fmaf(m10, e.m00, m11 * e.m10);
    r.m11 = fmaf(m10, e.m01, m11 * e.m11);
    r.d0 = fmaf(m00, e.d0, fmaf(m01, e.d1, d0));
    r.d1 = fmaf(m10, e.d0, fmaf(m11, e.d1, d1));
    return r;
  }
  __device__ float2 apply(float2 x) const {
    return make_float2(fmaf(m00, x.x, fmaf(m01, x.y, d0)), fmaf(m10, x.x, fmaf(m11, x.y, d1)));
  }
};

// Global record payload per lane: AGG fields and INCL fields never overlap,
// so a reader that saw either flag value reads consistent data.  Both kinds
// also carry the chunk's last state before this iteration's update ("last",
// written before the first flag), from which the successor re-anchors its
// boundary state each iteration.
//   Aff1: [P, d, incl, last]              (4 floats per lane)
//   Aff2: [m00 m01 m10 m11 | d0 d1 incl.c incl.h | last.c last.h - -] (12)
__device__ __forceinline__ void rec_put_agg(float* rec, int lane, const Aff1& e) {
  float* p = rec + lane * 4;
  *reinterpret_cast<float2*>(p) = make_float2(e.P, e.d);
}
__device__ __forceinline__ void rec_put_incl(float* rec, int lane, float v) { rec[lane * 4 + 2] = v; }
__device__ __forceinline__ void rec_get_agg(const float* rec, int lane, Aff1& e) {
  const float2 v = __ldcg(reinterpret_cast<const float2*>(rec + lane * 4));
  e.P = v.x;
  e.d = v.y;
}
__device__ __forceinline__ void rec_get_incl(const float* rec, int lane, float& v) {
  v = __ldcg(rec + lane * 4 + 2);
}
__device__ __forceinline__ void rec_put_last(float* rec, int lane, float v) { rec[lane * 4 + 3] = v; }
__device__ __forceinline__ void rec_get_last(const float* rec, int lane, float& v) {
  v = __ldcg(rec + lane * 4 + 3);
}
__device__ __forceinline__ void rec_put_agg(float* rec, int lane, const Aff2& e) {
  float* p = rec + lane * 12;
  *reinterpret_cast<float4*>(p) = make_float4(e.m00, e.m01, e.m10, e.m11);
  *reinterpret_cast<float2*>(p + 4) = make_float2(e.d0, e.d1);
}
__device__ __forceinline__ void rec_put_incl(float* rec, int lane, float2 v) {
  *reinterpret_cast<float2*>(rec + lane * 12 + 6) = v;
}
__device__ __forceinline__ void rec_put_last(float* rec, int lane, float2 v) {
  *reinterpret_cast<float2*>(rec + lane * 12 + 8) = v;
}
__device__ __forceinline__ void rec_get_last(const float* rec, int lane, float2& v) {
  v = __ldcg(reinterpret_cast<const float2*>(rec + lane * 12 + 8));
}
__device__ __forceinline__ void rec_get_agg(const float* rec, int lane, Aff2& e) {
  const float4 m = __ldcg(reinterpret_cast<const float4*>(rec + lane * 12));
  const float2 d = __ldcg(reinterpret_cast<const float2*>(rec + lane * 12 + 4));
  e = {m.x, m.y, m.z, m.w, d.x, d.y};
}
__device__ __forceinline__ void rec_get_incl(const float* rec, int lane, float2& v) {
  v = __ldcg(reinterpret_cast<const float2*>(rec + lane * 12 + 6));
}
template <class E> __host__ __device__ constexpr int rec_floats() { return sizeof(E) == sizeof(Aff1) ? 4 : 12; }

__device__ __forceinline__ unsigned make_flag(unsigned epoch, unsigned kind, bool ok) {
  return (epoch << 3) | (kind << 1) | (ok ? 1u : 0u);
}
__device__ __forceinline__ bool flag_valid(unsigned f, unsigned epoch) { return (f >> 3) == epoch; }

// Publish (warp-wide): payload already written by every lane; fence, then
// lane 0 releases the flag.
__device__ __forceinline__ void publish_flag(unsigned* fl, unsigned flag) {
  __threadfence();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) st_release(fl, flag);
}

// Decoupled look-back over the predecessors of cluster chunk `jc` (records of
// chunk q live at rec_base[(ticket0 + q) * stride + k]).  Warp-uniform.
// Returns false on timeout.  On success `din` is the incoming delta of chunk
// jc, `up_ok` tells whether every upstream chunk was below tol at k, and
// `plast` (if not null) is the immediate predecessor's last state before its
// update of iteration k.
template <class E, class V>
__device__ bool lookback(const unsigned* flags, const float* vals, int ticket0, int jc, int k,
                         int stride, unsigned epoch, uint64_t timeout_ns, V& din, bool& up_ok,
                         V* plast = nullptr) {
  const int lane = threadIdx.x & 31;
  constexpr int RF = rec_floats<E>();
  E acc = E::id();
  bool okall = true;
  int q0 = 0;  // predecessors already composed
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    const int n = min(32, jc - q0);  // predecessors jc-1-q0 .. jc-n-q0
    int window = 0, incl_at = -1;
    unsigned ns = 32, f_last = 0;
    for (;;) {  // phase 1: find a window that ends at an inclusive record
      unsigned f = 0;
      if (lane < n) {
        const size_t r = (size_t)(ticket0 + jc - 1 - q0 - lane) * stride + k;
        f = ld_acquire(&flags[r]);
      }
      const bool valid = lane < n && flag_valid(f, epoch);
      f_last = f;
      const unsigned vm = __ballot_sync(kFull, valid);
      const unsigned im = __ballot_sync(kFull, valid && ((f >> 1) & 3u) == kRecIncl);
      if (im) {
        const int qi = __ffs(im) - 1;
        const unsigned need = (qi == 31) ? kFull : ((2u << qi) - 1u);
        if ((vm & need) == need) {
          window = qi + 1;
          incl_at = qi;
          break;
        }
      } else if (n == 32 && vm == kFull) {
        window = 32;
        break;
      }
      const bool late = (globaltimer_ns() - t0) > timeout_ns;
      if (__shfl_sync(kFull, late, 0)) return false;
      __nanosleep(ns);
      ns = ns < 512 ? ns * 2 : 512;
    }
    // phase 2: the window's flags were acquired by their polling lanes; the
    // warp vote plus a fence in every lane orders each lane's payload reads
    // after those acquires.  Payload loads are independent (one round trip).
    {
      const unsigned okm = __ballot_sync(kFull, lane < window && (f_last & 1u));
      const unsigned need = (window == 32) ? kFull : ((1u << window) - 1u);
      okall = okall && ((okm & need) == need);
    }
    __threadfence();
#pragma unroll 4
    for (int q = 0; q < window; ++q) {
      const size_t r = (size_t)(ticket0 + jc - 1 - q0 - q) * stride + k;
      const float* rec = vals + r * (size_t)(kChan * RF);
      if (plast != nullptr && q0 == 0 && q == 0) rec_get_last(rec, lane, *plast);
      if (q == incl_at) {
        V v;
        rec_get_incl(rec, lane, v);
        din = acc.apply(v);
        up_ok = okall;
        return true;
      }
      E e;
      rec_get_agg(rec, lane, e);
      acc = acc.after(e);
    }
    q0 += window;
  }
}

}  // namespace pararnn
