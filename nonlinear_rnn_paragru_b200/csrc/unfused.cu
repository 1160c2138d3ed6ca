// unfused.cu -- the unfused ("CUDA-accelerated") tier of the Newton solve: an
// ablation that shows what fusing the iteration into one kernel buys.
//
// The pages describe three tiers of the same solver: plain framework code, a
// version whose parallel reduction runs in CUDA, and a fully fused kernel
// ("Apple научила классические RNN масштабироваться...", "Три уровня
// производительности").  This file is the middle one.  Every Newton
// iteration ("Параллельность RNN?", §1.2-§1.3) is three separate steps:
//   1. assemble: one thread per (b, t, d) evaluates the cell at the current
//      iterate and writes the Jacobian block A_t = df/ds (s_{t-1}) and the
//      right-hand side -r_t = f_t - s_t to HBM, and the residual maximum;
//   2. scan: the block-bidiagonal system ds_t = A_t ds_{t-1} - r_t, ds_{-1} =
//      0, is solved by a chunked scan in three kernels (chunk maps, a serial
//      pass over the chunk maps of each channel, the chunks re-run from their
//      true carry), which also adds ds to the iterate;
//   3. the host reads the residual maximum and decides whether to go on.
// The iterate lives in the output arrays (h, and c for ParaLSTM), starting at
// zero; the stopping rule is global: the update of the first iteration whose
// residual over the whole problem is below tol is applied, then the loop
// ends; at the cap a residual-only evaluation ends it with NOT_CONVERGED.
// Activations use CUDA's expf and tanhf.  Layout: u [B][T][G][D], states
// [B][T][D]; A and -r in the workspace, [B][T][D] per entry (ParaGRU: A, -r;
// ParaLSTM: A00, A01, A10, A11, -r_c, -r_h for the state order (c, h)).
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace pararnn {

namespace {

constexpr int kUfThreads = 256;
constexpr int kUfChunk = 64;  // steps per scan chunk

template <bool kBF16>
__device__ __forceinline__ float uf_u(const void* u, size_t i) {
  if constexpr (kBF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(u)[i]);
  else
    return reinterpret_cast<const float*>(u)[i];
}

__device__ __forceinline__ float uf_sig(float x) { return 1.f / (1.f + expf(-x)); }

// |v| as ordered bits: non-negative floats order like unsigned integers, and
// NaN is mapped above +inf so that it wins the maximum
__device__ __forceinline__ unsigned uf_abs_bits(float v) {
  return isnan(v) ? 0x7fc00000u : __float_as_uint(fabsf(v));
}

__device__ __forceinline__ void uf_block_max(unsigned bits, unsigned* out) {
  __shared__ unsigned wmax[kUfThreads / 32];
  bits = __reduce_max_sync(0xffffffffu, bits);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) wmax[warp] = bits;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned m = 0;
    for (int w = 0; w < kUfThreads / 32; ++w) m = max(m, wmax[w]);
    atomicMax(out, m);
  }
}

struct UfParams {
  const void* u;
  const float *a, *bias, *c0, *h0;
  float *c, *h;      // the iterate
  float* jac;        // A entries, one [B][T][D] plane each (1 or 4)
  float* rhs;        // -r, one [B][T][D] plane per state (1 or 2)
  float* agg;        // chunk maps: [B][nC][D] per entry (P then d)
  float* carry;      // carry entering each chunk: [B][nC][D] per state entry
  unsigned* rmax;    // residual maximum (ordered bits)
  const float* cin;  // delta entering the sequence [S][B][D] (a shard's), or null = 0
  int B, T, D, nC;
};

// ---------------------------------------------------------------- assemble --
template <bool kBF16>
__global__ void __launch_bounds__(kUfThreads) uf_assemble_gru(const UfParams p) {
  const size_t N = (size_t)p.B * p.T * p.D;
  unsigned m = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < N;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = i / p.D;
    const int d = (int)(i - bt * p.D);
    const int b = (int)(bt / p.T), t = (int)(bt - (size_t)b * p.T);
    const float hp = t > 0 ? p.h[i - p.D] : (p.h0 ? p.h0[(size_t)b * p.D + d] : 0.f);
    const size_t iu = bt * 3 * p.D + d;
    const float az = p.a[d], ar = p.a[p.D + d], ac = p.a[2 * p.D + d];
    const float z = uf_sig(fmaf(az, hp, uf_u<kBF16>(p.u, iu) + (p.bias ? p.bias[d] : 0.f)));
    const float r =
        uf_sig(fmaf(ar, hp, uf_u<kBF16>(p.u, iu + p.D) + (p.bias ? p.bias[p.D + d] : 0.f)));
    const float cc = tanhf(fmaf(ac, r * hp, uf_u<kBF16>(p.u, iu + 2 * (size_t)p.D) +
                                                (p.bias ? p.bias[2 * p.D + d] : 0.f)));
    const float f = fmaf(z, cc - hp, hp);
    // dh'/dh = (1 - z) + (c - h) z (1 - z) a_z + z (1 - c^2) a_c (r + a_r h r (1 - r))
    const float A = (1.f - z) + (cc - hp) * z * (1.f - z) * az +
                    z * (1.f - cc * cc) * ac * fmaf(ar * hp, r * (1.f - r), r);
    const float res = p.h[i] - f;
    p.jac[i] = A;
    p.rhs[i] = -res;
    m = max(m, uf_abs_bits(res));
  }
  uf_block_max(m, p.rmax);
}

template <bool kBF16>
__global__ void __launch_bounds__(kUfThreads) uf_assemble_lstm(const UfParams p) {
  const size_t N = (size_t)p.B * p.T * p.D;
  unsigned m = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < N;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t bt = i / p.D;
    const int d = (int)(i - bt * p.D);
    const int b = (int)(bt / p.T), t = (int)(bt - (size_t)b * p.T);
    const size_t i0 = (size_t)b * p.D + d;
    const float cp = t > 0 ? p.c[i - p.D] : (p.c0 ? p.c0[i0] : 0.f);
    const float hp = t > 0 ? p.h[i - p.D] : (p.h0 ? p.h0[i0] : 0.f);
    const size_t iu = bt * 4 * p.D + d;
    float aa[4], g[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      aa[q] = p.a[q * p.D + d];
      g[q] = fmaf(aa[q], hp,
                  uf_u<kBF16>(p.u, iu + (size_t)q * p.D) + (p.bias ? p.bias[q * p.D + d] : 0.f));
    }
    const float gi = uf_sig(g[0]), gf = uf_sig(g[1]), gg = tanhf(g[2]), go = uf_sig(g[3]);
    const float cn = fmaf(gf, cp, gi * gg);
    const float tc = tanhf(cn);
    const float hn = go * tc;
    // state (c, h): dc'/dc = f, dc'/dh = X, dh'/dc = o (1 - tanh^2) f,
    // dh'/dh = o (1 - o) a_o tanh(c') + o (1 - tanh^2) X
    const float X = cp * gf * (1.f - gf) * aa[1] + gg * gi * (1.f - gi) * aa[0] +
                    gi * (1.f - gg * gg) * aa[2];
    const float odt = go * (1.f - tc * tc);
    const size_t N1 = N;
    p.jac[i] = gf;
    p.jac[N1 + i] = X;
    p.jac[2 * N1 + i] = odt * gf;
    p.jac[3 * N1 + i] = go * (1.f - go) * aa[3] * tc + odt * X;
    const float rc = p.c[i] - cn, rh = p.h[i] - hn;
    p.rhs[i] = -rc;
    p.rhs[N1 + i] = -rh;
    m = max(m, max(uf_abs_bits(rc), uf_abs_bits(rh)));
  }
  uf_block_max(m, p.rmax);
}

// -------------------------------------------------------------------- scan --
// One thread per (b, chunk, d): the chunk's map x_out = P x_in + d from a
// zero incoming delta.  ParaGRU: agg planes P, d; ParaLSTM: P00 P01 P10 P11
// d0 d1.
template <bool kLSTM>
__global__ void __launch_bounds__(kUfThreads) uf_scan_chunks(const UfParams p) {
  const size_t M = (size_t)p.B * p.nC * p.D;
  const size_t N = (size_t)p.B * p.T * p.D;
  for (size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x; j < M;
       j += (size_t)gridDim.x * blockDim.x) {
    const size_t bk = j / p.D;
    const int d = (int)(j - bk * p.D);
    const int b = (int)(bk / p.nC), k = (int)(bk - (size_t)b * p.nC);
    const int t0 = k * kUfChunk, t1 = min(p.T, t0 + kUfChunk);
    size_t i = ((size_t)b * p.T + t0) * p.D + d;
    if constexpr (!kLSTM) {
      float P = 1.f, x = 0.f;
      for (int t = t0; t < t1; ++t, i += p.D) {
        const float A = p.jac[i];
        x = fmaf(A, x, p.rhs[i]);
        P *= A;
      }
      p.agg[j] = P;
      p.agg[M + j] = x;
    } else {
      float p00 = 1.f, p01 = 0.f, p10 = 0.f, p11 = 1.f, x0 = 0.f, x1 = 0.f;
      for (int t = t0; t < t1; ++t, i += p.D) {
        const float a00 = p.jac[i], a01 = p.jac[N + i], a10 = p.jac[2 * N + i],
                    a11 = p.jac[3 * N + i];
        const float y0 = fmaf(a00, x0, fmaf(a01, x1, p.rhs[i]));
        const float y1 = fmaf(a10, x0, fmaf(a11, x1, p.rhs[N + i]));
        x0 = y0;
        x1 = y1;
        const float q00 = fmaf(a00, p00, a01 * p10), q01 = fmaf(a00, p01, a01 * p11);
        const float q10 = fmaf(a10, p00, a11 * p10), q11 = fmaf(a10, p01, a11 * p11);
        p00 = q00;
        p01 = q01;
        p10 = q10;
        p11 = q11;
      }
      p.agg[j] = p00;
      p.agg[M + j] = p01;
      p.agg[2 * M + j] = p10;
      p.agg[3 * M + j] = p11;
      p.agg[4 * M + j] = x0;
      p.agg[5 * M + j] = x1;
    }
  }
}

// One thread per (b, d): the carry entering each chunk, in order.
template <bool kLSTM>
__global__ void __launch_bounds__(kUfThreads) uf_scan_carry(const UfParams p) {
  const size_t M = (size_t)p.B * p.nC * p.D;
  const size_t BD = (size_t)p.B * p.D;
  for (size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x; j < BD;
       j += (size_t)gridDim.x * blockDim.x) {
    const int b = (int)(j / p.D), d = (int)(j - (size_t)b * p.D);
    size_t g = (size_t)b * p.nC * p.D + d;
    if constexpr (!kLSTM) {
      float x = p.cin ? p.cin[j] : 0.f;
      for (int k = 0; k < p.nC; ++k, g += p.D) {
        p.carry[g] = x;
        x = fmaf(p.agg[g], x, p.agg[M + g]);
      }
    } else {
      float x0 = p.cin ? p.cin[j] : 0.f, x1 = p.cin ? p.cin[BD + j] : 0.f;
      for (int k = 0; k < p.nC; ++k, g += p.D) {
        p.carry[g] = x0;
        p.carry[M + g] = x1;
        const float y0 = fmaf(p.agg[g], x0, fmaf(p.agg[M + g], x1, p.agg[4 * M + g]));
        const float y1 = fmaf(p.agg[2 * M + g], x0, fmaf(p.agg[3 * M + g], x1, p.agg[5 * M + g]));
        x0 = y0;
        x1 = y1;
      }
    }
  }
}

// One thread per (b, chunk, d): the chunk re-run from its true carry; the
// deltas are added to the iterate.
template <bool kLSTM>
__global__ void __launch_bounds__(kUfThreads) uf_scan_apply(const UfParams p) {
  const size_t M = (size_t)p.B * p.nC * p.D;
  const size_t N = (size_t)p.B * p.T * p.D;
  for (size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x; j < M;
       j += (size_t)gridDim.x * blockDim.x) {
    const size_t bk = j / p.D;
    const int d = (int)(j - bk * p.D);
    const int b = (int)(bk / p.nC), k = (int)(bk - (size_t)b * p.nC);
    const int t0 = k * kUfChunk, t1 = min(p.T, t0 + kUfChunk);
    size_t i = ((size_t)b * p.T + t0) * p.D + d;
    if constexpr (!kLSTM) {
      float x = p.carry[j];
      for (int t = t0; t < t1; ++t, i += p.D) {
        x = fmaf(p.jac[i], x, p.rhs[i]);
        p.h[i] += x;
      }
    } else {
      float x0 = p.carry[j], x1 = p.carry[M + j];
      for (int t = t0; t < t1; ++t, i += p.D) {
        const float y0 = fmaf(p.jac[i], x0, fmaf(p.jac[N + i], x1, p.rhs[i]));
        const float y1 = fmaf(p.jac[2 * N + i], x0, fmaf(p.jac[3 * N + i], x1, p.rhs[N + i]));
        x0 = y0;
        x1 = y1;
        p.c[i] += x0;
        p.h[i] += x1;
      }
    }
  }
}

// ---------------------------------------------------------- sequence shards --
// A shard is a contiguous range of steps of every (b, d) channel, solved by
// one process (GPU).  Its part of the page's linear system couples to the
// shards before it only through the delta entering its first step, so a
// Newton iteration is: each shard solves its range from a zero incoming
// delta and composes its range's map ds_out = P ds_in + d; the maps of all
// shards are exchanged; each shard composes the maps of the shards before it
// into its incoming delta, and adds P_t ds_in to its local solution.

// One thread per (b, d): the shard's map (the chunk maps composed in order,
// first chunk innermost) and the shard's last states before the update.
// agg planes: ParaGRU P, d; ParaLSTM P00 P01 P10 P11 d0 d1 (state order c, h).
template <bool kLSTM>
__global__ void __launch_bounds__(kUfThreads) uf_shard_total(const UfParams p, float* agg,
                                                            float* last) {
  const size_t M = (size_t)p.B * p.nC * p.D;
  const size_t BD = (size_t)p.B * p.D;
  for (size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x; j < BD;
       j += (size_t)gridDim.x * blockDim.x) {
    const int b = (int)(j / p.D), d = (int)(j - (size_t)b * p.D);
    size_t g = (size_t)b * p.nC * p.D + d;
    const size_t il = ((size_t)b * p.T + p.T - 1) * p.D + d;
    if constexpr (!kLSTM) {
      float P = 1.f, x = 0.f;
      for (int k = 0; k < p.nC; ++k, g += p.D) {
        x = fmaf(p.agg[g], x, p.agg[M + g]);
        P *= p.agg[g];
      }
      agg[j] = P;
      agg[BD + j] = x;
      last[j] = p.h[il];
    } else {
      float p00 = 1.f, p01 = 0.f, p10 = 0.f, p11 = 1.f, x0 = 0.f, x1 = 0.f;
      for (int k = 0; k < p.nC; ++k, g += p.D) {
        const float a00 = p.agg[g], a01 = p.agg[M + g], a10 = p.agg[2 * M + g],
                    a11 = p.agg[3 * M + g];
        const float y0 = fmaf(a00, x0, fmaf(a01, x1, p.agg[4 * M + g]));
        const float y1 = fmaf(a10, x0, fmaf(a11, x1, p.agg[5 * M + g]));
        x0 = y0;
        x1 = y1;
        const float q00 = fmaf(a00, p00, a01 * p10), q01 = fmaf(a00, p01, a01 * p11);
        const float q10 = fmaf(a10, p00, a11 * p10), q11 = fmaf(a10, p01, a11 * p11);
        p00 = q00;
        p01 = q01;
        p10 = q10;
        p11 = q11;
      }
      agg[j] = p00;
      agg[BD + j] = p01;
      agg[2 * BD + j] = p10;
      agg[3 * BD + j] = p11;
      agg[4 * BD + j] = x0;
      agg[5 * BD + j] = x1;
      last[j] = p.c[il];
      last[BD + j] = p.h[il];
    }
  }
}

// One thread per (b, d): the delta entering shard r (the maps of shards
// 0 .. r-1 applied in order to the zero delta entering shard 0) and, for
// r > 0, shard r's new initial state: shard r-1's last state before the
// update plus that delta.
template <bool kLSTM>
__global__ void __launch_bounds__(kUfThreads) uf_shard_combine(const float* aggs,
                                                              const float* lasts, int r, int B,
                                                              int D, float* din, float* bound) {
  const size_t BD = (size_t)B * D;
  const int NA = kLSTM ? 6 : 2, S = kLSTM ? 2 : 1;
  for (size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x; j < BD;
       j += (size_t)gridDim.x * blockDim.x) {
    float x0 = 0.f, x1 = 0.f;
    for (int q = 0; q < r; ++q) {
      const float* A = aggs + (size_t)q * NA * BD + j;
      if constexpr (!kLSTM) {
        x0 = fmaf(A[0], x0, A[BD]);
      } else {
        const float y0 = fmaf(A[0], x0, fmaf(A[BD], x1, A[4 * BD]));
        const float y1 = fmaf(A[2 * BD], x0, fmaf(A[3 * BD], x1, A[5 * BD]));
        x0 = y0;
        x1 = y1;
      }
    }
    din[j] = x0;
    if (kLSTM) din[BD + j] = x1;
    if (r > 0) {
      const float* L = lasts + (size_t)(r - 1) * S * BD + j;
      bound[j] = L[0] + x0;
      if (kLSTM) bound[BD + j] = L[BD] + x1;
    }
  }
}

unsigned uf_grid(size_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  const size_t want = (n + kUfThreads - 1) / kUfThreads;
  return (unsigned)std::max<size_t>(1, std::min<size_t>(want, (size_t)sms * 8));
}

struct UfLayout {
  size_t rmax, jac, rhs, agg, carry, total;
};

UfLayout uf_layout(int cell, int B, int T, int D) {
  const bool lstm = cell == PARARNN_LSTM;
  const size_t N = (size_t)B * T * D;
  const size_t M = (size_t)B * ((T + kUfChunk - 1) / kUfChunk) * D;
  UfLayout L;
  L.rmax = 0;
  L.jac = 256;
  L.rhs = L.jac + align256(N * (lstm ? 4 : 1) * 4);
  L.agg = L.rhs + align256(N * (lstm ? 2 : 1) * 4);
  L.carry = L.agg + align256(M * (lstm ? 6 : 2) * 4);
  L.total = L.carry + align256(M * (lstm ? 2 : 1) * 4);
  return L;
}

}  // namespace

size_t unfused_ws_bytes(int cell, int B, int T, int D) { return uf_layout(cell, B, T, D).total; }

// The host-driven loop; arguments are validated by the caller.  Writes
// *stats (device) at the end.  Returns 0 or a CUDA error.
int unfused_solve(int cell, bool bf16, const void* u, const float* a, const float* bias,
                  const float* c0, const float* h0, float* c, float* h, int B, int T, int D,
                  float tol, int max_iters, pararnn_stats* stats, void* workspace,
                  cudaStream_t stream) {
  const bool lstm = cell == PARARNN_LSTM;
  const UfLayout L = uf_layout(cell, B, T, D);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  UfParams p;
  p.u = u;
  p.a = a;
  p.bias = bias;
  p.c0 = c0;
  p.h0 = h0;
  p.c = c;
  p.h = h;
  p.jac = reinterpret_cast<float*>(ws + L.jac);
  p.rhs = reinterpret_cast<float*>(ws + L.rhs);
  p.agg = reinterpret_cast<float*>(ws + L.agg);
  p.carry = reinterpret_cast<float*>(ws + L.carry);
  p.rmax = reinterpret_cast<unsigned*>(ws + L.rmax);
  p.cin = nullptr;
  p.B = B;
  p.T = T;
  p.D = D;
  p.nC = (T + kUfChunk - 1) / kUfChunk;
  const size_t N = (size_t)B * T * D, M = (size_t)B * p.nC * D, BD = (size_t)B * D;

  cudaError_t e = cudaMemsetAsync(h, 0, N * 4, stream);  // initial guess: zero
  if (e == cudaSuccess && lstm) e = cudaMemsetAsync(c, 0, N * 4, stream);
  if (e != cudaSuccess) return (int)e;
  pararnn_stats st = {0, 0.f, PARARNN_STATUS_CONVERGED, 0};
  for (int k = 0;; ++k) {
    e = cudaMemsetAsync(p.rmax, 0, sizeof(unsigned), stream);
    if (e != cudaSuccess) return (int)e;
    if (lstm) {
      if (bf16) uf_assemble_lstm<true><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
      else uf_assemble_lstm<false><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
    } else {
      if (bf16) uf_assemble_gru<true><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
      else uf_assemble_gru<false><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
    }
    unsigned bits = 0;
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaMemcpyAsync(&bits, p.rmax, sizeof(unsigned), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return (int)e;
    float r;
    std::memcpy(&r, &bits, sizeof r);  // the ordered bits are the float's own
    st.evals = k + 1;
    st.max_residual = r;
    if (!(r == r) || bits >= 0x7f800000u) {  // NaN or inf
      st.status = PARARNN_STATUS_NONFINITE;
      break;
    }
    if (k == max_iters) {  // residual-only evaluation at the cap
      if (!(r < tol)) st.status = PARARNN_STATUS_NOT_CONVERGED;
      break;
    }
    if (lstm) {
      uf_scan_chunks<true><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
      uf_scan_carry<true><<<uf_grid(BD), kUfThreads, 0, stream>>>(p);
      uf_scan_apply<true><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
    } else {
      uf_scan_chunks<false><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
      uf_scan_carry<false><<<uf_grid(BD), kUfThreads, 0, stream>>>(p);
      uf_scan_apply<false><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    st.iters = k + 1;
    if (r < tol) break;  // the update of the first certified iteration is applied
  }
  e = cudaMemcpyAsync(stats, &st, sizeof(st), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // st lives on this stack
  return (int)e;
}

namespace {
UfParams uf_shard_params(int cell, const void* u, const float* a, const float* bias,
                         const float* c_bound, const float* h_bound, float* c, float* h, int B,
                         int Ts, int D, void* workspace) {
  const UfLayout L = uf_layout(cell, B, Ts, D);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  UfParams p;
  p.u = u;
  p.a = a;
  p.bias = bias;
  p.c0 = c_bound;
  p.h0 = h_bound;
  p.c = c;
  p.h = h;
  p.jac = reinterpret_cast<float*>(ws + L.jac);
  p.rhs = reinterpret_cast<float*>(ws + L.rhs);
  p.agg = reinterpret_cast<float*>(ws + L.agg);
  p.carry = reinterpret_cast<float*>(ws + L.carry);
  p.rmax = nullptr;
  p.cin = nullptr;
  p.B = B;
  p.T = Ts;
  p.D = D;
  p.nC = (Ts + kUfChunk - 1) / kUfChunk;
  return p;
}
}  // namespace

// First half of a shard's Newton iteration: residual and Jacobians at the
// iterate (c, h) given the state before the shard (c_bound, h_bound), the
// shard's system solved from a zero incoming delta (chunk maps in the
// workspace), its map and last states to agg / last, and max|r| to *rmax.
// The iterate is not changed.  Arguments are validated by the caller.
int shard_eval(int cell, bool bf16, const void* u, const float* a, const float* bias,
               const float* c_bound, const float* h_bound, const float* c, const float* h, int B,
               int Ts, int D, float* agg, float* last, float* rmax, void* workspace,
               cudaStream_t stream) {
  const bool lstm = cell == PARARNN_LSTM;
  UfParams p = uf_shard_params(cell, u, a, bias, c_bound, h_bound, const_cast<float*>(c),
                               const_cast<float*>(h), B, Ts, D, workspace);
  p.rmax = reinterpret_cast<unsigned*>(rmax);  // ordered bits of |r| are the float's own
  const size_t N = (size_t)B * Ts * D, M = (size_t)B * p.nC * D, BD = (size_t)B * D;
  cudaError_t e = cudaMemsetAsync(rmax, 0, sizeof(float), stream);
  if (e != cudaSuccess) return (int)e;
  if (lstm) {
    if (bf16) uf_assemble_lstm<true><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
    else uf_assemble_lstm<false><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
    uf_scan_chunks<true><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
    uf_shard_total<true><<<uf_grid(BD), kUfThreads, 0, stream>>>(p, agg, last);
  } else {
    if (bf16) uf_assemble_gru<true><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
    else uf_assemble_gru<false><<<uf_grid(N), kUfThreads, 0, stream>>>(p);
    uf_scan_chunks<false><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
    uf_shard_total<false><<<uf_grid(BD), kUfThreads, 0, stream>>>(p, agg, last);
  }
  return (int)cudaGetLastError();
}

int shard_combine(int cell, const float* aggs, const float* lasts, int r, int B, int D,
                  float* din, float* bound, cudaStream_t stream) {
  const size_t BD = (size_t)B * D;
  if (cell == PARARNN_LSTM)
    uf_shard_combine<true><<<uf_grid(BD), kUfThreads, 0, stream>>>(aggs, lasts, r, B, D, din, bound);
  else
    uf_shard_combine<false><<<uf_grid(BD), kUfThreads, 0, stream>>>(aggs, lasts, r, B, D, din,
                                                                     bound);
  return (int)cudaGetLastError();
}

// Second half: the chunks re-run from their true carries, starting from the
// delta entering the shard, and the deltas added to the iterate.
int shard_apply(int cell, const float* din, float* c, float* h, int B, int Ts, int D,
                void* workspace, cudaStream_t stream) {
  UfParams p = uf_shard_params(cell, nullptr, nullptr, nullptr, nullptr, nullptr, c, h, B, Ts, D,
                               workspace);
  p.cin = din;
  const size_t M = (size_t)B * p.nC * D, BD = (size_t)B * D;
  if (cell == PARARNN_LSTM) {
    uf_scan_carry<true><<<uf_grid(BD), kUfThreads, 0, stream>>>(p);
    uf_scan_apply<true><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
  } else {
    uf_scan_carry<false><<<uf_grid(BD), kUfThreads, 0, stream>>>(p);
    uf_scan_apply<false><<<uf_grid(M), kUfThreads, 0, stream>>>(p);
  }
  return (int)cudaGetLastError();
}

}  // namespace pararnn
