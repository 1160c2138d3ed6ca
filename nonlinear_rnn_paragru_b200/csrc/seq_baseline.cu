// seq_baseline.cu -- naive step-by-step evaluation on the GPU, and the
// single-step update used for autoregressive decoding.
//
// One thread per (b, d) channel walks t = 1..T, applying the cell exactly as
// the sequential definition does ("Параллельность RNN?", §1.1: s_1 = f(s_0),
// s_2 = f(s_1), ...).  Lanes take consecutive channels so every load of u and
// every store of h is coalesced.  This is the reported baseline the parallel
// solve is compared with, not part of the solve.
//
// Decoding generates one token at a time, so its recurrent work per token is
// one update of the state, independent of the context length ("Apple научила
// классические RNN масштабироваться...", "Инференс быстрее и стабильнее по
// длине контекста", Figure 8).  The step kernels apply the same cell once,
// one thread per channel; the state may be updated in place (each thread
// reads its channel's state before writing it).
#include <cuda_bf16.h>

#include "common.cuh"

namespace pararnn {

template <bool kBF16>
__device__ __forceinline__ float load_u(const void* u, size_t i) {
  if constexpr (kBF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(u)[i]);
  else
    return reinterpret_cast<const float*>(u)[i];
}

__device__ __forceinline__ float sig(float x) { return rcp(1.f + ex2(-kLog2e * x)); }
__device__ __forceinline__ float tnh(float x) { return fmaf(-2.f, rcp(1.f + ex2(2.f * kLog2e * x)), 1.f); }

template <bool kBF16>
__global__ void gru_seq_kernel(const void* __restrict__ u, const float* __restrict__ a,
                               const float* __restrict__ bias, const float* __restrict__ h0,
                               float* __restrict__ h, int B, int T, int D) {
  const size_t ch = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (ch >= (size_t)B * D) return;
  const int b = (int)(ch / D), d = (int)(ch - (size_t)b * D);
  const float az = a[d], ar = a[D + d], ac = a[2 * D + d];
  const float bz = bias ? bias[d] : 0.f, br = bias ? bias[D + d] : 0.f,
              bc = bias ? bias[2 * D + d] : 0.f;
  float hp = h0 ? h0[ch] : 0.f;
  size_t iu = (size_t)b * T * 3 * D + d, ih = (size_t)b * T * D + d;
  for (int t = 0; t < T; ++t, iu += 3 * (size_t)D, ih += D) {
    const float uz = load_u<kBF16>(u, iu), ur = load_u<kBF16>(u, iu + D),
                uc = load_u<kBF16>(u, iu + 2 * (size_t)D);
    const float z = sig(fmaf(az, hp, uz + bz));
    const float r = sig(fmaf(ar, hp, ur + br));
    const float c = tnh(fmaf(ac, r * hp, uc + bc));
    hp = fmaf(z, c - hp, hp);
    h[ih] = hp;
  }
}

template <bool kBF16>
__global__ void lstm_seq_kernel(const void* __restrict__ u, const float* __restrict__ a,
                                const float* __restrict__ bias, const float* __restrict__ c0,
                                const float* __restrict__ h0, float* __restrict__ c,
                                float* __restrict__ h, int B, int T, int D) {
  const size_t ch = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (ch >= (size_t)B * D) return;
  const int b = (int)(ch / D), d = (int)(ch - (size_t)b * D);
  float aa[4], bb[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    aa[q] = a[q * D + d];
    bb[q] = bias ? bias[q * D + d] : 0.f;
  }
  float cp = c0 ? c0[ch] : 0.f, hp = h0 ? h0[ch] : 0.f;
  size_t iu = (size_t)b * T * 4 * D + d, ih = (size_t)b * T * D + d;
  for (int t = 0; t < T; ++t, iu += 4 * (size_t)D, ih += D) {
    const float gi = sig(fmaf(aa[0], hp, load_u<kBF16>(u, iu) + bb[0]));
    const float gf = sig(fmaf(aa[1], hp, load_u<kBF16>(u, iu + D) + bb[1]));
    const float gg = tnh(fmaf(aa[2], hp, load_u<kBF16>(u, iu + 2 * (size_t)D) + bb[2]));
    const float go = sig(fmaf(aa[3], hp, load_u<kBF16>(u, iu + 3 * (size_t)D) + bb[3]));
    cp = fmaf(gf, cp, gi * gg);
    hp = go * tnh(cp);
    c[ih] = cp;
    h[ih] = hp;
  }
}

// one step: u [B][3][D], state [B][D]; h_prev and h_next may be the same array
template <bool kBF16>
__global__ void gru_step_kernel(const void* __restrict__ u, const float* __restrict__ a,
                                const float* __restrict__ bias, const float* h_prev,
                                float* h_next, int B, int D) {
  const size_t ch = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (ch >= (size_t)B * D) return;
  const int b = (int)(ch / D), d = (int)(ch - (size_t)b * D);
  const size_t iu = (size_t)b * 3 * D + d;
  const float hp = h_prev ? h_prev[ch] : 0.f;
  const float z = sig(fmaf(a[d], hp, load_u<kBF16>(u, iu) + (bias ? bias[d] : 0.f)));
  const float r = sig(fmaf(a[D + d], hp, load_u<kBF16>(u, iu + D) + (bias ? bias[D + d] : 0.f)));
  const float c = tnh(fmaf(a[2 * D + d], r * hp,
                           load_u<kBF16>(u, iu + 2 * (size_t)D) + (bias ? bias[2 * D + d] : 0.f)));
  h_next[ch] = fmaf(z, c - hp, hp);
}

// one step: u [B][4][D], states [B][D]; *_prev and *_next may be the same arrays
template <bool kBF16>
__global__ void lstm_step_kernel(const void* __restrict__ u, const float* __restrict__ a,
                                 const float* __restrict__ bias, const float* c_prev,
                                 const float* h_prev, float* c_next, float* h_next, int B,
                                 int D) {
  const size_t ch = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (ch >= (size_t)B * D) return;
  const int b = (int)(ch / D), d = (int)(ch - (size_t)b * D);
  const size_t iu = (size_t)b * 4 * D + d;
  const float cp = c_prev ? c_prev[ch] : 0.f, hp = h_prev ? h_prev[ch] : 0.f;
  float pre[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    pre[q] = fmaf(a[q * D + d], hp,
                  load_u<kBF16>(u, iu + (size_t)q * D) + (bias ? bias[q * D + d] : 0.f));
  const float gi = sig(pre[0]), gf = sig(pre[1]), gg = tnh(pre[2]), go = sig(pre[3]);
  const float cn = fmaf(gf, cp, gi * gg);
  c_next[ch] = cn;
  h_next[ch] = go * tnh(cn);
}

int launch_decode_step(int cell, bool bf16, const void* u, const float* a, const float* bias,
                       const float* c_prev, const float* h_prev, float* c_next, float* h_next,
                       int B, int D, cudaStream_t stream) {
  const int threads = 128;
  const size_t n = (size_t)B * D;
  const unsigned grid = (unsigned)((n + threads - 1) / threads);
  if (cell == PARARNN_GRU) {
    if (bf16)
      gru_step_kernel<true><<<grid, threads, 0, stream>>>(u, a, bias, h_prev, h_next, B, D);
    else
      gru_step_kernel<false><<<grid, threads, 0, stream>>>(u, a, bias, h_prev, h_next, B, D);
  } else {
    if (bf16)
      lstm_step_kernel<true><<<grid, threads, 0, stream>>>(u, a, bias, c_prev, h_prev, c_next,
                                                           h_next, B, D);
    else
      lstm_step_kernel<false><<<grid, threads, 0, stream>>>(u, a, bias, c_prev, h_prev, c_next,
                                                            h_next, B, D);
  }
  return (int)cudaGetLastError();
}

int launch_seq_baseline(int cell, bool bf16, const void* u, const float* a, const float* bias,
                        const float* c0, const float* h0, float* c, float* h, int B, int T,
                        int D, cudaStream_t stream) {
  const int threads = 128;
  const size_t n = (size_t)B * D;
  const unsigned grid = (unsigned)((n + threads - 1) / threads);
  if (cell == PARARNN_GRU) {
    if (bf16)
      gru_seq_kernel<true><<<grid, threads, 0, stream>>>(u, a, bias, h0, h, B, T, D);
    else
      gru_seq_kernel<false><<<grid, threads, 0, stream>>>(u, a, bias, h0, h, B, T, D);
  } else {
    if (bf16)
      lstm_seq_kernel<true><<<grid, threads, 0, stream>>>(u, a, bias, c0, h0, c, h, B, T, D);
    else
      lstm_seq_kernel<false><<<grid, threads, 0, stream>>>(u, a, bias, c0, h0, c, h, B, T, D);
  }
  return (int)cudaGetLastError();
}

}  // namespace pararnn
