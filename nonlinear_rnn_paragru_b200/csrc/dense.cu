// dense.cu -- Newton solve for a general cell whose Jacobian is a full D x D
// matrix: the GRU with full recurrent matrices W_z, W_r, W_c.
//
// The pages derive the Newton step for any Markov cell: the Jacobian of the
// residual is block-bidiagonal, identities on the diagonal and -df/ds below
// it, a dense D x D block for a general cell ("Параллельность RNN?", §1.3),
// and the fully general solver of the pages works with such blocks ("Apple
// научила классические RNN масштабироваться...", "Три уровня
// производительности").  Cell (the reset gate on the recurrent term of the
// candidate):  z = sig(W_z h + u_z + b_z),  r = sig(W_r h + u_r + b_r),
// c = tanh(u_c + b_c + r (W_c h)),  h' = (1 - z) h + z c,  and
//   dh'/dh = diag(1 - z) + diag((c - h) z (1 - z)) W_z
//            + diag(z (1 - c^2)) [diag(r) W_c + diag((W_c h) r (1 - r)) W_r].
// Each Newton iteration, with the host checking the residual as in the
// unfused tier, runs (tensor-core path, the default):
//   pre-activations  Q = h W^T for every step: tcgen05 GEMMs of the states
//                    [B*T, D] by the stacked matrices [3D, D] (tc_gemm.cu) in
//                    split tf32 (three products of hi/lo parts), so they, the
//                    residual and the fixed point carry fp32 accuracy; W h0
//                    once per solve;
//   dn_assemble2     one CTA per (b, 8 steps, half of the rows): gates,
//                    residual, -r_t, the four coefficient vectors of J_t and
//                    the block J_t to HBM, row-major at odd positions of its
//                    16-step chunk and transposed at even ones;
//   chunk maps       each chunk's product J_15 ... J_0 as a tree of pairwise
//                    products, four levels of batched D x D tcgen05 GEMMs (left
//                    factor row-major, right factor transposed: both operands
//                    K-major; each level stores its products in the layout the
//                    next level reads them in);
//   dn_spass, dn_carry2, dn_spass
//                    the chunk offsets (every chunk's recurrence from a zero
//                    delta), the delta entering each chunk chunk by chunk
//                    (matrix-vector products with the chunk maps), and every
//                    chunk re-run from its delta, ds added to h; the two
//                    chunk passes take J_t through its structure, diag(co0)
//                    plus row-scaled W_z, W_c, W_r, all chains at once.
// The chunk maps' tf32 products make each Newton step inexact (about 1e-3
// relative); the residual is evaluated to fp32 accuracy, so the fixed point
// is that of the cell and the iteration still converges, linearly near the
// root.  The
// CUDA-core path (fp32 products, exact steps, D <= 128) is kept for
// comparison (PARARNN_FLAG_DENSE_SIMT): dn_pre, dn_assemble, dn_chunk_maps
// (a D x D x D product per step in shared memory), dn_carry, dn_apply.
// Layouts: u [B][T][3][D], W [3][D][D] row-major (row i of W_g feeds unit i),
// bias [3][D], h0 [B][D], h [B][T][D].  D <= 512.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace pararnn {

namespace {

constexpr int kDnThreads = 256;
constexpr int kDnChunk = 16;       // steps per scan chunk (four levels of pairwise products)
constexpr int kDnLevels = 4;
constexpr int kDnMaxDSimt = 128;   // three (D x (D+1)) fp32 tiles fit in shared memory
constexpr int kDnMaxD = 512;

template <bool kBF16>
__device__ __forceinline__ float dn_u(const void* u, size_t i) {
  if constexpr (kBF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(u)[i]);
  else
    return reinterpret_cast<const float*>(u)[i];
}

__device__ __forceinline__ float dn_sig(float x) { return 1.f / (1.f + expf(-x)); }

__device__ __forceinline__ unsigned dn_abs_bits(float v) {
  return isnan(v) ? 0x7fc00000u : __float_as_uint(fabsf(v));
}

struct DnParams {
  const void* u;
  const float *W, *bias, *h0;
  float* h;        // the iterate [B][T][D]
  float* Q;        // recurrent pre-activations [B][T][3][D]
  float* J;        // Jacobian blocks [B][T][D][D]
  float* rhs;      // -r [B][T][D]
  float* P;        // chunk maps [B][nC][D][D]
  float* d;        // chunk offsets [B][nC][D]
  float* carry;    // delta entering each chunk [B][nC][D]
  unsigned* rmax;  // residual maximum (ordered bits)
  int B, T, D, nC;
};

// ---------------------------------------------------------- pre-activations --
// Q[m][n] = sum_k S[m][k] W[n][k], m = b*T + t over the shifted states
// S[m] = h_{t-1} (h0 at t = 0), n over the 3D rows of W.  64 x 64 tiles, K in
// steps of 16, each thread a 4 x 4 block of outputs.
__global__ void __launch_bounds__(kDnThreads) dn_pre(const DnParams p) {
  __shared__ float As[16][64];
  __shared__ float Bs[16][64];
  const int M = p.B * p.T, N = 3 * p.D, K = p.D;
  const int m0 = blockIdx.x * 64, n0 = blockIdx.y * 64;  // rows on x: B*T may be large
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + r * kDnThreads;  // 0 .. 1023: 64 rows x 16 columns
      const int row = e / 16, col = e % 16;
      const int m = m0 + row, k = k0 + col;
      float a = 0.f;
      if (m < M && k < K) {
        const int b = m / p.T, t = m - b * p.T;
        a = t > 0 ? p.h[(size_t)(m - 1) * K + k] : (p.h0 ? p.h0[(size_t)b * K + k] : 0.f);
      }
      As[col][row] = a;
      const int n = n0 + row;
      Bs[col][row] = (n < N && k < K) ? p.W[(size_t)n * K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        w[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) p.Q[(size_t)m * N + n] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------- assemble --
template <bool kBF16>
__global__ void __launch_bounds__(kDnThreads) dn_assemble(const DnParams p) {
  __shared__ float co[4][kDnMaxD];  // per row i: 1 - z, (c - h) z (1 - z), z (1 - c^2) r, z (1 - c^2) q r (1 - r)
  __shared__ unsigned wmax[kDnThreads / 32];
  const int D = p.D;
  const size_t bt = blockIdx.x;  // b * T + t
  const int b = (int)(bt / p.T), t = (int)(bt - (size_t)b * p.T);
  unsigned m = 0;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const float hp = t > 0 ? p.h[(bt - 1) * D + i] : (p.h0 ? p.h0[(size_t)b * D + i] : 0.f);
    const size_t iu = bt * 3 * D + i;
    const float* q3 = p.Q + bt * 3 * D;
    const float z = dn_sig(q3[i] + dn_u<kBF16>(p.u, iu) + (p.bias ? p.bias[i] : 0.f));
    const float r = dn_sig(q3[D + i] + dn_u<kBF16>(p.u, iu + D) + (p.bias ? p.bias[D + i] : 0.f));
    const float q = q3[2 * D + i];
    const float c =
        tanhf(dn_u<kBF16>(p.u, iu + 2 * (size_t)D) + (p.bias ? p.bias[2 * D + i] : 0.f) + r * q);
    const float f = fmaf(z, c - hp, hp);
    const float res = p.h[bt * D + i] - f;
    p.rhs[bt * D + i] = -res;
    m = max(m, dn_abs_bits(res));
    const float gc = z * (1.f - c * c);
    co[0][i] = 1.f - z;
    co[1][i] = (c - hp) * z * (1.f - z);
    co[2][i] = gc * r;
    co[3][i] = gc * q * r * (1.f - r);
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned mm = 0;
    for (int w = 0; w < kDnThreads / 32; ++w) mm = max(mm, wmax[w]);
    atomicMax(p.rmax, mm);
  }
  const size_t DD = (size_t)D * D;
  float* Jt = p.J + bt * DD;
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e - i * D;
    Jt[e] = (i == j ? co[0][i] : 0.f) + co[1][i] * p.W[e] + co[2][i] * p.W[2 * DD + e] +
            co[3][i] * p.W[DD + e];
  }
}

// -------------------------------------------------------------------- scan --
// Shared memory of dn_chunk_maps: three D x (D + 1) tiles (J_t, P, the next
// P; the padding keeps column walks free of bank conflicts) and two D-vectors.
size_t dn_maps_smem(int D) { return ((size_t)3 * D * (D + 1) + 2 * (size_t)D) * 4; }
size_t dn_apply_smem(int D) { return ((size_t)D * (D + 1) + 2 * (size_t)D) * 4; }

// Loads J_t [D][D] into a padded shared tile.
__device__ __forceinline__ void dn_load_tile(float* dst, const float* src, int D) {
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e - i * D;
    dst[i * (D + 1) + j] = src[e];
  }
}

// One CTA per (b, chunk): the chunk's map x_out = P x_in + d.
__global__ void __launch_bounds__(kDnThreads) dn_chunk_maps(const DnParams p) {
  extern __shared__ float sm[];
  const int D = p.D, ld = D + 1;
  float* Js = sm;
  float* Pa = Js + (size_t)D * ld;
  float* Pb = Pa + (size_t)D * ld;
  float* xa = Pb + (size_t)D * ld;
  float* xb = xa + D;
  const int b = blockIdx.x / p.nC, k = blockIdx.x - b * p.nC;
  const int t0 = k * kDnChunk, t1 = min(p.T, t0 + kDnChunk);
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e - i * D;
    Pa[i * ld + j] = (i == j) ? 1.f : 0.f;
  }
  for (int i = threadIdx.x; i < D; i += blockDim.x) xa[i] = 0.f;
  for (int t = t0; t < t1; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    dn_load_tile(Js, p.J + bt * D * D, D);
    __syncthreads();
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
      const int i = e / D, j = e - i * D;
      float s = 0.f;
      for (int q = 0; q < D; ++q) s = fmaf(Js[i * ld + q], Pa[q * ld + j], s);
      Pb[i * ld + j] = s;
    }
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      float s = p.rhs[bt * D + i];
      for (int q = 0; q < D; ++q) s = fmaf(Js[i * ld + q], xa[q], s);
      xb[i] = s;
    }
    __syncthreads();
    float* tp = Pa;
    Pa = Pb;
    Pb = tp;
    float* tx = xa;
    xa = xb;
    xb = tx;
  }
  const size_t o = (size_t)blockIdx.x * D;  // (b * nC + k) * D
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e - i * D;
    p.P[o * D + e] = Pa[i * ld + j];
  }
  for (int i = threadIdx.x; i < D; i += blockDim.x) p.d[o + i] = xa[i];
}

// One CTA per b: the delta entering each chunk, chunk by chunk; a warp per
// row of the chunk map, so its loads are coalesced along the row.
__global__ void __launch_bounds__(kDnThreads) dn_carry(const DnParams p) {
  __shared__ float x[2][kDnMaxD];
  const int D = p.D, b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < D; i += blockDim.x) x[0][i] = 0.f;
  __syncthreads();
  int cur = 0;
  for (int k = 0; k < p.nC; ++k) {
    const size_t o = ((size_t)b * p.nC + k) * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) p.carry[o + i] = x[cur][i];
    for (int i = warp; i < D; i += kDnThreads / 32) {
      const float* Pi = p.P + (o + i) * D;
      float s = 0.f;
      for (int q = lane; q < D; q += 32) s = fmaf(Pi[q], x[cur][q], s);
#pragma unroll
      for (int sh = 16; sh > 0; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
      if (lane == 0) x[cur ^ 1][i] = s + p.d[o + i];
    }
    __syncthreads();
    cur ^= 1;
  }
}

// One CTA per (b, chunk): the chunk re-run from its carry; ds added to h.
__global__ void __launch_bounds__(kDnThreads) dn_apply(const DnParams p) {
  extern __shared__ float sm[];
  const int D = p.D, ld = D + 1;
  float* Js = sm;
  float* xa = Js + (size_t)D * ld;
  float* xb = xa + D;
  const int b = blockIdx.x / p.nC, k = blockIdx.x - b * p.nC;
  const int t0 = k * kDnChunk, t1 = min(p.T, t0 + kDnChunk);
  const size_t o = (size_t)blockIdx.x * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x) xa[i] = p.carry[o + i];
  for (int t = t0; t < t1; ++t) {
    const size_t bt = (size_t)b * p.T + t;
    dn_load_tile(Js, p.J + bt * D * D, D);
    __syncthreads();
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      float s = p.rhs[bt * D + i];
      for (int q = 0; q < D; ++q) s = fmaf(Js[i * ld + q], xa[q], s);
      xb[i] = s;
      p.h[bt * D + i] += s;
    }
    __syncthreads();
    float* tx = xa;
    xa = xb;
    xb = tx;
  }
}

// ------------------------------------------------------ tensor-core path --
struct Dn2Params {
  const void* u;
  const float *W, *Wt, *bias, *h0;
  float* h;        // the iterate [B][T][D]
  const float* Q;  // row b*T + t: W h_t, [B][T][3D]
  const float* Q0; // W h0 [B][3D] (zeros when h0 is absent)
  float* J;        // [B][Tp][D][D]: odd positions of a chunk row-major, even transposed
  const float* P;  // chunk maps [B][nC][D][D] row-major (the last tree level)
  float* rhs;      // -r [B][Tp][D], zero on padded steps
  // [B][Tp][4][D]: J_t = diag(co0) + diag(co1) W_z + diag(co2) W_c + diag(co3) W_r
  // (co0 = 1, the others 0 on padded steps)
  float* co;
  float* d;        // chunk offsets [B][nC][D]
  float* carry;    // delta entering each chunk [B][nC][D]
  unsigned* rmax;
  int B, T, D, nC, Tp;
};

// x = hi + lo with hi = x with the 13 low mantissa bits cleared (exactly the
// value a tf32 product reads) and lo = x - hi (exact in fp32).  A product
// hi_a hi_b + hi_a lo_b + lo_a hi_b then carries the fp32 product to about
// 2^-21 relative (the dropped lo_a lo_b and the tf32 reading of lo are below
// it): the split-tf32 technique, used here for the pre-activations, on which
// the residual and so the fixed point depend.
__global__ void dn_split(const float* __restrict__ x, float* __restrict__ hi,
                         float* __restrict__ lo, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    hi[i] = h;
    lo[i] = v - h;
  }
}

// W_g^T for each gate: Wt[g][j][i] = W[g][i][j]
__global__ void dn_transpose_w(const float* __restrict__ W, float* __restrict__ Wt, int D) {
  __shared__ float tile[32][33];
  const int g = blockIdx.z, i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const size_t off = (size_t)g * D * D;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = i0 + r, j = j0 + threadIdx.x;
    if (i < D && j < D) tile[r][threadIdx.x] = W[off + (size_t)i * D + j];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int j = j0 + r, i = i0 + threadIdx.x;
    if (i < D && j < D) Wt[off + (size_t)j * D + i] = tile[threadIdx.x][r];
  }
}

// One CTA per (b, eight consecutive padded steps t0..t0+7, half of the rows):
// gates from the pre-activations of h_{t-1}, residual, -r_t, the coefficients
// of J_t and, for its rows, J_t for each step; padded steps (t >= T) get J = I,
// -r = 0 and the identity's coefficients.  The four odd steps are stored
// row-major and the four even ones transposed, so every float4 of a W (Wt) row
// is loaded once for four steps.  The two CTAs of a step group compute the
// same gates; the one holding the first half of the rows stores the vectors.
constexpr int kDnAsm = 8;     // steps per assembly CTA (Tp is a multiple of 16)
constexpr int kDnAsmSplit = 2;  // CTAs per step group (row halves)
constexpr size_t kDnAsmSmem = (size_t)kDnAsm * 4 * kDnMaxD * 4;
template <bool kBF16>
__global__ void __launch_bounds__(kDnThreads) dn_assemble2(const Dn2Params p) {
  extern __shared__ __align__(16) float asm_sm[];
  float (*co)[4][kDnMaxD] = reinterpret_cast<float (*)[4][kDnMaxD]>(asm_sm);
  __shared__ unsigned wmax[kDnThreads / 32];
  const int D = p.D;
  const int groups = p.Tp / kDnAsm;
  const int half = (int)(blockIdx.x % kDnAsmSplit);
  const int gidx = (int)(blockIdx.x / kDnAsmSplit);
  const int b = gidx / groups, t0 = (gidx % groups) * kDnAsm;
  const bool vec_owner = half == 0;
  const size_t DD = (size_t)D * D;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned m = 0;
#pragma unroll 1
  for (int st = 0; st < kDnAsm; ++st) {
    const int t = t0 + st;
    const size_t bt = (size_t)b * p.Tp + t;
    if (t >= p.T) {
      if (vec_owner)
        for (int i = threadIdx.x; i < D; i += blockDim.x) {
          p.rhs[bt * D + i] = 0.f;
          p.co[(bt * 4 + 0) * D + i] = 1.f;
          p.co[(bt * 4 + 1) * D + i] = 0.f;
          p.co[(bt * 4 + 2) * D + i] = 0.f;
          p.co[(bt * 4 + 3) * D + i] = 0.f;
        }
      continue;
    }
    const size_t bs = (size_t)b * p.T + t;  // (b, t) in the unpadded arrays
    const float* q3 = t > 0 ? p.Q + (bs - 1) * 3 * D : p.Q0 + (size_t)b * 3 * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      const float hp = t > 0 ? p.h[(bs - 1) * D + i] : (p.h0 ? p.h0[(size_t)b * D + i] : 0.f);
      const size_t iu = bs * 3 * D + i;
      const float z = dn_sig(q3[i] + dn_u<kBF16>(p.u, iu) + (p.bias ? p.bias[i] : 0.f));
      const float r = dn_sig(q3[D + i] + dn_u<kBF16>(p.u, iu + D) + (p.bias ? p.bias[D + i] : 0.f));
      const float q = q3[2 * D + i];
      const float c =
          tanhf(dn_u<kBF16>(p.u, iu + 2 * (size_t)D) + (p.bias ? p.bias[2 * D + i] : 0.f) + r * q);
      const float f = fmaf(z, c - hp, hp);
      const float res = p.h[bs * D + i] - f;
      m = max(m, dn_abs_bits(res));
      const float gc = z * (1.f - c * c);
      const float c0 = 1.f - z, c1 = (c - hp) * z * (1.f - z), c2 = gc * r,
                  c3 = gc * q * r * (1.f - r);
      co[st][0][i] = c0;
      co[st][1][i] = c1;
      co[st][2][i] = c2;
      co[st][3][i] = c3;
      if (vec_owner) {
        p.rhs[bt * D + i] = -res;
        p.co[(bt * 4 + 0) * D + i] = c0;
        p.co[(bt * 4 + 1) * D + i] = c1;
        p.co[(bt * 4 + 2) * D + i] = c2;
        p.co[(bt * 4 + 3) * D + i] = c3;
      }
    }
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if (lane == 0) wmax[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0 && vec_owner) {
    unsigned mm = 0;
    for (int w = 0; w < kDnThreads / 32; ++w) mm = max(mm, wmax[w]);
    atomicMax(p.rmax, mm);
  }
  // J[i][j] = [i == j] (1 - z_i) + co1_i Wz[i][j] + co2_i Wc[i][j] + co3_i Wr[i][j];
  // a warp per stored row of this CTA's half, lanes along it in float4s
  // (coalesced, every load of the row in flight before the stores)
  constexpr int kQ4 = kDnMaxD / 128;
  constexpr int kPar = kDnAsm / 2;  // steps of one parity
  const int D4 = D >> 2;
  const int Dh = D / kDnAsmSplit, rlo = half * Dh, rhi = rlo + Dh;
#pragma unroll 1
  for (int parity = 1; parity >= 0; --parity) {  // odd steps row-major, even transposed
    const float* Wsrc = parity ? p.W : p.Wt;
    for (int row = rlo + warp; row < rhi; row += kDnThreads / 32) {
      float4 wz[kQ4], wr[kQ4], wc[kQ4];
#pragma unroll
      for (int k = 0; k < kQ4; ++k) {
        const int q4 = lane + 32 * k;
        if (q4 < D4) {
          const float4* base = reinterpret_cast<const float4*>(Wsrc + (size_t)row * D) + q4;
          wz[k] = __ldg(base);
          wr[k] = __ldg(base + DD / 4);
          wc[k] = __ldg(base + 2 * DD / 4);
        }
      }
#pragma unroll
      for (int k = 0; k < kQ4; ++k) {
        const int q4 = lane + 32 * k;
        if (q4 >= D4) continue;
#pragma unroll
        for (int which = 0; which < kPar; ++which) {
          const int s = parity + 2 * which;
          const bool valid = t0 + s < p.T;
          float* Jt = p.J + ((size_t)b * p.Tp + t0 + s) * DD;
          float4 o;
          if (!valid) {  // padded step: the identity
            o = make_float4(row == 4 * q4 ? 1.f : 0.f, row == 4 * q4 + 1 ? 1.f : 0.f,
                            row == 4 * q4 + 2 ? 1.f : 0.f, row == 4 * q4 + 3 ? 1.f : 0.f);
          } else if (parity) {  // row-major: element (row, j), row coefficients
            const float c1 = co[s][1][row], c2 = co[s][2][row], c3 = co[s][3][row];
            o.x = fmaf(c1, wz[k].x, fmaf(c2, wc[k].x, c3 * wr[k].x));
            o.y = fmaf(c1, wz[k].y, fmaf(c2, wc[k].y, c3 * wr[k].y));
            o.z = fmaf(c1, wz[k].z, fmaf(c2, wc[k].z, c3 * wr[k].z));
            o.w = fmaf(c1, wz[k].w, fmaf(c2, wc[k].w, c3 * wr[k].w));
            const int dj = row - 4 * q4;  // the diagonal element, if in this float4
            if (dj >= 0 && dj < 4) (&o.x)[dj] += co[s][0][row];
          } else {  // transposed: stored row j = row holds column j, element (i, j)
            const float4 c1 = reinterpret_cast<const float4*>(co[s][1])[q4];
            const float4 c2 = reinterpret_cast<const float4*>(co[s][2])[q4];
            const float4 c3 = reinterpret_cast<const float4*>(co[s][3])[q4];
            o.x = fmaf(c1.x, wz[k].x, fmaf(c2.x, wc[k].x, c3.x * wr[k].x));
            o.y = fmaf(c1.y, wz[k].y, fmaf(c2.y, wc[k].y, c3.y * wr[k].y));
            o.z = fmaf(c1.z, wz[k].z, fmaf(c2.z, wc[k].z, c3.z * wr[k].z));
            o.w = fmaf(c1.w, wz[k].w, fmaf(c2.w, wc[k].w, c3.w * wr[k].w));
            const int di = row - 4 * q4;
            if (di >= 0 && di < 4) (&o.x)[di] += co[s][0][row];
          }
          reinterpret_cast<float4*>(Jt + (size_t)row * D)[q4] = o;
        }
      }
    }
  }
}

// ---- the sequential passes, a cluster of CL CTAs per chain: CTA rank r owns
// the rows [r R, r R + R) of every matrix-vector product (R = D / CL), keeps the
// whole vector x in its shared memory, and sends its rows of the next x to
// every CTA of the cluster (distributed shared memory) before one cluster
// barrier per step.  Each chain reads its D x D matrices with CL SMs' worth
// of loads in flight instead of one.
namespace cgd = cooperative_groups;

struct DnVec {
  __align__(16) float x[2][kDnMaxD];  // the vector, double-buffered by step parity
  float part[2 * kDnMaxD];   // transposed layout: partial sums of the q groups, [qg][row]
};

// y[i] = sum_q M[i][q] x[q] + add[i] for this CTA's rows i in [r0, r0 + R),
// M row-major or stored transposed (M[q][i]); the result goes to x_next of
// every CTA of the cluster.  Ends with the cluster barrier.
__device__ __forceinline__ void dn_cmatvec(cgd::cluster_group& cl, DnVec& v, int cur,
                                           const float* __restrict__ M, bool rowmajor,
                                           const float* __restrict__ add, int D, int r0, int R,
                                           float* __restrict__ yout) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float* x = v.x[cur];
  float* y_local = v.x[cur ^ 1];
  const int ncl = (int)cl.num_blocks();
  if (rowmajor) {
    // a warp per row, lanes along it in float4s, four rows at a time: every
    // lane has its 4 x (D / 128) loads in flight before the first fma (the
    // chain reads a fresh D x D matrix each step, so the pass is bound by
    // how many loads are in flight)
    constexpr int kRows = 4, kQ4 = kDnMaxD / 128;
    const int D4 = D >> 2;
    const float4* x4 = reinterpret_cast<const float4*>(x);
    for (int i0 = warp * kRows; i0 < R; i0 += (kDnThreads / 32) * kRows) {
      float4 mv[kRows][kQ4];
#pragma unroll
      for (int rr = 0; rr < kRows; ++rr)
#pragma unroll
        for (int k = 0; k < kQ4; ++k) {
          const int q4 = lane + 32 * k;
          mv[rr][k] = (i0 + rr < R && q4 < D4)
                          ? __ldg(reinterpret_cast<const float4*>(M + (size_t)(r0 + i0 + rr) * D) + q4)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      float s[kRows];
#pragma unroll
      for (int rr = 0; rr < kRows; ++rr) {
        s[rr] = 0.f;
#pragma unroll
        for (int k = 0; k < kQ4; ++k) {
          const int q4 = lane + 32 * k;
          if (q4 < D4) {
            const float4 xv = x4[q4];
            s[rr] = fmaf(mv[rr][k].x, xv.x, s[rr]);
            s[rr] = fmaf(mv[rr][k].y, xv.y, s[rr]);
            s[rr] = fmaf(mv[rr][k].z, xv.z, s[rr]);
            s[rr] = fmaf(mv[rr][k].w, xv.w, s[rr]);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s[rr] += __shfl_xor_sync(0xffffffffu, s[rr], o);
      }
      if (lane < kRows && i0 + lane < R) {
        float sv = s[0];
#pragma unroll
        for (int rr = 1; rr < kRows; ++rr)
          if (lane == rr) sv = s[rr];
        const int i = r0 + i0 + lane;
        sv += add ? add[i] : 0.f;
        for (int r = 0; r < ncl; ++r) cl.map_shared_rank(y_local, r)[i] = sv;
        if (yout) yout[i] = sv;
      }
    }
  } else {  // threads over (row offset, quarter of q): rows contiguous in M[q][.]
    const int nq = kDnThreads / R >= 4 ? 4 : (kDnThreads / R >= 2 ? 2 : 1);
    const int qlen = (D + nq - 1) / nq;
    for (int e = threadIdx.x; e < R * nq; e += kDnThreads) {
      const int ii = e % R, qg = e / R;
      const int i = r0 + ii;
      const int q0 = qg * qlen, q1 = min(D, q0 + qlen);
      // eight independent sums, so that eight loads are in flight
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int q = q0;
      for (; q + 8 <= q1; q += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) s8[u] = fmaf(__ldg(M + (size_t)(q + u) * D + i), x[q + u], s8[u]);
      }
      for (; q < q1; ++q) s8[0] = fmaf(__ldg(M + (size_t)q * D + i), x[q], s8[0]);
      v.part[qg * R + ii] = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
    }
    __syncthreads();
    for (int ii = threadIdx.x; ii < R; ii += kDnThreads) {
      const int i = r0 + ii;
      float s = add ? add[i] : 0.f;
      for (int qg = 0; qg < nq; ++qg) s += v.part[qg * R + ii];
      for (int r = 0; r < ncl; ++r) cl.map_shared_rank(y_local, r)[i] = s;
      if (yout) yout[i] = s;
    }
  }
  cl.sync();
}

// One cluster per b: the delta entering each chunk, chunk by chunk
// (x <- P_k x + d_k).
__global__ void __launch_bounds__(kDnThreads) dn_carry2(const Dn2Params p) {
  __shared__ DnVec v;
  cgd::cluster_group cl = cgd::this_cluster();
  const int D = p.D, ncl = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int R = D / ncl, r0 = rank * R;
  const int b = blockIdx.x / ncl;
  for (int i = threadIdx.x; i < D; i += blockDim.x) v.x[0][i] = 0.f;
  cl.sync();
  int cur = 0;
  for (int k = 0; k < p.nC; ++k) {
    const size_t o = (size_t)b * p.nC + k;
    for (int ii = threadIdx.x; ii < R; ii += blockDim.x) p.carry[o * D + r0 + ii] = v.x[cur][r0 + ii];
    dn_cmatvec(cl, v, cur, p.P + o * D * D, true, p.d + o * D, D, r0, R, nullptr);
    cur ^= 1;
  }
}

// ---- the chunks' recurrences through the structure of J_t, for all chains
// at once.  J_t x = co0 x + co1 (W_z x) + co2 (W_c x) + co3 (W_r x): the
// three products with x take the stacked recurrent matrices, the same for
// every step, so a step of every chain is one product of W by the matrix of
// the chains' deltas, and a step reads 4 D coefficients instead of the D x D
// block.  One persistent CTA per SM owns up to 4 channels i (rows i of W_z,
// W_r, W_c, held in shared memory k-major); per step it stages the chains'
// deltas (X[j][chain], chains innermost) in blocks of 64 chains, its warps
// take eighths of k and their partial sums are added in warp order, and each
// thread finishes one (channel, chain) of the block.  A grid barrier (bounded
// wait) separates the steps.  Offsets: from a zero delta, the last step's
// delta is the chunk offset; apply: from the delta entering the chunk, every
// step's delta added to h.
constexpr int kSpCpc = 4;                    // channels per CTA, at most
constexpr int kSpCb = 64;                    // chains per staged block
constexpr int kSpThreads = 512;
constexpr int kSpKg = kSpThreads / 32;       // k groups (warps)
struct SpParams {
  Dn2Params p;
  float* X;             // [2][D][nchp] chain deltas, chains innermost
  unsigned* bar;        // grid barrier arrivals (zero at launch)
  int* err;             // set when a barrier wait runs out
  int cpc, nch, nchp;   // channels per CTA, chains (B * nC), padded to 4
  uint64_t timeout_ns;
};
constexpr size_t kSpSmem =
    (size_t)(kDnMaxD * 3 * kSpCpc + kDnMaxD * kSpCb + kSpKg * 6 * kSpCpc * 32) * 4;

// every CTA's stores before this point are visible to every CTA after it;
// false when the wait ran out
__device__ __forceinline__ bool sp_grid_sync(unsigned* bar, unsigned target, uint64_t timeout_ns) {
  __shared__ int ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
    int good = 1;
    if (ld_acquire(bar) < target) {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire(bar) < target) {
        if (globaltimer_ns() - t0 > timeout_ns) {
          good = 0;
          break;
        }
      }
    }
    __threadfence();
    ok = good;
  }
  __syncthreads();
  return ok != 0;
}

template <bool kApply>
__global__ void __launch_bounds__(kSpThreads, 1) dn_spass(const SpParams s) {
  extern __shared__ __align__(16) float sp_sm[];
  const Dn2Params& p = s.p;
  const int D = p.D, nch = s.nch, nchp = s.nchp, cpc = s.cpc;
  float* Ws = sp_sm;                            // [D][3][kSpCpc]
  float* Xs = Ws + kDnMaxD * 3 * kSpCpc;        // [D][kSpCb]
  float* part = Xs + kDnMaxD * kSpCb;           // [kSpKg][2][3][kSpCpc][32]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i0 = blockIdx.x * cpc;
  const unsigned G = gridDim.x;
  // this CTA's rows of W_z, W_r, W_c, k-major (rows past D or cpc: zero)
  for (int e = tid; e < D * 3 * kSpCpc; e += kSpThreads) {
    const int k = e / (3 * kSpCpc), rem = e % (3 * kSpCpc), m = rem / kSpCpc, il = rem % kSpCpc;
    const int i = i0 + il;
    Ws[e] = (il < cpc && i < D) ? p.W[((size_t)m * D + i) * D + k] : 0.f;
  }
  // the deltas entering the chunks: zero (offsets) or the carries (apply)
  float* X0 = s.X;
  for (int e = tid; e < cpc * nch; e += kSpThreads) {
    const int il = e / nch, cg = e % nch, i = i0 + il;
    if (i < D) X0[(size_t)i * nchp + cg] = kApply ? p.carry[(size_t)cg * D + i] : 0.f;
  }
  unsigned round = 1;
  if (!sp_grid_sync(s.bar, round * G, s.timeout_ns)) {
    if (tid == 0) atomicExch(s.err, 1);
    return;
  }
  const int kq = (D + kSpKg - 1) / kSpKg, k0 = warp * kq, k1 = min(D, k0 + kq);
  for (int pp = 0; pp < kDnChunk; ++pp) {
    const float* Xc = s.X + (size_t)(pp & 1) * D * nchp;
    float* Xn = s.X + (size_t)((pp & 1) ^ 1) * D * nchp;
    for (int cb0 = 0; cb0 < nch; cb0 += kSpCb) {
      const int ncb = min(kSpCb, nchp - cb0);    // a multiple of 4
      // this thread's output (channel il, chain c of the block): its
      // coefficients and -r loaded now, used after the products
      const int oil = tid / kSpCb, oc = tid % kSpCb;  // threads past 4 x 64: none
      const int oi = i0 + oil, ocg = cb0 + oc;
      const bool own = oil < cpc && oi < D && ocg < nch;
      const int ob = own ? ocg / p.nC : 0, okc = own ? ocg - ob * p.nC : 0;
      const int ot = okc * kDnChunk + pp;
      const size_t obt = (size_t)ob * p.Tp + ot;
      float cf0 = 0.f, cf1 = 0.f, cf2 = 0.f, cf3 = 0.f, orhs = 0.f;
      if (own) {
        const float* cof = p.co + obt * 4 * D + oi;
        cf0 = cof[0];
        cf1 = cof[D];
        cf2 = cof[2 * D];
        cf3 = cof[3 * D];
        orhs = p.rhs[obt * D + oi];
      }
      // stage X[.][cb0, cb0 + ncb) (float4s, L2: other CTAs wrote it)
      const int n4 = ncb >> 2;
#pragma unroll 16
      for (int e = tid; e < D * n4; e += kSpThreads) {
        const int j = e / n4, c4 = e % n4;
        const float4 v = __ldcg(reinterpret_cast<const float4*>(Xc + (size_t)j * nchp + cb0) + c4);
        reinterpret_cast<float4*>(Xs + j * kSpCb)[c4] = v;
      }
      __syncthreads();
      // y[m][il][c] over this warp's k range, chains lane and lane + 32
      float acc[2][3][kSpCpc];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int m = 0; m < 3; ++m)
#pragma unroll
          for (int il = 0; il < kSpCpc; ++il) acc[h2][m][il] = 0.f;
#pragma unroll 4
      for (int k = k0; k < k1; ++k) {
        const float xa = Xs[k * kSpCb + lane], xb = Xs[k * kSpCb + 32 + lane];
        const float4* w4 = reinterpret_cast<const float4*>(Ws + k * 3 * kSpCpc);
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          const float4 w = w4[m];
          acc[0][m][0] = fmaf(w.x, xa, acc[0][m][0]);
          acc[0][m][1] = fmaf(w.y, xa, acc[0][m][1]);
          acc[0][m][2] = fmaf(w.z, xa, acc[0][m][2]);
          acc[0][m][3] = fmaf(w.w, xa, acc[0][m][3]);
          acc[1][m][0] = fmaf(w.x, xb, acc[1][m][0]);
          acc[1][m][1] = fmaf(w.y, xb, acc[1][m][1]);
          acc[1][m][2] = fmaf(w.z, xb, acc[1][m][2]);
          acc[1][m][3] = fmaf(w.w, xb, acc[1][m][3]);
        }
      }
      float* pw = part + (size_t)warp * 2 * 3 * kSpCpc * 32;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
        for (int m = 0; m < 3; ++m)
#pragma unroll
          for (int il = 0; il < kSpCpc; ++il)
            pw[((h2 * 3 + m) * kSpCpc + il) * 32 + lane] = acc[h2][m][il];
      __syncthreads();
      // the thread's output: the warps' sums in order, then J_t x - r_t
      if (own) {
        const int h2 = oc >> 5, ln = oc & 31;
        float y3[3];
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          float sum = 0.f;
          for (int w = 0; w < kSpKg; ++w)
            sum += part[(size_t)w * 2 * 3 * kSpCpc * 32 + ((h2 * 3 + m) * kSpCpc + oil) * 32 + ln];
          y3[m] = sum;
        }
        const float x = Xs[oi * kSpCb + oc];
        // W rows: 0 = W_z, 1 = W_r, 2 = W_c
        const float y = fmaf(cf0, x, fmaf(cf1, y3[0], fmaf(cf2, y3[2], fmaf(cf3, y3[1], orhs))));
        Xn[(size_t)oi * nchp + ocg] = y;
        if (kApply) {
          if (ot < p.T) p.h[((size_t)ob * p.T + ot) * D + oi] += y;
        } else if (pp == kDnChunk - 1) {
          p.d[(size_t)ocg * D + oi] = y;
        }
      }
      __syncthreads();
    }
    if (pp + 1 < kDnChunk) {
      ++round;
      if (!sp_grid_sync(s.bar, round * G, s.timeout_ns)) {
        if (tid == 0) atomicExch(s.err, 1);
        return;
      }
    }
  }
}

// CTAs per chain of the sequential passes: D / 64, from 1 to 8, dividing D
int dn_cluster(int D) {
  for (int c = 8; c > 1; c /= 2)
    if (D % (8 * c) == 0 && D / c >= 64) return c;
  return 1;
}

// `wide`: a pass with few chains (the carry chain, one per b) takes clusters
// of 16 CTAs (a non-portable size) where the device can hold one per chain,
// so that twice as many SMs read each step's matrix
template <class K>
cudaError_t dn_launch_cluster(K kern, unsigned chains, int D, const Dn2Params& p,
                              cudaStream_t stream, bool wide = false) {
  int cl = dn_cluster(D);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kDnThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (wide && D % (8 * 16) == 0 && D / 16 >= 32 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess) {
    attr[0].val.clusterDim.x = 16;
    cfg.gridDim = dim3(chains * 16u);
    int fit = 0;
    if (cudaOccupancyMaxActiveClusters(&fit, kern, &cfg) == cudaSuccess && fit >= (int)chains)
      cl = 16;
  }
  cudaGetLastError();
  attr[0].val.clusterDim.x = cl;
  cfg.gridDim = dim3(chains * (unsigned)cl);
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// A structured pass, launched cooperatively (all its CTAs resident: its
// steps are separated by grid barriers), its barrier count zeroed first.
cudaError_t sp_launch(bool apply, const SpParams& sp, unsigned grid, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(sp.bar, 0, sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  SpParams a = sp;
  void* args[] = {&a};
  return cudaLaunchCooperativeKernel(apply ? (const void*)dn_spass<true> : (const void*)dn_spass<false>,
                                     dim3(grid), dim3(kSpThreads), args, kSpSmem, stream);
}

struct DnLayout {
  size_t rmax, Q, J, rhs, P, d, carry, total;
};

// tensor-core path workspace: [0, 256) residual maximum and the GEMMs' error
// flag, then W^T, Q, W h0, the level-0 blocks, tree levels 1..4, -r, d, carry
struct Dn2Layout {
  size_t Wt, Wsp, hsp, h0sp, Q, Q0, J, lvl[kDnLevels], rhs, d, carry, co, X, total;
};

Dn2Layout dn2_layout(int B, int T, int D) {
  const size_t nC = (size_t)(T + kDnChunk - 1) / kDnChunk, Tp = nC * kDnChunk;
  const size_t DD = (size_t)D * D;
  Dn2Layout L;
  L.Wt = 256;
  L.Wsp = L.Wt + align256(3 * DD * 4);                       // W hi, lo
  L.hsp = L.Wsp + 2 * align256(3 * DD * 4);                  // h hi, lo
  L.h0sp = L.hsp + 2 * align256((size_t)B * T * D * 4);      // h0 hi, lo
  L.Q = L.h0sp + 2 * align256((size_t)B * D * 4);
  L.Q0 = L.Q + align256((size_t)B * T * 3 * D * 4);
  L.J = L.Q0 + align256((size_t)B * 3 * D * 4);
  size_t o = L.J + align256((size_t)B * Tp * DD * 4);
  for (int l = 0; l < kDnLevels; ++l) {
    L.lvl[l] = o;
    o += align256((size_t)B * (Tp >> (l + 1)) * DD * 4);
  }
  L.rhs = o;
  L.d = L.rhs + align256((size_t)B * Tp * D * 4);
  L.carry = L.d + align256((size_t)B * nC * D * 4);
  L.co = L.carry + align256((size_t)B * nC * D * 4);
  L.X = L.co + align256((size_t)B * Tp * 4 * D * 4);
  const size_t nchp = ((size_t)B * nC + 3) & ~size_t(3);
  L.total = L.X + align256(2 * (size_t)D * nchp * 4);
  return L;
}

DnLayout dn_layout(int B, int T, int D) {
  const size_t BT = (size_t)B * T, nC = (size_t)(T + kDnChunk - 1) / kDnChunk;
  const size_t BC = (size_t)B * nC;
  DnLayout L;
  L.rmax = 0;
  L.Q = 256;
  L.J = L.Q + align256(BT * 3 * D * 4);
  L.rhs = L.J + align256(BT * D * D * 4);
  L.P = L.rhs + align256(BT * D * 4);
  L.d = L.P + align256(BC * D * D * 4);
  L.carry = L.d + align256(BC * D * 4);
  L.total = L.carry + align256(BC * D * 4);
  return L;
}

}  // namespace

int tc_operand_map(CUtensorMap* map, const float* base, int K, int rows, int Z, long long zstride);
int launch_tc_gemm(const CUtensorMap& ma, const CUtensorMap& mb, float* C, int M, int N, int K,
                   int Z, int store_mode, int* err, cudaStream_t stream);

int dense_max_d(bool simt) { return simt ? kDnMaxDSimt : kDnMaxD; }
size_t dense_ws_bytes(int B, int T, int D) {
  return std::max(dn_layout(B, T, D).total, dn2_layout(B, T, D).total);
}

namespace {
// Tensor-core path; see the file comment.
int dense_solve_tc(bool bf16, const void* u, const float* W, const float* bias, const float* h0,
                   float* h, int B, int T, int D, float tol, int max_iters, pararnn_stats* stats,
                   void* workspace, cudaStream_t stream) {
  const Dn2Layout L = dn2_layout(B, T, D);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  Dn2Params p;
  p.u = u;
  p.W = W;
  p.Wt = reinterpret_cast<float*>(ws + L.Wt);
  p.bias = bias;
  p.h0 = h0;
  p.h = h;
  float* Q = reinterpret_cast<float*>(ws + L.Q);
  float* Q0 = reinterpret_cast<float*>(ws + L.Q0);
  p.Q = Q;
  p.Q0 = Q0;
  p.J = reinterpret_cast<float*>(ws + L.J);
  p.P = reinterpret_cast<float*>(ws + L.lvl[kDnLevels - 1]);
  p.rhs = reinterpret_cast<float*>(ws + L.rhs);
  p.co = reinterpret_cast<float*>(ws + L.co);
  p.d = reinterpret_cast<float*>(ws + L.d);
  p.carry = reinterpret_cast<float*>(ws + L.carry);
  p.rmax = reinterpret_cast<unsigned*>(ws);
  int* err = reinterpret_cast<int*>(ws + 4);
  p.B = B;
  p.T = T;
  p.D = D;
  p.nC = (T + kDnChunk - 1) / kDnChunk;
  p.Tp = p.nC * kDnChunk;
  const size_t BT = (size_t)B * T, DD = (size_t)D * D;
  const int nprod0 = B * p.Tp;  // level-0 blocks

  // operand maps: the states and h0 against the stacked matrices; per tree
  // level, odd blocks (left factors) against even ones (right factors)
  // split-tf32 operands of the pre-activations: h, W and h0 as hi + lo
  float* Whi = reinterpret_cast<float*>(ws + L.Wsp);
  float* Wlo = reinterpret_cast<float*>(ws + L.Wsp + align256(3 * DD * 4));
  float* hhi = reinterpret_cast<float*>(ws + L.hsp);
  float* hlo = reinterpret_cast<float*>(ws + L.hsp + align256(BT * D * 4));
  float* h0hi = reinterpret_cast<float*>(ws + L.h0sp);
  float* h0lo = reinterpret_cast<float*>(ws + L.h0sp + align256((size_t)B * D * 4));
  CUtensorMap mhh, mhl, mh0h, mh0l, mwh, mwl, ml[kDnLevels], mr[kDnLevels];
  int rc = tc_operand_map(&mhh, hhi, D, (int)BT, 1, (long long)BT * D);
  rc |= tc_operand_map(&mhl, hlo, D, (int)BT, 1, (long long)BT * D);
  rc |= tc_operand_map(&mwh, Whi, D, 3 * D, 1, 3LL * DD);
  rc |= tc_operand_map(&mwl, Wlo, D, 3 * D, 1, 3LL * DD);
  if (h0) {
    rc |= tc_operand_map(&mh0h, h0hi, D, B, 1, (long long)B * D);
    rc |= tc_operand_map(&mh0l, h0lo, D, B, 1, (long long)B * D);
  }
  for (int l = 0; l < kDnLevels; ++l) {
    const float* in = l == 0 ? p.J : reinterpret_cast<float*>(ws + L.lvl[l - 1]);
    const int nout = nprod0 >> (l + 1);
    rc |= tc_operand_map(&ml[l], in + DD, D, D, nout, 2LL * DD);
    rc |= tc_operand_map(&mr[l], in, D, D, nout, 2LL * DD);
  }
  if (rc) return (int)cudaErrorInvalidValue;

  cudaError_t e = cudaMemsetAsync(h, 0, BT * D * 4, stream);  // initial guess: zero
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, 8, stream);  // residual maximum, error flag
  if (e != cudaSuccess) return (int)e;
  dn_transpose_w<<<dim3((D + 31) / 32, (D + 31) / 32, 3), dim3(32, 8), 0, stream>>>(
      W, reinterpret_cast<float*>(ws + L.Wt), D);
  const unsigned sgrid = 8 * 148;
  dn_split<<<sgrid, 256, 0, stream>>>(W, Whi, Wlo, 3 * DD);
  // C = A B^T to fp32 accuracy from split operands: hi hi, then + hi lo, + lo hi
  auto split_gemm = [&](const CUtensorMap& ah, const CUtensorMap& al, float* C, int M) {
    int r = launch_tc_gemm(ah, mwh, C, M, 3 * D, D, 1, 0, err, stream);
    if (!r) r = launch_tc_gemm(ah, mwl, C, M, 3 * D, D, 1, 3, err, stream);
    if (!r) r = launch_tc_gemm(al, mwh, C, M, 3 * D, D, 1, 3, err, stream);
    return r;
  };
  int ge = 0;
  if (h0) {
    dn_split<<<sgrid, 256, 0, stream>>>(h0, h0hi, h0lo, (size_t)B * D);
    ge = split_gemm(mh0h, mh0l, Q0, B);
  } else {
    e = cudaMemsetAsync(Q0, 0, (size_t)B * 3 * D * 4, stream);
  }
  if (ge) return ge;
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  // the structured passes: one CTA per SM, up to 4 channels each
  SpParams sp;
  sp.p = p;
  sp.X = reinterpret_cast<float*>(ws + L.X);
  sp.bar = reinterpret_cast<unsigned*>(ws + 8);
  sp.err = err;
  sp.nch = B * p.nC;
  sp.nchp = (sp.nch + 3) & ~3;
  sp.timeout_ns = 1000000000ull;
  unsigned sgrid_sp = 0;
  {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sp.cpc = std::min(kSpCpc, (D + sms - 1) / sms);
    sgrid_sp = (unsigned)((D + sp.cpc - 1) / sp.cpc);
    e = cudaFuncSetAttribute(dn_assemble2<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDnAsmSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(dn_assemble2<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kDnAsmSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(dn_spass<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSpSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(dn_spass<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSpSmem);
    if (e != cudaSuccess) return (int)e;
  }
  pararnn_stats st = {0, 0.f, PARARNN_STATUS_CONVERGED, 0};
  for (int k = 0;; ++k) {
    e = cudaMemsetAsync(p.rmax, 0, sizeof(unsigned), stream);
    if (e != cudaSuccess) return (int)e;
    dn_split<<<sgrid, 256, 0, stream>>>(h, hhi, hlo, BT * D);
    ge = split_gemm(mhh, mhl, Q, (int)BT);
    if (ge) return ge;
    const unsigned nblk = (unsigned)((size_t)B * (p.Tp / kDnAsm) * kDnAsmSplit);
    if (bf16)
      dn_assemble2<true><<<nblk, kDnThreads, kDnAsmSmem, stream>>>(p);
    else
      dn_assemble2<false><<<nblk, kDnThreads, kDnAsmSmem, stream>>>(p);
    unsigned hdr[2] = {0u, 0u};
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return (int)e;
    if (hdr[1] != 0u) {  // a tensor-core GEMM's wait ran out
      st.status = PARARNN_STATUS_TIMEOUT;
      break;
    }
    float r;
    std::memcpy(&r, &hdr[0], sizeof r);  // the ordered bits are the float's own
    st.evals = k + 1;
    st.max_residual = r;
    if (!(r == r) || hdr[0] >= 0x7f800000u) {  // NaN or inf
      st.status = PARARNN_STATUS_NONFINITE;
      break;
    }
    if (k == max_iters) {  // residual-only evaluation at the cap
      if (!(r < tol)) st.status = PARARNN_STATUS_NOT_CONVERGED;
      break;
    }
    // chunk maps: four levels of pairwise block products
    for (int l = 0; l < kDnLevels; ++l) {
      float* out = reinterpret_cast<float*>(ws + L.lvl[l]);
      ge = launch_tc_gemm(ml[l], mr[l], out, D, D, D, nprod0 >> (l + 1),
                          l + 1 < kDnLevels ? 2 : 0, err, stream);
      if (ge) return ge;
    }
    e = sp_launch(false, sp, sgrid_sp, stream);
    if (e == cudaSuccess) e = dn_launch_cluster(dn_carry2, (unsigned)B, D, p, stream, true);
    if (e == cudaSuccess) e = sp_launch(true, sp, sgrid_sp, stream);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    st.iters = k + 1;
    if (r < tol) break;  // the update of the first certified iteration is applied
  }
  e = cudaMemcpyAsync(stats, &st, sizeof(st), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // st lives on this stack
  return (int)e;
}
}  // namespace

// The host-driven loop; arguments are validated by the caller.  Writes
// *stats (device) at the end.  Returns 0 or a CUDA error.
int dense_gru_solve(bool bf16, bool simt, const void* u, const float* W, const float* bias,
                    const float* h0, float* h, int B, int T, int D, float tol, int max_iters,
                    pararnn_stats* stats, void* workspace, cudaStream_t stream) {
  if (!simt)
    return dense_solve_tc(bf16, u, W, bias, h0, h, B, T, D, tol, max_iters, stats, workspace,
                          stream);
  const DnLayout L = dn_layout(B, T, D);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  DnParams p;
  p.u = u;
  p.W = W;
  p.bias = bias;
  p.h0 = h0;
  p.h = h;
  p.Q = reinterpret_cast<float*>(ws + L.Q);
  p.J = reinterpret_cast<float*>(ws + L.J);
  p.rhs = reinterpret_cast<float*>(ws + L.rhs);
  p.P = reinterpret_cast<float*>(ws + L.P);
  p.d = reinterpret_cast<float*>(ws + L.d);
  p.carry = reinterpret_cast<float*>(ws + L.carry);
  p.rmax = reinterpret_cast<unsigned*>(ws + L.rmax);
  p.B = B;
  p.T = T;
  p.D = D;
  p.nC = (T + kDnChunk - 1) / kDnChunk;
  const size_t BT = (size_t)B * T;
  const unsigned nmaps = (unsigned)((size_t)B * p.nC);
  const size_t sm_maps = dn_maps_smem(D), sm_apply = dn_apply_smem(D);
  cudaError_t e = cudaFuncSetAttribute(dn_chunk_maps, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm_maps);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dn_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm_apply);
  if (e == cudaSuccess) e = cudaMemsetAsync(h, 0, BT * D * 4, stream);  // initial guess: zero
  if (e != cudaSuccess) return (int)e;
  const dim3 pre_grid((unsigned)((BT + 63) / 64), (unsigned)((3 * D + 63) / 64));
  pararnn_stats st = {0, 0.f, PARARNN_STATUS_CONVERGED, 0};
  for (int k = 0;; ++k) {
    e = cudaMemsetAsync(p.rmax, 0, sizeof(unsigned), stream);
    if (e != cudaSuccess) return (int)e;
    dn_pre<<<pre_grid, kDnThreads, 0, stream>>>(p);
    if (bf16)
      dn_assemble<true><<<(unsigned)BT, kDnThreads, 0, stream>>>(p);
    else
      dn_assemble<false><<<(unsigned)BT, kDnThreads, 0, stream>>>(p);
    unsigned bits = 0;
    e = cudaGetLastError();
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(&bits, p.rmax, sizeof(unsigned), cudaMemcpyDeviceToHost, stream);
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
    dn_chunk_maps<<<nmaps, kDnThreads, sm_maps, stream>>>(p);
    dn_carry<<<(unsigned)B, kDnThreads, 0, stream>>>(p);
    dn_apply<<<nmaps, kDnThreads, sm_apply, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    st.iters = k + 1;
    if (r < tol) break;  // the update of the first certified iteration is applied
  }
  e = cudaMemcpyAsync(stats, &st, sizeof(st), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);  // st lives on this stack
  return (int)e;
}

}  // namespace pararnn
