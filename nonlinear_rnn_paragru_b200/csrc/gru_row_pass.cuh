// gru_row_pass.cuh -- the ParaGRU cell pass of the 8-channel row kernels
// (whole-sequence / clustered solve and the segment-queue solve).
//
// A thread owns a 32-step chunk of one channel: its iterate h and running
// Jacobian product P in registers as 16 packed pairs (step i, step i + 16).
// The tile's gate arguments are fp32 in shared memory, pre-scaled with the
// bias folded in (-log2e u_z + b'_z, -log2e u_r + b'_r, 2 log2e u_c + b'_c),
// laid out per chunk as [gate][pair i][channel] {step i, step i + 16} with
// channel c at slot c ^ row_swizzle(i) of its pair row.
#pragma once
#include "common.cuh"

namespace pararnn {

constexpr int kRowC = 8;                     // channels per tile
constexpr int kRowK = 32 / kRowC;            // chunks per warp
constexpr int kRowL = 32;                    // steps per chunk (per thread)
constexpr int kRowH = kRowL / 2;             // step pairs per chunk
constexpr int kRowS = 3 * kRowL * kRowC * 4 + 64;     // chunk slot: 3072 bytes + 64
constexpr int kRowBox = 256;                          // steps per TMA box
constexpr int kRowBoxBytes = kRowBox * 3 * kRowC * 2;  // 12288
constexpr float kRowLn2 = 0.693147180559945309f;

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// channel slot of channel c in pair row i is c ^ row_swizzle(i)
__host__ __device__ constexpr int row_swizzle(int i) { return (i >> 1) & 7; }

// One pass over a chunk of 2 kH steps: H[i] = (h_i, h_{i+kH}) is the iterate, hb the state
// before the chunk.  With kFull the two half-chunks are scanned from a zero
// incoming delta: H becomes the local solution, P the running products, and
// DL / PA the halves' (delta out, product).  Returns max |h_t - f_t|.
// AZ2, AR2, AC2: the h coefficients of the three arguments (-log2e a_z,
// -log2e a_r, 2 log2e a_c); AZ = a_z.
template <int kH, bool kFull>
__device__ __forceinline__ float row_pass(const unsigned char* __restrict__ base, int c8, float hb,
                                          float2 (&H)[kH], float2 (&P)[kH], float2 AZ2,
                                          float2 AR2, float2 AC2, float2 AZ, float2& DLo,
                                          float2& PAo) {
  const float2 ONE = f2(1.f, 1.f), M1 = f2(-1.f, -1.f), M2 = f2(-2.f, -2.f);
  // a_r = -ln2 AR2 and 4 a_c = 2 ln2 AC2: the constants ride on r(1-r), t(1-t)
  const float2 NL = f2(-kRowLn2, -kRowLn2), PL = f2(kRowLn2, kRowLn2);
  const float2 TL = f2(2.f * kRowLn2, 2.f * kRowLn2), MTL = f2(-2.f * kRowLn2, -2.f * kRowLn2);
  float m = 0.f;
  float2 DL = f2(0.f, 0.f), PA = ONE;
  float2 HP = f2(hb, H[kH - 1].x);  // states before steps 0 and 16
  static_assert(kH % 2 == 0, "the pass takes its step pairs two at a time");
#pragma unroll
  for (int i = 0; i < kH; i += 2) {
    // two step pairs at a time: the gates of both, then one reciprocal for
    // the four tanh factors, then their Jacobians and scan steps
    float2 HPs[2], HTs[2], Z2[2], R2[2], PC2[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int ii = i + j;
      const unsigned char* bi = base + ((c8 ^ (row_swizzle(ii) * 8)) + ii * kRowC * 8);
      const float2 UZ = *reinterpret_cast<const float2*>(bi);
      const float2 UR = *reinterpret_cast<const float2*>(bi + 1 * kH * kRowC * 8);
      const float2 UC = *reinterpret_cast<const float2*>(bi + 2 * kH * kRowC * 8);
      const float2 hp = j == 0 ? HP : HTs[0];
      HPs[j] = hp;
      HTs[j] = H[ii];
      // z, r = 1/(1+e) with e = 2^(argument).  One reciprocal serves the four
      // sigmoids of a pair and one the four tanh of two pairs: every argument
      // is clamped at 31, so a product of four (1+e) stays below 2^124 (the
      // clamp moves a sigmoid or tanh by under 1e-9).
      const float2 TZ = ffma2(AZ2, hp, UZ), TR = ffma2(AR2, hp, UR);
      const float2 EZ = f2(ex2(fmin_nan(TZ.x, 31.f)), ex2(fmin_nan(TZ.y, 31.f)));
      const float2 ER = f2(ex2(fmin_nan(TR.x, 31.f)), ex2(fmin_nan(TR.y, 31.f)));
      const float2 PZ = fadd2(ONE, EZ), PR = fadd2(ONE, ER);
      const float2 PP = fmul2(PZ, PR);
      const float inv = rcp(PP.x * PP.y);
      const float2 INV = f2(PP.y * inv, PP.x * inv);        // 1/(pz pr) per step
      Z2[j] = fmul2(PR, INV);
      R2[j] = fmul2(PZ, INV);
      const float2 TC = ffma2(AC2, fmul2(R2[j], hp), UC);
      const float2 EC = f2(ex2(fmin_nan(TC.x, 31.f)), ex2(fmin_nan(TC.y, 31.f)));  // e^{2y}
      PC2[j] = fadd2(ONE, EC);
    }
    const float w0 = PC2[0].x * PC2[0].y, w1 = PC2[1].x * PC2[1].y;
    const float ic = rcp(w0 * w1);
    const float i0 = w1 * ic, i1 = w0 * ic;                  // 1/w0, 1/w1
    const float2 TTs[2] = {f2(PC2[0].y * i0, PC2[0].x * i0),
                           f2(PC2[1].y * i1, PC2[1].x * i1)};  // t = 1/(1+e^{2y})
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int ii = i + j;
      const float2 hp = HPs[j], HT = HTs[j], Z = Z2[j], R = R2[j], TT = TTs[j];
      const float2 C = ffma2(M2, TT, ONE);                  // tanh(y) = 1 - 2t
      const float2 CMH = ffma2(hp, M1, C);
      const float2 F = ffma2(Z, CMH, hp);
      const float2 DF = ffma2(F, M1, HT);
      m = fmax3_nan(m, fabsf(DF.x), fabsf(DF.y));
      if (kFull) {
        // A = (1-z) + a_z z(1-z)(c-h) + (1-c^2) z a_c (r + a_r h r(1-r)),
        // with 1-c^2 = 4t(1-t)
        const float2 OMZ = ffma2(Z, M1, ONE);
        const float2 A1 = ffma2(fmul2(AZ, fmul2(Z, OMZ)), CMH, OMZ);
        const float2 T1 = fmul2(TT, ffma2(TT, MTL, TL));   // 2 ln2 t(1-t)
        const float2 S = fmul2(fmul2(Z, T1), AC2);
        const float2 RR = fmul2(R, ffma2(R, PL, NL));      // -ln2 r(1-r)
        const float2 Q = ffma2(fmul2(AR2, hp), RR, R);
        const float2 A = ffma2(S, Q, A1);
        const float2 HN = ffma2(A, DL, F);
        DL = ffma2(HT, M1, HN);
        PA = fmul2(PA, A);
        H[ii] = HN;
        P[ii] = PA;
      }
    }
    HP = HTs[1];
  }
  DLo = DL;
  PAo = PA;
  return m;
}

// The pass of row_pass<kH, true> with every gate from the one-instruction
// tanh: sigma(x) = 1/2 + 1/2 tanh(x/2), c = tanh(y).  The stored arguments
// are -log2e x (z, r) and 2 log2e y (c), so x/2 and y are those times -ln2/2
// and ln2/2.  An inexact evaluation (gates within about 2^-11 relative) for
// the Newton iterations far from the root: the fixed point is fixed by the
// residual alone ("Параллельность RNN?", §1.2), so the solve takes these
// while the residual is large and decides convergence on exact evaluations
// only.  Same arguments and results as row_pass<kH, true>.
template <int kH>
__device__ __forceinline__ float row_pass_apx(const unsigned char* __restrict__ base, int c8,
                                              float hb, float2 (&H)[kH], float2 (&P)[kH],
                                              float2 AZ2, float2 AR2, float2 AC2, float2 AZ,
                                              float2& DLo, float2& PAo) {
  const float2 ONE = f2(1.f, 1.f), M1 = f2(-1.f, -1.f), HALF = f2(0.5f, 0.5f);
  const float2 KG = f2(-0.5f * kRowLn2, -0.5f * kRowLn2), KC = f2(0.5f * kRowLn2, 0.5f * kRowLn2);
  const float2 MKC = f2(-0.5f * kRowLn2, -0.5f * kRowLn2);
  // a_r = -ln2 AR2 and a_c = ln2/2 AC2: the constants ride on r(1-r), 1-c^2
  const float2 NL = f2(-kRowLn2, -kRowLn2), PL = f2(kRowLn2, kRowLn2);
  float m = 0.f;
  float2 DL = f2(0.f, 0.f), PA = ONE;
  float2 HP = f2(hb, H[kH - 1].x);  // states before steps 0 and 16
#pragma unroll
  for (int i = 0; i < kH; ++i) {
    const unsigned char* bi = base + ((c8 ^ (row_swizzle(i) * 8)) + i * kRowC * 8);
    const float2 UZ = *reinterpret_cast<const float2*>(bi);
    const float2 UR = *reinterpret_cast<const float2*>(bi + 1 * kH * kRowC * 8);
    const float2 UC = *reinterpret_cast<const float2*>(bi + 2 * kH * kRowC * 8);
    const float2 HT = H[i];
    const float2 XZ = fmul2(ffma2(AZ2, HP, UZ), KG), XR = fmul2(ffma2(AR2, HP, UR), KG);  // x/2
    const float2 Z = ffma2(HALF, f2(tanh_apx(XZ.x), tanh_apx(XZ.y)), HALF);
    const float2 R = ffma2(HALF, f2(tanh_apx(XR.x), tanh_apx(XR.y)), HALF);
    const float2 Y = fmul2(ffma2(AC2, fmul2(R, HP), UC), KC);                         // y
    const float2 C = f2(tanh_apx(Y.x), tanh_apx(Y.y));
    const float2 CMH = ffma2(HP, M1, C);
    const float2 F = ffma2(Z, CMH, HP);
    const float2 DF = ffma2(F, M1, HT);
    m = fmax3_nan(m, fabsf(DF.x), fabsf(DF.y));
    // A = (1-z) + a_z z(1-z)(c-h) + (1-c^2) z a_c (r + a_r h r(1-r))
    const float2 OMZ = ffma2(Z, M1, ONE);
    const float2 A1 = ffma2(fmul2(AZ, fmul2(Z, OMZ)), CMH, OMZ);
    const float2 OMC = ffma2(fmul2(C, MKC), C, KC);      // ln2/2 (1 - c^2)
    const float2 S = fmul2(fmul2(Z, OMC), AC2);
    const float2 RR = fmul2(R, ffma2(R, PL, NL));        // -ln2 r(1-r)
    const float2 Q = ffma2(fmul2(AR2, HP), RR, R);
    const float2 A = ffma2(S, Q, A1);
    const float2 HN = ffma2(A, DL, F);
    DL = ffma2(HT, M1, HN);
    PA = fmul2(PA, A);
    H[i] = HN;
    P[i] = PA;
    HP = HT;
  }
  DLo = DL;
  PAo = PA;
  return m;
}

}  // namespace pararnn
