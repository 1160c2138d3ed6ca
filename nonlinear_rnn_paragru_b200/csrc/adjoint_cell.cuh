// adjoint_cell.cuh -- the ParaGRU cell of the 8-channel adjoint kernels
// (whole-sequence and segment-queue), evaluated on packed step pairs, and the
// layout of a chunk's staged inputs.
//
// A thread owns a 16-step chunk of one channel, taken as 8 step pairs
// (i, i + 8).  Per chunk three TMA boxes land in a 2304-byte slot: u (bf16
// rows [t][gate][8 ch], 19 steps), the states h_{t-1} (fp32, 20 steps) and
// dL/dh (fp32, 19 steps); chunk k of a warp is loaded k steps early and read at
// a k-row offset, so the four chunks a warp reads at one step fall in disjoint
// bank windows.
#pragma once
#include "common.cuh"

namespace pararnn {

constexpr int kArC = 8;                       // channels per tile
constexpr int kArK = 32 / kArC;               // chunks per warp
constexpr int kArL = 16;                      // steps per chunk
constexpr int kArH = kArL / 2;                // step pairs per chunk
constexpr int kArUStep = 3 * kArC * 2;        // 48 bytes per step of u
constexpr int kArSStep = kArC * 4;            // 32 bytes per step of h or dL/dh
constexpr int kArUBox = kArL + kArK - 1;      // 19 steps
constexpr int kArHBox = kArL + kArK;          // 20 steps (one more: h_{t-1})
constexpr int kArGBox = kArL + kArK - 1;      // 19 steps
constexpr int kArUOff = 0, kArHOff = 1024, kArGOff = 1664;
constexpr int kArS = 2304;                    // chunk slot
static_assert(kArUBox * kArUStep <= kArHOff && kArHOff + kArHBox * kArSStep <= kArGOff &&
                  kArGOff + kArGBox * kArSStep <= kArS && kArS % 128 == 0 &&
                  kArHOff % 128 == 0 && kArGOff % 128 == 0,
              "chunk slot layout");

__device__ __forceinline__ float2 af2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 afma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 amul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 aadd(float2 a, float2 b) { return __fadd2_rn(a, b); }

// affine map x -> P x + d, as float2 (P, d); (f o g)(x) = f(g(x))
__device__ __forceinline__ float2 ar_after(float2 f, float2 g) {
  return af2(f.x * g.x, fmaf(f.x, g.y, f.y));
}

struct ArCell {
  float2 AZ2, AR2, AC2, AZ, AR, AC;  // scaled (argument) and raw weights, both lanes
};

// The cell at a step pair: from the previous state HP and the pre-scaled
// arguments UZ, UR, UC, the Jacobian A = df/dh and the pieces
// GZ = df/du_z, GR = df/du_r, GC = df/du_c, RH = r h.  Each sigmoid and the
// tanh take their own ex2 and reciprocal, unclamped (a saturating argument
// gives the gate's limit, a NaN stays NaN): 2% faster in the queue adjoint
// than one reciprocal shared by a step pair's four sigmoids.
__device__ __forceinline__ void ar_cell(const ArCell& k, float2 HP, float2 UZ, float2 UR,
                                        float2 UC, float2& A, float2& GZ, float2& GR,
                                        float2& GC, float2& RH) {
  const float2 ONE = af2(1.f, 1.f), M1 = af2(-1.f, -1.f), M2 = af2(-2.f, -2.f);
  const float2 F4 = af2(4.f, 4.f), M4 = af2(-4.f, -4.f);
  const float2 TZ = afma(k.AZ2, HP, UZ), TR = afma(k.AR2, HP, UR);
  const float2 PZ = aadd(ONE, af2(ex2(TZ.x), ex2(TZ.y)));
  const float2 PR = aadd(ONE, af2(ex2(TR.x), ex2(TR.y)));
  const float2 Z = af2(rcp(PZ.x), rcp(PZ.y)), R = af2(rcp(PR.x), rcp(PR.y));
  RH = amul(R, HP);
  const float2 TC = afma(k.AC2, RH, UC);
  const float2 PC = aadd(ONE, af2(ex2(TC.x), ex2(TC.y)));
  const float2 TT = af2(rcp(PC.x), rcp(PC.y));
  const float2 C = afma(M2, TT, ONE);                 // tanh
  const float2 CMH = afma(HP, M1, C);
  const float2 OMZ = afma(Z, M1, ONE);
  const float2 ZZ = amul(Z, OMZ);                     // z(1-z)
  const float2 RR = amul(R, afma(R, M1, ONE));        // r(1-r)
  GZ = amul(CMH, ZZ);                                 // (c-h) z(1-z)
  GC = amul(Z, amul(TT, afma(TT, M4, F4)));           // z (1-c^2)
  const float2 GCA = amul(GC, k.AC);
  GR = amul(GCA, amul(HP, RR));                       // z(1-c^2) a_c h r(1-r)
  const float2 Q = afma(amul(k.AR, HP), RR, R);       // r + a_r h r(1-r)
  A = afma(GCA, Q, afma(amul(k.AZ, ZZ), CMH, OMZ));
}

// pre-scaled arguments of a step pair: -log2e u_z + b'_z, ... from bf16 rows
__device__ __forceinline__ void ar_args(const unsigned char* ux, const unsigned char* uy, float2 S,
                                        float2 BZ, float2 BR, float2 BC, float2& UZ, float2& UR,
                                        float2& UC) {
  const unsigned short* rx = reinterpret_cast<const unsigned short*>(ux);
  const unsigned short* ry = reinterpret_cast<const unsigned short*>(uy);
  const float2 SC = af2(2.f * kLog2e, 2.f * kLog2e);
  UZ = afma(S, af2(__uint_as_float((unsigned)rx[0] << 16), __uint_as_float((unsigned)ry[0] << 16)), BZ);
  UR = afma(S, af2(__uint_as_float((unsigned)rx[kArC] << 16),
                   __uint_as_float((unsigned)ry[kArC] << 16)), BR);
  UC = afma(SC, af2(__uint_as_float((unsigned)rx[2 * kArC] << 16),
                    __uint_as_float((unsigned)ry[2 * kArC] << 16)), BC);
}

// ---------------------------------------------------------------- ParaLSTM --
// A chunk's staged inputs for the ParaLSTM adjoints: u (bf16 [t][i f g o]
// [8 ch], 19 steps), c_{t-1} and h_{t-1} (fp32, 20 steps) and dL/dh (fp32,
// 19 steps) in a 3200-byte slot.  The u rows are 64 bytes, so chunks k and
// k + 2 of a warp share bank windows there (two-way); the 32-byte state rows
// are conflict-free as for ParaGRU.
constexpr int kAlUStep = 4 * kArC * 2;        // 64 bytes per step of u
constexpr int kAlUOff = 0, kAlCOff = 1280, kAlHOff = 1920, kAlGOff = 2560;
constexpr int kAlS = 3200;                    // chunk slot

struct AlCell {
  float2 AI2, AF2, AG2, AO2;  // h coefficients of the arguments (-log2e a; 2 log2e a for g)
  float2 AI, AF, AG, AO;      // raw weights
};

// The cell at a step pair from (CP, HP) = (c_{t-1}, h_{t-1}) and the
// pre-scaled arguments: the Jacobian entries A00 = f, A01 = X = dc'/dh,
// A10 = dh'/dc, A11 = dh'/dh, and the pieces of du: du_{i,f,g} = (gci, gcf,
// gcg) (lambda_c + kk lambda_h), du_o = dot lambda_h.  Each gate and
// tanh(c') takes its own ex2 and reciprocal, unclamped: a saturating argument
// gives 2^x = inf and a reciprocal of 0, the gate's limit, and a NaN stays
// NaN (one reciprocal shared by the six sigmoids of a step pair needed
// clamped arguments and a longer dependency chain: 4% slower).
__device__ __forceinline__ void al_cell(const AlCell& k, float2 CP, float2 HP, float2 UI,
                                        float2 UF, float2 UG, float2 UO, float2& F, float2& X,
                                        float2& KK, float2& A11, float2& GCI, float2& GCF,
                                        float2& GCG, float2& DOT) {
  const float2 ONE = af2(1.f, 1.f), M1 = af2(-1.f, -1.f), M2 = af2(-2.f, -2.f);
  const float2 F4 = af2(4.f, 4.f), M4 = af2(-4.f, -4.f);
  const float2 TL = af2(2.f * kLog2e, 2.f * kLog2e);
  auto e2 = [](float2 v) { return af2(ex2(v.x), ex2(v.y)); };
  auto rc = [](float2 v) { return af2(rcp(v.x), rcp(v.y)); };
  const float2 I = rc(aadd(ONE, e2(afma(k.AI2, HP, UI))));
  F = rc(aadd(ONE, e2(afma(k.AF2, HP, UF))));
  const float2 O = rc(aadd(ONE, e2(afma(k.AO2, HP, UO))));
  const float2 TG = rc(aadd(ONE, e2(afma(k.AG2, HP, UG))));
  const float2 G = afma(M2, TG, ONE);
  const float2 CN = afma(F, CP, amul(I, G));
  const float2 TC1 = rc(aadd(ONE, e2(amul(TL, CN))));
  const float2 TC = afma(M2, TC1, ONE);
  const float2 DI = amul(I, afma(I, M1, ONE));
  const float2 DF = amul(F, afma(F, M1, ONE));
  const float2 DO = amul(O, afma(O, M1, ONE));
  const float2 DG = amul(TG, afma(TG, M4, F4));       // 1 - g^2
  const float2 DT = amul(TC1, afma(TC1, M4, F4));     // 1 - tanh^2(c')
  GCI = amul(G, DI);
  GCF = amul(CP, DF);
  GCG = amul(I, DG);
  KK = amul(O, DT);
  DOT = amul(DO, TC);
  X = afma(GCF, k.AF, afma(GCI, k.AI, amul(GCG, k.AG)));
  A11 = afma(DOT, k.AO, amul(KK, X));
}

// pre-scaled arguments of a step pair from bf16 rows [i f g o][8 ch]
__device__ __forceinline__ void al_args(const unsigned char* ux, const unsigned char* uy,
                                        const float2 (&BS)[4], float2& UI, float2& UF,
                                        float2& UG, float2& UO) {
  const unsigned short* rx = reinterpret_cast<const unsigned short*>(ux);
  const unsigned short* ry = reinterpret_cast<const unsigned short*>(uy);
  const float2 S = af2(-kLog2e, -kLog2e), SG = af2(2.f * kLog2e, 2.f * kLog2e);
  auto ld = [&](int g) {
    return af2(__uint_as_float((unsigned)rx[g * kArC] << 16),
               __uint_as_float((unsigned)ry[g * kArC] << 16));
  };
  UI = afma(S, ld(0), BS[0]);
  UF = afma(S, ld(1), BS[1]);
  UG = afma(SG, ld(2), BS[2]);
  UO = afma(S, ld(3), BS[3]);
}

}  // namespace pararnn
