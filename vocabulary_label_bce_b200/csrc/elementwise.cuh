// Per-logit BCE math of the tile engine, two logits at a time.
//
// For a logit z (section III-A, Eq. (2) of "Cut Binary Cross Entropy"):
//   u = e^{-|z|} in (0, 1],   w = 1 + u in (1, 2]
//   l(z, 0) = max(z, 0) + log(1 + e^{-|z|}) = max(z, 0) + ln 2 * log2(w)
//   sigmoid(z) = 1 / w  (z >= 0),   u / w  (z < 0)      (Eq. (4): G = sigmoid(Z) - Y)
//
// Pipe budget on B200 (measured with the library's pipe probes): the SFU
// (ex2, rcp, lg2, tanh) retires 16 results per clock per SM, the FMA pipe 128,
// so one SFU operation costs as much as eight FMAs.  Each logit therefore gets
// exactly one SFU operation (the exponential); the reciprocal runs on the FMA
// pipe, and the logarithm is taken once per 32 logits of a row as the log2 of
// the product of their w (each factor is in (1, 2], so 32 of them stay finite).
//
// Reciprocal, on the FMA pipe: a seed, then the cubically convergent step
// r1 = r0 (1 + e + e^2) with e = 1 - w r0, which leaves |1 - w r1| = |e|^3.
//  * item pass, w in (1, 2]: linear minimax seed (24 - 8 w) / 17, |e| <= 1/17,
//    so |1 - w r1| <= 2.1e-4;
//  * gradient-only passes, w in (1, 2^100]: exponent-flip seed
//    r0 = bits^-1(C - bits(w)) (the integer subtraction negates the exponent
//    and roughly reflects the mantissa; with C = 0x7EF31000, |e| <= 0.0506 for
//    every normal w), so |1 - w r1| <= 1.3e-4.
// Both seeds are formed from -w, which the FMA pipe produces in the same
// instruction as 1 + u (bits(-w) = bits(w) + 2^31 for the integer seed).
//
// Gradient-only passes move a share of their exponentials to the FMA pipe as
// well (exp2_poly3_pair below).
//
// Packed fp32x2 instructions (two lanes of work per instruction) halve the
// issue slots of the FMA-pipe part; the SFU and the selects stay scalar.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>
#include "ptx_sm100.cuh"

namespace cutbce {

constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kLn2F = 0.6931471805599453f;
constexpr uint32_t kRcpSeedNeg = 0x7EF31000u + 0x80000000u;   // C + 2^31: seed from bits(-w)

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// 1 / w from nw = -w (w normal and positive): seed plus cubic step, |rel err| <= 1.3e-4.
__device__ __forceinline__ float2 rcp2_cubic(float2 nw) {
  float2 r = f2(__uint_as_float(kRcpSeedNeg - __float_as_uint(nw.x)),
                __uint_as_float(kRcpSeedNeg - __float_as_uint(nw.y)));
  const float2 e = __ffma2_rn(nw, r, f2(1.f, 1.f));    // 1 - w r0
  const float2 t = __ffma2_rn(e, e, e);                // e + e^2
  return __ffma2_rn(r, t, r);                          // r0 (1 + e + e^2)
}

// 1 / w for w in [1, 2] from nw = -w: linear minimax seed r0 = (24 - 8 w) / 17
// (|rel err| <= 1/17), one FFMA2 instead of two integer subtractions, then the
// cubic step: |rel err| <= (1/17)^3 = 2.1e-4.
__device__ __forceinline__ float2 rcp2_unit_interval(float2 nw) {
  float2 r = __ffma2_rn(nw, f2(8.f / 17.f, 8.f / 17.f), f2(24.f / 17.f, 24.f / 17.f));
  const float2 e = __ffma2_rn(nw, r, f2(1.f, 1.f));    // 1 - w r0
  const float2 t = __ffma2_rn(e, e, e);                // e + e^2
  return __ffma2_rn(r, t, r);                          // r0 (1 + e + e^2)
}

// Item-owned pass, loss and gradient: returns sigmoid(z) for both logits and
// folds their loss terms into the running products `prod` (of w, sign-free
// over an even count of factors per component) and the running sum `relu`
// of max(z, 0).  z log2 e is formed for both logits in one packed multiply;
// the exponential takes -|.| of it as operand modifiers.
__device__ __forceinline__ float2 bce_pair_loss_grad(float2 z, float2& prod, float2& relu) {
  const float2 tz = __fmul2_rn(z, f2(kLog2eF, kLog2eF));
  const float2 u = f2(ex2_approx(-fabsf(tz.x)), ex2_approx(-fabsf(tz.y)));   // e^{-|z|}
  const float2 nw = __ffma2_rn(u, f2(-1.f, -1.f), f2(-1.f, -1.f));           // -(1 + u)
  prod = __fmul2_rn(prod, nw);
  relu = __fadd2_rn(relu, f2(fmaxf(z.x, 0.f), fmaxf(z.y, 0.f)));
  const float2 r = rcp2_unit_interval(nw);
  const float2 ur = __fmul2_rn(u, r);
  return f2(z.x >= 0.f ? r.x : ur.x, z.y >= 0.f ? r.y : ur.y);
}

// Item-owned pass, loss only.
__device__ __forceinline__ void bce_pair_loss(float2 z, float2& prod, float2& relu) {
  const float2 tz = __fmul2_rn(z, f2(kLog2eF, kLog2eF));
  const float2 u = f2(ex2_approx(-fabsf(tz.x)), ex2_approx(-fabsf(tz.y)));
  prod = __fmul2_rn(prod, __fadd2_rn(u, f2(1.f, 1.f)));
  relu = __fadd2_rn(relu, f2(fmaxf(z.x, 0.f), fmaxf(z.y, 0.f)));
}

// 1 for every normal x > 0, 0 for x <= 0 (and for a subnormal x, flushed to 0):
// the Cut Metrics decision, on the FMA pipe.
__device__ __forceinline__ float positive_mask(float x) {
  float r;
  asm("mul.rn.ftz.sat.f32 %0, %1, %2;" : "=f"(r) : "f"(x), "f"(0x1p126f));
  return r;
}

// 2^x for x in [-100, 100] on the FMA pipe: x = j + f with j = rint(x) taken from
// the low mantissa bits of x + 1.5 * 2^23, f in [-1/2, 1/2]; 2^f by a degree-3
// polynomial fitted by a Remez exchange for minimum relative error on
// [-1/2, 1/2] (max relative error 7.5e-5, float32 Horner included); the
// exponent j is added to the result's exponent field with one integer
// multiply-add (bits(x + 1.5 * 2^23) * 2^23 keeps j's low 9 bits, two's
// complement, and the polynomial's exponent is -1 or 0).
__device__ __forceinline__ float2 exp2_poly3_pair(float2 x) {
  constexpr float kShift = 12582912.0f;   // 1.5 * 2^23
  const float2 j = __fadd2_rn(x, f2(kShift, kShift));
  const float2 jr = __fadd2_rn(j, f2(-kShift, -kShift));             // rint(x), exact
  const float2 f = __ffma2_rn(jr, f2(-1.f, -1.f), x);                // x - rint(x), exact
  float2 p = __ffma2_rn(f2(0.0551716685f, 0.0551716685f), f, f2(0.2426111251f, 0.2426111251f));
  p = __ffma2_rn(p, f, f2(0.6932609677f, 0.6932609677f));
  p = __ffma2_rn(p, f, f2(0.9999280572f, 0.9999280572f));
  uint32_t rx, ry;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(rx) : "r"(__float_as_uint(j.x)), "r"(1u << 23), "r"(__float_as_uint(p.x)));
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(ry) : "r"(__float_as_uint(j.y)), "r"(1u << 23), "r"(__float_as_uint(p.y)));
  return f2(__uint_as_float(rx), __uint_as_float(ry));
}

// Pairs of every 16 (one 32-logit chunk) whose exponential the gradient-only
// passes evaluate on the FMA pipe instead of the SFU.  The SFU retires 16
// exponentials per clock per SM and the polynomial costs about four more issue
// slots than the SFU instruction, so only a small share moves (the best of
// 0, 1, 2, 3 and 4 of 16 measured on the position-owned pass).
constexpr int kPolyPairsPerChunk = 2;

// Gradient only (the position-owned pass, and the item pass without the loss):
// sigmoid(z) = 1 / (1 + 2^x), x = -z log2 e clamped to [-100, 100] as
// 200 * saturate(-z log2 e / 200 + 1/2) - 100 on the FMA pipe (error <= 200 *
// 2^-25 in x, 4e-6 relative in 2^x); below z = -69.3 the result is 2^-100
// instead of a smaller positive number.  2^x from the SFU, or (kPoly) from the
// FMA-pipe polynomial; then the exponent-flip seed and the cubic step
// (|rel err| <= 1.3e-4).  Total relative error <= 2.1e-4 plus rounding, well
// inside the bf16 rounding of G that follows (up to 2^-9).
template <bool kPoly>
__device__ __forceinline__ float2 sigmoid_pair(float2 z) {
  float ax, ay;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(ax) : "f"(z.x), "f"(-kLog2eF / 200.f), "f"(0.5f));
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(ay) : "f"(z.y), "f"(-kLog2eF / 200.f), "f"(0.5f));
  const float2 x = __ffma2_rn(f2(ax, ay), f2(200.f, 200.f), f2(-100.f, -100.f));
  const float2 v = kPoly ? exp2_poly3_pair(x) : f2(ex2_approx(x.x), ex2_approx(x.y));
  const float2 nw = __ffma2_rn(v, f2(-1.f, -1.f), f2(-1.f, -1.f));   // -(1 + v)
  return rcp2_cubic(nw);
}

}  // namespace cutbce
