// Per-logit BCE math of the tile engine, two logits at a time.
//
// For a logit z (section III-A, Eq. (2) of "Cut Binary Cross Entropy"):
//   l(z, 0) = max(z, 0) + log(1 + e^{-|z|})
//   sigmoid(z) = 1 / (1 + e^{-z})      (Eq. (4): G = sigmoid(Z) - Y)
//
// Pipe budget on B200 (measured with the library's pipe probes): the SFU
// (ex2, rcp, tanh, lg2) retires 16 results per clock per SM, the FMA pipe 128,
// and the SM issues one warp instruction per clock per sub-partition, so a
// packed fp32x2 FMA-pipe instruction does two lanes of work in one issue slot.
// The passes are bound by issue slots and the SFU, so each logit gets exactly
// one SFU operation and as few issued instructions as the accuracy allows.
// The tensor-core tiles hold zh = z / 2 (the compacted H is stored halved,
// exactly), which is the argument of the tanh below; the functions here take zh.
//
//  * passes with the loss (with or without the gradient): one tanh per logit.
//    With t = tanh(zh): sigmoid(z) = (1 + t)/2, and w = 1 + |t| = 2 sigmoid(|z|),
//    which is in [1, 2], so l(z, 0) = max(z, 0) + ln 2 - ln w.  The log is
//    taken once per tile slab of a row (up to 64 logits), as log2 of the
//    product of their w, and
//    max(z, 0) = z / 2 + |z| / 2: the tiles sum |z| / 2, the linear z / 2 is
//    summed over the whole problem as one dot product of column sums.
//  * gradient only: sigmoid(z) = (1 + tanh(z/2))/2 from one tanh, except for
//    two pairs in 16, whose sigmoid runs wholly on the FMA pipe (an FMA-pipe
//    2^x and a reciprocal by seed and cubic step) to take load off the SFU.
//
// tanh.approx.f32 is measured on B200 by the library's element-math self test
// (cutbce_selftest_element_math) over [-40, 40]: sigmoid from it is within
// 4.0e-6 of the exact value, ln w within 4.4e-6, and the mean error of ln w
// over z ~ N(0, 1) is 4e-8 of the mean element loss; the bf16 rounding of G
// that follows is up to 2^-9 relative.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>
#include "ptx_sm100.cuh"

namespace cutbce {

constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kLn2F = 0.6931471805599453f;
constexpr uint32_t kRcpSeedNeg = 0x7EF31000u + 0x80000000u;   // C + 2^31: seed from bits(-w)

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// 1 / w from nw = -w (w normal and positive) on the FMA pipe: the exponent-flip
// seed r0 = bits^-1(C - bits(w)), C = 0x7EF31000 (the integer subtraction
// negates the exponent and roughly reflects the mantissa: |1 - w r0| <= 0.0506
// for every normal w), formed from -w since bits(-w) = bits(w) + 2^31; then the
// cubically convergent step r1 = r0 (1 + e + e^2), e = 1 - w r0, which leaves
// |1 - w r1| = |e|^3 <= 1.3e-4.
__device__ __forceinline__ float2 rcp2_cubic(float2 nw) {
  float2 r = f2(__uint_as_float(kRcpSeedNeg - __float_as_uint(nw.x)),
                __uint_as_float(kRcpSeedNeg - __float_as_uint(nw.y)));
  const float2 e = __ffma2_rn(nw, r, f2(1.f, 1.f));    // 1 - w r0
  const float2 t = __ffma2_rn(e, e, e);                // e + e^2
  return __ffma2_rn(r, t, r);                          // r0 (1 + e + e^2)
}

// Passes with the loss and the gradient (the item-owned pass, and the
// position-owned pass when it takes the weighted loss): returns sigmoid(z) for
// both logits (zh = z / 2) and folds their loss terms into the running product
// `prod` of w = 1 + |tanh(zh)| and the running sum `absz` of |zh| = |z| / 2 (the
// other half of max(z, 0) = z / 2 + |z| / 2 is linear in z and summed once,
// from column sums, by the finish).
__device__ __forceinline__ float2 bce_pair_loss_grad(float2 zh, float2& prod, float2& absz) {
  const float2 t = f2(tanh_approx(zh.x), tanh_approx(zh.y));
  prod = __fmul2_rn(prod, f2(1.f + fabsf(t.x), 1.f + fabsf(t.y)));
  absz.x += fabsf(zh.x);
  absz.y += fabsf(zh.y);
  return __ffma2_rn(t, f2(0.5f, 0.5f), f2(0.5f, 0.5f));
}

// Loss only (the forward): the same terms as bce_pair_loss_grad, so that the
// forward and the fused call give the same loss bit for bit.
__device__ __forceinline__ void bce_pair_loss(float2 zh, float2& prod, float2& absz) {
  const float2 t = f2(tanh_approx(zh.x), tanh_approx(zh.y));
  prod = __fmul2_rn(prod, f2(1.f + fabsf(t.x), 1.f + fabsf(t.y)));
  absz.x += fabsf(zh.x);
  absz.y += fabsf(zh.y);
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

// Pairs of every 16 (one 32-logit chunk) whose sigmoid the gradient-only
// passes evaluate wholly on the FMA pipe instead of from the SFU's tanh.  The
// FMA-pipe path costs about ten more issue slots a pair, so only a small share
// moves (the best of 0 to 3 of 16, measured on the position-owned pass).
constexpr int kPolyPairsPerChunk = 2;

// Gradient only, on the FMA pipe alone, from zh = z / 2:
// sigmoid(z) = 1 / (1 + 2^x), x = -z log2 e clamped to [-100, 100] as
// 200 * saturate(-zh (2 log2 e) / 200 + 1/2) - 100 (the same bits as with z and
// log2 e / 200: both factors are scaled by exact powers of two; error <= 200 * 2^-25 in x,
// 4e-6 relative in 2^x); below z = -69.3 the result is 2^-100 instead of a
// smaller positive number.  2^x from the FMA-pipe polynomial (7.5e-5), then the
// exponent-flip seed and the cubic step (|rel err| <= 1.3e-4).  Total relative
// error <= 2.1e-4 plus rounding, inside the bf16 rounding of G that follows.
__device__ __forceinline__ float2 sigmoid_pair_fma(float2 zh) {
  float ax, ay;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(ax) : "f"(zh.x), "f"(-kLog2eF / 100.f), "f"(0.5f));
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(ay) : "f"(zh.y), "f"(-kLog2eF / 100.f), "f"(0.5f));
  const float2 x = __ffma2_rn(f2(ax, ay), f2(200.f, 200.f), f2(-100.f, -100.f));
  const float2 v = exp2_poly3_pair(x);
  const float2 nw = __ffma2_rn(v, f2(-1.f, -1.f), f2(-1.f, -1.f));   // -(1 + v)
  return rcp2_cubic(nw);
}

// Gradient only, one SFU operation and one packed FMA-pipe instruction per pair:
// sigmoid(z) = (1 + tanh(zh)) / 2, zh = z / 2.
__device__ __forceinline__ float2 sigmoid_pair_tanh(float2 zh) {
  return __ffma2_rn(f2(tanh_approx(zh.x), tanh_approx(zh.y)), f2(0.5f, 0.5f), f2(0.5f, 0.5f));
}

}  // namespace cutbce
