// exp2_poly.cuh -- 2^x on the FMA pipe, for part of the forward kernel's
// exponentials (the MUFU unit alone needs as many cycles per tile as both
// tensor-core products).
//
// Cody-Waite style range reduction: 2^x = 2^floor(x) * 2^f, f in [0, 1).
// floor(x) comes from one round-down add of 1.5 * 2^23 (its low mantissa
// bits then hold floor(x) as an integer), 2^f from a degree-3 polynomial
// fitted for minimax relative error on [0, 1) by Lawson's iteratively
// reweighted least squares with c0 = 1 (fit_exp2_poly.py prints these
// coefficients; max relative error 8.6e-5, far below bf16's 2^-9), and
// 2^floor(x) is added to the exponent field.  Inputs are clamped at -126 so
// the result stays a normal float; callers use it only where every input is
// finite (masked -inf logits go through ex2.approx, which returns 0).
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace lca {

constexpr float kExp2C1 = 0.6951163411140442f;
constexpr float kExp2C2 = 0.22764700651168823f;
constexpr float kExp2C3 = 0.07706519961357117f;
constexpr float kExp2Magic = 12582912.0f;  // 1.5 * 2^23

// Two lanes at once: x = (lo, hi) packed.
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x) {
  float a, b;
  f2_unpack(x, a, b);
  a = fmaxf(a, -126.0f);
  b = fmaxf(b, -126.0f);
  x = f2_pack(a, b);
  const uint64_t magic = f2_pack(kExp2Magic, kExp2Magic);
  const uint64_t t = f2_add_rm(x, magic);        // 1.5*2^23 + floor(x)
  const uint64_t fl = f2_sub(t, magic);           // floor(x), exact
  const uint64_t f = f2_sub(x, fl);               // in [0, 1)
  uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(1.0f, 1.0f));
  // exponent field += floor(x): the low 9 bits of t's pattern shifted into
  // bits 23..31 (two's complement wraps correctly)
  const uint32_t tlo = static_cast<uint32_t>(t), thi = static_cast<uint32_t>(t >> 32);
  const uint32_t plo = static_cast<uint32_t>(p) + (tlo << 23);
  const uint32_t phi = static_cast<uint32_t>(p >> 32) + (thi << 23);
  return (static_cast<uint64_t>(phi) << 32) | plo;
}

}  // namespace lca
