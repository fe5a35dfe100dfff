// Symmetric int8 quantiser code shared by the per-token quantisation kernels
// (activations before the W8A8 products, and the latent between them).
#pragma once

#include "common.cuh"

namespace lr {

// The int8 code of a symmetric quantiser, clamp(rint(fl(x / sc)), -127, 127)
// with the IEEE fp32 quotient, where |x| <= 127 sc (sc = fl(max / 127)), given
// inv = fl(1 / sc).  t = fl(x inv) carries two roundings of relative size
// 2^-24 against x / sc, and fl(x / sc) one, so |t - fl(x / sc)| < 2.3e-5 for
// |x / sc| <= 127.5: where t lies farther than 1/8192 from every
// half-integer, both round to the same integer and no division is needed.
// The rest (near-ties, and non-finite values) take the quotient itself.
LR_DEV float quant_code(float x, float sc, float inv) {
  const float t = x * inv;
  const float r = rintf(t);
  const float q = 0.5f - fabsf(t - r) > 1.0f / 8192.0f ? r : rintf(__fdiv_rn(x, sc));
  return fminf(fmaxf(q, -127.f), 127.f);
}

}  // namespace lr
