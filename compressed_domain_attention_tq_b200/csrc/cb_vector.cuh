// cb_vector.cuh -- one warp quantizes one d-vector into a codebook cache row
// (AdapTQ post: indices into a Max-Lloyd codebook with +-3 sigma clipping).
// Per group of 32 rotated coordinates y:
//   sigma = fl32(sqrt(S / 32)), S = sum y^2 accumulated in fp64
//   u     = clamp(fl32(y / sigma), -3, 3)          (u = 0 when sigma = 0)
//   index = #{ i : u > t_i },  t_i = fl32(fl32(C_i + C_{i+1}) * 0.5)
// A row holds its groups in order, each in 4 * BITS bytes; index j of a group
// occupies bits BITS*j .. BITS*j + BITS - 1 of the group's little-endian bit
// string.  Lane l holds coordinates E*l .. E*l+E-1 (E = D/32); the rotation is
// the int4 warp quantizer's.  Used by the codebook quantize kernel and by the
// decode kernel's fused append.
//
// With `uniform` the same row format holds the uniform low-bit variant (the
// int4 quantizer at BITS bits: Open-TQ-Metal forum summary, future work int2):
// m = 2^(BITS-1) - 1, s = fl32(amax / m), index = clamp(rne(fl32(y / s)), -m, m)
// + m, read back through the levels C[u] = u - m; `levels` is not read.
#pragma once
#include <math.h>
#include <stdint.h>

#include "quantize_vector.cuh"

namespace tq {

template <int D, int BITS>
__device__ __forceinline__ void cb_quantize_vector_warp(const void* src, bool bf16,
                                                        const int8_t* signs, const float* levels,
                                                        uint8_t* prow_bytes, float* srow,
                                                        int lane, bool uniform = false) {
  constexpr int E = D / 32;   // coordinates per lane (E consecutive ones)
  constexpr int GL = 32 / E;  // lanes per group
  constexpr int L = 1 << BITS;
  constexpr int M = (1 << (BITS - 1)) - 1;  // uniform: largest code

  float x[E];
  load_vector_warp<D>(src, bf16, x, lane);
  rotate_vector_warp<D>(x, signs, lane);

  // indices of this lane's E coordinates, packed at bit BITS * j0 of the group
  uint32_t bits = 0;
  float sigma;
  if (uniform) {
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
    for (int o = 1; o < GL; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    sigma = __fdiv_rn(amax, (float)M);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float c = amax > 0.0f ? rintf(__fdiv_rn(x[e], sigma)) : 0.0f;
      c = fminf(fmaxf(c, (float)-M), (float)M);
      bits |= (uint32_t)((int)c + M) << (BITS * e);
    }
  } else {
    float t[L - 1];  // thresholds between adjacent levels
#pragma unroll
    for (int i = 0; i + 1 < L; ++i) t[i] = __fmul_rn(__fadd_rn(levels[i], levels[i + 1]), 0.5f);
    // the group's sum of squares in fp64: this lane's E, then the group's GL lanes
    double S = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) S += (double)x[e] * (double)x[e];
#pragma unroll
    for (int o = 1; o < GL; o <<= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    sigma = (float)sqrt(S / 32.0);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float u = sigma > 0.0f ? __fdiv_rn(x[e], sigma) : 0.0f;
      u = fminf(fmaxf(u, -3.0f), 3.0f);
      uint32_t k = 0;
#pragma unroll
      for (int i = 0; i + 1 < L; ++i) k += u > t[i] ? 1u : 0u;
      bits |= k << (BITS * e);
    }
  }
  const int g = lane / GL, j0 = E * (lane % GL);
  const int off = BITS * j0;  // bit offset of this lane's indices in the group
  uint32_t* prow = reinterpret_cast<uint32_t*>(prow_bytes);
  const uint64_t wide = bits;
#pragma unroll
  for (int w = 0; w < BITS; ++w) {  // the group's BITS words
    const int sh = off - 32 * w;
    uint32_t c = 0;
    if (sh >= 0 && sh < 32) c = (uint32_t)(wide << sh);
    else if (sh < 0 && sh > -32) c = (uint32_t)(wide >> -sh);
#pragma unroll
    for (int o = 1; o < GL; o <<= 1) c |= __shfl_xor_sync(0xffffffffu, c, o);
    if (lane % GL == w) prow[BITS * g + w] = c;
  }
  if (lane % GL == 0) srow[g] = sigma;
}

}  // namespace tq
