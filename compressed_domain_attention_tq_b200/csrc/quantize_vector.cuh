// quantize_vector.cuh -- one warp quantizes one d-vector into its cache row.
//
// Sign flip + Walsh-Hadamard rotation (AdapTQ post, "Fast Hadamard Rotation
// (HAR)"; random signs: SRFT post, core method), group-32 abs-max scale and
// symmetric int4 codes with nibble packing (SRFT post, core method).  Lane l
// holds coordinates E*l .. E*l+E-1 (E = D/32).  The butterfly stages run in
// the order bits 1, 2, 4, ... with u + w / u - w in fp32, the same operations
// as the bulk kernel's, so both give bit-identical rotated values; codes use
// the IEEE division (c = rne(fl32(y / s)), s = fl32(amax / 7)).  Used by the
// small-append kernel and by the decode kernels' fused append.
#pragma once
#include <stdint.h>

namespace tq {

// Lane l loads coordinates E*l .. E*l+E-1 (E = D/32) of one fp32 or bf16 vector.
template <int D>
__device__ __forceinline__ void load_vector_warp(const void* src, bool bf16, float (&x)[D / 32],
                                                 int lane) {
  constexpr int E = D / 32;
  if (bf16) {
    const uint16_t* s16 = static_cast<const uint16_t*>(src) + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = __uint_as_float((uint32_t)s16[e] << 16);
  } else {
    const float* s32 = static_cast<const float*>(src) + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = s32[e];
  }
}

// In place: x <- H_D (signs (.) x) / sqrt(D) for the lane layout above (D = 128
// or 256), butterflies in the order bits 1, 2, 4, ...; nothing when signs is NULL.
template <int D>
__device__ __forceinline__ void rotate_vector_warp(float (&x)[D / 32], const int8_t* signs, int lane) {
  constexpr int E = D / 32;
  if (signs) {
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (signs[lane * E + e] < 0) x[e] = __uint_as_float(__float_as_uint(x[e]) ^ 0x80000000u);
#pragma unroll
    for (int bit = 1; bit < E; bit <<= 1)
#pragma unroll
      for (int e = 0; e < E; ++e)
        if ((e & bit) == 0) {
          const float u = x[e], w = x[e | bit];
          x[e] = u + w;
          x[e | bit] = u - w;
        }
#pragma unroll
    for (int lb = 1; lb < 32; lb <<= 1)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float v = __shfl_xor_sync(0xffffffffu, x[e], lb);
        x[e] = (lane & lb) ? v - x[e] : x[e] + v;
      }
    const float norm = (D == 128) ? 0.08838834764831844f : 0.0625f;  // 1/sqrt(D)
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] *= norm;
  }
}

template <int D>
__device__ __forceinline__ void quantize_vector_warp(const void* src, bool bf16, const int8_t* signs,
                                                     uint8_t* packed_row, float* scale_row, int lane) {
  constexpr int E = D / 32;   // coordinates per lane
  constexpr int GL = 32 / E;  // lanes per quantization group
  constexpr int NG = D / 32;
  float x[E];
  load_vector_warp<D>(src, bf16, x, lane);
  rotate_vector_warp<D>(x, signs, lane);
  float amax = 0.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int o = 1; o < GL; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 7.0f);
  uint32_t half[E / 4];  // 4 codes per 16-bit half-word
#pragma unroll
  for (int h = 0; h < E / 4; ++h) half[h] = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    float c = 0.0f;
    if (s > 0.0f) c = fminf(fmaxf(rintf(__fdiv_rn(x[e], s)), -7.0f), 7.0f);
    half[e / 4] |= ((uint32_t)(int)c & 0xFu) << (4 * (e % 4));
  }
  // coordinate i = E*lane + e: group g = lane / GL, in-group j = E*(lane % GL) + e,
  // sub-block j / 4, so half-word h sits at byte (j0/4 + h) * 2*NG + 2*g
  const int g = lane / GL;
  const int j0 = E * (lane % GL);
#pragma unroll
  for (int h = 0; h < E / 4; ++h)
    *reinterpret_cast<uint16_t*>(packed_row + (j0 / 4 + h) * 2 * NG + 2 * g) = (uint16_t)half[h];
  if (lane % GL == 0) scale_row[g] = s;
}

}  // namespace tq
