// quantize.cu -- fused on-the-fly int4 quantization of K/V vectors.
//
// One pass per vector: optional sign flip + Walsh-Hadamard butterflies
// (AdapTQ post, "Fast Hadamard Rotation (HAR)"; random signs as in the SRFT
// post's sign-randomized Hadamard), group-32 abs-max, symmetric int4 codes,
// nibble packing and 128-bit stores (SRFT post, core method: rotation, scale,
// group abs-max and int4 packing fused into a single kernel).
//
// Work decomposition: each thread owns 128 consecutive coordinates of one
// vector (d = 128: one thread per vector; d = 256: two neighbouring lanes per
// vector, joined by one shuffle butterfly stage).  Seven butterfly stages run
// in registers, so the rotation costs no shuffles at d = 128.
//
// Codes are c = rne(fl32(y / s)) with s = fl32(amax / 7) (fp32 IEEE
// division, round half to even).  Instead of one IEEE division per element,
// each element is rounded twice with reciprocals bracketing 1/s from below and
// above (relative distance 2^-21, far more than the rounding error of the
// reciprocal and of the quotient).  Rounding is monotone, so when both give
// the same integer it equals rne(fl32(y / s)); otherwise (an element within
// ~1e-5 of a half-integer, or a subnormal scale) the group is recomputed with
// the IEEE division.  With rotation off the result is bit-identical to the
// plain definition.
#include <cuda_bf16.h>
#include <math.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr float kRneMagic = 12582912.0f;  // 1.5 * 2^23: x + M rounds x to an integer
constexpr float kInvSqrt128 = 0.08838834764831844f;
constexpr float kBracketLo = 1.0f - 4.76837158203125e-07f;  // 1 - 2^-21 (exact)
constexpr float kBracketHi = 1.0f + 4.76837158203125e-07f;  // 1 + 2^-21 (exact)
constexpr int64_t kSmallAppendVectors = 8192;  // up to this many: one warp per vector

__device__ __forceinline__ uint32_t bfi4(uint32_t word, uint32_t nib_src, int pos) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, %3, 4;" : "=r"(r) : "r"(nib_src), "r"(word), "r"(pos));
  return r;
}

// 128 consecutive inputs -> fp32, sign flips applied (bf16 flips the sign bit
// before widening; fp32 flips it after).
template <bool BF16, bool ROT>
__device__ __forceinline__ void load_slice(const void* base, int64_t elem_off, bool valid,
                                           const uint32_t* __restrict__ smask,
                                           float (&x)[128]) {
  if (BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem_off);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      uint4 w = valid ? __ldcs(p + c) : make_uint4(0, 0, 0, 0);
      uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t u = ws[k];
        if (ROT) u ^= smask[c * 4 + k];   // bit 15 / bit 31 = sign of element 2k / 2k+1
        x[c * 8 + 2 * k] = __uint_as_float(u << 16);
        x[c * 8 + 2 * k + 1] = __uint_as_float(u & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_off);
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      float4 f = valid ? __ldcs(p + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      float fs[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t u = __float_as_uint(fs[k]);
        if (ROT) u ^= smask[64 + c * 4 + k];   // per-element masks (bit 31)
        x[c * 4 + k] = __uint_as_float(u);
      }
    }
  }
}

template <int D, bool BF16, bool ROT>
__global__ void __launch_bounds__(128) quantize_kernel(QuantizeArgs a) {
  constexpr int L = D / 128;  // threads per vector
  // Sign masks per 128-coordinate slice: [0, 64) XOR masks for bf16 pairs
  // (bit 15 / bit 31), [64, 192) XOR masks for single fp32 elements (bit 31).
  __shared__ uint32_t smask[192];
  __shared__ uint32_t smask_hi[192];
  if (ROT) {
    for (int i = threadIdx.x; i < 128 * L; i += blockDim.x) {
      const int e = i % 128;
      uint32_t* m = (i / 128) ? smask_hi : smask;
      m[64 + e] = (a.signs[i] < 0) ? 0x80000000u : 0u;
      if ((e & 1) == 0)
        m[e / 2] = ((a.signs[i] < 0) ? 0x00008000u : 0u) | ((a.signs[i + 1] < 0) ? 0x80000000u : 0u);
    }
    __syncthreads();
  }
  const int64_t per_kv = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t nvec = 2 * per_kv;
  const int sub = (L == 2) ? (int)(threadIdx.x & 1) : 0;
  const int64_t vec_stride = ((int64_t)gridDim.x * blockDim.x) / L;
  const uint32_t* mymask = sub ? smask_hi : smask;

  for (int64_t vec = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / L;; vec += vec_stride) {
    bool valid = vec < nvec;
    if (L == 1) {
      if (!valid) break;
    } else if (__all_sync(0xffffffffu, !valid)) {
      break;
    }
    const int kv = valid ? (int)(vec / per_kv) : 0;
    const int64_t rem = valid ? vec % per_kv : 0;
    const int64_t bh = rem / a.n_new;
    const int64_t n = rem % a.n_new;
    const int b = (int)(bh / a.Hkv);
    const int64_t p = valid ? (int64_t)a.pos[b] + n : -1;
    const bool store = valid && p >= 0 && p < a.capacity;

    float x[128];
    load_slice<BF16, ROT>(kv ? a.v : a.k, rem * D + sub * 128, valid, mymask, x);

    if (ROT) {
#pragma unroll
      for (int bit = 1; bit < 128; bit <<= 1) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          if ((i & bit) == 0) {
            const float u = x[i], w = x[i | bit];
            x[i] = u + w;
            x[i | bit] = u - w;
          }
        }
      }
      if (L == 2) {  // butterfly on coordinate bit 7 across the lane pair
        const float sgn = sub ? -1.0f : 1.0f;
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float other = __shfl_xor_sync(0xffffffffu, x[i], 1);
          x[i] = fmaf(sgn, x[i], other);
        }
      }
      const float norm = (D == 128) ? kInvSqrt128 : 0.0625f;
#pragma unroll
      for (int i = 0; i < 128; ++i) x[i] *= norm;
    }

    float scales[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float* xg = x + 32 * g;
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(xg[j]));
      const float s = __fdiv_rn(amax, 7.0f);
      scales[g] = s;
      const float r = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
      const bool big = !(r <= 3.0e38f);   // subnormal scale: use the division throughout
      const float rlo = r * kBracketLo, rhi = r * kBracketHi;
      float code[32];
      bool ambiguous = big;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float flo = fmaf(xg[j], rlo, kRneMagic);
        const float fhi = fmaf(xg[j], rhi, kRneMagic);
        ambiguous |= (flo != fhi);
        code[j] = flo;
      }
      if (ambiguous) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float c = rintf(__fdiv_rn(xg[j], s));
          c = fminf(fmaxf(c, -7.0f), 7.0f);
          code[j] = kRneMagic + c;   // exact: |c| <= 7
        }
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) xg[j] = code[j];
    }

    // Pack: group g (of this thread's 4), in-group j -> local word 2*(j/4) + g/2,
    // bit 16*(g%2) + 4*(j%4).  For d = 128 local words are the row's 16 words;
    // for d = 256 local word (2r + g/2) is row word 4r + 2*sub + g/2.
    uint32_t words[16];
#pragma unroll
    for (int w = 0; w < 16; ++w) words[w] = 0u;
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int j = 0; j < 32; ++j)
        words[2 * (j / 4) + g / 2] =
            bfi4(words[2 * (j / 4) + g / 2], __float_as_uint(x[32 * g + j]), 16 * (g % 2) + 4 * (j % 4));

    if (L == 2) {
      // Lane 0 keeps sub-blocks 0..3, lane 1 keeps 4..7; each needs the
      // partner's two words of those sub-blocks.
      uint32_t recv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r_send = sub ? (k / 2) : (4 + k / 2);
        const uint32_t send = words[2 * r_send + (k % 2)];
        recv[k] = __shfl_xor_sync(0xffffffffu, send, 1);
      }
      uint32_t out[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int r = sub ? 4 + q4 : q4;
        // row words 4r..4r+3 = [lane0 w(2r), lane0 w(2r+1), lane1 w(2r), lane1 w(2r+1)]
        const uint32_t own0 = words[2 * r], own1 = words[2 * r + 1];
        const uint32_t oth0 = recv[2 * q4], oth1 = recv[2 * q4 + 1];
        out[4 * q4 + 0] = sub ? oth0 : own0;
        out[4 * q4 + 1] = sub ? oth1 : own1;
        out[4 * q4 + 2] = sub ? own0 : oth0;
        out[4 * q4 + 3] = sub ? own1 : oth1;
      }
#pragma unroll
      for (int w = 0; w < 16; ++w) words[w] = out[w];
    }

    if (store) {
      const int64_t row = bh * a.capacity + p;
      uint8_t* packed = kv ? a.v_packed : a.k_packed;
      float* scl = kv ? a.v_scales : a.k_scales;
      uint4* dst = reinterpret_cast<uint4*>(packed + row * (D / 2) + sub * 64);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        dst[c] = make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
      *reinterpret_cast<float4*>(scl + row * (D / 32) + sub * 4) =
          make_float4(scales[0], scales[1], scales[2], scales[3]);
    }
  }
}

// Small appends (a decode step quantizes 2 * B * Hkv vectors): one warp per
// vector, lane l holding coordinates E*l .. E*l+E-1 (E = D/32), so a step's
// few vectors finish in a few hundred cycles instead of one long serial
// thread each.  The butterfly stages run in the same order and with the same
// operations as quantize_kernel's (bits 1, 2, 4, ...), so the rotated values
// are bit-identical; codes use the IEEE division directly.
template <int D>
__global__ void __launch_bounds__(128) quantize_warp_kernel(QuantizeArgs a) {
  constexpr int E = D / 32;        // coordinates per lane
  constexpr int GL = 32 / E;       // lanes per quantization group
  const int lane = threadIdx.x & 31;
  const int64_t per_kv = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t vec = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (vec >= 2 * per_kv) return;  // whole warp
  const int kv = (int)(vec / per_kv);
  const int64_t rem = vec % per_kv;
  const int64_t bh = rem / a.n_new, n = rem % a.n_new;
  const int b = (int)(bh / a.Hkv);
  const int64_t p = (int64_t)a.pos[b] + n;
  if (p < 0 || p >= a.capacity) return;  // whole warp
  float x[E];
  const int64_t off = rem * D + lane * E;
  const void* src = kv ? a.v : a.k;
  if (a.bf16) {
    const uint16_t* s16 = static_cast<const uint16_t*>(src) + off;
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = __uint_as_float((uint32_t)s16[e] << 16);
  } else {
    const float* s32 = static_cast<const float*>(src) + off;
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = s32[e];
  }
  if (a.signs) {
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (a.signs[lane * E + e] < 0) x[e] = __uint_as_float(__float_as_uint(x[e]) ^ 0x80000000u);
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
    const float norm = (D == 128) ? kInvSqrt128 : 0.0625f;
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] *= norm;
  }
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
  constexpr int NG = D / 32;
  const int g = lane / GL;
  const int j0 = E * (lane % GL);
  const int64_t row = bh * a.capacity + p;
  uint8_t* packed = (kv ? a.v_packed : a.k_packed) + row * (D / 2);
#pragma unroll
  for (int h = 0; h < E / 4; ++h)
    *reinterpret_cast<uint16_t*>(packed + (j0 / 4 + h) * 2 * NG + 2 * g) = (uint16_t)half[h];
  if (lane % GL == 0) (kv ? a.v_scales : a.k_scales)[row * NG + g] = s;
}

template <int D, bool BF16, bool ROT>
cudaError_t launch_q(const QuantizeArgs& a, cudaStream_t stream) {
  constexpr int L = D / 128;
  const int64_t threads = 2LL * a.B * a.Hkv * a.n_new * L;
  int64_t blocks = (threads + 127) / 128;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_kernel<D, BF16, ROT><<<(unsigned)blocks, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream) {
  const int64_t nvec = 2LL * a.B * a.Hkv * a.n_new;
  if (nvec <= kSmallAppendVectors) {
    const unsigned blocks = (unsigned)((nvec + 3) / 4);
    if (a.d == 128) quantize_warp_kernel<128><<<blocks, 128, 0, stream>>>(a);
    else quantize_warp_kernel<256><<<blocks, 128, 0, stream>>>(a);
    return cudaGetLastError();
  }
  const bool rot = a.signs != nullptr;
  if (a.d == 128) {
    if (a.bf16) return rot ? launch_q<128, true, true>(a, stream) : launch_q<128, true, false>(a, stream);
    return rot ? launch_q<128, false, true>(a, stream) : launch_q<128, false, false>(a, stream);
  }
  if (a.bf16) return rot ? launch_q<256, true, true>(a, stream) : launch_q<256, true, false>(a, stream);
  return rot ? launch_q<256, false, true>(a, stream) : launch_q<256, false, false>(a, stream);
}

}  // namespace tq
