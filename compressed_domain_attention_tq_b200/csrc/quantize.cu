// quantize.cu -- fused on-the-fly int4 quantization of K/V vectors.
//
// One pass per vector: optional sign flip + Walsh-Hadamard butterflies
// (AdapTQ post, "Fast Hadamard Rotation (HAR)"; random signs as in the SRFT
// post's sign-randomized Hadamard), group-32 abs-max, symmetric int4 codes,
// nibble packing and 128-bit stores (SRFT post, core method: rotation, scale,
// group abs-max and int4 packing fused into a single kernel).
//
// Work decomposition (bulk appends): each thread owns 128 consecutive
// coordinates of one vector (d = 128: one thread per vector; d = 256: two
// neighbouring lanes per vector, joined by one shuffle butterfly stage).
// Seven butterfly stages run in registers, so the rotation costs no shuffles
// at d = 128.  The inputs reach registers through shared memory: each warp
// copies its next batch of 32 slices with coalesced 16-byte cp.async while it
// computes the current one, and reads its slice at a padded pitch (no bank
// conflicts).  Small appends (a decode step) use one warp per vector instead.
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

#include "quantize_vector.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr float kRneMagic = 12582912.0f;  // 1.5 * 2^23: x + M rounds x to an integer
constexpr float kInvSqrt128 = 0.08838834764831844f;
constexpr float kBracketLo = 1.0f - 4.76837158203125e-07f;  // 1 - 2^-21 (exact)
constexpr float kBracketHi = 1.0f + 4.76837158203125e-07f;  // 1 + 2^-21 (exact)
constexpr int64_t kSmallAppendVectors = 8192;  // up to this many: one warp per vector

// Async 16-byte global -> shared copy; src_bytes = 0 zero-fills without reading.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bulk path layout.  A warp quantizes batches of 32 slices (a slice = 128
// consecutive coordinates of one vector: d = 128 -> 32 vectors, d = 256 -> 16
// vectors, two lanes each).  A batch is VPB consecutive input vectors, i.e.
// one contiguous span of the K (then V) input, copied with coalesced 16-byte
// cp.async into shared memory at a pitch of slice + 16 bytes, so that lane t
// then reads its own slice t without bank conflicts.  Two buffers per warp:
// the next batch is in flight while the current one is computed.
template <bool BF16>
struct QCfg {
  static constexpr int EB = BF16 ? 2 : 4;       // input bytes per element
  static constexpr int SLICE = 128 * EB;        // bytes of a 128-coordinate slice
  static constexpr int PITCH = SLICE + 16;      // shared-memory slice pitch
  static constexpr int BUF = 32 * PITCH;        // one batch buffer
  static constexpr int WARPS = BF16 ? 8 : 4;    // warps per CTA (one CTA per SM)
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int MASKS = 2 * 192 * 4;     // sign masks of the two 128-slices
  static constexpr int BYTES = MASKS + WARPS * 2 * BUF;
  static_assert(BYTES <= 227 * 1024, "shared memory");
};

// This lane's slice of a staged batch -> fp32, sign flips applied (bf16 flips
// the sign bit before widening; fp32 flips it after).
template <bool BF16, bool ROT>
__device__ __forceinline__ void read_slice(const unsigned char* slice, const uint32_t* smask,
                                           float (&x)[128]) {
  if (BF16) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const uint4 w = reinterpret_cast<const uint4*>(slice)[c];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t u = ws[k];
        if (ROT) u ^= smask[c * 4 + k];  // bit 15 / bit 31 = sign of element 2k / 2k+1
        x[c * 8 + 2 * k] = __uint_as_float(u << 16);
        x[c * 8 + 2 * k + 1] = __uint_as_float(u & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const uint4 w = reinterpret_cast<const uint4*>(slice)[c];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t u = ws[k];
        if (ROT) u ^= smask[64 + c * 4 + k];  // per-element masks (bit 31)
        x[c * 4 + k] = __uint_as_float(u);
      }
    }
  }
}

// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// a - b for two lanes at once (fma with -1 rounds like the subtraction)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// Rotation (unless !ROT), group-32 abs-max scales and int4 codes of one
// 128-coordinate slice, packed into the row layout: words[16] are the slice's
// packed row words (d = 128: the whole row; d = 256: after the lane-pair
// exchange, this lane's half of the row), scales[4] its groups' scales.
// Butterfly stages run in the order bits 1, 2, 4, ... with u + w / u - w in
// fp32 (two lanes at once from bit 2 on), the same operations as the
// small-append kernel, so both give bit-identical codes.
template <int D, bool ROT>
__device__ __forceinline__ void quantize_slice(float (&x)[128], int sub, uint32_t (&words)[16],
                                               float (&scales)[4]) {
  constexpr int L = D / 128;
  if (ROT) {
#pragma unroll
    for (int i = 0; i < 128; i += 2) {
      const float u = x[i], w = x[i + 1];
      x[i] = u + w;
      x[i + 1] = u - w;
    }
#pragma unroll
    for (int bit = 2; bit < 128; bit <<= 1)
#pragma unroll
      for (int i = 0; i < 128; i += 2)
        if ((i & bit) == 0) {
          const float2 u = make_float2(x[i], x[i + 1]), w = make_float2(x[i | bit], x[(i | bit) + 1]);
          const float2 s = __fadd2_rn(u, w), d = sub2(u, w);
          x[i] = s.x;
          x[i + 1] = s.y;
          x[i | bit] = d.x;
          x[(i | bit) + 1] = d.y;
        }
    if (L == 2) {  // butterfly on coordinate bit 7 across the lane pair
      const float sgn = sub ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, x[i], 1);
        x[i] = fmaf(sgn, x[i], other);
      }
    }
    const float2 norm = (D == 128) ? make_float2(kInvSqrt128, kInvSqrt128) : make_float2(0.0625f, 0.0625f);
#pragma unroll
    for (int i = 0; i < 128; i += 2) {
      const float2 v = __fmul2_rn(make_float2(x[i], x[i + 1]), norm);
      x[i] = v.x;
      x[i + 1] = v.y;
    }
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float* xg = x + 32 * g;
    float m[11];
#pragma unroll
    for (int j = 0; j < 10; ++j) m[j] = fmax3(fabsf(xg[3 * j]), fabsf(xg[3 * j + 1]), fabsf(xg[3 * j + 2]));
    m[10] = fmaxf(fabsf(xg[30]), fabsf(xg[31]));
    const float amax = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]),
                             fmax3(fmax3(m[6], m[7], m[8]), m[9], m[10]));
    const float s = __fdiv_rn(amax, 7.0f);
    scales[g] = s;
    const float r = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
    const bool big = !(r <= 3.0e38f);  // subnormal scale: use the division throughout
    const float2 rlo = make_float2(r * kBracketLo, r * kBracketLo);
    const float2 rhi = make_float2(r * kBracketHi, r * kBracketHi);
    const float2 magic = make_float2(kRneMagic, kRneMagic);
    float code[32];
    uint32_t diff = big ? 1u : 0u;
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float2 v = make_float2(xg[j], xg[j + 1]);
      const float2 flo = __ffma2_rn(v, rlo, magic), fhi = __ffma2_rn(v, rhi, magic);
      diff |= (__float_as_uint(flo.x) ^ __float_as_uint(fhi.x)) |
              (__float_as_uint(flo.y) ^ __float_as_uint(fhi.y));
      code[j] = flo.x;
      code[j + 1] = flo.y;
    }
    if (diff) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float c = rintf(__fdiv_rn(xg[j], s));
        c = fminf(fmaxf(c, -7.0f), 7.0f);
        code[j] = kRneMagic + c;  // exact: |c| <= 7
      }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) xg[j] = code[j];
  }

  // Pack: group g (of this slice's 4), in-group j -> local word 2*(j/4) + g/2,
  // bit 16*(g%2) + 4*(j%4).  For d = 128 local words are the row's 16 words;
  // for d = 256 local word (2r + g/2) is row word 4r + 2*sub + g/2.  Each code
  // is held as the float M + c (bits 0x4B400000 + c), so the bits minus
  // (0x4B400000 - 8) are c + 8 in 1..15: a word is sum_k (c_k + 8) 16^k, built
  // by shift-adds on the raw bits (wrapping; the constant is removed once),
  // and flipping bit 3 of each nibble gives the two's-complement nibbles.
  constexpr uint32_t kBias = (0x4B400000u - 8u) * 0x11111111u;
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {
      uint32_t w = 0u;
#pragma unroll
      for (int k = 7; k >= 0; --k) {
        const int g = 2 * gp + k / 4, j = 4 * r + k % 4;
        w = (w << 4) + __float_as_uint(x[32 * g + j]);
      }
      words[2 * r + gp] = (w - kBias) ^ 0x88888888u;
    }

  if (L == 2) {
    // Lane 0 keeps sub-blocks 0..3, lane 1 keeps 4..7; each needs the
    // partner's two words of those sub-blocks.
    uint32_t recv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      // lane 1 sends sub-block k / 2, lane 0 sub-block 4 + k / 2 (static indices)
      const uint32_t send = sub ? words[2 * (k / 2) + (k % 2)] : words[2 * (4 + k / 2) + (k % 2)];
      recv[k] = __shfl_xor_sync(0xffffffffu, send, 1);
    }
    uint32_t out[16];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      // r = sub ? 4 + q4 : q4; row words 4r..4r+3 =
      // [lane0 w(2r), lane0 w(2r+1), lane1 w(2r), lane1 w(2r+1)]
      const uint32_t own0 = sub ? words[2 * (4 + q4)] : words[2 * q4];
      const uint32_t own1 = sub ? words[2 * (4 + q4) + 1] : words[2 * q4 + 1];
      const uint32_t oth0 = recv[2 * q4], oth1 = recv[2 * q4 + 1];
      out[4 * q4 + 0] = sub ? oth0 : own0;
      out[4 * q4 + 1] = sub ? oth1 : own1;
      out[4 * q4 + 2] = sub ? own0 : oth0;
      out[4 * q4 + 3] = sub ? own1 : oth1;
    }
#pragma unroll
    for (int w = 0; w < 16; ++w) words[w] = out[w];
  }
}

template <int D, bool BF16, bool ROT>
__global__ void __launch_bounds__(QCfg<BF16>::THREADS, 1) quantize_staged_kernel(QuantizeArgs a) {
  using Q = QCfg<BF16>;
  constexpr int L = D / 128;         // lanes per vector
  constexpr int VPB = 32 / L;        // vectors per batch
  constexpr int VB = D * Q::EB;      // input bytes per vector
  constexpr int CPL = Q::SLICE / 16; // 16-byte copies per lane per batch
  extern __shared__ __align__(16) unsigned char smem[];
  // Sign masks per 128-coordinate slice (second slice at +192): [0, 64) XOR
  // masks for bf16 pairs (bit 15 / bit 31), [64, 192) for fp32 (bit 31).
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (ROT) {
    for (int i = threadIdx.x; i < 128 * L; i += blockDim.x) {
      const int e = i % 128;
      uint32_t* m = smask + (i / 128) * 192;
      m[64 + e] = (a.signs[i] < 0) ? 0x80000000u : 0u;
      if ((e & 1) == 0)
        m[e / 2] = ((a.signs[i] < 0) ? 0x00008000u : 0u) | ((a.signs[i + 1] < 0) ? 0x80000000u : 0u);
    }
  }
  __syncthreads();
  unsigned char* buf = smem + Q::MASKS + warp * 2 * Q::BUF;
  const int64_t per_kv = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t nvec = 2 * per_kv;
  const int64_t nbatch = (nvec + VPB - 1) / VPB;
  const int64_t nw = (int64_t)gridDim.x * Q::WARPS;
  const unsigned char* kin = static_cast<const unsigned char*>(a.k);
  const unsigned char* vin = static_cast<const unsigned char*>(a.v);
  const bool narrow = per_kv <= 0x7fffffffLL;  // 32-bit index arithmetic suffices

  // batch bi (VPB consecutive vectors: one contiguous span of K, then of V)
  // -> padded slices of buffer dst; vectors past the end are zero-filled
  auto issue = [&](int64_t bi, unsigned char* dst) {
    const int64_t v0 = bi * VPB;
    if (v0 + VPB <= per_kv || (v0 >= per_kv && v0 + VPB <= nvec)) {
      // the whole batch is one contiguous span of K or of V: lane offsets once,
      // then constant steps (the byte offset of copy c is 512 c + 16 lane)
      const unsigned char* src = (v0 < per_kv ? kin + v0 * VB : vin + (v0 - per_kv) * VB) + 16 * lane;
      const int o = 16 * lane;
      unsigned char* d0 = dst + ((o / VB) * L + (o % VB) / Q::SLICE) * Q::PITCH + (o % VB) % Q::SLICE;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        // 512 c is a whole number of slices (512 = 2 slices at bf16, 1 at fp32)
        cp_async16(d0 + (512 * c / Q::SLICE) * Q::PITCH, src + 512 * c, 16u);
      }
      cp_async_commit();
      return;
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int o = (c * 32 + lane) * 16;  // byte offset within the batch
      const int vi = o / VB, ov = o % VB;
      const int64_t v = v0 + vi;
      const bool ok = v < nvec;
      const unsigned char* src = ok ? (v < per_kv ? kin + v * VB : vin + (v - per_kv) * VB) + ov : kin;
      cp_async16(dst + (vi * L + ov / Q::SLICE) * Q::PITCH + ov % Q::SLICE, src, ok ? 16u : 0u);
    }
    cp_async_commit();
  };

  int64_t bi = (int64_t)blockIdx.x * Q::WARPS + warp;
  if (bi < nbatch) issue(bi, buf);
  for (int k = 0; bi < nbatch; ++k, bi += nw) {
    const unsigned char* cur = buf + (k & 1) * Q::BUF;
    if (bi + nw < nbatch) {
      issue(bi + nw, buf + ((k + 1) & 1) * Q::BUF);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const int sub = (L == 2) ? (lane & 1) : 0;
    float x[128];
    read_slice<BF16, ROT>(cur + lane * Q::PITCH, smask + sub * 192, x);
    __syncwarp();  // the next iteration refills the other buffer, and this one after it

    uint32_t words[16];
    float scales[4];
    quantize_slice<D, ROT>(x, sub, words, scales);

    const int64_t v = bi * VPB + lane / L;
    if (v < nvec) {
      const bool kv = v >= per_kv;
      const int64_t rem = kv ? v - per_kv : v;
      int64_t bh, n;
      if (narrow) {
        const uint32_t r32 = (uint32_t)rem, bh32 = r32 / (uint32_t)a.n_new;
        bh = bh32;
        n = r32 - bh32 * (uint32_t)a.n_new;
      } else {
        bh = rem / a.n_new;
        n = rem - bh * a.n_new;
      }
      const int b = (int)((uint32_t)bh / (uint32_t)a.Hkv);
      const int64_t p = (int64_t)a.pos[b] + n;
      if (p >= 0 && p < a.capacity) {
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
}

// Small appends (a decode step quantizes 2 * B * Hkv vectors): one warp per
// vector (quantize_vector_warp), so a step's few vectors finish in a few
// hundred cycles instead of one long serial thread each.
template <int D>
__global__ void __launch_bounds__(128) quantize_warp_kernel(QuantizeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t per_kv = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t vec = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (vec >= 2 * per_kv) return;  // whole warp
  const int kv = (int)(vec / per_kv);
  const int64_t rem = vec % per_kv;
  const int64_t bh = rem / a.n_new, n = rem % a.n_new;
  const int b = (int)(bh / a.Hkv);
  int64_t p = (int64_t)a.pos[b] + n;
  if (a.pos_is_ctx) p = (int64_t)min(max(a.pos[b], 1), a.max_ctx) - 1 + n;
  if (p < 0 || p >= a.capacity) return;  // whole warp
  const int64_t row = bh * a.capacity + p;
  const int eb = a.bf16 ? 2 : 4;
  quantize_vector_warp<D>(static_cast<const unsigned char*>(kv ? a.v : a.k) + rem * D * eb, a.bf16,
                          a.signs, (kv ? a.v_packed : a.k_packed) + row * (D / 2),
                          (kv ? a.v_scales : a.k_scales) + row * (D / 32), lane);
}

// d = 128 with bf16 inputs: two lanes per vector, 64 coordinates each (lane
// 2v + sub holds coordinates 64 sub .. 64 sub + 63, groups 2 sub, 2 sub + 1).
// Six butterfly stages run in registers and the seventh (coordinate bit 6)
// across the lane pair, in the same order and with the same operations as the
// other quantize kernels; half the registers per thread let 16 warps share an
// SM.  A warp batch is 16 vectors (32 slices of 128 bytes at a 144-byte pitch).
struct QHalf {
  static constexpr int SLICE = 128;         // 64 bf16
  static constexpr int PITCH = SLICE + 16;  // shared-memory slice pitch
  static constexpr int BUF = 32 * PITCH;
  static constexpr int WARPS = 16;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int MASKS = 2 * 32 * 4;  // bf16 pair masks of the two 64-slices
  static constexpr int BYTES = MASKS + WARPS * 2 * BUF;
  static_assert(BYTES <= 227 * 1024, "shared memory");
};

template <bool ROT>
__global__ void __launch_bounds__(QHalf::THREADS, 1) quantize_half_kernel(QuantizeArgs a) {
  using Q = QHalf;
  constexpr int D = 128, VPB = 16, VB = 256, CPL = 8;  // vectors / bytes per vector / copies per lane
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem);  // [2][32]: bit 15 / 31 = sign of 2k / 2k+1
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (ROT)
    for (int i = threadIdx.x; i < 64; i += blockDim.x)
      smask[i] = ((a.signs[2 * i] < 0) ? 0x00008000u : 0u) | ((a.signs[2 * i + 1] < 0) ? 0x80000000u : 0u);
  __syncthreads();
  unsigned char* buf = smem + Q::MASKS + warp * 2 * Q::BUF;
  const int64_t per_kv = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t nvec = 2 * per_kv;
  const int64_t nbatch = (nvec + VPB - 1) / VPB;
  const int64_t nw = (int64_t)gridDim.x * Q::WARPS;
  const unsigned char* kin = static_cast<const unsigned char*>(a.k);
  const unsigned char* vin = static_cast<const unsigned char*>(a.v);
  const bool narrow = per_kv <= 0x7fffffffLL;

  // batch bi -> padded slices of buffer dst; the byte offset of copy c is
  // 512 c + 16 lane: vector 2c + lane / 16, slice 2 (that) + (lane % 16) / 8
  auto issue = [&](int64_t bi, unsigned char* dst) {
    const int64_t v0 = bi * VPB;
    const int ov = 16 * (lane & 15);
    unsigned char* d0 = dst + (2 * (lane >> 4) + ov / Q::SLICE) * Q::PITCH + ov % Q::SLICE;
    if (v0 + VPB <= per_kv || (v0 >= per_kv && v0 + VPB <= nvec)) {
      const unsigned char* src = (v0 < per_kv ? kin + v0 * VB : vin + (v0 - per_kv) * VB) + 16 * lane;
#pragma unroll
      for (int c = 0; c < CPL; ++c) cp_async16(d0 + 4 * c * Q::PITCH, src + 512 * c, 16u);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int64_t v = v0 + 2 * c + (lane >> 4);
        const bool ok = v < nvec;
        const unsigned char* src = ok ? (v < per_kv ? kin + v * VB : vin + (v - per_kv) * VB) + ov : kin;
        cp_async16(d0 + 4 * c * Q::PITCH, src, ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  };

  int64_t bi = (int64_t)blockIdx.x * Q::WARPS + warp;
  if (bi < nbatch) issue(bi, buf);
  const int sub = lane & 1;
  for (int k = 0; bi < nbatch; ++k, bi += nw) {
    const unsigned char* cur = buf + (k & 1) * Q::BUF;
    if (bi + nw < nbatch) {
      issue(bi + nw, buf + ((k + 1) & 1) * Q::BUF);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    float x[64];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 w = reinterpret_cast<const uint4*>(cur + lane * Q::PITCH)[c];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t u = ws[kk];
        if (ROT) u ^= smask[sub * 32 + c * 4 + kk];
        x[c * 8 + 2 * kk] = __uint_as_float(u << 16);
        x[c * 8 + 2 * kk + 1] = __uint_as_float(u & 0xFFFF0000u);
      }
    }
    __syncwarp();  // the next iteration refills the other buffer, and this one after it

    if (ROT) {
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float u = x[i], w = x[i + 1];
        x[i] = u + w;
        x[i + 1] = u - w;
      }
#pragma unroll
      for (int bit = 2; bit < 64; bit <<= 1)
#pragma unroll
        for (int i = 0; i < 64; i += 2)
          if ((i & bit) == 0) {
            const float2 u = make_float2(x[i], x[i + 1]), w = make_float2(x[i | bit], x[(i | bit) + 1]);
            const float2 s = __fadd2_rn(u, w), d = sub2(u, w);
            x[i] = s.x;
            x[i + 1] = s.y;
            x[i | bit] = d.x;
            x[(i | bit) + 1] = d.y;
          }
      const float sgn = sub ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {  // coordinate bit 6, across the lane pair
        const float other = __shfl_xor_sync(0xffffffffu, x[i], 1);
        x[i] = fmaf(sgn, x[i], other);  // lane 0: u + w, lane 1: u - w (exact sign flip)
      }
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        const float2 v = __fmul2_rn(make_float2(x[i], x[i + 1]), make_float2(kInvSqrt128, kInvSqrt128));
        x[i] = v.x;
        x[i + 1] = v.y;
      }
    }
    float scales[2];
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      float* xg = x + 32 * g;
      float m[11];
#pragma unroll
      for (int j = 0; j < 10; ++j) m[j] = fmax3(fabsf(xg[3 * j]), fabsf(xg[3 * j + 1]), fabsf(xg[3 * j + 2]));
      m[10] = fmaxf(fabsf(xg[30]), fabsf(xg[31]));
      const float amax = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]),
                               fmax3(fmax3(m[6], m[7], m[8]), m[9], m[10]));
      const float s = __fdiv_rn(amax, 7.0f);
      scales[g] = s;
      const float r = (s > 0.0f) ? __frcp_rn(s) : 0.0f;
      const bool big = !(r <= 3.0e38f);
      const float2 rlo = make_float2(r * kBracketLo, r * kBracketLo);
      const float2 rhi = make_float2(r * kBracketHi, r * kBracketHi);
      const float2 magic = make_float2(kRneMagic, kRneMagic);
      float code[32];
      uint32_t diff = big ? 1u : 0u;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 v = make_float2(xg[j], xg[j + 1]);
        const float2 flo = __ffma2_rn(v, rlo, magic), fhi = __ffma2_rn(v, rhi, magic);
        diff |= (__float_as_uint(flo.x) ^ __float_as_uint(fhi.x)) |
                (__float_as_uint(flo.y) ^ __float_as_uint(fhi.y));
        code[j] = flo.x;
        code[j + 1] = flo.y;
      }
      if (diff) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float c = rintf(__fdiv_rn(xg[j], s));
          c = fminf(fmaxf(c, -7.0f), 7.0f);
          code[j] = kRneMagic + c;
        }
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) xg[j] = code[j];
    }
    // local word r: this lane's groups, in-group 4r .. 4r + 3 (group 0 in bits
    // 0..15, group 1 in 16..31) = row word 2r + sub; nibbles by shift-adds on
    // the magic-float bits (see quantize_slice)
    constexpr uint32_t kBias = (0x4B400000u - 8u) * 0x11111111u;
    uint32_t w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      uint32_t acc = 0u;
#pragma unroll
      for (int kk = 7; kk >= 0; --kk) acc = (acc << 4) + __float_as_uint(x[32 * (kk / 4) + 4 * r + kk % 4]);
      w[r] = (acc - kBias) ^ 0x88888888u;
    }
    // 16-byte chunk c = row words 4c .. 4c + 3 = [w0(2c), w1(2c), w0(2c+1), w1(2c+1)]
    // (wS = lane S's local words); lane 0 writes chunks 0, 1 and lane 1 chunks 2, 3
    uint32_t recv[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) recv[kk] = __shfl_xor_sync(0xffffffffu, sub ? w[kk] : w[4 + kk], 1);
    const int64_t v = bi * VPB + (lane >> 1);
    if (v < nvec) {
      const bool kv = v >= per_kv;
      const int64_t rem = kv ? v - per_kv : v;
      int64_t bh, n;
      if (narrow) {
        const uint32_t r32 = (uint32_t)rem, bh32 = r32 / (uint32_t)a.n_new;
        bh = bh32;
        n = r32 - bh32 * (uint32_t)a.n_new;
      } else {
        bh = rem / a.n_new;
        n = rem - bh * a.n_new;
      }
      const int b = (int)((uint32_t)bh / (uint32_t)a.Hkv);
      const int64_t p = (int64_t)a.pos[b] + n;
      if (p >= 0 && p < a.capacity) {
        const int64_t row = bh * a.capacity + p;
        uint4* dst = reinterpret_cast<uint4*>((kv ? a.v_packed : a.k_packed) + row * (D / 2) + 32 * sub);
        if (sub == 0) {
          dst[0] = make_uint4(w[0], recv[0], w[1], recv[1]);
          dst[1] = make_uint4(w[2], recv[2], w[3], recv[3]);
        } else {
          dst[0] = make_uint4(recv[0], w[4], recv[1], w[5]);
          dst[1] = make_uint4(recv[2], w[6], recv[3], w[7]);
        }
        *reinterpret_cast<float2*>((kv ? a.v_scales : a.k_scales) + row * 4 + 2 * sub) =
            make_float2(scales[0], scales[1]);
      }
    }
  }
}

template <bool ROT>
cudaError_t launch_half(const QuantizeArgs& a, cudaStream_t stream) {
  static SmemLimitSet smem_set;
  const cudaError_t e = ensure_smem_limit(quantize_half_kernel<ROT>, QHalf::BYTES, smem_set);
  if (e != cudaSuccess) return e;
  const int64_t nbatch = (2LL * a.B * a.Hkv * a.n_new + 15) / 16;
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (nbatch + QHalf::WARPS - 1) / QHalf::WARPS;
  if (blocks > sms) blocks = sms;
  quantize_half_kernel<ROT><<<(unsigned)blocks, QHalf::THREADS, QHalf::BYTES, stream>>>(a);
  return cudaGetLastError();
}

template <int D, bool BF16, bool ROT>
cudaError_t launch_q(const QuantizeArgs& a, cudaStream_t stream) {
  using Q = QCfg<BF16>;
  static SmemLimitSet smem_set;
  const cudaError_t e = ensure_smem_limit(quantize_staged_kernel<D, BF16, ROT>, Q::BYTES, smem_set);
  if (e != cudaSuccess) return e;
  const int64_t nbatch = (2LL * a.B * a.Hkv * a.n_new + 32 / (D / 128) - 1) / (32 / (D / 128));
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (nbatch + Q::WARPS - 1) / Q::WARPS;
  if (blocks > sms) blocks = sms;
  quantize_staged_kernel<D, BF16, ROT><<<(unsigned)blocks, Q::THREADS, Q::BYTES, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream) {
  const int64_t nvec = 2LL * a.B * a.Hkv * a.n_new;
  if (nvec <= kSmallAppendVectors || a.pos_is_ctx) {
    const unsigned blocks = (unsigned)((nvec + 3) / 4);
    if (a.d == 128) quantize_warp_kernel<128><<<blocks, 128, 0, stream>>>(a);
    else quantize_warp_kernel<256><<<blocks, 128, 0, stream>>>(a);
    return cudaGetLastError();
  }
  const bool rot = a.signs != nullptr;
  if (a.d == 128) {
    if (a.bf16 && rot && !a.butterfly_rotation && quantize_tc_supported(a)) return launch_quantize_tc(a, stream);
    if (a.bf16) return rot ? launch_half<true>(a, stream) : launch_half<false>(a, stream);
    return rot ? launch_q<128, false, true>(a, stream) : launch_q<128, false, false>(a, stream);
  }
  if (a.bf16 && rot && !a.butterfly_rotation && quantize_tc_supported(a)) return launch_quantize_tc(a, stream);
  if (a.bf16) return rot ? launch_q<256, true, true>(a, stream) : launch_q<256, true, false>(a, stream);
  return rot ? launch_q<256, false, true>(a, stream) : launch_q<256, false, false>(a, stream);
}

}  // namespace tq
