// quantize_tc.cu -- bulk quantize-append of bf16 K/V at head_dim 128 with the
// rotation on the fifth-generation tensor cores.
//
// The rotated vector is y = R x with R = H diag(signs) / sqrt(128) (AdapTQ
// post, "Fast Hadamard Rotation (HAR)"; the sign-randomized Hadamard of the
// SRFT post).  For bf16 inputs every product x_k * (+-1) is exact, so the
// unnormalised rotation of a tile of 128 vectors is one 128 x 128 x 128 bf16
// product with fp32 accumulation: D = X B, B[k][n] = signs[k] * H[k][n]
// (H[k][n] = (-1)^popcount(k & n), the Sylvester Hadamard matrix).  The
// butterfly form of the other quantize kernels spends about six of its ~16
// instructions per coordinate on this; here it costs eight tcgen05.mma per
// tile, and the CUDA cores only do the group abs-max, the codes and the
// packing (SRFT post, core method: scale, group abs-max and int4 packing
// fused into one pass).
//
// One persistent CTA per SM, warp-specialised:
//  - warp 8 (one thread) streams 128-vector input tiles into a ring of five
//    32 KB shared-memory stages with TMA (two 64-element boxes per tile, the
//    128-byte swizzle the MMA reads);
//  - warp 9 (one thread) issues the eight K = 16 MMAs of a tile into one of
//    two 128-column fp32 accumulators in tensor memory;
//  - warps 0-3 and 4-7 (one thread per vector, warp w reads tensor-memory
//    lanes 32 (w % 4) ..) take the accumulators of even and odd tiles in turn:
//    group-32 abs-max, scale, codes, nibble packing, 16-byte stores.  A tile's
//    groups are handled in two pairs; the second pair's tensor-memory loads
//    are in flight while the first is quantized.
// The epilogue warps build B in shared memory while the first input copies
// are in flight; the MMA issuer waits for it on a named barrier.
// Every wait is bounded (tc::mbar_wait); a CTA whose wait gives up writes NaN
// scales into every row it did not finish, so the failure shows in the cache.
//
// Codes.  With y = fl(D c), c = fl(1 / sqrt(128)), the stored values are
// s = fl(max|y| / 7) and q = rne(fl(y / s)), the definition the oracle and
// the other kernels follow.  max|y| = fl(max|D| c) (rounding is monotone).
// fl(a / 7) is computed as fl(a zh + fl(a zl)), zh = fl(1/7), zl = fl(1/7 -
// zh): division by a divisor known in advance (Brisebarre, Muller and Raina,
// IEEE Trans. Computers 2004).  It is exact here because a / 7 lies at least
// 1/14 of an ulp from every rounding midpoint while the two-term error is
// below 2^-24 ulp (checked over every significand on the CPU); below a =
// 2^-90, where a zl would lose bits, the IEEE division runs instead.
// q is found without forming y: D is rounded twice to an integer, with
// fl(fl(c r) (1 -+ 2^-21)) as factors, r the hardware reciprocal of s
// (relative error below 2^-23); the two bracket fl(y / s) (their relative
// distance, 2^-21, exceeds 2^-23 plus the four roundings of 2^-24 between
// them), so when both give the same integer it is q; otherwise (a value
// within ~1e-6 of a half-integer, or s below 2^-100, where y could be
// subnormal) the group is recomputed as fl(y / s) with the IEEE division.
// The accumulation order inside the tensor core is not the butterflies' one,
// so this kernel's rotated values can differ from theirs in the last bits;
// when every partial sum is exact (small-integer inputs) the two kernels
// give identical bits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include "tc_ptx.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace tc;

constexpr int kRows = 128;          // vectors per tile (MMA M)
constexpr int kNS = 5;              // input stages
constexpr int kStage = kRows * 256; // one tile of bf16 input (two 16 KB swizzled halves)
constexpr int kThreads = 320;       // 8 epilogue warps, producer, MMA issuer
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kTmemCols = 256;      // two 128-column accumulators

constexpr float kInvSqrt128 = 0.08838834764831844f;
constexpr float kRneMagic = 12582912.0f;                    // 1.5 * 2^23
constexpr float kBracketLo = 1.0f - 4.76837158203125e-07f;  // 1 - 2^-21
constexpr float kBracketHi = 1.0f + 4.76837158203125e-07f;  // 1 + 2^-21
constexpr float kFastScaleMin = 0x1p-100f;
constexpr float kDiv7Min = 0x1p-90f;          // fl(a / 7) by the two-constant form from here up
constexpr float kSeventhHi = 0x1.24924ap-3f;  // fl(1/7)
constexpr float kSeventhLo = -0x1.b6db6ep-28f;  // fl(1/7 - fl(1/7))

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int kOffB = 0;                         // B, 32 KB
constexpr int kOffStage = 32768;                 // kNS stages
constexpr int kOffBar = kOffStage + kNS * kStage;
constexpr int kFull = 0, kEmpty = kNS, kDFull = 2 * kNS, kDEmpty = 2 * kNS + 2, kMmaDone = 2 * kNS + 4;
constexpr int kNBar = 2 * kNS + 5;
constexpr int kOffMisc = kOffBar + 8 * kNBar;    // tensor-memory base, abort flag
constexpr int kSmemBytes = kOffMisc + 16 + 1024; // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// idesc: bf16 A and B (type 1), f32 accumulation, both K-major, M = N = 128
constexpr uint32_t kIdesc = idesc_f16(128, 128, 0, 0) | (1u << 7) | (1u << 10);

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

struct Tiles {
  int64_t rows;      // vectors per tensor (B * Hkv * n_new)
  int64_t per;       // tiles per tensor
  __device__ int64_t total() const { return 2 * per; }
};

// Destination row of input vector `row` of the K (kv = 0) or V tensor, or -1
// when its position falls outside the cache.
__device__ __forceinline__ int64_t dest_row(const QuantizeArgs& a, int64_t row) {
  const uint32_t r32 = (uint32_t)row, bh = r32 / (uint32_t)a.n_new;
  const uint32_t n = r32 - bh * (uint32_t)a.n_new;
  const int b = (int)(bh / (uint32_t)a.Hkv);
  const int64_t p = (int64_t)a.pos[b] + n;
  if (p < 0 || p >= a.capacity) return -1;
  return (int64_t)bh * a.capacity + p;
}

// fl(a / 7) for a >= 0 (NaN and infinity through the IEEE division)
__device__ __forceinline__ float div7(float a) {
  return (a >= kDiv7Min && a <= 3.4028234663852886e38f) ? __fmaf_rn(a, kSeventhHi, __fmul_rn(a, kSeventhLo))
                                                         : __fdiv_rn(a, 7.0f);
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The 32 registers written by a tensor-memory load are used only after this
// point (the load completes at tcgen05.wait::ld, which the compiler does not
// know about).
__device__ __forceinline__ void tie32(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]),
                 "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7]));
}

// One group of 32 coordinates of this thread's vector: d[] = unnormalised
// rotated values D (fp32 bits) -> the scale, and in hw[jb] the codes of
// in-group coordinates 4 jb .. 4 jb + 3 as sum_kk 16^kk (0x4B400000 + q)
// (mod 2^32; each code is the float kRneMagic + q).
__device__ __forceinline__ float quantize_group(const uint32_t (&d)[32], uint32_t (&hw)[8]) {
  float m[11];
#pragma unroll
  for (int j = 0; j < 10; ++j)
    m[j] = fmax3(fabsf(__uint_as_float(d[3 * j])), fabsf(__uint_as_float(d[3 * j + 1])),
                 fabsf(__uint_as_float(d[3 * j + 2])));
  m[10] = fmaxf(fabsf(__uint_as_float(d[30])), fabsf(__uint_as_float(d[31])));
  const float amax = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]),
                           fmax3(fmax3(m[6], m[7], m[8]), m[9], m[10]));
  const float s = div7(amax * kInvSqrt128);
  const float r = (s > 0.0f) ? rcp_approx(s) : 0.0f;
  const float cr = r * kInvSqrt128;
  const float2 rlo = make_float2(cr * kBracketLo, cr * kBracketLo);
  const float2 rhi = make_float2(cr * kBracketHi, cr * kBracketHi);
  const float2 magic = make_float2(kRneMagic, kRneMagic);
  uint32_t diff[4] = {(s > 0.0f && s < kFastScaleMin) || !(r <= 3.0e38f) ? 1u : 0u, 0u, 0u, 0u};
#pragma unroll
  for (int jb = 0; jb < 8; ++jb) {
    uint32_t c[4];
#pragma unroll
    for (int h = 0; h < 4; h += 2) {
      const int j = 4 * jb + h;
      const float2 v = make_float2(__uint_as_float(d[j]), __uint_as_float(d[j + 1]));
      const float2 flo = __ffma2_rn(v, rlo, magic), fhi = __ffma2_rn(v, rhi, magic);
      diff[jb & 3] |= (__float_as_uint(flo.x) ^ __float_as_uint(fhi.x)) |
                      (__float_as_uint(flo.y) ^ __float_as_uint(fhi.y));
      c[h] = __float_as_uint(flo.x);
      c[h + 1] = __float_as_uint(flo.y);
    }
    hw[jb] = ((((c[3] << 4) + c[2]) << 4) + c[1]) * 16u + c[0];
  }
  if (diff[0] | diff[1] | diff[2] | diff[3]) {
#pragma unroll
    for (int jb = 0; jb < 8; ++jb) {
      uint32_t c[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float y = __uint_as_float(d[4 * jb + h]) * kInvSqrt128;
        float q = rintf(__fdiv_rn(y, s));
        q = fminf(fmaxf(q, -7.0f), 7.0f);
        c[h] = __float_as_uint(kRneMagic + q);  // exact: |q| <= 7
      }
      hw[jb] = ((((c[3] << 4) + c[2]) << 4) + c[1]) * 16u + c[0];
    }
  }
  return s;
}

// Row words 2 jb + p of the pair of groups (2p + 1, 2p): nibbles from the
// top are in-group 4 jb + 3 .. 4 jb of group 2p + 1, then of group 2p.  The
// constant 0x4B400000 of each code is removed (leaving q + 8 per nibble, no
// borrows), then bit 3 of every nibble is flipped (two's complement nibbles).
__device__ __forceinline__ void pack_pair(const uint32_t (&hw_hi)[8], const uint32_t (&hw_lo)[8], int p,
                                          uint32_t (&words)[16]) {
  constexpr uint32_t kBias = (0x4B400000u - 8u) * 0x11111111u;
#pragma unroll
  for (int jb = 0; jb < 8; ++jb) words[2 * jb + p] = ((hw_hi[jb] << 16) + hw_lo[jb] - kBias) ^ 0x88888888u;
}

__global__ void __launch_bounds__(kThreads, 1)
    quantize_tc_kernel(const QuantizeArgs a, const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the 128-byte swizzle is a function of absolute shared-memory address bits
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  int* misc = reinterpret_cast<int*>(smem + kOffMisc);
  volatile int* abort = misc + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Tiles tl;
  tl.rows = (int64_t)a.B * a.Hkv * a.n_new;
  tl.per = (tl.rows + kRows - 1) / kRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar + kFull + s, 1);
      mbar_init(bar + kEmpty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar + kDFull + b, 1);
      mbar_init(bar + kDEmpty + b, 4);
    }
    mbar_init(bar + kMmaDone, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), kTmemCols);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = static_cast<uint32_t>(misc[0]);
  const int64_t t_first = blockIdx.x, t_step = gridDim.x;

  if (warp < 8) {
    // B^T[n][k] = signs[k] (-1)^popcount(n & k) as bf16 +-1, K-major: row n
    // of K-half h at h * 16 KB + 128 n, its 16-byte chunk c at (c ^ (n % 8)) * 16.
    // Thread t builds chunk t % 16 (k = 8 (t % 16) .. + 7) of rows t / 16 + 16 it.
    {
      const int kc = threadIdx.x & 15;
      uint32_t neg8 = 0;  // bit e: signs[8 kc + e] < 0
#pragma unroll
      for (int e = 0; e < 8; ++e) neg8 |= (a.signs[8 * kc + e] < 0 ? 1u : 0u) << e;
      // bit e of kWalsh[m] = parity(m & e), m < 8
      constexpr uint64_t kWalsh = 0x963C5AF066CCAA00ull;
      unsigned char* bsm = smem + kOffB;
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int n = (threadIdx.x >> 4) + 16 * it;
        const uint32_t par = (uint32_t)(__popc(n & (8 * kc)) & 1) * 0xFFu;
        const uint32_t neg = neg8 ^ par ^ (uint32_t)((kWalsh >> (8 * (n & 7))) & 0xFFu);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = 0x3F803F80u | (((neg >> (2 * e)) & 1u) << 15) | (((neg >> (2 * e + 1)) & 1u) << 31);
        *reinterpret_cast<uint4*>(bsm + (kc >> 3) * 16384 + n * 128 + (((kc & 7) ^ (n & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // operand for the tensor cores
      asm volatile("bar.arrive 1, 288;" ::: "memory");                // B is ready
    }
    // ============================================================ epilogue
    const int set = warp >> 2, quarter = warp & 3;
    const uint32_t taddr = tbase + ((uint32_t)(32 * quarter) << 16) + 128u * set;
    uint32_t u = 0;
    bool failed = false;
    for (int64_t t = t_first + set * t_step; t < tl.total(); t += 2 * t_step, ++u) {
      const int kv = t >= tl.per;
      const int64_t row = (t - kv * tl.per) * kRows + 32 * quarter + lane;
      const int64_t dst = row < tl.rows ? dest_row(a, row) : -1;
      if (!failed) {
        const bool ok = mbar_wait(bar + kDFull + set, u & 1, abort);
        failed = !__all_sync(0xffffffffu, ok);
      }
      if (failed) {
        if (dst >= 0)
          *reinterpret_cast<float4*>((kv ? a.v_scales : a.k_scales) + dst * 4) =
              make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                          __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
        continue;
      }
      fence_after();
      uint32_t d1[32], d0[32], d3[32], d2[32], hw_a[8], hw_b[8], words[16];
      float sc[4];
      tld_x32(taddr + 32u, d1);
      tld_x32(taddr, d0);
      wait_ld();
      tie32(d1);
      tie32(d0);
      tld_x32(taddr + 96u, d3);  // in flight while groups 1 and 0 are quantized
      tld_x32(taddr + 64u, d2);
      sc[1] = quantize_group(d1, hw_a);
      sc[0] = quantize_group(d0, hw_b);
      pack_pair(hw_a, hw_b, 0, words);
      wait_ld();
      tie32(d3);
      tie32(d2);
      fence_before();  // every load of the accumulator is done: hand it back
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kDEmpty + set);
      sc[3] = quantize_group(d3, hw_a);
      sc[2] = quantize_group(d2, hw_b);
      pack_pair(hw_a, hw_b, 1, words);
      if (dst >= 0) {
        uint4* out = reinterpret_cast<uint4*>((kv ? a.v_packed : a.k_packed) + dst * 64);
#pragma unroll
        for (int c = 0; c < 4; ++c) out[c] = make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
        *reinterpret_cast<float4*>((kv ? a.v_scales : a.k_scales) + dst * 4) = make_float4(sc[0], sc[1], sc[2], sc[3]);
      }
    }
  } else if (warp == kProducerWarp) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t i = 0;
      for (int64_t t = t_first; t < tl.total(); t += t_step, ++i) {
        const int s = i % kNS;
        if (i >= kNS && !mbar_wait(bar + kEmpty + s, ((i / kNS) - 1) & 1, abort)) break;
        if (a.test_starve && i == 0) continue;  // test hook: the first stage never arrives
        const int kv = t >= tl.per;
        const int y = (int)((t - kv * tl.per) * kRows);
        unsigned char* stg = smem + kOffStage + s * kStage;
        mbar_arrive_expect_tx(bar + kFull + s, (uint32_t)kStage);
        const CUtensorMap* m = kv ? &map_v : &map_k;
        tma_load_2d(stg, m, 0, y, bar + kFull + s);
        tma_load_2d(stg + kStage / 2, m, 64, y, bar + kFull + s);
      }
      // copies still in flight land before the CTA exits
      const uint32_t first = i > (uint32_t)kNS ? i - kNS : 0;
      for (uint32_t v = first; v < i; ++v) {
        if (a.test_starve && v == 0) continue;
        mbar_drain(bar + kFull + v % kNS, (v / kNS) & 1);
      }
    }
  } else {
    // ============================================================ MMA issuer
    asm volatile("bar.sync 1, 288;" ::: "memory");  // B built by the epilogue warps
    if (lane == 0) {
      const uint64_t db = smem_desc_sw128(smem_u32(smem + kOffB));
      const uint64_t da = smem_desc_sw128(smem_u32(smem + kOffStage));
      uint32_t i = 0;
      for (int64_t t = t_first; t < tl.total(); t += t_step, ++i) {
        const int s = i % kNS, b = i & 1;
        if (!mbar_wait(bar + kFull + s, (i / kNS) & 1, abort)) break;
        if (i >= 2 && !mbar_wait(bar + kDEmpty + b, ((i >> 1) - 1) & 1, abort)) break;
        fence_after();
        const uint64_t das = da + (uint64_t)((s * kStage) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // K step ks: K-half ks / 4 (16 KB apart), 32 bytes per step inside a row
          const uint64_t off = (uint64_t)((((ks >> 2) * 16384) + (ks & 3) * 32) >> 4);
          mma_ss(tbase + 128u * b, das + off, db + off, kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar + kEmpty + s);
        mma_commit(bar + kDFull + b);
      }
      mma_commit(bar + kMmaDone);
      mbar_drain(bar + kMmaDone, 0);
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tbase, kTmemCols);
}

// ----------------------------------------------------------------- d = 256
// H_256 = [[H, H], [H, -H]] with H = H_128: for x = (x_lo, x_hi) the rotation
// is (P + Q, P - Q) / 16 with P = H (sigma_lo (.) x_lo), Q = H (sigma_hi (.)
// x_hi), two 128 x 128 x 128 products per tile into the two halves of a
// 256-column accumulator.  y = fl(P +- Q) / 16 (exact scaling); groups g and
// g + 4 come from the same columns of P and Q.
namespace w256 {
constexpr int kNS = 2;                     // input stages of 64 KB
constexpr int kStage = kRows * 512;        // four 16 KB swizzled chunks of 64 elements
constexpr int kOffB = 0;                   // B_lo, B_hi: 32 KB each
constexpr int kOffStage = 65536;
constexpr int kOffBar = kOffStage + kNS * kStage;
constexpr int kFull = 0, kEmpty = kNS, kDFull = 2 * kNS, kDEmpty = 2 * kNS + 2, kMmaDone = 2 * kNS + 4;
constexpr int kNBar = 2 * kNS + 5;
constexpr int kOffMisc = kOffBar + 8 * kNBar;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
constexpr int kTmemCols = 512;             // two accumulators of 256 columns (P | Q)
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
}  // namespace w256

// One group of 32 coordinates with y = fl(Dv * norm), norm a power of two:
// the scale, and hw[r] = the group's codes of in-group coordinates 4r .. 4r + 3
// as a finished nibble half-word (two's complement).
__device__ __forceinline__ float quantize_group_pow2(const float (&dv)[32], float norm, uint32_t (&hw)[8]) {
  float m[11];
#pragma unroll
  for (int j = 0; j < 10; ++j) m[j] = fmax3(fabsf(dv[3 * j]), fabsf(dv[3 * j + 1]), fabsf(dv[3 * j + 2]));
  m[10] = fmaxf(fabsf(dv[30]), fabsf(dv[31]));
  const float amax = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]),
                           fmax3(fmax3(m[6], m[7], m[8]), m[9], m[10]));
  const float s = div7(amax * norm);
  const float r = (s > 0.0f) ? rcp_approx(s) : 0.0f;
  const float cr = r * norm;
  const float2 rlo = make_float2(cr * kBracketLo, cr * kBracketLo);
  const float2 rhi = make_float2(cr * kBracketHi, cr * kBracketHi);
  const float2 magic = make_float2(kRneMagic, kRneMagic);
  uint32_t diff[4] = {(s > 0.0f && s < kFastScaleMin) || !(r <= 3.0e38f) ? 1u : 0u, 0u, 0u, 0u};
  uint32_t c[32];
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 v = make_float2(dv[j], dv[j + 1]);
    const float2 flo = __ffma2_rn(v, rlo, magic), fhi = __ffma2_rn(v, rhi, magic);
    diff[(j >> 1) & 3] |= (__float_as_uint(flo.x) ^ __float_as_uint(fhi.x)) |
                          (__float_as_uint(flo.y) ^ __float_as_uint(fhi.y));
    c[j] = __float_as_uint(flo.x);
    c[j + 1] = __float_as_uint(flo.y);
  }
  if (diff[0] | diff[1] | diff[2] | diff[3]) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float q = rintf(__fdiv_rn(dv[j] * norm, s));
      q = fminf(fmaxf(q, -7.0f), 7.0f);
      c[j] = __float_as_uint(kRneMagic + q);
    }
  }
  constexpr uint32_t kBias16 = (0x4B400000u - 8u) * 0x1111u;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const uint32_t h = ((((c[4 * rr + 3] << 4) + c[4 * rr + 2]) << 4) + c[4 * rr + 1]) * 16u + c[4 * rr];
    hw[rr] = ((h - kBias16) ^ 0x8888u) & 0xFFFFu;
  }
  return s;
}

__global__ void __launch_bounds__(kThreads, 1)
    quantize_tc256_kernel(const QuantizeArgs a, const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_v) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + w256::kOffBar);
  int* misc = reinterpret_cast<int*>(smem + w256::kOffMisc);
  volatile int* abort = misc + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Tiles tl;
  tl.rows = (int64_t)a.B * a.Hkv * a.n_new;
  tl.per = (tl.rows + kRows - 1) / kRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < w256::kNS; ++s) {
      mbar_init(bar + w256::kFull + s, 1);
      mbar_init(bar + w256::kEmpty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar + w256::kDFull + b, 1);
      mbar_init(bar + w256::kDEmpty + b, 4);
    }
    mbar_init(bar + w256::kMmaDone, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), w256::kTmemCols);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = static_cast<uint32_t>(misc[0]);
  const int64_t t_first = blockIdx.x, t_step = gridDim.x;

  if (warp < 8) {
    // B_lo^T, B_hi^T [n][k] = sigma_{k (+128)} (-1)^popcount(n & k), K-major, 128-byte
    // swizzle (as the d = 128 kernel's B); thread t builds chunk t % 16 of rows t / 16 + 16 it
    {
      const int kc = threadIdx.x & 15;
      constexpr uint64_t kWalsh = 0x963C5AF066CCAA00ull;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t neg8 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) neg8 |= (a.signs[128 * half + 8 * kc + e] < 0 ? 1u : 0u) << e;
        unsigned char* bsm = smem + w256::kOffB + half * 32768;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int n = (threadIdx.x >> 4) + 16 * it;
          const uint32_t par = (uint32_t)(__popc(n & (8 * kc)) & 1) * 0xFFu;
          const uint32_t neg = neg8 ^ par ^ (uint32_t)((kWalsh >> (8 * (n & 7))) & 0xFFu);
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = 0x3F803F80u | (((neg >> (2 * e)) & 1u) << 15) | (((neg >> (2 * e + 1)) & 1u) << 31);
          *reinterpret_cast<uint4*>(bsm + (kc >> 3) * 16384 + n * 128 + (((kc & 7) ^ (n & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.arrive 1, 288;" ::: "memory");
    }
    // ============================================================ epilogue
    const int set = warp >> 2, quarter = warp & 3;
    const uint32_t taddr = tbase + ((uint32_t)(32 * quarter) << 16) + 256u * set;
    uint32_t u = 0;
    bool failed = false;
    for (int64_t t = t_first + set * t_step; t < tl.total(); t += 2 * t_step, ++u) {
      const int kv = t >= tl.per;
      const int64_t row = (t - kv * tl.per) * kRows + 32 * quarter + lane;
      const int64_t dst = row < tl.rows ? dest_row(a, row) : -1;
      if (!failed) {
        const bool ok = mbar_wait(bar + w256::kDFull + set, u & 1, abort);
        failed = !__all_sync(0xffffffffu, ok);
      }
      if (failed) {
        if (dst >= 0) {
          float4* sp = reinterpret_cast<float4*>((kv ? a.v_scales : a.k_scales) + dst * 8);
          const float nan = __int_as_float(0x7fc00000);
          sp[0] = make_float4(nan, nan, nan, nan);
          sp[1] = make_float4(nan, nan, nan, nan);
        }
        continue;
      }
      fence_after();
      uint32_t words[32];
#pragma unroll
      for (int w = 0; w < 32; ++w) words[w] = 0u;
      float sc[8];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t pv[32], qv[32];
        tld_x32(taddr + 32u * g, pv);
        tld_x32(taddr + 128u + 32u * g, qv);
        wait_ld();
        tie32(pv);
        tie32(qv);
        if (g == 3) {  // the last loads of the accumulator: hand it back
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar + w256::kDEmpty + set);
        }
        float dlo[32], dhi[32];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 p2 = make_float2(__uint_as_float(pv[j]), __uint_as_float(pv[j + 1]));
          const float2 q2 = make_float2(__uint_as_float(qv[j]), __uint_as_float(qv[j + 1]));
          const float2 s2 = __fadd2_rn(p2, q2);
          const float2 d2 = __ffma2_rn(q2, make_float2(-1.0f, -1.0f), p2);  // p - q
          dlo[j] = s2.x;
          dlo[j + 1] = s2.y;
          dhi[j] = d2.x;
          dhi[j + 1] = d2.y;
        }
        uint32_t hw[8];
        // half-word f = 8 r + g of the row holds in-group 4r .. 4r + 3 of group g
        sc[g] = quantize_group_pow2(dlo, 0.0625f, hw);
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) words[(8 * rr + g) >> 1] |= hw[rr] << (16 * (g & 1));
        sc[g + 4] = quantize_group_pow2(dhi, 0.0625f, hw);
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) words[(8 * rr + g + 4) >> 1] |= hw[rr] << (16 * (g & 1));
      }
      if (dst >= 0) {
        uint4* out = reinterpret_cast<uint4*>((kv ? a.v_packed : a.k_packed) + dst * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) out[c] = make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
        float4* sp = reinterpret_cast<float4*>((kv ? a.v_scales : a.k_scales) + dst * 8);
        sp[0] = make_float4(sc[0], sc[1], sc[2], sc[3]);
        sp[1] = make_float4(sc[4], sc[5], sc[6], sc[7]);
      }
    }
  } else if (warp == kProducerWarp) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t i = 0;
      for (int64_t t = t_first; t < tl.total(); t += t_step, ++i) {
        const int s = i % w256::kNS;
        if (i >= w256::kNS && !mbar_wait(bar + w256::kEmpty + s, ((i / w256::kNS) - 1) & 1, abort)) break;
        if (a.test_starve && i == 0) continue;  // test hook: the first stage never arrives
        const int kv = t >= tl.per;
        const int y = (int)((t - kv * tl.per) * kRows);
        unsigned char* stg = smem + w256::kOffStage + s * w256::kStage;
        mbar_arrive_expect_tx(bar + w256::kFull + s, (uint32_t)w256::kStage);
        const CUtensorMap* m = kv ? &map_v : &map_k;
#pragma unroll
        for (int c = 0; c < 4; ++c) tma_load_2d(stg + c * 16384, m, 64 * c, y, bar + w256::kFull + s);
      }
      const uint32_t first = i > (uint32_t)w256::kNS ? i - w256::kNS : 0;
      for (uint32_t v = first; v < i; ++v) {
        if (a.test_starve && v == 0) continue;
        mbar_drain(bar + w256::kFull + v % w256::kNS, (v / w256::kNS) & 1);
      }
    }
  } else {
    // ============================================================ MMA issuer
    asm volatile("bar.sync 1, 288;" ::: "memory");  // B built by the epilogue warps
    if (lane == 0) {
      const uint64_t db = smem_desc_sw128(smem_u32(smem + w256::kOffB));
      const uint64_t da = smem_desc_sw128(smem_u32(smem + w256::kOffStage));
      uint32_t i = 0;
      for (int64_t t = t_first; t < tl.total(); t += t_step, ++i) {
        const int s = i % w256::kNS, b = i & 1;
        if (!mbar_wait(bar + w256::kFull + s, (i / w256::kNS) & 1, abort)) break;
        if (i >= 2 && !mbar_wait(bar + w256::kDEmpty + b, ((i >> 1) - 1) & 1, abort)) break;
        fence_after();
        const uint64_t das = da + (uint64_t)((s * w256::kStage) >> 4);
#pragma unroll
        for (int half = 0; half < 2; ++half)  // P from x_lo and B_lo, Q from x_hi and B_hi
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t aoff = (uint64_t)((((2 * half + (ks >> 2)) * 16384) + (ks & 3) * 32) >> 4);
            const uint64_t boff = (uint64_t)(((half * 32768 + (ks >> 2) * 16384) + (ks & 3) * 32) >> 4);
            mma_ss(tbase + 256u * b + 128u * half, das + aoff, db + boff, kIdesc, ks > 0 ? 1u : 0u);
          }
        mma_commit(bar + w256::kEmpty + s);
        mma_commit(bar + w256::kDFull + b);
      }
      mma_commit(bar + w256::kMmaDone);
      mbar_drain(bar + w256::kMmaDone, 0);
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tbase, w256::kTmemCols);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// rows x d bf16, 64 x 128-element boxes with the 128-byte swizzle (rows
// past the end read as zeros)
bool input_map(CUtensorMap* m, const void* base, int64_t rows, int d) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kRows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool quantize_tc_supported(const QuantizeArgs& a) {
  const int64_t rows = (int64_t)a.B * a.Hkv * a.n_new;
  return (a.d == 128 || a.d == 256) && a.bf16 && a.signs != nullptr && !a.pos_is_ctx && a.cb_bits == 0 &&
         a.lambda_k == nullptr && a.lambda_v == nullptr && rows <= (int64_t)INT32_MAX - kRows &&
         encode_fn() != nullptr;
}

cudaError_t launch_quantize_tc(const QuantizeArgs& a, cudaStream_t stream) {
  if (!quantize_tc_supported(a)) return cudaErrorNotSupported;
  static SmemLimitSet smem_set, smem_set256;
  const bool w = a.d == 256;
  const cudaError_t e = w ? ensure_smem_limit(quantize_tc256_kernel, w256::kSmemBytes, smem_set256)
                          : ensure_smem_limit(quantize_tc_kernel, kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.B * a.Hkv * a.n_new;
  CUtensorMap mk, mv;
  if (!input_map(&mk, a.k, rows, a.d) || !input_map(&mv, a.v, rows, a.d)) return cudaErrorInvalidValue;
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = 2 * ((rows + kRows - 1) / kRows);
  const int grid = (int)(tiles < sms ? tiles : sms);
  if (w) quantize_tc256_kernel<<<grid, kThreads, w256::kSmemBytes, stream>>>(a, mk, mv);
  else quantize_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(a, mk, mv);
  return cudaGetLastError();
}

}  // namespace tq
