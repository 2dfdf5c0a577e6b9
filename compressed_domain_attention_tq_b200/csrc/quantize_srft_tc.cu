// quantize_srft_tc.cu -- bulk quantize-append of bf16 K/V with the SRFT
// rotation on the fifth-generation tensor cores, head_dim 32, 64, 96 or 128.
//
// The stored vector is y = lambda (.) F (sigma (.) x) (SRFT post, core method:
// a sign-randomized Fourier transform, usable at widths that are not powers
// of two, then a per-coordinate scale lambda), F the orthonormal Hartley
// transform F[k][j] = cas(2 pi k j / d) / sqrt(d).  For bf16 inputs the
// unnormalised transform of a tile of 128 vectors is one 128 x d x d product
// D = X B with B[j][k] = sigma_j cas(2 pi j k / d).  B is not exact in bf16,
// so it is split into three bf16 parts (hi + mid + lo, about 24 bits, each
// entry first formed in fp64); the three products accumulate in the same fp32
// tensor-memory accumulator.  The epilogue forms y = fl(lambda'_k D_k) with
// lambda'_k = fl(lambda_k / sqrt(d)), then the group abs-max, the scale, the
// codes and the row layout of the int4 path.
//
// Roles and pipeline as in the Hadamard kernel (quantize_tc.cu): one
// persistent CTA per SM; warp 8 streams 128-vector tiles with TMA (K split
// into 64-element chunks with the 128-byte swizzle and, at d = 32 and 96, one
// 32-element chunk with the 64-byte swizzle); warp 9 issues 3 d / 16 MMAs per
// tile into one of four accumulators (the 3 d / 16 MMAs of a tile take about
// as long as its epilogue, so the issuer runs ahead); warps 0-7 (one thread
// per vector) take even and odd tiles and build B while the first copies fly.  Waits are
// bounded; a CTA that gives up writes NaN scales into the rows it did not
// finish.
//
// Codes: s = fl(max|y| / 7) by the two-constant division of the Hadamard
// kernel, q = rne(fl(y / s)) from two roundings of y fl(r (1 -+ 2^-21)), r
// the hardware reciprocal of s, with the IEEE division where they disagree
// or s < 2^-100.  The accumulation order differs from the warp FFT of the
// other SRFT kernels, so rows can differ from theirs in the last bits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "tc_ptx.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace tc;

constexpr int kRows = 128;
constexpr int kThreads = 320;  // 8 epilogue warps, producer, MMA issuer
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kNAcc = 4;        // accumulators of up to 128 columns: the MMAs run up to 3 tiles ahead
constexpr int kTmemCols = 512;

constexpr float kRneMagic = 12582912.0f;
constexpr float kBracketLo = 1.0f - 4.76837158203125e-07f;  // 1 - 2^-21
constexpr float kBracketHi = 1.0f + 4.76837158203125e-07f;  // 1 + 2^-21
constexpr float kFastScaleMin = 0x1p-100f;
constexpr float kDiv7Min = 0x1p-90f;
constexpr float kSeventhHi = 0x1.24924ap-3f;
constexpr float kSeventhLo = -0x1.b6db6ep-28f;

// Shared-memory descriptor of a K-major swizzled operand: layout 2 (128-byte
// swizzle, 1024-byte atoms of 8 rows) or 4 (64-byte swizzle, 512-byte atoms).
__host__ __device__ constexpr uint64_t desc_sw(uint32_t addr, uint32_t layout, uint32_t atom_bytes) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
         ((uint64_t)((atom_bytes >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)layout << 61);
}

template <int D>
struct L {
  static constexpr int NG = D / 32;           // quantization groups
  static constexpr int NC = D / 64;           // 64-element K chunks (128-byte swizzle)
  static constexpr int R32 = (D % 64) / 32;   // one 32-element chunk (64-byte swizzle)
  static constexpr int STAGE = kRows * D * 2; // one input tile
  static constexpr int PART = D * D * 2;      // one bf16 part of B
  static constexpr int BBYTES = 3 * PART;
  static constexpr int NS = (200 * 1024 - BBYTES) / STAGE > 5 ? 5 : (200 * 1024 - BBYTES) / STAGE;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_STAGE = (BBYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_LAM = OFF_STAGE + NS * STAGE;  // float lambda'[2][D]
  static constexpr int OFF_CAS = OFF_LAM + 8 * D;         // double cas[D]
  static constexpr int OFF_BAR = OFF_CAS + 8 * D;
  static constexpr int FULL = 0, EMPTY = NS, DFULL = 2 * NS, DEMPTY = 2 * NS + kNAcc;
  static constexpr int MMADONE = 2 * NS + 2 * kNAcc;
  static constexpr int NBAR = 2 * NS + 2 * kNAcc + 1;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int BYTES = OFF_MISC + 16 + 1024;
  static_assert(D % 32 == 0 && D >= 32 && D <= 128, "head_dim");
  static_assert(NS >= 2 && BYTES <= 227 * 1024, "shared memory");
  static_assert(STAGE % 1024 == 0 && PART % 1024 == 0, "1024-byte regions");
  // byte offset inside a [rows][D] K-major swizzled block of element (row, k)
  __device__ static uint32_t at(int rows, int row, int k) {
    const int c = k >> 6;
    if (c < NC) {
      const int kk = k & 63;
      return c * rows * 128 + row * 128 + ((((kk >> 3) ^ (row & 7)) << 4) | ((kk & 7) << 1));
    }
    const int kk = k - 64 * NC;  // < 32: the 64-byte swizzled chunk
    return NC * rows * 128 + row * 64 + ((((kk >> 3) ^ ((row >> 1) & 3)) << 4) | ((kk & 7) << 1));
  }
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float div7(float a) {
  return (a >= kDiv7Min && a <= 3.4028234663852886e38f) ? __fmaf_rn(a, kSeventhHi, __fmul_rn(a, kSeventhLo))
                                                         : __fdiv_rn(a, 7.0f);
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tie32(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]),
                 "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7]));
}

// One group: d[] = unnormalised transform D (fp32 bits), lam = lambda' of the
// group's 32 coordinates (shared memory) -> scale; hw[r] = the 4 codes of
// in-group coordinates 4r .. 4r + 3 as a nibble half-word (two's complement).
__device__ __forceinline__ float quantize_group(const uint32_t (&d)[32], const float* lam, uint32_t (&hw)[8]) {
  float y[32];
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 l = *reinterpret_cast<const float4*>(lam + j);
    const float2 a = __fmul2_rn(make_float2(__uint_as_float(d[j]), __uint_as_float(d[j + 1])), make_float2(l.x, l.y));
    const float2 b = __fmul2_rn(make_float2(__uint_as_float(d[j + 2]), __uint_as_float(d[j + 3])), make_float2(l.z, l.w));
    y[j] = a.x;
    y[j + 1] = a.y;
    y[j + 2] = b.x;
    y[j + 3] = b.y;
  }
  float m[11];
#pragma unroll
  for (int j = 0; j < 10; ++j) m[j] = fmax3(fabsf(y[3 * j]), fabsf(y[3 * j + 1]), fabsf(y[3 * j + 2]));
  m[10] = fmaxf(fabsf(y[30]), fabsf(y[31]));
  const float amax = fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]),
                           fmax3(fmax3(m[6], m[7], m[8]), m[9], m[10]));
  const float s = div7(amax);
  const float r = (s > 0.0f) ? rcp_approx(s) : 0.0f;
  const float2 rlo = make_float2(r * kBracketLo, r * kBracketLo);
  const float2 rhi = make_float2(r * kBracketHi, r * kBracketHi);
  const float2 magic = make_float2(kRneMagic, kRneMagic);
  uint32_t diff[4] = {(s > 0.0f && s < kFastScaleMin) || !(r <= 3.0e38f) ? 1u : 0u, 0u, 0u, 0u};
  uint32_t c[32];
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const float2 v = make_float2(y[j], y[j + 1]);
    const float2 flo = __ffma2_rn(v, rlo, magic), fhi = __ffma2_rn(v, rhi, magic);
    diff[(j >> 1) & 3] |= (__float_as_uint(flo.x) ^ __float_as_uint(fhi.x)) |
                          (__float_as_uint(flo.y) ^ __float_as_uint(fhi.y));
    c[j] = __float_as_uint(flo.x);
    c[j + 1] = __float_as_uint(flo.y);
  }
  if (diff[0] | diff[1] | diff[2] | diff[3]) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float q = rintf(__fdiv_rn(y[j], s));
      q = fminf(fmaxf(q, -7.0f), 7.0f);
      c[j] = __float_as_uint(kRneMagic + q);
    }
  }
  // each code is 0x4B400000 + q: the sum of 16^kk times it, minus the constant
  // per nibble (leaving q + 8, no borrows), with bit 3 of each nibble flipped
  constexpr uint32_t kBias = (0x4B400000u - 8u) * 0x1111u;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const uint32_t h = ((((c[4 * rr + 3] << 4) + c[4 * rr + 2]) << 4) + c[4 * rr + 1]) * 16u + c[4 * rr];
    hw[rr] = ((h - kBias) ^ 0x8888u) & 0xFFFFu;
  }
  return s;
}

__device__ __forceinline__ int64_t dest_row(const QuantizeArgs& a, int64_t row) {
  const uint32_t r32 = (uint32_t)row, bh = r32 / (uint32_t)a.n_new;
  const uint32_t n = r32 - bh * (uint32_t)a.n_new;
  const int b = (int)(bh / (uint32_t)a.Hkv);
  const int64_t p = (int64_t)a.pos[b] + n;
  if (p < 0 || p >= a.capacity) return -1;
  return (int64_t)bh * a.capacity + p;
}

struct Maps {
  CUtensorMap k64, v64, k32, v32;  // 64-element chunks (128-byte swizzle), 32-element chunk
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    quantize_srft_tc_kernel(const QuantizeArgs a, const __grid_constant__ Maps maps) {
  using Q = L<D>;
  constexpr int NG = Q::NG, NS = Q::NS, KS = D / 16;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Q::OFF_BAR);
  int* misc = reinterpret_cast<int*>(smem + Q::OFF_MISC);
  volatile int* abort = misc + 1;
  float* lam = reinterpret_cast<float*>(smem + Q::OFF_LAM);
  double* cas = reinterpret_cast<double*>(smem + Q::OFF_CAS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t per = (rows + kRows - 1) / kRows, total = 2 * per;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar + Q::FULL + s, 1);
      mbar_init(bar + Q::EMPTY + s, 1);
    }
    for (int b = 0; b < kNAcc; ++b) {
      mbar_init(bar + Q::DFULL + b, 1);
      mbar_init(bar + Q::DEMPTY + b, 4);
    }
    mbar_init(bar + Q::MMADONE, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), kTmemCols);
    tmem_relinquish();
  }
  // cas(2 pi m / d) in fp64, lambda' = fl(lambda / sqrt(d)) for K and V
  for (int i = threadIdx.x; i < D; i += kThreads) {
    double sn, cs;
    sincospi(2.0 * (double)i / (double)D, &sn, &cs);
    cas[i] = cs + sn;
    const double rs = 1.0 / sqrt((double)D);
    lam[i] = (float)((a.lambda_k ? (double)a.lambda_k[i] : 1.0) * rs);
    lam[D + i] = (float)((a.lambda_v ? (double)a.lambda_v[i] : 1.0) * rs);
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = static_cast<uint32_t>(misc[0]);

  if (warp < 8) {
    // B^T[n][k] = sigma_k cas(2 pi n k / d) in three bf16 parts (K-major rows n)
    {
      unsigned char* bsm = smem + Q::OFF_B;
      for (int e = threadIdx.x; e < D * D; e += 256) {
        const int n = e / D, k = e - n * D;
        double v = cas[(n * k) % D];
        if (a.signs && a.signs[k] < 0) v = -v;
        const __nv_bfloat16 hi = __double2bfloat16(v);
        const double r1 = v - (double)__bfloat162float(hi);
        const __nv_bfloat16 mid = __double2bfloat16(r1);
        const __nv_bfloat16 lo = __double2bfloat16(r1 - (double)__bfloat162float(mid));
        const uint32_t off = Q::at(D, n, k);
        *reinterpret_cast<__nv_bfloat16*>(bsm + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(bsm + Q::PART + off) = mid;
        *reinterpret_cast<__nv_bfloat16*>(bsm + 2 * Q::PART + off) = lo;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("bar.arrive 1, 288;" ::: "memory");
    }
    // ============================================================ epilogue
    const int set = warp >> 2, quarter = warp & 3;
    uint32_t u = 0;  // this set's tiles so far: tile i = 2 u + set of the CTA, accumulator i % kNAcc
    bool failed = false;
    for (int64_t t = blockIdx.x + set * gridDim.x; t < total; t += 2 * gridDim.x, ++u) {
      const uint32_t i = 2 * u + set, b = i % kNAcc;
      const uint32_t taddr = tbase + ((uint32_t)(32 * quarter) << 16) + 128u * b;
      const int kv = t >= per;
      const int64_t row = (t - kv * per) * kRows + 32 * quarter + lane;
      const int64_t dst = row < rows ? dest_row(a, row) : -1;
      float* scl = (kv ? a.v_scales : a.k_scales) + (dst >= 0 ? dst : 0) * NG;
      if (!failed) {
        const bool ok = mbar_wait(bar + Q::DFULL + b, (i / kNAcc) & 1, abort);
        failed = !__all_sync(0xffffffffu, ok);
      }
      if (failed) {
        if (dst >= 0)
#pragma unroll
          for (int g = 0; g < NG; ++g) scl[g] = __int_as_float(0x7fc00000);
        continue;
      }
      fence_after();
      uint32_t dbuf[2][32], hw[NG][8];
      float sc[NG];
      tld_x32(taddr, dbuf[0]);
      wait_ld();
      tie32(dbuf[0]);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        if (g + 1 < NG) tld_x32(taddr + 32u * (g + 1), dbuf[(g + 1) & 1]);  // in flight
        else {
          fence_before();  // every load of the accumulator is done: hand it back
          __syncwarp();
          if (lane == 0) mbar_arrive(bar + Q::DEMPTY + b);
        }
        sc[g] = quantize_group(dbuf[g & 1], lam + kv * D + 32 * g, hw[g]);
        if (g + 1 < NG) {
          wait_ld();
          tie32(dbuf[(g + 1) & 1]);
        }
      }
      if (dst >= 0) {
        // half-word f = r NG + g holds in-group 4r .. 4r + 3 of group g; word w
        // holds half-words 2w (low) and 2w + 1
        uint32_t words[D / 8];
#pragma unroll
        for (int w = 0; w < D / 8; ++w) {
          const int f0 = 2 * w, f1 = 2 * w + 1;
          words[w] = hw[f0 % NG][f0 / NG] | (hw[f1 % NG][f1 / NG] << 16);
        }
        uint4* out = reinterpret_cast<uint4*>((kv ? a.v_packed : a.k_packed) + dst * (D / 2));
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
          out[c] = make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
#pragma unroll
        for (int g = 0; g < NG; ++g) scl[g] = sc[g];
      }
    }
  } else if (warp == kProducerWarp) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t i = 0;
      for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(bar + Q::EMPTY + s, ((i / NS) - 1) & 1, abort)) break;
        if (a.test_starve && i == 0) continue;  // test hook: the first stage never arrives
        const int kv = t >= per;
        const int y = (int)((t - kv * per) * kRows);
        unsigned char* stg = smem + Q::OFF_STAGE + s * Q::STAGE;
        mbar_arrive_expect_tx(bar + Q::FULL + s, (uint32_t)Q::STAGE);
#pragma unroll
        for (int c = 0; c < Q::NC; ++c)
          tma_load_2d(stg + c * kRows * 128, kv ? &maps.v64 : &maps.k64, 64 * c, y, bar + Q::FULL + s);
        if (Q::R32)
          tma_load_2d(stg + Q::NC * kRows * 128, kv ? &maps.v32 : &maps.k32, 64 * Q::NC, y, bar + Q::FULL + s);
      }
      const uint32_t first = i > (uint32_t)NS ? i - NS : 0;
      for (uint32_t v = first; v < i; ++v) {
        if (a.test_starve && v == 0) continue;
        mbar_drain(bar + Q::FULL + v % NS, (v / NS) & 1);
      }
    }
  } else {
    // ============================================================ MMA issuer
    asm volatile("bar.sync 1, 288;" ::: "memory");  // B built by the epilogue warps
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, D, 0, 0) | (1u << 7) | (1u << 10);
      const uint32_t b0 = smem_u32(smem + Q::OFF_B), a0 = smem_u32(smem + Q::OFF_STAGE);
      uint32_t i = 0;
      for (int64_t t = blockIdx.x; t < total; t += gridDim.x, ++i) {
        const int s = i % NS, b = i % kNAcc;
        if (!mbar_wait(bar + Q::FULL + s, (i / NS) & 1, abort)) break;
        if (i >= kNAcc && !mbar_wait(bar + Q::DEMPTY + b, ((i / kNAcc) - 1) & 1, abort)) break;
        fence_after();
        const uint32_t as = a0 + s * Q::STAGE;
#pragma unroll
        for (int p = 0; p < 3; ++p)
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            // K step ks: chunk ks / 4 (128-byte swizzle), or the 32-element chunk
            const int c = ks >> 2;
            uint64_t da, db;
            if (c < Q::NC) {
              da = desc_sw(as + c * kRows * 128 + (ks & 3) * 32, 2, 1024);
              db = desc_sw(b0 + p * Q::PART + c * D * 128 + (ks & 3) * 32, 2, 1024);
            } else {
              const int kk = ks - 4 * Q::NC;
              da = desc_sw(as + Q::NC * kRows * 128 + kk * 32, 4, 512);
              db = desc_sw(b0 + p * Q::PART + Q::NC * D * 128 + kk * 32, 4, 512);
            }
            mma_ss(tbase + 128u * b, da, db, idesc, (p > 0 || ks > 0) ? 1u : 0u);
          }
        mma_commit(bar + Q::EMPTY + s);
        mma_commit(bar + Q::DFULL + b);
      }
      mma_commit(bar + Q::MMADONE);
      mbar_drain(bar + Q::MMADONE, 0);
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tbase, kTmemCols);
}

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

// rows x d bf16; boxes of `box` elements x 128 rows with the given swizzle
bool input_map(CUtensorMap* m, const void* base, int64_t rows, int d, int box, CUtensorMapSwizzle sw) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t boxd[2] = {(cuuint32_t)box, (cuuint32_t)kRows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, boxd, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const QuantizeArgs& a, cudaStream_t stream) {
  using Q = L<D>;
  static SmemLimitSet smem_set;
  const cudaError_t e = ensure_smem_limit(quantize_srft_tc_kernel<D>, Q::BYTES, smem_set);
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)a.B * a.Hkv * a.n_new;
  Maps m;
  memset(&m, 0, sizeof(m));
  if (Q::NC > 0 && (!input_map(&m.k64, a.k, rows, D, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
                    !input_map(&m.v64, a.v, rows, D, 64, CU_TENSOR_MAP_SWIZZLE_128B)))
    return cudaErrorInvalidValue;
  if (Q::R32 && (!input_map(&m.k32, a.k, rows, D, 32, CU_TENSOR_MAP_SWIZZLE_64B) ||
                 !input_map(&m.v32, a.v, rows, D, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
    return cudaErrorInvalidValue;
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = 2 * ((rows + kRows - 1) / kRows);
  const int grid = (int)(tiles < sms ? tiles : sms);
  quantize_srft_tc_kernel<D><<<grid, kThreads, Q::BYTES, stream>>>(a, m);
  return cudaGetLastError();
}

}  // namespace

bool quantize_srft_tc_supported(const QuantizeArgs& a) {
  const int64_t rows = (int64_t)a.B * a.Hkv * a.n_new;
  return (a.d == 32 || a.d == 64 || a.d == 96 || a.d == 128) && a.bf16 && !a.pos_is_ctx &&
         !a.butterfly_rotation && a.cb_bits == 0 && rows <= (int64_t)INT32_MAX - kRows &&
         encode_fn() != nullptr;
}

cudaError_t launch_quantize_srft_tc(const QuantizeArgs& a, cudaStream_t stream) {
  if (!quantize_srft_tc_supported(a)) return cudaErrorNotSupported;
  switch (a.d) {
    case 32: return launch_d<32>(a, stream);
    case 64: return launch_d<64>(a, stream);
    case 96: return launch_d<96>(a, stream);
    default: return launch_d<128>(a, stream);
  }
}

}  // namespace tq
