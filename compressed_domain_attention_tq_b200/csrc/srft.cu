// srft.cu -- the SRFT variant of the rotation (SRFT post, core method): a
// sign-randomized Fourier transform in place of the Hadamard one, usable at
// any width d = 32 M (M = 1 .. 8, so also d = 96, 160, 192, 224), followed by
// a per-coordinate scale lambda before the group abs-max quantization.
//
// The transform is the orthonormal discrete Hartley transform F (real,
// symmetric, F F = I), computed two vectors at a time by srft.cuh.  With
// signs sigma and scales lambda_K, lambda_V:
//   stored K row  y_k = lambda_K (.) F (sigma (.) k)   (V likewise with lambda_V)
//   query         q_r = F (sigma (.) q) / lambda_K     so q_r . y_k = q . k
//   output        o   = sigma (.) F (o_r / lambda_V)
// Kernels:
//   srft_quantize_kernel  one warp per (sequence, kv head, token): K and V of
//                         the token form one complex transform; then group
//                         abs-max, int4 codes and the packed row layout of the
//                         Hadamard path.  For d = 128 and 256 the team kernel
//                         (srft_team.cuh: d / 16 lanes per token) does the same.
//   srft_query_kernel     one warp per pair of query heads -> q_r (fp32) in the
//                         decode workspace; the decode kernels read it instead
//                         of rotating q themselves.
//   srft_prep_kernel      one decode step's new-token quantization and query
//                         rotation in one launch (the fused step's first kernel).
//   srft_merge_kernel     one CTA per pair of query heads: the split-K log-sum-
//                         exp merge of each head, 1 / lambda_V, then one warp
//                         maps both heads back.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "srft.cuh"
#include "srft_team.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kQWarps = 8;  // warps per quantize CTA
constexpr int kTeamMinTokens = 64;  // appends of at least this many tokens per row use the team kernel
constexpr int64_t kSrftTcMinVectors = 8192;  // bulk appends of more vectors use the tensor-core kernel
constexpr float kRneMagic = 12582912.0f;                   // 1.5 * 2^23: x + M rounds x to an integer
constexpr float kBracketLo = 1.0f - 4.76837158203125e-07f;  // 1 - 2^-21 (exact)
constexpr float kBracketHi = 1.0f + 4.76837158203125e-07f;  // 1 + 2^-21 (exact)

// c = clamp(rne(fl32(x / s)), -7, 7) without a division per element: x is
// rounded with reciprocals bracketing 1/s from below and above (2^-21 apart,
// far more than their rounding error); rounding is monotone, so when both
// give the same integer it is rne(fl32(x / s)), else (x / s within ~1e-5 of a
// half-integer, or a subnormal s) the IEEE division decides.
__device__ __forceinline__ float int4_code(float x, float s, float r, bool big) {
  const float lo = fmaf(x, r * kBracketLo, kRneMagic), hi = fmaf(x, r * kBracketHi, kRneMagic);
  float c = lo - kRneMagic;
  if (big || lo != hi) c = rintf(__fdiv_rn(x, s));
  return fminf(fmaxf(c, -7.0f), 7.0f);
}

// Per-lane constants of the SRFT quantizer: signs at j = lane + 32 j2 and
// lambda / (2 sqrt d) at k = k2 + M brev5(lane).
template <int M>
struct SrftLaneConsts {
  float sg[M], mk[M], mv[M];
  __device__ __forceinline__ void load(const QuantizeArgs& a, int lane) {
    constexpr int D = 32 * M;
    const float norm = 0.5f / sqrtf((float)D);
#pragma unroll
    for (int j2 = 0; j2 < M; ++j2) sg[j2] = a.signs ? (float)a.signs[lane + 32 * j2] : 1.0f;
#pragma unroll
    for (int k2 = 0; k2 < M; ++k2) {
      const int k = k2 + M * brev5(lane);
      mk[k2] = a.lambda_k ? norm * a.lambda_k[k] : norm;
      mv[k2] = a.lambda_v ? norm * a.lambda_v[k] : norm;
    }
  }
};

// One warp quantizes the K and V rows of vector pair p ((sequence, kv head)
// row-major, then token) into the cache; yk, yv: this warp's 2 x d floats of
// shared memory for the transpose.
template <int M>
__device__ __forceinline__ void srft_quantize_pair(const QuantizeArgs& a, int p,
                                                   const HartleyTwiddles<M>& tw,
                                                   const SrftLaneConsts<M>& lc, float* yk, float* yv,
                                                   int lane) {
  constexpr int D = 32 * M;
  const int bh = p / a.n_new, n = p % a.n_new;
  const int b = bh / a.Hkv;
  int64_t pos = (int64_t)a.pos[b] + n;
  if (a.pos_is_ctx) pos = (int64_t)min(max(a.pos[b], 1), a.max_ctx) - 1 + n;
  if (pos < 0 || pos >= a.capacity) return;  // the whole warp
  const int64_t row = (int64_t)bh * a.capacity + pos;
  float re[M], im[M];
#pragma unroll
  for (int j2 = 0; j2 < M; ++j2) {
    const int64_t idx = (int64_t)p * D + lane + 32 * j2;
    float xk, xv;
    if (a.bf16) {
      xk = __uint_as_float((uint32_t)static_cast<const uint16_t*>(a.k)[idx] << 16);
      xv = __uint_as_float((uint32_t)static_cast<const uint16_t*>(a.v)[idx] << 16);
    } else {
      xk = static_cast<const float*>(a.k)[idx];
      xv = static_cast<const float*>(a.v)[idx];
    }
    re[j2] = lc.sg[j2] * xk;
    im[j2] = lc.sg[j2] * xv;
  }
  float hx[M], hy[M];
  hartley_pair_warp<M>(re, im, tw, hx, hy);
#pragma unroll
  for (int k2 = 0; k2 < M; ++k2) {
    const int k = k2 + M * brev5(lane);
    yk[k] = hx[k2] * lc.mk[k2];
    yv[k] = hy[k2] * lc.mv[k2];
  }
  __syncwarp();
  // lane holds in-group coordinate j = lane of every group g (coordinate 32 g + lane)
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    const float* y = kv ? yv : yk;
    uint8_t* prow = (kv ? a.v_packed : a.k_packed) + row * (D / 2);
    float* srow = (kv ? a.v_scales : a.k_scales) + row * M;
#pragma unroll
    for (int g = 0; g < M; ++g) {
      const float x = y[32 * g + lane];
      float amax = fabsf(x);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s = __fdiv_rn(amax, 7.0f);
      const float r = s > 0.0f ? __frcp_rn(s) : 0.0f;
      const float c = s > 0.0f ? int4_code(x, s, r, !(r <= 3.0e38f)) : 0.0f;
      // byte (j / 4) * 2M + 2 g + (j % 4) / 2, nibble j % 2: four lanes make one half-word
      // c + 1.5 * 2^23 has the bits 0x4B400000 + c: its low nibble is c's two's complement
      uint32_t nib = (__float_as_uint(c + kRneMagic) & 0xFu) << (4 * (lane & 3));
      nib |= __shfl_xor_sync(0xffffffffu, nib, 1);
      nib |= __shfl_xor_sync(0xffffffffu, nib, 2);
      if ((lane & 3) == 0)
        *reinterpret_cast<uint16_t*>(prow + (lane >> 2) * 2 * M + 2 * g) = (uint16_t)nib;
      if (lane == g) srow[g] = s;
    }
  }
  __syncwarp();
}

template <int M>
__global__ void __launch_bounds__(32 * kQWarps) srft_quantize_kernel(QuantizeArgs a) {
  constexpr int D = 32 * M;
  __shared__ float ybuf[kQWarps][2][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  HartleyTwiddles<M> tw;
  hartley_twiddles<M>(tw, lane);
  SrftLaneConsts<M> lc;
  lc.load(a, lane);
  const int pairs = a.B * a.Hkv * a.n_new;  // < 2^31 (checked on the host)
  for (int p = blockIdx.x * kQWarps + warp; p < pairs; p += gridDim.x * kQWarps)
    srft_quantize_pair<M>(a, p, tw, lc, ybuf[warp][0], ybuf[warp][1], lane);
}

// Per-CTA tables of the team quantizer: signs (+-1) and lambda / (2 sqrt d).
template <int D>
struct TeamTables {
  float sgn[D], lk[D], lv[D];
  __device__ __forceinline__ void build(const QuantizeArgs& a) {
    const float norm = 0.5f / sqrtf((float)D);
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      sgn[i] = a.signs ? (float)a.signs[i] : 1.0f;
      lk[i] = a.lambda_k ? norm * a.lambda_k[i] : norm;
      lv[i] = a.lambda_v ? norm * a.lambda_v[i] : norm;
    }
  }
};

// Cache row of vector pair p ((sequence, kv head) row-major, then token), or
// false when its position is outside the cache.
__device__ __forceinline__ bool team_pair_row(const QuantizeArgs& a, int p, int64_t& row) {
  const int bh = p / a.n_new, n = p - bh * a.n_new;
  const int b = bh / a.Hkv;
  int64_t pos = (int64_t)a.pos[b] + n;
  if (a.pos_is_ctx) pos = (int64_t)min(max(a.pos[b], 1), a.max_ctx) - 1 + n;
  row = (int64_t)bh * a.capacity + pos;
  return pos >= 0 && pos < a.capacity;
}

// Team lane t (of P) quantizes one vector pair from re = sigma (.) k and
// im = sigma (.) v at j = t + P j2 into cache row `row` (stores only if ok;
// a team without a pair still takes part in the shuffles).  After the
// transform the lane owns coordinates 16 k1 .. 16 k1 + 15 (k1 = brev(t)):
// half of group k1 / 2, whose other half is in lane t ^ P/2; its codes are
// four half-words of the packed row, at byte (j / 4) * 2 ng + 2 g for the
// in-group coordinates j = 16 (k1 % 2) + 4 q .. 4 q + 3.
template <int P>
__device__ __forceinline__ void srft_quantize_team(const QuantizeArgs& a, int64_t row, bool ok,
                                                   const float (&re)[16], const float (&im)[16],
                                                   const TeamConsts<P>& c,
                                                   const TeamTables<16 * P>& tb, int t,
                                                   int team_base) {
  constexpr int D = 16 * P, NG = D / 32, L = TeamConsts<P>::L;
  float hx[16], hy[16];
  hartley_pair_team<P>(re, im, c, team_base, hx, hy);
  const int k1 = brev_bits<L>(t), g = k1 >> 1, half = k1 & 1;
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
    const float* lam = (kv ? tb.lv : tb.lk) + 16 * k1;
    const float* h = kv ? hy : hx;
    float y[16];  // coordinate 16 k1 + k2 in y[k2]
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 l = reinterpret_cast<const float4*>(lam)[q];
      y[4 * q] = h[brev4c(4 * q)] * l.x;
      y[4 * q + 1] = h[brev4c(4 * q + 1)] * l.y;
      y[4 * q + 2] = h[brev4c(4 * q + 2)] * l.z;
      y[4 * q + 3] = h[brev4c(4 * q + 3)] * l.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int k2 = 0; k2 < 16; ++k2) amax = fmaxf(amax, fabsf(y[k2]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, P / 2));
    const float s = __fdiv_rn(amax, 7.0f);
    const float r = s > 0.0f ? __frcp_rn(s) : 0.0f;
    // int4_code's bracketed reciprocals, unrolled: where both brackets give the
    // same integer, x * r_lo + 1.5 * 2^23 has the bits 0x4B400000 + c, so its
    // low nibble is the code's two's complement (|x / s| <= 7, so no clamp
    // binds); if any of the lane's 16 disagree (or s is subnormal) the lane
    // redoes them with the IEEE division, as int4_code does
    const float rl = r * kBracketLo, rh = r * kBracketHi;
    bool slow = !(r <= 3.0e38f);
    uint32_t hw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      hw[q] = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = fmaf(y[4 * q + e], rl, kRneMagic), hi = fmaf(y[4 * q + e], rh, kRneMagic);
        slow |= lo != hi;
        hw[q] |= (__float_as_uint(lo) & 0xFu) << (4 * e);
      }
    }
    if (slow) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        hw[q] = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float cc =
              s > 0.0f ? fminf(fmaxf(rintf(__fdiv_rn(y[4 * q + e], s)), -7.0f), 7.0f) : 0.0f;
          hw[q] |= (__float_as_uint(cc + kRneMagic) & 0xFu) << (4 * e);
        }
      }
    }
    uint8_t* prow = (kv ? a.v_packed : a.k_packed) + row * (D / 2);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (ok) *reinterpret_cast<uint16_t*>(prow + (4 * half + q) * 2 * NG + 2 * g) = (uint16_t)hw[q];
    if (ok && half == 0) ((kv ? a.v_scales : a.k_scales) + row * NG)[g] = s;
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// Bulk quantize-append for d = 16 P: each warp takes 32 / P pairs per step,
// grid-stride.  bf16 inputs are staged in shared memory by 16-byte async
// copies one step ahead (two buffers per warp; a pair's K and V rows at a
// pitch of 4 d + 16 bytes, so the teams' 2-byte reads fall in distinct
// banks); fp32 inputs are loaded directly.
template <int P>
__global__ void __launch_bounds__(256) srft_quantize_team_kernel(QuantizeArgs a) {
  constexpr int D = 16 * P, TPW = 32 / P;
  constexpr int PITCH = 4 * D + 16;           // bytes per staged pair (bf16 K row, V row, pad)
  constexpr int CHUNKS = TPW * (4 * D / 16);  // 16-byte copies per warp step (= 128)
  static_assert(CHUNKS == 128, "four copies per lane");
  __shared__ __align__(16) TeamTables<D> tb;
  __shared__ __align__(16) unsigned char stage[8][2][TPW * PITCH];
  tb.build(a);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = lane & (P - 1), team_base = lane & ~(P - 1), q = lane / P;
  TeamConsts<P> c;
  team_consts<P>(c, t);
  const int pairs = a.B * a.Hkv * a.n_new;  // < 2^31 (checked on the host)
  const int stride = gridDim.x * 8 * TPW;
  const int base0 = (blockIdx.x * 8 + warp) * TPW;
  if (!a.bf16) {
    for (int base = base0; base < pairs; base += stride) {
      const int p = base + q;
      int64_t row = 0;
      const bool ok = p < pairs && team_pair_row(a, p, row);
      float re[16], im[16];
#pragma unroll
      for (int j2 = 0; j2 < 16; ++j2) {
        const int j = t + P * j2;
        const float sg = tb.sgn[j];
        re[j2] = ok ? sg * static_cast<const float*>(a.k)[(int64_t)p * D + j] : 0.0f;
        im[j2] = ok ? sg * static_cast<const float*>(a.v)[(int64_t)p * D + j] : 0.0f;
      }
      srft_quantize_team<P>(a, row, ok, re, im, c, tb, t, team_base);
    }
    return;
  }
  // copies of one warp step: chunk i covers bytes 16 w .. of pair base + qq's K (kv = 0) or V row
  auto issue = [&](int base, unsigned char* buf) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int ch = lane + 32 * r;
      const int qq = ch / (4 * D / 16), w = ch % (4 * D / 16);
      const int kv = w / (2 * D / 16), off = 16 * (w % (2 * D / 16));
      const int p = base + qq;
      if (p < pairs)
        cp_async16(buf + qq * PITCH + kv * 2 * D + off,
                   static_cast<const unsigned char*>(kv ? a.v : a.k) + (int64_t)p * 2 * D + off);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (base0 < pairs) issue(base0, stage[warp][0]);
  int it = 0;
  for (int base = base0; base < pairs; base += stride, ++it) {
    const int nb = base + stride;
    if (nb < pairs) issue(nb, stage[warp][(it + 1) & 1]);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncwarp();
    const unsigned char* buf = stage[warp][it & 1] + q * PITCH;
    const int p = base + q;
    int64_t row = 0;
    const bool ok = p < pairs && team_pair_row(a, p, row);
    float re[16], im[16];
#pragma unroll
    for (int j2 = 0; j2 < 16; ++j2) {
      const int j = t + P * j2;
      const float sg = tb.sgn[j];
      const uint32_t uk = reinterpret_cast<const uint16_t*>(buf)[j];
      const uint32_t uv = reinterpret_cast<const uint16_t*>(buf + 2 * D)[j];
      re[j2] = ok ? sg * __uint_as_float(uk << 16) : 0.0f;
      im[j2] = ok ? sg * __uint_as_float(uv << 16) : 0.0f;
    }
    srft_quantize_team<P>(a, row, ok, re, im, c, tb, t, team_base);
    __syncwarp();  // every lane is done with this buffer before it is refilled
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// One warp rotates query heads h0 = 2 (p mod ceil(Hq/2)) and h0 + 1 of sequence
// p / ceil(Hq/2) into the workspace: q_rot = F (signs (.) q) / lambda_K.
template <int M>
__device__ __forceinline__ void srft_query_pair(const DecodeArgs& a, int64_t p,
                                                const HartleyTwiddles<M>& tw, int lane) {
  constexpr int D = 32 * M;
  const int pairs_per_b = (a.Hq + 1) / 2;
  const int b = (int)(p / pairs_per_b), h0 = 2 * (int)(p % pairs_per_b);
  const bool two = h0 + 1 < a.Hq;
  float re[M], im[M];
  const int64_t base0 = ((int64_t)b * a.Hq + h0) * D;
#pragma unroll
  for (int j2 = 0; j2 < M; ++j2) {
    const int j = lane + 32 * j2;
    const float sg = a.signs ? (float)a.signs[j] : 1.0f;
    float x0, x1 = 0.0f;
    if (a.q_bf16) {
      const uint16_t* q = static_cast<const uint16_t*>(a.q);
      x0 = __uint_as_float((uint32_t)q[base0 + j] << 16);
      if (two) x1 = __uint_as_float((uint32_t)q[base0 + D + j] << 16);
    } else {
      const float* q = static_cast<const float*>(a.q);
      x0 = q[base0 + j];
      if (two) x1 = q[base0 + D + j];
    }
    re[j2] = sg * x0;
    im[j2] = sg * x1;
  }
  float hx[M], hy[M];
  hartley_pair_warp<M>(re, im, tw, hx, hy);
  const float norm = 0.5f / sqrtf((float)D);
  float* q_rot = const_cast<float*>(a.q_rot);
#pragma unroll
  for (int k2 = 0; k2 < M; ++k2) {
    const int k = k2 + M * brev5(lane);
    const float mul = a.lambda_k ? __fdiv_rn(norm, a.lambda_k[k]) : norm;
    q_rot[base0 + k] = hx[k2] * mul;
    if (two) q_rot[base0 + D + k] = hy[k2] * mul;
  }
}

template <int M>
__global__ void __launch_bounds__(128) srft_query_kernel(DecodeArgs a) {
  // the decode kernel may start streaming the cache now; it waits for this
  // grid (griddepcontrol.wait) before it reads the rotated queries
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t p = (int64_t)blockIdx.x * 4 + warp;
  if (p >= (int64_t)a.B * ((a.Hq + 1) / 2)) return;  // the whole warp
  HartleyTwiddles<M> tw;
  hartley_twiddles<M>(tw, lane);
  srft_query_pair<M>(a, p, tw, lane);
}

// One decode step's preparation in one launch: warps [0, npk) quantize the new
// token's K/V pairs (one per sequence and kv head) into the cache, the next
// warps rotate the query pairs.
template <int M>
__global__ void __launch_bounds__(128) srft_prep_kernel(QuantizeArgs qa, DecodeArgs a) {
  constexpr int D = 32 * M;
  // the decode may start streaming now: it waits for this grid before it reads the
  // rotated queries and before it copies a sequence's last (appended) row
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float ybuf[4][2][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * 4 + warp;
  const int npk = qa.B * qa.Hkv * qa.n_new;
  const int64_t npq = (int64_t)a.B * ((a.Hq + 1) / 2);
  if (w >= npk + npq) return;  // the whole warp
  HartleyTwiddles<M> tw;
  hartley_twiddles<M>(tw, lane);
  if (w < npk) {
    SrftLaneConsts<M> lc;
    lc.load(qa, lane);
    srft_quantize_pair<M>(qa, (int)w, tw, lc, ybuf[warp][0], ybuf[warp][1], lane);
  } else {
    srft_query_pair<M>(a, w - npk, tw, lane);
  }
}

template <int M>
__global__ void __launch_bounds__(32 * M) srft_merge_kernel(DecodeArgs a) {
  constexpr int D = 32 * M;
  __shared__ float z[2][D];
  const int pairs_per_b = (a.Hq + 1) / 2;
  const int b = blockIdx.x / pairs_per_b, h0 = 2 * (blockIdx.x % pairs_per_b);
  const bool two = h0 + 1 < a.Hq;
  const int i = threadIdx.x, lane = i & 31;
  // everything that does not depend on the split-K partials runs before the wait
  HartleyTwiddles<M> tw;
  if (i < 32) hartley_twiddles<M>(tw, lane);
  const int raw = a.ctx_lens[b];
  const int T = raw < 1 ? 1 : (raw > a.max_ctx ? a.max_ctx : raw);
  const int nc = (T + a.plan.chunk - 1) / a.plan.chunk;
  const int stride = a.plan.part_stride;
  const float lv = a.lambda_v ? a.lambda_v[i] : 1.0f;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float* p0 = reinterpret_cast<const float*>(static_cast<const unsigned char*>(a.workspace) +
                                                   a.plan.header_bytes) +
                    ((int64_t)b * a.Hq + h0) * a.plan.n_chunks * stride;
  const float* p1 = two ? p0 + (int64_t)a.plan.n_chunks * stride : p0;
  // log-sum-exp merge of both heads' chunks: M = max m_c, o = sum 2^(m_c - M) acc_c / sum 2^(m_c - M) l_c
  float M0 = -INFINITY, M1 = -INFINITY;
  for (int c = 0; c < nc; ++c) {
    M0 = fmaxf(M0, p0[(int64_t)c * stride + D]);
    M1 = fmaxf(M1, p1[(int64_t)c * stride + D]);
  }
  constexpr int U = 4;
  float a0[U], l0[U], a1[U], l1[U];
#pragma unroll
  for (int k = 0; k < U; ++k) a0[k] = l0[k] = a1[k] = l1[k] = 0.0f;
  for (int c0 = 0; c0 < nc; c0 += U) {
#pragma unroll
    for (int k = 0; k < U; ++k)
      if (c0 + k < nc) {
        const float* q0 = p0 + (int64_t)(c0 + k) * stride;
        const float* q1 = p1 + (int64_t)(c0 + k) * stride;
        const float w0 = exp2f(q0[D] - M0), w1 = exp2f(q1[D] - M1);
        l0[k] = fmaf(w0, q0[D + 1], l0[k]);
        a0[k] = fmaf(w0, q0[i], a0[k]);
        l1[k] = fmaf(w1, q1[D + 1], l1[k]);
        a1[k] = fmaf(w1, q1[i], a1[k]);
      }
  }
  const float L0 = (l0[0] + l0[2]) + (l0[1] + l0[3]), L1 = (l1[0] + l1[2]) + (l1[1] + l1[3]);
  z[0][i] = ((a0[0] + a0[2]) + (a0[1] + a0[3])) / L0 / lv;
  z[1][i] = two ? ((a1[0] + a1[2]) + (a1[1] + a1[3])) / L1 / lv : 0.0f;
  if (a.lse != nullptr && i == 0) {
    *reinterpret_cast<float2*>(a.lse + ((int64_t)b * a.Hq + h0) * 2) = make_float2(M0, L0);
    if (two) *reinterpret_cast<float2*>(a.lse + ((int64_t)b * a.Hq + h0 + 1) * 2) = make_float2(M1, L1);
  }
  __syncthreads();
  if (i >= 32) return;
  float re[M], im[M];
#pragma unroll
  for (int j2 = 0; j2 < M; ++j2) {
    re[j2] = z[0][lane + 32 * j2];
    im[j2] = z[1][lane + 32 * j2];
  }
  float hx[M], hy[M];
  hartley_pair_warp<M>(re, im, tw, hx, hy);
  const float norm = 0.5f / sqrtf((float)D);
  const int64_t base0 = ((int64_t)b * a.Hq + h0) * D;
#pragma unroll
  for (int k2 = 0; k2 < M; ++k2) {
    const int k = k2 + M * brev5(lane);
    const float sg = a.signs ? (float)a.signs[k] * norm : norm;
    a.out[base0 + k] = hx[k2] * sg;
    if (two) a.out[base0 + D + k] = hy[k2] * sg;
  }
}

template <int M>
cudaError_t launch_quantize_srft_m(const QuantizeArgs& a, cudaStream_t stream) {
  const int64_t pairs = (int64_t)a.B * a.Hkv * a.n_new;
  // bulk bf16 appends at d <= 128: the transform as a tensor-core product
  if (2 * pairs > kSrftTcMinVectors && quantize_srft_tc_supported(a)) return launch_quantize_srft_tc(a, stream);
  // d = 128, 256 with a prefill-sized n_new: d / 16 lanes per pair.  Appends of
  // fewer tokens keep the one-warp kernel, the transform of the decode step's
  // fused append, so both give the same rows; the team kernel's own rounding
  // (another factorisation of the same DFT) can differ from it in the last bit.
  if constexpr (M == 4 || M == 8) {
    if (a.n_new >= kTeamMinTokens) {
      constexpr int TPW = 16 / M;  // pairs per warp
      int64_t blocks = (pairs + 8 * TPW - 1) / (8 * TPW);
      const int64_t cap = (int64_t)kSmCount * 8;
      if (blocks > cap) blocks = cap;
      srft_quantize_team_kernel<2 * M><<<(unsigned)blocks, 256, 0, stream>>>(a);
      return cudaGetLastError();
    }
  }
  int64_t blocks = (pairs + kQWarps - 1) / kQWarps;
  const int64_t cap = (int64_t)kSmCount * (M <= 4 ? 8 : 4);
  if (blocks > cap) blocks = cap;
  srft_quantize_kernel<M><<<(unsigned)blocks, 32 * kQWarps, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int M>
cudaError_t launch_srft_query_m(const DecodeArgs& a, cudaStream_t stream) {
  const int64_t warps = (int64_t)a.B * ((a.Hq + 1) / 2);
  srft_query_kernel<M><<<(unsigned)((warps + 3) / 4), 128, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int M>
cudaError_t launch_srft_prep_m(const QuantizeArgs& qa, const DecodeArgs& a, cudaStream_t stream) {
  const int64_t warps = (int64_t)qa.B * qa.Hkv * qa.n_new + (int64_t)a.B * ((a.Hq + 1) / 2);
  srft_prep_kernel<M><<<(unsigned)((warps + 3) / 4), 128, 0, stream>>>(qa, a);
  return cudaGetLastError();
}

template <int M>
cudaError_t launch_srft_merge_m(const DecodeArgs& a, cudaStream_t stream) {
  static SmemLimitSet smem_set;
  const cudaError_t e = ensure_smem_limit(srft_merge_kernel<M>, kMergeSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * ((a.Hq + 1) / 2));
  cfg.blockDim = dim3(32 * M);
  cfg.dynamicSmemBytes = merge_smem_bytes((long long)a.B * ((a.Hq + 1) / 2));  // residency cap, not used
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, srft_merge_kernel<M>, a);
}

#define TQ_SRFT_DISPATCH(FN, ARG)            \
  switch (d / 32) {                          \
    case 1: return FN<1>(ARG, stream);       \
    case 2: return FN<2>(ARG, stream);       \
    case 3: return FN<3>(ARG, stream);       \
    case 4: return FN<4>(ARG, stream);       \
    case 5: return FN<5>(ARG, stream);       \
    case 6: return FN<6>(ARG, stream);       \
    case 7: return FN<7>(ARG, stream);       \
    case 8: return FN<8>(ARG, stream);       \
    default: return cudaErrorInvalidValue;   \
  }

}  // namespace

bool srft_head_dim_supported(int d) { return d >= 32 && d <= 256 && d % 32 == 0; }

cudaError_t launch_quantize_srft(const QuantizeArgs& a, cudaStream_t stream) {
  const int d = a.d;
  TQ_SRFT_DISPATCH(launch_quantize_srft_m, a)
}

cudaError_t launch_srft_query(const DecodeArgs& a, cudaStream_t stream) {
  const int d = a.d;
  TQ_SRFT_DISPATCH(launch_srft_query_m, a)
}

cudaError_t launch_merge_srft(const DecodeArgs& a, cudaStream_t stream) {
  const int d = a.d;
  TQ_SRFT_DISPATCH(launch_srft_merge_m, a)
}

cudaError_t launch_srft_prep(const QuantizeArgs& qa, const DecodeArgs& a, cudaStream_t stream) {
  switch (a.d / 32) {
    case 1: return launch_srft_prep_m<1>(qa, a, stream);
    case 2: return launch_srft_prep_m<2>(qa, a, stream);
    case 3: return launch_srft_prep_m<3>(qa, a, stream);
    case 4: return launch_srft_prep_m<4>(qa, a, stream);
    case 5: return launch_srft_prep_m<5>(qa, a, stream);
    case 6: return launch_srft_prep_m<6>(qa, a, stream);
    case 7: return launch_srft_prep_m<7>(qa, a, stream);
    case 8: return launch_srft_prep_m<8>(qa, a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
