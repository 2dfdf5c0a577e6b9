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
//                         Hadamard path.
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
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kQWarps = 8;  // warps per quantize CTA
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * ((a.Hq + 1) / 2));
  cfg.blockDim = dim3(32 * M);
  cfg.dynamicSmemBytes = 0;
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
