// merge.cu -- the second kernel of every decode call: combines the split-K
// partials of each (sequence, query head) by log-sum-exp and rotates the
// result back to the unrotated basis.
//
// Partial c of a head holds (acc[0..d), m, l): the chunk's unnormalized sum
// of p v in the rotated basis, its running max m (log2 units) and sum l.
//   M = max_c m_c,  w_c = 2^(m_c - M),  o_rot = sum_c w_c acc_c / sum_c w_c l_c
//   o = R^T o_rot = diag(signs) H o_rot / sqrt(d)   (R = H diag(signs) / sqrt(d))
// (Open-TQ-Metal abstract: the attention output is that of the compressed
// cache; the query was rotated by the cache's signs, so V's output is rotated
// back.)
//
// One CTA of d threads (thread i: output coordinate i) per (sequence, query
// head), launched with programmatic stream serialization: it may start while
// the split-K kernel drains and waits at griddepcontrol.wait before reading
// partials.
#include <math.h>

#include "tq_internal.h"

namespace tq {
namespace {

template <int D>
__global__ void __launch_bounds__(D) merge_kernel(DecodeArgs a) {
  __shared__ float o[D];  // cross-warp butterfly stages
  const int b = blockIdx.x / a.Hq;
  const int hq = blockIdx.x % a.Hq;
  const int i = threadIdx.x, lane = i & 31;
  // inputs the split-K kernel does not write are read before waiting for it
  const int raw = a.ctx_lens[b];
  const float sgn = a.signs ? (float)a.signs[i] : 1.0f;
  const int T = raw < 1 ? 1 : (raw > a.max_ctx ? a.max_ctx : raw);
  const int nc = (T + a.plan.chunk - 1) / a.plan.chunk;
  const int stride = a.plan.part_stride;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float* part = reinterpret_cast<const float*>(static_cast<const unsigned char*>(a.workspace) +
                                                     a.plan.header_bytes) +
                      ((int64_t)b * a.Hq + hq) * a.plan.n_chunks * stride;

  // Every thread reads the chunks' (m, l) itself (the same addresses across the
  // block: broadcast loads), so no block-wide reductions are needed.
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, part[(int64_t)c * stride + D]);
  constexpr int U = 8;  // chunks in flight per thread
  float acc[U], lsum[U];
#pragma unroll
  for (int k = 0; k < U; ++k) acc[k] = lsum[k] = 0.0f;
  for (int c0 = 0; c0 < nc; c0 += U) {
    float2 ml[U];
    float v[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const bool ok = c0 + k < nc;
      const float* pc = part + (int64_t)(c0 + k) * stride;
      ml[k] = ok ? *reinterpret_cast<const float2*>(pc + D) : make_float2(-INFINITY, 0.0f);
      v[k] = ok ? pc[i] : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < U; ++k)
      if (c0 + k < nc) {
        const float w = exp2f(ml[k].x - M);  // NaN if a partial is NaN
        lsum[k] = fmaf(w, ml[k].y, lsum[k]);
        acc[k] = fmaf(w, v[k], acc[k]);
      }
  }
#pragma unroll
  for (int k = U / 2; k > 0; k >>= 1)
#pragma unroll
    for (int j = 0; j < k; ++j) {
      acc[j] += acc[j + k];
      lsum[j] += lsum[j + k];
    }
  const float L = lsum[0];
  float x = acc[0] / L;

  if (a.signs) {  // o = diag(signs) H o / sqrt(d), H in Sylvester order, bits 1, 2, 4, ...
#pragma unroll
    for (int bit = 1; bit < 32; bit <<= 1) {  // coordinate bits within the warp
      const float other = __shfl_xor_sync(0xffffffffu, x, bit);
      x = (lane & bit) ? other - x : x + other;
    }
#pragma unroll
    for (int bit = 32; bit < D; bit <<= 1) {  // across warps
      o[i] = x;
      __syncthreads();
      const float other = o[i ^ bit];
      __syncthreads();
      x = (i & bit) ? other - x : x + other;
    }
    x = x * sgn * rsqrtf((float)D);
  }
  a.out[((int64_t)b * a.Hq + hq) * D + i] = x;
  if (a.lse != nullptr && i == 0)  // the head's softmax state, for merging across contexts
    *reinterpret_cast<float2*>(a.lse + ((int64_t)b * a.Hq + hq) * 2) = make_float2(M, L);
}

// Outputs of several context parts of the same heads (each normalized, with
// its (max, sum) in log2 units) -> the output over their union:
//   M = max_r m_r,  w_r = 2^(m_r - M) l_r,  o = sum_r w_r o_r / sum_r w_r.
__global__ void __launch_bounds__(256) merge_lse_kernel(const float* __restrict__ outs,
                                                        const float* __restrict__ lses, int n_parts,
                                                        int64_t n_heads, int d, float* __restrict__ out) {
  const int64_t total = n_heads * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t h = idx / d;
    float M = -INFINITY;
    for (int r = 0; r < n_parts; ++r) M = fmaxf(M, lses[((int64_t)r * n_heads + h) * 2]);
    float num = 0.0f, den = 0.0f;
    for (int r = 0; r < n_parts; ++r) {
      const float2 ml = *reinterpret_cast<const float2*>(lses + ((int64_t)r * n_heads + h) * 2);
      const float w = exp2f(ml.x - M) * ml.y;  // NaN if a part is NaN
      num = fmaf(w, outs[(int64_t)r * total + idx], num);
      den += w;
    }
    out[idx] = num / den;
  }
}

template <int D>
cudaError_t launch_merge_d(const DecodeArgs& a, cudaStream_t stream) {
  static SmemLimitSet smem_set;
  const cudaError_t e = ensure_smem_limit(merge_kernel<D>, kMergeSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Hq);
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = merge_smem_bytes((long long)a.B * a.Hq);  // residency cap, not used
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel<D>, a);
}

}  // namespace

cudaError_t launch_merge_lse(const float* outs, const float* lses, int n_parts, int64_t n_heads,
                             int d, float* out, cudaStream_t stream) {
  const int64_t total = n_heads * d;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  merge_lse_kernel<<<(unsigned)blocks, 256, 0, stream>>>(outs, lses, n_parts, n_heads, d, out);
  return cudaGetLastError();
}

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_merge_d<128>(a, stream) : launch_merge_d<256>(a, stream);
}

}  // namespace tq
