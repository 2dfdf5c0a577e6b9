// decode_simt.cu -- split-K decode attention on the packed int4 cache using
// CUDA cores (the path for GQA shapes the tensor-core decode does not cover).
//
// Attention runs directly on the packed codes ("fused sdpa_int4",
// Open-TQ-Metal abstract): codes are unpacked in registers and scaled by
// their group's fp32 scale inside the dot products; no dequantized K/V matrix
// is written anywhere (forum summary, section "eliminating intermediate
// matrices").  Softmax runs online with a running maximum and fp32 sums
// (section "numerical stability").
//
// CTA (chunk, kv head, sequence): loads the G = Hq/Hkv query rows, rotates
// them with the cache's signs, then streams the chunk's K/V tiles through
// shared memory.  Each chunk leaves (running max m in log2 units, sum l,
// unnormalized acc[d]) per query head in the workspace; merge.cu combines the
// chunks and rotates the result back.
#include <cuda_bf16.h>
#include <math.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTile = 64;

// code of in-group coordinate j of group g in a packed row (d = 32*ng)
__device__ __forceinline__ int nibble_at(const uint8_t* row, int ng, int g, int j) {
  const int byte = (j / 4) * (2 * ng) + 2 * g + (j % 4) / 2;
  const int v = (row[byte] >> (4 * (j % 2))) & 0xF;
  return v >= 8 ? v - 16 : v;
}

// In-place Walsh-Hadamard transform of `n` rows of length D in shared memory
// (Sylvester order), all threads of the block participating.
template <int D>
__device__ void fwht_rows(float* buf, int n) {
  for (int bit = 1; bit < D; bit <<= 1) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < n * (D / 2); idx += blockDim.x) {
      const int r = idx / (D / 2), k = idx % (D / 2);
      const int lo = ((k & ~(bit - 1)) << 1) | (k & (bit - 1));
      float* row = buf + r * D;
      const float u = row[lo], w = row[lo | bit];
      row[lo] = u + w;
      row[lo | bit] = u - w;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ float load_q(const void* q, int bf16, int64_t idx) {
  if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16*>(q)[idx]);
  return static_cast<const float*>(q)[idx];
}

__device__ __forceinline__ int clamp_ctx(int T, int max_ctx) {
  return T < 1 ? 1 : (T > max_ctx ? max_ctx : T);
}

template <int D>
__global__ void __launch_bounds__(128) decode_simt_kernel(DecodeArgs a) {
  constexpr int NG = D / 32, ROWB = D / 2, ROWP = ROWB + 16;
  constexpr int SLICES = D / 8;                 // 8-coordinate slices per head
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int raw_T = a.ctx_lens[b];
  const int T = clamp_ctx(raw_T, a.max_ctx);
  if (chunk == 0 && kvh == 0 && threadIdx.x == 0)
    static_cast<int32_t*>(a.workspace)[b] = (raw_T < 1 || raw_T > a.max_ctx) ? 1 : 0;
  const int t_begin = chunk * a.plan.chunk;
  if (t_begin >= T) return;
  const int t_end = min(T, t_begin + a.plan.chunk);

  extern __shared__ __align__(16) unsigned char smem[];
  float* qs = reinterpret_cast<float*>(smem);                  // [G][D]
  float* sp = qs + G * D;                                      // [G][kTile] scores / probs
  float* kscale = sp + G * kTile;                              // [kTile][NG]
  float* vscale = kscale + kTile * NG;                         // [kTile][NG]
  float* mstate = vscale + kTile * NG;                         // [G] running max (log2)
  float* lstate = mstate + 16;                                 // [G] running sum
  float* alpha = lstate + 16;                                  // [G] rescale of this tile
  uint8_t* ktile = reinterpret_cast<uint8_t*>(alpha + 16);     // [kTile][ROWP]
  uint8_t* vtile = ktile + kTile * ROWP;

  // q' = attn_scale * log2(e) * R q (the SRFT variant's R q comes rotated in q_rot)
  const int64_t qbase = ((int64_t)b * a.Hq + (int64_t)kvh * G) * D;
  const bool wht = a.signs != nullptr && a.q_rot == nullptr;
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    float x;
    if (a.q_rot != nullptr) {
      x = a.q_rot[qbase + i];
    } else {
      x = load_q(a.q, a.q_bf16, qbase + i);
      if (a.signs) x *= (float)a.signs[i % D];
    }
    qs[i] = x;
  }
  if constexpr ((D & (D - 1)) == 0) {
    if (wht) fwht_rows<D>(qs, G);
  }
  const float qmul = a.attn_scale * kLog2e * (wht ? rsqrtf((float)D) : 1.0f);
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) qs[i] *= qmul;
  if (threadIdx.x < 16) {
    mstate[threadIdx.x] = -INFINITY;
    lstate[threadIdx.x] = 0.0f;
  }

  // PV work items: (head, 8-coordinate slice); at most 4 per thread.
  const int items = G * SLICES;
  float acc[4][8];
#pragma unroll
  for (int it = 0; it < 4; ++it)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[it][e] = 0.0f;

  const int64_t rowbase = ((int64_t)b * a.Hkv + kvh) * a.capacity;
  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int nt = min(kTile, t_end - t0);
    __syncthreads();
    // stage the tile's packed rows and scales
    for (int idx = threadIdx.x; idx < nt * (ROWB / 16); idx += blockDim.x) {
      const int r = idx / (ROWB / 16), c = idx % (ROWB / 16);
      const int64_t src = (rowbase + t0 + r) * ROWB + c * 16;
      *reinterpret_cast<uint4*>(ktile + r * ROWP + c * 16) =
          *reinterpret_cast<const uint4*>(a.k_packed + src);
      *reinterpret_cast<uint4*>(vtile + r * ROWP + c * 16) =
          *reinterpret_cast<const uint4*>(a.v_packed + src);
    }
    for (int idx = threadIdx.x; idx < nt * NG; idx += blockDim.x) {
      kscale[idx] = a.k_scales[(rowbase + t0) * NG + idx];
      vscale[idx] = a.v_scales[(rowbase + t0) * NG + idx];
    }
    __syncthreads();

    // scores: thread -> (token tt, heads hh, hh+2, ...)
    {
      const int tt = threadIdx.x % kTile, hh = threadIdx.x / kTile;
      for (int h = hh; h < G; h += 2) {
        float s = -INFINITY;
        if (tt < nt) {
          const uint8_t* row = ktile + tt * ROWP;
          s = 0.0f;
          for (int g = 0; g < NG; ++g) {
            float dot = 0.0f;
#pragma unroll 8
            for (int j = 0; j < 32; ++j)
              dot = fmaf(qs[h * D + 32 * g + j], (float)nibble_at(row, NG, g, j), dot);
            s = fmaf(kscale[tt * NG + g], dot, s);
          }
        }
        sp[h * kTile + tt] = s;
      }
    }
    __syncthreads();
    // online softmax update: warp w handles heads w, w+4, ...
    {
      const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
      for (int h = warp; h < G; h += 4) {
        const float s0 = sp[h * kTile + lane], s1 = sp[h * kTile + lane + 32];
        float mx = fmaxf(s0, s1);
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_old = mstate[h];
        const float m_new = fmaxf(m_old, mx);
        const float p0 = exp2f(s0 - m_new), p1 = exp2f(s1 - m_new);
        sp[h * kTile + lane] = p0;
        sp[h * kTile + lane + 32] = p1;
        float sum = p0 + p1;
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
          const float al = exp2f(m_old - m_new);
          alpha[h] = al;
          lstate[h] = lstate[h] * al + sum;
          mstate[h] = m_new;
        }
      }
    }
    __syncthreads();
    // P.V on the packed values
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int item = threadIdx.x + it * 128;
      if (item < items) {
        const int h = item / SLICES, sl = item % SLICES;
        const int g = sl / 4, j0 = (sl % 4) * 8;
        const float al = alpha[h];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[it][e] *= al;
        for (int tt = 0; tt < nt; ++tt) {
          const float pw = sp[h * kTile + tt] * vscale[tt * NG + g];
          const uint8_t* row = vtile + tt * ROWP;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            acc[it][e] = fmaf(pw, (float)nibble_at(row, NG, g, j0 + e), acc[it][e]);
        }
      }
    }
  }

  // partials: ws[b][hq][chunk][0..D) = acc, [D] = m, [D+1] = l
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + a.plan.header_bytes);
  const int stride = a.plan.part_stride;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int item = threadIdx.x + it * 128;
    if (item < items) {
      const int h = item / SLICES, sl = item % SLICES;
      const int64_t hq = (int64_t)kvh * G + h;
      float* dst = part + (((int64_t)b * a.Hq + hq) * a.plan.n_chunks + chunk) * stride;
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[sl * 8 + e] = acc[it][e];
    }
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int64_t hq = (int64_t)kvh * G + threadIdx.x;
    float* dst = part + (((int64_t)b * a.Hq + hq) * a.plan.n_chunks + chunk) * stride;
    dst[D] = mstate[threadIdx.x];
    dst[D + 1] = lstate[threadIdx.x];
  }
}

template <int D>
size_t simt_smem_bytes(int G) {
  constexpr int NG = D / 32, ROWP = D / 2 + 16;
  return sizeof(float) * ((size_t)G * D + (size_t)G * kTile + 2 * kTile * NG + 48) +
         2 * (size_t)kTile * ROWP;
}


template <int D>
cudaError_t launch_simt_d(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  dim3 grid(a.plan.n_chunks, a.Hkv, a.B);
  static std::atomic<uint64_t> smem_set{0};
  // the limit covers every group size the host accepts (up to 16 query heads)
  const cudaError_t e =
      ensure_smem_limit(decode_simt_kernel<D>, (int)simt_smem_bytes<D>(16), smem_set);
  if (e != cudaSuccess) return e;
  decode_simt_kernel<D><<<grid, 128, simt_smem_bytes<D>(G), stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

// head_dim 128 or 256; with the SRFT variant (rotated queries given) any
// multiple of 32 up to 256
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 32: return launch_simt_d<32>(a, stream);
    case 64: return launch_simt_d<64>(a, stream);
    case 96: return launch_simt_d<96>(a, stream);
    case 128: return launch_simt_d<128>(a, stream);
    case 160: return launch_simt_d<160>(a, stream);
    case 192: return launch_simt_d<192>(a, stream);
    case 224: return launch_simt_d<224>(a, stream);
    case 256: return launch_simt_d<256>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
