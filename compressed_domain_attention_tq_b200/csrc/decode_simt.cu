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
// shared memory.  Template FMT selects the cache format: 0 = int4 codes in the
// interleaved layout; 2, 3, 4 = the codebook variant's indices of that many
// bits (codebook.cu), whose scores use lookup tables (AdapTQ post, section
// "precomputed lookup tables"): with 2 bits one table of 16 partial dot
// products per pair of coordinates and head, read with the pair's 4 index bits;
// with 3 and 4 bits the codebook level times the query coordinate.  Each chunk leaves (running max m in log2 units, sum l,
// unnormalized acc[d]) per query head in the workspace; merge.cu combines the
// chunks and rotates the result back.
#include <cuda_bf16.h>
#include <math.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTile = 64;      // tokens per shared-memory tile
constexpr int kThreads = 128;

// Token parts of the P.V work: the (head, 8-dim slice) items are split over
// TP interleaved token subsets, TP chosen (up to 32, at most 4 items per
// thread) to fill the block's threads best, so small G (MHA) still occupies
// every thread; the parts are summed once per chunk.  Shared by the host
// (shared-memory size) and the kernel.
__host__ __device__ constexpr int simt_token_parts(int G, int slices) {
  int best = 1, best_num = 0, best_den = 1;
  for (int tp = 1; tp <= 32 && G * slices * tp <= 4 * kThreads; tp *= 2) {
    const int items = G * slices * tp;
    const int den = ((items + kThreads - 1) / kThreads) * kThreads;  // thread slots used
    if (items * best_den > best_num * den) {  // strictly better fill
      best = tp;
      best_num = items;
      best_den = den;
    }
  }
  return best;
}

// Token parts of the shared-code P.V items of codebook caches: one item per
// (8-dim slice, part) fills the block's 128 threads.
template <int D>
__host__ __device__ constexpr int simt_shared_token_parts() { return kThreads / (D / 8); }

// Packed row size in 32-bit words, and the staged row pitch: odd, so lanes
// reading the same offset of consecutive rows hit distinct banks.
template <int D, int FMT>
__host__ __device__ constexpr int simt_row_words() { return FMT == 0 ? D / 8 : D * FMT / 32; }
template <int D, int FMT>
__host__ __device__ constexpr int simt_pitch_words() { return simt_row_words<D, FMT>() + 1; }

// Code m of a 16-bit half-word (in-group coordinates 4r .. 4r+3 of one group)
// as the exact float 16^m c.  t = hw ^ 0x8888 holds the biased nibbles c + 8;
// masking nibble m in place and setting the exponent bits of 2^23 gives the
// float 2^23 + 16^m (c + 8), from which one subtraction leaves 16^m c.  The
// factor 16^m is folded into the query (scores) or removed from the sums at
// the end (P.V), both exactly.
__device__ __forceinline__ float code16m(uint32_t t, int m) {
  return __int_as_float((int)((t & (0xFu << (4 * m))) | 0x4B000000u)) -
         (8388608.0f + 8.0f * (float)(1 << (4 * m)));
}

// Index j (0..31) of a codebook group held in words gw[0 .. FMT-1]: bits
// FMT*j .. FMT*j + FMT - 1 of the group's little-endian bit string.
template <int FMT>
__device__ __forceinline__ uint32_t cb_index(const uint32_t* gw, int j) {
  const int bit = FMT * j;
  if constexpr (FMT == 3) {  // may straddle two words
    return __funnelshift_r(gw[bit >> 5], gw[(bit >> 5) + 1], bit & 31) & 7u;
  } else {
    return (gw[bit >> 5] >> (bit & 31)) & ((1u << FMT) - 1u);
  }
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

__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ int clamp_ctx(int T, int max_ctx) {
  return T < 1 ? 1 : (T > max_ctx ? max_ctx : T);
}

template <int D, int FMT>
__global__ void __launch_bounds__(kThreads, FMT == 0 ? 5 : 3) decode_simt_kernel(DecodeArgs a) {
  constexpr int NG = D / 32;
  constexpr int RW = simt_row_words<D, FMT>();  // packed row (words)
  constexpr int PW = simt_pitch_words<D, FMT>();  // staged row pitch (words)
  constexpr int L = FMT == 0 ? 0 : 1 << FMT;   // codebook levels
  constexpr uint32_t LMASK = FMT == 0 ? 1u : (uint32_t)(L - 1);
  constexpr int SLICES = D / 8;                 // 8-coordinate slices per head
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int TP = simt_token_parts(G, SLICES);
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
  float* scl = sp + G * kTile;                                 // [2 buffers][K, V][kTile][NG]
  float* mstate = scl + 4 * kTile * NG;                        // [G] running max (log2)
  float* lstate = mstate + 16;                                 // [G] running sum
  float* alpha = lstate + 16;                                  // [G] rescale of this tile
  float* cbk = alpha + 16;                                     // [16] codebook levels
  float* qT = cbk + 16;                                        // [D][8] query, heads fastest (FMT != 0)
  float* spT = qT + (FMT != 0 ? D * 8 : 0);                    // [kTile][8] weights, heads fastest
  float* lut = spT + (FMT != 0 ? kTile * 8 : 0);               // [G][D/2][16] (FMT 2)
  // [2 buffers][K, V][kTile][PW] staged packed rows; after the last tile the same
  // space holds the token parts' sums [TP][G][D] (TP > 1)
  uint32_t* tiles = reinterpret_cast<uint32_t*>(lut + (FMT == 2 ? G * D * 8 : 0));
  float* red = reinterpret_cast<float*>(tiles);
  if (FMT != 0 && threadIdx.x < L) cbk[threadIdx.x] = a.levels[threadIdx.x];

  // q' = attn_scale * log2(e) * R q (the SRFT variant's R q comes rotated in q_rot)
  const int64_t qbase = ((int64_t)b * a.Hq + (int64_t)kvh * G) * D;
  const bool wht = a.signs != nullptr && a.q_rot == nullptr;
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
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
  // int4: 16^-(i mod 4), as the codes of the score loop come scaled by 16^(i mod 4)
  for (int i = threadIdx.x; i < G * D; i += kThreads)
    qs[i] *= FMT == 0 ? qmul * __int_as_float((127 - 4 * (i & 3)) << 23) : qmul;
  if constexpr (FMT != 0) {  // transposed copies for the shared-code path (absent heads: 0)
    __syncthreads();
    for (int i = threadIdx.x; i < D * 8; i += kThreads) {
      const int j = i >> 3, h = i & 7;
      qT[i] = h < G ? qs[h * D + j] : 0.0f;
    }
    for (int i = threadIdx.x; i < kTile * 8; i += kThreads) spT[i] = 0.0f;
  }
  if constexpr (FMT == 2) {  // pair tables: lut[h][p][e] = C[e & 3] q'[2p] + C[e >> 2] q'[2p + 1]
    __syncthreads();
    for (int i = threadIdx.x; i < G * D * 8; i += kThreads) {
      const int e = i & 15, hp = i >> 4;  // hp = h * (D/2) + p
      const int h = hp / (D / 2), pp = hp % (D / 2);
      lut[i] = fmaf(cbk[e & 3], qs[h * D + 2 * pp], cbk[e >> 2] * qs[h * D + 2 * pp + 1]);
    }
  }
  if (threadIdx.x < 16) {
    mstate[threadIdx.x] = -INFINITY;
    lstate[threadIdx.x] = 0.0f;
  }

  // P.V work items (head h, token part tp, slice sl), sl fastest; at most 4 per thread
  const int items = G * SLICES * TP;
  float acc[4][8];
#pragma unroll
  for (int it = 0; it < 4; ++it)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[it][e] = 0.0f;
  // score parts: two threads per token when there is a single head
  const int SP = G == 1 ? 2 : 1;
  // Codebook caches with 2..8 heads per kv head: every code is decoded once per
  // token and used by all heads (scores: thread = token half; P.V: item =
  // (8-dim slice, token part) over all heads, TPS = 128 / slices token parts).
  const bool shared = FMT != 0 && G >= 2 && G <= 8;
  constexpr int TPS = simt_shared_token_parts<D>();
  float acc2[FMT != 0 ? 8 : 1][8];
#pragma unroll
  for (int h = 0; h < (FMT != 0 ? 8 : 1); ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc2[h][e] = 0.0f;

  const int64_t rowbase = ((int64_t)b * a.Hkv + kvh) * a.capacity;
  // Tiles are staged by 4-byte cp.async into two buffers: tile i + 1 is in
  // flight while tile i is computed.
  auto stage = [&](int t0, int buf) {
    const int nt = min(kTile, t_end - t0);
    uint32_t* kt = tiles + buf * 2 * kTile * PW;
    uint32_t* vt = kt + kTile * PW;
    const uint32_t* kg = reinterpret_cast<const uint32_t*>(a.k_packed) + (rowbase + t0) * RW;
    const uint32_t* vg = reinterpret_cast<const uint32_t*>(a.v_packed) + (rowbase + t0) * RW;
    for (int idx = threadIdx.x; idx < nt * RW; idx += kThreads) {
      const int r = idx / RW, w = idx % RW;
      cp_async4(kt + r * PW + w, kg + idx);
      cp_async4(vt + r * PW + w, vg + idx);
    }
    float* ks = scl + buf * 2 * kTile * NG;
    for (int idx = threadIdx.x; idx < nt * NG; idx += kThreads) {
      cp_async4(ks + idx, a.k_scales + (rowbase + t0) * NG + idx);
      cp_async4(ks + kTile * NG + idx, a.v_scales + (rowbase + t0) * NG + idx);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  stage(t_begin, 0);
  int buf = 0;
  for (int t0 = t_begin; t0 < t_end; t0 += kTile, buf ^= 1) {
    const int nt = min(kTile, t_end - t0);
    if (t0 + kTile < t_end) {  // the other buffer was released by the barrier ending the last tile
      stage(t0 + kTile, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint32_t* ktile = tiles + buf * 2 * kTile * PW;
    const uint32_t* vtile = ktile + kTile * PW;
    const float* kscale = scl + buf * 2 * kTile * NG;
    const float* vscale = kscale + kTile * NG;

    // scores S[h][t] = sum_g s_k[t][g] sum_{j in g} c[t][j] q'[h][32 g + j]
    if (FMT != 0 && shared) {  // thread = (token, half of each group); all heads
      const int tt = threadIdx.x >> 1, half = threadIdx.x & 1;
      float s[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) s[h] = 0.0f;
      if (tt < nt) {
        const uint32_t* row = ktile + tt * PW;
        for (int g = 0; g < NG; ++g) {
          const uint32_t* gw = row + (FMT != 0 ? FMT : 1) * g;
          float dg[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) dg[h] = 0.0f;
          // this half's 16 indices (FMT * 16 bits from bit FMT * 16 * half) in one register pair
          constexpr int FB = FMT != 0 ? FMT : 2;
          const int b0 = FB * 16 * half;
          const uint64_t bits = ((uint64_t)gw[(b0 >> 5) + 1] << 32 | gw[b0 >> 5]) >> (b0 & 31);
#pragma unroll
          for (int jl = 0; jl < 16; ++jl) {
            const int j = 16 * half + jl;
            const float c = cbk[(uint32_t)(bits >> (FB * jl)) & ((1u << FB) - 1u)];
            const float4 qa = *reinterpret_cast<const float4*>(qT + (32 * g + j) * 8);
            const float4 qb = *reinterpret_cast<const float4*>(qT + (32 * g + j) * 8 + 4);
            dg[0] = fmaf(qa.x, c, dg[0]);
            dg[1] = fmaf(qa.y, c, dg[1]);
            dg[2] = fmaf(qa.z, c, dg[2]);
            dg[3] = fmaf(qa.w, c, dg[3]);
            dg[4] = fmaf(qb.x, c, dg[4]);
            dg[5] = fmaf(qb.y, c, dg[5]);
            dg[6] = fmaf(qb.z, c, dg[6]);
            dg[7] = fmaf(qb.w, c, dg[7]);
          }
          const float sk = kscale[tt * NG + g];
#pragma unroll
          for (int h = 0; h < 8; ++h) s[h] = fmaf(sk, dg[h], s[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G) {
          const float v = s[h] + __shfl_xor_sync(0xffffffffu, s[h], 1);
          if (half == 0) sp[h * kTile + tt] = tt < nt ? v : -INFINITY;
        }
    }
    for (int idx = threadIdx.x; idx < (shared ? 0 : kTile * G * SP); idx += kThreads) {
      const int part = SP == 2 ? (idx & 1) : 0;
      const int tt = SP == 2 ? (idx >> 1) : idx % kTile;
      const int h = SP == 2 ? 0 : idx / kTile;
      float s = 0.0f;
      if (tt < nt && FMT == 2) {  // pair tables: 16 pairs per group, two words
        const uint32_t* row = ktile + tt * PW;
        const float* lh = lut + h * D * 8;
        for (int g = 0; g < NG; ++g) {
          float d0 = 0.0f, d1 = 0.0f;
          for (int w = (SP == 2 ? part : 0); w < (SP == 2 ? part + 1 : 2); ++w) {
            const uint32_t word = row[2 * g + w];
            const float* lp = lh + (16 * g + 8 * w) * 16;
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              d0 += lp[16 * k + ((word >> (4 * k)) & 15u)];
              d1 += lp[16 * (k + 1) + ((word >> (4 * k + 4)) & 15u)];
            }
          }
          s = fmaf(kscale[tt * NG + g], d0 + d1, s);
        }
      } else if (tt < nt && FMT != 0) {  // codebook level x query coordinate
        const uint32_t* row = ktile + tt * PW;
        const int j_lo = SP == 2 ? 16 * part : 0, j_hi = SP == 2 ? j_lo + 16 : 32;
        for (int g = 0; g < NG; ++g) {
          const uint32_t* gw = row + FMT * g;
          float d0 = 0.0f, d1 = 0.0f;
          for (int j = j_lo; j < j_hi; j += 2) {
            d0 = fmaf(qs[h * D + 32 * g + j], cbk[cb_index<FMT>(gw, j)], d0);
            d1 = fmaf(qs[h * D + 32 * g + j + 1], cbk[cb_index<FMT>(gw, j + 1)], d1);
          }
          s = fmaf(kscale[tt * NG + g], d0 + d1, s);
        }
      } else if (tt < nt) {
        const uint16_t* row = reinterpret_cast<const uint16_t*>(ktile + tt * PW);
        const int r_lo = SP == 2 ? 4 * part : 0, r_hi = SP == 2 ? r_lo + 4 : 8;
        for (int g = 0; g < NG; ++g) {
          float d0 = 0.0f, d1 = 0.0f, d2 = 0.0f, d3 = 0.0f;  // four independent chains
          for (int r = r_lo; r < r_hi; ++r) {
            const uint32_t t = row[r * NG + g] ^ 0x8888u;   // half-word at byte r * 2NG + 2g
            const float4 qv = *reinterpret_cast<const float4*>(qs + h * D + 32 * g + 4 * r);
            d0 = fmaf(qv.x, code16m(t, 0), d0);
            d1 = fmaf(qv.y, code16m(t, 1), d1);
            d2 = fmaf(qv.z, code16m(t, 2), d2);
            d3 = fmaf(qv.w, code16m(t, 3), d3);
          }
          s = fmaf(kscale[tt * NG + g], (d0 + d1) + (d2 + d3), s);
        }
      }
      if (SP == 2) s += __shfl_xor_sync(0xffffffffu, s, 1);  // idx, idx ^ 1: the same token
      if (part == 0) sp[h * kTile + tt] = tt < nt ? s : -INFINITY;
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
        if (FMT != 0 && shared) {
          spT[lane * 8 + h] = p0;
          spT[(lane + 32) * 8 + h] = p1;
        }
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
    if (FMT != 0 && shared && threadIdx.x < SLICES * TPS) {  // item (sl, tp) for all heads
      const int sl = threadIdx.x % SLICES, tp = threadIdx.x / SLICES;
      const int g = sl / 4, bit = (FMT != 0 ? FMT : 1) * 8 * (sl % 4);
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G) {
          const float al = alpha[h];
          if (al != 1.0f) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc2[h][e] *= al;
          }
        }
      for (int tt = tp; tt < nt; tt += TPS) {
        const uint32_t* gw = vtile + tt * PW + (FMT != 0 ? FMT : 1) * g;
        const uint32_t v8 = __funnelshift_r(gw[bit >> 5], gw[(bit >> 5) + 1], bit & 31);
        float c[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) c[m] = cbk[(v8 >> ((FMT != 0 ? FMT : 1) * m)) & LMASK];
        const float sv = vscale[tt * NG + g];
        const float4 pa = *reinterpret_cast<const float4*>(spT + tt * 8);
        const float4 pb = *reinterpret_cast<const float4*>(spT + tt * 8 + 4);
        const float pw[8] = {pa.x * sv, pa.y * sv, pa.z * sv, pa.w * sv,
                             pb.x * sv, pb.y * sv, pb.z * sv, pb.w * sv};
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (h < G) {
#pragma unroll
            for (int m = 0; m < 8; ++m) acc2[h][m] = fmaf(pw[h], c[m], acc2[h][m]);
          }
      }
    }
    // P.V on the packed values: item (h, tp, sl) adds tokens tp, tp + TP, ... of the tile
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int item = threadIdx.x + it * kThreads;
      if (!shared && item < items) {
        const int sl = item % SLICES, rest = item / SLICES;
        const int tp = rest % TP, h = rest / TP;
        const int g = sl / 4, r0 = (sl % 4) * 2;
        const float al = alpha[h];
        if (al != 1.0f) {  // the running max moved
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[it][e] *= al;
        }
        for (int tt = tp; tt < nt; tt += TP) {
          const float pw = sp[h * kTile + tt] * vscale[tt * NG + g];
          if constexpr (FMT == 0) {
            const uint16_t* row = reinterpret_cast<const uint16_t*>(vtile + tt * PW);
            const uint32_t t0 = row[r0 * NG + g] ^ 0x8888u, t1 = row[(r0 + 1) * NG + g] ^ 0x8888u;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              acc[it][m] = fmaf(pw, code16m(t0, m), acc[it][m]);
              acc[it][4 + m] = fmaf(pw, code16m(t1, m), acc[it][4 + m]);
            }
          } else {  // the slice's 8 indices: FMT * 8 bits at bit FMT * 8 * (sl % 4) of the group
            const uint32_t* gw = vtile + tt * PW + FMT * g;
            const int bit = FMT * 8 * (sl % 4);
            const uint32_t v8 = __funnelshift_r(gw[bit >> 5], gw[(bit >> 5) + 1], bit & 31);
#pragma unroll
            for (int m = 0; m < 8; ++m)
              acc[it][m] = fmaf(pw, cbk[(v8 >> (FMT * m)) & LMASK], acc[it][m]);
          }
        }
      }
    }
    __syncthreads();  // the tile's buffers and scores are free for the next stage
  }

  if constexpr (FMT == 0) {  // slot e of a P.V item holds 16^(e mod 4) times its sum
#pragma unroll
    for (int it = 0; it < 4; ++it)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[it][e] *= __int_as_float((127 - 4 * (e & 3)) << 23);
  }

  // partials: ws[b][hq][chunk][0..D) = acc, [D] = m, [D+1] = l
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + a.plan.header_bytes);
  const int stride = a.plan.part_stride;
  if (shared) {  // sum the TPS token parts in shared memory (fixed order: deterministic)
    if (threadIdx.x < SLICES * TPS) {
      const int sl = threadIdx.x % SLICES, tp = threadIdx.x / SLICES;
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < G)
#pragma unroll
          for (int e = 0; e < 8; ++e) red[(tp * G + h) * D + sl * 8 + e] = acc2[h][e];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
      float v = 0.0f;
      for (int tp = 0; tp < TPS; ++tp) v += red[tp * G * D + i];
      const int h = i / D, c = i % D;
      const int64_t hq = (int64_t)kvh * G + h;
      part[(((int64_t)b * a.Hq + hq) * a.plan.n_chunks + chunk) * stride + c] = v;
    }
  } else if (TP == 1) {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int item = threadIdx.x + it * kThreads;
      if (item < items) {
        const int sl = item % SLICES, h = item / SLICES;
        const int64_t hq = (int64_t)kvh * G + h;
        float* dst = part + (((int64_t)b * a.Hq + hq) * a.plan.n_chunks + chunk) * stride;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[sl * 8 + e] = acc[it][e];
      }
    }
  } else {  // sum the token parts in shared memory (fixed order: deterministic)
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int item = threadIdx.x + it * kThreads;
      if (item < items) {
        const int sl = item % SLICES, rest = item / SLICES;
        const int tp = rest % TP, h = rest / TP;
#pragma unroll
        for (int e = 0; e < 8; ++e) red[(tp * G + h) * D + sl * 8 + e] = acc[it][e];
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
      float v = 0.0f;
      for (int tp = 0; tp < TP; ++tp) v += red[tp * G * D + i];
      const int h = i / D, c = i % D;
      const int64_t hq = (int64_t)kvh * G + h;
      part[(((int64_t)b * a.Hq + hq) * a.plan.n_chunks + chunk) * stride + c] = v;
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

template <int D, int FMT>
size_t simt_smem_bytes(int G) {
  constexpr int NG = D / 32;
  const int TP = simt_token_parts(G, D / 8);
  const size_t tile_words = 4 * (size_t)kTile * simt_pitch_words<D, FMT>();
  size_t red_words = TP > 1 ? (size_t)TP * G * D : 0;
  if (FMT != 0 && G >= 2 && G <= 8) red_words = (size_t)simt_shared_token_parts<D>() * G * D;
  const size_t lut_words = FMT == 2 ? (size_t)G * D * 8 : 0;
  const size_t tr_words = FMT != 0 ? (size_t)D * 8 + kTile * 8 : 0;  // qT, spT
  return sizeof(float) * ((size_t)G * D + (size_t)G * kTile + 4 * kTile * NG + 64 + lut_words +
                          tr_words) +
         sizeof(uint32_t) * (tile_words > red_words ? tile_words : red_words);
}

template <int D, int FMT>
size_t simt_smem_max() {  // over every group size the host accepts (up to 16 query heads)
  size_t m = 0;
  for (int G = 1; G <= 16; ++G) {
    const size_t b = simt_smem_bytes<D, FMT>(G);
    m = b > m ? b : m;
  }
  return m;
}

template <int D, int FMT = 0>
cudaError_t launch_simt_d(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  dim3 grid(a.plan.n_chunks, a.Hkv, a.B);
  static SmemLimitSet smem_set;
  const cudaError_t e =
      ensure_smem_limit(decode_simt_kernel<D, FMT>, (int)simt_smem_max<D, FMT>(), smem_set);
  if (e != cudaSuccess) return e;
  decode_simt_kernel<D, FMT><<<grid, kThreads, simt_smem_bytes<D, FMT>(G), stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_simt_cb(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.cb_bits) {
    case 2: return launch_simt_d<D, 2>(a, stream);
    case 3: return launch_simt_d<D, 3>(a, stream);
    case 4: return launch_simt_d<D, 4>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// int4: head_dim 128 or 256, and with the SRFT variant (rotated queries given)
// any multiple of 32 up to 256; codebook variant: head_dim 128 or 256
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream) {
  if (a.cb_bits != 0) return a.d == 128 ? launch_simt_cb<128>(a, stream) : launch_simt_cb<256>(a, stream);
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
