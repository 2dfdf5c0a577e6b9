// decode_mma.cu -- split-K decode attention on the packed int4 cache with the
// GQA contractions on tensor cores (mma.sync m16n8k16, f16 x f16 -> f32).
//
// Attention runs directly on the packed codes ("fused sdpa_int4",
// Open-TQ-Metal abstract): no dequantized K/V matrix exists anywhere (forum
// summary, section "eliminating intermediate matrices"); codes are widened to
// f16 in registers, and the fp32 group scales are applied around the
// contractions.  Softmax runs online with a running maximum, fp32 sums and
// exact exp2 (section "numerical stability": the scaling trick and
// high-precision accumulators, without an approximate softmax).
//
// Work: persistent CTAs, one per SM, walk a list of items (sequence b, kv
// head, context chunk).  A producer warp streams each item's rows (packed K,
// packed V, K scales, V scales) into a ring of shared-memory stages with 1-D
// bulk async copies completing on mbarriers; 8 consumer warps each take 16
// tokens of every stage.  Each warp keeps its own running (max, sum, acc) and
// the 8 are merged per item in shared memory into one split-K partial
// (max in log2 units, sum, unnormalized acc[d]) per query head; merge_kernel
// combines the chunks and rotates the output back.
//
// Exactness on the tensor cores.  Codes (-7..7) are exact in f16.  The fp32
// operand of each contraction is split into hi + lo f16 parts (about 22 bits):
//  - scores: rows of the A operand are [query hi; query lo], so the 16 rows of
//    m16n8k16 hold 8 heads x 2 parts and hi + lo is summed per thread after
//    the product.  Each head's rotated, scaled query is first multiplied by a
//    power of two so its largest element lies in [2^13, 2^14) (f16 range).
//    Per group of 32 dims the product is scaled by the token's fp32 K scale.
//  - P.V: the operand is P' = p * s_v[token, group] * 2^-F_g, split into
//    hi + lo.  F_g (per warp and group) keeps P' below 2^15: it is set from
//    the first tile's V scales and raised, with an exact power-of-two rescale
//    of that group's accumulators, whenever a later tile would overflow.
// Two arrangements (template PATH):
//  - PATH 0 (heads on rows, 5..8 query heads per kv head, d = 128): scores
//    C = [q hi; q lo] x K^T; P.V C = [P' hi; P' lo] x V, where the score
//    accumulator fragment is reused as the P.V A operand without shuffles.
//  - PATH 1 (dims on rows, 1..4 query heads, d = 128 or 256): scores as
//    above with each head on two neighbouring rows; P.V C = V^T x [P' hi,
//    P' lo per head] with dims on the rows, so the accumulator is d/16 x 4
//    registers.
// Token order: slot k of a 16-token tile holds tile row pi(k), chosen so that
// the K-code and scale loads of a warp hit distinct shared-memory banks.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kWarps = 8;                       // consumer warps per CTA
constexpr int kMmaThreads = (kWarps + 1) * 32;  // + one producer warp
constexpr int kStageTokens = 16 * kWarps;       // tokens per pipeline stage
constexpr float kLog2e = 1.4426950408889634f;
constexpr long long kWaitCycles = 4000000000LL; // ~2 s at 2 GHz: a wait never lasts this long
constexpr uint32_t kFull = 0xffffffffu;

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`, giving up after kWaitCycles or as soon as
// another thread of the CTA has set *abort.  Returns false when it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort || clock64() - t0 > kWaitCycles) {
      *abort = 1;
      return false;
    }
  }
  return true;
}

// 1-D bulk async copy global -> shared (16-byte aligned, size % 16 == 0),
// completing `bytes` of transaction count on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_barrier_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWarps * 32) : "memory");
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// (a & b) ^ c in one LOP3
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Two int4 codes -> f16x2.  x holds 4-bit two's-complement codes; the result's
// low half is the code in bits 0..3 (resp. 4..7) and the high half the code in
// bits 16..19 (resp. 20..23).  Flipping bit 3 turns a code c into c + 8 in
// 0..15; OR-ing it under the exponent of 1024.0 (0x6400) gives the f16 value
// 1024 + c + 8 exactly (bits 4..7: 1024 + 16 (c + 8)), from which one exact
// f16 subtraction (resp. fma with 1/16) leaves c.
__device__ __forceinline__ uint32_t codes_lo(uint32_t x) {
  return hsub2(and_xor(x, 0x000F000Fu, 0x64086408u), 0x64086408u);  // - 1032
}
__device__ __forceinline__ uint32_t codes_hi(uint32_t x) {
  return hfma2(and_xor(x, 0x00F000F0u, 0x64806480u), 0x2C002C00u, 0xD480D480u);  // /16 - 72
}

// fp32 pair -> f16x2 (low half = lo_elem)
__device__ __forceinline__ uint32_t f16x2(float lo_elem, float hi_elem) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi_elem), "f"(lo_elem));
  return d;
}

// Exact split x = hi + lo with hi holding x's top 11 significant bits.
__device__ __forceinline__ float split_hi(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
}

// Row of the 16-token tile held by MMA slot k (0..15).
__device__ __forceinline__ int slot_row(int k) {
  const int t = (k & 7) >> 1;
  const int a = (t & 1) | ((t & 2) << 1);  // 0, 1, 4, 5
  return (k & 8) | (a ^ (3 * (k & 1)));
}

// ------------------------------------------------------------ configuration

template <int D, int PATH>
struct Cfg {
  static constexpr int NG = D / 32;        // quantization groups per vector
  static constexpr int RB = D / 2;         // packed bytes per row
  static constexpr int SB = 2 * NG;        // bytes of one of a row's 8 sub-blocks
  static constexpr int NH = PATH == 0 ? 8 : 4;  // query heads per kv head (max)
  static constexpr int NACC = PATH == 0 ? 4 * NG : 2 * NG;  // accumulator fragments
  static constexpr int NS = D == 128 ? 4 : 3;                // pipeline stages
  static constexpr int KC = 0;                               // stage: packed K rows
  static constexpr int VC = kStageTokens * RB;               //        packed V rows
  static constexpr int KS = 2 * kStageTokens * RB;           //        K scales
  static constexpr int VS = KS + kStageTokens * NG * 4;      //        V scales
  static constexpr int STAGE = VS + kStageTokens * NG * 4;
  static constexpr int BAR = NS * STAGE;                     // full[NS], empty[NS]
  static constexpr int QS = BAR + 16 * NS;                   // float [NH][D] query
  static constexpr int QEXP = QS + 4 * NH * D;               // float [NH]
  static constexpr int MACC = QEXP + 4 * 8;                  // float [kWarps][NH][D]
  static constexpr int MM = MACC + 4 * kWarps * NH * D;      // float [kWarps][NH] max
  static constexpr int ML = MM + 4 * kWarps * NH;            // float [kWarps][NH] sum
  static constexpr int MW = ML + 4 * kWarps * NH;            // float [kWarps][NH] weight
  static constexpr int MTOT = MW + 4 * kWarps * NH;          // float [NH] max, [NH] sum
  static constexpr int ABORT = MTOT + 4 * 2 * NH;            // int
  static constexpr int BYTES = ABORT + 16;
};

__device__ __forceinline__ int clamp_ctx_mma(int T, int max_ctx) {
  return T < 1 ? 1 : (T > max_ctx ? max_ctx : T);
}

// Item it -> (sequence b, kv head, chunk c) and its token range [t0, t1).
// Returns false for an item past the end of its sequence.
__device__ __forceinline__ bool item_range(const DecodeArgs& a, int it, int& b, int& kvh, int& c,
                                           int& t0, int& t1) {
  const int nc = a.plan.n_chunks;
  c = it % nc;
  const int bh = it / nc;
  kvh = bh % a.Hkv;
  b = bh / a.Hkv;
  const int T = clamp_ctx_mma(a.ctx_lens[b], a.max_ctx);
  t0 = c * a.plan.chunk;
  t1 = min(T, t0 + a.plan.chunk);
  return t0 < t1;
}

// Per-thread state of one consumer warp for one item.
template <int D, int PATH>
struct WarpState {
  float acc[Cfg<D, PATH>::NACC][4];     // P.V accumulators (fragments)
  uint32_t qa[D / 32][2][4];            // score A fragments: [group][k-step][reg]
  float vsc[D / 32];                    // 2^-F_g: V-scale normalisation per group
  float m;                              // running max of this thread's head (log2 units)
  float l;                              // this thread's share of the running sum
  float qexp;                           // 2^E of this thread's head (query normalisation)
  bool vset;                            // vsc initialised for this item
};

// Rotated, scaled query of the item's G heads -> smem (normalised by a power
// of two per head), then every consumer thread builds its score A fragments.
// Warp w < NH prepares head w; the FWHT runs in registers and shuffles.
template <int D, int PATH>
__device__ __forceinline__ void prep_query(const DecodeArgs& a, int b, int kvh, unsigned char* smem,
                                           WarpState<D, PATH>& st) {
  using C = Cfg<D, PATH>;
  constexpr int E = D / 32;  // elements per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  float* qs = reinterpret_cast<float*>(smem + C::QS);
  float* qexp = reinterpret_cast<float*>(smem + C::QEXP);
  if (warp < C::NH) {
    const int h = warp;
    float x[E];
    if (h < G) {
      const int64_t base = ((int64_t)b * a.Hq + (int64_t)kvh * G + h) * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float v = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[base + e])
                           : static_cast<const float*>(a.q)[base + e];
        if (a.signs) v *= (float)a.signs[lane * E + e];
        x[e] = v;
      }
      if (a.signs) {
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
        for (int bit = 1; bit < 32; bit <<= 1)
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float v = __shfl_xor_sync(kFull, x[e], bit);
            x[e] = (lane & bit) ? v - x[e] : x[e] + v;
          }
      }
      const float mul = a.attn_scale * kLog2e * (a.signs ? rsqrtf((float)D) : 1.0f);
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x[e] *= mul;
        amax = fmaxf(amax, fabsf(x[e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
      int ex = 0;
      frexpf(amax, &ex);                       // amax = m * 2^ex, m in [0.5, 1)
      int sh = amax > 0.0f ? 14 - ex : 0;      // amax * 2^sh in [2^13, 2^14)
      sh = max(-120, min(120, sh));
      const float scale = ldexpf(1.0f, sh);
#pragma unroll
      for (int e = 0; e < E; ++e) qs[h * D + lane * E + e] = x[e] * scale;
      if (lane == 0) qexp[h] = ldexpf(1.0f, -sh);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qs[h * D + lane * E + e] = 0.0f;
      if (lane == 0) qexp[h] = 1.0f;
    }
  }
  named_barrier_consumers();
  const int gid = lane >> 2, tig = lane & 3;
  const int hrow = PATH == 0 ? gid : gid >> 1;
  const float* qr = qs + hrow * D;
#pragma unroll
  for (int g = 0; g < D / 32; ++g)
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int e0 = 32 * g + 8 * tig + 2 * ks;
      const float v0 = qr[e0], v1 = qr[e0 + 4], v2 = qr[e0 + 1], v3 = qr[e0 + 5];
      const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
      const __half h2 = __float2half_rn(v2), h3 = __float2half_rn(v3);
      st.qa[g][ks][0] = f16x2(__half2float(h0), __half2float(h1));
      st.qa[g][ks][1] = f16x2(v0 - __half2float(h0), v1 - __half2float(h1));
      st.qa[g][ks][2] = f16x2(__half2float(h2), __half2float(h3));
      st.qa[g][ks][3] = f16x2(v2 - __half2float(h2), v3 - __half2float(h3));
    }
  st.qexp = qexp[hrow];
}

// Multiply the accumulator fragments of group g by f.
template <int D, int PATH>
__device__ __forceinline__ void scale_group(WarpState<D, PATH>& st, int g, float f) {
  constexpr int PER = PATH == 0 ? 4 : 2;
#pragma unroll
  for (int j = 0; j < Cfg<D, PATH>::NACC; ++j)
    if (j / PER == g) {
#pragma unroll
      for (int r = 0; r < 4; ++r) st.acc[j][r] *= f;
    }
}

// One 16-token tile of one warp: rows r0 .. r0+15 of the stage, the first
// `valid` of them real tokens.  rho[i]: tile rows of this thread's MMA slots
// 2tig, 2tig+1, 8+2tig, 9+2tig; krow[nt]: tile row of score n-tile nt's
// column gid.
template <int D, int PATH>
__device__ __forceinline__ void process_tile(const unsigned char* stg, int r0, int valid, int gid,
                                             int tig, const int (&rho)[4], const int (&krow)[2],
                                             WarpState<D, PATH>& st) {
  using C = Cfg<D, PATH>;
  constexpr int NG = C::NG, RB = C::RB, SB = C::SB;
  const unsigned char* kc = stg + C::KC + r0 * RB;
  const unsigned char* vc = stg + C::VC + r0 * RB;
  const float* ks = reinterpret_cast<const float*>(stg + C::KS) + r0 * NG;
  const float* vs = reinterpret_cast<const float*>(stg + C::VS) + r0 * NG;

  // ---- scores S = qexp * sum_g s_k[t, g] * (q_hi + q_lo) . c_k[t, group g]
  float S[4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    uint32_t kw[NG];  // sub-blocks 2tig and 2tig+1 of the n-tile's token gid
    const uint4* kp = reinterpret_cast<const uint4*>(kc + krow[nt] * RB + 2 * SB * tig);
#pragma unroll
    for (int q = 0; q < NG / 4; ++q) {
      const uint4 v = kp[q];
      kw[4 * q] = v.x;
      kw[4 * q + 1] = v.y;
      kw[4 * q + 2] = v.z;
      kw[4 * q + 3] = v.w;
    }
    float sk0[NG], sk1[NG];
#pragma unroll
    for (int q = 0; q < NG / 4; ++q) {
      const float4 a0 = reinterpret_cast<const float4*>(ks + rho[2 * nt] * NG)[q];
      const float4 a1 = reinterpret_cast<const float4*>(ks + rho[2 * nt + 1] * NG)[q];
      sk0[4 * q] = a0.x; sk0[4 * q + 1] = a0.y; sk0[4 * q + 2] = a0.z; sk0[4 * q + 3] = a0.w;
      sk1[4 * q] = a1.x; sk1[4 * q + 1] = a1.y; sk1[4 * q + 2] = a1.z; sk1[4 * q + 3] = a1.w;
    }
    float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      // in-group coordinates 8tig .. 8tig+7 of group g, nibble j <-> 8tig + j
      const uint32_t X = prmt(kw[g / 2], kw[NG / 2 + g / 2], (g & 1) ? 0x7632u : 0x5410u);
      const uint32_t Y = X >> 8;
      float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      mma16816(c, st.qa[g][0][0], st.qa[g][0][1], st.qa[g][0][2], st.qa[g][0][3], codes_lo(X),
               codes_hi(X));
      mma16816(c, st.qa[g][1][0], st.qa[g][1][1], st.qa[g][1][2], st.qa[g][1][3], codes_lo(Y),
               codes_hi(Y));
      s0 = fmaf(sk0[g], c[0] + c[2], s0);
      s1 = fmaf(sk1[g], c[1] + c[3], s1);
    }
    S[2 * nt] = s0 * st.qexp;
    S[2 * nt + 1] = s1 * st.qexp;
  }

  // ---- online softmax (log2 units) for this thread's head
  bool vld[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    vld[i] = rho[i] < valid;
    if (!vld[i]) S[i] = -INFINITY;
  }
  float mx = fmaxf(fmaxf(S[0], S[1]), fmaxf(S[2], S[3]));
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
  const float m_new = fmaxf(st.m, mx);
  if (__any_sync(kFull, m_new > st.m)) {
    const float alpha = exp2f(st.m - m_new);  // 0 on the first tile, 1 if unchanged
    // PATH 1 accumulates head tig; its softmax state lives on lane 8 * tig
    const float al = PATH == 0 ? alpha : __shfl_sync(kFull, alpha, 8 * tig);
#pragma unroll
    for (int j = 0; j < C::NACC; ++j)
#pragma unroll
      for (int r = 0; r < 4; ++r) st.acc[j][r] *= al;
    st.l *= alpha;
    st.m = m_new;
  }
  float p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = exp2f(S[i] - st.m);
  st.l += (p[0] + p[1]) + (p[2] + p[3]);

  // ---- P' = p * s_v * 2^-F_g, with F_g kept so that P' < 2^15
  float sv[4][NG];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < NG / 4; ++q) {
      const float4 a = reinterpret_cast<const float4*>(vs + rho[i] * NG)[q];
      sv[i][4 * q] = vld[i] ? a.x : 0.0f;
      sv[i][4 * q + 1] = vld[i] ? a.y : 0.0f;
      sv[i][4 * q + 2] = vld[i] ? a.z : 0.0f;
      sv[i][4 * q + 3] = vld[i] ? a.w : 0.0f;
    }
  float pv[4][NG];
  float pmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      pv[i][g] = p[i] * (sv[i][g] * st.vsc[g]);
      pmax = fmaxf(pmax, pv[i][g]);
    }
  if (__any_sync(kFull, !st.vset || pmax > 16384.0f)) {
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float vm = fmaxf(fmaxf(sv[0][g], sv[1][g]), fmaxf(sv[2][g], sv[3][g]));
      vm = fmaxf(vm, __shfl_xor_sync(kFull, vm, 1));
      vm = fmaxf(vm, __shfl_xor_sync(kFull, vm, 2));
      if (!st.vset || vm * st.vsc[g] > 16384.0f) {
        int ex = 0;
        frexpf(vm, &ex);
        int sh = vm > 0.0f ? 7 - ex : 0;  // vm * 2^sh in [64, 128)
        sh = max(-120, min(120, sh));
        const float nv = ldexpf(1.0f, sh);
        if (st.vset) scale_group(st, g, nv / st.vsc[g]);  // exact: powers of two
        st.vsc[g] = nv;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) pv[i][g] = p[i] * (sv[i][g] * st.vsc[g]);
    }
    st.vset = true;
  }

  // ---- P.V on the packed values
  uint32_t vw[4][NG / 2];  // sub-block gid of rows rho[0..3]
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned char* vp = vc + rho[i] * RB + SB * gid;
    if (NG == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(vp);
      vw[i][0] = v.x;
      vw[i][1] = v.y;
    } else {
#pragma unroll
      for (int q = 0; q < NG / 8; ++q) {
        const uint4 v = reinterpret_cast<const uint4*>(vp)[q];
        vw[i][4 * q] = v.x;
        vw[i][4 * q + 1] = v.y;
        vw[i][4 * q + 2] = v.z;
        vw[i][4 * q + 3] = v.w;
      }
    }
  }
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;
    // codes c = 0..3 of dims 32g + 4gid + c: low halves rows rho0 / rho2,
    // high halves rows rho1 / rho3
    const uint32_t X = prmt(vw[0][g / 2], vw[1][g / 2], sel);
    const uint32_t Y = prmt(vw[2][g / 2], vw[3][g / 2], sel);
    const float h0 = split_hi(pv[0][g]), h1 = split_hi(pv[1][g]);
    const float h2 = split_hi(pv[2][g]), h3 = split_hi(pv[3][g]);
    if (PATH == 0) {
      const uint32_t a0 = f16x2(h0, h1), a1 = f16x2(pv[0][g] - h0, pv[1][g] - h1);
      const uint32_t a2 = f16x2(h2, h3), a3 = f16x2(pv[2][g] - h2, pv[3][g] - h3);
      mma16816(st.acc[4 * g + 0], a0, a1, a2, a3, codes_lo(X), codes_lo(Y));
      mma16816(st.acc[4 * g + 1], a0, a1, a2, a3, codes_hi(X), codes_hi(Y));
      mma16816(st.acc[4 * g + 2], a0, a1, a2, a3, codes_lo(X >> 8), codes_lo(Y >> 8));
      mma16816(st.acc[4 * g + 3], a0, a1, a2, a3, codes_hi(X >> 8), codes_hi(Y >> 8));
    } else {
      const bool lo = gid & 1;  // column gid = (head gid / 2, part gid % 2)
      const uint32_t b0 = f16x2(lo ? pv[0][g] - h0 : h0, lo ? pv[1][g] - h1 : h1);
      const uint32_t b1 = f16x2(lo ? pv[2][g] - h2 : h2, lo ? pv[3][g] - h3 : h3);
      mma16816(st.acc[2 * g + 0], codes_lo(X), codes_hi(X), codes_lo(Y), codes_hi(Y), b0, b1);
      mma16816(st.acc[2 * g + 1], codes_lo(X >> 8), codes_hi(X >> 8), codes_lo(Y >> 8),
               codes_hi(Y >> 8), b0, b1);
    }
  }
}

// Wait for phase `parity` of `bar` for at most kWaitCycles (used only to drain
// copies still in flight after the pipeline gave up).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return;
}

// End of an item: the 8 warps' (max, sum, acc) per head are merged in shared
// memory and written as the item's split-K partial.  If the pipeline gave up,
// the partial's max is NaN, so the decode's output for these heads is NaN.
template <int D, int PATH>
__device__ __forceinline__ void finish_item(const DecodeArgs& a, unsigned char* smem,
                                            const WarpState<D, PATH>& st, int b, int kvh, int c,
                                            bool aborted) {
  using C = Cfg<D, PATH>;
  constexpr int NH = C::NH, NG = C::NG;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = a.Hq / a.Hkv;
  float* macc = reinterpret_cast<float*>(smem + C::MACC);
  float* mm = reinterpret_cast<float*>(smem + C::MM);
  float* ml = reinterpret_cast<float*>(smem + C::ML);
  float* mw = reinterpret_cast<float*>(smem + C::MW);
  float* mtot = reinterpret_cast<float*>(smem + C::MTOT);

  float l = st.l;
  l += __shfl_xor_sync(kFull, l, 1);
  l += __shfl_xor_sync(kFull, l, 2);
  const float m = aborted ? __int_as_float(0x7fc00000) : st.m;
  if (PATH == 0) {
    if (tig == 0) {
      mm[warp * NH + gid] = m;
      ml[warp * NH + gid] = l;
    }
    float* dst = macc + (warp * NH + gid) * D;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float inv = 1.0f / st.vsc[g];  // exact: a power of two
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        dst[32 * g + 8 * tig + cc] = (st.acc[4 * g + cc][0] + st.acc[4 * g + cc][2]) * inv;
        dst[32 * g + 8 * tig + 4 + cc] = (st.acc[4 * g + cc][1] + st.acc[4 * g + cc][3]) * inv;
      }
    }
  } else {
    if (tig == 0 && (gid & 1) == 0) {
      mm[warp * NH + (gid >> 1)] = m;
      ml[warp * NH + (gid >> 1)] = l;
    }
    float* dst = macc + (warp * NH + tig) * D;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const float inv = 1.0f / st.vsc[g];
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        const int dim = 32 * g + 4 * gid + 2 * pp;
        dst[dim] = (st.acc[2 * g + pp][0] + st.acc[2 * g + pp][1]) * inv;
        dst[dim + 1] = (st.acc[2 * g + pp][2] + st.acc[2 * g + pp][3]) * inv;
      }
    }
  }
  named_barrier_consumers();
  const int tid = threadIdx.x;
  if (tid < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mm[w * NH + tid]);
    float L = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float wt = exp2f(mm[w * NH + tid] - M);  // NaN if that warp gave up
      mw[w * NH + tid] = wt;
      L = fmaf(wt, ml[w * NH + tid], L);
    }
    mtot[tid] = M;
    mtot[NH + tid] = L;
  }
  named_barrier_consumers();
  const int stride = a.plan.part_stride;
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) +
                                         a.plan.header_bytes);
  for (int idx = tid; idx < G * D; idx += kWarps * 32) {
    const int h = idx / D, i = idx % D;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s = fmaf(mw[w * NH + h], macc[(w * NH + h) * D + i], s);
    float* dst = part + (((int64_t)b * a.Hq + (int64_t)kvh * G + h) * a.plan.n_chunks + c) * stride;
    dst[i] = s;
    if (i == 0) {
      dst[D] = mtot[h];
      dst[D + 1] = mtot[NH + h];
    }
  }
}

// Producer: one thread streams every stage of this CTA's items.
template <int D, int PATH>
__device__ __forceinline__ void produce(const DecodeArgs& a, unsigned char* smem, uint64_t* full,
                                        uint64_t* empty, volatile int* abort, int n_items) {
  using C = Cfg<D, PATH>;
  uint32_t sc = 0;  // stages issued so far
  bool ok = true;
  for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
    int b, kvh, c, t0, t1;
    if (!item_range(a, it, b, kvh, c, t0, t1)) continue;
    const int64_t row0 = ((int64_t)b * a.Hkv + kvh) * a.capacity;
    for (int t = t0; t < t1; t += kStageTokens, ++sc) {
      const int slot = sc % C::NS;
      const uint32_t round = sc / C::NS;
      if (!mbar_wait(empty + slot, (round & 1) ^ 1, abort)) {
        ok = false;
        break;
      }
      const int n = min(kStageTokens, t1 - t);
      const uint32_t cb = n * C::RB, sb = n * C::NG * 4;
      unsigned char* stg = smem + slot * C::STAGE;
      const int64_t row = row0 + t;
      mbar_arrive_expect_tx(full + slot, 2 * cb + 2 * sb);
      bulk_g2s(stg + C::KC, a.k_packed + row * C::RB, cb, full + slot);
      bulk_g2s(stg + C::VC, a.v_packed + row * C::RB, cb, full + slot);
      bulk_g2s(stg + C::KS, a.k_scales + row * C::NG, sb, full + slot);
      bulk_g2s(stg + C::VS, a.v_scales + row * C::NG, sb, full + slot);
    }
  }
  if (!ok)  // copies still in flight must land before the CTA exits
    for (uint32_t s = sc > (uint32_t)C::NS ? sc - C::NS : 0; s < sc; ++s)
      mbar_drain(full + s % C::NS, (s / C::NS) & 1);
}

template <int D, int PATH>
__global__ void __launch_bounds__(kMmaThreads, 1) decode_mma_kernel(DecodeArgs a) {
  using C = Cfg<D, PATH>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR);
  uint64_t* empty = full + C::NS;
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::ABORT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kWarps);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int n_items = a.B * a.Hkv * a.plan.n_chunks;
  if (warp == kWarps) {
    if (lane == 0) produce<D, PATH>(a, smem, full, empty, abort, n_items);
    return;
  }
  const int gid = lane >> 2, tig = lane & 3;
  const int rho[4] = {slot_row(2 * tig), slot_row(2 * tig + 1), 8 + slot_row(2 * tig),
                      8 + slot_row(2 * tig + 1)};
  const int krow[2] = {slot_row(gid), 8 + slot_row(gid)};
  WarpState<D, PATH> st;
  uint32_t sc = 0;  // stages consumed so far
  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    int b, kvh, c, t0, t1;
    if (!item_range(a, it, b, kvh, c, t0, t1)) continue;
    if (threadIdx.x == 0 && kvh == 0 && c == 0) {
      const int raw = a.ctx_lens[b];
      static_cast<int32_t*>(a.workspace)[b] = (raw < 1 || raw > a.max_ctx) ? 1 : 0;
    }
    prep_query<D, PATH>(a, b, kvh, smem, st);
#pragma unroll
    for (int j = 0; j < C::NACC; ++j)
#pragma unroll
      for (int r = 0; r < 4; ++r) st.acc[j][r] = 0.0f;
#pragma unroll
    for (int g = 0; g < C::NG; ++g) st.vsc[g] = 1.0f;
    st.m = -INFINITY;
    st.l = 0.0f;
    st.vset = false;
    for (int t = t0; t < t1; t += kStageTokens, ++sc) {
      const int slot = sc % C::NS;
      const uint32_t round = sc / C::NS;
      const bool ok = mbar_wait(full + slot, round & 1, abort);
      const int valid = min(16, min(kStageTokens, t1 - t) - 16 * warp);
      if (ok && valid > 0)
        process_tile<D, PATH>(smem + slot * C::STAGE, 16 * warp, valid, gid, tig, rho, krow, st);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + slot);
    }
    finish_item<D, PATH>(a, smem, st, b, kvh, c, *abort != 0);
  }
}

template <int D, int PATH>
cudaError_t launch_mma(const DecodeArgs& a, cudaStream_t stream) {
  using C = Cfg<D, PATH>;
  cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel<D, PATH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = a.B * a.Hkv * a.plan.n_chunks;
  const int grid = n_items < sms ? n_items : sms;
  decode_mma_kernel<D, PATH><<<grid, kMmaThreads, C::BYTES, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool decode_mma_supported(int d, int G) {
  return (d == 128 && G >= 1 && G <= 8) || (d == 256 && G >= 1 && G <= 4);
}

cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  if (a.d == 128 && G >= 5 && G <= 8) return launch_mma<128, 0>(a, stream);
  if (a.d == 128 && G >= 1 && G <= 4) return launch_mma<128, 1>(a, stream);
  if (a.d == 256 && G >= 1 && G <= 4) return launch_mma<256, 1>(a, stream);
  return cudaErrorNotSupported;
}

}  // namespace tq
