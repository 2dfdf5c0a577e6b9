// decode_mma.cu -- split-K decode attention on the packed int4 cache with the
// GQA contractions on tensor cores (mma.sync m16n8k16, f16 x f16 -> f32).
//
// Attention runs directly on the packed codes ("fused sdpa_int4",
// Open-TQ-Metal abstract): no dequantized K/V matrix exists anywhere (forum
// summary, section "eliminating intermediate matrices"); codes are widened to
// f16 in registers, and the fp32 group scales are applied around the
// contractions.  Softmax runs online with a running maximum and fp32 sums
// (section "numerical stability": the scaling trick and high-precision
// accumulators); exp2 is the hardware approximation, relative error ~2^-22.
//
// Work: persistent CTAs, one per SM, walk a list of items (sequence b, kv
// head, context chunk).  Each item's rows (packed K, packed V, K scales, V
// scales) stream through a ring of shared-memory stages filled by 1-D bulk
// async copies that complete on mbarriers.  There is no producer warp: every
// warp takes TPW 16-token tiles of each stage; the last warp to finish a stage
// (counted with a shared-memory atomic) queues its refill, and the next warp to
// leave any stage issues the queued refills in stage order, so all warps of the
// CTA compute and the slowest warp does not also carry the refills.  Each warp keeps its own running (max, sum,
// acc); the warps are merged per item in shared memory into one split-K
// partial (max in log2 units, sum, unnormalized acc[d]) per query head, and
// merge.cu combines the chunks and rotates the output back.
//
// Exactness on the tensor cores.  Codes (-7..7) are exact in f16.  The fp32
// operand of each contraction is split into hi + lo f16 parts (about 22 bits):
//  - scores: rows of the A operand are [query hi; query lo], so the 16 rows of
//    m16n8k16 hold 8 heads x 2 parts and hi + lo is summed per thread after
//    the product.  Each head's rotated, scaled query is first multiplied by a
//    power of two so its largest element lies in [2^13, 2^14) (f16 range).
//    Per group of 32 dims the product is scaled by the token's fp32 K scale.
//    The K codes enter as exact f16 subnormals (c + 8) 2^-24 (one LOP3 per two
//    codes); the epilogue scales by 2^24 and removes the offset 8 sum_g q.
//  - P.V: the operand is P' = 2^(S - m - F) * s_v[token, group], split into
//    hi + lo.  F (per warp) keeps P' below 2^15: it is set from the first
//    tile's V scales and raised, with an exact power-of-two rescale of the
//    accumulators and the running sum, whenever a later tile would overflow.
//    The partial then reports max m + F.
// Three arrangements (template PATH):
//  - PATH 0 (heads on rows, 5..8 query heads per kv head, d = 128; the
//    codebook caches only): scores C = [q hi; q lo] x K^T; P.V C = [P' hi;
//    P' lo] x levels, where the score accumulator fragment is reused as the
//    P.V A operand without shuffles.  The accumulator holds the hi and lo rows
//    apart: d/8 x 4 registers.
//  - PATH 2 (5..8 query heads, d = 128, int4): scores as PATH 0; P.V with
//    dims on the rows, C = V^T x P' hi + V^T x P' lo (two MMAs into one
//    accumulator), where the score fragment of head gid is already the B
//    operand of column gid.  The same MMA count as PATH 0 with half the
//    accumulator registers (d/16 x 4), which buys a third 16-token tile per
//    warp: the kernel is bound by the latency of each tile's dependent chain
//    (scores, max, weights, P.V), so the number of tiles in flight per
//    scheduler sets the speed.
//  - PATH 1 (dims on rows, 1..4 query heads, d = 96, 128 or 256): scores as
//    above with each head on two neighbouring rows; P.V C = V^T x [P' hi,
//    P' lo per head] with dims on the rows, so the accumulator is d/16 x 4
//    registers.
// Cache formats (template FMT):
//  - FMT 0: int4 codes (above).
//  - FMT 2, 3, 4: codebook indices of that many bits (PATH 0 only).  Each CTA
//    first builds a table over index pairs holding the two levels as f16 hi
//    and lo parts (levels scaled by a power of two into [0.5, 1)).  Every MMA
//    operand register is then one 8-byte table read, and each k-step runs
//    twice (hi levels, lo levels) into the same accumulator; sigma is applied
//    per group as the int4 scale is.
// Token order: slot k of a 16-token tile holds tile row pi(k), chosen so that
// the K-code and scale loads of a warp hit distinct shared-memory banks.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>

#include "cb_vector.cuh"
#include "quantize_vector.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz: a wait never lasts this long
constexpr uint32_t kFull = 0xffffffffu;

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
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
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
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

// Bounded wait that ignores *abort (drains copies still in flight).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return;
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

// Score operand: two int4 codes -> f16x2 in one LOP3, without the subtraction.
// Flipping bit 3 gives u = c + 8 in 1..15, which OR-ed under a zero exponent is
// the subnormal f16 u * 2^-24 (bits 4..7: 16 u * 2^-24), exact.  The query
// entries that meet the bits 4..7 codes are divided by 16, so an MMA over a
// group yields 2^-24 sum_j q_j (c_j + 8); the tile epilogue scales it by 2^24
// and removes 8 sum_j q_j, a constant of (head, group).
__device__ __forceinline__ uint32_t kcodes_lo(uint32_t x) { return and_xor(x, 0x000F000Fu, 0x00080008u); }
__device__ __forceinline__ uint32_t kcodes_hi(uint32_t x) { return and_xor(x, 0x00F000F0u, 0x00800080u); }

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

// 2^x with the hardware approximation (relative error about 2^-22; results
// below 2^-126 flush to zero, which no softmax weight here needs)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^e as a float for |e| <= 126
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// The NG fp32 scales of one row (rows are NG * 4 bytes: 16-byte units when NG
// is a multiple of 4, else 4-byte aligned).
template <int NG>
__device__ __forceinline__ void load_row_scales(const float* p, float (&out)[NG]) {
  if constexpr (NG % 4 == 0) {
#pragma unroll
    for (int q = 0; q < NG / 4; ++q) {
      const float4 v = reinterpret_cast<const float4*>(p)[q];
      out[4 * q] = v.x;
      out[4 * q + 1] = v.y;
      out[4 * q + 2] = v.z;
      out[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int g = 0; g < NG; ++g) out[g] = p[g];
  }
}

// K codes of group g for one token: the half-words of sub-blocks 2tig and
// 2tig + 1 (in-group coordinates 8tig .. 8tig + 7) in one word.  kw holds the
// two sub-blocks' bytes as words: NG = 4, 8: sub-block 0 in words 0 .. NG/2 - 1,
// sub-block 1 after it; NG = 3: 12 bytes, g0 g1 | g2 g0' | g1' g2'.
template <int NG>
__device__ __forceinline__ uint32_t kcode_word(const uint32_t (&kw)[NG], int g) {
  if constexpr (NG == 3) {
    return g == 0 ? prmt(kw[0], kw[1], 0x7610u) : g == 1 ? prmt(kw[0], kw[2], 0x5432u)
                                                          : prmt(kw[1], kw[2], 0x7610u);
  } else {
    return prmt(kw[g / 2], kw[NG / 2 + g / 2], (g & 1) ? 0x7632u : 0x5410u);
  }
}

// ------------------------------------------------------------ configuration

// Batches up to this size use the list of non-empty items (its prefix sums
// live in shared memory); larger ones walk every (sequence, kv head, chunk).
constexpr int kMaxListB = 1024;

template <int D, int PATH, int FMT>
struct Cfg {
  static constexpr int NW = 8;                  // warps per CTA (all consumers)
  static constexpr int TPW = D == 256 ? 1 : PATH == 2 ? 3 : 2;  // 16-token tiles per warp per stage
  static constexpr int THREADS = 32 * NW;
  static constexpr int ST = 16 * TPW * NW;      // tokens per pipeline stage
  static constexpr int NG = D / 32;             // quantization groups per vector
  static constexpr int RB = FMT ? D * FMT / 8 : D / 2;  // packed bytes per row
  static constexpr int NH = PATH == 1 ? 4 : 8;  // query heads per kv head (max)
  static constexpr int NACC = PATH == 0 ? 4 * NG : 2 * NG;  // accumulator fragments
  static constexpr int NS = D == 256 || PATH == 2 ? 3 : 4;   // pipeline stages
  // scale rows of 12 bytes (d = 96) are not 16-byte copy units: a stage's
  // scales arrive as the 16-byte aligned superset, SPAD bytes more per region
  static constexpr int SPAD = (NG % 4) ? 32 : 0;
  static constexpr int KC = 0;                               // stage: packed K rows
  static constexpr int VC = ST * RB;                         //        packed V rows
  static constexpr int KS = 2 * ST * RB;                     //        K scales
  static constexpr int VS = KS + ST * NG * 4 + SPAD;         //        V scales
  static constexpr int STAGE = VS + ST * NG * 4 + SPAD;
  static constexpr int al(int x) { return (x + 127) / 128 * 128; }  // 128-byte regions
  static constexpr int BAR = NS * STAGE;                     // uint64 full[NS]
  static constexpr int CNT = al(BAR + 8 * NS);               // int finished-warp count[NS]
  static constexpr int CUR = al(CNT + 4 * NS);               // int refill cursor[8], queue[3]
  static constexpr int SKEW = al(CUR + 44);                  // int [NS] first scale row's byte offset
  static constexpr int QA = al(SKEW + 4 * NS);               // f16 [NG][2][16][16] score A
  static constexpr int QS = al(QA + NG * 2 * 16 * 16 * 2);   // float [NH][D] query
  static constexpr int QEXP = al(QS + 4 * NH * D);           // float [NH]
  static constexpr int QK8 = al(QEXP + 4 * 8);               // float [NH][NG] -8 sum_g q
  // the warps' accumulators merge through MB buffers (more than 8 warps: in rounds)
  static constexpr int MB = NW < 8 ? NW : 8;
  static constexpr int MACC = al(QK8 + 4 * NH * NG);         // float [MB][NH][D]
  static constexpr int MM = al(MACC + 4 * MB * NH * D);      // float [NW][NH] max
  static constexpr int ML = al(MM + 4 * NW * NH);            // float [NW][NH] sum
  static constexpr int MW = al(ML + 4 * NW * NH);            // float [NW][NH] weight
  static constexpr int MTOT = al(MW + 4 * NW * NH);          // float [NH] max, [NH] sum
  static constexpr int ABORT = al(MTOT + 4 * 2 * NH);        // int
  static constexpr int PFX = al(ABORT + 16);                 // int [kMaxListB + 1] item prefix
  static constexpr int LUT = al(PFX + 4 * (kMaxListB + 1));  // codebook: uint2 [2^(2 FMT)]
  static constexpr int BYTES = LUT + (FMT ? 8 << (2 * FMT) : 0);
  static_assert(BYTES <= 227 * 1024, "shared memory");
  static_assert(FMT == 0 || (PATH == 0 && D == 128), "codebook decode: heads on rows, d = 128");
  static_assert(STAGE % 16 == 0 && VC % 16 == 0 && KS % 16 == 0 && VS % 16 == 0, "alignment");
};

template <int THREADS>
__device__ __forceinline__ void barrier_all() {
  asm volatile("bar.sync 1, %0;" ::"n"(THREADS) : "memory");
}

__device__ __forceinline__ int clamp_ctx_mma(int T, int max_ctx) {
  return T < 1 ? 1 : (T > max_ctx ? max_ctx : T);
}

// Item it -> (sequence b, kv head, chunk c) and its token range [t0, t1).
// With the item list (pfx != nullptr) the items are only the chunks that hold
// tokens, sequence by sequence (pfx[b] = items of the sequences before b), so
// that CTAs taking every gridDim.x-th item get equal shares even when the
// sequences' lengths differ; otherwise every chunk of the max_ctx plan is an
// item and those past a sequence's end return false.
__device__ __forceinline__ bool item_range(const DecodeArgs& a, const int* pfx, int it, int& b,
                                           int& kvh, int& c, int& t0, int& t1) {
  if (pfx != nullptr) {
    int lo = 0, hi = a.B;  // pfx[0] = 0 <= it < pfx[B]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pfx[mid] <= it) lo = mid;
      else hi = mid;
    }
    b = lo;
    const int T = clamp_ctx_mma(a.ctx_lens[b], a.max_ctx);
    const int nc = (T + a.plan.chunk - 1) / a.plan.chunk;
    const int r = it - pfx[b];
    kvh = r / nc;
    c = r % nc;
    t0 = c * a.plan.chunk;
    t1 = min(T, t0 + a.plan.chunk);
    return true;
  }
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

// Refill cursor (shared memory, used by one thread at a time): cur[0] item,
// cur[1] next token, cur[2] end token, cur[3] sequence, cur[4] kv head,
// cur[5] stages issued; cur[6] items in the call, cur[7] 1 if the item list
// in smem + PFX is used (both set once at kernel start and only read after).
// Issues the next stage of this CTA's stage sequence
// into `slot`; returns false when the sequence is exhausted.
template <int D, int PATH, int FMT>
__device__ __forceinline__ bool issue_next(const DecodeArgs& a, unsigned char* smem, int* cur,
                                           uint64_t* full, int slot) {
  using C = Cfg<D, PATH, FMT>;
  const int n_items = cur[6];
  const int* pfx = cur[7] ? reinterpret_cast<const int*>(smem + C::PFX) : nullptr;
  int it = cur[0], t = cur[1], t1 = cur[2];
  int b = cur[3], kvh = cur[4];
  while (t >= t1) {
    it += gridDim.x;
    if (it >= n_items) {
      cur[0] = it;
      return false;
    }
    int c, t0;
    item_range(a, pfx, it, b, kvh, c, t0, t1);
    t = t0;
  }
  const int n = min(C::ST, t1 - t);
  if (a.q_rot_overlap == 2 && t + n == t1 &&
      t1 == clamp_ctx_mma(a.ctx_lens[b], a.max_ctx))  // holds the row the preceding grid appends
    asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t cb = n * C::RB;
  unsigned char* stg = smem + slot * C::STAGE;
  const int64_t row = ((int64_t)b * a.Hkv + kvh) * a.capacity + t;
  uint64_t* bar = full + slot;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // earlier reads of the slot
  // scales: bytes [s0, s1) of each scales tensor; with rows of 16-byte multiples
  // one copy, else the 16-byte aligned superset from a0 (the first row lands
  // s0 - a0 bytes into the region), its last few bytes by plain loads where the
  // superset would run past the end of the tensor
  const int64_t s0 = row * C::NG * 4, s1 = (row + n) * C::NG * 4;
  int64_t a0 = s0, bulk_end = s1;
  if constexpr (C::SPAD != 0) {
    const int64_t tot = (int64_t)a.B * a.Hkv * a.capacity * C::NG * 4;
    a0 = s0 & ~(int64_t)15;
    const int64_t a1 = (s1 + 15) & ~(int64_t)15;
    bulk_end = a1 <= tot ? a1 : (tot & ~(int64_t)15);
  }
  const uint32_t sb = (uint32_t)(bulk_end - a0);
  reinterpret_cast<int*>(smem + C::SKEW)[slot] = (int)(s0 - a0);
  if (!(a.test_starve && cur[5] == 0)) {  // test hook: the first stage never arrives
    if constexpr (C::SPAD != 0) {
      for (int64_t o = bulk_end; o < s1; o += 4) {  // < 16 bytes at the end of the tensor
        const uint32_t d = (uint32_t)(o - a0);
        *reinterpret_cast<float*>(stg + C::KS + d) = *reinterpret_cast<const float*>(
            reinterpret_cast<const unsigned char*>(a.k_scales) + o);
        *reinterpret_cast<float*>(stg + C::VS + d) = *reinterpret_cast<const float*>(
            reinterpret_cast<const unsigned char*>(a.v_scales) + o);
      }
    }
    mbar_arrive_expect_tx(bar, 2 * cb + 2 * sb);
    bulk_g2s(stg + C::KC, a.k_packed + row * C::RB, cb, bar);
    bulk_g2s(stg + C::VC, a.v_packed + row * C::RB, cb, bar);
    if (sb > 0) {
      bulk_g2s(stg + C::KS, reinterpret_cast<const unsigned char*>(a.k_scales) + a0, sb, bar);
      bulk_g2s(stg + C::VS, reinterpret_cast<const unsigned char*>(a.v_scales) + a0, sb, bar);
    }
  }
  cur[0] = it;
  cur[1] = t + C::ST;
  cur[2] = t1;
  cur[3] = b;
  cur[4] = kvh;
  cur[5] += 1;
  return true;
}

// Refill queue (cur[8] stages freed by every warp, cur[9] refills issued,
// cur[10] lock; lane 0 of a warp only).  A stage freed by the last warp to
// finish it is only queued; the refill is issued by the next warp to finish a
// stage, which is one of the fastest, instead of by the last one, whose
// refills would otherwise keep it last (and alone doing every refill) for the
// rest of the item.  Refills are issued in order under the lock.
template <int D, int PATH, int FMT>
__device__ __forceinline__ void service_refills(const DecodeArgs& a, unsigned char* smem, int* cur,
                                                uint64_t* full, volatile int* abort) {
  using C = Cfg<D, PATH, FMT>;
  volatile int* q = cur + 8;
  if (q[1] >= q[0] || *abort) return;
  if (atomicCAS(cur + 10, 0, 1) != 0) return;  // another warp is issuing
  __threadfence_block();
  while (q[1] < q[0] && !*abort) {
    const int r = q[1];
    issue_next<D, PATH, FMT>(a, smem, cur, full, r % C::NS);
    q[1] = r + 1;
  }
  __threadfence_block();
  atomicExch(cur + 10, 0);
}

// Per-thread state of one warp for one item.
template <int D, int PATH, int FMT>
struct WarpState {
  float acc[Cfg<D, PATH, FMT>::NACC][4];  // P.V accumulators (fragments), scaled by 2^-F
  uint32_t qa_addr;                  // this lane's ldmatrix row address of the score A tiles
  uint32_t k8_addr;                  // shared address of -8 sum_g q of this thread's head
  float m;                           // running max of this thread's head (log2 units)
  float2 l;                          // this thread's share of the running sum (two partial
                                     // sums, added at the end), scaled by 2^-F
  float qexp;                        // 2^E of this thread's head (query normalisation)
  float cexp;                        // codebook: 2^e, the levels' normalisation (else 1)
  uint32_t lut;                      // codebook: shared address of the level-pair table
  int F;                             // V-scale normalisation exponent
  bool fset;                         // F chosen for this item
};

// Rotated, scaled query of the item's G heads -> smem (normalised by a power
// of two per head), then every thread builds its score A fragments.  Warp
// w < NH prepares head w; the FWHT runs in registers and shuffles.
template <int D, int PATH, int FMT>
__device__ __forceinline__ void prep_query(const DecodeArgs& a, int b, int kvh, unsigned char* smem,
                                           WarpState<D, PATH, FMT>& st, bool start_stream,
                                           int* cur, uint64_t* full) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int E = D / 32;  // elements per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  float* qs = reinterpret_cast<float*>(smem + C::QS);
  float* qexp = reinterpret_cast<float*>(smem + C::QEXP);
  // Heads are prepared by warps 0 .. NW/2 - 1 (two heads each when NH == 8)
  // while the last warp issues the first copies; with a fused append it first
  // waits (named barrier 2, warps 4, 5 and NW - 1) for the new tokens' rows.
  constexpr int HPW = (C::NH + C::NW / 2 - 1) / (C::NW / 2);  // heads per warp
  if (start_stream && threadIdx.x >= C::THREADS - 32) {
    if (a.k_new != nullptr) asm volatile("bar.sync 2, 96;" ::: "memory");
    if (threadIdx.x == C::THREADS - 32)
      for (int s = 0; s < C::NS; ++s)
        if (!issue_next<D, PATH, FMT>(a, smem, cur, full, s)) break;
  }
  // every head of this warp is loaded first, so all their loads (and the signs)
  // are in flight together: one memory latency for the warp, not one per head
  float xs[HPW][E];
  int8_t sg[E];
  const bool wht = a.signs != nullptr && a.q_rot == nullptr;
  if (warp < C::NW / 2) {
    if (a.q_rot != nullptr || a.inputs_pending)
      asm volatile("griddepcontrol.wait;" ::: "memory");  // written by the preceding grid
    if (wht) {
#pragma unroll
      for (int e = 0; e < E; ++e) sg[e] = a.signs[lane * E + e];  // bytes: no alignment needed
    }
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
      const int h = warp * HPW + hh;
      float* x = xs[hh];
      if (h >= C::NH || h >= G) {
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = 0.0f;
        continue;
      }
      const int64_t base = ((int64_t)b * a.Hq + (int64_t)kvh * G + h) * D + lane * E;
      if (E % 4 != 0) {  // d = 96: E = 3 consecutive values, 4-byte loads
        const float* src = a.q_rot != nullptr ? a.q_rot + base : nullptr;
#pragma unroll
        for (int e = 0; e < E; ++e)
          x[e] = src ? src[e]
                     : a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[base + e])
                                : static_cast<const float*>(a.q)[base + e];
      } else if (a.q_rot != nullptr) {  // SRFT variant: the query is already rotated (fp32)
#pragma unroll
        for (int e = 0; e < (E % 4 == 0 ? E : 0); e += 4) {
          const float4 v = *reinterpret_cast<const float4*>(a.q_rot + base + e);
          x[e] = v.x;
          x[e + 1] = v.y;
          x[e + 2] = v.z;
          x[e + 3] = v.w;
        }
      } else if (a.q_bf16) {  // E consecutive bf16 values: one 8- or 16-byte load
        uint32_t u[E / 2];
        if (E == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.q) + base);
          u[0] = v.x;
          u[1] = v.y;
        } else {
          const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + base);
          u[0] = v.x;
          u[1] = v.y;
          u[E > 4 ? 2 : 0] = v.z;
          u[E > 4 ? 3 : 1] = v.w;
        }
#pragma unroll
        for (int e = 0; e < E; ++e)
          x[e] = __uint_as_float(e & 1 ? (u[e / 2] & 0xFFFF0000u) : (u[e / 2] << 16));
      } else {
#pragma unroll
        for (int e = 0; e < (E % 4 == 0 ? E : 0); e += 4) {
          const float4 v = *reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + base + e);
          x[e] = v.x;
          x[e + 1] = v.y;
          x[e + 2] = v.z;
          x[e + 3] = v.w;
        }
      }
    }
  }
  for (int hh = 0; hh < HPW; ++hh) {
    const int h = warp * HPW + hh;
    if (warp >= C::NW / 2 || h >= C::NH) break;
    float* x = xs[hh];
    if (h < G) {
      if constexpr ((E & (E - 1)) == 0) {  // the Hadamard rotation needs a power-of-two width
      if (wht) {
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] *= (float)sg[e];
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
      }
      const float mul = a.attn_scale * kLog2e * (wht ? rsqrtf((float)D) : 1.0f);
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x[e] *= mul;
        amax = fmaxf(amax, fabsf(x[e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
      int ex = 0;
      frexpf(amax, &ex);                   // amax = m * 2^ex, m in [0.5, 1)
      int sh = amax > 0.0f ? 14 - ex : 0;  // amax * 2^sh in [2^13, 2^14)
      sh = max(-120, min(120, sh));
#pragma unroll
      for (int e = 0; e < E; ++e) qs[h * D + lane * E + e] = x[e] * pow2i(sh);
      if (lane == 0) qexp[h] = pow2i(-sh);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qs[h * D + lane * E + e] = 0.0f;
      if (lane == 0) qexp[h] = 1.0f;
    }
  }
  barrier_all<C::THREADS>();
  // Score A tiles in shared memory, f16 [group][k-step][row][k]: row r < 8 is
  // the hi part of head h(r), row 8 + r its lo part.  int4: MMA index k of
  // k-step ks is coordinate 32g + 8((k%8)/2) + 2ks + k/8 + 4(k%2), the order in
  // which the K-code words are unpacked; k >= 8 meets the codes of bits 4..7,
  // whose operand carries a factor 16 (kcodes_hi), so those entries are q / 16.
  // Codebook: coordinate 32g + 8((k%8)/2) + 4ks + 2(k/8) + k%2, the index pairs
  // of tile_scores_cb.  The two 16-byte halves of a row swap when row bit 2 is
  // set, so ldmatrix phases hit distinct banks.  Beside them (int4), -8 sum_g q
  // per head and group.
  __half* qa = reinterpret_cast<__half*>(smem + C::QA);
  if (FMT == 0 && threadIdx.x < C::NH * C::NG) {
    const int h = threadIdx.x / C::NG, g = threadIdx.x % C::NG;
    float sum = 0.0f;
    for (int j = 0; j < 32; ++j) sum += qs[h * D + 32 * g + j];
    reinterpret_cast<float*>(smem + C::QK8)[threadIdx.x] = -8.0f * sum;
  }
  for (int idx = threadIdx.x; idx < (D / 32) * 2 * 256; idx += C::THREADS) {
    const int k = idx & 15, row = (idx >> 4) & 15, gks = idx >> 8;
    const int g = gks >> 1, ks = gks & 1;
    const int hr = PATH == 1 ? ((row & 7) >> 1) : (row & 7);
    const int dim = FMT ? 32 * g + 8 * ((k & 7) >> 1) + 4 * ks + 2 * (k >> 3) + (k & 1)
                        : 32 * g + 8 * ((k & 7) >> 1) + 2 * ks + (k >> 3) + 4 * (k & 1);
    const float v = qs[hr * D + dim] * ((FMT == 0 && (k >> 3)) ? 0.0625f : 1.0f);  // exact
    const __half hi = __float2half_rn(v);
    const __half val = row < 8 ? hi : __float2half_rn(v - __half2float(hi));
    const int half16 = (k >> 3) ^ ((row >> 2) & 1);
    qa[(gks * 16 + row) * 16 + half16 * 8 + (k & 7)] = val;
  }
  barrier_all<C::THREADS>();
  const int gid = lane >> 2;
  const int hrow = PATH == 1 ? gid >> 1 : gid;
  {
    const int mi = lane >> 3, row = (lane & 7) + 8 * (mi & 1), kb = mi >> 1;
    st.qa_addr = smem_u32(smem + C::QA) + row * 32 + ((kb ^ ((row >> 2) & 1)) * 16);
  }
  st.k8_addr = smem_u32(smem + C::QK8) + hrow * C::NG * 4;
  st.qexp = qexp[hrow] * st.cexp;
}

template <int D, int PATH, int FMT>
__device__ __forceinline__ void scale_acc2(WarpState<D, PATH, FMT>& st, float f0, float f1) {
  const float2 ff = make_float2(f0, f1);
#pragma unroll
  for (int j = 0; j < Cfg<D, PATH, FMT>::NACC; ++j)
#pragma unroll
    for (int r = 0; r < 4; r += 2) {
      const float2 v = __fmul2_rn(make_float2(st.acc[j][r], st.acc[j][r + 1]), ff);
      st.acc[j][r] = v.x;
      st.acc[j][r + 1] = v.y;
    }
}

template <int D, int PATH, int FMT>
__device__ __forceinline__ void scale_acc(WarpState<D, PATH, FMT>& st, float f) {
  const float2 ff = make_float2(f, f);
#pragma unroll
  for (int j = 0; j < Cfg<D, PATH, FMT>::NACC; ++j)
#pragma unroll
    for (int r = 0; r < 4; r += 2) {
      const float2 v = __fmul2_rn(make_float2(st.acc[j][r], st.acc[j][r + 1]), ff);
      st.acc[j][r] = v.x;
      st.acc[j][r + 1] = v.y;
    }
}

// The per-stage work of one warp is split so that the P.V of one stage and
// the scores of the next run as one straight-line block the compiler can
// interleave; the branchy softmax update follows it.  A warp owns TPW
// consecutive 16-token tiles of each stage: tile u covers rows r0 + 16u ..
// r0 + 16u + 15, of which the first `nvalid` rows from r0 on are real tokens.
// rho[i]: tile rows of this thread's MMA slots 2tig, 2tig+1, 8+2tig, 9+2tig;
// krow[nt]: tile row of score n-tile nt's column gid.

// Scores before the qexp factor, S = sum_g s_k[t, g] (q_hi + q_lo) . c_k[t, g];
// unless FULL, rows past nvalid get -inf.  Branch-free.  Per group the two
// MMAs give x = 2^-24 sum_j q_j (c_j + 8) (kcodes_lo / kcodes_hi), and the
// group's term is s_k (2^24 x - 8 sum_j q_j).
template <int D, int PATH, int FMT, int TPW, bool FULL>
__device__ __forceinline__ void tile_scores(const unsigned char* stg, int skew, int r0, int nvalid, int tig,
                                            const int (&rho)[4], const int (&krow)[2],
                                            const WarpState<D, PATH, FMT>& st, float (&S)[TPW][4]) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int NG = C::NG, RB = C::RB, SB = 2 * NG;  // SB: bytes of one of a row's 8 sub-blocks
  const unsigned char* kc = stg + C::KC + r0 * RB;
  const float* ks = reinterpret_cast<const float*>(stg + C::KS + skew) + r0 * NG;
  uint32_t kw[TPW][2][NG];  // per tile and n-tile: sub-blocks 2tig, 2tig+1 of token krow[nt]
  float sk[TPW][4][NG];
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const unsigned char* kb = kc + (16 * u + krow[nt]) * RB + 2 * SB * tig;
      if constexpr (NG % 4 == 0) {
        const uint4* kp = reinterpret_cast<const uint4*>(kb);
#pragma unroll
        for (int q = 0; q < NG / 4; ++q) {
          const uint4 v = kp[q];
          kw[u][nt][4 * q] = v.x;
          kw[u][nt][4 * q + 1] = v.y;
          kw[u][nt][4 * q + 2] = v.z;
          kw[u][nt][4 * q + 3] = v.w;
        }
      } else {  // 12 bytes at a 4-byte aligned offset
#pragma unroll
        for (int q = 0; q < NG; ++q) kw[u][nt][q] = reinterpret_cast<const uint32_t*>(kb)[q];
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) load_row_scales<NG>(ks + (16 * u + rho[i]) * NG, sk[u][i]);
  }
  float k8[NG];  // -8 sum_g q of this thread's head
  if constexpr (NG % 4 == 0) {
#pragma unroll
    for (int q = 0; q < NG / 4; ++q)
      asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                   : "=f"(k8[4 * q]), "=f"(k8[4 * q + 1]), "=f"(k8[4 * q + 2]), "=f"(k8[4 * q + 3])
                   : "r"(st.k8_addr + 16 * q));
  } else {
#pragma unroll
    for (int q = 0; q < NG; ++q)
      asm volatile("ld.shared.f32 %0, [%1];" : "=f"(k8[q]) : "r"(st.k8_addr + 4 * q));
  }
#pragma unroll
  for (int u = 0; u < TPW; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) S[u][i] = 0.0f;
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    uint32_t a[2][4];
    ldsm_x4(st.qa_addr + (2 * g) * 512, a[0][0], a[0][1], a[0][2], a[0][3]);
    ldsm_x4(st.qa_addr + (2 * g + 1) * 512, a[1][0], a[1][1], a[1][2], a[1][3]);
#pragma unroll
    for (int u = 0; u < TPW; ++u)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        // in-group coordinates 8tig .. 8tig+7 of group g, nibble j <-> 8tig + j
        const uint32_t X = kcode_word<NG>(kw[u][nt], g);
        const uint32_t Y = X >> 8;
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma16816(c, a[0][0], a[0][1], a[0][2], a[0][3], kcodes_lo(X), kcodes_hi(X));
        mma16816(c, a[1][0], a[1][1], a[1][2], a[1][3], kcodes_lo(Y), kcodes_hi(Y));
        const float2 x = __ffma2_rn(__fadd2_rn(make_float2(c[0], c[1]), make_float2(c[2], c[3])),
                                    make_float2(16777216.0f, 16777216.0f), make_float2(k8[g], k8[g]));
        S[u][2 * nt] = fmaf(sk[u][2 * nt][g], x.x, S[u][2 * nt]);
        S[u][2 * nt + 1] = fmaf(sk[u][2 * nt + 1][g], x.y, S[u][2 * nt + 1]);
      }
  }
  if (!FULL)
#pragma unroll
    for (int u = 0; u < TPW; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) S[u][i] = 16 * u + rho[i] < nvalid ? S[u][i] : -INFINITY;
}

// Codebook scores.  Per group the B operand is the levels C[index] of the
// token's coordinates, as f16 hi + lo parts read from the level-pair table
// (entry i0 | i1 << FMT holds C[i0], C[i1] as an f16x2 hi part and an f16x2 lo
// part), so the group's product sum_j (q_hi + q_lo)_j (C_hi + C_lo)[index_j]
// collects all four partial products in one accumulator; then
// S = sum_g sigma_k[t, g] x_g.  Thread tig takes in-group coordinates 8tig ..
// 8tig + 7 (bits 8 FMT tig .. of the group's bit string) as the index pairs
// (8tig + 2m, 8tig + 2m + 1), m = 0..3.  Branch-free.  EXACT: every level is
// an f16 (the lo parts are zero), so only the hi parts are read and multiplied.
template <int D, int PATH, int FMT, int TPW, bool FULL, bool EXACT>
__device__ __forceinline__ void tile_scores_cb(const unsigned char* stg, int skew, int r0, int nvalid, int tig,
                                               const int (&rho)[4], const int (&krow)[2],
                                               const WarpState<D, PATH, FMT>& st,
                                               const unsigned char* lutp, float (&S)[TPW][4]) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int NG = C::NG, RB = C::RB, GB = 4 * FMT;  // GB: bytes per group
  constexpr uint32_t KM = (1u << (2 * FMT)) - 1;  // key mask
  const unsigned char* kc = stg + C::KC + r0 * RB;
  const float* ks = reinterpret_cast<const float*>(stg + C::KS + skew) + r0 * NG;
  // the thread's 8 FMT bits of a group start at byte FMT tig of the group
  const int wo = (FMT * tig) >> 2, sh = 8 * ((FMT * tig) & 3);
  uint32_t pc[TPW][2][NG];
  float sk[TPW][4][NG];
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const uint32_t* gw =
            reinterpret_cast<const uint32_t*>(kc + (16 * u + krow[nt]) * RB + g * GB) + wo;
        pc[u][nt][g] = FMT == 3 ? __funnelshift_r(gw[0], gw[1], sh) : gw[0] >> sh;
      }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < NG / 4; ++q) {
        const float4 v = reinterpret_cast<const float4*>(ks + (16 * u + rho[i]) * NG)[q];
        sk[u][i][4 * q] = v.x;
        sk[u][i][4 * q + 1] = v.y;
        sk[u][i][4 * q + 2] = v.z;
        sk[u][i][4 * q + 3] = v.w;
      }
  }
#pragma unroll
  for (int u = 0; u < TPW; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) S[u][i] = 0.0f;
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    uint32_t a[2][4];
    ldsm_x4(st.qa_addr + (2 * g) * 512, a[0][0], a[0][1], a[0][2], a[0][3]);
    ldsm_x4(st.qa_addr + (2 * g + 1) * 512, a[1][0], a[1][1], a[1][2], a[1][3]);
#pragma unroll
    for (int u = 0; u < TPW; ++u)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const uint32_t x = pc[u][nt][g];
        uint2 e[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const unsigned char* ep = lutp + (((x >> (2 * FMT * m)) & KM) << 3);
          if (EXACT) e[m] = make_uint2(*reinterpret_cast<const uint32_t*>(ep), 0u);
          else e[m] = *reinterpret_cast<const uint2*>(ep);
        }
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        mma16816(c, a[0][0], a[0][1], a[0][2], a[0][3], e[0].x, e[1].x);
        if (!EXACT) mma16816(c, a[0][0], a[0][1], a[0][2], a[0][3], e[0].y, e[1].y);
        mma16816(c, a[1][0], a[1][1], a[1][2], a[1][3], e[2].x, e[3].x);
        if (!EXACT) mma16816(c, a[1][0], a[1][1], a[1][2], a[1][3], e[2].y, e[3].y);
        const float2 x2 = __fadd2_rn(make_float2(c[0], c[1]), make_float2(c[2], c[3]));
        S[u][2 * nt] = fmaf(sk[u][2 * nt][g], x2.x, S[u][2 * nt]);
        S[u][2 * nt + 1] = fmaf(sk[u][2 * nt + 1][g], x2.y, S[u][2 * nt + 1]);
      }
  }
  if (!FULL)
#pragma unroll
    for (int u = 0; u < TPW; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) S[u][i] = 16 * u + rho[i] < nvalid ? S[u][i] : -INFINITY;
}

// Running max of this thread's head (log2 units) over the tiles' scores; when
// it grows, the accumulators and the running sum are rescaled.
template <int D, int PATH, int FMT, int TPW>
__device__ __forceinline__ void tile_max(int tig, const float (&S)[TPW][4], WarpState<D, PATH, FMT>& st) {
  float mx = fmaxf(fmax3(S[0][0], S[0][1], S[0][2]), S[0][3]);
#pragma unroll
  for (int u = 1; u < TPW; ++u)
    mx = fmax3(mx, fmax3(S[u][0], S[u][1], S[u][2]), S[u][3]);
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
  const float m_new = fmaxf(st.m, mx * st.qexp);
  if (__any_sync(kFull, m_new > st.m)) {
    const float alpha = ex2(st.m - m_new);  // 0 on the first tile, 1 if unchanged
    if (PATH == 0) {
      scale_acc(st, alpha);
    } else if (PATH == 1) {  // accumulates head tig; its softmax state lives on lane 8 * tig
      scale_acc(st, __shfl_sync(kFull, alpha, 8 * tig));
    } else {  // accumulator columns: heads 2tig (lane 8 tig) and 2tig + 1 (lane 8 tig + 4)
      const float a0 = __shfl_sync(kFull, alpha, 8 * tig), a1 = __shfl_sync(kFull, alpha, 8 * tig + 4);
      scale_acc2(st, a0, a1);
    }
    st.l = __fmul2_rn(st.l, make_float2(alpha, alpha));
    st.m = m_new;
  }
}

// V scales of the warp's rows (unless FULL, zero past nvalid).
template <int D, int PATH, int FMT, int TPW, bool FULL>
__device__ __forceinline__ void load_vscales(const unsigned char* stg, int skew, int r0, int nvalid,
                                             const int (&rho)[4], float (&sv)[TPW][4][D / 32]) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int NG = C::NG;
  const float* vs = reinterpret_cast<const float*>(stg + C::VS + skew) + r0 * NG;
#pragma unroll
  for (int u = 0; u < TPW; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool ok = FULL || 16 * u + rho[i] < nvalid;
      float v[NG];
      load_row_scales<NG>(vs + (16 * u + rho[i]) * NG, v);
#pragma unroll
      for (int g = 0; g < NG; ++g) sv[u][i][g] = ok ? v[g] : 0.0f;
    }
}

// The weights p' = 2^(S - m - F), keeping p' * s_v below 2^14: the exponent F
// follows the largest V scale seen (raised with an exact power-of-two rescale
// of acc, l and these weights, which is rare, so the weights are computed
// first with the current F and the check runs beside them).
template <int D, int PATH, int FMT, int TPW>
__device__ __forceinline__ void tile_weights(const float (&S)[TPW][4],
                                             const float (&sv)[TPW][4][D / 32],
                                             WarpState<D, PATH, FMT>& st, float (&p)[TPW][4]) {
  constexpr int NG = D / 32, NV = 4 * TPW * NG;
  // m = -inf only while every score so far is -inf (no real token yet)
  const float mF = st.m == -INFINITY ? 0.0f : st.m + (float)st.F;
  const float2 qe = make_float2(st.qexp, st.qexp), nm = make_float2(-mF, -mF);
#pragma unroll
  for (int u = 0; u < TPW; ++u)
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      const float2 arg = __ffma2_rn(make_float2(S[u][i], S[u][i + 1]), qe, nm);
      p[u][i] = ex2(arg.x);
      p[u][i + 1] = ex2(arg.y);
    }
  // p' <= 2^-F, so P' stays below 2^14 while every V scale is at most
  // 2^(14+F); non-negative floats order like their bit patterns
  int w[NV];
#pragma unroll
  for (int u = 0; u < TPW; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int g = 0; g < NG; ++g) w[(u * 4 + i) * NG + g] = __float_as_int(sv[u][i][g]);
  int vbits = 0;
#pragma unroll
  for (int j = 0; j + 1 < NV; j += 2) vbits = __vimax3_s32(vbits, w[j], w[j + 1]);
  if (__any_sync(kFull, !st.fset || vbits > __float_as_int(pow2i(14 + st.F)))) {
    float vm = __int_as_float(vbits);
    vm = fmaxf(vm, __shfl_xor_sync(kFull, vm, 1));
    vm = fmaxf(vm, __shfl_xor_sync(kFull, vm, 2));
    int ex = 0;
    frexpf(vm, &ex);
    int Fn = vm > 0.0f ? ex - 7 : 0;  // vm * 2^-Fn in [64, 128)
    Fn = max(-60, min(60, Fn));
    // F stays 0 until the first non-zero V scale, then only rises
    const int Fnew = st.fset ? max(st.F, Fn) : (vm > 0.0f ? Fn : st.F);
    if (Fnew != st.F) {
      const float f = pow2i(st.F - Fnew);  // exact
      scale_acc(st, f);
      st.l = __fmul2_rn(st.l, make_float2(f, f));
#pragma unroll
      for (int u = 0; u < TPW; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) p[u][i] *= f;
      st.F = Fnew;
    }
    if (vm > 0.0f) st.fset = true;
  }
#pragma unroll
  for (int u = 0; u < TPW; ++u)
#pragma unroll
    for (int i = 0; i < 4; i += 2) st.l = __fadd2_rn(st.l, make_float2(p[u][i], p[u][i + 1]));
}

// P.V on the packed values with P' = p' * s_v split into hi + lo.  Branch-free.
template <int D, int PATH, int FMT, int TPW>
__device__ __forceinline__ void tile_pv(const unsigned char* stg, int r0, int gid,
                                        const int (&rho)[4], const float (&p)[TPW][4],
                                        const float (&sv)[TPW][4][D / 32],
                                        WarpState<D, PATH, FMT>& st) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int NG = C::NG, RB = C::RB, SB = 2 * NG;  // SB: bytes of one of a row's 8 sub-blocks
  const unsigned char* vc = stg + C::VC + r0 * RB;
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    uint32_t vw[4][(NG + 1) / 2];  // sub-block gid of rows rho[0..3] of tile u (group pairs)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const unsigned char* vp = vc + (16 * u + rho[i]) * RB + SB * gid;
      if constexpr (NG == 3) {  // 6 bytes at a 2-byte aligned offset: g0 g1 | g2
        const uint16_t* h = reinterpret_cast<const uint16_t*>(vp);
        vw[i][0] = (uint32_t)h[0] | ((uint32_t)h[1] << 16);
        vw[i][1] = h[2];
      } else if (NG == 4) {
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
    for (int gp = 0; gp < NG; gp += 2) {
      // P' = p' * s_v of rows rho[0..3] for groups gp, gp + 1, split exactly
      // into f16-representable hi + lo (two groups per packed multiply; an odd
      // last group repeats its own scale in the unused half)
      const int g1 = gp + 1 < NG ? gp + 1 : gp;
      float wh[4][2], wl[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = __fmul2_rn(make_float2(p[u][i], p[u][i]),
                                    make_float2(sv[u][i][gp], sv[u][i][g1]));
        const float2 h = make_float2(split_hi(x.x), split_hi(x.y));
        const float2 l = __ffma2_rn(h, make_float2(-1.0f, -1.0f), x);  // exact
        wh[i][0] = h.x;
        wh[i][1] = h.y;
        wl[i][0] = l.x;
        wl[i][1] = l.y;
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int g = gp + e;
        if (g >= NG) break;  // odd NG: the last pair has one group
        const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;
        // codes c = 0..3 of dims 32g + 4gid + c: low halves rows rho0 / rho2,
        // high halves rows rho1 / rho3
        const uint32_t X = prmt(vw[0][g / 2], vw[1][g / 2], sel);
        const uint32_t Y = prmt(vw[2][g / 2], vw[3][g / 2], sel);
        if (PATH == 0) {  // (no int4 launch takes PATH 0; the codebook caches use tile_pv_cb)
          const uint32_t a0 = f16x2(wh[0][e], wh[1][e]), a1 = f16x2(wl[0][e], wl[1][e]);
          const uint32_t a2 = f16x2(wh[2][e], wh[3][e]), a3 = f16x2(wl[2][e], wl[3][e]);
          mma16816(st.acc[4 * g + 0], a0, a1, a2, a3, codes_lo(X), codes_lo(Y));
          mma16816(st.acc[4 * g + 1], a0, a1, a2, a3, codes_hi(X), codes_hi(Y));
          mma16816(st.acc[4 * g + 2], a0, a1, a2, a3, codes_lo(X >> 8), codes_lo(Y >> 8));
          mma16816(st.acc[4 * g + 3], a0, a1, a2, a3, codes_hi(X >> 8), codes_hi(Y >> 8));
        } else if (PATH == 2) {  // B: the weights of head gid, hi part, then lo part
          const uint32_t bh0 = f16x2(wh[0][e], wh[1][e]), bh1 = f16x2(wh[2][e], wh[3][e]);
          const uint32_t bl0 = f16x2(wl[0][e], wl[1][e]), bl1 = f16x2(wl[2][e], wl[3][e]);
          const uint32_t x0 = codes_lo(X), x1 = codes_hi(X), y0 = codes_lo(Y), y1 = codes_hi(Y);
          mma16816(st.acc[2 * g + 0], x0, x1, y0, y1, bh0, bh1);
          mma16816(st.acc[2 * g + 0], x0, x1, y0, y1, bl0, bl1);
          const uint32_t x2 = codes_lo(X >> 8), x3 = codes_hi(X >> 8);
          const uint32_t y2 = codes_lo(Y >> 8), y3 = codes_hi(Y >> 8);
          mma16816(st.acc[2 * g + 1], x2, x3, y2, y3, bh0, bh1);
          mma16816(st.acc[2 * g + 1], x2, x3, y2, y3, bl0, bl1);
        } else {
          const bool lo = gid & 1;  // column gid = (head gid / 2, part gid % 2)
          const uint32_t b0 = f16x2(lo ? wl[0][e] : wh[0][e], lo ? wl[1][e] : wh[1][e]);
          const uint32_t b1 = f16x2(lo ? wl[2][e] : wh[2][e], lo ? wl[3][e] : wh[3][e]);
          mma16816(st.acc[2 * g + 0], codes_lo(X), codes_hi(X), codes_lo(Y), codes_hi(Y), b0, b1);
          mma16816(st.acc[2 * g + 1], codes_lo(X >> 8), codes_hi(X >> 8), codes_lo(Y >> 8),
                   codes_hi(Y >> 8), b0, b1);
        }
      }
    }
  }
}

// Codebook P.V (heads on rows): as tile_pv with the B operand the levels of
// coordinates 32g + 4 gid + e (n-tile e) of the token pairs (rho0, rho1) and
// (rho2, rho3), hi and lo parts from the level-pair table (one lookup per row
// and pair of coordinates), both products in the same accumulator.  Branch-free.
template <int D, int PATH, int FMT, int TPW, bool EXACT>
__device__ __forceinline__ void tile_pv_cb(const unsigned char* stg, int r0, int gid,
                                           const int (&rho)[4], const float (&p)[TPW][4],
                                           const float (&sv)[TPW][4][D / 32],
                                           WarpState<D, PATH, FMT>& st, const unsigned char* lutp) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int NG = C::NG, RB = C::RB, GB = 4 * FMT;  // GB: bytes per group
  constexpr uint32_t KM = (1u << (2 * FMT)) - 1;      // key mask (two indices)
  const unsigned char* vc = stg + C::VC + r0 * RB;
  const int bo = 4 * FMT * gid;  // bit offset of this thread's 4 indices in a group
#pragma unroll
  for (int u = 0; u < TPW; ++u) {
    uint32_t f[4][NG];  // row rho[i]'s indices of dims 32g + 4 gid .. + 3 (4 FMT bits)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const unsigned char* rp = vc + (16 * u + rho[i]) * RB + g * GB;
        if (FMT == 2) {
          f[i][g] = rp[gid];
        } else if (FMT == 4) {
          f[i][g] = reinterpret_cast<const uint16_t*>(rp)[gid];
        } else {
          const uint32_t* w = reinterpret_cast<const uint32_t*>(rp) + (bo >> 5);
          f[i][g] = __funnelshift_r(w[0], w[1], bo & 31);
        }
      }
#pragma unroll
    for (int gp = 0; gp < NG; gp += 2) {
      float wh[4][2], wl[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = __fmul2_rn(make_float2(p[u][i], p[u][i]),
                                    make_float2(sv[u][i][gp], sv[u][i][gp + 1]));
        const float2 h = make_float2(split_hi(x.x), split_hi(x.y));
        const float2 l = __ffma2_rn(h, make_float2(-1.0f, -1.0f), x);  // exact
        wh[i][0] = h.x;
        wh[i][1] = h.y;
        wl[i][0] = l.x;
        wl[i][1] = l.y;
      }
#pragma unroll
      for (int eg = 0; eg < 2; ++eg) {
        const int g = gp + eg;
        const uint32_t a0 = f16x2(wh[0][eg], wh[1][eg]), a1 = f16x2(wl[0][eg], wl[1][eg]);
        const uint32_t a2 = f16x2(wh[2][eg], wh[3][eg]), a3 = f16x2(wl[2][eg], wl[3][eg]);
        // level pairs of dims (4 gid, 4 gid + 1) and (4 gid + 2, 4 gid + 3) of each row,
        // then byte permutes pair the rows: n-tile e takes the half holding dim 4 gid + e
        uint2 lv[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const unsigned char* ep = lutp + (((f[i][g] >> (2 * FMT * m)) & KM) << 3);
            if (EXACT) lv[i][m] = make_uint2(*reinterpret_cast<const uint32_t*>(ep), 0u);
            else lv[i][m] = *reinterpret_cast<const uint2*>(ep);
          }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int m = e >> 1;
          const uint32_t sel = (e & 1) ? 0x7632u : 0x5410u;
          mma16816(st.acc[4 * g + e], a0, a1, a2, a3, prmt(lv[0][m].x, lv[1][m].x, sel),
                   prmt(lv[2][m].x, lv[3][m].x, sel));
          if (!EXACT)
            mma16816(st.acc[4 * g + e], a0, a1, a2, a3, prmt(lv[0][m].y, lv[1][m].y, sel),
                     prmt(lv[2][m].y, lv[3][m].y, sel));
        }
      }
    }
  }
}

// One warp's share of a stage: scores, softmax update and P.V of its TPW tiles
// (rows r0 .. r0 + 16 TPW - 1, of which the first nvalid are real tokens).
template <int D, int PATH, int FMT, int TPW, bool FULL, bool EXACT = false>
__device__ __forceinline__ void stage_tiles(const unsigned char* stg, int skew, int r0, int nvalid, int gid,
                                            int tig, const int (&rho)[4], const int (&krow)[2],
                                            WarpState<D, PATH, FMT>& st,
                                            const unsigned char* lutp) {
  float S[TPW][4], p[TPW][4], sv[TPW][4][D / 32];
  if constexpr (FMT == 0)
    tile_scores<D, PATH, FMT, TPW, FULL>(stg, skew, r0, nvalid, tig, rho, krow, st, S);
  else
    tile_scores_cb<D, PATH, FMT, TPW, FULL, EXACT>(stg, skew, r0, nvalid, tig, rho, krow, st, lutp, S);
  tile_max<D, PATH, FMT, TPW>(tig, S, st);
  load_vscales<D, PATH, FMT, TPW, FULL>(stg, skew, r0, nvalid, rho, sv);
  tile_weights<D, PATH, FMT, TPW>(S, sv, st, p);
  if constexpr (FMT == 0)
    tile_pv<D, PATH, FMT, TPW>(stg, r0, gid, rho, p, sv, st);
  else
    tile_pv_cb<D, PATH, FMT, TPW, EXACT>(stg, r0, gid, rho, p, sv, st, lutp);
}

// End of an item: the warps' (max, sum, acc) per head are merged in shared
// memory and written as the item's split-K partial (max reported as m + F,
// with sum and acc scaled by 2^-F).  If the pipeline gave up, the partial's
// max is NaN, so the decode's output for these heads is NaN.
template <int D, int PATH, int FMT>
__device__ __forceinline__ void finish_item(const DecodeArgs& a, unsigned char* smem,
                                            const WarpState<D, PATH, FMT>& st, int b, int kvh, int c,
                                            bool aborted) {
  using C = Cfg<D, PATH, FMT>;
  constexpr int NH = C::NH, NG = C::NG, NW = C::NW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int G = a.Hq / a.Hkv;
  float* macc = reinterpret_cast<float*>(smem + C::MACC);
  float* mm = reinterpret_cast<float*>(smem + C::MM);
  float* ml = reinterpret_cast<float*>(smem + C::ML);
  float* mw = reinterpret_cast<float*>(smem + C::MW);
  float* mtot = reinterpret_cast<float*>(smem + C::MTOT);

  float l = st.l.x + st.l.y;
  l += __shfl_xor_sync(kFull, l, 1);
  l += __shfl_xor_sync(kFull, l, 2);
  const float m = aborted ? __int_as_float(0x7fc00000) : st.m + (float)st.F;
  const int tid = threadIdx.x;
  if constexpr (PATH == 2) {
    // softmax states first; then each warp adds its accumulator, weighted, into
    // buffer warp % MB, one round of MB warps at a time
    constexpr int MB = C::MB;
    if (tig == 0) {
      mm[warp * NH + gid] = m;
      ml[warp * NH + gid] = l;
    }
    barrier_all<C::THREADS>();
    if (tid < NH) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, mm[w * NH + tid]);
      float L = 0.0f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float wt = exp2f(mm[w * NH + tid] - M);  // NaN if that warp gave up
        mw[w * NH + tid] = wt;
        L = fmaf(wt, ml[w * NH + tid], L);
      }
      mtot[tid] = M;
      mtot[NH + tid] = L;
    }
    barrier_all<C::THREADS>();
    // fragment 2g + pp: rows gid, gid + 8 are dims 32g + 4gid + 2pp (+1),
    // columns 2tig, 2tig + 1 are heads
    const float w0 = mw[warp * NH + 2 * tig], w1 = mw[warp * NH + 2 * tig + 1];
    float* d0 = macc + ((warp % MB) * NH + 2 * tig) * D;
    float* d1 = d0 + D;
    for (int r = 0; r * MB < NW; ++r) {
      if (warp / MB == r) {
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int pp = 0; pp < 2; ++pp) {
            const int dim = 32 * g + 4 * gid + 2 * pp;
            float2 v0 = make_float2(w0 * st.acc[2 * g + pp][0], w0 * st.acc[2 * g + pp][2]);
            float2 v1 = make_float2(w1 * st.acc[2 * g + pp][1], w1 * st.acc[2 * g + pp][3]);
            if (r > 0) {
              const float2 o0 = *reinterpret_cast<const float2*>(d0 + dim);
              const float2 o1 = *reinterpret_cast<const float2*>(d1 + dim);
              v0 = make_float2(v0.x + o0.x, v0.y + o0.y);
              v1 = make_float2(v1.x + o1.x, v1.y + o1.y);
            }
            *reinterpret_cast<float2*>(d0 + dim) = v0;
            *reinterpret_cast<float2*>(d1 + dim) = v1;
          }
      }
      barrier_all<C::THREADS>();
    }
    const int stride = a.plan.part_stride;
    float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) +
                                           a.plan.header_bytes);
    for (int idx = tid; idx < G * D; idx += C::THREADS) {
      const int h = idx / D, i = idx % D;
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < MB; ++w) s += macc[(w * NH + h) * D + i];
      float* dst = part + (((int64_t)b * a.Hq + (int64_t)kvh * G + h) * a.plan.n_chunks + c) * stride;
      dst[i] = s;
      if (i == 0) {
        dst[D] = mtot[h];
        dst[D + 1] = mtot[NH + h];
      }
    }
    return;
  } else if (PATH == 0) {
    if (tig == 0) {
      mm[warp * NH + gid] = m;
      ml[warp * NH + gid] = l;
    }
    float* dst = macc + (warp * NH + gid) * D;
    const float ce = FMT ? st.cexp : 1.0f;  // codebook: the levels' normalisation
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        dst[32 * g + 8 * tig + cc] = (st.acc[4 * g + cc][0] + st.acc[4 * g + cc][2]) * ce;
        dst[32 * g + 8 * tig + 4 + cc] = (st.acc[4 * g + cc][1] + st.acc[4 * g + cc][3]) * ce;
      }
  } else {
    if (tig == 0 && (gid & 1) == 0) {
      mm[warp * NH + (gid >> 1)] = m;
      ml[warp * NH + (gid >> 1)] = l;
    }
    float* dst = macc + (warp * NH + tig) * D;
#pragma unroll
    for (int g = 0; g < NG; ++g)
#pragma unroll
      for (int pp = 0; pp < 2; ++pp) {
        const int dim = 32 * g + 4 * gid + 2 * pp;
        dst[dim] = st.acc[2 * g + pp][0] + st.acc[2 * g + pp][1];
        dst[dim + 1] = st.acc[2 * g + pp][2] + st.acc[2 * g + pp][3];
      }
  }
  barrier_all<C::THREADS>();
  if (tid < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mm[w * NH + tid]);
    float L = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float wt = exp2f(mm[w * NH + tid] - M);  // NaN if that warp gave up
      mw[w * NH + tid] = wt;
      L = fmaf(wt, ml[w * NH + tid], L);
    }
    mtot[tid] = M;
    mtot[NH + tid] = L;
  }
  barrier_all<C::THREADS>();
  const int stride = a.plan.part_stride;
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) +
                                         a.plan.header_bytes);
  for (int idx = tid; idx < G * D; idx += C::THREADS) {
    const int h = idx / D, i = idx % D;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) s = fmaf(mw[w * NH + h], macc[(w * NH + h) * D + i], s);
    float* dst = part + (((int64_t)b * a.Hq + (int64_t)kvh * G + h) * a.plan.n_chunks + c) * stride;
    dst[i] = s;
    if (i == 0) {
      dst[D] = mtot[h];
      dst[D + 1] = mtot[NH + h];
    }
  }
}

template <int D, int PATH, int FMT>
__global__ void __launch_bounds__(Cfg<D, PATH, FMT>::THREADS, 1) decode_mma_kernel(DecodeArgs a) {
  using C = Cfg<D, PATH, FMT>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR);
  int* cnt = reinterpret_cast<int*>(smem + C::CNT);
  int* cur = reinterpret_cast<int*>(smem + C::CUR);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::ABORT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(full + s, 1);
      cnt[s] = 0;
    }
    *abort = 0;
    cur[0] = (int)blockIdx.x - (int)gridDim.x;  // before this CTA's first item
    cur[1] = cur[2] = cur[3] = cur[4] = cur[5] = 0;
    cur[8] = cur[9] = cur[10] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the merge kernel may be scheduled now; it waits for this grid's writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // The item list: pfx[b + 1] = Hkv * (chunks of sequence b), then an
  // inclusive scan by warp 0.
  // (Built only when some sequence has fewer chunks than the plan; otherwise
  // the list is the plain enumeration and no scan is needed.)
  int* pfx = reinterpret_cast<int*>(smem + C::PFX);
  bool shorter = false;
  if (a.B <= kMaxListB) {
    for (int b = threadIdx.x; b < a.B; b += C::THREADS) {
      const int T = clamp_ctx_mma(a.ctx_lens[b], a.max_ctx);
      const int nc = (T + a.plan.chunk - 1) / a.plan.chunk;
      pfx[b + 1] = a.Hkv * nc;
      shorter |= nc < a.plan.n_chunks;
    }
    if (threadIdx.x == 0) pfx[0] = 0;
  }
  if (!__syncthreads_or(shorter)) pfx = nullptr;
  if (pfx != nullptr) {
    if (warp == 0) {
      int carry = 0;
      for (int base = 1; base <= a.B; base += 32) {
        const int i = base + lane;
        int v = i <= a.B ? pfx[i] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, v, o);
          if (lane >= o) v += y;
        }
        if (i <= a.B) pfx[i] = v + carry;
        carry += __shfl_sync(kFull, v, 31);
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    cur[6] = pfx != nullptr ? pfx[a.B] : a.B * a.Hkv * a.plan.n_chunks;
    cur[7] = pfx != nullptr;
  }
  // Codebook: the level-pair table, the levels normalised by 2^-e so that the
  // largest magnitude lies in [0.5, 1) (exact; 2^e is put back on the scores
  // and the output): entry i0 | i1 << FMT = (C[i0], C[i1]) as f16x2 hi parts
  // (round to nearest) and f16x2 lo parts (the remainders, rounded).
  float cexp = 1.0f;
  bool exact = false;  // every normalised level is an f16: the lo parts are zero
  if constexpr (FMT != 0) {
    constexpr int L = 1 << FMT;
    float lmax = 0.0f;
    for (int i = 0; i < L; ++i) lmax = fmaxf(lmax, fabsf(a.levels[i]));
    int e = 0;
    if (lmax > 0.0f) frexpf(lmax, &e);
    cexp = ldexpf(1.0f, e);
    exact = true;
    for (int i = 0; i < L; ++i) {
      const float c = ldexpf(a.levels[i], -e);
      exact = exact && __half2float(__float2half_rn(c)) == c;
    }
    uint2* lut = reinterpret_cast<uint2*>(smem + C::LUT);
    for (int key = threadIdx.x; key < L * L; key += C::THREADS) {
      const float c0 = ldexpf(a.levels[key & (L - 1)], -e), c1 = ldexpf(a.levels[key >> FMT], -e);
      const __half h0 = __float2half_rn(c0), h1 = __float2half_rn(c1);
      const __half l0 = __float2half_rn(c0 - __half2float(h0));
      const __half l1 = __float2half_rn(c1 - __half2float(h1));
      lut[key] = make_uint2((uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16),
                            (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16));
    }
  }
  const unsigned char* lutp = smem + C::LUT;
  __syncthreads();

  // Fused append: for every (sequence, kv head) whose last chunk is one of this
  // CTA's items, warps 4 and 5 quantize that kv head's new K and V token into
  // row T - 1 (T the clamped context length) while warps 0 .. 3 prepare the
  // first query.  Only that chunk reads the row; the proxy fence orders these
  // generic writes before the bulk copies, which the last warp issues only
  // after named barrier 2 (both warps arrive here exactly once).
  static_assert(C::NW >= 8, "the fused append uses warps 4, 5 and the last");
  if (a.k_new != nullptr && (warp == 4 || warp == 5)) {
    const bool isv = warp == 5;
    const int eb = a.kv_bf16 ? 2 : 4;
    for (int it = blockIdx.x; it < cur[6]; it += gridDim.x) {
      int b, kvh, c, t0, t1;
      if (!item_range(a, pfx, it, b, kvh, c, t0, t1)) continue;
      if (t1 != clamp_ctx_mma(a.ctx_lens[b], a.max_ctx)) continue;  // not the last chunk
      const int64_t bh = (int64_t)b * a.Hkv + kvh;
      const int64_t row = bh * a.capacity + (t1 - 1);
      if (a.inputs_pending) asm volatile("griddepcontrol.wait;" ::: "memory");  // k_new, v_new
      const unsigned char* src = static_cast<const unsigned char*>(isv ? a.v_new : a.k_new) + bh * D * eb;
      uint8_t* prow = const_cast<uint8_t*>(isv ? a.v_packed : a.k_packed) + row * C::RB;
      float* srow = const_cast<float*>(isv ? a.v_scales : a.k_scales) + row * (D / 32);
      if constexpr (FMT == 0) {
        if constexpr (D == 128 || D == 256)  // other widths are SRFT caches, never fused here
          quantize_vector_warp<D>(src, a.kv_bf16, a.signs, prow, srow, lane);
      } else {
        cb_quantize_vector_warp<D, FMT>(src, a.kv_bf16, a.signs, a.levels, prow, srow, lane,
                                        a.cb_uniform != 0);
      }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    asm volatile("bar.arrive 2, 96;" ::: "memory");
  }

  const int gid = lane >> 2, tig = lane & 3;
  const int rho[4] = {slot_row(2 * tig), slot_row(2 * tig + 1), 8 + slot_row(2 * tig),
                      8 + slot_row(2 * tig + 1)};
  const int krow[2] = {slot_row(gid), 8 + slot_row(gid)};
  WarpState<D, PATH, FMT> st;
  st.cexp = cexp;
  uint32_t sc = 0;  // stages consumed so far
  for (int it = blockIdx.x; it < cur[6]; it += gridDim.x) {
    int b, kvh, c, t0, t1;
    if (!item_range(a, cur[7] ? reinterpret_cast<const int*>(smem + C::PFX) : nullptr, it, b, kvh,
                    c, t0, t1))
      continue;
    if (threadIdx.x == 0 && kvh == 0 && c == 0) {
      const int raw = a.ctx_lens[b];
      static_cast<int32_t*>(a.workspace)[b] = (raw < 1 || raw > a.max_ctx) ? 1 : 0;
    }
    prep_query<D, PATH, FMT>(a, b, kvh, smem, st, sc == 0, cur, full);
#pragma unroll
    for (int j = 0; j < C::NACC; ++j)
#pragma unroll
      for (int r = 0; r < 4; ++r) st.acc[j][r] = 0.0f;
    st.m = -INFINITY;
    st.l = make_float2(0.0f, 0.0f);
    st.F = 0;
    st.fset = false;
    const int nst = (t1 - t0 + C::ST - 1) / C::ST;
    const int r0 = 16 * C::TPW * warp;
    for (int k = 0; k < nst; ++k, ++sc) {
      const int slot = sc % C::NS;
      const unsigned char* stg = smem + slot * C::STAGE;
      mbar_wait(full + slot, (sc / C::NS) & 1, abort);
      const int skew = C::SPAD ? reinterpret_cast<const int*>(smem + C::SKEW)[slot] : 0;
      const int nv = min(C::ST, t1 - t0 - k * C::ST) - r0;  // real rows from r0 on
      if constexpr (FMT != 0) {
        if (exact) {
          if (nv >= 16 * C::TPW)
            stage_tiles<D, PATH, FMT, C::TPW, true, true>(stg, skew, r0, nv, gid, tig, rho, krow, st, lutp);
          else if (nv > 0)
            stage_tiles<D, PATH, FMT, C::TPW, false, true>(stg, skew, r0, nv, gid, tig, rho, krow, st, lutp);
        } else {
          if (nv >= 16 * C::TPW)
            stage_tiles<D, PATH, FMT, C::TPW, true>(stg, skew, r0, nv, gid, tig, rho, krow, st, lutp);
          else if (nv > 0)
            stage_tiles<D, PATH, FMT, C::TPW, false>(stg, skew, r0, nv, gid, tig, rho, krow, st, lutp);
        }
      } else {
        if (nv >= 16 * C::TPW)
          stage_tiles<D, PATH, FMT, C::TPW, true>(stg, skew, r0, nv, gid, tig, rho, krow, st, lutp);
        else if (nv > 0)
          stage_tiles<D, PATH, FMT, C::TPW, false>(stg, skew, r0, nv, gid, tig, rho, krow, st, lutp);
      }
      __syncwarp();
      if (lane == 0) {
        // first the refills queued by earlier stages, then this warp leaves the
        // stage; the last warp out only queues the stage's refill
        service_refills<D, PATH, FMT>(a, smem, cur, full, abort);
        __threadfence_block();
        if (atomicAdd(cnt + slot, 1) == C::NW - 1) {
          cnt[slot] = 0;
          __threadfence_block();
          atomicAdd(cur + 8, 1);
        }
      }
    }
    finish_item<D, PATH, FMT>(a, smem, st, b, kvh, c, *abort != 0);
  }
  if (threadIdx.x == 0 && *abort) {  // copies still in flight must land before exit
    const uint32_t issued = (uint32_t)cur[5];
    for (uint32_t s = issued > (uint32_t)C::NS ? issued - C::NS : 0; s < issued; ++s)
      mbar_drain(full + s % C::NS, (s / C::NS) & 1);
  }
}

template <int D, int PATH, int FMT>
cudaError_t launch_mma(const DecodeArgs& a, cudaStream_t stream) {
  using C = Cfg<D, PATH, FMT>;
  static SmemLimitSet smem_set;
  const cudaError_t e = ensure_smem_limit(decode_mma_kernel<D, PATH, FMT>, C::BYTES, smem_set);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = a.B * a.Hkv * a.plan.n_chunks;
  const int grid = n_items < sms ? n_items : sms;
  // overlap the preceding grid that rotates the queries or gathers the step's
  // inputs: programmatic dependent launch (the kernel waits where it reads them)
  if ((a.q_rot != nullptr && a.q_rot_overlap) || a.inputs_pending) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_mma_kernel<D, PATH, FMT>, a);
  }
  decode_mma_kernel<D, PATH, FMT><<<grid, C::THREADS, C::BYTES, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool decode_mma_supported(int d, int G) {
  return (d == 128 && G >= 1 && G <= 8) || ((d == 96 || d == 256) && G >= 1 && G <= 4);
}

bool decode_mma_cb_supported(int d, int G) { return d == 128 && G >= 5 && G <= 8; }

int decode_stage_tokens(int d, int G) {
  if (!decode_mma_supported(d, G)) return 128;
  return d == 128 ? (G >= 5 ? Cfg<128, 2, 0>::ST : Cfg<128, 1, 0>::ST)
                   : d == 96 ? Cfg<96, 1, 0>::ST : Cfg<256, 1, 0>::ST;
}

cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  if (a.cb_bits != 0) {
    if (!decode_mma_cb_supported(a.d, G)) return cudaErrorNotSupported;
    switch (a.cb_bits) {
      case 2: return launch_mma<128, 0, 2>(a, stream);
      case 3: return launch_mma<128, 0, 3>(a, stream);
      case 4: return launch_mma<128, 0, 4>(a, stream);
      default: return cudaErrorNotSupported;
    }
  }
  if (a.d == 128 && G >= 5 && G <= 8) return launch_mma<128, 2, 0>(a, stream);
  if (a.d == 128 && G >= 1 && G <= 4) return launch_mma<128, 1, 0>(a, stream);
  if (a.d == 256 && G >= 1 && G <= 4) return launch_mma<256, 1, 0>(a, stream);
  if (a.d == 96 && G >= 1 && G <= 4) return launch_mma<96, 1, 0>(a, stream);
  return cudaErrorNotSupported;
}

}  // namespace tq
