// decode_tc.cu -- split-K decode attention on the packed int4 cache with both
// contractions on the fifth-generation tensor cores (tcgen05.mma, f16 x f16 ->
// f32, accumulators in tensor memory).  Head width 128, up to 8 query heads
// per kv head, the Hadamard-rotated (or unrotated) int4 cache, and the SRFT
// variant's cache (its queries arrive already rotated).
//
// What it computes is the decode of decode_mma.cu: attention directly on the
// packed codes ("fused sdpa_int4", Open-TQ-Metal abstract) with no dequantized
// K/V matrix (forum summary, "eliminating intermediate matrices"), an online
// softmax in fp32 (section "numerical stability") and one split-K partial
// (unnormalized acc[d], max m in log2 units, sum l) per (sequence, query head,
// chunk) for merge.cu.
//
// Work: persistent CTAs (one per SM) walk (sequence, kv head, chunk) items in
// 128-token tiles.  Warp roles:
//   0..3   K/V warps.  Warp q unpacks K codes of tile tokens 32q..32q+31 into
//          tensor memory A_K (token = lane: the A operand of the score MMA),
//          and the V codes of 32 of the 128 dims into A_V (dim = lane: the A
//          operand of the P.V MMA, read from a 64-byte-swizzled TMA copy with
//          transposing ldmatrix, so no transposition costs instructions).  They
//          fold the P.V accumulator into registers when the softmax reference
//          changes, and write the item's partial.
//   4..11  softmax warps.  Warp (q, hh) takes the scores of tokens 32q..+31
//          for heads 4hh..4hh+3 from tensor memory, keeps the softmax state,
//          and writes P' = p * s_v (split into f16 hi + lo) as the B operand
//          of the P.V MMA into shared memory.
//   12     producer: bulk copies of K codes and scales, TMA of V codes.
//   13     MMA issuer (one thread).
//   14     query preparation (rotation, scaling, B operand of the score MMA)
//          and the fused append of the step's new token.
//
// Exactness on the tensor cores:
//  - scores: D = A_K x B_Q with A_K the codes as exact f16 subnormals
//    (c + 8) 2^-24 (times 16 for codes in bits 4..7, whose query entries are
//    divided by 16) and B_Q the query split into f16 hi and lo parts (22 bits;
//    each head normalised by a power of two into [2^13, 2^14)).  A third MMA
//    per group adds -8 2^-24 sum_g q from a constant A block, so each group's
//    accumulator holds 2^-24 sum_j c_j q_j; S = sum_g s_k[g] (D_hi + D_lo).
//  - P.V: O = A_V x B_P with A_V the codes as exact f16 (c, or 16c for codes
//    in bits 4..7, whose output lanes are divided by 16), B_P the weights
//    P' = 2^(S - m) s_v 2^-F split into hi (top 11 bits) + lo.  The N columns
//    are (group, head, part); a dim's output is its group's columns.
//  - Lazy rescaling: the reference max m per head only moves when a tile's
//    maximum exceeds it by more than kTau (2^8), so p <= 2^8; F keeps
//    P' < 2^15 (f16 range).  When either moves, the K/V warps fold the
//    accumulator into registers with the exact factor 2^(dm + dF) before the
//    tile's P.V starts a fresh accumulator.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include "quantize_vector.cuh"
#include "tc_ptx.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kTile = 128;   // tokens per tile
constexpr int kNS = 5;       // pipeline stages (one tile each)
constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kProducerWarp = 12, kScoreMmaWarp = 13, kQueryWarp = 14, kPvMmaWarp = 15;
constexpr float kTau = 8.0f;  // lazy-rescale threshold (log2 units)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxList = 1024;  // batches up to this size use the list of non-empty items

// tensor-memory columns
constexpr uint32_t kColAK = 0, kColDS = 128, kColAV = 256, kColO = 384;
constexpr uint32_t kTmemCols = 512;

// shared memory layout (bytes)
struct L {
  static constexpr int STAGE = 20480;  // K codes 8K, V codes 8K, K scales 2K, V scales 2K
  static constexpr int KC = 0, VC = 8192, KS = 16384, VS = 18432;
  static constexpr int BP = kNS * STAGE;            // 2 x 16384: P.V B operand
  static constexpr int BQ = BP + 2 * 16384;         // 2 x 4096: score B operand
  static constexpr int BQ_SIZE = 4096;
  static constexpr int QS = BQ + 2 * BQ_SIZE;       // float [8][128] query scratch
  static constexpr int CORR = QS + 4 * 8 * kD;      // float [2][4][8] -8 2^-24 sum_g q
  static constexpr int BAR = CORR + 4 * 64;         // mbarriers
  static constexpr int NBAR = 2 * kNS + 32;
  static constexpr int XCHG = BAR + 8 * NBAR;       // [2][8 warps] x {int event; float max[4], vmax; pad}
  static constexpr int LSUM = XCHG + 4 * 128;       // float [8 warps][4]
  static constexpr int EVT = LSUM + 4 * 32;         // [2] x {int flag; pad}
  static constexpr int EVT_SIZE = 16;
  static constexpr int CEXP = EVT + 2 * EVT_SIZE;   // float [2][8]
  static constexpr int MISC = CEXP + 4 * 16;        // tmem base, abort
  static constexpr int PFX = MISC + 64;             // int [kMaxList + 1]
  static constexpr int BYTES = PFX + 4 * (kMaxList + 1);
};
static_assert(L::BYTES + 1024 <= 227 * 1024, "shared memory");
static_assert(L::STAGE % 1024 == 0 && L::VC % 1024 == 0 && L::BP % 1024 == 0, "alignment");

// mbarrier indices
enum Bar : int {
  kFull = 0,                  // [kNS] stage landed (producer + tx)
  kEmpty = kNS,               // [kNS] stage consumed (4 K/V + 8 softmax warps)
  kAKFull = 2 * kNS,          // [2] A_K written (4 warps)
  kAKEmpty = kAKFull + 2,     // [2] score MMAs read A_K (commit)
  kDSFull = kAKEmpty + 2,     // [2] scores in tensor memory (commit)
  kDSEmpty = kDSFull + 2,     // [2] scores read (8 warps)
  kAVFull = kDSEmpty + 2,     // [2] A_V written (4 warps)
  kAVEmpty = kAVFull + 2,     // [2] P.V MMAs of that buffer done (commit): frees A_V and B_P
  kBPFull = kAVEmpty + 2,     // [2] B_P written (8 warps)
  kQFull = kBPFull + 2,       // [2] query operand ready (query warp)
  kQEmpty = kQFull + 2,       // [2] the item's score MMAs done (commit), factors read (8 warps)
  kAppDone = kQEmpty + 2,     // fused append written (query warp)
  kMmaDone = kAppDone + 1,    // every MMA complete (commit)
  kBarCount = kMmaDone + 1
};
static_assert(kBarCount <= L::NBAR, "barrier slots");

struct Evt {
  int flag;  // the softmax folded the accumulator before this tile: its P.V starts afresh
};

__device__ __forceinline__ int clamp_ctx(int T, int max_ctx) {
  return T < 1 ? 1 : (T > max_ctx ? max_ctx : T);
}

// Item it -> (sequence b, kv head, chunk c) and its token range [t0, t1); as
// in the tensor-core decode: with the list (pfx) only chunks holding tokens.
__device__ __forceinline__ bool item_range(const DecodeArgs& a, const int* pfx, int it, int& b,
                                           int& kvh, int& c, int& t0, int& t1) {
  if (pfx != nullptr) {
    int lo = 0, hi = a.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pfx[mid] <= it) lo = mid;
      else hi = mid;
    }
    b = lo;
    const int T = clamp_ctx(a.ctx_lens[b], a.max_ctx);
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
  const int T = clamp_ctx(a.ctx_lens[b], a.max_ctx);
  t0 = c * a.plan.chunk;
  t1 = min(T, t0 + a.plan.chunk);
  return t0 < t1;
}

// This CTA's items in order; every role walks the same sequence.
struct Items {
  const DecodeArgs* a;
  const int* pfx;
  int n_items;
  int it;
  int b, kvh, c, t0, t1;
  __device__ Items(const DecodeArgs& args, const int* p, int n) : a(&args), pfx(p), n_items(n) {
    it = (int)blockIdx.x - (int)gridDim.x;
  }
  __device__ bool next() {
    for (it += gridDim.x; it < n_items; it += gridDim.x)
      if (item_range(*a, pfx, it, b, kvh, c, t0, t1)) return true;
    return false;
  }
  __device__ int tiles() const { return (t1 - t0 + kTile - 1) / kTile; }
};

__device__ __forceinline__ uint32_t lane_base(int quarter) { return (uint32_t)(32 * quarter) << 16; }

// mbar_wait by every lane of a warp, reconverged afterwards: the warps that run
// .sync.aligned tensor-memory instructions must stay converged, also when a
// wait gives up (then every later wait returns at once and the work proceeds
// on whatever the buffers hold; the partials report NaN).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  __syncwarp();
  return __all_sync(0xffffffffu, ok);
}

// Registers written by tcgen05.ld are valid only after tcgen05.wait::ld; the
// empty volatile statements after the wait make every later use depend on it.
__device__ __forceinline__ void tie8(uint32_t (&r)[8]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
               "+r"(r[7]));
}

// ------------------------------------------------------------ K/V warps

// K codes of tile tokens 32q..32q+31 -> A_K (f16 subnormal offset codes).
// Thread t = 4r + a reads the 16-byte chunk a (sub-blocks 2a, 2a+1: in-group
// coordinates 8a..8a+7 of every group) of rows 32q + 16hf + r + 8m'.  Per
// group, one byte permute gathers that group's 8 coordinates; value v = 0..3
// is the f16x2 (coordinate 8a + v, coordinate 8a + 4 + v) and goes to column
// 16g + 8(v/2) + 2a + (v%2) of the token's lane.
__device__ __forceinline__ void unpack_k(const unsigned char* stg, uint32_t tbase, int q, int lane) {
  const int r = lane >> 2, a = lane & 3;
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    uint4 w[2];
#pragma unroll
    for (int mp = 0; mp < 2; ++mp)
      w[mp] = *reinterpret_cast<const uint4*>(stg + L::KC + (32 * q + 16 * hf + r + 8 * mp) * 64 + 16 * a);
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {  // groups 2gp, 2gp+1: one 16x256b.x4 store (4 chunks)
      uint32_t reg[16];
#pragma unroll
      for (int ge = 0; ge < 2; ++ge) {
        const int g = 2 * gp + ge;
#pragma unroll
        for (int mp = 0; mp < 2; ++mp) {
          const uint32_t lo = g < 2 ? w[mp].x : w[mp].y, hi = g < 2 ? w[mp].z : w[mp].w;
          const uint32_t x = prmt(lo, hi, (g & 1) ? 0x7632u : 0x5410u);
          const uint32_t xs = x >> 8;
          const uint32_t y0 = and_xor(x, 0x000F000Fu, 0x00080008u);
          const uint32_t y1 = and_xor(x, 0x00F000F0u, 0x00800080u);
          const uint32_t y2 = and_xor(xs, 0x000F000Fu, 0x00080008u);
          const uint32_t y3 = and_xor(xs, 0x00F000F0u, 0x00800080u);
          // chunk 2ge + v/2 of this store; reg 2mp + v%2
          reg[4 * (2 * ge + 0) + 2 * mp + 0] = y0;
          reg[4 * (2 * ge + 0) + 2 * mp + 1] = y1;
          reg[4 * (2 * ge + 1) + 2 * mp + 0] = y2;
          reg[4 * (2 * ge + 1) + 2 * mp + 1] = y3;
        }
      }
      tst_16x256b_x4(tbase + lane_base(q) + ((uint32_t)(16 * hf) << 16) + 32 * gp, reg);
    }
  }
}

// V codes -> A_V for this warp's 32 dims (lane l: halfword column l % 8 of the
// rows' 16-byte chunk q, coordinate l / 8 of that halfword), all 128 tokens.
// ldmatrix.trans over the swizzled rows gives thread t = 4r + a the halfword
// r of tokens 8b + 2a and 8b + 2a + 1 as one register; codes become exact f16
// (c, or 16c for the nibbles in bits 4..7).  Column 8cb + 2a + p holds tokens
// 16cb + 8p + 2a + {0, 1}.
__device__ __forceinline__ void unpack_v(const unsigned char* stg, uint32_t tbase, int q, int lane) {
  const uint32_t vbase = smem_u32(stg + L::VC);
#pragma unroll
  for (int ht = 0; ht < 2; ++ht) {
    uint32_t rr[8];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int rho = 32 * (2 * ht + e) + lane;  // row this lane addresses
      const uint32_t addr = vbase + rho * 64 + 16 * (q ^ ((rho >> 1) & 3));
      ldsm_x4_trans(addr, rr[4 * e + 0], rr[4 * e + 1], rr[4 * e + 2], rr[4 * e + 3]);
    }
    uint32_t lo[16], hi[16];  // coordinates m = 0, 1 (lanes +0) and m = 2, 3 (lanes +16)
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // block b = 8ht + i: chunk cc = i / 2, p = i % 2
      const uint32_t x = rr[i], xs = x >> 8;
      const int cc = i >> 1, p = i & 1;
      lo[4 * cc + 0 + p] = hsub2(and_xor(x, 0x000F000Fu, 0x64086408u), 0x64086408u);
      lo[4 * cc + 2 + p] = hsub2(and_xor(x, 0x00F000F0u, 0x64806480u), 0x64806480u);
      hi[4 * cc + 0 + p] = hsub2(and_xor(xs, 0x000F000Fu, 0x64086408u), 0x64086408u);
      hi[4 * cc + 2 + p] = hsub2(and_xor(xs, 0x00F000F0u, 0x64806480u), 0x64806480u);
    }
    tst_16x256b_x4(tbase + lane_base(q) + 32 * ht, lo);
    tst_16x256b_x4(tbase + lane_base(q) + (16u << 16) + 32 * ht, hi);
  }
}

// acc[h] = (acc[h] + O[dim, head 4hh + h]) * alpha[h] for this lane's dim:
// the accumulator columns 16g + 8hh + 4 part + h of the lane's group g.
__device__ __forceinline__ void fold_half(uint32_t tbase, int q, int hh, int lane, float (&acc)[4],
                                          const float (&alpha)[4]) {
  const int my_g = lane & 3;
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = 0u;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t r[8];
    tld_x8(tbase + lane_base(q) + kColO + 16 * g + 8 * hh, r);
    wait_ld();
    tie8(r);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = my_g == g ? r[i] : o[i];
  }
#pragma unroll
  for (int h = 0; h < 4; ++h)
    acc[h] = (acc[h] + (__uint_as_float(o[h]) + __uint_as_float(o[4 + h]))) * alpha[h];
}

// ------------------------------------------------------------ query warp

// Query of item (b, kvh) -> B_Q (score B operand), the offset corrections
// -8 2^-24 sum_g q per (group, head), and cexp (per-head factor from the MMA's
// sum to log2-unit scores).
__device__ void prep_query(const DecodeArgs& a, int b, int kvh, unsigned char* smem, int qb, int lane) {
  const int G = a.Hq / a.Hkv;
  float* qs = reinterpret_cast<float*>(smem + L::QS);
  float* cexp = reinterpret_cast<float*>(smem + L::CEXP) + 8 * qb;
  float* corr = reinterpret_cast<float*>(smem + L::CORR) + 32 * qb;
  for (int h = 0; h < 8; ++h) {
    float x[4];
    if (h < G) {
      const int64_t base = ((int64_t)b * a.Hq + (int64_t)kvh * G + h) * kD + 4 * lane;
      if (a.q_rot != nullptr) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const float4 v = *reinterpret_cast<const float4*>(a.q_rot + base);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
      } else {
        if (a.inputs_pending) asm volatile("griddepcontrol.wait;" ::: "memory");
        if (a.q_bf16) {
          const uint2 v = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.q) + base);
          x[0] = __uint_as_float(v.x << 16);
          x[1] = __uint_as_float(v.x & 0xFFFF0000u);
          x[2] = __uint_as_float(v.y << 16);
          x[3] = __uint_as_float(v.y & 0xFFFF0000u);
        } else {
          const float4 v = *reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + base);
          x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
        }
        rotate_vector_warp<kD>(x, a.signs, lane);  // H (signs . q) / sqrt(d), or nothing
      }
      float amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[e] *= a.attn_scale * kLog2e;
        amax = fmaxf(amax, fabsf(x[e]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      int ex = 0;
      frexpf(amax, &ex);
      int sh = amax > 0.0f ? 14 - ex : 0;  // amax 2^sh in [2^13, 2^14)
      sh = max(-100, min(100, sh));
#pragma unroll
      for (int e = 0; e < 4; ++e) qs[h * kD + 4 * lane + e] = x[e] * pow2i(sh);
      if (lane == 0) cexp[h] = pow2i(24 - sh);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) qs[h * kD + 4 * lane + e] = 0.0f;
      if (lane == 0) cexp[h] = 1.0f;
    }
  }
  __syncwarp();
  {  // corrections: lane = (group, head)
    const int g = lane >> 3, h = lane & 7;
    float s = 0.0f;
    for (int j = 0; j < 32; ++j) s += qs[h * kD + 32 * g + j];
    corr[lane] = -8.0f * 5.9604644775390625e-08f * s;  // -8 2^-24 sum
  }
  __syncwarp();
  __half* bq = reinterpret_cast<__half*>(smem + L::BQ + qb * L::BQ_SIZE);
  // B_Q[g][j]: element (k, n), k = 0..15 of K-half j, n = 0..15, at
  // (n/8) 256 + (k/8) 128 + (n%8) 16 + (k%8) 2 bytes.  K element kk = 16j + k
  // of group g meets coordinate 8a + v + 4h with cc = kk/2, h = kk%2,
  // a = (cc%8)/2, v = 2(cc/8) + cc%2 (the K unpack's column order); N column n
  // is head 4(n/8) + n%4, part (n/4)%2.
  for (int e = lane; e < 4 * 2 * 256; e += 32) {
    const int g = e >> 9, j = (e >> 8) & 1, n = (e >> 4) & 15, k = e & 15;
    const int kk = 16 * j + k, cc = kk >> 1, hbit = kk & 1, wc = cc & 7;
    const int v = 2 * (cc >> 3) + (wc & 1);
    const int coord = 8 * (wc >> 1) + v + 4 * hbit;
    const int head = 4 * (n >> 3) + (n & 3), part = (n >> 2) & 1;
    const float val = qs[head * kD + 32 * g + coord] * ((v & 1) ? 0.0625f : 1.0f);  // exact
    const __half hv = __float2half_rn(val);
    const __half out = part ? __float2half_rn(val - __half2float(hv)) : hv;
    bq[(g * 1024 + j * 512 + (n >> 3) * 256 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) / 2] = out;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // operands for the tensor cores
  __syncwarp();
}

// ------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_v) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the 64-byte TMA swizzle is a function of absolute shared-memory address
  // bits, so the stages start on a 1024-byte boundary (1 KB extra requested)
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
  int* misc = reinterpret_cast<int*>(smem + L::MISC);
  volatile int* abort = misc + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar + kFull + s, 1);
      mbar_init(bar + kEmpty + s, 12);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + kAKFull + i, 4);
      mbar_init(bar + kAKEmpty + i, 1);
      mbar_init(bar + kDSFull + i, 1);
      mbar_init(bar + kDSEmpty + i, 8);
      mbar_init(bar + kAVFull + i, 4);
      mbar_init(bar + kAVEmpty + i, 1);
      mbar_init(bar + kBPFull + i, 8);
      mbar_init(bar + kQFull + i, 1);
      mbar_init(bar + kQEmpty + i, 9);  // the item's score MMAs (commit) + 8 softmax warps
    }
    mbar_init(bar + kAppDone, 1);
    mbar_init(bar + kMmaDone, 2);  // both MMA issuers
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp == 0) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), kTmemCols);
    tmem_relinquish();
  }
  // the item list (as in the other decode kernels)
  int* pfx = reinterpret_cast<int*>(smem + L::PFX);
  bool shorter = false;
  if (a.B <= kMaxList) {
    for (int b = threadIdx.x; b < a.B; b += kThreads) {
      const int T = clamp_ctx(a.ctx_lens[b], a.max_ctx);
      const int nc = (T + a.plan.chunk - 1) / a.plan.chunk;
      pfx[b + 1] = a.Hkv * nc;
      shorter |= nc < a.plan.n_chunks;
    }
    if (threadIdx.x == 0) pfx[0] = 0;
  }
  fence_before();
  if (!__syncthreads_or(shorter)) pfx = nullptr;
  fence_after();
  if (pfx != nullptr) {
    if (warp == 0) {
      int carry = 0;
      for (int base = 1; base <= a.B; base += 32) {
        const int i = base + lane;
        int v = i <= a.B ? pfx[i] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += y;
        }
        if (i <= a.B) pfx[i] = v + carry;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
    }
    __syncthreads();
  }
  const int n_items = pfx != nullptr ? pfx[a.B] : a.B * a.Hkv * a.plan.n_chunks;
  const uint32_t tbase = static_cast<uint32_t>(misc[0]);


  const int G = a.Hq / a.Hkv;
  Items items(a, pfx, n_items);

  if (warp < 4) {
    // ================================================== K/V warps
    const int q = warp;
    uint32_t kt = 0;
    while (items.next()) {
      const int nt = items.tiles();
      if (q == 0 && lane == 0 && items.kvh == 0 && items.c == 0) {
        const int raw = a.ctx_lens[items.b];
        static_cast<int32_t*>(a.workspace)[items.b] = (raw < 1 || raw > a.max_ctx) ? 1 : 0;
      }
      for (int j = 0; j < nt; ++j, ++kt) {
        const int s = kt % kNS, bb = kt & 1;
        const uint32_t n = kt >> 1;
        const unsigned char* stg = smem + s * L::STAGE;
        warp_wait(bar + kFull + s, (kt / kNS) & 1, abort);
        if (kt >= 2) warp_wait(bar + kAKEmpty + bb, (n - 1) & 1, abort);  // scores of tile kt-2 done
        fence_after();
        unpack_k(stg, tbase + kColAK + 64 * bb, q, lane);
        wait_st();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + kAKFull + bb);
        if (kt >= 2) warp_wait(bar + kAVEmpty + bb, (n - 1) & 1, abort);  // P.V of tile kt-2 done
        fence_after();
        unpack_v(stg, tbase + kColAV + 64 * bb, q, lane);
        wait_st();
        fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar + kAVFull + bb);
          mbar_arrive(bar + kEmpty + s);
        }
      }
    }
  } else if (warp < 12) {
    // ================================================== softmax warps
    const int q = warp & 3, hh = (warp - 4) >> 2, sw = warp - 4;  // sw = 4 hh + q
    const int tau = 32 * q + lane;  // tile token of this thread (= its A_K lane)
    const int kk = 16 * (tau >> 4) + 4 * ((tau & 7) >> 1) + 2 * ((tau >> 3) & 1) + (tau & 1);  // B_P row
    float* xchg = reinterpret_cast<float*>(smem + L::XCHG);
    float* lsum = reinterpret_cast<float*>(smem + L::LSUM);
    // this lane's dim in the P.V accumulator (tensor-memory lane 32q + lane; see unpack_v),
    // and the factor 1/16 of the dims whose codes sit in bits 4..7
    const int dim = 32 * (lane & 3) + 8 * q + 4 * ((lane & 7) >> 2) + (lane >> 3);
    const float dsc = ((lane >> 3) & 1) ? 0.0625f : 1.0f;
    uint32_t kt = 0, ii = 0;
    while (items.next()) {
      const int nt = items.tiles(), ib = ii & 1;
      warp_wait(bar + kQFull + ib, (ii >> 1) & 1, abort);
      float ce[4], cor[4][4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        ce[h] = reinterpret_cast<const float*>(smem + L::CEXP)[8 * ib + 4 * hh + h];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          cor[g][h] = reinterpret_cast<const float*>(smem + L::CORR)[32 * ib + 8 * g + 4 * hh + h];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kQEmpty + ib);
      // softmax reference of all 8 heads (every softmax warp takes the same
      // decisions); sums and accumulator of this warp's 4 heads
      float mref[8], lacc[4], acc[4];
#pragma unroll
      for (int h = 0; h < 8; ++h) mref[h] = -INFINITY;
#pragma unroll
      for (int h = 0; h < 4; ++h) lacc[h] = acc[h] = 0.0f;
      int F = 0;
      for (int j = 0; j < nt; ++j, ++kt) {
        const int s = kt % kNS, bb = kt & 1;
        const uint32_t n = kt >> 1;
        const unsigned char* stg = smem + s * L::STAGE;
        const int nvalid = min(kTile, items.t1 - items.t0 - kTile * j);
        const bool valid = tau < nvalid;
        warp_wait(bar + kDSFull + bb, n & 1, abort);
        fence_after();
        uint32_t d[4][8];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          tld_x8(tbase + lane_base(q) + kColDS + 64 * bb + 16 * g + 8 * hh, d[g]);
        wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) tie8(d[g]);
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + kDSEmpty + bb);
        warp_wait(bar + kFull + s, (kt / kNS) & 1, abort);
        const float4 sk = *reinterpret_cast<const float4*>(stg + L::KS + 16 * tau);
        const float4 sv = *reinterpret_cast<const float4*>(stg + L::VS + 16 * tau);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + kEmpty + s);
        const float skg[4] = {sk.x, sk.y, sk.z, sk.w};
        // S = sum_g s_k[g] (D_hi + D_lo - 8 2^-24 sum_g q), in log2 units after ce
        float x[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          float acc_s = 0.0f;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            acc_s = fmaf(skg[g], __uint_as_float(d[g][h]), acc_s);
            acc_s = fmaf(skg[g], __uint_as_float(d[g][4 + h]), acc_s);
            acc_s = fmaf(skg[g], cor[g][h], acc_s);
          }
          x[h] = valid ? acc_s * ce[h] : -INFINITY;
        }
        const float vloc = valid ? fmaxf(fmaxf(sv.x, sv.y), fmaxf(sv.z, sv.w)) : 0.0f;
        // Does the reference have to move?  A tile's maximum more than kTau above a
        // head's reference, or V scales that would push P' past 2^15 (F); always on
        // an item's first tile.  One vote per warp, then every softmax warp reads the
        // eight votes; only then are the maxima exchanged (the same decision in all).
        bool need = j == 0 || vloc * pow2i(-F) >= 128.0f;
#pragma unroll
        for (int h = 0; h < 4; ++h) need |= x[h] > (hh ? mref[4 + h] : mref[h]) + kTau;
        int* xv = reinterpret_cast<int*>(xchg) + (bb * 8 + sw) * 8;
        need = __any_sync(0xffffffffu, need);
        if (lane == 0) xv[0] = need;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        bool any = false;
#pragma unroll
        for (int w = 0; w < 8; ++w) any |= reinterpret_cast<const int*>(xchg)[(bb * 8 + w) * 8] != 0;
        float alpha[4] = {1.0f, 1.0f, 1.0f, 1.0f};
        bool flag = false;
        if (any) {
          float* xc = xchg + (bb * 8 + sw) * 8;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float mx = redux_max(x[h]);
            if (lane == 0) xc[1 + h] = mx;
          }
          {
            const float vm = redux_max(vloc);
            if (lane == 0) xc[5] = vm;
          }
          asm volatile("bar.sync 1, 256;" ::: "memory");
          float mt[8], vmax = 0.0f;
#pragma unroll
          for (int h = 0; h < 8; ++h) mt[h] = -INFINITY;
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            const float* xo = xchg + (bb * 8 + w) * 8;
#pragma unroll
            for (int h = 0; h < 4; ++h) mt[4 * (w >> 2) + h] = fmaxf(mt[4 * (w >> 2) + h], xo[1 + h]);
            vmax = fmaxf(vmax, xo[5]);
          }
          int ev_ex = 0;
          if (vmax > 0.0f) frexpf(vmax, &ev_ex);
          const int Fv = max(-100, min(100, ev_ex - 3));  // vmax 2^-F in [4, 8)
          if (j == 0) {
#pragma unroll
            for (int h = 0; h < 8; ++h) mref[h] = mt[h];
            F = vmax > 0.0f ? Fv : 0;
          } else {
            const bool evf = vmax * pow2i(-F) >= 128.0f;
            const int Fn = evf ? Fv : F;
            float al[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              const bool evm = mt[h] > mref[h] + kTau;
              const float mn = evm ? mt[h] : mref[h];
              flag |= evm;
              al[h] = ex2(mref[h] - mn);  // the same factor for the sum and the accumulator
              mref[h] = mn;
            }
            flag |= evf;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float a4 = hh ? al[4 + h] : al[h];
              alpha[h] = a4 * pow2i(F - Fn);
              lacc[h] *= a4;
            }
            F = Fn;
          }
        }
        float p[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          p[h] = valid ? ex2(x[h] - (hh ? mref[4 + h] : mref[h])) : 0.0f;
          lacc[h] += p[h];
        }
        const float fsc = pow2i(-F);
        const float svg[4] = {valid ? sv.x * fsc : 0.0f, valid ? sv.y * fsc : 0.0f,
                              valid ? sv.z * fsc : 0.0f, valid ? sv.w * fsc : 0.0f};
        // B_P[bb] and the event record are free once tile kt-2's P.V is done
        if (kt >= 2) warp_wait(bar + kAVEmpty + bb, (n - 1) & 1, abort);
        if (flag) {
          // fold this half's accumulator (tiles up to kt-1: done once tile kt-1's P.V
          // is) into registers; tile kt's P.V starts it afresh
          const uint32_t kp = kt - 1;
          warp_wait(bar + kAVEmpty + (kp & 1), (kp >> 1) & 1, abort);
          fence_after();
          fold_half(tbase, q, hh, lane, acc, alpha);
          fence_before();
        }
        if (sw == 0 && lane == 0) reinterpret_cast<Evt*>(smem + L::EVT + bb * L::EVT_SIZE)->flag = flag;
        unsigned char* bp = smem + L::BP + bb * 16384 + (kk >> 3) * 128 + (kk & 7) * 16;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float hv[4], lv[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float w = p[h] * svg[g];
            hv[h] = __uint_as_float(__float_as_uint(w) & 0xFFFFE000u);
            lv[h] = w - hv[h];
          }
          uint4 v;
          v.x = f16x2(hv[0], hv[1]);
          v.y = f16x2(hv[2], hv[3]);
          v.z = f16x2(lv[0], lv[1]);
          v.w = f16x2(lv[2], lv[3]);
          *reinterpret_cast<uint4*>(bp + (2 * g + hh) * 2048) = v;  // N columns 16g + 8hh + ..
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + kBPFull + bb);
      }
      // item end: the last P.V, then this lane's dim of the partial for the half's heads
      {
        const uint32_t kl = kt - 1;
        warp_wait(bar + kAVEmpty + (kl & 1), (kl >> 1) & 1, abort);
        fence_after();
        const float ones[4] = {1.0f, 1.0f, 1.0f, 1.0f};
        fold_half(tbase, q, hh, lane, acc, ones);
        fence_before();
      }
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float v = lacc[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) lsum[sw * 4 + h] = v;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const int stride = a.plan.part_stride;
      float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + a.plan.header_bytes);
      const bool bad = __any_sync(0xffffffffu, *abort != 0);
      const float sc = pow2i(F) * dsc;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int head = 4 * hh + h;
        if (head >= G) break;
        float* dst = part + (((int64_t)items.b * a.Hq + (int64_t)items.kvh * G + head) * a.plan.n_chunks +
                             items.c) * stride;
        dst[dim] = acc[h] * sc;
        if (q == 0 && lane == 0) {
          float l = 0.0f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) l += lsum[(4 * hh + qq) * 4 + h];
          dst[kD] = bad ? __int_as_float(0x7fc00000) : (hh ? mref[4 + h] : mref[h]);
          dst[kD + 1] = l;
        }
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");  // lsum reused by the next item
      ++ii;
    }
  } else if (warp == kProducerWarp) {
    // ================================================== producer
    uint32_t kt = 0;
    if (lane == 0) {
      bool appended = a.k_new == nullptr;
      while (items.next()) {
        const int nt = items.tiles();
        const int T = clamp_ctx(a.ctx_lens[items.b], a.max_ctx);
        const int64_t bh = (int64_t)items.b * a.Hkv + items.kvh;
        for (int j = 0; j < nt; ++j, ++kt) {
          const int s = kt % kNS;
          if (kt >= kNS) mbar_wait(bar + kEmpty + s, ((kt / kNS) - 1) & 1, abort);
          if (*abort) break;
          const int t = items.t0 + kTile * j;
          const int rows = min(kTile, items.t1 - t);
          const bool last_row = t + rows == T;  // holds the row a fused append writes
          if (last_row && !appended) {
            mbar_wait(bar + kAppDone, 0, abort);
            appended = true;
          }
          if (last_row && a.q_rot_overlap == 2) asm volatile("griddepcontrol.wait;" ::: "memory");
          if (a.test_starve && kt == 0) continue;  // test hook: the first stage never arrives
          unsigned char* stg = smem + s * L::STAGE;
          const int64_t row = bh * a.capacity + t;
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive_expect_tx(bar + kFull + s, 8192u + (uint32_t)rows * 96u);
          tma_load_3d(stg + L::VC, &tmap_v, 0, t, (int)bh, bar + kFull + s);
          bulk_g2s(stg + L::KC, a.k_packed + row * 64, (uint32_t)rows * 64u, bar + kFull + s);
          bulk_g2s(stg + L::KS, a.k_scales + row * 4, (uint32_t)rows * 16u, bar + kFull + s);
          bulk_g2s(stg + L::VS, a.v_scales + row * 4, (uint32_t)rows * 16u, bar + kFull + s);
        }
        if (*abort) break;
      }
      // copies still in flight must land before the CTA exits
      const uint32_t first = kt > (uint32_t)kNS ? kt - kNS : 0;
      for (uint32_t u = first; u < kt; ++u) {
        if (a.test_starve && u == 0) continue;
        mbar_drain(bar + kFull + u % kNS, (u / kNS) & 1);
      }
    }
  } else if (warp == kScoreMmaWarp) {
    // ================================================== score MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 16, 0, 0);
      // descriptor of the buffer's first core matrix; a later block of the same
      // buffer adds its byte offset / 16 to the address field (no carry: every
      // shared-memory address is below 256 KB)
      const uint64_t dq0 = smem_desc(smem_u32(smem + L::BQ), 128, 256);
      uint32_t kt = 0, ii = 0;
      while (items.next()) {
        const int nt = items.tiles(), ib = ii & 1;
        mbar_wait(bar + kQFull + ib, (ii >> 1) & 1, abort);
        const uint64_t dq = dq0 + (uint64_t)((ib * L::BQ_SIZE) >> 4);
        for (int j = 0; j < nt; ++j, ++kt) {
          const int bb = kt & 1;
          const uint32_t n = kt >> 1;
          mbar_wait(bar + kAKFull + bb, n & 1, abort);
          if (kt >= 2) mbar_wait(bar + kDSEmpty + bb, (n - 1) & 1, abort);
          fence_after();
          if (!*abort) {
            const uint32_t ds = tbase + kColDS + 64 * bb, ak = tbase + kColAK + 64 * bb;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              mma_ts(ds + 16 * g, ak + 16 * g, dq + (uint64_t)(64 * g), idS, 0u);
              mma_ts(ds + 16 * g, ak + 16 * g + 8, dq + (uint64_t)(64 * g + 32), idS, 1u);
            }
          }
          mma_commit(bar + kDSFull + bb);
          mma_commit(bar + kAKEmpty + bb);
          if (j == nt - 1) mma_commit(bar + kQEmpty + ib);
        }
        ++ii;
      }
      mma_commit(bar + kMmaDone);
      mbar_drain(bar + kMmaDone, 0);
    }
  } else if (warp == kPvMmaWarp) {
    // ================================================== P.V MMA issuer
    // O[dim, 16g + 8hh + 4 part + h] (+)= A_V x B_P, 8 K-blocks of 16 tokens per
    // tile; afresh on an item's first tile or after the softmax folded
    if (lane == 0) {
      constexpr uint32_t idPV = idesc_f16(128, 64, 0, 1);
      const uint64_t dp0 = smem_desc(smem_u32(smem + L::BP), 128, 2048);
      uint32_t kt = 0;
      while (items.next()) {
        const int nt = items.tiles();
        for (int j = 0; j < nt; ++j, ++kt) {
          const int bb = kt & 1;
          const uint32_t n = kt >> 1;
          mbar_wait(bar + kAVFull + bb, n & 1, abort);
          mbar_wait(bar + kBPFull + bb, n & 1, abort);
          const bool fresh = j == 0 || reinterpret_cast<const Evt*>(smem + L::EVT + bb * L::EVT_SIZE)->flag;
          fence_after();
          if (!*abort) {
            const uint64_t dp = dp0 + (uint64_t)((bb * 16384) >> 4);
            const uint32_t av = tbase + kColAV + 64 * bb;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ts(tbase + kColO, av + 8 * k, dp + (uint64_t)(16 * k), idPV, (k > 0 || !fresh) ? 1u : 0u);
          }
          mma_commit(bar + kAVEmpty + bb);
        }
      }
      mma_commit(bar + kMmaDone);
      mbar_drain(bar + kMmaDone, 0);
    }
  } else if (warp == kQueryWarp) {
    // ================================================== query warp
    uint32_t ii = 0;
    bool appended = a.k_new == nullptr;
    while (items.next()) {
      const int ib = ii & 1;
      if (ii >= 2) warp_wait(bar + kQEmpty + ib, ((ii >> 1) - 1) & 1, abort);
      prep_query(a, items.b, items.kvh, smem, ib, lane);
      if (lane == 0) mbar_arrive(bar + kQFull + ib);
      ++ii;
      if (!appended) {
        // fused append: every (sequence, kv head) whose last chunk is one of
        // this CTA's items gets its new K and V token in row T - 1
        Items mine(a, pfx, n_items);
        while (mine.next()) {
          const int T = clamp_ctx(a.ctx_lens[mine.b], a.max_ctx);
          if (mine.t1 != T) continue;
          const int64_t bh = (int64_t)mine.b * a.Hkv + mine.kvh;
          const int64_t row = bh * a.capacity + (T - 1);
          if (a.inputs_pending) asm volatile("griddepcontrol.wait;" ::: "memory");
          const int eb = a.kv_bf16 ? 2 : 4;
          quantize_vector_warp<kD>(static_cast<const unsigned char*>(a.k_new) + bh * kD * eb, a.kv_bf16,
                                   a.signs, const_cast<uint8_t*>(a.k_packed) + row * 64,
                                   const_cast<float*>(a.k_scales) + row * 4, lane);
          quantize_vector_warp<kD>(static_cast<const unsigned char*>(a.v_new) + bh * kD * eb, a.kv_bf16,
                                   a.signs, const_cast<uint8_t*>(a.v_packed) + row * 64,
                                   const_cast<float*>(a.v_scales) + row * 4, lane);
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + kAppDone);
        appended = true;
      }
    }
    if (!appended) {  // no items: nothing to append here
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kAppDone);
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
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

}  // namespace

bool decode_tc_supported(int d, int G) { return d == 128 && G >= 1 && G <= 8; }

int decode_tc_tile_tokens() { return kTile; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  if (!decode_tc_supported(a.d, a.Hq / a.Hkv) || a.cb_bits != 0) return cudaErrorNotSupported;
  static SmemLimitSet smem_set;
  cudaError_t e = ensure_smem_limit(decode_tc_kernel, L::BYTES + 1024, smem_set);
  if (e != cudaSuccess) return e;
  // V codes as a 3-D uint8 tensor {64 bytes, capacity rows, B * Hkv}, 128-row
  // boxes with the 64-byte swizzle (rows past the capacity read as zeros)
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[3] = {64, (cuuint64_t)a.capacity, (cuuint64_t)a.B * a.Hkv};
  const cuuint64_t strides[2] = {64, (cuuint64_t)a.capacity * 64};
  const cuuint32_t box[3] = {64, (cuuint32_t)kTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(a.v_packed), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_items = a.B * a.Hkv * a.plan.n_chunks;
  const int grid = n_items < sms ? n_items : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::BYTES + 1024;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ((a.q_rot != nullptr && a.q_rot_overlap) || a.inputs_pending) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel, a, tmap);
}

}  // namespace tq
