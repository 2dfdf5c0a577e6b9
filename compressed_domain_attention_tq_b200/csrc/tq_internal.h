// tq_internal.h -- declarations shared by the libtq translation units.
// Not part of the public ABI (include/tq.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/tq.h"

namespace tq {

constexpr int kGroup = 32;  // quantization group (rotated coordinates)
constexpr int kSmCount = 148;  // B200; sizes the split-K plan (a host-only, device-free choice)

// Split-K work decomposition of one decode call (host side, deterministic).
struct DecodePlan {
  int chunk;        // context tokens per chunk (multiple of the decode's stage)
  int n_chunks;     // ceil(max_ctx / chunk)
  int part_stride;  // floats per (b, q head, chunk) partial: d + 4 (16-byte rows)
  size_t header_bytes;  // int32 flags[B], rounded up to 256 bytes
  size_t qrot_offset;   // SRFT variant: rotated queries float[B][Hq][d] at this offset (else 0)
  size_t ws_bytes;  // header + partials (+ rotated queries)
};

// kind: the int4 cache (head_dim 128 or 256), the SRFT variant (any head_dim
// accepted by srft_head_dim_supported, plus room for the rotated queries), or
// the codebook variant (head_dim 128 or 256, always the CUDA-core decode).
enum class PlanKind { kInt4, kSrft, kCodebook };
bool make_decode_plan(int B, int Hq, int Hkv, int d, int max_ctx, DecodePlan* plan,
                      PlanKind kind = PlanKind::kInt4);

struct QuantizeArgs {
  const void* k;
  const void* v;
  int bf16;
  int B, Hkv, n_new, d;
  const int32_t* pos;
  const int8_t* signs;
  uint8_t* k_packed;
  float* k_scales;
  uint8_t* v_packed;
  float* v_scales;
  int64_t capacity;
  int pos_is_ctx = 0;  // 1: token n of sequence b goes to row clamp(pos[b], 1, max_ctx) - 1 + n
  int max_ctx = 0;
  const float* lambda_k = nullptr;  // SRFT variant: per-coordinate scales (NULL = ones)
  const float* lambda_v = nullptr;
  int cb_bits = 0;                  // codebook variant: bits per index (2, 3, 4), else 0
  const float* levels = nullptr;    // codebook variant: 2^cb_bits increasing levels (device)
  int cb_uniform = 0;               // uniform low-bit variant (abs-max scale, index c + m) of cb_bits
  int test_starve = 0;              // test hook: the tensor-core kernel withholds its first copy
  int butterfly_rotation = 0;       // test hook: CUDA-core butterflies instead of the tensor cores
};

struct DequantizeArgs {
  const uint8_t* packed;
  const float* scales;
  int n_seq, rows, d;
  int64_t row_stride;
  void* out;
  int bf16;
};

struct DecodeArgs {
  const void* q;
  int q_bf16;
  int B, Hq, Hkv, d;
  const uint8_t* k_packed;
  const float* k_scales;
  const uint8_t* v_packed;
  const float* v_scales;
  int64_t capacity;
  const int32_t* ctx_lens;
  int max_ctx;
  const int8_t* signs;
  float attn_scale;
  float* out;
  void* workspace;
  DecodePlan plan;
  const void* k_new;  // fused append (decode_mma only): [B][Hkv][1][d] new K and V, or NULL
  const void* v_new;
  int kv_bf16;
  float* lse;  // NULL, or [B][Hq][2]: each head's (max in log2 units, sum) for merging contexts
  const float* q_rot = nullptr;     // SRFT variant: [B][Hq][d] rotated queries F(sigma q)/lambda_K;
                                    // the decode kernels read these instead of rotating q
  int test_starve = 0;              // test hook: the tensor-core decode withholds each CTA's
                                    // first copy, so its waits run out (the abort path)
  int q_rot_overlap = 0;            // the tensor-core decode may start while the preceding grid
                                    // runs (programmatic dependent launch): 1 = that grid only
                                    // rotates the queries; 2 = it also appends each sequence's
                                    // last row, so the copy of that row waits for it
  const float* lambda_k = nullptr;  // SRFT variant: per-coordinate scales (NULL = ones)
  const float* lambda_v = nullptr;
  int cb_bits = 0;                  // codebook variant: bits per index (2, 3, 4), else 0
  const float* levels = nullptr;    // codebook variant: 2^cb_bits increasing levels (device)
  int cb_uniform = 0;               // the fused append writes uniform low-bit indices
  int inputs_pending = 0;           // q, k_new and v_new are written by the preceding kernel:
                                    // the tensor-core decode is launched as its programmatic
                                    // dependent and waits for it before reading them
};

// Identity of the CUDA context current on the calling thread: unique for the
// life of the process (a device reset, or a context the caller creates with the
// driver API, gives a new one).  Returns false when no context is current yet
// (the runtime binds one on this thread's first runtime call) or the driver
// cannot be queried.
bool current_context_id(unsigned long long* id);

// The argument checks of tq_sdpa_int4_decode that precede the workspace check
// (returns TQ_OK or that call's error status).
tq_status validate_decode_args(const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t group, const uint8_t* k_packed,
                         const float* k_scales, const uint8_t* v_packed, const float* v_scales,
                         int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx, float attn_scale,
                         const float* out);

// Test hooks set by tq_set_test_hooks (bits TQ_TEST_HOOK_*), read once per call.
extern std::atomic<unsigned> g_test_hooks;

// Contexts in which a kernel's dynamic shared memory limit has been raised.
// Function attributes live in the context that loaded the kernel, so the
// limit is raised once per context (the first launch there); later launches,
// including those made while a stream is being captured into a CUDA graph,
// only enqueue work.
struct SmemLimitSet {
  static constexpr int kSlots = 8;
  std::atomic<unsigned long long> ctx[kSlots] = {};
  std::atomic<unsigned> next{0};
};

template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kernel, int bytes, SmemLimitSet& done) {
  unsigned long long id = 0;
  if (current_context_id(&id))
    for (int i = 0; i < SmemLimitSet::kSlots; ++i)
      if (done.ctx[i].load(std::memory_order_acquire) == id) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && (id != 0 || current_context_id(&id)))
    done.ctx[done.next.fetch_add(1) % SmemLimitSet::kSlots].store(id, std::memory_order_release);
  return e;
}

// The merge kernels follow the split-K decode as its programmatic dependents,
// so their CTAs may start while the decode's CTAs still hold their SMs.  Small
// as they are, every one of them would then start on the few SMs the decode
// leaves free and run the whole merge there.  Each merge CTA therefore asks
// for this much dynamic shared memory, which it does not use: at most two fit
// on an SM, and the rest start on the SMs the decode releases.  Grids of more
// than two CTAs per SM skip the cap, which would split them into waves.
constexpr int kMergeSmemBytes = 100 * 1024;
inline int merge_smem_bytes(long long merge_ctas) {
  return merge_ctas <= 2LL * kSmCount ? kMergeSmemBytes : 0;
}

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t stream);
bool quantize_tc_supported(const QuantizeArgs& a);  // bulk bf16, d = 128, rotation on
cudaError_t launch_quantize_tc(const QuantizeArgs& a, cudaStream_t stream);
cudaError_t launch_dequantize(const DequantizeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t stream);
bool decode_mma_supported(int d, int G);
bool decode_mma_cb_supported(int d, int G);  // codebook caches on the tensor-core decode
int decode_stage_tokens(int d, int G);  // tokens per pipeline stage of the decode path
cudaError_t launch_decode_mma(const DecodeArgs& a, cudaStream_t stream);
bool decode_tc_supported(int d, int G);  // the tcgen05 decode (int4 cache, d = 128, G <= 8)
int decode_tc_tile_tokens();
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream);
bool srft_head_dim_supported(int d);
cudaError_t launch_quantize_srft(const QuantizeArgs& a, cudaStream_t stream);
bool quantize_srft_tc_supported(const QuantizeArgs& a);  // bf16, d = 32 .. 128 (multiple of 32)
cudaError_t launch_quantize_srft_tc(const QuantizeArgs& a, cudaStream_t stream);
cudaError_t launch_srft_query(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_merge_srft(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_srft_prep(const QuantizeArgs& qa, const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_quantize_cb(const QuantizeArgs& a, cudaStream_t stream);
void lloyd_max_gaussian(int bits, double* levels);
cudaError_t launch_merge_lse(const float* outs, const float* lses, int n_parts, int64_t n_heads,
                             int d, float* out, cudaStream_t stream);

}  // namespace tq
