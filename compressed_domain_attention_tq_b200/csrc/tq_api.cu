// tq_api.cu -- the C ABI of libtq (declared in include/tq.h): host-side
// validation, the split-K plan, and kernel dispatch.  Nothing here allocates;
// every buffer belongs to the caller (as in the AdapTQ post, section "zero
// heap allocation": no allocation on the hot path).
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <cudaTypedefs.h>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {

static inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Driver entry points for the context identity, looked up once through the
// runtime (libtq links no driver library).
namespace {
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxFns& ctx_fns() {
  static const CtxFns fns = [] {
    CtxFns f;
    cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
    void* p1 = nullptr;
    void* p2 = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p1, 4000, cudaEnableDefault, &q1) ==
            cudaSuccess &&
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &p2, 12000, cudaEnableDefault, &q2) ==
            cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess && q2 == cudaDriverEntryPointSuccess) {
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p1);
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p2);
    }
    return f;
  }();
  return fns;
}
}  // namespace

bool current_context_id(unsigned long long* id) {
  const CtxFns& f = ctx_fns();
  if (f.get_current == nullptr || f.get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return f.get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

// Test hooks (bits of tq_set_test_hooks), off unless a test turns them on.
std::atomic<unsigned> g_test_hooks{0};

// Split the context into chunks (multiples of the decode's pipeline stage,
// 192 or 128 tokens): pick the chunk count per sequence that minimises
// (waves of items over the CTA slots) x (chunk + a fixed per-item cost), where
// an item is one (sequence, kv head, chunk).  The tensor-core decode runs
// persistent CTAs, one per SM; the CUDA-core decode runs one 128-thread CTA
// per item, several resident per SM.
static bool make_decode_plan_uncached(int B, int Hq, int Hkv, int d, int max_ctx, DecodePlan* plan,
                                      PlanKind kind);

// The plan depends only on its arguments; each thread keeps its last one, so
// a decode loop with fixed sizes does the search once.
bool make_decode_plan(int B, int Hq, int Hkv, int d, int max_ctx, DecodePlan* plan, PlanKind kind) {
  struct Last {
    int B = 0, Hq = 0, Hkv = 0, d = 0, max_ctx = 0;
    PlanKind kind = PlanKind::kInt4;
    DecodePlan plan{};
  };
  thread_local Last last;
  if (last.B == B && last.Hq == Hq && last.Hkv == Hkv && last.d == d && last.max_ctx == max_ctx &&
      last.kind == kind && B > 0) {
    *plan = last.plan;
    return true;
  }
  if (!make_decode_plan_uncached(B, Hq, Hkv, d, max_ctx, plan, kind)) return false;
  last.B = B;
  last.Hq = Hq;
  last.Hkv = Hkv;
  last.d = d;
  last.max_ctx = max_ctx;
  last.kind = kind;
  last.plan = *plan;
  return true;
}

static bool make_decode_plan_uncached(int B, int Hq, int Hkv, int d, int max_ctx, DecodePlan* plan,
                                      PlanKind kind) {
  if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0 || max_ctx < 1) return false;
  const bool srft = kind == PlanKind::kSrft;
  if (srft ? !srft_head_dim_supported(d) : (d != 128 && d != 256)) return false;
  const int64_t units = (int64_t)B * Hkv;
  const bool mma = kind == PlanKind::kCodebook ? decode_mma_cb_supported(d, Hq / Hkv)
                                              : decode_mma_supported(d, Hq / Hkv);
  const int64_t step = mma ? decode_stage_tokens(d, Hq / Hkv) : 128, per_item_cost = mma ? 384 : 256;
  const int64_t slots = mma ? kSmCount : 4 * kSmCount;
  const int64_t max_n = ceil_div(max_ctx, step);
  int64_t best_chunk = ceil_div(max_ctx, step) * step, best_cost = -1;
  for (int64_t n = 1; n <= max_n && n <= 4096; ++n) {
    const int64_t chunk = ceil_div(ceil_div(max_ctx, n), step) * step;
    const int64_t items = units * ceil_div(max_ctx, chunk);
    const int64_t cost = ceil_div(items, slots) * (chunk + per_item_cost);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_chunk = chunk;
    }
  }
  plan->chunk = (int)best_chunk;
  plan->n_chunks = (int)ceil_div(max_ctx, best_chunk);
  plan->part_stride = d + 4;
  plan->header_bytes = (size_t)ceil_div(4LL * B, 256) * 256;
  plan->ws_bytes = plan->header_bytes +
                   sizeof(float) * (size_t)B * Hq * plan->n_chunks * plan->part_stride;
  plan->qrot_offset = 0;
  if (srft) {  // the rotated queries follow the partials
    plan->qrot_offset = (size_t)ceil_div((int64_t)plan->ws_bytes, 256) * 256;
    plan->ws_bytes = plan->qrot_offset + sizeof(float) * (size_t)B * Hq * d;
  }
  return true;
}

// A failed CUDA call becomes TQ_ERR_CUDA; with the environment variable
// TQ_DEBUG set, its CUDA error string is also printed on stderr.
static tq_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return TQ_OK;
  if (getenv("TQ_DEBUG")) fprintf(stderr, "libtq: %s: %s\n", where, cudaGetErrorString(e));
  return TQ_ERR_CUDA;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// The variant of a call: the int4 cache with the Hadamard rotation (signs) or
// none; the SRFT variant (srft: signs, optional per-coordinate scales of K and
// V); or the codebook variant (cb_bits 2..4 with its levels, Hadamard or none).
struct Rotation {
  bool srft = false;
  const float* lambda_k = nullptr;
  const float* lambda_v = nullptr;
  int cb_bits = 0;
  const float* levels = nullptr;
  bool cb_uniform = false;  // uniform low-bit indices in the codebook layout (levels u - m)
};

static bool head_dim_ok(int d, const Rotation& rot) {
  return rot.srft ? srft_head_dim_supported(d) : (d == 128 || d == 256);
}

static bool codebook_ok(const Rotation& rot) {
  if (rot.cb_bits == 0) return true;
  if (rot.cb_bits < 2 || rot.cb_bits > 4) return false;
  if (rot.cb_uniform && rot.levels == nullptr) return true;  // a uniform quantize reads no levels
  return rot.levels != nullptr && (reinterpret_cast<uintptr_t>(rot.levels) & 3u) == 0;
}

}  // namespace tq

using namespace tq;

extern "C" {

void tq_set_test_hooks(uint32_t hooks) { g_test_hooks.store(hooks, std::memory_order_relaxed); }

const char* tq_status_string(tq_status status) {
  switch (status) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument (pointer, size, shape or alignment)";
    case TQ_ERR_UNSUPPORTED: return "unsupported configuration (head_dim, group or GQA ratio)";
    case TQ_ERR_WORKSPACE: return "workspace missing or smaller than tq_decode_workspace_bytes()";
    case TQ_ERR_CUDA: return "CUDA launch or runtime error";
    case TQ_ERR_SCRATCH_LIMIT:
      return "sizes need more decode scratch than the built-in TQ_STATIC_SCRATCH_BYTES";
  }
  return "unknown status";
}

}  // extern "C"

static tq_status quantize_impl(const void* k, const void* v, tq_dtype in_dtype, int32_t batch,
                               int32_t num_kv_heads, int32_t n_new, int32_t head_dim,
                               int32_t group, const int32_t* pos, const int8_t* signs,
                               const Rotation& rot, uint8_t* k_packed, float* k_scales,
                               uint8_t* v_packed, float* v_scales, int64_t capacity,
                               void* cuda_stream, const char* where) {
  if (!k || !v || !pos || !k_packed || !k_scales || !v_packed || !v_scales) return TQ_ERR_INVALID_ARG;
  if (in_dtype != TQ_F32 && in_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (batch < 1 || num_kv_heads < 1 || n_new < 1 || capacity < n_new) return TQ_ERR_INVALID_ARG;
  if ((int64_t)batch * num_kv_heads * n_new > INT32_MAX) return TQ_ERR_INVALID_ARG;
  if (!head_dim_ok(head_dim, rot)) return TQ_ERR_UNSUPPORTED;
  if (group != kGroup) return TQ_ERR_UNSUPPORTED;
  if (rot.cb_bits != 0 && (rot.cb_bits < 2 || rot.cb_bits > 4)) return TQ_ERR_UNSUPPORTED;
  if (!codebook_ok(rot)) return TQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_packed) || !aligned16(v_packed) ||
      !aligned16(k_scales) || !aligned16(v_scales) || !aligned4(rot.lambda_k) ||
      !aligned4(rot.lambda_v))
    return TQ_ERR_INVALID_ARG;
  QuantizeArgs a;
  a.k = k;
  a.v = v;
  a.bf16 = in_dtype == TQ_BF16;
  a.B = batch;
  a.Hkv = num_kv_heads;
  a.n_new = n_new;
  a.d = head_dim;
  a.pos = pos;
  a.signs = signs;
  a.k_packed = k_packed;
  a.k_scales = k_scales;
  a.v_packed = v_packed;
  a.v_scales = v_scales;
  a.capacity = capacity;
  a.lambda_k = rot.lambda_k;
  a.lambda_v = rot.lambda_v;
  a.cb_bits = rot.cb_bits;
  a.levels = rot.levels;
  a.cb_uniform = rot.cb_uniform ? 1 : 0;
  const unsigned hooks = g_test_hooks.load(std::memory_order_relaxed);
  a.test_starve = (hooks & TQ_TEST_HOOK_STARVE_PIPELINE) != 0;
  a.butterfly_rotation = (hooks & TQ_TEST_HOOK_BUTTERFLY_QUANTIZE) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const cudaError_t e = rot.srft ? launch_quantize_srft(a, s)
                        : rot.cb_bits ? launch_quantize_cb(a, s)
                                      : launch_quantize(a, s);
  return cuda_status(e, where);
}

extern "C" {

tq_status tq_quantize_append(const void* k, const void* v, tq_dtype in_dtype, int32_t batch,
                             int32_t num_kv_heads, int32_t n_new, int32_t head_dim,
                             int32_t group, const int32_t* pos, const int8_t* signs,
                             uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                             float* v_scales, int64_t capacity, void* cuda_stream) {
  return quantize_impl(k, v, in_dtype, batch, num_kv_heads, n_new, head_dim, group, pos, signs,
                       Rotation{}, k_packed, k_scales, v_packed, v_scales, capacity, cuda_stream,
                       "tq_quantize_append");
}

tq_status tq_quantize_append_srft(const void* k, const void* v, tq_dtype in_dtype, int32_t batch,
                                  int32_t num_kv_heads, int32_t n_new, int32_t head_dim,
                                  int32_t group, const int32_t* pos, const int8_t* signs,
                                  const float* lambda_k, const float* lambda_v,
                                  uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                                  float* v_scales, int64_t capacity, void* cuda_stream) {
  return quantize_impl(k, v, in_dtype, batch, num_kv_heads, n_new, head_dim, group, pos, signs,
                       Rotation{true, lambda_k, lambda_v}, k_packed, k_scales, v_packed,
                       v_scales, capacity, cuda_stream, "tq_quantize_append_srft");
}

tq_status tq_quantize_append_cb(const void* k, const void* v, tq_dtype in_dtype, int32_t batch,
                                int32_t num_kv_heads, int32_t n_new, int32_t head_dim,
                                int32_t group, int32_t bits, const float* levels,
                                const int32_t* pos, const int8_t* signs, uint8_t* k_packed,
                                float* k_scales, uint8_t* v_packed, float* v_scales,
                                int64_t capacity, void* cuda_stream) {
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  return quantize_impl(k, v, in_dtype, batch, num_kv_heads, n_new, head_dim, group, pos, signs, r,
                       k_packed, k_scales, v_packed, v_scales, capacity, cuda_stream,
                       "tq_quantize_append_cb");
}

tq_status tq_quantize_append_uniform(const void* k, const void* v, tq_dtype in_dtype,
                                     int32_t batch, int32_t num_kv_heads, int32_t n_new,
                                     int32_t head_dim, int32_t group, int32_t bits,
                                     const int32_t* pos, const int8_t* signs, uint8_t* k_packed,
                                     float* k_scales, uint8_t* v_packed, float* v_scales,
                                     int64_t capacity, void* cuda_stream) {
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.cb_uniform = true;
  return quantize_impl(k, v, in_dtype, batch, num_kv_heads, n_new, head_dim, group, pos, signs, r,
                       k_packed, k_scales, v_packed, v_scales, capacity, cuda_stream,
                       "tq_quantize_append_uniform");
}

tq_status tq_uniform_levels(int32_t bits, float* levels) {
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  if (!levels) return TQ_ERR_INVALID_ARG;
  const int m = (1 << (bits - 1)) - 1;
  for (int u = 0; u < (1 << bits); ++u) levels[u] = (float)(u - m);
  return TQ_OK;
}

tq_status tq_lloyd_max_gaussian(int32_t bits, float* levels) {
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  if (!levels) return TQ_ERR_INVALID_ARG;
  double c[16];
  lloyd_max_gaussian(bits, c);
  for (int i = 0; i < (1 << bits); ++i) levels[i] = (float)c[i];
  return TQ_OK;
}

size_t tq_decode_cb_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t max_ctx) {
  DecodePlan p;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &p,
                        PlanKind::kCodebook))
    return 0;
  return p.ws_bytes;
}

tq_status tq_dequantize(const uint8_t* packed, const float* scales, int32_t n_seq, int32_t rows,
                        int64_t row_stride, int32_t head_dim, int32_t group, void* out,
                        tq_dtype out_dtype, void* cuda_stream) {
  if (!packed || !scales || !out) return TQ_ERR_INVALID_ARG;
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (n_seq < 1 || rows < 1 || row_stride < rows) return TQ_ERR_INVALID_ARG;
  if (!srft_head_dim_supported(head_dim)) return TQ_ERR_UNSUPPORTED;
  if (group != kGroup) return TQ_ERR_UNSUPPORTED;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(out)) return TQ_ERR_INVALID_ARG;
  DequantizeArgs a;
  a.packed = packed;
  a.scales = scales;
  a.n_seq = n_seq;
  a.rows = rows;
  a.row_stride = row_stride;
  a.d = head_dim;
  a.out = out;
  a.bf16 = out_dtype == TQ_BF16;
  return cuda_status(launch_dequantize(a, static_cast<cudaStream_t>(cuda_stream)), "tq_dequantize");
}

size_t tq_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t max_ctx) {
  DecodePlan p;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &p)) return 0;
  return p.ws_bytes;
}

size_t tq_decode_srft_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t max_ctx) {
  DecodePlan p;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &p, PlanKind::kSrft))
    return 0;
  return p.ws_bytes;
}

int32_t tq_decode_chunk_tokens(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t max_ctx) {
  DecodePlan p;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &p)) return 0;
  return p.chunk;
}

}  // extern "C"

// Shared by tq_sdpa_int4_decode and tq_sdpa_int4_decode_append (k_new, v_new
// non-NULL: append the new token of every (sequence, kv head) first).
// A host-buffer step's inputs, moved into the workspace's staging space by
// decode_impl once the call is validated, before its first launch: by the
// gather kernel when the host buffers are mapped, else by three copies.
struct HostInputs {
  bool gather;
  const void *q, *k, *v;  // host buffers (their device addresses when gather)
  unsigned char *dq, *dk, *dv;
  size_t q_bytes, kv_bytes;
};

__global__ void host_gather_kernel(const uint4* q, uint4* dq, int64_t nq, const uint4* k, uint4* dk,
                                   const uint4* v, uint4* dv, int64_t nkv);

static cudaError_t move_host_inputs(const HostInputs& h, cudaStream_t s) {
  if (h.gather) {
    const int64_t nq = (int64_t)(h.q_bytes / 16), nkv = (int64_t)(h.kv_bytes / 16);
    const int64_t n = nq > nkv ? nq : nkv;
    const unsigned blocks = (unsigned)(n / 256 + 1 < 64 ? n / 256 + 1 : 64);
    host_gather_kernel<<<blocks, 256, 0, s>>>(
        static_cast<const uint4*>(h.q), reinterpret_cast<uint4*>(h.dq), nq,
        static_cast<const uint4*>(h.k), reinterpret_cast<uint4*>(h.dk),
        static_cast<const uint4*>(h.v), reinterpret_cast<uint4*>(h.dv), nkv);
    return cudaGetLastError();
  }
  cudaError_t e = cudaMemcpyAsync(h.dq, h.q, h.q_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(h.dk, h.k, h.kv_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(h.dv, h.v, h.kv_bytes, cudaMemcpyHostToDevice, s);
  return e;
}

namespace tq {

// The checks tq_sdpa_int4_decode makes before it looks at the workspace, in
// the same order and with the same results (used by the static-scratch call,
// which must report invalid arguments before its own size limit).
tq_status validate_decode_args(const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                               int32_t num_kv_heads, int32_t head_dim, int32_t group,
                               const uint8_t* k_packed, const float* k_scales, const uint8_t* v_packed,
                               const float* v_scales, int64_t capacity, const int32_t* ctx_lens,
                               int32_t max_ctx, float attn_scale, const float* out) {
  if (!q || !k_packed || !k_scales || !v_packed || !v_scales || !ctx_lens || !out)
    return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  if (batch < 1 || num_kv_heads < 1 || num_q_heads < num_kv_heads || num_q_heads % num_kv_heads != 0)
    return TQ_ERR_INVALID_ARG;
  if (max_ctx < 1 || capacity < max_ctx) return TQ_ERR_INVALID_ARG;
  if (!(attn_scale > 0.0f) || !isfinite(attn_scale)) return TQ_ERR_INVALID_ARG;
  if (!head_dim_ok(head_dim, Rotation{})) return TQ_ERR_UNSUPPORTED;
  if (group != kGroup) return TQ_ERR_UNSUPPORTED;
  if (num_q_heads / num_kv_heads > 16) return TQ_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_packed) || !aligned16(v_packed) ||
      !aligned16(k_scales) || !aligned16(v_scales))
    return TQ_ERR_INVALID_ARG;
  DecodePlan plan;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &plan))
    return TQ_ERR_INVALID_ARG;
  return TQ_OK;
}

}  // namespace tq

static tq_status decode_impl(const void* q, tq_dtype q_dtype, const void* k_new, const void* v_new,
                             tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads,
                             int32_t num_kv_heads, int32_t head_dim, int32_t group,
                             const uint8_t* k_packed, const float* k_scales,
                             const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                             const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                             float attn_scale, float* out, void* workspace, size_t workspace_bytes,
                             void* cuda_stream, const char* where, float* lse = nullptr,
                             const Rotation& rot = Rotation{},
                             const HostInputs* host_in = nullptr) {
  if (!q || !k_packed || !k_scales || !v_packed || !v_scales || !ctx_lens || !out)
    return TQ_ERR_INVALID_ARG;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
  const bool append = k_new != nullptr || v_new != nullptr;
  if (append && (!k_new || !v_new || (kv_dtype != TQ_F32 && kv_dtype != TQ_BF16) ||
                 !aligned16(k_new) || !aligned16(v_new)))
    return TQ_ERR_INVALID_ARG;
  if (batch < 1 || num_kv_heads < 1 || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads != 0)
    return TQ_ERR_INVALID_ARG;
  if (max_ctx < 1 || capacity < max_ctx) return TQ_ERR_INVALID_ARG;
  if (!(attn_scale > 0.0f) || !isfinite(attn_scale)) return TQ_ERR_INVALID_ARG;
  if (!head_dim_ok(head_dim, rot)) return TQ_ERR_UNSUPPORTED;
  if (group != kGroup) return TQ_ERR_UNSUPPORTED;
  if (num_q_heads / num_kv_heads > 16) return TQ_ERR_UNSUPPORTED;
  if (!codebook_ok(rot)) return TQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_packed) || !aligned16(v_packed) ||
      !aligned16(k_scales) || !aligned16(v_scales) || (lse && (reinterpret_cast<uintptr_t>(lse) & 7u)) ||
      !aligned4(rot.lambda_k) || !aligned4(rot.lambda_v))
    return TQ_ERR_INVALID_ARG;
  DecodeArgs a;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &a.plan,
                        rot.srft ? PlanKind::kSrft
                        : rot.cb_bits ? PlanKind::kCodebook
                                      : PlanKind::kInt4))
    return TQ_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < a.plan.ws_bytes) return TQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return TQ_ERR_INVALID_ARG;
  // Test hooks (tq_set_test_hooks; off in normal use): fail the call as a failed launch
  // would, before anything is enqueued; or make the tensor-core decode's bounded waits for
  // its first copies run out (its outputs are then NaN).
  const unsigned hooks = g_test_hooks.load(std::memory_order_relaxed);
  if (hooks & TQ_TEST_HOOK_FAIL_LAUNCH) return cuda_status(cudaErrorLaunchFailure, where);
  a.test_starve = (hooks & TQ_TEST_HOOK_STARVE_PIPELINE) != 0;
  if (host_in != nullptr) {
    const cudaError_t e = move_host_inputs(*host_in, static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) return cuda_status(e, where);
    a.inputs_pending = host_in->gather;  // the tensor-core decode overlaps the gather kernel
  }
  a.q = q;
  a.q_bf16 = q_dtype == TQ_BF16;
  a.B = batch;
  a.Hq = num_q_heads;
  a.Hkv = num_kv_heads;
  a.d = head_dim;
  a.k_packed = k_packed;
  a.k_scales = k_scales;
  a.v_packed = v_packed;
  a.v_scales = v_scales;
  a.capacity = capacity;
  a.ctx_lens = ctx_lens;
  a.max_ctx = max_ctx;
  a.signs = signs;
  a.attn_scale = attn_scale;
  a.out = out;
  a.workspace = workspace;
  a.k_new = nullptr;
  a.v_new = nullptr;
  a.kv_bf16 = kv_dtype == TQ_BF16;
  a.lse = lse;
  a.lambda_k = rot.lambda_k;
  a.lambda_v = rot.lambda_v;
  a.cb_bits = rot.cb_bits;
  a.levels = rot.levels;
  a.cb_uniform = rot.cb_uniform ? 1 : 0;
  a.q_rot = rot.srft ? reinterpret_cast<const float*>(static_cast<unsigned char*>(workspace) +
                                                      a.plan.qrot_offset)
                     : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const bool mma = rot.cb_bits ? decode_mma_cb_supported(head_dim, num_q_heads / num_kv_heads)
                               : decode_mma_supported(head_dim, num_q_heads / num_kv_heads);
  if (append && mma && !rot.srft) {  // the decode kernel quantizes the new tokens itself
    a.k_new = k_new;
    a.v_new = v_new;
  } else if (append && rot.srft) {  // new tokens and query rotation in one launch
    QuantizeArgs qa;
    qa.k = k_new;
    qa.v = v_new;
    qa.bf16 = kv_dtype == TQ_BF16;
    qa.B = batch;
    qa.Hkv = num_kv_heads;
    qa.n_new = 1;
    qa.d = head_dim;
    qa.pos = ctx_lens;
    qa.pos_is_ctx = 1;
    qa.max_ctx = max_ctx;
    qa.signs = signs;
    qa.k_packed = const_cast<uint8_t*>(k_packed);
    qa.k_scales = const_cast<float*>(k_scales);
    qa.v_packed = const_cast<uint8_t*>(v_packed);
    qa.v_scales = const_cast<float*>(v_scales);
    qa.capacity = capacity;
    qa.lambda_k = rot.lambda_k;
    qa.lambda_v = rot.lambda_v;
    const cudaError_t e = launch_srft_prep(qa, a, s);
    if (e != cudaSuccess) return cuda_status(e, where);
    a.q_rot_overlap = 2;
  } else if (append) {  // the CUDA-core decode: one small-append launch first
    QuantizeArgs qa;
    qa.k = k_new;
    qa.v = v_new;
    qa.bf16 = kv_dtype == TQ_BF16;
    qa.B = batch;
    qa.Hkv = num_kv_heads;
    qa.n_new = 1;
    qa.d = head_dim;
    qa.pos = ctx_lens;
    qa.pos_is_ctx = 1;
    qa.max_ctx = max_ctx;
    qa.signs = signs;
    qa.k_packed = const_cast<uint8_t*>(k_packed);
    qa.k_scales = const_cast<float*>(k_scales);
    qa.v_packed = const_cast<uint8_t*>(v_packed);
    qa.v_scales = const_cast<float*>(v_scales);
    qa.capacity = capacity;
    qa.lambda_k = rot.lambda_k;
    qa.lambda_v = rot.lambda_v;
    qa.cb_bits = rot.cb_bits;
    qa.levels = rot.levels;
    qa.cb_uniform = rot.cb_uniform ? 1 : 0;
    const cudaError_t e = rot.srft ? launch_quantize_srft(qa, s)
                          : rot.cb_bits ? launch_quantize_cb(qa, s)
                                        : launch_quantize(qa, s);
    if (e != cudaSuccess) return cuda_status(e, where);
  }
  if (rot.srft && !append) {  // rotated queries into the workspace, read by the decode kernel
    a.q_rot_overlap = 1;         // the rotation writes no cache rows: the decode may overlap it
    const cudaError_t e = launch_srft_query(a, s);
    if (e != cudaSuccess) return cuda_status(e, where);
  }
  const bool tc = rot.cb_bits == 0 && decode_tc_supported(head_dim, num_q_heads / num_kv_heads) &&
                  (hooks & TQ_TEST_HOOK_TCGEN05_DECODE);
  const cudaError_t e = tc ? launch_decode_tc(a, s) : mma ? launch_decode_mma(a, s) : launch_decode_simt(a, s);
  if (e != cudaSuccess) return cuda_status(e, where);
  return cuda_status(rot.srft ? launch_merge_srft(a, s) : launch_merge(a, s), where);
}

extern "C" {

tq_status tq_sdpa_int4_decode(const void* q, tq_dtype q_dtype, int32_t batch,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t group, const uint8_t* k_packed, const float* k_scales,
                              const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                              const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                              float attn_scale, float* out, void* workspace,
                              size_t workspace_bytes, void* cuda_stream) {
  return decode_impl(q, q_dtype, nullptr, nullptr, TQ_F32, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_int4_decode");
}

tq_status tq_sdpa_int4_decode_lse(const void* q, tq_dtype q_dtype, int32_t batch,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t group, const uint8_t* k_packed, const float* k_scales,
                                  const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                                  const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                                  float attn_scale, float* out, float* lse, void* workspace,
                                  size_t workspace_bytes, void* cuda_stream) {
  if (!lse) return TQ_ERR_INVALID_ARG;
  return decode_impl(q, q_dtype, nullptr, nullptr, TQ_F32, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_int4_decode_lse", lse);
}

tq_status tq_merge_lse(const float* outs, const float* lses, int32_t n_parts, int32_t batch,
                       int32_t num_q_heads, int32_t head_dim, float* out, void* cuda_stream) {
  if (!outs || !lses || !out) return TQ_ERR_INVALID_ARG;
  if (n_parts < 1 || batch < 1 || num_q_heads < 1 || head_dim < 1) return TQ_ERR_INVALID_ARG;
  if (!srft_head_dim_supported(head_dim)) return TQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(lses) & 7u) || !aligned16(outs) || !aligned16(out))
    return TQ_ERR_INVALID_ARG;
  return cuda_status(launch_merge_lse(outs, lses, n_parts, (int64_t)batch * num_q_heads, head_dim,
                                      out, static_cast<cudaStream_t>(cuda_stream)),
                     "tq_merge_lse");
}

tq_status tq_sdpa_int4_decode_srft(const void* q, tq_dtype q_dtype, int32_t batch,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t group, const uint8_t* k_packed, const float* k_scales,
                                   const uint8_t* v_packed, const float* v_scales,
                                   int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx,
                                   const int8_t* signs, const float* lambda_k,
                                   const float* lambda_v, float attn_scale, float* out,
                                   void* workspace, size_t workspace_bytes, void* cuda_stream) {
  return decode_impl(q, q_dtype, nullptr, nullptr, TQ_F32, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_int4_decode_srft", nullptr, Rotation{true, lambda_k, lambda_v});
}

tq_status tq_sdpa_int4_decode_append_srft(
    const void* q, tq_dtype q_dtype, const void* k_new, const void* v_new, tq_dtype kv_dtype,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t group,
    uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales, int64_t capacity,
    const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs, const float* lambda_k,
    const float* lambda_v, float attn_scale, float* out, void* workspace, size_t workspace_bytes,
    void* cuda_stream) {
  if (!k_new || !v_new) return TQ_ERR_INVALID_ARG;
  return decode_impl(q, q_dtype, k_new, v_new, kv_dtype, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_int4_decode_append_srft", nullptr, Rotation{true, lambda_k, lambda_v});
}

tq_status tq_sdpa_cb_decode(const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t group, int32_t bits,
                           const float* levels, const uint8_t* k_packed, const float* k_scales,
                           const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                           const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                           float attn_scale, float* out, void* workspace, size_t workspace_bytes,
                           void* cuda_stream) {
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  return decode_impl(q, q_dtype, nullptr, nullptr, TQ_F32, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_cb_decode", nullptr, r);
}

tq_status tq_sdpa_int4_decode_srft_lse(const void* q, tq_dtype q_dtype, int32_t batch,
                                       int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                       int32_t group, const uint8_t* k_packed,
                                       const float* k_scales, const uint8_t* v_packed,
                                       const float* v_scales, int64_t capacity,
                                       const int32_t* ctx_lens, int32_t max_ctx,
                                       const int8_t* signs, const float* lambda_k,
                                       const float* lambda_v, float attn_scale, float* out,
                                       float* lse, void* workspace, size_t workspace_bytes,
                                       void* cuda_stream) {
  if (!lse) return TQ_ERR_INVALID_ARG;
  return decode_impl(q, q_dtype, nullptr, nullptr, TQ_F32, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_int4_decode_srft_lse", lse, Rotation{true, lambda_k, lambda_v});
}

tq_status tq_sdpa_cb_decode_lse(const void* q, tq_dtype q_dtype, int32_t batch,
                                int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t group, int32_t bits, const float* levels,
                                const uint8_t* k_packed, const float* k_scales,
                                const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                                const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                                float attn_scale, float* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* cuda_stream) {
  if (!lse) return TQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  return decode_impl(q, q_dtype, nullptr, nullptr, TQ_F32, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_cb_decode_lse", lse, r);
}

tq_status tq_sdpa_uniform_decode_append(const void* q, tq_dtype q_dtype, const void* k_new,
                                        const void* v_new, tq_dtype kv_dtype, int32_t batch,
                                        int32_t num_q_heads, int32_t num_kv_heads,
                                        int32_t head_dim, int32_t group, int32_t bits,
                                        const float* levels, uint8_t* k_packed, float* k_scales,
                                        uint8_t* v_packed, float* v_scales, int64_t capacity,
                                        const int32_t* ctx_lens, int32_t max_ctx,
                                        const int8_t* signs, float attn_scale, float* out,
                                        void* workspace, size_t workspace_bytes,
                                        void* cuda_stream) {
  if (!k_new || !v_new || !levels) return TQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  r.cb_uniform = true;
  return decode_impl(q, q_dtype, k_new, v_new, kv_dtype, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_uniform_decode_append", nullptr, r);
}

tq_status tq_sdpa_cb_decode_append(const void* q, tq_dtype q_dtype, const void* k_new,
                                   const void* v_new, tq_dtype kv_dtype, int32_t batch,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t group, int32_t bits, const float* levels,
                                   uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                                   float* v_scales, int64_t capacity, const int32_t* ctx_lens,
                                   int32_t max_ctx, const int8_t* signs, float attn_scale,
                                   float* out, void* workspace, size_t workspace_bytes,
                                   void* cuda_stream) {
  if (!k_new || !v_new) return TQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  return decode_impl(q, q_dtype, k_new, v_new, kv_dtype, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_cb_decode_append", nullptr, r);
}

// Device staging of the host-buffer step call, after the decode workspace:
// q [B][Hq][d], k_new and v_new [B][Hkv][d], out [B][Hq][d] (each 256-byte aligned).
struct HostStaging {
  size_t q, k, v, out, total;
};

static bool host_staging(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t max_ctx, tq_dtype q_dtype, tq_dtype kv_dtype,
                         PlanKind kind, HostStaging* hs) {
  DecodePlan p;
  if (!make_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, &p, kind))
    return false;
  if ((q_dtype != TQ_F32 && q_dtype != TQ_BF16) || (kv_dtype != TQ_F32 && kv_dtype != TQ_BF16))
    return false;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t qb = (size_t)batch * num_q_heads * head_dim * (q_dtype == TQ_BF16 ? 2 : 4);
  const size_t kb = (size_t)batch * num_kv_heads * head_dim * (kv_dtype == TQ_BF16 ? 2 : 4);
  hs->q = up(p.ws_bytes);
  hs->k = hs->q + up(qb);
  hs->v = hs->k + up(kb);
  hs->out = hs->v + up(kb);
  hs->total = hs->out + (size_t)batch * num_q_heads * head_dim * 4;
  return true;
}

size_t tq_decode_append_host_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                             int32_t num_kv_heads, int32_t head_dim,
                                             int32_t max_ctx, tq_dtype q_dtype,
                                             tq_dtype kv_dtype) {
  HostStaging hs;
  if (!host_staging(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, q_dtype, kv_dtype,
                    PlanKind::kInt4, &hs))
    return 0;
  return hs.total;
}

size_t tq_decode_append_host_srft_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                                  int32_t num_kv_heads, int32_t head_dim,
                                                  int32_t max_ctx, tq_dtype q_dtype,
                                                  tq_dtype kv_dtype) {
  HostStaging hs;
  if (!host_staging(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, q_dtype, kv_dtype,
                    PlanKind::kSrft, &hs))
    return 0;
  return hs.total;
}

size_t tq_decode_append_host_cb_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                                int32_t num_kv_heads, int32_t head_dim,
                                                int32_t max_ctx, tq_dtype q_dtype,
                                                tq_dtype kv_dtype) {
  HostStaging hs;
  if (head_dim != 128 && head_dim != 256) return 0;
  if (!host_staging(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, q_dtype, kv_dtype,
                    PlanKind::kCodebook, &hs))
    return 0;
  return hs.total;
}

}  // extern "C"

// Copies the step's inputs from mapped host memory into the workspace's
// staging space: byte ranges that start 16-byte aligned and are multiples of
// 16 bytes long, as 16-byte loads spread over the grid, so each input crosses
// the bus once, in full coalesced requests (the decode then reads it from
// device memory: every CTA of a kv head reads its queries).
__global__ void host_gather_kernel(const uint4* q, uint4* dq, int64_t nq, const uint4* k, uint4* dk,
                                   const uint4* v, uint4* dv, int64_t nkv) {
  // the tensor-core decode may start streaming the cache now; it waits for
  // this grid before it reads q, k_new and v_new
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nq; i += stride) dq[i] = q[i];
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nkv; i += stride) {
    dk[i] = k[i];
    dv[i] = v[i];
  }
}

// The device address of a host buffer that kernels can access directly
// (page-locked and mapped under unified addressing) when it is 16-byte
// aligned there, else nullptr.
static void* device_view(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // clear the query's error
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) return nullptr;
  return aligned16(at.devicePointer) ? at.devicePointer : nullptr;
}

extern "C" {

}  // extern "C"

// The fused step with its inputs and output in host memory, for every cache
// format (rot): mapped host buffers through the gather kernel and direct
// output writes, else staging copies (see include/tq.h).
static tq_status host_step(const void* q_host, tq_dtype q_dtype, const void* k_new_host,
                           const void* v_new_host, tq_dtype kv_dtype, int32_t batch,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                           int32_t group, uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                           float* v_scales, int64_t capacity, const int32_t* ctx_lens,
                           int32_t max_ctx, const int8_t* signs, float attn_scale,
                           float* out_host, void* workspace, size_t workspace_bytes,
                           void* cuda_stream, const char* where, const Rotation& rot) {
  if (!q_host || !k_new_host || !v_new_host || !out_host) return TQ_ERR_INVALID_ARG;
  const PlanKind kind = rot.srft ? PlanKind::kSrft
                        : rot.cb_bits ? PlanKind::kCodebook
                                      : PlanKind::kInt4;
  HostStaging hs;
  if ((kind == PlanKind::kCodebook && head_dim != 128 && head_dim != 256) ||
      !host_staging(batch, num_q_heads, num_kv_heads, head_dim, max_ctx, q_dtype, kv_dtype, kind,
                    &hs)) {
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
    if (kv_dtype != TQ_F32 && kv_dtype != TQ_BF16) return TQ_ERR_INVALID_ARG;
    if (!head_dim_ok(head_dim, rot)) return TQ_ERR_UNSUPPORTED;
    return TQ_ERR_INVALID_ARG;
  }
  if (!workspace || workspace_bytes < hs.total) return TQ_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const size_t q_bytes = (size_t)batch * num_q_heads * head_dim * (q_dtype == TQ_BF16 ? 2 : 4);
  const size_t kv_bytes = (size_t)batch * num_kv_heads * head_dim * (kv_dtype == TQ_BF16 ? 2 : 4);
  const size_t out_bytes = (size_t)batch * num_q_heads * head_dim * 4;
  // mapped host buffers: one small kernel gathers the inputs into the staging
  // space and the merge writes the output into out_host, no copies
  const void* dq = device_view(q_host);
  const void* dk = device_view(k_new_host);
  const void* dv = device_view(v_new_host);
  void* dout = device_view(out_host);
  const bool mapped = dq && dk && dv && dout && q_bytes % 16 == 0 && kv_bytes % 16 == 0;
  HostInputs hin;
  hin.gather = mapped;
  hin.q = mapped ? dq : q_host;
  hin.k = mapped ? dk : k_new_host;
  hin.v = mapped ? dv : v_new_host;
  hin.dq = ws + hs.q;
  hin.dk = ws + hs.k;
  hin.dv = ws + hs.v;
  hin.q_bytes = q_bytes;
  hin.kv_bytes = kv_bytes;
  const tq_status st = decode_impl(
      ws + hs.q, q_dtype, ws + hs.k, ws + hs.v, kv_dtype, batch, num_q_heads, num_kv_heads,
      head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens, max_ctx, signs,
      attn_scale, mapped ? static_cast<float*>(dout) : reinterpret_cast<float*>(ws + hs.out),
      workspace, hs.q, cuda_stream, where, nullptr, rot, &hin);
  if (st != TQ_OK || mapped) return st;
  return cuda_status(cudaMemcpyAsync(out_host, ws + hs.out, out_bytes, cudaMemcpyDeviceToHost, s),
                     where);
}

extern "C" {

tq_status tq_sdpa_int4_decode_append_host(const void* q_host, tq_dtype q_dtype,
                                          const void* k_new_host, const void* v_new_host,
                                          tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads,
                                          int32_t num_kv_heads, int32_t head_dim, int32_t group,
                                          uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                                          float* v_scales, int64_t capacity,
                                          const int32_t* ctx_lens, int32_t max_ctx,
                                          const int8_t* signs, float attn_scale, float* out_host,
                                          void* workspace, size_t workspace_bytes,
                                          void* cuda_stream) {
  return host_step(q_host, q_dtype, k_new_host, v_new_host, kv_dtype, batch, num_q_heads,
                   num_kv_heads, head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity,
                   ctx_lens, max_ctx, signs, attn_scale, out_host, workspace, workspace_bytes,
                   cuda_stream, "tq_sdpa_int4_decode_append_host", Rotation{});
}

tq_status tq_sdpa_int4_decode_append_srft_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales,
    int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
    const float* lambda_k, const float* lambda_v, float attn_scale, float* out_host,
    void* workspace, size_t workspace_bytes, void* cuda_stream) {
  Rotation r;
  r.srft = true;
  r.lambda_k = lambda_k;
  r.lambda_v = lambda_v;
  return host_step(q_host, q_dtype, k_new_host, v_new_host, kv_dtype, batch, num_q_heads,
                   num_kv_heads, head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity,
                   ctx_lens, max_ctx, signs, attn_scale, out_host, workspace, workspace_bytes,
                   cuda_stream, "tq_sdpa_int4_decode_append_srft_host", r);
}

tq_status tq_sdpa_uniform_decode_append_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, int32_t bits, const float* levels, uint8_t* k_packed, float* k_scales,
    uint8_t* v_packed, float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out_host, void* workspace,
    size_t workspace_bytes, void* cuda_stream) {
  if (!levels) return TQ_ERR_INVALID_ARG;
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  r.cb_uniform = true;
  return host_step(q_host, q_dtype, k_new_host, v_new_host, kv_dtype, batch, num_q_heads,
                   num_kv_heads, head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity,
                   ctx_lens, max_ctx, signs, attn_scale, out_host, workspace, workspace_bytes,
                   cuda_stream, "tq_sdpa_uniform_decode_append_host", r);
}

tq_status tq_sdpa_cb_decode_append_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, int32_t bits, const float* levels, uint8_t* k_packed, float* k_scales,
    uint8_t* v_packed, float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out_host, void* workspace,
    size_t workspace_bytes, void* cuda_stream) {
  Rotation r;
  r.cb_bits = bits;
  r.levels = levels;
  if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
  return host_step(q_host, q_dtype, k_new_host, v_new_host, kv_dtype, batch, num_q_heads,
                   num_kv_heads, head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity,
                   ctx_lens, max_ctx, signs, attn_scale, out_host, workspace, workspace_bytes,
                   cuda_stream, "tq_sdpa_cb_decode_append_host", r);
}

tq_status tq_sdpa_int4_decode_append(const void* q, tq_dtype q_dtype, const void* k_new,
                                     const void* v_new, tq_dtype kv_dtype, int32_t batch,
                                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t group, uint8_t* k_packed, float* k_scales,
                                     uint8_t* v_packed, float* v_scales, int64_t capacity,
                                     const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                                     float attn_scale, float* out, void* workspace,
                                     size_t workspace_bytes, void* cuda_stream) {
  if (!k_new || !v_new) return TQ_ERR_INVALID_ARG;
  return decode_impl(q, q_dtype, k_new, v_new, kv_dtype, batch, num_q_heads, num_kv_heads,
                     head_dim, group, k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens,
                     max_ctx, signs, attn_scale, out, workspace, workspace_bytes, cuda_stream,
                     "tq_sdpa_int4_decode_append");
}

}  // extern "C"
