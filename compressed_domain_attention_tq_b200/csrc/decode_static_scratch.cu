// decode_static_scratch.cu -- tq_sdpa_int4_decode_static_scratch, the decode
// call for callers that cannot allocate device memory.
//
// Its scratch is one file-scope __device__ array of TQ_STATIC_SCRATCH_BYTES,
// which every GPU that loads libtq holds until the process exits.  In host
// code the array's name is only a host-side stand-in, so its device address
// is looked up with cudaGetSymbolAddress, with the calling thread's CUDA
// context current, the first time a call runs in that context, and kept per
// context (a device reset, or a context the caller creates with the driver
// API, loads the module again and gets its own array).  The decode then runs
// through tq_sdpa_int4_decode unchanged, with that address as its workspace.
// Nothing here allocates.
#include <mutex>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[TQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxContexts = 64;
struct Entry {
  unsigned long long ctx;  // context identity (0 = empty slot)
  void* addr;              // device address of g_decode_scratch in that context
};
std::mutex g_scratch_mu;
Entry g_scratch[kMaxContexts];
int g_scratch_next = 0;

// Device address of the scratch array in the calling thread's current context
// (looked up on the first call in that context).  Returns TQ_OK and sets
// *out, or an error.
tq_status scratch_in_current_context(void** out) {
  unsigned long long id = 0;
  if (!current_context_id(&id)) {
    // no context bound to this thread yet: the lookup below binds the device's
    // primary context (the runtime's usual behaviour), then the identity exists
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return TQ_ERR_CUDA;
    if (!current_context_id(&id)) return TQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  for (int i = 0; i < kMaxContexts; ++i)
    if (g_scratch[i].ctx == id) {
      *out = g_scratch[i].addr;
      return TQ_OK;
    }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return TQ_ERR_CUDA;
  g_scratch[g_scratch_next] = Entry{id, p};
  g_scratch_next = (g_scratch_next + 1) % kMaxContexts;
  *out = p;
  return TQ_OK;
}

}  // namespace
}  // namespace tq

extern "C" {

tq_status tq_sdpa_int4_decode_static_scratch(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, const uint8_t* k_packed, const float* k_scales,
    const uint8_t* v_packed, const float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out, void* cuda_stream) {
  // the arguments tq_sdpa_int4_decode would reject are reported as it would
  // report them; only then is the size checked against the array
  const tq_status st = tq::validate_decode_args(q, q_dtype, batch, num_q_heads, num_kv_heads, head_dim,
                                                group, k_packed, k_scales, v_packed, v_scales, capacity,
                                                ctx_lens, max_ctx, attn_scale, out);
  if (st != TQ_OK) return st;
  const size_t need =
      tq_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx);
  if (need > (size_t)TQ_STATIC_SCRATCH_BYTES) return TQ_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const tq_status sc = tq::scratch_in_current_context(&scratch);
  if (sc != TQ_OK) return sc;
  return tq_sdpa_int4_decode(q, q_dtype, batch, num_q_heads, num_kv_heads, head_dim, group,
                             k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens, max_ctx,
                             signs, attn_scale, out, scratch, TQ_STATIC_SCRATCH_BYTES, cuda_stream);
}

}  // extern "C"
