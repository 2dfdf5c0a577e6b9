// decode_static_scratch.cu -- tq_sdpa_int4_decode_static_scratch, the decode
// call for callers that cannot allocate device memory.
//
// Its scratch is one file-scope __device__ array of TQ_STATIC_SCRATCH_BYTES,
// which every GPU that loads libtq holds until the process exits.  In host
// code the array's name is only a host-side stand-in, so its device address
// is looked up once per device with cudaGetSymbolAddress (with that device
// current) and cached; the decode then runs through tq_sdpa_int4_decode
// unchanged, with that address as its workspace.  Nothing here allocates.
#include <mutex>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace tq {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[TQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

// Device address of the scratch array on the current device (looked up on the
// first call for that device).  Returns TQ_OK and sets *out, or an error.
tq_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return TQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
  const size_t need =
      tq_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_ctx);
  if (need > (size_t)TQ_STATIC_SCRATCH_BYTES) return TQ_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (need != 0) {  // need == 0: invalid sizes, reported by the call below
    const tq_status st = tq::scratch_on_current_device(&scratch);
    if (st != TQ_OK) return st;
  }
  return tq_sdpa_int4_decode(q, q_dtype, batch, num_q_heads, num_kv_heads, head_dim, group,
                             k_packed, k_scales, v_packed, v_scales, capacity, ctx_lens, max_ctx,
                             signs, attn_scale, out, scratch, scratch ? TQ_STATIC_SCRATCH_BYTES : 0,
                             cuda_stream);
}

}  // extern "C"
