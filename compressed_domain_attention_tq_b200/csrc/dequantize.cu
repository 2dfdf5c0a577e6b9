// dequantize.cu -- packed int4 rows -> dequantized values (scale * code), in
// the rotated basis of the cache.  A utility beside the decode path (which
// never forms these values): one thread per packed 32-bit word.
//
// Row layout (see tq.h): coordinate i = 32 g + j of a row sits in byte
// (j/4)*(2*ng) + 2g + (j%4)/2, low nibble for even j.  A 32-bit word w of a row
// therefore holds sub-block s = 4w / (2 ng) of two groups g0 = (4w mod 2 ng)/2
// and g0 + 1: its 16-bit half k carries coordinates 32 (g0 + k) + 4 s + n in
// nibble n (n = 0..3).
#include <cuda_bf16.h>

#include "tq_internal.h"

namespace tq {
namespace {

template <int D, bool BF16>
__global__ void __launch_bounds__(256) dequantize_kernel(DequantizeArgs a) {
  constexpr int NG = D / 32, WPR = D / 8;  // groups, packed words per row
  const int64_t total = (int64_t)a.n_seq * a.rows * WPR;
  for (int64_t gw = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gw < total;
       gw += (int64_t)gridDim.x * blockDim.x) {
    const int wi = (int)(gw % WPR);
    const int64_t rr = gw / WPR;                 // output row
    const int64_t seq = rr / a.rows, r = rr % a.rows;
    const int64_t src_row = seq * a.row_stride + r;
    const uint32_t word = reinterpret_cast<const uint32_t*>(a.packed + src_row * (D / 2))[wi];
    const int s = (4 * wi) / (2 * NG), g0 = ((4 * wi) % (2 * NG)) / 2;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int g = g0 + k;
      const float sc = a.scales[src_row * NG + g];
      float v[4];
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const int code = ((int)((word >> (16 * k + 4 * n)) & 0xFu) ^ 8) - 8;  // sign-extend
        v[n] = sc * (float)code;
      }
      const int64_t o = rr * D + 32 * g + 4 * s;
      if (BF16) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + o;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out) = pk;
      } else {
        *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) = make_float4(v[0], v[1], v[2], v[3]);
      }
    }
  }
}

template <int D, bool BF16>
cudaError_t launch_dq(const DequantizeArgs& a, cudaStream_t stream) {
  const int64_t total = (int64_t)a.n_seq * a.rows * (D / 8);
  int dev = 0, sms = kSmCount;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (total + 255) / 256;
  if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
  dequantize_kernel<D, BF16><<<(unsigned)blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequantize(const DequantizeArgs& a, cudaStream_t stream) {
  if (a.d == 128) return a.bf16 ? launch_dq<128, true>(a, stream) : launch_dq<128, false>(a, stream);
  return a.bf16 ? launch_dq<256, true>(a, stream) : launch_dq<256, false>(a, stream);
}

}  // namespace tq
