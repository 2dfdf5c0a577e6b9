// dequantize.cu -- packed int4 rows -> dequantized values (scale * code), in
// the rotated basis of the cache.  A utility beside the decode path (which
// never forms these values): one thread per packed 32-bit word.
//
// Row layout (see tq.h): coordinate i = 32 g + j of a row sits in byte
// (j/4)*(2*ng) + 2g + (j%4)/2, low nibble for even j.  The 16-bit half-word h
// of a row (bytes 2h, 2h + 1) therefore belongs to sub-block s = h / ng and
// group g = h mod ng, and carries coordinates 32 g + 4 s + n in nibble n
// (n = 0..3); a 32-bit word w holds half-words 2w and 2w + 1.
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
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int hw = 2 * wi + k, s = hw / NG, g = hw % NG;
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


template <int D>
cudaError_t launch_dq_d(const DequantizeArgs& a, cudaStream_t stream) {
  return a.bf16 ? launch_dq<D, true>(a, stream) : launch_dq<D, false>(a, stream);
}

}  // namespace

// head_dim: any multiple of 32 up to 256
cudaError_t launch_dequantize(const DequantizeArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 32: return launch_dq_d<32>(a, stream);
    case 64: return launch_dq_d<64>(a, stream);
    case 96: return launch_dq_d<96>(a, stream);
    case 128: return launch_dq_d<128>(a, stream);
    case 160: return launch_dq_d<160>(a, stream);
    case 192: return launch_dq_d<192>(a, stream);
    case 224: return launch_dq_d<224>(a, stream);
    case 256: return launch_dq_d<256>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tq
