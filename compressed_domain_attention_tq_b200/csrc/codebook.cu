// codebook.cu -- the codebook variant of the cache (AdapTQ post: 2-, 3- and
// 4-bit indices into a Max-Lloyd codebook, +-3 sigma clipping, dot products
// on the packed indices through lookup tables; int2 is Open-TQ-Metal's future
// work).  Per group of 32 rotated coordinates:
//   sigma = fl32(sqrt(S / 32)), S = sum y^2 accumulated in fp64
//   u     = clamp(fl32(y / sigma), -3, 3)          (u = 0 when sigma = 0)
//   index = #{ i : u > t_i },  t_i = fl32(fl32(C_i + C_{i+1}) * 0.5)
// and the value is sigma * C[index].  A row holds its groups in order, each in
// 4 * bits bytes; index j of a group occupies bits bits*j .. bits*j + bits - 1
// of the group's little-endian bit string.
//
// Here: the quantize-append kernel (one warp per vector: cb_vector.cuh) and the
// host-side Gaussian Max-Lloyd generator.  The decode is decode_mma.cu's
// tensor-core kernel (5..8 query heads per kv head, d = 128) or decode_simt.cu's
// kernel, both instantiated for the codebook formats.
#include <math.h>
#include <stdint.h>

#include "cb_vector.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

template <int D, int BITS>
__global__ void __launch_bounds__(128) cb_quantize_kernel(QuantizeArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t per_kv = (int64_t)a.B * a.Hkv * a.n_new;
  const int64_t vec = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (vec >= 2 * per_kv) return;  // the whole warp
  const int kv = (int)(vec / per_kv);
  const int64_t rem = vec % per_kv;
  const int64_t bh = rem / a.n_new, n = rem % a.n_new;
  const int b = (int)(bh / a.Hkv);
  int64_t p = (int64_t)a.pos[b] + n;
  if (a.pos_is_ctx) p = (int64_t)min(max(a.pos[b], 1), a.max_ctx) - 1 + n;
  if (p < 0 || p >= a.capacity) return;  // the whole warp
  const int64_t row = bh * a.capacity + p;
  const int eb = a.bf16 ? 2 : 4;
  cb_quantize_vector_warp<D, BITS>(static_cast<const unsigned char*>(kv ? a.v : a.k) + rem * D * eb,
                                   a.bf16, a.signs, a.levels,
                                   (kv ? a.v_packed : a.k_packed) + row * (D * BITS / 8),
                                   (kv ? a.v_scales : a.k_scales) + row * (D / 32), lane,
                                   a.cb_uniform != 0);
}

template <int D, int BITS>
cudaError_t launch_cb_q(const QuantizeArgs& a, cudaStream_t stream) {
  const int64_t nvec = 2LL * a.B * a.Hkv * a.n_new;
  cb_quantize_kernel<D, BITS><<<(unsigned)((nvec + 3) / 4), 128, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_cb_q_d(const QuantizeArgs& a, cudaStream_t stream) {
  switch (a.cb_bits) {
    case 2: return launch_cb_q<D, 2>(a, stream);
    case 3: return launch_cb_q<D, 3>(a, stream);
    case 4: return launch_cb_q<D, 4>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

double normal_pdf(double x) { return exp(-0.5 * x * x) * 0.3989422804014327; }
double normal_cdf(double x) { return 0.5 * erfc(-x * 0.7071067811865476); }

}  // namespace

cudaError_t launch_quantize_cb(const QuantizeArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_cb_q_d<128>(a, stream) : launch_cb_q_d<256>(a, stream);
}

// Gaussian Max-Lloyd codebook: start from the cell centres of equal-probability
// cells (inverse normal cdf by bisection), then alternate thresholds at the
// midpoints of the levels and levels at the N(0,1) means of their cells,
//   mean over (a, b) = (pdf(a) - pdf(b)) / (cdf(b) - cdf(a)),
// until no level moves by more than 1e-15.
void lloyd_max_gaussian(int bits, double* c) {
  const int L = 1 << bits;
  for (int i = 0; i < L; ++i) {
    const double pr = (i + 0.5) / L;
    double lo = -10.0, hi = 10.0;
    for (int it = 0; it < 200; ++it) {
      const double mid = 0.5 * (lo + hi);
      (normal_cdf(mid) < pr ? lo : hi) = mid;
    }
    c[i] = 0.5 * (lo + hi);
  }
  double t[256];
  for (int it = 0; it < 200000; ++it) {
    for (int i = 0; i + 1 < L; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
    double moved = 0.0;
    for (int i = 0; i < L; ++i) {
      const double pa = i == 0 ? 0.0 : normal_pdf(t[i - 1]);
      const double pb = i == L - 1 ? 0.0 : normal_pdf(t[i]);
      const double ca = i == 0 ? 0.0 : normal_cdf(t[i - 1]);
      const double cb = i == L - 1 ? 1.0 : normal_cdf(t[i]);
      const double m = (pa - pb) / (cb - ca);
      moved = fmax(moved, fabs(m - c[i]));
      c[i] = m;
    }
    if (moved < 1e-15) break;
  }
}

}  // namespace tq
