// srft.cuh -- one warp computes the orthonormal discrete Hartley transform
//   (F x)[k] = sum_j x[j] cas(2 pi k j / d) / sqrt(d),  cas = cos + sin,
// of two real d-vectors at once (d = 32 M, M = 1 .. 8).  This is the SRFT
// variant's rotation (SRFT post, core method: a sign-randomized Fourier
// transform in place of the Hadamard one, with a mixed-radix structure that
// suits widths that are not powers of two).
//
// Method: the two real inputs x, y form one complex vector z = x + i y, whose
// DFT Z = X + i Y is taken by a mixed-radix Cooley-Tukey step, d = 32 x M:
//   index j = lane + 32 j2 (lane < 32, j2 < M), k = k2 + M k1;
//   A. an M-point DFT inside each lane over its j2 (no communication);
//   B. a twiddle exp(-2 pi i lane k2 / d);
//   C. a 32-point radix-2 decimation-in-frequency FFT across the lanes by
//      shuffles, which leaves Z[k2 + M k1] in lane brev5(k1).
// The real transforms follow from the Hermitian symmetry of X and Y:
//   H_x[k] = (Re Z[k] + Re Z[d-k] - Im Z[k] + Im Z[d-k]) / 2
//   H_y[k] = (Im Z[k] + Im Z[d-k] + Re Z[k] - Re Z[d-k]) / 2
// (H = Re X - Im X for the e^{-i} DFT), where Z[d-k] sits in lane lane ^ 31,
// slot M - k2 (k2 > 0), or in lane brev5((32 - k1) mod 32), slot 0 (k2 = 0).
// Twiddles are computed once per warp in double (three sincospi calls per
// lane, the rest as exact powers and squares) and rounded to fp32; the
// transform's arithmetic is fp32.
// Each input is first scaled by a power of two that brings its largest
// magnitude into [0.5, 1), and its transform scaled back (both exact): the
// rounding error a transform of z leaves in X and Y is relative to |z|, so
// without this a vector much smaller than its partner (a token whose V is
// orders of magnitude below its K, say) would lose its precision.
#pragma once
#include <math.h>
#include <stdint.h>

namespace tq {

__device__ __forceinline__ int brev5(int x) { return (int)(__brev((unsigned)x) >> 27); }

template <int M>
struct HartleyTwiddles {
  float2 wm[M];  // exp(-2 pi i t / M), t < M
  float2 wb[M];  // exp(-2 pi i lane k2 / d), k2 < M
  float2 wc[5];  // radix-2 stage with half-size h = 16 >> s: exp(-2 pi i (lane mod h) / 2h)
                 // for lanes with bit h set, 1 for the others
  float sg[5];   // -1 for lanes with bit h set (they keep partner - own), +1 otherwise
  int src0;      // lane holding Z[d - k] for this lane's slot 0
};

// exp(-2 pi i num / den) in double
__device__ __forceinline__ double2 cis_neg(int num, int den) {
  double s, c;
  sincospi(2.0 * (double)num / (double)den, &s, &c);
  return make_double2(c, -s);
}

__device__ __forceinline__ double2 cmul_d(double2 a, double2 b) {
  return make_double2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

__device__ __forceinline__ float2 to_f2(double2 a) { return make_float2((float)a.x, (float)a.y); }

template <int M>
__device__ __forceinline__ void hartley_twiddles(HartleyTwiddles<M>& tw, int lane) {
  constexpr int D = 32 * M;
  // powers of exp(-2 pi i / M) and of exp(-2 pi i lane / d)
  const double2 bm = cis_neg(1, M), bb = cis_neg(lane, D);
  double2 pm = make_double2(1.0, 0.0), pb = make_double2(1.0, 0.0);
#pragma unroll
  for (int t = 0; t < M; ++t) {
    tw.wm[t] = to_f2(pm);
    tw.wb[t] = to_f2(pb);
    pm = cmul_d(pm, bm);
    pb = cmul_d(pb, bb);
  }
  // radix-2 stages: a_s = exp(-2 pi i u_s / 32) with u_s = (lane mod h) 2^s, h = 16 >> s;
  // u_{s+1} = 2 u_s - 16 b (b: bit 3 - s of lane), so a_{s+1} = a_s^2 (-1)^b
  double2 a = cis_neg(lane & 15, 32);
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int h = 16 >> s;
    const bool upper = (lane & h) != 0;
    tw.wc[s] = upper ? to_f2(a) : make_float2(1.0f, 0.0f);
    tw.sg[s] = upper ? -1.0f : 1.0f;
    if (s < 4) {
      a = cmul_d(a, a);
      if ((lane >> (3 - s)) & 1) a = make_double2(-a.x, -a.y);
    }
  }
  tw.src0 = brev5((32 - brev5(lane)) & 31);
}

// In: re[j2] = x[lane + 32 j2], im[j2] = y[lane + 32 j2].
// Out: hx[k2] = 2 sqrt(d) (F x)[k], hy[k2] = 2 sqrt(d) (F y)[k] for
// k = k2 + M brev5(lane); the caller applies the factor 1 / (2 sqrt(d)).
template <int M>
__device__ __forceinline__ void hartley_pair_warp(const float (&re_in)[M], const float (&im_in)[M],
                                                  const HartleyTwiddles<M>& tw, float (&hx)[M],
                                                  float (&hy)[M]) {
  // power-of-two normalization of each input (see above)
  float mx = 0.0f, my = 0.0f;
#pragma unroll
  for (int j2 = 0; j2 < M; ++j2) {
    mx = fmaxf(mx, fabsf(re_in[j2]));
    my = fmaxf(my, fabsf(im_in[j2]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, o));
  }
  int ex = 0, ey = 0;
  if (mx > 0.0f) frexpf(mx, &ex);
  if (my > 0.0f) frexpf(my, &ey);
  // multiplying by 2^-e and 2^e is what ldexpf computes (both are correctly
  // rounded); the float powers are exact while e stays in [-126, 126]
  const bool fast = ex >= -126 && ex <= 126 && ey >= -126 && ey <= 126;  // warp-uniform
  const float sxi = __int_as_float((127 - (fast ? ex : 0)) << 23);
  const float syi = __int_as_float((127 - (fast ? ey : 0)) << 23);
  float re[M], im[M];
#pragma unroll
  for (int j2 = 0; j2 < M; ++j2) {
    re[j2] = fast ? re_in[j2] * sxi : ldexpf(re_in[j2], -ex);
    im[j2] = fast ? im_in[j2] * syi : ldexpf(im_in[j2], -ey);
  }
  float ar[M], ai[M];
  // A: M-point DFT within the lane
#pragma unroll
  for (int k2 = 0; k2 < M; ++k2) {
    float sr = 0.0f, si = 0.0f;
#pragma unroll
    for (int j2 = 0; j2 < M; ++j2) {
      const float2 w = tw.wm[(j2 * k2) % M];
      sr = fmaf(re[j2], w.x, fmaf(-im[j2], w.y, sr));
      si = fmaf(re[j2], w.y, fmaf(im[j2], w.x, si));
    }
    ar[k2] = sr;
    ai[k2] = si;
  }
  // B: twiddles
#pragma unroll
  for (int k2 = 1; k2 < M; ++k2) {
    const float2 w = tw.wb[k2];
    const float r = ar[k2], i = ai[k2];
    ar[k2] = fmaf(r, w.x, -i * w.y);
    ai[k2] = fmaf(r, w.y, i * w.x);
  }
  // C: 32-point radix-2 DIF across the lanes: lower lane a + b, upper lane (a - b) w
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int h = 16 >> s;
    const float2 w = tw.wc[s];
    const float sg = tw.sg[s];
#pragma unroll
    for (int k2 = 0; k2 < M; ++k2) {
      const float pr = __shfl_xor_sync(0xffffffffu, ar[k2], h);
      const float pi = __shfl_xor_sync(0xffffffffu, ai[k2], h);
      const float tr = fmaf(sg, ar[k2], pr), ti = fmaf(sg, ai[k2], pi);
      ar[k2] = fmaf(tr, w.x, -ti * w.y);
      ai[k2] = fmaf(tr, w.y, ti * w.x);
    }
  }
  // Hartley transforms of x and y from Z[k] and Z[d - k]
#pragma unroll
  for (int k2 = 0; k2 < M; ++k2) {
    float qr, qi;
    if (k2 == 0) {
      qr = __shfl_sync(0xffffffffu, ar[0], tw.src0);
      qi = __shfl_sync(0xffffffffu, ai[0], tw.src0);
    } else {
      qr = __shfl_xor_sync(0xffffffffu, ar[M - k2], 31);
      qi = __shfl_xor_sync(0xffffffffu, ai[M - k2], 31);
    }
    // an all-zero input's transform is exactly zero (not its partner's rounding residue)
    const float vx = (ar[k2] + qr) + (qi - ai[k2]), vy = (ai[k2] + qi) + (ar[k2] - qr);
    if (fast) {
      hx[k2] = mx > 0.0f ? vx * __int_as_float((127 + ex) << 23) : 0.0f;
      hy[k2] = my > 0.0f ? vy * __int_as_float((127 + ey) << 23) : 0.0f;
    } else {
      hx[k2] = mx > 0.0f ? ldexpf(vx, ex) : 0.0f;
      hy[k2] = my > 0.0f ? ldexpf(vy, ey) : 0.0f;
    }
  }
}

}  // namespace tq
