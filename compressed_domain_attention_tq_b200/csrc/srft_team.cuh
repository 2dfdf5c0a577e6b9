// srft_team.cuh -- the SRFT quantizer for d = 16 P (P = 8: d = 128; P = 16:
// d = 256), P lanes (a team) per K/V pair, 32 / P pairs per warp (SRFT post,
// core method: sign flip, Fourier-type transform, per-coordinate scale, then
// group abs-max int4 with the Hadamard path's packing).
//
// The transform is srft.cuh's: the orthonormal Hartley transforms of x = K
// and y = V from one complex DFT of z = x + i y, split by the Hermitian
// symmetry of the two real transforms.  Only the DFT's factorisation differs,
// d = 16 x P instead of 32 x M, so that most of it runs inside a lane:
//   index j = t + P j2 (team lane t < P, j2 < 16), k = k2 + 16 k1;
//   A. a 16-point radix-2 DFT inside each lane over its j2 (decimation in
//      frequency, results in bit-reversed register order);
//   B. a twiddle exp(-2 pi i t k2 / d);
//   C. a P-point radix-2 DFT across the team by shuffles, which leaves
//      Z[k2 + 16 k1] in team lane brev(k1).
// Each lane then owns 16 consecutive coordinates 16 k1 .. 16 k1 + 15, half of
// one quantization group (the other half is in lane t ^ P/2), so the scale
// and the codes come from registers and one shuffle.  As in srft.cuh each
// input is first scaled by a power of two that brings its largest magnitude
// into [0.5, 1) and its transform scaled back, an all-zero input gives an
// exactly zero transform, and the twiddles are computed in double and
// rounded to fp32 once.
#pragma once
#include <math.h>
#include <stdint.h>

#include "srft.cuh"

namespace tq {

template <int P>
struct TeamConsts {
  static constexpr int L = P == 8 ? 3 : 4;  // log2 P
  float2 wb[16];  // exp(-2 pi i t k2 / d), k2 < 16
  float2 wc[L];   // stage s (half-size h = P/2 >> s): exp(-2 pi i (t mod h) / 2h) for lanes with
                  // bit h set, 1 for the others
  float sg[L];    // -1 for lanes with bit h set (they keep partner - own), +1 otherwise
  int src0;       // team lane holding Z[d - 16 k1] (this lane's register 0 holds Z[16 k1])
};

template <int L>
__device__ __forceinline__ int brev_bits(int x) {
  return (int)(__brev((unsigned)x) >> (32 - L));
}

// 16 - k within 4 bits, in bit-reversed register order: register holding
// k2' = (16 - k2) mod 16 for the register s holding k2 = brev4(s)
__host__ __device__ constexpr int team_mirror(int s) {
  int k = 0;
  for (int b = 0; b < 4; ++b) k |= ((s >> b) & 1) << (3 - b);
  const int m = (16 - k) & 15;
  int r = 0;
  for (int b = 0; b < 4; ++b) r |= ((m >> b) & 1) << (3 - b);
  return r;
}

__host__ __device__ constexpr int brev4c(int s) {
  int k = 0;
  for (int b = 0; b < 4; ++b) k |= ((s >> b) & 1) << (3 - b);
  return k;
}

template <int P>
__device__ __forceinline__ void team_consts(TeamConsts<P>& c, int t) {
  constexpr int D = 16 * P, L = TeamConsts<P>::L;
  const double2 b = cis_neg(t, D);
  double2 pw = make_double2(1.0, 0.0);
#pragma unroll
  for (int k2 = 0; k2 < 16; ++k2) {
    c.wb[k2] = to_f2(pw);
    pw = cmul_d(pw, b);
  }
#pragma unroll
  for (int s = 0; s < L; ++s) {
    const int h = (P / 2) >> s;
    const bool upper = (t & h) != 0;
    c.wc[s] = upper ? to_f2(cis_neg(t & (h - 1), 2 * h)) : make_float2(1.0f, 0.0f);
    c.sg[s] = upper ? -1.0f : 1.0f;
  }
  c.src0 = brev_bits<L>((P - brev_bits<L>(t)) & (P - 1));
}

// exp(-2 pi i n / 16), n < 8, rounded to fp32
__device__ __forceinline__ float2 w16(int n) {
  constexpr float c1 = 0.92387953251128674f, s1 = 0.38268343236508978f, h = 0.70710678118654752f;
  switch (n) {
    case 1: return make_float2(c1, -s1);
    case 2: return make_float2(h, -h);
    case 3: return make_float2(s1, -c1);
    case 5: return make_float2(-s1, -c1);
    case 6: return make_float2(-h, -h);
    case 7: return make_float2(-c1, -s1);
    default: return make_float2(1.0f, 0.0f);  // n = 0 (n = 4 is handled as -i)
  }
}

// (u, v) -> (u + v, (u - v) w16^n), n a compile-time constant after unrolling
__device__ __forceinline__ void dif_bfly(float& ur, float& ui, float& vr, float& vi, int n) {
  const float dr = ur - vr, di = ui - vi;
  ur += vr;
  ui += vi;
  if (n == 0) {
    vr = dr;
    vi = di;
  } else if (n == 4) {  // times -i
    vr = di;
    vi = -dr;
  } else {
    const float2 w = w16(n);
    vr = fmaf(dr, w.x, -di * w.y);
    vi = fmaf(dr, w.y, di * w.x);
  }
}

// In: re[j2] = x[t + P j2], im[j2] = y[t + P j2] (team lane t).
// Out: hx[s] = 2 sqrt(d) (F x)[k], hy[s] = 2 sqrt(d) (F y)[k] for
// k = brev4(s) + 16 brevL(t); the caller applies 1 / (2 sqrt(d)).
template <int P>
__device__ __forceinline__ void hartley_pair_team(const float (&re_in)[16], const float (&im_in)[16],
                                                  const TeamConsts<P>& c, int team_base,
                                                  float (&hx)[16], float (&hy)[16]) {
  constexpr int L = TeamConsts<P>::L;
  // power-of-two normalization of each input over the team
  float mx = 0.0f, my = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    mx = fmaxf(mx, fabsf(re_in[j]));
    my = fmaxf(my, fabsf(im_in[j]));
  }
#pragma unroll
  for (int o = P / 2; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    my = fmaxf(my, __shfl_xor_sync(0xffffffffu, my, o));
  }
  int ex = 0, ey = 0;
  if (mx > 0.0f) frexpf(mx, &ex);
  if (my > 0.0f) frexpf(my, &ey);
  // multiplying by 2^-e and 2^e is what ldexpf computes; the float powers are
  // exact while e stays in [-126, 126] (team-uniform)
  const bool fast = ex >= -126 && ex <= 126 && ey >= -126 && ey <= 126;
  const float sxi = __int_as_float((127 - (fast ? ex : 0)) << 23);
  const float syi = __int_as_float((127 - (fast ? ey : 0)) << 23);
  float ar[16], ai[16];
  if (fast) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      ar[j] = re_in[j] * sxi;
      ai[j] = im_in[j] * syi;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      ar[j] = ldexpf(re_in[j], -ex);
      ai[j] = ldexpf(im_in[j], -ey);
    }
  }
  // A: 16-point DIF inside the lane; afterwards register s holds k2 = brev4(s)
#pragma unroll
  for (int h = 8; h > 0; h >>= 1)
#pragma unroll
    for (int blk = 0; blk < 16; blk += 2 * h)
#pragma unroll
      for (int i = 0; i < h; ++i)
        dif_bfly(ar[blk + i], ai[blk + i], ar[blk + i + h], ai[blk + i + h], i * (8 / h));
  // B: twiddles exp(-2 pi i t k2 / d)
#pragma unroll
  for (int s = 1; s < 16; ++s) {
    const float2 w = c.wb[brev4c(s)];
    const float r = ar[s], i = ai[s];
    ar[s] = fmaf(r, w.x, -i * w.y);
    ai[s] = fmaf(r, w.y, i * w.x);
  }
  // C: P-point radix-2 DIF across the team: lower lane a + b, upper lane (a - b) w
#pragma unroll
  for (int st = 0; st < L; ++st) {
    const int h = (P / 2) >> st;
    const float2 w = c.wc[st];
    const float sg = c.sg[st];
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      const float pr = __shfl_xor_sync(0xffffffffu, ar[s], h);
      const float pi = __shfl_xor_sync(0xffffffffu, ai[s], h);
      const float tr = fmaf(sg, ar[s], pr), ti = fmaf(sg, ai[s], pi);
      ar[s] = fmaf(tr, w.x, -ti * w.y);
      ai[s] = fmaf(tr, w.y, ti * w.x);
    }
  }
  // Hartley transforms of x and y from Z[k] and Z[d - k]
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    float qr, qi;
    if (s == 0) {
      qr = __shfl_sync(0xffffffffu, ar[0], team_base + c.src0);
      qi = __shfl_sync(0xffffffffu, ai[0], team_base + c.src0);
    } else {
      qr = __shfl_xor_sync(0xffffffffu, ar[team_mirror(s)], P - 1);
      qi = __shfl_xor_sync(0xffffffffu, ai[team_mirror(s)], P - 1);
    }
    hx[s] = (ar[s] + qr) + (qi - ai[s]);
    hy[s] = (ai[s] + qi) + (ar[s] - qr);
  }
  // scale back; an all-zero input's transform is exactly zero (not its
  // partner's rounding residue)
  if (fast) {
    const float sx = mx > 0.0f ? __int_as_float((127 + ex) << 23) : 0.0f;
    const float sy = my > 0.0f ? __int_as_float((127 + ey) << 23) : 0.0f;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      hx[s] *= sx;
      hy[s] *= sy;
    }
  } else {
#pragma unroll
    for (int s = 0; s < 16; ++s) {
      hx[s] = mx > 0.0f ? ldexpf(hx[s], ex) : 0.0f;
      hy[s] = my > 0.0f ? ldexpf(hy[s], ey) : 0.0f;
    }
  }
}

}  // namespace tq
