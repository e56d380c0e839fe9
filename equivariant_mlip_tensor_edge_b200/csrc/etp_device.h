// Device helpers shared by the convolution kernels: the binding of the generated per-path code
// and the radial basis. Internal to libetp.
#pragma once

#include "etp_internal.h"
#include "generated/etp_paths.h"

namespace etp {

constexpr unsigned kFull = 0xffffffffu;

template <int L> struct Gen;
#define ETP_GEN_BIND(LL)                                                                          \
  template <> struct Gen<LL> {                                                                    \
    static constexpr int D = etp_gen::PathSet<LL>::D;                                             \
    static constexpr int P = etp_gen::PathSet<LL>::P;                                             \
    __device__ static void sh(float nx, float ny, float nz, float* Y) { etp_gen::sh_eval_##LL(nx, ny, nz, Y); } \
    __device__ static void sh_grad(float nx, float ny, float nz, const float* gY, float& gx,      \
                                   float& gy, float& gz, float& s) {                              \
      etp_gen::sh_grad_##LL(nx, ny, nz, gY, gx, gy, gz, s);                                       \
    }                                                                                             \
    template <int K, class WF>                                                                    \
    __device__ static void fwd(const float* Y, WF&& wf, const float (&x)[D][K], float (&acc)[D][K]) { \
      etp_gen::tp_fwd_##LL<K>(Y, wf, x, acc);                                                     \
    }                                                                                             \
    template <int K, class WF>                                                                    \
    __device__ static void bwd(const float* Y, WF&& wf, const float (&x)[D][K], const float (&g)[D][K], \
                               float (&gx)[D][K], float* gY, float& accd) {                       \
      etp_gen::tp_bwd_##LL<K>(Y, wf, x, g, gx, gY, accd);                                         \
    }                                                                                             \
  };
ETP_GEN_BIND(1)
ETP_GEN_BIND(2)
ETP_GEN_BIND(3)
#undef ETP_GEN_BIND

// ---------------------------------------------------------------- per-edge geometry

// R_b(d) = (2/r_c) sin(b pi t) / d * u(t), t = d / r_c, u(t) = 1 - 28 t^6 + 48 t^7 - 21 t^8.
// sin(b pi t) for b = 1..8 by the Chebyshev recurrence s_{b+1} = 2 cos(pi t) s_b - s_{b-1}.
// If dR is given, also dR_b/dd. Edges with t >= 1 (or d == 0) get R = dR = 0.
template <bool kDeriv>
__device__ __forceinline__ void radial_basis(float d, float inv_rc, float (&R)[kNumBasis],
                                             float (&dR)[kNumBasis]) {
  const float t = d * inv_rc;
  if (!(t < 1.0f) || !(d > 0.0f)) {
#pragma unroll
    for (int b = 0; b < kNumBasis; ++b) {
      R[b] = 0.0f;
      if (kDeriv) dR[b] = 0.0f;
    }
    return;
  }
  float s1, c1;
  sincospif(t, &s1, &c1);
  const float t2 = t * t;
  const float t3 = t2 * t;
  const float t6 = t3 * t3;
  const float u = fmaf(t6, fmaf(t, fmaf(-21.0f, t, 48.0f), -28.0f), 1.0f);
  const float inv_d = 1.0f / d;
  const float pref = 2.0f * inv_rc * inv_d;     // (2/r_c)/d
  const float two_c = 2.0f * c1;
  float sp = 0.0f, sc = s1;                      // sin((b-1) pi t), sin(b pi t)
  float cp = 1.0f, cc = c1;                      // cos((b-1) pi t), cos(b pi t)
  // du/dd = u'(t) / r_c,  u'(t) = -168 t^5 (1 - t)^2
  const float omt = 1.0f - t;
  const float du = -168.0f * (t3 * t2) * omt * omt * inv_rc;
  const float kpi = 3.14159265358979323846f * inv_rc;
#pragma unroll
  for (int b = 0; b < kNumBasis; ++b) {
    R[b] = pref * sc * u;
    if (kDeriv) {
      // d/dd [ (2/r_c) sin(k d)/d u ] = (2/r_c)/d [ k cos(k d) u + sin(k d) (du - u/d) ]
      dR[b] = pref * fmaf(kpi * static_cast<float>(b + 1) * cc, u, sc * (du - u * inv_d));
    }
    const float sn = fmaf(two_c, sc, -sp);
    sp = sc;
    sc = sn;
    if (kDeriv) {
      const float cn = fmaf(two_c, cc, -cp);
      cp = cc;
      cc = cn;
    }
  }
}

}  // namespace etp
