// 2x2 projective (Moebius) maps for the scans of one-scalar uncertainty recurrences.
//
// Kalman Delta Networks, Abstract: the scan-compatible KDN uncertainty recurrences are Moebius maps,
// which compose associatively.  A map c -> (a c + b) / (c' c + d) is the matrix [[a, b], [c', d]];
// products are renormalised so that the lower-right entry is 1 (the map is projective), which keeps every
// entry of a product of non-negative maps in range.
#pragma once

namespace kdn {
namespace mobius {

struct Mob {
  float a, b, c, d;
};

__device__ __forceinline__ Mob identity() { return Mob{1.f, 0.f, 0.f, 1.f}; }

// later o earlier (apply `earlier` first), renormalised
__device__ __forceinline__ Mob compose(const Mob& later, const Mob& earlier) {
  Mob m;
  m.a = fmaf(later.a, earlier.a, later.b * earlier.c);
  m.b = fmaf(later.a, earlier.b, later.b * earlier.d);
  m.c = fmaf(later.c, earlier.a, later.d * earlier.c);
  m.d = fmaf(later.c, earlier.b, later.d * earlier.d);
  const float inv = 1.f / m.d;
  m.a *= inv, m.b *= inv, m.c *= inv, m.d = 1.f;
  return m;
}

__device__ __forceinline__ Mob shfl_up(const Mob& m, int delta) {
  Mob r;
  r.a = __shfl_up_sync(0xffffffffu, m.a, delta);
  r.b = __shfl_up_sync(0xffffffffu, m.b, delta);
  r.c = __shfl_up_sync(0xffffffffu, m.c, delta);
  r.d = __shfl_up_sync(0xffffffffu, m.d, delta);
  return r;
}

__device__ __forceinline__ float apply(const Mob& m, float x) { return (m.a * x + m.b) / (m.c * x + m.d); }

// The isotropic-Kalman token map (divided through by d_k r): propagate c^- = a^2 c + Qn, then the
// isotropic projection c <- d_k c^- r / (d_k r + c^- ||k||^2); w = ||k||^2 / (d_k r).
__device__ __forceinline__ Mob iso_token(float a2, float qn, float w) { return Mob{a2, qn, w * a2, fmaf(w, qn, 1.f)}; }

}  // namespace mobius
}  // namespace kdn
