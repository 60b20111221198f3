// Device-side 3D-RoPE helpers shared by the kernels that rotate positional keys
// or queries [paperlayer App. C.1 separate t/h/w subspaces; App. D.3 (6,5,5) pairs].
#pragma once
#include "kernels.h"

namespace vmla {

// (cos, sin) of rotary pair p at integer grid position (t, h, w).
__device__ __forceinline__ float2 rope_cs(const Rope& rp, int p, int t, int h, int w) {
  const int pos = p < rp.n_t ? t : (p < rp.n_t + rp.n_h ? h : w);
  float s, c;
  sincosf((float)pos * rp.freq[p], &s, &c);
  return make_float2(c, s);
}

// (u, v) -> (u cos - v sin, u sin + v cos)
__device__ __forceinline__ void rope_apply(float& u, float& v, float2 cs) {
  const float a = u * cs.x - v * cs.y, b = u * cs.y + v * cs.x;
  u = a;
  v = b;
}

}  // namespace vmla
