// sta_common.cuh -- device helpers shared by the STA forward and backward
// kernels: token addressing in raster / tile-major order, TMA box coordinates
// of a run of tile rows, per-warp barrier arrival, bounded drains.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "sta_kernels.h"

namespace sta {

constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;  // 0.2 s

__device__ __forceinline__ bool drain_wait(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > (long long)(2 * kDrainLimitNs)) return false;
  return true;
}

// 2^x for two values at once on the FMA pipe, instead of the MUFU unit.
// Cody and Waite's argument reduction: x = n + r with n = round(x) (adding
// 1.5 * 2^23 rounds to an integer, which lands in the low mantissa bits) and r
// in [-1/2, 1/2]; 2^r by a degree-3 polynomial in Horner form; n added to the
// exponent field of the result.  The coefficients are this library's own
// minimax fit of 2^r on [-1/2, 1/2] in relative error (fit_exp2_poly.py in
// this directory): relative error <= 7.5e-5 for x >= -125 and <= 1.5e-4 down
// to -126, far below the bf16 rounding of P that follows.  Inputs below -126
// are clamped to -126 (2^-126 instead of a smaller value or 0): the softmax
// adds these terms to a row sum >= 1 and multiplies them into V rows that are
// zero for keys past the end of a list.
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 magic = make_float2(12582912.f, 12582912.f);
  const float2 t = add2(x, magic);
  const float2 r = sub2(x, sub2(t, magic));
  float2 p = fma2(make_float2(kExp2C3, kExp2C3), r, make_float2(kExp2C2, kExp2C2));
  p = fma2(p, r, make_float2(kExp2C1, kExp2C1));
  p = fma2(p, r, make_float2(kExp2C0, kExp2C0));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// Token index (in the tensor's own order) of row `o` of tile `tile`.
__device__ __forceinline__ long long token_row(const Geometry &g, int tiled, int bh, int tile, int o) {
  if (tiled) return (long long)bh * g.N + (long long)tile * g.tau + o;
  const int it = tile / (g.GH * g.GW), ih = (tile / g.GW) % g.GH, iw = tile % g.GW;
  const int a = o / (g.th * g.tw), b = (o / g.tw) % g.th, c = o % g.tw;
  const int t = it * g.tt + a, h = ih * g.th + b, w = iw * g.tw + c;
  return (long long)bh * g.N + ((long long)t * g.H + h) * g.W + w;
}

// Per-warp arrive: every lane has finished its part before lane 0 arrives.
__device__ __forceinline__ void warp_arrive(uint64_t *bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// TMA box coordinates of `piece_rows` consecutive tile-major rows starting at
// in-tile row `off` of tile `tile` in slice bh; an out-of-range coordinate
// (zero fill) when !valid.  Tiled maps use (row); raster maps (w, h, t*bh).
template <class P>
__device__ __forceinline__ int4 box_coords(const P &p, int bh, int tile, int off, bool valid) {
  const Geometry &g = p.g;
  if (p.kv_mode == kKvTiled) return make_int4(valid ? bh * g.N + tile * g.tau + off : p.oob_coord, 0, 0, 0);
  const int kt = tile / (g.GH * g.GW), kh = (tile / g.GW) % g.GH, kw = tile % g.GW;
  const int a = off / (g.th * g.tw), b = (off / g.tw) % g.th, c = off % g.tw;
  return make_int4(kw * g.tw + c, kh * g.th + b, valid ? bh * g.T + kt * g.tt + a : p.oob_coord, 0);
}

// Issue the TMA box(es) of one piece (all 64-column panels of a 128-row
// operand tile whose panels are `panel_bytes` apart) at `c`.
template <int D, class P>
__device__ __forceinline__ void load_box(const P &p, const CUtensorMap *map, uint8_t *dst, int4 c, uint64_t *bar) {
  constexpr uint32_t kPanelBytes = 128 * 128;
  const int boxes = (D / 64) / p.box_panels;
  for (int pn = 0; pn < boxes; ++pn) {
    uint8_t *pdst = dst + pn * kPanelBytes;
    if (p.kv_mode == kKvTiled) {
      if constexpr (D == 128) tma_load_3d(pdst, map, 0, c.x, pn, bar);
      else tma_load_2d(pdst, map, 0, c.x, bar);
    } else {
      if constexpr (D == 128) tma_load_5d(pdst, map, 0, c.x, c.y, c.z, pn, bar);
      else tma_load_4d(pdst, map, 0, c.x, c.y, c.z, bar);
    }
  }
}

}  // namespace sta
