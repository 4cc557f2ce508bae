// sta_permute.cu -- raster <-> tile-major token permutation (HBM-bound copy).
//
// Tiles are non-overlapping blocks of tile_t x tile_h x tile_w tokens
// ("Fast Video Generation with Sliding Tile Attention", summary page,
// Methodology).  In tile-major order a tile's tokens are contiguous, so every
// (query tile, key tile) pair is a dense block.  Token n = (t*H + h)*W + w goes
// to position tile*tau + in_tile, tile = ((t/tt)*GH + h/th)*GW + w/tw and
// in_tile = ((t%tt)*th + h%th)*tw + w%tw.
//
// One CTA per (batch x head slice, tile).  Inside a tile, the tokens of one
// (t, h) line form a run of tile_w consecutive tokens on both sides (raster
// and tile-major), so the CTA walks the tile run by run in 16-byte chunks:
// both sides are read and written in contiguous runs of tile_w * d * 2 bytes,
// and the only index arithmetic per chunk is two 32-bit divisions.  Each
// thread keeps four chunks in flight.
#include <cuda_bf16.h>

#include "sta_kernels.h"

namespace sta {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kThreads) permute_kernel(const PermuteParams p) {
  const Geometry &g = p.g;
  const int cpr = g.d / 8;        // 16-byte chunks per token row
  const int run = g.tw * cpr;     // chunks in one (t, h) line of the tile
  const int total = g.tt * g.th * run;
  const uint4 *src = static_cast<const uint4 *>(p.src);
  uint4 *dst = static_cast<uint4 *>(p.dst);
  for (long long slab = blockIdx.x; slab < (long long)g.B * g.Hh * g.n_tiles; slab += gridDim.x) {
    const int bh = (int)(slab / g.n_tiles), tile = (int)(slab - (long long)bh * g.n_tiles);
    const int it = tile / (g.GH * g.GW), ih = (tile / g.GW) % g.GH, iw = tile % g.GW;
    const long long tiled0 = ((long long)bh * g.N + (long long)tile * g.tau) * cpr;
    const long long raster0 = (long long)bh * g.N * cpr;
    auto offsets = [&](int idx, long long &raster, long long &tiled) {
      const int r = idx / run, c = idx - r * run;  // line of the tile, chunk in the line
      const int a = r / g.th, b = r - a * g.th;
      const long long n = ((long long)(it * g.tt + a) * g.H + (ih * g.th + b)) * g.W + iw * g.tw;
      raster = raster0 + n * cpr + c;
      tiled = tiled0 + (long long)r * run + c;
    };
    for (int base = threadIdx.x; base < total; base += kThreads * kUnroll) {
      long long from[kUnroll], to[kUnroll];
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int idx = base + u * kThreads;
        if (idx < total) {
          long long raster, tiled;
          offsets(idx, raster, tiled);
          from[u] = p.inverse ? tiled : raster;
          to[u] = p.inverse ? raster : tiled;
          v[u] = src[from[u]];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (base + u * kThreads < total) dst[to[u]] = v[u];
    }
  }
}

}  // namespace

cudaError_t launch_permute(const PermuteParams &p, int num_sms, cudaStream_t stream) {
  const long long slabs = (long long)p.g.B * p.g.Hh * p.g.n_tiles;
  if (slabs == 0) return cudaSuccess;
  const long long cap = (long long)num_sms * 8;  // 8 CTAs of 256 threads per SM
  const int blocks = (int)(slabs < cap ? slabs : cap);
  permute_kernel<<<blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace sta
