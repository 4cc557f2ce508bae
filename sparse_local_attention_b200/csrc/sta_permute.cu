// sta_permute.cu -- raster <-> tile-major token permutation (HBM-bound copy).
//
// Tiles are non-overlapping blocks of tile_t x tile_h x tile_w tokens
// ("Fast Video Generation with Sliding Tile Attention", summary page,
// Methodology).  In tile-major order a tile's tokens are contiguous, so every
// (query tile, key tile) pair is a dense block.  Token n = (t*H + h)*W + w goes
// to position tile*tau + in_tile, tile = ((t/tt)*GH + h/th)*GW + w/tw and
// in_tile = ((t%tt)*th + h%th)*tw + w%tw.
//
// One thread moves 16 bytes (8 bf16).  Threads walk the tile-major side in
// order, so that side is perfectly coalesced; on the raster side a warp still
// touches runs of tile_w whole token rows (tile_w * d * 2 contiguous bytes).
#include <cuda_bf16.h>

#include "sta_kernels.h"

namespace sta {
namespace {

__global__ void __launch_bounds__(256) permute_kernel(const PermuteParams p) {
  const Geometry &g = p.g;
  const int cpr = g.d / 8;  // 16-byte chunks per row
  const long long total = (long long)g.B * g.Hh * g.N * cpr;
  const uint4 *src = static_cast<const uint4 *>(p.src);
  uint4 *dst = static_cast<uint4 *>(p.dst);
  const int plane = g.th * g.tw;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / cpr;
    const int c = (int)(i - row * cpr);
    const long long bh = row / g.N;
    const int pos = (int)(row - bh * g.N);  // tile-major position
    const int tile = pos / g.tau, o = pos - (pos / g.tau) * g.tau;
    const int it = tile / (g.GH * g.GW), ih = (tile / g.GW) % g.GH, iw = tile % g.GW;
    const int a = o / plane, b = (o / g.tw) % g.th, cc = o % g.tw;
    const long long n = ((long long)(it * g.tt + a) * g.H + (ih * g.th + b)) * g.W + (iw * g.tw + cc);
    const long long raster = (bh * g.N + n) * cpr + c;
    const long long tiled = row * cpr + c;
    if (p.inverse)
      dst[raster] = src[tiled];
    else
      dst[tiled] = src[raster];
  }
}

}  // namespace

cudaError_t launch_permute(const PermuteParams &p, int num_sms, cudaStream_t stream) {
  const long long total = (long long)p.g.B * p.g.Hh * p.g.N * (p.g.d / 8);
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)num_sms * 16;
  if (blocks > cap) blocks = cap;
  permute_kernel<<<(int)blocks, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace sta
