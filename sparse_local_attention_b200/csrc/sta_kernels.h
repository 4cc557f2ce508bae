// sta_kernels.h -- parameter blocks and launchers shared by the host API
// (sta_api.cpp) and the CUDA kernels.  Internal to libsta.so.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/sta.h"

namespace sta {

// Status codes the kernels write into the workspace status word.
enum KernelError : int {
  kErrNone = 0,
  kErrWaitProducer = 0x101,  // producer: waited too long for a free stage
  kErrWaitMma = 0x102,       // MMA issuer: waited too long for data / softmax
  kErrWaitSoftmax = 0x103,   // softmax warps: waited too long for an MMA result
  kErrWaitEpilogue = 0x104,
  kErrBwdWait = 0x201,
};

// How the K/V tiles are read by TMA.
// Both maps split the head dimension into 64-element (128-byte) panels; for
// d = 128 the panel index is the outermost map dimension, so one box can
// bring both panels of a chunk in a single TMA instruction.
enum KvMode : int {
  kKvTiled = 0,   // (64, B*Hh*N rows[, 2 panels]) over a tile-major buffer
  kKvRaster = 1,  // (64, W, H, T*B*Hh[, 2 panels]) over the raster tensor
};

struct Geometry {
  int B, Hh, d, N;
  int T, H, W;
  int tt, th, tw;
  int GT, GH, GW;
  int n_tiles, tau;  // tiles per (b, h) slice, tokens per tile
};

struct FwdParams {
  Geometry g;
  const void *q;     // bf16, token order given by `tiled`
  void *o;           // bf16
  float *lse;        // fp32, nullable
  int tiled;         // q / o / lse are tile-major instead of raster
  int nqb;           // 128-row query blocks per tile = ceil(tau / 128)
  const int32_t *kv_list;   // [Hh][n_tiles][kv_stride]
  const int32_t *kv_count;  // [Hh]
  int kv_stride;
  // Work items (bh, a, b, 0): query block A = a % nqb of tile a / nqb and query
  // block B likewise from b, or b = -1 for a lone block.  A and B attend to the
  // same key tiles (the KV-tile list of A's tile).  Heaviest first within each
  // kind; the last n_work_lone items are the lone blocks.
  const int4 *work;
  int n_work;
  int n_work_lone;
  float scale_log2;  // softmax scale * log2(e)
  int *status;       // device status word
  unsigned long long wait_limit_ns;
  // K/V gather geometry
  int kv_mode;
  int piece_rows;            // rows per TMA box (divides both tau and 128)
  int box_w, box_h, box_t;   // raster box extents in tokens
  int box_panels;            // panels per box: 2 = whole chunk row in one instruction
  int oob_coord;             // row (tiled) or T*B*Hh (raster) coordinate past the end
};

struct BwdParams {
  Geometry g;
  int tiled;  // token order of every user tensor (q k v o dout lse dq dk dv)
  int nqb;    // 128-row blocks per tile = ceil(tau / 128)
  // operand TMA geometry (same meaning as in FwdParams)
  int kv_mode, piece_rows, box_w, box_h, box_t, box_panels, oob_coord;
  const void *o, *dout;  // preprocess inputs
  const float *lse;      // forward LSE (natural log)
  float *lse2_t, *dd_t;  // one 128-float run per query block: LSE*log2(e), D = rowsum(dO*O)
  // Per query block, one 4 KB K-major operand panel (no swizzle; 16 groups
  // of 8 rows at 256 bytes, the two 8-element halves of a row 128 bytes
  // apart): row q holds (a_hi, a_lo, d_hi, d_lo, 0, ..., 0) with a_hi + a_lo
  // = -LSE_q*log2(e) / scale_log2 and d_hi + d_lo = -D_q, all bf16.  The
  // dK/dV kernel adds them to S^T and dP^T with one more K step each, against
  // panels whose rows are (1, 1, 0, ...) and (0, 0, 1, 1, 0, ...), so that its
  // elementwise pass needs no per-query operand.
  uint8_t *aug;
  void *dq, *dk, *dv;    // bf16 outputs
  const int32_t *kv_list, *kv_count;  // forward lists (dQ kernel)
  int kv_stride;
  const int32_t *inv_off, *inv_idx;   // inverse lists, [Hh][n_tiles + 1] absolute offsets (dK/dV kernel)
  const int2 *work_kv;                // (bh, key tile * nqb + key block), heaviest first
  int n_work_kv;
  const int2 *work_q;                 // (bh, query tile * nqb + query block), heaviest first
  int n_work_q;
  float scale, scale_log2;
  int *status;
  unsigned long long wait_limit_ns;
};

struct PermuteParams {
  Geometry g;
  const void *src;
  void *dst;
  int inverse;
};

cudaError_t launch_forward(const FwdParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                           const CUtensorMap &tmap_v, int num_sms, cudaStream_t stream);
// The argument checks of sta_backward other than those of the workspace
// (null, host-only or forward-only plan, flags, alignment, current device).
sta_status check_backward_call(const sta_plan_s *plan, const void *const tensors[9], uint32_t flags);

cudaError_t launch_permute(const PermuteParams &p, int num_sms, cudaStream_t stream);
// Backward: preprocess (D, LSE*log2 e), dK/dV (key-block major) and dQ
// (query-block major), enqueued in that order on `stream`.
cudaError_t launch_backward(const BwdParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                            const CUtensorMap &tmap_v, const CUtensorMap &tmap_do, int num_sms,
                            cudaStream_t stream);

}  // namespace sta
