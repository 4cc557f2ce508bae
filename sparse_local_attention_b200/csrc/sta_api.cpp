// sta_api.cpp -- host side of libsta.so: argument checking, the planner
// (window starts, KV-tile lists, inverse lists, work order), TMA descriptors
// and kernel launches behind the C ABI of include/sta.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <new>
#include <numeric>
#include <vector>

#include "../../include/sta.h"
#include "sta_kernels.h"

using sta::Geometry;

struct sta_plan_s {
  sta_problem p{};
  Geometry g{};
  std::vector<int32_t> window;   // heads*3, as given
  std::vector<int32_t> wclamp;   // heads*3, clamped to the grid
  std::vector<int32_t> count;    // heads: key tiles per query tile
  int32_t kv_stride = 0;         // max(count)
  std::vector<int32_t> kv_list;  // [heads][n_tiles][kv_stride]
  std::vector<int32_t> inv_off;  // [heads][n_tiles + 1], absolute into inv_idx
  std::vector<int32_t> inv_idx;
  std::vector<int4> work;        // forward work items (see FwdParams::work)
  // sta_forward_host: the same items grouped by slice group (slices
  // [group_slice[g], group_slice[g + 1])), two-block items then lone ones
  std::vector<int4> work_host;
  std::vector<int> group_off, group_lone, group_slice;
  std::vector<int2> work_kv;     // backward dK/dV items (bh, key tile * nqb + key block)
  std::vector<int2> work_q;      // backward dQ items (bh, query tile * nqb + query block)
  int nqb = 1;  // 128-row query blocks per tile
  int n_work_lone = 0;  // forward items with one query block, at the end of `work`
  int kv_mode = sta::kKvTiled;
  int piece_rows = 0, box_w = 0, box_h = 0, box_t = 0;
  bool host_only = false;
  bool tiled = false;
  float scale = 0.f;
  int device = -1, num_sms = 0;
  // device copies
  int32_t *d_kv_list = nullptr, *d_count = nullptr, *d_inv_off = nullptr, *d_inv_idx = nullptr;
  int4 *d_work = nullptr, *d_work_host = nullptr;
  int2 *d_work_kv = nullptr, *d_work_q = nullptr;
};

namespace {

uint64_t g_wait_limit_ns = 2000ull * 1000 * 1000;  // 2 s per barrier wait

// Start of the window of `w` tiles (already clamped to G) around tile q,
// shifted inward so that [start, start + w) stays inside [0, G).
inline int window_start(int q, int w, int G) {
  int s = q - w / 2;
  if (s < 0) s = 0;
  if (s > G - w) s = G - w;
  return s;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

size_t tensor_bytes(const sta_plan_s *pl) {
  return (size_t)pl->g.B * pl->g.Hh * pl->g.N * pl->g.d * 2;
}

constexpr size_t kStatusBytes = 256;

size_t fwd_workspace(const sta_plan_s *pl) {
  size_t b = kStatusBytes;
  if (!pl->tiled && pl->kv_mode == sta::kKvTiled) b += 3 * tensor_bytes(pl);
  return b;
}

// Backward workspace: status word, then LSE*log2(e) and D = rowsum(dO*O), one
// 128-float run per (batch, head, tile, query block), then the two 4 KB
// operand panels per query block that fold LSE and D into the dK/dV kernel's
// S^T and dP^T products, then (only when tiles are not readable as boxes of
// the raster tensors) tile-major copies of Q, K, V and dO.
size_t bwd_blocks(const sta_plan_s *pl) { return (size_t)pl->g.B * pl->g.Hh * pl->g.n_tiles * pl->nqb; }
size_t bwd_vec_bytes(const sta_plan_s *pl) { return bwd_blocks(pl) * 128 * 4; }
constexpr size_t kAugBytesPerBlock = 4096;
// sta_forward_host workspace: device copies of Q, K, V, O and LSE (each at a
// 256-byte boundary), then sta_forward's own workspace (status word first).
constexpr int kHostGroups = 24;  // slice groups pipelined by sta_forward_host


size_t lse_bytes(const sta_plan_s *pl) { return (size_t)pl->g.B * pl->g.Hh * pl->g.N * 4; }

size_t host_copies_bytes(const sta_plan_s *pl) { return 4 * round256(tensor_bytes(pl)) + round256(lse_bytes(pl)); }

size_t host_workspace(const sta_plan_s *pl) { return host_copies_bytes(pl) + fwd_workspace(pl); }

size_t bwd_aug_offset(const sta_plan_s *pl) { return round256(kStatusBytes + 2 * bwd_vec_bytes(pl)); }
size_t bwd_gather_offset(const sta_plan_s *pl) { return bwd_aug_offset(pl) + bwd_blocks(pl) * kAugBytesPerBlock; }

size_t bwd_workspace(const sta_plan_s *pl) {
  size_t b = bwd_gather_offset(pl);
  if (!pl->tiled && pl->kv_mode == sta::kKvTiled) b += 4 * tensor_bytes(pl);
  return b;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Panels per TMA box: both 64-column panels of a 128-row chunk in one box
// when the chunk is a single piece and d = 128; otherwise one panel per box.
int box_panels(const sta_plan_s *pl) { return (pl->g.d == 128 && pl->piece_rows == 128) ? 2 : 1; }

// Tile-major buffer [rows][d] bf16 viewed as (64, rows[, 2 panels]); a box is
// `box_rows` rows by `panels` 64-column panels.
bool make_map_tiled_box(CUtensorMap *m, const void *base, const sta_plan_s *pl, int box_rows, int panels) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const Geometry &g = pl->g;
  const cuuint64_t rows = (cuuint64_t)g.B * g.Hh * g.N;
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {(cuuint64_t)g.d * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)panels};
  cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = g.d == 128 ? 3 : 2;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raster tensor viewed as (64, W, H, T*B*Hh[, 2 panels]); a box is a run of
// whole w-lines / h-planes of one tile (bw x bh x bt tokens) by `panels`
// 64-column panels, so tiles are gathered straight from the raster layout.
bool make_map_raster_box(CUtensorMap *m, const void *base, const sta_plan_s *pl, int bw, int bh, int bt,
                         int panels) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const Geometry &g = pl->g;
  const cuuint64_t row = (cuuint64_t)g.d * 2;
  cuuint64_t dims[5] = {64, (cuuint64_t)g.W, (cuuint64_t)g.H, (cuuint64_t)g.T * g.B * g.Hh, 2};
  cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.H, 128};
  cuuint32_t box[5] = {64, (cuuint32_t)bw, (cuuint32_t)bh, (cuuint32_t)bt, (cuuint32_t)panels};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const cuuint32_t rank = g.d == 128 ? 5 : 4;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_tiled(CUtensorMap *m, const void *base, const sta_plan_s *pl) {
  return make_map_tiled_box(m, base, pl, pl->piece_rows, box_panels(pl));
}

bool make_map_raster(CUtensorMap *m, const void *base, const sta_plan_s *pl) {
  return make_map_raster_box(m, base, pl, pl->box_w, pl->box_h, pl->box_t, box_panels(pl));
}

void free_device(sta_plan_s *pl) {
  cudaFree(pl->d_kv_list);
  cudaFree(pl->d_count);
  cudaFree(pl->d_inv_off);
  cudaFree(pl->d_inv_idx);
  cudaFree(pl->d_work);
  cudaFree(pl->d_work_host);
  cudaFree(pl->d_work_kv);
  cudaFree(pl->d_work_q);
  pl->d_kv_list = pl->d_count = pl->d_inv_off = pl->d_inv_idx = nullptr;
  pl->d_work = pl->d_work_host = nullptr;
  pl->d_work_kv = pl->d_work_q = nullptr;
}

template <class T>
bool upload(T **dst, const std::vector<T> &src) {
  if (src.empty()) return true;
  if (cudaMalloc(reinterpret_cast<void **>(dst), src.size() * sizeof(T)) != cudaSuccess) return false;
  return cudaMemcpy(*dst, src.data(), src.size() * sizeof(T), cudaMemcpyHostToDevice) == cudaSuccess;
}

int gcd_int(int a, int b) {
  while (b) {
    int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Plan the TMA gather of one piece of `rows` tokens of a tile directly from
// the raster tensor: the piece must be a box (whole w-runs, whole h-planes).
bool raster_box(const Geometry &g, int rows, int *bw, int *bh, int *bt) {
  const int plane = g.th * g.tw;
  if (rows % plane == 0) {
    const int t = rows / plane;
    if (g.tt % t) return false;
    *bw = g.tw, *bh = g.th, *bt = t;
  } else if (rows % g.tw == 0 && rows < plane) {
    const int h = rows / g.tw;
    if (g.th % h) return false;
    *bw = g.tw, *bh = h, *bt = 1;
  } else if (rows < g.tw && g.tw % rows == 0) {
    *bw = rows, *bh = 1, *bt = 1;
  } else {
    return false;
  }
  return *bw <= 256 && *bh <= 256 && *bt <= 256;
}

// Compute calls enqueue on the calling thread's current device, and the plan's
// tables live on the device that was current when it was created: a call made
// while another device is current is refused before anything is enqueued.
constexpr int kNoDevice = -2;

sta_status check_device(const sta_plan_s *pl) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return STA_ERR_CUDA;
  }
  return dev == pl->device ? STA_OK : STA_ERR_INVALID_ARG;
}

sta_status finish_call(const sta_plan_s *pl, void *workspace, cudaStream_t stream, uint32_t flags) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return STA_ERR_CUDA;
  if (flags & STA_CALL_CHECK) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return STA_ERR_CUDA;
    int st = 0;
    if (cudaMemcpy(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return STA_ERR_CUDA;
    if (st != 0) return STA_ERR_TIMEOUT;
  }
  (void)pl;
  return STA_OK;
}

struct ForwardMaps {
  CUtensorMap q, k, v;
  bool ok = false;
};

// Tensor maps of one forward call over Q, K, V at qbase / kbase / vbase (raster
// boxes, or tile-major rows when the tensors are tile-major or gathered).
ForwardMaps forward_maps(const sta_plan_s *pl, const void *qbase, const void *kbase, const void *vbase) {
  ForwardMaps m;
  const bool raster5d = pl->kv_mode == sta::kKvRaster;
  m.ok = raster5d ? (make_map_raster(&m.q, qbase, pl) && make_map_raster(&m.k, kbase, pl) &&
                     make_map_raster(&m.v, vbase, pl))
                  : (make_map_tiled(&m.q, qbase, pl) && make_map_tiled(&m.k, kbase, pl) &&
                     make_map_tiled(&m.v, vbase, pl));
  return m;
}

// Launch the forward kernel(s) over `n_work` items at `work` (the last
// `n_lone` of them lone blocks).
sta_status enqueue_forward(const sta_plan_s *pl, const ForwardMaps &maps, const void *q, void *o, float *lse,
                           int *status, cudaStream_t stream, const int4 *work, int n_work, int n_lone) {
  const bool raster5d = pl->kv_mode == sta::kKvRaster;
  sta::FwdParams fp{};
  fp.g = pl->g;
  fp.q = q, fp.o = o, fp.lse = lse;
  fp.tiled = pl->tiled ? 1 : 0;
  fp.nqb = pl->nqb;
  fp.kv_list = pl->d_kv_list, fp.kv_count = pl->d_count, fp.kv_stride = pl->kv_stride;
  fp.work = work, fp.n_work = n_work, fp.n_work_lone = n_lone;
  fp.scale_log2 = pl->scale * 1.4426950408889634f;
  fp.status = status;
  fp.wait_limit_ns = g_wait_limit_ns;
  fp.kv_mode = raster5d ? sta::kKvRaster : sta::kKvTiled;
  fp.piece_rows = pl->piece_rows;
  fp.box_w = pl->box_w, fp.box_h = pl->box_h, fp.box_t = pl->box_t;
  fp.box_panels = box_panels(pl);
  fp.oob_coord = raster5d ? pl->g.T * pl->g.B * pl->g.Hh : pl->g.B * pl->g.Hh * pl->g.N;
  const cudaError_t e = sta::launch_forward(fp, maps.q, maps.k, maps.v, pl->num_sms, stream);
  return e == cudaSuccess ? STA_OK : STA_ERR_CUDA;
}

}  // namespace

namespace sta {

// Every check of sta_backward except those of the workspace, in the order
// sta_backward applies them; the last is the device check.
sta_status check_backward_call(const sta_plan_s *pl, const void *const tensors[9], uint32_t flags) {
  if (!pl || pl->host_only) return STA_ERR_INVALID_ARG;
  for (int i = 0; i < 9; ++i)
    if (!tensors[i]) return STA_ERR_INVALID_ARG;
  if (pl->inv_off.empty()) return STA_ERR_INVALID_ARG;  // plan built without STA_PROBLEM_BACKWARD
  if (flags & ~STA_CALL_CHECK) return STA_ERR_INVALID_ARG;
  for (int i = 0; i < 9; ++i)
    if (!aligned16(tensors[i])) return STA_ERR_ALIGNMENT;
  return check_device(pl);
}

}  // namespace sta

extern "C" {

const char *sta_status_string(sta_status s) {
  switch (s) {
    case STA_OK: return "ok";
    case STA_ERR_INVALID_ARG: return "invalid argument";
    case STA_ERR_SHAPE: return "shape not supported (tile must divide the latent; sizes must be >= 1)";
    case STA_ERR_UNSUPPORTED: return "unsupported configuration (head_dim must be 64 or 128; tile volume a multiple of 8; sm_100 device)";
    case STA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case STA_ERR_WORKSPACE: return "workspace missing or too small";
    case STA_ERR_OOM: return "out of memory";
    case STA_ERR_CUDA: return "CUDA runtime error";
    case STA_ERR_TIMEOUT: return "kernel wait timed out; outputs are invalid";
  }
  return "unknown status";
}

void sta_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns; }

sta_status sta_plan_create(const sta_problem *prob, sta_plan_t *out) {
  if (!prob || !out || !prob->window) return STA_ERR_INVALID_ARG;
  const uint32_t known = STA_PROBLEM_BACKWARD | STA_PROBLEM_TILED | STA_PROBLEM_HOST_ONLY | STA_PROBLEM_DEVICE_CHECK_TEST;
  if (prob->flags & ~known) return STA_ERR_INVALID_ARG;
  if (prob->batch < 1 || prob->heads < 1 || prob->T < 1 || prob->H < 1 || prob->W < 1 || prob->tile_t < 1 ||
      prob->tile_h < 1 || prob->tile_w < 1)
    return STA_ERR_SHAPE;
  if (prob->T % prob->tile_t || prob->H % prob->tile_h || prob->W % prob->tile_w) return STA_ERR_SHAPE;
  if (prob->head_dim != 64 && prob->head_dim != 128) return STA_ERR_UNSUPPORTED;
  for (int i = 0; i < 3 * prob->heads; ++i)
    if (prob->window[i] < 1) return STA_ERR_INVALID_ARG;
  const long long N = (long long)prob->T * prob->H * prob->W;
  const long long rows = N * prob->batch * prob->heads;
  if (rows >= (1ll << 31) - 1024) return STA_ERR_SHAPE;
  const long long tau = (long long)prob->tile_t * prob->tile_h * prob->tile_w;
  if (tau % 8) return STA_ERR_UNSUPPORTED;

  sta_plan_s *pl = new (std::nothrow) sta_plan_s();
  if (!pl) return STA_ERR_OOM;
  pl->p = *prob;
  pl->host_only = (prob->flags & STA_PROBLEM_HOST_ONLY) != 0;
  pl->tiled = (prob->flags & STA_PROBLEM_TILED) != 0;
  Geometry &g = pl->g;
  g.B = prob->batch, g.Hh = prob->heads, g.d = prob->head_dim, g.N = (int)N;
  g.T = prob->T, g.H = prob->H, g.W = prob->W;
  g.tt = prob->tile_t, g.th = prob->tile_h, g.tw = prob->tile_w;
  g.GT = g.T / g.tt, g.GH = g.H / g.th, g.GW = g.W / g.tw;
  g.n_tiles = g.GT * g.GH * g.GW;
  g.tau = (int)tau;
  pl->scale = prob->scale > 0.f ? prob->scale : 1.0f / std::sqrt((float)g.d);
  pl->nqb = (g.tau + 127) / 128;

  try {
    // --- per-head clamped windows and list lengths
    pl->window.assign(prob->window, prob->window + 3 * g.Hh);
    pl->wclamp.resize(3 * g.Hh);
    pl->count.resize(g.Hh);
    const int G[3] = {g.GT, g.GH, g.GW};
    for (int h = 0; h < g.Hh; ++h) {
      int c = 1;
      for (int a = 0; a < 3; ++a) {
        pl->wclamp[3 * h + a] = std::min(pl->window[3 * h + a], G[a]);
        c *= pl->wclamp[3 * h + a];
      }
      pl->count[h] = c;
    }
    pl->kv_stride = *std::max_element(pl->count.begin(), pl->count.end());
    // list positions (and the inverse lists' offsets) are 32-bit on the device
    if ((long long)g.Hh * g.n_tiles * pl->kv_stride >= (1ll << 31) - 1) {
      delete pl;
      return STA_ERR_SHAPE;
    }

    // --- forward KV-tile lists: whole key tiles of each query tile's window,
    //     ascending tile-major index (t outer, w inner)
    pl->kv_list.assign((size_t)g.Hh * g.n_tiles * pl->kv_stride, -1);
    for (int h = 0; h < g.Hh; ++h) {
      const int *w = &pl->wclamp[3 * h];
      for (int qt = 0; qt < g.GT; ++qt)
        for (int qh = 0; qh < g.GH; ++qh)
          for (int qw = 0; qw < g.GW; ++qw) {
            const int qtile = (qt * g.GH + qh) * g.GW + qw;
            const int st = window_start(qt, w[0], g.GT), sh = window_start(qh, w[1], g.GH),
                      sw = window_start(qw, w[2], g.GW);
            int32_t *dst = &pl->kv_list[((size_t)h * g.n_tiles + qtile) * pl->kv_stride];
            int n = 0;
            for (int kt = st; kt < st + w[0]; ++kt)
              for (int kh = sh; kh < sh + w[1]; ++kh)
                for (int kw = sw; kw < sw + w[2]; ++kw) dst[n++] = (kt * g.GH + kh) * g.GW + kw;
          }
    }

    // --- inverse lists (key tile -> query tiles), CSR per head
    if (prob->flags & STA_PROBLEM_BACKWARD) {
      pl->inv_off.assign((size_t)g.Hh * (g.n_tiles + 1), 0);
      std::vector<std::vector<int32_t>> buckets(g.n_tiles);
      for (int h = 0; h < g.Hh; ++h) {
        for (auto &b : buckets) b.clear();
        for (int qtile = 0; qtile < g.n_tiles; ++qtile) {
          const int32_t *lst = &pl->kv_list[((size_t)h * g.n_tiles + qtile) * pl->kv_stride];
          for (int i = 0; i < pl->count[h]; ++i) buckets[lst[i]].push_back(qtile);
        }
        int32_t *off = &pl->inv_off[(size_t)h * (g.n_tiles + 1)];
        off[0] = (int32_t)pl->inv_idx.size();
        for (int k = 0; k < g.n_tiles; ++k) {
          pl->inv_idx.insert(pl->inv_idx.end(), buckets[k].begin(), buckets[k].end());
          off[k + 1] = (int32_t)pl->inv_idx.size();
        }
      }
    }

    // --- forward work items: pairs of 128-row query blocks that attend to the
    //     same key tiles, so that each K/V chunk brought in serves 256 rows.
    //     Blocks 2i, 2i+1 of a tile pair up.  When a tile has an odd number of
    //     blocks, its last block pairs with the last block of another tile of
    //     the same head whose KV-tile list is the same (tiles whose clamped
    //     windows coincide, as they do next to the grid borders); a block left
    //     without such a partner is a lone item.  Lone items go last: the
    //     one-CTA forward runs them as a launch of their own.  Within each
    //     kind the persistent grid takes items round-robin, so they are ordered
    //     by cost, largest first (query blocks x key tiles: a longest-
    //     processing-time order); within a cost, head by head and tile by tile,
    //     so consecutive items share most of their key tiles in L2.
    std::vector<int> heads(g.Hh);
    std::iota(heads.begin(), heads.end(), 0);
    std::stable_sort(heads.begin(), heads.end(), [&](int a, int b) { return pl->count[a] > pl->count[b]; });
    const int nqb = pl->nqb;
    std::vector<int4> lone_items;
    std::vector<int> partner(g.n_tiles);
    for (int h : heads) {
      // partner[t]: the tile whose last block shares an item with t's last block
      // (t itself when t leads such an item, -1 when t's last block is lone,
      // -2 when t's last block is taken by an earlier tile)
      std::fill(partner.begin(), partner.end(), -1);
      if (nqb % 2 == 1) {
        const int *w = &pl->wclamp[3 * h];
        std::map<std::array<int, 3>, int> open;  // window start -> tile waiting for a partner
        for (int t = 0; t < g.n_tiles; ++t) {
          const int qt = t / (g.GH * g.GW), qh = (t / g.GW) % g.GH, qw = t % g.GW;
          const std::array<int, 3> key = {window_start(qt, w[0], g.GT), window_start(qh, w[1], g.GH),
                                          window_start(qw, w[2], g.GW)};
          auto f = open.find(key);
          if (f == open.end()) {
            open[key] = t;
          } else {
            partner[f->second] = t;
            partner[t] = -2;
            open.erase(f);
          }
        }
      }
      for (int b = 0; b < g.B; ++b) {
        const int bh = b * g.Hh + h;
        for (int t = 0; t < g.n_tiles; ++t) {
          for (int qb = 0; qb + 1 < nqb; qb += 2)
            pl->work.push_back(make_int4(bh, t * nqb + qb, t * nqb + qb + 1, 0));
          if (nqb % 2 == 1) {
            const int last = t * nqb + nqb - 1;
            if (partner[t] >= 0) pl->work.push_back(make_int4(bh, last, partner[t] * nqb + nqb - 1, 0));
            else if (partner[t] == -1) lone_items.push_back(make_int4(bh, last, -1, 0));
          }
        }
      }
    }
    auto cost = [&](const int4 &w) { return (long long)(w.z >= 0 ? 2 : 1) * pl->count[w.x % g.Hh]; };
    auto by_cost = [&](const int4 &a, const int4 &b) { return cost(a) > cost(b); };
    std::stable_sort(pl->work.begin(), pl->work.end(), by_cost);
    std::stable_sort(lone_items.begin(), lone_items.end(), by_cost);
    pl->n_work_lone = (int)lone_items.size();
    pl->work.insert(pl->work.end(), lone_items.begin(), lone_items.end());
    {
      // slice groups for sta_forward_host: each group's items in the order
      // above (two-block items, then lone blocks)
      const int slices = g.B * g.Hh, groups = std::min(slices, kHostGroups);
      pl->group_slice.resize(groups + 1);
      for (int gi = 0; gi <= groups; ++gi) pl->group_slice[gi] = (int)((long long)slices * gi / groups);
      std::vector<int> group_of(slices);
      for (int gi = 0; gi < groups; ++gi)
        for (int sl = pl->group_slice[gi]; sl < pl->group_slice[gi + 1]; ++sl) group_of[sl] = gi;
      const int n_pairs = (int)pl->work.size() - pl->n_work_lone;
      pl->group_off.assign(groups + 1, 0);
      pl->group_lone.assign(groups, 0);
      for (int gi = 0; gi < groups; ++gi) {
        pl->group_off[gi] = (int)pl->work_host.size();
        for (int i = 0; i < (int)pl->work.size(); ++i)
          if (group_of[pl->work[i].x] == gi) {
            pl->work_host.push_back(pl->work[i]);
            if (i >= n_pairs) ++pl->group_lone[gi];
          }
      }
      pl->group_off[groups] = (int)pl->work_host.size();
    }

    if (prob->flags & STA_PROBLEM_BACKWARD) {
      // dQ: one 128-row query block per item, heaviest heads first.
      for (int h : heads)
        for (int b = 0; b < g.B; ++b)
          for (int t = 0; t < g.n_tiles; ++t)
            for (int qb = 0; qb < nqb; ++qb) pl->work_q.push_back(make_int2(b * g.Hh + h, t * nqb + qb));
      // dK/dV: one 128-row key block per item, slice by slice (the key blocks
      // running at the same time then read the query tiles of one slice,
      // which stay in L2), within a slice longest inverse list first.
      struct KvItem { int len, bh, key; };
      std::vector<KvItem> items;
      items.reserve((size_t)g.B * g.Hh * g.n_tiles * nqb);
      for (int h = 0; h < g.Hh; ++h)
        for (int b = 0; b < g.B; ++b)
          for (int t = 0; t < g.n_tiles; ++t) {
            const int32_t *off = &pl->inv_off[(size_t)h * (g.n_tiles + 1) + t];
            for (int kb = 0; kb < nqb; ++kb) items.push_back({off[1] - off[0], b * g.Hh + h, t * nqb + kb});
          }
      std::stable_sort(items.begin(), items.end(),
                       [](const KvItem &a, const KvItem &c) { return a.bh != c.bh ? a.bh < c.bh : a.len > c.len; });
      for (const KvItem &it : items) pl->work_kv.push_back(make_int2(it.bh, it.key));
    }
  } catch (const std::bad_alloc &) {
    delete pl;
    return STA_ERR_OOM;
  }

  // --- how K/V tiles reach shared memory
  pl->piece_rows = gcd_int(g.tau, 128);
  if (pl->tiled) {
    pl->kv_mode = sta::kKvTiled;
  } else if (raster_box(g, pl->piece_rows, &pl->box_w, &pl->box_h, &pl->box_t)) {
    pl->kv_mode = sta::kKvRaster;
  } else {
    pl->kv_mode = sta::kKvTiled;  // permute K and V into the workspace first
  }

  if (!pl->host_only) {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&pl->num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      delete pl;
      return STA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) {
      delete pl;
      return STA_ERR_UNSUPPORTED;
    }
    // (a plan made for the device-check test records a device that is never current)
    pl->device = (prob->flags & STA_PROBLEM_DEVICE_CHECK_TEST) ? kNoDevice : dev;
    std::vector<int32_t> cnt(pl->count);
    if (!upload(&pl->d_kv_list, pl->kv_list) || !upload(&pl->d_count, cnt) || !upload(&pl->d_work, pl->work) ||
        !upload(&pl->d_work_host, pl->work_host) ||
        !upload(&pl->d_inv_off, pl->inv_off) || !upload(&pl->d_inv_idx, pl->inv_idx) ||
        !upload(&pl->d_work_kv, pl->work_kv) || !upload(&pl->d_work_q, pl->work_q)) {
      cudaError_t e = cudaGetLastError();
      free_device(pl);
      delete pl;
      return e == cudaErrorMemoryAllocation ? STA_ERR_OOM : STA_ERR_CUDA;
    }
  }
  *out = pl;
  return STA_OK;
}

sta_status sta_plan_destroy(sta_plan_t pl) {
  if (!pl) return STA_OK;
  if (!pl->host_only) free_device(pl);
  delete pl;
  return STA_OK;
}

sta_status sta_plan_workspace_size(sta_plan_t pl, size_t *fwd, size_t *bwd) {
  if (!pl) return STA_ERR_INVALID_ARG;
  if (fwd) *fwd = fwd_workspace(pl);
  if (bwd) *bwd = bwd_workspace(pl);
  return STA_OK;
}

sta_status sta_plan_geometry(sta_plan_t pl, int32_t *n_tiles, int32_t *tile_volume) {
  if (!pl) return STA_ERR_INVALID_ARG;
  if (n_tiles) *n_tiles = pl->g.n_tiles;
  if (tile_volume) *tile_volume = pl->g.tau;
  return STA_OK;
}

sta_status sta_plan_work_items(sta_plan_t pl, int32_t which, int32_t *out, size_t cap_items, size_t *n_items,
                               int32_t *n_lone) {
  if (!pl || !n_items) return STA_ERR_INVALID_ARG;
  if (n_lone) *n_lone = pl->n_work_lone;
  if (which == STA_WORK_FORWARD || which == STA_WORK_FORWARD_HOST) {
    const std::vector<int4> &w = which == STA_WORK_FORWARD ? pl->work : pl->work_host;
    *n_items = w.size();
    if (!out) return STA_OK;
    if (cap_items < w.size()) return STA_ERR_INVALID_ARG;
    for (size_t i = 0; i < w.size(); ++i) {
      out[4 * i] = w[i].x, out[4 * i + 1] = w[i].y, out[4 * i + 2] = w[i].z, out[4 * i + 3] = w[i].w;
    }
    return STA_OK;
  }
  if (which == STA_WORK_DKDV || which == STA_WORK_DQ) {
    const std::vector<int2> &w = which == STA_WORK_DKDV ? pl->work_kv : pl->work_q;
    *n_items = w.size();
    if (!out) return STA_OK;
    if (cap_items < w.size()) return STA_ERR_INVALID_ARG;
    for (size_t i = 0; i < w.size(); ++i) out[2 * i] = w[i].x, out[2 * i + 1] = w[i].y;
    return STA_OK;
  }
  return STA_ERR_INVALID_ARG;
}

sta_status sta_plan_launches(sta_plan_t pl, int32_t *forward, int32_t *backward) {
  if (!pl) return STA_ERR_INVALID_ARG;
  const int n_work = (int)pl->work.size();
  const bool gather = !pl->tiled && pl->kv_mode != sta::kKvRaster;  // permute Q, K, V (and dO) first
  if (forward) {
    int f = gather ? 3 : 0;
    f += (n_work - pl->n_work_lone > 0 ? 1 : 0) + (pl->n_work_lone > 0 ? 1 : 0);
    *forward = f;
  }
  if (backward) {
    int b = 0;
    if (!pl->inv_off.empty()) {
      b = (gather ? 4 : 0) + 1;  // D / LSE preprocess
      b += pl->work_kv.empty() ? 0 : 1;
      b += pl->work_q.empty() ? 0 : 1;
    }
    *backward = b;
  }
  return STA_OK;
}

sta_status sta_plan_kv_tiles(sta_plan_t pl, int32_t head, int32_t *out, size_t cap, size_t *n) {
  if (!pl || !n || head < 0 || head >= pl->g.Hh) return STA_ERR_INVALID_ARG;
  const int per = pl->count[head];
  *n = (size_t)pl->g.n_tiles * per;
  if (!out) return STA_OK;
  if (cap < *n) return STA_ERR_INVALID_ARG;
  for (int q = 0; q < pl->g.n_tiles; ++q)
    std::memcpy(out + (size_t)q * per, &pl->kv_list[((size_t)head * pl->g.n_tiles + q) * pl->kv_stride],
                per * sizeof(int32_t));
  return STA_OK;
}

sta_status sta_plan_q_tiles(sta_plan_t pl, int32_t head, int32_t *offsets, int32_t *indices, size_t cap,
                            size_t *n_indices) {
  if (!pl || head < 0 || head >= pl->g.Hh) return STA_ERR_INVALID_ARG;
  if (pl->inv_off.empty()) return STA_ERR_INVALID_ARG;  // plan built without STA_PROBLEM_BACKWARD
  const int32_t *off = &pl->inv_off[(size_t)head * (pl->g.n_tiles + 1)];
  const size_t n = (size_t)(off[pl->g.n_tiles] - off[0]);
  if (n_indices) *n_indices = n;
  if (offsets)
    for (int k = 0; k <= pl->g.n_tiles; ++k) offsets[k] = off[k] - off[0];
  if (indices) {
    if (cap < n) return STA_ERR_INVALID_ARG;
    std::memcpy(indices, &pl->inv_idx[off[0]], n * sizeof(int32_t));
  }
  return STA_OK;
}

sta_status sta_permute(sta_plan_t pl, const void *src, void *dst, int32_t inverse, void *stream) {
  if (!pl || !src || !dst || pl->host_only) return STA_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return STA_ERR_ALIGNMENT;
  const size_t bytes = tensor_bytes(pl);
  const char *s = static_cast<const char *>(src), *d = static_cast<const char *>(dst);
  if (s < d + bytes && d < s + bytes) return STA_ERR_INVALID_ARG;
  if (const sta_status dev_st = check_device(pl)) return dev_st;
  sta::PermuteParams pp{};
  pp.g = pl->g;
  pp.src = src;
  pp.dst = dst;
  pp.inverse = inverse ? 1 : 0;
  if (sta::launch_permute(pp, pl->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STA_ERR_CUDA;
  return STA_OK;
}

sta_status sta_forward(sta_plan_t pl, const void *q, const void *k, const void *v, void *o, float *lse,
                       void *workspace, size_t ws_bytes, void *stream_, uint32_t flags) {
  if (!pl || !q || !k || !v || !o || pl->host_only) return STA_ERR_INVALID_ARG;
  if (flags & ~STA_CALL_CHECK) return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return STA_ERR_ALIGNMENT;
  if (!workspace || ws_bytes < fwd_workspace(pl)) return STA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return STA_ERR_ALIGNMENT;
  if (const sta_status dev_st = check_device(pl)) return dev_st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char *ws = static_cast<char *>(workspace);
  int *status = reinterpret_cast<int *>(ws);

  const void *qbase = q, *kbase = k, *vbase = v;
  if (!pl->tiled && pl->kv_mode != sta::kKvRaster) {
    // Tiles are not readable as TMA boxes of the raster tensor: gather Q, K
    // and V tile-major into the workspace first.
    char *dst = ws + kStatusBytes;
    const void *src[3] = {q, k, v};
    const void **base[3] = {&qbase, &kbase, &vbase};
    for (int i = 0; i < 3; ++i) {
      sta::PermuteParams pp{};
      pp.g = pl->g;
      pp.inverse = 0;
      pp.src = src[i], pp.dst = dst + i * tensor_bytes(pl);
      if (sta::launch_permute(pp, pl->num_sms, stream) != cudaSuccess) return STA_ERR_CUDA;
      *base[i] = pp.dst;
    }
  }
  if (flags & STA_CALL_CHECK)
    if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return STA_ERR_CUDA;
  const ForwardMaps maps = forward_maps(pl, qbase, kbase, vbase);
  if (!maps.ok) return STA_ERR_CUDA;
  const sta_status st = enqueue_forward(pl, maps, q, o, lse, status, stream, pl->d_work, (int)pl->work.size(),
                                        pl->n_work_lone);
  if (st != STA_OK) return st;
  return finish_call(pl, workspace, stream, flags);
}

sta_status sta_plan_host_workspace_size(sta_plan_t pl, size_t *bytes) {
  if (!pl || !bytes) return STA_ERR_INVALID_ARG;
  *bytes = host_workspace(pl);
  return STA_OK;
}

sta_status sta_forward_host(sta_plan_t pl, const void *q, const void *k, const void *v, void *o, float *lse,
                            void *workspace, size_t ws_bytes, void *stream_, uint32_t flags) {
  if (!pl || !q || !k || !v || !o || pl->host_only) return STA_ERR_INVALID_ARG;
  if (flags & ~STA_CALL_CHECK) return STA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < host_workspace(pl)) return STA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return STA_ERR_ALIGNMENT;
  if (const sta_status dev_st = check_device(pl)) return dev_st;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  const size_t tb = tensor_bytes(pl), tb_r = round256(tb);
  char *ws = static_cast<char *>(workspace);
  char *dq = ws, *dk = ws + tb_r, *dv = ws + 2 * tb_r, *dout = ws + 3 * tb_r;
  float *dlse = reinterpret_cast<float *>(ws + 4 * tb_r);
  char *ws_fwd = ws + host_copies_bytes(pl);
  const size_t fwd_bytes = fwd_workspace(pl);
  const bool gather = !pl->tiled && pl->kv_mode != sta::kKvRaster;

  if (gather) {
    // no slice pipeline on these paths: whole tensors in, one sta_forward, whole outputs out
    if ((flags & STA_CALL_CHECK) && cudaMemsetAsync(ws_fwd, 0, sizeof(int), stream) != cudaSuccess)
      return STA_ERR_CUDA;
    if (cudaMemcpyAsync(dq, q, tb, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(dk, k, tb, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(dv, v, tb, cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return STA_ERR_CUDA;
    sta_status st = sta_forward(pl, dq, dk, dv, dout, lse ? dlse : nullptr, ws_fwd, fwd_bytes, stream, 0);
    if (st != STA_OK) return st;
    if (cudaMemcpyAsync(o, dout, tb, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return STA_ERR_CUDA;
    if (lse && cudaMemcpyAsync(lse, dlse, lse_bytes(pl), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
      return STA_ERR_CUDA;
    return finish_call(pl, ws_fwd, stream, flags);
  }

  // Slice groups: the inputs of group g + 1 cross the bus while group g is
  // computed, and group g's outputs come back while later groups run.
  const int groups = (int)pl->group_slice.size() - 1;
  const size_t slice_bytes = (size_t)pl->g.N * pl->g.d * 2, slice_lse = (size_t)pl->g.N * 4;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> ev(2 * groups + 2, nullptr);  // in[g], comp[g], start, done
  auto cleanup = [&]() {
    for (cudaEvent_t e : ev)
      if (e) cudaEventDestroy(e);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
  };
  bool ok = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (size_t i = 0; i < ev.size() && ok; ++i) ok = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) == cudaSuccess;
  cudaEvent_t *ev_in = ev.data(), *ev_comp = ev.data() + groups, ev_start = ev[2 * groups], ev_done = ev[2 * groups + 1];
  int *status = reinterpret_cast<int *>(ws_fwd);
  if (ok && (flags & STA_CALL_CHECK)) ok = cudaMemsetAsync(status, 0, sizeof(int), stream) == cudaSuccess;
  ok = ok && cudaEventRecord(ev_start, stream) == cudaSuccess && cudaStreamWaitEvent(s_in, ev_start, 0) == cudaSuccess &&
       cudaStreamWaitEvent(s_out, ev_start, 0) == cudaSuccess;
  for (int gi = 0; gi < groups && ok; ++gi) {
    const size_t off = (size_t)pl->group_slice[gi] * slice_bytes;
    const size_t n = (size_t)(pl->group_slice[gi + 1] - pl->group_slice[gi]) * slice_bytes;
    ok = cudaMemcpyAsync(dq + off, static_cast<const char *>(q) + off, n, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaMemcpyAsync(dk + off, static_cast<const char *>(k) + off, n, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaMemcpyAsync(dv + off, static_cast<const char *>(v) + off, n, cudaMemcpyHostToDevice, s_in) == cudaSuccess &&
         cudaEventRecord(ev_in[gi], s_in) == cudaSuccess;
  }
  const ForwardMaps maps = forward_maps(pl, dq, dk, dv);
  ok = ok && maps.ok;
  sta_status st = STA_OK;
  for (int gi = 0; gi < groups && ok; ++gi) {
    ok = cudaStreamWaitEvent(stream, ev_in[gi], 0) == cudaSuccess;
    if (ok) {
      st = enqueue_forward(pl, maps, dq, dout, lse ? dlse : nullptr, status, stream,
                           pl->d_work_host + pl->group_off[gi], pl->group_off[gi + 1] - pl->group_off[gi],
                           pl->group_lone[gi]);
      ok = st == STA_OK && cudaEventRecord(ev_comp[gi], stream) == cudaSuccess;
    }
  }
  for (int gi = 0; gi < groups && ok; ++gi) {
    const size_t s0 = pl->group_slice[gi], ns = pl->group_slice[gi + 1] - s0;
    ok = cudaStreamWaitEvent(s_out, ev_comp[gi], 0) == cudaSuccess &&
         cudaMemcpyAsync(static_cast<char *>(o) + s0 * slice_bytes, dout + s0 * slice_bytes, ns * slice_bytes,
                         cudaMemcpyDeviceToHost, s_out) == cudaSuccess;
    if (ok && lse)
      ok = cudaMemcpyAsync(lse + s0 * pl->g.N, dlse + s0 * pl->g.N, ns * slice_lse, cudaMemcpyDeviceToHost, s_out) ==
           cudaSuccess;
  }
  ok = ok && cudaEventRecord(ev_done, s_out) == cudaSuccess && cudaStreamWaitEvent(stream, ev_done, 0) == cudaSuccess;
  cleanup();  // destruction waits for the enqueued work on the device side
  if (!ok) return st != STA_OK ? st : STA_ERR_CUDA;
  return finish_call(pl, ws_fwd, stream, flags);
}

sta_status sta_backward(sta_plan_t pl, const void *q, const void *k, const void *v, const void *o,
                        const float *lse, const void *dout, void *dq, void *dk, void *dv, void *workspace,
                        size_t ws_bytes, void *stream_, uint32_t flags) {
  const void *tensors[9] = {q, k, v, o, lse, dout, dq, dk, dv};
  sta_status st = sta::check_backward_call(pl, tensors, flags);
  if (st != STA_OK) return st;
  if (!workspace || ws_bytes < bwd_workspace(pl)) return STA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return STA_ERR_ALIGNMENT;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  char *ws = static_cast<char *>(workspace);
  int *status = reinterpret_cast<int *>(ws);
  float *lse2_t = reinterpret_cast<float *>(ws + kStatusBytes);
  float *dd_t = reinterpret_cast<float *>(ws + kStatusBytes + bwd_vec_bytes(pl));

  const void *base[4] = {q, k, v, dout};
  const bool raster = pl->kv_mode == sta::kKvRaster;
  if (!pl->tiled && !raster) {
    char *dst = ws + bwd_gather_offset(pl);
    for (int i = 0; i < 4; ++i) {
      sta::PermuteParams pp{};
      pp.g = pl->g;
      pp.inverse = 0;
      pp.src = base[i], pp.dst = dst + i * tensor_bytes(pl);
      if (sta::launch_permute(pp, pl->num_sms, stream) != cudaSuccess) return STA_ERR_CUDA;
      base[i] = pp.dst;
    }
  }
  CUtensorMap maps[4];
  for (int i = 0; i < 4; ++i) {
    const bool ok = raster ? make_map_raster(&maps[i], base[i], pl) : make_map_tiled(&maps[i], base[i], pl);
    if (!ok) return STA_ERR_CUDA;
  }

  sta::BwdParams bp{};
  bp.g = pl->g;
  bp.tiled = pl->tiled ? 1 : 0;
  bp.nqb = (pl->g.tau + 127) / 128;
  bp.kv_mode = raster ? sta::kKvRaster : sta::kKvTiled;
  bp.piece_rows = pl->piece_rows;
  bp.box_w = pl->box_w, bp.box_h = pl->box_h, bp.box_t = pl->box_t;
  bp.box_panels = box_panels(pl);
  bp.oob_coord = raster ? pl->g.T * pl->g.B * pl->g.Hh : pl->g.B * pl->g.Hh * pl->g.N;
  bp.o = o, bp.dout = dout, bp.lse = lse;
  bp.lse2_t = lse2_t, bp.dd_t = dd_t;
  bp.aug = reinterpret_cast<uint8_t *>(ws + bwd_aug_offset(pl));
  bp.dq = dq, bp.dk = dk, bp.dv = dv;
  bp.kv_list = pl->d_kv_list, bp.kv_count = pl->d_count, bp.kv_stride = pl->kv_stride;
  bp.inv_off = pl->d_inv_off, bp.inv_idx = pl->d_inv_idx;
  bp.work_kv = pl->d_work_kv, bp.n_work_kv = (int)pl->work_kv.size();
  bp.work_q = pl->d_work_q, bp.n_work_q = (int)pl->work_q.size();
  bp.scale = pl->scale;
  bp.scale_log2 = pl->scale * 1.4426950408889634f;
  bp.status = status;
  bp.wait_limit_ns = g_wait_limit_ns;

  if (flags & STA_CALL_CHECK)
    if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return STA_ERR_CUDA;
  if (sta::launch_backward(bp, maps[0], maps[1], maps[2], maps[3], pl->num_sms, stream) != cudaSuccess)
    return STA_ERR_CUDA;
  return finish_call(pl, workspace, stream, flags);
}

}  // extern "C"
