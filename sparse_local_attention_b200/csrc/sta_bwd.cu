// sta_bwd.cu -- Sliding Tile Attention backward kernels for sm_100a.
//
// Gradients of the windowed attention ("Fast Video Generation with Sliding
// Tile Attention", Abstract: fine-tuning with STA).  With P = softmax of the
// scores inside each query's window (recomputed from the forward LSE) and
// D_i = sum_c dO_ic O_ic:
//   dV = P^T dO,  dS = P o (dO V^T - D),  dK = scale dS^T Q,  dQ = scale dS K,
// every sum running only over the (query, key) pairs of the window.
//
// Three launches, no atomics (the result is deterministic):
//   1. bwd_pre: D and LSE * log2(e) per query row, stored tile-major so a
//      128-row block reads them as one contiguous run, and per query block
//      the operand panel that carries -LSE / scale and -D into the dK/dV
//      kernel's products (BwdParams::aug).
//   2. bwd_dkdv: one 128-row key block per work item (key-block major).  K and
//      V stay in shared memory; the query blocks of every query tile whose
//      window holds the key tile (the planner's inverse lists) stream through
//      a ring.  S^T = K Q^T and dP^T = V dO^T land in TMEM; the elementwise
//      warps (thread = key row) turn them into P^T and dS^T (bf16), then
//      dV += P^T dO and dK += dS^T Q accumulate in TMEM with P^T / dS^T as the
//      TMEM A operand.  With head dim 64, P^T / dS^T have TMEM columns of their
//      own and S^T / dP^T of the next query chunk are computed while the
//      elementwise warps work; with head dim 128 they are written over the
//      columns they come from.
//   3. bwd_dq: one 128-row query block per work item (query-block major, the
//      forward KV-tile lists).  S = Q K^T and dP = dO V^T per 128-key chunk,
//      dS in TMEM columns of its own, dQ += dS K; the next chunk's S / dP are
//      computed while the elementwise warps work on this one.
// Warp roles: NG warpgroups of elementwise warps that split each chunk's
// columns (thread = TMEM lane = row) -- four with head dim 64, two with head
// dim 128, whose in-place P^T / dS^T path needs 64 columns per thread -- then
// one TMA producer warp and one MMA issuer warp.  Every wait is bounded.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "sta_common.cuh"
#include "sta_kernels.h"

namespace sta {
namespace {

constexpr int kBM = 128;
constexpr int kMaxCoords = 1024;

// Warp roles of the dK/dV and dQ kernels: NG warpgroups of elementwise warps
// (warpgroup e takes columns [e kBM / NG, (e + 1) kBM / NG) of every chunk;
// thread = TMEM lane = row), then the TMA producer warp and the MMA warp.
// More warpgroups give each sub-partition more warps to hide the latency of
// the elementwise pass and each thread fewer live registers.
template <int NG>
struct Roles {
  static constexpr int kGroups = NG;
  static constexpr int kMathWarps = 4 * NG;
  static constexpr int kProducerWarp = kMathWarps, kMmaWarp = kMathWarps + 1;
  static constexpr int kThreads = 32 * (kMathWarps + 2);
  static constexpr int kCols = kBM / NG;  // chunk columns per warpgroup
  static_assert(kCols % 32 == 0, "whole 32-column TMEM loads");
};
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kAugPanelBytes = 4096, kAugBlockBytes = kAugPanelBytes;  // see BwdParams::aug
// pairs of exponentials (of every 8) that the dK/dV and the dQ elementwise
// passes compute on the FMA pipe (exp2_fma2) instead of the MUFU
constexpr int kEmuDkdv = 0, kEmuDq = 0;

// x as two bf16 (hi, lo) with hi + lo = x to within 2^-16 relative: hi in
// bits 0..15 (element 0 of the panel row), lo in bits 16..31 (element 1).
__device__ __forceinline__ uint32_t hi_lo_bf16(float x) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
  return uint32_t(__bfloat16_as_ushort(hi)) | (uint32_t(__bfloat16_as_ushort(lo)) << 16);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// LSE * log2(e) and D are stored per 128-row query block: run of block qb of
// tile t of slice bh = ((bh * n_tiles + t) * nqb + qb) * 128.  Rows past the
// tile's end hold LSE = +inf and D = 0, so P = exp2(S - LSE) is 0 there and
// no mask is needed.
__device__ __forceinline__ long long vec_run(const BwdParams &p, int bh, int tile, int qb) {
  return (((long long)bh * p.g.n_tiles + tile) * p.nqb + qb) * kBM;
}

// The elementwise pass over one thread's 64 columns of S and dP (TMEM lane =
// row): four quarters of 16 columns, the TMEM load of quarter q + 1 in flight
// while quarter q is computed.  compute(q, s, dp) gets the quarter's raw fp32
// bits; after_reads() runs once every load has completed (the columns may then
// be overwritten).
template <typename Compute, typename AfterReads>
__device__ __forceinline__ void quarters_pipelined(uint32_t s_addr, uint32_t dp_addr, Compute &&compute,
                                                   AfterReads &&after_reads) {
  uint32_t s0[16], d0[16], s1[16], d1[16];
  tmem_ld16(s_addr, s0);
  tmem_ld16(dp_addr, d0);
  tmem_ld_wait_regs(s0, d0);
  tmem_ld16(s_addr + 16, s1);
  tmem_ld16(dp_addr + 16, d1);
  compute(0, s0, d0);
  tmem_ld_wait_regs(s1, d1);
  tmem_ld16(s_addr + 32, s0);
  tmem_ld16(dp_addr + 32, d0);
  compute(1, s1, d1);
  tmem_ld_wait_regs(s0, d0);
  tmem_ld16(s_addr + 48, s1);
  tmem_ld16(dp_addr + 48, d1);
  compute(2, s0, d0);
  tmem_ld_wait_regs(s1, d1);
  after_reads();
  compute(3, s1, d1);
}

// ----------------------------------------------------------------------- 1. preprocess
// A group of D / 8 lanes per row (16-byte loads of O and dO, the row's LSE
// loaded beside them), 32 / (D / 8) rows per warp and iteration.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p) {
  const Geometry &g = p.g;
  constexpr int kLanes = D / 8, kRows = 32 / kLanes;
  static_assert(kLanes >= 2 && kLanes <= 32 && 32 % kLanes == 0, "whole rows per warp");
  const int lane = threadIdx.x & 31, sub = lane / kLanes, part = lane % kLanes;
  const long long nrows = (long long)g.B * g.Hh * g.n_tiles * p.nqb * kBM;  // padded runs, a multiple of kRows
  const long long step = (long long)gridDim.x * (blockDim.x / 32) * kRows;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32 * kRows + sub; r < nrows; r += step) {
    const long long run = r / kBM;
    const long long bt = run / p.nqb;  // bh * n_tiles + tile
    const int o = (int)(run - bt * p.nqb) * kBM + (int)(r - run * kBM);
    const int bh = (int)(bt / g.n_tiles), tile = (int)(bt - (long long)bh * g.n_tiles);
    // rows past the tile's end: P = dS = 0 (LSE = +inf, D = 0)
    const bool valid = o < g.tau;
    float acc = 0.f, lse = 0.f;
    if (valid) {
      const long long tok = token_row(g, p.tiled, bh, tile, o);
      const uint4 a = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.o) + tok * D)[part];
      const uint4 b = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.dout) + tok * D)[part];
      if (part == 0) lse = p.lse[tok];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 af = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&av[e]));
        const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&bv[e]));
        acc = fmaf(af.x, bf.x, fmaf(af.y, bf.y, acc));
      }
    }
    // sum over the row's lane group (every lane of the warp takes part)
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (part == 0) {
      p.dd_t[r] = valid ? acc : 0.f;
      p.lse2_t[r] = valid ? lse * kLog2e : INFINITY;
    }
    // row i of the block's operand panel: parts 0 / 1 write its two halves;
    // S^T + (-LSE / scale) times scale_log2 is S^T scale_log2 - LSE log2 e
    if (part < 2) {
      const int i = (int)(r - run * kBM);
      uint4 *cell = reinterpret_cast<uint4 *>(p.aug + run * kAugBlockBytes + (i / 8) * 256 + part * 128 + (i % 8) * 16);
      *cell = part == 0 ? make_uint4(hi_lo_bf16(valid ? -lse / p.scale : -1e30f), valid ? hi_lo_bf16(-acc) : 0u, 0u, 0u)
                        : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// ----------------------------------------------------------------------- 2. dK, dV
// Elementwise warpgroups (warpgroup e = query columns [kCW e, kCW e + kCW) of
// each 128-query chunk, kCW = 32 with head dim 64 and 64 with head dim 128;
// thread = key row = TMEM lane), then the TMA producer and the MMA issuer.
// With head dim 64, P^T and dS^T get TMEM columns of their own, so S^T / dP^T
// of chunk i + 1 are computed while the elementwise warps work on chunk i;
// with head dim 128 the accumulators leave no room and P^T / dS^T are written
// over the S^T / dP^T columns they come from.
template <int D>
struct DkvCfg {
  static constexpr uint32_t kTile = kBM * D * 2;           // one 128-row operand tile
  static constexpr uint32_t kPanel = kBM * 128;
  static constexpr bool kSep = D == 64;                    // P^T, dS^T in columns of their own
  using R = Roles<kSep ? 4 : 2>;                           // the in-place path assumes two warpgroups
  static constexpr int kStages = D == 128 ? 2 : 5;
  static constexpr uint32_t kStage = 2 * kTile + kAugBlockBytes;  // Q, dO, the block's LSE / D panel
  // two selector panels: rows (1, 1, 0, ..., 0) pick -LSE / scale, rows
  // (0, 0, 1, 1, 0, ..., 0) pick -D out of the block's panel
  static constexpr uint32_t kOnes = 2 * kAugPanelBytes;
  // barriers: st_full[S] st_empty[S] kv_full kv_free s_full s_read p_ready pd_free acc_done acc_free drain
  static constexpr int kNumBars = 2 * kStages + 9;
  static constexpr uint32_t kSmem = 2 * kTile + kStages * kStage + kOnes + kNumBars * 8 + 64 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static constexpr uint32_t kTmS = 0, kTmDP = 128;
  static constexpr uint32_t kTmP = kSep ? 256 : kTmS, kTmDS = kSep ? 320 : kTmDP;
  static constexpr uint32_t kTmDV = kSep ? 384 : 256, kTmDK = kTmDV + D;
  static_assert(kTmDK + D <= 512, "TMEM budget");
};

template <int D>
__global__ void __launch_bounds__(DkvCfg<D>::R::kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_do,
                    const BwdParams p) {
  using C = DkvCfg<D>;
  using R = typename C::R;
  constexpr int kMathWarps = R::kMathWarps, kProducerWarp = R::kProducerWarp, kMmaWarp = R::kMmaWarp;
  constexpr int kCW = R::kCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *k_s = smem, *v_s = smem + C::kTile;
  uint8_t *stages = smem + 2 * C::kTile;  // [stage]{Q tile, dO tile, LSE / D panel}
  uint8_t *ones_s = stages + C::kStages * C::kStage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(ones_s + C::kOnes);
  uint64_t *st_full = bars, *st_empty = bars + C::kStages;
  uint64_t *kv_full = bars + 2 * C::kStages, *kv_free = kv_full + 1;
  uint64_t *s_full = kv_full + 2;    // S^T, dP^T of a chunk are in TMEM
  uint64_t *s_read = kv_full + 3;    // ... and have been read (separate P / dS columns only)
  uint64_t *p_ready = kv_full + 4;   // P^T, dS^T written
  uint64_t *pd_free = kv_full + 5;   // the dV / dK MMAs have read them (separate columns only)
  uint64_t *acc_done = kv_full + 6, *acc_free = kv_full + 7, *drain = kv_full + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geometry &g = p.g;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 1);
    }
    mbar_init(kv_full, 1);
    mbar_init(kv_free, 1);
    mbar_init(s_full, 1);
    mbar_init(s_read, kMathWarps);
    mbar_init(p_ready, kMathWarps);
    mbar_init(pd_free, 1);
    mbar_init(acc_done, 1);
    mbar_init(acc_free, kMathWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // the selector panels (layout of BwdParams::aug): every row of the first
  // is (1, 1, 0, ..., 0), of the second (0, 0, 1, 1, 0, ..., 0)
  for (int c = threadIdx.x; c < (int)(C::kOnes / 16); c += blockDim.x) {
    const bool first_half = ((c * 16) % 256) < 128, second_panel = c * 16 >= (int)kAugPanelBytes;
    const uint32_t ones = first_half ? 0x3F803F80u : 0u;  // two bf16 1.0
    reinterpret_cast<uint4 *>(ones_s)[c] = second_panel ? make_uint4(0u, ones, 0u, 0u) : make_uint4(ones, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};
  const int pieces = kBM / p.piece_rows;

  auto item_info = [&](int item, int &bh, int &ktile, int &kb, int &off0, int &nq) {
    const int2 wi = p.work_kv[item];
    bh = wi.x, ktile = wi.y / p.nqb, kb = wi.y % p.nqb;
    const int32_t *io = p.inv_off + (long long)(bh % g.Hh) * (g.n_tiles + 1) + ktile;
    off0 = io[0];
    nq = (io[1] - io[0]) * p.nqb;
  };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      tma_prefetch_desc(&tmap_do);
      uint32_t ld = 0, item_ctr = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_work_kv && ok; item += gridDim.x) {
        int bh, ktile, kb, off0, nq;
        item_info(item, bh, ktile, kb, off0, nq);
        if (!mbar_wait(kv_free, (item_ctr & 1) ^ 1, ctl, kErrBwdWait)) { ok = false; break; }
        mbar_arrive_expect_tx(kv_full, 2 * C::kTile);
        for (int pc = 0; pc < pieces; ++pc) {
          const int off = kb * kBM + pc * p.piece_rows;
          const int4 c = box_coords(p, bh, ktile, off, off < g.tau);
          load_box<D>(p, &tmap_k, k_s + pc * p.piece_rows * 128, c, kv_full);
          load_box<D>(p, &tmap_v, v_s + pc * p.piece_rows * 128, c, kv_full);
        }
        for (int i = 0; i < nq && ok; ++i) {
          const int qt = p.inv_idx[off0 + i / p.nqb], qb = i % p.nqb;
          const uint32_t st = ld % C::kStages, ph = (ld / C::kStages) & 1;
          if (!mbar_wait(&st_empty[st], ph ^ 1, ctl, kErrBwdWait)) { ok = false; break; }
          uint8_t *sb = stages + st * C::kStage;
          mbar_arrive_expect_tx(&st_full[st], C::kStage);
          for (int pc = 0; pc < pieces; ++pc) {
            const int off = qb * kBM + pc * p.piece_rows;
            const int4 c = box_coords(p, bh, qt, off, off < g.tau);
            load_box<D>(p, &tmap_q, sb + pc * p.piece_rows * 128, c, &st_full[st]);
            load_box<D>(p, &tmap_do, sb + C::kTile + pc * p.piece_rows * 128, c, &st_full[st]);
          }
          const long long run = vec_run(p, bh, qt, qb) / kBM;
          bulk_load(sb + 2 * C::kTile, p.aug + run * kAugBlockBytes, kAugBlockBytes, &st_full[st]);
          ++ld;
        }
        ++item_ctr;
      }
      if (!ok) {
        const uint32_t first = ld > (uint32_t)C::kStages ? ld - C::kStages : 0;
        for (uint32_t i = first; i < ld; ++i) drain_wait(&st_full[i % C::kStages], (i / C::kStages) & 1);
        if (item_ctr > 0) drain_wait(kv_full, (item_ctr - 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // the whole warp issues (converged, warp-uniform operands; one elected lane per MMA)
    {
      constexpr uint32_t idesc_ss = idesc_bf16_f32(kBM, kBM, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kBM, D, false, true);
      const uint64_t kd = smem_desc_sw128(smem_u32(k_s), 16, 1024), vd = smem_desc_sw128(smem_u32(v_s), 16, 1024);
      const uint64_t sk0 = smem_desc_sw128(smem_u32(stages), 16, 1024);              // K-major Q / dO
      const uint64_t sm0 = smem_desc_sw128(smem_u32(stages), C::kPanel, 1024);       // MN-major Q / dO
      const uint64_t ones_d = smem_desc_plain(smem_u32(ones_s), 128, 256);                    // selects -LSE / scale
      const uint64_t ones_dd = smem_desc_plain(smem_u32(ones_s) + kAugPanelBytes, 128, 256);  // selects -D
      const uint64_t aug0 = smem_desc_plain(smem_u32(stages + 2 * C::kTile), 128, 256);  // stage 0's LSE / D panel
      uint32_t ld = 0, item_ctr = 0, p_waits = 0, r_waits = 0;
      bool ok = true, issued = false;
      // S^T = K Q^T and dP^T = V dO^T for the chunk in stage `st`
      auto issue_s = [&](uint32_t st) {
        const uint32_t so = (st * C::kStage) >> 4, dso = (st * C::kStage + C::kTile) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * C::kPanel + (kk % 4) * 32) >> 4;
          mma_ss_w(tmem + C::kTmS, kd + off, sk0 + so + off, idesc_ss, kk > 0 ? 1u : 0u);
        }
        // + (-LSE / scale) per query column
        mma_ss_w(tmem + C::kTmS, ones_d, aug0 + ((st * C::kStage) >> 4), idesc_ss, 1u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * C::kPanel + (kk % 4) * 32) >> 4;
          mma_ss_w(tmem + C::kTmDP, vd + off, sk0 + dso + off, idesc_ss, kk > 0 ? 1u : 0u);
        }
        // - D per query column
        mma_ss_w(tmem + C::kTmDP, ones_dd, aug0 + ((st * C::kStage) >> 4), idesc_ss, 1u);
        mma_commit_w(s_full);
      };
      auto wait_stage = [&](uint32_t l) -> bool {
        if (!mbar_wait_w(&st_full[l % C::kStages], (l / C::kStages) & 1, ctl, kErrBwdWait)) return false;
        tc_fence_after();
        return true;
      };
      for (int item = blockIdx.x; item < p.n_work_kv && ok; item += gridDim.x) {
        int bh, ktile, kb, off0, nq;
        item_info(item, bh, ktile, kb, off0, nq);
        if (!mbar_wait_w(kv_full, item_ctr & 1, ctl, kErrBwdWait)) { ok = false; break; }
        tc_fence_after();
        if (!wait_stage(ld)) { ok = false; break; }
        issue_s(ld % C::kStages);
        issued = true;
        for (int i = 0; i < nq && ok; ++i) {
          const uint32_t cur = ld + i, st = cur % C::kStages;
          if (C::kSep && i + 1 < nq) {
            // the next chunk's S^T / dP^T as soon as this chunk's have been read
            if (!mbar_wait_w(s_read, r_waits & 1, ctl, kErrBwdWait)) { ok = false; break; }
            ++r_waits;
            tc_fence_after();
            if (!wait_stage(cur + 1)) { ok = false; break; }
            issue_s((cur + 1) % C::kStages);
          }
          if (!mbar_wait_w(p_ready, p_waits & 1, ctl, kErrBwdWait)) { ok = false; break; }
          ++p_waits;
          if (i == 0 && item_ctr > 0 && !mbar_wait_w(acc_free, (item_ctr - 1) & 1, ctl, kErrBwdWait)) { ok = false; break; }
          tc_fence_after();
          // dV += P^T dO and dK += dS^T Q (queries are the contraction, 8 steps of 16)
          const uint32_t so = (st * C::kStage) >> 4, dso = (st * C::kStage + C::kTile) >> 4;
#pragma unroll
          for (int kk = 0; kk < kBM / 16; ++kk) {
            const uint32_t off = (kk * 16 * 128) >> 4;
            mma_ts_w(tmem + C::kTmDV, tmem + C::kTmP + kk * 8, sm0 + dso + off, idesc_acc, (i > 0 || kk > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < kBM / 16; ++kk) {
            const uint32_t off = (kk * 16 * 128) >> 4;
            mma_ts_w(tmem + C::kTmDK, tmem + C::kTmDS + kk * 8, sm0 + so + off, idesc_acc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_w(&st_empty[st]);
          if (C::kSep) mma_commit_w(pd_free);
          if (i + 1 == nq) mma_commit_w(kv_free);
          if (!C::kSep && i + 1 < nq) {
            // P^T / dS^T live in the S^T / dP^T columns: the next S^T / dP^T
            // are issued after the MMAs that read them (in-order execution)
            if (!wait_stage(cur + 1)) { ok = false; break; }
            issue_s((cur + 1) % C::kStages);
          }
        }
        if (!ok) break;
        ld += nq;
        mma_commit_w(acc_done);
        ++item_ctr;
      }
      if (!ok && issued) {
        mma_commit_w(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // elementwise warps: thread = key row of the block = TMEM lane; warpgroup
    // e owns query columns [kCW e, kCW e + kCW)
    const int e = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const float2 sl2x2 = make_float2(p.scale_log2, p.scale_log2);
    uint32_t s_waits = 0, f_waits = 0, item_ctr = 0, gchunk = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_work_kv && ok; item += gridDim.x) {
      int bh, ktile, kb, off0, nq;
      item_info(item, bh, ktile, kb, off0, nq);
      const int krow = kb * kBM + row;
      const bool row_valid = krow < g.tau;
      for (int i = 0; i < nq; ++i, ++gchunk) {
        bool okw = mbar_wait_w(s_full, s_waits & 1, ctl, kErrBwdWait);
        ++s_waits;
        okw = __all_sync(0xffffffffu, okw);
        // P^T = 2^(S^T scale_log2) and dS^T = P^T dP^T for this warpgroup's
        // kCW query columns, packed to bf16.  The MMAs have already added
        // -LSE / scale to S^T and -D to dP^T from the operand panels (query
        // rows past a tile's end get -1e30 and 0: P = dS = 0 there).
        uint32_t pp[kCW / 32][16], pd[kCW / 32][16];
        // columns q0 .. q0 + 2 n - 1 (of the warpgroup's kCW) from raw S^T / dP^T bits
        auto pds = [&](int q0, int n, const uint32_t *rs, const uint32_t *rd) {
#pragma unroll
          for (int k = 0; k < n; ++k) {
            const int w = q0 / 2 + k;  // packed column
            const float2 t = mul2(make_float2(__uint_as_float(rs[2 * k]), __uint_as_float(rs[2 * k + 1])), sl2x2);
            const float2 pr = (w % 8 >= 8 - kEmuDkdv) ? exp2_fma2(t) : make_float2(ex2_approx(t.x), ex2_approx(t.y));
            const float2 dr = mul2(pr, make_float2(__uint_as_float(rd[2 * k]), __uint_as_float(rd[2 * k + 1])));
            pp[w >> 4][w & 15] = pack_bf16(pr.x, pr.y);
            pd[w >> 4][w & 15] = pack_bf16(dr.x, dr.y);
          }
        };
        if constexpr (C::kSep) {
          // S^T and dP^T are read in one batch and their columns released at
          // once, before any arithmetic: the MMA warp computes the next
          // chunk's S^T / dP^T while this one is worked on.
          static_assert(kCW == 32, "one 32-column load of each");
          if (okw) {
            tc_fence_after();
            const uint32_t base = tmem + lane_off + kCW * e;
            uint32_t rs[32], rd[32];
            tmem_ld32(base + C::kTmS, rs);
            tmem_ld32(base + C::kTmDP, rd);
            tmem_ld_wait();
            reg_fence32(rs);
            reg_fence32(rd);
            if (i + 1 < nq) {
              tc_fence_before();
              warp_arrive(s_read, lane);
            }
            pds(0, 16, rs, rd);
          }
        } else {
          // P^T / dS^T are written over S^T / dP^T, so their columns are not
          // released early: four quarters, the next quarter's load in flight
          static_assert(kCW == 64, "the in-place path runs two warpgroups");
          if (okw) {
            tc_fence_after();
            const uint32_t base = tmem + lane_off + 64 * e;
            quarters_pipelined(
                base + C::kTmS, base + C::kTmDP,
                [&](int qt, const uint32_t(&rs)[16], const uint32_t(&rd)[16]) { pds(16 * qt, 8, rs, rd); },
                [&]() {});
          }
          // both warpgroups have read their S^T / dP^T columns before either
          // writes P^T / dS^T over the first half of them
          okw = named_bar_and(1, 32 * kMathWarps, okw);
        }
        if (!okw) { ok = false; break; }
        if (C::kSep && gchunk > 0) {
          // the dV / dK MMAs of the previous chunk have read P^T / dS^T
          bool okf = mbar_wait_w(pd_free, f_waits & 1, ctl, kErrBwdWait);
          ++f_waits;
          okf = __all_sync(0xffffffffu, okf);
          if (!okf) { ok = false; break; }
          tc_fence_after();
        }
        const uint32_t pbase = tmem + lane_off + (kCW / 2) * e;
#pragma unroll
        for (int h = 0; h < kCW / 32; ++h) {
          tmem_st16(pbase + C::kTmP + 16 * h, pp[h]);
          tmem_st16(pbase + C::kTmDS + 16 * h, pd[h]);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(p_ready, lane);
      }
      if (!ok) break;
      // epilogue: the first half of the warpgroups writes dV, the second half
      // scale * dK (rows of this key block), each warpgroup kOut columns
      bool oke = mbar_wait_w(acc_done, item_ctr & 1, ctl, kErrBwdWait);
      oke = __all_sync(0xffffffffu, oke);
      if (!C::kSep) oke = named_bar_and(1, 32 * kMathWarps, oke);
      if (!oke) { ok = false; break; }
      tc_fence_after();
      constexpr int kHalf = R::kGroups / 2, kOut = D / kHalf;
      static_assert(kOut % 32 == 0, "whole 32-column TMEM loads");
      const int which = e / kHalf, part = e % kHalf;
      const long long tok = row_valid ? token_row(g, p.tiled, bh, ktile, krow) : 0;
      const uint32_t col = (which ? C::kTmDK : C::kTmDV) + part * kOut;
      const float mul = which ? p.scale : 1.f;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(which ? p.dk : p.dv) + tok * D + part * kOut);
#pragma unroll
      for (int c = 0; c < kOut / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + col + c * 32, r);
        tmem_ld_wait();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(r[8 * v + 0]) * mul, __uint_as_float(r[8 * v + 1]) * mul);
            w.y = pack_bf16(__uint_as_float(r[8 * v + 2]) * mul, __uint_as_float(r[8 * v + 3]) * mul);
            w.z = pack_bf16(__uint_as_float(r[8 * v + 4]) * mul, __uint_as_float(r[8 * v + 5]) * mul);
            w.w = pack_bf16(__uint_as_float(r[8 * v + 6]) * mul, __uint_as_float(r[8 * v + 7]) * mul);
            dst[c * 4 + v] = w;
          }
        }
      }
      tc_fence_before();
      warp_arrive(acc_free, lane);
      ++item_ctr;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------- 3. dQ
// Elementwise warpgroups (warpgroup e = key columns [kCW e, kCW e + kCW) of
// each 128-key chunk, kCW = 32 with head dim 64 and 64 with head dim 128;
// thread = query row), then the producer and the MMA warp.  dS has TMEM
// columns of its own, so S / dP of chunk j + 1 are computed while the
// elementwise warps work on chunk j.
template <int D>
struct DqCfg {
  static constexpr uint32_t kTile = kBM * D * 2;
  static constexpr uint32_t kPanel = kBM * 128;
  static constexpr int kSlots = D == 128 ? 4 : 8;
  using R = Roles<D == 64 ? 4 : 2>;
  // barriers: full[S] empty[S] q_full q_free s_full s_read ds_ready ds_free acc_done acc_free drain
  static constexpr int kNumBars = 2 * kSlots + 9;
  static constexpr uint32_t kSmem = (2 + kSlots) * kTile + kNumBars * 8 + 64 + 16 + kMaxCoords * 16 + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static constexpr uint32_t kTmS = 0, kTmDP = 128, kTmDS = 256, kTmDQ = 320;
  static_assert(kTmDQ + D <= 512, "TMEM budget");
};

template <int D>
__global__ void __launch_bounds__(DqCfg<D>::R::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_do,
                  const BwdParams p) {
  using C = DqCfg<D>;
  using R = typename C::R;
  constexpr int kMathWarps = R::kMathWarps, kProducerWarp = R::kProducerWarp, kMmaWarp = R::kMmaWarp;
  constexpr int kCW = R::kCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_s = smem, *do_s = smem + C::kTile, *slots = smem + 2 * C::kTile;
  uint64_t *bars = reinterpret_cast<uint64_t *>(slots + C::kSlots * C::kTile);
  uint64_t *full = bars, *empty = bars + C::kSlots;
  uint64_t *q_full = bars + 2 * C::kSlots, *q_free = q_full + 1;
  uint64_t *s_full = q_full + 2;    // S, dP of a chunk are in TMEM
  uint64_t *s_read = q_full + 3;    // ... and have been read
  uint64_t *ds_ready = q_full + 4;  // dS written
  uint64_t *ds_free = q_full + 5;   // the dQ MMAs have read it
  uint64_t *acc_done = q_full + 6, *acc_free = q_full + 7, *drain = q_full + 8;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int4 *s_coord = reinterpret_cast<int4 *>((reinterpret_cast<uintptr_t>(tmem_slot) + 64 + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geometry &g = p.g;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    mbar_init(s_full, 1);
    mbar_init(s_read, kMathWarps);
    mbar_init(ds_ready, kMathWarps);
    mbar_init(ds_free, 1);
    mbar_init(acc_done, 1);
    mbar_init(acc_free, kMathWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};
  const int pieces = kBM / p.piece_rows;

  struct Item {
    int bh, tile, qb, head, nkeys, nc;
  };
  auto item_info = [&](int item) {
    const int2 wi = p.work_q[item];
    Item it;
    it.bh = wi.x, it.tile = wi.y / p.nqb, it.qb = wi.y % p.nqb, it.head = it.bh % g.Hh;
    it.nkeys = p.kv_count[it.head] * g.tau;
    it.nc = (it.nkeys + kBM - 1) / kBM;
    return it;
  };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      tma_prefetch_desc(&tmap_do);
    }
    uint32_t ld = 0, item_ctr = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_work_q && ok; item += gridDim.x) {
      const Item it = item_info(item);
      const int32_t *list = p.kv_list + ((long long)it.head * g.n_tiles + it.tile) * p.kv_stride;
      const int nbox = it.nc * pieces;
      const bool staged = nbox <= kMaxCoords;
      auto kv_coord = [&](int e) -> int4 {
        const int key = (e / pieces) * kBM + (e % pieces) * p.piece_rows;
        const bool valid = key < it.nkeys;
        const int li = key / g.tau;
        return box_coords(p, it.bh, valid ? __ldg(list + li) : 0, key - li * g.tau, valid);
      };
      __syncwarp();
      if (staged)
        for (int e = lane; e < nbox; e += 32) s_coord[e] = kv_coord(e);
      __syncwarp();
      if (lane == 0) {
        if (!mbar_wait(q_free, (item_ctr & 1) ^ 1, ctl, kErrBwdWait)) ok = false;
        if (ok) {
          mbar_arrive_expect_tx(q_full, 2 * C::kTile);
          for (int pc = 0; pc < pieces; ++pc) {
            const int off = it.qb * kBM + pc * p.piece_rows;
            const int4 c = box_coords(p, it.bh, it.tile, off, off < g.tau);
            load_box<D>(p, &tmap_q, q_s + pc * p.piece_rows * 128, c, q_full);
            load_box<D>(p, &tmap_do, do_s + pc * p.piece_rows * 128, c, q_full);
          }
        }
        for (int s = 0; s < 2 * it.nc && ok; ++s) {
          const int chunk = s >> 1, is_v = s & 1;
          const uint32_t slot = ld % C::kSlots, phase = (ld / C::kSlots) & 1;
          if (!mbar_wait(&empty[slot], phase ^ 1, ctl, kErrBwdWait)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[slot], C::kTile);
          for (int pc = 0; pc < pieces; ++pc) {
            const int e = chunk * pieces + pc;
            load_box<D>(p, is_v ? &tmap_v : &tmap_k, slots + slot * C::kTile + pc * p.piece_rows * 128,
                        staged ? s_coord[e] : kv_coord(e), &full[slot]);
          }
          ++ld;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ld = __shfl_sync(0xffffffffu, ld, 0);
      ++item_ctr;
    }
    if (!ok && lane == 0) {
      const uint32_t first = ld > (uint32_t)C::kSlots ? ld - C::kSlots : 0;
      for (uint32_t i = first; i < ld; ++i) drain_wait(&full[i % C::kSlots], (i / C::kSlots) & 1);
      if (item_ctr > 0) drain_wait(q_full, (item_ctr - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // the whole warp issues (converged, warp-uniform operands; one elected lane per MMA)
    {
      constexpr uint32_t idesc_ss = idesc_bf16_f32(kBM, kBM, false, false);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(kBM, D, false, true);
      const uint64_t qd = smem_desc_sw128(smem_u32(q_s), 16, 1024), dod = smem_desc_sw128(smem_u32(do_s), 16, 1024);
      const uint64_t sk0 = smem_desc_sw128(smem_u32(slots), 16, 1024);         // K-major K / V
      const uint64_t sm0 = smem_desc_sw128(smem_u32(slots), C::kPanel, 1024);  // MN-major K
      uint32_t ld = 0, item_ctr = 0, ds_waits = 0, r_waits = 0;
      bool ok = true, issued = false;
      // S = Q K^T and dP = dO V^T for chunk j (ring loads lk = K_j, lk + 1 = V_j)
      auto issue_s = [&](uint32_t lk) -> bool {
        const uint32_t lv = lk + 1, ks = lk % C::kSlots, vs = lv % C::kSlots;
        if (!mbar_wait_w(&full[ks], (lk / C::kSlots) & 1, ctl, kErrBwdWait) ||
            !mbar_wait_w(&full[vs], (lv / C::kSlots) & 1, ctl, kErrBwdWait))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * C::kPanel + (kk % 4) * 32) >> 4;
          mma_ss_w(tmem + C::kTmS, qd + off, sk0 + ((ks * C::kTile) >> 4) + off, idesc_ss, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * C::kPanel + (kk % 4) * 32) >> 4;
          mma_ss_w(tmem + C::kTmDP, dod + off, sk0 + ((vs * C::kTile) >> 4) + off, idesc_ss, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(s_full);
        mma_commit_w(&empty[vs]);  // V is read by dP only
        return true;
      };
      for (int item = blockIdx.x; item < p.n_work_q && ok; item += gridDim.x) {
        const Item it = item_info(item);
        if (!mbar_wait_w(q_full, item_ctr & 1, ctl, kErrBwdWait)) { ok = false; break; }
        tc_fence_after();
        if (!issue_s(ld)) { ok = false; break; }
        issued = true;
        if (it.nc == 1) mma_commit_w(q_free);
        for (int j = 0; j < it.nc && ok; ++j) {
          const uint32_t lk = ld + 2 * j;
          if (j + 1 < it.nc) {
            // the next chunk's S / dP as soon as this chunk's have been read
            if (!mbar_wait_w(s_read, r_waits & 1, ctl, kErrBwdWait)) { ok = false; break; }
            ++r_waits;
            tc_fence_after();
            if (!issue_s(lk + 2)) { ok = false; break; }
            if (j + 2 == it.nc) mma_commit_w(q_free);  // Q and dO are no longer read
          }
          if (!mbar_wait_w(ds_ready, ds_waits & 1, ctl, kErrBwdWait)) { ok = false; break; }
          ++ds_waits;
          if (j == 0 && item_ctr > 0 && !mbar_wait_w(acc_free, (item_ctr - 1) & 1, ctl, kErrBwdWait)) { ok = false; break; }
          tc_fence_after();
          // dQ += dS K (keys are the contraction)
          const uint32_t ks = lk % C::kSlots;
#pragma unroll
          for (int kk = 0; kk < kBM / 16; ++kk)
            mma_ts_w(tmem + C::kTmDQ, tmem + C::kTmDS + kk * 8, sm0 + ((ks * C::kTile + kk * 16 * 128) >> 4), idesc_dq,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(&empty[ks]);
          mma_commit_w(ds_free);
        }
        if (!ok) break;
        ld += 2 * it.nc;
        mma_commit_w(acc_done);
        ++item_ctr;
      }
      if (!ok && issued) {
        mma_commit_w(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // elementwise warps: thread = query row = TMEM lane; warpgroup e owns key
    // columns [kCW e, kCW e + kCW)
    const int e = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const float2 sl2x2 = make_float2(p.scale_log2, p.scale_log2);
    uint32_t s_waits = 0, f_waits = 0, item_ctr = 0, gchunk = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_work_q && ok; item += gridDim.x) {
      const Item it = item_info(item);
      const int qrow = it.qb * kBM + row;
      const bool row_valid = qrow < g.tau;
      const long long lo = vec_run(p, it.bh, it.tile, it.qb) + row;
      const float lse2 = p.lse2_t[lo], dd = p.dd_t[lo];
      const float2 nlse2 = make_float2(-lse2, -lse2), ndd = make_float2(-dd, -dd);
      for (int j = 0; j < it.nc; ++j, ++gchunk) {
        bool okw = mbar_wait_w(s_full, s_waits & 1, ctl, kErrBwdWait);
        ++s_waits;
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) { ok = false; break; }
        tc_fence_after();
        // dS for this warpgroup's kCW key columns, packed to bf16.  S and dP
        // are read in one batch so the MMA warp can reuse their columns at once;
        // keys past the list's end (only in the last chunk) are masked.
        const int kvalid = it.nkeys - j * kBM - kCW * e;
        const bool whole = kvalid >= kCW;
        uint32_t rs[kCW / 32][32], rd[kCW / 32][32];
        const uint32_t base = tmem + lane_off + kCW * e;
#pragma unroll
        for (int h = 0; h < kCW / 32; ++h) tmem_ld32(base + C::kTmS + 32 * h, rs[h]);
#pragma unroll
        for (int h = 0; h < kCW / 32; ++h) tmem_ld32(base + C::kTmDP + 32 * h, rd[h]);
        tmem_ld_wait();
        if (j + 1 < it.nc) {
          tc_fence_before();
          warp_arrive(s_read, lane);
        }
        uint32_t pd[kCW / 32][16];
#pragma unroll
        for (int hf = 0; hf < kCW / 32; ++hf) {
          float2 dr[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 t = fma2(make_float2(__uint_as_float(rs[hf][2 * k]), __uint_as_float(rs[hf][2 * k + 1])), sl2x2,
                                  nlse2);
            const float2 pr = (k % 8 >= 8 - kEmuDq) ? exp2_fma2(t) : make_float2(ex2_approx(t.x), ex2_approx(t.y));
            dr[k] = mul2(pr, add2(make_float2(__uint_as_float(rd[hf][2 * k]), __uint_as_float(rd[hf][2 * k + 1])), ndd));
          }
          if (!whole) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              if (32 * hf + 2 * k >= kvalid) dr[k].x = 0.f;
              if (32 * hf + 2 * k + 1 >= kvalid) dr[k].y = 0.f;
            }
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) pd[hf][k] = pack_bf16(dr[k].x, dr[k].y);
        }
        if (gchunk > 0) {
          // the dQ MMAs of the previous chunk have read dS
          bool okf = mbar_wait_w(ds_free, f_waits & 1, ctl, kErrBwdWait);
          ++f_waits;
          okf = __all_sync(0xffffffffu, okf);
          if (!okf) { ok = false; break; }
          tc_fence_after();
        }
#pragma unroll
        for (int h = 0; h < kCW / 32; ++h) tmem_st16(tmem + lane_off + C::kTmDS + (kCW / 2) * e + 16 * h, pd[h]);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(ds_ready, lane);
      }
      if (!ok) break;
      bool oke = mbar_wait_w(acc_done, item_ctr & 1, ctl, kErrBwdWait);
      oke = __all_sync(0xffffffffu, oke);
      if (!oke) { ok = false; break; }
      tc_fence_after();
      // warpgroup e writes dQ columns [e kOut, (e + 1) kOut)
      constexpr int kOut = D / R::kGroups;
      static_assert(kOut % 16 == 0, "whole 16-column TMEM loads");
      constexpr int kLd = kOut < 32 ? kOut : 32;  // columns per TMEM load
      const long long tok = row_valid ? token_row(g, p.tiled, it.bh, it.tile, qrow) : 0;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.dq) + tok * D + e * kOut);
      const float mul = p.scale;
#pragma unroll
      for (int c = 0; c < kOut / kLd; ++c) {
        uint32_t r[32];
        if constexpr (kLd == 32) {
          tmem_ld32(tmem + lane_off + C::kTmDQ + e * kOut + c * 32, r);
        } else {
          tmem_ld16(tmem + lane_off + C::kTmDQ + e * kOut + c * 16, *reinterpret_cast<uint32_t(*)[16]>(r));
        }
        tmem_ld_wait();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < kLd / 8; ++v) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(r[8 * v + 0]) * mul, __uint_as_float(r[8 * v + 1]) * mul);
            w.y = pack_bf16(__uint_as_float(r[8 * v + 2]) * mul, __uint_as_float(r[8 * v + 3]) * mul);
            w.z = pack_bf16(__uint_as_float(r[8 * v + 4]) * mul, __uint_as_float(r[8 * v + 5]) * mul);
            w.w = pack_bf16(__uint_as_float(r[8 * v + 6]) * mul, __uint_as_float(r[8 * v + 7]) * mul);
            dst[c * (kLd / 8) + v] = w;
          }
        }
      }
      tc_fence_before();
      warp_arrive(acc_free, lane);
      ++item_ctr;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_bwd_d(const BwdParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                         const CUtensorMap &tdo, int num_sms, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)DkvCfg<D>::kSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DqCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const long long rows = (long long)p.g.B * p.g.Hh * p.g.N;
  constexpr int kPreRows = 8 * (32 / (D / 8));  // rows per 256-thread block and iteration
  long long pre_blocks = (rows + kPreRows - 1) / kPreRows;
  if (pre_blocks > (long long)num_sms * 16) pre_blocks = (long long)num_sms * 16;
  bwd_pre_kernel<D><<<(int)pre_blocks, 256, 0, stream>>>(p);
  const int g1 = p.n_work_kv < num_sms ? p.n_work_kv : num_sms;
  if (g1 > 0) bwd_dkdv_kernel<D><<<g1, DkvCfg<D>::R::kThreads, DkvCfg<D>::kSmem, stream>>>(tq, tk, tv, tdo, p);
  const int g2 = p.n_work_q < num_sms ? p.n_work_q : num_sms;
  if (g2 > 0) bwd_dq_kernel<D><<<g2, DqCfg<D>::R::kThreads, DqCfg<D>::kSmem, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BwdParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                            const CUtensorMap &tmap_v, const CUtensorMap &tmap_do, int num_sms,
                            cudaStream_t stream) {
  if (p.g.d == 128) return launch_bwd_d<128>(p, tmap_q, tmap_k, tmap_v, tmap_do, num_sms, stream);
  if (p.g.d == 64) return launch_bwd_d<64>(p, tmap_q, tmap_k, tmap_v, tmap_do, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sta
