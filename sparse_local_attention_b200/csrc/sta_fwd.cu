// sta_fwd.cu -- fused Sliding Tile Attention forward kernel for sm_100a.
//
// What it computes ("Fast Video Generation with Sliding Tile Attention",
// Abstract; summary page, Methodology / Novelty): for each query tile, dense
// attention over the whole key tiles of its window, with no partly masked
// block.  The KV-tile list of each (head, query tile) comes from the planner.
//
// Design (B200):
//   * persistent grid, one CTA per SM, work items = (batch*head, query tile,
//     128-row query block), heaviest first;
//   * warp 8: TMA producer.  K and V chunks of 128 keys are gathered tile by
//     tile (a chunk may span several key tiles) into a ring of shared-memory
//     stages with 128-byte swizzle, in the order the MMA consumes them.  The
//     item's KV-tile list is staged in shared memory first, so no load waits
//     on a global read;
//   * warp 9: tcgen05 MMA issuer.  S = Q K^T with Q held in tensor memory
//     (A operand from TMEM, so only K is read from shared memory), two S
//     buffers in TMEM so the next S is computed while softmax runs, then
//     O += P V with P (bf16) from TMEM and V from shared memory.  P is
//     written over the first 64 columns of its own S buffer: tcgen05.mma
//     operations issued by one thread execute in order, so the P V of chunk c
//     has read P before the S of chunk c + 2 overwrites that buffer;
//   * warps 0-7: softmax, two warpgroups working on alternate chunks (chunk c
//     goes to warpgroup c % 2, which always uses S buffer c % 2).  Query row r
//     lives in TMEM lane r; a thread owns one whole row, so row max and sum
//     need no shuffles.  The running maximum is handed from one warpgroup to
//     the other through shared memory and an mbarrier, so one warpgroup's
//     exponentials overlap the other's loads and reductions.  fp32 online
//     softmax in the log2 domain with lazy rescaling of O (only when the
//     running max grows by more than 2^8); P is rounded to bf16 on the integer
//     pipe so the XU pipe only runs ex2.
//   * Tensor memory (512 columns): S0/P0 [0,128) S1/P1 [128,256) O [256,256+d)
//     Q [256+d, 256+1.5d).
// Every barrier wait is bounded; on a time-out the kernel records an error in
// the status word, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "sta_kernels.h"

namespace sta {
namespace {

constexpr int kBM = 128;  // query rows per block (MMA M)
constexpr int kBN = 128;  // keys per chunk (MMA N of Q K^T, K of P V)
constexpr int kThreads = 320;  // 8 softmax warps + producer + MMA
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kMaxList = 1024;  // KV-tile list entries staged in shared memory
constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;  // 0.2 s

template <int D>
struct FwdCfg {
  static constexpr int kSlots = D == 128 ? 6 : 10;
  static constexpr uint32_t kPanelBytes = kBN * 128;            // 128 rows x 64 bf16
  static constexpr uint32_t kSlotBytes = kBN * D * 2;          // one K or V chunk
  static constexpr int kPanels = D / 64;
  static constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO = 256;
  static constexpr uint32_t kTmQ = 256 + D;
  static constexpr uint32_t kTmCols = 512;
  // barriers: full[S] empty[S] s_full[2] p_ready pv_done[2] o_done q_ready o_free drain m_ready[2]
  static constexpr int kNumBars = 2 * kSlots + 12;
  static constexpr uint32_t kMiscBytes = 64;                       // tmem address, abort flag
  static constexpr uint32_t kXchgBytes = (2 * 128 + 4 * 128) * 4;  // m hand-over, epilogue (m, l)
  static constexpr uint32_t kListBytes = kMaxList * 4;
  static constexpr uint32_t kSmemBytes =
      kSlots * kSlotBytes + kNumBars * 8 + kMiscBytes + kXchgBytes + kListBytes + 1024;
  static_assert(kTmQ + D / 2 <= kTmCols, "TMEM budget");
};

__device__ __forceinline__ bool drain_wait(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > (long long)(2 * kDrainLimitNs)) return false;
  return true;
}

// Token index (in the tensor's own order) of row `o` of query tile `tile`.
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

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sta_fwd_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                   const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *slots = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kSlots * C::kSlotBytes);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kSlots;
  uint64_t *s_full = bars + 2 * C::kSlots;  // [2], buffer b <-> warpgroup b
  uint64_t *p_ready = s_full + 2;
  uint64_t *pv_done = p_ready + 1;          // [2], P V of chunk c -> pv_done[c % 2]
  uint64_t *o_done = pv_done + 2;           // last P V of an item
  uint64_t *q_ready = o_done + 1;
  uint64_t *o_free = q_ready + 1;
  uint64_t *drain = o_free + 1;
  uint64_t *m_ready = drain + 1;            // [2], running max published by warpgroup w
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *m_xchg = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(tmem_slot) + C::kMiscBytes);  // [2][128]
  float *e_xchg = m_xchg + 256;                                                                     // [2][2][128]
  int32_t *s_list = reinterpret_cast<int32_t *>(e_xchg + 512);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geometry &g = p.g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_ready, 4);  // the four warps of the warpgroup that owns the chunk
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(o_done, 1);
    mbar_init(q_ready, 8);
    mbar_init(o_free, 8);
    mbar_init(drain, 1);
    mbar_init(&m_ready[0], 4);
    mbar_init(&m_ready[1], 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
    }
    uint32_t ld = 0;
    bool ok = true;
    const int pieces = kBN / p.piece_rows;
    for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
      const int2 wi = p.work[item];
      const int bh = wi.x, tile = wi.y / p.nqb, head = bh % g.Hh;
      const int cnt = p.kv_count[head];
      const int nkeys = cnt * g.tau;
      const int nc = (nkeys + kBN - 1) / kBN;
      const int32_t *glist = p.kv_list + ((long long)head * g.n_tiles + tile) * p.kv_stride;
      const bool staged = cnt <= kMaxList;
      __syncwarp();
      if (staged)
        for (int i = lane; i < cnt; i += 32) s_list[i] = __ldg(glist + i);
      __syncwarp();
      if (lane == 0) {
        const int32_t *list = staged ? s_list : glist;
        // Loads in consumption order: K0, then (K_{j+1}, V_j) for every j.
        for (int s = 0; s < 2 * nc; ++s) {
          const int is_v = (s == 0) ? 0 : ((s & 1) == 0 || s == 2 * nc - 1) ? 1 : 0;
          int chunk;
          if (s == 0) chunk = 0;
          else if (s == 2 * nc - 1) chunk = nc - 1;
          else chunk = (s & 1) ? (s + 1) / 2 : s / 2 - 1;
          const CUtensorMap *map = is_v ? &tmap_v : &tmap_k;
          const uint32_t slot = ld % C::kSlots;
          const uint32_t phase = (ld / C::kSlots) & 1;
          if (!mbar_wait(&empty[slot], phase ^ 1, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[slot], C::kSlotBytes);
          uint8_t *dst = slots + slot * C::kSlotBytes;
          for (int pc = 0; pc < pieces; ++pc) {
            const int key = chunk * kBN + pc * p.piece_rows;
            const bool valid = key < nkeys;
            const int li = key / g.tau, off = key - (key / g.tau) * g.tau;
            const int ktile = valid ? list[li] : 0;
            const int boxes = C::kPanels / p.box_panels;
            for (int pn = 0; pn < boxes; ++pn) {
              uint8_t *pdst = dst + pn * C::kPanelBytes + pc * p.piece_rows * 128;
              if (p.kv_mode == kKvTiled) {
                const int y = valid ? bh * g.N + ktile * g.tau + off : p.oob_coord;
                if constexpr (D == 128) tma_load_3d(pdst, map, 0, y, pn, &full[slot]);
                else tma_load_2d(pdst, map, 0, y, &full[slot]);
              } else {
                const int kt = ktile / (g.GH * g.GW), kh = (ktile / g.GW) % g.GH, kw = ktile % g.GW;
                const int a = off / (g.th * g.tw), b = (off / g.tw) % g.th, c = off % g.tw;
                const int tz = valid ? bh * g.T + kt * g.tt + a : p.oob_coord;
                if constexpr (D == 128) tma_load_5d(pdst, map, 0, kw * g.tw + c, kh * g.th + b, tz, pn, &full[slot]);
                else tma_load_4d(pdst, map, 0, kw * g.tw + c, kh * g.th + b, tz, &full[slot]);
              }
            }
          }
          ++ld;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ld = __shfl_sync(0xffffffffu, ld, 0);
    }
    if (!ok && lane == 0) {
      // Let the copies already issued land before the CTA exits.
      const uint32_t first = ld > (uint32_t)C::kSlots ? ld - C::kSlots : 0;
      for (uint32_t i = first; i < ld; ++i) drain_wait(&full[i % C::kSlots], (i / C::kSlots) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t slots_addr = smem_u32(slots);
      uint32_t ld = 0, chunk_g = 0, item_ctr = 0;
      bool ok = true;
      bool issued = false;

      auto issue_s = [&](uint32_t gchunk) -> bool {
        const uint32_t slot = ld % C::kSlots, phase = (ld / C::kSlots) & 1;
        if (!mbar_wait(&full[slot], phase, ctl, kErrWaitMma)) return false;
        tc_fence_after();
        const uint32_t buf = gchunk & 1;
        const uint32_t d_tm = tmem + (buf ? C::kTmS1 : C::kTmS0);
        const uint32_t kbase = slots_addr + slot * C::kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a_tm = tmem + C::kTmQ + kk * 8;
          const uint64_t bdesc = smem_desc_sw128(kbase + (kk / 4) * C::kPanelBytes + (kk % 4) * 32, 16, 1024);
          mma_ts(d_tm, a_tm, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[buf]);
        mma_commit(&empty[slot]);
        ++ld;
        issued = true;
        return true;
      };
      auto issue_pv = [&](uint32_t gchunk, bool first, bool last) -> bool {
        const uint32_t slot = ld % C::kSlots, phase = (ld / C::kSlots) & 1;
        if (!mbar_wait(&full[slot], phase, ctl, kErrWaitMma)) return false;
        tc_fence_after();
        const uint32_t vbase = slots_addr + slot * C::kSlotBytes;
        const uint32_t p_tm = tmem + ((gchunk & 1) ? C::kTmS1 : C::kTmS0);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t a_tm = p_tm + kk * 8;
          const uint64_t bdesc = smem_desc_sw128(vbase + kk * 16 * 128, C::kPanelBytes, 1024);
          mma_ts(tmem + C::kTmO, a_tm, bdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&empty[slot]);
        mma_commit(&pv_done[gchunk & 1]);
        if (last) mma_commit(o_done);
        ++ld;
        issued = true;
        return true;
      };

      for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
        const int2 wi = p.work[item];
        const int head = wi.x % g.Hh;
        const int nkeys = p.kv_count[head] * g.tau;
        const int nc = (nkeys + kBN - 1) / kBN;
        if (!mbar_wait(q_ready, item_ctr & 1, ctl, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        ok = issue_s(chunk_g);
        if (ok && nc > 1) ok = issue_s(chunk_g + 1);
        for (int j = 0; j < nc && ok; ++j) {
          const uint32_t gc = chunk_g + j;
          if (!mbar_wait(p_ready, gc & 1, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          if (j == 0 && item_ctr > 0) {
            if (!mbar_wait(o_free, (item_ctr - 1) & 1, ctl, kErrWaitMma)) { ok = false; break; }
            tc_fence_after();
          }
          if (!issue_pv(gc, j == 0, j == nc - 1)) { ok = false; break; }
          if (j + 2 < nc && !issue_s(gc + 2)) { ok = false; break; }
        }
        chunk_g += nc;
        ++item_ctr;
      }
      if (!ok && issued) {
        // Wait for every MMA already issued before TMEM is released.
        mma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int wg = warp >> 2;                       // chunks c with c % 2 == wg
    const int quad = warp & 3;                      // TMEM lane quadrant
    const int row = quad * 32 + lane;               // query row = TMEM lane
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t s_col = wg ? C::kTmS1 : C::kTmS0;
    const float sl2 = p.scale_log2;
    uint32_t chunk_g = 0, item_ctr = 0;
    uint32_t s_waits = 0, pv_waits = 0, m_waits = 0;  // phases consumed on s_full[wg], pv_done[1-wg], m_ready[1-wg]
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
      const int2 wi = p.work[item];
      const int bh = wi.x, tile = wi.y / p.nqb, qb = wi.y % p.nqb, head = bh % g.Hh;
      const int nkeys = p.kv_count[head] * g.tau;
      const int nc = (nkeys + kBN - 1) / kBN;
      const int o_in_tile = qb * kBM + row;
      const bool row_valid = o_in_tile < g.tau;
      const long long tok = row_valid ? token_row(g, p.tiled, bh, tile, o_in_tile) : 0;

      // Q row -> TMEM (A operand of S = Q K^T), bf16 pairs packed per column;
      // warpgroup wg writes elements [wg*D/2, (wg+1)*D/2).
      {
        const uint4 *src =
            reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.q) + tok * D) + wg * (D / 16);
        if constexpr (D == 128) {
          uint32_t w[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = row_valid ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
            w[4 * v + 0] = x.x, w[4 * v + 1] = x.y, w[4 * v + 2] = x.z, w[4 * v + 3] = x.w;
          }
          tmem_st32(tmem + lane_off + C::kTmQ + wg * 32, w);
        } else {
          uint32_t w[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 x = row_valid ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
            w[4 * v + 0] = x.x, w[4 * v + 1] = x.y, w[4 * v + 2] = x.z, w[4 * v + 3] = x.w;
          }
          tmem_st16(tmem + lane_off + C::kTmQ + wg * 16, w);
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(q_ready, lane);
      }

      // The running max m is the same number in both warpgroups at every
      // chunk; each warpgroup keeps its own partial row sum l_w, expressed
      // relative to the m of the last chunk it processed (m_w).
      float m_w = -INFINITY, l_w = 0.f;
      // A failed wait is carried to the epilogue barrier (whose AND-reduction
      // makes the exit uniform); nobody may skip that named barrier.
      bool carry = true;
      for (int j = 0; j < nc; ++j) {
        const uint32_t gc = chunk_g + j;
        if ((int)(gc & 1) != wg) continue;
        if (!carry) continue;
        // ---- S_j
        bool okw = mbar_wait(&s_full[wg], s_waits & 1, ctl, kErrWaitSoftmax);
        ++s_waits;
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) { carry = false; continue; }
        tc_fence_after();
        float s[kBN];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          const uint32_t sb = tmem + lane_off + s_col;
          tmem_ld32(sb, r0);
          tmem_ld32(sb + 32, r1);
          tmem_ld32(sb + 64, r2);
          tmem_ld32(sb + 96, r3);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            s[i] = __uint_as_float(r0[i]);
            s[32 + i] = __uint_as_float(r1[i]);
            s[64 + i] = __uint_as_float(r2[i]);
            s[96 + i] = __uint_as_float(r3[i]);
          }
        }
        const int kvalid = nkeys - j * kBN;
        if (kvalid < kBN) {
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (i >= kvalid) s[i] = -INFINITY;
        }
        float t16[16];
#pragma unroll
        for (int a = 0; a < 16; ++a)
          t16[a] = max3(max3(s[8 * a], s[8 * a + 1], s[8 * a + 2]), max3(s[8 * a + 3], s[8 * a + 4], s[8 * a + 5]),
                        fmaxf(s[8 * a + 6], s[8 * a + 7]));
        float t4[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) t4[a] = fmaxf(fmaxf(t16[4 * a], t16[4 * a + 1]), fmaxf(t16[4 * a + 2], t16[4 * a + 3]));
        const float mloc = fmaxf(fmaxf(t4[0], t4[1]), fmaxf(t4[2], t4[3])) * sl2;

        // ---- running max: take the previous chunk's m from the other warpgroup
        float m_prev = -INFINITY;
        if (j > 0) {
          bool okm = mbar_wait(&m_ready[wg ^ 1], m_waits & 1, ctl, kErrWaitSoftmax);
          ++m_waits;
          okm = __all_sync(0xffffffffu, okm);
          if (!okm) { carry = false; continue; }
          m_prev = m_xchg[(wg ^ 1) * 128 + row];
        }
        const bool resc = mloc > m_prev + 8.0f;  // also true while m_prev == -inf
        const float m_new = resc ? mloc : m_prev;
        if (j + 1 < nc) {
          m_xchg[wg * 128 + row] = m_new;
          warp_arrive(&m_ready[wg], lane);
        }
        const bool warp_resc = __any_sync(0xffffffffu, resc) && j > 0;
        const float alpha_o = resc ? ex2_approx(m_prev - m_new) : 1.f;  // O rescale (j > 0)

        // ---- P = exp2(S * scale_log2 - m) as bf16 over the consumed S columns, row sum
        float ls[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) ls[a] = 0.f;
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float p0 = ex2_approx(fmaf(s[32 * c + i], sl2, -m_new));
            const float p1 = ex2_approx(fmaf(s[32 * c + i + 1], sl2, -m_new));
            ls[(i / 2) & 7] += p0 + p1;
            pk[i / 2] = pack_bf16_rna(p0, p1);
          }
          tmem_st16(tmem + lane_off + s_col + c * 16, pk);
        }
        const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        l_w = (m_w == m_new ? l_w : l_w * ex2_approx(m_w - m_new)) + lsum;
        m_w = m_new;

        // ---- O is complete up to the previous chunk once its P V is done
        if (gc > 0) {
          bool okp = mbar_wait(&pv_done[wg ^ 1], pv_waits & 1, ctl, kErrWaitSoftmax);
          ++pv_waits;
          okp = __all_sync(0xffffffffu, okp);
          if (!okp) { carry = false; continue; }
          tc_fence_after();
        }
        if (warp_resc) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + C::kTmO + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha_o);
            tmem_st32(tmem + lane_off + C::kTmO + c * 32, r);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(p_ready, lane);
      }
      chunk_g += nc;

      // ---- epilogue: O / l -> bf16 row (each warpgroup half of the columns), LSE
      bool oke = carry && mbar_wait(o_done, item_ctr & 1, ctl, kErrWaitEpilogue);
      oke = __all_sync(0xffffffffu, oke);
      e_xchg[(0 * 2 + wg) * 128 + row] = m_w;
      e_xchg[(1 * 2 + wg) * 128 + row] = l_w;
      if (!named_bar_and(1, kSoftmaxThreads, oke)) { ok = false; break; }
      tc_fence_after();
      const float m0 = e_xchg[row], m1 = e_xchg[128 + row];
      const float l0 = e_xchg[256 + row], l1 = e_xchg[384 + row];
      const float m_f = fmaxf(m0, m1);
      const float l_row = (l0 > 0.f ? l0 * ex2_approx(m0 - m_f) : 0.f) + (l1 > 0.f ? l1 * ex2_approx(m1 - m_f) : 0.f);
      const float inv_l = 1.f / l_row;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + tok * D) + wg * (D / 16);
      const uint32_t col_o = C::kTmO + wg * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + col_o + c * 32, r);
        tmem_ld_wait();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 x;
            x.x = pack_bf16(__uint_as_float(r[8 * v + 0]) * inv_l, __uint_as_float(r[8 * v + 1]) * inv_l);
            x.y = pack_bf16(__uint_as_float(r[8 * v + 2]) * inv_l, __uint_as_float(r[8 * v + 3]) * inv_l);
            x.z = pack_bf16(__uint_as_float(r[8 * v + 4]) * inv_l, __uint_as_float(r[8 * v + 5]) * inv_l);
            x.w = pack_bf16(__uint_as_float(r[8 * v + 6]) * inv_l, __uint_as_float(r[8 * v + 7]) * inv_l);
            dst[c * 4 + v] = x;
          }
        }
      }
      tc_fence_before();
      warp_arrive(o_free, lane);
      if (wg == 0 && row_valid && p.lse) p.lse[tok] = (m_f + __log2f(l_row)) * 0.69314718055994530942f;
      ++item_ctr;
      // e_xchg is rewritten by the next item's epilogue; make sure everyone
      // has read it first.
      named_bar_sync(2, kSoftmaxThreads);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

template <int D>
cudaError_t launch_fwd_d(const FwdParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int num_sms,
                         cudaStream_t stream) {
  using C = FwdCfg<D>;
  static bool attr_set = false;  // per process; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(sta_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = p.n_work < num_sms ? p.n_work : num_sms;
  if (grid <= 0) return cudaSuccess;
  sta_fwd_kernel<D><<<grid, kThreads, C::kSmemBytes, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward(const FwdParams &p, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v,
                           int num_sms, cudaStream_t stream) {
  if (p.g.d == 128) return launch_fwd_d<128>(p, tmap_k, tmap_v, num_sms, stream);
  if (p.g.d == 64) return launch_fwd_d<64>(p, tmap_k, tmap_v, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sta
