// sta_fwd_pair.cu -- Sliding Tile Attention forward on CTA pairs (sm_100a),
// for head dim 128 and tiles whose volume is a multiple of 128 tokens (the
// 720P video-latent workloads).  Same result as sta_fwd.cu.
//
// A cluster of two CTAs (on two SMs) takes a pair of 128-row query blocks of
// one query tile; both blocks attend to the same key tiles ("Fast Video
// Generation with Sliding Tile Attention", summary page, Methodology: dense
// attention between whole tiles).  The tensor-core work of the pair is issued
// as tcgen05 MMAs of the cta_group::2 kind (M = 256): CTA r holds query block r
// in its tensor memory, and each K/V chunk of 128 keys is split between the two
// shared memories -- CTA r loads keys [64 r, 64 r + 64) of K (both 64-column
// panels) and columns [64 r, 64 r + 64) of V (all 128 keys) -- so every SM
// brings in only half of each chunk.
//
// Per CTA: warps 0-7 softmax (two warpgroups on alternate chunks, thread =
// query row = TMEM lane, running max handed over through shared memory),
// warp 8 TMA producer, warp 9 MMA issuer (only the leader CTA issues).
// Tensor memory per CTA (512 columns): S0/P0 [0,128) S1/P1 [128,256)
// O [256,384) Q [384,448); with two S buffers the tensor core computes
// S(j + 1) while the softmax of chunk j runs.  P(j) is written over the first
// 64 columns of its S buffer; MMAs issued by one thread execute in order, so
// P V(j) has read P(j) before S(j + 2) overwrites that buffer.
// Cross-CTA signalling uses mbarrier arrivals and tcgen05.commit to the peer's
// shared::cluster addresses (no multicast).  Every wait is bounded.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "sta_common.cuh"
#include "sta_kernels.h"

namespace sta {
namespace {

constexpr int D = 128;
constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kMaxCoords = 2048;       // staged box coordinates (two per chunk)
constexpr int kSlots = 10;
constexpr uint32_t kSlotBytes = 16384;   // K half (64 keys x 128) or V half (128 keys x 64)
constexpr uint32_t kKPanelBytes = 64 * 128;
constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO = 256, kTmQ = 384, kTmCols = 512;
// barriers: full[S] empty[S] s_full[2] pv_done[2] o_done p_ready[2] q_ready o_free m_ready[2] drain
constexpr int kNumBars = 2 * kSlots + 12;
constexpr uint32_t kMiscBytes = 64;
constexpr uint32_t kXchgBytes = (2 * 128 + 4 * 128) * 4;
constexpr uint32_t kSmemBytes = kSlots * kSlotBytes + kNumBars * 8 + kMiscBytes + kXchgBytes + 16 +
                                kMaxCoords * 16 + 1024;

struct PairItem {
  int bh, tile, head, nkeys, nc;  // tile: whose KV-tile list the item walks
  int my_tile, my_qb;             // this CTA's query block (my_qb == -1: none)
};

__device__ __forceinline__ PairItem decode_pair(const FwdParams &p, int item) {
  const int4 wi = p.work[item];
  PairItem it;
  it.bh = wi.x;
  it.tile = wi.y / p.nqb;
  const int mine = cluster_ctarank() ? wi.z : wi.y;
  it.my_tile = mine >= 0 ? mine / p.nqb : it.tile;
  it.my_qb = mine >= 0 ? mine - it.my_tile * p.nqb : -1;
  it.head = it.bh % p.g.Hh;
  it.nkeys = p.kv_count[it.head] * p.g.tau;
  it.nc = (it.nkeys + kBN - 1) / kBN;
  return it;
}

// One TMA box (rows of a tile, as staged in `c`), completion counted on the
// leader's barrier.  K halves carry both 64-column panels; V halves one panel.
__device__ __forceinline__ void load_half(const FwdParams &p, const CUtensorMap *map, uint8_t *dst, int4 c,
                                          int panel, uint32_t bar_cluster) {
  if (p.kv_mode == kKvTiled) tma2_load_3d(dst, map, 0, c.x, panel, bar_cluster);
  else tma2_load_5d(dst, map, 0, c.x, c.y, c.z, panel, bar_cluster);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sta_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmap_kh, const __grid_constant__ CUtensorMap tmap_vh,
                        const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *slots = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(slots + kSlots * kSlotBytes);
  uint64_t *full = bars;                  // leader's are used: both CTAs' bytes
  uint64_t *empty = bars + kSlots;        // per CTA
  uint64_t *s_full = bars + 2 * kSlots;   // [2] per CTA
  uint64_t *pv_done = s_full + 2;         // [2] per CTA
  uint64_t *o_done = pv_done + 2;         // per CTA
  uint64_t *p_ready = o_done + 1;         // [2] leader: 8 warps (4 per CTA) per S buffer
  uint64_t *q_ready = p_ready + 2;        // leader: 16 warps
  uint64_t *o_free = q_ready + 1;         // leader: 16 warps
  uint64_t *m_ready = o_free + 1;         // [2] per CTA, between its two warpgroups
  uint64_t *drain = m_ready + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *m_xchg = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(tmem_slot) + kMiscBytes);  // [2][128]
  float *e_xchg = m_xchg + 256;                                                                   // [2][2][128]
  int4 *s_coord = reinterpret_cast<int4 *>((reinterpret_cast<uintptr_t>(e_xchg + 512) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
  const Geometry &g = p.g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&pv_done[x], 1);
      mbar_init(&m_ready[x], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(&p_ready[0], 8);
    mbar_init(&p_ready[1], 8);
    mbar_init(q_ready, 16);
    mbar_init(o_free, 16);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc2(tmem_slot, kTmCols);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};
  auto leader = [&](const void *local) { return mapa_shared(smem_u32(local), 0); };
  auto peer = [&](const void *local) { return mapa_shared(smem_u32(local), rank ^ 1); };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&tmap_kh);
      tma_prefetch_desc(&tmap_vh);
    }
    uint32_t ld = 0;
    bool ok = true;
    for (int item = cid; item < p.n_work && ok; item += ncl) {
      const PairItem it = decode_pair(p, item);
      const int32_t *list = p.kv_list + ((long long)it.head * g.n_tiles + it.tile) * p.kv_stride;
      const bool staged = 2 * it.nc <= kMaxCoords;
      // coordinates of this CTA's halves: e = 2 * chunk + (0: K rows, 1: V rows)
      auto coord = [&](int e) -> int4 {
        const int key0 = (e >> 1) * kBN;
        const int li = key0 / g.tau, off = key0 - li * g.tau;
        const int tile = __ldg(list + li);
        return box_coords(p, it.bh, tile, (e & 1) ? off : off + 64 * (int)rank, true);
      };
      __syncwarp();
      if (staged)
        for (int e = lane; e < 2 * it.nc; e += 32) s_coord[e] = coord(e);
      __syncwarp();
      if (lane == 0) {
        // consumption order: K0, then (K_{j+1}, V_j) for every j
        for (int s = 0; s < 2 * it.nc; ++s) {
          const int is_v = (s == 0) ? 0 : ((s & 1) == 0 || s == 2 * it.nc - 1) ? 1 : 0;
          int chunk;
          if (s == 0) chunk = 0;
          else if (s == 2 * it.nc - 1) chunk = it.nc - 1;
          else chunk = (s & 1) ? (s + 1) / 2 : s / 2 - 1;
          const uint32_t slot = ld % kSlots, phase = (ld / kSlots) & 1;
          if (!mbar_wait<true>(&empty[slot], phase ^ 1, ctl, kErrWaitProducer)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[slot], 2 * kSlotBytes);
          const int e = 2 * chunk + is_v;
          load_half(p, is_v ? &tmap_vh : &tmap_kh, slots + slot * kSlotBytes, staged ? s_coord[e] : coord(e),
                    is_v ? (int)rank : 0, leader(&full[slot]));
          ++ld;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ld = __shfl_sync(0xffffffffu, ld, 0);
    }
    if (!ok && lane == 0) {
      if (rank == 0) {
        const uint32_t first = ld > (uint32_t)kSlots ? ld - kSlots : 0;
        for (uint32_t i = first; i < ld; ++i) drain_wait(&full[i % kSlots], (i / kSlots) & 1);
      } else {
        // this CTA's copies complete on the leader's barriers: give them time to land
        const long long t0 = clock64();
        while (clock64() - t0 < 400000) {
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(2 * kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(2 * kBM, D, false, true);
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(slots), 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(slots), kKPanelBytes, 1024);
      uint32_t ld = 0, chunk_g = 0, item_ctr = 0;
      bool ok = true, issued = false;
      auto commit_both = [&](uint64_t *bar) {
        mma2_commit(smem_u32(bar));
        mma2_commit(peer(bar));
      };
      auto wait_full = [&](uint32_t slot_ld) -> bool {
        const uint32_t slot = slot_ld % kSlots, phase = (slot_ld / kSlots) & 1;
        if (!mbar_wait<true>(&full[slot], phase, ctl, kErrWaitMma)) return false;
        tc_fence_after();
        return true;
      };
      auto issue_s = [&](uint32_t gchunk) -> bool {
        if (!wait_full(ld)) return false;
        const uint32_t slot = ld % kSlots, buf = gchunk & 1;
        const uint64_t kd = kdesc0 + ((slot * kSlotBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma2_ts(tmem + (buf ? kTmS1 : kTmS0), tmem + kTmQ + kk * 8,
                  kd + (((kk / 4) * kKPanelBytes + (kk % 4) * 32) >> 4), idesc_s, kk > 0 ? 1u : 0u);
        commit_both(&s_full[buf]);
        commit_both(&empty[slot]);
        ++ld;
        issued = true;
        return true;
      };
      auto issue_pv = [&](uint32_t gchunk, bool first, bool last) -> bool {
        if (!wait_full(ld)) return false;
        const uint32_t slot = ld % kSlots, buf = gchunk & 1;
        const uint64_t vd = vdesc0 + ((slot * kSlotBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma2_ts(tmem + kTmO, tmem + (buf ? kTmS1 : kTmS0) + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_pv,
                  (first && kk == 0) ? 0u : 1u);
        commit_both(&empty[slot]);
        commit_both(&pv_done[buf]);
        if (last) commit_both(o_done);
        ++ld;
        issued = true;
        return true;
      };
      for (int item = cid; item < p.n_work && ok; item += ncl) {
        const PairItem it = decode_pair(p, item);
        if (!mbar_wait<true>(q_ready, item_ctr & 1, ctl, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        ok = issue_s(chunk_g);
        if (ok && it.nc > 1) ok = issue_s(chunk_g + 1);
        for (int j = 0; j < it.nc && ok; ++j) {
          const uint32_t gc = chunk_g + j;
          if (!mbar_wait<true>(&p_ready[gc & 1], (gc >> 1) & 1, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          if (j == 0 && item_ctr > 0) {
            if (!mbar_wait<true>(o_free, (item_ctr - 1) & 1, ctl, kErrWaitMma)) { ok = false; break; }
            tc_fence_after();
          }
          if (!issue_pv(gc, j == 0, j == it.nc - 1)) { ok = false; break; }
          if (j + 2 < it.nc && !issue_s(gc + 2)) { ok = false; break; }
        }
        chunk_g += it.nc;
        ++item_ctr;
      }
      if (!ok && issued) {
        mma2_commit(smem_u32(drain));
        drain_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-7 (both CTAs)
    const int wg = warp >> 2;          // chunks c with c % 2 == wg
    const int quad = warp & 3;         // TMEM lane quadrant
    const int row = quad * 32 + lane;  // query row of this CTA's block = TMEM lane
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t s_col = wg ? kTmS1 : kTmS0;
    const float sl2 = p.scale_log2;
    const uint32_t p_ready_l = leader(&p_ready[wg]), q_ready_l = leader(q_ready), o_free_l = leader(o_free);
    auto arrive_leader = [&](uint32_t bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(bar);
    };
    uint32_t chunk_g = 0, item_ctr = 0, s_waits = 0, m_waits = 0;
    bool ok = true;
    for (int item = cid; item < p.n_work && ok; item += ncl) {
      const PairItem it = decode_pair(p, item);
      const int o_in_tile = it.my_qb * kBM + row;  // negative when this CTA has no block
      const bool row_valid = it.my_qb >= 0 && o_in_tile < g.tau;
      const long long tok = row_valid ? token_row(g, p.tiled, it.bh, it.my_tile, o_in_tile) : 0;
      {
        // Q row -> TMEM; warpgroup wg writes elements [64 wg, 64 wg + 64)
        const uint4 *src =
            reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.q) + tok * D) + wg * 8;
        uint32_t w[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 x = row_valid ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
          w[4 * v + 0] = x.x, w[4 * v + 1] = x.y, w[4 * v + 2] = x.z, w[4 * v + 3] = x.w;
        }
        tmem_st32(tmem + lane_off + kTmQ + wg * 32, w);
        tmem_st_wait();
        tc_fence_before();
        arrive_leader(q_ready_l);
      }

      float m_w = -INFINITY, l_w = 0.f;
      bool carry = true;
      for (int j = 0; j < it.nc; ++j) {
        const uint32_t gc = chunk_g + j;
        if ((int)(gc & 1) != wg || !carry) continue;
        bool okw = mbar_wait<true>(&s_full[wg], s_waits & 1, ctl, kErrWaitSoftmax);
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
        float t16[16];
#pragma unroll
        for (int a = 0; a < 16; ++a)
          t16[a] = max3(max3(s[8 * a], s[8 * a + 1], s[8 * a + 2]), max3(s[8 * a + 3], s[8 * a + 4], s[8 * a + 5]),
                        fmaxf(s[8 * a + 6], s[8 * a + 7]));
        float t4[4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
          t4[a] = fmaxf(fmaxf(t16[4 * a], t16[4 * a + 1]), fmaxf(t16[4 * a + 2], t16[4 * a + 3]));
        const float mloc = fmaxf(fmaxf(t4[0], t4[1]), fmaxf(t4[2], t4[3])) * sl2;

        // running max of the previous chunk, from the other warpgroup
        float m_prev = -INFINITY;
        if (j > 0) {
          bool okm = mbar_wait<true>(&m_ready[wg ^ 1], m_waits & 1, ctl, kErrWaitSoftmax);
          ++m_waits;
          okm = __all_sync(0xffffffffu, okm);
          if (!okm) { carry = false; continue; }
          m_prev = m_xchg[(wg ^ 1) * 128 + row];
        }
        const bool resc = mloc > m_prev + 8.0f;  // also true while m_prev == -inf
        const float m_new = resc ? mloc : m_prev;
        if (j + 1 < it.nc) {
          m_xchg[wg * 128 + row] = m_new;
          warp_arrive(&m_ready[wg], lane);
        }
        const bool warp_resc = __any_sync(0xffffffffu, resc) && j > 0;
        const float alpha_o = resc ? ex2_approx(m_prev - m_new) : 1.f;

        // P = exp2(S * scale_log2 - m) as bf16 over the consumed S columns, row sum
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
            pk[i / 2] = pack_bf16(p0, p1);
          }
          tmem_st16(tmem + lane_off + s_col + c * 16, pk);
        }
        const float lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        l_w = (m_w == m_new ? l_w : l_w * ex2_approx(m_w - m_new)) + lsum;
        m_w = m_new;

        // Only a warp that rescales O waits for the previous P V (chunk gc - 1, the
        // other warpgroup's) to have landed in O; the others hand P over at once.
        // pv_done[b] completes once per chunk of parity b, so chunk gc - 1 is its
        // completion number (gc - 1) >> 1.  S(gc) being done means P V(gc - 2) is
        // (MMAs of one thread finish in issue order) and P V(gc + 1) cannot start
        // before this warp arrives below, so the barrier is at most one phase
        // short of that completion and the parity wait is exact.
        if (warp_resc) {
          bool okp = mbar_wait<true>(&pv_done[wg ^ 1], ((gc - 1) >> 1) & 1, ctl, kErrWaitSoftmax);
          okp = __all_sync(0xffffffffu, okp);
          if (!okp) { carry = false; continue; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + kTmO + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha_o);
            tmem_st32(tmem + lane_off + kTmO + c * 32, r);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        arrive_leader(p_ready_l);
      }
      chunk_g += it.nc;

      // epilogue: O / l -> bf16 row (each warpgroup half of the columns), LSE
      bool oke = carry && mbar_wait<true>(o_done, item_ctr & 1, ctl, kErrWaitEpilogue);
      oke = __all_sync(0xffffffffu, oke);
      e_xchg[wg * 128 + row] = m_w;
      e_xchg[(2 + wg) * 128 + row] = l_w;
      if (!named_bar_and(1, kSoftmaxThreads, oke)) { ok = false; break; }
      tc_fence_after();
      const float m0 = e_xchg[row], m1 = e_xchg[128 + row];
      const float l0 = e_xchg[256 + row], l1 = e_xchg[384 + row];
      const float m_f = fmaxf(m0, m1);
      const float l_row =
          (l0 > 0.f ? l0 * ex2_approx(m0 - m_f) : 0.f) + (l1 > 0.f ? l1 * ex2_approx(m1 - m_f) : 0.f);
      const float inv_l = 1.f / l_row;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + tok * D) + wg * 8;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + kTmO + wg * 64 + c * 32, r);
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
      arrive_leader(o_free_l);
      if (wg == 0 && row_valid && p.lse) p.lse[tok] = (m_f + __log2f(l_row)) * 0.69314718055994530942f;
      ++item_ctr;
      named_bar_sync(2, kSoftmaxThreads);  // e_xchg is read before the next item rewrites it
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // every pair MMA, remote arrival and copy of both CTAs is done
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem, kTmCols);
  }
}

}  // namespace

uint32_t forward_pair_smem_bytes() { return kSmemBytes; }

cudaError_t launch_forward_pair(const FwdParams &p, const CUtensorMap &tmap_kh, const CUtensorMap &tmap_vh,
                                int num_sms, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(sta_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int clusters = num_sms / 2;
  if (p.n_work < clusters) clusters = p.n_work;
  if (clusters <= 0) return cudaSuccess;
  sta_fwd_pair_kernel<<<2 * clusters, kThreads, kSmemBytes, stream>>>(tmap_kh, tmap_vh, p);
  return cudaGetLastError();
}

}  // namespace sta
