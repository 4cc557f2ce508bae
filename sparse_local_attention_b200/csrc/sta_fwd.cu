// sta_fwd.cu -- fused Sliding Tile Attention forward kernel for sm_100a.
//
// What it computes ("Fast Video Generation with Sliding Tile Attention",
// Abstract; summary page, Methodology / Novelty): for each query tile, dense
// attention over the whole key tiles of its window, with no partly masked
// block.  The KV-tile list of each (head, query tile) comes from the planner.
//
// Design (B200):
//   * persistent grid, one CTA per SM.  A work item is a pair of 128-row
//     query blocks (A, B) that attend to the same key tiles -- two blocks of
//     one query tile, or the last blocks of two tiles whose windows coincide
//     -- so every K/V chunk brought into shared memory serves 256 query rows.
//     A block left without a partner is a lone item; its key chunks are
//     divided between the two warpgroups (the first half to A, the rest to
//     B, both reading the same Q) and the epilogue merges the two partial
//     softmax states, so a lone block still keeps two MMA/softmax chains in
//     flight.  The two kinds of item run as two launches of two
//     instantiations (kMode 0 / 1), each over its part of the work list,
//     heaviest items first.
//   * warp 8: TMA producer.  Loads Q_A, Q_B (shared memory, 128-byte swizzle)
//     and streams K and V chunks of 128 keys into a ring of stages, gathering
//     them tile by tile from the KV-tile list.  At the start of an item the
//     whole warp turns the list into TMA box coordinates (one int4 per box,
//     shared by K and V), so issuing a load costs a shared-memory read.
//   * warp 9: tcgen05 MMA issuer.  S_X = Q_X K^T into TMEM, then O_X += P_X V
//     with P_X read from TMEM.  The two blocks ping-pong: while warpgroup A
//     runs the softmax of chunk j, the tensor core computes S_B(j), and so on.
//     P_X is written over the first 64 columns of S_X; tcgen05.mma operations
//     issued by one thread execute in order, so P V(j) has read P before the
//     S of chunk j + 1 overwrites that buffer.  What stands between the end
//     of a block's softmax pass and its next S is kept short: the ring slots
//     of a chunk are waited for before the softmax finishes, the P V products
//     of the first kLeadKeys keys are issued as soon as their P is written,
//     and the softmax takes S(j)'s arrival as proof that P V(j-1) is done.
//   * warps 0-3 / 4-7: softmax of block A / B.  Query row r lives in TMEM lane
//     r and a thread owns one whole row: row max and sum need no shuffles.
//     fp32 online softmax in the log2 domain with lazy rescaling of O (only
//     when the running max grows by more than 2^8).  ex2 runs on the XU pipe,
//     the bf16 packing (cvt) on another, so they overlap.
//   * Tensor memory (512 columns): S_A/P_A [0,128) S_B/P_B [128,256)
//     O_A [256,256+d) O_B [256+d,256+2d).
// Every barrier wait is bounded; on a time-out the kernel records an error in
// the status word, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "sta_kernels.h"
#include "sta_common.cuh"

namespace sta {
namespace {

constexpr int kBM = 128;  // query rows per block (MMA M)
constexpr int kBN = 128;  // keys per chunk (MMA N of Q K^T, K of P V)
constexpr int kThreads = 320;  // 8 softmax warps + producer + MMA
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kMaxCoords = 1024;  // per-item K/V box coordinates staged in shared memory

template <int D, int kMode>
struct FwdCfg {
  static constexpr uint32_t kPanelBytes = kBN * 128;  // 128 rows x 64 bf16
  static constexpr uint32_t kTileBytes = kBN * D * 2;  // one Q block or one K / V chunk
  static constexpr int kNumQ = kMode == 0 ? 2 : 1;     // Q blocks held (a lone block needs one)
  // K/V ring: what shared memory holds besides Q; a lone block's second K/V
  // stream gets the space of the Q block it does not need
  static constexpr int kSlots = (D == 128 ? 4 : 8) + (2 - kNumQ);
  static constexpr uint32_t kTmO0 = 256;  // O_X at kTmO0 + X * D; S_X at 128 * X
  static constexpr uint32_t kTmCols = 512;
  // P of a chunk's first kLeadKeys keys is published on its own (p_lead) and
  // its share of P V issued at once, so that only the rest of P V stands
  // between the end of the softmax and the next S (measured on B200: a lead of
  // 96 keys is the faster at head dim 128, 64 keys at head dim 64).
  static constexpr int kLeadKeys = D == 128 ? 96 : 64;
  static_assert(kLeadKeys % 32 == 0 && kLeadKeys < kBN, "whole 32-key groups of P");
  // barriers: full[S] empty[S] q_full q_free s_full[2] p_ready[2] pv_done[2] o_free[2] drain p_lead[2]
  static constexpr int kNumBars = 2 * kSlots + 13;
  static constexpr uint32_t kMiscBytes = 64 + 4 * 128 * 4;  // tmem address, abort flag, m/l exchange
  static constexpr uint32_t kListBytes = kMaxCoords * 16;
  static constexpr uint32_t kSmemBytes =
      (kNumQ + kSlots) * kTileBytes + kNumBars * 8 + kMiscBytes + 16 + kListBytes + 1024;
  static_assert(kTmO0 + 2 * D <= kTmCols, "TMEM budget");
};

struct ItemInfo {
  int bh, head, tile;      // tile: whose KV-tile list the item walks (block A's)
  int ta, qa, tb, qb;      // query block A = block qa of tile ta; B = block qb of tile tb
  bool has_b;              // a second query block shares the K/V chunks
  bool split;              // one query block, its chunks divided between the two warpgroups
  int nkeys, nc;
  int n0, n1, c1;          // chunks of warpgroup 0: 0 .. n0 - 1; of warpgroup 1: c1 .. c1 + n1 - 1
  __device__ __forceinline__ int n(int x) const { return x ? n1 : n0; }
  __device__ __forceinline__ int c0(int x) const { return x ? c1 : 0; }
};

// kMode 0: items of one or two query blocks whose chunks are shared; kMode 1:
// lone query blocks, their chunks split between the warpgroups when there are
// at least two.  The host launches one kernel per kind over its part of the
// work list, so that each instantiation carries only the code it runs.
template <int kMode>
__device__ __forceinline__ ItemInfo decode_item(const FwdParams &p, int item) {
  const int4 wi = p.work[item];
  ItemInfo it;
  it.bh = wi.x;
  it.ta = wi.y / p.nqb;
  it.qa = wi.y - it.ta * p.nqb;
  it.has_b = kMode == 0 && wi.z >= 0;
  it.tb = it.has_b ? wi.z / p.nqb : it.ta;
  it.qb = it.has_b ? wi.z - it.tb * p.nqb : it.qa;
  it.tile = it.ta;
  it.head = it.bh % p.g.Hh;
  it.nkeys = p.kv_count[it.head] * p.g.tau;
  it.nc = (it.nkeys + kBN - 1) / kBN;
  it.split = kMode == 1 && it.nc > 1;
  it.n0 = it.split ? (it.nc + 1) / 2 : it.nc;
  it.n1 = it.split ? it.nc - it.n0 : (it.has_b ? it.nc : 0);
  it.c1 = it.split ? it.n0 : 0;
  return it;
}

template <int D, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    sta_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const FwdParams p) {
  using C = FwdCfg<D, kMode>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_smem = smem;                                  // [kNumQ][D/64 panels][128 rows][64]
  uint8_t *slots = smem + C::kNumQ * C::kTileBytes;        // [kSlots][D/64][128][64]
  uint64_t *bars = reinterpret_cast<uint64_t *>(slots + C::kSlots * C::kTileBytes);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kSlots;
  uint64_t *q_full = bars + 2 * C::kSlots;  // Q_A (+ Q_B) landed
  uint64_t *q_free = q_full + 1;            // every S MMA of the item has completed
  uint64_t *s_full = q_free + 1;            // [2]
  uint64_t *p_ready = s_full + 2;           // [2]
  uint64_t *pv_done = p_ready + 2;          // [2]
  uint64_t *o_free = pv_done + 2;           // [2]
  uint64_t *drain = o_free + 2;
  uint64_t *p_lead = drain + 1;             // [2] P of the chunk's first kLeadKeys keys written
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *ml_xchg = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(tmem_slot) + 64);  // [m0 m1 l0 l1][128]
  int4 *s_coord =  // 16-byte aligned for the int4 accesses
      reinterpret_cast<int4 *>((reinterpret_cast<uintptr_t>(tmem_slot) + C::kMiscBytes + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geometry &g = p.g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_ready[x], 4);  // the four warps of the block's warpgroup
      mbar_init(&p_lead[x], 4);
      mbar_init(&pv_done[x], 1);
      mbar_init(&o_free[x], 4);
    }
    mbar_init(drain, 1);
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
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
    }
    uint32_t ld = 0, item_ctr = 0;
    bool ok = true;
    const int pieces = kBN / p.piece_rows;
    for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
      const ItemInfo it = decode_item<kMode>(p, item);
      const int32_t *list = p.kv_list + ((long long)it.head * g.n_tiles + it.tile) * p.kv_stride;
      const int nbox = it.nc * pieces;  // K/V boxes of the item (K and V share coordinates)
      const bool staged = nbox <= kMaxCoords;
      auto kv_coord = [&](int e) -> int4 {
        const int key = (e / pieces) * kBN + (e % pieces) * p.piece_rows;
        const bool valid = key < it.nkeys;
        const int li = key / g.tau;
        return box_coords(p, it.bh, valid ? __ldg(list + li) : 0, key - li * g.tau, valid);
      };
      __syncwarp();
      if (staged)
        for (int e = lane; e < nbox; e += 32) s_coord[e] = kv_coord(e);
      __syncwarp();
      if (lane == 0) {
        // Q_A, Q_B: once the previous item's S MMAs are done with them.
        if (!mbar_wait(q_free, (item_ctr & 1) ^ 1, ctl, kErrWaitProducer)) ok = false;
        if (ok) {
          mbar_arrive_expect_tx(q_full, (it.has_b ? 2 : 1) * C::kTileBytes);
          for (int x = 0; x < (it.has_b ? 2 : 1); ++x)
            for (int pc = 0; pc < pieces; ++pc) {
              const int off = (x ? it.qb : it.qa) * kBM + pc * p.piece_rows;
              load_box<D>(p, &tmap_q, q_smem + x * C::kTileBytes + pc * p.piece_rows * 128,
                          box_coords(p, it.bh, x ? it.tb : it.ta, off, off < g.tau), q_full);
            }
        }
        if constexpr (kMode == 0) {
          // K and V chunks in the order the MMA first uses them: K0 V0 K1 V1 ...
          for (int s = 0; s < 2 * it.nc && ok; ++s) {
            const int chunk = s >> 1, is_v = s & 1;
            const uint32_t slot = ld % C::kSlots, phase = (ld / C::kSlots) & 1;
            if (!mbar_wait(&empty[slot], phase ^ 1, ctl, kErrWaitProducer)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[slot], C::kTileBytes);
            uint8_t *dst = slots + slot * C::kTileBytes;
            for (int pc = 0; pc < pieces; ++pc) {
              const int e = chunk * pieces + pc;
              load_box<D>(p, is_v ? &tmap_v : &tmap_k, dst + pc * p.piece_rows * 128,
                          staged ? s_coord[e] : kv_coord(e), &full[slot]);
            }
            ++ld;
          }
        } else {
          // Lone block: with one chunk, K0 V0.  Split: K_A(0) K_B(0), then per
          // step j: V_A(j) K_A(j+1) V_B(j) K_B(j+1), warpgroup x's step j being
          // chunk c0(x) + j.
          auto emit = [&](int chunk, int is_v) -> bool {
            const uint32_t slot = ld % C::kSlots, phase = (ld / C::kSlots) & 1;
            if (!mbar_wait(&empty[slot], phase ^ 1, ctl, kErrWaitProducer)) return false;
            mbar_arrive_expect_tx(&full[slot], C::kTileBytes);
            uint8_t *dst = slots + slot * C::kTileBytes;
            for (int pc = 0; pc < pieces; ++pc) {
              const int e = chunk * pieces + pc;
              load_box<D>(p, is_v ? &tmap_v : &tmap_k, dst + pc * p.piece_rows * 128,
                          staged ? s_coord[e] : kv_coord(e), &full[slot]);
            }
            ++ld;
            return true;
          };
          const int nxk = it.split ? 2 : 1;  // K/V streams
          // step -1 loads each stream's first K; step j >= 0 its V(j), then K(j + 1)
#pragma unroll 1
          for (int st = -1; st < it.n0 && ok; ++st)
#pragma unroll 1
            for (int e = 0; e < 2 * nxk && ok; ++e) {
              const int x = e >> 1, is_v = (e & 1) ^ 1;
              const int j = is_v ? st : st + 1;  // step of the chunk this load serves
              if ((st < 0 && is_v) || j >= it.n(x)) continue;
              ok = emit(it.c0(x) + j, is_v);
            }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ld = __shfl_sync(0xffffffffu, ld, 0);
      ++item_ctr;
    }
    if (!ok && lane == 0) {
      // Let the copies already issued land before the CTA exits.
      const uint32_t first = ld > (uint32_t)C::kSlots ? ld - C::kSlots : 0;
      for (uint32_t i = first; i < ld; ++i) drain_wait(&full[i % C::kSlots], (i / C::kSlots) & 1);
      if (item_ctr > 0) drain_wait(q_full, (item_ctr - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (converged, operands warp-uniform); one
    // elected lane issues each MMA and commit.
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
      const uint32_t slots_addr = smem_u32(slots), q_addr = smem_u32(q_smem);
      uint32_t ld = 0, item_ctr = 0;
      uint32_t p_waits[2] = {0, 0}, o_waits[2] = {0, 0}, x_items[2] = {0, 0};
      bool ok = true, issued = false;

      // Shared-memory descriptors are built once; a k-step only adds to the
      // start-address field (bits 0..13, address >> 4), which cannot carry
      // because every operand lies below 256 KB.
      const uint64_t qdesc0 = smem_desc_sw128(q_addr, 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(slots_addr, 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(slots_addr, C::kPanelBytes, 1024);
      // S_X = Q_qx K^T for the K chunk in ring slot `slot` (qx = x, or 0 in a split item).
      auto mma_s = [&](int x, int qx, uint32_t slot) {
        const uint64_t qd = qdesc0 + ((qx * C::kTileBytes) >> 4), kd = kdesc0 + ((slot * C::kTileBytes) >> 4);
        const uint32_t d_tm = tmem + 128 * x;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * C::kPanelBytes + (kk % 4) * 32) >> 4;
          mma_ss_w(d_tm, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit_w(&s_full[x]);
      };
      // O_X += P_X V for the V chunk in ring slot `slot`, in two parts: the
      // first kLeadKeys keys as soon as the softmax has written P for them, the
      // rest (and the pv_done commit) once all of P is there.
      auto mma_pv = [&](int x, uint32_t slot, bool first, uint32_t ph) -> bool {
        const uint64_t vd = vdesc0 + ((slot * C::kTileBytes) >> 4);
        const uint32_t o_tm = tmem + C::kTmO0 + x * D, p_tm = tmem + 128 * x;
#pragma unroll
        for (int kk = 0; kk < C::kLeadKeys / 16; ++kk)
          mma_ts_w(o_tm, p_tm + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_pv, (first && kk == 0) ? 0u : 1u);
        if (!mbar_wait_w(&p_ready[x], ph, ctl, kErrWaitMma)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = C::kLeadKeys / 16; kk < kBN / 16; ++kk)
          mma_ts_w(o_tm, p_tm + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_pv, 1u);
        mma_commit_w(&pv_done[x]);
        return true;
      };
      auto wait_slot = [&](uint32_t slot_ld) -> bool {
        const uint32_t slot = slot_ld % C::kSlots, phase = (slot_ld / C::kSlots) & 1;
        if (!mbar_wait_w(&full[slot], phase, ctl, kErrWaitMma)) return false;
        tc_fence_after();
        return true;
      };

      if constexpr (kMode == 0)
        for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
          const ItemInfo it = decode_item<kMode>(p, item);
          const int nx = it.has_b ? 2 : 1;
          if (!mbar_wait_w(q_full, item_ctr & 1, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          // chunk 0: S_A(0) [, S_B(0)]
          const uint32_t k0 = ld;
          if (!wait_slot(k0)) { ok = false; break; }
          for (int x = 0; x < nx; ++x) mma_s(x, x, k0 % C::kSlots);
          issued = true;
          mma_commit_w(&empty[k0 % C::kSlots]);
          if (it.nc == 1) mma_commit_w(q_free);
          for (int j = 0; j < it.nc && ok; ++j) {
            const uint32_t vj = k0 + 2 * j + 1, kn = k0 + 2 * j + 2;  // V_j, K_{j+1} load indices
            // V_j and K_{j+1} land long before they are used: wait for them here,
            // while the softmax works, not between P V(j) and S(j + 1)
            if (!wait_slot(vj) || (j + 1 < it.nc && !wait_slot(kn))) { ok = false; break; }
            for (int x = 0; x < nx; ++x) {
              const uint32_t ph = p_waits[x] & 1;
              if (!mbar_wait_w(&p_lead[x], ph, ctl, kErrWaitMma)) { ok = false; break; }
              ++p_waits[x];
              tc_fence_after();
              if (j == 0 && x_items[x] > 0) {
                // the previous item of this block has read O_X in its epilogue
                if (!mbar_wait_w(&o_free[x], o_waits[x] & 1, ctl, kErrWaitMma)) { ok = false; break; }
                ++o_waits[x];
                tc_fence_after();
              }
              if (!mma_pv(x, vj % C::kSlots, j == 0, ph)) { ok = false; break; }
              if (x == nx - 1) mma_commit_w(&empty[vj % C::kSlots]);
              if (j + 1 < it.nc) {
                mma_s(x, x, kn % C::kSlots);
                if (x == nx - 1) {
                  mma_commit_w(&empty[kn % C::kSlots]);
                  if (j + 2 == it.nc) mma_commit_w(q_free);
                }
              }
            }
          }
          ld = k0 + 2 * it.nc;
          for (int x = 0; x < nx; ++x) ++x_items[x];
          ++item_ctr;
        }
      else
        for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
          const ItemInfo it = decode_item<kMode>(p, item);
          const int nx = it.split ? 2 : 1;
          if (!mbar_wait_w(q_full, item_ctr & 1, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          uint32_t l = ld, kslot = 0, vslot = 0;
          int s_left = it.nc;  // S groups still to issue (one per chunk)
          // Each warpgroup has its own K/V stream: every chunk takes the next ring slot.
          auto take = [&](uint32_t &slot) -> bool {
            if (!wait_slot(l)) return false;
            slot = l++;
            return true;
          };
          auto release = [&](uint32_t slot) { mma_commit_w(&empty[slot % C::kSlots]); };
          auto s_group_done = [&]() {
            if (--s_left == 0) mma_commit_w(q_free);  // Q is no longer read
          };
          // first chunk of each warpgroup
          for (int x = 0; x < nx && ok; ++x) {
            if (!take(kslot)) { ok = false; break; }
            mma_s(x, 0, kslot % C::kSlots);
            issued = true;
            release(kslot);
            s_group_done();
          }
          for (int j = 0; j < it.n(0) && ok; ++j) {
            for (int x = 0; x < nx; ++x) {
              if (j >= it.n(x)) continue;
              // V(j) and K(j + 1) of this stream, waited for while the softmax
              // works rather than between P V(j) and S(j + 1)
              if (!take(vslot) || (j + 1 < it.n(x) && !take(kslot))) { ok = false; break; }
              const uint32_t ph = p_waits[x] & 1;
              if (!mbar_wait_w(&p_lead[x], ph, ctl, kErrWaitMma)) { ok = false; break; }
              ++p_waits[x];
              tc_fence_after();
              if (j == 0 && x_items[x] > 0) {
                // the previous item of this warpgroup has read O_X in its epilogue
                if (!mbar_wait_w(&o_free[x], o_waits[x] & 1, ctl, kErrWaitMma)) { ok = false; break; }
                ++o_waits[x];
                tc_fence_after();
              }
              if (!mma_pv(x, vslot % C::kSlots, j == 0, ph)) { ok = false; break; }
              release(vslot);
              if (j + 1 < it.n(x)) {
                mma_s(x, 0, kslot % C::kSlots);
                release(kslot);
                s_group_done();
              }
            }
          }
          ld = l;
          for (int x = 0; x < nx; ++x) ++x_items[x];
          ++item_ctr;
        }
      if (!ok && issued) {
        // Wait for every MMA already issued before TMEM is released.
        mma_commit_w(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax: warpgroup x owns block x
    // (in a split item: the chunks c0(x) .. c0(x) + n(x) - 1 of block A's keys)
    const int x = warp >> 2;
    const int quad = warp & 3;         // TMEM lane quadrant
    const int row = quad * 32 + lane;  // query row of the block = TMEM lane
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const uint32_t s_col = 128 * x, o_col = C::kTmO0 + x * D;
    const float sl2 = p.scale_log2;
    // S chunks of this warpgroup so far, and its pv_done phases (one per chunk)
    uint32_t s_waits = 0, pv_waits = 0;
    // After a failed wait the warpgroup keeps walking the items without
    // touching barriers or TMEM, so that both warpgroups still meet at the
    // named barriers of split items.
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_work; item += gridDim.x) {
      const ItemInfo it = decode_item<kMode>(p, item);
      if (it.n(x) == 0) continue;
      const bool own_b = x == 1 && !it.split;  // warpgroup 1 holds block B
      const int o_in_tile = (own_b ? it.qb : it.qa) * kBM + row;
      const bool row_valid = o_in_tile < g.tau;
      const long long tok = row_valid ? token_row(g, p.tiled, it.bh, own_b ? it.tb : it.ta, o_in_tile) : 0;

      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < it.n(x) && ok; ++j) {
        bool okw = mbar_wait_w(&s_full[x], s_waits & 1, ctl, kErrWaitSoftmax);
        ++s_waits;
        // O_X holds every chunk before j: one thread issues every MMA and
        // commit, S(j) after P V(j-1), and a commit tracks the completion of
        // all earlier MMAs of its thread, so s_full(j) implies pv_done(j-1):
        // that phase is counted, not waited for.  (The lone-block kernel
        // derives the count from s_waits instead, which keeps it clear of
        // spills at head dim 64.)
        if (kMode == 0 && j > 0) ++pv_waits;
        okw = __all_sync(0xffffffffu, okw);
        if (!okw) { ok = false; break; }
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
        const int kvalid = it.nkeys - (it.c0(x) + j) * kBN;
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
        const bool resc = mloc > m + 8.0f;  // also true while m == -inf
        const float m_new = resc ? mloc : m;
        const float alpha = resc ? ex2_approx(m - m_new) : 1.f;
        const bool warp_resc = __any_sync(0xffffffffu, resc) && j > 0;
        m = m_new;

        // P = exp2(S * scale_log2 - m) as bf16 over the consumed S columns, row
        // sum.  The first kLeadKeys keys are published on their own (p_lead) so
        // that their share of P V runs while the rest of P is formed; O is
        // rescaled (rarely) before that, once the first half of S is no longer
        // held.
        float ls[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) ls[a] = 0.f;
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float p0 = ex2_approx(fmaf(s[32 * c + i], sl2, -m));
            const float p1 = ex2_approx(fmaf(s[32 * c + i + 1], sl2, -m));
            ls[(i / 2) & 7] += p0 + p1;
            pk[i / 2] = pack_bf16(p0, p1);
          }
          tmem_st16(tmem + lane_off + s_col + c * 16, pk);
          if (c == 1 && warp_resc) {
            // O holds every chunk before j (P V(j-1) finished before S(j))
#pragma unroll 1
            for (int oc = 0; oc < D / 16; ++oc) {
              uint32_t r[16];
              tmem_ld16(tmem + lane_off + o_col + oc * 16, r);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              tmem_st16(tmem + lane_off + o_col + oc * 16, r);
            }
          }
          if (c == C::kLeadKeys / 32 - 1) {
            tmem_st_wait();
            tc_fence_before();
            warp_arrive(&p_lead[x], lane);
          }
        }
        l = l * alpha + (((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7])));
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(&p_ready[x], lane);
      }

      // epilogue: O_X / l -> bf16 row, LSE
      bool oke = false;
      if (ok) {
        // the last chunk's phase
        oke = mbar_wait_w(&pv_done[x], (kMode == 0 ? pv_waits : s_waits - 1) & 1, ctl, kErrWaitEpilogue);
        ++pv_waits;
        oke = __all_sync(0xffffffffu, oke);
      }
      if (it.split) {
        // Merge the two partial states of the row (m_x, l_x, O_x); warpgroup x
        // writes output columns [x D / 2, (x + 1) D / 2).
        ml_xchg[x * 128 + row] = m;
        ml_xchg[(2 + x) * 128 + row] = l;
        const bool both = named_bar_and(1, 256, oke);
        ok = ok && both;
        if (both) {
          tc_fence_after();
          const float m0 = ml_xchg[row], m1 = ml_xchg[128 + row];
          const float mf = fmaxf(m0, m1);
          const float a0 = ex2_approx(m0 - mf), a1 = ex2_approx(m1 - mf);
          const float lf = ml_xchg[256 + row] * a0 + ml_xchg[384 + row] * a1;
          const float inv_l = 1.f / lf;
          const float f0 = a0 * inv_l, f1 = a1 * inv_l;
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + tok * D + x * (D / 2));
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t r0[32], r1[32];
            tmem_ld32(tmem + lane_off + C::kTmO0 + x * (D / 2) + c * 32, r0);
            tmem_ld32(tmem + lane_off + C::kTmO0 + D + x * (D / 2) + c * 32, r1);
            tmem_ld_wait();
            if (row_valid) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  o[e] = __uint_as_float(r0[8 * v + e]) * f0 + __uint_as_float(r1[8 * v + e]) * f1;
                uint4 w;
                w.x = pack_bf16(o[0], o[1]);
                w.y = pack_bf16(o[2], o[3]);
                w.z = pack_bf16(o[4], o[5]);
                w.w = pack_bf16(o[6], o[7]);
                dst[c * 4 + v] = w;
              }
            }
          }
          if (x == 0 && row_valid && p.lse) p.lse[tok] = (mf + __log2f(lf)) * 0.69314718055994530942f;
          tc_fence_before();
        }
        // both warpgroups are done with O_A, O_B and the exchange area
        named_bar_sync(2, 256);
        if (both) warp_arrive(&o_free[x], lane);
        continue;
      }
      if (!oke) {
        ok = false;
        continue;
      }
      tc_fence_after();
      const float inv_l = 1.f / l;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + tok * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + o_col + c * 32, r);
        tmem_ld_wait();
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(r[8 * v + 0]) * inv_l, __uint_as_float(r[8 * v + 1]) * inv_l);
            w.y = pack_bf16(__uint_as_float(r[8 * v + 2]) * inv_l, __uint_as_float(r[8 * v + 3]) * inv_l);
            w.z = pack_bf16(__uint_as_float(r[8 * v + 4]) * inv_l, __uint_as_float(r[8 * v + 5]) * inv_l);
            w.w = pack_bf16(__uint_as_float(r[8 * v + 6]) * inv_l, __uint_as_float(r[8 * v + 7]) * inv_l);
            dst[c * 4 + v] = w;
          }
        }
      }
      tc_fence_before();
      warp_arrive(&o_free[x], lane);
      if (row_valid && p.lse) p.lse[tok] = (m + __log2f(l)) * 0.69314718055994530942f;
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

template <int D, int kMode>
cudaError_t launch_fwd_mode(const FwdParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            int num_sms, cudaStream_t stream) {
  using C = FwdCfg<D, kMode>;
  static bool attr_set = false;  // per process; the attribute is per function
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(sta_fwd_kernel<D, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = p.n_work < num_sms ? p.n_work : num_sms;
  if (grid <= 0) return cudaSuccess;
  sta_fwd_kernel<D, kMode><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

// The work list holds the items of one or two shared blocks first and the
// lone blocks (n_work_lone of them) last; each part gets its own launch.
template <int D>
cudaError_t launch_fwd_d(const FwdParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                         int num_sms, cudaStream_t stream) {
  FwdParams part = p;
  part.n_work = p.n_work - p.n_work_lone;
  cudaError_t e = launch_fwd_mode<D, 0>(part, tq, tk, tv, num_sms, stream);
  if (e != cudaSuccess) return e;
  part.work = p.work + part.n_work;
  part.n_work = p.n_work_lone;
  return launch_fwd_mode<D, 1>(part, tq, tk, tv, num_sms, stream);
}

}  // namespace

cudaError_t launch_forward(const FwdParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                           const CUtensorMap &tmap_v, int num_sms, cudaStream_t stream) {
  if (p.g.d == 128) return launch_fwd_d<128>(p, tmap_q, tmap_k, tmap_v, num_sms, stream);
  if (p.g.d == 64) return launch_fwd_d<64>(p, tmap_q, tmap_k, tmap_v, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sta
