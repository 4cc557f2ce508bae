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
//   * warp 4: TMA producer.  K and V chunks of 128 keys are gathered tile by
//     tile (a chunk may span several key tiles) into a ring of shared-memory
//     stages with 128-byte swizzle, in the order the MMA consumes them;
//   * warp 5: tcgen05 MMA issuer.  S = Q K^T with Q held in tensor memory
//     (A operand from TMEM, so only K is read from shared memory), two S
//     buffers in TMEM so the next S is computed while softmax runs, then
//     O += P V with P (bf16) from TMEM and V from shared memory;
//   * warps 0-3: softmax.  Thread r owns query row r (= TMEM lane r), so row
//     max / sum need no shuffles.  fp32 online softmax in the log2 domain with
//     lazy rescaling of O (only when the running max grows by more than 2^8).
//   * Tensor memory (512 columns): S0 [0,128) S1 [128,256) O [256,256+d)
//     Q [256+d, 256+1.5d) P [256+1.5d, 256+1.5d+64).
// Every barrier wait is bounded; on a time-out the kernel records an error in
// the status word, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "sta_kernels.h"

namespace sta {
namespace {

constexpr int kBM = 128;  // query rows per block (MMA M)
constexpr int kBN = 128;  // keys per chunk (MMA N of Q K^T, K of P V)
constexpr int kThreads = 192;
constexpr uint64_t kDrainLimitNs = 200ull * 1000 * 1000;  // 0.2 s

template <int D>
struct FwdCfg {
  static constexpr int kSlots = D == 128 ? 6 : 10;
  static constexpr uint32_t kPanelBytes = kBN * 128;            // 128 rows x 64 bf16
  static constexpr uint32_t kSlotBytes = kBN * D * 2;          // one K or V chunk
  static constexpr int kPanels = D / 64;
  static constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO = 256;
  static constexpr uint32_t kTmQ = 256 + D, kTmP = 256 + D + D / 2;
  static constexpr uint32_t kTmCols = 512;
  static constexpr int kNumBars = 2 * kSlots + 8;
  static constexpr uint32_t kSmemBytes = kSlots * kSlotBytes + kNumBars * 8 + 64 + 1024;
  static_assert(kTmP + 64 <= kTmCols, "TMEM budget");
};

__device__ __forceinline__ bool drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kDrainLimitNs) return false;
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
  uint64_t *s_full = bars + 2 * C::kSlots;  // [2]
  uint64_t *p_ready = s_full + 2;
  uint64_t *pv_done = p_ready + 1;
  uint64_t *q_ready = pv_done + 1;
  uint64_t *o_free = q_ready + 1;
  uint64_t *drain = o_free + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geometry &g = p.g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_ready, 128);
    mbar_init(pv_done, 1);
    mbar_init(q_ready, 128);
    mbar_init(o_free, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      uint32_t ld = 0;
      bool ok = true;
      const int pieces = kBN / p.piece_rows;
      for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
        const int2 wi = p.work[item];
        const int bh = wi.x, tile = wi.y / p.nqb, head = bh % g.Hh;
        const int cnt = p.kv_count[head];
        const int nkeys = cnt * g.tau;
        const int nc = (nkeys + kBN - 1) / kBN;
        const int32_t *list = p.kv_list + ((long long)head * g.n_tiles + tile) * p.kv_stride;
        // Loads in consumption order: K0, then (K_{j+1}, V_j) for every j.
        for (int s = 0; s < 2 * nc && ok; ++s) {
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
            for (int pn = 0; pn < C::kPanels; ++pn) {
              uint8_t *pdst = dst + pn * C::kPanelBytes + pc * p.piece_rows * 128;
              if (p.kv_mode == kKvTiled2D) {
                const int y = valid ? bh * g.N + ktile * g.tau + off : p.oob_coord;
                tma_load_2d(pdst, map, pn * 64, y, &full[slot]);
              } else {
                const int kt = ktile / (g.GH * g.GW), kh = (ktile / g.GW) % g.GH, kw = ktile % g.GW;
                const int a = off / (g.th * g.tw), b = (off / g.tw) % g.th, c = off % g.tw;
                tma_load_5d(pdst, map, pn * 64, kw * g.tw + c, kh * g.th + b, kt * g.tt + a,
                            valid ? bh : p.oob_coord, &full[slot]);
              }
            }
          }
          ++ld;
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        const uint32_t first = ld > (uint32_t)C::kSlots ? ld - C::kSlots : 0;
        for (uint32_t i = first; i < ld; ++i) drain_wait(&full[i % C::kSlots], (i / C::kSlots) & 1);
        // the load whose empty-wait failed was never issued
      }
    }
  } else if (warp == 5) {
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
      auto issue_pv = [&](bool first) -> bool {
        const uint32_t slot = ld % C::kSlots, phase = (ld / C::kSlots) & 1;
        if (!mbar_wait(&full[slot], phase, ctl, kErrWaitMma)) return false;
        tc_fence_after();
        const uint32_t vbase = slots_addr + slot * C::kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t a_tm = tmem + C::kTmP + kk * 8;
          const uint64_t bdesc = smem_desc_sw128(vbase + kk * 16 * 128, C::kPanelBytes, 1024);
          mma_ts(tmem + C::kTmO, a_tm, bdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(&empty[slot]);
        mma_commit(pv_done);
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
          if (!issue_pv(j == 0)) { ok = false; break; }
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
    // ------------------------------------------------------------ softmax warps 0-3
    const int row = threadIdx.x;  // TMEM lane
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t chunk_g = 0, item_ctr = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_work && ok; item += gridDim.x) {
      const int2 wi = p.work[item];
      const int bh = wi.x, tile = wi.y / p.nqb, qb = wi.y % p.nqb, head = bh % g.Hh;
      const int nkeys = p.kv_count[head] * g.tau;
      const int nc = (nkeys + kBN - 1) / kBN;
      const int o_in_tile = qb * kBM + row;
      const bool row_valid = o_in_tile < g.tau;
      const long long tok = row_valid ? token_row(g, p.tiled, bh, tile, o_in_tile) : 0;

      // Q row -> TMEM (A operand of S = Q K^T), bf16 pairs packed per column.
      {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.q) + tok * D);
#pragma unroll
        for (int part = 0; part < D / 64; ++part) {
          uint32_t w[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            uint4 x = row_valid ? __ldg(src + part * 8 + v) : make_uint4(0, 0, 0, 0);
            w[4 * v + 0] = x.x;
            w[4 * v + 1] = x.y;
            w[4 * v + 2] = x.z;
            w[4 * v + 3] = x.w;
          }
          tmem_st32(tmem + lane_off + C::kTmQ + part * 32, w);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(q_ready);
      }

      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nc; ++j) {
        const uint32_t gc = chunk_g + j, buf = gc & 1;
        ok = mbar_wait(&s_full[buf], (gc >> 1) & 1, ctl, kErrWaitSoftmax);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float s[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + (buf ? C::kTmS1 : C::kTmS0) + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
        }
        const int kvalid = nkeys - j * kBN;
        if (kvalid < kBN) {
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (i >= kvalid) s[i] = -INFINITY;
        }
        float mx = s[0];
#pragma unroll
        for (int i = 1; i < kBN; ++i) mx = fmaxf(mx, s[i]);
        const float m_cand = fmaxf(m, mx * sl2);
        const bool resc = m_cand > m + 8.0f;  // also true while m == -inf
        float alpha = 1.f;
        if (resc) {
          alpha = ex2_approx(m - m_cand);
          m = m_cand;
        }
        const bool warp_resc = __any_sync(0xffffffffu, resc) && j > 0;
        l *= alpha;
        uint32_t pk[kBN / 2];
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int i = 0; i < kBN; i += 2) {
          const float p0 = ex2_approx(fmaf(s[i], sl2, -m));
          const float p1 = ex2_approx(fmaf(s[i + 1], sl2, -m));
          ls0 += p0;
          ls1 += p1;
          pk[i / 2] = pack_bf16(p0, p1);
        }
        l += ls0 + ls1;
        if (j > 0) {
          // P and O are free once the previous P V has completed.
          ok = mbar_wait(pv_done, (gc - 1) & 1, ctl, kErrWaitSoftmax);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < kBN / 64; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = pk[c * 32 + i];
          tmem_st32(tmem + lane_off + C::kTmP + c * 32, w);
        }
        if (warp_resc) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + C::kTmO + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(tmem + lane_off + C::kTmO + c * 32, r);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      if (!ok) break;
      chunk_g += nc;

      // Epilogue: O / l -> bf16 row, LSE.
      ok = mbar_wait(pv_done, (chunk_g - 1) & 1, ctl, kErrWaitEpilogue);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) + tok * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + C::kTmO + c * 32, r);
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
      mbar_arrive(o_free);
      if (row_valid && p.lse) p.lse[tok] = (m + __log2f(l)) * 0.69314718055994530942f;
      ++item_ctr;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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
