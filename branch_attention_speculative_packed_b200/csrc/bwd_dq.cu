// dQ pass of the backward on sm_100a (query-stationary, tcgen05 + TMEM).
//
// One persistent CTA per SM takes (row tile, query head) items, longest first,
// from a global counter.  Per key tile j of the item (main keys, then the
// branch-local keys of the tile's branches):
//   S_j  = Q K_j^T     -> TMEM buffer j % 2
//   dP_j = dO V_j^T    -> TMEM
//   threads: P = exp2(S * scale*log2e - L*log2e) under the row's key range,
//            dS = P * (dP - D), written as bf16 into the first 64 columns of
//            S_j's own TMEM buffer
//   dQ  += dS_j K_j    (A operand read from TMEM) -> TMEM accumulator
// and finally dQ * scale is written as bf16 to the row's place in dq / dqb.
// Because dS_j lives in S_j's buffer, the two S buffers double-buffer dS too;
// the in-order tensor pipe runs dQ_j (reading dS_j) before S_{j+2}, which
// overwrites that buffer.
//
// Q and dO come from the pre-pass's slot-ordered copies (one TMA box per 64
// columns); L and D are the pre-pass's per-slot values.  K and V travel in
// separate rings: V_j is released as soon as dP_j has run, K_j only after
// dQ_j, so K gets the deeper ring.
//
// Roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer X (S_j,
// dQ_j), warps 2-5 one query row per thread, warp 6 MMA issuer Y (dP_j).  Two
// issuers because a thread that waits on a barrier stops feeding the tensor
// pipe until its queued MMAs drain; the S/dQ chain and the dP chain wait on
// different events (K fills and dS from the threads; V fills and the threads
// freeing dP), so each keeps the pipe busy while the other waits.  Shared memory (D = head dim): Q | dO | 3 x K |
// 2 x V.  TMEM: S/dS buffers at columns 0 and 128, dP at 256, dQ at 384.
#include <cuda.h>
#include <cuda_bf16.h>

#include "bwd_kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

constexpr int kThreads = 224;
constexpr int kWarpY = 6;  // the second MMA issuer (dP)
constexpr uint32_t kKStages = 3, kVStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColDP = 256, kColDQ = 384;

template <int D>
struct Smem {
  static constexpr uint32_t kTileBytes = 128u * D * 2u;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kDO = kQ + kTileBytes;
  static constexpr uint32_t kK0 = kDO + kTileBytes;
  static constexpr uint32_t kV0 = kK0 + kKStages * kTileBytes;
  static constexpr uint32_t kBar = kV0 + kVStages * kTileBytes;
  // q_full, q_empty, k_full[3], k_empty[3], v_full[2], v_empty[2], s_full[2], dp_full,
  // dp_empty, ds_full[2], dq_done, drain, item_full[4], item_empty[4], drain_y
  static constexpr uint32_t kNumBars = 29;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8u;  // tmem base, abort, item slots[4]
  static constexpr uint32_t kTotal = kMisc + 32u;
  static constexpr uint32_t kAlloc = kTotal + 1024u;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// kGen: a window or bitmask words are in use (per-row lower bounds and mask
// bits); the plain instantiation keeps the original masking.
template <int D, bool kGen>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
                  const DqArgs a) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t b0 = sbase + L::kBar;
  const uint32_t bar_q_full = b0, bar_q_empty = b0 + 8;
  auto bar_k_full = [&](uint32_t s) { return b0 + 16 + 8 * s; };   // 3
  auto bar_k_empty = [&](uint32_t s) { return b0 + 40 + 8 * s; };  // 3
  auto bar_v_full = [&](uint32_t s) { return b0 + 64 + 8 * s; };   // 2
  auto bar_v_empty = [&](uint32_t s) { return b0 + 80 + 8 * s; };  // 2
  auto bar_s_full = [&](uint32_t s) { return b0 + 96 + 8 * s; };   // 2
  const uint32_t bar_dp_full = b0 + 112, bar_dp_empty = b0 + 120;
  auto bar_ds_full = [&](uint32_t s) { return b0 + 128 + 8 * s; };  // 2
  const uint32_t bar_dq_done = b0 + 144, bar_drain = b0 + 152;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  ptx::ItemRing ring;
  ring.slot = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
  ring.full = bar_drain + 8;
  ring.empty = ring.full + 8 * ptx::kItemSlots;
  const uint32_t bar_drain_y = ring.empty + 8 * ptx::kItemSlots;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_q_full, 1);
    ptx::mbar_init(bar_q_empty, 2);  // Q read by issuer X's S MMAs, dO by issuer Y's dP MMAs
    for (uint32_t i = 0; i < kKStages; ++i) {
      ptx::mbar_init(bar_k_full(i), 1);
      ptx::mbar_init(bar_k_empty(i), 1);
    }
    for (uint32_t i = 0; i < kVStages; ++i) {
      ptx::mbar_init(bar_v_full(i), 1);
      ptx::mbar_init(bar_v_empty(i), 1);
    }
    for (uint32_t i = 0; i < 2; ++i) {
      ptx::mbar_init(bar_s_full(i), 1);
      ptx::mbar_init(bar_ds_full(i), 128);
    }
    ptx::mbar_init(bar_dp_full, 1);
    ptx::mbar_init(bar_dp_empty, 128);
    ptx::mbar_init(bar_dq_done, 1);
    ptx::mbar_init(bar_drain, 1);
    ptx::mbar_init(bar_drain_y, 1);
    for (uint32_t i = 0; i < ptx::kItemSlots; ++i) {
      ptx::mbar_init(ring.full + 8 * i, 1);
      ptx::mbar_init(ring.empty + 8 * i, 130);  // two MMA issuers + 128 gradient threads
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmDO);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    ptx::prefetch_tmap(&tmKb);
    ptx::prefetch_tmap(&tmVb);
  }
  if (warp == 1) {
    ptx::tmem_alloc(sbase + L::kMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int Hq = a.Hq;
  const long long lim = a.wait_limit;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t ks = 0, kph = 0, vs = 0, vph = 0, q_phase = 0;
      // parity of each stage's last fill and whether it may still be in flight (abort drain)
      uint32_t kpend = 0, kpar = 0, vpend = 0, vpar = 0, q_fills = 0;
      bool ok = true;
      // The ring runs one item ahead of the loads, so the next item's tile
      // descriptor is fetched while this item's K/V tiles stream.
      int item = static_cast<int>(atomicAdd(a.counter, 1u));
      ok = ptx::ring_put(ring, 0, item, abort_flag, a.err, lim, ptx::wait_site(2, 0, 12));
      TileDesc td = {};
      if (ok && item < a.n_items) td = a.tiles[a.order[item / Hq]];
      for (uint32_t rn = 1; ok && item < a.n_items; ++rn) {
        const int nxt = static_cast<int>(atomicAdd(a.counter, 1u));
        if (!ptx::ring_put(ring, rn, nxt, abort_flag, a.err, lim, ptx::wait_site(2, 0, 12))) { ok = false; break; }
        TileDesc td_next = {};
        if (nxt < a.n_items) td_next = a.tiles[a.order[nxt / Hq]];
        const int h = item % Hq;
        const int g = h / a.G;
        if (!ptx::mbar_wait(bar_q_empty, q_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 0, 1))) { ok = false; break; }
        q_phase ^= 1u;
        ptx::mbar_expect_tx(bar_q_full, 2u * L::kTileBytes);
        ++q_fills;
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          ptx::tma_load_2d(sbase + L::kQ + cb * 16384u, &tmQ, bar_q_full, h * D + cb * 64, td.row_base);
          ptx::tma_load_2d(sbase + L::kDO + cb * 16384u, &tmDO, bar_q_full, h * D + cb * 64, td.row_base);
        }
        const int nkv = ceil_div(td.kv_end - td.kv_lo, 128);
        const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
        for (int j = 0; j < nkv + nbr; ++j) {
          const void* mk = &tmK;
          const void* mv = &tmV;
          int y;
          if (j < nkv) {
            y = td.kv_lo + 128 * j;
          } else {
            y = td.br_lo + 128 * (j - nkv);
            mk = &tmKb;
            mv = &tmVb;
          }
          if (!ptx::mbar_wait(bar_k_empty(ks), kph ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 0, 2))) { ok = false; break; }
          ptx::mbar_expect_tx(bar_k_full(ks), L::kTileBytes);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            ptx::tma_load_2d(sbase + L::kK0 + ks * L::kTileBytes + cb * 16384u, mk, bar_k_full(ks), g * D + cb * 64, y);
          kpend |= 1u << ks;
          kpar = (kpar & ~(1u << ks)) | (kph << ks);
          if (++ks == kKStages) { ks = 0; kph ^= 1u; }
          if (!ptx::mbar_wait(bar_v_empty(vs), vph ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 0, 3))) { ok = false; break; }
          ptx::mbar_expect_tx(bar_v_full(vs), L::kTileBytes);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            ptx::tma_load_2d(sbase + L::kV0 + vs * L::kTileBytes + cb * 16384u, mv, bar_v_full(vs), g * D + cb * 64, y);
          vpend |= 1u << vs;
          vpar = (vpar & ~(1u << vs)) | (vph << vs);
          if (++vs == kVStages) { vs = 0; vph ^= 1u; }
        }
        item = nxt;
        td = td_next;
      }
      {
        // our own copies land before the CTA exits (immediate on a normal exit)
        volatile int never = 0;
        const long long dl = ptx::kDrainCycles;
        for (uint32_t i = 0; i < kKStages; ++i)
          if (kpend & (1u << i)) ptx::mbar_wait(bar_k_full(i), (kpar >> i) & 1u, &never, a.err, dl);
        for (uint32_t i = 0; i < kVStages; ++i)
          if (vpend & (1u << i)) ptx::mbar_wait(bar_v_full(i), (vpar >> i) & 1u, &never, a.err, dl);
        if (q_fills) ptx::mbar_wait(bar_q_full, (q_fills - 1) & 1u, &never, a.err, dl);
      }
    }
  } else if (warp == 1 || warp == kWarpY) {
    // ------------------------------------------------------------ MMA issuers
    // Two issuing threads: X (warp 1) runs S_j and dQ_j, the users of the two
    // S/dS buffers, the K stages and dQ; Y (warp 6) runs dP_j, the user of the
    // dP buffer and the V stages.  Neither touches the other's TMEM columns; a
    // thread that waits on a barrier stops feeding the tensor pipe while the
    // other keeps it busy.  The item's Q / dO slot is released by both.
    if (lane == 0) {
      const bool X = warp == 1;
      constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdDQ = ptx::idesc_bf16_f32(128, D, false, true);
      uint32_t ks = 0, kph = 0, vs = 0, vph = 0, q_phase = 0, dp_phase = 0;
      uint32_t s_cnt = 0, ds_cnt = 0;  // S tiles issued, dQ MMAs issued
      bool ok = true;
      // Shared-memory descriptors of every tile and stage, built once.
      const uint64_t qd0 = ptx::sdesc_sw128(sbase + L::kQ, 16u, 1024u);
      const uint64_t od0 = ptx::sdesc_sw128(sbase + L::kDO, 16u, 1024u);
      static_assert(kKStages == 3 && kVStages == 2, "descriptor selects");
      const uint64_t kd0 = ptx::sdesc_sw128(sbase + L::kK0, 16u, 1024u);
      const uint64_t kd1 = ptx::sdesc_sw128(sbase + L::kK0 + L::kTileBytes, 16u, 1024u);
      const uint64_t kd2 = ptx::sdesc_sw128(sbase + L::kK0 + 2u * L::kTileBytes, 16u, 1024u);
      const uint64_t kg0 = ptx::sdesc_sw128(sbase + L::kK0, 16384u, 1024u);
      const uint64_t kg1 = ptx::sdesc_sw128(sbase + L::kK0 + L::kTileBytes, 16384u, 1024u);
      const uint64_t kg2 = ptx::sdesc_sw128(sbase + L::kK0 + 2u * L::kTileBytes, 16384u, 1024u);
      const uint64_t vd0 = ptx::sdesc_sw128(sbase + L::kV0, 16u, 1024u);
      const uint64_t vd1 = ptx::sdesc_sw128(sbase + L::kV0 + L::kTileBytes, 16u, 1024u);
      const uint32_t b_drain = X ? bar_drain : bar_drain_y;
      // dQ += dS K for the tile whose S went to buffer ds_cnt % 2 and whose K
      // sits in K stage `kstage`.
      auto issue_dq = [&](int jj, uint32_t kstage) -> bool {
        const uint32_t b = ds_cnt & 1u;
        if (!ptx::mbar_wait(bar_ds_full(b), (ds_cnt >> 1) & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 1, 3))) return false;
        ptx::tc_fence_after();
        const uint64_t bd0 = kstage == 0 ? kg0 : (kstage == 1 ? kg1 : kg2);
        const uint32_t acc0 = jj > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::umma_ts(tmem + kColDQ, tmem + kColS0 + b * 128u + kk * 8u, ptx::sdesc_add(bd0, kk * 2048u), kIdDQ,
                       kk > 0 ? 1u : acc0);
        ptx::umma_commit(bar_k_empty(kstage));
        ++ds_cnt;
        return true;
      };
      for (uint32_t rn = 0; ok; ++rn) {
        int item = 0;
        if (!ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(2, 1, 13))) { ok = false; break; }
        if (item >= a.n_items) break;
        const TileDesc td = a.tiles[a.order[item / Hq]];
        const int nkv = ceil_div(td.kv_end - td.kv_lo, 128);
        const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
        const int n = nkv + nbr;
        if (!ptx::mbar_wait(bar_q_full, q_phase, abort_flag, a.err, lim, ptx::wait_site(2, 1, 4))) { ok = false; break; }
        q_phase ^= 1u;
        ptx::tc_fence_after();
        if (X) {
          uint32_t prev_ks = 0;
          for (int j = 0; j < n; ++j) {
            // S_j = Q K_j^T.  Its buffer last held S/dS of tile j-2, whose dQ MMA
            // was issued before this point, so the in-order pipe keeps them apart.
            if (!ptx::mbar_wait(bar_k_full(ks), kph, abort_flag, a.err, lim, ptx::wait_site(2, 1, 5))) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t sb = s_cnt & 1u;
            const uint64_t bk0 = ks == 0 ? kd0 : (ks == 1 ? kd1 : kd2);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
              ptx::umma_ss(tmem + kColS0 + sb * 128u, ptx::sdesc_add(qd0, off), ptx::sdesc_add(bk0, off), kIdS,
                           kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar_s_full(sb));
            ++s_cnt;
            if (j == n - 1) ptx::umma_commit(bar_q_empty);
            if (j > 0 && !issue_dq(j - 1, prev_ks)) { ok = false; break; }
            prev_ks = ks;
            if (++ks == kKStages) { ks = 0; kph ^= 1u; }
          }
          if (!ok) break;
          if (!issue_dq(n - 1, prev_ks)) { ok = false; break; }
          ptx::umma_commit(bar_dq_done);
        } else {
          for (int j = 0; j < n; ++j) {
            // dP_j = dO V_j^T once the threads hold dP_{j-1} in registers
            if (!ptx::mbar_wait(bar_v_full(vs), vph, abort_flag, a.err, lim, ptx::wait_site(2, 1, 6))) { ok = false; break; }
            if (!ptx::mbar_wait(bar_dp_empty, dp_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 1, 7))) { ok = false; break; }
            dp_phase ^= 1u;
            ptx::tc_fence_after();
            const uint64_t bv0 = vs ? vd1 : vd0;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
              ptx::umma_ss(tmem + kColDP, ptx::sdesc_add(od0, off), ptx::sdesc_add(bv0, off), kIdS, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar_dp_full);
            ptx::umma_commit(bar_v_empty(vs));
            if (++vs == kVStages) { vs = 0; vph ^= 1u; }
            if (j == n - 1) ptx::umma_commit(bar_q_empty);
          }
          if (!ok) break;
        }
      }
      ptx::umma_commit(b_drain);
      volatile int never = 0;
      ptx::mbar_wait(b_drain, 0, &never, a.err, ptx::kDrainCycles);
    }
  } else {
    // ------------------------------------------------------------ dS / epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sl2 = a.scale_log2;
    uint32_t s_cnt = 0, dp_cnt = 0, items = 0;
    bool ok = true;
    for (uint32_t rn = 0; ok; ++rn) {
      int item = 0;
      if (!__all_sync(0xffffffffu, ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(2, 2, 14)))) {
        ok = false;
        break;
      }
      if (item >= a.n_items) break;
      const TileDesc td = a.tiles[a.order[item / Hq]];
      const int h = item % Hq;
      const int nkv = ceil_div(td.kv_end - td.kv_lo, 128);
      const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
      const int n = nkv + nbr;
      const int64_t slot = int64_t(td.row_base) + row;
      const SlotMeta m = a.meta[slot];
      const float neg_l2 = a.ls[int64_t(h) * a.n_slots + slot];
      const float dval = a.ds[int64_t(h) * a.n_slots + slot];
      // the row's first visible main key and, for a bitmask branch row, its mask word
      const int rlo = (kGen && a.window > 0) ? max(td.doc_start, m.limit - a.window + 1) : td.doc_start;
      const uint64_t bits = (kGen && a.mode == 2 && m.row >= a.S) ? a.bmask[m.row - a.S] : 0ull;
      for (int j = 0; j < n; ++j) {
        const uint32_t sb = s_cnt & 1u;
        bool w = ptx::mbar_wait(bar_s_full(sb), (s_cnt >> 1) & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 2, 8));
        w = w && ptx::mbar_wait(bar_dp_full, dp_cnt & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 2, 9));
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        ++dp_cnt;
        ptx::tc_fence_after();
        uint32_t dp[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tl + kColDP + c * 32u, dp[c]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_regs_ready(dp[c]);
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar_dp_empty);
        int lo, hi, sh = 0;
        bool bitm = false;
        if (j < nkv) {
          const int y = td.kv_lo + 128 * j;
          lo = kGen ? rlo - y : 0;
          hi = m.limit - y + 1;
        } else {
          const int kr0 = td.br_lo + 128 * (j - nkv);
          lo = m.blo - kr0;
          hi = m.bhi - kr0;
          sh = lo;  // column c is branch key c - sh of the row's branch
          bitm = kGen && a.mode == 2;
        }
        lo = max(lo, 0);
        hi = min(hi, 128);
        const bool full = lo == 0 && hi == 128 && !bitm;
        const float2 c2 = make_float2(sl2, sl2), nl2 = make_float2(neg_l2, neg_l2), d2 = make_float2(dval, dval);
        // dS in two halves of 64 keys: the S columns of a half are all read
        // before its 32 packed dS columns overwrite the front of the buffer.
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = hf * 2 + cc;
            uint32_t sr[32];
            ptx::tmem_ld32(tl + kColS0 + sb * 128u + c * 32u, sr);
            ptx::tmem_wait_ld();
            ptx::tmem_regs_ready(sr);
            // exponent arguments S * scale*log2(e) - L*log2(e), two keys per instruction
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 x = ptx::fma2(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), c2, nl2);
              sr[i] = __float_as_uint(x.x);
              sr[i + 1] = __float_as_uint(x.y);
            }
            if (!full) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int col = c * 32 + i;
                bool out = col < lo || col >= hi;
                if constexpr (kGen) out = out || (bitm && !((bits >> (col - sh)) & 1ull));
                if (out) sr[i] = __float_as_uint(-INFINITY);
              }
            }
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 p = ptx::exp2_sfu(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])));
              const float2 g = ptx::mul2(p, ptx::sub2(make_float2(__uint_as_float(dp[c][i]), __uint_as_float(dp[c][i + 1])), d2));
              pk[cc * 16 + (i >> 1)] = ptx::pack_bf16x2(g.x, g.y);
            }
          }
          ptx::tmem_st32(tl + kColS0 + sb * 128u + hf * 32u, pk);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar_ds_full(sb));
        ++s_cnt;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_dq_done, items & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 2, 11)))) {
        ok = false;
        break;
      }
      ++items;
      ptx::tc_fence_after();
      const int r = m.row;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t qv[32];
        ptx::tmem_ld32(tl + kColDQ + c * 32u, qv);
        ptx::tmem_wait_ld();
        ptx::tmem_regs_ready(qv);
        if (r >= 0) {
          __nv_bfloat16* dst = (r < a.S ? a.dq + (int64_t(r) * Hq + h) * D
                                        : a.dqb + (int64_t(r - a.S) * Hq + h) * D) + c * 32;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 wv;
            wv.x = ptx::pack_bf16x2(__uint_as_float(qv[q4 * 8 + 0]) * a.scale, __uint_as_float(qv[q4 * 8 + 1]) * a.scale);
            wv.y = ptx::pack_bf16x2(__uint_as_float(qv[q4 * 8 + 2]) * a.scale, __uint_as_float(qv[q4 * 8 + 3]) * a.scale);
            wv.z = ptx::pack_bf16x2(__uint_as_float(qv[q4 * 8 + 4]) * a.scale, __uint_as_float(qv[q4 * 8 + 5]) * a.scale);
            wv.w = ptx::pack_bf16x2(__uint_as_float(qv[q4 * 8 + 6]) * a.scale, __uint_as_float(qv[q4 * 8 + 7]) * a.scale);
            reinterpret_cast<uint4*>(dst)[q4] = wv;
          }
        }
      }
      ptx::tc_fence_before();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kGen>
cudaError_t launch_d(const DqMaps& m, const DqArgs& a, int num_sms, cudaStream_t st) {
  using L = Smem<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D, kGen>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kAlloc));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  bwd_dq_kernel<D, kGen><<<grid, kThreads, L::kAlloc, st>>>(m.qg, m.dog, m.k, m.v, m.kb, m.vb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq(const DqMaps& m, const DqArgs& a, int num_sms, cudaStream_t st) {
  const bool gen = a.window > 0 || a.mode == 2;
  if (a.d == 128) return gen ? launch_d<128, true>(m, a, num_sms, st) : launch_d<128, false>(m, a, num_sms, st);
  if (a.d == 64) return gen ? launch_d<64, true>(m, a, num_sms, st) : launch_d<64, false>(m, a, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace ba
