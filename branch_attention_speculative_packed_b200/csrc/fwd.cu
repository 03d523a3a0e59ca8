// Branch-attention forward on sm_100a: tcgen05 MMA with TMEM accumulators,
// TMA-staged tiles, warp-specialised pipeline.
//
// Paper: arXiv 2609.07108 §3.2 / Eq. 2 (rcap.io post, branch-attention
// paragraph; cere-bro wiki, "Obstacle one, context parallelism").  One
// persistent CTA per SM walks (row tile, query head) work items, longest
// first.  For each item it streams the item's main key tiles (the causal
// prefix [doc start, largest limit]) and, in the fused variant, the key tiles
// of the branch-local keys, through one online softmax.  Visiting key tiles
// one after another with a running (max, sum) is the same log-sum-exp merge
// ring attention applies between ring steps (Eq. 2), so the main-sequence
// component, the branch-local component and their merge all happen here.
//
// Roles (192 threads):
//   warp 0      producer: claims work items (one item ahead of the consumers)
//               and streams the K/V key tiles through a 3-stage TMA ring.
//   warp 1      TMEM allocator and single-thread MMA issuer:
//               S[sb] = Q K^T into one of two TMEM buffers, then O += P V
//               with P read from TMEM (A operand in tensor memory).
//   warps 2-5   softmax / epilogue, one query row per thread.  Each thread
//               copies its own query row into shared memory (cp.async): the
//               next item's rows go in as soon as the current item's last
//               S MMA, the only reader of Q, has finished, so the copy
//               overlaps the last softmax step and the epilogue.  Per key
//               tile: load S from
//               TMEM, mask by the row's key range, update the running max
//               (lazily: O in TMEM is rescaled only when the max grows by
//               more than 2^8), write P (bf16) into one of two TMEM buffers
//               for the P.V MMA, and finally normalise O and write O and LSE.
//
// Shared memory (D = head dim): Q [128 x D] | 3 x (K [128 x D], V [128 x D]),
// bf16 in the 128-byte-swizzled layout (TMA writes K / V; the threads write Q
// in the same pattern).
// TMEM: S buffers at columns 0 and 128, O at 256, P buffers at 384 and 448
// (128 rows x 128 bf16 keys = 64 columns each).
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

constexpr int kThreads = 192;
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Smem {
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kTileBytes = 128u * D * 2u;  // one 128-row bf16 tile
  static constexpr uint32_t kK0 = kQ + kTileBytes;
  static constexpr uint32_t kStageBytes = 2u * kTileBytes;  // K + V
  static constexpr uint32_t kBar = kK0 + kStages * kStageBytes;
  // barriers: q_full, kv_full[3], kv_empty[3], s_full[2], s_empty[2], p_full[2], o_done[2],
  // drain, item_full[4], item_empty[4]
  static constexpr uint32_t kNumBars = 24;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8u;  // tmem base, abort, item slots[4]
  static constexpr uint32_t kTotal = kMisc + 32u;
  static constexpr uint32_t kAlloc = kTotal + 1024u;  // slack to align the base to 1024
};

struct Bars {
  uint32_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], s_empty[2], p_full[2],
      o_done[2], drain;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmKb, const __grid_constant__ CUtensorMap tmVb,
               const FwdArgs a) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  Bars bar;
  {
    uint32_t b = sbase + L::kBar;
    bar.q_full = b; b += 8;
    for (int i = 0; i < kStages; ++i) { bar.kv_full[i] = b; b += 8; }
    for (int i = 0; i < kStages; ++i) { bar.kv_empty[i] = b; b += 8; }
    for (int i = 0; i < 2; ++i) { bar.s_full[i] = b; b += 8; }
    for (int i = 0; i < 2; ++i) { bar.s_empty[i] = b; b += 8; }
    for (int i = 0; i < 2; ++i) { bar.p_full[i] = b; b += 8; }
    for (int i = 0; i < 2; ++i) { bar.o_done[i] = b; b += 8; }
    bar.drain = b;
  }
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  ptx::ItemRing ring;
  ring.slot = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
  ring.full = bar.drain + 8;
  ring.empty = ring.full + 8 * ptx::kItemSlots;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar.q_full, 128);  // one arrival per softmax thread (its copied row)
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(bar.kv_full[i], 1);
      ptx::mbar_init(bar.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar.s_full[i], 1);
      ptx::mbar_init(bar.s_empty[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar.p_full[i], 128);
      ptx::mbar_init(bar.o_done[i], 1);
    }
    ptx::mbar_init(bar.drain, 1);
    for (uint32_t i = 0; i < ptx::kItemSlots; ++i) {
      ptx::mbar_init(ring.full + 8 * i, 1);
      ptx::mbar_init(ring.empty + 8 * i, 129);  // MMA issuer + 128 softmax threads
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
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
      uint32_t kv_stage = 0, kv_phase = 0;
      // Parity of each stage's last fill and whether it may still be in flight (abort drain).
      uint32_t pend_mask = 0, pend_par = 0;
      // The ring runs one item ahead of the K/V stream, so the consumers learn
      // the next item (and copy its query rows) before the current one ends.
      int cur = static_cast<int>(atomicAdd(a.counter, 1u));
      bool ok = ptx::ring_put(ring, 0, cur, abort_flag, a.err, lim, ptx::wait_site(1, 0, 12));
      for (uint32_t rn = 1; ok && cur < a.n_items; ++rn) {
        const int nxt = static_cast<int>(atomicAdd(a.counter, 1u));
        if (!ptx::ring_put(ring, rn, nxt, abort_flag, a.err, lim, ptx::wait_site(1, 0, 12))) { ok = false; break; }
        const TileDesc td = a.tiles[a.order[cur / Hq]];
        const int g = (cur % Hq) / a.G;
        const int nkv = ceil_div(td.kv_end - td.doc_start, 128);
        const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
        for (int j = 0; j < nkv + nbr; ++j) {
          if (!ptx::mbar_wait(bar.kv_empty[kv_stage], kv_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(1, 0, 2))) {
            ok = false;
            break;
          }
          ptx::mbar_expect_tx(bar.kv_full[kv_stage], 2u * L::kTileBytes);
          const void* mk = &tmK;
          const void* mv = &tmV;
          int y;
          if (j < nkv) {
            y = td.doc_start + 128 * j;
          } else {
            y = td.br_lo + 128 * (j - nkv);
            mk = &tmKb;
            mv = &tmVb;
          }
          const uint32_t sk = sbase + L::kK0 + kv_stage * L::kStageBytes;
          const uint32_t sv = sk + L::kTileBytes;
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            ptx::tma_load_2d(sk + cb * 16384u, mk, bar.kv_full[kv_stage], g * D + cb * 64, y);
            ptx::tma_load_2d(sv + cb * 16384u, mv, bar.kv_full[kv_stage], g * D + cb * 64, y);
          }
          pend_mask |= 1u << kv_stage;
          pend_par = (pend_par & ~(1u << kv_stage)) | (kv_phase << kv_stage);
          if (++kv_stage == kStages) { kv_stage = 0; kv_phase ^= 1u; }
        }
        cur = nxt;
      }
      if (*abort_flag) {
        // Let our own copies in flight land before the CTA exits (bounded).
        volatile int never = 0;
        for (int i = 0; i < kStages; ++i)
          if (pend_mask & (1u << i))
            ptx::mbar_wait(bar.kv_full[i], (pend_par >> i) & 1u, &never, a.err, lim / 8);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPV = ptx::idesc_bf16_f32(128, D, false, true);
      uint32_t kv_stage = 0, kv_phase = 0, q_phase = 0, s_cnt = 0, pv_cnt = 0;
      bool ok = true;
      const uint32_t sQ = sbase + L::kQ;
      // O += P V for key tile jj: P from TMEM buffer pv_cnt % 2, V from the stage.
      auto issue_pv = [&](int jj, uint32_t stage) -> bool {
        const uint32_t pb = pv_cnt & 1u;
        if (!ptx::mbar_wait(bar.p_full[pb], (pv_cnt >> 1) & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 1, 3))) return false;
        ptx::tc_fence_after();
        const uint32_t sv = sbase + L::kK0 + stage * L::kStageBytes + L::kTileBytes;
        const uint64_t bd0 = ptx::sdesc_sw128(sv, 16384u, 1024u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = ptx::sdesc_add(bd0, kk * 2048u);
          ptx::umma_ts(tmem + kColO, tmem + kColP + pb * 64u + kk * 8u, bd, kIdPV,
                       (jj > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit(bar.o_done[pb]);
        ptx::umma_commit(bar.kv_empty[stage]);
        ++pv_cnt;
        return true;
      };
      for (uint32_t rn = 0; ok; ++rn) {
        int item = 0;
        if (!ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(1, 1, 13))) { ok = false; break; }
        if (item >= a.n_items) break;
        const TileDesc td = a.tiles[a.order[item / Hq]];
        const int nkv = ceil_div(td.kv_end - td.doc_start, 128);
        const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
        const int n = nkv + nbr;
        if (!ptx::mbar_wait(bar.q_full, q_phase, abort_flag, a.err, lim, ptx::wait_site(1, 1, 4))) { ok = false; break; }
        q_phase ^= 1u;
        ptx::tc_fence_after();
        uint32_t prev_stage = 0;
        for (int j = 0; j < n; ++j) {
          if (!ptx::mbar_wait(bar.kv_full[kv_stage], kv_phase, abort_flag, a.err, lim, ptx::wait_site(1, 1, 5))) { ok = false; break; }
          const uint32_t sb = s_cnt & 1u;
          const uint32_t sph = (s_cnt >> 1) & 1u;
          if (!ptx::mbar_wait(bar.s_empty[sb], sph ^ 1u, abort_flag, a.err, lim, ptx::wait_site(1, 1, 6))) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t sk = sbase + L::kK0 + kv_stage * L::kStageBytes;
          const uint64_t ad0 = ptx::sdesc_sw128(sQ, 16u, 1024u);
          const uint64_t bd0 = ptx::sdesc_sw128(sk, 16u, 1024u);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
            const uint64_t ad = ptx::sdesc_add(ad0, off);
            const uint64_t bd = ptx::sdesc_add(bd0, off);
            ptx::umma_ss(tmem + kColS0 + sb * 128u, ad, bd, kIdS, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar.s_full[sb]);
          ++s_cnt;
          if (j > 0 && !issue_pv(j - 1, prev_stage)) { ok = false; break; }
          prev_stage = kv_stage;
          if (++kv_stage == kStages) { kv_stage = 0; kv_phase ^= 1u; }
        }
        if (!ok) break;
        if (!issue_pv(n - 1, prev_stage)) { ok = false; break; }
      }
      // Drain: every MMA this thread issued completes before TMEM is freed.
      ptx::umma_commit(bar.drain);
      volatile int never = 0;
      ptx::mbar_wait(bar.drain, 0, &never, a.err, lim);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sl2 = a.scale_log2;
    uint32_t s_cnt = 0, pv_cnt = 0;  // S tiles consumed, P tiles produced

    // This thread's row of a work item.
    struct RowItem {
      bool valid;
      int h, n, nkv, doc_start, br_lo, r, limit, blo, bhi;
    };
    auto fetch = [&](uint32_t rn, RowItem& it) -> bool {
      int item = 0;
      if (!__all_sync(0xffffffffu, ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(1, 2, 14))))
        return false;
      it.valid = item < a.n_items;
      if (!it.valid) return true;
      const TileDesc td = a.tiles[a.order[item / Hq]];
      it.h = item % Hq;
      it.doc_start = td.doc_start;
      it.br_lo = td.br_lo;
      it.nkv = ceil_div(td.kv_end - td.doc_start, 128);
      it.n = it.nkv + ((a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0);
      it.r = a.row_table[td.row_base + row];
      it.limit = td.doc_start;  // padding rows see one key: keeps their math finite
      it.blo = it.bhi = 0;      // visible branch key rows [blo, bhi)
      if (it.r >= 0 && it.r < a.S) {
        it.limit = it.r;
      } else if (it.r >= a.S) {
        const int b = (it.r - a.S) / a.B;
        const int t = (it.r - a.S) - b * a.B;
        it.limit = a.anchors[b];
        it.blo = b * a.B;
        it.bhi = it.blo + (a.mode == 1 ? a.B : t + 1);
      }
      return true;
    };
    // Copy this thread's query row (bf16, D values) into row `row` of the
    // swizzled Q tile; padding rows are zero-filled.
    auto copy_q = [&](const RowItem& it) {
      const __nv_bfloat16* src = a.q;
      uint32_t bytes = 0;
      if (it.r >= 0 && it.r < a.S) {
        src = a.q + (int64_t(it.r) * Hq + it.h) * D;
        bytes = 16;
      } else if (it.r >= a.S) {
        src = a.qb + (int64_t(it.r - a.S) * Hq + it.h) * D;
        bytes = 16;
      }
      const uint32_t dst = sbase + L::kQ + static_cast<uint32_t>(row) * 128u;
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::cp_async16(dst + cb * 16384u + ((static_cast<uint32_t>(c) ^ (row & 7)) << 4),
                          src + (bytes ? cb * 64 + c * 8 : 0), bytes);
      ptx::cp_async_commit();
    };
    // The copies have landed: make them visible to the tensor core, then tell the MMA issuer.
    auto publish_q = [&]() {
      ptx::cp_async_wait_all();
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(bar.q_full);
    };

    RowItem cur;
    bool ok = fetch(0, cur);
    if (ok && cur.valid) {
      copy_q(cur);
      publish_q();
    }
    for (uint32_t rn = 1; ok && cur.valid; ++rn) {
      const int h = cur.h, n = cur.n, nkv = cur.nkv, r = cur.r;
      const int limit = cur.limit, blo = cur.blo, bhi = cur.bhi;
      RowItem nxt;
      nxt.valid = false;
      float m_used = -INFINITY;
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        if (j == n - 1 && !fetch(rn, nxt)) {
          ok = false;
          break;
        }
        const uint32_t sb = s_cnt & 1u;
        const uint32_t sph = (s_cnt >> 1) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar.s_full[sb], sph, abort_flag, a.err, lim, ptx::wait_site(1, 2, 7)))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tl + kColS0 + sb * 128u + c * 32u, sr[c]);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar.s_empty[sb]);
        ++s_cnt;
        // The item's last S MMA has finished: the next item's rows may overwrite Q.
        if (j == n - 1 && nxt.valid) copy_q(nxt);
        // visible columns [lo, hi) of this key tile
        int lo, hi;
        if (j < nkv) {
          lo = 0;
          hi = limit - (cur.doc_start + 128 * j) + 1;
        } else {
          const int kr0 = cur.br_lo + 128 * (j - nkv);
          lo = blo - kr0;
          hi = bhi - kr0;
        }
        lo = max(lo, 0);
        hi = min(hi, 128);
        if (!(lo == 0 && hi == 128)) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = c * 32 + i;
              if (col < lo || col >= hi) sr[c][i] = __float_as_uint(-INFINITY);
            }
        }
        // Row max over 8 independent accumulators, two new values per instruction.
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mx8[(i >> 1) & 7] = ptx::max3(mx8[(i >> 1) & 7], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
        const float mx = fmaxf(ptx::max3(mx8[0], mx8[1], mx8[2]),
                               fmaxf(ptx::max3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const float mxs = mx * sl2;
        float alpha = 1.f;
        bool rescale = false;
        if (m_used == -INFINITY) {
          m_used = mxs;
        } else if (mxs > m_used + kRescaleThreshold) {
          alpha = ptx::ex2(m_used - mxs);
          m_used = mxs;
          rescale = true;
        }
        // P = exp2(S * scale*log2(e) - m), row sum over 4 paired accumulators
        const float2 c2 = make_float2(sl2, sl2);
        const float2 nm2 = make_float2(-m_used, -m_used);
        float2 rs4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) rs4[u] = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 x = ptx::fma2(make_float2(__uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1])), c2, nm2);
            const float2 p = ptx::exp2_sfu(x);
            rs4[(i >> 1) & 3] = ptx::add2(rs4[(i >> 1) & 3], p);
            sr[c][i] = __float_as_uint(p.x);
            sr[c][i + 1] = __float_as_uint(p.y);
          }
        const float2 rsa = ptx::add2(ptx::add2(rs4[0], rs4[1]), ptx::add2(rs4[2], rs4[3]));
        l = l * alpha + (rsa.x + rsa.y);
        const uint32_t pb = pv_cnt & 1u;
        // P buffer pb is free once the P.V that last read it (two tiles ago) finished.
        bool w = true;
        if (pv_cnt >= 2)
          w = ptx::mbar_wait(bar.o_done[pb], ((pv_cnt >> 1) - 1u) & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 2, 9));
        // Rescaling O needs the previous P.V (the other buffer) to have finished.
        const bool any_rescale = __any_sync(0xffffffffu, rescale);
        if (any_rescale && j > 0)
          w = w && ptx::mbar_wait(bar.o_done[pb ^ 1u], ((pv_cnt - 1u) >> 1) & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 2, 10));
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        ptx::tc_fence_after();
        if (any_rescale && j > 0) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            ptx::tmem_ld32(tl + kColO + c * 32u, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            ptx::tmem_st32(tl + kColO + c * 32u, ov);
          }
        }
        // P (bf16, two keys per 32-bit column) -> TMEM buffer pb
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t pw[32];
#pragma unroll
          for (int wi = 0; wi < 32; ++wi) {
            const int key = (h2 * 32 + wi) * 2;
            pw[wi] = ptx::pack_bf16x2(__uint_as_float(sr[key >> 5][key & 31]),
                                      __uint_as_float(sr[key >> 5][(key & 31) + 1]));
          }
          ptx::tmem_st32(tl + kColP + pb * 64u + h2 * 32u, pw);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar.p_full[pb]);
        ++pv_cnt;
      }
      if (!ok) break;
      // The next item's S MMAs may start while this item's epilogue runs.
      if (nxt.valid) publish_q();
      // ---------------------------------------------------------- epilogue
      {  // the item's last P.V (and, in order, every earlier one) finished
        const uint32_t last = pv_cnt - 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar.o_done[last & 1u], (last >> 1) & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 2, 11)))) {
          ok = false;
          break;
        }
      }
      ptx::tc_fence_after();
      const float inv_l = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        ptx::tmem_ld32(tl + kColO + c * 32u, ov);
        ptx::tmem_wait_ld();
        if (r >= 0) {
          if (a.out_bf16) {
            __nv_bfloat16* dst = (r < a.S ? a.o + (int64_t(r) * Hq + h) * D
                                          : a.ob + (int64_t(r - a.S) * Hq + h) * D) + c * 32;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 w;
              w.x = ptx::pack_bf16x2(__uint_as_float(ov[q4 * 8 + 0]) * inv_l, __uint_as_float(ov[q4 * 8 + 1]) * inv_l);
              w.y = ptx::pack_bf16x2(__uint_as_float(ov[q4 * 8 + 2]) * inv_l, __uint_as_float(ov[q4 * 8 + 3]) * inv_l);
              w.z = ptx::pack_bf16x2(__uint_as_float(ov[q4 * 8 + 4]) * inv_l, __uint_as_float(ov[q4 * 8 + 5]) * inv_l);
              w.w = ptx::pack_bf16x2(__uint_as_float(ov[q4 * 8 + 6]) * inv_l, __uint_as_float(ov[q4 * 8 + 7]) * inv_l);
              reinterpret_cast<uint4*>(dst)[q4] = w;
            }
          } else {
            float* dst = a.o_part + (int64_t(r) * Hq + h) * D + c * 32;
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              float4 w;
              w.x = __uint_as_float(ov[q4 * 4 + 0]) * inv_l;
              w.y = __uint_as_float(ov[q4 * 4 + 1]) * inv_l;
              w.z = __uint_as_float(ov[q4 * 4 + 2]) * inv_l;
              w.w = __uint_as_float(ov[q4 * 4 + 3]) * inv_l;
              reinterpret_cast<float4*>(dst)[q4] = w;
            }
          }
        }
      }
      if (r >= 0) a.lse[int64_t(h) * a.lse_ld + r] = (m_used + __log2f(l)) * 0.69314718055994531f;
      ptx::tc_fence_before();
      cur = nxt;
    }
    // Copies this thread issued must land before the CTA's shared memory goes away.
    ptx::cp_async_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_fwd_d(const FwdMaps& m, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  using L = Smem<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kAlloc));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  fwd_kernel<D><<<grid, kThreads, L::kAlloc, stream>>>(m.k, m.v, m.kb, m.vb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const FwdMaps& maps, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  if (a.d == 128) return launch_fwd_d<128>(maps, a, num_sms, stream);
  if (a.d == 64) return launch_fwd_d<64>(maps, a, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ba
