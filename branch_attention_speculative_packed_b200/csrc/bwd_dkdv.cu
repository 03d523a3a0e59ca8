// dK/dV pass of the backward on sm_100a (key-stationary, tcgen05 + TMEM).
//
// One persistent CTA per SM takes (main key tile, KV head) items, most work
// first, from a global counter.  The item's K and V tiles (128 keys) stay in
// shared memory; the CTA visits every row tile that can see them (a
// contiguous range of the plan's tiles), for each of the G query heads of the
// KV head.  Per (row tile, head) sub-tile i of 128 query rows:
//   S^T_i  = K Q_i^T     [128 keys x 128 rows]  -> TMEM buffer SB
//   dP^T_i = V dO_i^T                           -> TMEM buffer DB
//   threads (one key per thread, two warpgroups of 64 rows each):
//       P^T = exp2(S^T*scale*log2e - L*log2e) where key <= the row's limit
//       (and, under a window W, key >= limit - W + 1),
//       written as bf16 over the front of each warpgroup's half of SB;
//       dS^T = P^T (dP^T - D), written as bf16 the same way into DB
//   dV += P^T dO_i,  dK += dS^T Q_i             (A operand read from TMEM)
// and finally dK * scale and dV are written as bf16 for the keys this item
// owns (a key tile may run past its document's end; those keys belong to the
// next document's items and are not written here).
//
// The tensor pipe executes in issue order
//     S_i, dK_{i-1}, dP_i, dV_i, S_{i+1}, dK_i, ...
// so S_{i+1} overwrites SB only after dV_i has read P^T_i, and dP_{i+1}
// overwrites DB only after dK_i has read dS^T_i; while the threads turn S_i
// into P^T_i the pipe runs dK_{i-1} and dP_i, and while they form dS^T_i it
// runs dV_i and S_{i+1}.  Every MMA is 128 x 128 x 16 (N = 128 runs the
// tensor core at full rate; N = 64 costs nearly as much per instruction).
//
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 2-9 one key row each (warps w and w + 4 share TMEM lane
// quarter w % 4 and split the 128 query rows of a sub-tile).
// TMEM: dK 0..127, dV 128..255, SB 256..383, DB 384..511.
// Shared memory: K | V | 2 x (Q tile, L, D, limits) | 2 x dO tile.  Q_i is
// released after dK_i and dO_i after dV_i.
#include <cuda.h>
#include <cuda_bf16.h>

#include "bwd_kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

// Gradient warpgroups: each takes 128 / NWG of a sub-tile's query rows for
// its keys (one key per thread).  Four of them (d = 128) halve every thread's
// share of the S^T / dP^T work and put four gradient warps on each scheduler.
template <int D>
struct Roles {
  static constexpr int kNWG = D == 128 ? 4 : 2;
  static constexpr int kCW = 128 / kNWG;              // query rows (columns of S^T) per warpgroup
  static constexpr int kGrad = 128 * kNWG;            // gradient threads
  static constexpr int kThreads = 64 + kGrad;         // + TMA producer warp, MMA warp
};
constexpr int kSlots = 2;  // Q and dO ring depth
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDK = 0, kColDV = 128, kColS = 256, kColDP = 384;

template <int D>
struct Smem {
  static constexpr uint32_t kTile = 128u * D * 2u;  // K, V, Q or dO tile (128 rows)
  static constexpr uint32_t kMeta = 3u * 128u * 4u;  // L, D, limits of 128 rows
  static constexpr uint32_t kQSlot = (kTile + kMeta + 1023u) / 1024u * 1024u;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTile;
  static constexpr uint32_t kQ0 = kV + kTile;
  static constexpr uint32_t kO0 = kQ0 + kSlots * kQSlot;
  static constexpr uint32_t kBar = kO0 + kSlots * kTile;
  // kv_full, kv_empty, q_full[2], q_empty[2], o_full[2], o_empty[2], s_full, p_ready, dp_full,
  // ds_ready, acc_full, acc_free, drain, item_full[4], item_empty[4]
  static constexpr uint32_t kNumBars = 25;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8u;  // tmem base, abort, item slots[4]
  static constexpr uint32_t kTotal = kMisc + 32u;
  static constexpr uint32_t kAlloc = kTotal + 1024u;
  // offsets inside a Q slot
  static constexpr uint32_t kSL = kTile, kSD = kTile + 512u, kSLim = kTile + 1024u;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// kWin: a main-prefix window is in use (masking from below as well).
template <int D, bool kWin>
__global__ void __launch_bounds__(Roles<D>::kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const DkdvArgs a) {
  using L = Smem<D>;
  constexpr int kNWG = Roles<D>::kNWG, kCW = Roles<D>::kCW, kGrad = Roles<D>::kGrad;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t b0 = sbase + L::kBar;
  const uint32_t bar_kv_full = b0, bar_kv_empty = b0 + 8;
  auto bar_q_full = [&](uint32_t s) { return b0 + 16 + 8 * s; };
  auto bar_q_empty = [&](uint32_t s) { return b0 + 32 + 8 * s; };
  auto bar_o_full = [&](uint32_t s) { return b0 + 48 + 8 * s; };
  auto bar_o_empty = [&](uint32_t s) { return b0 + 64 + 8 * s; };
  const uint32_t bar_s_full = b0 + 80, bar_p_ready = b0 + 88, bar_dp_full = b0 + 96, bar_ds_ready = b0 + 104;
  const uint32_t bar_acc_full = b0 + 112, bar_acc_free = b0 + 120, bar_drain = b0 + 128;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  ptx::ItemRing ring;
  ring.slot = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
  ring.full = bar_drain + 8;
  ring.empty = ring.full + 8 * ptx::kItemSlots;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_kv_full, 1);
    ptx::mbar_init(bar_kv_empty, 1);
    for (uint32_t i = 0; i < kSlots; ++i) {
      ptx::mbar_init(bar_q_full(i), 1);
      ptx::mbar_init(bar_q_empty(i), 1);
      ptx::mbar_init(bar_o_full(i), 1);
      ptx::mbar_init(bar_o_empty(i), 1);
    }
    ptx::mbar_init(bar_s_full, 1);
    ptx::mbar_init(bar_p_ready, kGrad);
    ptx::mbar_init(bar_dp_full, 1);
    ptx::mbar_init(bar_ds_ready, kGrad);
    ptx::mbar_init(bar_acc_full, 1);
    ptx::mbar_init(bar_acc_free, kGrad);
    ptx::mbar_init(bar_drain, 1);
    for (uint32_t i = 0; i < ptx::kItemSlots; ++i) {
      ptx::mbar_init(ring.full + 8 * i, 1);
      ptx::mbar_init(ring.empty + 8 * i, 1 + kGrad);  // MMA issuer + the gradient threads
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmDO);
  }
  if (warp == 1) {
    ptx::tmem_alloc(sbase + L::kMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int G = a.G;
  const long long lim = a.wait_limit;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_phase = 0, qs = 0, qph = 0, os = 0, oph = 0;
      // fills that may still be in flight when an abort drains the CTA
      uint32_t qpend = 0, qpar = 0, opend = 0, opar = 0, kv_fills = 0;
      bool ok = true;
      for (uint32_t rn = 0; ok; ++rn) {
        const int item = static_cast<int>(atomicAdd(a.counter, 1u));
        if (!ptx::ring_put(ring, rn, item, abort_flag, a.err, lim, ptx::wait_site(3, 0, 13))) { ok = false; break; }
        if (item >= a.n_items) break;
        const int code = a.order[item];
        const KvItem it = a.items[code / a.Hkv];
        const int g = code % a.Hkv;
        if (!ptx::mbar_wait(bar_kv_empty, kv_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 0, 1))) { ok = false; break; }
        kv_phase ^= 1u;
        ptx::mbar_expect_tx(bar_kv_full, 2u * L::kTile);
        ++kv_fills;
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          ptx::tma_load_2d(sbase + L::kK + cb * 16384u, &tmK, bar_kv_full, g * D + cb * 64, it.key0);
          ptx::tma_load_2d(sbase + L::kV + cb * 16384u, &tmV, bar_kv_full, g * D + cb * 64, it.key0);
        }
        for (int ti = 0; ti < it.t_count && ok; ++ti) {
          const TileDesc td = a.tiles[it.t_first + it.t_count - 1 - ti];
          for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            if (!ptx::mbar_wait(bar_q_empty(qs), qph ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 0, 2))) { ok = false; break; }
            const uint32_t sq = sbase + L::kQ0 + qs * L::kQSlot;
            ptx::mbar_expect_tx(bar_q_full(qs), L::kTile + L::kMeta);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
              ptx::tma_load_2d(sq + cb * 16384u, &tmQ, bar_q_full(qs), h * D + cb * 64, td.row_base);
            bulk_load(sq + L::kSL, a.ls + int64_t(h) * a.n_slots + td.row_base, 512u, bar_q_full(qs));
            bulk_load(sq + L::kSD, a.ds + int64_t(h) * a.n_slots + td.row_base, 512u, bar_q_full(qs));
            bulk_load(sq + L::kSLim, a.lims + td.row_base, 512u, bar_q_full(qs));
            qpend |= 1u << qs;
            qpar = (qpar & ~(1u << qs)) | (qph << qs);
            if (++qs == kSlots) { qs = 0; qph ^= 1u; }
            if (!ptx::mbar_wait(bar_o_empty(os), oph ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 0, 3))) { ok = false; break; }
            const uint32_t so = sbase + L::kO0 + os * L::kTile;
            ptx::mbar_expect_tx(bar_o_full(os), L::kTile);
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
              ptx::tma_load_2d(so + cb * 16384u, &tmDO, bar_o_full(os), h * D + cb * 64, td.row_base);
            opend |= 1u << os;
            opar = (opar & ~(1u << os)) | (oph << os);
            if (++os == kSlots) { os = 0; oph ^= 1u; }
          }
        }
      }
      {
        // our own copies land before the CTA exits (immediate on a normal exit)
        volatile int never = 0;
        const long long dl = ptx::kDrainCycles;
        for (uint32_t i = 0; i < kSlots; ++i) {
          if (qpend & (1u << i)) ptx::mbar_wait(bar_q_full(i), (qpar >> i) & 1u, &never, a.err, dl);
          if (opend & (1u << i)) ptx::mbar_wait(bar_o_full(i), (opar >> i) & 1u, &never, a.err, dl);
        }
        if (kv_fills) ptx::mbar_wait(bar_kv_full, (kv_fills - 1) & 1u, &never, a.err, dl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdG = ptx::idesc_bf16_f32(128, D, false, true);
      uint32_t kv_phase = 0, qs = 0, qph = 0, os = 0, oph = 0, acc_phase = 0, sub = 0;
      bool ok = true;
      const uint64_t kd0 = ptx::sdesc_sw128(sbase + L::kK, 16u, 1024u);
      const uint64_t vd0 = ptx::sdesc_sw128(sbase + L::kV, 16u, 1024u);
      for (uint32_t rn = 0; ok; ++rn) {
        int item = 0;
        if (!ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(3, 1, 14))) { ok = false; break; }
        if (item >= a.n_items) break;
        const KvItem it = a.items[a.order[item] / a.Hkv];
        if (!ptx::mbar_wait(bar_kv_full, kv_phase, abort_flag, a.err, lim, ptx::wait_site(3, 1, 3))) { ok = false; break; }
        kv_phase ^= 1u;
        ptx::tc_fence_after();
        bool first_dv = true, first_dk = true, have_prev = false;
        uint32_t prev_qs = 0;
        // dK += dS^T Q for the previous sub-tile (its dS^T in DB, its Q in slot qslot)
        auto issue_dk = [&](uint32_t qslot) -> bool {
          if (!ptx::mbar_wait(bar_ds_ready, (sub - 1u) & 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 4))) return false;
          ptx::tc_fence_after();
          const uint64_t qd0 = ptx::sdesc_sw128(sbase + L::kQ0 + qslot * L::kQSlot, 16384u, 1024u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::umma_ts(tmem + kColDK, tmem + kColDP + (kk / (kCW / 16)) * kCW + (kk % (kCW / 16)) * 8u,
                         ptx::sdesc_add(qd0, kk * 2048u), kIdG, (!first_dk || kk > 0) ? 1u : 0u);
          first_dk = false;
          ptx::umma_commit(bar_q_empty(qslot));
          return true;
        };
        for (int ti = 0; ti < it.t_count && ok; ++ti) {
          for (int hh = 0; hh < G; ++hh) {
            // S^T_i = K Q_i^T -> SB (SB's last reader, dV_{i-1}, was issued before)
            if (!ptx::mbar_wait(bar_q_full(qs), qph, abort_flag, a.err, lim, ptx::wait_site(3, 1, 5))) { ok = false; break; }
            ptx::tc_fence_after();
            const uint64_t qd0 = ptx::sdesc_sw128(sbase + L::kQ0 + qs * L::kQSlot, 16u, 1024u);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
              ptx::umma_ss(tmem + kColS, ptx::sdesc_add(kd0, off), ptx::sdesc_add(qd0, off), kIdS, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar_s_full);
            if (have_prev && !issue_dk(prev_qs)) { ok = false; break; }
            // dP^T_i = V dO_i^T -> DB (DB's last reader, dK_{i-1}, was issued just above)
            if (!ptx::mbar_wait(bar_o_full(os), oph, abort_flag, a.err, lim, ptx::wait_site(3, 1, 6))) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t so = sbase + L::kO0 + os * L::kTile;
            const uint64_t od0 = ptx::sdesc_sw128(so, 16u, 1024u);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
              ptx::umma_ss(tmem + kColDP, ptx::sdesc_add(vd0, off), ptx::sdesc_add(od0, off), kIdS, kk > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar_dp_full);
            // dV += P^T_i dO_i once the threads have written P^T_i
            if (!ptx::mbar_wait(bar_p_ready, sub & 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 7))) { ok = false; break; }
            if (first_dv) {  // the previous item's epilogue has read dK / dV
              if (!ptx::mbar_wait(bar_acc_free, acc_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 8))) { ok = false; break; }
              acc_phase ^= 1u;
            }
            ptx::tc_fence_after();
            const uint64_t ogd0 = ptx::sdesc_sw128(so, 16384u, 1024u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              ptx::umma_ts(tmem + kColDV, tmem + kColS + (kk / (kCW / 16)) * kCW + (kk % (kCW / 16)) * 8u,
                           ptx::sdesc_add(ogd0, kk * 2048u), kIdG, (!first_dv || kk > 0) ? 1u : 0u);
            first_dv = false;
            ptx::umma_commit(bar_o_empty(os));
            prev_qs = qs;
            have_prev = true;
            ++sub;
            if (++qs == kSlots) { qs = 0; qph ^= 1u; }
            if (++os == kSlots) { os = 0; oph ^= 1u; }
          }
        }
        if (!ok) break;
        if (have_prev && !issue_dk(prev_qs)) { ok = false; break; }
        if (first_dv) {  // no sub-tile in this item: still pair the epilogue handshake
          if (!ptx::mbar_wait(bar_acc_free, acc_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 9))) { ok = false; break; }
          acc_phase ^= 1u;
        }
        ptx::umma_commit(bar_kv_empty);
        ptx::umma_commit(bar_acc_full);
      }
      ptx::umma_commit(bar_drain);
      volatile int never = 0;
      ptx::mbar_wait(bar_drain, 0, &never, a.err, ptx::kDrainCycles);
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T / epilogue
    constexpr int kNC = kCW / 32;          // 32-column chunks per warpgroup
    const int quarter = warp & 3;
    const int wg = (warp - 2) >> 2;        // which kCW query rows of a sub-tile
    const int row = quarter * 32 + lane;   // key row within the tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t wg_col = static_cast<uint32_t>(wg) * kCW;
    const float sl2 = a.scale_log2;
    // window: a row with limit l sees keys >= l - W + 1; with no window W is
    // huge, so that bound never bites
    const int W = a.window > 0 ? a.window : 0x3fffffff;
    uint32_t qs = 0, qph = 0, sub = 0, acc_cnt = 0;
    bool ok = true;
    for (uint32_t rn = 0; ok; ++rn) {
      int item = 0;
      if (!__all_sync(0xffffffffu, ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(3, 2, 15)))) {
        ok = false;
        break;
      }
      if (item >= a.n_items) break;
      const int code = a.order[item];
      const KvItem it = a.items[code / a.Hkv];
      const int g = code % a.Hkv;
      const int kp = it.key0 + row;  // this thread's key position
      const int warp_last_key = it.key0 + quarter * 32 + 31;
      const int warp_first_key = it.key0 + quarter * 32;
      bool any = false;
      for (int ti = 0; ti < it.t_count && ok; ++ti) {
        for (int hh = 0; hh < G; ++hh) {
          // The slot's L, D and limits landed (TMA completion, seen by this thread);
          // usually long before S^T_i, so this wait costs nothing on the critical path.
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_q_full(qs), qph, abort_flag, a.err, lim, ptx::wait_site(3, 2, 12)))) {
            ok = false;
            break;
          }
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_s_full, sub & 1u, abort_flag, a.err, lim, ptx::wait_site(3, 2, 9)))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint32_t sv[kNC][32];
#pragma unroll
          for (int c = 0; c < kNC; ++c) ptx::tmem_ld32(tl + kColS + wg_col + c * 32u, sv[c]);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kNC; ++c) ptx::tmem_regs_ready(sv[c]);
          const uint8_t* sq = smem + L::kQ0 + qs * L::kQSlot;
          const float4* L4 = reinterpret_cast<const float4*>(sq + L::kSL) + wg * (kCW / 4);  // -L * log2(e)
          const float4* D4 = reinterpret_cast<const float4*>(sq + L::kSD) + wg * (kCW / 4);
          const int* Lim = reinterpret_cast<const int*>(sq + L::kSLim) + wg * kCW;
          // exponent arguments S^T * scale*log2(e) - L*log2(e), two rows per instruction
          const float2 c2 = make_float2(sl2, sl2);
#pragma unroll
          for (int q = 0; q < kCW / 4; ++q) {
            const float4 l = L4[q];
            const int c = q >> 3, i = (q & 7) * 4;
            const float2 x0 = ptx::fma2(make_float2(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1])), c2,
                                        make_float2(l.x, l.y));
            const float2 x1 = ptx::fma2(make_float2(__uint_as_float(sv[c][i + 2]), __uint_as_float(sv[c][i + 3])), c2,
                                        make_float2(l.z, l.w));
            sv[c][i] = __float_as_uint(x0.x);
            sv[c][i + 1] = __float_as_uint(x0.y);
            sv[c][i + 2] = __float_as_uint(x1.x);
            sv[c][i + 3] = __float_as_uint(x1.y);
          }
          // The rows are sorted by limit (padding, limit -1, only at a tile's end, and
          // neutralised by its L), so when the warp's last key is visible to this
          // warpgroup's first row, every pair is -- unless a window cuts the front of
          // a row's range: that needs the warp's first key at or after the largest
          // limit's window start as well.
          bool full = warp_last_key <= Lim[0];
          if constexpr (kWin) {
            int mx = Lim[lane];
#pragma unroll
            for (int c = 1; c < kNC; ++c) mx = max(mx, Lim[c * 32 + lane]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            full = full && warp_first_key >= mx - W + 1;
          }
          if (!full) {
#pragma unroll
            for (int col = 0; col < kCW; ++col)
              if (kp > Lim[col] || (kWin && kp < Lim[col] - W + 1)) sv[col >> 5][col & 31] = __float_as_uint(-INFINITY);
          }
          uint32_t pk[kCW / 2];
#pragma unroll
          for (int j = 0; j < kCW / 2; ++j) {
            const int c = j >> 4, i = (j & 15) * 2;
            // every other pair on the FMA pipe, the rest on the special-function unit
            const float2 xx = make_float2(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1]));
            const float2 pp = (j & 1) ? ptx::exp2_poly(xx) : ptx::exp2_sfu(xx);
            sv[c][i] = __float_as_uint(pp.x);
            sv[c][i + 1] = __float_as_uint(pp.y);
            pk[j] = ptx::pack_bf16x2(pp.x, pp.y);  // lower row in the low half
          }
          if constexpr (kCW == 64) ptx::tmem_st32(tl + kColS + wg_col, pk); else ptx::tmem_st16(tl + kColS + wg_col, pk);
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar_p_ready);
          // dS^T = P^T (dP^T - D)
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_dp_full, sub & 1u, abort_flag, a.err, lim, ptx::wait_site(3, 2, 10)))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          uint32_t pv[kNC][32];
#pragma unroll
          for (int c = 0; c < kNC; ++c) ptx::tmem_ld32(tl + kColDP + wg_col + c * 32u, pv[c]);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kNC; ++c) ptx::tmem_regs_ready(pv[c]);
#pragma unroll
          for (int q = 0; q < kCW / 4; ++q) {
            const float4 dd = D4[q];
            const int c = q >> 3, i = (q & 7) * 4;
            const float2 g0 = ptx::mul2(make_float2(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1])),
                                        ptx::sub2(make_float2(__uint_as_float(pv[c][i]), __uint_as_float(pv[c][i + 1])),
                                                  make_float2(dd.x, dd.y)));
            const float2 g1 = ptx::mul2(make_float2(__uint_as_float(sv[c][i + 2]), __uint_as_float(sv[c][i + 3])),
                                        ptx::sub2(make_float2(__uint_as_float(pv[c][i + 2]), __uint_as_float(pv[c][i + 3])),
                                                  make_float2(dd.z, dd.w)));
            pk[q * 2] = ptx::pack_bf16x2(g0.x, g0.y);
            pk[q * 2 + 1] = ptx::pack_bf16x2(g1.x, g1.y);
          }
          if constexpr (kCW == 64) ptx::tmem_st32(tl + kColDP + wg_col, pk); else ptx::tmem_st16(tl + kColDP + wg_col, pk);
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar_ds_ready);
          any = true;
          ++sub;
          if (++qs == kSlots) { qs = 0; qph ^= 1u; }
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_acc_full, acc_cnt & 1u, abort_flag, a.err, lim, ptx::wait_site(3, 2, 11)))) {
        ok = false;
        break;
      }
      ++acc_cnt;
      ptx::tc_fence_after();
      const bool own = kp < it.key_end && any;
      const bool zero = kp < it.key_end && !any;
      // each warpgroup writes D / kNWG (= 32) of the D columns of dK and of dV
      static_assert(D / kNWG == 32, "one 32-column chunk per warpgroup");
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = which == 0 ? a.dk : a.dv;
        const float mul = which == 0 ? a.scale : 1.f;
        const uint32_t col0 = (which == 0 ? kColDK : kColDV) + static_cast<uint32_t>(wg) * (D / kNWG);
#pragma unroll
        for (int c = 0; c < D / kNWG / 32; ++c) {
          uint32_t v[32];
          ptx::tmem_ld32(tl + col0 + c * 32u, v);
          ptx::tmem_wait_ld();
          ptx::tmem_regs_ready(v);
          if (own || zero) {
            __nv_bfloat16* dst = out + (int64_t(kp) * a.Hkv + g) * D + wg * (D / kNWG) + c * 32;
            const float z = zero ? 0.f : mul;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 wv;
              wv.x = ptx::pack_bf16x2(__uint_as_float(v[q4 * 8 + 0]) * z, __uint_as_float(v[q4 * 8 + 1]) * z);
              wv.y = ptx::pack_bf16x2(__uint_as_float(v[q4 * 8 + 2]) * z, __uint_as_float(v[q4 * 8 + 3]) * z);
              wv.z = ptx::pack_bf16x2(__uint_as_float(v[q4 * 8 + 4]) * z, __uint_as_float(v[q4 * 8 + 5]) * z);
              wv.w = ptx::pack_bf16x2(__uint_as_float(v[q4 * 8 + 6]) * z, __uint_as_float(v[q4 * 8 + 7]) * z);
              reinterpret_cast<uint4*>(dst)[q4] = wv;
            }
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar_acc_free);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kWin>
cudaError_t launch_d(const DkdvMaps& m, const DkdvArgs& a, int num_sms, cudaStream_t st) {
  using L = Smem<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, kWin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kAlloc));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  bwd_dkdv_kernel<D, kWin><<<grid, Roles<D>::kThreads, L::kAlloc, st>>>(m.k, m.v, m.qg, m.dog, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkdv(const DkdvMaps& m, const DkdvArgs& a, int num_sms, cudaStream_t st) {
  const bool win = a.window > 0;
  if (a.d == 128) return win ? launch_d<128, true>(m, a, num_sms, st) : launch_d<128, false>(m, a, num_sms, st);
  if (a.d == 64) return win ? launch_d<64, true>(m, a, num_sms, st) : launch_d<64, false>(m, a, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace ba
