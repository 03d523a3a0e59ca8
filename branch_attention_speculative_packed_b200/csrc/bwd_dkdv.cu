// dK/dV pass of the backward on sm_100a (key-stationary, tcgen05 + TMEM).
//
// One persistent CTA per SM walks (main key tile, KV head) items, most work
// first.  The item's K and V tiles (128 keys) stay in shared memory; the CTA
// visits every row tile that can see them (a contiguous range of the plan's
// tiles), for each of the G query heads of the KV head, in halves of 64 rows:
//   S^T  = K Q^T      [128 keys x 64 rows]  -> TMEM (two buffers)
//   dP^T = V dO^T     [128 x 64]            -> TMEM (two buffers)
//   threads (one key per thread): P^T = exp2(S^T*scale*log2e - L*log2e) where
//       key <= the row's limit, dS^T = P^T (dP^T - D), written as bf16 into
//       the first 32 columns of S^T's and dP^T's own TMEM buffers
//   dV += P^T dO,  dK += dS^T Q             (A operand read from TMEM)
// and finally dK * scale and dV are written as bf16 for the keys this item
// owns (a key tile may run past its document's end; those keys belong to the
// next document's items and are not written here).
//
// The tensor pipe runs the gradient MMAs of sub-tile i (reading P^T_i and
// dS^T_i) before the S^T / dP^T MMAs of sub-tile i + 2, which overwrite those
// buffers, so the two S^T / dP^T buffers double-buffer P^T / dS^T as well.
//
// Roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-5
// one key row each.  TMEM: dK 0..127, dV 128..255, S^T 256 / 320, dP^T 384 / 448.
// Shared memory: K | V | 4 stages of (Q half, dO half, L, D, slot metadata).
#include <cuda.h>
#include <cuda_bf16.h>

#include "bwd_kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kHalf = 64;  // query rows per sub-tile
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDK = 0, kColDV = 128, kColS = 256, kColDP = 384;

template <int D>
struct Smem {
  static constexpr uint32_t kKVBytes = 128u * D * 2u;       // K or V tile
  static constexpr uint32_t kHalfBytes = kHalf * D * 2u;    // Q or dO half tile
  static constexpr uint32_t kMetaBytes = kHalf * (4u + 4u + 16u);  // L, D, SlotMeta
  static constexpr uint32_t kStageBytes = ((2u * kHalfBytes + kMetaBytes) + 1023u) / 1024u * 1024u;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kKVBytes;
  static constexpr uint32_t kStage0 = kV + kKVBytes;
  static constexpr uint32_t kBar = kStage0 + kStages * kStageBytes;
  // kv_full, kv_empty, st_full[4], st_empty[4], sd_full[2], pd_full[2], acc_full, acc_free,
  // drain, item_full[4], item_empty[4]
  static constexpr uint32_t kNumBars = 25;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8u;  // tmem base, abort, item slots[4]
  static constexpr uint32_t kTotal = kMisc + 32u;
  static constexpr uint32_t kAlloc = kTotal + 1024u;
  // offsets inside a stage
  static constexpr uint32_t kSQ = 0, kSDO = kHalfBytes, kSL = 2u * kHalfBytes;
  static constexpr uint32_t kSD = kSL + kHalf * 4u, kSM = kSD + kHalf * 4u;
  static constexpr uint32_t kStageTx = 2u * kHalfBytes + kMetaBytes;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                    const DkdvArgs a) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t b0 = sbase + L::kBar;
  const uint32_t bar_kv_full = b0, bar_kv_empty = b0 + 8;
  auto bar_st_full = [&](uint32_t s) { return b0 + 16 + 8 * s; };   // 4
  auto bar_st_empty = [&](uint32_t s) { return b0 + 48 + 8 * s; };  // 4
  auto bar_sd_full = [&](uint32_t s) { return b0 + 80 + 8 * s; };   // 2
  auto bar_pd_full = [&](uint32_t s) { return b0 + 96 + 8 * s; };   // 2
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
    for (uint32_t i = 0; i < kStages; ++i) {
      ptx::mbar_init(bar_st_full(i), 1);
      ptx::mbar_init(bar_st_empty(i), 1);
    }
    for (uint32_t i = 0; i < 2; ++i) {
      ptx::mbar_init(bar_sd_full(i), 1);
      ptx::mbar_init(bar_pd_full(i), 128);
    }
    ptx::mbar_init(bar_acc_full, 1);
    ptx::mbar_init(bar_acc_free, 128);
    ptx::mbar_init(bar_drain, 1);
    for (uint32_t i = 0; i < ptx::kItemSlots; ++i) {
      ptx::mbar_init(ring.full + 8 * i, 1);
      ptx::mbar_init(ring.empty + 8 * i, 129);  // MMA issuer + 128 gradient threads
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
      uint32_t kv_phase = 0, st = 0, st_phase = 0;
      uint32_t pend_mask = 0, pend_par = 0, kv_fills = 0;
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
        ptx::mbar_expect_tx(bar_kv_full, 2u * L::kKVBytes);
        ++kv_fills;
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          ptx::tma_load_2d(sbase + L::kK + cb * 16384u, &tmK, bar_kv_full, g * D + cb * 64, it.key0);
          ptx::tma_load_2d(sbase + L::kV + cb * 16384u, &tmV, bar_kv_full, g * D + cb * 64, it.key0);
        }
        for (int ti = 0; ti < it.t_count && ok; ++ti) {
          const TileDesc td = a.tiles[it.t_first + it.t_count - 1 - ti];
          const int nh = (td.n_rows + kHalf - 1) / kHalf;
          for (int hh = 0; hh < G && ok; ++hh) {
            const int h = g * G + hh;
            for (int half = 0; half < nh; ++half) {
              if (!ptx::mbar_wait(bar_st_empty(st), st_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 0, 2))) { ok = false; break; }
              const uint32_t sb = sbase + L::kStage0 + st * L::kStageBytes;
              const int slot0 = td.row_base + half * kHalf;
              ptx::mbar_expect_tx(bar_st_full(st), L::kStageTx);
#pragma unroll
              for (int cb = 0; cb < D / 64; ++cb) {
                ptx::tma_load_2d(sb + L::kSQ + cb * 8192u, &tmQ, bar_st_full(st), h * D + cb * 64, slot0);
                ptx::tma_load_2d(sb + L::kSDO + cb * 8192u, &tmDO, bar_st_full(st), h * D + cb * 64, slot0);
              }
              bulk_load(sb + L::kSL, a.ls + int64_t(h) * a.n_slots + slot0, kHalf * 4u, bar_st_full(st));
              bulk_load(sb + L::kSD, a.ds + int64_t(h) * a.n_slots + slot0, kHalf * 4u, bar_st_full(st));
              bulk_load(sb + L::kSM, a.meta + slot0, kHalf * 16u, bar_st_full(st));
              pend_mask |= 1u << st;
              pend_par = (pend_par & ~(1u << st)) | (st_phase << st);
              if (++st == kStages) { st = 0; st_phase ^= 1u; }
            }
          }
        }
      }
      if (*abort_flag) {
        volatile int never = 0;
        for (int i = 0; i < kStages; ++i)
          if (pend_mask & (1u << i))
            ptx::mbar_wait(bar_st_full(i), (pend_par >> i) & 1u, &never, a.err, lim / 8);
        if (kv_fills) ptx::mbar_wait(bar_kv_full, (kv_fills - 1) & 1u, &never, a.err, lim / 8);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, kHalf, false, false);
      constexpr uint32_t kIdG = ptx::idesc_bf16_f32(128, D, false, true);
      uint32_t kv_phase = 0, st = 0, st_phase = 0, pd_phase = 0, acc_phase = 0, sd_cnt = 0;
      bool ok = true;
      const uint32_t sK = sbase + L::kK, sV = sbase + L::kV;
      for (uint32_t rn = 0; ok; ++rn) {
        int item = 0;
        if (!ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(3, 1, 14))) { ok = false; break; }
        if (item >= a.n_items) break;
        const KvItem it = a.items[a.order[item] / a.Hkv];
        if (!ptx::mbar_wait(bar_kv_full, kv_phase, abort_flag, a.err, lim, ptx::wait_site(3, 1, 3))) { ok = false; break; }
        kv_phase ^= 1u;
        ptx::tc_fence_after();
        bool first_grad = true;
        uint32_t prev_st = 0, prev_b = 0;
        bool have_prev = false;
        auto issue_grad = [&](uint32_t stg, uint32_t pb) -> bool {
          // pd_phase bit pb: parity of buffer pb's next P^T / dS^T hand-over
          if (!ptx::mbar_wait(bar_pd_full(pb), (pd_phase >> pb) & 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 4))) return false;
          pd_phase ^= 1u << pb;
          if (first_grad) {  // the previous item's epilogue has read dK / dV
            if (!ptx::mbar_wait(bar_acc_free, acc_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 5))) return false;
            acc_phase ^= 1u;
          }
          ptx::tc_fence_after();
          const uint32_t sb = sbase + L::kStage0 + stg * L::kStageBytes;
          const uint64_t od0 = ptx::sdesc_sw128(sb + L::kSDO, 8192u, 1024u);
          const uint64_t qd0 = ptx::sdesc_sw128(sb + L::kSQ, 8192u, 1024u);
          const uint32_t pt = tmem + kColS + pb * kHalf, dst = tmem + kColDP + pb * kHalf;
#pragma unroll
          for (int kk = 0; kk < kHalf / 16; ++kk) {
            const uint32_t acc = (!first_grad || kk > 0) ? 1u : 0u;
            ptx::umma_ts(tmem + kColDV, pt + kk * 8u, ptx::sdesc_add(od0, kk * 2048u), kIdG, acc);
            ptx::umma_ts(tmem + kColDK, dst + kk * 8u, ptx::sdesc_add(qd0, kk * 2048u), kIdG, acc);
          }
          first_grad = false;
          ptx::umma_commit(bar_st_empty(stg));
          return true;
        };
        for (int ti = 0; ti < it.t_count && ok; ++ti) {
          const TileDesc td = a.tiles[it.t_first + it.t_count - 1 - ti];
          const int nh = (td.n_rows + kHalf - 1) / kHalf;
          for (int hh = 0; hh < G && ok; ++hh) {
            for (int half = 0; half < nh; ++half) {
              if (!ptx::mbar_wait(bar_st_full(st), st_phase, abort_flag, a.err, lim, ptx::wait_site(3, 1, 6))) { ok = false; break; }
              // buffer b last held sub-tile sd_cnt - 2, whose gradient MMAs were issued above
              const uint32_t b = sd_cnt & 1u;
              ptx::tc_fence_after();
              const uint32_t sb = sbase + L::kStage0 + st * L::kStageBytes;
              const uint64_t kd0 = ptx::sdesc_sw128(sK, 16u, 1024u);
              const uint64_t vd0 = ptx::sdesc_sw128(sV, 16u, 1024u);
              const uint64_t qd0 = ptx::sdesc_sw128(sb + L::kSQ, 16u, 1024u);
              const uint64_t od0 = ptx::sdesc_sw128(sb + L::kSDO, 16u, 1024u);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t offA = (kk >> 2) * 16384u + (kk & 3) * 32u;
                const uint32_t offB = (kk >> 2) * 8192u + (kk & 3) * 32u;
                ptx::umma_ss(tmem + kColS + b * kHalf, ptx::sdesc_add(kd0, offA), ptx::sdesc_add(qd0, offB),
                             kIdS, kk > 0 ? 1u : 0u);
              }
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t offA = (kk >> 2) * 16384u + (kk & 3) * 32u;
                const uint32_t offB = (kk >> 2) * 8192u + (kk & 3) * 32u;
                ptx::umma_ss(tmem + kColDP + b * kHalf, ptx::sdesc_add(vd0, offA), ptx::sdesc_add(od0, offB),
                             kIdS, kk > 0 ? 1u : 0u);
              }
              ptx::umma_commit(bar_sd_full(b));
              ++sd_cnt;
              if (have_prev && !issue_grad(prev_st, prev_b)) { ok = false; break; }
              prev_st = st;
              prev_b = b;
              have_prev = true;
              if (++st == kStages) { st = 0; st_phase ^= 1u; }
            }
          }
        }
        if (!ok) break;
        if (have_prev && !issue_grad(prev_st, prev_b)) { ok = false; break; }
        if (first_grad) {  // no gradient MMA in this item: still pair the epilogue handshake
          if (!ptx::mbar_wait(bar_acc_free, acc_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(3, 1, 8))) { ok = false; break; }
          acc_phase ^= 1u;
        }
        ptx::umma_commit(bar_kv_empty);
        ptx::umma_commit(bar_acc_full);
      }
      ptx::umma_commit(bar_drain);
      volatile int never = 0;
      ptx::mbar_wait(bar_drain, 0, &never, a.err, lim);
    }
  } else {
    // ------------------------------------------------------------ P^T, dS^T / epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row within the tile
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sl2 = a.scale_log2;
    uint32_t st = 0, st_phase = 0, sd_cnt = 0, acc_cnt = 0;
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
      bool any = false;
      for (int ti = 0; ti < it.t_count && ok; ++ti) {
        const TileDesc td = a.tiles[it.t_first + it.t_count - 1 - ti];
        const int nh = (td.n_rows + kHalf - 1) / kHalf;
        for (int hh = 0; hh < G && ok; ++hh) {
          for (int half = 0; half < nh; ++half) {
            const uint32_t b = sd_cnt & 1u;
            const uint32_t bph = (sd_cnt >> 1) & 1u;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_sd_full(b), bph, abort_flag, a.err, lim, ptx::wait_site(3, 2, 9)))) {
              ok = false;
              break;
            }
            ++sd_cnt;
            ptx::tc_fence_after();
            uint32_t sv[2][32], pv[2][32];
            ptx::tmem_ld32(tl + kColS + b * kHalf, sv[0]);
            ptx::tmem_ld32(tl + kColS + b * kHalf + 32u, sv[1]);
            ptx::tmem_ld32(tl + kColDP + b * kHalf, pv[0]);
            ptx::tmem_ld32(tl + kColDP + b * kHalf + 32u, pv[1]);
            ptx::tmem_wait_ld();
            // the stage's L, D and metadata landed (TMA completion, seen by this thread)
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_st_full(st), st_phase, abort_flag, a.err, lim, ptx::wait_site(3, 2, 12)))) {
              ok = false;
              break;
            }
            const uint8_t* sb = smem + L::kStage0 + st * L::kStageBytes;
            const float4* L4 = reinterpret_cast<const float4*>(sb + L::kSL);  // -L * log2(e)
            const float4* D4 = reinterpret_cast<const float4*>(sb + L::kSD);
            const SlotMeta* Ms = reinterpret_cast<const SlotMeta*>(sb + L::kSM);
            // exponent arguments S^T * scale*log2(e) - L*log2(e), two rows per instruction
            const float2 c2 = make_float2(sl2, sl2);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
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
            // The half's rows are sorted by limit (padding, limit -1, only at a tile's end), so
            // when the warp's last key is visible to the first row, every pair is visible.
            if (!(warp_last_key <= Ms[0].limit)) {
#pragma unroll
              for (int col = 0; col < 64; ++col)
                if (kp > Ms[col].limit) sv[col >> 5][col & 31] = __float_as_uint(-INFINITY);
            }
            // P^T and dS^T = P^T (dP^T - D) of this key row over the 64 query rows
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float4 dd = D4[q];
              const int c = q >> 3, i = (q & 7) * 4;
              const float2 p0 = make_float2(ptx::ex2(__uint_as_float(sv[c][i])), ptx::ex2(__uint_as_float(sv[c][i + 1])));
              const float2 p1 = make_float2(ptx::ex2(__uint_as_float(sv[c][i + 2])), ptx::ex2(__uint_as_float(sv[c][i + 3])));
              const float2 g0 = ptx::mul2(p0, ptx::sub2(make_float2(__uint_as_float(pv[c][i]), __uint_as_float(pv[c][i + 1])),
                                                       make_float2(dd.x, dd.y)));
              const float2 g1 = ptx::mul2(p1, ptx::sub2(make_float2(__uint_as_float(pv[c][i + 2]), __uint_as_float(pv[c][i + 3])),
                                                       make_float2(dd.z, dd.w)));
              sv[c][i] = __float_as_uint(p0.x);
              sv[c][i + 1] = __float_as_uint(p0.y);
              sv[c][i + 2] = __float_as_uint(p1.x);
              sv[c][i + 3] = __float_as_uint(p1.y);
              pv[c][i] = __float_as_uint(g0.x);
              pv[c][i + 1] = __float_as_uint(g0.y);
              pv[c][i + 2] = __float_as_uint(g1.x);
              pv[c][i + 3] = __float_as_uint(g1.y);
            }
            // bf16 pairs (lower row in the low half) over S^T's / dP^T's first 32 columns
            uint32_t pk[32], dk[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = j >> 4, i = (j & 15) * 2;
              pk[j] = ptx::pack_bf16x2(__uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1]));
              dk[j] = ptx::pack_bf16x2(__uint_as_float(pv[c][i]), __uint_as_float(pv[c][i + 1]));
            }
            ptx::tmem_st32(tl + kColS + b * kHalf, pk);
            ptx::tmem_st32(tl + kColDP + b * kHalf, dk);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_pd_full(b));
            any = true;
            if (++st == kStages) { st = 0; st_phase ^= 1u; }
          }
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
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = which == 0 ? a.dk : a.dv;
        const float mul = which == 0 ? a.scale : 1.f;
        const uint32_t col0 = which == 0 ? kColDK : kColDV;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          ptx::tmem_ld32(tl + col0 + c * 32u, v);
          ptx::tmem_wait_ld();
          if (own || zero) {
            __nv_bfloat16* dst = out + (int64_t(kp) * a.Hkv + g) * D + c * 32;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 wv;
              const float z = zero ? 0.f : mul;
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

template <int D>
cudaError_t launch_d(const DkdvMaps& m, const DkdvArgs& a, int num_sms, cudaStream_t st) {
  using L = Smem<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kAlloc));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  bwd_dkdv_kernel<D><<<grid, kThreads, L::kAlloc, st>>>(m.k, m.v, m.qg, m.dog, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkdv(const DkdvMaps& m, const DkdvArgs& a, int num_sms, cudaStream_t st) {
  if (a.d == 128) return launch_d<128>(m, a, num_sms, st);
  if (a.d == 64) return launch_d<64>(m, a, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace ba
