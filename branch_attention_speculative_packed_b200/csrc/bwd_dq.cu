// dQ pass of the backward on sm_100a (query-stationary, tcgen05 + TMEM).
//
// One persistent CTA per SM walks (row tile, query head) items, longest first,
// like the forward.  Per key tile j of the item (main keys, then the
// branch-local keys of the tile's branches):
//   S  = Q K_j^T      -> TMEM (two buffers)
//   dP = dO V_j^T     -> TMEM
//   threads: P = exp2(S * scale*log2e - L*log2e) under the row's key range,
//            dS = P * (dP - D)  -> shared memory (bf16)
//   dQ += dS K_j      -> TMEM accumulator
// and finally dQ * scale is written as bf16 to the row's place in dq / dqb.
// Q and dO come from the pre-pass's slot-ordered copies, so each is one TMA
// box per 64 columns; L and D are the pre-pass's per-slot values.
//
// Roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2-5
// one query row per thread.  Shared memory (D = head dim): Q | dO |
// 2 x (K, V) | dS.  TMEM: S at columns 0 / 128, dP at 256, dQ at 384.
#include <cuda.h>
#include <cuda_bf16.h>

#include "bwd_kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColDP = 256, kColDQ = 384;

template <int D>
struct Smem {
  static constexpr uint32_t kTileBytes = 128u * D * 2u;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kDO = kQ + kTileBytes;
  static constexpr uint32_t kK0 = kDO + kTileBytes;
  static constexpr uint32_t kStageBytes = 2u * kTileBytes;
  static constexpr uint32_t kDS = kK0 + kStages * kStageBytes;
  static constexpr uint32_t kBar = kDS + 128u * 128u * 2u;
  // q_full, q_empty, kv_full[2], kv_empty[2], s_full[2], s_empty[2], dp_full, dp_empty,
  // ds_full, ds_free, drain, item_full[4], item_empty[4]
  static constexpr uint32_t kNumBars = 23;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8u;  // tmem base, abort, item slots[4]
  static constexpr uint32_t kTotal = kMisc + 32u;
  static constexpr uint32_t kAlloc = kTotal + 1024u;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

template <int D>
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
  auto bar_kv_full = [&](uint32_t s) { return b0 + 16 + 8 * s; };
  auto bar_kv_empty = [&](uint32_t s) { return b0 + 32 + 8 * s; };
  auto bar_s_full = [&](uint32_t s) { return b0 + 48 + 8 * s; };
  auto bar_s_empty = [&](uint32_t s) { return b0 + 64 + 8 * s; };
  const uint32_t bar_dp_full = b0 + 80, bar_dp_empty = b0 + 88;
  const uint32_t bar_ds_full = b0 + 96, bar_ds_free = b0 + 104, bar_drain = b0 + 112;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  ptx::ItemRing ring;
  ring.slot = reinterpret_cast<volatile int*>(smem + L::kMisc + 16);
  ring.full = bar_drain + 8;
  ring.empty = ring.full + 8 * ptx::kItemSlots;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_q_full, 1);
    ptx::mbar_init(bar_q_empty, 1);
    for (uint32_t i = 0; i < kStages; ++i) {
      ptx::mbar_init(bar_kv_full(i), 1);
      ptx::mbar_init(bar_kv_empty(i), 1);
    }
    for (uint32_t i = 0; i < 2; ++i) {
      ptx::mbar_init(bar_s_full(i), 1);
      ptx::mbar_init(bar_s_empty(i), 128);
    }
    ptx::mbar_init(bar_dp_full, 1);
    ptx::mbar_init(bar_dp_empty, 128);
    ptx::mbar_init(bar_ds_full, 128);
    ptx::mbar_init(bar_ds_free, 1);
    ptx::mbar_init(bar_drain, 1);
    for (uint32_t i = 0; i < ptx::kItemSlots; ++i) {
      ptx::mbar_init(ring.full + 8 * i, 1);
      ptx::mbar_init(ring.empty + 8 * i, 129);  // MMA issuer + 128 gradient threads
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
      uint32_t kv_stage = 0, kv_phase = 0, q_phase = 0;
      uint32_t pend_mask = 0, pend_par = 0, q_fills = 0;
      bool ok = true;
      for (uint32_t rn = 0; ok; ++rn) {
        const int item = static_cast<int>(atomicAdd(a.counter, 1u));
        if (!ptx::ring_put(ring, rn, item, abort_flag, a.err, lim, ptx::wait_site(2, 0, 12))) { ok = false; break; }
        if (item >= a.n_items) break;
        const TileDesc td = a.tiles[a.order[item / Hq]];
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
        const int nkv = ceil_div(td.kv_end - td.doc_start, 128);
        const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
        for (int j = 0; j < nkv + nbr; ++j) {
          if (!ptx::mbar_wait(bar_kv_empty(kv_stage), kv_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 0, 2))) { ok = false; break; }
          ptx::mbar_expect_tx(bar_kv_full(kv_stage), 2u * L::kTileBytes);
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
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            ptx::tma_load_2d(sk + cb * 16384u, mk, bar_kv_full(kv_stage), g * D + cb * 64, y);
            ptx::tma_load_2d(sk + L::kTileBytes + cb * 16384u, mv, bar_kv_full(kv_stage), g * D + cb * 64, y);
          }
          pend_mask |= 1u << kv_stage;
          pend_par = (pend_par & ~(1u << kv_stage)) | (kv_phase << kv_stage);
          if (++kv_stage == kStages) { kv_stage = 0; kv_phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        volatile int never = 0;
        for (int i = 0; i < kStages; ++i)
          if (pend_mask & (1u << i))
            ptx::mbar_wait(bar_kv_full(i), (pend_par >> i) & 1u, &never, a.err, lim / 8);
        if (q_fills) ptx::mbar_wait(bar_q_full, (q_fills - 1) & 1u, &never, a.err, lim / 8);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdDQ = ptx::idesc_bf16_f32(128, D, false, true);
      uint32_t kv_stage = 0, kv_phase = 0, q_phase = 0, dp_phase = 0, ds_phase = 0, s_cnt = 0;
      bool ok = true;
      const uint32_t sQ = sbase + L::kQ, sDO = sbase + L::kDO, sDS = sbase + L::kDS;
      auto issue_dq = [&](int jj, uint32_t stage) -> bool {
        if (!ptx::mbar_wait(bar_ds_full, ds_phase, abort_flag, a.err, lim, ptx::wait_site(2, 1, 3))) return false;
        ds_phase ^= 1u;
        ptx::tc_fence_after();
        const uint32_t sk = sbase + L::kK0 + stage * L::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = ptx::sdesc_sw128(sDS + (kk >> 2) * 16384u + (kk & 3) * 32u, 16u, 1024u);
          const uint64_t bd = ptx::sdesc_sw128(sk + kk * 2048u, 16384u, 1024u);
          ptx::umma_ss(tmem + kColDQ, ad, bd, kIdDQ, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit(bar_ds_free);
        ptx::umma_commit(bar_kv_empty(stage));
        return true;
      };
      for (uint32_t rn = 0; ok; ++rn) {
        int item = 0;
        if (!ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(2, 1, 13))) { ok = false; break; }
        if (item >= a.n_items) break;
        const TileDesc td = a.tiles[a.order[item / Hq]];
        const int nkv = ceil_div(td.kv_end - td.doc_start, 128);
        const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
        const int n = nkv + nbr;
        if (!ptx::mbar_wait(bar_q_full, q_phase, abort_flag, a.err, lim, ptx::wait_site(2, 1, 4))) { ok = false; break; }
        q_phase ^= 1u;
        ptx::tc_fence_after();
        uint32_t prev_stage = 0;
        for (int j = 0; j < n; ++j) {
          if (!ptx::mbar_wait(bar_kv_full(kv_stage), kv_phase, abort_flag, a.err, lim, ptx::wait_site(2, 1, 5))) { ok = false; break; }
          const uint32_t sb = s_cnt & 1u;
          const uint32_t sph = (s_cnt >> 1) & 1u;
          if (!ptx::mbar_wait(bar_s_empty(sb), sph ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 1, 6))) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t sk = sbase + L::kK0 + kv_stage * L::kStageBytes;
          const uint32_t sv = sk + L::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
            ptx::umma_ss(tmem + kColS0 + sb * 128u, ptx::sdesc_sw128(sQ + off, 16u, 1024u),
                         ptx::sdesc_sw128(sk + off, 16u, 1024u), kIdS, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar_s_full(sb));
          ++s_cnt;
          if (!ptx::mbar_wait(bar_dp_empty, dp_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(2, 1, 7))) { ok = false; break; }
          dp_phase ^= 1u;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
            ptx::umma_ss(tmem + kColDP, ptx::sdesc_sw128(sDO + off, 16u, 1024u),
                         ptx::sdesc_sw128(sv + off, 16u, 1024u), kIdS, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar_dp_full);
          if (j == n - 1) ptx::umma_commit(bar_q_empty);
          if (j > 0 && !issue_dq(j - 1, prev_stage)) { ok = false; break; }
          prev_stage = kv_stage;
          if (++kv_stage == kStages) { kv_stage = 0; kv_phase ^= 1u; }
        }
        if (!ok) break;
        if (!issue_dq(n - 1, prev_stage)) { ok = false; break; }
      }
      ptx::umma_commit(bar_drain);
      volatile int never = 0;
      ptx::mbar_wait(bar_drain, 0, &never, a.err, lim);
    }
  } else {
    // ------------------------------------------------------------ dS / epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t sDS = sbase + L::kDS;
    const float sl2 = a.scale_log2;
    uint32_t s_cnt = 0, dp_cnt = 0, ds_cnt = 0;
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
      const int nkv = ceil_div(td.kv_end - td.doc_start, 128);
      const int nbr = (a.with_branch && td.br_hi > td.br_lo) ? ceil_div(td.br_hi - td.br_lo, 128) : 0;
      const int n = nkv + nbr;
      const int64_t slot = int64_t(td.row_base) + row;
      const SlotMeta m = a.meta[slot];
      const float neg_l2 = -a.ls[int64_t(h) * a.n_slots + slot];
      const float dval = a.ds[int64_t(h) * a.n_slots + slot];
      for (int j = 0; j < n; ++j) {
        const uint32_t sb = s_cnt & 1u;
        const uint32_t sph = (s_cnt >> 1) & 1u;
        bool w = ptx::mbar_wait(bar_s_full(sb), sph, abort_flag, a.err, lim, ptx::wait_site(2, 2, 8));
        w = w && ptx::mbar_wait(bar_dp_full, dp_cnt & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 2, 9));
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        ++dp_cnt;
        ptx::tc_fence_after();
        uint32_t dp[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tl + kColDP + c * 32u, dp[c]);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar_dp_empty);
        int lo, hi;
        if (j < nkv) {
          lo = 0;
          hi = m.limit - (td.doc_start + 128 * j) + 1;
        } else {
          const int kr0 = td.br_lo + 128 * (j - nkv);
          lo = m.blo - kr0;
          hi = m.bhi - kr0;
        }
        lo = max(lo, 0);
        hi = min(hi, 128);
        if (j > 0) {
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_ds_free, ds_cnt & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 2, 10)))) {
            ok = false;
            break;
          }
          ++ds_cnt;
        }
        // S in chunks of 32 columns; the load of chunk c+1 overlaps the math of chunk c.
        uint32_t sbuf[2][32];
        ptx::tmem_ld32(tl + kColS0 + sb * 128u, sbuf[0]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < 3) ptx::tmem_ld32(tl + kColS0 + sb * 128u + (c + 1) * 32u, sbuf[(c + 1) & 1]);
          const uint32_t* sr = sbuf[c & 1];
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float v2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = c * 32 + i + e;
              const float p = (col >= lo && col < hi)
                                  ? ptx::ex2(fmaf(__uint_as_float(sr[i + e]), sl2, neg_l2))
                                  : 0.f;
              v2[e] = p * (__uint_as_float(dp[c][i + e]) - dval);
            }
            pk[i >> 1] = ptx::pack_bf16x2(v2[0], v2[1]);
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int ch = c * 4 + q4;
            const uint32_t addr = sDS + (ch >> 3) * 16384u + row * 128u + (((ch & 7) ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[q4 * 4 + 0]),
                         "r"(pk[q4 * 4 + 1]), "r"(pk[q4 * 4 + 2]), "r"(pk[q4 * 4 + 3])
                         : "memory");
          }
          ptx::tmem_wait_ld();
          if (c == 2) {  // all four chunks of S are in registers now
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_s_empty(sb));
          }
        }
        ++s_cnt;
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar_ds_full);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_ds_free, ds_cnt & 1u, abort_flag, a.err, lim, ptx::wait_site(2, 2, 11)))) {
        ok = false;
        break;
      }
      ++ds_cnt;
      ptx::tc_fence_after();
      const int r = m.row;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t qv[32];
        ptx::tmem_ld32(tl + kColDQ + c * 32u, qv);
        ptx::tmem_wait_ld();
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

template <int D>
cudaError_t launch_d(const DqMaps& m, const DqArgs& a, int num_sms, cudaStream_t st) {
  using L = Smem<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kAlloc));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  bwd_dq_kernel<D><<<grid, kThreads, L::kAlloc, st>>>(m.qg, m.dog, m.k, m.v, m.kb, m.vb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dq(const DqMaps& m, const DqArgs& a, int num_sms, cudaStream_t st) {
  if (a.d == 128) return launch_d<128>(m, a, num_sms, st);
  if (a.d == 64) return launch_d<64>(m, a, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace ba
