// Branch-attention forward on sm_100a: tcgen05 MMA with TMEM accumulators,
// TMA-staged tiles, warp-specialised pipeline over two query tiles.
//
// Paper: arXiv 2609.07108 §3.2 / Eq. 2 (rcap.io post, branch-attention
// paragraph; cere-bro wiki, "Obstacle one, context parallelism").  One
// persistent CTA per SM walks (tile pair, query head) work items, longest
// first.  A pair is two consecutive row tiles A and B of one document; they
// share the document's main key tiles, so one K/V stream serves both: the
// main key tiles [doc start, larger limit] (each tile takes those up to its
// own limit), then A's branch-local key tiles, then B's.  Visiting key tiles
// one after another with a running (max, sum) is the same log-sum-exp merge
// ring attention applies between ring steps (Eq. 2), so the main-sequence
// component, the branch-local component and their merge all happen here.
//
// Per tile t in {A, B} and key tile j:
//   S_t = Q_t K_j^T                   -> TMEM buffer S_t
//   softmax warpgroup t: P = exp2(S * scale*log2e - m), bf16, written over
//       the first 64 columns of S_t
//   O_t += P V_j   (P read from TMEM) -> TMEM accumulator O_t
// The tensor pipe runs, in issue order, ... PV_A(j), S_A(j+1), PV_B(j),
// S_B(j+1) ...: S_t(j+1) overwrites S_t only after PV_t(j) has read P, and
// while one warpgroup computes its softmax the pipe works on the other tile.
//
// Roles (320 threads):
//   warp 0      producer: claims work items (one item ahead of the consumers)
//               and streams the K/V key tiles through a 2-stage TMA ring.
//   warp 1      TMEM allocator and single-thread MMA issuer.
//   warps 2-5   softmax / epilogue of tile A, warps 6-9 of tile B, one query
//               row per thread.  Each thread copies its own query row into
//               shared memory (cp.async); the next item's row goes in as soon
//               as the tile's last S MMA, the only reader of Q, has finished.
//               Per key tile: load S, mask by the row's key range, update the
//               running max (lazily: O is rescaled only when the max grows by
//               more than 2^8), write P; finally normalise O, write O and LSE.
//               A thread reads its S row twice, 32 columns at a time (once
//               for the row max, once for P), rather than holding all of it.
//
// Shared memory (D = head dim): Q_A | Q_B [128 x D each] | 2 x (K, V [128 x D]),
// bf16 in the 128-byte-swizzled layout (TMA writes K / V; the threads write Q
// in the same pattern).  TMEM: S_A 0, S_B 128, O_A 256, O_B 384.
#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

constexpr int kThreads = 320;
constexpr int kWarpProducer = 0, kWarpMma = 1;  // warps 2-9: softmax
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;  // tile t: S at kColS + 128 t, O at kColO + 128 t
constexpr float kRescaleThreshold = 8.0f;   // log2 units

template <int D>
struct Smem {
  static constexpr uint32_t kTileBytes = 128u * D * 2u;  // one 128-row bf16 tile
  static constexpr uint32_t kQ0 = 0;                     // Q_A, then Q_B
  static constexpr uint32_t kK0 = 2u * kTileBytes;
  static constexpr uint32_t kStageBytes = 2u * kTileBytes;  // K + V
  static constexpr uint32_t kBar = kK0 + kStages * kStageBytes;
  // barriers: q_full[2], kv_full[2], kv_empty[2], s_full[2], p_full[2], o_done[2], drain,
  // item_full[4], item_empty[4]
  static constexpr uint32_t kNumBars = 21;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8u;  // tmem base, abort, item slots[4]
  static constexpr uint32_t kTotal = kMisc + 32u;
  static constexpr uint32_t kAlloc = kTotal + 1024u;  // slack to align the base to 1024
};

struct Bars {
  uint32_t q_full[2], kv_full[kStages], kv_empty[kStages], s_full[2], p_full[2], o_done[2], drain;
};

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// The key-tile stream of a tile pair.  The main keys come as up to two
// segments [sl, sh), each cut into 128-key tiles from its first key:
//   - full rows: one segment from the first tile's first key (its document
//     start, or later under a window) to the larger limit + 1; two segments
//     when a window leaves a gap of at least a key tile between the tiles;
//   - ring partial k (virtual rank k): the keys of the document's zigzag
//     chunks k and 2R-1-k within that range.
// Then A's branch-local key tiles, then B's.
struct PairPlan {
  TileDesc t[2];
  bool on[2];   // tile present (the second tile of a pair may be absent)
  int lo[2], hi[2];  // each tile's main key range [lo, hi)
  int nkv[2];   // plain stream: main key tiles of each tile
  int nbr[2];   // branch key tiles of each tile
  int sl[2], sh[2], sn[2];  // main segments and their key tiles
  int nmain;    // main key tiles streamed: sn[0] + sn[1]
  int n;        // key tiles streamed
  int k;        // ring partial (virtual rank) of the item, 0 for full rows
};

// kGen selects the general stream (window, ring partials, bitmask words); the
// plain instantiation (full rows, chain or block masks, no window) keeps the
// one-segment stream [doc start, larger limit] with no per-tile range checks.
template <bool kGen>
__device__ __forceinline__ PairPlan load_pair(const FwdArgs& a, int item) {
  PairPlan pp;
  const int per = a.Hq * (a.ring > 0 ? a.ring : 1);
  const int pair = item / per;
  pp.k = a.ring > 0 ? (item / a.Hq) % a.ring : 0;
  const int2 ids = reinterpret_cast<const int2*>(a.pairs)[pair];
  const int id[2] = {ids.x, ids.y};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    pp.on[t] = id[t] >= 0;
    pp.nbr[t] = 0;
    if (pp.on[t]) {
      pp.t[t] = a.tiles[id[t]];
      if (a.with_branch && pp.t[t].br_hi > pp.t[t].br_lo)
        pp.nbr[t] = ceil_div(pp.t[t].br_hi - pp.t[t].br_lo, 128);
    } else {
      pp.t[t] = pp.t[0];
    }
    pp.lo[t] = pp.t[t].kv_lo;
    pp.hi[t] = pp.on[t] ? pp.t[t].kv_end : pp.t[t].kv_lo;
    pp.nkv[t] = pp.on[t] ? ceil_div(pp.t[t].kv_end - pp.t[t].doc_start, 128) : 0;
  }
  if constexpr (!kGen) {
    pp.sl[0] = pp.t[0].doc_start;
    pp.sn[0] = max(pp.nkv[0], pp.nkv[1]);
    pp.sh[0] = pp.sl[0] + 128 * pp.sn[0];
    pp.sl[1] = pp.sh[1] = pp.sh[0];
    pp.sn[1] = 0;
    pp.nmain = pp.sn[0];
    pp.n = pp.nmain + pp.nbr[0] + pp.nbr[1];
    return pp;
  }
  const int rlo = pp.lo[0], rhi = max(pp.hi[0], pp.hi[1]);
  if (a.ring > 0) {
    const int s = pp.t[0].doc_start;
    const int64_t L = pp.t[0].doc_end - s;
    const int64_t R2 = 2 * a.ring;
    const int c[2] = {pp.k, static_cast<int>(R2) - 1 - pp.k};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      pp.sl[g] = max(rlo, s + static_cast<int>(c[g] * L / R2));
      pp.sh[g] = min(rhi, s + static_cast<int>((c[g] + 1) * L / R2));
    }
  } else if (pp.on[1] && pp.lo[1] - pp.hi[0] >= 128) {
    pp.sl[0] = pp.lo[0];
    pp.sh[0] = pp.hi[0];
    pp.sl[1] = pp.lo[1];
    pp.sh[1] = pp.hi[1];
  } else {
    pp.sl[0] = rlo;
    pp.sh[0] = rhi;
    pp.sl[1] = pp.sh[1] = rhi;
  }
#pragma unroll
  for (int g = 0; g < 2; ++g) pp.sn[g] = pp.sh[g] > pp.sl[g] ? ceil_div(pp.sh[g] - pp.sl[g], 128) : 0;
  pp.nmain = pp.sn[0] + pp.sn[1];
  pp.n = pp.nmain + pp.nbr[0] + pp.nbr[1];
  return pp;
}

// (Fields are picked with selects, never indexed by a runtime value, so
// PairPlan stays in registers.)
// First key of main key tile j (< nmain) and whether it lies in segment 1.
__device__ __forceinline__ int main_key0(const PairPlan& pp, int j, bool& s1) {
  s1 = j >= pp.sn[0];
  return (s1 ? pp.sl[1] : pp.sl[0]) + 128 * (j - (s1 ? pp.sn[0] : 0));
}

// Does tile t take key tile j of the stream?
template <bool kGen>
__device__ __forceinline__ bool takes(const PairPlan& pp, int t, int j) {
  if (!(t ? pp.on[1] : pp.on[0])) return false;
  if (j < pp.nmain) {
    if constexpr (!kGen) return j < (t ? pp.nkv[1] : pp.nkv[0]);
    bool s1;
    const int y = main_key0(pp, j, s1);
    return max(y, t ? pp.lo[1] : pp.lo[0]) <
           min(min(y + 128, s1 ? pp.sh[1] : pp.sh[0]), t ? pp.hi[1] : pp.hi[0]);
  }
  j -= pp.nmain;
  return t == 0 ? j < pp.nbr[0] : j >= pp.nbr[0];
}

// Index of the last key tile tile t takes (-1: none).
template <bool kGen>
__device__ __forceinline__ int last_taken(const PairPlan& pp, int t) {
  if (!(t ? pp.on[1] : pp.on[0])) return -1;
  if ((t ? pp.nbr[1] : pp.nbr[0]) > 0) return t == 0 ? pp.nmain + pp.nbr[0] - 1 : pp.n - 1;
  if constexpr (!kGen) return (t ? pp.nkv[1] : pp.nkv[0]) - 1;
  const int lo = t ? pp.lo[1] : pp.lo[0], hi = t ? pp.hi[1] : pp.hi[0];
  const int e1 = min(pp.sh[1], hi);
  if (max(pp.sl[1], lo) < e1) return pp.sn[0] + (e1 - 1 - pp.sl[1]) / 128;
  const int e0 = min(pp.sh[0], hi);
  if (max(pp.sl[0], lo) < e0) return (e0 - 1 - pp.sl[0]) / 128;
  return -1;
}

template <int D, bool kGen>
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
    for (int i = 0; i < 2; ++i) { bar.q_full[i] = b; b += 8; }
    for (int i = 0; i < kStages; ++i) { bar.kv_full[i] = b; b += 8; }
    for (int i = 0; i < kStages; ++i) { bar.kv_empty[i] = b; b += 8; }
    for (int i = 0; i < 2; ++i) { bar.s_full[i] = b; b += 8; }
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
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar.q_full[i], 128);  // one arrival per softmax thread (its copied row)
      ptx::mbar_init(bar.s_full[i], 1);
      ptx::mbar_init(bar.p_full[i], 128);
      ptx::mbar_init(bar.o_done[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(bar.kv_full[i], 1);
      ptx::mbar_init(bar.kv_empty[i], 1);
    }
    ptx::mbar_init(bar.drain, 1);
    for (uint32_t i = 0; i < ptx::kItemSlots; ++i) {
      ptx::mbar_init(ring.full + 8 * i, 1);
      ptx::mbar_init(ring.empty + 8 * i, 257);  // MMA issuer + 256 softmax threads
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    ptx::prefetch_tmap(&tmKb);
    ptx::prefetch_tmap(&tmVb);
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(sbase + L::kMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int Hq = a.Hq;
  const long long lim = a.wait_limit;

  if (warp == kWarpProducer) {
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
        const PairPlan pp = load_pair<kGen>(a, cur);
        const int g = (cur % Hq) / a.G;
        for (int j = 0; j < pp.n; ++j) {
          if (!ptx::mbar_wait(bar.kv_empty[kv_stage], kv_phase ^ 1u, abort_flag, a.err, lim, ptx::wait_site(1, 0, 2))) {
            ok = false;
            break;
          }
          ptx::mbar_expect_tx(bar.kv_full[kv_stage], 2u * L::kTileBytes);
          const void* mk = &tmK;
          const void* mv = &tmV;
          int y;
          if (j < pp.nmain) {
            bool s1;
            y = main_key0(pp, j, s1);
          } else {
            const int jb = j - pp.nmain;
            y = jb < pp.nbr[0] ? pp.t[0].br_lo + 128 * jb : pp.t[1].br_lo + 128 * (jb - pp.nbr[0]);
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
      {
        // Our own copies land before the CTA exits (on a normal exit every
        // fill was consumed, so these waits return at once).
        volatile int never = 0;
        for (int i = 0; i < kStages; ++i)
          if (pend_mask & (1u << i))
            ptx::mbar_wait(bar.kv_full[i], (pend_par >> i) & 1u, &never, a.err, ptx::kDrainCycles);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = ptx::idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPV = ptx::idesc_bf16_f32(128, D, false, true);
      uint32_t kv_stage = 0, kv_phase = 0;
      uint32_t q_phase[2] = {0u, 0u};
      uint32_t p_cnt[2] = {0u, 0u};  // P tiles consumed per tile slot (p_full parity)
      // Shared-memory descriptors of every tile and stage, built once: rebuilding
      // them per MMA group costs the issuing thread more than an MMA takes.
      const uint64_t dq0 = ptx::sdesc_sw128(sbase + L::kQ0, 16u, 1024u);
      const uint64_t dq1 = ptx::sdesc_sw128(sbase + L::kQ0 + L::kTileBytes, 16u, 1024u);
      const uint64_t dk0 = ptx::sdesc_sw128(sbase + L::kK0, 16u, 1024u);
      const uint64_t dk1 = ptx::sdesc_sw128(sbase + L::kK0 + L::kStageBytes, 16u, 1024u);
      const uint64_t dv0 = ptx::sdesc_sw128(sbase + L::kK0 + L::kTileBytes, 16384u, 1024u);
      const uint64_t dv1 = ptx::sdesc_sw128(sbase + L::kK0 + L::kStageBytes + L::kTileBytes, 16384u, 1024u);
      bool ok = true;
      for (uint32_t rn = 0; ok; ++rn) {
        int item = 0;
        if (!ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(1, 1, 13))) { ok = false; break; }
        if (item >= a.n_items) break;
        const PairPlan pp = load_pair<kGen>(a, item);
        bool first_s[2] = {true, true}, first_pv[2] = {true, true};
        // S_t(j) = Q_t K_j^T into tile t's S buffer (the P.V that last read it was issued before).
        auto issue_s = [&](int t, uint32_t stage) -> bool {
          if (first_s[t]) {  // this tile's query rows have been copied in
            if (!ptx::mbar_wait(bar.q_full[t], q_phase[t], abort_flag, a.err, lim, ptx::wait_site(1, 1, 4))) return false;
            q_phase[t] ^= 1u;
            ptx::tc_fence_after();
            first_s[t] = false;
          }
          const uint64_t ad0 = t ? dq1 : dq0;
          const uint64_t bd0 = stage ? dk1 : dk0;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
            ptx::umma_ss(tmem + kColS + t * 128u, ptx::sdesc_add(ad0, off), ptx::sdesc_add(bd0, off), kIdS,
                         kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit(bar.s_full[t]);
          return true;
        };
        // O_t += P_t V_j with P_t read from tile t's S buffer in TMEM.
        auto issue_pv = [&](int t, uint32_t stage) -> bool {
          if (!ptx::mbar_wait(bar.p_full[t], p_cnt[t] & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 1, 3))) return false;
          ++p_cnt[t];
          ptx::tc_fence_after();
          const uint64_t bd0 = stage ? dv1 : dv0;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::umma_ts(tmem + kColO + t * 128u, tmem + kColS + t * 128u + kk * 8u, ptx::sdesc_add(bd0, kk * 2048u),
                         kIdPV, (!first_pv[t] || kk > 0) ? 1u : 0u);
          first_pv[t] = false;
          ptx::umma_commit(bar.o_done[t]);
          return true;
        };
        if (pp.n == 0) continue;
        // prologue: the S MMAs of key tile 0
        if (!ptx::mbar_wait(bar.kv_full[kv_stage], kv_phase, abort_flag, a.err, lim, ptx::wait_site(1, 1, 5))) { ok = false; break; }
        ptx::tc_fence_after();
        for (int t = 0; t < 2 && ok; ++t)
          if (takes<kGen>(pp, t, 0) && !issue_s(t, kv_stage)) ok = false;
        for (int j = 0; j < pp.n && ok; ++j) {
          const uint32_t st_j = kv_stage;
          uint32_t st_n = kv_stage + 1, ph_n = kv_phase;
          if (st_n == kStages) { st_n = 0; ph_n ^= 1u; }
          const bool more = j + 1 < pp.n;
          if (takes<kGen>(pp, 0, j) && !issue_pv(0, st_j)) { ok = false; break; }
          if (more) {
            if (!ptx::mbar_wait(bar.kv_full[st_n], ph_n, abort_flag, a.err, lim, ptx::wait_site(1, 1, 5))) { ok = false; break; }
            ptx::tc_fence_after();
            if (takes<kGen>(pp, 0, j + 1) && !issue_s(0, st_n)) { ok = false; break; }
          }
          if (takes<kGen>(pp, 1, j) && !issue_pv(1, st_j)) { ok = false; break; }
          ptx::umma_commit(bar.kv_empty[st_j]);
          if (more && takes<kGen>(pp, 1, j + 1) && !issue_s(1, st_n)) { ok = false; break; }
          kv_stage = st_n;
          kv_phase = ph_n;
        }
      }
      // Drain: every MMA this thread issued completes before TMEM is freed.
      ptx::umma_commit(bar.drain);
      volatile int never = 0;
      ptx::mbar_wait(bar.drain, 0, &never, a.err, ptx::kDrainCycles);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int t = (warp - 2) >> 2;  // tile of the pair this warpgroup serves
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t colS = kColS + static_cast<uint32_t>(t) * 128u;
    const uint32_t colO = kColO + static_cast<uint32_t>(t) * 128u;
    const uint32_t sQ = sbase + L::kQ0 + static_cast<uint32_t>(t) * L::kTileBytes;
    // this warpgroup's barriers (selected, not indexed, so `bar` stays in registers)
    const uint32_t my_q_full = t ? bar.q_full[1] : bar.q_full[0];
    const uint32_t my_s_full = t ? bar.s_full[1] : bar.s_full[0];
    const uint32_t my_p_full = t ? bar.p_full[1] : bar.p_full[0];
    const uint32_t my_o_done = t ? bar.o_done[1] : bar.o_done[0];
    const float sl2 = a.scale_log2;
    uint32_t s_cnt = 0, p_cnt = 0;  // S tiles consumed, P tiles produced

    // This thread's row of the warpgroup's tile in a work item.
    struct RowItem {
      bool valid, on;
      int h, k, n, nmain, nkv, sn0, nbr0, last;
      int sl0, sh0, sl1, sh1, tlo, thi;  // main segments and the tile's main key range
      int br_lo, r, limit, rlo, blo, bhi;  // the row: main keys [rlo, limit], branch [blo, bhi)
      uint64_t bits;                        // the row's branch mask word (BA_MASK_BITMASK)
    };
    auto get_item = [&](uint32_t rn, int& item) -> bool {
      return __all_sync(0xffffffffu, ptx::ring_get(ring, rn, &item, abort_flag, a.err, lim, ptx::wait_site(1, 2, 14)));
    };
    auto make_row = [&](int item, RowItem& it) {
      it.valid = item < a.n_items;
      it.on = false;
      if (!it.valid) return;
      const PairPlan pp = load_pair<kGen>(a, item);
      it.on = t ? pp.on[1] : pp.on[0];
      if (!it.on) return;
      const TileDesc td = t ? pp.t[1] : pp.t[0];
      it.h = item % Hq;
      it.k = pp.k;
      it.n = pp.n;
      it.nmain = pp.nmain;
      it.nkv = t ? pp.nkv[1] : pp.nkv[0];
      it.sn0 = pp.sn[0];
      it.nbr0 = pp.nbr[0];
      it.last = last_taken<kGen>(pp, t);
      it.sl0 = pp.sl[0];
      it.sh0 = pp.sh[0];
      it.sl1 = pp.sl[1];
      it.sh1 = pp.sh[1];
      it.tlo = t ? pp.lo[1] : pp.lo[0];
      it.thi = t ? pp.hi[1] : pp.hi[0];
      it.br_lo = td.br_lo;
      it.r = a.row_table[td.row_base + row];
      it.limit = td.doc_start;  // padding rows see at most one key: keeps their math finite
      it.rlo = td.doc_start;
      it.blo = it.bhi = 0;      // visible branch key rows [blo, bhi)
      it.bits = 0;
      if (it.r >= 0 && it.r < a.S) {
        it.limit = it.r;
      } else if (it.r >= a.S) {
        const int b = (it.r - a.S) / a.B;
        const int tt = (it.r - a.S) - b * a.B;
        it.limit = a.anchors[b];
        it.blo = b * a.B;
        it.bhi = it.blo + (a.mode == 0 ? tt + 1 : a.B);
        if (kGen && a.mode == 2) it.bits = a.bmask[it.r - a.S];
      }
      if (kGen && a.window > 0 && it.r >= 0) it.rlo = max(td.doc_start, it.limit - a.window + 1);
    };
    // Where this thread's query row of `item` lives (false: the tile is absent
    // or takes no key tile of the item, so no S MMA reads its Q).
    auto q_src = [&](int item, const __nv_bfloat16*& src, uint32_t& bytes) -> bool {
      if (item >= a.n_items) return false;
      int row_base;
      if constexpr (kGen) {
        const PairPlan pp = load_pair<kGen>(a, item);
        if (last_taken<kGen>(pp, t) < 0) return false;
        row_base = (t ? pp.t[1] : pp.t[0]).row_base;
      } else {  // every present tile takes at least its first main key tile
        const int2 ids = reinterpret_cast<const int2*>(a.pairs)[item / Hq];
        const int id = t == 0 ? ids.x : ids.y;
        if (id < 0) return false;
        row_base = a.tiles[id].row_base;
      }
      const int r = a.row_table[row_base + row];
      const int h = item % Hq;
      src = a.q;  // padding row: zero-filled
      bytes = 0;
      if (r >= 0 && r < a.S) {
        src = a.q + (int64_t(r) * Hq + h) * D;
        bytes = 16;
      } else if (r >= a.S) {
        src = a.qb + (int64_t(r - a.S) * Hq + h) * D;
        bytes = 16;
      }
      return true;
    };
    // Does this warpgroup's tile take key tile j of the item's stream?
    auto takes_own = [&](const RowItem& it, int j) -> bool {
      if (j < it.nmain) {
        if constexpr (!kGen) return j < it.nkv;  // the plain stream: a prefix of the main tiles
        const bool s1 = j >= it.sn0;
        const int y = (s1 ? it.sl1 : it.sl0) + 128 * (j - (s1 ? it.sn0 : 0));
        return max(y, it.tlo) < min(min(y + 128, s1 ? it.sh1 : it.sh0), it.thi);
      }
      return t == 0 ? j - it.nmain < it.nbr0 : j - it.nmain >= it.nbr0;
    };
    // Copy this thread's query row (bf16, D values) into row `row` of the
    // swizzled Q tile; padding rows are zero-filled.
    auto copy_q = [&](const __nv_bfloat16* src, uint32_t bytes) {
      const uint32_t dst = sQ + static_cast<uint32_t>(row) * 128u;
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
      ptx::mbar_arrive(my_q_full);
    };

    RowItem cur;
    int item0 = 0;
    bool ok = get_item(0, item0);
    if (ok) {
      make_row(item0, cur);
      const __nv_bfloat16* src;
      uint32_t bytes;
      if (q_src(item0, src, bytes)) {
        copy_q(src, bytes);
        publish_q();
      }
    }
    for (uint32_t rn = 1; ok && cur.valid; ++rn) {
      int nxt_item = 0;
      bool nxt_on = false, fetched = false;
      const __nv_bfloat16* nsrc = a.q;
      uint32_t nbytes = 0;
      if (cur.on) {
        const int h = cur.h, nmain = cur.nmain, r = cur.r;
        const int limit = cur.limit, blo = cur.blo, bhi = cur.bhi;
        const bool use_bits = kGen && a.mode == 2;
        float m_used = -INFINITY;
        float l = 0.f;
        bool first = true;
        for (int j = 0; j < cur.n; ++j) {
          if (!takes_own(cur, j)) continue;
          if (j == cur.last) {
            if (!get_item(rn, nxt_item)) {
              ok = false;
              break;
            }
            fetched = true;
            nxt_on = q_src(nxt_item, nsrc, nbytes);
          }
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(my_s_full, s_cnt & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 2, 7)))) {
            ok = false;
            break;
          }
          ++s_cnt;
          ptx::tc_fence_after();
          // The tile's last S MMA has finished: the next item's rows may overwrite Q.
          if (j == cur.last && nxt_on) copy_q(nsrc, nbytes);
          // visible columns [lo, hi) of this key tile (and, for a bitmask
          // branch tile, those whose bit is set: column c is branch key c - sh)
          int lo, hi, sh = 0;
          bool bitm = false;
          if (j < nmain) {
            if constexpr (kGen) {
              const bool s1 = j >= cur.sn0;
              const int y = (s1 ? cur.sl1 : cur.sl0) + 128 * (j - (s1 ? cur.sn0 : 0));
              lo = max(cur.rlo, s1 ? cur.sl1 : cur.sl0) - y;
              hi = min(limit + 1, s1 ? cur.sh1 : cur.sh0) - y;
            } else {
              lo = 0;
              hi = limit - (cur.sl0 + 128 * j) + 1;
            }
          } else {
            const int kb = t == 0 ? j - nmain : j - nmain - cur.nbr0;
            const int kr0 = cur.br_lo + 128 * kb;
            lo = blo - kr0;
            hi = bhi - kr0;
            sh = lo;
            bitm = use_bits;
          }
          lo = max(lo, 0);
          hi = min(hi, 128);
          const bool full = lo == 0 && hi == 128 && !bitm;
          const uint64_t bits = cur.bits;
          auto masked = [&](int col) -> bool {
            if constexpr (!kGen) return col < lo || col >= hi;
            return col < lo || col >= hi || (bitm && !((bits >> (col - sh)) & 1ull));
          };
          // Pass 1: row max, 32 columns at a time, 8 independent accumulators.
          float mx8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t sr[32];
            ptx::tmem_ld32(tl + colS + c * 32u, sr);
            ptx::tmem_wait_ld();
            ptx::tmem_regs_ready(sr);
            if (!full) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (masked(c * 32 + i)) sr[i] = __float_as_uint(-INFINITY);
            }
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              mx8[(i >> 1) & 7] = ptx::max3(mx8[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
          }
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
          // Rescaling O needs this tile's previous P.V to have finished.
          const bool any_rescale = __any_sync(0xffffffffu, rescale);
          if (any_rescale && !first) {
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(my_o_done, (p_cnt - 1u) & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 2, 10)))) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t ov[32];
              ptx::tmem_ld32(tl + colO + c * 32u, ov);
              ptx::tmem_wait_ld();
              ptx::tmem_regs_ready(ov);
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              ptx::tmem_st32(tl + colO + c * 32u, ov);
            }
          }
          // Pass 2: P = exp2(S * scale*log2(e) - m) as bf16 pairs over the first
          // 64 columns of S, row sum over 4 paired accumulators.
          const float2 c2 = make_float2(sl2, sl2);
          // a row with no visible key so far keeps m = -inf; subtract 0 then, so P = 0 exactly
          const float mref = (kGen && m_used == -INFINITY) ? 0.f : m_used;
          const float2 nm2 = make_float2(-mref, -mref);
          float2 rs4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) rs4[u] = make_float2(0.f, 0.f);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t sr[32];
            ptx::tmem_ld32(tl + colS + c * 32u, sr);
            ptx::tmem_wait_ld();
            ptx::tmem_regs_ready(sr);
            if (!full) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (masked(c * 32 + i)) sr[i] = __float_as_uint(-INFINITY);
            }
            uint32_t pw[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 x = ptx::fma2(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), c2, nm2);
              // every other pair on the FMA pipe: two warpgroups share one special-function unit
              const float2 p = ((i >> 1) & 1) ? ptx::exp2_poly(x) : ptx::exp2_sfu(x);
              rs4[(i >> 1) & 3] = ptx::add2(rs4[(i >> 1) & 3], p);
              pw[i >> 1] = ptx::pack_bf16x2(p.x, p.y);
            }
            // keys 32c..32c+31 -> P columns 16c..16c+15, S columns read in this or an earlier chunk
            ptx::tmem_st16(tl + colS + c * 16u, pw);
          }
          const float2 rsa = ptx::add2(ptx::add2(rs4[0], rs4[1]), ptx::add2(rs4[2], rs4[3]));
          l = l * alpha + (rsa.x + rsa.y);
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          ptx::mbar_arrive(my_p_full);
          ++p_cnt;
          first = false;
        }
        if (!ok) break;
        // The next item's S MMAs may start while this item's epilogue runs.
        if (nxt_on) publish_q();
        // ---------------------------------------------------------- epilogue
        // the tile's last P.V (and, in order, every earlier one) finished
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(my_o_done, (p_cnt - 1u) & 1u, abort_flag, a.err, lim, ptx::wait_site(1, 2, 11)))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // l == 0: the row saw no key of this item (a ring partial may be
        // empty): O = 0, LSE = -inf, whatever TMEM holds
        const bool empty = kGen && !(l > 0.f);
        const float inv_l = empty ? 0.f : 1.f / l;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          ptx::tmem_ld32(tl + colO + c * 32u, ov);
          ptx::tmem_wait_ld();
          ptx::tmem_regs_ready(ov);
          if (empty) {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0u;
          }
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
              float* dst = a.o_part + (kGen ? int64_t(cur.k) * a.o_part_stride : 0) +
                           (int64_t(r) * Hq + h) * D + c * 32;
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
        if (r >= 0)
          a.lse[(kGen ? int64_t(cur.k) * a.lse_stride : 0) + int64_t(h) * a.lse_ld + r] =
              empty ? -INFINITY : (m_used + __log2f(l)) * 0.69314718055994531f;
        ptx::tc_fence_before();
      }
      if (!fetched) {
        // This tile had no part in the item: take the next one now; the tile's
        // Q buffer is free (its last S MMA finished before this item began).
        if (!get_item(rn, nxt_item)) {
          ok = false;
          break;
        }
        if (q_src(nxt_item, nsrc, nbytes)) {
          copy_q(nsrc, nbytes);
          publish_q();
        }
      }
      make_row(nxt_item, cur);
    }
    // Copies this thread issued must land before the CTA's shared memory goes away.
    ptx::cp_async_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kGen>
cudaError_t launch_fwd_d(const FwdMaps& m, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  using L = Smem<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(fwd_kernel<D, kGen>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::kAlloc));
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  fwd_kernel<D, kGen><<<grid, kThreads, L::kAlloc, stream>>>(m.k, m.v, m.kb, m.vb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const FwdMaps& maps, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  // the general stream only where a window, ring partials or mask words need it
  const bool gen = a.window > 0 || a.ring > 0 || a.mode == 2;
  if (a.d == 128) return gen ? launch_fwd_d<128, true>(maps, a, num_sms, stream)
                             : launch_fwd_d<128, false>(maps, a, num_sms, stream);
  if (a.d == 64) return gen ? launch_fwd_d<64, true>(maps, a, num_sms, stream)
                            : launch_fwd_d<64, false>(maps, a, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ba
