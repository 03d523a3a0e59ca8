// Host planner: validation, zigzag chunks, row tiles, longest-first order.
#include "plan.h"

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <utility>

namespace ba {

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// First index i in [lo, hi) with a[i] >= x.
int lower_bound_i(const int32_t* a, int lo, int hi, int64_t x) {
  return static_cast<int>(std::lower_bound(a + lo, a + hi, x) - a);
}

}  // namespace

int64_t pair_main_tiles(const TileDesc& a, const TileDesc& b) {
  // One stream [a.kv_lo, b.kv_end) unless a gap of at least a whole key tile
  // separates the two tiles' ranges; then two streams.
  const int64_t K = kKeysPerTile;
  if (int64_t(b.kv_lo) - a.kv_end >= K)
    return (int64_t(a.kv_end) - a.kv_lo + K - 1) / K + (int64_t(b.kv_end) - b.kv_lo + K - 1) / K;
  const int64_t hi = std::max(a.kv_end, b.kv_end);
  return (hi - a.kv_lo + K - 1) / K;
}

ba_status validate(const ba_problem* p, bool need_tensors) {
  if (!p) return BA_ERR_INVALID_ARG;
  if (p->S < 1 || p->ndoc < 1 || p->ndoc > p->S) return BA_ERR_INVALID_ARG;
  if (p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv != 0) return BA_ERR_INVALID_ARG;
  if (p->d < 1 || p->Nb < 0 || p->R < 1 || p->R > 64) return BA_ERR_INVALID_ARG;
  if (p->mode != BA_MASK_CHAIN && p->mode != BA_MASK_BLOCK && p->mode != BA_MASK_BITMASK)
    return BA_ERR_INVALID_ARG;
  if (p->mode == BA_MASK_BITMASK && p->Nb > 0) {
    if (!p->branch_mask_h || !p->branch_mask_d || !aligned16(p->branch_mask_d))
      return BA_ERR_INVALID_ARG;
  }
  if (p->Nb > 0 && (p->B < 1 || p->B > 64)) return BA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return BA_ERR_UNSUPPORTED;
  if (p->cp_select != 0 && (p->cp_select != 1 || p->cp_rank < 0 || p->cp_rank >= p->R))
    return BA_ERR_INVALID_ARG;
  // Row indices and head-major LSE offsets must fit the kernels' int32 row math.
  const int64_t rows = (int64_t)p->S + (int64_t)p->Nb * (p->Nb > 0 ? p->B : 0);
  if (rows >= (int64_t(1) << 31) - kRowsPerTile * 4) return BA_ERR_UNSUPPORTED;
  if (!p->cu_seqlens_h || !p->cu_seqlens_d) return BA_ERR_INVALID_ARG;
  if (p->Nb > 0 && (!p->anchors_h || !p->anchors_d)) return BA_ERR_INVALID_ARG;
  const int32_t* cu = p->cu_seqlens_h;
  if (cu[0] != 0 || cu[p->ndoc] != p->S) return BA_ERR_INVALID_ARG;
  for (int i = 0; i < p->ndoc; ++i)
    if (cu[i + 1] <= cu[i]) return BA_ERR_INVALID_ARG;  // empty or decreasing document
  for (int b = 0; b < p->Nb; ++b) {
    const int32_t a = p->anchors_h[b];
    if (a < 0 || a >= p->S) return BA_ERR_INVALID_ARG;
    if (b > 0 && a < p->anchors_h[b - 1]) return BA_ERR_INVALID_ARG;
  }
  if (!aligned16(p->cu_seqlens_d) || (p->Nb > 0 && !aligned16(p->anchors_d)))
    return BA_ERR_INVALID_ARG;
  if (need_tensors) {
    if (!p->q || !p->k || !p->v) return BA_ERR_INVALID_ARG;
    if (!aligned16(p->q) || !aligned16(p->k) || !aligned16(p->v)) return BA_ERR_INVALID_ARG;
    if (p->Nb > 0) {
      if (!p->qb || !p->kb || !p->vb) return BA_ERR_INVALID_ARG;
      if (!aligned16(p->qb) || !aligned16(p->kb) || !aligned16(p->vb)) return BA_ERR_INVALID_ARG;
    }
  }
  return BA_OK;
}

void build_plan(const ba_problem* p, Plan* plan) {
  const int S = p->S, R = p->R;
  const int Nb = p->Nb, B = (p->Nb > 0 ? p->B : 0);
  const int32_t* cu = p->cu_seqlens_h;
  const int32_t* anc = p->anchors_h;
  plan->S = S;
  plan->Nb = Nb;
  plan->B = B;
  plan->R = R;
  plan->ndoc = p->ndoc;
  plan->chunks.clear();
  plan->tiles.clear();
  plan->chunks_dev.clear();
  plan->n_tile_pairs = plan->n_branch_tile_pairs = plan->n_visible_pairs = 0;
  plan->rank_pairs.assign(R, 0);

  const int64_t W = p->window > 0 ? p->window : 0;
  const bool one_rank = p->cp_select != 0;
  // sum over n in [n0, n1] of min(n, W) (W = 0: no window)
  auto prefix_sum = [&](int64_t n0, int64_t n1) -> int64_t {
    if (n1 < n0) return 0;
    auto upto = [&](int64_t n) -> int64_t {  // sum over [1, n]
      if (W > 0 && n > W) return W * (W + 1) / 2 + (n - W) * W;
      return n * (n + 1) / 2;
    };
    return upto(n1) - upto(n0 - 1);
  };
  int64_t vis = 0;  // exact visible pairs per head of the rows this plan covers

  int tile_count = 0;
  for (int di = 0; di < p->ndoc; ++di) {
    const int s = cu[di], e = cu[di + 1];
    const int64_t L = e - s;
    // Zigzag chunks of this document and their owning virtual ranks.
    const size_t chunk0 = plan->chunks.size();
    for (int k = 0; k < 2 * R; ++k) {
      Chunk c;
      c.doc = di;
      c.k = k;
      c.rank = k < R ? k : 2 * R - 1 - k;
      c.c0 = s + static_cast<int>((int64_t(k) * L) / (2 * R));
      c.c1 = s + static_cast<int>((int64_t(k + 1) * L) / (2 * R));
      c.b0 = Nb ? lower_bound_i(anc, 0, Nb, c.c0) : 0;
      c.b1 = Nb ? lower_bound_i(anc, c.b0, Nb, c.c1) : 0;
      c.n_rows = int64_t(c.c1 - c.c0) + int64_t(B) * (c.b1 - c.b0);
      c.tile0 = c.ntiles = 0;
      plan->chunks.push_back(c);
    }
    // The row segments of this document the plan covers: the whole document,
    // or (one rank's rows) the rank's two zigzag chunks, positions [c0, c1)
    // with the branches anchored there.
    int seg_lo[2], seg_hi[2], nseg = 0;
    if (!one_rank) {
      seg_lo[0] = s;
      seg_hi[0] = e;
      nseg = 1;
    } else {
      const Chunk& ca = plan->chunks[chunk0 + p->cp_rank];
      const Chunk& cb = plan->chunks[chunk0 + 2 * R - 1 - p->cp_rank];
      if (ca.c1 > ca.c0) { seg_lo[nseg] = ca.c0; seg_hi[nseg] = ca.c1; ++nseg; }
      if (cb.c1 > cb.c0) { seg_lo[nseg] = cb.c0; seg_hi[nseg] = cb.c1; ++nseg; }
    }
    for (int sg = 0; sg < nseg; ++sg) {
      // Row tiles over the segment's rows in limit order (main row p, then
      // the branch rows anchored at p).  A tile may cross a zigzag chunk edge
      // (whole documents); it is owned by the virtual rank whose chunk holds
      // its first row.
      const int c0 = seg_lo[sg], c1 = seg_hi[sg];
      const int b0 = Nb ? lower_bound_i(anc, 0, Nb, c0) : 0;
      const int b1 = Nb ? lower_bound_i(anc, b0, Nb, c1) : 0;
      const int64_t n_rows = int64_t(c1 - c0) + int64_t(B) * (b1 - b0);
      const int ntiles = static_cast<int>((n_rows + kRowsPerTile - 1) / kRowsPerTile);
      vis += prefix_sum(c0 - s + 1, c1 - s);
      for (int b = b0; b < b1; ++b) {
        vis += int64_t(B) * prefix_sum(anc[b] - s + 1, anc[b] - s + 1);
        if (p->mode == BA_MASK_CHAIN) {
          vis += int64_t(B) * (B + 1) / 2;
        } else if (p->mode == BA_MASK_BLOCK) {
          vis += int64_t(B) * B;
        } else {
          const uint64_t keep = B >= 64 ? ~uint64_t(0) : ((uint64_t(1) << B) - 1);
          for (int t = 0; t < B; ++t) vis += __builtin_popcountll(p->branch_mask_h[int64_t(b) * B + t] & keep);
        }
      }
      ChunkDev cd;
      cd.c0 = c0;
      cd.b0 = b0;
      cd.slot_base = tile_count * kRowsPerTile;
      cd.pad = c1;
      plan->chunks_dev.push_back(cd);
      // merged index of main position q within the segment
      auto main_index = [&](int q) -> int64_t {
        const int lb = Nb ? lower_bound_i(anc, b0, b1, q) : 0;
        return int64_t(q - c0) + int64_t(B) * (lb - b0);
      };
      // limit of the row at merged index m: largest q in [c0, c1) with main_index(q) <= m
      auto limit_at = [&](int64_t m) -> int {
        int lo = c0, hi = c1 - 1;
        while (lo < hi) {
          const int mid = lo + (hi - lo + 1) / 2;
          if (main_index(mid) <= m) lo = mid; else hi = mid - 1;
        }
        return lo;
      };
      // first merged index of branch b's rows
      auto branch_start = [&](int b) -> int64_t {
        return int64_t(anc[b] - c0) + 1 + int64_t(B) * (b - b0);
      };
      for (int t = 0; t < ntiles; ++t) {
        const int64_t m0 = int64_t(t) * kRowsPerTile;
        const int64_t m1 = std::min<int64_t>(n_rows, m0 + kRowsPerTile);
        TileDesc td;
        td.row_base = (tile_count + t) * kRowsPerTile;
        td.n_rows = static_cast<int32_t>(m1 - m0);
        td.doc_start = s;
        td.min_limit = limit_at(m0);
        td.kv_end = limit_at(m1 - 1) + 1;
        td.kv_lo = W > 0 ? static_cast<int32_t>(std::max<int64_t>(s, td.min_limit - W + 1)) : s;
        td.doc_end = e;
        td.pad0 = td.pad1 = 0;
        td.rank = 0;
        for (int k = 0; k < 2 * R; ++k) {
          const Chunk& c = plan->chunks[chunk0 + k];
          if (c.c0 <= td.min_limit && td.min_limit < c.c1) td.rank = c.rank;
        }
        td.br_lo = td.br_hi = 0;
        if (b1 > b0) {
          // branches whose rows [start, start + B) meet [m0, m1)
          int lo = b0, hi = b1;  // first b with start(b) + B > m0
          while (lo < hi) {
            const int mid = (lo + hi) / 2;
            if (branch_start(mid) + B > m0) hi = mid; else lo = mid + 1;
          }
          const int blo = lo;
          lo = b0;
          hi = b1;  // first b with start(b) >= m1
          while (lo < hi) {
            const int mid = (lo + hi) / 2;
            if (branch_start(mid) >= m1) hi = mid; else lo = mid + 1;
          }
          const int bhi = lo;  // exclusive
          if (bhi > blo) {
            td.br_lo = blo * B;
            td.br_hi = bhi * B;
          }
        }
        const int64_t nkv = (int64_t(td.kv_end) - td.kv_lo + kKeysPerTile - 1) / kKeysPerTile;
        const int64_t nbr = (int64_t(td.br_hi) - td.br_lo + kKeysPerTile - 1) / kKeysPerTile;
        plan->n_tile_pairs += nkv;
        plan->n_branch_tile_pairs += std::max<int64_t>(0, nbr);
        plan->rank_pairs[td.rank] += nkv;
        plan->tiles.push_back(td);
      }
      tile_count += ntiles;
    }
  }
  plan->n_visible_pairs = vis;
  // Longest-processing-time-first order over the key tiles each row tile visits.
  const int nt = static_cast<int>(plan->tiles.size());
  plan->order.resize(nt);
  std::iota(plan->order.begin(), plan->order.end(), 0);
  std::vector<int64_t> cost(nt);
  for (int i = 0; i < nt; ++i) {
    const TileDesc& td = plan->tiles[i];
    cost[i] = (int64_t(td.kv_end) - td.kv_lo + kKeysPerTile - 1) / kKeysPerTile +
              (int64_t(td.br_hi) - td.br_lo + kKeysPerTile - 1) / kKeysPerTile;
  }
  std::stable_sort(plan->order.begin(), plan->order.end(),
                   [&](int a, int b) { return cost[a] > cost[b]; });
  // Forward pairs: tiles 2k and 2k+1 of each document share the document's
  // main key tiles; a pair streams max(main tiles) plus both branch ranges.
  std::vector<std::pair<int32_t, int32_t>> prs;
  std::vector<int64_t> pcost;
  for (int i = 0; i < nt;) {
    const bool two = i + 1 < nt && plan->tiles[i + 1].doc_start == plan->tiles[i].doc_start;
    const TileDesc& ta = plan->tiles[i];
    int64_t c = cost[i];
    if (two) {
      // the pair streams its main key tiles once (see pair_main_tiles)
      const TileDesc& tb = plan->tiles[i + 1];
      const int64_t ma = (int64_t(ta.kv_end) - ta.kv_lo + kKeysPerTile - 1) / kKeysPerTile;
      const int64_t mb = (int64_t(tb.kv_end) - tb.kv_lo + kKeysPerTile - 1) / kKeysPerTile;
      c = cost[i] + cost[i + 1] - ma - mb + pair_main_tiles(ta, tb);
    }
    prs.emplace_back(i, two ? i + 1 : -1);
    pcost.push_back(c);
    i += two ? 2 : 1;
  }
  std::vector<int> pidx(prs.size());
  std::iota(pidx.begin(), pidx.end(), 0);
  std::stable_sort(pidx.begin(), pidx.end(), [&](int a, int b) { return pcost[a] > pcost[b]; });
  plan->pairs.clear();
  for (int k : pidx) {
    plan->pairs.push_back(prs[k].first);
    plan->pairs.push_back(prs[k].second);
  }
}

void build_kv_plan(const ba_problem* p, Plan* plan) {
  plan->kv_items.clear();
  plan->n_kv_pairs = 0;
  const int32_t* cu = p->cu_seqlens_h;
  const int nt = static_cast<int>(plan->tiles.size());
  int t = 0;
  for (int di = 0; di < p->ndoc; ++di) {
    const int s = cu[di], e = cu[di + 1];
    // row tiles of this document: contiguous, kv_end non-decreasing
    const int t_lo = t;
    while (t < nt && plan->tiles[t].doc_start == s) ++t;
    const int t_hi = t;
    for (int k0 = s; k0 < e; k0 += kKeysPerTile) {
      int lo = t_lo, hi = t_hi;  // first tile with kv_end > k0
      while (lo < hi) {
        const int mid = (lo + hi) / 2;
        if (plan->tiles[mid].kv_end > k0) hi = mid; else lo = mid + 1;
      }
      KvItem it;
      it.key0 = k0;
      it.key_end = std::min(e, k0 + kKeysPerTile);
      it.t_first = lo;
      int t_end = t_hi;
      if (p->window > 0) {
        // rows see this tile only while limit - W + 1 <= key_end - 1
        int a = lo, c = t_hi;  // first tile whose smallest limit is beyond that
        while (a < c) {
          const int mid = (a + c) / 2;
          if (int64_t(plan->tiles[mid].min_limit) - p->window + 1 > int64_t(it.key_end) - 1) c = mid;
          else a = mid + 1;
        }
        t_end = a;
      }
      it.t_count = t_end - lo;
      plan->n_kv_pairs += it.t_count;
      plan->kv_items.push_back(it);
    }
  }
  // Work order: documents longest first, then KV head, then key tiles in
  // order, so the CTAs running at the same time share one (document, KV head)
  // and stream the same query tiles through L2.  Entry = item * Hkv + head.
  plan->kv_order.clear();
  std::vector<int> docs(p->ndoc);
  std::iota(docs.begin(), docs.end(), 0);
  std::stable_sort(docs.begin(), docs.end(), [&](int a, int b) {
    return (cu[a + 1] - cu[a]) > (cu[b + 1] - cu[b]);
  });
  std::vector<int> first_item(p->ndoc + 1, 0);
  {
    int k = 0;
    for (int di = 0; di < p->ndoc; ++di) {
      first_item[di] = k;
      k += (cu[di + 1] - cu[di] + kKeysPerTile - 1) / kKeysPerTile;
    }
    first_item[p->ndoc] = k;
  }
  for (int di : docs)
    for (int g = 0; g < p->Hkv; ++g)
      for (int k = first_item[di]; k < first_item[di + 1]; ++k)
        plan->kv_order.push_back(k * p->Hkv + g);
}

WorkspaceLayout workspace_layout(const ba_problem* p, const Plan& plan, int which) {
  // Layout: counters | tiles | order | chunks | pairs | kv items | kv order |
  // rows | backward buffers.  Everything in [tiles_off, rows_off) comes from
  // the host plan (one upload image); the row table is scattered on the
  // device; the rest is written by the kernels.
  WorkspaceLayout w;
  const size_t nt = plan.tiles.size();
  w.n_slots = int64_t(nt) * kRowsPerTile;
  size_t off = 0;
  w.counters_off = off;
  off = align_up(off + 4 * sizeof(uint32_t), 256);
  w.tiles_off = off;
  off = align_up(off + nt * sizeof(TileDesc), 256);
  w.order_off = off;
  off = align_up(off + nt * sizeof(int32_t), 256);
  w.chunks_off = off;
  off = align_up(off + plan.chunks_dev.size() * sizeof(ChunkDev), 256);
  w.pairs_off = off;
  off = align_up(off + plan.pairs.size() * sizeof(int32_t), 256);
  w.kv_items_off = off;
  off = align_up(off + plan.kv_items.size() * sizeof(KvItem), 256);
  w.kv_order_off = off;
  off = align_up(off + plan.kv_order.size() * sizeof(int32_t), 256);
  w.rows_off = off;
  off = align_up(off + size_t(w.n_slots) * sizeof(int32_t), 256);
  if (which == BA_WS_BWD) {
    const size_t rows = size_t(p->S) + size_t(p->Nb) * (p->Nb > 0 ? p->B : 0);
    const size_t slots = size_t(w.n_slots);
    w.qg_off = off;
    off = align_up(off + slots * p->Hq * p->d * 2, 1024);
    w.dog_off = off;
    off = align_up(off + slots * p->Hq * p->d * 2, 1024);
    w.ls_off = off;
    off = align_up(off + slots * p->Hq * sizeof(float), 256);
    w.ds_off = off;
    off = align_up(off + slots * p->Hq * sizeof(float), 256);
    w.meta_off = off;
    off = align_up(off + slots * sizeof(SlotMeta), 256);
    w.lims_off = off;
    off = align_up(off + slots * sizeof(int32_t), 256);
    w.drow_off = off;
    off = align_up(off + rows * p->Hq * sizeof(float), 256);
  }
  w.total = off;
  return w;
}

void build_image(const Plan& plan, const WorkspaceLayout& w, std::vector<uint8_t>* image) {
  image->assign(w.rows_off - w.tiles_off, 0);
  uint8_t* base = image->data() - w.tiles_off;  // so that base + x_off addresses region x
  auto put = [&](size_t off, const void* src, size_t bytes) {
    if (bytes) std::memcpy(base + off, src, bytes);
  };
  put(w.tiles_off, plan.tiles.data(), plan.tiles.size() * sizeof(TileDesc));
  put(w.order_off, plan.order.data(), plan.order.size() * sizeof(int32_t));
  put(w.chunks_off, plan.chunks_dev.data(), plan.chunks_dev.size() * sizeof(ChunkDev));
  put(w.pairs_off, plan.pairs.data(), plan.pairs.size() * sizeof(int32_t));
  put(w.kv_items_off, plan.kv_items.data(), plan.kv_items.size() * sizeof(KvItem));
  put(w.kv_order_off, plan.kv_order.data(), plan.kv_order.size() * sizeof(int32_t));
}

}  // namespace ba
