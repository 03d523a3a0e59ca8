// Host planner for branch attention: zigzag split into R virtual ranks, row
// tiles, key-tile ranges and the longest-first work order.
//
// Paper: arXiv 2609.07108 §3.2 as described on the rcap.io post: the
// main-sequence part runs on packed zigzag ring attention, whose zigzag split
// balances the triangular causal work across ranks, and the branch-local part
// runs on the rank that holds the branch's anchor.  The chunk rule itself is
// not printed on the pages; the reading taken here is: a document [s, s+L) is
// cut into 2R chunks, chunk k = [s + floor(kL/2R), s + floor((k+1)L/2R)),
// virtual rank r owns chunks r and 2R-1-r, and a branch belongs to the rank
// owning the chunk that holds its anchor.
#pragma once
#include <cstddef>
#include <cstdint>
#include <vector>

#include "../../include/ba.h"
#include "tile_desc.h"

namespace ba {

constexpr int kRowsPerTile = 128;  // query rows per tile (the tcgen05 M)
constexpr int kKeysPerTile = 128;  // keys per key tile (the tcgen05 N of S = QK^T)

struct Chunk {
  int doc, k, rank;
  int c0, c1;   // main positions [c0, c1)
  int b0, b1;   // branches whose anchor lies in [c0, c1)
  int64_t n_rows;
  int tile0, ntiles;  // unused: row tiles are cut per document
};

struct Plan {
  int S = 0, Nb = 0, B = 0, R = 1, ndoc = 0;
  std::vector<Chunk> chunks;       // doc-major, chunk-index minor (= position order)
  std::vector<TileDesc> tiles;     // in position order
  std::vector<int32_t> order;      // tile indices, longest (most key tiles) first
  // Forward work items: two consecutive row tiles of one document (the second
  // -1 when the document has an odd tile left), two int32 per pair, longest first.
  std::vector<int32_t> pairs;
  std::vector<ChunkDev> chunks_dev;
  std::vector<int64_t> rank_pairs; // main (row tile, key tile) pairs per virtual rank
  std::vector<KvItem> kv_items;    // key tiles of the dK/dV pass
  std::vector<int32_t> kv_order;   // work order: kv item * Hkv + KV head
  int64_t n_kv_pairs = 0;          // (key tile, row tile) pairs of the dK/dV pass
  int64_t n_tile_pairs = 0;        // main key tiles visited, per query head
  int64_t n_branch_tile_pairs = 0; // branch key tiles visited (fused forward), per head
  int64_t n_visible_pairs = 0;     // exact visible (row, key) pairs per head
};

// Host-side validation of every argument; `need_tensors` also checks the
// device tensor pointers.  Returns BA_OK or the first error found.
ba_status validate(const ba_problem* p, bool need_tensors);

// Builds the plan from the host copies of cu_seqlens and anchors.
// Precondition: validate(p, ...) == BA_OK.
void build_plan(const ba_problem* p, Plan* plan);

// Main key tiles a forward tile pair streams (the device kernel's rule).
int64_t pair_main_tiles(const TileDesc& a, const TileDesc& b);

// Builds the key-tile list of the dK/dV pass (after build_plan).
void build_kv_plan(const ba_problem* p, Plan* plan);

// Workspace layout shared by the forward and backward paths.
struct WorkspaceLayout {
  size_t counters_off = 0;  // uint32 work-item counters (forward, dQ pass, dK/dV pass)
  size_t tiles_off = 0, order_off = 0, chunks_off = 0, rows_off = 0, pairs_off = 0;
  // backward only
  size_t kv_items_off = 0, kv_order_off = 0;
  size_t qg_off = 0, dog_off = 0;    // Q and dO gathered into slot order, bf16 [slots, Hq, d]
  size_t ls_off = 0, ds_off = 0;     // log2-scaled LSE and D = rowsum(dO*O), fp32 [Hq, slots]
  size_t meta_off = 0;               // SlotMeta [slots]
  size_t lims_off = 0;               // main-key limit per slot, int32 [slots]
  size_t drow_off = 0;               // D in row order, fp32 [Hq, rows]
  size_t total = 0;
  int64_t n_slots = 0;               // row-table entries (ntiles * 128)
};
WorkspaceLayout workspace_layout(const ba_problem* p, const Plan& plan, int which);

// The host bytes of the workspace region [tiles_off, rows_off): tiles, order,
// chunks, pairs and the dK/dV key-tile list, at their layout offsets.  The
// region is the same for the forward and the backward layout.
void build_image(const Plan& plan, const WorkspaceLayout& w, std::vector<uint8_t>* image);

}  // namespace ba
