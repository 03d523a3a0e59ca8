// Plain structs shared by the host planner and the device kernels.
#pragma once
#include <cstdint>

namespace ba {

// One row tile: up to 128 query rows of one document, ordered by their last
// visible main key ("limit"); ties put the main row first, then the branch
// rows anchored there (branch-major, depth-minor).  The tile belongs to the
// virtual rank whose zigzag chunk holds its first row.
struct TileDesc {
  int32_t row_base;   // first slot in the row table (tile index * 128)
  int32_t n_rows;     // valid rows, 1..128 (slots beyond hold -1)
  int32_t doc_start;  // first main key of the tile's document
  int32_t kv_end;     // one past the largest limit in the tile
  int32_t min_limit;  // smallest limit in the tile
  int32_t br_lo;      // branch key rows (flattened b*B+u) the tile's branch
  int32_t br_hi;      //   rows can see: [br_lo, br_hi); empty if br_lo >= br_hi
  int32_t rank;       // owning virtual rank
  int32_t kv_lo;      // first main key any row of the tile sees (doc_start
                      //   unless a window cuts the prefix)
  int32_t doc_end;    // one past the last main key of the tile's document
  int32_t pad0, pad1;
};
static_assert(sizeof(TileDesc) == 48, "TileDesc must stay 48 bytes");

// A row segment of the plan (a whole document, or one zigzag chunk of it
// when the plan covers one virtual rank's rows): what the device row scatter
// needs.
struct ChunkDev {
  int32_t c0;        // first main position of the segment
  int32_t b0;        // first branch anchored in the segment
  int32_t slot_base; // row-table slot of merged index 0
  int32_t pad;       // one past the last main position of the segment
};
static_assert(sizeof(ChunkDev) == 16, "ChunkDev must stay 16 bytes");

// One main key tile of the key-stationary dK/dV pass: 128 keys of one
// document and the row tiles (a contiguous range) whose rows can see them.
struct KvItem {
  int32_t key0;     // first key (packed main position), document start + 128 j
  int32_t key_end;  // one past the last key this item owns: min(doc end, key0 + 128)
  int32_t t_first;  // first row tile with a row whose limit >= key0
  int32_t t_count;  // row tiles to visit: [t_first, t_first + t_count)
};
static_assert(sizeof(KvItem) == 16, "KvItem must stay 16 bytes");

// Per row-table slot metadata written by the backward pre-pass.
struct SlotMeta {
  int32_t limit;  // last visible main key (-1 for padding)
  int32_t blo;    // visible branch key rows [blo, bhi) (flattened b*B+u)
  int32_t bhi;
  int32_t row;    // concatenated row index (-1 for padding)
};
static_assert(sizeof(SlotMeta) == 16, "SlotMeta must stay 16 bytes");

}  // namespace ba
