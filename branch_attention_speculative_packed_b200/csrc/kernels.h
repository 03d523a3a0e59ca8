// Launch wrappers of the device kernels (host side).  Every wrapper enqueues
// on `stream` and returns the cudaError_t of the launch.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tile_desc.h"

namespace ba {

// ---------------------------------------------------------------- forward
struct FwdArgs {
  const __nv_bfloat16* q;    // [S, Hq, d]
  const __nv_bfloat16* qb;   // [Nb*B, Hq, d] (q when there are no branches)
  const int32_t* anchors;    // [Nb]
  const int32_t* row_table;  // [ntiles * 128], -1 = padding
  const TileDesc* tiles;     // [ntiles]
  const int32_t* pairs;      // [n_pairs][2] tile indices (second -1: single), longest first
  const uint64_t* bmask;     // BA_MASK_BITMASK: [Nb*B] words (row (b,t) sees branch key u iff bit u)
  int S, Nb, B, mode, Hq, G, d;
  int window;                // main-prefix window (> 0), else none
  int ring;                  // R > 0: one partial per virtual rank's zigzag keys; 0: full rows
  int n_items;               // n_pairs * Hq (* ring when ring > 0)
  float scale_log2;          // softmax scale * log2(e)
  int with_branch;           // also visit the branch key tiles (fused forward)
  int out_bf16;              // 1: bf16 o / ob; 0: fp32 o_part
  float* o_part;             // [rows, Hq, d] (ring: [ring, rows, Hq, d])
  int64_t o_part_stride;     // elements between ring partials of o_part
  int64_t lse_stride;        // elements between ring partials of lse
  __nv_bfloat16* o;          // [S, Hq, d]
  __nv_bfloat16* ob;         // [Nb*B, Hq, d]
  float* lse;                // element (h, r) at lse[h * lse_ld + r]
  int64_t lse_ld;
  uint32_t* err;             // device error word
  uint32_t* counter;         // work-item counter, zero at launch
  long long wait_limit;      // cycles per bounded wait
};

struct FwdMaps {
  CUtensorMap k, v, kb, vb;  // [rows, Hkv*d], box 64 x 128
};

cudaError_t launch_fwd(const FwdMaps& maps, const FwdArgs& a, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- planning
cudaError_t launch_plan_rows(const ChunkDev* segs, int nseg, const int32_t* anchors, int S, int Nb,
                             int B, int32_t* row_table, int64_t n_slots, cudaStream_t stream);

// ---------------------------------------------------------------- branch part / merge
cudaError_t launch_branch_fwd(const __nv_bfloat16* qb, const __nv_bfloat16* kb,
                              const __nv_bfloat16* vb, const uint64_t* bmask, int Nb, int B,
                              int mode, int Hq, int Hkv, int d, float scale, float* o_part,
                              float* lse_part, cudaStream_t stream);

// One thread waits, with the bounded wait every kernel uses, on a barrier no
// one arrives on: it gives up after `limit` cycles and records wait site
// (kernel 4, role 0, site 1) in the device error word.
cudaError_t launch_bounded_wait_probe(uint32_t* err, long long limit, cudaStream_t stream);

struct MergeArgs {
  int nparts, rows, H, d;
  const float* o[16];
  const float* lse[16];
  int64_t lse_ld[16];
  __nv_bfloat16* o_out;
  float* lse_out;
  int64_t lse_out_ld;
};
cudaError_t launch_lse_merge(const MergeArgs& a, cudaStream_t stream);

}  // namespace ba
