// Launch wrappers and argument blocks of the backward kernels (host side).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tile_desc.h"

namespace ba {

struct PrepArgs {
  const int32_t* row_table;  // [n_slots]
  const int32_t* anchors;
  const __nv_bfloat16 *q, *qb, *o, *ob, *dout, *dob;
  const float* lse;          // [Hq, rows], natural log
  int S, B, mode, Hq;
  int64_t rows, n_slots;
  __nv_bfloat16* qg;         // [n_slots, Hq, d]
  __nv_bfloat16* dog;        // [n_slots, Hq, d]
  float* ls;                 // [Hq, n_slots], -LSE * log2(e) (-inf for padding)
  float* ds;                 // [Hq, n_slots]
  float* drow;               // [Hq, rows]
  SlotMeta* meta;            // [n_slots]
  int32_t* lims;             // [n_slots], meta[].limit on its own (-1 for padding)
};
cudaError_t launch_bwd_prep(const PrepArgs& a, int d, cudaStream_t st);

struct BranchBwdArgs {
  const __nv_bfloat16 *qb, *kb, *vb, *dob;
  const float* lse;   // [Hq, rows]
  const float* drow;  // [Hq, rows]
  const uint64_t* bmask;  // BA_MASK_BITMASK: [Nb*B] words
  const int32_t* cu;      // [ndoc + 1] (one rank's rows: to find a branch's owner)
  const int32_t* anchors; // [Nb]
  int ndoc, R;
  int cp_rank;            // >= 0: only the branches whose anchor virtual rank cp_rank owns
  int S, Nb, B, mode, Hq, Hkv;
  int64_t rows;
  float scale;
  __nv_bfloat16 *dkb, *dvb;
  uint32_t* err;          // device error word
  long long wait_limit;   // bound of the copy wait, in cycles
};
cudaError_t launch_branch_bwd(const BranchBwdArgs& a, int d, cudaStream_t st);

// Query-stationary dQ pass (tcgen05).
struct DqArgs {
  const TileDesc* tiles;
  const int32_t* order;
  const SlotMeta* meta;
  const float* ls;  // [Hq, n_slots], -LSE * log2(e)
  const float* ds;  // [Hq, n_slots]
  const uint64_t* bmask;  // BA_MASK_BITMASK: [Nb*B] words, else unused
  int S, Hq, G, d;
  int mode, window;
  int64_t n_slots;
  int n_items;      // ntiles * Hq
  int with_branch;
  float scale_log2, scale;
  __nv_bfloat16* dq;   // [S, Hq, d]
  __nv_bfloat16* dqb;  // [Nb*B, Hq, d]
  uint32_t* err;
  uint32_t* counter;   // work-item counter, zero at launch
  long long wait_limit;
};
struct DqMaps {
  CUtensorMap qg, dog;  // [n_slots, Hq*d], box 64 x 128
  CUtensorMap k, v;     // [S, Hkv*d], box 64 x 128
  CUtensorMap kb, vb;   // [Nb*B, Hkv*d], box 64 x 128
};
cudaError_t launch_bwd_dq(const DqMaps& m, const DqArgs& a, int num_sms, cudaStream_t st);

// Key-stationary dK/dV pass (tcgen05), main keys.
struct DkdvArgs {
  const KvItem* items;
  const int32_t* order;
  const TileDesc* tiles;
  const int32_t* lims;  // [n_slots]: a row sees main keys <= its limit
  const float* ls;  // [Hq, n_slots], -LSE * log2(e)
  const float* ds;  // [Hq, n_slots]
  int Hq, Hkv, G, d;
  int window;   // main-prefix window (> 0), else none
  int64_t n_slots;
  int n_items;  // n_kv * Hkv
  float scale_log2, scale;
  __nv_bfloat16 *dk, *dv;  // [S, Hkv, d]
  uint32_t* err;
  uint32_t* counter;       // work-item counter, zero at launch
  long long wait_limit;
};
struct DkdvMaps {
  CUtensorMap k, v;      // [S, Hkv*d], box 64 x 128
  CUtensorMap qg, dog;   // [n_slots, Hq*d], box 64 x 128
};
cudaError_t launch_bwd_dkdv(const DkdvMaps& m, const DkdvArgs& a, int num_sms, cudaStream_t st);

}  // namespace ba
