// extern "C" entry points of libba_b200.so (declared in include/ba.h).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/ba.h"
#include "kernels.h"
#include "plan.h"

namespace ba {

// Device error word (bounded waits that expired).  Kernels get its address
// as an argument; host code reads it through cudaGetSymbolAddress.
__device__ uint32_t g_error_word;

namespace {

constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at B200 clocks

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  uint32_t* err = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[64];
EncodeTiledFn g_encode = nullptr;

ba_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    if (cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BA_ERR_CUDA;
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return BA_ERR_UNSUPPORTED;  // built for sm_100a only
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return BA_ERR_CUDA;
    di.err = static_cast<uint32_t*>(p);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return BA_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    di.ready = true;
  }
  *out = di;
  return BA_OK;
}

// 2-D bf16 tensor map over a [rows, cols] row-major matrix, box [box_rows, 64]
// with 128-byte swizzle.
ba_status encode_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
  if (rows < 1) rows = 1;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BA_OK : BA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

float scale_of(const ba_problem* p) {
  return p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->d));
}

// Uploads the plan into the workspace and scatters the row table.
ba_status stage_plan(const ba_problem* p, const Plan& plan, const WorkspaceLayout& w,
                     cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  const size_t nt = plan.tiles.size();
  if (nt == 0) return BA_OK;
  if (cudaMemcpyAsync(ws + w.tiles_off, plan.tiles.data(), nt * sizeof(TileDesc),
                      cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(ws + w.order_off, plan.order.data(), nt * sizeof(int32_t),
                      cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(ws + w.chunks_off, plan.chunks_dev.data(),
                      plan.chunks_dev.size() * sizeof(ChunkDev), cudaMemcpyHostToDevice,
                      st) != cudaSuccess ||
      cudaMemsetAsync(ws + w.rows_off, 0xFF, size_t(w.n_slots) * sizeof(int32_t), st) !=
          cudaSuccess)
    return BA_ERR_CUDA;
  if (launch_plan_rows(p->cu_seqlens_d, p->ndoc, p->anchors_d, p->S, p->Nb, plan.B, p->R,
                       reinterpret_cast<const ChunkDev*>(ws + w.chunks_off),
                       reinterpret_cast<int32_t*>(ws + w.rows_off), w.n_slots,
                       st) != cudaSuccess)
    return BA_ERR_CUDA;
  return BA_OK;
}

ba_status check_workspace(const ba_problem* p, const WorkspaceLayout& w) {
  if (!p->workspace || (reinterpret_cast<uintptr_t>(p->workspace) & 255u) != 0)
    return BA_ERR_WORKSPACE;
  if (p->workspace_bytes < w.total) return BA_ERR_WORKSPACE;
  return BA_OK;
}

ba_status run_fwd(const ba_problem* p, bool fused, float* o_part, void* o, void* ob, float* lse,
                  cudaStream_t st) {
  ba_status s = validate(p, true);
  if (s != BA_OK) return s;
  if (!lse || !aligned16(lse)) return BA_ERR_INVALID_ARG;
  if (fused) {
    if (!o || !aligned16(o) || (p->Nb > 0 && (!ob || !aligned16(ob)))) return BA_ERR_INVALID_ARG;
  } else if (!o_part || !aligned16(o_part)) {
    return BA_ERR_INVALID_ARG;
  }
  DeviceInfo di;
  if ((s = device_info(&di)) != BA_OK) return s;
  Plan plan;
  build_plan(p, &plan);
  const WorkspaceLayout w = workspace_layout(p, plan, BA_WS_FWD);
  if ((s = check_workspace(p, w)) != BA_OK) return s;
  if ((s = stage_plan(p, plan, w, st)) != BA_OK) return s;

  const int64_t nbr_rows = int64_t(p->Nb) * plan.B;
  const int64_t rows = int64_t(p->S) + nbr_rows;
  FwdMaps maps;
  const void* qb = p->Nb > 0 ? p->qb : p->q;
  const void* kb = p->Nb > 0 ? p->kb : p->k;
  const void* vb = p->Nb > 0 ? p->vb : p->v;
  const int64_t nb_rows_map = p->Nb > 0 ? nbr_rows : p->S;
  if (encode_2d(&maps.q, p->q, p->S, int64_t(p->Hq) * p->d, 1) != BA_OK ||
      encode_2d(&maps.qb, qb, nb_rows_map, int64_t(p->Hq) * p->d, 1) != BA_OK ||
      encode_2d(&maps.k, p->k, p->S, int64_t(p->Hkv) * p->d, 128) != BA_OK ||
      encode_2d(&maps.v, p->v, p->S, int64_t(p->Hkv) * p->d, 128) != BA_OK ||
      encode_2d(&maps.kb, kb, nb_rows_map, int64_t(p->Hkv) * p->d, 128) != BA_OK ||
      encode_2d(&maps.vb, vb, nb_rows_map, int64_t(p->Hkv) * p->d, 128) != BA_OK)
    return BA_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.anchors = p->anchors_d;
  a.row_table = reinterpret_cast<const int32_t*>(ws + w.rows_off);
  a.tiles = reinterpret_cast<const TileDesc*>(ws + w.tiles_off);
  a.order = reinterpret_cast<const int32_t*>(ws + w.order_off);
  a.S = p->S;
  a.Nb = p->Nb;
  a.B = plan.B > 0 ? plan.B : 1;
  a.mode = p->mode;
  a.Hq = p->Hq;
  a.G = p->Hq / p->Hkv;
  a.d = p->d;
  const int64_t items = int64_t(plan.tiles.size()) * p->Hq;
  if (items > 0x7fffffff) return BA_ERR_UNSUPPORTED;
  a.n_items = static_cast<int>(items);
  a.scale_log2 = scale_of(p) * 1.4426950408889634f;
  a.with_branch = fused && p->Nb > 0 ? 1 : 0;
  a.out_bf16 = fused ? 1 : 0;
  a.o_part = o_part;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.ob = static_cast<__nv_bfloat16*>(ob);
  a.lse = lse;
  a.lse_ld = rows;
  a.err = di.err;
  a.wait_limit = kWaitLimitCycles;
  if (launch_fwd(maps, a, di.num_sms, st) != cudaSuccess) return BA_ERR_CUDA;
  return BA_OK;
}

}  // namespace
}  // namespace ba

using namespace ba;

extern "C" {

size_t ba_workspace_size(const ba_problem* p, int which) {
  if (validate(p, false) != BA_OK) return 0;
  if (which != BA_WS_FWD && which != BA_WS_BWD) return 0;
  Plan plan;
  build_plan(p, &plan);
  return workspace_layout(p, plan, which).total;
}

ba_status ba_plan_stats(const ba_problem* p, int64_t* n_row_tiles, int64_t* n_tile_pairs,
                        int64_t* n_visible_pairs) {
  ba_status s = validate(p, false);
  if (s != BA_OK) return s;
  Plan plan;
  build_plan(p, &plan);
  if (n_row_tiles) *n_row_tiles = static_cast<int64_t>(plan.tiles.size());
  if (n_tile_pairs) *n_tile_pairs = plan.n_tile_pairs;
  if (n_visible_pairs) *n_visible_pairs = plan.n_visible_pairs;
  return BA_OK;
}

ba_status ba_main_fwd(const ba_problem* p, float* o_part, float* lse_part, ba_stream_t stream) {
  return run_fwd(p, false, o_part, nullptr, nullptr, lse_part, reinterpret_cast<cudaStream_t>(stream));
}

ba_status ba_fused_fwd(const ba_problem* p, void* o, void* ob, float* lse, ba_stream_t stream) {
  return run_fwd(p, true, nullptr, o, ob, lse, reinterpret_cast<cudaStream_t>(stream));
}

ba_status ba_branch_fwd(const ba_problem* p, float* o_part, float* lse_part, ba_stream_t stream) {
  ba_status s = validate(p, true);
  if (s != BA_OK) return s;
  if (p->Nb == 0) return BA_OK;
  if (!o_part || !lse_part || !aligned16(o_part) || !aligned16(lse_part)) return BA_ERR_INVALID_ARG;
  DeviceInfo di;
  if ((s = device_info(&di)) != BA_OK) return s;
  if (launch_branch_fwd(static_cast<const __nv_bfloat16*>(p->qb),
                        static_cast<const __nv_bfloat16*>(p->kb),
                        static_cast<const __nv_bfloat16*>(p->vb), p->Nb, p->B, p->mode, p->Hq,
                        p->Hkv, p->d, scale_of(p), o_part, lse_part,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BA_ERR_CUDA;
  return BA_OK;
}

ba_status ba_lse_merge(int nparts, int rows, int H, int d, const float* const* o_parts,
                       const float* const* lse_parts, const int64_t* lse_ld, void* o_out,
                       float* lse_out, int64_t lse_out_ld, ba_stream_t stream) {
  if (nparts < 1 || nparts > 16 || rows < 0 || H < 1) return BA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return BA_ERR_UNSUPPORTED;
  if (!o_parts || !lse_parts || !lse_ld || !o_out || !lse_out) return BA_ERR_INVALID_ARG;
  if (!aligned16(o_out) || lse_out_ld < rows) return BA_ERR_INVALID_ARG;
  MergeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.nparts = nparts;
  a.rows = rows;
  a.H = H;
  a.d = d;
  for (int i = 0; i < nparts; ++i) {
    if (!o_parts[i] || !lse_parts[i] || !aligned16(o_parts[i]) || lse_ld[i] < rows)
      return BA_ERR_INVALID_ARG;
    a.o[i] = o_parts[i];
    a.lse[i] = lse_parts[i];
    a.lse_ld[i] = lse_ld[i];
  }
  a.o_out = static_cast<__nv_bfloat16*>(o_out);
  a.lse_out = lse_out;
  a.lse_out_ld = lse_out_ld;
  if (rows == 0) return BA_OK;
  DeviceInfo di;
  ba_status s = device_info(&di);
  if (s != BA_OK) return s;
  if (launch_lse_merge(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BA_ERR_CUDA;
  return BA_OK;
}

ba_status ba_bwd(const ba_problem* p, const void* o, const void* ob, const float* lse,
                 const void* dout, const void* doutb, void* dq, void* dk, void* dv, void* dqb,
                 void* dkb, void* dvb, ba_stream_t stream);

const char* ba_status_string(ba_status s) {
  switch (s) {
    case BA_OK: return "ok";
    case BA_ERR_INVALID_ARG: return "invalid argument";
    case BA_ERR_UNSUPPORTED: return "unsupported configuration";
    case BA_ERR_CUDA: return "CUDA runtime error";
    case BA_ERR_TIMEOUT: return "device-side bounded wait expired";
    case BA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

ba_status ba_sync_status(ba_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return BA_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    return BA_ERR_TIMEOUT;
  }
  return BA_OK;
}

}  // extern "C"
