// extern "C" entry points of libba_b200.so (declared in include/ba.h).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <cmath>
#include <cstring>
#include <list>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <unordered_map>
#include <utility>
#include <vector>

#include "../../include/ba.h"
#include "bwd_kernels.h"
#include "kernels.h"
#include "plan.h"

namespace ba {

// Device error word (bounded waits that expired).  Kernels get its address
// as an argument; host code reads it through cudaGetSymbolAddress.
__device__ uint32_t g_error_word;

namespace {

constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at B200 clocks
// The limit every launch passes to its bounded waits (ba_set_wait_limit).
std::atomic<long long> g_wait_limit{kWaitLimitCycles};

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
  // bf16 matrix [rows, cols], box [box_rows, 64 columns = 128 bytes], 128-byte swizzle
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

// ------------------------------------------------------------------ profiling
struct ProfRecord {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;

// Brackets one kernel launch with events on `st` while profiling is enabled.
struct ProfScope {
  ProfRecord rec{nullptr, nullptr, nullptr};
  cudaStream_t st;
  ProfScope(const char* name, cudaStream_t s) : st(s) {
    if (!g_prof_on) return;
    if (cudaEventCreate(&rec.start) != cudaSuccess) return;
    if (cudaEventCreate(&rec.stop) != cudaSuccess) {
      cudaEventDestroy(rec.start);
      return;
    }
    rec.name = name;
    cudaEventRecord(rec.start, st);
  }
  ~ProfScope() {
    if (!rec.name) return;
    cudaEventRecord(rec.stop, st);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back(rec);
  }
};

float scale_of(const ba_problem* p) {
  return p->scale > 0.f ? p->scale : 1.0f / std::sqrt(static_cast<float>(p->d));
}

// ------------------------------------------------------------------ plan cache
// A host plan depends only on the problem's sizes and on the contents of its
// host cu_seqlens and anchors.  Plans are kept, least recently used first
// out, so repeated calls on one packing (every training step, forward and
// backward) plan once.  Each entry also holds the bytes the workspace needs
// from the host, in pageable memory and, once a device call has used it, in a
// page-locked copy so the upload is a plain asynchronous copy.
constexpr size_t kPlanCacheCapacity = 16;

struct CachedPlan {
  Plan plan;
  WorkspaceLayout ws_fwd, ws_bwd;
  std::vector<uint8_t> image;  // workspace bytes [tiles_off, rows_off), same for both layouts
  double build_ms = 0.0;       // host time it took to build this entry
  std::mutex mu;               // guards the fields below
  void* pinned = nullptr;      // page-locked copy of `image`
  bool pinned_failed = false;
  // one event per stream that uploaded from `pinned`: its last upload there
  std::vector<std::pair<cudaStream_t, cudaEvent_t>> uploads;

  ~CachedPlan() {
    // The page-locked copy goes only after every upload from it has finished.
    for (auto& u : uploads) {
      cudaEventSynchronize(u.second);
      cudaEventDestroy(u.second);
    }
    if (pinned) cudaFreeHost(pinned);
  }
};

struct PlanCache {
  std::mutex mu;
  std::list<std::pair<std::string, std::shared_ptr<CachedPlan>>> lru;  // most recent first
  std::unordered_map<std::string, decltype(lru)::iterator> index;
  int64_t hits = 0, misses = 0;
};

// Never destroyed: entries may hold CUDA resources, which must not be
// released from a static destructor after the runtime has shut down.
PlanCache& plan_cache() {
  static PlanCache* c = new PlanCache;
  return *c;
}

std::string plan_key(const ba_problem* p) {
  const int32_t dims[] = {p->S, p->ndoc, p->Hq, p->Hkv, p->d, p->Nb, p->Nb > 0 ? p->B : 0,
                          p->mode, p->R, p->window > 0 ? p->window : 0, p->cp_select,
                          p->cp_select ? p->cp_rank : 0};
  std::string key(reinterpret_cast<const char*>(dims), sizeof(dims));
  key.append(reinterpret_cast<const char*>(p->cu_seqlens_h), size_t(p->ndoc + 1) * sizeof(int32_t));
  if (p->Nb > 0) key.append(reinterpret_cast<const char*>(p->anchors_h), size_t(p->Nb) * sizeof(int32_t));
  if (p->Nb > 0 && p->mode == BA_MASK_BITMASK)
    key.append(reinterpret_cast<const char*>(p->branch_mask_h), size_t(p->Nb) * p->B * sizeof(uint64_t));
  return key;
}

// The cached plan of a validated problem (built on a miss).  Without
// `may_evict` a miss never drops older entries (dropping one may free its
// page-locked copy); the next call that may evict trims the cache.
std::shared_ptr<CachedPlan> get_plan(const ba_problem* p, bool may_evict = true) {
  PlanCache& c = plan_cache();
  std::string key = plan_key(p);
  {
    std::lock_guard<std::mutex> lk(c.mu);
    auto it = c.index.find(key);
    if (it != c.index.end()) {
      c.lru.splice(c.lru.begin(), c.lru, it->second);
      ++c.hits;
      return it->second->second;
    }
  }
  auto e = std::make_shared<CachedPlan>();
  const auto t0 = std::chrono::steady_clock::now();
  build_plan(p, &e->plan);
  build_kv_plan(p, &e->plan);
  e->ws_fwd = workspace_layout(p, e->plan, BA_WS_FWD);
  e->ws_bwd = workspace_layout(p, e->plan, BA_WS_BWD);
  build_image(e->plan, e->ws_fwd, &e->image);
  e->build_ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
  std::vector<std::shared_ptr<CachedPlan>> evicted;  // released after the lock
  std::lock_guard<std::mutex> lk(c.mu);
  ++c.misses;
  auto it = c.index.find(key);
  if (it != c.index.end()) return it->second->second;  // built concurrently by another caller
  c.lru.emplace_front(key, e);
  c.index.emplace(std::move(key), c.lru.begin());
  while (may_evict && c.lru.size() > kPlanCacheCapacity) {
    c.index.erase(c.lru.back().first);
    evicted.push_back(std::move(c.lru.back().second));
    c.lru.pop_back();
  }
  return e;
}

// Uploads the plan into the workspace and scatters the row table.  With
// `pinned_ok` the bytes come from the entry's page-locked copy (made on first
// use); otherwise straight from pageable memory.
ba_status stage_plan(const ba_problem* p, CachedPlan& e, const WorkspaceLayout& w, void* workspace,
                     bool pinned_ok, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (e.plan.tiles.empty()) return BA_OK;
  const size_t n = e.image.size();
  const void* src = e.image.data();
  cudaEvent_t* done = nullptr;
  std::unique_lock<std::mutex> lk(e.mu, std::defer_lock);
  if (pinned_ok) {
    lk.lock();
    if (!e.pinned && !e.pinned_failed) {
      void* h = nullptr;
      if (cudaHostAlloc(&h, n, cudaHostAllocPortable) == cudaSuccess && h) {
        std::memcpy(h, e.image.data(), n);
        e.pinned = h;
      } else {
        cudaGetLastError();  // not sticky; fall back to the pageable copy
        e.pinned_failed = true;
      }
    }
    if (e.pinned) {
      src = e.pinned;
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone) {
        for (auto& u : e.uploads)
          if (u.first == st) done = &u.second;
        if (!done) {
          cudaEvent_t ev;
          if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return BA_ERR_CUDA;
          e.uploads.emplace_back(st, ev);
          done = &e.uploads.back().second;
        }
      }
    }
  }
  if (cudaMemcpyAsync(ws + w.tiles_off, src, n, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BA_ERR_CUDA;
  if (done && cudaEventRecord(*done, st) != cudaSuccess) return BA_ERR_CUDA;
  if (lk.owns_lock()) lk.unlock();
  if (cudaMemsetAsync(ws + w.rows_off, 0xFF, size_t(w.n_slots) * sizeof(int32_t), st) != cudaSuccess ||
      cudaMemsetAsync(ws + w.counters_off, 0, 4 * sizeof(uint32_t), st) != cudaSuccess)
    return BA_ERR_CUDA;
  ProfScope prof("plan_rows", st);
  if (launch_plan_rows(reinterpret_cast<const ChunkDev*>(ws + w.chunks_off),
                       static_cast<int>(e.plan.chunks_dev.size()), p->anchors_d, p->S, p->Nb,
                       e.plan.B, reinterpret_cast<int32_t*>(ws + w.rows_off), w.n_slots,
                       st) != cudaSuccess)
    return BA_ERR_CUDA;
  return BA_OK;
}

ba_status check_workspace(const void* ws, size_t bytes, const WorkspaceLayout& w) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BA_ERR_WORKSPACE;
  if (bytes < w.total) return BA_ERR_WORKSPACE;
  return BA_OK;
}

// The forward (fused or main component only).  `scratch` / `scratch_bytes`
// replace the caller's workspace when set (the no-allocation entry point);
// there a plan too large for the scratch is refused with `too_big` before
// anything is enqueued, and the plan is uploaded from pageable memory.
ba_status run_fwd(const ba_problem* p, bool fused, float* o_part, void* o, void* ob, float* lse,
                  cudaStream_t st, void* scratch = nullptr, size_t scratch_bytes = 0,
                  ba_status too_big = BA_ERR_WORKSPACE, bool ring = false) {
  ba_status s = validate(p, true);
  if (s != BA_OK) return s;
  if (!lse || !aligned16(lse)) return BA_ERR_INVALID_ARG;
  if (fused) {
    if (!o || !aligned16(o) || (p->Nb > 0 && (!ob || !aligned16(ob)))) return BA_ERR_INVALID_ARG;
  } else if (!o_part || !aligned16(o_part)) {
    return BA_ERR_INVALID_ARG;
  }
  const std::shared_ptr<CachedPlan> cp = get_plan(p, scratch == nullptr);
  const Plan& plan = cp->plan;
  const WorkspaceLayout& w = cp->ws_fwd;
  void* ws_ptr = scratch ? scratch : p->workspace;
  if (scratch) {
    if (w.total > scratch_bytes) return too_big;
  } else if ((s = check_workspace(p->workspace, p->workspace_bytes, w)) != BA_OK) {
    return s;
  }
  const int64_t items = int64_t(plan.pairs.size() / 2) * p->Hq * (ring ? p->R : 1);
  if (items > 0x7fffffff) return BA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((s = device_info(&di)) != BA_OK) return s;
  if ((s = stage_plan(p, *cp, w, ws_ptr, scratch == nullptr, st)) != BA_OK) return s;

  const int64_t nbr_rows = int64_t(p->Nb) * plan.B;
  const int64_t rows = int64_t(p->S) + nbr_rows;
  FwdMaps maps;
  const void* qb = p->Nb > 0 ? p->qb : p->q;
  const void* kb = p->Nb > 0 ? p->kb : p->k;
  const void* vb = p->Nb > 0 ? p->vb : p->v;
  const int64_t nb_rows_map = p->Nb > 0 ? nbr_rows : p->S;
  if (encode_2d(&maps.k, p->k, p->S, int64_t(p->Hkv) * p->d, 128) != BA_OK ||
      encode_2d(&maps.v, p->v, p->S, int64_t(p->Hkv) * p->d, 128) != BA_OK ||
      encode_2d(&maps.kb, kb, nb_rows_map, int64_t(p->Hkv) * p->d, 128) != BA_OK ||
      encode_2d(&maps.vb, vb, nb_rows_map, int64_t(p->Hkv) * p->d, 128) != BA_OK)
    return BA_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(ws_ptr);
  FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = static_cast<const __nv_bfloat16*>(p->q);
  a.qb = static_cast<const __nv_bfloat16*>(qb);
  a.anchors = p->anchors_d;
  a.row_table = reinterpret_cast<const int32_t*>(ws + w.rows_off);
  a.tiles = reinterpret_cast<const TileDesc*>(ws + w.tiles_off);
  a.pairs = reinterpret_cast<const int32_t*>(ws + w.pairs_off);
  a.bmask = (p->mode == BA_MASK_BITMASK && p->Nb > 0) ? p->branch_mask_d : nullptr;
  a.S = p->S;
  a.Nb = p->Nb;
  a.B = plan.B > 0 ? plan.B : 1;
  a.mode = p->mode;
  a.Hq = p->Hq;
  a.G = p->Hq / p->Hkv;
  a.d = p->d;
  a.window = p->window > 0 ? p->window : 0;
  a.ring = ring ? p->R : 0;
  a.n_items = static_cast<int>(items);
  a.scale_log2 = scale_of(p) * 1.4426950408889634f;
  a.with_branch = fused && p->Nb > 0 ? 1 : 0;
  a.out_bf16 = fused ? 1 : 0;
  a.o_part = o_part;
  a.o_part_stride = ring ? rows * p->Hq * p->d : 0;
  a.lse_stride = ring ? rows * p->Hq : 0;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.ob = static_cast<__nv_bfloat16*>(ob);
  a.lse = lse;
  a.lse_ld = rows;
  a.err = di.err;
  a.counter = reinterpret_cast<uint32_t*>(ws + w.counters_off);
  a.wait_limit = g_wait_limit.load();
  ProfScope prof(fused ? "fused_fwd" : ring ? "main_fwd_ring" : "main_fwd", st);
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
  const std::shared_ptr<CachedPlan> cp = get_plan(p);
  return (which == BA_WS_FWD ? cp->ws_fwd : cp->ws_bwd).total;
}

ba_status ba_plan_stats(const ba_problem* p, int64_t* n_row_tiles, int64_t* n_tile_pairs,
                        int64_t* n_visible_pairs) {
  ba_status s = validate(p, false);
  if (s != BA_OK) return s;
  const std::shared_ptr<CachedPlan> cp = get_plan(p);
  if (n_row_tiles) *n_row_tiles = static_cast<int64_t>(cp->plan.tiles.size());
  if (n_tile_pairs) *n_tile_pairs = cp->plan.n_tile_pairs;
  if (n_visible_pairs) *n_visible_pairs = cp->plan.n_visible_pairs;
  return BA_OK;
}

int ba_plan_rank_work(const ba_problem* p, int64_t* pairs, int cap) {
  ba_status s = validate(p, false);
  if (s != BA_OK) return s;
  const std::shared_ptr<CachedPlan> cp = get_plan(p);
  for (int r = 0; r < cap && r < p->R; ++r)
    if (pairs) pairs[r] = cp->plan.rank_pairs[r];
  return p->R;
}

int64_t ba_plan_fwd_pairs(const ba_problem* p, int32_t* tiles, int64_t cap) {
  ba_status s = validate(p, false);
  if (s != BA_OK) return s;
  const std::shared_ptr<CachedPlan> cp = get_plan(p);
  const Plan& plan = cp->plan;
  const int64_t n = static_cast<int64_t>(plan.pairs.size() / 2);
  for (int64_t i = 0; tiles && i < cap && i < n; ++i) {
    tiles[2 * i] = plan.pairs[2 * i];
    tiles[2 * i + 1] = plan.pairs[2 * i + 1];
  }
  return n;
}

ba_status ba_plan_prepare(const ba_problem* p, double* build_ms) {
  ba_status s = validate(p, false);
  if (s != BA_OK) return s;
  const std::shared_ptr<CachedPlan> cp = get_plan(p);
  if (build_ms) *build_ms = cp->build_ms;
  return BA_OK;
}

void ba_clear_cache(void) {
  PlanCache& c = plan_cache();
  std::list<std::pair<std::string, std::shared_ptr<CachedPlan>>> dropped;
  {
    std::lock_guard<std::mutex> lk(c.mu);
    c.index.clear();
    dropped.swap(c.lru);
  }
  // entries still used by a call in progress go when that call returns
}

void ba_plan_cache_stats(int64_t* entries, int64_t* hits, int64_t* misses) {
  PlanCache& c = plan_cache();
  std::lock_guard<std::mutex> lk(c.mu);
  if (entries) *entries = static_cast<int64_t>(c.lru.size());
  if (hits) *hits = c.hits;
  if (misses) *misses = c.misses;
}

ba_status ba_main_fwd(const ba_problem* p, float* o_part, float* lse_part, ba_stream_t stream) {
  return run_fwd(p, false, o_part, nullptr, nullptr, lse_part, reinterpret_cast<cudaStream_t>(stream));
}

ba_status ba_main_fwd_ring(const ba_problem* p, float* o_parts, float* lse_parts,
                           ba_stream_t stream) {
  return run_fwd(p, false, o_parts, nullptr, nullptr, lse_parts,
                 reinterpret_cast<cudaStream_t>(stream), nullptr, 0, BA_ERR_WORKSPACE, true);
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
  ProfScope prof("branch_fwd", reinterpret_cast<cudaStream_t>(stream));
  if (launch_branch_fwd(static_cast<const __nv_bfloat16*>(p->qb),
                        static_cast<const __nv_bfloat16*>(p->kb),
                        static_cast<const __nv_bfloat16*>(p->vb),
                        p->mode == BA_MASK_BITMASK ? p->branch_mask_d : nullptr, p->Nb, p->B, p->mode, p->Hq,
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
  ProfScope prof("lse_merge", reinterpret_cast<cudaStream_t>(stream));
  if (launch_lse_merge(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BA_ERR_CUDA;
  return BA_OK;
}

ba_status ba_bwd(const ba_problem* p, const void* o, const void* ob, const float* lse,
                 const void* dout, const void* doutb, void* dq, void* dk, void* dv, void* dqb,
                 void* dkb, void* dvb, ba_stream_t stream) {
  ba_status s = validate(p, true);
  if (s != BA_OK) return s;
  const bool nb = p->Nb > 0;
  const void* need[] = {o, lse, dout, dq, dk, dv};
  for (const void* x : need)
    if (!x || !aligned16(x)) return BA_ERR_INVALID_ARG;
  if (nb) {
    const void* needb[] = {ob, doutb, dqb, dkb, dvb};
    for (const void* x : needb)
      if (!x || !aligned16(x)) return BA_ERR_INVALID_ARG;
  }
  DeviceInfo di;
  if ((s = device_info(&di)) != BA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const std::shared_ptr<CachedPlan> cp = get_plan(p);
  const Plan& plan = cp->plan;
  const WorkspaceLayout& w = cp->ws_bwd;
  if ((s = check_workspace(p->workspace, p->workspace_bytes, w)) != BA_OK) return s;
  const size_t nkv = plan.kv_items.size();
  const int64_t items_q = int64_t(plan.tiles.size()) * p->Hq;
  const int64_t items_kv = int64_t(nkv) * p->Hkv;
  if (items_q > 0x7fffffff || items_kv > 0x7fffffff) return BA_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  if ((s = stage_plan(p, *cp, w, p->workspace, true, st)) != BA_OK) return s;
  const int64_t rows = int64_t(p->S) + int64_t(p->Nb) * plan.B;
  const float scale = scale_of(p);
  const int G = p->Hq / p->Hkv;

  // 1. pre-pass
  PrepArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  pa.row_table = reinterpret_cast<const int32_t*>(ws + w.rows_off);
  pa.anchors = p->anchors_d;
  pa.q = static_cast<const __nv_bfloat16*>(p->q);
  pa.qb = static_cast<const __nv_bfloat16*>(nb ? p->qb : p->q);
  pa.o = static_cast<const __nv_bfloat16*>(o);
  pa.ob = static_cast<const __nv_bfloat16*>(nb ? ob : o);
  pa.dout = static_cast<const __nv_bfloat16*>(dout);
  pa.dob = static_cast<const __nv_bfloat16*>(nb ? doutb : dout);
  pa.lse = lse;
  pa.S = p->S;
  pa.B = plan.B > 0 ? plan.B : 1;
  pa.mode = p->mode;
  pa.Hq = p->Hq;
  pa.rows = rows;
  pa.n_slots = w.n_slots;
  pa.qg = reinterpret_cast<__nv_bfloat16*>(ws + w.qg_off);
  pa.dog = reinterpret_cast<__nv_bfloat16*>(ws + w.dog_off);
  pa.ls = reinterpret_cast<float*>(ws + w.ls_off);
  pa.ds = reinterpret_cast<float*>(ws + w.ds_off);
  pa.drow = reinterpret_cast<float*>(ws + w.drow_off);
  pa.meta = reinterpret_cast<SlotMeta*>(ws + w.meta_off);
  pa.lims = reinterpret_cast<int32_t*>(ws + w.lims_off);
  const uint64_t* bmask = (nb && p->mode == BA_MASK_BITMASK) ? p->branch_mask_d : nullptr;
  {
    ProfScope prof("bwd_prep", st);
    if (launch_bwd_prep(pa, p->d, st) != cudaSuccess) return BA_ERR_CUDA;
  }

  // tensor maps
  const int64_t qcols = int64_t(p->Hq) * p->d, kcols = int64_t(p->Hkv) * p->d;
  const int64_t nb_rows_map = nb ? int64_t(p->Nb) * plan.B : p->S;
  DqMaps dm;
  DkdvMaps km;
  if (encode_2d(&dm.qg, pa.qg, w.n_slots, qcols, 128) != BA_OK ||
      encode_2d(&dm.dog, pa.dog, w.n_slots, qcols, 128) != BA_OK ||
      encode_2d(&dm.k, p->k, p->S, kcols, 128) != BA_OK ||
      encode_2d(&dm.v, p->v, p->S, kcols, 128) != BA_OK ||
      encode_2d(&dm.kb, nb ? p->kb : p->k, nb_rows_map, kcols, 128) != BA_OK ||
      encode_2d(&dm.vb, nb ? p->vb : p->v, nb_rows_map, kcols, 128) != BA_OK ||
      encode_2d(&km.qg, pa.qg, w.n_slots, qcols, 128) != BA_OK ||
      encode_2d(&km.dog, pa.dog, w.n_slots, qcols, 128) != BA_OK)
    return BA_ERR_CUDA;
  km.k = dm.k;
  km.v = dm.v;

  // 2. dQ (main and branch keys)
  DqArgs qa;
  std::memset(&qa, 0, sizeof(qa));
  qa.tiles = reinterpret_cast<const TileDesc*>(ws + w.tiles_off);
  qa.order = reinterpret_cast<const int32_t*>(ws + w.order_off);
  qa.meta = pa.meta;
  qa.ls = pa.ls;
  qa.ds = pa.ds;
  qa.bmask = bmask;
  qa.mode = p->mode;
  qa.window = p->window > 0 ? p->window : 0;
  qa.S = p->S;
  qa.Hq = p->Hq;
  qa.G = G;
  qa.d = p->d;
  qa.n_slots = w.n_slots;
  qa.n_items = static_cast<int>(items_q);
  qa.with_branch = nb ? 1 : 0;
  qa.scale_log2 = scale * 1.4426950408889634f;
  qa.scale = scale;
  qa.dq = static_cast<__nv_bfloat16*>(dq);
  qa.dqb = static_cast<__nv_bfloat16*>(nb ? dqb : dq);
  qa.err = di.err;
  qa.counter = reinterpret_cast<uint32_t*>(ws + w.counters_off) + 1;
  qa.wait_limit = g_wait_limit.load();
  {
    ProfScope prof("bwd_dq", st);
    if (launch_bwd_dq(dm, qa, di.num_sms, st) != cudaSuccess) return BA_ERR_CUDA;
  }

  // 3. dK, dV of the main keys
  DkdvArgs ka;
  std::memset(&ka, 0, sizeof(ka));
  ka.items = reinterpret_cast<const KvItem*>(ws + w.kv_items_off);
  ka.order = reinterpret_cast<const int32_t*>(ws + w.kv_order_off);
  ka.tiles = qa.tiles;
  ka.lims = pa.lims;
  ka.ls = pa.ls;
  ka.ds = pa.ds;
  ka.window = p->window > 0 ? p->window : 0;
  ka.Hq = p->Hq;
  ka.Hkv = p->Hkv;
  ka.G = G;
  ka.d = p->d;
  ka.n_slots = w.n_slots;
  ka.n_items = static_cast<int>(items_kv);
  ka.scale_log2 = qa.scale_log2;
  ka.scale = scale;
  ka.dk = static_cast<__nv_bfloat16*>(dk);
  ka.dv = static_cast<__nv_bfloat16*>(dv);
  ka.err = di.err;
  ka.counter = reinterpret_cast<uint32_t*>(ws + w.counters_off) + 2;
  ka.wait_limit = g_wait_limit.load();
  {
    ProfScope prof("bwd_dkdv", st);
    if (launch_bwd_dkdv(km, ka, di.num_sms, st) != cudaSuccess) return BA_ERR_CUDA;
  }

  // 4. dK, dV of the branch keys
  if (nb) {
    BranchBwdArgs ba_;
    std::memset(&ba_, 0, sizeof(ba_));
    ba_.qb = static_cast<const __nv_bfloat16*>(p->qb);
    ba_.kb = static_cast<const __nv_bfloat16*>(p->kb);
    ba_.vb = static_cast<const __nv_bfloat16*>(p->vb);
    ba_.dob = static_cast<const __nv_bfloat16*>(doutb);
    ba_.lse = lse;
    ba_.drow = pa.drow;
    ba_.bmask = bmask;
    ba_.cu = p->cu_seqlens_d;
    ba_.anchors = p->anchors_d;
    ba_.ndoc = p->ndoc;
    ba_.R = p->R;
    ba_.cp_rank = p->cp_select ? p->cp_rank : -1;
    ba_.S = p->S;
    ba_.Nb = p->Nb;
    ba_.B = p->B;
    ba_.mode = p->mode;
    ba_.Hq = p->Hq;
    ba_.Hkv = p->Hkv;
    ba_.rows = rows;
    ba_.scale = scale;
    ba_.dkb = static_cast<__nv_bfloat16*>(dkb);
    ba_.dvb = static_cast<__nv_bfloat16*>(dvb);
    ba_.err = di.err;
    ba_.wait_limit = g_wait_limit.load();
    ProfScope prof("branch_bwd", st);
    if (launch_branch_bwd(ba_, p->d, st) != cudaSuccess) return BA_ERR_CUDA;
  }
  return BA_OK;
}

const char* ba_status_string(ba_status s) {
  switch (s) {
    case BA_OK: return "ok";
    case BA_ERR_INVALID_ARG: return "invalid argument";
    case BA_ERR_UNSUPPORTED: return "unsupported configuration";
    case BA_ERR_CUDA: return "CUDA runtime error";
    case BA_ERR_TIMEOUT: return "device-side bounded wait expired";
    case BA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case BA_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the library's static array holds (BA_STATIC_SCRATCH_BYTES)";
  }
  return "unknown status";
}

void ba_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
}

int ba_profile_collect(const char** names, double* total_ms, int* launches, int cap) {
  std::vector<ProfRecord> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    recs.swap(g_prof);
  }
  std::map<std::string, std::pair<double, int>> acc;
  std::map<std::string, const char*> name_of;
  bool ok = true;
  for (const ProfRecord& r : recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      ok = false;
    auto& e = acc[r.name];
    e.first += ms;
    e.second += 1;
    name_of[r.name] = r.name;
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  int i = 0;
  for (const auto& kv : acc) {
    if (i < cap) {
      if (names) names[i] = name_of[kv.first];
      if (total_ms) total_ms[i] = kv.second.first;
      if (launches) launches[i] = kv.second.second;
    }
    ++i;
  }
  return ok ? i : -1;
}

void ba_set_wait_limit(long long cycles) {
  g_wait_limit.store(cycles > 0 ? cycles : kWaitLimitCycles);
}

ba_status ba_check_bounded_wait(ba_stream_t stream) {
  DeviceInfo di;
  ba_status s = device_info(&di);
  if (s != BA_OK) return s;
  if (launch_bounded_wait_probe(di.err, g_wait_limit.load(), reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return BA_ERR_CUDA;
  return BA_OK;
}

static uint32_t g_last_error_word = 0;

uint32_t ba_last_error_word(void) { return g_last_error_word; }

ba_status ba_sync_status(ba_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return BA_ERR_CUDA;
  if (word != 0) {
    g_last_error_word = word;
    const uint32_t zero = 0;
    cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    return BA_ERR_TIMEOUT;
  }
  return BA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Entry point that allocates nothing: ba_fused_fwd with its scratch in a
// file-scope device array (see ba_fused_fwd_noalloc in include/ba.h).
namespace ba {
namespace {

static __device__ __align__(256) uint8_t g_static_scratch[BA_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// Device address of g_static_scratch on the current device, looked up once
// per device.  In host code the symbol itself is only a host-side stand-in.
ba_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return BA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return BA_OK;
}

}  // namespace
}  // namespace ba

extern "C" ba_status ba_fused_fwd_noalloc(const ba_problem* p, void* o, void* ob, float* lse,
                                           ba_stream_t stream) {
  void* scratch = nullptr;
  ba_status s = static_scratch(&scratch);
  if (s != BA_OK) return s;
  return run_fwd(p, true, nullptr, o, ob, lse, reinterpret_cast<cudaStream_t>(stream), scratch,
                 BA_STATIC_SCRATCH_BYTES, BA_ERR_SCRATCH_LIMIT);
}
