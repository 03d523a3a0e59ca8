// Small kernels: row-table scatter of the plan, the standalone branch-local
// component (step a3) and the k-way LSE merge (step a4, Eq. 2).
#include <cuda_bf16.h>

#include <cmath>

#include "kernels.h"
#include "ptx.cuh"

namespace ba {
namespace {

// ------------------------------------------------------------------ plan rows
// Writes every covered concatenated row index r (main rows 0..S-1, then
// branch rows S + b*B + t) into its slot of the row table.  The plan covers
// row segments (whole documents, or one virtual rank's zigzag chunks): main
// positions [c0, c1) and the branches anchored there, in position order.
// Within a segment the rows are ordered by limit (main row p: p; branch row:
// its anchor), main row first on ties, then branches in index order,
// depth-minor:
//   main p:       m = (p - c0) + B * (#anchors in [c0, p))
//   branch (b,t): m = (a_b - c0) + 1 + B * (b - b0) + t
// where b0 is the segment's first branch.  Rows outside every segment are
// skipped.
__global__ void plan_rows_kernel(const ChunkDev* __restrict__ segs, int nseg,
                                 const int32_t* __restrict__ anchors, int S, int Nb, int B,
                                 int32_t* __restrict__ rows, int64_t n_slots) {
  const int64_t total = int64_t(S) + int64_t(Nb) * B;
  for (int64_t r = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; r < total;
       r += int64_t(gridDim.x) * blockDim.x) {
    int lim, b = 0, t = 0;
    const bool br = r >= S;
    if (!br) {
      lim = static_cast<int>(r);
    } else {
      const int64_t q = r - S;
      b = static_cast<int>(q / B);
      t = static_cast<int>(q - int64_t(b) * B);
      lim = anchors[b];
    }
    int lo = 0, hi = nseg - 1;  // last segment with c0 <= lim
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (segs[mid].c0 <= lim) lo = mid; else hi = mid - 1;
    }
    const ChunkDev c = segs[lo];
    if (lim < c.c0 || lim >= c.pad) continue;  // not a covered row
    int64_t m;
    if (!br) {
      int a0 = 0, a1 = Nb;  // first anchor >= lim
      while (a0 < a1) {
        const int mid = (a0 + a1) >> 1;
        if (anchors[mid] < lim) a0 = mid + 1; else a1 = mid;
      }
      m = int64_t(lim - c.c0) + int64_t(B) * (a0 - c.b0);
    } else {
      m = int64_t(lim - c.c0) + 1 + int64_t(B) * (b - c.b0) + t;
    }
    const int64_t slot = int64_t(c.slot_base) + m;
    if (slot >= 0 && slot < n_slots) rows[slot] = static_cast<int32_t>(r);
  }
}

// ------------------------------------------------------------------ branch part
// One block per (branch b, KV head g), one warp per query head of the group.
// The branch's B keys and values of head g are staged in shared memory; each
// warp walks the B rows of its head: scores against the visible branch keys
// (chain: u <= t; block: all; bitmask: the row's bits), softmax, O = P V.
// Output fp32 O and LSE.
template <int D>
__global__ void branch_fwd_kernel(const __nv_bfloat16* __restrict__ qb,
                                  const __nv_bfloat16* __restrict__ kb,
                                  const __nv_bfloat16* __restrict__ vb,
                                  const uint64_t* __restrict__ bmask, int Nb, int B, int mode,
                                  int Hq, int Hkv, float scale, float* __restrict__ o_part,
                                  float* __restrict__ lse_part) {
  constexpr int E = D / 32;  // elements per lane
  extern __shared__ float sm[];  // [2][B][D]
  const int b = blockIdx.x / Hkv;
  const int g = blockIdx.x % Hkv;
  const int G = Hq / Hkv;
  float* sk = sm;
  float* sv = sm + B * D;
  for (int i = threadIdx.x; i < B * D; i += blockDim.x) {
    const int u = i / D, e = i % D;
    const int64_t off = ((int64_t(b) * B + u) * Hkv + g) * D + e;
    sk[i] = __bfloat162float(kb[off]);
    sv[i] = __bfloat162float(vb[off]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= G) return;
  const int h = g * G + warp;
  const int64_t nbr = int64_t(Nb) * B;
  for (int t = 0; t < B; ++t) {
    const int64_t row = int64_t(b) * B + t;
    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = __bfloat162float(qb[(row * Hq + h) * D + lane * E + e]);
    const int nvis = mode == 0 ? t + 1 : B;
    const uint64_t bits = mode == 2 ? bmask[row] : ~0ull;
    float mx = -INFINITY, l = 0.f;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int u = 0; u < nvis; ++u) {
      if (!((bits >> u) & 1ull)) continue;  // bitmask: row t sees key u iff bit u is set
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) s = fmaf(qv[e], sk[u * D + lane * E + e], s);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      s *= scale;
      const float mn = fmaxf(mx, s);
      const float c = expf(mx - mn);
      const float p = expf(s - mn);
      l = l * c + p;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = acc[e] * c + p * sv[u * D + lane * E + e];
      mx = mn;
    }
    // a bitmask row may see no branch key at all: the empty partial (0, -inf)
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o_part[(row * Hq + h) * D + lane * E + e] = acc[e] * inv;
    if (lane == 0) lse_part[int64_t(h) * nbr + row] = l > 0.f ? mx + logf(l) : -INFINITY;
  }
}

// ------------------------------------------------------------------ LSE merge
// One warp per (head h, group of 32 rows).  Lane j first merges the LSEs of
// row r0 + j (coalesced over rows); then D/8 lanes cover one row, each lane 8
// consecutive elements: two 16-byte fp32 loads per part and one 16-byte bf16
// store, 32/(D/8) rows per warp instruction and two such row sets in flight.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const MergeArgs a) {
  constexpr int TPR = D / 8;      // lanes per row
  constexpr int RPI = 32 / TPR;   // rows per warp instruction
  constexpr int U = 2;            // row sets per iteration
  const int64_t groups = (int64_t(a.rows) + 31) / 32;
  const int64_t nwarps = groups * a.H;
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPR, rsel = lane / TPR;
  for (int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / 32; w < nwarps;
       w += (int64_t(gridDim.x) * blockDim.x) / 32) {
    const int h = static_cast<int>(w % a.H);
    const int64_t r0 = (w / a.H) * 32;
    const int64_t my = r0 + lane;
    const bool live = my < a.rows;
    float lp[16];
    float mx = -INFINITY;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      lp[p] = -INFINITY;
      if (p < a.nparts && live) lp[p] = a.lse[p][int64_t(h) * a.lse_ld[p] + my];
      mx = fmaxf(mx, lp[p]);
    }
    float Lr = -INFINITY;
    float wt[16];
    if (mx != -INFINITY) {
      float tot = 0.f;
#pragma unroll
      for (int p = 0; p < 16; ++p) tot += (lp[p] == -INFINITY) ? 0.f : expf(lp[p] - mx);
      Lr = mx + logf(tot);
    }
#pragma unroll
    for (int p = 0; p < 16; ++p) wt[p] = (Lr == -INFINITY || lp[p] == -INFINITY) ? 0.f : expf(lp[p] - Lr);
    if (live) a.lse_out[int64_t(h) * a.lse_out_ld + my] = Lr;
    const int64_t left = int64_t(a.rows) - r0;
    const int nr = left < 32 ? static_cast<int>(left) : 32;
    for (int i0 = 0; i0 < nr; i0 += RPI * U) {
      float acc[U][8];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        if (p >= a.nparts) break;
        float4 v[U][2];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = i0 + u * RPI + rsel;
          v[u][0] = v[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < nr) {
            const float4* src = reinterpret_cast<const float4*>(a.o[p] + ((r0 + i) * a.H + h) * D + sub * 8);
            v[u][0] = src[0];
            v[u][1] = src[1];
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const float wp = __shfl_sync(0xffffffffu, wt[p], (i0 + u * RPI + rsel) & 31);
          acc[u][0] = fmaf(wp, v[u][0].x, acc[u][0]);
          acc[u][1] = fmaf(wp, v[u][0].y, acc[u][1]);
          acc[u][2] = fmaf(wp, v[u][0].z, acc[u][2]);
          acc[u][3] = fmaf(wp, v[u][0].w, acc[u][3]);
          acc[u][4] = fmaf(wp, v[u][1].x, acc[u][4]);
          acc[u][5] = fmaf(wp, v[u][1].y, acc[u][5]);
          acc[u][6] = fmaf(wp, v[u][1].z, acc[u][6]);
          acc[u][7] = fmaf(wp, v[u][1].w, acc[u][7]);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * RPI + rsel;
        if (i >= nr) continue;
        uint4 o;
        o.x = ptx::pack_bf16x2(acc[u][0], acc[u][1]);
        o.y = ptx::pack_bf16x2(acc[u][2], acc[u][3]);
        o.z = ptx::pack_bf16x2(acc[u][4], acc[u][5]);
        o.w = ptx::pack_bf16x2(acc[u][6], acc[u][7]);
        *reinterpret_cast<uint4*>(a.o_out + ((r0 + i) * a.H + h) * D + sub * 8) = o;
      }
    }
  }
}

// ------------------------------------------------------------------ bounded-wait probe
__global__ void bounded_wait_probe_kernel(uint32_t* err, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    const uint32_t b = ptx::smem_u32(&bar);
    ptx::mbar_init(b, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
    // nothing ever arrives: the wait gives up after `limit` cycles and reports
    ptx::mbar_wait(b, 0, &abort_flag, err, limit, ptx::wait_site(4, 0, 1));
  }
}

int grid_for(int64_t work, int per_block, int cap) {
  int64_t g = (work + per_block - 1) / per_block;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_plan_rows(const ChunkDev* segs, int nseg, const int32_t* anchors, int S, int Nb,
                             int B, int32_t* row_table, int64_t n_slots, cudaStream_t stream) {
  const int64_t total = int64_t(S) + int64_t(Nb) * B;
  if (nseg <= 0) return cudaSuccess;
  plan_rows_kernel<<<grid_for(total, 256, 148 * 16), 256, 0, stream>>>(
      segs, nseg, anchors, S, Nb, B, row_table, n_slots);
  return cudaGetLastError();
}

cudaError_t launch_branch_fwd(const __nv_bfloat16* qb, const __nv_bfloat16* kb,
                              const __nv_bfloat16* vb, const uint64_t* bmask, int Nb, int B,
                              int mode, int Hq, int Hkv, int d, float scale, float* o_part,
                              float* lse_part, cudaStream_t stream) {
  if (Nb == 0) return cudaSuccess;
  const int G = Hq / Hkv;
  const int threads = G * 32 < 64 ? 64 : G * 32;
  const size_t smem = size_t(2) * B * d * sizeof(float);
  const int64_t blocks = int64_t(Nb) * Hkv;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (d == 128) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(branch_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
    branch_fwd_kernel<128><<<static_cast<unsigned>(blocks), threads, smem, stream>>>(
        qb, kb, vb, bmask, Nb, B, mode, Hq, Hkv, scale, o_part, lse_part);
  } else {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(branch_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
    branch_fwd_kernel<64><<<static_cast<unsigned>(blocks), threads, smem, stream>>>(
        qb, kb, vb, bmask, Nb, B, mode, Hq, Hkv, scale, o_part, lse_part);
  }
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_probe(uint32_t* err, long long limit, cudaStream_t stream) {
  bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(err, limit);
  return cudaGetLastError();
}

cudaError_t launch_lse_merge(const MergeArgs& a, cudaStream_t stream) {
  const int64_t warps = (int64_t(a.rows) + 31) / 32 * a.H;
  const int grid = grid_for(warps, 8, 148 * 32);
  if (a.d == 128)
    lse_merge_kernel<128><<<grid, 256, 0, stream>>>(a);
  else
    lse_merge_kernel<64><<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ba
