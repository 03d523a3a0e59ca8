// Backward pass: pre-pass, branch-local dK/dV and the host orchestration of
// ba_bwd.  The pages do not describe the backward; it is the softmax-attention
// gradient of the same masked attention, recomputed from the merged LSE:
//   D_i = <dO_i, O_i>,  P_ij = exp(s_ij - L_i),  dS_ij = P_ij (<dO_i, v_j> - D_i)
//   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,  dV_j = sum_i P_ij dO_i
// With the merged L and D, each component's backward is plain attention
// backward restricted to that component's keys, and the two add; no separate
// backward of the Eq. 2 merge is needed.
//
// Kernels, in launch order:
//   1. bwd_prep (HBM-bound): D = rowsum(dO * O); Q and dO gathered into
//      row-tile slot order (so both tensor-core passes load whole tiles with
//      plain TMA boxes); per-slot log2-scaled L, D and key-range metadata.
//   2. bwd_dq (tcgen05, query-stationary): dQ over main and branch keys.
//   3. bwd_dkdv (tcgen05, key-stationary): dK, dV of the main keys.
//   4. branch_bwd (SIMT): dK, dV of the branch keys (a handful of pairs each).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "../../include/ba.h"
#include "bwd_kernels.h"
#include "plan.h"
#include "ptx.cuh"

namespace ba {
namespace {

// ------------------------------------------------------------------ pre-pass
// One group of D/8 threads per (slot, head); each thread moves 16 bytes of
// the row.  Slots are the row-table entries (tile * 128 + i).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const PrepArgs a) {
  constexpr int TPR = D / 8;  // threads per (slot, head)
  const int64_t pairs = a.n_slots * a.Hq;
  const int sub = threadIdx.x % TPR;
  const int64_t stride = (int64_t(gridDim.x) * blockDim.x) / TPR;
  for (int64_t pr = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / TPR; pr < pairs; pr += stride) {
    const int64_t slot = pr / a.Hq;
    const int h = static_cast<int>(pr % a.Hq);
    const int r = a.row_table[slot];
    uint4 qv = make_uint4(0, 0, 0, 0), dv = make_uint4(0, 0, 0, 0);
    float dsum = 0.f;
    if (r >= 0) {
      const bool br = r >= a.S;
      const int64_t rr = br ? r - a.S : r;
      const int64_t off = (rr * a.Hq + h) * D + sub * 8;
      qv = *reinterpret_cast<const uint4*>((br ? a.qb : a.q) + off);
      dv = *reinterpret_cast<const uint4*>((br ? a.dob : a.dout) + off);
      const uint4 ov = *reinterpret_cast<const uint4*>((br ? a.ob : a.o) + off);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(d2[i]);
        const float2 y = __bfloat1622float2(o2[i]);
        dsum = fmaf(x.x, y.x, dsum);
        dsum = fmaf(x.y, y.y, dsum);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off, TPR);
    const int64_t goff = (slot * a.Hq + h) * D + sub * 8;
    *reinterpret_cast<uint4*>(a.qg + goff) = qv;
    *reinterpret_cast<uint4*>(a.dog + goff) = dv;
    if (sub == 0) {
      const int64_t hs = int64_t(h) * a.n_slots + slot;
      if (r >= 0) {
        a.ls[hs] = -a.lse[int64_t(h) * a.rows + r] * 1.4426950408889634f;
        a.ds[hs] = dsum;
        a.drow[int64_t(h) * a.rows + r] = dsum;
      } else {
        a.ls[hs] = -INFINITY;  // padding: P = exp2(s - inf) = 0
        a.ds[hs] = 0.f;
      }
      if (h == 0) {
        SlotMeta m;
        m.limit = -1;
        m.blo = m.bhi = 0;
        m.row = r;
        if (r >= 0 && r < a.S) {
          m.limit = r;
        } else if (r >= a.S) {
          const int b = (r - a.S) / a.B;
          const int t = (r - a.S) - b * a.B;
          m.limit = a.anchors[b];
          m.blo = b * a.B;
          m.bhi = m.blo + (a.mode == 0 ? t + 1 : a.B);
        }
        a.meta[slot] = m;
        a.lims[slot] = m.limit;
      }
    }
  }
}

// ------------------------------------------------------------------ branch dK/dV
// Virtual rank owning main position p: the zigzag chunk k of its document
// [s, s + L) with s + floor(kL/2R) <= p < s + floor((k+1)L/2R) belongs to
// rank k (k < R) or 2R-1-k.
__device__ __forceinline__ int zigzag_owner(const int32_t* cu, int ndoc, int R, int p) {
  int lo = 0, hi = ndoc - 1;  // last document with start <= p
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= p) lo = mid; else hi = mid - 1;
  }
  const int64_t s = cu[lo], L = cu[lo + 1] - cu[lo], R2 = 2 * R;
  int64_t k = (int64_t(p) - s) * R2 / L;  // floor(kL/2R) <= p - s for this k
  while (k + 1 < R2 && s + (k + 1) * L / R2 <= p) ++k;
  return static_cast<int>(k < R ? k : R2 - 1 - k);
}

// One block per (branch b, KV head g); one warp per branch key u (strided).
// The block's inputs are contiguous runs of the input layouts: for each of the
// B rows, the G query heads of q and of dO (G * D values), and for each of the
// B keys, k and v (D values).  Thread 0 moves them into shared memory with
// 4B bulk copies (the TMA engine, completion counted on one mbarrier), so all
// of a block's bytes are in flight at once instead of one row per warp at a
// time; the warps then work from shared memory.  Lane l holds elements
// [l*E, l*E + E) of k_u, v_u and of the accumulators.  For every query head of
// the group and every row t that sees u (chain: t >= u; block: all; bitmask:
// bit u of row t's word):
//   s = scale <q_t, k_u>, P = exp(s - L_t), dS = P (<dO_t, v_u> - D_t),
//   dV_u += P dO_t, dK_u += scale dS q_t.
// E consecutive bf16 values of shared memory (8 or 4 bytes, aligned) as floats.
template <int E>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* p, float (&f)[E]) {
  static_assert(E == 4 || E == 2, "4 or 2 values per lane");
  if constexpr (E == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
    f[0] = lo.x; f[1] = lo.y; f[2] = hi.x; f[3] = hi.y;
  } else {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    f[0] = v.x; f[1] = v.y;
  }
}

template <int D>
__global__ void __launch_bounds__(256) branch_bwd_kernel(const BranchBwdArgs a) {
  constexpr int E = D / 32;
  const int b = blockIdx.x / a.Hkv;
  const int g = blockIdx.x % a.Hkv;
  // one rank's rows: the branch belongs to the rank owning its anchor
  if (a.cp_rank >= 0 && zigzag_owner(a.cu, a.ndoc, a.R, a.anchors[b]) != a.cp_rank) return;
  const int G = a.Hq / a.Hkv;
  const int B = a.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  extern __shared__ __align__(128) uint8_t sm[];
  __nv_bfloat16* sq = reinterpret_cast<__nv_bfloat16*>(sm);  // [B][G][D]
  __nv_bfloat16* sdo = sq + B * G * D;                        // [B][G][D]
  __nv_bfloat16* sk = sdo + B * G * D;                        // [B][D]
  __nv_bfloat16* sv = sk + B * D;                             // [B][D]
  float* sL = reinterpret_cast<float*>(sv + B * D);           // [B][G] natural-log LSE
  float* sD = sL + B * G;                                     // [B][G]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sL + ((2 * B * G + 1) & ~1));  // after L, D; 8-byte aligned
  const uint32_t bar_a = ptx::smem_u32(bar);
  const int64_t row0 = int64_t(b) * B;  // flattened branch row / key of (b, 0)
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_a, 1);
    ptx::fence_mbar_init();
    const uint32_t rowb = static_cast<uint32_t>(G * D * 2), keyb = static_cast<uint32_t>(D * 2);
    ptx::mbar_expect_tx(bar_a, 2u * B * (rowb + keyb));
    for (int t = 0; t < B; ++t) {
      const int64_t qo = ((row0 + t) * a.Hq + int64_t(g) * G) * D;
      const int64_t ko = ((row0 + t) * a.Hkv + g) * D;
      ptx::bulk_g2s(ptx::smem_u32(sq + t * G * D), a.qb + qo, rowb, bar_a);
      ptx::bulk_g2s(ptx::smem_u32(sdo + t * G * D), a.dob + qo, rowb, bar_a);
      ptx::bulk_g2s(ptx::smem_u32(sk + t * D), a.kb + ko, keyb, bar_a);
      ptx::bulk_g2s(ptx::smem_u32(sv + t * D), a.vb + ko, keyb, bar_a);
    }
  }
  for (int i = threadIdx.x; i < B * G; i += blockDim.x) {
    const int64_t row = int64_t(a.S) + row0 + i / G;
    const int64_t h = int64_t(g) * G + i % G;
    sL[i] = a.lse[h * a.rows + row];
    sD[i] = a.drow[h * a.rows + row];
  }
  __syncthreads();  // the barrier's initialisation and L, D
  {
    volatile int never = 0;
    if (!ptx::mbar_wait(bar_a, 0, &never, a.err, a.wait_limit, ptx::wait_site(5, 2, 1))) {
      // the copies still land before the block's shared memory goes away
      ptx::mbar_wait(bar_a, 0, &never, a.err, ptx::kDrainCycles);
      return;
    }
  }
  for (int u = warp; u < B; u += nw) {
    float kf[E], vf[E], dk[E], dv[E];
    load_bf16<E>(sk + u * D + lane * E, kf);
    load_bf16<E>(sv + u * D + lane * E, vf);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dk[e] = 0.f;
      dv[e] = 0.f;
    }
    for (int hh = 0; hh < G; ++hh) {
      for (int t = (a.mode == 0 ? u : 0); t < B; ++t) {
        // bitmask: row t sees key u iff bit u of its word
        if (a.mode == 2 && !((a.bmask[row0 + t] >> u) & 1ull)) continue;
        const int o = (t * G + hh) * D + lane * E;
        float qf[E], df[E];
        load_bf16<E>(sq + o, qf);
        load_bf16<E>(sdo + o, df);
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s = fmaf(qf[e], kf[e], s);
          dp = fmaf(df[e], vf[e], dp);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          s += __shfl_xor_sync(0xffffffffu, s, off);
          dp += __shfl_xor_sync(0xffffffffu, dp, off);
        }
        const float P = expf(s * a.scale - sL[t * G + hh]);
        const float dS = P * (dp - sD[t * G + hh]);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dv[e] = fmaf(P, df[e], dv[e]);
          dk[e] = fmaf(dS, qf[e], dk[e]);
        }
      }
    }
    const int64_t ku = ((row0 + u) * a.Hkv + g) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      a.dkb[ku + e] = __float2bfloat16_rn(dk[e] * a.scale);
      a.dvb[ku + e] = __float2bfloat16_rn(dv[e]);
    }
  }
}

// The same computation for shapes whose rows do not fit in one block's shared
// memory (large B x G): each warp loads its rows from global memory one at a
// time.
template <int D>
__global__ void branch_bwd_rows_kernel(const BranchBwdArgs a) {
  constexpr int E = D / 32;
  const int b = blockIdx.x / a.Hkv;
  const int g = blockIdx.x % a.Hkv;
  // one rank's rows: the branch belongs to the rank owning its anchor
  if (a.cp_rank >= 0 && zigzag_owner(a.cu, a.ndoc, a.R, a.anchors[b]) != a.cp_rank) return;
  const int G = a.Hq / a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const int64_t base_row = int64_t(a.S) + int64_t(b) * a.B;  // concatenated row of (b, 0)
  for (int u = warp; u < a.B; u += nw) {
    const int64_t ku = ((int64_t(b) * a.B + u) * a.Hkv + g) * D + lane * E;
    float kf[E], vf[E], dk[E], dv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kf[e] = __bfloat162float(a.kb[ku + e]);
      vf[e] = __bfloat162float(a.vb[ku + e]);
      dk[e] = 0.f;
      dv[e] = 0.f;
    }
    for (int hh = 0; hh < G; ++hh) {
      const int h = g * G + hh;
      for (int t = (a.mode == 0 ? u : 0); t < a.B; ++t) {
        // bitmask: row t sees key u iff bit u of its word
        if (a.mode == 2 && !((a.bmask[int64_t(b) * a.B + t] >> u) & 1ull)) continue;
        const int64_t qo = ((int64_t(b) * a.B + t) * a.Hq + h) * D + lane * E;
        float qf[E], df[E];
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          qf[e] = __bfloat162float(a.qb[qo + e]);
          df[e] = __bfloat162float(a.dob[qo + e]);
          s = fmaf(qf[e], kf[e], s);
          dp = fmaf(df[e], vf[e], dp);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          s += __shfl_xor_sync(0xffffffffu, s, off);
          dp += __shfl_xor_sync(0xffffffffu, dp, off);
        }
        const int64_t row = base_row + t;
        const float P = expf(s * a.scale - a.lse[int64_t(h) * a.rows + row]);
        const float dS = P * (dp - a.drow[int64_t(h) * a.rows + row]);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dv[e] = fmaf(P, df[e], dv[e]);
          dk[e] = fmaf(dS, qf[e], dk[e]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      a.dkb[ku + e] = __float2bfloat16_rn(dk[e] * a.scale);
      a.dvb[ku + e] = __float2bfloat16_rn(dv[e]);
    }
  }
}

// Shared memory of one branch-key block: q, dO [B][G][D], k, v [B][D] (bf16),
// L, D [B][G] (fp32, padded to 8 bytes) and the copy barrier.
size_t branch_bwd_smem(int B, int G, int d) {
  return size_t(2) * B * G * d * 2 + size_t(2) * B * d * 2 + size_t((2 * B * G + 1) & ~1) * 4 + 8;
}

int grid_cap(int64_t work, int per_block, int cap) {
  int64_t g = (work + per_block - 1) / per_block;
  if (g < 1) g = 1;
  if (g > cap) g = cap;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_bwd_prep(const PrepArgs& a, int d, cudaStream_t st) {
  const int tpr = d / 8;
  const int64_t threads = a.n_slots * a.Hq * tpr;
  const int grid = grid_cap(threads, 256, 148 * 32);
  if (d == 128)
    bwd_prep_kernel<128><<<grid, 256, 0, st>>>(a);
  else
    bwd_prep_kernel<64><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_branch_bwd(const BranchBwdArgs& a, int d, cudaStream_t st) {
  if (a.Nb == 0) return cudaSuccess;
  const int64_t blocks = int64_t(a.Nb) * a.Hkv;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  const int warps = a.B < 8 ? a.B : 8;
  const size_t smem = branch_bwd_smem(a.B, a.Hq / a.Hkv, d);
  if (smem > 232448) {  // B x G too large for one block's rows in shared memory
    if (d == 128)
      branch_bwd_rows_kernel<128><<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(a);
    else
      branch_bwd_rows_kernel<64><<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(a);
    return cudaGetLastError();
  }
  cudaError_t e = d == 128 ? cudaFuncSetAttribute(branch_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem))
                           : cudaFuncSetAttribute(branch_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (d == 128)
    branch_bwd_kernel<128><<<static_cast<unsigned>(blocks), warps * 32, smem, st>>>(a);
  else
    branch_bwd_kernel<64><<<static_cast<unsigned>(blocks), warps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace ba
