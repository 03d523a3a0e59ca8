/*
 * ba.h -- branch attention for speculative-draft training on B200 (sm_100a).
 *
 * C ABI of libba_b200.so.  Plain pointers and sizes only.
 *
 * The operation.  Source: "Online Draft Co-Training for Speculative Decoding
 * in Large-Scale, Long-Context RL Post-Training" (arXiv 2609.07108), §3.2 and
 * Eq. 2, as described on the rcap.io post (paragraph on branch attention under
 * context parallelism) and the evolve.pub review (Summary; FAQ on branch
 * attention under CP).  A packed main sequence of S tokens (documents given by
 * cu_seqlens, no padding) carries Nb draft branches; branch b hangs off the
 * main position anchors[b] and has B rows.  Every query row attends with a
 * softmax over its visible keys:
 *   - main row i:        main keys j in [s(i), i]      (s = document start)
 *   - branch row (b, t): main keys j in [s(a_b), a_b]  (causal prefix up to
 *                        and including the anchor) plus its own branch keys
 *                        (b, u) with u <= t (BA_MASK_CHAIN, EAGLE-3 training-
 *                        time test) or all u < B (BA_MASK_BLOCK, DFlash-style
 *                        block draft).
 * Main rows never see branch keys; branches never see each other's keys.
 * The library computes it the way the paper decomposes it: a causal
 * main-sequence component over a load-balanced zigzag split (R virtual ranks
 * on one GPU), a rank-local branch component, and the online-softmax
 * (log-sum-exp) merge of the two, Eq. 2:
 *     L = log(exp(L1) + exp(L2)),  O = exp(L1 - L) O1 + exp(L2 - L) O2.
 * The backward pass (dQ, dK, dV through both parts) is not described on the
 * pages; it is the textbook softmax-attention gradient of the same definition,
 * recomputed from the merged LSE.
 *
 * Conventions (all entry points):
 *   - Tensors are row-major with the last dimension contiguous:
 *       q  bf16 [S, Hq, d]        k, v   bf16 [S, Hkv, d]
 *       qb bf16 [Nb, B, Hq, d]    kb, vb bf16 [Nb, B, Hkv, d]
 *     GQA: query head h uses KV head h / (Hq / Hkv).
 *   - "Rows" are the S main rows followed by the Nb*B branch rows (b-major,
 *     depth-minor).  LSE arrays are fp32 [Hq, rows] (head-major), natural log.
 *   - Every device pointer must be 16-byte aligned.  Supported: d in {64, 128},
 *     Hq % Hkv == 0, 1 <= B <= 64, 1 <= R <= 64.  anchors ascending (ties
 *     allowed), each in [0, S).  Nb may be 0 (plain packed causal attention).
 *   - scale <= 0 selects 1/sqrt(d).
 *   - Ownership: the caller owns every buffer, including the workspace whose
 *     size ba_workspace_size() returns.  The library allocates no device
 *     memory on these paths.  Its only state between calls is a cache of host
 *     plans (see ba_plan_prepare / ba_clear_cache).
 *   - Work is enqueued on `stream` and runs asynchronously.  Argument errors are
 *     detected on the host before anything is enqueued.  A device-side bounded
 *     wait that expires sets a device error word and the kernel returns;
 *     ba_sync_status() reports it as BA_ERR_TIMEOUT.
 *   - Results do not depend on R beyond floating-point summation order.
 */
#ifndef BA_B200_H
#define BA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BA_API __attribute__((visibility("default")))
#else
#define BA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* ba_stream_t;

typedef enum {
  BA_OK = 0,
  BA_ERR_INVALID_ARG = -1, /* bad size, pointer, layout or ordering */
  BA_ERR_UNSUPPORTED = -2, /* valid but not implemented (e.g. d = 96) */
  BA_ERR_CUDA = -3,        /* a CUDA runtime call failed */
  BA_ERR_TIMEOUT = -4,     /* a device-side bounded wait expired */
  BA_ERR_WORKSPACE = -5,   /* workspace missing or too small */
  BA_ERR_SCRATCH_LIMIT = -6 /* problem needs more than the static scratch array holds */
} ba_status;

typedef enum {
  BA_MASK_CHAIN = 0,  /* EAGLE-3 training-time test: depth t sees branch keys u <= t */
  BA_MASK_BLOCK = 1,  /* DFlash-style block draft: all B keys of its own block */
  BA_MASK_BITMASK = 2 /* any per-branch pattern, e.g. for DSpark's Markov head (the
                         pages do not spell that mask out): row (b, t) sees branch
                         key (b, u) iff bit u of branch_mask[b * B + t] is set */
} ba_mask_mode;

enum { BA_WS_FWD = 0, BA_WS_BWD = 1 };

typedef struct {
  int S;      /* packed main tokens (sum of document lengths), >= 1 */
  int ndoc;   /* documents, >= 1; cu_seqlens has ndoc + 1 entries */
  int Hq;     /* query heads */
  int Hkv;    /* key/value heads, Hq % Hkv == 0 */
  int d;      /* head dimension: 64 or 128 */
  int Nb;     /* branches (may be 0) */
  int B;      /* branch depth (chain) or block size (block) */
  int mode;   /* ba_mask_mode */
  int R;      /* virtual zigzag ranks, >= 1 */
  float scale;/* softmax scale; <= 0 selects 1/sqrt(d) */
  const int32_t* cu_seqlens_h; /* host copy, [ndoc + 1], 0 = c0 < c1 < ... = S */
  const int32_t* cu_seqlens_d; /* device copy of the same */
  const int32_t* anchors_h;    /* host copy, [Nb], ascending, in [0, S) */
  const int32_t* anchors_d;    /* device copy of the same */
  const void* q;  const void* k;  const void* v;   /* device, bf16 */
  const void* qb; const void* kb; const void* vb;  /* device, bf16 (ignored if Nb == 0) */
  void* workspace;        /* device, 256-byte aligned, caller-owned */
  size_t workspace_bytes; /* its size */
  int window;             /* main-prefix window W: if > 0, a row whose last main key is l
                             sees only main keys [max(s(l), l - W + 1), l]; branch keys
                             are not affected; <= 0: no window */
  const uint64_t* branch_mask_h; /* BA_MASK_BITMASK only: host copy, [Nb * B] words */
  const uint64_t* branch_mask_d; /* device copy of the same (16-byte aligned) */
  int cp_select;          /* 0: every row; 1: only the rows the zigzag split gives
                             virtual rank cp_rank (its two chunks of every document
                             and the branches anchored there) -- one rank's share
                             under context parallelism; see the notes below */
  int cp_rank;            /* 0 <= cp_rank < R when cp_select = 1 */
} ba_problem;

/* One rank's rows (cp_select = 1).  Every entry point then computes only the
 * rows of virtual rank cp_rank, against the full main K/V (which a context-
 * parallel caller all-gathers first): the forward writes O / LSE of those rows
 * alone; ba_bwd writes dQ of those rows, dK / dV of the branches anchored in
 * the rank's chunks, and a partial dK / dV of every main key -- the
 * contributions of this rank's rows only, zero for keys none of them sees --
 * which the ranks then sum.  Rows, keys and branches outside stay untouched
 * except for those partial main-key gradients.  ba_plan_stats counts the
 * rank's rows. */

/* Bytes of workspace that ba_main_fwd / ba_fused_fwd (which = BA_WS_FWD) or
 * ba_bwd (which = BA_WS_BWD) need for this problem.  Returns 0 if the problem
 * is invalid.  Host only; reads cu_seqlens_h and anchors_h. */
BA_API size_t ba_workspace_size(const ba_problem* p, int which);

/* Step a2: the causal main-sequence component of every row (main rows, then
 * branch rows), i.e. each row against main keys [s(limit), limit] with
 * limit = i for main row i and a_b for branch row (b, t), over the zigzag
 * split into R virtual ranks.
 *   o_part   device fp32 [S + Nb*B, Hq, d]: the normalised output of this
 *            component alone (its softmax runs over main keys only)
 *   lse_part device fp32 [Hq, S + Nb*B]: its log-sum-exp
 * Needs ba_workspace_size(p, BA_WS_FWD) bytes of workspace.
 * Paper: §3.2 (rcap.io post: the main-sequence part is computed by the
 * existing packed, load-balanced zigzag ring attention). */
BA_API ba_status ba_main_fwd(const ba_problem* p, float* o_part, float* lse_part, ba_stream_t stream);

/* Step a2 as the ring computes it: per-virtual-rank partials of the main
 * component.  The zigzag split gives virtual rank k the keys of chunks k and
 * 2R-1-k of every document; partial k of a row is its attention over the
 * visible main keys among those, i.e. what the row's rank computes at the
 * ring step where rank k's K/V visit it.  Merging the R partials of a row
 * with ba_lse_merge (Eq. 2; R <= 16 there) gives ba_main_fwd's result.
 *   o_parts   device fp32 [R, S + Nb*B, Hq, d]
 *   lse_parts device fp32 [R, Hq, S + Nb*B]
 * A row with no visible key in rank k's chunks gets the empty partial
 * (O = 0, LSE = -inf).  Needs ba_workspace_size(p, BA_WS_FWD) bytes of
 * workspace.  Paper: §3.2 (rcap.io post: the main-sequence part rides the
 * packed, load-balanced zigzag ring attention, whose ring steps are merged
 * with the log-sum-exp rule); the zigzag chunk rule itself is this library's
 * reading: a document [s, s+L) is cut at s + floor(kL/2R). */
BA_API ba_status ba_main_fwd_ring(const ba_problem* p, float* o_parts, float* lse_parts,
                                  ba_stream_t stream);

/* Step a3: the rank-local branch component: each branch row against its own
 * branch keys only (chain: u <= t; block: all B).  Needs no workspace.
 *   o_part   device fp32 [Nb*B, Hq, d]
 *   lse_part device fp32 [Hq, Nb*B]
 * Paper: §3.2 (rcap.io post; evolve.pub FAQ: the branch-local part is
 * computed on the rank that holds the branch's anchor, so branch K/V never
 * move). */
BA_API ba_status ba_branch_fwd(const ba_problem* p, float* o_part, float* lse_part, ba_stream_t stream);

/* Step a4: k-way online-softmax merge, Eq. 2, of nparts partial results over
 * the same rows:  L = log sum_p exp(L_p),  O = sum_p exp(L_p - L) O_p.
 * A partial with L_p = -inf is empty and contributes nothing; if all are
 * empty the row gets O = 0, L = -inf.
 *   o_parts    host array of nparts device pointers, each fp32 [rows, H, d]
 *   lse_parts  host array of nparts device pointers; element (h, r) of part p
 *              is lse_parts[p][h * lse_ld[p] + r]
 *   lse_ld     host array of nparts head strides (>= rows)
 *   o_out      device bf16 [rows, H, d] (round to nearest even)
 *   lse_out    device fp32, element (h, r) at lse_out[h * lse_out_ld + r]
 * 1 <= nparts <= 16; d in {64, 128}.  Needs no workspace.
 * Paper: Eq. 2 (evolve.pub "Scope & Claims"); the rcap.io post calls it the
 * log-sum-exp rule ring attention uses between ring steps. */
BA_API ba_status ba_lse_merge(int nparts, int rows, int H, int d,
                       const float* const* o_parts, const float* const* lse_parts,
                       const int64_t* lse_ld, void* o_out, float* lse_out,
                       int64_t lse_out_ld, ba_stream_t stream);

/* Steps a2 + a3 + a4 in one persistent kernel: the branch-local keys are
 * visited as extra key tiles of the same online softmax, so the Eq. 2 merge
 * happens in registers and TMEM.
 *   o    device bf16 [S, Hq, d]         final output of the main rows
 *   ob   device bf16 [Nb, B, Hq, d]     final output of the branch rows
 *   lse  device fp32 [Hq, S + Nb*B]     merged LSE (input to ba_bwd)
 * Needs ba_workspace_size(p, BA_WS_FWD) bytes of workspace.
 * Paper: §3.2; the cere-bro wiki page ("Obstacle one, context parallelism")
 * describes the merge as happening within the ring pass itself. */
BA_API ba_status ba_fused_fwd(const ba_problem* p, void* o, void* ob, float* lse, ba_stream_t stream);

/* ba_fused_fwd for callers that cannot allocate device memory.  The paper has
 * no counterpart; this is a deployment convenience.  Some callers cannot call
 * cudaMalloc or hand the library a freshly allocated workspace: a runtime
 * whose allocator owns every byte of device memory and forbids side
 * allocations, code running under a strict device-memory budget fixed at
 * start-up, or a caller that must not trigger an allocation's implicit
 * synchronisation in the middle of a stream.  This entry point computes
 * exactly what ba_fused_fwd computes (same kernels, same plan, same outputs)
 * but takes its scratch space (the plan: tile table, order, tile pairs, chunk
 * table and row table) from a file-scope device array inside the library instead of
 * p->workspace, which is ignored along with p->workspace_bytes.
 *   - Capacity: BA_STATIC_SCRATCH_BYTES (8 MiB), enough for problems of up to
 *     about 1.8 million rows (S + Nb*B).  Every GPU that loads the library
 *     holds this array until the process exits.  A problem whose plan needs
 *     more returns BA_ERR_SCRATCH_LIMIT before anything is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on that device.
 *   - All calls share the one array, and it keeps the last call's contents.
 *     Each call rewrites every part of it that it reads (the row table is
 *     reset to -1 on every call), so nothing relies on earlier contents.
 *     Calls whose work overlaps on the GPU (different streams, or different
 *     host threads, on the same device) race on the array: serialise them.
 *   - Allocates no device memory and calls no allocating library routine.
 *     The host plan comes from the plan cache (built on the host if absent;
 *     this call never evicts an entry) and is uploaded into the array with a
 *     copy from pageable host memory on every call, so the call returns only
 *     after the driver has staged those bytes. */
#define BA_STATIC_SCRATCH_BYTES ((size_t)8 << 20)
BA_API ba_status ba_fused_fwd_noalloc(const ba_problem* p, void* o, void* ob, float* lse,
                                      ba_stream_t stream);

/* Backward (steps a5-a8; not on the pages): gradients of sum(O * dO) through
 * both components, recomputed from the merged LSE.
 *   o, ob, lse      the outputs of ba_fused_fwd
 *   dout, doutb     bf16, layouts of o and ob
 *   dq, dk, dv      bf16 [S, Hq, d], [S, Hkv, d], [S, Hkv, d]   (written)
 *   dqb, dkb, dvb   bf16 [Nb, B, Hq, d], [Nb, B, Hkv, d] x2      (written)
 * Needs ba_workspace_size(p, BA_WS_BWD) bytes of workspace (fp32 dQ
 * accumulator, D = rowsum(dO * O), plan). */
BA_API ba_status ba_bwd(const ba_problem* p, const void* o, const void* ob, const float* lse,
                 const void* dout, const void* doutb, void* dq, void* dk, void* dv,
                 void* dqb, void* dkb, void* dvb, ba_stream_t stream);

/* Plan cache (no counterpart on the pages; the plan is this library's own
 * work list).  Every entry point plans on the host from cu_seqlens_h and
 * anchors_h: the zigzag split, row tiles, their order and the key tiles of the
 * backward.  Plans are cached, keyed by the problem's sizes (S, ndoc, Hq,
 * Hkv, d, Nb, B, mode, R, window) and the contents of cu_seqlens_h, anchors_h
 * and (bitmask mode) branch_mask_h, so
 * the forward and backward of one packing, and later steps over the same
 * packing, plan once.  The cache keeps the 16 most recently used plans.  A
 * cached plan also keeps a page-locked copy of the bytes a device call
 * uploads into the workspace (made by the first device call that uses it), so
 * that upload is one asynchronous copy; an entry's page-locked copy is freed
 * only after every upload from it has finished.
 *
 * ba_plan_prepare builds (or finds) the plan of a problem without touching a
 * GPU and reports, in *build_ms (may be NULL), how long building it took on
 * the host.  It returns BA_ERR_INVALID_ARG / BA_ERR_UNSUPPORTED as
 * ba_plan_stats does.  Host only; reads cu_seqlens_h and anchors_h. */
BA_API ba_status ba_plan_prepare(const ba_problem* p, double* build_ms);

/* Drops every cached plan (an entry still in use by a call in progress goes
 * when that call returns).  Freeing a page-locked copy waits for the uploads
 * from it to finish. */
BA_API void ba_clear_cache(void);

/* Number of cached plans and the cache's hit and miss counts since the
 * library was loaded (any argument may be NULL).  Host only. */
BA_API void ba_plan_cache_stats(int64_t* entries, int64_t* hits, int64_t* misses);

/* Static description of a status code. */
BA_API const char* ba_status_string(ba_status s);

/* Synchronises `stream`, then reports (and clears) the device error word of
 * the current device: BA_ERR_TIMEOUT if a bounded wait expired, BA_ERR_CUDA
 * if the synchronisation failed, else BA_OK. */
BA_API ba_status ba_sync_status(ba_stream_t stream);

/* Failure detection (no counterpart on the pages).  Every wait inside the
 * library's kernels is bounded: when it expires the kernel records where it
 * gave up in the device error word, lets its own copies and tensor-core work
 * in flight finish (a separate, fixed bound of about 2 s), frees its tensor
 * memory and returns; the CUDA context stays usable.
 * ba_set_wait_limit sets the bound, in SM clock cycles, that later launches
 * use for their waits (<= 0 restores the default, about 2 s).  Shortening it
 * to a few hundred cycles makes ordinary waits expire, which is how the
 * failure path is tested; results of launches that expired are garbage.  Not
 * thread-safe with respect to concurrent calls of the library. */
BA_API void ba_set_wait_limit(long long cycles);

/* Launches a one-thread check of the bounded wait on `stream`: it waits, with
 * the current limit, on a barrier that nothing arrives on.  After it,
 * ba_sync_status() must report BA_ERR_TIMEOUT with an error word naming
 * kernel 4, role 0, wait site 1.  Returns BA_OK if the check was enqueued. */
BA_API ba_status ba_check_bounded_wait(ba_stream_t stream);

/* The device error word that the last failing ba_sync_status() reported
 * (0 if none): bit 31 set for an expired bounded wait, bits 24-30 the kernel
 * (1 forward, 2 dQ pass, 3 dK/dV pass, 4 the check above, 5 the branch-key
 * backward), bits 16-23 the
 * role (0 TMA producer,
 * 1 MMA issuer, 2 softmax / gradient threads), bits 8-15 the wait site in that
 * role, bit 0 the phase parity waited for.  For diagnosing a timeout. */
BA_API uint32_t ba_last_error_word(void);

/* Planner statistics for a problem (host only, no GPU needed): number of row
 * tiles, (row tile, key tile) pairs the forward kernel visits per query head,
 * and the exact count of visible (row, key) pairs per query head.  Returns
 * BA_ERR_INVALID_ARG for an invalid problem. */
BA_API ba_status ba_plan_stats(const ba_problem* p, int64_t* n_row_tiles, int64_t* n_tile_pairs,
                        int64_t* n_visible_pairs);

/* Kernel timing for benchmarks (no counterpart on the pages).  While enabled,
 * every kernel the library launches is bracketed by two CUDA events recorded
 * on the launching stream; the library creates and destroys these events
 * itself (host-side handles, no device memory).  Enabling and disabling are
 * not thread-safe with respect to concurrent calls of the library. */
BA_API void ba_profile_enable(int on);

/* Waits for the recorded events, sums the elapsed time per kernel name, writes
 * up to `cap` entries (name, total milliseconds, number of launches) and
 * forgets the records.  Returns the number of distinct kernel names (may be
 * larger than cap), or -1 if an event query failed.  Names are static strings
 * owned by the library. */
BA_API int ba_profile_collect(const char** names, double* total_ms, int* launches, int cap);

/* Work per virtual rank of the zigzag split (host only, no GPU needed):
 * writes, for r < min(cap, R), the number of (row tile, main key tile) pairs
 * of the row tiles owned by virtual rank r, and returns R (or a negative
 * status for an invalid problem).  A row tile is owned by the rank whose
 * zigzag chunk holds its first row.  With the zigzag split these totals are
 * nearly equal (the pages: the split balances the triangular causal work). */
BA_API int ba_plan_rank_work(const ba_problem* p, int64_t* pairs, int cap);

/* Work items of the fused / main forward (host only, no GPU needed): each
 * item is a pair of consecutive row tiles of one document (tile indices in
 * position order; the second is -1 when a document has an odd tile left),
 * which share the document's main key tiles, in the order the kernel claims
 * them (most key tiles first).  Writes min(cap, n) pairs as 2 x int32 each to
 * `tiles` (may be NULL) and returns n, the number of pairs, or a negative
 * status for an invalid problem.  Each forward work item is one pair times
 * one query head. */
BA_API int64_t ba_plan_fwd_pairs(const ba_problem* p, int32_t* tiles, int64_t cap);

#ifdef __cplusplus
}
#endif
#endif /* BA_B200_H */
