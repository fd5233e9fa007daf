/*
 * spava.h -- C ABI of the B200 (sm_100a) approximate-attention prefill layer
 * of Spava / APB-V, with all 2H ZigZag virtual hosts emulated on one GPU.
 *
 * Sources (page title and the part of the page that defines each call):
 *   [SC] "Spava: Accelerating Long-Video Understanding via Sequence-
 *        Parallelism-aware Approximate Attention" (sciencestack.ai),
 *        TL;DR and Fig. 2-5 captions.
 *   [PR] "APB-V: Accelerating Long-Video Understanding via Sequence-
 *        Parallelism-aware Approximate Attention" (pith.science review):
 *        "What carries the argument", "Core claim", referee major comment 1,
 *        minor comment 2, "Axiom & Free-Parameter Ledger".
 *   [GN] "Technische Samenvatting: APB-V" (gist.science, nl), Methodologie.
 *
 * Sequence and layouts.  The token sequence is
 *     A | B^(0) | B^(1) | ... | B^(V-1) | B_qr,     V = 2H virtual hosts,
 * an anchor block of la tokens, V context blocks of L_h tokens and a query
 * block of lq tokens; n = la + sum L_h + lq.  Virtual hosts h and 2H-1-h form
 * ZigZag pairs on the pages' physical hosts; on one GPU the pairing only
 * shapes the work order.  All tensors are contiguous, row-major:
 *     Q, O       [n, Hq,  d]  bf16
 *     K, V       [n, Hkv, d]  bf16
 *     lse        [Hq, n]      fp32, natural log of sum exp(scale * q.k)
 *     qsum       [Hkv, d]     fp32
 *     scores     [Hkv, S]     fp32, S = sum_{h<V-1} L_h (block h at column
 *                             start_h - la)
 *     idx        [V-1, Hkv, lp] int32, block-relative, ascending; entries past
 *                             lp_eff(h) = min(lp, L_h) are -1
 *     Kp, Vp     [P, Hkv, d]  bf16, P = sum_{h<V-1} lp_eff(h); block h's rows
 *                             start at row off_h = sum_{j<h} lp_eff(j)
 *     O_part     [V, lq, Hq, d] fp32, lse_part [V, Hq, lq] fp32
 * Query head g reads KV head g / (Hq/Hkv).
 *
 * Ownership and errors.  Every tensor pointer is device memory owned by the
 * caller (the library allocates nothing and keeps no per-call state).  Q, K,
 * V, Kp, Vp and O must be 16-byte aligned.  Calls are asynchronous on
 * `stream`.  Argument errors are returned before anything is launched.  A
 * failed launch returns SPAVA_ERR_CUDA.  The attention kernel bounds every
 * wait; if one gives up it records a device error word that
 * spava_device_error() reports (the results of that call are then invalid).
 */
#ifndef SPAVA_H_
#define SPAVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* spava_stream_t;

typedef enum {
  SPAVA_OK = 0,
  SPAVA_ERR_INVALID_ARG = 1, /* bad shape, null or misaligned pointer       */
  SPAVA_ERR_UNSUPPORTED = 2, /* valid but outside this library's limits     */
  SPAVA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
  SPAVA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed           */
  SPAVA_ERR_DEVICE = 5       /* a kernel reported a device-side failure     */
} spava_status_t;

#define SPAVA_MAX_HOSTS 16   /* H; V = 2H <= 32 virtual hosts */

/* Passing-key selectors (spava_problem_t.score_kind).  LINEAR is the pages'
 * rule (Q_qr K^(h)T summed per key); the other two are the alternatives the
 * review asks to compare it with ([PR] major comment 1, "What would settle
 * it"); they change which keys pass, nothing else. */
#define SPAVA_SCORE_LINEAR 0   /* sum over query-block rows of scale <q, k>              */
#define SPAVA_SCORE_SOFTMAX 1  /* sum over query-block rows of softmax over the block    */
#define SPAVA_SCORE_CONTEXT 2  /* sum over the block's own rows of their causal softmax
                                  within the block (cumulative context attention)        */

/* One layer's problem ([SC] Fig. 2 caption; [GN] Context Splitting;
 * [PR] ledger for la and lp). */
typedef struct {
  int32_t num_hosts;         /* H >= 1 physical hosts; V = 2H context blocks */
  int32_t anchor_len;        /* la >= 0 (0 = the "w/o anchor" ablation)      */
  const int32_t* block_lens; /* HOST array of 2H lengths, each >= 1          */
  int32_t query_len;         /* lq >= 1                                       */
  int32_t lp;                /* passing length >= 0 (0 = "w/o passing");
                                clamped per block to min(lp, L_h)            */
  int32_t num_q_heads;       /* Hq >= 1                                       */
  int32_t num_kv_heads;      /* Hkv >= 1, Hq % Hkv == 0                       */
  int32_t head_dim;          /* d in {64, 128}                                */
  float softmax_scale;       /* <= 0 selects 1/sqrt(d)                        */
  int32_t score_kind;        /* SPAVA_SCORE_*; 0 = the pages' selector        */
  uint32_t host_mask;        /* 0 = every virtual host (the whole layer on one
                                GPU).  Otherwise the virtual hosts this caller
                                computes, bit h for host h (bits >= V must be
                                0): the compression of block h (h < V-1), the
                                context rows of block h and host h's query
                                partial; the anchor rows go with bit 0.  This
                                is the pages' own split of the 2H virtual
                                hosts over GPUs ([SC] Fig. 2 and Fig. 4
                                captions: GPU p holds hosts p and 2H-1-p; [PR]
                                "What carries the argument": the passing
                                blocks are all-gathered across hosts): each
                                GPU runs spava_compress and spava_attn_fwd
                                with its mask, the caller exchanges the Kp/Vp
                                rows and the query partials between the GPUs,
                                and spava_lse_merge merges all V partials.
                                spava_compress, spava_attn_fwd,
                                spava_problem_sizes and spava_lse_merge
                                accept a partial mask (lse_merge always merges
                                all V partials); every other call returns
                                SPAVA_ERR_UNSUPPORTED for it.                 */
} spava_problem_t;

/* Derived sizes, filled by spava_problem_sizes().  attn_pairs, attn_flops and
 * attn_tiles count the rows host_mask selects. */
typedef struct {
  int64_t seq_len;        /* n                                               */
  int64_t query_start;    /* la + sum L_h                                     */
  int64_t score_cols;     /* S = sum_{h<V-1} L_h                              */
  int64_t passing_rows;   /* P = sum_{h<V-1} min(lp, L_h)                     */
  int64_t attn_pairs;     /* visible (row, key) pairs per query head          */
  double attn_flops;      /* 4 * d * Hq * attn_pairs                          */
  int64_t attn_tiles;     /* 128-row work items of the attention launch       */
  size_t workspace_bytes; /* what spava_layer_fwd needs                       */
} spava_sizes_t;

/* Check a problem and fill its derived sizes.  No CUDA call. */
spava_status_t spava_problem_sizes(const spava_problem_t* prob, spava_sizes_t* out);

/* Workspace spava_layer_fwd needs (bytes). No CUDA call. */
spava_status_t spava_workspace_size(const spava_problem_t* prob, size_t* bytes);

/* Step 1, KV importance ([SC] Fig. 5 caption: Q_qr K^(h)T estimates KV
 * importance; [PR] "What carries the argument").  The score of key j of
 * block h < V-1 for KV head kv is the sum, over the query block's rows i and
 * the query heads g of that KV head, of scale * <q_ig, k_j>.  By linearity it
 * equals <qsum_kv, k_j> with qsum_kv = scale * sum_{i,g} q_ig, which this
 * call writes to `qsum` and then streams K once to form `scores`. */
spava_status_t spava_score(const spava_problem_t* prob, const void* Q,
                           const void* K, float* qsum, float* scores,
                           spava_stream_t stream);

/* Step 1 under the selector prob->score_kind (any of SPAVA_SCORE_*), into
 * `scores` (same layout as spava_score).  The two alternatives need two
 * passes: the attention kernel computes every scoring row's log-normaliser
 * over the block (softmax: the query block's rows over block h; context:
 * block h's rows, causally over its own keys), then a tensor-core kernel
 * sums exp(scale <q, k> - lse) per key.  `workspace` (>= spava_workspace_size
 * bytes for this problem, 256-byte aligned) holds the first pass's output.
 * spava_score itself returns SPAVA_ERR_UNSUPPORTED for these selectors. */
spava_status_t spava_score_variant(const spava_problem_t* prob, const void* Q,
                                   const void* K, float* scores, void* workspace,
                                   size_t ws_bytes, spava_stream_t stream);

/* Step 2, top-lp per block and KV head ([PR] "What carries the argument":
 * each context block compressed to its top-lp key-value pairs).  Larger
 * score first; equal scores keep the lower index; -0.0 equals +0.0.
 * Writes `idx` (ascending, -1 padded).  One cluster of CTAs per (block, KV
 * head) selects across its slices of the scores (the fused compression's
 * select); blocks too long for that use one CTA each. */
spava_status_t spava_select_topk(const spava_problem_t* prob,
                                 const float* scores, int32_t* idx,
                                 spava_stream_t stream);

/* Step 3, the passing blocks of all hosts compacted into Kp, Vp: row
 * off_h + t of KV head kv is key start_h + idx[h][kv][t].  This in-HBM
 * gather replaces the pages' cross-host all-gather ([PR] "What carries the
 * argument"; [SC] Fig. 2 caption): host h reads the prefix of off_h rows. */
spava_status_t spava_gather_passing(const spava_problem_t* prob, const void* K,
                                    const void* V, const int32_t* idx,
                                    void* Kp, void* Vp, spava_stream_t stream);

/* Steps 1-3 fused in two launches: the same qsum, scores, idx, Kp and Vp as
 * spava_score + spava_select_topk + spava_gather_passing ([SC] Fig. 5 caption:
 * importance estimation, then the essential KVs).  The query-block sum (the
 * scoring stage's own kernel, so both calls see the same qsum bits), then,
 * started at once as its programmatic dependent, one cluster of CTAs per
 * (block, KV head) -- 8, or 4 when 8-CTA clusters would not fit the GPU in one
 * wave -- streams K^(h) once (each CTA one slice), selects across the cluster
 * by exchanging radix counts in distributed shared memory and copies the kept
 * rows, an equal share per CTA.  Every block length must be <= 24576
 * (SPAVA_ERR_UNSUPPORTED otherwise; the separate stage calls have no such
 * limit).  With lp = 0 it does nothing.  With a partial host_mask only the
 * selected blocks are compressed: their scores, idx and Kp/Vp rows (at their
 * offsets off_h of the full buffer) are written, and qsum if any block is
 * selected; nothing else. */
spava_status_t spava_compress(const spava_problem_t* prob, const void* Q,
                              const void* K, const void* V, float* qsum,
                              float* scores, int32_t* idx, void* Kp, void* Vp,
                              spava_stream_t stream);

/* Step 4, one launch of causal attention over mixed key segments ([PR]
 * minor comment 2: Eq. 4 key list [K_a, K_p, K^(h)]; [SC] Fig. 3 fused
 * context and query forward; Fig. 4 load balancing):
 *   anchor rows r < la: keys 0..r;
 *   context rows of host h: A, Kp rows [0, off_h), and B^(h) keys up to r;
 *   query rows, partial of host h: B^(h) (host 0 also A and B_qr up to r).
 * Writes O / lse for anchor and context rows, and O_part / lse_part.  With a
 * partial host_mask only the selected hosts' rows and partials are written
 * (context rows of host h still read Kp rows [0, off_h), which the caller must
 * have filled with the other hosts' passing rows). */
spava_status_t spava_attn_fwd(const spava_problem_t* prob, const void* Q,
                              const void* K, const void* V, const void* Kp,
                              const void* Vp, void* O, float* lse,
                              float* O_part, float* lse_part,
                              spava_stream_t stream);

/* Step 5, merge of the query partials ([PR] ledger: lse merging is exact;
 * [GN] fused context and query forward): lse = log sum_h exp(lse_h),
 * O = sum_h exp(lse_h - lse) O_h, written to the query rows of O and lse. */
spava_status_t spava_lse_merge(const spava_problem_t* prob, const float* O_part,
                               const float* lse_part, void* O, float* lse,
                               spava_stream_t stream);

/* The whole layer: steps 1-5 in order on `stream`, with every intermediate
 * carved from `workspace` (device memory, >= spava_workspace_size bytes,
 * 256-byte aligned).  Outputs O [n, Hq, d] bf16 and lse [Hq, n] fp32.
 * Three launches: the compression of steps 1-3 (query sum, then scores,
 * selection and gather in one cluster launch), then attention with
 * the merge of step 5 in the same launch (the last of the V partial CTAs of
 * a query tile pair merges it; [SC] Fig. 5 caption: the passing-block
 * exchange and the merge overlap the attention).  The attention launch may
 * start while the compression runs (programmatic dependent launch): it waits
 * for it only before reading the passing buffer.  The work list is checked
 * before anything is launched (SPAVA_ERR_UNSUPPORTED: more than 6144 work
 * items of two 128-row tiles).  Blocks longer than 24576 keys fall back to
 * the three stage kernels of steps 1-3, and so do the selectors other than
 * SPAVA_SCORE_LINEAR (spava_score_variant, top-lp, gather). */
spava_status_t spava_layer_fwd(const spava_problem_t* prob, const void* Q,
                               const void* K, const void* V, void* O,
                               float* lse, void* workspace, size_t ws_bytes,
                               spava_stream_t stream);

/* The whole layer, like spava_layer_fwd, for callers that cannot allocate
 * device memory: code that only receives input and output pointers from a
 * host framework which owns the device allocator (a plugin or operator
 * interface), or whose memory budget leaves no room to reserve a separate
 * workspace, and so cannot hand this library a workspace.  The pages describe
 * no such entry; it has no counterpart in the paper.
 *
 * The intermediates live instead in one fixed array of 64 MiB inside this
 * library: every GPU that loads the library holds it until the process
 * exits.  A problem whose workspace (spava_workspace_size) exceeds 64 MiB is
 * rejected with SPAVA_ERR_WORKSPACE before anything is launched.  The call
 * allocates no device memory.  Its first call on a device looks up the
 * array's device address on that device (cudaGetSymbolAddress); make that
 * first call before any stream capture.  That address stays valid until the
 * device is reset: after cudaDeviceReset the library holds a stale address,
 * so a process that resets a device must not call this entry on it again.
 * All calls on a device share the array and it keeps the last call's
 * contents (nothing in it needs to start at zero: each call writes every
 * byte it reads, and zeroes its merge counters itself).  Calls whose work
 * overlaps on the GPU (other streams, other host threads) race on the array
 * and give wrong results: serialise them. */
spava_status_t spava_layer_fwd_noalloc(const spava_problem_t* prob, const void* Q,
                                       const void* K, const void* V, void* O,
                                       float* lse, spava_stream_t stream);

/* Device-side error word of the current device (0 = none); synchronizes the
 * device, then clears the word.  Bit 0: a bounded wait in the attention
 * kernel gave up; bit 1: the gather met an index outside its block. */
spava_status_t spava_device_error(uint32_t* code);

/* Test hook, not part of the layer: one thread of a one-CTA kernel waits on
 * an mbarrier that nothing completes, through the same bounded waits the
 * kernels use, with a limit of limit_ns (0 < limit_ns <= 4 s).  The wait gives
 * up, raises the CTA's abort flag and sets bit 0 of the device error word;
 * then the drain wait gives up too.  out (device, 4 x int64): the wait's
 * result (0), the abort flag (1), the drain's result (0), the nanoseconds
 * both took.  The context stays usable. */
spava_status_t spava_debug_wait_timeout(int64_t* out, uint64_t limit_ns, spava_stream_t stream);

/* Test hook, not part of the layer: spava_attn_fwd with one key tile left
 * unloaded.  The producer of every CTA skips its key tile skip_k_tile (>= 0),
 * and every wait of the launch gives up after limit_ns (0 < limit_ns <= 4 s)
 * instead of 4 s, so the CTAs that reach that tile take the kernel's abort
 * path: the MMA warp's wait runs out, the abort flag stops the other roles,
 * the copies and MMAs in flight are drained (bounded), TMEM is freed and bit
 * 0 of the device error word is set.  The outputs of the call are invalid;
 * the context stays usable. */
spava_status_t spava_debug_attn_abort(const spava_problem_t* prob, const void* Q, const void* K,
                                      const void* V, const void* Kp, const void* Vp, void* O, float* lse,
                                      float* O_part, float* lse_part, int32_t skip_k_tile,
                                      uint64_t limit_ns, spava_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* spava_status_string(spava_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SPAVA_H_ */
