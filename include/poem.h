/*
 * poem.h -- C ABI of libpoem, a B200 (sm_100a) implementation of the hot path of
 * POEM-style output-relative block-sparse attention prefill.
 *
 * The method (Wu et al., "POEM: Output-Relative Block-Sparse Attention for
 * Long-Context Prefilling", as summarised in the reading note "Attention
 * deletion error", Section 4.1 and Equations (3)-(4)): for one query and one
 * head, a visible key block b has softmax mass m_b and attention-weighted mean
 * value v_b; the dense output is o = sum_b m_b v_b; dropping a set D of blocks
 * with mass delta < 1 gives o~ = (o - sum_D m_b v_b) / (1 - delta), and
 *     || o - o~ || <= sum_{b in D} I_b / (1 - delta),   I_b = m_b || v_b - o ||.
 *
 * Three calls form one prefill layer, all asynchronous on the caller's stream:
 *   poem_score   exact m_b and I_b on a strided subset of the queries of each
 *                query tile, max-aggregated per (head, tile, visible block)
 *   poem_select  mandatory blocks + blocks in descending I_b until the bound
 *                above is <= tau; CSR block list per (head, tile)
 *   bsa_fwd      causal GQA block-sparse attention over the listed blocks
 *   bsa_fwd_grouped  the same, with two query heads of a KV group sharing K/V tiles
 *
 * Conventions for every entry point
 *   - All pointers are device pointers unless stated, 16-byte aligned.  The
 *     caller owns every buffer; the library never allocates device memory and
 *     never synchronises a stream (poem_check excepted).
 *   - q, k, v, o hold bf16 values (poem_bf16 = raw bf16 bits); the head
 *     dimension is contiguous; token and head strides are given in elements
 *     and must be multiples of 8 (16 bytes).
 *   - Each call validates its arguments on the host before any launch and
 *     returns POEM_ERR_INVALID_ARG / POEM_ERR_UNSUPPORTED without launching.
 *   - Conditions found on the device (a bounded wait that gave up, a block id
 *     outside the causal range, a col_idx buffer that is too small) are OR-ed
 *     into an error word at the start of the call's workspace; poem_check
 *     reads and clears it.  Workspaces must be zero-filled once before first
 *     use (the library keeps the error word clear otherwise).
 *   - Supported in this version: head_dim in {64, 128}, block in {64, 128},
 *     n_sample in {16} dividing block, n_tokens % block == 0,
 *     n_q_heads % n_kv_heads == 0.  Anything else: POEM_ERR_UNSUPPORTED.
 *   - There is no CPU fallback and no other backend.
 */
#ifndef POEM_H
#define POEM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t poem_bf16; /* raw bfloat16 bit pattern */

typedef enum poem_status {
  POEM_OK = 0,
  POEM_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, tau < 0 or NaN ...   */
  POEM_ERR_UNSUPPORTED = 2, /* valid but not implemented (head_dim, block, n_sample)    */
  POEM_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed; see poem_last_error  */
  POEM_ERR_TIMEOUT = 4,     /* device: a bounded wait gave up (reported by poem_check)  */
  POEM_ERR_CAPACITY = 5,    /* col_capacity too small (device: reported by poem_check)  */
  POEM_ERR_WORKSPACE = 6,   /* ws_bytes smaller than poem_workspace_size reports        */
  POEM_ERR_BAD_LIST = 7,    /* device: a listed block id outside 0..tile (skipped)      */
  POEM_ERR_BOUNDS = 8       /* device, debug build only: an index outside its buffer   */
} poem_status;

/*
 * Problem shape of one attention layer.
 *   q: [n_tokens, n_q_heads, head_dim], element (t, h, c) at
 *      q[t*q_stride_tok + h*q_stride_head + c]; o like q with o_stride_*.
 *   k, v: [q_offset + n_tokens, n_kv_heads, head_dim] with kv_stride_*.
 *   Query head h reads KV head h / (n_q_heads / n_kv_heads) (GQA).
 *   block: key block size = query tile size B; T = n_tokens / B query tiles.
 *   q_offset: position of the first query among the keys (chunked prefill: the
 *      queries are the last n_tokens of the q_offset + n_tokens visible tokens;
 *      0 for a whole prefill).  Must be a multiple of block.  Query tile i holds
 *      the queries at key positions q_offset + iB .. q_offset + iB + B - 1, is
 *      global tile t0 + i (t0 = q_offset / B) and sees key blocks 0..t0+i
 *      (causal).
 *   n_sample: S sampled queries per tile for scoring, rows iB + j*(B/S).
 *   softmax_scale: logit scale; 0 selects 1/sqrt(head_dim).
 * Per-(head, query tile, visible block) arrays (scores, estimates) hold row
 * (h, i) at h*E + i*t0 + i*(i+1)/2, E = T*t0 + T*(T+1)/2 entries per head
 * (t0 = 0: the packed lower triangle h*T*(T+1)/2 + i*(i+1)/2).
 */
typedef struct poem_shape {
  int32_t n_tokens;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t block;
  int32_t n_sample;
  float softmax_scale;
  int32_t q_offset;
  int64_t q_stride_tok, q_stride_head;
  int64_t kv_stride_tok, kv_stride_head;
  int64_t o_stride_tok, o_stride_head;
} poem_shape;

/*
 * Workspace bytes each call needs for this shape (any output pointer may be
 * NULL).  Every workspace starts with a 256-byte header holding the error word.
 */
poem_status poem_workspace_size(const poem_shape* shape, size_t* score_bytes, size_t* select_bytes,
                                size_t* fwd_bytes);

/*
 * poem_score -- exact block scores on the sampled queries.
 * Section 4.1 (m_b, v_b, o) and Equation (4) (I_b = m_b ||v_b - o||) of the
 * reading note; sampling (S strided queries per tile) and max-aggregation are
 * this library's choices.
 * For each query head h, query tile i (global tile g = t0 + i) and visible
 * block b <= g:
 *   I_hat[h, i, b] = max_j I_b(q_j),  m_hat[h, i, b] = max_j m_b(q_j)
 * over the sampled queries q_j = iB + j*(B/S), j = 0..S-1, with dense causal
 * softmax attention of q_j over keys 0..q_j.
 * Outputs (fp32, packed per (head, query tile) row, see poem_shape): entry
 *   (h, i, b) at h*E + i*t0 + i*(i+1)/2 + b; n_q_heads*E entries each.
 * ws: at least score_bytes (holds per-sampled-query dense outputs and
 *   log-sum-exps between the two passes).
 */
poem_status poem_score(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                       float* I_hat, float* m_hat, void* ws, size_t ws_bytes, void* stream);

/*
 * poem_select -- threshold selection per (head, tile), Equation (4).
 * Row r = h*T + i; below, i stands for the row's global tile t0 + i (block ids
 * are global).  Mandatory: sink block 0, local block i-1 (i >= 1) and the
 * diagonal block i.  Candidates 1..i-2 are ranked by (I_hat desc, id asc) --
 * equal scores favour the smaller id, the convention of the "Block-Filtered
 * Long-Context Attention" page, Appendix "Block ordering".  With D_k the
 * candidates ranked k, k+1, ..., S_I = sum_{D_k} I_hat and S_m = sum_{D_k}
 * m_hat (fp64), the row keeps the top k for the smallest k with
 *     S_m < 1  and  S_I <= tau * (1 - S_m).
 * Shapes whose lists could exceed int32 offsets (n_q_heads*E > 2^31 - 1) are
 * POEM_ERR_UNSUPPORTED.
 * Outputs: row_ptr[n_q_heads*T + 1] (int32, exclusive scan of list lengths)
 *   and col_idx[row_ptr[r] .. row_ptr[r+1]) the kept ids of row r in
 *   ascending order.  col_capacity: entries available in col_idx; when the
 *   lists need more, col_idx holds a truncated prefix and POEM_ERR_CAPACITY is
 *   reported by poem_check (n_q_heads*E always suffices).
 * order (nullable): int32[n_q_heads*T], a work order for bsa_fwd -- rows grouped
 *   by KV head, longest list first, ties by row id.
 * tau: absolute bound on the per-query head-output error in V's units; must be
 *   finite and >= 0 (tau = 0 keeps every candidate with I_hat > 0).
 */
poem_status poem_select(const poem_shape* shape, const float* I_hat, const float* m_hat, float tau,
                        int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * poem_select_per_head -- poem_select with one tau per query head: the pages
 * calibrate retention thresholds offline for each head group; a caller passes
 * its calibrated values here (a group's value repeated over its heads).
 * tau_per_head: device array of n_q_heads floats, read by the kernel (so a
 * captured CUDA graph picks up new values without re-capture).  Entries must be
 * finite and >= 0; a bad entry makes its head's rows keep every candidate and
 * poem_check reports POEM_ERR_INVALID_ARG.  Outputs and workspace as poem_select.
 */
poem_status poem_select_per_head(const poem_shape* shape, const float* I_hat, const float* m_hat,
                                 const float* tau_per_head, int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                 int32_t* order, void* ws, size_t ws_bytes, void* stream);

/*
 * poem_select_mass_only -- the mass-only baseline at a matched budget: row r
 * keeps the mandatory blocks and the (ref_row_ptr[r+1] - ref_row_ptr[r] -
 * |mandatory|) candidates of largest m_hat (ties: smaller id).  Same outputs
 * and workspace as poem_select.  ref_row_ptr is a device pointer.
 */
poem_status poem_select_mass_only(const poem_shape* shape, const float* m_hat, const int32_t* ref_row_ptr,
                                  int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order,
                                  void* ws, size_t ws_bytes, void* stream);

/*
 * poem_select_ranked_budget -- fixed-budget ranking by any per-block score: row r
 * keeps the mandatory blocks and the (ref_row_ptr[r+1] - ref_row_ptr[r] -
 * |mandatory|) candidates of largest score (ties: smaller id).  With score =
 * m_hat this is poem_select_mass_only; with score = I_hat it is POEM's ranking
 * at a given block count, which compares selectors at matched budgets (the
 * evaluation the reading note's last section proposes).  score is packed
 * lower-triangular like poem_score's outputs.  Same outputs and workspace as
 * poem_select.
 */
poem_status poem_select_ranked_budget(const poem_shape* shape, const float* score, const int32_t* ref_row_ptr,
                                      int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order,
                                      void* ws, size_t ws_bytes, void* stream);

/*
 * poem_select_noalloc -- poem_select for callers that cannot allocate device
 * memory.  (An addition of this library; the method description has no
 * counterpart.)  Some callers own no allocator: a serving runtime that reserves
 * all device memory up front and must not let a library grow its footprint while
 * it serves, or a plug-in that is only handed pointers by its host.  This entry
 * point takes the same inputs and outputs as poem_select but no workspace: its
 * scratch lives in a fixed 8 MiB array inside the library's device image.  It
 * calls no allocator of any kind.
 *   - When the 8 MiB is committed: CUDA loads the array's device module on a
 *     device lazily, at the first poem_select_noalloc call made with that device
 *     current; from then on the device holds the 8 MiB until the process exits.
 *     A caller that reserves device memory up front makes one call (any valid
 *     shape) before its reservation, so that this first call cannot run out of
 *     memory.
 *   - Shapes whose selection scratch (poem_workspace_size's select_bytes) exceeds
 *     8 MiB are rejected with POEM_ERR_WORKSPACE (e.g. 32 heads x 256 tiles fits;
 *     32 heads x 1024 tiles does not).  Every refusal leaves a message in
 *     poem_last_error.
 *   - All calls share the array and each call overwrites it: calls whose kernels
 *     overlap on the GPU (other streams, other host threads) race; serialise them.
 *   - The first call on a device resolves the array's device address with that
 *     device current; make that first call before any stream capture.  After a
 *     device reset (cudaDeviceReset) the next call finds the old address gone and
 *     resolves it again.
 *   - There is no workspace error word to poll: a col_idx that is too small is
 *     seen by comparing row_ptr[n_q_heads*T] with col_capacity after the call.
 */
poem_status poem_select_noalloc(const poem_shape* shape, const float* I_hat, const float* m_hat, float tau,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int32_t* order,
                                void* stream);

/*
 * Practical POEM selector (reading note "Attention deletion error", the
 * paragraph on Equation (6) and Appendix B): the dense reference output and the
 * block outputs are estimated from pooled features, candidates are preselected
 * by mass, reranked by log mass + w * log deviation, and kept in that order
 * until the accumulated pooled mass reaches a threshold.  The pages print
 * neither the estimators nor w; this library's estimators are mean pooling:
 *   q~_{h,i}  mean of the B queries of tile i, head h
 *   k~_{g,b}, v~_{g,b}  means of the B keys / values of block b, KV head g
 *   m~[h, i, b] = softmax over b <= i of softmax_scale * <q~_{h,i}, k~_{g,b}>
 *   o~ = sum_b m~ v~_b,   d~[h, i, b] = || v~_b - o~ ||
 * (with one token per block and one query per tile these are the exact m_b and
 * ||v_b - o||).
 */

/* Workspace bytes of poem_score_pooled: a 256-byte header, then the fp32 means
 * q~ (row-major), k~ (channel-major), v~ (row- and channel-major). */
poem_status poem_pooled_workspace_size(const poem_shape* shape, size_t* pooled_bytes);

/*
 * poem_score_pooled -- m~ and d~ for every (head, tile, visible block).
 * Outputs (fp32, in poem_score's row layout): entry (h, i, b) at
 *   h*E + i*t0 + i*(i+1)/2 + b.  fp32 arithmetic throughout.
 * ws: at least pooled_bytes; holds the pooled means after the call.
 * n_sample is ignored.
 */
poem_status poem_score_pooled(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                              float* m_pool, float* d_pool, void* ws, size_t ws_bytes, void* stream);

/*
 * poem_select_practical -- two-stage selection per (head, tile) from m~, d~.
 * Row r = h*T + i (i below: the row's global tile t0 + i).  Mandatory: blocks
 * 0, i-1 (i >= 1) and i.  Candidates 1..i-2:
 *   stage 1: ranked by (m~ desc, id asc); the first ceil(rho * |Cand|) form the
 *            shortlist (rho in [0, 1]);
 *   stage 2: the shortlist ranked by (log m~ + w * log d~ desc, id asc), in
 *            fp64 with log 0 = -inf (w finite, >= 0);
 *   the row keeps the mandatory blocks and the shortest prefix of the stage-2
 *   order with  sum_{mandatory} m~ + sum_{prefix} m~ >= gamma  (fp64; the
 *   whole shortlist when the sum never reaches gamma).
 * Outputs, col_capacity, order and workspace: as poem_select (select_bytes).
 * NaN gamma, rho outside [0, 1] or a negative / non-finite w: INVALID_ARG.
 */
poem_status poem_select_practical(const poem_shape* shape, const float* m_pool, const float* d_pool, double w,
                                  double gamma, double rho, int32_t* row_ptr, int32_t* col_idx,
                                  int64_t col_capacity, int32_t* order, void* ws, size_t ws_bytes, void* stream);

/*
 * poem_select_practical_per_head -- poem_select_practical with one gamma per
 * query head (device array of n_q_heads floats, read by the kernel).  A NaN or
 * infinite entry keeps its head's whole shortlist and poem_check reports
 * POEM_ERR_INVALID_ARG.
 */
poem_status poem_select_practical_per_head(const poem_shape* shape, const float* m_pool, const float* d_pool, double w,
                                           const float* gamma_per_head, double rho, int32_t* row_ptr,
                                           int32_t* col_idx, int64_t col_capacity, int32_t* order, void* ws,
                                           size_t ws_bytes, void* stream);

/*
 * bsa_fwd -- causal GQA block-sparse attention forward.
 * Query t of head h in query tile i (key position q_offset + t, global tile
 * g = t0 + i) attends, with softmax, to the keys u <= q_offset + t whose
 * block is listed in col_idx[row_ptr[r] .. row_ptr[r+1]), r = h*T + i
 * (the renormalised output o~ of Section 4.1).  Lists must be ascending and
 * hold ids in 0..g; an id outside that range is skipped and reported as
 * POEM_ERR_BAD_LIST by poem_check.  A row with no visible key outputs 0 and
 * lse = -inf.
 * o: bf16 output with o_stride_*; lse (nullable): fp32 [n_q_heads, n_tokens],
 *   natural-log log-sum-exp of the scaled logits over the kept keys.
 * order (nullable): permutation of the rows giving the launch order; NULL
 *   selects KV-head-major, last tile first.
 */
poem_status bsa_fwd(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                    const int32_t* row_ptr, const int32_t* col_idx, const int32_t* order, poem_bf16* o,
                    float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * bsa_fwd_grouped -- the same computation and outputs as bsa_fwd (every row's
 * renormalised output over its own list, Section 4.1), scheduled so that two
 * query heads of one KV group share K/V tiles: one CTA takes query heads
 * 2p, 2p + 1 of a group at one query tile and walks the union of their two
 * lists, loading each block's K and V once for both heads; each head runs its
 * attention only on the blocks of its own list.  Work order: KV head major,
 * last tile first (no order argument).  Arguments, list rules, errors and
 * workspace as bsa_fwd.
 * NOT the fast path: it halves the K/V traffic from L2 but is slower than
 * bsa_fwd (on the Llama-shaped 128K layer 136.0 vs 123.2 ms on the exact lists,
 * 35.8 vs 30.7 ms on the practical lists); it is kept as a comparison schedule
 * for the per-KV-group union lists.  Use bsa_fwd.
 */
poem_status bsa_fwd_grouped(const poem_shape* shape, const poem_bf16* q, const poem_bf16* k, const poem_bf16* v,
                            const int32_t* row_ptr, const int32_t* col_idx, poem_bf16* o, float* lse, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * Synchronise `stream`, read and clear the error word at the start of `ws`
 * (a workspace passed to one of the calls above) and map it to a status:
 * POEM_ERR_TIMEOUT, POEM_ERR_BAD_LIST, POEM_ERR_CAPACITY, POEM_ERR_INVALID_ARG
 * (a bad per-head threshold), POEM_ERR_BOUNDS (a failed bounds check of the
 * debug build, see below), or POEM_OK.
 *
 * Debug build: the library compiled with -DPOEM_CHECKS (libpoem_checks.so, built
 * by the package's build script) adds device-side bounds checks on the packed
 * score writes, the sampled-query workspace and the selection scratch; an index
 * outside its buffer skips the access and sets POEM_ERR_BOUNDS.  Release builds
 * compile the checks away.
 */
poem_status poem_check(void* stream, void* ws);

/* Upper bound, in nanoseconds, of every on-device wait (default 2e9).  A
 * process-wide setting read at launch time. */
void poem_set_wait_limit_ns(uint64_t ns);

const char* poem_status_string(poem_status s);

/* Text of the last CUDA error seen by this thread (empty if none). */
const char* poem_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* POEM_H */
