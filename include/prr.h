/*
 * prr.h -- C ABI of the PRR decode-step library (sm_100a).
 *
 * PRR (Predict, Reuse, and Repair: Accelerating Dynamic Sparse Attention for
 * Long-Context LLM Decoding) removes the wait between block selection and attention
 * in dynamic sparse attention (DSA) decoding: an EMA of past selections predicts the
 * blocks, attention over the predicted blocks runs while the true top-K is being
 * selected, predicted blocks outside the true set are dropped, and the missed blocks
 * are repaired and merged through online-softmax statistics.  The result equals plain
 * top-K DSA attention whatever the prediction (PRR abstract; method summary;
 * contributions (1)-(3)).
 *
 * Conventions shared by every entry point
 *  - All array pointers are DEVICE pointers owned by the caller.  The library never
 *    allocates, frees or synchronises device memory; only prr_get_device_status
 *    synchronises (to read the status word back).
 *  - bf16 arrays are passed as uint16_t bit patterns.
 *  - NULL: every buffer a call takes is required (PRR_ERR_INVALID_ARG if NULL) except
 *    where its description says otherwise; with P = 0 (no speculation budget) the
 *    predicted-slot buffers (pred, pred_next, keep, part_m, part_l, part_O) may be
 *    NULL, and prr_speculate returns PRR_OK without doing anything.
 *  - Alignment: q where a call attends with it (prr_speculate, prr_repair_merge and
 *    both decode steps), and k_cache, v_cache, summ, part_O, out, k_new and v_new
 *    wherever a call takes them, start on a 16-byte boundary; otherwise the call
 *    returns PRR_ERR_INVALID_ARG before enqueuing anything.
 *  - Shapes (row-major, innermost last), with units = B*Hkv (B*Hq under
 *    PRR_SELECT_PER_HEAD), G = Hq/Hkv, maxnb = ceil(cap_tokens/bs):
 *      q            [B][Hq][d]               bf16   query of the step
 *      k_cache/v_cache [B][Hkv][cap_tokens][d] bf16 (16-byte aligned base), or a paged
 *                   pool [pages][Hkv][bs][d] with a block table (see prr_dims)
 *      seq_lens     [B]                      int32  tokens n in the cache, 1 <= n <= cap
 *      summ         [B][Hkv][maxnb][2][d]    bf16   per block: min row then max row
 *      ema          [B][Hkv][maxnb]          fp64   EMA state, starts at 0
 *      pred, pred_next [B][Hkv][P]           int32  ascending block ids, -1 when empty
 *      sel, missed  [B][Hkv][K]              int32  ascending block ids, -1 when empty
 *      n_missed     [B][Hkv]                 int32
 *      keep         [B][Hkv][P]              uint8  keep[j] = Pred_j in S_t
 *      part_m, part_l [B][Hq][P]             fp32   speculative partials, one per slot
 *      part_O       [B][Hq][P][d]            fp32
 *      out          [B][Hq][d]               fp32   attention output
 *      lse          [B][Hq]                  fp32   natural-log log-sum-exp of the logits
 *    Partials use base-2 logits: part_m = max_i scale*log2(e)*q.k_i over the block,
 *    part_l = sum_i 2^(logit_i - part_m), part_O = sum_i 2^(logit_i - part_m) v_i.
 *  - Supported shapes: d in {64, 128}; bs in {64, 128}; 1 <= G <= 8; 1 <= K <= 128;
 *    0 <= P <= 128; 1 <= cap_tokens <= 2^30; at most 65,535 selection units (B*Hkv, or
 *    B*Hq under PRR_SELECT_PER_HEAD); pages*Hkv below 2^31.  Others return
 *    PRR_ERR_SHAPE (prr_workspace_bytes returns 0).
 *  - Shared-memory ceilings on maxnb = ceil(cap_tokens/bs), checked before anything is
 *    enqueued (PRR_ERR_SHAPE beyond them), all within 227 KB per CTA:
 *    - the selection finisher keeps a unit's keys and bitmaps on chip, so
 *      prr_select_topk, prr_select_topk_static and prr_decode_step take maxnb up to
 *      19,715 blocks at d = 128 (34,800 at d = 64);
 *    - the predictor keeps a unit's fp64 EMA state on chip (7,232 bytes plus 8 per
 *      block plus 12 per 32 blocks), so prr_ema_predict takes maxnb up to 26,890
 *      blocks, and prr_decode_step the smaller of its two limits (19,715 at d = 128,
 *      26,890 at d = 64);
 *    - prr_decode_step_fused holds the same predictor state plus 1,080 bytes of its
 *      own (alignment slack and barriers), so it takes maxnb up to 26,760 blocks.
 *  - Errors: argument and shape checks happen on the host before anything is
 *    enqueued and return a prr_status.  A failed launch returns PRR_ERR_CUDA.
 *    Problems that only the device can see (a seq_len out of range, a malformed
 *    predicted list, a wait that timed out) set the status word in the workspace
 *    (first error wins) and never trap; read it with prr_get_device_status.  After a
 *    non-zero device status, re-initialise the workspace before the next call.
 *  - Calls are asynchronous on the given stream(s).  Two calls that share a
 *    workspace must not overlap on the GPU.
 */
#ifndef PRR_H
#define PRR_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PRR_OK = 0,
  PRR_ERR_INVALID_ARG = 1,   /* null pointer or misaligned buffer */
  PRR_ERR_SHAPE = 2,         /* unsupported or inconsistent dimensions */
  PRR_ERR_CAPACITY = 3,      /* workspace smaller than prr_workspace_bytes() */
  PRR_ERR_CUDA = 4,          /* a CUDA runtime call failed */
  PRR_ERR_DEVICE_STATUS = 5, /* prr_get_device_status found a device-side error */
  PRR_ERR_TIMEOUT = 6        /* reserved: a bounded wait gave up (device code 4) */
} prr_status;

/* Device status codes (the value prr_get_device_status stores in *code). */
#define PRR_DEV_OK 0
#define PRR_DEV_BAD_SEQ_LEN 1  /* seq_lens[b] < 1 or > cap_tokens (that sequence is skipped) */
#define PRR_DEV_BAD_PRED 2     /* predicted list entry out of range or not ascending */
#define PRR_DEV_BAD_MISSED 3   /* missed list entry out of range */
#define PRR_DEV_WAIT_TIMEOUT 4 /* a bounded wait for a TMA copy gave up */
#define PRR_DEV_BAD_RANGE 5    /* summary update range outside [0, cap_tokens] or longer than max_range_tokens, or a block-table entry outside [0, pages) */

typedef struct {
  int32_t B;          /* sequences */
  int32_t Hq;         /* query heads */
  int32_t Hkv;        /* KV heads (Hq % Hkv == 0) */
  int32_t d;          /* head dim */
  int32_t bs;         /* tokens per KV block */
  int32_t cap_tokens; /* KV capacity per (sequence, KV head) */
  int32_t K;          /* top-K blocks selected per (sequence, KV head) */
  int32_t P;          /* speculation budget: predicted blocks per (sequence, KV head) */
  double alpha;       /* EMA decay, 0 <= alpha <= 1 */
  float scale;        /* softmax scale applied to q.k (usually 1/sqrt(d)) */
  /* Block selector (the DSA method whose top-K PRR accelerates; PRR abstract: results
   * across representative DSA methods).  Zero-initialised dims give the default.
   *   PRR_SELECT_GROUP_SUM  one selection per KV head; block score = the sum over the
   *                         group's query heads of each head's Quest bound
   *   PRR_SELECT_GROUP_MAX  one selection per KV head; score = the largest of the
   *                         group's per-head bounds
   *   PRR_SELECT_PER_HEAD   every query head selects its own top-K with its own bound;
   *                         then a "unit" is a (sequence, query head) pair, and the
   *                         per-unit arrays below are [B][Hq][...] instead of
   *                         [B][Hkv][...] (summaries and KV stay per KV head).
   *   PRR_SELECT_REPRESENTATIVE  one selection per KV head; each block is represented by
   *                         n_rep of its own tokens (rep_offsets, below; InfLLM-style,
   *                         the InfLLM title is in PRR's reference list) and scores
   *                         sum_h sum_j q_h . k_rep_j over the group's query heads.
   *                         It reads the key cache, so only the decode steps take it;
   *                         prr_select_topk and prr_select_topk_static return
   *                         PRR_ERR_SHAPE for it. */
  int32_t selector;
  int32_t n_sink;     /* the first n_sink blocks are always selected (attention sinks), 0..2^22 */
  int32_t n_local;    /* the newest n_local blocks are always selected (local window), 0..2^22;
                       * the rest of the min(K, nb) budget goes to the best other blocks; when
                       * the forced blocks alone exceed it, sinks come first (lowest index
                       * first), then local blocks from the newest backwards */
  /* KV cache layout.  pages == 0 (block_table NULL): contiguous, k_cache / v_cache
   * [B][Hkv][cap_tokens][d].  pages > 0: paged (as in PagedAttention / vLLM and
   * FlashInfer serving, in PRR's reference list) -- k_cache / v_cache are pools of
   * `pages` pages [pages][Hkv][bs][d], one page holding one block of bs tokens of every
   * KV head, and block_table (device int32 [B][maxnb]) maps block j of sequence b to its
   * page.  cap_tokens stays the per-sequence capacity.  Only entries of blocks below a
   * sequence's length are read; an entry outside [0, pages) sets PRR_DEV_BAD_RANGE and
   * that block is not read. */
  int32_t pages;
  const int32_t* block_table;
  /* PRR_SELECT_REPRESENTATIVE only (the other selectors ignore them): n_rep (1..16)
   * representative tokens per block, and rep_offsets (device uint8
   * [B][Hkv][maxnb][n_rep]) their offsets inside the block, chosen when the block was
   * built.  An offset at or past a ragged tail's valid tokens stands for the block's
   * last valid token. */
  int32_t n_rep;
  const uint8_t* rep_offsets;
} prr_dims;

#define PRR_SELECT_GROUP_SUM 0
#define PRR_SELECT_GROUP_MAX 1
#define PRR_SELECT_PER_HEAD 2
#define PRR_SELECT_REPRESENTATIVE 3

/* Buffers of one decode step (see the shapes above). */
typedef struct {
  const uint16_t* q;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  const int32_t* seq_lens;
  uint16_t* summ;
  double* ema;
  const int32_t* pred;  /* Pred_t (read) */
  int32_t* pred_next;   /* Pred_{t+1} (written); must not alias pred */
  int32_t* sel;
  int32_t* missed;
  int32_t* n_missed;
  uint8_t* keep;
  float* part_m;
  float* part_l;
  float* part_O;
  float* out;
  float* lse;
  /* Optional, both or neither (NULL: the caller appended the step's token already).
   * The step's new token [B][Hkv][d] bf16 (16-byte aligned).  The step then appends it
   * itself: it writes the rows at position seq_lens[b] of the caches, works on
   * seq_lens[b] + 1 tokens and advances seq_lens[b] when it is done (a full cache sets
   * PRR_DEV_BAD_SEQ_LEN and skips that sequence).  prr_decode_step_fused does this
   * inside its one launch; prr_decode_step launches the append first. */
  const uint16_t* k_new;
  const uint16_t* v_new;
  /* Optional (NULL: off).  prr_decode_step_fused records, for every work item its CTAs
   * run, trace[4i..4i+3] = {start ns, end ns, (SM id << 32) | CTA, kind} (%globaltimer;
   * kind 1 selection chunk, 6 top-K finisher, 4 predictor update, 2 speculative block,
   * 3 repair item, 5 merge), i = the item's ticket.  Items: units*ceil(maxnb/C)
   * selection chunks (C blocks each: units*maxnb/512 rounded up to a multiple of 32,
   * clamped to [32, 128]), units finishers, units predictor updates, units*P
   * speculative slots, units*R repair items (R = min(K, max(4, ceil(1024/units)))) and
   * units*G merges; the tickets of a unit's repair items and merges follow its
   * speculative slots a few units later.  Items that did not run stay zero.  Size:
   * 4 * (the number of items) words. */
  unsigned long long* trace;
  /* Optional (NULL: off).  Eight counters the step adds to (atomically; the caller
   * zeroes them):  [0] units whose top-K came straight from the 32-block group tie
   * masks, [1] units whose top-K needed the search over the block keys, [2] units
   * that took every block (K_eff = nb), [3] speculative blocks attended, [4]
   * speculative blocks skipped because selection had already dropped them, [5]
   * repaired (missed) blocks attended, [6], [7] zero. */
  unsigned long long* stats;
} prr_step_buffers;

/* Events of one decode step.  fork, sel_done, spec_done and join are required (any
 * flags); they order the two streams.  The timing marks are optional (NULL to skip);
 * when given they must be created with timing enabled, and under stream capture they
 * become event-record nodes of the graph. */
typedef struct {
  cudaEvent_t fork;          /* select_stream -> spec_stream: start of the step */
  cudaEvent_t sel_done;      /* select_stream -> spec_stream: S_t is known (predictor may run) */
  cudaEvent_t spec_done;     /* spec_stream -> select_stream: speculative partials written */
  cudaEvent_t join;          /* spec_stream -> select_stream: end of the spec stream's work */
  cudaEvent_t t_begin;       /* select_stream: before selection */
  cudaEvent_t t_select_end;  /* select_stream: after selection */
  cudaEvent_t t_repair_end;  /* select_stream: after repair */
  cudaEvent_t t_combine_begin; /* select_stream: before the LSE merge (after its wait) */
  cudaEvent_t t_combine_end; /* select_stream: after the LSE merge */
  cudaEvent_t t_spec_begin;  /* spec_stream: before speculation */
  cudaEvent_t t_spec_end;    /* spec_stream: after speculation */
  cudaEvent_t t_ema_begin;   /* spec_stream: before the predictor */
  cudaEvent_t t_ema_end;     /* spec_stream: after the predictor */
} prr_step_events;

/* Library version (major*10000 + minor*100 + patch).  Library plumbing, like the
 * status, workspace and append calls below: no passage of the pages defines them. */
int prr_version(void);

/* Human-readable name of a status. */
const char* prr_status_string(prr_status s);

/* Bytes of workspace the calls below need for these dims (0 if the dims are
 * unsupported).  The workspace holds the status word, the selection tickets, one
 * 32-bit score key per block, one (max key, tie mask) summary per 32-block group, the
 * repair partials and the fused step's control words (two copies, one per parity). */
size_t prr_workspace_bytes(const prr_dims* dims);

/* Byte offset of a workspace word reserved for failure-detection tests.  A test may set
 * it to a non-zero int32 (with a plain copy into the workspace) to make
 * prr_decode_step_fused skip its selection chunks: no unit's top-K completes, so the
 * launch's end-of-step wait runs out after its one-second limit and the launch returns
 * with the device status PRR_DEV_WAIT_TIMEOUT, without a fault.  Leave it zero
 * otherwise; prr_workspace_init clears it. */
#define PRR_WS_TEST_SKIP_SELECTION_OFFSET 4

/* Zero-fill a workspace (required once before first use, and after a device error).
 * The kernels leave their tickets re-armed, so steady-state calls need no reset. */
prr_status prr_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream);

/* Wait for all work on the current device (cudaDeviceSynchronize, whatever streams the
 * calls ran on), then read the workspace status word into *code (0 = no error).
 * Returns PRR_OK if the code is 0, PRR_ERR_DEVICE_STATUS otherwise, PRR_ERR_CUDA if the
 * wait or the copy fails.  Not for use while a stream capture is in progress. */
prr_status prr_get_device_status(const void* ws, int32_t* code);

/* Write one new token per (sequence, KV head): k_new/v_new [B][Hkv][d] go to position
 * seq_lens[b] of the caches, then seq_lens[b] is incremented (a full cache leaves
 * seq_lens unchanged and sets PRR_DEV_BAD_SEQ_LEN).  The pages take the decode loop's
 * one-token-per-step cache growth as given; this is that step, not part of PRR. */
prr_status prr_append_kv(const prr_dims* dims, const uint16_t* k_new, const uint16_t* v_new,
                         int32_t* seq_lens, uint16_t* k_cache, uint16_t* v_cache, void* ws,
                         cudaStream_t stream);

/* Block key summaries (step a1).  For every sequence b and KV head, the summaries of
 * the blocks touched by tokens [tok_begin[b], tok_end[b]) become the per-channel
 * min/max over the block's tokens [block start, tok_end[b]): a range that starts
 * inside a block is folded into the stored summary of that block's earlier tokens.
 * tok_begin/tok_end are device int32 [B]; both NULL means "the token just appended":
 * [seq_lens[b]-1, seq_lens[b]).  max_range_tokens bounds tok_end-tok_begin over all
 * sequences (it sizes the grid); a longer range sets PRR_DEV_BAD_RANGE and leaves that
 * sequence's summaries as they were.  Summary per Quest (Query-Aware Sparsity for
 * Efficient Long-Context LLM Inference, in the PRR reference list). */
prr_status prr_update_summaries(const prr_dims* dims, const uint16_t* k_cache,
                                const int32_t* tok_begin, const int32_t* tok_end,
                                const int32_t* seq_lens, int32_t max_range_tokens, uint16_t* summ,
                                void* ws, cudaStream_t stream);

/* Block scoring + top-K (steps a2-a3).  For each (b, KV head): the score of every
 * block below nb = ceil(n/bs) is the sum over the G query heads of
 * sum_c max(q_hc*min_bc, q_hc*max_bc); sel = the min(K, nb) best blocks under (score
 * desc, block asc), written ascending; missed = sel \ pred ascending, n_missed its
 * size; keep[j] = (pred[j] in sel).  A predicted slot is active when 0 <= pred[j] < nb.
 * PRR abstract: the true selected set; method summary: repair only the missed blocks. */
prr_status prr_select_topk(const prr_dims* dims, const uint16_t* q, const uint16_t* summ,
                           const int32_t* seq_lens, const int32_t* pred, int32_t* sel,
                           int32_t* missed, int32_t* n_missed, uint8_t* keep, void* ws,
                           cudaStream_t stream);

/* EMA predictor (step a4).  If sel is not NULL: e_b <- alpha*e_b + (1-alpha)*[b in sel]
 * for every block b < nb (fp64, multiplies and add rounded separately).  Then
 * pred_next = the min(P, nb) best blocks under (e desc, block asc), ascending, -1
 * beyond.  With sel NULL the state is only read (the zero state predicts 0..P-1).
 * PRR abstract and contribution (1): a lightweight EMA-based predictor. */
prr_status prr_ema_predict(const prr_dims* dims, double* ema, const int32_t* sel,
                           const int32_t* seq_lens, int32_t* pred_next, void* ws,
                           cudaStream_t stream);

/* Speculative attention (step a5): one (m, l, O) partial per active predicted slot j
 * and query head, over the tokens of block pred[j] below n.  Inactive slots are left
 * untouched.  PRR abstract: attention over the predicted blocks while selection is
 * still running. */
prr_status prr_speculate(const prr_dims* dims, const uint16_t* q, const uint16_t* k_cache,
                         const uint16_t* v_cache, const int32_t* seq_lens, const int32_t* pred,
                         float* part_m, float* part_l, float* part_O, void* ws,
                         cudaStream_t stream);

/* Repair + merge (step a6): attention partials over the missed blocks, then the LSE
 * merge of the kept speculative partials (keep[j] = 1) and the repair partials:
 *   m* = max m_j, l* = sum l_j 2^(m_j-m*), out = sum O_j 2^(m_j-m*) / l*,
 *   lse = (m* + log2 l*) ln 2.
 * The speculative partials must come from prr_speculate on the same pred and q.
 * PRR method summary and contribution (3): fold the missed blocks into the partial
 * state with online-softmax statistics, no recomputation. */
prr_status prr_repair_merge(const prr_dims* dims, const uint16_t* q, const uint16_t* k_cache,
                            const uint16_t* v_cache, const int32_t* seq_lens,
                            const int32_t* missed, const int32_t* n_missed, const uint8_t* keep,
                            const int32_t* pred, const float* part_m, const float* part_l,
                            const float* part_O, float* out, float* lse, void* ws,
                            cudaStream_t stream);

/* One full decode step (a1-a7) after the caller appended the step's token:
 *   select_stream: [tail summary + scoring + top-K] -> repair -> (wait spec) LSE merge
 *   spec_stream:   speculation over buf->pred -> (wait selection) EMA predictor
 * Speculation runs while selection is in flight; the predictor for step t+1 runs while
 * the missed blocks are repaired and merged.  Selection, repair and merge are launched
 * at the highest stream priority, speculation and prediction at the lowest.  On return
 * the work is enqueued; select_stream waits for spec_stream at the end (event join), so
 * completion of select_stream means the step is done.  The caller swaps pred/pred_next
 * between steps.  No allocation and no synchronisation, so the step can be captured
 * into a CUDA graph (after one uncaptured call on the device).  PRR method summary:
 * speculation overlaps selection and is kept off the critical path. */
prr_status prr_decode_step(const prr_dims* dims, const prr_step_buffers* buf, void* ws,
                           size_t ws_bytes, cudaStream_t select_stream, cudaStream_t spec_stream,
                           const prr_step_events* events);

/* The same decode step (a1-a7) in ONE persistent launch on `stream`: resident CTAs of
 * 128 threads (three per SM at the usual shapes) take work items from one counter --
 * every unit's selection chunks first, then its top-K finishers, predictor updates,
 * speculative blocks, repairs and merges.  A dependent item waits, bounded, in the CTA
 * that took it for the items it reads, which always hold lower tickets; a speculative
 * block that selection has already dropped is skipped.  step_parity (0 or 1) must
 * alternate between consecutive calls that share `ws`: each launch uses one copy of the
 * workspace control words and clears the other for the next launch.  Same buffers,
 * results and error behaviour as prr_decode_step; capturable in a CUDA graph (one
 * graph per parity).  Size limit: a CTA's shared memory holds one item's scratch at a
 * time, at long contexts the predictor's per-unit state (about 7.1 KB + 8.4 bytes per
 * block), within 227 KB, so maxnb = ceil(cap_tokens/bs) up to 26,760 blocks;
 * beyond that the call returns PRR_ERR_SHAPE.  Above about 8,000 blocks fewer CTAs fit
 * per SM and the step slows down.
 * PRR abstract / method summary: speculation overlaps selection and stays off the
 * critical path; repair merges the missed blocks without recomputation. */
prr_status prr_decode_step_fused(const prr_dims* dims, const prr_step_buffers* buf, void* ws,
                                 size_t ws_bytes, int32_t step_parity, cudaStream_t stream);

/* Profiling-guided speculation budget (PRR abstract: the speculation budget comes from
 * profiling and keeps speculative work off the critical path; limitations: overheads
 * at context lengths off the profiled grid, between or beyond its points, come from
 * polynomial regressions).
 * Host functions: they touch no device memory and need no GPU.
 *
 * prr_budget_fit: least-squares polynomial of degree `degree` (0..3) through the n
 * points (context_tokens[i], us[i]), in x = context_tokens / 65536; coef[0..degree]
 * receives the coefficients, lowest order first.  PRR_ERR_SHAPE if n <= degree or the
 * degree is outside 0..3; PRR_ERR_INVALID_ARG for a null pointer or a singular system
 * (fewer distinct contexts than coefficients). */
prr_status prr_budget_fit(const double* context_tokens, const double* us, int32_t n, int32_t degree,
                          double* coef);

/* prr_budget_choose (same passages as prr_budget_fit): the speculation budget for a
 * context of context_tokens: the largest p_grid[j] whose predicted speculation time
 * (polynomial spec_coef[j], [np][degree+1]) does not exceed the predicted selection
 * time (polynomial sel_coef, [degree+1]), or 0 if none does.  p_grid must be strictly
 * ascending.  *p_out receives the budget. */
prr_status prr_budget_choose(const double* sel_coef, const double* spec_coef, const int32_t* p_grid,
                             int32_t np, int32_t degree, int32_t context_tokens, int32_t* p_out);

/* Largest units*ceil(cap_tokens/bs) that prr_select_topk_static accepts, and the bytes
 * of device memory its fixed scratch array occupies on every GPU that loads the
 * library (status word + 65536 chunk tickets + one 32-bit key per block). */
#define PRR_SELECT_STATIC_MAX_BLOCKS (1 << 20)
#define PRR_SELECT_STATIC_SCRATCH_BYTES (256 + 65536 * 4 + (size_t)PRR_SELECT_STATIC_MAX_BLOCKS * 4)

/* prr_select_topk without a caller-supplied workspace, for callers that cannot
 * allocate device memory: code running inside another runtime's memory pool with no
 * access to its allocator, hosts that forbid cudaMalloc once serving has started
 * (an allocation can synchronise the device or invalidate an ongoing stream capture),
 * and deployments that fix every buffer at build time.  The paper has no counterpart:
 * this is a packaging variant of the selection step, not a step of the method.
 *
 * Same arguments, results and shape rules as prr_select_topk, minus `ws`; the caller
 * still passes every input and output.  The kernel's scratch (status word, per-unit
 * chunk tickets, per-block score keys) lives in one fixed array inside the library,
 * PRR_SELECT_STATIC_SCRATCH_BYTES per GPU, held from the moment the library's device
 * code is loaded on that GPU until the process exits.
 *   status: optional device int32; receives this call's device-side status code
 *           (0 = ok, else one of PRR_DEV_*), written on `stream` after the kernel.
 * Returns PRR_ERR_CAPACITY, without enqueuing anything, when
 * units*ceil(cap_tokens/bs) > PRR_SELECT_STATIC_MAX_BLOCKS.  Calls no cudaMalloc,
 * cudaFree or other allocating routine.  The first call in each CUDA context (made
 * with that context current) looks up the array's device address and keeps it for
 * that context, so a context created later on the same device (for instance after
 * cudaDeviceReset) gets the address again; make that first call before any stream
 * capture.  Every call clears the status word and the
 * tickets on `stream` (the keys are always rewritten before use).  All calls share
 * the one array: calls whose work may overlap on the GPU (different streams without
 * ordering between them) race and give undefined results; order them on one stream. */
prr_status prr_select_topk_static(const prr_dims* dims, const uint16_t* q, const uint16_t* summ,
                                  const int32_t* seq_lens, const int32_t* pred, int32_t* sel,
                                  int32_t* missed, int32_t* n_missed, uint8_t* keep,
                                  int32_t* status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PRR_H */
