// prr_params.h -- kernel parameter block and workspace layout shared by the host
// launchers and the device kernels of the PRR decode step.
#pragma once

#include <cstddef>
#include <cstdint>

namespace prr {

// Device status codes written (first error wins) into the workspace status word.
enum : int {
  kDevOk = 0,
  kDevBadSeqLen = 1,      // seq_lens[b] < 1 or > cap_tokens
  kDevBadPred = 2,         // predicted list not strictly ascending / out of range
  kDevBadMissed = 3,       // missed list entry out of range
  kDevWaitTimeout = 4,     // a bounded mbarrier wait gave up
  kDevBadRange = 5,        // summary update range outside [0, cap_tokens]
};

// Counters of prr_step_buffers::stats.
enum : int {
  kStatTieMasks = 0,
  kStatKeySearch = 1,
  kStatTakeAll = 2,
  kStatSpecAttended = 3,
  kStatSpecSkipped = 4,
  kStatRepaired = 5,
};

// A bounded wait gives up after this long (one second).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Byte offsets inside the caller-owned workspace (all 256-byte aligned).
struct WsLayout {
  size_t status;     // int32 status word
  size_t sel_cnt;    // uint32 [units] chunk tickets of the selection kernel
  size_t keys;       // uint32 [units][maxnb] order-preserving block-score keys
  size_t gsum;       // uint32x2 [units][ceil(maxnb/32)] per 32-block group: max key, tie mask
  size_t rm;         // float [units*G][K] repair partial max (base-2 logits)
  size_t rl;         // float [units*G][K] repair partial sum
  size_t rO;         // float [units*G][K][d] repair partial numerator
  size_t ctl;        // uint32 [2][ctl_words] control words of the fused step (see fused_step.cu)
  size_t total;
};

struct Params {
  // shape.  A unit is one selection: a (sequence, KV head) pair, or a (sequence, query
  // head) pair under per-head selection.  G = query heads per unit (1 per head).
  int B, Hq, Hkv, G, d, bs, cap, K, P, maxnb, units;
  int upb;      // units per sequence: sequence of unit u = u / upb
  int kv_div;   // KV (and summary) slice of unit u = u / kv_div
  int sel_max;  // block score = largest per-head bound of the group instead of their sum
  int n_sink;   // forced first blocks
  int n_local;  // forced newest blocks
  // paged KV: pools [pages][Hkv][bs][d], table [B][maxnb] block -> page (null: contiguous)
  int pages;
  const int* table;
  // representative-key selector (null: summary bounds): offsets [units][maxnb][n_rep]
  const uint8_t* rep;
  int n_rep;
  float scale_log2;  // softmax scale * log2(e): logits are handled in base 2
  double alpha;      // EMA decay
  int append_summary;  // selection also folds token n-1 into its block summary
  int append_kv;       // the fused step appends k_new/v_new itself: n = seq_lens[b] + 1
  // selection geometry
  int chunk_blocks;  // blocks per selection CTA (multiple of 32)
  int nchunks;       // selection CTAs per unit
  // fused single-launch step
  int parity;        // which copy of the control words this launch uses
  int ctl_words;     // words per copy
  int fchunks;       // SEL items per unit
  int fchunk_blocks; // blocks per SEL item (multiple of 32, at most 128)
  int fregion;       // bytes of the per-CTA shared-memory union of the fused step
  int rep_items;     // REPAIR items per unit of the fused step: item r repairs missed slots r, r + rep_items, ...
  int dep_lag;       // units between a unit's SPEC tickets and its REPAIR / COMBINE tickets
  // caller buffers (any may be null when the kernel does not use it)
  const uint16_t* q;        // [B][Hq][d] bf16
  const uint16_t* k_new;    // [B][Hkv][d] bf16 token appended by the fused step (append_kv)
  const uint16_t* v_new;    // [B][Hkv][d] bf16
  const uint16_t* kc;       // [B][Hkv][cap][d] bf16
  const uint16_t* vc;       // [B][Hkv][cap][d] bf16
  const int* seq_lens;      // [B]
  uint16_t* summ;           // [B][Hkv][maxnb][2][d] bf16 (min row, max row)
  double* ema;              // [B][Hkv][maxnb]
  const int* pred;          // [B][Hkv][P]  Pred_t
  int* pred_next;           // [B][Hkv][P]  Pred_{t+1}
  int* sel;                 // [B][Hkv][K]
  int* missed;              // [B][Hkv][K]
  int* n_missed;            // [B][Hkv]
  uint8_t* keep;            // [B][Hkv][P]
  float* pm;                // [B][Hq][P]
  float* pl;                // [B][Hq][P]
  float* pO;                // [B][Hq][P][d]
  float* out;               // [B][Hq][d]
  float* lse;               // [B][Hq]
  // workspace views
  int* status;
  unsigned* sel_cnt;
  uint32_t* keys;
  uint2* gsum;               // null: the finisher derives group maxima from the keys
  float* rm;
  float* rl;
  float* rO;
  unsigned* ctl;
  unsigned long long* trace;  // optional: per fused item {start ns, end ns, sm, item}
  unsigned long long* stats;  // optional: step counters (see prr_step_buffers::stats)
  // summary update range (null: append of token seq_lens[b]-1)
  const int* tok_begin;
  const int* tok_end;
};

}  // namespace prr
