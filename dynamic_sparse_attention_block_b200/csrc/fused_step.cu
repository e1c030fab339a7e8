// fused_step.cu -- the whole PRR decode step in ONE persistent, warp-specialised launch.
//
// This is the PRR runtime (abstract; method summary; contributions (1)-(3)) scheduled
// as a dataflow over a 148-SM part.  One CTA per SM: a producer warp, two consumer
// groups of four warps and a bookkeeper warp share a ring of item slots in shared
// memory.
//
//  * The producer takes work, resolves what each item needs to load, and issues the
//    copies (1-D bulk copies for summary rows and query rows, 3-D TMA for K/V tiles)
//    into the next free slot, up to a full ring ahead of the consumers, so every SM
//    keeps several items' bytes in flight while the consumers compute.
//  * Work comes from three places.  This CTA's FINISH mailbox (taken first); the ready
//    queue in the workspace: REPAIR (unit, missed slot, block), EMA (unit) and COMBINE
//    (unit, query head); and the main tickets (one atomic counter, claimed in small
//    batches): first every selection chunk (SEL: unit, 32-128 blocks), then every
//    speculative slot (SPEC: unit, predicted slot j).  No item ever waits for
//    another: a task exists only once everything it reads does.
//  * SEL folds the appended key into its block's summary (a1) and scores the chunk's
//    blocks (a2).  FINISH runs a unit's top-K (a3) once all its chunks are scored,
//    publishes S_t, M_t = S_t \ Pred_t and the keep mask, and queues one REPAIR per
//    missed block (a4).  SPEC attends one predicted block (a5); a predicted block that
//    selection has already dropped is skipped by the producer.  REPAIR attends one
//    missed block (a6); COMBINE is the LSE merge of one query head (a6); EMA is the
//    unit's predictor update (a4).
//  * Consumers never wait on global memory ordering.  Whatever must be published to
//    other CTAs with release semantics -- a chunk scored, a partial written, a
//    finisher's outputs, a merge or predictor update done -- a consumer group posts as
//    a record to the bookkeeper warp through shared memory.  The bookkeeper takes the
//    records in batches: one release fence covers all of them, then the counter
//    updates (one lane each), then, for the counts that complete, one acquire fence
//    and the follow-up tasks: FINISH into this CTA's mailbox when a unit's last chunk
//    is counted, the unit's EMA task when its finisher is done, and its COMBINE tasks
//    when its partial count completes (the finisher adds a large constant minus the
//    expected count, so whichever add lands last completes it).
//  * The launch ends when every unit's merges and predictor update are done; the
//    producers then send their consumer groups an exit item.
//
// Waits: consumers wait for their slot's copies (bounded), the producer for a free
// slot (bounded) and, at the end, for the last tasks of other CTAs (bounded); none of
// them depends on CTAs that have not started, so the launch needs no co-residency.  A
// wait that times out records PRR_DEV_WAIT_TIMEOUT and raises an abort flag that makes
// every CTA stop taking work; copies already issued are waited for (bounded) first.
//
// Control words live in the workspace in two copies selected by the step parity: a
// launch works on copy[parity] and clears copy[1 - parity] for the next launch.
//
// When the caller passes the step's new token (k_new, v_new), the launch appends it:
// every item works on n = seq_lens[b] + 1 tokens, the SEL chunk that owns the new
// token writes its K/V row into the cache, attention over the tail block takes that
// row from k_new/v_new (a concurrent copy may still hold the old row), and the
// launch's last CTA advances seq_lens once no item can read it any more.
#include <algorithm>

#include "prr_attn.cuh"
#include "prr_parts.cuh"

namespace prr {

constexpr int kFusedThreads = 320;       // two consumer groups of 128, a producer and a bookkeeper warp
constexpr int kProducerWarp = 8;
constexpr int kBookWarp = 9;
constexpr int kAuxBytes = 4096;          // per slot: q rows, key row, reductions, descriptor
constexpr int kAuxQ = 0;                 // G*D bf16 query rows (<= 2048 bytes)
constexpr int kAuxNewK = 3072;           // the appended key row (D bf16)
constexpr int kAuxRed = 3328;            // 80 floats of attention reductions
constexpr int kAuxDesc = 3712;           // ItemDesc
constexpr unsigned kBig = 1u << 30;      // per-unit partial-count completion value

// Control words of one copy (word offsets).
enum : int {
  kCtlWork = 0,      // next main ticket
  kCtlAbort = 1,     // set when a bounded wait gave up
  kCtlRqHead = 2,    // next ready-queue entry to take
  kCtlRqTail = 3,    // next ready-queue entry to fill
  kCtlCombined = 4,  // finished COMBINE tasks
  kCtlEmaDone = 5,   // finished EMA tasks
  kCtlFinal = 6,     // set by the CTA that advances seq_lens
  kCtlUnits = 16,    // per-unit words start here
};

enum : int {
  kItemExit = 0, kItemSel = 1, kItemSpec = 2, kItemRepair = 3, kItemEma = 4, kItemCombine = 5, kItemFinish = 6
};

// What a consumer finds in its slot.
struct ItemDesc {
  int kind;
  int u;          // unit
  int idx;        // SEL: chunk; SPEC: predicted slot; REPAIR: missed slot; COMBINE: query head
  int blk;        // SPEC / REPAIR: block
  int n;          // tokens of the unit's sequence this step (0 if seq_lens was invalid)
  int trace;      // trace record index
  unsigned seq;   // ring sequence number of this use of the slot
  unsigned pad;
  unsigned long long t_issue;  // debug builds: when the copies were issued
};
constexpr unsigned kNoSeq = 0xFFFFFFFFu;  // a slot's descriptor before its first use

struct FusedCtl {
  unsigned* words;          // the fixed words above
  unsigned* sel_cnt;        // [units] scored SEL chunks
  unsigned* done;           // [units] finished partials (+ kBig - expected, added by the finisher)
  unsigned* keepf;          // [units][P] 0 until S_t is known, then 1 | keep << 1
  unsigned long long* rq;   // [rq_cap] ready tasks (0 = not yet written)
};

__host__ __device__ inline size_t fused_ctl_words(int units, int P, int K, int G) {
  const size_t U = static_cast<size_t>(units);
  size_t w = kCtlUnits + 2 * U + U * static_cast<size_t>(P);
  w = (w + 1) & ~static_cast<size_t>(1);  // the queue holds 8-byte words
  return w + 2 * U * static_cast<size_t>(1 + K + G);
}

__device__ __forceinline__ FusedCtl ctl_view(const Params& p, int parity) {
  unsigned* b = p.ctl + static_cast<size_t>(parity) * p.ctl_words;
  const size_t U = p.units;
  size_t q = kCtlUnits + 2 * U + U * static_cast<size_t>(p.P);
  q = (q + 1) & ~static_cast<size_t>(1);
  return FusedCtl{b, b + kCtlUnits, b + kCtlUnits + U, b + kCtlUnits + 2 * U,
                  reinterpret_cast<unsigned long long*>(b + q)};
}

// Task words: kind (bits 60-63), unit (32-47), index (24-31), block (0-23).
__device__ __forceinline__ unsigned long long make_task(int kind, int u, int idx, int blk) {
  return (static_cast<unsigned long long>(kind) << 60) | (static_cast<unsigned long long>(u) << 32) |
         (static_cast<unsigned long long>(idx & 0xFF) << 24) | static_cast<unsigned long long>(blk & 0xFFFFFF);
}

// Blocks per SEL item: a multiple of 32 in [32, 128], about units*maxnb / (2*SMs), so a
// short context spreads its scan over many SMs and a long one moves 64 KB per item.
__host__ __device__ inline int fused_chunk_blocks(int units, int maxnb, int sms) {
  long long c = (static_cast<long long>(units) * maxnb + 2LL * sms - 1) / (2LL * sms);
  c = ((c + 31) / 32) * 32;
  return static_cast<int>(c < 32 ? 32 : (c > 128 ? 128 : c));
}

// Bytes of one slot's main area: two K/V tiles, a SEL chunk of summary rows, or the
// scratch of the finisher, the predictor or a merge -- whichever is largest.
template <int D, int BS>
size_t fused_slot_bytes(const Params& p) {
  size_t b = 2 * static_cast<size_t>(AttnTile<D, BS>::TILEB);
  b = std::max(b, static_cast<size_t>(p.fchunk_blocks) * 4 * D);
  b = std::max(b, finish_scratch_bytes(p.maxnb));
  b = std::max(b, ema_scratch_bytes(p.maxnb));
  b = std::max(b, combine_scratch_bytes(p.P, p.K, D));
  return (b + 1023) & ~static_cast<size_t>(1023);
}

// ---------------------------------------------------------------- ready queue
// Tasks are appended by reserving entries (atomic add on the tail) and publishing each
// word with a store that follows a release fence (or needs none: a repair's word is all
// it reads), so a taker that reads the word non-zero also sees what the task reads.
// Takers claim entry indices one at a time with an atomic add on the head (no
// compare-and-swap retries, so many idle CTAs do not contend): a claimed index may lie
// ahead of the tail, and the claimer checks it without blocking until a task lands
// there or the step is over.

// ---------------------------------------------------------------- bookkeeping records
// A record is one 64-bit word: op (bits 56-63), unit (32-55), argument (0-31).  Three
// single-writer rings (consumer group 0, group 1, producer) feed the bookkeeper warp.
enum : unsigned {
  kRecSelDone = 1,   // a SEL chunk of the unit is scored (keys and group summaries written)
  kRecPartial = 2,   // a speculative or repair partial of the unit is written, or skipped
  kRecFinDone = 3,   // the unit's finisher is done; argument: kBig - expected partials
  kRecEmaDone = 4,   // a predictor update is done
  kRecCombDone = 5,  // a merge is done
  kRecExit = 6,      // the writer has stopped
};
constexpr int kRecRing = 64;   // records per ring
constexpr int kFinBox = 32;    // FINISH mailbox entries

struct BookSmem {
  unsigned long long rec[3][kRecRing];
  unsigned tail[3];    // written by each ring's writer (release)
  unsigned head[3];    // written by the bookkeeper once the records are read
  unsigned fin[kFinBox];
  unsigned fin_tail;   // written by the bookkeeper (release)
  unsigned fin_head;   // written by the producer
};

__device__ __forceinline__ unsigned long long make_rec(unsigned op, int u, unsigned arg) {
  return (static_cast<unsigned long long>(op) << 56) | (static_cast<unsigned long long>(u & 0xFFFFFF) << 32) | arg;
}

__device__ __forceinline__ void st_release_cta(unsigned* a, unsigned v) {
  asm volatile("st.release.cta.shared.u32 [%0], %1;" ::"r"(smem_addr(a)), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_cta(const unsigned* a) {
  unsigned v;
  asm volatile("ld.acquire.cta.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(a)) : "memory");
  return v;
}

// One thread (the ring's only writer): append a record.  What the writer's group wrote
// before its last group barrier is ordered before the record (release at CTA scope);
// the bookkeeper's fence then publishes it at GPU scope.  Bounded wait for room.
__device__ inline bool post_record(BookSmem* bk, int ring, unsigned& tail, unsigned long long rec, int* status) {
  if (tail - ld_acquire_cta(&bk->head[ring]) >= static_cast<unsigned>(kRecRing)) {
    const uint64_t t0 = global_ns();
    while (tail - ld_acquire_cta(&bk->head[ring]) >= static_cast<unsigned>(kRecRing)) {
      if (global_ns() - t0 > kWaitLimitNs) {
        report(status, kDevWaitTimeout);
        return false;
      }
      __nanosleep(64);
    }
  }
  bk->rec[ring][tail % kRecRing] = rec;
  st_release_cta(&bk->tail[ring], ++tail);
  return true;
}

// ---------------------------------------------------------------- consumer items
template <int D>
__device__ void sel_scores(const Params& p, const ItemDesc& it, unsigned char* rows, unsigned char* aux,
                           float4* coef, const Grp& grp) {
  constexpr int ROWB = 4 * D;
  const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
  const int u = it.u, n = it.n;
  const int kvu = u / p.kv_div;  // KV slice (several units share it under per-head selection)
  const int c0 = it.idx * p.fchunk_blocks;
  const int nb = (n + p.bs - 1) / p.bs;
  const int cnt = max(0, min(p.fchunk_blocks, nb - c0));
  const int tail = n > 0 ? (n - 1) / p.bs : -1;
  const bool own_tail = p.append_summary && tail >= c0 && tail < c0 + cnt;
  uint16_t* newk = reinterpret_cast<uint16_t*>(aux + kAuxNewK);
  uint16_t* summ_unit = p.summ + static_cast<size_t>(kvu) * p.maxnb * 2 * D;

  load_coef<D>(p, reinterpret_cast<const uint16_t*>(aux + kAuxQ), coef, grp);
  const long long trow = own_tail ? kv_row(p, kvu, n - 1) : -1;  // the new token's row in the cache
  if (own_tail && trow >= 0) {
    const size_t ukv = static_cast<size_t>(kvu) * D;
    const uint16_t* krow = p.append_kv ? p.k_new + ukv : p.kc + static_cast<size_t>(trow) * D;
    if (tid < D / 8) reinterpret_cast<uint4*>(newk)[tid] = reinterpret_cast<const uint4*>(krow)[tid];
    if (p.append_kv && tid >= 32 && tid < 32 + D / 4) {  // the new row enters the cache
      const int c = tid - 32;
      const size_t dst = static_cast<size_t>(trow) * D;
      if (c < D / 8) {
        reinterpret_cast<uint4*>(const_cast<uint16_t*>(p.kc) + dst)[c] =
            reinterpret_cast<const uint4*>(p.k_new + ukv)[c];
      } else {
        reinterpret_cast<uint4*>(const_cast<uint16_t*>(p.vc) + dst)[c - D / 8] =
            reinterpret_cast<const uint4*>(p.v_new + ukv)[c - D / 8];
      }
    }
  }
  gsync(grp);
  const int first = c0 + 32 * warp;
  const int wrows = min(32, cnt - 32 * warp);
  if (wrows > 0) {
    unsigned char* tile = rows + warp * 32 * ROWB;
    if (own_tail && trow >= 0 && tail >= first && tail < first + wrows)
      fold_tail_row<D>(reinterpret_cast<uint32_t*>(tile + (tail - first) * ROWB), newk, ((n - 1) % p.bs) == 0,
                       reinterpret_cast<uint32_t*>(summ_unit + static_cast<size_t>(tail) * 2 * D), lane);
    uint32_t key = 0u;
    if (lane < wrows) {
      key = block_key(p, first + lane, nb, score_row<D>(p, tile + lane * ROWB, coef, lane));
      p.keys[static_cast<size_t>(u) * p.maxnb + first + lane] = key;
    }
    write_group_summary(p, u, first / 32, key, lane < wrows);
  }
}

// FINISH: the unit's selection is complete (every chunk's keys are visible): top-K,
// missed set, keep mask; queue its repairs.  Returns the partial-count adjustment for
// the bookkeeper (kBig - active predicted slots - missed blocks).  The finisher leaves
// the missed blocks (+1) in the first K words of `scratch`, which it does not use
// otherwise, so queueing them needs no global round trip.
__device__ unsigned finish_unit(const Params& p, const FusedCtl& C, int u, int n, unsigned char* scratch,
                                const Grp& grp) {
  const int nb = (n + p.bs - 1) / p.bs;
  unsigned* mlist = reinterpret_cast<unsigned*>(scratch);
  const FinishOut f = select_finish(p, u, nb, scratch, grp, C.keepf + static_cast<size_t>(u) * p.P, mlist);
  gsync(grp);  // mlist is complete
  const int tid = grp.tid;
  const int nm = min(max(f.n_missed, 0), p.K);
  if (tid < 32 && nm > 0) {  // one warp queues the repairs, lane-parallel; a repair reads only its word
    unsigned pos = 0;
    if (tid == 0) pos = atomicAdd(C.words + kCtlRqTail, static_cast<unsigned>(nm));
    pos = __shfl_sync(kFull, pos, 0);
    for (int i = tid; i < nm; i += 32) {
      if (pos + i < static_cast<unsigned>(p.rq_cap)) {
        st_relaxed64(C.rq + pos + i, make_task(kItemRepair, u, i, static_cast<int>(mlist[i]) - 1));
      } else {
        report(p.status, kDevWaitTimeout);  // cannot happen: the queue holds every task of a step
        atomicExch(C.words + kCtlAbort, 1u);
      }
    }
  }
  return kBig - static_cast<unsigned>(f.p_active + nm);
}

// ---------------------------------------------------------------- shared memory
struct FusedSmem {
  unsigned char* slots;  // fslots * fslot_bytes
  unsigned char* aux;    // fslots * kAuxBytes
  float4* coef;          // [2 groups][coef_bytes(D, sets) / 16] scoring coefficients
  uint64_t* fullK;       // [fslots] K tile (or summary rows) + query rows landed
  uint64_t* fullV;       // [fslots] V tile landed
  uint64_t* empty;       // [fslots] the consumer group is done with the slot
  int* claim;            // [1] next slot sequence number a consumer group takes
  int* bcast;            // [2][8] per-group broadcast words
  BookSmem* bk;          // records for the bookkeeper, FINISH mailbox
};

template <int D>
__host__ __device__ inline size_t group_coef_bytes(const Params& p) {
  return coef_bytes(D, p.sel_max ? p.G : 1);
}

template <int D>
__device__ __forceinline__ FusedSmem fused_smem(const Params& p, unsigned char* base) {
  FusedSmem s;
  s.slots = base;
  s.aux = base + static_cast<size_t>(p.fslots) * p.fslot_bytes;
  s.coef = reinterpret_cast<float4*>(s.aux + static_cast<size_t>(p.fslots) * kAuxBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(s.coef) + 2 * group_coef_bytes<D>(p));
  s.fullK = bars;
  s.fullV = bars + p.fslots;
  s.empty = bars + 2 * p.fslots;
  s.claim = reinterpret_cast<int*>(bars + 3 * p.fslots);
  s.bcast = s.claim + 4;
  s.bk = reinterpret_cast<BookSmem*>(s.bcast + 16);
  return s;
}

__host__ __device__ inline size_t fused_smem_total(int slots, int slot_bytes, size_t group_coef) {
  return 1024 + static_cast<size_t>(slots) * (slot_bytes + kAuxBytes) + 2 * group_coef +
         3 * 8 * static_cast<size_t>(slots) + 4 * 4 + 16 * 4 + sizeof(BookSmem);
}

// ---------------------------------------------------------------- producer
// Lane 0 of the producer warp: fill slot `seq % fslots` with an item and start its
// copies.  Waits (bounded) until the slot's previous use is done; false if it was not.
template <int D, int BS>
__device__ bool prod_emit(const Params& p, const FusedSmem& S, const CUtensorMap* kmap, const CUtensorMap* vmap,
                          uint32_t& seq, const ItemDesc& it) {
  const uint32_t use = seq / p.fslots;
  const int s = seq % p.fslots;
  if (use > 0 && !mbar_wait_idle(&S.empty[s], (use - 1) & 1u, p.status)) return false;
  unsigned char* slot = S.slots + static_cast<size_t>(s) * p.fslot_bytes;
  unsigned char* aux = S.aux + static_cast<size_t>(s) * kAuxBytes;
  {
    ItemDesc d = it;
    d.seq = seq;
#ifdef PRR_PHASE_DEBUG
    d.t_issue = global_ns();
#endif
    *reinterpret_cast<ItemDesc*>(aux + kAuxDesc) = d;
  }
  const uint32_t qbytes = static_cast<uint32_t>(p.G) * D * 2;
  const uint16_t* qsrc = p.q + static_cast<size_t>(it.u) * p.G * D;
  fence_proxy_async();  // the consumers' generic writes to this slot precede the new copies
  if (it.kind == kItemSel) {
    const int c0 = it.idx * p.fchunk_blocks;
    const int rows = max(0, min(p.fchunk_blocks, p.maxnb - c0));  // up to the allocation, not n
    const uint32_t bytes = static_cast<uint32_t>(rows) * 4 * D;
    mbar_expect_tx(&S.fullK[s], bytes + qbytes);
    if (bytes)
      bulk_load(slot, p.summ + (static_cast<size_t>(it.u / p.kv_div) * p.maxnb + c0) * 2 * D, bytes, &S.fullK[s]);
    bulk_load(aux + kAuxQ, qsrc, qbytes, &S.fullK[s]);
    mbar_arrive(&S.fullV[s]);
  } else if (it.kind == kItemSpec || it.kind == kItemRepair) {
    using L = AttnTile<D, BS>;
    unsigned char* sK = slot;
    unsigned char* sV = slot + L::TILEB;
    int tok0;
    const int slice = kv_tile(p, it.u / p.kv_div, it.blk, &tok0);
    mbar_expect_tx(&S.fullK[s], L::TILEB + qbytes);
#pragma unroll
    for (int r = 0; r < D / 64; ++r) tma_load_3d(sK + r * L::REGB, kmap, &S.fullK[s], r * 64, tok0, slice);
    bulk_load(aux + kAuxQ, qsrc, qbytes, &S.fullK[s]);
    mbar_expect_tx(&S.fullV[s], L::TILEB);
#pragma unroll
    for (int r = 0; r < D / 64; ++r) tma_load_3d(sV + r * L::REGB, vmap, &S.fullV[s], r * 64, tok0, slice);
  } else {  // no copy: the arrivals publish the descriptor
    mbar_arrive(&S.fullK[s]);
    mbar_arrive(&S.fullV[s]);
  }
  ++seq;
  return true;
}

__device__ __forceinline__ bool warp_flag(bool v) { return __shfl_sync(kFull, v ? 1 : 0, 0) != 0; }

// Producer warp.  Lane 0 drives; lanes resolve a claimed batch of main tickets in
// parallel (one round trip for all of them).  Each pass looks first at this CTA's
// FINISH mailbox, then at the one claimed ready-queue index lane 0 always holds (one
// load, no waiting), then emits the batch in hand; the next batch's tickets are claimed
// one batch ahead.
template <int D, int BS>
__device__ void producer(const Params& p, const FusedCtl& C, const FusedSmem& S, const CUtensorMap* kmap,
                         const CUtensorMap* vmap) {
  const int lane = threadIdx.x & 31;
  const Grp solo{0, 32, -1};  // reports from any lane (checked_len reports when tid == 0)
  const int U = p.units;
  const unsigned n_sel = static_cast<unsigned>(U) * p.fchunks;
  const unsigned n_main = n_sel + static_cast<unsigned>(U) * p.P;
  const unsigned B = static_cast<unsigned>(p.fbatch);
  uint32_t seq = 0;
  unsigned rec_tail = 0;  // lane 0: records posted to the bookkeeper
  unsigned fin_head = 0;  // lane 0: FINISH mailbox entries taken
  bool ok = true, exhausted = false;
  // failure-detection tests set the word after the status word: selection never runs
  const bool skip_sel = p.status != nullptr && p.status[1] != 0;
  unsigned next_base = 0, pend = 0;  // lane 0: next batch's first ticket, claimed queue index
  if (lane == 0) {
    next_base = atomicAdd(C.words + kCtlWork, B);
    pend = atomicAdd(C.words + kCtlRqHead, 1u);
  }
  uint64_t idle_t0 = 0;

  for (;;) {
    // ---- a unit whose selection this CTA completed: its finisher first (critical path)
    bool fin_emitted = false;
    if (lane == 0 && fin_head != ld_acquire_cta(&S.bk->fin_tail)) {
      ItemDesc it{};
      it.kind = kItemFinish;
      it.u = static_cast<int>(S.bk->fin[fin_head % kFinBox]);
      it.n = checked_len(p, it.u / p.upb, solo);
      it.trace = static_cast<int>(n_main + p.rq_cap + it.u);
      st_release_cta(&S.bk->fin_head, ++fin_head);
      ok = prod_emit<D, BS>(p, S, kmap, vmap, seq, it);
      fin_emitted = true;
    }
    ok = warp_flag(ok);
    if (!ok) break;
    fin_emitted = warp_flag(fin_emitted);

    // One round trip per pass: lane 0 loads its claimed queue word and the abort flag
    // while the lanes load the metadata of the batch in hand; all of it is looked at
    // afterwards.
    unsigned long long tq = 0ull;
    unsigned abort_seen = 0u;
    if (lane == 0) {
      if (pend < static_cast<unsigned>(p.rq_cap)) tq = ld_relaxed64(C.rq + pend);
      abort_seen = ld_relaxed(C.words + kCtlAbort);
    }
    unsigned base = 0, cnt = 0;
    ItemDesc mine{};
    bool emit = false, skip_done = false;
    if (!exhausted) {
      base = __shfl_sync(kFull, next_base, 0);
      if (base >= n_main) {
        exhausted = true;
      } else {
        if (lane == 0) next_base = atomicAdd(C.words + kCtlWork, B);  // claimed a batch ahead
        cnt = min(B, n_main - base);
        if (static_cast<unsigned>(lane) < cnt) {  // lane i resolves ticket base + i
          const unsigned tk = base + lane;
          mine.trace = static_cast<int>(tk);
          if (tk < n_sel) {
            mine.kind = kItemSel;
            mine.u = static_cast<int>(tk / p.fchunks);
            mine.idx = static_cast<int>(tk % p.fchunks);
            mine.n = checked_len(p, mine.u / p.upb, solo);
            emit = !skip_sel;
          } else {
            const unsigned sp = tk - n_sel;
            mine.kind = kItemSpec;
            mine.u = static_cast<int>(sp / p.P);
            mine.idx = static_cast<int>(sp % p.P);
            const size_t pj = static_cast<size_t>(mine.u) * p.P + mine.idx;
            const int blk = p.pred[pj];
            const unsigned kf = __ldcg(C.keepf + pj);
            mine.n = checked_len(p, mine.u / p.upb, solo);
            mine.blk = blk;
            const int nb = (mine.n + BS - 1) / BS;
            if (blk >= 0 && blk < nb) {
              if (kf == 1u) {
                skip_done = true;  // selection already dropped it: nothing to attend
              } else {
                emit = true;
              }
            }
          }
        }
      }
    }
    if (__shfl_sync(kFull, abort_seen, 0)) {
      ok = false;
      break;
    }

    // ---- the claimed queue entry (repairs and merges are on the critical path)
    const bool have_task = __shfl_sync(kFull, tq != 0ull ? 1 : 0, 0) != 0;
    if (have_task) {
      if (lane == 0) {
        const unsigned long long task = ld_acquire64(C.rq + pend);  // orders what the task reads
        ItemDesc it{};
        it.kind = static_cast<int>(task >> 60);
        it.u = static_cast<int>((task >> 32) & 0xFFFF);
        it.idx = static_cast<int>((task >> 24) & 0xFF);
        it.blk = static_cast<int>(task & 0xFFFFFF);
        it.n = checked_len(p, it.u / p.upb, solo);
        it.trace = static_cast<int>(n_main + pend);
        pend = atomicAdd(C.words + kCtlRqHead, 1u);  // the next claim; its value is needed next pass
        ok = prod_emit<D, BS>(p, S, kmap, vmap, seq, it);
      }
      ok = warp_flag(ok);
      if (!ok) break;
    }

    // ---- the batch of main tickets
    for (unsigned i = 0; i < cnt; ++i) {  // warp-uniform loop; lane 0 emits lane i's item
      ItemDesc it{};
      it.kind = __shfl_sync(kFull, mine.kind, i);
      it.u = __shfl_sync(kFull, mine.u, i);
      it.idx = __shfl_sync(kFull, mine.idx, i);
      it.blk = __shfl_sync(kFull, mine.blk, i);
      it.n = __shfl_sync(kFull, mine.n, i);
      it.trace = __shfl_sync(kFull, mine.trace, i);
      const bool e = __shfl_sync(kFull, emit ? 1 : 0, i) != 0;
      const bool sd = __shfl_sync(kFull, skip_done ? 1 : 0, i) != 0;
      if (lane == 0) {
        if (e) {
          ok = prod_emit<D, BS>(p, S, kmap, vmap, seq, it);
        } else if (sd) {
          bump(p.stats, kStatSpecSkipped);
          ok = post_record(S.bk, 2, rec_tail, make_rec(kRecPartial, it.u, 1u), p.status);
        }
      }
      ok = warp_flag(ok);
      if (!ok) break;
    }
    if (!ok) break;
    if (cnt > 0 || have_task || fin_emitted) {
      idle_t0 = 0;
      continue;
    }
    if (!exhausted) continue;

    // ---- no work in hand: done, or wait for other CTAs' tasks
    bool all_done = false;
    if (lane == 0) {
      all_done = ld_acquire(C.words + kCtlCombined) >= static_cast<unsigned>(U * p.G) &&
                 ld_acquire(C.words + kCtlEmaDone) >= static_cast<unsigned>(U);
      if (!all_done) {
        const uint64_t now = global_ns();
        if (idle_t0 == 0) idle_t0 = now;
        if (now - idle_t0 > kWaitLimitNs) {
          report(p.status, kDevWaitTimeout);
          ok = false;
        } else {
          __nanosleep(100);
        }
      }
    }
    all_done = warp_flag(all_done);
    ok = warp_flag(ok);
    if (!ok) break;
    if (all_done) {
      // the step appended its token: advance seq_lens once nothing can read it any more
      if (p.append_kv && lane == 0 && atomicCAS(C.words + kCtlFinal, 0u, 1u) == 0u) {
        for (int b = 0; b < p.B; ++b) {
          const int n0 = p.seq_lens[b];
          if (n0 >= 0 && n0 < p.cap) const_cast<int*>(p.seq_lens)[b] = n0 + 1;
        }
      }
      break;
    }
  }

  // ---- exit items for both consumer groups, then let issued copies land
  if (lane == 0) {
    if (!ok) atomicExch(C.words + kCtlAbort, 1u);
    ItemDesc ex{};
    ex.kind = kItemExit;
    bool sent = true;
    for (int g = 0; g < 2 && sent; ++g) sent = prod_emit<D, BS>(p, S, kmap, vmap, seq, ex);
    const uint32_t first = seq > static_cast<uint32_t>(p.fslots) ? seq - p.fslots : 0u;
    for (uint32_t q = first; q < seq; ++q) {  // bounded waits; completed phases return at once
      const int s = q % p.fslots;
      const uint32_t ph = (q / p.fslots) & 1u;
      mbar_wait(&S.fullK[s], ph, p.status);
      mbar_wait(&S.fullV[s], ph, p.status);
    }
    post_record(S.bk, 2, rec_tail, make_rec(kRecExit, 0, 0u), p.status);
  }
  __syncwarp();
}

// One thread: bounded wait until the slot descriptor's sequence number is `k`.
__device__ bool wait_seq(const unsigned* seq, uint32_t k, int* status) {
  const volatile unsigned* v = seq;
  if (*v == k) return true;
  const uint64_t t0 = global_ns();
  for (int spin = 0; *v != k; ++spin) {
    if (spin > 4) __nanosleep(64);
    if (global_ns() - t0 > kWaitLimitNs) {
      report(status, kDevWaitTimeout);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- consumer groups
// A group takes the next slot in sequence, runs its item and hands the slot back as
// soon as it no longer reads it; what other CTAs wait for goes to the bookkeeper as a
// record, so the group never waits for its own global writes to complete.
template <int D, int BS>
__device__ void consumer(const Params& p, const FusedCtl& C, const FusedSmem& S, int group) {
  const Grp grp{static_cast<int>(threadIdx.x) - 128 * group, 128, 1 + group};
  const int tid = grp.tid;
  int* bc = S.bcast + 8 * group;
  unsigned rec_tail = 0;  // thread 0: records posted
  bool posted_ok = true;  // thread 0: every post went through
  for (;;) {
    bool filled = true;
    if (tid == 0) {
      const uint32_t kc = static_cast<uint32_t>(atomicAdd(S.claim, 1));
      bc[0] = static_cast<int>(kc);
      // The slot's barriers are waited on by parity, which tells apart only two
      // consecutive uses: the other group may still hold the slot's previous use (this
      // group can run a whole ring ahead of it), so first wait until the producer has
      // filled THIS use, which it does only once the previous one is handed back.
      const ItemDesc* d = reinterpret_cast<const ItemDesc*>(S.aux + static_cast<size_t>(kc % p.fslots) * kAuxBytes +
                                                            kAuxDesc);
      filled = wait_seq(&d->seq, kc, p.status);
    }
    const bool filled_all = gsync_and(grp, filled);
    const uint32_t k = static_cast<uint32_t>(bc[0]);
    const int s = k % p.fslots;
    const uint32_t ph = (k / p.fslots) & 1u;
    unsigned char* slot = S.slots + static_cast<size_t>(s) * p.fslot_bytes;
    unsigned char* aux = S.aux + static_cast<size_t>(s) * kAuxBytes;
    if (!filled_all || !gsync_and(grp, mbar_wait_idle(&S.fullK[s], ph, p.status))) {
      if (tid == 0) {
        atomicExch(C.words + kCtlAbort, 1u);
        post_record(S.bk, group, rec_tail, make_rec(kRecExit, 0, 0u), p.status);
      }
      return;  // the producer waits for this slot's copies before the CTA exits
    }
    const ItemDesc it = *reinterpret_cast<const ItemDesc*>(aux + kAuxDesc);
    if (it.kind == kItemExit) {
      if (tid == 0) post_record(S.bk, group, rec_tail, make_rec(kRecExit, 0, 0u), p.status);
      return;
    }
#ifdef PRR_PHASE_DEBUG
    unsigned long long* dbg_item =
        (it.trace >= 0 && it.trace < (1 << 16)) ? g_item[it.trace] : nullptr;
    if (dbg_item && tid == 0) {
      dbg_item[0] = it.t_issue;
      dbg_item[1] = global_ns();
    }
#else
    unsigned long long* dbg_item = nullptr;
#endif
    if (p.trace && tid == 0) {
      unsigned smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      unsigned long long* tr = p.trace + 4 * static_cast<size_t>(it.trace);
      tr[0] = global_ns();
      tr[2] = (static_cast<unsigned long long>(smid) << 32) | (static_cast<unsigned>(group) << 16) | blockIdx.x;
      tr[3] = static_cast<unsigned long long>(it.kind);
    }
    bool ok = true;
    bool released = false;                 // (every thread) the slot was handed back early
    unsigned long long rec = 0ull;         // thread 0: the record this item ends with
    if (it.kind == kItemSel) {
      sel_scores<D>(p, it, slot, aux, S.coef + group * (group_coef_bytes<D>(p) / 16), grp);
      rec = make_rec(kRecSelDone, it.u, 0u);
    } else if (it.kind == kItemFinish) {
      const unsigned adj = finish_unit(p, C, it.u, it.n, slot, grp);  // the slot is the finisher's scratch
      rec = make_rec(kRecFinDone, it.u, adj);
    } else if (it.kind == kItemSpec || it.kind == kItemRepair) {
      using L = AttnTile<D, BS>;
      const bool spec = it.kind == kItemSpec;
      const size_t rs = static_cast<size_t>(spec ? p.P : p.K);
      const size_t row0 = static_cast<size_t>(it.u) * p.G * rs + it.idx;
      const PartialDst dst = spec ? PartialDst{p.pm + row0, p.pl + row0, p.pO + row0 * D, rs, rs * D}
                                  : PartialDst{p.rm + row0, p.rl + row0, p.rO + row0 * D, rs, rs * D};
      const bool tail_new = p.append_kv && it.n > 0 && it.blk == (it.n - 1) / BS;
      const size_t kvrow = static_cast<size_t>(it.u / p.kv_div) * D;
      const uint16_t* pk = tail_new ? p.k_new + kvrow : nullptr;
      const uint16_t* pv = tail_new ? p.v_new + kvrow : nullptr;
      if (it.blk >= 0 && it.blk < (it.n + BS - 1) / BS) {
        // the slot goes back as soon as the tiles are read, before the partial is written
        ok = attn_compute<D, BS>(p, reinterpret_cast<const uint16_t*>(aux + kAuxQ), it.blk, it.n, dst, slot,
                                 slot + L::TILEB, reinterpret_cast<float*>(aux + kAuxRed), &S.fullK[s],
                                 &S.fullV[s], ph, grp,
                                 [&] {
                                   released = true;
                                   if (tid == 0) {
                                     mbar_arrive(&S.empty[s]);
                                     if (dbg_item) dbg_item[3] = global_ns();
                                   }
                                 },
                                 pk, pv, dbg_item ? dbg_item + 2 : nullptr);
      } else {  // a missed entry out of range: contribute nothing (copies still land)
        if (tid == 0) {
          report(p.status, kDevBadMissed);
          mbar_wait(&S.fullV[s], ph, p.status);
        }
        write_empty_partial(dst, p.G, D, grp);
      }
      if (tid == 0 && ok) bump(p.stats, spec ? kStatSpecAttended : kStatRepaired);
      rec = make_rec(kRecPartial, it.u, 1u);
    } else if (it.kind == kItemEma) {
      ema_unit(p, it.u, slot, [] { return true; }, grp);
      rec = make_rec(kRecEmaDone, it.u, 0u);
    } else if (it.kind == kItemCombine) {
      combine_head<D>(p, it.u, it.idx, slot, [] { return true; }, grp);
      rec = make_rec(kRecCombDone, it.u, 0u);
    }
    if (!released) fence_proxy_async();  // generic writes to the slot precede the copies that refill it
    // every thread's outputs (and reads of the slot) precede the slot's release and the record
    if (!gsync_and(grp, ok)) {
      if (tid == 0) {
        atomicExch(C.words + kCtlAbort, 1u);
        post_record(S.bk, group, rec_tail, make_rec(kRecExit, 0, 0u), p.status);
      }
      return;
    }
    if (tid == 0) {
      if (!released) mbar_arrive(&S.empty[s]);
      if (rec != 0ull && posted_ok) {
        posted_ok = post_record(S.bk, group, rec_tail, rec, p.status);
        if (!posted_ok) atomicExch(C.words + kCtlAbort, 1u);
      }
      if (p.trace) p.trace[4 * static_cast<size_t>(it.trace) + 1] = global_ns();
    }
  }
}

// ---------------------------------------------------------------- bookkeeper
// One warp.  Takes up to 32 records per round (one per lane) from the three rings,
// publishes them with one release fence, applies them (one atomic per lane) and
// queues the follow-up work of the counts that completed, after one acquire fence.
// Ends once all three writers have posted their exit record.
__device__ void bookkeeper(const Params& p, const FusedCtl& C, const FusedSmem& S) {
  const int lane = threadIdx.x & 31;
  BookSmem* bk = S.bk;
  unsigned hd[3] = {0u, 0u, 0u};  // records taken, per ring (every lane keeps the same copy)
  unsigned fin_tail = 0u;         // FINISH entries posted (lane 0)
  int exits = 0;
  uint64_t idle_t0 = global_ns();
  for (;;) {
    unsigned tl[3];
#pragma unroll
    for (int r = 0; r < 3; ++r) tl[r] = __shfl_sync(kFull, lane == 0 ? ld_acquire_cta(&bk->tail[r]) : 0u, 0);
    // this round's records: ring 0 first, then 1, then 2, at most 32 in all
    int take[3], total = 0;
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      take[r] = min(static_cast<int>(tl[r] - hd[r]), 32 - total);
      total += take[r];
    }
    if (total == 0) {
      if (exits >= 3) break;
      if (global_ns() - idle_t0 > kWaitLimitNs) {  // a writer never finished
        if (lane == 0) {
          report(p.status, kDevWaitTimeout);
          atomicExch(C.words + kCtlAbort, 1u);
        }
        break;
      }
      __nanosleep(32);
      continue;
    }
    idle_t0 = global_ns();
    unsigned long long rec = 0ull;
    {
      int r = 0, i = lane;
      while (r < 3 && i >= take[r]) i -= take[r++];
      if (r < 3) rec = bk->rec[r][(hd[r] + i) % kRecRing];
    }
#pragma unroll
    for (int r = 0; r < 3; ++r) hd[r] += take[r];
    __syncwarp();
    if (lane < 3) st_release_cta(&bk->head[lane], lane == 0 ? hd[0] : (lane == 1 ? hd[1] : hd[2]));
    const unsigned op = static_cast<unsigned>(rec >> 56);
    const int u = static_cast<int>((rec >> 32) & 0xFFFFFF);
    const unsigned arg = static_cast<unsigned>(rec);
    exits += __popc(__ballot_sync(kFull, op == kRecExit));
    if (!__any_sync(kFull, op != 0u && op != kRecExit)) continue;

    fence_acq_rel_gpu();  // release: every record's writes (ordered before it at CTA scope)
    bool fin = false, comb = false, ema = false;
    if (op == kRecSelDone) {
      fin = atomicAdd(C.sel_cnt + u, 1u) == static_cast<unsigned>(p.fchunks - 1);
    } else if (op == kRecPartial || op == kRecFinDone) {
      comb = atomicAdd(C.done + u, arg) + arg == kBig;
      ema = op == kRecFinDone;
    } else if (op == kRecEmaDone) {
      atomicAdd(C.words + kCtlEmaDone, 1u);
    } else if (op == kRecCombDone) {
      atomicAdd(C.words + kCtlCombined, 1u);
    }
    if (!__any_sync(kFull, fin || comb || ema)) continue;
    fence_acq_rel_gpu();  // acquire: what the completed counts' adders published; release for the tasks

    // global tasks: the unit's predictor update, its G merges
    const int ntask = (ema ? 1 : 0) + (comb ? p.G : 0);
    const int inc = warp_inclusive_sum(ntask);
    const int all = __shfl_sync(kFull, inc, 31);
    if (all > 0) {
      unsigned pos = 0;
      if (lane == 0) pos = atomicAdd(C.words + kCtlRqTail, static_cast<unsigned>(all));
      pos = __shfl_sync(kFull, pos, 0) + static_cast<unsigned>(inc - ntask);
      for (int t = 0; t < ntask; ++t, ++pos) {
        const unsigned long long w = (ema && t == 0) ? make_task(kItemEma, u, 0, 0)
                                                     : make_task(kItemCombine, u, t - (ema ? 1 : 0), 0);
        if (pos < static_cast<unsigned>(p.rq_cap)) {
          st_relaxed64(C.rq + pos, w);
        } else {
          report(p.status, kDevWaitTimeout);  // cannot happen: the queue holds every task of a step
          atomicExch(C.words + kCtlAbort, 1u);
        }
      }
    }
    // FINISH of the units whose selection completed here: this CTA's mailbox, in lane order
    if (__any_sync(kFull, fin)) {
      unsigned m = __ballot_sync(kFull, fin);
      while (m) {
        const int l = __ffs(m) - 1;
        m &= m - 1u;
        const int fu = __shfl_sync(kFull, u, l);
        if (lane == 0) {
          bool room = fin_tail - ld_acquire_cta(&bk->fin_head) < static_cast<unsigned>(kFinBox);
          if (!room) {
            const uint64_t t0 = global_ns();
            while (!(room = fin_tail - ld_acquire_cta(&bk->fin_head) < static_cast<unsigned>(kFinBox))) {
              if (global_ns() - t0 > kWaitLimitNs) break;
              __nanosleep(64);
            }
          }
          if (room) {
            bk->fin[fin_tail % kFinBox] = static_cast<unsigned>(fu);
            st_release_cta(&bk->fin_tail, ++fin_tail);
          } else {
            report(p.status, kDevWaitTimeout);
            atomicExch(C.words + kCtlAbort, 1u);
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- the kernel
template <int D, int BS>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_step_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const FusedSmem S = fused_smem<D>(p, base);
  const FusedCtl C = ctl_view(p, p.parity);
  const int tid = threadIdx.x;

  if (blockIdx.x == 0) {  // clear the other copy of the control words for the next launch
    unsigned* other = p.ctl + static_cast<size_t>(1 - p.parity) * p.ctl_words;
    for (int i = tid; i < p.ctl_words; i += blockDim.x) other[i] = 0u;
  }
  if (tid < 3) {
    S.bk->tail[tid] = 0u;
    S.bk->head[tid] = 0u;
  }
  if (tid == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    for (int i = 0; i < p.fslots; ++i) {
      mbar_init(&S.fullK[i], 1);
      mbar_init(&S.fullV[i], 1);
      mbar_init(&S.empty[i], 1);
      reinterpret_cast<ItemDesc*>(S.aux + static_cast<size_t>(i) * kAuxBytes + kAuxDesc)->seq = kNoSeq;
    }
    S.claim[0] = 0;
    S.bk->fin_tail = 0u;
    S.bk->fin_head = 0u;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = tid >> 5;
  if (warp == kProducerWarp) {
    producer<D, BS>(p, C, S, &kmap, &vmap);
  } else if (warp == kBookWarp) {
    bookkeeper(p, C, S);
  } else {
    consumer<D, BS>(p, C, S, warp / 4);
  }
}

// ---------------------------------------------------------------- host side
void fused_geometry(Params& p, int sms) {
  p.fchunk_blocks = fused_chunk_blocks(p.units, p.maxnb, sms);
  p.fchunks = (p.maxnb + p.fchunk_blocks - 1) / p.fchunk_blocks;
  const long long n_main = static_cast<long long>(p.units) * (p.fchunks + p.P);
  const long long b = n_main / (4LL * sms);
  p.fbatch = static_cast<int>(b < 1 ? 1 : (b > 4 ? 4 : b));
  p.rq_cap = p.units * (1 + p.K + p.G);
  p.ctl_words = static_cast<int>(fused_ctl_words(p.units, p.P, p.K, p.G));
}

template <int D, int BS>
static size_t fused_smem_for(Params& p) {
  p.fslot_bytes = static_cast<int>(fused_slot_bytes<D, BS>(p));
  const long long room = 227LL * 1024 - 1024 - 128 - static_cast<long long>(sizeof(BookSmem)) -
                         2 * static_cast<long long>(group_coef_bytes<D>(p));
  const long long slots = room / (p.fslot_bytes + kAuxBytes + 24);
  p.fslots = static_cast<int>(slots < 8 ? (slots < 0 ? 0 : slots) : 8);
  return fused_smem_total(p.fslots, p.fslot_bytes, group_coef_bytes<D>(p));
}

template <int D, int BS>
static cudaError_t launch_fused_t(Params p, const CUtensorMap& kmap, const CUtensorMap& vmap, cudaStream_t s,
                                  int priority, int sms, int* grid_out) {
  fused_geometry(p, sms);
  const size_t smem = fused_smem_for<D, BS>(p);
  if (p.fslots < 2) return cudaErrorInvalidConfiguration;
  const void* fn = reinterpret_cast<const void*>(fused_step_kernel<D, BS>);
  cudaError_t e = allow_max_smem(fn);
  if (e != cudaSuccess) return e;
  if (grid_out) *grid_out = sms;
  return launch_kernel(fused_step_kernel<D, BS>, dim3(static_cast<unsigned>(sms)), dim3(kFusedThreads), smem, s,
                       priority, kmap, vmap, p);
}

cudaError_t launch_fused(const Params& p, const CUtensorMap& kmap, const CUtensorMap& vmap, cudaStream_t s,
                         int priority, int sms, int* grid_out) {
  if (p.d == 128) {
    if (p.bs == 128) return launch_fused_t<128, 128>(p, kmap, vmap, s, priority, sms, grid_out);
    return launch_fused_t<128, 64>(p, kmap, vmap, s, priority, sms, grid_out);
  }
  if (p.bs == 128) return launch_fused_t<64, 128>(p, kmap, vmap, s, priority, sms, grid_out);
  return launch_fused_t<64, 64>(p, kmap, vmap, s, priority, sms, grid_out);
}

// Shared memory the fused step needs for these dims (SIZE_MAX if fewer than two slots fit).
size_t fused_smem_bytes(const Params& p, int sms) {
  Params q = p;
  fused_geometry(q, sms);
  size_t r;
  if (p.d == 128) r = p.bs == 128 ? fused_smem_for<128, 128>(q) : fused_smem_for<128, 64>(q);
  else r = p.bs == 128 ? fused_smem_for<64, 128>(q) : fused_smem_for<64, 64>(q);
  return q.fslots < 2 ? static_cast<size_t>(-1) : r;
}

size_t fused_ctl_words_for(int units, int P, int K, int G) { return fused_ctl_words(units, P, K, G); }

}  // namespace prr

#ifdef PRR_PHASE_DEBUG
// Debug builds only: copy the per-unit phase timestamps of the finisher and predictor.
extern "C" int prr_debug_phases(void* dst) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, prr::g_phase, sizeof(prr::g_phase)));
}

extern "C" int prr_debug_items(void* dst) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, prr::g_item, sizeof(prr::g_item)));
}
#endif
