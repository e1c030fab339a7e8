// fused_step.cu -- the whole PRR decode step in ONE persistent launch.
//
// This is the PRR runtime (abstract; method summary; contributions (1)-(3)) scheduled
// for a 148-SM part.  Resident CTAs of 128 threads (as many per SM as shared memory and
// registers allow, three for the usual shapes) take work items from one atomic
// counter, in this order:
//   1. SEL     (unit, chunk of 32-128 blocks): fold the appended key into its block's
//              summary (a1), score the chunk's blocks (a2) into keys.
//   2. FIN     (unit): once the unit's chunks are scored, the top-K finisher (a3);
//              publishes S_t, the missed set M_t = S_t \ Pred_t and the keep mask.
//   3. EMA     (unit): predictor update with S_t and Pred_{t+1} (a4); starts copying
//              its state at once and waits for S_t.
//   4. SPEC    (unit, predicted slot): speculative partial of block Pred_t[slot] (a5).
//              A speculative item that starts after its unit's selection is published
//              skips a block that selection dropped (its partial would be discarded).
//   5. REPAIR  (unit, r < R): partials of the missed blocks in slots r, r + R, ... (a6);
//              each slot's block arrives in a descriptor word the finisher publishes.
//   6. COMBINE (unit, query head): LSE merge of kept + repaired partials (a6).
// Selection work is handed out first, so the critical path (select -> repair -> merge)
// starts at once and speculation streams while it runs; a dependent item waits for
// its inputs in the CTA that took it, so a result is picked up the moment it exists.
// After the predictor updates, each unit's REPAIR and COMBINE tickets follow its SPEC
// tickets a fixed lag later (about two rounds of the resident grid), so the merges of
// the early units run while the later units still stream instead of all waiting for the
// last speculative block.
//
// Waits only ever target items with a smaller index, which were taken by CTAs that are
// already running, so every wait ends without any co-residency assumption.  The counts
// and the ticket order are defined in prr_schedule.h, which a host test enumerates.  Each wait
// is bounded (kWaitLimitNs); a timeout records PRR_DEV_WAIT_TIMEOUT and raises an abort
// flag that makes every later wait give up at once.
//
// Control words live in the workspace in two copies selected by the step parity: a
// launch works on copy[parity] and clears copy[1 - parity] for the next launch, so no
// reset launch is needed and a late CTA can never see the next step's counters.
//
// When the caller passes the step's new token (k_new, v_new), the launch appends it:
// every item works on n = seq_lens[b] + 1 tokens, the SEL chunk that owns the new
// token writes its K/V row into the cache, attention over the tail block takes that
// row from k_new/v_new (a concurrent copy may still hold the old row), and the CTA that
// finishes the launch's last merge or predictor update advances seq_lens.
#include <algorithm>

#include "prr_attn.cuh"
#include "prr_parts.cuh"
#include "prr_schedule.h"

namespace prr {

constexpr int kFusedThreads = 128;

// Control words of one copy (word offsets).
enum : int {
  kCtlWork = 0,      // next item
  kCtlAbort = 1,     // set when a bounded wait gave up
  kCtlTail = 2,      // finished merges + predictor updates (the last one ends the step)
  kCtlUnits = 16,    // per-unit words start here
};

struct FusedCtl {
  unsigned* words;       // the fixed words above
  unsigned* sel_cnt;     // [units] scored SEL chunks
  unsigned* sel_done;    // [units] 0, then 1 + |M_t| once S_t is published
  unsigned* p_act;       // [units] active speculative slots (published with S_t)
  unsigned* spec_done;   // [units] finished (or skipped) speculative items
  unsigned* rep_done;    // [units] finished repairs
  unsigned* keepf;       // [units][P] 0 until S_t is known, then 1 | keep << 1
  unsigned* rdesc;       // [units][K] 0 until S_t is known, then missed block + 1 or kNoRepair
};

__host__ __device__ inline size_t fused_ctl_words(int units, int P, int K) {
  const size_t U = static_cast<size_t>(units);
  return kCtlUnits + 5 * U + U * static_cast<size_t>(P) + U * static_cast<size_t>(K);
}

__device__ __forceinline__ FusedCtl ctl_view(const Params& p, int parity) {
  unsigned* b = p.ctl + static_cast<size_t>(parity) * p.ctl_words;
  const size_t U = p.units;
  unsigned* u0 = b + kCtlUnits;
  return FusedCtl{b, u0, u0 + U, u0 + 2 * U, u0 + 3 * U, u0 + 4 * U, u0 + 5 * U,
                  u0 + 5 * U + U * static_cast<size_t>(p.P)};
}

// CTA-wide bounded wait until *flag >= target.  Thread 0 polls; the verdict is shared,
// and every thread gets the flag value thread 0 saw last in *seen (if given).
static __device__ bool wait_geq(const unsigned* flag, unsigned target, const FusedCtl& C, int* status, int* sh,
                         unsigned* seen = nullptr) {
  if (threadIdx.x == 0) {
    int ok = 1;
    unsigned v = ld_acquire(flag);
    if (v < target) {
      const uint64_t t0 = global_ns();
      for (;;) {
        v = ld_acquire(flag);
        if (v >= target) break;
        if (ld_acquire(C.words + kCtlAbort)) {
          ok = 0;
          break;
        }
        if (global_ns() - t0 > kWaitLimitNs) {
          report(status, kDevWaitTimeout);
          atomicExch(C.words + kCtlAbort, 1u);
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    sh[0] = ok;
    sh[4] = static_cast<int>(v);
  }
  __syncthreads();
  const bool ok = sh[0] != 0;
  if (seen) *seen = static_cast<unsigned>(sh[4]);
  __syncthreads();
  return ok;
}

// Signal that this CTA's item is complete: the barrier orders every thread's writes
// before thread 0's release, which a consumer pairs with an acquire load of the counter.
__device__ __forceinline__ void count_done(unsigned* counter) {
  __syncthreads();
  if (threadIdx.x == 0) red_release_add(counter, 1u);
}

// A merge or predictor update is done; the CTA that finishes the last one of the step
// advances seq_lens when the launch appended the step's token (every item has read
// seq_lens by then: each reads it as it starts, and all of them start before the last
// merge can finish).
static __device__ void count_tail(const Params& p, const FusedCtl& C) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned total = static_cast<unsigned>(p.units) * (p.G + 1);
    if (atom_add_acq_rel(C.words + kCtlTail, 1u) + 1u == total && p.append_kv) {
      for (int b = 0; b < p.B; ++b) {
        const int n0 = p.seq_lens[b];
        if (n0 >= 0 && n0 < p.cap) const_cast<int*>(p.seq_lens)[b] = n0 + 1;
      }
    }
  }
}

template <int D>
__host__ __device__ inline size_t group_coef_bytes(const Params& p) {
  return coef_bytes(D, p.sel_max ? p.G : 1);
}

// Shared memory of a SEL item: the chunk's summary rows, then the scoring
// coefficients and the appended key row (the finisher's scratch may be larger).
template <int D>
__host__ __device__ inline size_t sel_aux_offset(const Params& p) {
  size_t a = static_cast<size_t>(kFusedChunk) * 4 * D;
  const size_t f = finish_scratch_bytes(p.maxnb);
  if (f > a) a = f;
  return (a + 15) & ~static_cast<size_t>(15);
}

// ---------------------------------------------------------------- SEL item
template <int D>
__device__ void sel_item(const Params& p, const FusedCtl& C, int u, int chunk, unsigned char* smem, uint64_t* bar,
                         uint32_t& ph, bool skip) {
  constexpr int ROWB = 4 * D;
  const Grp grp = cta_grp();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = chunk * p.fchunk_blocks;
  const int kvu = u / p.kv_div;  // KV (summary) slice: several units share it under per-head selection
  uint16_t* summ_unit = p.summ + static_cast<size_t>(kvu) * p.maxnb * 2 * D;
  if (skip) {  // failure-detection tests: the selection never completes
    __syncthreads();
    return;
  }
  // The copy covers the chunk's rows up to the allocation (not the sequence length), so
  // it starts before seq_lens has been read; rows past the last block are never used.
  const int alloc_rows = max(0, min(p.fchunk_blocks, p.maxnb - c0));
  if (tid == 0 && alloc_rows > 0) {
    fence_proxy_async();
    mbar_expect_tx(bar, static_cast<uint32_t>(alloc_rows) * ROWB);
    const unsigned char* src = reinterpret_cast<const unsigned char*>(summ_unit) + static_cast<size_t>(c0) * ROWB;
    for (int w = 0; w < 4; ++w) {
      const int rows = min(32, alloc_rows - 32 * w);
      if (rows > 0) bulk_load(smem + w * 32 * ROWB, src + static_cast<size_t>(w) * 32 * ROWB, rows * ROWB, bar);
    }
  }
  const int n = checked_len(p, u / p.upb, grp);
  const int nb = (n + p.bs - 1) / p.bs;
  const int cnt = max(0, min(p.fchunk_blocks, nb - c0));
  const int tail = n > 0 ? (n - 1) / p.bs : -1;
  const bool own_tail = p.append_summary && tail >= c0 && tail < c0 + cnt;
  float4* coef = reinterpret_cast<float4*>(smem + sel_aux_offset<D>(p));
  uint16_t* newk = reinterpret_cast<uint16_t*>(reinterpret_cast<unsigned char*>(coef) + group_coef_bytes<D>(p));

  load_coef<D>(p, p.q + static_cast<size_t>(u) * p.G * D, coef, grp);
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
  __syncthreads();
  if (alloc_rows > 0) {
    const bool ok = __syncthreads_and(mbar_wait(bar, ph, p.status));
    ph ^= 1u;
    if (!ok) {
      if (tid == 0) atomicExch(C.words + kCtlAbort, 1u);
      return;
    }
  }
  const int first = c0 + 32 * warp;
  const int wrows = min(32, cnt - 32 * warp);
  if (wrows > 0) {
    unsigned char* tile = smem + warp * 32 * ROWB;
    if (own_tail && trow >= 0 && tail >= first && tail < first + wrows)
      fold_tail_row<D>(reinterpret_cast<uint32_t*>(tile + (tail - first) * ROWB), newk, ((n - 1) % p.bs) == 0,
                       reinterpret_cast<uint32_t*>(summ_unit + static_cast<size_t>(tail) * 2 * D), lane);
    uint32_t key = 0u;
    if (lane < wrows) {
      key = block_key(p, first + lane, nb, score_block<D>(p, tile + lane * ROWB, coef, lane, kvu, first + lane, n));
      p.keys[static_cast<size_t>(u) * p.maxnb + first + lane] = key;
    }
    write_group_summary(p, u, first / 32, key, lane < wrows);
  }
  count_done(C.sel_cnt + u);  // the unit's FIN item waits for all its chunks
}

// ---------------------------------------------------------------- FIN item
static __device__ void fin_item(const Params& p, const FusedCtl& C, int u, unsigned char* smem, int* sh) {
  if (!wait_geq(C.sel_cnt + u, static_cast<unsigned>(p.fchunks), C, p.status, sh)) return;
  const int n = checked_len(p, u / p.upb, cta_grp());
  const int nb = (n + p.bs - 1) / p.bs;
  const FinishOut f = select_finish(p, u, nb, smem, cta_grp(), C.keepf + static_cast<size_t>(u) * p.P,
                                    C.rdesc + static_cast<size_t>(u) * p.K);
  __syncthreads();  // every thread's outputs precede the release below
  if (threadIdx.x == 0) {
    C.p_act[u] = static_cast<unsigned>(f.p_active);
    st_release(C.sel_done + u, 1u + static_cast<unsigned>(f.n_missed));
  }
}

// ---------------------------------------------------------------- the kernel
template <int D, int BS>
__global__ void __launch_bounds__(kFusedThreads, 3) fused_step_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                      const __grid_constant__ CUtensorMap vmap,
                                                                      const __grid_constant__ Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.fregion);  // K tile, V tile, summaries
  int* sh = reinterpret_cast<int*>(bars + 3);                        // broadcast words [8]
  const int tid = threadIdx.x;
  const FusedCtl C = ctl_view(p, p.parity);

  if (blockIdx.x == 0) {  // clear the other copy of the control words for the next launch
    unsigned* other = p.ctl + static_cast<size_t>(1 - p.parity) * p.ctl_words;
    for (int i = tid; i < p.ctl_words; i += blockDim.x) other[i] = 0u;
  }
  if (tid == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  uint32_t ph_attn = 0u, ph_sel = 0u;
  const int U = p.units;
  const int R = p.rep_items;
  const int n_sel = U * p.fchunks, n_fin = U, n_ema = U, n_spec = U * p.P, n_rep = U * R;
  const int total = n_sel + n_fin + n_ema + n_spec + n_rep + U * p.G;
  // failure-detection tests set the word after the status word: selection never completes
  const bool skip_sel = p.status != nullptr && p.status[1] != 0;

  // SEL, SPEC and REPAIR items take their CTA's next ticket as they start (thread 0),
  // so the streaming phases never wait for the work counter.  FIN, EMA and COMBINE
  // items do not: a long finisher or wait must not hold back a ticket that an idle CTA
  // could run.  Still deadlock-free: the lowest unfinished item is always being
  // processed, because a CTA holding a prefetched ticket is working on a lower item.
  constexpr unsigned kNoTicket = 0xFFFFFFFFu;
  unsigned next_ticket = kNoTicket;
  for (;;) {
    if (tid == 0) {
      sh[2] = static_cast<int>(next_ticket != kNoTicket ? next_ticket : atomicAdd(C.words + kCtlWork, 1u));
      next_ticket = kNoTicket;
    }
    __syncthreads();
    int it = sh[2];
    __syncthreads();
    if (it >= total) break;
    fence_proxy_async();  // generic shared-memory writes of the last item precede new copies
    const int item_id = it;
    int kind = 0, kind_tail = 0;
    if (p.trace && tid == 0) {
      unsigned smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      p.trace[4 * static_cast<size_t>(it) + 0] = global_ns();
      p.trace[4 * static_cast<size_t>(it) + 2] = (static_cast<unsigned long long>(smid) << 32) | blockIdx.x;
    }

    if (it < n_sel) {
      kind = 1;
      if (tid == 0) next_ticket = atomicAdd(C.words + kCtlWork, 1u);
      sel_item<D>(p, C, it / p.fchunks, it % p.fchunks, smem, &bars[2], ph_sel, skip_sel);
    } else if ((it -= n_sel) < n_fin) {
      kind = 6;
      fin_item(p, C, it, smem, sh);
    } else if ((it -= n_fin) < n_ema) {  // predictor for step t+1
      kind = 4;
      ema_unit(p, it, smem, [&] { return wait_geq(C.sel_done + it, 1u, C, p.status, sh); }, cta_grp());
      count_tail(p, C);
    } else if (!decode_tail(p.P, p.G, p.dep_lag, it - n_ema, U, R, &it, &kind_tail)) {  // speculation
      kind = 2;
      if (tid == 0) next_ticket = atomicAdd(C.words + kCtlWork, 1u);
      const int u = it / p.P, j = it % p.P;
      // the predicted block, the sequence length and the slot's keep flag in one round
      // trip (the keep flag may change under us: thread 0 reads it and shares its verdict)
      if (tid == 0) sh[3] = (__ldcg(C.keepf + static_cast<size_t>(u) * p.P + j) == 1u) ? 1 : 0;
      const int blk = p.pred[static_cast<size_t>(u) * p.P + j];
      const int n = checked_len(p, u / p.upb, cta_grp());
      const int nb = (n + BS - 1) / BS;
      __syncthreads();
      const bool dropped = sh[3] != 0;
      __syncthreads();
      if (blk >= 0 && blk < nb) {
        if (!dropped) {
          const size_t row0 = static_cast<size_t>(u) * p.G * p.P + j;
          const PartialDst dst{p.pm + row0, p.pl + row0, p.pO + row0 * D, static_cast<size_t>(p.P),
                               static_cast<size_t>(p.P) * D};
          const bool tail_new = p.append_kv && blk == (n - 1) / BS;
          const size_t kvrow = static_cast<size_t>(u / p.kv_div) * D;
          if (!block_partial<D, BS>(p, &kmap, &vmap, u, blk, n, dst, smem, bars, ph_attn, cta_grp(),
                                    tail_new ? p.k_new + kvrow : nullptr, tail_new ? p.v_new + kvrow : nullptr) &&
              tid == 0)
            atomicExch(C.words + kCtlAbort, 1u);
          ph_attn ^= 1u;
          if (tid == 0) bump(p.stats, kStatSpecAttended);
        } else if (tid == 0) {
          bump(p.stats, kStatSpecSkipped);
        }
        count_done(C.spec_done + u);
      }
    } else if (kind_tail == 3) {  // repair (it: unit * R + r)
      kind = 3;
      if (tid == 0) next_ticket = atomicAdd(C.words + kCtlWork, 1u);
      const int u = it / R;
      const int n = checked_len(p, u / p.upb, cta_grp());
      const int nb = (n + BS - 1) / BS;
      // slots r, r + R, ...: each slot's descriptor (the missed block + 1, or kNoRepair)
      // is published by the finisher, so one acquire load hands over the block
      for (int i = it % R; i < p.K; i += R) {
        unsigned desc = 0u;
        if (!wait_geq(C.rdesc + static_cast<size_t>(u) * p.K + i, 1u, C, p.status, sh, &desc)) break;
        if (desc == kNoRepair) break;
        const int blk = static_cast<int>(desc) - 1;
        const size_t row0 = static_cast<size_t>(u) * p.G * p.K + i;
        const PartialDst dst{p.rm + row0, p.rl + row0, p.rO + row0 * D, static_cast<size_t>(p.K),
                             static_cast<size_t>(p.K) * D};
        if (blk >= 0 && blk < nb) {
          const bool tail_new = p.append_kv && blk == (n - 1) / BS;
          const size_t kvrow = static_cast<size_t>(u / p.kv_div) * D;
          if (!block_partial<D, BS>(p, &kmap, &vmap, u, blk, n, dst, smem, bars, ph_attn, cta_grp(),
                                    tail_new ? p.k_new + kvrow : nullptr, tail_new ? p.v_new + kvrow : nullptr) &&
              tid == 0)
            atomicExch(C.words + kCtlAbort, 1u);
          ph_attn ^= 1u;
          if (tid == 0) bump(p.stats, kStatRepaired);
        } else {
          if (tid == 0) report(p.status, kDevBadMissed);
          write_empty_partial(dst, p.G, D, cta_grp());
        }
        count_done(C.rep_done + u);
      }
    } else {  // LSE merge of (unit, head) (it: unit * G + h)
      kind = 5;
      const int u = it / p.G, h = it % p.G;
      unsigned flag = 0u;
      if (wait_geq(C.sel_done + u, 1u, C, p.status, sh, &flag)) {
        const unsigned nm = static_cast<unsigned>(min(static_cast<int>(flag) - 1, p.K));
        const unsigned pa = __ldcg(C.p_act + u);
        // fold the speculative partials as soon as they are all written, then the repairs
        if (wait_geq(C.spec_done + u, pa, C, p.status, sh))
          combine_head<D>(p, u, h, smem, [&] { return wait_geq(C.rep_done + u, nm, C, p.status, sh); },
                          cta_grp());
      }
      count_tail(p, C);
    }
    __syncthreads();
    if (p.trace && tid == 0) {
      p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
      p.trace[4 * static_cast<size_t>(item_id) + 3] = static_cast<unsigned long long>(kind);
    }
  }
}

// ---------------------------------------------------------------- host side
template <int D, int BS>
static size_t fused_region_bytes(const Params& p) {
  size_t r = sel_aux_offset<D>(p) + group_coef_bytes<D>(p) + 2 * D;
  r = std::max(r, AttnTile<D, BS>::bytes);
  r = std::max(r, ema_scratch_bytes(p.maxnb));
  r = std::max(r, combine_scratch_bytes(p.P, D));
  return (r + 15) & ~static_cast<size_t>(15);
}

void fused_geometry(Params& p, int sms) {
  (void)sms;
  p.fchunk_blocks = fused_chunk_blocks(p.units, p.maxnb);
  p.fchunks = (p.maxnb + p.fchunk_blocks - 1) / p.fchunk_blocks;
  p.rep_items = fused_rep_items(p.units, p.K);
  p.ctl_words = static_cast<int>(fused_ctl_words(p.units, p.P, p.K));
}

template <int D, int BS>
static size_t fused_smem_for(Params& p) {
  p.fregion = static_cast<int>(fused_region_bytes<D, BS>(p));
  return 1024 + static_cast<size_t>(p.fregion) + 3 * 8 + 8 * 4;
}

template <int D, int BS>
static cudaError_t launch_fused_t(Params p, const CUtensorMap& kmap, const CUtensorMap& vmap, cudaStream_t s,
                                  int priority, int sms, int* grid_out) {
  fused_geometry(p, sms);
  const size_t smem = fused_smem_for<D, BS>(p);
  const void* fn = reinterpret_cast<const void*>(fused_step_kernel<D, BS>);
  cudaError_t e = allow_max_smem(fn);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_step_kernel<D, BS>, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long long items = fused_total_items(p.units, p.fchunks, p.P, p.rep_items, p.G);
  long long grid = static_cast<long long>(per_sm) * sms;
  if (grid > items) grid = items;
  if (grid_out) *grid_out = static_cast<int>(grid);
  // dependent tickets about two rounds of the grid after their unit's SPEC tickets
  p.dep_lag = fused_dep_lag(grid, p.P, p.units);
  return launch_kernel(fused_step_kernel<D, BS>, dim3(static_cast<unsigned>(grid)), dim3(kFusedThreads), smem, s,
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

// Shared memory the fused step needs for these dims.
size_t fused_smem_bytes(const Params& p, int sms) {
  Params q = p;
  fused_geometry(q, sms);
  if (p.d == 128) return p.bs == 128 ? fused_smem_for<128, 128>(q) : fused_smem_for<128, 64>(q);
  return p.bs == 128 ? fused_smem_for<64, 128>(q) : fused_smem_for<64, 64>(q);
}

size_t fused_ctl_words_for(int units, int P, int K, int G) {
  (void)G;
  return fused_ctl_words(units, P, K);
}

}  // namespace prr

#ifdef PRR_PHASE_DEBUG
// Debug builds only: copy the per-unit phase timestamps of the finisher and predictor.
extern "C" int prr_debug_phases(void* dst) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, prr::g_phase, sizeof(prr::g_phase)));
}
#endif
