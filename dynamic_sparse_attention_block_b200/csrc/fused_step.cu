// fused_step.cu -- the whole PRR decode step in ONE persistent launch.
//
// Resident CTAs (128 threads) take work items from one atomic counter, in this order:
//   1. SEL     (unit, chunk of 32-128 blocks): tail-summary fold, block scores -> keys.
//   2. FIN     (unit): once the unit's chunks are scored, the top-K finisher; publishes
//              S_t, the missed set and the keep mask.
//   3. EMA     (unit): predictor update with S_t and Pred_{t+1}; starts copying its
//              state at once and waits for S_t, then runs while speculation streams.
//   4. SPEC    (unit, predicted slot): speculative partial of block Pred_t[slot].  A
//              speculative item that starts after its unit's selection is published
//              skips a block that selection dropped (its partial would be discarded).
//   5. REPAIR  (unit, r < R): partials of the missed blocks in slots r, r + R, ...;
//              each slot's block arrives in a descriptor word the finisher publishes.
//   6. COMBINE (unit, query head): LSE merge of kept + repaired partials (waits for all
//              of the unit's speculative and repair partials).
// This is the PRR runtime (abstract; method summary; contributions (1)-(3)) scheduled
// for a 148-SM part: speculation overlaps selection inside the launch, selection work
// is handed out first so the critical path (select -> repair -> merge) starts at once,
// and no kernel boundary separates the phases.
//
// Waits only ever target items with a smaller index, which were taken by CTAs that are
// already running, so every wait ends without any co-residency assumption.  Each wait
// is bounded (kWaitLimitNs); a timeout records kDevWaitTimeout and raises an abort flag
// that makes every later wait give up at once.
//
// Control words live in the workspace in two copies selected by the step parity: a
// launch works on copy[parity] and clears copy[1 - parity] for the next launch, so no
// reset launch is needed and a late CTA can never see the next step's counters.
#include "prr_attn.cuh"
#include "prr_parts.cuh"

namespace prr {

constexpr int kFusedChunk = 128;  // most blocks per SEL item (4 warps x 32 rows)

// Blocks per SEL item: a multiple of 32 in [32, 128], about units*maxnb/512, so that a
// short context still spreads its scan over many CTAs and a long one moves 64 KB per item.
__host__ __device__ inline int fused_chunk_blocks(int units, int maxnb) {
  long long c = (static_cast<long long>(units) * maxnb + 511) / 512;
  c = ((c + 31) / 32) * 32;
  return static_cast<int>(c < 32 ? 32 : (c > kFusedChunk ? kFusedChunk : c));
}

struct FusedCtl {
  unsigned* work;        // next item
  unsigned* abort;       // set on a timed-out wait
  unsigned* sel_loaded;  // SEL items whose summary tile has landed
  unsigned* sel_finished;  // units whose S_t is published
  unsigned* sel_cnt;     // [units] scored SEL chunks
  unsigned* sel_done;    // [units] 0, then 1 + |M_t| once S_t is published
  unsigned* p_act;       // [units] active speculative slots (published with S_t)
  unsigned* spec_done;   // [units] finished (or skipped) speculative items
  unsigned* rep_done;    // [units] finished repair items
  unsigned* keepf;       // [units][P] 0 until S_t is known, then 1 | keep << 1
  unsigned* rdesc;       // [units][K] 0 until S_t is known, then missed block + 1 or kNoRepair
};

__device__ __forceinline__ FusedCtl ctl_view(const Params& p, int parity) {
  unsigned* b = p.ctl + static_cast<size_t>(parity) * p.ctl_words;
  const int U = p.units;
  return FusedCtl{b,          b + 1,          b + 2,          b + 3,          b + 16,
                  b + 16 + U, b + 16 + 2 * U, b + 16 + 3 * U, b + 16 + 4 * U, b + 16 + 5 * U,
                  b + 16 + 5 * U + static_cast<size_t>(U) * p.P};
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// CTA-wide bounded wait until *flag >= target.  Thread 0 polls; the verdict is shared,
// and every thread gets the flag value thread 0 saw last in *seen (if given).
__device__ bool wait_geq(const unsigned* flag, unsigned target, const FusedCtl& C, int* status, int* sh,
                         unsigned* seen = nullptr) {
  if (threadIdx.x == 0) {
    int ok = 1;
    unsigned v = ld_acquire(flag);
    if (v < target) {
      const uint64_t t0 = global_ns();
      for (;;) {
        v = ld_acquire(flag);
        if (v >= target) break;
        if (ld_acquire(C.abort)) {
          ok = 0;
          break;
        }
        if (global_ns() - t0 > kWaitLimitNs) {
          report(status, kDevWaitTimeout);
          atomicExch(C.abort, 1u);
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

template <int D>
struct FusedSel {
  static constexpr int ROWB = 4 * D;
  static constexpr int C = ROWB / 16;
  __host__ __device__ static size_t aux(int maxnb) {  // coefficient area follows tiles / finisher scratch
    size_t a = static_cast<size_t>(kFusedChunk) * ROWB;
    const size_t f = finish_scratch_bytes(maxnb);
    if (f > a) a = f;
    return (a + 15) & ~static_cast<size_t>(15);
  }
  __host__ __device__ static size_t bytes(int maxnb) { return aux(maxnb) + 2 * C * 16 + 2 * D; }
};

// ---------------------------------------------------------------- SEL item
template <int D>
__device__ void sel_item(const Params& p, const FusedCtl& C, int u, int chunk, unsigned char* smem, uint64_t* bar,
                         uint32_t& ph) {
  using L = FusedSel<D>;
  constexpr int ROWB = L::ROWB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = chunk * p.fchunk_blocks;
  uint16_t* summ_unit = p.summ + static_cast<size_t>(u) * p.maxnb * 2 * D;
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
  const int n = checked_len(p, u / p.Hkv);
  const int nb = (n + p.bs - 1) / p.bs;
  const int cnt = max(0, min(p.fchunk_blocks, nb - c0));
  const int tail = n > 0 ? (n - 1) / p.bs : -1;
  const bool own_tail = p.append_summary && tail >= c0 && tail < c0 + cnt;
  const size_t aux = L::aux(p.maxnb);
  float4* coef_lo = reinterpret_cast<float4*>(smem + aux);
  float4* coef_hi = coef_lo + L::C;
  uint16_t* newk = reinterpret_cast<uint16_t*>(coef_hi + L::C);

  load_group_coef<D>(p, u, coef_lo, coef_hi);
  if (own_tail) {
    const uint16_t* krow = p.kc + (static_cast<size_t>(u) * p.cap + (n - 1)) * D;
    for (int c = tid; c < D / 8; c += blockDim.x)
      reinterpret_cast<uint4*>(newk)[c] = __ldg(reinterpret_cast<const uint4*>(krow) + c);
  }
  __syncthreads();
  if (alloc_rows > 0) {
    const bool ok = __syncthreads_and(mbar_wait(bar, ph, p.status));
    ph ^= 1u;
    if (!ok) {
      if (tid == 0) atomicExch(C.abort, 1u);
      return;
    }
  }
  if (tid == 0) atomicAdd(C.sel_loaded, 1u);  // this chunk no longer needs bandwidth
  const int first = c0 + 32 * warp;
  const int rows = min(32, cnt - 32 * warp);
  if (rows > 0) {
    unsigned char* tile = smem + warp * 32 * ROWB;
    if (own_tail && tail >= first && tail < first + rows)
      fold_tail_row<D>(reinterpret_cast<uint32_t*>(tile + (tail - first) * ROWB), newk, ((n - 1) % p.bs) == 0,
                       reinterpret_cast<uint32_t*>(summ_unit + static_cast<size_t>(tail) * 2 * D), lane);
    uint32_t key = 0u;
    if (lane < rows) {
      key = orderable(score_summary_row<D>(tile + lane * ROWB, coef_lo, coef_hi, lane));
      p.keys[static_cast<size_t>(u) * p.maxnb + first + lane] = key;
    }
    write_group_summary(p, u, first / 32, key, lane < rows);
  }
  count_done(C.sel_cnt + u);  // the unit's FIN item waits for all its chunks
}

// ---------------------------------------------------------------- FIN item
__device__ void fin_item(const Params& p, const FusedCtl& C, int u, unsigned char* smem, int* sh) {
  if (!wait_geq(C.sel_cnt + u, static_cast<unsigned>(p.fchunks), C, p.status, sh)) return;
  const int n = checked_len(p, u / p.Hkv);
  const int nb = (n + p.bs - 1) / p.bs;
  const FinishOut f = select_finish(p, u, nb, smem, C.keepf + static_cast<size_t>(u) * p.P,
                                    C.rdesc + static_cast<size_t>(u) * p.K);
  __syncthreads();  // every thread's outputs precede the release below
  if (threadIdx.x == 0) {
    C.p_act[u] = static_cast<unsigned>(f.p_active);
    st_release(C.sel_done + u, 1u + static_cast<unsigned>(f.n_missed));
    red_release_add(C.sel_finished, 1u);
  }
}

// ---------------------------------------------------------------- fused kernel
template <int D, int BS>
__global__ void __launch_bounds__(128, 3) fused_step_kernel(const __grid_constant__ CUtensorMap kmap,
                                                         const __grid_constant__ CUtensorMap vmap,
                                                         const __grid_constant__ Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.fused_region);  // K tile, V tile, summaries
  int* sh = reinterpret_cast<int*>(bars + 3);                              // broadcast slots [8]
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
  const int n_sel = U * p.fchunks, n_fin = U, n_spec = U * p.P, n_ema = U, n_rep = U * R;
  const int n_comb = U * p.G;
  const int total = n_sel + n_fin + n_spec + n_ema + n_rep + n_comb;

  // SEL, SPEC and REPAIR items take their CTA's next ticket as they start (thread 0),
  // so the streaming phases never wait for the work counter.  FIN, EMA and COMBINE
  // items do not: a long finisher or wait must not hold back a ticket that an idle CTA
  // could run.
  // Still deadlock-free: the lowest unfinished item is always being processed, because
  // a CTA holding a prefetched ticket is working on a lower item.
  constexpr unsigned kNoTicket = 0xFFFFFFFFu;
  unsigned next_ticket = kNoTicket;
  for (;;) {
    if (tid == 0) {
      sh[2] = static_cast<int>(next_ticket != kNoTicket ? next_ticket : atomicAdd(C.work, 1u));
      next_ticket = kNoTicket;
    }
    __syncthreads();
    int it = sh[2];
    __syncthreads();
    if (it >= total) break;
    fence_proxy_async();  // generic shared-memory writes of the last item precede new copies
    if (p.trace && tid == 0) {
      unsigned smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      p.trace[4 * static_cast<size_t>(it) + 0] = global_ns();
      p.trace[4 * static_cast<size_t>(it) + 2] = (static_cast<unsigned long long>(smid) << 32) | blockIdx.x;
      p.trace[4 * static_cast<size_t>(it) + 3] = static_cast<unsigned long long>(it);
    }
    const int item_id = it;

    if (it < n_sel) {
      if (tid == 0) next_ticket = atomicAdd(C.work, 1u);
      sel_item<D>(p, C, it / p.fchunks, it % p.fchunks, smem, &bars[2], ph_sel);
      __syncthreads();
      if (p.trace && tid == 0) p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
      continue;
    }
    it -= n_sel;
    if (it < n_fin) {
      fin_item(p, C, it, smem, sh);
      __syncthreads();
      if (p.trace && tid == 0) p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
      continue;
    }
    it -= n_fin;
    if (it < n_ema) {  // predictor for step t+1
      ema_unit(p, it, smem, [&] { return wait_geq(C.sel_done + it, 1u, C, p.status, sh); });
      __syncthreads();
      if (p.trace && tid == 0) p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
      continue;
    }
    it -= n_ema;
    if (it < n_spec) {  // speculation
      if (tid == 0) next_ticket = atomicAdd(C.work, 1u);
      const int u = it / p.P, j = it % p.P;
      // the predicted block, the sequence length and the slot's keep flag in one round trip
      // (the keep flag may change under us: thread 0 reads it and shares its verdict)
      if (tid == 0) sh[3] = (__ldcg(C.keepf + static_cast<size_t>(u) * p.P + j) == 1u) ? 1 : 0;
      const int blk = p.pred[static_cast<size_t>(u) * p.P + j];
      const int n = checked_len(p, u / p.Hkv);
      const int nb = (n + BS - 1) / BS;
      __syncthreads();
      bool dropped = sh[3] != 0;
      __syncthreads();
      if (blk >= 0 && blk < nb) {
        const bool skip = dropped;
        if (!skip) {
          const size_t row0 = static_cast<size_t>(u) * p.G * p.P + j;
          const PartialDst dst{p.pm + row0, p.pl + row0, p.pO + row0 * D, static_cast<size_t>(p.P),
                               static_cast<size_t>(p.P) * D};
          if (!block_partial<D, BS>(p, &kmap, &vmap, u, blk, n, dst, smem, bars, ph_attn) && tid == 0)
            atomicExch(C.abort, 1u);
          ph_attn ^= 1u;
        }
        count_done(C.spec_done + u);
      }
      __syncthreads();
      if (p.trace && tid == 0) p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
      continue;
    }
    it -= n_spec;
    if (it < n_rep) {  // repair
      if (tid == 0) next_ticket = atomicAdd(C.work, 1u);
      const int u = it / R;
      const int n = checked_len(p, u / p.Hkv);
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
          if (!block_partial<D, BS>(p, &kmap, &vmap, u, blk, n, dst, smem, bars, ph_attn) && tid == 0)
            atomicExch(C.abort, 1u);
          ph_attn ^= 1u;
        } else {
          if (tid == 0) report(p.status, kDevBadMissed);
          write_empty_partial(dst, p.G, D);
        }
        count_done(C.rep_done + u);
      }
      __syncthreads();
      if (p.trace && tid == 0) p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
      continue;
    }
    it -= n_rep;
    {  // LSE merge of (unit, head)
      const int u = it / p.G, h = it % p.G;
      unsigned flag = 0u;
      if (wait_geq(C.sel_done + u, 1u, C, p.status, sh, &flag)) {
        const unsigned nm = static_cast<unsigned>(min(static_cast<int>(flag) - 1, p.K));
        const unsigned pa = __ldcg(C.p_act + u);
        // fold the speculative partials as soon as they are all written, then the repairs
        if (wait_geq(C.spec_done + u, pa, C, p.status, sh))
          combine_head<D>(p, u, h, smem, [&] { return wait_geq(C.rep_done + u, nm, C, p.status, sh); });
      }
      __syncthreads();
      if (p.trace && tid == 0) p.trace[4 * static_cast<size_t>(item_id) + 1] = global_ns();
    }
  }
}

template <int D, int BS>
static size_t fused_region_bytes(const Params& p) {
  size_t r = FusedSel<D>::bytes(p.maxnb);
  r = r > AttnTile<D, BS>::bytes ? r : AttnTile<D, BS>::bytes;
  const size_t e = ema_scratch_bytes(p.maxnb);
  r = r > e ? r : e;
  const size_t c = combine_scratch_bytes(p.P, p.K, D);
  r = r > c ? r : c;
  return (r + 15) & ~static_cast<size_t>(15);
}

template <int D, int BS>
static cudaError_t launch_fused_t(Params p, const CUtensorMap& kmap, const CUtensorMap& vmap, cudaStream_t s,
                                  int priority, int sms, int* grid_out) {
  p.fchunk_blocks = fused_chunk_blocks(p.units, p.maxnb);
  p.fchunks = (p.maxnb + p.fchunk_blocks - 1) / p.fchunk_blocks;
  p.fused_region = static_cast<int>(fused_region_bytes<D, BS>(p));
  const size_t smem = 1024 + static_cast<size_t>(p.fused_region) + 3 * 8 + 8 * 4;
  const void* fn = reinterpret_cast<const void*>(fused_step_kernel<D, BS>);
  cudaError_t e = allow_max_smem(fn);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_step_kernel<D, BS>, 128, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long long items = static_cast<long long>(p.units) * (p.fchunks + 1 + p.P + 1 + p.rep_items + p.G);
  long long grid = static_cast<long long>(per_sm) * sms;
  if (grid > items) grid = items;
  if (grid_out) *grid_out = static_cast<int>(grid);
  return launch_kernel(fused_step_kernel<D, BS>, dim3(static_cast<unsigned>(grid)), dim3(128), smem, s, priority,
                       kmap, vmap, p);
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

size_t fused_smem_bytes(const Params& p) {
  Params q = p;
  q.fchunk_blocks = fused_chunk_blocks(q.units, q.maxnb);
  q.fchunks = (q.maxnb + q.fchunk_blocks - 1) / q.fchunk_blocks;
  size_t r;
  if (p.d == 128) r = p.bs == 128 ? fused_region_bytes<128, 128>(q) : fused_region_bytes<128, 64>(q);
  else r = p.bs == 128 ? fused_region_bytes<64, 128>(q) : fused_region_bytes<64, 64>(q);
  return 1024 + r + 3 * 8 + 8 * 4;
}

}  // namespace prr

#ifdef PRR_PHASE_DEBUG
// Debug builds only: copy the phase timestamps of the fused kernel's translation unit.
extern "C" int prr_debug_phases(void* dst) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, prr::g_phase, sizeof(prr::g_phase)));
}
#endif
