// select_topk.cu -- block scoring fused with top-K selection, the missed set and the
// keep mask of the predicted slots.
//
// Score (Quest's channel-wise bound, summed over the GQA group -- the group shares
// one selection per KV head):
//   s_b = sum_h sum_c max(q_hc*min_bc, q_hc*max_bc)
//       = sum_c (sum_h max(q_hc,0)) * max_bc + (sum_h min(q_hc,0)) * min_bc
// so one block costs 2d fused multiply-adds against its 2d summary values whatever the
// group size.  On the dyadic {-8..8}/8 grid every product is a multiple of 1/64 and
// every partial sum stays below 2^24 units of 1/64, so the fp32 score is exact in any
// order.  True selected set (PRR abstract): the K best blocks under (score desc, index
// asc).  Missed set M = S \ Pred and keep[j] = [Pred_j in S] drive reuse and repair
// (PRR method summary, contributions (2)-(3)).
//
// Work split: grid (chunk, unit).  Each CTA owns `chunk_blocks` consecutive blocks of
// one (sequence, KV head); each of its 4 warps streams 32-block tiles of summaries into
// its own 2-stage shared-memory ring with 1-D TMA bulk copies, scores one block per
// lane and keeps a sorted top-N list (N = 32R >= K) in registers.  The CTA's list goes
// to the workspace; the last CTA of the unit to finish (atomic ticket, no waiting)
// merges the unit's lists and writes the outputs.
#include "prr_kernels.cuh"

namespace prr {

template <int D, int R>
struct SelectSmem {
  static constexpr int N = 32 * R;
  static constexpr int ROWB = 4 * D;        // bytes of one block summary (min row + max row)
  static constexpr int STAGE = 32 * ROWB;   // one 32-block tile
  static constexpr int C = ROWB / 16;       // 16-byte chunks per summary row
  static constexpr size_t stages = 0;
  static constexpr size_t coef = stages + 8 * STAGE;           // 4 warps x 2 stages
  static constexpr size_t lists = coef + 2 * C * 16;           // float4 lo/hi per chunk
  static constexpr size_t bars = lists + 4 * N * 8;
  static constexpr size_t misc = bars + 8 * 8;
  static constexpr size_t bitmaps = misc + 8 * 4;
  static size_t bytes(int maxnb) { return bitmaps + 2 * static_cast<size_t>((maxnb + 31) / 32) * 4; }
};

template <int D, int R>
__global__ void __launch_bounds__(128, 1) select_topk_kernel(const __grid_constant__ Params p) {
  using L = SelectSmem<D, R>;
  constexpr int N = L::N, ROWB = L::ROWB, STAGE = L::STAGE, C = L::C;
  extern __shared__ __align__(1024) unsigned char smem[];
  float4* coef_lo = reinterpret_cast<float4*>(smem + L::coef);
  float4* coef_hi = coef_lo + C;
  uint64_t* lists = reinterpret_cast<uint64_t*>(smem + L::lists);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  int* misc = reinterpret_cast<int*>(smem + L::misc);
  const int W = (p.maxnb + 31) / 32;
  unsigned* bm_pred = reinterpret_cast<unsigned*>(smem + L::bitmaps);
  unsigned* bm_sel = bm_pred + W;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, u = blockIdx.y;
  const int n = checked_len(p, u / p.Hkv);
  const int nb = (n + p.bs - 1) / p.bs;
  const int c0 = chunk * p.chunk_blocks;
  const int cnt = max(0, min(p.chunk_blocks, nb - c0));
  const int nrounds = (cnt + 31) / 32;

  // group coefficients: element e of the [min | max] summary row multiplies coef[e]
  {
    float* lo = reinterpret_cast<float*>(coef_lo);
    float* hi = reinterpret_cast<float*>(coef_hi);
    const uint16_t* qg = p.q + static_cast<size_t>(u) * p.G * D;
    for (int c = tid; c < D; c += blockDim.x) {
      float neg = 0.f, pos = 0.f;
      for (int h = 0; h < p.G; ++h) {
        const float x = __uint_as_float(static_cast<uint32_t>(qg[h * D + c]) << 16);
        neg += fminf(x, 0.f);
        pos += fmaxf(x, 0.f);
      }
      const int e0 = c, e1 = D + c;  // min part, max part
      ((e0 & 7) < 4 ? lo[(e0 >> 3) * 4 + (e0 & 3)] : hi[(e0 >> 3) * 4 + (e0 & 3)]) = neg;
      ((e1 & 7) < 4 ? lo[(e1 >> 3) * 4 + (e1 & 3)] : hi[(e1 >> 3) * 4 + (e1 & 3)]) = pos;
    }
  }
  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  const unsigned char* src = reinterpret_cast<const unsigned char*>(p.summ) +
                             (static_cast<size_t>(u) * p.maxnb + c0) * ROWB;
  unsigned char* ring = smem + L::stages + warp * 2 * STAGE;
  uint64_t* wbar = bars + warp * 2;
  bool pending[2] = {false, false};
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int r = warp + 4 * s;
      if (r < nrounds) {
        const uint32_t bytes = min(32, cnt - r * 32) * ROWB;
        mbar_expect_tx(&wbar[s], bytes);
        bulk_load(ring + s * STAGE, src + static_cast<size_t>(r) * STAGE, bytes, &wbar[s]);
        pending[s] = true;
      }
    }
  }

  uint64_t list[R];
#pragma unroll
  for (int r = 0; r < R; ++r) list[r] = 0ull;
  uint32_t phase[2] = {0u, 0u};
  bool alive = true;
  int it = 0;
  for (int r = warp; r < nrounds; r += 4, ++it) {
    const int s = it & 1;
    if (!mbar_wait(&wbar[s], phase[s], p.status)) {
      alive = false;
      break;
    }
    phase[s] ^= 1u;
    pending[s] = false;
    const int rows = min(32, cnt - r * 32);
    uint64_t key = 0ull;
    if (lane < rows) {
      const unsigned char* row = ring + s * STAGE + lane * ROWB;
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < C; ++i) {
        const int cc = (i + lane) & (C - 1);  // rotated start: conflict-free rows
        const uint4 w = *reinterpret_cast<const uint4*>(row + cc * 16);
        const float4 a = coef_lo[cc], z = coef_hi[cc];
        acc = fmaf(a.x, bf16_lo(w.x), acc);
        acc = fmaf(a.y, bf16_hi(w.x), acc);
        acc = fmaf(a.z, bf16_lo(w.y), acc);
        acc = fmaf(a.w, bf16_hi(w.y), acc);
        acc = fmaf(z.x, bf16_lo(w.z), acc);
        acc = fmaf(z.y, bf16_hi(w.z), acc);
        acc = fmaf(z.z, bf16_lo(w.w), acc);
        acc = fmaf(z.w, bf16_hi(w.w), acc);
      }
      key = score_key(acc, c0 + r * 32 + lane);
    }
    __syncwarp();
    if (lane == 0 && r + 8 < nrounds) {
      const uint32_t bytes = min(32, cnt - (r + 8) * 32) * ROWB;
      mbar_expect_tx(&wbar[s], bytes);
      bulk_load(ring + s * STAGE, src + static_cast<size_t>(r + 8) * STAGE, bytes, &wbar[s]);
      pending[s] = true;
    }
    const uint64_t worst = shfl_idx(list[R - 1], 31);
    if (__any_sync(0xFFFFFFFFu, key > worst)) insert32<R>(list, key);
  }
  if (__syncthreads_or(!alive)) {
    // a copy did not land in time: let this warp's copies in flight finish (bounded)
    // before the CTA gives up its shared memory, then leave the unit unfinished.
    if (lane == 0) {
      for (int s = 0; s < 2; ++s)
        if (pending[s]) mbar_wait(&wbar[s], phase[s], p.status);
    }
    return;
  }

  // CTA top-N: warp 0 merges the four warp lists
#pragma unroll
  for (int r = 0; r < R; ++r) lists[warp * N + r * 32 + lane] = list[r];
  __syncthreads();
  if (warp == 0) {
    for (int w = 1; w < 4; ++w) {
      uint64_t o[R];
#pragma unroll
      for (int r = 0; r < R; ++r) o[r] = lists[w * N + r * 32 + lane];
      merge_sorted<R>(list, o);
    }
    uint64_t* dst = p.cand + (static_cast<size_t>(u) * p.nchunks + chunk) * N;
#pragma unroll
    for (int r = 0; r < R; ++r) dst[r * 32 + lane] = list[r];
  }

  // chunk ticket: the last CTA of this unit finishes the selection
  __threadfence();
  __syncthreads();
  if (tid == 0) misc[0] = (atomicAdd(p.sel_cnt + u, 1u) == static_cast<unsigned>(p.nchunks - 1));
  __syncthreads();
  if (!misc[0]) return;
  __threadfence();
  if (tid == 0) p.sel_cnt[u] = 0u;

  const int used = (nb + p.chunk_blocks - 1) / p.chunk_blocks;
#pragma unroll
  for (int r = 0; r < R; ++r) list[r] = 0ull;
  for (int c = warp; c < used; c += 4) {
    const uint64_t* cl = p.cand + (static_cast<size_t>(u) * p.nchunks + c) * N;
    uint64_t o[R];
#pragma unroll
    for (int r = 0; r < R; ++r) o[r] = __ldcg(cl + r * 32 + lane);
    merge_sorted<R>(list, o);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) lists[warp * N + r * 32 + lane] = list[r];
  for (int i = tid; i < W; i += blockDim.x) {
    bm_pred[i] = 0u;
    bm_sel[i] = 0u;
  }
  __syncthreads();

  const int keff = min(p.K, nb);
  int sel_idx[R];
  if (warp == 0) {
    for (int w = 1; w < 4; ++w) {
      uint64_t o[R];
#pragma unroll
      for (int r = 0; r < R; ++r) o[r] = lists[w * N + r * 32 + lane];
      merge_sorted<R>(list, o);
    }
    // the K best, re-sorted by ascending block index
    uint64_t ord[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = r * 32 + lane;
      ord[r] = e < keff ? static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(key_index(list[r]))) + 1ull
                        : 0ull;
    }
    bitonic_sort<R>(ord);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int e = r * 32 + lane;
      const int idx = ord[r] ? static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(ord[r] - 1ull)) : -1;
      sel_idx[r] = idx;
      if (e < p.K) p.sel[static_cast<size_t>(u) * p.K + e] = idx;
      if (idx >= 0) atomicOr(&bm_sel[idx >> 5], 1u << (idx & 31));
    }
  }
  // predicted slots: active iff 0 <= Pred_j < nb (the speculation kernel uses the same rule)
  int active = 0, pv = -1;
  if (tid < p.P) {
    pv = p.pred[static_cast<size_t>(u) * p.P + tid];
    active = (pv >= 0 && pv < nb) ? 1 : 0;
    if (active) {
      atomicOr(&bm_pred[pv >> 5], 1u << (pv & 31));
      if (tid > 0 && p.pred[static_cast<size_t>(u) * p.P + tid - 1] >= pv) report(p.status, kDevBadPred);
    } else if (pv != -1) {
      report(p.status, kDevBadPred);
    }
  }
  const int p_active = __syncthreads_count(active);
  if (warp == 0) {
    int base = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int idx = sel_idx[r];
      const bool miss = idx >= 0 && !((bm_pred[idx >> 5] >> (idx & 31)) & 1u);
      const unsigned mask = __ballot_sync(0xFFFFFFFFu, miss);
      if (miss) p.missed[static_cast<size_t>(u) * p.K + base + __popc(mask & ((1u << lane) - 1u))] = idx;
      base += __popc(mask);
    }
    for (int e = base + lane; e < p.K; e += 32) p.missed[static_cast<size_t>(u) * p.K + e] = -1;
    if (lane == 0) {
      p.n_missed[u] = base;
      misc[2] = base;
    }
  }
  if (tid < p.P)
    p.keep[static_cast<size_t>(u) * p.P + tid] =
        (active && ((bm_sel[pv >> 5] >> (pv & 31)) & 1u)) ? 1 : 0;
  __syncthreads();
  if (p.mode == MODE_STEP) {
    // selection's share of the merge ticket: everything except one per active
    // speculative slot and one per repair item
    const unsigned add = kMergeTarget - static_cast<unsigned>(p_active + misc[2]);
    merge_ticket<D>(p, u, add, reinterpret_cast<float*>(smem + L::stages), &misc[3]);
  }
}

size_t select_smem_bytes(int d, int list_len, int maxnb) {
  const int R = list_len / 32;
  if (d == 128) {
    if (R == 1) return SelectSmem<128, 1>::bytes(maxnb);
    if (R == 2) return SelectSmem<128, 2>::bytes(maxnb);
    return SelectSmem<128, 4>::bytes(maxnb);
  }
  if (R == 1) return SelectSmem<64, 1>::bytes(maxnb);
  if (R == 2) return SelectSmem<64, 2>::bytes(maxnb);
  return SelectSmem<64, 4>::bytes(maxnb);
}

template <int D, int R>
static cudaError_t launch_select_t(const Params& p, cudaStream_t s, int priority) {
  const size_t smem = SelectSmem<D, R>::bytes(p.maxnb);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(select_topk_kernel<D, R>));
  if (e != cudaSuccess) return e;
  return launch_kernel(select_topk_kernel<D, R>, dim3(p.nchunks, p.units), dim3(128), smem, s, priority, p);
}

cudaError_t launch_select(const Params& p, cudaStream_t s, int priority) {
  const int R = p.list_len / 32;
  if (p.d == 128) {
    if (R == 1) return launch_select_t<128, 1>(p, s, priority);
    if (R == 2) return launch_select_t<128, 2>(p, s, priority);
    return launch_select_t<128, 4>(p, s, priority);
  }
  if (R == 1) return launch_select_t<64, 1>(p, s, priority);
  if (R == 2) return launch_select_t<64, 2>(p, s, priority);
  return launch_select_t<64, 4>(p, s, priority);
}

}  // namespace prr
