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
// Work split: grid (chunk, unit), 256 threads.  Warps 0-3 of each CTA stream 32-block
// tiles of summaries through private 2-stage shared-memory rings (1-D TMA bulk copies)
// and score one block per lane; the order-preserving 32-bit keys go to the workspace.
// Each warp also writes its 32-block group's largest key and tie mask.  The last CTA of
// a unit to finish (atomic ticket, no waiting) selects the top K (select_finish) and
// emits the selected set in block order.
// In decode-step mode the CTA owning the block of the newly appended token first folds
// that token into the block's summary (step a1) and writes it back.
#include "prr_parts.cuh"

namespace prr {

template <int D>
struct SelectSmem {
  static constexpr int ROWB = 4 * D;        // bytes of one block summary (min row + max row)
  static constexpr int STAGE = 32 * ROWB;   // one 32-block tile
  static constexpr int C = ROWB / 16;       // 16-byte chunks per summary row
  static constexpr size_t stages = 0;       // 4 streaming warps x 2 stages
  static constexpr size_t coef = stages + 8 * STAGE;
  static constexpr size_t newk = coef + 8 * 2 * C * 16;  // coefficients: up to 8 per-head sets; then the key row
  static constexpr size_t bars = newk + 2 * D;
  static constexpr size_t misc = bars + 8 * 8;
  static constexpr size_t fin = misc + 16 * 4;  // finisher scratch
  static size_t bytes(int maxnb) { return fin + finish_scratch_bytes(maxnb); }
};

template <int D>
__global__ void __launch_bounds__(256, 1) select_topk_kernel(const __grid_constant__ Params p) {
  using L = SelectSmem<D>;
  constexpr int ROWB = L::ROWB, STAGE = L::STAGE;
  extern __shared__ __align__(1024) unsigned char smem[];
  float4* coef = reinterpret_cast<float4*>(smem + L::coef);
  uint16_t* newk = reinterpret_cast<uint16_t*>(smem + L::newk);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bars);
  int* misc = reinterpret_cast<int*>(smem + L::misc);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, u = blockIdx.y;
  const int n = checked_len(p, u / p.upb);
  const int nb = (n + p.bs - 1) / p.bs;
  const int c0 = chunk * p.chunk_blocks;
  const int cnt = max(0, min(p.chunk_blocks, nb - c0));
  const int nrounds = (cnt + 31) / 32;
  const int tail = n > 0 ? (n - 1) / p.bs : -1;
  const bool own_tail = p.append_summary && tail >= c0 && tail < c0 + cnt;
  const int kvu = u / p.kv_div;  // KV slice (several units share it under per-head selection)
  uint16_t* summ_unit = p.summ + static_cast<size_t>(kvu) * p.maxnb * 2 * D;

  const Grp grp = cta_grp();
  load_coef<D>(p, p.q + static_cast<size_t>(u) * p.G * D, coef, grp);
  const long long trow = own_tail ? kv_row(p, kvu, n - 1) : -1;
  if (own_tail && trow >= 0) {  // the appended token's key row
    const uint16_t* krow = p.kc + static_cast<size_t>(trow) * D;
    for (int c = tid; c < D / 8; c += blockDim.x)
      reinterpret_cast<uint4*>(newk)[c] = __ldg(reinterpret_cast<const uint4*>(krow) + c);
  }
  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ---- streaming + scoring (warps 0-3, private 2-stage rings)
  bool alive = true;
  if (warp < 4) {
    const unsigned char* src = reinterpret_cast<const unsigned char*>(summ_unit) + static_cast<size_t>(c0) * ROWB;
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
    uint32_t phase[2] = {0u, 0u};
    uint32_t* keys_out = p.keys + static_cast<size_t>(u) * p.maxnb;
    int it = 0;
    for (int r = warp; r < nrounds; r += 4, ++it) {
      const int s = it & 1;
      if (!__all_sync(kFull, mbar_wait(&wbar[s], phase[s], p.status))) {  // warp-uniform verdict
        alive = false;
        break;
      }
      phase[s] ^= 1u;
      pending[s] = false;
      const int first = c0 + r * 32;
      const int rows = min(32, cnt - r * 32);
      unsigned char* tile = ring + s * STAGE;
      if (own_tail && trow >= 0 && tail >= first && tail < first + rows)
        fold_tail_row<D>(reinterpret_cast<uint32_t*>(tile + (tail - first) * ROWB), newk, ((n - 1) % p.bs) == 0,
                         reinterpret_cast<uint32_t*>(summ_unit + static_cast<size_t>(tail) * 2 * D), lane);
      uint32_t key = 0u;
      if (lane < rows) {
        key = block_key(p, first + lane, nb, score_block<D>(p, tile + lane * ROWB, coef, lane, kvu, first + lane, n));
        keys_out[first + lane] = key;
      }
      write_group_summary(p, u, first / 32, key, lane < rows);
      __syncwarp();
      if (lane == 0 && r + 8 < nrounds) {
        const uint32_t bytes = min(32, cnt - (r + 8) * 32) * ROWB;
        mbar_expect_tx(&wbar[s], bytes);
        bulk_load(ring + s * STAGE, src + static_cast<size_t>(r + 8) * STAGE, bytes, &wbar[s]);
        pending[s] = true;
      }
    }
    if (!alive && lane == 0) {  // let this warp's copies in flight land (bounded)
      for (int s = 0; s < 2; ++s)
        if (pending[s]) mbar_wait(&wbar[s], phase[s], p.status);
    }
  }
  if (__syncthreads_or(!alive)) return;  // unit left unfinished; the status word says why

  // ---- chunk ticket: the last CTA of this unit selects
  __threadfence();
  __syncthreads();
  if (tid == 0) misc[0] = (atomicAdd(p.sel_cnt + u, 1u) == static_cast<unsigned>(p.nchunks - 1));
  __syncthreads();
  if (!misc[0]) return;
  __threadfence();
  if (tid == 0) p.sel_cnt[u] = 0u;
  select_finish(p, u, nb, smem + L::fin, grp);
}

size_t select_smem_bytes(int d, int maxnb) {
  return d == 128 ? SelectSmem<128>::bytes(maxnb) : SelectSmem<64>::bytes(maxnb);
}

template <int D>
static cudaError_t launch_select_t(const Params& p, cudaStream_t s, int priority) {
  const size_t smem = SelectSmem<D>::bytes(p.maxnb);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(select_topk_kernel<D>));
  if (e != cudaSuccess) return e;
  return launch_kernel(select_topk_kernel<D>, dim3(p.nchunks, p.units), dim3(256), smem, s, priority, p);
}

cudaError_t launch_select(const Params& p, cudaStream_t s, int priority) {
  return p.d == 128 ? launch_select_t<128>(p, s, priority) : launch_select_t<64>(p, s, priority);
}

}  // namespace prr
