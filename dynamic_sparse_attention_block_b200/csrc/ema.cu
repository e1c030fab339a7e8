// ema.cu -- the EMA predictor: update the per-block moving average with the true
// selected set S_t and emit the predicted set for the next step.
//
// PRR abstract and method summary: a lightweight predictor built on an exponential
// moving average of past selections forecasts the next step's top-K blocks.  The
// pages print no formula; the reading taken here is
//   e_b <- alpha*e_b + beta*[b in S_t],  beta = 1 - alpha,  e starts at 0,
// evaluated in fp64 with separately rounded multiplies and add (no fused multiply-
// add), so the state and the predicted set are bit-exact against the fp64 CPU
// oracle.  Pred_{t+1} = the min(P, nb) best blocks under (e desc, index asc), written
// in ascending block order, -1 beyond.
//
// One CTA (8 warps) per (sequence, KV head); each warp keeps a sorted register list
// of the best N = 32R >= P (value, index) pairs, merged across warps at the end.
#include "prr_kernels.cuh"

namespace prr {

template <int R>
__global__ void __launch_bounds__(256) ema_predict_kernel(const __grid_constant__ Params p) {
  constexpr int N = 32 * R;
  constexpr int NW = 8;
  extern __shared__ __align__(16) unsigned char smem[];
  const int W = (p.maxnb + 31) / 32;
  unsigned* bm = reinterpret_cast<unsigned*>(smem);
  EmaKey* lists = reinterpret_cast<EmaKey*>(smem + ((static_cast<size_t>(W) * 4 + 15) & ~static_cast<size_t>(15)));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x;
  const int n = checked_len(p, u / p.Hkv);
  const int nb = (n + p.bs - 1) / p.bs;
  double* e = p.ema + static_cast<size_t>(u) * p.maxnb;
  const bool update = p.sel != nullptr;

  if (update) {
    for (int i = tid; i < W; i += blockDim.x) bm[i] = 0u;
    __syncthreads();
    for (int i = tid; i < p.K; i += blockDim.x) {
      const int v = p.sel[static_cast<size_t>(u) * p.K + i];
      if (v >= 0 && v < nb) atomicOr(&bm[v >> 5], 1u << (v & 31));
    }
    __syncthreads();
  }
  const double alpha = p.alpha;
  const double beta = __dsub_rn(1.0, alpha);

  const EmaKey empty = {0ull, 0xFFFFFFFFu};
  EmaKey list[R];
#pragma unroll
  for (int r = 0; r < R; ++r) list[r] = empty;
  for (int base = warp * 32; base < nb; base += NW * 32) {
    const int idx = base + lane;
    EmaKey k = empty;
    if (idx < nb) {
      double x = e[idx];
      if (update) {
        const double ind = ((bm[idx >> 5] >> (idx & 31)) & 1u) ? 1.0 : 0.0;
        x = __dadd_rn(__dmul_rn(alpha, x), __dmul_rn(beta, ind));
        e[idx] = x;
      }
      k.ev = static_cast<uint64_t>(__double_as_longlong(x)) + 1ull;  // e >= 0: bits order as values
      k.idx = static_cast<uint32_t>(idx);
    }
    const EmaKey worst = shfl_idx(list[R - 1], 31);
    if (__any_sync(0xFFFFFFFFu, better(k, worst))) insert32<R>(list, k);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) lists[warp * N + r * 32 + lane] = list[r];
  __syncthreads();
  if (warp != 0) return;
  for (int w = 1; w < NW; ++w) {
    EmaKey o[R];
#pragma unroll
    for (int r = 0; r < R; ++r) o[r] = lists[w * N + r * 32 + lane];
    merge_sorted<R>(list, o);
  }
  const int peff = min(p.P, nb);
  uint64_t ord[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int el = r * 32 + lane;
    ord[r] = el < peff ? static_cast<uint64_t>(0xFFFFFFFFu - list[r].idx) + 1ull : 0ull;
  }
  bitonic_sort<R>(ord);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int el = r * 32 + lane;
    if (el < p.P)
      p.pred_next[static_cast<size_t>(u) * p.P + el] =
          ord[r] ? static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(ord[r] - 1ull)) : -1;
  }
}

static size_t ema_smem_bytes(int R, int maxnb) {
  const size_t W = static_cast<size_t>((maxnb + 31) / 32);
  return ((W * 4 + 15) & ~static_cast<size_t>(15)) + 8 * 32 * R * sizeof(EmaKey);
}

template <int R>
static cudaError_t launch_ema_t(const Params& p, cudaStream_t s, int priority) {
  const size_t smem = ema_smem_bytes(R, p.maxnb);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(ema_predict_kernel<R>));
  if (e != cudaSuccess) return e;
  return launch_kernel(ema_predict_kernel<R>, dim3(p.units), dim3(256), smem, s, priority, p);
}

cudaError_t launch_ema(const Params& p, cudaStream_t s, int priority) {
  const int R = p.P <= 32 ? 1 : (p.P <= 64 ? 2 : 4);
  if (R == 1) return launch_ema_t<1>(p, s, priority);
  if (R == 2) return launch_ema_t<2>(p, s, priority);
  return launch_ema_t<4>(p, s, priority);
}

}  // namespace prr
