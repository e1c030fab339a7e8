// ema.cu -- standalone EMA predictor launch: one CTA (256 threads) per (sequence, KV
// head) runs ema_unit (prr_parts.cuh).
#include "prr_parts.cuh"

namespace prr {

__global__ void __launch_bounds__(256) ema_predict_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(16) unsigned char smem[];
  ema_unit(p, blockIdx.x, smem, [] { return true; }, cta_grp());
}

size_t ema_smem_bytes(int maxnb) { return ema_scratch_bytes(maxnb); }

cudaError_t launch_ema(const Params& p, cudaStream_t s, int priority) {
  const size_t smem = ema_scratch_bytes(p.maxnb);
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(ema_predict_kernel));
  if (e != cudaSuccess) return e;
  return launch_kernel(ema_predict_kernel, dim3(p.units), dim3(256), smem, s, priority, p);
}

}  // namespace prr
