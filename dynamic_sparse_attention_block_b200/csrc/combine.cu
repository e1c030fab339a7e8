// combine.cu -- standalone LSE merge launch: one CTA (4 warps) per (query head of the
// group, unit) runs combine_head (prr_parts.cuh).
#include "prr_parts.cuh"

namespace prr {

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(16) unsigned char smem[];
  combine_head<D>(p, blockIdx.y, blockIdx.x, smem, [] { return true; }, cta_grp());
}

cudaError_t launch_combine(const Params& p, cudaStream_t s, int priority) {
  const dim3 grid(p.G, p.units);
  const size_t smem = combine_scratch_bytes(p.P, p.d);
  if (p.d == 128) return launch_kernel(combine_kernel<128>, grid, dim3(128), smem, s, priority, p);
  return launch_kernel(combine_kernel<64>, grid, dim3(128), smem, s, priority, p);
}

}  // namespace prr
