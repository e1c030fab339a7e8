// attention.cu -- standalone speculation / repair launches: one CTA per (slot, unit)
// runs block_partial (prr_attn.cuh) on Pred_t[slot] (speculation) or on missed[slot]
// (repair) and writes one (m, l, O) partial per query head.
#include "prr_attn.cuh"

namespace prr {

template <int D, int BS, int KIND>
__global__ void __launch_bounds__(128) attn_block_kernel(const __grid_constant__ CUtensorMap kmap,
                                                         const __grid_constant__ CUtensorMap vmap,
                                                         const __grid_constant__ Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnTile<D, BS>::bytes);
  const int tid = threadIdx.x;
  const int slot = blockIdx.x, u = blockIdx.y;
  const int G = p.G;
  const int n = checked_len(p, u / p.upb);
  const int nb = (n + BS - 1) / BS;

  int blk = -1;
  bool active;
  if (KIND == 0) {  // speculation: slot j of Pred_t
    blk = p.pred[static_cast<size_t>(u) * p.P + slot];
    active = blk >= 0 && blk < nb;
  } else {  // repair: slot i of the missed set
    int nm = p.n_missed[u];
    if (nm < 0 || nm > p.K) {  // a caller-supplied count outside [0, K]
      if (tid == 0 && slot == 0) report(p.status, kDevBadMissed);
      nm = nm < 0 ? 0 : p.K;
    }
    active = slot < nm;
    if (active) blk = p.missed[static_cast<size_t>(u) * p.K + slot];
  }
  if (!active) return;

  PartialDst dst;
  if (KIND == 0) {
    const size_t row0 = static_cast<size_t>(u) * G * p.P + slot;
    dst = {p.pm + row0, p.pl + row0, p.pO + row0 * D, static_cast<size_t>(p.P), static_cast<size_t>(p.P) * D};
  } else {
    const size_t row0 = static_cast<size_t>(u) * G * p.K + slot;
    dst = {p.rm + row0, p.rl + row0, p.rO + row0 * D, static_cast<size_t>(p.K), static_cast<size_t>(p.K) * D};
  }
  if (!(blk >= 0 && blk < nb)) {  // a missed entry out of range: contribute nothing
    if (tid == 0) report(p.status, kDevBadMissed);
    write_empty_partial(dst, G, D, cta_grp());
    return;
  }
  if (tid == 0) {
    bump(p.stats, KIND == 0 ? kStatSpecAttended : kStatRepaired);
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  block_partial<D, BS>(p, &kmap, &vmap, u, blk, n, dst, smem, bars, 0u, cta_grp());
}

template <int D, int BS>
static size_t attn_smem() {
  return 1024 + AttnTile<D, BS>::bytes + 2 * 8;
}

template <int D, int BS>
static cudaError_t launch_attn_t(const Params& p, const CUtensorMap& kmap, const CUtensorMap& vmap, int kind,
                                 cudaStream_t s, int priority) {
  const size_t smem = attn_smem<D, BS>();
  const int slots = kind == 0 ? p.P : p.K;
  if (slots == 0) return cudaSuccess;
  const dim3 grid(slots, p.units);
  if (kind == 0) {
    cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(attn_block_kernel<D, BS, 0>));
    if (e != cudaSuccess) return e;
    return launch_kernel(attn_block_kernel<D, BS, 0>, grid, dim3(128), smem, s, priority, kmap, vmap, p);
  }
  cudaError_t e = allow_max_smem(reinterpret_cast<const void*>(attn_block_kernel<D, BS, 1>));
  if (e != cudaSuccess) return e;
  return launch_kernel(attn_block_kernel<D, BS, 1>, grid, dim3(128), smem, s, priority, kmap, vmap, p);
}

cudaError_t launch_attention(const Params& p, const CUtensorMap& kmap, const CUtensorMap& vmap, int kind,
                             cudaStream_t s, int priority) {
  if (p.d == 128) {
    if (p.bs == 128) return launch_attn_t<128, 128>(p, kmap, vmap, kind, s, priority);
    return launch_attn_t<128, 64>(p, kmap, vmap, kind, s, priority);
  }
  if (p.bs == 128) return launch_attn_t<64, 128>(p, kmap, vmap, kind, s, priority);
  return launch_attn_t<64, 64>(p, kmap, vmap, kind, s, priority);
}

}  // namespace prr
