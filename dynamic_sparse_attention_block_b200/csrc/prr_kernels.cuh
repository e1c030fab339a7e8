// prr_kernels.cuh -- internal declarations shared by the kernel translation units:
// the launch helper, the shared-memory ceiling helper, the sequence-length guard and
// the host launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

#include "prr_device.cuh"
#include "prr_params.h"

namespace prr {

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, int priority, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributePriority;
  attr[0].val.priority = priority;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory ceiling to the per-CTA maximum, once per
// (kernel, device).  Kept out of the launch path so that launches stay capturable.
cudaError_t allow_max_smem(const void* kernel);

// Tokens n of sequence b this launch works on -- seq_lens[b], plus the token the fused
// step appends itself -- if n lies in [1, cap], otherwise 0 (and the status word says so).
__device__ __forceinline__ int checked_len(const Params& p, int b, const Grp& g) {
  const int n = p.seq_lens[b] + p.append_kv;
  if (n < 1 || n > p.cap) {
    if (g.tid == 0) report(p.status, kDevBadSeqLen);
    return 0;
  }
  return n;
}

__device__ __forceinline__ int checked_len(const Params& p, int b) { return checked_len(p, b, cta_grp()); }

// Row of token t of KV slice kvu (a (sequence, KV head) pair) in the cache, counted in
// rows of d elements: contiguous [B][Hkv][cap][d], or paged through the block table
// ([pages][Hkv][bs][d]).  -1 (and PRR_DEV_BAD_RANGE) for a table entry outside the pool.
__device__ __forceinline__ long long kv_row(const Params& p, int kvu, int t) {
  if (!p.table) return static_cast<long long>(kvu) * p.cap + t;
  const int b = kvu / p.Hkv, h = kvu % p.Hkv;
  const int pg = p.table[static_cast<size_t>(b) * p.maxnb + t / p.bs];
  if (pg < 0 || pg >= p.pages) {
    report(p.status, kDevBadRange);
    return -1;
  }
  return (static_cast<long long>(pg) * p.Hkv + h) * p.bs + t % p.bs;
}

// TMA coordinates of block blk of KV slice kvu: the tile's first token (*tok0) and its
// slice (the tensor maps' third coordinate).  A table entry outside the pool reports
// PRR_DEV_BAD_RANGE and yields a slice past the map, whose copy lands zeros.
__device__ __forceinline__ int kv_tile(const Params& p, int kvu, int blk, int* tok0) {
  if (!p.table) {
    *tok0 = blk * p.bs;
    return kvu;
  }
  *tok0 = 0;
  const int b = kvu / p.Hkv, h = kvu % p.Hkv;
  const int pg = p.table[static_cast<size_t>(b) * p.maxnb + blk];
  if (pg < 0 || pg >= p.pages) {
    report(p.status, kDevBadRange);
    return p.pages * p.Hkv;
  }
  return pg * p.Hkv + h;
}

// launchers (host)
cudaError_t launch_update_summaries(const Params& p, int max_range_tokens, cudaStream_t s,
                                    int priority);
cudaError_t launch_append_kv(const Params& p, const uint16_t* k_new, const uint16_t* v_new,
                             uint16_t* kc, uint16_t* vc, int* seq_lens, cudaStream_t s);
cudaError_t launch_select(const Params& p, cudaStream_t s, int priority);
cudaError_t launch_ema(const Params& p, cudaStream_t s, int priority);
cudaError_t launch_attention(const Params& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                             int kind, cudaStream_t s, int priority);
cudaError_t launch_combine(const Params& p, cudaStream_t s, int priority);
cudaError_t launch_fused(const Params& p, const CUtensorMap& kmap, const CUtensorMap& vmap, cudaStream_t s,
                         int priority, int sms, int* grid_out);
size_t fused_smem_bytes(const Params& p, int sms);
size_t fused_ctl_words_for(int units, int P, int K, int G);
void fused_geometry(Params& p, int sms);
size_t select_smem_bytes(int d, int maxnb);
size_t ema_smem_bytes(int maxnb);

}  // namespace prr
