// prr_kernels.cuh -- internal declarations shared by the kernel translation units:
// the launch helper, the sequence-length guard and the online-softmax (m, l, O)
// merge that the last contributor of a (sequence, KV head) runs.
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

// seq_lens[b] if it lies in [1, cap], otherwise 0 (and the status word says so).
__device__ __forceinline__ int checked_len(const Params& p, int b) {
  const int n = p.seq_lens[b];
  if (n < 1 || n > p.cap) {
    if (threadIdx.x == 0) report(p.status, kDevBadSeqLen);
    return 0;
  }
  return n;
}

// Scratch the merge needs, in floats: slot list (P+K) + weights G*(P+K).
__host__ __device__ constexpr int merge_scratch_floats(int P, int K) { return (P + K) * 9 + 8; }

// LSE merge of one (sequence, KV head).  The PRR method summary has the repair step
// combine the attention of the missed blocks with the partial state of the kept
// speculative blocks through online-softmax statistics.  Inputs are the
// kept speculative partials (keep[j] = 1, slot j of pm/pl/pO) and the repair partials
// (slot i < n_missed of rm/rl/rO), all with logits in base 2:
//   m* = max m_j,  l* = sum l_j 2^(m_j - m*),  out = sum O_j 2^(m_j - m*) / l*,
//   lse = (m* + log2 l*) ln 2.
// Run by every thread of one CTA (blockDim.x threads, multiple of 32).  Partials were
// written by other CTAs: read through L2 (ld.global.cg).
template <int D>
__device__ __noinline__ void merge_unit(const Params& p, int u, float* scratch) {
  const int G = p.G, P = p.P, K = p.K;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  int* slots = reinterpret_cast<int*>(scratch);           // [P + K]
  float* wts = scratch + (P + K);                          // [G][P + K]
  int* count = reinterpret_cast<int*>(wts + G * (P + K));  // [1]
  const int nm = min(max(__ldcg(p.n_missed + u), 0), K);  // same clamp as the repair kernel
  if (warp == 0) {
    int cnt = 0;
    for (int base = 0; base < P; base += 32) {
      const int j = base + lane;
      const bool kept = j < P && __ldcg(p.keep + static_cast<size_t>(u) * P + j) != 0;
      const unsigned mask = __ballot_sync(0xFFFFFFFFu, kept);
      if (kept) slots[cnt + __popc(mask & ((1u << lane) - 1u))] = j;
      cnt += __popc(mask);
    }
    for (int i = lane; i < nm; i += 32) slots[cnt + i] = P + i;
    if (lane == 0) count[0] = cnt + nm;
  }
  __syncthreads();
  const int ns = count[0];
  // per-head max and normaliser; one warp per head
  for (int h = warp; h < G; h += nwarps) {
    const size_t row = static_cast<size_t>(u) * G + h;
    float mloc = -INFINITY;
    for (int s = lane; s < ns; s += 32) {
      const int j = slots[s];
      const float m = j < P ? __ldcg(p.pm + row * P + j) : __ldcg(p.rm + row * K + (j - P));
      wts[h * (P + K) + s] = m;
      mloc = fmaxf(mloc, m);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xFFFFFFFFu, mloc, o));
    float lsum = 0.0f;
    if (mloc == -INFINITY) {
      for (int s = lane; s < ns; s += 32) wts[h * (P + K) + s] = 0.0f;
    } else {
      for (int s = lane; s < ns; s += 32) {
        const int j = slots[s];
        const float l = j < P ? __ldcg(p.pl + row * P + j) : __ldcg(p.rl + row * K + (j - P));
        const float w = exp2f(wts[h * (P + K) + s] - mloc);
        wts[h * (P + K) + s] = w;
        lsum += l * w;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xFFFFFFFFu, lsum, o);
    __syncwarp();
    const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
    for (int s = lane; s < ns; s += 32) wts[h * (P + K) + s] *= inv;
    if (lane == 0)
      p.lse[row] = lsum > 0.0f ? (mloc + log2f(lsum)) * 0.69314718055994530942f : -INFINITY;
  }
  __syncthreads();
  // weighted sum of the numerators, 4 channels per thread
  constexpr int C4 = D / 4;
  for (int e = tid; e < G * C4; e += blockDim.x) {
    const int h = e / C4, c4 = e % C4;
    const size_t row = static_cast<size_t>(u) * G + h;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < ns; ++s) {
      const int j = slots[s];
      const float w = wts[h * (P + K) + s];
      const float4* src = j < P
          ? reinterpret_cast<const float4*>(p.pO + (row * P + j) * D) + c4
          : reinterpret_cast<const float4*>(p.rO + (row * K + (j - P)) * D) + c4;
      const float4 o = __ldcg(src);
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
    }
    reinterpret_cast<float4*>(p.out + row * D)[c4] = acc;
  }
}

// Add `add` to the merge ticket of unit u; the contributor that completes it runs the
// merge and re-arms the ticket.  Every thread of the CTA calls this.  `flag` is a
// shared int.
template <int D>
__device__ __forceinline__ void merge_ticket(const Params& p, int u, unsigned add, float* scratch,
                                             int* flag) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned old = atomicAdd(p.merge_cnt + u, add);
    *flag = (old + add == kMergeTarget) ? 1 : 0;
  }
  __syncthreads();
  if (*flag) {
    __threadfence();
    merge_unit<D>(p, u, scratch);
    __syncthreads();
    if (threadIdx.x == 0) p.merge_cnt[u] = 0u;
  }
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
size_t select_smem_bytes(int d, int list_len, int maxnb);

}  // namespace prr
