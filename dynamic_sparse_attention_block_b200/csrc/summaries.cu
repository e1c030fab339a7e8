// summaries.cu -- per-block key summaries (per-channel min and max of the keys of a
// block), built over a token range or updated for the token just appended.
//
// Dynamic sparse attention as the PRR abstract describes it attends only to the K
// highest-scoring KV blocks of each query; scoring a block needs a compact
// description of its keys.  The summary is the
// per-channel min/max pair of Quest (Query-Aware Sparsity for Efficient Long-Context
// LLM Inference, in PRR's reference list).  Values stay bf16: min and max of bf16
// inputs are exact.
#include "prr_kernels.cuh"

namespace prr {

// One CTA per (block touched by the range, unit).  128 threads: D/8 column chunks of
// 8 channels (one 16-byte load each) x 128/(D/8) row groups.
template <int D>
__global__ void __launch_bounds__(128) update_summaries_kernel(const __grid_constant__ Params p) {
  constexpr int C = D / 8;      // 16-byte column chunks per key row
  constexpr int RG = 128 / C;   // row groups
  __shared__ uint4 red_lo[RG][C];
  __shared__ uint4 red_hi[RG][C];

  const int u = blockIdx.y;
  const int b = u / p.Hkv;
  int begin, end;
  if (p.tok_begin) {
    begin = p.tok_begin[b];
    end = p.tok_end[b];
  } else {
    end = p.seq_lens[b];
    begin = end - 1;
  }
  if (begin < 0 || end > p.cap || begin > end) {
    if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, kDevBadRange);
    return;
  }
  if (begin == end) return;
  // a range longer than the call's max_range_tokens touches more blocks than the grid has
  if ((end - 1) / p.bs - begin / p.bs >= static_cast<int>(gridDim.x)) {
    if (threadIdx.x == 0 && blockIdx.x == 0) report(p.status, kDevBadRange);
    return;
  }
  const int blk = begin / p.bs + blockIdx.x;
  const int t0 = blk * p.bs;
  const int lo_t = max(begin, t0), hi_t = min(end, t0 + p.bs);
  if (lo_t >= hi_t) return;
  const bool fresh = (lo_t == t0);  // range covers the block from its first token

  const int c = threadIdx.x % C, rg = threadIdx.x / C;
  const long long r0 = kv_row(p, u, t0);  // the block's rows are contiguous in the cache
  if (r0 < 0) return;
  // +inf / -inf bf16 pairs as the identities of min / max
  __nv_bfloat162 mn[4], mx[4];
  const __nv_bfloat162 pinf = __halves2bfloat162(__ushort_as_bfloat16(0x7F80), __ushort_as_bfloat16(0x7F80));
  const __nv_bfloat162 ninf = __halves2bfloat162(__ushort_as_bfloat16(0xFF80), __ushort_as_bfloat16(0xFF80));
#pragma unroll
  for (int i = 0; i < 4; ++i) { mn[i] = pinf; mx[i] = ninf; }

  const uint16_t* base = p.kc + static_cast<size_t>(r0) * D + c * 8;
  for (int t = lo_t + rg; t < hi_t; t += RG) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t - t0) * D));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&ws[i]);
      mn[i] = __hmin2(mn[i], x);
      mx[i] = __hmax2(mx[i], x);
    }
  }
  red_lo[rg][c] = *reinterpret_cast<uint4*>(mn);
  red_hi[rg][c] = *reinterpret_cast<uint4*>(mx);
  __syncthreads();
  if (rg != 0) return;
  for (int r = 1; r < RG; ++r) {
    const uint4 a = red_lo[r][c], z = red_hi[r][c];
    const __nv_bfloat162* ap = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* zp = reinterpret_cast<const __nv_bfloat162*>(&z);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mn[i] = __hmin2(mn[i], ap[i]);
      mx[i] = __hmax2(mx[i], zp[i]);
    }
  }
  uint16_t* srow = p.summ + (static_cast<size_t>(u) * p.maxnb + blk) * 2 * D;
  uint4* dlo = reinterpret_cast<uint4*>(srow + c * 8);
  uint4* dhi = reinterpret_cast<uint4*>(srow + D + c * 8);
  if (!fresh) {  // fold in the summary of the block's earlier tokens
    const uint4 a = *dlo, z = *dhi;
    const __nv_bfloat162* ap = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* zp = reinterpret_cast<const __nv_bfloat162*>(&z);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mn[i] = __hmin2(mn[i], ap[i]);
      mx[i] = __hmax2(mx[i], zp[i]);
    }
  }
  *dlo = *reinterpret_cast<uint4*>(mn);
  *dhi = *reinterpret_cast<uint4*>(mx);
}

// Append one token per (sequence, KV head) at position seq_lens[b], then advance
// seq_lens[b].  One CTA per sequence.
template <int D>
__global__ void __launch_bounds__(128) append_kv_kernel(const Params p, const uint16_t* k_new,
                                                        const uint16_t* v_new, uint16_t* kc,
                                                        uint16_t* vc, int* seq_lens) {
  const int b = blockIdx.x;
  const int pos = seq_lens[b];
  bool ok = pos >= 0 && pos < p.cap;
  if (ok) {
    constexpr int C = D / 8;
    for (int i = threadIdx.x; i < p.Hkv * C; i += blockDim.x) {
      const int h = i / C, c = i % C;
      const long long row = kv_row(p, b * p.Hkv + h, pos);
      if (row < 0) continue;  // bad block-table entry (reported)
      const size_t src = (static_cast<size_t>(b) * p.Hkv + h) * D + c * 8;
      const size_t dst = static_cast<size_t>(row) * D + c * 8;
      *reinterpret_cast<uint4*>(kc + dst) = *reinterpret_cast<const uint4*>(k_new + src);
      *reinterpret_cast<uint4*>(vc + dst) = *reinterpret_cast<const uint4*>(v_new + src);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (ok) seq_lens[b] = pos + 1;
    else report(p.status, kDevBadSeqLen);
  }
}

cudaError_t launch_update_summaries(const Params& p, int max_range_tokens, cudaStream_t s,
                                    int priority) {
  const int nx = (max_range_tokens + p.bs - 2) / p.bs + 1;
  const dim3 grid(nx, p.units);
  if (p.d == 128) return launch_kernel(update_summaries_kernel<128>, grid, dim3(128), 0, s, priority, p);
  return launch_kernel(update_summaries_kernel<64>, grid, dim3(128), 0, s, priority, p);
}

cudaError_t launch_append_kv(const Params& p, const uint16_t* k_new, const uint16_t* v_new,
                             uint16_t* kc, uint16_t* vc, int* seq_lens, cudaStream_t s) {
  if (p.d == 128)
    return launch_kernel(append_kv_kernel<128>, dim3(p.B), dim3(128), 0, s, 0, p, k_new, v_new, kc, vc, seq_lens);
  return launch_kernel(append_kv_kernel<64>, dim3(p.B), dim3(128), 0, s, 0, p, k_new, v_new, kc, vc, seq_lens);
}

}  // namespace prr
