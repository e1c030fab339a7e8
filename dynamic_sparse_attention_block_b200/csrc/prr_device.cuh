// prr_device.cuh -- device-side building blocks for the PRR decode-step kernels
// (sm_100a): inline-PTX wrappers for mbarrier / TMA bulk copies / ldmatrix /
// mma.sync / movmatrix, bounded waits that report through the workspace status word,
// and warp-register bitonic lists used for top-K selection and EMA prediction.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "prr_params.h"

namespace prr {

// ------------------------------------------------------------------ small helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Record a device-side error code (first writer wins; never traps).
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ mbarrier + TMA

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

// make barrier initialisation visible to the async (TMA) proxy
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}

// Wait for the barrier's phase to complete, giving up after kWaitLimitNs.  On time-out
// the status word records kDevWaitTimeout and false is returned; callers then
// skip the dependent work (they never touch a buffer a copy may still be writing).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t phase, int* status) {
  if (mbar_try_wait(bar, phase)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, phase)) {
    if (global_ns() - t0 > kWaitLimitNs) {
      report(status, kDevWaitTimeout);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 3-D tiled TMA load (box described by the tensor map), completion on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ tensor-core fragments

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// transpose of an 8x8 b16 matrix held one row-pair per thread (fragment layout)
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ------------------------------------------------------------------ ranking keys

// Order-preserving map of an fp32 score onto uint32 (larger float -> larger integer).
// -0.0 is folded onto +0.0 first so that equal scores tie.
__device__ __forceinline__ uint32_t orderable(float s) {
  if (s == 0.0f) s = 0.0f;
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Higher key ranks first: score descending, then block index ascending.  0 = empty.
__device__ __forceinline__ uint64_t score_key(float s, int idx) {
  return (static_cast<uint64_t>(orderable(s)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int key_index(uint64_t k) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
}

// EMA ranking element: value descending, then index ascending; ev == 0 is empty.
struct EmaKey {
  uint64_t ev;   // bit pattern of e (e >= 0) plus one
  uint32_t idx;
};

__device__ __forceinline__ bool better(uint64_t a, uint64_t b) { return a > b; }
__device__ __forceinline__ bool better(const EmaKey& a, const EmaKey& b) {
  return a.ev != b.ev ? a.ev > b.ev : a.idx < b.idx;
}
__device__ __forceinline__ uint64_t shfl_xor(uint64_t v, int m) {
  return __shfl_xor_sync(0xFFFFFFFFu, v, m);
}
__device__ __forceinline__ EmaKey shfl_xor(const EmaKey& v, int m) {
  EmaKey r;
  r.ev = __shfl_xor_sync(0xFFFFFFFFu, v.ev, m);
  r.idx = __shfl_xor_sync(0xFFFFFFFFu, v.idx, m);
  return r;
}
__device__ __forceinline__ uint64_t shfl_idx(uint64_t v, int src) {
  return __shfl_sync(0xFFFFFFFFu, v, src);
}
__device__ __forceinline__ EmaKey shfl_idx(const EmaKey& v, int src) {
  EmaKey r;
  r.ev = __shfl_sync(0xFFFFFFFFu, v.ev, src);
  r.idx = __shfl_sync(0xFFFFFFFFu, v.idx, src);
  return r;
}
template <typename T>
__device__ __forceinline__ T pick_better(const T& a, const T& b) {
  return better(a, b) ? a : b;
}
template <typename T>
__device__ __forceinline__ T pick_worse(const T& a, const T& b) {
  return better(a, b) ? b : a;
}

// ------------------------------------------------------------------ warp bitonic lists
//
// A list of N = 32*R elements lives in one warp: element e = r*32 + lane is register r
// of that lane.  "Sorted" means best first.

// Bitonic half-cleaner cascade: turns a bitonic list into a sorted one (best first).
template <int R, typename T>
__device__ __forceinline__ void bitonic_clean(T (&v)[R]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int jr = R / 2; jr >= 1; jr >>= 1) {  // partners in the same lane
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if ((r & jr) == 0) {
        T a = v[r], b = v[r | jr];
        v[r] = pick_better(a, b);
        v[r | jr] = pick_worse(a, b);
      }
    }
  }
#pragma unroll
  for (int j = 16; j >= 1; j >>= 1) {  // partners across lanes
    const bool lower = (lane & j) == 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      T o = shfl_xor(v[r], j);
      v[r] = lower ? pick_better(v[r], o) : pick_worse(v[r], o);
    }
  }
}

// Full bitonic sort of the N = 32*R elements, best first.
template <int R, typename T>
__device__ __forceinline__ void bitonic_sort(T (&v)[R]) {
  const int lane = threadIdx.x & 31;
  // stages with k <= 32: every register row sorted independently, alternating
  // direction by row so that pairs of rows form bitonic sequences.
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j >= 1; j >>= 1) {
      const bool lower = (lane & j) == 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        // element index e = r*32 + lane; block of size k is "best-first" when
        // (e & k) == 0 (k == 32 uses the row bit)
        const int e = r * 32 + lane;
        const bool best_first = (e & k) == 0;
        T o = shfl_xor(v[r], j);
        const bool take_better = (lower == best_first);
        v[r] = take_better ? pick_better(v[r], o) : pick_worse(v[r], o);
      }
    }
  }
  // stages with k > 32: compare across rows first, then within rows
#pragma unroll
  for (int kr = 2; kr <= R; kr <<= 1) {  // k = 32*kr
#pragma unroll
    for (int jr = kr >> 1; jr >= 1; jr >>= 1) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if ((r & jr) == 0) {
          const bool best_first = ((r * 32) & (kr * 32)) == 0;
          T a = v[r], b = v[r | jr];
          if (best_first) {
            v[r] = pick_better(a, b);
            v[r | jr] = pick_worse(a, b);
          } else {
            v[r] = pick_worse(a, b);
            v[r | jr] = pick_better(a, b);
          }
        }
      }
    }
#pragma unroll
    for (int j = 16; j >= 1; j >>= 1) {
      const bool lower = (lane & j) == 0;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const bool best_first = ((r * 32) & (kr * 32)) == 0;
        T o = shfl_xor(v[r], j);
        const bool take_better = (lower == best_first);
        v[r] = take_better ? pick_better(v[r], o) : pick_worse(v[r], o);
      }
    }
  }
}

// Keep the best N of (sorted list `v`) U (sorted list `w`), result sorted in `v`.
template <int R, typename T>
__device__ __forceinline__ void merge_sorted(T (&v)[R], const T (&w)[R]) {
  const int lane = threadIdx.x & 31;
  // element e of v meets element N-1-e of w: register R-1-r of lane 31-lane
#pragma unroll
  for (int r = 0; r < R; ++r) {
    T o = shfl_idx(w[R - 1 - r], 31 - lane);
    v[r] = pick_better(v[r], o);
  }
  bitonic_clean<R>(v);
}

// Insert 32 unsorted candidates (one per lane) into the sorted list `v`.
template <int R, typename T>
__device__ __forceinline__ void insert32(T (&v)[R], T cand) {
  T c1[1] = {cand};
  bitonic_sort<1>(c1);
  const int lane = threadIdx.x & 31;
  // positions N-32..N-1 of v meet the reversed candidates
  T o = shfl_idx(c1[0], 31 - lane);
  v[R - 1] = pick_better(v[R - 1], o);
  bitonic_clean<R>(v);
}

}  // namespace prr
