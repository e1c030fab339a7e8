// prr_select.cuh -- CTA-wide ranking primitives: radix selection of the k-th largest
// 32-bit key, and bitmap-based selection and ordered emission.
//
// Ranking order everywhere: larger key first, ties broken by the lower index.  The
// top-k set is therefore {key > T} plus the lowest-index entries with key == T, where
// T is the k-th largest key (with multiplicity).  T is found MSB-first, 8 bits per
// pass, from a shared-memory histogram (one shared-memory reduction per key).  Sets
// are then held as bitmaps (one ballot per 32 entries); trimming the ties and writing
// a set in ascending index order take one warp, popcounts and a shuffle prefix sum.  These routines run once per step on the
// critical path, so they use few barriers and no CTA-wide scans.  Every thread of the
// group must call the functions that synchronise it (marked "Group"; see Grp).
#pragma once

#include <cstdint>

#include "prr_device.cuh"

namespace prr {

constexpr unsigned kFull = 0xFFFFFFFFu;

// Inclusive warp prefix sum.
__device__ __forceinline__ int warp_inclusive_sum(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Group.  k-th largest key (1 <= k <= number of members) among entries i < n with
// member(i).  Returns T; *n_gt = number of members with key > T.  `hist`: 256
// unsigned of 16-byte aligned shared scratch; `bc`: 2 ints of shared scratch.
// Leading bytes shared by every member key (one min/max reduction) need no pass, so
// scores in a narrow range usually take two or three passes.
template <typename KeyFn, typename MemberFn>
__device__ uint32_t radix_kth_largest(int n, int k, KeyFn key, MemberFn member, unsigned* hist, int* bc,
                                      int* n_gt, const Grp& grp) {
  const int tid = grp.tid, lane = tid & 31, warp = tid >> 5, NT = grp.nt, nw = NT >> 5;
  constexpr int U = 4;  // keys per thread per round: independent loads in flight
  unsigned kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int base = 0; base < n; base += U * NT) {
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const int i = base + q * NT + tid;
      if (i < n && member(i)) {
        const uint32_t v = key(i);
        kmin = min(kmin, v);
        kmax = max(kmax, v);
      }
    }
  }
  kmin = __reduce_min_sync(kFull, kmin);
  kmax = __reduce_max_sync(kFull, kmax);
  if (lane == 0) {
    hist[warp] = kmin;
    hist[32 + warp] = kmax;
  }
  gsync(grp);
  unsigned gmin = 0xFFFFFFFFu, gmax = 0u;
  for (int w = 0; w < nw; ++w) {
    gmin = min(gmin, hist[w]);
    gmax = max(gmax, hist[32 + w]);
  }
  gsync(grp);  // hist is reused below
  if (gmin == gmax) {  // all member keys equal
    *n_gt = 0;
    return gmin;
  }
  const int skip = __clz(gmin ^ gmax) / 8;  // leading bytes common to all keys
  uint32_t pmask = skip ? (0xFFFFFFFFu << (32 - 8 * skip)) : 0u;
  uint32_t prefix = gmin & pmask;
  int krem = k, above_total = 0;
#pragma unroll 1
  for (int shift = 24 - 8 * skip; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0u;
    gsync(grp);
    for (int base = 0; base < n; base += U * NT) {  // warp-uniform trip count
      unsigned dg[U];
      bool act[U];
#pragma unroll
      for (int q = 0; q < U; ++q) {
        const int i = base + q * NT + tid;
        dg[q] = 0u;
        act[q] = false;
        if (i < n && member(i)) {
          const uint32_t kv = key(i);
          act[q] = (kv & pmask) == prefix;
          dg[q] = (kv >> shift) & 0xFFu;
        }
      }
      // One shared-memory reduction per key (no return value, so the issuing warp does
      // not wait for it); aggregating equal digits first costs more than it saves.
#pragma unroll
      for (int q = 0; q < U; ++q)
        if (act[q]) red_shared_add(&hist[dg[q]], 1u);
    }
    gsync(grp);
    if (warp == 0) {
      // lane l owns bins 8l..8l+7; suffix sums run from the top bin down
      const uint4 a = reinterpret_cast<const uint4*>(hist)[2 * lane];
      const uint4 b = reinterpret_cast<const uint4*>(hist)[2 * lane + 1];
      const int c[8] = {static_cast<int>(a.x), static_cast<int>(a.y), static_cast<int>(a.z), static_cast<int>(a.w),
                        static_cast<int>(b.x), static_cast<int>(b.y), static_cast<int>(b.z), static_cast<int>(b.w)};
      int sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) sum += c[j];
      int suf = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(kFull, suf, o);
        if (lane + o < 32) suf += y;
      }
      const int higher = suf - sum;  // members in the bins of higher lanes
      if (higher < krem && suf >= krem) {
        int acc = higher;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          if (acc + c[j] >= krem) {
            bc[0] = 8 * lane + j;
            bc[1] = acc;
            break;
          }
          acc += c[j];
        }
      }
    }
    gsync(grp);
    const uint32_t dsel = static_cast<uint32_t>(bc[0]);
    const int above = bc[1];
    above_total += above;
    krem -= above;
    prefix |= dsel << shift;
    pmask |= 0xFFu << shift;
  }
  gsync(grp);  // bc / hist reusable
  *n_gt = above_total;
  return prefix;
}

// Group.  Bitmap `bm` (ceil(n/32) words) of the entries with cmp(i) > 0 plus the
// `take_equal` lowest-index entries with cmp(i) == 0 (cmp(i) < 0: not selected).
// `eq` is scratch of the same size.  On return bm is complete and visible to all.
template <typename CmpFn>
__device__ void select_bitmap(int n, int take_equal, CmpFn cmp, unsigned* bm, unsigned* eq, const Grp& grp) {
  const int lane = grp.tid & 31, warp = grp.tid >> 5, nw = grp.nt >> 5;
  const int W = (n + 31) / 32;
  constexpr int U = 4;  // words per warp per round: independent comparisons in flight
  for (int w0 = warp; w0 < W; w0 += U * nw) {
    int c[U];
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const int i = (w0 + q * nw) * 32 + lane;
      c[q] = i < n ? cmp(i) : -1;
    }
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const int wd = w0 + q * nw;
      const unsigned gt = __ballot_sync(kFull, c[q] > 0);
      const unsigned e = __ballot_sync(kFull, c[q] == 0);
      if (lane == 0 && wd < W) {
        bm[wd] = gt;
        eq[wd] = e;
      }
    }
  }
  gsync(grp);
  if (warp == 0 && take_equal > 0) {  // the first take_equal tie bits, in index order
    int base = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
      const int wd = w0 + lane;
      unsigned e = wd < W ? eq[wd] : 0u;
      const int c = __popc(e);
      const int inc = warp_inclusive_sum(c);
      const int exc = base + inc - c;
      if (e && exc < take_equal) {
        const int need = take_equal - exc;
        unsigned keepm = e;
        if (need < c) {
          keepm = 0u;
          for (int r = 0; r < need; ++r) {
            const unsigned low = e & (0u - e);
            keepm |= low;
            e ^= low;
          }
        }
        bm[wd] |= keepm;
      }
      base += __shfl_sync(kFull, inc, 31);
      if (base >= take_equal) break;
    }
  }
  gsync(grp);
}

// One warp.  Write the set bits of bm[0..W) (optionally masked by ~exclude) as
// ascending indices to out[0..), then -1 up to `cap`; on_emit(pos, index) is called
// for every index written.  Returns the count.
template <typename EmitFn>
__device__ __forceinline__ int warp_emit_bitmap(const unsigned* bm, const unsigned* exclude, int W, int* out, int cap,
                                                EmitFn on_emit) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int wd = w0 + lane;
    unsigned b = wd < W ? (exclude ? (bm[wd] & ~exclude[wd]) : bm[wd]) : 0u;
    const int c = __popc(b);
    const int inc = warp_inclusive_sum(c);
    int pos = base + inc - c;
    while (b) {
      const int bit = __ffs(b) - 1;
      if (pos < cap) {
        out[pos] = wd * 32 + bit;
        on_emit(pos, wd * 32 + bit);
      }
      ++pos;
      b &= b - 1u;
    }
    base += __shfl_sync(kFull, inc, 31);
  }
  for (int e = base + lane; e < cap; e += 32) out[e] = -1;
  return base;
}

__device__ __forceinline__ int warp_emit_bitmap(const unsigned* bm, const unsigned* exclude, int W, int* out,
                                                int cap) {
  return warp_emit_bitmap(bm, exclude, W, out, cap, [](int, int) {});
}

}  // namespace prr
