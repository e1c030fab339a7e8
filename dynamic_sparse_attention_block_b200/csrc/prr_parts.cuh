// prr_parts.cuh -- CTA-level pieces of the decode step shared by the standalone
// kernels and the fused single-launch step: block scoring, the selection finisher,
// the EMA predictor of one unit and the LSE merge of one query head.
//
// Data written by other CTAs of the same launch is read through L2 (ld.global.cg).
#pragma once

#include "prr_kernels.cuh"
#include "prr_select.cuh"

namespace prr {

#ifdef PRR_PHASE_DEBUG
// Debug builds only: per-unit phase timestamps of the finisher / predictor.
__device__ unsigned long long g_phase[2][4096][8];
#define PRR_PHASE(kind, u, k) \
  do {                        \
    if (threadIdx.x == 0 && (u) < 4096) g_phase[kind][u][k] = global_ns(); \
  } while (0)
#else
#define PRR_PHASE(kind, u, k) \
  do {                        \
  } while (0)
#endif

// ------------------------------------------------------------------ block scoring
//
// Quest's channel-wise bound summed over the GQA group (one selection per KV head):
//   s_b = sum_h sum_c max(q_hc*min_bc, q_hc*max_bc)
//       = sum_c (sum_h max(q_hc,0)) * max_bc + (sum_h min(q_hc,0)) * min_bc
// One block costs 2d fused multiply-adds against its 2d summary values.  On the dyadic
// {-8..8}/8 grid every product is a multiple of 1/64 and every partial sum stays below
// 2^24 units of 1/64, so the fp32 score is exact in any order.

// Coefficients of the [min | max] summary row, element e in chunk e/8: positions 0-3
// in lo[chunk], 4-7 in hi[chunk].  All threads call; synchronise before use.
template <int D>
__device__ __forceinline__ void load_group_coef(const Params& p, int u, float4* lo4, float4* hi4) {
  float* lo = reinterpret_cast<float*>(lo4);
  float* hi = reinterpret_cast<float*>(hi4);
  const uint16_t* qg = p.q + static_cast<size_t>(u) * p.G * D;
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float neg = 0.f, pos = 0.f;
    for (int h = 0; h < p.G; ++h) {
      const float x = __uint_as_float(static_cast<uint32_t>(qg[h * D + c]) << 16);
      neg += fminf(x, 0.f);
      pos += fmaxf(x, 0.f);
    }
    const int e0 = c, e1 = D + c;  // min part, max part
    ((e0 & 7) < 4 ? lo[(e0 >> 3) * 4 + (e0 & 3)] : hi[(e0 >> 3) * 4 + (e0 & 3)]) = neg;
    ((e1 & 7) < 4 ? lo[(e1 >> 3) * 4 + (e1 & 3)] : hi[(e1 >> 3) * 4 + (e1 & 3)]) = pos;
  }
}

// Bound of one block from its summary row in shared memory.  Lanes start at rotated
// chunks, so 32 lanes reading 32 consecutive rows hit distinct banks.
template <int D>
__device__ __forceinline__ float score_summary_row(const unsigned char* row, const float4* lo4,
                                                   const float4* hi4, int lane) {
  constexpr int C = 4 * D / 16;  // 16-byte chunks per row
  float acc = 0.f;
#pragma unroll 8
  for (int i = 0; i < C; ++i) {
    const int cc = (i + lane) & (C - 1);
    const uint4 w = *reinterpret_cast<const uint4*>(row + cc * 16);
    const float4 a = lo4[cc], z = hi4[cc];
    acc = fmaf(a.x, bf16_lo(w.x), acc);
    acc = fmaf(a.y, bf16_hi(w.x), acc);
    acc = fmaf(a.z, bf16_lo(w.y), acc);
    acc = fmaf(a.w, bf16_hi(w.y), acc);
    acc = fmaf(z.x, bf16_lo(w.z), acc);
    acc = fmaf(z.y, bf16_hi(w.z), acc);
    acc = fmaf(z.z, bf16_lo(w.w), acc);
    acc = fmaf(z.w, bf16_hi(w.w), acc);
  }
  return acc;
}

// Fold the appended token's key row (newk, d bf16 in shared memory) into the summary
// row of its block (in shared memory) and write the row back to global memory.  A
// block that starts with this token takes min = max = k.  One warp calls it.
template <int D>
__device__ __forceinline__ void fold_tail_row(uint32_t* row, const uint16_t* newk, bool fresh, uint32_t* grow,
                                              int lane) {
  for (int e = lane; e < D; e += 32) {  // bf16 pairs of [min | max]
    const int part = e / (D / 2);       // 0: min row, 1: max row
    const int ch2 = e % (D / 2);        // channel pair
    const __nv_bfloat162 kv = reinterpret_cast<const __nv_bfloat162*>(newk)[ch2];
    const uint32_t old = row[e];
    const __nv_bfloat162 cur = *reinterpret_cast<const __nv_bfloat162*>(&old);
    const __nv_bfloat162 nw = fresh ? kv : (part == 0 ? __hmin2(cur, kv) : __hmax2(cur, kv));
    const uint32_t bits = *reinterpret_cast<const uint32_t*>(&nw);
    row[e] = bits;
    grow[e] = bits;
  }
  __syncwarp();
}

// ------------------------------------------------------------------ selection finisher
//
// True selected set (PRR abstract): the K best blocks under (score desc, index asc),
// written in ascending block order.  missed = S \ Pred ascending, keep[j] = [Pred_j in S]
// (PRR method summary, contributions (2)-(3)).  A predicted slot is active iff
// 0 <= Pred_j < nb.  Keys come from p.keys (written by this or other CTAs); the keys
// and the predicted list are fetched together (one round trip).

struct FinishOut {
  int p_active;  // active predicted slots
  int n_missed;
};

__host__ __device__ constexpr size_t finish_scratch_bytes(int maxnb) {
  return static_cast<size_t>(maxnb) * 4 + 4 * static_cast<size_t>((maxnb + 31) / 32) * 4 + 256 * 4 + 128 * 4 +
         16 * 4;
}

__device__ inline FinishOut select_finish(const Params& p, int u, int nb, unsigned char* scratch) {
  const int tid = threadIdx.x, warp = tid >> 5;
  const int W = (p.maxnb + 31) / 32;
  uint32_t* skeys = reinterpret_cast<uint32_t*>(scratch);
  unsigned* bm_pred = reinterpret_cast<unsigned*>(skeys + p.maxnb);
  unsigned* bm_sel = bm_pred + W;
  unsigned* bm_eq = bm_sel + W;
  unsigned* hist = bm_eq + W;
  int* spred = reinterpret_cast<int*>(hist + 256);  // [128]
  int* misc = spred + 128;                          // bc[2], counts

  PRR_PHASE(0, u, 0);
  const uint32_t* keys_in = p.keys + static_cast<size_t>(u) * p.maxnb;
  for (int i = tid; i < nb; i += blockDim.x) skeys[i] = __ldcg(keys_in + i);
  for (int j = tid; j < p.P; j += blockDim.x) spred[j] = p.pred[static_cast<size_t>(u) * p.P + j];
  for (int i = tid; i < W; i += blockDim.x) bm_pred[i] = 0u;
  __syncthreads();
  PRR_PHASE(0, u, 1);
  int active_local = 0;
  for (int j = tid; j < p.P; j += blockDim.x) {
    const int pv = spred[j];
    if (pv >= 0 && pv < nb) {
      ++active_local;
      atomicOr(&bm_pred[pv >> 5], 1u << (pv & 31));
      if (j > 0 && spred[j - 1] >= pv) report(p.status, kDevBadPred);
    } else if (pv != -1) {
      report(p.status, kDevBadPred);
    }
  }
  const int keff = min(p.K, nb);
  uint32_t T = 0u;
  int n_gt = 0;
  const bool take_all = keff >= nb;
  if (keff > 0 && !take_all)
    T = radix_kth_largest(
        nb, keff, [&](int i) { return skeys[i]; }, [&](int) { return true; }, hist, misc, &n_gt);
  PRR_PHASE(0, u, 2);
  select_bitmap(
      nb, take_all ? 0 : keff - n_gt,
      [&](int i) {
        if (take_all) return 1;
        const uint32_t kv = skeys[i];
        return kv > T ? 1 : (kv == T ? 0 : -1);
      },
      bm_sel, bm_eq);
  PRR_PHASE(0, u, 3);
  // three warps in parallel: selected list, missed list, keep mask
  int nm = 0;
  const int Wn = (nb + 31) / 32;
  if (warp == 0) {
    warp_emit_bitmap(bm_sel, nullptr, Wn, p.sel + static_cast<size_t>(u) * p.K, p.K);
  } else if (warp == 1) {
    nm = warp_emit_bitmap(bm_sel, bm_pred, Wn, p.missed + static_cast<size_t>(u) * p.K, p.K);
    if ((tid & 31) == 0) {
      p.n_missed[u] = nm;
      misc[2] = nm;
    }
  }
  for (int j = tid; j < p.P; j += blockDim.x) {
    const int pv = spred[j];
    p.keep[static_cast<size_t>(u) * p.P + j] =
        (pv >= 0 && pv < nb && ((bm_sel[pv >> 5] >> (pv & 31)) & 1u)) ? 1 : 0;
  }
  // active predicted slots (CTA sum of the per-thread counts)
  if (tid == 0) misc[3] = 0;
  __syncthreads();
  if (active_local) atomicAdd(&misc[3], active_local);
  __syncthreads();
  PRR_PHASE(0, u, 4);
  PRR_PHASE(0, u, 5);
  return FinishOut{misc[3], misc[2]};
}

// ------------------------------------------------------------------ EMA predictor
//
// PRR abstract and method summary: an exponential moving average of past selections
// forecasts the next step's blocks.  Reading taken (the pages print no formula):
//   e_b <- alpha*e_b + beta*[b in S_t],  beta = 1 - alpha,  e starts at 0,
// in fp64 with separately rounded multiplies and add (no fused multiply-add), so the
// state and the predicted set are bit-exact against the fp64 CPU oracle.
// Pred_{t+1} = the min(P, nb) best blocks under (e desc, index asc), ascending, -1
// beyond.  e >= 0, so its IEEE bit pattern orders like its value: the P-th largest
// pattern is found by radix selection on the high word, then (unless the tied entries
// agree on the low word) on the low word among entries tied on the high word; exact
// ties go to the lowest block indices.

__host__ __device__ constexpr size_t ema_scratch_bytes(int maxnb) {
  return static_cast<size_t>(maxnb) * 8 + 3 * static_cast<size_t>((maxnb + 31) / 32) * 4 + 256 * 4 + 16 * 4;
}

__device__ inline void ema_unit(const Params& p, int u, unsigned char* scratch) {
  const int W = (p.maxnb + 31) / 32;
  uint32_t* hi = reinterpret_cast<uint32_t*>(scratch);
  uint32_t* lo = hi + p.maxnb;
  unsigned* bm = lo + p.maxnb;  // selected blocks of this step
  unsigned* bsel = bm + W;      // predicted set
  unsigned* beq = bsel + W;
  unsigned* hist = beq + W;
  int* misc = reinterpret_cast<int*>(hist + 256);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  PRR_PHASE(1, u, 0);
  const int n = checked_len(p, u / p.Hkv);
  const int nb = (n + p.bs - 1) / p.bs;
  double* e = p.ema + static_cast<size_t>(u) * p.maxnb;
  const bool update = p.sel != nullptr;

  // fetch the state and S_t together
  for (int i = tid; i < nb; i += blockDim.x) {
    const unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(e[i]));
    hi[i] = static_cast<uint32_t>(bits >> 32);
    lo[i] = static_cast<uint32_t>(bits);
  }
  int sv = -1;
  if (update && tid < p.K) sv = __ldcg(p.sel + static_cast<size_t>(u) * p.K + tid);
  for (int i = tid; i < W; i += blockDim.x) bm[i] = 0u;
  __syncthreads();
  if (update) {
    for (int i = tid; i < p.K; i += blockDim.x) {
      const int v = i == tid ? sv : __ldcg(p.sel + static_cast<size_t>(u) * p.K + i);
      if (v >= 0 && v < nb) atomicOr(&bm[v >> 5], 1u << (v & 31));
    }
    __syncthreads();
    const double alpha = p.alpha;
    const double beta = __dsub_rn(1.0, alpha);
    for (int i = tid; i < nb; i += blockDim.x) {
      const double x0 = __longlong_as_double(static_cast<long long>((static_cast<unsigned long long>(hi[i]) << 32) | lo[i]));
      const double ind = ((bm[i >> 5] >> (i & 31)) & 1u) ? 1.0 : 0.0;
      const double x = __dadd_rn(__dmul_rn(alpha, x0), __dmul_rn(beta, ind));
      e[i] = x;
      const unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(x));
      hi[i] = static_cast<uint32_t>(bits >> 32);
      lo[i] = static_cast<uint32_t>(bits);
    }
    __syncthreads();
  }
  PRR_PHASE(1, u, 1);

  const int peff = min(p.P, nb);
  int* out = p.pred_next + static_cast<size_t>(u) * p.P;
  if (peff <= 0) {
    for (int j = tid; j < p.P; j += blockDim.x) out[j] = -1;
    return;
  }
  if (peff >= nb) {
    select_bitmap(nb, 0, [&](int) { return 1; }, bsel, beq);
  } else {
    int gt_hi = 0, gt_lo = 0;
    const uint32_t Thi = radix_kth_largest(
        nb, peff, [&](int i) { return hi[i]; }, [&](int) { return true; }, hist, misc, &gt_hi);
    PRR_PHASE(1, u, 2);
    const int need = peff - gt_hi;  // taken from the entries tied on the high word
    // do the tied entries agree on the low word?  (then the low-word pass is moot)
    unsigned mn = 0xFFFFFFFFu, mx = 0u;
    for (int i = tid; i < nb; i += blockDim.x)
      if (hi[i] == Thi) {
        mn = min(mn, lo[i]);
        mx = max(mx, lo[i]);
      }
    mn = __reduce_min_sync(kFull, mn);
    mx = __reduce_max_sync(kFull, mx);
    if (lane == 0) {
      misc[4 + warp] = static_cast<int>(mn);
      misc[8 + warp] = static_cast<int>(mx);
    }
    __syncthreads();
    unsigned gmin = 0xFFFFFFFFu, gmax = 0u;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
      gmin = min(gmin, static_cast<unsigned>(misc[4 + w]));
      gmax = max(gmax, static_cast<unsigned>(misc[8 + w]));
    }
    uint32_t Tlo = gmin;
    if (gmin != gmax)
      Tlo = radix_kth_largest(
          nb, need, [&](int i) { return lo[i]; }, [&](int i) { return hi[i] == Thi; }, hist, misc, &gt_lo);
    PRR_PHASE(1, u, 3);
    select_bitmap(
        nb, need - gt_lo,
        [&](int i) {
          const uint32_t h = hi[i];
          if (h != Thi) return h > Thi ? 1 : -1;
          const uint32_t l = lo[i];
          return l > Tlo ? 1 : (l == Tlo ? 0 : -1);
        },
        bsel, beq);
  }
  if (warp == 0) warp_emit_bitmap(bsel, nullptr, (nb + 31) / 32, out, p.P);
  __syncthreads();
  PRR_PHASE(1, u, 4);
}

// ------------------------------------------------------------------ LSE merge
//
// PRR method summary and contribution (3): the missed blocks are attended once the
// true set is known and combined with the reusable speculative state through
// online-softmax statistics, with no recomputation.  With base-2 logits:
//   m* = max_j m_j,  l* = sum_j l_j 2^(m_j - m*),  out = sum_j O_j 2^(m_j - m*) / l*,
//   lse = (m* + log2 l*) ln 2,
// over the slots j with keep[j] = 1 (speculation) and the first n_missed repair slots.
// 128 threads: the weighted numerator sum is split over the 4 warps, each lane one
// float4 column with 16 slot loads in flight.

__host__ __device__ constexpr size_t combine_scratch_bytes(int P, int K, int D) {
  return static_cast<size_t>(P + K) * 16 + 16 * 4 + 4 * static_cast<size_t>(D) * 4 + 32;
}

template <int D>
__device__ void combine_head(const Params& p, int u, int h, unsigned char* scratch) {
  constexpr int C4 = D / 4;
  const int P = p.P, K = p.K, S = P + K;
  int* slots = reinterpret_cast<int*>(scratch);   // compacted active slots
  float* wt = reinterpret_cast<float*>(slots + S);  // per slot: m, then weight
  float* lv = wt + S;                               // per slot: l
  int* actf = reinterpret_cast<int*>(lv + S);       // per slot: contributes?
  float* red = reinterpret_cast<float*>(actf + S);  // 8 floats + count
  int* count = reinterpret_cast<int*>(red + 8);
  float4* part = reinterpret_cast<float4*>((reinterpret_cast<uintptr_t>(red + 16) + 15) &
                                           ~static_cast<uintptr_t>(15));  // [4][C4]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t row = static_cast<size_t>(u) * p.G + h;

  // round trip 1: every slot's flag and statistics at once
  const int nm = min(max(__ldcg(p.n_missed + u), 0), K);
  float mloc = -INFINITY;
  for (int s = tid; s < S; s += blockDim.x) {
    bool act;
    float m, l;
    if (s < P) {
      act = __ldcg(p.keep + static_cast<size_t>(u) * P + s) != 0;
      m = __ldcg(p.pm + row * P + s);
      l = __ldcg(p.pl + row * P + s);
    } else {
      act = (s - P) < nm;
      m = act ? __ldcg(p.rm + row * K + (s - P)) : 0.f;
      l = act ? __ldcg(p.rl + row * K + (s - P)) : 0.f;
    }
    wt[s] = act ? m : -INFINITY;
    lv[s] = act ? l : 0.f;
    actf[s] = act ? 1 : 0;
    if (act) mloc = fmaxf(mloc, m);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xFFFFFFFFu, mloc, o));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  const float mstar = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float lsum = 0.f;
  for (int s = tid; s < S; s += blockDim.x) {
    const float w = (wt[s] == -INFINITY || mstar == -INFINITY) ? 0.f : exp2f(wt[s] - mstar);
    wt[s] = w;
    lsum += lv[s] * w;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xFFFFFFFFu, lsum, o);
  if (lane == 0) red[4 + warp] = lsum;
  if (warp == 0) {  // compact the contributing slots
    int cnt = 0;
    for (int base = 0; base < S; base += 32) {
      const int s = base + lane;
      const bool a = s < S && actf[s] != 0;
      const unsigned mask = __ballot_sync(0xFFFFFFFFu, a);
      if (a) slots[cnt + __popc(mask & ((1u << lane) - 1u))] = s;
      cnt += __popc(mask);
    }
    if (lane == 0) count[0] = cnt;
  }
  __syncthreads();
  const float lstar = red[4] + red[5] + red[6] + red[7];
  const int ns = count[0];

  // round trip 2: the numerators of the contributing slots, 16 loads in flight per lane
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int BATCH = 16;
  for (int s0 = warp; s0 < ns; s0 += 4 * BATCH) {
    float4 v[BATCH];
    float w[BATCH];
#pragma unroll
    for (int q = 0; q < BATCH; ++q) {
      const int si = s0 + 4 * q;
      v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      w[q] = 0.f;
      if (si < ns && lane < C4) {
        const int j = slots[si];
        const float4* src = j < P ? reinterpret_cast<const float4*>(p.pO + (row * P + j) * D)
                                  : reinterpret_cast<const float4*>(p.rO + (row * K + (j - P)) * D);
        v[q] = __ldcg(src + lane);
        w[q] = wt[j];
      }
    }
#pragma unroll
    for (int q = 0; q < BATCH; ++q) {
      acc.x = fmaf(w[q], v[q].x, acc.x);
      acc.y = fmaf(w[q], v[q].y, acc.y);
      acc.z = fmaf(w[q], v[q].z, acc.z);
      acc.w = fmaf(w[q], v[q].w, acc.w);
    }
  }
  if (lane < C4) part[warp * C4 + lane] = acc;
  __syncthreads();
  if (tid < C4) {
    float4 o = part[tid];
#pragma unroll
    for (int w2 = 1; w2 < 4; ++w2) {
      o.x += part[w2 * C4 + tid].x;
      o.y += part[w2 * C4 + tid].y;
      o.z += part[w2 * C4 + tid].z;
      o.w += part[w2 * C4 + tid].w;
    }
    const float inv = lstar > 0.f ? 1.0f / lstar : 0.f;
    o.x *= inv;
    o.y *= inv;
    o.z *= inv;
    o.w *= inv;
    reinterpret_cast<float4*>(p.out + row * D)[tid] = o;
  }
  if (tid == 0) p.lse[row] = lstar > 0.f ? (mstar + log2f(lstar)) * 0.69314718055994530942f : -INFINITY;
  __syncthreads();
}

}  // namespace prr
