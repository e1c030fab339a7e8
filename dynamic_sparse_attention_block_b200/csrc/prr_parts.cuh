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
    if ((threadIdx.x & 127) == 0 && (u) < 4096) g_phase[kind][u][k] = global_ns(); \
  } while (0)
#else
#define PRR_PHASE(kind, u, k) \
  do {                        \
  } while (0)
#endif

// ------------------------------------------------------------------ batched loads
//
// Copy n 32-bit words (global, written by other CTAs: read through L2) into shared
// memory with kBatch loads in flight per thread before any is consumed; a plain loop
// would wait one memory round trip per element.
constexpr int kBatch = 16;

__device__ __forceinline__ void load_words_cg(uint32_t* dst, const uint32_t* src, int n, const Grp& g) {
  for (int base = 0; base < n; base += kBatch * g.nt) {
    uint32_t v[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int i = base + q * g.nt + g.tid;
      v[q] = i < n ? __ldcg(src + i) : 0u;
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int i = base + q * g.nt + g.tid;
      if (i < n) dst[i] = v[q];
    }
  }
}

// ------------------------------------------------------------------ block scoring
//
// Quest's channel-wise bound summed over the GQA group (one selection per KV head):
//   s_b = sum_h sum_c max(q_hc*min_bc, q_hc*max_bc)
//       = sum_c (sum_h max(q_hc,0)) * max_bc + (sum_h min(q_hc,0)) * min_bc
// One block costs 2d fused multiply-adds against its 2d summary values.  On the dyadic
// {-8..8}/8 grid every product is a multiple of 1/64 and every partial sum stays below
// 2^24 units of 1/64, so the fp32 score is exact in any order.

// Coefficients of the [min | max] summary row, element e in chunk e/8: positions 0-3
// in lo[chunk], 4-7 in hi[chunk], from the G query rows qg ([G][D] bf16, global or
// shared).  The group's threads call; synchronise before use.
template <int D>
__device__ __forceinline__ void load_group_coef(const Params& p, const uint16_t* qg, float4* lo4, float4* hi4,
                                                const Grp& g) {
  float* lo = reinterpret_cast<float*>(lo4);
  float* hi = reinterpret_cast<float*>(hi4);
  for (int c = g.tid; c < D; c += g.nt) {
    uint16_t qv[8];  // G <= 8: every head's load in flight before the first is used
#pragma unroll
    for (int h = 0; h < 8; ++h) qv[h] = h < p.G ? qg[h * D + c] : static_cast<uint16_t>(0);
    float neg = 0.f, pos = 0.f;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < p.G) {
        const float x = __uint_as_float(static_cast<uint32_t>(qv[h]) << 16);
        neg += fminf(x, 0.f);
        pos += fmaxf(x, 0.f);
      }
    }
    const int e0 = c, e1 = D + c;  // min part, max part
    ((e0 & 7) < 4 ? lo[(e0 >> 3) * 4 + (e0 & 3)] : hi[(e0 >> 3) * 4 + (e0 & 3)]) = neg;
    ((e1 & 7) < 4 ? lo[(e1 >> 3) * 4 + (e1 & 3)] : hi[(e1 >> 3) * 4 + (e1 & 3)]) = pos;
  }
}

// Bound of one block from its summary row in shared memory.  Lanes start at rotated
// chunks, so 32 lanes reading 32 consecutive rows hit distinct banks.  Four
// independent accumulators (one per pair of products of a chunk) keep four fused
// multiply-add chains in flight instead of one; exact on the dyadic grid in any order.
template <int D>
__device__ __forceinline__ float score_summary_row(const unsigned char* row, const float4* lo4,
                                                   const float4* hi4, int lane) {
  constexpr int C = 4 * D / 16;  // 16-byte chunks per row
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
  for (int i = 0; i < C; ++i) {
    const int cc = (i + lane) & (C - 1);
    const uint4 w = *reinterpret_cast<const uint4*>(row + cc * 16);
    const float4 a = lo4[cc], z = hi4[cc];
    a0 = fmaf(a.x, bf16_lo(w.x), a0);
    a1 = fmaf(a.z, bf16_lo(w.y), a1);
    a2 = fmaf(z.x, bf16_lo(w.z), a2);
    a3 = fmaf(z.z, bf16_lo(w.w), a3);
    a0 = fmaf(a.y, bf16_hi(w.x), a0);
    a1 = fmaf(a.w, bf16_hi(w.y), a1);
    a2 = fmaf(z.y, bf16_hi(w.z), a2);
    a3 = fmaf(z.w, bf16_hi(w.w), a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// Selector variant (group max): the block score is the LARGEST of the group's per-head
// bounds, max_h sum_c max(q_hc*min_bc, q_hc*max_bc).  Per head the bound is again one
// dot product, with coefficients min(q_hc, 0) against the min row and max(q_hc, 0)
// against the max row; coef holds G such sets, set h at coef + 2*C*h (lo parts) and
// coef + 2*C*h + C (hi parts), C = 4D/16 chunks, laid out as in load_group_coef.
template <int D>
__device__ __forceinline__ void load_head_coef(const Params& p, const uint16_t* qg, float4* coef, const Grp& g) {
  constexpr int C = 4 * D / 16;
  for (int i = g.tid; i < p.G * D; i += g.nt) {
    const int h = i / D, c = i % D;
    const float x = __uint_as_float(static_cast<uint32_t>(qg[h * D + c]) << 16);
    float* lo = reinterpret_cast<float*>(coef + 2 * C * h);
    float* hi = reinterpret_cast<float*>(coef + 2 * C * h + C);
    const int e0 = c, e1 = D + c;  // min part, max part
    ((e0 & 7) < 4 ? lo[(e0 >> 3) * 4 + (e0 & 3)] : hi[(e0 >> 3) * 4 + (e0 & 3)]) = fminf(x, 0.f);
    ((e1 & 7) < 4 ? lo[(e1 >> 3) * 4 + (e1 & 3)] : hi[(e1 >> 3) * 4 + (e1 & 3)]) = fmaxf(x, 0.f);
  }
}

// Largest per-head bound of one block (row in shared memory); every head's products of
// a 16-byte chunk reuse the chunk's unpacked values.  Exact on the dyadic grid.
template <int D>
__device__ __forceinline__ float score_summary_row_max(const unsigned char* row, const float4* coef, int G,
                                                       int lane) {
  constexpr int C = 4 * D / 16;
  float acc[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) acc[h] = 0.f;
#pragma unroll 2
  for (int i = 0; i < C; ++i) {
    const int cc = (i + lane) & (C - 1);
    const uint4 w = *reinterpret_cast<const uint4*>(row + cc * 16);
    const float x0 = bf16_lo(w.x), x1 = bf16_hi(w.x), x2 = bf16_lo(w.y), x3 = bf16_hi(w.y);
    const float x4 = bf16_lo(w.z), x5 = bf16_hi(w.z), x6 = bf16_lo(w.w), x7 = bf16_hi(w.w);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < G) {
        const float4 a = coef[2 * C * h + cc], z = coef[2 * C * h + C + cc];
        float s = acc[h];
        s = fmaf(a.x, x0, s);
        s = fmaf(a.y, x1, s);
        s = fmaf(a.z, x2, s);
        s = fmaf(a.w, x3, s);
        s = fmaf(z.x, x4, s);
        s = fmaf(z.y, x5, s);
        s = fmaf(z.z, x6, s);
        s = fmaf(z.w, x7, s);
        acc[h] = s;
      }
    }
  }
  float m = acc[0];
#pragma unroll
  for (int h = 1; h < 8; ++h)
    if (h < G) m = fmaxf(m, acc[h]);
  return m;
}

// Bytes of the scoring coefficients: one set for the group sum, G sets for the max.
__host__ __device__ constexpr size_t coef_bytes(int D, int sets) { return static_cast<size_t>(sets) * 2 * (4 * D / 16) * 16; }

// Selector variant (representative keys, InfLLM-style): block b is represented by
// n_rep of its own tokens, offsets rep[(kvu*maxnb + b)*n_rep + j] inside the block (an
// offset at or past the valid tokens of a ragged tail stands for the last valid one),
// and scores sum_h sum_j q_h . k_rep_j = sum_j qsum . k_rep_j, qsum = sum_h q_h.  The
// coefficient area then holds qsum (D floats).  On the dyadic grid every product is a
// multiple of 1/64 and every partial sum stays below 2^24 units, so the fp32 score is
// exact in any order.  The key rows are read through L2: the step may have written the
// appended row in this launch.
template <int D>
__device__ __forceinline__ void load_qsum(const Params& p, const uint16_t* qg, float* qs, const Grp& g) {
  for (int c = g.tid; c < D; c += g.nt) {
    float acc = 0.f;
    for (int h = 0; h < p.G; ++h) acc += __uint_as_float(static_cast<uint32_t>(qg[h * D + c]) << 16);
    qs[c] = acc;
  }
}

template <int D>
__device__ __forceinline__ float score_rep_block(const Params& p, int kvu, int b, int n, const float* qs) {
  const int valid = min(p.bs, n - b * p.bs);
  const uint8_t* offs = p.rep + (static_cast<size_t>(kvu) * p.maxnb + b) * p.n_rep;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int j = 0; j < p.n_rep; ++j) {
    const int off = min(static_cast<int>(offs[j]), valid - 1);
    const long long row = kv_row(p, kvu, b * p.bs + off);
    if (row < 0) continue;  // a bad block-table entry (reported by kv_row)
    const uint4* kr = reinterpret_cast<const uint4*>(p.kc + static_cast<size_t>(row) * D);
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint4 w = __ldcg(kr + c8);
      const float* q8 = qs + 8 * c8;
      a0 = fmaf(q8[0], bf16_lo(w.x), a0);
      a1 = fmaf(q8[2], bf16_lo(w.y), a1);
      a2 = fmaf(q8[4], bf16_lo(w.z), a2);
      a3 = fmaf(q8[6], bf16_lo(w.w), a3);
      a0 = fmaf(q8[1], bf16_hi(w.x), a0);
      a1 = fmaf(q8[3], bf16_hi(w.y), a1);
      a2 = fmaf(q8[5], bf16_hi(w.z), a2);
      a3 = fmaf(q8[7], bf16_hi(w.w), a3);
    }
  }
  return (a0 + a1) + (a2 + a3);
}

// Every variant: coefficients for unit u's query rows qg (group-synchronise before use).
template <int D>
__device__ __forceinline__ void load_coef(const Params& p, const uint16_t* qg, float4* coef, const Grp& g) {
  if (p.rep) {
    load_qsum<D>(p, qg, reinterpret_cast<float*>(coef), g);
  } else if (p.sel_max) {
    load_head_coef<D>(p, qg, coef, g);
  } else {
    load_group_coef<D>(p, qg, coef, coef + (4 * D / 16), g);
  }
}

template <int D>
__device__ __forceinline__ float score_row(const Params& p, const unsigned char* row, const float4* coef, int lane) {
  if (p.sel_max) return score_summary_row_max<D>(row, coef, p.G, lane);
  return score_summary_row<D>(row, coef, coef + (4 * D / 16), lane);
}

// The score of block b of KV slice kvu (n tokens): its summary row, or its
// representative keys under the representative-key selector.
template <int D>
__device__ __forceinline__ float score_block(const Params& p, const unsigned char* row, const float4* coef, int lane,
                                             int kvu, int b, int n) {
  if (p.rep) return score_rep_block<D>(p, kvu, b, n, reinterpret_cast<const float*>(coef));
  return score_row<D>(p, row, coef, lane);
}

// Ranking key of block b (of nb) with score s: forced sink blocks rank above
// everything, then forced local blocks, newest first, then every other block by its
// score (orderable keys of finite scores stay below 0xFF800001).  Top-K over these keys
// takes the sinks first, then the newest local blocks, then the best of the rest.
__device__ __forceinline__ uint32_t block_key(const Params& p, int b, int nb, float s) {
  if (b < p.n_sink) return 0xFFFFFFFFu;
  if (b >= nb - p.n_local) return 0xFFFFFFFEu - static_cast<uint32_t>(nb - 1 - b);
  return orderable(s);
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
// 0 <= Pred_j < nb.
//
// S = {key > T} plus the lowest-index blocks with key == T, T the K_eff-th largest key.
// Group summaries: each scoring warp writes, for its group of 32 blocks, the group's
// largest key and the mask of the blocks holding it.  From those alone the finisher
// sees whether at least K_eff blocks tie at the overall maximum; then T is that maximum
// and S is the first K_eff set bits of the maximal groups' masks -- no key is loaded
// (this is the usual case when every block's bound saturates).  Otherwise T comes from
// a radix selection over the keys by the whole group (radix_kth_largest).

constexpr int kEagerKeys = 4096;  // up to this many keys are fetched with the group summaries

// One warp (all lanes): summary of the warp's group of 32 blocks (`valid` lanes).
__device__ __forceinline__ void write_group_summary(const Params& p, int u, int group, uint32_t key, bool valid) {
  if (!p.gsum) return;
  const uint32_t mx = __reduce_max_sync(kFull, valid ? key : 0u);
  const unsigned mask = __ballot_sync(kFull, valid && key == mx);
  if ((threadIdx.x & 31) == 0) p.gsum[static_cast<size_t>(u) * ((p.maxnb + 31) / 32) + group] = make_uint2(mx, mask);
}

struct FinishOut {
  int p_active;  // active predicted slots
  int n_missed;
  int path;      // kStatTakeAll, kStatTieMasks or kStatKeySearch
};

__host__ __device__ constexpr size_t finish_scratch_bytes(int maxnb) {
  return 256 * 4 + 128 * 4 + 16 * 4 + static_cast<size_t>((maxnb + 31) / 32) * 8 + static_cast<size_t>(maxnb) * 4 +
         3 * static_cast<size_t>((maxnb + 31) / 32) * 4;
}

// Optional outputs for the fused step: keepf [P], per predicted slot, 1 | keep << 1;
// rdesc [K], per missed slot, block + 1 (kNoRepair past the last missed block).
constexpr unsigned kNoRepair = 0xFFFFFFFFu;

__device__ inline FinishOut select_finish(const Params& p, int u, int nb, unsigned char* scratch, const Grp& grp,
                                          unsigned* keepf = nullptr, unsigned* rdesc = nullptr) {
  const int tid = grp.tid, warp = tid >> 5, lane = tid & 31, NT = grp.nt;
  const int W = (p.maxnb + 31) / 32;
  int* spred = reinterpret_cast<int*>(scratch + 256 * 4);  // [128]
  int* misc = spred + 128;                                 // counts, T, n_gt
  uint2* gs = reinterpret_cast<uint2*>(misc + 16);         // [W] group summaries
  uint32_t* skeys = reinterpret_cast<uint32_t*>(gs + W);
  unsigned* bm_pred = skeys + p.maxnb;
  unsigned* bm_sel = bm_pred + W;
  unsigned* bm_eq = bm_sel + W;
  const int Wn = (nb + 31) / 32;

  PRR_PHASE(0, u, 0);
  const int keff = min(p.K, nb);
  const bool take_all = keff >= nb;
  const bool use_gs = p.gsum != nullptr && !take_all && keff > 0;
  bool have_keys = false;
  for (int j = tid; j < p.P; j += NT) spred[j] = p.pred[static_cast<size_t>(u) * p.P + j];
  if (use_gs) {
    const uint2* src = p.gsum + static_cast<size_t>(u) * W;
    for (int g = tid; g < Wn; g += NT) gs[g] = __ldcg(src + g);
  }
  if (!take_all && nb <= kEagerKeys) {  // with the summaries: no second round trip if no tie
    load_words_cg(skeys, p.keys + static_cast<size_t>(u) * p.maxnb, nb, grp);
    have_keys = true;
  }
  for (int i = tid; i < W; i += NT) bm_pred[i] = 0u;
  if (tid < 16) misc[tid] = 0;
  gsync(grp);
  PRR_PHASE(0, u, 1);
  int active_local = 0;
  for (int j = tid; j < p.P; j += NT) {
    const int pv = spred[j];
    if (pv >= 0 && pv < nb) {
      ++active_local;
      atomicOr(&bm_pred[pv >> 5], 1u << (pv & 31));
      if (j > 0 && spred[j - 1] >= pv) report(p.status, kDevBadPred);
    } else if (pv != -1) {
      report(p.status, kDevBadPred);
    }
  }
  uint32_t T = 0u;
  int n_gt = 0;
  bool tie_masks = false;  // S comes straight from the group tie masks
  if (!take_all && keff > 0) {
    unsigned* ms = reinterpret_cast<unsigned*>(misc);
    // largest key and the number of blocks holding it
    uint32_t mx = 0u;
    if (use_gs) {
      for (int g = tid; g < Wn; g += NT) mx = max(mx, gs[g].x);
    } else {
      for (int i = tid; i < nb; i += NT) mx = max(mx, skeys[i]);
    }
    mx = __reduce_max_sync(kFull, mx);
    if (lane == 0) atomicMax(&ms[6], mx);
    gsync(grp);
    const uint32_t gmax = ms[6];
    int ce = 0;
    if (use_gs) {
      for (int g = tid; g < Wn; g += NT) ce += gs[g].x == gmax ? __popc(gs[g].y) : 0;
    } else {
      for (int i = tid; i < nb; i += NT) ce += skeys[i] == gmax ? 1 : 0;
    }
    ce = __reduce_add_sync(kFull, ce);
    if (lane == 0 && ce) atomicAdd(&misc[7], ce);
    gsync(grp);
    if (misc[7] >= keff) {
      T = gmax;
      tie_masks = use_gs;
    } else {
      if (!have_keys && !take_all) {
        load_words_cg(skeys, p.keys + static_cast<size_t>(u) * p.maxnb, nb, grp);
        have_keys = true;
        gsync(grp);
      }
      // T: the K_eff-th largest key, by radix selection over the whole group (8-bit
      // digits from the first byte the keys differ in; lanes of a warp that fall in the
      // same bin add in one atomic, so ties at the threshold stay cheap)
      unsigned* hist = reinterpret_cast<unsigned*>(scratch);  // first 1 KB of the scratch
      int gt = 0;
      T = radix_kth_largest(
          nb, keff, [&](int i) { return skeys[i]; }, [](int) { return true; }, hist, misc + 10, &gt, grp);
      n_gt = gt;
    }
  }
  PRR_PHASE(0, u, 2);
  if (tie_masks) {
    // the first K_eff tied blocks in index order: trim the maximal groups' masks
    if (warp == 0) {
      int base = 0;
      for (int w0 = 0; w0 < Wn; w0 += 32) {
        const int wd = w0 + lane;
        unsigned m = 0u;
        if (wd < Wn) {
          const uint2 g = gs[wd];
          m = g.x == T ? g.y : 0u;
        }
        const int c = __popc(m);
        const int inc = warp_inclusive_sum(c);
        const int exc = base + inc - c;
        unsigned keepm = 0u;
        if (exc < keff) {
          const int need = keff - exc;
          keepm = m;
          if (need < c) {
            keepm = 0u;
            unsigned e = m;
            for (int r = 0; r < need; ++r) {
              const unsigned low = e & (0u - e);
              keepm |= low;
              e ^= low;
            }
          }
        }
        if (wd < Wn) bm_sel[wd] = keepm;
        base += __shfl_sync(kFull, inc, 31);
      }
    }
    gsync(grp);
  } else {
    select_bitmap(
        nb, take_all ? 0 : keff - n_gt,
        [&](int i) {
          if (take_all) return 1;
          const uint32_t kv = skeys[i];
          return kv > T ? 1 : (kv == T ? 0 : -1);
        },
        bm_sel, bm_eq, grp);
  }
  PRR_PHASE(0, u, 3);
  // three warps in parallel: selected list, missed list, keep mask
  int nm = 0;
  if (warp == 0) {
    warp_emit_bitmap(bm_sel, nullptr, Wn, p.sel + static_cast<size_t>(u) * p.K, p.K);
  } else if (warp == 1) {
    // missed list; each missed block is handed to its repair slot and, since the repair
    // reads it next, started toward L2
    nm = warp_emit_bitmap(bm_sel, bm_pred, Wn, p.missed + static_cast<size_t>(u) * p.K, p.K, [&](int pos, int b) {
      if (rdesc) rdesc[pos] = static_cast<unsigned>(b) + 1u;
      if (p.kc && p.vc) {
        const int rows = p.table ? p.bs : min(p.bs, p.cap - b * p.bs);
        const long long r0 = kv_row(p, u / p.kv_div, b * p.bs);  // a block's rows are contiguous
        if (r0 >= 0) {
          const size_t off = static_cast<size_t>(r0) * p.d;
          prefetch_l2(p.kc + off, static_cast<uint32_t>(rows) * p.d * 2);
          prefetch_l2(p.vc + off, static_cast<uint32_t>(rows) * p.d * 2);
        }
      }
    });
    if (rdesc)
      for (int e = nm + lane; e < p.K; e += 32) rdesc[e] = kNoRepair;
    if ((tid & 31) == 0) {
      p.n_missed[u] = nm;
      misc[2] = nm;
    }
  }
  for (int j = tid; j < p.P; j += NT) {
    const int pv = spred[j];
    const unsigned kv = (pv >= 0 && pv < nb && ((bm_sel[pv >> 5] >> (pv & 31)) & 1u)) ? 1u : 0u;
    p.keep[static_cast<size_t>(u) * p.P + j] = static_cast<uint8_t>(kv);
    if (keepf) keepf[j] = 1u | (kv << 1);
  }
  PRR_PHASE(0, u, 4);
  // active predicted slots (CTA sum of the per-thread counts)
  if (tid == 0) misc[3] = 0;
  gsync(grp);
  if (active_local) atomicAdd(&misc[3], active_local);
  gsync(grp);
  PRR_PHASE(0, u, 5);
  const int path = take_all ? kStatTakeAll : (tie_masks ? kStatTieMasks : kStatKeySearch);
  if (tid == 0 && keff > 0) bump(p.stats, path);
  return FinishOut{misc[3], misc[2], path};
}

// ------------------------------------------------------------------ EMA predictor
//
// PRR abstract and method summary: an exponential moving average of past selections
// forecasts the next step's blocks.  Reading taken (the pages print no formula):
//   e_b <- alpha*e_b + beta*[b in S_t],  beta = 1 - alpha,  e starts at 0,
// in fp64 with separately rounded multiplies and add (no fused multiply-add), so the
// state and the predicted set are bit-exact against the fp64 CPU oracle.
// Pred_{t+1} = the min(P, nb) best blocks under (e desc, index asc), ascending, -1
// beyond.  e >= 0, so its IEEE bit pattern orders like its value.
//
// Candidate filter (exact): after the update every block of S_t holds e >= beta (a
// rounded sum of beta and a non-negative term), so when P_eff <= |S_t| the P-th
// largest e is >= beta and the whole predicted set lies among the blocks with
// e >= beta.  Those candidates (typically about K of them, given temporal locality)
// are collected during the update and ranked by counting: rank(i) = #{j : e_j > e_i,
// or e_j == e_i and j < i}; rank < P_eff is selected.  Otherwise (P > |S_t|, no
// update, or too many candidates) the general path runs: radix selection on the
// high word, then on the low word among the entries tied on the high word.

constexpr int kEmaCand = 512;  // candidates ranked by counting; more take the radix path

__host__ __device__ constexpr size_t ema_scratch_bytes(int maxnb) {
  return 256 * 4 + 16 * 4 + static_cast<size_t>(kEmaCand) * 12 + static_cast<size_t>(maxnb) * 8 +
         3 * static_cast<size_t>((maxnb + 31) / 32) * 4;
}

// Every thread of the CTA calls it.  wait_sel() (CTA-wide) returns once S_t may be read,
// false to give up; the state copy is started before it, so its latency is hidden.
template <typename WaitFn>
__device__ inline void ema_unit(const Params& p, int u, unsigned char* scratch, WaitFn wait_sel, const Grp& grp) {
  const int W = (p.maxnb + 31) / 32;
  unsigned* hist = reinterpret_cast<unsigned*>(scratch);  // 16-byte aligned
  int* misc = reinterpret_cast<int*>(hist + 256);         // [4] candidates, [5] |S_t|
  unsigned long long* ckey = reinterpret_cast<unsigned long long*>(misc + 16);
  int* cidx = reinterpret_cast<int*>(ckey + kEmaCand);
  double* ev = reinterpret_cast<double*>(cidx + kEmaCand);  // state, up to the allocation
  unsigned* bm = reinterpret_cast<unsigned*>(ev + p.maxnb);  // selected blocks of this step
  unsigned* bsel = bm + W;                                    // predicted set
  unsigned* beq = bsel + W;

  const int tid = grp.tid, warp = tid >> 5, lane = tid & 31, NT = grp.nt;
  PRR_PHASE(1, u, 0);
  double* e = p.ema + static_cast<size_t>(u) * p.maxnb;
  const bool update = p.sel != nullptr;
  // state copy up to the allocation (entries >= nb are unused), before any wait
  for (int i = tid; i < p.maxnb; i += NT) cp_async_8(ev + i, e + i);
  for (int i = tid; i < W; i += NT) {
    bm[i] = 0u;
    bsel[i] = 0u;
  }
  if (tid == 0) {
    misc[4] = 0;
    misc[5] = 0;
  }
  if (!wait_sel()) {
    cp_async_wait_all();
    gsync(grp);
    return;
  }
  int sv = -1;
  if (update && tid < p.K) sv = __ldcg(p.sel + static_cast<size_t>(u) * p.K + tid);
  const int n = checked_len(p, u / p.upb, grp);
  const int nb = (n + p.bs - 1) / p.bs;
  const int Wn = (nb + 31) / 32;
  const int peff = min(p.P, nb);
  cp_async_wait_all();
  gsync(grp);
  bool ranked = false;
  if (update) {
    for (int i = tid; i < p.K; i += NT) {
      const int v = i == tid ? sv : __ldcg(p.sel + static_cast<size_t>(u) * p.K + i);
      if (v >= 0 && v < nb) atomicOr(&bm[v >> 5], 1u << (v & 31));
    }
    gsync(grp);
    int nsel = 0;
    for (int i = tid; i < Wn; i += NT) nsel += __popc(bm[i]);
    if (nsel) atomicAdd(&misc[5], nsel);
    gsync(grp);
    const bool filter = peff > 0 && peff < nb && peff <= misc[5];
    const double alpha = p.alpha;
    const double beta = __dsub_rn(1.0, alpha);
    for (int base = 0; base < nb; base += NT) {  // warp-uniform trip count
      const int i = base + tid;
      bool cand = false;
      unsigned long long bits = 0ull;
      if (i < nb) {
        const double ind = ((bm[i >> 5] >> (i & 31)) & 1u) ? 1.0 : 0.0;
        const double x = __dadd_rn(__dmul_rn(alpha, ev[i]), __dmul_rn(beta, ind));
        e[i] = x;
        ev[i] = x;
        bits = static_cast<unsigned long long>(__double_as_longlong(x));
        cand = filter && x >= beta;
      }
      const unsigned bal = __ballot_sync(kFull, cand);
      if (bal) {
        int wbase = 0;
        if (lane == 0) wbase = atomicAdd(&misc[4], __popc(bal));
        wbase = __shfl_sync(kFull, wbase, 0);
        const int slot = wbase + __popc(bal & ((1u << lane) - 1u));
        if (cand && slot < kEmaCand) {
          ckey[slot] = bits;
          cidx[slot] = i;
        }
      }
    }
    gsync(grp);
    const int cnt = misc[4];
    if (filter && cnt <= kEmaCand) {
      ranked = true;
      for (int c = tid; c < cnt; c += NT) {
        const unsigned long long kc = ckey[c];
        const int ic = cidx[c];
        int rank = 0;
        for (int j = 0; j < cnt; ++j) {
          const unsigned long long kj = ckey[j];
          rank += (kj > kc) | ((kj == kc) & (cidx[j] < ic));
        }
        if (rank < peff) atomicOr(&bsel[ic >> 5], 1u << (ic & 31));
      }
      gsync(grp);
    }
  }
  PRR_PHASE(1, u, 1);

  int* out = p.pred_next + static_cast<size_t>(u) * p.P;
  if (peff <= 0) {
    for (int j = tid; j < p.P; j += NT) out[j] = -1;
    return;
  }
  auto hi = [&](int i) { return static_cast<uint32_t>(static_cast<unsigned long long>(__double_as_longlong(ev[i])) >> 32); };
  auto lo = [&](int i) { return static_cast<uint32_t>(static_cast<unsigned long long>(__double_as_longlong(ev[i]))); };
  if (ranked) {
    // bsel holds the predicted set
  } else if (peff >= nb) {
    select_bitmap(nb, 0, [&](int) { return 1; }, bsel, beq, grp);
  } else {
    int gt_hi = 0, gt_lo = 0;
    const uint32_t Thi = radix_kth_largest(nb, peff, hi, [&](int) { return true; }, hist, misc, &gt_hi, grp);
    PRR_PHASE(1, u, 2);
    const int need = peff - gt_hi;  // taken from the entries tied on the high word
    // low word among the entries tied on the high word (no pass at all when they agree)
    const uint32_t Tlo = radix_kth_largest(
        nb, need, lo, [&](int i) { return hi(i) == Thi; }, hist, misc, &gt_lo, grp);
    PRR_PHASE(1, u, 3);
    select_bitmap(
        nb, need - gt_lo,
        [&](int i) {
          const uint32_t h = hi(i);
          if (h != Thi) return h > Thi ? 1 : -1;
          const uint32_t l = lo(i);
          return l > Tlo ? 1 : (l == Tlo ? 0 : -1);
        },
        bsel, beq, grp);
  }
  if (warp == 0) warp_emit_bitmap(bsel, nullptr, Wn, out, p.P);
  gsync(grp);
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
// 128 threads.  Each warp folds its share of the slots into a running (m, l, O) state
// (O: one float4 column per lane), rescaling when a larger max arrives, so loads never
// wait for a CTA-wide maximum; the four warp states are combined at the end.  The
// speculative slots are folded first; `wait_repair()` (CTA-uniform) runs between the
// two phases, so a caller can start on the speculative part before repair is done.

__host__ __device__ constexpr size_t combine_scratch_bytes(int P, int D) {
  return static_cast<size_t>(P) * 12 + 16 * 4 + 4 * static_cast<size_t>(D) * 4 + 64;
}

struct WarpState {
  float m;  // running max (base-2 logits), -inf when empty
  float l;  // running sum, relative to m (meaningful in lane 0; all lanes agree)
  float4 o; // running numerator column of this lane, relative to m
};

// Fold up to B slots (values already loaded) into the warp state.
template <int B>
__device__ __forceinline__ void fold_batch(WarpState& st, const float (&m)[B], const float (&l)[B],
                                           const float4 (&o)[B]) {
  float mb = st.m;
#pragma unroll
  for (int q = 0; q < B; ++q) mb = fmaxf(mb, m[q]);
  if (mb == -INFINITY) return;
  const float sc = st.m == -INFINITY ? 0.f : exp2f(st.m - mb);
  st.l *= sc;
  st.o.x *= sc;
  st.o.y *= sc;
  st.o.z *= sc;
  st.o.w *= sc;
#pragma unroll
  for (int q = 0; q < B; ++q) {
    const float w = m[q] == -INFINITY ? 0.f : exp2f(m[q] - mb);
    st.l = fmaf(w, l[q], st.l);
    st.o.x = fmaf(w, o[q].x, st.o.x);
    st.o.y = fmaf(w, o[q].y, st.o.y);
    st.o.z = fmaf(w, o[q].z, st.o.z);
    st.o.w = fmaf(w, o[q].w, st.o.w);
  }
  st.m = mb;
}

template <int D, typename WaitFn>
__device__ void combine_head(const Params& p, int u, int h, unsigned char* scratch, WaitFn wait_repair,
                             const Grp& grp) {
  constexpr int C4 = D / 4;
  constexpr int B = 8;  // slots per batch and warp: 8 float4 loads in flight per lane
  const int P = p.P, K = p.K;
  float* km = reinterpret_cast<float*>(scratch);  // [P] kept slot max or -inf
  float* kl = km + P;                             // [P]
  int* slots = reinterpret_cast<int*>(kl + P);    // [P] compacted kept slots
  float* red = reinterpret_cast<float*>(slots + P);  // [4] m, [4] l, count
  int* count = reinterpret_cast<int*>(red + 8);
  float4* part = reinterpret_cast<float4*>((reinterpret_cast<uintptr_t>(red + 16) + 15) &
                                           ~static_cast<uintptr_t>(15));  // [4][C4]
  const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
  const size_t row = static_cast<size_t>(u) * p.G + h;
  const bool col = lane < C4;
  WarpState st{-INFINITY, 0.f, make_float4(0.f, 0.f, 0.f, 0.f)};

  // ---- speculative slots: flags and statistics in one round trip, then numerators
  for (int j = tid; j < P; j += grp.nt) {
    const bool act = __ldcg(p.keep + static_cast<size_t>(u) * P + j) != 0;
    const float m = __ldcg(p.pm + row * P + j);
    const float l = __ldcg(p.pl + row * P + j);
    km[j] = act ? m : -INFINITY;
    kl[j] = act ? l : 0.f;
  }
  gsync(grp);
  if (warp == 0) {
    int cnt = 0;
    for (int base = 0; base < P; base += 32) {
      const int j = base + lane;
      const bool a = j < P && km[j] != -INFINITY;
      const unsigned mask = __ballot_sync(0xFFFFFFFFu, a);
      if (a) slots[cnt + __popc(mask & ((1u << lane) - 1u))] = j;
      cnt += __popc(mask);
    }
    if (lane == 0) count[0] = cnt;
  }
  gsync(grp);
  const int ns = count[0];
  for (int s0 = warp; s0 < ns; s0 += 4 * B) {
    float m[B], l[B];
    float4 o[B];
#pragma unroll
    for (int q = 0; q < B; ++q) {
      const int si = s0 + 4 * q;
      m[q] = -INFINITY;
      l[q] = 0.f;
      o[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (si < ns) {
        const int j = slots[si];
        m[q] = km[j];
        l[q] = kl[j];
        if (col) o[q] = __ldcg(reinterpret_cast<const float4*>(p.pO + (row * P + j) * D) + lane);
      }
    }
    fold_batch<B>(st, m, l, o);
  }

  // ---- repair slots: statistics and numerators in one round trip
  if (wait_repair()) {
    const int nm = min(max(__ldcg(p.n_missed + u), 0), K);
    for (int i0 = warp; i0 < nm; i0 += 4 * B) {
      float m[B], l[B];
      float4 o[B];
#pragma unroll
      for (int q = 0; q < B; ++q) {
        const int i = i0 + 4 * q;
        m[q] = -INFINITY;
        l[q] = 0.f;
        o[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < nm) {
          m[q] = __ldcg(p.rm + row * K + i);
          l[q] = __ldcg(p.rl + row * K + i);
          if (col) o[q] = __ldcg(reinterpret_cast<const float4*>(p.rO + (row * K + i) * D) + lane);
        }
      }
      fold_batch<B>(st, m, l, o);
    }
  }

  // ---- combine the four warp states
  if (lane == 0) {
    red[warp] = st.m;
    red[4 + warp] = st.l;
  }
  if (col) part[warp * C4 + lane] = st.o;
  gsync(grp);
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float L = 0.f, f[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    f[w] = (red[w] == -INFINITY || M == -INFINITY) ? 0.f : exp2f(red[w] - M);
    L = fmaf(f[w], red[4 + w], L);
  }
  if (tid < C4) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float4 v = part[w * C4 + tid];
      o.x = fmaf(f[w], v.x, o.x);
      o.y = fmaf(f[w], v.y, o.y);
      o.z = fmaf(f[w], v.z, o.z);
      o.w = fmaf(f[w], v.w, o.w);
    }
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    o.x *= inv;
    o.y *= inv;
    o.z *= inv;
    o.w *= inv;
    reinterpret_cast<float4*>(p.out + row * D)[tid] = o;
  }
  if (tid == 0) p.lse[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
  gsync(grp);
}

}  // namespace prr
