// prr_schedule.h -- work items of one fused decode-step launch: how many of each kind
// it runs and the order in which its ticket counter hands them out.
//
// Plain C++ with no CUDA types, so that the host and the kernel share one definition
// and a host program can check the order (every item exactly once; every item after
// all the items it waits for, which is what keeps the persistent grid free of
// deadlock).
//
// Tickets, per launch, with U units, F selection chunks per unit, P predicted slots,
// R repair items and G merges (one per query head of the group) per unit:
//   [0, U*F)                 SEL      unit-major: unit t / F scores chunk t % F
//   [U*F, U*F + U)           FIN      the finisher of one unit (waits for its F chunks)
//   next U                   EMA      the predictor update of one unit (waits for FIN)
//   the rest                 SPEC, REPAIR and COMBINE, interleaved by decode_tail:
//                            REPAIR waits for its unit's FIN; COMBINE for its unit's
//                            FIN, every SPEC and every REPAIR.
#pragma once

#include <cstddef>

#if defined(__CUDACC__)
#define PRR_HD __host__ __device__ __forceinline__
#else
#define PRR_HD inline
#endif

namespace prr {

constexpr int kFusedChunk = 128;  // most blocks per SEL item (4 warps x 32 rows)

// Blocks per SEL item: a multiple of 32 in [32, 128], about units*maxnb/512, so that a
// short context still spreads its scan over many CTAs and a long one moves 64 KB per item.
PRR_HD int fused_chunk_blocks(int units, int maxnb) {
  long long c = (static_cast<long long>(units) * maxnb + 511) / 512;
  c = ((c + 31) / 32) * 32;
  return static_cast<int>(c < 32 ? 32 : (c > kFusedChunk ? kFusedChunk : c));
}

// REPAIR items per unit: enough that a unit with many misses spreads them over CTAs,
// few enough that most items have work.
PRR_HD int fused_rep_items(int units, int K) {
  const int r = (1024 + units - 1) / units;
  const int lo = r > 4 ? r : 4;
  return K < lo ? K : lo;
}

// Units whose SPEC tickets separate a unit's last SPEC ticket from its first dependent
// ticket: enough for about two rounds of a grid of `grid` CTAs, so that by the time a
// CTA takes a REPAIR or COMBINE ticket its unit's selection has long been published.
PRR_HD int fused_dep_lag(long long grid, int P, int units) {
  return P > 0 ? static_cast<int>((2 * grid + P - 1) / P) : units;
}

// Items of one launch (the ticket counter runs over [0, this)).
PRR_HD long long fused_total_items(int units, int fchunks, int P, int R, int G) {
  return static_cast<long long>(units) * (fchunks + 1 + 1 + P + R + G);
}

// Tickets after the predictor updates (t counts from the first of them), with
// Lc = min(dep_lag, U) and M = R + G dependent items per unit: first the SPEC tickets
// of units 0..Lc-1 (P each); then, for k = 0..U-Lc-1, the SPEC tickets of unit Lc+k
// followed by unit k's R REPAIR and G COMBINE tickets; last the dependent tickets of
// units U-Lc..U-1.  Every dependent ticket comes after all of its unit's SPEC tickets.
// Returns false for a SPEC ticket (*idx = unit * P + slot), true for a dependent one
// (*kind 3 with *idx = unit * R + r, or 5 with *idx = unit * G + h).
PRR_HD bool decode_tail(int P, int G, int dep_lag, int t, int U, int R, int* idx, int* kind) {
  const int M = R + G;
  const int Lc = dep_lag < U ? dep_lag : U;
  int v, r;  // unit and index of a dependent ticket
  if (t < Lc * P) {
    *idx = t;
    return false;
  }
  t -= Lc * P;
  const int mid = (U - Lc) * (P + M);
  if (t < mid) {
    const int k = t / (P + M), q = t % (P + M);
    if (q < P) {
      *idx = (Lc + k) * P + q;
      return false;
    }
    v = k;
    r = q - P;
  } else {
    t -= mid;
    v = U - Lc + t / M;
    r = t % M;
  }
  if (r < R) {
    *kind = 3;
    *idx = v * R + r;
  } else {
    *kind = 5;
    *idx = v * G + (r - R);
  }
  return true;
}

}  // namespace prr
