// prr_attn.cuh -- online-softmax statistics of ONE KV block for all G query heads of a
// GQA group: the unit of speculation and of repair.
//
// PRR abstract / method summary: attention over the predicted blocks runs while the
// selection is in flight; once the true set is known the missed blocks are attended
// and everything is merged through online-softmax statistics.  Per block and head:
//   m = max_i s_i,  l = sum_i 2^(s_i - m),  O = sum_i 2^(s_i - m) v_i
// with s_i = scale*log2(e) * q.k_i (base-2 logits) over the block's tokens below n.
// One partial per block means a predicted block that selection drops is simply never
// merged (reuse = keep the partials of Pred n S).
//
// Data path (sm_100a): the block's K and V tiles ([bs][d] bf16, contiguous in the
// cache) arrive by 3-D TMA with the 128-byte swizzle, one mbarrier each, so the
// ldmatrix reads below are bank-conflict free.  Each staged tile is shared by all G
// heads.  Both products run on the tensor cores with mma.m16n8k16 in swap-AB form:
//   S^T[tok][h] = K[tok][:] . Q^T[:][h]     (M = 16 tokens, N = 8 heads, K = d)
//   O^T[c][h]   = V^T[c][tok] . P^T[tok][h] (M = 16 channels, N = 8 heads, K = tokens)
// P is split as bf16 hi + bf16 lo (two MMAs) so the PV product keeps ~16 mantissa
// bits.  For S^T and the softmax the four warps own token slices; P goes through a
// small buffer in the dead K tile, and for O^T they own channel slices over all
// tokens, so each warp finishes whole output columns and the tiles are free before the
// partial is written out.
//
// The copies and the arithmetic are separate steps (attn_issue, attn_compute): one
// thread issues the copies, then the whole CTA computes (block_partial runs both).
#pragma once

#include "prr_kernels.cuh"

namespace prr {

template <int D, int BS>
struct AttnTile {
  static constexpr int TILEB = BS * D * 2;  // one K or V tile
  static constexpr int REGB = BS * 128;     // one 64-channel swizzle region of a tile
  static constexpr int REDB = 80 * 4;       // cross-warp reductions
  static constexpr size_t bytes = 2 * static_cast<size_t>(TILEB) + REDB;  // tiles + reductions
};

// Where one block's partial goes: m/l of head h at m[h*rstride], O at O[h*ostride].
struct PartialDst {
  float* m;
  float* l;
  float* O;
  size_t rstride;
  size_t ostride;
};

__device__ __forceinline__ void write_empty_partial(const PartialDst& dst, int G, int D, const Grp& g) {
  for (int e = g.tid; e < G * D; e += g.nt) dst.O[(e / D) * dst.ostride + (e % D)] = 0.f;
  if (g.tid < G) {
    dst.m[g.tid * dst.rstride] = -INFINITY;
    dst.l[g.tid * dst.rstride] = 0.f;
  }
}

// One thread: start the K and V tiles of block `blk` of KV slice `slice` (the
// tensor maps' third coordinate) towards sK / sV, completing on barK / barV.  Earlier
// generic writes of this thread to the tiles are ordered before the copies.
template <int D, int BS>
__device__ __forceinline__ void attn_issue(const CUtensorMap* kmap, const CUtensorMap* vmap, int slice, int tok0,
                                           unsigned char* sK, unsigned char* sV, uint64_t* barK, uint64_t* barV) {
  using L = AttnTile<D, BS>;
  constexpr int NREG = D / 64;
  fence_proxy_async();
  mbar_expect_tx(barK, L::TILEB);
#pragma unroll
  for (int r = 0; r < NREG; ++r) tma_load_3d(sK + r * L::REGB, kmap, barK, r * 64, tok0, slice);
  mbar_expect_tx(barV, L::TILEB);
#pragma unroll
  for (int r = 0; r < NREG; ++r) tma_load_3d(sV + r * L::REGB, vmap, barV, r * 64, tok0, slice);
}

// Write one token row (d bf16, 16-byte aligned, global) into row r of a staged tile in
// its 128-byte swizzled position.  The group's first D/8 threads each move 16 bytes.
template <int D, int BS>
__device__ __forceinline__ void tile_put_row(unsigned char* tile, int r, const uint16_t* row, const Grp& g) {
  using L = AttnTile<D, BS>;
  if (g.tid < D / 8) {
    const int rr = g.tid >> 3, c16 = g.tid & 7;
    *reinterpret_cast<uint4*>(tile + rr * L::REGB + r * 128 + ((c16 ^ (r & 7)) << 4)) =
        *reinterpret_cast<const uint4*>(row + g.tid * 8);
  }
}

// Partial of the block whose K/V tiles are (being) staged in sK / sV, tokens below n of
// block `blk`.  Every thread of a 128-thread group calls it.  `q` points at the G query
// rows of the unit ([G][D] bf16, global or shared).  barK / barV are the tiles'
// mbarriers, waited on with parity `phase` (bounded).  When `patch_k` is not null, the
// token n-1 (which lies in this block) is taken from patch_k / patch_v instead of the
// staged tiles (the caller has not written it to the cache yet).  `red` is 80 floats of
// shared scratch.  tiles_free() is called by every thread once no thread reads the
// tiles any more -- before the partial is written out -- so a caller can hand the
// buffers back early.  Returns false if a copy did not land in time (status word set;
// tiles_free is then not called).
//
// Work split: for S^T and the softmax each warp owns a slice of the tokens; P (bf16
// high and low parts) then goes through a small buffer in the dead K tile, and for
// O^T = V^T P^T each warp owns a slice of the channels over all tokens, so every warp
// finishes whole output columns and no cross-warp sum of O is needed.
template <int D, int BS, typename TilesFree>
__device__ bool attn_compute(const Params& p, const uint16_t* q, int blk, int n, const PartialDst& dst,
                             unsigned char* sK, unsigned char* sV, float* red, uint64_t* barK, uint64_t* barV,
                             uint32_t phase, const Grp& grp, TilesFree tiles_free, const uint16_t* patch_k = nullptr,
                             const uint16_t* patch_v = nullptr, unsigned long long* t_v = nullptr) {
  using L = AttnTile<D, BS>;
  constexpr int REGB = L::REGB, NREG = D / 64;
  constexpr int MTW = BS / 64;  // 16-token m-tiles per warp for S^T (4 warps)
  constexpr int KS = D / 16;    // k-steps of QK^T == 16-channel tiles of PV
  constexpr int CT = KS / 4;    // 16-channel tiles per warp for O^T
  constexpr int PST = BS + 8;   // row stride (bf16) of the P buffer; the pad spreads rows over banks
  static_assert(2 * 8 * PST * 2 <= L::TILEB, "P buffer fits in the K tile");
  const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;

  // Q^T fragments (B operand of the score product): lane (g, t) holds head g,
  // channels 16ks + 2t, +1 and 16ks + 2t + 8, +9.  Heads >= G are zero.
  const int g = lane >> 2, t = lane & 3;
  uint32_t qf[KS][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(q + (g < G ? g : 0) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qf[ks][0] = g < G ? qrow[ks * 8 + t] : 0u;
      qf[ks][1] = g < G ? qrow[ks * 8 + 4 + t] : 0u;
    }
  }

  const int nv = min(BS, n - blk * BS);  // valid tokens of this block
  const int prow = n - 1 - blk * BS;      // row of token n-1 when a patch is given
  if (!gsync_and(grp, mbar_wait(barK, phase, p.status))) {
    if (tid == 0) mbar_wait(barV, phase, p.status);  // let the V copy land (bounded)
    return false;
  }
  if (patch_k) {
    tile_put_row<D, BS>(sK, prow, patch_k, grp);
    gsync(grp);
  }

  // ---- S^T = K Q^T on the tensor cores (this warp's tokens)
  const uint32_t sK_addr = smem_addr(sK), sV_addr = smem_addr(sV);
  float sc[MTW][4];
#pragma unroll
  for (int mi = 0; mi < MTW; ++mi) {
    const int mt = warp * MTW + mi;
    sc[mi][0] = sc[mi][1] = sc[mi][2] = sc[mi][3] = 0.f;
    const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int ch = 2 * ks + (lane >> 4);
      const uint32_t addr = sK_addr + (ch >> 3) * REGB + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
      uint32_t a[4];
      ldsm_x4(addr, a);
      mma_16816(sc[mi], a, qf[ks][0], qf[ks][1]);
    }
  }
  // base-2 logits; tokens >= nv masked.  sc[mi][0..1]: token 16mt+g, heads 2t, 2t+1;
  // sc[mi][2..3]: token 16mt+g+8.
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int mi = 0; mi < MTW; ++mi) {
    const int tok = (warp * MTW + mi) * 16 + g;
    const bool v0 = tok < nv, v1 = tok + 8 < nv;
    sc[mi][0] = v0 ? sc[mi][0] * p.scale_log2 : -INFINITY;
    sc[mi][1] = v0 ? sc[mi][1] * p.scale_log2 : -INFINITY;
    sc[mi][2] = v1 ? sc[mi][2] * p.scale_log2 : -INFINITY;
    sc[mi][3] = v1 ? sc[mi][3] * p.scale_log2 : -INFINITY;
    mx0 = fmaxf(mx0, fmaxf(sc[mi][0], sc[mi][2]));
    mx1 = fmaxf(mx1, fmaxf(sc[mi][1], sc[mi][3]));
  }
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, o));
  }
  if (g == 0) {
    red[warp * 8 + 2 * t] = mx0;
    red[warp * 8 + 2 * t + 1] = mx1;
  }
  gsync(grp);  // the maxima are visible, and every warp is past its reads of the K tile
  float m0 = red[2 * t], m1 = red[2 * t + 1];
#pragma unroll
  for (int w = 1; w < 4; ++w) {
    m0 = fmaxf(m0, red[w * 8 + 2 * t]);
    m1 = fmaxf(m1, red[w * 8 + 2 * t + 1]);
  }

  // ---- P = 2^(s - m) as bf16 high + low parts, [head][token] in the dead K tile
  uint16_t* Ph = reinterpret_cast<uint16_t*>(sK);
  uint16_t* Pl = Ph + 8 * PST;
  float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
  for (int mi = 0; mi < MTW; ++mi) {
    const int tok = (warp * MTW + mi) * 16 + g;
    const float pv[4] = {exp2f(sc[mi][0] - m0), exp2f(sc[mi][1] - m1), exp2f(sc[mi][2] - m0),
                         exp2f(sc[mi][3] - m1)};
    ls0 += pv[0] + pv[2];
    ls1 += pv[1] + pv[3];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * t + (e & 1), tk = tok + (e >> 1) * 8;
      const __nv_bfloat16 hi = __float2bfloat16_rn(pv[e]);
      const __nv_bfloat16 lo = __float2bfloat16_rn(pv[e] - __bfloat162float(hi));
      Ph[h * PST + tk] = __bfloat16_as_ushort(hi);
      Pl[h * PST + tk] = __bfloat16_as_ushort(lo);
    }
  }
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1) {
    ls0 += __shfl_xor_sync(0xFFFFFFFFu, ls0, o);
    ls1 += __shfl_xor_sync(0xFFFFFFFFu, ls1, o);
  }
  if (g == 0) {
    red[32 + warp * 8 + 2 * t] = ls0;
    red[32 + warp * 8 + 2 * t + 1] = ls1;
  }

  if (!gsync_and(grp, mbar_wait(barV, phase, p.status))) return false;  // also publishes P
  if (t_v && tid == 0) *t_v = global_ns();  // debug timelines: the V tile is usable
  if (nv < BS) {  // tokens past the end of the sequence: zero V so 0 * V stays 0
    uint4* v4 = reinterpret_cast<uint4*>(sV);
    const int rows = BS - nv;
    for (int i = tid; i < rows * NREG * 8; i += grp.nt) {
      const int r = nv + i / (NREG * 8), rem = i % (NREG * 8);
      v4[((rem >> 3) * REGB + r * 128) / 16 + (rem & 7)] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (patch_v) tile_put_row<D, BS>(sV, prow, patch_v, grp);
  gsync(grp);
  if (warp == 0 && g == 0) {
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      l0 += red[32 + w * 8 + 2 * t];
      l1 += red[32 + w * 8 + 2 * t + 1];
    }
    red[64 + 2 * t] = m0;
    red[64 + 2 * t + 1] = m1;
    red[72 + 2 * t] = l0;
    red[72 + 2 * t + 1] = l1;
  }

  // ---- O^T = V^T P^T on the tensor cores (this warp's channels, all tokens)
  float oacc[CT][4];
#pragma unroll
  for (int ct = 0; ct < CT; ++ct) oacc[ct][0] = oacc[ct][1] = oacc[ct][2] = oacc[ct][3] = 0.f;
  const uint32_t pb_addr = smem_addr(((lane >> 4) ? Pl : Ph) + (lane & 7) * PST + ((lane >> 3) & 1) * 8);
#pragma unroll
  for (int kt = 0; kt < BS / 16; ++kt) {
    uint32_t b[4];  // P^T fragments of tokens 16kt..: high part (k 0-7, 8-15), low part
    ldsm_x4(pb_addr + kt * 32, b);
    const int row = kt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
    for (int ct = 0; ct < CT; ++ct) {
      const int dt = warp * CT + ct;
      const int ch = 2 * dt + ((lane >> 3) & 1);
      const uint32_t addr = sV_addr + (ch >> 3) * REGB + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
      uint32_t a[4];
      ldsm_x4_trans(addr, a);
      mma_16816(oacc[ct], a, b[0], b[1]);
      mma_16816(oacc[ct], a, b[2], b[3]);
    }
  }
  fence_proxy_async();  // this thread's generic writes to the tiles precede later copies
  gsync(grp);           // no thread reads the tiles any more
  tiles_free();

  // ---- the partial: whole columns from each warp, m and l from the reductions
#pragma unroll
  for (int ct = 0; ct < CT; ++ct) {
    const int c0 = (warp * CT + ct) * 16 + g;
    const int h0 = 2 * t, h1 = 2 * t + 1;
    if (h0 < G) {
      dst.O[h0 * dst.ostride + c0] = oacc[ct][0];
      dst.O[h0 * dst.ostride + c0 + 8] = oacc[ct][2];
    }
    if (h1 < G) {
      dst.O[h1 * dst.ostride + c0] = oacc[ct][1];
      dst.O[h1 * dst.ostride + c0 + 8] = oacc[ct][3];
    }
  }
  if (tid < G) {
    dst.m[tid * dst.rstride] = red[64 + tid];
    dst.l[tid * dst.rstride] = red[72 + tid];
  }
  return true;
}

// Both steps in one group: partial of block `blk` of unit u.  `smem` is 1024-byte
// aligned with AttnTile::bytes free; bars[0], bars[1] are initialised mbarriers (count
// 1) whose current phase parity is `phase`.  patch_k / patch_v: see attn_compute.
template <int D, int BS>
__device__ bool block_partial(const Params& p, const CUtensorMap* kmap, const CUtensorMap* vmap, int u,
                              int blk, int n, const PartialDst& dst, unsigned char* smem, uint64_t* bars,
                              uint32_t phase, const Grp& grp, const uint16_t* patch_k = nullptr,
                              const uint16_t* patch_v = nullptr) {
  using L = AttnTile<D, BS>;
  unsigned char* sK = smem;
  unsigned char* sV = smem + L::TILEB;
  if (grp.tid == 0) {
    int tok0;
    const int slice = kv_tile(p, u / p.kv_div, blk, &tok0);
    attn_issue<D, BS>(kmap, vmap, slice, tok0, sK, sV, &bars[0], &bars[1]);
  }
  return attn_compute<D, BS>(p, p.q + static_cast<size_t>(u) * p.G * D, blk, n, dst, sK, sV,
                             reinterpret_cast<float*>(smem + 2 * L::TILEB), &bars[0], &bars[1], phase, grp,
                             [] {}, patch_k, patch_v);
}

}  // namespace prr
