// attention.cu -- split-KV block attention for speculation and repair.
//
// One CTA computes the online-softmax statistics of ONE KV block for all G query
// heads of a GQA group (PRR abstract / method summary: speculative attention over
// the predicted blocks while selection runs, then repair of the missed blocks once
// the true set is known, merged through online-softmax statistics):
//   m = max_i s_i,  l = sum_i 2^(s_i - m),  O = sum_i 2^(s_i - m) v_i
// with s_i = scale*log2(e) * q.k_i (base-2 logits), tokens i of the block below n.
// One partial per block means a predicted block that selection drops is simply never
// merged (reuse = keep the partials of Pred n S).
//
// Data path (sm_100a): the block's K and V tiles ([bs][d] bf16, contiguous in the
// cache) arrive by 3-D TMA with the 128-byte swizzle, one mbarrier each, so the
// ldmatrix reads below are bank-conflict free.  Each staged tile is shared by all G
// heads.  Both products run on the tensor cores with mma.m16n8k16 in swap-AB form:
//   S^T[tok][h] = K[tok][:] . Q^T[:][h]     (M = 16 tokens, N = 8 heads, K = d)
//   O^T[c][h]   = V^T[c][tok] . P^T[tok][h] (M = 16 channels, N = 8 heads, K = tokens)
// The S^T accumulator fragment becomes the P^T operand fragment through movmatrix
// (an in-register 8x8 transpose).  P is split as bf16 hi + bf16 lo (two MMAs) so the
// PV product keeps ~16 mantissa bits.  Warps own disjoint token slices; their O^T
// partial sums are added in shared memory.
#include "prr_kernels.cuh"

namespace prr {

template <int D, int BS>
struct AttnSmem {
  static constexpr int TILEB = BS * D * 2;   // one K or V tile
  static constexpr int REGB = BS * 128;      // one 64-channel swizzle region of a tile
  static size_t bytes(int P, int K) {
    size_t work = 2 * static_cast<size_t>(TILEB);
    const size_t scratch = (static_cast<size_t>(merge_scratch_floats(P, K)) * 4 + 15) & ~static_cast<size_t>(15);
    if (scratch > work) work = scratch;
    return 1024 /* alignment slack */ + work + 80 * 4 /* red */ + 2 * 8 /* bars */ + 16;
  }
};

template <int D, int BS, int KIND>
__global__ void __launch_bounds__(128) attn_block_kernel(const __grid_constant__ CUtensorMap kmap,
                                                         const __grid_constant__ CUtensorMap vmap,
                                                         const __grid_constant__ Params p) {
  using L = AttnSmem<D, BS>;
  constexpr int TILEB = L::TILEB, REGB = L::REGB, NREG = D / 64;
  constexpr int MTW = BS / 64;  // 16-token m-tiles per warp (4 warps)
  constexpr int KS = D / 16;    // k-steps of QK^T == 16-channel tiles of PV
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  size_t work = 2 * static_cast<size_t>(TILEB);
  {
    const size_t scratch =
        (static_cast<size_t>(merge_scratch_floats(p.P, p.K)) * 4 + 15) & ~static_cast<size_t>(15);
    if (scratch > work) work = scratch;
  }
  unsigned char* sK = smem;
  unsigned char* sV = smem + TILEB;
  float* red = reinterpret_cast<float*>(smem + work);  // [0,32) max, [32,64) sum, [64,72) m, [72,80) l
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 80);
  int* flag = reinterpret_cast<int*>(bars + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slot = blockIdx.x, u = blockIdx.y;
  const int G = p.G;
  const int n = checked_len(p, u / p.Hkv);
  const int nb = (n + BS - 1) / BS;

  int blk = -1;
  bool active;
  unsigned add;
  if (KIND == 0) {  // speculation: slot j of Pred_t
    blk = p.pred[static_cast<size_t>(u) * p.P + slot];
    active = blk >= 0 && blk < nb;
    add = (p.mode == MODE_STEP && active) ? 1u : 0u;
  } else {  // repair: slot i of the missed set
    int nm = p.n_missed[u];
    if (nm < 0 || nm > p.K) {  // a caller-supplied count outside [0, K]
      if (tid == 0 && slot == 0) report(p.status, kDevBadMissed);
      nm = nm < 0 ? 0 : p.K;
    }
    active = slot < nm;
    if (active) blk = p.missed[static_cast<size_t>(u) * p.K + slot];
    add = active ? 1u : 0u;
    if (p.mode == MODE_STANDALONE && slot == 0) add += kMergeTarget - static_cast<unsigned>(nm);
  }
  if (!active) {
    if (add) merge_ticket<D>(p, u, add, reinterpret_cast<float*>(smem), flag);
    return;
  }

  float* pm_dst;
  float* pl_dst;
  float* pO_dst;
  size_t rstride, ostride;  // per-head strides of the destination partial arrays
  if (KIND == 0) {
    const size_t row0 = static_cast<size_t>(u) * G * p.P + slot;
    pm_dst = p.pm + row0;
    pl_dst = p.pl + row0;
    pO_dst = p.pO + row0 * D;
    rstride = p.P;
    ostride = static_cast<size_t>(p.P) * D;
  } else {
    const size_t row0 = static_cast<size_t>(u) * G * p.K + slot;
    pm_dst = p.rm + row0;
    pl_dst = p.rl + row0;
    pO_dst = p.rO + row0 * D;
    rstride = p.K;
    ostride = static_cast<size_t>(p.K) * D;
  }

  if (!(blk >= 0 && blk < nb)) {  // a missed entry out of range: contribute nothing
    if (tid == 0) report(p.status, kDevBadMissed);
    for (int e = tid; e < G * D; e += blockDim.x) pO_dst[(e / D) * ostride + (e % D)] = 0.f;
    if (tid < G) {
      pm_dst[tid * rstride] = -INFINITY;
      pl_dst[tid * rstride] = 0.f;
    }
    if (add) merge_ticket<D>(p, u, add, reinterpret_cast<float*>(smem), flag);
    return;
  }

  if (tid == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
    mbar_expect_tx(&bars[0], TILEB);
#pragma unroll
    for (int r = 0; r < NREG; ++r) tma_load_3d(sK + r * REGB, &kmap, &bars[0], r * 64, blk * BS, u);
    mbar_expect_tx(&bars[1], TILEB);
#pragma unroll
    for (int r = 0; r < NREG; ++r) tma_load_3d(sV + r * REGB, &vmap, &bars[1], r * 64, blk * BS, u);
  }

  // Q^T fragments (B operand of the score product): lane (g, t) holds head g,
  // channels 16ks + 2t, +1 and 16ks + 2t + 8, +9.  Heads >= G are zero.
  const int g = lane >> 2, t = lane & 3;
  uint32_t qf[KS][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.q + (static_cast<size_t>(u) * G + (g < G ? g : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qf[ks][0] = g < G ? __ldg(qrow + ks * 8 + t) : 0u;
      qf[ks][1] = g < G ? __ldg(qrow + ks * 8 + 4 + t) : 0u;
    }
  }
  __syncthreads();  // barrier initialisation visible to all threads

  const int nv = min(BS, n - blk * BS);  // valid tokens of this block
  if (!__syncthreads_and(mbar_wait(&bars[0], 0, p.status))) {
    if (tid == 0) mbar_wait(&bars[1], 0, p.status);  // let the V copy land (bounded)
    return;
  }

  // ---- S^T = K Q^T on the tensor cores
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
  __syncthreads();
  float m0 = red[2 * t], m1 = red[2 * t + 1];
#pragma unroll
  for (int w = 1; w < 4; ++w) {
    m0 = fmaxf(m0, red[w * 8 + 2 * t]);
    m1 = fmaxf(m1, red[w * 8 + 2 * t + 1]);
  }

  // ---- P = 2^(s - m), split hi/lo, transposed into B fragments
  float ls0 = 0.f, ls1 = 0.f;
  uint32_t bh[MTW][2], bl[MTW][2];
#pragma unroll
  for (int mi = 0; mi < MTW; ++mi) {
    const float p0 = exp2f(sc[mi][0] - m0), p1 = exp2f(sc[mi][1] - m1);
    const float p2 = exp2f(sc[mi][2] - m0), p3 = exp2f(sc[mi][3] - m1);
    ls0 += p0 + p2;
    ls1 += p1 + p3;
    const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
    const uint32_t l01 = pack_bf16x2(p0 - bf16_lo(h01), p1 - bf16_hi(h01));
    const uint32_t l23 = pack_bf16x2(p2 - bf16_lo(h23), p3 - bf16_hi(h23));
    bh[mi][0] = movmatrix_trans(h01);
    bh[mi][1] = movmatrix_trans(h23);
    bl[mi][0] = movmatrix_trans(l01);
    bl[mi][1] = movmatrix_trans(l23);
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

  if (!__syncthreads_and(mbar_wait(&bars[1], 0, p.status))) return;
  if (nv < BS) {  // tokens past the end of the sequence: zero V so 0 * V stays 0
    uint4* v4 = reinterpret_cast<uint4*>(sV);
    const int rows = BS - nv;
    for (int i = tid; i < rows * NREG * 8; i += blockDim.x) {
      const int r = nv + i / (NREG * 8), rem = i % (NREG * 8);
      v4[((rem >> 3) * REGB + r * 128) / 16 + (rem & 7)] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();
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

  // ---- O^T = V^T P^T on the tensor cores
  float oacc[KS][4];
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) oacc[dt][0] = oacc[dt][1] = oacc[dt][2] = oacc[dt][3] = 0.f;
#pragma unroll
  for (int mi = 0; mi < MTW; ++mi) {
    const int mt = warp * MTW + mi;
    const int row = mt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
    for (int dt = 0; dt < KS; ++dt) {
      const int ch = 2 * dt + ((lane >> 3) & 1);
      const uint32_t addr = sV_addr + (ch >> 3) * REGB + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
      uint32_t a[4];
      ldsm_x4_trans(addr, a);
      mma_16816(oacc[dt], a, bh[mi][0], bh[mi][1]);
      mma_16816(oacc[dt], a, bl[mi][0], bl[mi][1]);
    }
  }
  // per-warp O^T into the (dead) K tile: redO[warp][h][c ^ 4h], conflict-free
  float* redO = reinterpret_cast<float*>(sK);
#pragma unroll
  for (int dt = 0; dt < KS; ++dt) {
    const int c0 = dt * 16 + g;
    redO[(warp * 8 + 2 * t) * D + (c0 ^ (8 * t))] = oacc[dt][0];
    redO[(warp * 8 + 2 * t + 1) * D + (c0 ^ (8 * t + 4))] = oacc[dt][1];
    redO[(warp * 8 + 2 * t) * D + ((c0 + 8) ^ (8 * t))] = oacc[dt][2];
    redO[(warp * 8 + 2 * t + 1) * D + ((c0 + 8) ^ (8 * t + 4))] = oacc[dt][3];
  }
  __syncthreads();
  constexpr int C4 = D / 4;
  for (int e = tid; e < G * C4; e += blockDim.x) {
    const int h = e / C4, c4 = e % C4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float4 v = *reinterpret_cast<const float4*>(redO + (w * 8 + h) * D + ((4 * c4) ^ (4 * h)));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<float4*>(pO_dst + h * ostride)[c4] = acc;
  }
  if (tid < G) {
    pm_dst[tid * rstride] = red[64 + tid];
    pl_dst[tid * rstride] = red[72 + tid];
  }
  if (add) merge_ticket<D>(p, u, add, reinterpret_cast<float*>(smem), flag);
}

template <int D, int BS>
static cudaError_t launch_attn_t(const Params& p, const CUtensorMap& kmap, const CUtensorMap& vmap, int kind,
                                 cudaStream_t s, int priority) {
  const size_t smem = AttnSmem<D, BS>::bytes(p.P, p.K);
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
