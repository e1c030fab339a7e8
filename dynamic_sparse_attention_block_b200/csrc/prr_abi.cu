// prr_abi.cu -- host side of the C ABI declared in include/prr.h: argument and shape
// validation, workspace layout, TMA tensor maps, kernel launches and the two-stream
// orchestration of one decode step.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "prr.h"
#include "prr_kernels.cuh"

using namespace prr;

namespace {

// Shared-memory ceilings of the kernels that keep a unit's per-block state on chip: the
// selection finisher (keys and bitmaps) and the predictor (the fp64 EMA state).
constexpr size_t kMaxSmemPerCta = 227 * 1024;

int maxnb_of(const prr_dims* d) { return static_cast<int>((d->cap_tokens + d->bs - 1) / d->bs); }

bool select_fits(const prr_dims* d) { return prr::select_smem_bytes(d->d, maxnb_of(d)) <= kMaxSmemPerCta; }

bool ema_fits(const prr_dims* d) { return prr::ema_smem_bytes(maxnb_of(d)) <= kMaxSmemPerCta; }

constexpr int kVersion = 100;  // 0.1.0

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool dims_ok(const prr_dims* d) {
  if (!d) return false;
  if (d->B < 1 || d->Hkv < 1 || d->Hq < d->Hkv || d->Hq % d->Hkv) return false;
  const int G = d->Hq / d->Hkv;
  if (G > 8) return false;
  if (d->d != 64 && d->d != 128) return false;
  if (d->bs != 64 && d->bs != 128) return false;
  if (d->cap_tokens < 1 || d->cap_tokens > (1 << 30)) return false;  // ceil(cap/bs) stays in int
  if (d->K < 1 || d->K > 128 || d->P < 0 || d->P > 128) return false;
  if (!(d->alpha >= 0.0 && d->alpha <= 1.0)) return false;
  if (!std::isfinite(d->scale)) return false;
  if (d->selector < PRR_SELECT_GROUP_SUM || d->selector > PRR_SELECT_REPRESENTATIVE) return false;
  if (d->selector == PRR_SELECT_REPRESENTATIVE && (d->n_rep < 1 || d->n_rep > 16 || !d->rep_offsets)) return false;
  if (d->n_sink < 0 || d->n_sink > (1 << 22) || d->n_local < 0 || d->n_local > (1 << 22)) return false;
  if (d->pages < 0 || (d->pages > 0) != (d->block_table != nullptr)) return false;
  if (static_cast<long long>(d->pages) * d->Hkv >= (1LL << 31)) return false;
  const long long units = static_cast<long long>(d->B) * (d->selector == PRR_SELECT_PER_HEAD ? d->Hq : d->Hkv);
  if (units > 65535) return false;  // grid.y
  return true;
}

// Selection units and the query heads each one scores with.
struct SelShape {
  size_t units;
  size_t G;
};

SelShape sel_shape(const prr_dims* d) {
  if (d->selector == PRR_SELECT_PER_HEAD) return {static_cast<size_t>(d->B) * d->Hq, 1};
  return {static_cast<size_t>(d->B) * d->Hkv, static_cast<size_t>(d->Hq / d->Hkv)};
}

WsLayout layout_for(const prr_dims* d) {
  WsLayout L = {};
  const SelShape sh = sel_shape(d);
  const size_t units = sh.units;
  const size_t G = sh.G;
  const size_t maxnb = static_cast<size_t>((d->cap_tokens + d->bs - 1) / d->bs);
  size_t off = 0;
  L.status = off;
  off = align256(off + 4);
  L.sel_cnt = off;
  off = align256(off + 4 * units);
  L.keys = off;
  off = align256(off + 4 * units * maxnb);
  L.gsum = off;
  off = align256(off + 8 * units * ((maxnb + 31) / 32));
  L.rm = off;
  off = align256(off + 4 * units * G * d->K);
  L.rl = off;
  off = align256(off + 4 * units * G * d->K);
  L.rO = off;
  off = align256(off + 4 * units * G * d->K * d->d);
  L.ctl = off;
  off = align256(off + 4 * 2 * fused_ctl_words_for(static_cast<int>(units), d->P, d->K, static_cast<int>(G)));
  L.total = off;
  return L;
}

struct DeviceInfo {
  int sms = 0;
  int prio_high = 0, prio_low = 0;
};

DeviceInfo device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!have[dev]) {
    DeviceInfo di;
    cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetStreamPriorityRange(&di.prio_low, &di.prio_high);
    if (di.sms <= 0) di.sms = 148;
    cache[dev] = di;
    have[dev] = true;
  }
  return cache[dev];
}

// Blocks per selection CTA: about one CTA per SM over the whole (units x blocks) scan,
// a multiple of 128 so every warp of the CTA streams at least one 32-block tile.
int select_chunk(int units, int maxnb, int sms) {
  const long long total = static_cast<long long>(units) * maxnb;
  long long c = (total + sms - 1) / sms;
  c = ((c + 127) / 128) * 128;
  if (c < 128) c = 128;
  if (c > 2048) c = 2048;
  return static_cast<int>(c);
}

// Kernel parameters.  `kv_units`: the call works on KV heads whatever the selector
// (summaries, appends); otherwise units follow the selector.
Params base_params(const prr_dims* d, void* ws, bool kv_units = false) {
  Params p;
  std::memset(&p, 0, sizeof p);
  p.B = d->B;
  p.Hq = d->Hq;
  p.Hkv = d->Hkv;
  p.G = d->Hq / d->Hkv;
  p.upb = d->Hkv;
  p.kv_div = 1;
  if (!kv_units && d->selector == PRR_SELECT_PER_HEAD) {
    p.kv_div = p.G;
    p.G = 1;
    p.upb = d->Hq;
  }
  p.sel_max = d->selector == PRR_SELECT_GROUP_MAX && p.G > 1;
  p.n_sink = d->n_sink;
  p.n_local = d->n_local;
  p.pages = d->pages;
  p.table = d->block_table;
  if (d->selector == PRR_SELECT_REPRESENTATIVE) {
    p.rep = d->rep_offsets;
    p.n_rep = d->n_rep;
  }
  p.d = d->d;
  p.bs = d->bs;
  p.cap = d->cap_tokens;
  p.K = d->K;
  p.P = d->P;
  p.maxnb = (d->cap_tokens + d->bs - 1) / d->bs;
  p.units = d->B * p.upb;
  p.scale_log2 = static_cast<float>(static_cast<double>(d->scale) * 1.4426950408889634074);
  p.alpha = d->alpha;
  p.chunk_blocks = select_chunk(p.units, p.maxnb, device_info().sms);
  p.nchunks = (p.maxnb + p.chunk_blocks - 1) / p.chunk_blocks;
  const WsLayout L = layout_for(d);
  unsigned char* w = static_cast<unsigned char*>(ws);
  if (w) {
    p.status = reinterpret_cast<int*>(w + L.status);
    p.sel_cnt = reinterpret_cast<unsigned*>(w + L.sel_cnt);
    p.keys = reinterpret_cast<uint32_t*>(w + L.keys);
    p.gsum = reinterpret_cast<uint2*>(w + L.gsum);
    p.rm = reinterpret_cast<float*>(w + L.rm);
    p.rl = reinterpret_cast<float*>(w + L.rl);
    p.rO = reinterpret_cast<float*>(w + L.rO);
    p.ctl = reinterpret_cast<unsigned*>(w + L.ctl);
  }
  p.ctl_words = static_cast<int>(fused_ctl_words_for(p.units, p.P, p.K, p.G));
  return p;
}

// Record a timing mark; under stream capture it must become a real event-record node.
cudaError_t record_mark(cudaEvent_t ev, cudaStream_t s) {
  if (!ev) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                                             : cudaEventRecord(ev, s);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D map over a KV cache, box {64 channels, bs tokens, 1 slice}, 128-byte swizzle, zero
// fill outside the tensor.  Contiguous caches [B*Hkv][cap][d]: a slice is one
// (sequence, KV head) pair.  Paged pools [pages*Hkv][bs][d]: a slice is one (page, KV
// head) tile.
bool make_kv_map(CUtensorMap* map, const void* base, const prr_dims* d) {
  auto fn = encode_fn();
  if (!fn) return false;
  const bool paged = d->pages > 0;
  const cuuint64_t rows = static_cast<cuuint64_t>(paged ? d->bs : d->cap_tokens);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d->d), rows,
                              static_cast<cuuint64_t>(paged ? d->pages : d->B) * d->Hkv};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d->d) * 2, static_cast<cuuint64_t>(d->d) * 2 * rows};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(d->bs), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

prr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PRR_OK : PRR_ERR_CUDA; }

}  // namespace

namespace prr {

cudaError_t allow_max_smem(const void* kernel) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

}  // namespace prr

extern "C" {

int prr_version(void) { return kVersion; }

const char* prr_status_string(prr_status s) {
  switch (s) {
    case PRR_OK: return "ok";
    case PRR_ERR_INVALID_ARG: return "invalid argument";
    case PRR_ERR_SHAPE: return "unsupported or inconsistent dimensions";
    case PRR_ERR_CAPACITY: return "workspace too small";
    case PRR_ERR_CUDA: return "CUDA runtime error";
    case PRR_ERR_DEVICE_STATUS: return "device-side error recorded in the workspace";
    case PRR_ERR_TIMEOUT: return "bounded wait timed out";
  }
  return "unknown status";
}

size_t prr_workspace_bytes(const prr_dims* dims) {
  if (!dims_ok(dims)) return 0;
  return layout_for(dims).total;
}

prr_status prr_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ws || ws_bytes == 0) return PRR_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, stream));
}

prr_status prr_get_device_status(const void* ws, int32_t* code) {
  if (!ws || !code) return PRR_ERR_INVALID_ARG;
  int32_t v = 0;
  // every call that may still write the word can run on any stream, blocking or not
  if (cudaDeviceSynchronize() != cudaSuccess) return PRR_ERR_CUDA;
  if (cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return PRR_ERR_CUDA;
  *code = v;
  return v == 0 ? PRR_OK : PRR_ERR_DEVICE_STATUS;
}

prr_status prr_append_kv(const prr_dims* dims, const uint16_t* k_new, const uint16_t* v_new,
                         int32_t* seq_lens, uint16_t* k_cache, uint16_t* v_cache, void* ws,
                         cudaStream_t stream) {
  if (!dims_ok(dims)) return PRR_ERR_SHAPE;
  if (!k_new || !v_new || !seq_lens || !k_cache || !v_cache || !ws) return PRR_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return PRR_ERR_INVALID_ARG;
  Params p = base_params(dims, ws, true);
  return cuda_status(launch_append_kv(p, k_new, v_new, k_cache, v_cache, seq_lens, stream));
}

prr_status prr_update_summaries(const prr_dims* dims, const uint16_t* k_cache,
                                const int32_t* tok_begin, const int32_t* tok_end,
                                const int32_t* seq_lens, int32_t max_range_tokens, uint16_t* summ,
                                void* ws, cudaStream_t stream) {
  if (!dims_ok(dims)) return PRR_ERR_SHAPE;
  if (!k_cache || !summ || !ws) return PRR_ERR_INVALID_ARG;
  if ((tok_begin == nullptr) != (tok_end == nullptr)) return PRR_ERR_INVALID_ARG;
  if (!tok_begin && !seq_lens) return PRR_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(summ)) return PRR_ERR_INVALID_ARG;
  if (max_range_tokens < 1 || max_range_tokens > dims->cap_tokens) return PRR_ERR_SHAPE;
  if (!tok_begin && max_range_tokens != 1) return PRR_ERR_SHAPE;
  Params p = base_params(dims, ws, true);
  p.kc = k_cache;
  p.summ = summ;
  p.seq_lens = seq_lens;
  p.tok_begin = tok_begin;
  p.tok_end = tok_end;
  return cuda_status(launch_update_summaries(p, max_range_tokens, stream, 0));
}

prr_status prr_select_topk(const prr_dims* dims, const uint16_t* q, const uint16_t* summ,
                           const int32_t* seq_lens, const int32_t* pred, int32_t* sel,
                           int32_t* missed, int32_t* n_missed, uint8_t* keep, void* ws,
                           cudaStream_t stream) {
  if (!dims_ok(dims) || !select_fits(dims)) return PRR_ERR_SHAPE;
  if (dims->selector == PRR_SELECT_REPRESENTATIVE) return PRR_ERR_SHAPE;  // needs the key cache: the step calls
  if (!q || !summ || !seq_lens || !sel || !missed || !n_missed || !ws) return PRR_ERR_INVALID_ARG;
  if (dims->P > 0 && (!pred || !keep)) return PRR_ERR_INVALID_ARG;
  if (!aligned16(summ)) return PRR_ERR_INVALID_ARG;
  Params p = base_params(dims, ws);
  p.q = q;
  p.summ = const_cast<uint16_t*>(summ);
  p.seq_lens = seq_lens;
  p.pred = pred;
  p.sel = sel;
  p.missed = missed;
  p.n_missed = n_missed;
  p.keep = keep;
  return cuda_status(launch_select(p, stream, 0));
}

prr_status prr_ema_predict(const prr_dims* dims, double* ema, const int32_t* sel,
                           const int32_t* seq_lens, int32_t* pred_next, void* ws,
                           cudaStream_t stream) {
  if (!dims_ok(dims) || !ema_fits(dims)) return PRR_ERR_SHAPE;
  if (!ema || !seq_lens || !ws || (dims->P > 0 && !pred_next)) return PRR_ERR_INVALID_ARG;
  Params p = base_params(dims, ws);
  p.ema = ema;
  p.sel = const_cast<int*>(sel);
  p.seq_lens = seq_lens;
  p.pred_next = pred_next;
  return cuda_status(launch_ema(p, stream, 0));
}

prr_status prr_speculate(const prr_dims* dims, const uint16_t* q, const uint16_t* k_cache,
                         const uint16_t* v_cache, const int32_t* seq_lens, const int32_t* pred,
                         float* part_m, float* part_l, float* part_O, void* ws,
                         cudaStream_t stream) {
  if (!dims_ok(dims)) return PRR_ERR_SHAPE;
  if (dims->P == 0) return PRR_OK;
  if (!q || !k_cache || !v_cache || !seq_lens || !pred || !part_m || !part_l || !part_O || !ws)
    return PRR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(part_O)) return PRR_ERR_INVALID_ARG;
  Params p = base_params(dims, ws);
  p.q = q;
  p.kc = k_cache;
  p.vc = v_cache;
  p.seq_lens = seq_lens;
  p.pred = pred;
  p.pm = part_m;
  p.pl = part_l;
  p.pO = part_O;
  CUtensorMap km, vm;
  if (!make_kv_map(&km, k_cache, dims) || !make_kv_map(&vm, v_cache, dims)) return PRR_ERR_CUDA;
  return cuda_status(launch_attention(p, km, vm, 0, stream, 0));
}

prr_status prr_repair_merge(const prr_dims* dims, const uint16_t* q, const uint16_t* k_cache,
                            const uint16_t* v_cache, const int32_t* seq_lens,
                            const int32_t* missed, const int32_t* n_missed, const uint8_t* keep,
                            const int32_t* pred, const float* part_m, const float* part_l,
                            const float* part_O, float* out, float* lse, void* ws,
                            cudaStream_t stream) {
  if (!dims_ok(dims)) return PRR_ERR_SHAPE;
  if (!q || !k_cache || !v_cache || !seq_lens || !missed || !n_missed || !out || !lse || !ws)
    return PRR_ERR_INVALID_ARG;
  if (dims->P > 0 && (!keep || !pred || !part_m || !part_l || !part_O)) return PRR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return PRR_ERR_INVALID_ARG;
  if (part_O && !aligned16(part_O)) return PRR_ERR_INVALID_ARG;
  Params p = base_params(dims, ws);
  p.q = q;
  p.kc = k_cache;
  p.vc = v_cache;
  p.seq_lens = seq_lens;
  p.missed = const_cast<int*>(missed);
  p.n_missed = const_cast<int*>(n_missed);
  p.keep = const_cast<uint8_t*>(keep);
  p.pred = pred;
  p.pm = const_cast<float*>(part_m);
  p.pl = const_cast<float*>(part_l);
  p.pO = const_cast<float*>(part_O);
  p.out = out;
  p.lse = lse;
  CUtensorMap km, vm;
  if (!make_kv_map(&km, k_cache, dims) || !make_kv_map(&vm, v_cache, dims)) return PRR_ERR_CUDA;
  cudaError_t e = launch_attention(p, km, vm, 1, stream, 0);
  if (e == cudaSuccess) e = launch_combine(p, stream, 0);
  return cuda_status(e);
}

}  // extern "C"

namespace {

// Shared validation of the step buffers; fills the kernel parameter block.
prr_status step_params(const prr_dims* dims, const prr_step_buffers* b, void* ws, size_t ws_bytes, Params* out) {
  if (!dims_ok(dims)) return PRR_ERR_SHAPE;
  if (!b || !ws) return PRR_ERR_INVALID_ARG;
  if (ws_bytes < layout_for(dims).total) return PRR_ERR_CAPACITY;
  if (!b->q || !b->k_cache || !b->v_cache || !b->seq_lens || !b->summ || !b->ema || !b->sel ||
      !b->missed || !b->n_missed || !b->out || !b->lse)
    return PRR_ERR_INVALID_ARG;
  if (dims->P > 0 && (!b->pred || !b->pred_next || !b->keep || !b->part_m || !b->part_l || !b->part_O))
    return PRR_ERR_INVALID_ARG;
  if (dims->P > 0 && b->pred == b->pred_next) return PRR_ERR_INVALID_ARG;
  if (!aligned16(b->k_cache) || !aligned16(b->v_cache) || !aligned16(b->summ) || !aligned16(b->out) ||
      !aligned16(b->q))
    return PRR_ERR_INVALID_ARG;
  if (b->part_O && !aligned16(b->part_O)) return PRR_ERR_INVALID_ARG;
  Params p = base_params(dims, ws);
  p.q = b->q;
  p.kc = b->k_cache;
  p.vc = b->v_cache;
  p.seq_lens = b->seq_lens;
  p.summ = b->summ;
  p.ema = b->ema;
  p.pred = b->pred;
  p.pred_next = b->pred_next;
  p.sel = b->sel;
  p.missed = b->missed;
  p.n_missed = b->n_missed;
  p.keep = b->keep;
  p.pm = b->part_m;
  p.pl = b->part_l;
  p.pO = b->part_O;
  p.out = b->out;
  p.lse = b->lse;
  p.append_summary = 1;
  if ((b->k_new == nullptr) != (b->v_new == nullptr)) return PRR_ERR_INVALID_ARG;
  if (b->k_new && (!aligned16(b->k_new) || !aligned16(b->v_new))) return PRR_ERR_INVALID_ARG;
  p.k_new = b->k_new;
  p.v_new = b->v_new;
  p.append_kv = b->k_new ? 1 : 0;
  p.trace = b->trace;
  p.stats = b->stats;
  *out = p;
  return PRR_OK;
}

}  // namespace

extern "C" {

prr_status prr_decode_step(const prr_dims* dims, const prr_step_buffers* b, void* ws,
                           size_t ws_bytes, cudaStream_t select_stream, cudaStream_t spec_stream,
                           const prr_step_events* ev) {
  if (!ev || !ev->fork || !ev->sel_done || !ev->spec_done || !ev->join) return PRR_ERR_INVALID_ARG;
  Params p;
  const prr_status st = step_params(dims, b, ws, ws_bytes, &p);
  if (st != PRR_OK) return st;
  if (!select_fits(dims) || !ema_fits(dims)) return PRR_ERR_SHAPE;
  CUtensorMap km, vm;
  if (!make_kv_map(&km, b->k_cache, dims) || !make_kv_map(&vm, b->v_cache, dims)) return PRR_ERR_CUDA;
  const DeviceInfo di = device_info();
  const int hi = di.prio_high, lo = di.prio_low;

#define PRR_TRY(x)                               \
  do {                                           \
    if ((x) != cudaSuccess) return PRR_ERR_CUDA; \
  } while (0)
  cudaStream_t A = select_stream, B = spec_stream;
  if (p.append_kv) {  // the step's token first: the kernels below then see it in the cache
    PRR_TRY(launch_append_kv(p, p.k_new, p.v_new, const_cast<uint16_t*>(p.kc), const_cast<uint16_t*>(p.vc),
                             const_cast<int*>(p.seq_lens), A));
    p.append_kv = 0;
  }
  PRR_TRY(cudaEventRecord(ev->fork, A));
  PRR_TRY(cudaStreamWaitEvent(B, ev->fork, 0));
  // spec stream: speculation over Pred_t, independent of selection
  PRR_TRY(record_mark(ev->t_spec_begin, B));
  PRR_TRY(launch_attention(p, km, vm, 0, B, lo));
  PRR_TRY(record_mark(ev->t_spec_end, B));
  PRR_TRY(cudaEventRecord(ev->spec_done, B));
  // critical path: tail summary + scoring + top-K, then repair of the missed blocks
  PRR_TRY(record_mark(ev->t_begin, A));
  PRR_TRY(launch_select(p, A, hi));
  PRR_TRY(record_mark(ev->t_select_end, A));
  PRR_TRY(cudaEventRecord(ev->sel_done, A));
  PRR_TRY(launch_attention(p, km, vm, 1, A, hi));
  PRR_TRY(record_mark(ev->t_repair_end, A));
  // spec stream: the predictor for step t+1 needs S_t only; it overlaps repair/merge
  PRR_TRY(cudaStreamWaitEvent(B, ev->sel_done, 0));
  PRR_TRY(record_mark(ev->t_ema_begin, B));
  PRR_TRY(launch_ema(p, B, lo));  // the state advances even with no speculation budget
  PRR_TRY(record_mark(ev->t_ema_end, B));
  PRR_TRY(cudaEventRecord(ev->join, B));
  // merge once speculation and repair are both done
  PRR_TRY(cudaStreamWaitEvent(A, ev->spec_done, 0));
  PRR_TRY(record_mark(ev->t_combine_begin, A));
  PRR_TRY(launch_combine(p, A, hi));
  PRR_TRY(record_mark(ev->t_combine_end, A));
  PRR_TRY(cudaStreamWaitEvent(A, ev->join, 0));
#undef PRR_TRY
  return PRR_OK;
}

prr_status prr_decode_step_fused(const prr_dims* dims, const prr_step_buffers* b, void* ws, size_t ws_bytes,
                                 int32_t step_parity, cudaStream_t stream) {
  if (step_parity != 0 && step_parity != 1) return PRR_ERR_INVALID_ARG;
  Params p;
  const prr_status st = step_params(dims, b, ws, ws_bytes, &p);
  if (st != PRR_OK) return st;
  const DeviceInfo di = device_info();
  if (fused_smem_bytes(p, di.sms) > 227 * 1024) return PRR_ERR_SHAPE;
  p.parity = step_parity;
  CUtensorMap km, vm;
  if (!make_kv_map(&km, b->k_cache, dims) || !make_kv_map(&vm, b->v_cache, dims)) return PRR_ERR_CUDA;
  return cuda_status(launch_fused(p, km, vm, stream, di.prio_high, di.sms, nullptr));
}

}  // extern "C"
