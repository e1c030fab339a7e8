// select_static.cu -- prr_select_topk for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory for a workspace: code that runs
// inside another framework's memory pool without access to its allocator, a plugin
// whose host process forbids cudaMalloc after start-up (allocation can synchronise the
// device and break latency guarantees or an ongoing stream capture), or a tiny
// embedded deployment that sizes every buffer at build time.  For them this entry
// point keeps the selection kernel's scratch (status word, chunk tickets, one 32-bit
// score key per block) in a fixed array inside the library itself.  The caller still
// passes all inputs and outputs.
//
// The array is a file-scope __device__ variable, so every GPU that loads the library
// holds it (PRR_SELECT_STATIC_SCRATCH_BYTES, about 4.3 MB) until the process exits.
// Host code cannot use the array's name as a device pointer: the device address is
// looked up with cudaGetSymbolAddress on the first call made in a CUDA context (with
// that context current) and then passed to the kernel like any workspace pointer.  The
// address is cached per context, keyed by the context's process-unique id, so a
// context created later on the same device (after cudaDeviceReset, say) looks the
// address up again instead of writing through one that died with the old module.
#include <cudaTypedefs.h>

#include <cstring>
#include <map>
#include <mutex>

#include "prr.h"
#include "prr_kernels.cuh"

namespace {

// Layout: status word (256 B), one chunk ticket per unit (65536 units at most, the
// shape rules' limit), one score key per block of every unit.
constexpr size_t kHeaderBytes = 256;
constexpr size_t kTicketBytes = static_cast<size_t>(65536) * 4;
constexpr size_t kKeyBytes = static_cast<size_t>(PRR_SELECT_STATIC_MAX_BLOCKS) * 4;
constexpr size_t kScratchBytes = kHeaderBytes + kTicketBytes + kKeyBytes;
static_assert(kScratchBytes == PRR_SELECT_STATIC_SCRATCH_BYTES, "header and library disagree");

__device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

std::mutex g_mu;
std::map<unsigned long long, void*> g_addr;  // context id -> device address of the array

// The driver's cuCtxGetCurrent and cuCtxGetId through the runtime's entry-point query
// (the library does not link libcuda directly).
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 current = nullptr;
  PFN_cuCtxGetId_v12000 id = nullptr;
};

CtxFns ctx_fns() {
  static const CtxFns fns = [] {
    CtxFns f;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.id = reinterpret_cast<PFN_cuCtxGetId_v12000>(ptr);
    return f;
  }();
  return fns;
}

// Device address of the scratch array in the current context (looked up once per context).
cudaError_t scratch_address(void** out) {
  const CtxFns f = ctx_fns();
  if (!f.current || !f.id) return cudaErrorDeviceUninitialized;
  CUcontext ctx = nullptr;
  void* fresh = nullptr;
  if (f.current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (!ctx) {  // no context yet on this thread: the lookup itself brings up the device's
    cudaError_t e = cudaGetSymbolAddress(&fresh, g_select_scratch);  // primary context
    if (e != cudaSuccess) return e;
    if (f.current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
  }
  unsigned long long id = 0;
  if (f.id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> g(g_mu);
  auto it = g_addr.find(id);
  if (it == g_addr.end()) {
    if (!fresh) {
      cudaError_t e = cudaGetSymbolAddress(&fresh, g_select_scratch);
      if (e != cudaSuccess) return e;
    }
    it = g_addr.emplace(id, fresh).first;
  }
  *out = it->second;
  return cudaSuccess;
}

}  // namespace

extern "C" prr_status prr_select_topk_static(const prr_dims* dims, const uint16_t* q, const uint16_t* summ,
                                             const int32_t* seq_lens, const int32_t* pred, int32_t* sel,
                                             int32_t* missed, int32_t* n_missed, uint8_t* keep,
                                             int32_t* status, cudaStream_t stream) {
  if (prr_workspace_bytes(dims) == 0) return PRR_ERR_SHAPE;  // same shape rules as the other calls
  if (dims->selector == PRR_SELECT_REPRESENTATIVE) return PRR_ERR_SHAPE;  // summary selectors only
  if (prr::select_smem_bytes(dims->d, static_cast<int>((dims->cap_tokens + dims->bs - 1) / dims->bs)) >
      227 * 1024)
    return PRR_ERR_SHAPE;  // the finisher's on-chip scratch, as prr_select_topk
  if (!q || !summ || !seq_lens || !sel || !missed || !n_missed) return PRR_ERR_INVALID_ARG;
  if (dims->P > 0 && (!pred || !keep)) return PRR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(summ) & 15u) != 0) return PRR_ERR_INVALID_ARG;

  const bool per_head = dims->selector == PRR_SELECT_PER_HEAD;
  const int upb = per_head ? dims->Hq : dims->Hkv;  // selection units per sequence
  const int units = dims->B * upb;
  const int maxnb = (dims->cap_tokens + dims->bs - 1) / dims->bs;
  if (static_cast<long long>(units) * maxnb > PRR_SELECT_STATIC_MAX_BLOCKS) return PRR_ERR_CAPACITY;

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return PRR_ERR_CUDA;
  unsigned char* s = static_cast<unsigned char*>(base);
  // the status word and the tickets must start at zero; the keys are overwritten
  if (cudaMemsetAsync(s, 0, sizeof(int32_t), stream) != cudaSuccess) return PRR_ERR_CUDA;
  if (cudaMemsetAsync(s + kHeaderBytes, 0, static_cast<size_t>(units) * 4, stream) != cudaSuccess)
    return PRR_ERR_CUDA;

  prr::Params p;
  std::memset(&p, 0, sizeof p);
  p.B = dims->B;
  p.Hq = dims->Hq;
  p.Hkv = dims->Hkv;
  p.G = per_head ? 1 : dims->Hq / dims->Hkv;
  p.upb = upb;
  p.kv_div = per_head ? dims->Hq / dims->Hkv : 1;
  p.sel_max = dims->selector == PRR_SELECT_GROUP_MAX && p.G > 1;
  p.n_sink = dims->n_sink;
  p.n_local = dims->n_local;
  p.pages = dims->pages;
  p.table = dims->block_table;
  p.d = dims->d;
  p.bs = dims->bs;
  p.cap = dims->cap_tokens;
  p.K = dims->K;
  p.P = dims->P;
  p.maxnb = maxnb;
  p.units = units;
  p.chunk_blocks = 256;
  p.nchunks = (maxnb + p.chunk_blocks - 1) / p.chunk_blocks;
  p.q = q;
  p.summ = const_cast<uint16_t*>(summ);
  p.seq_lens = seq_lens;
  p.pred = pred;
  p.sel = sel;
  p.missed = missed;
  p.n_missed = n_missed;
  p.keep = keep;
  p.status = reinterpret_cast<int*>(s);
  p.sel_cnt = reinterpret_cast<unsigned*>(s + kHeaderBytes);
  p.keys = reinterpret_cast<uint32_t*>(s + kHeaderBytes + kTicketBytes);
  if (prr::launch_select(p, stream, 0) != cudaSuccess) return PRR_ERR_CUDA;
  if (status && cudaMemcpyAsync(status, s, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return PRR_ERR_CUDA;
  return PRR_OK;
}
