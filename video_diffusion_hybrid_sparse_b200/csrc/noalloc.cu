// noalloc.cu - vdn_hybrid_attn_fwd_static: the whole hybrid-attention call
// for callers that cannot allocate device memory.
//
// Who needs it: code that runs inside another runtime's plugin or operator
// interface, which hands over input and output tensors but no allocator and
// no way to reserve extra device memory; and latency-critical loops in which
// a cudaMalloc (it may synchronise the device and can fail under memory
// pressure) is not acceptable.  Such callers still own q, k, v, text, gates
// and out, but cannot provide the scratch workspace the regular entry point
// takes.
//
// How: the scratch lives in a file-scope static device array of
// kStaticScratchBytes (32 MiB).  Every GPU that loads this library holds that
// array until the process exits.  Host code cannot pass the array's name to a
// kernel (on the host it is only a stand-in symbol), so the first call on each
// device, with that device current, looks up its device address with
// cudaGetSymbolAddress and caches it together with the id of the CUDA context
// it was looked up in; that first call should therefore come before any
// stream capture.  The address is only valid in that context: if the context
// is replaced (cudaDeviceReset, or a primary context released and made again)
// the module is loaded afresh, the array may move, and the next call looks
// the address up again (and should again precede any capture).  The call
// then runs the regular whole-call path with cfg->workspace replaced by that
// address.  Nothing is allocated: no cudaMalloc, cudaFree or allocating
// library routine is called.
//
// All calls on a device share the one array and it keeps the last call's
// contents; the status slot at its start is cleared on every call.  Calls
// whose GPU work overlaps (two streams, or two host threads without
// ordering) race on the array: the caller must order them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "vdnattn.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct CachedAddress {
  unsigned long long ctx_id;  // id of the context the address belongs to (0: none yet)
  void* addr;
};

std::mutex g_mu;
CachedAddress g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Id of the context current on this thread; 0 when there is none yet.
bool current_ctx_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  return !ctx || get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_static_scratch in the current device's current context
// (looked up once per device, and again whenever that context has changed).
vdn_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VDN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = 0;
  if (!current_ctx_id(&id)) return VDN_ERR_CUDA;
  CachedAddress& c = g_scratch[dev];
  if (id == 0 || c.ctx_id != id || !c.addr) {
    void* p = nullptr;  // the lookup makes the device's primary context current if none was
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return VDN_ERR_CUDA;
    if (!current_ctx_id(&id) || id == 0) return VDN_ERR_CUDA;
    c.ctx_id = id;
    c.addr = p;
  }
  *out = c.addr;
  return VDN_OK;
}

bool bad_ptr(const void* p) { return !p || (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

extern "C" VDN_API size_t vdn_static_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" VDN_API vdn_status vdn_hybrid_attn_fwd_static(const void* q, const void* k, const void* v,
                                                         const void* text_k, const void* text_v,
                                                         const void* gate_s, const void* gate_l, void* out,
                                                         const vdn_cfg* cfg, void* stream) {
  if (!cfg) return VDN_ERR_INVALID_ARG;
  vdn_cfg c = *cfg;
  c.workspace = nullptr;
  c.workspace_bytes = 0;
  const vdn_status valid = vdn_validate(&c);
  if (valid != VDN_OK) return valid;
  // Problems whose scratch does not fit the static array are rejected before any CUDA call.
  if (vdn_workspace_bytes(&c) > kStaticScratchBytes) return VDN_ERR_WORKSPACE;
  // Every pointer rule of the regular call, checked here because the status
  // slot is cleared on the stream before that call runs: an error return
  // means nothing was queued and no CUDA call was made.
  for (const void* p : {q, k, v, gate_s, gate_l, static_cast<const void*>(out)})
    if (bad_ptr(p)) return p ? VDN_ERR_ALIGNMENT : VDN_ERR_INVALID_ARG;
  if (cfg->text_tokens > 0)
    for (const void* p : {text_k, text_v})
      if (bad_ptr(p)) return p ? VDN_ERR_ALIGNMENT : VDN_ERR_INVALID_ARG;
  if (cfg->output_mode == VDN_OUTPUT_SPLIT && bad_ptr(cfg->out_linear))
    return cfg->out_linear ? VDN_ERR_ALIGNMENT : VDN_ERR_INVALID_ARG;
  if ((cfg->debug_flags & VDN_EXPORT_STATES) && (!cfg->export_fwd || !cfg->export_bwd)) return VDN_ERR_INVALID_ARG;
  if (cfg->status_word && (reinterpret_cast<uintptr_t>(cfg->status_word) & 3u) != 0) return VDN_ERR_ALIGNMENT;
  if (cfg->rms_weight && (reinterpret_cast<uintptr_t>(cfg->rms_weight) & 15u) != 0) return VDN_ERR_ALIGNMENT;
  void* scratch = nullptr;
  const vdn_status s = scratch_address(&scratch);
  if (s != VDN_OK) return s;
  c.workspace = scratch;
  c.workspace_bytes = kStaticScratchBytes;
  if (cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess) return VDN_ERR_CUDA;
  return vdn_hybrid_attn_fwd(q, k, v, text_k, text_v, gate_s, gate_l, out, &c, stream);
}
