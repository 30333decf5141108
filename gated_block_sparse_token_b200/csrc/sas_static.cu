// sas_decode_step_static: the fused decode step for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where cudaMalloc (or any allocator) is off
// limits -- a serving loop that must not allocate once it is warmed up
// (cudaMalloc can synchronise the device and fragments a caching pool), a
// plugin inside a host framework that owns all GPU memory, a plain C caller
// with no allocator of its own.  Such callers cannot hand sas_decode_step the
// small workspace it keeps its device status word in.  This entry point keeps
// that scratch in a file-scope __device__ array instead; the caller passes
// inputs and outputs only.
//
// Limits, stated once: the array is kStaticScratchBytes (256 bytes), enough
// for the fused step's scratch at any problem size (its only scratch is the
// status word); a build that needs more (the phase-trace build) is refused
// with SAS_ERR_WORKSPACE.  Every GPU that loads the library holds the array
// until the process exits.  All calls share it: the status word is cleared at
// the start of every call, and calls that overlap on the GPU (concurrent
// streams) race on it.
#include <mutex>

#include "sas.h"
#include "sas_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Driver calls that identify the current context (looked up through the
// runtime, like the library's other driver entry points).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

std::mutex g_scratch_mu;
std::once_flag g_ctx_fn_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
// per device: the context the address was looked up in, and the address
unsigned long long g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_addr[kMaxDevices] = {};

void load_ctx_fns() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  fn = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(fn);
  (void)cudaGetLastError();
}

// Device address of g_decode_scratch in the current device's context.  The
// host-side symbol is only a stand-in, never a device address.  The address
// is looked up once per device and looked up again when the device's context
// has changed since (after cudaDeviceReset the module is loaded anew and the
// array may sit elsewhere).
sas_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SAS_ERR_UNSUPPORTED;
  std::call_once(g_ctx_fn_once, load_ctx_fns);
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) return SAS_ERR_CUDA;
  // id of the current context; 0 while none is bound yet (first call)
  auto current_ctx_id = [](unsigned long long* id) -> bool {
    CUcontext ctx = nullptr;
    *id = 0;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return false;
    return ctx == nullptr || g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
  };
  unsigned long long ctx_id = 0;
  if (!current_ctx_id(&ctx_id)) return SAS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (ctx_id == 0 || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != ctx_id) {
    void* p = nullptr;
    // binds (or creates) the device's primary context if none is current
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return SAS_ERR_CUDA;
    }
    if (!current_ctx_id(&ctx_id) || ctx_id == 0) return SAS_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx_id;
  }
  *out = g_scratch_addr[dev];
  return SAS_OK;
}

}  // namespace

extern "C" sas_status sas_decode_step_static(const sas_config* cfg, const void* q,
                                             const sas_kv* kv, const void* w_q,
                                             const float* gamma_q, const void* w_k,
                                             const float* gamma_k, void* gate_keys,
                                             int32_t max_gate_blocks, void* out,
                                             int32_t* sel_idx, int32_t* sel_count,
                                             float* group_scores, uint32_t* status_out,
                                             sas_stream_t stream) {
  if (cfg == nullptr || kv == nullptr) return SAS_ERR_INVALID_ARG;
  // a decode step needs the workspace of no batch and no prefill length
  if (sas_workspace_bytes(cfg, 0, 0) > kStaticScratchBytes) return SAS_ERR_WORKSPACE;
  if (status_out != nullptr && (reinterpret_cast<uintptr_t>(status_out) % 4) != 0)
    return SAS_ERR_INVALID_ARG;
  // every host check of the step first (any 256-aligned stand-in passes the
  // workspace check), so that a refused call enqueues nothing at all
  bool launch = false;
  sas_status st = sas::check_decode_step_args(
      cfg, q, kv, w_q, gamma_q, w_k, gamma_k, gate_keys, max_gate_blocks, out, sel_idx, sel_count,
      group_scores, reinterpret_cast<const void*>(static_cast<uintptr_t>(256)), kStaticScratchBytes,
      &launch);
  if (st != SAS_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_for_current_device(&scratch)) != SAS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the array keeps the last call's contents: the status word starts at zero
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s) != cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  if (launch) {
    st = sas_decode_step(cfg, q, kv, w_q, gamma_q, w_k, gamma_k, gate_keys, max_gate_blocks, out,
                         sel_idx, sel_count, group_scores, scratch, kStaticScratchBytes, stream);
    if (st != SAS_OK) return st;
  }
  if (status_out != nullptr &&
      cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  return SAS_OK;
}
