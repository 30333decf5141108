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

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, looked up once per
// device (the host-side symbol is only a stand-in, never a device address).
sas_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SAS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return SAS_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
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
  if (sas_workspace_bytes(cfg, kv->batch, 0) > kStaticScratchBytes) return SAS_ERR_WORKSPACE;
  if (status_out != nullptr && (reinterpret_cast<uintptr_t>(status_out) % 4) != 0)
    return SAS_ERR_INVALID_ARG;
  void* scratch = nullptr;
  sas_status st = scratch_for_current_device(&scratch);
  if (st != SAS_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the array keeps the last call's contents: the status word starts at zero
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s) != cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  st = sas_decode_step(cfg, q, kv, w_q, gamma_q, w_k, gamma_k, gate_keys, max_gate_blocks, out,
                       sel_idx, sel_count, group_scores, scratch, kStaticScratchBytes, stream);
  if (st != SAS_OK) return st;
  if (status_out != nullptr &&
      cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  return SAS_OK;
}
