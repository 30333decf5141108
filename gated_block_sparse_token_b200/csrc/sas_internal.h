// Internal (not exported) launch parameters shared by the libsas host API and
// its kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "sas_device.cuh"

namespace sas {

enum DecodeMode : int { kModeGate = 0, kModeAttend = 1, kModeFused = 2 };

// Byte offsets (from a 1024-byte aligned base) of the shared-memory regions
// of the cluster decode kernel.  `u_*` regions share one union: the gate
// weights slice and raw query are dead before the selection arrays are used.
struct DecodeSmem {
  int slots;   // NST stage slots of 16 KiB (gate-key chunks, then K/V tiles)
  int sslice;  // fp32 [slice_cap]  this CTA's share of the group scores
  int u_wq;    // bf16 [G][128][dpc] W_q column slice          (phase 0)
  int u_qs;    // fp32 [G][128] query staged for the gate GEMV (phase 0)
  int u_sall;  // fp32 [mg] all group scores of the (seq, head) (phase 2)
  int u_sel;   // int32 [max_sel] selected blocks             (phase 2, 3)
  int u_hist;  // uint32 [2][256] radix histograms            (phase 2)
  int u_scan;  // int32 [16] scan scratch
  int qv;      // fp32 [G][128] gate query v, then q~ in place
  int qbar;    // fp32 [128] group-mean gate query (fused mode)
  int qatt;    // fp32 [G][128] attention query (fp32 K/V only)
  int pml;     // fp32 m[4][8], l[4][8] per-warp softmax state
  int bars;    // uint64 [NST] mbarriers
  int total;   // bytes to request, including alignment slack
  int slice_cap;
};

inline DecodeSmem plan_decode_smem(int G, int mg, int cs, int nst, int max_sel, bool f32_kv) {
  DecodeSmem p{};
  int off = 0;
  auto take = [&](int bytes, int align) {
    off = (off + align - 1) / align * align;
    const int o = off;
    off += bytes;
    return o;
  };
  const int dpc = kDim / cs;
  p.slice_cap = (std::max(mg, 1) + cs - 1) / cs;
  p.slots = take(nst * kTileBytes, 1024);
  p.sslice = take(p.slice_cap * 4, 16);
  // union region
  const int ustart = (off + 15) / 16 * 16;
  const int wq_bytes = G * kDim * dpc * 2;
  const int qs_bytes = G * kDim * 4;
  p.u_wq = ustart;
  p.u_qs = ustart + wq_bytes;
  const int part_a = wq_bytes + qs_bytes;
  int o2 = ustart;
  p.u_sall = o2;
  o2 += (std::max(mg, 1) * 4 + 15) / 16 * 16;
  p.u_sel = o2;
  o2 += (max_sel * 4 + 15) / 16 * 16;
  p.u_hist = o2;
  o2 += 512 * 4;
  p.u_scan = o2;
  o2 += 16 * 4;
  off = ustart + std::max(part_a, o2 - ustart);
  p.qv = take(G * kDim * 4, 16);
  p.qbar = take(kDim * 4, 16);
  p.qatt = f32_kv ? take(G * kDim * 4, 16) : 0;
  p.pml = take(2 * kWarps * kMaxGroup * 4, 16);
  p.bars = take(nst * 8, 8);
  p.total = off + 1024;
  return p;
}

struct DecodeParams {
  int hq, hkv, G;
  int topk;     // historical blocks kept: budget/64 - 1
  int max_sel;  // budget/64
  int mg;       // rows of the gate-key cache per (seq, head)
  float rope_base, eps, attn_scale_log2, gate_scale;
  const void* q;
  const __nv_bfloat16* w_q;
  const float* gamma_q;
  const float* gate_keys;
  KvView kv;
  float* head_scores;
  float* group_scores;
  int32_t* sel_idx;
  int32_t* sel_count;
  void* out;
  uint32_t* status;
  DecodeSmem sm;
};

struct TopkParams {
  int hkv, topk, max_sel, mg;
  const float* group_scores;
  const int32_t* seq_lens;
  int32_t* sel_idx;
  int32_t* sel_count;
  uint32_t* status;
};

struct PoolParams {
  int hkv, mg, num_blocks;
  float rope_base, eps;
  KvView kv;
  const int32_t* blk_begin;
  const __nv_bfloat16* w_k;
  const float* gamma_k;
  float* gate_keys;
  float* pooled_raw;
  uint32_t* status;
};

constexpr int kPoolBlocksPerCta = 8;

// Launchers (return the cudaError_t of the launch).
cudaError_t launch_decode(int mode, bool f32_kv, bool f32_out, int cs, int nst,
                          const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                          int batch, cudaStream_t stream);
cudaError_t launch_topk(const TopkParams& p, int batch, cudaStream_t stream);
cudaError_t launch_pool(bool f32_kv, const PoolParams& p, int batch, cudaStream_t stream);
size_t topk_smem_bytes(int mg, int max_sel);
size_t pool_smem_bytes();

// One-time per-process set-up of kernel attributes.
cudaError_t prepare_kernels();

}  // namespace sas
