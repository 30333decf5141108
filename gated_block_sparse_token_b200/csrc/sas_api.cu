// libsas C ABI: host-side validation, TMA tensor-map encoding and kernel
// dispatch.  Every entry point validates on the host, enqueues on the given
// stream and returns; nothing here allocates or synchronises except
// sas_get_device_status.
#include <math.h>
#include <string.h>

#include <mutex>

#include "sas.h"
#include "sas_internal.h"

namespace sas {
cudaError_t prepare_decode_kernels();
cudaError_t prepare_pool_kernels();
cudaError_t prepare_prefill_kernels();
cudaError_t prepare_backward_kernels();
cudaError_t prepare_prefill_backward_kernels();
}

namespace {

using sas::kDim;

constexpr int32_t kAbiVersion = 10;
constexpr size_t kStatusBytes = 256;  // status word + padding
constexpr int kMaxBudget = 16384;
constexpr int kMaxGateBlocks = 16384;
constexpr int kClusterSize = 8;
constexpr int kStages = 2;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::once_flag g_once;
cudaError_t g_prep_err = cudaSuccess;
EncodeTiledFn g_encode = nullptr;

cudaError_t prepare() {
  std::call_once(g_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                                     cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) {
      g_prep_err = (e != cudaSuccess) ? e : cudaErrorSymbolNotFound;
      return;
    }
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    g_prep_err = sas::prepare_decode_kernels();
    if (g_prep_err == cudaSuccess) g_prep_err = sas::prepare_pool_kernels();
    if (g_prep_err == cudaSuccess) g_prep_err = sas::prepare_prefill_kernels();
    if (g_prep_err == cudaSuccess) g_prep_err = sas::prepare_backward_kernels();
    if (g_prep_err == cudaSuccess) g_prep_err = sas::prepare_prefill_backward_kernels();
  });
  return g_prep_err;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool finite_pos(float x) { return isfinite(x) && x > 0.f; }

sas_status check_config(const sas_config* c) {
  if (c == nullptr) return SAS_ERR_INVALID_ARG;
  if (c->block_size != 64 || c->gate_hidden != 128) return SAS_ERR_INVALID_ARG;
  if (c->head_dim != 128) return SAS_ERR_UNSUPPORTED;
  if (c->num_q_heads < 1 || c->num_kv_heads < 1) return SAS_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads != 0) return SAS_ERR_INVALID_ARG;
  if (c->num_q_heads / c->num_kv_heads > sas::kMaxGroup) return SAS_ERR_UNSUPPORTED;
  if (c->token_budget < 64 || c->token_budget % 64 != 0) return SAS_ERR_INVALID_ARG;
  if (c->token_budget > kMaxBudget) return SAS_ERR_UNSUPPORTED;
  if (!finite_pos(c->rope_base) || !finite_pos(c->attn_scale) || !finite_pos(c->gate_scale))
    return SAS_ERR_INVALID_ARG;
  if (!isfinite(c->norm_eps) || c->norm_eps < 0.f) return SAS_ERR_INVALID_ARG;
  if (c->kv_dtype != SAS_DTYPE_BF16 && c->kv_dtype != SAS_DTYPE_F32) return SAS_ERR_INVALID_ARG;
  if (c->out_dtype != SAS_DTYPE_BF16 && c->out_dtype != SAS_DTYPE_F32) return SAS_ERR_INVALID_ARG;
  if (c->gate_mode != SAS_GATE_SELECT_ONLY && c->gate_mode != SAS_GATE_LOGSIGMOID_BIAS)
    return SAS_ERR_INVALID_ARG;
  if (c->gate_keys_bf16 != 0 && c->gate_keys_bf16 != 1) return SAS_ERR_INVALID_ARG;
  if (c->static_weights != 0 && c->static_weights != 1) return SAS_ERR_INVALID_ARG;
  return SAS_OK;
}

sas_status check_ws(const sas_config* cfg, void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned(ws, 16)) return SAS_ERR_WORKSPACE;
  if (ws_bytes < sas_workspace_bytes(cfg, 0, 0)) return SAS_ERR_WORKSPACE;
  return SAS_OK;
}

sas_status check_kv(const sas_config* cfg, const sas_kv* kv) {
  if (kv == nullptr) return SAS_ERR_INVALID_ARG;
  if (kv->batch < 0) return SAS_ERR_INVALID_ARG;
  if (kv->batch == 0) return SAS_OK;
  if (kv->k == nullptr || kv->v == nullptr || kv->seq_lens == nullptr) return SAS_ERR_INVALID_ARG;
  if (!aligned(kv->k, 16) || !aligned(kv->v, 16) || !aligned(kv->seq_lens, 4))
    return SAS_ERR_INVALID_ARG;
  long long rows;
  if (kv->block_table != nullptr) {
    if (!aligned(kv->block_table, 4) || kv->num_pages < 1 || kv->max_blocks_per_seq < 1)
      return SAS_ERR_INVALID_ARG;
    rows = static_cast<long long>(kv->num_pages) * cfg->num_kv_heads * 64;
  } else {
    if (kv->capacity < 64 || kv->capacity % 64 != 0) return SAS_ERR_INVALID_ARG;
    rows = static_cast<long long>(kv->batch) * cfg->num_kv_heads * kv->capacity;
  }
  if (rows > 0x7fffffffLL) return SAS_ERR_UNSUPPORTED;  // TMA row coordinate is int32
  return SAS_OK;
}

sas::KvView make_view(const sas_config* cfg, const sas_kv* kv) {
  sas::KvView v{};
  v.k = kv->k;
  v.v = kv->v;
  v.block_table = kv->block_table;
  v.seq_lens = kv->seq_lens;
  v.hkv = cfg->num_kv_heads;
  v.capacity = kv->capacity;
  v.num_pages = kv->num_pages;
  v.max_blocks_per_seq = kv->max_blocks_per_seq;
  v.token_budgets = kv->token_budgets;
  v.max_budget = cfg->token_budget;
  return v;
}

// 2-D view [rows][128] of a bf16 K or V cache, 64x64 boxes, 128-byte swizzle.
bool encode_kv_map(CUtensorMap* m, const void* ptr, long long rows) {
  memset(m, 0, sizeof(*m));
  if (g_encode == nullptr) return false;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(kDim * 2)};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim,
                              gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D view [Hq*128][128] of bf16 W_q; one box = the 128 rows of one query
// head restricted to the 128/CS columns a cluster CTA projects.
bool encode_wq_map(CUtensorMap* m, const void* w_q, int hq) {
  memset(m, 0, sizeof(*m));
  if (g_encode == nullptr) return false;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(hq) * kDim};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(kDim * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kDim / kClusterSize), static_cast<cuuint32_t>(kDim)};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w_q), gdim,
                              gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D view [Hkv*384][128] of bf16 W_k; one box = 128 rows x the 128/CS
// columns a cluster CTA projects.
bool encode_wk_map(CUtensorMap* m, const void* w_k, int hkv) {
  memset(m, 0, sizeof(*m));
  if (g_encode == nullptr) return false;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(hkv) * sas::kPool};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(kDim * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kDim / kClusterSize), 128};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w_k), gdim,
                              gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

long long kv_rows(const sas_config* cfg, const sas_kv* kv) {
  return kv->block_table != nullptr
             ? static_cast<long long>(kv->num_pages) * cfg->num_kv_heads * 64
             : static_cast<long long>(kv->batch) * cfg->num_kv_heads * kv->capacity;
}

void fill_common(sas::DecodeParams& p, const sas_config* cfg, int mg) {
  p.hq = cfg->num_q_heads;
  p.hkv = cfg->num_kv_heads;
  p.G = cfg->num_q_heads / cfg->num_kv_heads;
  p.max_sel = cfg->token_budget / 64;
  p.topk = p.max_sel - 1;
  p.mg = mg;
  p.rope_base = cfg->rope_base;
  p.eps = cfg->norm_eps;
  p.attn_scale_log2 = cfg->attn_scale * 1.4426950408889634f;
  p.gate_scale = cfg->gate_scale;
  p.gated = cfg->gate_mode == SAS_GATE_LOGSIGMOID_BIAS ? 1 : 0;
  p.gk16 = cfg->gate_keys_bf16;
  p.static_weights = cfg->static_weights;
  p.sm = sas::plan_decode_smem(p.G, mg, kClusterSize, kStages, p.max_sel,
                               cfg->kv_dtype == SAS_DTYPE_F32, p.gated != 0);
  sas::fill_rope_table(p.rope, cfg->rope_base);
}

bool plan_ok(const sas::DecodeParams& p) {
  return p.sm.total <= 227 * 1024 && sas::decode_smem_aligned(p.sm, p.G, kDim / kClusterSize);
}

unsigned long long* trace_region(void* ws) {
#ifdef SAS_PHASE_TRACE
  return reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(ws) + kStatusBytes);
#else
  (void)ws;
  return nullptr;
#endif
}

size_t ws_header_bytes() {
#ifdef SAS_PHASE_TRACE
  return kStatusBytes + static_cast<size_t>(sas::kTraceCtas) * sas::kTraceSlots * 8;
#else
  return kStatusBytes;
#endif
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// gate queries, block lists, list lengths
size_t prefill_scratch_bytes(size_t batch, int hq, int hkv, size_t nblk, int max_sel) {
  return up256(batch * hq * nblk * kDim * 4) + up256(batch * hkv * nblk * max_sel * 4) +
         up256(batch * hkv * nblk * 4);
}

sas_status launch_result(cudaError_t e) {
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  return SAS_OK;
}

}  // namespace

extern "C" {

int32_t sas_abi_version(void) { return kAbiVersion; }

const char* sas_status_string(sas_status s) {
  switch (s) {
    case SAS_OK: return "ok";
    case SAS_ERR_INVALID_ARG: return "invalid argument";
    case SAS_ERR_UNSUPPORTED: return "unsupported configuration";
    case SAS_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SAS_ERR_CUDA: return "CUDA runtime error";
    case SAS_ERR_DEVICE_BOUNDS: return "device-detected out-of-range length, page or block index";
    case SAS_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

// Workspace layout: status header, then (batch > 0) the gate backward's
// per-pair terms, then (batch > 0 and max_seq_len > 0) the prefill scratch
// and the prefill gate backward's terms.
size_t bwd_scratch_bytes(const sas_config* cfg, int32_t batch) {
  if (cfg == nullptr || batch <= 0 || cfg->num_kv_heads <= 0 || cfg->num_q_heads <= 0 || cfg->token_budget < 64)
    return 0;
  return sas::gate_bwd_scratch_bytes(static_cast<size_t>(batch), cfg->num_q_heads, cfg->num_kv_heads,
                                     cfg->token_budget / 64);
}

size_t sas_workspace_bytes(const sas_config* cfg, int32_t batch, int32_t max_seq_len) {
  size_t bytes = ws_header_bytes() + bwd_scratch_bytes(cfg, batch);
  if (cfg != nullptr && batch > 0 && max_seq_len > 0 && cfg->num_kv_heads > 0 &&
      cfg->num_q_heads > 0 && cfg->token_budget >= 64) {
    // prefill scratch: gate queries, block lists and their lengths
    const size_t nblk = static_cast<size_t>((max_seq_len + 63) / 64);
    bytes += prefill_scratch_bytes(batch, cfg->num_q_heads, cfg->num_kv_heads, nblk,
                                   cfg->token_budget / 64);
    // the prefill gate backward's per-(sequence, head, block) terms
    bytes += sas::prefill_bwd_scratch_bytes(static_cast<size_t>(batch), cfg->num_q_heads, cfg->num_kv_heads,
                                            nblk, cfg->token_budget / 64);
  }
  return bytes;
}

sas_status sas_reset_device_status(void* ws, sas_stream_t stream) {
  if (ws == nullptr || !aligned(ws, 16)) return SAS_ERR_WORKSPACE;
  return launch_result(cudaMemsetAsync(ws, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_get_device_status(const void* ws, sas_stream_t stream, sas_status* out) {
  if (ws == nullptr || out == nullptr || !aligned(ws, 16)) return SAS_ERR_INVALID_ARG;
  uint32_t word = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return SAS_ERR_CUDA;
  }
  if (word & sas::kStatusBounds)
    *out = SAS_ERR_DEVICE_BOUNDS;
  else if (word & sas::kStatusTimeout)
    *out = SAS_ERR_TIMEOUT;
  else
    *out = SAS_OK;
  return SAS_OK;
}

sas_status sas_pool_keys(const sas_config* cfg, const sas_kv* kv, const int32_t* blk_begin,
                         int32_t num_blocks, const void* w_k, const float* gamma_k,
                         void* gate_keys, int32_t max_gate_blocks, float* pooled_raw, void* ws,
                         size_t ws_bytes, sas_stream_t stream) {
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if ((st = check_kv(cfg, kv)) != SAS_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != SAS_OK) return st;
  if (num_blocks < 0 || max_gate_blocks < 1 || max_gate_blocks > kMaxGateBlocks)
    return SAS_ERR_INVALID_ARG;
  if (kv->batch == 0 || num_blocks == 0) return SAS_OK;
  if (w_k == nullptr || gamma_k == nullptr || gate_keys == nullptr) return SAS_ERR_INVALID_ARG;
  if (!aligned(w_k, 16) || !aligned(gamma_k, 4) || !aligned(gate_keys, 16) ||
      (pooled_raw != nullptr && !aligned(pooled_raw, 4)) ||
      (blk_begin != nullptr && !aligned(blk_begin, 4)))
    return SAS_ERR_INVALID_ARG;
  if (kv->batch > 65535) return SAS_ERR_UNSUPPORTED;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  sas::PoolParams p{};
  p.hkv = cfg->num_kv_heads;
  p.mg = max_gate_blocks;
  p.num_blocks = num_blocks;
  p.rope_base = cfg->rope_base;
  p.eps = cfg->norm_eps;
  sas::fill_rope_table(p.rope, cfg->rope_base);
  p.kv = make_view(cfg, kv);
  p.blk_begin = blk_begin;
  p.w_k = static_cast<const __nv_bfloat16*>(w_k);
  p.gamma_k = gamma_k;
  p.gate_keys = gate_keys;
  p.gk16 = cfg->gate_keys_bf16;
  p.pooled_raw = pooled_raw;
  p.status = static_cast<uint32_t*>(ws);
  if (cfg->kv_dtype == SAS_DTYPE_F32)
    return launch_result(sas::launch_pool(true, p, kv->batch, reinterpret_cast<cudaStream_t>(stream)));
  CUtensorMap tmwk;
  if (!encode_kv_map(&tmwk, w_k, static_cast<long long>(cfg->num_kv_heads) * sas::kPool)) return SAS_ERR_CUDA;
  return launch_result(sas::launch_pool_project(p, tmwk, kv->batch, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_gate_scores(const sas_config* cfg, const void* q, const int32_t* seq_lens,
                           int32_t batch, const void* w_q, const float* gamma_q,
                           const void* gate_keys, int32_t max_gate_blocks, float* head_scores,
                           float* group_scores, void* ws, size_t ws_bytes, sas_stream_t stream) {
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != SAS_OK) return st;
  if (batch < 0 || max_gate_blocks < 1 || max_gate_blocks > kMaxGateBlocks) return SAS_ERR_INVALID_ARG;
  if (batch == 0) return SAS_OK;
  if (q == nullptr || seq_lens == nullptr || w_q == nullptr || gamma_q == nullptr ||
      gate_keys == nullptr || group_scores == nullptr)
    return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(seq_lens, 4) || !aligned(w_q, 16) || !aligned(gamma_q, 16) ||
      !aligned(gate_keys, 16) || !aligned(group_scores, 4) ||
      (head_scores != nullptr && !aligned(head_scores, 4)))
    return SAS_ERR_INVALID_ARG;
  if (static_cast<long long>(batch) * cfg->num_kv_heads > 65535) return SAS_ERR_UNSUPPORTED;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  sas::DecodeParams p{};
  fill_common(p, cfg, max_gate_blocks);
  if (!plan_ok(p)) return SAS_ERR_UNSUPPORTED;
  p.q = q;
  p.w_q = static_cast<const __nv_bfloat16*>(w_q);
  p.gamma_q = gamma_q;
  p.gate_keys = gate_keys;
  p.kv.seq_lens = seq_lens;
  p.kv.hkv = cfg->num_kv_heads;
  p.head_scores = head_scores;
  p.group_scores = group_scores;
  p.status = static_cast<uint32_t*>(ws);
  p.trace = trace_region(ws);
  CUtensorMap dummy, tmw;
  memset(&dummy, 0, sizeof(dummy));
  if (!encode_wq_map(&tmw, w_q, cfg->num_q_heads)) return SAS_ERR_CUDA;
  return launch_result(sas::launch_decode(sas::kModeGate, cfg->kv_dtype == SAS_DTYPE_F32, false,
                                          kClusterSize, kStages, p, dummy, dummy, tmw, dummy, batch,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_topk_blocks(const sas_config* cfg, const float* group_scores,
                           const int32_t* seq_lens, const int32_t* token_budgets, int32_t batch,
                           int32_t max_gate_blocks, int32_t* sel_idx, int32_t* sel_count, void* ws,
                           size_t ws_bytes, sas_stream_t stream) {
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != SAS_OK) return st;
  if (batch < 0 || max_gate_blocks < 1 || max_gate_blocks > kMaxGateBlocks) return SAS_ERR_INVALID_ARG;
  if (batch == 0) return SAS_OK;
  if (group_scores == nullptr || seq_lens == nullptr || sel_idx == nullptr || sel_count == nullptr)
    return SAS_ERR_INVALID_ARG;
  if (!aligned(group_scores, 4) || !aligned(seq_lens, 4) || !aligned(sel_idx, 4) ||
      !aligned(sel_count, 4) || !aligned(token_budgets, 4))
    return SAS_ERR_INVALID_ARG;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  sas::TopkParams p{};
  p.hkv = cfg->num_kv_heads;
  p.max_sel = cfg->token_budget / 64;
  p.topk = p.max_sel - 1;
  p.mg = max_gate_blocks;
  p.group_scores = group_scores;
  p.seq_lens = seq_lens;
  p.token_budgets = token_budgets;
  p.sel_idx = sel_idx;
  p.sel_count = sel_count;
  p.status = static_cast<uint32_t*>(ws);
  return launch_result(sas::launch_topk(p, batch, reinterpret_cast<cudaStream_t>(stream)));
}

// Host checks of a decode-attention call (everything attention_call checks
// before it enqueues anything).  *launch is false when there is nothing to do.
static sas_status check_attention_args(int mode, const sas_config* cfg, const void* q,
                                       const sas_kv* kv, const void* w_q, const float* gamma_q,
                                       const void* w_k, const float* gamma_k,
                                       const void* gate_keys, int32_t max_gate_blocks,
                                       const void* out, const int32_t* sel_idx,
                                       const int32_t* sel_count, const float* group_scores,
                                       const void* ws, size_t ws_bytes, bool* launch) {
  *launch = false;
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if ((st = check_kv(cfg, kv)) != SAS_OK) return st;
  if ((st = check_ws(cfg, const_cast<void*>(ws), ws_bytes)) != SAS_OK) return st;
  if (kv->batch == 0) return SAS_OK;
  if (q == nullptr || out == nullptr || !aligned(q, 16) || !aligned(out, 4)) return SAS_ERR_INVALID_ARG;
  if (mode == sas::kModeFused) {
    if (max_gate_blocks < 1 || max_gate_blocks > kMaxGateBlocks) return SAS_ERR_INVALID_ARG;
    if (w_q == nullptr || gamma_q == nullptr || gate_keys == nullptr) return SAS_ERR_INVALID_ARG;
    if (!aligned(w_q, 16) || !aligned(gamma_q, 16) || !aligned(gate_keys, 16)) return SAS_ERR_INVALID_ARG;
    if ((w_k == nullptr) != (gamma_k == nullptr)) return SAS_ERR_INVALID_ARG;
    if (w_k != nullptr && (!aligned(w_k, 16) || !aligned(gamma_k, 16))) return SAS_ERR_INVALID_ARG;
    if ((sel_idx != nullptr && !aligned(sel_idx, 4)) || (sel_count != nullptr && !aligned(sel_count, 4)) ||
        (group_scores != nullptr && !aligned(group_scores, 4)))
      return SAS_ERR_INVALID_ARG;
  } else {
    if (sel_idx == nullptr || sel_count == nullptr || !aligned(sel_idx, 4) || !aligned(sel_count, 4))
      return SAS_ERR_INVALID_ARG;
    // the gated mode needs the gate query and keys, which this call has not
    if (cfg->gate_mode != SAS_GATE_SELECT_ONLY) return SAS_ERR_UNSUPPORTED;
    max_gate_blocks = 1;
  }
  if (static_cast<long long>(kv->batch) * cfg->num_kv_heads > 65535) return SAS_ERR_UNSUPPORTED;
  sas::DecodeParams p{};
  fill_common(p, cfg, max_gate_blocks);
  if (!plan_ok(p)) return SAS_ERR_UNSUPPORTED;
  *launch = true;
  return SAS_OK;
}

static sas_status attention_call(int mode, const sas_config* cfg, const void* q, const sas_kv* kv,
                                 const void* w_q, const float* gamma_q, const void* w_k,
                                 const float* gamma_k, void* gate_keys, int32_t max_gate_blocks,
                                 void* out, int32_t* sel_idx, int32_t* sel_count,
                                 float* group_scores, void* ws, size_t ws_bytes,
                                 sas_stream_t stream, bool q_mapped = false) {
  bool launch = false;
  sas_status st = check_attention_args(mode, cfg, q, kv, w_q, gamma_q, w_k, gamma_k, gate_keys,
                                       max_gate_blocks, out, sel_idx, sel_count, group_scores, ws,
                                       ws_bytes, &launch);
  if (st != SAS_OK || !launch) return st;
  if (mode != sas::kModeFused) max_gate_blocks = 1;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  sas::DecodeParams p{};
  fill_common(p, cfg, max_gate_blocks);
  p.q = q;
  p.q_mapped = q_mapped ? 1 : 0;
  p.w_q = static_cast<const __nv_bfloat16*>(w_q);
  p.gamma_q = gamma_q;
  p.gate_keys = gate_keys;
  p.gamma_k = (mode == sas::kModeFused) ? gamma_k : nullptr;
  p.gate_keys_out = gate_keys;
  p.kv = make_view(cfg, kv);
  p.group_scores = group_scores;
  p.sel_idx = sel_idx;
  p.sel_count = sel_count;
  p.out = out;
  p.status = static_cast<uint32_t*>(ws);
  p.trace = trace_region(ws);
  const bool f32_kv = cfg->kv_dtype == SAS_DTYPE_F32;
  CUtensorMap tmk, tmv, tmw, tmwk;
  memset(&tmk, 0, sizeof(tmk));
  memset(&tmv, 0, sizeof(tmv));
  memset(&tmw, 0, sizeof(tmw));
  memset(&tmwk, 0, sizeof(tmwk));
  if (!f32_kv) {
    const long long rows = kv_rows(cfg, kv);
    if (!encode_kv_map(&tmk, kv->k, rows) || !encode_kv_map(&tmv, kv->v, rows)) return SAS_ERR_CUDA;
  }
  if (mode == sas::kModeFused && !encode_wq_map(&tmw, w_q, cfg->num_q_heads)) return SAS_ERR_CUDA;
  if (p.gamma_k != nullptr && !encode_wk_map(&tmwk, w_k, cfg->num_kv_heads)) return SAS_ERR_CUDA;
  return launch_result(sas::launch_decode(mode, f32_kv, cfg->out_dtype == SAS_DTYPE_F32,
                                          kClusterSize, kStages, p, tmk, tmv, tmw, tmwk, kv->batch,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_prefill_block_sparse(const sas_config* cfg, const void* q, const void* k,
                                    const void* v, int32_t batch, int32_t seq_len,
                                    const int32_t* token_budgets, const void* w_q, const float* gamma_q, const void* w_k,
                                    const float* gamma_k, void* gate_keys,
                                    int32_t max_gate_blocks, void* out, int32_t* sel_idx,
                                    int32_t* sel_count, void* ws, size_t ws_bytes,
                                    sas_stream_t stream) {
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if (batch < 0 || seq_len < 0) return SAS_ERR_INVALID_ARG;
  if (batch == 0 || seq_len == 0) return SAS_OK;
  if (cfg->kv_dtype != SAS_DTYPE_BF16 || cfg->out_dtype != SAS_DTYPE_BF16) return SAS_ERR_UNSUPPORTED;
  const int G = cfg->num_q_heads / cfg->num_kv_heads;
  if (seq_len % 64 != 0) return SAS_ERR_UNSUPPORTED;
  if (cfg->token_budget / 64 > sas::kPfMaxSel) return SAS_ERR_UNSUPPORTED;
  const int nblk = seq_len / 64;
  if (max_gate_blocks < nblk || max_gate_blocks > kMaxGateBlocks) return SAS_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || w_q == nullptr || gamma_q == nullptr ||
      w_k == nullptr || gamma_k == nullptr || gate_keys == nullptr || out == nullptr)
    return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(w_q, 16) ||
      !aligned(gamma_q, 16) || !aligned(w_k, 16) || !aligned(gamma_k, 16) ||
      !aligned(gate_keys, 16) || !aligned(out, 16) || (sel_idx != nullptr && !aligned(sel_idx, 4)) ||
      (sel_count != nullptr && !aligned(sel_count, 4)) || !aligned(token_budgets, 4))
    return SAS_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, 256)) return SAS_ERR_WORKSPACE;
  if (ws_bytes < sas_workspace_bytes(cfg, batch, seq_len)) return SAS_ERR_WORKSPACE;
  const long long qrows = static_cast<long long>(batch) * cfg->num_q_heads * seq_len;
  if (qrows > 0x7fffffffLL) return SAS_ERR_UNSUPPORTED;
  if (static_cast<long long>(batch) * cfg->num_kv_heads * nblk * ((G + 1) / 2) > 0x7fffffffLL)
    return SAS_ERR_UNSUPPORTED;
  if (batch > 65535 || cfg->num_q_heads > 65535) return SAS_ERR_UNSUPPORTED;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // 1. pooled gate keys of every block
  sas_kv kv{};
  kv.k = k;
  kv.v = v;
  kv.block_table = nullptr;
  kv.seq_lens = nullptr;  // every sequence has seq_len tokens
  kv.batch = batch;
  kv.capacity = seq_len;
  sas::PoolParams pp{};
  pp.hkv = cfg->num_kv_heads;
  pp.mg = max_gate_blocks;
  pp.num_blocks = nblk;
  pp.rope_base = cfg->rope_base;
  pp.eps = cfg->norm_eps;
  sas::fill_rope_table(pp.rope, cfg->rope_base);
  pp.kv = make_view(cfg, &kv);
  pp.blk_begin = nullptr;
  pp.w_k = static_cast<const __nv_bfloat16*>(w_k);
  pp.gamma_k = gamma_k;
  pp.gate_keys = gate_keys;
  pp.gk16 = cfg->gate_keys_bf16;
  pp.pooled_raw = nullptr;
  pp.status = static_cast<uint32_t*>(ws);
  CUtensorMap tmwk;
  if (!encode_kv_map(&tmwk, w_k, static_cast<long long>(cfg->num_kv_heads) * sas::kPool)) return SAS_ERR_CUDA;
  cudaError_t e = sas::launch_pool_project(pp, tmwk, batch, s);
  if (e != cudaSuccess) return launch_result(e);

  // 2-4. gate queries, selection, tensor-core block-sparse attention
  sas::PrefillParams p{};
  sas::fill_rope_table(p.rope, cfg->rope_base);
  p.batch = batch;
  p.hq = cfg->num_q_heads;
  p.hkv = cfg->num_kv_heads;
  p.G = G;
  p.T = seq_len;
  p.nblk = nblk;
  p.max_sel = cfg->token_budget / 64;
  p.topk = p.max_sel - 1;
  p.mg = max_gate_blocks;
  p.eps = cfg->norm_eps;
  p.attn_scale_log2 = cfg->attn_scale * 1.4426950408889634f;
  p.gate_scale = cfg->gate_scale;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.w_q = static_cast<const __nv_bfloat16*>(w_q);
  p.gamma_q = gamma_q;
  p.gate_keys = gate_keys;
  p.gk16 = cfg->gate_keys_bf16;
  uint8_t* scratch = static_cast<uint8_t*>(ws) + ws_header_bytes() + bwd_scratch_bytes(cfg, batch);
  p.qt = reinterpret_cast<float*>(scratch);
  scratch += up256(static_cast<size_t>(batch) * p.hq * nblk * kDim * 4);
  p.sel = reinterpret_cast<int32_t*>(scratch);
  scratch += up256(static_cast<size_t>(batch) * p.hkv * nblk * p.max_sel * 4);
  p.cnt = reinterpret_cast<int32_t*>(scratch);
  p.gated = (cfg->gate_mode == SAS_GATE_LOGSIGMOID_BIAS) ? 1 : 0;
  p.token_budgets = token_budgets;
  p.sel_out = sel_idx;
  p.cnt_out = sel_count;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = static_cast<uint32_t*>(ws);
  p.trace = trace_region(ws);
  CUtensorMap tmq, tmk, tmv;
  if (!encode_kv_map(&tmq, q, qrows) ||
      !encode_kv_map(&tmk, k, static_cast<long long>(batch) * p.hkv * seq_len) ||
      !encode_kv_map(&tmv, v, static_cast<long long>(batch) * p.hkv * seq_len))
    return SAS_ERR_CUDA;
  return launch_result(sas::launch_prefill(p, tmq, tmk, tmv, s));
}

sas_status sas_gate_backward(const sas_config* cfg, const void* q, const sas_kv* kv,
                             const void* w_q, const float* gamma_q, const void* w_k,
                             const float* gamma_k, const int32_t* sel_idx,
                             const int32_t* sel_count, const float* d_out, float* dw_q,
                             float* dw_k, float* dgamma_q, float* dgamma_k, void* ws,
                             size_t ws_bytes, sas_stream_t stream) {
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if ((st = check_kv(cfg, kv)) != SAS_OK) return st;
  if ((st = check_ws(cfg, ws, ws_bytes)) != SAS_OK) return st;
  if (kv->batch == 0) return SAS_OK;
  if (q == nullptr || w_q == nullptr || gamma_q == nullptr || w_k == nullptr || gamma_k == nullptr ||
      sel_idx == nullptr || sel_count == nullptr || d_out == nullptr || dw_q == nullptr ||
      dw_k == nullptr || dgamma_q == nullptr || dgamma_k == nullptr)
    return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 4) || !aligned(w_q, 4) || !aligned(gamma_q, 4) || !aligned(w_k, 16) ||
      !aligned(gamma_k, 4) || !aligned(sel_idx, 4) || !aligned(sel_count, 4) ||
      !aligned(d_out, 4) || !aligned(dw_q, 4) || !aligned(dw_k, 4) || !aligned(dgamma_q, 4) ||
      !aligned(dgamma_k, 4))
    return SAS_ERR_INVALID_ARG;
  if (cfg->kv_dtype != SAS_DTYPE_BF16) return SAS_ERR_UNSUPPORTED;
  const int G = cfg->num_q_heads / cfg->num_kv_heads;
  const int max_sel = cfg->token_budget / 64;
  // as many K/V stages (up to 4) as fit beside the list's pooled keys
  int stages = 4;
  while (stages > 1 && sas::gate_bwd_smem_bytes(G, max_sel, stages) > 227 * 1024) --stages;
  if (max_sel > sas::kBwMaxSel || sas::gate_bwd_smem_bytes(G, max_sel, stages) > 227 * 1024)
    return SAS_ERR_UNSUPPORTED;
  if (static_cast<long long>(kv->batch) * cfg->num_kv_heads > 0x7fffffffLL) return SAS_ERR_UNSUPPORTED;
  if (kv_rows(cfg, kv) > 0x7fffffffLL) return SAS_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  // the select-only mode gives the gate parameters no gradient
  if (cfg->gate_mode == SAS_GATE_SELECT_ONLY) return SAS_OK;
  // the per-pair terms the reduction sums live in the workspace
  if (ws_bytes < sas_workspace_bytes(cfg, kv->batch, 0)) return SAS_ERR_WORKSPACE;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  sas::GateBwdParams p{};
  sas::fill_rope_table(p.rope, cfg->rope_base);
  p.hq = cfg->num_q_heads;
  p.hkv = cfg->num_kv_heads;
  p.G = G;
  p.max_sel = max_sel;
  p.eps = cfg->norm_eps;
  p.attn_scale = cfg->attn_scale;
  p.gate_scale = cfg->gate_scale;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kv = make_view(cfg, kv);
  p.w_q = static_cast<const __nv_bfloat16*>(w_q);
  p.gamma_q = gamma_q;
  p.w_k = static_cast<const __nv_bfloat16*>(w_k);
  p.gamma_k = gamma_k;
  p.sel_idx = sel_idx;
  p.sel_count = sel_count;
  p.d_out = d_out;
  p.stages = stages;
  p.batch = kv->batch;
  p.dw_q = dw_q;
  p.dw_k = dw_k;
  p.dgamma_q = dgamma_q;
  p.dgamma_k = dgamma_k;
  p.status = static_cast<uint32_t*>(ws);
  {
    const size_t B = static_cast<size_t>(kv->batch), pairs = B * cfg->num_kv_heads;
    uint8_t* w = static_cast<uint8_t*>(ws) + ws_header_bytes();
    p.ws_dv = reinterpret_cast<float*>(w);
    w += up256(B * cfg->num_q_heads * kDim * 4);
    p.ws_p = reinterpret_cast<float*>(w);
    w += up256(pairs * max_sel * sas::kPool * 4);
    p.ws_du = reinterpret_cast<float*>(w);
    w += up256(pairs * max_sel * kDim * 4);
    p.ws_dg = reinterpret_cast<float*>(w);
    w += up256(pairs * 2 * kDim * 4);
    p.ws_nh = reinterpret_cast<int32_t*>(w);
  }
  p.trace = trace_region(ws);
  CUtensorMap tmk, tmv, tmwk;
  const long long rows = kv_rows(cfg, kv);
  if (!encode_kv_map(&tmk, kv->k, rows) || !encode_kv_map(&tmv, kv->v, rows)) return SAS_ERR_CUDA;
  // W_k as [Hkv * 384][128] in 64 x 64 boxes (64-row chunks of the projection)
  if (!encode_kv_map(&tmwk, w_k, static_cast<long long>(cfg->num_kv_heads) * sas::kPool)) return SAS_ERR_CUDA;
  return launch_result(sas::launch_gate_backward(p, tmk, tmv, tmwk, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_prefill_gate_backward(const sas_config* cfg, const void* q, const void* k, const void* v,
                                     int32_t batch, int32_t seq_len, const void* w_q, const float* gamma_q,
                                     const void* w_k, const float* gamma_k, const void* gate_keys,
                                     int32_t max_gate_blocks, const int32_t* sel_idx, const int32_t* sel_count,
                                     const float* d_out, float* dw_q, float* dw_k, float* dgamma_q,
                                     float* dgamma_k, void* ws, size_t ws_bytes, sas_stream_t stream) {
  sas_status st = check_config(cfg);
  if (st != SAS_OK) return st;
  if (batch < 0 || seq_len < 0) return SAS_ERR_INVALID_ARG;
  if (batch == 0 || seq_len == 0) return SAS_OK;
  if (q == nullptr || k == nullptr || v == nullptr || w_q == nullptr || gamma_q == nullptr || w_k == nullptr ||
      gamma_k == nullptr || gate_keys == nullptr || sel_idx == nullptr || sel_count == nullptr ||
      d_out == nullptr || dw_q == nullptr || dw_k == nullptr || dgamma_q == nullptr || dgamma_k == nullptr)
    return SAS_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(w_q, 2) || !aligned(gamma_q, 4) ||
      !aligned(w_k, 2) || !aligned(gamma_k, 4) || !aligned(gate_keys, 16) || !aligned(sel_idx, 4) ||
      !aligned(sel_count, 4) || !aligned(d_out, 16) || !aligned(dw_q, 4) || !aligned(dw_k, 4) ||
      !aligned(dgamma_q, 4) || !aligned(dgamma_k, 4))
    return SAS_ERR_INVALID_ARG;
  if (cfg->kv_dtype != SAS_DTYPE_BF16 || cfg->gate_keys_bf16 != 0) return SAS_ERR_UNSUPPORTED;
  if (seq_len % 64 != 0) return SAS_ERR_UNSUPPORTED;
  const int nblk = seq_len / 64;
  const int max_sel = cfg->token_budget / 64;
  if (max_gate_blocks < nblk || max_gate_blocks > kMaxGateBlocks) return SAS_ERR_INVALID_ARG;
  if (max_sel > sas::kPbMaxSel) return SAS_ERR_UNSUPPORTED;
  const int stages = sas::prefill_bwd_smem_bytes(max_sel, 2) <= 113 * 1024 ? 2 : 1;
  if (sas::prefill_bwd_smem_bytes(max_sel, stages) > 227 * 1024) return SAS_ERR_UNSUPPORTED;
  if (static_cast<long long>(nblk) * (sas::kPbChunk / 32 + 1) * 4 > 227 * 1024) return SAS_ERR_UNSUPPORTED;
  if (static_cast<long long>(batch) * cfg->num_q_heads * seq_len > 0x7fffffffLL) return SAS_ERR_UNSUPPORTED;
  if (batch > 65535 || cfg->num_q_heads > 65535 || nblk > 0x7fffffff) return SAS_ERR_UNSUPPORTED;
  if (ws == nullptr || !aligned(ws, 256)) return SAS_ERR_WORKSPACE;
  // the select-only mode gives the gate parameters no gradient
  if (cfg->gate_mode == SAS_GATE_SELECT_ONLY) return SAS_OK;
  if (ws_bytes < sas_workspace_bytes(cfg, batch, seq_len)) return SAS_ERR_WORKSPACE;
  if (prepare() != cudaSuccess) return SAS_ERR_CUDA;
  sas::PrefillBwdParams p{};
  sas::fill_rope_table(p.rope, cfg->rope_base);
  p.batch = batch;
  p.hq = cfg->num_q_heads;
  p.hkv = cfg->num_kv_heads;
  p.G = cfg->num_q_heads / cfg->num_kv_heads;
  p.T = seq_len;
  p.nblk = nblk;
  p.max_sel = max_sel;
  p.mg = max_gate_blocks;
  p.stages = stages;
  p.eps = cfg->norm_eps;
  p.attn_scale = cfg->attn_scale;
  p.gate_scale = cfg->gate_scale;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.w_q = static_cast<const __nv_bfloat16*>(w_q);
  p.gamma_q = gamma_q;
  p.w_k = static_cast<const __nv_bfloat16*>(w_k);
  p.gamma_k = gamma_k;
  p.gate_keys = static_cast<const float*>(gate_keys);
  p.sel_idx = sel_idx;
  p.sel_count = sel_count;
  p.d_out = d_out;
  p.dw_q = dw_q;
  p.dw_k = dw_k;
  p.dgamma_q = dgamma_q;
  p.dgamma_k = dgamma_k;
  p.status = static_cast<uint32_t*>(ws);
  {
    // after the header, the decode backward's terms and the prefill scratch
    const size_t B = static_cast<size_t>(batch);
    uint8_t* w = static_cast<uint8_t*>(ws) + ws_header_bytes() + bwd_scratch_bytes(cfg, batch) +
                 prefill_scratch_bytes(B, p.hq, p.hkv, nblk, max_sel);
    const size_t qh = B * p.hq * nblk, kh = B * p.hkv * nblk;
    p.ws_qbar = reinterpret_cast<float*>(w);
    w += up256(qh * kDim * 4);
    p.ws_qt = reinterpret_cast<float*>(w);
    w += up256(qh * kDim * 4);
    p.ws_dv = reinterpret_cast<float*>(w);
    w += up256(qh * kDim * 4);
    p.ws_dgq = reinterpret_cast<float*>(w);
    w += up256(qh * kDim * 4);
    p.ws_ds = reinterpret_cast<float*>(w);
    w += up256(qh * max_sel * 4);
    p.ws_p = reinterpret_cast<float*>(w);
    w += up256(kh * sas::kPool * 4);
    p.ws_du = reinterpret_cast<float*>(w);
    w += up256(kh * kDim * 4);
    p.ws_dgk = reinterpret_cast<float*>(w);
    w += up256(kh * kDim * 4);
    p.ws_gpart = reinterpret_cast<float*>(w);
  }
  CUtensorMap tmq, tmk, tmv;
  const long long qrows = static_cast<long long>(batch) * p.hq * seq_len;
  const long long krows = static_cast<long long>(batch) * p.hkv * seq_len;
  if (!encode_kv_map(&tmq, q, qrows) || !encode_kv_map(&tmk, k, krows) || !encode_kv_map(&tmv, v, krows))
    return SAS_ERR_CUDA;
  return launch_result(sas::launch_prefill_gate_backward(p, tmq, tmk, tmv, reinterpret_cast<cudaStream_t>(stream)));
}

sas_status sas_sparse_decode(const sas_config* cfg, const void* q, const sas_kv* kv,
                             const int32_t* sel_idx, const int32_t* sel_count, void* out,
                             void* ws, size_t ws_bytes, sas_stream_t stream) {
  return attention_call(sas::kModeAttend, cfg, q, kv, nullptr, nullptr, nullptr, nullptr, nullptr,
                        0, out, const_cast<int32_t*>(sel_idx), const_cast<int32_t*>(sel_count),
                        nullptr, ws, ws_bytes, stream);
}

}  // extern "C"

namespace sas {
sas_status check_decode_step_args(const sas_config* cfg, const void* q, const sas_kv* kv,
                                  const void* w_q, const float* gamma_q, const void* w_k,
                                  const float* gamma_k, const void* gate_keys,
                                  int32_t max_gate_blocks, const void* out, const int32_t* sel_idx,
                                  const int32_t* sel_count, const float* group_scores,
                                  const void* ws, size_t ws_bytes, bool* launch) {
  return check_attention_args(kModeFused, cfg, q, kv, w_q, gamma_q, w_k, gamma_k, gate_keys,
                              max_gate_blocks, out, sel_idx, sel_count, group_scores, ws, ws_bytes,
                              launch);
}
}  // namespace sas

extern "C" {

sas_status sas_decode_step(const sas_config* cfg, const void* q, const sas_kv* kv, const void* w_q,
                           const float* gamma_q, const void* w_k, const float* gamma_k,
                           void* gate_keys, int32_t max_gate_blocks, void* out,
                           int32_t* sel_idx, int32_t* sel_count, float* group_scores, void* ws,
                           size_t ws_bytes, sas_stream_t stream) {
  return attention_call(sas::kModeFused, cfg, q, kv, w_q, gamma_q, w_k, gamma_k, gate_keys,
                        max_gate_blocks, out, sel_idx, sel_count, group_scores, ws, ws_bytes,
                        stream);
}

// The device address of page-locked host memory (cudaHostAlloc,
// cudaHostRegister) that this context can reach, else nullptr (pageable
// memory).
static void* mapped_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

sas_status sas_decode_step_host(const sas_config* cfg, const void* q_host, void* q_dev,
                                const sas_kv* kv, const void* w_q, const float* gamma_q,
                                const void* w_k, const float* gamma_k, void* gate_keys,
                                int32_t max_gate_blocks, void* out_dev, void* out_host,
                                int32_t* sel_idx, int32_t* sel_count, float* group_scores,
                                void* ws, size_t ws_bytes, sas_stream_t stream) {
  bool launch = false;
  sas_status st = check_attention_args(sas::kModeFused, cfg, q_dev, kv, w_q, gamma_q, w_k, gamma_k,
                                       gate_keys, max_gate_blocks, out_dev, sel_idx, sel_count,
                                       group_scores, ws, ws_bytes, &launch);
  if (st != SAS_OK || !launch) return st;
  if (q_host == nullptr || out_host == nullptr) return SAS_ERR_INVALID_ARG;
  const size_t elems = static_cast<size_t>(kv->batch) * cfg->num_q_heads * kDim;
  const size_t q_bytes = elems * (cfg->kv_dtype == SAS_DTYPE_F32 ? 4 : 2);
  const size_t out_bytes = elems * (cfg->out_dtype == SAS_DTYPE_F32 ? 4 : 2);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // page-locked buffers move over the host link inside the step kernel (no
  // copy engine next to the launch); pageable ones take a runtime copy
  const void* q_src = mapped_host(q_host);
  void* out_dst = mapped_host(out_host);
  const bool q_mapped = q_src != nullptr && aligned(q_src, 16);
  if (!q_mapped) {
    st = launch_result(cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, s));
    if (st != SAS_OK) return st;
  }
  void* out_target = (out_dst != nullptr && aligned(out_dst, 4)) ? out_dst : out_dev;
  st = attention_call(sas::kModeFused, cfg, q_mapped ? q_src : q_dev, kv, w_q, gamma_q, w_k, gamma_k,
                      gate_keys, max_gate_blocks, out_target, sel_idx, sel_count, group_scores, ws,
                      ws_bytes, stream, q_mapped);
  if (st != SAS_OK || out_target != out_dev) return st;
  return launch_result(cudaMemcpyAsync(out_host, out_dev, out_bytes, cudaMemcpyDeviceToHost, s));
}

}  // extern "C"
