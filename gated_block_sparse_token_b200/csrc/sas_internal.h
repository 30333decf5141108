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
// of the cluster decode kernel.  Region R is reused across phases:
//   phases 0-1  [ qv | wq | qs ]
//   phases 2-4  [ inbox | pool P | pool u | keys | hist | selbits | scan ]
//               with the W_k slice of the fused pooling over keys.. once the
//               selection is done (rank 0) or the scores are sent (others)
// inbox (written by other CTAs after the attention phase) covers at least
// qv, and keys (written by the other CTAs of the cluster into rank 0 during
// their phase 1) starts past the inbox, so no remote write can land on data
// this CTA still reads.
constexpr int kSelBins = 1024;  // value buckets of the Top-K selection
constexpr int kSelCand = 256;   // candidates ranked exactly in the boundary bucket
// Distributed Top-K of the fused step (every CTA ranks its own gate-key rows,
// the clusters' CTAs exchange their sorted local candidates, every CTA ranks
// the union): taken when the sequence keeps at most kFastTopk historical
// blocks and no CTA holds more than kFastRows of them.
constexpr int kFastTopk = 64;
constexpr int kFastRows = 256;

struct DecodeSmem {
  int slots;     // NST stage slots of 16 KiB (gate-key chunks, then K/V tiles)
  int sel;       // int32 [max_sel] selected blocks (phases 2-3)
  int rows;      // int64 [ceil(max_sel / CS)] cache rows of this CTA's entries (paged)
  int gbias;     // fp32 [max_sel][G] gated mode: log-sigmoid gate per entry and head
  int qraw;      // T [G][128] query as stored (bf16 or fp32), bulk copy
  int qbar;      // fp32 [128] group-mean gate query (fused mode)
  int pml;       // fp32 m[4][8], l[4][8] per-warp softmax state
  int bars;      // uint64 [NST] mbarriers
  int r_qv;      // fp32 [G][128] gate query v, then q~ in place   (phases 0-1)
  int r_wq;      // bf16 [wq_heads][128][dpc] W_q column slice (TMA) (phase 0)
  int wq_heads;  // heads of the slice resident at once (G, or ceil(G / 2): two passes)
  int gam;       // fp32 [128] gamma_q (bulk copy)
  int r_inbox;   // fp32 [CS][G][dpc] o, then [CS][G][2] (m, l)     (phases 3-4)
  int r_pool_p;  // fp32 [384] pooled current block (fused pooling)  (phases 3-4)
  int r_pool_u;  // fp32 [CS][17] projected slices + sum of squares  (phases 3-4)
  int r_wk;      // bf16 [384][dpc] W_k column slice (TMA)           (phases 3-4)
  int gamk;      // fp32 [128] gamma_k (bulk copy, fused pooling)
  int r_keys;    // fp32 scores -> uint32 keys [mg] (rank 0)        (phases 1-2)
  int r_hist;    // uint32 [kSelBins], then int32 candidates        (phase 2)
  int r_selbits; // uint32 [(mg + 31) / 32]                         (phase 2)
  int r_scan;    // int32 [16]                                      (phase 2)
  // distributed Top-K (phases 1-2; over keys.., like the rank-0 selection)
  int r_lkeys;   // uint64 [kFastRows] this CTA's (score, block) keys
  int r_gather;  // uint64 [CS][kFastTopk] sorted local candidates of every CTA
  int total;     // bytes to request, including alignment slack
};

// Shared memory a CTA may take for four to fit on one SM (228 KiB per SM,
// 1 KiB of it reserved per CTA).
constexpr int kFourPerSmBytes = 228 * 1024 / 4 - 1024;

// wq_heads: heads of the W_q slice resident at once (G: one pass; fewer:
// phase 0 loads the slice in two passes through the same region).
inline DecodeSmem plan_decode_smem_heads(int G, int mg, int cs, int nst, int max_sel, bool f32_kv, bool gated,
                                         int wq_heads) {
  DecodeSmem p{};
  int off = 0;
  auto take = [&](int bytes, int align) {
    off = (off + align - 1) / align * align;
    const int o = off;
    off += bytes;
    return o;
  };
  auto up16 = [](int x) { return (x + 15) / 16 * 16; };
  const int dpc = kDim / cs;
  mg = std::max(mg, 1);
  p.wq_heads = wq_heads;
  p.slots = take(nst * kTileBytes, 1024);
  p.sel = take(max_sel * 4, 16);
  p.rows = take((max_sel + cs - 1) / cs * 8, 16);
  p.gbias = take(gated ? max_sel * G * 4 : 0, 16);
  p.qraw = take(G * kDim * (f32_kv ? 4 : 2), 16);
  p.qbar = take(kDim * 4, 16);
  p.pml = take(2 * kWarps * kMaxGroup * 4, 16);
  p.gam = take(kDim * 4, 16);
  p.gamk = take(kDim * 4, 16);
  // ring slots, prologue, pooled P, W_k slice, scores (rank 0), list, v,
  // attention partials, pooled slices (rank 0), second W_q pass
  p.bars = take((nst + 9) * 8, 8);
  auto up128 = [](int x) { return (x + 127) / 128 * 128; };
  const int r = up128(off);
  // phases 0-1 (the W_q slice is a tensor-TMA destination: 128-byte aligned)
  p.r_qv = r;
  p.r_wq = up128(r + G * kDim * 4);
  const int end01 = p.r_wq + up16(wq_heads * kDim * dpc * 2);
  // phases 2-4 (gated mode: clear of q~, which the gates read after the list)
  p.r_inbox = gated ? up16(r + G * kDim * 4) : r;
  p.r_pool_p = p.r_inbox + up16(cs * G * (dpc + 2) * 4);
  p.r_pool_u = p.r_pool_p + up16(kPool * 4);
  p.r_keys = up128(p.r_pool_u + up16(cs * 17 * 4));
  p.r_wk = p.r_keys;
  p.r_hist = p.r_keys + up16(mg * 4);
  p.r_selbits = p.r_hist + up16(std::max(kSelBins, kSelCand) * 4);
  p.r_scan = p.r_selbits + up16((mg + 31) / 32 * 4);
  p.r_lkeys = p.r_keys;
  p.r_gather = p.r_lkeys + kFastRows * 8;
  const int end_fast = p.r_gather + cs * kFastTopk * 8;
  const int end24 = std::max(std::max(p.r_scan + 16 * 4, end_fast), p.r_wk + kPool * dpc * 2);
  p.total = std::max(end01, end24) + 1024;
  return p;
}

// One pass over W_q when four CTAs fit on an SM that way (or two passes
// would not make them fit); else two passes of ceil(G / 2) heads.
inline DecodeSmem plan_decode_smem(int G, int mg, int cs, int nst, int max_sel, bool f32_kv,
                                   bool gated = false) {
  const DecodeSmem one = plan_decode_smem_heads(G, mg, cs, nst, max_sel, f32_kv, gated, G);
  if (one.total <= kFourPerSmBytes || G < 2) return one;
  const DecodeSmem two = plan_decode_smem_heads(G, mg, cs, nst, max_sel, f32_kv, gated, (G + 1) / 2);
  return two.total <= kFourPerSmBytes ? two : one;
}

// TMA destinations of the plan: tensor boxes need 128-byte (swizzled: 1024-
// byte) aligned shared addresses, bulk copies 16-byte ones.
inline bool decode_smem_aligned(const DecodeSmem& p, int G, int dpc) {
  return p.slots % 1024 == 0 && p.r_wq % 128 == 0 && (G * kDim * dpc * 2) % 128 == 0 &&
         p.r_wk % 128 == 0 && p.qraw % 16 == 0 && p.gam % 16 == 0 && p.gamk % 16 == 0 &&
         p.bars % 8 == 0;
}

struct DecodeParams {
  RopeTable rope;
  unsigned long long* trace;  // phase timestamps (tracing builds only), else null
  int hq, hkv, G;
  int topk;     // historical blocks kept: budget/64 - 1
  int max_sel;  // budget/64
  int mg;       // rows of the gate-key cache per (seq, head)
  float rope_base, eps, attn_scale_log2, gate_scale;
  int gated;    // 1: log-sigmoid gate bias on the selected historical blocks
  const void* q;
  const __nv_bfloat16* w_q;
  const float* gamma_q;
  const void* gate_keys;  // fp32, or bf16 when gk16 [B][Hkv][mg][128]
  const float* gamma_k;  // fused pooling of a completed current block (null: off)
  void* gate_keys_out;   // same array as gate_keys, written at row c when pooling
  int gk16;              // gate keys stored as bf16
  // 1: W_q, gamma_q and gamma_k are read before the kernels ahead on the
  // stream have finished (the caller guarantees that none writes them);
  // 0: every input is read after they have finished
  int static_weights;
  int q_mapped;          // q is page-locked host memory at its device address:
                         // the cluster's CTAs each load a share and broadcast it
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
  const int32_t* token_budgets;  // null: topk for every sequence
  int32_t* sel_idx;
  int32_t* sel_count;
  uint32_t* status;
};

struct PoolParams {
  RopeTable rope;
  int hkv, mg, num_blocks;
  float rope_base, eps;
  KvView kv;
  const int32_t* blk_begin;
  const __nv_bfloat16* w_k;
  const float* gamma_k;
  void* gate_keys;  // fp32, or bf16 when gk16
  int gk16;
  float* pooled_raw;
  uint32_t* status;
};

struct PrefillParams {
  RopeTable rope;
  int batch, hq, hkv, G, T, nblk, topk, max_sel, mg;
  float eps, attn_scale_log2, gate_scale;
  const __nv_bfloat16* q;     // [B][Hq][T][128]
  const __nv_bfloat16* w_q;   // [Hq][128][128]
  const float* gamma_q;       // [128]
  const void* gate_keys;      // [B][Hkv][mg][128], fp32 or bf16 (gk16)
  int gk16;
  float* qt;                  // workspace: gate queries [B][Hq][nblk][128]
  int32_t* sel;               // workspace: block lists [B][Hkv][nblk][max_sel]
  int32_t* cnt;               // workspace: list lengths [B][Hkv][nblk]
  int32_t* sel_out;           // optional copies of the lists
  int32_t* cnt_out;
  int gated;                  // gated mode: + log(sigmoid(gate score)) on kept historical blocks
  const int32_t* token_budgets;  // [B] per-sequence budgets, or null (topk for every sequence)
  __nv_bfloat16* out;         // [B][Hq][T][128]
  uint32_t* status;
  unsigned long long* trace;  // per-CTA timings (tracing builds only), else null
};

// Gradient through the gates of the gated decode step (one CTA per
// (sequence, KV head), the block list held fixed).
constexpr int kBwThreads = 256;
constexpr int kBwMaxSel = 64;  // block lists of up to 64 entries (4,096 tokens)

struct GateBwdParams {
  RopeTable rope;
  int hq, hkv, G, max_sel;
  float eps, attn_scale, gate_scale;
  const __nv_bfloat16* q;     // [B][Hq][128]
  KvView kv;
  const __nv_bfloat16* w_q;   // [Hq][128][128]
  const float* gamma_q;       // [128]
  const __nv_bfloat16* w_k;   // [Hkv][384][128]
  const float* gamma_k;       // [128]
  const int32_t* sel_idx;     // [B][Hkv][max_sel]
  const int32_t* sel_count;   // [B][Hkv]
  const float* d_out;         // [B][Hq][128]
  int stages;                 // K/V ring stages (2, or 1 when two do not fit)
  int batch;                  // B
  float* dw_q;                // [Hq][128][128]  (accumulated)
  float* dw_k;                // [Hkv][384][128] (accumulated)
  float* dgamma_q;            // [128]           (accumulated)
  float* dgamma_k;            // [128]           (accumulated)
  // per-pair terms the reduction kernel sums (workspace)
  float* ws_dv;               // [B][Hq][128]        dL/dv_g
  float* ws_p;                // [B*Hkv][max_sel][384] pooled keys of the historical entries
  float* ws_du;               // [B*Hkv][max_sel][128] dL/du_e
  float* ws_dg;               // [B*Hkv][2][128]     gain gradients (q, k)
  int32_t* ws_nh;             // [B*Hkv]             historical entries (-1: pair skipped)
  uint32_t* status;
  unsigned long long* trace;  // per-CTA step timings (tracing builds only), else null
};

// Workspace bytes of the backward's per-pair terms (after the status header).
inline size_t gate_bwd_scratch_bytes(size_t batch, int hq, int hkv, int max_sel) {
  auto up256 = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t pairs = batch * static_cast<size_t>(hkv);
  return up256(batch * hq * kDim * 4) + up256(pairs * max_sel * kPool * 4) + up256(pairs * max_sel * kDim * 4) +
         up256(pairs * 2 * kDim * 4) + up256(pairs * 4);
}

// Gradient through the gates of the gated prefill (block lists held fixed).
constexpr int kPbThreads = 128;  // attention pass: 4 warps of 16 query tokens
constexpr int kPbMaxSel = 64;    // block lists of up to 64 entries (4,096 tokens)
constexpr int kPbChunk = 128;    // key blocks per CTA of the gate-key pass

struct PrefillBwdParams {
  RopeTable rope;
  int batch, hq, hkv, G, T, nblk, max_sel, mg, stages;
  float eps, attn_scale, gate_scale;
  const __nv_bfloat16* q;      // [B][Hq][T][128]
  const __nv_bfloat16* k;      // [B][Hkv][T][128]
  const __nv_bfloat16* w_q;    // [Hq][128][128]
  const float* gamma_q;        // [128]
  const __nv_bfloat16* w_k;    // [Hkv][384][128]
  const float* gamma_k;        // [128]
  const float* gate_keys;      // [B][Hkv][mg][128] fp32 (the forward's)
  const int32_t* sel_idx;      // [B][Hkv][nblk][max_sel]
  const int32_t* sel_count;    // [B][Hkv][nblk]
  const float* d_out;          // [B][Hq][T][128]
  float* dw_q;                 // [Hq][128][128]  (accumulated)
  float* dw_k;                 // [Hkv][384][128] (accumulated)
  float* dgamma_q;             // [128]           (accumulated)
  float* dgamma_k;             // [128]           (accumulated)
  // per-(sequence, head, block) terms (workspace)
  float* ws_qbar;   // [B][Hq][nblk][128] block-mean gate query
  float* ws_qt;     // [B][Hq][nblk][128] q~
  float* ws_dv;     // [B][Hq][nblk][128] dL/dv
  float* ws_dgq;    // [B][Hq][nblk][128] dL/dgamma_q terms
  float* ws_ds;     // [B][Hq][nblk][max_sel] dL/ds of each list entry
  float* ws_p;      // [B][Hkv][nblk][384] pooled keys
  float* ws_du;     // [B][Hkv][nblk][128] dL/du
  float* ws_dgk;    // [B][Hkv][nblk][128] dL/dgamma_k terms
  float* ws_gpart;  // [Hq + Hkv][128] gain sums per head
  uint32_t* status;
};

inline size_t prefill_bwd_scratch_bytes(size_t batch, int hq, int hkv, size_t nblk, int max_sel) {
  auto up256 = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t qh = batch * hq * nblk, kh = batch * hkv * nblk;
  return 4 * up256(qh * kDim * 4) + up256(qh * max_sel * 4) + up256(kh * kPool * 4) + 2 * up256(kh * kDim * 4) +
         up256(static_cast<size_t>(hq + hkv) * kDim * 4);
}

// Shared memory of the prefill backward's attention pass: the K/V ring, the
// per-(entry, token) statistics (the Q tile first lands in the same region),
// the list and its gate terms, the gate-query vectors.
inline int prefill_bwd_smem_bytes(int max_sel, int stages) {
  const int stats = 3 * max_sel * 64 * 4;
  return stages * 2 * kTileBytes + (stats > kTileBytes ? stats : kTileBytes) + 4 * max_sel * 4 + 6 * kDim * 4 +
         64 + 1024;
}

// Shared-memory bytes of the backward kernel for a group of G heads and
// block lists of max_sel entries.
// Row stride (floats) of the pooled keys in the backward's shared memory:
// 8 floats of padding put the 8 rows of one tensor-core fragment load in
// different banks.
constexpr int kBwPoolStride = kPool + 8;

inline int gate_bwd_smem_bytes(int G, int max_sel, int stages = 2) {
  return stages * 2 * kTileBytes       // K and V tiles, 1 to 4 stages
         + max_sel * kBwPoolStride * 4 // pooled keys of the list
         + max_sel * kDim * 4          // u, then dL/du, per entry
         + 4 * G * kDim * 4            // q, d_out, v (then dL/dv), q~
         + 3 * max_sel * G * 4         // per-entry softmax statistics
         + 2 * max_sel * G * 4         // gate scores and their gradients
         + 2 * G * kBlock * 4          // logits and d_out . v of one block
         + 2 * max_sel * 4             // list, RMS of u
         + G * kDim * 2                // q as bf16 (the tensor-core operand)
         + G * kDim * 4                // dL/dq~ per head
         + 2 * kDim * 4                // dL/dgamma_q, dL/dgamma_k
         + 2 * (kBwThreads / 32) * kDim * 4  // their per-warp partial sums
         + 4 * kPool * 4               // pooling partials of one block (4 token quarters)
         + 8 * 8 + 1024;               // barriers, alignment slack
}

constexpr int kPfQb = 16;      // query blocks per gate-query CTA
constexpr int kPfMaxSel = 256;  // prefill budget up to 16,384 tokens (two CTAs per SM up to 4,096)

constexpr int kPoolBlocksPerCta = 8;
constexpr int kPoolWkBytes = kPool * kDim * 2;  // W_k of one KV head, bf16 (96 KiB)

// Phase-trace builds (-DSAS_PHASE_TRACE) record per-CTA timestamps after the
// status word; ordinary builds compile the hooks out.
constexpr int kTraceSlots = 32;
constexpr int kTraceCtas = 4096;

// Launchers (return the cudaError_t of the launch).
cudaError_t launch_decode(int mode, bool f32_kv, bool f32_out, int cs, int nst,
                          const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                          const CUtensorMap& tmw, const CUtensorMap& tmwk, int batch,
                          cudaStream_t stream);
cudaError_t launch_topk(const TopkParams& p, int batch, cudaStream_t stream);
cudaError_t launch_pool(bool f32_kv, const PoolParams& p, int batch, cudaStream_t stream);
// bf16 caches: pooling on the CUDA cores, projection on the tensor cores
// (tmwk: W_k as a [Hkv*384][128] bf16 map, 64x64 boxes, 128-byte swizzle)
cudaError_t launch_pool_project(const PoolParams& p, const CUtensorMap& tmwk, int batch, cudaStream_t stream);
size_t topk_smem_bytes(int mg, int max_sel);
size_t pool_smem_bytes();
void fill_rope_table(RopeTable& t, float base);
cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmq, const CUtensorMap& tmk,
                           const CUtensorMap& tmv, cudaStream_t stream);
size_t prefill_attn_smem_bytes(int max_sel);
cudaError_t launch_gate_backward(const GateBwdParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                 const CUtensorMap& tmwk, cudaStream_t stream);
cudaError_t launch_prefill_gate_backward(const PrefillBwdParams& p, const CUtensorMap& tmq, const CUtensorMap& tmk,
                                         const CUtensorMap& tmv, cudaStream_t stream);

// One-time per-process set-up of kernel attributes.
cudaError_t prepare_kernels();

}  // namespace sas

#include "sas.h"

namespace sas {

// Every host check sas_decode_step makes before it enqueues anything (the
// workspace check against ws / ws_bytes included); *launch is false when the
// call has nothing to do (batch 0).
sas_status check_decode_step_args(const sas_config* cfg, const void* q, const sas_kv* kv,
                                  const void* w_q, const float* gamma_q, const void* w_k,
                                  const float* gamma_k, const void* gate_keys,
                                  int32_t max_gate_blocks, const void* out, const int32_t* sel_idx,
                                  const int32_t* sel_count, const float* group_scores,
                                  const void* ws, size_t ws_bytes, bool* launch);

}  // namespace sas
