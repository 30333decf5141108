/*
 * sas.h -- C ABI of libsas: SAS (Simple-Attention-Sparsification) gated
 * Top-K KV-block selection feeding block-sparse GQA attention, for NVIDIA
 * B200 (sm_100a).
 *
 * What the method fixes (release pages: "Tencent released
 * Simple-Attention-Sparsification, a method for efficient sparse attention
 * in Qwen3 models", aigc.news 2026-09-14, release paragraph; "Simple-Attention-
 * Sparsification Text Generation Model: 12GB+ VRAM", localmodelwatch,
 * "Specifications and Configuration Table"):
 *   64-token KV blocks; a 128-wide gate; the query goes through a projection
 *   the pages call Qproj; each key block is summarised by its maximum,
 *   minimum and average; queries and keys are normalised and the gate applies
 *   RoPE; the top historical blocks are kept under a 1,024, 2,048 (default)
 *   or 4,096-token budget, the current block always kept (31 + 1 = 2,048/64).
 *
 * Readings of what the pages leave open (one per item, used by every entry
 * point):
 *   - gate weights: W_q [128][128] per query head, W_k [384][128] per KV head,
 *     bf16, applied as x @ W (row vector times matrix), no bias; one RMSNorm
 *     gain [128] for q and one for k per layer (the printed parameter counts
 *     33.0M / 42.0M fit exactly this layout);
 *   - pooled key of block b = [max ; min ; mean] over its 64 tokens, per dim;
 *   - k~_b = RoPE(RMSNorm(pooled_b @ W_k) * gamma_k, position b);
 *     q~_g = RoPE(RMSNorm(q_g @ W_q[g]) * gamma_q, position c), c the current
 *     block index floor((L-1)/64); RMSNorm x / sqrt(mean(x^2) + eps);
 *     RoPE rotate-half, pairs (i, i+64), angle pos * base^(-2i/128);
 *   - s_{g,b} = (q~_g . k~_b) * gate_scale; group score S_b = mean over the
 *     G = Hq/Hkv query heads of a KV head; one block set per KV head;
 *   - selection: the min(budget/64 - 1, c) historical blocks of largest S
 *     (ties: lower index), plus block c, listed in ascending order;
 *   - attention: softmax(q . k_j * attn_scale) over every token j <= L-1 of
 *     the selected blocks, each selected block weighted 1.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are caller-owned DEVICE memory (sas_decode_step_host
 *     also takes two host buffers); the library never
 *     allocates, frees or synchronises (except sas_get_device_status, which
 *     synchronises the given stream).
 *   - Every call validates its arguments on the host, enqueues its kernels on
 *     `stream` and returns.  Host-detected problems return an error code and
 *     enqueue nothing.  A failed launch returns SAS_ERR_CUDA.
 *   - Problems only the device can see (a sequence length beyond the cache,
 *     a page id out of range, a selected block beyond the current block)
 *     skip the affected (sequence, KV head), write zeros to its outputs and
 *     set a bit in the status word at the start of `ws`; read it with
 *     sas_get_device_status.  No device-side trap or assert is used.
 *   - Every bounded device wait that runs out (1 s) sets SAS_ERR_TIMEOUT's
 *     bit in the same status word and the kernel returns.
 *   - The first call that launches kernels performs one-time set-up (kernel
 *     attributes, driver entry point for tensor maps); make it before any
 *     CUDA stream capture.
 *   - Layouts are row-major C arrays; the shapes below use
 *     B = batch, Hq/Hkv = query/KV heads, D = 128, MG = max_gate_blocks.
 */
#ifndef SAS_H_
#define SAS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAS_API __attribute__((visibility("default")))
#else
#define SAS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t.  NULL means the legacy default stream. */
typedef struct CUstream_st* sas_stream_t;

typedef enum {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = 1,   /* a host-checked argument is wrong */
  SAS_ERR_UNSUPPORTED = 2,   /* valid request this build does not handle */
  SAS_ERR_WORKSPACE = 3,     /* ws NULL, misaligned or smaller than needed */
  SAS_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  SAS_ERR_DEVICE_BOUNDS = 5, /* device saw an out-of-range length/page/index */
  SAS_ERR_TIMEOUT = 6        /* a bounded device wait ran out */
} sas_status;

typedef enum { SAS_DTYPE_BF16 = 0, SAS_DTYPE_F32 = 1 } sas_dtype;

/* How the selected blocks enter the decode attention.
 *   SAS_GATE_SELECT_ONLY: every selected block weighs 1 (the gate only
 *     selects).
 *   SAS_GATE_LOGSIGMOID_BIAS: the attention logits of every token of a
 *     selected historical block b, for query head g, get + log(sigmoid(s_gb)),
 *     s_gb = (q~_g . k~_b) * gate_scale the head's gate score; the current
 *     block gets 0.  One plain reading of the continuous gates that the
 *     pages say weight the selected blocks (aigc.news release paragraph of
 *     2026-09-14). */
typedef enum { SAS_GATE_SELECT_ONLY = 0, SAS_GATE_LOGSIGMOID_BIAS = 1 } sas_gate_mode;

typedef struct {
  int32_t num_q_heads;   /* Hq >= 1 */
  int32_t num_kv_heads;  /* Hkv >= 1, Hq % Hkv == 0, 1 <= Hq/Hkv <= 8 */
  int32_t head_dim;      /* must be 128 */
  int32_t block_size;    /* must be 64 (KV block size of the method) */
  int32_t gate_hidden;   /* must be 128 (gate hidden size of the method) */
  int32_t token_budget;  /* multiple of 64, 64 .. 16384; default 2048 */
  float rope_base;       /* gate RoPE base, > 0; default 10000 */
  float norm_eps;        /* RMSNorm epsilon, >= 0; default 1e-6 */
  float attn_scale;      /* attention logit scale, > 0; default 1/sqrt(128) */
  float gate_scale;      /* gate score scale, > 0; default 1/sqrt(128) */
  int32_t kv_dtype;      /* sas_dtype of q, K and V (and of prefill Q) */
  int32_t out_dtype;     /* sas_dtype of the attention output */
  int32_t gate_mode;     /* sas_gate_mode; default SAS_GATE_SELECT_ONLY.
                            sas_decode_step(_static) and sas_prefill_block_sparse
                            implement the gated mode (prefill: gates from each
                            query block's gate query); sas_sparse_decode returns
                            SAS_ERR_UNSUPPORTED for it (it has no gate inputs);
                            the gate-score, Top-K and pooling calls ignore it. */
  int32_t gate_keys_bf16;  /* 0 (default): the gate-key cache is fp32
                              [B][Hkv][MG][128].  1: it is bf16, keys rounded to
                              nearest-even when written (half the bytes the
                              scores stream).  Every call that reads or writes
                              gate keys follows it. */
  int32_t static_weights; /* 0 (default) or 1.  The decode kernels are launched
                            with programmatic stream serialization: they may
                            start while kernels ahead of them on the stream
                            are still running, and read their inputs and
                            write their outputs only once those have
                            finished.  With 1, the caller guarantees that
                            w_q, gamma_q, w_k and gamma_k are not written by
                            any kernel that may still be running (weights of
                            an inference model never are), and the kernels
                            read them before that point. */
} sas_config;

/* KV cache description (device pointers, caller-owned). */
typedef struct {
  const void* k;               /* keys, kv_dtype, 16-byte aligned */
  const void* v;               /* values, same layout as k */
  const int32_t* block_table;  /* NULL: contiguous layout [B][Hkv][capacity][D].
                                  Else paged layout [num_pages][Hkv][64][D] and
                                  block_table [B][max_blocks_per_seq] holds the
                                  page id of each 64-token block. */
  const int32_t* seq_lens;     /* [B] context length L_s >= 1 of each sequence,
                                  including the token being decoded */
  int32_t batch;               /* B >= 0 (0: nothing to do) */
  int32_t capacity;            /* contiguous: tokens per (seq, head), multiple
                                  of 64; paged: ignored */
  int32_t num_pages;           /* paged: pages in the pool; contiguous: ignored */
  int32_t max_blocks_per_seq;  /* paged: row length of block_table */
  const int32_t* token_budgets; /* NULL: cfg->token_budget for every sequence.
                                   Else [B] per-sequence budgets (pages: 1,024,
                                   2,048 or 4,096 usable without retraining),
                                   each a multiple of 64 in 64 ..
                                   cfg->token_budget; cfg->token_budget sizes
                                   the block lists.  A sequence with a bad
                                   budget is skipped and reported as
                                   SAS_ERR_DEVICE_BOUNDS. */
} sas_kv;

/* Bytes of device workspace `ws` every entry point below needs for this
 * configuration (status word plus any scratch).  batch and max_seq_len are
 * the largest B and L_s (decode) or T (prefill) of the calls that will use
 * it; decode steps need neither (0, 0), sas_gate_backward the batch,
 * sas_prefill_block_sparse and sas_prefill_gate_backward both. */
SAS_API size_t sas_workspace_bytes(const sas_config* cfg, int32_t batch, int32_t max_seq_len);

/* Zero the status word at the start of ws (cudaMemsetAsync on `stream`). */
SAS_API sas_status sas_reset_device_status(void* ws, sas_stream_t stream);

/* Synchronise `stream`, read the status word of ws and return it as a
 * sas_status in *out (SAS_OK, SAS_ERR_DEVICE_BOUNDS or SAS_ERR_TIMEOUT; bounds
 * wins when both bits are set). */
SAS_API sas_status sas_get_device_status(const void* ws, sas_stream_t stream, sas_status* out);

SAS_API const char* sas_status_string(sas_status s);

/* ABI version of this header; bumped on any signature or layout change. */
SAS_API int32_t sas_abi_version(void);

/*
 * Pooling and gate keys (pages: keys pooled per block by max, min and
 * average; Q/K normalisation and gate RoPE on; gate hidden size 128).
 *
 * For each sequence s and KV head h, pools blocks
 *   b = blk_begin[s] .. blk_begin[s] + num_blocks - 1
 * (blk_begin may be NULL: 0 for every sequence), skipping blocks that are not
 * complete (64*(b+1) > L_s) or have b >= max_gate_blocks, and writes
 *   gate_keys[s][h][b][:] = RoPE(RMSNorm(P_b @ W_k[h]) * gamma_k, b)   (fp32)
 *   pooled_raw[s][h][b][:] = P_b = [max ; min ; mean]                 (fp32,
 *   optional, NULL to skip).
 * Call it for new complete blocks as tokens are appended (incremental), or
 * with blk_begin NULL and num_blocks = L/64 after a prefill.
 *   w_k       bf16 [Hkv][384][128]     gamma_k  fp32 [128]
 *   gate_keys fp32 [B][Hkv][MG][128]   pooled_raw fp32 [B][Hkv][MG][384]
 */
SAS_API sas_status sas_pool_keys(const sas_config* cfg, const sas_kv* kv,
                         const int32_t* blk_begin, int32_t num_blocks,
                         const void* w_k, const float* gamma_k,
                         void* gate_keys, int32_t max_gate_blocks,
                         float* pooled_raw, void* ws, size_t ws_bytes,
                         sas_stream_t stream);

/*
 * Gate scores of every historical block (pages: the gate ranks the KV
 * blocks so that the best can be selected; the query side goes through
 * the projection the pages name Qproj).
 *   q            kv_dtype [B][Hq][128]  query of token L_s - 1
 *   w_q          bf16 [Hq][128][128]    gamma_q fp32 [128]
 *   gate_keys    fp32 [B][Hkv][MG][128] (from sas_pool_keys)
 *   head_scores  fp32 [B][Hq][MG]  s_{g,b} for b < c_s (optional, NULL)
 *   group_scores fp32 [B][Hkv][MG] S_b for b < c_s
 * Entries b >= c_s are left untouched.  Requires c_s <= MG.
 */
SAS_API sas_status sas_gate_scores(const sas_config* cfg, const void* q, const int32_t* seq_lens,
                           int32_t batch, const void* w_q, const float* gamma_q,
                           const void* gate_keys, int32_t max_gate_blocks,
                           float* head_scores, float* group_scores,
                           void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * Top-K block selection under the token budget (pages: training Top-K 31,
 * default budget 2,048; 1,024 and 4,096 usable without retraining).
 *   group_scores fp32 [B][Hkv][MG]
 *   token_budgets: NULL (cfg->token_budget for all) or int32 [B], as in sas_kv
 *   sel_idx   int32 [B][Hkv][cfg budget/64]: ascending block ids, the current
 *             block c_s last; entries past sel_count are left untouched
 *   sel_count int32 [B][Hkv] = min(budget_s/64, c_s + 1)
 */
SAS_API sas_status sas_topk_blocks(const sas_config* cfg, const float* group_scores,
                           const int32_t* seq_lens, const int32_t* token_budgets, int32_t batch,
                           int32_t max_gate_blocks, int32_t* sel_idx, int32_t* sel_count,
                           void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * Block-sparse flash-decoding attention over given block lists (the sparse
 * decode backend the pages name for inference).
 *   q    kv_dtype [B][Hq][128]
 *   sel_idx / sel_count as produced by sas_topk_blocks (any ascending list of
 *   blocks <= c_s whose last entry is c_s is accepted)
 *   out  out_dtype [B][Hq][128]
 */
SAS_API sas_status sas_sparse_decode(const sas_config* cfg, const void* q, const sas_kv* kv,
                             const int32_t* sel_idx, const int32_t* sel_count,
                             void* out, void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * Fused decode step (pages: for each decoded token the gate ranks the
 * historical blocks, the best are kept under the token budget with the
 * current block, and attention runs over those blocks only; aigc.news
 * release paragraph of 2026-09-14): gate query, scores, Top-K and
 * block-sparse attention in
 * one launch (one thread-block cluster per (sequence, KV head); the cluster's
 * CTAs split the gate keys and the selected blocks and merge through
 * distributed shared memory).
 *   q, w_q, gamma_q, gate_keys as for sas_gate_scores (q and gamma_q 16-byte
 *   aligned); out as for sas_sparse_decode.
 *   w_k, gamma_k: optional (both NULL or both set).  When set, and the decoded
 *   token completes its block (L_s % 64 == 0) and c_s < max_gate_blocks, the
 *   step also writes gate_keys[s][h][c_s] -- the gate key of that block, as
 *   sas_pool_keys computes it -- so decoding maintains the gate keys without
 *   a separate launch.  Row c_s is not read by the same step.
 *   sel_idx, sel_count, group_scores: optional outputs (NULL to skip), layouts
 *   as above.
 */
SAS_API sas_status sas_decode_step(const sas_config* cfg, const void* q, const sas_kv* kv,
                                   const void* w_q, const float* gamma_q, const void* w_k,
                                   const float* gamma_k, void* gate_keys,
                                   int32_t max_gate_blocks, void* out, int32_t* sel_idx,
                                   int32_t* sel_count, float* group_scores, void* ws,
                                   size_t ws_bytes, sas_stream_t stream);

/*
 * The fused decode step with the query and the output in host memory.  The
 * release pages have no counterpart: the operation is sas_decode_step's, for
 * a serving loop that makes one call per step: enqueues on `stream` the move of
 * q_host into q_dev, sas_decode_step on q_dev, and the move of the output
 * into out_host.  out_host holds the step's output once the stream has
 * passed this call (synchronise on the stream, or on an event recorded after
 * the call).
 *   q_host   host memory, kv_dtype [B][Hq][128]
 *   q_dev    device memory of the same size, 16-byte aligned (overwritten
 *            when q_host is pageable, else untouched)
 *   out_dev  device memory, out_dtype [B][Hq][128] (overwritten when
 *            out_host is pageable, else untouched)
 *   out_host host memory of the same size
 * Page-locked host memory (cudaHostAlloc, cudaHostRegister) that the
 * stream's device can address moves without the copy engine: the step
 * kernel reads q_host over the host link (a 16-byte aligned q_host; each
 * byte crosses the link once) and writes its output rows straight into
 * out_host.  It may read q_host before kernels ahead of it on the stream
 * have finished, so q_host must hold the query when the call is made and
 * must not be written by device work enqueued before the call.  Pageable
 * memory takes a runtime copy instead (the CUDA runtime stages it; the call
 * may block until the copy is done).  The host buffers are the caller's and must stay valid
 * until the stream has passed the call.  Every other argument is that of
 * sas_decode_step.  All arguments are checked before anything is enqueued
 * (a bad one enqueues nothing); SAS_ERR_CUDA from a copy or a launch leaves
 * what was enqueued before it in place.
 */
SAS_API sas_status sas_decode_step_host(const sas_config* cfg, const void* q_host, void* q_dev,
                                        const sas_kv* kv, const void* w_q, const float* gamma_q,
                                        const void* w_k, const float* gamma_k, void* gate_keys,
                                        int32_t max_gate_blocks, void* out_dev, void* out_host,
                                        int32_t* sel_idx, int32_t* sel_count,
                                        float* group_scores, void* ws, size_t ws_bytes,
                                        sas_stream_t stream);

/*
 * Block-sparse chunked prefill (pages: training Top-K 31 historical blocks
 * over 32,768-token sequences, 64-token blocks, gate with Qproj, Q/K
 * normalisation and gate RoPE).  For every 64-token query block i of every
 * sequence and KV head: gate query = per-head mean of the block's 64 queries
 * through Qproj, RMSNorm and RoPE at position i; group scores against the
 * gate keys of blocks b < i; the min(budget/64 - 1, i) best blocks plus block
 * i; token t of block i attends to all tokens of the kept blocks and to
 * tokens 64i..t of its own block.
 *   token_budgets: NULL (cfg->token_budget for every sequence) or int32 [B]
 *   per-sequence budgets, each a multiple of 64 in 64 .. cfg->token_budget
 *   (cfg->token_budget sizes the lists and the workspace).  A sequence with
 *   a bad budget is skipped (its out rows set to 0, sel_count 0) and reported as
 *   SAS_ERR_DEVICE_BOUNDS.
 *   q      bf16 [B][Hq][T][128]      k, v bf16 [B][Hkv][T][128]
 *   out    bf16 [B][Hq][T][128]      (all 16-byte aligned)
 *   w_q, gamma_q, w_k, gamma_k as for the decode entry points.
 *   gate_keys [B][Hkv][MG][128] (output; fp32, bf16 when cfg->gate_keys_bf16):
 *   rows 0..T/64-1 are written, so decoding can continue from them.
 *   MG >= T/64.
 *   sel_idx int32 [B][Hkv][T/64][budget/64], sel_count int32 [B][Hkv][T/64]:
 *   optional outputs (NULL to skip), the block list of every query block.
 *   ws: 256-byte aligned, at least sas_workspace_bytes(cfg, B, T) bytes
 *   (gate queries and block lists live there).
 * This build requires bf16 inputs and output and T a multiple of 64; other
 * requests return SAS_ERR_UNSUPPORTED.  Budgets up to the configuration's
 * limit of 16,384 tokens and GQA groups of 1 to 8 heads are handled (the
 * tensor-core tile holds two query heads; an odd group's last tile one).
 */
SAS_API sas_status sas_prefill_block_sparse(const sas_config* cfg, const void* q, const void* k,
                                            const void* v, int32_t batch, int32_t seq_len,
                                            const int32_t* token_budgets,
                                            const void* w_q, const float* gamma_q,
                                            const void* w_k, const float* gamma_k,
                                            void* gate_keys, int32_t max_gate_blocks, void* out,
                                            int32_t* sel_idx, int32_t* sel_count, void* ws,
                                            size_t ws_bytes, sas_stream_t stream);

/*
 * Gradient through the gates (pages: the continuous gates on the selected
 * blocks let a gradient reach the gate despite the discrete Top-K;
 * aigc.news release paragraph of 2026-09-14).  For the gated decode step
 * (cfg->gate_mode = SAS_GATE_LOGSIGMOID_BIAS) with the block lists held fixed
 * and an upstream gradient d_out of its output, ADDS to
 *   dw_q     fp32 [Hq][128][128]   dL/dW_q
 *   dw_k     fp32 [Hkv][384][128]  dL/dW_k
 *   dgamma_q fp32 [128]            dL/dgamma_q
 *   dgamma_k fp32 [128]            dL/dgamma_k
 * (zero them first for a fresh gradient; the sums over sequences and block
 * list entries run in a fixed order, so repeated calls add identical values).
 * The gate of a selected
 * historical block b for query head g is log(sigmoid(s_gb)) on its tokens'
 * logits; its gradient reaches W_q and gamma_q through the gate query (q_g
 * @ W_q[g], RMSNorm, gain, RoPE at the current block) and W_k and gamma_k
 * through the gate key of b (pooled block @ W_k, RMSNorm, gain, RoPE at b),
 * recomputed here from the cache.  The Top-K itself has no gradient.  In the
 * select-only mode the gate parameters get no gradient: the call returns
 * SAS_OK and enqueues nothing.
 *   q        bf16 [B][Hq][128], the step's queries
 *   kv       the cache the step read (bf16)
 *   sel_idx, sel_count: the block lists of the step (as sas_decode_step
 *            returns them); a list that is not ascending, does not end with
 *            the current block or names a block outside the cache skips its
 *            (sequence, KV head) and sets SAS_ERR_DEVICE_BOUNDS's bit
 *   d_out    fp32 [B][Hq][128]  dL/dout
 *   ws       at least sas_workspace_bytes(cfg, B, 0) bytes (per-pair terms
 *            that a second kernel sums into the gradients), else
 *            SAS_ERR_WORKSPACE
 * This build handles budgets up to 4,096 tokens (lists of up to 64 blocks)
 * and bf16 caches; others return SAS_ERR_UNSUPPORTED.
 */
SAS_API sas_status sas_gate_backward(const sas_config* cfg, const void* q, const sas_kv* kv,
                                     const void* w_q, const float* gamma_q, const void* w_k,
                                     const float* gamma_k, const int32_t* sel_idx,
                                     const int32_t* sel_count, const float* d_out, float* dw_q,
                                     float* dw_k, float* dgamma_q, float* dgamma_k, void* ws,
                                     size_t ws_bytes, sas_stream_t stream);

/*
 * Gradient through the gates of the gated block-sparse prefill (pages: the
 * continuous gates on the selected blocks let a gradient reach the gate past
 * the discrete Top-K selection; aigc.news release paragraph of 2026-09-14).
 * For sas_prefill_block_sparse in the gated mode (cfg->gate_mode =
 * SAS_GATE_LOGSIGMOID_BIAS), its block lists held fixed, and an upstream
 * gradient d_out of its output, ADDS to dw_q, dw_k, dgamma_q and dgamma_k
 * (shapes as for sas_gate_backward; zero them first for a fresh gradient;
 * every sum runs in a fixed order, so repeated calls add identical values).
 * Query block i of head g carries the gate log(sigmoid(s_gib)) on the tokens
 * of each selected historical block b, s_gib = q~_gi . k~_b * gate_scale with
 * q~_gi from the mean of the block's 64 queries (q_bar @ W_q[g], RMSNorm,
 * gain, RoPE at i); the gradient reaches W_q and gamma_q through every
 * query block's gate query and W_k and gamma_k through the gate keys (pooled
 * block @ W_k, RMSNorm, gain, RoPE at b, recomputed from the cache), summed
 * over the query blocks that kept each key block.  The select-only mode
 * gives no gradient: the call returns SAS_OK and enqueues nothing.
 *   q, k, v     bf16, as for sas_prefill_block_sparse (16-byte aligned)
 *   gate_keys   fp32 [B][Hkv][max_gate_blocks][128], the keys the forward
 *               wrote (scores are recomputed from them); cfg->gate_keys_bf16
 *               must be 0
 *   sel_idx, sel_count: the forward's block lists [B][Hkv][T/64][budget/64]
 *               and lengths [B][Hkv][T/64]; a list that is not ascending or
 *               does not end with its query block skips that query block
 *               and sets SAS_ERR_DEVICE_BOUNDS's bit
 *   d_out       fp32 [B][Hq][T][128]  dL/dout (16-byte aligned)
 *   ws          at least sas_workspace_bytes(cfg, B, T) bytes
 * This build handles bf16 inputs, T a multiple of 64 and budgets up to
 * 4,096 tokens; others return SAS_ERR_UNSUPPORTED.
 */
SAS_API sas_status sas_prefill_gate_backward(const sas_config* cfg, const void* q, const void* k, const void* v,
                                             int32_t batch, int32_t seq_len, const void* w_q,
                                             const float* gamma_q, const void* w_k, const float* gamma_k,
                                             const void* gate_keys, int32_t max_gate_blocks,
                                             const int32_t* sel_idx, const int32_t* sel_count,
                                             const float* d_out, float* dw_q, float* dw_k, float* dgamma_q,
                                             float* dgamma_k, void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * Allocation-free variant of sas_decode_step.  The release pages have no
 * counterpart: this exists for callers that cannot allocate device memory
 * (a serving loop that must not allocate after warm-up, a plugin whose host
 * framework owns all GPU memory, a C caller without an allocator) and so
 * cannot provide the workspace `ws`.
 *   Same arguments and results as sas_decode_step, minus ws / ws_bytes.  The
 *   scratch (the device status word) lives in a 256-byte file-scope device
 *   array of the library that every GPU loading the library keeps until exit.
 *   status_out: optional device uint32; receives the status bits of this call
 *   (bit 0: out-of-range length / page / block, bit 1: a bounded wait timed
 *   out; 0 when clean).
 *   The first call on a device looks up the array's device address; make it
 *   before any CUDA stream capture.  Every call clears the status word first;
 *   calls that overlap on the GPU share the array and race on it.  A build
 *   whose scratch need exceeds 256 bytes is refused with SAS_ERR_WORKSPACE.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
SAS_API sas_status sas_decode_step_static(const sas_config* cfg, const void* q, const sas_kv* kv,
                                          const void* w_q, const float* gamma_q, const void* w_k,
                                          const float* gamma_k, void* gate_keys,
                                          int32_t max_gate_blocks, void* out, int32_t* sel_idx,
                                          int32_t* sel_count, float* group_scores,
                                          uint32_t* status_out, sas_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SAS_H_ */
