// SAS block-sparse chunked prefill.
//
// Method (release pages: "Tencent released Simple-Attention-Sparsification
// ..." aigc.news 2026-09-14, release paragraph: training Top-K 31 historical
// blocks over 32,768-token sequences, 64-token blocks, gate with Qproj, Q/K
// normalisation and gate RoPE): for every 64-token query block i of a
// sequence and every KV head h,
//   q~_g = RoPE(RMSNorm(mean_t q_{g,t} @ W_q[g]) * gamma_q, i)   (g in the group)
//   S_b  = mean_g(q~_g . k~_b) * gate_scale                    (b < i)
//   keep the min(topk_s, i) blocks of largest S_b (ties: lower index) + block
//   i, topk_s = budget_s / 64 - 1 (one budget per sequence, or the
//   configured one); token t of block i attends to every token of the kept
//   blocks and to the tokens of block i up to t (causal); gated mode: the
//   logits of a kept historical block b for head g get + log(sigmoid(s_gb)),
//   s_gb = q~_g . k~_b * gate_scale.
//
// Kernels:
//   prefill_gate_query_kernel  q~ for every (sequence, query head, block):
//                              W_q[g] staged in shared memory once per CTA,
//                              16 blocks projected at once.
//   prefill_select_kernel      scores and exact Top-K per (seq, head, block).
//   prefill_attn_kernel        tcgen05 block-sparse attention (gated mode: a
//                              second instance): one CTA per
//                              (seq, KV head, query block, pair of query
//                              heads); the 128 query rows (2 heads x 64
//                              tokens) are the M dimension of
//                              S = Q K^T (N = 64 keys) and O += P V (N = 128),
//                              accumulators in tensor memory.
#include "sas_internal.h"
#include "sas_select.cuh"

namespace sas {

// ------------------------------------------------------------ gate queries
// grid (ceil(nblk / kPfQb), Hq, B), 128 threads; one CTA per kPfQb query
// blocks of one (sequence, query head).
//   A. block sums: warp w sums the 64 queries of blocks w, w + 4, ... (lane:
//      16-byte column chunk lane % 16, rows of parity lane / 16; 16 rows'
//      loads in flight per lane), into qm[dim][block];
//   B. u = mean @ W_q[g] for all the CTA's blocks at once, thread d owning
//      output dimension d (W_q read from shared memory once per CTA);
//   C. RMSNorm (gain gamma_q) and gate RoPE at each block's index.
__global__ void __launch_bounds__(kThreads) prefill_gate_query_kernel(const __grid_constant__ PrefillParams p) {
  constexpr int NB = kPfQb;
  const int g = blockIdx.y;
  const int s = blockIdx.z;
  const int i0 = blockIdx.x * NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* wq = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // [128][128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + kDim * kDim * 2);
  __shared__ __align__(16) float qm[kDim][NB];  // block sums, [dim][block]
  __shared__ float xs[NB][kDim];                // normalised u, [block][dim]
  __shared__ float ssq[kWarps][NB];
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, kDim * kDim * 2);
    bulk_g2s(wq, p.w_q + static_cast<size_t>(g) * kDim * kDim, kDim * kDim * 2, bar);
  }
  const int nb = min(NB, p.nblk - i0);  // blocks of this CTA (>= 1)

  // ---- A. sums of the 64 queries of each block
  {
    const int cvec = lane & 15, par = lane >> 4;
    for (int bi = warp; bi < NB; bi += kWarps) {  // warp-uniform
      float acc[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[v] = 0.f;
      if (bi < nb) {
        const __nv_bfloat16* qb =
            p.q + ((static_cast<size_t>(s) * p.hq + g) * p.T + static_cast<size_t>(i0 + bi) * kBlock + par) * kDim +
            cvec * 8;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint4 raw[16];
#pragma unroll
          for (int r = 0; r < 16; ++r)
            raw[r] = *reinterpret_cast<const uint4*>(qb + static_cast<size_t>(2 * (16 * half + r)) * kDim);
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const uint32_t u[4] = {raw[r].x, raw[r].y, raw[r].z, raw[r].w};
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              acc[2 * v] += bf16_lo(u[v]);
              acc[2 * v + 1] += bf16_hi(u[v]);
            }
          }
        }
      }
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], 16);
      if (par == 0) {
#pragma unroll
        for (int v = 0; v < 8; ++v) qm[cvec * 8 + v][bi] = acc[v];
      }
    }
  }
  __syncthreads();
  const bool ok = mbar_wait(bar, 0, p.status);

  // ---- B. u_b[d] = (sum_b / 64) . W_q[:, d]
  const int d = tid;
  float u[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) u[b] = 0.f;
  if (ok) {
#pragma unroll 4
    for (int r = 0; r < kDim; ++r) {
      const float w = __bfloat162float(wq[r * kDim + d]);
      const float4* m4 = reinterpret_cast<const float4*>(&qm[r][0]);
#pragma unroll
      for (int c = 0; c < NB / 4; ++c) {
        const float4 x = m4[c];
        u[4 * c] = fmaf(x.x, w, u[4 * c]);
        u[4 * c + 1] = fmaf(x.y, w, u[4 * c + 1]);
        u[4 * c + 2] = fmaf(x.z, w, u[4 * c + 2]);
        u[4 * c + 3] = fmaf(x.w, w, u[4 * c + 3]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) u[b] *= (1.f / kBlock);  // a power of two: exact

  // ---- C. RMSNorm and RoPE per block
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float sq = u[b] * u[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) ssq[warp][b] = sq;
  }
  __syncthreads();
  const float gam = p.gamma_q[d];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const float tot = ssq[0][b] + ssq[1][b] + ssq[2][b] + ssq[3][b];
    xs[b][d] = u[b] * (1.f / sqrtf(tot / kDim + p.eps)) * gam;
  }
  __syncthreads();
  for (int b = 0; b < nb; ++b) {
    const int i = i0 + b;
    float cs, sn;
    rope_cos_sin(p.rope.theta_over_pi[d & 63], i, cs, sn);
    const float y = (d < 64) ? xs[b][d] * cs - xs[b][d + 64] * sn : xs[b][d] * cs + xs[b][d - 64] * sn;
    p.qt[((static_cast<size_t>(s) * p.hq + g) * p.nblk + i) * kDim + d] = y;
  }
}

// ------------------------------------------------------------ selection
// grid (nblk, Hkv, B), 128 threads.
// kPfSelQb consecutive query blocks per CTA: every gate-key row is loaded
// once and scored against their kPfSelQb group-mean gate queries, then the
// exact selection runs for each query block in turn.  One: with four the
// kernel took 125 us instead of 107 us per 32k-token sequence (the exact
// selection, not the gate-key reads, bounds it, and a quarter of the CTAs
// run it).
constexpr int kPfSelQb = 1;

template <bool kMedium>
__global__ void __launch_bounds__(kThreads) prefill_select_kernel(const __grid_constant__ PrefillParams p) {
  const int i0 = blockIdx.x * kPfSelQb;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;
  const int nq = min(kPfSelQb, p.nblk - i0);  // query blocks of this CTA
  const size_t base0 = (static_cast<size_t>(s) * p.hkv + h) * p.nblk + i0;
  // this sequence's Top-K: budget / 64 - 1; a bad budget skips the sequence
  // (empty lists, which the attention kernel reports and skips as well)
  int topk = p.topk;
  if (p.token_budgets != nullptr) {
    const int b = p.token_budgets[s];
    topk = (b >= kBlock && b <= p.max_sel * kBlock && b % kBlock == 0) ? b / kBlock - 1 : -1;
  }
  if (topk < 0) {
    if (tid == 0) raise_status(p.status, kStatusBounds);
    if (tid < nq) {
      p.cnt[base0 + tid] = 0;
      if (p.cnt_out != nullptr) p.cnt_out[base0 + tid] = 0;
    }
    return;
  }
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* vals = reinterpret_cast<float*>(smem_raw);  // [kPfSelQb][nblk]
  const int vstride = (p.nblk + 3) / 4 * 4;
  uint8_t* q = smem_raw + (kPfSelQb * vstride * 4 + 15) / 16 * 16;
  int* sel = reinterpret_cast<int*>(q);
  q += (p.max_sel * 4 + 15) / 16 * 16;
  uint32_t* hist = reinterpret_cast<uint32_t*>(q);
  q += kSelBins * 4;
  uint32_t* selbits = reinterpret_cast<uint32_t*>(q);
  q += ((p.nblk + 31) / 32 * 4 + 15) / 16 * 16;
  int* scan = reinterpret_cast<int*>(q);
  q += 16 * 4;
  float* qbar = reinterpret_cast<float*>(q);  // [kPfSelQb][128]
  // S_b = mean_g(q~_g . k~_b) * scale = (scale/G * sum_g q~_g) . k~_b
  for (int x = tid; x < kPfSelQb * kDim; x += kThreads) {
    const int qq = x / kDim, d = x - qq * kDim;
    float a = 0.f;
    if (qq < nq)
      for (int g = 0; g < G; ++g)
        a += p.qt[((static_cast<size_t>(s) * p.hq + h * G + g) * p.nblk + i0 + qq) * kDim + d];
    qbar[x] = a * (p.gate_scale / static_cast<float>(G));
  }
  __syncthreads();
  const int grp = lane >> 3, sub = lane & 7;
  const size_t gk_base = (static_cast<size_t>(s) * p.hkv + h) * p.mg * kDim;  // elements
  const int ilast = i0 + nq - 1;  // the last query block scores blocks 0 .. ilast - 1
  for (int b0 = 0; b0 < ilast; b0 += 16) {
    const int b = b0 + warp * 4 + grp;
    float kr[16];
    if (b < ilast) {
      const size_t off = gk_base + static_cast<size_t>(b) * kDim + sub * 16;
      if (p.gk16) {
        const uint4* row = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.gate_keys) + off);
        const uint4 r0 = row[0], r1 = row[1];
        const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          kr[2 * k] = bf16_lo(w[k]);
          kr[2 * k + 1] = bf16_hi(w[k]);
        }
      } else {
        const float4* row = reinterpret_cast<const float4*>(static_cast<const float*>(p.gate_keys) + off);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 v = row[k];
          kr[4 * k] = v.x;
          kr[4 * k + 1] = v.y;
          kr[4 * k + 2] = v.z;
          kr[4 * k + 3] = v.w;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) kr[k] = 0.f;
    }
#pragma unroll
    for (int qq = 0; qq < kPfSelQb; ++qq) {
      const float4* qv = reinterpret_cast<const float4*>(qbar + qq * kDim + sub * 16);
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 qk = qv[k];
        acc = fmaf(qk.x, kr[4 * k], acc);
        acc = fmaf(qk.y, kr[4 * k + 1], acc);
        acc = fmaf(qk.z, kr[4 * k + 2], acc);
        acc = fmaf(qk.w, kr[4 * k + 3], acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (b < i0 + qq && sub == 0) vals[qq * vstride + b] = acc;
    }
  }
  __syncthreads();
  for (int qq = 0; qq < nq; ++qq) {
    const int i = i0 + qq;
    const size_t base = base0 + qq;
    const int m = select_blocks<kMedium>(vals + qq * vstride, i, topk, i, sel, hist, selbits, scan);
    for (int j = tid; j < m; j += kThreads) {
      p.sel[base * p.max_sel + j] = sel[j];
      if (p.sel_out != nullptr) p.sel_out[base * p.max_sel + j] = sel[j];
    }
    if (tid == 0) {
      p.cnt[base] = m;
      if (p.cnt_out != nullptr) p.cnt_out[base] = m;
    }
    __syncthreads();  // sel and the selection scratch are reused by the next query block
  }
}

size_t prefill_select_smem_bytes(int nblk, int max_sel) {
  return static_cast<size_t>((kPfSelQb * ((nblk + 3) / 4 * 4) * 4 + 15) / 16 * 16 + (max_sel * 4 + 15) / 16 * 16 +
                             kSelBins * 4 + ((nblk + 31) / 32 * 4 + 15) / 16 * 16 + 16 * 4 + kPfSelQb * kDim * 4);
}

// ------------------------------------------------------------ tcgen05 attention
// 160 threads: warps 0-3 own one query row each per thread (softmax, O
// rescaling, epilogue); warp 4 lane 0 issues the TMA copies and the MMAs.
// Shared memory (1024-aligned): Q 32 KiB | K ring 3 x 16 KiB | V ring 2 x 16 KiB
// | barriers | block list.  Tensor memory, 256 columns: two S buffers of 64
// fp32 columns and O (128 columns).  The softmax writes P_e as bf16 pairs over
// the first 32 columns of S buffer e % 2, and P V reads it from there (A
// operand in tensor memory), so P never goes through shared memory and the
// softmax of tile e + 1 does not wait for P V of tile e.
//
// Per tile e (m tiles, ascending block ids, the diagonal block last):
//   QK_e    S[e%2] = Q K_e^T          needs K_e and P V_{e-2} done (S[e%2] free)
//   soft_e  P_e = exp2(S log2e/sqrt(d) - m), into S[e%2]; O *= alpha when the
//           running maximum grew by more than 2^8 (then after P V_{e-1})
//   PV_e    O += P_e V_e              needs soft_e and V_e
// The issuer runs PV_e, waits for it, then QK_{e+2}; soft_{e+1} overlaps both.
constexpr int kPfAttnThreads = 160;
constexpr uint32_t kPfTmemCols = 256;
constexpr int kPfKStages = 3, kPfVStages = 2;
constexpr int kPfSmemQ = 0, kPfSmemK = 32768, kPfSmemV = kPfSmemK + kPfKStages * 16384,
              kPfSmemBars = kPfSmemV + kPfVStages * 16384;
enum { kBarQ = 0, kBarK0 = 1, kBarV0 = kBarK0 + kPfKStages, kBarS0 = kBarV0 + kPfVStages,
       kBarP0 = kBarS0 + 2, kBarO = kBarP0 + 2, kNumPfBars = kBarO + 1 };

size_t prefill_attn_smem_bytes(int max_sel) {
  // barriers, TMEM slot, block list, gates of the list for the CTA's 2 heads
  return static_cast<size_t>(kPfSmemBars + kNumPfBars * 8 + 16 + max_sel * 4 + max_sel * 2 * 4);
}

// Tracing builds: the issuer and softmax thread 0 add up the SM cycles they
// spend in each wait and phase; CTA k < kTraceCtas writes them to slots of
// trace row k.  Ordinary builds compile the hooks out.
#ifdef SAS_PHASE_TRACE
#define PF_TIC(v) const long long v = clock64()
#define PF_TOC(acc, v) (acc) += clock64() - (v)
#else
#define PF_TIC(v) \
  do {            \
  } while (0)
#define PF_TOC(acc, v) \
  do {                 \
  } while (0)
#endif

// kGated: the gated mode (a separate instance, so that the select-only
// softmax loop carries no gate load)
template <bool kGated>
__global__ void __launch_bounds__(kPfAttnThreads, 2)
    prefill_attn_kernel(const __grid_constant__ PrefillParams p,
                        const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int npair = (p.G + 1) / 2;
  int idx = static_cast<int>(blockIdx.x);
  const int pair = idx % npair;
  idx /= npair;
  const int h = idx % p.hkv;
  idx /= p.hkv;
  const int s = idx % p.batch;
  const int i = p.nblk - 1 - idx / p.batch;  // longest block lists first
  const int g0 = h * p.G + 2 * pair;
  // an odd group's last tile holds one head: rows 64..127 repeat it and are
  // not stored
  const bool lone = 2 * pair + 1 >= p.G;
#ifdef SAS_PHASE_TRACE
  unsigned long long* trc =
      (p.trace != nullptr && blockIdx.x < static_cast<unsigned>(kTraceCtas)) ? p.trace + blockIdx.x * kTraceSlots : nullptr;
  const unsigned long long t_start = global_timer_ns();
  long long acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#endif

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kPfSmemBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumPfBars);
  int* sel_s = reinterpret_cast<int*>(tmem_slot + 4);
  float* gb_s = reinterpret_cast<float*>(sel_s + p.max_sel);  // gated mode: gates [entry][2 heads]
  // the plan assumes a 1024-byte aligned dynamic shared window (swizzled
  // TMA boxes and UMMA descriptors); anything else is reported, not used
  const bool misaligned = (smem_u32(base) & 1023u) != 0;

  const size_t lbase = (static_cast<size_t>(s) * p.hkv + h) * p.nblk + i;
  bool err = misaligned;
  int m = 0;
  if (!err) {
    m = p.cnt[lbase];
    if (m < 1 || m > p.max_sel) err = true;
  }
  if (!err) {
    const int32_t* sl = p.sel + lbase * p.max_sel;
    for (int j = tid; j < m; j += kPfAttnThreads) {
      const int b = sl[j];
      sel_s[j] = b;
      if (b < 0 || b > i || (j == m - 1 && b != i) || (j > 0 && sl[j - 1] >= b)) err = true;
    }
  }
  if (tid == 0 && !misaligned) {
    for (int b = 0; b < kNumPfBars; ++b)
      mbar_init(&bars[b], (b == kBarP0 || b == kBarP0 + 1) ? 128u : 1u);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  const bool bad = __syncthreads_or(err) != 0;
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (bad && tid == 0) raise_status(p.status, kStatusBounds);
  if (bad) m = 0;

  uint8_t* sQ = base + kPfSmemQ;
  uint8_t* sK = base + kPfSmemK;
  uint8_t* sV = base + kPfSmemV;
  const float sl2 = p.attn_scale_log2;

  if (warp == 4) {
    if (lane == 0 && m > 0) {
      // ---------------------------------------------------- producer / MMA issuer
#ifdef SAS_PHASE_TRACE
      const long long t_prod0 = clock64();
#endif
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, false, true);
      // descriptors of the stage-0 operands; later k-steps and stages add
      // their byte offset >> 4 to the start-address field
      const uint64_t dQ = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = umma_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV = umma_desc_sw128(smem_u32(sV), 8192, 1024);
      const int rowq0 = static_cast<int>((static_cast<size_t>(s) * p.hq + g0) * p.T) + kBlock * i;
      const int rowq1 = lone ? rowq0 : rowq0 + p.T;
      const int rowkv = static_cast<int>((static_cast<size_t>(s) * p.hkv + h) * p.T);
      mbar_arrive_expect_tx(&bars[kBarQ], 32768);
      tma_load_2d(sQ + 0, &tmq, 0, rowq0, &bars[kBarQ]);
      tma_load_2d(sQ + 8192, &tmq, 0, rowq1, &bars[kBarQ]);
      tma_load_2d(sQ + 16384, &tmq, 64, rowq0, &bars[kBarQ]);
      tma_load_2d(sQ + 24576, &tmq, 64, rowq1, &bars[kBarQ]);
      auto load_k = [&](int e) {
        const int st = e % kPfKStages;
        mbar_arrive_expect_tx(&bars[kBarK0 + st], 16384);
        const int row = rowkv + kBlock * sel_s[e];
        tma_load_2d(sK + st * 16384, &tmk, 0, row, &bars[kBarK0 + st]);
        tma_load_2d(sK + st * 16384 + 8192, &tmk, 64, row, &bars[kBarK0 + st]);
      };
      auto load_v = [&](int e) {
        const int st = e % kPfVStages;
        mbar_arrive_expect_tx(&bars[kBarV0 + st], 16384);
        const int row = rowkv + kBlock * sel_s[e];
        tma_load_2d(sV + st * 16384, &tmv, 0, row, &bars[kBarV0 + st]);
        tma_load_2d(sV + st * 16384 + 8192, &tmv, 64, row, &bars[kBarV0 + st]);
      };
      auto issue_qk = [&](int e) {  // K_e has landed, S[e % 2] is free
        const int st = e % kPfKStages;
        PF_TIC(tk);
        mbar_wait(&bars[kBarK0 + st], (e / kPfKStages) & 1, p.status);
        PF_TOC(acc[3], tk);
        tc_fence_after_sync();
        PF_TIC(tiq);
        const uint64_t dk = dK + static_cast<uint64_t>(st * (16384 >> 4));
        const uint32_t d_tmem = tmem + (e & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ss(d_tmem, dQ + static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                       dk + static_cast<uint64_t>(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), idesc_qk, kk > 0);
        umma_commit(&bars[kBarS0 + (e & 1)]);
        PF_TOC(acc[6], tiq);
      };
      for (int e = 0; e < m && e < kPfKStages; ++e) load_k(e);
      for (int e = 0; e < m && e < kPfVStages; ++e) load_v(e);
      PF_TIC(tq);
      mbar_wait(&bars[kBarQ], 0, p.status);
      PF_TOC(acc[4], tq);
      issue_qk(0);
      if (m > 1) issue_qk(1);
      for (int e = 0; e < m; ++e) {
        // P_e written (and so S_e read, Q K_e done: its K slot is free)
        PF_TIC(tp);
        mbar_wait(&bars[kBarP0 + (e & 1)], (e >> 1) & 1, p.status);
        PF_TOC(acc[0], tp);
        if (e + kPfKStages < m) load_k(e + kPfKStages);
        PF_TIC(tv);
        mbar_wait(&bars[kBarV0 + e % kPfVStages], (e / kPfVStages) & 1, p.status);
        PF_TOC(acc[1], tv);
        tc_fence_after_sync();
        PF_TIC(tip);
        const uint32_t aP = tmem + (e & 1) * 64;
        const uint64_t dv = dV + static_cast<uint64_t>((e % kPfVStages) * (16384 >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ts(tmem + 128, aP + kk * 8, dv + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                       e > 0 || kk > 0);
        umma_commit(&bars[kBarO]);
        PF_TOC(acc[5], tip);
        if (e + 2 < m) {
          PF_TIC(to);
          mbar_wait(&bars[kBarO], e & 1, p.status);  // P V_e done: V slot and S[e % 2] free
          PF_TOC(acc[2], to);
          if (e + kPfVStages < m) load_v(e + kPfVStages);
          issue_qk(e + 2);
        }
      }
      mbar_wait(&bars[kBarO], (m - 1) & 1, p.status);  // nothing of ours in flight at teardown
#ifdef SAS_PHASE_TRACE
      if (trc != nullptr) {
        for (int k = 0; k < 5; ++k) trc[2 + k] = static_cast<unsigned long long>(acc[k]);
        trc[12] = static_cast<unsigned long long>(acc[5]);
        trc[13] = static_cast<unsigned long long>(acc[6]);
        trc[14] = static_cast<unsigned long long>(clock64() - t_prod0);
      }
#endif
    }
  } else {
    // ------------------------------------------------------ softmax / epilogue
    const int r = tid;            // query row: head g0 + (r >> 6), token r & 63
    const int t = r & 63;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    float m_run = -INFINITY, l_run = 0.f;  // running maximum in log2 units, row sum
    if (kGated && m > 0) {
      // gated mode: gate log(sigmoid(q~_g(i) . k~_b * gate_scale)) of every kept
      // historical block b for the CTA's two heads, computed while the first
      // Q / K copies and S tile are in flight.  Eight lanes per block (16
      // dimensions each), 16 blocks per pass; the diagonal block gets 0.
      const int grp = lane >> 3, sub = lane & 7;
      const float4* qa = reinterpret_cast<const float4*>(
          p.qt + ((static_cast<size_t>(s) * p.hq + g0) * p.nblk + i) * kDim + sub * 16);
      const float4* qb = qa + (lone ? 0 : static_cast<size_t>(p.nblk) * (kDim / 4));  // head g0 + 1
      float4 q0[4], q1[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        q0[c] = qa[c];
        q1[c] = qb[c];
      }
      const size_t gk_base = (static_cast<size_t>(s) * p.hkv + h) * p.mg * kDim + sub * 16;  // elements
      for (int j0 = 0; j0 < m - 1; j0 += 16) {
        const int j = j0 + 4 * warp + grp;
        const bool ok = j < m - 1;
        float kr[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) kr[x] = 0.f;
        if (ok) {
          const size_t off = gk_base + static_cast<size_t>(sel_s[j]) * kDim;
          if (p.gk16) {
            const uint4* row = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.gate_keys) + off);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 w = row[c];
              const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                kr[8 * c + 2 * x] = bf16_lo(u[x]);
                kr[8 * c + 2 * x + 1] = bf16_hi(u[x]);
              }
            }
          } else {
            const float4* row = reinterpret_cast<const float4*>(static_cast<const float*>(p.gate_keys) + off);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 w = row[c];
              kr[4 * c] = w.x;
              kr[4 * c + 1] = w.y;
              kr[4 * c + 2] = w.z;
              kr[4 * c + 3] = w.w;
            }
          }
        }
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          a0 = fmaf(q0[c].x, kr[4 * c], fmaf(q0[c].y, kr[4 * c + 1], fmaf(q0[c].z, kr[4 * c + 2], fmaf(q0[c].w, kr[4 * c + 3], a0))));
          a1 = fmaf(q1[c].x, kr[4 * c], fmaf(q1[c].y, kr[4 * c + 1], fmaf(q1[c].z, kr[4 * c + 2], fmaf(q1[c].w, kr[4 * c + 3], a1))));
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          a0 += __shfl_xor_sync(0xffffffffu, a0, o);
          a1 += __shfl_xor_sync(0xffffffffu, a1, o);
        }
        if (ok && sub == 0) {
          const float s0 = a0 * p.gate_scale, s1 = a1 * p.gate_scale;
          gb_s[2 * j] = (s0 >= 0.f) ? -log1pf(expf(-s0)) : s0 - log1pf(expf(s0));
          gb_s[2 * j + 1] = (s1 >= 0.f) ? -log1pf(expf(-s1)) : s1 - log1pf(expf(s1));
        }
      }
      if (tid < 2) gb_s[2 * (m - 1) + tid] = 0.f;
      named_bar_sync(1, 128);  // the four softmax warps
    }
    for (int e = 0; e < m; ++e) {
      PF_TIC(ts);
      mbar_wait(&bars[kBarS0 + (e & 1)], (e >> 1) & 1, p.status);
      PF_TOC(acc[5], ts);
      PF_TIC(tc);
      tc_fence_after_sync();
      float sv[64];
      tmem_ld32(tl + (e & 1) * 64, sv);
      tmem_ld32(tl + (e & 1) * 64 + 32, sv + 32);
      tmem_wait_ld();
      if (e == m - 1) {  // the diagonal block: causal mask
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (j > t) sv[j] = -INFINITY;
      }
      float mx0 = fmax3(sv[0], sv[1], sv[2]), mx1 = fmax3(sv[3], sv[4], sv[5]);
#pragma unroll
      for (int j = 6; j < 62; j += 4) {
        mx0 = fmax3(mx0, sv[j], sv[j + 1]);
        mx1 = fmax3(mx1, sv[j + 2], sv[j + 3]);
      }
      // gated mode: + the block's gate for this row's head, in log2 units
      const float beta2 = kGated ? gb_s[2 * e + (r >> 6)] * kLog2e : 0.f;
      const float mx = fmaf(fmax3(mx0, mx1, fmaxf(sv[62], sv[63])), sl2, beta2);
      const float m_new = fmaxf(m_run, mx);
      // rescale O only when the running maximum grows by more than 2^8:
      // probabilities stay below 256 in between, exact after normalisation
      const bool resc = (m_new > m_run + 8.f);
      const float m_use = resc ? m_new : m_run;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const float p0 = exp2_approx(fmaf(sv[j], sl2, beta2 - m_use));
        const float p1 = exp2_approx(fmaf(sv[j + 1], sl2, beta2 - m_use));
        rs[(j >> 1) & 3] += p0 + p1;
        pk[j >> 1] = pack_bf16x2(p0, p1);
      }
      const float alpha = exp2_approx(m_run - m_use);
      if (e > 0 && __any_sync(0xffffffffu, resc)) {
#ifdef SAS_PHASE_TRACE
        acc[7] += 1;
#endif
        mbar_wait(&bars[kBarO], (e - 1) & 1, p.status);  // P V_{e-1} done: O is stable
        tc_fence_after_sync();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tl + 128 + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(tl + 128 + 32 * c, o);
        }
      }
      tmem_st32(tl + (e & 1) * 64, pk);
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarP0 + (e & 1)]);
      PF_TOC(acc[6], tc);
      l_run = l_run * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
      m_run = m_use;
    }
#ifdef SAS_PHASE_TRACE
    if (trc != nullptr && tid == 0) trc[11] = global_timer_ns();  // end of the tile loop
#endif
    // epilogue: O / l, bf16, one row per thread
    __nv_bfloat16* dst = p.out + ((static_cast<size_t>(s) * p.hq + g0 + (r >> 6)) * p.T +
                                  static_cast<size_t>(i) * kBlock + t) * kDim;
    if (m > 0) {
      mbar_wait(&bars[kBarO], (m - 1) & 1, p.status);
      tc_fence_after_sync();
      const float inv = 1.f / l_run;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tl + 128 + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 pk;
          pk.x = pack_bf16x2(o[8 * k + 0] * inv, o[8 * k + 1] * inv);
          pk.y = pack_bf16x2(o[8 * k + 2] * inv, o[8 * k + 3] * inv);
          pk.z = pack_bf16x2(o[8 * k + 4] * inv, o[8 * k + 5] * inv);
          pk.w = pack_bf16x2(o[8 * k + 6] * inv, o[8 * k + 7] * inv);
          if (!(lone && r >= kBlock)) *reinterpret_cast<uint4*>(dst + 32 * c + 8 * k) = pk;
        }
      }
    } else if (!(lone && r >= kBlock)) {
      for (int c = 0; c < kDim / 8; ++c) *reinterpret_cast<uint4*>(dst + 8 * c) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 0) tmem_dealloc(tmem, kPfTmemCols);
#ifdef SAS_PHASE_TRACE
  if (trc != nullptr && tid == 0) {
    trc[0] = t_start;
    trc[1] = global_timer_ns();
    trc[7] = static_cast<unsigned long long>(acc[5]);
    trc[8] = static_cast<unsigned long long>(acc[6]);
    trc[9] = static_cast<unsigned long long>(acc[7]);
    trc[10] = static_cast<unsigned long long>(m);
  }
#endif
}

// ------------------------------------------------------------ launchers
cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmq, const CUtensorMap& tmk,
                           const CUtensorMap& tmv, cudaStream_t stream) {
  {
    const dim3 grid(static_cast<unsigned>((p.nblk + kPfQb - 1) / kPfQb), static_cast<unsigned>(p.hq),
                    static_cast<unsigned>(p.batch));
    prefill_gate_query_kernel<<<grid, kThreads, kDim * kDim * 2 + 16, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    const dim3 grid(static_cast<unsigned>((p.nblk + kPfSelQb - 1) / kPfSelQb), static_cast<unsigned>(p.hkv),
                    static_cast<unsigned>(p.batch));
    const size_t smem = prefill_select_smem_bytes(p.nblk, p.max_sel);
    if (p.nblk - 1 > 4 * kThreads)  // more than 512 historical blocks can occur
      prefill_select_kernel<true><<<grid, kThreads, smem, stream>>>(p);
    else
      prefill_select_kernel<false><<<grid, kThreads, smem, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const unsigned ctas = static_cast<unsigned>(p.batch) * p.hkv * p.nblk * ((p.G + 1) / 2);
  const size_t smem = prefill_attn_smem_bytes(p.max_sel);
  if (p.gated)
    prefill_attn_kernel<true><<<ctas, kPfAttnThreads, smem, stream>>>(p, tmq, tmk, tmv);
  else
    prefill_attn_kernel<false><<<ctas, kPfAttnThreads, smem, stream>>>(p, tmq, tmk, tmv);
  return cudaGetLastError();
}

cudaError_t prepare_prefill_kernels() {
  cudaError_t e = cudaFuncSetAttribute(prefill_gate_query_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kDim * kDim * 2 + 16);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(prefill_select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(prefill_select_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(prefill_attn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(prefill_attn_smem_bytes(kPfMaxSel)));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_attn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(prefill_attn_smem_bytes(kPfMaxSel)));
}

}  // namespace sas
