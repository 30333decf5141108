// SAS block-sparse chunked prefill.
//
// Method (release pages: "Tencent released Simple-Attention-Sparsification
// ..." aigc.news 2026-09-14, release paragraph: training Top-K 31 historical
// blocks over 32,768-token sequences, 64-token blocks, gate with Qproj, Q/K
// normalisation and gate RoPE): for every 64-token query block i of a
// sequence and every KV head h,
//   q~_g = RoPE(RMSNorm(mean_t q_{g,t} @ W_q[g]) * gamma_q, i)   (g in the group)
//   S_b  = mean_g(q~_g . k~_b) * gate_scale                    (b < i)
//   keep the min(topk, i) blocks of largest S_b (ties: lower index) + block i;
//   token t of block i attends to every token of the kept blocks and to the
//   tokens of block i up to t (causal).
//
// Kernels:
//   prefill_gate_query_kernel  q~ for every (sequence, query head, block):
//                              W_q[g] staged in shared memory once per CTA.
//   prefill_select_kernel      scores and exact Top-K per (seq, head, block).
//   prefill_attn_kernel        tcgen05 block-sparse attention: one CTA per
//                              (seq, KV head, query block, pair of query
//                              heads); the 128 query rows (2 heads x 64
//                              tokens) are the M dimension of
//                              S = Q K^T (N = 64 keys) and O += P V (N = 128),
//                              accumulators in tensor memory.
#include "sas_internal.h"
#include "sas_select.cuh"

namespace sas {

// ------------------------------------------------------------ gate queries
// grid (ceil(nblk / kPfQb), Hq, B), 128 threads.  Thread d owns dimension d.
__global__ void __launch_bounds__(kThreads) prefill_gate_query_kernel(const __grid_constant__ PrefillParams p) {
  const int g = blockIdx.y;
  const int s = blockIdx.z;
  const int i0 = blockIdx.x * kPfQb;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* wq = reinterpret_cast<__nv_bfloat16*>(smem_raw);  // [128][128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + kDim * kDim * 2);
  __shared__ float red[8][kDim];
  __shared__ float qbar[kDim];
  __shared__ float xn[kDim];
  __shared__ float ssq[kWarps];
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, kDim * kDim * 2);
    bulk_g2s(wq, p.w_q + static_cast<size_t>(g) * kDim * kDim, kDim * kDim * 2, bar);
  }
  __syncthreads();
  const bool ok = mbar_wait(bar, 0, p.status);
  const float gam = p.gamma_q[tid];
  const int cvec = tid & 15, rg = tid >> 4;  // 8 dims x rows rg, rg+8, ...
  const int i1 = min(p.nblk, i0 + kPfQb);
  for (int i = i0; i < i1; ++i) {
    const __nv_bfloat16* qb = p.q + ((static_cast<size_t>(s) * p.hq + g) * p.T + static_cast<size_t>(i) * kBlock) * kDim;
    uint4 raw[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      raw[r] = *reinterpret_cast<const uint4*>(qb + static_cast<size_t>(rg + 8 * r) * kDim + cvec * 8);
    float acc[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) acc[v] = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw[r]);
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[v] += __bfloat162float(e[v]);
    }
#pragma unroll
    for (int v = 0; v < 8; ++v) red[rg][cvec * 8 + v] = acc[v];
    __syncthreads();
    {
      float sm = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) sm += red[r][tid];
      qbar[tid] = sm * (1.f / kBlock);  // per-head mean of the block's 64 queries
    }
    __syncthreads();
    float u = 0.f;
    if (ok) {
      float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 16
      for (int r = 0; r < kDim; ++r) a4[r & 3] = fmaf(qbar[r], __bfloat162float(wq[r * kDim + tid]), a4[r & 3]);
      u = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    }
    float sq = u * u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) ssq[warp] = sq;
    __syncthreads();
    const float tot = ssq[0] + ssq[1] + ssq[2] + ssq[3];
    xn[tid] = u * (1.f / sqrtf(tot / kDim + p.eps)) * gam;
    __syncthreads();
    float cs, sn;
    rope_cos_sin(p.rope.theta_over_pi[tid & 63], i, cs, sn);
    const float y = (tid < 64) ? xn[tid] * cs - xn[tid + 64] * sn : xn[tid] * cs + xn[tid - 64] * sn;
    p.qt[((static_cast<size_t>(s) * p.hq + g) * p.nblk + i) * kDim + tid] = y;
    __syncthreads();  // red / qbar / xn / ssq are reused by the next block
  }
}

// ------------------------------------------------------------ selection
// grid (nblk, Hkv, B), 128 threads.
__global__ void __launch_bounds__(kThreads) prefill_select_kernel(const __grid_constant__ PrefillParams p) {
  const int i = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* vals = reinterpret_cast<float*>(smem_raw);
  uint8_t* q = smem_raw + (p.nblk * 4 + 15) / 16 * 16;
  int* sel = reinterpret_cast<int*>(q);
  q += (p.max_sel * 4 + 15) / 16 * 16;
  uint32_t* hist = reinterpret_cast<uint32_t*>(q);
  q += kSelBins * 4;
  uint32_t* selbits = reinterpret_cast<uint32_t*>(q);
  q += ((p.nblk + 31) / 32 * 4 + 15) / 16 * 16;
  int* scan = reinterpret_cast<int*>(q);
  q += 16 * 4;
  float* qbar = reinterpret_cast<float*>(q);
  // S_b = mean_g(q~_g . k~_b) * scale = (scale/G * sum_g q~_g) . k~_b
  {
    float a = 0.f;
    for (int g = 0; g < G; ++g)
      a += p.qt[((static_cast<size_t>(s) * p.hq + h * G + g) * p.nblk + i) * kDim + tid];
    qbar[tid] = a * (p.gate_scale / static_cast<float>(G));
  }
  __syncthreads();
  const int grp = lane >> 3, sub = lane & 7;
  float4 qr[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) qr[k] = *reinterpret_cast<const float4*>(qbar + sub * 16 + 4 * k);
  const float* gk = p.gate_keys + (static_cast<size_t>(s) * p.hkv + h) * p.mg * kDim;
  for (int b0 = 0; b0 < i; b0 += 16) {
    const int b = b0 + warp * 4 + grp;
    float acc = 0.f;
    if (b < i) {
      const float4* row = reinterpret_cast<const float4*>(gk + static_cast<size_t>(b) * kDim + sub * 16);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 kv = row[k];
        acc = fmaf(qr[k].x, kv.x, acc);
        acc = fmaf(qr[k].y, kv.y, acc);
        acc = fmaf(qr[k].z, kv.z, acc);
        acc = fmaf(qr[k].w, kv.w, acc);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (b < i && sub == 0) vals[b] = acc;
  }
  __syncthreads();
  const int m = select_blocks(vals, i, p.topk, i, sel, hist, selbits, scan);
  const size_t base = (static_cast<size_t>(s) * p.hkv + h) * p.nblk + i;
  for (int j = tid; j < m; j += kThreads) {
    p.sel[base * p.max_sel + j] = sel[j];
    if (p.sel_out != nullptr) p.sel_out[base * p.max_sel + j] = sel[j];
  }
  if (tid == 0) {
    p.cnt[base] = m;
    if (p.cnt_out != nullptr) p.cnt_out[base] = m;
  }
}

size_t prefill_select_smem_bytes(int nblk, int max_sel) {
  return static_cast<size_t>((nblk * 4 + 15) / 16 * 16 + (max_sel * 4 + 15) / 16 * 16 + kSelBins * 4 +
                             ((nblk + 31) / 32 * 4 + 15) / 16 * 16 + 16 * 4 + kDim * 4);
}

// ------------------------------------------------------------ tcgen05 attention
// 160 threads: warps 0-3 own one query row each per thread (softmax, O
// rescaling, epilogue); warp 4 lane 0 issues the TMA copies and the MMAs.
// Shared memory (1024-aligned): Q 32 KiB | K ring 2 x 16 KiB | V ring 2 x 16 KiB
// | P 16 KiB | barriers | block list.  Tensor memory: S double buffer
// (2 x 64 columns) and O (128 columns), 256 columns in all.
constexpr int kPfAttnThreads = 160;
constexpr uint32_t kPfTmemCols = 256;
constexpr int kPfSmemQ = 0, kPfSmemK = 32768, kPfSmemV = 65536, kPfSmemP = 98304,
              kPfSmemBars = 114688;
enum { kBarQ = 0, kBarK0 = 1, kBarV0 = 3, kBarS0 = 5, kBarSfree0 = 7, kBarP = 9, kBarO = 10,
       kNumPfBars = 11 };

size_t prefill_attn_smem_bytes(int max_sel) {
  return static_cast<size_t>(kPfSmemBars + kNumPfBars * 8 + 16 + max_sel * 4);
}

__global__ void __launch_bounds__(kPfAttnThreads, 2)
    prefill_attn_kernel(const __grid_constant__ PrefillParams p,
                        const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int npair = p.G / 2;
  int idx = static_cast<int>(blockIdx.x);
  const int pair = idx % npair;
  idx /= npair;
  const int h = idx % p.hkv;
  idx /= p.hkv;
  const int s = idx % p.batch;
  const int i = p.nblk - 1 - idx / p.batch;  // longest block lists first
  const int g0 = h * p.G + 2 * pair;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kPfSmemBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumPfBars);
  int* sel_s = reinterpret_cast<int*>(tmem_slot + 4);
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
      mbar_init(&bars[b], (b == kBarSfree0 || b == kBarSfree0 + 1 || b == kBarP) ? 128u : 1u);
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
  uint8_t* sP = base + kPfSmemP;
  const float sl2 = p.attn_scale_log2;

  if (warp == 4) {
    if (lane == 0 && m > 0) {
      // ---------------------------------------------------- producer / MMA issuer
      const uint32_t idesc_qk = umma_idesc_bf16(128, 64, false, false);
      const uint32_t idesc_pv = umma_idesc_bf16(128, 128, false, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      const int rowq0 = static_cast<int>((static_cast<size_t>(s) * p.hq + g0) * p.T) + kBlock * i;
      const int rowq1 = rowq0 + p.T;
      const int rowkv = static_cast<int>((static_cast<size_t>(s) * p.hkv + h) * p.T);
      mbar_arrive_expect_tx(&bars[kBarQ], 32768);
      tma_load_2d(sQ + 0, &tmq, 0, rowq0, &bars[kBarQ]);
      tma_load_2d(sQ + 8192, &tmq, 0, rowq1, &bars[kBarQ]);
      tma_load_2d(sQ + 16384, &tmq, 64, rowq0, &bars[kBarQ]);
      tma_load_2d(sQ + 24576, &tmq, 64, rowq1, &bars[kBarQ]);
      auto load_k = [&](int e) {
        const int st = e & 1;
        mbar_arrive_expect_tx(&bars[kBarK0 + st], 16384);
        const int row = rowkv + kBlock * sel_s[e];
        tma_load_2d(sK + st * 16384, &tmk, 0, row, &bars[kBarK0 + st]);
        tma_load_2d(sK + st * 16384 + 8192, &tmk, 64, row, &bars[kBarK0 + st]);
      };
      auto load_v = [&](int e) {
        const int st = e & 1;
        mbar_arrive_expect_tx(&bars[kBarV0 + st], 16384);
        const int row = rowkv + kBlock * sel_s[e];
        tma_load_2d(sV + st * 16384, &tmv, 0, row, &bars[kBarV0 + st]);
        tma_load_2d(sV + st * 16384 + 8192, &tmv, 64, row, &bars[kBarV0 + st]);
      };
      auto issue_qk = [&](int e) {
        const int st = e & 1;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = umma_desc_sw128(aQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(aK + st * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
          umma_bf16_ss(tmem + st * 64, a, b, idesc_qk, kk > 0);
        }
        umma_commit(&bars[kBarS0 + st]);
      };
      load_k(0);
      load_v(0);
      if (m > 1) {
        load_k(1);
        load_v(1);
      }
      mbar_wait(&bars[kBarQ], 0, p.status);
      mbar_wait(&bars[kBarK0], 0, p.status);
      tc_fence_after_sync();
      issue_qk(0);
      for (int e = 0; e < m; ++e) {
        if (e + 1 < m) {
          mbar_wait(&bars[kBarK0 + ((e + 1) & 1)], ((e + 1) >> 1) & 1, p.status);
          if (e >= 1) mbar_wait(&bars[kBarSfree0 + ((e + 1) & 1)], ((e - 1) >> 1) & 1, p.status);
          tc_fence_after_sync();
          issue_qk(e + 1);
        }
        if (e + 2 < m) {
          mbar_wait(&bars[kBarS0 + (e & 1)], (e >> 1) & 1, p.status);  // QK_e done: K slot free
          load_k(e + 2);
        }
        mbar_wait(&bars[kBarP], e & 1, p.status);
        mbar_wait(&bars[kBarV0 + (e & 1)], (e >> 1) & 1, p.status);
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t a = umma_desc_sw128(aP + kk * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(aV + (e & 1) * 16384 + kk * 2048, 8192, 1024);
          umma_bf16_ss(tmem + 128, a, b, idesc_pv, e > 0 || kk > 0);
        }
        umma_commit(&bars[kBarO]);
        if (e + 2 < m) {
          mbar_wait(&bars[kBarO], e & 1, p.status);  // PV_e done: V slot free
          load_v(e + 2);
        }
      }
      mbar_wait(&bars[kBarO], (m - 1) & 1, p.status);  // nothing of ours in flight at teardown
    }
  } else {
    // ------------------------------------------------------ softmax / epilogue
    const int r = tid;            // query row: head g0 + (r >> 6), token r & 63
    const int t = r & 63;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    float m_run = -INFINITY, l_run = 0.f;
    for (int e = 0; e < m; ++e) {
      mbar_wait(&bars[kBarS0 + (e & 1)], (e >> 1) & 1, p.status);
      tc_fence_after_sync();
      float sv[64];
      tmem_ld32(tl + (e & 1) * 64, sv);
      tmem_ld32(tl + (e & 1) * 64 + 32, sv + 32);
      tmem_wait_ld();
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarSfree0 + (e & 1)]);
      const bool diag = (sel_s[e] == i);
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float x = (diag && j > t) ? -INFINITY : sv[j] * sl2;
        sv[j] = x;
        mx = fmaxf(mx, x);
      }
      const float m_new = fmaxf(m_run, mx);
      // rescale O only when the running maximum grows by more than 2^8:
      // probabilities stay below 256 in between, exact after normalisation
      const bool resc = (m_new > m_run + 8.f);
      const float m_use = resc ? m_new : m_run;
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float pj = (sv[j] == -INFINITY) ? 0.f : exp2f(sv[j] - m_use);
        sv[j] = pj;
        rs += pj;
      }
      if (e > 0) {
        mbar_wait(&bars[kBarO], (e - 1) & 1, p.status);  // PV_{e-1} done: O and P free
        tc_fence_after_sync();
      }
      const float alpha = resc ? exp2f(m_run - m_use) : 1.f;
      if (e > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tl + 128 + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(tl + 128 + 32 * c, o);
        }
        tmem_wait_st();
      }
      l_run = l_run * alpha + rs;
      m_run = m_use;
      // P row r as bf16, 128-byte swizzled (chunk jc of row r at jc ^ (r & 7))
#pragma unroll
      for (int jc = 0; jc < 8; ++jc) {
        uint4 pk;
        pk.x = pack_bf16x2(sv[8 * jc + 0], sv[8 * jc + 1]);
        pk.y = pack_bf16x2(sv[8 * jc + 2], sv[8 * jc + 3]);
        pk.z = pack_bf16x2(sv[8 * jc + 4], sv[8 * jc + 5]);
        pk.w = pack_bf16x2(sv[8 * jc + 6], sv[8 * jc + 7]);
        *reinterpret_cast<uint4*>(sP + r * 128 + ((jc ^ (r & 7)) << 4)) = pk;
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(&bars[kBarP]);
    }
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
          *reinterpret_cast<uint4*>(dst + 32 * c + 8 * k) = pk;
        }
      }
    } else {
      for (int c = 0; c < kDim / 8; ++c) *reinterpret_cast<uint4*>(dst + 8 * c) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 0) tmem_dealloc(tmem, kPfTmemCols);
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
    const dim3 grid(static_cast<unsigned>(p.nblk), static_cast<unsigned>(p.hkv), static_cast<unsigned>(p.batch));
    prefill_select_kernel<<<grid, kThreads, prefill_select_smem_bytes(p.nblk, p.max_sel), stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const unsigned ctas = static_cast<unsigned>(p.batch) * p.hkv * p.nblk * (p.G / 2);
  prefill_attn_kernel<<<ctas, kPfAttnThreads, prefill_attn_smem_bytes(p.max_sel), stream>>>(p, tmq, tmk, tmv);
  return cudaGetLastError();
}

cudaError_t prepare_prefill_kernels() {
  cudaError_t e = cudaFuncSetAttribute(prefill_gate_query_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kDim * kDim * 2 + 16);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(prefill_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(prefill_attn_smem_bytes(kPfMaxSel)));
}

}  // namespace sas
