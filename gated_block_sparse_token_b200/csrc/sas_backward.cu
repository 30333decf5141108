// SAS gate backward: the gradient of the gated decode step with respect to
// the gate parameters W_q, W_k, gamma_q and gamma_k.
//
// Method (release pages: "Tencent released Simple-Attention-Sparsification
// ..." aigc.news 2026-09-14, release paragraph -- continuous gates on the
// selected blocks make the discrete Top-K selection differentiable): in the
// gated mode every token of a selected historical block b carries, for query
// head g, the logit bias log(sigmoid(s_gb)) with s_gb = q~_g . k~_b *
// gate_scale.  For an upstream gradient dL/dout the gate parameters receive
//   dL/ds_gb = (sum over the block's tokens j of dL/dlogit_gj) * sigmoid(-s_gb),
//   dL/dlogit_gj = p_gj (dout_g . v_j - dout_g . out_g),
// then back through the score, the gate RoPE, the RMSNorms and the two
// projections.  The block list is held fixed (the Top-K has no gradient).
//
// Two kernels.  gate_backward_kernel, one CTA (256 threads) per (sequence,
// KV head):
//   1. q, dout and the gains into shared memory; v_g = q_g @ W_q[g]; RMSNorm,
//      gain, RoPE -> q~_g.
//   2. one pass over the block list, K and V blocks by 2-D TMA (128-byte
//      swizzle) into a ring of as many stages (up to 4) as shared memory
//      holds beside the list's terms: the pooled key [max; min; mean]
//      of every historical entry; the logits q_g . k_j (warps 0-3) and
//      dout_g . v_j (warps 4-7, dout split into two bf16 terms) on bf16
//      mma.sync with fp32 accumulation; per (entry, head) the softmax
//      statistics of the block without its bias -- max m', sum z' of
//      exp(logit - m'), sum y' of exp(logit - m') (dout . v_j).  A bias
//      constant over the block only shifts m', so the biased statistics
//      follow once the gates are known.
//   3. u_e = P_e @ W_k[h] for every historical entry on the tensor cores
//      (W_k read once through the idle ring, P split into two bf16 terms);
//      RMSNorm, gain, RoPE -> k~_e; s_ge.
//   4. per head: the global max, sum and D_g = dout_g . out_g from the
//      per-entry statistics with the biases; dL/dbias_ge and dL/ds_ge.
//   5. dL/dq~_g and dL/dk~_e; RoPE transposed (rotation by -pos); RMSNorm
//      backward; dL/dv_g, dL/du_e and the gain gradients.
//   6. dL/dv_g, the pooled keys P_e, dL/du_e and the pair's gain gradients
//      into the workspace.
// gate_grad_reduce_kernel then adds, with no atomics (a fixed summation
// order, so the result is reproducible bit for bit),
//   dL/dW_q[g] = sum over sequences of q_g (x) dL/dv_g,
//   dL/dW_k[h] = sum over sequences and historical entries of P_e (x) dL/du_e,
// and the gain gradients summed over the pairs, to the caller's arrays.
#include <cmath>

#include "sas_internal.h"

namespace sas {

// Step-trace hook: thread 0 of each CTA stamps the SM clock at step
// boundaries (tracing builds only; slot 0 is the global timer).
#ifdef SAS_PHASE_TRACE
#define BWD_TRACE(k)                                                                         \
  do {                                                                                       \
    if (p.trace != nullptr && threadIdx.x == 0 && blockIdx.x < static_cast<unsigned>(kTraceCtas)) { \
      p.trace[blockIdx.x * kTraceSlots + (k)] = ((k) == 0) ? global_timer_ns() : clock64();  \
      if ((k) == 0) p.trace[blockIdx.x * kTraceSlots + 23] = clock64();                      \
    }                                                                                        \
  } while (0)
#else
#define BWD_TRACE(k) \
  do {               \
  } while (0)
#endif

namespace {

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// log(sigmoid(x)) without overflow for either sign
__device__ __forceinline__ float log_sigmoid_f(float x) {
  return (x >= 0.f) ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

__device__ __forceinline__ float sigmoid_f(float x) {
  return (x >= 0.f) ? 1.f / (1.f + expf(-x)) : expf(x) / (1.f + expf(x));
}

}  // namespace

__global__ void __launch_bounds__(kBwThreads, 1)
    gate_backward_kernel(const __grid_constant__ GateBwdParams p, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmwk) {
  constexpr int kW = kBwThreads / 32;  // warps
  // a cluster of two CTAs per (sequence, KV head) pair: CTA 1 streams and
  // pools every other list entry and hands its rows to CTA 0, which carries
  // the rest of the pass alone
  uint32_t crank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int s = pair / p.hkv;
  const int h = pair - s * p.hkv;
  const int G = p.G;
  const int MS = p.max_sel;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  BWD_TRACE(0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // carve (the order of gate_bwd_smem_bytes)
  const int NS = p.stages;                                            // K/V ring stages (1 or 2)
  uint8_t* tiles = base;                                              // [NS stages][K, V] bf16 [64][128]
  constexpr int kPs = kBwPoolStride;
  float* P = reinterpret_cast<float*>(tiles + 2 * NS * kTileBytes);   // [MS][kPs] pooled keys
  float* U = P + MS * kPs;                                            // [MS][128] u, then dL/du
  float* qf = U + MS * kDim;                                          // [G][128] q
  float* dof = qf + G * kDim;                                         // [G][128] dout
  float* vq = dof + G * kDim;                                         // [G][128] v, then dL/dv
  float* qt = vq + G * kDim;                                          // [G][128] q~
  float* st_m = qt + G * kDim;                                        // [MS][G] block max (no bias)
  float* st_z = st_m + MS * G;                                        // [MS][G]
  float* st_y = st_z + MS * G;                                        // [MS][G]
  float* sg = st_y + MS * G;                                          // [MS][G] gate scores
  float* dsg = sg + MS * G;                                           // [MS][G] dL/ds
  float* lg = dsg + MS * G;                                           // [G][64] logits of one block
  float* wg = lg + G * kBlock;                                        // [G][64] dout . v_j
  int* sel = reinterpret_cast<int*>(wg + G * kBlock);                 // [MS]
  float* ru = reinterpret_cast<float*>(sel + MS);                     // [MS] RMS of u_e
  __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(ru + MS);     // [G][128] q as bf16
  float* dqt = reinterpret_cast<float*>(qb + G * kDim);               // [G][128] dL/dq~
  float* dgq = dqt + G * kDim;                                        // [128]
  float* dgk = dgq + kDim;                                            // [128]
  float* red = dgk + kDim;                                            // [2][warps][128] gain partials
  float* poolp = red + 2 * kW * kDim;                                 // [4][384] pooling partials
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(poolp + 4 * kPool) + 7) & ~uintptr_t(7));
  // k~ of every historical entry (steps 3-5), over the K/V ring, idle by then
  float* ktl = reinterpret_cast<float*>(tiles);                       // [MS][128]
  static_assert(kBwMaxSel * kDim * 4 <= 2 * kTileBytes, "k~ of a full list fits one ring stage");

  // ---- the block list, checked like the attention call checks it
  const int L = p.kv.seq_lens[s];
  const int m = p.sel_count[pair];
  const int c = (L >= 1) ? (L - 1) / kBlock : 0;
  bool err = (L < 1) || m < 1 || m > MS;
  if (!err) {
    const int32_t* si = p.sel_idx + static_cast<size_t>(pair) * MS;
    for (int j = tid; j < m; j += kBwThreads) {
      const int b = si[j];
      sel[j] = b;
      if (b < 0 || b > c) err = true;
      if (j == m - 1 && b != c) err = true;
      if (j > 0 && si[j - 1] >= b) err = true;
      if (p.kv.block_row(s, h, b) < 0) err = true;
    }
  }
  if (__syncthreads_or(err)) {  // both CTAs see the same list and leave together
    if (tid == 0 && crank == 0) {
      raise_status(p.status, kStatusBounds);
      p.ws_nh[pair] = -1;
    }
    return;
  }
  const int nh = m - 1;  // historical entries (the current block, last, has no gate)
  // entries e = crank, crank + 2, ...; CTA 1's rows reach CTA 0 as
  // (pooled row unless e is the current block) + 3 G statistics each
  const int n1 = m >> 1;
  const int hist1 = n1 - (((m - 1) & 1) ? 1 : 0);
  const uint32_t x_bytes = static_cast<uint32_t>(n1 * 3 * G * 4 + hist1 * kPool * 4);

  // ---- K/V ring: the CTA's k-th entry (e = crank + 2k) in stage k % NS
  // (16 KiB K then 16 KiB V)
  auto issue = [&](int k) {
    const int st = k % NS;
    const int row0 = static_cast<int>(p.kv.block_row(s, h, sel[static_cast<int>(crank) + 2 * k]));
    uint8_t* kd = tiles + (2 * st) * kTileBytes;
    uint8_t* vd = kd + kTileBytes;
    mbar_arrive_expect_tx(&bars[st], 2 * kTileBytes);
    tma_load_2d(kd, &tmk, 0, row0, &bars[st]);
    tma_load_2d(kd + 8192, &tmk, 64, row0, &bars[st]);
    tma_load_2d(vd, &tmv, 0, row0, &bars[st]);
    tma_load_2d(vd + 8192, &tmv, 64, row0, &bars[st]);
  };
  uint64_t* bar_w = &bars[4];  // W_k chunks (step 3)
  uint64_t* bar_x = &bars[5];  // CTA 0: the rows CTA 1 hands over
  const int mine = (m - static_cast<int>(crank) + 1) >> 1;  // entries of this CTA
  if (tid == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    prefetch_tensormap(&tmwk);
    for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
    mbar_init(bar_w, 1);
    mbar_init(bar_x, 1);
    fence_mbar_init();
    if (crank == 0) mbar_arrive_expect_tx(bar_x, x_bytes);
    for (int k = 0; k < NS && k < mine; ++k) issue(k);
  }
  // thread 0 arrives after its barrier initialisation: CTA 1 stores into
  // CTA 0 only after the wait that follows its list pass
  cluster_arrive_relaxed();

  BWD_TRACE(1);  // list checked, ring started
  // ---- 1. gate query: v_g = q_g @ W_q[g], RMSNorm, gain, RoPE at c
  const size_t qoff = (static_cast<size_t>(s) * p.hq + static_cast<size_t>(h) * G) * kDim;
  for (int i = tid; i < G * kDim; i += kBwThreads) {
    const __nv_bfloat16 x = p.q[qoff + i];
    qb[i] = x;
    qf[i] = __bfloat162float(x);
    dof[i] = p.d_out[qoff + i];
  }
  __syncthreads();
  // two adjacent columns per thread (one 4-byte load per row, 256 bytes per
  // warp and row)
  for (int o = tid; o < G * (kDim / 2); o += kBwThreads) {
    const int g = o / (kDim / 2), j = 2 * (o - g * (kDim / 2));
    const uint32_t* wcol =
        reinterpret_cast<const uint32_t*>(p.w_q + (static_cast<size_t>(h * G + g) * kDim) * kDim + j);
    const float* qrow = qf + g * kDim;
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll 16
    for (int i = 0; i < kDim; i += 2) {
      const uint32_t w0 = wcol[static_cast<size_t>(i) * (kDim / 2)];
      const uint32_t w1 = wcol[static_cast<size_t>(i + 1) * (kDim / 2)];
      a0 = fmaf(qrow[i], bf16_lo(w0), a0);
      a1 = fmaf(qrow[i], bf16_hi(w0), a1);
      b0 = fmaf(qrow[i + 1], bf16_lo(w1), b0);
      b1 = fmaf(qrow[i + 1], bf16_hi(w1), b1);
    }
    vq[g * kDim + j] = a0 + b0;
    vq[g * kDim + j + 1] = a1 + b1;
  }
  __syncthreads();
  for (int g = warp; g < G; g += kW) {
    float x[4], ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[k] = vq[g * kDim + lane + 32 * k];
      ss = fmaf(x[k], x[k], ss);
    }
    ss = warp_sum(ss);
    const float inv = 1.f / sqrtf(ss / kDim + p.eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = x[k] * inv * p.gamma_q[lane + 32 * k];
    float c0, s0, c1, s1;
    rope_cos_sin(p.rope.theta_over_pi[lane], c, c0, s0);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], c, c1, s1);
    qt[g * kDim + lane] = x[0] * c0 - x[2] * s0;
    qt[g * kDim + lane + 64] = x[2] * c0 + x[0] * s0;
    qt[g * kDim + lane + 32] = x[1] * c1 - x[3] * s1;
    qt[g * kDim + lane + 96] = x[3] * c1 + x[1] * s1;
  }

  BWD_TRACE(2);  // gate query done
  // ---- 2. pass over the list: pooled keys and unbiased block statistics
  const float alpha = p.attn_scale;
#ifdef SAS_PHASE_TRACE
  unsigned long long seg[6] = {0, 0, 0, 0, 0, 0}, tseg = clock64();
#define BWD_SEG(i)                      \
  do {                                  \
    const unsigned long long t_ = clock64(); \
    seg[i] += t_ - tseg;                \
    tseg = t_;                          \
  } while (0)
#else
#define BWD_SEG(i) \
  do {             \
  } while (0)
#endif
  for (int k = 0; k < mine; ++k) {
    const int e = static_cast<int>(crank) + 2 * k;
    const int st = k % NS;
    const bool ok = mbar_wait(&bars[st], (k / NS) & 1, p.status);
    BWD_SEG(0);
    const int b = sel[e];
    const int nvalid = (b == c) ? (L - b * kBlock) : kBlock;
    const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(tiles + (2 * st) * kTileBytes);
    const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(tiles + (2 * st + 1) * kTileBytes);
    // pooling partials: thread (quarter, pair) takes dimensions 2 pr, 2 pr + 1
    // over tokens 16 quarter .. + 15 (4-byte loads; every warp shares it)
    if (b != c) {
      const int pr = tid & 63, qt4 = tid >> 6;
      float mx0 = -INFINITY, mx1 = -INFINITY, mn0 = INFINITY, mn1 = INFINITY, s0 = 0.f, s1 = 0.f;
      if (ok) {
        const uint8_t* kt8 = reinterpret_cast<const uint8_t*>(kt) + (pr & 3) * 4;
#pragma unroll
        for (int t = 16 * qt4; t < 16 * qt4 + 16; ++t) {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(kt8 + swz_tile_offset(t, pr >> 2));
          const float x0 = bf16_lo(w), x1 = bf16_hi(w);
          mx0 = fmaxf(mx0, x0);
          mx1 = fmaxf(mx1, x1);
          mn0 = fminf(mn0, x0);
          mn1 = fminf(mn1, x1);
          s0 += x0;
          s1 += x1;
        }
      }
      float* pp = poolp + qt4 * kPool;
      *reinterpret_cast<float2*>(pp + 2 * pr) = make_float2(mx0, mx1);
      *reinterpret_cast<float2*>(pp + kDim + 2 * pr) = make_float2(mn0, mn1);
      *reinterpret_cast<float2*>(pp + 2 * kDim + 2 * pr) = make_float2(s0, s1);
    }
    BWD_SEG(1);
    // logits q_g . k_j (warps 0-3) and dout_g . v_j (warps 4-7) on the
    // tensor cores: the group's heads are rows 0..G-1 of the A operand, each
    // warp takes 16 tokens as two 8-column tiles; dout enters as hi + lo
    // bf16 terms (its fp32 value to about 2^-16)
    {
      const bool is_w = warp >= 4;
      const int wt = warp & 3;
      const int tq = lane & 3, gq = lane >> 2;
      const int mat = lane >> 3;
      const int tok = 16 * wt + (mat >> 1) * 8 + (lane & 7);
      const uint32_t tb = smem_u32(tiles + (2 * st + (is_w ? 1 : 0)) * kTileBytes);
      const int gr = min(gq, G - 1);
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      if (ok) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(tb + swz_tile_offset(tok, 2 * ks + (mat & 1)), r0, r1, r2, r3);
          if (!is_w) {
            const uint32_t* q2 = reinterpret_cast<const uint32_t*>(qb + gr * kDim + 16 * ks + 2 * tq);
            const uint32_t a0 = q2[0], a2 = q2[4];
            mma_rows0_7(acc[0][0], acc[0][1], a0, a2, r0, r1);
            mma_rows0_7(acc[1][0], acc[1][1], a0, a2, r2, r3);
          } else {
            const float* d = dof + gr * kDim + 16 * ks + 2 * tq;
            const float x0 = d[0], x1 = d[1], x8 = d[8], x9 = d[9];
            const uint32_t h0 = pack_bf16x2(x0, x1), h2 = pack_bf16x2(x8, x9);
            const uint32_t l0 = pack_bf16x2(x0 - bf16_lo(h0), x1 - bf16_hi(h0));
            const uint32_t l2 = pack_bf16x2(x8 - bf16_lo(h2), x9 - bf16_hi(h2));
            mma_rows0_7(acc[0][0], acc[0][1], h0, h2, r0, r1);
            mma_rows0_7(acc[0][0], acc[0][1], l0, l2, r0, r1);
            mma_rows0_7(acc[1][0], acc[1][1], h0, h2, r2, r3);
            mma_rows0_7(acc[1][0], acc[1][1], l0, l2, r2, r3);
          }
        }
      }
      if (gq < G) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int j = 16 * wt + 8 * nt + 2 * tq + q;
            const bool live = ok && j < nvalid;  // rows past the context may hold anything
            if (!is_w)
              lg[gq * kBlock + j] = live ? acc[nt][q] * alpha : -INFINITY;
            else
              wg[gq * kBlock + j] = live ? acc[nt][q] : 0.f;
          }
      }
    }
    BWD_SEG(2);
    __syncthreads();  // every read of this stage is done, the block's values are in
    if (tid == 0 && k + NS < mine) {
      fence_proxy_async_smem();
      issue(k + NS);
    }
    BWD_SEG(3);
    if (b != c) {  // the pooled key: quarters combined in order
      for (int i = tid; i < kPool; i += kBwThreads) {
        const float a0 = poolp[i], a1 = poolp[kPool + i], a2 = poolp[2 * kPool + i], a3 = poolp[3 * kPool + i];
        float r;
        if (i < kDim)
          r = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
        else if (i < 2 * kDim)
          r = fminf(fminf(a0, a1), fminf(a2, a3));
        else
          r = ((a0 + a1) + (a2 + a3)) * (1.f / kBlock);
        P[e * kPs + i] = r;
      }
    }
    for (int g = warp; g < G; g += kW) {
      const float l0 = lg[g * kBlock + lane], l1 = lg[g * kBlock + lane + 32];
      const float mx = warp_max(fmaxf(l0, l1));
      float z = 0.f, y = 0.f;
      if (mx != -INFINITY) {
        const float e0 = (l0 == -INFINITY) ? 0.f : expf(l0 - mx);
        const float e1 = (l1 == -INFINITY) ? 0.f : expf(l1 - mx);
        z = e0 + e1;
        y = e0 * wg[g * kBlock + lane] + e1 * wg[g * kBlock + lane + 32];
      }
      z = warp_sum(z);
      y = warp_sum(y);
      if (lane == 0) {
        st_m[e * G + g] = mx;
        st_z[e * G + g] = z;
        st_y[e * G + g] = y;
      }
    }
    BWD_SEG(4);
    __syncthreads();  // lg / wg are rewritten by the next entry
    BWD_SEG(5);
  }
#ifdef SAS_PHASE_TRACE
  if (p.trace != nullptr && tid == 0 && blockIdx.x < static_cast<unsigned>(kTraceCtas))
    for (int i = 0; i < 6; ++i) p.trace[blockIdx.x * kTraceSlots + 10 + i] = seg[i];
#endif

  // ---- hand-over: CTA 1's pooled rows and statistics into CTA 0's arrays
  // (the same places CTA 0 would have written them), 16-byte and 4-byte
  // asynchronous stores completing bar_x's bytes; CTA 1 then leaves
  cluster_wait();
  if (crank == 1) {
    const uint32_t rbar = dsmem_addr(bar_x, 0);
    for (int i = tid; i < hist1 * (kPool / 4); i += kBwThreads) {
      const int e = 1 + 2 * (i / (kPool / 4)), q4 = i - (i / (kPool / 4)) * (kPool / 4);
      const float4 v = *reinterpret_cast<const float4*>(P + e * kPs + 4 * q4);
      st_async_v4_f32(dsmem_addr(P + e * kPs + 4 * q4, 0), v.x, v.y, v.z, v.w, rbar);
    }
    for (int i = tid; i < n1 * G; i += kBwThreads) {
      const int e = 1 + 2 * (i / G), g = i - (i / G) * G;
      const int o = e * G + g;
      st_async_f32(dsmem_addr(st_m + o, 0), st_m[o], rbar);
      st_async_f32(dsmem_addr(st_z + o, 0), st_z[o], rbar);
      st_async_f32(dsmem_addr(st_y + o, 0), st_y[o], rbar);
    }
  } else if (x_bytes > 0) {
    mbar_wait_cluster(bar_x, 0, p.status);  // acquire at cluster scope: stores of CTA 1
  }
  // CTA 1 stays until CTA 0 holds every row
  cluster_arrive_relaxed();
  cluster_wait();
  if (crank == 1) return;

  BWD_TRACE(3);  // list pass done
  // ---- 3. gate keys of the historical entries: u_e = P_e @ W_k[h], on the
  // tensor cores.  W_k[h] streams through the idle K/V ring in 64-row
  // chunks (2-D TMA, 128-byte swizzle, two chunks per round); warp w owns
  // output columns 16w .. 16w + 15 of every 16-entry tile; P enters as hi +
  // lo bf16 terms (its fp32 value to about 2^-16), W_k is bf16 already.
  {
    const int tq = lane & 3, gq = lane >> 2, mat = lane >> 3;
    const int nmt = (nh + 15) >> 4;  // 16-entry tiles
    float acc[kBwMaxSel / 16][2][4];
#pragma unroll
    for (int mt = 0; mt < kBwMaxSel / 16; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
    constexpr int kChunks = kPool / 64;
    constexpr int kPerRound = 2;  // one ring stage holds two 16 KiB tiles
    for (int c0 = 0; c0 < kChunks; c0 += kPerRound) {
      __syncthreads();  // every read of the region (list pass, last round) is done
      if (tid == 0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar_w, kPerRound * kTileBytes);
        for (int cc = 0; cc < kPerRound; ++cc) {
          const int y = h * kPool + (c0 + cc) * 64;
          tma_load_2d(tiles + cc * kTileBytes, &tmwk, 0, y, bar_w);
          tma_load_2d(tiles + cc * kTileBytes + 8192, &tmwk, 64, y, bar_w);
        }
      }
      if (!mbar_wait(bar_w, (c0 / kPerRound) & 1, p.status)) continue;
      for (int cc = 0; cc < kPerRound; ++cc) {
        const uint32_t tb = smem_u32(tiles + cc * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 rows of the chunk
          uint32_t r0, r1, r2, r3;
          ldsm_x4_trans(tb + swz_tile_offset(16 * kk + (mat & 1) * 8 + (lane & 7), 2 * warp + (mat >> 1)), r0,
                        r1, r2, r3);
          const int k0 = (c0 + cc) * 64 + 16 * kk + 2 * tq;  // pooled dimension
#pragma unroll
          for (int mt = 0; mt < kBwMaxSel / 16; ++mt) {
            if (mt < nmt) {
              const int e0 = 16 * mt + gq, e1 = e0 + 8;
              const float2 z = make_float2(0.f, 0.f);
              const float2 x00 = e0 < nh ? *reinterpret_cast<const float2*>(P + e0 * kPs + k0) : z;
              const float2 x02 = e0 < nh ? *reinterpret_cast<const float2*>(P + e0 * kPs + k0 + 8) : z;
              const float2 x10 = e1 < nh ? *reinterpret_cast<const float2*>(P + e1 * kPs + k0) : z;
              const float2 x12 = e1 < nh ? *reinterpret_cast<const float2*>(P + e1 * kPs + k0 + 8) : z;
              const uint32_t h0 = pack_bf16x2(x00.x, x00.y), h1 = pack_bf16x2(x10.x, x10.y);
              const uint32_t h2 = pack_bf16x2(x02.x, x02.y), h3 = pack_bf16x2(x12.x, x12.y);
              const uint32_t l0 = pack_bf16x2(x00.x - bf16_lo(h0), x00.y - bf16_hi(h0));
              const uint32_t l1 = pack_bf16x2(x10.x - bf16_lo(h1), x10.y - bf16_hi(h1));
              const uint32_t l2 = pack_bf16x2(x02.x - bf16_lo(h2), x02.y - bf16_hi(h2));
              const uint32_t l3 = pack_bf16x2(x12.x - bf16_lo(h3), x12.y - bf16_hi(h3));
              mma_bf16_16816(acc[mt][0], h0, h1, h2, h3, r0, r1);
              mma_bf16_16816(acc[mt][0], l0, l1, l2, l3, r0, r1);
              mma_bf16_16816(acc[mt][1], h0, h1, h2, h3, r2, r3);
              mma_bf16_16816(acc[mt][1], l0, l1, l2, l3, r2, r3);
            }
          }
        }
      }
    }
#pragma unroll
    for (int mt = 0; mt < kBwMaxSel / 16; ++mt) {
      if (mt < nmt) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int j = 16 * warp + 8 * nt + 2 * tq;
          const int e0 = 16 * mt + gq, e1 = e0 + 8;
          if (e0 < nh) *reinterpret_cast<float2*>(U + e0 * kDim + j) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
          if (e1 < nh) *reinterpret_cast<float2*>(U + e1 * kDim + j) = make_float2(acc[mt][nt][2], acc[mt][nt][3]);
        }
      }
    }
  }
  __syncthreads();
  BWD_TRACE(4);  // u = P W_k done
  // RMS, k~_e and the gate scores s_ge (warp per entry)
  auto key_of = [&](int e, float* kk, float& inv) {
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      kk[k] = U[e * kDim + lane + 32 * k];
      ss = fmaf(kk[k], kk[k], ss);
    }
    ss = warp_sum(ss);
    inv = 1.f / sqrtf(ss / kDim + p.eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) kk[k] = kk[k] * inv * p.gamma_k[lane + 32 * k];
    float c0, s0, c1, s1;
    rope_cos_sin(p.rope.theta_over_pi[lane], sel[e], c0, s0);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], sel[e], c1, s1);
    const float y0 = kk[0] * c0 - kk[2] * s0, y2 = kk[2] * c0 + kk[0] * s0;
    const float y1 = kk[1] * c1 - kk[3] * s1, y3 = kk[3] * c1 + kk[1] * s1;
    kk[0] = y0;
    kk[1] = y1;
    kk[2] = y2;
    kk[3] = y3;
  };
  for (int e = warp; e < nh; e += kW) {
    float kk[4], inv;
    key_of(e, kk, inv);
    if (lane == 0) ru[e] = inv;
#pragma unroll
    for (int k = 0; k < 4; ++k) ktl[e * kDim + lane + 32 * k] = kk[k];
    for (int g = 0; g < G; ++g) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) a = fmaf(qt[g * kDim + lane + 32 * k], kk[k], a);
      a = warp_sum(a);
      if (lane == 0) sg[e * G + g] = a * p.gate_scale;
    }
  }
  __syncthreads();

  BWD_TRACE(5);  // gate keys and scores done
  // ---- 4. biased statistics per head; dL/dbias and dL/ds per entry
  for (int g = warp; g < G; g += kW) {
    float mx = -INFINITY;
    for (int e = lane; e < m; e += 32) {
      const float bias = (e < nh) ? log_sigmoid_f(sg[e * G + g]) : 0.f;
      mx = fmaxf(mx, st_m[e * G + g] + bias);
    }
    mx = warp_max(mx);
    float l = 0.f, yy = 0.f;
    for (int e = lane; e < m; e += 32) {
      const float bias = (e < nh) ? log_sigmoid_f(sg[e * G + g]) : 0.f;
      const float me = st_m[e * G + g] + bias;
      const float f = (me == -INFINITY) ? 0.f : expf(me - mx);
      l = fmaf(f, st_z[e * G + g], l);
      yy = fmaf(f, st_y[e * G + g], yy);
    }
    l = warp_sum(l);
    yy = warp_sum(yy);
    const float D = yy / l;  // dout_g . out_g
    for (int e = lane; e < nh; e += 32) {
      const float se = sg[e * G + g];
      const float me = st_m[e * G + g] + log_sigmoid_f(se);
      const float f = (me == -INFINITY) ? 0.f : expf(me - mx) / l;
      const float dbias = f * (st_y[e * G + g] - st_z[e * G + g] * D);
      dsg[e * G + g] = dbias * sigmoid_f(-se);  // d log(sigmoid(s)) / ds = sigmoid(-s)
    }
  }
  __syncthreads();

  BWD_TRACE(6);  // gate gradients done
  // ---- 5. dL/dq~_g = sum_e dL/ds_ge * gate_scale * k~_e: warp g owns head g
  // (entries in order)
  for (int g = warp; g < G; g += kW) {
    float a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int e = 0; e < nh; ++e) {
      const float d = dsg[e * G + g] * p.gate_scale;
#pragma unroll
      for (int k = 0; k < 4; ++k) a[k] = fmaf(d, ktl[e * kDim + lane + 32 * k], a[k]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) dqt[g * kDim + lane + 32 * k] = a[k];
  }
  // dL/dk~_e -> dL/du_e (in place of u); dL/dgamma_k per warp
  float pgk[4] = {0.f, 0.f, 0.f, 0.f};
  for (int e = warp; e < nh; e += kW) {
    const float inv = ru[e];
    float dk[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g = 0; g < G; ++g) {
      const float d = dsg[e * G + g] * p.gate_scale;
#pragma unroll
      for (int k = 0; k < 4; ++k) dk[k] = fmaf(d, qt[g * kDim + lane + 32 * k], dk[k]);
    }
    // RoPE transposed: rotation by -b
    float c0, s0, c1, s1;
    rope_cos_sin(p.rope.theta_over_pi[lane], sel[e], c0, s0);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], sel[e], c1, s1);
    float dh[4];
    dh[0] = dk[0] * c0 + dk[2] * s0;
    dh[2] = dk[2] * c0 - dk[0] * s0;
    dh[1] = dk[1] * c1 + dk[3] * s1;
    dh[3] = dk[3] * c1 - dk[1] * s1;
    // RMSNorm backward: x = u_e, y = x * inv * gamma_k
    float u[4], dot = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      u[k] = U[e * kDim + lane + 32 * k];
      dot = fmaf(p.gamma_k[lane + 32 * k] * dh[k], u[k], dot);
    }
    dot = warp_sum(dot);
    const float inv3 = inv * inv * inv;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int d = lane + 32 * k;
      pgk[k] = fmaf(dh[k] * u[k], inv, pgk[k]);
      U[e * kDim + d] = p.gamma_k[d] * dh[k] * inv - u[k] * dot * inv3 / kDim;
    }
  }
  __syncthreads();  // dqt complete
  // dL/dq^_g -> dL/dv_g (in place of v); dL/dgamma_q per warp
  float pgq[4] = {0.f, 0.f, 0.f, 0.f};
  for (int g = warp; g < G; g += kW) {
    float c0, s0, c1, s1;
    rope_cos_sin(p.rope.theta_over_pi[lane], c, c0, s0);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], c, c1, s1);
    const float* dq = dqt + g * kDim;
    float dh[4];
    dh[0] = dq[lane] * c0 + dq[lane + 64] * s0;
    dh[2] = dq[lane + 64] * c0 - dq[lane] * s0;
    dh[1] = dq[lane + 32] * c1 + dq[lane + 96] * s1;
    dh[3] = dq[lane + 96] * c1 - dq[lane + 32] * s1;
    float x[4], ss = 0.f, dot = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[k] = vq[g * kDim + lane + 32 * k];
      ss = fmaf(x[k], x[k], ss);
      dot = fmaf(p.gamma_q[lane + 32 * k] * dh[k], x[k], dot);
    }
    ss = warp_sum(ss);
    dot = warp_sum(dot);
    const float inv = 1.f / sqrtf(ss / kDim + p.eps);
    const float inv3 = inv * inv * inv;
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int d = lane + 32 * k;
      pgq[k] = fmaf(dh[k] * x[k], inv, pgq[k]);
      vq[g * kDim + d] = p.gamma_q[d] * dh[k] * inv - x[k] * dot * inv3 / kDim;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    red[warp * kDim + lane + 32 * k] = pgq[k];
    red[(kW + warp) * kDim + lane + 32 * k] = pgk[k];
  }
  __syncthreads();
  // the gain gradients: warps summed in order
  {
    const int d = tid & (kDim - 1), which = tid >> 7;  // 0: gamma_q, 1: gamma_k
    float a = 0.f;
    for (int w = 0; w < kW; ++w) a += red[(which * kW + w) * kDim + d];
    (which == 0 ? dgq : dgk)[d] = a;
  }
  __syncthreads();

  BWD_TRACE(7);  // back through the norms done
  // ---- 6. the pair's terms into the workspace (the reduction adds them up)
  for (int i = tid; i < G * kDim; i += kBwThreads) p.ws_dv[qoff + i] = vq[i];
  {
    float* wp = p.ws_p + static_cast<size_t>(pair) * MS * kPool;
    float* wu = p.ws_du + static_cast<size_t>(pair) * MS * kDim;
    for (int i = tid; i < nh * kPool; i += kBwThreads) wp[i] = P[(i / kPool) * kPs + i % kPool];
    for (int i = tid; i < nh * kDim; i += kBwThreads) wu[i] = U[i];
  }
  if (tid < kDim) {
    p.ws_dg[(static_cast<size_t>(pair) * 2) * kDim + tid] = dgq[tid];
    p.ws_dg[(static_cast<size_t>(pair) * 2 + 1) * kDim + tid] = dgk[tid];
  }
  if (tid == 0) p.ws_nh[pair] = nh;
  BWD_TRACE(8);
}

// Sums of the per-pair terms, added to the caller's gradient arrays.  Blocks
// [0, Hq * 8): 16 rows of dW_q[hq] each; then Hkv * 24 blocks of 16 rows of
// dW_k[h]; the last block the two gain gradients.  Thread (rp, j) owns
// column j of rows rp, rp + 2, .. of its block's 16 and sums in a fixed order
// (sequences, then entries).  A pair the kernel skipped (a bad block list)
// contributes nothing.
constexpr int kRedRows = 16;

__global__ void __launch_bounds__(kBwThreads) gate_grad_reduce_kernel(const __grid_constant__ GateBwdParams p) {
  const int tid = threadIdx.x;
  const int j = tid & (kDim - 1), rp = tid >> 7;
  constexpr int kPer = kRedRows / (kBwThreads / kDim);  // rows per thread
  const int nq = p.hq * (kDim / kRedRows);
  const int nk = p.hkv * (kPool / kRedRows);
  const int blk = blockIdx.x;
  const int MS = p.max_sel;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  if (blk < nq) {
    const int hq = blk / (kDim / kRedRows);
    const int i0 = (blk - hq * (kDim / kRedRows)) * kRedRows + rp;
    const int h = hq / p.G;
#pragma unroll 4
    for (int s = 0; s < p.batch; ++s) {
      const bool live = p.ws_nh[s * p.hkv + h] >= 0;
      const float dv = live ? p.ws_dv[(static_cast<size_t>(s) * p.hq + hq) * kDim + j] : 0.f;
      const __nv_bfloat16* qr = p.q + (static_cast<size_t>(s) * p.hq + hq) * kDim;
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] = fmaf(__bfloat162float(qr[i0 + 2 * k]), dv, acc[k]);
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) p.dw_q[(static_cast<size_t>(hq) * kDim + i0 + 2 * k) * kDim + j] += acc[k];
  } else if (blk < nq + nk) {
    // rounds of up to 32 entries of one sequence (sequences ascending, then
    // entries): the dL/du rows and this block's 16 pooled columns staged in
    // shared memory, double-buffered -- the next round's 16-byte loads are
    // in flight in registers while this round is summed in order
    __shared__ __align__(16) float sdu[2][32][kDim];
    __shared__ __align__(16) float sp[2][32][kRedRows];
    const int b = blk - nq;
    const int h = b / (kPool / kRedRows);
    const int r0 = (b - h * (kPool / kRedRows)) * kRedRows;
    constexpr int kDuVec = 32 * (kDim / 4) / kBwThreads;  // float4 of dL/du per thread and round
    auto nh_of = [&](int s) { return max(p.ws_nh[s * p.hkv + h], 0); };
    float4 rdu[kDuVec];
    float4 rsp = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fetch = [&](int s, int e0, int ne) {
      const size_t pr = static_cast<size_t>(s) * p.hkv + h;
      const float4* src = reinterpret_cast<const float4*>(p.ws_du + (pr * MS + e0) * kDim);
#pragma unroll
      for (int q = 0; q < kDuVec; ++q) {
        const int i = tid + q * kBwThreads;
        rdu[q] = (i < ne * (kDim / 4)) ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (tid < ne * (kRedRows / 4)) {
        const int e = tid / (kRedRows / 4), c4 = tid % (kRedRows / 4);
        rsp = reinterpret_cast<const float4*>(p.ws_p + (pr * MS + e0 + e) * kPool + r0)[c4];
      }
    };
    auto stash = [&](int buf, int ne) {
#pragma unroll
      for (int q = 0; q < kDuVec; ++q) {
        const int i = tid + q * kBwThreads;
        if (i < ne * (kDim / 4)) reinterpret_cast<float4*>(&sdu[buf][0][0])[i] = rdu[q];
      }
      if (tid < ne * (kRedRows / 4))
        reinterpret_cast<float4*>(&sp[buf][tid / (kRedRows / 4)][0])[tid % (kRedRows / 4)] = rsp;
    };
    int s = 0, e0 = 0;
    while (s < p.batch && nh_of(s) == 0) ++s;
    int ne = (s < p.batch) ? min(32, nh_of(s)) : 0;
    if (s < p.batch) fetch(s, e0, ne);
    for (int buf = 0; s < p.batch; buf ^= 1) {
      // the reads of this buffer two rounds ago ended before the barrier of
      // the last round
      stash(buf, ne);
      __syncthreads();
      int s2 = s, e2 = e0 + 32;
      if (e2 >= nh_of(s2)) {
        e2 = 0;
        ++s2;
        while (s2 < p.batch && nh_of(s2) == 0) ++s2;
      }
      const int ne2 = (s2 < p.batch) ? min(32, nh_of(s2) - e2) : 0;
      if (s2 < p.batch) fetch(s2, e2, ne2);
      for (int e = 0; e < ne; ++e) {
        const float d = sdu[buf][e][j];
#pragma unroll
        for (int k = 0; k < kPer; ++k) acc[k] = fmaf(sp[buf][e][rp + 2 * k], d, acc[k]);
      }
      s = s2;
      e0 = e2;
      ne = ne2;
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) p.dw_k[(static_cast<size_t>(h) * kPool + r0 + rp + 2 * k) * kDim + j] += acc[k];
  } else {
    // thread (rp, j): gamma_q (rp = 0) or gamma_k (rp = 1), element j
    float a = 0.f;
#pragma unroll 16
    for (int pair = 0; pair < p.batch * p.hkv; ++pair) {
      const float x = p.ws_dg[(static_cast<size_t>(pair) * 2 + rp) * kDim + j];
      a += (p.ws_nh[pair] >= 0) ? x : 0.f;
    }
    (rp == 0 ? p.dgamma_q : p.dgamma_k)[j] += a;
  }
}

cudaError_t launch_gate_backward(const GateBwdParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                 const CUtensorMap& tmwk, cudaStream_t stream) {
  const int smem = gate_bwd_smem_bytes(p.G, p.max_sel, p.stages);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * p.batch * p.hkv), 1, 1);
  cfg.blockDim = dim3(kBwThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gate_backward_kernel, p, tmk, tmv, tmwk);
  if (e != cudaSuccess) return e;
  const unsigned nblk = static_cast<unsigned>(p.hq * (kDim / kRedRows) + p.hkv * (kPool / kRedRows) + 1);
  gate_grad_reduce_kernel<<<nblk, kBwThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t prepare_backward_kernels() {
  return cudaFuncSetAttribute(gate_backward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

}  // namespace sas
