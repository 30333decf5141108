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
// One CTA (256 threads) per (sequence, KV head):
//   1. q, dout and the gains into shared memory; v_g = q_g @ W_q[g]; RMSNorm,
//      gain, RoPE -> q~_g.
//   2. one pass over the block list, K and V blocks by TMA bulk copy into a
//      two-stage ring (one stage for 8-head groups at lists of 64 blocks,
//      where two do not fit): the pooled key [max; min; mean] of every historical
//      entry, and per (entry, head) the softmax statistics of the block
//      without its bias -- max m', sum z' of exp(logit - m'), sum y' of
//      exp(logit - m') (dout . v_j).  A bias constant over the block only
//      shifts m', so the biased statistics follow once the gates are known.
//   3. u_e = P_e @ W_k[h] for every historical entry (W_k read once, each
//      element used for all entries); RMSNorm, gain, RoPE -> k~_e; s_ge.
//   4. per head: the global max, sum and D_g = dout_g . out_g from the
//      per-entry statistics with the biases; dL/dbias_ge and dL/ds_ge.
//   5. dL/dq~_g and dL/dk~_e; RoPE transposed (rotation by -pos); RMSNorm
//      backward; dL/dv_g, dL/du_e and the gain gradients.
//   6. dL/dW_q[g] += q_g (x) dL/dv_g, dL/dW_k[h] += sum_e P_e (x) dL/du_e and
//      the gain gradients, added to the caller's arrays with atomics.
#include <cmath>

#include "sas_internal.h"

namespace sas {

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

__global__ void __launch_bounds__(kBwThreads, 1) gate_backward_kernel(const __grid_constant__ GateBwdParams p) {
  constexpr int kW = kBwThreads / 32;  // warps
  const int pair = blockIdx.x;
  const int s = pair / p.hkv;
  const int h = pair - s * p.hkv;
  const int G = p.G;
  const int MS = p.max_sel;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // carve (the order of gate_bwd_smem_bytes)
  const int NS = p.stages;                                            // K/V ring stages (1 or 2)
  uint8_t* tiles = base;                                              // [NS stages][K, V] bf16 [64][128]
  float* P = reinterpret_cast<float*>(tiles + 2 * NS * kTileBytes);   // [MS][384]
  float* U = P + MS * kPool;                                          // [MS][128] u, then dL/du
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
  float* scratch = ru + MS;                                           // [3][128] (unused slack)
  float* dqt = scratch + 3 * kDim;                                    // [G][128] dL/dq~
  float* dgq = dqt + G * kDim;                                        // [128]
  float* dgk = dgq + kDim;                                            // [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(dgk + kDim) + 7) & ~uintptr_t(7));

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
  if (__syncthreads_or(err)) {
    if (tid == 0) raise_status(p.status, kStatusBounds);
    return;
  }
  const int nh = m - 1;  // historical entries (the current block, last, has no gate)

  // ---- K/V ring: entry e in stage e % NS (16 KiB K then 16 KiB V)
  auto issue = [&](int e) {
    const int st = e % NS;
    const long long row0 = p.kv.block_row(s, h, sel[e]);
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.kv.k) + row0 * kDim;
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(p.kv.v) + row0 * kDim;
    mbar_arrive_expect_tx(&bars[st], 2 * kTileBytes);
    bulk_g2s(tiles + (2 * st) * kTileBytes, kb, kTileBytes, &bars[st]);
    bulk_g2s(tiles + (2 * st + 1) * kTileBytes, vb, kTileBytes, &bars[st]);
  };
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    issue(0);
    if (m > 1 && NS > 1) issue(1);
  }

  // ---- 1. gate query: v_g = q_g @ W_q[g], RMSNorm, gain, RoPE at c
  const size_t qoff = (static_cast<size_t>(s) * p.hq + static_cast<size_t>(h) * G) * kDim;
  for (int i = tid; i < G * kDim; i += kBwThreads) {
    qf[i] = __bfloat162float(p.q[qoff + i]);
    dof[i] = p.d_out[qoff + i];
  }
  if (tid < kDim) {
    dgq[tid] = 0.f;
    dgk[tid] = 0.f;
  }
  for (int i = tid; i < G * kDim; i += kBwThreads) dqt[i] = 0.f;
  __syncthreads();
  for (int o = tid; o < G * kDim; o += kBwThreads) {
    const int g = o >> 7, j = o & (kDim - 1);
    const __nv_bfloat16* wcol = p.w_q + (static_cast<size_t>(h * G + g) * kDim) * kDim + j;
    const float* qrow = qf + g * kDim;
    float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int i = 0; i < kDim; ++i) a4[i & 3] = fmaf(qrow[i], __bfloat162float(wcol[static_cast<size_t>(i) * kDim]), a4[i & 3]);
    vq[o] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
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

  // ---- 2. pass over the list: pooled keys and unbiased block statistics
  const float alpha = p.attn_scale;
  for (int e = 0; e < m; ++e) {
    const int st = e % NS;
    const bool ok = mbar_wait(&bars[st], (e / NS) & 1, p.status);
    const int b = sel[e];
    const int nvalid = (b == c) ? (L - b * kBlock) : kBlock;
    const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(tiles + (2 * st) * kTileBytes);
    const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(tiles + (2 * st + 1) * kTileBytes);
    if (b != c && tid < kDim) {
      float mx = -INFINITY, mn = INFINITY, sm = 0.f;
      if (ok) {
#pragma unroll 8
        for (int t = 0; t < kBlock; ++t) {
          const float x = __bfloat162float(kt[t * kDim + tid]);
          mx = fmaxf(mx, x);
          mn = fminf(mn, x);
          sm += x;
        }
      }
      P[e * kPool + tid] = mx;
      P[e * kPool + kDim + tid] = mn;
      P[e * kPool + 2 * kDim + tid] = sm * (1.f / kBlock);
    }
    // logits and dout . v_j: warp w takes tokens w, w + 8, ...; lane l holds
    // dimensions 4l .. 4l + 3
    for (int j = warp; j < kBlock; j += kW) {
      if (j >= nvalid) {
        if (lane < G) {
          lg[lane * kBlock + j] = -INFINITY;
          wg[lane * kBlock + j] = 0.f;
        }
        continue;
      }
      const uint2 kr = *reinterpret_cast<const uint2*>(kt + j * kDim + 4 * lane);
      const uint2 vr = *reinterpret_cast<const uint2*>(vt + j * kDim + 4 * lane);
      const float k0 = bf16_lo(kr.x), k1 = bf16_hi(kr.x), k2 = bf16_lo(kr.y), k3 = bf16_hi(kr.y);
      const float v0 = bf16_lo(vr.x), v1 = bf16_hi(vr.x), v2 = bf16_lo(vr.y), v3 = bf16_hi(vr.y);
      for (int g = 0; g < G; ++g) {
        const float4 q4 = *reinterpret_cast<const float4*>(qf + g * kDim + 4 * lane);
        const float4 d4 = *reinterpret_cast<const float4*>(dof + g * kDim + 4 * lane);
        float a = q4.x * k0 + q4.y * k1 + q4.z * k2 + q4.w * k3;
        float w = d4.x * v0 + d4.y * v1 + d4.z * v2 + d4.w * v3;
        a = warp_sum(a);
        w = warp_sum(w);
        if (lane == 0) {
          lg[g * kBlock + j] = ok ? a * alpha : -INFINITY;
          wg[g * kBlock + j] = ok ? w : 0.f;
        }
      }
    }
    __syncthreads();  // every read of this stage is done, the block's values are in
    if (tid == 0 && e + NS < m) {
      fence_proxy_async_smem();
      issue(e + NS);
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
    __syncthreads();  // lg / wg are rewritten by the next entry
  }

  // ---- 3. gate keys of the historical entries: u_e = P_e @ W_k[h]
  {
    const int j = tid & (kDim - 1);
    const int half = tid >> 7;  // entries half, half + 2, ...
    const __nv_bfloat16* wk = p.w_k + static_cast<size_t>(h) * kPool * kDim + j;
    constexpr int kMaxRows = kBwMaxSel / 2;
    float acc[kMaxRows];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
    const int nrows = (nh - half + 1) / 2;  // entries of this thread
    for (int i = 0; i < kPool; ++i) {
      const float w = __bfloat162float(wk[static_cast<size_t>(i) * kDim]);
#pragma unroll
      for (int r = 0; r < kMaxRows; ++r)
        if (r < nrows) acc[r] = fmaf(P[(half + 2 * r) * kPool + i], w, acc[r]);
    }
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < nrows) U[(half + 2 * r) * kDim + j] = acc[r];
  }
  __syncthreads();
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
    for (int g = 0; g < G; ++g) {
      float a = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) a = fmaf(qt[g * kDim + lane + 32 * k], kk[k], a);
      a = warp_sum(a);
      if (lane == 0) sg[e * G + g] = a * p.gate_scale;
    }
  }
  __syncthreads();

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

  // ---- 5. dL/dq~_g (summed over entries), dL/dk~_e -> dL/du_e, dL/dgamma_k
  for (int e = warp; e < nh; e += kW) {
    float kk[4], inv;
    key_of(e, kk, inv);
    float dk[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g = 0; g < G; ++g) {
      const float d = dsg[e * G + g] * p.gate_scale;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        atomicAdd(&dqt[g * kDim + lane + 32 * k], d * kk[k]);
        dk[k] = fmaf(d, qt[g * kDim + lane + 32 * k], dk[k]);
      }
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
      atomicAdd(&dgk[d], dh[k] * u[k] * inv);
      U[e * kDim + d] = p.gamma_k[d] * dh[k] * inv - u[k] * dot * inv3 / kDim;
    }
  }
  __syncthreads();
  // dL/dq^_g -> dL/dv_g (in place of v), dL/dgamma_q
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
      atomicAdd(&dgq[d], dh[k] * x[k] * inv);
      vq[g * kDim + d] = p.gamma_q[d] * dh[k] * inv - x[k] * dot * inv3 / kDim;
    }
  }
  __syncthreads();

  // ---- 6. weight and gain gradients into the caller's arrays
  for (int o = tid; o < G * kDim * kDim; o += kBwThreads) {
    const int g = o / (kDim * kDim);
    const int r = o - g * kDim * kDim;
    const int i = r >> 7, j = r & (kDim - 1);
    atomicAdd(&p.dw_q[(static_cast<size_t>(h * G + g) * kDim + i) * kDim + j], qf[g * kDim + i] * vq[g * kDim + j]);
  }
  {
    const int j = tid & (kDim - 1);
    for (int i = tid >> 7; i < kPool; i += kBwThreads / kDim) {
      float a = 0.f;
      for (int e = 0; e < nh; ++e) a = fmaf(P[e * kPool + i], U[e * kDim + j], a);
      if (nh > 0) atomicAdd(&p.dw_k[(static_cast<size_t>(h) * kPool + i) * kDim + j], a);
    }
  }
  if (tid < kDim) {
    atomicAdd(&p.dgamma_q[tid], dgq[tid]);
    atomicAdd(&p.dgamma_k[tid], dgk[tid]);
  }
}

cudaError_t launch_gate_backward(const GateBwdParams& p, int batch, cudaStream_t stream) {
  const int smem = gate_bwd_smem_bytes(p.G, p.max_sel, p.stages);
  gate_backward_kernel<<<static_cast<unsigned>(batch * p.hkv), kBwThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t prepare_backward_kernels() {
  return cudaFuncSetAttribute(gate_backward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

}  // namespace sas
