// SAS prefill gate backward: the gradient of the gated block-sparse prefill
// with respect to the gate parameters W_q, W_k, gamma_q and gamma_k.
//
// Method (release pages: "Tencent released Simple-Attention-Sparsification
// ..." aigc.news 2026-09-14, release paragraph -- continuous gates on the
// selected blocks make the discrete Top-K selection trainable): in the gated
// mode every token of a selected historical block b gets, for query head g
// of query block i, the logit bias log(sigmoid(s_gib)), s_gib = q~_gi .
// k~_b * gate_scale, where q~_gi is built from the mean of the block's 64
// queries.  For an upstream gradient dL/dout, with the block lists held
// fixed,
//   dL/ds_gib = sum over the block's query tokens t and key tokens j of
//               p_tj (dout_t . v_j - dout_t . out_t), times sigmoid(-s_gib),
// then back through the score, the RoPEs, the RMSNorms and the projections;
// a gate key's gradient sums over the query blocks that kept it.
//
// Four kernels:
//   prefill_bwd_attn_kernel, one CTA (4 warps) per (sequence, query head,
//     query block i): the block-mean gate query q_bar, v = q_bar @ W_q[g],
//     RMSNorm, RoPE at i -> q~; one pass over the block list with K and V by
//     2-D TMA (128-byte swizzle) through a ring: the logits q_t . k_j and
//     dout_t . v_j on bf16 mma.sync (each warp 16 query tokens x 64 keys; Q
//     and dout held as register fragments for the whole pass, dout as hi +
//     lo bf16 terms), and per (entry, token) the block's unbiased softmax
//     statistics m', z', y'.  The gates only shift a block's logits, so the
//     biased log-sum-exp, dout . out and dL/dbias follow from those
//     statistics once the gate scores are known.  dL/ds per entry, then
//     dL/dq~ -> RoPE transposed -> RMSNorm backward -> dL/dv; q_bar, q~,
//     dL/dv, the gamma_q term and every entry's dL/ds into the workspace.
//   prefill_bwd_keys_kernel, one CTA per (sequence, KV head, 128 key
//     blocks): which query blocks kept each key block (a bitmap built from
//     the lists); dL/dk~_b summed over them in a fixed order; the pooled
//     key P_b and u_b = P_b @ W_k[h] recomputed from the cache; RoPE
//     transposed, RMSNorm backward -> dL/du_b; P_b, dL/du_b and the gamma_k
//     term into the workspace.
//   prefill_grad_reduce_kernel: dW_q[g] += sum_(s,i) q_bar (x) dL/dv and
//     dW_k[h] += sum_(s,b) P_b (x) dL/du_b (rounds of 32 terms staged in
//     shared memory), and per-head sums of the gain terms;
//   prefill_gamma_final_kernel: the gain gradients from the per-head sums.
// Every sum runs in a fixed order (no atomics): repeated calls add identical
// values.
#include <cmath>

#include "sas_internal.h"

namespace sas {

namespace {

__device__ __forceinline__ float warp_sum_pb(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float log_sigmoid_pb(float x) {
  return (x >= 0.f) ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

__device__ __forceinline__ float sigmoid_pb(float x) {
  return (x >= 0.f) ? 1.f / (1.f + expf(-x)) : expf(x) / (1.f + expf(x));
}

}  // namespace

__global__ void __launch_bounds__(kPbThreads, 2)
    prefill_bwd_attn_kernel(const __grid_constant__ PrefillBwdParams p, const __grid_constant__ CUtensorMap tmq,
                            const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  const int i = blockIdx.x, hq = blockIdx.y, s = blockIdx.z;
  const int h = hq / p.G;
  const int MS = p.max_sel, NS = p.stages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tq = lane & 3, gq = lane >> 2, mat = lane >> 3;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = base;                                  // [NS][K, V] swizzled 64 x 128 bf16
  uint8_t* region = tiles + NS * 2 * kTileBytes;          // Q tile, then the statistics
  const int stats_bytes = 3 * MS * 64 * 4;
  float* st_m = reinterpret_cast<float*>(region);         // [MS][64] block max (no bias)
  float* st_z = st_m + MS * 64;                           // [MS][64] sum exp, then dL/dbias terms
  float* st_y = st_z + MS * 64;                           // [MS][64] sum exp * (dout . v)
  int* sel = reinterpret_cast<int*>(region + (stats_bytes > kTileBytes ? stats_bytes : kTileBytes));
  float* sc = reinterpret_cast<float*>(sel + MS);          // [MS] gate scores
  float* beta = sc + MS;                                   // [MS] log-sigmoid gates
  float* dsv = beta + MS;                                  // [MS] dL/ds
  float* qbar = dsv + MS;                                  // [128]
  float* vq = qbar + kDim;                                 // [128] v, then dL/dv
  float* qt = vq + kDim;                                   // [128] q~
  float* dqt = qt + kDim;                                  // [128] dL/dq~
  float* red = dqt + kDim;                                 // [8] reductions
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * kDim);  // [NS] ring, [4] Q

  const size_t vrow = ((static_cast<size_t>(s) * p.hq + hq) * p.nblk + i) * kDim;  // [B][Hq][nblk][128]
  const size_t lrow = (static_cast<size_t>(s) * p.hkv + h) * p.nblk + i;           // list index

  // ---- the block list (checked like the forward's)
  const int m = p.sel_count[lrow];
  bool err = m < 1 || m > MS;
  if (!err) {
    const int32_t* si = p.sel_idx + lrow * MS;
    for (int e = tid; e < m; e += kPbThreads) {
      const int b = si[e];
      sel[e] = b;
      if (b < 0 || b > i) err = true;
      if (e == m - 1 && b != i) err = true;
      if (e > 0 && si[e - 1] >= b) err = true;
    }
  }
  const bool bad = __syncthreads_or(err) != 0;
  const int nh = bad ? 0 : m - 1;  // historical entries
  if (bad && tid == 0) raise_status(p.status, kStatusBounds);
  if (nh == 0) {  // nothing kept (or a bad list): no gate, no gradient
    for (int d = tid; d < kDim; d += kPbThreads) {
      p.ws_qbar[vrow + d] = 0.f;
      p.ws_qt[vrow + d] = 0.f;
      p.ws_dv[vrow + d] = 0.f;
      p.ws_dgq[vrow + d] = 0.f;
    }
    return;
  }

  // ---- ring of K/V tiles; the Q tile first, into the statistics region
  const int qrow0 = static_cast<int>((static_cast<size_t>(s) * p.hq + hq) * p.T + static_cast<size_t>(i) * kBlock);
  const int krow_base = static_cast<int>((static_cast<size_t>(s) * p.hkv + h) * p.T);
  auto issue = [&](int e) {
    const int st = e % NS;
    uint8_t* kd = tiles + (2 * st) * kTileBytes;
    const int row0 = krow_base + sel[e] * kBlock;
    mbar_arrive_expect_tx(&bars[st], 2 * kTileBytes);
    tma_load_2d(kd, &tmk, 0, row0, &bars[st]);
    tma_load_2d(kd + 8192, &tmk, 64, row0, &bars[st]);
    tma_load_2d(kd + kTileBytes, &tmv, 0, row0, &bars[st]);
    tma_load_2d(kd + kTileBytes + 8192, &tmv, 64, row0, &bars[st]);
  };
  uint64_t* bar_q = &bars[4];
  if (tid == 0) {
    prefetch_tensormap(&tmq);
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
    for (int st = 0; st < NS; ++st) mbar_init(&bars[st], 1);
    mbar_init(bar_q, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar_q, kTileBytes);
    tma_load_2d(region, &tmq, 0, qrow0, bar_q);
    tma_load_2d(region + 8192, &tmq, 64, qrow0, bar_q);
    for (int e = 0; e < NS && e < m; ++e) issue(e);
  }
  __syncthreads();

  // ---- dout fragments (rows 16 warp + gq, + 8; 8 k-steps), as hi + lo bf16
  const int t0 = 16 * warp + gq, t1 = t0 + 8;
  uint32_t dh[8][4], dl[8][4];
  {
    const float* d0 = p.d_out + (static_cast<size_t>(qrow0) + t0) * kDim;
    const float* d1 = p.d_out + (static_cast<size_t>(qrow0) + t1) * kDim;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c = 16 * ks + 2 * tq;
      const float2 x00 = *reinterpret_cast<const float2*>(d0 + c), x02 = *reinterpret_cast<const float2*>(d0 + c + 8);
      const float2 x10 = *reinterpret_cast<const float2*>(d1 + c), x12 = *reinterpret_cast<const float2*>(d1 + c + 8);
      dh[ks][0] = pack_bf16x2(x00.x, x00.y);
      dh[ks][1] = pack_bf16x2(x10.x, x10.y);
      dh[ks][2] = pack_bf16x2(x02.x, x02.y);
      dh[ks][3] = pack_bf16x2(x12.x, x12.y);
      dl[ks][0] = pack_bf16x2(x00.x - bf16_lo(dh[ks][0]), x00.y - bf16_hi(dh[ks][0]));
      dl[ks][1] = pack_bf16x2(x10.x - bf16_lo(dh[ks][1]), x10.y - bf16_hi(dh[ks][1]));
      dl[ks][2] = pack_bf16x2(x02.x - bf16_lo(dh[ks][2]), x02.y - bf16_hi(dh[ks][2]));
      dl[ks][3] = pack_bf16x2(x12.x - bf16_lo(dh[ks][3]), x12.y - bf16_hi(dh[ks][3]));
    }
  }

  // ---- Q: register fragments and the block mean
  const bool okq = mbar_wait(bar_q, 0, p.status);
  uint32_t qa[8][4];
  {
    const uint32_t qb = smem_u32(region);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      ldsm_x4(qb + swz_tile_offset(16 * warp + (lane & 15), 2 * ks + (lane >> 4)), qa[ks][0], qa[ks][1], qa[ks][2],
              qa[ks][3]);
  }
  if (tid < kDim) {
    const uint8_t* q8 = region + (tid & 7) * 2;
    float a = 0.f;
    if (okq) {
#pragma unroll 8
      for (int t = 0; t < kBlock; ++t)
        a += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(q8 + swz_tile_offset(t, tid >> 3)));
    }
    qbar[tid] = a * (1.f / kBlock);
  }
  __syncthreads();  // the Q tile is read (fragments, mean): the region holds statistics from here on
  // gate query: v = q_bar @ W_q[hq] (thread j owns column j), RMSNorm, RoPE at i
  if (tid < kDim) {
    const __nv_bfloat16* wcol = p.w_q + static_cast<size_t>(hq) * kDim * kDim + tid;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 16
    for (int r = 0; r < kDim; r += 2) {
      a0 = fmaf(qbar[r], __bfloat162float(wcol[static_cast<size_t>(r) * kDim]), a0);
      a1 = fmaf(qbar[r + 1], __bfloat162float(wcol[static_cast<size_t>(r + 1) * kDim]), a1);
    }
    vq[tid] = a0 + a1;
  }
  __syncthreads();
  if (warp == 0) {
    float x[4], ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[k] = vq[lane + 32 * k];
      ss = fmaf(x[k], x[k], ss);
    }
    ss = warp_sum_pb(ss);
    const float inv = 1.f / sqrtf(ss / kDim + p.eps);
    if (lane == 0) red[0] = inv;
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = x[k] * inv * p.gamma_q[lane + 32 * k];
    float c0, s0, c1, s1;
    rope_cos_sin(p.rope.theta_over_pi[lane], i, c0, s0);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], i, c1, s1);
    qt[lane] = x[0] * c0 - x[2] * s0;
    qt[lane + 64] = x[2] * c0 + x[0] * s0;
    qt[lane + 32] = x[1] * c1 - x[3] * s1;
    qt[lane + 96] = x[3] * c1 + x[1] * s1;
  }

  // ---- one pass over the list: unbiased statistics per (entry, token)
  const float alpha = p.attn_scale;
  for (int e = 0; e < m; ++e) {
    const int st = e % NS;
    const bool ok = mbar_wait(&bars[st], (e / NS) & 1, p.status);
    const uint32_t kb = smem_u32(tiles + (2 * st) * kTileBytes);
    const uint32_t vb = kb + kTileBytes;
    float as[8][4], aw[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) as[nt][0] = as[nt][1] = as[nt][2] = as[nt][3] = aw[nt][0] = aw[nt][1] = aw[nt][2] = aw[nt][3] = 0.f;
    if (ok) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int tok = 16 * np + (mat >> 1) * 8 + (lane & 7);
          const uint32_t off = swz_tile_offset(tok, 2 * ks + (mat & 1));
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kb + off, r0, r1, r2, r3);
          mma_bf16_16816(as[2 * np], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r0, r1);
          mma_bf16_16816(as[2 * np + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r2, r3);
          ldsm_x4(vb + off, r0, r1, r2, r3);
          mma_bf16_16816(aw[2 * np], dh[ks][0], dh[ks][1], dh[ks][2], dh[ks][3], r0, r1);
          mma_bf16_16816(aw[2 * np], dl[ks][0], dl[ks][1], dl[ks][2], dl[ks][3], r0, r1);
          mma_bf16_16816(aw[2 * np + 1], dh[ks][0], dh[ks][1], dh[ks][2], dh[ks][3], r2, r3);
          mma_bf16_16816(aw[2 * np + 1], dl[ks][0], dl[ks][1], dl[ks][2], dl[ks][3], r2, r3);
        }
      }
    }
    __syncthreads();  // every read of this stage is done
    if (tid == 0 && e + NS < m) {
      fence_proxy_async_smem();
      issue(e + NS);
    }
    const bool diag = (e == m - 1);
#pragma unroll
    for (int r = 0; r < 2; ++r) {  // row t0 (r = 0) or t1 (r = 1)
      const int t = r ? t1 : t0;
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int j = 8 * nt + 2 * tq + c;
          const bool live = ok && (!diag || j <= t);
          if (live) mx = fmaxf(mx, as[nt][2 * r + c] * alpha);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float z = 0.f, y = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int j = 8 * nt + 2 * tq + c;
          const bool live = ok && (!diag || j <= t);
          if (live) {
            const float w = expf(as[nt][2 * r + c] * alpha - mx);
            z += w;
            y = fmaf(w, aw[nt][2 * r + c], y);
          }
        }
      z += __shfl_xor_sync(0xffffffffu, z, 1);
      z += __shfl_xor_sync(0xffffffffu, z, 2);
      y += __shfl_xor_sync(0xffffffffu, y, 1);
      y += __shfl_xor_sync(0xffffffffu, y, 2);
      if (tq == 0) {
        st_m[e * 64 + t] = mx;
        st_z[e * 64 + t] = z;
        st_y[e * 64 + t] = y;
      }
    }
  }

  // ---- gate scores of the historical entries (warp per entry), gates
  for (int e = warp; e < nh; e += kPbThreads / 32) {
    const float* kr = p.gate_keys + ((static_cast<size_t>(s) * p.hkv + h) * p.mg + sel[e]) * kDim;
    float a = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) a = fmaf(qt[lane + 32 * k], kr[lane + 32 * k], a);
    a = warp_sum_pb(a) * p.gate_scale;
    if (lane == 0) {
      sc[e] = a;
      beta[e] = log_sigmoid_pb(a);
    }
  }
  if (tid == 0) beta[m - 1] = 0.f;
  __syncthreads();

  // ---- per token: biased log-sum-exp and dout . out; dL/dbias terms
  if (tid < kBlock) {
    const int t = tid;
    float M = -INFINITY;
    for (int e = 0; e < m; ++e) M = fmaxf(M, st_m[e * 64 + t] + beta[e]);
    float l = 0.f, yy = 0.f;
    for (int e = 0; e < m; ++e) {
      const float me = st_m[e * 64 + t] + beta[e];
      const float f = (me == -INFINITY) ? 0.f : expf(me - M);
      l = fmaf(f, st_z[e * 64 + t], l);
      yy = fmaf(f, st_y[e * 64 + t], yy);
    }
    const float D = yy / l;  // dout_t . out_t
    for (int e = 0; e < nh; ++e) {
      const float me = st_m[e * 64 + t] + beta[e];
      const float f = (me == -INFINITY) ? 0.f : expf(me - M) / l;
      st_z[e * 64 + t] = f * (st_y[e * 64 + t] - st_z[e * 64 + t] * D);
    }
  }
  __syncthreads();
  // dL/ds per entry (tokens summed in order)
  for (int e = tid; e < nh; e += kPbThreads) {
    float a = 0.f;
    for (int t = 0; t < kBlock; ++t) a += st_z[e * 64 + t];
    const float ds = a * sigmoid_pb(-sc[e]);
    dsv[e] = ds;
  }
  __syncthreads();
  {
    float* wds = p.ws_ds + ((static_cast<size_t>(s) * p.hq + hq) * p.nblk + i) * MS;
    for (int e = tid; e < nh; e += kPbThreads) wds[e] = dsv[e];
  }
  // dL/dq~ = gate_scale * sum_e ds_e k~_e (thread d, entries in order)
  if (tid < kDim) {
    float a = 0.f;
    const float* kb0 = p.gate_keys + (static_cast<size_t>(s) * p.hkv + h) * p.mg * kDim + tid;
    for (int e = 0; e < nh; ++e) a = fmaf(dsv[e], kb0[static_cast<size_t>(sel[e]) * kDim], a);
    dqt[tid] = a * p.gate_scale;
  }
  __syncthreads();
  // RoPE transposed (rotation by -i), RMSNorm backward -> dL/dv; gamma_q term
  if (warp == 0) {
    float c0, s0, c1, s1;
    rope_cos_sin(p.rope.theta_over_pi[lane], i, c0, s0);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], i, c1, s1);
    float dhv[4];
    dhv[0] = dqt[lane] * c0 + dqt[lane + 64] * s0;
    dhv[2] = dqt[lane + 64] * c0 - dqt[lane] * s0;
    dhv[1] = dqt[lane + 32] * c1 + dqt[lane + 96] * s1;
    dhv[3] = dqt[lane + 96] * c1 - dqt[lane + 32] * s1;
    const float inv = red[0];
    float x[4], dot = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[k] = vq[lane + 32 * k];
      dot = fmaf(p.gamma_q[lane + 32 * k] * dhv[k], x[k], dot);
    }
    dot = warp_sum_pb(dot);
    const float inv3 = inv * inv * inv;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int d = lane + 32 * k;
      p.ws_dgq[vrow + d] = dhv[k] * x[k] * inv;
      p.ws_dv[vrow + d] = p.gamma_q[d] * dhv[k] * inv - x[k] * dot * inv3 / kDim;
      p.ws_qbar[vrow + d] = qbar[d];
      p.ws_qt[vrow + d] = qt[d];
    }
  }
}

// Gate keys: dL/dk~_b summed over the query blocks that kept b, then back to
// dL/du_b.  CTA (chunk, h, s) takes key blocks [kPbChunk * chunk, + kPbChunk);
// bit (i, b) of `keep` says query block i kept block b, `base` the list slot
// of i's first entry in the chunk.  Warp w takes blocks b0 + w, b0 + w + 8, ..
__global__ void __launch_bounds__(256) prefill_bwd_keys_kernel(const __grid_constant__ PrefillBwdParams p) {
  const int s = blockIdx.z, h = blockIdx.y;
  const int c0 = blockIdx.x * kPbChunk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int MS = p.max_sel, nblk = p.nblk;
  extern __shared__ uint8_t smem_raw[];
  uint32_t* keep = reinterpret_cast<uint32_t*>(smem_raw);   // [nblk][kPbChunk / 32]
  int* sbase = reinterpret_cast<int*>(keep + static_cast<size_t>(nblk) * (kPbChunk / 32));  // [nblk]
  const size_t pr = static_cast<size_t>(s) * p.hkv + h;
  for (int w = tid; w < nblk * (kPbChunk / 32); w += blockDim.x) keep[w] = 0u;
  __syncthreads();
  // rows: query block i > c0 (only those can keep a block of the chunk)
  for (int i = c0 + 1 + tid; i < nblk; i += blockDim.x) {
    const size_t li = pr * nblk + i;
    const int m = p.sel_count[li];
    int first = -1;
    if (m >= 2 && m <= MS) {
      const int32_t* si = p.sel_idx + li * MS;
      // the list as the attention pass checked it: ascending, ending with i
      // (a rejected list has no dL/ds terms)
      bool ok = si[m - 1] == i;
      for (int e = 0; e < m - 1 && ok; ++e) ok = si[e] >= 0 && si[e] < si[e + 1];
      if (ok) {
        for (int e = 0; e < m - 1; ++e) {
          const int b = si[e];
          if (b >= c0 && b < c0 + kPbChunk) {
            if (first < 0) first = e;
            keep[i * (kPbChunk / 32) + ((b - c0) >> 5)] |= 1u << ((b - c0) & 31);
          }
        }
      }
    }
    sbase[i] = first;
  }
  __syncthreads();
  const int G = p.G;
  for (int bl = warp; bl < kPbChunk; bl += 8) {
    const int b = c0 + bl;
    if (b >= nblk) break;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int wb = bl >> 5;
    const uint32_t below = (1u << (bl & 31)) - 1u;
    for (int i0 = b + 1; i0 < nblk; i0 += 32) {
      const int i = i0 + lane;
      const bool hit = i < nblk && (keep[i * (kPbChunk / 32) + wb] >> (bl & 31) & 1u);
      int slot = 0;
      if (hit) {
        slot = sbase[i] + __popc(keep[i * (kPbChunk / 32) + wb] & below);
        for (int w2 = 0; w2 < wb; ++w2) slot += __popc(keep[i * (kPbChunk / 32) + w2]);
      }
      uint32_t mask = __ballot_sync(0xffffffffu, hit);
      while (mask != 0u) {
        const int src = __ffs(mask) - 1;
        mask &= mask - 1u;
        const int ii = __shfl_sync(0xffffffffu, i, src);
        const int sl = __shfl_sync(0xffffffffu, slot, src);
        for (int g = 0; g < G; ++g) {
          const size_t hr = (static_cast<size_t>(s) * p.hq + h * G + g) * nblk + ii;
          const float d = p.ws_ds[hr * MS + sl];
          const float* qtv = p.ws_qt + hr * kDim;
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[k] = fmaf(d, qtv[lane + 32 * k], acc[k]);
        }
      }
    }
    const size_t kr = pr * nblk + b;
    const bool any = __any_sync(0xffffffffu, acc[0] != 0.f || acc[1] != 0.f || acc[2] != 0.f || acc[3] != 0.f);
    if (!any) {  // no query block kept b: no gradient reaches its gate key
      for (int r = lane; r < kPool; r += 32) p.ws_p[kr * kPool + r] = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        p.ws_du[kr * kDim + lane + 32 * k] = 0.f;
        p.ws_dgk[kr * kDim + lane + 32 * k] = 0.f;
      }
      continue;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] *= p.gate_scale;
    // pooled key of b: lane owns dims lane + 32 k
    float mx[4], mn[4], sm[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mx[k] = -INFINITY;
      mn[k] = INFINITY;
      sm[k] = 0.f;
    }
    const __nv_bfloat16* kblk = p.k + (pr * p.T + static_cast<size_t>(b) * kBlock) * kDim;
    for (int t = 0; t < kBlock; ++t) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x = __bfloat162float(kblk[t * kDim + lane + 32 * k]);
        mx[k] = fmaxf(mx[k], x);
        mn[k] = fminf(mn[k], x);
        sm[k] += x;
      }
    }
    float P[12];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      P[k] = mx[k];
      P[4 + k] = mn[k];
      P[8 + k] = sm[k] * (1.f / kBlock);
    }
    // u = P @ W_k[h]: row r of W_k belongs to pooled dim r, held by lane r % 32 slot r / 32
    float u[4] = {0.f, 0.f, 0.f, 0.f};
    const __nv_bfloat16* wk = p.w_k + static_cast<size_t>(h) * kPool * kDim;
#pragma unroll
    for (int sl = 0; sl < 12; ++sl) {
      for (int l = 0; l < 32; ++l) {
        const float pv = __shfl_sync(0xffffffffu, P[sl], l);
        const __nv_bfloat16* wr = wk + static_cast<size_t>(32 * sl + l) * kDim;
#pragma unroll
        for (int k = 0; k < 4; ++k) u[k] = fmaf(pv, __bfloat162float(wr[lane + 32 * k]), u[k]);
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) ss = fmaf(u[k], u[k], ss);
    ss = warp_sum_pb(ss);
    const float inv = 1.f / sqrtf(ss / kDim + p.eps);
    // RoPE transposed (rotation by -b): pairs (lane, lane + 64) and (lane + 32, lane + 96)
    float c0r, s0r, c1r, s1r;
    rope_cos_sin(p.rope.theta_over_pi[lane], b, c0r, s0r);
    rope_cos_sin(p.rope.theta_over_pi[lane + 32], b, c1r, s1r);
    float dhv[4];
    dhv[0] = acc[0] * c0r + acc[2] * s0r;
    dhv[2] = acc[2] * c0r - acc[0] * s0r;
    dhv[1] = acc[1] * c1r + acc[3] * s1r;
    dhv[3] = acc[3] * c1r - acc[1] * s1r;
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) dot = fmaf(p.gamma_k[lane + 32 * k] * dhv[k], u[k], dot);
    dot = warp_sum_pb(dot);
    const float inv3 = inv * inv * inv;
#pragma unroll
    for (int sl = 0; sl < 12; ++sl) p.ws_p[kr * kPool + 32 * sl + lane] = P[sl];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int d = lane + 32 * k;
      p.ws_dgk[kr * kDim + d] = dhv[k] * u[k] * inv;
      p.ws_du[kr * kDim + d] = p.gamma_k[d] * dhv[k] * inv - u[k] * dot * inv3 / kDim;
    }
  }
}

// dW_q, dW_k and the per-head gain sums.  Blocks [0, Hq * 8): 16 rows of
// dW_q[hq]; then Hkv * 24 blocks of 16 rows of dW_k[h].  Thread (rp, j) owns
// column j of rows rp, rp + 2, .. of its block's 16; the N = B * nblk terms
// are staged 32 at a time.  The first row block of each head also sums that
// head's gain terms (column j, terms in order).
constexpr int kPbRed = 16;

__global__ void __launch_bounds__(256) prefill_grad_reduce_kernel(const __grid_constant__ PrefillBwdParams p) {
  __shared__ __align__(16) float sx[32][kDim];
  __shared__ __align__(16) float sv[32][kPbRed];
  __shared__ __align__(16) float sg[32][kDim];
  const int tid = threadIdx.x, j = tid & (kDim - 1), rp = tid >> 7;
  constexpr int kPer = kPbRed / 2;
  const int nq = p.hq * (kDim / kPbRed);
  const int blk = blockIdx.x;
  const int N = p.batch * p.nblk;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  const bool is_q = blk < nq;
  const int head = is_q ? blk / (kDim / kPbRed) : (blk - nq) / (kPool / kPbRed);
  const int r0 = is_q ? (blk - head * (kDim / kPbRed)) * kPbRed : (blk - nq - head * (kPool / kPbRed)) * kPbRed;
  // term n = (s, block): left vector (q_bar or P) rows r0 .., right vector (dL/dv or dL/du)
  auto left = [&](int n) -> const float* {
    const int s = n / p.nblk, b = n - s * p.nblk;
    const size_t row = (static_cast<size_t>(s) * (is_q ? p.hq : p.hkv) + head) * p.nblk + b;
    return is_q ? p.ws_qbar + row * kDim : p.ws_p + row * kPool;
  };
  auto right = [&](int n) -> const float* {
    const int s = n / p.nblk, b = n - s * p.nblk;
    const size_t row = (static_cast<size_t>(s) * (is_q ? p.hq : p.hkv) + head) * p.nblk + b;
    return (is_q ? p.ws_dv : p.ws_du) + row * kDim;
  };
  // the first row block of each head also sums that head's gain terms
  const bool gains = (r0 == 0);
  const float* gterm = is_q ? p.ws_dgq : p.ws_dgk;
  float ga = 0.f;
  for (int n0 = 0; n0 < N; n0 += 32) {
    const int nn = min(32, N - n0);
    __syncthreads();
    // 16-byte loads, all of a thread's in flight at once
#pragma unroll 4
    for (int x = tid; x < nn * (kDim / 4); x += 256)
      reinterpret_cast<float4*>(&sx[x / (kDim / 4)][0])[x % (kDim / 4)] =
          reinterpret_cast<const float4*>(right(n0 + x / (kDim / 4)))[x % (kDim / 4)];
    if (tid < nn * (kPbRed / 4))
      reinterpret_cast<float4*>(&sv[tid / (kPbRed / 4)][0])[tid % (kPbRed / 4)] =
          reinterpret_cast<const float4*>(left(n0 + tid / (kPbRed / 4)) + r0)[tid % (kPbRed / 4)];
    if (gains) {
#pragma unroll 4
      for (int x = tid; x < nn * (kDim / 4); x += 256) {
        const int n = n0 + x / (kDim / 4), s = n / p.nblk, b = n - s * p.nblk;
        reinterpret_cast<float4*>(&sg[x / (kDim / 4)][0])[x % (kDim / 4)] = reinterpret_cast<const float4*>(
            gterm + ((static_cast<size_t>(s) * (is_q ? p.hq : p.hkv) + head) * p.nblk + b) * kDim)[x % (kDim / 4)];
      }
    }
    __syncthreads();
    for (int n = 0; n < nn; ++n) {
      const float d = sx[n][j];
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] = fmaf(sv[n][rp + 2 * k], d, acc[k]);
    }
    if (gains && rp == 0)
      for (int n = 0; n < nn; ++n) ga += sg[n][j];
  }
  float* dw = is_q ? p.dw_q + static_cast<size_t>(head) * kDim * kDim : p.dw_k + static_cast<size_t>(head) * kPool * kDim;
#pragma unroll
  for (int k = 0; k < kPer; ++k) dw[static_cast<size_t>(r0 + rp + 2 * k) * kDim + j] += acc[k];
  if (gains && rp == 0) p.ws_gpart[static_cast<size_t>(is_q ? head : p.hq + head) * kDim + j] = ga;
}

__global__ void __launch_bounds__(256) prefill_gamma_final_kernel(const __grid_constant__ PrefillBwdParams p) {
  const int j = threadIdx.x & (kDim - 1), which = threadIdx.x >> 7;  // 0: gamma_q, 1: gamma_k
  const int h0 = which ? p.hq : 0, nh = which ? p.hkv : p.hq;
  float a = 0.f;
  for (int h = 0; h < nh; ++h) a += p.ws_gpart[static_cast<size_t>(h0 + h) * kDim + j];
  (which ? p.dgamma_k : p.dgamma_q)[j] += a;
}

cudaError_t launch_prefill_gate_backward(const PrefillBwdParams& p, const CUtensorMap& tmq, const CUtensorMap& tmk,
                                         const CUtensorMap& tmv, cudaStream_t stream) {
  const int smem = prefill_bwd_smem_bytes(p.max_sel, p.stages);
  prefill_bwd_attn_kernel<<<dim3(p.nblk, p.hq, p.batch), kPbThreads, smem, stream>>>(p, tmq, tmk, tmv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t ksmem = static_cast<size_t>(p.nblk) * (kPbChunk / 32 + 1) * 4;
  prefill_bwd_keys_kernel<<<dim3((p.nblk + kPbChunk - 1) / kPbChunk, p.hkv, p.batch), 256, ksmem, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const unsigned nred = static_cast<unsigned>(p.hq * (kDim / kPbRed) + p.hkv * (kPool / kPbRed));
  prefill_grad_reduce_kernel<<<nred, 256, 0, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prefill_gamma_final_kernel<<<1, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t prepare_prefill_backward_kernels() {
  cudaError_t e = cudaFuncSetAttribute(prefill_bwd_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_bwd_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

}  // namespace sas
