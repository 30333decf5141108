// SAS key-block pooling and gate keys.
//
// Method (release pages, "key block pooling max + min + average", "Q/K
// normalization enabled", "gate RoPE enabled", gate hidden size 128): for a
// complete 64-token block b of (sequence s, KV head h)
//   P_b  = [max_j K_j ; min_j K_j ; mean_j K_j]          (384 = 3 x 128)
//   k~_b = RoPE(RMSNorm(P_b @ W_k[h]) * gamma_k, position b)
// One CTA handles up to kPoolBlocksPerCta consecutive blocks of one (s, h)
// so that every W_k row it reads from L2 serves all of them; thread d owns
// dimension d (coalesced 128-wide rows of K and of W_k).
#include "sas_internal.h"

namespace sas {

template <typename T>
__global__ void __launch_bounds__(kThreads) pool_keys_kernel(const __grid_constant__ PoolParams p) {
  constexpr int NB = kPoolBlocksPerCta;
  const int s = blockIdx.z;
  const int h = blockIdx.y;
  const int d = threadIdx.x;
  const int warp = d >> 5, lane = d & 31;
  __shared__ float P[NB][kPool];
  __shared__ float xn[NB][kDim];
  __shared__ float red[kWarps][NB];

  const int L = p.kv.seq_lens[s];
  const int first = p.blk_begin != nullptr ? p.blk_begin[s] : 0;
  const int b0 = first + static_cast<int>(blockIdx.x) * NB;
  const int b_end = first + p.num_blocks;

  long long rows[NB];
  int nb = 0;
  bool err = false;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int b = b0 + i;
    rows[i] = -1;
    // only complete blocks that have a gate-key row are pooled
    if (b >= 0 && b < b_end && b < p.mg && L >= 1 &&
        static_cast<long long>(b + 1) * kBlock <= static_cast<long long>(L)) {
      rows[i] = p.kv.block_row(s, h, b);
      if (rows[i] < 0) err = true;
      else nb = i + 1;
    }
  }
  if (err && d == 0) raise_status(p.status, kStatusBounds);
  if (nb == 0) return;  // uniform over the CTA

  const T* kbase = static_cast<const T*>(p.kv.k);
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    if (i < nb && rows[i] >= 0) {
      const T* col = kbase + rows[i] * kDim + d;
      float mx = -INFINITY, mn = INFINITY, sum = 0.f;
#pragma unroll 16
      for (int t = 0; t < kBlock; ++t) {
        const float x = to_float(col[static_cast<size_t>(t) * kDim]);
        mx = fmaxf(mx, x);
        mn = fminf(mn, x);
        sum += x;
      }
      P[i][d] = mx;
      P[i][kDim + d] = mn;
      P[i][2 * kDim + d] = sum * (1.f / kBlock);
      if (p.pooled_raw != nullptr) {
        float* pr = p.pooled_raw + ((static_cast<size_t>(s) * p.hkv + h) * p.mg + (b0 + i)) * kPool;
        pr[d] = mx;
        pr[kDim + d] = mn;
        pr[2 * kDim + d] = sum * (1.f / kBlock);
      }
    }
  }
  __syncthreads();

  // u = P @ W_k[h]
  float u[NB];
#pragma unroll
  for (int i = 0; i < NB; ++i) u[i] = 0.f;
  const __nv_bfloat16* wk = p.w_k + static_cast<size_t>(h) * kPool * kDim + d;
#pragma unroll 8
  for (int r = 0; r < kPool; ++r) {
    const float w = __bfloat162float(wk[static_cast<size_t>(r) * kDim]);
#pragma unroll
    for (int i = 0; i < NB; ++i) u[i] = fmaf(P[i][r], w, u[i]);
  }

  // RMSNorm per block
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    float sq = u[i] * u[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) red[warp][i] = sq;
  }
  __syncthreads();
  const float g = p.gamma_k[d];
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const float ss = red[0][i] + red[1][i] + red[2][i] + red[3][i];
    xn[i][d] = u[i] * (1.f / sqrtf(ss / kDim + p.eps)) * g;
  }
  __syncthreads();

  // gate RoPE at the block index, rotate-half pairs (j, j + 64)
  const int j = d & 63;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    if (i < nb && rows[i] >= 0) {
      const int b = b0 + i;
      float cs, sn;
      rope_cos_sin(j, b, p.rope_base, cs, sn);
      const float y = (d < 64) ? xn[i][d] * cs - xn[i][d + 64] * sn : xn[i][d] * cs + xn[i][d - 64] * sn;
      p.gate_keys[((static_cast<size_t>(s) * p.hkv + h) * p.mg + b) * kDim + d] = y;
    }
  }
}

cudaError_t launch_pool(bool f32_kv, const PoolParams& p, int batch, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((p.num_blocks + kPoolBlocksPerCta - 1) / kPoolBlocksPerCta),
                  static_cast<unsigned>(p.hkv), static_cast<unsigned>(batch));
  if (f32_kv)
    pool_keys_kernel<float><<<grid, kThreads, 0, stream>>>(p);
  else
    pool_keys_kernel<__nv_bfloat16><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

size_t pool_smem_bytes() { return 0; }

}  // namespace sas
