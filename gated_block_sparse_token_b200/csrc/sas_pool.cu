// SAS key-block pooling and gate keys.
//
// Method (release pages, "key block pooling max + min + average", "Q/K
// normalization enabled", "gate RoPE enabled", gate hidden size 128): for a
// complete 64-token block b of (sequence s, KV head h)
//   P_b  = [max_j K_j ; min_j K_j ; mean_j K_j]          (384 = 3 x 128)
//   k~_b = RoPE(RMSNorm(P_b @ W_k[h]) * gamma_k, position b)
//
// One CTA handles up to kPoolBlocksPerCta consecutive blocks of one (s, h).
// W_k[h] (96 KiB bf16) comes into shared memory with one TMA bulk copy that
// overlaps the pooling; the block's K rows are read with 16-byte loads (all
// rows of a block in flight at once), reduced per row group in registers and
// across row groups in shared memory.  The 384x128 projection then runs out
// of shared memory, thread d owning output dimension d.
#include <cmath>

#include "sas_internal.h"

namespace sas {

template <typename T>
__global__ void __launch_bounds__(kThreads) pool_keys_kernel(const __grid_constant__ PoolParams p) {
  constexpr int NB = kPoolBlocksPerCta;
  constexpr int VEC = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte load
  constexpr int TPR = kDim / VEC;                       // threads per K row
  constexpr int RG = kThreads / TPR;                    // row groups
  constexpr int RPT = kBlock / RG;                      // rows per thread
  const int s = blockIdx.z;
  const int h = blockIdx.y;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* wk_s = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + kPoolWkBytes);
  __shared__ float P[NB][kPool];
  __shared__ float red[RG][3][kDim];
  __shared__ float xn[kDim];
  __shared__ float ssq[kWarps];

  const int L = (p.kv.seq_lens != nullptr) ? p.kv.seq_lens[s] : p.kv.capacity;  // prefill: full length
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
      if (rows[i] < 0)
        err = true;
      else
        nb = i + 1;
    }
  }
  if (err && tid == 0) raise_status(p.status, kStatusBounds);
  if (nb == 0) return;  // uniform over the CTA

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, kPoolWkBytes);
    bulk_g2s(wk_s, p.w_k + static_cast<size_t>(h) * kPool * kDim, kPoolWkBytes, bar);
  }

  // ---- pooling: max, min, mean over the 64 tokens, per dimension
  const T* kbase = static_cast<const T*>(p.kv.k);
  const int cvec = tid % TPR;  // dims cvec*VEC .. +VEC
  const int rg = tid / TPR;    // rows rg, rg+RG, ...
  for (int i = 0; i < nb; ++i) {
    if (rows[i] < 0) continue;  // uniform
    const T* blk = kbase + rows[i] * kDim + cvec * VEC;
    uint4 raw[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r)
      raw[r] = *reinterpret_cast<const uint4*>(blk + static_cast<size_t>(rg + r * RG) * kDim);
    float mx[VEC], mn[VEC], sm[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      mx[v] = -INFINITY;
      mn[v] = INFINITY;
      sm[v] = 0.f;
    }
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const T* e = reinterpret_cast<const T*>(&raw[r]);
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        const float x = to_float(e[v]);
        mx[v] = fmaxf(mx[v], x);
        mn[v] = fminf(mn[v], x);
        sm[v] += x;
      }
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      red[rg][0][cvec * VEC + v] = mx[v];
      red[rg][1][cvec * VEC + v] = mn[v];
      red[rg][2][cvec * VEC + v] = sm[v];
    }
    __syncthreads();
    {
      const int d = tid;
      float a = red[0][0][d], b = red[0][1][d], c = red[0][2][d];
#pragma unroll
      for (int g = 1; g < RG; ++g) {
        a = fmaxf(a, red[g][0][d]);
        b = fminf(b, red[g][1][d]);
        c += red[g][2][d];
      }
      c *= (1.f / kBlock);
      P[i][d] = a;
      P[i][kDim + d] = b;
      P[i][2 * kDim + d] = c;
      if (p.pooled_raw != nullptr) {
        float* pr = p.pooled_raw + ((static_cast<size_t>(s) * p.hkv + h) * p.mg + (b0 + i)) * kPool;
        pr[d] = a;
        pr[kDim + d] = b;
        pr[2 * kDim + d] = c;
      }
    }
    __syncthreads();
  }

  // ---- u = P @ W_k[h] from shared memory
  const bool ok = mbar_wait(bar, 0, p.status);
  const int d = tid;
  float u[NB];
#pragma unroll
  for (int i = 0; i < NB; ++i) u[i] = 0.f;
  if (ok) {
#pragma unroll 4
    for (int r = 0; r < kPool; ++r) {
      const float w = __bfloat162float(wk_s[r * kDim + d]);
#pragma unroll
      for (int i = 0; i < NB; ++i)
        if (i < nb) u[i] = fmaf(P[i][r], w, u[i]);
    }
  }

  // ---- RMSNorm (gain gamma_k) and gate RoPE at the block index, per block
  const float gk = p.gamma_k[d];
  const int j = d & 63;
  for (int i = 0; i < nb; ++i) {
    float sq = u[0] * u[0];
#pragma unroll
    for (int k = 1; k < NB; ++k)
      if (k == i) sq = u[k] * u[k];
    float ui = u[0];
#pragma unroll
    for (int k = 1; k < NB; ++k)
      if (k == i) ui = u[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) ssq[warp] = sq;
    __syncthreads();
    const float tot = ssq[0] + ssq[1] + ssq[2] + ssq[3];
    xn[d] = ui * (1.f / sqrtf(tot / kDim + p.eps)) * gk;
    __syncthreads();
    if (rows[i] >= 0) {
      const int b = b0 + i;
      float cs, sn;
      rope_cos_sin(p.rope.theta_over_pi[j], b, cs, sn);
      const float y = (d < 64) ? xn[d] * cs - xn[d + 64] * sn : xn[d] * cs + xn[d - 64] * sn;
      const size_t gi = ((static_cast<size_t>(s) * p.hkv + h) * p.mg + b) * kDim + d;
      if (p.gk16)
        static_cast<__nv_bfloat16*>(p.gate_keys)[gi] = __float2bfloat16_rn(y);
      else
        static_cast<float*>(p.gate_keys)[gi] = y;
    }
    __syncthreads();
  }
}

cudaError_t launch_pool(bool f32_kv, const PoolParams& p, int batch, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((p.num_blocks + kPoolBlocksPerCta - 1) / kPoolBlocksPerCta),
                  static_cast<unsigned>(p.hkv), static_cast<unsigned>(batch));
  const size_t smem = pool_smem_bytes();
  if (f32_kv)
    pool_keys_kernel<float><<<grid, kThreads, smem, stream>>>(p);
  else
    pool_keys_kernel<__nv_bfloat16><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

size_t pool_smem_bytes() { return static_cast<size_t>(kPoolWkBytes) + 16; }

cudaError_t prepare_pool_kernels() {
  cudaError_t e = cudaFuncSetAttribute(pool_keys_kernel<float>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(pool_smem_bytes()));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(pool_keys_kernel<__nv_bfloat16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(pool_smem_bytes()));
}

void fill_rope_table(RopeTable& t, float base) {
  for (int i = 0; i < 64; ++i)
    t.theta_over_pi[i] = std::pow(static_cast<double>(base), -2.0 * i / kDim) / M_PI;
}

}  // namespace sas
