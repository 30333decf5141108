// SAS key-block pooling and gate keys.
//
// Method (release pages: keys pooled per block by max, min and average, Q/K
// normalisation and gate RoPE on, gate hidden size 128): for a
// complete 64-token block b of (sequence s, KV head h)
//   P_b  = [max_j K_j ; min_j K_j ; mean_j K_j]          (384 = 3 x 128)
//   k~_b = RoPE(RMSNorm(P_b @ W_k[h]) * gamma_k, position b)
//
// One CTA handles up to kPoolBlocksPerCta consecutive blocks of one (s, h).
// W_k[h] (96 KiB bf16) comes into shared memory with one TMA bulk copy that
// overlaps the pooling; each warp pools whole blocks (16-byte loads, 16 rows
// in flight per lane, reduced in registers and across the lanes that share
// a column chunk).  The 384x128 projection of all the CTA's blocks then runs
// out of shared memory at once, thread d owning output dimension d.
#include <cmath>

#include "sas_internal.h"

namespace sas {

template <typename T>
__global__ void __launch_bounds__(kThreads) pool_keys_kernel(const __grid_constant__ PoolParams p) {
  constexpr int NB = kPoolBlocksPerCta;
  constexpr int VEC = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte load
  constexpr int TPR = kDim / VEC;                       // lanes per K row
  const int s = blockIdx.z;
  const int h = blockIdx.y;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __nv_bfloat16* wk_s = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + kPoolWkBytes);
  // pooled blocks, [pooled dim][block]; reused for the normalised u, [block][dim]
  __shared__ __align__(16) float Pt[kPool][NB];
  float (*xs)[kDim] = reinterpret_cast<float (*)[kDim]>(&Pt[0][0]);
  __shared__ float ssq[kWarps][NB];

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
    mbar_arrive_expect_tx(bar, kPoolWkBytes);
    bulk_g2s(wk_s, p.w_k + static_cast<size_t>(h) * kPool * kDim, kPoolWkBytes, bar);
  }

  // ---- pooling: max, min, mean over the 64 tokens, per dimension.  Warp w
  // pools blocks w, w + 4, ...: lane l reads the 16-byte chunk l % TPR of
  // rows l / TPR, l / TPR + RPW, ... (16 rows' loads in flight per lane)
  {
    constexpr int RPW = 32 / TPR;          // rows per warp step (2 bf16, 1 fp32)
    constexpr int ROWS = kBlock / RPW;     // rows per lane
    const T* kbase = static_cast<const T*>(p.kv.k);
    const int cvec = lane % TPR, par = lane / TPR;
    for (int i = warp; i < NB; i += kWarps) {  // warp-uniform
      float mx[VEC], mn[VEC], sm[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) {
        mx[v] = -INFINITY;
        mn[v] = INFINITY;
        sm[v] = 0.f;
      }
      if (rows[i] >= 0) {
        const T* blk = kbase + (rows[i] + par) * kDim + cvec * VEC;
#pragma unroll
        for (int part = 0; part < ROWS / 16; ++part) {
          uint4 raw[16];
#pragma unroll
          for (int r = 0; r < 16; ++r)
            raw[r] = *reinterpret_cast<const uint4*>(blk + static_cast<size_t>(RPW * (16 * part + r)) * kDim);
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const T* e = reinterpret_cast<const T*>(&raw[r]);
#pragma unroll
            for (int v = 0; v < VEC; ++v) {
              const float x = to_float(e[v]);
              mx[v] = fmaxf(mx[v], x);
              mn[v] = fminf(mn[v], x);
              sm[v] += x;
            }
          }
        }
      }
#pragma unroll
      for (int o = TPR; o < 32; o <<= 1) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          mx[v] = fmaxf(mx[v], __shfl_xor_sync(0xffffffffu, mx[v], o));
          mn[v] = fminf(mn[v], __shfl_xor_sync(0xffffffffu, mn[v], o));
          sm[v] += __shfl_xor_sync(0xffffffffu, sm[v], o);
        }
      }
      if (par == 0) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          const int dd = cvec * VEC + v;
          const float mean = sm[v] * (1.f / kBlock);
          Pt[dd][i] = rows[i] >= 0 ? mx[v] : 0.f;
          Pt[kDim + dd][i] = rows[i] >= 0 ? mn[v] : 0.f;
          Pt[2 * kDim + dd][i] = mean;
          if (p.pooled_raw != nullptr && rows[i] >= 0) {
            float* pr = p.pooled_raw + ((static_cast<size_t>(s) * p.hkv + h) * p.mg + (b0 + i)) * kPool;
            pr[dd] = mx[v];
            pr[kDim + dd] = mn[v];
            pr[2 * kDim + dd] = mean;
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- u = P @ W_k[h] from shared memory, thread d owning output dimension d
  const bool ok = mbar_wait(bar, 0, p.status);
  const int d = tid;
  float u[NB];
#pragma unroll
  for (int i = 0; i < NB; ++i) u[i] = 0.f;
  if (ok) {
#pragma unroll 4
    for (int r = 0; r < kPool; ++r) {
      const float w = __bfloat162float(wk_s[r * kDim + d]);
      const float4* p4 = reinterpret_cast<const float4*>(&Pt[r][0]);
#pragma unroll
      for (int c = 0; c < NB / 4; ++c) {
        const float4 x = p4[c];
        u[4 * c] = fmaf(x.x, w, u[4 * c]);
        u[4 * c + 1] = fmaf(x.y, w, u[4 * c + 1]);
        u[4 * c + 2] = fmaf(x.z, w, u[4 * c + 2]);
        u[4 * c + 3] = fmaf(x.w, w, u[4 * c + 3]);
      }
    }
  }

  // ---- RMSNorm (gain gamma_k) and gate RoPE at the block index, per block
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    float sq = u[i] * u[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) ssq[warp][i] = sq;
  }
  __syncthreads();  // every Pt read is done: xs may overwrite it
  const float gk = p.gamma_k[d];
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const float tot = ssq[0][i] + ssq[1][i] + ssq[2][i] + ssq[3][i];
    xs[i][d] = u[i] * (1.f / sqrtf(tot / kDim + p.eps)) * gk;
  }
  __syncthreads();
  const int j = d & 63;
  for (int i = 0; i < nb; ++i) {
    if (rows[i] < 0) continue;
    const int b = b0 + i;
    float cs, sn;
    rope_cos_sin(p.rope.theta_over_pi[j], b, cs, sn);
    const float y = (d < 64) ? xs[i][d] * cs - xs[i][d + 64] * sn : xs[i][d] * cs + xs[i][d - 64] * sn;
    const size_t gi = ((static_cast<size_t>(s) * p.hkv + h) * p.mg + b) * kDim + d;
    if (p.gk16)
      static_cast<__nv_bfloat16*>(p.gate_keys)[gi] = __float2bfloat16_rn(y);
    else
      static_cast<float*>(p.gate_keys)[gi] = y;
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
