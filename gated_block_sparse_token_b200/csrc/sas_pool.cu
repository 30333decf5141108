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

cudaError_t prepare_pool_project_kernel();

cudaError_t prepare_pool_kernels() {
  const cudaError_t e0 = prepare_pool_project_kernel();
  if (e0 != cudaSuccess) return e0;
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

// ---------------------------------------------------------------- tensor-core pooling and projection
// The same pooled keys and gate keys for bf16 caches, with the projection on
// the 5th-generation tensor cores.  One CTA (256 threads) per 128 blocks of
// one (sequence, KV head):
//   1. W_k[h] (96 KiB bf16) comes in by TMA, 128-byte swizzled, as the
//      MN-major B operand [384 x 128]; tensor memory: 128 fp32 columns.
//   2. the 8 warps pool the tile's blocks straight from global memory
//      (16-byte loads, 16 per lane in flight) and write row i of the A
//      operand [128 x 512] bf16, K-major and 128-byte swizzled:
//      [max | min | mean_hi | mean_lo], where mean_hi = bf16(mean) and
//      mean_lo = bf16(mean - mean_hi).  max and min are elements of K (exact
//      in bf16) and hi + lo carries the fp32 mean to within 2^-17 of it, so
//      the bf16 x bf16 products the tensor core accumulates in fp32 give
//      u = P @ W_k to fp32 accuracy (the mean's W_k rows serve both hi and lo).
//   3. one thread issues the 32 MMAs (M = 128 blocks, N = 128, K = 16 each).
//   4. the epilogue reads u from tensor memory (a thread per block, two
//      warps per lane quarter, each half the rotate-half pairs), applies
//      RMSNorm, gamma_k and the gate RoPE at the block index, and stores the
//      gate keys.
constexpr int kPpRows = 128;          // blocks per CTA (the MMA's M)
constexpr int kPpThreads = 256;
constexpr int kPpA = kPpRows * 512 * 2;           // A operand bytes (8 chunks of 16 KiB)
constexpr int kPpB = kPool * kDim * 2;            // B operand bytes (2 N-halves of 48 KiB)
constexpr int kPpSmem = kPpA + kPpB + 2 * kPpRows * 4 + 64 + 1024;

__global__ void __launch_bounds__(kPpThreads, 1) pool_project_kernel(const __grid_constant__ PoolParams p,
                                                                     const __grid_constant__ CUtensorMap tmwk) {
  const int s = blockIdx.z;
  const int h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + kPpA;
  float* ssq = reinterpret_cast<float*>(sB + kPpB);  // [2][128] partial sums of squares
  uint64_t* bars = reinterpret_cast<uint64_t*>(ssq + 2 * kPpRows);  // W_k, MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  const int L = (p.kv.seq_lens != nullptr) ? p.kv.seq_lens[s] : p.kv.capacity;  // prefill: full length
  const int first = p.blk_begin != nullptr ? p.blk_begin[s] : 0;
  const int b0 = first + static_cast<int>(blockIdx.x) * kPpRows;
  const int b_end = first + p.num_blocks;
  auto row_of = [&](int i) -> long long {  // cache row of tile row i; -1: not pooled; -2: out of range
    const int b = b0 + i;
    if (b < 0 || b >= b_end || b >= p.mg || L < 1 || static_cast<long long>(b + 1) * kBlock > L) return -1;
    const long long r = p.kv.block_row(s, h, b);
    return r < 0 ? -2 : r;
  };
  // rows that may hold work: blocks max(b0, 0) .. min(b0 + 128, b_end, mg, L / 64) - 1
  {
    const int lo = max(b0, 0);
    const int hi = min(min(b0 + kPpRows, b_end), min(p.mg, L >= 1 ? L / kBlock : 0));
    if (lo >= hi) return;  // uniform over the CTA
  }

  if (tid == 0) {
    prefetch_tensormap(&tmwk);
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bars[0], kPpB);
    for (int c = 0; c < 2; ++c)
      for (int r = 0; r < kPool / 64; ++r)
        tma_load_2d(sB + c * (kPool * 128) + r * 8192, &tmwk, 64 * c, h * kPool + 64 * r, &bars[0]);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }

  // ---- pooling into the A operand
  {
    constexpr int TPR = 16;             // lanes per K row (16-byte loads)
    const int cvec = lane % TPR, par = lane / TPR;
    const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.kv.k);
    bool err = false;
    for (int i = warp; i < kPpRows; i += kPpThreads / 32) {  // warp-uniform
      const long long row = row_of(i);
      if (row == -2) err = true;
      float mx[8], mn[8], sm[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        mx[v] = -INFINITY;
        mn[v] = INFINITY;
        sm[v] = 0.f;
      }
      if (row >= 0) {
        const __nv_bfloat16* blk = kbase + (row + par) * kDim + cvec * 8;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint4 raw[16];
#pragma unroll
          for (int r = 0; r < 16; ++r)
            raw[r] = *reinterpret_cast<const uint4*>(blk + static_cast<size_t>(2 * (16 * part + r)) * kDim);
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const uint32_t w4[4] = {raw[r].x, raw[r].y, raw[r].z, raw[r].w};
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float x0 = bf16_lo(w4[v]), x1 = bf16_hi(w4[v]);
              mx[2 * v] = fmaxf(mx[2 * v], x0);
              mn[2 * v] = fminf(mn[2 * v], x0);
              sm[2 * v] += x0;
              mx[2 * v + 1] = fmaxf(mx[2 * v + 1], x1);
              mn[2 * v + 1] = fminf(mn[2 * v + 1], x1);
              sm[2 * v + 1] += x1;
            }
          }
        }
      }
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        mx[v] = fmaxf(mx[v], __shfl_xor_sync(0xffffffffu, mx[v], 16));
        mn[v] = fminf(mn[v], __shfl_xor_sync(0xffffffffu, mn[v], 16));
        sm[v] += __shfl_xor_sync(0xffffffffu, sm[v], 16);
      }
      if (par == 0) {
        uint32_t pk[4][4];  // [max, min, hi, lo][4 bf16 pairs]
        float mean[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) mean[v] = (row >= 0) ? sm[v] * (1.f / kBlock) : 0.f;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float a0 = row >= 0 ? mx[2 * v] : 0.f, a1 = row >= 0 ? mx[2 * v + 1] : 0.f;
          const float n0 = row >= 0 ? mn[2 * v] : 0.f, n1 = row >= 0 ? mn[2 * v + 1] : 0.f;
          const __nv_bfloat16 h0 = __float2bfloat16_rn(mean[2 * v]), h1 = __float2bfloat16_rn(mean[2 * v + 1]);
          pk[0][v] = pack_bf16x2(a0, a1);
          pk[1][v] = pack_bf16x2(n0, n1);
          pk[2][v] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
          pk[3][v] = pack_bf16x2(mean[2 * v] - __bfloat162float(h0), mean[2 * v + 1] - __bfloat162float(h1));
        }
        // K index sec * 128 + 8 cvec: chunk 2 sec + cvec / 8, 16-byte unit cvec % 8
#pragma unroll
        for (int sec = 0; sec < 4; ++sec) {
          const int kc = 2 * sec + (cvec >> 3);
          const int j = cvec & 7;
          *reinterpret_cast<uint4*>(sA + kc * (kPpRows * 128) + i * 128 + ((j ^ (i & 7)) << 4)) =
              make_uint4(pk[sec][0], pk[sec][1], pk[sec][2], pk[sec][3]);
        }
        if (p.pooled_raw != nullptr && row >= 0) {
          float* pr = p.pooled_raw + ((static_cast<size_t>(s) * p.hkv + h) * p.mg + (b0 + i)) * kPool + cvec * 8;
#pragma unroll
          for (int v = 0; v < 8; ++v) {  // 4-byte aligned: scalar stores
            pr[v] = mx[v];
            pr[kDim + v] = mn[v];
            pr[2 * kDim + v] = mean[v];
          }
        }
      }
    }
    if (err && lane == 0) raise_status(p.status, kStatusBounds);
  }
  fence_proxy_async_smem();  // the A rows written here are read by the tensor core (async proxy)
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // ---- u = A @ B on the tensor cores
  if (tid == 0) {
    const bool okb = mbar_wait(&bars[0], 0, p.status);
    tc_fence_after_sync();
    if (okb) {
      const uint64_t dA = umma_desc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t dB = umma_desc_sw128(smem_u32(sB), kPool * 128, 1024);
      constexpr uint32_t idesc = umma_idesc_bf16(kPpRows, kDim, false, true);
#pragma unroll
      for (int kk = 0; kk < 32; ++kk) {
        const uint32_t a_off = (kk >> 2) * (kPpRows * 128) + (kk & 3) * 32;
        const uint32_t brow = (kk < 24) ? 16 * kk : 16 * (kk - 8);  // the mean rows serve hi and lo
        umma_bf16_ss(tmem, dA + (a_off >> 4), dB + ((brow * 128) >> 4), idesc, kk > 0);
      }
    }
    umma_commit(&bars[1]);  // also when nothing was issued: the barrier still completes
  }
  const bool okm = mbar_wait(&bars[1], 0, p.status);
  tc_fence_after_sync();

  // ---- epilogue: RMSNorm, gain, RoPE at the block index, store
  {
    const int q4 = warp & 3, hf = warp >> 2;  // lane quarter; half of the rotate-half pairs
    const int i = 32 * q4 + lane;             // tile row = block b0 + i
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    float lo[32], hi[32];
    tmem_ld32(tl + 32 * hf, lo);       // columns 32 hf .. 32 hf + 31
    tmem_ld32(tl + 64 + 32 * hf, hi);  // their rotate-half partners
    tmem_wait_ld();
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) ss = fmaf(lo[k], lo[k], fmaf(hi[k], hi[k], ss));
    ssq[hf * kPpRows + i] = ss;
    __syncthreads();
    const long long row = row_of(i);
    if (row >= 0 && okm) {
      const int b = b0 + i;
      const float inv = 1.f / sqrtf((ssq[i] + ssq[kPpRows + i]) / kDim + p.eps);
      const size_t gi = ((static_cast<size_t>(s) * p.hkv + h) * p.mg + b) * kDim;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int d = 32 * hf + k;
        const float x0 = lo[k] * inv * p.gamma_k[d];
        const float x1 = hi[k] * inv * p.gamma_k[d + 64];
        float cs, sn;
        rope_cos_sin(p.rope.theta_over_pi[d], b, cs, sn);
        lo[k] = x0 * cs - x1 * sn;
        hi[k] = x1 * cs + x0 * sn;
      }
      if (p.gk16) {
        __nv_bfloat16* g = static_cast<__nv_bfloat16*>(p.gate_keys) + gi;
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
          *reinterpret_cast<uint4*>(g + 32 * hf + k) =
              make_uint4(pack_bf16x2(lo[k], lo[k + 1]), pack_bf16x2(lo[k + 2], lo[k + 3]),
                         pack_bf16x2(lo[k + 4], lo[k + 5]), pack_bf16x2(lo[k + 6], lo[k + 7]));
          *reinterpret_cast<uint4*>(g + 64 + 32 * hf + k) =
              make_uint4(pack_bf16x2(hi[k], hi[k + 1]), pack_bf16x2(hi[k + 2], hi[k + 3]),
                         pack_bf16x2(hi[k + 4], hi[k + 5]), pack_bf16x2(hi[k + 6], hi[k + 7]));
        }
      } else {
        float* g = static_cast<float*>(p.gate_keys) + gi;
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          *reinterpret_cast<float4*>(g + 32 * hf + k) = make_float4(lo[k], lo[k + 1], lo[k + 2], lo[k + 3]);
          *reinterpret_cast<float4*>(g + 64 + 32 * hf + k) = make_float4(hi[k], hi[k + 1], hi[k + 2], hi[k + 3]);
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

cudaError_t launch_pool_project(const PoolParams& p, const CUtensorMap& tmwk, int batch, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((p.num_blocks + kPpRows - 1) / kPpRows), static_cast<unsigned>(p.hkv),
                  static_cast<unsigned>(batch));
  pool_project_kernel<<<grid, kPpThreads, kPpSmem, stream>>>(p, tmwk);
  return cudaGetLastError();
}

cudaError_t prepare_pool_project_kernel() {
  return cudaFuncSetAttribute(pool_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPpSmem);
}

}  // namespace sas
