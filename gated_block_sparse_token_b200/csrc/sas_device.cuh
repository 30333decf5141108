// Device-side helpers shared by the libsas kernels (sm_100a only).
//
// Hand-written inline PTX for: mbarrier transaction barriers, TMA bulk and
// tensor copies global -> shared, ldmatrix, bf16 mma.sync, the global timer
// used to bound every wait, and the RoPE / order-preserving key helpers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sas {

constexpr int kBlock = 64;         // KV block size (tokens)
constexpr int kDim = 128;          // head_dim == gate hidden size
constexpr int kPool = 3 * kDim;    // pooled key width: max, min, mean
constexpr int kThreads = 128;      // threads per CTA of every kernel here
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroup = 8;       // largest GQA group (Hq / Hkv) handled
constexpr int kTileBytes = 16384;  // one stage slot: a 64x128 bf16 tile
constexpr int kGkChunk = kTileBytes / (kDim * 4);  // gate keys per slot (32)
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

// Bits of the device status word (first 4 bytes of the workspace).
constexpr uint32_t kStatusBounds = 1u;
constexpr uint32_t kStatusTimeout = 2u;

__device__ __forceinline__ void raise_status(uint32_t* status, uint32_t bit) {
  if (status != nullptr) atomicOr(status, bit);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Cluster-scope variants: a CTA arrives on another CTA's barrier (release at
// cluster scope), the owner waits with acquire at cluster scope.
__device__ __forceinline__ void mbar_remote_arrive(uint64_t* local_bar, uint32_t rank) {
  uint32_t raddr;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local_bar)), "r"(rank));
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(raddr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      raise_status(status, kStatusTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void fence_acq_rel_cluster() {
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
}

// Wait for phase `parity` of `bar` to complete, for at most kWaitLimitNs.
// Returns false (and raises the timeout bit) if the limit is reached.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      raise_status(status, kStatusTimeout);
      return false;
    }
  }
}

// ---------------------------------------------------------------- cluster barrier
// Split arrive / wait of the hardware cluster barrier (all threads of every
// CTA of the cluster).  Arriving at kernel start and waiting before the first
// distributed-shared-memory access guarantees every CTA of the cluster is
// running when its shared memory is touched.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- TMA copies
// Contiguous bytes global -> this CTA's shared memory; completes `bytes` of
// transaction count on `bar`.  dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Ask L2 to fetch `bytes` contiguous bytes from global memory (no shared
// memory involved, nothing to wait for).  src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Prefetch the 128-byte line holding `p` into L2 (load/store unit path, so it
// does not queue behind the TMA copies of the same SM).
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 2-D tiled tensor copy (box given by the tensor map) at element coordinates
// (x = innermost, y = row) into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- ldmatrix / mma
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8, f32) = A(16x16 bf16, row) * B(16x8 bf16, col) + C, keeping only the
// rows 0..7 of the result (rows 8..15 enter as zero and are dropped): the
// callers pad a GQA group of <= 8 heads to the 16 rows of the instruction.
// (a0, a2) are the A fragment registers of rows 0..7; d0, d1 accumulate.
__device__ __forceinline__ void mma_rows0_7(float& d0, float& d1, uint32_t a0, uint32_t a2,
                                            uint32_t b0, uint32_t b1) {
  float x2, x3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%10,%10};"
      : "+f"(d0), "+f"(d1), "=f"(x2), "=f"(x3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(0.f));
  (void)x2;
  (void)x3;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of (row, 16-byte chunk j in 0..15) of a 64-row x 128-col bf16
// tile stored as two 64x64 boxes written by TMA with 128-byte swizzling.
__device__ __forceinline__ uint32_t swz_tile_offset(int row, int j) {
  return static_cast<uint32_t>((j >> 3) * 8192 + row * 128 + (((j & 7) ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename OutT>
__device__ __forceinline__ OutT from_float(float x);
template <>
__device__ __forceinline__ float from_float<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Monotone map float -> uint32 (larger float, larger key).  -0 maps like +0;
// NaN maps below every number.
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x != x) return 0u;
  if (x == 0.f) x = 0.f;
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Gate RoPE factors at integer position pos for a pair whose frequency is
// theta = base^(-2i/128), given as theta_over_pi = theta / pi (double, from the
// host).  The angle is pos * theta; with a = pos * theta / pi, a - 2*floor(a/2)
// is exact in double, so sincospif sees a reduced argument in [0, 2).
__device__ __forceinline__ void rope_cos_sin(double theta_over_pi, int pos, float& c, float& s) {
  const double a = static_cast<double>(pos) * theta_over_pi;
  const double r = a - 2.0 * floor(0.5 * a);
  sincospif(static_cast<float>(r), &s, &c);
}

// Frequencies of the 64 rotate-half pairs, divided by pi (host-computed).
struct RopeTable {
  double theta_over_pi[64];
};

// KV cache addressing: row (in the [rows][128] view of K or V) of the first
// token of block b of (sequence s, KV head h); -1 if the block lies outside
// the cache.
struct KvView {
  const void* k;
  const void* v;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int32_t hkv;
  int32_t capacity;
  int32_t num_pages;
  int32_t max_blocks_per_seq;

  __device__ __forceinline__ long long block_row(int s, int h, int b) const {
    if (b < 0) return -1;
    if (block_table == nullptr) {
      if (static_cast<long long>(b + 1) * kBlock > capacity) return -1;
      return (static_cast<long long>(s) * hkv + h) * capacity + static_cast<long long>(b) * kBlock;
    }
    if (b >= max_blocks_per_seq) return -1;
    const int page = block_table[static_cast<long long>(s) * max_blocks_per_seq + b];
    if (page < 0 || page >= num_pages) return -1;
    return (static_cast<long long>(page) * hkv + h) * kBlock;
  }
};

}  // namespace sas
