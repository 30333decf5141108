// Exact Top-K block selection shared by the decode and prefill kernels.
#pragma once

#include "sas_internal.h"

namespace sas {
namespace {

// Exclusive prefix sum of v over the kThreads threads (thread order).
__device__ __forceinline__ int block_exclusive_scan(int v, int* scan) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) scan[warp] = inc;
  __syncthreads();
  int off = 0;
  for (int w = 0; w < warp; ++w) off += scan[w];
  __syncthreads();
  return off + inc - v;
}

// Top-K selection (pages: training Top-K 31 under the 2,048-token budget).
// Keeps the min(topk, n) largest of vals[0..n) -- ties go to the lower index
// -- lists them ascending in sel[], appends the current block `cur` and
// returns the count.  Exact: scores map to order-preserving 32-bit keys,
// which fall into kSelBins buckets by a monotone map (the leading 10 bits of
// key - min key); the bucket holding the topk-th key is found from the
// histogram, every bucket above it is kept, and the members of that bucket
// are ranked exactly by (key descending, index ascending).  One warp does the
// work with ballots and warp reductions (no CTA barrier inside); all threads
// of the CTA call it and meet at the final barrier.  Overwrites vals with keys.
__device__ int select_blocks(float* vals, int n, int topk, int cur, int* sel, uint32_t* hist,
                             uint32_t* selbits, int* scan, unsigned long long* tr = nullptr) {
#ifdef SAS_PHASE_TRACE
#define SEL_TRACE(k, v) \
  if (tr != nullptr && threadIdx.x == 0) tr[k] = (v)
#else
#define SEL_TRACE(k, v)
#endif
  (void)scan;
  const int tid = threadIdx.x, lane = tid & 31;
  if (topk <= 0) {  // a 64-token budget keeps the current block only
    if (tid == 0) sel[0] = cur;
    __syncthreads();
    return 1;
  }
  if (n <= topk) {
    for (int i = tid; i < n; i += kThreads) sel[i] = i;
    if (tid == 0) sel[n] = cur;
    __syncthreads();
    return n + 1;
  }
  if (tid < 32) {
    const unsigned full = 0xffffffffu;
    const unsigned lt = (1u << lane) - 1u;
    uint32_t* keys = reinterpret_cast<uint32_t*>(vals);
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int base = 0; base < n; base += 128) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        v[u] = (i < n) ? vals[i] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        if (i < n) {
          const uint32_t k = order_key(v[u]);
          keys[i] = k;
          lo = min(lo, k);
          hi = max(hi, k);
        }
      }
    }
    for (int i = lane; i < kSelBins; i += 32) hist[i] = 0u;
    for (int i = lane; i < (n + 31) / 32; i += 32) selbits[i] = 0u;
    lo = __reduce_min_sync(full, lo);
    hi = __reduce_max_sync(full, hi);
    const int shift = max(0, 32 - __clz(static_cast<int>((hi - lo) | 1u)) - 10);
    __syncwarp();
    SEL_TRACE(0, global_timer_ns());
    for (int base = 0; base < n; base += 128) {
      uint32_t kk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        kk[u] = (i < n) ? keys[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (base + 32 * u + lane < n) atomicAdd(&hist[(kk[u] - lo) >> shift], 1u);
    }
    __syncwarp();
    SEL_TRACE(1, global_timer_ns());
    // buckets in descending order, 32 groups of 32: lane g sums group g
    uint32_t gsum = 0u;
#pragma unroll 8
    for (int g = 0; g < kSelBins / 32; ++g) {
      const uint32_t v = __reduce_add_sync(full, hist[kSelBins - 1 - 32 * g - lane]);
      if (lane == g) gsum = v;
    }
    uint32_t ginc = gsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(full, ginc, o);
      if (lane >= o) ginc += y;
    }
    const uint32_t want = static_cast<uint32_t>(topk);
    const unsigned hitg = __ballot_sync(full, ginc - gsum < want && want <= ginc);
    const int gstar = __ffs(hitg) - 1;
    const uint32_t gexcl = __shfl_sync(full, ginc - gsum, gstar);
    const uint32_t bc = hist[kSelBins - 1 - 32 * gstar - lane];  // lane i: i-th bucket of the group
    uint32_t binc = bc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(full, binc, o);
      if (lane >= o) binc += y;
    }
    const unsigned hitb = __ballot_sync(full, gexcl + binc - bc < want && want <= gexcl + binc);
    const int lstar = __ffs(hitb) - 1;
    const uint32_t bstar = static_cast<uint32_t>(kSelBins - 1 - 32 * gstar - lstar);
    const int take = static_cast<int>(want - gexcl - __shfl_sync(full, binc - bc, lstar));
    __syncwarp();
    SEL_TRACE(2, global_timer_ns());
    // members of the boundary bucket (the histogram is no longer needed)
    int* cand = reinterpret_cast<int*>(hist);
    int nc = 0;
    for (int base = 0; base < n; base += 128) {
      uint32_t kk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        kk[u] = (i < n) ? keys[i] : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        const bool in = i < n && ((kk[u] - lo) >> shift) == bstar;
        const unsigned bal = __ballot_sync(full, in);
        if (in) {
          const int pos = nc + __popc(bal & lt);
          if (pos < kSelCand) cand[pos] = i;
        }
        nc += __popc(bal);
      }
    }
    __syncwarp();
    SEL_TRACE(3, global_timer_ns());
    SEL_TRACE(5, static_cast<unsigned long long>(nc));
    if (nc <= kSelCand) {
      for (int ci = lane; ci < nc; ci += 32) {
        const int i = cand[ci];
        const uint32_t ki = keys[i];
        int r = 0;
        for (int cj = 0; cj < nc; ++cj) {
          const int j = cand[cj];
          const uint32_t kj = keys[j];
          r += (kj > ki || (kj == ki && j < i)) ? 1 : 0;
        }
        if (r < take) atomicOr(&selbits[i >> 5], 1u << (i & 31));
      }
    } else {
      // a crowded boundary bucket (many equal scores): rank against all members
      for (int i = lane; i < n; i += 32) {
        const uint32_t ki = keys[i];
        if (((ki - lo) >> shift) != bstar) continue;
        int r = 0;
        for (int j = 0; j < n; ++j) {
          const uint32_t kj = keys[j];
          r += (((kj - lo) >> shift) == bstar && (kj > ki || (kj == ki && j < i))) ? 1 : 0;
        }
        if (r < take) atomicOr(&selbits[i >> 5], 1u << (i & 31));
      }
    }
    __syncwarp();
    SEL_TRACE(4, global_timer_ns());
    // ascending list: every bucket above the boundary plus the marked members
    int pos = 0;
    for (int base = 0; base < n; base += 128) {
      uint32_t kk[4], sb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        kk[u] = (i < n) ? keys[i] : 0u;
        sb[u] = (i < n) ? selbits[i >> 5] : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + 32 * u + lane;
        bool keep = false;
        if (i < n) {
          const uint32_t b = (kk[u] - lo) >> shift;
          keep = b > bstar || (b == bstar && ((sb[u] >> (i & 31)) & 1u));
        }
        const unsigned bal = __ballot_sync(full, keep);
        if (keep) sel[pos + __popc(bal & lt)] = i;
        pos += __popc(bal);
      }
    }
    if (lane == 0) sel[topk] = cur;
  }
  __syncthreads();
  return topk + 1;
}


}  // namespace
}  // namespace sas
