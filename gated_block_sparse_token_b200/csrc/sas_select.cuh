// Exact Top-K block selection shared by the decode and prefill kernels.
#pragma once

#include "sas_internal.h"

namespace sas {
namespace {

// Phase stamps of the selection (tracing builds only).
#ifdef SAS_PHASE_TRACE
#define SEL_TRACE(k, v) \
  if (tr != nullptr && threadIdx.x == 0) tr[k] = (v)
#else
#define SEL_TRACE(k, v)
#endif

// Exact Top-K of n <= PER * kThreads scores, the register path (PER = 4:
// every decode context up to 32,768 tokens; PER = 16: up to 131,072): each
// thread keeps the keys of indices PER t .. PER t + PER - 1 in registers;
// buckets are linear in the score value between the finite minimum and
// maximum (monotone in key order: NaN and -inf fall in bucket 0, +inf in
// the last), so the boundary bucket holds few members; the kept set is a bit
// mask, turned into the ascending list by one warp.  Requires topk >= 1 and
// n > topk; same result as the general path.
template <int PER>
__device__ __forceinline__ int select_regs(float* vals, int n, int topk, int cur, int* sel, uint32_t* hist,
                                           uint32_t* selmask, int* scan, unsigned long long* tr) {
  static_assert(PER == 4 || PER == 8 || PER == 16, "4, 8 or 16 keys per thread");
  constexpr int TPW = 32 / PER;                     // threads per 32-bit mask word
  constexpr int WPL = (PER * kThreads / 32 + 31) / 32;  // mask words per lane of warp 0
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned full = 0xffffffffu;
  uint32_t* keys = reinterpret_cast<uint32_t*>(vals);
  const int i0 = PER * tid;
  float x[PER];
  uint32_t k[PER];
  bool valid[PER];
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const float4 v = (i0 + 4 * q < n) ? *reinterpret_cast<const float4*>(vals + i0 + 4 * q)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    x[4 * q] = v.x;
    x[4 * q + 1] = v.y;
    x[4 * q + 2] = v.z;
    x[4 * q + 3] = v.w;
  }
  float fmn = INFINITY, fmx = -INFINITY;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    valid[u] = (i0 + u) < n;
    k[u] = order_key(x[u]);
    if (valid[u] && isfinite(x[u])) {
      fmn = fminf(fmn, x[u]);
      fmx = fmaxf(fmx, x[u]);
    }
  }
  // keys over the scores: each thread rewrites only its own range
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const int b = i0 + 4 * q;
    if (b + 3 < n) {
      *reinterpret_cast<uint4*>(keys + b) = make_uint4(k[4 * q], k[4 * q + 1], k[4 * q + 2], k[4 * q + 3]);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (b + u < n) keys[b + u] = k[4 * q + u];
    }
  }
  *reinterpret_cast<uint4*>(hist + 8 * tid) = make_uint4(0u, 0u, 0u, 0u);
  *reinterpret_cast<uint4*>(hist + 8 * tid + 4) = make_uint4(0u, 0u, 0u, 0u);
  const int words = (n + 31) / 32;  // mask words (selmask holds this many)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    fmn = fminf(fmn, __shfl_xor_sync(full, fmn, o));
    fmx = fmaxf(fmx, __shfl_xor_sync(full, fmx, o));
  }
  float* red = reinterpret_cast<float*>(scan);
  if (lane == 0) {
    red[warp] = fmn;
    red[4 + warp] = fmx;
  }
  if (tid == 0) scan[10] = 0;  // candidate counter
  __syncthreads();
  fmn = fminf(fminf(red[0], red[1]), fminf(red[2], red[3]));
  fmx = fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]));
  SEL_TRACE(0, global_timer_ns());
  const float span = fmx - fmn;
  const float scale = (span > 0.f && isfinite(span)) ? static_cast<float>(kSelBins - 1) / span : 0.f;
  int bk[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    int b = 0;
    if (isfinite(x[u]))
      b = min(kSelBins - 1, static_cast<int>((x[u] - fmn) * scale));
    else if (x[u] > 0.f)
      b = kSelBins - 1;  // +inf; NaN and -inf stay in bucket 0
    bk[u] = b;
    if (valid[u]) atomicAdd(&hist[b], 1u);
  }
  __syncthreads();
  SEL_TRACE(1, global_timer_ns());

  // ---- boundary bucket: thread t sums buckets 1023-8t .. 1016-8t (descending)
  const int hb = kSelBins - 8 * (tid + 1);
  {
    const uint4 h0 = *reinterpret_cast<const uint4*>(hist + hb);
    const uint4 h1 = *reinterpret_cast<const uint4*>(hist + hb + 4);
    const int hv[8] = {static_cast<int>(h0.x), static_cast<int>(h0.y), static_cast<int>(h0.z),
                       static_cast<int>(h0.w), static_cast<int>(h1.x), static_cast<int>(h1.y),
                       static_cast<int>(h1.z), static_cast<int>(h1.w)};
    const int sum = ((hv[0] + hv[1]) + (hv[2] + hv[3])) + ((hv[4] + hv[5]) + (hv[6] + hv[7]));
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) scan[12 + warp] = inc;
    __syncthreads();
    int excl = inc - sum;
    for (int w = 0; w < warp; ++w) excl += scan[12 + w];
    if (excl < topk && topk <= excl + sum) {
      int cum = excl;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (cum < topk && topk <= cum + hv[j]) {
          scan[8] = hb + j;      // the boundary bucket
          scan[9] = topk - cum;  // members of it to keep
        }
        cum += hv[j];
      }
    }
  }
  __syncthreads();
  const int bstar = scan[8];
  const int take = scan[9];
  SEL_TRACE(2, global_timer_ns());

  // ---- kept-above bits (one 32-bit word per TPW threads) and boundary members
  int* cand = reinterpret_cast<int*>(hist);
  uint32_t* candk = hist + kSelCand;
  {
    uint32_t bits = 0u;
    int cnt = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      if (valid[u] && bk[u] > bstar) bits |= 1u << (PER * (tid % TPW) + u);
      cnt += (valid[u] && bk[u] == bstar) ? 1 : 0;
    }
#pragma unroll
    for (int o = 1; o < TPW; o <<= 1) bits |= __shfl_xor_sync(full, bits, o);
    if ((tid % TPW) == 0 && (tid / TPW) < words) selmask[tid / TPW] = bits;
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    int base = 0;
    if (lane == 31 && inc > 0) base = atomicAdd(&scan[10], inc);
    base = __shfl_sync(full, base, 31);
    int pos = base + inc - cnt;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      if (valid[u] && bk[u] == bstar) {
        if (pos < kSelCand) {
          cand[pos] = i0 + u;
          candk[pos] = k[u];
        }
        ++pos;
      }
    }
  }
  __syncthreads();
  const int nc = scan[10];
  SEL_TRACE(3, global_timer_ns());
  SEL_TRACE(5, static_cast<unsigned long long>(nc));

  // ---- exact rank inside the boundary bucket: (key descending, index ascending)
  if (nc <= kSelCand) {
    for (int ci = tid; ci < nc; ci += kThreads) {
      const int i = cand[ci];
      const uint32_t ki = candk[ci];
      int r = 0;
      for (int cj = 0; cj < nc; ++cj) {
        const uint32_t kj = candk[cj];
        r += (kj > ki || (kj == ki && cand[cj] < i)) ? 1 : 0;
      }
      if (r < take) atomicOr(&selmask[i >> 5], 1u << (i & 31));
    }
  } else {
    // a crowded boundary bucket (many equal scores): rank against all members
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      if (!(valid[u] && bk[u] == bstar)) continue;
      const int i = i0 + u;
      int r = 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t kj = keys[j];
        if (kj > k[u] || (kj == k[u] && j < i)) {
          // member of the boundary bucket? (recomputed from the key's value)
          const float xj = __uint_as_float((kj & 0x80000000u) ? (kj & 0x7FFFFFFFu) : ~kj);
          int bj = 0;
          if (kj == 0u)
            bj = 0;
          else if (isfinite(xj))
            bj = min(kSelBins - 1, static_cast<int>((xj - fmn) * scale));
          else if (xj > 0.f)
            bj = kSelBins - 1;
          r += (bj == bstar) ? 1 : 0;
        }
      }
      if (r < take) atomicOr(&selmask[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();
  SEL_TRACE(4, global_timer_ns());

  // ---- ascending list from the mask (one warp: lane l owns words
  // WPL l .. WPL l + WPL - 1)
  if (warp == 0) {
    uint32_t wmask[WPL];
    int c = 0;
#pragma unroll
    for (int w = 0; w < WPL; ++w) {
      const int wi = WPL * lane + w;
      wmask[w] = (wi < words) ? selmask[wi] : 0u;
      c += __popc(wmask[w]);
    }
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    int pos = inc - c;
#pragma unroll
    for (int w = 0; w < WPL; ++w) {
      uint32_t mm = wmask[w];
      while (mm != 0u) {
        const int b = __ffs(mm) - 1;
        sel[pos++] = 32 * (WPL * lane + w) + b;
        mm &= mm - 1u;
      }
    }
    if (lane == 0) sel[topk] = cur;
  }
  __syncthreads();
  return topk + 1;
}

__device__ int select_small(float* vals, int n, int topk, int cur, int* sel, uint32_t* hist, uint32_t* selmask,
                            int* scan, unsigned long long* tr) {
  return select_regs<4>(vals, n, topk, cur, sel, hist, selmask, scan, tr);
}

// contexts of 513 .. 2,048 blocks; out of line so that its 16 keys per
// thread do not weigh on the registers of the kernels that inline the rest
__device__ __noinline__ int select_medium(float* vals, int n, int topk, int cur, int* sel, uint32_t* hist,
                                          uint32_t* selmask, int* scan, unsigned long long* tr) {
  return select_regs<16>(vals, n, topk, cur, sel, hist, selmask, scan, tr);
}

// Top-K selection, general path (pages: training Top-K 31 under the 2,048-token budget).
// Keeps the min(topk, n) largest of vals[0..n) -- ties go to the lower index
// -- lists them ascending in sel[], appends the current block `cur` and
// returns the count.  Exact: scores map to order-preserving 32-bit keys,
// which fall into kSelBins buckets by a monotone map (the leading 10 bits of
// key - min key); the bucket holding the topk-th key is found from the
// histogram, every bucket above it is kept, and the members of that bucket
// are ranked exactly by (key descending, index ascending).
//
// All kThreads threads take part; thread t owns the contiguous index range
// [t * per, (t + 1) * per) with per a multiple of 4 (16-byte key loads), so
// the final ascending list comes from one block-wide prefix sum.  vals must
// be 16-byte aligned with room for ceil(n / 4) * 4 entries; it is
// overwritten with the keys.  hist needs kSelBins words, selbits
// ceil(n / 32) words, scan 16 words.
__device__ __noinline__ int select_large(float* vals, int n, int topk, int cur, int* sel, uint32_t* hist,
                                         uint32_t* selbits, int* scan, unsigned long long* tr) {
  static_assert(kThreads == 128 && kSelBins == 8 * kThreads, "one thread per 8 histogram bins");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned full = 0xffffffffu;
  uint32_t* keys = reinterpret_cast<uint32_t*>(vals);
  const int per = (n + 4 * kThreads - 1) / (4 * kThreads) * 4;
  const int i0 = tid * per;
  const int i1 = min(n, i0 + per);

  // ---- keys, their range; clear the histogram, the marks and the counter
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int i = i0; i < i1; i += 4) {
    const float4 v = *reinterpret_cast<const float4*>(vals + i);
    uint4 k;
    k.x = order_key(v.x);
    k.y = order_key(v.y);
    k.z = order_key(v.z);
    k.w = order_key(v.w);
    if (i + 3 < n) {
      *reinterpret_cast<uint4*>(keys + i) = k;
      lo = min(min(lo, min(k.x, k.y)), min(k.z, k.w));
      hi = max(max(hi, max(k.x, k.y)), max(k.z, k.w));
    } else {
      const uint32_t kk[4] = {k.x, k.y, k.z, k.w};
      for (int u = 0; u < n - i; ++u) {
        keys[i + u] = kk[u];
        lo = min(lo, kk[u]);
        hi = max(hi, kk[u]);
      }
    }
  }
  *reinterpret_cast<uint4*>(hist + 8 * tid) = make_uint4(0u, 0u, 0u, 0u);
  *reinterpret_cast<uint4*>(hist + 8 * tid + 4) = make_uint4(0u, 0u, 0u, 0u);
  for (int w = tid; w < (n + 31) / 32; w += kThreads) selbits[w] = 0u;
  lo = __reduce_min_sync(full, lo);
  hi = __reduce_max_sync(full, hi);
  if (lane == 0) {
    scan[warp] = static_cast<int>(lo);
    scan[4 + warp] = static_cast<int>(hi);
  }
  if (tid == 0) scan[10] = 0;  // candidate counter
  __syncthreads();
  lo = min(min(static_cast<uint32_t>(scan[0]), static_cast<uint32_t>(scan[1])),
           min(static_cast<uint32_t>(scan[2]), static_cast<uint32_t>(scan[3])));
  hi = max(max(static_cast<uint32_t>(scan[4]), static_cast<uint32_t>(scan[5])),
           max(static_cast<uint32_t>(scan[6]), static_cast<uint32_t>(scan[7])));
  const int shift = max(0, 32 - __clz(static_cast<int>((hi - lo) | 1u)) - 10);
  SEL_TRACE(0, global_timer_ns());

  // ---- histogram of buckets
  for (int i = i0; i < i1; ++i) atomicAdd(&hist[(keys[i] - lo) >> shift], 1u);
  __syncthreads();
  SEL_TRACE(1, global_timer_ns());

  // ---- boundary bucket: thread t sums buckets 1023-8t .. 1016-8t (descending)
  const int hb = kSelBins - 8 * (tid + 1);
  const uint4 h0 = *reinterpret_cast<const uint4*>(hist + hb);
  const uint4 h1 = *reinterpret_cast<const uint4*>(hist + hb + 4);
  const uint32_t hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  const int want = topk;
  {
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) sum += static_cast<int>(hv[j]);
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) scan[12 + warp] = inc;
    __syncthreads();
    int excl = inc - sum;
    for (int w = 0; w < warp; ++w) excl += scan[12 + w];
    if (excl < want && want <= excl + sum) {
      int cum = excl;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const int hj = static_cast<int>(hv[j]);
        if (cum < want && want <= cum + hj) {
          scan[8] = hb + j;      // the boundary bucket
          scan[9] = want - cum;  // members of it to keep
        }
        cum += hj;
      }
    }
  }
  __syncthreads();
  const uint32_t bstar = static_cast<uint32_t>(scan[8]);
  const int take = scan[9];
  SEL_TRACE(2, global_timer_ns());

  // ---- members of the boundary bucket, with their keys (the histogram is done)
  int* cand = reinterpret_cast<int*>(hist);
  uint32_t* candk = hist + kSelCand;
  {
    int cnt = 0;
    for (int i = i0; i < i1; ++i) cnt += (((keys[i] - lo) >> shift) == bstar) ? 1 : 0;
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    int base = 0;
    if (lane == 31 && inc > 0) base = atomicAdd(&scan[10], inc);
    base = __shfl_sync(full, base, 31);
    int pos = base + inc - cnt;
    if (cnt > 0) {
      for (int i = i0; i < i1; ++i) {
        const uint32_t k = keys[i];
        if (((k - lo) >> shift) == bstar) {
          if (pos < kSelCand) {
            cand[pos] = i;
            candk[pos] = k;
          }
          ++pos;
        }
      }
    }
  }
  __syncthreads();
  const int nc = scan[10];
  SEL_TRACE(3, global_timer_ns());
  SEL_TRACE(5, static_cast<unsigned long long>(nc));

  // ---- exact rank inside the boundary bucket: (key descending, index ascending)
  if (nc <= kSelCand) {
    for (int ci = tid; ci < nc; ci += kThreads) {
      const int i = cand[ci];
      const uint32_t ki = candk[ci];
      int r = 0;
#pragma unroll 4
      for (int cj = 0; cj < nc; ++cj) {
        const uint32_t kj = candk[cj];
        r += (kj > ki || (kj == ki && cand[cj] < i)) ? 1 : 0;
      }
      if (r < take) atomicOr(&selbits[i >> 5], 1u << (i & 31));
    }
  } else {
    // a crowded boundary bucket (many equal scores): rank against all members
    for (int i = i0; i < i1; ++i) {
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
  __syncthreads();
  SEL_TRACE(4, global_timer_ns());

  // ---- ascending list: every bucket above the boundary plus the marked members
  {
    int cnt = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t b = (keys[i] - lo) >> shift;
      cnt += (b > bstar || (b == bstar && ((selbits[i >> 5] >> (i & 31)) & 1u))) ? 1 : 0;
    }
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(full, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) scan[12 + warp] = inc;
    __syncthreads();
    int pos = inc - cnt;
    for (int w = 0; w < warp; ++w) pos += scan[12 + w];
    if (cnt > 0) {
      for (int i = i0; i < i1; ++i) {
        const uint32_t b = (keys[i] - lo) >> shift;
        if (b > bstar || (b == bstar && ((selbits[i >> 5] >> (i & 31)) & 1u))) sel[pos++] = i;
      }
    }
    if (tid == 0) sel[topk] = cur;
  }
  __syncthreads();
  return topk + 1;
}


// Entry point: trivial budgets, then the short path (n <= 512) inline, the
// 16-keys-per-thread path (n <= 2,048) and the general path out of line
// (keeping their code out of the caller keeps its instruction footprint
// small).  kMedium = false leaves the 16-key path out, for kernels that never
// see more than 512 blocks and should not carry its registers.
template <bool kMedium = true>
__device__ __forceinline__ int select_blocks(float* vals, int n, int topk, int cur, int* sel, uint32_t* hist,
                                             uint32_t* selbits, int* scan, unsigned long long* tr = nullptr) {
  const int tid = threadIdx.x;
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
  if (n <= 4 * kThreads) return select_small(vals, n, topk, cur, sel, hist, selbits, scan, tr);
  if (kMedium && n <= 16 * kThreads) return select_medium(vals, n, topk, cur, sel, hist, selbits, scan, tr);
  return select_large(vals, n, topk, cur, sel, hist, selbits, scan, tr);
}

}  // namespace
}  // namespace sas
