// SAS decode kernels: gate scores, Top-K block selection and block-sparse
// flash-decoding attention, as one thread-block cluster per (sequence, KV
// head).
//
// Method (release pages: "Tencent released Simple-Attention-Sparsification
// ..." aigc.news 2026-09-14, release paragraph; "Simple-Attention-
// Sparsification Text Generation Model: 12GB+ VRAM", "Specifications and
// Configuration Table"): a 128-wide gate scores every historical 64-token
// block from the Qproj-projected query and the projected, Q/K-normalised,
// RoPE'd max+min+average pooled keys; the top blocks under the token budget
// plus the current block are attended.
//
// Work split of one cluster of CS CTAs (128 threads each) for (s, h):
//   start    the launch may overlap the kernel ahead on the stream
//            (programmatic dependent launch): barriers are set up, and with
//            static weights the W_q column slice and gains requested, before
//            waiting for it; then every load that does not depend on the
//            sequence length (q, the first gate-key chunks) is issued;
//            the length, and for a paged cache every page id of the
//            sequence, is validated.
//   phase 0  each CTA computes 128/CS columns of v_g = q_g @ W_q[g] for the G
//            query heads of the group, one warp per head (large groups: the
//            W_q slice in two passes of ceil(G/2) heads), and stores them into
//            every CTA of the cluster (st.async into distributed shared
//            memory, bytes counted on the receiver's mbarrier); RMSNorm +
//            RoPE -> q~_g.
//   phase 1  each CTA streams 1/CS of the gate keys k~_b (TMA bulk copies
//            into a ring of 16 KiB stage slots), scores its blocks and stores
//            each score into CTA 0.
//   phase 2  CTA 0 runs the exact selection once for the cluster (value
//            buckets, exact ranking inside the boundary bucket, ties to the
//            lower index) and sends the ascending block list to the others.
//            Gated mode: each CTA then computes the gates of its own entries.
//   phase 3  CTA r attends to list entries j = r (mod CS): K and V tiles come
//            in by 2-D TMA (128-byte swizzle); each warp runs flash-decoding
//            over 16 tokens of every tile on bf16 mma.sync (the GQA group as
//            the M=16 rows, fp32 accumulate, online softmax).
//   phase 4  each CTA folds its 4 warps' partials (m, l, o) and stores the
//            128/CS-column slices into the owning CTAs (st.async, counted on
//            the owner's barrier); CTA r merges the CS partials of its columns
//            once all have arrived.
// The CTA that owns the current block (always selected) prefetches its
// tiles before the selection finishes and, when the decoded token completes
// the block, pools it and sends the pooled vector to every CTA; each CTA
// projects it on its 16 W_k columns inside its attention loop (after its
// second list entry, while its warps mostly wait on tiles) and CTA 0
// normalises and rotates the result into the block's gate key before it
// waits for the attention partials.  No cluster barrier follows the start,
// and every wait is bounded.
#include <cooperative_groups.h>

#include <type_traits>

#include "sas_internal.h"
#include "sas_select.cuh"

namespace cg = cooperative_groups;

namespace sas {

// Phase-trace hook: thread 0 of each CTA stamps the global timer at phase
// boundaries (tracing builds only).
#ifdef SAS_PHASE_TRACE
// Slot 0 holds the global timer at the CTA's start (for alignment across
// CTAs) and slot 23 the SM clock there; slot 22 the global timer at the end;
// every other slot the SM clock.
#define SAS_TRACE(k)                                                                        \
  do {                                                                                      \
    const unsigned cta_ = blockIdx.y * gridDim.x + blockIdx.x;                              \
    if (p.trace != nullptr && threadIdx.x == 0 && cta_ < static_cast<unsigned>(kTraceCtas)) { \
      unsigned long long* t_ = p.trace + cta_ * kTraceSlots;                                \
      if ((k) == 0) {                                                                       \
        t_[0] = global_timer_ns();                                                          \
        t_[23] = clock64();                                                                 \
      } else {                                                                              \
        t_[(k)] = clock64();                                                                \
        if ((k) == 8) t_[22] = global_timer_ns();                                           \
      }                                                                                     \
    }                                                                                       \
  } while (0)
#else
#define SAS_TRACE(k) \
  do {               \
  } while (0)
#endif

namespace {

__device__ __forceinline__ uint8_t* align_smem_1024(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return raw + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  acc = fmaf(a.w, b.w, acc);
  return acc;
}

}  // namespace

// Bitonic merge of two descending lists of 32*E keys held by one warp (lane l
// holds elements l + 32 i, i < E): the elementwise maximum of A and reversed B
// holds the 32*E largest keys of both as a bitonic sequence, which the
// cleaning stages sort descending.  Returns them in the same layout.
template <int E>
__device__ __forceinline__ void merge_desc(unsigned long long (&a)[E], const unsigned long long (&b)[E]) {
  const int lane = threadIdx.x & 31;
  unsigned long long c[E];
#pragma unroll
  for (int i = 0; i < E; ++i) {
    // reversed B: element 32E-1-(l+32i) = lane 31-l, slot E-1-i
    const unsigned long long br = __shfl_sync(0xffffffffu, b[E - 1 - i], 31 - lane);
    c[i] = a[i] > br ? a[i] : br;
  }
#pragma unroll
  for (int j = 16 * E; j > 0; j >>= 1) {
    if (j >= 32) {  // partner in another slot of the same lane
      const int js = j / 32;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        if ((i & js) == 0) {
          const unsigned long long x = c[i], y = c[i | js];
          c[i] = x > y ? x : y;
          c[i | js] = x > y ? y : x;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, c[i], j);
        const bool keep_max = (lane & j) == 0;
        c[i] = keep_max ? (c[i] > y ? c[i] : y) : (c[i] > y ? y : c[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < E; ++i) a[i] = c[i];
}

// Distributed exact Top-K of one cluster of 8 CTAs (the fused step's
// selection when the sequence keeps at most kFastTopk historical blocks).
// Every CTA holds the (score, block) keys of its own gate-key rows in lkeys
// (keys are distinct: the block index breaks score ties toward the lower
// block; key 0 sorts below every key).  (1) each CTA ranks its keys by
// counting and sends its best plen[rank], in descending order, to every CTA
// of the cluster (st.async into gather[rank][.], bytes counted on bar);
// (2) every CTA merges the 8 sorted lists with a bitonic merge tree (four
// warps, then two, then one; lists of 32*E keys, E = 1 or 2) -- the global
// best topk always lie among them, each being among its own CTA's best topk
// -- whose first topk are the kept blocks; (3) warp 0 sorts their block
// ids ascending (a bitonic network over the warp) into sel[0 .. topk), then
// sel[topk] = cur.  lkeys and gather are scratch from step (2) on.
// Returns false if the candidates did not all arrive (bounded wait; the
// timeout bit is then set).  Ends with a block-wide barrier.
// Ascending bitonic sort of 32*E values held by one warp (lane l holds
// elements l + 32 i, i < E).
template <int E>
__device__ __forceinline__ void warp_sort_asc(uint32_t (&x)[E]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {  // partner in another slot of the same lane
        const int js = j / 32;
#pragma unroll
        for (int i = 0; i < E; ++i) {
          if ((i & js) == 0) {
            const bool asc = ((lane + 32 * i) & k) == 0;
            const uint32_t lo = min(x[i], x[i | js]), hi = max(x[i], x[i | js]);
            x[i] = asc ? lo : hi;
            x[i | js] = asc ? hi : lo;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const uint32_t y = __shfl_xor_sync(0xffffffffu, x[i], j);
          const bool asc = ((lane + 32 * i) & k) == 0;
          const bool lower = (lane & j) == 0;
          x[i] = (lower == asc) ? min(x[i], y) : max(x[i], y);
        }
      }
    }
  }
}

template <int E>
__device__ __forceinline__ void load_list(unsigned long long (&v)[E], const unsigned long long* lst, int len) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] = (lane + 32 * i < len) ? lst[lane + 32 * i] : 0ull;
}

template <int CS, int E>
__device__ __noinline__ bool distributed_topk(unsigned long long* lkeys, unsigned long long* gather,
                                              const int* plen, int topk, int cur,
                                              int rank, int* sel, uint64_t* bar, uint32_t* status,
                                              unsigned long long* tr) {
  static_assert(CS == 8, "the merge tree has three levels");
  constexpr int LEN = 32 * E;  // list length of the merge
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // rows this CTA holds (plen[CS]); only the first plen[rank] ranks are sent
  const int nl = plen[CS];
  const int P = plen[rank];
  const int split = (nl <= 32) ? 4 : ((nl <= 64) ? 2 : 1);  // threads per key
  for (int base0 = 0; base0 < nl * split; base0 += kThreads) {
    const int idx = base0 + tid;
    const int i = idx / split, part = idx - i * split;
    const bool live = i < nl;
    const unsigned long long x = live ? lkeys[i] : 0ull;
    int r = 0;
    if (live) {
#pragma unroll 8
      for (int jj = part; jj < nl; jj += split) r += (lkeys[jj] > x) ? 1 : 0;
    }
    if (split >= 2) r += __shfl_xor_sync(0xffffffffu, r, 1);
    if (split >= 4) r += __shfl_xor_sync(0xffffffffu, r, 2);
    if (live && part == 0 && r < P) {
#pragma unroll
      for (int dst = 0; dst < CS; ++dst)
        st_async_u64(dsmem_addr(gather + rank * kFastTopk + r, dst), x, dsmem_addr(bar, dst));
    }
  }
  if (tr != nullptr && tid == 0) tr[0] = clock64();  // candidates sent
  bool ok = mbar_wait_cluster(bar, 0, status);  // every CTA's candidates
  ok = __syncthreads_and(ok) != 0;             // (and every read of lkeys is done)
  if (!ok) return false;
  if (tr != nullptr && tid == 0) tr[1] = clock64();  // candidates in
  // merge tree: level 1 into lkeys (4 lists), level 2 into gather (2 lists)
  unsigned long long a[E], b[E];
  {
    load_list<E>(a, gather + (2 * warp) * kFastTopk, plen[2 * warp]);
    load_list<E>(b, gather + (2 * warp + 1) * kFastTopk, plen[2 * warp + 1]);
    merge_desc<E>(a, b);
#pragma unroll
    for (int i = 0; i < E; ++i) lkeys[warp * LEN + lane + 32 * i] = a[i];
  }
  __syncthreads();
  if (warp < 2) {
    load_list<E>(a, lkeys + (2 * warp) * LEN, LEN);
    load_list<E>(b, lkeys + (2 * warp + 1) * LEN, LEN);
    merge_desc<E>(a, b);
#pragma unroll
    for (int i = 0; i < E; ++i) gather[warp * LEN + lane + 32 * i] = a[i];
  }
  __syncthreads();
  if (warp == 0) {
    load_list<E>(a, gather, LEN);
    load_list<E>(b, gather + LEN, LEN);
    merge_desc<E>(a, b);
    if (tr != nullptr && lane == 0) tr[2] = clock64();  // merged
    // the first topk of the merged list are the kept blocks: their ids,
    // sorted ascending (the rest sort last), give the list
    uint32_t blk[E];
#pragma unroll
    for (int i = 0; i < E; ++i)
      blk[i] = (lane + 32 * i < topk) ? ~static_cast<uint32_t>(a[i] & 0xFFFFFFFFull) : 0xFFFFFFFFu;
    warp_sort_asc<E>(blk);
#pragma unroll
    for (int i = 0; i < E; ++i)
      if (lane + 32 * i < topk) sel[lane + 32 * i] = static_cast<int>(blk[i]);
    if (lane == 0) sel[topk] = cur;
  }
  __syncthreads();
  return true;
}

template <typename T, typename OutT, int CS, int NST, int MODE>
__global__ void __launch_bounds__(kThreads, 4)
    decode_cluster_kernel(const __grid_constant__ DecodeParams p,
                          const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv,
                          const __grid_constant__ CUtensorMap tmw,
                          const __grid_constant__ CUtensorMap tmwk) {
  constexpr bool kF32 = std::is_same<T, float>::value;
  constexpr int kDpc = kDim / CS;               // output / W_q columns per CTA
  constexpr int kTilesPerBlock = kF32 ? 4 : 2;  // 16 KiB tiles per K+V block
  static_assert(kDpc == 16, "the gate-query GEMV maps 8 row groups x 4 column quads to a warp");
  static_assert((CS & (CS - 1)) == 0, "power-of-two clusters");

  cg::cluster_group cluster = cg::this_cluster();
  SAS_TRACE(0);
  const int rank = static_cast<int>(cluster.block_rank());
  const int pair = blockIdx.y;
  const int s = pair / p.hkv;
  const int h = pair - s * p.hkv;
  const int G = p.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem_1024(smem_raw);
  uint8_t* slots = base + p.sm.slots;
  int* sel = reinterpret_cast<int*>(base + p.sm.sel);
  T* qraw = reinterpret_cast<T*>(base + p.sm.qraw);
  float* qbar = reinterpret_cast<float*>(base + p.sm.qbar);
  float* pm = reinterpret_cast<float*>(base + p.sm.pml);
  float* pl = pm + kWarps * kMaxGroup;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + p.sm.bars);
  float* qv = reinterpret_cast<float*>(base + p.sm.r_qv);
  __nv_bfloat16* wq_s = reinterpret_cast<__nv_bfloat16*>(base + p.sm.r_wq);
  float* gam_s = reinterpret_cast<float*>(base + p.sm.gam);
  uint64_t* bar_pro = bars + NST;     // prologue copies: q, W_q slice, gamma_q (, gamma_k)
  uint64_t* bar_p = bars + NST + 1;   // pooled current block has arrived (cluster scope)
  uint64_t* bar_wk = bars + NST + 2;  // W_k column slice has arrived
  // Cluster exchanges: the sender stores into the receiver's shared memory
  // with st.async, which completes the bytes on the receiver's barrier; the
  // receiver registers the bytes it expects (its own single arrival).
  uint64_t* bar_sc = bars + NST + 3;  // rank 0: the scores of every CTA
  uint64_t* bar_sel = bars + NST + 4; // ranks > 0: the block list from rank 0
  uint64_t* bar_v = bars + NST + 5;   // the gate query v (a slice from each CTA)
  uint64_t* bar_m = bars + NST + 6;   // attention partials of this CTA's columns
  uint64_t* bar_u = bars + NST + 7;   // rank 0: projected pooled slices
  uint64_t* bar_wq2 = bars + NST + 8; // second pass of the W_q slice (large groups)
  const int wq_heads = p.sm.wq_heads;  // heads of the W_q slice resident at once
  float* pool_p = reinterpret_cast<float*>(base + p.sm.r_pool_p);
  float* pool_u = reinterpret_cast<float*>(base + p.sm.r_pool_u);
  __nv_bfloat16* wk_s = reinterpret_cast<__nv_bfloat16*>(base + p.sm.r_wk);
  float* gamk_s = reinterpret_cast<float*>(base + p.sm.gamk);
  const bool pool_on = (MODE == kModeFused) && (p.gamma_k != nullptr);
  float* inbox_o = reinterpret_cast<float*>(base + p.sm.r_inbox);  // [CS][G][kDpc]
  float* inbox_ml = inbox_o + CS * G * kDpc;                         // [CS][G][2]
  float* keys = reinterpret_cast<float*>(base + p.sm.r_keys);
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + p.sm.r_hist);
  uint32_t* selbits = reinterpret_cast<uint32_t*>(base + p.sm.r_selbits);
  int* scan = reinterpret_cast<int*>(base + p.sm.r_scan);
  float* po = reinterpret_cast<float*>(slots);  // [4][G][128], after the last tile
  // gated mode: log-sigmoid gate of list entry j for head g at gbias[j * G + g]
  float* gbias = reinterpret_cast<float*>(base + p.sm.gbias);
  const bool gated = (MODE == kModeFused) && p.gated != 0;
  // paged cache: rows of this CTA's list entries, looked up once in parallel
  // when the list is in hand (the issuer then needs no page-table load per tile)
  long long* rows_s = reinterpret_cast<long long*>(base + p.sm.rows);
  const bool paged = p.kv.block_table != nullptr;
  bool rows_cached = false;  // meaningful in thread 0 only

  // ------------------------------------------------------------ gate-key partition
  // The gate-key rows of (s, h) are split over the cluster in chunks of one
  // 16 KiB ring slot (32 fp32 or 64 bf16 rows): chunk j goes to CTA j % CS.
  // The split does not depend on the sequence length, so each CTA requests
  // its first NST chunks that lie inside the gate-key cache before the length
  // is known (a chunk past the historical blocks is then not scored).
  const int gk_rows = p.gk16 ? 2 * kGkChunk : kGkChunk;
  const int gk_shift = p.gk16 ? 6 : 5;  // log2(gk_rows)
  static_assert(kGkChunk == 32, "gate-key chunks of 32 fp32 or 64 bf16 rows");
  const uint32_t gk_row_bytes = p.gk16 ? kDim * 2u : kDim * 4u;
  const uint8_t* gk_pair = static_cast<const uint8_t*>(p.gate_keys) + static_cast<size_t>(pair) * p.mg * gk_row_bytes;
  int nspec = 0;  // chunks requested before the length is known (tiles 0 .. nspec-1)
  if (MODE != kModeAttend)
    while (nspec < NST && (rank + nspec * CS) * gk_rows < p.mg) ++nspec;

  // ------------------------------------------------------------ prologue copies
  // The launch may overlap the kernels ahead on the stream (programmatic
  // dependent launch).  Thread 0 initialises the barriers before waiting for
  // them; when the caller declares the weights static, it also requests
  // gamma_q, gamma_k and the CTA's W_q column slice (one 2-D TMA box per
  // head) before the wait.  q, the length, the budget, the gate keys and
  // the cache are always read after it.
  int* len_s = reinterpret_cast<int*>(qbar);  // qbar is written only after the validation
  auto issue_weights = [&]() {
    if (MODE != kModeAttend) {
      bulk_g2s(gam_s, p.gamma_q, kDim * 4, bar_pro);
      for (int g = 0; g < wq_heads; ++g)
        tma_load_2d(wq_s + static_cast<size_t>(g) * kDim * kDpc, &tmw, rank * kDpc, (h * G + g) * kDim, bar_pro);
    }
    if (pool_on) bulk_g2s(gamk_s, p.gamma_k, kDim * 4, bar_pro);
  };
  if (tid == 0) {
    // the kernel behind this one may be scheduled from now on: it reads
    // nothing this grid writes before this grid has completed
    griddep_launch_dependents();
    if (MODE != kModeAttend) prefetch_tensormap(&tmw);
    if constexpr (!kF32 && MODE != kModeGate) {
      prefetch_tensormap(&tmk);
      prefetch_tensormap(&tmv);
    }
    if (pool_on) prefetch_tensormap(&tmwk);
    for (int i = 0; i < NST + 9; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    const uint32_t qbytes = static_cast<uint32_t>(G * kDim * sizeof(T));
    uint32_t tx = qbytes;
    if (MODE != kModeAttend) tx += static_cast<uint32_t>(wq_heads * kDim * kDpc * 2 + kDim * 4);
    if (pool_on) tx += kDim * 4;
    mbar_arrive_expect_tx(bar_pro, tx);
    // the gate query v arrives from every CTA whatever the length holds
    if (MODE != kModeAttend) mbar_arrive_expect_tx(bar_v, static_cast<uint32_t>(G * kDim * 4));
    if (p.static_weights) issue_weights();
  }
  // q in page-locked host memory: each CTA loads one eighth of the cluster's
  // query over the host link (16 bytes a lane of warp 1) and, after the
  // cluster barrier, stores it into every CTA's q buffer, so the link carries
  // each byte once.  The caller guarantees that no earlier device work writes
  // that memory, so the loads go out before the wait.
  constexpr int kQWords = kDim * static_cast<int>(sizeof(T)) / (16 * CS);  // words per head and CTA
  static_assert(kQWords * 16 * CS == kDim * static_cast<int>(sizeof(T)), "q rows split evenly over the cluster");
  const bool q_sender = p.q_mapped && warp == 1 && lane < G * kQWords;
  uint4 q_word = make_uint4(0u, 0u, 0u, 0u);
  if (q_sender)
    q_word = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                            (static_cast<size_t>(s) * p.hq + static_cast<size_t>(h) * G) *
                                                kDim)[rank * G * kQWords + lane];
  griddep_wait();
  if (tid == 0) {
    const int L0 = p.kv.seq_lens[s];
    const int topk0 = (MODE == kModeFused) ? p.kv.topk_of(s) : 0;  // this sequence's budget
    if (!p.q_mapped)
      bulk_g2s(qraw,
               static_cast<const T*>(p.q) + (static_cast<size_t>(s) * p.hq + static_cast<size_t>(h) * G) * kDim,
               G * kDim * static_cast<uint32_t>(sizeof(T)), bar_pro);
    if (!p.static_weights) issue_weights();
    for (int k = 0; k < nspec; ++k) {
      const int r0 = (rank + k * CS) * gk_rows;
      const uint32_t bytes = static_cast<uint32_t>(min(gk_rows, p.mg - r0)) * gk_row_bytes;
      mbar_arrive_expect_tx(&bars[k], bytes);
      bulk_g2s(slots + k * kTileBytes, gk_pair + static_cast<size_t>(r0) * gk_row_bytes, bytes, &bars[k]);
    }
    len_s[0] = L0;
    len_s[1] = topk0;
  }
  SAS_TRACE(16);  // thread 0: prologue copies requested
  // thread 0 arrives after its barrier initialisation: no CTA of the cluster
  // passes cluster_wait() (and stores into this one) before it
  cluster_arrive_relaxed();
  double th0 = 0.0, th1 = 0.0;
  if (MODE != kModeAttend) {
    th0 = p.rope.theta_over_pi[lane];
    th1 = p.rope.theta_over_pi[lane + 32];
  }

  // ------------------------------------------------------------ phase 0: gate query projection
  // v_g = q_g @ W_q[g] needs no length: it runs while the length load is in
  // flight.  One warp per head: each lane accumulates 16 rows (8 apart) of
  // 4 columns, shuffles sum the 8 row groups, and every CTA of the cluster
  // receives every column (one 16-byte asynchronous store per lane).
  // Large groups take the W_q slice in two passes through the same region
  // (the second copy is requested once every read of the first is done).
  // the cluster barrier first: every thread of the cluster has arrived, so
  // thread 0's barrier initialisation (fenced before its arrival) is visible
  // before any thread waits on those barriers, and every CTA runs before
  // stores reach it
  cluster_wait();
  if (q_sender) {
    const uint32_t off = static_cast<uint32_t>(rank * G * kQWords + lane) * 16u;
#pragma unroll 1
    for (int r = 0; r < CS; ++r)
      st_async_v4_f32(dsmem_addr(reinterpret_cast<const char*>(qraw) + off, r), __uint_as_float(q_word.x),
                      __uint_as_float(q_word.y), __uint_as_float(q_word.z), __uint_as_float(q_word.w),
                      dsmem_addr(bar_pro, r));
  }
  const bool pro_ok = mbar_wait(bar_pro, 0, p.status);
  SAS_TRACE(21);  // prologue copies in
  if (MODE != kModeAttend) {
    bool wq_ok = pro_ok;
    for (int g0 = 0; g0 < G; g0 += wq_heads) {
      const int gn = min(wq_heads, G - g0);
      if (g0 > 0) {
        __syncthreads();
        if (tid == 0) {
          fence_proxy_async_smem();  // the slice's generic reads before the async-proxy overwrite
          mbar_arrive_expect_tx(bar_wq2, static_cast<uint32_t>(gn * kDim * kDpc * 2));
          for (int g = 0; g < gn; ++g)
            tma_load_2d(wq_s + static_cast<size_t>(g) * kDim * kDpc, &tmw, rank * kDpc,
                        (h * G + g0 + g) * kDim, bar_wq2);
        }
        wq_ok = mbar_wait(bar_wq2, 0, p.status) && wq_ok;
      }
      // warp w: heads w, w + 4, ..; lane (rg, cq): rows rg, rg + 8, .., rg +
      // 120 of columns 4 cq .. 4 cq + 3 of the CTA's slice (one load step
      // reads 8 consecutive 32-byte rows: no bank conflicts)
      const int cq = lane & 3, rg = lane >> 2;
      for (int gl = warp; gl < gn; gl += kWarps) {
        const int g = g0 + gl;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        if (wq_ok) {
          const __nv_bfloat16* wrow = wq_s + (static_cast<size_t>(gl) * kDim + rg) * kDpc + 4 * cq;
          const T* qcol = qraw + g * kDim + rg;
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float x = to_float(qcol[8 * u]);
            const uint2 w = *reinterpret_cast<const uint2*>(wrow + 8 * u * kDpc);
            a0 = fmaf(x, __uint_as_float(w.x << 16), a0);
            a1 = fmaf(x, __uint_as_float(w.x & 0xffff0000u), a1);
            a2 = fmaf(x, __uint_as_float(w.y << 16), a2);
            a3 = fmaf(x, __uint_as_float(w.y & 0xffff0000u), a3);
          }
        }
        if (gl == 0) SAS_TRACE(24);  // thread 0: products summed
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          a0 += __shfl_xor_sync(0xffffffffu, a0, o);
          a1 += __shfl_xor_sync(0xffffffffu, a1, o);
          a2 += __shfl_xor_sync(0xffffffffu, a2, o);
          a3 += __shfl_xor_sync(0xffffffffu, a3, o);
        }
        if (gl == 0) SAS_TRACE(25);  // thread 0: row groups combined
        // the lanes of row group r deliver the four columns to CTA r
        st_async_v4_f32(dsmem_addr(qv + g * kDim + rank * kDpc + 4 * cq, rg), a0, a1, a2, a3,
                        dsmem_addr(bar_v, rg));
      }
    }
  }
  SAS_TRACE(1);

  // ------------------------------------------------------------ validation
  __syncthreads();
  const int L = len_s[0];
  const int topk = len_s[1];  // fused mode: historical blocks kept for this sequence
  bool err = (L < 1) || topk < 0;
  const int c = err ? 0 : (L - 1) / kBlock;  // current block
  if (MODE != kModeAttend && c > p.mg) err = true;
  if (MODE == kModeFused && !err) {
    // every block 0..c must map to cache rows.  Contiguous: one bound (rows
    // grow with the block index).  Paged: every page id of the sequence in
    // the pool, 16 independent loads in flight per thread.
    if (p.kv.block_table == nullptr) {
      if (p.kv.block_row(s, h, c) < 0) err = true;
    } else if (c >= p.kv.max_blocks_per_seq) {
      err = true;
    } else {
      const int32_t* trow = p.kv.block_table + static_cast<long long>(s) * p.kv.max_blocks_per_seq;
      for (int b0 = tid; b0 <= c; b0 += 16 * kThreads) {
        int pg[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int b = b0 + u * kThreads;
          pg[u] = (b <= c) ? trow[b] : 0;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (pg[u] < 0 || pg[u] >= p.kv.num_pages) err = true;
      }
    }
  }
  int m = 0;  // entries of the block list (current block last)
  if (MODE == kModeAttend && !err) {
    const int mm = p.sel_count[pair];
    if (mm < 1 || mm > p.max_sel) {
      err = true;
    } else {
      const int32_t* si = p.sel_idx + static_cast<size_t>(pair) * p.max_sel;
      for (int j = tid; j < mm; j += kThreads) {
        const int b = si[j];
        sel[j] = b;
        if (b < 0 || b > c) err = true;
        if (j == mm - 1 && b != c) err = true;
        if (j > 0 && si[j - 1] >= b) err = true;
        if (p.kv.block_row(s, h, b) < 0) err = true;
      }
      m = mm;
    }
  }
  const bool bad = __syncthreads_or(err) != 0;
  SAS_TRACE(17);  // length read and validated
  if (bad && rank == 0 && tid == 0) raise_status(p.status, kStatusBounds);
  const int n = bad ? 0 : c;  // historical blocks
  // the decoded token completes block c: pool it into gate-key row c
  const bool do_pool = pool_on && !bad && (L % kBlock == 0) && (c < p.mg);
  if (MODE == kModeFused) m = bad ? 0 : min(topk, n) + 1;
  if (MODE == kModeAttend && bad) m = 0;

  // gate-key chunks of this CTA: global chunks rank, rank + CS, ... below
  // ceil(n / gk_rows); the speculative ones are tiles 0 .. nspec-1 whatever
  // the length turned out to be
  const int nch_all = (n + gk_rows - 1) >> gk_shift;
  const int nch_need = (MODE == kModeAttend || nch_all <= rank) ? 0 : (nch_all - rank + CS - 1) / CS;
  const int nchunks = (MODE == kModeAttend) ? 0 : max(nch_need, nspec);
  // historical blocks (gate-key rows) CTA r scores: its full chunks plus the
  // partial last chunk if it owns it
  auto rows_of = [&](int r) -> int {
    const int full = n >> gk_shift, rem = n & (gk_rows - 1);
    const int nf = (full > r) ? (full - r + CS - 1) / CS : 0;
    return nf * gk_rows + ((rem > 0 && (full & (CS - 1)) == r) ? rem : 0);
  };
  // Top-K route: nothing to choose (a 64-token budget, or every historical
  // block kept); the distributed selection; or every score to rank 0, which
  // selects for the cluster (budgets above kFastTopk + 1 blocks, very long
  // contexts)
  const bool sel_local = (MODE == kModeFused) && (topk <= 0 || n <= topk);
  const bool sel_fast = (MODE == kModeFused) && !sel_local && topk <= kFastTopk &&
                        ((nch_all + CS - 1) / CS) * gk_rows <= kFastRows;
  const int cnt_mine = (rank < m) ? (m - 1 - rank) / CS + 1 : 0;
  const bool own_cur = (m > 0) && ((m - 1) % CS == rank);
  unsigned long long* lkeys = reinterpret_cast<unsigned long long*>(base + p.sm.r_lkeys);
  unsigned long long* gather = reinterpret_cast<unsigned long long*>(base + p.sm.r_gather);

  // bytes this CTA will receive from the cluster (bad is uniform over it)
  if (tid == 0) {
    if (MODE == kModeFused && !bad) {
      if (sel_fast) {
        uint32_t bytes = 0;
        for (int r = 0; r < CS; ++r) bytes += static_cast<uint32_t>(min(topk, rows_of(r))) * 8u;
        mbar_arrive_expect_tx(bar_sc, bytes);
      } else if (!sel_local) {
        if (rank == 0)
          mbar_arrive_expect_tx(bar_sc, static_cast<uint32_t>(n * 4));
        else
          mbar_arrive_expect_tx(bar_sel, static_cast<uint32_t>(m * 4));
      } else {
        mbar_arrive_expect_tx(bar_sc, static_cast<uint32_t>(CS * 4));  // one token per CTA
      }
    }
    if (do_pool) {
      mbar_arrive_expect_tx(bar_p, kPool * 4);
      if (rank == 0) mbar_arrive_expect_tx(bar_u, CS * 17 * 4);
    }
    if (MODE != kModeGate) mbar_arrive_expect_tx(bar_m, static_cast<uint32_t>(CS * G * (kDpc + 2) * 4));
  }

  // list entry e of this CTA -> block id (the current block first if owned)
  auto entry_index = [&](int e) -> int {
    if (own_cur) return (e == 0) ? (m - 1) : rank + (e - 1) * CS;
    return rank + e * CS;
  };
  auto entry_block = [&](int e) -> int {
    const int j = entry_index(e);
    return (j == m - 1) ? c : sel[j];
  };

  // ------------------------------------------------------------ tile ring
  // Tile t lives in slot t % NST, phase (t / NST) & 1.  Tiles 0..nchunks-1
  // are gate-key chunks, then kTilesPerBlock tiles per list entry.  Thread 0
  // issues tile t once tile t - NST has been released by every thread.
  int issued = nspec;  // meaningful in thread 0 only
  auto issue = [&](int t, bool traced) {
    const int slot = t % NST;
    uint8_t* dst = slots + slot * kTileBytes;
    if (t < nchunks) {
      const int b0 = (rank + t * CS) * gk_rows;
      const int cntb = min(gk_rows, n - b0);
      const uint32_t bytes = static_cast<uint32_t>(cntb) * gk_row_bytes;
      mbar_arrive_expect_tx(&bars[slot], bytes);
      bulk_g2s(dst, gk_pair + static_cast<size_t>(b0) * gk_row_bytes, bytes, &bars[slot]);
      return;
    }
    const int k = t - nchunks;
    const int e = k / kTilesPerBlock;
    const int part = k - e * kTilesPerBlock;
    const long long row0 = rows_cached ? rows_s[e] : p.kv.block_row(s, h, entry_block(e));
    if (traced) SAS_TRACE(9);
    mbar_arrive_expect_tx(&bars[slot], kTileBytes);
    if (traced) SAS_TRACE(19);
    if constexpr (kF32) {
      const float* src = static_cast<const float*>(part < 2 ? p.kv.k : p.kv.v) +
                         (row0 + (part & 1) * 32) * kDim;
      bulk_g2s(dst, src, kTileBytes, &bars[slot]);
    } else {
      const CUtensorMap* map = (part == 0) ? &tmk : &tmv;
      tma_load_2d(dst, map, 0, static_cast<int>(row0), &bars[slot]);
      if (traced) SAS_TRACE(26);
      tma_load_2d(dst + 8192, map, 64, static_cast<int>(row0), &bars[slot]);
    }
  };
  auto pump = [&](int consumed, int known, bool traced = false) {
    if (tid != 0) return;
    if (traced) SAS_TRACE(27);
    fence_proxy_async_smem();
    if (traced) SAS_TRACE(28);
    bool first = traced;
    while (issued < known && issued < consumed + NST) {
      issue(issued++, first);
      first = false;
    }
    if (traced) SAS_TRACE(29);
  };

  // before the selection only the gate-key chunks and the current block are known
  int known = nchunks + ((MODE == kModeAttend) ? kTilesPerBlock * cnt_mine
                                               : (own_cur ? kTilesPerBlock : 0));
  pump(0, known);
  if (tid == 0) {
    // the ring holds NST chunks: ask L2 for this CTA's later chunks now
    for (int t = NST; t < nch_need; ++t) {
      const int b0 = (rank + t * CS) * gk_rows;
      prefetch_l2(gk_pair + static_cast<size_t>(b0) * gk_row_bytes,
                  static_cast<uint32_t>(min(gk_rows, n - b0)) * gk_row_bytes);
    }
  }

  // ------------------------------------------------------------ gate query: norm and RoPE
  // the rotation at position c needs only the length: computed while v is
  // still on its way
  float c0 = 1.f, s0 = 0.f, c1 = 1.f, s1 = 0.f;
  if (MODE != kModeAttend && !bad) {
    rope_cos_sin(th0, c, c0, s0);
    rope_cos_sin(th1, c, c1, s1);
  }
  if (MODE != kModeAttend) mbar_wait_cluster(bar_v, 0, p.status);  // every column of v is here
  SAS_TRACE(2);

  if (MODE != kModeAttend) {
    if (!bad) {
      // Q normalisation (RMSNorm, gain gamma_q) and gate RoPE at position c.
      for (int g = warp; g < G; g += kWarps) {
        float x[4];
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[k] = qv[g * kDim + lane + 32 * k];
          ss = fmaf(x[k], x[k], ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = 1.f / sqrtf(ss / kDim + p.eps);
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = x[k] * inv * gam_s[lane + 32 * k];
        qv[g * kDim + lane] = x[0] * c0 - x[2] * s0;
        qv[g * kDim + lane + 64] = x[2] * c0 + x[0] * s0;
        qv[g * kDim + lane + 32] = x[1] * c1 - x[3] * s1;
        qv[g * kDim + lane + 96] = x[3] * c1 + x[1] * s1;
      }
    }
    __syncthreads();
    if (MODE == kModeFused && !bad) {
      // S_b = mean_g(q~_g . k~_b) * scale = (scale/G * sum_g q~_g) . k~_b
      const float f = p.gate_scale / static_cast<float>(G);
      for (int d = tid; d < kDim; d += kThreads) {
        float a = 0.f;
        for (int g = 0; g < G; ++g) a += qv[g * kDim + d];
        qbar[d] = a * f;
      }
    }
    __syncthreads();

    // ---------------------------------------------------------- phase 1: scores
    const int grp = lane >> 3;  // 4 blocks per warp at a time, 8 lanes per block
    const int sub = lane & 7;   // lane covers dims sub*16 .. sub*16+15
    // fp32 keys: chunk rotation for conflict-free 16-byte loads; bf16 keys:
    // natural order (each lane reads 32 contiguous bytes)
    const int rot = p.gk16 ? 0 : sub >> 1;
    float4 qr[4];
    if (MODE == kModeFused) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        qr[i] = *reinterpret_cast<const float4*>(qbar + sub * 16 + ((i + rot) & 3) * 4);
    }
    SAS_TRACE(14);  // q~ and the head mean ready
    for (int ci = 0; ci < nchunks; ++ci) {
      const int slot = ci % NST;
      const bool ok = mbar_wait(&bars[slot], (ci / NST) & 1, p.status);
      if (ci == 0) SAS_TRACE(15);  // first gate-key chunk in
      const int b0 = (rank + ci * CS) * gk_rows;
      const int cntb = max(0, min(gk_rows, n - b0));  // 0 for a speculative chunk past n
      const float* gk = reinterpret_cast<const float*>(slots + slot * kTileBytes);
      const uint8_t* gk16 = slots + slot * kTileBytes;
      for (int it = 0; it < gk_rows / 16; ++it) {
        const int bb = it * 16 + warp * 4 + grp;
        const bool act = ok && bb < cntb;
        const float* row = gk + bb * kDim + sub * 16;
        const uint8_t* row16 = gk16 + bb * (kDim * 2) + sub * 32;
        float S = 0.f;
        if (MODE == kModeFused) {
          float acc = 0.f;
          if (act) {
            if (p.gk16) {
              acc = dot8_bf16(qr[0], qr[1], *reinterpret_cast<const uint4*>(row16), acc);
              acc = dot8_bf16(qr[2], qr[3], *reinterpret_cast<const uint4*>(row16 + 16), acc);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                acc = dot4(qr[i], *reinterpret_cast<const float4*>(row + ((i + rot) & 3) * 4), acc);
            }
          }
          acc += __shfl_xor_sync(0xffffffffu, acc, 1);
          acc += __shfl_xor_sync(0xffffffffu, acc, 2);
          acc += __shfl_xor_sync(0xffffffffu, acc, 4);
          S = acc;
          if (sub == 0 && bb < cntb) {
            if (sel_fast) {
              // (score, block) key: larger score first, then the lower block
              lkeys[ci * gk_rows + bb] = (static_cast<unsigned long long>(order_key(S)) << 32) |
                                         static_cast<unsigned long long>(~static_cast<uint32_t>(b0 + bb));
            } else if (!sel_local) {
              // rank 0 of the cluster receives every score and selects
              st_async_f32(dsmem_addr(keys + b0 + bb, 0), S, dsmem_addr(bar_sc, 0));
            }
          }
        } else {
          for (int g = 0; g < G; ++g) {
            float acc = 0.f;
            if (act) {
              const float* qrow = qv + g * kDim + sub * 16;
              if (p.gk16) {
                const float4* q4 = reinterpret_cast<const float4*>(qrow);
                acc = dot8_bf16(q4[0], q4[1], *reinterpret_cast<const uint4*>(row16), acc);
                acc = dot8_bf16(q4[2], q4[3], *reinterpret_cast<const uint4*>(row16 + 16), acc);
              } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int ch = ((i + rot) & 3) * 4;
                  acc = dot4(*reinterpret_cast<const float4*>(qrow + ch),
                             *reinterpret_cast<const float4*>(row + ch), acc);
                }
              }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            const float sg = acc * p.gate_scale;
            S += sg;
            if (act && sub == 0 && p.head_scores != nullptr)
              p.head_scores[(static_cast<size_t>(s) * p.hq + h * G + g) * p.mg + b0 + bb] = sg;
          }
          S = S / static_cast<float>(G);
        }
        if (act && sub == 0 && p.group_scores != nullptr)
          p.group_scores[static_cast<size_t>(pair) * p.mg + b0 + bb] = S;
      }
      if (ci == 0) SAS_TRACE(30);  // first chunk scored (thread 0)
      // chunks that all fit the ring (requested up front) need no slot
      // recycling: one barrier after the last
      if (nchunks > NST || ci == nchunks - 1) {
        __syncthreads();
        if (ci == 0) SAS_TRACE(31);
        pump(ci + 1, known);
      }
    }
  }
  SAS_TRACE(3);
  if (MODE == kModeGate) return;  // everything sent to this CTA (v) has arrived

  // ------------------------------------------------------------ phase 2: Top-K
  if (MODE == kModeFused) {
    SAS_TRACE(4);
    auto issue_wk = [&]() {
      // this CTA's 16 columns of W_k[h] (384 rows as three 128-row boxes);
      // they land over the key region, unused from here on
      if (do_pool && tid == 0) {
        fence_proxy_async_smem();  // the key region's generic accesses before the async-proxy overwrite
        mbar_arrive_expect_tx(bar_wk, kPool * kDpc * 2);
        for (int part = 0; part < 3; ++part)
          tma_load_2d(wk_s + part * 128 * kDpc, &tmwk, rank * kDpc, h * kPool + part * 128, bar_wk);
      }
    };
    bool list_ok = true;
    if (bad) {
      if (rank == 0 && tid == 0 && p.sel_count != nullptr) p.sel_count[pair] = 0;
    } else if (sel_local) {
      // every historical block kept (or none): the list needs no scores.  A
      // token from every CTA still marks the end of its scores, so that no
      // CTA's merge partials reach another's inbox (over its gate query)
      // while that CTA is still scoring.
      if (tid < CS) st_async_u32(dsmem_addr(scan + rank, tid), 1u, dsmem_addr(bar_sc, tid));
      list_ok = mbar_wait_cluster(bar_sc, 0, p.status);
      const int kept = m - 1;
      for (int j = tid; j < kept; j += kThreads) sel[j] = j;
      if (tid == 0) sel[kept] = c;
      __syncthreads();
      if (rank == 0) {
        for (int j = tid; j < m; j += kThreads)
          if (p.sel_idx != nullptr) p.sel_idx[static_cast<size_t>(pair) * p.max_sel + j] = sel[j];
        if (p.sel_count != nullptr && tid == 0) p.sel_count[pair] = m;
      }
      issue_wk();
    } else if (sel_fast) {
      // Distributed exact Top-K.  (1) each CTA ranks its own (score, block)
      // keys by counting (keys are distinct: the block index breaks ties) and
      // sends its best min(topk, rows) in descending order to every CTA;
      // (2) every CTA merges the sorted lists (bitonic merge tree) and keeps
      // the topk best; (3) their block ids, sorted, give the ascending list.
      // The global best topk always lie in the union: each is among its own
      // CTA's best topk.
      int plen[CS + 1];  // kept candidates of every CTA, then this CTA's row count
#pragma unroll
      for (int r = 0; r < CS; ++r) plen[r] = min(topk, rows_of(r));
      plen[CS] = rows_of(rank);
      SAS_TRACE(10);  // scores of this CTA done
#ifdef SAS_PHASE_TRACE
      unsigned long long* ttr = (p.trace != nullptr && blockIdx.y * gridDim.x + blockIdx.x < kTraceCtas)
                                    ? p.trace + (blockIdx.y * gridDim.x + blockIdx.x) * kTraceSlots + 11
                                    : nullptr;
#else
      unsigned long long* ttr = nullptr;
#endif
      list_ok = (topk <= 32)
                    ? distributed_topk<CS, 1>(lkeys, gather, plen, topk, c, rank, sel, bar_sc, p.status, ttr)
                    : distributed_topk<CS, 2>(lkeys, gather, plen, topk, c, rank, sel, bar_sc, p.status, ttr);
      __syncthreads();
      SAS_TRACE(18);
      if (rank == 0) {
        if (p.sel_idx != nullptr)
          for (int j = tid; j < m; j += kThreads) p.sel_idx[static_cast<size_t>(pair) * p.max_sel + j] = sel[j];
        if (p.sel_count != nullptr && tid == 0) p.sel_count[pair] = list_ok ? m : 0;
      }
      issue_wk();
    } else {
      // Rank 0 selects once for the cluster: it waits for every score, ranks
      // them and sends the block list to every other CTA the same way.
      if (rank == 0) {
        list_ok = mbar_wait_cluster(bar_sc, 0, p.status);
        SAS_TRACE(9);  // rank 0: every score of the cluster is in
#ifdef SAS_PHASE_TRACE
        unsigned long long* tr = (p.trace != nullptr && blockIdx.y * gridDim.x + blockIdx.x < kTraceCtas)
                                     ? p.trace + (blockIdx.y * gridDim.x + blockIdx.x) * kTraceSlots + 10
                                     : nullptr;
#else
        unsigned long long* tr = nullptr;
#endif
        list_ok = __syncthreads_and(list_ok) != 0;
        if (list_ok) {
          select_blocks(keys, n, topk, c, sel, hist, selbits, scan, tr);
        } else {  // scores missing (timeout, in the status word): a valid stand-in list
          for (int j = tid; j < m; j += kThreads) sel[j] = c;
          __syncthreads();
        }
        SAS_TRACE(18);  // rank 0: list ready
        for (int j = tid; j < m; j += kThreads) {
          const int b = sel[j];
          for (int r = 1; r < CS; ++r)
            st_async_u32(dsmem_addr(sel + j, r), static_cast<uint32_t>(b), dsmem_addr(bar_sel, r));
          if (p.sel_idx != nullptr) p.sel_idx[static_cast<size_t>(pair) * p.max_sel + j] = b;
        }
        if (p.sel_count != nullptr && tid == 0) p.sel_count[pair] = list_ok ? m : 0;
        SAS_TRACE(19);  // rank 0: list sent
        issue_wk();
      } else {
        issue_wk();
        list_ok = mbar_wait_cluster(bar_sel, 0, p.status);
      }
    }
    // a list that never came (timeout, already in the status word) is not
    // read: the current block, always valid, stands in for every entry
    if (__syncthreads_and(list_ok) == 0) {
      for (int j = tid; j < m; j += kThreads) sel[j] = c;
      __syncthreads();
    }
    known = nchunks + kTilesPerBlock * cnt_mine;
    SAS_TRACE(20);  // list in hand
    // the cache rows of this CTA's entries, looked up in parallel (paged:
    // one page-table read each), so that issuing a tile reads one word
    for (int e = tid; e < cnt_mine; e += kThreads) rows_s[e] = p.kv.block_row(s, h, entry_block(e));
    __syncthreads();
    rows_cached = true;
    pump(nchunks, known, true);
    if (gated && !bad) {
      // gated mode: each CTA computes the gates of its own list entries,
      // log(sigmoid(s_gb)), s_gb = (q~_g . k~_b) * gate_scale, while its K/V
      // copies are in flight; q~ (v, rotated in place) is still intact (the
      // gated plan keeps every later region clear of it).  The current block
      // (and a stand-in list, all entries the current block) gets 0.  As in
      // the score phase: 8 lanes per key row (16 dimensions each), 4 rows per
      // warp; one 8-lane reduction per (row, head).
      const int grp = lane >> 3, sub = lane & 7;
      for (int e0 = 0; e0 < cnt_mine; e0 += 4 * kWarps) {
        const int e = e0 + 4 * warp + grp;
        const bool live = e < cnt_mine;
        const int b = live ? entry_block(e) : c;
        uint4 kr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) kr[i] = make_uint4(0u, 0u, 0u, 0u);
        if (b != c) {
          const uint8_t* krow = gk_pair + static_cast<size_t>(b) * gk_row_bytes;
          if (p.gk16) {
            kr[0] = *reinterpret_cast<const uint4*>(krow + 32 * sub);
            kr[1] = *reinterpret_cast<const uint4*>(krow + 32 * sub + 16);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) kr[i] = *reinterpret_cast<const uint4*>(krow + 64 * sub + 16 * i);
          }
        }
        const int jg = live ? entry_index(e) * G : 0;
        for (int g = 0; g < G; ++g) {
          const float4* q4 = reinterpret_cast<const float4*>(qv + g * kDim + 16 * sub);
          float a = 0.f;
          if (p.gk16) {
            a = dot8_bf16(q4[0], q4[1], kr[0], a);
            a = dot8_bf16(q4[2], q4[3], kr[1], a);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 k = kr[i];
              a = dot4(q4[i], make_float4(__uint_as_float(k.x), __uint_as_float(k.y),
                                          __uint_as_float(k.z), __uint_as_float(k.w)), a);
            }
          }
          a += __shfl_xor_sync(0xffffffffu, a, 1);
          a += __shfl_xor_sync(0xffffffffu, a, 2);
          a += __shfl_xor_sync(0xffffffffu, a, 4);
          const float sg = a * p.gate_scale;
          if (sub == 0 && live)
            gbias[jg + g] = (b == c) ? 0.f : ((sg >= 0.f) ? -log1pf(expf(-sg)) : sg - log1pf(expf(sg)));
        }
      }
      __syncthreads();
    }
    SAS_TRACE(5);
  }

  // ------------------------------------------------------------ phase 3: attention
  const int tq = lane & 3, gq = lane >> 2;
  float m_run = -INFINITY, l_run = 0.f;  // bf16 path: head gq of this warp
  float o_acc[16][2];                      // bf16 path: O[gq][8nt + 2tq + e]
  float fm[kMaxGroup], fl[kMaxGroup], fo[kMaxGroup][4];  // fp32 path
  // bf16 path: this lane's q fragments (head gq, columns 16ks + 2tq (+8)) are
  // read from shared memory at each K tile rather than held in registers
  const uint32_t* qfrag = reinterpret_cast<const uint32_t*>(
      reinterpret_cast<const __nv_bfloat16*>(qraw) + min(gq, G - 1) * kDim + 2 * tq);
  const bool qlive = gq < G;
  if constexpr (!kF32) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o_acc[nt][0] = o_acc[nt][1] = 0.f;
  } else {
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
      fm[g] = -INFINITY;
      fl[g] = 0.f;
      fo[g][0] = fo[g][1] = fo[g][2] = fo[g][3] = 0.f;
    }
  }
  const float sl2 = p.attn_scale_log2;

  if (do_pool && own_cur) {
    // key-block pooling (max, min, mean over the 64 tokens) of the current
    // block, straight from its K tile (list entry 0 of this CTA, already
    // requested), sent to every CTA of the cluster
    const int t0 = nchunks;
    float mx = -INFINITY, mn = INFINITY, sm = 0.f;
    const int d = tid;
    if constexpr (!kF32) {
      const bool ok = mbar_wait(&bars[t0 % NST], (t0 / NST) & 1, p.status);
      const uint8_t* kt = slots + (t0 % NST) * kTileBytes;
      const int jc = d >> 3, el = d & 7;
      if (ok) {
#pragma unroll 8
        for (int t = 0; t < kBlock; ++t) {
          const float x = __bfloat162float(
              *reinterpret_cast<const __nv_bfloat16*>(kt + swz_tile_offset(t, jc) + el * 2));
          mx = fmaxf(mx, x);
          mn = fminf(mn, x);
          sm += x;
        }
      }
    } else {
      bool ok = mbar_wait(&bars[t0 % NST], (t0 / NST) & 1, p.status);
      ok = mbar_wait(&bars[(t0 + 1) % NST], ((t0 + 1) / NST) & 1, p.status) && ok;
      const float* k0 = reinterpret_cast<const float*>(slots + (t0 % NST) * kTileBytes);
      const float* k1 = reinterpret_cast<const float*>(slots + ((t0 + 1) % NST) * kTileBytes);
      if (ok) {
        for (int t = 0; t < kBlock; ++t) {
          const float x = (t < 32 ? k0 : k1)[(t & 31) * kDim + d];
          mx = fmaxf(mx, x);
          mn = fminf(mn, x);
          sm += x;
        }
      }
    }
    sm *= (1.f / kBlock);
#pragma unroll
    for (int r = 0; r < CS; ++r) {
      const uint32_t rb = dsmem_addr(bar_p, r);
      st_async_f32(dsmem_addr(pool_p + d, r), mx, rb);
      st_async_f32(dsmem_addr(pool_p + kDim + d, r), mn, rb);
      st_async_f32(dsmem_addr(pool_p + 2 * kDim + d, r), sm, rb);
    }
  }

  // u = P @ W_k[h] for this CTA's 16 columns; slices and their sums of
  // squares go to CTA 0, which normalises and rotates once all have come.
  // Run inside the attention loop (after the CTA's second list entry), where
  // the warps mostly wait on tiles; qbar (dead since the scores) is scratch.
  bool pooled_done = false;
  auto project_pooled = [&]() {
    // u = P @ W_k[h] for this CTA's 16 columns; slices and their sums of
    // squares go to CTA 0, which normalises and rotates once all have come
    const bool okp = mbar_wait_cluster(bar_p, 0, p.status);  // the pooled block
    const bool okw = mbar_wait(bar_wk, 0, p.status);
    const int j = tid & (kDpc - 1);
    const int rg = tid / kDpc;  // kThreads / kDpc row groups
    constexpr int kRowsPer = kPool / (kThreads / kDpc);
    float acc = 0.f;
    if (okp && okw) {
      float a2[2] = {0.f, 0.f};
#pragma unroll 16
      for (int r = 0; r < kRowsPer; ++r)
        a2[r & 1] = fmaf(pool_p[rg * kRowsPer + r], __bfloat162float(wk_s[(rg * kRowsPer + r) * kDpc + j]),
                         a2[r & 1]);
      acc = a2[0] + a2[1];
    }
    qbar[tid] = acc;  // qbar (dead since the scores) holds the row-group sums
    __syncthreads();
    if (tid < kDpc) {
      float u = 0.f;
      for (int g = 0; g < kThreads / kDpc; ++g) u += qbar[g * kDpc + tid];
      float sq = u * u;
#pragma unroll
      for (int o = kDpc / 2; o > 0; o >>= 1) sq += __shfl_xor_sync(0x0000ffffu, sq, o);
      const uint32_t rb = dsmem_addr(bar_u, 0);
      st_async_f32(dsmem_addr(pool_u + rank * 17 + tid, 0), u, rb);
      if (tid == 0) st_async_f32(dsmem_addr(pool_u + rank * 17 + 16, 0), sq, rb);
    }
    pooled_done = true;
  };

  for (int e = 0; e < cnt_mine; ++e) {
    const int b = entry_block(e);
    const int jg = entry_index(e) * G;  // gated mode: this entry's gates at gbias[jg + g]
    const int nvalid = (b == c) ? (L - b * kBlock) : kBlock;
    const int t0 = nchunks + e * kTilesPerBlock;
    if constexpr (!kF32) {
      // ---- K tile: S = q K^T for this warp's 16 tokens
      const int slotK = t0 % NST;
      bool ok = mbar_wait(&bars[slotK], (t0 / NST) & 1, p.status);
      float sacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      if (ok) {
        const uint32_t kbase = smem_u32(slots + slotK * kTileBytes);
        const int mat = lane >> 3;
        const int tok = 16 * warp + (mat >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kbase + swz_tile_offset(tok, 2 * ks + (mat & 1)), r0, r1, r2, r3);
          const uint32_t qa0 = qlive ? qfrag[8 * ks] : 0u;      // q[16ks + 2tq], [+1]
          const uint32_t qa2 = qlive ? qfrag[8 * ks + 4] : 0u;  // q[16ks + 8 + 2tq], [+1]
          mma_rows0_7(sacc[0][0], sacc[0][1], qa0, qa2, r0, r1);
          mma_rows0_7(sacc[1][0], sacc[1][1], qa0, qa2, r2, r3);
        }
      }
      __syncthreads();
      pump(t0 + 1, known);
      // ---- online softmax (per warp, head gq); gated mode: + the entry's
      // log-sigmoid gate, in log2 units like the scaled logits
      const float beta2 = (gated && gq < G) ? gbias[jg + gq] * kLog2e : 0.f;
      float x[2][2];
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int tl = 16 * warp + 8 * nt + 2 * tq + q;
          x[nt][q] = (tl < nvalid) ? fmaf(sacc[nt][q], sl2, beta2) : -INFINITY;
          mx = fmaxf(mx, x[nt][q]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(m_run, mx);
      const float alpha = (mnew == -INFINITY) ? 1.f : exp2f(m_run - mnew);
      float pr[2][2];
      float psum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          pr[nt][q] = (x[nt][q] == -INFINITY) ? 0.f : exp2f(x[nt][q] - mnew);
          psum += pr[nt][q];
        }
      l_run = l_run * alpha + psum;
      m_run = mnew;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        o_acc[nt][0] *= alpha;
        o_acc[nt][1] *= alpha;
      }
      const uint32_t pa0 = pack_bf16x2(pr[0][0], pr[0][1]);
      const uint32_t pa2 = pack_bf16x2(pr[1][0], pr[1][1]);
      // ---- V tile: O += P V
      const int t1 = t0 + 1;
      const int slotV = t1 % NST;
      ok = mbar_wait(&bars[slotV], (t1 / NST) & 1, p.status);
      if (ok) {
        uint8_t* vtile = slots + slotV * kTileBytes;
        if (nvalid < kBlock) {
          // rows past the context may hold anything (even NaN): zero this
          // warp's invalid rows so that P = 0 there gives exactly 0
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int idx = it * 32 + lane;
            const int row = 16 * warp + (idx >> 4);
            const int ch = idx & 15;
            if (row >= nvalid)
              *reinterpret_cast<uint4*>(vtile + (ch >> 3) * 8192 + row * 128 + (ch & 7) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();  // the slot is refilled by TMA later
          __syncwarp();
        }
        const uint32_t vbase = smem_u32(vtile);
        const int mat = lane >> 3;
        const int tok = 16 * warp + (mat & 1) * 8 + (lane & 7);
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4_trans(vbase + swz_tile_offset(tok, 2 * np + (mat >> 1)), r0, r1, r2, r3);
          mma_rows0_7(o_acc[2 * np][0], o_acc[2 * np][1], pa0, pa2, r0, r1);
          mma_rows0_7(o_acc[2 * np + 1][0], o_acc[2 * np + 1][1], pa0, pa2, r2, r3);
        }
      }
      __syncthreads();
      pump(t1 + 1, known);
    } else {
      // ---- fp32 K/V: SIMT path (small parity configurations)
      const float* qatt = reinterpret_cast<const float*>(qraw);
      const int half = warp >> 1;  // tokens 0..31 in tile t0 (t0+2 for V), 32..63 in t0+1
      const int tK = t0 + half;
      bool ok = mbar_wait(&bars[t0 % NST], (t0 / NST) & 1, p.status);
      ok = mbar_wait(&bars[(t0 + 1) % NST], ((t0 + 1) / NST) & 1, p.status) && ok;
      const int tt = lane >> 1, hh = lane & 1;
      const int tl = 16 * warp + tt;
      float lg[kMaxGroup];
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) lg[g] = 0.f;
      if (ok) {
        const float* krow = reinterpret_cast<const float*>(slots + (tK % NST) * kTileBytes) +
                            (tl & 31) * kDim + hh * 64;
        for (int i = 0; i < 64; ++i) {
          const int d = (i + tt) & 63;
          const float kv = krow[d];
#pragma unroll
          for (int g = 0; g < kMaxGroup; ++g)
            if (g < G) lg[g] = fmaf(qatt[g * kDim + hh * 64 + d], kv, lg[g]);
        }
      }
      __syncthreads();
      pump(t0 + 2, known);
      float pg[kMaxGroup];
#pragma unroll
      for (int g = 0; g < kMaxGroup; ++g) {
        float xv = lg[g] + __shfl_xor_sync(0xffffffffu, lg[g], 1);
        const float bg = (gated && g < G) ? gbias[jg + g] * kLog2e : 0.f;
        xv = (tl < nvalid) ? fmaf(xv, sl2, bg) : -INFINITY;
        float mx = xv;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mnew = fmaxf(fm[g], mx);
        const float alpha = (mnew == -INFINITY) ? 1.f : exp2f(fm[g] - mnew);
        pg[g] = (xv == -INFINITY) ? 0.f : exp2f(xv - mnew);
        float ps = pg[g];
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        fl[g] = fl[g] * alpha + ps;
        fm[g] = mnew;
#pragma unroll
        for (int k = 0; k < 4; ++k) fo[g][k] *= alpha;
      }
      const int t2 = t0 + 2;
      ok = mbar_wait(&bars[t2 % NST], (t2 / NST) & 1, p.status);
      ok = mbar_wait(&bars[(t2 + 1) % NST], ((t2 + 1) / NST) & 1, p.status) && ok;
      if (ok) {
        float* vt = reinterpret_cast<float*>(slots + ((t2 + half) % NST) * kTileBytes);
        if (nvalid < kBlock) {
          for (int it = 0; it < 16; ++it) {
            const int idx = it * 32 + lane;
            const int row = 16 * warp + (idx >> 5);
            if (row >= nvalid)
              *reinterpret_cast<float4*>(vt + (row & 31) * kDim + (idx & 31) * 4) =
                  make_float4(0.f, 0.f, 0.f, 0.f);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        for (int tk = 0; tk < 16; ++tk) {
          const float4 v4 =
              *reinterpret_cast<const float4*>(vt + ((16 * warp + tk) & 31) * kDim + 4 * lane);
#pragma unroll
          for (int g = 0; g < kMaxGroup; ++g) {
            const float pv = __shfl_sync(0xffffffffu, pg[g], 2 * tk);
            if (g < G) {
              fo[g][0] = fmaf(pv, v4.x, fo[g][0]);
              fo[g][1] = fmaf(pv, v4.y, fo[g][1]);
              fo[g][2] = fmaf(pv, v4.z, fo[g][2]);
              fo[g][3] = fmaf(pv, v4.w, fo[g][3]);
            }
          }
        }
      }
      __syncthreads();
      pump(t0 + 4, known);
    }
    if (do_pool && e == min(1, cnt_mine - 1)) project_pooled();
  }
  SAS_TRACE(6);

  // ------------------------------------------------------------ phase 4: merge
  // per-warp partials (the stage slots are free: every issued tile was consumed)
  if constexpr (!kF32) {
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
    if (gq < G) {
      if (tq == 0) {
        pm[warp * kMaxGroup + gq] = m_run;
        pl[warp * kMaxGroup + gq] = l_run;
      }
      float* dst = po + (static_cast<size_t>(warp) * G + gq) * kDim;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<float2*>(dst + 8 * nt + 2 * tq) = make_float2(o_acc[nt][0], o_acc[nt][1]);
    }
  } else {
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
      if (g < G) {
        if (lane == 0) {
          pm[warp * kMaxGroup + g] = fm[g];
          pl[warp * kMaxGroup + g] = fl[g];
        }
        *reinterpret_cast<float4*>(po + (static_cast<size_t>(warp) * G + g) * kDim + 4 * lane) =
            make_float4(fo[g][0], fo[g][1], fo[g][2], fo[g][3]);
      }
    }
  }
  __syncthreads();
  // fold the 4 warps; thread d owns column d of every head and sends it to
  // the CTA that writes that column
  {
    const int d = tid;
    const int dst = d / kDpc;
    const int dd = d - dst * kDpc;
    const uint32_t rb = dsmem_addr(bar_m, dst);
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, pm[w * kMaxGroup + g]);
      float lsum = 0.f, osum = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float f = exp2f(pm[w * kMaxGroup + g] - M);
          lsum = fmaf(pl[w * kMaxGroup + g], f, lsum);
          osum = fmaf(po[(static_cast<size_t>(w) * G + g) * kDim + d], f, osum);
        }
      }
      st_async_f32(dsmem_addr(inbox_o + (rank * G + g) * kDpc + dd, dst), osum, rb);
      if (dd == 0) {
        st_async_f32(dsmem_addr(inbox_ml + (rank * G + g) * 2 + 0, dst), M, rb);
        st_async_f32(dsmem_addr(inbox_ml + (rank * G + g) * 2 + 1, dst), lsum, rb);
      }
    }
  }
  if (do_pool && !pooled_done) project_pooled();
  if (do_pool && rank == 0) {
    // RMSNorm (gain gamma_k) and gate RoPE at position c of the pooled block
    mbar_wait_cluster(bar_u, 0, p.status);
    const int d = tid;
    float ss = 0.f;
#pragma unroll
    for (int r = 0; r < CS; ++r) ss += pool_u[r * 17 + 16];
    const float x = pool_u[(d / kDpc) * 17 + (d % kDpc)] * (1.f / sqrtf(ss / kDim + p.eps)) * gamk_s[d];
    qbar[d] = x;
    __syncthreads();
    float cs, sn;
    rope_cos_sin(p.rope.theta_over_pi[d & 63], c, cs, sn);
    const float y = (d < 64) ? qbar[d] * cs - qbar[d + 64] * sn : qbar[d] * cs + qbar[d - 64] * sn;
    const size_t gi = (static_cast<size_t>(pair) * p.mg + c) * kDim + d;
    if (p.gk16)
      static_cast<__nv_bfloat16*>(p.gate_keys_out)[gi] = __float2bfloat16_rn(y);
    else
      static_cast<float*>(p.gate_keys_out)[gi] = y;
  }
  mbar_wait_cluster(bar_m, 0, p.status);  // every partial of this CTA's columns
  __syncthreads();                         // qbar is reused below
  SAS_TRACE(7);
  {
    OutT* out = static_cast<OutT*>(p.out);
    for (int it = tid; it < G * kDpc; it += kThreads) {
      const int g = it / kDpc;
      const int dd = it - g * kDpc;
      float res = 0.f;
      if (!bad) {
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < CS; ++r) M = fmaxf(M, inbox_ml[(r * G + g) * 2]);
        float den = 0.f, num = 0.f;
#pragma unroll
        for (int r = 0; r < CS; ++r) {
          const float mr = inbox_ml[(r * G + g) * 2];
          if (mr != -INFINITY) {
            const float f = exp2f(mr - M);
            den = fmaf(inbox_ml[(r * G + g) * 2 + 1], f, den);
            num = fmaf(inbox_o[(r * G + g) * kDpc + dd], f, num);
          }
        }
        res = num / den;
      }
      out[(static_cast<size_t>(s) * p.hq + h * G + g) * kDim + rank * kDpc + dd] =
          from_float<OutT>(res);
    }
  }
  SAS_TRACE(8);
}

// ------------------------------------------------------------ Top-K kernel
template <bool kMedium>
__global__ void __launch_bounds__(kThreads) topk_kernel(const __grid_constant__ TopkParams p) {
  const int pair = blockIdx.x;
  const int s = pair / p.hkv;
  const int tid = threadIdx.x;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* vals = reinterpret_cast<float*>(smem_raw);
  uint8_t* q = smem_raw + (p.mg * 4 + 15) / 16 * 16;
  int* sel = reinterpret_cast<int*>(q);
  q += (p.max_sel * 4 + 15) / 16 * 16;
  uint32_t* hist = reinterpret_cast<uint32_t*>(q);
  q += kSelBins * 4;
  uint32_t* selbits = reinterpret_cast<uint32_t*>(q);
  q += ((p.mg + 31) / 32 * 4 + 15) / 16 * 16;
  int* scan = reinterpret_cast<int*>(q);
  const int L = p.seq_lens[s];
  int topk = p.topk;
  if (p.token_budgets != nullptr) {
    const int b = p.token_budgets[s];
    topk = (b >= kBlock && b <= (p.topk + 1) * kBlock && b % kBlock == 0) ? b / kBlock - 1 : -1;
  }
  if (L < 1 || (L - 1) / kBlock > p.mg || topk < 0) {
    if (tid == 0) {
      raise_status(p.status, kStatusBounds);
      p.sel_count[pair] = 0;
    }
    return;
  }
  const int c = (L - 1) / kBlock;
  for (int b = tid; b < c; b += kThreads) vals[b] = p.group_scores[static_cast<size_t>(pair) * p.mg + b];
  __syncthreads();
  const int m = select_blocks<kMedium>(vals, c, topk, c, sel, hist, selbits, scan);
  for (int j = tid; j < m; j += kThreads) p.sel_idx[static_cast<size_t>(pair) * p.max_sel + j] = sel[j];
  if (tid == 0) p.sel_count[pair] = m;
}

size_t topk_smem_bytes(int mg, int max_sel) {
  return static_cast<size_t>((mg * 4 + 15) / 16 * 16 + (max_sel * 4 + 15) / 16 * 16 + kSelBins * 4 +
                             ((mg + 31) / 32 * 4 + 15) / 16 * 16 + 16 * 4);
}

// ------------------------------------------------------------ launchers
namespace {

template <typename T, typename OutT, int CS, int NST, int MODE>
cudaError_t launch_cluster(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                           const CUtensorMap& tmw, const CUtensorMap& tmwk, int batch,
                           cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, static_cast<unsigned>(batch * p.hkv), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.sm.total);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the CTAs may start while the kernel ahead
  // on the stream drains; the kernel waits for it before reading its inputs
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_cluster_kernel<T, OutT, CS, NST, MODE>, p, tmk, tmv, tmw,
                            tmwk);
}

template <typename T, typename OutT, int CS, int NST, int MODE>
cudaError_t set_attrs() {
  auto k = decode_cluster_kernel<T, OutT, CS, NST, MODE>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  if (CS > 8) e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int MODE>
cudaError_t dispatch_types(bool f32_kv, bool f32_out, int cs, int nst, const DecodeParams& p,
                           const CUtensorMap& tmk, const CUtensorMap& tmv, const CUtensorMap& tmw,
                           const CUtensorMap& tmwk, int batch, cudaStream_t st) {
  using bf = __nv_bfloat16;
  if (cs != 8 || nst != 2) return cudaErrorInvalidValue;
  if (!f32_kv && !f32_out) return launch_cluster<bf, bf, 8, 2, MODE>(p, tmk, tmv, tmw, tmwk, batch, st);
  if (!f32_kv && f32_out) return launch_cluster<bf, float, 8, 2, MODE>(p, tmk, tmv, tmw, tmwk, batch, st);
  if (f32_kv && !f32_out) return launch_cluster<float, bf, 8, 2, MODE>(p, tmk, tmv, tmw, tmwk, batch, st);
  return launch_cluster<float, float, 8, 2, MODE>(p, tmk, tmv, tmw, tmwk, batch, st);
}

template <int MODE>
cudaError_t attrs_for_mode() {
  using bf = __nv_bfloat16;
  cudaError_t e;
  if ((e = set_attrs<bf, bf, 8, 2, MODE>()) != cudaSuccess) return e;
  if ((e = set_attrs<bf, float, 8, 2, MODE>()) != cudaSuccess) return e;
  if ((e = set_attrs<float, bf, 8, 2, MODE>()) != cudaSuccess) return e;
  return set_attrs<float, float, 8, 2, MODE>();
}

}  // namespace

cudaError_t launch_decode(int mode, bool f32_kv, bool f32_out, int cs, int nst,
                          const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                          const CUtensorMap& tmw, const CUtensorMap& tmwk, int batch,
                          cudaStream_t stream) {
  switch (mode) {
    case kModeGate:
      return dispatch_types<kModeGate>(f32_kv, false, cs, nst, p, tmk, tmv, tmw, tmwk, batch, stream);
    case kModeAttend:
      return dispatch_types<kModeAttend>(f32_kv, f32_out, cs, nst, p, tmk, tmv, tmw, tmwk, batch, stream);
    default:
      return dispatch_types<kModeFused>(f32_kv, f32_out, cs, nst, p, tmk, tmv, tmw, tmwk, batch, stream);
  }
}

cudaError_t launch_topk(const TopkParams& p, int batch, cudaStream_t stream) {
  const size_t smem = topk_smem_bytes(p.mg, p.max_sel);
  if (p.mg > 4 * kThreads)  // more than 512 historical blocks can occur
    topk_kernel<true><<<static_cast<unsigned>(batch * p.hkv), kThreads, smem, stream>>>(p);
  else
    topk_kernel<false><<<static_cast<unsigned>(batch * p.hkv), kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t prepare_decode_kernels() {
  cudaError_t e;
  if ((e = attrs_for_mode<kModeGate>()) != cudaSuccess) return e;
  if ((e = attrs_for_mode<kModeAttend>()) != cudaSuccess) return e;
  if ((e = attrs_for_mode<kModeFused>()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024)) !=
      cudaSuccess)
    return e;
  return cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
}

}  // namespace sas
