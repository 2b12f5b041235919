// Exact per-query top-k over the indexer's candidate lists (sm_100a).
//
// Token selection of the DeepSeek Sparse Attention page (kwkr.cn/news/60693,
// section 3.3): query t keeps min(top_k, t+1) keys ranked by (score desc,
// key index asc).  The indexer stores each candidate as the 64-bit word
// (raw accumulator bits << 32) | (0xFFFFFFFF - s), in kCandParts lists per
// row (one per column part of its tile), each in ascending key order.
//
// select_kernel: one CTA per row.  The lists are merged into one
// ascending-key run of sort keys: relu(acc) when that orders exactly like
// the score relu(fp32(acc) * scale) (checked per row), else the score word
// (non-negative, so its bits order like the value).  Stable LSD radix passes
// over the span of key bits that differ within the row (digits of up to 9
// bits) then order the run by key, descending; equal keys keep ascending key
// index, so the first min(top_k, t+1) entries are the answer.  Rows whose
// lists overflowed, or hold fewer keys than needed, go to the fallback.
//
// Fallback: fb_score_kernel recomputes every causal score of up to one
// queued row per SM on CUDA cores (FP32, exact for integer-valued inputs)
// over the whole grid and bins the scores; fb_select_kernel keeps the keys
// from the bin of the k-th score up and sorts them like select_kernel.
// fallback_kernel (one CTA per row) takes the rest: it builds the 64-bit keys
// (score_bits << 32) | (0xFFFFFFFF - s) -- larger key, better rank -- and
// selects by MSD radix passes plus a bitonic sort of the winners.
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "sort.cuh"

namespace dsa {

namespace {

constexpr int kSelThreads = 256;
constexpr int kFbBins = 4096;   // fallback histogram: bits 19..30 of a non-negative score word
constexpr int kFbChunk = 4096;  // keys per scoring work item
constexpr uint32_t kZeroModeTauBits = 1u;  // tau of a row whose threshold is "score > 0"

__device__ __forceinline__ void block_find_from_top(const unsigned int* hist, int R, int* out) {
  // Warp 0 scans the 256 bins from the top; out[0] = bin, out[1] = rank in bin.
  const int lane = threadIdx.x & 31;
  unsigned int local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) local += hist[255 - 8 * lane - i];
  unsigned int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned int ballot = __ballot_sync(0xFFFFFFFFu, incl >= static_cast<unsigned int>(R));
  const int src = __ffs(ballot) - 1;
  if (lane == src) {
    unsigned int run = incl - local;
    for (int i = 0; i < 8; ++i) {
      const int bb = 255 - 8 * lane - i;
      if (run + hist[bb] >= static_cast<unsigned int>(R)) {
        out[0] = bb;
        out[1] = R - static_cast<int>(run);
        break;
      }
      run += hist[bb];
    }
  }
}

// The R-th largest (1-based) of n distinct 64-bit keys.  Keys may live in
// shared or global memory; every thread of the block must call.
template <typename KeyPtr>
__device__ unsigned long long block_radix_select(KeyPtr keys, int n, int R, unsigned int* hist,
                                                 int* shared2) {
  unsigned long long prefix = 0, mask = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned long long k = keys[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) block_find_from_top(hist, R, shared2);
    __syncthreads();
    const int b = shared2[0];
    R = shared2[1];
    prefix |= static_cast<unsigned long long>(b) << shift;
    mask |= 0xFFull << shift;
    __syncthreads();
  }
  return prefix;
}

// Sort P (a power of two) keys descending in shared memory.
__device__ void block_bitonic_desc(unsigned long long* a, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < P / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const unsigned long long x = a[lo], y = a[hi];
        if ((x < y) == desc) {
          a[lo] = y;
          a[hi] = x;
        }
      }
    }
  }
  __syncthreads();
}

__device__ __forceinline__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Given the keys of one row (n of them, m <= n to keep), write indices[0..k).
template <typename KeyPtr>
__device__ void finish_row(KeyPtr keys, int n, int m, int top_k, int32_t* out,
                           unsigned long long* sel, unsigned int* hist, int* shared2) {
  const unsigned long long kth = (n > m) ? block_radix_select(keys, n, m, hist, shared2) : 0ull;
  if (threadIdx.x == 0) shared2[2] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long k = keys[i];
    if (k >= kth) {
      const int pos = atomicAdd(&shared2[2], 1);
      if (pos < m) sel[pos] = k;
    }
  }
  const int P = next_pow2(max(m, 2));
  __syncthreads();
  for (int i = m + threadIdx.x; i < P; i += blockDim.x) sel[i] = 0ull;
  block_bitonic_desc(sel, P);
  for (int i = threadIdx.x; i < top_k; i += blockDim.x)
    out[i] = i < m ? static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(sel[i])) : -1;
  __syncthreads();
}

// ---- sort-based select of one row ----------------------------------------------------
//
// The filter writes each row's candidates as kCandParts lists (one per
// column part of the indexer tile), each already in ascending key order.
// The select merges them into one ascending-index run (pairwise merge
// paths: lists 0+1 and 2+3 side by side, then the two results), then sorts
// it by key with
// stable LSD counting passes (descending digit), so equal keys keep
// ascending index: the result is the (score desc, index asc) order, and the
// first m entries are the answer.  Only the span of key bits that differ
// within the row is sorted, in digits of up to 9 bits (integer-valued inputs
// need one pass).  Ranks inside a warp come from __match_any_sync, so the
// passes use no atomics.

// Two block shapes: most rows (up to 3584 candidates) take 256 threads with
// three CTAs per SM; rows with more (up to 5632) are queued for a second
// launch with 512 threads and two CTAs per SM, which the grid-wide fallback's
// select also uses.  At 32K rows of 1434 candidates the small shape ran the
// select in 0.69 ms against 0.93 ms for the large one alone.
template <int WARPS, int SLOTS>
struct SelCfg {
  static constexpr int kWarps = WARPS;
  static constexpr int kSlots = SLOTS;                   // items per lane per radix pass
  static constexpr int kThreads = WARPS * 32;
  static constexpr int kCap = WARPS * 32 * SLOTS;        // keys per row
  static constexpr size_t kSmem =
      static_cast<size_t>(kCap) * (8 + 4 + 4) + (WARPS * 256 + 512 + WARPS + 8) * 4;
};
using SelSmall = SelCfg<8, 14>;    // 3584 keys
using SelBig = SelCfg<16, 11>;     // 5632 keys
constexpr int kSortCap = SelBig::kCap;

__device__ __forceinline__ uint32_t key_index(unsigned long long k) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(k);
}

// Row statistics of the sort keys: minimum, maximum, OR of all keys, number
// of non-zero keys.  Per-thread partials are combined with warp reductions
// and shared-memory atomics into misc[0..3], which thread 0 set to
// (~0, 0, 0, 0) before a barrier; every thread calls, then a barrier.
struct KeyStats {
  uint32_t kmin, kmax, kor;
  int npos;
};

__device__ __forceinline__ void stats_add(uint32_t w, uint32_t& lo, uint32_t& hi, uint32_t& orr,
                                          uint32_t& pos) {
  lo = min(lo, w);
  hi = max(hi, w);
  orr |= w;
  pos += w != 0u;
}

__device__ __forceinline__ void stats_init(uint32_t* misc) {
  misc[0] = 0xFFFFFFFFu;
  misc[1] = 0u;
  misc[2] = 0u;
  misc[3] = 0u;
}

__device__ __forceinline__ void stats_reduce(uint32_t lo, uint32_t hi, uint32_t orr, uint32_t pos,
                                             uint32_t* misc) {
  lo = __reduce_min_sync(0xFFFFFFFFu, lo);
  hi = __reduce_max_sync(0xFFFFFFFFu, hi);
  orr = __reduce_or_sync(0xFFFFFFFFu, orr);
  pos = __reduce_add_sync(0xFFFFFFFFu, pos);
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&misc[0], lo);
    atomicMax(&misc[1], hi);
    atomicOr(&misc[2], orr);
    atomicAdd(&misc[3], pos);
  }
}

__device__ __forceinline__ KeyStats stats_read(const uint32_t* misc) {
  return KeyStats{misc[0], misc[1], misc[2], static_cast<int>(misc[3])};
}

// Merge two ascending-index runs of 64-bit candidate keys a[0, na) and
// b[0, nb) into out[0, na + nb), threads tid < nthr of the block taking equal
// slices of the output (merge path: each finds its split by binary search).
__device__ void merge_keys_by_index(const unsigned long long* a, int na, const unsigned long long* b,
                                    int nb, unsigned long long* out, int tid, int nthr) {
  const int n = na + nb;
  const int per = (n + nthr - 1) / nthr;
  const int p0 = min(n, tid * per), p1 = min(n, p0 + per);
  if (p0 >= p1) return;
  int lo = max(0, p0 - nb), hi = min(p0, na);
  while (lo < hi) {  // smallest i such that a[i] does not precede b[p0 - i - 1]
    const int i = (lo + hi) >> 1;
    if (key_index(a[i]) < key_index(b[p0 - i - 1]))
      lo = i + 1;
    else
      hi = i;
  }
  int i = lo, j = p0 - lo;
  for (int p = p0; p < p1; ++p) {
    const bool take_a = j >= nb || (i < na && key_index(a[i]) < key_index(b[j]));
    out[p] = take_a ? a[i++] : b[j++];
  }
}

// Merge two ascending-index runs a[0, na) and b[0, nb) (64-bit candidate
// keys) into one ascending-index run, written as relu(accumulator) words `sc`
// and key indices `ix` (merge path: each thread finds its split by binary
// search); the thread's partial key statistics and, over the positive keys,
// largest exponent field and lowest set bit are accumulated on the way.
__device__ void merge_by_index(const unsigned long long* a, int na, const unsigned long long* b,
                               int nb, uint32_t* sc, uint32_t* ix, uint32_t& klo, uint32_t& khi,
                               uint32_t& orr, uint32_t& pos, uint32_t& emax, uint32_t& pmin) {
  const int n = na + nb;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int p0 = min(n, static_cast<int>(threadIdx.x) * per), p1 = min(n, p0 + per);
  if (p0 >= p1) return;
  int lo = max(0, p0 - nb), hi = min(p0, na);
  while (lo < hi) {  // smallest i such that a[i] does not precede b[p0 - i - 1]
    const int i = (lo + hi) >> 1;
    if (key_index(a[i]) < key_index(b[p0 - i - 1]))
      lo = i + 1;
    else
      hi = i;
  }
  int i = lo, j = p0 - lo;
  for (int p = p0; p < p1; ++p) {
    const bool take_a = j >= nb || (i < na && key_index(a[i]) < key_index(b[j]));
    const unsigned long long k = take_a ? a[i++] : b[j++];
    // the filter stored the raw accumulator; the sort key starts as relu(acc)
    const uint32_t acc = static_cast<uint32_t>(k >> 32);
    const uint32_t w = __uint_as_float(acc) > 0.0f ? acc : 0u;
    sc[p] = w;
    ix[p] = key_index(k);
    stats_add(w, klo, khi, orr, pos);
    if (w) {  // exponent field and lowest set bit (exponent of 2, biased by 150)
      const uint32_t e = w >> 23;
      const uint32_t mant = (w & 0x7FFFFFu) | (e ? 0x800000u : 0u);
      emax = max(emax, e);
      pmin = min(pmin, e ? e + static_cast<uint32_t>(__ffs(static_cast<int>(mant)) - 1) : 0u);
    }
  }
}

struct SelParams {
  int64_t L;       // query rows
  int64_t q0;      // query row t sits at key position q0 + t
  int top_k, cap;
  float scale;
  const unsigned long long* cand;
  const int* cand_n;
  const float* tau;
  int32_t* indices;
  int* fb_rows;
  int* counters;          // [0] fallback rows, [1] overflow rows, [2] candidates, [4] big rows
  int force_fb_period;
  int* big_rows;          // rows queued for the large block shape
};

// Two regions of 8 * kSortCap bytes.  Region 1 first holds the candidate
// lists as loaded (raw), then the merged score words sc0 and key indices ix;
// region 2 holds the first-level merges (tmp), then the sort's scratch sc1,
// ps0, ps1.  With two lists they are loaded into region 2 and merged once.
struct SelSmem {
  unsigned long long* raw;  // region 1: [kSortCap] candidate keys
  unsigned long long* tmp;  // region 2: [kSortCap] keys of the first-level merges
  uint32_t* sc1;            // region 2 after the merge: sc1 [kSortCap], ps0, ps1 [kSortCap]
  uint16_t* ps0;
  uint16_t* ps1;
  uint32_t* sc0;            // region 1 after the merge: [kSortCap] score words
  uint32_t* ix;             //   and [kSortCap] key indices
  uint32_t* cnt;            // [warps][256] words: 16-bit radix counters [warps][512] / bitmap
  uint32_t* base;           // [512 + warps]
  uint32_t* misc;           // [8]
};
template <class Cfg>
__device__ __forceinline__ SelSmem carve_sel_smem(unsigned long long* smem) {
  constexpr int cap = Cfg::kCap;
  SelSmem sm;
  sm.raw = smem;
  sm.tmp = smem + cap;
  sm.sc0 = reinterpret_cast<uint32_t*>(sm.raw);
  sm.ix = sm.sc0 + cap;
  sm.sc1 = reinterpret_cast<uint32_t*>(sm.tmp);
  sm.ps0 = reinterpret_cast<uint16_t*>(sm.sc1 + cap);
  sm.ps1 = sm.ps0 + cap;
  sm.cnt = reinterpret_cast<uint32_t*>(smem + 2 * cap);
  sm.base = sm.cnt + Cfg::kWarps * 256;
  sm.misc = sm.base + 512 + Cfg::kWarps;
  return sm;
}

// The n kept candidates of row t (score words sc0 and key indices ix, in
// ascending index order; n <= kSortCap) are sorted by score, descending and
// stable, and the first m key indices are written to out, padded with -1 up
// to top_k.  zero_mode: every positive score of the row is among the
// candidates and the zeros are ranked by index.  Every thread calls.
template <class Cfg>
__device__ void sort_emit(const SelSmem& sm, int n, int m, bool zero_mode, int64_t t, int top_k,
                          int32_t* out, const KeyStats& st) {
  uint32_t* sc0 = sm.sc0;
  uint32_t* sc1 = sm.sc1;
  uint16_t* ps0 = sm.ps0;
  uint16_t* ps1 = sm.ps1;
  uint32_t* ix = sm.ix;
  uint32_t* cnt = sm.cnt;
  uint32_t* base = sm.base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Keys of non-negative floats order like the values; the passes sort
  // key - minimum over the bits where the keys can differ: from the lowest
  // bit any key sets (all keys are multiples of it) to the top bit of the
  // range.
  const int npos = st.npos;
  int lo = 0, hi = -1;
  if (st.kmax > st.kmin) {
    lo = __ffs(static_cast<int>(st.kor)) - 1;
    hi = 31 - __clz(static_cast<int>(st.kmax - st.kmin));
  }
  uint32_t* ks = sc0;
  uint16_t* ps = nullptr;
  stable_sort32_by_score<Cfg::kWarps, Cfg::kSlots>(&ks, &ps, sc1, ps1, ps0, n, st.kmin, lo, hi,
                                                    reinterpret_cast<uint16_t*>(cnt), base);
    if (!zero_mode || npos >= m) {
      for (int i = threadIdx.x; i < top_k; i += blockDim.x)
        out[i] = i < m ? static_cast<int32_t>(ix[ps ? ps[i] : i]) : -1;
    } else {
      // Every positive score is a candidate; the rest of the row ranks the
      // zero scores by ascending key index.  Within keys [0, R) there are at
      // least m - npos zeros.
      const int R = static_cast<int>(min64(t + 1, static_cast<int64_t>(m) + npos));
      const int words = (R + 31) / 32;
      uint32_t* bm = cnt;
      for (int wd = threadIdx.x; wd < words; wd += blockDim.x) bm[wd] = 0u;
      __syncthreads();
      for (int i = threadIdx.x; i < npos; i += blockDim.x) {
        const uint32_t sidx = ix[ps ? ps[i] : i];
        if (sidx < static_cast<uint32_t>(R)) atomicOr(&bm[sidx >> 5], 1u << (sidx & 31));
        out[i] = static_cast<int32_t>(sidx);
      }
      __syncthreads();
      uint32_t z = 0u;
      if (threadIdx.x < words) {
        const int wd = threadIdx.x;
        const uint32_t valid = (wd * 32 + 32 <= R) ? 0xFFFFFFFFu : ((1u << (R - wd * 32)) - 1u);
        z = __popc(~bm[wd] & valid);
      }
      if (threadIdx.x < 128) {
        uint32_t incl = z;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
          if (lane >= off) incl += y;
        }
        if (lane == 31) base[warp] = incl;
        __syncwarp();
        base[8 + threadIdx.x] = incl - z;  // exclusive within the warp
      }
      __syncthreads();
      if (threadIdx.x < words) {
        const int wd = threadIdx.x;
        uint32_t rank = base[8 + wd];
        for (int w2 = 0; w2 < warp; ++w2) rank += base[w2];
        const uint32_t valid = (wd * 32 + 32 <= R) ? 0xFFFFFFFFu : ((1u << (R - wd * 32)) - 1u);
        uint32_t zeros = ~bm[wd] & valid;
        while (zeros) {
          const int bit = __ffs(zeros) - 1;
          zeros &= zeros - 1u;
          if (rank < static_cast<uint32_t>(m - npos)) out[npos + rank] = wd * 32 + bit;
          ++rank;
        }
      }
      for (int i = m + threadIdx.x; i < top_k; i += blockDim.x) out[i] = -1;
    }
}

// BIG = false: every row; rows with more candidates than Cfg holds (but at
// most SelBig's) are queued in big_rows.  BIG = true: the queued rows.
template <class Cfg, bool BIG>
__global__ void __launch_bounds__(Cfg::kThreads, BIG ? 2 : 3) select_kernel(const SelParams p) {
  extern __shared__ unsigned long long sel_smem[];
  const SelSmem sm = carve_sel_smem<Cfg>(sel_smem);
  const int lane = threadIdx.x & 31;
  static_assert(kCandParts == 2 || kCandParts == 4, "two or four candidate lists per row");
  unsigned long long* lists = kCandParts == 4 ? sm.raw : sm.tmp;
  const int64_t nrows = BIG ? static_cast<int64_t>(*(volatile const int*)(p.counters + 4)) : p.L;
  for (int64_t w = blockIdx.x; w < nrows; w += gridDim.x) {
    const int64_t t = BIG ? p.big_rows[w] : w;
    const int64_t qpos = p.q0 + t;   // the query's key position: keys 0 .. qpos are causal
    const int m = static_cast<int>(min64(p.top_k, qpos + 1));
    int nl[kCandParts];
    int n = 0;
    bool overflow = false;
#pragma unroll
    for (int q = 0; q < kCandParts; ++q) {
      nl[q] = p.cand_n[kCandParts * t + q];
      overflow |= nl[q] > p.cap;
      n += nl[q];
    }
    overflow |= n > SelBig::kCap;
    const bool zero_mode = __float_as_uint(p.tau[t]) == kZeroModeTauBits;
    const bool forced = p.force_fb_period > 0 && t % p.force_fb_period == 0;
    if (!BIG && !overflow && n > Cfg::kCap && !forced) {   // a row for the large block shape
      if (threadIdx.x == 0) p.big_rows[atomicAdd(&p.counters[4], 1)] = static_cast<int>(t);
      continue;
    }
    if (overflow || forced || (!zero_mode && n < m)) {
      if (threadIdx.x == 0) {
        const int pos = atomicAdd(&p.counters[0], 1);
        p.fb_rows[pos] = static_cast<int>(t);
        if (overflow) atomicAdd(&p.counters[1], 1);
      }
      continue;
    }
    if (threadIdx.x == 0) atomicAdd(&p.counters[2], n);
    const unsigned long long* c0 = p.cand + kCandParts * t * static_cast<int64_t>(p.cap);
    // Every list in flight at once (8-byte asynchronous copies), one wait.
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      int q = 0, off = i;
#pragma unroll
      for (int r = 0; r + 1 < kCandParts; ++r)
        if (q == r && off >= nl[r]) {
          off -= nl[r];
          q = r + 1;
        }
      const unsigned long long* src = c0 + q * static_cast<int64_t>(p.cap) + off;
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(lists + i)), "l"(src)
                   : "memory");
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // First level (four lists): 0+1 and 2+3 into region 2, half the block each.
    int na = nl[0], nb = n - nl[0];
    if (kCandParts == 4) {
      const int half = blockDim.x / 2;
      na = nl[0] + nl[1];
      nb = n - na;
      if (threadIdx.x < half)
        merge_keys_by_index(lists, nl[0], lists + nl[0], nl[1], sm.tmp, threadIdx.x, half);
      else
        merge_keys_by_index(lists + na, nl[2], lists + na + nl[2], nl[kCandParts - 1], sm.tmp + na,
                            threadIdx.x - half, half);
      __syncthreads();
    }
    const unsigned long long* runs = kCandParts == 4 ? sm.tmp : lists;
    if (threadIdx.x == 0) {
      stats_init(sm.misc);
      sm.misc[4] = 0u;           // largest exponent field of a positive accumulator
      sm.misc[5] = 0xFFFFFFFFu;  // lowest set bit (exponent of 2) over them, biased by 150
    }
    __syncthreads();
    uint32_t lo = 0xFFFFFFFFu, hi = 0u, orr = 0u, pos = 0u, emax = 0u, pmin = 0xFFFFFFFFu;
    merge_by_index(runs, na, runs + na, nb, sm.sc0, sm.ix, lo, hi, orr, pos, emax, pmin);
    stats_reduce(lo, hi, orr, pos, sm.misc);
    emax = __reduce_max_sync(0xFFFFFFFFu, emax);
    pmin = __reduce_min_sync(0xFFFFFFFFu, pmin);
    if (lane == 0) {
      atomicMax(&sm.misc[4], emax);
      atomicMin(&sm.misc[5], pmin);
    }
    __syncthreads();
    // Ordering by relu(acc) is ordering by score = relu(fp32(acc) * scale), ties
    // included, when the scale is positive and no two distinct accumulators of
    // the row round to the same score: so when every positive accumulator is a
    // normal multiple of 4 ulps of the largest one (then the exact products
    // differ by 2 ulps of the larger score) and the smallest scores stay
    // normal.  Integer-valued index inputs give that.  Otherwise the keys
    // become the score words.
    KeyStats st = stats_read(sm.misc);
    const uint32_t em = sm.misc[4], pm = sm.misc[5];
    // every positive accumulator is a multiple of 2^(pm - 150) >= 4 ulps of
    // the largest (2^(em - 148)); the smallest score, >= 2^(pm - 150) * scale,
    // is normal, and the largest score is finite (no ties at +inf)
    const bool by_acc =
        p.scale > 0.0f &&
        (pm == 0xFFFFFFFFu ||
         (pm >= em + 2u && __fmul_rn(ldexpf(1.0f, static_cast<int>(pm) - 150), p.scale) >= 1.17549435e-38f &&
          __fmul_rn(__uint_as_float(st.kmax), p.scale) < INFINITY));
    if (!by_acc) {
      __syncthreads();  // everyone has read misc
      if (threadIdx.x == 0) stats_init(sm.misc);
      __syncthreads();
      lo = 0xFFFFFFFFu, hi = 0u, orr = 0u, pos = 0u;
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float sc = __fmul_rn(__uint_as_float(sm.sc0[i]), p.scale);
        const uint32_t w = sc > 0.0f ? __float_as_uint(sc) : 0u;
        sm.sc0[i] = w;
        stats_add(w, lo, hi, orr, pos);
      }
      stats_reduce(lo, hi, orr, pos, sm.misc);
      __syncthreads();
      st = stats_read(sm.misc);
    }
    sort_emit<Cfg>(sm, n, m, zero_mode, qpos, p.top_k, p.indices + t * p.top_k, st);
    __syncthreads();
  }
}

struct FbParams {
  int64_t L;                     // key rows (stride of the scratch rows)
  int64_t q0;                    // query row t sits at key position q0 + t
  int top_k;
  const void* q_idx;
  const void* k_idx;
  int esize, d;
  float scale;
  const int* fb_rows;
  int* counters;                 // [0] fallback rows, [3] rows left to the one-CTA path
  int32_t* indices;
  unsigned long long* scratch;   // [slots, L]: keys of fallback row f (f < slots) / of a CTA
  unsigned int* hist;            // [slots, kFbBins]
  int* slow;                     // [slots] fallback slots left to the one-CTA path
  int slots;
};

template <int ESIZE>
__device__ __forceinline__ void load_row_f32(const void* base, int64_t row, int d, float* out) {
  // Decodes one index row into float (FP8 E4M3 via the cuda_fp8 conversion).
  if (ESIZE == 1) {
    const __nv_fp8_storage_t* r = static_cast<const __nv_fp8_storage_t*>(base) + row * d;
    for (int j = threadIdx.x; j < d; j += blockDim.x)
      out[j] = __half2float(__half(__nv_cvt_fp8_to_halfraw(r[j], __NV_E4M3)));
  } else {
    const __nv_bfloat16* r = static_cast<const __nv_bfloat16*>(base) + row * d;
    for (int j = threadIdx.x; j < d; j += blockDim.x) out[j] = __bfloat162float(r[j]);
  }
}

// q . row in FP32 with one accumulator per 16-byte chunk of the row (eight
// independent FMA chains for 128 FP8 values); exact whenever the inputs and
// every partial sum are integers below 2^24.
template <int ESIZE>
__device__ __forceinline__ float dot_row(const float* q, const void* base, int64_t row, int d) {
  constexpr int kMaxChunks = DSA_MAX_INDEX_DIM * ESIZE / 16;
  float acc[kMaxChunks];
  const uint8_t* r = static_cast<const uint8_t*>(base) + row * d * ESIZE;
  const int chunks = d * ESIZE / 16;
#pragma unroll
  for (int u = 0; u < kMaxChunks; ++u) {
    acc[u] = 0.0f;
    if (u < chunks) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(r + u * 16));
      const uint32_t words[4] = {w.x, w.y, w.z, w.w};
      if (ESIZE == 1) {
        const float* qq = q + u * 16;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const __nv_fp8x2_storage_t pair =
                static_cast<__nv_fp8x2_storage_t>((words[k] >> (16 * h)) & 0xFFFFu);
            const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3)));
            acc[u] = fmaf(qq[4 * k + 2 * h], f.x, acc[u]);
            acc[u] = fmaf(qq[4 * k + 2 * h + 1], f.y, acc[u]);
          }
        }
      } else {
        const float* qq = q + u * 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&words[k]));
          acc[u] = fmaf(qq[2 * k], f.x, acc[u]);
          acc[u] = fmaf(qq[2 * k + 1], f.y, acc[u]);
        }
      }
    }
  }
#pragma unroll
  for (int w = 1; w < kMaxChunks; w <<= 1)
#pragma unroll
    for (int u = 0; u + w < kMaxChunks; u += 2 * w) acc[u] += acc[u + w];
  return acc[0];
}

// Scores of fallback rows f < slots, spread over the whole grid: work item
// (f, c) computes keys c * kFbChunk .. +kFbChunk of row fb_rows[f] as 64-bit
// keys (score word << 32 | ~s) into scratch[f] and adds them to the row's
// histogram of score bits 19..30.
template <int ESIZE>
__global__ void __launch_bounds__(kSelThreads) fb_score_kernel(const FbParams p) {
  __shared__ float qf[DSA_MAX_INDEX_DIM];
  __shared__ unsigned int h[kFbBins];
  const int lane = threadIdx.x & 31;
  const int nf = min(*(volatile const int*)p.counters, p.slots);
  const int cpr = static_cast<int>((p.L + kFbChunk - 1) / kFbChunk);
  const int64_t items = static_cast<int64_t>(nf) * cpr;
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const int f = static_cast<int>(item / cpr), c = static_cast<int>(item % cpr);
    const int64_t t = p.fb_rows[f];
    const int64_t pos = p.q0 + t;   // keys 0 .. pos are causal
    const int64_t s0 = static_cast<int64_t>(c) * kFbChunk;
    if (s0 > pos) continue;
    const int64_t s1 = min64(pos + 1, s0 + kFbChunk);
    load_row_f32<ESIZE>(p.q_idx, t, p.d, qf);
    for (int i = threadIdx.x; i < kFbBins; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    unsigned long long* out = p.scratch + static_cast<int64_t>(f) * p.L;
    for (int64_t s = s0 + threadIdx.x; s < s0 + kFbChunk; s += blockDim.x) {
      const bool ok = s < s1;
      uint32_t bits = 0u;
      if (ok) {
        const float sc = __fmul_rn(dot_row<ESIZE>(qf, p.k_idx, s, p.d), p.scale);
        bits = sc > 0.0f ? __float_as_uint(sc) : 0u;
        out[s] = (static_cast<unsigned long long>(bits) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(s));
      }
      // ReLU zeros are common: one add per warp for them
      const uint32_t zeros = __ballot_sync(0xFFFFFFFFu, ok && bits == 0u);
      if (lane == 0 && zeros) atomicAdd(&h[0], static_cast<unsigned int>(__popc(zeros)));
      if (ok && bits != 0u) atomicAdd(&h[bits >> 19], 1u);
    }
    __syncthreads();
    unsigned int* gh = p.hist + static_cast<int64_t>(f) * kFbBins;
    for (int i = threadIdx.x; i < kFbBins; i += blockDim.x)
      if (h[i]) atomicAdd(&gh[i], h[i]);
    __syncthreads();
  }
}

// Select of fallback rows f < slots from their scored keys: the histogram
// gives the bin b holding the m-th largest score; the keys in bins >= b are
// compacted in ascending index order into shared memory and go through the
// same sort as the candidates of the main select.  Rows whose keys in bins
// >= b do not fit (b = 0, where the ReLU zeros are) are left to the one-CTA
// path.
__global__ void __launch_bounds__(SelBig::kThreads, 1) fb_select_kernel(const FbParams p) {
  constexpr int kSortThreads = SelBig::kThreads, kSortWarps = SelBig::kWarps;
  extern __shared__ unsigned long long sel_smem[];
  const SelSmem sm = carve_sel_smem<SelBig>(sel_smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* wsum = sm.base;   // [kSortWarps] per-warp counts, then the scan
  uint32_t* misc = sm.misc;
  const int nf = min(*(volatile const int*)p.counters, p.slots);
  constexpr int kPer = kFbBins / kSortThreads;  // bins per thread
  static_assert(kPer * kSortThreads == kFbBins, "bins per thread");
  for (int f = blockIdx.x; f < nf; f += gridDim.x) {
    const int64_t t = p.fb_rows[f];
    const int n = static_cast<int>(p.q0 + t + 1);
    const int m = min(p.top_k, n);
    const unsigned int* gh = p.hist + static_cast<int64_t>(f) * kFbBins;
    // thread i owns bins kFbBins-1-kPer*i .. kFbBins-kPer*(i+1) (descending)
    unsigned int loc = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) loc += gh[kFbBins - 1 - kPer * threadIdx.x - q];
    unsigned int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    if (threadIdx.x == 0) misc[4] = 0xFFFFFFFFu;
    __syncthreads();
    unsigned int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    const unsigned int ex = before + incl - loc;  // count in bins above my range
    if (ex < static_cast<unsigned int>(m) && ex + loc >= static_cast<unsigned int>(m)) {
      unsigned int run = ex;
      for (int q = 0; q < kPer; ++q) {
        const int b = kFbBins - 1 - kPer * threadIdx.x - q;
        if (run + gh[b] >= static_cast<unsigned int>(m)) {
          misc[4] = static_cast<uint32_t>(b);
          misc[5] = run + gh[b];  // keys in bins >= b
          break;
        }
        run += gh[b];
      }
    }
    __syncthreads();
    const uint32_t b = misc[4];
    const uint32_t total = misc[5];
    __syncthreads();
    if (b == 0xFFFFFFFFu || b == 0u || total > static_cast<uint32_t>(kSortCap)) {
      if (threadIdx.x == 0) p.slow[atomicAdd(&p.counters[3], 1)] = f;
      continue;
    }
    // stable compaction of the keys in bins >= b, four consecutive keys per thread
    const unsigned long long* keys = p.scratch + static_cast<int64_t>(f) * p.L;
    uint32_t done = 0;
    uint32_t slo = 0xFFFFFFFFu, shi = 0u, sor = 0u, spos = 0u;
    if (threadIdx.x == 0) stats_init(misc);  // misc[0..3]; b and total are held in registers
    for (int s0 = 0; s0 < n; s0 += 4 * kSortThreads) {
      const int sb = s0 + 4 * threadIdx.x;
      unsigned long long k4[4];
      int c = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        k4[q] = sb + q < n ? keys[sb + q] : 0ull;
        c += (sb + q < n && static_cast<uint32_t>(k4[q] >> 51) >= b) ? 1 : 0;
      }
      int ic = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, ic, o);
        if (lane >= o) ic += y;
      }
      if (lane == 31) wsum[warp] = static_cast<uint32_t>(ic);
      __syncthreads();
      uint32_t pos = done;
      for (int w = 0; w < warp; ++w) pos += wsum[w];
      uint32_t all = 0;
      for (int w = 0; w < kSortWarps; ++w) all += wsum[w];
      pos += static_cast<uint32_t>(ic - c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (sb + q < n && static_cast<uint32_t>(k4[q] >> 51) >= b) {
          const uint32_t w = static_cast<uint32_t>(k4[q] >> 32);
          sm.sc0[pos] = w;
          sm.ix[pos] = static_cast<uint32_t>(sb + q);
          stats_add(w, slo, shi, sor, spos);
          ++pos;
        }
      }
      done += all;
      __syncthreads();
    }
    stats_reduce(slo, shi, sor, spos, misc);
    __syncthreads();
    sort_emit<SelBig>(sm, static_cast<int>(total), m, false, p.q0 + t, p.top_k, p.indices + t * p.top_k,
              stats_read(misc));
    __syncthreads();
  }
}

// One CTA per row, scores recomputed into the CTA's own scratch row: the
// fallback slots the shared-memory select left (p.slow) and the fallback
// rows beyond the slots.
template <int ESIZE>
__global__ void __launch_bounds__(kSelThreads) fallback_kernel(const FbParams p) {
  extern __shared__ unsigned long long fb_smem[];
  unsigned long long* sel = fb_smem;                                   // [pow2(top_k)]
  unsigned int* hist = reinterpret_cast<unsigned int*>(sel + next_pow2(max(p.top_k, 2)));
  int* shared2 = reinterpret_cast<int*>(hist + 256);
  float* qf = reinterpret_cast<float*>(shared2 + 4);                   // [d]
  unsigned long long* scratch = p.scratch + static_cast<int64_t>(blockIdx.x) * p.L;
  const int nfb = *(volatile const int*)p.counters;
  const int nslow = *(volatile const int*)(p.counters + 3);
  const int extra = max(0, nfb - p.slots);
  for (int w = blockIdx.x; w < nslow + extra; w += gridDim.x) {
    const int f = w < nslow ? p.slow[w] : p.slots + (w - nslow);
    const int64_t t = p.fb_rows[f];
    const int n = static_cast<int>(p.q0 + t + 1);
    const int m = min(p.top_k, n);
    load_row_f32<ESIZE>(p.q_idx, t, p.d, qf);
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += blockDim.x) {
      float sc = __fmul_rn(dot_row<ESIZE>(qf, p.k_idx, s, p.d), p.scale);
      sc = sc > 0.0f ? sc : 0.0f;
      scratch[s] = (static_cast<unsigned long long>(__float_as_uint(sc)) << 32) |
                   (0xFFFFFFFFu - static_cast<uint32_t>(s));
    }
    __syncthreads();
    finish_row(scratch, n, m, p.top_k, p.indices + t * p.top_k, sel, hist, shared2);
  }
}

}  // namespace

dsa_status launch_select(const SelectLaunch& a, cudaStream_t stream) {
  const int P = 1 << (32 - __builtin_clz(std::max(a.top_k, 2) - 1));
  SelParams p{a.L,      a.q0,    a.top_k,   a.cap,     a.scale,    a.cand,
              a.cand_n, a.tau,   a.indices, a.fb_rows,  a.counters, a.force_fb_period, a.big_rows};
  cudaError_t e = cudaFuncSetAttribute(select_kernel<SelSmall, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SelSmall::kSmem));
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  e = cudaFuncSetAttribute(select_kernel<SelBig, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(SelBig::kSmem));
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>(a.L, 3 * num_sms()));
  select_kernel<SelSmall, false><<<grid, SelSmall::kThreads, SelSmall::kSmem, stream>>>(p);
  // rows with more candidates than the small shape holds (their number is known on the device)
  const int grid_big = static_cast<int>(std::min<int64_t>(a.L, 2 * num_sms()));
  select_kernel<SelBig, true><<<grid_big, SelBig::kThreads, SelBig::kSmem, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;

  // Fallback rows (their number is known on the device only): scores on the
  // whole grid, select in shared memory, the rest on one CTA per row.  The
  // histograms start from zero.
  if (cudaMemsetAsync(a.fb_hist, 0, static_cast<size_t>(a.fb_ctas) * kFbBins * sizeof(unsigned int),
                      stream) != cudaSuccess)
    return DSA_ERR_CUDA;
  FbParams f{a.Lk,      a.q0,         a.top_k,   a.q_idx,   a.k_idx,  a.esize, a.d,     a.scale,
             a.fb_rows, a.counters,   a.indices, a.fb_scratch, a.fb_hist, a.fb_slow, a.fb_ctas};
  if (a.esize == 1)
    fb_score_kernel<1><<<4 * num_sms(), kSelThreads, 0, stream>>>(f);
  else
    fb_score_kernel<2><<<4 * num_sms(), kSelThreads, 0, stream>>>(f);
  e = cudaFuncSetAttribute(fb_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(SelBig::kSmem));
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  fb_select_kernel<<<a.fb_ctas, SelBig::kThreads, SelBig::kSmem, stream>>>(f);
  const size_t fsmem = static_cast<size_t>(P) * 8 + 256 * 4 + 16 + a.d * 4;
  if (a.esize == 1) {
    e = cudaFuncSetAttribute(fallback_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(fsmem));
    if (e == cudaSuccess) fallback_kernel<1><<<a.fb_ctas, kSelThreads, fsmem, stream>>>(f);
  } else {
    e = cudaFuncSetAttribute(fallback_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(fsmem));
    if (e == cudaSuccess) fallback_kernel<2><<<a.fb_ctas, kSelThreads, fsmem, stream>>>(f);
  }
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
