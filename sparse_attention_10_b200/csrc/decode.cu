// Decode step: indexer scan over the cache and per-sequence top-k (sm_100a).
//
// One new query per sequence attends over that sequence's cached rows (the
// DeepSeek Sparse Attention page, kwkr.cn/news/60693, sections 3.2-3.3; the
// scan streams the index cache once, section 4.2).
//
// decode_scan_kernel: grid (chunks, B).  Each thread scores whole cache rows:
// 16-byte loads of the row, FP32 FMA in index order (exact for integer
// inputs), relu(fp32(dot) * scale) into a score array, plus a shared-memory
// histogram of the top 11 bits of each score, added to a per-sequence
// histogram in global memory.
//
// decode_select_kernel: a cluster of two CTAs per query (one CTA once the
// queries alone fill the SMs).  The histogram gives the bin of the m-th best
// score; every key at or above that bin is compacted into shared memory (or,
// when too many, into a global scratch row) and the exact select plus sort of
// the prefill path finishes the row.
//
// validate -> scan -> select -> attention -> combine are launched
// programmatically: each kernel lets the next one's CTAs be placed once all of
// its own have started, and the next one waits (griddepcontrol.wait) before
// reading anything.  With the histograms cleared by the counters' memset this
// took the 64-sequence decode step from 0.2246 to 0.2170 ms.
#include <cooperative_groups.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "sort.cuh"

namespace dsa {

// Shared with select.cu (same translation-unit-free helpers re-declared here).
namespace {

constexpr int kScanThreads = 256;
constexpr int kScanRowsPerCta = 2048;
constexpr int kHistBins = 2048;           // score bits 30..20 (scores are >= +0)
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelSlots = 8;
constexpr int kSmemKeys = kSelWarps * 32 * kSelSlots;   // 8192 candidates held in shared memory

__device__ __forceinline__ unsigned long long score_key(float sc, uint32_t s) {
  return (static_cast<unsigned long long>(__float_as_uint(sc)) << 32) | (0xFFFFFFFFu - s);
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

// seq_start must start at 0, end at total_rows, and give lengths in [nq, max_len]
// (nq new tokens per sequence sit at its last nq rows).
__global__ void validate_kernel(const int64_t* seq_start, int B, int64_t total_rows,
                                int64_t max_len, int nq, int* invalid) {
  griddep_launch_dependents();
  bool bad = false;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int64_t len = seq_start[b + 1] - seq_start[b];
    bad |= len < nq || len > max_len;
  }
  if (threadIdx.x == 0) bad |= seq_start[0] != 0 || seq_start[B] != total_rows;
  if (__syncthreads_or(bad) && threadIdx.x == 0) {
    *invalid = 1;
    record_error(DSA_ERR_INVALID_ARG);
  }
}

// Paged cache: every length in [1, max_len] and within its block-table row,
// every block a sequence reaches in [0, num_blocks).  CTA b also writes the
// sum of the lengths before sequence b (and, for the last, the total), which
// the later stages use as seq_start.
__global__ void validate_paged_kernel(const int32_t* seq_lens, int B, int64_t max_len, int nq,
                                      const int32_t* table, int bt_ld, int bs_log2,
                                      int64_t num_blocks, int64_t* seq_start_out, int* invalid) {
  __shared__ long long wsum[32];
  griddep_launch_dependents();
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long before = 0;
  for (int i = threadIdx.x; i < b; i += blockDim.x) before += seq_lens[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xFFFFFFFFu, before, o);
  if (lane == 0) wsum[warp] = before;
  const int64_t len = seq_lens[b];
  bool bad = len < nq || len > max_len || ((len - 1) >> bs_log2) >= bt_ld;
  if (!bad) {
    const int64_t nblk = ((len - 1) >> bs_log2) + 1;
    const int32_t* row = table + static_cast<int64_t>(b) * bt_ld;
    for (int64_t j = threadIdx.x; j < nblk; j += blockDim.x) {
      const int32_t v = row[j];
      bad |= v < 0 || v >= num_blocks;
    }
  }
  const int any_bad = __syncthreads_or(bad);
  if (threadIdx.x == 0) {
    long long start = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) start += wsum[w];
    seq_start_out[b] = start;
    if (b == B - 1) seq_start_out[B] = start + len;
    if (any_bad) {
      *invalid = 1;
      record_error(DSA_ERR_INVALID_ARG);
    }
  }
}

struct ScanParams {
  const void* k_idx;
  const void* q_idx;            // [B * nq, d]
  int d;
  const int64_t* seq_start;
  float scale;
  float* scores;                // query v's scores at score_base(v)
  unsigned int* hist;           // [B * nq, kHistBins]
  const int* invalid;
  const int32_t* block_table;   // paged cache (PAGED kernels only)
  int bt_ld, bs_log2;
  int nq;                       // new tokens per sequence
  int q_first;                  // multi-query scans: first of this launch's queries (0 .. nq-1)
};

// Several new tokens per sequence: query j (0 .. nq-1) of sequence b is query
// v = b * nq + j; it sits at position len_b - nq + j and sees the first
// len_b - nq + 1 + j rows.  Its scores are stored from score_base(v) on: the
// queries' score arrays follow one another in v order.
__device__ __forceinline__ int64_t query_len(const int64_t* seq_start, int b, int j, int nq) {
  return seq_start[b + 1] - seq_start[b] - (nq - 1 - j);
}
__device__ __forceinline__ int64_t score_base(const int64_t* seq_start, int b, int j, int nq) {
  const int64_t len = seq_start[b + 1] - seq_start[b];
  return static_cast<int64_t>(nq) * seq_start[b] - static_cast<int64_t>(b) * (nq * (nq - 1) / 2) +
         static_cast<int64_t>(j) * (len - nq + 1) + j * (j - 1) / 2;
}

// Cache row of row s of sequence b in a paged cache.
__device__ __forceinline__ int64_t paged_row(const ScanParams& p, int b, int64_t s) {
  const int32_t blk = __ldg(p.block_table + static_cast<int64_t>(b) * p.bt_ld + (s >> p.bs_log2));
  return (static_cast<int64_t>(blk) << p.bs_log2) | (s & ((int64_t(1) << p.bs_log2) - 1));
}

template <int ESIZE, bool PAGED>
__global__ void __launch_bounds__(kScanThreads) decode_scan_kernel(const ScanParams p) {
  __shared__ float qf[DSA_MAX_INDEX_DIM];
  __shared__ unsigned int hist[kHistBins];
  griddep_launch_dependents();
  griddep_wait();   // the validation
  if (*p.invalid) return;
  const int b = blockIdx.y;
  const int64_t base = p.seq_start[b];
  const int64_t len = p.seq_start[b + 1] - base;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kScanRowsPerCta;
  if (c0 >= len) return;
  const int64_t c1 = min64(len, c0 + kScanRowsPerCta);
  for (int j = threadIdx.x; j < p.d; j += blockDim.x) {
    if (ESIZE == 1) {
      const __nv_fp8_storage_t v = static_cast<const __nv_fp8_storage_t*>(p.q_idx)[b * p.d + j];
      qf[j] = __half2float(__half(__nv_cvt_fp8_to_halfraw(v, __NV_E4M3)));
    } else {
      qf[j] = __bfloat162float(static_cast<const __nv_bfloat16*>(p.q_idx)[b * p.d + j]);
    }
  }
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  // Zero scores are not counted (the select recovers them as len - sum of
  // bins); lanes that hit the same bin add once through their leader.
  for (int64_t s0 = c0; s0 < c1; s0 += blockDim.x) {
    const int64_t s = s0 + threadIdx.x;
    uint32_t bin = 0;
    if (s < c1) {
      const int64_t row = PAGED ? paged_row(p, b, s) : base + s;
      float sc = __fmul_rn(dot_row<ESIZE>(qf, p.k_idx, row, p.d), p.scale);
      sc = sc > 0.0f ? sc : 0.0f;
      p.scores[base + s] = sc;
      bin = __float_as_uint(sc) >> 20;
    }
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
    if (bin != 0 && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (hist[i]) atomicAdd(&p.hist[static_cast<int64_t>(b) * kHistBins + i], hist[i]);
}

// Coalesced variant for rows of LPR x 16 bytes (LPR a power of two): LPR
// lanes share a row, each holding its 16-byte slice of the query in
// registers; a warp load covers 32 / LPR consecutive rows, eight loads are in
// flight per lane, and log2(LPR) shuffles finish each row's dot product.
//
// PAGED: the cache is block-paged; the CTA's slice of its sequence's block
// table (at most kScanRowsPerCta entries, block sizes being powers of two) is
// staged in shared memory, and each row address is looked up there.
//
// NQ > 1: NQ of the sequence's nq new tokens (q_first .. q_first + NQ - 1)
// are scored against each row at once, so one pass over the index cache serves
// them all; query j keeps the rows up to its position only.  Four queries per
// thread need 148 registers (one CTA per SM) and ran slower than two passes of
// two.  PASS: the launch is one of several (q_first and nq read at run time);
// otherwise NQ is the whole count, which keeps the single-query kernel at 80
// registers (three CTAs per SM).
template <int ESIZE, int LPR, bool PAGED, int NQ, bool PASS>
__global__ void __launch_bounds__(kScanThreads) decode_scan_rows_kernel(const ScanParams p) {
  constexpr int RPL = 32 / LPR;                 // rows per warp load
  constexpr int U = 8;                          // loads in flight per lane
  constexpr int VALS = 16 / ESIZE;              // index values per 16-byte slice
  __shared__ unsigned int hist[NQ][kHistBins];
  __shared__ int32_t blk[PAGED ? kScanRowsPerCta : 1];
  griddep_launch_dependents();
  griddep_wait();   // the validation (and, for a later pass, nothing: launched plainly)
  if (*p.invalid) return;
  const int b = blockIdx.y;
  const int64_t base = p.seq_start[b];
  const int64_t len = p.seq_start[b + 1] - base;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kScanRowsPerCta;
  if (c0 >= len) return;
  const int64_t c1 = min64(len, c0 + kScanRowsPerCta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPR, rsub = lane / LPR;
  const int nq = PASS ? p.nq : NQ;
  const int q_first = PASS ? p.q_first : 0;
  float qv[NQ][VALS];
#pragma unroll
  for (int t = 0; t < NQ; ++t) {
    const int64_t qrow = static_cast<int64_t>(b) * nq + q_first + t;
#pragma unroll
    for (int i = 0; i < VALS; ++i) {
      const int j = sub * VALS + i;
      if (ESIZE == 1) {
        const __nv_fp8_storage_t v = static_cast<const __nv_fp8_storage_t*>(p.q_idx)[qrow * p.d + j];
        qv[t][i] = __half2float(__half(__nv_cvt_fp8_to_halfraw(v, __NV_E4M3)));
      } else {
        qv[t][i] = __bfloat162float(static_cast<const __nv_bfloat16*>(p.q_idx)[qrow * p.d + j]);
      }
    }
  }
  int64_t sbase[NQ];
#pragma unroll
  for (int t = 0; t < NQ; ++t) sbase[t] = score_base(p.seq_start, b, q_first + t, nq);
  for (int i = threadIdx.x; i < NQ * kHistBins; i += blockDim.x) (&hist[0][0])[i] = 0;
  const int64_t j0 = PAGED ? c0 >> p.bs_log2 : 0;
  const int64_t off_mask = (int64_t(1) << p.bs_log2) - 1;
  if (PAGED) {
    const int64_t j1 = (c1 - 1) >> p.bs_log2;
    const int32_t* trow = p.block_table + static_cast<int64_t>(b) * p.bt_ld;
    for (int64_t j = j0 + threadIdx.x; j <= j1; j += blockDim.x) blk[j - j0] = trow[j];
  }
  __syncthreads();
  const uint8_t* rows = static_cast<const uint8_t*>(p.k_idx) + (PAGED ? 0 : base * (LPR * 16));
  // A warp step covers RPL * U rows starting at a multiple of RPL * U; when a
  // block holds at least that many rows they all lie in one block, so one
  // lookup per step serves every load.
  constexpr int kStepLog2 = LPR == 4 ? 6 : LPR == 8 ? 5 : 4;   // log2(RPL * U)
  static_assert((1 << kStepLog2) == RPL * U, "rows per warp step");
  const bool one_block = PAGED && p.bs_log2 >= kStepLog2;
  for (int64_t r0 = c0 + warp * RPL * U; r0 < c1; r0 += (kScanThreads / 32) * RPL * U) {
    uint4 w[U];
    int64_t step_cr = 0;   // cache row of r0 (one-block steps)
    if (one_block)
      step_cr = (static_cast<int64_t>(blk[(r0 >> p.bs_log2) - j0]) << p.bs_log2) | (r0 & off_mask);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = r0 + u * RPL + rsub;
      int64_t cr = r;   // cache row
      if (PAGED) {
        if (one_block) {
          cr = step_cr + (u * RPL + rsub);
        } else {
          const int64_t rr = r < c1 ? r : c0;
          cr = (static_cast<int64_t>(blk[(rr >> p.bs_log2) - j0]) << p.bs_log2) | (rr & off_mask);
        }
      }
      // streaming loads: the cache is read once and should not evict what
      // the attention will gather
      w[u] = r < c1 ? __ldcs(reinterpret_cast<const uint4*>(rows + cr * (LPR * 16) + sub * 16))
                    : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
      float acc[NQ];
#pragma unroll
      for (int t = 0; t < NQ; ++t) acc[t] = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (ESIZE == 1) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const __nv_fp8x2_storage_t pair =
                static_cast<__nv_fp8x2_storage_t>((words[k] >> (16 * h)) & 0xFFFFu);
            const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3)));
#pragma unroll
            for (int t = 0; t < NQ; ++t) {
              acc[t] = fmaf(qv[t][4 * k + 2 * h], f.x, acc[t]);
              acc[t] = fmaf(qv[t][4 * k + 2 * h + 1], f.y, acc[t]);
            }
          }
        } else {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&words[k]));
#pragma unroll
          for (int t = 0; t < NQ; ++t) {
            acc[t] = fmaf(qv[t][2 * k], f.x, acc[t]);
            acc[t] = fmaf(qv[t][2 * k + 1], f.y, acc[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NQ; ++t)
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xFFFFFFFFu, acc[t], o);
      const int64_t r = r0 + u * RPL + rsub;
      if (sub == 0 && r < c1) {
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          if (r < len - (nq - 1 - (q_first + t))) {   // causal for query q_first + t
            float sc = __fmul_rn(acc[t], p.scale);
            sc = sc > 0.0f ? sc : 0.0f;
            p.scores[sbase[t] + r] = sc;
            const uint32_t bin = __float_as_uint(sc) >> 20;
            if (bin) atomicAdd(&hist[t][bin], 1u);  // zero scores are recovered by the select
          }
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NQ * kHistBins; i += blockDim.x) {
    const unsigned int h = (&hist[0][0])[i];
    if (h) atomicAdd(&p.hist[(static_cast<int64_t>(b) * nq + q_first) * kHistBins + i], h);
  }
}

// ---- select ------------------------------------------------------------------

__device__ __forceinline__ void find_from_top_256(const unsigned int* hist, int R, int* out) {
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

template <typename KeyPtr>
__device__ unsigned long long radix_select(KeyPtr keys, int n, int R, unsigned int* hist,
                                           int* sh) {
  unsigned long long prefix = 0, mask = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const unsigned long long k = keys[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) find_from_top_256(hist, R, sh);
    __syncthreads();
    const int bsel = sh[0];
    R = sh[1];
    prefix |= static_cast<unsigned long long>(bsel) << shift;
    mask |= 0xFFull << shift;
    __syncthreads();
  }
  return prefix;
}

__device__ void bitonic_desc(unsigned long long* a, int P) {
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

struct DSelParams {
  const float* scores;
  const unsigned int* hist;
  const int64_t* seq_start;
  int top_k;
  int32_t* indices;
  unsigned long long* scratch;   // [scores] (query v's keys from score_base(v) on)
  const int* invalid;
  int nq;
};

// CL = 2: a cluster of two CTAs per query: both find the boundary bin, each
// compacts the candidates of one half of the query's scores (index order is
// kept: the first CTA takes the lower half), and the first CTA gathers the
// second's list from its shared memory (distributed shared memory) and
// finishes the select.  CL = 1: one CTA per query (queries enough to fill
// the GPU on their own, e.g. several new tokens per sequence).
template <int CL>
__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(kSelThreads)
    decode_select_kernel(const DSelParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned int crank = cluster.block_rank();
  extern __shared__ unsigned long long ds_smem[];
  unsigned long long* bufA = ds_smem;                              // [kSmemKeys]
  unsigned long long* bufB = bufA + kSmemKeys;                     // [kSmemKeys]
  uint32_t* cnt = reinterpret_cast<uint32_t*>(bufB + kSmemKeys);   // [warps][256]
  uint32_t* dbase = cnt + kSelWarps * 256;                         // [256]
  uint32_t* wsum = dbase + 256;                                    // [2][warps]
  int* sh = reinterpret_cast<int*>(wsum + 2 * kSelWarps);          // [8]
  unsigned int* h256 = dbase;                                      // fallback path histogram
  griddep_wait();   // the scan's scores and histograms
  griddep_launch_dependents();
  if (*p.invalid) return;
  const int v = blockIdx.x / CL;              // query v = b * nq + j
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t base = score_base(p.seq_start, v / p.nq, v % p.nq, p.nq);
  const int n = static_cast<int>(query_len(p.seq_start, v / p.nq, v % p.nq, p.nq));
  const int m = min(p.top_k, n);
  const float* sc = p.scores + base;
  const unsigned int* hist = p.hist + static_cast<int64_t>(v) * kHistBins;
  int32_t* out = p.indices + static_cast<int64_t>(v) * p.top_k;

  // Bin of the m-th best score.  The histogram is staged in shared memory
  // (bufB is free until the sort); thread i owns bins 2047 - 2i and 2046 - 2i,
  // a block-wide prefix from the top finds the bin.  Bin 0 (score +0) is not
  // counted by the scan: it holds every key not counted in a higher bin.
  {
    unsigned int* hs = reinterpret_cast<unsigned int*>(bufB);
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hs[i] = i > 0 ? hist[i] : 0u;
    if (threadIdx.x == 0) {
      sh[3] = 0;            // OR of score words
      sh[4] = -1;           // AND of score words
    }
    __syncthreads();
    constexpr int kBinsPer = kHistBins / kSelThreads;
    unsigned int loc[kBinsPer], local = 0;
#pragma unroll
    for (int q = 0; q < kBinsPer; ++q) {
      loc[q] = hs[kHistBins - 1 - kBinsPer * threadIdx.x - q];
      local += loc[q];
    }
    unsigned int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    unsigned int before = 0, above0 = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      const unsigned int x = wsum[w];
      before += w < warp ? x : 0u;
      above0 += x;
    }
    unsigned int run = before + incl - local;
    if (threadIdx.x == kSelThreads - 1) {        // its last bin is bin 0
      loc[kBinsPer - 1] = static_cast<unsigned int>(n) - above0;
      local += loc[kBinsPer - 1];
    }
    if (run < static_cast<unsigned int>(m) && run + local >= static_cast<unsigned int>(m)) {
#pragma unroll
      for (int q = 0; q < kBinsPer; ++q) {
        if (run < static_cast<unsigned int>(m) && run + loc[q] >= static_cast<unsigned int>(m)) {
          sh[0] = kHistBins - 1 - kBinsPer * threadIdx.x - q;
          sh[1] = static_cast<int>(run + loc[q]);  // keys in bins >= that bin
        }
        run += loc[q];
      }
    }
    __syncthreads();
  }
  const uint32_t bin = static_cast<uint32_t>(sh[0]);
  const int ncand = sh[1];

  if (ncand <= kSmemKeys) {
    // Stable compaction of the candidates (score bin >= bin) in index order.
    // Eight consecutive scores per thread and round; the next round's scores
    // are loaded before this round's block scan, and the per-warp counts
    // alternate between two arrays, so a round needs one barrier.
    uint32_t o_or = 0u, o_and = 0xFFFFFFFFu;
    constexpr int kPer = 8;
    constexpr int kRound = kSelThreads * kPer;
    const int half = ((n + 1) / 2 + kPer - 1) / kPer * kPer;
    const int lo = crank ? min(n, half) : 0;      // this CTA's scores: [lo, hi)
    const int hi = (crank || CL == 1) ? n : min(n, half);
    const int rounds = (hi - lo + kRound - 1) / kRound;
    float vn[kPer];
    auto load = [&](int r) {
      const int s = lo + r * kRound + threadIdx.x * kPer;
#pragma unroll
      for (int k = 0; k < kPer; ++k) vn[k] = s + k < hi ? sc[s + k] : 0.0f;
    };
    load(0);
    uint32_t done = 0;
    for (int r = 0; r < rounds; ++r) {
      float v[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) v[k] = vn[k];
      if (r + 1 < rounds) load(r + 1);
      const int s = lo + r * kRound + threadIdx.x * kPer;
      uint32_t flags = 0;
#pragma unroll
      for (int k = 0; k < kPer; ++k)
        if (s + k < hi && (__float_as_uint(v[k]) >> 20) >= bin) flags |= 1u << k;
      const uint32_t c = __popc(flags);
      uint32_t incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t* ws = wsum + (r & 1) * kSelWarps;
      if (lane == 31) ws[warp] = incl;
      __syncthreads();
      const uint32_t x = ws[lane];
      uint32_t wi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
        if (lane >= o) wi += y;
      }
      const uint32_t woff = __shfl_sync(0xFFFFFFFFu, wi - x, warp);
      const uint32_t total = __shfl_sync(0xFFFFFFFFu, wi, 31);
      uint32_t pos = done + woff + incl - c;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        if (flags & (1u << k)) {
          const uint32_t bits = __float_as_uint(v[k]);
          o_or |= bits;
          o_and &= bits;
          if (pos < static_cast<uint32_t>(kSmemKeys)) bufA[pos] = score_key(v[k], static_cast<uint32_t>(s + k));
          ++pos;
        }
      }
      done += total;
    }
    if (threadIdx.x == 0) sh[2] = static_cast<int>(done);
    o_or = __reduce_or_sync(0xFFFFFFFFu, o_or);
    o_and = __reduce_and_sync(0xFFFFFFFFu, o_and);
    if (lane == 0) {
      atomicOr(reinterpret_cast<unsigned int*>(&sh[3]), o_or);
      atomicAnd(reinterpret_cast<unsigned int*>(&sh[4]), o_and);
    }
    if constexpr (CL == 2) {
      cluster.sync();   // both halves compacted (also a barrier of each CTA)
      if (crank == 0) {
        const unsigned long long* rkeys = cluster.map_shared_rank(bufA, 1);
        const int* rsh = cluster.map_shared_rank(sh, 1);
        const int c0 = sh[2], c1 = rsh[2];
        for (int i = threadIdx.x; i < c1; i += blockDim.x)
          if (c0 + i < kSmemKeys) bufA[c0 + i] = rkeys[i];
        __syncthreads();
        if (threadIdx.x == 0) {
          sh[2] = c0 + c1;
          sh[3] |= rsh[3];
          sh[4] &= rsh[4];
        }
      }
      cluster.sync();   // the second CTA's shared memory is no longer read
      if (crank != 0) return;
    } else {
      __syncthreads();
    }
    const int nc = min(sh[2], kSmemKeys);
    const uint32_t vary = static_cast<uint32_t>(sh[3]) ^ static_cast<uint32_t>(sh[4]);
    const unsigned long long* cur =
        stable_sort_by_score<kSelWarps, kSelSlots>(bufA, bufB, nc, vary, cnt, dbase);
    for (int i = threadIdx.x; i < p.top_k; i += blockDim.x)
      out[i] = i < m && i < nc ? static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(cur[i]))
                               : -1;
    return;
  }

  // Many candidates (wide ties): compact into the global scratch row, select
  // the m-th key by radix passes there, then sort the m winners (first CTA of
  // the cluster only).
  if (crank != 0) return;
  unsigned long long* cand = p.scratch + base;
  if (threadIdx.x == 0) sh[2] = 0;
  __syncthreads();
  for (int s = threadIdx.x; s < n; s += blockDim.x) {
    const float v = sc[s];
    if ((__float_as_uint(v) >> 20) >= bin) {
      const int pos = atomicAdd(&sh[2], 1);
      if (pos < ncand) cand[pos] = score_key(v, s);
    }
  }
  __syncthreads();
  const unsigned long long kth = ncand > m ? radix_select(cand, ncand, m, h256, sh) : 0ull;
  unsigned long long* sel = bufA;
  if (threadIdx.x == 0) sh[3] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < ncand; i += blockDim.x) {
    const unsigned long long k = cand[i];
    if (k >= kth) {
      const int pos = atomicAdd(&sh[3], 1);
      if (pos < m) sel[pos] = k;
    }
  }
  int P = 2;
  while (P < m) P <<= 1;
  __syncthreads();
  for (int i = m + threadIdx.x; i < P; i += blockDim.x) sel[i] = 0ull;
  bitonic_desc(sel, P);
  for (int i = threadIdx.x; i < p.top_k; i += blockDim.x)
    out[i] = i < m ? static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(sel[i])) : -1;
}

// pdl: launched programmatically after the validation kernel (first pass only)
template <bool PAGED, int NQ, bool PASS>
bool launch_scan_rows(const ScanParams& sp, dim3 grid, int esize, int lpr, cudaStream_t stream, bool pdl) {
  const dim3 block(kScanThreads);
  if (esize == 1 && lpr == 8)
    launch_maybe_programmatic(decode_scan_rows_kernel<1, 8, PAGED, NQ, PASS>, grid, block, 0, stream, pdl, sp);
  else if (esize == 1 && lpr == 4)
    launch_maybe_programmatic(decode_scan_rows_kernel<1, 4, PAGED, NQ, PASS>, grid, block, 0, stream, pdl, sp);
  else if (esize == 1 && lpr == 16)
    launch_maybe_programmatic(decode_scan_rows_kernel<1, 16, PAGED, NQ, PASS>, grid, block, 0, stream, pdl, sp);
  else if (esize == 2 && lpr == 8)
    launch_maybe_programmatic(decode_scan_rows_kernel<2, 8, PAGED, NQ, PASS>, grid, block, 0, stream, pdl, sp);
  else if (esize == 2 && lpr == 16)
    launch_maybe_programmatic(decode_scan_rows_kernel<2, 16, PAGED, NQ, PASS>, grid, block, 0, stream, pdl, sp);
  else
    return false;
  return true;
}

// Returns false when no kernel serves these rows (several new tokens with an
// index row that is not 64, 128 or 256 bytes).  Several tokens are scanned in
// passes of two (and one for an odd count).
template <bool PAGED>
bool launch_scan(ScanParams sp, dim3 grid, int esize, int lpr, cudaStream_t stream) {
  sp.q_first = 0;
  if (sp.nq == 2) return launch_scan_rows<PAGED, 2, false>(sp, grid, esize, lpr, stream, true);
  if (sp.nq == 1) {
    if (launch_scan_rows<PAGED, 1, false>(sp, grid, esize, lpr, stream, true)) return true;
    if (esize == 1)
      launch_maybe_programmatic(decode_scan_kernel<1, PAGED>, grid, dim3(kScanThreads), 0, stream, true, sp);
    else
      launch_maybe_programmatic(decode_scan_kernel<2, PAGED>, grid, dim3(kScanThreads), 0, stream, true, sp);
    return true;
  }
  for (int q = 0; q < sp.nq; q += 2) {
    sp.q_first = q;
    const bool ok = q + 1 < sp.nq ? launch_scan_rows<PAGED, 2, true>(sp, grid, esize, lpr, stream, q == 0)
                                  : launch_scan_rows<PAGED, 1, true>(sp, grid, esize, lpr, stream, q == 0);
    if (!ok) return false;
  }
  return true;
}

}  // namespace

dsa_status launch_decode_select(const DecodeLaunch& a, cudaStream_t stream) {
  // a.hist was cleared together with the counters
  if (a.seq_lens)
    validate_paged_kernel<<<a.B, 256, 0, stream>>>(a.seq_lens, a.B, a.max_len, a.nq, a.block_table,
                                                   a.bt_ld, a.bs_log2, a.num_blocks,
                                                   a.seq_start_out, a.invalid);
  else
    validate_kernel<<<1, 256, 0, stream>>>(a.seq_start, a.B, a.total_rows, a.max_len, a.nq, a.invalid);
  ScanParams sp{a.k_idx,   a.q_idx,   a.d,           a.seq_start, a.scale,    a.scores,
                a.hist,    a.invalid, a.block_table, a.bt_ld,     a.bs_log2, a.nq, 0};
  const dim3 grid(static_cast<unsigned int>((a.max_len + kScanRowsPerCta - 1) / kScanRowsPerCta),
                  static_cast<unsigned int>(a.B));
  const int lpr = a.d * a.esize / 16;  // 16-byte slices per index row
  const bool launched = a.seq_lens ? launch_scan<true>(sp, grid, a.esize, lpr, stream)
                                   : launch_scan<false>(sp, grid, a.esize, lpr, stream);
  if (!launched) return DSA_ERR_UNSUPPORTED;   // checked by the caller before any launch
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;

  DSelParams dp{a.scores, a.hist, a.seq_start, a.top_k, a.indices, a.keys, a.invalid, a.nq};
  const size_t smem = static_cast<size_t>(2 * kSmemKeys) * 8 +
                      (kSelWarps * 256 + 256 + 2 * kSelWarps + 8) * 4;
  // two CTAs per query while the queries fill at most half the SMs (one CTA per SM)
  const int64_t queries = static_cast<int64_t>(a.B) * a.nq;
  // launched programmatically: its CTAs may be placed while the scan's last wave runs
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (2 * queries <= num_sms()) {
    if (cudaFuncSetAttribute(decode_select_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    cfg.gridDim = dim3(static_cast<unsigned int>(2 * queries));
    e = cudaLaunchKernelEx(&cfg, decode_select_kernel<2>, dp);
  } else {
    if (cudaFuncSetAttribute(decode_select_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return DSA_ERR_CUDA;
    cfg.gridDim = dim3(static_cast<unsigned int>(queries));
    e = cudaLaunchKernelEx(&cfg, decode_select_kernel<1>, dp);
  }
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
