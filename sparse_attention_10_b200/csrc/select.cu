// Exact per-query top-k over the indexer's candidate lists (sm_100a).
//
// Token selection of the DeepSeek Sparse Attention page (kwkr.cn/news/60693,
// section 3.3): query t keeps min(top_k, t+1) keys ranked by (score desc,
// key index asc).  A candidate is one 64-bit key (score_bits << 32) |
// (0xFFFFFFFF - s): scores are non-negative floats after ReLU, so their bits
// order like the values, and the low word makes the lower key index win a
// tie.  Larger key = better rank, all keys of a row are distinct.
//
// select_kernel: one CTA per row; loads the row's two candidate lists (one
// per indexer column half) into shared memory, finds the m-th largest key by
// an 8-bit MSD radix select, compacts the m winners and sorts them (bitonic,
// descending) into indices[t].  Rows whose lists overflowed, or hold fewer
// than m keys, are queued for the fallback.
//
// fallback_kernel: recomputes every causal score of a queued row on CUDA
// cores (sequential FP32 FMA, exact for integer-valued inputs), then runs the
// same select over the whole row from a global scratch row.
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kSelThreads = 256;

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

struct SelParams {
  int64_t L;
  int top_k, cap;
  const unsigned long long* cand;
  const int* cand_n;
  int32_t* indices;
  int* fb_rows;
  int* counters;
};

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelParams p) {
  extern __shared__ unsigned long long sel_smem[];
  unsigned long long* keys = sel_smem;                        // [2 * cap]
  unsigned long long* sel = keys + 2 * p.cap;                 // [top_k rounded to pow2]
  unsigned int* hist = reinterpret_cast<unsigned int*>(sel + next_pow2(max(p.top_k, 2)));
  int* shared2 = reinterpret_cast<int*>(hist + 256);
  for (int64_t t = blockIdx.x; t < p.L; t += gridDim.x) {
    const int m = static_cast<int>(min64(p.top_k, t + 1));
    const int n0 = p.cand_n[2 * t], n1 = p.cand_n[2 * t + 1];
    const bool overflow = n0 > p.cap || n1 > p.cap;
    const int n = n0 + n1;
    if (overflow || n < m) {
      if (threadIdx.x == 0) {
        const int pos = atomicAdd(&p.counters[0], 1);
        p.fb_rows[pos] = static_cast<int>(t);
        if (overflow) atomicAdd(&p.counters[1], 1);
      }
      continue;
    }
    if (threadIdx.x == 0) atomicAdd(&p.counters[2], n);
    const unsigned long long* c0 = p.cand + 2 * t * static_cast<int64_t>(p.cap);
    const unsigned long long* c1 = c0 + p.cap;
    for (int i = threadIdx.x; i < n0; i += blockDim.x) keys[i] = c0[i];
    for (int i = threadIdx.x; i < n1; i += blockDim.x) keys[n0 + i] = c1[i];
    __syncthreads();
    finish_row(keys, n, m, p.top_k, p.indices + t * p.top_k, sel, hist, shared2);
  }
}

struct FbParams {
  int64_t L;
  int top_k;
  const void* q_idx;
  const void* k_idx;
  int esize, d;
  float scale;
  const int* fb_rows;
  const int* counters;
  int32_t* indices;
  unsigned long long* scratch;   // [gridDim.x, L]
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

template <int ESIZE>
__device__ __forceinline__ float dot_row(const float* q, const void* base, int64_t row, int d) {
  float acc = 0.0f;
  if (ESIZE == 1) {
    const uint8_t* r = static_cast<const uint8_t*>(base) + row * d;
    for (int j = 0; j < d; j += 16) {
      const uint4 w = *reinterpret_cast<const uint4*>(r + j);
      const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const __nv_fp8x2_storage_t pair =
              static_cast<__nv_fp8x2_storage_t>((words[u] >> (16 * h)) & 0xFFFFu);
          const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3)));
          acc = fmaf(q[j + 4 * u + 2 * h], f.x, acc);
          acc = fmaf(q[j + 4 * u + 2 * h + 1], f.y, acc);
        }
      }
    }
  } else {
    const __nv_bfloat16* r = static_cast<const __nv_bfloat16*>(base) + row * d;
    for (int j = 0; j < d; j += 8) {
      const uint4 w = *reinterpret_cast<const uint4*>(r + j);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(h2[u]);
        acc = fmaf(q[j + 2 * u], f.x, acc);
        acc = fmaf(q[j + 2 * u + 1], f.y, acc);
      }
    }
  }
  return acc;
}

template <int ESIZE>
__global__ void __launch_bounds__(kSelThreads) fallback_kernel(const FbParams p) {
  extern __shared__ unsigned long long fb_smem[];
  unsigned long long* sel = fb_smem;                                   // [pow2(top_k)]
  unsigned int* hist = reinterpret_cast<unsigned int*>(sel + next_pow2(max(p.top_k, 2)));
  int* shared2 = reinterpret_cast<int*>(hist + 256);
  float* qf = reinterpret_cast<float*>(shared2 + 4);                   // [d]
  unsigned long long* scratch = p.scratch + static_cast<int64_t>(blockIdx.x) * p.L;
  const int nfb = *(volatile const int*)p.counters;
  for (int f = blockIdx.x; f < nfb; f += gridDim.x) {
    const int64_t t = p.fb_rows[f];
    const int n = static_cast<int>(t + 1);
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
  SelParams p{a.L, a.top_k, a.cap, a.cand, a.cand_n, a.indices, a.fb_rows, a.counters};
  const size_t smem = (2 * static_cast<size_t>(a.cap) + P) * 8 + 256 * 4 + 16;
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  const int grid = static_cast<int>(std::min<int64_t>(a.L, 4 * num_sms()));
  select_kernel<<<grid, kSelThreads, smem, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;

  FbParams f{a.L, a.top_k, a.q_idx, a.k_idx, a.esize, a.d, a.scale, a.fb_rows, a.counters,
             a.indices, a.fb_scratch};
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
