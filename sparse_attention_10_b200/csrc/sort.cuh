// Block-wide stable radix pass used by the per-row selects (sm_100a).
#pragma once

#include <stdint.h>

namespace dsa {

// One stable counting pass over n <= WARPS * 32 * SLOTS 64-bit keys:
// out = in ordered by byte (key >> shift) & 255, DESCENDING; keys with equal
// bytes keep their input order.  Warp w owns a contiguous chunk of the input,
// lanes take consecutive items, so (warp, slot, lane) order is input order.
// Ranks inside a warp come from __match_any_sync and a per-warp digit count
// in shared memory, so there are no atomics.  cnt: [WARPS][256], base: [256].
// Every thread of the block (WARPS warps) must call it.
template <int WARPS, int SLOTS>
__device__ void radix_pass_desc(const unsigned long long* in, unsigned long long* out, int n,
                                int shift, uint32_t* cnt, uint32_t* base) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = (n + WARPS * 32 - 1) / (WARPS * 32) * 32;  // items per warp
  const int slots = chunk / 32;
  uint32_t* wc = cnt + warp * 256;
  for (int d = lane; d < 256; d += 32) wc[d] = 0;
  __syncwarp();
  const uint32_t lt = (1u << lane) - 1u;
  unsigned long long v[SLOTS];
  uint32_t dg[SLOTS], rk[SLOTS];
#pragma unroll
  for (int j = 0; j < SLOTS; ++j) {
    if (j < slots) {
      const int i = warp * chunk + j * 32 + lane;
      const bool ok = i < n;
      v[j] = ok ? in[i] : 0ull;
      const uint32_t d = ok ? 255u - static_cast<uint32_t>((v[j] >> shift) & 255u) : 256u;
      dg[j] = d;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, d);
      const uint32_t before = ok ? wc[d] : 0u;
      rk[j] = before + __popc(peers & lt);
      __syncwarp();
      if (ok && lane == __ffs(peers) - 1) wc[d] = before + __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  if (threadIdx.x < 256) {  // per digit: warp-exclusive prefix, digit total
    const int d = threadIdx.x;
    uint32_t run = 0;
    for (int w = 0; w < WARPS; ++w) {
      const uint32_t c = cnt[w * 256 + d];
      cnt[w * 256 + d] = run;
      run += c;
    }
    base[d] = run;
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // exclusive scan of the 256 digit totals
    uint32_t loc[8], sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      loc[q] = base[lane * 8 + q];
      sum += loc[q];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t ex = incl - sum;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      base[lane * 8 + q] = ex;
      ex += loc[q];
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < SLOTS; ++j) {
    if (j < slots && dg[j] < 256u) out[base[dg[j]] + cnt[warp * 256 + dg[j]] + rk[j]] = v[j];
  }
  __syncthreads();
}

// Sort the n keys of `a` by their score word (bits 32..63), descending and
// stable, with one pass per score byte that differs among the keys
// (`vary` = OR ^ AND of the score words).  Returns the buffer holding the
// result (a or b).
template <int WARPS, int SLOTS>
__device__ unsigned long long* stable_sort_by_score(unsigned long long* a, unsigned long long* b,
                                                    int n, uint32_t vary, uint32_t* cnt,
                                                    uint32_t* base) {
  unsigned long long* cur = a;
  unsigned long long* nxt = b;
  for (int byte = 0; byte < 4; ++byte) {
    if ((vary >> (8 * byte)) & 255u) {
      radix_pass_desc<WARPS, SLOTS>(cur, nxt, n, 32 + 8 * byte, cnt, base);
      unsigned long long* t = cur;
      cur = nxt;
      nxt = t;
    }
  }
  return cur;
}

}  // namespace dsa
