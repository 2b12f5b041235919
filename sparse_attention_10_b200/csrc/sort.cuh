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

namespace dsa {

// Stable pass on 32-bit keys with 16-bit payloads (positions):
// (kout, pout) = (kin, pin) ordered by the `width`-bit digit ((key - kmin) >> shift),
// width <= 9, DESCENDING, equal digits in input order.  pin == nullptr means
// the identity payload.  Warp w owns items [w * chunk, (w + 1) * chunk), lane
// order within each 32-item slot; ranks inside a warp come from
// __match_any_sync on the digit, so no atomics.  Per-warp digit counters are
// 16-bit (a warp holds at most 32 * SLOTS items): cnt16 is [WARPS][512],
// base [512].
template <int WARPS, int SLOTS>
__device__ void radix_pass32_var(const uint32_t* kin, const uint16_t* pin, uint32_t* kout,
                                 uint16_t* pout, int n, uint32_t kmin, int shift, int width,
                                 uint16_t* cnt16, uint32_t* base) {
  constexpr int kBins = 512;
  constexpr int DPT = (kBins + WARPS * 32 - 1) / (WARPS * 32);   // digits per thread
  static_assert(DPT * WARPS * 32 == kBins, "digits spread evenly over the threads");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = (n + WARPS * 32 - 1) / (WARPS * 32) * 32;  // items per warp
  const int slots = chunk / 32;
  const uint32_t nd = 1u << width, top = nd - 1u;
  uint16_t* wc = cnt16 + warp * kBins;
  for (int d = lane; d < kBins; d += 32) wc[d] = 0;
  __syncwarp();
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t dr[SLOTS];  // digit (bits 16..25, 512 = no item) | rank in warp (bits 0..15)
#pragma unroll
  for (int j = 0; j < SLOTS; ++j) {
    if (j < slots) {
      const int i = warp * chunk + j * 32 + lane;
      const bool ok = i < n;
      const uint32_t d = ok ? top - (((kin[i] - kmin) >> shift) & top) : 512u;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, d);
      const uint32_t before = ok ? wc[d] : 0u;
      dr[j] = (d << 16) | (before + __popc(peers & lt));
      __syncwarp();
      if (ok && lane == __ffs(peers) - 1) wc[d] = static_cast<uint16_t>(before + __popc(peers));
      __syncwarp();
    }
  }
  __syncthreads();
  // per digit (thread t owns digits DPT t .. DPT t + DPT - 1): exclusive prefix
  // over the warps (in place), digit totals
  uint32_t tot[DPT], total = 0;
#pragma unroll
  for (int q = 0; q < DPT; ++q) {
    const int d = DPT * threadIdx.x + q;
    uint32_t run = 0;
#pragma unroll 4
    for (int w = 0; w < WARPS; ++w) {
      const uint32_t c = cnt16[w * kBins + d];
      cnt16[w * kBins + d] = static_cast<uint16_t>(run);
      run += c;
    }
    tot[q] = run;
    total += run;
  }
  // exclusive scan of the digit totals over the block (digits in thread order)
  uint32_t incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) base[kBins + warp] = incl;  // warp sums after the digit bases
  __syncthreads();
  {
    uint32_t off = 0;
    for (int w = 0; w < warp; ++w) off += base[kBins + w];
    off += incl - total;
#pragma unroll
    for (int q = 0; q < DPT; ++q) {
      base[DPT * threadIdx.x + q] = off;
      off += tot[q];
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < SLOTS; ++j) {
    if (j < slots) {
      const uint32_t dg = dr[j] >> 16;
      if (dg < 512u) {
        const int i = warp * chunk + j * 32 + lane;
        const uint32_t pos = base[dg] + cnt16[warp * kBins + dg] + (dr[j] & 0xFFFFu);
        kout[pos] = kin[i];
        pout[pos] = pin ? pin[i] : static_cast<uint16_t>(i);
      }
    }
  }
  __syncthreads();
}

// Stable sort of (key, position) pairs, descending by key, over bits lo..hi
// of key - kmin (the bits where the keys can differ; hi < lo: all keys
// equal): the span is cut into equal digits of at most 9 bits, one pass
// each, least significant first.  Returns through *k / *p the buffers holding
// the result; *p == nullptr means no pass ran (input order).  cnt16 needs
// WARPS * 512 16-bit counters, base 512 + WARPS words.
template <int WARPS, int SLOTS>
__device__ void stable_sort32_by_score(uint32_t** k, uint16_t** p, uint32_t* k_alt,
                                       uint16_t* p_alt, uint16_t* p_first, int n, uint32_t kmin,
                                       int lo, int hi, uint16_t* cnt16, uint32_t* base) {
  uint32_t* kc = *k;
  uint16_t* pc = nullptr;             // identity until the first pass
  uint32_t* kn = k_alt;
  uint16_t* pn = p_first;
  uint16_t* spare = p_alt;
  if (hi >= lo) {
    const int span = hi - lo + 1;
    const int passes = (span + 8) / 9;
    const int width = (span + passes - 1) / passes;
    for (int q = 0; q < passes; ++q) {
      const int sh = lo + q * width;
      const int wd = min(width, hi + 1 - sh);
      radix_pass32_var<WARPS, SLOTS>(kc, pc, kn, pn, n, kmin, sh, wd, cnt16, base);
      uint32_t* tk = kc;
      kc = kn;
      kn = tk;
      uint16_t* tp = pc ? pc : spare;
      pc = pn;
      pn = tp;
    }
  }
  *k = kc;
  *p = pc;  // nullptr: no pass ran, order is the input order
}

}  // namespace dsa
