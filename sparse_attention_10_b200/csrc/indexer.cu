// Lightning indexer on 5th-generation tensor cores (sm_100a).
//
// Computes the DSA indexer of the DeepSeek Sparse Attention page
// (kwkr.cn/news/60693, section 3.2): I[t, s] = relu(fp32(q_idx[t] . k_idx[s])
// * scale), FP8 E4M3 (kind::f8f6f4) or BF16 (kind::f16) inputs, FP32
// accumulate in tensor memory.  One CTA per SM, persistent over 128-query
// tiles; for each tile it streams 256-key tiles through a TMA -> shared memory
// ring, issues tcgen05.mma into one of two TMEM accumulators (128 lanes x 256
// columns each) and lets the epilogue warps read the other one.
//
// The epilogue never writes the L x L matrix (section 3.3 / 4.3: the
// selection consumes scores where they are produced).  Three modes:
//   dense   write every score (check / small sizes only);
//   sample  write 16-bit keys of the scores against a few evenly spaced key
//           tiles, from which the per-row threshold is estimated;
//   filter  keep (raw accumulator, key) pairs whose accumulator reaches the
//           row's threshold, appending them to the row's candidate list.
// Causal: key tiles entirely above the diagonal are never issued; the
// diagonal tile is masked per key in the epilogue.
//
// Warp roles (64 + 128 * kCandParts threads): warp 0 issues TMA, warp 1 owns
// TMEM and issues MMAs (one lane), the rest are the epilogue.  Warp w reads
// TMEM lanes 32*(w%4)..+31 (the rule for tcgen05.ld) and columns part p =
// (w-2)/4 of a tile (256 / kCandParts columns), so each query row has one
// candidate list per column part, each in ascending key order.  Two parts
// (eight epilogue warps) measured best over the whole step: four parts cut
// the 128K filter from 5.85 to 5.14 ms but the select's four-way merge cost
// 1.2 ms more.  A chunk that is wholly causal and fits the list takes one
// predicated compare-and-store per column (the column a constant); walking
// each lane's hits instead (a divergent loop and a register select per hit)
// took 5.97 against 4.55 ms on the 128K filter.  Every wait is bounded; on timeout the CTA drains its own copies
// and MMAs, frees TMEM and exits with DSA_ERR_TIMEOUT recorded.
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kEpiWarps = 4 * kCandParts;   // four TMEM lane quarters x column parts
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kPartCols = kBN / kCandParts;  // columns of a tile one epilogue warp reads
constexpr int kChunk = 16;        // columns per TMEM load in the epilogue
constexpr int kMiscBytes = 1024;  // barriers, TMEM slot, abort flag
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kTileA = kBM * 32;   // bytes of one 32-byte K slice of the A tile
constexpr uint32_t kTileB = kBN * 32;   // bytes of one 32-byte K slice of a B tile

// A row of d_bytes is split into column slices of 128 bytes (128-byte
// swizzle), then at most one of 64 bytes (64-byte swizzle) and one of 32
// bytes (32-byte swizzle); each slice is one TMA box per tile and gives
// width/32 MMA K-steps.
constexpr int kMaxSlices = 5;
struct Slices {
  int n;
  int width[kMaxSlices];    // bytes: 128, 64 or 32
  int col[kMaxSlices];      // byte offset of the slice in a row
  int a_off[kMaxSlices];    // shared-memory offset of the slice in the A tile (128 rows)
  int b_off[kMaxSlices];    // ... in a B stage (256 rows)
  int kind[kMaxSlices];     // 0: 128-byte, 1: 64-byte, 2: 32-byte swizzle
};

struct Maps {                // tensor maps per swizzle kind
  CUtensorMap q[3];          // query index rows, 128-row boxes
  CUtensorMap k[3];          // key index rows, 256-row boxes
  CUtensorMap k8[3];         // key index rows, 8-row boxes (sampled mini-tiles)
};

struct Params {
  const void* k_idx;
  int64_t Lq, Lk;
  int64_t q0;     // causal modes: query row i sits at key position q0 + i
  int nkb, stages;
  Slices sl;
  uint32_t off_b, off_bar;
  float scale;
  int mode;
  int n_items;
  const float* tau;
  unsigned long long* cand;
  int* cand_n;
  int cap;        // filter: per-part capacity; sample: full capacity (rows below are kept whole)
  uint16_t* samp;
  int samp_ld;
  float* scores;
  uint64_t limit_ns;
};

__device__ __forceinline__ int sched_item(int round, int cta, int G) {
  // Snake order: descending work in item index, so pair big with small.
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

__device__ __forceinline__ int64_t item_qtile(const Params& p, int item) {
  const int64_t nqt = (p.Lq + kBM - 1) / kBM;
  return p.mode == kModeDense ? item : nqt - 1 - item;
}

__device__ __forceinline__ int64_t sample_span(int64_t r0) {
  // Key tiles entirely below the band of 128 positions before the query tile
  // whose first row sits at key position r0.
  return r0 >= 128 ? (r0 - 128) / kBN : 0;
}

__device__ __forceinline__ int item_ntiles(const Params& p, int64_t qt) {
  if (p.mode == kModeDense) return static_cast<int>((p.Lk + kBN - 1) / kBN);
  const int64_t r0 = qt * kBM;
  if (p.mode == kModeFilter) {
    const int64_t last = p.q0 + min(r0 + kBM, p.Lq) - 1;   // position of the tile's last row
    return static_cast<int>(last / kBN + 1);
  }
  if (p.q0 + r0 + kBM <= p.cap) return 0;  // every row of the tile keeps all its keys
  return static_cast<int>(min64(sample_span(p.q0 + r0), kSampTilesMax));
}

__device__ __forceinline__ int item_ktile(const Params& p, int64_t qt, int j, int nt) {
  if (p.mode != kModeSample) return j;
  return static_cast<int>((static_cast<int64_t>(j) * sample_span(p.q0 + qt * kBM)) / nt);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// tcgen05.wait::ld that also names the 16 registers of the load it completes,
// so the compiler keeps every use of them after the wait.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}

__device__ __forceinline__ uint32_t sample_key16(uint32_t acc_bits) {
  const float f = __uint_as_float(acc_bits);
  return (f > 0.0f ? acc_bits : 0u) >> 16;  // non-negative float bits are monotone
}

constexpr int kMiniRows = 8;                       // rows per sampled mini-tile
constexpr int kMinisPerTile = kBN / kMiniRows;     // 32

// First key of mini-tile i (0 .. nt*32-1) of the query tile whose first row
// sits at position r0: the mini-tiles are spread evenly over the keys below
// the band [r0 - 128, r0 + 128), so every region of the prefix is
// represented (a stratified sample), and each stays inside it.
__device__ __forceinline__ int mini_tile_row(int64_t r0, int i, int nt) {
  const uint64_t span = static_cast<uint64_t>(r0 - 128);           // keys [0, span)
  const uint64_t nmini = static_cast<uint64_t>(nt) * kMinisPerTile;
  const uint64_t room = span - kMiniRows;                          // span >= 256 * nt
  return static_cast<int>((static_cast<uint64_t>(i) * room) / (nmini - 1 > 0 ? nmini - 1 : 1));
}

template <int ESIZE>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + p.off_b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  const int S = p.stages;
  // barrier slots
  const int FULL = 0, EMPTY = S, A_FULL = 2 * S, A_EMPTY = 2 * S + 1, ACC_FULL = 2 * S + 2,
            ACC_EMPTY = 2 * S + 4, DRAIN = 2 * S + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t stage_bytes = static_cast<uint32_t>(p.nkb) * kTileB;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(bar(FULL + i), 1);
      mbar_init(bar(EMPTY + i), 1);
    }
    mbar_init(bar(A_FULL), 1);
    mbar_init(bar(A_EMPTY), 1);
    mbar_init(bar(ACC_FULL), 1);
    mbar_init(bar(ACC_FULL + 1), 1);
    mbar_init(bar(ACC_EMPTY), kEpiWarps);
    mbar_init(bar(ACC_EMPTY + 1), kEpiWarps);
    mbar_init(bar(DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < p.sl.n; ++i) {
      tma_prefetch_desc(&maps.q[p.sl.kind[i]]);
      tma_prefetch_desc(&maps.k[p.sl.kind[i]]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Lane 0 issues the TMA copies and barrier operations.  In sample mode the
    // whole warp issues them, one 8-row mini-tile per lane.
    const bool gather = p.mode == kModeSample;
    if (gather || lane == 0) {
      uint32_t it = 0, item_it = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int item = sched_item(round, blockIdx.x, gridDim.x);
        if (item >= p.n_items) break;
        const int64_t qt = item_qtile(p, item);
        const int nt = item_ntiles(p, qt);
        if (nt == 0) continue;
        if (lane == 0) {
          ok = mbar_wait(bar(A_EMPTY), (item_it & 1) ^ 1, p.limit_ns, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(bar(A_FULL), p.nkb * kTileA);
            for (int i = 0; i < p.sl.n; ++i)
              tma_load_2d(sA + p.sl.a_off[i], &maps.q[p.sl.kind[i]], p.sl.col[i] / ESIZE,
                          static_cast<int>(qt * kBM), bar(A_FULL));
          }
        }
        if (gather) ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++item_it;
        for (int j = 0; j < nt; ++j) {
          const uint32_t s = it % S, ph = (it / S) & 1;
          if (lane == 0) ok = mbar_wait(bar(EMPTY + s), ph ^ 1, p.limit_ns, abort_flag);
          if (gather) ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          const uint32_t dst = sB + s * stage_bytes;
          if (!gather) {
            mbar_arrive_expect_tx(bar(FULL + s), stage_bytes);
            const int kt = item_ktile(p, qt, j, nt);
            for (int i = 0; i < p.sl.n; ++i)
              tma_load_2d(dst + p.sl.b_off[i], &maps.k[p.sl.kind[i]], p.sl.col[i] / ESIZE, kt * kBN,
                          bar(FULL + s));
          } else {
            // 32 mini-tiles of 8 consecutive keys; each lane loads one mini-tile
            // (all 32-byte slices) into rows 8*lane .. 8*lane+7 of the stage.
            if (lane == 0) mbar_arrive_expect_tx(bar(FULL + s), stage_bytes);
            __syncwarp();
            const int y = mini_tile_row(p.q0 + qt * kBM, j * kMinisPerTile + lane, nt);
            for (int i = 0; i < p.sl.n; ++i)
              tma_load_2d(dst + p.sl.b_off[i] + lane * kMiniRows * p.sl.width[i], &maps.k8[p.sl.kind[i]],
                          p.sl.col[i] / ESIZE, y, bar(FULL + s));
          }
          ++it;
        }
      }
      if (lane == 0) {
        const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0;
        if (ok) {
          // Every stage still held is released by an MMA commit; wait for those
          // arrivals so none lands after the CTA exits.
          for (uint32_t i = first; i < it; ++i)
            mbar_wait(bar(EMPTY + i % S), (i / S) & 1, p.limit_ns, nullptr);
        } else {
          // Aborted: wait for the data of every copy still in flight.
          for (uint32_t i = first; i < it; ++i)
            mbar_wait(bar(FULL + i % S), (i / S) & 1, p.limit_ns, nullptr);
          if (item_it) mbar_wait(bar(A_FULL), (item_it - 1) & 1, p.limit_ns, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(ESIZE == 1 ? 0u : 1u, kBM, kBN);
      uint32_t it = 0, acc_it = 0, item_it = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int item = sched_item(round, blockIdx.x, gridDim.x);
        if (item >= p.n_items) break;
        const int64_t qt = item_qtile(p, item);
        const int nt = item_ntiles(p, qt);
        if (nt == 0) continue;
        if (!mbar_wait(bar(A_FULL), item_it & 1, p.limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < nt; ++j) {
          const uint32_t s = it % S, ph = (it / S) & 1;
          const uint32_t buf = acc_it & 1;
          if (!mbar_wait(bar(FULL + s), ph, p.limit_ns, abort_flag) ||
              !mbar_wait(bar(ACC_EMPTY + buf), ((acc_it >> 1) & 1) ^ 1, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + buf * kBN;
          const uint32_t bstage = sB + s * stage_bytes;
          uint32_t acc = 0;
          for (int i = 0; i < p.sl.n; ++i) {
            for (int k = 0; k < p.sl.width[i]; k += 32) {  // one MMA per 32 bytes of K
              const uint64_t ad = smem_desc_kmajor(sA + p.sl.a_off[i] + k, p.sl.kind[i]);
              const uint64_t bd = smem_desc_kmajor(bstage + p.sl.b_off[i] + k, p.sl.kind[i]);
              if (ESIZE == 1)
                mma_f8(d_tmem, ad, bd, idesc, acc);
              else
                mma_bf16(d_tmem, ad, bd, idesc, acc);
              acc = 1;
            }
          }
          mma_commit(bar(EMPTY + s));
          mma_commit(bar(ACC_FULL + buf));
          ++it;
          ++acc_it;
        }
        if (!ok) break;
        mma_commit(bar(A_EMPTY));
        ++item_it;
      }
      // Drain: every MMA issued so far (and the arrivals of its commits) done.
      mma_commit(bar(DRAIN));
      mbar_wait(bar(DRAIN), 0, p.limit_ns, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int part = ew >> 2;
    const int row_local = quarter * 32 + lane;
    uint32_t acc_it = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int item = sched_item(round, blockIdx.x, gridDim.x);
      if (item >= p.n_items) break;
      const int64_t qt = item_qtile(p, item);
      const int nt = item_ntiles(p, qt);
      if (nt == 0) continue;
      const int64_t t = qt * kBM + row_local;
      const bool row_ok = t < p.Lq;
      float tau = INFINITY;
      if (p.mode == kModeFilter && row_ok) tau = p.tau[t];
      int count = 0;
      unsigned long long* my_cand =
          p.mode == kModeFilter && row_ok ? p.cand + (kCandParts * t + part) * static_cast<int64_t>(p.cap)
                                          : nullptr;
      for (int j = 0; j < nt; ++j) {
        const uint32_t buf = acc_it & 1;
        if (!mbar_wait(bar(ACC_FULL + buf), (acc_it >> 1) & 1, p.limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kt = item_ktile(p, qt, j, nt);
        const uint32_t tbase =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kBN + part * kPartCols;
        // Chunk c+1's TMEM load is in flight while chunk c is processed.
        auto process = [&](int c, uint32_t (&v)[kChunk]) {
            const int64_t s0 = static_cast<int64_t>(kt) * kBN + part * kPartCols + c * kChunk;
            if (p.mode == kModeFilter) {
              const int64_t lim0 = p.q0 + t - s0;
              if (row_ok && lim0 >= kChunk - 1 && count + kChunk <= p.cap) {
                // Whole chunk causal and room for every column: one predicated
                // compare-and-store per column, with the column index a constant.
                uint2* dst = reinterpret_cast<uint2*>(my_cand + count);
                const uint32_t nbase = 0xFFFFFFFFu - static_cast<uint32_t>(s0);
                int n = 0;
#pragma unroll
                for (int q = 0; q < kChunk; ++q) {
                  if (__uint_as_float(v[q]) >= tau) {
                    dst[n] = make_uint2(nbase - q, v[q]);
                    ++n;
                  }
                }
                count += n;
                return;
              }
              uint32_t pass = 0;
#pragma unroll
              for (int q = 0; q < kChunk; ++q) pass |= (__uint_as_float(v[q]) >= tau ? 1u : 0u) << q;
              const int64_t lim = p.q0 + t - s0;  // keys s0 .. q0 + t are causal
              if (lim < kChunk - 1) pass &= lim < 0 ? 0u : ((2u << lim) - 1u);
              if (!row_ok) pass = 0;
              if (pass) {
                // Each hit is stored as (raw accumulator bits, ~key); the select
                // turns the accumulator into relu(fp32(acc) * scale).
                const int hits = __popc(pass);
                if (count + hits <= p.cap) {
                  uint2* dst = reinterpret_cast<uint2*>(my_cand + count);
                  const uint32_t nbase = 0xFFFFFFFFu - static_cast<uint32_t>(s0);
                  while (pass) {
                    const int q = __ffs(pass) - 1;
                    pass &= pass - 1;
                    // v[q] by a select tree over the 16 registers
                    uint32_t t8[8], t4[4], t2[2];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t8[e] = (q & 1) ? v[2 * e + 1] : v[2 * e];
#pragma unroll
                    for (int e = 0; e < 4; ++e) t4[e] = (q & 2) ? t8[2 * e + 1] : t8[2 * e];
#pragma unroll
                    for (int e = 0; e < 2; ++e) t2[e] = (q & 4) ? t4[2 * e + 1] : t4[2 * e];
                    *dst++ = make_uint2(nbase - q, (q & 8) ? t2[1] : t2[0]);
                  }
                }
                count += hits;
              }
            } else if (p.mode == kModeSample) {
              if (row_ok) {
                uint32_t w[kChunk / 2];
#pragma unroll
                for (int q = 0; q < kChunk / 2; ++q)
                  w[q] = sample_key16(v[2 * q]) | (sample_key16(v[2 * q + 1]) << 16);
                uint4* dst = reinterpret_cast<uint4*>(p.samp + t * p.samp_ld + j * kBN + part * kPartCols +
                                                      c * kChunk);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
              }
            } else {
              if (row_ok) {
                float* out = p.scores + t * p.Lk;
#pragma unroll
                for (int q = 0; q < kChunk; ++q) {
                  const int64_t s = s0 + q;
                  if (s < p.Lk) {
                    const float sc = __fmul_rn(__uint_as_float(v[q]), p.scale);
                    out[s] = sc > 0.0f ? sc : 0.0f;
                  }
                }
              }
            }
          };
        uint32_t va[kChunk], vb[kChunk];
        tmem_ld16(tbase, va);
        tmem_ld_wait_regs(va);
#pragma unroll
        for (int c = 0; c < kPartCols / kChunk; c += 2) {
          tmem_ld16(tbase + (c + 1) * kChunk, vb);
          process(c, va);
          __syncwarp();
          tmem_ld_wait_regs(vb);
          if (c + 2 < kPartCols / kChunk) tmem_ld16(tbase + (c + 2) * kChunk, va);
          process(c + 1, vb);
          __syncwarp();
          if (c + 2 < kPartCols / kChunk) tmem_ld_wait_regs(va);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ACC_EMPTY + buf));
        ++acc_it;
      }
      if (!ok) break;
      if (p.mode == kModeFilter && row_ok) p.cand_n[kCandParts * t + part] = count;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();
    tmem_dealloc(tmem_base, 2 * kBN);
  }
}

// ---- threshold from the sample --------------------------------------------------

// Lane l owns bins 255-8l .. 248-8l (top first).  Finds the bin holding the
// R-th largest key (1-based) and the rank of that key inside the bin.
__device__ __forceinline__ void warp_find_from_top(const unsigned int* hist, int R, int* bin,
                                                   int* rank_in_bin) {
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
  int b = 0, r = 0;
  if (lane == src) {
    unsigned int run = incl - local;
    for (int i = 0; i < 8; ++i) {
      const int bb = 255 - 8 * lane - i;
      if (run + hist[bb] >= static_cast<unsigned int>(R)) {
        b = bb;
        r = R - static_cast<int>(run);
        break;
      }
      run += hist[bb];
    }
  }
  *bin = __shfl_sync(0xFFFFFFFFu, b, src);
  *rank_in_bin = __shfl_sync(0xFFFFFFFFu, r, src);
}

// One warp per query row t.  Rows with t + 1 <= cap keep every key (tau =
// -inf).  Otherwise the R-th largest sampled 16-bit key, with R chosen so that
// about `target` keys of the whole row reach it, gives a raw-accumulator
// threshold; it is lowered to the smallest accumulator whose scaled score
// equals that key's score, so the filter keeps whole ties.
__global__ void __launch_bounds__(256) tau_kernel(const uint16_t* samp, int samp_ld, int64_t L,
                                                  int64_t q0, int cap, int target, float scale,
                                                  float* tau) {
  __shared__ unsigned int hist_all[8][256];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + w;
  if (row >= L) return;
  const int64_t t = q0 + row;          // the query's key position
  unsigned int* hist = hist_all[w];
  if (t + 1 <= cap) {
    if (lane == 0) tau[row] = -INFINITY;
    return;
  }
  const int64_t qt = row / kBM;
  const int ns = static_cast<int>(min64(sample_span(q0 + qt * kBM), kSampTilesMax));
  if (ns == 0) {
    if (lane == 0) tau[row] = -INFINITY;
    return;
  }
  const int n = ns * kBN;
  const uint16_t* src = samp + row * samp_ld;
  int R = static_cast<int>((static_cast<int64_t>(n) * target + t) / (t + 1));
  R = max(1, min(R, n));
  for (int i = lane; i < 256; i += 32) hist[i] = 0;
  __syncwarp();
  for (int i = lane; i < n; i += 32) atomicAdd(&hist[src[i] >> 8], 1u);
  __syncwarp();
  int b1, r1;
  warp_find_from_top(hist, R, &b1, &r1);
  __syncwarp();
  for (int i = lane; i < 256; i += 32) hist[i] = 0;
  __syncwarp();
  for (int i = lane; i < n; i += 32) {
    const uint32_t k = src[i];
    if (static_cast<int>(k >> 8) == b1) atomicAdd(&hist[k & 255], 1u);
  }
  __syncwarp();
  int b2, r2;
  warp_find_from_top(hist, r1, &b2, &r2);
  if (lane == 0) {
    float a = __uint_as_float(static_cast<uint32_t>((b1 << 8) | b2) << 16);
    const float sigma = __fmul_rn(a, scale);
    if (!(a > 0.0f) || !(sigma > 0.0f)) {
      // The sampled rank falls among ReLU zeros: keep every positive score
      // (smallest positive threshold) and let the select add zeros by index.
      tau[row] = __uint_as_float(1u);
      return;
    }
    for (int i = 0; i < 64; ++i) {
      const float prev = __uint_as_float(__float_as_uint(a) - 1u);
      if (prev > 0.0f && __fmul_rn(prev, scale) >= sigma)
        a = prev;
      else
        break;
    }
    tau[row] = a;
  }
}

// ---- host side -----------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Row-major [rows, d] matrix, boxes of `width` bytes x box_rows, swizzle
// matching the width (128, 64 or 32 bytes).
bool make_map(CUtensorMap* m, const void* base, int esize, int d, int64_t rows, int box_rows,
              int width) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(width / esize), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = width == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : width == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(m, esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

Slices make_slices(int d_bytes) {
  Slices sl{};
  int col = 0;
  auto add = [&](int w, int kind) {
    sl.width[sl.n] = w;
    sl.col[sl.n] = col;
    sl.a_off[sl.n] = col * kBM;
    sl.b_off[sl.n] = col * kBN;
    sl.kind[sl.n] = kind;
    ++sl.n;
    col += w;
  };
  while (d_bytes - col >= 128) add(128, 0);
  if (d_bytes - col >= 64) add(64, 1);
  if (d_bytes - col >= 32) add(32, 2);
  return sl;
}

}  // namespace

dsa_status launch_indexer(const IndexerLaunch& a, cudaStream_t stream) {
  const int d_bytes = a.d * a.esize;
  if (d_bytes % 32 != 0 || d_bytes <= 0 || a.d > DSA_MAX_INDEX_DIM) return DSA_ERR_UNSUPPORTED;
  const int nkb = d_bytes / 32;
  const uint32_t a_bytes = nkb * kTileA, stage_bytes = nkb * kTileB;
  const int avail = kSmemLimit - 1024 - static_cast<int>(a_bytes) - kMiscBytes;
  const int stages = std::min(8, avail / static_cast<int>(stage_bytes));
  if (stages < 1) return DSA_ERR_UNSUPPORTED;

  Params p{};
  p.k_idx = a.k_idx;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.q0 = a.q0;
  p.nkb = nkb;
  p.stages = stages;
  p.off_b = a_bytes;
  p.off_bar = a_bytes + stages * stage_bytes;
  p.scale = a.scale;
  p.mode = a.mode;
  p.n_items = static_cast<int>((a.Lq + kBM - 1) / kBM);
  p.tau = a.tau;
  p.cand = a.cand;
  p.cand_n = a.cand_n;
  p.cap = a.cap;
  p.samp = a.samp;
  p.samp_ld = a.samp_ld;
  p.scores = a.scores;
  p.limit_ns = a.limit_ns;
  // At least 116 KB so two CTAs never share an SM (each holds all 512 TMEM columns).
  const size_t smem = std::max<size_t>(p.off_bar + kMiscBytes + 1024, 116 * 1024);

  p.sl = make_slices(d_bytes);
  Maps maps{};
  const int widths[3] = {128, 64, 32};
  for (int kind = 0; kind < 3; ++kind) {
    bool used = false;
    for (int i = 0; i < p.sl.n; ++i) used |= p.sl.kind[i] == kind;
    if (!used) continue;  // maps of unused kinds stay zero and are never read
    const int w = widths[kind];
    if (!make_map(&maps.q[kind], a.q_idx, a.esize, a.d, a.Lq, kBM, w) ||
        !make_map(&maps.k[kind], a.k_idx, a.esize, a.d, a.Lk, kBN, w) ||
        !make_map(&maps.k8[kind], a.k_idx, a.esize, a.d, a.Lk, kMiniRows, w))
      return DSA_ERR_CUDA;
  }

  const int grid = std::max(1, std::min(p.n_items, num_sms()));
  cudaError_t e;
  if (a.esize == 1) {
    e = cudaFuncSetAttribute(indexer_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess) indexer_kernel<1><<<grid, kThreads, smem, stream>>>(maps, p);
  } else {
    e = cudaFuncSetAttribute(indexer_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess) indexer_kernel<2><<<grid, kThreads, smem, stream>>>(maps, p);
  }
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status launch_tau_select(const uint16_t* samp, int samp_ld, int64_t L, int64_t q0, int cap,
                             int target, float scale, float* tau, cudaStream_t stream) {
  const int64_t blocks = (L + 7) / 8;
  tau_kernel<<<static_cast<unsigned int>(blocks), 256, 0, stream>>>(samp, samp_ld, L, q0, cap, target,
                                                                    scale, tau);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
