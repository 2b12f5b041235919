// Sparse MQA attention over the selected keys (sm_100a).
//
// Attention stage of the DeepSeek Sparse Attention page (kwkr.cn/news/60693,
// section 3.3 "standard attention" over the kept keys; section 4.1 BF16;
// section 4.2 one K/V shared by every query head, 128-byte rows, prefetch of
// the next block while the current one is computed):
//   O[q, h] = sum_{s in S_q} softmax_s(Q[q, h] . K[s] * scale) V[s].
//
// One CTA (4 warps) per (query, split).  The selected K and V rows are
// gathered with 16-byte cp.async into padded shared-memory tiles of 64 keys,
// double buffered, so one gathered row serves all H heads.  Each warp takes 16
// keys of a tile: S = Q K^T with mma.sync m16n8k16 (the H <= 16 heads are the
// M dimension), online softmax in FP32 with quad shuffles, P (BF16) V with
// mma.sync.  The four warps' partial (max, sum, O) are merged at the end.
// With more than one split per query (decode), each split writes its
// partial state and a combine kernel merges them (log-sum-exp).
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kAttnThreads = 128;
constexpr int kKeysPerTile = 64;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, FP32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct AttnParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const int32_t* idx;
  int ld_idx;
  int64_t nq;
  int H;
  float scale_log2;
  int top_k;
  const int64_t* seq_start;
  int nsplit;
  __nv_bfloat16* O;
  float* part;
  const int* invalid;
  const int32_t* block_table;   // paged decode cache, else null
  int bt_ld, bs_log2;
  int64_t q0;                   // prefill: query q sits at key position q0 + q
  int qpt;                      // decode: queries per sequence
};

template <int D>
struct AttnSmem {
  static constexpr int kRowQ = 2 * D + 16;            // padded Q row (bytes)
  static constexpr int kRowKV = 2 * D;                // K/V rows are XOR-swizzled, not padded
  static constexpr int kTile = kKeysPerTile * kRowKV; // one K (or V) tile
  static constexpr int kStages = D == 64 ? 4 : 3;
  static constexpr int kQ = 16 * kRowQ;
  static constexpr int kIds = DSA_MAX_TOP_K * 4;
  static constexpr int kMergeRow = D + 8;             // padded merge rows (floats)
  static constexpr int kBytes = kQ + kIds + kStages * 2 * kTile;
};

// Byte offset of 16-byte chunk c of row r in a swizzled K/V tile: the chunk
// index is XORed with the row's low three bits, so the eight rows an
// ldmatrix reads at one logical chunk fall in eight different bank groups.
template <int D>
__device__ __forceinline__ uint32_t kv_off(int r, int c) {
  return static_cast<uint32_t>(r * (2 * D) + ((c ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads) attn_kernel(const AttnParams p) {
  using SM = AttnSmem<D>;
  constexpr int PIECES = D / 8;                  // 16-byte pieces per row
  constexpr int NST = SM::kStages;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;                                         // 16 padded rows
  int32_t* sIds = reinterpret_cast<int32_t*>(smem + SM::kQ);  // this item's key list
  uint8_t* sKV = smem + SM::kQ + SM::kIds;                    // [stages][K tile, V tile]
  const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tig = lane & 3;
  const int64_t n_items = p.nq * p.nsplit;

  griddep_wait();   // the select's indices
  griddep_launch_dependents();
  if (p.invalid && *p.invalid) return;
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int64_t q = item / p.nsplit;
    const int sp = static_cast<int>(item % p.nsplit);
    int64_t row_base = 0;
    int count;
    const int64_t sq = p.seq_start ? q / p.qpt : q;   // decode: the query's sequence
    int64_t qlen = 0;                                   // decode: rows the query sees
    if (p.seq_start) {
      row_base = p.seq_start[sq];
      qlen = p.seq_start[sq + 1] - row_base - (p.qpt - 1 - q % p.qpt);
      count = static_cast<int>(min64(p.top_k, qlen));
    } else {
      count = static_cast<int>(min64(p.top_k, p.q0 + q + 1));
    }
    const int per = (count + p.nsplit - 1) / p.nsplit;
    const int begin = min(count, sp * per), end = min(count, begin + per);
    const int n = end - begin;
    const int32_t* ids = p.idx + q * p.ld_idx + begin;
    // rows a query may read: its causal prefix (prefill) or its sequence (decode)
    const int row_limit = p.seq_start ? static_cast<int>(qlen)
                                      : static_cast<int>(min64(p.q0 + q + 1, 0x7FFFFFFF));
    // a paged cache's key rows are absolute (translated below)
    const int64_t kv_base = p.block_table ? 0 : row_base;
    const __nv_bfloat16* Kb = p.K + kv_base * D;
    const __nv_bfloat16* Vb = p.V + kv_base * D;

    // Q rows (heads >= H are zero) and this item's key list, clamped.
    // (asynchronous copies: every row of Q and the whole key list in flight at once)
    for (int i = tid; i < 16 * PIECES; i += kAttnThreads) {
      const int r = i / PIECES, c = i % PIECES;
      cp_async16(smem_u32(sQ + r * SM::kRowQ + c * 16), p.Q + (q * p.H + min(r, p.H - 1)) * D + c * 8,
                 r < p.H ? 16u : 0u);
    }
    for (int i = tid; i < n; i += kAttnThreads)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(sIds + i)), "l"(ids + i)
                   : "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    for (int i = tid; i < n; i += kAttnThreads) {
      const int s = sIds[i];
      int r = (s >= 0 && s < row_limit) ? s : -1;
      if (p.block_table && r >= 0)   // position in the sequence -> row of the block pool
        r = (__ldg(p.block_table + sq * p.bt_ld + (r >> p.bs_log2)) << p.bs_log2) |
            (r & ((1 << p.bs_log2) - 1));
      sIds[i] = r;
    }
    __syncthreads();

    const int ntiles = (n + kKeysPerTile - 1) / kKeysPerTile;
    // Eight lanes share a key: lane l8 copies 16-byte chunks l8, l8+8, ... of
    // its K row and its V row (each group of eight lanes reads 128 contiguous
    // bytes), with the row address computed once per key; a warp covers four
    // keys per step.  Chunk c of row r lands at kv_off(r, c); with c = l8 + 8h
    // that is the row's base + ((l8 ^ (r & 7)) << 4) + 128 h.
    auto issue = [&](int tile) {
      if (tile < ntiles) {
        const uint32_t st = sKVa + (tile % NST) * 2 * SM::kTile;
        const int l8 = lane & 7, kq = lane >> 3;
#pragma unroll
        for (int it = 0; it < kKeysPerTile / 16; ++it) {
          const int r = it * 16 + warp * 4 + kq;
          const int j = tile * kKeysPerTile + r;
          const int s = j < n ? sIds[j] : -1;
          const uint32_t sz = s < 0 ? 0u : 16u;
          const int64_t row = static_cast<int64_t>(s < 0 ? 0 : s) * D + l8 * 8;
          const uint32_t dk = st + r * (2 * D) + ((l8 ^ (r & 7)) << 4);
#pragma unroll
          for (int h = 0; h < PIECES / 8; ++h) {
            cp_async16(dk + h * 128, Kb + row + h * 64, sz);
            cp_async16(dk + SM::kTile + h * 128, Vb + row + h * 64, sz);
          }
        }
      }
      cp_async_commit();  // possibly empty: keeps one group per tile
    };
#pragma unroll
    for (int t = 0; t < NST - 1; ++t) issue(t);

    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int r = (lane & 7) + ((lane >> 3) & 1) * 8, c = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(sQa + r * SM::kRowQ + c * 2, qa[kk]);
    }
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;

    for (int tile = 0; tile < ntiles; ++tile) {
      cp_async_wait<NST - 2>();   // this tile's copies (issued NST-1 tiles ago) are done
      __syncthreads();            // ... for every thread; the oldest stage is free again
      issue(tile + NST - 1);
      const uint32_t sK = sKVa + (tile % NST) * 2 * SM::kTile;
      const uint32_t sV = sK + SM::kTile;
      // All K fragments first, then S = Q K^T in four independent accumulator
      // chains (even / odd K slices), then the V fragments, whose latency the
      // softmax below hides.
      uint32_t kf[D / 16][4], vf[D / 16][4];
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 7) + (lane >> 4) * 8, c = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(sK + kv_off<D>(r, c), kf[kk]);
      }
      float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float sb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        float (&acc)[2][4] = (kk & 1) ? sb : sa;
        mma16816(acc[0], qa[kk], kf[kk][0], kf[kk][1]);
        mma16816(acc[1], qa[kk], kf[kk][2], kf[kk][3]);
      }
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, c = dt * 2 + (lane >> 4);
        ldsm_x4_t(sV + kv_off<D>(r, c), vf[dt]);
      }
      float s[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = sa[nt][e] + sb[nt][e];
      // scale (log2 domain) and mask keys past the end of this item's list
      const int key0 = tile * kKeysPerTile + warp * 16;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = key0 + nt * 8 + tig * 2 + (e & 1);
          s[nt][e] = j < n ? s[nt][e] * p.scale_log2 : -INFINITY;
        }
      float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
      float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float r0 = n0 == -INFINITY ? 0.0f : n0, r1 = n1 == -INFINITY ? 0.0f : n1;
      const bool same = n0 == m0 && n1 == m1;
      const float c0 = fast_exp2(m0 - r0), c1 = fast_exp2(m1 - r1);
      m0 = n0;
      m1 = n1;
      float pr[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        pr[nt][0] = fast_exp2(s[nt][0] - r0);
        pr[nt][1] = fast_exp2(s[nt][1] - r0);
        pr[nt][2] = fast_exp2(s[nt][2] - r1);
        pr[nt][3] = fast_exp2(s[nt][3] - r1);
      }
      const float ps0 = pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
      const float ps1 = pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
      if (__all_sync(0xFFFFFFFFu, same)) {   // no row max moved: nothing to rescale
        l0 += ps0;
        l1 += ps1;
      } else {
        l0 = l0 * c0 + ps0;
        l1 = l1 * c1 + ps1;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          o[i][0] *= c0;
          o[i][1] *= c0;
          o[i][2] *= c1;
          o[i][3] *= c1;
        }
      }
      uint32_t pa[4];
      pa[0] = pack_bf16(pr[0][0], pr[0][1]);
      pa[1] = pack_bf16(pr[0][2], pr[0][3]);
      pa[2] = pack_bf16(pr[1][0], pr[1][1]);
      pa[3] = pack_bf16(pr[1][2], pr[1][3]);
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        mma16816(o[2 * dt], pa, vf[dt][0], vf[dt][1]);
        mma16816(o[2 * dt + 1], pa, vf[dt][2], vf[dt][3]);
      }
    }
    cp_async_wait<0>();
    __syncthreads();  // all warps done with the tiles: the stage area becomes the merge area

    // ---- merge the four warps' partial states
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    constexpr int MR = SM::kMergeRow;
    float* wm = reinterpret_cast<float*>(sKV);          // [4][16]
    float* wl = wm + 4 * 16;                            // [4][16]
    float* wo = wl + 4 * 16;                            // [4][16][MR]
    if (tig == 0) {
      wm[warp * 16 + g] = m0;
      wm[warp * 16 + g + 8] = m1;
      wl[warp * 16 + g] = l0;
      wl[warp * 16 + g + 8] = l1;
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const int col = i * 8 + tig * 2;
      *reinterpret_cast<float2*>(wo + (warp * 16 + g) * MR + col) = make_float2(o[i][0], o[i][1]);
      *reinterpret_cast<float2*>(wo + (warp * 16 + g + 8) * MR + col) = make_float2(o[i][2], o[i][3]);
    }
    __syncthreads();
    for (int i = tid; i < p.H * (D / 2); i += kAttnThreads) {
      const int h = i / (D / 2), col = (i % (D / 2)) * 2;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * 16 + h]);
      const float Mr = M == -INFINITY ? 0.0f : M;
      float Ls = 0.0f, ox = 0.0f, oy = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = fast_exp2(wm[w * 16 + h] - Mr);
        Ls += f * wl[w * 16 + h];
        const float2 v = *reinterpret_cast<const float2*>(wo + (w * 16 + h) * MR + col);
        ox += f * v.x;
        oy += f * v.y;
      }
      if (p.nsplit == 1) {
        const float inv = Ls > 0.0f ? 1.0f / Ls : 0.0f;
        *reinterpret_cast<__nv_bfloat162*>(p.O + (q * p.H + h) * D + col) =
            __floats2bfloat162_rn(ox * inv, oy * inv);
      } else {
        float* dst = p.part + ((q * p.nsplit + sp) * p.H + h) * (D + 2);
        dst[2 + col] = ox;
        dst[2 + col + 1] = oy;
        if (col == 0) {
          dst[0] = M;
          dst[1] = Ls;
        }
      }
    }
    __syncthreads();  // shared memory is reused by the next item
  }
}

// Merge split partials: O = sum_s 2^(M_s - M) O_s / sum_s 2^(M_s - M) L_s.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(const float* part, int nsplit, int H,
                                                    __nv_bfloat16* O, const int* invalid) {
  griddep_wait();   // the attention's partials
  if (invalid && *invalid) return;
  const int64_t qh = blockIdx.x;
  const int64_t q = qh / H, h = qh % H;
  const int col = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, part[((q * nsplit + s) * H + h) * (D + 2)]);
  const float Mr = M == -INFINITY ? 0.0f : M;
  float num = 0.0f, den = 0.0f;
  for (int s = 0; s < nsplit; ++s) {
    const float* src = part + ((q * nsplit + s) * H + h) * (D + 2);
    const float f = fast_exp2(src[0] - Mr);
    num += f * src[2 + col];
    den += f * src[1];
  }
  O[(q * H + h) * D + col] = __float2bfloat16_rn(den > 0.0f ? num / den : 0.0f);
}

// Split partials -> final output (nothing to do with one split).
template <int D>
dsa_status launch_combine(const AttnLaunch& a, cudaStream_t stream) {
  if (a.nsplit == 1) return DSA_OK;
  const cudaError_t e = launch_maybe_programmatic(combine_kernel<D>, dim3(static_cast<unsigned int>(a.nq * a.H)),
                                                  dim3(D), 0, stream, a.seq_start != nullptr, a.part,
                                                  a.nsplit, a.H, a.O, a.invalid);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

template <int D>
dsa_status launch_d(const AttnLaunch& a, cudaStream_t stream) {
  AttnParams p{a.Q,      a.K,    a.V,       a.idx,         a.ld_idx, a.nq,
               a.H,      a.scale_log2, a.top_k, a.seq_start, a.nsplit, a.O,
               a.part,   a.invalid, a.block_table, a.bt_ld, a.bs_log2, a.q0, std::max(a.qpt, 1)};
  const size_t smem = AttnSmem<D>::kBytes;
  static_assert(AttnSmem<D>::kStages * 2 * AttnSmem<D>::kTile >=
                    (4 * 16 * 2 + 4 * 16 * AttnSmem<D>::kMergeRow) * 4,
                "merge area must fit in the tiles");
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_kernel<D>, kAttnThreads, smem);
  const int64_t items = a.nq * a.nsplit;
  const int grid = static_cast<int>(std::min<int64_t>(items, std::max(1, per_sm) * num_sms()));
  // decode (seq_start set) follows the select kernel: launched programmatically
  const cudaError_t e2 = launch_maybe_programmatic(attn_kernel<D>, dim3(grid), dim3(kAttnThreads), smem, stream,
                                                   a.seq_start != nullptr, p);
  if (e2 != cudaSuccess || cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  return launch_combine<D>(a, stream);
}

}  // namespace

dsa_status launch_attention(const AttnLaunch& a, cudaStream_t stream) {
  // Split launches (decode: 2-8 splits per query) are short items, where the
  // mma.sync kernel's lower per-item latency wins (0.030 vs 0.039 ms for
  // 64 x 2048 keys in 256-key items).  Paged caches take the mma.sync kernel.
  if (a.nsplit == 1 && !a.block_table && attention_tc_supported(a)) {
    const dsa_status st = launch_attention_tc(a, stream);
    return st != DSA_OK ? st : launch_combine<128>(a, stream);
  }
  if (a.D == 64) return launch_d<64>(a, stream);
  if (a.D == 128) return launch_d<128>(a, stream);
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
