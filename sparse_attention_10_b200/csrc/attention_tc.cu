// Sparse MQA attention over the selected keys on the fifth-generation tensor
// cores (sm_100a), for head dim 128.
//
// Attention stage of the DeepSeek Sparse Attention page (kwkr.cn/news/60693,
// section 3.3 "standard attention" over the kept keys; section 4.1 BF16;
// section 4.2 one K/V shared by every query head):
//   O[q, h] = sum_{s in S_q} softmax_s(Q[q, h] . K[s] * scale) V[s].
//
// The H <= 16 query heads share every gathered K/V row, so the keys, not the
// heads, are the 128-row M side of both products:
//   S^T[key, head] = K[key] . Q[head]           tcgen05.mma M=128 N=16 K=D
//   O^T[dim, head] = sum_key V[key, dim] P[key, head]   M=128 (dims) N=16 K=16 keys
// Every 128-key tile of S^T gets its own 16 TMEM columns (up to 16 tiles = 256
// columns), so the softmax sees the whole row at once: one max and one sum per
// head, no online rescaling.  P goes to shared memory in BF16 one tile at a
// time and O^T accumulates in TMEM columns 0..15 (tile 0's S columns, which
// the softmax has read before the first P tile is released).
//
// Roles (288 threads, two CTAs per SM, persistent over (query, split) items):
//   warps 0-3  softmax and epilogue; thread i owns TMEM lane i (a key of each
//              S tile, a dim of O);
//   warps 4-7  gather the kept K and V rows with 16-byte cp.async into a ring
//              of 128-key tiles (eight lanes per 256-byte row), laid out as
//              128-byte-swizzled atoms: the K-major A operand of S and, for V,
//              the MN-major A operand of O (the same bytes);
//   warp 8     allocates TMEM and issues the MMAs (one thread).
// Every wait is bounded; a wait that runs out records DSA_ERR_TIMEOUT and
// every role leaves its loop.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kD = 128;            // head dim served by this kernel
constexpr int kKeys = 128;         // keys per tile = TMEM lanes of S^T
constexpr int kN = 16;             // heads padded to the MMA's N
constexpr int kNst = 3;            // K/V tile ring
constexpr int kNp = 2;             // P tile slots
constexpr int kThreads = 288;
constexpr uint32_t kCols = 256;    // TMEM columns: 16 tiles x 16 heads
constexpr int kMaxTiles = DSA_MAX_TOP_K / kKeys;
static_assert(kMaxTiles * kN <= static_cast<int>(kCols), "S of a full item must fit TMEM");

// Shared-memory layout (offsets from a 1024-byte-aligned base).
constexpr int kTileBytes = kKeys * 2 * kD;              // 32 KB: K or V rows of one tile
constexpr int kOffQ = kNst * kTileBytes;                // Q: 16 rows, 2 atoms of 128 B
constexpr int kOffP = kOffQ + kN * 2 * kD;              // P slots: 128 keys x 32 B
constexpr int kPBytes = kKeys * kN * 2;
constexpr int kOffRed = kOffP + kNp * kPBytes;          // [2][16 heads][4 warps] floats
constexpr int kOffBar = kOffRed + 2 * kN * 4 * 4;
enum {
  FULL = 0,
  EMPTY = FULL + kNst,
  Q_FULL = EMPTY + kNst,
  Q_EMPTY,
  S_FULL,
  O_FULL,
  P_FULL,
  P_EMPTY = P_FULL + kNp,
  TM_EMPTY = P_EMPTY + kNp,
  RED_MAX,
  RED_SUM,
  DRAIN,
  NBAR
};
constexpr int kOffSlot = kOffBar + NBAR * 8;            // TMEM base address, abort flag
constexpr int kSmemBytes = kOffSlot + 16 + 1024;        // + alignment slack

struct TcParams {
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
  uint64_t limit_ns;
  int64_t q0;          // prefill: query q sits at key position q0 + q
};

struct Item {
  int64_t q;
  int sp;
  int n;             // kept keys of this item
  int row_limit;     // rows the query may read
  int64_t row_base;  // first K/V row of its sequence
  const int32_t* ids;
};

__device__ __forceinline__ Item make_item(const TcParams& p, int64_t item) {
  Item it;
  it.q = item / p.nsplit;
  it.sp = static_cast<int>(item % p.nsplit);
  int count;
  if (p.seq_start) {
    it.row_base = p.seq_start[it.q];
    const int64_t len = p.seq_start[it.q + 1] - it.row_base;
    count = static_cast<int>(min64(p.top_k, len));
    it.row_limit = static_cast<int>(min64(len, 0x7FFFFFFF));
  } else {
    it.row_base = 0;
    count = static_cast<int>(min64(p.top_k, p.q0 + it.q + 1));
    it.row_limit = static_cast<int>(min64(p.q0 + it.q + 1, 0x7FFFFFFF));
  }
  const int per = (count + p.nsplit - 1) / p.nsplit;
  const int begin = min(count, it.sp * per), end = min(count, begin + per);
  it.n = end - begin;
  it.ids = p.idx + it.q * p.ld_idx + begin;
  return it;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// This thread's shared-memory stores become visible to the tensor cores'
// (async proxy) reads that follow.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
// tcgen05.wait::ld naming the registers of the load it completes, so no use
// of them is scheduled before the wait.
__device__ __forceinline__ void tmem_wait16(uint32_t (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15])
               :
               : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Shared-memory matrix descriptor (tcgen05, version 1) with explicit leading
// and stride byte offsets; layout 2 = 128-byte swizzle, 6 = 32-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}

// S: A = K tile (K-major), B = Q (K-major).  O: A = V tile read as V^T
// (MN-major), B = P read as P^T (MN-major): bits 15 and 16.
constexpr uint32_t kIdescS = make_idesc(1u, kKeys, kN);
constexpr uint32_t kIdescO = make_idesc(1u, kD, kN) | (1u << 15) | (1u << 16);

// Reduce 16 per-thread values over a warp with `op`: lane l ends with head
// l >> 1 (each value halves the lanes that still need it: 8+4+2+1+1 shuffles).
template <typename Op>
__device__ __forceinline__ float warp_reduce16(float (&x)[16], int lane, Op op) {
  float a[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    const bool up = lane & 16;
    const float send = up ? x[h] : x[h + 8];
    const float keep = up ? x[h + 8] : x[h];
    a[h] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 16));
  }
  float b[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const bool up = lane & 8;
    const float send = up ? a[h] : a[h + 4];
    const float keep = up ? a[h + 4] : a[h];
    b[h] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 8));
  }
  float c[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const bool up = lane & 4;
    const float send = up ? b[h] : b[h + 2];
    const float keep = up ? b[h + 2] : b[h];
    c[h] = op(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 4));
  }
  const bool up = lane & 2;
  float d = op(up ? c[1] : c[0], __shfl_xor_sync(0xFFFFFFFFu, up ? c[0] : c[1], 2));
  return op(d, __shfl_xor_sync(0xFFFFFFFFu, d, 1));
}

__global__ void __launch_bounds__(kThreads, 2) attn_tc_kernel(const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sRing = sbase, sQ = sbase + kOffQ, sP = sbase + kOffP;
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffSlot + 4);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kNst; ++i) {
      mbar_init(bar(FULL + i), 128);
      mbar_init(bar(EMPTY + i), 1);
    }
    for (int i = 0; i < kNp; ++i) {
      mbar_init(bar(P_FULL + i), 128);
      mbar_init(bar(P_EMPTY + i), 1);
    }
    mbar_init(bar(Q_FULL), 128);
    mbar_init(bar(Q_EMPTY), 1);
    mbar_init(bar(S_FULL), 1);
    mbar_init(bar(O_FULL), 1);
    mbar_init(bar(TM_EMPTY), 128);
    mbar_init(bar(RED_MAX), 128);
    mbar_init(bar(RED_SUM), 128);
    mbar_init(bar(DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool skip = p.invalid && *p.invalid;
  const int64_t n_items = skip ? 0 : p.nq * p.nsplit;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ gather
    // Eight lanes per key row: lane l8 copies 16-byte chunks l8 (dims 0..63)
    // and l8 + 8 (dims 64..127); chunk c of row r goes to atom c / 8 at
    // r * 128 + ((c % 8) ^ (r % 8)) * 16.  A warp covers four rows per step.
    // Key ids live in registers: for tile kt, lane L of gather warp pw holds
    // the id (or -1) of key kt * 128 + (L / 4) * 16 + pw * 4 + L % 4 (the
    // keys this warp copies) and hands it to the copying lanes by shuffle.
    // The next item's ids are loaded while the current item is copied.  Each
    // thread's copies of a tile are tracked by an asynchronous arrival on the
    // tile's FULL barrier (cp.async.mbarrier.arrive.noinc, 128 expected), so
    // the gather never waits for its own copies.
    const int pw = warp - 4, l8 = lane & 7, kq = lane >> 3;
    const int pt = pw * 32 + lane;
    uint32_t g = 0, ait = 0;
    auto find = [&](int64_t& scan, Item& it, int& nt) -> bool {
      for (; scan < n_items; scan += gridDim.x) {
        it = make_item(p, scan);
        nt = (it.n + kKeys - 1) / kKeys;
        if (nt > 0) {
          scan += gridDim.x;
          return true;
        }
      }
      return false;
    };
    auto load_ids = [&](const Item& it, int nt, int32_t (&v)[kMaxTiles]) {
#pragma unroll
      for (int kt = 0; kt < kMaxTiles; ++kt) {
        const int j = kt * kKeys + (lane >> 2) * 16 + pw * 4 + (lane & 3);
        v[kt] = kt < nt && j < it.n ? __ldg(it.ids + j) : -1;
      }
    };
    // one tile: K or V rows of keys kt * 128 .. +127 into the next stage
    auto tile = [&](const __nv_bfloat16* src, int32_t my_id, bool with_q) -> bool {
      const uint32_t stage = g % kNst;
      if (!mbar_wait(bar(EMPTY + stage), ((g / kNst) & 1) ^ 1, p.limit_ns, abort_flag))
        return false;
      const uint32_t dst = sRing + stage * kTileBytes;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int r = s * 16 + pw * 4 + kq;
        const int32_t id = __shfl_sync(0xFFFFFFFFu, my_id, s * 4 + kq);
        const __nv_bfloat16* row = src + static_cast<int64_t>(id < 0 ? 0 : id) * kD + l8 * 8;
        const uint32_t d = dst + r * 128 + ((l8 ^ (r & 7)) << 4);
        cp_async16(d, row, id < 0 ? 0u : 16u);
        cp_async16(d + kKeys * 128, row + 64, id < 0 ? 0u : 16u);
      }
      cp_async_arrive(bar(FULL + stage));
      if (with_q) cp_async_arrive(bar(Q_FULL));
      ++g;
      return true;
    };
    int64_t scan = blockIdx.x;
    Item cur{}, nxt{};
    int cur_nt = 0, nxt_nt = 0;
    int32_t ids[kMaxTiles], nids[kMaxTiles];
    bool have = find(scan, cur, cur_nt);
    if (have) load_ids(cur, cur_nt, ids);
    bool ok = true;
    while (have && ok) {
      const bool have_nxt = find(scan, nxt, nxt_nt);
      if (have_nxt) load_ids(nxt, nxt_nt, nids);
#pragma unroll
      for (int kt = 0; kt < kMaxTiles; ++kt)
        ids[kt] = ids[kt] >= 0 && ids[kt] < cur.row_limit ? ids[kt] : -1;
      if (!mbar_wait(bar(Q_EMPTY), (ait & 1) ^ 1, p.limit_ns, abort_flag)) break;
      // Q rows (heads >= H zero), same 128-byte-swizzled K-major layout; they
      // complete with the first K tile.
      for (int i = pt; i < kN * 16; i += 128) {
        const int h = i >> 4, c = i & 15;
        cp_async16(sQ + (c >> 3) * (kN * 128) + h * 128 + (((c & 7) ^ (h & 7)) << 4),
                   p.Q + (cur.q * p.H + min(h, p.H - 1)) * kD + c * 8, h < p.H ? 16u : 0u);
      }
      const __nv_bfloat16* Kb = p.K + cur.row_base * kD;
      const __nv_bfloat16* Vb = p.V + cur.row_base * kD;
#pragma unroll
      for (int kt = 0; kt < kMaxTiles; ++kt)
        if (kt < cur_nt && ok) ok = tile(Kb, ids[kt], kt == 0);
#pragma unroll
      for (int kt = 0; kt < kMaxTiles; ++kt)
        if (kt < cur_nt && ok) ok = tile(Vb, ids[kt], false);
      ++ait;
#pragma unroll
      for (int kt = 0; kt < kMaxTiles; ++kt) ids[kt] = nids[kt];
      cur = nxt;
      cur_nt = nxt_nt;
      have = have_nxt;
    }
    cp_async_wait_all();
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t g = 0, pc = 0, ait = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const Item it = make_item(p, item);
        const int nt = (it.n + kKeys - 1) / kKeys;
        if (nt == 0) continue;
        if (!mbar_wait(bar(TM_EMPTY), (ait & 1) ^ 1, p.limit_ns, abort_flag) ||
            !mbar_wait(bar(Q_FULL), ait & 1, p.limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int i = 0; i < nt && ok; ++i) {
          const uint32_t stage = g % kNst;
          if (!mbar_wait(bar(FULL + stage), (g / kNst) & 1, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sRing + stage * kTileBytes;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint32_t off = (ks >> 2) * (kKeys * 128) + (ks & 3) * 32;
            const uint32_t qoff = (ks >> 2) * (kN * 128) + (ks & 3) * 32;
            mma_bf16(tmem_base + i * kN, smem_desc(a0 + off, 16, 1024, 2),
                     smem_desc(sQ + qoff, 16, 1024, 2), kIdescS, ks > 0);
          }
          mma_commit(bar(EMPTY + stage));
          ++g;
        }
        if (!ok) break;
        mma_commit(bar(S_FULL));
        mma_commit(bar(Q_EMPTY));
        for (int i = 0; i < nt && ok; ++i) {
          const uint32_t stage = g % kNst, slot = pc % kNp;
          if (!mbar_wait(bar(FULL + stage), (g / kNst) & 1, p.limit_ns, abort_flag) ||
              !mbar_wait(bar(P_FULL + slot), (pc / kNp) & 1, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sRing + stage * kTileBytes, b0 = sP + slot * kPBytes;
#pragma unroll
          for (int ks = 0; ks < kKeys / 16; ++ks)
            mma_bf16(tmem_base, smem_desc(a0 + ks * 2048, kKeys * 128, 1024, 2),
                     smem_desc(b0 + ks * 512, 16, 256, 6), kIdescO, (i > 0 || ks > 0));
          mma_commit(bar(EMPTY + stage));
          mma_commit(bar(P_EMPTY + slot));
          ++g;
          ++pc;
        }
        if (!ok) break;
        mma_commit(bar(O_FULL));
        ++ait;
      }
      // every MMA issued so far (and its commits' arrivals) done
      mma_commit(bar(DRAIN));
      mbar_wait(bar(DRAIN), 0, p.limit_ns, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = warp * 32 + lane;                       // TMEM lane: key of a tile / dim of O
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    float* red_max = red;                                 // [16 heads][4 warps]
    float* red_sum = red + kN * 4;
    uint32_t pc = 0, ait = 0;
    bool ok = true;
    for (int64_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const Item it = make_item(p, item);
      const int nt = (it.n + kKeys - 1) / kKeys;
      if (nt == 0) {
        if (p.nsplit > 1) {
          // empty split: a partial that the combine weighs by zero
          for (int h = 0; h < p.H; ++h) {
            float* dst = p.part + ((it.q * p.nsplit + it.sp) * p.H + h) * (kD + 2);
            dst[2 + r] = 0.0f;
            if (r == 0) {
              dst[0] = -INFINITY;
              dst[1] = 0.0f;
            }
          }
        } else {
          for (int h = 0; h < p.H; ++h) p.O[(it.q * p.H + h) * kD + r] = __float2bfloat16_rn(0.0f);
        }
        continue;
      }
      uint32_t vmask = 0;
      for (int i = 0; i < nt; ++i) {
        const int j = i * kKeys + r;
        const int32_t id = j < it.n ? __ldg(it.ids + j) : -1;
        vmask |= (id >= 0 && id < it.row_limit ? 1u : 0u) << i;
      }
      if (!mbar_wait(bar(S_FULL), ait & 1, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // pass 1: per-head maximum of the scaled scores (log2 domain)
      float mx[kN];
#pragma unroll
      for (int h = 0; h < kN; ++h) mx[h] = -INFINITY;
      for (int i = 0; i < nt; i += 2) {  // two tiles' loads per wait
        uint32_t v0[16], v1[16];
        const bool two = i + 1 < nt;
        tmem_ld16(tl + i * kN, v0);
        if (two) tmem_ld16(tl + (i + 1) * kN, v1);
        tmem_wait16(v0);
        tmem_wait16(v1);
        if ((vmask >> i) & 1u) {
#pragma unroll
          for (int h = 0; h < kN; ++h) mx[h] = fmaxf(mx[h], __uint_as_float(v0[h]) * p.scale_log2);
        }
        if (two && ((vmask >> (i + 1)) & 1u)) {
#pragma unroll
          for (int h = 0; h < kN; ++h) mx[h] = fmaxf(mx[h], __uint_as_float(v1[h]) * p.scale_log2);
        }
      }
      {
        const float m = warp_reduce16(mx, lane, [](float a, float b) { return fmaxf(a, b); });
        if ((lane & 1) == 0) red_max[(lane >> 1) * 4 + warp] = m;
      }
      mbar_arrive(bar(RED_MAX));
      if (!mbar_wait(bar(RED_MAX), ait & 1, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      float mr[kN];
#pragma unroll
      for (int h = 0; h < kN; ++h) {
        const float4 w = *reinterpret_cast<const float4*>(red_max + h * 4);
        const float m = fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w));
        mr[h] = m == -INFINITY ? 0.0f : m;
      }
      // pass 2: P = 2^(s - max) in BF16 to shared memory, sums in FP32
      float sum[kN];
#pragma unroll
      for (int h = 0; h < kN; ++h) sum[h] = 0.0f;
      // Tile i goes to P slot (pc + i) % kNp.
      auto emit = [&](int i, uint32_t (&v)[16]) -> bool {
        const uint32_t t = pc + i, slot = t % kNp;
        if (!mbar_wait(bar(P_EMPTY + slot), ((t / kNp) & 1) ^ 1, p.limit_ns, abort_flag))
          return false;
        const bool valid = (vmask >> i) & 1u;
        float pr[kN];
#pragma unroll
        for (int h = 0; h < kN; ++h) {
          pr[h] = valid ? fast_exp2(fmaf(__uint_as_float(v[h]), p.scale_log2, -mr[h])) : 0.0f;
          sum[h] += pr[h];
        }
        // key r's 16 heads: 32 bytes, 16-byte halves swapped on rows 4..7 of
        // each 8-row group (32-byte swizzle, MN-major B operand)
        uint8_t* dst = smem + kOffP + slot * kPBytes + r * 32;
        const int sw = (r >> 2) & 1;
        *reinterpret_cast<uint4*>(dst + (sw << 4)) =
            make_uint4(pack_bf16(pr[0], pr[1]), pack_bf16(pr[2], pr[3]), pack_bf16(pr[4], pr[5]),
                       pack_bf16(pr[6], pr[7]));
        *reinterpret_cast<uint4*>(dst + ((sw ^ 1) << 4)) =
            make_uint4(pack_bf16(pr[8], pr[9]), pack_bf16(pr[10], pr[11]),
                       pack_bf16(pr[12], pr[13]), pack_bf16(pr[14], pr[15]));
        fence_proxy_async();
        tc_fence_before();
        mbar_arrive(bar(P_FULL + slot));
        return true;
      };
      for (int i = 0; i < nt; ++i) {
        uint32_t v[16];
        tmem_ld16(tl + i * kN, v);
        tmem_wait16(v);
        if (!emit(i, v)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      pc += nt;
      if (!ok) break;
      {
        const float s = warp_reduce16(sum, lane, [](float a, float b) { return a + b; });
        if ((lane & 1) == 0) red_sum[(lane >> 1) * 4 + warp] = s;
      }
      mbar_arrive(bar(RED_SUM));
      if (!mbar_wait(bar(RED_SUM), ait & 1, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      // Everything but O first: 1 / sum per head in registers and, for split
      // partials, the (max, sum) words; red_max and red_sum are not read
      // after TM_EMPTY, whose completion lets the next item overwrite them.
      float inv[kN];
#pragma unroll
      for (int h = 0; h < kN; ++h) {
        const float4 w = *reinterpret_cast<const float4*>(red_sum + h * 4);
        const float l = (w.x + w.y) + (w.z + w.w);
        if (p.nsplit == 1) {
          inv[h] = l > 0.0f ? 1.0f / l : 0.0f;
        } else {
          inv[h] = 1.0f;
          if (r == 0 && h < p.H) {
            const float4 m = *reinterpret_cast<const float4*>(red_max + h * 4);
            float* dst = p.part + ((it.q * p.nsplit + it.sp) * p.H + h) * (kD + 2);
            dst[0] = fmaxf(fmaxf(m.x, m.y), fmaxf(m.z, m.w));
            dst[1] = l;
          }
        }
      }
      if (!mbar_wait(bar(O_FULL), ait & 1, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t o[16];
      tmem_ld16(tl, o);
      tmem_wait16(o);
      tc_fence_before();
      mbar_arrive(bar(TM_EMPTY));  // O is in registers: the next item's S may start
#pragma unroll
      for (int h = 0; h < kN; ++h) {
        if (h >= p.H) break;
        const float ov = __uint_as_float(o[h]) * inv[h];
        if (p.nsplit == 1)
          p.O[(it.q * p.H + h) * kD + r] = __float2bfloat16_rn(ov);
        else
          p.part[((it.q * p.nsplit + it.sp) * p.H + h) * (kD + 2) + 2 + r] = ov;
      }
      ++ait;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kCols);
  }
}

}  // namespace

bool attention_tc_supported(const AttnLaunch& a) { return a.D == kD && a.H >= 1 && a.H <= kN; }

dsa_status launch_attention_tc(const AttnLaunch& a, cudaStream_t stream) {
  TcParams p{a.Q,         a.K,      a.V,       a.idx, a.ld_idx,  a.nq,     a.H,
             a.scale_log2, a.top_k, a.seq_start, a.nsplit, a.O, a.part, a.invalid,
             wait_limit_ns(), a.q0};
  static_assert(kSmemBytes <= 113 * 1024, "two CTAs per SM");
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  const int64_t items = a.nq * a.nsplit;
  const int grid = static_cast<int>(std::min<int64_t>(items, 2 * static_cast<int64_t>(num_sms())));
  if (grid <= 0) return DSA_OK;
  attn_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace dsa
