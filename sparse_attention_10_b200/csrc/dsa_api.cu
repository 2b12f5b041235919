// C ABI of the DSA library: argument checks, workspace layout, launch order.
//
// dsa_prefill runs, in stream order:
//   1. indexer (sample mode)  scores against a few key tiles per query tile;
//   2. tau_kernel             per-row raw-accumulator threshold from the sample;
//   3. indexer (filter mode)  every causal score, candidates >= threshold;
//   4. select_kernel          exact top-k + order per row (fallback queue);
//      fallback_kernel        exact recomputation for queued rows;
//   5. attn_kernel            gathered sparse MQA attention.
// dsa_decode runs the scan, the per-sequence select and split attention.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dsa {

__device__ unsigned int g_status = 0;

// dsa_debug_force_fallback's period (0: off).
std::atomic<int> g_force_fb_period{0};

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int esize_of(int idx_dtype) {
  return idx_dtype == DSA_IDX_FP8_E4M3 ? 1 : (idx_dtype == DSA_IDX_BF16 ? 2 : 0);
}

dsa_status check_index_dims(int idx_dtype, int d_idx) {
  const int es = esize_of(idx_dtype);
  if (es == 0) return DSA_ERR_INVALID_ARG;
  if (d_idx <= 0 || d_idx > DSA_MAX_INDEX_DIM) return DSA_ERR_INVALID_ARG;
  if ((d_idx * es) % 32 != 0) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

float default_scale(float s, int dim) {
  return std::isnan(s) ? static_cast<float>(1.0 / std::sqrt(static_cast<double>(dim))) : s;
}

// ---- prefill workspace ----------------------------------------------------------

struct PrefillPlan {
  int cap_part;     // candidates kept per (row, column part of the indexer tile)
  int cap_all;      // rows with t + 1 <= cap_all keep every key
  int target;       // candidates aimed for per row by the threshold
  int samp_ld;
  int fb_ctas;
  size_t off_counters, off_tau, off_cand_n, off_cand, off_samp, off_fb_rows, off_fb_scratch,
      off_fb_hist, off_fb_slow, off_big_rows, total;
};

// L query rows against Lk key rows (Lk = L for a whole sequence).
PrefillPlan plan_prefill(int64_t L, int top_k, int64_t Lk) {
  PrefillPlan p{};
  // 1.4 k: on the synthetic workloads the realized count has a spread of
  // about 0.1 k around the target, so fewer than k survivors (a fallback
  // row) is a > 4-sigma event; each extra 0.1 k costs filter stores and
  // select work in proportion.
  p.target = (top_k * 7 + 2) / 5;
  // Per part about target / kCandParts candidates arrive; the capacity leaves twice that plus
  // 128.  Rows with t + 1 <= cap_all (1.25 k + 128) keep every key: at most
  // ceil(cap_all / 256) * 256 / kCandParts of them fall in one part, below cap_part.
  p.cap_part = ((top_k * 14 / (5 * kCandParts) + 128) + 15) / 16 * 16;
  p.cap_all = ((top_k * 5 / 4 + 128) + 15) / 16 * 16;
  p.samp_ld = kSampTilesMax * kBN;
  p.fb_ctas = std::max(1, num_sms());
  size_t o = 0;
  p.off_counters = o;
  o = align_up(o + 64 * sizeof(int));
  p.off_tau = o;
  o = align_up(o + L * sizeof(float));
  p.off_cand_n = o;
  o = align_up(o + kCandParts * L * sizeof(int));
  p.off_cand = o;
  o = align_up(o + static_cast<size_t>(kCandParts * L) * p.cap_part * sizeof(unsigned long long));
  p.off_samp = o;
  o = align_up(o + static_cast<size_t>(L) * p.samp_ld * sizeof(uint16_t));
  p.off_fb_rows = o;
  o = align_up(o + L * sizeof(int));
  p.off_fb_scratch = o;
  o = align_up(o + static_cast<size_t>(p.fb_ctas) * Lk * sizeof(unsigned long long));
  p.off_fb_hist = o;
  o = align_up(o + static_cast<size_t>(p.fb_ctas) * 4096 * sizeof(unsigned int));
  p.off_fb_slow = o;
  o = align_up(o + static_cast<size_t>(p.fb_ctas) * sizeof(int));
  p.off_big_rows = o;
  o = align_up(o + L * sizeof(int));
  p.total = o;
  return p;
}

// ---- decode workspace -------------------------------------------------------------

// Upper bound on the key splits per decode sequence (sizes the partials).  A launch uses as
// many as fill one wave of two attention CTAs per SM, at least 2: at 64 sequences on 148 SMs
// that is 4 splits, which timed 15% faster than 8 (two waves of shorter items).
constexpr int kDecodeSplits = 8;

static int decode_splits(int queries) {
  return std::clamp(2 * num_sms() / std::max(queries, 1), 2, kDecodeSplits);
}

struct DecodePlan {
  size_t off_counters, off_scores, off_hist, off_keys, off_indices, off_part, off_seq, total;
};

// paged: one more array, the running sum of the lengths [B + 1] (int64).
// nq new tokens per sequence: B * nq queries, at most nq * total_rows scores.
DecodePlan plan_decode(int B, int64_t total_rows, int H, int D, int top_k, bool paged = false,
                       int nq = 1) {
  DecodePlan p{};
  const size_t nqry = static_cast<size_t>(B) * nq;
  const size_t nscore = static_cast<size_t>(total_rows) * nq;
  size_t o = 0;
  p.off_counters = o;
  o = align_up(o + 64 * sizeof(int));
  p.off_hist = o;   // right after the counters: one memset clears both
  o = align_up(o + nqry * 2048 * sizeof(unsigned int));
  p.off_scores = o;
  o = align_up(o + nscore * sizeof(float));
  p.off_keys = o;
  o = align_up(o + nscore * sizeof(unsigned long long));
  p.off_indices = o;
  o = align_up(o + nqry * top_k * sizeof(int32_t));
  p.off_part = o;
  o = align_up(o + nqry * kDecodeSplits * H * (D + 2) * sizeof(float));
  if (paged) {
    p.off_seq = o;
    o = align_up(o + static_cast<size_t>(B + 1) * sizeof(int64_t));
  }
  p.total = o;
  return p;
}

// ---- stage timing (diagnostic) -------------------------------------------------------

struct StageRec {
  cudaEvent_t a, b;
  int stage, launches;
};
bool g_timing = false;
std::mutex g_timing_mu;
std::vector<StageRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;
double g_ms[DSA_NUM_STAGES];
int64_t g_launches[DSA_NUM_STAGES];

cudaEvent_t pooled_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Records an event on `s` at construction and at destruction (when enabled).
class StageScope {
 public:
  StageScope(int stage, int launches, cudaStream_t s) : stage_(stage), launches_(launches), s_(s) {
    if (!g_timing) return;
    std::lock_guard<std::mutex> g(g_timing_mu);
    a_ = pooled_event();
    if (a_) cudaEventRecord(a_, s_);
  }
  ~StageScope() {
    if (!g_timing || !a_) return;
    std::lock_guard<std::mutex> g(g_timing_mu);
    cudaEvent_t b = pooled_event();
    if (!b) return;
    cudaEventRecord(b, s_);
    g_recs.push_back({a_, b, stage_, launches_});
  }

 private:
  int stage_, launches_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr;
};

__global__ void wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, limit_ns, nullptr);  // nothing arrives
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(smem_u32(&bar));  // leave the barrier complete
}

constexpr int64_t kMaxDecodeLen = (int64_t(1) << 31) - 1;
constexpr int kMaxDecodeBatch = 65535;  // sequences are the scan grid's y extent
constexpr int kMaxBlockSize = 1 << 16;

// One decode call: a contiguous cache (seq_start) or a paged one (seq_lens,
// block_table); the entry points check what is particular to each.
struct DecodeCall {
  const void* k_idx;
  const void* K;
  const void* V;
  const int64_t* seq_start;      // contiguous cache, else null
  const int32_t* seq_lens;       // paged cache, else null
  const int32_t* block_table;
  int bt_ld, bs_log2;
  int64_t num_blocks;
  int B;
  int nq;                        // new tokens per sequence (the last nq rows of each)
  int64_t total_rows;            // rows the workspace is planned for
  int64_t max_len;
  int idx_dtype, d_idx, D;
  const void* q_idx;
  const void* Q;
  int H, top_k;
  float idx_scale, attn_scale;
  void* O;
  int32_t* indices;
  void* workspace;
  size_t workspace_bytes;
  cudaStream_t stream;
};

dsa_status run_decode(const DecodeCall& c) {
  const bool paged = c.seq_lens != nullptr;
  if (!c.k_idx || !c.K || !c.V || !c.q_idx || !c.Q || !c.O || !c.workspace)
    return DSA_ERR_INVALID_ARG;
  for (const void* ptr : {c.k_idx, c.K, c.V, c.q_idx, c.Q, static_cast<const void*>(c.O)})
    if (!aligned16(ptr)) return DSA_ERR_INVALID_ARG;
  if (c.indices && !aligned16(c.indices)) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(c.workspace) & 255) != 0) return DSA_ERR_INVALID_ARG;
  if (c.B < 1 || c.B > kMaxDecodeBatch || c.max_len < 1 || c.max_len > kMaxDecodeLen)
    return DSA_ERR_INVALID_ARG;
  if (c.top_k < 1 || c.top_k > DSA_MAX_TOP_K) return DSA_ERR_INVALID_ARG;
  if (c.H < 1 || c.H > DSA_MAX_HEADS) return DSA_ERR_INVALID_ARG;
  if (c.D != 64 && c.D != 128) return DSA_ERR_UNSUPPORTED;
  dsa_status st = check_index_dims(c.idx_dtype, c.d_idx);
  if (st != DSA_OK) return st;
  if (c.nq < 1 || c.nq > 4 || static_cast<int64_t>(c.B) * c.nq > kMaxDecodeBatch) return DSA_ERR_INVALID_ARG;
  if (!decode_nq_supported(c.nq, esize_of(c.idx_dtype), c.d_idx)) return DSA_ERR_UNSUPPORTED;
  const DecodePlan plan = plan_decode(c.B, c.total_rows, c.H, c.D, c.top_k, paged, c.nq);
  if (c.workspace_bytes < plan.total) return DSA_ERR_WORKSPACE;
  cudaStream_t s = c.stream;
  uint8_t* ws = static_cast<uint8_t*>(c.workspace);
  int32_t* idx = c.indices ? c.indices : reinterpret_cast<int32_t*>(ws + plan.off_indices);
  const size_t cleared = plan.off_hist + static_cast<size_t>(c.B) * c.nq * 2048 * sizeof(unsigned int);
  if (cudaMemsetAsync(ws + plan.off_counters, 0, cleared - plan.off_counters, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  int64_t* seq_ws = paged ? reinterpret_cast<int64_t*>(ws + plan.off_seq) : nullptr;
  const int64_t* seq_start = paged ? seq_ws : c.seq_start;

  DecodeLaunch dl{};
  dl.k_idx = c.k_idx;
  dl.q_idx = c.q_idx;
  dl.esize = esize_of(c.idx_dtype);
  dl.d = c.d_idx;
  dl.seq_start = seq_start;
  dl.B = c.B;
  dl.total_rows = c.total_rows;
  dl.max_len = c.max_len;
  dl.scale = default_scale(c.idx_scale, c.d_idx);
  dl.top_k = c.top_k;
  dl.scores = reinterpret_cast<float*>(ws + plan.off_scores);
  dl.hist = reinterpret_cast<unsigned int*>(ws + plan.off_hist);
  dl.indices = idx;
  dl.keys = reinterpret_cast<unsigned long long*>(ws + plan.off_keys);
  dl.invalid = reinterpret_cast<int*>(ws + plan.off_counters) + 8;
  dl.seq_lens = c.seq_lens;
  dl.block_table = c.block_table;
  dl.bt_ld = c.bt_ld;
  dl.bs_log2 = c.bs_log2;
  dl.num_blocks = c.num_blocks;
  dl.seq_start_out = seq_ws;
  dl.nq = c.nq;
  {
    StageScope scope(5, 3, s);  // validate + scan + select (timed together)
    if ((st = launch_decode_select(dl, s)) != DSA_OK) return st;
  }

  AttnLaunch at{};
  at.Q = static_cast<const __nv_bfloat16*>(c.Q);
  at.K = static_cast<const __nv_bfloat16*>(c.K);
  at.V = static_cast<const __nv_bfloat16*>(c.V);
  at.kv_rows = paged ? c.num_blocks << c.bs_log2 : c.total_rows;
  at.idx = idx;
  at.ld_idx = c.top_k;
  at.nq = static_cast<int64_t>(c.B) * c.nq;
  at.qpt = c.nq;
  at.H = c.H;
  at.D = c.D;
  at.scale_log2 = default_scale(c.attn_scale, c.D) * 1.4426950408889634f;
  at.top_k = c.top_k;
  at.seq_start = seq_start;
  at.nsplit = decode_splits(c.B * c.nq);
  at.O = static_cast<__nv_bfloat16*>(c.O);
  at.part = reinterpret_cast<float*>(ws + plan.off_part);
  at.invalid = dl.invalid;
  at.block_table = c.block_table;
  at.bt_ld = c.bt_ld;
  at.bs_log2 = c.bs_log2;
  StageScope scope(7, 2, s);
  return launch_attention(at, s);
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

uint64_t wait_limit_ns() { return 2000000000ull; }  // 2 s per wait

}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA runtime error";
    case DSA_ERR_TIMEOUT: return "device-side wait timed out";
    case DSA_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

const char* dsa_version(void) { return "0.1.0"; }

dsa_status dsa_indexer_scores(const void* q_idx, const void* k_idx, int idx_dtype, int d_idx,
                              float idx_scale, int64_t Lq, int64_t Lk, float* scores,
                              void* stream) {
  if (!q_idx || !k_idx || !scores || Lq < 1 || Lk < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (Lq > (int64_t(1) << 31) - 1 || Lk > (int64_t(1) << 31) - 1) return DSA_ERR_UNSUPPORTED;
  dsa_status st = check_index_dims(idx_dtype, d_idx);
  if (st != DSA_OK) return st;
  IndexerLaunch a{};
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.esize = esize_of(idx_dtype);
  a.d = d_idx;
  a.Lq = Lq;
  a.Lk = Lk;
  a.scale = default_scale(idx_scale, d_idx);
  a.mode = kModeDense;
  a.scores = scores;
  a.limit_ns = wait_limit_ns();
  return launch_indexer(a, static_cast<cudaStream_t>(stream));
}

size_t dsa_prefill_workspace_size(int64_t L, int d_idx, int idx_dtype, int H, int D, int top_k) {
  (void)d_idx; (void)idx_dtype; (void)H; (void)D;
  if (L < 1 || top_k < 1) return 0;
  return plan_prefill(L, top_k, L).total;
}

size_t dsa_prefill_chunk_workspace_size(int64_t Lq, int64_t Lk, int d_idx, int idx_dtype, int H,
                                        int D, int top_k) {
  (void)d_idx; (void)idx_dtype; (void)H; (void)D;
  if (Lq < 1 || Lk < Lq || top_k < 1) return 0;
  return plan_prefill(Lq, top_k, Lk).total;
}

dsa_status dsa_prefill(const void* q_idx, const void* k_idx, int idx_dtype, int d_idx,
                       float idx_scale, const void* Q, const void* K, const void* V, int64_t L,
                       int H, int D, float attn_scale, int top_k, int32_t* indices, void* O,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return dsa_prefill_chunk(q_idx, k_idx, idx_dtype, d_idx, idx_scale, Q, K, V, L, L, H, D,
                           attn_scale, top_k, indices, O, workspace, workspace_bytes, stream);
}

dsa_status dsa_prefill_chunk(const void* q_idx, const void* k_idx, int idx_dtype, int d_idx,
                             float idx_scale, const void* Q, const void* K, const void* V,
                             int64_t Lq, int64_t Lk, int H, int D, float attn_scale, int top_k,
                             int32_t* indices, void* O, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!q_idx || !k_idx || !Q || !K || !V || !indices || !O || !workspace) return DSA_ERR_INVALID_ARG;
  for (const void* ptr : {q_idx, k_idx, Q, K, V, static_cast<const void*>(indices),
                          static_cast<const void*>(O)})
    if (!aligned16(ptr)) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return DSA_ERR_INVALID_ARG;
  if (Lq < 1 || Lk < Lq || Lk > (int64_t(1) << 31) - 1) return DSA_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > DSA_MAX_TOP_K) return DSA_ERR_INVALID_ARG;
  if (H < 1 || H > DSA_MAX_HEADS) return DSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DSA_ERR_UNSUPPORTED;
  dsa_status st = check_index_dims(idx_dtype, d_idx);
  if (st != DSA_OK) return st;
  const int64_t L = Lq;
  const int64_t q0 = Lk - Lq;   // query row t sits at key position q0 + t
  const PrefillPlan plan = plan_prefill(L, top_k, Lk);
  if (workspace_bytes < plan.total) return DSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* counters = reinterpret_cast<int*>(ws + plan.off_counters);
  float* tau = reinterpret_cast<float*>(ws + plan.off_tau);
  int* cand_n = reinterpret_cast<int*>(ws + plan.off_cand_n);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(ws + plan.off_cand);
  uint16_t* samp = reinterpret_cast<uint16_t*>(ws + plan.off_samp);
  int* fb_rows = reinterpret_cast<int*>(ws + plan.off_fb_rows);
  unsigned long long* fb_scratch = reinterpret_cast<unsigned long long*>(ws + plan.off_fb_scratch);
  const int es = esize_of(idx_dtype);
  const float iscale = default_scale(idx_scale, d_idx);
  const float ascale = default_scale(attn_scale, D);

  if (cudaMemsetAsync(counters, 0, 64 * sizeof(int), s) != cudaSuccess) return DSA_ERR_CUDA;

  IndexerLaunch a{};
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.esize = es;
  a.d = d_idx;
  a.Lq = L;
  a.Lk = Lk;
  a.q0 = q0;
  a.scale = iscale;
  a.limit_ns = wait_limit_ns();
  if (Lk > plan.cap_all) {   // some row (the last, at position Lk - 1) needs a threshold
    StageScope scope(0, 1, s);
    a.mode = kModeSample;
    a.samp = samp;
    a.samp_ld = plan.samp_ld;
    a.cap = plan.cap_all;
    if ((st = launch_indexer(a, s)) != DSA_OK) return st;
  }
  {
    StageScope scope(1, 1, s);
    st = launch_tau_select(samp, plan.samp_ld, L, q0, plan.cap_all, plan.target, iscale, tau, s);
    if (st != DSA_OK) return st;
  }
  a.mode = kModeFilter;
  a.tau = tau;
  a.cand = cand;
  a.cand_n = cand_n;
  a.cap = plan.cap_part;
  {
    StageScope scope(2, 1, s);
    if ((st = launch_indexer(a, s)) != DSA_OK) return st;
  }

  SelectLaunch sl{};
  sl.L = L;
  sl.q0 = q0;
  sl.Lk = Lk;
  sl.top_k = top_k;
  sl.cap = plan.cap_part;
  sl.cand = cand;
  sl.cand_n = cand_n;
  sl.tau = tau;
  sl.indices = indices;
  sl.fb_rows = fb_rows;
  sl.counters = counters;
  sl.q_idx = q_idx;
  sl.k_idx = k_idx;
  sl.esize = es;
  sl.d = d_idx;
  sl.scale = iscale;
  sl.fb_scratch = fb_scratch;
  sl.fb_hist = reinterpret_cast<unsigned int*>(ws + plan.off_fb_hist);
  sl.fb_slow = reinterpret_cast<int*>(ws + plan.off_fb_slow);
  sl.big_rows = reinterpret_cast<int*>(ws + plan.off_big_rows);
  sl.fb_ctas = plan.fb_ctas;
  sl.force_fb_period = g_force_fb_period.load();
  {
    StageScope scope(3, 5, s);
    if ((st = launch_select(sl, s)) != DSA_OK) return st;
  }

  AttnLaunch at{};
  at.Q = static_cast<const __nv_bfloat16*>(Q);
  at.K = static_cast<const __nv_bfloat16*>(K);
  at.V = static_cast<const __nv_bfloat16*>(V);
  at.kv_rows = Lk;
  at.q0 = q0;
  at.idx = indices;
  at.ld_idx = top_k;
  at.nq = L;
  at.H = H;
  at.D = D;
  at.scale_log2 = ascale * 1.4426950408889634f;
  at.top_k = top_k;
  at.seq_start = nullptr;
  at.nsplit = 1;
  at.O = static_cast<__nv_bfloat16*>(O);
  StageScope scope(4, 1, s);
  return launch_attention(at, s);
}

size_t dsa_decode_workspace_size(int B, int64_t total_rows, int d_idx, int idx_dtype, int H,
                                 int D, int top_k) {
  return dsa_decode_multi_workspace_size(B, 1, total_rows, d_idx, idx_dtype, H, D, top_k);
}

size_t dsa_decode_multi_workspace_size(int B, int T, int64_t total_rows, int d_idx, int idx_dtype,
                                       int H, int D, int top_k) {
  (void)d_idx; (void)idx_dtype;
  if (B < 1 || T < 1 || T > 4 || total_rows < 1 || H < 1 || top_k < 1) return 0;
  return plan_decode(B, total_rows, H, D, top_k, false, T).total;
}

dsa_status dsa_decode(const void* k_idx, const void* K, const void* V, const int64_t* seq_start,
                      int B, int64_t total_rows, int64_t max_len, int idx_dtype, int d_idx, int D,
                      const void* q_idx, const void* Q, int H, int top_k, float idx_scale,
                      float attn_scale, void* O, int32_t* indices, void* workspace,
                      size_t workspace_bytes, void* stream) {
  return dsa_decode_multi(k_idx, K, V, seq_start, B, 1, total_rows, max_len, idx_dtype, d_idx, D,
                          q_idx, Q, H, top_k, idx_scale, attn_scale, O, indices, workspace,
                          workspace_bytes, stream);
}

dsa_status dsa_decode_multi(const void* k_idx, const void* K, const void* V,
                            const int64_t* seq_start, int B, int T, int64_t total_rows,
                            int64_t max_len, int idx_dtype, int d_idx, int D, const void* q_idx,
                            const void* Q, int H, int top_k, float idx_scale, float attn_scale,
                            void* O, int32_t* indices, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!seq_start || (reinterpret_cast<uintptr_t>(seq_start) & 7) != 0 || total_rows < 1)
    return DSA_ERR_INVALID_ARG;
  DecodeCall c{};
  c.k_idx = k_idx;
  c.K = K;
  c.V = V;
  c.seq_start = seq_start;
  c.B = B;
  c.nq = T;
  c.total_rows = total_rows;
  c.max_len = max_len;
  c.idx_dtype = idx_dtype;
  c.d_idx = d_idx;
  c.D = D;
  c.q_idx = q_idx;
  c.Q = Q;
  c.H = H;
  c.top_k = top_k;
  c.idx_scale = idx_scale;
  c.attn_scale = attn_scale;
  c.O = O;
  c.indices = indices;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  c.stream = static_cast<cudaStream_t>(stream);
  return run_decode(c);
}

size_t dsa_decode_paged_workspace_size(int B, int64_t max_len, int d_idx, int idx_dtype, int H,
                                       int D, int top_k) {
  return dsa_decode_paged_multi_workspace_size(B, 1, max_len, d_idx, idx_dtype, H, D, top_k);
}

size_t dsa_decode_paged_multi_workspace_size(int B, int T, int64_t max_len, int d_idx,
                                             int idx_dtype, int H, int D, int top_k) {
  (void)d_idx; (void)idx_dtype;
  if (B < 1 || T < 1 || T > 4 || max_len < 1 || max_len > kMaxDecodeLen || H < 1 || top_k < 1)
    return 0;
  return plan_decode(B, static_cast<int64_t>(B) * max_len, H, D, top_k, true, T).total;
}

dsa_status dsa_decode_paged(const void* k_idx, const void* K, const void* V, int64_t num_blocks,
                            int block_size, const int32_t* block_table, int max_blocks,
                            const int32_t* seq_lens, int B, int64_t max_len, int idx_dtype,
                            int d_idx, int D, const void* q_idx, const void* Q, int H, int top_k,
                            float idx_scale, float attn_scale, void* O, int32_t* indices,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return dsa_decode_paged_multi(k_idx, K, V, num_blocks, block_size, block_table, max_blocks,
                                seq_lens, B, 1, max_len, idx_dtype, d_idx, D, q_idx, Q, H, top_k,
                                idx_scale, attn_scale, O, indices, workspace, workspace_bytes,
                                stream);
}

dsa_status dsa_decode_paged_multi(const void* k_idx, const void* K, const void* V,
                                  int64_t num_blocks, int block_size, const int32_t* block_table,
                                  int max_blocks, const int32_t* seq_lens, int B, int T,
                                  int64_t max_len, int idx_dtype, int d_idx, int D,
                                  const void* q_idx, const void* Q, int H, int top_k,
                                  float idx_scale, float attn_scale, void* O, int32_t* indices,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!block_table || !seq_lens || (reinterpret_cast<uintptr_t>(block_table) & 3) != 0 ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3) != 0)
    return DSA_ERR_INVALID_ARG;
  if (block_size < 1 || block_size > kMaxBlockSize || (block_size & (block_size - 1)) != 0)
    return DSA_ERR_INVALID_ARG;
  if (num_blocks < 1 || num_blocks > INT32_MAX / block_size || max_blocks < 1 || B < 1 ||
      max_len < 1 || max_len > kMaxDecodeLen)
    return DSA_ERR_INVALID_ARG;
  DecodeCall c{};
  c.k_idx = k_idx;
  c.K = K;
  c.V = V;
  c.seq_lens = seq_lens;
  c.block_table = block_table;
  c.bt_ld = max_blocks;
  int lg = 0;
  while ((1 << lg) < block_size) ++lg;
  c.bs_log2 = lg;
  c.num_blocks = num_blocks;
  c.B = B;
  c.nq = T;
  c.total_rows = static_cast<int64_t>(B) * max_len;
  c.max_len = max_len;
  c.idx_dtype = idx_dtype;
  c.d_idx = d_idx;
  c.D = D;
  c.q_idx = q_idx;
  c.Q = Q;
  c.H = H;
  c.top_k = top_k;
  c.idx_scale = idx_scale;
  c.attn_scale = attn_scale;
  c.O = O;
  c.indices = indices;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  c.stream = static_cast<cudaStream_t>(stream);
  return run_decode(c);
}

dsa_status dsa_sync_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return DSA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess)
    return DSA_ERR_CUDA;
  return static_cast<dsa_status>(v);
}

dsa_status dsa_last_stats(const void* workspace, int64_t out[4], void* stream) {
  if (!workspace || !out) return DSA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  int c[4] = {0, 0, 0, 0};
  if (cudaMemcpy(c, workspace, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  for (int i = 0; i < 4; ++i) out[i] = c[i];
  return DSA_OK;
}

dsa_status dsa_stage_timing(int enable) {
  std::lock_guard<std::mutex> g(g_timing_mu);
  g_timing = enable != 0;
  return DSA_OK;
}

dsa_status dsa_stage_times(double* ms, int64_t* launches, int n) {
  if (n < 0 || n > DSA_NUM_STAGES) return DSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(g_timing_mu);
  dsa_status st = DSA_OK;
  for (const StageRec& r : g_recs) {
    float t = 0.0f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = DSA_ERR_CUDA;
    g_ms[r.stage] += t;
    g_launches[r.stage] += r.launches;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_recs.clear();
  for (int i = 0; i < n; ++i) {
    if (ms) ms[i] = g_ms[i];
    if (launches) launches[i] = g_launches[i];
  }
  for (int i = 0; i < DSA_NUM_STAGES; ++i) {
    g_ms[i] = 0.0;
    g_launches[i] = 0;
  }
  return st;
}

dsa_status dsa_debug_force_fallback(int period) {
  if (period < 0) return DSA_ERR_INVALID_ARG;
  dsa::g_force_fb_period.store(period);
  return DSA_OK;
}

dsa_status dsa_debug_wait_timeout(uint64_t limit_ns, void* stream) {
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // extern "C"

// ---- decode without allocation --------------------------------------------------------
//
// Scratch for dsa_decode_static: one block per device, in the library's own
// device memory, so callers that may not allocate need no workspace.  Host
// code cannot use the symbol's name as a device address; each device's
// address is looked up once with cudaGetSymbolAddress while that device is
// current.

namespace {

static __device__ __align__(256) unsigned char g_decode_static_scratch[DSA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_scratch[kMaxDevices] = {};

}  // namespace

extern "C" dsa_status dsa_decode_static(const void* k_idx, const void* K, const void* V,
                                        const int64_t* seq_start, int B, int64_t total_rows,
                                        int64_t max_len, int idx_dtype, int d_idx, int D,
                                        const void* q_idx, const void* Q, int H, int top_k,
                                        float idx_scale, float attn_scale, void* O,
                                        int32_t* indices, void* stream) {
  const size_t need = dsa_decode_workspace_size(B, total_rows, d_idx, idx_dtype, H, D, top_k);
  if (need == 0) return DSA_ERR_INVALID_ARG;
  if (need > DSA_DECODE_STATIC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  // The block's address is only valid on the device it was looked up for: the
  // output must live on the current device.
  if (O) {
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, O) != cudaSuccess) {
      cudaGetLastError();
      return DSA_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice || attr.device != dev) return DSA_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> g(g_static_mu);
    if (!g_static_scratch[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_decode_static_scratch) != cudaSuccess || !ptr)
        return DSA_ERR_CUDA;
      g_static_scratch[dev] = ptr;
    }
    scratch = g_static_scratch[dev];
  }
  return dsa_decode(k_idx, K, V, seq_start, B, total_rows, max_len, idx_dtype, d_idx, D, q_idx, Q,
                    H, top_k, idx_scale, attn_scale, O, indices, scratch,
                    DSA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
