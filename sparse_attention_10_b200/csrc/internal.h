// Host-side declarations shared by the DSA translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// ---- indexer (tcgen05) -------------------------------------------------------

enum IndexerMode { kModeDense = 0, kModeSample = 1, kModeFilter = 2 };

constexpr int kBM = 128;          // query rows per tile = TMEM lanes
constexpr int kBN = 256;          // keys per tile = TMEM columns per accumulator
constexpr int kSampTilesMax = 16; // key tiles sampled per query tile for the threshold
constexpr int kCandParts = 2;     // candidate lists per query row: one per column part of a tile

struct IndexerLaunch {
  const void* q_idx;
  const void* k_idx;
  int esize;          // 1 = FP8 E4M3, 2 = BF16
  int d;              // index dim (elements)
  int64_t Lq, Lk;
  int64_t q0;         // causal modes: query row i sits at key position q0 + i
  float scale;
  int mode;
  // filter
  const float* tau;
  unsigned long long* cand;
  int* cand_n;
  int cap;
  // sample
  uint16_t* samp;
  int samp_ld;
  // dense
  float* scores;
  uint64_t limit_ns;
};

dsa_status launch_indexer(const IndexerLaunch& a, cudaStream_t stream);

// Threshold per query row from the sampled scores (raw accumulator domain).
dsa_status launch_tau_select(const uint16_t* samp, int samp_ld, int64_t L, int64_t q0, int cap,
                             int target, float scale, float* tau, cudaStream_t stream);

// ---- select -------------------------------------------------------------------

struct SelectLaunch {
  int64_t L;             // query rows
  int64_t q0;            // query row t sits at key position q0 + t
  int64_t Lk;            // key rows (q0 + L)
  int top_k;
  int cap;
  const unsigned long long* cand;
  const int* cand_n;
  const float* tau;      // per-row threshold (zero-mode rows are marked by its bits)
  int32_t* indices;
  int* fb_rows;          // [L] rows that need the exact fallback
  int force_fb_period;   // > 0: rows t % period == 0 go to the fallback (test hook)
  int* counters;         // [0] fallback rows, [1] overflow rows, [2] candidates,
                         // [3] fallback rows left to the one-CTA path, [4] big rows
  int* big_rows;         // [L] rows whose candidates need the large select shape
  // fallback inputs
  const void* q_idx;
  const void* k_idx;
  int esize, d;
  float scale;
  unsigned long long* fb_scratch;  // [fb_ctas, Lk]
  unsigned int* fb_hist;           // [fb_ctas, 4096]
  int* fb_slow;                    // [fb_ctas]
  int fb_ctas;                     // fallback rows handled by the grid-wide path
};

dsa_status launch_select(const SelectLaunch& a, cudaStream_t stream);

// ---- attention ---------------------------------------------------------------

struct AttnLaunch {
  const __nv_bfloat16* Q;      // [nq, H, D]
  const __nv_bfloat16* K;      // [rows, D]
  const __nv_bfloat16* V;
  int64_t kv_rows;             // rows of K and V
  const int32_t* idx;          // [nq, ld_idx]
  int ld_idx;
  int64_t nq;
  int H, D;
  float scale_log2;            // softmax scale * log2(e)
  int top_k;
  // prefill: count(q) = min(top_k, q0 + q + 1), row base 0
  // decode:  count(q) = min(top_k, len_q), row base seq_start[q]
  const int64_t* seq_start;    // null for prefill
  int nsplit;                  // splits of the key list per query (1 = final output)
  __nv_bfloat16* O;            // [nq, H, D] (nsplit == 1)
  float* part;                 // [nq, nsplit, H, D + 2] (nsplit > 1)
  const int* invalid;          // nonzero: skip all work (decode inputs failed validation)
  // paged decode cache (null: K/V rows of query q start at seq_start[q]): key s of query q
  // is row (block_table[q * bt_ld + (s >> bs_log2)] << bs_log2) | (s & (2^bs_log2 - 1))
  const int32_t* block_table;
  int bt_ld, bs_log2;
  int64_t q0;                  // prefill: query q sits at key position q0 + q (chunked prefill)
  int qpt;                     // decode: queries per sequence (query q belongs to sequence
                               // q / qpt and sees its first len - (qpt - 1 - q % qpt) rows)
};

dsa_status launch_attention(const AttnLaunch& a, cudaStream_t stream);

// tcgen05 attention (head dim 128, up to 16 heads); launch_attention routes
// the shapes it supports there.
bool attention_tc_supported(const AttnLaunch& a);
dsa_status launch_attention_tc(const AttnLaunch& a, cudaStream_t stream);

// ---- decode ------------------------------------------------------------------

struct DecodeLaunch {
  const void* k_idx;
  const void* q_idx;
  int esize, d;
  const int64_t* seq_start;
  int B;
  int64_t total_rows, max_len;
  float scale;
  int top_k;
  float* scores;               // [total_rows]
  unsigned int* hist;          // [B, 2048]
  int32_t* indices;            // [B, top_k]
  unsigned long long* keys;    // [total_rows] scratch (many-candidate rows)
  int* invalid;                // set when seq_start (or the paged inputs) fail validation
  // Paged cache (seq_lens non-null): row s of sequence b is k_idx row
  // (block_table[b * bt_ld + (s >> bs_log2)] << bs_log2) | (s & (2^bs_log2 - 1)).
  // The validator writes the running sum of the lengths into seq_start_out (then
  // seq_start == seq_start_out), so scores and scratch stay indexed by sequence.
  const int32_t* seq_lens;
  const int32_t* block_table;
  int bt_ld, bs_log2;
  int64_t num_blocks;
  int64_t* seq_start_out;
  // nq new tokens per sequence (1 .. 4): query v = b * nq + j sits at position
  // len_b - nq + j; q_idx is [B * nq, d], scores, histograms and indices are
  // per query v (scores of query v from nq * seq_start[b] - b * nq(nq-1)/2 +
  // j (len_b - nq + 1) + j(j-1)/2 on).  nq > 1 needs index rows of 64, 128 or
  // 256 bytes (decode_nq_supported).
  int nq;
};

dsa_status launch_decode_select(const DecodeLaunch& a, cudaStream_t stream);
inline bool decode_nq_supported(int nq, int esize, int d) {
  const int lpr = d * esize / 16;
  if (nq == 1) return true;
  return nq >= 2 && nq <= 4 && (lpr == 4 || lpr == 8 || lpr == 16) && (esize == 1 || lpr != 4);
}

int num_sms();
uint64_t wait_limit_ns();

}  // namespace dsa
