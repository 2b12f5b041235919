/*
 * dsa.h — C ABI of a B200 (sm_100a) implementation of DeepSeek Sparse
 * Attention (DSA): lightning indexer -> per-query top-k -> softmax attention
 * of H query heads over only the kept keys of one MQA-shared K/V.
 *
 * What is computed follows the DeepSeek Sparse Attention page
 * (kwkr.cn/news/60693):
 *   section 3.2  lightning indexer: I = relu(matmul(q_idx, k_idx^T) * scale),
 *                scale = index_dim^-0.5, FP8 inputs in a low index dimension;
 *   section 3.3  fine-grained token selection: each query keeps its top-k
 *                keys, then ordinary softmax attention runs over those keys;
 *   section 4.1  precision: FP8 index stage, BF16 attention stage;
 *   section 4.2  memory: all query heads share one K/V (MQA); rows are laid
 *                out on 128-byte boundaries, the cache in token blocks
 *                (dsa_decode_paged);
 *   section 7.2  per-length settings (FP8 at 32K/64K, BF16 index at 128K).
 * Readings where the page is silent (stated once here, used everywhere):
 *   - causal: query t sees keys s <= t, the diagonal included;
 *   - the indexer score of a pair is fp32(fp32(q.k) * scale), then ReLU maps
 *     every non-positive score (and -0) to +0;
 *   - order: keys are ranked by (score descending, key index ascending), so
 *     ties go to the lower key index; a query keeps min(top_k, t+1) keys;
 *   - indices[t] lists the kept keys in that rank order and pads with -1;
 *   - attention softmax scale defaults to D^-0.5; output is BF16 (nearest).
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers on the current
 *     device; the caller owns every buffer.  No call allocates memory.
 *   - Tensors are dense row-major.  Device pointers must be 16-byte aligned;
 *     128-byte alignment is recommended (row starts then fall on 128 B).
 *   - `stream` is a cudaStream_t passed as void*.  Calls only enqueue work;
 *     they are asynchronous and keep no state between calls, so calls on
 *     distinct workspaces may run concurrently.  No compute call synchronises
 *     with the host (only dsa_sync_status, dsa_last_stats and
 *     dsa_stage_times do), so after one ordinary call with the same shapes
 *     (which loads the kernels) a dsa_prefill* or dsa_decode* call with a
 *     caller's workspace may be captured into a CUDA graph and replayed with
 *     the same pointers and sizes.
 *   - Argument errors are reported synchronously by the return value and
 *     nothing is enqueued.  Errors found on the device (a bounded wait that
 *     ran out; decode lengths or block ids that fail the device-side checks)
 *     are recorded in a per-device status word that dsa_sync_status() reads
 *     and clears.
 *   - idx_scale / attn_scale: pass NaN to use index_dim^-0.5 / D^-0.5
 *     (each rounded to float32).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, size out of range  */
  DSA_ERR_UNSUPPORTED = 2,  /* shape the kernels do not handle              */
  DSA_ERR_WORKSPACE = 3,    /* workspace smaller than *_workspace_size()    */
  DSA_ERR_CUDA = 4,         /* a CUDA runtime call failed                   */
  DSA_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out           */
  DSA_ERR_DEVICE = 6        /* other device-side fault recorded by a kernel */
} dsa_status;

typedef enum {
  DSA_IDX_FP8_E4M3 = 0,     /* OCP FP8 E4M3 bytes                            */
  DSA_IDX_BF16 = 1          /* bfloat16                                      */
} dsa_idx_dtype;

/* Limits of this implementation. */
#define DSA_MAX_TOP_K 2048
#define DSA_MAX_INDEX_DIM 256
#define DSA_MAX_HEADS 16

/* Human-readable name of a status code (static string). */
const char* dsa_status_string(dsa_status s);

/* Library version as "major.minor.patch" (static string). */
const char* dsa_version(void);

/*
 * dsa_indexer_scores — the lightning indexer of section 3.2 exactly as the
 * page's snippet writes it: the dense matrix
 *     scores[t, s] = relu(fp32(q_idx[t] . k_idx[s]) * idx_scale)
 * for t < Lq, s < Lk, with no causal mask and no selection.  Runs on the same
 * tcgen05 tensor-core tiles as dsa_prefill.  Meant for checking and small
 * sizes: it writes Lq*Lk floats.
 *   q_idx   device [Lq, d_idx]   FP8 E4M3 or BF16 (idx_dtype)
 *   k_idx   device [Lk, d_idx]
 *   scores  device [Lq, Lk] float32, written
 * d_idx must be a multiple of 32 bytes of the element type and <= 256.
 * Returns DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED on bad arguments.
 */
dsa_status dsa_indexer_scores(const void* q_idx, const void* k_idx, int idx_dtype, int d_idx,
                              float idx_scale, int64_t Lq, int64_t Lk, float* scores,
                              void* stream);

/* Bytes of device workspace dsa_prefill needs for these sizes. */
size_t dsa_prefill_workspace_size(int64_t L, int d_idx, int idx_dtype, int H, int D, int top_k);

/*
 * dsa_prefill — DSA over one causal sequence of length L (sections 3.1-3.3,
 * 4.1-4.3): indexer scores of every causal pair, per-query top-k, then
 * softmax attention of H heads over the kept keys.  The L x L score matrix
 * is never written to memory.
 *   q_idx, k_idx  device [L, d_idx]  FP8 E4M3 or BF16 (idx_dtype); d_idx a
 *                 multiple of 32 bytes of the element type, <= 256
 *   Q             device [L, H, D] BF16 (query heads)
 *   K, V          device [L, D]    BF16 (one K/V shared by all heads)
 *   indices       device [L, top_k] int32, written: kept keys of query t in
 *                 rank order, -1 padded (t+1 < top_k)
 *   O             device [L, H, D] BF16, written
 *   workspace     device, >= dsa_prefill_workspace_size(...) bytes, 256-byte
 *                 aligned; contents on entry are ignored
 * Limits: 1 <= top_k <= 2048, 1 <= H <= 16, D in {64, 128}, L >= 1.
 */
dsa_status dsa_prefill(const void* q_idx, const void* k_idx, int idx_dtype, int d_idx,
                       float idx_scale, const void* Q, const void* K, const void* V, int64_t L,
                       int H, int D, float attn_scale, int top_k, int32_t* indices, void* O,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace dsa_prefill_chunk needs for Lq queries against Lk keys. */
size_t dsa_prefill_chunk_workspace_size(int64_t Lq, int64_t Lk, int d_idx, int idx_dtype, int H,
                                        int D, int top_k);

/*
 * dsa_prefill_chunk — dsa_prefill for the last Lq positions of a causal
 * sequence of Lk tokens: the same three stages (sections 3.2, 3.3, 4.1-4.2)
 * for query rows that sit at key positions Lk - Lq .. Lk - 1.  Query row i
 * (position p = Lk - Lq + i) sees keys 0 .. p, keeps min(top_k, p + 1) of
 * them, and its indices are key positions.  With Lq = Lk this is
 * dsa_prefill.  It serves chunked prefill (a long prompt in pieces, each
 * chunk against every key before it), several new tokens of one sequence at
 * once (speculative or multi-token decode over a contiguous cache), and a
 * split of one sequence's query rows over GPUs (each GPU runs its chunks
 * against the key prefix they need).
 *   q_idx    device [Lq, d_idx]   index rows of the queries
 *   k_idx    device [Lk, d_idx]   index rows of all keys 0 .. Lk - 1
 *   Q        device [Lq, H, D] BF16;  K, V  device [Lk, D] BF16
 *   indices  device [Lq, top_k] int32, written (-1 padded)
 *   O        device [Lq, H, D] BF16, written
 *   workspace >= dsa_prefill_chunk_workspace_size(Lq, Lk, ...) bytes
 * Limits as dsa_prefill, and 1 <= Lq <= Lk.
 */
dsa_status dsa_prefill_chunk(const void* q_idx, const void* k_idx, int idx_dtype, int d_idx,
                             float idx_scale, const void* Q, const void* K, const void* V,
                             int64_t Lq, int64_t Lk, int H, int D, float attn_scale, int top_k,
                             int32_t* indices, void* O, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Bytes of device workspace dsa_decode needs.  total_rows = sum of lengths. */
size_t dsa_decode_workspace_size(int B, int64_t total_rows, int d_idx, int idx_dtype, int H,
                                 int D, int top_k);

/*
 * dsa_decode — one decode step for a batch of B cached sequences (the same
 * three stages as dsa_prefill for one new query per sequence; the indexer
 * scan streams the cache, section 4.2).  The cache is ragged and contiguous
 * per sequence: rows seq_start[b] .. seq_start[b+1]-1 belong to sequence b.
 * The new token's rows are already in the cache, so the query of sequence b
 * sits at position len_b - 1 and sees all len_b rows.
 *   k_idx      device [total_rows, d_idx] FP8 E4M3 or BF16
 *   K, V       device [total_rows, D] BF16
 *   seq_start  device [B+1] int64, nondecreasing, seq_start[0] = 0,
 *              seq_start[B] = total_rows; every length >= 1
 *   q_idx      device [B, d_idx];  Q device [B, H, D] BF16
 *   O          device [B, H, D] BF16, written
 *   indices    device [B, top_k] int32, written when non-null (rank order,
 *              -1 padded), positions relative to the sequence's first row
 *   max_len    host bound on every len_b (sizes the scan grid)
 * Limits as dsa_prefill; 1 <= B <= 65535, max_len <= 2^31 - 1.
 */
dsa_status dsa_decode(const void* k_idx, const void* K, const void* V, const int64_t* seq_start,
                      int B, int64_t total_rows, int64_t max_len, int idx_dtype, int d_idx, int D,
                      const void* q_idx, const void* Q, int H, int top_k, float idx_scale,
                      float attn_scale, void* O, int32_t* indices, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Bytes of device workspace dsa_decode_paged needs (planned for B * max_len rows). */
size_t dsa_decode_paged_workspace_size(int B, int64_t max_len, int d_idx, int idx_dtype, int H,
                                       int D, int top_k);

/*
 * dsa_decode_paged — dsa_decode over a block-paged cache.  The DeepSeek
 * Sparse Attention page (section 4.2) keeps the cache in token blocks laid
 * out on 128-byte boundaries; read here as pools of fixed-size blocks and a
 * per-sequence block table, so a sequence grows by appending a block and
 * blocks need not be contiguous or in order (several sequences may share
 * one).  Row s of sequence b (0 <= s < seq_lens[b]) is row
 * s % block_size of block block_table[b * max_blocks + s / block_size].
 *   k_idx        device [num_blocks, block_size, d_idx] FP8 E4M3 or BF16
 *   K, V         device [num_blocks, block_size, D] BF16
 *   block_table  device [B, max_blocks] int32; entries past a sequence's
 *                last block are not read
 *   seq_lens     device [B] int32, each in [1, max_len] and at most
 *                max_blocks * block_size
 *   block_size   a power of two in [1, 65536];
 *                num_blocks * block_size <= 2^31 - 1
 *   max_len      host bound on every seq_lens[b] (sizes the scan grid and
 *                the workspace: dsa_decode_paged_workspace_size)
 * Every other argument, output and limit is that of dsa_decode; indices are
 * positions within the sequence (0 .. len_b - 1), not pool rows.  The
 * device checks the lengths and every block id a sequence reaches
 * (0 <= id < num_blocks) before any kernel reads through the table; a
 * failure makes the call a no-op that records DSA_ERR_INVALID_ARG in the
 * status word (dsa_sync_status).  Host-side argument errors return
 * DSA_ERR_INVALID_ARG at once and enqueue nothing.
 */
dsa_status dsa_decode_paged(const void* k_idx, const void* K, const void* V, int64_t num_blocks,
                            int block_size, const int32_t* block_table, int max_blocks,
                            const int32_t* seq_lens, int B, int64_t max_len, int idx_dtype,
                            int d_idx, int D, const void* q_idx, const void* Q, int H, int top_k,
                            float idx_scale, float attn_scale, void* O, int32_t* indices,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace dsa_decode_multi needs (T new tokens per sequence). */
size_t dsa_decode_multi_workspace_size(int B, int T, int64_t total_rows, int d_idx, int idx_dtype,
                                       int H, int D, int top_k);

/*
 * dsa_decode_multi — dsa_decode with T new tokens per sequence (1 <= T <= 4):
 * speculative drafts, or a short chunk of prompt appended to each sequence.
 * The T tokens' rows are the last T rows of each sequence in the cache; token
 * j (0-based) of sequence b sits at position len_b - T + j and sees rows
 * 0 .. len_b - T + j (causal among the new tokens too), as sections 3.2-3.3
 * define for any query.  The index cache is read once for all T tokens.
 *   q_idx    device [B, T, d_idx];  Q device [B, T, H, D] BF16
 *   O        device [B, T, H, D] BF16, written
 *   indices  device [B, T, top_k] int32, written when non-null (positions
 *            within the sequence, -1 padded)
 * Every other argument is that of dsa_decode; every length must be >= T.
 * T > 1 needs index rows of 64, 128 or 256 bytes (FP8 d 64/128/256, BF16 d
 * 64/128); other shapes return DSA_ERR_UNSUPPORTED.  T = 1 is dsa_decode.
 */
dsa_status dsa_decode_multi(const void* k_idx, const void* K, const void* V,
                            const int64_t* seq_start, int B, int T, int64_t total_rows,
                            int64_t max_len, int idx_dtype, int d_idx, int D, const void* q_idx,
                            const void* Q, int H, int top_k, float idx_scale, float attn_scale,
                            void* O, int32_t* indices, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Bytes of device workspace dsa_decode_paged_multi needs. */
size_t dsa_decode_paged_multi_workspace_size(int B, int T, int64_t max_len, int d_idx,
                                             int idx_dtype, int H, int D, int top_k);

/*
 * dsa_decode_paged_multi — dsa_decode_multi over a block-paged cache: the
 * layout, block table and checks of dsa_decode_paged, T new tokens per
 * sequence as in dsa_decode_multi (seq_lens[b] counts them; each >= T).
 */
dsa_status dsa_decode_paged_multi(const void* k_idx, const void* K, const void* V,
                                  int64_t num_blocks, int block_size, const int32_t* block_table,
                                  int max_blocks, const int32_t* seq_lens, int B, int T,
                                  int64_t max_len, int idx_dtype, int d_idx, int D,
                                  const void* q_idx, const void* Q, int H, int top_k,
                                  float idx_scale, float attn_scale, void* O, int32_t* indices,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * dsa_sync_status — synchronise `stream`, then read and clear the current
 * device's status word (the first device-side error since the last read).
 * Returns DSA_OK when no kernel recorded an error, DSA_ERR_CUDA when the
 * synchronisation itself failed.
 */
dsa_status dsa_sync_status(void* stream);

/*
 * dsa_last_stats — host copy of counters the last dsa_prefill/dsa_decode
 * call left in `workspace` (synchronises `stream`):
 *   out[0] rows that took the exact fallback select, out[1] rows whose
 *   candidate list overflowed, out[2] total candidates emitted.
 * Diagnostic only.
 */
dsa_status dsa_last_stats(const void* workspace, int64_t out[4], void* stream);

/*
 * Stage timing (diagnostic).  While enabled (per process), dsa_prefill and
 * dsa_decode record a CUDA event before and after each of their stages on
 * the call's stream.  dsa_stage_times synchronises those events, writes the
 * summed time in milliseconds and the number of kernel launches of each stage
 * into ms[i] / launches[i] for i < n (n <= DSA_NUM_STAGES), and resets them.
 * Stages: 0 indexer sample, 1 threshold, 2 indexer filter, 3 select +
 * fallback, 4 attention, 5 decode scan, 6 decode select, 7 decode attention
 * + combine (stage 5 covers the whole decode scan and select; stage 6 is
 * unused).  Events are created on demand and kept for reuse.
 */
#define DSA_NUM_STAGES 8
dsa_status dsa_stage_timing(int enable);
dsa_status dsa_stage_times(double* ms, int64_t* launches, int n);

/*
 * dsa_debug_wait_timeout — runs one tiny kernel whose only work is a
 * bounded wait on a shared-memory barrier that nothing completes, with a
 * limit of `limit_ns` nanoseconds.  The kernel records DSA_ERR_TIMEOUT in the
 * status word and returns normally, so the context stays usable.  Exists to
 * test the timeout path without hanging or faulting a GPU.
 */
dsa_status dsa_debug_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * dsa_debug_force_fallback — test hook for the exact fallback of the select
 * stage.  With period > 0, every later dsa_prefill call sends each query row
 * t with t % period == 0 to the fallback (scores recomputed for the whole
 * row and selected exactly), whatever its candidate list holds; period = 0
 * restores the normal behaviour.  The results are the same either way; only
 * the path and the time differ.  Process-wide setting, not thread-safe.
 * Returns DSA_ERR_INVALID_ARG for period < 0.
 */
dsa_status dsa_debug_force_fallback(int period);

/*
 * dsa_index_to_fp8 — lossless FP8 copy of BF16 indexer inputs.  Section 7.2
 * of the page runs the 128K indexer in BF16 and section 4.1 the index stage
 * in FP8; when every BF16 value is exactly an FP8 E4M3 value (small integers,
 * for instance), the E4M3 copy gives bit-identical indexer scores, so
 * dsa_prefill can take it (idx_dtype FP8) and run the indexer on the FP8
 * tensor-core path.  Writes out_fp8[i] = E4M3(in_bf16[i]) (round to nearest,
 * saturating) and counts in *inexact the values whose copy differs from the
 * input (NaN included).  Use the copy only when *inexact == 0 (read it after
 * synchronising the stream); the count is reset by the call.
 *   in_bf16  device [n] BF16, 16-byte aligned
 *   out_fp8  device [n] bytes, 8-byte aligned, written
 *   inexact  device uint64, written
 * n must be a positive multiple of 8 (any index dim of 16 or more does).
 */
dsa_status dsa_index_to_fp8(const void* in_bf16, int64_t n, void* out_fp8, uint64_t* inexact,
                            void* stream);

/*
 * dsa_gather_probe — diagnostic: the memory ceiling of the attention's
 * gather.  The attention of section 3.3 reads, for each query, the K and V
 * rows of its kept keys (section 4.2: one K/V shared by every head), random
 * rows that mostly hit in L2.  This call copies, for every query row t < L,
 * the rows indices[t, 0 : min(t + 1, top_k)] of K and then of V into a
 * shared-memory ring (16-byte asynchronous copies, stages of 16 KB) and does
 * nothing else with them, on num_SMs * ctas_per_sm CTAs of 128 threads with
 * `stages` stages each.  Timing it gives the rate at which this device
 * gathers exactly the attention's rows.
 *   indices  device [L, top_k] int32 (a dsa_prefill output); ids outside
 *            [0, L) read row 0
 *   K, V     device [L, D] BF16, D in {64, 128}, 16-byte aligned
 *   sink     device, 8 bytes, may be written (keeps the loads live)
 * ctas_per_sm in [1, 8]; stages in {2, 3, 4, 6}.
 */
dsa_status dsa_gather_probe(const int32_t* indices, int64_t L, int top_k, const void* K,
                            const void* V, int D, int ctas_per_sm, int stages, uint64_t* sink,
                            void* stream);

/*
 * dsa_decode_static — dsa_decode for callers that cannot allocate device
 * memory: a plugin whose host application owns every device allocation, or
 * a serving loop that must not call cudaMalloc (it can synchronise the device
 * and stall other streams) once it is running.  The pages describe no such
 * entry point; it has no counterpart there.
 *
 * Arguments, outputs and errors are those of dsa_decode without the
 * workspace: the scratch comes from one block of device memory built into
 * the library (DSA_DECODE_STATIC_SCRATCH_BYTES = 18 MiB per device, held by
 * every device that loads the library until the process exits).  That is
 * enough for B <= 64 sequences holding up to 2^20 cached rows in total, with
 * H <= 16, D <= 128, top_k <= 2048; sizes whose workspace
 * (dsa_decode_workspace_size) exceeds it return DSA_ERR_WORKSPACE and enqueue
 * nothing.  The caller still owns and passes every input and output.
 *
 * The first call on a device looks up that device's address of the block
 * (cudaGetSymbolAddress, with the device current); make that first call
 * before any stream capture.  Every call on a device uses the same block and
 * leaves its contents behind (each call clears what it needs zeroed), so
 * calls whose work overlaps on the GPU — on different streams, or from
 * different threads — race and corrupt each other: serialise them.
 *
 * The block belongs to the device that is current when the call is made:
 * `stream` must be a stream of that device's primary context, and O must be
 * device memory of that device (checked: DSA_ERR_INVALID_ARG otherwise).
 * There is no workspace to hand to dsa_last_stats, so its counters are not
 * available for calls made through this entry point.
 */
#define DSA_DECODE_STATIC_SCRATCH_BYTES (18u << 20)
dsa_status dsa_decode_static(const void* k_idx, const void* K, const void* V,
                             const int64_t* seq_start, int B, int64_t total_rows, int64_t max_len,
                             int idx_dtype, int d_idx, int D, const void* q_idx, const void* Q, int H,
                             int top_k, float idx_scale, float attn_scale, void* O,
                             int32_t* indices, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
