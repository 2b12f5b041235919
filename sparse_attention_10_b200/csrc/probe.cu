// Gather probe: the memory ceiling of the sparse attention's access pattern.
//
// The attention of the DeepSeek Sparse Attention page (sections 3.3 and 4.2)
// reads, for every query, the K and V rows of its kept keys: 2 x top_k random
// rows of 256 bytes (head dim 128) out of tensors small enough to stay in L2.
// Its bound is therefore neither the HBM copy rate nor the tensor cores but
// how fast the SMs can pull random rows through L2 into shared memory.  This
// kernel does exactly that and nothing else: for every query row t it copies
// the rows listed in indices[t, 0 : min(t + 1, top_k)] of K and then of V into
// a ring of 16 KB shared-memory stages with 16-byte cp.async, each thread
// reading back one word of its own copies once they land.  Its rate over a
// few launch shapes is the ceiling the attention kernel is measured against.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr int kProbeThreads = 128;
constexpr int kProbeStage = 16384;

__device__ __forceinline__ void probe_cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int NST>
__device__ __forceinline__ void probe_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(NST) : "memory");
}

template <int NST>
__global__ void __launch_bounds__(kProbeThreads) gather_probe_kernel(const int32_t* __restrict__ idx,
                                                                      int64_t L, int top_k,
                                                                      const uint8_t* __restrict__ K,
                                                                      const uint8_t* __restrict__ V,
                                                                      int row_bytes,
                                                                      unsigned long long* sink) {
  constexpr int kPasses = 8;   // rows of a stage per thread: 64 rows of 256 B or 128 of 128 B
  extern __shared__ __align__(128) uint8_t ring[];
  const int lanes_per_row = row_bytes / 16;                     // 16 (D = 128) or 8 (D = 64)
  const int rows_per_pass = kProbeThreads / lanes_per_row;      // 8 or 16
  const int tile_rows = rows_per_pass * kPasses;                // 64 or 128: one 16 KB stage
  const int sub = threadIdx.x % lanes_per_row, r0 = threadIdx.x / lanes_per_row;
  uint32_t acc = 0;
  uint32_t issued = 0;
  for (int64_t t = blockIdx.x; t < L; t += gridDim.x) {
    const int m = static_cast<int>(min64(t + 1, top_k));
    const int32_t* ids = idx + t * top_k;
    for (int j0 = 0; j0 < m; j0 += tile_rows) {
      // the tile's row ids first (independent loads), then the copies
      int64_t rows[kPasses];
#pragma unroll
      for (int u = 0; u < kPasses; ++u) {
        const int j = j0 + r0 + u * rows_per_pass;
        int64_t s = j < m ? __ldg(ids + j) : -1;
        rows[u] = (s < 0 || s >= L) ? (j < m ? 0 : -1) : s;
      }
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint8_t* src = which ? V : K;
        const uint32_t stage = smem_u32(ring + (issued % NST) * kProbeStage);
#pragma unroll
        for (int u = 0; u < kPasses; ++u)
          if (rows[u] >= 0)
            probe_cp16(stage + (r0 + u * rows_per_pass) * row_bytes + sub * 16,
                       src + rows[u] * row_bytes + sub * 16);
        asm volatile("cp.async.commit_group;" ::: "memory");
        ++issued;
        // The ring holds NST tiles.  With at most NST - 1 groups pending, the
        // tile in the slot the next copy reuses has landed: read one word of
        // this thread's own copies there before the slot is overwritten.
        probe_wait<NST - 1>();
        acc ^= *reinterpret_cast<const volatile uint32_t*>(ring + (issued % NST) * kProbeStage +
                                                           r0 * row_bytes + sub * 16);
      }
    }
  }
  probe_wait<0>();
  acc = __reduce_xor_sync(0xFFFFFFFFu, acc);
  if ((threadIdx.x & 31) == 0 && acc == 0x9E3779B9u) atomicXor(sink, 1ull);   // keeps the loads live
}

template <int NST>
cudaError_t launch_probe(const int32_t* idx, int64_t L, int top_k, const uint8_t* K, const uint8_t* V,
                         int row_bytes, int grid, unsigned long long* sink, cudaStream_t s) {
  const int smem = NST * kProbeStage;
  cudaError_t e = cudaFuncSetAttribute(gather_probe_kernel<NST>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gather_probe_kernel<NST><<<grid, kProbeThreads, smem, s>>>(idx, L, top_k, K, V, row_bytes, sink);
  return cudaGetLastError();
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status dsa_gather_probe(const int32_t* indices, int64_t L, int top_k, const void* K,
                                       const void* V, int D, int ctas_per_sm, int stages,
                                       uint64_t* sink, void* stream) {
  using namespace dsa;
  if (!indices || !K || !V || !sink || L < 1 || top_k < 1 || top_k > DSA_MAX_TOP_K) return DSA_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || ctas_per_sm < 1 || ctas_per_sm > 8) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15) return DSA_ERR_INVALID_ARG;
  const int64_t grid64 = min64(static_cast<int64_t>(num_sms()) * ctas_per_sm, L);
  const int grid = static_cast<int>(grid64);
  const int row_bytes = D * 2;
  auto s = static_cast<cudaStream_t>(stream);
  auto Kb = static_cast<const uint8_t*>(K);
  auto Vb = static_cast<const uint8_t*>(V);
  auto sk = reinterpret_cast<unsigned long long*>(sink);
  cudaError_t e;
  switch (stages) {
    case 2: e = launch_probe<2>(indices, L, top_k, Kb, Vb, row_bytes, grid, sk, s); break;
    case 3: e = launch_probe<3>(indices, L, top_k, Kb, Vb, row_bytes, grid, sk, s); break;
    case 4: e = launch_probe<4>(indices, L, top_k, Kb, Vb, row_bytes, grid, sk, s); break;
    case 6: e = launch_probe<6>(indices, L, top_k, Kb, Vb, row_bytes, grid, sk, s); break;
    default: return DSA_ERR_INVALID_ARG;
  }
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
