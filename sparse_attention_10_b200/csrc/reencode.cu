// Lossless FP8 re-encoding of BF16 indexer inputs.
//
// The DeepSeek Sparse Attention page sets the indexer's precision per length
// (section 7.2: FP8 at 32K and 64K, BF16 at 128K) and runs the index stage in
// FP8 (section 4.1).  When every BF16 value of q_idx / k_idx is exactly
// representable in FP8 E4M3, the FP8 copy gives bit-identical indexer scores
// (every product and partial sum is the same number), so the indexer can run
// on the FP8 tensor-core path at twice the BF16 rate.  This kernel writes the
// E4M3 copy and counts the values that do not survive the round trip; the
// copy may only be used when that count is zero.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

// Eight BF16 values (16 bytes) per thread and iteration, eight E4M3 bytes out.
__global__ void __launch_bounds__(256) bf16_to_e4m3_kernel(const uint4* __restrict__ in, int64_t n8,
                                                           uint2* __restrict__ out,
                                                           unsigned long long* inexact) {
  unsigned int bad = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 w = __ldg(in + i);
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162_raw pair;
      pair.x = static_cast<unsigned short>(words[k] & 0xFFFFu);
      pair.y = static_cast<unsigned short>(words[k] >> 16);
      const __nv_fp8x2_storage_t f8 = __nv_cvt_bfloat16raw2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
      const float2 back = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(f8, __NV_E4M3)));
      const float a = __uint_as_float((words[k] & 0xFFFFu) << 16);
      const float b = __uint_as_float(words[k] & 0xFFFF0000u);
      bad += (back.x == a ? 0u : 1u) + (back.y == b ? 0u : 1u);   // NaN never compares equal
      o[k >> 1] |= static_cast<uint32_t>(f8) << (16 * (k & 1));
    }
    out[i] = make_uint2(o[0], o[1]);
  }
  bad = __reduce_add_sync(0xFFFFFFFFu, bad);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(inexact, static_cast<unsigned long long>(bad));
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status dsa_index_to_fp8(const void* in_bf16, int64_t n, void* out_fp8,
                                       uint64_t* inexact, void* stream) {
  using namespace dsa;
  if (!in_bf16 || !out_fp8 || !inexact || n < 1 || n % 8 != 0) return DSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(in_bf16) & 15) || (reinterpret_cast<uintptr_t>(out_fp8) & 7) ||
      (reinterpret_cast<uintptr_t>(inexact) & 7))
    return DSA_ERR_INVALID_ARG;
  auto s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(inexact, 0, sizeof(uint64_t), s) != cudaSuccess) return DSA_ERR_CUDA;
  const int64_t n8 = n / 8;
  const int grid = static_cast<int>(min64((n8 + 255) / 256, 8 * static_cast<int64_t>(num_sms())));
  bf16_to_e4m3_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(in_bf16), n8,
                                           static_cast<uint2*>(out_fp8),
                                           reinterpret_cast<unsigned long long*>(inexact));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}
