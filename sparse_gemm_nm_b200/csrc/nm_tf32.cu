// nm_tf32.cu -- 1:2 sparsity of float32 weights for the TF32 tensor cores.
//
// "M:N sparsity on NVIDIA tensor cores" (the passage on the formats the
// sparse tensor cores take): for TF32 the 2:4 block halves to 1:2, still
// 50 percent.  Selection follows the bf16 rule on the float32 value: of each
// pair along K the larger magnitude survives, equal magnitudes go to the lower
// index, a NaN ranks above every number (all NaNs equal).  Values are the
// survivors' float32 bits pushed left (R x K/2); the positions take one bit
// each, survivor j of a row in word j / 32 at bit j % 32 (the row-wise packing
// of the bf16 path with b = 1).
//
// Compress: one warp per (row, metadata word): lane l takes pair 32 c + l,
// loads its two values (the warp reads 256 contiguous bytes), stores the
// survivor (128 contiguous bytes per warp) and the warp's ballot of the
// positions is the metadata word.  Decompress: one thread per pair.  The GEMM
// decompresses into a staged dense copy and runs the dense pair kernel's
// kind::tf32 form (dense_pair_kernel).
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

static int grid_of(int64_t n, int threads) {
  const int64_t want = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count_current() * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

// Order key of a float32 magnitude: larger key = larger |w|; every NaN maps to one key above +Inf.
__device__ __forceinline__ uint32_t f32_key(uint32_t bits) { return min(bits & 0x7FFFFFFFu, 0x7F800001u); }

__global__ void __launch_bounds__(256) compress_1of2_f32_kernel(const uint32_t* __restrict__ W, int64_t R, int64_t K,
                                                               int64_t ldw, uint32_t* __restrict__ values,
                                                               uint32_t* __restrict__ meta) {
  pdl_gate();
  const int lane = threadIdx.x & 31;
  const int64_t pairs = K / 2, words = (pairs + 31) / 32;
  const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = warp0; w < R * words; w += nwarps) {
    const int64_t r = w / words, c = w - r * words;
    const int64_t p = 32 * c + lane;
    uint32_t pos = 0;
    if (p < pairs) {
      const uint32_t a = __ldg(W + r * ldw + 2 * p), b = __ldg(W + r * ldw + 2 * p + 1);
      pos = f32_key(a) >= f32_key(b) ? 0u : 1u;
      values[r * pairs + p] = pos ? b : a;
    }
    const uint32_t word = __ballot_sync(0xffffffffu, pos != 0);
    if (lane == 0) meta[r * words + c] = word;
  }
}

__global__ void __launch_bounds__(256) decompress_1of2_f32_kernel(const uint32_t* __restrict__ values,
                                                                 const uint32_t* __restrict__ meta, int64_t R,
                                                                 int64_t K, uint32_t* __restrict__ W_out,
                                                                 int64_t ldw) {
  pdl_gate();
  const int64_t pairs = K / 2, words = (pairs + 31) / 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < R * pairs;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / pairs, p = i - r * pairs;
    const uint32_t bit = (__ldg(meta + r * words + p / 32) >> (p % 32)) & 1u;
    const uint32_t v = __ldg(values + i);
    W_out[r * ldw + 2 * p] = bit ? 0u : v;
    W_out[r * ldw + 2 * p + 1] = bit ? v : 0u;
  }
}

cudaError_t launch_compress_tf32(const float* W, int64_t R, int64_t K, int64_t ldw, float* values, uint32_t* meta,
                                 cudaStream_t s) {
  const int64_t warps = R * ((K / 2 + 31) / 32);
  cudaError_t e = launch_pdl(compress_1of2_f32_kernel, dim3(grid_of(warps * 32, 256)), dim3(256), 0, s,
                             reinterpret_cast<const uint32_t*>(W), R, K, ldw, reinterpret_cast<uint32_t*>(values),
                             meta);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decompress_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, float* W_out,
                                   int64_t ldw, cudaStream_t s) {
  cudaError_t e = launch_pdl(decompress_1of2_f32_kernel, dim3(grid_of(R * (K / 2), 256)), dim3(256), 0, s,
                             reinterpret_cast<const uint32_t*>(values), meta, R, K,
                             reinterpret_cast<uint32_t*>(W_out), ldw);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nmk
