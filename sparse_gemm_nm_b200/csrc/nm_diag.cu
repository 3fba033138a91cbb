// nm_diag.cu -- diagonal sparsity under the index-map permutation.
//
// SHUFFLESPARSE applies one permutation primitive to block, N:M and diagonal
// patterns; DynaDiag keeps a diagonal pattern through training (90 % sparse ViT
// linears).  The pages give no format, so the library reads it plainly:
// diagonal o (0 <= o < K) of an R x K weight is {(r, (r + o) mod K)}, one entry
// per row; a diagonal operand keeps D distinct offsets (ascending) and
// V[d][r] = W[r][(r + o_d) mod K].  One-shot selection keeps the D diagonals
// with the largest score s(o) = sum_r |W[r][(r + o) mod K]|, an fp32 sum in
// ascending r (NaN above every number, ties to the lower offset).
//
// Kernels: scores (one thread per offset, the fixed-order sum), rank (one
// thread per offset counts the offsets that beat it), place (the kept offsets
// in ascending order), gather (V), and the scatter that writes a dense copy for
// the GEMM, which then runs as a dense tcgen05 GEMM on SM pairs: at 90 %
// sparsity the dense tensor-core rate beats multiplying only the kept entries
// on the CUDA cores (see the design notes).
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

__global__ void __launch_bounds__(256) diag_scores_kernel(const uint16_t* __restrict__ W, int64_t R, int64_t K,
                                                         int64_t ldw, float* __restrict__ scores) {
  pdl_gate();
  const int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (o >= K) return;
  float acc = 0.0f;
  int64_t col = o;
  for (int64_t r = 0; r < R; ++r) {
    const float w = __uint_as_float((uint32_t)__ldg(W + r * ldw + col) << 16);
    acc = __fadd_rn(acc, fabsf(w));
    if (++col == K) col = 0;
  }
  scores[o] = acc;
}

__device__ __forceinline__ bool diag_beats(float sa, int64_t a, float sb, int64_t b) {
  const bool na = isnan(sa), nb = isnan(sb);
  if (na || nb) return (na && !nb) || (na && nb && a < b);
  return sa > sb || (sa == sb && a < b);
}

// keep[o] = 1 when fewer than D offsets beat o.
__global__ void __launch_bounds__(256) diag_rank_kernel(const float* __restrict__ scores, int64_t K, int64_t D,
                                                       uint8_t* __restrict__ keep) {
  pdl_gate();
  __shared__ float s[2048];
  const int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const float so = o < K ? scores[o] : 0.0f;
  int64_t rank = 0;
  for (int64_t base = 0; base < K; base += 2048) {
    __syncthreads();
    for (int64_t i = threadIdx.x; i < 2048 && base + i < K; i += blockDim.x) s[i] = scores[base + i];
    __syncthreads();
    const int64_t n = K - base < 2048 ? K - base : 2048;
    if (o < K)
      for (int64_t i = 0; i < n; ++i)
        if (base + i != o && diag_beats(s[i], base + i, so, o)) ++rank;
  }
  if (o < K) keep[o] = rank < D ? 1 : 0;
}

// offsets[#kept below o] = o for every kept o.
__global__ void __launch_bounds__(256) diag_place_kernel(const uint8_t* __restrict__ keep, int64_t K,
                                                        int32_t* __restrict__ offsets) {
  pdl_gate();
  const int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (o >= K || !keep[o]) return;
  int64_t pos = 0;
  for (int64_t p = 0; p < o; ++p) pos += keep[p];
  offsets[pos] = (int32_t)o;
}

// V[d][r] = W[r][(r + o_d) mod K]
__global__ void __launch_bounds__(256) diag_gather_kernel(const uint16_t* __restrict__ W, int64_t R, int64_t K,
                                                         int64_t ldw, const int32_t* __restrict__ offsets,
                                                         int64_t D, uint16_t* __restrict__ V) {
  pdl_gate();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < D * R; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t d = i / R, r = i - d * R;
    V[i] = W[r * ldw + (r + offsets[d]) % K];
  }
}

// W_out[r][(r + o_d) mod K] = V[d][r] (the rest of W_out zeroed before)
__global__ void __launch_bounds__(256) diag_scatter_kernel(const uint16_t* __restrict__ V,
                                                          const int32_t* __restrict__ offsets, int64_t D, int64_t R,
                                                          int64_t K, uint16_t* __restrict__ W_out, int64_t ldw) {
  pdl_gate();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < D * R; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t d = i / R, r = i - d * R;
    const int64_t o = offsets[d];
    if (o < 0 || o >= K) continue;  // not a valid offset: nothing to place
    W_out[r * ldw + (r + o) % K] = V[i];
  }
}

static int grid_of(int64_t n, int threads) {
  const int64_t want = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count_current() * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_diag_select(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D, float* scores,
                               uint8_t* keep, int32_t* offsets, uint16_t* values, cudaStream_t s) {
  const int blocks = (int)((K + 255) / 256);
  cudaError_t e = launch_pdl(diag_scores_kernel, dim3(blocks), dim3(256), 0, s, W, R, K, ldw, scores);
  count_launch();
  if (e == cudaSuccess) e = launch_pdl(diag_rank_kernel, dim3(blocks), dim3(256), 0, s, (const float*)scores, K, D, keep);
  count_launch();
  if (e == cudaSuccess) e = launch_pdl(diag_place_kernel, dim3(blocks), dim3(256), 0, s, (const uint8_t*)keep, K, offsets);
  count_launch();
  if (e == cudaSuccess && D > 0)
    e = launch_pdl(diag_gather_kernel, dim3(grid_of(D * R, 256)), dim3(256), 0, s, W, R, K, ldw,
                   (const int32_t*)offsets, D, values);
  if (D > 0) count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_diag_expand(const uint16_t* V, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                               uint16_t* W_out, int64_t ldw, cudaStream_t s) {
  cudaError_t e = launch_fill_zero(W_out, R, K, ldw, 2, s);
  if (e == cudaSuccess && D > 0) {
    e = launch_pdl(diag_scatter_kernel, dim3(grid_of(D * R, 256)), dim3(256), 0, s, V, offsets, D, R, K, W_out, ldw);
    count_launch();
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nmk
