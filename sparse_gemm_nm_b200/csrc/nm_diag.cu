// nm_diag.cu -- diagonal sparsity under the index-map permutation.
//
// SHUFFLESPARSE applies one permutation primitive to block, N:M and diagonal
// patterns; DynaDiag keeps a diagonal pattern through training (90 % sparse ViT
// linears).  The pages give no format, so the library reads it plainly:
// diagonal o (0 <= o < K) of an R x K weight is {(r, (r + o) mod K)}, one entry
// per row; a diagonal operand keeps D distinct offsets (ascending) and
// V[d][r] = W[r][(r + o_d) mod K].  One-shot selection keeps the D diagonals
// with the largest score s(o) = sum_r |W[r][(r + o) mod K]|, in fp32 and a
// fixed order: 32-row chunk sums (r ascending), then the chunk sums in
// ascending order (NaN above every number, ties to the lower offset).
//
// Kernels: partial scores (one thread per offset and 32-row chunk), scores
// (one thread per offset adds the chunk sums in order), rank (offset tile x
// competitor tile blocks count the offsets that beat each offset), place (one
// block: a prefix sum puts the kept offsets in ascending order), gather (V), and
// the scatter that writes a dense copy for the GEMM, which then runs as a
// dense tcgen05 GEMM on SM pairs: at 90 %
// sparsity the dense tensor-core rate beats multiplying only the kept entries
// on the CUDA cores (see the design notes).
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

static int grid_of(int64_t n, int threads) {
  const int64_t want = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count_current() * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}


// Partial scores: thread (o, c) sums |W[r][(r + o) mod K]| over the 32 rows of chunk c, r ascending;
// part[c * K + o].  Consecutive threads take consecutive offsets, so the loads of a row are coalesced.
__global__ void __launch_bounds__(256) diag_part_kernel(const uint16_t* __restrict__ W, int64_t R, int64_t K,
                                                       int64_t ldw, float* __restrict__ part) {
  pdl_gate();
  const int64_t chunks = (R + 31) / 32;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < chunks * K;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i / K, o = i - c * K;
    const int64_t r0 = 32 * c, r1 = r0 + 32 < R ? r0 + 32 : R;
    int64_t col = (r0 + o) % K;
    float acc = 0.0f;
    for (int64_t r = r0; r < r1; ++r) {
      acc = __fadd_rn(acc, fabsf(__uint_as_float((uint32_t)__ldg(W + r * ldw + col) << 16)));
      if (++col == K) col = 0;
    }
    part[i] = acc;
  }
}

// s(o) = the chunk sums in ascending chunk order.
__global__ void __launch_bounds__(256) diag_scores_kernel(const float* __restrict__ part, int64_t R, int64_t K,
                                                         float* __restrict__ scores) {
  pdl_gate();
  const int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (o >= K) return;
  const int64_t chunks = (R + 31) / 32;
  float acc = 0.0f;
  for (int64_t c = 0; c < chunks; ++c) acc = __fadd_rn(acc, part[c * K + o]);
  scores[o] = acc;
}

__device__ __forceinline__ bool diag_beats(float sa, int64_t a, float sb, int64_t b) {
  const bool na = isnan(sa), nb = isnan(sb);
  if (na || nb) return (na && !nb) || (na && nb && a < b);
  return sa > sb || (sa == sb && a < b);
}

// rank[o] += #{p in this block's 256-offset slice of competitors : p beats o}; blocks cover (offset tile,
// competitor tile) pairs, so the count is an exact integer whatever the order of the additions.
__global__ void __launch_bounds__(256) diag_rank_kernel(const float* __restrict__ scores, int64_t K,
                                                       uint32_t* __restrict__ rank) {
  pdl_gate();
  __shared__ float s[256];
  const int64_t tiles = (K + 255) / 256;
  const int64_t ot = blockIdx.x % tiles, pt = blockIdx.x / tiles;
  const int64_t o = ot * 256 + threadIdx.x, p0 = pt * 256;
  if (p0 + threadIdx.x < K) s[threadIdx.x] = scores[p0 + threadIdx.x];
  __syncthreads();
  if (o >= K) return;
  const float so = scores[o];
  const int64_t n = K - p0 < 256 ? K - p0 : 256;
  uint32_t cnt = 0;
  for (int64_t i = 0; i < n; ++i)
    if (p0 + i != o && diag_beats(s[i], p0 + i, so, o)) ++cnt;
  if (cnt) atomicAdd(rank + o, cnt);
}

// One block: keep[o] = rank[o] < D, then each kept offset goes to position #kept below it
// (a block-wide prefix sum over 1024-offset slices, in ascending order).
__global__ void __launch_bounds__(1024) diag_place_kernel(const uint32_t* __restrict__ rank, int64_t K, int64_t D,
                                                         int32_t* __restrict__ offsets) {
  pdl_gate();
  __shared__ uint32_t warp_sum[32];
  __shared__ uint32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t base = 0; base < K; base += 1024) {
    const int64_t o = base + threadIdx.x;
    const uint32_t keep = (o < K && (int64_t)rank[o] < D) ? 1u : 0u;
    uint32_t incl = keep;  // inclusive scan inside the warp
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      uint32_t w = warp_sum[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += v;
      }
      warp_sum[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const uint32_t before = carry + (warp ? warp_sum[warp - 1] : 0u) + incl - keep;
    if (keep) offsets[before] = (int32_t)o;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sum[31];
    __syncthreads();
  }
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

cudaError_t launch_diag_select(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D, float* part,
                               float* scores, uint8_t* keep, int32_t* offsets, uint16_t* values, cudaStream_t s) {
  const int blocks = (int)((K + 255) / 256);
  cudaError_t e = launch_pdl(diag_part_kernel, dim3(grid_of((R + 31) / 32 * K, 256)), dim3(256), 0, s, W, R, K, ldw,
                             part);
  count_launch();
  if (e == cudaSuccess)
    e = launch_pdl(diag_scores_kernel, dim3(blocks), dim3(256), 0, s, (const float*)part, R, K, scores);
  count_launch();
  uint32_t* rank = reinterpret_cast<uint32_t*>(keep);
  if (e == cudaSuccess) e = cudaMemsetAsync(rank, 0, (size_t)K * 4, s);
  if (e == cudaSuccess)
    e = launch_pdl(diag_rank_kernel, dim3((unsigned)(blocks * blocks)), dim3(256), 0, s, (const float*)scores, K, rank);
  count_launch();
  if (e == cudaSuccess)
    e = launch_pdl(diag_place_kernel, dim3(1), dim3(1024), 0, s, (const uint32_t*)rank, K, D, offsets);
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
