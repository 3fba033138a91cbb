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
// Selection kernels: partial scores (one thread per offset and 32-row chunk),
// scores (a block per 32 offsets adds their chunk sums in order from shared
// memory), rank (blocks of 256 offsets x 64 competitors count, by one 64-bit
// key compare each, the offsets that beat each offset), place (one block: a
// prefix sum puts the kept offsets in ascending order), gather (V).
//
// The GEMM runs on a dense copy of the operand with a dense tcgen05 GEMM on SM
// pairs: at 90 % sparsity the dense tensor-core rate beats multiplying only
// the kept entries on the CUDA cores.  The copy is written by lookup, every
// element once with 16-byte stores: entry (r, k) sits on diagonal
// (k - r) mod K, whose slot in V comes from a K-entry table.  With an index
// map that is a permutation (checked on the device), the copy's columns are
// placed through it, W''[r][idx[k]] = W'[r][k], so that W'' X = W' X[idx] and
// the GEMM reads X itself instead of a gathered copy of it.
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

static int grid_of(int64_t n, int threads) {
  const int64_t want = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count_current() * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

__device__ __forceinline__ float abs_bf16(uint16_t b) { return fabsf(__uint_as_float((uint32_t)b << 16)); }

// Partial scores: thread (o, c) sums |W[r][(r + o) mod K]| over the 32 rows of chunk c, r ascending;
// part[c * K + o].  Consecutive threads take consecutive offsets, so the loads of a row are coalesced.
// A full chunk (and K >= 32, so the column wraps at most once) loads its 32 values before adding.
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
    if (r1 - r0 == 32 && K >= 32) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int64_t cc = col + j < K ? col + j : col + j - K;
        v[j] = abs_bf16(__ldg(W + (r0 + j) * ldw + cc));
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) acc = __fadd_rn(acc, v[j]);
    } else {
      for (int64_t r = r0; r < r1; ++r) {
        acc = __fadd_rn(acc, abs_bf16(__ldg(W + r * ldw + col)));
        if (++col == K) col = 0;
      }
    }
    part[i] = acc;
  }
}

// s(o) = the chunk sums in ascending chunk order.  A block takes 32 offsets: its eight warps stage slabs
// of 64 chunk rows (coalesced 128-byte rows) in shared memory, and warp 0 adds them in order.
__global__ void __launch_bounds__(256) diag_scores_kernel(const float* __restrict__ part, int64_t R, int64_t K,
                                                         float* __restrict__ scores) {
  pdl_gate();
  __shared__ float slab[64][33];
  const int64_t chunks = (R + 31) / 32;
  const int64_t o0 = (int64_t)blockIdx.x * 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const bool in = o0 + lane < K;
  float acc = 0.0f;
  for (int64_t c0 = 0; c0 < chunks; c0 += 64) {
    const int nc = chunks - c0 < 64 ? (int)(chunks - c0) : 64;
    for (int cc = w; cc < nc; cc += 8) slab[cc][lane] = in ? part[(c0 + cc) * K + o0 + lane] : 0.0f;
    __syncthreads();
    if (w == 0)
      for (int cc = 0; cc < nc; ++cc) acc = __fadd_rn(acc, slab[cc][lane]);
    __syncthreads();
  }
  if (w == 0 && in) scores[o0 + lane] = acc;
}

// Order key of offset o with score s: p beats o exactly when key(p) > key(o).  The score maps to an
// unsigned integer in the order of the floats (NaN above +Inf and all NaNs equal, -0 equal to +0);
// the low word ranks equal scores by lower offset.
__device__ __forceinline__ uint64_t diag_key(float s, int64_t o) {
  uint32_t u = __float_as_uint(s);
  if (isnan(s))
    u = 0xFFFFFFFFu;
  else if (s == 0.0f)
    u = 0x80000000u;
  else
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)u << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)o);
}

constexpr int kRankTile = 64;  // competitors per block

// rank[o] += #{p in this block's slice of competitors : p beats o}; blocks cover (offset tile of 256,
// competitor tile of 64) pairs (x: competitor tile, y: offset tile), so the count is an exact integer
// whatever the order of the additions.
__global__ void __launch_bounds__(256) diag_rank_kernel(const float* __restrict__ scores, int64_t K,
                                                       uint32_t* __restrict__ rank) {
  pdl_gate();
  __shared__ uint64_t key[kRankTile];
  const int64_t p0 = (int64_t)blockIdx.x * kRankTile;
  const int64_t o = (int64_t)blockIdx.y * 256 + threadIdx.x;
  if (threadIdx.x < kRankTile && p0 + threadIdx.x < K) key[threadIdx.x] = diag_key(scores[p0 + threadIdx.x], p0 + threadIdx.x);
  __syncthreads();
  if (o >= K) return;
  const uint64_t ko = diag_key(scores[o], o);
  const int n = K - p0 < kRankTile ? (int)(K - p0) : kRankTile;
  uint32_t cnt = 0;
#pragma unroll 8
  for (int i = 0; i < n; ++i) cnt += key[i] > ko ? 1u : 0u;
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

// Tables of the dense copy (filled with 0xFF bytes before): slot[o] = d for each kept offset o_d in
// [0, K), else -1; with idx, cnt[j] counts (from -1) the entries naming j, inv[j] = the k with
// idx[k] = j, and *is_perm drops to 0 when an entry is out of range or a second entry names the
// same j -- so *is_perm stays nonzero exactly when idx is a permutation of [0, K).
__global__ void __launch_bounds__(256) diag_tables_kernel(const int32_t* __restrict__ offsets, int64_t D, int64_t K,
                                                         const int32_t* __restrict__ idx, int32_t* __restrict__ slot,
                                                         int32_t* __restrict__ cnt, int32_t* __restrict__ inv,
                                                         uint32_t* __restrict__ is_perm) {
  pdl_gate();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < K; i += (int64_t)gridDim.x * blockDim.x) {
    if (i < D) {
      const int32_t o = offsets[i];
      if (o >= 0 && (int64_t)o < K) slot[o] = (int32_t)i;
    }
    if (idx) {
      const int32_t j = idx[i];
      if (j < 0 || (int64_t)j >= K) {
        *is_perm = 0u;
      } else {
        if (atomicAdd(cnt + j, 1) != -1) *is_perm = 0u;
        inv[j] = (int32_t)i;
      }
    }
  }
}

// W[r][j] for j in [0, K): the entry of column k = inv[j] (a permutation) or k = j (otherwise), which is
// V[slot[(k - r) mod K]][r] when that diagonal is kept, else +0.  A thread writes 8 columns of a row,
// consecutive threads consecutive column groups (16-byte stores when the rows allow them).
__global__ void __launch_bounds__(256) diag_dense_kernel(const uint16_t* __restrict__ V, const int32_t* __restrict__ slot,
                                                        int64_t R, int64_t K, const int32_t* __restrict__ inv,
                                                        const uint32_t* is_perm, uint16_t* __restrict__ W,
                                                        int64_t ldw, int vec) {
  pdl_gate();
  const bool perm = inv && *reinterpret_cast<const volatile uint32_t*>(is_perm);
  const int64_t groups = (K + 7) / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < R * groups;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / groups, j0 = (i - r * groups) * 8;
    const int64_t rm = r % K;
    uint32_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int64_t j = j0 + e;
      uint32_t b = 0;
      if (j < K) {
        const int64_t k = perm ? (int64_t)__ldg(inv + j) : j;
        int64_t o = k - rm;
        if (o < 0) o += K;
        const int32_t d = __ldg(slot + o);
        if (d >= 0) b = __ldg(V + (int64_t)d * R + r);
      }
      h[e] = b;
    }
    uint16_t* dst = W + r * ldw + j0;
    if (vec && j0 + 8 <= K) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                                                  h[6] | (h[7] << 16));
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (j0 + e < K) dst[e] = (uint16_t)h[e];
    }
  }
}

cudaError_t launch_diag_select(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D, float* part,
                               float* scores, uint8_t* keep, int32_t* offsets, uint16_t* values, cudaStream_t s) {
  const int64_t otiles = (K + 255) / 256, ptiles = (K + kRankTile - 1) / kRankTile;
  cudaError_t e = launch_pdl(diag_part_kernel, dim3(grid_of((R + 31) / 32 * K, 256)), dim3(256), 0, s, W, R, K, ldw,
                             part);
  count_launch();
  if (e == cudaSuccess)
    e = launch_pdl(diag_scores_kernel, dim3((unsigned)((K + 31) / 32)), dim3(256), 0, s, (const float*)part, R, K,
                   scores);
  count_launch();
  uint32_t* rank = reinterpret_cast<uint32_t*>(keep);
  if (e == cudaSuccess) e = cudaMemsetAsync(rank, 0, (size_t)K * 4, s);
  if (e == cudaSuccess)
    e = launch_pdl(diag_rank_kernel, dim3((unsigned)ptiles, (unsigned)otiles), dim3(256), 0, s, (const float*)scores,
                   K, rank);
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

int64_t diag_table_words(int64_t K, bool with_idx) { return with_idx ? 3 * K + 1 : K; }

cudaError_t launch_diag_dense(const uint16_t* V, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                              const int32_t* idx, int32_t* tables, uint16_t* W_out, int64_t ldw, cudaStream_t s,
                              const uint32_t** is_perm) {
  int32_t* slot = tables;
  int32_t* cnt = idx ? tables + K : nullptr;
  int32_t* inv = idx ? tables + 2 * K : nullptr;
  uint32_t* flag = idx ? reinterpret_cast<uint32_t*>(tables + 3 * K) : nullptr;
  if (is_perm) *is_perm = flag;
  cudaError_t e = cudaMemsetAsync(tables, 0xFF, (size_t)diag_table_words(K, idx != nullptr) * 4, s);
  if (e == cudaSuccess)
    e = launch_pdl(diag_tables_kernel, dim3(grid_of(K, 256)), dim3(256), 0, s, offsets, D, K, idx, slot, cnt, inv, flag);
  count_launch();
  const int vec = (reinterpret_cast<uintptr_t>(W_out) % 16 == 0 && ldw % 8 == 0) ? 1 : 0;
  if (e == cudaSuccess)
    e = launch_pdl(diag_dense_kernel, dim3(grid_of(R * ((K + 7) / 8), 256)), dim3(256), 0, s, V,
                   (const int32_t*)slot, R, K, (const int32_t*)inv, (const uint32_t*)flag, W_out, ldw, vec);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nmk
