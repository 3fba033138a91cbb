// nm_compress.cu -- N:M magnitude prune + push-left compression, and the
// inverse scatter, as streaming (HBM-bound) kernels.
//
// Selection rule ("M:N sparsity on NVIDIA tensor cores": opening passage and
// "The recipe", step 2): in every group of M consecutive weights along a row
// keep the N of largest magnitude; equal magnitudes go to the lower index.
// Magnitudes are compared as the 15-bit magnitude field of the bf16 pattern,
// which orders finite values and infinities exactly as |w| does; NaNs are
// folded to one key just above +Inf so they tie among themselves.
// Storage (same page, storage paragraphs of "Where this sits among the three
// case studies"): survivors pushed left in ascending position; b-bit
// positions, survivor j of a row in word j/S at bit b*(j%S).
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

__device__ __forceinline__ uint32_t mag_key(uint32_t bits16) {
  const uint32_t k = bits16 & 0x7FFFu;
  return k > 0x7F80u ? 0x7F81u : k;
}

// One group of four (e[0..3] as 16-bit patterns) -> 2:4 nibble (p0 | p1 << 2)
// and the two survivors packed lo | hi << 16.
__device__ __forceinline__ void select_2of4(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3, uint32_t& nib,
                                            uint32_t& packed) {
  // Composite keys are distinct: magnitude first, then the lower index.
  const uint32_t c0 = (mag_key(e0) << 2) | 3u, c1 = (mag_key(e1) << 2) | 2u;
  const uint32_t c2 = (mag_key(e2) << 2) | 1u, c3 = (mag_key(e3) << 2) | 0u;
  const uint32_t r0 = (c1 > c0) + (c2 > c0) + (c3 > c0);
  const uint32_t r1 = (c0 > c1) + (c2 > c1) + (c3 > c1);
  const uint32_t r2 = (c0 > c2) + (c1 > c2) + (c3 > c2);
  const uint32_t r3 = (c0 > c3) + (c1 > c3) + (c2 > c3);
  const uint32_t keep = (r0 < 2u) | ((r1 < 2u) << 1) | ((r2 < 2u) << 2) | ((r3 < 2u) << 3);
  const uint32_t p0 = __ffs(keep) - 1u;
  const uint32_t p1 = 31u - __clz(keep);
  nib = p0 | (p1 << 2);
  const uint32_t v0 = p0 == 0 ? e0 : p0 == 1 ? e1 : e2;  // p0 <= 2
  const uint32_t v1 = p1 == 3 ? e3 : p1 == 2 ? e2 : e1;  // p1 >= 1
  packed = v0 | (v1 << 16);
}

// 2:4 fast path.  A warp walks the matrix in 512-byte pieces (32 lanes x 8
// weights = 8 metadata words); each lane loads 16 contiguous bytes, selects
// its two groups, stores 8 bytes of values, and four neighbouring lanes merge
// their metadata bytes into one word with shuffles.  Loads and stores of a
// warp instruction are contiguous.  U pieces per lane are kept in flight.
constexpr int kCompressUnroll = 4;

__global__ void __launch_bounds__(256) compress_2of4_kernel(const uint16_t* __restrict__ W, uint32_t R,
                                                            uint32_t K, int64_t ldw, uint16_t* __restrict__ V,
                                                            uint32_t* __restrict__ meta) {
  // R * K / 8 < 2^32 is checked by the launcher: 32-bit index arithmetic.
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t cpr = K >> 3;           // 8-weight chunks per row
  const uint32_t total = R * cpr;        // chunks in the matrix
  const uint32_t warp_id = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t base = warp_id * 32u * kCompressUnroll; base < total; base += nwarps * 32u * kCompressUnroll) {
    uint4 in[kCompressUnroll];
    uint32_t rr[kCompressUnroll], cc[kCompressUnroll];
#pragma unroll
    for (int u = 0; u < kCompressUnroll; ++u) {
      const uint32_t c = base + u * 32u + lane;
      rr[u] = c / cpr;
      cc[u] = c - rr[u] * cpr;
      in[u] = c < total ? __ldg(reinterpret_cast<const uint4*>(W + (int64_t)rr[u] * ldw + (cc[u] << 3)))
                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kCompressUnroll; ++u) {
      uint32_t nib0, nib1, pk0, pk1;
      select_2of4(in[u].x & 0xFFFFu, in[u].x >> 16, in[u].y & 0xFFFFu, in[u].y >> 16, nib0, pk0);
      select_2of4(in[u].z & 0xFFFFu, in[u].z >> 16, in[u].w & 0xFFFFu, in[u].w >> 16, nib1, pk1);
      // byte of this lane inside its metadata word: lanes 4q..4q+3 -> bytes 0..3
      uint32_t word = (nib0 | (nib1 << 4)) << (8 * (lane & 3));
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      if (base + u * 32u + lane < total) {
        const int64_t r = rr[u];
        *reinterpret_cast<uint2*>(V + r * (K >> 1) + (cc[u] << 2)) = make_uint2(pk0, pk1);
        if ((lane & 3) == 0) meta[r * (K >> 5) + (cc[u] >> 2)] = word;
      }
    }
  }
}

// Generic path: one thread per metadata word.  The thread re-derives the
// selection of every group its survivors belong to (a group may straddle two
// words when S is not a multiple of N) and writes only its own survivors.
template <int M>
__global__ void __launch_bounds__(256) compress_generic_kernel(const uint16_t* __restrict__ W, int64_t R,
                                                               int64_t K, int64_t ldw, int n,
                                                               uint16_t* __restrict__ V,
                                                               uint32_t* __restrict__ meta) {
  constexpr int B = M == 2 ? 1 : M == 4 ? 2 : M == 8 ? 3 : 4;
  constexpr int S = 32 / B;
  const int64_t vcols = K / M * n;
  const int64_t mcols = (vcols + S - 1) / S;
  const int64_t total = R * mcols;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = w / mcols;
    const int64_t c = w - r * mcols;
    const int64_t j0 = c * S;
    const int64_t j1 = (j0 + S < vcols) ? j0 + S : vcols;
    uint32_t word = 0;
    int64_t cur_g = -1;
    uint32_t keep = 0;
    for (int64_t j = j0; j < j1; ++j) {
      const int64_t g = j / n;
      if (g != cur_g) {
        cur_g = g;
        const uint16_t* grp = W + r * ldw + g * M;
        uint32_t ck[M];
#pragma unroll
        for (int i = 0; i < M; ++i) ck[i] = (mag_key(grp[i]) << 4) | (uint32_t)(15 - i);
        keep = 0;
#pragma unroll
        for (int i = 0; i < M; ++i) {
          int rank = 0;
#pragma unroll
          for (int t = 0; t < M; ++t) rank += (ck[t] > ck[i]);
          keep |= (uint32_t)(rank < n) << i;
        }
      }
      // position of survivor s = j - g*n: the s-th set bit of keep
      uint32_t rest = keep;
      for (int64_t s = j - g * n; s > 0; --s) rest &= rest - 1u;
      const uint32_t p = __ffs(rest) - 1u;
      V[r * vcols + j] = W[r * ldw + g * M + p];
      word |= p << (B * (int)(j - j0));
    }
    meta[w] = word;
  }
}

// 2:4 fast decompress: one thread per metadata word -> 32 output weights.
__global__ void __launch_bounds__(256) decompress_2of4_kernel(const uint16_t* __restrict__ V,
                                                              const uint32_t* __restrict__ meta, int64_t R,
                                                              int64_t K, uint16_t* __restrict__ W, int64_t ldw) {
  const int64_t wpr = K >> 5;
  const int64_t total = R * wpr;
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = w / wpr;
    const int64_t c = w - r * wpr;
    const uint32_t word = __ldg(meta + w);
    const uint4* src = reinterpret_cast<const uint4*>(V + r * (K >> 1) + (c << 4));
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    const uint32_t vals[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[16];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      const uint32_t nib = (word >> (4 * g)) & 0xFu;
      const uint32_t p0 = nib & 3u, p1 = nib >> 2;
      const uint32_t v0 = vals[g] & 0xFFFFu, v1 = vals[g] >> 16;
      uint32_t e[4];
#pragma unroll
      for (uint32_t i = 0; i < 4; ++i) e[i] = (i == p0) ? v0 : (i == p1) ? v1 : 0u;
      out[2 * g] = e[0] | (e[1] << 16);
      out[2 * g + 1] = e[2] | (e[3] << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(W + r * ldw + (c << 5));
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
  }
}

// Generic decompress: one thread per group.
template <int M>
__global__ void __launch_bounds__(256) decompress_generic_kernel(const uint16_t* __restrict__ V,
                                                                 const uint32_t* __restrict__ meta, int64_t R,
                                                                 int64_t K, int n, uint16_t* __restrict__ W,
                                                                 int64_t ldw) {
  constexpr int B = M == 2 ? 1 : M == 4 ? 2 : M == 8 ? 3 : 4;
  constexpr int S = 32 / B;
  const int64_t groups = K / M;
  const int64_t vcols = groups * n;
  const int64_t mcols = (vcols + S - 1) / S;
  const int64_t total = R * groups;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t / groups;
    const int64_t g = t - r * groups;
    uint16_t e[M];
#pragma unroll
    for (int i = 0; i < M; ++i) e[i] = 0;
    for (int s = 0; s < n; ++s) {
      const int64_t j = g * n + s;
      const uint32_t word = __ldg(meta + r * mcols + j / S);
      const uint32_t p = (word >> (B * (int)(j % S))) & ((1u << B) - 1u);
      const uint16_t v = V[r * vcols + j];
#pragma unroll
      for (int i = 0; i < M; ++i)
        if ((uint32_t)i == p) e[i] = v;
    }
    uint16_t* dst = W + r * ldw + g * M;
#pragma unroll
    for (int i = 0; i < M; ++i) dst[i] = e[i];
  }
}

__global__ void fill_zero_kernel(uint8_t* Y, int64_t R, int64_t row_bytes, int64_t ld_bytes) {
  const int64_t total = R * row_bytes;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / row_bytes;
    Y[r * ld_bytes + (i - r * row_bytes)] = 0;
  }
}

static int grid_for(int64_t work, int threads) {
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count_current() * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaError_t launch_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint16_t* values,
                            uint32_t* meta, cudaStream_t s) {
  const int threads = 256;
  if (n == 2 && m == 4 && K % 32 == 0 && ldw % 8 == 0 && aligned16(W) && aligned16(values) &&
      R * (K / 8) < (int64_t(1) << 32) - 4096 * kCompressUnroll) {
    const int64_t work = R * (K / 8) / kCompressUnroll;
    compress_2of4_kernel<<<grid_for(work, threads), threads, 0, s>>>(W, (uint32_t)R, (uint32_t)K, ldw, values,
                                                                     meta);
  } else {
    const int64_t work = R * meta_cols(K, n, m);
    const int grid = grid_for(work, threads);
    switch (m) {
      case 2: compress_generic_kernel<2><<<grid, threads, 0, s>>>(W, R, K, ldw, n, values, meta); break;
      case 4: compress_generic_kernel<4><<<grid, threads, 0, s>>>(W, R, K, ldw, n, values, meta); break;
      case 8: compress_generic_kernel<8><<<grid, threads, 0, s>>>(W, R, K, ldw, n, values, meta); break;
      default: compress_generic_kernel<16><<<grid, threads, 0, s>>>(W, R, K, ldw, n, values, meta); break;
    }
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_decompress(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K, int n, int m,
                              uint16_t* W_out, int64_t ldw, cudaStream_t s) {
  const int threads = 256;
  if (n == 2 && m == 4 && K % 32 == 0 && ldw % 8 == 0 && aligned16(W_out) && aligned16(values)) {
    const int64_t work = R * (K / 32);
    decompress_2of4_kernel<<<grid_for(work, threads), threads, 0, s>>>(values, meta, R, K, W_out, ldw);
  } else {
    const int64_t work = R * (K / m);
    const int grid = grid_for(work, threads);
    switch (m) {
      case 2: decompress_generic_kernel<2><<<grid, threads, 0, s>>>(values, meta, R, K, n, W_out, ldw); break;
      case 4: decompress_generic_kernel<4><<<grid, threads, 0, s>>>(values, meta, R, K, n, W_out, ldw); break;
      case 8: decompress_generic_kernel<8><<<grid, threads, 0, s>>>(values, meta, R, K, n, W_out, ldw); break;
      default: decompress_generic_kernel<16><<<grid, threads, 0, s>>>(values, meta, R, K, n, W_out, ldw); break;
    }
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fill_zero(void* Y, int64_t R, int64_t T, int64_t ldy, int esize, cudaStream_t s) {
  const int threads = 256;
  fill_zero_kernel<<<grid_for(R * T * esize, threads), threads, 0, s>>>(static_cast<uint8_t*>(Y), R, T * esize,
                                                                         ldy * esize);
  count_launch();
  return cudaGetLastError();
}

}  // namespace nmk
