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
// case studies"): survivors pushed left in ascending position.  2:4 positions
// are tiled in the sparse tensor core's order (one nibble per group, see
// compress_2of4_tiled_kernel); other patterns are packed row-wise, b-bit
// positions, survivor j of a row in word j/S at bit b*(j%S).
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

__device__ __forceinline__ uint32_t mag_key(uint32_t bits16) {
  const uint32_t k = bits16 & 0x7FFFu;
  return k > 0x7F80u ? 0x7F81u : k;
}

// 2:4 with tiled metadata.  One warp per metadata block (16 rows x 128
// columns): lane i takes row 16*rb + i/2, columns 128*cb + 64*(i%2) .. +63
// (sixteen groups), so every 16-byte load of the warp covers 16 rows x 32
// bytes.  The lane selects its sixteen groups, stores its 32 survivors
// (64 contiguous bytes) and keeps the sixteen nibbles; the block's 64 words
// are then assembled with shuffles, 2 per lane.
//
// Selection of one group (keys k_i = bf16 magnitude field, NaNs folded just
// above +Inf): with s_ij = (k_i >= k_j) for i < j, element i beats j iff
// s_ij, and j beats i iff !s_ij (equal keys go to the lower index).  An
// element survives iff it beats at least two of the other three, a 3-input
// majority.
__device__ __forceinline__ uint32_t maj3(uint32_t a, uint32_t b, uint32_t c) { return (a & b) | (a & c) | (b & c); }

// Nibble p0 | p1 << 2 for each of the six 2-of-4 keep masks (others unused).
__device__ __forceinline__ uint32_t nibble_of_keep(uint32_t kb) {
  constexpr uint64_t lut = (0x4ull << (4 * 3)) | (0x8ull << (4 * 5)) | (0x9ull << (4 * 6)) | (0xCull << (4 * 9)) |
                           (0xDull << (4 * 10)) | (0xEull << (4 * 12));
  return (uint32_t)(lut >> (4 * kb)) & 0xFu;
}

// Group of four in (lo, hi) = (e0 | e1 << 16, e2 | e3 << 16): returns the
// nibble, and in `pk` the two survivors (first in the low half).
__device__ __forceinline__ uint32_t select_pair(uint32_t lo, uint32_t hi, uint32_t& pk) {
  const uint32_t k0 = min(lo & 0x7FFFu, 0x7F81u), k1 = min((lo >> 16) & 0x7FFFu, 0x7F81u);
  const uint32_t k2 = min(hi & 0x7FFFu, 0x7F81u), k3 = min((hi >> 16) & 0x7FFFu, 0x7F81u);
  const uint32_t s01 = k0 >= k1, s02 = k0 >= k2, s03 = k0 >= k3;
  const uint32_t s12 = k1 >= k2, s13 = k1 >= k3, s23 = k2 >= k3;
  const uint32_t keep = maj3(s01, s02, s03) | (maj3(s01 ^ 1u, s12, s13) << 1) | (maj3(s02 ^ 1u, s12 ^ 1u, s23) << 2) |
                        (maj3(s03 ^ 1u, s13 ^ 1u, s23 ^ 1u) << 3);
  const uint32_t nib = nibble_of_keep(keep);
  const uint32_t p0 = nib & 3u, p1 = nib >> 2;
  pk = __byte_perm(lo, hi, 0x1010u + p0 * 0x22u + p1 * 0x2200u);
  return nib;
}

__global__ void __launch_bounds__(256) compress_2of4_tiled_kernel(const uint16_t* __restrict__ W, uint32_t R,
                                                                  uint32_t K, int64_t ldw,
                                                                  uint16_t* __restrict__ V,
                                                                  uint32_t* __restrict__ meta, uint32_t cblocks,
                                                                  uint32_t nblocks, bool vec) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t blk = warp; blk < nblocks; blk += nwarps) {
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint32_t r = rb * 16 + (lane >> 1);
    const uint32_t c0 = cb * 128 + (lane & 1u) * 64;  // first of this lane's 64 columns
    uint32_t nib_lo = 0x44444444u, nib_hi = 0x44444444u;  // groups 0..7, 8..15
    if (r < R && c0 < K) {
      const uint16_t* wrow = W + (int64_t)r * ldw + c0;
      uint32_t* vrow = reinterpret_cast<uint32_t*>(V + (int64_t)r * (K >> 1) + c0 / 2);
      if (vec && c0 + 64 <= K) {
        uint4 in[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) in[i] = __ldg(reinterpret_cast<const uint4*>(wrow) + i);
        uint32_t pk[16];
        uint32_t n0 = 0, n1 = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t a = select_pair(in[i].x, in[i].y, pk[2 * i]);
          const uint32_t b = select_pair(in[i].z, in[i].w, pk[2 * i + 1]);
          const uint32_t two = a | (b << 4);
          if (i < 4) n0 |= two << (8 * i);
          else n1 |= two << (8 * (i - 4));
        }
        nib_lo = n0;
        nib_hi = n1;
        uint4* vout = reinterpret_cast<uint4*>(vrow);
#pragma unroll
        for (int i = 0; i < 4; ++i) vout[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      } else {
        uint32_t n0 = 0, n1 = 0;
        for (int g = 0; g < 16; ++g) {
          const uint32_t cg = c0 + 4 * g;
          uint32_t nib = 0x4u;
          if (cg < K) {
            const uint32_t lo = (uint32_t)wrow[4 * g] | ((uint32_t)wrow[4 * g + 1] << 16);
            const uint32_t hi = (uint32_t)wrow[4 * g + 2] | ((uint32_t)wrow[4 * g + 3] << 16);
            uint32_t pk;
            nib = select_pair(lo, hi, pk);
            vrow[g] = pk;
          }
          if (g < 8) n0 |= nib << (4 * g);
          else n1 |= nib << (4 * (g - 8));
        }
        nib_lo = n0;
        nib_hi = n1;
      }
    }
    // Words 2L, 2L+1 of the block: lane l = L/2 of the tile (row l%8 and row
    // 8 + l%8), quarters q = 2*(L%2) and 2*(L%2)+1, K half h = l/8.  Their
    // 16-bit halves live in lanes 2*(l%8) + L%2 (low row) and 2*(l%8 + 8) +
    // L%2 (high row), in 16-bit chunk h of nib_lo (q even) and nib_hi (q odd).
    const uint32_t l = lane >> 1, rr = l & 7u, h = l >> 3;
    const uint32_t src_lo = 2 * rr + (lane & 1u), src_hi = 2 * (rr + 8) + (lane & 1u);
    const uint32_t a_lo = __shfl_sync(0xffffffffu, nib_lo, src_lo);
    const uint32_t a_hi = __shfl_sync(0xffffffffu, nib_hi, src_lo);
    const uint32_t b_lo = __shfl_sync(0xffffffffu, nib_lo, src_hi);
    const uint32_t b_hi = __shfl_sync(0xffffffffu, nib_hi, src_hi);
    const uint32_t w0 = ((a_lo >> (16 * h)) & 0xFFFFu) | (((b_lo >> (16 * h)) & 0xFFFFu) << 16);
    const uint32_t w1 = ((a_hi >> (16 * h)) & 0xFFFFu) | (((b_hi >> (16 * h)) & 0xFFFFu) << 16);
    *reinterpret_cast<uint2*>(meta + (int64_t)blk * 64 + 2 * lane) = make_uint2(w0, w1);
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

// 2:4 decompress from tiled metadata: one thread per word -> 2 x 16 weights.
__device__ __forceinline__ void decompress_half16(const uint16_t* __restrict__ vrow, uint16_t* __restrict__ wrow,
                                                  uint32_t nibs, uint32_t k0, uint32_t K, bool vec) {
  uint32_t out[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t nib = (nibs >> (4 * t)) & 0xFu;
    const uint32_t p0 = nib & 3u, p1 = nib >> 2;
    uint32_t v = 0;
    if (k0 + 4 * t < K) v = *reinterpret_cast<const uint32_t*>(vrow + k0 / 2 + 2 * t);
    const uint32_t v0 = v & 0xFFFFu, v1 = v >> 16;
    uint32_t e[4];
#pragma unroll
    for (uint32_t i = 0; i < 4; ++i) e[i] = (i == p0) ? v0 : (i == p1) ? v1 : 0u;
    out[2 * t] = e[0] | (e[1] << 16);
    out[2 * t + 1] = e[2] | (e[3] << 16);
  }
  if (vec && k0 + 16 <= K) {
    uint4* dst = reinterpret_cast<uint4*>(wrow + k0);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  } else {
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (k0 + 4 * t < K) {
        *reinterpret_cast<uint32_t*>(wrow + k0 + 4 * t) = out[2 * t];
        *reinterpret_cast<uint32_t*>(wrow + k0 + 4 * t + 2) = out[2 * t + 1];
      }
  }
}

__global__ void __launch_bounds__(256) decompress_2of4_tiled_kernel(const uint16_t* __restrict__ V,
                                                                    const uint32_t* __restrict__ meta, uint32_t R,
                                                                    uint32_t K, uint16_t* __restrict__ W,
                                                                    int64_t ldw, uint32_t cblocks, uint32_t total,
                                                                    bool vec) {
  for (uint32_t w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += gridDim.x * blockDim.x) {
    const uint32_t blk = w >> 6, wi = w & 63u;
    const uint32_t l = wi >> 2, q = wi & 3u;
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint32_t r_lo = rb * 16 + (l & 7u);
    const uint32_t k0 = cb * 128 + q * 32 + (l >> 3) * 16;
    if (k0 >= K) continue;
    const uint32_t word = __ldg(meta + w);
    if (r_lo < R)
      decompress_half16(V + (int64_t)r_lo * (K >> 1), W + (int64_t)r_lo * ldw, word & 0xFFFFu, k0, K, vec);
    if (r_lo + 8 < R)
      decompress_half16(V + (int64_t)(r_lo + 8) * (K >> 1), W + (int64_t)(r_lo + 8) * ldw, word >> 16, k0, K, vec);
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

// Row gather Xp[k][0..T) = X[idx[k]][0..T): one warp per row, 16-byte pieces,
// all of a lane's pieces loaded before any is stored.  Entries of idx outside
// [0, K) give zero rows.  X and Xp rows are 16-byte aligned (T % 8 == 0 on
// the vector path).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ X, int64_t ldx,
                                                          const int32_t* __restrict__ idx, int64_t K, int64_t T,
                                                          uint16_t* __restrict__ Xp, int64_t ldp) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t pieces = T >> 3;  // 16-byte pieces per row
  for (int64_t k = warp; k < K; k += nwarps) {
    const int32_t src = __ldg(idx + k);
    const bool valid = src >= 0 && (int64_t)src < K;
    const uint4* in = reinterpret_cast<const uint4*>(X + (valid ? (int64_t)src : 0) * ldx);
    uint4* out = reinterpret_cast<uint4*>(Xp + k * ldp);
    for (int64_t c0 = 0; c0 < pieces; c0 += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t c = c0 + u * 32 + lane;
        v[u] = (valid && c < pieces) ? __ldg(in + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t c = c0 + u * 32 + lane;
        if (c < pieces) out[c] = v[u];
      }
    }
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
  if (tiled_meta(n, m)) {
    const int64_t nblocks = meta_row_blocks(R) * meta_col_blocks(K);
    const bool vec = K % 16 == 0 && ldw % 8 == 0 && aligned16(W) && aligned16(values);
    compress_2of4_tiled_kernel<<<grid_for(nblocks * 32, threads), threads, 0, s>>>(
        W, (uint32_t)R, (uint32_t)K, ldw, values, meta, (uint32_t)meta_col_blocks(K), (uint32_t)nblocks, vec);
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
  if (tiled_meta(n, m)) {
    const int64_t total = meta_words(R, K, n, m);
    const bool vec = K % 16 == 0 && ldw % 8 == 0 && aligned16(W_out) && aligned16(values);
    decompress_2of4_tiled_kernel<<<grid_for(total, threads), threads, 0, s>>>(
        values, meta, (uint32_t)R, (uint32_t)K, W_out, ldw, (uint32_t)meta_col_blocks(K), (uint32_t)total, vec);
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

cudaError_t launch_gather_rows(const uint16_t* X, int64_t ldx, const int32_t* idx, int64_t K, int64_t T,
                               uint16_t* Xp, int64_t ldp, cudaStream_t s) {
  const int threads = 256;
  gather_rows_kernel<<<grid_for(K * 32, threads), threads, 0, s>>>(X, ldx, idx, K, T, Xp, ldp);
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
