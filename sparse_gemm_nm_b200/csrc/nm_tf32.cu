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
// Compress: one warp per 64 pairs of a row (two metadata words), 16 bytes
// per lane in, 8 bytes out; decompress: one thread per two pairs, 8 bytes in,
// 16 bytes out (scalar accesses where rows are not aligned).  The GEMM
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

// One warp per 64 pairs (two metadata words) of a row: lane l takes pairs 2l and 2l + 1 (one 16-byte load
// when rows are 16-byte aligned), writes both survivors (8 bytes), and the 16 lanes of each half OR their
// position bits into that half's metadata word.
__global__ void __launch_bounds__(256) compress_1of2_f32_kernel(const uint32_t* __restrict__ W, int64_t R, int64_t K,
                                                               int64_t ldw, uint32_t* __restrict__ values,
                                                               uint32_t* __restrict__ meta, int vec_in, int vec_out) {
  pdl_gate();
  const int lane = threadIdx.x & 31;
  const int64_t pairs = K / 2, words = (pairs + 31) / 32, items = (words + 1) / 2;
  const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t w = warp0; w < R * items; w += nwarps) {
    const int64_t r = w / items, q = w - r * items;
    const int64_t p0 = 64 * q + 2 * lane;
    const bool v0 = p0 < pairs, v1 = p0 + 1 < pairs;
    const uint32_t* src = W + r * ldw + 2 * p0;
    uint32_t e0 = 0, e1 = 0, e2 = 0, e3 = 0;
    if (vec_in && v1) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
      e0 = v.x, e1 = v.y, e2 = v.z, e3 = v.w;
    } else {
      if (v0) e0 = __ldg(src), e1 = __ldg(src + 1);
      if (v1) e2 = __ldg(src + 2), e3 = __ldg(src + 3);
    }
    const uint32_t pa = f32_key(e0) >= f32_key(e1) ? 0u : 1u, pb = f32_key(e2) >= f32_key(e3) ? 0u : 1u;
    const uint32_t sa = pa ? e1 : e0, sb = pb ? e3 : e2;
    uint32_t* dst = values + r * pairs + p0;
    if (vec_out && v1) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(sa, sb);
    } else {
      if (v0) dst[0] = sa;
      if (v1) dst[1] = sb;
    }
    uint32_t c = ((v0 ? pa : 0u) << ((2 * lane) & 31)) | ((v1 ? pb : 0u) << ((2 * lane + 1) & 31));
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) c |= __shfl_xor_sync(0xffffffffu, c, off);  // within each 16-lane half
    const int64_t word = 2 * q + (lane >> 4);
    if ((lane & 15) == 0 && word < words) meta[r * words + word] = c;
  }
}

// One thread per two pairs (16 bytes of output): W_out[r][2p + bit] = values[r][p], +0.0 at the other position.
__global__ void __launch_bounds__(256) decompress_1of2_f32_kernel(const uint32_t* __restrict__ values,
                                                                 const uint32_t* __restrict__ meta, int64_t R,
                                                                 int64_t K, uint32_t* __restrict__ W_out,
                                                                 int64_t ldw, int vec_in, int vec_out) {
  pdl_gate();
  const int64_t pairs = K / 2, words = (pairs + 31) / 32, halves = (pairs + 1) / 2;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < R * halves;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / halves, p0 = 2 * (i - r * halves);
    const bool v1 = p0 + 1 < pairs;
    const uint32_t word = __ldg(meta + r * words + p0 / 32);
    const uint32_t ba = (word >> (p0 % 32)) & 1u, bb = (word >> ((p0 + 1) % 32)) & 1u;
    const uint32_t* vsrc = values + r * pairs + p0;
    uint32_t va, vb = 0;
    if (vec_in && v1) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(vsrc));
      va = v.x, vb = v.y;
    } else {
      va = __ldg(vsrc);
      if (v1) vb = __ldg(vsrc + 1);
    }
    uint32_t* dst = W_out + r * ldw + 2 * p0;
    const uint4 o = make_uint4(ba ? 0u : va, ba ? va : 0u, bb ? 0u : vb, bb ? vb : 0u);
    if (vec_out && v1) {
      *reinterpret_cast<uint4*>(dst) = o;
    } else {
      dst[0] = o.x, dst[1] = o.y;
      if (v1) dst[2] = o.z, dst[3] = o.w;
    }
  }
}

// Metadata of the sparse kind::tf32 MMA (TMEM order in tc_mma_sp_pair_tf32): per 128-row block and
// 64-deep K stage (32 pairs: one stored word per row), one 4 KB chunk that tcgen05.cp (128 lanes x 256
// bits, no swizzle) moves into 8 TMEM columns; the four K = 16 steps of the stage take columns 0, 2, 4, 6
// (odd columns stay 0).  Lane L of the chunk: rows 16 (L / 16) + L % 8 and + 8, pairs 4 ((L % 16) / 8) ..
// + 3 of each step.  Pairs or rows outside R x K/2 get the nibble 0x4 (their values are zero).  Chunk
// layout as the int8 one: half c of lanes 8j .. 8j + 7 at 256 j + 128 c, 16 bytes per lane.
__global__ void __launch_bounds__(256) relayout_meta_tf32_kernel(const uint32_t* __restrict__ meta, int64_t R,
                                                                int64_t npairs, int64_t mcols, uint32_t kblocks,
                                                                uint32_t* __restrict__ out, uint32_t total) {
  pdl_gate();
  // one thread per (chunk, lane L): its four metadata words (even columns) and four zeros, two 16-byte stores
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t chunk = i >> 7, L = i & 127u;
    const uint32_t rb128 = chunk / kblocks, kb = chunk - rb128 * kblocks;
    const uint32_t l = L & 15u, h = l >> 3;
    const int64_t r0 = (int64_t)rb128 * 128 + 16 * (L >> 4) + (l & 7u);
    uint32_t m[2] = {0u, 0u};  // the stage's stored word of rows r0 and r0 + 8 (bit p: position of pair p)
    int64_t valid[2] = {0, 0};  // pairs of the stage inside K / 2
    const int64_t p0 = (int64_t)kb * 32;
    const int64_t inside = npairs - p0 < 32 ? npairs - p0 : 32;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int64_t r = r0 + 8 * half;
      if (r < R && inside > 0) {
        m[half] = __ldg(meta + r * mcols + kb);
        valid[half] = inside;
      }
    }
    uint32_t w[4];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t word = 0x44444444u;
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int q = kk * 8 + 4 * (int)h + t;  // pair of the stage
          if (q < valid[half] && ((m[half] >> q) & 1u)) word ^= 0xAu << (16 * half + 4 * t);  // 0x4 -> 0xE
        }
      w[kk] = word;
    }
    // words 0..7 of lane L: half c (words 4c .. 4c + 3) at 256 (L / 8) + 128 c + 16 (L % 8) bytes
    uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)chunk * 1024 + (L >> 3) * 64 + (L & 7u) * 4);
    dst[0] = make_uint4(w[0], 0u, w[1], 0u);
    dst[8] = make_uint4(w[2], 0u, w[3], 0u);
  }
}

cudaError_t launch_relayout_meta_tf32(const uint32_t* meta, int64_t R, int64_t K, uint32_t* out, int64_t rblocks128,
                                      cudaStream_t s) {
  const int64_t kblocks = (K + 63) / 64;
  const int64_t total = rblocks128 * kblocks * 128;  // one thread per chunk lane
  const int64_t npairs = K / 2, mcols = (npairs + 31) / 32;
  cudaError_t e = launch_pdl(relayout_meta_tf32_kernel, dim3(grid_of(total, 256)), dim3(256), 0, s, meta, R, npairs,
                             mcols, (uint32_t)kblocks, out, (uint32_t)total);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

static int aligned16_rows(const void* p, int64_t ld) { return (reinterpret_cast<uintptr_t>(p) % 16 == 0 && ld % 4 == 0) ? 1 : 0; }
static int aligned8_rows(const void* p, int64_t ld) { return (reinterpret_cast<uintptr_t>(p) % 8 == 0 && ld % 2 == 0) ? 1 : 0; }

cudaError_t launch_compress_tf32(const float* W, int64_t R, int64_t K, int64_t ldw, float* values, uint32_t* meta,
                                 cudaStream_t s) {
  const int64_t warps = R * (((K / 2 + 31) / 32 + 1) / 2);
  cudaError_t e = launch_pdl(compress_1of2_f32_kernel, dim3(grid_of(warps * 32, 256)), dim3(256), 0, s,
                             reinterpret_cast<const uint32_t*>(W), R, K, ldw, reinterpret_cast<uint32_t*>(values),
                             meta, aligned16_rows(W, ldw), aligned8_rows(values, K / 2));
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decompress_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, float* W_out,
                                   int64_t ldw, cudaStream_t s) {
  cudaError_t e = launch_pdl(decompress_1of2_f32_kernel, dim3(grid_of(R * ((K / 2 + 1) / 2), 256)), dim3(256), 0, s,
                             reinterpret_cast<const uint32_t*>(values), meta, R, K,
                             reinterpret_cast<uint32_t*>(W_out), ldw, aligned8_rows(values, K / 2),
                             aligned16_rows(W_out, ldw));
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nmk
