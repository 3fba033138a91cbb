// nm_int8.cu -- 2:4 structured sparsity on INT8 weights.
//
// "M:N sparsity on NVIDIA tensor cores": the sparse tensor cores take 2:4 for
// FP16, BF16 and INT8 weights, and with a 2-bit index per stored value an INT8
// 2:4 matrix keeps 62.5 % of its dense bytes.  The selection rule is the one of
// the bf16 path on int8 magnitudes (|-128| = 128 ranks above 127, equal
// magnitudes to the lower index); values are pushed left (R x K/2 int8) and the
// positions use the same tiled 2:4 metadata as bf16.  Requires K % 16 == 0.
//
// compress_2of4_i8_kernel: one warp per 16-row x 128-column block; lane
// (half, piece) takes rows 2i + half and columns 8*piece .. +7 (two groups),
// the block's 64 metadata words assembled with shuffles as in the bf16 kernel.
// decompress_2of4_i8_kernel: one thread per metadata word (two rows x 16
// columns), 16-byte stores of the dense rows.
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

// One group of four int8 (bytes of v): returns p0 | p1 << 2 (p0 < p1) and in
// `pk` the two survivors in bytes 0 and 1.  Composite keys |v_i| * 4 + (3 - i)
// are distinct; the two largest win (max/min of each pair, then the larger
// maximum and the larger of the smaller maximum and the larger minimum).
__device__ __forceinline__ uint32_t select_pair_i8(uint32_t v, uint32_t& pk) {
  const uint32_t m = __vabs4(v);  // per-byte |v|; -128 gives 0x80 = 128
  const uint32_t c0 = ((m & 0xFFu) << 2) | 3u, c1 = (((m >> 8) & 0xFFu) << 2) | 2u;
  const uint32_t c2 = (((m >> 16) & 0xFFu) << 2) | 1u, c3 = (m >> 24) << 2;
  const uint32_t m01 = max(c0, c1), n01 = min(c0, c1), m23 = max(c2, c3), n23 = min(c2, c3);
  const uint32_t top = max(m01, m23), second = max(min(m01, m23), max(n01, n23));
  const uint32_t pa = (top & 3u) ^ 3u, pb = (second & 3u) ^ 3u;
  const uint32_t p0 = min(pa, pb), p1 = max(pa, pb);
  pk = __byte_perm(v, 0u, p0 | (p1 << 4) | 0x4400u) & 0xFFFFu;
  return p0 | (p1 << 2);
}

__global__ void __launch_bounds__(256) compress_2of4_i8_kernel(const int8_t* __restrict__ W, uint32_t R, uint32_t K,
                                                              int64_t ldw, int8_t* __restrict__ V,
                                                              uint32_t* __restrict__ meta, uint32_t cblocks,
                                                              uint32_t nblocks) {
  pdl_gate();
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t half = lane >> 4, piece = lane & 15u;
  for (uint32_t blk = warp; blk < nblocks; blk += nwarps) {
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint32_t col = cb * 128 + 8 * piece;
    uint2 in[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t row = rb * 16 + 2 * i + half;
      in[i] = (row < R && col < K) ? __ldg(reinterpret_cast<const uint2*>(W + (int64_t)row * ldw + col))
                                   : make_uint2(0u, 0u);
    }
    uint32_t lo8 = 0, hi8 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t row = rb * 16 + 2 * i + half;
      uint32_t pa, pb;
      const uint32_t byte = select_pair_i8(in[i].x, pa) | (select_pair_i8(in[i].y, pb) << 4);
      if (row < R && col < K)
        *reinterpret_cast<uint32_t*>(V + (int64_t)row * (K >> 1) + col / 2) = pa | (pb << 16);
      if (i < 4) lo8 |= byte << (8 * i);
      else hi8 |= byte << (8 * (i - 4));
    }
    // metadata words: the same assembly as the bf16 compress (rows of a zero group select (0, 1) = 0x4)
    const uint32_t l = lane >> 1, r = l & 7u, h = l >> 3, k = r >> 1;
    const uint32_t s0 = 16 * (r & 1u) + 8 * (lane & 1u) + 2 * h;
    const uint32_t a0 = __shfl_sync(0xffffffffu, lo8, s0), a1 = __shfl_sync(0xffffffffu, lo8, s0 + 1);
    const uint32_t b0 = __shfl_sync(0xffffffffu, hi8, s0), b1 = __shfl_sync(0xffffffffu, hi8, s0 + 1);
    const uint32_t c0 = __shfl_sync(0xffffffffu, lo8, s0 + 4), c1 = __shfl_sync(0xffffffffu, lo8, s0 + 5);
    const uint32_t d0 = __shfl_sync(0xffffffffu, hi8, s0 + 4), d1 = __shfl_sync(0xffffffffu, hi8, s0 + 5);
    const uint32_t pick = k | ((k + 4) << 4);
    const uint32_t w0 = __byte_perm(__byte_perm(a0, a1, pick), __byte_perm(b0, b1, pick), 0x5410u);
    const uint32_t w1 = __byte_perm(__byte_perm(c0, c1, pick), __byte_perm(d0, d1, pick), 0x5410u);
    *reinterpret_cast<uint2*>(meta + (int64_t)blk * 64 + 2 * lane) = make_uint2(w0, w1);
  }
}

// One thread per tiled metadata word: rows 16rb + (l % 8) (bits 0..15) and
// 16rb + 8 + (l % 8) (bits 16..31), columns 128cb + 32q + 16h .. +15.
__global__ void __launch_bounds__(256) decompress_2of4_i8_kernel(const int8_t* __restrict__ V,
                                                                const uint32_t* __restrict__ meta, uint32_t R,
                                                                uint32_t K, int8_t* __restrict__ Wout, int64_t ldw,
                                                                uint32_t cblocks, uint32_t total) {
  pdl_gate();
  for (uint32_t w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += gridDim.x * blockDim.x) {
    const uint32_t blk = w >> 6, i = w & 63u, l = i >> 2, q = i & 3u;
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint32_t c0 = cb * 128 + 32 * q + 16 * (l >> 3);
    if (c0 >= K) continue;
    const uint32_t word = __ldg(meta + w);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t row = rb * 16 + 8 * hh + (l & 7u);
      if (row >= R) continue;
      const uint2 vals = __ldg(reinterpret_cast<const uint2*>(V + (int64_t)row * (K >> 1) + c0 / 2));
      const uint32_t nib16 = word >> (16 * hh);
      uint32_t out[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const uint32_t nib = (nib16 >> (4 * g)) & 0xFu, p0 = nib & 3u, p1 = nib >> 2;
        const uint32_t src = g < 2 ? vals.x : vals.y;
        const uint32_t b0 = (src >> (16 * (g & 1))) & 0xFFu, b1 = (src >> (16 * (g & 1) + 8)) & 0xFFu;
        out[g] = (b0 << (8 * p0)) | (b1 << (8 * p1));
      }
      *reinterpret_cast<uint4*>(Wout + (int64_t)row * ldw + c0) = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

// Metadata of the sparse kind::i8 MMA.  That MMA reads its positions per row in
// plain K order (TMEM lane = row; the 16 groups of one K = 64 step in two
// columns, group g at column g / 8, bits 4 (g % 8)), unlike the kind::f16 order
// of the stored tiled words (rows r and r + 8 share a word).  This pass
// rewrites the tiled words, per 128-row block and 256-column K block, into one
// 4 KB chunk that tcgen05.cp (128 lanes x 256 bits, no swizzle) moves into 8
// TMEM columns: row r's 32 bytes (64 groups, two per byte, low nibble first)
// as two 16-byte halves, half c of rows 8j .. 8j + 7 at 256 j + 128 c.
// Groups or rows outside the tiled words (padding) get the nibble 0x4.
// One thread per output 16-byte half (row r, half c: words 4c .. 4c + 3, groups
// 32c .. 32c + 31 of the chunk's 64): they are the 16-bit row halves of four
// consecutive tiled words (lo) and of the four 32 words later (hi), so a thread
// makes two 16-byte loads (four 4-byte ones each when meta is not 16-byte
// aligned, vec == false) and one 16-byte store.
__global__ void __launch_bounds__(256) relayout_meta_i8_kernel(const uint32_t* __restrict__ meta, uint32_t rblocks16,
                                                              uint32_t cblocks128, uint32_t kblocks256,
                                                              uint32_t* __restrict__ out, uint32_t total, bool vec) {
  pdl_gate();
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t chunk = i >> 8, within = i & 255u;  // 256 halves per chunk
    const uint32_t r = within >> 1, c = within & 1u;   // row of the 128, half of the row's two
    const uint32_t rb128 = chunk / kblocks256, kb = chunk - rb128 * kblocks256;
    const uint32_t row = rb128 * 128 + r;
    const uint32_t rb = row >> 4, cb = 2 * kb + c;     // tiled block: 16 rows x 128 columns (32 groups)
    uint4 v = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    if (rb < rblocks16 && cb < cblocks128) {
      const uint32_t* src = meta + (rb * cblocks128 + cb) * 64 + 4 * (row & 7u);
      uint4 lo, hi;  // quarters 0..3 of rows (row & 7) and +8: groups 8q .. 8q + 3; lane + 8: groups 8q + 4 .. 8q + 7
      if (vec) {
        lo = __ldg(reinterpret_cast<const uint4*>(src));
        hi = __ldg(reinterpret_cast<const uint4*>(src + 32));
      } else {
        lo = make_uint4(__ldg(src), __ldg(src + 1), __ldg(src + 2), __ldg(src + 3));
        hi = make_uint4(__ldg(src + 32), __ldg(src + 33), __ldg(src + 34), __ldg(src + 35));
      }
      const uint32_t sh = 16 * ((row >> 3) & 1u);
      auto join = [&](uint32_t l, uint32_t h) { return ((l >> sh) & 0xFFFFu) | (((h >> sh) & 0xFFFFu) << 16); };
      v = make_uint4(join(lo.x, hi.x), join(lo.y, hi.y), join(lo.z, hi.z), join(lo.w, hi.w));
    }
    // words 4c .. 4c + 3 of row r at byte 128 c + 16 (r % 8) of the 8-row group r / 8
    *reinterpret_cast<uint4*>(out + (int64_t)chunk * 1024 + (r >> 3) * 64 + c * 32 + (r & 7u) * 4) = v;
  }
}

cudaError_t launch_relayout_meta_i8(const uint32_t* meta, int64_t R, int64_t K, uint32_t* out, int64_t rblocks128,
                                    cudaStream_t s) {
  const int64_t kblocks256 = (K + 255) / 256;
  const int64_t total = rblocks128 * kblocks256 * 256;
  const int64_t want = (total + 255) / 256;
  const int64_t cap = (int64_t)sm_count_current() * 8;
  const int grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
  cudaError_t e = launch_pdl(relayout_meta_i8_kernel, dim3(grid), dim3(256), 0, s, meta, (uint32_t)meta_row_blocks(R),
                             (uint32_t)meta_col_blocks(K), (uint32_t)kblocks256, out, (uint32_t)total,
                             (reinterpret_cast<uintptr_t>(meta) & 15u) == 0);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_compress_i8(const int8_t* W, int64_t R, int64_t K, int64_t ldw, int8_t* values, uint32_t* meta,
                               cudaStream_t s) {
  const int64_t cblocks = meta_col_blocks(K), nblocks = meta_row_blocks(R) * cblocks;
  const int64_t warps_per_cta = 8;
  const int64_t want = (nblocks + warps_per_cta - 1) / warps_per_cta;
  const int64_t cap = (int64_t)sm_count_current() * 8;
  const int grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
  cudaError_t e = launch_pdl(compress_2of4_i8_kernel, dim3(grid), dim3(256), 0, s, W, (uint32_t)R, (uint32_t)K, ldw,
                             values, meta, (uint32_t)cblocks, (uint32_t)nblocks);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_decompress_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, int8_t* W_out,
                                 int64_t ldw, cudaStream_t s) {
  const int64_t cblocks = meta_col_blocks(K);
  const int64_t total = meta_row_blocks(R) * cblocks * 64;
  const int64_t want = (total + 255) / 256;
  const int64_t cap = (int64_t)sm_count_current() * 8;
  const int grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
  cudaError_t e = launch_pdl(decompress_2of4_i8_kernel, dim3(grid), dim3(256), 0, s, values, meta, (uint32_t)R,
                             (uint32_t)K, W_out, ldw, (uint32_t)cblocks, (uint32_t)total);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nmk
