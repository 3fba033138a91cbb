// nm_internal.h -- declarations shared by the host entry points and the
// kernel launchers of libnm_b200 (not part of the public ABI).
#pragma once
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

namespace nmk {

// Bits per stored position and positions per 32-bit word for a group of m.
inline int index_bits(int m) { return m == 2 ? 1 : m == 4 ? 2 : m == 8 ? 3 : m == 16 ? 4 : 0; }
inline int positions_per_word(int m) { return 32 / index_bits(m); }
inline bool pattern_ok(int n, int m) { return index_bits(m) > 0 && n >= 1 && n < m; }
inline int64_t value_cols(int64_t K, int n, int m) { return K / m * n; }
inline int64_t meta_cols(int64_t K, int n, int m) {
  const int64_t s = positions_per_word(m);
  return (value_cols(K, n, m) + s - 1) / s;
}
// 2:4 metadata is tiled for the sparse tensor core: 64 words per block of
// 16 rows x 128 columns, rows and columns padded up to whole blocks.
inline bool tiled_meta(int n, int m) { return n == 2 && m == 4; }
inline int64_t meta_row_blocks(int64_t R) { return (R + 15) / 16; }
inline int64_t meta_col_blocks(int64_t K) { return (K + 127) / 128; }
inline int64_t meta_words(int64_t R, int64_t K, int n, int m) {
  return tiled_meta(n, m) ? meta_row_blocks(R) * meta_col_blocks(K) * 64 : R * meta_cols(K, n, m);
}

// Patterns whose survivors never exceed two per aligned group of four, so a
// tile of them can be re-encoded as 2:4 for the sparse MMA.
inline bool fits_2of4(int n, int m) { return (m == 2 && n == 1) || ((m == 4 || m == 8) && n <= 2); }

// Every kernel of the library is launched as a programmatic dependent of the
// previous kernel in its stream and starts with pdl_gate(): it waits until
// that kernel has completed and its writes are visible (griddepcontrol.wait),
// touching no global memory before, then lets its own successor be scheduled.
// Stream order is unchanged; the successor's launch and setup overlap the tail
// of the kernel before it.
// Gather of permuted input rows, Xp[k] = X[idx[k]] (K x T bf16; an entry of idx
// outside [0, K) gives a zero row).  Work items are (row, 4 KB chunk).
struct GatherJob {
  const uint16_t* X;
  int64_t ldx;
  const int32_t* idx;
  int64_t K, T;
  uint16_t* Xp;
  int64_t ldp;
  const uint32_t* skip_if;  // gather_rows_kernel does nothing when this word is set and nonzero at run time
};

#ifdef __CUDACC__
__device__ __forceinline__ void pdl_gate() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Items warp, warp + nwarps, ... of a gather: each lane moves 16-byte pieces of
// one row; when T % 8 != 0 the partial last piece is read element by element,
// so the reads stay inside the row's T columns.
__device__ __forceinline__ void gather_rows_items(const GatherJob& g, int64_t warp, int64_t nwarps, int lane) {
  const int64_t whole = g.T >> 3;         // 16-byte pieces inside the row's T columns
  const int64_t pieces = (g.T + 7) >> 3;  // + a partial last piece when T % 8 != 0
  const int64_t chunks = (pieces + 255) / 256;
  const int64_t items = g.K * chunks;
  for (int64_t it = warp; it < items; it += nwarps) {
    const int64_t k = it / chunks, c0 = (it - k * chunks) * 256;
    const int32_t src = __ldg(g.idx + k);
    const bool valid = src >= 0 && (int64_t)src < g.K;
    const uint16_t* row = g.X + (valid ? (int64_t)src : 0) * g.ldx;
    const uint4* in = reinterpret_cast<const uint4*>(row);
    uint4* out = reinterpret_cast<uint4*>(g.Xp + k * g.ldp);
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t c = c0 + u * 32 + lane;
      v[u] = (valid && c < whole) ? __ldg(in + c) : make_uint4(0, 0, 0, 0);
      if (valid && c == whole && c < pieces) {  // columns 8c .. T-1 one by one, zeros after them
        uint32_t w[4] = {0, 0, 0, 0};
        for (int64_t j = 0; 8 * c + j < g.T; ++j) w[j >> 1] |= (uint32_t)__ldg(row + 8 * c + j) << (16 * (j & 1));
        v[u] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t c = c0 + u * 32 + lane;
      if (c < pieces) out[c] = v[u];
    }
  }
}
#endif

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int sm_count_current();
void count_launch();

cudaError_t launch_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint16_t* values,
                            uint32_t* meta, cudaStream_t s);
cudaError_t launch_decompress(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K, int n, int m,
                              uint16_t* W_out, int64_t ldw, cudaStream_t s);
// 2:4 decompress of the 128 x 128 tiles that the SM-pair hybrid kernel reads as
// dense tiles: tile_map entry non-zero (tile map ceil(R/128) x ceil(K/128)) and
// the partner row tile (row tile index ^ 1) present and zero in the same column;
// other tiles of W_out are not written.
cudaError_t launch_decompress_tiles(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K,
                                    const uint8_t* tile_map, uint16_t* W_out, int64_t ldw, cudaStream_t s);
// Xp[k] = X[idx[k]] (zero rows for idx outside [0, K)); with skip_if set, the
// launch does nothing when that device word is nonzero when it runs.
cudaError_t launch_gather_rows(const uint16_t* X, int64_t ldx, const int32_t* idx, int64_t K, int64_t T,
                               uint16_t* Xp, int64_t ldp, cudaStream_t s, const uint32_t* skip_if = nullptr);
cudaError_t launch_reencode_2of4(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K, int n, int m,
                                 uint16_t* values2, uint32_t* meta2, cudaStream_t s);
cudaError_t launch_fill_zero(void* Y, int64_t R, int64_t T, int64_t ldy, int esize, cudaStream_t s);

}  // namespace nmk
