// nm_spmm.h -- parameter block of the tcgen05 GEMM kernel (internal).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"

namespace nmk {

enum AMode : int {
  A_TMA_SPARSE = 0,    // 2:4 values by TMA, metadata re-laid by the builders
  A_BUILD_SPARSE = 1,  // builders re-encode an N:M row segment as 2:4 (values + metadata)
  A_BUILD_DENSE = 2,   // builders expand an N:M row segment into a dense tile
  A_HYBRID = 3         // per 128x128 tile: dense W by TMA, or 2:4 values by TMA
};

// Height of the A and B boxes of the SM-pair kernel: each stage's 128 rows
// of values and 128 rows of X arrive as 64-row boxes from separate warps.
constexpr uint32_t kPairBoxRows = 64;

enum Pattern : int { PAT_2_4 = 0, PAT_1_2 = 1, PAT_1_4 = 2, PAT_1_8 = 3, PAT_2_8 = 4, PAT_OTHER = 5 };

struct SpmmParams {
  CUtensorMap tm_vals;  // compressed values R x K*n/m, box {32, 128} 64B swizzle (one SM) or {64, kPairBoxRows} 128B (SM pair)
  CUtensorMap tm_w;     // dense W R x K, box {64, 128}, 128B swizzle (hybrid)
  CUtensorMap tm_x;     // X K x T, box {strip, 64} (one SM) or {64, kPairBoxRows} (SM pair)
  CUtensorMap tm_wm;    // W under the 2:4 mask (staged), box {64, 64}, 128B swizzle (SM-pair hybrid)
  CUtensorMap tm_y;     // Y R x T bf16, box {64, 32}, 128B swizzle (SM-pair epilogue stores)
  CUtensorMap tm_y32;   // Y R x T bf16, box {32, 32}, no swizzle (last 32 columns of a 224-column SM-pair tile)
  CUtensorMap tm_meta;  // tiled 2:4 metadata {64 words, col blocks, row blocks}, box {64, 1, 8} (SM pair)
  const uint16_t* vals;
  const uint32_t* meta;
  const int32_t* idx;
  const uint16_t* X;  // K x T, row stride ldx (read directly when permuted)
  int64_t ldx;
  const uint8_t* tile_map;
  void* Y;
  uint32_t* status;
  int64_t ldy;
  int64_t R, K, T;
  int64_t vcols, mcols;             // mcols: row-wise patterns
  int64_t meta_rblocks, meta_cblocks; // tiled 2:4 metadata blocks (16 rows x 128 columns)
  int64_t k_tiles;
  int n, m;
  int pattern;
  int a_mode;
  int permuted;
  int out_f32;
  int tiles_m, tiles_n, num_tiles;
  int n_major;  // SM-pair kernel: column tiles go fastest (set when the compressed weights are larger than X)
  int hyb_tiles_k;
  int hyb_rows;  // tile-map rows, ceil(R / 128)
  int stages;
  uint32_t a_slot_bytes;
  // skinny (small T) split-K kernel: K tiles of 128 split into `splits`
  // ranges of `kt_per_split`; fp32 partials in ws[splits][R][bn] when splits > 1
  int splits;
  int kt_per_split;
  int bn;
  int kd;  // skinny stage depth (logical K per stage: 128 or 256)
  float* ws;
  // fused prune + compress + GEMM: optional outputs of the compressed operand
  uint16_t* out_vals;
  uint32_t* out_meta;
};

// Dense bf16 GEMM on SM pairs for the backward products: C (M x N) = A (M x Kr) B (Kr x N),
// fp32 accumulation.  A and B are read with TMA boxes of 64 x 64 (128-byte swizzle), K-major
// (the reduction axis contiguous) or MN-major.  Epilogue 0 stores C, row m of C going to row
// row_map[m] of `out` when row_map is set (rows mapped outside [0, rows_out) are dropped);
// epilogue 1 stores only the entries at the survivor columns of an N:M pattern of an
// M x N weight (meta), as out[m][j] for survivor j of row m.
struct DenseParams {
  CUtensorMap tm_a, tm_b;
  CUtensorMap tm_b_alt;     // read instead of tm_b when use_alt is set and *use_alt is nonzero at run time
  CUtensorMap tm_out;       // epilogue 0 with tma_store: C (M x N), box {64 bf16 | 32 four-byte, 32 rows}, 128B swizzle
  const uint32_t* use_alt;
  int tma_store;            // epilogue 0 without row_map: whole-line TMA stores through tm_out
  int64_t M, N, Kr;
  int64_t k_tiles;
  int tiles_m, tiles_n, num_tiles;
  int n_major;  // tile order: column tiles fastest, so pairs running together share A's row block (A larger than B)
  uint32_t* status;
  void* out;
  int64_t ldo;
  int out_f32;
  const int32_t* row_map;
  int64_t rows_out;
  const uint32_t* meta;
  int n, m;
  int64_t vcols, mcols, meta_cblocks;
  int vec_out;  // epilogue 1, 2:4: K % 16 == 0 and `out` 16-byte aligned (vector stores of whole chunks)
};
enum DenseEpi : int { EPI_STORE = 0, EPI_SURVIVORS = 1 };
cudaError_t launch_dense_pair(const DenseParams& p, bool a_mn, bool b_mn, int epi, cudaStream_t stream);
cudaError_t launch_dense_pair_i8(const DenseParams& p, cudaStream_t stream);
cudaError_t launch_dense_pair_tf32(const DenseParams& p, cudaStream_t stream);
// 1:2 float32 operand for the TF32 path (values R x K/2, metadata R x ceil(K/64) words, one bit per survivor).
cudaError_t launch_compress_tf32(const float* W, int64_t R, int64_t K, int64_t ldw, float* values, uint32_t* meta,
                                 cudaStream_t s);
cudaError_t launch_decompress_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, float* W_out,
                                   int64_t ldw, cudaStream_t s);
cudaError_t launch_diag_select(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D, float* part,
                               float* scores, uint8_t* keep, int32_t* offsets, uint16_t* values, cudaStream_t s);
// Dense copy of a diagonal operand, columns [0, K) of rows [0, R) of W_out.
// `tables` is device scratch of diag_table_words(K, idx != nullptr) words.
// With idx: when idx is a permutation of [0, K) the copy's columns are placed
// through it (column idx[k] holds what column k would), so that the product
// with X equals the product of the plain copy with X[idx]; the word returned
// in *is_perm (inside `tables`) is nonzero exactly then.
int64_t diag_table_words(int64_t K, bool with_idx);
cudaError_t launch_diag_dense(const uint16_t* V, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                              const int32_t* idx, int32_t* tables, uint16_t* W_out, int64_t ldw, cudaStream_t s,
                              const uint32_t** is_perm);
cudaError_t launch_compress_i8(const int8_t* W, int64_t R, int64_t K, int64_t ldw, int8_t* values, uint32_t* meta,
                               cudaStream_t s);
cudaError_t launch_decompress_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, int8_t* W_out,
                                 int64_t ldw, cudaStream_t s);

int spmm_max_stages(int bn, uint32_t a_slot);
cudaError_t launch_spmm(SpmmParams& p, int bn, cudaStream_t stream);
cudaError_t read_and_clear_status(uint32_t* out);
cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream);
uint32_t* status_word_ptr();
bool pair_kernel_fits(const SpmmParams& p);
cudaError_t launch_spmm_pair(SpmmParams& p, cudaStream_t stream);
cudaError_t launch_spmm_pair_hybrid(SpmmParams& p, cudaStream_t stream);
// INT8 2:4 on SM pairs (sparse kind::i8): tm_vals int8 values R x K/2 (box {128, 64}), tm_x int8 X (box
// {128, 64}), tm_meta the re-laid-out metadata as rows of 256 bytes (box {256, 16}), meta_cblocks = its
// 256-column K blocks; int32 results through the fp32 store path (out_f32 = 1).
cudaError_t launch_spmm_pair_i8(SpmmParams& p, cudaStream_t stream);
cudaError_t launch_relayout_meta_i8(const uint32_t* meta, int64_t R, int64_t K, uint32_t* out, int64_t rblocks128,
                                    cudaStream_t s);
// TF32 1:2 on SM pairs (sparse kind::tf32): tm_vals fp32 values R x K/2 (box {32, 64}), tm_x fp32 X (box {32, 64},
// 128-byte swizzle in 32-byte units), tm_meta the re-laid-out metadata (box {256, 16}), meta_cblocks = its 64-deep
// K blocks; Y bf16 or fp32.
cudaError_t launch_spmm_pair_tf32(SpmmParams& p, cudaStream_t stream);
cudaError_t launch_relayout_meta_tf32(const uint32_t* meta, int64_t R, int64_t K, uint32_t* out, int64_t rblocks128,
                                      cudaStream_t s);
bool skinny_kernel_fits(int64_t T);
int skinny_bn(int64_t T);
int skinny_kd(int64_t K, int64_t T);
cudaError_t launch_spmm_skinny(SpmmParams& p, cudaStream_t stream);
cudaError_t launch_skinny_reduce(const SpmmParams& p, cudaStream_t stream);
cudaError_t launch_prune_spmm_skinny(SpmmParams& p, cudaStream_t stream);
cudaError_t launch_compress_stream(const CUtensorMap& tm_w, int64_t R, int64_t K, uint16_t* values, uint32_t* meta,
                                   uint32_t* status, cudaStream_t s, const GatherJob* gather = nullptr);

}  // namespace nmk
