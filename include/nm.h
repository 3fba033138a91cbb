/*
 * nm.h -- C ABI of libnm_b200, N:M structured weight sparsity on NVIDIA B200
 * (sm_100a): magnitude prune + push-left compression, decompression, and the
 * sparse x dense GEMM y = (W Pi) x in plain, column-permuted and PATCH-style
 * hybrid forms; further down, the one-call prune + GEMM, the two backward
 * products, INT8 2:4, TF32 1:2 (float32 data) and the diagonal pattern, each
 * with its own conventions where they differ from the ones below.
 *
 * Conventions shared by every call
 *  - bf16 data is passed as its 16-bit pattern (uint16_t).  All matrices are
 *    row-major.  W is R x K (R output features, K the reduction axis), X is
 *    K x T (T tokens, contiguous), Y is R x T.
 *  - An N:M pattern groups M consecutive weights along K.  Supported M is 2,
 *    4, 8 or 16 with 1 <= N < M, and K must be a multiple of M.
 *  - Compressed form ("values" + "meta"):
 *      values  R x (K*N/M) bf16, the N survivors of each group pushed left in
 *              ascending position order; row stride K*N/M.
 *      meta    nm_meta_words(R,K,N,M) uint32 words of in-group positions.
 *        2:4   "tiled": one nibble p0 | p1 << 2 per group (first survivor in
 *              the low bits), tiled in the order a sparse tensor-core MMA
 *              reads them.  Rows go 16 at a time and columns 128 at a time;
 *              block (rb, cb) is 64 words at word (rb*ceil(K/128) + cb)*64.
 *              Word 4*l + q of a block (lane l = 0..15, quarter q = 0..3)
 *              covers block columns 32q + 16h .. 32q + 16h + 15, h = l/8: row
 *              16rb + (l%8) in bits 0..15 and row 16rb + 8 + (l%8) in bits
 *              16..31, four nibbles in column order.  Groups past R or K in
 *              the padded blocks hold 0x4, the positions (0,1) of a zero group.
 *        other "row-wise": survivor j of row r stores its position
 *              (b = ceil(log2 M) bits) in word r*ceil(K*N/M/S) + floor(j/S) at
 *              bit b*(j mod S), S = floor(32/b); unused bits 0.
 *  - Every pointer is DEVICE memory owned by the caller (none is freed or
 *    retained).  The library allocates no device memory, except stream-ordered
 *    staging buffers from its own pool in the calls that document them (the
 *    GEMMs on the two-SM path, the backward, INT8, TF32 and diagonal calls).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are detected on the host and returned
 *    before anything is launched.  Each successful call launches one kernel
 *    (none when the output is empty), except the GEMM calls that stage an
 *    operand first (a re-encoding and/or a gather pass; see nm_spmm).
 *  - Device pointers given to the GEMMs must be 16-byte aligned, and leading
 *    dimensions of X and Y must keep every row 16-byte aligned
 *    (NM_ERR_MISALIGNED otherwise).
 *  - Waits inside the GEMM kernels are bounded (about 2 s); a kernel that gives
 *    up records it in a device status word read by nm_device_status().
 *  - Inputs are expected to be finite.  With an Inf or NaN in X the result may
 *    differ from the sum over stored survivors (zeros padded in by the kernel
 *    can meet it).
 */
#ifndef NM_B200_H
#define NM_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NM_API __attribute__((visibility("default")))
#else
#define NM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nm_status {
  NM_OK = 0,
  NM_ERR_INVALID_ARG = 1, /* null pointer, bad shape or pattern, ld too small */
  NM_ERR_UNSUPPORTED = 2, /* valid request outside what this build implements */
  NM_ERR_MISALIGNED = 3,  /* pointer / leading dimension breaks 16-byte rows   */
  NM_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed              */
  NM_ERR_TIMEOUT = 5,     /* a kernel's bounded wait gave up (device status)   */
  NM_ERR_NO_DEVICE = 6    /* no sm_100 device is current                       */
} nm_status;

typedef enum nm_out_dtype { NM_OUT_BF16 = 0, NM_OUT_F32 = 1 } nm_out_dtype;

/* Kernel design for nm_spmm_algo.  AUTO: 2:4 and patterns that fit inside
 * 2:4 (1:2, 1:4, 1:8, 2:8) use the sparse tensor-core MMA, other patterns the
 * dense expansion. */
typedef enum nm_algo {
  NM_ALGO_AUTO = 0,
  NM_ALGO_SPARSE_TC = 1, /* tcgen05.mma.sp; 1:4 / 1:8 re-encoded as 2:4 while loading */
  NM_ALGO_DENSE_TC = 2   /* survivors expanded into a dense tile, dense tcgen05.mma   */
} nm_algo;

/* ------------------------------------------------------------------ sizes */
/* Bits per stored position, ceil(log2 m); 0 for an unsupported m. */
NM_API int nm_index_bits(int m);
/* Columns of the value block, K*n/m (-1 on a bad pattern or K % m != 0). */
NM_API int64_t nm_value_cols(int64_t K, int n, int m);
/* 32-bit metadata words of an R x K matrix (-1 on a bad pattern or K % m != 0). */
NM_API int64_t nm_meta_words(int64_t R, int64_t K, int n, int m);

/* ------------------------------------------------------------- compress */
/*
 * nm_prune_compress -- keep the n largest-magnitude weights of every group of
 * m consecutive weights along each row of W, ties going to the lower index,
 * and write them in compressed form.
 * Source: "M:N sparsity on NVIDIA tensor cores" -- opening passage (groups of
 * four along a row, two survivors anywhere inside, metadata [[0,3],[1,2]] of
 * the worked row), "The recipe" step 2 (zero the smallest magnitudes), and the
 * storage paragraphs of "Where this sits among the three case studies"
 * (survivors pushed left into an R x C/2 block plus 2-bit positions).
 *   W       [in]  R x K bf16, row stride ldw >= K (elements)
 *   values  [out] R x nm_value_cols(K,n,m) bf16
 *   meta    [out] nm_meta_words(R,K,n,m) uint32, every word written
 * Magnitudes are compared on the bf16 value: +0 and -0 tie, a NaN ranks above
 * every number.  Exactly n survivors are stored per group, zeros included.
 * Errors: NM_ERR_INVALID_ARG (bad pattern, K % m, ldw < K, null pointer).
 */
NM_API nm_status nm_prune_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int n, int m,
                            uint16_t* values, uint32_t* meta, void* stream);

/*
 * nm_decompress -- scatter the survivors back to their positions; every other
 * element becomes +0 (bits 0x0000).  decompress(compress(W)) is W with the
 * pruned weights replaced by +0.
 * Source: same storage paragraphs (a survivor's place follows from its group
 * and its stored position; no pointers are needed).
 *   values, meta [in]  compressed form of an R x K matrix (layout above)
 *   W_out        [out] R x K bf16, row stride ldw >= K
 * Errors: NM_ERR_INVALID_ARG.
 */
NM_API nm_status nm_decompress(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K, int n, int m,
                        uint16_t* W_out, int64_t ldw, void* stream);

/* ----------------------------------------------------------------- GEMM */
/*
 * nm_spmm -- Y = W' X with W' the decompressed weights, computed from the
 * compressed operand (only the weights are compressed; X and Y are dense).
 * Products are exact and accumulate in fp32 on the tensor cores; Y is rounded
 * once (bf16 round-to-nearest-even, or stored as fp32).
 * Source: "M:N sparsity on NVIDIA tensor cores", GEMM paragraphs of "Where
 * this sits among the three case studies" (the indices pick the elements of
 * the dense operand; sparse x dense = dense) and the K-axis rule.
 *   values, meta [in] compressed R x K weights, pattern n:m
 *   X            [in] K x T bf16, row stride ldx >= T, ldx % 8 == 0
 *   Y            [out] R x T, bf16 or fp32 (y_dtype), row stride ldy >= T
 * Kernel choice: shapes with K % 128 == 0, T >= 192 and T % 8 == 0 run on two
 * SMs per 256 x 256 tile (256 x 224 tiles with two accumulators when K <= 1024).
 * 2:4 reads the caller's operand directly.  1:2, 1:4,
 * 1:8 and 2:8 (at most two survivors per aligned group of four) are first
 * re-encoded as 2:4 into a staging buffer (R*K bytes of values plus R*K/8
 * bytes of metadata) from the library's pool (see nm_spmm_permuted and
 * nm_release_staging), one extra launch.  On the same shapes, the dense
 * design (NM_ALGO_DENSE_TC, or any pattern the 2:4 MMA cannot take under
 * NM_ALGO_AUTO) decompresses the operand into a staged dense copy (R*K*2
 * bytes) and runs dense MMAs on SM pairs.  Shapes with K % 128 == 0 and
 * T <= 64 run a split-K kernel (one 128-row tile and one range of K per work
 * unit, persistent over the SMs); when K is split into s > 1 ranges it stages
 * s*R*bn*4 bytes of fp32 partials (bn = T rounded up to 16, 32 or 64) and a
 * second launch sums them in range order.  Every other case runs on one SM
 * per 128-row tile and stages nothing.
 * Errors: NM_ERR_INVALID_ARG, NM_ERR_MISALIGNED, NM_ERR_CUDA.
 */
NM_API nm_status nm_spmm(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                  const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype,
                  void* stream);

/*
 * nm_spmm_permuted -- Y = (W' Pi) X with the hard column permutation Pi given
 * as an index map: row k of the permuted input is X[idx[k]], so
 * y[r][t] = sum_k W'[r][k] * X[idx[k]][t].  The FLOP count is that of
 * nm_spmm, and an identity map gives nm_spmm's result.  How X is read:
 *  - the two-SM path (see nm_spmm): a gather pass first writes
 *    Xp[k] = X[idx[k]] into a staging buffer of K x ceil8(T) bf16, which the
 *    GEMM then streams like X.  The
 *    buffer comes from a stream-ordered pool that the library owns (one per
 *    device) and goes back to it, on `stream`, when the call's kernels are
 *    done; the pool keeps its memory for later calls (high-water mark: the
 *    largest staged bytes of one call, K x ceil8(T) x 2 plus a re-encoded
 *    operand if any, times the calls in flight on different streams) until
 *    nm_release_staging().  A failed allocation returns
 *    NM_ERR_CUDA.
 *  - every other shape: the GEMM kernel reads the mapped rows of X while it
 *    stages its tiles; there is no separate pass and no allocation.
 * Source: "Technische Samenvatting: SHUFFLESPARSE", section "2. Methodologie"
 * (y = (W Pi) x; at inference Pi is a precomputed index map and the structured
 * sparse GEMM reads its input at the permuted addresses).
 *   idx [in] K int32 device array; entries outside [0, K) read as zero rows.
 * Other arguments as nm_spmm.
 */
NM_API nm_status nm_spmm_permuted(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                           const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                           nm_out_dtype y_dtype, void* stream);

/*
 * nm_hybrid_spmm -- PATCH-style hybrid GEMM: W is split into tile x tile
 * blocks; block (i, j) uses the dense weights when tile_map[i][j] == 0 and the
 * 2:4-pruned weights when it is 1.  Dense blocks are read from W, 2:4 blocks
 * from the 2:4 compressed form of the whole W (nm_prune_compress(W, 2, 4));
 * both accumulate into one output tile.
 * Source: "Structured Sparsity" topic cards, PATCH abstract (weight matrices
 * partitioned into tiles, each tile either dense or 2:4 sparse).
 *   W        [in] R x K bf16, row stride ldw >= K, ldw % 8 == 0 (dense tiles)
 *   values, meta [in] nm_prune_compress(W, 2, 4) (2:4 tiles)
 *   tile_map [in] ceil(R/tile) x ceil(K/tile) uint8, 0 = dense, 1 = 2:4
 *   tile     [in] must be 128
 * Shapes with K % 128 == 0, T >= 192 and T % 8 == 0 run on SM pairs: a K
 * stage of a 256-row tile uses the 2:4 MMA when both 128-row tiles are 2:4,
 * else dense MMAs; the 2:4 tiles of such stages come from a staged copy of W
 * under the mask (R*K*2 bytes from the library's pool, one extra launch).
 * Other arguments as nm_spmm.  Errors: as nm_spmm, NM_ERR_UNSUPPORTED for
 * tile != 128 or K % 16 != 0.
 */
NM_API nm_status nm_hybrid_spmm(const uint16_t* W, int64_t ldw, const uint16_t* values, const uint32_t* meta,
                         const uint8_t* tile_map, int tile, int64_t R, int64_t K, const uint16_t* X,
                         int64_t ldx, int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype, void* stream);

/*
 * nm_prune_spmm -- prune and multiply in one call, for masks that change from
 * call to call (weights re-pruned during training): Y = (W' Pi) X where W' is
 * W under the n:m magnitude mask of nm_prune_compress, and Pi is the index
 * map of nm_spmm_permuted (idx may be NULL for none).  The result equals
 * nm_prune_compress followed by nm_spmm_permuted on its output.
 * Source: "Structured Sparsity" topic cards, RNM-TD3 abstract (N:M structured
 * sparsity kept through the whole of training, so the mask is recomputed as
 * the weights move) and "M:N sparsity on NVIDIA tensor cores" (the mask).
 *   W      [in]  R x K bf16, row stride ldw >= K
 *   values, meta [out, optional] both NULL, or both set: they receive
 *          exactly what nm_prune_compress(W, n, m) writes
 *   other arguments as nm_spmm_permuted.
 * 2:4 with K % 128 == 0, T <= 64, ldw % 8 == 0 and 16-byte aligned W (and
 * values/meta when given) runs one fused kernel: each 128 x 128 tile of W is
 * read once by TMA, selected in shared memory and fed to the sparse MMA, so
 * W is read from HBM once and the compressed form is only written when
 * asked for; split-K partials and the gather of permuted rows are staged as
 * in nm_spmm_permuted (a second launch sums the partials).  Every other case
 * runs nm_prune_compress into `values`/`meta` (or, when those are NULL, into
 * a staging buffer of R*K*9/16 bytes for 2:4 from the library's pool) and
 * then the nm_spmm_permuted path.
 * Errors: as nm_prune_compress and nm_spmm_permuted; NM_ERR_INVALID_ARG when
 * only one of values and meta is given.
 */
NM_API nm_status nm_prune_spmm(const uint16_t* W, int64_t ldw, int n, int m, int64_t R, int64_t K,
                               const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                               nm_out_dtype y_dtype, uint16_t* values, uint32_t* meta, void* stream);

/* ----------------------------------------------------------------- INT8 */
/*
 * INT8 2:4 weights.  Source: "M:N sparsity on NVIDIA tensor cores" -- the
 * sparse tensor cores take 2:4 for FP16, BF16 and INT8 weights; with a 2-bit
 * index per stored value INT8 2:4 keeps 62.5 % of the dense bytes (a 37.5 %
 * saving).  Same selection rule as nm_prune_compress on int8 magnitudes
 * (|-128| = 128 ranks above 127, equal magnitudes to the lower index), values
 * pushed left (R x K/2 int8), and the same tiled 2:4 metadata
 * (nm_meta_words(R, K, 2, 4) words).  All three need K % 16 == 0
 * (NM_ERR_UNSUPPORTED otherwise).
 *
 * nm_prune_compress_i8: W R x K int8 (row stride ldw >= K, ldw % 8 == 0,
 *   8-byte aligned); values 4-byte and meta 8-byte aligned.
 * nm_decompress_i8: W_out R x K int8 (ldw % 16 == 0, 16-byte aligned), 0 at
 *   the pruned positions.
 * nm_spmm_i8: Y = W' X exactly in int32, X K x T int8 (ldx % 16 == 0, 16-byte
 *   aligned), Y R x T int32 (ldy % 4 == 0, 16-byte aligned).  With T >= 192,
 *   K % 32 == 0 and 16-byte aligned values it runs on the sparse tensor cores
 *   (tcgen05 kind::i8 on SM pairs): the tiled metadata is first re-laid out
 *   into the order that MMA reads (one launch, 4 KB per 128 rows and 256
 *   columns staged from the library's pool), then the GEMM (a second
 *   launch).  Other shapes: the operand is decompressed into a staging buffer
 *   (R x K bytes) and multiplied by a dense kind::i8 GEMM.  |W'| <= 128 and
 *   |X| <= 128, so a sum overflows int32 only for K > 131072; the call does
 *   not check.
 * Errors: NM_ERR_INVALID_ARG, NM_ERR_UNSUPPORTED, NM_ERR_MISALIGNED, NM_ERR_CUDA.
 */
NM_API nm_status nm_prune_compress_i8(const int8_t* W, int64_t R, int64_t K, int64_t ldw, int8_t* values,
                                      uint32_t* meta, void* stream);
NM_API nm_status nm_decompress_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, int8_t* W_out,
                                  int64_t ldw, void* stream);
NM_API nm_status nm_spmm_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, const int8_t* X,
                            int64_t ldx, int64_t T, int32_t* Y, int64_t ldy, void* stream);

/* ----------------------------------------------------------------- TF32 */
/*
 * 1:2 sparsity of float32 weights for the TF32 tensor cores.  Source: "M:N
 * sparsity on NVIDIA tensor cores", the passage on the formats the sparse
 * tensor cores take (for TF32 the block halves to 1:2, still 50 percent).
 *
 * nm_prune_compress_tf32: W float32 R x K (row stride ldw >= K, K even),
 *   4-byte aligned.  Of each pair (W[r][2p], W[r][2p+1]) the larger
 *   magnitude survives; equal magnitudes go to the first; a NaN ranks above
 *   every number (NaNs tie).  values: R x K/2 float32, the survivors' bits.
 *   meta: R x ceil(K/64) words (nm_meta_words(R, K, 1, 2)); survivor p of a
 *   row is bit p % 32 of word p / 32: its position in the pair (0 or 1);
 *   unused bits 0.  One launch.
 * nm_decompress_tf32: W_out[r][2p + bit] = values[r][p], +0.0 at the other
 *   position (row stride ldw >= K).
 * nm_spmm_tf32: Y = W' X, X float32 K x T (row stride ldx >= T, ldx % 4 == 0,
 *   16-byte aligned), Y R x T bf16 or fp32 (y_dtype) as nm_spmm.  With
 *   T >= 192, K % 8 == 0 and 16-byte aligned values it runs on the sparse
 *   tensor cores (tcgen05 kind::tf32 on SM pairs) after one pass that re-lays
 *   the positions out into that MMA's metadata order (4 KB per 128 rows and
 *   64 columns staged from the library's pool).  Other shapes: the operand
 *   is decompressed into a staged dense copy (R x ceil4(K) float32) and
 *   multiplied by a dense kind::tf32 GEMM.  Either way the tensor cores read
 *   W' and X as TF32 (10 explicit mantissa bits) and accumulate in fp32, so Y
 *   meets the GEMM tolerance (|y - y_ref| <= 2^-7 sum |w||x|), not bit
 *   equality with an fp32 product.
 * Errors: NM_ERR_INVALID_ARG (odd K, negative sizes, ld too small, null),
 *   NM_ERR_MISALIGNED, NM_ERR_UNSUPPORTED (a dimension >= 2^31), NM_ERR_CUDA.
 */
NM_API nm_status nm_prune_compress_tf32(const float* W, int64_t R, int64_t K, int64_t ldw, float* values,
                                        uint32_t* meta, void* stream);
NM_API nm_status nm_decompress_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, float* W_out,
                                    int64_t ldw, void* stream);
NM_API nm_status nm_spmm_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, const float* X,
                              int64_t ldx, int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype, void* stream);

/* ------------------------------------------------------------- diagonal */
/*
 * Diagonal sparsity under the index map.  Source: the SHUFFLESPARSE technical
 * summary, section "3. Belangrijkste Bijdragen" (one permutation primitive
 * over block, N:M and diagonal patterns), and the DynaDiag abstract on the
 * SHUFFLESPARSE author page (a diagonal pattern kept through training, 90 %
 * sparse ViT linears).  The pages give no format; this library reads it as:
 * diagonal o (0 <= o < K) of an R x K matrix is {(r, (r + o) mod K)}, one
 * entry per row; a diagonal operand is D distinct offsets (int32, ascending)
 * and values V (D x R bf16), V[d][r] = W[r][(r + o_d) mod K].
 *
 * nm_diag_prune_compress: keep the D diagonals of largest score
 *   s(o) = sum_r |W[r][(r + o) mod K]| (NaN ranks above every number; ties
 *   to the lower offset); writes offsets[D] and values (D x R).  The device
 *   adds the scores in float32 (32-row chunk sums with r ascending, then the
 *   chunk sums in ascending order), so where two diagonals' exact scores
 *   differ by less than the rounding of R float32 additions, either one may
 *   be kept: the set is one that a float32 evaluation of s ranks first, and
 *   no dropped diagonal's exact score exceeds a kept one's by more than
 *   that rounding.  Stages ceil(R/32)*K*4 + K*8 bytes from the library's
 *   pool; a memset and five launches (partial sums, scores, ranks,
 *   placement, gather).
 * nm_diag_expand: the dense R x K copy (+0 off the kept diagonals), row
 *   stride ldw >= K (columns K..ldw-1 are not written); offsets outside
 *   [0, K) place nothing; offsets must be distinct (of a repeated offset,
 *   one of its diagonals is placed).  Every element is written once, by lookup in a
 *   K-entry table staged from the library's pool (K*4 bytes).
 * nm_diag_spmm: y[r][t] = sum_d V[d][r] * X[idx[(r + o_d) mod K]][t]
 *   (X[k] when idx is NULL; idx entries outside [0, K) read zero rows).
 *   Offsets must be distinct.  The operand is expanded into a staged dense
 *   copy (R x ceil8(K) bf16) and multiplied by a dense tcgen05 GEMM on SM
 *   pairs.  With idx the device checks whether idx is a permutation of
 *   [0, K): if so, the copy's columns are placed through idx (column idx[k]
 *   holds the entries of column k) and the GEMM reads X itself; otherwise a
 *   gather pass stages X[idx] and the GEMM reads that.  Staging: the copy,
 *   (3K+1)*4 bytes of tables, and K x ceil8(T) bf16 for the gather (reserved
 *   in both cases).  X, Y as nm_spmm.
 * Errors: NM_ERR_INVALID_ARG (D > K, ld too small, null), NM_ERR_MISALIGNED,
 *   NM_ERR_UNSUPPORTED, NM_ERR_CUDA.
 */
NM_API nm_status nm_diag_prune_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D,
                                        int32_t* offsets, uint16_t* values, void* stream);
NM_API nm_status nm_diag_expand(const uint16_t* values, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                                uint16_t* W_out, int64_t ldw, void* stream);
NM_API nm_status nm_diag_spmm(const uint16_t* values, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                              const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                              nm_out_dtype dtype, void* stream);

/* ------------------------------------------------------------- backward */
/*
 * nm_spmm_t -- input gradient of y = (W' Pi) x: dX = (W' Pi)^T dY, i.e.
 * dXp = W'^T dY (K x T) and dX[idx[k]] = dXp[k] (dX = dXp when idx is NULL).
 * Source: "Structured Sparsity" topic cards, RNM-TD3 abstract (N:M sparsity
 * kept through training), and the DynaDiag page's abstract (sparse forward
 * and backward passes); the gather of nm_spmm_permuted, whose adjoint this is.
 * W'^T is N:M along its output axis, not along the reduction axis R, so the
 * sparse MMA cannot take it: W' is decompressed into a staging buffer
 * (R x ceil8(K) bf16 from the library's pool, one launch) and a dense
 * tcgen05 GEMM on SM pairs reads it transposed (a second launch).
 *   values, meta [in] compressed R x K weights, pattern n:m
 *   idx  [in] NULL, or a permutation of [0, K) (the forward's index map):
 *        row k of W'^T dY is written to row idx[k] of dX; entries outside
 *        [0, K) drop their row; repeated entries are not supported (their
 *        rows race), and rows of dX that no entry names are not written
 *   dY   [in]  R x T bf16, row stride lddy >= T, lddy % 8 == 0
 *   dX   [out] K x T, bf16 or fp32 (dtype), row stride lddx >= T, 16-byte rows
 * Errors: as nm_spmm.
 */
NM_API nm_status nm_spmm_t(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                           const int32_t* idx, const uint16_t* dY, int64_t lddy, int64_t T, void* dX, int64_t lddx,
                           nm_out_dtype dtype, void* stream);

/*
 * nm_sddmm -- gradient of the stored values of y = (W' Pi) x:
 * dV[r][j] = sum_t dY[r][t] * X[idx[k_j]][t], with k_j the column of
 * survivor j of row r (group j / n, position from meta; X[idx[k]] = X[k]
 * when idx is NULL, a zero row for an entry outside [0, K)).  These are the
 * entries of dY Xp^T at the survivors, in the layout of `values`.
 * Source: same passages as nm_spmm_t.
 * The full product dY Xp^T runs as a dense tcgen05 GEMM on SM pairs and the
 * epilogue stores only the survivor entries.  With idx, one gather pass first
 * stages Xp (K x ceil8(T) bf16 from the library's pool).
 *   meta [in]  metadata of the compressed R x K weights, pattern n:m
 *   dY   [in]  R x T bf16, row stride lddy >= T, lddy % 8 == 0
 *   X    [in]  K x T bf16, row stride ldx >= T, ldx % 8 == 0
 *   dV   [out] R x nm_value_cols(K,n,m), bf16 or fp32 (dtype), contiguous rows
 * Errors: as nm_spmm.
 */
NM_API nm_status nm_sddmm(const uint32_t* meta, int n, int m, int64_t R, int64_t K, const int32_t* idx,
                          const uint16_t* dY, int64_t lddy, const uint16_t* X, int64_t ldx, int64_t T, void* dV,
                          nm_out_dtype dtype, void* stream);

/*
 * nm_spmm_algo --nm_spmm / nm_spmm_permuted (idx may be NULL) with the kernel
 * design chosen explicitly, to compare the sparse tensor-core path with the
 * dense expansion on the same pattern.  NM_ERR_UNSUPPORTED when the pattern
 * does not fit the requested design (NM_ALGO_SPARSE_TC with 3:4, say).
 */
NM_API nm_status nm_spmm_algo(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                       const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                       nm_out_dtype y_dtype, nm_algo algo, void* stream);

/*
 * nm_release_staging -- return the memory that nm_spmm_permuted's staging pools
 * keep reserved (all devices) to the driver.  Memory still in use by calls
 * in flight stays reserved.  The pages have no counterpart to this
 * call; it exists because the pool deliberately keeps its memory between calls.
 * Errors: NM_ERR_CUDA.
 */
NM_API nm_status nm_release_staging(void);

/*
 * nm_selftest_wait_timeout -- exercise the failure-reporting path.  The pages
 * have no counterpart to this call; it exists so that the bounded waits of the
 * kernels can be tested without a fault.  It launches one block on `stream`
 * in which a thread waits, with the same bounded wait the GEMM kernels use, on
 * a barrier that nothing completes; after limit_us microseconds (1..1000000)
 * the wait gives up and records a timeout in the device status word, and the
 * kernel returns.  The next nm_device_status(stream) returns NM_ERR_TIMEOUT
 * (and clears the word); the context stays usable.
 * Errors: NM_ERR_INVALID_ARG (limit out of range), NM_ERR_NO_DEVICE, NM_ERR_CUDA.
 */
NM_API nm_status nm_selftest_wait_timeout(uint32_t limit_us, void* stream);

/*
 * nm_spmm_permuted_noalloc -- nm_spmm_permuted without any device allocation.
 * The pages have no counterpart to this call; it exists for callers that
 * cannot let a library allocate device memory: runtimes that budget every
 * byte up front, processes whose memory pool belongs to another allocator, or
 * loops that cannot afford a pool that has to grow.  nm_spmm_permuted stages
 * the gathered input X[idx[k]] in a buffer taken from a library-owned memory
 * pool on `stream`; this call stages it instead in a fixed 32 MiB array inside the
 * library, which every device that loads the library holds until the process
 * exits, and works through the columns of X in chunks that fit it (chunks of
 * floor(16 Mi / K / 256) * 256 columns, one gather and one GEMM launch each).
 * For 2:4, columns that a two-SM chunk serves are bit-identical to
 * nm_spmm_permuted's; a last chunk of fewer than 192 columns runs on the one-SM
 * kernel, and other patterns always do, so those agree with nm_spmm_permuted
 * within the GEMM tolerance (different summation order).  Arguments and
 * errors as nm_spmm_permuted (the same checks), plus:
 *  - NM_ERR_UNSUPPORTED when K > 65536 on the two-SM path (a 256-column chunk
 *    of K rows must fit the array);
 *  - the first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) and keeps it for the life of the process; make
 *    that first call before any stream capture, and do not use the call
 *    after cudaDeviceReset on that device (the kept address would be stale);
 *  - all calls share the one array and each leaves its last chunk in it: calls
 *    that may overlap on the GPU (different streams, or other host threads)
 *    race and must be serialised by the caller.  Nothing in the array needs to
 *    start at zero: each chunk writes every element it later reads.
 * Every other case (patterns other than 2:4, K % 128 != 0, T < 192,
 * T % 8 != 0) runs on the one-SM kernel, which reads the mapped rows of X
 * itself and stages nothing (patterns other than 2:4 are not re-encoded
 * here, unlike nm_spmm_permuted).
 */
NM_API nm_status nm_spmm_permuted_noalloc(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R,
                                          int64_t K, const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T,
                                          void* Y, int64_t ldy, nm_out_dtype y_dtype, void* stream);

/* ------------------------------------------------------------ utilities */
/* Synchronises `stream`, then returns NM_ERR_TIMEOUT if any kernel of this
 * library recorded a bounded wait that gave up since the previous call (and
 * clears the record), NM_ERR_CUDA on a pending CUDA error, else NM_OK. */
NM_API nm_status nm_device_status(void* stream);

/* Static description of a status code. */
NM_API const char* nm_status_string(nm_status s);

/* Text of the most recent error of the calling host thread ("" if none). */
NM_API const char* nm_last_error(void);

/* Number of kernels this library has launched in this process. */
NM_API uint64_t nm_launch_count(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
NM_API int nm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NM_B200_H */
