/*
 * nm_oracle.c -- plain, slow, obviously-correct CPU definition of N:M
 * structured weight sparsity: magnitude prune, push-left compression,
 * decompression, and the sparse x dense GEMM (plain, column-permuted and
 * PATCH-style hybrid).  Every sum is accumulated in double precision.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header or table
 * with the CUDA library.
 *
 * Sources (page title, then the passage):
 *  [MN-def]   "M:N sparsity on NVIDIA tensor cores", opening passage: a 2:4
 *             row is read four cells at a time; every group of four
 *             consecutive weights along a row keeps exactly two survivors,
 *             anywhere inside the group; the metadata of the worked row
 *             [v,0,0,v | 0,v,v,0] is [[0,3],[1,2]]; the general a:b form.
 *  [MN-fine]  same page, "Fine-grained in what it removes, structured in how
 *             many": two bits per survivor say which slot it came from; the
 *             groups run along the row of W, which is the reduction axis K.
 *  [MN-fmt]   same page, "Where this sits among the three case studies",
 *             storage paragraphs: an R x C matrix is stored as an R x C/2
 *             block of values with all survivors pushed left, plus an
 *             R x C/2 block of 2-bit indices; 36 bits per group of four
 *             FP16 weights.
 *  [MN-gemm]  same page and section, GEMM paragraphs: only the first operand
 *             is compressed; the indices pick the elements of the dense
 *             second operand that the kept weights multiply (the K = 8
 *             example); the result is a dense matrix.
 *  [MN-prune] same page, "The recipe: one prune, one retrain, no search",
 *             step 2: in every group of four along the row, zero the two
 *             with the smallest absolute value.
 *  [SS-perm]  "Technische Samenvatting: SHUFFLESPARSE ...", section
 *             "2. Methodologie": y = (W Pi) x; at inference the hard Pi is
 *             a precomputed index map and the structured sparse GEMM reads
 *             its input at the permuted addresses (same FLOP count).
 *  [PATCH]    "Structured Sparsity" topic cards, the PATCH abstract: weight
 *             matrices are split into tiles, each tile either dense or 2:4.
 *  [MN-int8]  "M:N sparsity on NVIDIA tensor cores", passage on the formats
 *             the sparse tensor cores accept (2:4 for FP16, BF16 and INT8
 *             weights) and the storage paragraphs (a 2-bit index per stored
 *             value: 25 % of an INT8 value, so INT8 2:4 saves 37.5 %).
 *  [MN-tf32]  "M:N sparsity on NVIDIA tensor cores", the same passage on the
 *             formats: for TF32 the block halves to 1:2, still 50 percent.
 *  [DIAG]     SHUFFLESPARSE (the technical summary's contributions and the
 *             author page's abstract): one permutation primitive over block,
 *             N:M and diagonal patterns; the DynaDiag abstract on the same
 *             author page: a diagonal sparsity pattern kept through training,
 *             90 % sparse ViT linears.  The pages give no format; the
 *             readings are below.
 *  [TRAIN]    "Structured Sparsity" topic cards, RNM-TD3 abstract (N:M
 *             sparsity kept through the whole of training) and the
 *             DynaDiag page's abstract (sparse computation in the forward
 *             and the backward pass): the gradients of y = (W' Pi) x.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - ties in magnitude go to the lower index inside the group;
 *  - exactly N survivors are always stored, zeros included, so the format
 *    stays fixed-rate;
 *  - survivors of a group are stored in ascending position order, as in the
 *    worked row;
 *  - magnitudes are compared on the bf16 value; +0 and -0 tie; a NaN ranks
 *    above every number (Inf included) and NaNs tie among themselves;
 *  - positions use b = ceil(log2 M) bits.  For every pattern except 2:4,
 *    survivor j of a row goes to 32-bit word floor(j/S) at bit b*(j mod S),
 *    S = floor(32/b), rows one after the other, unused bits zero
 *    ("row-wise" packing).  For 2:4 a group's two positions form one nibble
 *    p0 | p1 << 2 (first survivor low), and the nibbles are tiled in the order
 *    a B200 sparse tensor-core instruction reads them ("tiled" packing, see
 *    meta_slot_2of4 below); groups past R or K in the padded tiles hold the
 *    nibble of an all-zero group, positions (0,1);
 *  - the permutation is applied as X_perm[k][t] = X[idx[k]][t]; an entry of
 *    idx outside [0, K) reads a zero row;
 *  - diagonal pattern: diagonal o (0 <= o < K) of an R x K matrix is the set
 *    {(r, (r + o) mod K)}, one entry per row (wrapping); a diagonally sparse
 *    weight keeps D distinct offsets (ascending) and stores V[d][r] =
 *    W[r][(r + o_d) mod K] (D x R); one-shot selection keeps the D diagonals
 *    of largest score s(o) = sum_r |W[r][(r + o) mod K]| (the plain sum in
 *    double, r ascending; a NaN on the diagonal ranks it above every number),
 *    ties to the lower offset.  A device that sums in float32 may keep a
 *    different but equally valid set when two scores differ by less than its
 *    rounding error; the tests accept any set that no dropped diagonal beats
 *    by more than that error;
 *  - backward: dX is the adjoint of that gather (row k of W'^T dY is added to
 *    row idx[k] of dX; entries outside [0, K) drop their row, repeated
 *    entries add up), and the gradient of the stored values is
 *    dV[r][j] = sum_t dY[r][t] * X_perm[k_j][t] for the survivor's column k_j;
 *  - TF32: 1:2 selection compares the float32 values (the same rules); the
 *    values and W hold float32 bit patterns (uint32); the oracle's GEMM is
 *    exact in double and the TF32 device path is held to the GEMM tolerance;
 *  - W (dense, R x K) and the compressed values hold bf16 bit patterns
 *    (uint16); X is K x T row-major; Y is R x T (double here).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bf16 <-> double.  bf16 is the upper half of an IEEE binary32, so the */
/* conversion to double is exact.                                       */
/* ------------------------------------------------------------------ */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Bits per stored position for a group of M: ceil(log2 M). */
int oracle_index_bits(int m)
{
    int b = 0;
    while ((1 << b) < m) b++;
    return b;
}

/* Positions packed into one 32-bit word (row-wise packing). */
int oracle_positions_per_word(int m)
{
    return 32 / oracle_index_bits(m);
}

/* Columns of the value block: K * N / M. */
int64_t oracle_value_cols(int64_t K, int n, int m)
{
    return K / m * n;
}

/* 32-bit metadata words per row (row-wise packing): ceil(value_cols / S). */
int64_t oracle_meta_cols(int64_t K, int n, int m)
{
    int64_t s = oracle_positions_per_word(m);
    return (oracle_value_cols(K, n, m) + s - 1) / s;
}

/* Total 32-bit metadata words of an R x K matrix.  Tiled 2:4: one block of
 * 64 words per 16 rows x 128 columns, rows and columns padded up. */
int64_t oracle_meta_words(int64_t R, int64_t K, int n, int m)
{
    if (n == 2 && m == 4) return (R + 15) / 16 * ((K + 127) / 128) * 64;
    return R * oracle_meta_cols(K, n, m);
}

/* Tiled 2:4 packing: word and bit offset of the nibble of group g (columns
 * 4g..4g+3) of row r.  Rows are taken 16 at a time and columns 128 at a
 * time; block (rb, cb) holds 64 words at word (rb * ceil(K/128) + cb) * 64.
 * Inside a block, word 4*l + q (lane l = 0..15, quarter q = 0..3) covers
 * columns 32q + 16h .. 32q + 16h + 15 of the block, h = l / 8, for row
 * (l mod 8) of the 16 in bits 0..15 and row 8 + (l mod 8) in bits 16..31,
 * four nibbles each in column order. */
static int64_t meta_slot_2of4(int64_t r, int64_t g, int64_t K, int *bit)
{
    int64_t cblocks = (K + 127) / 128;
    int64_t rb = r / 16, cb = g / 32;
    int q = (int)((g % 32) / 8), h = (int)((g % 8) / 4), t = (int)(g % 4);
    int l = (int)(r % 8) + 8 * h;
    *bit = 16 * (int)((r / 8) % 2) + 4 * t;
    return (rb * cblocks + cb) * 64 + 4 * l + q;
}

static int pattern_ok(int n, int m)
{
    return (m == 2 || m == 4 || m == 8 || m == 16) && n >= 1 && n < m;
}

/* ------------------------------------------------------------------ */
/* Selection [MN-def], [MN-prune].                                      */
/* ------------------------------------------------------------------ */

/* Does element a of a group beat element b (a != b)?  Larger magnitude
 * wins; a NaN beats every number; equal magnitudes (and NaN vs NaN) go to
 * the lower index. */
static int beats(double wa, int a, double wb, int b)
{
    int na = isnan(wa), nb = isnan(wb);
    if (na || nb) {
        if (na && !nb) return 1;
        if (nb && !na) return 0;
        return a < b;
    }
    double ma = fabs(wa), mb = fabs(wb);
    if (ma != mb) return ma > mb;
    return a < b;
}

/* mask[r*K + k] = 1 if W[r][k] survives N:M pruning, else 0.  An element
 * survives when fewer than N elements of its group beat it. */
int oracle_prune_mask(const uint16_t *W, int64_t R, int64_t K, int64_t ldw,
                      int n, int m, uint8_t *mask)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t g = 0; g < K / m; g++) {
            const uint16_t *grp = W + r * ldw + g * m;
            for (int i = 0; i < m; i++) {
                int rank = 0;
                for (int j = 0; j < m; j++)
                    if (j != i && beats(bf16_value(grp[j]), j, bf16_value(grp[i]), i))
                        rank++;
                mask[r * K + g * m + i] = (uint8_t)(rank < n);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Push-left compression [MN-fmt].                                      */
/* values: R x (K*N/M) bf16 bits, survivors in ascending position.      */
/* meta:   oracle_meta_words words (tiled 2:4, else row-wise b-bit).    */
/* ------------------------------------------------------------------ */
int oracle_compress(const uint16_t *W, int64_t R, int64_t K, int64_t ldw,
                    int n, int m, uint16_t *values, uint32_t *meta)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    int64_t mcols = oracle_meta_cols(K, n, m);
    int b = oracle_index_bits(m);
    int s = oracle_positions_per_word(m);
    uint8_t *mask = (uint8_t *)malloc((size_t)(R * K > 0 ? R * K : 1));
    if (!mask) return 2;
    oracle_prune_mask(W, R, K, ldw, n, m, mask);
    int tiled = (n == 2 && m == 4);
    int64_t words = oracle_meta_words(R, K, n, m);
    for (int64_t i = 0; i < words; i++) meta[i] = tiled ? 0x44444444u : 0u;
    for (int64_t r = 0; r < R; r++) {
        int64_t j = 0; /* survivor index inside the row */
        for (int64_t g = 0; g < K / m; g++) {
            uint32_t nib = 0;
            int seen = 0;
            for (int p = 0; p < m; p++) {
                if (!mask[r * K + g * m + p]) continue;
                values[r * vcols + j] = W[r * ldw + g * m + p];
                if (tiled)
                    nib |= (uint32_t)p << (2 * seen);
                else
                    meta[r * mcols + j / s] |= (uint32_t)p << (b * (j % s));
                seen++;
                j++;
            }
            if (tiled) {
                int bit;
                int64_t w = meta_slot_2of4(r, g, K, &bit);
                meta[w] = (meta[w] & ~(0xFu << bit)) | (nib << bit);
            }
        }
    }
    free(mask);
    return 0;
}

/* In-group position of survivor j of row r (an R x K matrix). */
static int position_of(const uint32_t *meta, int64_t K, int64_t r, int64_t j, int n, int m)
{
    if (n == 2 && m == 4) {
        int bit;
        int64_t w = meta_slot_2of4(r, j / 2, K, &bit);
        return (int)((meta[w] >> (bit + 2 * (int)(j % 2))) & 3u);
    }
    int b = oracle_index_bits(m);
    int s = oracle_positions_per_word(m);
    int64_t mcols = oracle_meta_cols(K, n, m);
    uint32_t word = meta[r * mcols + j / s];
    return (int)((word >> (b * (j % s))) & ((1u << b) - 1u));
}

/* positions[r * vcols + j] = in-group position of survivor j of row r. */
int oracle_positions(const uint32_t *meta, int64_t R, int64_t K, int n, int m, uint8_t *positions)
{
    if (!pattern_ok(n, m) || K % m != 0) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++)
        for (int64_t j = 0; j < vcols; j++)
            positions[r * vcols + j] = (uint8_t)position_of(meta, K, r, j, n, m);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Decompression: put every survivor back at its position, +0 (bits     */
/* 0x0000) everywhere else.                                             */
/* ------------------------------------------------------------------ */
int oracle_decompress(const uint16_t *values, const uint32_t *meta, int64_t R, int64_t K,
                      int n, int m, uint16_t *W_out, int64_t ldw)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t k = 0; k < K; k++) W_out[r * ldw + k] = 0;
        for (int64_t j = 0; j < vcols; j++) {
            int64_t g = j / n;
            int p = position_of(meta, K, r, j, n, m);
            W_out[r * ldw + g * m + p] = values[r * vcols + j];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Sparse x dense GEMM on the compressed operand [MN-gemm], [SS-perm]:  */
/*   y[r][t] = sum_j V[r][j] * X[pi(g*M + pos_j)][t],  g = j / N,       */
/* pi(k) = idx[k] when idx is given, else k.  Products and the sum are  */
/* in double, in survivor order.                                         */
/* ------------------------------------------------------------------ */
int oracle_spmm(const uint16_t *values, const uint32_t *meta, int n, int m,
                int64_t R, int64_t K, const uint16_t *X, int64_t ldx, int64_t T,
                const int32_t *idx, double *Y, int64_t ldy)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldx < T || ldy < T) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0;
            for (int64_t j = 0; j < vcols; j++) {
                int64_t k = (j / n) * m + position_of(meta, K, r, j, n, m);
                int64_t src = idx ? (int64_t)idx[k] : k;
                if (src < 0 || src >= K) continue; /* a zero row */
                acc += bf16_value(values[r * vcols + j]) * bf16_value(X[src * ldx + t]);
            }
            Y[r * ldy + t] = acc;
        }
    }
    return 0;
}

/* The same sum for a list of (row, column) output coordinates only: the
 * per-element form used to check full-size results by sampling. */
int oracle_spmm_sampled(const uint16_t *values, const uint32_t *meta, int n, int m,
                        int64_t R, int64_t K, const uint16_t *X, int64_t ldx, int64_t T,
                        const int32_t *idx, const int64_t *rows, const int64_t *cols,
                        int64_t count, double *out, double *out_abs)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldx < T) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t i = 0; i < count; i++) {
        int64_t r = rows[i], t = cols[i];
        if (r < 0 || r >= R || t < 0 || t >= T) return 3;
        double acc = 0.0, mag = 0.0;
        for (int64_t j = 0; j < vcols; j++) {
            int64_t k = (j / n) * m + position_of(meta, K, r, j, n, m);
            int64_t src = idx ? (int64_t)idx[k] : k;
            double w = bf16_value(values[r * vcols + j]);
            double x = (src < 0 || src >= K) ? 0.0 : bf16_value(X[src * ldx + t]);
            acc += w * x;
            mag += fabs(w) * fabs(x);
        }
        out[i] = acc;
        if (out_abs) out_abs[i] = mag;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Plain dense GEMM of a bf16 matrix, the closed form a sparse GEMM     */
/* must equal once the pruned weights are written out densely:          */
/*   y[r][t] = sum_k W[r][k] * X[pi(k)][t].                              */
/* y_abs (optional) receives sum_k |W[r][k]| * |X[pi(k)][t]|, the scale */
/* of the floating-point tolerance.                                     */
/* ------------------------------------------------------------------ */
int oracle_dense_gemm(const uint16_t *W, int64_t R, int64_t K, int64_t ldw,
                      const uint16_t *X, int64_t ldx, int64_t T, const int32_t *idx,
                      double *Y, double *Y_abs, int64_t ldy)
{
    if (ldw < K || ldx < T || ldy < T) return 1;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; k++) {
                int64_t src = idx ? (int64_t)idx[k] : k;
                double w = bf16_value(W[r * ldw + k]);
                double x = (src < 0 || src >= K) ? 0.0 : bf16_value(X[src * ldx + t]);
                acc += w * x;
                mag += fabs(w) * fabs(x);
            }
            Y[r * ldy + t] = acc;
            if (Y_abs) Y_abs[r * ldy + t] = mag;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* PATCH-style hybrid [PATCH]: tile (i, j) of size tile x tile uses the */
/* dense weights when tile_map[i][j] == 0, and the 2:4-pruned weights   */
/* (survivors kept, +0 elsewhere) when it is 1.  W_eff is written out   */
/* and multiplied densely.  tile_map is ceil(R/tile) x ceil(K/tile).    */
/* ------------------------------------------------------------------ */
int oracle_hybrid_weights(const uint16_t *W, int64_t R, int64_t K, int64_t ldw,
                          const uint8_t *tile_map, int64_t tile, uint16_t *W_eff)
{
    if (K % 4 != 0 || tile <= 0 || tile % 4 != 0 || ldw < K) return 1;
    uint8_t *mask = (uint8_t *)malloc((size_t)(R * K > 0 ? R * K : 1));
    if (!mask) return 2;
    oracle_prune_mask(W, R, K, ldw, 2, 4, mask);
    int64_t tiles_k = (K + tile - 1) / tile;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t k = 0; k < K; k++) {
            int sparse = tile_map[(r / tile) * tiles_k + k / tile] != 0;
            uint16_t w = W[r * ldw + k];
            W_eff[r * K + k] = (sparse && !mask[r * K + k]) ? (uint16_t)0 : w;
        }
    }
    free(mask);
    return 0;
}

int oracle_hybrid_spmm(const uint16_t *W, int64_t R, int64_t K, int64_t ldw,
                       const uint8_t *tile_map, int64_t tile,
                       const uint16_t *X, int64_t ldx, int64_t T, double *Y, double *Y_abs,
                       int64_t ldy)
{
    uint16_t *W_eff = (uint16_t *)malloc((size_t)(R * K > 0 ? R * K : 1) * sizeof(uint16_t));
    if (!W_eff) return 2;
    int rc = oracle_hybrid_weights(W, R, K, ldw, tile_map, tile, W_eff);
    if (rc == 0) rc = oracle_dense_gemm(W_eff, R, K, K, X, ldx, T, NULL, Y, Y_abs, ldy);
    free(W_eff);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Backward products of y = (W' Pi) x [TRAIN], [SS-perm], [MN-gemm].    */
/* dY is R x T (the gradient of y).                                     */
/*                                                                      */
/* Input gradient: with Xp[k] = X[pi(k)], y = W' Xp gives               */
/*   dXp[k][t] = sum_r W'[r][k] * dY[r][t],  and dX[pi(k)] += dXp[k].    */
/* Only survivors are non-zero in W', so the sum runs over the stored   */
/* values: survivor j of row r sits in column k = (j/N)*M + pos_j.      */
/* dX (K x T) is overwritten; dX_abs (optional) gets the sums of        */
/* |products|.  Entries of idx outside [0, K) drop their row.           */
/* ------------------------------------------------------------------ */
int oracle_spmm_t(const uint16_t *values, const uint32_t *meta, int n, int m,
                  int64_t R, int64_t K, const uint16_t *dY, int64_t lddy, int64_t T,
                  const int32_t *idx, double *dX, double *dX_abs, int64_t lddx)
{
    if (!pattern_ok(n, m) || K % m != 0 || lddy < T || lddx < T) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t k = 0; k < K; k++)
        for (int64_t t = 0; t < T; t++) {
            dX[k * lddx + t] = 0.0;
            if (dX_abs) dX_abs[k * lddx + t] = 0.0;
        }
    for (int64_t r = 0; r < R; r++) {
        for (int64_t j = 0; j < vcols; j++) {
            int64_t k = (j / n) * m + position_of(meta, K, r, j, n, m);
            int64_t dst = idx ? (int64_t)idx[k] : k;
            if (dst < 0 || dst >= K) continue;
            double w = bf16_value(values[r * vcols + j]);
            for (int64_t t = 0; t < T; t++) {
                double g = bf16_value(dY[r * lddy + t]);
                dX[dst * lddx + t] += w * g;
                if (dX_abs) dX_abs[dst * lddx + t] += fabs(w) * fabs(g);
            }
        }
    }
    return 0;
}

/* Gradient of the stored values: dV[r][j] = sum_t dY[r][t] * Xp[k_j][t], */
/* the entries of dY Xp^T at the survivors' columns only (a sampled      */
/* dense-dense product).  dV is R x K*N/M; dV_abs (optional) gets the     */
/* sums of |products|.                                                    */
int oracle_sddmm(const uint32_t *meta, int n, int m, int64_t R, int64_t K,
                 const uint16_t *dY, int64_t lddy, const uint16_t *X, int64_t ldx, int64_t T,
                 const int32_t *idx, double *dV, double *dV_abs)
{
    if (!pattern_ok(n, m) || K % m != 0 || lddy < T || ldx < T) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t j = 0; j < vcols; j++) {
            int64_t k = (j / n) * m + position_of(meta, K, r, j, n, m);
            int64_t src = idx ? (int64_t)idx[k] : k;
            double acc = 0.0, mag = 0.0;
            if (src >= 0 && src < K) {
                for (int64_t t = 0; t < T; t++) {
                    double g = bf16_value(dY[r * lddy + t]);
                    double x = bf16_value(X[src * ldx + t]);
                    acc += g * x;
                    mag += fabs(g) * fabs(x);
                }
            }
            dV[r * vcols + j] = acc;
            if (dV_abs) dV_abs[r * vcols + j] = mag;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* INT8 weights [MN-int8].  The same rule on int8 values: the larger    */
/* |w| wins (|-128| = 128 ranks above 127), equal magnitudes go to the  */
/* lower index; values are pushed left and the positions use the same   */
/* metadata packing as bf16 (tiled for 2:4).  The GEMM is exact integer */
/* arithmetic: y[r][t] = sum_j V[r][j] * X[k_j][t] in 64 bits.           */
/* ------------------------------------------------------------------ */
int oracle_prune_mask_i8(const int8_t *W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint8_t *mask)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t g = 0; g < K / m; g++) {
            const int8_t *grp = W + r * ldw + g * m;
            for (int i = 0; i < m; i++) {
                int rank = 0, mi = abs((int)grp[i]);
                for (int j = 0; j < m; j++) {
                    int mj = abs((int)grp[j]);
                    if (j != i && (mj > mi || (mj == mi && j < i))) rank++;
                }
                mask[r * K + g * m + i] = (uint8_t)(rank < n);
            }
        }
    }
    return 0;
}

int oracle_compress_i8(const int8_t *W, int64_t R, int64_t K, int64_t ldw, int n, int m, int8_t *values,
                       uint32_t *meta)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    int64_t mcols = oracle_meta_cols(K, n, m);
    int b = oracle_index_bits(m);
    int s = oracle_positions_per_word(m);
    uint8_t *mask = (uint8_t *)malloc((size_t)(R * K > 0 ? R * K : 1));
    if (!mask) return 2;
    oracle_prune_mask_i8(W, R, K, ldw, n, m, mask);
    int tiled = (n == 2 && m == 4);
    int64_t words = oracle_meta_words(R, K, n, m);
    for (int64_t i = 0; i < words; i++) meta[i] = tiled ? 0x44444444u : 0u;
    for (int64_t r = 0; r < R; r++) {
        int64_t j = 0;
        for (int64_t g = 0; g < K / m; g++) {
            uint32_t nib = 0;
            int seen = 0;
            for (int p = 0; p < m; p++) {
                if (!mask[r * K + g * m + p]) continue;
                values[r * vcols + j] = W[r * ldw + g * m + p];
                if (tiled)
                    nib |= (uint32_t)p << (2 * seen);
                else
                    meta[r * mcols + j / s] |= (uint32_t)p << (b * (j % s));
                seen++;
                j++;
            }
            if (tiled) {
                int bit;
                int64_t w = meta_slot_2of4(r, g, K, &bit);
                meta[w] = (meta[w] & ~(0xFu << bit)) | (nib << bit);
            }
        }
    }
    free(mask);
    return 0;
}

int oracle_decompress_i8(const int8_t *values, const uint32_t *meta, int64_t R, int64_t K, int n, int m,
                         int8_t *W_out, int64_t ldw)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t k = 0; k < K; k++) W_out[r * ldw + k] = 0;
        for (int64_t j = 0; j < vcols; j++)
            W_out[r * ldw + (j / n) * m + position_of(meta, K, r, j, n, m)] = values[r * vcols + j];
    }
    return 0;
}

int oracle_spmm_i8(const int8_t *values, const uint32_t *meta, int n, int m, int64_t R, int64_t K,
                   const int8_t *X, int64_t ldx, int64_t T, int64_t *Y, int64_t ldy)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldx < T || ldy < T) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t t = 0; t < T; t++) {
            int64_t acc = 0;
            for (int64_t j = 0; j < vcols; j++) {
                int64_t k = (j / n) * m + position_of(meta, K, r, j, n, m);
                acc += (int64_t)values[r * vcols + j] * (int64_t)X[k * ldx + t];
            }
            Y[r * ldy + t] = acc;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* FP32 weights for the TF32 tensor cores [MN-tf32]: the block halves   */
/* to 1:2 for TF32.  The same selection rule on the float32 value       */
/* (converted to double exactly; NaN above every number, equal          */
/* magnitudes to the lower index), the same push-left values (float32   */
/* bits, copied) and the same metadata packing as bf16.  The GEMM is    */
/* the exact sum of the exact products of the stored float32 values, in */
/* double; a device that rounds its inputs to TF32 is held to the GEMM  */
/* tolerance, not to bit equality.                                      */
/* ------------------------------------------------------------------ */
static double f32_value(uint32_t bits)
{
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_prune_mask_f32(const uint32_t *W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint8_t *mask)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t g = 0; g < K / m; g++) {
            const uint32_t *grp = W + r * ldw + g * m;
            for (int i = 0; i < m; i++) {
                int rank = 0;
                for (int j = 0; j < m; j++)
                    if (j != i && beats(f32_value(grp[j]), j, f32_value(grp[i]), i)) rank++;
                mask[r * K + g * m + i] = (uint8_t)(rank < n);
            }
        }
    }
    return 0;
}

int oracle_compress_f32(const uint32_t *W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint32_t *values,
                        uint32_t *meta)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    int64_t mcols = oracle_meta_cols(K, n, m);
    int b = oracle_index_bits(m);
    int s = oracle_positions_per_word(m);
    uint8_t *mask = (uint8_t *)malloc((size_t)(R * K > 0 ? R * K : 1));
    if (!mask) return 2;
    oracle_prune_mask_f32(W, R, K, ldw, n, m, mask);
    int tiled = (n == 2 && m == 4);
    int64_t words = oracle_meta_words(R, K, n, m);
    for (int64_t i = 0; i < words; i++) meta[i] = tiled ? 0x44444444u : 0u;
    for (int64_t r = 0; r < R; r++) {
        int64_t j = 0;
        for (int64_t g = 0; g < K / m; g++) {
            uint32_t nib = 0;
            int seen = 0;
            for (int p = 0; p < m; p++) {
                if (!mask[r * K + g * m + p]) continue;
                values[r * vcols + j] = W[r * ldw + g * m + p];
                if (tiled)
                    nib |= (uint32_t)p << (2 * seen);
                else
                    meta[r * mcols + j / s] |= (uint32_t)p << (b * (j % s));
                seen++;
                j++;
            }
            if (tiled) {
                int bit;
                int64_t w = meta_slot_2of4(r, g, K, &bit);
                meta[w] = (meta[w] & ~(0xFu << bit)) | (nib << bit);
            }
        }
    }
    free(mask);
    return 0;
}

int oracle_decompress_f32(const uint32_t *values, const uint32_t *meta, int64_t R, int64_t K, int n, int m,
                          uint32_t *W_out, int64_t ldw)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldw < K) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t k = 0; k < K; k++) W_out[r * ldw + k] = 0u; /* +0.0 */
        for (int64_t j = 0; j < vcols; j++)
            W_out[r * ldw + (j / n) * m + position_of(meta, K, r, j, n, m)] = values[r * vcols + j];
    }
    return 0;
}

/* y[r][t] = sum_j V[r][j] * X[k_j][t] (float32 values, double sums);    */
/* Y_abs (optional) receives sum_j |V[r][j]| |X[k_j][t]|.                */
int oracle_spmm_f32(const uint32_t *values, const uint32_t *meta, int n, int m, int64_t R, int64_t K,
                    const uint32_t *X, int64_t ldx, int64_t T, double *Y, double *Y_abs, int64_t ldy)
{
    if (!pattern_ok(n, m) || K % m != 0 || ldx < T || ldy < T) return 1;
    int64_t vcols = oracle_value_cols(K, n, m);
    for (int64_t r = 0; r < R; r++) {
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t j = 0; j < vcols; j++) {
                int64_t k = (j / n) * m + position_of(meta, K, r, j, n, m);
                double w = f32_value(values[r * vcols + j]), x = f32_value(X[k * ldx + t]);
                acc += w * x;
                mag += fabs(w) * fabs(x);
            }
            Y[r * ldy + t] = acc;
            if (Y_abs) Y_abs[r * ldy + t] = mag;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Diagonal sparsity [DIAG] (readings in the header).                   */
/* ------------------------------------------------------------------ */
/* s(o) = sum_r |W[r][(r + o) mod K]|, accumulated in double with r
 * ascending.  A bf16 magnitude is exact in double, and for the sizes used
 * here (R <= 2^20 rows of bf16 magnitudes) the rounding of this sum is far
 * below the gap a float32 sum could resolve. */
int oracle_diag_scores(const uint16_t *W, int64_t R, int64_t K, int64_t ldw, double *scores)
{
    if (K <= 0 || ldw < K) return 1;
    for (int64_t o = 0; o < K; o++) {
        double total = 0.0;
        for (int64_t r = 0; r < R; r++) total += fabs(bf16_value(W[r * ldw + (r + o) % K]));
        scores[o] = total;
    }
    return 0;
}

/* Does offset a (score sa) rank above offset b (score sb)? */
static int diag_beats(double sa, int64_t a, double sb, int64_t b)
{
    int na = isnan(sa), nb = isnan(sb);
    if (na || nb) {
        if (na && !nb) return 1;
        if (nb && !na) return 0;
        return a < b;
    }
    if (sa != sb) return sa > sb;
    return a < b;
}

/* The D best offsets by score, written in ascending order. */
int oracle_diag_select(const uint16_t *W, int64_t R, int64_t K, int64_t ldw, int64_t D, int32_t *offsets)
{
    if (K <= 0 || D < 0 || D > K || ldw < K) return 1;
    double *s = (double *)malloc((size_t)K * sizeof(double));
    if (!s) return 2;
    oracle_diag_scores(W, R, K, ldw, s);
    int64_t n = 0;
    for (int64_t o = 0; o < K; o++) {
        int64_t rank = 0;
        for (int64_t p = 0; p < K; p++)
            if (p != o && diag_beats(s[p], p, s[o], o)) rank++;
        if (rank < D) offsets[n++] = (int32_t)o;
    }
    free(s);
    return n == D ? 0 : 3;
}

/* V[d][r] = W[r][(r + o_d) mod K]. */
int oracle_diag_compress(const uint16_t *W, int64_t R, int64_t K, int64_t ldw, int64_t D, const int32_t *offsets,
                         uint16_t *values)
{
    if (K <= 0 || ldw < K) return 1;
    for (int64_t d = 0; d < D; d++)
        for (int64_t r = 0; r < R; r++) values[d * R + r] = W[r * ldw + (r + offsets[d]) % K];
    return 0;
}

/* The dense R x K matrix of a diagonal operand: +0 off the kept diagonals. */
int oracle_diag_expand(const uint16_t *values, const int32_t *offsets, int64_t D, int64_t R, int64_t K,
                       uint16_t *W_out, int64_t ldw)
{
    if (K <= 0 || ldw < K) return 1;
    for (int64_t r = 0; r < R; r++)
        for (int64_t k = 0; k < K; k++) W_out[r * ldw + k] = 0;
    for (int64_t d = 0; d < D; d++)
        for (int64_t r = 0; r < R; r++) W_out[r * ldw + (r + offsets[d]) % K] = values[d * R + r];
    return 0;
}

/* y[r][t] = sum_d V[d][r] * X[pi((r + o_d) mod K)][t] in double; y_abs gets the sums of |products|. */
int oracle_diag_spmm(const uint16_t *values, const int32_t *offsets, int64_t D, int64_t R, int64_t K,
                     const uint16_t *X, int64_t ldx, int64_t T, const int32_t *idx, double *Y, double *Y_abs,
                     int64_t ldy)
{
    if (K <= 0 || ldx < T || ldy < T) return 1;
    for (int64_t r = 0; r < R; r++) {
        for (int64_t t = 0; t < T; t++) {
            double acc = 0.0, mag = 0.0;
            for (int64_t d = 0; d < D; d++) {
                int64_t k = (r + offsets[d]) % K;
                int64_t src = idx ? (int64_t)idx[k] : k;
                double w = bf16_value(values[d * R + r]);
                double x = (src < 0 || src >= K) ? 0.0 : bf16_value(X[src * ldx + t]);
                acc += w * x;
                mag += fabs(w) * fabs(x);
            }
            Y[r * ldy + t] = acc;
            if (Y_abs) Y_abs[r * ldy + t] = mag;
        }
    }
    return 0;
}
