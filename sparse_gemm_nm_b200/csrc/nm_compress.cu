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
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_select.cuh"

namespace nmk {

__device__ __forceinline__ uint32_t mag_key(uint32_t bits16) {
  const uint32_t k = bits16 & 0x7FFFu;
  return k > 0x7F80u ? 0x7F81u : k;
}

// 2:4 with tiled metadata.  One warp per metadata block (16 rows x 128
// columns).  Load i (0..7) of the warp reads rows 2i and 2i+1 of the block,
// 256 contiguous bytes each: lane l takes row 2i + l/16 and the eight
// columns 8*(l%16) .. +7 (two groups).  So a lane holds the same two groups of
// eight rows, every load and every value store of the warp covers whole
// 128-byte lines, and each lane keeps one byte of nibbles per row (rows
// 2k + l/16: k = 0..3 in `lo8`, k = 4..7 in `hi8`).  The block's 64 words are
// assembled with shuffles, two per lane.  The group selection is select_quad
// (two groups per call, nm_select.cuh); select_pair for a lone group at a ragged edge.
__global__ void __launch_bounds__(256, 4) compress_2of4_tiled_kernel(const uint16_t* __restrict__ W, uint32_t R,
                                                                  uint32_t K, int64_t ldw,
                                                                  uint16_t* __restrict__ V,
                                                                  uint32_t* __restrict__ meta, uint32_t cblocks,
                                                                  uint32_t nblocks, bool vec) {
  pdl_gate();
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  const uint32_t half = lane >> 4, piece = lane & 15u;
  for (uint32_t blk = warp; blk < nblocks; blk += nwarps) {
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint32_t col = cb * 128 + 8 * piece;  // this lane's first column
    uint32_t lo8 = 0x44444444u, hi8 = 0x44444444u;
    if (vec) {  // K % 8 == 0: a piece is wholly inside or wholly outside
      uint4 in[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t row = rb * 16 + 2 * i + half;
        if (row < R && col < K) in[i] = __ldg(reinterpret_cast<const uint4*>(W + (int64_t)row * ldw + col));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t row = rb * 16 + 2 * i + half;
        uint32_t byte = 0x44u;
        if (row < R && col < K) {
          uint32_t v0, v1;
          byte = select_quad(in[i], v0, v1);
          *reinterpret_cast<uint2*>(V + (int64_t)row * (K >> 1) + col / 2) = make_uint2(v0, v1);
        }
        if (i < 4) lo8 = (lo8 & ~(0xFFu << (8 * i))) | (byte << (8 * i));
        else hi8 = (hi8 & ~(0xFFu << (8 * (i - 4)))) | (byte << (8 * (i - 4)));
      }
    } else {
      for (int i = 0; i < 8; ++i) {
        const uint32_t row = rb * 16 + 2 * i + half;
        uint32_t byte = 0x44u;
        if (row < R) {
          const uint16_t* wrow = W + (int64_t)row * ldw;
          uint32_t* vrow = reinterpret_cast<uint32_t*>(V + (int64_t)row * (K >> 1));
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const uint32_t cg = col + 4 * g;
            if (cg < K) {
              const uint32_t lo = (uint32_t)wrow[cg] | ((uint32_t)wrow[cg + 1] << 16);
              const uint32_t hi = (uint32_t)wrow[cg + 2] | ((uint32_t)wrow[cg + 3] << 16);
              uint32_t pk;
              const uint32_t nib = select_pair(lo, hi, pk);
              vrow[cg / 4] = pk;  // value column cg / 2
              byte = (byte & ~(0xFu << (4 * g))) | (nib << (4 * g));
            }
          }
        }
        if (i < 4) lo8 = (lo8 & ~(0xFFu << (8 * i))) | (byte << (8 * i));
        else hi8 = (hi8 & ~(0xFFu << (8 * (i - 4)))) | (byte << (8 * (i - 4)));
      }
    }
    // Words 2L (quarter q = 2*(L%2)) and 2L+1 (q + 1) of tile lane l = L/2:
    // row r = l%8 (low half) and 8 + r (high half), column half h = l/8.
    // The nibble byte of (row r, piece p) sits in lane 16*(r%2) + p, byte
    // r/2 of lo8 (low row) or hi8 (high row); quarter q takes pieces
    // 4q + 2h and 4q + 2h + 1.
    const uint32_t l = lane >> 1, r = l & 7u, h = l >> 3, k = r >> 1;
    const uint32_t s0 = 16 * (r & 1u) + 8 * (lane & 1u) + 2 * h;  // source lane of quarter q's first piece
    const uint32_t a0 = __shfl_sync(0xffffffffu, lo8, s0), a1 = __shfl_sync(0xffffffffu, lo8, s0 + 1);
    const uint32_t b0 = __shfl_sync(0xffffffffu, hi8, s0), b1 = __shfl_sync(0xffffffffu, hi8, s0 + 1);
    const uint32_t c0 = __shfl_sync(0xffffffffu, lo8, s0 + 4), c1 = __shfl_sync(0xffffffffu, lo8, s0 + 5);
    const uint32_t d0 = __shfl_sync(0xffffffffu, hi8, s0 + 4), d1 = __shfl_sync(0xffffffffu, hi8, s0 + 5);
    const uint32_t pick = k | ((k + 4) << 4);  // byte k of the first operand, then byte k of the second
    const uint32_t w0 = __byte_perm(__byte_perm(a0, a1, pick), __byte_perm(b0, b1, pick), 0x5410u);
    const uint32_t w1 = __byte_perm(__byte_perm(c0, c1, pick), __byte_perm(d0, d1, pick), 0x5410u);
    *reinterpret_cast<uint2*>(meta + (int64_t)blk * 64 + 2 * lane) = make_uint2(w0, w1);
  }
}

// Row-wise patterns with whole 16-byte pieces (K % 8 == 0, 16-byte aligned
// rows): 1:2, 1:4, 3:4, 1:8, 2:8, 3:8, 4:8.  Lanes read consecutive 16-byte
// pieces of one row (a warp load is 512 contiguous bytes); a piece is 8/M
// groups for M <= 8.  Each group keeps its N largest combined keys
// (magnitude key, then the lower index: key << log2(M) | (M - 1 - i), all
// distinct), found by N rounds of a max over the group; the kept positions
// are then emitted in ascending order.  A work unit is one row and one span of
// groups whose survivors fill whole metadata words (UNITS pieces per lane);
// every lane parks its survivors' position codes in shared memory, and after
// a warp barrier each lane ORs the codes of its own words (S codes of b bits)
// and stores them.  Value stores are 2-byte per survivor, contiguous across the
// warp.
template <int M, int N>
struct RowwisePlan {
  static constexpr int B = M == 2 ? 1 : M == 4 ? 2 : 3;        // position bits
  static constexpr int S = 32 / B;                              // positions per word
  static constexpr int G = 8 / M;                               // groups per 16-byte piece
  static constexpr int PER_PIECE = G * N;                       // survivors per piece
  static constexpr int gcd(int a, int b) { return b == 0 ? a : gcd(b, a % b); }
  static constexpr int BASE = S / gcd(S, 32 * PER_PIECE);       // pieces per lane to fill whole words
  static constexpr int UNITS = BASE >= 4 ? BASE : BASE * ((4 + BASE - 1) / BASE);  // >= 4 loads in flight
  static constexpr int SURV = 32 * PER_PIECE * UNITS;           // survivors per work unit
  static constexpr int WORDS = SURV / S;                        // metadata words per work unit
  static constexpr int GROUPS = 32 * G * UNITS;                 // groups per work unit
};

template <int M, int N>
__global__ void __launch_bounds__(256) compress_rowwise_warp_kernel(const uint16_t* __restrict__ W, int64_t R,
                                                                    int64_t K, int64_t ldw,
                                                                    uint16_t* __restrict__ V,
                                                                    uint32_t* __restrict__ meta) {
  using P = RowwisePlan<M, N>;
  static_assert(P::SURV % P::S == 0, "a work unit must fill whole words");
  constexpr int LOGM = M == 2 ? 1 : M == 4 ? 2 : 3;
  __shared__ uint8_t codes[8][P::SURV];
  pdl_gate();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t ngroups = K / M;
  const int64_t vcols = ngroups * N;
  const int64_t mcols = (vcols + P::S - 1) / P::S;
  const int64_t units_per_row = (ngroups + P::GROUPS - 1) / P::GROUPS;
  const int64_t units = R * units_per_row;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  uint8_t* my = codes[wib];
  for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib; u < units; u += nwarps) {
    const int64_t row = u / units_per_row;
    const int64_t g0 = (u - row * units_per_row) * P::GROUPS;  // first group of the unit
    const uint16_t* wrow = W + row * ldw;
    uint4 in[P::UNITS];
#pragma unroll
    for (int i = 0; i < P::UNITS; ++i) {
      const int64_t g = g0 + (int64_t)(i * 32 + lane) * P::G;
      in[i] = g < ngroups ? __ldg(reinterpret_cast<const uint4*>(wrow + g * M)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < P::UNITS; ++i) {
      const int piece = i * 32 + lane;
      const int64_t gp = g0 + (int64_t)piece * P::G;
      const uint32_t w4[4] = {in[i].x, in[i].y, in[i].z, in[i].w};
#pragma unroll
      for (int gg = 0; gg < P::G; ++gg) {
        uint32_t ck[M];
#pragma unroll
        for (int e = 0; e < M; ++e) {
          const int flat = gg * M + e;  // element of the piece
          const uint32_t b16 = (w4[flat >> 1] >> (16 * (flat & 1))) & 0xFFFFu;
          ck[e] = (mag_key(b16) << LOGM) | (uint32_t)(M - 1 - e);
        }
        uint32_t keep = 0;  // bit e: element e survives
#pragma unroll
        for (int t = 0; t < N; ++t) {
          uint32_t best = 0;
#pragma unroll
          for (int e = 0; e < M; ++e) best = max(best, (keep >> e) & 1u ? 0u : ck[e]);
          keep |= 1u << (M - 1 - (best & (M - 1)));
        }
        const bool valid = gp + gg < ngroups;
        const int64_t j0 = (gp + gg) * N;  // first survivor of the group in the row
        const int sc0 = (piece * P::G + gg) * N;  // its slot in the unit
#pragma unroll
        for (int t = 0; t < N; ++t) {
          const uint32_t p = __ffs(keep) - 1u;
          keep &= keep - 1u;
          const int flat = gg * M + (int)p;
          const uint32_t word = (flat >> 1) == 0 ? w4[0] : (flat >> 1) == 1 ? w4[1] : (flat >> 1) == 2 ? w4[2] : w4[3];
          if (valid) V[row * vcols + j0 + t] = (uint16_t)((word >> (16 * (flat & 1))) & 0xFFFFu);
          my[sc0 + t] = valid ? (uint8_t)p : (uint8_t)0;
        }
      }
    }
    __syncwarp();
    const int64_t w0 = (g0 * N) / P::S;  // first word of the unit (units start on word boundaries)
#pragma unroll
    for (int w = lane; w < P::WORDS; w += 32) {
      if (w0 + w < mcols) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < P::S; ++j) word |= (uint32_t)my[w * P::S + j] << (P::B * j);
        meta[row * mcols + w0 + w] = word;
      }
    }
    __syncwarp();
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
  pdl_gate();
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
                                                                    bool vec, const uint8_t* __restrict__ tile_map,
                                                                    uint32_t rtiles) {
  pdl_gate();
  for (uint32_t w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += gridDim.x * blockDim.x) {
    const uint32_t blk = w >> 6, wi = w & 63u;
    const uint32_t l = wi >> 2, q = wi & 3u;
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint32_t r_lo = rb * 16 + (l & 7u);
    const uint32_t k0 = cb * 128 + q * 32 + (l >> 3) * 16;
    if (k0 >= K) continue;
    // With a tile map (128 x 128 tiles, one column block each): the 2:4 tiles
    // that the SM-pair hybrid kernel reads as dense tiles, i.e. those whose
    // partner row tile (the other 128 rows of the pair's 256) exists and is
    // dense in the same column block.  Where both are 2:4 the stage runs the
    // sparse MMA on the compressed form; a lone last row tile pairs with itself.
    if (tile_map) {
      const uint32_t t = r_lo >> 7, partner = t ^ 1u;
      if (__ldg(tile_map + (int64_t)t * cblocks + cb) == 0 || partner >= rtiles ||
          __ldg(tile_map + (int64_t)partner * cblocks + cb) != 0)
        continue;
    }
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
  pdl_gate();
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
  pdl_gate();
  const int64_t total = R * row_bytes;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / row_bytes;
    Y[r * ld_bytes + (i - r * row_bytes)] = 0;
  }
}

// Row gather Xp[k][0..T) = X[idx[k]][0..T).  Work items are (row, 4 KB chunk)
// pairs so that long rows (large T) spread over many warps; a warp loads its
// chunk as 8 x 16 bytes per lane, all in flight, then stores it.  Entries of
// idx outside [0, K) give zero rows.  X and Xp rows are 16-byte aligned
// (T % 8 == 0).  Persistent grid of kGatherCtasPerSm CTAs per SM (the dynamic
// shared memory it requests, unused, caps residency there): as a programmatic
// dependent the kernel is placed on SMs while the previous kernel drains, and
// without the cap all of it could land on the first few SMs to free up.
constexpr int kGatherCtasPerSm = 4;
constexpr size_t kGatherSmemCap = 56 * 1024;

__global__ void __launch_bounds__(256) gather_rows_kernel(const GatherJob g) {
  pdl_gate();
  if (g.skip_if && *reinterpret_cast<const volatile uint32_t*>(g.skip_if)) return;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  gather_rows_items(g, warp, nwarps, threadIdx.x & 31);
}

// Re-encoding of an N:M operand whose survivors never exceed two per aligned
// group of four (1:2, 1:4, 2:4, 1:8, 2:8) as a 2:4 operand with tiled
// metadata, so that the two-SM sparse GEMM can run it.  A group of four keeps
// its survivors (ascending); one survivor is paired with a +0.0 at the lowest
// other position, none gives (0, 1) with two zeros.  One thread per row and
// 16-column chunk (one 16-bit half of a tiled metadata word); rows and
// columns of the padded blocks get the padding nibbles 0x4.
template <int M>
__global__ void __launch_bounds__(256) reencode_2of4_kernel(const uint16_t* __restrict__ V,
                                                            const uint32_t* __restrict__ meta, uint32_t R,
                                                            uint32_t K, int n, uint32_t vcols, uint32_t mcols,
                                                            uint16_t* __restrict__ V2, uint16_t* __restrict__ meta2,
                                                            uint32_t cblocks, uint32_t total) {
  pdl_gate();
  constexpr int B = M == 2 ? 1 : M == 4 ? 2 : 3;
  constexpr int S = 32 / B;
  const uint32_t chunks = cblocks * 8;
  for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
    const uint32_t r = t / chunks, c = t - r * chunks;
    const uint32_t cb = c >> 3, qh = c & 7u;  // block column 16*qh = 32q + 16h
    const uint32_t k0 = cb * 128 + 16 * qh;
    const uint32_t word = ((r >> 4) * cblocks + cb) * 64 + 4 * ((r & 7u) + 8 * (qh & 1u)) + (qh >> 1);
    uint32_t nib16 = 0x4444u;
    if (r < R && k0 < K) {
      nib16 = 0;
      uint32_t out[4];
      for (int g4 = 0; g4 < 4; ++g4) {
        const uint32_t c4 = k0 + 4 * g4;  // first column of this group of four
        uint32_t pos[2] = {0, 1}, val[2] = {0, 0};
        int cnt = 0;
        if (c4 < K) {
          const uint32_t g_first = c4 / M, g_last = (c4 + 3) / M;  // N:M groups overlapping [c4, c4 + 4)
          for (uint32_t g = g_first; g <= g_last; ++g) {
            for (int s = 0; s < n; ++s) {
              const uint32_t j = g * n + s;
              const uint32_t pw = __ldg(meta + (int64_t)r * mcols + j / S);
              const uint32_t col = g * M + ((pw >> (B * (j % S))) & ((1u << B) - 1u));
              if (col >= c4 && col < c4 + 4 && cnt < 2) {
                pos[cnt] = col - c4;
                val[cnt] = V[(int64_t)r * vcols + j];
                ++cnt;
              }
            }
          }
        }
        uint32_t p0 = pos[0], p1 = pos[1], v0 = val[0], v1 = val[1];
        if (cnt == 1) {  // pair the survivor with a zero at the lowest other position
          if (pos[0] == 0) { p0 = 0; p1 = 1; v0 = val[0]; v1 = 0; }
          else { p0 = 0; p1 = pos[0]; v0 = 0; v1 = val[0]; }
        }
        nib16 |= (p0 | (p1 << 2)) << (4 * g4);
        out[g4] = v0 | (v1 << 16);
      }
      uint32_t* vrow = reinterpret_cast<uint32_t*>(V2 + (int64_t)r * (K >> 1) + k0 / 2);
      for (int g4 = 0; g4 < 4; ++g4)
        if (k0 + 4 * g4 < K) vrow[g4] = out[g4];
    }
    meta2[2 * (int64_t)word + ((r >> 3) & 1u)] = (uint16_t)nib16;
  }
}

static int grid_for(int64_t work, int threads) {
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count_current() * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Row-wise patterns served by compress_rowwise_warp_kernel.
static bool rowwise_warp_pattern(int n, int m) {
  return (m == 2 && n == 1) || (m == 4 && (n == 1 || n == 3)) || (m == 8 && n >= 1 && n <= 4);
}

cudaError_t launch_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint16_t* values,
                            uint32_t* meta, cudaStream_t s) {
  const int threads = 256;
  if (tiled_meta(n, m)) {
    const int64_t nblocks = meta_row_blocks(R) * meta_col_blocks(K);
    const bool vec = K % 8 == 0 && ldw % 8 == 0 && aligned16(W) && aligned16(values);
    launch_pdl(compress_2of4_tiled_kernel, grid_for(nblocks * 32, threads), threads, 0, s,
        W, (uint32_t)R, (uint32_t)K, ldw, values, meta, (uint32_t)meta_col_blocks(K), (uint32_t)nblocks, vec);
  } else if (K % 8 == 0 && ldw % 8 == 0 && aligned16(W) && rowwise_warp_pattern(n, m)) {
    // one warp per work unit (a row's span of groups filling whole words); 8 warps per block
    auto units = [&](int groups) { return R * ((K / m + groups - 1) / groups); };
    auto go = [&](auto kernel, int groups) {
      const int64_t want = (units(groups) + 7) / 8;
      const int64_t cap = (int64_t)sm_count_current() * 8;
      launch_pdl(kernel, (int)(want < cap ? (want > 0 ? want : 1) : cap), threads, 0, s, W, R, K, ldw, values, meta);
    };
    if (n == 1 && m == 2) go(compress_rowwise_warp_kernel<2, 1>, RowwisePlan<2, 1>::GROUPS);
    else if (n == 1 && m == 4) go(compress_rowwise_warp_kernel<4, 1>, RowwisePlan<4, 1>::GROUPS);
    else if (n == 3 && m == 4) go(compress_rowwise_warp_kernel<4, 3>, RowwisePlan<4, 3>::GROUPS);
    else if (n == 1 && m == 8) go(compress_rowwise_warp_kernel<8, 1>, RowwisePlan<8, 1>::GROUPS);
    else if (n == 2 && m == 8) go(compress_rowwise_warp_kernel<8, 2>, RowwisePlan<8, 2>::GROUPS);
    else if (n == 3 && m == 8) go(compress_rowwise_warp_kernel<8, 3>, RowwisePlan<8, 3>::GROUPS);
    else go(compress_rowwise_warp_kernel<8, 4>, RowwisePlan<8, 4>::GROUPS);
  } else {
    const int64_t work = R * meta_cols(K, n, m);
    const int grid = grid_for(work, threads);
    switch (m) {
      case 2: launch_pdl(compress_generic_kernel<2>, grid, threads, 0, s, W, R, K, ldw, n, values, meta); break;
      case 4: launch_pdl(compress_generic_kernel<4>, grid, threads, 0, s, W, R, K, ldw, n, values, meta); break;
      case 8: launch_pdl(compress_generic_kernel<8>, grid, threads, 0, s, W, R, K, ldw, n, values, meta); break;
      default: launch_pdl(compress_generic_kernel<16>, grid, threads, 0, s, W, R, K, ldw, n, values, meta); break;
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
    launch_pdl(decompress_2of4_tiled_kernel, grid_for(total, threads), threads, 0, s,
        values, meta, (uint32_t)R, (uint32_t)K, W_out, ldw, (uint32_t)meta_col_blocks(K), (uint32_t)total, vec,
        nullptr, 0u);
  } else {
    const int64_t work = R * (K / m);
    const int grid = grid_for(work, threads);
    switch (m) {
      case 2: launch_pdl(decompress_generic_kernel<2>, grid, threads, 0, s, values, meta, R, K, n, W_out, ldw); break;
      case 4: launch_pdl(decompress_generic_kernel<4>, grid, threads, 0, s, values, meta, R, K, n, W_out, ldw); break;
      case 8: launch_pdl(decompress_generic_kernel<8>, grid, threads, 0, s, values, meta, R, K, n, W_out, ldw); break;
      default: launch_pdl(decompress_generic_kernel<16>, grid, threads, 0, s, values, meta, R, K, n, W_out, ldw); break;
    }
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_decompress_tiles(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K,
                                    const uint8_t* tile_map, uint16_t* W_out, int64_t ldw, cudaStream_t s) {
  const int threads = 256;
  const int64_t total = meta_words(R, K, 2, 4);
  const bool vec = K % 16 == 0 && ldw % 8 == 0 && aligned16(W_out) && aligned16(values);
  launch_pdl(decompress_2of4_tiled_kernel, grid_for(total, threads), threads, 0, s,
      values, meta, (uint32_t)R, (uint32_t)K, W_out, ldw, (uint32_t)meta_col_blocks(K), (uint32_t)total, vec,
      tile_map, (uint32_t)((R + 127) / 128));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* X, int64_t ldx, const int32_t* idx, int64_t K, int64_t T,
                               uint16_t* Xp, int64_t ldp, cudaStream_t s, const uint32_t* skip_if) {
  const int threads = 256;
  static std::atomic<bool> configured[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gather_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kGatherSmemCap);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int64_t items = K * (((T + 7) / 8 + 255) / 256);
  const int64_t want = (items + 7) / 8;  // 8 warps per CTA
  const int64_t cap = (int64_t)sm_count_current() * kGatherCtasPerSm;
  const int grid = (int)(want < cap ? (want > 0 ? want : 1) : cap);
  const GatherJob g{X, ldx, idx, K, T, Xp, ldp, skip_if};
  cudaError_t e = launch_pdl(gather_rows_kernel, grid, threads, kGatherSmemCap, s, g);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_fill_zero(void* Y, int64_t R, int64_t T, int64_t ldy, int esize, cudaStream_t s) {
  const int threads = 256;
  launch_pdl(fill_zero_kernel, grid_for(R * T * esize, threads), threads, 0, s, static_cast<uint8_t*>(Y), R, T * esize,
                                                                         ldy * esize);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_reencode_2of4(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K, int n, int m,
                                 uint16_t* values2, uint32_t* meta2, cudaStream_t s) {
  const int threads = 256;
  const int64_t cblocks = meta_col_blocks(K);
  const int64_t total = meta_row_blocks(R) * 16 * cblocks * 8;
  const int grid = grid_for(total, threads);
  const uint32_t vcols = (uint32_t)value_cols(K, n, m), mcols = (uint32_t)meta_cols(K, n, m);
  uint16_t* m16 = reinterpret_cast<uint16_t*>(meta2);
  switch (m) {
    case 2: launch_pdl(reencode_2of4_kernel<2>, grid, threads, 0, s, values, meta, (uint32_t)R, (uint32_t)K, n, vcols, mcols,
                                                                values2, m16, (uint32_t)cblocks, (uint32_t)total); break;
    case 4: launch_pdl(reencode_2of4_kernel<4>, grid, threads, 0, s, values, meta, (uint32_t)R, (uint32_t)K, n, vcols, mcols,
                                                                values2, m16, (uint32_t)cblocks, (uint32_t)total); break;
    case 8: launch_pdl(reencode_2of4_kernel<8>, grid, threads, 0, s, values, meta, (uint32_t)R, (uint32_t)K, n, vcols, mcols,
                                                                values2, m16, (uint32_t)cblocks, (uint32_t)total); break;
    default: return cudaErrorInvalidValue;
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace nmk
