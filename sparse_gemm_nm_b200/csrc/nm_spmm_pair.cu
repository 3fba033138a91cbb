// nm_spmm_pair.cu -- 2:4 sparse x dense GEMM on a pair of SMs (tcgen05 cta_group::2).
//
// Same operation as nm_spmm.cu (Y = W' X with W' stored as 2:4 values plus
// row-wise 2-bit positions; "M:N sparsity on NVIDIA tensor cores", GEMM
// paragraphs of "Where this sits among the three case studies"), laid out so
// that the tensor cores of two SMs share one 256 x 256 output tile: each CTA
// of the cluster stages its own 128 rows of the compressed weights and its own
// 128 columns of X, and one MMA instruction of the leader CTA consumes both.
// Per SM this halves the X bytes per useful FLOP compared with a 128 x 256
// tile on one SM, which is what bounds a 2:4 GEMM: the sparse MMA reads a
// dense X tile twice as fast as the dense MMA would.
//
// Pipeline (per CTA, 4 stages of 128 logical K):
//   A  compressed values, 128 rows x 64 (16 KB) as two 64-row boxes, TMA,
//      128-byte swizzle
//   B  X rows k0..k0+127, this CTA's 128 columns (32 KB) as four boxes of
//      64 rows x 64 columns, TMA
//   E  2:4 metadata of the 128 rows (2 KB): eight tiled 16-row blocks, already
//      in the order tcgen05.cp hands to the tensor core, one 3-D TMA box
// The seven boxes of a stage are issued by seven different warps (in an
// isolated copy test on B200, boxes from separate issuing warps overlapped
// about 2.5x better than the same boxes queued by one thread; in this kernel
// the split measures neutral, because the MMA issue rate, not the copies,
// sets the stage period).  No issuer waits for anything but a free stage.  All copies of both CTAs complete on the
// leader's barrier, which expects the bytes of both.  The leader's MMA thread
// copies E into TMEM (tcgen05.cp, both CTAs) and issues four tcgen05.mma.sp
// (M = 256, N = 256, K = 32) per stage; its commits release the stage in both
// CTAs.  Each CTA drains its own 128 x 256 fp32 accumulator.
//
// Tile order: the persistent pairs take consecutive tiles.  Row tiles go
// fastest, unless the compressed weights are well larger than X (n_major):
// then column tiles go fastest, the pairs running together share a row block
// of the weights, and the weights stream from HBM about once (a TF32 launch
// list read 605 MB of DRAM for 215 MB of operands with row tiles fastest).
//
// Short tiles (DB): a tile of few stages spends about as long handing its
// accumulator over (MMA completion, TMEM drain, release) as computing it; on a
// six-stage ViT tile a trace showed ~2.3 us of MMAs and ~1.6 us until the next
// tile's first MMA.  Two accumulators let the next tile's MMAs run while the
// epilogue drains, but two 256-column fp32 accumulators fill all 512 TMEM
// columns and leave none for the sparse metadata.  So the DB form uses 256 x 224
// tiles (each CTA supplies 112 columns of X: its first 64-column strip and 48
// columns of its second) and two 224-column accumulators (TMEM columns 0 and 256,
// metadata from column 480).  A stage costs about the same at N = 192, 224 or 256
// (each CTA loads both 64-column strips whole), so the widest N whose two
// accumulators leave room for the metadata covers the most columns per stage.  It keeps four stages: a trace of the three-stage form on the
// ViT shape showed the MMA thread waiting ~240 ns of each ~600 ns stage for data
// (X rows 100 KB apart, a third of them from HBM).
//
// INT8 (I8): the same pipeline on the sparse kind::i8 MMA.  A stage covers 256
// logical K: A is 128 rows x 128 stored bytes (16 KB), B 256 rows x this CTA's
// 128 int8 columns (32 KB, four 64-row boxes), and the metadata 4 KB per CTA in
// the per-row order that MMA reads (relayout_meta_i8_kernel), copied into 8
// TMEM columns; four K = 64 MMAs per stage, int32 accumulators stored as such.
// TF32 1:2 (TF32): the same on the sparse kind::tf32 MMA.  A stage covers 64
// logical K: A 128 rows x 32 stored fp32, B 64 rows x 128 fp32 columns (four
// 32-column strips in the 32-byte-unit swizzle the MMA reads for MN-major
// 32-bit operands), 4 KB of metadata (relayout_meta_tf32_kernel); four K = 16
// MMAs per stage, each with its own even TMEM metadata column.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_spmm.h"

namespace nmk {

namespace pair {
constexpr int kThreads = 384;  // warps 0,2-5,10,11 copies; 1 MMA; 6-9 epilogue
constexpr uint32_t kB = 32768;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kIdescDense = idesc_bf16(256, false, 256);
constexpr uint32_t kEpi = 4096;  // per epilogue warp: 32 rows x 64 bf16 columns, 128-byte swizzle

struct Layout {
  uint32_t a, b, e, epi, bar, total;
};
// HYB = false: 2:4 only, A slots of 16 KB (compressed values), four stages.
// HYB = true (PATCH hybrid): A slots of 32 KB so that a stage can hold the
// dense 128 x 128 tile instead, three stages.
// DB = true (2:4, short tiles): 256 x 224 tiles, two accumulators, four stages.
template <bool HYB, bool DB = false, bool I8 = false, bool TF32 = false>
struct Cfg {
  static_assert(!((I8 || TF32) && (HYB || DB)) && !(I8 && TF32), "int8 / tf32 run the 256 x 256 sparse form only");
  static constexpr bool kWideE = I8 || TF32;  // 4 KB metadata chunks staged per row block and stage
  static constexpr int kStages = HYB ? 3 : 4;
  static constexpr uint32_t kN = DB ? 224u : 256u;  // pair tile columns (per CTA: kN / 2 of X)
  static constexpr int kAcc = DB ? 2 : 1;           // accumulators, 256 TMEM columns apart
  static constexpr uint32_t kECol = DB ? 480u : 256u;
  static constexpr uint32_t kE = kWideE ? 4096u : 2048u;  // metadata bytes per stage and CTA
  static constexpr uint32_t kECols = kWideE ? 8u : 4u;    // its TMEM columns
  static constexpr int kEpiBufs = 1;
  static constexpr uint32_t kIdesc = I8     ? (idesc_s8_major(256, 256, false, true) | (1u << 2))
                                     : TF32 ? (idesc_tf32_major(256, 256, false, true) | (1u << 2))
                                            : idesc_bf16(kN, true, 256);
  static constexpr uint32_t kA = HYB ? 32768u : 16384u;
  static constexpr uint32_t kTxSparse = 2u * (16384u + kB + kE);  // both CTAs' A, B and E bytes
  static constexpr uint32_t kTxDense = 2u * (32768u + kB);        // both CTAs' dense A and B bytes
  static constexpr uint32_t kBars = (2 * kStages + 6) * 8;        // full, empty, acc_full[2], acc_empty[2], spare[2]
  __host__ __device__ static constexpr Layout layout() {
    return Layout{0u, kStages * kA, kStages * (kA + kB), kStages * (kA + kB + kE),
                  kStages * (kA + kB + kE) + 4 * kEpiBufs * kEpi,
                  kStages * (kA + kB + kE) + 4 * kEpiBufs * kEpi + kBars + 64};
  }
  static_assert(kStages * (kA + kB + kE) + 4 * kEpiBufs * kEpi + kBars + 64 + 1024 <= 232448, "shared memory");
  static_assert(kN <= 256 && (kN / 2) % 16 == 0, "each CTA supplies a multiple of 16 columns of X");
  static_assert(kECol >= 256u * (kAcc - 1) + kN && kECol + kECols * kStages <= kTmemCols, "TMEM columns");
};
}  // namespace pair

template <bool HYB, bool DB, bool I8, bool TF32>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::kThreads, 1)
    spmm_pair_kernel(const __grid_constant__ SpmmParams p) {
  using namespace pair;
  using C = Cfg<HYB, DB, I8, TF32>;
  constexpr uint32_t kE = C::kE;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kA = C::kA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr Layout L = C::layout();
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* spare = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(spare + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: follower
  const int pair_id = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);  // the leader's expect_tx; bytes from both CTAs
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);
    }
    mbar_init(spare, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_vals);
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_meta);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_gate();  // no global memory touched before this point

  const int64_t k_tiles = p.k_tiles;  // 128-deep stages (bf16) or 256-deep (int8), set by the host
  const uint32_t lead_full0 = map_to_cta(smem_u32(&full[0]), 0);
  const uint32_t lead_acc_empty0 = map_to_cta(smem_u32(acc_empty), 0);
  bool ok = true;
  // Hybrid: is the 128 x 128 weight tile (row block 2*tm + rr, k block kt) 2:4?
  // A stage runs the sparse MMA only when both CTAs' tiles are 2:4; otherwise
  // both CTAs stage dense tiles (W, or W with the 2:4 mask applied).
  auto tile_sparse = [&](int tm, int64_t kt, int rr) -> bool {
    if (!HYB) return true;
    if (!p.tile_map) return false;  // dense design: every stage dense (W is the staged decompressed operand)
    int rb = 2 * tm + rr;
    if (rb >= p.hyb_rows) rb = 2 * tm;
    return __ldg(p.tile_map + (int64_t)rb * p.hyb_tiles_k + kt) != 0;
  };

  if (warp < 6 || warp >= 10) {
    if (warp == 1) {
      // ---------------------------------------------------------- MMA (leader)
      if (rank == 0 && lane == 0) {
        int s = 0, acc = 0;
        uint32_t ph = 0, aph = 0;  // aph bit a: phase of accumulator a
        for (int tile = pair_id; tile < p.num_tiles && ok; tile += npairs) {
          const int tm = p.n_major ? tile / p.tiles_n : tile % p.tiles_m;
          ok = mbar_wait(&acc_empty[acc], ((aph >> acc) & 1u) ^ 1u, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + 256u * (uint32_t)acc;
          for (int64_t kt = 0; kt < k_tiles; ++kt) {
            ok = mbar_wait(&full[s], ph, abort_flag, p.status, kWaitNs);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + L.a + s * kA);
            const uint32_t b_addr = smem_u32(smem + L.b + s * kB);
            const uint32_t e_tmem = tmem_base + C::kECol + C::kECols * s;
            if (I8) {  // four K = 64 steps: 32 stored bytes of A and 64 rows (8 KB) of B each
              tc_cp_128x256b_pair(e_tmem, smem_desc(smem_u32(smem + L.e + s * kE), 128, 256, SWZ_NONE));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024, SWZ_128B);
                const uint64_t bd = smem_desc(b_addr + kk * 8192, 32768, 1024, SWZ_128B);
                tc_mma_sp_pair_i8(d_tmem, ad, bd, e_tmem + 2u * (uint32_t)kk, C::kIdesc,
                                  (kt > 0 || kk > 0) ? 1u : 0u);
              }
            } else if (TF32) {  // four K = 16 steps: 32 bytes of A and 16 rows (2 KB per strip) of B each
              tc_cp_128x256b_pair(e_tmem, smem_desc(smem_u32(smem + L.e + s * kE), 128, 256, SWZ_NONE));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024, SWZ_128B);
                const uint64_t bd = smem_desc(b_addr + kk * 2048, 8192, 512, SWZ_128B_BASE32B);
                tc_mma_sp_pair_tf32(d_tmem, ad, bd, e_tmem + 2u * (uint32_t)kk, C::kIdesc,
                                    (kt > 0 || kk > 0) ? 1u : 0u);
              }
            } else if (tile_sparse(tm, kt, 0) && tile_sparse(tm, kt, 1)) {
              tc_cp_128x128b_pair(e_tmem, smem_desc(smem_u32(smem + L.e + s * kE), 2048, 128, SWZ_NONE));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024, SWZ_128B);
                const uint64_t bd = smem_desc(b_addr + kk * 4096, 16384, 1024, SWZ_128B);
                tc_mma_sp_pair(d_tmem, ad, bd, e_tmem + (uint32_t)(kk & 2), C::kIdesc | (uint32_t)(kk & 1),
                               (kt > 0 || kk > 0) ? 1u : 0u);
              }
            } else if (HYB) {  // dense A tile: [K half][128 rows][128 B], eight K = 16 MMAs
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t ad = smem_desc(a_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, SWZ_128B);
                const uint64_t bd = smem_desc(b_addr + kk * 2048, 16384, 1024, SWZ_128B);
                tc_mma_pair(d_tmem, ad, bd, kIdescDense, (kt > 0 || kk > 0) ? 1u : 0u);
              }
            }
            tc_commit_pair(&empty[s], 0x3);
            if (++s == kStages) { s = 0; ph ^= 1u; }
          }
          if (!ok) break;
          tc_commit_pair(&acc_full[acc], 0x3);
          aph ^= 1u << acc;
          if (C::kAcc == 2) acc ^= 1;
        }
        if (!ok) {
          tc_commit_pair(spare, 0x1);
          volatile int dummy = 0;
          mbar_wait(spare, 0, &dummy, p.status, 100000000ull);
        }
      }
    } else {
      // ------ copy issuers: warps 0/10 A halves, warps 2-5 B boxes, warp 11 metadata (E)
      if (lane == 0) {
        int s = 0;
        uint32_t ph = 0;
        for (int tile = pair_id; tile < p.num_tiles && ok; tile += npairs) {
          const int tm = p.n_major ? tile / p.tiles_n : tile % p.tiles_m;
          const int tn = p.n_major ? tile % p.tiles_n : tile / p.tiles_m;
          const int32_t row0 = tm * 256 + 128 * (int)rank;
          const int32_t col0 = tn * (int32_t)C::kN + (int32_t)(C::kN / 2) * (int)rank;
          for (int64_t kt = 0; kt < k_tiles; ++kt) {
            ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitNs);
            if (!ok) break;
            const uint32_t lead_full = lead_full0 + 8u * s;
            const bool sparse = tile_sparse(tm, kt, 0) && tile_sparse(tm, kt, 1);
            if (warp == 0 || warp == 10) {
              const int h = warp == 10;
              if (rank == 0 && h == 0) mbar_arrive_expect_tx(&full[s], sparse ? C::kTxSparse : C::kTxDense);
              if (sparse) {
                tma_load_2d_pair(smem + L.a + s * kA + h * 8192, &p.tm_vals, lead_full,
                                 (int32_t)(kt * (I8 ? 128 : TF32 ? 32 : 64)), row0 + 64 * h);
              } else if (HYB) {  // this CTA's dense tile: W, or W under the 2:4 mask if the tile is 2:4
                const CUtensorMap* src = tile_sparse(tm, kt, (int)rank) ? &p.tm_wm : &p.tm_w;
#pragma unroll
                for (int kh = 0; kh < 2; ++kh)
                  tma_load_2d_pair(smem + L.a + s * kA + kh * 16384 + h * 8192, src, lead_full,
                                   (int32_t)(kt * 128 + 64 * kh), row0 + 64 * h);
              }
            } else if (warp <= 5) {
              if (I8) {  // box K quarter q: 128 int8 columns x 64 rows of X
                const int q = warp - 2;
                tma_load_2d_pair(smem + L.b + s * kB + q * 8192, &p.tm_x, lead_full, col0,
                                 (int32_t)(kt * 256 + 64 * q));
              } else if (TF32) {  // strip j: 32 fp32 columns x 64 rows of X
                const int j = warp - 2;
                tma_load_2d_pair(smem + L.b + s * kB + j * 8192, &p.tm_x, lead_full, col0 + 32 * j,
                                 (int32_t)(kt * 64));
              } else {  // box (strip j, K half h): 64 columns x 64 rows of X
                const int j = (warp - 2) >> 1, h = (warp - 2) & 1;
                tma_load_2d_pair(smem + L.b + s * kB + j * 16384 + h * 8192, &p.tm_x, lead_full, col0 + 64 * j,
                                 (int32_t)(kt * 128 + 64 * h));
              }
            } else if (C::kWideE) {  // the 4 KB chunk (128-row block, K block kt): 16 rows of 256 bytes
              tma_load_2d_pair(smem + L.e + s * kE, &p.tm_meta, lead_full, 0,
                               (int32_t)(((int64_t)(row0 / 128) * p.meta_cblocks + kt) * 16));
            } else if (sparse) {  // eight 16-row metadata blocks of column block kt
              tma_load_3d_pair(smem + L.e + s * kE, &p.tm_meta, lead_full, 0, (int32_t)kt, row0 / 16);
            }
            if (++s == kStages) { s = 0; ph ^= 1u; }
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    uint32_t aph = 0;  // bit a: phase of accumulator a
    int acc = 0;
    for (int tile = pair_id; tile < p.num_tiles && ok; tile += npairs) {
      const int tm = p.n_major ? tile / p.tiles_n : tile % p.tiles_m;
      const int tn = p.n_major ? tile % p.tiles_n : tile / p.tiles_m;
      const int64_t n0 = (int64_t)tn * C::kN;
      ok = mbar_wait(&acc_full[acc], (aph >> acc) & 1u, abort_flag, p.status, kWaitNs);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + 256u * (uint32_t)acc + ((uint32_t)(quarter * 32) << 16);
      const uint32_t lead_acc_empty = lead_acc_empty0 + 8u * (uint32_t)acc;
      if (DB && !p.out_f32) {
        // Column chunks of 64, 64, 64 and 32 through the warp's staging buffer,
        // one TMA store each (the last through the 32-column map tm_y32).  The
        // accumulator is released after the last TMEM load; the next tile's MMAs
        // run in the other accumulator meanwhile, so this epilogue has a whole
        // tile period to finish.
        static_assert(!DB || C::kN == 224u, "the chunk split below covers 224 columns");
        const int32_t wrow0 = (int32_t)(tm * 256 + 128 * rank + quarter * 32);
        uint8_t* ebuf = smem + L.epi + quarter * (C::kEpiBufs * kEpi);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v0[32], v1[32];
          tmem_ld_32x32b_x32(t_addr + c * 64, v0);
          if (c < 3) tmem_ld_32x32b_x32(t_addr + c * 64 + 32, v1);
          tc_wait_ld();
          if (c == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
          }
          if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read the buffer
          __syncwarp();
          if (c < 3) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              *reinterpret_cast<uint4*>(ebuf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v0[8 * j]), __uint_as_float(v0[8 * j + 1])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 2]), __uint_as_float(v0[8 * j + 3])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 4]), __uint_as_float(v0[8 * j + 5])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 6]), __uint_as_float(v0[8 * j + 7])));
              *reinterpret_cast<uint4*>(ebuf + lane * 128 + (((j + 4) ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v1[8 * j]), __uint_as_float(v1[8 * j + 1])),
                             pack_bf16x2(__uint_as_float(v1[8 * j + 2]), __uint_as_float(v1[8 * j + 3])),
                             pack_bf16x2(__uint_as_float(v1[8 * j + 4]), __uint_as_float(v1[8 * j + 5])),
                             pack_bf16x2(__uint_as_float(v1[8 * j + 6]), __uint_as_float(v1[8 * j + 7])));
            }
          } else {  // 32 columns: 64-byte rows, unswizzled
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(ebuf + lane * 64 + (j << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v0[8 * j]), __uint_as_float(v0[8 * j + 1])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 2]), __uint_as_float(v0[8 * j + 3])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 4]), __uint_as_float(v0[8 * j + 5])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 6]), __uint_as_float(v0[8 * j + 7])));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && n0 + 64 * c < p.T && wrow0 < p.R) {
            tma_store_2d(c < 3 ? &p.tm_y : &p.tm_y32, ebuf, (int32_t)(n0 + 64 * c), wrow0);
            bulk_commit_group();
          }
        }
      } else if (!DB && !p.out_f32) {
        // Whole accumulator row into registers (bf16), release TMEM, then four
        // 64-column chunks through this warp's swizzled staging buffer and a
        // TMA store each: every store writes whole lines, and parts of the box
        // beyond R or T are not written.
        uint32_t pk[128];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_addr + c * 32, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[c * 16 + i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
        const int32_t wrow0 = (int32_t)(tm * 256 + 128 * rank + quarter * 32);
        uint8_t* ebuf = smem + L.epi + quarter * (C::kEpiBufs * kEpi);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read the buffer
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(ebuf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(pk[32 * c + 4 * j], pk[32 * c + 4 * j + 1], pk[32 * c + 4 * j + 2], pk[32 * c + 4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && n0 + 64 * c < p.T && wrow0 < p.R) {
            tma_store_2d(&p.tm_y, ebuf, (int32_t)(n0 + 64 * c), wrow0);
            bulk_commit_group();
          }
        }
      } else {
        // 32-bit results (fp32, or the int32 accumulator bits): 32-column chunks
        // (128-byte rows) through the warp's 128-byte-swizzled staging buffer, one
        // TMA store each (tm_y encodes 4-byte elements, box 32 x 32).  The next
        // chunk's TMEM load is issued before waiting for the previous store to
        // read the buffer; the accumulator is released after the last load.
        const int32_t wrow0 = (int32_t)(tm * 256 + 128 * rank + quarter * 32);
        uint8_t* ebufs = smem + L.epi + quarter * (C::kEpiBufs * kEpi);
        constexpr int kChunks = (int)(C::kN / 32);
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_addr, v);
        tc_wait_ld();
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c) {
          uint8_t* ebuf = ebufs + (c % C::kEpiBufs) * kEpi;
          if (lane == 0) bulk_wait_group_read<C::kEpiBufs - 1>();  // this buffer's last store has read it
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(ebuf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && n0 + 32 * c < p.T && wrow0 < p.R) {
            tma_store_2d(&p.tm_y, ebuf, (int32_t)(n0 + 32 * c), wrow0);
            bulk_commit_group();
          }
          if (c + 1 < kChunks) {
            tmem_ld_32x32b_x32(t_addr + (c + 1) * 32, v);
            tc_wait_ld();
          }
          if (c + 2 == kChunks || kChunks == 1) {  // the last TMEM load is done
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
          }
        }
      }
      aph ^= 1u << acc;
      if (C::kAcc == 2) acc ^= 1;
    }
    if (lane == 0) bulk_wait_group<0>();  // every store of this warp has landed
  }

  // -------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    sleep_about_ns(200000ull);
  }
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

bool pair_kernel_fits(const SpmmParams& p) {
  return p.a_mode == A_TMA_SPARSE && p.K % 128 == 0 && p.K > 0 && p.T >= 192 && p.R >= 1 && p.T % 8 == 0;
}

template <bool HYB, bool DB, bool I8 = false, bool TF32 = false>
static cudaError_t launch_pair(SpmmParams& p, cudaStream_t stream) {
  constexpr pair::Layout L = pair::Cfg<HYB, DB, I8, TF32>::layout();
  const size_t bytes = L.total + 1024;
  static std::atomic<bool> configured[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(spmm_pair_kernel<HYB, DB, I8, TF32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int pairs_avail = sm_count_current() / 2;
  const int pairs = p.num_tiles < pairs_avail ? p.num_tiles : pairs_avail;
  cudaError_t e =
      launch_pdl(spmm_pair_kernel<HYB, DB, I8, TF32>, dim3(2 * pairs), dim3(pair::kThreads), bytes, stream, p);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Tiles of at most kDbMaxStages 128-deep stages take the double-buffered
// form (256 x 224 tiles).  Measured on B200 with 256 x 192 tiles (nm_spmm,
// event-timed loops): ViT 3072 x 768 x 50432 at 1:8 (6 stages) 174 -> 166 us;
// at 24 stages (768 x 3072) 125 -> 143 us, at 32 (4096 x 4096 x 2048) 33 -> 44
// us.  A narrower stage costs about as much as a 256-column one, so the
// double-buffered form pays only where the hidden hand-over is a large part of
// a tile.
constexpr int64_t kDbMaxStages = 8;

cudaError_t launch_spmm_pair(SpmmParams& p, cudaStream_t stream) {
  if (p.k_tiles <= kDbMaxStages) {
    p.tiles_n = (int)((p.T + 223) / 224);
    p.num_tiles = p.tiles_m * p.tiles_n;
    return launch_pair<false, true>(p, stream);
  }
  return launch_pair<false, false>(p, stream);
}

cudaError_t launch_spmm_pair_hybrid(SpmmParams& p, cudaStream_t stream) { return launch_pair<true, false>(p, stream); }

cudaError_t launch_spmm_pair_i8(SpmmParams& p, cudaStream_t stream) { return launch_pair<false, false, true>(p, stream); }

cudaError_t launch_spmm_pair_tf32(SpmmParams& p, cudaStream_t stream) {
  return launch_pair<false, false, false, true>(p, stream);
}

}  // namespace nmk
