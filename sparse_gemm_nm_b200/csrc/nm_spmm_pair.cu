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
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_spmm.h"

namespace nmk {

namespace pair {
constexpr int kThreads = 384;  // warps 0,2-5,10,11 copies; 1 MMA; 6-9 epilogue
constexpr uint32_t kB = 32768, kE = 2048;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kECol = 256;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kIdesc = idesc_bf16(256, true, 256);
constexpr uint32_t kIdescDense = idesc_bf16(256, false, 256);
constexpr uint32_t kEpi = 4096;  // per epilogue warp: 32 rows x 64 bf16 columns, 128-byte swizzle

struct Layout {
  uint32_t a, b, e, epi, bar, total;
};
// HYB = false: 2:4 only, A slots of 16 KB (compressed values), four stages.
// HYB = true (PATCH hybrid): A slots of 32 KB so that a stage can hold the
// dense 128 x 128 tile instead, three stages.
// SHORT (2:4, few stages per tile): three stages, and four 4 KB staging
// buffers per epilogue warp instead of one.  A warp's 32 x 256 bf16 output is
// then written to shared memory while the accumulator drains and leaves as
// four TMA stores issued together; with one buffer each 4 KB chunk waited for
// the previous store to read it, a chain (~4 us) that a long tile hides behind
// its MMAs but a six-stage tile (~2.8 us of MMAs) does not.
template <bool HYB, bool SHORT = false>
struct Cfg {
  static constexpr int kStages = (HYB || SHORT) ? 3 : 4;
  static constexpr int kEpiBufs = SHORT ? 4 : 1;
  static constexpr uint32_t kA = HYB ? 32768u : 16384u;
  static constexpr uint32_t kTxSparse = 2u * (16384u + kB + kE);  // both CTAs' A, B and E bytes
  static constexpr uint32_t kTxDense = 2u * (32768u + kB);        // both CTAs' dense A and B bytes
  __host__ __device__ static constexpr Layout layout() {
    return Layout{0u, kStages * kA, kStages * (kA + kB), kStages * (kA + kB + kE),
                  kStages * (kA + kB + kE) + 4 * kEpiBufs * kEpi,
                  kStages * (kA + kB + kE) + 4 * kEpiBufs * kEpi + (2 * kStages + 4) * 8 + 64};
  }
  static_assert(kStages * (kA + kB + kE) + 4 * kEpiBufs * kEpi + (2 * kStages + 4) * 8 + 64 + 1024 <= 232448,
                "shared memory");
};
}  // namespace pair

// Work of one SM pair.  Data-parallel: whole tiles pair_id, pair_id + npairs,
// ...  Stream-K (p.sk): the num_tiles * k_tiles (tile, 128-deep stage) units in
// tile-major order are cut into npairs contiguous ranges of equal length, so
// every pair gets the same number of stages; a tile whose stages fall in two
// ranges is finished by whichever of its pairs completes last (epilogue).
__device__ __forceinline__ int64_t sk_begin(int64_t units, int npairs, int q) { return units * q / npairs; }

__device__ __forceinline__ int sk_pair_of(int64_t u, int64_t units, int npairs) {
  int q = (int)((u * npairs) / units);
  while (q + 1 < npairs && sk_begin(units, npairs, q + 1) <= u) ++q;
  while (q > 0 && sk_begin(units, npairs, q) > u) --q;
  return q;
}

struct PairWork {
  int64_t u, end, k_tiles;
  int tile, npairs, num_tiles;
  bool sk;
  __device__ PairWork(const SpmmParams& p, int pair_id, int npairs_)
      : k_tiles(p.k_tiles), tile(pair_id), npairs(npairs_), num_tiles(p.num_tiles), sk(p.sk != 0) {
    const int64_t units = (int64_t)p.num_tiles * p.k_tiles;
    u = sk ? sk_begin(units, npairs, pair_id) : 0;
    end = sk ? sk_begin(units, npairs, pair_id + 1) : 0;
  }
  // next (tile, stages [kt0, kt1)) of this pair
  __device__ bool next(int& t, int64_t& kt0, int64_t& kt1) {
    if (!sk) {
      if (tile >= num_tiles) return false;
      t = tile;
      kt0 = 0;
      kt1 = k_tiles;
      tile += npairs;
      return true;
    }
    if (u >= end) return false;
    t = (int)(u / k_tiles);
    kt0 = u - (int64_t)t * k_tiles;
    kt1 = kt0 + (end - u) < k_tiles ? kt0 + (end - u) : k_tiles;
    u += kt1 - kt0;
    return true;
  }
};

// Stream-K partial accumulator of one CTA: 128 rows x 256 fp32 columns, stored
// as [column quad][row] float4s so that a warp's access to one quad of its 32
// rows covers 512 contiguous bytes.  Slot 2q holds the first segment of pair
// q's range, 2q + 1 its last.
__device__ __forceinline__ float4* sk_slot(const SpmmParams& p, int q, bool later, uint32_t rank) {
  return reinterpret_cast<float4*>(p.sk_ws) + ((int64_t)(2 * q + (later ? 1 : 0)) * 2 + rank) * (128 * 64);
}

template <bool HYB, bool SHORT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::kThreads, 1)
    spmm_pair_kernel(const __grid_constant__ SpmmParams p) {
  using namespace pair;
  using C = Cfg<HYB, SHORT>;
  constexpr int kStages = C::kStages;
  constexpr uint32_t kA = C::kA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr Layout L = C::layout();
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* spare = acc_empty + 1;
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
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(spare, 1);
    mbar_init(spare + 1, 4);  // the four epilogue warps (stream-K hand-off)
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

  const uint32_t lead_full0 = map_to_cta(smem_u32(&full[0]), 0);
  const uint32_t lead_acc_empty = map_to_cta(smem_u32(acc_empty), 0);
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
        int s = 0;
        uint32_t ph = 0, aph = 0;
        PairWork work(p, pair_id, npairs);
        int tile;
        int64_t kt0, kt1;
        while (ok && work.next(tile, kt0, kt1)) {
          const int tm = tile % p.tiles_m;
          ok = mbar_wait(acc_empty, aph ^ 1u, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          for (int64_t kt = kt0; kt < kt1; ++kt) {
            ok = mbar_wait(&full[s], ph, abort_flag, p.status, kWaitNs);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + L.a + s * kA);
            const uint32_t b_addr = smem_u32(smem + L.b + s * kB);
            const uint32_t e_tmem = tmem_base + kECol + 4u * s;
            if (tile_sparse(tm, kt, 0) && tile_sparse(tm, kt, 1)) {
              tc_cp_128x128b_pair(e_tmem, smem_desc(smem_u32(smem + L.e + s * kE), 2048, 128, SWZ_NONE));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024, SWZ_128B);
                const uint64_t bd = smem_desc(b_addr + kk * 4096, 16384, 1024, SWZ_128B);
                tc_mma_sp_pair(tmem_base, ad, bd, e_tmem + (uint32_t)(kk & 2), kIdesc | (uint32_t)(kk & 1),
                               (kt > kt0 || kk > 0) ? 1u : 0u);
              }
            } else if (HYB) {  // dense A tile: [K half][128 rows][128 B], eight K = 16 MMAs
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t ad = smem_desc(a_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, SWZ_128B);
                const uint64_t bd = smem_desc(b_addr + kk * 2048, 16384, 1024, SWZ_128B);
                tc_mma_pair(tmem_base, ad, bd, kIdescDense, (kt > kt0 || kk > 0) ? 1u : 0u);
              }
            }
            tc_commit_pair(&empty[s], 0x3);
            if (++s == kStages) { s = 0; ph ^= 1u; }
          }
          if (!ok) break;
          tc_commit_pair(acc_full, 0x3);
          aph ^= 1u;
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
        PairWork work(p, pair_id, npairs);
        int tile;
        int64_t kt0, kt1;
        while (ok && work.next(tile, kt0, kt1)) {
          const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
          const int32_t row0 = tm * 256 + 128 * (int)rank;
          const int32_t col0 = tn * 256 + 128 * (int)rank;
          for (int64_t kt = kt0; kt < kt1; ++kt) {
            ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitNs);
            if (!ok) break;
            const uint32_t lead_full = lead_full0 + 8u * s;
            const bool sparse = tile_sparse(tm, kt, 0) && tile_sparse(tm, kt, 1);
            if (warp == 0 || warp == 10) {
              const int h = warp == 10;
              if (rank == 0 && h == 0) mbar_arrive_expect_tx(&full[s], sparse ? C::kTxSparse : C::kTxDense);
              if (sparse) {
                tma_load_2d_pair(smem + L.a + s * kA + h * 8192, &p.tm_vals, lead_full, (int32_t)(kt * 64),
                                 row0 + 64 * h);
              } else if (HYB) {  // this CTA's dense tile: W, or W under the 2:4 mask if the tile is 2:4
                const CUtensorMap* src = tile_sparse(tm, kt, (int)rank) ? &p.tm_wm : &p.tm_w;
#pragma unroll
                for (int kh = 0; kh < 2; ++kh)
                  tma_load_2d_pair(smem + L.a + s * kA + kh * 16384 + h * 8192, src, lead_full,
                                   (int32_t)(kt * 128 + 64 * kh), row0 + 64 * h);
              }
            } else if (warp <= 5) {  // box (strip j, K half h): 64 columns x 64 rows of X
              const int j = (warp - 2) >> 1, h = (warp - 2) & 1;
              tma_load_2d_pair(smem + L.b + s * kB + j * 16384 + h * 8192, &p.tm_x, lead_full, col0 + 64 * j,
                               (int32_t)(kt * 128 + 64 * h));
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
    uint32_t aph = 0, ephase = 0;
    uint64_t* epi_bar = spare + 1;
    volatile uint32_t* sk_flag = reinterpret_cast<volatile uint32_t*>(tmem_slot + 2);
    const int64_t units = (int64_t)p.num_tiles * p.k_tiles;
    const int64_t my_beg = p.sk ? sk_begin(units, npairs, pair_id) : 0;
    // all four epilogue warps meet (bounded wait; orders the shared flag and, with the
    // fences before it, this CTA's workspace stores)
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_bar);
      const bool r = mbar_wait(epi_bar, ephase, abort_flag, p.status, kWaitNs);
      ephase ^= 1u;
      return r;
    };
    PairWork work(p, pair_id, npairs);
    int tile;
    int64_t kt0, kt1;
    while (ok && work.next(tile, kt0, kt1)) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const int64_t row = (int64_t)tm * 256 + 128 * rank + quarter * 32 + lane;
      const int64_t n0 = (int64_t)tn * 256;
      ok = mbar_wait(acc_full, aph, abort_flag, p.status, kWaitNs);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
      const bool row_ok = row < p.R;
      if (kt0 == 0 && kt1 == p.k_tiles) {
        if (C::kEpiBufs == 4 && !p.out_f32) {
          // 64-column chunk c of the warp's 32 rows: two TMEM loads, bf16 pairs
          // into staging buffer c (128-byte swizzled rows); TMEM released after
          // the last load, then the four stores leave together.
          const int32_t wrow0 = (int32_t)(tm * 256 + 128 * rank + quarter * 32);
          uint8_t* ebuf = smem + L.epi + quarter * (C::kEpiBufs * kEpi);
          if (lane == 0) bulk_wait_group_read<0>();  // the previous tile's stores have read the buffers
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t v0[32], v1[32];
            tmem_ld_32x32b_x32(t_addr + c * 64, v0);
            tmem_ld_32x32b_x32(t_addr + c * 64 + 32, v1);
            tc_wait_ld();
            uint8_t* buf = ebuf + c * kEpi;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v0[8 * j]), __uint_as_float(v0[8 * j + 1])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 2]), __uint_as_float(v0[8 * j + 3])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 4]), __uint_as_float(v0[8 * j + 5])),
                             pack_bf16x2(__uint_as_float(v0[8 * j + 6]), __uint_as_float(v0[8 * j + 7])));
              *reinterpret_cast<uint4*>(buf + lane * 128 + (((j + 4) ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(__uint_as_float(v1[8 * j]), __uint_as_float(v1[8 * j + 1])),
                             pack_bf16x2(__uint_as_float(v1[8 * j + 2]), __uint_as_float(v1[8 * j + 3])),
                             pack_bf16x2(__uint_as_float(v1[8 * j + 4]), __uint_as_float(v1[8 * j + 5])),
                             pack_bf16x2(__uint_as_float(v1[8 * j + 6]), __uint_as_float(v1[8 * j + 7])));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && wrow0 < p.R) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              if (n0 + 64 * c < p.T) tma_store_2d(&p.tm_y, ebuf + c * kEpi, (int32_t)(n0 + 64 * c), wrow0);
            bulk_commit_group();
          }
        } else if (C::kEpiBufs == 1 && !p.out_f32) {
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
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_addr + c * 16, v);
            tc_wait_ld();
            if (!row_ok) continue;
            const int64_t col0 = n0 + c * 16;
            if (p.out_f32) {
              float* yrow = static_cast<float*>(p.Y) + row * p.ldy;
#pragma unroll
              for (int e = 0; e < 16; ++e)
                if (col0 + e < p.T) yrow[col0 + e] = __uint_as_float(v[e]);
            } else {
              uint16_t* yrow = static_cast<uint16_t*>(p.Y) + row * p.ldy;
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                const uint32_t pk = pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                if (col0 + e < p.T) yrow[col0 + e] = (uint16_t)(pk & 0xFFFFu);
                if (col0 + e + 1 < p.T) yrow[col0 + e + 1] = (uint16_t)(pk >> 16);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
        }
      } else {
        // Stream-K segment of a split tile.  If the tile's other segments are
        // already in the workspace, this CTA adds them to its accumulator as it
        // drains TMEM and stores the tile.  Otherwise its partial goes to its
        // workspace slot, and the last segment to arrive adds all partials in
        // range order.  Either way the sum runs over the segments in range
        // order, so the result does not depend on which pair finishes last.
        const int rr = quarter * 32 + lane;  // row within this CTA's 128
        const int64_t tu0 = (int64_t)tile * p.k_tiles;
        const int q0 = sk_pair_of(tu0, units, npairs);
        const int q1 = sk_pair_of(tu0 + p.k_tiles - 1, units, npairs);
        const bool q0_later = tu0 > sk_begin(units, npairs, q0);
        const int32_t wrow0 = (int32_t)(tm * 256 + 128 * rank + quarter * 32);
        uint8_t* ebuf = smem + L.epi + quarter * (C::kEpiBufs * kEpi);
        uint32_t* cnt = p.sk_cnt + 2 * tile + (int)rank;
        // Only a tile's first segment, which ends its pair's range, checks first:
        // the other segment starts a later range and is usually long finished.
        if (kt0 == 0) {
          if (warp == 6 && lane == 0) {
            *sk_flag = atomicAdd(cnt, 0u);
            __threadfence();
          }
          ok = epi_sync();
          if (!ok) break;
        }
        // 64-column chunk c of this warp's rows to the output (staging + TMA store, or fp32 rows)
        auto emit = [&](int c, const float* a) {
          if (!p.out_f32) {
            uint8_t* buf = ebuf + (C::kEpiBufs == 4 ? c * kEpi : 0);
            if (C::kEpiBufs == 1 || c == 0) {
              if (lane == 0) bulk_wait_group_read<0>();  // earlier stores have read the buffer(s)
              __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(a[8 * j], a[8 * j + 1]), pack_bf16x2(a[8 * j + 2], a[8 * j + 3]),
                             pack_bf16x2(a[8 * j + 4], a[8 * j + 5]), pack_bf16x2(a[8 * j + 6], a[8 * j + 7]));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && n0 + 64 * c < p.T && wrow0 < p.R) {
              tma_store_2d(&p.tm_y, buf, (int32_t)(n0 + 64 * c), wrow0);
              bulk_commit_group();
            }
          } else if (row_ok) {
            float* yrow = static_cast<float*>(p.Y) + row * p.ldy;
#pragma unroll
            for (int j = 0; j < 64; ++j)
              if (n0 + 64 * c + j < p.T) yrow[n0 + 64 * c + j] = a[j];
          }
        };
        if (kt0 == 0 && *sk_flag == (uint32_t)(q1 - q0)) {
          // every other segment is in the workspace (nseg <= 2 here: the host
          // enables stream-K only with at least one tile per pair)
          const int qo = pair_id == q0 ? q1 : q0;
          const float4* other = sk_slot(p, qo, qo == q0 && q0_later, rank);
          __threadfence();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t v[64];
            tmem_ld_32x32b_x32(t_addr + c * 64, *reinterpret_cast<uint32_t(*)[32]>(v));
            tmem_ld_32x32b_x32(t_addr + c * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
            tc_wait_ld();
            float a[64];
#pragma unroll
            for (int g = 0; g < 16; ++g) {
              const float4 o = __ldcg(other + (16 * c + g) * 128 + rr);
              a[4 * g] = __uint_as_float(v[4 * g]) + o.x;
              a[4 * g + 1] = __uint_as_float(v[4 * g + 1]) + o.y;
              a[4 * g + 2] = __uint_as_float(v[4 * g + 2]) + o.z;
              a[4 * g + 3] = __uint_as_float(v[4 * g + 3]) + o.w;
            }
            if (c == 3) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
            }
            emit(c, a);
          }
        } else {
          float4* mine = sk_slot(p, pair_id, tu0 + kt0 > my_beg, rank);
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(t_addr + c * 32, v);
            tc_wait_ld();
#pragma unroll
            for (int g = 0; g < 8; ++g)
              mine[(8 * c + g) * 128 + rr] = make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                                         __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(lead_acc_empty);
          __threadfence();
          ok = epi_sync();
          if (!ok) break;
          if (warp == 6 && lane == 0) *sk_flag = atomicAdd(cnt, 1u);
          ok = epi_sync();
          if (!ok) break;
          if (*sk_flag == (uint32_t)(q1 - q0)) {
            __threadfence();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float a[64];
#pragma unroll
              for (int j = 0; j < 64; ++j) a[j] = 0.0f;
              for (int q = q0; q <= q1; ++q) {
                const float4* src = sk_slot(p, q, q == q0 && q0_later, rank);
#pragma unroll
                for (int g = 0; g < 16; ++g) {
                  const float4 o = __ldcg(src + (16 * c + g) * 128 + rr);
                  a[4 * g] += o.x;
                  a[4 * g + 1] += o.y;
                  a[4 * g + 2] += o.z;
                  a[4 * g + 3] += o.w;
                }
              }
              emit(c, a);
            }
          }
        }
      }
      aph ^= 1u;
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

template <bool HYB, bool SHORT>
static cudaError_t launch_pair(SpmmParams& p, cudaStream_t stream) {
  constexpr pair::Layout L = pair::Cfg<HYB, SHORT>::layout();
  const size_t bytes = L.total + 1024;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(spmm_pair_kernel<HYB, SHORT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int pairs_avail = sm_count_current() / 2;
  const int pairs = p.num_tiles < pairs_avail ? p.num_tiles : pairs_avail;
  cudaError_t e = launch_pdl(spmm_pair_kernel<HYB, SHORT>, dim3(2 * pairs), dim3(pair::kThreads), bytes, stream, p);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Tiles of at most eight 128-deep stages take the short-tile configuration
// (three stages, four staging buffers per epilogue warp).
cudaError_t launch_spmm_pair(SpmmParams& p, cudaStream_t stream) {
  return p.k_tiles <= 8 ? launch_pair<false, true>(p, stream) : launch_pair<false, false>(p, stream);
}

cudaError_t launch_spmm_pair_hybrid(SpmmParams& p, cudaStream_t stream) { return launch_pair<true, false>(p, stream); }

}  // namespace nmk
