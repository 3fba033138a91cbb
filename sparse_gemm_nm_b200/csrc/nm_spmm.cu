// nm_spmm.cu -- sparse x dense GEMM on the sm_100a tensor cores.
//
// Y (R x T) = W' (R x K, N:M along K) * X (K x T), optionally with the input
// rows permuted through an index map, optionally with per-tile dense / 2:4
// weights.  Sources: "M:N sparsity on NVIDIA tensor cores" (GEMM paragraphs
// of "Where this sits among the three case studies": only the weights are
// compressed, their positions select the rows of the dense operand);
// "Technische Samenvatting: SHUFFLESPARSE", "2. Methodologie" (y = (W Pi) x,
// the kernel reads its input at the permuted addresses); "Structured
// Sparsity" topic cards, PATCH abstract (tiles either dense or 2:4).
//
// One persistent CTA per SM walks output tiles of 128 x BN.  Warp roles:
//   warp 0      TMA producer: compressed A tile (or dense W tile) and, without
//               an index map, the X tile.
//   warp 1      TMEM owner and MMA issuer (one thread): per stage it copies
//               the metadata tile into TMEM (tcgen05.cp) and issues
//               tcgen05.mma.sp (2:4) or tcgen05.mma (dense) into the fp32
//               accumulator in TMEM.
//   warps 2-5   builders, one thread per tile row: re-lay the row-wise
//               metadata into the tensor-core metadata order, or build the A
//               tile in shared memory from the compressed operand (1:4 / 1:8
//               re-encoded as 2:4, or any N:M expanded to a dense tile).  With
//               an index map they also gather the X rows X[idx[k]] with
//               coalesced 16-byte cp.async straight into the swizzled B tile.
//   warps 6-9   epilogue: TMEM -> registers -> bf16/fp32 -> global.
// Stages of the shared-memory ring are handed over with mbarriers; every wait
// is bounded in time and reports through a device status word.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_spmm.h"

namespace nmk {

__device__ uint32_t g_status;  // bit 0: a bounded wait gave up

constexpr int kThreads = 320;
constexpr int kBuilderWarp0 = 2;
constexpr int kEpilogueWarp0 = 6;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kEColBase = 256;     // TMEM columns of the metadata ring
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct SmemLayout {
  uint32_t a_off, b_off, e_off, bar_off, total;
};

__host__ __device__ inline SmemLayout smem_layout(int stages, uint32_t a_slot, uint32_t b_slot) {
  SmemLayout L;
  L.a_off = 0;
  L.b_off = L.a_off + stages * a_slot;
  L.e_off = L.b_off + stages * b_slot;
  L.bar_off = L.e_off + stages * 2048u;
  // full[stages], empty[stages], acc_full[2], acc_empty[2], misc words
  L.total = L.bar_off + (2 * stages + 4) * 8 + 64;
  return L;
}

// ----------------------------------------------------------------------------
// Builders: metadata re-layout.  The tensor core reads 2:4 metadata for a
// 128-row x 32-K MMA from one TMEM column: lane (r%8) + 8*h + 16*(r/16) holds,
// in bits 16*((r/8)%2) .. +15, the sixteen position bits of row r for K half h
// (nibble per group of four, first position in the low bits).  The shared tile
// handed to tcgen05.cp is 128 lanes x 16 bytes, row = lane.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void put_e_word(uint8_t* e_slot, int r, int kk, uint32_t w) {
  const int lane_lo = (r & 7) | (r & ~15);
  const int half = (r >> 3) & 1;
  uint16_t* lo = reinterpret_cast<uint16_t*>(e_slot + lane_lo * 16 + kk * 4 + half * 2);
  uint16_t* hi = reinterpret_cast<uint16_t*>(e_slot + (lane_lo + 8) * 16 + kk * 4 + half * 2);
  *lo = static_cast<uint16_t>(w & 0xFFFFu);
  *hi = static_cast<uint16_t>(w >> 16);
}

// Position of survivor j of a row (row-wise packing: b-bit fields, S per word).
__device__ __forceinline__ uint32_t pos_of(const uint32_t* mrow, int64_t j, int b, int s) {
  const uint32_t w = __ldg(mrow + j / s);
  return (w >> (b * (int)(j % s))) & ((1u << b) - 1u);
}

// 2:4 nibble (p0 | p1 << 2) of group g of row `row` in the tiled packing.
__device__ __forceinline__ uint32_t nibble_2of4(const SpmmParams& p, int64_t row, int64_t g) {
  const int64_t blk = (row >> 4) * p.meta_cblocks + (g >> 5);
  const int l = (int)(row & 7) + 8 * (int)((g >> 2) & 1);
  const int q = (int)((g >> 3) & 3);
  const int bit = 16 * (int)((row >> 3) & 1) + 4 * (int)(g & 3);
  return (__ldg(p.meta + blk * 64 + 4 * l + q) >> bit) & 0xFu;
}

// One 2:4 group from a single survivor at in-group position q (0..3) value v.
__device__ __forceinline__ void one_in_four(uint32_t q, uint32_t v, uint32_t& nib, uint32_t& pk) {
  nib = q == 0 ? 0x4u : (q << 2);             // (0,1) or (0,q)
  pk = q == 0 ? v : (v << 16);                // value sits at the slot of position q
}

// Re-encode one row of stage kt (64 logical K) as 2:4: 16 groups -> 16 packed
// value words (two bf16 each) and two metadata words.
template <int N, int M>
__device__ __forceinline__ void reencode_row(const SpmmParams& p, int64_t row, int64_t kt, uint32_t (&vals)[16],
                                             uint32_t& w0, uint32_t& w1) {
  w0 = w1 = 0x44444444u;
#pragma unroll
  for (int i = 0; i < 16; ++i) vals[i] = 0;
  if (row >= p.R) return;
  const int64_t k0 = kt * 64;
  const uint16_t* vrow = p.vals + row * p.vcols;
  const uint32_t* mrow = p.meta + row * p.mcols;  // row-wise patterns only
  constexpr int B = M == 2 ? 1 : M == 4 ? 2 : 3;
  constexpr int S = 32 / B;
  uint32_t nibs[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) nibs[q] = 0x4u;
  if (N == 2 && M == 4) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int64_t g = k0 / 4 + q;
      if (g * 4 < p.K) {
        vals[q] = (uint32_t)vrow[2 * g] | ((uint32_t)vrow[2 * g + 1] << 16);
        nibs[q] = nibble_2of4(p, row, g);
      }
    }
  } else if (N == 1 && M == 2) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int64_t g = k0 / 2 + 2 * q;  // first 1:2 group of this block of four
      if (g * 2 < p.K) {
        const bool second = (g + 1) * 2 < p.K;  // K % 4 == 2 leaves half a block
        const uint32_t pa = pos_of(mrow, g, B, S), pb = second ? pos_of(mrow, g + 1, B, S) : 0u;
        vals[q] = (uint32_t)vrow[g] | (second ? ((uint32_t)vrow[g + 1] << 16) : 0u);
        nibs[q] = pa | ((2u + pb) << 2);
      }
    }
  } else if (N == 1 && M == 4) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int64_t g = k0 / 4 + q;
      if (g * 4 < p.K) one_in_four(pos_of(mrow, g, B, S), vrow[g], nibs[q], vals[q]);
    }
  } else if (M == 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // 1:8 or 2:8 group i -> 2:4 groups 2i, 2i+1
      const int64_t g = k0 / 8 + i;
      if (g * 8 >= p.K) continue;
      if (N == 1) {
        const uint32_t q = pos_of(mrow, g, B, S);
        const uint32_t v = vrow[g];
        uint32_t nb, pk;
        one_in_four(q & 3u, v, nb, pk);
        if (q < 4) { nibs[2 * i] = nb; vals[2 * i] = pk; }
        else { nibs[2 * i + 1] = nb; vals[2 * i + 1] = pk; }
      } else {
        const uint32_t qa = pos_of(mrow, 2 * g, B, S), qb = pos_of(mrow, 2 * g + 1, B, S);
        const uint32_t va = vrow[2 * g], vb = vrow[2 * g + 1];
        if (qb < 4) {  // both in the low half
          nibs[2 * i] = qa | (qb << 2);
          vals[2 * i] = va | (vb << 16);
        } else if (qa >= 4) {  // both in the high half
          nibs[2 * i + 1] = (qa - 4) | ((qb - 4) << 2);
          vals[2 * i + 1] = va | (vb << 16);
        } else {
          one_in_four(qa, va, nibs[2 * i], vals[2 * i]);
          one_in_four(qb - 4, vb, nibs[2 * i + 1], vals[2 * i + 1]);
        }
      }
    }
  }
  w0 = w1 = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    w0 |= nibs[q] << (4 * q);
    w1 |= nibs[q + 8] << (4 * q);
  }
}

// Write one 64-byte row of a K-major SWIZZLE_64B tile (8-row atoms of 512 B).
__device__ __forceinline__ void store_row_sw64(uint8_t* tile, int r, const uint32_t (&v)[16]) {
  uint8_t* base = tile + r * 64;
  const int x = (r >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(base + ((c ^ x) << 4)) =
        make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// Dense expansion of one row of stage kt into a K-major SWIZZLE_128B tile
// (128-byte rows, 8-row atoms of 1 KB): zeros, then each survivor at its K.
__device__ __forceinline__ void expand_row_sw128(const SpmmParams& p, uint8_t* tile, int r, int64_t row,
                                                 int64_t kt) {
  uint8_t* base = tile + r * 128;
  const int x = r & 7;
#pragma unroll
  for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(base + (c << 4)) = make_uint4(0, 0, 0, 0);
  if (row >= p.R) return;
  const int n = p.n, m = p.m;
  const int b = m == 2 ? 1 : m == 4 ? 2 : m == 8 ? 3 : 4;
  const int s = 32 / b;
  const int64_t k0 = kt * 64;
  const int64_t g0 = k0 / m;
  int64_t g1 = (k0 + 64) / m;
  if (g1 * m > p.K) g1 = p.K / m;
  const uint16_t* vrow = p.vals + row * p.vcols;
  const uint32_t* mrow = p.meta + row * p.mcols;
  const bool tiled = n == 2 && m == 4;
  for (int64_t j = g0 * n; j < g1 * n; ++j) {
    const int64_t g = j / n;
    const uint32_t pos = tiled ? (nibble_2of4(p, row, g) >> (2 * (j & 1))) & 3u : pos_of(mrow, j, b, s);
    const int kr = (int)(g * m + pos - k0);  // 0..63
    const int c = kr >> 3;
    *reinterpret_cast<uint16_t*>(base + (((c ^ x) << 4) | ((kr & 7) << 1))) = vrow[j];
  }
}

// ----------------------------------------------------------------------------
// The kernel
// ----------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(kThreads, 1) spmm_kernel(const __grid_constant__ SpmmParams p) {
  constexpr int NUM_ACC = (BN <= 128) ? 2 : 1;
  constexpr int BSW = BN >= 64 ? 128 : BN * 2;          // bytes per swizzled B row
  constexpr int STRIP_COLS = BSW / 2;                    // columns per B strip
  constexpr int N_STRIPS = BN / STRIP_COLS;
  constexpr uint32_t STRIP_BYTES = 64u * BSW;            // 64 K-rows per stage
  constexpr uint32_t B_BYTES = 64u * BN * 2u;
  constexpr uint32_t B_SWZ = BSW == 128 ? SWZ_128B : BSW == 64 ? SWZ_64B : SWZ_32B;
  constexpr uint32_t IDESC_SP = idesc_bf16(BN, true);
  constexpr uint32_t IDESC_DN = idesc_bf16(BN, false);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  const SmemLayout L = smem_layout(stages, p.a_slot_bytes, B_BYTES);
  uint8_t* a_base = smem + L.a_off;
  uint8_t* b_base = smem + L.b_off;
  uint8_t* e_base = smem + L.e_off;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* empty = full + stages;
  uint64_t* acc_full = empty + stages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* spare_bar = reinterpret_cast<uint64_t*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1 + 4 + (p.permuted ? 128 : 0));
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(spare_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_x);
    if (p.a_mode == A_TMA_SPARSE || p.a_mode == A_HYBRID) tma_prefetch_desc(&p.tm_vals);
    if (p.a_mode == A_HYBRID) tma_prefetch_desc(&p.tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_gate();  // no global memory touched before this point

  const int64_t k_tiles = p.k_tiles;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int s = 0;
    uint32_t ph = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const int m0 = tm * 128, n0 = tn * BN;
      for (int64_t kt = 0; kt < k_tiles; ++kt) {
        ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitLimitNs);
        if (!ok) break;
        int a_kind = 0;  // 0 none, 1 compressed via TMA, 2 dense W via TMA
        if (p.a_mode == A_TMA_SPARSE) a_kind = 1;
        else if (p.a_mode == A_HYBRID) a_kind = __ldg(p.tile_map + (int64_t)tm * p.hyb_tiles_k + kt / 2) ? 1 : 2;
        const uint32_t a_bytes = a_kind == 1 ? 128u * 64u : a_kind == 2 ? 128u * 128u : 0u;
        uint8_t* a_dst = a_base + s * p.a_slot_bytes;
        uint8_t* b_dst = b_base + s * B_BYTES;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], a_bytes + (p.permuted ? 0u : B_BYTES));
          if (a_kind == 1) tma_load_2d(a_dst, &p.tm_vals, &full[s], (int32_t)(kt * 32), m0);
          else if (a_kind == 2) tma_load_2d(a_dst, &p.tm_w, &full[s], (int32_t)(kt * 64), m0);
        }
        __syncwarp();
        if (!p.permuted && lane < N_STRIPS)
          tma_load_2d(b_dst + lane * STRIP_BYTES, &p.tm_x, &full[s], n0 + lane * STRIP_COLS, (int32_t)(kt * 64));
        if (++s == stages) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int tm = tile % p.tiles_m;
        ok = mbar_wait(&acc_empty[acc], aph ^ 1u, abort_flag, p.status, kWaitLimitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int64_t kt = 0; kt < k_tiles; ++kt) {
          ok = mbar_wait(&full[s], ph, abort_flag, p.status, kWaitLimitNs);
          if (!ok) break;
          tc_fence_after();
          bool sparse = p.a_mode != A_BUILD_DENSE;
          if (p.a_mode == A_HYBRID) sparse = __ldg(p.tile_map + (int64_t)tm * p.hyb_tiles_k + kt / 2) != 0;
          const uint32_t a_addr = smem_u32(a_base + s * p.a_slot_bytes);
          const uint32_t b_addr = smem_u32(b_base + s * B_BYTES);
          if (sparse) {
            const uint32_t e_tmem = tmem_base + kEColBase + 4u * s;
            tc_cp_128x128b(e_tmem, smem_desc(smem_u32(e_base + s * 2048), 2048, 128, SWZ_NONE));
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 512, SWZ_64B);
              const uint64_t bd = smem_desc(b_addr + kk * 32 * BSW, STRIP_BYTES, 8 * BSW, B_SWZ);
              // The metadata operand address stays column-pair aligned; the
              // descriptor's sparsity selector picks the column within the pair.
              tc_mma_sp(d_tmem, ad, bd, e_tmem, IDESC_SP | (uint32_t)kk, (kt > 0 || kk > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024, SWZ_128B);
              const uint64_t bd = smem_desc(b_addr + kk * 16 * BSW, STRIP_BYTES, 8 * BSW, B_SWZ);
              tc_mma(d_tmem, ad, bd, IDESC_DN, (kt > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(&empty[s]);
          if (++s == stages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == NUM_ACC) { acc = 0; aph ^= 1u; }
      }
      if (!ok) {  // let issued tensor-core work drain before TMEM is released
        tc_commit(spare_bar);
        volatile int dummy = 0;
        mbar_wait(spare_bar, 0, &dummy, p.status, 100000000ull);
      }
    }
  } else if (warp < kEpilogueWarp0) {
    // ------------------------------------------------------------ builders
    const int r = threadIdx.x - 32 * kBuilderWarp0;  // tile row 0..127
    const int bw = r >> 5;                           // builder warp 0..3
    const bool e_from_meta = p.a_mode == A_TMA_SPARSE || p.a_mode == A_HYBRID;
    // The stages of this CTA in order: tile blockIdx.x + j*gridDim.x, kt.
    const int64_t my_tiles = (p.num_tiles - 1 - blockIdx.x) / gridDim.x + 1;
    const int64_t total = my_tiles * k_tiles;
    // Prefetch ring, PF stages ahead: this row's two 2:4 metadata words, and
    // (permuted) the source row of X for K-row 16*bw + lane of the stage.
    constexpr int PF = 6;
    uint2 mq[PF];
    int32_t iq[PF];
    // prefetch cursor (stage it + PF) advanced incrementally, no divisions
    int f_tile = blockIdx.x;
    int64_t f_kt = 0, f_it = 0;
    auto fetch = [&](uint2& mw, int32_t& ix) {
      mw = make_uint2(0x44444444u, 0x44444444u);
      ix = -1;
      if (f_it < total) {
        if (e_from_meta) {
          // TMEM lane r of the tile is lane r%16 of row block (m0 + r)/16 in the
          // tiled 2:4 metadata; this stage's 64 columns are words q = 2*(kt%2), +1.
          const int64_t rb = (int64_t)(f_tile % p.tiles_m) * 8 + (r >> 4);
          if (rb < p.meta_rblocks) {
            const uint32_t* blk = p.meta + (rb * p.meta_cblocks + (f_kt >> 1)) * 64;
            mw = __ldg(reinterpret_cast<const uint2*>(blk + 4 * (r & 15) + 2 * (f_kt & 1)));
          }
        }
        if (p.permuted && lane < 16) {
          const int64_t k = f_kt * 64 + bw * 16 + lane;
          if (k < p.K) ix = __ldg(p.idx + k);
        }
      }
      ++f_it;
      if (++f_kt == k_tiles) { f_kt = 0; f_tile += gridDim.x; }
    };
#pragma unroll
    for (int j = 0; j < PF; ++j) fetch(mq[j], iq[j]);
    int s = 0;
    uint32_t ph = 0;
    int tile = blockIdx.x;
    int64_t kt = 0;
    for (int64_t it = 0; it < total; ++it) {
      const uint2 mw = mq[0];
      const int32_t ix = iq[0];
#pragma unroll
      for (int j = 0; j < PF - 1; ++j) {
        mq[j] = mq[j + 1];
        iq[j] = iq[j + 1];
      }
      fetch(mq[PF - 1], iq[PF - 1]);
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const int64_t row = (int64_t)tm * 128 + r;
      ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitLimitNs);
      if (!ok) break;
      uint8_t* a_dst = a_base + s * p.a_slot_bytes;
      uint8_t* e_dst = e_base + s * 2048;
      if (p.a_mode == A_TMA_SPARSE) {
        *reinterpret_cast<uint2*>(e_dst + r * 16) = mw;
      } else if (p.a_mode == A_HYBRID) {
        if (__ldg(p.tile_map + (int64_t)tm * p.hyb_tiles_k + kt / 2)) *reinterpret_cast<uint2*>(e_dst + r * 16) = mw;
      } else if (p.a_mode == A_BUILD_SPARSE) {
        uint32_t vals[16], w0, w1;
        switch (p.pattern) {
          case PAT_2_4: reencode_row<2, 4>(p, row, kt, vals, w0, w1); break;
          case PAT_1_2: reencode_row<1, 2>(p, row, kt, vals, w0, w1); break;
          case PAT_1_4: reencode_row<1, 4>(p, row, kt, vals, w0, w1); break;
          case PAT_1_8: reencode_row<1, 8>(p, row, kt, vals, w0, w1); break;
          default: reencode_row<2, 8>(p, row, kt, vals, w0, w1); break;
        }
        store_row_sw64(a_dst, r, vals);
        put_e_word(e_dst, r, 0, w0);
        put_e_word(e_dst, r, 1, w1);
      } else {  // A_BUILD_DENSE
        expand_row_sw128(p, a_dst, r, row, kt);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
      if (p.permuted) {
        // Gather K-rows 16*bw .. 16*bw+15 of the stage: row k of the tile is
        // X[idx[k]][n0 .. n0+BN), 16 bytes per lane, written at its swizzled
        // place in the MN-major B tile.
        constexpr int LPR = BN / 8;       // lanes per row segment
        constexpr int RPI = 32 / LPR;     // rows per warp instruction
        uint8_t* b_dst = b_base + s * B_BYTES;
        const int chunk = lane % LPR;
        const int64_t col = (int64_t)tn * BN + chunk * 8;
        const uint32_t cbytes = col >= p.T ? 0u : (col + 8 <= p.T ? 16u : (uint32_t)(p.T - col) * 2u);
        const int strip = (chunk * 8) / STRIP_COLS;
        const int cis = ((chunk * 8) % STRIP_COLS) / 8;  // 16-byte chunk inside the strip row
#pragma unroll
        for (int q = 0; q < 16 / RPI; ++q) {
          const int i = q * RPI + lane / LPR;   // 0..15
          const int32_t src = __shfl_sync(0xffffffffu, ix, i);
          const int kr = bw * 16 + i;           // K-row inside the stage
          const bool valid = src >= 0 && (int64_t)src < p.K;
          const uint32_t nbytes = valid ? cbytes : 0u;
          const uint16_t* g = nbytes ? p.X + (int64_t)src * p.ldx + col : p.X;
          const int sw = cis ^ ((kr * BSW >> 7) & (BSW / 16 - 1));
          cp_async_16(b_dst + strip * STRIP_BYTES + kr * BSW + (sw << 4), g, nbytes);
        }
        cp_async_arrive_noinc(&full[s]);
      }
      if (++s == stages) { s = 0; ph ^= 1u; }
      if (++kt == k_tiles) { kt = 0; tile += gridDim.x; }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    int acc = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const int64_t row = (int64_t)tm * 128 + quarter * 32 + lane;
      const int64_t n0 = (int64_t)tn * BN;
      ok = mbar_wait(&acc_full[acc], aph, abort_flag, p.status, kWaitLimitNs);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      const bool row_ok = row < p.R;
      if (!p.out_f32 && NUM_ACC == 1 && n0 + BN <= p.T) {
        // Drain the whole accumulator into registers (bf16 pairs), release it
        // to the MMA warp, then write out while the next tile accumulates.
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_addr + c * 32, v);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[c * 16 + i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        if (row_ok) {
          uint4* yrow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.Y) + row * p.ldy + n0);
#pragma unroll
          for (int c8 = 0; c8 < BN / 8; ++c8)
            yrow[c8] = make_uint4(pk[4 * c8], pk[4 * c8 + 1], pk[4 * c8 + 2], pk[4 * c8 + 3]);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(t_addr + c * 16, v);
          tc_wait_ld();
          if (!row_ok) continue;
          const int64_t col0 = n0 + c * 16;
          if (p.out_f32) {
            float* yrow = static_cast<float*>(p.Y) + row * p.ldy;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int64_t col = col0 + 4 * q;
              if (col + 4 <= p.T) {
                *reinterpret_cast<uint4*>(yrow + col) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (col + e < p.T) yrow[col + e] = __uint_as_float(v[4 * q + e]);
              }
            }
          } else {
            uint16_t* yrow = static_cast<uint16_t*>(p.Y) + row * p.ldy;
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int64_t col = col0 + 8 * h;
              if (col + 8 <= p.T) {
                *reinterpret_cast<uint4*>(yrow + col) = make_uint4(pk[4 * h], pk[4 * h + 1], pk[4 * h + 2], pk[4 * h + 3]);
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  if (col + e < p.T) yrow[col + e] = (uint16_t)(pk[4 * h + e / 2] >> (16 * (e & 1)));
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
      if (++acc == NUM_ACC) { acc = 0; aph ^= 1u; }
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // give TMA copies that were already issued time to land (bounded)
    sleep_about_ns(200000ull);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------------------
// Host launcher
// ----------------------------------------------------------------------------
template <int BN>
static cudaError_t launch_bn(const SpmmParams& p, int grid, cudaStream_t stream) {
  const SmemLayout L = smem_layout(p.stages, p.a_slot_bytes, 64u * BN * 2u);
  const size_t bytes = L.total + 1024;
  static std::atomic<bool> configured[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(spmm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         232448);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  cudaError_t e = launch_pdl(spmm_kernel<BN>, dim3(grid), dim3(kThreads), bytes, stream, p);
  return e != cudaSuccess ? e : cudaGetLastError();
}

int spmm_max_stages(int bn, uint32_t a_slot) {
  const uint32_t b = 64u * bn * 2u;
  const uint32_t budget = 232448u - 1024u - 256u;
  int st = 1;
  while (st < 16 && smem_layout(st + 1, a_slot, b).total <= budget) ++st;
  return st;
}

// Device address of the status word on the current device (looked up once per device; devices past the
// cache are looked up on every call).
uint32_t* status_word_ptr() {
  static std::atomic<uint32_t*> status_ptr[64];  // zero-initialised: not looked up yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  const bool cached = dev >= 0 && dev < 64;
  if (cached) {
    uint32_t* p = status_ptr[dev].load(std::memory_order_relaxed);
    if (p) return p;
  }
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) return nullptr;
  if (cached) status_ptr[dev].store(static_cast<uint32_t*>(addr), std::memory_order_relaxed);
  return static_cast<uint32_t*>(addr);
}

cudaError_t launch_spmm(SpmmParams& p, int bn, cudaStream_t stream) {
  const int sms = sm_count_current();
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  cudaError_t e;
  switch (bn) {
    case 16: e = launch_bn<16>(p, grid, stream); break;
    case 32: e = launch_bn<32>(p, grid, stream); break;
    case 64: e = launch_bn<64>(p, grid, stream); break;
    case 128: e = launch_bn<128>(p, grid, stream); break;
    default: e = launch_bn<256>(p, grid, stream); break;
  }
  count_launch();
  return e;
}

// Self-test of the failure path: one thread waits, with the library's bounded
// wait, on a barrier that nothing completes; the wait gives up after limit_ns
// and records the timeout in the status word.  Nothing else is touched.
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t stream) {
  uint32_t* st = status_word_ptr();
  if (!st) return cudaErrorInvalidSymbol;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(st, limit_ns);
  count_launch();
  return cudaGetLastError();
}

cudaError_t read_and_clear_status(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_status, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_status, &zero, sizeof(uint32_t));
}

}  // namespace nmk
