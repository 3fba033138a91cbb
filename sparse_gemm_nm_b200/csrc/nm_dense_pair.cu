// nm_dense_pair.cu -- dense GEMMs on SM pairs: the backward pass of an N:M layer,
// and the forward GEMM of the formats run on a staged dense copy (the diagonal
// pattern in bf16, INT8 2:4 as kind::i8, TF32 1:2 as kind::tf32).
//
// Training keeps the N:M structure of W' through every step ("Structured
// Sparsity" topic cards, RNM-TD3 abstract; the DynaDiag page's abstract asks
// for sparse forward and backward passes).  The forward product y = (W' Pi) x
// runs on the sparse tensor cores because W' is N:M along its reduction axis K.
// The two gradients are not of that form:
//   dX = (W' Pi)^T dY  reduces over R, and W'^T is N:M along its output axis;
//   dV = the survivor entries of dY Xp^T, a product sampled at the survivors.
// The sparse MMA takes sparsity only on A along the reduction axis, so both
// run here as dense MMAs: dX on the decompressed W' (A = W'^T read MN-major
// from the R x K matrix), dV as the full product with only the survivor
// entries stored.
//
// Layout per CTA of the pair (cta_group::2, M = 256 = 2 x 128 rows, N = 256):
// three stages of 128 reduction steps, A 128 rows x 128 (32 KB) and B 128 x
// this CTA's 128 columns (32 KB), each as four TMA boxes of 64 x 64 with the
// 128-byte swizzle.  A K-major stage is [K half][128 rows][128 B]; an MN-major
// stage is [64-wide M (or N) strip][128 reduction rows][128 B].  The leader's
// MMA thread issues eight tcgen05.mma (K = 16) per stage; its commits release
// the stage in both CTAs.  Each CTA drains its own 128 x 256 fp32 accumulator;
// two accumulators (512 TMEM columns) let the next tile's MMAs run meanwhile.
// The int8 and tf32 forms keep the stage bytes (256 and 64 reduction steps),
// with K = 32 and K = 8 per MMA.  The plain store epilogue sends whole
// 128-byte row chunks through a swizzled staging tile and TMA stores; with a
// row map (dX under an index map) rows are stored one per lane.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_spmm.h"

namespace nmk {

namespace dpair {
constexpr int kThreads = 256;  // warp 0 copies, 1 MMA, 4-7 epilogue
constexpr int kStages = 3;
constexpr uint32_t kA = 32768, kB = 32768;
constexpr uint32_t kTx = 2u * (kA + kB);  // both CTAs' bytes of a stage
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators
constexpr uint32_t kRowPad = 33;          // epilogue row buffer: 32 floats + 1 (no bank conflicts)
constexpr uint32_t kEpiBuf = 5120;        // per epilogue warp: the row buffer, or a 4 KB TMA-store tile (1024-aligned)
static_assert(kEpiBuf >= 32 * kRowPad * 4 && kEpiBuf % 1024 == 0, "epilogue buffer");
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kOffBuf = kStages * (kA + kB);
constexpr uint32_t kOffBar = kOffBuf + 4 * kEpiBuf;
constexpr uint32_t kSmemBytes = kOffBar + (2 * kStages + 5) * 8 + 16 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
}  // namespace dpair

// Column of survivor j of weight row r (stored position read from the
// metadata): 2:4 tiled metadata or the row-wise packing of other patterns.
__device__ __forceinline__ int64_t survivor_col(const DenseParams& p, int64_t r, int64_t j) {
  const int64_t g = j / p.n;
  if (p.n == 2 && p.m == 4) {
    const int64_t k = 4 * g, c = k & 127;
    const int64_t word = ((r >> 4) * p.meta_cblocks + (k >> 7)) * 64 + 4 * ((r & 7) + 8 * ((c >> 4) & 1)) + (c >> 5);
    const uint32_t nib = (__ldg(p.meta + word) >> (16 * ((r >> 3) & 1) + 4 * ((c >> 2) & 3))) & 0xFu;
    return k + ((j & 1) ? (nib >> 2) : (nib & 3u));
  }
  const int b = p.m == 2 ? 1 : p.m == 4 ? 2 : p.m == 8 ? 3 : 4;
  const int S = 32 / b;
  const uint32_t w = __ldg(p.meta + r * p.mcols + j / S);
  return g * p.m + ((w >> (b * (int)(j % S))) & ((1u << b) - 1u));
}

// I8: signed int8 operands and int32 accumulation (kind::i8).  A stage then holds 256 reduction steps in
// the same bytes: A K-major as two 128-byte halves, B MN-major as one 128-column strip of 256 rows.
template <bool A_MN, bool B_MN, int EPI, bool I8 = false, bool TF32 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(dpair::kThreads, 1)
    dense_pair_kernel(const __grid_constant__ DenseParams p) {
  using namespace dpair;
  static_assert(!I8 || (!A_MN && B_MN), "int8: K-major A and MN-major B");
  static_assert(!TF32 || (!A_MN && B_MN && !I8), "tf32: K-major A and MN-major B");
  constexpr uint32_t kIdesc = I8     ? idesc_s8_major(256, 256, A_MN, B_MN)
                              : TF32 ? idesc_tf32_major(256, 256, A_MN, B_MN)
                                     : idesc_bf16_major(256, 256, A_MN, B_MN);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* spare = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(spare + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs)
  const int pair_id = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);  // four epilogue warps in each CTA
    }
    mbar_init(spare, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_a);
    tma_prefetch_desc(&p.tm_b);
    if (p.use_alt) tma_prefetch_desc(&p.tm_b_alt);
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
  const uint32_t lead_acc_empty0 = map_to_cta(smem_u32(acc_empty), 0);
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------- copies
    if (lane == 0) {
      const CUtensorMap* tmb =
          (p.use_alt && *reinterpret_cast<const volatile uint32_t*>(p.use_alt)) ? &p.tm_b_alt : &p.tm_b;
      int s = 0;
      uint32_t ph = 0;
      for (int tile = pair_id; tile < p.num_tiles && ok; tile += npairs) {
        const int tm = p.n_major ? tile / p.tiles_n : tile % p.tiles_m;
        const int tn = p.n_major ? tile % p.tiles_n : tile / p.tiles_m;
        const int32_t m0 = tm * 256 + 128 * (int)rank;  // this CTA's 128 rows of C
        const int32_t n0 = tn * 256 + 128 * (int)rank;  // this CTA's 128 columns of B
        for (int64_t kt = 0; kt < p.k_tiles; ++kt) {
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          const uint32_t bar = lead_full0 + 8u * s;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], kTx);
          uint8_t* a = smem + s * (kA + kB);
          uint8_t* b = a + kA;
          if (TF32) {  // A: two 32-step halves x two 64-row halves; B: four 32-column strips of 64 rows (their
                       // tensor map swizzles 128-byte rows in 32-byte units, the layout the MMA reads)
            const int32_t k0 = (int32_t)(kt * 64);
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_2d_pair(a + i * 16384 + h * 8192, &p.tm_a, bar, k0 + 32 * i, m0 + 64 * h);
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d_pair(b + j * 8192, tmb, bar, n0 + 32 * j, k0);
            if (++s == kStages) { s = 0; ph ^= 1u; }
            continue;
          }
          if (I8) {  // A: two 128-step halves x two 64-row halves; B: four 64-row boxes of one 128-column strip
            const int32_t k0 = (int32_t)(kt * 256);
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tma_load_2d_pair(a + i * 16384 + h * 8192, &p.tm_a, bar, k0 + 128 * i, m0 + 64 * h);
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d_pair(b + j * 8192, tmb, bar, n0, k0 + 64 * j);
            if (++s == kStages) { s = 0; ph ^= 1u; }
            continue;
          }
          const int32_t k0 = (int32_t)(kt * 128);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // A: MN-major box (64 M columns at m0 + 64 i, reduction rows k0 + 64 h) or K-major box
              // (reduction columns k0 + 64 i, rows m0 + 64 h); same smem slot either way.
              if (A_MN)
                tma_load_2d_pair(a + i * 16384 + h * 8192, &p.tm_a, bar, m0 + 64 * i, k0 + 64 * h);
              else
                tma_load_2d_pair(a + i * 16384 + h * 8192, &p.tm_a, bar, k0 + 64 * i, m0 + 64 * h);
              if (B_MN)
                tma_load_2d_pair(b + i * 16384 + h * 8192, tmb, bar, n0 + 64 * i, k0 + 64 * h);
              else
                tma_load_2d_pair(b + i * 16384 + h * 8192, tmb, bar, k0 + 64 * i, n0 + 64 * h);
            }
          }
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA (leader)
    if (rank == 0 && lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int i = 0;  // tile counter: accumulator i % 2, its use i / 2
      for (int tile = pair_id; tile < p.num_tiles && ok; tile += npairs, ++i) {
        const int ab = i & 1;
        ok = mbar_wait(&acc_empty[ab], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, p.status, kWaitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + 256u * (uint32_t)ab;
        for (int64_t kt = 0; kt < p.k_tiles; ++kt) {
          ok = mbar_wait(&full[s], ph, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * (kA + kB));
          const uint32_t b_addr = a_addr + kA;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // K = 16 step kk: K-major operands advance 32 B inside a 64-wide half (halves 16 KB
            // apart); MN-major operands advance 16 rows of 128 B (strips 16 KB apart).
            const uint64_t ad = A_MN ? smem_desc(a_addr + kk * 2048, 16384, 1024, SWZ_128B)
                                     : smem_desc(a_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, SWZ_128B);
            // int8 MN-major B: K = 32 step kk advances 32 rows of 128 B.  tf32 (K = 8 steps of 32 B for A):
            // B is MN-major in the 128-byte / 32-byte-unit swizzle (four-row atoms 512 B apart), advances
            // 8 rows of 128 B, and its four 32-column strips are 8 KB apart
            const uint64_t bd = I8     ? smem_desc(b_addr + kk * 4096, 32768, 1024, SWZ_128B)
                                : TF32 ? smem_desc(b_addr + kk * 1024, 8192, 512, SWZ_128B_BASE32B)
                                : B_MN ? smem_desc(b_addr + kk * 2048, 16384, 1024, SWZ_128B)
                                       : smem_desc(b_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, SWZ_128B);
            if (I8)
              tc_mma_pair_i8(d_tmem, ad, bd, kIdesc, (kt > 0 || kk > 0) ? 1u : 0u);
            else if (TF32)
              tc_mma_pair_tf32(d_tmem, ad, bd, kIdesc, (kt > 0 || kk > 0) ? 1u : 0u);
            else
              tc_mma_pair(d_tmem, ad, bd, kIdesc, (kt > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair(&empty[s], 0x3);
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[ab], 0x3);
      }
      if (!ok) {
        tc_commit_pair(spare, 0x1);
        volatile int dummy = 0;
        mbar_wait(spare, 0, &dummy, p.status, 100000000ull);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    float* buf = reinterpret_cast<float*>(smem + kOffBuf + (warp - 4) * kEpiBuf) + lane * kRowPad;
    int i = 0;
    for (int tile = pair_id; tile < p.num_tiles && ok; tile += npairs, ++i) {
      const int ab = i & 1;
      const int tm = p.n_major ? tile / p.tiles_n : tile % p.tiles_m;
      const int tn = p.n_major ? tile % p.tiles_n : tile / p.tiles_m;
      const int64_t row = (int64_t)tm * 256 + 128 * rank + quarter * 32 + lane;
      const int64_t n0 = (int64_t)tn * 256;
      ok = mbar_wait(&acc_full[ab], (uint32_t)(i >> 1) & 1u, abort_flag, p.status, kWaitNs);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + 256u * (uint32_t)ab;
      if (EPI == EPI_STORE && p.tma_store) {
        // Whole-line stores: each chunk (64 bf16 or 32 four-byte columns = 128-byte rows) goes through
        // this warp's 128-byte-swizzled staging tile and one TMA store of 32 rows; parts of the box past
        // M or N are not written.  The accumulator is released after its last TMEM load.
        const bool wide = p.out_f32 != 0;
        const int chunks = wide ? 8 : 4;
        const int32_t wrow0 = (int32_t)(tm * 256 + 128 * rank + quarter * 32);
        uint8_t* sbuf = smem + kOffBuf + (warp - 4) * kEpiBuf;
#pragma unroll 1
        for (int c = 0; c < chunks; ++c) {
          uint32_t w[32];
          if (wide) {
            tmem_ld_32x32b_x32(t_addr + c * 32, w);
            tc_wait_ld();
          } else {
            uint32_t v[32];
            tmem_ld_32x32b_x32(t_addr + c * 64, v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            tmem_ld_32x32b_x32(t_addr + c * 64 + 32, v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              w[16 + j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          }
          if (c == chunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_acc_empty0 + 8u * (uint32_t)ab);
          }
          const int64_t col0 = n0 + (wide ? 32 : 64) * c;
          if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read the tile
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(sbuf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && col0 < p.N && (int64_t)wrow0 < p.M) {
            tma_store_2d(&p.tm_out, sbuf, (int32_t)col0, wrow0);
            bulk_commit_group();
          }
        }
        continue;
      }
      bool row_ok = row < p.M;
      int64_t orow = row;
      if (EPI == EPI_STORE && row_ok && p.row_map) {
        const int32_t v = __ldg(p.row_map + row);
        row_ok = v >= 0 && (int64_t)v < p.rows_out;
        orow = v;
      }
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_addr + c * 32, v);
        tc_wait_ld();
        const int64_t col0 = n0 + 32 * c;
        if (!row_ok || col0 >= p.N) continue;
        if (EPI == EPI_STORE) {
          if (p.out_f32) {
            float* y = static_cast<float*>(p.out) + orow * p.ldo + col0;
            if (col0 + 32 <= p.N) {
#pragma unroll
              for (int q = 0; q < 8; ++q)
                reinterpret_cast<float4*>(y)[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                              __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (col0 + e < p.N) y[e] = __uint_as_float(v[e]);
            }
          } else {
            uint16_t* y = static_cast<uint16_t*>(p.out) + orow * p.ldo + col0;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (col0 + 32 <= p.N) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<uint4*>(y)[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (col0 + e < p.N) y[e] = (uint16_t)(pk[e >> 1] >> (16 * (e & 1)));
            }
          }
        } else if (p.vec_out && col0 + 32 <= p.N) {
          // 2:4: the chunk's eight groups take their nibbles from two tiled metadata words (column
          // halves h = 0, 1 of the chunk's 32-column quarter q); the sixteen survivors are picked from
          // registers and stored as 32 (bf16) or 64 (fp32) contiguous bytes of the row.
          const uint32_t* mb =
              p.meta + ((row >> 4) * p.meta_cblocks + (col0 >> 7)) * 64 + 4 * (row & 7) + ((col0 >> 5) & 3);
          const uint32_t wh[2] = {__ldg(mb), __ldg(mb + 32)};
          const int sh = 16 * (int)((row >> 3) & 1);
          float o[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t nib = (wh[i >> 2] >> (sh + 4 * (i & 3))) & 0xFu;
            const uint32_t p0 = nib & 3u, p1 = nib >> 2;
            const float a0 = __uint_as_float(v[4 * i]), a1 = __uint_as_float(v[4 * i + 1]);
            const float a2 = __uint_as_float(v[4 * i + 2]), a3 = __uint_as_float(v[4 * i + 3]);
            o[2 * i] = p0 == 0 ? a0 : (p0 == 1 ? a1 : a2);
            o[2 * i + 1] = p1 == 3 ? a3 : (p1 == 2 ? a2 : a1);
          }
          if (p.out_f32) {
            float4* y = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.ldo + (col0 >> 1));
#pragma unroll
            for (int q = 0; q < 4; ++q) y[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          } else {
            uint4* y = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.ldo + (col0 >> 1));
            y[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                              pack_bf16x2(o[6], o[7]));
            y[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                              pack_bf16x2(o[14], o[15]));
          }
        } else {
          // survivors of weight row `row` among columns col0 .. col0 + 31 (M divides 32)
#pragma unroll
          for (int e = 0; e < 32; ++e) buf[e] = __uint_as_float(v[e]);
          const int64_t cend = col0 + 32 < p.N ? col0 + 32 : p.N;
          const int64_t j0 = col0 / p.m * p.n, j1 = cend / p.m * p.n;
          for (int64_t j = j0; j < j1; ++j) {
            const float val = buf[survivor_col(p, row, j) - col0];
            if (p.out_f32)
              static_cast<float*>(p.out)[row * p.ldo + j] = val;
            else
              static_cast<uint16_t*>(p.out)[row * p.ldo + j] = (uint16_t)(pack_bf16x2(val, 0.0f) & 0xFFFFu);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_acc_empty0 + 8u * (uint32_t)ab);
    }
    if (lane == 0) bulk_wait_group<0>();  // every TMA store of this warp has landed
  }

  // -------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) sleep_about_ns(200000ull);
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, dpair::kTmemCols);
  }
}

template <bool A_MN, bool B_MN, int EPI, bool I8 = false, bool TF32 = false>
static cudaError_t launch_dp(const DenseParams& p, cudaStream_t stream) {
  static std::atomic<bool> configured[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(dense_pair_kernel<A_MN, B_MN, EPI, I8, TF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dpair::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int pairs_avail = sm_count_current() / 2;
  const int pairs = p.num_tiles < pairs_avail ? p.num_tiles : pairs_avail;
  // Tile order: the pairs running at one time take consecutive tiles.  With A (M x Kr) larger than B
  // (Kr x N), column tiles go fastest so that they share A's row block and each block of A streams from
  // HBM about once (a float32 W' of 11008 x 4096 is 180 MB, above the 126 MB L2); otherwise row tiles.
  DenseParams q = p;
  q.n_major = p.M > p.N ? 1 : 0;
  cudaError_t e = launch_pdl(dense_pair_kernel<A_MN, B_MN, EPI, I8, TF32>, dim3(2 * pairs), dim3(dpair::kThreads),
                             (size_t)dpair::kSmemBytes, stream, q);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_dense_pair(const DenseParams& p, bool a_mn, bool b_mn, int epi, cudaStream_t stream) {
  if (p.num_tiles <= 0) return cudaSuccess;
  if (a_mn && b_mn && epi == EPI_STORE) return launch_dp<true, true, EPI_STORE>(p, stream);
  if (!a_mn && !b_mn && epi == EPI_SURVIVORS) return launch_dp<false, false, EPI_SURVIVORS>(p, stream);
  if (!a_mn && b_mn && epi == EPI_STORE) return launch_dp<false, true, EPI_STORE>(p, stream);
  return cudaErrorInvalidValue;
}

// int8 forward GEMM on the decompressed operand: A K-major, B MN-major, int32 stored through the 32-bit path
// (p.out_f32 = 1 moves the accumulator bits unchanged).
cudaError_t launch_dense_pair_i8(const DenseParams& p, cudaStream_t stream) {
  if (p.num_tiles <= 0) return cudaSuccess;
  return launch_dp<false, true, EPI_STORE, true>(p, stream);
}

// tf32 forward GEMM on the decompressed 1:2 operand: A (float32) K-major, B (float32) MN-major, a stage of
// 64 reduction steps in the same bytes as a bf16 stage.
cudaError_t launch_dense_pair_tf32(const DenseParams& p, cudaStream_t stream) {
  if (p.num_tiles <= 0) return cudaSuccess;
  return launch_dp<false, true, EPI_STORE, false, true>(p, stream);
}

}  // namespace nmk
