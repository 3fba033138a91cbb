// nm_spmm_fused.cu -- prune + compress + 2:4 GEMM in one kernel, for few columns (T <= 64).
//
// Y = W' X where W' is W under the 2:4 magnitude mask ("M:N sparsity on
// NVIDIA tensor cores": keep the 2 of every 4 consecutive weights along K with
// the largest magnitude, equal magnitudes to the lower index), computed from
// the dense W without a separate compress pass: the selection runs on each
// weight tile in shared memory, feeding the sparse MMA directly, and the
// compressed operand (values + tiled metadata, exactly nm_prune_compress's
// output) is optionally written on the way.  For shapes whose weights are
// read once (decode, T <= 64) this removes the compress pass's write and the
// GEMM's re-read of the compressed operand: HBM traffic is W read once, plus
// the compressed form if it is requested.
//
// Work units as in nm_spmm_skinny.cu (one 128-row tile and one range of
// 128-deep K stages, persistent CTAs, fp32 partials + range-ordered reduction
// when K is split).  Per stage: TMA brings the dense 128 x 128 W tile (32 KB,
// one box) and the X rows; eight selector warps, one per 16-row block, read
// the tile from shared memory, select, and write the compressed values into
// the MMA's A slot (128-byte swizzled K-major rows) and the 16-row block's 64
// metadata words into the E slot (the layout tcgen05.cp expects); the MMA
// thread then copies E into TMEM and issues four tcgen05.mma.sp (M = 128,
// N = bn, K = 32).  Two groups of eight selector warps take alternate stages:
// the selection is integer work on the ALU pipe, which one group cannot run
// at the rate the tiles arrive.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_select.cuh"
#include "nm_spmm.h"

namespace nmk {

namespace fused {
constexpr int kSelectors = 8;  // warps per stage, one per 16-row block
constexpr int kGroups = 2;     // selector groups, taking alternate stages
static_assert(kGroups == 2, "full barriers are laid out per (slot, group) for two groups");
constexpr int kSelWarps = kSelectors * kGroups;
constexpr int kThreads = 32 * (2 + kSelWarps + 4);  // 0 copies, 1 MMA, 2..17 select, 18..21 epilogue
constexpr int kAcc = 4;
constexpr uint32_t kW = 32768, kA = 16384, kE = 2048;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kSmemBudget = 222 * 1024;
__host__ __device__ constexpr uint32_t b_bytes(int bn) { return 128u * (uint32_t)bn * 2u; }
__host__ __device__ constexpr uint32_t stage_bytes(int bn) { return kW + kA + kE + b_bytes(bn); }
__host__ __device__ constexpr int stages(int bn) {
  return (int)((kSmemBudget - 1024) / stage_bytes(bn)) > 4 ? 4 : (int)((kSmemBudget - 1024) / stage_bytes(bn));
}
__host__ __device__ constexpr uint32_t tmem_cols(int bn) {
  return (uint32_t)(kAcc * bn + 4 * stages(bn)) <= 128 ? 128u
         : (uint32_t)(kAcc * bn + 4 * stages(bn)) <= 256 ? 256u : 512u;
}
}  // namespace fused

template <int BN>
__global__ void __launch_bounds__(fused::kThreads, 1) prune_spmm_skinny_kernel(const __grid_constant__ SpmmParams p) {
  using namespace fused;
  constexpr int S = stages(BN);
  constexpr uint32_t kB = b_bytes(BN);
  constexpr uint32_t BSW = (uint32_t)BN * 2u;
  constexpr uint32_t B_SWZ = BSW == 128 ? SWZ_128B : BSW == 64 ? SWZ_64B : SWZ_32B;
  constexpr uint32_t kIdesc = idesc_bf16(BN, true, 128);
  constexpr uint32_t kCols = tmem_cols(BN);
  constexpr uint32_t kECol = kAcc * BN;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* w_base = smem;                // S x 32 KB: dense W tiles, 256-byte rows
  uint8_t* a_base = w_base + S * kW;     // S x 16 KB: compressed values, SW128 K-major
  uint8_t* b_base = a_base + S * kA;     // S x kB: X rows
  uint8_t* e_base = b_base + S * kB;     // S x 2 KB: metadata blocks
  // full[2 s + g]: the copies of a stage in slot s taken by selector group g.  With S odd
  // the uses of one slot alternate between the groups; a barrier per (slot, group) keeps
  // every barrier's phases consumed in order by one group, as its parity waits need.
  uint64_t* full = reinterpret_cast<uint64_t*>(e_base + S * kE);
  uint64_t* built = full + 2 * S;
  uint64_t* empty = built + S;
  uint64_t* acc_full = empty + S;
  uint64_t* acc_empty = acc_full + kAcc;
  uint64_t* spare = acc_empty + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(spare + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int units = p.tiles_m * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[2 * s], 1);
      mbar_init(&full[2 * s + 1], 1);
      mbar_init(&built[s], kSelectors);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(spare, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_w);
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;
  pdl_gate();  // no global memory touched before this point

  auto unit_range = [&](int u, int& tm, int64_t& kt0, int64_t& kt1) {
    tm = u % p.tiles_m;
    const int sp = u / p.tiles_m;
    kt0 = (int64_t)sp * p.kt_per_split;
    kt1 = kt0 + p.kt_per_split < p.k_tiles ? kt0 + p.kt_per_split : p.k_tiles;
  };

  if (warp == 0) {
    // -------------------------------------------------------------- copies
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, j = 0;  // j: the CTA's stage counter (stage j goes to group j % kGroups)
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int tm;
        int64_t kt0, kt1;
        unit_range(u, tm, kt0, kt1);
        for (int64_t kt = kt0; kt < kt1; ++kt, ++j) {
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          uint64_t* fb = &full[2 * s + (int)(j % kGroups)];
          mbar_arrive_expect_tx(fb, kW + kB);
          tma_load_2d(w_base + s * kW, &p.tm_w, fb, (int32_t)(kt * 128), tm * 128);
          tma_load_2d(b_base + s * kB, &p.tm_x, fb, 0, (int32_t)(kt * 128));
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      int s = 0, i = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
        int tm;
        int64_t kt0, kt1;
        unit_range(u, tm, kt0, kt1);
        const int a = i % kAcc;
        ok = mbar_wait(&acc_empty[a], ((uint32_t)(i / kAcc) & 1u) ^ 1u, abort_flag, p.status, kWaitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(a * BN);
        for (int64_t kt = kt0; kt < kt1; ++kt) {
          ok = mbar_wait(&built[s], ph, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(a_base + s * kA);
          const uint32_t b_addr = smem_u32(b_base + s * kB);
          const uint32_t e_tmem = tmem_base + kECol + 4u * s;
          tc_cp_128x128b(e_tmem, smem_desc(smem_u32(e_base + s * kE), 2048, 128, SWZ_NONE));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(a_addr + kk * 32, 16, 1024, SWZ_128B);
            const uint64_t bd = smem_desc(b_addr + kk * 32 * BSW, 128 * BSW, 8 * BSW, B_SWZ);
            tc_mma_sp(d_tmem, ad, bd, e_tmem + (uint32_t)(kk & 2), kIdesc | (uint32_t)(kk & 1),
                      (kt > kt0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[a]);
      }
      if (!ok) {
        tc_commit(spare);
        volatile int dummy = 0;
        mbar_wait(spare, 0, &dummy, p.status, 100000000ull);
      }
    }
  } else if (warp < 2 + kSelWarps) {
    // ---------------------------------------- selectors: one 16-row block each
    // Group g takes the CTA's stages j with j % kGroups == g, so that two
    // stages are selected at once.  Lane (half, piece) = (lane / 16, lane % 16)
    // takes rows 2i + half of the block and columns 8*piece .. +7 (two groups),
    // as in the compress kernels.
    const int blk16 = (warp - 2) % kSelectors;
    const int group = (warp - 2) / kSelectors;
    const uint32_t half = lane >> 4, piece = lane & 15u;
    const uint32_t l = lane >> 1, rr = l & 7u, hh = l >> 3, kb = rr >> 1;
    const uint32_t src0 = 16 * (rr & 1u) + 8 * (lane & 1u) + 2 * hh;  // see store of the metadata words
    const uint32_t pick = kb | ((kb + 4) << 4);
    uint32_t j = 0;  // the CTA's stage counter
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int tm;
      int64_t kt0, kt1;
      unit_range(u, tm, kt0, kt1);
      for (int64_t kt = kt0; kt < kt1; ++kt, ++j) {
        if ((int)(j % kGroups) != group) continue;
        // the group's uses of barrier (slot s, group) are its stages j = r mod lcm(S, kGroups)
        constexpr uint32_t kCycle = S % kGroups == 0 ? S : S * kGroups;
        const uint32_t s = j % S, ph = (j / kCycle) & 1u;
        ok = mbar_wait(&full[2 * s + group], ph, abort_flag, p.status, kWaitNs);
        if (!ok) break;
        const uint8_t* wt = w_base + s * kW + blk16 * 16 * 256;
        uint4 in[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) in[i] = *reinterpret_cast<const uint4*>(wt + (2 * i + half) * 256 + piece * 16);
        uint32_t pk[16], by[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          by[i] = select_quad(in[i], pk[2 * i], pk[2 * i + 1]);
        // compressed values into the A slot: tile row r, 128 bytes, 16-byte chunks swizzled by r % 8
        uint8_t* at = a_base + s * kA;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t r = 16 * blk16 + 2 * i + half;
          *reinterpret_cast<uint2*>(at + r * 128 + ((((piece >> 1) ^ (r & 7u)) << 4) | ((piece & 1u) << 3))) =
              make_uint2(pk[2 * i], pk[2 * i + 1]);
        }
        // the block's 64 metadata words (tiled order), two per lane
        const uint32_t lo8 = by[0] | (by[1] << 8) | (by[2] << 16) | (by[3] << 24);
        const uint32_t hi8 = by[4] | (by[5] << 8) | (by[6] << 16) | (by[7] << 24);
        const uint32_t a0 = __shfl_sync(0xffffffffu, lo8, src0), a1 = __shfl_sync(0xffffffffu, lo8, src0 + 1);
        const uint32_t b0 = __shfl_sync(0xffffffffu, hi8, src0), b1 = __shfl_sync(0xffffffffu, hi8, src0 + 1);
        const uint32_t c0 = __shfl_sync(0xffffffffu, lo8, src0 + 4), c1 = __shfl_sync(0xffffffffu, lo8, src0 + 5);
        const uint32_t d0 = __shfl_sync(0xffffffffu, hi8, src0 + 4), d1 = __shfl_sync(0xffffffffu, hi8, src0 + 5);
        const uint32_t w0 = __byte_perm(__byte_perm(a0, a1, pick), __byte_perm(b0, b1, pick), 0x5410u);
        const uint32_t w1 = __byte_perm(__byte_perm(c0, c1, pick), __byte_perm(d0, d1, pick), 0x5410u);
        *reinterpret_cast<uint2*>(e_base + s * kE + blk16 * 256 + 8 * lane) = make_uint2(w0, w1);
        fence_proxy_async_smem();  // the A and E slots are read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&built[s]);
        // optional outputs: the compressed operand, exactly as nm_prune_compress writes it
        // (after the arrival, so that the MMA need not wait for these stores)
        if (p.out_vals) {
          const int64_t col = kt * 128 + 8 * piece;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int64_t row = (int64_t)tm * 128 + 16 * blk16 + 2 * i + half;
            if (row < p.R)
              *reinterpret_cast<uint2*>(p.out_vals + row * (p.K >> 1) + col / 2) = make_uint2(pk[2 * i], pk[2 * i + 1]);
          }
        }
        if (p.out_meta) {
          const int64_t rbg = (int64_t)tm * 8 + blk16;
          if (rbg < p.meta_rblocks)
            *reinterpret_cast<uint2*>(p.out_meta + (rbg * p.meta_cblocks + kt) * 64 + 2 * lane) = make_uint2(w0, w1);
        }
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    int i = 0;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++i) {
      int tm;
      int64_t kt0, kt1;
      unit_range(u, tm, kt0, kt1);
      const int sp = u / p.tiles_m;
      const int a = i % kAcc;
      ok = mbar_wait(&acc_full[a], (uint32_t)(i / kAcc) & 1u, abort_flag, p.status, kWaitNs);
      if (!ok) break;
      tc_fence_after();
      const int64_t row = (int64_t)tm * 128 + quarter * 32 + lane;
      const bool row_ok = row < p.R;
      const uint32_t t_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * BN);
      float acc[BN];
#pragma unroll
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(t_addr + c * 16, v);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[c * 16 + e] = __uint_as_float(v[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
      if (!row_ok) continue;
      if (p.splits > 1) {
        float4* part = reinterpret_cast<float4*>(p.ws + ((int64_t)sp * p.R + row) * BN);
#pragma unroll
        for (int q = 0; q < BN / 4; ++q) part[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
      } else if (p.out_f32) {
        float* y = static_cast<float*>(p.Y) + row * p.ldy;
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e < p.T) y[e] = acc[e];
      } else {
        uint16_t* y = static_cast<uint16_t*>(p.Y) + row * p.ldy;
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
          const uint32_t pk = pack_bf16x2(acc[e], acc[e + 1]);
          if (e < p.T) y[e] = (uint16_t)(pk & 0xFFFFu);
          if (e + 1 < p.T) y[e + 1] = (uint16_t)(pk >> 16);
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    sleep_about_ns(200000ull);
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kCols);
  }
}

template <int BN>
static cudaError_t launch_fused_bn(SpmmParams& p, cudaStream_t stream) {
  using namespace fused;
  constexpr int S = stages(BN);
  const size_t bytes = (size_t)S * stage_bytes(BN) + (4 * S + 2 * kAcc + 1) * 8 + 16 + 1024;
  static std::atomic<bool> configured[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(prune_spmm_skinny_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int units = p.tiles_m * p.splits;
  const int sms = sm_count_current();
  cudaError_t e = launch_pdl(prune_spmm_skinny_kernel<BN>, dim3(units < sms ? units : sms), dim3(kThreads), bytes,
                             stream, p);
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  return launch_skinny_reduce(p, stream);
}

cudaError_t launch_prune_spmm_skinny(SpmmParams& p, cudaStream_t stream) {
  switch (p.bn) {
    case 16: return launch_fused_bn<16>(p, stream);
    case 32: return launch_fused_bn<32>(p, stream);
    case 64: return launch_fused_bn<64>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nmk
