// nm_spmm_skinny.cu -- 2:4 sparse x dense GEMM for few columns (T <= 64), split along K.
//
// Same operation as nm_spmm.cu ("M:N sparsity on NVIDIA tensor cores", GEMM
// paragraphs of "Where this sits among the three case studies"), for the
// decode-like shapes where X has a handful of columns: the whole cost is
// streaming the compressed weights once, so the kernel is built for bytes in
// flight, not for MMA throughput.  A work unit is one 128-row tile and one
// range of 128-deep K stages; persistent CTAs (one per SM) walk the units, so
// the row tiles times the K ranges cover every SM even when R / 128 is below
// the SM count.  Per stage, TMA brings the compressed values (two 64-row
// boxes, 128-byte swizzle), the tiled 2:4 metadata (one 3-D box of eight
// 16-row blocks) and the X rows (one box of bn columns); the MMA thread copies
// the metadata into TMEM and issues four tcgen05.mma.sp (M = 128, N = bn,
// K = 32).  Accumulators rotate through four TMEM buffers, so the epilogue of
// one unit overlaps the next.  With one K range the epilogue writes Y; with
// several it writes fp32 partials, which skinny_reduce_kernel (launched as a
// programmatic dependent of this kernel) sums in range order into Y.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_spmm.h"

namespace nmk {

namespace skinny {
constexpr int kThreads = 256;  // warp 0 A copies, 1 MMA, 2 E + B copies, 4..7 epilogue
constexpr int kAcc = 4;
// Stage depth KD (128 or 256 logical K): A = 128 rows x KD/2 values as
// 64-row x 64-value boxes, E = KD/128 metadata boxes of 2 KB, B = KD rows.
__host__ __device__ constexpr uint32_t a_bytes(int kd) { return 128u * (uint32_t)kd; }
__host__ __device__ constexpr uint32_t e_bytes(int kd) { return 2048u * (uint32_t)(kd / 128); }
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kSmemBudget = 220 * 1024;

__host__ __device__ constexpr uint32_t b_bytes(int bn, int kd) { return (uint32_t)kd * (uint32_t)bn * 2u; }
__host__ __device__ constexpr uint32_t stage_bytes(int bn, int kd) { return a_bytes(kd) + e_bytes(kd) + b_bytes(bn, kd); }
__host__ __device__ constexpr int stages(int bn, int kd) {
  return (int)((kSmemBudget - 1024) / stage_bytes(bn, kd)) > 8 ? 8 : (int)((kSmemBudget - 1024) / stage_bytes(bn, kd));
}
__host__ __device__ constexpr uint32_t tmem_cols(int bn, int kd) {
  // kAcc accumulators of bn columns plus kd/32 metadata columns per stage, as a power of two >= 32
  return (uint32_t)(kAcc * bn + (kd / 32) * stages(bn, kd)) <= 128 ? 128u
         : (uint32_t)(kAcc * bn + (kd / 32) * stages(bn, kd)) <= 256 ? 256u : 512u;
}
}  // namespace skinny

template <int BN, int KD>
__global__ void __launch_bounds__(skinny::kThreads, 1) spmm_skinny_kernel(const __grid_constant__ SpmmParams p) {
  using namespace skinny;
  constexpr int S = stages(BN, KD);
  constexpr uint32_t kA = a_bytes(KD), kE = e_bytes(KD);
  constexpr uint32_t kB = b_bytes(BN, KD);
  constexpr uint32_t kStage = stage_bytes(BN, KD);
  constexpr int KC = KD / 128;  // 128-deep chunks per stage
  constexpr uint32_t BSW = (uint32_t)BN * 2u;  // bytes per swizzled X row in smem (32, 64 or 128)
  constexpr uint32_t B_SWZ = BSW == 128 ? SWZ_128B : BSW == 64 ? SWZ_64B : SWZ_32B;
  constexpr uint32_t kIdesc = idesc_bf16(BN, true, 128);
  constexpr uint32_t kCols = tmem_cols(BN, KD);
  constexpr uint32_t kECol = kAcc * BN;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: A at s*kA, then all B slots, then all E slots (1024-byte aligned slots)
  uint8_t* a_base = smem;
  uint8_t* b_base = smem + S * kA;
  uint8_t* e_base = b_base + S * kB;
  uint64_t* full = reinterpret_cast<uint64_t*>(e_base + S * kE);
  uint64_t* empty = full + S;
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
      mbar_init(&full[s], 1);
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
    tma_prefetch_desc(&p.tm_vals);
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_meta);
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

  if (warp == 0 || warp == 2) {
    // ------------------------------------------- copies: warp 0 A (two boxes), warp 2 E and B
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int tm;
        int64_t kt0, kt1;
        unit_range(u, tm, kt0, kt1);
        for (int64_t kt = kt0; kt < kt1; ++kt) {
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          if (warp == 0) {
            mbar_arrive_expect_tx(&full[s], kStage);
#pragma unroll
            for (int c = 0; c < KC; ++c) {  // chunk c: values (kt*KC + c)*64 .. +63, rows in two boxes
              tma_load_2d(a_base + s * kA + c * 16384, &p.tm_vals, &full[s], (int32_t)((kt * KC + c) * 64), tm * 128);
              tma_load_2d(a_base + s * kA + c * 16384 + 8192, &p.tm_vals, &full[s], (int32_t)((kt * KC + c) * 64),
                          tm * 128 + 64);
            }
          } else {
#pragma unroll
            for (int c = 0; c < KC; ++c)
              tma_load_3d(e_base + s * kE + c * 2048, &p.tm_meta, &full[s], 0, (int32_t)(kt * KC + c), tm * 8);
            tma_load_2d(b_base + s * kB, &p.tm_x, &full[s], 0, (int32_t)(kt * KD));
          }
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
          ok = mbar_wait(&full[s], ph, abort_flag, p.status, kWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(a_base + s * kA);
          const uint32_t b_addr = smem_u32(b_base + s * kB);
          const uint32_t e_tmem = tmem_base + kECol + (uint32_t)(KD / 32) * s;
#pragma unroll
          for (int c = 0; c < KC; ++c)
            tc_cp_128x128b(e_tmem + 4u * c, smem_desc(smem_u32(e_base + s * kE + c * 2048), 2048, 128, SWZ_NONE));
#pragma unroll
          for (int kk = 0; kk < KD / 32; ++kk) {
            const uint64_t ad = smem_desc(a_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, SWZ_128B);
            const uint64_t bd = smem_desc(b_addr + kk * 32 * BSW, (uint32_t)KD * BSW, 8 * BSW, B_SWZ);
            tc_mma_sp(d_tmem, ad, bd, e_tmem + 4u * (kk >> 2) + (uint32_t)(kk & 2), kIdesc | (uint32_t)(kk & 1),
                      (kt > kt0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&acc_full[a]);
      }
      if (!ok) {  // let MMAs already issued finish before TMEM is freed
        tc_commit(spare);
        volatile int dummy = 0;
        mbar_wait(spare, 0, &dummy, p.status, 100000000ull);
      }
    }
  } else if (warp >= 4) {
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
      if (lane == 0) mbar_arrive(&acc_empty[a]);  // the accumulator is in registers now
      if (p.splits > 1) {
        if (row_ok) {
          float4* part = reinterpret_cast<float4*>(p.ws + ((int64_t)sp * p.R + row) * BN);
#pragma unroll
          for (int q = 0; q < BN / 4; ++q) part[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        }
        continue;
      }
      if (row_ok) {
        if (p.out_f32) {
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

// Y[r][t] = sum over K ranges s (in order) of ws[s][r][t], t < T.  Launched as
// a programmatic dependent of the GEMM: it may start while the GEMM drains
// and waits (griddepcontrol.wait) for the GEMM's writes before reading ws.
__global__ void __launch_bounds__(256) skinny_reduce_kernel(const float* __restrict__ ws, int splits, int64_t R,
                                                            int bn, int64_t T, void* Y, int64_t ldy, int out_f32) {
  pdl_gate();
  const int64_t total = R * T;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / T, t = i - r * T;
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += __ldcg(ws + ((int64_t)s * R + r) * bn + t);
    if (out_f32) static_cast<float*>(Y)[r * ldy + t] = acc;
    else static_cast<uint16_t*>(Y)[r * ldy + t] = (uint16_t)(pack_bf16x2(acc, 0.f) & 0xFFFFu);
  }
}

bool skinny_kernel_fits(int64_t T) { return T >= 1 && T <= 64; }

int skinny_bn(int64_t T) { return T <= 16 ? 16 : T <= 32 ? 32 : 64; }

// Sum of the K ranges' fp32 partials into Y (when the skinny kernels split K).
cudaError_t launch_skinny_reduce(const SpmmParams& p, cudaStream_t stream) {
  const int sms = sm_count_current();
  const int64_t total = p.R * p.T;
  const int64_t want = (total + 255) / 256;
  const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  cudaError_t e = launch_pdl(skinny_reduce_kernel, dim3(grid), dim3(256), 0, stream, (const float*)p.ws, p.splits,
                             p.R, p.bn, p.T, p.Y, p.ldy, p.out_f32);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int BN, int KD>
static cudaError_t launch_bn(SpmmParams& p, cudaStream_t stream) {
  using namespace skinny;
  constexpr int S = stages(BN, KD);
  const size_t bytes = (size_t)S * stage_bytes(BN, KD) + (2 * S + 2 * kAcc + 1) * 8 + 16 + 1024;  // + slots, align
  static std::atomic<bool> configured[64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(spmm_skinny_kernel<BN, KD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const int units = p.tiles_m * p.splits;
  const int sms = sm_count_current();
  cudaError_t e = launch_pdl(spmm_skinny_kernel<BN, KD>, dim3(units < sms ? units : sms), dim3(kThreads), bytes,
                             stream, p);
  count_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  return launch_skinny_reduce(p, stream);
}

int skinny_kd(int64_t K, int64_t T) { (void)T; return K % 128 == 0 ? 128 : 0; }

cudaError_t launch_spmm_skinny(SpmmParams& p, cudaStream_t stream) {
  const bool deep = p.kd == 256;
  switch (p.bn) {
    case 16: return deep ? launch_bn<16, 256>(p, stream) : launch_bn<16, 128>(p, stream);
    case 32: return deep ? launch_bn<32, 256>(p, stream) : launch_bn<32, 128>(p, stream);
    case 64: return deep ? launch_bn<64, 256>(p, stream) : launch_bn<64, 128>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nmk
