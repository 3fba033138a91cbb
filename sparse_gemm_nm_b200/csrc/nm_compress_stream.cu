// nm_compress_stream.cu -- 2:4 prune + compress as a TMA-fed stream.
//
// Same result as compress_2of4_tiled_kernel (nm_compress.cu; selection and
// storage rules from "M:N sparsity on NVIDIA tensor cores": keep the 2 of
// every 4 consecutive weights along K with the largest magnitude, equal
// magnitudes to the lower index, survivors pushed left, 2:4 metadata in the
// tiled tensor-core order), built to keep HBM busy: a producer warp streams
// 16-row x 128-column blocks of W (4 KB TMA boxes) into a 16-slot shared-memory
// ring, and eight consumer warps select from shared memory and store values and
// metadata while the next blocks are in flight.  Blocks past R or K arrive
// zero-filled, which selects positions (0, 1): exactly the padding nibble 0x4;
// values are stored only inside R x K.  Optionally the same grid also gathers
// the permuted rows of a GEMM input (see kGatherWarps).
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "nm_internal.h"
#include "nm_ptx.cuh"
#include "nm_select.cuh"

namespace nmk {

namespace cstream {
constexpr int kConsumers = 8;
constexpr int kThreads = 32 * (kConsumers + 1);  // warps 0..7 consume, warp 8 produces
// With a gather job the CTA also runs kGatherWarps warps (9 ..) that copy the
// permuted rows of an input X: integer-bound selection leaves HBM bandwidth
// to spare, which the copy uses.
constexpr int kGatherWarps = 4;
constexpr int kThreadsGather = kThreads + 32 * kGatherWarps;
constexpr int kSlots = 16;
constexpr uint32_t kBlockBytes = 16 * 128 * 2;
constexpr uint64_t kWaitNs = 2000000000ull;
// Dynamic shared memory requested per CTA: the ring needs ~66 KB, but the
// request is sized so that at most two CTAs fit on an SM.  Launched as a
// programmatic dependent, the persistent grid is placed while the previous
// kernel drains; without the cap three CTAs could land on each early-freed SM
// and leave the last SMs to free up without work.
constexpr size_t kSmem = 100 * 1024;
static_assert(kSlots * kBlockBytes + 2 * kSlots * 8 + 64 + 1024 <= kSmem, "ring does not fit");
// Block j goes to slot j % kSlots and to consumer warp j % kConsumers, and the
// waits test barrier phases by parity.  With kSlots a multiple of kConsumers
// every slot is always read by the same warp, which takes its uses in order, so
// a warp never waits on use u of a slot before use u - 1 has completed (the
// parity of use u - 2 would otherwise pass for use u).
static_assert(kSlots % kConsumers == 0, "each ring slot must belong to one consumer warp");
}  // namespace cstream

template <bool GATHER>
__global__ void __launch_bounds__(GATHER ? cstream::kThreadsGather : cstream::kThreads, 2)
    compress_2of4_stream_kernel(const __grid_constant__ CUtensorMap tm_w, uint32_t R, uint32_t K,
                                uint16_t* __restrict__ V, uint32_t* __restrict__ meta, uint32_t cblocks,
                                uint32_t nblocks, uint32_t* status, const __grid_constant__ GatherJob gj) {
  using namespace cstream;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kSlots * kBlockBytes);
  uint64_t* empty = full + kSlots;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kSlots);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kConsumers && lane == 0) tma_prefetch_desc(&tm_w);
  __syncthreads();
  pdl_gate();  // no global memory touched before this point

  // this CTA's blocks: blockIdx.x + j * gridDim.x, j = 0, 1, ...; slot j % kSlots; consumer j % kConsumers
  const uint32_t nmine = blockIdx.x < nblocks ? (nblocks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (GATHER && warp > kConsumers) {
    gather_rows_items(gj, (int64_t)blockIdx.x * kGatherWarps + (warp - kConsumers - 1),
                      (int64_t)gridDim.x * kGatherWarps, lane);
    return;
  }
  if (warp == kConsumers) {
    if (lane == 0) {
      for (uint32_t j = 0; j < nmine; ++j) {
        const uint32_t slot = j % kSlots, use = j / kSlots;
        if (!mbar_wait(&empty[slot], (use & 1u) ^ 1u, abort_flag, status, kWaitNs)) break;
        const uint32_t blk = blockIdx.x + j * gridDim.x;
        const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
        mbar_arrive_expect_tx(&full[slot], kBlockBytes);
        tma_load_2d(ring + slot * kBlockBytes, &tm_w, &full[slot], (int32_t)(cb * 128), (int32_t)(rb * 16));
      }
    }
    return;
  }
  const uint32_t half = lane >> 4, piece = lane & 15u;
  for (uint32_t j = warp; j < nmine; j += kConsumers) {
    const uint32_t slot = j % kSlots, use = j / kSlots;
    if (!mbar_wait(&full[slot], use & 1u, abort_flag, status, kWaitNs)) break;
    const uint32_t blk = blockIdx.x + j * gridDim.x;
    const uint32_t rb = blk / cblocks, cb = blk - rb * cblocks;
    const uint8_t* src = ring + slot * kBlockBytes;
    uint4 in[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)  // row 2i + half, columns 8*piece .. +7 of the block
      in[i] = *reinterpret_cast<const uint4*>(src + (2 * i + half) * 256 + piece * 16);
    uint32_t pk[16], by[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      by[i] = select_quad(in[i], pk[2 * i], pk[2 * i + 1]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);  // the block's registers are consumed
    const uint32_t col = cb * 128 + 8 * piece;
    if (col < K) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t row = rb * 16 + 2 * i + half;
        if (row < R)
          *reinterpret_cast<uint2*>(V + (int64_t)row * (K >> 1) + col / 2) = make_uint2(pk[2 * i], pk[2 * i + 1]);
      }
    }
    const uint32_t lo8 = by[0] | (by[1] << 8) | (by[2] << 16) | (by[3] << 24);
    const uint32_t hi8 = by[4] | (by[5] << 8) | (by[6] << 16) | (by[7] << 24);
    // Words 2L, 2L+1: tile lane l = L/2 (rows l%8 and 8 + l%8), column half h = l/8;
    // the nibble byte of (row r, piece p) is in lane 16*(r%2) + p, byte r/2 of lo8/hi8.
    const uint32_t l = lane >> 1, r = l & 7u, h = l >> 3, k = r >> 1;
    const uint32_t s0 = 16 * (r & 1u) + 8 * (lane & 1u) + 2 * h;
    const uint32_t a0 = __shfl_sync(0xffffffffu, lo8, s0), a1 = __shfl_sync(0xffffffffu, lo8, s0 + 1);
    const uint32_t b0 = __shfl_sync(0xffffffffu, hi8, s0), b1 = __shfl_sync(0xffffffffu, hi8, s0 + 1);
    const uint32_t c0 = __shfl_sync(0xffffffffu, lo8, s0 + 4), c1 = __shfl_sync(0xffffffffu, lo8, s0 + 5);
    const uint32_t d0 = __shfl_sync(0xffffffffu, hi8, s0 + 4), d1 = __shfl_sync(0xffffffffu, hi8, s0 + 5);
    const uint32_t pick = k | ((k + 4) << 4);
    const uint32_t w0 = __byte_perm(__byte_perm(a0, a1, pick), __byte_perm(b0, b1, pick), 0x5410u);
    const uint32_t w1 = __byte_perm(__byte_perm(c0, c1, pick), __byte_perm(d0, d1, pick), 0x5410u);
    *reinterpret_cast<uint2*>(meta + (int64_t)blk * 64 + 2 * lane) = make_uint2(w0, w1);
  }
}

cudaError_t launch_compress_stream(const CUtensorMap& tm_w, int64_t R, int64_t K, uint16_t* values, uint32_t* meta,
                                   uint32_t* status, cudaStream_t s, const GatherJob* gather) {
  using namespace cstream;
  static std::atomic<bool> configured[2][64];  // zero-initialised: false
  int dev = 0;
  cudaGetDevice(&dev);
  const int gi = gather ? 1 : 0;
  if (dev >= 0 && dev < 64 && !configured[gi][dev]) {
    cudaError_t e = gather ? cudaFuncSetAttribute(compress_2of4_stream_kernel<true>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem)
                           : cudaFuncSetAttribute(compress_2of4_stream_kernel<false>,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    configured[gi][dev] = true;
  }
  const int64_t nblocks = meta_row_blocks(R) * meta_col_blocks(K);
  const int64_t cap = (int64_t)sm_count_current() * 2;
  // with a gather job every CTA of the persistent grid also copies rows
  const int grid = gather ? (int)cap : (int)(nblocks < cap ? nblocks : cap);
  const GatherJob none{};
  cudaError_t e =
      gather ? launch_pdl(compress_2of4_stream_kernel<true>, dim3(grid), dim3(kThreadsGather), kSmem, s, tm_w,
                          (uint32_t)R, (uint32_t)K, values, meta, (uint32_t)meta_col_blocks(K), (uint32_t)nblocks,
                          status, *gather)
             : launch_pdl(compress_2of4_stream_kernel<false>, dim3(grid), dim3(kThreads), kSmem, s, tm_w, (uint32_t)R,
                          (uint32_t)K, values, meta, (uint32_t)meta_col_blocks(K), (uint32_t)nblocks, status, none);
  count_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nmk
