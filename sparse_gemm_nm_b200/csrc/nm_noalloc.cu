// nm_noalloc.cu -- a permuted 2:4 GEMM entry point that allocates no device memory.
//
// nm_spmm_permuted stages the gathered input Xp[k] = X[idx[k]] in a buffer it
// takes from the device's memory pool on the caller's stream.  Some callers
// cannot allow that: a runtime that plans every byte of device memory up front
// and treats any allocation it did not make as a failure, a process whose pool
// is exhausted or shared with an allocator that must stay the only owner, or a
// latency-critical loop where an allocation call that has to grow the pool is
// not acceptable.  nm_spmm_permuted_noalloc computes the same result with the
// same kernels, but stages the gathered input in a fixed array that lives in
// the library's module for as long as the process runs (32 MiB on every device
// that loads the library).  Columns of X are processed in chunks that fit the
// array; each chunk is gathered into it and multiplied before the next one.
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nm.h"
#include "nm_internal.h"
#include "nm_spmm.h"

namespace nmk {

void set_last_error(const char* msg);
bool pair_path_for(int n, int m, int64_t R, int64_t K, int64_t T, const void* values, const void* meta);
nm_status check_permuted_args(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                              const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                              nm_out_dtype y_dtype);
nm_status spmm_permuted_unstaged(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                                 const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y,
                                 int64_t ldy, nm_out_dtype y_dtype, cudaStream_t stream);
nm_status build_pair_params(SpmmParams& p, const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K,
                            const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy, bool out_f32);

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int64_t kNoAllocScratchElems = (int64_t)(kNoAllocScratchBytes / 2);

// The staging array.  Host code must not use its name as an address (on the
// host it is only a stand-in); the device address comes from
// cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) uint16_t g_noalloc_scratch[kNoAllocScratchElems];

static std::mutex g_noalloc_mu;
static uint16_t* g_noalloc_ptr[64];

// Device address of the staging array on the current device (set up on the
// first call for that device).
static nm_status scratch_for_current_device(uint16_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    set_last_error("no usable current CUDA device");
    return NM_ERR_NO_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      char msg[256];
      snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the staging array failed: %s", cudaGetErrorString(e));
      set_last_error(msg);
      return NM_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<uint16_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return NM_OK;
}

}  // namespace nmk

using namespace nmk;

extern "C" NM_API nm_status nm_spmm_permuted_noalloc(const uint16_t* values, const uint32_t* meta, int n, int m,
                                                     int64_t R, int64_t K, const int32_t* idx, const uint16_t* X,
                                                     int64_t ldx, int64_t T, void* Y, int64_t ldy,
                                                     nm_out_dtype y_dtype, void* stream) {
  // Other shapes and patterns run on the one-SM kernel, which gathers X rows
  // itself and stages nothing (no re-encoded operand either).
  if (!pair_path_for(n, m, R, K, T, values, meta) || R <= 0 || K <= 0 || T <= 0)
    return spmm_permuted_unstaged(values, meta, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype,
                                  static_cast<cudaStream_t>(stream));
  // The same checks, statuses and texts as nm_spmm_permuted.
  nm_status st = check_permuted_args(values, meta, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype);
  if (st != NM_OK) return st;
  const int esize = y_dtype == NM_OUT_F32 ? 4 : 2;
  // Each chunk stages K rows x `chunk` columns; chunks are multiples of 256
  // columns, so at least one 256-column chunk must fit.
  const int64_t chunk = kNoAllocScratchElems / K / 256 * 256;
  if (chunk < 256) {
    char msg[200];
    snprintf(msg, sizeof msg,
             "K = %lld is too large for the %zu MiB staging array of the allocation-free call (K <= %lld)",
             (long long)K, kNoAllocScratchBytes >> 20, (long long)(kNoAllocScratchElems / 256));
    set_last_error(msg);
    return NM_ERR_UNSUPPORTED;
  }
  uint16_t* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != NM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left; every element a chunk
  // reads is written by that chunk's gather first, so nothing is cleared.
  for (int64_t t0 = 0; t0 < T; t0 += chunk) {
    const int64_t tc = (T - t0 < chunk) ? T - t0 : chunk;
    uint8_t* y0 = static_cast<uint8_t*>(Y) + t0 * esize;
    if (!pair_path_for(n, m, R, K, tc, values, meta)) {
      // A last chunk too narrow for the two-SM kernel (fewer than 192
      // columns): the one-SM kernel reads its mapped rows of X itself and
      // stages nothing.  t0 is a multiple of 256, so X + t0 and y0 stay
      // 16-byte aligned.
      st = spmm_permuted_unstaged(values, meta, n, m, R, K, idx, X + t0, ldx, tc, y0, ldy, y_dtype, s);
      if (st != NM_OK) return st;
      continue;
    }
    cudaError_t e = launch_gather_rows(X + t0, ldx, idx, K, tc, scratch, tc, s);
    if (e != cudaSuccess) {
      set_last_error(cudaGetErrorString(e));
      return NM_ERR_CUDA;
    }
    SpmmParams p;
    st = build_pair_params(p, values, meta, R, K, scratch, tc, tc, y0, ldy, y_dtype == NM_OUT_F32);
    if (st != NM_OK) return st;
    e = launch_spmm_pair(p, s);
    if (e != cudaSuccess) {
      set_last_error(cudaGetErrorString(e));
      return NM_ERR_CUDA;
    }
  }
  return NM_OK;
}
