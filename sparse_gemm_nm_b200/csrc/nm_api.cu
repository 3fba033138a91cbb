// nm_api.cu -- the C ABI of libnm_b200 (declared in include/nm.h): argument
// checks on the host, tensor-map encoding, choice of kernel variant, launch.
#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/nm.h"
#include "nm_internal.h"
#include "nm_spmm.h"

namespace nmk {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static thread_local std::string t_last_error;

static nm_status fail(nm_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
static nm_status fail(nm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

static nm_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool known = false;
};
static DeviceInfo g_dev[64];
static std::mutex g_dev_mu;

static const DeviceInfo* device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.known) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
    if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
    d.known = true;
  }
  return &d;
}

int sm_count_current() {
  const DeviceInfo* d = device_info();
  return d ? d->sms : 148;
}

static nm_status require_device() {
  const DeviceInfo* d = device_info();
  if (!d) return fail(NM_ERR_NO_DEVICE, "no CUDA device is current");
  if (d->major != 10) return fail(NM_ERR_NO_DEVICE, "device is sm_%d0, this library is built for sm_100a", d->major);
  return NM_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Library-owned stream-ordered pool for the permuted GEMM's staging buffers,
// one per device.  Its release threshold is "never", so memory returned by
// cudaFreeAsync stays reserved for the next call instead of going back to the
// driver at each synchronisation: re-mapping tens of MB on every call costs
// far more than the GEMM.  nm_release_staging() hands the memory back.
static std::mutex g_pool_mu;
static cudaMemPool_t g_pool[64];

static cudaError_t staging_pool(cudaMemPool_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = ~0ull;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    g_pool[dev] = pool;
  }
  *out = g_pool[dev];
  return cudaSuccess;
}

// Per-thread cache of encoded tensor maps: a call that repeats the previous
// calls' buffers and shapes (an inference loop) skips cuTensorMapEncodeTiled.
// The key is every encode argument; a map depends on nothing else.
struct TmapKey {
  const void* base;
  uint64_t d0, d1, d2, s0, s1;
  uint32_t b0, b1, b2;
  int swizzle, dtype, rank;
  bool operator==(const TmapKey& o) const {
    return base == o.base && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && s0 == o.s0 && s1 == o.s1 && b0 == o.b0 &&
           b1 == o.b1 && b2 == o.b2 && swizzle == o.swizzle && dtype == o.dtype && rank == o.rank;
  }
};
struct TmapCache {
  static constexpr int kEntries = 32;
  TmapKey key[kEntries];
  CUtensorMap map[kEntries];
  bool used[kEntries] = {};
  int next = 0;
  bool find(const TmapKey& k, CUtensorMap* out) const {
    for (int i = 0; i < kEntries; ++i)
      if (used[i] && key[i] == k) {
        *out = map[i];
        return true;
      }
    return false;
  }
  void put(const TmapKey& k, const CUtensorMap& m) {
    key[next] = k;
    map[next] = m;
    used[next] = true;
    next = (next + 1) % kEntries;
  }
};
static thread_local TmapCache t_tmaps;

// swizzle_bytes code of the 128-byte swizzle with 32-byte units (MN-major tf32 operands of the MMA).
constexpr int kSwizzle128Atom32B = -32;

static nm_status make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                           uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes,
                           const char* what, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  const TmapKey key{base, inner, outer, 0, row_bytes, 0, box_inner, box_outer, 0, swizzle_bytes, (int)dtype, 2};
  if (t_tmaps.find(key, tm)) return NM_OK;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle swz = swizzle_bytes == 128                 ? CU_TENSOR_MAP_SWIZZLE_128B
                           : swizzle_bytes == kSwizzle128Atom32B ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                           : swizzle_bytes == 64                ? CU_TENSOR_MAP_SWIZZLE_64B
                           : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with %d", what, (int)r);
  t_tmaps.put(key, *tm);
  return NM_OK;
}

// Whole-line TMA stores for the dense pair kernel's plain epilogue: C is rows x cols with row stride ldo
// elements (bf16, or four-byte values when wide); the caller has checked 16-byte rows.
static nm_status set_store_map(DenseParams& p, void* out, int64_t rows, int64_t cols, int64_t ldo, bool wide) {
  p.tma_store = 1;
  return wide ? make_tmap(&p.tm_out, out, (uint64_t)cols, (uint64_t)rows, (uint64_t)ldo * 4, 32, 32, 128,
                          "C (four-byte)", CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
              : make_tmap(&p.tm_out, out, (uint64_t)cols, (uint64_t)rows, (uint64_t)ldo * 2, 64, 32, 128, "C (bf16)");
}

// 3-D map of the tiled 2:4 metadata: {64 words of a block, column blocks, row blocks}.
static nm_status make_meta_tmap(CUtensorMap* tm, const void* meta, int64_t rblocks, int64_t cblocks) {
  const TmapKey key{meta, 64, (uint64_t)cblocks, (uint64_t)rblocks, 256, (uint64_t)cblocks * 256, 64, 1, 8, 0,
                    (int)CU_TENSOR_MAP_DATA_TYPE_UINT32, 3};
  if (t_tmaps.find(key, tm)) return NM_OK;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {64, (cuuint64_t)cblocks, (cuuint64_t)rblocks};
  cuuint64_t strides[2] = {256, (cuuint64_t)cblocks * 256};
  cuuint32_t box[3] = {64, 1, 8};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(meta), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NM_ERR_CUDA, "cuTensorMapEncodeTiled(meta) failed with %d", (int)r);
  t_tmaps.put(key, *tm);
  return NM_OK;
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tile order of the SM-pair kernel: column tiles fastest when the compressed weights (R x vcols) exceed
// 1.5x the dense input (K x T; same element size), so that the weights stream from HBM about once.
static int pair_n_major(int64_t R, int64_t vcols, int64_t K, int64_t T) {
  return (double)R * (double)vcols > 1.5 * (double)K * (double)T ? 1 : 0;
}

// Store map of the SM-pair kernel's epilogue: bf16 Y in 64-column x 32-row boxes, 32-bit Y (fp32,
// or int32 accumulator bits) in 32 x 32 boxes; both 128-byte rows with the 128-byte swizzle.
// Store maps of the SM-pair epilogues: p.tm_y, and for bf16 Y also p.tm_y32
// (the last 32 columns of the double-buffered form's 224-column tiles).
static nm_status make_pair_store_maps(SpmmParams& p, void* Y, int64_t R, int64_t T, int64_t ldy, bool out32) {
  if (out32)
    return make_tmap(&p.tm_y, Y, (uint64_t)T, (uint64_t)R, (uint64_t)ldy * 4, 32, 32, 128, "Y (32-bit)",
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  nm_status st = make_tmap(&p.tm_y, Y, (uint64_t)T, (uint64_t)R, (uint64_t)ldy * 2, 64, 32, 128, "Y");
  if (st == NM_OK) st = make_tmap(&p.tm_y32, Y, (uint64_t)T, (uint64_t)R, (uint64_t)ldy * 2, 32, 32, 0, "Y (32 columns)");
  return st;
}

static int pattern_id(int n, int m) {
  if (n == 2 && m == 4) return PAT_2_4;
  if (n == 1 && m == 2) return PAT_1_2;
  if (n == 1 && m == 4) return PAT_1_4;
  if (n == 1 && m == 8) return PAT_1_8;
  if (n == 2 && m == 8) return PAT_2_8;
  return PAT_OTHER;
}

static int pick_bn(int64_t T) {
  int bn = 16;
  while (bn < T && bn < 256) bn *= 2;
  return bn;
}

struct GemmRequest {
  const uint16_t* values;
  const uint32_t* meta;
  int n, m;
  int64_t R, K, T;
  const int32_t* idx;
  const uint16_t* X;
  int64_t ldx;
  void* Y;
  int64_t ldy;
  int y_dtype;
  nm_algo algo;
  // hybrid
  bool hybrid;
  const uint16_t* W;
  int64_t ldw;
  const uint8_t* tile_map;
  int tile;
  // false: never stage anything (no re-encoded operand); used by the
  // allocation-free entry point for shapes it does not chunk itself
  bool allow_staging = true;
};

// Split of the K stages for the skinny kernel: the number of ranges that
// keeps the persistent CTAs best balanced (units per CTA / its ceiling), each
// range at least two stages, fewest ranges on ties.  Every range is non-empty.
static void choose_splits(SpmmParams& p, int sms) {
  const int64_t kt = p.k_tiles;
  int best_s = 1, best_kps = (int)kt;
  double best = -1.0;
  for (int s = 1; s <= 16 && s <= kt; ++s) {
    const int64_t kps = (kt + s - 1) / s;
    if (kps < 2 && s > 1) break;
    const int64_t se = (kt + kps - 1) / kps;  // ranges actually used
    const int64_t units = (int64_t)p.tiles_m * se;
    const int64_t waves = (units + sms - 1) / sms;
    const double eff = (double)units / (double)(waves * sms);
    if (eff > best + 1e-9) {
      best = eff;
      best_s = (int)se;
      best_kps = (int)kps;
    }
  }
  p.splits = best_s;
  p.kt_per_split = best_kps;
}

// Argument checks of the sparse GEMM calls, in three steps so that every
// entry point reports the same status and text for the same mistake:
// shape/pattern/dtype, then the output (and a usable device), then the operands.
static nm_status check_gemm_shape(const GemmRequest& q) {
  if (q.R < 0 || q.K < 0 || q.T < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (!pattern_ok(q.n, q.m)) return fail(NM_ERR_INVALID_ARG, "pattern %d:%d not supported (M in 2,4,8,16; 1<=N<M)", q.n, q.m);
  if (q.K % q.m != 0) return fail(NM_ERR_INVALID_ARG, "K=%lld is not a multiple of M=%d", (long long)q.K, q.m);
  if (q.y_dtype != NM_OUT_BF16 && q.y_dtype != NM_OUT_F32) return fail(NM_ERR_INVALID_ARG, "bad output dtype");
  if (q.algo != NM_ALGO_AUTO && q.algo != NM_ALGO_SPARSE_TC && q.algo != NM_ALGO_DENSE_TC)
    return fail(NM_ERR_INVALID_ARG, "bad algorithm");
  return NM_OK;
}

static nm_status check_gemm_output(const GemmRequest& q) {
  if (!q.Y) return fail(NM_ERR_INVALID_ARG, "Y is null");
  if (q.ldy < q.T) return fail(NM_ERR_INVALID_ARG, "ldy < T");
  const int esize = q.y_dtype == NM_OUT_F32 ? 4 : 2;
  if (!al16(q.Y) || (q.ldy * esize) % 16 != 0) return fail(NM_ERR_MISALIGNED, "Y rows must be 16-byte aligned");
  return require_device();
}

static nm_status check_gemm_operands(const GemmRequest& q) {
  if (!q.values || !q.meta || !q.X) return fail(NM_ERR_INVALID_ARG, "null operand");
  if (q.ldx < q.T) return fail(NM_ERR_INVALID_ARG, "ldx < T");
  if (!al16(q.X) || q.ldx % 8 != 0) return fail(NM_ERR_MISALIGNED, "X rows must be 16-byte aligned");
  if (q.R >= (1ll << 31) || q.K >= (1ll << 31) || q.T >= (1ll << 31))
    return fail(NM_ERR_UNSUPPORTED, "dimensions must stay below 2^31");
  return NM_OK;
}

static nm_status run_gemm(const GemmRequest& q, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_gemm_shape(q);
  if (st != NM_OK) return st;
  if (q.R == 0 || q.T == 0) return NM_OK;
  st = check_gemm_output(q);
  if (st != NM_OK) return st;
  const int esize = q.y_dtype == NM_OUT_F32 ? 4 : 2;
  if (q.K == 0) {
    cudaError_t e = launch_fill_zero(q.Y, q.R, q.T, q.ldy, esize, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  st = check_gemm_operands(q);
  if (st != NM_OK) return st;

  SpmmParams p;
  std::memset(&p, 0, sizeof p);
  p.vals = q.values;
  p.meta = q.meta;
  p.idx = q.idx;
  p.X = q.X;
  p.ldx = q.ldx;
  p.Y = q.Y;
  p.ldy = q.ldy;
  p.R = q.R;
  p.K = q.K;
  p.T = q.T;
  p.n = q.n;
  p.m = q.m;
  p.vcols = value_cols(q.K, q.n, q.m);
  p.mcols = meta_cols(q.K, q.n, q.m);
  p.meta_rblocks = meta_row_blocks(q.R);
  p.meta_cblocks = meta_col_blocks(q.K);
  p.pattern = pattern_id(q.n, q.m);
  p.permuted = q.idx != nullptr;
  p.out_f32 = q.y_dtype == NM_OUT_F32;

  const bool tma_values_ok = q.n == 2 && q.m == 4 && q.K % 16 == 0 && al16(q.values);
  if (q.hybrid) {
    if (q.tile != 128) return fail(NM_ERR_UNSUPPORTED, "hybrid tile must be 128");
    if (!q.W || !q.tile_map) return fail(NM_ERR_INVALID_ARG, "null hybrid operand");
    if (q.ldw < q.K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
    if (!tma_values_ok) return fail(NM_ERR_UNSUPPORTED, "hybrid needs K %% 16 == 0 and 16-byte aligned values");
    if (!al16(q.W) || q.ldw % 8 != 0) return fail(NM_ERR_MISALIGNED, "W rows must be 16-byte aligned");
    p.a_mode = A_HYBRID;
    p.tile_map = q.tile_map;
    p.hyb_tiles_k = (int)((q.K + 127) / 128);
  } else if (q.algo == NM_ALGO_DENSE_TC) {
    p.a_mode = A_BUILD_DENSE;
  } else if (tma_values_ok) {
    p.a_mode = A_TMA_SPARSE;
  } else if (fits_2of4(q.n, q.m)) {
    p.a_mode = A_BUILD_SPARSE;
  } else if (q.algo == NM_ALGO_AUTO) {
    p.a_mode = A_BUILD_DENSE;
  } else {
    return fail(NM_ERR_UNSUPPORTED, "pattern %d:%d does not fit the 2:4 sparse MMA", q.n, q.m);
  }

  p.status = status_word_ptr();
  if (!p.status) return fail(NM_ERR_CUDA, "device status word is unavailable");

  // Two SMs per 256 x 256 tile when the shape allows it (2:4 from TMA, K % 128 == 0).
  // Other patterns that fit the 2:4 MMA take the same kernel on shapes it
  // serves, after a re-encoding pass into a staged 2:4 operand.
  // PATCH hybrid on SM pairs: a stage runs the sparse MMA when both CTAs' 128 x 128
  // tiles are 2:4, else the dense MMA on W, with the 2:4 tiles taken from a staged
  // copy of W under the mask (one tile-filtered decompress pass).
  if (q.hybrid && q.allow_staging && q.K % 128 == 0 && q.T >= 192 && q.T % 8 == 0 && al16(q.meta)) {
    cudaMemPool_t pool = nullptr;
    cudaError_t e = staging_pool(&pool);
    if (e != cudaSuccess) return cuda_fail(e, "staging pool");
    void* wm = nullptr;
    e = cudaMallocFromPoolAsync(&wm, (size_t)(q.R * q.K * 2), pool, stream);
    if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the masked 2:4 tiles");
    e = launch_decompress_tiles(q.values, q.meta, q.R, q.K, q.tile_map, static_cast<uint16_t*>(wm), q.K, stream);
    if (e != cudaSuccess) {
      cudaFreeAsync(wm, stream);
      return cuda_fail(e, "masked-tile decompress launch");
    }
    p.tiles_m = (int)((q.R + 255) / 256);
    p.tiles_n = (int)((q.T + 255) / 256);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.k_tiles = q.K / 128;
    p.hyb_tiles_k = (int)(q.K / 128);
    p.hyb_rows = (int)((q.R + 127) / 128);
    st = make_tmap(&p.tm_x, q.X, (uint64_t)q.T, (uint64_t)q.K, (uint64_t)q.ldx * 2, 64, kPairBoxRows, 128, "X");
    if (st == NM_OK)
      st = make_tmap(&p.tm_vals, q.values, (uint64_t)p.vcols, (uint64_t)q.R, (uint64_t)p.vcols * 2, 64,
                     kPairBoxRows, 128, "values");
    if (st == NM_OK) st = make_meta_tmap(&p.tm_meta, q.meta, p.meta_rblocks, p.meta_cblocks);
    if (st == NM_OK)
      st = make_tmap(&p.tm_w, q.W, (uint64_t)q.K, (uint64_t)q.R, (uint64_t)q.ldw * 2, 64, kPairBoxRows, 128, "W");
    if (st == NM_OK)
      st = make_tmap(&p.tm_wm, wm, (uint64_t)q.K, (uint64_t)q.R, (uint64_t)q.K * 2, 64, kPairBoxRows, 128, "W masked");
    if (st == NM_OK) st = make_pair_store_maps(p, q.Y, q.R, q.T, q.ldy, p.out_f32 != 0);
    if (st == NM_OK) e = launch_spmm_pair_hybrid(p, stream);
    cudaFreeAsync(wm, stream);
    if (st != NM_OK) return st;
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "hybrid pair launch");
  }

  // Few columns (T <= 64): the split-K skinny kernel on the same staged operands.
  const bool pair_shape = q.K % 128 == 0 && q.T >= 192 && q.T % 8 == 0;
  const bool skinny_shape = q.K % 128 == 0 && skinny_kernel_fits(q.T) && q.allow_staging;
  const bool tma_2of4 = p.a_mode == A_TMA_SPARSE && al16(q.meta) && q.algo != NM_ALGO_DENSE_TC;
  const bool reencode = q.allow_staging && !q.hybrid && p.a_mode == A_BUILD_SPARSE && !(q.n == 2 && q.m == 4) &&
                        (pair_shape || skinny_shape);
  const bool use_skinny = skinny_shape && (tma_2of4 || reencode);
  // Dense design on SM pairs (NM_ALGO_DENSE_TC, or a pattern the 2:4 MMA cannot
  // take): decompress into a staged dense operand, then the pair kernel's dense stages.
  const bool dense_pair = q.allow_staging && !q.hybrid && p.a_mode == A_BUILD_DENSE && pair_shape;
  if (dense_pair || reencode || use_skinny || (q.algo != NM_ALGO_DENSE_TC && pair_kernel_fits(p) && al16(q.meta))) {
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaSuccess;
    const uint16_t* vals = q.values;
    const uint32_t* meta = q.meta;
    void* staged_a = nullptr;  // re-encoded values, then tiled metadata
    if (dense_pair) {
      e = staging_pool(&pool);
      if (e != cudaSuccess) return cuda_fail(e, "staging pool");
      e = cudaMallocFromPoolAsync(&staged_a, (size_t)(q.R * q.K * 2), pool, stream);
      if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the decompressed weights");
      e = launch_decompress(q.values, q.meta, q.R, q.K, q.n, q.m, static_cast<uint16_t*>(staged_a), q.K, stream);
      if (e != cudaSuccess) {
        cudaFreeAsync(staged_a, stream);
        return cuda_fail(e, "decompress launch");
      }
      p.tile_map = nullptr;
    } else if (reencode) {
      e = staging_pool(&pool);
      if (e != cudaSuccess) return cuda_fail(e, "staging pool");
      const size_t vbytes = (size_t)(q.R * (q.K / 2) * 2 + 255) / 256 * 256;
      const size_t mbytes = (size_t)meta_words(q.R, q.K, 2, 4) * 4;
      e = cudaMallocFromPoolAsync(&staged_a, vbytes + mbytes, pool, stream);
      if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the re-encoded weights");
      uint16_t* v2 = static_cast<uint16_t*>(staged_a);
      uint32_t* m2 = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(staged_a) + vbytes);
      e = launch_reencode_2of4(q.values, q.meta, q.R, q.K, q.n, q.m, v2, m2, stream);
      if (e != cudaSuccess) {
        cudaFreeAsync(staged_a, stream);
        return cuda_fail(e, "re-encode launch");
      }
      vals = v2;
      meta = m2;
      p.n = 2;
      p.m = 4;
      p.pattern = PAT_2_4;
      p.a_mode = A_TMA_SPARSE;
      p.vcols = q.K / 2;
      p.mcols = 0;
    }
    // With an index map, one gather pass stages Xp[k] = X[idx[k]] in a
    // stream-ordered buffer from the staging pool and the pair kernel streams
    // Xp with TMA boxes.
    const uint16_t* xsrc = q.X;
    int64_t ldsrc = q.ldx;
    void* staged = nullptr;
    auto release = [&]() {
      if (staged) cudaFreeAsync(staged, stream);
      if (staged_a) cudaFreeAsync(staged_a, stream);
    };
    if (p.permuted) {
      const int64_t ldp = (q.T + 7) / 8 * 8;
      if (!pool) e = staging_pool(&pool);
      if (e != cudaSuccess) {
        release();
        return cuda_fail(e, "staging pool");
      }
      e = cudaMallocFromPoolAsync(&staged, (size_t)(q.K * ldp * 2), pool, stream);
      if (e != cudaSuccess) {
        staged = nullptr;
        release();
        return cuda_fail(e, "staging buffer for the permuted input");
      }
      e = launch_gather_rows(q.X, q.ldx, q.idx, q.K, q.T, static_cast<uint16_t*>(staged), ldp, stream);
      if (e != cudaSuccess) {
        release();
        return cuda_fail(e, "gather launch");
      }
      xsrc = static_cast<const uint16_t*>(staged);
      ldsrc = ldp;
      p.permuted = 0;
    }
    p.k_tiles = q.K / 128;
    void* ws = nullptr;
    if (use_skinny) {
      p.bn = skinny_bn(q.T);
      p.kd = skinny_kd(q.K, q.T);
      p.k_tiles = q.K / p.kd;
      p.tiles_m = (int)((q.R + 127) / 128);
      if ((int64_t)p.tiles_m * p.k_tiles >= (1ll << 31)) {
        release();
        return fail(NM_ERR_UNSUPPORTED, "too many tiles");
      }
      choose_splits(p, sm_count_current());
      p.tiles_n = 1;
      p.num_tiles = p.tiles_m;
      if (p.splits > 1) {
        if (!pool) e = staging_pool(&pool);
        if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&ws, (size_t)p.splits * q.R * p.bn * 4, pool, stream);
        if (e != cudaSuccess) {
          ws = nullptr;
          release();
          return cuda_fail(e, "split-K workspace");
        }
        p.ws = static_cast<float*>(ws);
      }
      st = make_tmap(&p.tm_x, xsrc, (uint64_t)q.T, (uint64_t)q.K, (uint64_t)ldsrc * 2, (uint32_t)p.bn,
                     (uint32_t)p.kd, p.bn * 2, "X");
    } else {
      p.tiles_m = (int)((q.R + 255) / 256);
      p.tiles_n = (int)((q.T + 255) / 256);
      if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) {
        release();
        return fail(NM_ERR_UNSUPPORTED, "too many tiles");
      }
      p.num_tiles = p.tiles_m * p.tiles_n;
      st = make_tmap(&p.tm_x, xsrc, (uint64_t)q.T, (uint64_t)q.K, (uint64_t)ldsrc * 2, 64, kPairBoxRows, 128, "X");
    }
    if (st == NM_OK && dense_pair)
      st = make_tmap(&p.tm_w, staged_a, (uint64_t)q.K, (uint64_t)q.R, (uint64_t)q.K * 2, 64, kPairBoxRows, 128,
                     "decompressed W");
    if (st == NM_OK && !dense_pair)
      st = make_tmap(&p.tm_vals, vals, (uint64_t)p.vcols, (uint64_t)q.R, (uint64_t)p.vcols * 2, 64, kPairBoxRows,
                     128, "values");
    if (st == NM_OK && !dense_pair) st = make_meta_tmap(&p.tm_meta, meta, p.meta_rblocks, p.meta_cblocks);
    if (st == NM_OK && !use_skinny) st = make_pair_store_maps(p, q.Y, q.R, q.T, q.ldy, p.out_f32 != 0);
    if (!use_skinny && !dense_pair) p.n_major = pair_n_major(q.R, p.vcols, q.K, q.T);
    if (st == NM_OK)
      e = use_skinny   ? launch_spmm_skinny(p, stream)
          : dense_pair ? launch_spmm_pair_hybrid(p, stream)
                       : launch_spmm_pair(p, stream);
    if (ws) cudaFreeAsync(ws, stream);
    release();
    if (st != NM_OK) return st;
    return e == cudaSuccess ? NM_OK : cuda_fail(e, use_skinny ? "spmm skinny launch" : "spmm pair launch");
  }

  const int bn = pick_bn(q.T);
  const int bsw = bn >= 64 ? 128 : bn * 2;
  p.a_slot_bytes = (p.a_mode == A_BUILD_DENSE || p.a_mode == A_HYBRID) ? 16384u : 8192u;
  p.stages = spmm_max_stages(bn, p.a_slot_bytes);
  p.tiles_m = (int)((q.R + 127) / 128);
  p.tiles_n = (int)((q.T + bn - 1) / bn);
  if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "too many tiles");
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.k_tiles = (q.K + 63) / 64;

  st = make_tmap(&p.tm_x, q.X, (uint64_t)q.T, (uint64_t)q.K, (uint64_t)q.ldx * 2, bsw / 2, 64, bsw, "X");
  if (st != NM_OK) return st;
  if (p.a_mode == A_TMA_SPARSE || p.a_mode == A_HYBRID) {
    st = make_tmap(&p.tm_vals, q.values, (uint64_t)p.vcols, (uint64_t)q.R, (uint64_t)p.vcols * 2, 32, 128, 64,
                   "values");
    if (st != NM_OK) return st;
  }
  if (p.a_mode == A_HYBRID) {
    st = make_tmap(&p.tm_w, q.W, (uint64_t)q.K, (uint64_t)q.R, (uint64_t)q.ldw * 2, 64, 128, 128, "W");
    if (st != NM_OK) return st;
  }
  cudaError_t e = launch_spmm(p, bn, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "spmm launch");
}

// ---- helpers for entry points defined in other files (additive) ----
void set_last_error(const char* msg) { t_last_error = msg ? msg : ""; }

// nm_spmm_permuted for shapes the allocation-free call does not stage itself:
// the same kernels, but never a staged (re-encoded) operand.
nm_status spmm_permuted_unstaged(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                                 const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y,
                                 int64_t ldy, nm_out_dtype y_dtype, cudaStream_t stream) {
  if (!idx && R > 0 && K > 0 && T > 0) return fail(NM_ERR_INVALID_ARG, "idx is null");
  GemmRequest q{};
  q.values = values;
  q.meta = meta;
  q.n = n;
  q.m = m;
  q.R = R;
  q.K = K;
  q.T = T;
  q.idx = idx;
  q.X = X;
  q.ldx = ldx;
  q.Y = Y;
  q.ldy = ldy;
  q.y_dtype = (int)y_dtype;
  q.algo = NM_ALGO_AUTO;
  q.hybrid = false;
  q.allow_staging = false;
  return run_gemm(q, stream);
}

// The checks nm_spmm_permuted makes before it launches anything, for a shape
// with R, K, T > 0 (same statuses and texts).
nm_status check_permuted_args(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                              const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                              nm_out_dtype y_dtype) {
  t_last_error.clear();
  if (!idx) return fail(NM_ERR_INVALID_ARG, "idx is null");
  GemmRequest q{};
  q.values = values;
  q.meta = meta;
  q.n = n;
  q.m = m;
  q.R = R;
  q.K = K;
  q.T = T;
  q.idx = idx;
  q.X = X;
  q.ldx = ldx;
  q.Y = Y;
  q.ldy = ldy;
  q.y_dtype = (int)y_dtype;
  q.algo = NM_ALGO_AUTO;
  nm_status st = check_gemm_shape(q);
  if (st == NM_OK) st = check_gemm_output(q);
  if (st == NM_OK) st = check_gemm_operands(q);
  return st;
}

bool pair_path_for(int n, int m, int64_t R, int64_t K, int64_t T, const void* values, const void* meta) {
  SpmmParams p;
  std::memset(&p, 0, sizeof p);
  p.a_mode = (n == 2 && m == 4 && K % 16 == 0 && al16(values)) ? A_TMA_SPARSE : A_BUILD_SPARSE;
  p.R = R;
  p.K = K;
  p.T = T;
  return pair_kernel_fits(p) && al16(meta);
}

nm_status build_pair_params(SpmmParams& p, const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K,
                            const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy, bool out_f32) {
  std::memset(&p, 0, sizeof p);
  p.vals = values;
  p.meta = meta;
  p.X = X;
  p.ldx = ldx;
  p.Y = Y;
  p.ldy = ldy;
  p.R = R;
  p.K = K;
  p.T = T;
  p.n = 2;
  p.m = 4;
  p.vcols = value_cols(K, 2, 4);
  p.mcols = meta_cols(K, 2, 4);
  p.meta_rblocks = meta_row_blocks(R);
  p.meta_cblocks = meta_col_blocks(K);
  p.pattern = PAT_2_4;
  p.a_mode = A_TMA_SPARSE;
  p.out_f32 = out_f32 ? 1 : 0;
  p.status = status_word_ptr();
  if (!p.status) return fail(NM_ERR_CUDA, "device status word is unavailable");
  p.tiles_m = (int)((R + 255) / 256);
  p.tiles_n = (int)((T + 255) / 256);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.k_tiles = K / 128;
  nm_status st = make_tmap(&p.tm_x, X, (uint64_t)T, (uint64_t)K, (uint64_t)ldx * 2, 64, kPairBoxRows, 128, "X");
  if (st == NM_OK)
    st = make_tmap(&p.tm_vals, values, (uint64_t)p.vcols, (uint64_t)R, (uint64_t)p.vcols * 2, 64, kPairBoxRows, 128,
                   "values");
  if (st == NM_OK) st = make_meta_tmap(&p.tm_meta, meta, p.meta_rblocks, p.meta_cblocks);
  if (st == NM_OK) st = make_pair_store_maps(p, Y, R, T, ldy, out_f32);
  p.n_major = pair_n_major(R, p.vcols, K, T);
  return st;
}


// Prune + GEMM.  2:4 on skinny shapes: one fused kernel selects each W tile in
// shared memory and feeds the sparse MMA (W read from HBM once).  Otherwise:
// compress (into the caller's buffers or a staged pair), then the GEMM path.
static nm_status run_prune_gemm(const uint16_t* W, int64_t ldw, int n, int m, int64_t R, int64_t K,
                                const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                                nm_out_dtype y_dtype, uint16_t* values, uint32_t* meta, cudaStream_t stream) {
  t_last_error.clear();
  if (R < 0 || K < 0 || T < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (!pattern_ok(n, m)) return fail(NM_ERR_INVALID_ARG, "pattern %d:%d not supported", n, m);
  if (K % m != 0) return fail(NM_ERR_INVALID_ARG, "K=%lld is not a multiple of M=%d", (long long)K, m);
  if ((values == nullptr) != (meta == nullptr)) return fail(NM_ERR_INVALID_ARG, "values and meta: give both or neither");
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (y_dtype != NM_OUT_BF16 && y_dtype != NM_OUT_F32) return fail(NM_ERR_INVALID_ARG, "bad output dtype");
  if (R == 0) return NM_OK;
  if (K > 0 && !W) return fail(NM_ERR_INVALID_ARG, "W is null");
  if (T == 0 || K == 0) {
    nm_status st = values ? nm_prune_compress(W, R, K, ldw, n, m, values, meta, stream) : NM_OK;
    if (st != NM_OK || T == 0) return st;
    return nm_spmm_algo(nullptr, nullptr, n, m, R, K, nullptr, X, ldx, T, Y, ldy, y_dtype, NM_ALGO_AUTO, stream);
  }
  if (!X) return fail(NM_ERR_INVALID_ARG, "X is null");
  const bool fused = n == 2 && m == 4 && K % 128 == 0 && skinny_kernel_fits(T) && ldw % 8 == 0 && al16(W) &&
                     (!values || (al16(values) && al16(meta))) && R < (1ll << 31) && K < (1ll << 31);
  if (!fused) {
    void* staged = nullptr;
    uint16_t* v = values;
    uint32_t* mt = meta;
    if (!values) {
      cudaMemPool_t pool = nullptr;
      cudaError_t e = staging_pool(&pool);
      if (e != cudaSuccess) return cuda_fail(e, "staging pool");
      const size_t vbytes = (size_t)(R * value_cols(K, n, m) * 2 + 255) / 256 * 256;
      const size_t mbytes = (size_t)meta_words(R, K, n, m) * 4;
      e = cudaMallocFromPoolAsync(&staged, vbytes + mbytes, pool, stream);
      if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the compressed weights");
      v = static_cast<uint16_t*>(staged);
      mt = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(staged) + vbytes);
    }
    // 2:4 on SM-pair shapes with an index map: the compress grid also gathers
    // Xp[k] = X[idx[k]] (its selection is integer-bound and leaves HBM
    // bandwidth over), then the GEMM reads Xp like an unpermuted input.
    const bool combined = idx && X && n == 2 && m == 4 && K % 128 == 0 && T >= 192 && T % 8 == 0 &&
                          ldw % 8 == 0 && al16(W) && al16(v) && al16(mt) && al16(X) && ldx % 8 == 0 && ldx >= T &&
                          R < (1ll << 31) && K < (1ll << 31);
    nm_status st = NM_OK;
    if (combined) {
      st = require_device();
      void* xp = nullptr;
      cudaError_t e = cudaSuccess;
      if (st == NM_OK) {
        cudaMemPool_t pool = nullptr;
        e = staging_pool(&pool);
        if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&xp, (size_t)(K * T * 2), pool, stream);
        if (e != cudaSuccess) {
          xp = nullptr;
          st = cuda_fail(e, "staging buffer for the permuted input");
        }
      }
      CUtensorMap tm;
      if (st == NM_OK) st = make_tmap(&tm, W, (uint64_t)K, (uint64_t)R, (uint64_t)ldw * 2, 128, 16, 0, "W");
      uint32_t* status = status_word_ptr();
      if (st == NM_OK && !status) st = fail(NM_ERR_CUDA, "device status word is unavailable");
      if (st == NM_OK) {
        const GatherJob g{X, ldx, idx, K, T, static_cast<uint16_t*>(xp), T};
        e = launch_compress_stream(tm, R, K, v, mt, status, stream, &g);
        if (e != cudaSuccess) st = cuda_fail(e, "compress + gather launch");
      }
      if (st == NM_OK)
        st = nm_spmm_algo(v, mt, 2, 4, R, K, nullptr, static_cast<const uint16_t*>(xp), T, T, Y, ldy, y_dtype,
                          NM_ALGO_AUTO, stream);
      if (xp) cudaFreeAsync(xp, stream);
    } else {
      st = nm_prune_compress(W, R, K, ldw, n, m, v, mt, stream);
      if (st == NM_OK) st = nm_spmm_algo(v, mt, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype, NM_ALGO_AUTO, stream);
    }
    if (staged) cudaFreeAsync(staged, stream);
    return st;
  }

  // fused kernel: same argument rules as the GEMM calls
  if (!Y) return fail(NM_ERR_INVALID_ARG, "Y is null");
  if (ldy < T) return fail(NM_ERR_INVALID_ARG, "ldy < T");
  const int esize = y_dtype == NM_OUT_F32 ? 4 : 2;
  if (!al16(Y) || (ldy * esize) % 16 != 0) return fail(NM_ERR_MISALIGNED, "Y rows must be 16-byte aligned");
  if (!X) return fail(NM_ERR_INVALID_ARG, "X is null");
  if (ldx < T) return fail(NM_ERR_INVALID_ARG, "ldx < T");
  if (!al16(X) || ldx % 8 != 0) return fail(NM_ERR_MISALIGNED, "X rows must be 16-byte aligned");
  nm_status st = require_device();
  if (st != NM_OK) return st;

  SpmmParams p;
  std::memset(&p, 0, sizeof p);
  p.Y = Y;
  p.ldy = ldy;
  p.R = R;
  p.K = K;
  p.T = T;
  p.n = 2;
  p.m = 4;
  p.pattern = PAT_2_4;
  p.vcols = K / 2;
  p.meta_rblocks = meta_row_blocks(R);
  p.meta_cblocks = meta_col_blocks(K);
  p.out_f32 = y_dtype == NM_OUT_F32;
  p.out_vals = values;
  p.out_meta = meta;
  p.status = status_word_ptr();
  if (!p.status) return fail(NM_ERR_CUDA, "device status word is unavailable");
  p.bn = skinny_bn(T);
  p.kd = 128;
  p.k_tiles = K / 128;
  p.tiles_m = (int)((R + 127) / 128);
  if ((int64_t)p.tiles_m * p.k_tiles >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "too many tiles");
  choose_splits(p, sm_count_current());
  p.tiles_n = 1;
  p.num_tiles = p.tiles_m;

  cudaMemPool_t pool = nullptr;
  cudaError_t e = cudaSuccess;
  void* staged = nullptr;
  void* ws = nullptr;
  auto release = [&]() {
    if (staged) cudaFreeAsync(staged, stream);
    if (ws) cudaFreeAsync(ws, stream);
  };
  const uint16_t* xsrc = X;
  int64_t ldsrc = ldx;
  if (idx || p.splits > 1) {
    e = staging_pool(&pool);
    if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  }
  if (idx) {
    const int64_t ldp = (T + 7) / 8 * 8;
    e = cudaMallocFromPoolAsync(&staged, (size_t)(K * ldp * 2), pool, stream);
    if (e != cudaSuccess) {
      staged = nullptr;
      return cuda_fail(e, "staging buffer for the permuted input");
    }
    e = launch_gather_rows(X, ldx, idx, K, T, static_cast<uint16_t*>(staged), ldp, stream);
    if (e != cudaSuccess) {
      release();
      return cuda_fail(e, "gather launch");
    }
    xsrc = static_cast<const uint16_t*>(staged);
    ldsrc = ldp;
  }
  if (p.splits > 1) {
    e = cudaMallocFromPoolAsync(&ws, (size_t)p.splits * R * p.bn * 4, pool, stream);
    if (e != cudaSuccess) {
      ws = nullptr;
      release();
      return cuda_fail(e, "split-K workspace");
    }
    p.ws = static_cast<float*>(ws);
  }
  // W: one 128 x 128 box per stage, unswizzled (256-byte rows in shared memory)
  st = make_tmap(&p.tm_w, W, (uint64_t)K, (uint64_t)R, (uint64_t)ldw * 2, 128, 128, 0, "W");
  if (st == NM_OK)
    st = make_tmap(&p.tm_x, xsrc, (uint64_t)T, (uint64_t)K, (uint64_t)ldsrc * 2, (uint32_t)p.bn, 128, p.bn * 2, "X");
  if (st == NM_OK) e = launch_prune_spmm_skinny(p, stream);
  release();
  if (st != NM_OK) return st;
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "fused prune + GEMM launch");
}


// Backward products of y = (W' Pi) x on the dense SM-pair GEMM.
static nm_status check_bwd_common(int n, int m, int64_t R, int64_t K, int64_t T, nm_out_dtype dtype) {
  if (R < 0 || K < 0 || T < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (!pattern_ok(n, m)) return fail(NM_ERR_INVALID_ARG, "pattern %d:%d not supported", n, m);
  if (K % m != 0) return fail(NM_ERR_INVALID_ARG, "K=%lld is not a multiple of M=%d", (long long)K, m);
  if (dtype != NM_OUT_BF16 && dtype != NM_OUT_F32) return fail(NM_ERR_INVALID_ARG, "bad output dtype");
  if (R >= (1ll << 31) || K >= (1ll << 31) || T >= (1ll << 31))
    return fail(NM_ERR_UNSUPPORTED, "dimensions must stay below 2^31");
  return NM_OK;
}

static nm_status run_spmm_t(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                            const int32_t* idx, const uint16_t* dY, int64_t lddy, int64_t T, void* dX, int64_t lddx,
                            nm_out_dtype dtype, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_bwd_common(n, m, R, K, T, dtype);
  if (st != NM_OK) return st;
  if (K == 0 || T == 0) return NM_OK;
  if (!dX) return fail(NM_ERR_INVALID_ARG, "dX is null");
  if (lddx < T) return fail(NM_ERR_INVALID_ARG, "lddx < T");
  const int esize = dtype == NM_OUT_F32 ? 4 : 2;
  if (!al16(dX) || (lddx * esize) % 16 != 0) return fail(NM_ERR_MISALIGNED, "dX rows must be 16-byte aligned");
  st = require_device();
  if (st != NM_OK) return st;
  if (R == 0) {  // no rows of W': the gradient is zero
    cudaError_t e = launch_fill_zero(dX, K, T, lddx, esize, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  if (!values || !meta || !dY) return fail(NM_ERR_INVALID_ARG, "null operand");
  if (lddy < T) return fail(NM_ERR_INVALID_ARG, "lddy < T");
  if (!al16(dY) || lddy % 8 != 0) return fail(NM_ERR_MISALIGNED, "dY rows must be 16-byte aligned");
  // W' written out densely (R x ldk bf16, rows padded to 16 bytes) in a staging buffer
  cudaMemPool_t pool = nullptr;
  cudaError_t e = staging_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  const int64_t ldk = (K + 7) / 8 * 8;
  void* wd = nullptr;
  e = cudaMallocFromPoolAsync(&wd, (size_t)(R * ldk * 2), pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the decompressed weights");
  e = launch_decompress(values, meta, R, K, n, m, static_cast<uint16_t*>(wd), ldk, stream);
  DenseParams p;
  std::memset(&p, 0, sizeof p);
  p.M = K;
  p.N = T;
  p.Kr = R;
  p.k_tiles = (R + 127) / 128;
  p.tiles_m = (int)((K + 255) / 256);
  p.tiles_n = (int)((T + 255) / 256);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.status = status_word_ptr();
  p.out = dX;
  p.ldo = lddx;
  p.out_f32 = dtype == NM_OUT_F32;
  p.row_map = idx;
  p.rows_out = K;
  if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
  if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_a, wd, (uint64_t)K, (uint64_t)R, (uint64_t)ldk * 2, 64, 64, 128, "W' (dense)");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_b, dY, (uint64_t)T, (uint64_t)R, (uint64_t)lddy * 2, 64, 64, 128, "dY");
  if (e == cudaSuccess && st == NM_OK && !idx) st = set_store_map(p, dX, K, T, lddx, p.out_f32 != 0);
  if (e == cudaSuccess && st == NM_OK) e = launch_dense_pair(p, true, true, EPI_STORE, stream);
  cudaFreeAsync(wd, stream);
  if (st != NM_OK) return st;
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "transposed GEMM launch");
}

static nm_status run_sddmm(const uint32_t* meta, int n, int m, int64_t R, int64_t K, const int32_t* idx,
                           const uint16_t* dY, int64_t lddy, const uint16_t* X, int64_t ldx, int64_t T, void* dV,
                           nm_out_dtype dtype, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_bwd_common(n, m, R, K, T, dtype);
  if (st != NM_OK) return st;
  if (R == 0 || K == 0) return NM_OK;
  if (!dV || !meta) return fail(NM_ERR_INVALID_ARG, "null operand");
  const int esize = dtype == NM_OUT_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(dV) & (uintptr_t)(esize - 1)) != 0) return fail(NM_ERR_MISALIGNED, "dV misaligned");
  st = require_device();
  if (st != NM_OK) return st;
  const int64_t vcols = value_cols(K, n, m);
  if (T == 0) {  // an empty reduction: every gradient entry is zero
    cudaError_t e = launch_fill_zero(dV, R, vcols, vcols, esize, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  if (!dY || !X) return fail(NM_ERR_INVALID_ARG, "null operand");
  if (lddy < T || ldx < T) return fail(NM_ERR_INVALID_ARG, "leading dimension < T");
  if (!al16(dY) || lddy % 8 != 0 || !al16(X) || ldx % 8 != 0)
    return fail(NM_ERR_MISALIGNED, "dY and X rows must be 16-byte aligned");
  cudaError_t e = cudaSuccess;
  void* staged = nullptr;
  const uint16_t* xsrc = X;
  int64_t ldsrc = ldx;
  if (idx) {  // Xp[k] = X[idx[k]] staged once, then read as the K-major B operand
    cudaMemPool_t pool = nullptr;
    e = staging_pool(&pool);
    if (e != cudaSuccess) return cuda_fail(e, "staging pool");
    const int64_t ldp = (T + 7) / 8 * 8;
    e = cudaMallocFromPoolAsync(&staged, (size_t)(K * ldp * 2), pool, stream);
    if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the permuted input");
    e = launch_gather_rows(X, ldx, idx, K, T, static_cast<uint16_t*>(staged), ldp, stream);
    xsrc = static_cast<const uint16_t*>(staged);
    ldsrc = ldp;
  }
  DenseParams p;
  std::memset(&p, 0, sizeof p);
  p.M = R;
  p.N = K;
  p.Kr = T;
  p.k_tiles = (T + 127) / 128;
  p.tiles_m = (int)((R + 255) / 256);
  p.tiles_n = (int)((K + 255) / 256);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.status = status_word_ptr();
  p.out = dV;
  p.ldo = vcols;
  p.out_f32 = dtype == NM_OUT_F32;
  p.meta = meta;
  p.n = n;
  p.m = m;
  p.vcols = vcols;
  p.mcols = meta_cols(K, n, m);
  p.meta_cblocks = meta_col_blocks(K);
  p.vec_out = n == 2 && m == 4 && K % 16 == 0 && al16(dV);
  if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
  if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_a, dY, (uint64_t)T, (uint64_t)R, (uint64_t)lddy * 2, 64, 64, 128, "dY");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_b, xsrc, (uint64_t)T, (uint64_t)K, (uint64_t)ldsrc * 2, 64, 64, 128, "X");
  if (e == cudaSuccess && st == NM_OK) e = launch_dense_pair(p, false, false, EPI_SURVIVORS, stream);
  if (staged) cudaFreeAsync(staged, stream);
  if (st != NM_OK) return st;
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "value-gradient GEMM launch");
}


// INT8 2:4 (compress, decompress, GEMM on the decompressed operand).
static bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

static nm_status check_i8_shape(int64_t R, int64_t K) {
  if (R < 0 || K < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (K % 16 != 0) return fail(NM_ERR_UNSUPPORTED, "int8 calls need K %% 16 == 0 (K = %lld)", (long long)K);
  if (R >= (1ll << 31) || K >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "matrix too large for one call");
  return NM_OK;
}

static nm_status run_compress_i8(const int8_t* W, int64_t R, int64_t K, int64_t ldw, int8_t* values, uint32_t* meta,
                                 cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_i8_shape(R, K);
  if (st != NM_OK) return st;
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W || !values || !meta) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (!aligned_to(W, 8) || ldw % 8 != 0 || !aligned_to(values, 4) || !aligned_to(meta, 8))
    return fail(NM_ERR_MISALIGNED, "int8 compress: W rows 8-byte aligned, values 4-byte, meta 8-byte");
  st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e = launch_compress_i8(W, R, K, ldw, values, meta, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "int8 compress launch");
}

static nm_status run_decompress_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, int8_t* W_out,
                                   int64_t ldw, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_i8_shape(R, K);
  if (st != NM_OK) return st;
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W_out || !values || !meta) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (!aligned_to(W_out, 16) || ldw % 16 != 0 || !aligned_to(values, 8) || !aligned_to(meta, 4))
    return fail(NM_ERR_MISALIGNED, "int8 decompress: W_out rows 16-byte aligned, values 8-byte");
  st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e = launch_decompress_i8(values, meta, R, K, W_out, ldw, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "int8 decompress launch");
}

static nm_status run_spmm_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, const int8_t* X,
                             int64_t ldx, int64_t T, int32_t* Y, int64_t ldy, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_i8_shape(R, K);
  if (st != NM_OK) return st;
  if (T < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (R == 0 || T == 0) return NM_OK;
  if (!Y) return fail(NM_ERR_INVALID_ARG, "Y is null");
  if (ldy < T) return fail(NM_ERR_INVALID_ARG, "ldy < T");
  if (!al16(Y) || ldy % 4 != 0) return fail(NM_ERR_MISALIGNED, "Y rows must be 16-byte aligned");
  if (T >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "dimensions must stay below 2^31");
  st = require_device();
  if (st != NM_OK) return st;
  if (K == 0) {
    cudaError_t e = launch_fill_zero(Y, R, T, ldy, 4, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  if (!values || !meta || !X) return fail(NM_ERR_INVALID_ARG, "null operand");
  if (ldx < T) return fail(NM_ERR_INVALID_ARG, "ldx < T");
  if (!al16(X) || ldx % 16 != 0) return fail(NM_ERR_MISALIGNED, "X rows must be 16-byte aligned");
  if (!aligned_to(values, 8) || !aligned_to(meta, 4)) return fail(NM_ERR_MISALIGNED, "values must be 8-byte aligned");
  cudaMemPool_t pool = nullptr;
  cudaError_t e = staging_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  // The sparse tensor cores (kind::i8 on SM pairs) when the shape fills pair tiles: the tiled metadata is
  // re-laid out per row (R x K / 8 bytes staged) and the compressed values are read as they are.
  if (T >= 192 && K % 32 == 0 && al16(values) && R < (1ll << 31) && K < (1ll << 31)) {
    const int64_t rblocks128 = (R + 255) / 256 * 2, kblocks = (K + 255) / 256;
    void* em = nullptr;
    e = cudaMallocFromPoolAsync(&em, (size_t)(rblocks128 * kblocks * 4096), pool, stream);
    if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the int8 metadata");
    e = launch_relayout_meta_i8(meta, R, K, static_cast<uint32_t*>(em), rblocks128, stream);
    SpmmParams p;
    std::memset(&p, 0, sizeof p);
    p.R = R;
    p.K = K;
    p.T = T;
    p.n = 2;
    p.m = 4;
    p.Y = Y;
    p.ldy = ldy;
    p.out_f32 = 1;  // the int32 accumulator bits, stored unchanged
    p.a_mode = A_TMA_SPARSE;
    p.pattern = PAT_2_4;
    p.vcols = K / 2;
    p.meta_cblocks = kblocks;
    p.k_tiles = kblocks;
    p.tiles_m = (int)((R + 255) / 256);
    p.tiles_n = (int)((T + 255) / 256);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.status = status_word_ptr();
    if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
    if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
    if (e == cudaSuccess && st == NM_OK)
      st = make_tmap(&p.tm_vals, values, (uint64_t)(K / 2), (uint64_t)R, (uint64_t)(K / 2), 128, kPairBoxRows, 128,
                     "values (int8)", CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (e == cudaSuccess && st == NM_OK)
      st = make_tmap(&p.tm_x, X, (uint64_t)T, (uint64_t)K, (uint64_t)ldx, 128, kPairBoxRows, 128, "X (int8)",
                     CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (e == cudaSuccess && st == NM_OK)
      st = make_tmap(&p.tm_meta, em, 256, (uint64_t)(rblocks128 * kblocks * 16), 256, 256, 16, 0,
                     "metadata (int8 order)", CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (e == cudaSuccess && st == NM_OK) st = make_pair_store_maps(p, Y, R, T, ldy, true);
    p.n_major = pair_n_major(R, K / 2, K, T);
    if (e == cudaSuccess && st == NM_OK) e = launch_spmm_pair_i8(p, stream);
    cudaFreeAsync(em, stream);
    if (st != NM_OK) return st;
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "int8 sparse GEMM launch");
  }
  void* wd = nullptr;
  e = cudaMallocFromPoolAsync(&wd, (size_t)(R * K), pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the decompressed int8 weights");
  e = launch_decompress_i8(values, meta, R, K, static_cast<int8_t*>(wd), K, stream);
  DenseParams p;
  std::memset(&p, 0, sizeof p);
  p.M = R;
  p.N = T;
  p.Kr = K;
  p.k_tiles = (K + 255) / 256;
  p.tiles_m = (int)((R + 255) / 256);
  p.tiles_n = (int)((T + 255) / 256);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.status = status_word_ptr();
  p.out = Y;
  p.ldo = ldy;
  p.out_f32 = 1;  // the int32 accumulator bits, stored unchanged
  if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
  if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_a, wd, (uint64_t)K, (uint64_t)R, (uint64_t)K, 128, 64, 128, "W' (int8, dense)",
                   CU_TENSOR_MAP_DATA_TYPE_UINT8);
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_b, X, (uint64_t)T, (uint64_t)K, (uint64_t)ldx, 128, 64, 128, "X (int8)",
                   CU_TENSOR_MAP_DATA_TYPE_UINT8);
  if (e == cudaSuccess && st == NM_OK) st = set_store_map(p, Y, R, T, ldy, true);
  if (e == cudaSuccess && st == NM_OK) e = launch_dense_pair_i8(p, stream);
  cudaFreeAsync(wd, stream);
  if (st != NM_OK) return st;
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "int8 GEMM launch");
}


// TF32 path: 1:2 float32 weights, GEMM on a staged dense copy with the kind::tf32 pair kernel.
static nm_status check_tf32_shape(int64_t R, int64_t K) {
  if (R < 0 || K < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (K % 2 != 0) return fail(NM_ERR_INVALID_ARG, "K must be even (1:2)");
  if (R >= (1ll << 31) || K >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "dimensions must stay below 2^31");
  return NM_OK;
}

static nm_status run_compress_tf32(const float* W, int64_t R, int64_t K, int64_t ldw, float* values, uint32_t* meta,
                                   cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_tf32_shape(R, K);
  if (st != NM_OK) return st;
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W || !values || !meta) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (!aligned_to(W, 4) || !aligned_to(values, 4) || !aligned_to(meta, 4))
    return fail(NM_ERR_MISALIGNED, "float32 operands must be 4-byte aligned");
  st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e = launch_compress_tf32(W, R, K, ldw, values, meta, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "tf32 compress launch");
}

static nm_status run_decompress_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, float* W_out,
                                     int64_t ldw, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_tf32_shape(R, K);
  if (st != NM_OK) return st;
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W_out || !values || !meta) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (!aligned_to(W_out, 4) || !aligned_to(values, 4) || !aligned_to(meta, 4))
    return fail(NM_ERR_MISALIGNED, "float32 operands must be 4-byte aligned");
  st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e = launch_decompress_tf32(values, meta, R, K, W_out, ldw, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "tf32 decompress launch");
}

static nm_status run_spmm_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, const float* X,
                               int64_t ldx, int64_t T, void* Y, int64_t ldy, nm_out_dtype dtype, cudaStream_t stream) {
  t_last_error.clear();
  nm_status st = check_tf32_shape(R, K);
  if (st != NM_OK) return st;
  if (T < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (dtype != NM_OUT_BF16 && dtype != NM_OUT_F32) return fail(NM_ERR_INVALID_ARG, "bad output dtype");
  if (R == 0 || T == 0) return NM_OK;
  if (!Y) return fail(NM_ERR_INVALID_ARG, "Y is null");
  if (ldy < T) return fail(NM_ERR_INVALID_ARG, "ldy < T");
  const int esize = dtype == NM_OUT_F32 ? 4 : 2;
  if (!al16(Y) || (ldy * esize) % 16 != 0) return fail(NM_ERR_MISALIGNED, "Y rows must be 16-byte aligned");
  if (T >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "dimensions must stay below 2^31");
  st = require_device();
  if (st != NM_OK) return st;
  if (K == 0) {
    cudaError_t e = launch_fill_zero(Y, R, T, ldy, esize, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  if (!values || !meta || !X) return fail(NM_ERR_INVALID_ARG, "null operand");
  if (ldx < T) return fail(NM_ERR_INVALID_ARG, "ldx < T");
  if (!al16(X) || ldx % 4 != 0) return fail(NM_ERR_MISALIGNED, "X rows must be 16-byte aligned");
  if (!aligned_to(values, 4) || !aligned_to(meta, 4)) return fail(NM_ERR_MISALIGNED, "values must be 4-byte aligned");
  cudaMemPool_t pool = nullptr;
  cudaError_t e = staging_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  // The sparse tensor cores (kind::tf32 on SM pairs) when the shape fills pair tiles: the 1-bit row-wise
  // positions are re-laid out into the MMA's metadata order (R x K / 8 bytes staged) and the compressed
  // values are read as they are.
  if (T >= 192 && K % 8 == 0 && al16(values)) {
    const int64_t rblocks128 = (R + 255) / 256 * 2, kblocks = (K + 63) / 64;
    void* em = nullptr;
    e = cudaMallocFromPoolAsync(&em, (size_t)(rblocks128 * kblocks * 4096), pool, stream);
    if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the tf32 metadata");
    e = launch_relayout_meta_tf32(meta, R, K, static_cast<uint32_t*>(em), rblocks128, stream);
    SpmmParams p;
    std::memset(&p, 0, sizeof p);
    p.R = R;
    p.K = K;
    p.T = T;
    p.n = 1;
    p.m = 2;
    p.Y = Y;
    p.ldy = ldy;
    p.out_f32 = dtype == NM_OUT_F32;
    p.a_mode = A_TMA_SPARSE;
    p.pattern = PAT_1_2;
    p.vcols = K / 2;
    p.meta_cblocks = kblocks;
    p.k_tiles = kblocks;
    p.tiles_m = (int)((R + 255) / 256);
    p.tiles_n = (int)((T + 255) / 256);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.status = status_word_ptr();
    if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
    if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
    if (e == cudaSuccess && st == NM_OK)
      st = make_tmap(&p.tm_vals, values, (uint64_t)(K / 2), (uint64_t)R, (uint64_t)(K / 2) * 4, 32, kPairBoxRows, 128,
                     "values (float32)", CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
    if (e == cudaSuccess && st == NM_OK)
      st = make_tmap(&p.tm_x, X, (uint64_t)T, (uint64_t)K, (uint64_t)ldx * 4, 32, kPairBoxRows, kSwizzle128Atom32B,
                     "X (float32)", CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
    if (e == cudaSuccess && st == NM_OK)
      st = make_tmap(&p.tm_meta, em, 256, (uint64_t)(rblocks128 * kblocks * 16), 256, 256, 16, 0,
                     "metadata (tf32 order)", CU_TENSOR_MAP_DATA_TYPE_UINT8);
    if (e == cudaSuccess && st == NM_OK) st = make_pair_store_maps(p, Y, R, T, ldy, p.out_f32 != 0);
    p.n_major = pair_n_major(R, K / 2, K, T);
    if (e == cudaSuccess && st == NM_OK) e = launch_spmm_pair_tf32(p, stream);
    cudaFreeAsync(em, stream);
    if (st != NM_OK) return st;
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "tf32 sparse GEMM launch");
  }
  const int64_t ldk = (K + 3) / 4 * 4;  // 16-byte rows for the TMA
  void* wd = nullptr;
  e = cudaMallocFromPoolAsync(&wd, (size_t)(R * ldk * 4), pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the decompressed float32 weights");
  e = launch_decompress_tf32(values, meta, R, K, static_cast<float*>(wd), ldk, stream);
  DenseParams p;
  std::memset(&p, 0, sizeof p);
  p.M = R;
  p.N = T;
  p.Kr = K;
  p.k_tiles = (K + 63) / 64;
  p.tiles_m = (int)((R + 255) / 256);
  p.tiles_n = (int)((T + 255) / 256);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.status = status_word_ptr();
  p.out = Y;
  p.ldo = ldy;
  p.out_f32 = dtype == NM_OUT_F32;
  if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
  if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_a, wd, (uint64_t)K, (uint64_t)R, (uint64_t)ldk * 4, 32, 64, 128, "W' (float32, dense)",
                   CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_b, X, (uint64_t)T, (uint64_t)K, (uint64_t)ldx * 4, 32, 64, kSwizzle128Atom32B,
                   "X (float32)", CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  if (e == cudaSuccess && st == NM_OK) st = set_store_map(p, Y, R, T, ldy, p.out_f32 != 0);
  if (e == cudaSuccess && st == NM_OK) e = launch_dense_pair_tf32(p, stream);
  cudaFreeAsync(wd, stream);
  if (st != NM_OK) return st;
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "tf32 GEMM launch");
}

// Diagonal sparsity: selection + gather, dense copy, GEMM on the dense copy.
static nm_status run_diag_prune_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D,
                                         int32_t* offsets, uint16_t* values, cudaStream_t stream) {
  t_last_error.clear();
  if (R < 0 || K < 0 || D < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (D > K) return fail(NM_ERR_INVALID_ARG, "D > K");
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (K == 0 || D == 0) return NM_OK;
  if (!W || !offsets || (R > 0 && !values)) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (R >= (1ll << 31) || K >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "matrix too large for one call");
  if (K > 65535ll * 256) return fail(NM_ERR_UNSUPPORTED, "K > 16776960 (the rank grid's offset tiles)");
  nm_status st = require_device();
  if (st != NM_OK) return st;
  cudaMemPool_t pool = nullptr;
  cudaError_t e = staging_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  void* buf = nullptr;
  const size_t pbytes = (size_t)(((R + 31) / 32 * K * 4 + 255) / 256 * 256);
  const size_t sbytes = (size_t)((K * 4 + 255) / 256 * 256);
  e = cudaMallocFromPoolAsync(&buf, pbytes + sbytes + (size_t)K * 4, pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the diagonal scores");
  uint8_t* b8 = static_cast<uint8_t*>(buf);
  e = launch_diag_select(W, R, K, ldw, D, reinterpret_cast<float*>(b8), reinterpret_cast<float*>(b8 + pbytes),
                         b8 + pbytes + sbytes, offsets, values, stream);
  cudaFreeAsync(buf, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "diagonal selection launch");
}

static nm_status run_diag_expand(const uint16_t* values, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                                 uint16_t* W_out, int64_t ldw, cudaStream_t stream) {
  t_last_error.clear();
  if (R < 0 || K < 0 || D < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (D > K || ldw < K) return fail(NM_ERR_INVALID_ARG, "D > K or ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W_out || (D > 0 && (!values || !offsets))) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (R >= (1ll << 31) || K >= (1ll << 31)) return fail(NM_ERR_UNSUPPORTED, "matrix too large for one call");
  nm_status st = require_device();
  if (st != NM_OK) return st;
  if (D == 0) {
    cudaError_t e = launch_fill_zero(W_out, R, K, ldw, 2, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  cudaMemPool_t pool = nullptr;
  cudaError_t e = staging_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  void* tables = nullptr;
  e = cudaMallocFromPoolAsync(&tables, (size_t)diag_table_words(K, false) * 4, pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the diagonal table");
  e = launch_diag_dense(values, offsets, D, R, K, nullptr, static_cast<int32_t*>(tables), W_out, ldw, stream, nullptr);
  cudaFreeAsync(tables, stream);
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "diagonal expand launch");
}

static nm_status run_diag_spmm(const uint16_t* values, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                               const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                               nm_out_dtype dtype, cudaStream_t stream) {
  t_last_error.clear();
  if (R < 0 || K < 0 || D < 0 || T < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (D > K) return fail(NM_ERR_INVALID_ARG, "D > K");
  if (dtype != NM_OUT_BF16 && dtype != NM_OUT_F32) return fail(NM_ERR_INVALID_ARG, "bad output dtype");
  if (R == 0 || T == 0) return NM_OK;
  if (!Y) return fail(NM_ERR_INVALID_ARG, "Y is null");
  if (ldy < T) return fail(NM_ERR_INVALID_ARG, "ldy < T");
  const int esize = dtype == NM_OUT_F32 ? 4 : 2;
  if (!al16(Y) || (ldy * esize) % 16 != 0) return fail(NM_ERR_MISALIGNED, "Y rows must be 16-byte aligned");
  if (R >= (1ll << 31) || K >= (1ll << 31) || T >= (1ll << 31))
    return fail(NM_ERR_UNSUPPORTED, "dimensions must stay below 2^31");
  nm_status st = require_device();
  if (st != NM_OK) return st;
  if (K == 0 || D == 0) {
    cudaError_t e = launch_fill_zero(Y, R, T, ldy, esize, stream);
    return e == cudaSuccess ? NM_OK : cuda_fail(e, "zero fill");
  }
  if (!values || !offsets || !X) return fail(NM_ERR_INVALID_ARG, "null operand");
  if (ldx < T) return fail(NM_ERR_INVALID_ARG, "ldx < T");
  if (!al16(X) || ldx % 8 != 0) return fail(NM_ERR_MISALIGNED, "X rows must be 16-byte aligned");
  cudaMemPool_t pool = nullptr;
  cudaError_t e = staging_pool(&pool);
  if (e != cudaSuccess) return cuda_fail(e, "staging pool");
  // Staging: the dense copy (R x ceil8(K)) with its lookup tables, and with idx
  // a gathered X[idx] that the gather pass fills only when idx is not a
  // permutation (otherwise the copy's columns are placed through idx and the
  // GEMM reads X itself; the device-side check decides at run time).
  const int64_t ldk = (K + 7) / 8 * 8;
  const size_t wbytes = (size_t)((R * ldk * 2 + 255) / 256 * 256);
  void* wd = nullptr;
  void* xp = nullptr;
  e = cudaMallocFromPoolAsync(&wd, wbytes + (size_t)diag_table_words(K, idx != nullptr) * 4, pool, stream);
  if (e != cudaSuccess) return cuda_fail(e, "staging buffer for the dense diagonal operand");
  const uint32_t* is_perm = nullptr;
  e = launch_diag_dense(values, offsets, D, R, K, idx, reinterpret_cast<int32_t*>(static_cast<uint8_t*>(wd) + wbytes),
                        static_cast<uint16_t*>(wd), ldk, stream, &is_perm);
  const uint16_t* xsrc = X;
  int64_t ldsrc = ldx;
  if (e == cudaSuccess && idx) {
    const int64_t ldp = (T + 7) / 8 * 8;
    e = cudaMallocFromPoolAsync(&xp, (size_t)(K * ldp * 2), pool, stream);
    if (e == cudaSuccess)
      e = launch_gather_rows(X, ldx, idx, K, T, static_cast<uint16_t*>(xp), ldp, stream, is_perm);
    xsrc = static_cast<const uint16_t*>(xp);
    ldsrc = ldp;
  }
  DenseParams p;
  std::memset(&p, 0, sizeof p);
  p.M = R;
  p.N = T;
  p.Kr = K;
  p.k_tiles = (K + 127) / 128;
  p.tiles_m = (int)((R + 255) / 256);
  p.tiles_n = (int)((T + 255) / 256);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.status = status_word_ptr();
  p.out = Y;
  p.ldo = ldy;
  p.out_f32 = dtype == NM_OUT_F32;
  if (e == cudaSuccess && !p.status) e = cudaErrorInvalidSymbol;
  if ((int64_t)p.tiles_m * p.tiles_n >= (1ll << 31)) st = fail(NM_ERR_UNSUPPORTED, "too many tiles");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_a, wd, (uint64_t)K, (uint64_t)R, (uint64_t)ldk * 2, 64, 64, 128, "diagonal operand (dense)");
  if (e == cudaSuccess && st == NM_OK)
    st = make_tmap(&p.tm_b, xsrc, (uint64_t)T, (uint64_t)K, (uint64_t)ldsrc * 2, 64, 64, 128, "X");
  if (e == cudaSuccess && st == NM_OK && idx) {
    st = make_tmap(&p.tm_b_alt, X, (uint64_t)T, (uint64_t)K, (uint64_t)ldx * 2, 64, 64, 128, "X (direct)");
    p.use_alt = is_perm;
  }
  if (e == cudaSuccess && st == NM_OK) st = set_store_map(p, Y, R, T, ldy, p.out_f32 != 0);
  if (e == cudaSuccess && st == NM_OK) e = launch_dense_pair(p, false, true, EPI_STORE, stream);
  cudaFreeAsync(wd, stream);
  if (xp) cudaFreeAsync(xp, stream);
  if (st != NM_OK) return st;
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "diagonal GEMM launch");
}

}  // namespace nmk

using namespace nmk;

extern "C" {

int nm_index_bits(int m) { return index_bits(m); }

int64_t nm_value_cols(int64_t K, int n, int m) {
  if (!pattern_ok(n, m) || K < 0 || K % m != 0) return -1;
  return value_cols(K, n, m);
}

int64_t nm_meta_words(int64_t R, int64_t K, int n, int m) {
  if (!pattern_ok(n, m) || R < 0 || K < 0 || K % m != 0) return -1;
  return meta_words(R, K, n, m);
}

nm_status nm_prune_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int n, int m, uint16_t* values,
                            uint32_t* meta, void* stream) {
  t_last_error.clear();
  if (R < 0 || K < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (!pattern_ok(n, m)) return fail(NM_ERR_INVALID_ARG, "pattern %d:%d not supported", n, m);
  if (K % m != 0) return fail(NM_ERR_INVALID_ARG, "K=%lld is not a multiple of M=%d", (long long)K, m);
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W || !values || !meta) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (R >= (1ll << 31) || K >= (1ll << 31) || meta_words(R, K, n, m) >= (1ll << 31))
    return fail(NM_ERR_UNSUPPORTED, "matrix too large for one call");
  nm_status st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e;
  if (tiled_meta(n, m) && K % 8 == 0 && ldw % 8 == 0 && al16(W) && al16(values) && al16(meta)) {
    // 2:4 on aligned rows: the TMA-fed stream kernel (16-row x 128-column boxes)
    CUtensorMap tm;
    st = make_tmap(&tm, W, (uint64_t)K, (uint64_t)R, (uint64_t)ldw * 2, 128, 16, 0, "W");
    if (st != NM_OK) return st;
    uint32_t* status = status_word_ptr();
    if (!status) return fail(NM_ERR_CUDA, "device status word is unavailable");
    e = launch_compress_stream(tm, R, K, values, meta, status, static_cast<cudaStream_t>(stream));
  } else {
    e = launch_compress(W, R, K, ldw, n, m, values, meta, static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "compress launch");
}

nm_status nm_decompress(const uint16_t* values, const uint32_t* meta, int64_t R, int64_t K, int n, int m,
                        uint16_t* W_out, int64_t ldw, void* stream) {
  t_last_error.clear();
  if (R < 0 || K < 0) return fail(NM_ERR_INVALID_ARG, "negative dimension");
  if (!pattern_ok(n, m)) return fail(NM_ERR_INVALID_ARG, "pattern %d:%d not supported", n, m);
  if (K % m != 0) return fail(NM_ERR_INVALID_ARG, "K=%lld is not a multiple of M=%d", (long long)K, m);
  if (ldw < K) return fail(NM_ERR_INVALID_ARG, "ldw < K");
  if (R == 0 || K == 0) return NM_OK;
  if (!W_out || !values || !meta) return fail(NM_ERR_INVALID_ARG, "null pointer");
  if (R >= (1ll << 31) || K >= (1ll << 31) || meta_words(R, K, n, m) >= (1ll << 31))
    return fail(NM_ERR_UNSUPPORTED, "matrix too large for one call");
  nm_status st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e = launch_decompress(values, meta, R, K, n, m, W_out, ldw, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "decompress launch");
}

nm_status nm_spmm_algo(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                       const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                       nm_out_dtype y_dtype, nm_algo algo, void* stream) {
  GemmRequest q{};
  q.values = values;
  q.meta = meta;
  q.n = n;
  q.m = m;
  q.R = R;
  q.K = K;
  q.T = T;
  q.idx = idx;
  q.X = X;
  q.ldx = ldx;
  q.Y = Y;
  q.ldy = ldy;
  q.y_dtype = (int)y_dtype;
  q.algo = algo;
  q.hybrid = false;
  return run_gemm(q, static_cast<cudaStream_t>(stream));
}

nm_status nm_spmm(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                  const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype,
                  void* stream) {
  return nm_spmm_algo(values, meta, n, m, R, K, nullptr, X, ldx, T, Y, ldy, y_dtype, NM_ALGO_AUTO, stream);
}

nm_status nm_spmm_permuted(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                           const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                           nm_out_dtype y_dtype, void* stream) {
  if (!idx && R > 0 && K > 0 && T > 0) return fail(NM_ERR_INVALID_ARG, "idx is null");
  return nm_spmm_algo(values, meta, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype, NM_ALGO_AUTO, stream);
}

nm_status nm_hybrid_spmm(const uint16_t* W, int64_t ldw, const uint16_t* values, const uint32_t* meta,
                         const uint8_t* tile_map, int tile, int64_t R, int64_t K, const uint16_t* X, int64_t ldx,
                         int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype, void* stream) {
  GemmRequest q{};
  q.values = values;
  q.meta = meta;
  q.n = 2;
  q.m = 4;
  q.R = R;
  q.K = K;
  q.T = T;
  q.idx = nullptr;
  q.X = X;
  q.ldx = ldx;
  q.Y = Y;
  q.ldy = ldy;
  q.y_dtype = (int)y_dtype;
  q.algo = NM_ALGO_AUTO;
  q.hybrid = true;
  q.W = W;
  q.ldw = ldw;
  q.tile_map = tile_map;
  q.tile = tile;
  return run_gemm(q, static_cast<cudaStream_t>(stream));
}

nm_status nm_prune_spmm(const uint16_t* W, int64_t ldw, int n, int m, int64_t R, int64_t K, const int32_t* idx,
                        const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype,
                        uint16_t* values, uint32_t* meta, void* stream) {
  return run_prune_gemm(W, ldw, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype, values, meta,
                        static_cast<cudaStream_t>(stream));
}

nm_status nm_spmm_t(const uint16_t* values, const uint32_t* meta, int n, int m, int64_t R, int64_t K,
                    const int32_t* idx, const uint16_t* dY, int64_t lddy, int64_t T, void* dX, int64_t lddx,
                    nm_out_dtype dtype, void* stream) {
  return run_spmm_t(values, meta, n, m, R, K, idx, dY, lddy, T, dX, lddx, dtype, static_cast<cudaStream_t>(stream));
}

nm_status nm_sddmm(const uint32_t* meta, int n, int m, int64_t R, int64_t K, const int32_t* idx, const uint16_t* dY,
                   int64_t lddy, const uint16_t* X, int64_t ldx, int64_t T, void* dV, nm_out_dtype dtype,
                   void* stream) {
  return run_sddmm(meta, n, m, R, K, idx, dY, lddy, X, ldx, T, dV, dtype, static_cast<cudaStream_t>(stream));
}

nm_status nm_prune_compress_i8(const int8_t* W, int64_t R, int64_t K, int64_t ldw, int8_t* values, uint32_t* meta,
                               void* stream) {
  return run_compress_i8(W, R, K, ldw, values, meta, static_cast<cudaStream_t>(stream));
}

nm_status nm_decompress_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, int8_t* W_out,
                           int64_t ldw, void* stream) {
  return run_decompress_i8(values, meta, R, K, W_out, ldw, static_cast<cudaStream_t>(stream));
}

nm_status nm_spmm_i8(const int8_t* values, const uint32_t* meta, int64_t R, int64_t K, const int8_t* X, int64_t ldx,
                     int64_t T, int32_t* Y, int64_t ldy, void* stream) {
  return run_spmm_i8(values, meta, R, K, X, ldx, T, Y, ldy, static_cast<cudaStream_t>(stream));
}

nm_status nm_prune_compress_tf32(const float* W, int64_t R, int64_t K, int64_t ldw, float* values, uint32_t* meta,
                                 void* stream) {
  return run_compress_tf32(W, R, K, ldw, values, meta, static_cast<cudaStream_t>(stream));
}

nm_status nm_decompress_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, float* W_out, int64_t ldw,
                             void* stream) {
  return run_decompress_tf32(values, meta, R, K, W_out, ldw, static_cast<cudaStream_t>(stream));
}

nm_status nm_spmm_tf32(const float* values, const uint32_t* meta, int64_t R, int64_t K, const float* X, int64_t ldx,
                       int64_t T, void* Y, int64_t ldy, nm_out_dtype y_dtype, void* stream) {
  return run_spmm_tf32(values, meta, R, K, X, ldx, T, Y, ldy, y_dtype, static_cast<cudaStream_t>(stream));
}

nm_status nm_diag_prune_compress(const uint16_t* W, int64_t R, int64_t K, int64_t ldw, int64_t D, int32_t* offsets,
                                 uint16_t* values, void* stream) {
  return run_diag_prune_compress(W, R, K, ldw, D, offsets, values, static_cast<cudaStream_t>(stream));
}

nm_status nm_diag_expand(const uint16_t* values, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                         uint16_t* W_out, int64_t ldw, void* stream) {
  return run_diag_expand(values, offsets, D, R, K, W_out, ldw, static_cast<cudaStream_t>(stream));
}

nm_status nm_diag_spmm(const uint16_t* values, const int32_t* offsets, int64_t D, int64_t R, int64_t K,
                       const int32_t* idx, const uint16_t* X, int64_t ldx, int64_t T, void* Y, int64_t ldy,
                       nm_out_dtype dtype, void* stream) {
  return run_diag_spmm(values, offsets, D, R, K, idx, X, ldx, T, Y, ldy, dtype, static_cast<cudaStream_t>(stream));
}

nm_status nm_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  e = read_and_clear_status(&word);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word & 1u) return fail(NM_ERR_TIMEOUT, "a kernel's bounded wait gave up");
  return NM_OK;
}

const char* nm_status_string(nm_status s) {
  switch (s) {
    case NM_OK: return "ok";
    case NM_ERR_INVALID_ARG: return "invalid argument";
    case NM_ERR_UNSUPPORTED: return "unsupported";
    case NM_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case NM_ERR_CUDA: return "CUDA error";
    case NM_ERR_TIMEOUT: return "bounded wait gave up";
    case NM_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

const char* nm_last_error(void) { return t_last_error.c_str(); }

uint64_t nm_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int nm_version(void) { return 100; }

nm_status nm_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  t_last_error.clear();
  if (limit_us < 1 || limit_us > 1000000) return fail(NM_ERR_INVALID_ARG, "limit_us must be in [1, 1000000]");
  nm_status st = require_device();
  if (st != NM_OK) return st;
  cudaError_t e = launch_selftest_wait((uint64_t)limit_us * 1000ull, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NM_OK : cuda_fail(e, "self-test launch");
}

nm_status nm_release_staging(void) {
  set_last_error("");
  std::lock_guard<std::mutex> lk(g_pool_mu);
  for (int d = 0; d < 64; ++d) {
    if (!g_pool[d]) continue;
    cudaError_t e = cudaMemPoolTrimTo(g_pool[d], 0);
    if (e != cudaSuccess) return cuda_fail(e, "trimming the staging pool");
  }
  return NM_OK;
}

}  // extern "C"
