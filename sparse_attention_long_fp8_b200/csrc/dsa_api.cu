// Host side of the DSA C ABI (include/dsa.h): argument validation, tile
// dispatch, TMA descriptor set-up and launches on the caller's stream.
// One translation unit holds every kernel so the device error word is a
// single symbol per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdarg>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/dsa.h"
#include "indexer.cuh"
#include "indexer_topk.cuh"
#include "sparse_attn.cuh"
#include "sparse_attn_vh.cuh"
#include "topk.cuh"
#include "selftest.cuh"
#include "quantize.cuh"
#include "indexer_kl.cuh"

namespace {

thread_local std::string g_last_error;

dsa_status fail(dsa_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
dsa_status fail(dsa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

dsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define DSA_CUDA_TRY(expr, what)                 \
  do {                                           \
    cudaError_t e_ = (expr);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

constexpr int kMaxDevices = 64;
// SM count assumed when no device is current (host-only size queries).
constexpr int kDefaultSms = 148;

// SM count of the current device, read once per device. It sizes grids and
// decides the split plans, so dsa_workspace_size and the launches that use
// the workspace see the same value on the same device.
int num_sms() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();   // no device: clear the non-sticky error
    return kDefaultSms;
  }
  static std::atomic<int> sms[kMaxDevices];
  int n = sms[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = kDefaultSms;
    }
    sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// ------------------------------------------------------------------ device check

dsa_status current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail(DSA_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  if (*dev < 0 || *dev >= kMaxDevices) return fail(DSA_ERR_NO_DEVICE, "device ordinal out of range");
  // Cached per device; host threads may race to fill it, with equal values.
  static std::atomic<int> major[kMaxDevices];
  int mj = major[*dev].load(std::memory_order_relaxed);
  if (mj == 0) {
    cudaDeviceGetAttribute(&mj, cudaDevAttrComputeCapabilityMajor, *dev);
    major[*dev].store(mj, std::memory_order_relaxed);
  }
  if (mj != 10)
    return fail(DSA_ERR_NO_DEVICE, "device %d is sm_%d0, this library is built for sm_100a", *dev,
                mj);
  return DSA_OK;
}

// ------------------------------------------------------------------ TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D byte tensor [rows, row_bytes] with a box of [box_rows, row_bytes] and the
// swizzle that matches the row width (32, 64 or 128 bytes).
dsa_status make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes,
                        uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {row_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DSA_OK;
}

// 2D byte tensor [rows, row_bytes] with a box of [box_rows, 128 bytes] and
// the 128-byte swizzle (the attention's output stores).
dsa_status make_tmap_rows128(CUtensorMap* map, void* base, uint64_t rows, uint32_t row_bytes,
                             uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DSA_OK;
}

// ------------------------------------------------------------------ validation

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

dsa_status check_shape_common(const dsa_shape* s) {
  if (!s) return fail(DSA_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 1 || s->n_q < 1 || s->n_kv < 1)
    return fail(DSA_ERR_INVALID_ARG, "batch, n_q and n_kv must be >= 1 (got %d, %d, %d)",
                s->batch, s->n_q, s->n_kv);
  if (static_cast<int64_t>(s->batch) * s->n_q > (1ll << 30) ||
      static_cast<int64_t>(s->batch) * s->n_kv > (1ll << 30))
    return fail(DSA_ERR_INVALID_ARG, "batch * rows exceeds 2^30");
  return DSA_OK;
}

dsa_status check_indexer_shape(const dsa_shape* s) {
  if (dsa_status st = check_shape_common(s)) return st;
  const bool ok = (s->idx_heads == 64 && s->idx_dim == 128) || (s->idx_heads == 4 && s->idx_dim == 32);
  if (!ok)
    return fail(DSA_ERR_UNSUPPORTED, "indexer shape (H^I=%d, d^I=%d) is not compiled in; supported: (64,128), (4,32)",
                s->idx_heads, s->idx_dim);
  if (static_cast<int64_t>(s->batch) * s->n_q * s->idx_heads >= (1ll << 31))
    return fail(DSA_ERR_INVALID_ARG, "batch * n_q * H^I exceeds the TMA coordinate range");
  return DSA_OK;
}

dsa_status check_topk_shape(const dsa_shape* s) {
  if (dsa_status st = check_shape_common(s)) return st;
  if (s->topk < 1) return fail(DSA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", s->topk);
  if (static_cast<int64_t>(s->batch) * s->n_q * s->topk >= (1ll << 40))
    return fail(DSA_ERR_INVALID_ARG, "index array too large");
  return DSA_OK;
}

dsa_status check_attn_shape(const dsa_shape* s) {
  if (dsa_status st = check_topk_shape(s)) return st;
  const bool big = s->qk_dim == 576 && s->v_dim == 512;
  const bool tiny = s->qk_dim == 64 && s->v_dim == 64;
  if (!big && !tiny)
    return fail(DSA_ERR_UNSUPPORTED, "(qk_dim=%d, v_dim=%d) is not compiled in; supported: (576,512), (64,64)",
                s->qk_dim, s->v_dim);
  if (s->heads < 1 || s->heads > 128)
    return fail(DSA_ERR_UNSUPPORTED, "heads must be in [1, 128] (got %d)", s->heads);
  if (!(std::isfinite(s->softmax_scale)))
    return fail(DSA_ERR_INVALID_ARG, "softmax_scale must be finite");
  return DSA_OK;
}

// ------------------------------------------------------------------ layouts

// Key rows and query positions of one call (dsa_layout, or the contiguous
// default when it is NULL).
struct HostLayout {
  dsa::KeyMap km;
  const int32_t* row_pos;
};

dsa_status resolve_layout(const dsa_shape* s, const dsa_layout* L, HostLayout* out) {
  out->row_pos = L ? L->row_pos : nullptr;
  out->km.block_table = nullptr;
  out->km.max_pages = 0;
  out->km.page_shift = 0;
  out->km.pool_rows = static_cast<int64_t>(s->batch) * s->n_kv;
  if (out->row_pos && reinterpret_cast<uintptr_t>(out->row_pos) % 4)
    return fail(DSA_ERR_INVALID_ARG, "row_pos must be 4-byte aligned");
  if (!L || !L->block_table) return DSA_OK;
  const int32_t page = L->page_size;
  if (page < 128 || page > 65536 || (page & (page - 1)))
    return fail(DSA_ERR_INVALID_ARG, "page_size must be a power of two in [128, 65536] (got %d)",
                page);
  const int64_t need_pages = (static_cast<int64_t>(s->n_kv) + page - 1) / page;
  if (L->max_pages < need_pages)
    return fail(DSA_ERR_INVALID_ARG, "max_pages %d < ceil(n_kv / page_size) = %lld", L->max_pages,
                static_cast<long long>(need_pages));
  if (L->pool_rows < page || L->pool_rows % page != 0 || L->pool_rows > (1ll << 31) - 256)
    return fail(DSA_ERR_INVALID_ARG,
                "pool_rows must be a positive multiple of page_size below 2^31 - 256 (got %lld)",
                static_cast<long long>(L->pool_rows));
  if (reinterpret_cast<uintptr_t>(L->block_table) % 4)
    return fail(DSA_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
  out->km.block_table = L->block_table;
  out->km.max_pages = L->max_pages;
  out->km.page_shift = __builtin_ctz(static_cast<unsigned>(page));
  out->km.pool_rows = L->pool_rows;
  return DSA_OK;
}

// ------------------------------------------------------------------ kernel attributes

template <class K>
dsa_status set_smem(K kernel, int bytes, int dev, std::atomic<bool>* done_flags) {
  // Once per device and kernel; concurrent first calls both set the same
  // attribute, which is harmless.
  if (!done_flags[dev].load(std::memory_order_acquire)) {
    DSA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                 "cudaFuncSetAttribute");
    done_flags[dev].store(true, std::memory_order_release);
  }
  return DSA_OK;
}

// ------------------------------------------------------------------ indexer launch

// Key tiles per CTA of the score kernel. The kernel streams key tiles from
// HBM, so the grid is sized by its wave count: the split that minimises
// (waves) x (tiles per CTA + a setup cost of about two tiles), with as many
// CTAs resident per SM as shared memory and TMEM allow, and at least 4 tiles
// per CTA to amortise the setup.
int indexer_tiles_per_split(int n_tiles, int64_t groups, int smem_bytes, uint32_t tmem_cols) {
  constexpr int kSmemPerSm = 233472;           // shared memory of one SM
  const int per_sm = std::max(1, std::min(kSmemPerSm / (smem_bytes + 1024),
                                          static_cast<int>(512 / tmem_cols)));
  const int64_t slots = static_cast<int64_t>(per_sm) * num_sms();
  int best_tps = n_tiles;
  int64_t best_cost = -1;
  for (int want = 1; want <= std::min(n_tiles, 256); ++want) {
    const int tps = (n_tiles + want - 1) / want;
    if (tps < 4 && tps < n_tiles) break;
    const int splits = (n_tiles + tps - 1) / tps;
    const int64_t waves = (groups * splits + slots - 1) / slots;
    const int64_t cost = waves * (tps + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_tps = tps;
    }
  }
  return best_tps;
}

template <int HI, int DI, int QG>
dsa_status launch_indexer_t(const dsa_shape* s, const HostLayout& lay, const uint8_t* q_fp8,
                            const float* q_scale, const float* w, const uint8_t* k_fp8,
                            const float* k_scale, const int32_t* q_pos0, const int32_t* kv_len,
                            int32_t row_begin, int32_t rows, float* scores, int write_invalid,
                            cudaStream_t stream, int dev, uint64_t* signs = nullptr) {
  using T = dsa::IndexerTile<HI, DI, QG>;
  static std::atomic<bool> attr_done[kMaxDevices];
  if (dsa_status st = set_smem(dsa::indexer_scores_kernel<HI, DI, QG>, T::SMEM_BYTES, dev, attr_done))
    return st;
  CUtensorMap tq, tk;
  if (dsa_status st = make_tmap_u8(&tq, q_fp8, static_cast<uint64_t>(s->batch) * s->n_q * HI, DI, T::N))
    return st;
  if (dsa_status st = make_tmap_u8(&tk, k_fp8, static_cast<uint64_t>(lay.km.pool_rows), DI, T::M))
    return st;
  dsa::IndexerParams p{};
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.rp = dsa::RowPos{q_pos0, lay.row_pos, s->n_q};
  p.km = lay.km;
  p.kv_len = kv_len;
  p.scores = scores;
  p.signs = signs;
  p.B = s->batch;
  p.n_q = s->n_q;
  p.n_kv = s->n_kv;
  p.row_begin = row_begin;
  p.rows = rows;
  p.n_groups = (rows + QG - 1) / QG;
  const int n_tiles = (s->n_kv + T::M - 1) / T::M;
  const int64_t groups = static_cast<int64_t>(s->batch) * p.n_groups;
  p.tiles_per_split = indexer_tiles_per_split(n_tiles, groups, T::SMEM_BYTES, T::TMEM_COLS);
  p.write_invalid = write_invalid;
  const int n_splits = (n_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  if (p.n_groups > 65535 || s->batch > 65535)
    return fail(DSA_ERR_INVALID_ARG, "row range too large for one indexer launch");
  dim3 grid(n_splits, p.n_groups, s->batch);
  dsa::indexer_scores_kernel<HI, DI, QG><<<grid, T::THREADS, T::SMEM_BYTES, stream>>>(tq, tk, p);
  DSA_CUDA_TRY(cudaGetLastError(), "indexer launch");
  return DSA_OK;
}

dsa_status launch_indexer(const dsa_shape* s, const HostLayout& lay, const uint8_t* q_fp8,
                          const float* q_scale, const float* w, const uint8_t* k_fp8,
                          const float* k_scale, const int32_t* q_pos0, const int32_t* kv_len,
                          int32_t row_begin, int32_t rows, float* scores, int write_invalid,
                          cudaStream_t stream, int dev, uint64_t* signs = nullptr) {
  if (s->idx_heads == 64) {
    if (rows == 1)
      return launch_indexer_t<64, 128, 1>(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0,
                                          kv_len, row_begin, rows, scores, write_invalid, stream,
                                          dev, signs);
    return launch_indexer_t<64, 128, 4>(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                                        row_begin, rows, scores, write_invalid, stream, dev, signs);
  }
  if (rows <= 4)
    return launch_indexer_t<4, 32, 4>(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                                      row_begin, rows, scores, write_invalid, stream, dev, signs);
  return launch_indexer_t<4, 32, 64>(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                                     row_begin, rows, scores, write_invalid, stream, dev, signs);
}

// Scores and selection in one kernel: H^I = 64, d^I = 128, k <= 2048.
bool indexer_topk_supported(const dsa_shape* s) {
  using T = dsa::IndexerTopkTile<64, 128, 4>;
  return s->idx_heads == 64 && s->idx_dim == 128 && s->topk <= T::MAX_K;
}

dsa_status launch_indexer_topk(const dsa_shape* s, const HostLayout& lay, const uint8_t* q_fp8,
                               const float* q_scale, const float* w, const uint8_t* k_fp8,
                               const float* k_scale, const int32_t* q_pos0,
                               const int32_t* kv_len, int32_t row_begin, int32_t rows,
                               int32_t* indices, int32_t out_rows, cudaStream_t stream, int dev) {
  using T = dsa::IndexerTopkTile<64, 128, 4>;
  static std::atomic<bool> attr_done[kMaxDevices];
  if (dsa_status st = set_smem(dsa::indexer_topk_kernel<64, 128, 4>, T::SMEM_BYTES, dev, attr_done))
    return st;
  if (rows <= 0) return DSA_OK;
  CUtensorMap tq, tk;
  if (dsa_status st = make_tmap_u8(&tq, q_fp8, static_cast<uint64_t>(s->batch) * s->n_q * 64, 128, T::N))
    return st;
  if (dsa_status st = make_tmap_u8(&tk, k_fp8, static_cast<uint64_t>(lay.km.pool_rows), 128, T::M))
    return st;
  dsa::IndexerTopkParams p{};
  p.q_scale = q_scale;
  p.w = w;
  p.k_scale = k_scale;
  p.rp = dsa::RowPos{q_pos0, lay.row_pos, s->n_q};
  p.km = lay.km;
  p.kv_len = kv_len;
  p.indices = indices;
  p.B = s->batch;
  p.n_q = s->n_q;
  p.n_kv = s->n_kv;
  p.k = s->topk;
  p.row_begin = row_begin;
  p.rows = rows;
  p.n_groups = (rows + 3) / 4;
  p.out_rows = out_rows;
  if (s->batch > 65535) return fail(DSA_ERR_INVALID_ARG, "batch > 65535");
  dim3 grid(p.n_groups, s->batch);
  dsa::indexer_topk_kernel<64, 128, 4><<<grid, T::THREADS, T::SMEM_BYTES, stream>>>(tq, tk, p);
  DSA_CUDA_TRY(cudaGetLastError(), "fused indexer top-k launch");
  return DSA_OK;
}

// A launch that may overlap the previous kernel of the stream (programmatic
// stream serialization); the kernel waits (griddep_wait) before it reads
// anything that kernel writes. Used only for the second and later kernels of
// dsa_forward, whose first kernel is an ordinary launch.
template <class... Params, class... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, int smem,
                             cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ------------------------------------------------------------------ top-k launch

dsa_status launch_topk(const dsa_shape* s, const HostLayout& lay, const float* scores,
                       int32_t row_begin, int32_t rows, const int32_t* q_pos0,
                       const int32_t* kv_len, int32_t* indices, int32_t out_rows,
                       int32_t out_row0, cudaStream_t stream, int dev, bool dependent = false) {
  static std::atomic<bool> attr_done[kMaxDevices];
  const int smem = static_cast<int>(sizeof(dsa::TopkSmem));
  if (dsa_status st = set_smem(dsa::topk_kernel, smem, dev, attr_done)) return st;
  if (s->batch > 65535) return fail(DSA_ERR_INVALID_ARG, "batch > 65535");
  dsa::TopkParams p{};
  p.scores = scores;
  p.rp = dsa::RowPos{q_pos0, lay.row_pos, s->n_q};
  p.kv_len = kv_len;
  p.indices = indices;
  p.rows = rows;
  p.row_begin = row_begin;
  p.n_kv = s->n_kv;
  p.k = s->topk;
  p.out_rows = out_rows;
  p.out_row0 = out_row0;
  dim3 grid(2 * rows, s->batch);   // a cluster of two CTAs per row
  if (dependent)
    DSA_CUDA_TRY(launch_dependent(dsa::topk_kernel, grid, dim3(dsa::kTopkThreads), smem, stream, p),
                 "top-k launch");
  else
    dsa::topk_kernel<<<grid, dsa::kTopkThreads, smem, stream>>>(p);
  DSA_CUDA_TRY(cudaGetLastError(), "top-k launch");
  return DSA_OK;
}

// ------------------------------------------------------------------ attention launch

struct AttnPlan {
  int vsplit, splits, slots_per_split;
  size_t ws_bytes;
};

AttnPlan plan_attn(const dsa_shape* s) {
  AttnPlan pl{};
  pl.vsplit = s->qk_dim == 576 ? 2 : 1;
  const int64_t rows = static_cast<int64_t>(s->batch) * s->n_q;
  const int64_t ctas = rows * pl.vsplit;
  const int max_splits = (s->topk + 31) / 32;
  int splits = 1;
  const int sms = num_sms();
  if (ctas < sms / 2) {
    splits = static_cast<int>(std::min<int64_t>(max_splits, (sms + ctas - 1) / ctas));
    splits = std::max(1, std::min(splits, 16));
  }
  int sps = (s->topk + splits - 1) / splits;
  sps = (sps + 31) / 32 * 32;
  splits = (s->topk + sps - 1) / sps;
  pl.splits = splits;
  pl.slots_per_split = sps;
  pl.ws_bytes = 0;
  if (splits > 1) {
    const size_t po = static_cast<size_t>(rows) * splits * s->heads * s->v_dim * sizeof(float);
    const size_t pl_ = static_cast<size_t>(rows) * splits * s->heads * sizeof(float);
    pl.ws_bytes = (po + 255) / 256 * 256 + (pl_ + 255) / 256 * 256;
  }
  return pl;
}

template <int DQK, int DV, int VSPLIT>
dsa_status launch_attn_t(const dsa_shape* s, const dsa::KeyMap& km, const AttnPlan& pl,
                         const uint16_t* q, const uint16_t* kv, const int32_t* indices, void* out,
                         int out_bf16, float* lse, void* ws, cudaStream_t stream, int dev) {
  using T = dsa::AttnTile<DQK, DV, VSPLIT>;
  static std::atomic<bool> attr_done[kMaxDevices];
  if (dsa_status st = set_smem(dsa::sparse_attn_kernel<DQK, DV, VSPLIT>, T::SMEM_BYTES, dev, attr_done))
    return st;
  dsa::AttnParams p{};
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.kv = reinterpret_cast<const __nv_bfloat16*>(kv);
  p.km = km;
  p.indices = indices;
  p.out = out;
  p.lse = lse;
  p.B = s->batch;
  p.n_q = s->n_q;
  p.n_kv = s->n_kv;
  p.topk = s->topk;
  p.H = s->heads;
  p.splits = pl.splits;
  p.slots_per_split = pl.slots_per_split;
  p.out_bf16 = out_bf16;
  p.scale_log2 = s->softmax_scale * 1.4426950408889634f;
  const int64_t rows = static_cast<int64_t>(s->batch) * s->n_q;
  if (pl.splits > 1) {
    const size_t po = static_cast<size_t>(rows) * pl.splits * s->heads * s->v_dim * sizeof(float);
    p.part_o = static_cast<float*>(ws);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + (po + 255) / 256 * 256);
  }
  const int64_t nblocks = rows * pl.splits * VSPLIT;
  if (nblocks >= (1ll << 31)) return fail(DSA_ERR_INVALID_ARG, "too many attention rows");
  dsa::sparse_attn_kernel<DQK, DV, VSPLIT>
      <<<static_cast<unsigned>(nblocks), T::THREADS, T::SMEM_BYTES, stream>>>(p);
  DSA_CUDA_TRY(cudaGetLastError(), "sparse attention launch");
  if (pl.splits > 1) {
    if (rows > 0x7fffffffll) return fail(DSA_ERR_INVALID_ARG, "too many rows");
    dim3 grid(static_cast<unsigned>(rows), s->heads);
    dsa::attn_combine_kernel<<<grid, 128, 0, stream>>>(p, DV);
    DSA_CUDA_TRY(cudaGetLastError(), "attention combine launch");
  }
  return DSA_OK;
}

// 576/512 latent: two CTAs per (row, split), one per value half, see sparse_attn_vh.cuh.
dsa_status launch_attn_vh(const dsa_shape* s, const dsa::KeyMap& km, const AttnPlan& pl,
                          const uint16_t* q, const uint16_t* kv, const int32_t* indices,
                          void* out, int out_bf16, float* lse, void* ws, cudaStream_t stream,
                          int dev, bool dependent) {
  using T = dsa::VhTile;
  static std::atomic<bool> attr_done[kMaxDevices];
  if (dsa_status st = set_smem(dsa::sparse_attn_vh_kernel, T::SMEM_BYTES, dev, attr_done))
    return st;
  dsa::AttnParams p{};
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.kv = reinterpret_cast<const __nv_bfloat16*>(kv);
  p.km = km;
  p.indices = indices;
  p.out = out;
  p.lse = lse;
  p.B = s->batch;
  p.n_q = s->n_q;
  p.n_kv = s->n_kv;
  p.topk = s->topk;
  p.H = s->heads;
  p.splits = pl.splits;
  p.slots_per_split = pl.slots_per_split;
  p.out_bf16 = out_bf16;
  p.scale_log2 = s->softmax_scale * 1.4426950408889634f;
  const int64_t rows = static_cast<int64_t>(s->batch) * s->n_q;
  if (pl.splits > 1) {
    const size_t po = static_cast<size_t>(rows) * pl.splits * s->heads * s->v_dim * sizeof(float);
    p.part_o = static_cast<float*>(ws);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + (po + 255) / 256 * 256);
  }
  // the output as rows of DV elements for the kernel's TMA stores
  CUtensorMap to;
  {
    const bool direct = pl.splits == 1;
    const uint32_t esz = (direct && out_bf16) ? 2u : 4u;
    const uint64_t orows = static_cast<uint64_t>(rows) * (direct ? 1 : pl.splits) * s->heads;
    if (dsa_status st = make_tmap_rows128(&to, direct ? out : static_cast<void*>(p.part_o), orows,
                                          static_cast<uint32_t>(s->v_dim) * esz,
                                          static_cast<uint32_t>(s->heads)))
      return st;
  }
  // persistent CTAs (one per SM, an even number so that a CTA keeps its
  // value half), each walking units c, c + grid, ...
  const int64_t n_units = rows * pl.splits * 2;
  if (n_units >= (1ll << 31)) return fail(DSA_ERR_INVALID_ARG, "too many attention rows");
  const int64_t grid = std::min<int64_t>(n_units, std::max(2, num_sms() / 2 * 2));
  if (dependent)
    DSA_CUDA_TRY(launch_dependent(dsa::sparse_attn_vh_kernel, dim3(static_cast<unsigned>(grid)),
                                  dim3(T::THREADS), T::SMEM_BYTES, stream, to, p, n_units),
                 "sparse attention launch");
  else
    dsa::sparse_attn_vh_kernel<<<static_cast<unsigned>(grid), T::THREADS, T::SMEM_BYTES, stream>>>(
        to, p, n_units);
  DSA_CUDA_TRY(cudaGetLastError(), "sparse attention launch");
  if (pl.splits > 1) {
    dim3 grid(static_cast<unsigned>(rows), s->heads);
    dsa::attn_combine_kernel<<<grid, 128, 0, stream>>>(p, s->v_dim);
    DSA_CUDA_TRY(cudaGetLastError(), "attention combine launch");
  }
  return DSA_OK;
}

dsa_status launch_attn(const dsa_shape* s, const dsa::KeyMap& km, const uint16_t* q,
                       const uint16_t* kv, const int32_t* indices, void* out, int out_bf16,
                       float* lse, void* ws, size_t ws_bytes, cudaStream_t stream, int dev,
                       bool dependent = false) {
  const AttnPlan pl = plan_attn(s);
  if (pl.ws_bytes > 0) {
    if (!ws || ws_bytes < pl.ws_bytes)
      return fail(DSA_ERR_WORKSPACE, "attention needs %zu workspace bytes, got %zu", pl.ws_bytes,
                  ws ? ws_bytes : size_t(0));
    if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  if (s->qk_dim == 576)
    return launch_attn_vh(s, km, pl, q, kv, indices, out, out_bf16, lse, ws, stream, dev,
                          dependent);
  return launch_attn_t<64, 64, 1>(s, km, pl, q, kv, indices, out, out_bf16, lse, ws, stream, dev);
}

// ------------------------------------------------------------------ forward plan

struct FwdPlan {
  int chunk_rows;
  bool fused;   // scores and selection in one kernel: no score buffer at all
  size_t scores_bytes, attn_bytes, total;
};

FwdPlan plan_forward(const dsa_shape* s) {
  FwdPlan f{};
  f.attn_bytes = plan_attn(s).ws_bytes;
  // The fused kernel runs one CTA per 4 query rows over all of their keys;
  // with fewer groups than SMs (decode) the split score kernel plus the
  // separate selection keeps more of the GPU busy.
  const int64_t groups = static_cast<int64_t>(s->batch) * ((s->n_q + 3) / 4);
  if (indexer_topk_supported(s) && groups >= num_sms()) {
    f.fused = true;
    f.chunk_rows = s->n_q;
    f.scores_bytes = 0;
    f.total = f.attn_bytes;
    return f;
  }
  const size_t row_bytes = static_cast<size_t>(s->batch) * s->n_kv * sizeof(float);
  const size_t budget = 256ull << 20;   // scores of one row chunk (L2-sized pieces at 64K+)
  int64_t chunk = static_cast<int64_t>(budget / row_bytes);
  chunk = std::max<int64_t>(chunk, 64);
  chunk = std::min<int64_t>(chunk, s->n_q);
  if (chunk < s->n_q) chunk = std::max<int64_t>(64, chunk / 64 * 64);
  f.chunk_rows = static_cast<int>(chunk);
  f.scores_bytes = (row_bytes * chunk + 255) / 256 * 256;
  f.total = f.scores_bytes + f.attn_bytes;
  return f;
}

// ------------------------------------------------------------------ warm-up loss plan

// Rows per chunk of dsa_indexer_kl: per (row, key) it stores p (then g), the
// score I and the sign mask, 16 bytes; a chunk of every sequence's rows
// takes at most ~512 MB of workspace.
struct KlPlan {
  int chunk_rows, k_split;
  size_t pbar_bytes, scores_bytes, signs_bytes, part_bytes, total;
};

KlPlan plan_kl(const dsa_shape* s) {
  KlPlan k{};
  const size_t per_row = static_cast<size_t>(s->batch) * s->n_kv;
  const size_t budget = 512ull << 20;
  int64_t chunk = static_cast<int64_t>(budget / (16 * per_row));
  chunk = std::max<int64_t>(1, std::min<int64_t>(chunk, s->n_q));
  k.chunk_rows = static_cast<int>(chunk);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  k.pbar_bytes = up(per_row * chunk * 4);
  k.scores_bytes = up(per_row * chunk * 4);
  k.signs_bytes = up(per_row * chunk * 8);
  // dk partials: the chunk's rows split so that key tiles x splits fill the
  // SMs about twice
  const int64_t tiles = static_cast<int64_t>(s->batch) * ((s->n_kv + 63) / 64);
  k.k_split = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>({16, chunk, (2 * num_sms() + tiles - 1) / tiles})));
  k.part_bytes = up(static_cast<size_t>(k.k_split) * per_row * s->idx_dim * 4);
  k.total = k.pbar_bytes + k.scores_bytes + k.signs_bytes + k.part_bytes;
  return k;
}

dsa_status check_kl_shape(const dsa_shape* s) {
  if (dsa_status st = check_indexer_shape(s)) return st;
  if (dsa_status st = check_attn_shape(s)) return st;
  return DSA_OK;
}

template <int DQK>
dsa_status launch_kl_probs(const dsa_shape* s, const uint16_t* q, const uint16_t* kv,
                           const int32_t* q_pos0, const int32_t* kv_len, int32_t row_begin,
                           int32_t rows, float* pbar, cudaStream_t stream, int dev) {
  using T = dsa::KlProbTile<DQK>;
  static std::atomic<bool> attr_done[kMaxDevices];
  if (dsa_status st = set_smem(dsa::kl_probs_kernel<DQK>, T::SMEM_BYTES, dev, attr_done)) return st;
  dsa::KlProbParams p{};
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.kv = reinterpret_cast<const __nv_bfloat16*>(kv);
  p.q_pos0 = q_pos0;
  p.kv_len = kv_len;
  p.pbar = pbar;
  p.B = s->batch;
  p.n_q = s->n_q;
  p.n_kv = s->n_kv;
  p.H = s->heads;
  p.row_begin = row_begin;
  p.rows = rows;
  p.scale_log2 = s->softmax_scale * 1.4426950408889634f;
  dim3 grid(rows, s->batch);
  dsa::kl_probs_kernel<DQK><<<grid, T::THREADS, T::SMEM_BYTES, stream>>>(p);
  DSA_CUDA_TRY(cudaGetLastError(), "warm-up loss probabilities launch");
  return DSA_OK;
}

template <int HI, int DI>
dsa_status launch_kl_grads(const dsa::KlGradParams& p, int32_t rows, int32_t batch, int32_t n_kv,
                           float* part, int32_t k_split, cudaStream_t stream, int dev) {
  using Map = dsa::KlGradUMap<HI, DI>;
  using KMap = dsa::KlGradKMap<HI, DI>;
  static std::atomic<bool> attr_done[kMaxDevices];
  if (dsa_status st = set_smem(dsa::kl_grad_k_kernel<HI, DI>, KMap::SMEM_BYTES, dev, attr_done))
    return st;
  dsa::kl_grad_u_kernel<HI, DI><<<dim3(rows, batch), Map::THREADS, 0, stream>>>(p);
  DSA_CUDA_TRY(cudaGetLastError(), "warm-up loss gradient (q, w) launch");
  dsa::kl_grad_k_kernel<HI, DI><<<dim3((n_kv + KMap::KT - 1) / KMap::KT, k_split, batch),
                                   dsa::kKlGradThreads, KMap::SMEM_BYTES, stream>>>(p, part,
                                                                                    k_split);
  DSA_CUDA_TRY(cudaGetLastError(), "warm-up loss gradient (k) launch");
  const int64_t n = static_cast<int64_t>(batch) * n_kv * DI;
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 4 * num_sms()));
  dsa::kl_grad_k_reduce_kernel<<<blocks, 256, 0, stream>>>(part, p.dk, n, k_split);
  DSA_CUDA_TRY(cudaGetLastError(), "warm-up loss gradient (k) reduce launch");
  return DSA_OK;
}

dsa_status check_ptrs(std::initializer_list<const void*> ptrs, const char* what) {
  for (const void* p : ptrs)
    if (!p) return fail(DSA_ERR_INVALID_ARG, "%s: required pointer is NULL", what);
  return DSA_OK;
}

}  // namespace

// ======================================================================== no-alloc scratch

// Split-K partials of dsa_sparse_attn_noalloc. Host code may not use this
// name as a device address: it is a host-side stand-in. The device address
// comes from cudaGetSymbolAddress once per device.
static constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on `dev` (the current device).
dsa_status noalloc_scratch_addr(int dev, void** addr) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return DSA_OK;
}
}  // namespace

// ======================================================================== C ABI

extern "C" {

const char* dsa_version(void) { return "0.1.0"; }

dsa_status dsa_quantize_e4m3(int64_t rows, int32_t dim, const uint16_t* x, uint8_t* codes,
                             float* scales, void* stream) {
  if (rows < 0) return fail(DSA_ERR_INVALID_ARG, "rows must be >= 0 (got %lld)", static_cast<long long>(rows));
  if (dim != 32 && dim != 64 && dim != 128)
    return fail(DSA_ERR_UNSUPPORTED, "dsa_quantize_e4m3 supports dim 32, 64, 128 (got %d)", dim);
  if (dsa_status st = check_ptrs({x, codes, scales}, "dsa_quantize_e4m3")) return st;
  const int per = dim / 32;
  if (!aligned(x, 2 * per) || !aligned(codes, per) || !aligned(scales, 4))
    return fail(DSA_ERR_INVALID_ARG, "x must be %d-byte and codes %d-byte aligned", 2 * per, per);
  const long long blocks = (rows + dsa::kQuantRowsPerCta - 1) / dsa::kQuantRowsPerCta;
  if (blocks >= (1ll << 31)) return fail(DSA_ERR_INVALID_ARG, "too many rows");
  if (rows == 0) return DSA_OK;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>(blocks);
  constexpr int threads = 32 * dsa::kQuantWarps;
  if (per == 4)
    dsa::quantize_e4m3_rows_kernel<4><<<grid, threads, 0, st_>>>(x, codes, scales, rows);
  else if (per == 2)
    dsa::quantize_e4m3_rows_kernel<2><<<grid, threads, 0, st_>>>(x, codes, scales, rows);
  else
    dsa::quantize_e4m3_rows_kernel<1><<<grid, threads, 0, st_>>>(x, codes, scales, rows);
  DSA_CUDA_TRY(cudaGetLastError(), "quantiser launch");
  return DSA_OK;
}

dsa_status dsa_selftest_wait_timeout(uint32_t limit_ms, void* stream) {
  if (limit_ms == 0 || limit_ms > 10000)
    return fail(DSA_ERR_INVALID_ARG, "limit_ms must be in [1, 10000] (got %u)", limit_ms);
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  dsa::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ms) * 1000000ull);
  DSA_CUDA_TRY(cudaGetLastError(), "wait self-test launch");
  return DSA_OK;
}

const char* dsa_status_string(dsa_status st) {
  switch (st) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape";
    case DSA_ERR_WORKSPACE: return "workspace missing or too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device wait timed out";
    case DSA_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

const char* dsa_last_error(void) { return g_last_error.c_str(); }

dsa_status dsa_workspace_size(const dsa_shape* s, int32_t op, size_t* bytes) {
  if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = 0;
  switch (op) {
    case DSA_OP_INDEXER:
      return check_indexer_shape(s);
    case DSA_OP_TOPK:
      return check_topk_shape(s);
    case DSA_OP_SPARSE_ATTN: {
      if (dsa_status st = check_attn_shape(s)) return st;
      *bytes = plan_attn(s).ws_bytes;
      return DSA_OK;
    }
    case DSA_OP_FORWARD: {
      if (dsa_status st = check_indexer_shape(s)) return st;
      if (dsa_status st = check_attn_shape(s)) return st;
      *bytes = plan_forward(s).total;
      return DSA_OK;
    }
    case DSA_OP_INDEXER_KL: {
      if (dsa_status st = check_kl_shape(s)) return st;
      *bytes = plan_kl(s).total;
      return DSA_OK;
    }
    default:
      return fail(DSA_ERR_INVALID_ARG, "unknown op %d", op);
  }
}

dsa_status dsa_forward_chunk_rows(const dsa_shape* s, int32_t* rows) {
  if (!rows) return fail(DSA_ERR_INVALID_ARG, "rows is NULL");
  if (dsa_status st = check_indexer_shape(s)) return st;
  if (dsa_status st = check_attn_shape(s)) return st;
  *rows = plan_forward(s).chunk_rows;
  return DSA_OK;
}

dsa_status dsa_forward_plan(const dsa_shape* s, int32_t* fused, int32_t* chunk_rows,
                            int32_t* attn_splits) {
  if (!fused || !chunk_rows || !attn_splits)
    return fail(DSA_ERR_INVALID_ARG, "dsa_forward_plan: output pointer is NULL");
  if (dsa_status st = check_indexer_shape(s)) return st;
  if (dsa_status st = check_attn_shape(s)) return st;
  const FwdPlan f = plan_forward(s);
  *fused = f.fused ? 1 : 0;
  *chunk_rows = f.chunk_rows;
  *attn_splits = plan_attn(s).splits;
  return DSA_OK;
}

dsa_status dsa_indexer_scores_ex(const dsa_shape* s, const dsa_layout* layout,
                                 const uint8_t* q_fp8, const float* q_scale, const float* w,
                                 const uint8_t* k_fp8, const float* k_scale,
                                 const int32_t* q_pos0, const int32_t* kv_len, int32_t row_begin,
                                 int32_t row_end, int32_t flags, float* scores, void* stream) {
  if (dsa_status st = check_indexer_shape(s)) return st;
  if (flags != DSA_SCORES_ALL && flags != DSA_SCORES_VISIBLE_ONLY)
    return fail(DSA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if (dsa_status st = check_ptrs({q_fp8, q_scale, w, k_fp8, k_scale, scores}, "dsa_indexer_scores"))
    return st;
  if (row_begin < 0 || row_end > s->n_q || row_begin >= row_end)
    return fail(DSA_ERR_INVALID_ARG, "row range [%d, %d) outside [0, %d) or empty", row_begin,
                row_end, s->n_q);
  if (!aligned(q_fp8, 16) || !aligned(k_fp8, 16))
    return fail(DSA_ERR_INVALID_ARG, "q_fp8 and k_fp8 must be 16-byte aligned");
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, layout, &lay)) return st;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  return launch_indexer(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len, row_begin,
                        row_end - row_begin, scores, flags == DSA_SCORES_ALL ? 1 : 0,
                        static_cast<cudaStream_t>(stream), dev);
}

dsa_status dsa_indexer_scores(const dsa_shape* s, const uint8_t* q_fp8, const float* q_scale,
                              const float* w, const uint8_t* k_fp8, const float* k_scale,
                              const int32_t* q_pos0, const int32_t* kv_len, int32_t row_begin,
                              int32_t row_end, int32_t flags, float* scores, void* stream) {
  return dsa_indexer_scores_ex(s, nullptr, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                               row_begin, row_end, flags, scores, stream);
}

dsa_status dsa_indexer_topk_ex(const dsa_shape* s, const dsa_layout* layout, const uint8_t* q_fp8,
                               const float* q_scale, const float* w, const uint8_t* k_fp8,
                               const float* k_scale, const int32_t* q_pos0,
                               const int32_t* kv_len, int32_t row_begin, int32_t row_end,
                               int32_t* indices, void* stream) {
  if (dsa_status st = check_indexer_shape(s)) return st;
  if (dsa_status st = check_topk_shape(s)) return st;
  if (!indexer_topk_supported(s))
    return fail(DSA_ERR_UNSUPPORTED,
                "dsa_indexer_topk supports idx_heads = 64, idx_dim = 128, topk <= 2048 "
                "(got %d, %d, %d)",
                s->idx_heads, s->idx_dim, s->topk);
  if (dsa_status st = check_ptrs({q_fp8, q_scale, w, k_fp8, k_scale, indices}, "dsa_indexer_topk"))
    return st;
  if (row_begin < 0 || row_end > s->n_q || row_begin >= row_end)
    return fail(DSA_ERR_INVALID_ARG, "row range [%d, %d) outside [0, %d) or empty", row_begin,
                row_end, s->n_q);
  if (!aligned(q_fp8, 16) || !aligned(k_fp8, 16))
    return fail(DSA_ERR_INVALID_ARG, "q_fp8 and k_fp8 must be 16-byte aligned");
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, layout, &lay)) return st;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  return launch_indexer_topk(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len, row_begin,
                             row_end - row_begin, indices, row_end - row_begin,
                             static_cast<cudaStream_t>(stream), dev);
}

dsa_status dsa_indexer_topk(const dsa_shape* s, const uint8_t* q_fp8, const float* q_scale,
                            const float* w, const uint8_t* k_fp8, const float* k_scale,
                            const int32_t* q_pos0, const int32_t* kv_len, int32_t row_begin,
                            int32_t row_end, int32_t* indices, void* stream) {
  return dsa_indexer_topk_ex(s, nullptr, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                             row_begin, row_end, indices, stream);
}

dsa_status dsa_topk_ex(const dsa_shape* s, const dsa_layout* layout, const float* scores,
                       int32_t row_begin, int32_t row_end, const int32_t* q_pos0,
                       const int32_t* kv_len, int32_t* indices, void* ws, size_t ws_bytes,
                       void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (dsa_status st = check_topk_shape(s)) return st;
  if (dsa_status st = check_ptrs({scores, indices}, "dsa_topk")) return st;
  if (row_begin < 0 || row_end > s->n_q || row_begin >= row_end)
    return fail(DSA_ERR_INVALID_ARG, "row range [%d, %d) outside [0, %d) or empty", row_begin,
                row_end, s->n_q);
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, layout, &lay)) return st;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  return launch_topk(s, lay, scores, row_begin, row_end - row_begin, q_pos0, kv_len, indices,
                     row_end - row_begin, 0, static_cast<cudaStream_t>(stream), dev);
}

dsa_status dsa_topk(const dsa_shape* s, const float* scores, int32_t row_begin, int32_t row_end,
                    const int32_t* q_pos0, const int32_t* kv_len, int32_t* indices, void* ws,
                    size_t ws_bytes, void* stream) {
  return dsa_topk_ex(s, nullptr, scores, row_begin, row_end, q_pos0, kv_len, indices, ws,
                     ws_bytes, stream);
}

dsa_status dsa_sparse_attn_ex(const dsa_shape* s, const dsa_layout* layout, const uint16_t* q,
                              const uint16_t* kv, const int32_t* indices, void* out,
                              int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                              void* stream) {
  if (dsa_status st = check_attn_shape(s)) return st;
  if (dsa_status st = check_ptrs({q, kv, indices, out}, "dsa_sparse_attn")) return st;
  if (out_dtype != DSA_OUT_F32 && out_dtype != DSA_OUT_BF16)
    return fail(DSA_ERR_INVALID_ARG, "out_dtype must be DSA_OUT_F32 or DSA_OUT_BF16");
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16))
    return fail(DSA_ERR_INVALID_ARG, "q, kv and out must be 16-byte aligned");
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, layout, &lay)) return st;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  return launch_attn(s, lay.km, q, kv, indices, out, out_dtype == DSA_OUT_BF16, lse, ws, ws_bytes,
                     static_cast<cudaStream_t>(stream), dev);
}

dsa_status dsa_sparse_attn(const dsa_shape* s, const uint16_t* q, const uint16_t* kv,
                           const int32_t* indices, void* out, int32_t out_dtype, float* lse,
                           void* ws, size_t ws_bytes, void* stream) {
  return dsa_sparse_attn_ex(s, nullptr, q, kv, indices, out, out_dtype, lse, ws, ws_bytes, stream);
}

dsa_status dsa_sparse_attn_noalloc(const dsa_shape* s, const uint16_t* q, const uint16_t* kv,
                                   const int32_t* indices, void* out, int32_t out_dtype,
                                   float* lse, void* stream) {
  if (dsa_status st = check_attn_shape(s)) return st;
  if (dsa_status st = check_ptrs({q, kv, indices, out}, "dsa_sparse_attn_noalloc")) return st;
  if (out_dtype != DSA_OUT_F32 && out_dtype != DSA_OUT_BF16)
    return fail(DSA_ERR_INVALID_ARG, "out_dtype must be DSA_OUT_F32 or DSA_OUT_BF16");
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16))
    return fail(DSA_ERR_INVALID_ARG, "q, kv and out must be 16-byte aligned");
  const AttnPlan pl = plan_attn(s);
  if (pl.ws_bytes > kNoAllocScratchBytes)
    return fail(DSA_ERR_WORKSPACE,
                "this shape needs %zu bytes of split-K scratch; dsa_sparse_attn_noalloc holds at "
                "most %zu (use dsa_sparse_attn with a workspace)",
                pl.ws_bytes, kNoAllocScratchBytes);
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, nullptr, &lay)) return st;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  void* scratch = nullptr;
  if (pl.ws_bytes > 0) {
    if (dsa_status st = noalloc_scratch_addr(dev, &scratch)) return st;
  }
  return launch_attn(s, lay.km, q, kv, indices, out, out_dtype == DSA_OUT_BF16, lse, scratch,
                     pl.ws_bytes > 0 ? kNoAllocScratchBytes : 0,
                     static_cast<cudaStream_t>(stream), dev);
}

dsa_status dsa_forward_ex(const dsa_shape* s, const dsa_layout* layout, const uint8_t* q_fp8,
                          const float* q_scale, const float* w, const uint8_t* k_fp8,
                          const float* k_scale, const int32_t* q_pos0, const int32_t* kv_len,
                          const uint16_t* q, const uint16_t* kv, int32_t* indices_out, void* out,
                          int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                          void* stream) {
  if (dsa_status st = check_indexer_shape(s)) return st;
  if (dsa_status st = check_attn_shape(s)) return st;
  if (dsa_status st = check_ptrs({q_fp8, q_scale, w, k_fp8, k_scale, q, kv, indices_out, out},
                                 "dsa_forward"))
    return st;
  if (out_dtype != DSA_OUT_F32 && out_dtype != DSA_OUT_BF16)
    return fail(DSA_ERR_INVALID_ARG, "out_dtype must be DSA_OUT_F32 or DSA_OUT_BF16");
  if (!aligned(q_fp8, 16) || !aligned(k_fp8, 16) || !aligned(q, 16) || !aligned(kv, 16) ||
      !aligned(out, 16))
    return fail(DSA_ERR_INVALID_ARG, "q_fp8, k_fp8, q, kv and out must be 16-byte aligned");
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, layout, &lay)) return st;
  const FwdPlan f = plan_forward(s);
  if (f.total > 0) {
    if (!ws || ws_bytes < f.total)
      return fail(DSA_ERR_WORKSPACE, "dsa_forward needs %zu workspace bytes, got %zu", f.total,
                  ws ? ws_bytes : size_t(0));
    if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  float* scores = static_cast<float*>(ws);
  void* attn_ws = static_cast<char*>(ws) + f.scores_bytes;
  if (f.fused) {
    if (dsa_status e = launch_indexer_topk(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0,
                                           kv_len, 0, s->n_q, indices_out, s->n_q, st_, dev))
      return e;
    return launch_attn(s, lay.km, q, kv, indices_out, out, out_dtype == DSA_OUT_BF16, lse, attn_ws,
                       f.attn_bytes, st_, dev);
  }
  for (int r0 = 0; r0 < s->n_q; r0 += f.chunk_rows) {
    const int rows = std::min(f.chunk_rows, s->n_q - r0);
    if (dsa_status e = launch_indexer(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                                      r0, rows, scores, 0, st_, dev))
      return e;
    // The chunk's selections go straight to their rows of indices_out. The
    // top-k and the attention are dependent launches: each may start its
    // set-up while the kernel before it finishes, and waits for that kernel
    // before reading its output; the indexer is an ordinary launch (the
    // scores buffer it writes is read by the previous chunk's top-k).
    if (dsa_status e = launch_topk(s, lay, scores, r0, rows, q_pos0, kv_len, indices_out, s->n_q,
                                   r0, st_, dev, true))
      return e;
  }
  return launch_attn(s, lay.km, q, kv, indices_out, out, out_dtype == DSA_OUT_BF16, lse, attn_ws,
                     f.attn_bytes, st_, dev, true);
}

dsa_status dsa_forward(const dsa_shape* s, const uint8_t* q_fp8, const float* q_scale,
                       const float* w, const uint8_t* k_fp8, const float* k_scale,
                       const int32_t* q_pos0, const int32_t* kv_len, const uint16_t* q,
                       const uint16_t* kv, int32_t* indices_out, void* out, int32_t out_dtype,
                       float* lse, void* ws, size_t ws_bytes, void* stream) {
  return dsa_forward_ex(s, nullptr, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len, q, kv,
                        indices_out, out, out_dtype, lse, ws, ws_bytes, stream);
}

dsa_status dsa_indexer_kl(const dsa_shape* s, const uint8_t* q_fp8, const float* q_scale,
                          const float* w, const uint8_t* k_fp8, const float* k_scale,
                          const int32_t* q_pos0, const int32_t* kv_len, const uint16_t* q,
                          const uint16_t* kv, float* loss, float* dw, float* dq, float* dk,
                          void* ws, size_t ws_bytes, void* stream) {
  if (dsa_status st = check_kl_shape(s)) return st;
  if (dsa_status st = check_ptrs({q_fp8, q_scale, w, k_fp8, k_scale, q, kv, loss, dw, dq, dk},
                                 "dsa_indexer_kl"))
    return st;
  if (!aligned(q_fp8, 16) || !aligned(k_fp8, 16) || !aligned(q, 16) || !aligned(kv, 16))
    return fail(DSA_ERR_INVALID_ARG, "q_fp8, k_fp8, q and kv must be 16-byte aligned");
  const KlPlan plan = plan_kl(s);
  if (!ws || ws_bytes < plan.total)
    return fail(DSA_ERR_WORKSPACE, "dsa_indexer_kl needs %zu workspace bytes, got %zu", plan.total,
                ws ? ws_bytes : size_t(0));
  if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  HostLayout lay;
  if (dsa_status st = resolve_layout(s, nullptr, &lay)) return st;
  int dev;
  if (dsa_status st = current_device(&dev)) return st;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  float* pbar = static_cast<float*>(ws);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + plan.pbar_bytes);
  uint64_t* signs =
      reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + plan.pbar_bytes + plan.scores_bytes);
  float* part = reinterpret_cast<float*>(static_cast<char*>(ws) + plan.pbar_bytes +
                                         plan.scores_bytes + plan.signs_bytes);
  // dk is a sum over every row chunk
  DSA_CUDA_TRY(cudaMemsetAsync(dk, 0,
                               static_cast<size_t>(s->batch) * s->n_kv * s->idx_dim * sizeof(float),
                               st_),
               "clear dk");
  for (int r0 = 0; r0 < s->n_q; r0 += plan.chunk_rows) {
    const int rows = std::min(plan.chunk_rows, s->n_q - r0);
    if (s->qk_dim == 576) {
      if (dsa_status e = launch_kl_probs<576>(s, q, kv, q_pos0, kv_len, r0, rows, pbar, st_, dev))
        return e;
    } else {
      if (dsa_status e = launch_kl_probs<64>(s, q, kv, q_pos0, kv_len, r0, rows, pbar, st_, dev))
        return e;
    }
    if (dsa_status e = launch_indexer(s, lay, q_fp8, q_scale, w, k_fp8, k_scale, q_pos0, kv_len,
                                      r0, rows, scores, 1, st_, dev, signs))
      return e;
    dsa::KlRowParams rp{};
    rp.scores = scores;
    rp.pbar = pbar;
    rp.loss = loss;
    rp.q_pos0 = q_pos0;
    rp.kv_len = kv_len;
    rp.n_q = s->n_q;
    rp.n_kv = s->n_kv;
    rp.row_begin = r0;
    rp.rows = rows;
    dsa::kl_rows_kernel<<<dim3(rows, s->batch), dsa::kKlRowThreads, 0, st_>>>(rp);
    DSA_CUDA_TRY(cudaGetLastError(), "warm-up loss rows launch");
    dsa::KlGradParams gp{};
    gp.q_fp8 = q_fp8;
    gp.q_scale = q_scale;
    gp.w = w;
    gp.k_fp8 = k_fp8;
    gp.k_scale = k_scale;
    gp.g = pbar;
    gp.signs = signs;
    gp.q_pos0 = q_pos0;
    gp.kv_len = kv_len;
    gp.dw = dw;
    gp.dq = dq;
    gp.dk = dk;
    gp.n_q = s->n_q;
    gp.n_kv = s->n_kv;
    gp.row_begin = r0;
    gp.rows = rows;
    const int ksplit = std::min(plan.k_split, rows);
    dsa_status e = s->idx_heads == 64
                       ? launch_kl_grads<64, 128>(gp, rows, s->batch, s->n_kv, part, ksplit, st_, dev)
                       : launch_kl_grads<4, 32>(gp, rows, s->batch, s->n_kv, part, ksplit, st_, dev);
    if (e) return e;
  }
  return DSA_OK;
}

dsa_status dsa_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, dsa::g_error_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (word) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(dsa::g_error_word, &zero, sizeof(zero));
    if (word & dsa::kErrTimeout)
      return fail(DSA_ERR_TIMEOUT, "a device-side wait exceeded its limit (error word 0x%x)", word);
    if (word & dsa::kErrInternal)
      return fail(DSA_ERR_CUDA, "a kernel invariant failed (error word 0x%x)", word);
    if (word & dsa::kErrBadInput)
      return fail(DSA_ERR_INVALID_ARG,
                  "a block-table page was outside the key pool; its keys were skipped "
                  "(error word 0x%x)",
                  word);
    return fail(DSA_ERR_CUDA, "device error word 0x%x", word);
  }
  return DSA_OK;
}

}  // extern "C"
