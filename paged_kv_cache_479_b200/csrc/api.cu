// api.cu -- the C ABI of libpkv (declared in include/pkv.h): host-side
// argument checks, workspace sizing, the bulk-tensor map of the KV pool, and
// kernel launches.  No memory is allocated and no stream is synchronised
// here, except in pkv_read_error_word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "partition.cuh"
#include "pkv.h"

namespace {

thread_local char g_err[512] = "";

pkv_status fail(pkv_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

pkv_status ok() {
  g_err[0] = '\0';
  return PKV_OK;
}

pkv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

bool is_fp8(int dtype) { return dtype == PKV_FP8_E4M3 || dtype == PKV_FP8_E5M2; }

bool valid_page_size(int ps) { return ps == 16 || ps == 32 || ps == 64 || ps == 128 || ps == 256; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kDecodeHeadDim = 128;
constexpr int kMaxGroup = 8;
constexpr int kMaxShortCols = 16;  // short chunks: q_len * G columns per (request, kv head)
constexpr int kMaxPartitions = 1 << 20;

// workspace layout: counters int32[N] | part_lse float[2N][C] | part_o float[2N][C][128],
// C = state columns per slot (G for the decode, 8 or 16 for short chunks)
struct WsLayout {
  size_t counters, part_lse, part_o, total;
};

WsLayout ws_layout(int group, int N) {
  WsLayout w;
  w.counters = 0;
  w.part_lse = align_up((size_t)N * 4, 256);
  w.part_o = w.part_lse + align_up((size_t)2 * N * group * 4, 256);
  w.total = w.part_o + align_up((size_t)2 * N * group * kDecodeHeadDim * 4, 256);
  return w;
}

int current_device_partitions() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return pkv_default_partitions(dev);
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

struct MapKey {
  const void* pool;
  long long pages;
  int ps, hkv, dtype, layout, device, halves;
  bool operator==(const MapKey& o) const {
    return pool == o.pool && pages == o.pages && ps == o.ps && hkv == o.hkv && dtype == o.dtype &&
           layout == o.layout && device == o.device && halves == o.halves;
  }
};

// Tensor map of the pool for the kernels' bulk-tensor loads.  Preferred form,
// 5-D: (dim % 64, slot, dim / 64, kv head, 2 page + K/V) with boxes of
// [2][16 slots][64 dims] -- one load brings a tile's whole K (or V) into
// shared memory as two 128-byte-swizzled [16][64] halves.  Both pool layouts
// (HND [page][2][head][slot][dim], NHD [page][2][slot][head][dim]) are this
// view with different strides.  If the driver rejected the 5-D form (its
// strides are not increasing), the HND pool falls back to the 4-D form
// (dim, slot, K/V * Hkv + head, page) with [16][64] boxes: two loads per K or
// V tile, same shared-memory layout.
// halves: dim-halves per box of the 16-bit 5-D view -- 2 (the decode and prefix
// kernels: a [2][16][64] box is one K or V tile) or 1 (the tcgen05 kernel: a
// [16][64] box per half, so each half of a 64-token tile is contiguous).
pkv_status pool_tensor_map(const void* pool, long long pages, int ps, int hkv, int dtype, int layout,
                           CUtensorMap* out, int* one_box, int halves = 2) {
  static std::mutex mu;
  static MapKey keys[16];
  static CUtensorMap maps[16];
  static int kinds[16];
  static int used = 0, next = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  const MapKey key{pool, pages, ps, hkv, dtype, layout, dev, is_fp8(dtype) ? 2 : halves};
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
      if (keys[i] == key) {
        *out = maps[i];
        *one_box = kinds[i];
        return PKV_OK;
      }
  }
  auto encode = get_encode();
  if (!encode) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (is_fp8(dtype)) {
    // 8-bit pool: 4-D view (byte of the row, slot, kv head, 2 page + K/V) with
    // [2][16 slots][128 bytes] boxes -- one load brings a tile's K and V
    const bool nhd = layout == PKV_LAYOUT_NHD;
    const cuuint64_t row = kDecodeHeadDim;  // one token's K (or V) row: 128 bytes
    cuuint64_t dims[4] = {row, (cuuint64_t)ps, (cuuint64_t)hkv, (cuuint64_t)2 * pages};
    cuuint64_t strides[3] = {nhd ? (cuuint64_t)hkv * row : row, nhd ? row : (cuuint64_t)ps * row,
                             (cuuint64_t)hkv * ps * row};
    cuuint32_t box[4] = {(cuuint32_t)row, (cuuint32_t)pkv::kTileTokens, 1, 2};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap m8;
    const CUresult r8 = encode(&m8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(pool), dims,
                               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r8 != CUDA_SUCCESS)
      return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed for the 8-bit pool (%d)", (int)r8);
    std::lock_guard<std::mutex> lk(mu);
    keys[next] = key;
    maps[next] = m8;
    kinds[next] = 2;
    next = (next + 1) % 16;
    if (used < 16) ++used;
    *out = m8;
    *one_box = 2;
    return PKV_OK;
  }
  const CUtensorMapDataType dt =
      dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t row = (cuuint64_t)kDecodeHeadDim * 2;  // bytes of one token's K (or V) row
  CUtensorMap m;
  int kind = 0;
  CUresult r = CUDA_ERROR_INVALID_VALUE;
#ifndef PKV_FORCE_4D_MAP
  {
    const bool nhd = layout == PKV_LAYOUT_NHD;
    cuuint64_t dims[5] = {64, (cuuint64_t)ps, 2, (cuuint64_t)hkv, (cuuint64_t)2 * pages};
    cuuint64_t strides[4] = {nhd ? (cuuint64_t)hkv * row : row, 128,
                             nhd ? row : (cuuint64_t)ps * row, (cuuint64_t)hkv * ps * row};
    cuuint32_t box[5] = {64, (cuuint32_t)pkv::kTileTokens, (cuuint32_t)halves, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    r = encode(&m, dt, 5, const_cast<void*>(pool), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    kind = 1;
  }
#endif
  if (r != CUDA_SUCCESS && layout == PKV_LAYOUT_NHD)
    return fail(PKV_ERR_UNSUPPORTED, "the driver rejected the 5-D tensor map the NHD layout needs");
  if (r != CUDA_SUCCESS) {
    cuuint64_t dims[4] = {(cuuint64_t)kDecodeHeadDim, (cuuint64_t)ps, (cuuint64_t)2 * hkv,
                          (cuuint64_t)pages};
    cuuint64_t strides[3] = {row, (cuuint64_t)ps * row, (cuuint64_t)2 * hkv * ps * row};
    cuuint32_t box[4] = {64, (cuuint32_t)pkv::kTileTokens, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    r = encode(&m, dt, 4, const_cast<void*>(pool), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    kind = 0;
  }
  if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  {
    std::lock_guard<std::mutex> lk(mu);
    keys[next] = key;
    maps[next] = m;
    kinds[next] = kind;
    next = (next + 1) % 16;
    if (used < 16) ++used;
  }
  *out = m;
  *one_box = kind;
  return PKV_OK;
}

}  // namespace

namespace pkv {

// q [nnz_q][hq][128] (16-bit) as (dim % 64, dim / 64, head, token): a box of
// [128 / G tokens][G heads][64 dims] is one dim half of a 128-row tile of the
// tcgen05 kernel, rows (token, head) in order, 128-byte swizzled
bool chunk_q_map(const void* q, long long nnz_q, int hq, int group, bool bf16, CUtensorMap* m) {
  auto encode = get_encode();
  if (!encode || group < 1 || 128 % group != 0 || hq < group || nnz_q < 1 ||
      nnz_q > 0x7fffffffLL || !aligned(q, 16))
    return false;
  cuuint64_t dims[4] = {64, 2, (cuuint64_t)hq, (cuuint64_t)nnz_q};
  cuuint64_t strides[3] = {128, 256, (cuuint64_t)hq * 256};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)group, (cuuint32_t)(128 / group)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 states [nnz_q][states][hq][128] as (dim % 32, dim / 32, head, slot,
// token): a box of [128 / G tokens][G heads][32 dims] is a quarter of a
// 128-row tile's states in one slot, 128-byte swizzled
bool chunk_state_map(float* state_o, long long nnz_q, int states, int hq, int group,
                     CUtensorMap* m) {
  auto encode = get_encode();
  if (!encode || !state_o || group < 1 || 128 % group != 0 || hq < group || states < 1 ||
      nnz_q < 1 || nnz_q > 0x7fffffffLL || !aligned(state_o, 16))
    return false;
  cuuint64_t dims[5] = {32, 4, (cuuint64_t)hq, (cuuint64_t)states, (cuuint64_t)nnz_q};
  cuuint64_t strides[4] = {128, 512, (cuuint64_t)hq * 512, (cuuint64_t)states * hq * 512};
  cuuint32_t box[5] = {32, 1, (cuuint32_t)group, 1, (cuuint32_t)(128 / group)};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, state_o, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pkv

namespace {
// the decode kernel's wait limit (pkv_set_wait_limit_ns); 0 selects the default
std::atomic<unsigned long long> g_wait_ns{0};
}  // namespace

size_t pkv::decode_counter_bytes(int group, int num_partitions) {
  const int N = num_partitions ? num_partitions : current_device_partitions();
  if (N <= 0 || N > kMaxPartitions || group < 1) return 0;
  return ws_layout(group, N).part_lse;
}

unsigned long long pkv::decode_wait_limit_ns() {
  const unsigned long long v = g_wait_ns.load(std::memory_order_relaxed);
  return v ? v : (unsigned long long)pkv::kWaitLimitNs;
}

cudaError_t pkv::ensure_smem_opt_in(const void* func, size_t bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({func, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  done.insert({func, dev});
  return cudaSuccess;
}

pkv_status pkv::set_error(pkv_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

// dtype: type of q and out; kv_dtype: the pool's (dtype, or PKV_FP8_E4M3 /
// PKV_FP8_E5M2 with k_scale / v_scale)
static pkv_status decode_impl(const void* q, int num_qo_heads, const void* pool, int64_t num_pages,
                      int page_size, int num_kv_heads, int head_dim, int dtype, int layout,
                      const pkv::TableView& tv, const int32_t* page_ids, int batch, float sm_scale,
                      int num_partitions, void* workspace, size_t workspace_bytes, void* out,
                      float* lse, int32_t* error_word, void* stream, int out_f32,
                      long long out_rs, long long lse_rs, int kv_dtype = -1,
                      float k_scale = 1.f, float v_scale = 1.f,
                      const int32_t* qo_indptr = nullptr, int64_t nnz_q = 0, int max_q_len = 1,
                      const void* k_new = nullptr, const void* v_new = nullptr,
                      const int32_t* append_indptr = nullptr, int64_t nnz_new = 0,
                      int early_table = 0) {
  if (kv_dtype < 0) kv_dtype = dtype;
  if (batch < 0 || num_pages < 1 || num_kv_heads < 1 || num_qo_heads < 1)
    return fail(PKV_ERR_INVALID_ARG, "sizes out of range");
  if (dtype != PKV_F16 && dtype != PKV_BF16)
    return fail(PKV_ERR_INVALID_ARG, "dtype must be PKV_F16 or PKV_BF16");
  if (kv_dtype != dtype && !is_fp8(kv_dtype))
    return fail(PKV_ERR_INVALID_ARG, "the pool must hold q's type or 8-bit (E4M3 / E5M2) codes");
  if (is_fp8(kv_dtype) &&
      !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
    return fail(PKV_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive");
  if (num_qo_heads % num_kv_heads != 0)
    return fail(PKV_ERR_INVALID_ARG, "num_qo_heads must be a multiple of num_kv_heads");
  if (head_dim != kDecodeHeadDim) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 128");
  const int group = num_qo_heads / num_kv_heads;
  // columns per (request, kv head): G heads of each of up to max_q_len tokens
  const int64_t cols = (int64_t)group * (qo_indptr ? max_q_len : 1);
  if (qo_indptr && (max_q_len < 1 || cols > kMaxShortCols))
    return fail(PKV_ERR_UNSUPPORTED, "short chunks need 1 <= max_q_len and max_q_len * G <= 16");
  if (!qo_indptr && group > kMaxGroup) return fail(PKV_ERR_UNSUPPORTED, "GQA group must be 1..8");
  const int nq = cols > kMaxGroup ? 2 : 1;
  const int pcols = qo_indptr ? kMaxGroup * nq : group;
  if (!valid_page_size(page_size))
    return fail(PKV_ERR_UNSUPPORTED, "page_size must be 16, 32, 64, 128 or 256");
  if (num_pages > 0x7fffffffLL) return fail(PKV_ERR_UNSUPPORTED, "more than 2^31-1 pages");
  if (!std::isfinite(sm_scale)) return fail(PKV_ERR_INVALID_ARG, "sm_scale is not finite");
  if (num_partitions < 0 || num_partitions > kMaxPartitions)
    return fail(PKV_ERR_INVALID_ARG, "num_partitions out of range");
  if (layout != PKV_LAYOUT_HND && layout != PKV_LAYOUT_NHD)
    return fail(PKV_ERR_INVALID_ARG, "layout must be PKV_LAYOUT_HND or PKV_LAYOUT_NHD");
  if (batch == 0) return ok();
  if (!q || !pool || !page_ids || !out || !workspace ||
      (tv.indptr ? !tv.last_len : (!tv.context_lens || tv.max_blocks < 1)))
    return fail(PKV_ERR_INVALID_ARG, "null pointer or empty block table");
  if (!aligned(q, 16) || !aligned(pool, 16) || !aligned(out, 16))
    return fail(PKV_ERR_INVALID_ARG, "q, pool and out must be 16-byte aligned");
  if (out == q || out == pool) return fail(PKV_ERR_INVALID_ARG, "out aliases q or pool");
  const bool fused = nnz_new > 0;
  if (nnz_new < 0) return fail(PKV_ERR_INVALID_ARG, "nnz_new < 0");
  if (fused) {
    if (kv_dtype != dtype) return fail(PKV_ERR_INVALID_ARG, "a fused append needs a 16-bit pool");
    if (!k_new || !v_new || !append_indptr)
      return fail(PKV_ERR_INVALID_ARG, "null k_new, v_new or append_indptr");
    if (!aligned(k_new, 16) || !aligned(v_new, 16))
      return fail(PKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
    if (nnz_new * (int64_t)num_kv_heads > (int64_t)1 << 40)
      return fail(PKV_ERR_UNSUPPORTED, "too many new rows");
  }
  int N = num_partitions;
  if (N == 0) N = current_device_partitions();
  if (N <= 0) return fail(PKV_ERR_CUDA, "cannot query the SM count");
  const WsLayout L = ws_layout(pcols, N);
  if (!aligned(workspace, 256)) return fail(PKV_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (workspace_bytes < L.total)
    return fail(PKV_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, L.total);

  CUtensorMap tmap;
  int one_box = 0;
  pkv_status st =
      pool_tensor_map(pool, num_pages, page_size, num_kv_heads, kv_dtype, layout, &tmap, &one_box);
  if (st != PKV_OK) return st;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pkv::DecodeArgs a;
  a.q = q;
  a.out = out;
  a.lse = lse;
  a.tv = tv;
  a.indices = page_ids;
  a.counters = reinterpret_cast<int*>(ws + L.counters);
  a.part_lse = reinterpret_cast<float*>(ws + L.part_lse);
  a.part_o = reinterpret_cast<float*>(ws + L.part_o);
  a.err = reinterpret_cast<int*>(error_word);
  a.num_pages = num_pages;
  a.batch = batch;
  a.hq = num_qo_heads;
  a.hkv = num_kv_heads;
  a.group = group;
  a.page_size = page_size;
  const bool fp8 = is_fp8(kv_dtype);
  a.scale_log2 = (float)((double)sm_scale * 1.4426950408889634 * (fp8 ? (double)k_scale : 1.0));
  a.v_scale = fp8 ? v_scale : 1.f;
  a.one_box = one_box;
  a.out_f32 = out_f32;
  a.out_rs = out_rs;
  a.lse_rs = lse_rs;
  a.qo_indptr = qo_indptr;
  a.nnz_q = nnz_q;
  a.pcols = pcols;
  a.max_cols = (int)cols;
  a.pool = const_cast<void*>(pool);
  a.layout = layout;
  a.k_new = fused ? k_new : nullptr;
  a.v_new = fused ? v_new : nullptr;
  a.append_indptr = fused ? append_indptr : nullptr;
  a.nnz_new = fused ? nnz_new : 0;
  a.wait_ns = pkv::decode_wait_limit_ns();
  a.early_table = early_table;
  cudaError_t e =
      pkv::launch_decode(tmap, a, dtype == PKV_BF16,
                         kv_dtype == PKV_FP8_E4M3 ? pkv::kKvE4M3
                         : kv_dtype == PKV_FP8_E5M2 ? pkv::kKvE5M2 : pkv::kKv16,
                         nq, N, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

// dtype: type of k_new / v_new; kv_dtype: the pool's (dtype, or an 8-bit
// type: the rows are quantised with k_scale / v_scale)
static pkv_status append_impl(void* pool, int64_t num_pages, int page_size, int num_kv_heads,
                              int head_dim, int dtype, int layout, const pkv::TableView& tv,
                              const int32_t* page_ids, int batch, const void* k_new,
                              const void* v_new, const int32_t* append_indptr, int64_t nnz_new,
                              int32_t* error_word, void* stream, int kv_dtype = -1,
                              float k_scale = 1.f, float v_scale = 1.f) {
  if (kv_dtype < 0) kv_dtype = dtype;
  if (batch < 0 || nnz_new < 0 || num_pages < 0 || page_size < 1 || num_kv_heads < 1)
    return fail(PKV_ERR_INVALID_ARG, "negative or zero size");
  if (dtype != PKV_F16 && dtype != PKV_BF16)
    return fail(PKV_ERR_INVALID_ARG, "dtype must be PKV_F16 or PKV_BF16");
  if (kv_dtype != dtype && !is_fp8(kv_dtype))
    return fail(PKV_ERR_INVALID_ARG, "the pool must hold the rows' type or 8-bit codes");
  if (is_fp8(kv_dtype) &&
      !(k_scale > 0.f && v_scale > 0.f && std::isfinite(k_scale) && std::isfinite(v_scale)))
    return fail(PKV_ERR_INVALID_ARG, "k_scale and v_scale must be finite and positive");
  if (layout != PKV_LAYOUT_HND && layout != PKV_LAYOUT_NHD)
    return fail(PKV_ERR_INVALID_ARG, "layout must be PKV_LAYOUT_HND or PKV_LAYOUT_NHD");
  if (head_dim < 8 || head_dim % 8 != 0)
    return fail(PKV_ERR_UNSUPPORTED, "append needs head_dim a positive multiple of 8");
  if (nnz_new == 0 || batch == 0) return ok();
  if (!pool || !page_ids || !k_new || !v_new || !append_indptr ||
      (tv.indptr ? !tv.last_len : (!tv.context_lens || tv.max_blocks < 1)))
    return fail(PKV_ERR_INVALID_ARG, "null pointer or empty block table");
  if (!aligned(pool, 16) || !aligned(k_new, 16) || !aligned(v_new, 16))
    return fail(PKV_ERR_INVALID_ARG, "pool, k_new and v_new must be 16-byte aligned");
  if (nnz_new * (int64_t)num_kv_heads > (int64_t)1 << 40)
    return fail(PKV_ERR_UNSUPPORTED, "too many new rows");
  pkv::AppendArgs a;
  a.pool = pool;
  a.tv = tv;
  a.indices = page_ids;
  a.append_indptr = append_indptr;
  a.k_new = k_new;
  a.v_new = v_new;
  a.err = reinterpret_cast<int*>(error_word);
  a.num_pages = num_pages;
  a.nnz = nnz_new;
  a.batch = batch;
  a.hkv = num_kv_heads;
  a.head_dim = head_dim;
  a.page_size = page_size;
  a.layout = layout;
  a.fp8 = kv_dtype == PKV_FP8_E4M3 ? pkv::kKvE4M3 : kv_dtype == PKV_FP8_E5M2 ? pkv::kKvE5M2 : 0;
  a.in_bf16 = dtype == PKV_BF16;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  cudaError_t e = pkv::launch_append(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return ok();
}

// unpack the descriptors of the _ex calls
static pkv_status table_view(const pkv_table_desc* t, pkv::TableView* tv, const int32_t** ids) {
  if (!t) return fail(PKV_ERR_INVALID_ARG, "null table descriptor");
  if (t->flags & ~PKV_TABLE_READY_AT_LAUNCH)
    return fail(PKV_ERR_INVALID_ARG, "unknown table flags 0x%x", (unsigned)t->flags);
  if (t->kind == PKV_TABLE_CSR) {
    *tv = pkv::csr_view(t->page_indptr, t->last_page_len);
    *ids = t->page_indices;
    if (t->batch > 0 && !t->page_indptr) return fail(PKV_ERR_INVALID_ARG, "null page_indptr");
    return PKV_OK;
  }
  if (t->kind == PKV_TABLE_BLOCK) {
    tv->indptr = nullptr;
    tv->last_len = nullptr;
    tv->context_lens = t->context_lens;
    tv->max_blocks = t->max_blocks_per_seq;
    *ids = t->block_table;
    return PKV_OK;
  }
  return fail(PKV_ERR_INVALID_ARG, "table kind must be PKV_TABLE_CSR or PKV_TABLE_BLOCK");
}

extern "C" {

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "PKV_OK";
    case PKV_ERR_INVALID_ARG: return "PKV_ERR_INVALID_ARG";
    case PKV_ERR_UNSUPPORTED: return "PKV_ERR_UNSUPPORTED";
    case PKV_ERR_WORKSPACE: return "PKV_ERR_WORKSPACE";
    case PKV_ERR_CUDA: return "PKV_ERR_CUDA";
    case PKV_ERR_DEVICE: return "PKV_ERR_DEVICE";
    default: return "PKV_ERR_UNKNOWN";
  }
}

const char* pkv_last_error(void) { return g_err; }

uint64_t pkv_set_wait_limit_ns(uint64_t nanoseconds) {
  const unsigned long long prev = pkv::decode_wait_limit_ns();
  g_wait_ns.store(nanoseconds, std::memory_order_relaxed);
  return prev;
}

int pkv_default_partitions(int device) {
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return -1;
  return sms * pkv::kDecodeCtasPerSm;  // persistent decode CTAs resident at once
}

size_t pkv_decode_workspace_bytes(int batch, int num_qo_heads, int num_kv_heads, int head_dim,
                                  int num_partitions) {
  if (batch < 0 || num_kv_heads < 1 || num_qo_heads < num_kv_heads ||
      num_qo_heads % num_kv_heads != 0 || head_dim != kDecodeHeadDim)
    return 0;
  const int group = num_qo_heads / num_kv_heads;
  if (group > kMaxGroup) return 0;
  int N = num_partitions;
  if (N == 0) N = current_device_partitions();
  if (N <= 0 || N > kMaxPartitions) return 0;
  return ws_layout(group, N).total;
}

pkv_status pkv_check_table(const int32_t* page_indptr_h, const int32_t* page_indices_h,
                           const int32_t* last_page_len_h, int batch, int64_t num_pages,
                           int page_size) {
  if (batch < 0 || page_size < 1 || num_pages < 0)
    return fail(PKV_ERR_INVALID_ARG, "batch, page_size or num_pages out of range");
  if (batch > 0 && (!page_indptr_h || !last_page_len_h))
    return fail(PKV_ERR_INVALID_ARG, "null table pointer");
  if (batch == 0) return ok();
  if (page_indptr_h[0] < 0) return fail(PKV_ERR_INVALID_ARG, "page_indptr[0] < 0");
  for (int b = 0; b < batch; ++b) {
    const pkv::ReqInfo r = pkv::request_info(pkv::csr_view(page_indptr_h, last_page_len_h), b, page_size);
    if (r.err & pkv::kErrIndptr)
      return fail(PKV_ERR_INVALID_ARG, "page_indptr decreases at request %d", b);
    if (r.err & pkv::kErrLastLen)
      return fail(PKV_ERR_INVALID_ARG, "last_page_len[%d] = %d outside [1, %d]", b,
                  last_page_len_h[b], page_size);
  }
  if (page_indptr_h[batch] > 0 && !page_indices_h)
    return fail(PKV_ERR_INVALID_ARG, "null page_indices");
  for (int32_t i = page_indptr_h[0]; i < page_indptr_h[batch]; ++i)
    if (page_indices_h[i] < 0 || page_indices_h[i] >= num_pages)
      return fail(PKV_ERR_INVALID_ARG, "page_indices[%d] = %d outside [0, %lld)", i,
                  page_indices_h[i], (long long)num_pages);
  return ok();
}

int64_t pkv_plan_segments(const int32_t* page_indptr_h, const int32_t* last_page_len_h,
                          int batch, int page_size, int num_kv_heads, int num_partitions,
                          int64_t* segments, int64_t max_segments) {
  if (batch < 0 || !valid_page_size(page_size) || num_kv_heads < 1 || num_partitions < 1 ||
      num_partitions > kMaxPartitions || (batch > 0 && (!page_indptr_h || !last_page_len_h)))
    return -1;
  long long total = 0;
  for (int b = 0; b < batch; ++b)
    total += pkv::request_info(pkv::csr_view(page_indptr_h, last_page_len_h), b, page_size).units;
  const long long W = (long long)num_kv_heads * total;
  if (W == 0) return 0;
  // the kernel uses min(num_partitions, W) partitions: none of them is empty
  const int N = W < num_partitions ? (int)W : num_partitions;
  int64_t count = 0;
  for (int c = 0; c < N; ++c) {
    const long long f0 = pkv::part_start(W, N, c), f1 = pkv::part_start(W, N, c + 1);
    if (f0 >= f1) continue;
    // locate the request holding f0 (the device does this with a block scan)
    long long Cb = 0;
    int b0 = -1;
    pkv::ReqInfo r0{};
    for (int b = 0; b < batch; ++b) {
      const pkv::ReqInfo r = pkv::request_info(pkv::csr_view(page_indptr_h, last_page_len_h), b, page_size);
      if (r.units > 0 && (long long)num_kv_heads * Cb <= f0 &&
          f0 < (long long)num_kv_heads * (Cb + r.units)) {
        b0 = b;
        r0 = r;
        break;
      }
      Cb += r.units;
    }
    if (b0 < 0) return -1;
    pkv::Walk wk;
    wk.tv = pkv::csr_view(page_indptr_h, last_page_len_h);
    wk.B = batch;
    wk.ps = page_size;
    wk.Hkv = num_kv_heads;
    wk.start(b0, Cb, r0, f0, f1);
    while (!wk.done()) {
      const long long t0 = wk.t0(), t1 = wk.t1();
      if (t1 > t0) {
        // the kernel's form (no division for pair ends inside the share)
        const pkv::SegPlace pl = pkv::seg_place_in(W, N, wk.pair_start(), wk.ri.units, c, f0, f1);
        if (segments && count < max_segments) {
          int64_t* row = segments + 7 * count;
          row[0] = c;
          row[1] = wk.b;
          row[2] = wk.kvh;
          row[3] = t0;
          row[4] = t1;
          row[5] = pl.slot;
          row[6] = pl.ncover;
        }
        ++count;
      }
      wk.advance();
    }
  }
  return count;
}

pkv_status pkv_append(void* pool, int64_t num_pages, int page_size, int num_kv_heads,
                      int head_dim, int dtype, const int32_t* page_indptr,
                      const int32_t* page_indices, const int32_t* last_page_len, int batch,
                      const void* k_new, const void* v_new, const int32_t* append_indptr,
                      int64_t nnz_new, int32_t* error_word, void* stream) {
  return append_impl(pool, num_pages, page_size, num_kv_heads, head_dim, dtype, PKV_LAYOUT_HND,
                     pkv::csr_view(page_indptr, last_page_len), page_indices, batch, k_new, v_new,
                     append_indptr, nnz_new, error_word, stream);
}

pkv_status pkv_decode(const void* q, int num_qo_heads, const void* pool, int64_t num_pages,
                      int page_size, int num_kv_heads, int head_dim, int dtype,
                      const int32_t* page_indptr, const int32_t* page_indices,
                      const int32_t* last_page_len, int batch, float sm_scale,
                      int num_partitions, void* workspace, size_t workspace_bytes, void* out,
                      float* lse, int32_t* error_word, void* stream) {
  return decode_impl(q, num_qo_heads, pool, num_pages, page_size, num_kv_heads, head_dim, dtype,
                     PKV_LAYOUT_HND, pkv::csr_view(page_indptr, last_page_len), page_indices,
                     batch, sm_scale, num_partitions, workspace, workspace_bytes, out, lse,
                     error_word, stream, 0, (long long)num_qo_heads * kDecodeHeadDim,
                     num_qo_heads);
}

pkv_status pkv_decode_append(const void* q, int num_qo_heads, const pkv_pool_desc* pool,
                             const pkv_table_desc* table, const void* k_new, const void* v_new,
                             const int32_t* append_indptr, int64_t nnz_new, float sm_scale,
                             int num_partitions, void* workspace, size_t workspace_bytes,
                             void* out, float* lse, int32_t* error_word, void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  if (is_fp8(pool->dtype))
    return fail(PKV_ERR_INVALID_ARG, "the fused append takes 16-bit pools (8-bit: pkv_append_fp8)");
  if (nnz_new < 0) return fail(PKV_ERR_INVALID_ARG, "nnz_new < 0");
  if (nnz_new > 0 && (pool->data == k_new || pool->data == v_new || out == k_new || out == v_new))
    return fail(PKV_ERR_INVALID_ARG, "k_new / v_new alias the pool or out");
  return decode_impl(q, num_qo_heads, pool->data, pool->num_pages, pool->page_size,
                     pool->num_kv_heads, pool->head_dim, pool->dtype, pool->layout, tv, ids,
                     table->batch, sm_scale, num_partitions, workspace, workspace_bytes, out, lse,
                     error_word, stream, 0, (long long)num_qo_heads * kDecodeHeadDim,
                     num_qo_heads, -1, 1.f, 1.f, nullptr, 0, 1, k_new, v_new, append_indptr,
                     nnz_new, table->flags & PKV_TABLE_READY_AT_LAUNCH);
}

pkv_status pkv_decode_ex(const void* q, int num_qo_heads, const pkv_pool_desc* pool,
                         const pkv_table_desc* table, float sm_scale, int num_partitions,
                         void* workspace, size_t workspace_bytes, void* out, float* lse,
                         int32_t* error_word, void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  if (is_fp8(pool->dtype))
    return fail(PKV_ERR_INVALID_ARG, "an 8-bit pool needs pkv_decode_fp8 (it carries the scales)");
  return decode_impl(q, num_qo_heads, pool->data, pool->num_pages, pool->page_size,
                     pool->num_kv_heads, pool->head_dim, pool->dtype, pool->layout, tv, ids,
                     table->batch, sm_scale, num_partitions, workspace, workspace_bytes, out, lse,
                     error_word, stream, 0, (long long)num_qo_heads * kDecodeHeadDim,
                     num_qo_heads, -1, 1.f, 1.f, nullptr, 0, 1, nullptr, nullptr, nullptr, 0,
                     table->flags & PKV_TABLE_READY_AT_LAUNCH);
}

pkv_status pkv_append_ex(const pkv_pool_desc* pool, const pkv_table_desc* table,
                         const void* k_new, const void* v_new, const int32_t* append_indptr,
                         int64_t nnz_new, int32_t* error_word, void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  if (is_fp8(pool->dtype))
    return fail(PKV_ERR_INVALID_ARG, "an 8-bit pool needs pkv_append_fp8 (it carries the scales)");
  return append_impl(pool->data, pool->num_pages, pool->page_size, pool->num_kv_heads,
                     pool->head_dim, pool->dtype, pool->layout, tv, ids, table->batch, k_new,
                     v_new, append_indptr, nnz_new, error_word, stream);
}

pkv_status pkv_decode_fp8(const void* q, int q_dtype, int num_qo_heads, const pkv_pool_desc* pool,
                          float k_scale, float v_scale, const pkv_table_desc* table,
                          float sm_scale, int num_partitions, void* workspace,
                          size_t workspace_bytes, void* out, float* lse, int32_t* error_word,
                          void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  if (!is_fp8(pool->dtype))
    return fail(PKV_ERR_INVALID_ARG, "pool dtype must be PKV_FP8_E4M3 or PKV_FP8_E5M2");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  return decode_impl(q, num_qo_heads, pool->data, pool->num_pages, pool->page_size,
                     pool->num_kv_heads, pool->head_dim, q_dtype, pool->layout, tv, ids,
                     table->batch, sm_scale, num_partitions, workspace, workspace_bytes, out, lse,
                     error_word, stream, 0, (long long)num_qo_heads * kDecodeHeadDim,
                     num_qo_heads, pool->dtype, k_scale, v_scale, nullptr, 0, 1, nullptr, nullptr,
                     nullptr, 0, table->flags & PKV_TABLE_READY_AT_LAUNCH);
}

pkv_status pkv_append_fp8(const pkv_pool_desc* pool, float k_scale, float v_scale,
                          const pkv_table_desc* table, const void* k_new, const void* v_new,
                          int new_dtype, const int32_t* append_indptr, int64_t nnz_new,
                          int32_t* error_word, void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  if (!is_fp8(pool->dtype))
    return fail(PKV_ERR_INVALID_ARG, "pool dtype must be PKV_FP8_E4M3 or PKV_FP8_E5M2");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  return append_impl(pool->data, pool->num_pages, pool->page_size, pool->num_kv_heads,
                     pool->head_dim, new_dtype, pool->layout, tv, ids, table->batch, k_new, v_new,
                     append_indptr, nnz_new, error_word, stream, pool->dtype, k_scale, v_scale);
}

}  // extern "C"

namespace {

// Shared-prefix cascade: the prefix step's grid (row blocks x kv heads x key
// splits) and the fp32 attention states it and the suffix decode write.
struct CascadePlan {
  int row_blocks, splits, states;
  size_t state_o, state_lse, decode_ws, total;  // byte offsets / size
};

CascadePlan cascade_plan(int batch, int hq, int hkv, long long prefix_len, int N, int sms) {
  CascadePlan p;
  const int G = hq / hkv;
  const long long rows = (long long)batch * G;
  const int R = pkv::chunk_rows_per_cta(), T = pkv::chunk_tile_tokens();
  p.row_blocks = (int)((rows + R - 1) / R);
  const long long tiles = (prefix_len + T - 1) / T;
  const long long units = (long long)p.row_blocks * hkv;
  // key splits: the count that minimises (waves of CTAs) x (tiles per CTA), one
  // CTA per SM being resident, plus half a tile per split for its state's share
  // of the merge -- ceil(sms / units) splits can spill a few CTAs into a second
  // wave that doubles the step (32 units on 148 SMs: 5 splits = 160 CTAs)
  long long splits = 1;
  if (units < sms && tiles > 1) {
    double best = 1e300;
    for (long long sp = 1; sp <= tiles && sp <= 64; ++sp) {
      const long long waves = (units * sp + sms - 1) / sms;
      const double cost = (double)(waves * ((tiles + sp - 1) / sp)) + 0.5 * (double)sp;
      if (cost < best) {
        best = cost;
        splits = sp;
      }
    }
  }
  p.splits = (int)splits;
  p.states = p.splits + 1;
  p.state_o = 0;
  p.state_lse = align_up((size_t)batch * p.states * hq * kDecodeHeadDim * 4, 256);
  p.decode_ws = p.state_lse + align_up((size_t)batch * p.states * hq * 4, 256);
  p.total = p.decode_ws + ws_layout(G, N).total;
  return p;
}

int current_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return sms;
}

}  // namespace

extern "C" {

size_t pkv_cascade_workspace_bytes(int batch, int num_qo_heads, int num_kv_heads, int head_dim,
                                   int64_t prefix_len, int num_partitions) {
  const size_t dec = pkv_decode_workspace_bytes(batch, num_qo_heads, num_kv_heads, head_dim,
                                                num_partitions);
  if (dec == 0 || prefix_len < 0) return 0;
  if (prefix_len == 0) return dec;
  int N = num_partitions ? num_partitions : current_device_partitions();
  const int sms = current_sms();
  if (N <= 0 || sms <= 0) return 0;
  return cascade_plan(batch, num_qo_heads, num_kv_heads, prefix_len, N, sms).total;
}

pkv_status pkv_cascade_decode(const void* q, int num_qo_heads, const void* pool, int64_t num_pages,
                              int page_size, int num_kv_heads, int head_dim, int dtype,
                              const int32_t* prefix_page_indices, int64_t prefix_len,
                              const int32_t* page_indptr, const int32_t* page_indices,
                              const int32_t* last_page_len, int batch, float sm_scale,
                              int num_partitions, void* workspace, size_t workspace_bytes,
                              void* out, float* lse, int32_t* error_word, void* stream) {
  if (prefix_len < 0) return fail(PKV_ERR_INVALID_ARG, "prefix_len < 0");
  if (prefix_len == 0 || batch == 0)
    return pkv_decode(q, num_qo_heads, pool, num_pages, page_size, num_kv_heads, head_dim, dtype,
                      page_indptr, page_indices, last_page_len, batch, sm_scale, num_partitions,
                      workspace, workspace_bytes, out, lse, error_word, stream);
  if (batch < 0 || num_pages < 1 || num_kv_heads < 1 || num_qo_heads < 1 ||
      num_qo_heads % num_kv_heads != 0)
    return fail(PKV_ERR_INVALID_ARG, "sizes out of range");
  if (dtype != PKV_F16 && dtype != PKV_BF16)
    return fail(PKV_ERR_INVALID_ARG, "dtype must be PKV_F16 or PKV_BF16");
  if (head_dim != kDecodeHeadDim) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 128");
  const int group = num_qo_heads / num_kv_heads;
  if (group > kMaxGroup) return fail(PKV_ERR_UNSUPPORTED, "GQA group must be 1..8");
  if (!valid_page_size(page_size))
    return fail(PKV_ERR_UNSUPPORTED, "page_size must be 16, 32, 64, 128 or 256");
  if (prefix_len > (int64_t)num_pages * page_size)
    return fail(PKV_ERR_INVALID_ARG, "prefix longer than the pool");
  if (!std::isfinite(sm_scale)) return fail(PKV_ERR_INVALID_ARG, "sm_scale is not finite");
  if (num_partitions < 0 || num_partitions > kMaxPartitions)
    return fail(PKV_ERR_INVALID_ARG, "num_partitions out of range");
  if (!q || !pool || !prefix_page_indices || !page_indptr || !page_indices || !last_page_len ||
      !out || !workspace)
    return fail(PKV_ERR_INVALID_ARG, "null pointer");
  if (!aligned(q, 16) || !aligned(pool, 16) || !aligned(out, 16))
    return fail(PKV_ERR_INVALID_ARG, "q, pool and out must be 16-byte aligned");
  if (out == q || out == pool) return fail(PKV_ERR_INVALID_ARG, "out aliases q or pool");
  if (!aligned(workspace, 256)) return fail(PKV_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  int N = num_partitions ? num_partitions : current_device_partitions();
  const int sms = current_sms();
  if (N <= 0 || sms <= 0) return fail(PKV_ERR_CUDA, "cannot query the SM count");
  const CascadePlan P = cascade_plan(batch, num_qo_heads, num_kv_heads, prefix_len, N, sms);
  if (workspace_bytes < P.total)
    return fail(PKV_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, P.total);

  CUtensorMap tmap;
  int one_box = 0;
  pkv_status st = pool_tensor_map(pool, num_pages, page_size, num_kv_heads, dtype, PKV_LAYOUT_HND,
                                  &tmap, &one_box, /*halves=*/1);
  if (st != PKV_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* state_o = reinterpret_cast<float*>(ws + P.state_o);
  float* state_lse = reinterpret_cast<float*>(ws + P.state_lse);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // 1. the shared prefix, once for every request's queries: state slots 0 .. splits-1
  pkv::ChunkArgs pa = {};
  pa.q = q;
  pa.prefix_pages = prefix_page_indices;
  pa.prefix_len = prefix_len;
  pa.state_o = state_o;
  pa.state_lse = state_lse;
  pa.states = P.states;
  pa.out_states = 1;
  pa.err = reinterpret_cast<int*>(error_word);
  pa.num_pages = num_pages;
  pa.nnz_q = batch;
  pa.page_size = page_size;
  pa.batch = batch;
  pa.hq = num_qo_heads;
  pa.hkv = num_kv_heads;
  pa.group = group;
  pa.splits = P.splits;
  pa.window_left = -1;
  pa.sink = 0;
  pa.scale_log2 = sm_scale * 1.4426950408889634f;
  pa.one_box = one_box;
  CUtensorMap qmap = {}, omap = {};
  pa.q_tma = pkv::chunk_q_map(q, batch, num_qo_heads, group, dtype == PKV_BF16, &qmap) ? 1 : 0;
  pa.o_tma = pkv::chunk_state_map(state_o, batch, P.states, num_qo_heads, group, &omap) ? 1 : 0;
  cudaError_t e = pkv::launch_chunk_tc(tmap, qmap, omap, pa, dtype == PKV_BF16, P.row_blocks, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefix launch");
  // 2. each request's own pages: the last state slot, as an fp32 state.  The
  // prefix launch lets it start once the prefix has waited for the kernels
  // before the cascade, and nothing in the cascade writes the own-page table:
  // it is read before this launch's dependency wait (its CTAs fill the SMs
  // the prefix leaves idle); q, the pool and the state slot only after it.
  st = decode_impl(q, num_qo_heads, pool, num_pages, page_size, num_kv_heads, head_dim, dtype,
                   PKV_LAYOUT_HND, pkv::csr_view(page_indptr, last_page_len), page_indices,
                   batch, sm_scale, N,
                   ws + P.decode_ws, workspace_bytes - P.decode_ws,
                   state_o + (size_t)P.splits * num_qo_heads * kDecodeHeadDim,
                   state_lse + (size_t)P.splits * num_qo_heads, error_word, stream, 1,
                   (long long)P.states * num_qo_heads * kDecodeHeadDim,
                   (long long)P.states * num_qo_heads, -1, 1.f, 1.f, nullptr, 0, 1, nullptr,
                   nullptr, nullptr, 0, /*early_table=*/1);
  if (st != PKV_OK) return st;
  // 3. merge the prefix and suffix states of every (request, head)
  pkv::MergeArgs ma;
  ma.v = state_o;
  ma.s = state_lse;
  ma.v_out = out;
  ma.s_out = lse;
  ma.rows = batch;
  ma.states = P.states;
  ma.heads = num_qo_heads;
  ma.head_dim = kDecodeHeadDim;
  ma.out_dtype = dtype;
  ma.vec4 = 1;
  ma.rows_ok = 1;
  e = pkv::launch_merge(ma, s);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

// ------------------------------------------------------------ append attention

int64_t pkv_append_attention_plan(const int32_t* qo_indptr_h, const int32_t* kv_len_h, int batch,
                                  int num_qo_heads, int num_kv_heads, int window_left,
                                  int sink_tokens, int num_sms, int32_t* plan_h,
                                  int64_t capacity, int32_t* num_splits) {
  if (batch < 0 || num_kv_heads < 1 || num_qo_heads < num_kv_heads ||
      num_qo_heads % num_kv_heads != 0 || sink_tokens < 0 || (batch > 0 && !qo_indptr_h) ||
      capacity < 0 || (batch > 0 && qo_indptr_h[0] != 0))
    return -1;
  const int G = num_qo_heads / num_kv_heads;
  const int R = pkv::chunk_rows_per_cta(), T = pkv::chunk_tile_tokens();
  struct Block {
    long long tiles;
    int32_t b, r0, n;
  };
  std::vector<Block> blocks;
  int64_t ctas = 0;
  long long max_tiles = 0;
  for (int b = 0; b < batch; ++b) {
    const long long q_len = (long long)qo_indptr_h[b + 1] - qo_indptr_h[b];
    if (q_len < 0) return -1;
    const long long rows = q_len * G;
    const long long L = kv_len_h ? kv_len_h[b] : q_len;
    if (kv_len_h && (L < q_len)) return -1;
    for (long long r0 = 0; r0 < rows; r0 += R) {
      const long long n = rows - r0 < R ? rows - r0 : R;
      if (r0 > 0x7fffffffLL) return -1;
      // the kernel's key range for this row block, in tiles (host mirror)
      const long long base = L - q_len, pf = base + r0 / G, pl = base + (r0 + n - 1) / G;
      long long lo = window_left >= 0 ? pf - window_left : 0;
      lo = lo < 0 ? 0 : lo;
      const long long lo16 = lo & ~15LL;
      const long long a_end = window_left >= 0 ? (sink_tokens < lo16 ? sink_tokens : lo16) : 0;
      const long long tiles = (a_end + T - 1) / T + (pl + 1 - lo16 + T - 1) / T;
      if (tiles > max_tiles) max_tiles = tiles;
      blocks.push_back({tiles, b, (int32_t)r0, (int32_t)n});
    }
  }
  // longest first: CTAs are dispatched in block order as SMs free up, so the
  // launch ends on short blocks (ties keep request and row order)
  std::stable_sort(blocks.begin(), blocks.end(),
                   [](const Block& x, const Block& y) { return x.tiles > y.tiles; });
  const int64_t count = (int64_t)blocks.size();
  if (plan_h) {
    for (int64_t i = 0; i < count && i < capacity; ++i) {
      int32_t* e = plan_h + 4 * i;
      e[0] = blocks[i].b;
      e[1] = blocks[i].r0;
      e[2] = blocks[i].n;
      e[3] = 0;
    }
  }
  ctas = count * num_kv_heads;
  if (num_splits) {
    // cut the key range when there are too few CTAs for the SMs, keeping at
    // least two tiles per split
    long long s = 1;
    if (kv_len_h && num_sms > 0 && ctas > 0 && ctas < num_sms) {
      s = (2LL * num_sms + ctas - 1) / ctas;
      const long long cap = max_tiles / 2 > 1 ? max_tiles / 2 : 1;
      s = s < cap ? s : cap;
      s = s < 32 ? s : 32;
    }
    *num_splits = (int32_t)s;
  }
  return count;
}

size_t pkv_append_attention_short_workspace_bytes(int num_qo_heads, int num_kv_heads,
                                                  int max_q_len, int num_partitions) {
  if (num_kv_heads < 1 || num_qo_heads < num_kv_heads || num_qo_heads % num_kv_heads != 0 ||
      max_q_len < 1)
    return 0;
  const int64_t cols = (int64_t)(num_qo_heads / num_kv_heads) * max_q_len;
  if (cols > kMaxShortCols) return 0;
  int N = num_partitions;
  if (N == 0) N = current_device_partitions();
  if (N <= 0 || N > kMaxPartitions) return 0;
  return ws_layout(cols > kMaxGroup ? 2 * kMaxGroup : kMaxGroup, N).total;
}

pkv_status pkv_append_attention_short(const void* q, const int32_t* qo_indptr, int64_t nnz_q,
                                      int max_q_len, int num_qo_heads, const pkv_pool_desc* pool,
                                      const pkv_table_desc* table, const void* k_new,
                                      const void* v_new, const int32_t* append_indptr,
                                      int64_t nnz_new, float sm_scale, int num_partitions,
                                      void* workspace, size_t workspace_bytes, void* out,
                                      float* lse, int32_t* error_word, void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  if (pool->dtype != PKV_F16 && pool->dtype != PKV_BF16)
    return fail(PKV_ERR_INVALID_ARG, "pool dtype must be PKV_F16 or PKV_BF16");
  if (nnz_q < 0) return fail(PKV_ERR_INVALID_ARG, "nnz_q < 0");
  if (table->batch > 0 && !qo_indptr) return fail(PKV_ERR_INVALID_ARG, "null qo_indptr");
  if (nnz_new < 0) return fail(PKV_ERR_INVALID_ARG, "nnz_new < 0");
  if (nnz_new > 0 && (pool->data == k_new || pool->data == v_new || out == k_new || out == v_new))
    return fail(PKV_ERR_INVALID_ARG, "k_new / v_new alias the pool or out");
  if (nnz_q == 0 && nnz_new > 0)
    return pkv_append_ex(pool, table, k_new, v_new, append_indptr, nnz_new, error_word, stream);
  if (nnz_q == 0) return ok();
  return decode_impl(q, num_qo_heads, pool->data, pool->num_pages, pool->page_size,
                     pool->num_kv_heads, pool->head_dim, pool->dtype, pool->layout, tv, ids,
                     table->batch, sm_scale, num_partitions, workspace, workspace_bytes, out, lse,
                     error_word, stream, 0, (long long)num_qo_heads * kDecodeHeadDim,
                     num_qo_heads, -1, 1.f, 1.f, qo_indptr, nnz_q, max_q_len, k_new, v_new,
                     append_indptr, nnz_new);
}

size_t pkv_append_attention_workspace_bytes(int64_t nnz_q, int num_qo_heads, int num_splits) {
  if (nnz_q < 0 || num_qo_heads < 1 || num_splits < 1) return 0;
  if (num_splits == 1) return 0;
  const size_t states = (size_t)nnz_q * num_splits * num_qo_heads;
  return align_up(states * kDecodeHeadDim * 4, 256) + align_up(states * 4, 256);
}

pkv_status pkv_append_attention(const void* q, const int32_t* qo_indptr, int64_t nnz_q,
                                int num_qo_heads, const pkv_pool_desc* pool,
                                const pkv_table_desc* table, const int32_t* plan,
                                int64_t num_row_blocks, int num_splits, int window_left,
                                int sink_tokens, float sm_scale, void* workspace,
                                size_t workspace_bytes, void* out, float* lse,
                                int32_t* error_word, void* stream) {
  if (!pool) return fail(PKV_ERR_INVALID_ARG, "null pool descriptor");
  pkv::TableView tv;
  const int32_t* ids = nullptr;
  pkv_status st = table_view(table, &tv, &ids);
  if (st != PKV_OK) return st;
  const int batch = table->batch;
  if (batch < 0 || nnz_q < 0 || num_row_blocks < 0 || pool->num_pages < 1 ||
      pool->num_kv_heads < 1 || num_qo_heads < pool->num_kv_heads ||
      num_qo_heads % pool->num_kv_heads != 0)
    return fail(PKV_ERR_INVALID_ARG, "sizes out of range");
  if (pool->dtype != PKV_F16 && pool->dtype != PKV_BF16)
    return fail(PKV_ERR_INVALID_ARG, "pool dtype must be PKV_F16 or PKV_BF16");
  if (pool->layout != PKV_LAYOUT_HND && pool->layout != PKV_LAYOUT_NHD)
    return fail(PKV_ERR_INVALID_ARG, "layout must be PKV_LAYOUT_HND or PKV_LAYOUT_NHD");
  if (pool->head_dim != kDecodeHeadDim) return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 128");
  if (!valid_page_size(pool->page_size))
    return fail(PKV_ERR_UNSUPPORTED, "page_size must be 16, 32, 64, 128 or 256");
  if (pool->num_pages > 0x7fffffffLL) return fail(PKV_ERR_UNSUPPORTED, "more than 2^31-1 pages");
  if (num_splits < 1 || num_splits > 1024)
    return fail(PKV_ERR_INVALID_ARG, "num_splits must be 1..1024");
  if (sink_tokens < 0) return fail(PKV_ERR_INVALID_ARG, "sink_tokens < 0");
  if (!std::isfinite(sm_scale)) return fail(PKV_ERR_INVALID_ARG, "sm_scale is not finite");
  if (num_row_blocks > 0x7fffffffLL || num_row_blocks * pool->num_kv_heads > 0x7fffffffLL)
    return fail(PKV_ERR_UNSUPPORTED, "too many row blocks");
  if (num_row_blocks == 0 || nnz_q == 0 || batch == 0) return ok();
  if (!q || !qo_indptr || !pool->data || !ids || !plan || !out ||
      (tv.indptr ? !tv.last_len : (!tv.context_lens || tv.max_blocks < 1)))
    return fail(PKV_ERR_INVALID_ARG, "null pointer or empty block table");
  if (!aligned(q, 16) || !aligned(pool->data, 16) || !aligned(out, 16) || !aligned(plan, 16))
    return fail(PKV_ERR_INVALID_ARG, "q, pool, out and plan must be 16-byte aligned");
  if (out == q || out == pool->data) return fail(PKV_ERR_INVALID_ARG, "out aliases q or pool");
  const size_t need = pkv_append_attention_workspace_bytes(nnz_q, num_qo_heads, num_splits);
  if (need > 0 && (!workspace || !aligned(workspace, 256)))
    return fail(PKV_ERR_WORKSPACE, "workspace must be non-null and 256-byte aligned");
  if (workspace_bytes < need)
    return fail(PKV_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, need);

  CUtensorMap tmap;
  int one_box = 0;
  st = pool_tensor_map(pool->data, pool->num_pages, pool->page_size, pool->num_kv_heads,
                       pool->dtype, pool->layout, &tmap, &one_box, /*halves=*/1);
  if (st != PKV_OK) return st;
  const size_t states = (size_t)nnz_q * num_splits * num_qo_heads;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pkv::ChunkArgs a;
  a.q = q;
  a.qo_indptr = qo_indptr;
  a.tv = tv;
  a.indices = ids;
  a.plan = reinterpret_cast<const int4*>(plan);
  a.out = out;
  a.lse = lse;
  a.prefix_pages = nullptr;
  a.prefix_len = 0;
  a.states = num_splits;
  a.out_states = num_splits > 1;
  a.state_o = num_splits > 1 ? reinterpret_cast<float*>(ws) : nullptr;
  a.state_lse = num_splits > 1
                    ? reinterpret_cast<float*>(ws + align_up(states * kDecodeHeadDim * 4, 256))
                    : nullptr;
  a.err = reinterpret_cast<int*>(error_word);
  a.num_pages = pool->num_pages;
  a.nnz_q = nnz_q;
  a.batch = batch;
  a.hq = num_qo_heads;
  a.hkv = pool->num_kv_heads;
  a.group = num_qo_heads / pool->num_kv_heads;
  a.page_size = pool->page_size;
  a.splits = num_splits;
  a.window_left = window_left < 0 ? -1 : window_left;
  a.sink = sink_tokens;
  a.scale_log2 = sm_scale * 1.4426950408889634f;
  a.one_box = one_box;
  CUtensorMap qmap = {}, omap = {};
  a.q_tma = pkv::chunk_q_map(q, nnz_q, num_qo_heads, a.group, pool->dtype == PKV_BF16, &qmap) ? 1 : 0;
  a.o_tma = num_splits > 1 && pkv::chunk_state_map(a.state_o, nnz_q, num_splits, num_qo_heads,
                                                   a.group, &omap)
                ? 1
                : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = pkv::launch_chunk_tc(tmap, qmap, omap, a, pool->dtype == PKV_BF16,
                                       (int)num_row_blocks, s);
  if (e != cudaSuccess) return cuda_fail(e, "append attention launch");
  if (num_splits > 1) {
    pkv::MergeArgs ma;
    ma.v = a.state_o;
    ma.s = a.state_lse;
    ma.v_out = out;
    ma.s_out = lse;
    ma.rows = nnz_q;
    ma.states = num_splits;
    ma.heads = num_qo_heads;
    ma.head_dim = kDecodeHeadDim;
    ma.out_dtype = pool->dtype;
    ma.vec4 = 1;
    ma.rows_ok = 1;
    e = pkv::launch_merge(ma, s);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return ok();
}

pkv_status pkv_merge_states(const float* v, const float* s, int64_t num_rows, int num_states,
                            int num_heads, int head_dim, void* v_out, int out_dtype,
                            float* s_out, void* stream) {
  if (num_rows < 0 || num_states < 1 || num_heads < 1 || head_dim < 1)
    return fail(PKV_ERR_INVALID_ARG, "sizes out of range");
  if (out_dtype != PKV_F16 && out_dtype != PKV_BF16 && out_dtype != PKV_F32)
    return fail(PKV_ERR_INVALID_ARG, "out_dtype must be PKV_F16, PKV_BF16 or PKV_F32");
  if (num_rows == 0) return ok();
  if (!v || !s || !v_out) return fail(PKV_ERR_INVALID_ARG, "null pointer");
  pkv::MergeArgs a;
  a.v = v;
  a.s = s;
  a.v_out = v_out;
  a.s_out = s_out;
  a.rows = num_rows;
  a.states = num_states;
  a.heads = num_heads;
  a.head_dim = head_dim;
  a.out_dtype = out_dtype;
  a.vec4 = head_dim == 128 && aligned(v, 16) && aligned(v_out, 16);
  a.rows_ok = aligned(s, 16);
  cudaError_t e = pkv::launch_merge(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

pkv_status pkv_read_error_word(int32_t* error_word, int32_t* value, int clear, void* stream) {
  if (!error_word || !value) return fail(PKV_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(value, error_word, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (clear && *value) {
    e = cudaMemsetAsync(error_word, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  }
  if (*value) return fail(PKV_ERR_DEVICE, "device error bits 0x%x", *value);
  return ok();
}

pkv_status paged_kv_append(void* pool, int64_t num_pages, int page_size, int num_kv_heads,
                           int head_dim, int dtype, const int32_t* page_indptr,
                           const int32_t* page_indices, const int32_t* last_page_len,
                           int batch, const void* k_new, const void* v_new,
                           const int32_t* append_indptr, int64_t nnz_new, int32_t* error_word,
                           void* stream) {
  return pkv_append(pool, num_pages, page_size, num_kv_heads, head_dim, dtype, page_indptr,
                    page_indices, last_page_len, batch, k_new, v_new, append_indptr, nnz_new,
                    error_word, stream);
}

pkv_status paged_decode_attention(const void* q, int num_qo_heads, const void* pool,
                                  int64_t num_pages, int page_size, int num_kv_heads,
                                  int head_dim, int dtype, const int32_t* page_indptr,
                                  const int32_t* page_indices, const int32_t* last_page_len,
                                  int batch, float sm_scale, int num_partitions,
                                  void* workspace, size_t workspace_bytes, void* out, float* lse,
                                  int32_t* error_word, void* stream) {
  return pkv_decode(q, num_qo_heads, pool, num_pages, page_size, num_kv_heads, head_dim, dtype,
                    page_indptr, page_indices, last_page_len, batch, sm_scale, num_partitions,
                    workspace, workspace_bytes, out, lse, error_word, stream);
}

pkv_status merge_states(const float* v, const float* s, int64_t num_rows, int num_states,
                        int num_heads, int head_dim, void* v_out, int out_dtype, float* s_out,
                        void* stream) {
  return pkv_merge_states(v, s, num_rows, num_states, num_heads, head_dim, v_out, out_dtype,
                          s_out, stream);
}

}  // extern "C"
