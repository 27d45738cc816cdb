// static_ws.cu -- pkv_decode_static_workspace: decode attention for callers
// that cannot provide a workspace buffer.
//
// pkv_decode needs a little device scratch (split-KV arrival counters and
// partial (o, lse) states) that the caller normally allocates and passes in.
// Some callers cannot allocate device memory when they call: a serving
// engine that has already reserved all free HBM for its KV pool and owns no
// spare buffer, a plugin inside a host framework whose allocator it cannot
// reach, or code on a latency-critical path where cudaMalloc (which may
// synchronise the whole device) is not allowed.  For them this entry point
// runs the same decode kernel on scratch that lives in this library: a
// file-scope device array of kStaticScratchBytes, which every GPU that loads
// the library holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "pkv.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)4 << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of this device's copy of g_decode_scratch.  The array's name
// in host code is only a host-side stand-in, so the address is looked up once
// per device, with that device current, and cached.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

pkv_status pkv_decode_static_workspace(const void* q, int num_qo_heads, const void* pool,
                                       int64_t num_pages, int page_size, int num_kv_heads,
                                       int head_dim, int dtype, const int32_t* page_indptr,
                                       const int32_t* page_indices,
                                       const int32_t* last_page_len, int batch,
                                       float sm_scale, int num_partitions, void* out,
                                       float* lse, int32_t* error_word, void* stream) {
  const size_t need =
      pkv_decode_workspace_bytes(batch, num_qo_heads, num_kv_heads, head_dim, num_partitions);
  if (need > kStaticScratchBytes)
    return pkv::set_error(PKV_ERR_WORKSPACE,
                          "needs %zu bytes of scratch but the static scratch holds %zu; use "
                          "fewer partitions or pkv_decode with a caller-owned workspace",
                          need, kStaticScratchBytes);
  if (need == 0 || batch == 0) {
    // invalid shapes or nothing to do: pkv_decode reports it without launching
    return pkv_decode(q, num_qo_heads, pool, num_pages, page_size, num_kv_heads, head_dim,
                      dtype, page_indptr, page_indices, last_page_len, batch, sm_scale,
                      num_partitions, nullptr, 0, out, lse, error_word, stream);
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess)
    return pkv::set_error(PKV_ERR_CUDA, "locating the static scratch: %s", cudaGetErrorString(e));
  // The scratch keeps whatever the previous call left.  Only its arrival
  // counters must start at zero (every partial state is written before it is
  // read), so clear the counters of this call's partition count.
  const size_t counters =
      pkv::decode_counter_bytes(num_qo_heads / num_kv_heads, num_partitions);
  if (counters == 0 || counters > need)
    return pkv::set_error(PKV_ERR_CUDA, "cannot size the static scratch's counters");
  e = cudaMemsetAsync(scratch, 0, counters, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return pkv::set_error(PKV_ERR_CUDA, "clearing the static scratch: %s", cudaGetErrorString(e));
  return pkv_decode(q, num_qo_heads, pool, num_pages, page_size, num_kv_heads, head_dim, dtype,
                    page_indptr, page_indices, last_page_len, batch, sm_scale, num_partitions,
                    scratch, kStaticScratchBytes, out, lse, error_word, stream);
}

}  // extern "C"
