// internal.h -- launch entry points shared between the kernel files and the
// C ABI layer (api.cu).  Not installed; the public interface is include/pkv.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

// record the detail that pkv_last_error() reports on this thread; returns s
pkv_status set_error(pkv_status s, const char* fmt, ...);

struct DecodeArgs {
  const void* q;          // [B][Hq][128]
  void* out;              // [B][Hq][128]
  float* lse;             // [B][Hq] or null
  const int32_t* indptr;  // [B+1]
  const int32_t* indices;
  const int32_t* last_len;  // [B]
  int* counters;          // [N] arrival counters (zero between launches)
  float* part_lse;        // [2N][G], log2 domain
  float* part_o;          // [2N][G][128]
  int* err;               // device error word or null
  long long num_pages;
  int batch, hq, hkv, group, page_size;
  float scale_log2;       // sm_scale * log2(e)
  int one_box;            // 1: 5-D tensor map, one box per K/V tile; 0: 4-D map, two boxes
};

constexpr int kDecodeThreads = 288;  // 8 consumer warps + 1 producer warp
#ifndef PKV_STAGES
#define PKV_STAGES 16
#endif
#ifndef PKV_CTAS_PER_SM
#define PKV_CTAS_PER_SM 1
#endif
constexpr int kDecodeStages = PKV_STAGES;        // K/V ring slots (8 KiB each) per CTA
constexpr int kDecodeCtasPerSm = PKV_CTAS_PER_SM; // resident decode CTAs per SM

size_t decode_smem_bytes();
cudaError_t launch_decode(const CUtensorMap& tmap, const DecodeArgs& a, bool bf16, int grid,
                          cudaStream_t stream);

struct AppendArgs {
  void* pool;
  const int32_t* indptr;
  const int32_t* indices;
  const int32_t* last_len;
  const int32_t* append_indptr;
  const void* k_new;
  const void* v_new;
  int* err;
  long long num_pages;
  long long nnz;
  int batch, hkv, head_dim, page_size;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

struct MergeArgs {
  const float* v;
  const float* s;
  void* v_out;
  float* s_out;
  long long rows;
  int states, heads, head_dim, out_dtype;
};
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream);

}  // namespace pkv
