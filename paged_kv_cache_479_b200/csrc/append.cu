// append.cu -- scatter newly decoded tokens' K and V into their pages.
//
// Works on either page-table form (CSR or dense block table) and either pool
// layout (HND or NHD).
//
// Blocks take requests (grid-stride over b, blockIdx.y splits a request's new
// rows further when requests append many tokens); a warp copies one
// (new token, kv head) row pair.  Position pos of request b lives at page
// page_indices[indptr[b] + pos / page_size], slot pos % page_size -- the O(1)
// translation of "Flash Attention与Paged KV Cache优化大模型推理实战" section 3.2.
// The K row and the V row are copied with 16-byte vector loads and stores;
// the pool ends up bit-identical to a byte-wise scatter.  Into an 8-bit pool
// each element x is stored as fp8(x / scale) instead (binary32 division, then
// round to nearest even with saturation at the format's largest finite value,
// 448 for E4M3 and 57344 for E5M2): 8 elements per lane, 16 bytes in, 8 out.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "partition.cuh"

namespace pkv {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) append_kernel(const AppendArgs a) {
  // PDL: the next kernel (the decode) may start its prologue now; this one
  // waits for the kernel before it, which may have produced k_new / v_new
  grid_dependents_launch();
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int b = blockIdx.x; b < a.batch; b += gridDim.x) {
    const int a0 = a.append_indptr[b], a1 = a.append_indptr[b + 1];
    const ReqInfo r = request_info(a.tv, b, a.page_size);
    const long long n_new = (long long)a1 - a0;
    if (n_new == 0) continue;
    if (a0 < 0 || n_new < 0 || a1 > a.nnz || r.err || n_new > r.len) {
      if (threadIdx.x == 0 && blockIdx.y == 0 && a.err) atomicOr(a.err, r.err ? r.err : kErrAppend);
      continue;
    }
    const long long rows = n_new * a.hkv;
    for (long long row = (long long)blockIdx.y * kWarps + warp; row < rows;
         row += (long long)gridDim.y * kWarps) {
      const long long i = row / a.hkv;  // new token within the request
      const int h = (int)(row % a.hkv);
      const long long pos = r.len - n_new + i;
      const int page = a.indices[(long long)r.page_base + pos / a.page_size];
      if (page < 0 || (long long)page >= a.num_pages) {
        if (lane == 0 && a.err) atomicOr(a.err, kErrPageId);
        continue;
      }
      const long long slot = pos % a.page_size;
      const int vecs = a.head_dim / 8;  // 16-byte vectors per row
      const size_t src = ((size_t)(a0 + i) * a.hkv + h) * a.head_dim;
      // HND: [page][K/V][head][slot][dim]; NHD: [page][K/V][slot][head][dim]
      const size_t dk = a.layout == PKV_LAYOUT_NHD
          ? ((((size_t)page * 2 + 0) * a.page_size + slot) * a.hkv + h) * a.head_dim
          : ((((size_t)page * 2 + 0) * a.hkv + h) * a.page_size + slot) * a.head_dim;
      const size_t dv = dk + (size_t)a.hkv * a.page_size * a.head_dim;
      const uint16_t* kn = static_cast<const uint16_t*>(a.k_new);
      const uint16_t* vn = static_cast<const uint16_t*>(a.v_new);
      if (a.fp8) {
        uint8_t* pool8 = static_cast<uint8_t*>(a.pool);
        for (int e = lane; e < 2 * vecs; e += 32) {
          const bool is_v = e >= vecs;
          const int x = (is_v ? e - vecs : e) * 8;
          const uint4 val = *reinterpret_cast<const uint4*>((is_v ? vn : kn) + src + x);
          const float sc = is_v ? a.v_scale : a.k_scale;
          const uint32_t w[4] = {val.x, val.y, val.z, val.w};
          uint16_t c[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = a.in_bf16 ? unpack2<true>(w[j]) : unpack2<false>(w[j]);
            const float x0 = __fdiv_rn(f.x, sc), x1 = __fdiv_rn(f.y, sc);
            c[j] = a.fp8 == kKvE5M2 ? f32x2_to_e5m2x2(x0, x1) : f32x2_to_e4m3x2(x0, x1);
          }
          *reinterpret_cast<uint2*>(pool8 + (is_v ? dv : dk) + x) =
              make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16), (uint32_t)c[2] | ((uint32_t)c[3] << 16));
        }
        continue;
      }
      uint16_t* pool = static_cast<uint16_t*>(a.pool);
      for (int e = lane; e < 2 * vecs; e += 32) {
        const bool is_v = e >= vecs;
        const int x = (is_v ? e - vecs : e) * 8;
        const uint4 val = *reinterpret_cast<const uint4*>((is_v ? vn : kn) + src + x);
        *reinterpret_cast<uint4*>(pool + (is_v ? dv : dk) + x) = val;
      }
    }
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.nnz == 0 || a.batch == 0) return cudaSuccess;
  const unsigned gx = (unsigned)(a.batch < 65535 ? a.batch : 65535);
  // split a request's rows over more blocks when the average request appends many
  const long long avg_rows = (a.nnz * a.hkv + a.batch - 1) / a.batch;
  long long gy = (avg_rows + 4 * kWarps - 1) / (4 * kWarps);
  gy = gy < 1 ? 1 : (gy > 1024 ? 1024 : gy);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, (unsigned)gy);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, append_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
