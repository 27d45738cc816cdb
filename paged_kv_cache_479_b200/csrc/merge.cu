// merge.cu -- merge attention states of disjoint key sets (pkv_merge_states).
//
// One warp per (row, head): with M = max_j s_j and w_j = exp(s_j - M),
// v_out = sum_j w_j v_j / sum_j w_j and s_out = M + log sum_j w_j, states
// taken in ascending j.  This is the exact log-sum-exp combination that the
// blockwise/ring sketch of "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的
// 生产级部署" section 4.2 approximates by averaging.  The same combination is
// fused into the decode kernel for its own split-KV partitions; this kernel
// serves callers that combine states computed elsewhere (another launch, a
// shared prefix, another GPU).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "internal.h"

namespace pkv {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) merge_kernel(const MergeArgs a) {
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (gw >= a.rows * a.heads) return;
  const long long r = gw / a.heads;
  const int h = (int)(gw % a.heads);
  const int S = a.states, H = a.heads, D = a.head_dim;

  float M = -INFINITY;
  for (int j = 0; j < S; ++j) M = fmaxf(M, a.s[((size_t)r * S + j) * H + h]);
  const size_t orow = ((size_t)r * H + h) * D;
  if (M == -INFINITY) {
    for (int d = lane; d < D; d += 32) {
      if (a.out_dtype == 2) static_cast<float*>(a.v_out)[orow + d] = 0.f;
      else static_cast<uint16_t*>(a.v_out)[orow + d] = 0;
    }
    if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = -INFINITY;
    return;
  }
  float wsum = 0.f;
  for (int j = 0; j < S; ++j) {
    const float sj = a.s[((size_t)r * S + j) * H + h];
    if (sj != -INFINITY) wsum += expf(sj - M);
  }
  for (int d = lane; d < D; d += 32) {
    float acc = 0.f;
    for (int j = 0; j < S; ++j) {
      const float sj = a.s[((size_t)r * S + j) * H + h];
      if (sj == -INFINITY) continue;  // no weight, whatever its values hold
      acc += expf(sj - M) * a.v[(((size_t)r * S + j) * H + h) * D + d];
    }
    const float val = acc / wsum;
    if (a.out_dtype == 2) {
      static_cast<float*>(a.v_out)[orow + d] = val;
    } else if (a.out_dtype == 1) {
      __nv_bfloat16 x = __float2bfloat16_rn(val);
      static_cast<__nv_bfloat16*>(a.v_out)[orow + d] = x;
    } else {
      __half x = __float2half_rn(val);
      static_cast<__half*>(a.v_out)[orow + d] = x;
    }
  }
  if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = M + logf(wsum);
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  const long long warps = a.rows * a.heads;
  if (warps == 0) return cudaSuccess;
  const long long blocks = (warps + kWarps - 1) / kWarps;
  merge_kernel<<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
