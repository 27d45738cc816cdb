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
//
// Lane L handles dims 4L .. 4L+3 (float4 loads) when head_dim is 128, every
// 32nd dim otherwise; the state weights are computed once per warp, 32 states
// at a time (lane j holds state j's weight), and broadcast with shuffles.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ void store_val(const MergeArgs& a, size_t i, float v) {
  if (a.out_dtype == 2) {
    static_cast<float*>(a.v_out)[i] = v;
  } else if (a.out_dtype == 1) {
    static_cast<__nv_bfloat16*>(a.v_out)[i] = __float2bfloat16_rn(v);
  } else {
    static_cast<__half*>(a.v_out)[i] = __float2half_rn(v);
  }
}

constexpr int kBatch = 8;  // states whose values are loaded together (head_dim 128)

__global__ void __launch_bounds__(kWarps * 32) merge_kernel(const MergeArgs a) {
  // programmatic dependent launch: the CTAs may be resident before the kernel
  // that writes the states has finished; wait for it before reading them
  grid_dependency_wait();
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (gw >= a.rows * a.heads) return;
  const long long r = gw / a.heads;
  const int h = (int)(gw % a.heads);
  const int S = a.states, H = a.heads, D = a.head_dim;
  const float* s_row = a.s + (size_t)r * S * H + h;           // stride H between states
  const float* v_row = a.v + ((size_t)r * S * H + h) * D;     // stride H * D between states

  float M = -INFINITY;
  for (int j = lane; j < S; j += 32) M = fmaxf(M, s_row[(size_t)j * H]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const size_t orow = ((size_t)r * H + h) * D;
  if (M == -INFINITY) {  // no keys at all
    for (int d = lane; d < D; d += 32) store_val(a, orow + d, 0.f);
    if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = -INFINITY;
    return;
  }
  const bool vec = a.vec4 != 0;
  if (vec) {
    // head_dim 128: each lane owns dims 4L .. 4L+3; the values of kBatch states
    // are loaded together, one round trip per batch, then weighted in state order
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    for (int j0 = 0; j0 < S; j0 += kBatch) {
      float sj[kBatch];
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        sj[u] = j0 + u < S ? s_row[(size_t)(j0 + u) * H] : -INFINITY;
        v[u] = j0 + u < S ? *reinterpret_cast<const float4*>(v_row + (size_t)(j0 + u) * H * D + 4 * lane)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (sj[u] == -INFINITY) continue;  // (uniform) no keys: its values may be anything, even NaN
        const float wk = expf(sj[u] - M);
        wsum += wk;
        acc.x += wk * v[u].x;
        acc.y += wk * v[u].y;
        acc.z += wk * v[u].z;
        acc.w += wk * v[u].w;
      }
    }
    const float inv = 1.f / wsum;
    store_val(a, orow + 4 * lane + 0, acc.x * inv);
    store_val(a, orow + 4 * lane + 1, acc.y * inv);
    store_val(a, orow + 4 * lane + 2, acc.z * inv);
    store_val(a, orow + 4 * lane + 3, acc.w * inv);
    if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = M + logf(wsum);
    return;
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);  // vec: dims 4L..4L+3
  float accs[4] = {0.f, 0.f, 0.f, 0.f};          // otherwise: dims L, L+32, L+64, L+96
  float wsum = 0.f;
  for (int j0 = 0; j0 < S; j0 += 32) {
    const int j = j0 + lane;
    const float sj = j < S ? s_row[(size_t)j * H] : -INFINITY;
    const float wj = sj == -INFINITY ? 0.f : expf(sj - M);  // a state with no keys: weight 0
    wsum += wj;
    const int cnt = S - j0 < 32 ? S - j0 : 32;
    for (int k = 0; k < cnt; ++k) {
      const float wk = __shfl_sync(0xffffffffu, wj, k);
      if (wk == 0.f) continue;  // (uniform) its values may be anything, even NaN
      const float* vj = v_row + (size_t)(j0 + k) * H * D;
      if (vec) {
        const float4 v = *reinterpret_cast<const float4*>(vj + 4 * lane);
        acc.x += wk * v.x;
        acc.y += wk * v.y;
        acc.z += wk * v.z;
        acc.w += wk * v.w;
      } else {
        for (int i = 0, d = lane; d < D && i < 4; ++i, d += 32) accs[i] += wk * vj[d];
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  const float inv = 1.f / wsum;
  if (vec) {
    store_val(a, orow + 4 * lane + 0, acc.x * inv);
    store_val(a, orow + 4 * lane + 1, acc.y * inv);
    store_val(a, orow + 4 * lane + 2, acc.z * inv);
    store_val(a, orow + 4 * lane + 3, acc.w * inv);
  } else {
    for (int i = 0, d = lane; d < D && i < 4; ++i, d += 32) store_val(a, orow + d, accs[i] * inv);
    // head_dim above 128: the remaining dims, one state pass each
    for (int d = lane + 128; d < D; d += 32) {
      float x = 0.f;
      for (int j = 0; j < S; ++j) {
        const float sj = s_row[(size_t)j * H];
        if (sj == -INFINITY) continue;
        x += expf(sj - M) * v_row[(size_t)j * H * D + d];
      }
      store_val(a, orow + d, x * inv);
    }
  }
  if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = M + logf(wsum);
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  const long long warps = a.rows * a.heads;
  if (warps == 0) return cudaSuccess;
  const long long blocks = (warps + kWarps - 1) / kWarps;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, merge_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
