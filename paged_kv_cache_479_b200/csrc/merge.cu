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
// head_dim 128: lane L handles dims 4L .. 4L+3 (16-byte loads and stores) in
// one pass over the states, 8 at a time against a running maximum.  Other head
// dims: every 32nd dim per lane, the maximum taken first, the weights
// computed 32 states at a time (lane j holds state j's) and broadcast with
// shuffles.
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

  const size_t orow = ((size_t)r * H + h) * D;
  if (a.vec4) {
    // head_dim 128: each lane owns dims 4L .. 4L+3.  The lse and values of
    // kBatch states are loaded together, one round trip per batch, and weighted
    // in state order against the running maximum; a later batch with a larger
    // maximum rescales what is summed (up to kBatch states: the maximum of all
    // of them, as in the definition)
    float M = -INFINITY, wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < S; j0 += kBatch) {
      float sj[kBatch];
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        sj[u] = j0 + u < S ? s_row[(size_t)(j0 + u) * H] : -INFINITY;
        v[u] = j0 + u < S ? *reinterpret_cast<const float4*>(v_row + (size_t)(j0 + u) * H * D + 4 * lane)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mb = M;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) mb = fmaxf(mb, sj[u]);
      if (mb == -INFINITY) continue;  // (uniform) no state with keys yet
      if (mb > M) {
        const float f = M == -INFINITY ? 0.f : expf(M - mb);
        wsum *= f;
        acc.x *= f;
        acc.y *= f;
        acc.z *= f;
        acc.w *= f;
        M = mb;
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
    // no keys at all: 0 and -inf
    const float inv = M == -INFINITY ? 0.f : 1.f / wsum;
    const float4 o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (a.out_dtype == 2) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.v_out) + orow + 4 * lane) = o;
    } else {
      const uint2 w = a.out_dtype == 1 ? make_uint2(pack2<true>(o.x, o.y), pack2<true>(o.z, o.w))
                                       : make_uint2(pack2<false>(o.x, o.y), pack2<false>(o.z, o.w));
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.v_out) + orow + 4 * lane) = w;
    }
    if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = M == -INFINITY ? -INFINITY : M + logf(wsum);
    return;
  }
  float M = -INFINITY;
  for (int j = lane; j < S; j += 32) M = fmaxf(M, s_row[(size_t)j * H]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (M == -INFINITY) {  // no keys at all
    for (int d = lane; d < D; d += 32) store_val(a, orow + d, 0.f);
    if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = -INFINITY;
    return;
  }
  // other head dims: lane L owns dims L, L + 32, L + 64, L + 96; the weights of
  // 32 states at a time (lane j holds state j's) are broadcast with shuffles
  float accs[4] = {0.f, 0.f, 0.f, 0.f};
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
      for (int i = 0, d = lane; d < D && i < 4; ++i, d += 32) accs[i] += wk * vj[d];
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  const float inv = 1.f / wsum;
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
  if (lane == 0 && a.s_out) a.s_out[(size_t)r * H + h] = M + logf(wsum);
}

// One CTA per row when its states fit in shared memory (head_dim 128): the
// row's values [S][H][128] and lse [S][H], contiguous in both arrays, arrive
// by two bulk copies -- one round trip for the whole row -- and warp w merges
// heads w, w + 8, ... with lane L on dims 4L .. 4L+3, in the same arithmetic
// as the per-warp path (the maximum of all states, then ascending states).
constexpr int kRowThreads = 256;
constexpr size_t kRowSmemMax = 112 * 1024;  // two CTAs per SM at the largest

__global__ void __launch_bounds__(kRowThreads) merge_rows_kernel(const MergeArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const int S = a.states, H = a.heads;
  const uint32_t vbytes = (uint32_t)S * H * 128 * 4, sbytes = (uint32_t)S * H * 4;
  const float* sv = reinterpret_cast<const float*>(sm);
  const float* ss = reinterpret_cast<const float*>(sm + vbytes);
  const long long r = blockIdx.x;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // programmatic dependent launch: wait for the kernel that writes the states
  grid_dependency_wait();
  grid_dependents_launch();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(smem_u32(&bar), vbytes + sbytes);
    bulk_load(smem_u32(sm), a.v + (size_t)r * S * H * 128, vbytes, smem_u32(&bar));
    bulk_load(smem_u32(sm + vbytes), a.s + (size_t)r * S * H, sbytes, smem_u32(&bar));
  }
  if (!mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, nullptr)) {
    // never expected; the copies land before this CTA's shared memory is released
    if (threadIdx.x == 0) {
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(smem_u32(&bar), 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  for (int h = threadIdx.x >> 5; h < H; h += kRowThreads / 32) {
    float M = -INFINITY;
    for (int j = 0; j < S; ++j) M = fmaxf(M, ss[j * H + h]);
    float wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int j = 0; j < S; ++j) {
        const float sj = ss[j * H + h];
        if (sj == -INFINITY) continue;  // (uniform) no keys: its values may be anything, even NaN
        const float wk = expf(sj - M);
        const float4 v = *reinterpret_cast<const float4*>(sv + ((size_t)j * H + h) * 128 + 4 * lane);
        wsum += wk;
        acc.x += wk * v.x;
        acc.y += wk * v.y;
        acc.z += wk * v.z;
        acc.w += wk * v.w;
      }
    }
    const float inv = M == -INFINITY ? 0.f : 1.f / wsum;
    const float4 o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    const size_t orow = ((size_t)r * H + h) * 128;
    if (a.out_dtype == 2) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.v_out) + orow + 4 * lane) = o;
    } else {
      const uint2 w = a.out_dtype == 1 ? make_uint2(pack2<true>(o.x, o.y), pack2<true>(o.z, o.w))
                                       : make_uint2(pack2<false>(o.x, o.y), pack2<false>(o.z, o.w));
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.v_out) + orow + 4 * lane) = w;
    }
    if (lane == 0 && a.s_out)
      a.s_out[(size_t)r * H + h] = M == -INFINITY ? -INFINITY : M + logf(wsum);
  }
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  const long long warps = a.rows * a.heads;
  if (warps == 0) return cudaSuccess;
  // whole rows through shared memory when they fit and the bulk copies'
  // alignment rules hold (16-byte aligned rows of lse: S * H a multiple of 4)
  const size_t row_bytes = (size_t)a.states * a.heads * (128 + 1) * 4;
  const bool rows = a.vec4 && a.rows_ok && ((long long)a.states * a.heads) % 4 == 0 &&
                    row_bytes <= kRowSmemMax && a.rows <= 0x7fffffffLL;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (rows) {
    e = ensure_smem_opt_in(reinterpret_cast<const void*>(merge_rows_kernel), kRowSmemMax);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((unsigned)a.rows);
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = row_bytes;
    e = cudaLaunchKernelEx(&cfg, merge_rows_kernel, a);
  } else {
    const long long blocks = (warps + kWarps - 1) / kWarps;
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = 0;
    e = cudaLaunchKernelEx(&cfg, merge_kernel, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
