// append.cu -- scatter newly decoded tokens' K and V into their pages.
//
// One warp per (new token, kv head): the warp finds the token's request by
// binary search over append_indptr, maps its logical position to
// (page, slot) through the page table -- page = page_indices[indptr[b] + pos / page_size],
// slot = pos % page_size, the O(1) translation of "Flash Attention与Paged KV Cache
// 优化大模型推理实战" section 3.2 -- and copies the head's K row and V row with
// 16-byte vector loads and stores.  Pure copies: the pool is bit-identical to
// what a byte-wise scatter would produce.
#include <cuda_runtime.h>

#include "internal.h"
#include "partition.cuh"

namespace pkv {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) append_kernel(const AppendArgs a) {
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (gw >= a.nnz * a.hkv) return;
  const long long i = gw / a.hkv;     // new token
  const int h = (int)(gw % a.hkv);    // kv head

  // request b: append_indptr[b] <= i < append_indptr[b+1]
  int lo = 0, hi = a.batch;           // invariant: append_indptr[lo] <= i < append_indptr[hi]
  if (a.append_indptr[0] > i || a.append_indptr[a.batch] <= i) {
    if (lane == 0 && a.err) atomicOr(a.err, kErrAppend);
    return;
  }
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.append_indptr[mid] <= i) lo = mid; else hi = mid;
  }
  const int b = lo;
  const ReqInfo r = request_info(a.indptr, a.last_len, b, a.page_size);
  const long long n_new = (long long)a.append_indptr[b + 1] - a.append_indptr[b];
  const long long pos = r.len - n_new + (i - a.append_indptr[b]);
  if (r.err || pos < 0 || pos >= r.len) {
    if (lane == 0 && a.err) atomicOr(a.err, r.err ? r.err : kErrAppend);
    return;
  }
  const int page = a.indices[(long long)r.page_base + pos / a.page_size];
  if (page < 0 || (long long)page >= a.num_pages) {
    if (lane == 0 && a.err) atomicOr(a.err, kErrPageId);
    return;
  }
  const long long slot = pos % a.page_size;
  const int vecs = a.head_dim / 8;    // 16-byte vectors per row
  const size_t src = ((size_t)i * a.hkv + h) * a.head_dim;
  const size_t dk = ((((size_t)page * 2 + 0) * a.hkv + h) * a.page_size + slot) * a.head_dim;
  const size_t dv = ((((size_t)page * 2 + 1) * a.hkv + h) * a.page_size + slot) * a.head_dim;
  const uint16_t* kn = static_cast<const uint16_t*>(a.k_new);
  const uint16_t* vn = static_cast<const uint16_t*>(a.v_new);
  uint16_t* pool = static_cast<uint16_t*>(a.pool);
  for (int e = lane; e < 2 * vecs; e += 32) {
    const bool is_v = e >= vecs;
    const int x = (is_v ? e - vecs : e) * 8;
    const uint4 val = *reinterpret_cast<const uint4*>((is_v ? vn : kn) + src + x);
    *reinterpret_cast<uint4*>(pool + (is_v ? dv : dk) + x) = val;
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  const long long warps = a.nnz * a.hkv;
  if (warps == 0) return cudaSuccess;
  const long long blocks = (warps + kWarps - 1) / kWarps;
  append_kernel<<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
