// chunk.cu -- multi-token append attention: each request's chunk of new query
// tokens attends over its paged cache with a causal mask (and an optional
// window with sink tokens).
//
// Chunked prefill processes a long prompt a chunk at a time, each chunk
// attending over the cache that already holds the earlier chunks ("大模型长上下文
// 窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署" section 3.1); several
// speculative tokens verified at once are the same computation with a short
// chunk.  The table passed is the table after the chunk's K/V were appended,
// so query i of a chunk of q_len sits at position pos = L - q_len + i and
// sees keys t <= pos; with window_left >= 0 only t >= pos - window_left or
// t < sink_tokens (the window-plus-global-tokens mask of the same article's
// section 2.3, cut to its causal half).
//
// Rows: row r of request b's chunk is query token r / G of the chunk and
// query head kvh * G + r % G, so a block of 128 rows shares every K/V tile of
// its KV head (GQA reuse) -- the M dimension of a dense contraction that runs
// on the tensor cores (attn_tile.cuh).  The host plan lists the row blocks;
// the grid is (row block, kv head, split).  A row block's keys are the
// visible range of its rows: the sink tokens [0, min(sink, lo)) followed by
// [lo, last row's position] with lo the first row's window start, in 64-token
// tiles; `splits` cuts that tile list into equal shares.  With one split the
// CTA writes the final output; otherwise it writes its rows' fp32 states
// (o / l, natural-log lse) for pkv_merge_states' kernel to combine.
//
// CTA: 8 consumer warps (16 rows each) and 1 producer warp issuing the 64-token
// K/V tiles as 16-token bulk-tensor boxes into a 3-stage ring.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "attn_tile.cuh"
#include "common.cuh"
#include "internal.h"
#include "partition.cuh"

namespace pkv {
namespace {

using tile::kBoxBytes;
using tile::kBoxes;
using tile::kD;
using tile::kHalf;
using tile::kKVBytes;
using tile::kTile;
constexpr int kWarps = 8;
constexpr int kRows = kWarps * 16;
constexpr int kStageBytes = 2 * kKVBytes;
constexpr int kStages = 3;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(16) Ctl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int t0[kStages];     // first key position of the stage's tile
  int valid[kStages];  // keys present in the stage's tile
  int abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + sizeof(Ctl);

// key visibility (same rule as the host-side description above)
__device__ __forceinline__ bool visible(long long t, long long pos, int window_left, int sink) {
  return t <= pos && (window_left < 0 || t >= pos - window_left || t < sink);
}

template <bool BF16>
__global__ void __launch_bounds__((kWarps + 1) * 32, 1)
    chunk_kernel(const __grid_constant__ CUtensorMap tmap, const ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + (size_t)kStages * kStageBytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kvh = blockIdx.y, split = blockIdx.z;
  const int G = a.group;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctl.full[s]), 1);
      mbar_init(smem_u32(&ctl.empty[s]), kWarps * 32);
    }
    ctl.abort = 0;
    fence_barrier_init();
  }
  if (warp == kWarps && lane == 0) prefetch_tensormap(&tmap);
  grid_dependency_wait();
  __syncthreads();

  // ---- this CTA's row block and the keys its rows may see
  const int4 item = a.plan[blockIdx.x];
  const int b = item.x, row0 = item.y, nrows = item.z;
  bool bad = (unsigned)b >= (unsigned)a.batch || nrows < 1 || nrows > kRows || row0 < 0;
  ReqInfo r{};
  long long q_len = 0, q_first = 0;
  if (!bad) {
    r = request_info(a.tv, b, a.page_size);
    q_first = a.qo_indptr[b];
    q_len = (long long)a.qo_indptr[b + 1] - q_first;
    bad = r.err != 0 || q_len < 0 || q_len > r.len || q_first < 0 ||
          q_first + q_len > a.nnz_q || (long long)row0 + nrows > q_len * G;
  }
  if (bad) {
    // a malformed plan or table: flag it; the rows (if addressable) stay unwritten
    if (tid == 0 && a.err) atomicOr(a.err, r.err ? r.err : kErrAppend);
    return;
  }
  const long long base = r.len - q_len;                  // position of chunk token 0
  const long long pos_first = base + row0 / G, pos_last = base + (row0 + nrows - 1) / G;
  const long long hi = pos_last + 1;                      // keys [.., hi)
  long long lo = a.window_left >= 0 ? pos_first - a.window_left : 0;
  lo = lo < 0 ? 0 : lo;
  const long long lo16 = lo & ~15LL;                      // boxes start on 16-token rows
  long long a_end = a.window_left >= 0 ? (a.sink < lo16 ? a.sink : lo16) : 0;
  const int nA = (int)((a_end + kTile - 1) / kTile);
  const int nB = (int)((hi - lo16 + kTile - 1) / kTile);
  const int ntiles_all = nA + nB;
  const int per = (ntiles_all + a.splits - 1) / a.splits;
  const int j0 = split * per;
  const int j1 = j0 + per < ntiles_all ? j0 + per : ntiles_all;
  const int ntiles = j1 > j0 ? j1 - j0 : 0;
  auto tile_range = [&](int j, long long& t0, long long& t1) {
    if (j < nA) {
      t0 = (long long)j * kTile;
      t1 = t0 + kTile < a_end ? t0 + kTile : a_end;
    } else {
      t0 = lo16 + (long long)(j - nA) * kTile;
      t1 = t0 + kTile < hi ? t0 + kTile : hi;
    }
  };

  if (warp == kWarps) {
    // =========================== producer ===========================
    const uint32_t ring0 = smem_u32(smem);
    const int* ids = a.indices + r.page_base;
    bool ok = true;
    for (int i = 0; ok && i < ntiles; ++i) {
      const int s = i % kStages;
      long long t0, t1;
      tile_range(j0 + i, t0, t1);
      const int valid = (int)(t1 - t0);
      int page = -1, yoff = 0;
      if (lane < kBoxes && lane * kTileTokens < valid) {
        const long long tok = t0 + lane * kTileTokens;
        page = ids[tok / a.page_size];
        if (page < 0 || (long long)page >= a.num_pages) {
          if (a.err) atomicOr(a.err, kErrPageId);
          page = -1;
        }
        yoff = (int)(tok % a.page_size);
      }
      const unsigned have = __ballot_sync(0xffffffffu, page >= 0);
      int okl = 1;
      if (lane == 0) {
        okl = mbar_wait_bounded(smem_u32(&ctl.empty[s]), ((i / kStages) & 1) ^ 1, &ctl.abort, a.err);
        if (okl) {
          ctl.t0[s] = (int)t0;
          ctl.valid[s] = valid;
          mbar_arrive_expect_tx(smem_u32(&ctl.full[s]), (uint32_t)__popc(have) * 2 * kBoxBytes);
        }
      }
      ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
      if (!ok) break;
      if (page >= 0) {
        const uint32_t full = smem_u32(&ctl.full[s]);
        const uint32_t kdst = ring0 + (uint32_t)s * kStageBytes + (uint32_t)lane * kBoxBytes;
        const uint32_t vdst = kdst + kKVBytes;
        if (a.one_box) {  // 5-D view: (dim % 64, slot, dim / 64, kv head, 2 page + K/V)
          tma_load_5d(kdst, &tmap, 0, yoff, 0, kvh, 2 * page, full);
          tma_load_5d(vdst, &tmap, 0, yoff, 0, kvh, 2 * page + 1, full);
        } else {
          tma_load_4d(kdst, &tmap, 0, yoff, kvh, page, full);
          tma_load_4d(kdst + kHalf, &tmap, 64, yoff, kvh, page, full);
          tma_load_4d(vdst, &tmap, 0, yoff, a.hkv + kvh, page, full);
          tma_load_4d(vdst + kHalf, &tmap, 64, yoff, a.hkv + kvh, page, full);
        }
      }
    }
    if (!ok && lane == 0) {
      // aborted: let the copies already issued land before the CTA exits
      for (int s = 0; s < kStages; ++s) {
        const uint64_t t0 = global_timer_ns();
        const uint32_t bar = smem_u32(&ctl.full[s]);
        for (int ph = 0; ph < 2; ++ph)
          while (!mbar_try_wait(bar, ph) && global_timer_ns() - t0 < kWaitLimitNs) {
          }
      }
    }
    return;
  }

  // =========================== consumers ===========================
  const int g = lane >> 2, cq = lane & 3;
  const int wrow0 = row0 + warp * 16;              // this warp's first row
  const bool active = warp * 16 < nrows;           // warps past the block's rows only pace the ring
  long long pos[2];                                // positions of rows g and g + 8 (-1: no row)
  uint32_t qa[8][4];
  {
    const uint16_t* qp[2];
    for (int hr = 0; hr < 2; ++hr) {
      const int rr = wrow0 + g + 8 * hr;
      const bool v = rr < row0 + nrows;
      pos[hr] = v ? base + rr / G : -1;
      qp[hr] = v ? static_cast<const uint16_t*>(a.q) +
                       ((size_t)(q_first + rr / G) * a.hq + (size_t)kvh * G + rr % G) * kD
                 : nullptr;
    }
    if (active) tile::load_q(qp[0], qp[1], cq, qa);
  }
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale_log2;
  const uint32_t ring0 = smem_u32(smem);

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % kStages;
    if (!mbar_wait_bounded(smem_u32(&ctl.full[s]), (i / kStages) & 1, &ctl.abort, a.err)) return;
    const int valid = ctl.valid[s];
    const long long t0 = ctl.t0[s];
    if (active) {
      const uint32_t kb = ring0 + (uint32_t)s * kStageBytes, vb = kb + kKVBytes;
      float sc[8][4];
      tile::qk<BF16>(qa, kb, lane, sc);
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int t = n * 8 + 2 * cq;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tt = t + (e & 1);
          const long long p = pos[e >> 1];
          sc[n][e] = (tt < valid && visible(t0 + tt, p, a.window_left, a.sink))
                         ? sc[n][e] * sl2 : -INFINITY;
        }
      }
      tile::online_softmax(sc, m0, m1, l0, l1, o);
      if (valid < kTile) tile::zero_v_rows(smem + (size_t)s * kStageBytes + kKVBytes, valid, lane);
      tile::pv<BF16>(sc, vb, lane, o);
      if (valid < kTile) fence_proxy_async_smem();
    }
    __syncwarp();
    mbar_arrive(smem_u32(&ctl.empty[s]));
  }
  if (!active) return;

  // ---- rows: final output (one split) or fp32 state (o / l, natural-log lse)
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  for (int hr = 0; hr < 2; ++hr) {
    if (pos[hr] < 0) continue;
    const int rr = wrow0 + g + 8 * hr;
    const size_t tok = (size_t)(q_first + rr / G);
    const size_t h = (size_t)kvh * G + rr % G;
    const float l = hr ? l1 : l0, m = hr ? m1 : m0;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float lse = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    if (a.splits == 1) {
      uint16_t* op = static_cast<uint16_t*>(a.out) + (tok * a.hq + h) * kD;
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<uint32_t*>(op + n * 8 + 2 * cq) =
            pack2<BF16>(o[n][2 * hr] * inv, o[n][2 * hr + 1] * inv);
      if (cq == 0 && a.lse) a.lse[tok * a.hq + h] = lse;
    } else {
      float* op = a.state_o + ((tok * a.splits + split) * a.hq + h) * kD;
#pragma unroll
      for (int n = 0; n < 16; ++n)
        *reinterpret_cast<float2*>(op + n * 8 + 2 * cq) =
            make_float2(o[n][2 * hr] * inv, o[n][2 * hr + 1] * inv);
      if (cq == 0) a.state_lse[(tok * a.splits + split) * a.hq + h] = lse;
    }
  }
}

}  // namespace

size_t chunk_smem_bytes() { return kSmemBytes; }
int chunk_rows_per_cta() { return kRows; }
int chunk_tile_tokens() { return kTile; }

cudaError_t launch_chunk(const CUtensorMap& tmap, const ChunkArgs& a, bool bf16, int row_blocks,
                         cudaStream_t stream) {
  auto kern = bf16 ? chunk_kernel<true> : chunk_kernel<false>;
  static bool attr_set[2][64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_set[bf16][dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set[bf16][dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)row_blocks, (unsigned)a.hkv, (unsigned)a.splits);
  cfg.blockDim = dim3((kWarps + 1) * 32);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmap, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
