// prefix.cu -- attention of many requests' queries over ONE shared prefix.
//
// When requests share a prefix (a system prompt stored once in shared pages:
// "大模型推理极致优化：FlashAttention+PageAttention联合调优" section 3.2; automatic
// prefix sharing, "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署"
// section 3.3), decoding each request separately re-reads the prefix's K/V
// once per request.  Here the prefix is read once per block of 128 query
// rows, where a row is one (request, query head) of one KV head's group:
// B * G rows per KV head become the M dimension of a dense contraction,
//     S[128 x 64]  = Q[128 x 128] . K_tile^T      (m16n8k16, fp32 accumulate)
//     O[128 x 128] += P[128 x 64] . V_tile         (P split into bf16 high + low)
// with online softmax over the prefix tokens (FlashAttention-style, "大模型推理
// 极致优化：FlashAttention+PageAttention联合调优" section 2.2).  The prefix tokens are
// cut into `splits` chunks so the grid fills the GPU; each CTA writes its rows'
// normalised partial state (o, natural-log lse) as fp32 into state slot
// `split` of [B][S][Hq][128]; the states are merged with the requests' own
// (suffix) attention afterwards (pkv_merge_states).
//
// CTA: 8 consumer warps (16 query rows each) and 1 producer warp issuing the
// K/V of 64-token tiles as 16-token bulk-tensor boxes into a 3-stage ring.
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
constexpr int kWarps = 8;                       // consumer warps
constexpr int kRows = kWarps * 16;              // query rows per CTA
constexpr int kStageBytes = 2 * kKVBytes;
constexpr int kStages = 3;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(16) Ctl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int valid[kStages];  // prefix tokens present in the stage's tile
  int abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + sizeof(Ctl);

template <bool BF16>
__global__ void __launch_bounds__((kWarps + 1) * 32, 1)
    prefix_kernel(const __grid_constant__ CUtensorMap tmap, const PrefixArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + (size_t)kStages * kStageBytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rb = blockIdx.x, split = blockIdx.y, kvh = blockIdx.z;
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

  const long long t_begin = (long long)split * a.tokens_per_split;
  const long long t_end = t_begin + a.tokens_per_split < a.prefix_len
                              ? t_begin + a.tokens_per_split : a.prefix_len;
  const int ntiles = t_end > t_begin ? (int)((t_end - t_begin + kTile - 1) / kTile) : 0;

  if (warp == kWarps) {
    // =========================== producer ===========================
    const uint32_t ring0 = smem_u32(smem);
    bool ok = true;
    for (int i = 0; ok && i < ntiles; ++i) {
      const int s = i % kStages;
      const long long t0 = t_begin + (long long)i * kTile;
      const int valid = (int)((t_end - t0) < kTile ? (t_end - t0) : kTile);
      // lanes 0..kBoxes-1 each handle one 16-token box
      int page = -1, yoff = 0;
      if (lane < kBoxes && lane * kTileTokens < valid) {
        const long long tok = t0 + lane * kTileTokens;
        page = a.prefix_pages[tok / a.page_size];
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
  const long long nrows = (long long)a.batch * G;
  const long long row0 = (long long)rb * kRows + warp * 16;  // this warp's first row
  // query rows as A fragments: row r -> request r / G, query head kvh * G + r % G
  uint32_t qa[8][4];
  {
    const uint16_t* qp[2];
    for (int hr = 0; hr < 2; ++hr) {
      const long long r = row0 + g + 8 * hr;
      qp[hr] = r < nrows ? static_cast<const uint16_t*>(a.q) +
                               ((size_t)(r / G) * a.hq + (size_t)kvh * G + r % G) * kD
                         : nullptr;
    }
    tile::load_q(qp[0], qp[1], cq, qa);
  }
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows g and g + 8
  const float sl2 = a.scale_log2;
  const uint32_t ring0 = smem_u32(smem);

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % kStages;
    if (!mbar_wait_bounded(smem_u32(&ctl.full[s]), (i / kStages) & 1, &ctl.abort, a.err)) return;
    const int valid = ctl.valid[s];
    const uint32_t kb = ring0 + (uint32_t)s * kStageBytes, vb = kb + kKVBytes;
    float sc[8][4];
    tile::qk<BF16>(qa, kb, lane, sc);
    // tokens past the prefix are not keys
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int t = n * 8 + 2 * cq;
      sc[n][0] = t < valid ? sc[n][0] * sl2 : -INFINITY;
      sc[n][1] = t + 1 < valid ? sc[n][1] * sl2 : -INFINITY;
      sc[n][2] = t < valid ? sc[n][2] * sl2 : -INFINITY;
      sc[n][3] = t + 1 < valid ? sc[n][3] * sl2 : -INFINITY;
    }
    tile::online_softmax(sc, m0, m1, l0, l1, o);
    if (valid < kTile) tile::zero_v_rows(smem + (size_t)s * kStageBytes + kKVBytes, valid, lane);
    tile::pv<BF16>(sc, vb, lane, o);
    if (valid < kTile) fence_proxy_async_smem();
    __syncwarp();
    mbar_arrive(smem_u32(&ctl.empty[s]));
  }

  // ---- rows' partial states: o / l (fp32) and lse (natural log)
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  for (int hr = 0; hr < 2; ++hr) {
    const long long r = row0 + g + 8 * hr;
    if (r >= nrows) continue;
    const long long b = r / G, h = (long long)kvh * G + r % G;
    const float l = hr ? l1 : l0, m = hr ? m1 : m0;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* op = a.state_o + (((size_t)b * a.states + split) * a.hq + h) * kD;
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<float2*>(op + n * 8 + 2 * cq) =
          make_float2(o[n][2 * hr] * inv, o[n][2 * hr + 1] * inv);
    if (cq == 0)
      a.state_lse[((size_t)b * a.states + split) * a.hq + h] =
          l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

}  // namespace

size_t prefix_smem_bytes() { return kSmemBytes; }
int prefix_rows_per_cta() { return kRows; }
int prefix_tile_tokens() { return kTile; }

cudaError_t launch_prefix(const CUtensorMap& tmap, const PrefixArgs& a, bool bf16, int row_blocks,
                          cudaStream_t stream) {
  auto kern = bf16 ? prefix_kernel<true> : prefix_kernel<false>;
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
  cfg.gridDim = dim3((unsigned)row_blocks, (unsigned)a.splits, (unsigned)a.hkv);
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
