// decode.cu -- batched decode attention over the paged KV cache, sm_100a.
//
// One persistent CTA per partition (see partition.cuh): 8 consumer warps and
// 1 producer warp.
//
//  producer warp   walks the partition's (request, kv head, tile) sequence,
//                  looks the physical page up in the page table and issues
//                  bulk-tensor (TMA) loads of the tile's K and V
//                  ([16 tokens][128 dims] each, two 128-byte-swizzled boxes
//                  of 64 dims) into a 16-slot shared-memory ring guarded by
//                  full/empty mbarriers.  This is the "load the next block
//                  while the current one is being computed" pipeline of
//                  "大模型推理极致优化：FlashAttention+PageAttention联合调优"
//                  section 5.2, with the K/V of each page reached through the
//                  page table ("上下文窗口优化实战：如何用PagedAttention+FlashInfer
//                  将Llama3-70B的128K上下文吞吐提升3.8倍？", section 4.3 names this
//                  gather as the decode hot spot).
//  consumer warps  take ring slots round-robin.  Per tile, with tokens on the
//                  MMA's M axis and the (up to 8) query heads of the GQA group
//                  on N, one warp computes
//                      S^T[16 x 8]  = K_tile[16 x 128] . Q_g^T   (m16n8k16, fp32 acc)
//                  applies the online-softmax update (running max and sum in
//                  log2 units, "大模型推理极致优化：FlashAttention+PageAttention
//                  联合调优" section 2.2: recursive block-wise softmax), turns
//                  P^T into the B operand of the second MMA with movmatrix,
//                  and accumulates
//                      O^T[128 x 8] += V_tile^T[128 x 16] . P^T[16 x 8]
//                  so every K/V element read from HBM serves all G query
//                  heads of its KV head (GQA reuse).  For bf16, P is split
//                  into a bf16 high part and a bf16 remainder (two MMAs) so
//                  the probabilities keep ~16 significant bits.
//                  At the end of each (request, kv head) segment the 8 warps'
//                  states are merged through shared memory (rows padded from
//                  128 to 132 floats against bank conflicts, the padding trick of
//                  "Flash Attention与Paged KV Cache优化大模型推理实战" section 3.1),
//                  then either written as the final output or, when the pair
//                  spans several partitions, as a partial (o, lse) state; the
//                  last partition to arrive (atomic counter, no waiting)
//                  merges the partial states by their log-sum-exp weights.
//
// Short chunks (DecodeArgs::qo_indptr set): a request's q_len chunk tokens
// (q_len * G <= 16) each attend causally over the cache; the pair's columns
// are then (chunk token i, head h) at i * G + h, in two n8 column tiles when
// there are more than 8 (NQ = 2), and the keys of column i end at position
// L - q_len + i.  Every K/V tile is still read once per (request, kv head).
//
// Tokens past a request's length in its last tile are excluded by setting
// their scores to -inf (a select, never a multiply) and zeroing their V rows
// in shared memory, so whatever those slots hold (even NaN) never reaches
// the output.  Every wait has a time limit; see common.cuh.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "partition.cuh"

namespace pkv {
namespace {

constexpr int kD = 128;
constexpr int kConsumerWarps = 8;    // consumer warps of every variant but one (below)
constexpr int kMaxWarps = 16;        // consumer warps + the producer, at most
constexpr int kStages = kDecodeStages;
// GQA groups of at most 4 need half the query-block and merge-scratch room, which
// buys a 24-slot ring (192 KiB in flight instead of 128 KiB); wider groups and
// short chunks keep kStages slots
constexpr int kStagesNarrow = kStages + kStages / 2;
constexpr int kIssueLanes = kStages < 16 ? kStages : 16;  // producer lanes issuing at once
// Consumer warp w takes ring positions w, w+8, w+16, ...  With the slot count
// a multiple of the warp count, every slot has ONE consumer warp, so a warp
// only ever waits on the next round of a slot it has itself finished.  (A
// parity wait cannot tell the round before last from the next one: if another
// warp could still own the current round, the wait might return early.)
static_assert(kStages % kConsumerWarps == 0 && 32 % kIssueLanes == 0,
              "each ring slot must have a single consumer warp");
constexpr int kHalfBytes = kTileTokens * 64 * 2;  // one [16][64] box: 2 KiB
constexpr int kTileBytes = 2 * kHalfBytes;        // K or V of one 16-bit tile: 4 KiB
constexpr int kSlotBytes = 2 * kTileBytes;        // K + V: 8 KiB
// An 8-bit (E4M3) tile is half the bytes; its ring has twice the slots, so the
// same bytes are in flight.
constexpr int kMaxStages = 2 * kStagesNarrow;
constexpr int kSegRecs = 16;                      // segment records in flight
constexpr int kMaxGroup = 8;                      // columns of one n8 MMA tile
constexpr int kQBufs = 8;                         // staged query blocks in flight
// a staged query block: the pair's columns (up to gc NQ rows of 128 dims)
__host__ __device__ constexpr int q_buf_bytes(int nq, int gc) { return nq * gc * 128 * 2; }
// The producer refills query buffer (and record) seg % n for segment seg + n
// only after issuing every tile of segments seg .. seg+n-1 (each a multiple of
// 8 tiles, at least 8).  With S ring slots that means the tiles up to
// start(seg) + 8n - 1 - S have been released, which includes every consumer
// warp's first tile of segment seg -- where it reads the buffer -- as long as
// S <= 8 (n - 1).  The consumer's parity (sid / kQBufs) & 1 needs the record
// index to run over at least two buffer rounds.
static_assert(kMaxStages <= kConsumerWarps * (kQBufs - 1) &&
                  kMaxStages <= kConsumerWarps * (kSegRecs - 1) && kSegRecs % (2 * kQBufs) == 0,
              "a query buffer or segment record could be refilled before every warp read it");
// 8-bit pools with GQA groups of at most 4: their tiles carry half the bytes
// of a 16-bit tile for the same MMA work, so the consumers, not the loads, set
// the pace; 12 consumer warps on a 36-slot ring (144 KiB in flight) keep more
// tiles in work per SM than 8 on 48 (the 12 warps' merge scratch leaves no room
// for 48 slots)
constexpr int kFp8Warps = 12;
constexpr int kFp8WarpsStages = 36;
// Short chunks with two column tiles (q_len * G up to 16): twice the MMA work
// per tile on 168 registers, so again the consumers set the pace; 10 consumer
// warps (three warps of 168 registers per scheduler still fit) on a 20-slot
// ring (160 KiB in flight), with 4 staged query blocks to make the room
constexpr int kChunkWarps = 10;
constexpr int kChunkWarpsStages = 20;
constexpr int kChunkQBufs = 4;
// ring slots of a variant: 16-bit tiles (8 KiB), 8-bit tiles (4 KiB)
__host__ __device__ constexpr int ring_slots(int gc, bool fp8, int cw) {
  return !fp8 ? (cw == kChunkWarps ? kChunkWarpsStages : (gc <= 4 ? kStagesNarrow : kStages))
              : (cw == kFp8Warps ? kFp8WarpsStages : 2 * (gc <= 4 ? kStagesNarrow : kStages));
}
// staged query blocks of a variant
__host__ __device__ constexpr int q_bufs(int cw) { return cw == kChunkWarps ? kChunkQBufs : kQBufs; }
constexpr int kScratchStride = kD + 4;
constexpr float kLn2 = 0.6931471805599453f;

// a partition's first and last pair are the only ones it can share with others
constexpr int kMaxPending = 2;

// TileMeta bits
constexpr int kMetaValid = 0x1f;
constexpr int kMetaSegLast = 1 << 8;
constexpr int kMetaEnd = 1 << 9;
constexpr int kMetaSegShift = 12;

struct SegRec {
  int b, kvh, slot, c_first, ncover;
  int ncol;             // columns with a query row (G, or q_len * G; 0 = none)
  long long pair_start;
  long long q_row;      // row of q / out of the first column's token
};

// A (request, kv head) pair this partition shares with others: the partition
// holding its first tile owns counters[c_first]; ncover partitions hold its
// tiles (ncover = 0: no such pair).
struct SplitPair {
  int c_first, ncover;
};

struct __align__(16) Ctl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t cons;                      // consumer-only barrier (every consumer thread)
  uint64_t qfull[kQBufs];             // a segment's query rows landed in qbuf[i]
  int meta[kMaxStages];
  int last_it[kMaxStages];            // ring position of the last hand-over of each slot (-1: none)
  SegRec seg[kSegRecs];
  long long warp_tot[kMaxWarps];
  long long Cb0;
  SegRec pend[kMaxPending];   // split pairs this CTA wrote partial states for
  int pend_last[kMaxPending]; // 1 when this CTA arrived last for that pair
  SplitPair split[kMaxPending];  // the pairs holding this share's first and last unit
  int npend;
  int b0;
  int abort;
  int counted;                // 1 once this CTA has counted itself in on its split pairs
};

// the CW consumer warps' states of up to GC columns, merged at a segment end
template <int GC, int CW>
struct Scratch {
  float m[CW][GC];
  float l[CW][GC];
  float o[CW][GC][kScratchStride];
};

constexpr size_t scratch_bytes(int gc, int cw) {
  return (size_t)cw * gc * (2 + kScratchStride) * sizeof(float);
}
constexpr size_t smem_bytes(int nq, int gc, bool fp8 = false, int cw = kConsumerWarps) {
  return 1024 /*alignment slack*/ + (size_t)ring_slots(gc, fp8, cw) * (fp8 ? kSlotBytes / 2 : kSlotBytes) +
         (size_t)q_bufs(cw) * q_buf_bytes(nq, gc) + sizeof(Ctl) + scratch_bytes(gc <= 4 ? 4 : kMaxGroup, cw);
}
static_assert(smem_bytes(1, 4) <= 227 * 1024 && smem_bytes(1, kMaxGroup) <= 227 * 1024 &&
                  smem_bytes(2, kMaxGroup) <= 227 * 1024 &&
                  smem_bytes(1, 4, true, kFp8Warps) <= 227 * 1024 &&
                  smem_bytes(2, kMaxGroup, false, kChunkWarps) <= 227 * 1024,
              "shared memory per CTA");

// output of (request b, query head h): 16-bit final outputs, or fp32 attention
// states at a caller-chosen request stride (used when the result is merged later)
template <bool BF16>
__device__ __forceinline__ void store_out1(const DecodeArgs& a, size_t b, size_t h, int d, float v) {
  const size_t i = b * (size_t)a.out_rs + h * kD + d;
  if (a.out_f32) static_cast<float*>(a.out)[i] = v;
  else static_cast<uint16_t*>(a.out)[i] = to_bits16<BF16>(v);
}

template <bool BF16>
__device__ __forceinline__ void store_out4(const DecodeArgs& a, size_t b, size_t h, int d, float4 v) {
  const size_t i = b * (size_t)a.out_rs + h * kD + d;
  if (a.out_f32)
    *reinterpret_cast<float4*>(static_cast<float*>(a.out) + i) = v;
  else
    *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + i) =
        make_uint2(pack2<BF16>(v.x, v.y), pack2<BF16>(v.z, v.w));
}

__device__ __forceinline__ void store_lse(const DecodeArgs& a, size_t b, size_t h, float v) {
  if (a.lse) a.lse[b * (size_t)a.lse_rs + h] = v;
}

// inclusive scan over the whole block (NW warps); returns the prefix for this
// thread and the block total in *total
template <int NW>
__device__ long long block_incl_scan(long long v, long long* warp_tot, long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  long long before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const long long t = warp_tot[w];
    if (w < warp) before += t;
    all += t;
  }
  __syncthreads();
  *total = all;
  return x + before;
}

__device__ __forceinline__ uint32_t ld_u32(const void* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// all consumer threads meet; bounded
__device__ __forceinline__ bool cons_sync(Ctl& ctl, uint32_t& phase, int* err, uint64_t limit) {
  mbar_arrive(smem_u32(&ctl.cons));
  const bool ok = mbar_wait_bounded(smem_u32(&ctl.cons), phase, &ctl.abort, err, limit);
  phase ^= 1u;
  return ok;
}

// The pair holding unit `off` of request r (whose units start at flat unit
// Hkv * Cb), if partition c holds one of its tiles and shares it with others.
__device__ __forceinline__ SplitPair split_pair_at(long long W, int N, int c, int Hkv,
                                                   long long Cb, const ReqInfo& r, long long off) {
  SplitPair sp;
  sp.c_first = 0;
  sp.ncover = 0;
  const long long kvh = off / r.units;
  const SegPlace pl = seg_place(W, N, (long long)Hkv * Cb + kvh * r.units, r.units, c);
  if (pl.ncover > 1 && c >= pl.c_first && c < pl.c_first + pl.ncover) {
    sp.c_first = pl.c_first;
    sp.ncover = pl.ncover;
  }
  return sp;
}

// Count this partition in on each pair it shares (at most two: the ones
// holding its first and its last unit; every pair in between lies wholly
// inside its share).  The last arrival resets the pair's counter and, when
// this partition finished cleanly, merges the pair (pend_last).  Called once
// per CTA on every path out of the kernel, so the counters are back at zero
// when the launch ends, even after a wait ran out.
__device__ void count_in(const DecodeArgs& a, Ctl& ctl, bool clean) {
#pragma unroll
  for (int k = 0; k < kMaxPending; ++k) {
    const SplitPair sp = ctl.split[k];
    if (sp.ncover <= 1) continue;
    if (k == 1 && ctl.split[0].ncover > 1 && ctl.split[0].c_first == sp.c_first) continue;
    const int old = atomicAdd(&a.counters[sp.c_first], 1);
    if (old != sp.ncover - 1) continue;
    a.counters[sp.c_first] = 0;  // the last arrival is the counter's only remaining user
    if (!clean) continue;
    for (int j = 0; j < ctl.npend && j < kMaxPending; ++j)
      if (ctl.pend[j].c_first == sp.c_first) ctl.pend_last[j] = 1;
  }
}

// two 8-bit codes (bytes 0-1, or 2-3, of r) widened exactly to an fp16 pair:
// E4M3 by conversion, E5M2 (the top byte of a half) by placing each code in
// the high byte of its lane
template <int KV>
__device__ __forceinline__ uint32_t widen_lo(uint32_t r) {
  if constexpr (KV == kKvE4M3) return e4m3x2_to_f16x2((uint16_t)r);
  else return prmt(r, 0u, 0x1404u);
}
template <int KV>
__device__ __forceinline__ uint32_t widen_hi(uint32_t r) {
  if constexpr (KV == kKvE4M3) return e4m3x2_to_f16x2((uint16_t)(r >> 16));
  else return prmt(r, 0u, 0x3424u);
}

// Fused append: the new rows of (request b, kv head kvh) at positions in
// [tok_lo, tok_hi) are copied from k_new / v_new into their pages (16-byte
// pieces spread over the warp's lanes), then each lane orders its stores
// before the async-proxy (bulk-tensor) loads the warp issues next.  Each
// position lies in exactly one tile, and only the CTA that owns that tile
// reads it in this launch.
__device__ __forceinline__ void write_new_rows(const DecodeArgs& a, const ReqInfo& ri, int b,
                                               int kvh, long long tok_lo, long long tok_hi,
                                               int lane) {
  const long long a0 = a.append_indptr[b], a1 = a.append_indptr[b + 1];
  const long long n_new = a1 - a0;
  if (n_new <= 0) return;
  if (a0 < 0 || a1 > a.nnz_new || n_new > ri.len) {
    if (lane == 0 && a.err) atomicOr(a.err, kErrAppend);
    return;
  }
  const long long first = ri.len - n_new;  // position of the first new row
  const long long lo = tok_lo > first ? tok_lo : first;
  const long long hi = tok_hi < ri.len ? tok_hi : ri.len;
  if (lo >= hi) return;
  const int ps = a.page_size;
  const long long pieces = (hi - lo) * 2 * (kD / 8);  // rows x (K, V) x 16-byte pieces
  // up to 4 pieces per lane per round: every load of the round is issued
  // before its stores, so a round costs one load latency, not four
  constexpr int kU = 4;
  for (long long e0 = 0; e0 < pieces; e0 += 32 * kU) {
    uint4 val[kU];
    size_t dst[kU];
    bool put[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long long e = e0 + u * 32 + lane;
      put[u] = false;
      dst[u] = 0;
      if (e < pieces) {
        const long long pos = lo + e / (2 * (kD / 8));
        const int kv = (int)((e / (kD / 8)) & 1), c = (int)(e % (kD / 8));
        const int page = __ldg(a.indices + ri.page_base + pos / ps);
        const long long slot = pos % ps;
        const size_t src = ((size_t)(a0 + pos - first) * a.hkv + kvh) * kD + (size_t)c * 8;
        const uint16_t* from = static_cast<const uint16_t*>(kv ? a.v_new : a.k_new);
        val[u] = __ldg(reinterpret_cast<const uint4*>(from + src));
        if (page < 0 || (long long)page >= a.num_pages) {
          if (a.err) atomicOr(a.err, kErrPageId);
        } else {
          put[u] = true;
          dst[u] = (a.layout == PKV_LAYOUT_NHD
                        ? ((((size_t)page * 2 + kv) * ps + slot) * a.hkv + kvh) * kD
                        : ((((size_t)page * 2 + kv) * a.hkv + kvh) * ps + slot) * kD) +
                   (size_t)c * 8;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (put[u]) *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.pool) + dst[u]) = val[u];
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// KV: the pool's element type -- kKv16 (q's own 16-bit type), kKvE4M3, kKvE5M2;
// NQ: n8 column tiles per pair (2 only for short chunks over 16-bit pools);
// CHUNK: short chunks (causal limits per column), else decode (one token per request)
// GC: the GQA groups the variant takes, 8 (any) or 4 (a deeper ring)
template <bool BF16, int KV, int NQ, bool CHUNK, int GC, int CW = kConsumerWarps>
__global__ void __launch_bounds__((CW + 1) * 32, kDecodeCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  constexpr bool FP8 = KV != kKv16;
  constexpr int kThreads = (CW + 1) * 32;  // CW consumer warps, then the producer warp
  static_assert(CW == kConsumerWarps || (CW == kFp8Warps && FP8 && GC == 4) ||
                    (CW == kChunkWarps && CHUNK && NQ == 2),
                "12 consumer warps: 8-bit pools, narrow groups; 10: short chunks, two column tiles");
  constexpr int kQB = q_bufs(CW);  // staged query blocks (a power of two)
  static_assert((kQB & (kQB - 1)) == 0 && kQB <= kQBufs && kSegRecs % (2 * kQB) == 0,
                "query blocks");
  static_assert(CW + 1 <= kMaxWarps, "warp count");
  static_assert(NQ == 1 || (NQ == 2 && !FP8), "two column tiles only for 16-bit pools");
  static_assert(!CHUNK || !FP8, "short chunks only for 16-bit pools");
  static_assert(CHUNK || NQ == 1, "the decode has one column tile");
  static_assert(GC == kMaxGroup || (GC == 4 && NQ == 1 && !CHUNK), "narrow groups: decode only");
  constexpr int kCols = NQ * GC;  // columns with a query row at most
  constexpr int kQBufBytes = q_buf_bytes(NQ, GC);
  // ring geometry of this variant (16-bit: 16 or 24 slots of 8 KiB; 8-bit: 32,
  // 36 or 48 of 4 KiB)
  constexpr int kSt = ring_slots(GC, FP8, CW);
  constexpr int kTileB = FP8 ? kTileBytes / 2 : kTileBytes;
  constexpr int kSlotB = 2 * kTileB;
  constexpr int kRingBytes = kSt * kSlotB;
  constexpr int kIssue = kSt < 16 ? kSt : 16;
  static_assert(kSt % CW == 0 && 32 % kIssue == 0 && kSt <= kMaxStages,
                "each ring slot must have a single consumer warp");
  static_assert(kSt <= CW * (kQB - 1) && kSt <= CW * (kSegRecs - 1),
                "a query buffer or segment record could be refilled before every warp read it");
  // MMA operand type: 16-bit pools use their own type; E4M3 codes are widened
  // to fp16 (exact), so those tiles run the fp16 MMA
  constexpr bool kMmaBF16 = BF16 && !FP8;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte-swizzled TMA boxes need 1024-byte aligned shared addresses
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = smem;
  uint8_t* qbuf = smem + kRingBytes;
  Ctl& ctl = *reinterpret_cast<Ctl*>(qbuf + (size_t)kQB * kQBufBytes);
  Scratch<GC, CW>& scr =
      *reinterpret_cast<Scratch<GC, CW>*>(reinterpret_cast<uint8_t*>(&ctl) + sizeof(Ctl));

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int c = blockIdx.x;
  const int B = a.batch;
  const int Hkv = a.hkv;

  if (tid == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(smem_u32(&ctl.full[s]), 1);
      mbar_init(smem_u32(&ctl.empty[s]), 32);
    }
    mbar_init(smem_u32(&ctl.cons), CW * 32);
    for (int i = 0; i < kQB; ++i) mbar_init(smem_u32(&ctl.qfull[i]), 1);
    for (int s = 0; s < kSt; ++s) ctl.last_it[s] = -1;
    for (int k = 0; k < kMaxPending; ++k) {
      ctl.pend_last[k] = 0;
      ctl.split[k].c_first = 0;
      ctl.split[k].ncover = 0;
    }
    ctl.abort = 0;
    ctl.counted = 0;
    ctl.b0 = -1;
    ctl.npend = 0;
    fence_barrier_init();
  }
  if (warp == CW && lane == 0) prefetch_tensormap(&tmap);
  // With programmatic dependent launch this CTA may start while the previous
  // kernel in the stream still runs; everything above touched no input.  When
  // the caller promises that kernel does not write the page table
  // (early_table), the prologue and the producer's first page-id loads run
  // before the wait; every thread waits before it reads q, the pool or new
  // rows, and before it writes anything.
  const bool early = a.early_table != 0;
  if (!early) grid_dependency_wait();
  grid_dependents_launch();

  // ---- prologue: total work W, this partition's share [f0, f1), its first request
  long long mine = 0;
  int errs = 0;
  for (int b = tid; b < B; b += kThreads) {
    const ReqInfo r = request_info(a.tv, b, a.page_size);
    mine += r.units;
    errs |= r.err;
  }
  if (errs && c == 0 && a.err) {
    if (early) grid_dependency_wait();
    atomicOr(a.err, errs);
  }
  long long total_units;
  (void)block_incl_scan<CW + 1>(mine, ctl.warp_tot, &total_units);
  const long long W = (long long)Hkv * total_units;
  // with fewer units than CTAs only the first W partitions get work, so that
  // every partition that covers a (request, kv head) pair is non-empty
  const int N = W < (long long)gridDim.x ? (int)W : (int)gridDim.x;
  const long long f0 = c < N ? part_start(W, N, c) : 0;
  const long long f1 = c < N ? part_start(W, N, c + 1) : 0;

  long long carry = 0;
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + tid;
    ReqInfo r;
    r.tiles = 0;
    r.units = 0;
    r.len = 0;
    if (b < B) r = request_info(a.tv, b, a.page_size);
    long long chunk_total;
    const long long incl = block_incl_scan<CW + 1>(r.units, ctl.warp_tot, &chunk_total);
    const long long excl = incl - r.units;
    if (b < B && r.units > 0 && f0 < f1) {
      const long long s0 = (long long)Hkv * (carry + excl), s1 = (long long)Hkv * (carry + incl);
      // the pair holding this share's last unit, if it is shared with others
      if (s0 <= f1 - 1 && f1 - 1 < s1)
        ctl.split[1] = split_pair_at(W, N, c, Hkv, carry + excl, r, f1 - 1 - s0);
      if (s0 <= f0 && f0 < s1) {
        ctl.b0 = b;
        ctl.Cb0 = carry + excl;
        ctl.split[0] = split_pair_at(W, N, c, Hkv, carry + excl, r, f0 - s0);
        // warm L2 with the first page ids and query rows this partition needs,
        // while the rest of the prologue runs
        const long long u = (f0 - s0) % r.units;
        const long long t0 = u > kSegmentCost ? u - kSegmentCost : 0;
        const int kvh0 = (int)((f0 - s0) / r.units);
        prefetch_l2(a.indices + r.page_base + (t0 * kTileTokens) / a.page_size);
        const long long qr = a.qo_indptr ? a.qo_indptr[b] : b;
        prefetch_l2(static_cast<const uint16_t*>(a.q) + ((size_t)qr * a.hq + (size_t)kvh0 * a.group) * kD);
      }
    }
    if (b < B && r.tiles == 0 && (b % (int)gridDim.x) == c) {
      if (early) grid_dependency_wait();
      if (!a.qo_indptr) {
        // a request with no tokens: attention over no keys -> o = 0, lse = -inf
        for (int h = 0; h < a.hq; ++h) {
          for (int d = 0; d < kD; d += 4) store_out4<BF16>(a, b, h, d, make_float4(0.f, 0.f, 0.f, 0.f));
          store_lse(a, b, h, -INFINITY);
        }
      } else if (a.qo_indptr[b + 1] != a.qo_indptr[b] && a.err) {
        atomicOr(a.err, kErrAppend);  // chunk tokens but no cache: they were never appended
      }
    }
    carry += chunk_total;
  }
  __syncthreads();
  if (f0 >= f1 || ctl.b0 < 0) {
    // no work: still wait, so that this launch never completes before the
    // kernels it depends on (a dependent launch relies on that)
    if (early) grid_dependency_wait();
    return;
  }

  const int G = a.group;

  if (warp == CW) {
    // =========================== producer ===========================
    Walk wk;
    wk.tv = a.tv;
    wk.B = B;
    wk.ps = a.page_size;
    wk.Hkv = Hkv;
    wk.start(ctl.b0, ctl.Cb0, request_info(a.tv, ctl.b0, a.page_size), f0, f1);
    const uint32_t ring0 = smem_u32(ring);
    const long long ps = a.page_size;
    const int ps_shift = __ffs(a.page_size) - 1;  // page sizes are powers of two
    uint32_t i = 0;  // tiles handed to the ring so far
    int seg = 0;
    bool ok = true;
    // page ids of the previous segment's first 32 tiles: the kv heads of one
    // request share its pages, so the next head's segment over the same
    // tiles reuses them instead of loading them again
    long long ids_base = -1, ids_t0 = -1, ids_n = 0;
    int ids_first = -1;
    while (ok && !wk.done()) {
      if (wk.seg_units() <= 0) {  // only possible if the table changed under the kernel
        if (lane == 0) {
          if (a.err) atomicOr(a.err, kErrIndptr);
          ctl.abort = 1;
        }
        ok = false;
        break;
      }
      const long long t0 = wk.t0();
      const long long n = wk.t1() - t0;
      if (n == 0) {  // this share of the pair holds only its fixed-cost units
        wk.advance();
        continue;
      }
      const long long n_pad = (n + CW - 1) / CW * CW;
      const long long pstart = wk.pair_start();
      // page ids, one tile per lane, loaded one 32-tile batch ahead of their use
      const int* idx = a.indices + wk.ri.page_base;
      int page_next = -1;
      if (wk.ri.page_base == ids_base && t0 == ids_t0 && (n < 32 ? n : 32) <= ids_n) {
        page_next = lane < n ? ids_first : -1;
      } else if (lane < n) {
        page_next = idx[((t0 + lane) * kTileTokens) >> ps_shift];
      }
      ids_base = wk.ri.page_base;
      ids_t0 = t0;
      ids_n = n < 32 ? n : 32;
      ids_first = page_next;
      if (early && seg == 0) grid_dependency_wait();  // before q, the pool or new rows
      if (lane == 0) {
        const SegPlace pl = seg_place_in(W, N, pstart, wk.ri.units, c, f0, f1);
        SegRec& r = ctl.seg[seg & (kSegRecs - 1)];
        r.b = wk.b;
        r.kvh = wk.kvh;
        r.slot = pl.slot;
        r.c_first = pl.c_first;
        r.ncover = pl.ncover;
        r.pair_start = pstart;
        // the pair's query rows: its G heads of one token (decode) or of each
        // of the chunk's tokens; a chunk that does not fit gets no columns
        long long q_row = wk.b;
        int q_len = 1;
        if (CHUNK) {
          q_row = a.qo_indptr[wk.b];
          const long long ql = (long long)a.qo_indptr[wk.b + 1] - q_row;
          const bool fits = ql >= 1 && ql * G <= a.max_cols && ql * G <= kCols &&
                            ql <= wk.ri.len && q_row >= 0 && q_row + ql <= a.nnz_q;
          if (!fits && ql != 0 && a.err) atomicOr(a.err, kErrAppend);
          q_len = fits ? (int)ql : 0;
        }
        r.ncol = q_len * G;
        r.q_row = q_row;
        // stage them (G contiguous rows per token) for the consumers
        const int qb = seg & (kQB - 1);
        const uint32_t qbar = smem_u32(&ctl.qfull[qb]);
        const uint32_t qbytes = (uint32_t)G * kD * 2;
        mbar_arrive_expect_tx(qbar, qbytes * (uint32_t)q_len);
        for (int i = 0; i < q_len; ++i)
          bulk_load(smem_u32(qbuf + (size_t)qb * kQBufBytes + (size_t)i * qbytes),
                    static_cast<const uint16_t*>(a.q) +
                        ((size_t)(q_row + i) * a.hq + (size_t)wk.kvh * G) * kD,
                    qbytes, qbar);
        // last segment of this request: warm L2 with the next request's table entries
        if (wk.kvh == Hkv - 1 && wk.b + 1 < B) {
          if (a.tv.indptr) {
            prefetch_l2(a.tv.indptr + wk.b + 2);
            prefetch_l2(a.tv.last_len + wk.b + 1);
            prefetch_l2(a.indices + wk.ri.page_base + (wk.ri.len + ps - 1) / ps);
          } else {
            prefetch_l2(a.tv.context_lens + wk.b + 1);
            prefetch_l2(a.indices + wk.ri.page_base + a.tv.max_blocks);
          }
        }
      }
      __syncwarp();  // the record is written before any lane publishes a tile of it
      for (long long k0 = 0; ok && k0 < n_pad; k0 += 32) {
        int page = page_next;
        if (k0 + 32 + lane < n)
          page_next = idx[((t0 + k0 + 32 + lane) * kTileTokens) >> ps_shift];
        const long long k = k0 + lane;
        int yoff = 0, valid = 0;
        if (k < n) {
          if (page < 0 || (long long)page >= a.num_pages) {
            if (a.err) atomicOr(a.err, kErrPageId);
            page = -1;
          }
          const long long tok0 = (t0 + k) * kTileTokens;
          yoff = (int)(tok0 & (ps - 1));
          // tokens from the tile's first to the request's end, capped at 31: the
          // tile's valid count, and (for short chunks) each key's distance from
          // the end, which decides the causal mask
          const long long left = wk.ri.len - tok0;
          valid = left < kMetaValid ? (int)left : kMetaValid;
        } else {
          page = -1;
        }
        if constexpr (!FP8) {
          if (a.k_new) {  // fused append: this batch's tiles' new rows, before their loads
            const long long tiles_here = (n - k0) < 32 ? (n - k0) : 32;
            write_new_rows(a, wk.ri, wk.b, wk.kvh, (t0 + k0) * kTileTokens,
                           (t0 + k0 + (tiles_here > 0 ? tiles_here : 0)) * kTileTokens, lane);
            __syncwarp();
          }
        }
        const int flags = ((k >= n_pad - CW) ? kMetaSegLast : 0) |
                          ((seg & (kSegRecs - 1)) << kMetaSegShift);
        const int cnt = (int)((n_pad - k0) < 32 ? (n_pad - k0) : 32);
        // lanes [jb, jb + kIssue) publish their tiles concurrently (distinct ring slots)
        for (int jb = 0; jb < cnt; jb += kIssue) {
          int okl = 1;
          if (lane >= jb && lane < jb + kIssue && lane < cnt) {
            const uint32_t it = i + (uint32_t)(lane - jb);
            const int s = (int)(it % kSt);
            okl = mbar_wait_bounded(smem_u32(&ctl.empty[s]), ((it / kSt) & 1u) ^ 1u,
                                    &ctl.abort, a.err, a.wait_ns);
            if (okl) {
              const uint32_t full = smem_u32(&ctl.full[s]);
              ctl.last_it[s] = (int)it;
              if (page >= 0 && valid > 0) {
                ctl.meta[s] = valid | flags;
                mbar_arrive_expect_tx(full, kSlotB);
                const uint32_t dst = ring0 + (uint32_t)s * kSlotB;
                const int zk = wk.kvh, zv = Hkv + wk.kvh;
                if constexpr (FP8) {
                  // 4-D view (byte of the row, slot, kv head, 2 page + K/V): one
                  // [2][16][128] box brings the tile's K and V
                  tma_load_4d(dst, &tmap, 0, yoff, wk.kvh, 2 * page, full);
                } else if (a.one_box) {  // 5-D view: (dim % 64, slot, dim / 64, kv head, 2 page + K/V)
                  tma_load_5d(dst, &tmap, 0, yoff, 0, wk.kvh, 2 * page, full);
                  tma_load_5d(dst + kTileB, &tmap, 0, yoff, 0, wk.kvh, 2 * page + 1, full);
                } else {  // 4-D view of the HND layout: (dim, slot, K/V * Hkv + head, page)
                  tma_load_4d(dst, &tmap, 0, yoff, zk, page, full);
                  tma_load_4d(dst + kHalfBytes, &tmap, 64, yoff, zk, page, full);
                  tma_load_4d(dst + 2 * kHalfBytes, &tmap, 0, yoff, zv, page, full);
                  tma_load_4d(dst + 3 * kHalfBytes, &tmap, 64, yoff, zv, page, full);
                }
              } else {
                ctl.meta[s] = flags;  // no data: padding, or a skipped bad page
                mbar_arrive(full);
              }
            }
          }
          ok = __all_sync(0xffffffffu, okl) != 0;
          const int issued = (cnt - jb) < kIssue ? (cnt - jb) : kIssue;
          i += (uint32_t)issued;
          if (!ok) break;
        }
      }
      ++seg;
      wk.advance();
    }
    // one end marker per consumer warp
    if (ok) {
      int okl = 1;
      if (lane < CW) {
        const uint32_t it = i + lane;
        const int s = (int)(it % kSt);
        okl = mbar_wait_bounded(smem_u32(&ctl.empty[s]), ((it / kSt) & 1u) ^ 1u, &ctl.abort,
                                a.err, a.wait_ns);
        if (okl) {
          ctl.last_it[s] = (int)it;
          ctl.meta[s] = kMetaEnd;
          mbar_arrive(smem_u32(&ctl.full[s]));
        }
      }
      ok = __all_sync(0xffffffffu, okl) != 0;
      i += CW;
    }
    __syncwarp();
    if (lane == 0) {
      // Never leave with copies in flight, whoever gave up (the consumers may
      // have stopped waiting while this warp finished cleanly): wait for the
      // last hand-over of every slot to land, and for every staged query block.
      for (int s = 0; s < kSt; ++s) {
        const int it = ctl.last_it[s];
        if (it < 0) continue;
        const uint32_t bar = smem_u32(&ctl.full[s]);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, ((uint32_t)it / kSt) & 1u) &&
               global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
      for (int qb = 0; qb < kQB && qb < seg; ++qb) {
        const int last = seg - 1 - ((seg - 1 - qb) % kQB);  // latest segment using qbuf qb
        const uint32_t bar = smem_u32(&ctl.qfull[qb]);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, (uint32_t)(last / kQB) & 1u) &&
               global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    return;
  }

  // =========================== consumers ===========================
  if (early) grid_dependency_wait();  // before any output is written
  const int g = lane >> 2;     // MMA row group: token g / g+8 of the tile, column g of P^T
  const int cq = lane & 3;     // MMA column pair: columns 2cq, 2cq+1 of S^T (per n8 tile)
  const int mi = lane >> 3;    // ldmatrix: which 8x8 matrix this lane addresses
  const int r8 = lane & 7;     // ldmatrix: row within it
  const float sl2 = a.scale_log2;
  const int ct = warp * 32 + lane;
  const uint32_t ring0 = smem_u32(ring);

  uint32_t qf[NQ][8][2];
  float qsc0 = sl2, qsc1 = sl2;  // score scale of S^T columns 2cq, 2cq+1 (E4M3 pools)
  float o[NQ][8][4];
  float m0[NQ], m1[NQ], l0[NQ], l1[NQ];
  // a key at distance e - r from the request's end is visible to column
  // (token i, head h) of a chunk of q_len tokens when e - r >= q_len - i;
  // decode (q_len = 1) and columns without a query row need only e - r >= 1
  int need0[NQ], need1[NQ];
#pragma unroll
  for (int nt = 0; nt < NQ; ++nt) {
    m0[nt] = m1[nt] = -INFINITY;
    l0[nt] = l1[nt] = 0.f;
    need0[nt] = need1[nt] = 1;
  }
  int cur_seg = -1;
  SegRec rec;
  rec.b = 0;
  rec.kvh = 0;
  rec.ncol = 0;
  uint32_t cons_phase = 0;
  bool clean = true;

  for (uint32_t i = warp;; i += CW) {
    const int s = (int)(i % kSt);
    if (!mbar_wait_bounded(smem_u32(&ctl.full[s]), (i / kSt) & 1u, &ctl.abort, a.err, a.wait_ns)) {
      clean = false;
      break;
    }
    const int info = ctl.meta[s];
    if (info & kMetaEnd) break;
    const int sid = (info >> kMetaSegShift) & (kSegRecs - 1);
    if (sid != cur_seg) {
      cur_seg = sid;
      rec = ctl.seg[sid];
      if ((unsigned)rec.b >= (unsigned)B || (unsigned)rec.kvh >= (unsigned)Hkv ||
          (unsigned)rec.ncol > (unsigned)kCols) {
        // never expected: a corrupted record would address out of bounds
        if (lane == 0 && a.err) atomicOr(a.err, kErrTimeout);
        ctl.abort = 1;
        clean = false;
        break;
      }
      // the segment's query rows, staged by the producer
      const int qb = sid & (kQB - 1);
      if (!mbar_wait_bounded(smem_u32(&ctl.qfull[qb]), (uint32_t)(sid / kQB) & 1u, &ctl.abort,
                             a.err, a.wait_ns)) {
        clean = false;
        break;
      }
      if constexpr (FP8) {
        // B fragments of the fp16 MMA against widened E4M3 keys.  Head g's dims
        // are taken in the order the 8-bit K fragments deliver them: k slots
        // 2cq, 2cq+1, 2cq+8, 2cq+9 of chunk ch are dims 16ch + 4cq + 0..3.  A
        // bf16 row is first multiplied by a power of two that puts its largest
        // magnitude in [2^14, 2^15) (inside fp16's range; only elements 2^28
        // below that maximum lose bits), and the score scale undoes it.
        uint2 raw[8];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) raw[ch] = make_uint2(0u, 0u);
        if (g < rec.ncol) {
          const uint8_t* qp = qbuf + (size_t)qb * kQBufBytes + ((size_t)g * kD + 4 * cq) * 2;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) raw[ch] = *reinterpret_cast<const uint2*>(qp + ch * 32);
        }
        int qexp = 0;  // head g's row was multiplied by 2^qexp
        if constexpr (BF16) {
          float mx = 0.f;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const float2 u = unpack2<true>(raw[ch].x), v = unpack2<true>(raw[ch].y);
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(u.x), fabsf(u.y)), fmaxf(fabsf(v.x), fabsf(v.y))));
          }
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          int e = (mx > 0.f && mx <= 3.0e38f) ? ((__float_as_int(mx) >> 23) & 0xff) - 127 : 0;
          e = e < -100 ? -100 : e;
          qexp = 14 - e;
          const float f = __int_as_float((127 + qexp) << 23);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const float2 u = unpack2<true>(raw[ch].x), v = unpack2<true>(raw[ch].y);
            qf[0][ch][0] = pack2<false>(u.x * f, u.y * f);
            qf[0][ch][1] = pack2<false>(v.x * f, v.y * f);
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            qf[0][ch][0] = raw[ch].x;
            qf[0][ch][1] = raw[ch].y;
          }
        }
        // this lane's S^T columns are heads 2cq and 2cq+1 (held by lanes 8cq and 8cq+4)
        const int e0 = __shfl_sync(0xffffffffu, qexp, 8 * cq);
        const int e1 = __shfl_sync(0xffffffffu, qexp, 8 * cq + 4);
        qsc0 = sl2 * __int_as_float((127 - e0) << 23);
        qsc1 = sl2 * __int_as_float((127 - e1) << 23);
      } else {
#pragma unroll
        for (int nt = 0; nt < NQ; ++nt) {
          const int col = nt * kMaxGroup + g;
          if (col < rec.ncol) {
            const uint16_t* qp =
                reinterpret_cast<const uint16_t*>(qbuf + (size_t)qb * kQBufBytes) + col * kD + 2 * cq;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              qf[nt][j][0] = ld_u32(qp + j * 16);
              qf[nt][j][1] = ld_u32(qp + j * 16 + 8);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) qf[nt][j][0] = qf[nt][j][1] = 0u;
          }
        }
      }
      const int q_len = CHUNK ? rec.ncol / G : 1;
#pragma unroll
      for (int nt = 0; nt < NQ; ++nt) {
        const int c0 = nt * kMaxGroup + 2 * cq, c1 = c0 + 1;
        need0[nt] = CHUNK && c0 < rec.ncol ? q_len - c0 / G : 1;
        need1[nt] = CHUNK && c1 < rec.ncol ? q_len - c1 / G : 1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
        m0[nt] = m1[nt] = -INFINITY;
        l0[nt] = l1[nt] = 0.f;
      }
    }
    const int e_end = info & kMetaValid;  // tokens from the tile's first to the end (<= 31)
    const int valid = e_end > kTileTokens ? kTileTokens : e_end;
    const uint32_t kb = ring0 + (uint32_t)s * kSlotB;
    const uint32_t vb = kb + kTileB;
    bool wrote_smem = false;
    if (valid > 0) {
      // ---- S^T = K_tile . Q^T  (tokens on M, columns on N)
      float sa[NQ][4], sb[NQ][4];
#pragma unroll
      for (int nt = 0; nt < NQ; ++nt)
#pragma unroll
        for (int k = 0; k < 4; ++k) sa[nt][k] = sb[nt][k] = 0.f;
      if constexpr (FP8) {
        // one ldmatrix.x4 = tokens (0-7 | 8-15) x chunks (2jj | 2jj+1) of 16 codes;
        // lane (g, cq) gets codes 4cq .. 4cq+3 of token g's chunk, widened in pairs
        const int tok = ((mi & 1) << 3) + r8;
        const uint32_t rowb = kb + (uint32_t)tok * 128u;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int chunk = 2 * jj + (mi >> 1);
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4(rowb + (uint32_t)(((chunk & 7) ^ r8) << 4), r0, r1, r2, r3);
          mma_16816<false>(sa[0], widen_lo<KV>(r0), widen_lo<KV>(r1), widen_hi<KV>(r0),
                           widen_hi<KV>(r1), qf[0][2 * jj][0], qf[0][2 * jj][1]);
          mma_16816<false>(sb[0], widen_lo<KV>(r2), widen_lo<KV>(r3), widen_hi<KV>(r2),
                           widen_hi<KV>(r3), qf[0][2 * jj + 1][0], qf[0][2 * jj + 1][1]);
        }
      } else {
        const int tok = ((mi & 1) << 3) + r8;
        const uint32_t rowb = kb + (uint32_t)tok * 128u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int chunk = 2 * j + (mi >> 1);
          const uint32_t addr =
              rowb + (uint32_t)(j >> 2) * kHalfBytes + (uint32_t)(((chunk & 7) ^ r8) << 4);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(addr, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt) {
            if (j & 1)
              mma_16816<BF16>(sb[nt], a0, a1, a2, a3, qf[nt][j][0], qf[nt][j][1]);
            else
              mma_16816<BF16>(sa[nt], a0, a1, a2, a3, qf[nt][j][0], qf[nt][j][1]);
          }
        }
      }
      // ---- mask (past the end; causal within a chunk), online softmax (log2 units)
      const float sc0 = FP8 ? qsc0 : sl2, sc1 = FP8 ? qsc1 : sl2;
      const int dlo = e_end - g, dhi = e_end - g - 8;  // distances of tokens g, g+8 from the end
      uint32_t bh0[NQ], bh1[NQ], bl0[NQ], bl1[NQ];
#pragma unroll
      for (int nt = 0; nt < NQ; ++nt) {
        const int nd0 = CHUNK ? need0[nt] : 1, nd1 = CHUNK ? need1[nt] : 1;
        const float x0 = dlo >= nd0 ? (sa[nt][0] + sb[nt][0]) * sc0 : -INFINITY;  // token g,   col 2cq
        const float x1 = dlo >= nd1 ? (sa[nt][1] + sb[nt][1]) * sc1 : -INFINITY;  // token g,   col 2cq+1
        const float x2 = dhi >= nd0 ? (sa[nt][2] + sb[nt][2]) * sc0 : -INFINITY;  // token g+8, col 2cq
        const float x3 = dhi >= nd1 ? (sa[nt][3] + sb[nt][3]) * sc1 : -INFINITY;  // token g+8, col 2cq+1
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m0[nt], mx0), mn1 = fmaxf(m1[nt], mx1);
        // a chunk column that has seen no visible key yet keeps m = -inf:
        // subtract 0 (every decode tile has a visible key for every column)
        const float ms0 = CHUNK && mn0 == -INFINITY ? 0.f : mn0;
        const float ms1 = CHUNK && mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = ex2(m0[nt] - ms0), al1 = ex2(m1[nt] - ms1);
        const float p0 = ex2(x0 - ms0), p1 = ex2(x1 - ms1);
        const float p2 = ex2(x2 - ms0), p3 = ex2(x3 - ms1);
        l0[nt] = l0[nt] * al0 + (p0 + p2);
        l1[nt] = l1[nt] * al1 + (p1 + p3);
        m0[nt] = mn0;
        m1[nt] = mn1;
        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[nt][mt][0] *= al0;
            o[nt][mt][1] *= al1;
            o[nt][mt][2] *= al0;
            o[nt][mt][3] *= al1;
          }
        }
        // ---- P^T as the B operand of the PV MMA (movmatrix transposes S^T's layout)
        const uint32_t ph0 = pack2<kMmaBF16>(p0, p1), ph1 = pack2<kMmaBF16>(p2, p3);
        bh0[nt] = movmatrix_trans(ph0);
        bh1[nt] = movmatrix_trans(ph1);
        bl0[nt] = bl1[nt] = 0u;
        if constexpr (kMmaBF16) {
          const float2 f0 = unpack2<true>(ph0), f1 = unpack2<true>(ph1);
          bl0[nt] = movmatrix_trans(pack2<true>(p0 - f0.x, p1 - f0.y));
          bl1[nt] = movmatrix_trans(pack2<true>(p2 - f1.x, p3 - f1.y));
        }
      }
      // ---- zero V rows past the end (their slots may hold anything, even NaN)
      if (valid < kTileTokens) {
        uint8_t* vrow = ring + (size_t)s * kSlotB + kTileB;
        if constexpr (FP8) {  // one [16][128]-byte box
          for (int idx = lane; idx < (kTileTokens - valid) * 8; idx += 32) {
            const int tok = valid + (idx >> 3), ch = idx & 7;
            *reinterpret_cast<uint4*>(vrow + tok * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
        } else {  // two [16][64]-element boxes
          for (int idx = lane; idx < (kTileTokens - valid) * 16; idx += 32) {
            const int tok = valid + (idx >> 4), half = (idx >> 3) & 1, ch = idx & 7;
            *reinterpret_cast<uint4*>(vrow + half * kHalfBytes + tok * 128 + ch * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        wrote_smem = true;
        __syncwarp();
      }
      // ---- O^T += V_tile^T . P^T   (dims on M, columns on N, tokens on K)
      if constexpr (FP8) {
        // ldmatrix.trans of tokens (0-7 | 8-15) x chunks (2jj | 2jj+1) hands lane
        // (g, cq) codes V[2cq][2g], V[2cq][2g+1], V[2cq+1][2g], V[2cq+1][2g+1];
        // a byte permute pairs them by dim, so accumulator o[2jj] holds dims
        // 32jj + 2g (row g) and 32jj + 16 + 2g (row g+8), o[2jj+1] those + 1
        const int tok = ((mi >> 1) << 3) + r8;
        const uint32_t rowb = vb + (uint32_t)tok * 128u;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int chunk = 2 * jj + (mi & 1);
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4_trans(rowb + (uint32_t)(((chunk & 7) ^ r8) << 4), r0, r1, r2, r3);
          uint32_t x[4], y[4];  // dim 2g (x) and 2g+1 (y), tokens 2cq and 2cq+1
          const uint32_t rr[4] = {r0, r1, r2, r3};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if constexpr (KV == kKvE4M3) {
              const uint32_t p = prmt(rr[k], 0u, 0x3120u);
              x[k] = widen_lo<KV>(p);
              y[k] = widen_hi<KV>(p);
            } else {  // E5M2: pair and widen in one byte permute each
              x[k] = prmt(rr[k], 0u, 0x2404u);
              y[k] = prmt(rr[k], 0u, 0x3414u);
            }
          }
          mma_16816<false>(o[0][2 * jj], x[0], x[1], x[2], x[3], bh0[0], bh1[0]);
          mma_16816<false>(o[0][2 * jj + 1], y[0], y[1], y[2], y[3], bh0[0], bh1[0]);
        }
      } else {
        const int tok = ((mi >> 1) << 3) + r8;
        const uint32_t rowb = vb + (uint32_t)tok * 128u;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int chunk = 2 * mt + (mi & 1);
          const uint32_t addr =
              rowb + (uint32_t)(mt >> 2) * kHalfBytes + (uint32_t)(((chunk & 7) ^ r8) << 4);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(addr, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NQ; ++nt) {
            mma_16816<BF16>(o[nt][mt], a0, a1, a2, a3, bh0[nt], bh1[nt]);
            if constexpr (BF16) mma_16816<BF16>(o[nt][mt], a0, a1, a2, a3, bl0[nt], bl1[nt]);
          }
        }
      }
    }
    if (wrote_smem) fence_proxy_async_smem();
    __syncwarp();
    mbar_arrive(smem_u32(&ctl.empty[s]));

    if (info & kMetaSegLast) {
      // ================= end of segment: merge the CW warps' states =================
      // one n8 column tile at a time through the scratch area
      const bool direct = rec.ncover == 1;
#pragma unroll
      for (int nt = 0; nt < NQ; ++nt) {
        if (!cons_sync(ctl, cons_phase, a.err, a.wait_ns)) {  // previous merge done with scratch
          clean = false;
          break;
        }
        float la = l0[nt], lb = l1[nt];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          la += __shfl_xor_sync(0xffffffffu, la, off);
          lb += __shfl_xor_sync(0xffffffffu, lb, off);
        }
        // this lane's columns 2cq, 2cq + 1 (a narrow variant keeps the first GC)
        if (2 * cq < GC) {
          if (g == 0) {
            scr.m[warp][2 * cq] = m0[nt];
            scr.m[warp][2 * cq + 1] = m1[nt];
            scr.l[warp][2 * cq] = la;
            scr.l[warp][2 * cq + 1] = lb;
          }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            // dims of accumulator rows g and g+8 (see the PV MMA of each KV type)
            const int d0 = FP8 ? 32 * (mt >> 1) + 2 * g + (mt & 1) : mt * 16 + g;
            const int d1 = FP8 ? d0 + 16 : d0 + 8;
            scr.o[warp][2 * cq][d0] = o[nt][mt][0];
            scr.o[warp][2 * cq + 1][d0] = o[nt][mt][1];
            scr.o[warp][2 * cq][d1] = o[nt][mt][2];
            scr.o[warp][2 * cq + 1][d1] = o[nt][mt][3];
          }
        }
        if (!cons_sync(ctl, cons_phase, a.err, a.wait_ns)) {
          clean = false;
          break;
        }
        const int ncols = rec.ncol - nt * kMaxGroup;  // columns of this tile with a query row
        for (int e = ct; e < ncols * kD && e < GC * kD; e += CW * 32) {
          const int h = e >> 7, d = e & (kD - 1);
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < CW; ++w) M = fmaxf(M, scr.m[w][h]);
          const float Ms = CHUNK && M == -INFINITY ? 0.f : M;  // no visible key in this share
          float L = 0.f, acc = 0.f;
#pragma unroll
          for (int w = 0; w < CW; ++w) {
            const float wt = ex2(scr.m[w][h] - Ms);
            L += wt * scr.l[w][h];
            acc += wt * scr.o[w][h][d];
          }
          const float val = !CHUNK || L > 0.f ? (FP8 ? acc * a.v_scale / L : acc / L) : 0.f;
          const int col = nt * kMaxGroup + h;
          if (direct) {
            const size_t hq = (size_t)rec.kvh * G + col % G;
            const size_t row = (size_t)rec.q_row + col / G;
            store_out1<BF16>(a, row, hq, d, val);
            if (d == 0) store_lse(a, row, hq, (M + log2f(L)) * kLn2);
          } else {
            a.part_o[((size_t)rec.slot * a.pcols + col) * kD + d] = val;
            if (d == 0) a.part_lse[(size_t)rec.slot * a.pcols + col] = M + log2f(L);
          }
        }
      }
      if (!clean) break;
      if (!direct && ct == 0 && ctl.npend < kMaxPending) ctl.pend[ctl.npend++] = rec;
    }
  }
  // ============ end of the partition: split pairs, last arrival merges ============
  // On the clean path thread 0 counts the CTA in after every consumer has
  // written its partial states; on a failed path (a wait ran out, a bad
  // record) the first thread out counts it in and nothing is merged -- the
  // launch's outputs are invalid then (PKV_DEVERR_TIMEOUT or _INDPTR), but
  // the workspace stays reusable.
  bool synced = clean && !ctl.abort;
  if (synced) {
    __threadfence();  // this CTA's partial states are visible before it counts itself in
    synced = cons_sync(ctl, cons_phase, a.err, a.wait_ns);
  }
  if ((!synced || ct == 0) && atomicCAS(&ctl.counted, 0, 1) == 0) count_in(a, ctl, synced);
  if (!synced) return;
  const int npend = ctl.npend;
  if (!cons_sync(ctl, cons_phase, a.err, a.wait_ns)) return;
  __threadfence();
  // one warp per (pair, column); lane L owns dims 4L .. 4L+3
  const int P = a.pcols;  // state columns per slot
  for (int item = warp; item < npend * kCols; item += CW) {
    const int k = item / kCols, h = item % kCols;
    if (!ctl.pend_last[k] || h >= ctl.pend[k].ncol) continue;
    const SegRec pr = ctl.pend[k];
    auto slot_of = [&](int j) { return state_slot(pr.c_first, j); };
    constexpr int kBatch = 8;  // partial states loaded together
    float wt[kBatch];
    float4 v[kBatch];
    auto load_batch = [&](int j0) {
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = j0 + u;
        if (j < pr.ncover) {
          const int sl = slot_of(j);
          wt[u] = __ldcg(a.part_lse + (size_t)sl * P + h);
          v[u] = __ldcg(reinterpret_cast<const float4*>(a.part_o + ((size_t)sl * P + h) * kD) + lane);
        } else {
          wt[u] = -INFINITY;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    // the first batch's loads go out with the maximum's: up to kBatch states,
    // one round trip
    load_batch(0);
    float M = -INFINITY;
    for (int j = lane; j < pr.ncover; j += 32)
      M = fmaxf(M, __ldcg(a.part_lse + (size_t)slot_of(j) * P + h));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (CHUNK) M = M == -INFINITY ? 0.f : M;  // (every column of a chunk sees key 0: not expected)
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < pr.ncover; j0 += kBatch) {
      if (j0 > 0) load_batch(j0);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float w = ex2(wt[u] - M);
        L += w;
        acc.x += w * v[u].x;
        acc.y += w * v[u].y;
        acc.z += w * v[u].z;
        acc.w += w * v[u].w;
      }
    }
    const float inv = !CHUNK || L > 0.f ? 1.f / L : 0.f;
    const size_t hq = (size_t)pr.kvh * G + h % G;
    const size_t row = (size_t)pr.q_row + h / G;
    store_out4<BF16>(a, row, hq, 4 * lane,
                     make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
    if (lane == 0) store_lse(a, row, hq, !CHUNK || L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY);
  }
}

}  // namespace

size_t decode_smem_bytes(int nq) { return smem_bytes(nq, kMaxGroup); }

cudaError_t launch_decode(const CUtensorMap& tmap, const DecodeArgs& a, bool bf16, int kv, int nq,
                          int grid, cudaStream_t stream) {
  static_assert(sizeof(Ctl) % 16 == 0, "Ctl must keep Scratch 16-byte aligned");
  if (kv != kKv16 && kv != kKvE4M3 && kv != kKvE5M2) return cudaErrorInvalidValue;
  const bool chunk = a.qo_indptr != nullptr;
  if ((nq != 1 && nq != 2) || (chunk && kv != kKv16) || (!chunk && nq != 1))
    return cudaErrorInvalidValue;
  using Kern = void (*)(const CUtensorMap, const DecodeArgs);
  // decode: 16-bit, E4M3, E5M2 pools (fp16, bf16 each), for any GQA group and
  // for groups of at most 4 (16-bit: the deeper ring; 8-bit: 12 consumer
  // warps); short chunks: one or two column tiles over 16-bit pools (fp16,
  // bf16 each)
  static const Kern kKerns[16] = {
      decode_kernel<false, kKv16, 1, false, 8>,   decode_kernel<true, kKv16, 1, false, 8>,
      decode_kernel<false, kKvE4M3, 1, false, 8>, decode_kernel<true, kKvE4M3, 1, false, 8>,
      decode_kernel<false, kKvE5M2, 1, false, 8>, decode_kernel<true, kKvE5M2, 1, false, 8>,
      decode_kernel<false, kKv16, 1, true, 8>,    decode_kernel<true, kKv16, 1, true, 8>,
      decode_kernel<false, kKv16, 2, true, 8, kChunkWarps>,
      decode_kernel<true, kKv16, 2, true, 8, kChunkWarps>,
      decode_kernel<false, kKv16, 1, false, 4>,   decode_kernel<true, kKv16, 1, false, 4>,
      decode_kernel<false, kKvE4M3, 1, false, 4, kFp8Warps>,
      decode_kernel<true, kKvE4M3, 1, false, 4, kFp8Warps>,
      decode_kernel<false, kKvE5M2, 1, false, 4, kFp8Warps>,
      decode_kernel<true, kKvE5M2, 1, false, 4, kFp8Warps>};
  // the narrow variants pay where many (request, kv head) pairs (at least one
  // per CTA) each stream a short run of tiles; a few long pairs split across
  // many CTAs stream as fast with the default ring and slow down with 24 slots
  const bool narrow = !chunk && a.group <= 4 && (long long)a.batch * a.hkv >= grid;
  const int variant = (chunk ? 4 + 2 * nq : 2 * kv + (narrow ? 10 : 0)) + (bf16 ? 1 : 0);
  const Kern kern = kKerns[variant];
  const bool fp8 = kv != kKv16;
  const int cw = chunk && nq == 2 ? kChunkWarps : narrow && fp8 ? kFp8Warps : kConsumerWarps;
  const size_t smem = smem_bytes(nq, narrow ? 4 : kMaxGroup, fp8, cw);
  cudaError_t e = ensure_smem_opt_in(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: CTAs may become resident while the previous
  // kernel drains; the kernel waits for it before reading any input
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)(cw + 1) * 32);
  cfg.dynamicSmemBytes = smem;
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
