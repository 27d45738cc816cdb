// chunk_tc.cu -- multi-token append attention on the fifth-generation tensor
// cores (tcgen05, accumulators in tensor memory).
//
// Each request's chunk of new query tokens attends over its paged cache with
// a causal mask and an optional window with sink tokens (chunked prefill,
// "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署" section 3.1;
// the window of section 2.3 cut to its causal half).  A CTA owns a block of up
// to 256 rows of one request and KV head -- row r = (chunk token r / G, query
// head kvh * G + r % G) -- as two 128-row tiles A and B that share every K/V
// tile their rows may see.  Keys come in pairs of 64-token tiles; per pair,
// tile and row tile:
//     S[128 x 128] = Q[128 x 128] . K_pair^T     tcgen05.mma, A and B in shared memory
//     online softmax per 64-key tile, one thread per row reading S from tensor memory
//     O[128 x 128] += P[128 x 64] . V_tile        tcgen05.mma, P in tensor memory
// (An MMA costs about the same issue time at N = 64 as at N = 128 -- ~95
// cycles for M = 128, K = 16 -- so S is taken 128 keys at a time.)
// -- the blockwise recursive softmax of "大模型推理极致优化：FlashAttention+
// PageAttention联合调优" section 2.2 with a row tile as one MMA.  While one row
// tile's softmax runs, the tensor core works on the other's products.
//
// The same kernel computes the shared-prefix step of the cascade: for a
// prefix stored once in shared pages (prefix page sharing, "大模型推理极致优化：
// FlashAttention+PageAttention联合调优" section 3.2), rows are the (request,
// query head) pairs of every request for one KV head -- row r = (request
// r / G, head kvh * G + r % G) -- and the keys are the prefix's, unmasked, so
// the prefix's K/V is read once per 256 rows instead of once per request.
// Its result is a fp32 state per row and key split, merged afterwards with
// the state of the request's own pages.
//
// Warp roles (320 threads): warp 0 issues the bulk-tensor loads of K and V
// into a 2-stage ring of 128-key pairs; warp 1 allocates tensor memory and one of its lanes
// issues every MMA; warps 2..5 own row tile A and warps 6..9 row tile B (one
// warp per 32-lane quarter of tensor memory): they stage Q, run the softmax
// and the epilogue.
//
// Tensor memory (512 columns x 128 lanes of 32 bits): S of row tile t for
// the first / second tile of a pair in columns [64(2t+b), +64) -- rewritten in place
// by P (bf16: the high 16 bits of each fp32 probability in the first 32
// columns, the rounded remainder in the next 32, two MMAs; fp16: one part)
// -- and O of row tile t in [256 + 128t, +128).
//
// The running maximum is only moved (and O, l rescaled) when a tile's
// maximum exceeds it by more than 8 (log2 units); otherwise exponentials are
// taken against the stale maximum, which bounds P by 2^8 and changes nothing
// in o = O / l.
//
// Every wait is bounded (common.cuh); on a timeout the kernel sets the
// timeout bit, lets its own copies and MMAs drain (bounded), frees tensor
// memory and returns.  Tensor-memory loads and stores are warp-collective, so
// every branch around them is warp-uniform.  An mbarrier parity wait cannot
// tell a phase from the one two phases later or earlier, so a thread waits for
// a phase only when the phase before it is known complete and the phase after
// it cannot have completed yet (it needs something this thread does first);
// where that cannot be arranged (the end of a row tile) the barrier has one
// phase.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "partition.cuh"
#include "umma.cuh"

namespace pkv {
namespace {

constexpr int kD = 128;
constexpr int kTileRows = 128;                    // rows of one row tile (the MMA's M)
constexpr int kRowTiles = 2;
constexpr int kRows = kRowTiles * kTileRows;      // rows per CTA
constexpr int kTile = 64;                         // keys per softmax / P.V tile
constexpr int kPairKeys = 2 * kTile;              // keys per S product and ring stage
constexpr int kStages = 2;                        // ring stages (pairs)
constexpr int kThreads = 64 + kRows;              // producer, MMA, 8 softmax warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr int kQTileBytes = kTileRows * kD * 2;   // 32 KiB: two 64-dim halves of [128][64]
constexpr int kQHalf = kTileRows * 128;           // 16 KiB
constexpr int kKVHalf = kPairKeys * 128;          // 16 KiB: [128 tokens][64 dims]
constexpr int kKBytes = 2 * kKVHalf;              // 32 KiB
constexpr int kStageBytes = 2 * kKBytes;          // K then V: 64 KiB
constexpr int kBoxBytes = kTileTokens * 128;      // one [16][64] box: 2 KiB
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;
constexpr unsigned kAll = 0xffffffffu;
constexpr long long kNoCausalLimit = 1LL << 60;  // position of a prefix row: sees every key

struct __align__(16) Ctl {
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t q_full[kRowTiles];
  uint64_t s_full[kRowTiles];      // S of a pair
  uint64_t p_full[kRowTiles][2];
  uint64_t o_done[kRowTiles];   // one phase per P.V tile (the softmax's rescale waits)
  uint64_t o_final[kRowTiles];  // one phase: the row tile's last P.V done
  uint64_t drained;  // one phase: every MMA of the CTA completed
  uint64_t staged[kRowTiles];  // one phase: the row tile's states are in shared memory
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes =
    1024 + (size_t)kRowTiles * kQTileBytes + (size_t)kStages * kStageBytes + sizeof(Ctl);

// the visible key range of a row block, as a list of 64-token tiles:
// sink tiles [0, a_end) then window tiles [lo16, hi)
struct KeyRange {
  long long a_end, lo16, hi;
  int nA, n;
  __device__ void tile(int j, long long& t0, long long& t1) const {
    if (j < nA) {
      t0 = (long long)j * kTile;
      t1 = t0 + kTile < a_end ? t0 + kTile : a_end;
    } else {
      t0 = lo16 + (long long)(j - nA) * kTile;
      t1 = t0 + kTile < hi ? t0 + kTile : hi;
    }
  }
};

// mbar_wait_bounded with a suspend-time hint on the try-wait: a waiting
// thread sleeps until the phase completes (or 10 ms pass) instead of spinning,
// which leaves the issue slots to the warps that have work (the softmax warps
// of one row tile wait while the other's compute).  Same bound, abort and
// error behaviour.
__device__ __forceinline__ bool try_wait_sleeping(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(10000000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_sleeping(uint32_t bar, uint32_t parity, volatile int* abort,
                                              int* err) {
  if (try_wait_sleeping(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (*abort) return false;
    if (try_wait_sleeping(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      if (err) atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, float x, float y, float z, float w) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(x), "f"(y), "f"(z),
               "f"(w)
               : "memory");
}

__device__ __forceinline__ int clamp64(long long v) { return v <= 0 ? 0 : (v >= kTile ? kTile : (int)v); }

// qmap (when a.q_tma): q as (dim % 64, dim / 64, head, token) with boxes of
// [128 / G tokens][G heads][64 dims] -- one row tile's half, 128-byte swizzled.
// omap (when a.o_tma): the fp32 states as (dim % 32, dim / 32, head, slot,
// token) with boxes of [128 / G tokens][G heads][32 dims].
template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap omap, const ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* qs = smem;                                        // Q of both row tiles
  uint8_t* ring = smem + (size_t)kRowTiles * kQTileBytes;    // K/V stages
  Ctl& ctl = *reinterpret_cast<Ctl*>(ring + (size_t)kStages * kStageBytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // blocks in launch order: the kv heads of a row block, then the next row
  // block (the planner lists the row blocks longest first); key splits on y
  const int kvh = (int)(blockIdx.x % (unsigned)a.hkv), split = blockIdx.y;
  const int rblock = (int)(blockIdx.x / (unsigned)a.hkv);
  const int G = a.group;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&ctl.kv_full[s]), 1);
      mbar_init(smem_u32(&ctl.kv_empty[s]), 1);
    }
    for (int t = 0; t < kRowTiles; ++t) {
      mbar_init(smem_u32(&ctl.q_full[t]), kTileRows);
      mbar_init(smem_u32(&ctl.o_done[t]), 1);
      mbar_init(smem_u32(&ctl.o_final[t]), 1);
      mbar_init(smem_u32(&ctl.staged[t]), kTileRows);
      mbar_init(smem_u32(&ctl.s_full[t]), 1);
      for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&ctl.p_full[t][b]), kTileRows);
    }
    mbar_init(smem_u32(&ctl.drained), 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    umma::tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
    umma::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap);
    if (a.q_tma) prefetch_tensormap(&qmap);
    if (a.o_tma) prefetch_tensormap(&omap);
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tbase = ctl.tmem_base;
  grid_dependency_wait();
  // the shared-prefix step (one wave) lets the next launch -- the cascade's
  // own-page decode, which does not read its output -- start on the SMs it
  // leaves idle; append attention, whose CTAs come in several waves, does not
  if (a.prefix_pages != nullptr) grid_dependents_launch();

  // ---- this CTA's row block and the keys its rows may see
  const bool prefix = a.prefix_pages != nullptr;
  int b = 0, row0, nrows;
  if (prefix) {  // rows of every request, in blocks of kRows
    row0 = rblock * kRows;
    const long long left = (long long)a.batch * G - row0;
    nrows = left < kRows ? (int)left : kRows;
  } else {
    const int4 item = a.plan[rblock];
    b = item.x;
    row0 = item.y;
    nrows = item.z;
  }
  bool bad = (!prefix && (unsigned)b >= (unsigned)a.batch) || nrows < 1 || nrows > kRows ||
             row0 < 0 || (prefix && a.prefix_len < 1);
  ReqInfo r{};
  long long q_len = 0, q_first = 0;
  if (!bad && !prefix) {
    r = request_info(a.tv, b, a.page_size);
    q_first = a.qo_indptr[b];
    q_len = (long long)a.qo_indptr[b + 1] - q_first;
    bad = r.err != 0 || q_len < 0 || q_len > r.len || q_first < 0 ||
          q_first + q_len > a.nnz_q || (long long)row0 + nrows > q_len * G;
  }
  if (bad && tid == 0 && a.err) atomicOr(a.err, r.err ? r.err : kErrAppend);
  const long long base = r.len - q_len;  // position of chunk token 0
  const int tiles = nrows > kTileRows ? 2 : 1;  // row tiles with rows
  KeyRange kr{};
  int j0 = 0, n = 0;
  if (!bad && prefix) {  // every prefix token, unmasked
    kr.hi = a.prefix_len;
    kr.n = (int)((kr.hi + kTile - 1) / kTile);
  } else if (!bad) {
    const long long pos_first = base + row0 / G, pos_last = base + (row0 + nrows - 1) / G;
    kr.hi = pos_last + 1;
    long long lo = a.window_left >= 0 ? pos_first - a.window_left : 0;
    lo = lo < 0 ? 0 : lo;
    kr.lo16 = lo & ~15LL;
    kr.a_end = a.window_left >= 0 ? (a.sink < kr.lo16 ? a.sink : kr.lo16) : 0;
    kr.nA = (int)((kr.a_end + kTile - 1) / kTile);
    kr.n = kr.nA + (int)((kr.hi - kr.lo16 + kTile - 1) / kTile);
  }
  if (!bad) {  // this split's share of the key tiles
    const int per = (kr.n + a.splits - 1) / a.splits;
    j0 = split * per;
    const int j1 = j0 + per < kr.n ? j0 + per : kr.n;
    n = j1 > j0 ? j1 - j0 : 0;
  }

  if (!bad && warp == 0) {
    // =========================== producer ===========================
    const uint32_t ring0 = smem_u32(ring);
    const int* ids = prefix ? a.prefix_pages : a.indices + r.page_base;
    bool ok = true;
    int issued = 0;
    const int np = (n + 1) / 2;  // pairs of tiles
    for (int i = 0; ok && i < np; ++i) {
      const int s = i % kStages;
      // lane L < 8 looks up box L: tokens 16 (L % 4) .. of tile 2i + L / 4
      int page = -1, yoff = 0;
      if (lane < 8 && 2 * i + (lane >> 2) < n) {
        long long t0, t1;
        kr.tile(j0 + 2 * i + (lane >> 2), t0, t1);
        const int sub = lane & 3;
        if (sub * kTileTokens < (int)(t1 - t0)) {
          const long long tok = t0 + sub * kTileTokens;
          page = ids[tok / a.page_size];
          if (page < 0 || (long long)page >= a.num_pages) {
            if (a.err) atomicOr(a.err, kErrPageId);
            page = -1;
          }
          yoff = (int)(tok % a.page_size);
        }
      }
      const unsigned have = __ballot_sync(kAll, page >= 0) & 0xffu;
      // every lane loads one box (K / V = L / 16, dim half = L / 8 % 2, box = L % 8)
      const int box = lane & 7, half = (lane >> 3) & 1, kv = lane >> 4;
      const int bpage = __shfl_sync(kAll, page, box);
      const int byoff = __shfl_sync(kAll, yoff, box);
      int okl = 1;
      if (lane == 0) {
        okl = wait_sleeping(smem_u32(&ctl.kv_empty[s]), ((i / kStages) & 1) ^ 1, &ctl.abort,
                                a.err);
        if (okl) mbar_arrive_expect_tx(smem_u32(&ctl.kv_full[s]), __popc(have) * 4u * kBoxBytes);
      }
      ok = __shfl_sync(kAll, okl, 0) != 0;
      if (!ok) break;
      if (bpage >= 0) {
        const uint32_t dst = ring0 + (uint32_t)s * kStageBytes + (uint32_t)kv * kKBytes +
                             (uint32_t)half * kKVHalf + (uint32_t)box * kBoxBytes;
        const uint32_t full = smem_u32(&ctl.kv_full[s]);
        if (a.one_box)  // 5-D view (dim % 64, slot, dim / 64, kv head, 2 page + K/V), [16][64] boxes
          tma_load_5d(dst, &tmap, 0, byoff, half, kvh, 2 * bpage + kv, full);
        else            // 4-D view of the HND layout (dim, slot, K/V * Hkv + head, page)
          tma_load_4d(dst, &tmap, 64 * half, byoff, kv * a.hkv + kvh, bpage, full);
      }
      issued = i + 1;
    }
    if (lane == 0) {
      // never leave with copies in flight, whoever gave up (the MMA or softmax
      // warps may have stopped waiting while this warp finished cleanly)
      const int first = issued > kStages ? issued - kStages : 0;
      for (int k = first; k < issued; ++k) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(smem_u32(&ctl.kv_full[k % kStages]), (k / kStages) & 1) &&
               global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (!bad && warp == 1) {
    // =========================== MMA issuer ===========================
    if (lane == 0) {
      const uint32_t ring0 = smem_u32(ring);
      const uint32_t idesc_s = umma::instr_desc(BF16, kTileRows, kPairKeys, false, false);
      const uint32_t idesc_pv = umma::instr_desc(BF16, kTileRows, kD, false, true);
      auto issue_s = [&](int p, int t) {  // S_t of pair p into both buffers of row tile t
        const uint32_t qb = smem_u32(qs) + (uint32_t)t * kQTileBytes;
        const uint32_t kbase = ring0 + (uint32_t)(p % kStages) * kStageBytes;
        const uint32_t d = tbase + (uint32_t)(2 * t) * kTile;
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {  // 16 dims per MMA: 32 bytes along a swizzled row
          const uint32_t off = (uint32_t)(k & 3) * 32u;
          const uint64_t ad = umma::smem_desc(qb + (uint32_t)(k >> 2) * kQHalf + off, 16, 1024);
          const uint64_t bd = umma::smem_desc(kbase + (uint32_t)(k >> 2) * kKVHalf + off, 16, 1024);
          umma::mma_ss(d, ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        umma::commit(smem_u32(&ctl.s_full[t]));
      };
      auto issue_pv = [&](int j, int t) {  // O_t += P_t(j) . V(j)
        const uint32_t vbase = ring0 + (uint32_t)((j >> 1) % kStages) * kStageBytes + kKBytes +
                               (uint32_t)(j & 1) * (kTile * 128);
        const uint32_t p_cols = tbase + (uint32_t)(2 * t + (j & 1)) * kTile;
        const uint32_t o = tbase + kColO + (uint32_t)t * kD;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {  // 16 keys per MMA: 8 columns of P, 2 KiB of V
          const uint64_t bd = umma::smem_desc(vbase + (uint32_t)k * 2048u, kKVHalf, 1024);
          umma::mma_ts(o, p_cols + 8u * k, bd, idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
        }
        if constexpr (BF16) {
#pragma unroll
          for (int k = 0; k < kTile / 16; ++k) {
            const uint64_t bd = umma::smem_desc(vbase + (uint32_t)k * 2048u, kKVHalf, 1024);
            umma::mma_ts(o, p_cols + 32u + 8u * k, bd, idesc_pv, 1u);
          }
        }
        umma::commit(smem_u32(&ctl.o_done[t]));
      };
      bool ok = true;
      for (int t = 0; ok && t < tiles; ++t)
        ok = wait_sleeping(smem_u32(&ctl.q_full[t]), 0, &ctl.abort, a.err);
      if (ok && n > 0) {
        ok = wait_sleeping(smem_u32(&ctl.kv_full[0]), 0, &ctl.abort, a.err);
        if (ok) {
          umma::fence_after_sync();
          for (int t = 0; t < tiles; ++t) issue_s(0, t);
        }
      }
      const int np = (n + 1) / 2;
      // per pair: PV of its first tile for A and B; then, per row tile, PV of
      // its second tile followed at once by S of the next pair, so the tensor
      // core alternates between the row tiles (A's next S runs while B's
      // softmax still works on its second tile)
      for (int p = 0; ok && p < np; ++p) {
        const int ja = 2 * p, jb = 2 * p + 1;
        for (int t = 0; ok && t < tiles; ++t) {
          ok = wait_sleeping(smem_u32(&ctl.p_full[t][0]), p & 1, &ctl.abort, a.err);
          if (!ok) break;
          umma::fence_after_sync();
          issue_pv(ja, t);
          if (ja == n - 1) umma::commit(smem_u32(&ctl.o_final[t]));
        }
        if (ok && jb < n) {
          const bool next = p + 1 < np;
          if (next)
            ok = wait_sleeping(smem_u32(&ctl.kv_full[(p + 1) % kStages]), ((p + 1) / kStages) & 1,
                               &ctl.abort, a.err);
          for (int t = 0; ok && t < tiles; ++t) {
            ok = wait_sleeping(smem_u32(&ctl.p_full[t][1]), p & 1, &ctl.abort, a.err);
            if (!ok) break;
            umma::fence_after_sync();
            issue_pv(jb, t);
            if (jb == n - 1) umma::commit(smem_u32(&ctl.o_final[t]));
            // S of the next pair overwrites both P buffers of this row tile: no
            // wait, the MMAs of one thread run in issue order, so both PVs
            // have read P before it writes (and the softmax wrote P before
            // its p_full arrival)
            if (next) issue_s(p + 1, t);
          }
        }
        if (ok) umma::commit(smem_u32(&ctl.kv_empty[p % kStages]));
      }
      // let every MMA issued land before tensor memory is freed (a commit
      // arrives once all MMAs this thread issued before it completed)
      umma::commit(smem_u32(&ctl.drained));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(smem_u32(&ctl.drained), 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else if (!bad && warp >= 2 && (warp - 2) / 4 < tiles) {
    // =========================== softmax warps ===========================
    const int t = (warp - 2) / 4;                  // row tile
    const int quarter = warp & 3;                  // tensor-memory lane quarter
    const int row = quarter * 32 + lane;           // row within the tile
    const uint32_t trow = tbase + ((uint32_t)(quarter * 32) << 16);
    const uint32_t t_o = trow + kColO + (uint32_t)t * kD;
    const int rr = row0 + t * kTileRows + row;     // row within the request's chunk rows
    const bool has_row = t * kTileRows + row < nrows;
    const bool full_tile = t * kTileRows + kTileRows <= nrows;
    const long long pos = has_row ? (prefix ? kNoCausalLimit : base + rr / G) : -1;
    uint8_t* qt = qs + (size_t)t * kQTileBytes;
    // the row tile's first row is (token q_first + (row0 + 128 t) / G, head
    // kvh * G) when G divides its start
    if (a.q_tma && (row0 + t * kTileRows) % G == 0) {
      // ---- Q by two bulk-tensor loads (rows past the tensor read as zeros;
      // rows past the block, another request's, are masked like any such row:
      // the rows of a tile never mix in its products)
      if (warp == 2 + 4 * t && lane == 0) {
        const uint32_t bar = smem_u32(&ctl.q_full[t]);
        mbar_arrive_expect_tx(bar, kQTileBytes);
        for (int half = 0; half < 2; ++half)
          tma_load_4d(smem_u32(qt) + (uint32_t)half * kQHalf, &qmap, 0, half, kvh * G,
                      (int)(q_first + (row0 + t * kTileRows) / G), bar);
      } else {
        mbar_arrive(smem_u32(&ctl.q_full[t]));
      }
    } else {
      // ---- stage this row of Q in the 128-byte-swizzled K-major layout
      const uint4* src = has_row ? reinterpret_cast<const uint4*>(
                                       static_cast<const uint16_t*>(a.q) +
                                       ((size_t)(q_first + rr / G) * a.hq + (size_t)kvh * G + rr % G) * kD)
                                 : nullptr;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = src ? src[c] : make_uint4(0, 0, 0, 0);
        const int half = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(qt + half * kQHalf + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&ctl.q_full[t]));
    }
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int bj = j & 1;  // tile within its pair: the S / P buffer
      const uint32_t t_s = trow + (uint32_t)(2 * t + bj) * kTile;
      if (bj == 0) {  // one S product covers both tiles of the pair
        ok = __all_sync(kAll, wait_sleeping(smem_u32(&ctl.s_full[t]), (j >> 1) & 1, &ctl.abort,
                                            a.err));
        if (!ok) break;
      }
      umma::fence_after_sync();
      uint32_t s0[32], s1[32];
      umma::ld32(t_s, s0);
      umma::ld32(t_s + 32u, s1);
      long long t0, t1;
      kr.tile(j0 + j, t0, t1);
      const int valid = (int)(t1 - t0);
      // visible keys of this row in the tile: k < hk (causal), and k >= lk or k < sk (window)
      const int hk = pos - t0 + 1 >= valid ? valid : clamp64(pos - t0 + 1);
      const int lk = a.window_left >= 0 ? clamp64(pos - a.window_left - t0) : 0;
      const int sk = a.window_left >= 0 ? clamp64((long long)a.sink - t0) : 0;
      umma::wait_ld();
      float x[64];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        x[k] = __uint_as_float(s0[k]);
        x[32 + k] = __uint_as_float(s1[k]);
      }
      if (!__all_sync(kAll, hk == kTile && lk == 0)) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
          x[k] = ((k < hk) & ((k >= lk) | (k < sk))) ? x[k] : -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = x[u];
#pragma unroll
      for (int k = 8; k < 64; k += 16) {
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = max3(mx[u], x[k + u], x[k + 8 + u < 64 ? k + 8 + u : k + u]);
      }
      const float mt = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl2;
      const bool move = mt > m_used + kRescaleThreshold;
      // O (and l) were accumulated against m_used: rescale the rows that move
      // their maximum, once PV(j-1) is done (the whole warp loads and stores)
      const bool rescale = move && j > 0 && m_used != -INFINITY;
      if (__any_sync(kAll, rescale)) {
        ok = __all_sync(kAll, wait_sleeping(smem_u32(&ctl.o_done[t]), (j - 1) & 1,
                                                &ctl.abort, a.err));
        if (!ok) break;
        umma::fence_after_sync();
        const float f = rescale ? ex2(m_used - mt) : 1.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          umma::ld32(t_o + 32u * c, o);
          umma::wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
          umma::st32(t_o + 32u * c, o);
        }
        l *= f;
      }
      if (move) m_used = mt;
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      // P = 2^(x * scale - m): high part = top 16 bits (bf16 truncation), low
      // part = the exact remainder rounded to bf16; fp16: one rounding.  Two
      // keys per paired-fp32 instruction.
      uint32_t hi[32], lo[32];
      const uint64_t scale2 = f2_pack(sl2, sl2), neg_m2 = f2_pack(-mref, -mref);
      uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 e = f2_unpack(f2_fma(f2_pack(x[2 * k], x[2 * k + 1]), scale2, neg_m2));
        const float p0 = ex2(e.x), p1 = ex2(e.y);
        const uint64_t pp = f2_pack(p0, p1);
        acc[k & 1] = f2_add(acc[k & 1], pp);
        if constexpr (BF16) {
          const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
          hi[k] = prmt(b0, b1, 0x7632u);
          const float2 rem = f2_unpack(f2_sub(pp, f2_pack(__uint_as_float(b0 & 0xffff0000u),
                                                          __uint_as_float(b1 & 0xffff0000u))));
          lo[k] = pack2<true>(rem.x, rem.y);
        } else {
          hi[k] = pack2<false>(p0, p1);
        }
      }
      const float2 s2 = f2_unpack(f2_add(acc[0], acc[1]));
      l += s2.x + s2.y;
      umma::st32(t_s, hi);
      if constexpr (BF16) umma::st32(t_s + 32u, lo);
      // V rows past the tile's keys may hold anything (even NaN): row tile A
      // zeroes them before the first PV of this tile (B's is issued after A's)
      if (t == 0 && valid < kTile) {
        uint8_t* vt = ring + (size_t)((j >> 1) % kStages) * kStageBytes + kKBytes + bj * (kTile * 128);
        const int chunks = (kTile - valid) * 16;  // 16-byte chunks over both dim halves
        for (int idx = row; idx < chunks; idx += kTileRows) {
          const int tk = valid + (idx >> 4), half = (idx >> 3) & 1, c = idx & 7;
          *reinterpret_cast<uint4*>(vt + half * kKVHalf + tk * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      umma::wait_st();
      umma::fence_before_sync();
      mbar_arrive(smem_u32(&ctl.p_full[t][bj]));
    }
    // ---- epilogue: o = O / l of this row (every lane loads; rows past the block store nothing)
    if (ok) {
      // the row tile's last P.V (and every MMA before it): a one-phase barrier,
      // so the wait cannot alias however far the P.V phases have run
      bool have_o = n > 0;
      if (have_o)
        have_o = __all_sync(kAll, wait_sleeping(smem_u32(&ctl.o_final[t]), 0, &ctl.abort, a.err));
      if (n == 0 || have_o) {
        umma::fence_after_sync();
        const size_t tok = has_row ? (size_t)(q_first + rr / G) : 0;
        const size_t h = has_row ? (size_t)kvh * G + rr % G : 0;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float lse = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
        // fp32 states of a row tile whose rows are all its own (or past the
        // tensor: the prefix's last block) go out as four bulk-tensor stores
        // of [128 rows][32 dims], staged 128-byte swizzled in a ring stage no
        // MMA reads any more: A takes the stage of the pair before the last (its
        // last P.V completed every MMA issued before it, B's of that pair
        // included), B the last pair's (its last P.V is the CTA's last MMA)
        const bool st_tma = a.out_states && a.o_tma && (row0 + t * kTileRows) % G == 0 &&
                            (a.prefix_pages != nullptr || full_tile);
        if (st_tma) {
          const uint32_t stg = smem_u32(ring) + (uint32_t)((((n + 1) >> 1) + t) & 1) * kStageBytes;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            if (have_o) {
              umma::ld32(t_o + 32u * c, o);
              umma::wait_ld();
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = 0u;
            }
            const uint32_t box = stg + (uint32_t)(c * kTileRows * 128 + row * 128);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              st_shared_v4(box + (uint32_t)((k ^ (row & 7)) << 4),
                           __uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                           __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
          }
          fence_proxy_async_smem();
          mbar_arrive(smem_u32(&ctl.staged[t]));
          if (warp == 2 + 4 * t && lane == 0 &&
              wait_sleeping(smem_u32(&ctl.staged[t]), 0, &ctl.abort, a.err)) {
            for (int c = 0; c < 4; ++c)
              tma_store_5d(&omap, stg + (uint32_t)(c * kTileRows * 128), 0, c, kvh * G,
                           split, (int)(q_first + (row0 + t * kTileRows) / G));
            bulk_store_commit_and_wait_read();
          }
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            if (have_o) {
              umma::ld32(t_o + 32u * c, o);
              umma::wait_ld();
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = 0u;
            }
            if (!has_row) continue;
            if (!a.out_states) {
              uint16_t* op = static_cast<uint16_t*>(a.out) + (tok * a.hq + h) * kD + 32 * c;
#pragma unroll
              for (int k = 0; k < 32; k += 8) {
                uint4 w;
                w.x = pack2<BF16>(__uint_as_float(o[k + 0]) * inv, __uint_as_float(o[k + 1]) * inv);
                w.y = pack2<BF16>(__uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
                w.z = pack2<BF16>(__uint_as_float(o[k + 4]) * inv, __uint_as_float(o[k + 5]) * inv);
                w.w = pack2<BF16>(__uint_as_float(o[k + 6]) * inv, __uint_as_float(o[k + 7]) * inv);
                *reinterpret_cast<uint4*>(op + k) = w;
              }
            } else {
              float* op = a.state_o + ((tok * a.states + split) * a.hq + h) * kD + 32 * c;
#pragma unroll
              for (int k = 0; k < 32; k += 4)
                *reinterpret_cast<float4*>(op + k) =
                    make_float4(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv,
                                __uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
            }
          }
        }
        if (has_row) {
          if (!a.out_states) {
            if (a.lse) a.lse[tok * a.hq + h] = lse;
          } else {
            a.state_lse[(tok * a.states + split) * a.hq + h] = lse;
          }
        }
      }
    }
  }

  // ---- free tensor memory once every warp is done with it
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

size_t chunk_tc_smem_bytes() { return kSmemBytes; }
int chunk_rows_per_cta() { return kRows; }
int chunk_tile_tokens() { return kTile; }

cudaError_t launch_chunk_tc(const CUtensorMap& tmap, const CUtensorMap& qmap,
                            const CUtensorMap& omap, const ChunkArgs& a, bool bf16, int row_blocks,
                            cudaStream_t stream) {
  auto kern = bf16 ? chunk_tc_kernel<true> : chunk_tc_kernel<false>;
  cudaError_t e = ensure_smem_opt_in(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)row_blocks * (unsigned)a.hkv, (unsigned)a.splits);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmap, qmap, omap, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
