// partition.cuh -- split-KV work partition, shared by the decode kernel and
// by its host mirror (pkv_plan_segments).
//
// The decode work is the flattened sequence of (request b, kv head g) pairs,
// b-major then g; pair (b, g) contributes kSegmentCost "units" of fixed cost
// (starting the pair and merging its state costs about that many tiles'
// time) followed by its tiles(b) = ceil(len_b / 16) 16-token tiles.  With
// W = the total unit count, partition c of N takes the contiguous share of
// units [floor(c W / N), floor((c+1) W / N)), so every CTA gets the same
// amount of time-weighted work whatever the length mix: one long sequence is
// spread over all SMs, many short ones are packed together.  This is the
// split-KV idea (a long sequence's keys cut into blocks whose partial
// softmax states are combined afterwards); the pages describe the
// combination step as blockwise/ring attention ("大模型长上下文窗口工程化实战：
// 从RoPE扩展到百万Token推理的生产级部署", section 4.2) and size the launch from
// the work actually present rather than a fixed grid ("上下文窗口优化实战：
// 如何用PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？",
// section 2.4).
//
// A pair whose tiles fall in several partitions leaves one partial (o, lse)
// state per partition.  Partition c writes slot 2c + 1 for the pair that
// starts in its share and continues past it, and slot 2c for the pair that
// started before its share, so 2N slots always suffice.  The pair's first
// partition owns its arrival counter; the partition that arrives last merges.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define PKV_HD __host__ __device__ __forceinline__
#else
#define PKV_HD inline
#endif

#ifndef PKV_SEG_COST
#define PKV_SEG_COST 16
#endif

namespace pkv {

constexpr int kTileTokens = 16;
constexpr int kSegmentCost = PKV_SEG_COST;  // units charged per (request, kv head) pair

// device error bits (same values as PKV_DEVERR_* in pkv.h)
constexpr int kErrPageId = 0x01;
constexpr int kErrIndptr = 0x02;
constexpr int kErrLastLen = 0x04;
constexpr int kErrAppend = 0x08;
constexpr int kErrTimeout = 0x10;
constexpr int kErrContextLen = 0x20;

// A page table in one of two forms:
//   CSR:   request b owns ids[indptr[b] .. indptr[b+1]) and holds
//          (np - 1) * page_size + last_len[b] tokens;
//   dense: request b owns ids[b * max_blocks ..] (a [batch][max_blocks] block
//          table, vLLM-style) and holds context_lens[b] tokens.
struct TableView {
  const int32_t* indptr;        // CSR, or null for the dense form
  const int32_t* last_len;      // CSR
  const int32_t* context_lens;  // dense
  int max_blocks;               // dense: row length of the block table
};

struct ReqInfo {
  int64_t page_base;  // first entry of the request's page ids
  int32_t err;        // error bits (request then counts as empty)
  int64_t len;        // tokens
  int64_t tiles;      // ceil(len / 16)
  int64_t units;      // kSegmentCost + tiles per kv head, 0 for an empty request
};

PKV_HD ReqInfo request_info(const TableView& tv, int b, int ps) {
  ReqInfo r;
  r.err = 0;
  r.len = 0;
  r.tiles = 0;
  r.units = 0;
  if (tv.indptr) {
    r.page_base = tv.indptr[b];
    const int64_t np = (int64_t)tv.indptr[b + 1] - r.page_base;
    if (r.page_base < 0 || np < 0) {
      r.err = kErrIndptr;
      return r;
    }
    if (np == 0) return r;
    const int ll = tv.last_len[b];
    if (ll < 1 || ll > ps) {
      r.err = kErrLastLen;
      return r;
    }
    r.len = (np - 1) * (int64_t)ps + ll;
  } else {
    r.page_base = (int64_t)b * tv.max_blocks;
    const int64_t len = tv.context_lens[b];
    if (len < 0 || len > (int64_t)tv.max_blocks * ps) {
      r.err = kErrContextLen;
      return r;
    }
    r.len = len;
  }
  r.tiles = (r.len + kTileTokens - 1) / kTileTokens;
  r.units = r.len ? r.tiles + kSegmentCost : 0;
  return r;
}

// CSR view of (indptr, last_len)
PKV_HD TableView csr_view(const int32_t* indptr, const int32_t* last_len) {
  TableView t;
  t.indptr = indptr;
  t.last_len = last_len;
  t.context_lens = nullptr;
  t.max_blocks = 0;
  return t;
}

// First flat unit of partition c.
PKV_HD int64_t part_start(int64_t W, int N, int64_t c) { return (W * c) / N; }

// Partition holding flat unit f (0 <= f < W): the largest c with part_start(c) <= f.
PKV_HD int part_of(int64_t W, int N, int64_t f) { return (int)(((f + 1) * N - 1) / W); }

// Where a segment's result goes.  pair_start = first flat unit of the
// (request, kv head) pair, pair_units = its unit count, c = this partition.
struct SegPlace {
  int c_first;   // first partition holding a tile of the pair (owns the counter)
  int ncover;    // partitions holding tiles of the pair
  int slot;      // partial-state slot of (pair, c), -1 if ncover == 1
};

// slot of covering partition c_first + j
PKV_HD int state_slot(int c_first, int j) { return 2 * (c_first + j) + (j == 0 ? 1 : 0); }

PKV_HD SegPlace seg_place(int64_t W, int N, int64_t pair_start, int64_t pair_units, int c) {
  SegPlace p;
  p.c_first = part_of(W, N, pair_start + kSegmentCost);  // first tile, after the fixed cost
  const int c_last = part_of(W, N, pair_start + pair_units - 1);
  p.ncover = c_last - p.c_first + 1;
  p.slot = p.ncover == 1 ? -1 : state_slot(p.c_first, c - p.c_first);
  return p;
}

// seg_place for partition c whose share is [f0, f1) (f0 = part_start(c),
// f1 = part_start(c + 1)) and which holds at least one tile of the pair: a
// pair end inside the share belongs to c, so the divisions of part_of are only
// needed for an end outside it (the share's first and last pair).
PKV_HD SegPlace seg_place_in(int64_t W, int N, int64_t pair_start, int64_t pair_units, int c,
                             int64_t f0, int64_t f1) {
  SegPlace p;
  const int64_t first = pair_start + kSegmentCost, last = pair_start + pair_units - 1;
  p.c_first = first >= f0 ? c : part_of(W, N, first);
  const int c_last = last < f1 ? c : part_of(W, N, last);
  p.ncover = c_last - p.c_first + 1;
  p.slot = p.ncover == 1 ? -1 : state_slot(p.c_first, c - p.c_first);
  return p;
}

// Sequential walk over the segments of one partition.  Table pointers may be
// host or device memory (whichever side runs the walk).  A segment whose
// share of the pair holds only fixed-cost units has no tiles (t0 == t1).
struct Walk {
  TableView tv;
  int B, ps, Hkv;
  int b, kvh;
  int64_t u;      // unit within the pair
  int64_t Cb;     // sum of units(b') for b' < b
  int64_t f, f1;  // current flat unit, end of the partition
  ReqInfo ri;     // info of request b

  // start at flat unit f0 inside request b0 (whose units start at Cb0 per kv head)
  PKV_HD void start(int b0, int64_t Cb0, const ReqInfo& ri0, int64_t f0, int64_t f_end) {
    b = b0;
    Cb = Cb0;
    ri = ri0;
    f = f0;
    f1 = f_end;
    const int64_t r = f0 - (int64_t)Hkv * Cb0;
    kvh = ri0.units ? (int)(r / ri0.units) : 0;
    u = ri0.units ? r % ri0.units : 0;
  }
  PKV_HD bool done() const { return f >= f1; }
  PKV_HD int64_t seg_units() const {
    const int64_t a = ri.units - u, bnd = f1 - f;
    return a < bnd ? a : bnd;
  }
  // the segment's tiles of the pair: [t0, t1)
  PKV_HD int64_t t0() const { return u > kSegmentCost ? u - kSegmentCost : 0; }
  PKV_HD int64_t t1() const {
    const int64_t e = u + seg_units() - kSegmentCost;
    return e > 0 ? e : 0;
  }
  PKV_HD int64_t pair_start() const { return (int64_t)Hkv * Cb + (int64_t)kvh * ri.units; }
  // move past the current segment
  PKV_HD void advance() {
    f += seg_units();
    u = 0;
    if (++kvh < Hkv) return;
    kvh = 0;
    Cb += ri.units;
    if (f >= f1) return;
    do {
      ++b;
      ri = request_info(tv, b, ps);
    } while (ri.units == 0 && b + 1 < B);
  }
};

}  // namespace pkv
