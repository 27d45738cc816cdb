// partition.cuh -- split-KV work partition, shared by the decode kernel and
// by its host mirror (pkv_plan_segments).
//
// The decode work is the flattened sequence of 16-token tiles
//     (request b, kv head g, tile t),  b-major, then g, then t,
// W = num_kv_heads * sum_b tiles(b) tiles in all.  Partition c of N takes the
// contiguous share [floor(c W / N), floor((c+1) W / N)), so every CTA streams
// the same number of tiles (+-1) whatever the length mix: one long sequence
// is spread over all SMs, many short ones are packed together.  This is the
// split-KV idea (a long sequence's keys cut into blocks whose partial
// softmax states are combined afterwards); the pages describe the
// combination step as blockwise/ring attention ("大模型长上下文窗口工程化实战：
// 从RoPE扩展到百万Token推理的生产级部署", section 4.2) and the launch sized from
// the non-zero work rather than a fixed grid ("上下文窗口优化实战：如何用
// PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？", section 2.4).
//
// A (request, kv head) pair whose tiles fall in several partitions leaves one
// partial (o, lse) state per partition.  Partition c owns state slots 2c (its
// first pair) and 2c+1 (its last pair, when that pair started before c's
// share), so 2N slots always suffice.  The pair's first partition owns its
// arrival counter; the partition that arrives last merges.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define PKV_HD __host__ __device__ __forceinline__
#else
#define PKV_HD inline
#endif

namespace pkv {

constexpr int kTileTokens = 16;

// device error bits (same values as PKV_DEVERR_* in pkv.h)
constexpr int kErrPageId = 0x01;
constexpr int kErrIndptr = 0x02;
constexpr int kErrLastLen = 0x04;
constexpr int kErrAppend = 0x08;
constexpr int kErrTimeout = 0x10;

struct ReqInfo {
  int32_t page_base;  // page_indptr[b]
  int32_t err;        // error bits (request then counts as empty)
  int64_t len;        // tokens
  int64_t tiles;      // ceil(len / 16)
};

// Length of request b from the CSR table: (np - 1) * page_size + last_page_len.
PKV_HD ReqInfo request_info(const int32_t* indptr, const int32_t* last_len, int b, int ps) {
  ReqInfo r;
  r.page_base = indptr[b];
  r.err = 0;
  r.len = 0;
  r.tiles = 0;
  const int64_t np = (int64_t)indptr[b + 1] - (int64_t)r.page_base;
  if (r.page_base < 0 || np < 0) {
    r.err = kErrIndptr;
    return r;
  }
  if (np == 0) return r;
  const int ll = last_len[b];
  if (ll < 1 || ll > ps) {
    r.err = kErrLastLen;
    return r;
  }
  r.len = (np - 1) * (int64_t)ps + ll;
  r.tiles = (r.len + kTileTokens - 1) / kTileTokens;
  return r;
}

// First flat tile of partition c.
PKV_HD int64_t part_start(int64_t W, int N, int64_t c) { return (W * c) / N; }

// Partition holding flat tile f (0 <= f < W): the largest c with part_start(c) <= f.
PKV_HD int part_of(int64_t W, int N, int64_t f) { return (int)(((f + 1) * N - 1) / W); }

// Where a segment's result goes.  pair_start = first flat tile of the
// (request, kv head) pair, pair_tiles = its tile count, c = this partition.
struct SegPlace {
  int c_first;   // first partition covering the pair (owns the counter)
  int ncover;    // partitions covering the pair
  int slot;      // partial-state slot of (pair, c), -1 if ncover == 1
};

PKV_HD int state_slot(int64_t W, int N, int64_t pair_start, int c_first, int c) {
  return 2 * c + ((c == c_first && pair_start != part_start(W, N, c)) ? 1 : 0);
}

PKV_HD SegPlace seg_place(int64_t W, int N, int64_t pair_start, int64_t pair_tiles, int c) {
  SegPlace p;
  p.c_first = part_of(W, N, pair_start);
  const int c_last = part_of(W, N, pair_start + pair_tiles - 1);
  p.ncover = c_last - p.c_first + 1;
  p.slot = p.ncover == 1 ? -1 : state_slot(W, N, pair_start, p.c_first, c);
  return p;
}

// Sequential walk over the segments of one partition.  Table pointers may be
// host or device memory (whichever side runs the walk).
struct Walk {
  const int32_t* indptr;
  const int32_t* last_len;
  int B, ps, Hkv;
  int b, kvh;
  int64_t t;      // tile within the pair
  int64_t Cb;     // sum of tiles(b') for b' < b
  int64_t f, f1;  // current flat tile, end of the partition
  ReqInfo ri;     // info of request b

  // start at flat tile f0 inside request b0 (whose tiles start at Cb0)
  PKV_HD void start(int b0, int64_t Cb0, const ReqInfo& ri0, int64_t f0, int64_t f_end) {
    b = b0;
    Cb = Cb0;
    ri = ri0;
    f = f0;
    f1 = f_end;
    const int64_t r = f0 - (int64_t)Hkv * Cb0;
    kvh = ri0.tiles ? (int)(r / ri0.tiles) : 0;
    t = ri0.tiles ? r % ri0.tiles : 0;
  }
  PKV_HD bool done() const { return f >= f1; }
  PKV_HD int64_t seg_tiles() const {
    const int64_t a = ri.tiles - t, bnd = f1 - f;
    return a < bnd ? a : bnd;
  }
  PKV_HD int64_t pair_start() const { return (int64_t)Hkv * Cb + (int64_t)kvh * ri.tiles; }
  // move past the current segment
  PKV_HD void advance() {
    f += seg_tiles();
    t = 0;
    if (++kvh < Hkv) return;
    kvh = 0;
    Cb += ri.tiles;
    if (f >= f1) return;
    do {
      ++b;
      ri = request_info(indptr, last_len, b, ps);
    } while (ri.tiles == 0 && b + 1 < B);
  }
};

}  // namespace pkv
