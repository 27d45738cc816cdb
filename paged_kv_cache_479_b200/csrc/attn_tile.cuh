// attn_tile.cuh -- one consumer warp's share of a FlashAttention-style tile
// step with many query rows: 16 query rows against a 64-token K/V tile in
// shared memory, on the m16n8k16 tensor-core MMA with fp32 accumulation.
//
//     S[16 x 64]  = Q[16 x 128] . K_tile^T
//     online softmax over S (running max and sum in log2 units)
//     O[16 x 128] += P[16 x 64] . V_tile     (bf16: P split into high + low parts)
//
// This is the blockwise recursive softmax of "大模型推理极致优化：FlashAttention+
// PageAttention联合调优" section 2.2 for a block of query rows, used by the
// shared-prefix kernel (prefix.cu).
//
// Shared-memory tile: K (then V) of 64 tokens as four 16-token bulk-tensor
// boxes, each [2][16][64] elements with the 128-byte swizzle.
#pragma once
#include <math.h>

#include "common.cuh"
#include "partition.cuh"

namespace pkv {
namespace tile {

constexpr int kD = 128;
constexpr int kTile = 64;                        // tokens per tile
constexpr int kBoxes = kTile / kTileTokens;      // 16-token boxes per K (or V) tile
constexpr int kBoxBytes = kTileTokens * kD * 2;  // 4 KiB
constexpr int kHalf = kBoxBytes / 2;             // one [16][64] half of a box
constexpr int kKVBytes = kBoxes * kBoxBytes;     // 16 KiB for K (and for V) of a tile

// byte offset of (token t of the tile, 16-byte chunk c of its 128 dims)
__device__ __forceinline__ uint32_t tile_off(int t, int c) {
  const int bx = t >> 4, tt = t & 15;
  return (uint32_t)(bx * kBoxBytes + (c >> 3) * kHalf + tt * 128 + (((c & 7) ^ (tt & 7)) << 4));
}

// this lane's query rows g and g+8 (q0 / q1, null = no row) as A fragments
__device__ __forceinline__ void load_q(const uint16_t* q0, const uint16_t* q1, int cq,
                                       uint32_t (&qa)[8][4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int d0 = j * 16 + 2 * cq;
    qa[j][0] = q0 ? *reinterpret_cast<const uint32_t*>(q0 + d0) : 0u;
    qa[j][1] = q1 ? *reinterpret_cast<const uint32_t*>(q1 + d0) : 0u;
    qa[j][2] = q0 ? *reinterpret_cast<const uint32_t*>(q0 + d0 + 8) : 0u;
    qa[j][3] = q1 ? *reinterpret_cast<const uint32_t*>(q1 + d0 + 8) : 0u;
  }
}

// S = Q K^T: sc[n] holds tokens n*8 + 2cq, +1 of rows g (0, 1) and g+8 (2, 3)
template <bool BF16>
__device__ __forceinline__ void qk(const uint32_t (&qa)[8][4], uint32_t kb, int lane,
                                   float (&sc)[8][4]) {
  const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int n = 0; n < 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {  // n-tile pair (2np, 2np+1)
      const int tok = np * 16 + (mi >> 1) * 8 + r8;
      const int chunk = j * 2 + (mi & 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(kb + tile_off(tok, chunk), b0, b1, b2, b3);
      mma_16816<BF16>(sc[2 * np], qa[j][0], qa[j][1], qa[j][2], qa[j][3], b0, b1);
      mma_16816<BF16>(sc[2 * np + 1], qa[j][0], qa[j][1], qa[j][2], qa[j][3], b2, b3);
    }
  }
}

// Online-softmax step over scores already scaled to log2 units, -inf where a
// key is not visible; sc becomes P.  A row that has seen no visible key yet
// keeps m = -inf and l = 0 (its P is 0: the exponent is taken against 0).
__device__ __forceinline__ void online_softmax(float (&sc)[8][4], float& m0, float& m1, float& l0,
                                               float& l1, float (&o)[16][4]) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    mx0 = fmaxf(mx0, fmaxf(sc[n][0], sc[n][1]));
    mx1 = fmaxf(mx1, fmaxf(sc[n][2], sc[n][3]));
  }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
  const float al0 = mn0 == -INFINITY ? 1.f : ex2(m0 - mn0);
  const float al1 = mn1 == -INFINITY ? 1.f : ex2(m1 - mn1);
  const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
  m0 = mn0;
  m1 = mn1;
  float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    sc[n][0] = ex2(sc[n][0] - b0);
    sc[n][1] = ex2(sc[n][1] - b0);
    sc[n][2] = ex2(sc[n][2] - b1);
    sc[n][3] = ex2(sc[n][3] - b1);
    ps0 += sc[n][0] + sc[n][1];
    ps1 += sc[n][2] + sc[n][3];
  }
  l0 = l0 * al0 + ps0;
  l1 = l1 * al1 + ps1;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    o[n][0] *= al0;
    o[n][1] *= al0;
    o[n][2] *= al1;
    o[n][3] *= al1;
  }
}

// V rows at and past `valid` may hold anything (even NaN): zero them.  The
// caller issues fence_proxy_async_smem() before the slot is refilled by TMA.
__device__ __forceinline__ void zero_v_rows(uint8_t* vtile, int valid, int lane) {
  for (int idx = lane; idx < (kTile - valid) * 16; idx += 32) {
    const int t = valid + (idx >> 4), c = idx & 15;
    *reinterpret_cast<uint4*>(vtile + tile_off(t, c)) = make_uint4(0, 0, 0, 0);
  }
  __syncwarp();
}

// O += P V (P of two adjacent n-tiles is the A fragment of one k-step)
template <bool BF16>
__device__ __forceinline__ void pv(const float (&sc)[8][4], uint32_t vb, int lane,
                                   float (&o)[16][4]) {
  const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t ah[4], al[4];
    const float* p0 = sc[2 * kk];
    const float* p1 = sc[2 * kk + 1];
    ah[0] = pack2<BF16>(p0[0], p0[1]);
    ah[1] = pack2<BF16>(p0[2], p0[3]);
    ah[2] = pack2<BF16>(p1[0], p1[1]);
    ah[3] = pack2<BF16>(p1[2], p1[3]);
    if constexpr (BF16) {
      float2 f;
      f = unpack2<true>(ah[0]); al[0] = pack2<true>(p0[0] - f.x, p0[1] - f.y);
      f = unpack2<true>(ah[1]); al[1] = pack2<true>(p0[2] - f.x, p0[3] - f.y);
      f = unpack2<true>(ah[2]); al[2] = pack2<true>(p1[0] - f.x, p1[1] - f.y);
      f = unpack2<true>(ah[3]); al[3] = pack2<true>(p1[2] - f.x, p1[3] - f.y);
    }
#pragma unroll
    for (int np = 0; np < 8; ++np) {  // dim n-tile pair (2np, 2np+1)
      const int tok = kk * 16 + (mi & 1) * 8 + r8;
      const int chunk = 2 * np + (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(vb + tile_off(tok, chunk), b0, b1, b2, b3);
      mma_16816<BF16>(o[2 * np], ah[0], ah[1], ah[2], ah[3], b0, b1);
      mma_16816<BF16>(o[2 * np + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
      if constexpr (BF16) {
        mma_16816<BF16>(o[2 * np], al[0], al[1], al[2], al[3], b0, b1);
        mma_16816<BF16>(o[2 * np + 1], al[0], al[1], al[2], al[3], b2, b3);
      }
    }
  }
}

}  // namespace tile
}  // namespace pkv
