// internal.h -- launch entry points shared between the kernel files and the
// C ABI layer (api.cu).  Not installed; the public interface is include/pkv.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "partition.cuh"
#include "pkv.h"

namespace pkv {

// record the detail that pkv_last_error() reports on this thread; returns s
pkv_status set_error(pkv_status s, const char* fmt, ...);

struct DecodeArgs {
  const void* q;          // [B][Hq][128]
  void* out;              // [B][Hq][128]
  float* lse;             // [B][Hq] or null
  TableView tv;           // page table (CSR or dense block table)
  const int32_t* indices; // page ids: CSR indices, or the [B][max_blocks] block table
  int* counters;          // [N] arrival counters (zero between launches)
  float* part_lse;        // [2N][pcols], log2 domain
  float* part_o;          // [2N][pcols][128]
  int* err;               // device error word or null
  long long num_pages;
  int batch, hq, hkv, group, page_size;
  float scale_log2;       // sm_scale * log2(e) (* k_scale for an E4M3 pool)
  float v_scale;          // 8-bit pool: value of a V code = code value * v_scale
  int one_box;            // 1: 5-D tensor map, one box per K/V tile; 0: 4-D map, two boxes
  int out_f32;            // 1: out is fp32 (an attention state for a later merge)
  long long out_rs;       // elements of out between consecutive requests (Hq * 128 when packed)
  long long lse_rs;       // elements of lse between consecutive requests (Hq when packed)
  // short chunks: request b's query tokens are rows qo_indptr[b] .. of q / out
  // (null for decode: one token, row b)
  const int32_t* qo_indptr;
  long long nnz_q;        // rows of q (short chunks)
  int pcols;              // columns per partial-state slot (G for decode)
  int max_cols;           // short chunks: the caller's bound on q_len * G
  // fused append (16-bit pools; k_new null = none): the step's new rows
  // k_new / v_new [nnz_new][Hkv][128], request b's at append_indptr[b] ..,
  // written into the pool (layout: PKV_LAYOUT_*) before the tiles holding them
  // are loaded
  void* pool;
  int layout;
  const void* k_new;
  const void* v_new;
  const int32_t* append_indptr;
  long long nnz_new;
  // time limit of every pipeline wait (ns); the drain of a CTA's own copies
  // before it exits always uses the full kWaitLimitNs
  unsigned long long wait_ns;
  // 1: the table is not written by the preceding kernel in the stream, so it
  // is read (and the partition planned) before waiting for that kernel
  int early_table;
};

// wait limit of the decode kernel's pipeline waits (pkv_set_wait_limit_ns)
unsigned long long decode_wait_limit_ns();

// Bytes at the start of pkv_decode's workspace that hold its arrival
// counters (the only part that must be zero before a launch), for the GQA
// group and partition count given (0 = the current device's default).
size_t decode_counter_bytes(int group, int num_partitions);

// Raise `func`'s dynamic shared-memory limit to `bytes` on the current device,
// once per (function, device); safe to call from several host threads.
cudaError_t ensure_smem_opt_in(const void* func, size_t bytes);

#ifndef PKV_STAGES
#define PKV_STAGES 16
#endif
#ifndef PKV_CTAS_PER_SM
#define PKV_CTAS_PER_SM 1
#endif
constexpr int kDecodeStages = PKV_STAGES;        // K/V ring slots (8 KiB each) per CTA
constexpr int kDecodeCtasPerSm = PKV_CTAS_PER_SM; // resident decode CTAs per SM

size_t decode_smem_bytes(int nq);
// pool element types of the decode kernel
constexpr int kKv16 = 0;    // q's own 16-bit type
constexpr int kKvE4M3 = 1;  // FP8 E4M3 codes
constexpr int kKvE5M2 = 2;  // FP8 E5M2 codes
// bf16: q/out type (else fp16); kv: one of the pool element types above
// nq: n8 column tiles per (request, kv head) -- 1, or 2 (16-bit pools only)
cudaError_t launch_decode(const CUtensorMap& tmap, const DecodeArgs& a, bool bf16, int kv, int nq,
                          int grid, cudaStream_t stream);

// many-row attention on tcgen05 (chunk_tc.cu): multi-token append attention
// (rows from a host plan, each request's own pages, causal), or the shared
// prefix of a cascade (prefix_pages set: rows = (request, head) pairs of every
// request, keys = the prefix, no mask, fp32 states)
struct ChunkArgs {
  const void* q;               // [nnz_q][Hq][128]
  const int32_t* qo_indptr;    // [B+1], qo_indptr[0] = 0
  TableView tv;                // the table after the append
  const int32_t* indices;
  const int4* plan;            // row blocks {request, first row, rows, 0}
  void* out;                   // [nnz_q][Hq][128] (one split)
  float* lse;                  // [nnz_q][Hq] or null (one split)
  float* state_o;              // [nnz_q][states][Hq][128]: slot `split` written
  float* state_lse;            // [nnz_q][states][Hq]
  const int32_t* prefix_pages; // shared prefix: its page ids (null for append attention)
  long long prefix_len;        // shared prefix: tokens
  int states;                  // state slots per row
  int out_states;              // 1: write fp32 states, 0: the final 16-bit output
  int* err;
  long long num_pages;
  long long nnz_q;             // rows of q / out
  int batch, hq, hkv, group, page_size, splits, window_left, sink;
  float scale_log2;
  int one_box;
  int q_tma;                   // 1: qmap describes q (G divides 128), Q comes in by bulk-tensor loads
  int o_tma;                   // 1: omap describes state_o, full row tiles' states go out by bulk-tensor stores
};
// chunk_tc.cu (tcgen05); its tensor map has [16][64] boxes (one dim half each)
int chunk_rows_per_cta();
int chunk_tile_tokens();
size_t chunk_tc_smem_bytes();
// q / state tensor maps for ChunkArgs::q_tma / o_tma; false when the shapes do
// not allow them (the kernel then stages Q and writes states per thread)
bool chunk_q_map(const void* q, long long nnz_q, int hq, int group, bool bf16, CUtensorMap* m);
bool chunk_state_map(float* state_o, long long nnz_q, int states, int hq, int group, CUtensorMap* m);
cudaError_t launch_chunk_tc(const CUtensorMap& tmap, const CUtensorMap& qmap,
                            const CUtensorMap& omap, const ChunkArgs& a, bool bf16, int row_blocks,
                            cudaStream_t stream);

struct AppendArgs {
  void* pool;
  TableView tv;
  const int32_t* indices;
  const int32_t* append_indptr;
  const void* k_new;
  const void* v_new;
  int* err;
  long long num_pages;
  long long nnz;
  int batch, hkv, head_dim, page_size;
  int layout;  // PKV_LAYOUT_HND or PKV_LAYOUT_NHD
  int fp8;     // kKvE4M3 / kKvE5M2: rows are quantised as fp8(x / scale); 0: 16-bit copy
  int in_bf16; // fp8 only: k_new / v_new are bf16 (else fp16)
  float k_scale, v_scale;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

struct MergeArgs {
  const float* v;
  const float* s;
  void* v_out;
  float* s_out;
  long long rows;
  int states, heads, head_dim, out_dtype;
  int vec4;  // 1: head_dim 128, v and v_out 16-byte aligned (16-byte loads, 8- or 16-byte stores)
  int rows_ok;  // 1: s 16-byte aligned too (whole rows may be bulk-copied to shared memory)
};
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream);

}  // namespace pkv
