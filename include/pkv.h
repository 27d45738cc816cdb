/*
 * pkv.h -- C ABI of libpkv: batched decode attention over a paged KV cache
 * on NVIDIA B200 (sm_100a).
 *
 * The operation (PagedAttention computed FlashAttention-style):
 *   For each request b and query head h, one new query token q[b][h][:]
 *   attends over the request's cached keys and values:
 *       o[b][h] = softmax(sm_scale * q K^T) V,   lse[b][h] = log sum_t exp(sm_scale * q.k_t)
 *   which is the standard attention Attention(Q,K,V) = softmax(QK^T/sqrt(d))V
 *   ("大模型推理极致优化：FlashAttention+PageAttention联合调优", section 2.1)
 *   for one query row.  K and V sit in fixed-size physical pages reached
 *   through a per-request page table ("上下文窗口优化实战：如何用PagedAttention+FlashInfer
 *   将Llama3-70B的128K上下文吞吐提升3.8倍？", chapter 1 and section 2.3: the decode
 *   kernel takes the page table and the block size directly).  Scores are
 *   never written to memory: softmax is computed online over blocks of keys
 *   ("大模型推理极致优化：FlashAttention+PageAttention联合调优", section 2.2).
 *
 * Memory layout (all arrays are the caller's, row-major, on the device
 * unless a name ends in _h):
 *   pool            [num_pages][2][num_kv_heads][page_size][head_dim]  fp16/bf16
 *                   index 0 of the second axis holds K, index 1 holds V.
 *   page_indptr     int32 [batch+1]   request b owns page_indices[page_indptr[b] ..
 *                                     page_indptr[b+1]) in logical order
 *   page_indices    int32 [page_indptr[batch]]   physical page ids in [0, num_pages)
 *   last_page_len   int32 [batch]     tokens in the request's last page, in
 *                                     [1, page_size] when it owns a page
 *   The request holds len_b = (np_b - 1) * page_size + last_page_len[b] tokens,
 *   np_b = page_indptr[b+1] - page_indptr[b]; len_b = 0 when np_b = 0.  The
 *   same physical page may appear in several requests (a shared prefix).
 *   q, out          [batch][num_qo_heads][head_dim], same 16-bit type as the pool
 *   lse             float [batch][num_qo_heads], natural log
 *   Query head h reads KV head h / (num_qo_heads / num_kv_heads).
 *
 * Ownership and errors: the library allocates no memory and never
 * synchronises the stream (except pkv_read_error_word).  Every call checks
 * its scalar arguments on the host and returns a status without launching
 * when they are invalid; pkv_last_error() then describes the problem.
 * Table CONTENTS live on the device and are checked by the kernels: a bad
 * page id, indptr or last_page_len sets a bit in the optional caller-owned
 * device word `error_word` (PKV_DEVERR_*), the offending page or request is
 * skipped, and the kernel still completes.  No kernel traps or waits without
 * a time limit; a wait that runs past its limit sets PKV_DEVERR_TIMEOUT.
 * `stream` is a cudaStream_t (NULL = the legacy default stream).
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,   /* a scalar argument or pointer is invalid */
  PKV_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels implement */
  PKV_ERR_WORKSPACE = 3,     /* workspace too small or misaligned */
  PKV_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  PKV_ERR_DEVICE = 5         /* pkv_read_error_word found device error bits */
} pkv_status;

typedef enum pkv_dtype {
  PKV_F16 = 0,
  PKV_BF16 = 1,
  PKV_F32 = 2,               /* only as the output type of pkv_merge_states */
  PKV_FP8_E4M3 = 3,          /* only as a pool type, with pkv_decode_fp8 / pkv_append_fp8 */
  PKV_FP8_E5M2 = 4           /* likewise */
} pkv_dtype;

/* Pool layouts (the simple calls use HND). */
typedef enum pkv_layout {
  PKV_LAYOUT_HND = 0,  /* pool[page][2][kv_head][slot][head_dim]: one head's slots contiguous */
  PKV_LAYOUT_NHD = 1   /* pool[page][2][slot][kv_head][head_dim]: one slot's heads contiguous */
} pkv_layout;

/* A KV pool: `data` holds num_pages pages of 2 (K, V) x num_kv_heads x page_size
 * x head_dim elements of `dtype`, in `layout` order. */
typedef struct pkv_pool_desc {
  void* data;
  int64_t num_pages;
  int32_t page_size;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t dtype;   /* pkv_dtype */
  int32_t layout;  /* pkv_layout */
  int32_t reserved;
} pkv_pool_desc;

/* Page-table forms. */
typedef enum pkv_table_kind {
  PKV_TABLE_CSR = 0,   /* page_indptr / page_indices / last_page_len, as in the simple calls */
  PKV_TABLE_BLOCK = 1  /* dense block table + context lengths (the vLLM form, "上下文窗口优化实战：
                          如何用PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？"
                          section 4.3: block_table [batch, max_blocks_per_seq], context_lens [batch]) */
} pkv_table_kind;

/* A page table (device arrays).  CSR: request b owns page_indices[page_indptr[b] ..
 * page_indptr[b+1]) and holds (np-1)*page_size + last_page_len[b] tokens.  BLOCK:
 * request b owns block_table[b][0 .. ceil(context_lens[b]/page_size)) and holds
 * context_lens[b] tokens (at most max_blocks_per_seq * page_size; more sets
 * PKV_DEVERR_CONTEXT_LEN and the request is treated as empty). */
typedef struct pkv_table_desc {
  int32_t kind;   /* pkv_table_kind */
  int32_t batch;
  const int32_t* page_indptr;
  const int32_t* page_indices;
  const int32_t* last_page_len;
  const int32_t* block_table;
  const int32_t* context_lens;
  int32_t max_blocks_per_seq;
  int32_t flags;  /* PKV_TABLE_* bits, 0 for none */
} pkv_table_desc;

/*
 * PKV_TABLE_READY_AT_LAUNCH: the caller promises that the page table (indptr /
 * indices / last_page_len, or block_table / context_lens) is not written by
 * the kernel that runs just before this call in the stream.  The decode then
 * reads the table and plans its split-KV partition while that kernel is still
 * finishing (programmatic dependent launch), and waits for it only before it
 * reads q, the pool or new rows and before it writes anything.  Host-to-device
 * copies of the table before the call are fine: a copy is not a kernel and
 * the decode starts after it.  Without the flag the decode waits first.
 */
#define PKV_TABLE_READY_AT_LAUNCH 0x1

/* Bits the kernels OR into *error_word. */
#define PKV_DEVERR_PAGE_ID   0x01  /* page id outside [0, num_pages): page skipped */
#define PKV_DEVERR_INDPTR    0x02  /* page_indptr decreasing or negative: request treated as empty */
#define PKV_DEVERR_LAST_LEN  0x04  /* last_page_len outside [1, page_size]: request treated as empty */
#define PKV_DEVERR_APPEND    0x08  /* append_indptr malformed or more new tokens than the request holds */
#define PKV_DEVERR_TIMEOUT   0x10  /* an internal wait ran past its time limit; outputs invalid */
#define PKV_DEVERR_CONTEXT_LEN 0x20 /* block table: context_lens[b] < 0 or beyond its row: request treated as empty */

/* Human-readable name of a status code (static string). */
PKV_API const char* pkv_status_string(int status);

/* Detail of the last non-OK status returned on this host thread ("" if none). */
PKV_API const char* pkv_last_error(void);

/*
 * Time limit, in nanoseconds, of every wait inside the decode kernel
 * (pkv_decode and the calls built on it) for launches made after this call;
 * 0 restores the default of one second.  Returns the previous limit.  A wait
 * that runs past it sets PKV_DEVERR_TIMEOUT and the CTA gives up: it still
 * lets its own copies in flight land (with the full one-second limit) and
 * counts itself in on the split pairs it shares, so the launch completes,
 * the CUDA context stays usable and the workspace can be reused as it is by
 * the next call; only that launch's outputs are invalid.  The library never
 * needs a limit below the default; a short one exists so that tests can make
 * a wait run out and check this error path.  Process-wide; safe to call from
 * any host thread.  (No counterpart in the pages: it is part of the failure
 * handling of this library.)
 */
PKV_API uint64_t pkv_set_wait_limit_ns(uint64_t nanoseconds);

/* Number of split-KV partitions pkv_decode uses when num_partitions = 0 on
 * `device`: one persistent CTA per SM.  Returns a value < 0 on error. */
PKV_API int pkv_default_partitions(int device);

/*
 * Workspace bytes pkv_decode needs for these shapes and this partition
 * count (num_partitions = 0 means pkv_default_partitions(current device)).
 * The workspace holds one arrival counter per partition and at most two
 * partial (o, lse) states per partition.  It must be 256-byte aligned and
 * ZERO-FILLED before its first use; every launch leaves the counters at zero
 * when it completes -- also a launch that set a PKV_DEVERR_* bit -- so the
 * same workspace can be reused by later calls on the same stream without
 * clearing.  Calls that overlap on the GPU must not share a workspace.
 * Returns 0 for invalid shapes.
 */
PKV_API size_t pkv_decode_workspace_bytes(int batch, int num_qo_heads, int num_kv_heads,
                                  int head_dim, int num_partitions);

/*
 * pkv_append -- scatter new tokens' K and V into their pages
 * (a1 of the decode step: pages are allocated on demand by the caller,
 * "大模型推理极致优化：FlashAttention+PageAttention联合调优" section 3.2;
 * position p of a request lives at page page_indices[page_indptr[b] + p / page_size],
 * slot p % page_size, "Flash Attention与Paged KV Cache优化大模型推理实战" section 3.2).
 *
 *   pool                the KV pool (written in place)
 *   page_indptr, page_indices, last_page_len, batch
 *                       the page table AFTER the append (pages already allocated)
 *   k_new, v_new        [nnz_new][num_kv_heads][head_dim] in the pool's dtype
 *   append_indptr       int32 [batch+1]; request b appends rows
 *                       append_indptr[b] .. append_indptr[b+1]) at its last
 *                       n_b positions: len_b - n_b + i
 *   nnz_new             append_indptr[batch] (rows in k_new / v_new)
 * Bit-exact copies; no other byte of the pool changes.  head_dim must be a
 * multiple of 8 and all data pointers 16-byte aligned.
 */
PKV_API pkv_status pkv_append(void* pool, int64_t num_pages, int page_size, int num_kv_heads,
                      int head_dim, int dtype,
                      const int32_t* page_indptr, const int32_t* page_indices,
                      const int32_t* last_page_len, int batch,
                      const void* k_new, const void* v_new, const int32_t* append_indptr,
                      int64_t nnz_new, int32_t* error_word, void* stream);

/*
 * pkv_decode -- batched decode attention over the paged KV cache.
 *
 *   q                [batch][num_qo_heads][head_dim], dtype = pool dtype, 16-byte aligned
 *   pool, num_pages, page_size, num_kv_heads, head_dim, dtype
 *                    the KV pool (16-byte aligned); head_dim must be 128,
 *                    page_size one of 16, 32, 64, 128, 256,
 *                    num_qo_heads / num_kv_heads (the GQA group) in 1..8
 *   page_indptr, page_indices, last_page_len, batch   the page table (device)
 *   sm_scale         score scale (1/sqrt(head_dim) for standard attention)
 *   num_partitions   split-KV partitions, 0 = pkv_default_partitions().  The
 *                    flattened work (request, kv head, 16-token tile) is cut
 *                    into this many equal contiguous shares, one per CTA; a
 *                    (request, kv head) cut across shares is merged exactly
 *                    by log-sum-exp weights inside the same launch.  Results
 *                    depend on the partition count only through fp32
 *                    rounding; for a fixed count they are bitwise
 *                    reproducible and independent of physical page placement.
 *   workspace        see pkv_decode_workspace_bytes (device, zero-filled once)
 *   out              [batch][num_qo_heads][head_dim] in dtype (must not alias q or pool)
 *   lse              float [batch][num_qo_heads] or NULL
 *   error_word       int32 device word for PKV_DEVERR_* bits, or NULL
 * A request with no tokens gets out = 0 and lse = -inf.
 */
PKV_API pkv_status pkv_decode(const void* q, int num_qo_heads,
                      const void* pool, int64_t num_pages, int page_size, int num_kv_heads,
                      int head_dim, int dtype,
                      const int32_t* page_indptr, const int32_t* page_indices,
                      const int32_t* last_page_len, int batch,
                      float sm_scale, int num_partitions,
                      void* workspace, size_t workspace_bytes,
                      void* out, float* lse, int32_t* error_word, void* stream);

/*
 * pkv_decode_ex / pkv_append_ex -- pkv_decode / pkv_append on a pool and a page
 * table given by descriptors, which adds the NHD pool layout and the dense
 * block-table form.  Same semantics, workspace (pkv_decode_workspace_bytes)
 * and error behaviour as the simple calls; with PKV_TABLE_BLOCK the table to
 * pass to pkv_append_ex is the table after the append (context_lens counts
 * the new tokens).
 */
PKV_API pkv_status pkv_decode_ex(const void* q, int num_qo_heads, const pkv_pool_desc* pool,
                                 const pkv_table_desc* table, float sm_scale, int num_partitions,
                                 void* workspace, size_t workspace_bytes, void* out, float* lse,
                                 int32_t* error_word, void* stream);
PKV_API pkv_status pkv_append_ex(const pkv_pool_desc* pool, const pkv_table_desc* table,
                                 const void* k_new, const void* v_new,
                                 const int32_t* append_indptr, int64_t nnz_new,
                                 int32_t* error_word, void* stream);

/*
 * pkv_decode_append -- one decode step in one launch: pkv_append_ex of the
 * step's new rows followed by pkv_decode_ex, fused.  The decode kernel writes
 * each new row into its page just before it loads the tile that holds it (the
 * one CTA that reads that tile), so the append costs no launch of its own.
 *   q, pool, table, sm_scale, num_partitions, workspace, out, lse, error_word,
 *   stream   as in pkv_decode_ex (the table is the one after the append)
 *   k_new, v_new, append_indptr, nnz_new   as in pkv_append_ex; the pool must be
 *            16-bit (PKV_F16 / PKV_BF16, as k_new / v_new; 8-bit pools:
 *            pkv_append_fp8 then pkv_decode_fp8); nnz_new = 0 is a plain decode
 * On return (stream order) the pool holds exactly what pkv_append_ex would have
 * written and out / lse what pkv_decode_ex would have computed on it.  A
 * request whose append_indptr entries start below 0, end past nnz_new or claim
 * more rows than the request holds sets PKV_DEVERR_APPEND and gets no rows
 * written (a decreasing pair appends nothing).  k_new / v_new must not alias
 * the pool or out.
 */
PKV_API pkv_status pkv_decode_append(const void* q, int num_qo_heads, const pkv_pool_desc* pool,
                                     const pkv_table_desc* table, const void* k_new,
                                     const void* v_new, const int32_t* append_indptr,
                                     int64_t nnz_new, float sm_scale, int num_partitions,
                                     void* workspace, size_t workspace_bytes, void* out,
                                     float* lse, int32_t* error_word, void* stream);

/*
 * pkv_decode_fp8 / pkv_append_fp8 -- the 8-bit KV cache: a pool of FP8 codes
 * ("fp8_e4m3" KV-cache dtype of the serving configurations in "上下文窗口优化
 * 实战：如何用PagedAttention+FlashInfer将Llama3-70B的128K上下文吞吐提升3.8倍？"
 * section 4.1; "fp8_e5m2" in "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token
 * 推理的生产级部署" sections 3.1 and 3.2), half the bytes of a 16-bit pool.
 *
 * E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits, subnormals,
 * no infinity, codes 0x7f / 0xff are NaN; largest finite magnitude 448.
 * E5M2: the top byte of an IEEE half (bias 15, 2 fraction bits, infinities
 * and NaNs); largest finite magnitude 57344.  One binary32 scale for all keys
 * and one for all values: a key element is value(code) * k_scale, a value
 * element value(code) * v_scale.
 *
 *   pool       descriptor with dtype PKV_FP8_E4M3 or PKV_FP8_E5M2 (either
 *              layout; head_dim 128 for the decode, a multiple of 8 for the
 *              append); element bytes
 *   k_scale, v_scale  finite and > 0, else PKV_ERR_INVALID_ARG
 *   q_dtype    PKV_F16 or PKV_BF16: the type of q and out (decode)
 *   new_dtype  PKV_F16 or PKV_BF16: the type of k_new / v_new (append)
 *
 * pkv_decode_fp8 computes what pkv_decode_ex computes on the widened keys and
 * values (same table forms, workspace, out / lse and error behaviour).
 * pkv_append_fp8 scatters like pkv_append_ex and stores each new element x
 * as fp8(float(x) / scale): the quotient rounded to binary32, then to the
 * nearest finite value of the format, ties to even, larger magnitudes
 * (infinity included) saturating to +-448 (E4M3) or +-57344 (E5M2).  The _ex
 * calls reject 8-bit pools (they carry no scales); pkv_cascade_decode and
 * pkv_append_attention take 16-bit pools only.
 */
PKV_API pkv_status pkv_decode_fp8(const void* q, int q_dtype, int num_qo_heads,
                                  const pkv_pool_desc* pool, float k_scale, float v_scale,
                                  const pkv_table_desc* table, float sm_scale,
                                  int num_partitions, void* workspace, size_t workspace_bytes,
                                  void* out, float* lse, int32_t* error_word, void* stream);
PKV_API pkv_status pkv_append_fp8(const pkv_pool_desc* pool, float k_scale, float v_scale,
                                  const pkv_table_desc* table, const void* k_new,
                                  const void* v_new, int new_dtype,
                                  const int32_t* append_indptr, int64_t nnz_new,
                                  int32_t* error_word, void* stream);

/*
 * Multi-token append attention: each request's chunk of new query tokens
 * attends over its paged cache with a causal mask -- chunked prefill (a long
 * prompt processed a chunk at a time against the cache that holds the earlier
 * chunks, "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署"
 * section 3.1) and the verification of several speculative tokens at once.
 *
 * Request b's q_len_b = qo_indptr[b+1] - qo_indptr[b] query tokens are rows
 * qo_indptr[b] .. of q (qo_indptr[0] = 0, nnz_q = qo_indptr[batch]).  The
 * table is the table AFTER the chunk's K/V were appended (pkv_append*): the
 * request holds L_b >= q_len_b tokens and query i sits at position
 * pos = L_b - q_len_b + i.  Key t is visible to it when t <= pos and, if
 * window_left >= 0, also t >= pos - window_left or t < sink_tokens (the
 * sliding window with global tokens of the same article's section 2.3, cut
 * to its causal half; window_left < 0 = no window).  Query head h reads KV
 * head h / (Hq / Hkv); out / lse as in pkv_decode, per query token.
 *
 * pkv_append_attention_plan (host only) -- the row blocks of the launch:
 *   qo_indptr_h  host int32 [batch+1]
 *   kv_len_h     host int32 [batch]: L_b (tokens after the append), or NULL
 *   plan_h       host int32 [capacity][4] or NULL: {request, first row, rows, 0}
 *                per block of up to 256 rows (row r = chunk token r / G, query
 *                head kv_head * G + r % G), the blocks with the most key tiles
 *                first (the launch runs them in plan order, every kv head of a
 *                block before the next block, so it ends on short ones)
 *   num_splits   if not NULL, receives a split count for the launch: 1 when
 *                the row blocks fill num_sms SMs (or kv_len_h is NULL), else
 *                enough key splits for about two CTAs per SM
 *   returns the number of row blocks (entries beyond capacity are not
 *   written), or -1 for invalid arguments.
 *
 * pkv_append_attention_workspace_bytes -- fp32 partial states needed with
 *   num_splits > 1 (0 with one split).
 *
 * pkv_append_attention -- the launch:
 *   q             [nnz_q][num_qo_heads][128], the pool's dtype, 16-byte aligned
 *   qo_indptr     device int32 [batch+1]
 *   pool, table   descriptors (16-bit pools, either layout, either table form)
 *   plan          device int32 [num_row_blocks][4] from the planner, 16-byte aligned
 *   num_splits    1..1024; the same value the workspace was sized for
 *   workspace     device, 256-byte aligned (may be NULL with one split)
 *   out           [nnz_q][num_qo_heads][128] pool dtype;  lse float [nnz_q][Hq] or NULL
 * Errors as in pkv_decode; a plan entry or request that does not fit the table
 * sets PKV_DEVERR_APPEND (or the table's bit) and leaves its rows unwritten.
 */
PKV_API int64_t pkv_append_attention_plan(const int32_t* qo_indptr_h, const int32_t* kv_len_h,
                                          int batch, int num_qo_heads, int num_kv_heads,
                                          int window_left, int sink_tokens, int num_sms,
                                          int32_t* plan_h, int64_t capacity, int32_t* num_splits);
PKV_API size_t pkv_append_attention_workspace_bytes(int64_t nnz_q, int num_qo_heads,
                                                    int num_splits);
PKV_API pkv_status pkv_append_attention(const void* q, const int32_t* qo_indptr, int64_t nnz_q,
                                        int num_qo_heads, const pkv_pool_desc* pool,
                                        const pkv_table_desc* table, const int32_t* plan,
                                        int64_t num_row_blocks, int num_splits, int window_left,
                                        int sink_tokens, float sm_scale, void* workspace,
                                        size_t workspace_bytes, void* out, float* lse,
                                        int32_t* error_word, void* stream);

/*
 * pkv_append_attention_short -- pkv_append_attention (no window) for chunks of
 * at most max_q_len tokens with max_q_len * G <= 16 (G = num_qo_heads /
 * num_kv_heads), e.g. the verification of a few speculative tokens.  It runs
 * the decode kernel's split-KV schedule with the chunk's (token, head) pairs
 * as the columns of its MMAs, so each K/V tile is read once per (request, kv
 * head) and the work is spread over the SMs by cost whatever the length mix.
 *   q, qo_indptr, nnz_q, out, lse  as in pkv_append_attention
 *   max_q_len    host bound on every request's q_len (1 <= max_q_len, max_q_len
 *                * G <= 16, else PKV_ERR_UNSUPPORTED); a request whose q_len is
 *                larger, or larger than its cache, sets PKV_DEVERR_APPEND and its
 *                rows are left unwritten; requests with q_len = 0 write nothing
 *   pool, table  descriptors (16-bit pools, head_dim 128, either layout and form)
 *   k_new, v_new, append_indptr, nnz_new   optional (nnz_new = 0: none): the
 *                chunk's own K/V rows as in pkv_append_ex, written into the pool
 *                by the same launch before the tiles that hold them are loaded
 *                (the pool ends bitwise as after pkv_append_ex; 16-bit rows)
 *   num_partitions, workspace  as in pkv_decode, the workspace sized by
 *                pkv_append_attention_short_workspace_bytes (device, zero-filled
 *                once; the kernel leaves its counters zeroed)
 * Same results as pkv_append_attention up to rounding order.
 */
PKV_API size_t pkv_append_attention_short_workspace_bytes(int num_qo_heads, int num_kv_heads,
                                                          int max_q_len, int num_partitions);
PKV_API pkv_status pkv_append_attention_short(const void* q, const int32_t* qo_indptr,
                                              int64_t nnz_q, int max_q_len, int num_qo_heads,
                                              const pkv_pool_desc* pool,
                                              const pkv_table_desc* table, const void* k_new,
                                              const void* v_new, const int32_t* append_indptr,
                                              int64_t nnz_new, float sm_scale,
                                              int num_partitions, void* workspace,
                                              size_t workspace_bytes, void* out, float* lse,
                                              int32_t* error_word, void* stream);

/*
 * pkv_cascade_decode -- pkv_decode for a batch whose requests all begin with
 * the same shared prefix (a system prompt stored once in shared pages: physical
 * page sharing between requests with a common prefix, "大模型推理极致优化：
 * FlashAttention+PageAttention联合调优" section 3.2; automatic prefix reuse,
 * "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署" section 3.3).
 *
 * Request b attends over the prefix's prefix_len tokens followed by its own
 * tokens; the result equals pkv_decode on the concatenated page lists up to
 * fp32 rounding.  Instead of reading the prefix once per request, the prefix's
 * K/V are read once per block of 256 (request, query head) rows and multiplied
 * on tensor cores against all requests' queries; each request's own pages go
 * through the decode kernel; the two attention states are merged by their
 * log-sum-exp weights.
 *
 *   prefix_page_indices  device int32 [ceil(prefix_len / page_size)]: the prefix's
 *                        pages in order (the last one holds the remainder)
 *   prefix_len           prefix tokens (0: plain pkv_decode)
 *   page_indptr, page_indices, last_page_len, batch
 *                        each request's OWN pages after the prefix (CSR; a request
 *                        with no own tokens has no pages)
 *   workspace            pkv_cascade_workspace_bytes(), 256-byte aligned, zero-filled
 *                        before first use (as for pkv_decode)
 * Other arguments as pkv_decode.  Three launches on `stream`; no allocation.
 */
PKV_API size_t pkv_cascade_workspace_bytes(int batch, int num_qo_heads, int num_kv_heads,
                                           int head_dim, int64_t prefix_len,
                                           int num_partitions);
PKV_API pkv_status pkv_cascade_decode(const void* q, int num_qo_heads, const void* pool,
                                      int64_t num_pages, int page_size, int num_kv_heads,
                                      int head_dim, int dtype,
                                      const int32_t* prefix_page_indices, int64_t prefix_len,
                                      const int32_t* page_indptr, const int32_t* page_indices,
                                      const int32_t* last_page_len, int batch, float sm_scale,
                                      int num_partitions, void* workspace,
                                      size_t workspace_bytes, void* out, float* lse,
                                      int32_t* error_word, void* stream);

/*
 * pkv_merge_states -- merge attention states of disjoint key sets.
 *
 *   v       float [num_rows][num_states][num_heads][head_dim]  normalised partial outputs
 *   s       float [num_rows][num_states][num_heads]            their natural-log lse
 *   v_out   [num_rows][num_heads][head_dim] in out_dtype (PKV_F32, PKV_F16, PKV_BF16)
 *   s_out   float [num_rows][num_heads] or NULL
 * With M = max_j s_j, w_j = exp(s_j - M): v_out = sum_j w_j v_j / sum_j w_j,
 * s_out = M + log sum_j w_j.  A state with s = -inf carries no weight; if all
 * do, v_out = 0 and s_out = -inf.  This is the exact form of the blockwise
 * combination sketched in "大模型长上下文窗口工程化实战：从RoPE扩展到百万Token推理的生产级部署"
 * section 4.2 (that sketch averages per-block softmax outputs, which is not exact).
 */
PKV_API pkv_status pkv_merge_states(const float* v, const float* s, int64_t num_rows, int num_states,
                            int num_heads, int head_dim, void* v_out, int out_dtype,
                            float* s_out, void* stream);

/*
 * pkv_read_error_word -- synchronise `stream`, copy the device error word to
 * *value (host), and zero it on the device when `clear` is non-zero.
 * Returns PKV_ERR_DEVICE when any bit is set, PKV_OK otherwise.
 */
PKV_API pkv_status pkv_read_error_word(int32_t* error_word, int32_t* value, int clear, void* stream);

/*
 * pkv_check_table -- host-side check of a page table the caller holds on the
 * host (the consistency rules of "Flash Attention与Paged KV Cache优化大模型推理实战"
 * section 6.2: a page's valid length never exceeds the page size; plus
 * monotone indptr and page ids inside the pool).  No GPU needed.
 */
PKV_API pkv_status pkv_check_table(const int32_t* page_indptr_h, const int32_t* page_indices_h,
                           const int32_t* last_page_len_h, int batch, int64_t num_pages,
                           int page_size);

/*
 * pkv_plan_segments -- host mirror of the device-side split-KV partition, for
 * inspection and tests (no GPU needed).  For the table held on the host it
 * lists every segment the `num_partitions` CTAs of pkv_decode process, seven
 * int64 per segment: partition, request, kv head, first tile, end tile
 * (16-token tiles), partial-state slot (-1 when the segment covers its whole
 * (request, kv head) and writes the output directly), partitions covering
 * that (request, kv head).  Writes at most max_segments rows to `segments`
 * and returns the total number of segments, or -1 on invalid arguments.
 */
PKV_API int64_t pkv_plan_segments(const int32_t* page_indptr_h, const int32_t* last_page_len_h,
                          int batch, int page_size, int num_kv_heads, int num_partitions,
                          int64_t* segments, int64_t max_segments);

/*
 * pkv_decode_static_workspace -- pkv_decode without a caller-provided workspace.
 *
 * The pages describe no such call; it exists for users of this library who
 * cannot allocate device memory at the point where they decode, and have no
 * spare device buffer to lend as workspace -- for example a serving engine
 * that reserved all free HBM for its KV pool up front, a plugin running
 * inside a host framework whose allocator it cannot reach, or a
 * latency-critical loop where cudaMalloc (which can synchronise the device)
 * is not allowed.
 *
 * Same arguments and results as pkv_decode, minus workspace and
 * workspace_bytes.  The scratch is a file-scope device array of 4 MiB inside
 * libpkv, present on every GPU that loads the library until the process
 * exits; it fits the default partition count for up to 8 query heads per KV
 * head (about 1.2 MiB on a 148-SM B200).  Calls needing more return
 * PKV_ERR_WORKSPACE without launching.  The call allocates nothing: its first
 * call on a device looks the array's device address up (make that first call
 * before any stream capture), and every call clears the part of the array it
 * uses with cudaMemsetAsync on `stream` before the kernel.  All calls share
 * the one array, which keeps the last call's contents: calls that can
 * overlap on the GPU (different streams, or different host threads) race on
 * it and must be serialised by the caller.
 */
PKV_API pkv_status pkv_decode_static_workspace(const void* q, int num_qo_heads,
                                               const void* pool, int64_t num_pages,
                                               int page_size, int num_kv_heads, int head_dim,
                                               int dtype, const int32_t* page_indptr,
                                               const int32_t* page_indices,
                                               const int32_t* last_page_len, int batch,
                                               float sm_scale, int num_partitions, void* out,
                                               float* lse, int32_t* error_word, void* stream);

/* The same three operations under the names used in the paged-attention literature. */
PKV_API pkv_status paged_kv_append(void* pool, int64_t num_pages, int page_size, int num_kv_heads,
                           int head_dim, int dtype,
                           const int32_t* page_indptr, const int32_t* page_indices,
                           const int32_t* last_page_len, int batch,
                           const void* k_new, const void* v_new, const int32_t* append_indptr,
                           int64_t nnz_new, int32_t* error_word, void* stream);
PKV_API pkv_status paged_decode_attention(const void* q, int num_qo_heads,
                                  const void* pool, int64_t num_pages, int page_size,
                                  int num_kv_heads, int head_dim, int dtype,
                                  const int32_t* page_indptr, const int32_t* page_indices,
                                  const int32_t* last_page_len, int batch,
                                  float sm_scale, int num_partitions,
                                  void* workspace, size_t workspace_bytes,
                                  void* out, float* lse, int32_t* error_word, void* stream);
PKV_API pkv_status merge_states(const float* v, const float* s, int64_t num_rows, int num_states,
                        int num_heads, int head_dim, void* v_out, int out_dtype,
                        float* s_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
