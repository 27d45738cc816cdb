"""paged_kv_cache_479_b200 -- batched decode attention over a paged KV cache on B200.

A thin Python binding of libpkv (include/pkv.h).  Every function marshals
torch tensors into the C ABI (data pointers, sizes, the current CUDA
stream) and calls the library; all arithmetic runs in the library's CUDA
kernels.  There is no CPU fallback: if libpkv.so is missing or cannot be
loaded, importing the binding's functions raises.

Functions (C names in parentheses):
  paged_kv_append        (pkv_append)          scatter new tokens into pages
  paged_decode_attention (pkv_decode)          decode attention + split-KV merge
  merge_states           (pkv_merge_states)    merge (o, lse) states
  decode_workspace_bytes (pkv_decode_workspace_bytes)
  default_partitions     (pkv_default_partitions)
  read_error_word        (pkv_read_error_word)
  set_wait_limit_ns      (pkv_set_wait_limit_ns)  time limit of the decode's internal waits
  check_table            (pkv_check_table)     host-side table check
  plan_segments          (pkv_plan_segments)   host mirror of the split-KV partition
  decode_static_workspace (pkv_decode_static_workspace)  decode on the library's own scratch
  cascade_decode         (pkv_cascade_decode)  decode for a batch sharing one prefix
  paged_decode_attention_ex / paged_kv_append_ex (pkv_decode_ex / pkv_append_ex)
                         NHD pools and dense (vLLM-style) block tables
  paged_decode_append    (pkv_decode_append)   append + decode of a step in one launch
  paged_decode_attention_fp8 / paged_kv_append_fp8 (pkv_decode_fp8 / pkv_append_fp8)
                         the 8-bit (FP8 E4M3 / E5M2) KV cache with per-tensor K / V scales
  append_attention       (pkv_append_attention)  a chunk of query tokens per request,
                         causal over its cache (chunked prefill, speculative tokens)
  append_attention_plan  (pkv_append_attention_plan)  its host-side row-block plan
  append_attention_short (pkv_append_attention_short)  the same for chunks of at most
                         16 / G tokens (speculative verification) on the decode schedule
"""
from ._binding import (  # noqa: F401
    BF16,
    append_attention,
    append_attention_plan,
    append_attention_short,
    append_attention_short_workspace_bytes,
    append_attention_workspace_bytes,
    F16,
    F32,
    FP8_E4M3,
    FP8_E5M2,
    PkvError,
    PoolDesc,
    TableDesc,
    block_table,
    cascade_decode,
    cascade_workspace_bytes,
    check_table,
    csr_table,
    decode_static_workspace,
    decode_workspace_bytes,
    default_partitions,
    lib,
    merge_states,
    paged_decode_attention,
    paged_decode_append,
    paged_decode_attention_ex,
    paged_decode_attention_fp8,
    paged_kv_append,
    paged_kv_append_ex,
    set_wait_limit_ns,
    paged_kv_append_fp8,
    pool_desc,
    plan_segments,
    read_error_word,
    DEVERR_APPEND,
    DEVERR_CONTEXT_LEN,
    DEVERR_INDPTR,
    DEVERR_LAST_LEN,
    DEVERR_PAGE_ID,
    DEVERR_TIMEOUT,
    LAYOUT_HND,
    LAYOUT_NHD,
    TABLE_BLOCK,
    TABLE_CSR,
)

pkv_append = paged_kv_append
pkv_decode = paged_decode_attention
pkv_decode_static_workspace = decode_static_workspace
pkv_merge_states = merge_states
pkv_cascade_decode = cascade_decode
pkv_decode_ex = paged_decode_attention_ex
pkv_decode_append = paged_decode_append
pkv_append_ex = paged_kv_append_ex
pkv_decode_fp8 = paged_decode_attention_fp8
pkv_append_attention = append_attention
pkv_append_attention_short = append_attention_short
pkv_append_fp8 = paged_kv_append_fp8
