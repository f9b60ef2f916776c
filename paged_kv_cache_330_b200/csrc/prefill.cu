// Chunked prefill over the paged cache (host validation; kernel follows).
#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_prefill)

extern "C" int pa_prefill_chunk(const void* q, const int32_t* query_start_loc, int total_q_tokens, int max_chunk_len,
                                const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, int dtype,
                                void* out, void* stream) {
  if (batch < 0 || total_q_tokens < 0 || max_chunk_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      num_blocks < 0 || max_blocks_per_seq < 0)
    return PA_ERR_INVALID;
  if (!pa::valid_dtype(dtype) || head_dim != 128 || !pa::valid_block_size(block_size)) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads) return PA_ERR_INVALID;
  if (!pa::valid_group(num_q_heads / num_kv_heads)) return PA_ERR_UNSUPPORTED;
  if (batch == 0 || total_q_tokens == 0) return PA_OK;
  if (!q || !query_start_loc || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID;
  if (!pa::aligned16(q) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache) || !pa::aligned16(out))
    return PA_ERR_ALIGN;
  (void)scale; (void)stream;
  return PA_ERR_UNSUPPORTED;
}
