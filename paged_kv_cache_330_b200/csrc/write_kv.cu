// KV write: scatter the K/V rows of new tokens into their cache slots.
//
// Layout from the Block structure of "Nano-vLLM-Ascend: lightweight LLM
// inference framework for Ascend NPU", section 2.1 (per block
// [block_size, num_heads, head_dim], here stacked into one pool
// [num_blocks][block_size][Hkv][D]); the write is the "fill into fixed-size
// blocks" step of the PagedAttention operator on "Ascend NPU LLM inference
// optimisation: the vLLM-Ascend approach", section 2.2.
//
// A slot s addresses cache row s (block s / bs, row s % bs), and one row is
// Hkv*D contiguous elements, so a token's K (or V) is one contiguous run of
// Hkv*D*2 bytes at both ends.  Each thread moves one 16-byte vector; adjacent
// threads move adjacent vectors of the same token, so every warp reads and
// writes whole 512-byte runs (coalesced, full sectors).  The copy is bitwise.

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_write_kv)

namespace {

// vecs_per_row = Hkv*D*2/16.  Grid-stride over num_tokens * vecs_per_row
// vectors; each thread handles the same vector index of K and of V.
__global__ void __launch_bounds__(256) write_kv_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                       const int64_t* __restrict__ slot_mapping, int64_t total_vecs,
                                                       int vecs_per_row, int64_t num_slots, uint4* __restrict__ kc,
                                                       uint4* __restrict__ vc) {
  // a decode launched after this may start its set-up now; it waits for this grid to complete
  // before it reads the cache (programmatic dependent launch)
  asm volatile("griddepcontrol.launch_dependents;");
  // this grid may itself have started early (launched programmatically behind a decode that is still
  // reading the cache): wait for the preceding grid before reading inputs or writing slots
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total_vecs;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / vecs_per_row;
    const int c = (int)(i - t * vecs_per_row);
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {  // broken caller invariant: record, do not write
      PA_RECORD_ERROR(PA_ERRBIT_INDEX);
      continue;
    }
    const uint4 kk = pa::ld_nc_v4(k + i);
    const uint4 vv = pa::ld_nc_v4(v + i);
    pa::st_v4(kc + slot * vecs_per_row + c, kk);
    pa::st_v4(vc + slot * vecs_per_row + c, vv);
  }
}

// One CTA per (pair, 16-byte vector chunk): copies block src -> dst of both caches.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const int32_t* __restrict__ pairs, int num_pairs,
                                                          int64_t vecs_per_block, int num_blocks,
                                                          uint4* __restrict__ kc, uint4* __restrict__ vc) {
  const int p = blockIdx.y;
  if (p >= num_pairs) return;
  const int32_t src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    return;
  }
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < vecs_per_block;
       i += (int64_t)gridDim.x * blockDim.x) {
    pa::st_v4(kc + dst * vecs_per_block + i, pa::ld_nc_v4(kc + src * vecs_per_block + i));
    pa::st_v4(vc + dst * vecs_per_block + i, pa::ld_nc_v4(vc + src * vecs_per_block + i));
  }
}

int check_cache_args(const void* k_cache, const void* v_cache, int num_blocks, int block_size, int num_kv_heads,
                     int head_dim, int dtype) {
  if (!k_cache || !v_cache || num_blocks < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return PA_ERR_INVALID;
  if (!pa::valid_dtype(dtype)) return PA_ERR_UNSUPPORTED;
  if (!pa::valid_block_size(block_size) || (head_dim * 2) % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (!pa::aligned16(k_cache) || !pa::aligned16(v_cache)) return PA_ERR_ALIGN;
  return PA_OK;
}

}  // namespace

extern "C" int pa_write_kv(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens, void* k_cache,
                           void* v_cache, int num_blocks, int block_size, int num_kv_heads, int head_dim, int dtype,
                           void* stream) {
  int s = check_cache_args(k_cache, v_cache, num_blocks, block_size, num_kv_heads, head_dim, dtype);
  if (s != PA_OK) return s;
  if (num_tokens < 0) return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping) return PA_ERR_INVALID;
  if (!pa::aligned16(k) || !pa::aligned16(v) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)) return PA_ERR_ALIGN;
  const int vecs_per_row = num_kv_heads * head_dim * 2 / 16;
  const int64_t total = (int64_t)num_tokens * vecs_per_row;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = (int64_t)pa::sm_count() * 8;
  if (blocks > cap) blocks = cap;
  return pa::launch_programmatic(write_kv_kernel, dim3((unsigned)blocks), dim3(threads), 0, (cudaStream_t)stream,
                                 (const uint4*)k, (const uint4*)v, slot_mapping, total, vecs_per_row,
                                 (int64_t)num_blocks * block_size, (uint4*)k_cache, (uint4*)v_cache);
}

extern "C" int pa_copy_blocks(const int32_t* pairs, int num_pairs, void* k_cache, void* v_cache, int num_blocks,
                              int block_size, int num_kv_heads, int head_dim, int dtype, void* stream) {
  int s = check_cache_args(k_cache, v_cache, num_blocks, block_size, num_kv_heads, head_dim, dtype);
  if (s != PA_OK) return s;
  if (num_pairs < 0) return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!pairs || num_pairs > 65535) return PA_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(pairs) & 3u) return PA_ERR_ALIGN;
  const int64_t vecs_per_block = (int64_t)block_size * num_kv_heads * head_dim * 2 / 16;
  int gx = (int)((vecs_per_block + 255) / 256);
  if (gx > 64) gx = 64;
  dim3 grid(gx, num_pairs);
  copy_blocks_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(pairs, num_pairs, vecs_per_block, num_blocks,
                                                             (uint4*)k_cache, (uint4*)v_cache);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
