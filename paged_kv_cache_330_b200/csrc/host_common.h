// Host-side helpers shared by the launch wrappers (internal, not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "paged_attn.h"

namespace pa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_dtype(int dt) { return dt == PA_F16 || dt == PA_BF16; }
inline bool valid_block_size(int bs) { return bs == 16 || bs == 32 || bs == 64 || bs == 128 || bs == 256; }
inline bool valid_head_dim(int d) { return d == 64 || d == 128; }
inline bool valid_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

// Encode a 2-D tiled tensor map over a row-major [rows][cols] matrix of 16-bit
// elements with a 128-byte swizzle: box = box_cols x box_rows elements
// (box_cols * 2 must be <= 128).  Returns PA_OK or PA_ERR_CUDA.
int encode_2d_sw128(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                    uint32_t box_cols, uint32_t box_rows);

// The same with the swizzle chosen by its span in bytes (128 or 64; box_cols * 2 must equal it) and the
// L2 fill granularity (256 or 128 bytes: a box row of 128 bytes takes 128, so that a fill does not bring
// in the neighbouring head's row).
int encode_2d_u16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_cols, uint32_t box_rows, uint32_t swizzle_bytes, uint32_t l2_fill_bytes = 256);

// Number of SMs of the current device (cached per device).
int sm_count();

// The cascade decode's shared-prefix pass on the CTA-pair tensor-core kernel (head_dim 128; prefill.cu).
int prefix_pass_pairs(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      int max_blocks_per_seq, int num_groups, const int32_t* group_start, const int32_t* seq_prefix,
                      int max_group_size, const float* lse_s, int num_q_heads, int num_kv_heads, int block_size,
                      int num_blocks, float scale, int dtype, void* out, cudaStream_t st);

// Launch with programmatic stream serialization: the kernel may start while the preceding kernel on the
// stream is still running (once that kernel signals griddepcontrol.launch_dependents or exits), so it
// must execute griddepcontrol.wait before it reads or writes memory the preceding kernel may touch.
template <typename... Params, typename... Args>
int launch_programmatic(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) return PA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
