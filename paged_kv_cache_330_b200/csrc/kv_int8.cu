// INT8 KV cache: the quantising cache write and the block copy of an INT8 cache.
//
// The pages list KV-cache compression and INT8 among the tuning steps ("Nano-
// vLLM-Ascend: lightweight LLM inference framework for Ascend NPU", section
// 4.3) and name INT8 as the next throughput step once the accuracy of the
// attention scores is handled ("Ascend NPU LLM inference optimisation: the
// vLLM-Ascend approach", section 5).  They give no format; the one built here:
// every (token, KV head) row of D values is stored as D int8 codes with one
// fp32 scale, symmetric around zero, from the row's largest magnitude:
//
//   amax = max_d |x_d|;  inv = 127 / amax;  code_d = rint(x_d * inv) in [-127, 127];
//   scale = amax / 127   (all fp32, IEEE division and multiply, rounding half to even;
//                         amax == 0 gives zero codes and a zero scale)
//
// One scale per row means appending a token never re-quantises the rest of its
// block.  Codes use the 16-bit caches' layout [num_blocks][block_size][Hkv][D]
// (one byte per element); scales are [num_blocks][Hkv][block_size] fp32, so the
// 16 scales of one head over a 16-token chunk are one contiguous 64-byte run
// that a bulk copy can fetch.
//
// The write: one warp per (token, KV head) row.  Each lane holds D/32 values;
// the row's amax comes from warp shuffles (max is exact), then every lane
// forms its codes with the same fp32 steps and stores them as one 4-byte (D
// 128) or 2-byte (D 64) word, so a warp writes the row's D bytes in one
// coalesced store; lane 0 writes the scale.

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_int8)

namespace {

using namespace pa;

__device__ __forceinline__ int quant_code(float x, float inv) {
  const int c = __float2int_rn(__fmul_rn(x, inv));  // fp32 product, then round half to even
  return c < -127 ? -127 : (c > 127 ? 127 : c);
}

// Quantise one D-value row held by a warp (EPL values per lane) and store codes and scale.
template <int DT, int D>
__device__ __forceinline__ void quant_row(const void* src_row, int8_t* dst_codes, float* dst_scale, int lane) {
  constexpr int EPL = D / 32;
  float x[EPL];
  if constexpr (EPL == 4) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(src_row) + lane);
    const float2 a = Elt<DT>::to_f2(u.x), b = Elt<DT>::to_f2(u.y);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    const float2 a = Elt<DT>::to_f2(__ldg(reinterpret_cast<const uint32_t*>(src_row) + lane));
    x[0] = a.x; x[1] = a.y;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) packed |= (uint32_t)(quant_code(x[i], inv) & 0xff) << (8 * i);
  if constexpr (EPL == 4)
    reinterpret_cast<uint32_t*>(dst_codes)[lane] = packed;
  else
    reinterpret_cast<uint16_t*>(dst_codes)[lane] = (uint16_t)packed;
  if (lane == 0) *dst_scale = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
}

template <int DT, int D>
__global__ void __launch_bounds__(256) write_kv_int8_kernel(const void* __restrict__ k, const void* __restrict__ v,
                                                            const int64_t* __restrict__ slot_mapping, int num_tokens,
                                                            int hkv, int block_size, int64_t num_slots,
                                                            int8_t* __restrict__ kq, int8_t* __restrict__ vq,
                                                            float* __restrict__ ks, float* __restrict__ vs) {
  // a decode launched after this may start its set-up now; it waits for this grid before reading the cache
  asm volatile("griddepcontrol.launch_dependents;");
  // launched programmatically itself: wait for the preceding grid before reading inputs or writing slots
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t items = (int64_t)num_tokens * hkv;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t it = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); it < items; it += warps) {
    const int64_t t = it / hkv;
    const int h = (int)(it - t * hkv);
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {  // broken caller invariant: record, do not write
      if (lane == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
      continue;
    }
    const int64_t blk = slot / block_size;
    const int row = (int)(slot - blk * block_size);
    const size_t src_off = (size_t)it * D * 2;                 // [t][h][D] 16-bit
    const size_t code_off = ((size_t)slot * hkv + h) * D;      // [slot][h][D] int8
    const size_t scale_off = ((size_t)blk * hkv + h) * block_size + row;
    quant_row<DT, D>(reinterpret_cast<const uint8_t*>(k) + src_off, kq + code_off, ks + scale_off, lane);
    quant_row<DT, D>(reinterpret_cast<const uint8_t*>(v) + src_off, vq + code_off, vs + scale_off, lane);
  }
}

// One CTA row per pair: copies block src -> dst of the codes (code_vecs 16-byte vectors per block) and of
// the scales (scale_vecs per block) of both caches.
__global__ void __launch_bounds__(256) copy_blocks_int8_kernel(const int32_t* __restrict__ pairs, int num_pairs,
                                                               int64_t code_vecs, int64_t scale_vecs, int num_blocks,
                                                               uint4* __restrict__ kq, uint4* __restrict__ vq,
                                                               uint4* __restrict__ ks, uint4* __restrict__ vs) {
  const int p = blockIdx.y;
  if (p >= num_pairs) return;
  const int32_t src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.x == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    return;
  }
  const int64_t per = code_vecs + scale_vecs;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < per; i += (int64_t)gridDim.x * blockDim.x) {
    if (i < code_vecs) {
      st_v4(kq + dst * code_vecs + i, ld_nc_v4(kq + src * code_vecs + i));
      st_v4(vq + dst * code_vecs + i, ld_nc_v4(vq + src * code_vecs + i));
    } else {
      const int64_t j = i - code_vecs;
      st_v4(ks + dst * scale_vecs + j, ld_nc_v4(ks + src * scale_vecs + j));
      st_v4(vs + dst * scale_vecs + j, ld_nc_v4(vs + src * scale_vecs + j));
    }
  }
}

int check_int8_cache(const void* kq, const void* vq, const void* ks, const void* vs, int num_blocks, int block_size,
                     int num_kv_heads, int head_dim) {
  if (!kq || !vq || !ks || !vs || num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0) return PA_ERR_INVALID;
  if (!valid_block_size(block_size) || !valid_head_dim(head_dim)) return PA_ERR_UNSUPPORTED;
  if (!aligned16(kq) || !aligned16(vq) || !aligned16(ks) || !aligned16(vs)) return PA_ERR_ALIGN;
  return PA_OK;
}

}  // namespace

extern "C" int pa_write_kv_int8(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens,
                                void* k_codes, void* v_codes, float* k_scales, float* v_scales, int num_blocks,
                                int block_size, int num_kv_heads, int head_dim, int dtype, void* stream) {
  int s = check_int8_cache(k_codes, v_codes, k_scales, v_scales, num_blocks, block_size, num_kv_heads, head_dim);
  if (s != PA_OK) return s;
  if (!valid_dtype(dtype)) return PA_ERR_UNSUPPORTED;
  if (num_tokens < 0) return PA_ERR_INVALID;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u)) return PA_ERR_ALIGN;
  const int64_t items = (int64_t)num_tokens * num_kv_heads;
  int64_t blocks = (items + 7) / 8;  // 8 warps per CTA, one row per warp
  const int64_t cap = (int64_t)sm_count() * 16;
  if (blocks > cap) blocks = cap;
  const int64_t slots = (int64_t)num_blocks * block_size;
  auto* kq = reinterpret_cast<int8_t*>(k_codes);
  auto* vq = reinterpret_cast<int8_t*>(v_codes);
  cudaStream_t st = (cudaStream_t)stream;
  const unsigned g = (unsigned)blocks;
  auto kern = dtype == PA_BF16 ? (head_dim == 128 ? write_kv_int8_kernel<PA_BF16, 128> : write_kv_int8_kernel<PA_BF16, 64>)
                               : (head_dim == 128 ? write_kv_int8_kernel<PA_F16, 128> : write_kv_int8_kernel<PA_F16, 64>);
  return launch_programmatic(kern, dim3(g), dim3(256), 0, st, k, v, slot_mapping, num_tokens, num_kv_heads, block_size,
                             slots, kq, vq, k_scales, v_scales);
}

extern "C" int pa_copy_blocks_int8(const int32_t* pairs, int num_pairs, void* k_codes, void* v_codes, float* k_scales,
                                   float* v_scales, int num_blocks, int block_size, int num_kv_heads, int head_dim,
                                   void* stream) {
  int s = check_int8_cache(k_codes, v_codes, k_scales, v_scales, num_blocks, block_size, num_kv_heads, head_dim);
  if (s != PA_OK) return s;
  if (num_pairs < 0) return PA_ERR_INVALID;
  if (num_pairs == 0) return PA_OK;
  if (!pairs || num_pairs > 65535) return PA_ERR_INVALID;
  if (reinterpret_cast<uintptr_t>(pairs) & 3u) return PA_ERR_ALIGN;
  const int64_t code_vecs = (int64_t)block_size * num_kv_heads * head_dim / 16;
  const int64_t scale_vecs = (int64_t)num_kv_heads * block_size * 4 / 16;
  int gx = (int)((code_vecs + scale_vecs + 255) / 256);
  if (gx > 64) gx = 64;
  dim3 grid(gx, num_pairs);
  copy_blocks_int8_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(pairs, num_pairs, code_vecs, scale_vecs, num_blocks,
                                                                  (uint4*)k_codes, (uint4*)v_codes, (uint4*)k_scales,
                                                                  (uint4*)v_scales);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
