// Decode with each sequence's context split across devices: the host-side split rule and the merge of
// the devices' intermediate results.
//
// Page "In-depth analysis of vllm-ascend: LLM inference architecture on Ascend hardware", sections 1.1
// and 3.1 (DCP): the KV cache of a long sequence is spread over several devices, each device attends
// over the part it holds, the intermediate results of all devices are gathered (AllGather) and combined.
// The pages fix neither the split nor the combination.  Here:
//
//   * split: logical block j of every sequence lives on rank j mod W (block-interleaved), so every
//     rank's share differs by at most one block and an appended token goes to rank (pos / bs) mod W;
//     within a rank, logical block j is local block j / W, so every local block but the last is full
//     and a rank's blocks form an ordinary paged sequence of local_len tokens;
//   * intermediate result: the rank's attention output normalised over its own tokens (pa_decode_lse)
//     and the log-sum-exp of its scores;
//   * merge: out = sum_r exp(lse_r - M) o_r / sum_r exp(lse_r - M), M = max_r lse_r (the softmax over
//     all tokens), one warp per (sequence, head) row.

#include "common.cuh"
#include "host_common.h"

namespace {

using namespace pa;

constexpr float kLog2eF = 1.4426950408889634f;

// parts: [P][rows][D] 16-bit; lses: [P][rows] fp32; out: [rows][D].
template <int DT, int D>
__global__ void __launch_bounds__(256) merge_states_kernel(const uint8_t* __restrict__ parts,
                                                           const float* __restrict__ lses, int P, int64_t rows,
                                                           uint8_t* __restrict__ out) {
  using T = typename Elt<DT>::T;
  constexpr int CH = D / 4;  // 4-element (8-byte) chunks per row
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    float M = -INFINITY;
    for (int p = lane; p < P; p += 32) M = fmaxf(M, __ldg(lses + (size_t)p * rows + r));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    uint2* dst = reinterpret_cast<uint2*>(out + (size_t)r * D * sizeof(T));
    if (M == -INFINITY) {  // no part holds a token of this row
      if (lane < CH) dst[lane] = make_uint2(0u, 0u);
      continue;
    }
    float den = 0.f;
    for (int p = lane; p < P; p += 32) den += fast_exp2((__ldg(lses + (size_t)p * rows + r) - M) * kLog2eF);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = 1.f / den;
    if (lane < CH) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int p = 0; p < P; ++p) {
        const float w = fast_exp2((__ldg(lses + (size_t)p * rows + r) - M) * kLog2eF) * inv;
        if (w == 0.f) continue;  // an empty part (lse -inf) contributes nothing, whatever its bytes
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(parts + ((size_t)p * rows + r) * D * sizeof(T)) + lane);
        const float2 x = Elt<DT>::to_f2(u.x), y = Elt<DT>::to_f2(u.y);
        a0 = fmaf(w, x.x, a0); a1 = fmaf(w, x.y, a1);
        a2 = fmaf(w, y.x, a2); a3 = fmaf(w, y.y, a3);
      }
      dst[lane] = make_uint2(Elt<DT>::from_f2(a0, a1), Elt<DT>::from_f2(a2, a3));
    }
  }
}

int64_t local_len_of(int64_t L, int bs, int world, int rank) {
  if (L <= 0) return 0;
  const int64_t nfull = L / bs, rem = L % bs;
  const int64_t full_here = nfull > rank ? (nfull - 1 - rank) / world + 1 : 0;
  return full_here * bs + ((rem > 0 && nfull % world == rank) ? rem : 0);
}

}  // namespace

extern "C" int pa_dcp_owner(int64_t position, int block_size, int world) {
  if (position < 0 || block_size <= 0 || world <= 0) return PA_ERR_INVALID;
  return (int)((position / block_size) % world);
}

extern "C" int64_t pa_dcp_local_position(int64_t position, int block_size, int world) {
  if (position < 0 || block_size <= 0 || world <= 0) return PA_ERR_INVALID;
  const int64_t j = position / block_size;
  return (j / world) * block_size + position % block_size;
}

extern "C" int pa_dcp_local_lens(const int32_t* context_lens, int batch, int block_size, int world, int rank,
                                 int32_t* local_lens_out) {
  if (batch < 0 || block_size <= 0 || world <= 0 || rank < 0 || rank >= world) return PA_ERR_INVALID;
  if (batch > 0 && (!context_lens || !local_lens_out)) return PA_ERR_INVALID;
  for (int b = 0; b < batch; ++b) {
    if (context_lens[b] < 0) return PA_ERR_INVALID;
  }
  for (int b = 0; b < batch; ++b) local_lens_out[b] = (int32_t)local_len_of(context_lens[b], block_size, world, rank);
  return PA_OK;
}

extern "C" int pa_merge_attn_states(const void* parts, const float* lses, int num_parts, int batch, int num_heads,
                                    int head_dim, int dtype, void* out, void* stream) {
  if (num_parts < 0 || batch < 0 || num_heads < 0) return PA_ERR_INVALID;
  if (!valid_dtype(dtype) || !valid_head_dim(head_dim)) return PA_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)batch * num_heads;
  if (rows == 0) return PA_OK;
  if (num_parts == 0 || !parts || !lses || !out) return PA_ERR_INVALID;
  if (!aligned16(parts) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lses) & 3u)) return PA_ERR_ALIGN;
  int64_t blocks = (rows + 7) / 8;  // 8 warps per CTA, one row per warp
  const int64_t cap = (int64_t)sm_count() * 16;
  if (blocks > cap) blocks = cap;
  const auto* pp = reinterpret_cast<const uint8_t*>(parts);
  auto* op = reinterpret_cast<uint8_t*>(out);
  cudaStream_t st = (cudaStream_t)stream;
  const unsigned g = (unsigned)blocks;
  if (dtype == PA_BF16) {
    if (head_dim == 128) merge_states_kernel<PA_BF16, 128><<<g, 256, 0, st>>>(pp, lses, num_parts, rows, op);
    else merge_states_kernel<PA_BF16, 64><<<g, 256, 0, st>>>(pp, lses, num_parts, rows, op);
  } else {
    if (head_dim == 128) merge_states_kernel<PA_F16, 128><<<g, 256, 0, st>>>(pp, lses, num_parts, rows, op);
    else merge_states_kernel<PA_F16, 64><<<g, 256, 0, st>>>(pp, lses, num_parts, rows, op);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
