// Rotary position embedding of new tokens' queries and keys, fused with the
// KV write.
//
// The rotation is the rotary multiply of "Nano-vLLM-Ascend: lightweight LLM
// inference framework for Ascend NPU", section 5.1 (x turned by per-position
// cos/sin tables; the backward is the same operator with sin negated), in the
// rotate-half pairing: element i of a head turns with element i + D/2 by the
// angle of table column i.  Section 3.1 of the same page is where each model
// brings its own rotary embedding; it runs right before the cache write of
// "Ascend NPU LLM inference optimisation: the vLLM-Ascend approach",
// section 2.2, so the two are one pass here: a key row is read once, turned
// in registers and stored straight into its cache slot, and V moves bitwise.
//
// Work items, per token (all 16-byte vectors):
//   [0, Hq*D/16)            rotate 8 pairs of one query head   (q -> q_out)
//   [.., + Hkv*D/16)        rotate 8 pairs of one key head     (k -> k_cache)
//   [.., + Hkv*D/8)         copy one 16-byte vector of V       (v -> v_cache)
// Adjacent items touch adjacent 16-byte vectors of the same head, so a warp
// reads and writes whole runs of the first and second half of each head.
// The fp32 cos/sin row of a position is read by every head of the token and
// stays in L1.  HBM traffic is the algorithmic minimum: q, k, v read once,
// q_out and the cache rows written once.

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_rope)

namespace {

struct RopeArgs {
  const uint4* q;        // [T][Hq][D] (may alias q_out: plain loads, never the read-only path)
  uint4* q_out;          // [T][Hq][D]
  const uint4* k;        // [T][Hkv][D]
  const uint4* v;        // [T][Hkv][D]
  const int64_t* positions;
  const float4* cos_t;   // [max_position][D/2]
  const float4* sin_t;
  const int64_t* slots;
  uint4* kc;             // [num_slots][Hkv][D]
  uint4* vc;
  int64_t num_slots;
  int64_t max_position;
  int total;             // num_tokens * items per token
  int hq, hkv;
  int rot;               // 16-byte vectors in half a head (D/16) = rotation items per head
};

__device__ __forceinline__ uint4 ld_plain_v4(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Turns the 8 pairs (x1[m], x2[m]) by the angles whose cos/sin are c[m], s[m].
template <int DT>
__device__ __forceinline__ void rotate8(uint4& x1, uint4& x2, const float* c, const float* s) {
  using E = pa::Elt<DT>;
  uint32_t* a = reinterpret_cast<uint32_t*>(&x1);
  uint32_t* b = reinterpret_cast<uint32_t*>(&x2);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float2 u = E::to_f2(a[w]), v = E::to_f2(b[w]);
    const float c0 = c[2 * w], c1 = c[2 * w + 1], s0 = s[2 * w], s1 = s[2 * w + 1];
    a[w] = E::from_f2(fmaf(u.x, c0, -v.x * s0), fmaf(u.y, c1, -v.y * s1));
    b[w] = E::from_f2(fmaf(v.x, c0, u.x * s0), fmaf(v.y, c1, u.y * s1));
  }
}

template <int DT>
__global__ void __launch_bounds__(256) rope_write_kv_kernel(const RopeArgs a) {
  // a decode kernel launched after this one may start its set-up now; it waits for this grid to
  // complete before it reads q_out or the cache (programmatic dependent launch)
  asm volatile("griddepcontrol.launch_dependents;");
  // launched programmatically itself: wait for the preceding grid before reading inputs or writing
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int rot = a.rot, vec = 2 * rot;  // 16-byte vectors per half head / per head
  const int rq = a.hq * rot, rk = a.hkv * rot;
  const int ipt = rq + rk + a.hkv * vec;
  for (int64_t ii = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; ii < a.total;
       ii += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)ii;  // a.total < 2^31
    const int t = i / ipt;
    const int c = i - t * ipt;
    const int64_t pos = __ldg(a.positions + t);
    if (pos < 0 || pos >= a.max_position) {  // broken caller invariant: record once per token, write nothing
      if (c == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
      continue;
    }
    int64_t slot = -1;
    if (c >= rq) {
      slot = __ldg(a.slots + t);
      if (slot < 0) continue;
      if (slot >= a.num_slots) {
        if (c == rq) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
        continue;
      }
    }
    if (c < rq + rk) {
      const bool isq = c < rq;
      const int cc = isq ? c : c - rq;
      const int h = cc / rot, r = cc - h * rot;
      uint4 x1, x2;
      if (isq) {
        const uint4* src = a.q + ((int64_t)t * a.hq + h) * vec;
        x1 = ld_plain_v4(src + r);
        x2 = ld_plain_v4(src + rot + r);
      } else {
        const uint4* src = a.k + ((int64_t)t * a.hkv + h) * vec;
        x1 = pa::ld_nc_v4(src + r);
        x2 = pa::ld_nc_v4(src + rot + r);
      }
      // table row pos, columns 8r .. 8r+7: two float4 of cos, two of sin
      const int64_t tb = pos * vec + 2 * r;
      const float4 c0 = __ldg(a.cos_t + tb), c1 = __ldg(a.cos_t + tb + 1);
      const float4 s0 = __ldg(a.sin_t + tb), s1 = __ldg(a.sin_t + tb + 1);
      const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      rotate8<DT>(x1, x2, cv, sv);
      uint4* dst = isq ? a.q_out + ((int64_t)t * a.hq + h) * vec : a.kc + (slot * a.hkv + h) * vec;
      pa::st_v4(dst + r, x1);
      pa::st_v4(dst + rot + r, x2);
    } else {
      const int vi = c - rq - rk;  // vector index within the token's V row
      pa::st_v4(a.vc + slot * (a.hkv * vec) + vi, pa::ld_nc_v4(a.v + (int64_t)t * a.hkv * vec + vi));
    }
  }
}

}  // namespace

extern "C" int pa_rope_write_kv(const void* q, void* q_out, const void* k, const void* v, const int64_t* positions,
                                const float* cos_table, const float* sin_table, int max_position,
                                const int64_t* slot_mapping, int num_tokens, int num_q_heads, void* k_cache,
                                void* v_cache, int num_blocks, int block_size, int num_kv_heads, int head_dim,
                                int dtype, void* stream) {
  if (num_tokens < 0 || num_blocks < 0 || block_size <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || max_position <= 0)
    return PA_ERR_INVALID;
  if (!pa::valid_dtype(dtype) || !pa::valid_block_size(block_size) || !pa::valid_head_dim(head_dim))
    return PA_ERR_UNSUPPORTED;
  if (!k_cache || !v_cache) return PA_ERR_INVALID;
  if (!pa::aligned16(k_cache) || !pa::aligned16(v_cache)) return PA_ERR_ALIGN;
  if (num_tokens == 0) return PA_OK;
  if (!q || !q_out || !k || !v || !positions || !cos_table || !sin_table || !slot_mapping) return PA_ERR_INVALID;
  if (!pa::aligned16(q) || !pa::aligned16(q_out) || !pa::aligned16(k) || !pa::aligned16(v) ||
      !pa::aligned16(cos_table) || !pa::aligned16(sin_table) || (reinterpret_cast<uintptr_t>(positions) & 7u) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_ALIGN;
  const int rot = head_dim / 16;
  const int64_t ipt = (int64_t)(num_q_heads + num_kv_heads) * rot + (int64_t)num_kv_heads * 2 * rot;
  const int64_t total = (int64_t)num_tokens * ipt;
  if (total > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  RopeArgs a;
  a.q = (const uint4*)q;
  a.q_out = (uint4*)q_out;
  a.k = (const uint4*)k;
  a.v = (const uint4*)v;
  a.positions = positions;
  a.cos_t = (const float4*)cos_table;
  a.sin_t = (const float4*)sin_table;
  a.slots = slot_mapping;
  a.kc = (uint4*)k_cache;
  a.vc = (uint4*)v_cache;
  a.num_slots = (int64_t)num_blocks * block_size;
  a.max_position = max_position;
  a.total = (int)total;
  a.hq = num_q_heads;
  a.hkv = num_kv_heads;
  a.rot = rot;
  // one resident wave: every CTA strides over the same number of items
  const int threads = 256;
  auto kern = dtype == PA_BF16 ? rope_write_kv_kernel<PA_BF16> : rope_write_kv_kernel<PA_F16>;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess || per_sm < 1)
    return PA_ERR_CUDA;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = (int64_t)pa::sm_count() * per_sm;
  if (blocks > cap) blocks = cap;
  return pa::launch_programmatic(kern, dim3((unsigned)blocks), dim3(threads), 0, (cudaStream_t)stream, a);
}
