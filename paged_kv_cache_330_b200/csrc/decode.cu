// Paged decode attention, split-K, for sm_100a.
//
// What it computes (page "Nano-vLLM-Ascend: lightweight LLM inference
// framework for Ascend NPU", section 2.2.1 attention = softmax(q k^T/sqrt(d)) v
// and section 2.1 block table; page "Ascend NPU LLM inference optimisation:
// the vLLM-Ascend approach", section 2.2 PagedAttention operator and
// section 3.1 fp32 softmax): for every sequence b and query head h,
//   out[b][h] = sum_t softmax_t(scale <q[b][h], K_b[t][h/G]>) V_b[t][h/G],
// where token t of sequence b lives in physical block block_tables[b][t/bs],
// row t%bs of the cache.
//
// Work split.  One CTA per (sequence b, KV head g, split s); a split is
// `split_len` consecutive tokens (a multiple of 64), so long contexts spread
// over many SMs (the single-device reading of the context-parallel split on
// "In-depth analysis of vllm-ascend", section 3.1).  All G query heads of the
// group share every K/V tile the CTA loads.
//
// Data movement.  One producer warp gathers 16-row K and V boxes through the
// block table with TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast)
// into an NSTAGES-deep shared-memory ring guarded by mbarriers (the pages'
// prefetch-depth / pipeline-stage lesson, vLLM-Ascend page section 2.2).
// NW consumer warps each take 32 tokens of every stage.
//
// Math.  fp32 scores in the log2 domain (scale*log2(e) folded into q),
// online softmax with fp32 running max and sum, fp32 accumulators.
//   * G <= 4: CUDA cores.  QK^T: lane = token, full dot product per lane;
//     row max/sum by warp shuffles; PV: lane = slice of head_dim.
//   * G >= 8: the FP32 pipe cannot keep up with HBM at 8 flop per KV byte,
//     so QK^T and PV use warp-level mma.m16n8k16 (bf16/f16 in, fp32 out) with
//     the G query heads as rows; softmax rows are reduced with quad shuffles.
// Each consumer warp keeps its own (max, sum, acc); the warps merge through
// shared memory at the end.  A sequence that fits one split writes `out`
// directly; otherwise the split writes fp32 (max, sum, acc) to the workspace
// and a reduce kernel merges splits by the log-sum-exp rule.

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_decode)

namespace {

using namespace pa;

constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
  const void* q;
  void* out;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_m;  // [B][Hq][max_splits]  running max (log2 domain)
  float* ws_l;  // [B][Hq][max_splits]  sum of exp2(x - m)
  float* ws_o;  // [B][Hq][max_splits][D] sum of exp2(x - m) * v
  int max_blocks_per_seq;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int split_len;
  int max_splits;
  float scale_log2;
};

template <int D, int G, int NW, int NSTAGES>
struct Layout {
  static constexpr int TOK = NW * 32;                 // tokens per stage
  static constexpr int HALVES = D / 64;               // 128-byte column boxes per row
  static constexpr int STAGE_BYTES = TOK * D * 2;     // K (or V) bytes per stage
  static constexpr int BOXES = TOK / 16;              // 16-row boxes per stage
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + NSTAGES * STAGE_BYTES;
  static constexpr int Q_OFF = V_OFF + NSTAGES * STAGE_BYTES;           // fp32 [G][D]
  static constexpr int P_OFF = Q_OFF + G * D * 4;                       // fp32 [NW][32][G]
  static constexpr int BT_OFF = P_OFF + NW * 32 * G * 4;                // int32 [BT_MAX]
  // merge area, fp32 [NW][G][D] then [NW][G][2]; aliases the stage buffers,
  // which are free once every consumer has passed the pipeline
  static constexpr int M_OFF = K_OFF;
  static constexpr int ML_OFF = M_OFF + NW * G * D * 4;
  static_assert(ML_OFF + NW * G * 2 * 4 <= Q_OFF, "merge area must fit in the stage buffers");
  static constexpr int BT_MAX = 512;                                    // block-table entries per split
  static constexpr int BAR_OFF = BT_OFF + BT_MAX * 4;                   // uint64 full[NSTAGES], empty[NSTAGES]
  static constexpr int BYTES = BAR_OFF + 2 * NSTAGES * 8;
  static constexpr int ALLOC = BYTES + 1024;                            // slack for 1024-byte alignment
};

// Address of element (row r, column d) inside a stage buffer laid out as
// [half][TOK rows][128 bytes] with the TMA 128-byte swizzle (16-byte chunk
// index XOR row%8).
template <int TOK>
__device__ __forceinline__ uint32_t swz_addr(uint32_t base, int r, int d) {
  const int half = d >> 6;
  const int chunk = (d >> 3) & 7;
  return base + half * (TOK * 128) + r * 128 + ((chunk ^ (r & 7)) << 4) + ((d & 7) << 1);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}

template <int DT>
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  if constexpr (DT == PA_BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ CUDA-core consumer (G <= 4)
template <int DT, int D, int G, int NW, int NSTAGES>
struct CoreConsumer {
  using LY = Layout<D, G, NW, NSTAGES>;
  static constexpr int DPL = D / 32;  // head_dim elements per lane in PV
  float m[G], l[G], o[G][DPL];

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int j = 0; j < DPL; ++j) o[h][j] = 0.f;
    }
  }

  // One 32-token tile: rows r0 .. r0+31 of the stage, nv of them valid.
  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, uint32_t qbase, uint32_t pbase, int r0,
                                       int nv, int lane) {
    // ---- scores: lane = token
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
    const int r = r0 + lane;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const uint4 kv = lds128(swz_addr<LY::TOK>(kbase, r, c * 8));
      const float2 k01 = Elt<DT>::to_f2(kv.x), k23 = Elt<DT>::to_f2(kv.y), k45 = Elt<DT>::to_f2(kv.z),
                   k67 = Elt<DT>::to_f2(kv.w);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint4 qa = lds128(qbase + (h * D + c * 8) * 4);
        const uint4 qb = lds128(qbase + (h * D + c * 8 + 4) * 4);
        float a = acc[h];
        a = fmaf(k01.x, __uint_as_float(qa.x), a);
        a = fmaf(k01.y, __uint_as_float(qa.y), a);
        a = fmaf(k23.x, __uint_as_float(qa.z), a);
        a = fmaf(k23.y, __uint_as_float(qa.w), a);
        a = fmaf(k45.x, __uint_as_float(qb.x), a);
        a = fmaf(k45.y, __uint_as_float(qb.y), a);
        a = fmaf(k67.x, __uint_as_float(qb.z), a);
        a = fmaf(k67.y, __uint_as_float(qb.w), a);
        acc[h] = a;
      }
    }
    // ---- online softmax (log2 domain), fp32
    float p[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float s = lane < nv ? acc[h] : -INFINITY;
      const float mn = fmaxf(m[h], warp_max(s));
      const float alpha = fast_exp2(m[h] - mn);
      p[h] = fast_exp2(s - mn);
      l[h] = l[h] * alpha + warp_sum(p[h]);
      m[h] = mn;
#pragma unroll
      for (int j = 0; j < DPL; ++j) o[h][j] *= alpha;
    }
    // ---- p to shared memory, [token][G]
    const uint32_t pa = pbase + lane * G * 4;
    if constexpr (G == 1) {
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(pa), "f"(p[0]) : "memory");
    } else if constexpr (G == 2) {
      asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(pa), "f"(p[0]), "f"(p[1]) : "memory");
    } else {
      asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(pa), "f"(p[0]), "f"(p[1]), "f"(p[2]), "f"(p[3])
                   : "memory");
    }
    __syncwarp();
    // ---- PV: lane = DPL consecutive columns
    const int d0 = lane * DPL;
    for (int t = 0; t < nv; ++t) {
      float v[DPL];
      const uint32_t va = swz_addr<LY::TOK>(vbase, r0 + t, d0);
      if constexpr (DPL == 4) {
        const uint2 u = lds64(va);
        const float2 a = Elt<DT>::to_f2(u.x), b = Elt<DT>::to_f2(u.y);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
      } else {
        const float2 a = Elt<DT>::to_f2(lds32(va));
        v[0] = a.x; v[1] = a.y;
      }
      float pt[G];
      const uint32_t pr = pbase + t * G * 4;
      if constexpr (G == 1) {
        pt[0] = __uint_as_float(lds32(pr));
      } else if constexpr (G == 2) {
        const uint2 u = lds64(pr);
        pt[0] = __uint_as_float(u.x); pt[1] = __uint_as_float(u.y);
      } else {
        const uint4 u = lds128(pr);
        pt[0] = __uint_as_float(u.x); pt[1] = __uint_as_float(u.y);
        pt[2] = __uint_as_float(u.z); pt[3] = __uint_as_float(u.w);
      }
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int j = 0; j < DPL; ++j) o[h][j] = fmaf(pt[h], v[j], o[h][j]);
    }
    __syncwarp();
  }

  // Write this warp's (m, l, o) to the merge area: o as [G][D], ml as [G][2].
  __device__ __forceinline__ void stash(float* merge_o, float* merge_ml, int lane) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int j = 0; j < DPL; ++j) merge_o[h * D + lane * DPL + j] = o[h][j];
      if (lane == 0) {
        merge_ml[h * 2] = m[h];
        merge_ml[h * 2 + 1] = l[h];
      }
    }
  }
};

// ------------------------------------------------------------------ tensor-core consumer (G >= 8)
template <int DT, int D, int G, int NW, int NSTAGES>
struct MmaConsumer {
  using LY = Layout<D, G, NW, NSTAGES>;
  static constexpr int KS = D / 16;   // k-steps of QK^T
  static constexpr int ND = D / 8;    // n-tiles of PV
  uint32_t qa[KS][4];                 // A fragments of q (rows = heads, padded to 16)
  float o[ND][4];                     // rows lane/4 and lane/4+8, columns of an n-tile
  float m[2], l[2];                   // per row owned by this thread (lane/4, lane/4+8); l is a partial sum

  __device__ __forceinline__ void load_q(const typename Elt<DT>::T* qg, int lane) {
    const int r0 = lane >> 2, r1 = r0 + 8;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qg);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c = ks * 16 + (lane & 3) * 2;
      qa[ks][0] = r0 < G ? __ldg(q32 + (r0 * D + c) / 2) : 0u;
      qa[ks][1] = r1 < G ? __ldg(q32 + (r1 * D + c) / 2) : 0u;
      qa[ks][2] = r0 < G ? __ldg(q32 + (r0 * D + c + 8) / 2) : 0u;
      qa[ks][3] = r1 < G ? __ldg(q32 + (r1 * D + c + 8) / 2) : 0u;
    }
  }

  __device__ __forceinline__ void init() {
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  }

  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, float scale_log2, int r0, int nv, int lane) {
    // ---- S = Q K^T : 16 head-rows x 32 tokens (4 n-tiles)
    float s[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int pair = 0; pair < 2; ++pair) {
        const int tok = r0 + pair * 16 + ((lane >> 4) << 3) + (lane & 7);
        const int d = ks * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(swz_addr<LY::TOK>(kbase, tok, d), b0, b1, b2, b3);
        mma16816<DT>(s[pair * 2], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
        mma16816<DT>(s[pair * 2 + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
      }
    }
    // ---- mask, scale, row max (rows lane/4 and lane/4+8)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int t = n * 8 + (lane & 3) * 2;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = (t + e) < nv;
        s[n][e] = ok ? s[n][e] * scale_log2 : -INFINITY;
        s[n][2 + e] = ok ? s[n][2 + e] * scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[n][e]);
        mx1 = fmaxf(mx1, s[n][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float al0 = fast_exp2(m[0] - mn0), al1 = fast_exp2(m[1] - mn1);
    m[0] = mn0;
    m[1] = mn1;
    float ls0 = 0.f, ls1 = 0.f;
    uint32_t pa[2][4];  // A fragments of P for the two 16-token k-steps
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const float p0 = fast_exp2(s[n][0] - mn0), p1 = fast_exp2(s[n][1] - mn0);
      const float p2 = fast_exp2(s[n][2] - mn1), p3 = fast_exp2(s[n][3] - mn1);
      ls0 += p0 + p1;
      ls1 += p2 + p3;
      pa[n >> 1][(n & 1) * 2 + 0] = Elt<DT>::from_f2(p0, p1);
      pa[n >> 1][(n & 1) * 2 + 1] = Elt<DT>::from_f2(p2, p3);
    }
    l[0] = l[0] * al0 + ls0;
    l[1] = l[1] * al1 + ls1;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      o[n][0] *= al0; o[n][1] *= al0;
      o[n][2] *= al1; o[n][3] *= al1;
    }
    // ---- O += P V : k = tokens (2 steps of 16), n = head_dim (ND tiles of 8)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j * 16 >= nv) break;
#pragma unroll
      for (int dp = 0; dp < ND / 2; ++dp) {
        const int tok = r0 + j * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int d = dp * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(swz_addr<LY::TOK>(vbase, tok, d), b0, b1, b2, b3);
        if (nv < 32) {  // zero V of tokens past the end (their bytes may be anything, even NaN)
          const int tb = j * 16 + (lane & 3) * 2;
          const uint32_t lo0 = (tb < nv ? 0xffffu : 0u) | (tb + 1 < nv ? 0xffff0000u : 0u);
          const uint32_t lo1 = (tb + 8 < nv ? 0xffffu : 0u) | (tb + 9 < nv ? 0xffff0000u : 0u);
          b0 &= lo0; b2 &= lo0;
          b1 &= lo1; b3 &= lo1;
        }
        mma16816<DT>(o[dp * 2], pa[j][0], pa[j][1], pa[j][2], pa[j][3], b0, b1);
        mma16816<DT>(o[dp * 2 + 1], pa[j][0], pa[j][1], pa[j][2], pa[j][3], b2, b3);
      }
    }
  }

  __device__ __forceinline__ void stash(float* merge_o, float* merge_ml, int lane) {
    // complete the row sums across the quad
    float l0 = l[0], l1 = l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const int r0 = lane >> 2, r1 = r0 + 8;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      const int c = n * 8 + (lane & 3) * 2;
      if (r0 < G) { merge_o[r0 * D + c] = o[n][0]; merge_o[r0 * D + c + 1] = o[n][1]; }
      if (r1 < G) { merge_o[r1 * D + c] = o[n][2]; merge_o[r1 * D + c + 1] = o[n][3]; }
    }
    if ((lane & 3) == 0) {
      if (r0 < G) { merge_ml[r0 * 2] = m[0]; merge_ml[r0 * 2 + 1] = l0; }
      if (r1 < G) { merge_ml[r1 * 2] = m[1]; merge_ml[r1 * 2 + 1] = l1; }
    }
  }
};

// ------------------------------------------------------------------ split kernel
template <int DT, int D, int G, int NW, int NSTAGES, bool MMA>
__global__ void __launch_bounds__((NW + 1) * 32) decode_split_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                     const __grid_constant__ CUtensorMap vmap,
                                                                     const DecodeParams p) {
  using LY = Layout<D, G, NW, NSTAGES>;
  using T = typename Elt<DT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::BAR_OFF);
  uint64_t* empty = full + NSTAGES;
  int32_t* bt_s = reinterpret_cast<int32_t*>(smem + LY::BT_OFF);

  const int Hkv = p.num_kv_heads;
  const int u = blockIdx.x;
  const int g = u % Hkv;
  const int s = (u / Hkv) % p.max_splits;
  const int b = u / (Hkv * p.max_splits);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int L = __ldg(p.context_lens + b);
  {  // a length beyond what the grid or the block-table row covers is a caller error: clamp and record
    const int cap = min(p.max_splits * p.split_len, p.max_blocks_per_seq * p.block_size);
    if (L < 0 || L > cap) {
      if (threadIdx.x == 0 && s == 0 && g == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
      L = L < 0 ? 0 : cap;
    }
  }
  const int t0 = s * p.split_len;
  if (t0 >= L) {
    if (s == 0) {  // empty sequence: out = 0 (documented)
      T* ob = reinterpret_cast<T*>(p.out) + ((size_t)b * p.num_q_heads + (size_t)g * G) * D;
      for (int i = threadIdx.x; i < G * D; i += blockDim.x) ob[i] = Elt<DT>::from_f(0.f);
    }
    return;
  }
  const int t1 = min(L, t0 + p.split_len);
  const int nsplit = (L + p.split_len - 1) / p.split_len;
  const int nstages = (t1 - t0 + LY::TOK - 1) / LY::TOK;
  const int first_blk = t0 / p.block_size;
  const int nblk = (t1 - 1) / p.block_size - first_blk + 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    fence_mbar_init();
  }
  const T* qg = reinterpret_cast<const T*>(p.q) + ((size_t)b * p.num_q_heads + (size_t)g * G) * D;
  if (warp == NW) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    const int32_t* bt = p.block_tables + (size_t)b * p.max_blocks_per_seq + first_blk;
    for (int i = lane; i < nblk; i += 32) bt_s[i] = __ldg(bt + i);
  } else if constexpr (!MMA) {
    float* q_s = reinterpret_cast<float*>(smem + LY::Q_OFF);
    for (int i = threadIdx.x; i < G * D; i += NW * 32) q_s[i] = (float)qg[i] * p.scale_log2;
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------ producer: TMA gather through the block table
    bool ok = true;
    for (int k = 0; k < nstages && ok; ++k) {
      const int st = k % NSTAGES;
      if (k >= NSTAGES) ok = mbar_wait(&empty[st], ((k / NSTAGES) - 1) & 1);
      if (!ok) break;
      const int tok_base = t0 + k * LY::TOK;
      const int nbox = min(LY::BOXES, (t1 - tok_base + 15) >> 4);
      if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)(nbox * 16 * D * 2 * 2));
      __syncwarp();
      if (lane < nbox) {
        const int tok = tok_base + lane * 16;
        const int phys = bt_s[tok / p.block_size - first_blk];
        if (phys < 0 || phys >= p.num_blocks) PA_RECORD_ERROR(PA_ERRBIT_INDEX);  // TMA zero-fills out of range
        const int y = phys * p.block_size + (tok % p.block_size);
        uint8_t* kd = smem + LY::K_OFF + st * LY::STAGE_BYTES + lane * 16 * 128;
        uint8_t* vd = smem + LY::V_OFF + st * LY::STAGE_BYTES + lane * 16 * 128;
#pragma unroll
        for (int h = 0; h < LY::HALVES; ++h) {
          tma_load_2d(kd + h * LY::TOK * 128, &kmap, g * D + h * 64, y, &full[st]);
          tma_load_2d(vd + h * LY::TOK * 128, &vmap, g * D + h * 64, y, &full[st]);
        }
      }
    }
    if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    // drain: make sure every TMA this CTA issued has landed before the CTA can exit
    if (lane == 0) {
      for (int k = max(0, nstages - NSTAGES); k < nstages; ++k)
        if (!mbar_wait(&full[k % NSTAGES], (k / NSTAGES) & 1)) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    }
    return;
  }

  // -------------------------------------------------- consumers
  using C = typename std::conditional<MMA, MmaConsumer<DT, D, G, NW, NSTAGES>, CoreConsumer<DT, D, G, NW, NSTAGES>>::type;
  C c;
  c.init();
  if constexpr (MMA) c.load_q(qg, lane);
  const uint32_t qbase = sbase + LY::Q_OFF;
  const uint32_t pbase = sbase + LY::P_OFF + warp * 32 * G * 4;
  bool ok = true;
  for (int k = 0; k < nstages; ++k) {
    const int st = k % NSTAGES;
    if (!mbar_wait(&full[st], (k / NSTAGES) & 1)) {
      ok = false;
      break;
    }
    const int nv = min(32, max(0, t1 - (t0 + k * LY::TOK + warp * 32)));
    if (nv > 0) {
      const uint32_t kb = sbase + LY::K_OFF + st * LY::STAGE_BYTES;
      const uint32_t vb = sbase + LY::V_OFF + st * LY::STAGE_BYTES;
      if constexpr (MMA)
        c.tile(kb, vb, p.scale_log2, warp * 32, nv, lane);
      else
        c.tile(kb, vb, qbase, pbase, warp * 32, nv, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);

  // -------------------------------------------------- merge the NW warps, write out or a split partial
  float* merge_o = reinterpret_cast<float*>(smem + LY::M_OFF);
  float* merge_ml = reinterpret_cast<float*>(smem + LY::ML_OFF);
  named_barrier_sync(1, NW * 32);  // every consumer is done reading the stage buffers
  c.stash(merge_o + warp * G * D, merge_ml + warp * G * 2, lane);
  named_barrier_sync(1, NW * 32);
  const int hq0 = g * G;
  for (int i = threadIdx.x; i < G * D; i += NW * 32) {
    const int h = i / D, d = i - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, merge_ml[(w * G + h) * 2]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float sc = fast_exp2(merge_ml[(w * G + h) * 2] - M);
      num = fmaf(sc, merge_o[(w * G + h) * D + d], num);
      den = fmaf(sc, merge_ml[(w * G + h) * 2 + 1], den);
    }
    const size_t row = (size_t)b * p.num_q_heads + hq0 + h;
    if (nsplit == 1) {
      reinterpret_cast<T*>(p.out)[row * D + d] = Elt<DT>::from_f(num / den);
    } else {
      const size_t srow = row * p.max_splits + s;
      p.ws_o[srow * D + d] = num;
      if (d == 0) {
        p.ws_m[srow] = M;
        p.ws_l[srow] = den;
      }
    }
  }
}

// ------------------------------------------------------------------ split-K reduce
// One warp per (b, h): out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, M = max_s m_s.
template <int DT, int D>
__global__ void __launch_bounds__(128) decode_reduce_kernel(const DecodeParams p) {
  using T = typename Elt<DT>::T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;  // b * Hq + h
  if (row >= p.batch * p.num_q_heads) return;
  const int b = row / p.num_q_heads;
  const int L = __ldg(p.context_lens + b);
  const int ns = min((max(L, 0) + p.split_len - 1) / p.split_len, p.max_splits);
  if (ns <= 1) return;  // written directly by the split kernel
  const float* m = p.ws_m + (size_t)row * p.max_splits;
  const float* l = p.ws_l + (size_t)row * p.max_splits;
  float M = -INFINITY;
  for (int i = lane; i < ns; i += 32) M = fmaxf(M, m[i]);
  M = warp_max(M);
  constexpr int DPL = D / 32;
  float acc[DPL];
#pragma unroll
  for (int j = 0; j < DPL; ++j) acc[j] = 0.f;
  float den = 0.f;
  const float* o = p.ws_o + (size_t)row * p.max_splits * D + lane * DPL;
  for (int i = 0; i < ns; ++i) {
    const float w = fast_exp2(m[i] - M);
    den = fmaf(w, l[i], den);
    if constexpr (DPL == 4) {
      const float4 v = *reinterpret_cast<const float4*>(o + (size_t)i * D);
      acc[0] = fmaf(w, v.x, acc[0]); acc[1] = fmaf(w, v.y, acc[1]);
      acc[2] = fmaf(w, v.z, acc[2]); acc[3] = fmaf(w, v.w, acc[3]);
    } else {
      const float2 v = *reinterpret_cast<const float2*>(o + (size_t)i * D);
      acc[0] = fmaf(w, v.x, acc[0]); acc[1] = fmaf(w, v.y, acc[1]);
    }
  }
  const float inv = 1.f / den;
  T* out = reinterpret_cast<T*>(p.out) + (size_t)row * D + lane * DPL;
  if constexpr (DPL == 4) {
    uint2 w;
    w.x = Elt<DT>::from_f2(acc[0] * inv, acc[1] * inv);
    w.y = Elt<DT>::from_f2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(out) = w;
  } else {
    *reinterpret_cast<uint32_t*>(out) = Elt<DT>::from_f2(acc[0] * inv, acc[1] * inv);
  }
}

// ------------------------------------------------------------------ host side
constexpr int kNW = 2;        // consumer warps per CTA (64-token stages)
constexpr int kStages = 2;    // ring depth

struct Plan {
  int split_len;
  int max_splits;
  size_t ws_bytes;
  size_t off_l, off_o;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool make_plan(int batch, int Hq, int Hkv, int D, int max_ctx, int num_splits, Plan* pl) {
  if (batch < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_ctx < 0 || num_splits < 0) return false;
  const int gran = 64;
  const int max_split_len = 8192;  // keeps a split's block-table slice within BT_MAX entries
  int sl;
  if (num_splits > 0) {
    sl = (max_ctx + num_splits - 1) / num_splits;
    sl = std::max(gran, (sl + gran - 1) / gran * gran);
  } else {
    // Enough CTAs to fill the GPU several times over, but splits long enough
    // to amortise their partial write and pipeline fill.
    const long units = (long)batch * Hkv;
    const long target = 148L * 16;
    sl = 256;
    while (sl * 2 <= 4096 && units * ((max_ctx + 2 * sl - 1) / (2 * sl)) >= target) sl *= 2;
  }
  if (max_ctx > 0 && sl > ((max_ctx + gran - 1) / gran) * gran) sl = ((max_ctx + gran - 1) / gran) * gran;
  if (sl > max_split_len) sl = max_split_len;
  pl->split_len = sl;
  pl->max_splits = max_ctx > 0 ? (max_ctx + sl - 1) / sl : 1;
  const size_t rows = (size_t)batch * Hq * pl->max_splits;
  if (pl->max_splits <= 1) {
    pl->ws_bytes = 0;
    pl->off_l = pl->off_o = 0;
    return true;
  }
  pl->off_l = align256(rows * 4);
  pl->off_o = pl->off_l + align256(rows * 4);
  pl->ws_bytes = pl->off_o + align256(rows * D * 4);
  return true;
}

template <int DT, int D, int G>
int launch(const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p, cudaStream_t st) {
  constexpr bool MMA = G >= 8;
  using LY = Layout<D, G, kNW, kStages>;
  auto kern = decode_split_kernel<DT, D, G, kNW, kStages, MMA>;
  static bool attr_set[64] = {};  // per instantiation and device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::ALLOC) != cudaSuccess)
      return PA_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const long grid = (long)p.batch * p.max_splits * p.num_kv_heads;
  if (grid > 0) {
    kern<<<(unsigned)grid, (kNW + 1) * 32, LY::ALLOC, st>>>(km, vm, p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  if (p.max_splits > 1) {
    const int rows = p.batch * p.num_q_heads;
    decode_reduce_kernel<DT, D><<<(rows + 3) / 4, 128, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <int DT, int D>
int dispatch_g(int G, const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p, cudaStream_t st) {
  switch (G) {
    case 1: return launch<DT, D, 1>(km, vm, p, st);
    case 2: return launch<DT, D, 2>(km, vm, p, st);
    case 4: return launch<DT, D, 4>(km, vm, p, st);
    case 8: return launch<DT, D, 8>(km, vm, p, st);
    case 16: return launch<DT, D, 16>(km, vm, p, st);
  }
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" int pa_decode_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                              int num_splits_or_0, int* split_len_out, int* max_splits_out,
                              size_t* workspace_bytes_out) {
  Plan pl;
  if (!make_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_splits_or_0, &pl))
    return PA_ERR_INVALID;
  if (split_len_out) *split_len_out = pl.split_len;
  if (max_splits_out) *max_splits_out = pl.max_splits;
  if (workspace_bytes_out) *workspace_bytes_out = pl.ws_bytes;
  return PA_OK;
}

extern "C" size_t pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                           int max_context_len, int num_splits_or_0) {
  Plan pl;
  if (!make_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_splits_or_0, &pl)) return 0;
  return pl.ws_bytes;
}

extern "C" int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
                         float scale, int dtype, void* workspace, size_t workspace_bytes, int num_splits_or_0,
                         void* out, void* stream) {
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks < 0 ||
      max_context_len < 0 || max_blocks_per_seq < 0 || num_splits_or_0 < 0)
    return PA_ERR_INVALID;
  if (!pa::valid_dtype(dtype) || !pa::valid_head_dim(head_dim) || !pa::valid_block_size(block_size))
    return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID;
  const int G = num_q_heads / num_kv_heads;
  if (!pa::valid_group(G)) return PA_ERR_UNSUPPORTED;
  if (batch == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID;
  if (!pa::aligned16(q) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache) || !pa::aligned16(out) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_ALIGN;
  if ((long)max_blocks_per_seq * block_size < max_context_len) return PA_ERR_INVALID;
  if (num_blocks == 0 && max_context_len > 0) return PA_ERR_INVALID;
  Plan pl;
  if (!make_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_splits_or_0, &pl))
    return PA_ERR_INVALID;
  if (pl.max_splits > 1) {
    if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PA_ERR_ALIGN;
  }
  if ((long)batch * pl.max_splits * num_kv_heads > 0x7fffffffL) return PA_ERR_UNSUPPORTED;

  DecodeParams p;
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  p.ws_m = reinterpret_cast<float*>(ws);
  p.ws_l = reinterpret_cast<float*>(ws ? ws + pl.off_l : nullptr);
  p.ws_o = reinterpret_cast<float*>(ws ? ws + pl.off_o : nullptr);
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.split_len = pl.split_len;
  p.max_splits = pl.max_splits;
  p.scale_log2 = scale * kLog2e;

  // One tensor map per cache over the [num_blocks*block_size][Hkv*D] row view; 16-row x 64-column boxes.
  CUtensorMap km, vm;
  const uint64_t rows = (uint64_t)std::max(num_blocks, 1) * block_size;
  const uint64_t cols = (uint64_t)num_kv_heads * head_dim;
  if (pa::encode_2d_sw128(&km, k_cache, cols, rows, cols * 2, 64, 16) != PA_OK) return PA_ERR_CUDA;
  if (pa::encode_2d_sw128(&vm, v_cache, cols, rows, cols * 2, 64, 16) != PA_OK) return PA_ERR_CUDA;

  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == PA_BF16)
    return head_dim == 128 ? dispatch_g<PA_BF16, 128>(G, km, vm, p, st) : dispatch_g<PA_BF16, 64>(G, km, vm, p, st);
  return head_dim == 128 ? dispatch_g<PA_F16, 128>(G, km, vm, p, st) : dispatch_g<PA_F16, 64>(G, km, vm, p, st);
}
