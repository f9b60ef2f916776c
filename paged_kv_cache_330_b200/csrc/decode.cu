// Paged decode attention for sm_100a: persistent, evenly partitioned split-K.
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
// Work split.  A segment is one (sequence b, KV head g); it holds
// ceil(L_b/16) chunks of 16 tokens.  All segments, laid end to end in (b, g)
// order, form one line of C chunks.  CTA c of the persistent grid takes chunks
// [C*c/grid, C*(c+1)/grid): every CTA reads the same number of KV bytes,
// whatever the length mix.  The part of a segment that falls in one CTA is a
// piece; a piece that is a whole segment writes `out` directly, otherwise it
// writes fp32 (max, sum, acc) to the workspace; the CTA that writes a segment's
// last piece merges them (log-sum-exp rule).  This is the single-device reading
// of the context split on "In-depth analysis of vllm-ascend", section 3.1.
//
// Data movement.  One producer warp walks the CTA's chunk range, looks up each
// chunk's physical block (several stages ahead, cp.async into a plan ring) and
// gathers 16-row K and V boxes
// with TMA (cp.async.bulk.tensor, 128-byte swizzle, no multicast) into an
// NSTAGES-deep shared-memory ring guarded by mbarriers, straight across piece
// and segment boundaries (the pages' prefetch-depth / pipeline-stage lesson,
// vLLM-Ascend page section 2.2).  Each stage also carries a small descriptor
// and, at a piece's first stage, the G query rows of the group (bulk copy).
// NW consumer warps take 32 tokens of every stage each.
//
// Math.  fp32 scores in the log2 domain (scale*log2(e)), online softmax with
// fp32 running max and sum, fp32 accumulators.
//   * G <= 4: CUDA cores.  QK^T: lane = token, one full dot product per lane;
//     max/sum by warp shuffles; PV: lane = slice of head_dim.
//   * G >= 8: the FP32 pipe cannot keep up with HBM at 8 flop per KV byte, so
//     QK^T and PV use warp-level mma.m16n8k16 (bf16/f16 in, fp32 out) with the
//     G query heads as rows.  P enters PV as two 16-bit terms (hi + lo), which
//     keeps it exact to about 2^-17 instead of the 2^-9 of one bf16 rounding.

#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_decode)

namespace {

using namespace pa;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kChunk = 16;  // tokens per chunk = rows per TMA box
constexpr int kPlanRing = 8;  // producer plan ring slots
constexpr int kMaxPieces = 32;  // pieces per segment the epilogue merges with precomputed weights
constexpr int kLookahead = 3; // stages planned (block-table entries in flight) ahead of the one issued
static_assert(kPlanRing > kLookahead, "plan ring must hold the stages in flight plus the one issued");

struct DecodeParams {
  const void* q;
  void* out;
  const float* k_scales;  // int8 cache only: fp32 [num_blocks][Hkv][block_size]
  const float* v_scales;
  float* lse;             // optional fp32 [batch][Hq]: ln sum_t exp(scale <q, K_t>) (-inf for an empty context)
  const int32_t* ctx_start;  // optional int32 [batch]: tokens skipped at the head of each context (multiple of 16)
  const int32_t* block_tables;
  const int32_t* context_lens;
  int* ws_cnt;        // [B*Hkv] pieces of each segment written so far (zero between calls)
  float* ws_m;        // [nslots][G] running max of a piece (log2 domain)
  float* ws_l;        // [nslots][G] sum of exp2(x - m)
  float* ws_o;        // [nslots][G][D] sum of exp2(x - m) * v
  int max_blocks_per_seq;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int grid;
  float scale_log2;
};

enum : int { F_FIRST = 1, F_LAST = 2, F_DIRECT = 4, F_END = 8 };

// One stage as the producer planned it.  vid: the CTA that walks it; its piece's partial goes to workspace
// slot segment + vid.  c0/npieces (set on a piece's last stage) name the first CTA holding a piece of this
// segment and how many pieces the segment has, for the merge.
struct StageMeta {
  int b, g, tok0, ntok, flags, vid, c0, npieces;
};

__device__ __forceinline__ int stage_chunks(const StageMeta& d) { return (d.ntok + 15) / 16; }

// Shared-memory layout of one CTA.  Q8: the cache holds int8 codes (one byte per element) and per-token
// fp32 scales, which each stage carries next to the codes.
template <int D, int G, int NW, int NSTAGES, bool MMA, bool Q8 = false>
struct Layout {
  static constexpr int TOK = NW * 32;             // tokens per stage
  static constexpr int CPS = TOK / kChunk;        // chunks (16-row boxes) per stage
  static constexpr int ROWB = Q8 ? D : 2 * D;     // bytes of one (token, KV head) cache row
  static constexpr int BOXB = ROWB >= 128 ? 128 : ROWB;  // bytes per row of one TMA box
  static constexpr int HALVES = ROWB / BOXB;      // column boxes per row
  static constexpr int STAGE_BYTES = TOK * ROWB;  // K (or V) bytes per stage
  static constexpr int QSLOT = G * D * 2;         // the group's q rows
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + NSTAGES * STAGE_BYTES;
  static constexpr int SK_OFF = V_OFF + NSTAGES * STAGE_BYTES;                // fp32 K scales [NSTAGES][TOK] (Q8)
  static constexpr int SV_OFF = SK_OFF + (Q8 ? NSTAGES * TOK * 4 : 0);        // fp32 V scales [NSTAGES][TOK] (Q8)
  static constexpr int QS_OFF = SV_OFF + (Q8 ? NSTAGES * TOK * 4 : 0);
  static constexpr int META_OFF = QS_OFF + NSTAGES * QSLOT;
  static constexpr int PLAN_OFF = META_OFF + NSTAGES * (int)sizeof(StageMeta);  // producer plan ring
  static constexpr int PLAN_BYTES = kPlanRing * ((int)sizeof(StageMeta) + 8 * 4);
  static constexpr int QF_OFF = PLAN_OFF + PLAN_BYTES;                        // fp32 q per warp (CUDA-core path)
  static constexpr int QF_BYTES = MMA ? 0 : NW * G * D * 4;
  static constexpr int P_OFF = QF_OFF + QF_BYTES;                             // fp32 p per warp (CUDA-core path)
  static constexpr int P_BYTES = MMA ? 0 : NW * 32 * G * 4;
  // two merge buffers handed from the consumers to the epilogue warp:
  // fp32 o [NW][G][D], fp32 (m, l) [NW][G][2], then the piece's descriptor
  static constexpr int MB_O = 0;
  static constexpr int MB_ML = NW * G * D * 4;
  static constexpr int MB_DESC = MB_ML + NW * G * 2 * 4;
  static constexpr int MB_BYTES = (MB_DESC + (int)sizeof(StageMeta) + 15) / 16 * 16;
  static constexpr int M_OFF = P_OFF + P_BYTES;
  static constexpr int WTS_OFF = M_OFF + 2 * MB_BYTES;                        // merge weights fp32 [G][kMaxPieces]
  static constexpr int VIDS_OFF = WTS_OFF + G * kMaxPieces * 4;               // merge: slot of each piece, int32
  static constexpr int MISC_OFF = VIDS_OFF + kMaxPieces * 4;                  // int64 total chunks on the line
  static constexpr int BAR_OFF = MISC_OFF + 16;  // full[NSTAGES], empty[NSTAGES], mfull[2], mempty[2]
  static constexpr int BYTES = BAR_OFF + (2 * NSTAGES + 4) * 8;
  static constexpr int ALLOC = BYTES + 1024;                                  // slack for 1024-byte alignment
  static_assert(QS_OFF % 16 == 0 && QSLOT % 16 == 0 && BAR_OFF % 8 == 0, "alignment");
  static_assert(CPS <= 8, "plan ring holds 8 block lookups per stage");
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

// Address of byte `byte` (a multiple of 4 within its 16-byte chunk is what callers use) of row r of an
// int8 stage buffer of ROWB-byte rows written by TMA: 128-byte rows carry the 128-byte swizzle (16-byte
// chunk index XOR r%8), 64-byte rows the 64-byte swizzle (chunk index XOR (r/2)%4).
template <int ROWB>
__device__ __forceinline__ uint32_t swz8_addr(uint32_t base, int r, int byte) {
  if constexpr (ROWB == 128)
    return base + r * 128 + ((((byte >> 4) ^ (r & 7)) & 7) << 4) + (byte & 15);
  else
    return base + r * 64 + ((((byte >> 4) ^ (r >> 1)) & 3) << 4) + (byte & 15);
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
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ long long warp_incl_scan_ll(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// 1-D bulk copy global -> shared, completion in bytes on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cp_async4(void* smem_dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ CUDA-core consumer (G <= 4)
template <int DT, int D, int G, int NW, int NSTAGES>
struct CoreConsumer {
  using LY = Layout<D, G, NW, NSTAGES, false>;
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

  // The group's q rows (16-bit, [G][D]) -> this warp's fp32 copy scaled by scale*log2(e).
  __device__ __forceinline__ void load_q(const uint8_t* qslot, float* qf, float scale_log2, int lane) {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qslot);
    for (int i = lane; i < G * D / 2; i += 32) {
      const float2 f = Elt<DT>::to_f2(q32[i]);
      qf[2 * i] = f.x * scale_log2;
      qf[2 * i + 1] = f.y * scale_log2;
    }
    __syncwarp();
  }

  // One 32-token tile: rows r0 .. r0+31 of the stage, nv of them valid.
  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, uint32_t qbase, uint32_t pbase, int r0,
                                       int nv, int lane) {
    // ---- scores: lane = token; four partial sums per head keep the FMA chains short
    float acc[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
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
        acc[h][0] = fmaf(k01.x, __uint_as_float(qa.x), acc[h][0]);
        acc[h][1] = fmaf(k01.y, __uint_as_float(qa.y), acc[h][1]);
        acc[h][2] = fmaf(k23.x, __uint_as_float(qa.z), acc[h][2]);
        acc[h][3] = fmaf(k23.y, __uint_as_float(qa.w), acc[h][3]);
        acc[h][0] = fmaf(k45.x, __uint_as_float(qb.x), acc[h][0]);
        acc[h][1] = fmaf(k45.y, __uint_as_float(qb.y), acc[h][1]);
        acc[h][2] = fmaf(k67.x, __uint_as_float(qb.z), acc[h][2]);
        acc[h][3] = fmaf(k67.y, __uint_as_float(qb.w), acc[h][3]);
      }
    }
    // ---- online softmax (log2 domain), fp32
    float p[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float s = lane < nv ? (acc[h][0] + acc[h][1]) + (acc[h][2] + acc[h][3]) : -INFINITY;
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
#pragma unroll 4
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
// LO_ALL: P always enters PV as hi + lo (exact to ~2^-17).  Otherwise the lo term's products are issued
// only for a tile in which some row's share of its running softmax mass is at least 1/16 (the first tile,
// and tiles holding dominant keys); elsewhere the hi term alone moves an output by at most 2^-9 of that
// tile's share of |v|, which is under 1/16 of the row's mass.
template <int DT, int D, int G, int NW, int NSTAGES, bool LO_ALL = true>
struct MmaConsumer {
  using LY = Layout<D, G, NW, NSTAGES, true>;
  static constexpr int KS = D / 16;   // k-steps of QK^T
  static constexpr int ND = D / 8;    // n-tiles of PV
  uint32_t qa[KS][4];                 // A fragments of q (rows = heads, padded to 16)
  float o[ND][4];                     // rows lane/4 and lane/4+8, columns of an n-tile
  float m[2], l[2];                   // per row owned by this thread (lane/4, lane/4+8); l is a partial sum

  __device__ __forceinline__ void load_q(const uint8_t* qslot, float*, float, int lane) {
    const int r0 = lane >> 2, r1 = r0 + 8;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qslot);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int c = ks * 16 + (lane & 3) * 2;
      qa[ks][0] = r0 < G ? q32[(r0 * D + c) / 2] : 0u;
      qa[ks][1] = r1 < G ? q32[(r1 * D + c) / 2] : 0u;
      qa[ks][2] = r0 < G ? q32[(r0 * D + c + 8) / 2] : 0u;
      qa[ks][3] = r1 < G ? q32[(r1 * D + c + 8) / 2] : 0u;
    }
  }

  __device__ __forceinline__ void init() {
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int n = 0; n < ND; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  }

  template <int DT2 = DT>
  static __device__ __forceinline__ void split_hi_lo(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = Elt<DT2>::from_f2(a, b);
    const float2 h = Elt<DT2>::to_f2(hi);
    lo = Elt<DT2>::from_f2(a - h.x, b - h.y);
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
    uint32_t ph[2][4], pl[2][4];  // A fragments of P = hi + lo for the two 16-token k-steps
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const float p0 = fast_exp2(s[n][0] - mn0), p1 = fast_exp2(s[n][1] - mn0);
      const float p2 = fast_exp2(s[n][2] - mn1), p3 = fast_exp2(s[n][3] - mn1);
      ls0 += p0 + p1;
      ls1 += p2 + p3;
      split_hi_lo(p0, p1, ph[n >> 1][(n & 1) * 2 + 0], pl[n >> 1][(n & 1) * 2 + 0]);
      split_hi_lo(p2, p3, ph[n >> 1][(n & 1) * 2 + 1], pl[n >> 1][(n & 1) * 2 + 1]);
    }
    l[0] = l[0] * al0 + ls0;
    l[1] = l[1] * al1 + ls1;
    // this lane's columns of the tile against this lane's columns of the running sum (both partial sums
    // over the same column subset)
    const bool lo = LO_ALL || __any_sync(0xffffffffu, ls0 >= 0.0625f * l[0] || ls1 >= 0.0625f * l[1]);
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
        mma16816<DT>(o[dp * 2], ph[j][0], ph[j][1], ph[j][2], ph[j][3], b0, b1);
        mma16816<DT>(o[dp * 2 + 1], ph[j][0], ph[j][1], ph[j][2], ph[j][3], b2, b3);
        if (lo) {
          mma16816<DT>(o[dp * 2], pl[j][0], pl[j][1], pl[j][2], pl[j][3], b0, b1);
          mma16816<DT>(o[dp * 2 + 1], pl[j][0], pl[j][1], pl[j][2], pl[j][3], b2, b3);
        }
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

// ------------------------------------------------------------------ int8-cache consumer (every G)
// Scores and PV on mma.m16n8k16 with fp16 operands and tokens as the M rows, so a group of G <= 8 heads
// fills one n-tile of 8 columns instead of padding 16 rows:
//   S^T[t][h] = sum_d code_k[t][d] q[h][d]           (A = K codes, B = q^T)
//   O^T[d][h] += sum_t code_v[t][d] P'[h][t]          (A = V^T codes, B = P'^T)
// The codes become fp16 exactly (|code| <= 127): biased by 128 (XOR 0x80), two bytes are placed under
// the fp16 exponent of 1024 by one byte permute, and 1152 is subtracted (HSUB2).  The head_dim order
// inside a k-step is permuted so that every lane's operand bytes are contiguous: the sum over d does not
// depend on the order as long as q uses the same one, and O^T's row order is undone when it is stored.
// q is converted to fp16 once per piece after an exact power-of-two prescale that puts its largest
// magnitude in [2^14, 2^15); the prescale is undone in the score scale.  The dequantisation costs one
// multiply per token and head for K, s = scale_k[t] * (q . code_k[t]), and folds scale_v into the
// softmax weight that enters PV: with m the running score maximum, u = (s - m) + log2(scale_v[t]) (formed
// relative to m so that fp32 keeps the scale's bits however large the logits) and P' = 2^(u - rho), rho
// the running maximum of u, so the largest weight of a head is exactly 1 and every P' lies in [0, 1]
// (fp16 holds it to 2^-11 relative).  O is kept relative to (m, rho): O relative to m is O * 2^rho; the
// sum l is relative to m; both are rescaled when a maximum moves.
template <int D, int G, int NW, int NSTAGES>
struct Q8Consumer {
  using LY = Layout<D, G, NW, NSTAGES, true, true>;
  static constexpr int NT = (G + 7) / 8;  // n-tiles of 8 heads
  static constexpr int KS = D / 16;       // k-steps of QK^T, and m-tiles (16 rows of d) of O^T
  static constexpr int QB = D / 4;        // bytes of a K row one lane reads (its quarter of the row)
  static constexpr bool kPieceV = G <= 4;  // V codes read as one piece per row (see tile)
  uint32_t qb[NT][KS][2];                 // B fragments of q^T (fp16, prescaled)
  float o[NT][KS][4];                     // O^T relative to (m, rho): rows d (permuted), columns heads
  float m[NT][2], l[NT][2];               // heads 8nt + 2(lane%4) + {0,1}; l is this lane's partial sum
  float rho[NT][2];                       // running max of (s - m) + log2(scale_v) per head
  float qbias[NT][2];                     // -1152 * sum over d of the fp16 q^T of heads 8nt + 2(lane%4) + {0,1}
  float qs;                               // scale * log2(e) / prescale

  static __device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
  }
  // fp16x2 of bytes 0,1 (lo) or 2,3 (hi) of a word of codes already XORed with 0x80808080: the byte lands in
  // the low mantissa bits under the exponent of 1024, so each half is exactly 1152 + code (codes -128 .. 127
  // give 1024 .. 1279, integers fp16 holds exactly).  The 1152 is taken out in fp32 instead of here: for K it
  // starts the score accumulators (qbias), for V one product of the tile's P with a constant -1152 operand
  // comes off O in the rescale (a per-head term, the same for every row d).
  static constexpr uint32_t kNegBias = 0xE480E480u;  // fp16x2 (-1152, -1152)
  static __device__ __forceinline__ uint32_t to_h2(uint32_t xb, uint32_t sel) { return prmt(xb, 0x64646464u, sel); }
  static __device__ __forceinline__ void mma_f16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t trans8x8(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
  }
  static __device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      rho[nt][0] = rho[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int i = 0; i < KS; ++i) o[nt][i][0] = o[nt][i][1] = o[nt][i][2] = o[nt][i][3] = 0.f;
    }
  }

  // The group's q rows (16-bit [G][D], element type DT) -> fp16 B fragments after the prescale.
  template <int DT>
  __device__ __forceinline__ void load_q(const uint8_t* qslot, float scale_log2, int lane) {
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qslot);
    float amax = 0.f;
    for (int i = lane; i < G * D / 2; i += 32) {
      const float2 f = Elt<DT>::to_f2(q32[i]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    amax = warp_max(amax);
    int e = 0;
    if (amax > 0.f) {
      int k;
      frexpf(amax, &k);  // amax in [2^(k-1), 2^k)
      e = 15 - k;
      e = e < -60 ? -60 : (e > 60 ? 60 : e);
    }
    const float f = __int_as_float((127 + e) << 23), finv = __int_as_float((127 - e) << 23);
    qs = scale_log2 * finv;
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 8 + g;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0 = 0u, b1 = 0u;
        if (h < G) {
          const int d0 = c * QB + 4 * ks;
          const float2 x01 = Elt<DT>::to_f2(q32[(h * D + d0) / 2]);
          const float2 x23 = Elt<DT>::to_f2(q32[(h * D + d0) / 2 + 1]);
          b0 = pack_h2(x01.x * f, x01.y * f);
          b1 = pack_h2(x23.x * f, x23.y * f);
        }
        qb[nt][ks][0] = b0;
        qb[nt][ks][1] = b1;
      }
      // -1152 * sum_d q^T[d][h] in fp32, in the layout of the score accumulators (rows tokens, columns heads)
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) mma_f16(acc, kNegBias, kNegBias, kNegBias, kNegBias, qb[nt][ks][0], qb[nt][ks][1]);
      qbias[nt][0] = acc[0];
      qbias[nt][1] = acc[1];
    }
  }

  // One 32-token tile: rows r0 .. r0+31 of the stage, nv of them valid.  skb/svb: shared-memory addresses of
  // the stage's fp32 K and V scales.
  __device__ __forceinline__ void tile(uint32_t kbase, uint32_t vbase, uint32_t skb, uint32_t svb, int r0, int nv,
                                       int lane) {
    const int g = lane >> 2, c = lane & 3;
    // ---- S^T = K q^T: 2 m-tiles of 16 tokens x NT n-tiles of 8 heads
    float s[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        s[mt][nt][0] = s[mt][nt][2] = qbias[nt][0];  // the codes enter as 1152 + code: start at -1152 * sum q
        s[mt][nt][1] = s[mt][nt][3] = qbias[nt][1];
      }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int ta = r0 + 16 * mt + g, tb = ta + 8;
      uint32_t ka[KS], kb[KS];
#pragma unroll
      for (int i = 0; i < QB / 16; ++i) {
        const uint4 u = lds128(swz8_addr<LY::ROWB>(kbase, ta, c * QB + 16 * i));
        const uint4 w = lds128(swz8_addr<LY::ROWB>(kbase, tb, c * QB + 16 * i));
        ka[4 * i + 0] = u.x ^ 0x80808080u; ka[4 * i + 1] = u.y ^ 0x80808080u;
        ka[4 * i + 2] = u.z ^ 0x80808080u; ka[4 * i + 3] = u.w ^ 0x80808080u;
        kb[4 * i + 0] = w.x ^ 0x80808080u; kb[4 * i + 1] = w.y ^ 0x80808080u;
        kb[4 * i + 2] = w.z ^ 0x80808080u; kb[4 * i + 3] = w.w ^ 0x80808080u;
      }
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t a0 = to_h2(ka[ks], 0x4140u), a2 = to_h2(ka[ks], 0x4342u);
        const uint32_t a1 = to_h2(kb[ks], 0x4140u), a3 = to_h2(kb[ks], 0x4342u);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16(s[mt][nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
      }
    }
    // ---- per-token K scales, mask, online softmax per head (column), fp32 in the log2 domain
    float lsv[2][2];  // log2 of the V scale of this lane's rows (-inf for invalid tokens and zero scales)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * mt + g + 8 * hh;  // token within the tile
        const bool ok = t < nv;
        const float sk = __uint_as_float(lds32(skb + (r0 + t) * 4)) * qs;
        const float sv = __uint_as_float(lds32(svb + (r0 + t) * 4));
        lsv[mt][hh] = (ok && sv > 0.f) ? __log2f(sv) : -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          s[mt][nt][2 * hh] = ok ? s[mt][nt][2 * hh] * sk : -INFINITY;
          s[mt][nt][2 * hh + 1] = ok ? s[mt][nt][2 * hh + 1] * sk : -INFINITY;
        }
      }
    }
    uint32_t pb[NT][2][2];  // B fragments of P'^T per n-tile and k-step (16 tokens)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float beta[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(fmaxf(s[0][nt][e], s[0][nt][e + 2]), fmaxf(s[1][nt][e], s[1][nt][e + 2]));
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
        const float mn = fmaxf(m[nt][e], mx);  // finite: the tile holds a valid token
        const float alpha = fast_exp2(m[nt][e] - mn);
        const float rho_old = rho[nt][e] + (m[nt][e] - mn);  // rho relative to the new maximum (-inf stays -inf)
        m[nt][e] = mn;
        float u[2][2];
        float ux = -INFINITY, ls = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const float d0 = s[mt][nt][e] - mn, d1 = s[mt][nt][e + 2] - mn;
          ls += fast_exp2(d0) + fast_exp2(d1);
          u[mt][0] = d0 + lsv[mt][0];
          u[mt][1] = d1 + lsv[mt][1];
          ux = fmaxf(ux, fmaxf(u[mt][0], u[mt][1]));
        }
#pragma unroll
        for (int o2 = 4; o2 < 32; o2 <<= 1) ux = fmaxf(ux, __shfl_xor_sync(0xffffffffu, ux, o2));
        const float rn = fmaxf(rho_old, ux);
        const bool any = rn > -INFINITY;  // some token so far has a non-zero V scale
        beta[e] = any ? fast_exp2(rho_old - rn) : 1.f;
        rho[nt][e] = rn;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          s[mt][nt][e] = any ? fast_exp2(u[mt][0] - rn) : 0.f;
          s[mt][nt][e + 2] = any ? fast_exp2(u[mt][1] - rn) : 0.f;
        }
        l[nt][e] = l[nt][e] * alpha + ls;
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        pb[nt][mt][0] = trans8x8(pack_h2(s[mt][nt][0], s[mt][nt][1]));  // tokens 2c, 2c+1 of head g
        pb[nt][mt][1] = trans8x8(pack_h2(s[mt][nt][2], s[mt][nt][3]));  // tokens 2c+8, 2c+9
      }
      // -1152 * (sum of the tile's fp16 P' per head), laid out as O^T (every row d the same): the V codes
      // below enter as 1152 + code, so this comes off O as it is rescaled
      float pv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) mma_f16(pv, kNegBias, kNegBias, kNegBias, kNegBias, pb[nt][ks][0], pb[nt][ks][1]);
#pragma unroll
      for (int i = 0; i < KS; ++i) {
        o[nt][i][0] = fmaf(o[nt][i][0], beta[0], pv[0]); o[nt][i][2] = fmaf(o[nt][i][2], beta[0], pv[2]);
        o[nt][i][1] = fmaf(o[nt][i][1], beta[1], pv[1]); o[nt][i][3] = fmaf(o[nt][i][3], beta[1], pv[3]);
      }
    }
    // ---- O^T += V^T P'^T, k-steps of 16 tokens.  Rows t0, t0+1, t0+8, t0+9 (t0 = 16ks + 2c) give the
    // A operands of two m-tiles per 4-byte word (bytes d .. d+3 of each row): m-tile i0 holds d (row g) and
    // d+1 (row g+8), m-tile i0+1 holds d+2 and d+3.  Two load forms, chosen per group size by measurement
    // (same box, alternated): one 16-byte (D 64: 8-byte) load per row piece, d = VB*g + 4w, is faster at
    // G 2 (Qwen batch 46.6 -> 45.4 us, a long-context G 2 batch 156.9 -> 154.9 us) and slower at G 8 (Llama
    // batch 194.7 -> 197.2 us, a short-context G 8 batch 83.1 -> 84.0 us) than 4-byte loads, d = 4g + 32j;
    // stash() undoes the m-tile order of the form in use
    auto pv_word = [&](int ks, int i0, uint32_t wa, uint32_t wb, uint32_t wc, uint32_t wd) {
      const uint32_t xab = prmt(wa, wb, 0x5140u) ^ 0x80808080u, yab = prmt(wa, wb, 0x7362u) ^ 0x80808080u;
      const uint32_t xcd = prmt(wc, wd, 0x5140u) ^ 0x80808080u, ycd = prmt(wc, wd, 0x7362u) ^ 0x80808080u;
      const uint32_t a00 = to_h2(xab, 0x4140u), a01 = to_h2(xab, 0x4342u);
      const uint32_t a02 = to_h2(xcd, 0x4140u), a03 = to_h2(xcd, 0x4342u);
      const uint32_t a10 = to_h2(yab, 0x4140u), a11 = to_h2(yab, 0x4342u);
      const uint32_t a12 = to_h2(ycd, 0x4140u), a13 = to_h2(ycd, 0x4342u);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_f16(o[nt][i0], a00, a01, a02, a03, pb[nt][ks][0], pb[nt][ks][1]);
        mma_f16(o[nt][i0 + 1], a10, a11, a12, a13, pb[nt][ks][0], pb[nt][ks][1]);
      }
    };
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      if (ks * 16 >= nv) break;
      const int t0 = r0 + 16 * ks + 2 * c;
      if constexpr (kPieceV) {
        constexpr int VB = LY::ROWB / 8, VW = VB / 4;  // bytes and words of a lane's piece of a row
        uint32_t wv[4][VW];                            // rows t0, t0 + 1, t0 + 8, t0 + 9
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t a = swz8_addr<LY::ROWB>(vbase, t0 + (q & 1) + 8 * (q >> 1), VB * g);
          if constexpr (VW == 4) {
            const uint4 u = lds128(a);
            wv[q][0] = u.x; wv[q][1] = u.y; wv[q][2] = u.z; wv[q][3] = u.w;
          } else {
            const uint2 u = lds64(a);
            wv[q][0] = u.x; wv[q][1] = u.y;
          }
        }
#pragma unroll
        for (int w = 0; w < VW; ++w) pv_word(ks, 2 * w, wv[0][w], wv[1][w], wv[2][w], wv[3][w]);
      } else {
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          const int byte = 4 * g + 32 * j;
          pv_word(ks, 2 * j, lds32(swz8_addr<LY::ROWB>(vbase, t0, byte)), lds32(swz8_addr<LY::ROWB>(vbase, t0 + 1, byte)),
                  lds32(swz8_addr<LY::ROWB>(vbase, t0 + 8, byte)), lds32(swz8_addr<LY::ROWB>(vbase, t0 + 9, byte)));
        }
      }
    }
  }

  __device__ __forceinline__ void stash(float* merge_o, float* merge_ml, int lane) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float rel[2];  // O relative to m = O relative to (m, rho) times 2^rho
#pragma unroll
      for (int e = 0; e < 2; ++e) rel[e] = rho[nt][e] > -INFINITY ? exp2f(rho[nt][e]) : 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float le = l[nt][e];
        le += __shfl_xor_sync(0xffffffffu, le, 4);
        le += __shfl_xor_sync(0xffffffffu, le, 8);
        le += __shfl_xor_sync(0xffffffffu, le, 16);
        const int h = nt * 8 + 2 * c + e;
        if (g == 0 && h < G) {
          merge_ml[h * 2] = m[nt][e];
          merge_ml[h * 2 + 1] = le;
        }
      }
#pragma unroll
      for (int i = 0; i < KS; ++i) {
        const int d = kPieceV ? (LY::ROWB / 8) * g + 4 * (i >> 1) + 2 * (i & 1)  // the m-tile order of the PV
                              : 4 * g + 32 * (i >> 1) + 2 * (i & 1);           // products (see tile)
        const int h0 = nt * 8 + 2 * c;
        if (h0 < G) {
          merge_o[h0 * D + d] = o[nt][i][0] * rel[0];
          merge_o[h0 * D + d + 1] = o[nt][i][2] * rel[0];
        }
        if (h0 + 1 < G) {
          merge_o[(h0 + 1) * D + d] = o[nt][i][1] * rel[1];
          merge_o[(h0 + 1) * D + d + 1] = o[nt][i][3] * rel[1];
        }
      }
    }
  }
};

// ------------------------------------------------------------------ producer: walk of a CTA's chunk range
// Lane-uniform state (every lane of the producer warp holds the same values).
struct Walker {
  long long pos, end;         // current chunk, end of this CTA's range (global chunk line)
  long long seg_start;        // first chunk of the current segment
  long long piece_start;      // first chunk of the current piece
  int b, g, L, nch;           // current segment: sequence, KV head, clamped length, chunks
  int win_base, win_len;      // lens window: lane i holds the clamped length of sequence win_base + i
  int batch, hkv, cap, grid;
  long long total;            // chunks on the whole line
  bool narrow;                // total * grid < 2^32: every division of the walk fits in 32 bits
  int vid;                    // this CTA (see StageMeta)
  const int32_t* lens;
  const int32_t* starts;      // per-sequence first token (null: 0); the walk sees L - start tokens
  // sub-ranges still to walk after the current one, in order (at most two)
  int nq;
  long long q0_start, q0_end, q0_pre, q1_start, q1_end, q1_pre;
  int q0_b, q1_b;
  // batches of at most kRegBatch sequences: lane l holds the walk lengths of sequences 8l .. 8l+7 and the
  // chunks of all sequences before them, so lookups are shuffles instead of loads
  bool regs;
  int le[8];
  long long lane_pre;
};

constexpr int kRegBatch = 256;

// Counter add at device scope with release (writes ordered before it, including other lanes' through a
// preceding warp barrier, are visible before the count) and acquire (writes of the CTAs counted before
// are visible after it): one L2 round trip where a fence and then an atomic take two.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* ptr, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
  return old;
}

// Floor division of a >= 0 by b > 0; `narrow` (uniform over the warp) says a and b fit in 32 bits, and then
// the division is the 32-bit one: 64-bit integer division is a long software sequence, and the producer's
// set-up runs several before its first load.
__device__ __forceinline__ long long udiv(long long a, long long b, bool narrow) {
  return narrow ? (long long)((uint32_t)a / (uint32_t)b) : a / b;
}

// CTA that owns chunk x of the line: the largest c with total*c/grid <= x.
__device__ __forceinline__ long long owner_of(long long x, long long total, long long grid, bool narrow) {
  return udiv((x + 1) * grid - 1, total, narrow);
}

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// First token attended of sequence i: ctx_start[i] rounded down to a multiple of the 16-token chunk
// (callers pass multiples of 16; anything else is recorded as an index error where it is first read).
__device__ __forceinline__ int start_of(const int32_t* starts, int i) {
  return starts ? (max(0, __ldg(starts + i)) & ~(kChunk - 1)) : 0;
}
// Tokens of sequence i the walk covers: its clamped length minus its start.
__device__ __forceinline__ int eff_len(const int32_t* lens, const int32_t* starts, int i, int cap) {
  const int L = clamp_len(__ldg(lens + i), cap), s0 = start_of(starts, i);
  return L > s0 ? L - s0 : 0;
}

// Walk length of sequence s (each lane its own s) from the lanes' registers: lane s/8, entry s%8.
__device__ __forceinline__ int reg_len(const Walker& w, int s) {
  const int src = (s >> 3) & 31, e = s & 7;
  int r = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int t = __shfl_sync(0xffffffffu, w.le[j], src);
    if (e == j) r = t;
  }
  return s >= 0 && s < w.batch ? r : 0;
}

__device__ __forceinline__ void load_window(Walker& w, int base, int lane) {
  w.win_base = base;
  const int i = base + lane;
  if (w.regs)
    w.win_len = reg_len(w, i);
  else
    w.win_len = i < w.batch ? eff_len(w.lens, w.starts, i, w.cap) : 0;
}

// Sequence b holding chunk x of the line (x < total) and pre = chunks of all sequences before it.
// Warp-cooperative scan over the lengths, 256 per pass.
__device__ __forceinline__ void find_seq(const Walker& w, long long x, int lane, int& fb, long long& fpre) {
  long long run = 0;
  fb = -1;
  fpre = 0;
  if (w.regs) {  // the same search over the register-held lengths: no loads, one ballot
    long long pre = w.lane_pre;
    int found = -1;
    long long found_pre = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int v = (w.le[j] + kChunk - 1) / kChunk;
      if (v > 0 && pre * w.hkv <= x && x < (pre + v) * w.hkv) {
        found = lane * 8 + j;
        found_pre = pre;
      }
      pre += v;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, found >= 0);
    if (hit) {
      const int src = __ffs(hit) - 1;
      fb = __shfl_sync(0xffffffffu, found, src);
      fpre = __shfl_sync(0xffffffffu, found_pre, src);
    }
    return;
  }
  for (int base = 0; base < w.batch; base += 256) {
    int v[8];
    long long s = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = base + lane * 8 + j;
      v[j] = i < w.batch ? (eff_len(w.lens, w.starts, i, w.cap) + kChunk - 1) / kChunk : 0;
      s += v[j];
    }
    const long long incl = warp_incl_scan_ll(s, lane);
    long long pre = run + incl - s;
    int found = -1;
    long long found_pre = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (v[j] > 0 && pre * w.hkv <= x && x < (pre + v[j]) * w.hkv) {
        found = base + lane * 8 + j;
        found_pre = pre;
      }
      pre += v[j];
    }
    const unsigned hit = __ballot_sync(0xffffffffu, found >= 0);
    if (hit) {
      const int src = __ffs(hit) - 1;
      fb = __shfl_sync(0xffffffffu, found, src);
      fpre = __shfl_sync(0xffffffffu, found_pre, src);
      return;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Start walking chunks [x, end) from the segment that holds x (sequence b, pre chunks before it).
__device__ __forceinline__ void walker_seek(Walker& w, long long x, long long end, int b, long long pre, int lane) {
  if (b < w.win_base || b >= w.win_base + 32) load_window(w, b, lane);
  w.b = b;
  w.L = __shfl_sync(0xffffffffu, w.win_len, b - w.win_base);
  w.nch = (w.L + kChunk - 1) / kChunk;
  w.g = (int)udiv(x - pre * w.hkv, w.nch, w.narrow);
  w.seg_start = pre * w.hkv + (long long)w.g * w.nch;
  w.pos = x;
  w.piece_start = x;
  w.end = end;
}

__device__ __forceinline__ void walker_push(Walker& w, long long start, long long end, int b, long long pre) {
  if (w.nq == 0) {
    w.q0_start = start; w.q0_end = end; w.q0_b = b; w.q0_pre = pre;
  } else {
    w.q1_start = start; w.q1_end = end; w.q1_b = b; w.q1_pre = pre;
  }
  ++w.nq;
}

// Move to the next sequence with at least one chunk (b must stay < batch while chunks remain).
__device__ __forceinline__ void next_sequence(Walker& w, int lane) {
  for (;;) {
    w.b += 1;
    if (w.b >= w.batch) return;
    if (w.b - w.win_base >= 32) load_window(w, w.b, lane);
    w.L = __shfl_sync(0xffffffffu, w.win_len, w.b - w.win_base);
    w.nch = (w.L + kChunk - 1) / kChunk;
    if (w.nch > 0) return;
  }
}

template <int CPS>
__device__ __forceinline__ StageMeta walker_next(Walker& w, int cta, int lane) {
  StageMeta d;
  if (w.pos >= w.end && w.nq > 0) {  // next sub-range
    walker_seek(w, w.q0_start, w.q0_end, w.q0_b, w.q0_pre, lane);
    w.q0_start = w.q1_start; w.q0_end = w.q1_end; w.q0_b = w.q1_b; w.q0_pre = w.q1_pre;
    --w.nq;
  }
  if (w.pos >= w.end) {
    d.flags = F_END;
    d.b = d.g = d.tok0 = d.ntok = d.vid = d.c0 = d.npieces = 0;
    return d;
  }
  const long long seg_end = w.seg_start + w.nch;
  const long long piece_end = seg_end < w.end ? seg_end : w.end;
  long long stop = w.pos + CPS;
  if (stop > piece_end) stop = piece_end;
  d.b = w.b;
  d.g = w.g;
  d.tok0 = (int)(w.pos - w.seg_start) * kChunk;
  const int tok1 = min((int)(stop - w.seg_start) * kChunk, w.L);
  d.ntok = tok1 - d.tok0;
  d.vid = w.vid;
  d.flags = (w.pos == w.piece_start ? F_FIRST : 0) | (stop == piece_end ? F_LAST : 0) |
            (w.piece_start == w.seg_start && piece_end == seg_end ? F_DIRECT : 0);
  d.c0 = w.vid;
  d.npieces = 1;
  if ((d.flags & F_LAST) && !(d.flags & F_DIRECT)) {
    const long long c0 = owner_of(w.seg_start, w.total, w.grid, w.narrow);
    const long long c1 = owner_of(seg_end - 1, w.total, w.grid, w.narrow);
    int n = (int)(c1 - c0 + 1);
    if (w.total < w.grid) {  // some CTAs have an empty range and hold no piece
      n = 0;
      for (long long c = c0; c <= c1; ++c)
        n += (udiv(w.total * c, w.grid, w.narrow) != udiv(w.total * (c + 1), w.grid, w.narrow));
    }
    d.c0 = (int)c0;
    d.npieces = n;
  }
  w.pos = stop;
  if (stop == piece_end && stop < w.end) {  // next piece starts a new segment
    w.piece_start = stop;
    w.seg_start = seg_end;
    if (++w.g == w.hkv) {
      w.g = 0;
      next_sequence(w, lane);
    }
  }
  return d;
}

// ------------------------------------------------------------------ decode kernel
template <int DT, int D, int G, int NW, int NSTAGES, bool MMA, bool Q8>
__global__ void __launch_bounds__((NW + 2) * 32, Q8 ? 3 : 1) decode_kernel(const __grid_constant__ CUtensorMap kmap,
                                                               const __grid_constant__ CUtensorMap vmap,
                                                               const DecodeParams p) {
  using LY = Layout<D, G, NW, NSTAGES, MMA, Q8>;
  using T = typename Elt<DT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::BAR_OFF);
  uint64_t* empty = full + NSTAGES;
  uint64_t* mfull = empty + NSTAGES;   // merge buffer j filled by the NW consumer warps
  uint64_t* mempty = mfull + 2;        // merge buffer j released by the epilogue warp
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + LY::META_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    for (int j = 0; j < 2; ++j) {  // every lane arrives, so each lane's own smem writes/reads are ordered
      mbar_init(&mfull[j], NW * 32);
      mbar_init(&mempty[j], 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ================================================= producer warp
    const int B = p.batch, Hkv = p.num_kv_heads;
    const int cap = p.max_blocks_per_seq * p.block_size;
    // pass 1: total chunks over all sequences (lane l takes sequences base + 8l .. base + 8l + 7); the
    // first 256 sequences' walk lengths and chunk prefixes stay in registers for the lookups below
    Walker w;
    w.regs = B <= kRegBatch;
    w.lane_pre = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) w.le[j] = 0;
    long long tot = 0;
    bool clamped = false;
    for (int base = 0; base < B; base += 256) {
      long long s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + lane * 8 + j;
        int Le = 0;
        if (i < B) {
          const int L = __ldg(p.context_lens + i);
          clamped |= (L < 0 || L > cap);
          int s0 = 0;
          if (p.ctx_start) {
            const int s0raw = __ldg(p.ctx_start + i);
            clamped |= (s0raw < 0 || (s0raw & (kChunk - 1)) != 0);
            s0 = max(0, s0raw) & ~(kChunk - 1);  // as start_of()
          }
          const int Lc = clamp_len(L, cap);
          Le = Lc > s0 ? Lc - s0 : 0;            // as eff_len()
        }
        if (base == 0) w.le[j] = Le;
        s += (Le + kChunk - 1) / kChunk;
      }
      const long long incl = warp_incl_scan_ll(s, lane);
      if (base == 0) w.lane_pre = incl - s;
      tot += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (clamped && cta == 0 && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    const long long C = tot * Hkv;
    if (lane == 0) *reinterpret_cast<long long*>(smem + LY::MISC_OFF) = C;  // published by the first full barrier
    const bool narrow = C * p.grid < (1LL << 32);
    const long long x0 = udiv(C * cta, p.grid, narrow), x1 = udiv(C * (cta + 1), p.grid, narrow);
    // Walk order: the first piece, then the last piece, then the whole segments between.  Only
    // those two pieces can be partial, so both halves of every segment cut between two CTAs
    // finish early and its merge overlaps the rest of the stream instead of trailing it.
    w.pos = w.end = 0;
    w.batch = B;
    w.hkv = Hkv;
    w.cap = cap;
    w.grid = p.grid;
    w.total = C;
    w.narrow = narrow;
    w.vid = cta;
    w.lens = p.context_lens;
    w.starts = p.ctx_start;
    w.win_base = -64;
    w.nq = 0;
    if (x0 < x1) {
      int b0, bl;
      long long p0, pl;
      find_seq(w, x0, lane, b0, p0);
      find_seq(w, x1 - 1, lane, bl, pl);
      walker_seek(w, x0, x1, b0, p0, lane);
      const long long s0 = w.seg_start, e0 = s0 + w.nch;
      const int Ll = w.regs ? reg_len(w, bl) : eff_len(p.context_lens, p.ctx_start, bl, cap);
      const int nl = (Ll + kChunk - 1) / kChunk;
      const long long sl = pl * Hkv + udiv(x1 - 1 - pl * Hkv, nl, narrow) * nl, el = sl + nl;
      const bool last_sep = sl > s0 && x1 < el;
      const long long first_end = e0 < x1 ? e0 : x1, mid_end = last_sep ? sl : x1;
      w.end = first_end;
      if (last_sep) walker_push(w, sl, x1, bl, pl);
      if (first_end < mid_end) {
        int bm;
        long long pm;
        find_seq(w, first_end, lane, bm, pm);
        walker_push(w, first_end, mid_end, bm, pm);
      }
    }
    // The walk runs kLookahead stages ahead of the TMA issue: each planned
    // stage's block-table entries are fetched with cp.async into the plan
    // ring, so no lookup latency sits between a freed stage and its refill.
    const int32_t* bt_all = p.block_tables;
    const int mb = p.max_blocks_per_seq, bs = p.block_size;
    const int bs_shift = __ffs(bs) - 1;  // block sizes are powers of two
    StageMeta* plan = reinterpret_cast<StageMeta*>(smem + LY::PLAN_OFF);
    int32_t* plan_phys = reinterpret_cast<int32_t*>(smem + LY::PLAN_OFF + kPlanRing * sizeof(StageMeta));
    auto plan_push = [&](int j) {
      const StageMeta dn = walker_next<LY::CPS>(w, cta, lane);
      const int slot = j % kPlanRing;
      if (lane == 0) plan[slot] = dn;
      if (!(dn.flags & F_END) && lane < stage_chunks(dn))
        cp_async4(plan_phys + slot * 8 + lane,
                  bt_all + (size_t)dn.b * mb + ((start_of(p.ctx_start, dn.b) + dn.tok0 + lane * kChunk) >> bs_shift));
      cp_async_commit();
    };
    for (int j = 0; j < kLookahead; ++j) plan_push(j);
    // The cache rows read from here on may have just been written by pa_write_kv, which lets this
    // kernel launch while it runs (programmatic dependent launch; q, the block tables and the lengths
    // are not its outputs): wait for it to complete before the first load, and before any write (an
    // earlier kernel on the stream may still be writing the same output).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // 16-bit caches: let the next programmatically launched kernel on the stream (the next step's cache
    // write, or the next decode) begin now.  It waits for this grid's completion before it touches memory
    // this grid reads or writes, and meanwhile sits beside this grid's CTAs (they leave room for it), so
    // its launch and set-up overlap this grid's tail.
    if constexpr (!Q8) asm volatile("griddepcontrol.launch_dependents;");
    if (cta == 0) {  // out = 0 (and log-sum-exp -inf) for sequences with no token to attend to
      for (int i = lane; i < B; i += 32) {
        if (eff_len(p.context_lens, p.ctx_start, i, cap) != 0) continue;
        uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) + (size_t)i * p.num_q_heads * D);
        for (int e = 0; e < p.num_q_heads * D * 2 / 16; ++e) o4[e] = make_uint4(0, 0, 0, 0);
        if (p.lse)
          for (int h = 0; h < p.num_q_heads; ++h) p.lse[(size_t)i * p.num_q_heads + h] = -INFINITY;
      }
    }
    bool ok = true;
    int k = 0;
    for (;; ++k) {
      cp_async_wait<kLookahead - 1>();  // this lane's lookups for stage k have landed
      __syncwarp();
      const StageMeta d = plan[k % kPlanRing];
      const int nchunk = stage_chunks(d);
      const int phys = lane < nchunk ? plan_phys[(k % kPlanRing) * 8 + lane] : 0;
      const int st = k % NSTAGES;
      if (k >= NSTAGES && !mbar_wait(&empty[st], ((k / NSTAGES) - 1) & 1)) {
        ok = false;
        break;
      }
      if (lane == 0) meta[st] = d;
      if (d.flags & F_END) {
        if (lane == 0) mbar_arrive(&full[st]);
        break;
      }
      const bool first = d.flags & F_FIRST;
      constexpr uint32_t kChunkBytes = kChunk * LY::ROWB * 2 + (Q8 ? 2 * kChunk * 4 : 0);  // K + V (+ scales)
      if (lane == 0)
        mbar_arrive_expect_tx(&full[st], (uint32_t)nchunk * kChunkBytes + (first ? LY::QSLOT : 0));
      __syncwarp();
      if (lane < nchunk) {
        const bool in_range = phys >= 0 && phys < p.num_blocks;
        if (!in_range) PA_RECORD_ERROR(PA_ERRBIT_INDEX);  // TMA zero-fills out of range
        const int tok = start_of(p.ctx_start, d.b) + d.tok0 + lane * kChunk;  // token of the sequence
        const int y = phys * bs + (tok & (bs - 1));
        uint8_t* kd = smem + LY::K_OFF + st * LY::STAGE_BYTES + lane * kChunk * LY::BOXB;
        uint8_t* vd = smem + LY::V_OFF + st * LY::STAGE_BYTES + lane * kChunk * LY::BOXB;
        // tensor-map columns are 16-bit units: a row of one KV head starts at column g * ROWB / 2
#pragma unroll
        for (int h = 0; h < LY::HALVES; ++h) {
          tma_load_2d(kd + h * LY::TOK * LY::BOXB, &kmap, d.g * (LY::ROWB / 2) + h * 64, y, &full[st]);
          tma_load_2d(vd + h * LY::TOK * LY::BOXB, &vmap, d.g * (LY::ROWB / 2) + h * 64, y, &full[st]);
        }
        if constexpr (Q8) {
          // the chunk's 16 scales of KV head g: one 64-byte run of [num_blocks][Hkv][block_size] (a block id
          // out of range reads block 0 instead; the error bit is set above)
          const size_t so = ((size_t)(in_range ? phys : 0) * p.num_kv_heads + d.g) * bs + (tok & (bs - 1));
          bulk_load(smem + LY::SK_OFF + (st * LY::TOK + lane * kChunk) * 4, p.k_scales + so, kChunk * 4, &full[st]);
          bulk_load(smem + LY::SV_OFF + (st * LY::TOK + lane * kChunk) * 4, p.v_scales + so, kChunk * 4, &full[st]);
        }
      }
      if (first && lane == 31) {
        const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q) +
                              ((size_t)d.b * p.num_q_heads + (size_t)d.g * G) * D * 2;
        bulk_load(smem + LY::QS_OFF + st * LY::QSLOT, qsrc, LY::QSLOT, &full[st]);
      }
      plan_push(k + kLookahead);
    }
    cp_async_wait<0>();
    // int8 caches: the same signal once every load of this CTA is issued (three int8 CTAs per SM leave no
    // registers for a waiting write kernel, and the early signal measured slower there)
    if constexpr (Q8) asm volatile("griddepcontrol.launch_dependents;");
    if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    // drain: every copy this CTA issued has landed before the warp leaves
    if (lane == 0) {
      for (int j = max(0, k - NSTAGES + 1); j < k; ++j)
        if (!mbar_wait(&full[j % NSTAGES], (j / NSTAGES) & 1)) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    }
    return;
  }

  if (warp == NW + 1) {
    // ================================================= epilogue warp
    // Per finished piece: merge the NW consumer warps' states, then write the
    // output (whole segment) or an fp32 partial.  A partial is counted (atomic
    // add after a fence, no waiting); the CTA that completes a segment's last
    // piece merges all of its partials by the log-sum-exp rule and writes the
    // output.  Only a CTA's first and last pieces can be partial, and the
    // producer walks them first, so these merges overlap the stream.
    const long long* line_total = reinterpret_cast<const long long*>(smem + LY::MISC_OFF);
    bool ok = true;
    for (int pc = 0;; ++pc) {
      const int j = pc & 1;
      if (!mbar_wait(&mfull[j], (pc >> 1) & 1)) {
        ok = false;
        break;
      }
      uint8_t* mb = smem + LY::M_OFF + j * LY::MB_BYTES;
      const float* mo = reinterpret_cast<const float*>(mb + LY::MB_O);
      const float* mml = reinterpret_cast<const float*>(mb + LY::MB_ML);
      const StageMeta d = *reinterpret_cast<const StageMeta*>(mb + LY::MB_DESC);
      if (d.flags & F_END) break;
      const bool direct = d.flags & F_DIRECT;
      const size_t slot = (size_t)d.b * p.num_kv_heads + d.g + d.vid;
      T* outp = reinterpret_cast<T*>(p.out) + ((size_t)d.b * p.num_q_heads + (size_t)d.g * G) * D;
      for (int i = lane; i < G * D; i += 32) {
        const int h = i / D, dd = i - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) M = fmaxf(M, mml[(w2 * G + h) * 2]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) {
          const float sc = fast_exp2(mml[(w2 * G + h) * 2] - M);
          num = fmaf(sc, mo[(w2 * G + h) * D + dd], num);
          den = fmaf(sc, mml[(w2 * G + h) * 2 + 1], den);
        }
        if (direct) {
          outp[i] = Elt<DT>::from_f(num / den);
          if (p.lse && dd == 0)
            p.lse[(size_t)d.b * p.num_q_heads + (size_t)d.g * G + h] = (M + __log2f(den)) * kLn2;
        } else {
          const size_t srow = slot * G + h;
          p.ws_o[srow * D + dd] = num;
          if (dd == 0) {
            p.ws_m[srow] = M;
            p.ws_l[srow] = den;
          }
        }
      }
      mbar_arrive(&mempty[j]);  // this lane is done with the buffer
      if (direct) continue;
      __threadfence();  // this piece's partial is visible device-wide before it is counted
      __syncwarp();
      const long long C_s = *line_total;
      {
        const int sg = d.b * p.num_kv_heads + d.g;
        int last = 0;
        if (lane == 0) {
          last = atomicAdd(p.ws_cnt + sg, 1) == d.npieces - 1;
          if (last) atomicExch(p.ws_cnt + sg, 0);  // leave the counter at zero for the next call
        }
        if (!__shfl_sync(0xffffffffu, last, 0)) continue;  // another CTA finishes this segment
        __threadfence();
        // CTAs holding a piece of this segment: c0, c0+1, ... (when the line has fewer chunks than
        // CTAs, some CTAs hold nothing and are skipped)
        const bool dense = C_s >= p.grid;
        const int np = d.npieces;
        auto piece_cta = [&](int n) -> long long {
          if (dense) return d.c0 + n;
          for (long long k2 = d.c0, m2 = 0;; ++k2)
            if (C_s * k2 / p.grid != C_s * (k2 + 1) / p.grid && m2++ == n) return k2;
        };
        // Normalised weight of each piece per head, w[h][n] = 2^(m_n - M) / sum_n 2^(m_n - M) l_n, with
        // lane n holding piece n (its m and l loads all independent, the max and sum by warp shuffles);
        // then out = sum_n w[h][n] o_n with the pieces' loads issued four at a time.  The merge so costs
        // a few L2 round trips, not one per piece.
        float* wts = reinterpret_cast<float*>(smem + LY::WTS_OFF);
        int* vids = reinterpret_cast<int*>(smem + LY::VIDS_OFF);
        if (np <= kMaxPieces) {
          const size_t myrow = lane < np ? ((size_t)sg + piece_cta(lane)) * G : 0;
          if (lane < np) vids[lane] = (int)(myrow / G - sg);
#pragma unroll 1
          for (int h0 = 0; h0 < G; h0 += 4) {
            float mh[4], lh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const bool on = lane < np && h0 + e < G;
              mh[e] = on ? __ldcg(p.ws_m + myrow + h0 + e) : -INFINITY;
              lh[e] = on ? __ldcg(p.ws_l + myrow + h0 + e) : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (h0 + e >= G) break;
              const float Mh = warp_max(mh[e]);
              const float w = lane < np ? fast_exp2(mh[e] - Mh) : 0.f;
              const float den = warp_sum(w * lh[e]);
              if (lane < np) wts[(h0 + e) * np + lane] = w / den;
              if (p.lse && lane == 0)
                p.lse[(size_t)d.b * p.num_q_heads + (size_t)d.g * G + h0 + e] = (Mh + __log2f(den)) * kLn2;
            }
          }
          __syncwarp();
          T* outp = reinterpret_cast<T*>(p.out) + ((size_t)d.b * p.num_q_heads + (size_t)d.g * G) * D;
#pragma unroll 1
          for (int i0 = lane * 4; i0 < G * D; i0 += 128) {
            const int h = i0 / D, dd = i0 - h * D;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
            for (int n0 = 0; n0 < np; n0 += 4) {
              float4 o4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                o4[e] = n0 + e < np ? __ldcg(reinterpret_cast<const float4*>(
                                          p.ws_o + (((size_t)sg + vids[n0 + e]) * G + h) * D + dd))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float w = n0 + e < np ? wts[h * np + n0 + e] : 0.f;
                acc.x = fmaf(w, o4[e].x, acc.x); acc.y = fmaf(w, o4[e].y, acc.y);
                acc.z = fmaf(w, o4[e].z, acc.z); acc.w = fmaf(w, o4[e].w, acc.w);
              }
            }
            uint2 pk;
            pk.x = Elt<DT>::from_f2(acc.x, acc.y);
            pk.y = Elt<DT>::from_f2(acc.z, acc.w);
            *reinterpret_cast<uint2*>(outp + i0) = pk;
          }
          __syncwarp();
        } else {  // more pieces than the weight area holds (only with far more CTAs than chunks)
          T* outp = reinterpret_cast<T*>(p.out) + ((size_t)d.b * p.num_q_heads + (size_t)d.g * G) * D;
          for (int i = lane; i < G * D; i += 32) {
            const int h = i / D, dd = i - h * D;
            float M = -INFINITY, num = 0.f, den = 0.f;
            for (int n = 0; n < np; ++n) M = fmaxf(M, __ldcg(p.ws_m + ((size_t)sg + piece_cta(n)) * G + h));
            for (int n = 0; n < np; ++n) {
              const size_t srow = ((size_t)sg + piece_cta(n)) * G + h;
              const float w = fast_exp2(__ldcg(p.ws_m + srow) - M);
              num = fmaf(w, __ldcg(p.ws_o + srow * D + dd), num);
              den = fmaf(w, __ldcg(p.ws_l + srow), den);
            }
            outp[i] = Elt<DT>::from_f(num / den);
            if (p.lse && dd == 0)
              p.lse[(size_t)d.b * p.num_q_heads + (size_t)d.g * G + h] = (M + __log2f(den)) * kLn2;
          }
        }
      }
    }
    if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    return;
  }

  // =================================================== consumer warps
  using C = typename std::conditional<
      Q8, Q8Consumer<D, G, NW, NSTAGES>,
      typename std::conditional<MMA, MmaConsumer<DT, D, G, NW, NSTAGES>,
                                CoreConsumer<DT, D, G, NW, NSTAGES>>::type>::type;
  C c;
  c.init();
  float* qf = reinterpret_cast<float*>(smem + LY::QF_OFF) + warp * G * D;
  const uint32_t qbase = smem_u32(qf);
  const uint32_t pbase = sbase + LY::P_OFF + warp * 32 * G * 4;
  bool ok = true;
  int pc = 0;  // pieces handed to the epilogue warp
  // Hand a finished piece (or the end marker) to the epilogue through merge buffer pc%2.
  auto hand_over = [&](const StageMeta& d, bool end) -> bool {
    const int j = pc & 1;
    if (pc >= 2 && !mbar_wait(&mempty[j], ((pc >> 1) - 1) & 1)) return false;
    uint8_t* mb = smem + LY::M_OFF + j * LY::MB_BYTES;
    if (!end) c.stash(reinterpret_cast<float*>(mb + LY::MB_O) + warp * G * D,
                      reinterpret_cast<float*>(mb + LY::MB_ML) + warp * G * 2, lane);
    if (warp == 0 && lane == 0) {
      StageMeta dd = d;
      if (end) dd.flags = F_END;
      *reinterpret_cast<StageMeta*>(mb + LY::MB_DESC) = dd;
    }
    mbar_arrive(&mfull[j]);
    ++pc;
    return true;
  };
  for (int k = 0;; ++k) {
    const int st = k % NSTAGES;
    if (!mbar_wait(&full[st], (k / NSTAGES) & 1)) {
      ok = false;
      break;
    }
    const StageMeta d = meta[st];
    if (d.flags & F_END) {
      ok = hand_over(d, true);
      break;
    }
    if (d.flags & F_FIRST) {
      c.init();
      if constexpr (Q8)
        c.template load_q<DT>(smem + LY::QS_OFF + st * LY::QSLOT, p.scale_log2, lane);
      else
        c.load_q(smem + LY::QS_OFF + st * LY::QSLOT, qf, p.scale_log2, lane);
    }
    const int nv = min(32, max(0, d.ntok - warp * 32));
    if (nv > 0) {
      const uint32_t kb = sbase + LY::K_OFF + st * LY::STAGE_BYTES;
      const uint32_t vb = sbase + LY::V_OFF + st * LY::STAGE_BYTES;
      if constexpr (Q8)
        c.tile(kb, vb, sbase + LY::SK_OFF + st * LY::TOK * 4, sbase + LY::SV_OFF + st * LY::TOK * 4, warp * 32, nv,
               lane);
      else if constexpr (MMA)
        c.tile(kb, vb, p.scale_log2, warp * 32, nv, lane);
      else
        c.tile(kb, vb, qbase, pbase, warp * 32, nv, lane);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    if ((d.flags & F_LAST) && !hand_over(d, false)) {
      ok = false;
      break;
    }
  }
  if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
}

// ------------------------------------------------------------------ cascade decode: the shared-prefix pass
// Sequences forked from one parent share the blocks of their common prefix (page "Nano-vLLM-Ascend:
// lightweight LLM inference framework for Ascend NPU", section 2.1: reference-counted blocks; page "Ascend
// NPU LLM inference optimisation: the vLLM-Ascend approach", section 4: block sharing for long contexts).
// Plain decode reads every shared block once per sharer.  The cascade reads it once for all of them: the
// decode kernel first attends over each sequence's private suffix (ctx_start = prefix length) and leaves
// (out, lse) per (sequence, head); then this kernel attends over the shared prefix of every group with
// the query rows of all its members at once, and merges the two parts by the log-sum-exp rule.
//
// Work: CTA (group, KV head, row tile, split) holds up to 64 query rows (member, head of the KV head's
// group) and the split's share of the prefix's 16-token chunks.  One producer warp bulk-copies the q rows
// and gathers K/V boxes through the first member's block table with TMA into a 2-stage ring; four
// consumer warps own 16 rows each and run every 64-token stage through the warp-MMA consumer (QK^T and PV
// on mma.m16n8k16, fp32 online softmax; P as its high 16-bit term, plus the low term for tiles that carry
// at least 1/16 of some row's running mass).  The pass is bound by the warp-MMA rate, so the low term's
// products are spent only where they change the result measurably.  Each CTA writes fp32 (m, l, o) per
// row; the CTA that completes a row tile's last split (atomic count, no waiting) merges the splits with
// the suffix part and writes out.

constexpr int kCasRows = 64;  // query rows per CTA (4 consumer warps x 16)

struct CascadeParams {
  const void* q;
  void* out;                   // on entry the suffix result, on exit the final result
  const float* lse_s;          // [batch][Hq] suffix log-sum-exp (natural log)
  const int32_t* block_tables;
  const int32_t* group_start;  // [num_groups + 1]
  const int32_t* seq_prefix;   // [batch] shared prefix tokens of each sequence (the group's value)
  int* cnt;                    // [num_groups * Hkv * tiles] splits done per row tile (zero between calls)
  float* pm;                   // [units * splits][kCasRows]
  float* pl;
  float* po;                   // [units * splits][kCasRows][D]
  int max_blocks_per_seq, batch, num_q_heads, num_kv_heads, block_size, num_blocks, num_groups, tiles, splits;
  float scale_log2;
};

template <int D, int NSTAGES, int CT>
struct CasLayout {
  static constexpr int TOK = CT * kChunk;  // tokens per stage (CT chunks)
  static constexpr int HALVES = D / 64;
  static constexpr int STAGE_BYTES = TOK * D * 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = NSTAGES * STAGE_BYTES;
  static constexpr int Q_OFF = 2 * NSTAGES * STAGE_BYTES;
  static constexpr int MISC_OFF = Q_OFF + kCasRows * D * 2;
  static constexpr int BAR_OFF = MISC_OFF + 16;  // full[NSTAGES], empty[NSTAGES], qbar
  static constexpr int BYTES = BAR_OFF + (2 * NSTAGES + 1) * 8;
  static constexpr int ALLOC = BYTES + 1024;
};

template <int DT, int D, int G, int NSTAGES, int CT, int MINB>
__global__ void __launch_bounds__(160, MINB) cascade_prefix_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                   const __grid_constant__ CUtensorMap vmap,
                                                                   const CascadeParams p) {
  using LY = CasLayout<D, NSTAGES, CT>;
  using T = typename Elt<DT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LY::BAR_OFF);
  uint64_t* empty = full + NSTAGES;
  uint64_t* qbar = empty + NSTAGES;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.splits;
  const int sp = blockIdx.x % S;
  const int unit = blockIdx.x / S;  // (group, KV head, row tile)
  const int rt = unit % p.tiles;
  const int kvh = (unit / p.tiles) % p.num_kv_heads;
  const int gi = unit / (p.tiles * p.num_kv_heads);
  const int gs = __ldg(p.group_start + gi), ge = __ldg(p.group_start + gi + 1);
  const int nrows = max(0, ge - gs) * G;
  const int r0 = rt * kCasRows;
  if (ge <= gs || r0 >= nrows) return;  // the same decision in every thread of the CTA
  const int P0 = __ldg(p.seq_prefix + gs);
  const int cap = p.max_blocks_per_seq * p.block_size;
  const int P = min(max(0, P0), cap) & ~(kChunk - 1);
  if (P == 0) return;  // no shared prefix: the suffix result already is the answer
  const int C = P / kChunk;
  const int c_begin = (int)((long long)C * sp / S), c_end = (int)((long long)C * (sp + 1) / S);
  const int my_tok = (c_end - c_begin) * kChunk;
  const int nstages = (my_tok + LY::TOK - 1) / LY::TOK;

  if (threadIdx.x == 0) {
    if (P0 != P || ((P0 & (kChunk - 1)) != 0)) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    for (int i = 0; i < NSTAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    mbar_init(qbar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ================================================= producer warp
    // q rows of the tile: row i = member gs + (r0+i)/G, query head kvh*G + (r0+i)%G; rows past the group
    // are zero.
    int valid = 0;
    for (int i = lane; i < kCasRows; i += 32) {
      const int rr = r0 + i;
      uint8_t* dst = smem + LY::Q_OFF + i * D * 2;
      if (rr < nrows) {
        ++valid;
      } else {
        for (int e = 0; e < D * 2 / 16; ++e) reinterpret_cast<uint4*>(dst)[e] = make_uint4(0, 0, 0, 0);
      }
    }
    for (int o = 16; o > 0; o >>= 1) valid += __shfl_xor_sync(0xffffffffu, valid, o);
    __syncwarp();
    if (lane == 0) mbar_arrive_expect_tx(qbar, (uint32_t)valid * D * 2);
    __syncwarp();
    for (int i = lane; i < kCasRows; i += 32) {
      const int rr = r0 + i;
      if (rr < nrows) {
        const int b = gs + rr / G, h = kvh * G + rr % G;
        bulk_load(smem + LY::Q_OFF + i * D * 2,
                  reinterpret_cast<const uint8_t*>(p.q) + ((size_t)b * p.num_q_heads + h) * D * 2, D * 2, qbar);
      }
    }
    const int32_t* bt = p.block_tables + (size_t)gs * p.max_blocks_per_seq;
    const int bs = p.block_size;
    bool ok = true;
    // block of this lane's chunk of stage k (lanes 0..CT-1), fetched one stage ahead
    auto lookup = [&](int k) -> int {
      const int c = c_begin + k * CT + lane;
      return (lane < CT && c < c_end) ? __ldg(bt + (c * kChunk) / bs) : 0;
    };
    int phys = lookup(0);
    int k = 0;
    for (; k < nstages; ++k) {
      const int st = k % NSTAGES;
      const int next = lookup(k + 1);
      if (k >= NSTAGES && !mbar_wait(&empty[st], ((k / NSTAGES) - 1) & 1)) {
        ok = false;
        break;
      }
      const int nch = min(CT, c_end - (c_begin + k * CT));
      if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)(nch * kChunk * D * 2 * 2));
      __syncwarp();
      if (lane < nch) {
        if (phys < 0 || phys >= p.num_blocks) PA_RECORD_ERROR(PA_ERRBIT_INDEX);  // TMA zero-fills out of range
        const int tok = (c_begin + k * CT + lane) * kChunk;
        const int y = phys * bs + (tok % bs);
        uint8_t* kd = smem + LY::K_OFF + st * LY::STAGE_BYTES + lane * kChunk * 128;
        uint8_t* vd = smem + LY::V_OFF + st * LY::STAGE_BYTES + lane * kChunk * 128;
#pragma unroll
        for (int h = 0; h < LY::HALVES; ++h) {
          tma_load_2d(kd + h * LY::TOK * 128, &kmap, kvh * D + h * 64, y, &full[st]);
          tma_load_2d(vd + h * LY::TOK * 128, &vmap, kvh * D + h * 64, y, &full[st]);
        }
      }
      phys = next;
    }
    if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    // drain: every copy this CTA issued has landed before the warp leaves
    if (lane == 0) {
      if (!mbar_wait(qbar, 0)) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
      for (int j = max(0, k - NSTAGES); j < k; ++j)
        if (!mbar_wait(&full[j % NSTAGES], (j / NSTAGES) & 1)) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
    }
    return;
  }

  // =================================================== consumer warps (16 rows each)
  MmaConsumer<DT, D, 16, CT / 2, NSTAGES, false> c;  // its stage layout: CT/2 x 32 tokens; lo term on demand
  c.init();
  bool ok = mbar_wait(qbar, 0);
  if (ok) c.load_q(smem + LY::Q_OFF + warp * 16 * D * 2, nullptr, 0.f, lane);
  for (int k = 0; ok && k < nstages; ++k) {
    const int st = k % NSTAGES;
    if (!mbar_wait(&full[st], (k / NSTAGES) & 1)) {
      ok = false;
      break;
    }
    const int ntok = min(LY::TOK, my_tok - k * LY::TOK);
    const uint32_t kb = sbase + LY::K_OFF + st * LY::STAGE_BYTES;
    const uint32_t vb = sbase + LY::V_OFF + st * LY::STAGE_BYTES;
#pragma unroll
    for (int r0 = 0; r0 < LY::TOK; r0 += 32)
      if (r0 < ntok) c.tile(kb, vb, p.scale_log2, r0, min(32, ntok - r0), lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
  // ---- this split's partial (m, l, o) of the warp's 16 rows
  {
    float l0 = c.l[0], l1 = c.l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const size_t slot = (size_t)unit * S + sp;
    const int ra = warp * 16 + (lane >> 2), rb = ra + 8;
    float* po = p.po + slot * kCasRows * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int col = n * 8 + (lane & 3) * 2;
      *reinterpret_cast<float2*>(po + (size_t)ra * D + col) = make_float2(c.o[n][0], c.o[n][1]);
      *reinterpret_cast<float2*>(po + (size_t)rb * D + col) = make_float2(c.o[n][2], c.o[n][3]);
    }
    if ((lane & 3) == 0) {
      p.pm[slot * kCasRows + ra] = c.m[0];
      p.pl[slot * kCasRows + ra] = l0;
      p.pm[slot * kCasRows + rb] = c.m[1];
      p.pl[slot * kCasRows + rb] = l1;
    }
  }
  __threadfence();                // this split's partial is visible device-wide before it is counted
  named_barrier_sync(1, 128);     // all four consumer warps
  int* last_flag = reinterpret_cast<int*>(smem + LY::MISC_OFF);
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.cnt + unit, 1);
    const int last = prev == S - 1;
    if (last) atomicExch(p.cnt + unit, 0);  // leave the counter at zero for the next call
    *last_flag = last;
  }
  named_barrier_sync(1, 128);
  if (!*last_flag) return;
  __threadfence();
  // ---- merge the S splits with the suffix part: row i of the tile = (b, h)
  const float* pm = p.pm + (size_t)unit * S * kCasRows;
  const float* pl = p.pl + (size_t)unit * S * kCasRows;
  const float* po = p.po + (size_t)unit * S * kCasRows * D;
  for (int i = warp; i < kCasRows; i += 4) {
    const int rr = r0 + i;
    if (rr >= nrows) break;
    const int b = gs + rr / G, h = kvh * G + rr % G;
    const float ms = __ldg(p.lse_s + (size_t)b * p.num_q_heads + h) * kLog2e;  // suffix, log2 domain, l = 1
    float M = ms;
    for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, __ldcg(pm + (size_t)s2 * kCasRows + i));
    const float ws = fast_exp2(ms - M);  // 0 when the suffix is empty (ms = -inf)
    float den = ws;
    for (int s2 = 0; s2 < S; ++s2)
      den = fmaf(fast_exp2(__ldcg(pm + (size_t)s2 * kCasRows + i) - M), __ldcg(pl + (size_t)s2 * kCasRows + i), den);
    const float inv = 1.f / den;
    T* orow = reinterpret_cast<T*>(p.out) + ((size_t)b * p.num_q_heads + h) * D;
    for (int d0 = lane * 2; d0 < D; d0 += 64) {
      const float2 so = Elt<DT>::to_f2(*reinterpret_cast<const uint32_t*>(orow + d0));
      float a0 = ws * so.x, a1 = ws * so.y;
      for (int s2 = 0; s2 < S; ++s2) {
        const float w = fast_exp2(__ldcg(pm + (size_t)s2 * kCasRows + i) - M);
        const float2 o2 = __ldcg(reinterpret_cast<const float2*>(po + ((size_t)s2 * kCasRows + i) * D + d0));
        a0 = fmaf(w, o2.x, a0);
        a1 = fmaf(w, o2.y, a1);
      }
      *reinterpret_cast<uint32_t*>(orow + d0) = Elt<DT>::from_f2(a0 * inv, a1 * inv);
    }
  }
}

// ------------------------------------------------------------------ host side
// Consumer warps per CTA and ring depth.  16-bit cache: 2 warps (64-token stages), 2 stages, three CTAs per
// SM.  int8 cache: a 64-token stage holds half the bytes and the int8 consumer is the bound, so 3 warps
// (96-token stages), 2 stages and three CTAs per SM (nine consumer warps per SM; measured against 2 warps x 4
// stages, 4 x 2 and 4 x 3 on the Qwen and Llama shapes).
template <bool Q8>
struct Shape {
  static constexpr int NW = Q8 ? 3 : 2;
  static constexpr int NS = 2;
};

template <int D, int G, bool Q8>
constexpr int alloc_bytes() {
  return Layout<D, G, Shape<Q8>::NW, Shape<Q8>::NS, Q8 || (G >= 8), Q8>::ALLOC;
}

template <bool Q8>
int smem_per_cta_t(int D, int G) {
  switch (D * 100 + G) {
    case 6401: return alloc_bytes<64, 1, Q8>();
    case 6402: return alloc_bytes<64, 2, Q8>();
    case 6404: return alloc_bytes<64, 4, Q8>();
    case 6408: return alloc_bytes<64, 8, Q8>();
    case 6416: return alloc_bytes<64, 16, Q8>();
    case 12801: return alloc_bytes<128, 1, Q8>();
    case 12802: return alloc_bytes<128, 2, Q8>();
    case 12804: return alloc_bytes<128, 4, Q8>();
    case 12808: return alloc_bytes<128, 8, Q8>();
    case 12816: return alloc_bytes<128, 16, Q8>();
  }
  return 0;
}

int smem_per_cta(int D, int G, bool q8) { return q8 ? smem_per_cta_t<true>(D, G) : smem_per_cta_t<false>(D, G); }

struct Plan {
  int grid;
  size_t ws_bytes;
  size_t off_m, off_l, off_o;  // the piece counters sit at offset 0
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool make_plan(int batch, int Hq, int Hkv, int D, int num_partitions, bool q8, Plan* pl) {
  if (batch < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || num_partitions < 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  const int smem = smem_per_cta(D, G, q8);
  if (smem == 0) return false;
  int grid = num_partitions;
  if (grid == 0) {
    int dev = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
      per_sm = 228 * 1024;
    int occ = per_sm / (smem + 1024);
    occ = std::max(1, std::min(occ, 4));
    grid = pa::sm_count() * occ;
  }
  pl->grid = grid;
  const size_t slots = (size_t)batch * Hkv + grid;
  pl->off_m = align256((size_t)batch * Hkv * 4);
  pl->off_l = pl->off_m + align256(slots * G * 4);
  pl->off_o = pl->off_l + align256(slots * G * 4);
  pl->ws_bytes = pl->off_o + align256(slots * G * D * 4);
  return true;
}

template <int DT, int D, int G, bool Q8>
int launch(const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p, cudaStream_t st) {
  constexpr bool MMA = Q8 || G >= 8;
  constexpr int NW = Shape<Q8>::NW, NS = Shape<Q8>::NS;
  using LY = Layout<D, G, NW, NS, MMA, Q8>;
  auto kern = decode_kernel<DT, D, G, NW, NS, MMA, Q8>;
  // per instantiation and device; host threads may race to set it, which only repeats an idempotent call
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::ALLOC) != cudaSuccess)
      return PA_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  // programmatic dependent launch: may start while the preceding cache write runs (it signals
  // its dependents at entry); the producer waits for it before the first cache load
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3((NW + 2) * 32);
  cfg.dynamicSmemBytes = LY::ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, km, vm, p) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

template <int DT, int D, bool Q8>
int dispatch_g(int G, const CUtensorMap& km, const CUtensorMap& vm, const DecodeParams& p, cudaStream_t st) {
  switch (G) {
    case 1: return launch<DT, D, 1, Q8>(km, vm, p, st);
    case 2: return launch<DT, D, 2, Q8>(km, vm, p, st);
    case 4: return launch<DT, D, 4, Q8>(km, vm, p, st);
    case 8: return launch<DT, D, 8, Q8>(km, vm, p, st);
    case 16: return launch<DT, D, 16, Q8>(km, vm, p, st);
  }
  return PA_ERR_UNSUPPORTED;
}

int decode_plan_impl(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                     int num_partitions_or_0, bool q8, int* grid_out, int* max_pieces_out,
                     size_t* workspace_bytes_out) {
  if (max_context_len < 0 || !pa::valid_head_dim(head_dim)) return PA_ERR_INVALID;
  Plan pl;
  if (!make_plan(batch, num_q_heads, num_kv_heads, head_dim, num_partitions_or_0, q8, &pl)) return PA_ERR_INVALID;
  if (grid_out) *grid_out = pl.grid;
  if (max_pieces_out) *max_pieces_out = batch * num_kv_heads + pl.grid;
  if (workspace_bytes_out) *workspace_bytes_out = pl.ws_bytes;
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                              int num_partitions_or_0, int* grid_out, int* max_pieces_out,
                              size_t* workspace_bytes_out) {
  return decode_plan_impl(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions_or_0, false,
                          grid_out, max_pieces_out, workspace_bytes_out);
}

extern "C" size_t pa_decode_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                           int max_context_len, int num_partitions_or_0) {
  size_t ws = 0;
  if (decode_plan_impl(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions_or_0, false,
                       nullptr, nullptr, &ws) != PA_OK)
    return 0;
  return ws;
}

extern "C" int pa_decode_int8_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                                   int num_partitions_or_0, int* grid_out, int* max_pieces_out,
                                   size_t* workspace_bytes_out) {
  return decode_plan_impl(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions_or_0, true,
                          grid_out, max_pieces_out, workspace_bytes_out);
}

extern "C" size_t pa_decode_int8_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                                int max_context_len, int num_partitions_or_0) {
  size_t ws = 0;
  if (decode_plan_impl(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions_or_0, true,
                       nullptr, nullptr, &ws) != PA_OK)
    return 0;
  return ws;
}

namespace {

// Everything a decode call does before it enqueues work: argument checks, the plan, the kernel parameters
// and the two tensor maps.  Enqueues nothing; returns PA_OK with *launchable = false when there is nothing
// to run (batch 0).  q8: the caches are int8 codes with fp32 scales (k_scales, v_scales).
struct DecodeCall {
  DecodeParams p;
  CUtensorMap km, vm;
  int dtype, head_dim, G;
  bool q8, launchable;
};

int decode_prepare(const void* q, const void* k_cache, const void* v_cache, const float* k_scales,
                   const float* v_scales, bool q8, const int32_t* block_tables, int max_blocks_per_seq,
                   const int32_t* context_lens, int batch, int num_q_heads, int num_kv_heads, int head_dim,
                   int block_size, int num_blocks, int max_context_len, float scale, int dtype, void* workspace,
                   size_t workspace_bytes, int num_partitions_or_0, void* out, float* lse, DecodeCall* call) {
  call->launchable = false;
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks < 0 ||
      max_context_len < 0 || max_blocks_per_seq < 0 || num_partitions_or_0 < 0)
    return PA_ERR_INVALID;
  if (!pa::valid_dtype(dtype) || !pa::valid_head_dim(head_dim) || !pa::valid_block_size(block_size))
    return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID;
  const int G = num_q_heads / num_kv_heads;
  if (!pa::valid_group(G)) return PA_ERR_UNSUPPORTED;
  if (batch == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID;
  if (q8 && (!k_scales || !v_scales)) return PA_ERR_INVALID;
  if (!pa::aligned16(q) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache) || !pa::aligned16(out) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_ALIGN;
  if (q8 && (!pa::aligned16(k_scales) || !pa::aligned16(v_scales))) return PA_ERR_ALIGN;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return PA_ERR_ALIGN;
  if ((long)max_blocks_per_seq * block_size < max_context_len) return PA_ERR_INVALID;
  if (num_blocks == 0 && max_context_len > 0) return PA_ERR_INVALID;
  if ((long)num_blocks * block_size >= (1L << 31)) return PA_ERR_UNSUPPORTED;
  Plan pl;
  if (!make_plan(batch, num_q_heads, num_kv_heads, head_dim, num_partitions_or_0, q8, &pl)) return PA_ERR_INVALID;
  if (!workspace || workspace_bytes < pl.ws_bytes) return PA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PA_ERR_ALIGN;

  DecodeParams& p = call->p;
  p.q = q;
  p.out = out;
  p.k_scales = k_scales;
  p.v_scales = v_scales;
  p.lse = lse;
  p.ctx_start = nullptr;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  p.ws_cnt = reinterpret_cast<int*>(ws);
  p.ws_m = reinterpret_cast<float*>(ws + pl.off_m);
  p.ws_l = reinterpret_cast<float*>(ws + pl.off_l);
  p.ws_o = reinterpret_cast<float*>(ws + pl.off_o);
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.grid = pl.grid;
  p.scale_log2 = scale * kLog2e;

  // One tensor map per cache over the [num_blocks*block_size][Hkv*D] row view, in 16-bit units (an int8
  // row of D codes is D/2 units); boxes of 16 rows x 128 bytes (128-byte swizzle), or 16 rows x 64 bytes
  // (64-byte swizzle) for the int8 rows of head_dim 64.
  const uint64_t rows = (uint64_t)std::max(num_blocks, 1) * block_size;
  const uint64_t row_bytes = (uint64_t)num_kv_heads * head_dim * (q8 ? 1 : 2);
  const uint32_t box_bytes = (q8 && head_dim == 64) ? 64u : 128u;
  // L2 fills match one head's row: 256 bytes for a 16-bit row of head_dim 128, 128 bytes for int8 rows
  const uint32_t fill = (uint32_t)head_dim * (q8 ? 1 : 2) >= 256 ? 256u : 128u;
  if (pa::encode_2d_u16(&call->km, k_cache, row_bytes / 2, rows, row_bytes, box_bytes / 2, 16, box_bytes, fill) !=
      PA_OK)
    return PA_ERR_CUDA;
  if (pa::encode_2d_u16(&call->vm, v_cache, row_bytes / 2, rows, row_bytes, box_bytes / 2, 16, box_bytes, fill) !=
      PA_OK)
    return PA_ERR_CUDA;
  call->dtype = dtype;
  call->head_dim = head_dim;
  call->G = G;
  call->q8 = q8;
  call->launchable = true;
  return PA_OK;
}

template <bool Q8>
int decode_launch_t(const DecodeCall& c, cudaStream_t st) {
  if (c.dtype == PA_BF16)
    return c.head_dim == 128 ? dispatch_g<PA_BF16, 128, Q8>(c.G, c.km, c.vm, c.p, st)
                             : dispatch_g<PA_BF16, 64, Q8>(c.G, c.km, c.vm, c.p, st);
  return c.head_dim == 128 ? dispatch_g<PA_F16, 128, Q8>(c.G, c.km, c.vm, c.p, st)
                           : dispatch_g<PA_F16, 64, Q8>(c.G, c.km, c.vm, c.p, st);
}

int decode_launch(const DecodeCall& c, cudaStream_t st) {
  return c.q8 ? decode_launch_t<true>(c, st) : decode_launch_t<false>(c, st);
}

}  // namespace

extern "C" int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
                         float scale, int dtype, void* workspace, size_t workspace_bytes, int num_partitions_or_0,
                         void* out, void* stream) {
  DecodeCall call;
  const int s = decode_prepare(q, k_cache, v_cache, nullptr, nullptr, false, block_tables, max_blocks_per_seq,
                               context_lens, batch, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                               max_context_len, scale, dtype, workspace, workspace_bytes, num_partitions_or_0, out,
                               nullptr, &call);
  if (s != PA_OK || !call.launchable) return s;
  return decode_launch(call, (cudaStream_t)stream);
}

extern "C" int pa_decode_lse(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
                             float scale, int dtype, void* workspace, size_t workspace_bytes, int num_partitions_or_0,
                             void* out, float* lse_out, void* stream) {
  if (!lse_out && batch > 0) return PA_ERR_INVALID;
  DecodeCall call;
  const int s = decode_prepare(q, k_cache, v_cache, nullptr, nullptr, false, block_tables, max_blocks_per_seq,
                               context_lens, batch, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                               max_context_len, scale, dtype, workspace, workspace_bytes, num_partitions_or_0, out,
                               lse_out, &call);
  if (s != PA_OK || !call.launchable) return s;
  return decode_launch(call, (cudaStream_t)stream);
}

extern "C" int pa_decode_int8(const void* q, const void* k_codes, const void* v_codes, const float* k_scales,
                              const float* v_scales, const int32_t* block_tables, int max_blocks_per_seq,
                              const int32_t* context_lens, int batch, int num_q_heads, int num_kv_heads, int head_dim,
                              int block_size, int num_blocks, int max_context_len, float scale, int dtype,
                              void* workspace, size_t workspace_bytes, int num_partitions_or_0, void* out,
                              void* stream) {
  DecodeCall call;
  const int s = decode_prepare(q, k_codes, v_codes, k_scales, v_scales, true, block_tables, max_blocks_per_seq,
                               context_lens, batch, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                               max_context_len, scale, dtype, workspace, workspace_bytes, num_partitions_or_0, out,
                               nullptr, &call);
  if (s != PA_OK || !call.launchable) return s;
  return decode_launch(call, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ cascade decode (shared prefixes)
namespace {

// Prefix pass ring: stages of kCasChunks 16-token chunks, kCasStages deep, kCasMinBlocks CTAs per SM.
constexpr int kCasStages = 2;
constexpr int kCasChunks = 4;
constexpr int kCasMinBlocks = 2;

struct CascadePlan {
  Plan dec;
  size_t off_lse, off_cnt, off_pm, off_pl, off_po, total;
  int tiles, splits, units;
};

bool make_cascade_plan(int batch, int Hq, int Hkv, int D, int num_partitions, int num_groups, int max_group_size,
                       int max_prefix_len, CascadePlan* cp) {
  if (num_groups < 0 || max_group_size < 0 || max_prefix_len < 0) return false;
  if (!make_plan(batch, Hq, Hkv, D, num_partitions, false, &cp->dec)) return false;
  const int G = Hq / Hkv;
  cp->tiles = std::max(1, (max_group_size * G + kCasRows - 1) / kCasRows);
  cp->units = num_groups * Hkv * cp->tiles;
  // as many splits as keep the grid within one wave of two CTAs per SM (a partial second wave would double
  // the pass), at least one, at most one per 64-token stage of the longest prefix
  const int wave = pa::sm_count() * kCasMinBlocks;
  const int by_work = std::max(1, max_prefix_len / 64);
  cp->splits = cp->units > 0 ? std::max(1, std::min(by_work, wave / cp->units)) : 1;
  const size_t slots = (size_t)cp->units * cp->splits;
  cp->off_lse = align256(cp->dec.ws_bytes);
  cp->off_cnt = cp->off_lse + align256((size_t)batch * Hq * 4);
  cp->off_pm = cp->off_cnt + align256((size_t)cp->units * 4);
  cp->off_pl = cp->off_pm + align256(slots * kCasRows * 4);
  cp->off_po = cp->off_pl + align256(slots * kCasRows * 4);
  cp->total = cp->off_po + align256(slots * kCasRows * D * 4);
  return true;
}

template <int DT, int D, int G>
int launch_cascade(const CUtensorMap& km, const CUtensorMap& vm, const CascadeParams& cp, int grid, cudaStream_t st) {
  using LY = CasLayout<D, kCasStages, kCasChunks>;
  auto kern = cascade_prefix_kernel<DT, D, G, kCasStages, kCasChunks, kCasMinBlocks>;
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::ALLOC) != cudaSuccess)
      return PA_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  kern<<<grid, 160, LY::ALLOC, st>>>(km, vm, cp);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int DT, int D>
int dispatch_cascade(int G, const CUtensorMap& km, const CUtensorMap& vm, const CascadeParams& cp, int grid,
                     cudaStream_t st) {
  switch (G) {
    case 1: return launch_cascade<DT, D, 1>(km, vm, cp, grid, st);
    case 2: return launch_cascade<DT, D, 2>(km, vm, cp, grid, st);
    case 4: return launch_cascade<DT, D, 4>(km, vm, cp, grid, st);
    case 8: return launch_cascade<DT, D, 8>(km, vm, cp, grid, st);
    case 16: return launch_cascade<DT, D, 16>(km, vm, cp, grid, st);
  }
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" size_t pa_decode_cascade_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                                   int max_context_len, int num_partitions_or_0, int num_groups,
                                                   int max_group_size, int max_prefix_len) {
  if (max_context_len < 0 || !pa::valid_head_dim(head_dim)) return 0;
  CascadePlan cp;
  if (!make_cascade_plan(batch, num_q_heads, num_kv_heads, head_dim, num_partitions_or_0, num_groups, max_group_size,
                         max_prefix_len, &cp))
    return 0;
  return cp.total;
}

extern "C" int pa_decode_cascade(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                 int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                                 int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_context_len,
                                 float scale, int dtype, int num_groups, const int32_t* group_start,
                                 const int32_t* seq_prefix_len, int max_group_size, int max_prefix_len,
                                 void* workspace, size_t workspace_bytes, int num_partitions_or_0, void* out,
                                 void* stream) {
  if (num_groups < 0 || max_group_size < 0 || max_prefix_len < 0 || max_prefix_len > max_context_len)
    return PA_ERR_INVALID;
  if (batch > 0 && (!seq_prefix_len || (num_groups > 0 && !group_start))) return PA_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(seq_prefix_len) & 3u) || (reinterpret_cast<uintptr_t>(group_start) & 3u))
    return PA_ERR_ALIGN;
  if (num_groups > batch || (num_groups > 0 && max_group_size < 1)) return PA_ERR_INVALID;
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads) return PA_ERR_INVALID;
  CascadePlan cp;
  if (!make_cascade_plan(batch, num_q_heads, num_kv_heads, head_dim, num_partitions_or_0, num_groups, max_group_size,
                         max_prefix_len, &cp))
    return PA_ERR_INVALID;
  if (workspace && workspace_bytes < cp.total) return PA_ERR_WORKSPACE;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  DecodeCall call;
  int s = decode_prepare(q, k_cache, v_cache, nullptr, nullptr, false, block_tables, max_blocks_per_seq, context_lens,
                         batch, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, max_context_len, scale,
                         dtype, workspace, workspace ? cp.dec.ws_bytes : 0, num_partitions_or_0, out,
                         ws ? reinterpret_cast<float*>(ws + cp.off_lse) : nullptr, &call);
  if (s != PA_OK || !call.launchable) return s;
  // pass 1: every sequence's private suffix (tokens from its prefix length on), with its log-sum-exp
  call.p.ctx_start = seq_prefix_len;
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = decode_launch(call, st)) != PA_OK) return s;
  if (num_groups == 0 || max_prefix_len < kChunk) return PA_OK;
  // pass 2: the shared prefix of every group, once for all of its members, merged with pass 1; on the
  // CTA-pair tensor-core kernel at head_dim 128, on warp MMA otherwise
  if (head_dim == 128)
    return pa::prefix_pass_pairs(q, k_cache, v_cache, block_tables, max_blocks_per_seq, num_groups, group_start,
                                 seq_prefix_len, max_group_size, reinterpret_cast<const float*>(ws + cp.off_lse),
                                 num_q_heads, num_kv_heads, block_size, num_blocks, scale, dtype, out, st);
  CascadeParams c;
  c.q = q;
  c.out = out;
  c.lse_s = reinterpret_cast<const float*>(ws + cp.off_lse);
  c.block_tables = block_tables;
  c.group_start = group_start;
  c.seq_prefix = seq_prefix_len;
  c.cnt = reinterpret_cast<int*>(ws + cp.off_cnt);
  c.pm = reinterpret_cast<float*>(ws + cp.off_pm);
  c.pl = reinterpret_cast<float*>(ws + cp.off_pl);
  c.po = reinterpret_cast<float*>(ws + cp.off_po);
  c.max_blocks_per_seq = max_blocks_per_seq;
  c.batch = batch;
  c.num_q_heads = num_q_heads;
  c.num_kv_heads = num_kv_heads;
  c.block_size = block_size;
  c.num_blocks = num_blocks;
  c.num_groups = num_groups;
  c.tiles = cp.tiles;
  c.splits = cp.splits;
  c.scale_log2 = scale * kLog2e;
  const int grid = cp.units * cp.splits;
  if (dtype == PA_BF16)
    return head_dim == 128 ? dispatch_cascade<PA_BF16, 128>(call.G, call.km, call.vm, c, grid, st)
                           : dispatch_cascade<PA_BF16, 64>(call.G, call.km, call.vm, c, grid, st);
  return head_dim == 128 ? dispatch_cascade<PA_F16, 128>(call.G, call.km, call.vm, c, grid, st)
                         : dispatch_cascade<PA_F16, 64>(call.G, call.km, call.vm, c, grid, st);
}

// ------------------------------------------------------------------ decode with library-owned scratch
// Some callers cannot allocate device memory at the point where they run
// decode: code that runs while a CUDA graph is being captured (cudaMalloc is
// not allowed there), engines that hand out memory only from a pool fixed at
// start-up, or hosts that forbid allocation on the serving path because an
// allocation can block on the device.  For them the scratch lives in a static
// array of this file, set aside once per GPU when the library is loaded.
static __device__ __align__(256) unsigned char g_decode_scratch[PA_DECODE_STATIC_SCRATCH_BYTES];

namespace {

// Device address of g_decode_scratch on the current device, looked up once per
// device (the array's host-side name is not a device address).
int static_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_static_scratch(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int batch, int num_q_heads, int num_kv_heads,
                                        int head_dim, int block_size, int num_blocks, int max_context_len, float scale,
                                        int dtype, int num_partitions_or_0, void* out, void* stream) {
  // A plan larger than the static scratch is refused first, whatever the other arguments.
  size_t need = 0;
  int s = pa_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions_or_0, nullptr,
                         nullptr, &need);
  if (s != PA_OK) return s;
  if (need > PA_DECODE_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;  // batch too large for the static scratch
  void* scratch = nullptr;
  if ((s = static_scratch_ptr(&scratch)) != PA_OK) return s;
  // Every check pa_decode makes, before anything is enqueued: a rejected call leaves the stream and the
  // scratch untouched.
  DecodeCall call;
  s = decode_prepare(q, k_cache, v_cache, nullptr, nullptr, false, block_tables, max_blocks_per_seq, context_lens,
                     batch, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, max_context_len, scale, dtype,
                     scratch, PA_DECODE_STATIC_SCRATCH_BYTES, num_partitions_or_0, out, nullptr, &call);
  if (s != PA_OK || !call.launchable) return s;
  // The head of the scratch holds the per-segment piece counters, which must start at zero.  A completed
  // call leaves them at zero, but they are cleared anyway so that an earlier call that gave up (a timed-out
  // wait) cannot leak into this one.  The clear is a stream operation between the preceding kernel and the
  // decode kernel, so on this entry point decode does not start early under a preceding pa_write_kv.
  if (cudaMemsetAsync(scratch, 0, (size_t)batch * num_kv_heads * sizeof(int), (cudaStream_t)stream) != cudaSuccess)
    return PA_ERR_CUDA;
  return decode_launch(call, (cudaStream_t)stream);
}
