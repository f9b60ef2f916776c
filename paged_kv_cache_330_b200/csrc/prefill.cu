// Chunked prefill attention over the paged cache, tcgen05 / TMEM / TMA (sm_100a).
//
// What it computes (page "In-depth analysis of vllm-ascend: LLM inference
// architecture on Ascend hardware", section 1.1: prefill cut into chunks on one
// device; page "Nano-vLLM-Ascend: lightweight LLM inference framework for
// Ascend NPU", sections 2.1 and 2.2.1: block table, softmax(q k^T/sqrt(d)) v):
// sequence b appends C_b query tokens whose K/V are already in the cache, so
// that it now holds L_b tokens; query i sits at position p = L_b - C_b + i and
//   out[i][h] = sum_{t <= p} softmax_t(scale <q[i][h], K_b[t][h/G]>) V_b[t][h/G].
//
// One CTA per (128 query rows, query head, sequence).  Keys are walked in
// tiles of 128 (the only dense contraction on the path, so it runs on the
// 5th-generation tensor cores):
//   * a TMA producer warp loads the Q tile once and, per key tile, 16-row K
//     and V boxes gathered through the block table (128-byte swizzle, no
//     multicast) into a two-stage ring;
//   * one thread of the MMA warp issues S = Q K^T (M 128, N 128, K 128) into
//     one of two TMEM buffers and O += P V into a TMEM accumulator
//     (tcgen05.mma kind::f16, fp32 accumulate), completions signalled with
//     tcgen05.commit on mbarriers;
//   * four softmax warps (thread r = query row r = TMEM lane r) read S with
//     tcgen05.ld, apply the causal mask, keep fp32 running max / sum (the
//     vLLM-Ascend page, section 3.1, keeps softmax out of fp16), rescale O in
//     TMEM only when the running max grows by more than 2^8 (exact: O and the
//     sum always share the same reference max), and write P as bf16/f16 into
//     shared memory in the operand layout.  A key tile in which some row gets
//     at least 1/16 of its running mass (always the first tile, and tiles
//     with dominant keys) issues P as two 16-bit terms (hi + lo), exact to
//     ~2^-17; other tiles use one term, whose rounding then moves each output
//     by at most 2^-9 |v| / 16.
// S is double-buffered so S_{j+1} = Q K_{j+1}^T runs while the softmax warps
// work on tile j.

#include <algorithm>

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_prefill)

namespace {

using namespace pa;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int BM = 128;                 // query rows per CTA (TMEM lanes)
constexpr int BN = 128;                 // keys per tile
constexpr int HD = 128;                 // head_dim
constexpr int kStages = 2;              // K/V ring depth
constexpr float kRescaleLog2 = 8.f;     // rescale O only when the max grows by more than 2^8
// A key tile whose P carries at least 1/16 of some row's running softmax mass also issues P's low
// 16-bit term: its one-term rounding error (2^-9 relative) would otherwise reach ~2^-9 |v| of that
// row's output.  The first tile always qualifies (it holds all the mass so far).
constexpr float kLoFraction = 1.f / 16.f;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int TILE_HALF = BM * 128;                     // 128 rows x 128 bytes = 16 KB (64 columns)
constexpr int TILE = 2 * TILE_HALF;                     // 128 x 128 16-bit values = 32 KB
constexpr int Q_OFF = 0;
constexpr int K_OFF = Q_OFF + TILE;
constexpr int V_OFF = K_OFF + kStages * TILE;
constexpr int P_OFF = V_OFF + kStages * TILE;    // P, high 16-bit term
constexpr int PL_OFF = P_OFF + TILE;             // P, low 16-bit term (tiles that need it)
constexpr int BAR_OFF = PL_OFF + TILE;
// barriers: q_full, k_full[2], v_full[2], kv_empty[2], s_full[2], s_free[2], p_full, o_done
constexpr int NBAR = 1 + 2 * kStages + kStages + 2 + 2 + 2;
constexpr int TMEM_SLOT_OFF = BAR_OFF + NBAR * 8;
constexpr int LOFLAG_OFF = TMEM_SLOT_OFF + 4;    // int [2]: tile index + 1 when that tile needs the low term
constexpr int SMEM_BYTES = LOFLAG_OFF + 8 + 4;
static_assert(SMEM_BYTES + 1024 <= 232448, "shared memory budget");
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

constexpr int TMEM_COLS = 512;  // S0 [0,128), S1 [128,256), O [256,384)
constexpr int O_COL = 256;

struct PrefillParams {
  void* out;
  const int32_t* query_start_loc;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int max_blocks_per_seq;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int mtiles;         // ceil(max_chunk_len / BM)
  float scale_log2;
};

// --------------------------------------------------------------- tcgen05 helpers
// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand (rows of 128 bytes, 8-row groups 1024 bytes apart): k-step ks of 16 elements.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  return sdesc(tile + (ks >> 2) * TILE_HALF + (ks & 3) * 32, 16, 1024);
}
// MN-major operand (V: key rows of 128 bytes = 64 head_dim values; the two 64-column halves
// 16 KB apart): k-step ks covers keys 16*ks .. 16*ks+15.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int ks) {
  return sdesc(tile + ks * 16 * 128, TILE_HALF, 1024);
}
// Instruction descriptor, kind::f16: fp32 accumulate, A/B 16-bit (0 = f16, 1 = bf16), M 128, N 128.
__host__ __device__ constexpr uint32_t idesc(int fmt, bool b_mn_major) {
  return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(id), "r"(accumulate), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// Byte offset of (row r, column c) in a 128 x 128 tile stored as two 64-column halves with the
// 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (c >> 6) * TILE_HALF + r * 128 + ((((c >> 3) & 7) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

// --------------------------------------------------------------- kernel
template <int DT>
__global__ void __launch_bounds__(192, 1) prefill_kernel(const __grid_constant__ CUtensorMap qmap,
                                                          const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap,
                                                          const PrefillParams p) {
  using T = typename Elt<DT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStages;
  uint64_t* kv_empty = v_full + kStages;
  uint64_t* s_full = kv_empty + kStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + TMEM_SLOT_OFF);
  volatile int* lo_flag = reinterpret_cast<volatile int*>(smem + LOFLAG_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.num_q_heads / p.num_kv_heads;
  // CTA -> (query head, m-tile, sequence); the G heads of a KV group are adjacent so their K/V
  // tiles are read from L2 by neighbouring CTAs.
  int u = blockIdx.x;
  const int j_in_group = u % G;
  u /= G;
  const int mt = u % p.mtiles;
  u /= p.mtiles;
  const int g = u % p.num_kv_heads;
  const int b = u / p.num_kv_heads;
  const int h = g * G + j_in_group;

  const int q0 = __ldg(p.query_start_loc + b), q1 = __ldg(p.query_start_loc + b + 1);
  const int C = q1 - q0;
  const int m0 = mt * BM;
  if (m0 >= C) return;
  int L = __ldg(p.context_lens + b);
  const int cap = p.max_blocks_per_seq * p.block_size;
  if (L > cap || L < C) {  // broken caller invariant: record and produce nothing for this tile
    if (threadIdx.x == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    return;
  }
  const int pos0 = L - C + m0;                              // position of this tile's first query row
  const int kend = min(L, pos0 + BM);                       // keys [0, kend) are visible to some row
  const int nkv = (kend + BN - 1) / BN;

  if (threadIdx.x == 0) {
    lo_flag[0] = lo_flag[1] = 0;
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], BM);
    }
    mbar_init(p_full, BM);
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  if (warp == 5) {  // TMEM: S0, S1, O
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 4) {
    // ============================================ producer: Q once, then K/V tiles through the block table
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      mbar_arrive_expect_tx(q_full, TILE);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_2d(smem + Q_OFF + hf * TILE_HALF, &qmap, h * HD + hf * 64, q0 + m0, q_full);
    }
    const int32_t* bt = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    auto lookup = [&](int j) -> int {
      const int key = j * BN + lane * 16;
      return (j < nkv && lane < 8 && key < kend) ? __ldg(bt + key / p.block_size) : 0;
    };
    int phys = lookup(0);
    for (int j = 0; j < nkv && ok; ++j) {
      const int st = j % kStages;
      if (j >= kStages && !mbar_wait(&kv_empty[st], ((j / kStages) - 1) & 1)) {
        ok = false;
        break;
      }
      const int nbox = min(8, (kend - j * BN + 15) / 16);
      if (lane == 0) {
        mbar_arrive_expect_tx(&k_full[st], nbox * 16 * HD * 2);
        mbar_arrive_expect_tx(&v_full[st], nbox * 16 * HD * 2);
      }
      __syncwarp();
      if (lane < nbox) {
        if (phys < 0 || phys >= p.num_blocks) PA_RECORD_ERROR(PA_ERRBIT_INDEX);  // TMA zero-fills out of range
        const int key = j * BN + lane * 16;
        const int y = phys * p.block_size + key % p.block_size;
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_2d(smem + K_OFF + st * TILE + hf * TILE_HALF + lane * 16 * 128, &kmap, g * HD + hf * 64, y,
                      &k_full[st]);
          tma_load_2d(smem + V_OFF + st * TILE + hf * TILE_HALF + lane * 16 * 128, &vmap, g * HD + hf * 64, y,
                      &v_full[st]);
        }
      }
      phys = lookup(j + 1);
    }
  } else if (warp == 5) {
    // ============================================ MMA issuer (one thread issues; the warp zeroes V tails)
    const uint32_t id_s = idesc(DT == PA_BF16 ? 1 : 0, false);
    const uint32_t id_pv = idesc(DT == PA_BF16 ? 1 : 0, true);
    auto issue_pv = [&](int i) -> bool {
      const int st = i % kStages;
      if (!mbar_wait(&v_full[st], (i / kStages) & 1)) return false;
      const int valid = kend - i * BN;
      if (valid < BN) {  // keys past the end: zero their V rows (their bytes may be anything, even NaN)
        for (int idx = lane; idx < (BN - valid) * 16; idx += 32) {
          const int r = valid + idx / 16, c = (idx % 16) * 8;
          sts128(sb + V_OFF + st * TILE + tile_off(r, c), 0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (!mbar_wait(p_full, i & 1)) return false;
      tc_fence_after();
      const bool lo = lo_flag[i & 1] == i + 1;
      if (lane == 0) {
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_f16(tmem + O_COL, kmajor_desc(sb + P_OFF, ks), mnmajor_desc(sb + V_OFF + st * TILE, ks), id_pv,
                  (i > 0 || ks > 0) ? 1u : 0u);
        if (lo)
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_f16(tmem + O_COL, kmajor_desc(sb + PL_OFF, ks), mnmajor_desc(sb + V_OFF + st * TILE, ks), id_pv, 1u);
        mma_commit(o_done);
        mma_commit(&kv_empty[st]);
      }
      __syncwarp();
      return true;
    };
    if (!mbar_wait(q_full, 0)) ok = false;
    for (int j = 0; j < nkv && ok; ++j) {
      const int st = j % kStages, s2 = j & 1;
      if (!mbar_wait(&k_full[st], (j / kStages) & 1) || (j >= 2 && !mbar_wait(&s_free[s2], ((j >> 1) - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        for (int ks = 0; ks < HD / 16; ++ks)
          mma_f16(tmem + s2 * BN, kmajor_desc(sb + Q_OFF, ks), kmajor_desc(sb + K_OFF + st * TILE, ks), id_s,
                  ks > 0 ? 1u : 0u);
        mma_commit(&s_full[s2]);
      }
      __syncwarp();
      if (j >= 1 && !issue_pv(j - 1)) ok = false;
    }
    if (ok && !issue_pv(nkv - 1)) ok = false;
  } else {
    // ============================================ softmax warps: thread r owns query row m0 + r
    const int r = threadIdx.x;
    const int pos = pos0 + r;                                 // this row's position (keys 0..pos visible)
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lane quarter
    float m_ref = -INFINITY;                                  // reference max (log2 units) shared by O and l
    float l = 0.f;
    float s[BN];
    for (int j = 0; j < nkv && ok; ++j) {
      const int s2 = j & 1;
      if (!mbar_wait(&s_full[s2], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BN; c += 32) tmem_ld32(tmem + lane_base + s2 * BN + c, s + c);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[s2]);
      // causal mask: key k visible iff k <= pos (and k < L)
      const int k0 = j * BN;
      const int lim = min(pos, L - 1) - k0;  // last visible column of this tile
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        s[c] = c <= lim ? s[c] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleLog2 || m_ref == -INFINITY) {
        alpha = m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - mx);
        rescale = m_ref != -INFINITY;
        m_ref = mx;
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        s[c] = fast_exp2(s[c] - m_ref);
        rs += s[c];
      }
      l = l * alpha + rs;
      // does this tile carry a large share of some row's mass?  (CTA-wide decision: tile j needs
      // the low term iff lo_flag[j&1] == j+1 after the softmax warps have all voted)
      if (__any_sync(0xffffffffu, rs >= kLoFraction * l) && lane == 0) lo_flag[j & 1] = j + 1;
      named_barrier_sync(1, BM);
      const bool lo = lo_flag[j & 1] == j + 1;
      // the previous tile's PV must be done (P buffers free, O complete) before we touch either
      if (j > 0 && !mbar_wait(o_done, (j - 1) & 1)) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + O_COL + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tmem + lane_base + O_COL + c, o);
        }
        tmem_wait_st();
      }
#pragma unroll
      for (int c = 0; c < BN; c += 8) {
        uint32_t w[4], wl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = s[c + 2 * e], bb = s[c + 2 * e + 1];
          w[e] = Elt<DT>::from_f2(a, bb);
          const float2 hv = Elt<DT>::to_f2(w[e]);
          wl[e] = Elt<DT>::from_f2(a - hv.x, bb - hv.y);
        }
        sts128(sb + P_OFF + tile_off(r, c), w[0], w[1], w[2], w[3]);
        if (lo) sts128(sb + PL_OFF + tile_off(r, c), wl[0], wl[1], wl[2], wl[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // epilogue: O / l -> out
    if (ok && mbar_wait(o_done, (nkv - 1) & 1)) {
      tc_fence_after();
      const int row = m0 + r;
      T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(q0 + row) * p.num_q_heads + h) * HD;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + O_COL + c, o);
        tmem_wait_ld();
        if (row < C) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v;
            v.x = Elt<DT>::from_f2(o[e] * inv, o[e + 1] * inv);
            v.y = Elt<DT>::from_f2(o[e + 2] * inv, o[e + 3] * inv);
            v.z = Elt<DT>::from_f2(o[e + 4] * inv, o[e + 5] * inv);
            v.w = Elt<DT>::from_f2(o[e + 6] * inv, o[e + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c + e) = v;
          }
        }
      }
    } else {
      ok = false;
    }
  }
  if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

int encode_q_map(CUtensorMap* map, const void* q, int total_q, int Hq) {
  return pa::encode_2d_sw128(map, q, (uint64_t)Hq * HD, (uint64_t)std::max(total_q, 1), (uint64_t)Hq * HD * 2, 64,
                             BM);
}

}  // namespace

extern "C" int pa_prefill_chunk(const void* q, const int32_t* query_start_loc, int total_q_tokens, int max_chunk_len,
                                const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens, int batch, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, int dtype,
                                void* out, void* stream) {
  if (batch < 0 || total_q_tokens < 0 || max_chunk_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      num_blocks < 0 || max_blocks_per_seq < 0)
    return PA_ERR_INVALID;
  if (!pa::valid_dtype(dtype) || head_dim != HD || !pa::valid_block_size(block_size)) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads) return PA_ERR_INVALID;
  if (!pa::valid_group(num_q_heads / num_kv_heads)) return PA_ERR_UNSUPPORTED;
  if (batch == 0 || total_q_tokens == 0 || max_chunk_len == 0) return PA_OK;
  if (!q || !query_start_loc || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID;
  if (!pa::aligned16(q) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache) || !pa::aligned16(out) ||
      (reinterpret_cast<uintptr_t>(query_start_loc) & 3u) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_ALIGN;
  if (num_blocks == 0) return PA_ERR_INVALID;
  if ((long)num_blocks * block_size >= (1L << 31)) return PA_ERR_UNSUPPORTED;
  const int mtiles = (max_chunk_len + BM - 1) / BM;
  const long grid = (long)batch * num_kv_heads * mtiles * (num_q_heads / num_kv_heads);
  if (grid > 0x7fffffffL) return PA_ERR_UNSUPPORTED;

  PrefillParams p;
  p.out = out;
  p.query_start_loc = query_start_loc;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.mtiles = mtiles;
  p.scale_log2 = scale * kLog2e;

  CUtensorMap qm, km, vm;
  const uint64_t rows = (uint64_t)num_blocks * block_size;
  const uint64_t cols = (uint64_t)num_kv_heads * HD;
  if (encode_q_map(&qm, q, total_q_tokens, num_q_heads) != PA_OK) return PA_ERR_CUDA;
  if (pa::encode_2d_sw128(&km, k_cache, cols, rows, cols * 2, 64, 16) != PA_OK) return PA_ERR_CUDA;
  if (pa::encode_2d_sw128(&vm, v_cache, cols, rows, cols * 2, 64, 16) != PA_OK) return PA_ERR_CUDA;

  auto kern = dtype == PA_BF16 ? prefill_kernel<PA_BF16> : prefill_kernel<PA_F16>;
  static bool attr_set[2][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const int di = dtype == PA_BF16 ? 1 : 0;
  if (dev < 0 || dev >= 64 || !attr_set[di][dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) != cudaSuccess)
      return PA_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[di][dev] = true;
  }
  kern<<<(unsigned)grid, 192, SMEM_ALLOC, (cudaStream_t)stream>>>(qm, km, vm, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
