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
// This is the one dense contraction on the path, so it runs on the
// 5th-generation tensor cores.  One CTA owns two 128-row query tiles that read
// the same keys: two query heads of one KV group over the same rows (or, when
// a group has one head, two consecutive row tiles of it).  Keys are walked in
// tiles of 64:
//   * a TMA producer warp loads both query tiles once and, per key tile, 16-row
//     K and V boxes gathered through the block table (128-byte swizzle, no
//     multicast) into separate three-stage K and V rings shared by both query
//     tiles (a K slot frees after the S products, a V slot after the PVs, so
//     K runs ahead);
//   * one thread of the MMA warp issues, per key tile, S_t = Q_t K^T for both
//     query tiles (M 128, N 64, K 128) into per-tile double-buffered TMEM, then
//     O_t += P_t V for the previous key tile (M 128, N 128, K 64), with fp32
//     accumulation (tcgen05.mma kind::f16) and completions signalled with
//     tcgen05.commit on mbarriers;
//   * two softmax warpgroups, one per query tile (thread r = row r = TMEM lane
//     r), read S with tcgen05.ld, apply the causal mask, keep fp32 running max
//     and sum (the vLLM-Ascend page, section 3.1, keeps softmax out of fp16),
//     rescale O in TMEM only when the running max grows by more than 2^8
//     (exact: O and the sum always share one reference max), and write P in
//     the operand layout into shared memory.  A key tile in which some row of
//     the tile gets at least 1/16 of its running mass (always the first one,
//     and tiles with dominant keys) also issues P's low 16-bit term, exact to
//     ~2^-17; elsewhere one term moves an output by at most 2^-9 |v| / 16.
// With two query tiles and double-buffered S, the tensor core always has an
// S or a PV product to run while either warpgroup is in its softmax.

#include <algorithm>

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_prefill)

namespace {

using namespace pa;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int BM = 128;                 // query rows per query tile (TMEM lanes)
constexpr int BN = 64;                  // keys per key tile
constexpr int HD = 128;                 // head_dim
constexpr int kStages = 3;              // K and V ring depth (separate rings)
constexpr float kRescaleLog2 = 8.f;     // rescale O only when the max grows by more than 2^8
constexpr float kLoFraction = 1.f / 16.f;

// shared memory map (offsets from a 1024-byte aligned base).  Operand tiles have rows of
// 128 bytes (64 16-bit values) with the 128-byte swizzle; wider tiles are split into
// 64-column "halves" placed one after the other.
constexpr int QHALF = BM * 128;                 // 16 KB: 128 rows x 64 columns
constexpr int QTILE = 2 * QHALF;                // 32 KB: 128 rows x 128 columns (head_dim)
constexpr int KVHALF = BN * 128;                // 8 KB: 64 keys x 64 columns
constexpr int KVTILE = 2 * KVHALF;              // 16 KB: 64 keys x 128 columns
constexpr int PTILE = BM * 128;                 // 16 KB: 128 rows x 64 keys
constexpr int Q_OFF = 0;                        // Q[2]
constexpr int K_OFF = Q_OFF + 2 * QTILE;        // K[kStages]
constexpr int V_OFF = K_OFF + kStages * KVTILE; // V[kStages]
constexpr int P_OFF = V_OFF + kStages * KVTILE; // P high term [2 query tiles]
constexpr int PL_OFF = P_OFF + 2 * PTILE;       // P low term [2 query tiles]
constexpr int BAR_OFF = PL_OFF + 2 * PTILE;
// barriers: q_full, k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2][2], s_free[2][2], p_full[2],
// o_done[2][2]
constexpr int NBAR = 1 + 4 * kStages + 4 + 4 + 2 + 4;
constexpr int MISC_OFF = BAR_OFF + NBAR * 8;    // tmem base (4 B), lo flags int[2][2]
constexpr int SMEM_BYTES = MISC_OFF + 4 + 16 + 12;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// TMEM columns: S_t buffers [t*128 + buf*64, +64), O_t [256 + t*128, +128)
constexpr int TMEM_COLS = 512;
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
  int units;          // query-tile pairs per (sequence, KV head)
  float scale_log2;
};

// --------------------------------------------------------------- tcgen05 helpers
// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major operand whose 64-column halves are `half` bytes apart (rows 128 bytes, 8-row groups
// 1024 bytes apart): k-step ks of 16 elements.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int half, int ks) {
  return sdesc(tile + (ks >> 2) * half + (ks & 3) * 32, 16, 1024);
}
// MN-major V tile (key rows of 128 bytes = 64 head_dim values; the two halves KVHALF apart):
// k-step ks covers keys 16*ks .. 16*ks+15.
__device__ __forceinline__ uint64_t v_desc(uint32_t tile, int ks) {
  return sdesc(tile + ks * 16 * 128, KVHALF, 1024);
}
// Instruction descriptor, kind::f16: fp32 accumulate, A/B 16-bit (0 = f16, 1 = bf16), M 128.
__host__ __device__ constexpr uint32_t idesc(int fmt, bool b_mn_major, int n) {
  return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
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

// Byte offset of (row r, 16-bit column c) in a tile of 128-byte rows split into 64-column halves
// `half` bytes apart, with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t tile_off(int r, int c, int half) {
  return (c >> 6) * half + r * 128 + ((((c >> 3) & 7) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

// --------------------------------------------------------------- kernel
template <int DT>
__global__ void __launch_bounds__(320, 1) prefill_kernel(const __grid_constant__ CUtensorMap qmap,
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
  uint64_t* k_empty = v_full + kStages;    // K slot free: both S products of its key tile are done
  uint64_t* v_empty = k_empty + kStages;   // V slot free: both PV products of its key tile are done
  uint64_t* s_full = v_empty + kStages;    // [t][buf] at s_full[t * 2 + buf]
  uint64_t* s_free = s_full + 4;           // [t][buf]
  uint64_t* p_full = s_free + 4;           // [t]
  uint64_t* o_done = p_full + 2;           // [t][key tile & 1]: O_t += P_t V of that key tile is complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* lo_flag = reinterpret_cast<volatile int*>(smem + MISC_OFF + 4);  // [t][j & 1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.num_q_heads / p.num_kv_heads;
  // CTA -> (pair unit, KV head, sequence).  G >= 2: two heads of the group over the same 128 rows;
  // G == 1: the group's single head over two consecutive 128-row tiles.
  int u = blockIdx.x;
  const int unit = u % p.units;
  u /= p.units;
  const int g = u % p.num_kv_heads;
  const int b = u / p.num_kv_heads;
  int head[2], mrow[2];
  if (G >= 2) {
    const int pair = unit % (G / 2), mt = unit / (G / 2);
    head[0] = g * G + 2 * pair;
    head[1] = head[0] + 1;
    mrow[0] = mrow[1] = mt * BM;
  } else {
    head[0] = head[1] = g;
    mrow[0] = unit * 2 * BM;
    mrow[1] = mrow[0] + BM;
  }

  const int q0 = __ldg(p.query_start_loc + b), q1 = __ldg(p.query_start_loc + b + 1);
  const int C = q1 - q0;
  if (mrow[0] >= C) return;
  const int L = __ldg(p.context_lens + b);
  const int cap = p.max_blocks_per_seq * p.block_size;
  if (L > cap || L < C) {  // broken caller invariant: record and produce nothing for this tile
    if (threadIdx.x == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    return;
  }
  // keys [0, kend) are visible to some row of either tile
  const int kend = min(L, L - C + max(mrow[0], mrow[1]) + BM);
  const int nkv = (kend + BN - 1) / BN;

  if (threadIdx.x == 0) {
    lo_flag[0] = lo_flag[1] = lo_flag[2] = lo_flag[3] = 0;
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], BM);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&p_full[t], BM);
      mbar_init(&o_done[t * 2], 1);
      mbar_init(&o_done[t * 2 + 1], 1);
    }
    fence_mbar_init();
  }
  if (warp == 9) {  // TMEM: S_0 x2, S_1 x2, O_0, O_1
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

  if (warp == 8) {
    // ============================================ producer: both Q tiles once, then K/V tiles
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      mbar_arrive_expect_tx(q_full, 2 * QTILE);
      for (int t = 0; t < 2; ++t)
        for (int hf = 0; hf < 2; ++hf)
          tma_load_2d(smem + Q_OFF + t * QTILE + hf * QHALF, &qmap, head[t] * HD + hf * 64, q0 + mrow[t], q_full);
    }
    const int32_t* bt = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    auto lookup = [&](int j) -> int {
      const int key = j * BN + lane * 16;
      return (j < nkv && lane < BN / 16 && key < kend) ? __ldg(bt + key / p.block_size) : 0;
    };
    // K and V tiles are issued as their own slots free up: K slots early (after the S products),
    // V slots late (after the PV products), so K runs ahead of V.
    int jk = 0, jv = 0;
    int physk = lookup(0), physv = physk;
    auto issue = [&](int j, int phys, uint64_t* full, const CUtensorMap* map, int off) {
      const int st = j % kStages;
      const int nbox = min(BN / 16, (kend - j * BN + 15) / 16);
      if (lane == 0) mbar_arrive_expect_tx(&full[st], nbox * 16 * HD * 2);
      __syncwarp();
      if (lane < nbox) {
        if (phys < 0 || phys >= p.num_blocks) PA_RECORD_ERROR(PA_ERRBIT_INDEX);  // TMA zero-fills out of range
        const int key = j * BN + lane * 16;
        const int y = phys * p.block_size + key % p.block_size;
        for (int hf = 0; hf < 2; ++hf)
          tma_load_2d(smem + off + st * KVTILE + hf * KVHALF + lane * 16 * 128, map, g * HD + hf * 64, y, &full[st]);
      }
    };
    // lane 0 polls both rings and broadcasts, so the warp never splits on a wait; the time spent with
    // neither ring ready is bounded like every other wait
    uint64_t idle_since = 0;
    while (jk < nkv || jv < nkv) {
      int go = 0;  // 1: issue K, 2: issue V
      if (lane == 0) {
        if (jk < nkv && (jk < kStages || mbar_try_wait(&k_empty[jk % kStages], ((jk / kStages) - 1) & 1)))
          go = 1;
        else if (jv < jk && (jv < kStages || mbar_try_wait(&v_empty[jv % kStages], ((jv / kStages) - 1) & 1)))
          go = 2;
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (go == 1) {
        issue(jk, physk, k_full, &kmap, K_OFF);
        ++jk;
        physk = lookup(jk);
        idle_since = 0;
      } else if (go == 2) {
        issue(jv, physv, v_full, &vmap, V_OFF);
        ++jv;
        physv = lookup(jv);
        idle_since = 0;
      } else {
        int late = 0;
        if (lane == 0) {
          const uint64_t now = global_ns();
          if (idle_since == 0) idle_since = now;
          late = now - idle_since > PA_WAIT_LIMIT_NS;
        }
        if (__shfl_sync(0xffffffffu, late, 0)) {
          ok = false;
          break;
        }
      }
    }
  } else if (warp == 9) {
    // ============================================ MMA issuer (one thread issues; the warp zeroes V tails)
    const uint32_t id_s = idesc(DT == PA_BF16 ? 1 : 0, false, BN);
    const uint32_t id_pv = idesc(DT == PA_BF16 ? 1 : 0, true, HD);
    auto issue_pv = [&](int i) -> bool {
      const int st = i % kStages;
      if (!mbar_wait(&v_full[st], (i / kStages) & 1)) return false;
      const int valid = kend - i * BN;
      if (valid < BN) {  // keys past the end: zero their V rows (their bytes may be anything, even NaN)
        for (int idx = lane; idx < (BN - valid) * 16; idx += 32) {
          const int r = valid + idx / 16, c = (idx % 16) * 8;
          sts128(sb + V_OFF + st * KVTILE + tile_off(r, c, KVHALF), 0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      for (int t = 0; t < 2; ++t) {
        if (!mbar_wait(&p_full[t], i & 1)) return false;
        tc_fence_after();
        const bool lo = lo_flag[t * 2 + (i & 1)] == i + 1;
        if (lane == 0) {
          const uint32_t od = tmem + O_COL + t * HD;
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_f16(od, kmajor_desc(sb + P_OFF + t * PTILE, 0, ks), v_desc(sb + V_OFF + st * KVTILE, ks), id_pv,
                    (i > 0 || ks > 0) ? 1u : 0u);
          if (lo)
            for (int ks = 0; ks < BN / 16; ++ks)
              mma_f16(od, kmajor_desc(sb + PL_OFF + t * PTILE, 0, ks), v_desc(sb + V_OFF + st * KVTILE, ks), id_pv,
                      1u);
          mma_commit(&o_done[t * 2 + (i & 1)]);
          if (t == 1) mma_commit(&v_empty[st]);
        }
        __syncwarp();
      }
      return true;
    };
    if (!mbar_wait(q_full, 0)) ok = false;
    for (int j = 0; j < nkv && ok; ++j) {
      const int st = j % kStages, buf = j & 1;
      if (!mbar_wait(&k_full[st], (j / kStages) & 1)) {
        ok = false;
        break;
      }
      for (int t = 0; t < 2; ++t) {
        if (j >= 2 && !mbar_wait(&s_free[t * 2 + buf], ((j >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          for (int ks = 0; ks < HD / 16; ++ks)
            mma_f16(tmem + t * 128 + buf * BN, kmajor_desc(sb + Q_OFF + t * QTILE, QHALF, ks),
                    kmajor_desc(sb + K_OFF + st * KVTILE, KVHALF, ks), id_s, ks > 0 ? 1u : 0u);
          mma_commit(&s_full[t * 2 + buf]);
          if (t == 1) mma_commit(&k_empty[st]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (j >= 1 && !issue_pv(j - 1)) ok = false;
    }
    if (ok && !issue_pv(nkv - 1)) ok = false;
  } else {
    // ============================================ softmax warpgroups: warpgroup t, thread r owns row mrow[t] + r
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const int pos = L - C + mrow[t] + r;                      // this row's position (keys 0..pos visible)
    const int last_key = min(pos, L - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lane quarter
    const uint32_t p_lo = sb + PL_OFF + t * PTILE;
    float m_ref = -INFINITY;  // reference max (log2 units) shared by O and l
    float l = 0.f;
    float s[BN];
    for (int j = 0; j < nkv && ok; ++j) {
      const int buf = j & 1;
      if (!mbar_wait(&s_full[t * 2 + buf], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_ld32(tmem + lane_base + t * 128 + buf * BN, s);
      tmem_ld32(tmem + lane_base + t * 128 + buf * BN + 32, s + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[t * 2 + buf]);
      const int lim = last_key - j * BN;  // last visible column of this key tile
      if (lim < BN - 1) {
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = c <= lim ? s[c] : -INFINITY;
      }
      // eight independent partial maxima: short dependency chains
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = s[e];
#pragma unroll
      for (int c = 8; c < BN; ++c) pm[c & 7] = fmaxf(pm[c & 7], s[c]);
      float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      mx *= p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleLog2 || (m_ref == -INFINITY && mx != -INFINITY)) {
        alpha = m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - mx);
        rescale = m_ref != -INFINITY;
        m_ref = mx;
      }
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      float ps[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ps[e] = 0.f;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        s[c] = fast_exp2(fmaf(s[c], p.scale_log2, neg_m));
        ps[c & 7] += s[c];
      }
      const float rs = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      l = l * alpha + rs;
      // does this key tile carry a large share of some row's mass?  (decided per query tile:
      // tile j needs the low term iff lo_flag[t][j&1] == j+1 once the warpgroup has voted)
      if (__any_sync(0xffffffffu, rs >= kLoFraction * l) && lane == 0) lo_flag[t * 2 + (j & 1)] = j + 1;
      named_barrier_sync(1 + t, BM);
      const bool lo = lo_flag[t * 2 + (j & 1)] == j + 1;
      const uint32_t p_hi = sb + P_OFF + t * PTILE;
      // the P buffers and O are touched only after the PV of key tile j-1 is complete
      if (j >= 1 && !mbar_wait(&o_done[t * 2 + ((j - 1) & 1)], ((j - 1) >> 1) & 1)) {
        ok = false;
        break;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + O_COL + t * HD + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tmem + lane_base + O_COL + t * HD + c, o);
        }
        tmem_wait_st();
      }
#pragma unroll
      for (int c = 0; c < BN; c += 8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = Elt<DT>::from_f2(s[c + 2 * e], s[c + 2 * e + 1]);
        sts128(p_hi + tile_off(r, c, 0), w[0], w[1], w[2], w[3]);
        if (lo) {
          uint32_t wl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 hv = Elt<DT>::to_f2(w[e]);
            wl[e] = Elt<DT>::from_f2(s[c + 2 * e] - hv.x, s[c + 2 * e + 1] - hv.y);
          }
          sts128(p_lo + tile_off(r, c, 0), wl[0], wl[1], wl[2], wl[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    // epilogue: O / l -> out
    if (ok && mbar_wait(&o_done[t * 2 + ((nkv - 1) & 1)], ((nkv - 1) >> 1) & 1)) {
      tc_fence_after();
      const int row = mrow[t] + r;
      T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(q0 + row) * p.num_q_heads + head[t]) * HD;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + O_COL + t * HD + c, o);
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
  if (warp == 9)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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
  const int G = num_q_heads / num_kv_heads;
  if (!pa::valid_group(G)) return PA_ERR_UNSUPPORTED;
  if (batch == 0 || total_q_tokens == 0 || max_chunk_len == 0) return PA_OK;
  if (!q || !query_start_loc || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID;
  if (!pa::aligned16(q) || !pa::aligned16(k_cache) || !pa::aligned16(v_cache) || !pa::aligned16(out) ||
      (reinterpret_cast<uintptr_t>(query_start_loc) & 3u) || (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PA_ERR_ALIGN;
  if (num_blocks == 0) return PA_ERR_INVALID;
  if ((long)num_blocks * block_size >= (1L << 31)) return PA_ERR_UNSUPPORTED;
  const int mtiles = (max_chunk_len + BM - 1) / BM;
  const int units = G >= 2 ? (G / 2) * mtiles : (mtiles + 1) / 2;
  const long grid = (long)batch * num_kv_heads * units;
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
  p.units = units;
  p.scale_log2 = scale * kLog2e;

  CUtensorMap qm, km, vm;
  const uint64_t rows = (uint64_t)num_blocks * block_size;
  const uint64_t cols = (uint64_t)num_kv_heads * HD;
  if (pa::encode_2d_sw128(&qm, q, (uint64_t)num_q_heads * HD, (uint64_t)total_q_tokens, (uint64_t)num_q_heads * HD * 2,
                          64, BM) != PA_OK)
    return PA_ERR_CUDA;
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
  kern<<<(unsigned)grid, 320, SMEM_ALLOC, (cudaStream_t)stream>>>(qm, km, vm, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
