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
// 5th-generation tensor cores, as CTA pairs (a cluster of two CTAs on one
// TPC).  Each CTA owns 128 query rows: two heads of one KV group over the same
// rows, or, when a group has one head, two consecutive row tiles of it.  The
// pair walks the keys in tiles of 128 and the even CTA issues every product for
// both (tcgen05.mma cta_group::2, M = 256):
//   * S = Q K^T (N 128, K 128): A = the CTA's query tile in its own TMEM
//     (64 columns of packed 16-bit pairs), B = K split by key: each CTA holds
//     64 of the tile's 128 keys;
//   * O += P V (N 128, K 128): A = P, written by the softmax over its own S
//     buffer in TMEM, B = V split by head_dim: each CTA holds 64 columns.
// So each CTA streams half of every K and V tile from L2 (the bound of the
// one-CTA form) and the paired product runs at ~0.8 of the tensor peak where a
// one-CTA 128 x 128 x 16 product with A in TMEM stops near 0.6.
// Two TMA producer warps per CTA (one for K, one for V: a TMA issue stalls
// while the unit is busy) gather its 16-row K and V boxes through the block
// table (128-byte swizzle, no multicast) into four-stage K and V rings;
// the copies of both CTAs complete on the even CTA's barriers (TMA
// .cta_group::2), slots are released by a multicast tcgen05.commit, and the
// last, partial V tile is loaded against a local barrier and zero-filled past
// the end before it is signalled.  Two threads of the even CTA issue the
// products, one S(j) and one O += P(j) V, so the tensor core runs PV(j-1) and
// S(j+1) while the softmax works on S(j).  In each CTA two softmax warpgroups split every key tile in
// halves (keys 0-63 and 64-127; thread r = row r = TMEM lane r): they swap
// their half-tile maxima through shared memory, keep fp32 running sums per
// half (added at the end), rescale O in TMEM only when the running max grows
// by more than 2^8 (exact: O and the sums always share one reference max), and
// write P's high 16-bit term.  A warp in which some row puts at least 1/4 of
// that half's running mass in the half-tile (the first tiles, and tiles with
// dominant keys) also writes P's low term, exact to ~2^-17, and the other
// warps write zeros there; the even CTA issues the low term's product for a
// half when any warp of the pair asked.  Without it a tile's high term alone
// moves an output by at most 2^-9 |v| / 4 = 2^-11 |v| (the rounding of P
// relative to that tile's share of the row's mass); the low terms' extra
// products took 15 % of the kernel's time at a threshold of 1/16 and 4 % at 1/4, and
// dropping them altogether breaks the 2e-3 + 1e-2|ref| tolerance on a
// dominant key.  3 of every 8 exponentials run
// as a polynomial on the FMA pipe to relieve the MUFU unit.
//
// The same kernel serves the cascade decode's shared-prefix pass (pages "Nano-vLLM-Ascend..." section
// 2.1, reference-counted shared blocks, and "Ascend NPU LLM inference optimisation..." section 4, block
// sharing): a "sequence" is then a group of decode sequences forked from one parent, its query rows are
// the members' single decode queries (consecutive rows of the decode q), every row attends to the whole
// shared prefix through the first member's block table (no causal limit; keys past the prefix are masked
// in the last tile), and the epilogue merges the prefix's softmax with the member's suffix result already
// in `out` by their log-sum-exps.

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "host_common.h"

PA_DEFINE_ERROR_WORD(pa__err_prefill)
namespace {
// Bounded wait that polls with test_wait (never suspends the warp), for a wait on the critical path whose
// phase completes within a few hundred nanoseconds: the PV issuer's wait for P.  Measured: +1 % for the
// kernel; the same for every wait of both issuers; -2 % when the eight softmax warps also spin.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(pa::smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_spin_warp(uint64_t* bar, uint32_t parity) {
  bool done = mbar_test(bar, parity);
  if (!done) {
    const uint64_t start = pa::global_ns();
    for (;;) {
      for (int k = 0; k < 256 && !done; ++k) done = mbar_test(bar, parity);
      if (done || pa::global_ns() - start > PA_WAIT_LIMIT_NS) break;
    }
  }
  return __all_sync(0xffffffffu, done) != 0;
}
}  // namespace


namespace {

using namespace pa;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int BM = 128;                 // query rows per CTA (TMEM lanes); the pair covers 256
constexpr int BN = 128;                 // keys per key tile
constexpr int HD = 128;                 // head_dim
constexpr int KS = 4;                   // K ring depth
constexpr int VS = 4;                   // V ring depth
constexpr float kRescaleLog2 = 8.f;     // rescale O only when the max grows by more than 2^8
constexpr float kLoFraction = 1.f / 4.f;

// shared memory map (offsets from a 1024-byte aligned base).  Tiles have rows of 128 bytes
// (64 16-bit values) with the 128-byte swizzle.
constexpr int KHALF = (BN / 2) * 128;           // 8 KB: this CTA's 64 keys x 64 head_dim columns
constexpr int KTILE = 2 * KHALF;                // 16 KB: this CTA's 64 keys x 128 columns
constexpr int VTILE = BN * 128;                 // 16 KB: 128 keys x this CTA's 64 columns
constexpr int K_OFF = 0;                        // K[KS]
constexpr int V_OFF = K_OFF + KS * KTILE;       // V[VS]
constexpr int XCH_OFF = V_OFF + VS * VTILE;     // float m_part[2][2][128], l_part[2][128]
constexpr int BAR_OFF = XCH_OFF + 6 * BM * 4;
// barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], v_tail, s_full[2], p_full[2],
// o_done[2], drain[2].  The full barriers, q_full, p_full and drain are used in the even CTA only.
constexpr int NBAR = 1 + 2 * KS + 2 * VS + 1 + 2 + 2 + 2 + 2;
constexpr int MISC_OFF = BAR_OFF + NBAR * 8;    // tmem base (4 B), lo flags int[2 ranks][2][2 halves]
constexpr int SMEM_BYTES = MISC_OFF + 4 + 32 + 28;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// TMEM columns (both CTAs): Q [0, 64) (packed pairs), S buffers [128, 256) and [256, 384),
// O [384, 512).  Within an S buffer, P of key half h sits at h*64 (high term, 32 columns) and
// h*64 + 32 (low term), inside the columns that half's own S values occupied.
constexpr int TMEM_COLS = 512;
constexpr int Q_COL = 0;
constexpr int S_COL = 128;
constexpr int O_COL = 384;
constexpr int kSoftmaxWarps = 8;        // per CTA; q_full and p_full count one arrival per warp of the pair
// warps 0-7 softmax, 8 K producer, 9 S issuer (even CTA) and TMEM allocator, 10 V producer,
// 11 PV issuer (even CTA)
constexpr int kThreads = 12 * 32;

struct PrefillParams {
  const void* q;
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
  int units;          // CTA pairs per (sequence, KV head)
  float scale_log2;
  // Shared-prefix mode (the cascade decode's prefix pass): "sequence" b is a group of decode sequences
  // group_start[b] .. group_start[b+1]-1 sharing their first seq_prefix[group_start[b]] tokens; query row i
  // is member group_start[b] + i (its one decode query), every row attends to the whole prefix (no causal
  // limit) through the first member's block table, and the epilogue merges the prefix's softmax with the
  // member's suffix result (out, lse_s) already in `out`.
  int prefix_mode;
  const int32_t* group_start;
  const int32_t* seq_prefix;
  const float* lse_s;
};

// --------------------------------------------------------------- cluster / tcgen05 helpers
__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The address of this CTA's shared variable `local` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// All threads of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on a barrier of the other CTA.  The release form publishes this thread's earlier
// shared-memory writes to the pair and costs ~1-2 us, so it is kept for the few arrivals that
// follow generic writes; the relaxed form serves arrivals whose data is already ordered (TMA bytes
// counted by the barrier itself, TMEM stores completed by tcgen05.wait::st).
__device__ __forceinline__ void arrive_cluster_release(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void arrive_cluster_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// 2-D tiled load into this CTA's shared memory whose completion is counted on a barrier of
// either CTA of the pair (`bar` is a shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// This CTA's K half-tile as the K-major B operand of S (64 key rows of 128 bytes per head_dim
// half, the halves KHALF apart, 8-row groups 1024 bytes apart): k-step ks of 16 head_dim values.
__device__ __forceinline__ uint64_t k_desc(uint32_t tile, int ks) {
  return sdesc(tile + (ks >> 2) * KHALF + (ks & 3) * 32, 16, 1024);
}
// This CTA's V tile as the MN-major B operand of PV (128 key rows of 128 bytes = its 64
// head_dim columns): k-step ks covers keys 16*ks .. 16*ks+15.
__device__ __forceinline__ uint64_t v_desc(uint32_t tile, int ks) {
  return sdesc(tile + ks * 16 * 128, VTILE, 1024);
}
// Instruction descriptor, kind::f16: fp32 accumulate, A/B 16-bit (0 = f16, 1 = bf16), A K-major,
// M 256 (the pair).
__host__ __device__ constexpr uint32_t idesc(int fmt, bool b_mn_major, int n) {
  return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)((2 * BM) >> 4) << 24);
}
// D (TMEM of both CTAs) [+]= A (TMEM of both CTAs, 128 lanes x 16 elements each as 8 columns of
// packed pairs) * B (shared memory of both CTAs, split along N).
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs when every product issued so far is done.
__device__ __forceinline__ void commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// ... on this CTA's barrier only.
__device__ __forceinline__ void commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- softmax arithmetic
// Packed pairs of fp32 (Blackwell's f32x2 FMA/add issue two lanes' worth in one instruction).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// 2^x for a pair, on the FMA pipe instead of the MUFU unit (which issues 16 exp2 per clock per SM
// and bounds the softmax otherwise).  x is clamped to [-125, +inf) (every x here is <= 8), split
// as x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f is a degree-4 polynomial fitted here for minimal relative error on that
// interval (weighted least squares driven toward equioscillation; max relative error 2.7e-6,
// below the 2^-17 of the two-term P), and 2^n enters as n added to the exponent field.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  upk2(x2, x0, x1);
  x2 = pk2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t one = pk2(1.f, 1.f), neg_one = pk2(-1.f, -1.f);
  const uint64_t magic = pk2(12582912.f, 12582912.f), neg_magic = pk2(-12582912.f, -12582912.f);
  const uint64_t t = fma2(x2, one, magic);       // n in the low mantissa bits
  const uint64_t n = fma2(t, one, neg_magic);    // n as a float
  const uint64_t f = fma2(n, neg_one, x2);       // x - n
  uint64_t q = pk2(9.570068680e-03f, 9.570068680e-03f);
  q = fma2(q, f, pk2(5.591780692e-02f, 5.591780692e-02f));
  q = fma2(q, f, pk2(2.402474433e-01f, 2.402474433e-01f));
  q = fma2(q, f, pk2(6.931218505e-01f, 6.931218505e-01f));
  q = fma2(q, f, pk2(9.999992847e-01f, 9.999992847e-01f));
  float q0, q1, t0, t1;
  upk2(q, q0, q1);
  upk2(t, t0, t1);
  // the bits of t are 0x4B400000 + n, so (bits << 23) is n << 23 modulo 2^32
  return pk2(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
             __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}
constexpr int kPolyPairs = 3;  // of every 8 pairs of a row's half-tile, this many take exp2_poly2

// --------------------------------------------------------------- kernel
template <int DT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const PrefillParams p) {
  using T = typename Elt<DT>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* q_full = bars;                 // [even CTA] queries in TMEM, one arrival per softmax warp
  uint64_t* k_full = bars + 1;             // [even CTA] both K halves landed
  uint64_t* k_empty = k_full + KS;         // K slot free: S of its key tile is done
  uint64_t* v_full = k_empty + KS;         // [even CTA] both V halves landed (two producer arrivals)
  uint64_t* v_empty = v_full + VS;         // V slot free: PV of its key tile is done
  uint64_t* v_tail = v_empty + VS;         // this CTA's partial last V tile landed
  uint64_t* s_full = v_tail + 1;           // [key tile & 1]
  uint64_t* p_full = s_full + 2;           // [even CTA][key tile & 1]: P written, one arrival per softmax warp
  uint64_t* o_done = p_full + 2;           // [key tile & 1]: O += P V of that key tile is complete
  uint64_t* drain = o_done + 2;            // [even CTA][issuer] every product it issued has completed
  float* m_part = reinterpret_cast<float*>(smem + XCH_OFF);  // [key tile & 1][half][row]
  float* l_part = m_part + 4 * BM;                            // [half][row]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* lo_flag = reinterpret_cast<volatile int*>(smem + MISC_OFF + 4);  // [rank][j & 1][half], even CTA

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  const int G = p.num_q_heads / p.num_kv_heads;
  // pair -> (unit, KV head, sequence); the pairs reading the same K/V are adjacent
  int u = blockIdx.x >> 1;
  const int unit = u % p.units;
  u /= p.units;
  const int g = u % p.num_kv_heads;
  const int b = u / p.num_kv_heads;
  int head, mrow, mrow_lo, mrow_hi;  // this CTA's head and first row; the pair's first and last row tiles
  if (G >= 2) {
    const int hp = unit % (G / 2), mt = unit / (G / 2);
    head = g * G + 2 * hp + (int)rank;
    mrow = mrow_lo = mrow_hi = mt * BM;
  } else {
    head = g;
    mrow = (2 * unit + (int)rank) * BM;
    mrow_lo = 2 * unit * BM;
    mrow_hi = mrow_lo + BM;
  }

  const int32_t* rowstart = p.prefix_mode ? p.group_start : p.query_start_loc;
  const int q0 = __ldg(rowstart + b), q1 = __ldg(rowstart + b + 1);
  const int C = q1 - q0;
  // both CTAs of a pair take the same early exits (they depend on the pair only)
  if (mrow_lo >= C) return;
  const int cap = p.max_blocks_per_seq * p.block_size;
  int L, kend;
  if (p.prefix_mode) {  // keys [0, P) for every row: the group's shared prefix (a multiple of 16)
    const int P0 = __ldg(p.seq_prefix + q0);
    const int P = min(max(P0, 0), cap) & ~15;
    if (P != P0 && threadIdx.x == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
    if (P == 0) return;  // no shared prefix: the suffix result already is the answer
    L = P;
    kend = P;
  } else {
    L = __ldg(p.context_lens + b);
    if (L > cap || L < C) {  // broken caller invariant: record and produce nothing for this pair
      if (threadIdx.x == 0) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
      return;
    }
    // keys [0, kend) are visible to some row of the pair
    kend = L - C + min(mrow_hi + BM, C);
  }
  const int nkv = (kend + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 8; ++i) lo_flag[i] = 0;
    mbar_init(q_full, 2 * kSoftmaxWarps);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&v_full[i], 2);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(v_tail, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 2 * kSoftmaxWarps);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    fence_mbar_init();
  }
  if (warp == 9) {  // the same warp in both CTAs allocates the pair's TMEM
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 8 || warp == 10) {
    // ============================================ producers: this CTA's K halves (warp 8) and V
    // halves (warp 10); a TMA issue stalls while the unit is busy, so K and V get a warp each
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
    }
    const int32_t* bt = p.block_tables + (size_t)(p.prefix_mode ? q0 : b) * p.max_blocks_per_seq;
    const uint32_t kfull0 = map_rank(smem_u32(k_full), 0), vfull0 = map_rank(smem_u32(v_full), 0);
    // first key of box i of key tile j: K boxes cover this CTA's 64 keys, V boxes all 128
    auto kbox_key = [&](int j, int i) { return j * BN + (int)rank * (BN / 2) + i * 16; };
    auto vbox_key = [&](int j, int i) { return j * BN + i * 16; };
    auto nbox = [&](int key0, int maxb) { return max(0, min(maxb, (kend - key0 + 15) / 16)); };
    auto phys_of = [&](int key) -> int { return key < kend ? __ldg(bt + key / p.block_size) : 0; };
    auto wait1 = [&](uint64_t* bar, uint32_t parity) -> bool {
      int r = 1;
      if (lane == 0) r = mbar_wait(bar, parity) ? 1 : 0;
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    auto put_k = [&](int j) -> bool {
      const int st = j % KS;
      if (j >= KS && !wait1(&k_empty[st], ((j / KS) - 1) & 1)) return false;
      const int mine = nbox(kbox_key(j, 0), 4);
      if (leader && lane == 0) {  // bytes of both CTAs' boxes
        const int peer = nbox(j * BN + BN / 2, 4);
        mbar_arrive_expect_tx(&k_full[st], (mine + peer) * 2 * 16 * 128);
      }
      __syncwarp();
      if (lane < mine) {
        const int key = kbox_key(j, lane);
        const int phys = phys_of(key);
        if (phys < 0 || phys >= p.num_blocks) PA_RECORD_ERROR(PA_ERRBIT_INDEX);  // TMA zero-fills out of range
        const int y = phys * p.block_size + key % p.block_size;
        for (int hf = 0; hf < 2; ++hf)
          tma_load_2d_pair(sb + K_OFF + st * KTILE + hf * KHALF + lane * 16 * 128, &kmap, g * HD + hf * 64, y,
                           kfull0 + 8 * st);
      }
      __syncwarp();
      return true;
    };
    auto put_v = [&](int j) -> bool {
      const int st = j % VS;
      if (j >= VS && !wait1(&v_empty[st], ((j / VS) - 1) & 1)) return false;
      const int nb = nbox(vbox_key(j, 0), 8);
      const int valid = kend - j * BN;  // keys of this tile that exist
      const int x = g * HD + (int)rank * 64;
      auto box = [&](int i, bool pair_bar) {
        const int key = vbox_key(j, i);
        const int phys = phys_of(key);
        if (phys < 0 || phys >= p.num_blocks) PA_RECORD_ERROR(PA_ERRBIT_INDEX);
        const int y = phys * p.block_size + key % p.block_size;
        if (pair_bar)
          tma_load_2d_pair(sb + V_OFF + st * VTILE + i * 16 * 128, &vmap, x, y, vfull0 + 8 * st);
        else
          tma_load_2d(smem + V_OFF + st * VTILE + i * 16 * 128, &vmap, x, y, v_tail);
      };
      if (valid >= BN) {
        if (leader && lane == 0) mbar_arrive_expect_tx(&v_full[st], 2 * nb * 16 * 128);
        __syncwarp();
        if (lane < nb) box(lane, true);
        __syncwarp();
        if (!leader && lane == 0) arrive_cluster_relaxed(vfull0 + 8 * st);
        return true;
      }
      // last, partial tile: land it here, zero the rows past the end (their bytes may be anything,
      // even NaN, and P is 0 there), then signal the even CTA
      if (lane == 0) mbar_arrive_expect_tx(v_tail, nb * 16 * 128);
      __syncwarp();
      if (lane < nb) box(lane, false);
      __syncwarp();
      if (!wait1(v_tail, 0)) return false;
      uint8_t* vt = smem + V_OFF + st * VTILE;
      for (int off = valid * 128 + lane * 16; off < VTILE; off += 32 * 16)
        *reinterpret_cast<uint4*>(vt + off) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&v_full[st]);
        else
          arrive_cluster_release(vfull0 + 8 * st);
      }
      __syncwarp();
      return true;
    };
    int jk = 0, jv = 0;
    if (warp == 8) {
      for (; jk < nkv; ++jk)
        if (!put_k(jk)) {
          ok = false;
          break;
        }
    } else {
      for (; jv < nkv; ++jv)
        if (!put_v(jv)) {
          ok = false;
          break;
        }
    }
    // the even CTA's full barriers count both CTAs' bytes: wait there for the last copies to land
    // before the pair can exit (bounded)
    if (leader) {
      for (int j = max(0, jk - KS); j < jk; ++j)
        if (!wait1(&k_full[j % KS], (j / KS) & 1)) ok = false;
      for (int j = max(0, jv - VS); j < jv; ++j)
        if (!wait1(&v_full[j % VS], (j / VS) & 1)) ok = false;
    }
  } else if (warp == 9 || warp == 11) {
    // ============================================ MMA issuers, even CTA: S products from warp 9, PV
    // products from warp 11.  tcgen05.commit holds its thread until the products ahead of it have
    // gone to the tensor core, so one thread issuing both would leave the tensor core idle around
    // every commit; with two, S(j+1) runs while PV(j) is being issued.  The two streams are not
    // ordered with each other, so S(j) waits for PV(j-2) (which read P(j-2) from the same TMEM
    // buffer) to complete.
    if (leader) {
      const uint32_t id_s = idesc(DT == PA_BF16 ? 1 : 0, false, BN);
      const uint32_t id_pv = idesc(DT == PA_BF16 ? 1 : 0, true, HD);
      bool issued = false;
      uint64_t* my_drain = drain + (warp == 9 ? 0 : 1);
      if (warp == 9) {
        if (!mbar_wait_warp(q_full, 0)) ok = false;
        for (int j = 0; j < nkv && ok; ++j) {
          const int st = j % KS, buf = j & 1;
          if (!mbar_wait_warp(&k_full[st], (j / KS) & 1) ||
              (j >= 2 && !mbar_wait_warp(&o_done[buf], ((j - 2) >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            for (int ks = 0; ks < HD / 16; ++ks)
              mma_pair(tmem + S_COL + buf * BN, tmem + Q_COL + ks * 8, k_desc(sb + K_OFF + st * KTILE, ks), id_s,
                       ks > 0 ? 1u : 0u);
            commit_both(&s_full[buf]);
            commit_both(&k_empty[st]);
          }
          issued = true;
          __syncwarp();
        }
      } else {
        for (int i = 0; i < nkv && ok; ++i) {
          const int st = i % VS, buf = i & 1;
          if (!mbar_wait_warp(&v_full[st], (i / VS) & 1) || !mbar_spin_warp(&p_full[buf], (i >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          bool lo[2];
          for (int h = 0; h < 2; ++h)
            lo[h] = lo_flag[0 * 4 + buf * 2 + h] == i + 1 || lo_flag[1 * 4 + buf * 2 + h] == i + 1;
          if (lane == 0) {
            const uint32_t pb = tmem + S_COL + buf * BN;
            for (int ks = 0; ks < BN / 16; ++ks)
              mma_pair(tmem + O_COL, pb + (ks >> 2) * 64 + (ks & 3) * 8, v_desc(sb + V_OFF + st * VTILE, ks), id_pv,
                       (i > 0 || ks > 0) ? 1u : 0u);
            for (int ks = 0; ks < BN / 16; ++ks)
              if (lo[ks >> 2])
                mma_pair(tmem + O_COL, pb + (ks >> 2) * 64 + 32 + (ks & 3) * 8, v_desc(sb + V_OFF + st * VTILE, ks),
                         id_pv, 1u);
            commit_both(&o_done[buf]);
            commit_both(&v_empty[st]);
          }
          issued = true;
          __syncwarp();
        }
      }
      // every product this thread issued completes before the pair releases its TMEM (bounded)
      if (issued) {
        if (lane == 0) commit_local(my_drain);
        __syncwarp();
        if (!mbar_wait_warp(my_drain, 0)) ok = false;
      }
    }
  } else {
    // ============================================ softmax warpgroups: half hf = warp / 4, thread r = row r
    const int hf = warp >> 2;
    const int r = threadIdx.x & 127;
    const int row = mrow + r;
    const int pos = L - C + row;                              // this row's position (keys 0..pos visible)
    const int last_key = p.prefix_mode ? L - 1 : min(pos, L - 1);
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lane quarter
    const int pair_bar = 3 + (warp & 3);                      // the two warps that own rows 32*(warp&3)..
    const uint32_t qfull0 = map_rank(smem_u32(q_full), 0), pfull0 = map_rank(smem_u32(p_full), 0);
    const uint32_t flag0 = map_rank(smem_u32((const void*)lo_flag), 0) + 4u * (rank * 4 + hf);
    // one arrival per warp on the even CTA's barrier, after every lane's TMEM stores are complete
    // (the even CTA arrives locally; the odd CTA releases only after it wrote a low-term flag)
    auto warp_arrive = [&](uint64_t* bar, uint32_t bar0, bool wrote_flag) {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(bar);
        else if (wrote_flag)
          arrive_cluster_release(bar0);
        else
          arrive_cluster_relaxed(bar0);
      }
    };
    // the query row's half hf of head_dim into TMEM (packed pairs: the low half holds the even element)
    {
      uint32_t w[32];
      if (row < C) {
        const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                           ((size_t)(q0 + row) * p.num_q_heads + head) * HD + hf * 64);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = __ldg(src + i);
          w[4 * i] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = 0u;
      }
      tmem_st32(tmem + lane_base + Q_COL + hf * 32, w);
      warp_arrive(q_full, qfull0, false);
    }
    float m_ref = -INFINITY;  // reference max (log2 units) shared by O and l
    float l = 0.f;            // running sum over this half's keys
    float s[64];
    for (int j = 0; j < nkv && ok; ++j) {
      const int buf = j & 1;
      const uint32_t sbuf = tmem + lane_base + S_COL + buf * BN + hf * 64;
      if (!mbar_wait_warp(&s_full[buf], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        // both column halves in flight before the one wait (it covers every earlier load of the thread)
        uint32_t raw0[32], raw1[32];
        tmem_ld32(sbuf, raw0);
        tmem_ld32(sbuf + 32, raw1);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = __uint_as_float(raw0[c]);
          s[32 + c] = __uint_as_float(raw1[c]);
        }
      }
      const int lim = last_key - (j * BN + hf * 64);  // last visible column of this half-tile
      const bool diag = lim < 63;
      if (diag) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = c <= lim ? s[c] : -INFINITY;
      }
      float pm[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pm[e] = max3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
      for (int c = 24; c < 64; c += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = max3(pm[e], s[c + e], s[c + 8 + e]);
      float mx = max3(max3(pm[0], pm[1], pm[2]), max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      // swap half-tile maxima with the warp that owns the same rows; the barrier also orders both
      // warps' S reads before either writes P over its half of the buffer
      m_part[(buf * 2 + hf) * BM + r] = mx;
      named_barrier_sync(pair_bar, 64);
      mx = fmaxf(mx, m_part[(buf * 2 + (hf ^ 1)) * BM + r]) * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleLog2 || (m_ref == -INFINITY && mx != -INFINITY)) {
        alpha = m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - mx);
        rescale = m_ref != -INFINITY;
        m_ref = mx;
      }
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      // P = 2^(s * scale_log2 - m_ref), pairwise: 5 of every 8 pairs on the MUFU unit, 3 on the
      // FMA pipe; exact zeros where the causal mask applies
      const uint64_t sc2 = pk2(p.scale_log2, p.scale_log2), nm2 = pk2(neg_m, neg_m);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const uint64_t x2 = fma2(pk2(s[2 * e], s[2 * e + 1]), sc2, nm2);
        uint64_t p2;
        if ((e & 7) < kPolyPairs) {
          p2 = exp2_poly2(x2);
        } else {
          float x0, x1;
          upk2(x2, x0, x1);
          p2 = pk2(fast_exp2(x0), fast_exp2(x1));
        }
        upk2(p2, s[2 * e], s[2 * e + 1]);
      }
      if (diag) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = c <= lim ? s[c] : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) acc[e & 3] = add2(acc[e & 3], pk2(s[2 * e], s[2 * e + 1]));
      float a0, a1, a2, a3;
      upk2(add2(acc[0], acc[1]), a0, a1);
      upk2(add2(acc[2], acc[3]), a2, a3);
      const float rs = (a0 + a2) + (a1 + a3);
      l = l * alpha + rs;
      // does this half-tile carry a large share of some row's mass in this half?  Such a warp
      // writes P's low term and flags the half, which makes the even CTA issue the low term's
      // product for it; every other warp writes zeros there, so each row gets its low term or none
      const bool flag = __any_sync(0xffffffffu, rs >= kLoFraction * l);
      if (flag && lane == 0) {
        if (leader)
          lo_flag[rank * 4 + buf * 2 + hf] = j + 1;
        else
          st_cluster(flag0 + 8u * buf, (uint32_t)(j + 1));
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold PV(j-1) before it is scaled; PV(j) waits for this tile's P
        if (j >= 1 && !mbar_wait_warp(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + O_COL + hf * 64 + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem + lane_base + O_COL + hf * 64 + c, o);
        }
      }
      {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = Elt<DT>::from_f2(s[2 * e], s[2 * e + 1]);
        tmem_st32(sbuf, w);
        if (flag) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 hv = Elt<DT>::to_f2(w[e]);
            w[e] = Elt<DT>::from_f2(s[2 * e] - hv.x, s[2 * e + 1] - hv.y);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = 0u;
        }
        tmem_st32(sbuf + 32, w);
      }
      warp_arrive(&p_full[buf], pfull0 + 8u * buf, flag);
    }
    // epilogue: O / (l_0 + l_1) -> out
    l_part[hf * BM + r] = l;
    named_barrier_sync(pair_bar, 64);
    const float lsum = l + l_part[(hf ^ 1) * BM + r];
    if (ok && mbar_wait_warp(&o_done[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1)) {
      tc_fence_after();
      T* orow = reinterpret_cast<T*>(p.out) + ((size_t)(q0 + row) * p.num_q_heads + head) * HD + hf * 64;
      // out = wp * O + ws * (what out holds): wp = 1/l and ws = 0 for prefill; in shared-prefix mode the
      // prefix's softmax and the member's suffix result are weighted by their log-sum-exps, the prefix's
      // being m_ref + log2(l) in the log2 domain and the suffix's lse_s (natural log; -inf when empty)
      float wp = 1.f / lsum, ws = 0.f;
      // shared-prefix mode is launched while the suffix decode may still run: its (out, lse) are read only
      // after that grid has completed (everything before reads inputs and older cache rows only)
      if (p.prefix_mode) asm volatile("griddepcontrol.wait;" ::: "memory");
      if (p.prefix_mode && row < C) {
        const float mp = m_ref + __log2f(lsum);
        const float ms = __ldg(p.lse_s + (size_t)(q0 + row) * p.num_q_heads + head) * kLog2e;
        const float M = fmaxf(mp, ms);
        const float ep = exp2f(mp - M), es = exp2f(ms - M);
        wp = ep / ((ep + es) * lsum);
        ws = es / (ep + es);
      }
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + O_COL + hf * 64 + c, o);
        tmem_wait_ld();
        if (row < C) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(o[e + i]) * wp;
            if (p.prefix_mode) {
              const uint4 u = *reinterpret_cast<const uint4*>(orow + c + e);
              const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 sv = Elt<DT>::to_f2(w4[i]);
                f[2 * i] = fmaf(ws, sv.x, f[2 * i]);
                f[2 * i + 1] = fmaf(ws, sv.y, f[2 * i + 1]);
              }
            }
            uint4 v;
            v.x = Elt<DT>::from_f2(f[0], f[1]);
            v.y = Elt<DT>::from_f2(f[2], f[3]);
            v.z = Elt<DT>::from_f2(f[4], f[5]);
            v.w = Elt<DT>::from_f2(f[6], f[7]);
            *reinterpret_cast<uint4*>(orow + c + e) = v;
          }
        }
      }
    } else {
      ok = false;
    }
  }
  if (!ok && lane == 0) PA_RECORD_ERROR(PA_ERRBIT_TIMEOUT);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // no product, copy or remote arrival of the pair is still in flight
  tc_fence_after();
  if (warp == 9)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

}  // namespace

namespace {

// One launch of the pair kernel: tensor maps over the caches, the dynamic shared-memory attribute set once
// per dtype and device, grid 2 * batch * Hkv * units CTAs.
int launch_pairs(PrefillParams& p, const void* k_cache, const void* v_cache, int dtype, long grid, cudaStream_t st) {
  CUtensorMap km, vm;
  const uint64_t rows = (uint64_t)p.num_blocks * p.block_size;
  const uint64_t cols = (uint64_t)p.num_kv_heads * HD;
  if (pa::encode_2d_sw128(&km, k_cache, cols, rows, cols * 2, 64, 16) != PA_OK) return PA_ERR_CUDA;
  if (pa::encode_2d_sw128(&vm, v_cache, cols, rows, cols * 2, 64, 16) != PA_OK) return PA_ERR_CUDA;
  auto kern = dtype == PA_BF16 ? prefill_kernel<PA_BF16> : prefill_kernel<PA_F16>;
  // per dtype and device; host threads may race to set it, which only repeats an idempotent call
  static std::atomic<bool> attr_set[2][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const int di = dtype == PA_BF16 ? 1 : 0;
  if (dev < 0 || dev >= 64 || !attr_set[di][dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) != cudaSuccess)
      return PA_ERR_CUDA;
    if (dev >= 0 && dev < 64) attr_set[di][dev].store(true, std::memory_order_release);
  }
  if (p.prefix_mode)  // programmatic: its CTAs may take the SMs the suffix decode frees in its tail
    return pa::launch_programmatic(kern, dim3((unsigned)grid), dim3(kThreads), SMEM_ALLOC, st, km, vm, p);
  kern<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(km, vm, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
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
  const long grid = 2L * batch * num_kv_heads * units;
  if (grid > 0x7fffffffL) return PA_ERR_UNSUPPORTED;

  PrefillParams p = {};
  p.q = q;
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
  p.prefix_mode = 0;
  return launch_pairs(p, k_cache, v_cache, dtype, grid, (cudaStream_t)stream);
}

namespace pa {

// The cascade decode's shared-prefix pass on the tensor cores (head_dim 128): for every group g of
// decode sequences group_start[g] .. group_start[g+1]-1, its members' queries attend to the group's
// shared prefix (seq_prefix of its first member, read through that member's block table), and the
// result is merged in place with each member's suffix result (out, lse_s).  Arguments are checked by the
// caller.
int prefix_pass_pairs(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      int max_blocks_per_seq, int num_groups, const int32_t* group_start, const int32_t* seq_prefix,
                      int max_group_size, const float* lse_s, int num_q_heads, int num_kv_heads, int block_size,
                      int num_blocks, float scale, int dtype, void* out, cudaStream_t st) {
  const int G = num_q_heads / num_kv_heads;
  const int mtiles = (max_group_size + BM - 1) / BM;
  const int units = G >= 2 ? (G / 2) * mtiles : (mtiles + 1) / 2;
  const long grid = 2L * num_groups * num_kv_heads * units;
  if (grid == 0) return PA_OK;
  if (grid > 0x7fffffffL) return PA_ERR_UNSUPPORTED;
  PrefillParams p = {};
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.batch = num_groups;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  p.mtiles = mtiles;
  p.units = units;
  p.scale_log2 = scale * kLog2e;
  p.prefix_mode = 1;
  p.group_start = group_start;
  p.seq_prefix = seq_prefix;
  p.lse_s = lse_s;
  return launch_pairs(p, k_cache, v_cache, dtype, grid, st);
}

}  // namespace pa
