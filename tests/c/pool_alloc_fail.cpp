// Host memory exhaustion inside the block pool's batched calls, made on the host: this program replaces the
// global operator new (the library resolves it to this definition at load time) with one that throws
// std::bad_alloc once a countdown reaches zero.  Every batched call must then fail with a status and leave
// the pool exactly as it was: no sequence lost or added, every block's reference count unchanged (the
// leak check of "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend NPU", section 4.2).
// Prints "ok" and exits 0, or names the first failed check and exits 1.
#include <cstdio>
#include <cstdlib>
#include <new>
#include <vector>

#include "paged_attn.h"

static long g_fail_after = -1;  // < 0: never fail; otherwise the number of allocations still allowed

void* operator new(std::size_t n) {
  if (g_fail_after == 0) throw std::bad_alloc();
  if (g_fail_after > 0) --g_fail_after;
  void* p = std::malloc(n ? n : 1);
  if (!p) throw std::bad_alloc();
  return p;
}
void operator delete(void* p) noexcept { std::free(p); }
void operator delete(void* p, std::size_t) noexcept { std::free(p); }

#define CHECK(cond)                                                      \
  do {                                                                   \
    if (!(cond)) {                                                       \
      std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                          \
    }                                                                    \
  } while (0)

struct Snapshot {
  pa_pool_stats_t st;
  std::vector<int> refs;
};

static Snapshot snap(const pa_pool* p, int nb) {
  Snapshot s{};
  pa_pool_stats(p, &s.st);
  for (int b = 0; b < nb; ++b) s.refs.push_back(pa_pool_ref_count(p, b));
  return s;
}

static bool same(const Snapshot& a, const Snapshot& b) {
  return a.st.free_blocks == b.st.free_blocks && a.st.used_blocks == b.st.used_blocks &&
         a.st.num_seqs == b.st.num_seqs && a.st.tokens == b.st.tokens && a.st.table_refs == b.st.table_refs &&
         a.st.ref_sum == b.st.ref_sum && a.refs == b.refs;
}

int main() {
  enum { NB = 64, BS = 16 };
  pa_pool* p = pa_pool_create(NB, BS, nullptr);
  CHECK(p != nullptr);
  CHECK(pa_seq_alloc(p, 5, 40) == PA_OK);  // a live sequence holding 3 blocks
  CHECK(pa_seq_fork(p, 5, 7, 32) == PA_OK);
  const Snapshot before = snap(p, NB);

  // A batch that names the live id 5: with allocation working the call is refused (PA_ERR_NOT_FOUND); with
  // the id check's own allocation failing, it must still leave sequence 5 and its blocks alone.
  const int64_t ids[3] = {6, 5, 8};
  const int32_t toks[3] = {20, 10, 1};
  CHECK(pa_pool_alloc_batch(p, ids, toks, 3) == PA_ERR_NOT_FOUND);
  CHECK(same(before, snap(p, NB)));
  for (long k = 0; k < 12; ++k) {  // fail the k-th allocation of the call, for every k the call reaches
    g_fail_after = k;
    const int st = pa_pool_alloc_batch(p, ids, toks, 3);
    g_fail_after = -1;
    CHECK(st == PA_ERR_OOM || st == PA_ERR_NOT_FOUND);
    CHECK(same(before, snap(p, NB)));
    int len = 0;
    CHECK(pa_seq_info(p, 5, &len, nullptr) == PA_OK && len == 40);
  }

  // A batch of fresh ids: a failure at any allocation leaves none of them behind; with allocation working
  // the batch goes in whole.
  const int64_t fresh[3] = {10, 11, 12};
  for (long k = 0; k < 12; ++k) {
    g_fail_after = k;
    const int st = pa_pool_alloc_batch(p, fresh, toks, 3);
    g_fail_after = -1;
    if (st == PA_OK) {  // the call needed fewer than k allocations: undo it and stop
      CHECK(pa_pool_free_batch(p, fresh, 3) == PA_OK);
      CHECK(same(before, snap(p, NB)));
      break;
    }
    CHECK(st == PA_ERR_OOM);
    CHECK(same(before, snap(p, NB)));
    for (int i = 0; i < 3; ++i) CHECK(pa_seq_info(p, fresh[i], nullptr, nullptr) == PA_ERR_NOT_FOUND);
  }

  // The appending and freeing batches under the same failures: all or nothing.
  const int64_t live[2] = {5, 7};
  const int32_t one[2] = {1, 1};
  for (long k = 0; k < 12; ++k) {
    g_fail_after = k;
    const int st = pa_pool_append_batch(p, live, one, 2, nullptr, nullptr, nullptr);
    g_fail_after = -1;
    if (st == PA_OK) break;
    CHECK(st == PA_ERR_OOM);
    CHECK(same(before, snap(p, NB)));
  }
  pa_pool_destroy(p);
  std::printf("ok\n");
  return 0;
}
