// Host-side check of the dataflow factorisation's task numbering
// (csrc/chol_tasks.cuh, compiled for the host), for one block count N:
//  * decoding every number 0 .. total−1 yields each tile task of the
//    algorithm exactly once (PANEL, TRAIL, MROW, MTRAIL of every step);
//  * every task a task waits for comes earlier in the numbering, and every
//    task that waits for a step of the chain comes after the worker tasks
//    that step of the chain (and every step before it) waits for.
// With tasks claimed in numbering order by running CTAs, that makes the
// single launch free of deadlock.  Used by test_chol_tasks_host.py.
//
// usage: chol_tasks_sim N        prints "ok N total" or a failure and exits 1
#include <cstdio>
#include <cstdlib>
#include <map>
#include <tuple>
#include <vector>

#include "../post_weight_quantization_08_b200/csrc/chol_tasks.cuh"

using namespace gptq;
using Key = std::tuple<int, int, int, int>;

static int fail(const char* what, int N, int p) {
  std::printf("FAIL N=%d task %d: %s\n", N, p, what);
  return 1;
}

int main(int argc, char** argv) {
  const int N = std::atoi(argv[1]);
  std::vector<int> prefix(task_slots(N) + 1);
  build_slot_prefix(N, prefix.data());
  const int total = prefix[task_slots(N)];
  if ((int64_t)total != total_tasks(N)) return fail("total", N, -1);

  // the expected task set
  std::map<Key, int> pos;
  int expected = 0;
  for (int k = 0; k < N; ++k) {
    for (int i = k + 2; i < N; ++i) pos[Key(T_PANEL, k, i, k)] = -1, ++expected;
    for (int i = k + 2; i < N; ++i) pos[Key(T_TRAIL, k, i, k + 1)] = -1, ++expected;
    for (int i = k + 2; i < N; ++i)
      for (int j = k + 2; j <= i; ++j) pos[Key(T_TRAIL, k, i, j)] = -1, ++expected;
    for (int c = 0; c < k; ++c) pos[Key(T_MROW, k, k, c)] = -1, ++expected;
    for (int i = k + 1; i < N; ++i)
      for (int c = 0; c <= k; ++c) pos[Key(T_MTRAIL, k, i, c)] = -1, ++expected;
  }
  if (expected != total) return fail("count differs from the algorithm's task set", N, -1);
  std::vector<Key> order(total);
  for (int p = 0; p < total; ++p) {
    int kind, k, i, j;
    decode_task(p, N, prefix.data(), kind, k, i, j);
    Key key(kind, k, i, j);
    auto it = pos.find(key);
    if (it == pos.end()) return fail("decoded a task outside the set", N, p);
    if (it->second != -1) return fail("decoded a task twice", N, p);
    it->second = p;
    order[p] = key;
  }
  auto at = [&](int kind, int k, int i, int j) { return pos.at(Key(kind, k, i, j)); };
  // the chain's step k waits for tiles (k+1,k) and (k+1,k+1) after k updates:
  // TRAIL(k−1,k+1,k) and TRAIL(k−1,k+1,k+1); steps run in order
  std::vector<int> chain_ready(N, -1);
  for (int k = 0; k < N; ++k) {
    int r = k > 0 ? chain_ready[k - 1] : -1;
    if (k >= 1 && k + 1 < N) {
      r = std::max(r, at(T_TRAIL, k - 1, k + 1, k));
      r = std::max(r, at(T_TRAIL, k - 1, k + 1, k + 1));
    }
    chain_ready[k] = r;
  }
  for (int p = 0; p < total; ++p) {
    const int kind = std::get<0>(order[p]), k = std::get<1>(order[p]);
    const int i = std::get<2>(order[p]), j = std::get<3>(order[p]);
    std::vector<int> deps;        // worker tasks
    std::vector<int> chain;       // chain steps
    auto panel = [&](int kk, int ii) {      // L_{ii,kk} final
      if (ii == kk + 1) chain.push_back(kk); else deps.push_back(at(T_PANEL, kk, ii, kk));
    };
    if (kind == T_PANEL) {
      chain.push_back(k);
      if (k >= 1) deps.push_back(at(T_TRAIL, k - 1, i, k));
    } else if (kind == T_MROW) {
      chain.push_back(k);
      if (k - 1 >= j) deps.push_back(at(T_MTRAIL, k - 1, k, j));
    } else if (kind == T_TRAIL) {
      panel(k, i);
      panel(k, j);
      if (k >= 1) deps.push_back(at(T_TRAIL, k - 1, i, j));
    } else {
      panel(k, i);
      if (j < k) deps.push_back(at(T_MROW, k, k, j)); else chain.push_back(k);
      if (k - 1 >= j) deps.push_back(at(T_MTRAIL, k - 1, i, j));
    }
    for (int d : deps)
      if (d >= p) return fail("waits for a later task", N, p);
    for (int c : chain)
      if (chain_ready[c] >= p) return fail("waits for a chain step that waits for it", N, p);
  }
  std::printf("ok %d %d\n", N, total);
  return 0;
}
