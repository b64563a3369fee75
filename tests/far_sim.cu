// Host-side check of the trailing update's schedule (far_range in
// csrc/kernels.cuh, compiled for the host) for one (n, block, S): every
// (block e of errors, later column block c) pair receives block e's errors
// exactly once, from sweep e+1's prologue (c = e + 1) or from one far
// application, and a far application only uses errors of blocks that are
// finished when it runs (sweep b's launch: blocks < b).  Used by
// test_far_schedule_host.py.
//
// usage: far_sim n block S      prints "ok" or a failure and exits 1
#include <cstdio>
#include <cstdlib>
#include <set>
#include <utility>

#include "../post_weight_quantization_08_b200/csrc/kernels.cuh"

using namespace gptq;

int main(int argc, char** argv) {
  const int64_t n = std::atoll(argv[1]);
  const int block = std::atoi(argv[2]);
  const int S = std::atoi(argv[3]);
  const int64_t nb = (n + block - 1) / block;
  std::set<std::pair<int64_t, int64_t>> got;
  auto add = [&](int64_t e, int64_t c) -> bool {
    if (e >= c) return false;
    return got.insert({e, c}).second;
  };
  for (int64_t b = 1; b < nb; ++b) {
    if (!add(b - 1, b)) { std::printf("FAIL prologue %lld\n", (long long)b); return 1; }
    const FarRange r = far_range(n, block, S, b);
    if (r.c0 >= r.c1) continue;
    if (r.c0 % block != 0 || (r.c1 % block != 0 && r.c1 != n)) {
      std::printf("FAIL columns not on block edges at b=%lld\n", (long long)b);
      return 1;
    }
    const int64_t e0 = r.k0 / block, e1 = (r.k0 + r.kw) / block;
    if (r.k0 % block != 0 || r.kw % block != 0 || e0 < 0 || e1 > b) {
      std::printf("FAIL errors not finished at b=%lld\n", (long long)b);
      return 1;
    }
    for (int64_t e = e0; e < e1; ++e)
      for (int64_t c = r.c0 / block; c * block < r.c1; ++c)
        if (!add(e, c)) {
          std::printf("FAIL pair (%lld, %lld) twice at b=%lld\n", (long long)e, (long long)c,
                      (long long)b);
          return 1;
        }
  }
  const int64_t want = nb * (nb - 1) / 2;
  if ((int64_t)got.size() != want) {
    std::printf("FAIL %lld of %lld pairs\n", (long long)got.size(), (long long)want);
    return 1;
  }
  std::printf("ok\n");
  return 0;
}
