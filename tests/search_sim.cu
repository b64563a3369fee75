// Host-side run of the library's own binary-search logic (csrc/search.cuh:
// search_step, search_plan, search_decide, compiled for the host) on a
// pseudo-random measure of α, one pass a step and in lookahead rounds.  Used
// by test_search_host.py, which compares both traces with the oracle's
// bisection on the same measure.
//
// usage: search_sim seed span limit iters lo hi
// prints: "seq" and "rnd" lines of: final α, then (α, measure) per trace entry
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../post_weight_quantization_08_b200/csrc/search.cuh"

using namespace gptq;

// the measure: SplitMix64 (Steele, Lea, Flood 2014) of α's float bits xor a
// seed, modulo `span`; deliberately not monotone in α
static unsigned long long measure(float a, unsigned long long seed, unsigned long long span) {
  uint32_t b;
  std::memcpy(&b, &a, 4);
  unsigned long long x = (unsigned long long)b ^ seed;
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  x ^= x >> 31;
  return x % span;
}

static void init(SearchState* st, float lo, float hi) {
  std::memset(st, 0, sizeof(*st));
  st->lo = lo;
  st->hi = hi;
  st->a = hi;
}

static void print(const char* tag, const SearchState& st, const float* ta, const int64_t* tc,
                  int iters) {
  std::printf("%s %.9g", tag, (double)st.hi);
  for (int k = 0; k <= iters; ++k) std::printf(" %.9g %lld", (double)ta[k], (long long)tc[k]);
  std::printf("\n");
}

int main(int argc, char** argv) {
  if (argc != 7) return 2;
  const unsigned long long seed = std::strtoull(argv[1], nullptr, 10);
  const unsigned long long span = std::strtoull(argv[2], nullptr, 10);
  const long long limit = std::strtoll(argv[3], nullptr, 10);
  const int iters = std::atoi(argv[4]);
  const float lo = std::strtof(argv[5], nullptr), hi = std::strtof(argv[6], nullptr);
  float ta[80];
  int64_t tc[80];
  SearchState st;
  // one pass a step
  init(&st, lo, hi);
  for (int k = 0; k <= iters; ++k) {
    st.count = measure(st.a, seed, span);
    search_step(&st, k, limit, ta, tc);
  }
  print("seq", st, ta, tc, iters);
  // pass 0, then rounds of three candidates
  float ra[80];
  int64_t rc[80];
  init(&st, lo, hi);
  st.count = measure(st.a, seed, span);
  search_step(&st, 0, limit, ra, rc);
  for (int k0 = 1; k0 <= iters; k0 += 2) {
    search_plan(&st);
    for (int slot = 0; slot < 3; ++slot) st.ccount[slot] = measure(st.cand[slot], seed, span);
    search_decide(&st, k0, iters, limit, ra, rc);
  }
  print("rnd", st, ra, rc, iters);
  return 0;
}
