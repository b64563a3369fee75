// Task numbering of the dataflow factorisation in prepare.cu, for the host
// and the device: the CTAs of the one launch take tasks by number (an atomic
// counter), and a number must map to its tile task in O(log N).
//
// With N 64-column block steps, slot s holds the factor tasks of step s
// (r = N − s − 1 block rows below it):
//   PANEL(s,i)    i = s+2 .. N−1             (r − 1 tasks)
//   TRAIL(s,i,s+1) i = s+2 .. N−1            (r − 1 tasks)
//   TRAIL(s,i,j)  s+2 ≤ j ≤ i ≤ N−1, row by row  (r(r−1)/2 tasks)
// and then the inverse tasks of step k = s − kMLag (r = N − k − 1):
//   MROW(k,c)     c = 0 .. k−1               (k tasks)
//   MTRAIL(k,k+1,c) c = 0 .. k               (k + 1 tasks, none when r = 0)
//   MTRAIL(k,i,c) i = k+2 .. N−1, c = 0 .. k (row by row)
// The chain CTA itself does DIAG(s), PANEL(s,s+1) and TRAIL(s,s+1,s+1).
#pragma once

#include <cmath>
#include <cstdint>

namespace gptq {

constexpr int kMLag = 2;

enum TaskKind { T_PANEL = 0, T_MROW, T_TRAIL, T_MTRAIL };

__host__ __device__ inline int64_t factor_tasks(int N, int k) {
  const int64_t r = N - k - 1;
  return r <= 0 ? 0 : 2 * (r - 1) + (r - 1) * r / 2;
}
__host__ __device__ inline int64_t inverse_tasks(int N, int k) {
  const int64_t r = N - k - 1;
  return r <= 0 ? k : k + (k + 1) + (r - 1) * (k + 1);
}
__host__ __device__ inline int64_t slot_tasks(int N, int s) {
  return (s < N ? factor_tasks(N, s) : 0) +
         (s >= kMLag && s - kMLag < N ? inverse_tasks(N, s - kMLag) : 0);
}
__host__ __device__ inline int task_slots(int N) { return N + kMLag; }

// prefix[s] = tasks in slots before s, s = 0 .. task_slots(N) (the last entry
// is the total).  The caller keeps the total below 2^31.
__host__ __device__ inline void build_slot_prefix(int N, int* prefix) {
  int64_t t = 0;
  for (int s = 0; s < task_slots(N); ++s) {
    prefix[s] = (int)t;
    t += slot_tasks(N, s);
  }
  prefix[task_slots(N)] = (int)t;
}

inline int64_t total_tasks(int N) {
  int64_t t = 0;
  for (int s = 0; s < task_slots(N); ++s) t += slot_tasks(N, s);
  return t;
}

// Row ii of the lower-triangle enumeration (ii·(ii+1)/2 ≤ t < (ii+1)·(ii+2)/2).
__host__ __device__ inline int64_t tri_row(int64_t t) {
  int64_t ii = (int64_t)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while ((ii + 1) * (ii + 2) / 2 <= t) ++ii;
  while (ii > 0 && ii * (ii + 1) / 2 > t) --ii;
  return ii;
}

// Task number → (kind, k, i, j); for MROW and MTRAIL j is the column block c.
__host__ __device__ inline void decode_task(int task, int N, const int* prefix, int& kind,
                                            int& k, int& i, int& j) {
  int lo = 0, hi = task_slots(N);            // prefix[lo] ≤ task < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= task) lo = mid; else hi = mid;
  }
  const int s = lo;
  int64_t t = task - prefix[s];
  if (s < N) {
    const int64_t nf = factor_tasks(N, s);
    if (t < nf) {
      k = s;
      const int64_t r = N - k - 1;
      if (t < r - 1) { kind = T_PANEL; i = (int)(k + 2 + t); j = k; return; }
      t -= r - 1;
      if (t < r - 1) { kind = T_TRAIL; i = (int)(k + 2 + t); j = k + 1; return; }
      t -= r - 1;
      const int64_t ii = tri_row(t);
      kind = T_TRAIL;
      i = (int)(k + 2 + ii);
      j = (int)(k + 2 + (t - ii * (ii + 1) / 2));
      return;
    }
    t -= nf;
  }
  k = s - kMLag;
  const int r = N - k - 1;
  if (r <= 0 || t < k) { kind = T_MROW; i = k; j = (int)t; return; }
  t -= k;
  if (t < k + 1) { kind = T_MTRAIL; i = k + 1; j = (int)t; return; }
  t -= k + 1;
  kind = T_MTRAIL;
  i = (int)(k + 2 + t / (k + 1));
  j = (int)(t % (k + 1));
}

}  // namespace gptq
