// Host-side check of the decode work split (kvk_internal.cuh): on random batches, lengths,
// CTA counts and per-piece costs, every token is owned by exactly one CTA, the CTAs' token
// ranges are contiguous and in order, and the pieces the merge combines for a sequence are
// exactly the CTAs that own its tokens (CTAs that own nothing are skipped).  Built and run
// by tests/test_split_host.py; prints "ok <count>" or the first failure.
#include <cstdio>
#include <random>
#include <vector>

#include "kvk_internal.cuh"

int main() {
  std::mt19937 rng(12345);
  long checked = 0;
  for (int trial = 0; trial < 100000; ++trial) {
    const int batch = 1 + rng() % 6, G = 1 + rng() % 40;
    const int X = (trial % 3 == 0) ? 0 : (int)(rng() % 200);
    std::vector<int32_t> off(batch + 1, 0);
    for (int i = 0; i < batch; ++i) off[i + 1] = off[i] + ((rng() % 3 == 0) ? 0 : rng() % 300);
    const int64_t N = off[batch], C = N + (int64_t)X * batch;
    if (C == 0) continue;
    std::vector<int> owner(N, -1);
    int64_t prev = 0;
    for (int c = 0; c < G; ++c) {
      const int64_t lo = kvk::split_token(off.data(), batch, X, kvk::split_cost(c, C, G));
      const int64_t hi = kvk::split_token(off.data(), batch, X, kvk::split_cost(c + 1, C, G));
      if (lo != prev || hi < lo) {
        printf("trial %d: CTA %d range [%lld, %lld) after %lld\n", trial, c, (long long)lo,
               (long long)hi, (long long)prev);
        return 1;
      }
      for (int64_t t = lo; t < hi; ++t) owner[t] = c;
      prev = hi;
    }
    if (prev != N) {
      printf("trial %d: tokens [%lld, %lld) unowned\n", trial, (long long)prev, (long long)N);
      return 1;
    }
    for (int i = 0; i < batch; ++i) {
      const int64_t s0 = off[i], s1 = off[i + 1];
      if (s1 <= s0) continue;
      const int64_t u = (int64_t)X * (i + 1);
      const int c0 = kvk::split_cta(s0 + u, C, G), c1 = kvk::split_cta(s1 - 1 + u, C, G);
      std::vector<int> want, got;
      for (int64_t t = s0; t < s1; ++t)
        if (want.empty() || want.back() != owner[t]) want.push_back(owner[t]);
      for (int c = c0; c <= c1; ++c)
        if (C >= G || kvk::split_cost(c + 1, C, G) > kvk::split_cost(c, C, G)) got.push_back(c);
      if (want != got) {
        printf("trial %d: sequence %d merges %zu pieces, owners %zu (X %d, G %d)\n", trial, i,
               got.size(), want.size(), X, G);
        return 1;
      }
      ++checked;
    }
  }
  printf("ok %ld\n", checked);
  return 0;
}
