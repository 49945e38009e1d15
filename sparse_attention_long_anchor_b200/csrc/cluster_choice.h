// Cluster size of the fused decode select (host side, plain C++ with no CUDA
// dependency, so the rule is unit-tested on the CPU).
//
// One thread-block cluster handles one (batch, kv head) problem; its CTAs
// split the problem's keys, so K streams at a rate that grows with the
// cluster size, while the Top-k that follows is latency-bound.  How many
// clusters of each size run at once is a property of the device (a cluster
// must sit inside one GPC).  The rule: the fewest waves of `problems`
// clusters, then the largest size among those.
#pragma once

namespace kascade {

// sizes[i] in decreasing order; active[i] = clusters of sizes[i] that run at
// once on the device (<= 0: none); fits[i] = the kernel's shared memory at
// that size fits one SM.  Returns the chosen size, or 0 if none qualifies.
inline int choose_cluster_size(long long problems, const int* sizes, const int* active, const bool* fits, int n) {
  int best = 0;
  long long best_waves = 0;
  for (int i = 0; i < n; ++i) {
    if (active[i] <= 0 || !fits[i]) continue;
    const long long waves = problems <= 0 ? 1 : (problems + active[i] - 1) / active[i];
    if (best == 0 || waves < best_waves) {
      best = sizes[i];
      best_waves = waves;
    }
  }
  return best;
}

}  // namespace kascade
