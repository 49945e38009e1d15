// Cluster sizes of the decode select and the sparse decode (host side, plain
// C++ with no CUDA dependency, so the rules are unit-tested on the CPU).
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

// Short-list sparse decode: a launch is latency-bound and, with programmatic
// dependent launch, the next launch's clusters start early and gather their
// rows while this one runs, but only if both launches' clusters are resident
// at once.  So the largest size at which twice the problems fit the device
// (active >= 2 problems) is taken; else the largest at which all problems
// run in one wave; else 0 (the caller's long-list mode, which moves more
// keys per CTA, takes over).
inline int choose_overlap_cluster_size(long long problems, const int* sizes, const int* active, const bool* fits,
                                       int n) {
  for (int i = 0; i < n; ++i)
    if (fits[i] && active[i] > 0 && (long long)active[i] >= 2 * problems) return sizes[i];
  for (int i = 0; i < n; ++i)
    if (fits[i] && active[i] > 0 && (long long)active[i] >= problems) return sizes[i];
  return 0;
}

// Waves that `problems` clusters of the chosen size take (0 if `chosen` is
// not one of sizes[] or none of it runs).
inline long long cluster_waves(long long problems, const int* sizes, const int* active, int n, int chosen) {
  for (int i = 0; i < n; ++i)
    if (sizes[i] == chosen && active[i] > 0) return problems <= 0 ? 1 : (problems + active[i] - 1) / active[i];
  return 0;
}

// The fused decode select keeps a problem's scores on chip and runs its
// Top-k right after the scoring, so the SMs of a finished wave wait out the
// Top-k of the slowest cluster before the next wave's K stream starts.  It
// is taken only when every problem runs in one wave; with more, scoring into
// global memory at full occupancy and selecting in a second kernel is
// faster (batch 8 of the 8-kv-head shape at 64K keys: 271 us against 348).
inline int choose_fused_select_size(long long problems, const int* sizes, const int* active, const bool* fits,
                                    int n) {
  const int cs = choose_cluster_size(problems, sizes, active, fits, n);
  return cs && cluster_waves(problems, sizes, active, n, cs) == 1 ? cs : 0;
}

}  // namespace kascade
