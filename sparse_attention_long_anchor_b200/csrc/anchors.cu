// Anchor-layer selection (Kascade README, Abstract: the anchor layers are
// chosen by a dynamic program that maximises cross-layer similarity over a
// development set; Reproducibility, Figure 4, --run_type select_layers).
//
// Two pieces:
//   kascade_index_overlap   per (batch row, list): sum over the tiles of
//                           |A_t and B_t| for two index buffers of one
//                           shape (ascending lists), on the GPU;
//   kascade_plan_anchors    host: given sim[a][l] (layer l's similarity to
//                           an earlier layer a), the M anchors, layer 0
//                           among them, that maximise the sum over layers of
//                           the similarity to the nearest preceding anchor.
// The similarity a caller feeds the planner is its own choice; the overlap
// counts divided by the list length give the index-set overlap.
#include <stdint.h>
#include <string.h>

#include <vector>

#include "../../include/kascade.h"
#include "common.cuh"

namespace kascade {
namespace {

constexpr int kOvThreads = 256;

// one CTA per (batch row, list); tiles in turn; thread per entry of A,
// binary search in B (both ascending)
__global__ void __launch_bounds__(kOvThreads) index_overlap_kernel(const int32_t* __restrict__ a,
                                                                   const int32_t* __restrict__ b, int64_t row_len,
                                                                   int n_tiles, int n_ctx, int num, int den,
                                                                   bool decode, long long* __restrict__ counts) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ long long warp_sum[kOvThreads / 32];
  const int prob = blockIdx.x;
  const int32_t* ra = a + (size_t)prob * row_len;
  const int32_t* rb = b + (size_t)prob * row_len;
  long long mine = 0;
  for (int t = 0; t < n_tiles; ++t) {
    const int64_t off = decode ? 0 : tile_list_offset(t, 32, num, den);
    const int len = decode ? (int)row_len : topk_count(min(32 * (t + 1), n_ctx), num, den);
    const int32_t* la = ra + off;
    const int32_t* lb = rb + off;
    for (int i = threadIdx.x; i < len; i += kOvThreads) {
      const int32_t x = la[i];
      int lo = 0, hi = len;   // first position in B with value >= x
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (lb[mid] < x) lo = mid + 1;
        else hi = mid;
      }
      mine += lo < len && lb[lo] == x;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    for (int w = 0; w < kOvThreads / 32; ++w) tot += warp_sum[w];
    counts[prob] = tot;
  }
}

}  // namespace
}  // namespace kascade

using namespace kascade;

extern "C" {

int kascade_index_overlap(const kascade_shape* s, const int32_t* a, const int32_t* b, int64_t* counts,
                          void* stream) {
  const int64_t total = kascade_index_count(s);
  if (total < 0) return kascade_select(s, nullptr, nullptr, nullptr, nullptr, 0, nullptr);   // the shape's status
  if (!a || !b || !counts) return KASCADE_ERR_INVALID_ARG;
  if (((uintptr_t)a | (uintptr_t)b) % 4 || (uintptr_t)counts % 8) return KASCADE_ERR_UNSUPPORTED;
  const int lists = s->select_mode == KASCADE_SELECT_PER_HEAD   ? s->num_q_heads
                    : s->select_mode == KASCADE_SELECT_ALL_HEADS ? 1
                                                                 : s->num_kv_heads;
  const int problems = s->batch * lists;
  const int64_t row_len = total / problems;
  const bool decode = s->q_len == 1;
  const int n_tiles = decode ? 1 : (s->kv_len + 31) / 32;
  const cudaError_t e =
      launch_ex(index_overlap_kernel, dim3(problems), dim3(kOvThreads), 0, static_cast<cudaStream_t>(stream),
                (s->flags & KASCADE_FLAG_PDL) != 0, 1, a, b, row_len, n_tiles, s->kv_len, s->topk_num, s->topk_den,
                decode, reinterpret_cast<long long*>(counts));
  return e == cudaSuccess ? KASCADE_OK : KASCADE_ERR_CUDA;
}

int kascade_plan_anchors(const double* sim, int32_t n_layers, int32_t n_anchors, int32_t* anchors,
                         double* objective) {
  if (!sim || !anchors || n_layers < 1 || n_anchors < 1 || n_anchors > n_layers) return KASCADE_ERR_INVALID_ARG;
  const int L = n_layers, M = n_anchors;
  // run[j][i] = sum_{l = j}^{i - 1} sim[j][l]: layers j .. i-1 reusing anchor j
  std::vector<double> pre((size_t)L * (L + 1), 0.0);
  for (int j = 0; j < L; ++j)
    for (int i = j; i < L; ++i) pre[(size_t)j * (L + 1) + i + 1] = pre[(size_t)j * (L + 1) + i] + sim[(size_t)j * L + i];
  auto run = [&](int j, int i) { return pre[(size_t)j * (L + 1) + i] - pre[(size_t)j * (L + 1) + j]; };
  // best[m][j]: layers j.. with an anchor at j and m more after it;
  // nxt[m][j]: where the next anchor goes (smallest on ties)
  std::vector<double> best((size_t)M * L, 0.0);
  std::vector<int> nxt((size_t)M * L, -1);
  for (int j = 0; j < L; ++j) best[j] = run(j, L);
  for (int m = 1; m < M; ++m) {
    for (int j = 0; j < L; ++j) {
      double bv = 0.0;
      int bi = -1;
      for (int i = j + 1; i <= L - m; ++i) {
        const double v = run(j, i) + best[(size_t)(m - 1) * L + i];
        if (bi < 0 || v > bv) {
          bv = v;
          bi = i;
        }
      }
      best[(size_t)m * L + j] = bv;
      nxt[(size_t)m * L + j] = bi;
    }
  }
  int j = 0;
  for (int m = M - 1; m >= 0; --m) {
    anchors[M - 1 - m] = j;
    if (m > 0) j = nxt[(size_t)m * L + j];
  }
  if (objective) *objective = best[(size_t)(M - 1) * L + 0];
  return KASCADE_OK;
}

}  // extern "C"
