// Validation of the index inputs of the attention and refine calls
// (KASCADE_FLAG_CHECK_INDICES), a debugging aid with no counterpart in the
// method itself.
//
// The kernel reads the caller's index lists, head_map and kv_lens and writes
// checked copies into the workspace; the consumer kernels then read the
// copies.  An entry out of its range is raised in the device error word
// (KASCADE_DEVERR_INDEX_LIST) and clamped into range in the copy, so every
// later load stays inside the caller's K and V buffers; a list that is not
// strictly ascending is raised and copied as it is.  The call's results are
// not valid once the word is set.  Nothing traps.
//
// Ranges, for batch row b with n_b keys (kv_lens[b] clamped to [0, N], or N):
//   decode lists    the first ceil(frac n_b) entries in [0, n_b), ascending
//                   (a varlen row's tail past them is copied unchecked);
//   prefill lists   tile t's ceil(frac e_t) entries in [0, e_t),
//                   e_t = min(32 (t + 1), N), ascending;
//   refine pools    all pool_len entries in [0, N), ascending;
//   head_map        [0, lists per row);
//   kv_lens         [1, N].
#include "common.cuh"
#include "kernels.h"

namespace kascade {
namespace {

constexpr int kCheckThreads = 256;
constexpr int kErrIndexList = 7;

__device__ __forceinline__ int row_keys(const CheckArgs& c, int b) {
  return c.kv_lens ? min(max(c.kv_lens[b], 0), c.N) : c.N;
}

// entries [0, cnt) of one list: range [0, bound), strictly ascending
__device__ void check_list(const CheckArgs& c, const int32_t* src, int32_t* dst, int cnt, int bound) {
  bool bad = false;
  for (int i = threadIdx.x; i < cnt; i += kCheckThreads) {
    const int v = src[i];
    const bool in = v >= 0 && v < bound;
    bad |= !in || (i > 0 && src[i - 1] >= v);
    dst[i] = in ? v : min(max(v, 0), max(bound - 1, 0));
  }
  if (bad) raise_error(c.err, kErrIndexList);
}

// blocks [0, B L): one (batch row, list) row each; block B L: head_map and
// kv_lens
__global__ void __launch_bounds__(kCheckThreads) check_lists_kernel(const CheckArgs c) {
  pdl_wait();
  pdl_launch_dependents();
  const int row = blockIdx.x;
  if (row == c.B * c.L) {
    bool bad = false;
    for (int i = threadIdx.x; i < c.n_map; i += kCheckThreads) {
      const int v = c.head_map[i];
      const bool in = v >= 0 && v < c.L;
      bad |= !in;
      c.hm_out[i] = in ? v : 0;
    }
    if (c.kv_lens)
      for (int i = threadIdx.x; i < c.B; i += kCheckThreads) {
        const int v = c.kv_lens[i];
        bad |= v < 1 || v > c.N;
        c.kv_out[i] = min(max(v, 0), c.N);
      }
    if (bad) raise_error(c.err, kErrIndexList);
    return;
  }
  if (!c.idx) return;   // dense form: only head_map and kv_lens
  const int b = row / c.L;
  const int32_t* src = c.idx + (size_t)row * c.row_len;
  int32_t* dst = c.idx_out + (size_t)row * c.row_len;
  if (c.pool) {
    check_list(c, src, dst, (int)c.row_len, c.N);
  } else if (!c.prefill) {
    const int n_b = row_keys(c, b);
    const int cnt = topk_count(n_b, c.num, c.den);
    check_list(c, src, dst, cnt, n_b);
    for (int i = cnt + threadIdx.x; i < c.row_len; i += kCheckThreads) dst[i] = src[i];
  } else {
    const int T = (c.N + 31) / 32;
    for (int t = c.t0; t < T; ++t) {
      const int64_t off = chunk_list_offset(t, c.t0, 32, c.num, c.den);
      const int e_t = min(32 * (t + 1), c.N);
      check_list(c, src + off, dst + off, topk_count(e_t, c.num, c.den), e_t);
    }
  }
}

}  // namespace

cudaError_t launch_check_lists(const CheckArgs& c, cudaStream_t stream) {
  return launch_ex(check_lists_kernel, dim3(c.B * c.L + 1), dim3(kCheckThreads), 0, stream, c.pdl, 1, c);
}

}  // namespace kascade
