// Exact Top-k selection over pooled post-softmax scores (Kascade README,
// Abstract: "exact Top-k indices" in the anchor layers; strategy
// post_softmax_pooled_prefill_topk).
//
// One problem = one (batch, kv head) in decode or one (batch, kv head, query
// tile) in prefill: n candidate keys with pooled scores P_j >= 0, pick the k
// largest, equal scores going to the lower index, write them ascending.
//
// 1. fp32 pooled values v_j (decode: from the raw scores and softmax stats;
//    prefill: read from the score-and-pool kernel's output).
// 2. Radix select on the fp32 bit patterns (non-negative floats order like
//    their uint32 patterns): three histogram passes of 11/11/10 bits in shared
//    memory give the exact k-th largest fp32 value tau.
// 3. Keys with v in [tau (1 - delta), tau (1 + delta)] form the band; v is
//    accurate to far better than delta/3 relative, so keys above the band are
//    certainly in the true Top-k and keys below it certainly out.  Band
//    members get their pooled score recomputed in fp64 from the bf16 inputs
//    (exact products, fp64 sums, fp64 exp2) and the remaining slots go to the
//    largest of those, lower index first on equal values.
// 4. One ascending pass over the keys writes the selected indices with a
//    block-wide prefix sum.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace kascade {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelCtasPerSM = 4;   // problems in flight per SM
constexpr int kBins = 2048;
constexpr float kBandDelta = 1.0f / 8192.0f;
constexpr float kBandFloor = 0x1p-96f;   // below this fp32 exp2 underflow may hide mass
constexpr int kMaxD = 128;
constexpr int kMaxHeads = 64;   // query heads one problem may pool (all heads of a row)

struct SelShared {
  unsigned hist[kBins];
  int scan_buf[kSelThreads / 32 + 1];
  int bin, above;
  int nb, chi;
  int need_eq_ticket;
  float m2[kMaxHeads];
  double l[kMaxHeads];
  float inv_l[kMaxHeads];
  int b_idx[kSelThreads];
  double b_val[kSelThreads];
};

// dynamic shared memory after SelShared (rounded up to 128 bytes): decode q
// rows as float [heads][D], then a per-warp key row as double [warps][D]
constexpr size_t kSelHead = (sizeof(SelShared) + 127) / 128 * 128;
constexpr size_t kSelQ = (size_t)kMaxHeads * kMaxD * 4;
__host__ __device__ constexpr size_t sel_dyn_bytes() {
  return kSelHead + kSelQ + (size_t)(kSelThreads / 32) * kMaxD * 8;
}

template <int NT>
__device__ void find_bin(const unsigned* hist, int need, SelShared& sh) {
  constexpr int BPT = kBins / NT;
  const int tid = threadIdx.x;
  int local = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) local += (int)hist[kBins - 1 - tid * BPT - i];
  const int incl = block_inclusive_scan<NT>(local, sh.scan_buf, nullptr);
  const int excl = incl - local;
  if (excl < need && need <= incl) {
    int cum = excl;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int bin = kBins - 1 - tid * BPT - i;
      const int hc = (int)hist[bin];
      if (cum + hc >= need) {
        sh.bin = bin;
        sh.above = cum;
        break;
      }
      cum += hc;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void clear_hist(SelShared& sh) {
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) sh.hist[i] = 0;
  __syncthreads();
}

// f(j, v[j]) for j = tid, tid + NT, ... < n.  The loads of kBatch indices
// are issued before any of them is used, so a thread waits on the memory
// latency once per batch rather than once per element (each pass over a
// problem's scores is otherwise a chain of dependent L2 round trips).
constexpr int kBatch = 8;
template <int NT, class F>
__device__ __forceinline__ void for_each_value(const float* v, int n, F&& f) {
  int j = threadIdx.x;
  for (; j + (kBatch - 1) * NT < n; j += kBatch * NT) {
    float x[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) x[u] = v[j + u * NT];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) f(j + u * NT, x[u]);
  }
  for (; j < n; j += NT) f(j, v[j]);
}

// Problem description handed to the per-problem routine.
struct Problem {
  int b, h, t;
  int n, k;
  int i0, rows;            // prefill tile rows [i0, i0 + rows)
  const float* v;          // pooled values (prefill) / scratch (decode)
  int32_t* out;
  const int32_t* cand;     // decode refine: candidate j is key cand[j] (NULL: key j)
};

// element i of a q or k tensor of the input type (0 bf16, 1 fp32, 2 fp16)
__device__ __forceinline__ float elem(const __nv_bfloat16* base, size_t i, int in_type) {
  if (in_type == 1) return __ldg(reinterpret_cast<const float*>(base) + i);
  if (in_type == 2) return __half2float(reinterpret_cast<const __half*>(base)[i]);
  return __bfloat162float(base[i]);
}

// fp64 pooled score of key j, computed by one warp (all lanes return it).
// Head g of the problem is query head p.h G + g, scored against its own kv
// head's key row.
__device__ double refine_decode(const SelArgs& a, const Problem& p, int j, const float* qf,
                                const SelShared& sh, double c2) {
  const int lane = threadIdx.x & 31;
  double total = 0.0;
  for (int g = 0; g < a.G; ++g) {
    const int slab = kv_slab_of(p.b, p.h * a.G + g, a.Hkv, a.Gkv);
    const size_t krow = ((size_t)slab * (p.cand ? a.n_ctx : a.N) + (p.cand ? p.cand[j] : j)) * a.D;
    double dot = 0.0;
    for (int e = lane; e < a.D; e += 32) dot += (double)qf[g * a.D + e] * (double)elem(a.k, krow + e, a.in_type);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    total += exp2(dot * c2 - (double)sh.m2[g]) / sh.l[g];
  }
  return total / (double)a.G;
}

__device__ double refine_prefill(const SelArgs& a, const Problem& p, int j, double* kbuf, double c2) {
  const int lane = threadIdx.x & 31;
  double total = 0.0;
  // the problem's heads [h0, h0 + G), a run of heads per kv head: one key
  // row per run, then the tile's rows of those heads
  const int h0 = p.h * a.G;
  for (int g0 = 0; g0 < a.G;) {
    const int qh0 = h0 + g0;
    const int run = min(a.G - g0, a.Gkv - qh0 % a.Gkv);
    const size_t krow = ((size_t)kv_slab_of(p.b, qh0, a.Hkv, a.Gkv) * a.N + j) * a.D;
    __syncwarp();
    for (int e = lane; e < a.D; e += 32) kbuf[e] = (double)elem(a.k, krow + e, a.in_type);
    __syncwarp();
    const int nrows = run * a.tile;
    for (int r = lane; r < nrows; r += 32) {
      const int g = r / a.tile, il = r - g * a.tile;
      const int i = p.i0 + il;
      if (il >= p.rows || j > i) continue;
      const size_t qoff = ((size_t)(p.b * a.Hq + qh0 + g) * a.Lq + (i - a.q0)) * a.D;
      double dot = 0.0;
      if (a.in_type != 0) {
        for (int e = 0; e < a.D; ++e) dot += (double)elem(a.q, qoff + e, a.in_type) * kbuf[e];
      } else {
        const __nv_bfloat16* qr = a.q + qoff;
        for (int e = 0; e < a.D; e += 2) {
          const __nv_bfloat162 q2 = __ldg(reinterpret_cast<const __nv_bfloat162*>(qr + e));
          dot += (double)__low2float(q2) * kbuf[e] + (double)__high2float(q2) * kbuf[e + 1];
        }
      }
      const size_t srow = (size_t)(p.b * a.Hq + qh0 + g) * a.Lq + (i - a.q0);
      total += exp2(dot * c2 - (double)a.row_m2[srow]) / a.row_l[srow];
    }
    g0 += run;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  __syncwarp();
  return total / (double)(a.G * p.rows);
}

template <int NT>
__device__ void run_problem(const SelArgs& a, Problem& p, SelShared& sh, float* vscr,
                            int32_t* band_idx, double* band_val, uint8_t* state, char* dyn) {
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const double c2 = 1.4426950408889634 / sqrt((double)a.D);

  // fast path: everything is selected
  if (p.k >= p.n) {
    for (int j = tid; j < p.n; j += NT) p.out[j] = p.cand ? p.cand[j] : j;
    return;
  }

  float* qf = reinterpret_cast<float*>(dyn);                      // decode
  double* kbuf = reinterpret_cast<double*>(dyn + kSelQ) + warp * kMaxD;

  const float* v = p.v;
  clear_hist(sh);
  if (!a.prefill) {
    // combine split statistics of the G query heads (fp64), a warp per head
    for (int hw = warp; hw < a.G; hw += NT / 32) {
      const size_t row = (size_t)(p.b * a.Hq + p.h * a.G + hw) * a.splits;
      float m = -INFINITY;
      for (int s = lane; s < a.splits; s += 32) m = fmaxf(m, a.m_part[row + s]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      double l = 0.0;
      for (int s = lane; s < a.splits; s += 32)
        l += a.l_part[row + s] * exp2((double)a.m_part[row + s] - (double)m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) {
        sh.m2[hw] = m;
        sh.l[hw] = l;
        sh.inv_l[hw] = (float)(1.0 / l);
      }
    }
    for (int e = tid; e < a.G * a.D; e += NT) {
      const int g = e / a.D, dd = e - g * a.D;
      qf[e] = elem(a.q, (size_t)(p.b * a.Hq + p.h * a.G + g) * a.D + dd, a.in_type);
    }
    __syncthreads();
    const float* srow = a.s2 + (size_t)(p.b * a.Hq + p.h * a.G) * a.N;
    const float invG = 1.0f / (float)a.G;
    for (int j = tid; j < p.n; j += NT) {
      float acc = 0.f;
      for (int g = 0; g < a.G; ++g) acc += exp2f(srow[(size_t)g * a.N + j] - sh.m2[g]) * sh.inv_l[g];
      acc *= invG;
      vscr[j] = acc;
      atomicAdd(&sh.hist[__float_as_uint(acc) >> 21], 1u);
    }
    v = vscr;
  } else {
    for_each_value<NT>(v, p.n, [&](int, float x) { atomicAdd(&sh.hist[__float_as_uint(x) >> 21], 1u); });
  }
  __syncthreads();

  // radix select: bits [31:21], [20:10], [9:0]
  int need = p.k;
  unsigned prefix = 0;
  find_bin<NT>(sh.hist, need, sh);
  prefix = (unsigned)sh.bin << 21;
  need -= sh.above;
  __syncthreads();
  clear_hist(sh);
  for_each_value<NT>(v, p.n, [&](int, float xf) {
    const unsigned x = __float_as_uint(xf);
    if ((x >> 21) == (prefix >> 21)) atomicAdd(&sh.hist[(x >> 10) & 2047u], 1u);
  });
  __syncthreads();
  find_bin<NT>(sh.hist, need, sh);
  prefix |= (unsigned)sh.bin << 10;
  need -= sh.above;
  __syncthreads();
  clear_hist(sh);
  for_each_value<NT>(v, p.n, [&](int, float xf) {
    const unsigned x = __float_as_uint(xf);
    if ((x >> 10) == (prefix >> 10)) atomicAdd(&sh.hist[x & 1023u], 1u);
  });
  __syncthreads();
  find_bin<NT>(sh.hist, need, sh);
  prefix |= (unsigned)sh.bin;
  __syncthreads();

  // band around the k-th fp32 value
  const float tau = __uint_as_float(prefix);
  const float lo = tau < kBandFloor ? 0.0f : tau * (1.0f - kBandDelta);
  const float hi = fmaxf(tau * (1.0f + kBandDelta), kBandFloor);
  if (tid == 0) {
    sh.nb = 0;
    sh.chi = 0;
  }
  __syncthreads();
  int my_hi = 0;
  for_each_value<NT>(v, p.n, [&](int j, float x) {
    if (x > hi) {
      ++my_hi;
    } else if (x >= lo) {
      const int pos = atomicAdd(&sh.nb, 1);
      band_idx[pos] = j;
    }
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_hi += __shfl_xor_sync(0xffffffffu, my_hi, o);
  if (lane == 0) atomicAdd(&sh.chi, my_hi);
  __syncthreads();
  const int nb = sh.nb;
  const int need_band = p.k - sh.chi;

  // fp64 pooled scores of the band members, one warp per member
  for (int i = warp; i < nb; i += NT / 32) {
    const int j = band_idx[i];
    const double val = a.prefill ? refine_prefill(a, p, j, kbuf, c2)
                                 : refine_decode(a, p, j, qf, sh, c2);
    if (lane == 0) band_val[i] = val;
  }
  __syncthreads();

  int need_tie = 0;
  if (nb <= NT) {
    // rank by (value desc, index asc)
    if (tid < nb) {
      sh.b_idx[tid] = band_idx[tid];
      sh.b_val[tid] = band_val[tid];
    }
    __syncthreads();
    if (tid < nb) {
      const double my_v = sh.b_val[tid];
      const int my_j = sh.b_idx[tid];
      int rank = 0;
      for (int m = 0; m < nb; ++m) {
        const double ov = sh.b_val[m];
        rank += (ov > my_v) || (ov == my_v && sh.b_idx[m] < my_j);
      }
      state[my_j] = rank < need_band ? 1 : 0;
    }
  } else {
    // radix select on the fp64 bit patterns: 11-bit digits from bit 63 down
    unsigned long long pre = 0;
    int nd = need_band;
    const int shifts[6] = {53, 42, 31, 20, 9, 0};
    for (int pass = 0; pass < 6; ++pass) {
      const int sft = shifts[pass];
      clear_hist(sh);
      for (int i = tid; i < nb; i += NT) {
        const unsigned long long x = (unsigned long long)__double_as_longlong(band_val[i]);
        const bool match = pass == 0 || (x >> (shifts[pass - 1])) == (pre >> (shifts[pass - 1]));
        if (match) atomicAdd(&sh.hist[(x >> sft) & 2047ull], 1u);
      }
      __syncthreads();
      find_bin<NT>(sh.hist, nd, sh);
      pre |= (unsigned long long)sh.bin << sft;
      nd -= sh.above;
      __syncthreads();
    }
    const double tau64 = __longlong_as_double((long long)pre);
    need_tie = nd;
    for (int i = tid; i < nb; i += NT) {
      const double x = band_val[i];
      state[band_idx[i]] = x > tau64 ? 1 : (x == tau64 ? 2 : 0);
    }
  }
  __syncthreads();

  // ascending compaction
  if (need_tie == 0) {
    // warp w owns the consecutive keys [s0, s1) and walks them 32 at a time
    // (coalesced loads, ballot counts): one pass counts, the warps' counts
    // give each warp its output offset, a second pass writes
    constexpr int W = NT / 32;
    constexpr int C = 4;   // 32-key chunks whose loads are in flight together
    const int seg = ((p.n + W - 1) / W + 31) & ~31;
    const int s0 = min(p.n, warp * seg), s1 = min(p.n, s0 + seg);
    auto flags = [&](int base, uint32_t (&m)[C]) {
      float x[C];
#pragma unroll
      for (int u = 0; u < C; ++u) {
        const int j = base + 32 * u + lane;
        x[u] = j < s1 ? v[j] : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < C; ++u) {
        const int j = base + 32 * u + lane;
        const bool f = j < s1 && (x[u] > hi || (x[u] >= lo && state[j] == 1));
        m[u] = __ballot_sync(0xffffffffu, f);
      }
    };
    int c = 0;
    for (int base = s0; base < s1; base += 32 * C) {
      uint32_t m[C];
      flags(base, m);
#pragma unroll
      for (int u = 0; u < C; ++u) c += __popc(m[u]);
    }
    if (lane == 0) sh.scan_buf[warp] = c;
    __syncthreads();
    int w = 0;
#pragma unroll
    for (int u = 0; u < W; ++u) w += u < warp ? sh.scan_buf[u] : 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int base = s0; base < s1; base += 32 * C) {
      uint32_t m[C];
      flags(base, m);
#pragma unroll
      for (int u = 0; u < C; ++u) {
        const int j = base + 32 * u + lane;
        if ((m[u] >> lane) & 1u) p.out[w + __popc(m[u] & lt)] = p.cand ? p.cand[j] : j;
        w += __popc(m[u]);
      }
    }
    return;
  }
  int written = 0, ties_taken = 0;
  for (int base = 0; base < p.n; base += NT) {
    const int j = base + tid;
    int flag = 0, tie = 0;
    if (j < p.n) {
      const float x = v[j];
      if (x > hi) {
        flag = 1;
      } else if (x >= lo) {
        const uint8_t st = state[j];
        flag = st == 1;
        tie = st == 2;
      }
    }
    if (need_tie > 0) {
      int ties_total;
      const int tincl = block_inclusive_scan<NT>(tie, sh.scan_buf, &ties_total);
      if (tie && ties_taken + tincl - 1 < need_tie) flag = 1;
      ties_taken += ties_total;
    }
    int total;
    const int incl = block_inclusive_scan<NT>(flag, sh.scan_buf, &total);
    if (flag) p.out[written + incl - 1] = p.cand ? p.cand[j] : j;
    written += total;
  }
}

template <int NT>
__global__ void __launch_bounds__(NT, kSelCtasPerSM) select_kernel(const SelArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) char smem_raw[];
  SelShared& sh = *reinterpret_cast<SelShared*>(smem_raw);
  char* dyn = smem_raw + kSelHead;
  const int cta = blockIdx.x;
  float* vscr = a.v_scratch ? a.v_scratch + (size_t)cta * a.n_max : nullptr;
  int32_t* band_idx = a.band_idx + (size_t)cta * a.n_max;
  double* band_val = a.band_val + (size_t)cta * a.n_max;
  uint8_t* state = a.state + (size_t)cta * a.n_max;

  const int BH = a.B * a.Hp;   // problems: (batch row, problem of the row)
  if (!a.prefill) {
    // with candidates, N counts the candidates and k follows the context
    const int64_t K = topk_count(a.cand ? a.n_ctx : a.N, a.num, a.den);
    for (int prob = cta; prob < BH; prob += gridDim.x) {
      Problem p;
      p.b = prob / a.Hp;
      p.h = prob - p.b * a.Hp;
      p.t = 0;
      p.n = a.N;
      p.k = (int)K;
      if (a.kv_lens) {   // varlen row: its own candidates and budget
        p.n = min(a.N, a.kv_lens[p.b]);
        p.k = topk_count(p.n, a.num, a.den);
      }
      p.cand = nullptr;
      if (a.cand) {
        int hm = a.cand_map ? a.cand_map[p.h] : p.h;
        if (hm < 0 || hm >= a.cand_lists) hm = 0;
        p.cand = a.cand + (size_t)(p.b * a.cand_lists + hm) * a.N;
      }
      p.i0 = 0;
      p.rows = 1;
      p.v = vscr;
      p.out = a.idx + (size_t)prob * K;
      run_problem<NT>(a, p, sh, vscr, band_idx, band_val, state, dyn);
      for (int j = p.k + threadIdx.x; j < K; j += NT) p.out[j] = -1;   // a varlen row's unused tail
      __syncthreads();
    }
  } else {
    const int T = (a.N + a.tile - 1) / a.tile;
    const int t0 = a.q0 / a.tile;   // first query tile of the call (rolling chunks)
    const int64_t row_len = chunk_row_len(a.N, t0, a.tile, a.num, a.den);
    const int64_t pooled_len = chunk_pooled_len(a.N, t0, a.tile);
    const int64_t total = (int64_t)(T - t0) * BH;
    for (int64_t prob = cta; prob < total; prob += gridDim.x) {
      const int t = T - 1 - (int)(prob / BH);   // longest tiles first
      const int bh = (int)(prob % BH);
      Problem p;
      p.b = bh / a.Hp;
      p.h = bh - p.b * a.Hp;
      p.t = t;
      p.i0 = t * a.tile;
      p.n = min((t + 1) * a.tile, a.N);
      p.rows = p.n - p.i0;
      p.k = topk_count(p.n, a.num, a.den);
      p.v = a.pooled + (size_t)bh * pooled_len + chunk_pooled_offset(t, t0, a.tile);
      p.cand = nullptr;
      p.out = a.idx + (size_t)bh * row_len + chunk_list_offset(t, t0, a.tile, a.num, a.den);
      run_problem<NT>(a, p, sh, vscr, band_idx, band_val, state, dyn);
      __syncthreads();
    }
  }
}

}  // namespace

// pooled scores of all heads: the mean over a batch row's kv-head rows (each
// already the mean over its G query heads, so this is the mean over all Hq)
__global__ void pool_mean_kernel(const float* __restrict__ in, float* __restrict__ out, int Hkv, int64_t row) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const float inv = 1.0f / (float)Hkv;
  for (int64_t x = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; x < row; x += (int64_t)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int h = 0; h < Hkv; ++h) acc += in[((int64_t)b * Hkv + h) * row + x];
    out[(int64_t)b * row + x] = acc * inv;
  }
}

cudaError_t launch_pool_mean(const float* in, float* out, int B, int Hkv, int64_t row, int flags,
                             cudaStream_t stream) {
  int blocks = (int)((row + 255) / 256);
  if (blocks > 4096) blocks = 4096;
  return launch_ex(pool_mean_kernel, dim3(blocks, B), dim3(256), 0, stream, (flags & 1) != 0, 1, in, out, Hkv, row);
}

size_t select_scratch_bytes_per_cta(int n_max) {
  return (size_t)n_max * (sizeof(float) + sizeof(int32_t) + sizeof(double) + 1);
}

int select_grid(bool prefill, int problems, int num_sms) {
  (void)prefill;
  const int cap = num_sms * kSelCtasPerSM;
  return problems < cap ? problems : cap;
}

cudaError_t launch_select(const SelArgs& a, cudaStream_t stream) {
  const size_t smem = sel_dyn_bytes();
  const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(select_kernel<kSelThreads>), smem, false);
  if (e != cudaSuccess) return e;
  return launch_ex(select_kernel<kSelThreads>, dim3(a.grid), dim3(kSelThreads), smem, stream, (a.flags & 1) != 0, 1, a);
}

}  // namespace kascade
