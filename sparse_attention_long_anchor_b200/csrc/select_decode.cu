// Exact Top-k of the anchor decode layer with one thread-block cluster per
// (batch, kv head) (Kascade README, Abstract: exact Top-k indices computed in
// the anchor layers; selection is head-aware).
//
// The N candidate keys are split across the kCS CTAs of a cluster; each CTA
// keeps the fp32 pooled scores of its keys in shared memory:
//   P_j = (1/G) sum_g exp2(s2_gj - m2_g) / l_g
// (s2 and the per-split softmax statistics come from the scoring kernel).
// Radix select runs on the fp32 bit patterns with 8-bit digits: every CTA
// histograms its own keys, the histograms are summed over distributed
// shared memory, and every CTA derives the same digit.  The band of keys
// within delta (relative) of the k-th fp32 value is then re-scored in fp64
// (exact bf16 products, fp64 sums and exp2) and settled by (value desc,
// index asc); counts are exchanged over DSMEM and each CTA writes its
// selected keys, ascending, at its prefix offset.  No CTA waits on anything
// but cluster barriers, which every CTA of the cluster reaches.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace kascade {

namespace {

constexpr int kCS = 8;            // CTAs per cluster
constexpr int kCNT = 512;         // threads per CTA
constexpr int kCBins = 256;       // 8-bit digits
constexpr int kSmallBand = 1024;  // band sizes settled by direct ranking
constexpr float kBandDelta = 1.0f / 8192.0f;
constexpr float kBandFloor = 0x1p-96f;

struct CSh {
  unsigned hist[2][kCBins];
  int scan_buf[kCNT / 32 + 1];
  int bin, above;
  int nb, chi;
  int xchg[4];            // published to the cluster: c_hi, nb, ties, selected
  float m2[8];
  double l[8];
  float inv_l[8];
  int b_idx[kSmallBand];
  double b_val[kSmallBand];
};

constexpr size_t kCHead = (sizeof(CSh) + 127) / 128 * 128;

__host__ __device__ constexpr size_t cluster_dyn_bytes(int keys_per_cta) {
  // q rows fp32 [8][128], v[keys] fp32, state[keys] bytes
  return kCHead + 8 * 128 * 4 + (size_t)keys_per_cta * 4 + (size_t)keys_per_cta;
}

// Sum the cluster's histograms (buffer `buf`) and find the digit holding the
// need-th largest element.  Every CTA computes the same (bin, above).
__device__ void cluster_find_bin(cg::cluster_group& cluster, CSh& sh, int buf, int need) {
  __syncthreads();
  cluster.sync();
  const int t = threadIdx.x;
  int local = 0;
  int bin = -1;
  if (t < kCBins) {
    bin = kCBins - 1 - t;   // thread 0 holds the largest digit
#pragma unroll
    for (int r = 0; r < kCS; ++r) {
      const unsigned* rh = cluster.map_shared_rank(&sh.hist[buf][0], r);
      local += (int)rh[bin];
    }
  }
  const int incl = block_inclusive_scan<kCNT>(local, sh.scan_buf, nullptr);
  const int excl = incl - local;
  if (t < kCBins && excl < need && need <= incl) {
    sh.bin = bin;
    sh.above = excl;
  }
  __syncthreads();
}

// zero one histogram buffer; the barrier orders the stores before any
// thread's next atomicAdd into it
__device__ __forceinline__ void clear_hist(CSh& sh, int buf) {
  for (int i = threadIdx.x; i < kCBins; i += kCNT) sh.hist[buf][i] = 0;
  __syncthreads();
}

// exchange one int per CTA: returns the total and the sum over lower ranks
__device__ void cluster_exchange(cg::cluster_group& cluster, CSh& sh, int slot, int mine, int rank,
                                 int* total, int* below) {
  if (threadIdx.x == 0) sh.xchg[slot] = mine;
  __syncthreads();
  cluster.sync();
  int tot = 0, bel = 0;
#pragma unroll
  for (int r = 0; r < kCS; ++r) {
    const int x = *cluster.map_shared_rank(&sh.xchg[slot], r);
    tot += x;
    bel += r < rank ? x : 0;
  }
  *total = tot;
  *below = bel;
}

__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(kCNT)
    select_decode_cluster_kernel(const SelArgs a, int keys_per_cta) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) char smem_raw[];
  CSh& sh = *reinterpret_cast<CSh*>(smem_raw);
  float* qf = reinterpret_cast<float*>(smem_raw + kCHead);
  float* v = qf + 8 * 128;
  uint8_t* st = reinterpret_cast<uint8_t*>(v + keys_per_cta);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv;
  const int G = a.G, D = a.D, N = a.N;
  const int K = topk_count(N, a.num, a.den);
  const int j0 = rank * keys_per_cta;
  const int j1 = min(N, j0 + keys_per_cta);
  const int cnt = max(0, j1 - j0);
  int32_t* out = a.idx + (size_t)bh * K;
  int32_t* band_idx = a.band_idx + (size_t)bh * kCS * keys_per_cta + (size_t)rank * keys_per_cta;
  double* band_val = a.band_val + (size_t)bh * kCS * keys_per_cta + (size_t)rank * keys_per_cta;

  if (K >= N) {   // everything is selected (same branch in every CTA)
    for (int i = tid; i < cnt; i += kCNT) out[j0 + i] = j0 + i;
    return;
  }

  // softmax statistics of the G query heads from the scoring kernel's splits
  for (int g = warp; g < G; g += kCNT / 32) {
    const size_t row = (size_t)(b * a.Hq + h * G + g) * a.splits;
    float m = -INFINITY;
    for (int s = lane; s < a.splits; s += 32) m = fmaxf(m, a.m_part[row + s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    double l = 0.0;
    for (int s = lane; s < a.splits; s += 32) l += a.l_part[row + s] * exp2((double)a.m_part[row + s] - (double)m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      sh.m2[g] = m;
      sh.l[g] = l;
      sh.inv_l[g] = (float)(1.0 / l);
    }
  }
  for (int e = tid; e < G * D; e += kCNT) {
    const int g = e / D, dd = e - g * D;
    qf[e] = __bfloat162float(a.q[(size_t)(b * a.Hq + h * G + g) * D + dd]);
  }
  clear_hist(sh, 0);
  clear_hist(sh, 1);
  __syncthreads();

  // pooled fp32 scores of this CTA's keys + histogram of the top digit
  const float* srow = a.s2 + (size_t)(b * a.Hq + h * G) * N;
  const float invG = 1.0f / (float)G;
  for (int i = tid; i < cnt; i += kCNT) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) acc += exp2f(srow[(size_t)g * N + j0 + i] - sh.m2[g]) * sh.inv_l[g];
    acc *= invG;
    v[i] = acc;
    atomicAdd(&sh.hist[0][__float_as_uint(acc) >> 24], 1u);
  }

  // radix select over the cluster: digits [31:24] [23:16] [15:8] [7:0]
  int need = K;
  unsigned prefix = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const int buf = pass & 1;
    if (pass > 0) {
      for (int i = tid; i < cnt; i += kCNT) {
        const unsigned x = __float_as_uint(v[i]);
        if ((x >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&sh.hist[buf][(x >> shift) & 255u], 1u);
      }
    }
    cluster_find_bin(cluster, sh, buf, need);
    prefix |= (unsigned)sh.bin << shift;
    need -= sh.above;
    clear_hist(sh, buf ^ 1);   // the other buffer's readers have all passed this pass's barrier
  }

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
  for (int i = tid; i < cnt; i += kCNT) {
    const float x = v[i];
    if (x > hi) {
      ++my_hi;
    } else if (x >= lo) {
      band_idx[atomicAdd(&sh.nb, 1)] = j0 + i;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_hi += __shfl_xor_sync(0xffffffffu, my_hi, o);
  if (lane == 0 && my_hi) atomicAdd(&sh.chi, my_hi);
  __syncthreads();
  const int nb = sh.nb, chi = sh.chi;
  int chi_total, chi_below, nb_total, nb_below;
  cluster_exchange(cluster, sh, 0, chi, rank, &chi_total, &chi_below);
  cluster_exchange(cluster, sh, 1, nb, rank, &nb_total, &nb_below);
  const int need_band = K - chi_total;

  // fp64 pooled scores of this CTA's band members, one warp per member
  const double c2 = 1.4426950408889634 / sqrt((double)D);
  const __nv_bfloat16* kb = a.k + (size_t)bh * N * D;
  for (int i = warp; i < nb; i += kCNT / 32) {
    const int j = band_idx[i];
    const __nv_bfloat16* krow = kb + (size_t)j * D;
    float kv[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) kv[t] = lane + 32 * t < D ? __bfloat162float(krow[lane + 32 * t]) : 0.f;
    double total = 0.0;
    for (int g = 0; g < G; ++g) {
      double dot = 0.0;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (lane + 32 * t < D) dot += (double)qf[g * D + lane + 32 * t] * (double)kv[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      total += exp2(dot * c2 - (double)sh.m2[g]) / sh.l[g];
    }
    if (lane == 0) band_val[i] = total / (double)G;
  }
  __threadfence();
  __syncthreads();
  cluster.sync();

  int tie_quota = 0;
  if (nb_total <= kSmallBand) {
    // every CTA gathers the whole band and ranks its own members
    const int32_t* base_idx = a.band_idx + (size_t)bh * kCS * keys_per_cta;
    const double* base_val = a.band_val + (size_t)bh * kCS * keys_per_cta;
    for (int t = tid; t < nb_total; t += kCNT) {
      int r = 0, off = t;
      while (r < kCS) {
        const int nr = *cluster.map_shared_rank(&sh.xchg[1], r);
        if (off < nr) break;
        off -= nr;
        ++r;
      }
      sh.b_idx[t] = __ldcg(base_idx + (size_t)r * keys_per_cta + off);
      sh.b_val[t] = __ldcg(base_val + (size_t)r * keys_per_cta + off);
    }
    __syncthreads();
    for (int i = tid; i < nb; i += kCNT) {
      const int me = nb_below + i;
      const double mv = sh.b_val[me];
      const int mj = sh.b_idx[me];
      int rk = 0;
      for (int t = 0; t < nb_total; ++t) {
        const double ov = sh.b_val[t];
        rk += (ov > mv) || (ov == mv && sh.b_idx[t] < mj);
      }
      st[mj - j0] = rk < need_band ? 1 : 0;
    }
  } else {
    // large band (degenerate inputs): cluster radix select on the fp64 bits
    unsigned long long pre = 0;
    int nd = need_band;
    clear_hist(sh, 0);
    clear_hist(sh, 1);
    __syncthreads();
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      const int buf = pass & 1;
      for (int i = tid; i < nb; i += kCNT) {
        const unsigned long long x = (unsigned long long)__double_as_longlong(band_val[i]);
        if (pass == 0 || (x >> (shift + 8)) == (pre >> (shift + 8)))
          atomicAdd(&sh.hist[buf][(x >> shift) & 255ull], 1u);
      }
      cluster_find_bin(cluster, sh, buf, nd);
      pre |= (unsigned long long)sh.bin << shift;
      nd -= sh.above;
      clear_hist(sh, buf ^ 1);
    }
    const double tau64 = __longlong_as_double((long long)pre);
    int my_ties = 0;
    for (int i = tid; i < nb; i += kCNT) {
      const double x = band_val[i];
      const uint8_t s = x > tau64 ? 1 : (x == tau64 ? 2 : 0);
      st[band_idx[i] - j0] = s;
      my_ties += s == 2;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) my_ties += __shfl_xor_sync(0xffffffffu, my_ties, o);
    if (tid == 0) sh.nb = 0;
    __syncthreads();
    if (lane == 0 && my_ties) atomicAdd(&sh.nb, my_ties);
    __syncthreads();
    int ties_total, ties_below;
    cluster_exchange(cluster, sh, 2, sh.nb, rank, &ties_total, &ties_below);
    tie_quota = min(max(nd - ties_below, 0), sh.nb);   // lower ranks hold lower indices
  }
  __syncthreads();

  // count, exchange offsets, then write ascending
  int mine = 0;
  for (int i = tid; i < cnt; i += kCNT) {
    const float x = v[i];
    mine += x > hi || (x >= lo && st[i] == 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if (tid == 0) sh.chi = 0;
  __syncthreads();
  if (lane == 0 && mine) atomicAdd(&sh.chi, mine);
  __syncthreads();
  int sel_total, sel_below;
  cluster_exchange(cluster, sh, 3, sh.chi + tie_quota, rank, &sel_total, &sel_below);
  int written = sel_below, ties_taken = 0;
  for (int base = 0; base < cnt; base += kCNT) {
    const int i = base + tid;
    int flag = 0, tie = 0;
    if (i < cnt) {
      const float x = v[i];
      if (x > hi) {
        flag = 1;
      } else if (x >= lo) {
        flag = st[i] == 1;
        tie = st[i] == 2;
      }
    }
    if (tie_quota > 0) {
      int tt;
      const int tincl = block_inclusive_scan<kCNT>(tie, sh.scan_buf, &tt);
      if (tie && ties_taken + tincl - 1 < tie_quota) flag = 1;
      ties_taken += tt;
    }
    int total;
    const int incl = block_inclusive_scan<kCNT>(flag, sh.scan_buf, &total);
    if (flag) out[written + incl - 1] = j0 + i;
    written += total;
  }
  // no CTA may leave while another can still read its shared memory
  cluster.sync();
}

}  // namespace

int select_decode_cluster_keys(int N) { return (N + kCS - 1) / kCS; }

bool select_decode_cluster_ok(int N) { return select_decode_cluster_keys(N) <= 16384; }

size_t select_decode_cluster_scratch(int B, int Hkv, int N) {
  return (size_t)B * Hkv * kCS * select_decode_cluster_keys(N);
}

cudaError_t launch_select_decode_cluster(const SelArgs& a, cudaStream_t stream) {
  const int per = select_decode_cluster_keys(a.N);
  const size_t smem = cluster_dyn_bytes(per);
  cudaError_t e = cudaFuncSetAttribute(select_decode_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(kCS, a.B * a.Hkv);
  return launch_ex(select_decode_cluster_kernel, grid, dim3(kCNT), smem, stream, (a.flags & 1) != 0, 1, a, per);
}

}  // namespace kascade
