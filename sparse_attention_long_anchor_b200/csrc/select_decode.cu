// Exact Top-k of the anchor decode layer with one thread-block cluster per
// (batch, kv head) (Kascade README, Abstract: exact Top-k indices computed in
// the anchor layers; selection is head-aware).
//
// The N candidate keys are split across the CS CTAs of a cluster; each CTA
// keeps the fp32 pooled scores of its keys in shared memory:
//   P_j = (1/G) sum_g exp2(s2_gj - m2_g) / l_g,   s2 = q . k_j log2(e)/sqrt(d)
// Two kernels produce them:
//   * anchor_select_kernel (the usual path) streams the CTA's contiguous K
//     rows into shared memory with bulk TMA copies, scores them with warp
//     MMAs (keys as the MMA rows, the <= 8 query heads of the group as its
//     columns), keeps the scores in shared memory and takes the softmax
//     statistics of every head over the cluster through distributed shared
//     memory: one launch, no score round trip through global memory.
//     The cluster size (16, 12, 10, 9 or 8 CTAs) is chosen per device and
//     shape by choose_cluster_size;
//   * select_decode_cluster_kernel (fallback for contexts too long to keep
//     the scores on chip at any of those sizes) reads the scores and
//     per-split statistics written by the scoring kernel.
// Both then run the same cluster Top-k: radix select on the top 24 bits of
// the fp32 bit patterns (three 8-bit digits), histograms, counts and band
// entries sent to every CTA of the cluster with one-sided stores into its
// shared memory; the band of keys within delta (relative) of the 2^-15-wide
// bin holding the k-th fp32 value is re-scored in fp64 (exact bf16
// products, fp64 sums and exp2) and settled by (value desc, index asc); each
// CTA writes its selected keys, ascending, at its prefix offset.
#include <cooperative_groups.h>

#include "cluster_choice.h"
#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace kascade {

namespace {

constexpr int kCNT = 512;         // threads per CTA
constexpr int kWarpsC = kCNT / 32;
constexpr int kCBins = 256;       // 8-bit digits
constexpr int kSmallBand = 1024;  // band sizes settled by direct ranking
constexpr float kBandDelta = 1.0f / 8192.0f;
constexpr float kBandFloor = 0x1p-96f;
constexpr int kFallbackCS = 8;    // cluster size of the fallback kernel
constexpr int kRoundKeys = 256;   // fused kernel: K rows per streamed round
constexpr int kSlots = 2;         // fused kernel: rounds in flight
constexpr int kErrTimeout = 5;
constexpr int kMaxCS = 16;        // largest cluster
constexpr int kRadixPasses = 3;   // 8-bit digits [31:24] [23:16] [15:8]
// exchange barriers: one per radix pass, counts, band entries, softmax stats
constexpr int kBarCnt = kRadixPasses, kBarBand = kRadixPasses + 1, kBarStats = kRadixPasses + 2;
constexpr int kNumXBars = kRadixPasses + 3;
constexpr size_t kRxBytes(int cs) { return (size_t)kRadixPasses * cs * 256 * 4; }   // radix receive slots

struct CSh {
  unsigned hist[2][kCBins];   // large-band path: fp64 radix histograms, read by the cluster
  int scan_buf[kCNT / 32 + 1];
  int bin, above;
  int nb, chi;
  int xchg[4];            // large-band path, read by the cluster: slots 2 (ties) and 3 (selected)
  float m2[8];
  double l[8];
  float inv_l[8];
  float wpool[8];         // fused: weight exp2(cmax - m2) / l of the stored terms
  float wmax[kWarpsC][8];
  double wsum[kWarpsC][8];
  unsigned long long full[kSlots];   // fused: K round barriers
  unsigned long long xbar[kNumXBars];  // one-sided exchanges (see exchange_init)
  // slot r of these arrays is written by CTA r of the cluster
  int2 rx_cnt[kMaxCS];               // (count above the band, band size)
  float rx_cmax[kMaxCS][8];          // fused: CTA r's max score of each head
  double rx_csum[kMaxCS][8];         // fused: CTA r's sum of exp2(s2 - max) of each head
  int b_idx[kSmallBand];             // the cluster's band, ordered by CTA rank
  double b_val[kSmallBand];
};

constexpr size_t kCHead = (sizeof(CSh) + 127) / 128 * 128;

// Exchanges between the CTAs of a cluster are one-sided: each CTA stores its
// share into every other CTA's shared memory with st.async, which completes
// on the receiver's mbarrier, and the receiver waits on its own barrier only
// (no cluster-wide barrier, no remote loads).  Thread 0 sets the barriers up
// with the bytes of every fixed-size exchange; the band's size is added once
// the counts are known.  The caller then arrives on the cluster barrier and
// waits on it before its first store into another CTA, which orders the
// initialisation before any remote completion.
template <int CS>
__device__ void exchange_init(CSh& sh, int stats_bytes_per_cta) {
  const uint32_t xb = smem_u32(&sh.xbar[0]);
  for (int i = 0; i < kNumXBars; ++i) mbar_init(xb + 8u * i, 1);
  mbar_fence_init();
  for (int p = 0; p < kRadixPasses; ++p) mbar_arrive_expect_tx(xb + 8u * p, (CS - 1) * kCBins * 4);
  mbar_arrive_expect_tx(xb + 8u * kBarCnt, (CS - 1) * 8);
  if (stats_bytes_per_cta > 0) mbar_arrive_expect_tx(xb + 8u * kBarStats, (CS - 1) * stats_bytes_per_cta);
}

__device__ __forceinline__ int peer_of(int rank, int l, int cs) { return rank + l < cs ? rank + l : rank + l - cs; }

// Thread t < 256 holds c, the count of digit 255 - t; find the digit holding
// the need-th largest element into (sh.bin, sh.above): a scan over the eight
// warps that hold digits, two barriers.
__device__ __forceinline__ void find_digit(CSh& sh, int c, int need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int x = c;
  if (warp < kCBins / 32) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh.scan_buf[warp] = x;
  }
  __syncthreads();
  if (warp < kCBins / 32) {
    int pre = 0;
#pragma unroll
    for (int w = 0; w < kCBins / 32 - 1; ++w) pre += w < warp ? sh.scan_buf[w] : 0;
    const int incl = pre + x, excl = incl - c;
    if (excl < need && need <= incl) {
      sh.bin = kCBins - 1 - tid;
      sh.above = excl;
    }
  }
  __syncthreads();
}

// exclusive prefix over the CTA of one count per thread, and the total: one
// barrier (the caller must not reuse sh.scan_buf before another barrier)
__device__ __forceinline__ int cta_exclusive_scan(CSh& sh, int c, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh.scan_buf[warp] = x;
  __syncthreads();
  int pre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarpsC; ++w) {
    const int t = sh.scan_buf[w];
    pre += w < warp ? t : 0;
    tot += t;
  }
  *total = tot;
  return pre + x - c;
}

// Large-band path only (degenerate inputs): sum the cluster's histograms
// (buffer `buf`) over cluster barriers and remote loads, and find the digit
// holding the need-th largest element.  Every CTA computes the same
// (bin, above).
template <int CS>
__device__ void cluster_find_bin(cg::cluster_group& cluster, CSh& sh, int buf, int need) {
  __syncthreads();
  cluster.sync();
  const int t = threadIdx.x;
  int local = 0;
  int bin = -1;
  if (t < kCBins) {
    bin = kCBins - 1 - t;   // thread 0 holds the largest digit
#pragma unroll
    for (int r = 0; r < CS; ++r) {
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

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory"); }

// large-band path: exchange one int per CTA over a cluster barrier; returns
// the total and the sum over lower ranks
template <int CS>
__device__ void cluster_exchange(cg::cluster_group& cluster, CSh& sh, int slot, int mine, int rank, int* total,
                                 int* below) {
  if (threadIdx.x == 0) sh.xchg[slot] = mine;
  __syncthreads();
  cluster.sync();
  int tot = 0, bel = 0;
#pragma unroll
  for (int r = 0; r < CS; ++r) {
    const int x = *cluster.map_shared_rank(&sh.xchg[slot], r);
    tot += x;
    bel += r < rank ? x : 0;
  }
  *total = tot;
  *below = bel;
}

// Everything after the pooled scores: exact Top-K over the cluster of the
// pooled values v[0, cnt) of this CTA (keys j0 + i), written ascending into
// out[0, K).  sh.m2 / sh.l hold the softmax statistics of the G heads and
// qf the fp32 query rows (for the fp64 band).  rx: kRxBytes(CS) of shared
// memory at the same offset in every CTA, receiving the radix histograms.
// Band scratch for degenerate (large) bands: this CTA's `per` entries at
// band_idx / band_val.  The exchanges must have been set up (exchange_init,
// cluster barrier) before the call.
template <int CS>
__device__ void cluster_topk(cg::cluster_group& cluster, CSh& sh, uint32_t* rx, const float* v, uint8_t* st, int cnt,
                             int j0, int rank, int K, int32_t* out, int32_t* band_idx, double* band_val,
                             const float* qf, const __nv_bfloat16* kb, int G, int D, int* err) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t xb = smem_u32(&sh.xbar[0]);
  // this CTA's histogram slots start at zero (the others only ever receive)
  for (int i = tid; i < kRadixPasses * kCBins; i += kCNT)
    rx[((i / kCBins) * CS + rank) * kCBins + (i % kCBins)] = 0u;
  __syncthreads();

  // radix select over the cluster on digits [31:24] [23:16] [15:8]: the K-th
  // largest fp32 value lies in the bin [prefix, prefix | 0xff], 2^-15
  // relative wide, which the band below covers.  Each pass: local histogram,
  // sent to the other CTAs in 16-byte pieces, summed over the CS slots.
  int need = K;
  unsigned prefix = 0;
#pragma unroll 1   // one copy of the pass: passes 2 and 3 run from the instruction cache pass 1 filled
  for (int pass = 0; pass < kRadixPasses; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* mine = rx + (pass * CS + rank) * kCBins;
    for (int i = tid; i < cnt; i += kCNT) {
      const unsigned x = __float_as_uint(v[i]);
      if (pass == 0 || (x >> (shift + 8)) == (prefix >> (shift + 8))) atomicAdd(&mine[(x >> shift) & 255u], 1u);
    }
    __syncthreads();
    for (int t = tid; t < (CS - 1) * (kCBins / 4); t += kCNT) {
      const int pr = peer_of(rank, 1 + t / (kCBins / 4), CS), ch = t % (kCBins / 4);
      const uint32_t src = smem_u32(mine) + 16u * ch;
      st_async_v4u(mapa(src, pr), reinterpret_cast<const uint4*>(mine)[ch], mapa(xb + 8u * pass, pr));
    }
    if (!mbar_wait_cluster_bounded(xb + 8u * pass, 0)) raise_error(err, kErrTimeout);
    int local = 0;
    if (tid < kCBins) {   // thread 0 holds the largest digit
#pragma unroll
      for (int r = 0; r < CS; ++r) local += (int)rx[(pass * CS + r) * kCBins + (kCBins - 1 - tid)];
    }
    find_digit(sh, local, need);
    prefix |= (unsigned)sh.bin << shift;
    need -= sh.above;
  }

  // band around the bin holding the K-th fp32 value: fewer than K values lie
  // above hi and at least K at or above lo
  const float tau_lo = __uint_as_float(prefix), tau_hi = __uint_as_float(prefix | 0xffu);
  const float lo = tau_lo < kBandFloor ? 0.0f : tau_lo * (1.0f - kBandDelta);
  const float hi = fmaxf(tau_hi * (1.0f + kBandDelta), kBandFloor);
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
  // one exchange of (count above the band, band size)
  if (tid < CS) {
    const unsigned long long pair = (unsigned long long)(unsigned)chi | ((unsigned long long)(unsigned)nb << 32);
    if (tid == 0) {
      sh.rx_cnt[rank] = make_int2(chi, nb);
    } else {
      const int pr = peer_of(rank, tid, CS);
      st_async_u64(mapa(smem_u32(&sh.rx_cnt[rank]), pr), pair, mapa(xb + 8u * kBarCnt, pr));
    }
  }
  __syncthreads();
  if (!mbar_wait_cluster_bounded(xb + 8u * kBarCnt, 0)) raise_error(err, kErrTimeout);
  int chi_total = 0, chi_below = 0, nb_total = 0, nb_below = 0;
#pragma unroll
  for (int r = 0; r < CS; ++r) {
    const int2 xy = sh.rx_cnt[r];
    chi_total += xy.x;
    nb_total += xy.y;
    chi_below += r < rank ? xy.x : 0;
    nb_below += r < rank ? xy.y : 0;
  }
  const int need_band = K - chi_total;
  // small bands (the usual case) are sent whole to every CTA: entry i of CTA
  // r lands at position (entries of lower ranks) + i
  const bool small = nb_total <= kSmallBand;
  if (small && tid == 0) mbar_arrive_expect_tx(xb + 8u * kBarBand, (uint32_t)(nb_total - nb) * 12u);

  // fp64 pooled scores of this CTA's band members, one warp per member
  const double c2 = 1.4426950408889634 / sqrt((double)D);
  for (int i = warp; i < nb; i += kWarpsC) {
    const int j = band_idx[i];
    // lane holds dims [4 lane, 4 lane + 4) (d = 128) or [2 lane, 2 lane + 2)
    // (d = 64).  The head loop stays rolled: this runs once per launch,
    // mostly from a cold instruction cache, where code size is the cost.
    float kv[4] = {0.f, 0.f, 0.f, 0.f};
    const int dl = D / 32;
    if (dl == 4) {
      const uint2 r = *reinterpret_cast<const uint2*>(kb + (size_t)j * D + 4 * lane);
      kv[0] = bf16_lo(r.x), kv[1] = bf16_hi(r.x), kv[2] = bf16_lo(r.y), kv[3] = bf16_hi(r.y);
    } else {
      const uint32_t r = *reinterpret_cast<const uint32_t*>(kb + (size_t)j * D + 2 * lane);
      kv[0] = bf16_lo(r), kv[1] = bf16_hi(r);
    }
    double total = 0.0;
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
      double dot = 0.0;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (t < dl) dot += (double)qf[g * D + dl * lane + t] * (double)kv[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      total += exp2(dot * c2 - (double)sh.m2[g]) / sh.l[g];
    }
    const double val = total / (double)G;   // every lane holds it
    if (!small) {
      if (lane == 0) band_val[i] = val;
    } else if (lane == 0) {
      sh.b_idx[nb_below + i] = j;
      sh.b_val[nb_below + i] = val;
    } else if (lane < CS) {
      const int pr = peer_of(rank, lane, CS);
      const uint32_t bar = mapa(xb + 8u * kBarBand, pr);
      st_async_u32(mapa(smem_u32(&sh.b_idx[nb_below + i]), pr), (uint32_t)j, bar);
      st_async_u64(mapa(smem_u32(&sh.b_val[nb_below + i]), pr), (unsigned long long)__double_as_longlong(val), bar);
    }
  }
  __syncthreads();

  int tie_quota = 0, sel_below = 0;
  auto flag_of = [&](int i) -> int {
    const float x = v[i];
    return x > hi || (x >= lo && st[i] == 1);
  };
  if (small) {
    // every CTA holds the whole band (ordered by CTA rank) and ranks the
    // members of the lower CTAs and its own: its own are marked, the lower
    // ones give this CTA's output offset
    // every byte another CTA sends here has now arrived, and no CTA reads
    // another's shared memory on this path: no closing cluster barrier
    if (!mbar_wait_cluster_bounded(xb + 8u * kBarBand, 0)) raise_error(err, kErrTimeout);
    int low_sel = 0;
    for (int t = tid; t < nb_below + nb; t += kCNT) {
      const double mv = sh.b_val[t];
      const int mj = sh.b_idx[t];
      int rk = 0;
      for (int u = 0; u < nb_total; ++u) {
        const double ov = sh.b_val[u];
        rk += (ov > mv) || (ov == mv && sh.b_idx[u] < mj);
      }
      if (t < nb_below) low_sel += rk < need_band;
      else st[mj - j0] = rk < need_band ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) low_sel += __shfl_xor_sync(0xffffffffu, low_sel, o);
    if (tid == 0) sh.chi = 0;
    __syncthreads();
    if (lane == 0 && low_sel) atomicAdd(&sh.chi, low_sel);
    __syncthreads();
    sel_below = chi_below + sh.chi;
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
      cluster_find_bin<CS>(cluster, sh, buf, nd);
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
    cluster_exchange<CS>(cluster, sh, 2, sh.nb, rank, &ties_total, &ties_below);
    tie_quota = min(max(nd - ties_below, 0), sh.nb);   // lower ranks hold lower indices
    __syncthreads();
    int mine = 0;
    for (int i = tid; i < cnt; i += kCNT) mine += flag_of(i);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
    if (tid == 0) sh.chi = 0;
    __syncthreads();
    if (lane == 0 && mine) atomicAdd(&sh.chi, mine);
    __syncthreads();
    int sel_total;
    cluster_exchange<CS>(cluster, sh, 3, sh.chi + tie_quota, rank, &sel_total, &sel_below);
    cluster_arrive();   // the last reads of other CTAs' shared memory
  }
  __syncthreads();

  // write ascending at this CTA's offset
  if (tie_quota == 0) {
    // one scan: thread t owns the consecutive keys [t * kpt, (t + 1) * kpt)
    const int kpt = (cnt + kCNT - 1) / kCNT;
    const int b0 = min(cnt, tid * kpt), b1 = min(cnt, b0 + kpt);
    int c = 0;
    for (int i = b0; i < b1; ++i) c += flag_of(i);
    int unused;
    int w = sel_below + cta_exclusive_scan(sh, c, &unused);
    for (int i = b0; i < b1; ++i)
      if (flag_of(i)) out[w++] = j0 + i;
  } else {
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
      int tt;
      const int tincl = block_inclusive_scan<kCNT>(tie, sh.scan_buf, &tt);
      if (tie && ties_taken + tincl - 1 < tie_quota) flag = 1;
      ties_taken += tt;
      int total;
      const int incl = block_inclusive_scan<kCNT>(flag, sh.scan_buf, &total);
      if (flag) out[written + incl - 1] = j0 + i;
      written += total;
    }
  }
  // large bands: no CTA may leave while another can still read its shared memory
  if (!small) cluster_wait();
}

// ---------------------------------------------------------------- fallback

__host__ __device__ constexpr size_t cluster_dyn_bytes(int keys_per_cta) {
  // q rows fp32 [8][128], radix receive slots, v[keys] fp32, state[keys] bytes
  return kCHead + 8 * 128 * 4 + kRxBytes(kFallbackCS) + (size_t)keys_per_cta * 4 + (size_t)keys_per_cta;
}

__global__ void __cluster_dims__(kFallbackCS, 1, 1) __launch_bounds__(kCNT)
    select_decode_cluster_kernel(const SelArgs a, int keys_per_cta) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) char smem_raw[];
  CSh& sh = *reinterpret_cast<CSh*>(smem_raw);
  float* qf = reinterpret_cast<float*>(smem_raw + kCHead);
  uint32_t* rx = reinterpret_cast<uint32_t*>(qf + 8 * 128);
  float* v = reinterpret_cast<float*>(smem_raw + kCHead + 8 * 128 * 4 + kRxBytes(kFallbackCS));
  uint8_t* st = reinterpret_cast<uint8_t*>(v + keys_per_cta);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int b = bh / a.Hp, h = bh - b * a.Hp;   // problem h of batch row b
  const int G = a.G, D = a.D, N = a.N;
  const int K = topk_count(N, a.num, a.den);
  const int j0 = rank * keys_per_cta;
  const int j1 = min(N, j0 + keys_per_cta);
  const int cnt = max(0, j1 - j0);
  int32_t* out = a.idx + (size_t)bh * K;
  const size_t bbase = (size_t)bh * kFallbackCS * keys_per_cta;

  if (K >= N) {   // everything is selected (same branch in every CTA)
    for (int i = tid; i < cnt; i += kCNT) out[j0 + i] = j0 + i;
    return;
  }
  if (tid == 0) exchange_init<kFallbackCS>(sh, 0);
  __syncthreads();
  cluster_arrive();

  // softmax statistics of the G query heads from the scoring kernel's splits
  for (int g = warp; g < G; g += kWarpsC) {
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
  __syncthreads();

  // pooled fp32 scores of this CTA's keys
  const float* srow = a.s2 + (size_t)(b * a.Hq + h * G) * N;
  const float invG = 1.0f / (float)G;
  for (int i = tid; i < cnt; i += kCNT) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) acc += exp2f(srow[(size_t)g * N + j0 + i] - sh.m2[g]) * sh.inv_l[g];
    v[i] = acc * invG;
  }
  __syncthreads();
  cluster_wait();   // every CTA's exchange barriers are initialised
  cluster_topk<kFallbackCS>(cluster, sh, rx, v, st, cnt, j0, rank, K, out,
                            a.band_idx + bbase + (size_t)rank * keys_per_cta,
                            a.band_val + bbase + (size_t)rank * keys_per_cta, qf,
                            a.k + (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv) * N * D, G, D,
                            a.err);
}

// ------------------------------------------------------------ fused select

template <int D>
struct ASL {
  static constexpr size_t qf = kCHead;                               // [8][128] f32
  static constexpr size_t ring = qf + 8 * 128 * 4;                    // [kSlots][kRoundKeys][D] bf16
  static constexpr size_t RB = (size_t)kRoundKeys * D * 2;
  static constexpr size_t sc = ring + kSlots * RB;                         // [G][per + 4] f32 scores
  static size_t bytes(int G, int per) { return sc + (size_t)G * (per + 4) * 4 + (size_t)per + 16; }
  static_assert(ring % 128 == 0, "bulk copy destination alignment");
  static_assert(kSlots * RB >= kRxBytes(kMaxCS), "the ring doubles as the radix receive buffer");
};

template <int CS, int D>
__global__ void __launch_bounds__(kCNT, 1) anchor_select_kernel(const SelArgs a, int per) {
  using L = ASL<D>;
  constexpr int KS = D / 32;
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) char smem_raw[];
  CSh& sh = *reinterpret_cast<CSh*>(smem_raw);
  float* qf = reinterpret_cast<float*>(smem_raw + L::qf);
  const uint32_t ring = smem_u32(smem_raw) + (uint32_t)L::ring;
  float* sc = reinterpret_cast<float*>(smem_raw + L::sc);
  const int SCS = per + 4;   // score row stride (floats)

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int bh = blockIdx.y;
  const int b = bh / a.Hp, h = bh - b * a.Hp;   // problem h of batch row b
  const int G = a.G, N = a.N;
  const int K = topk_count(N, a.num, a.den);
  const int j0 = rank * per;
  const int j1 = min(N, j0 + per);
  const int cnt = max(0, j1 - j0);
  uint8_t* st = reinterpret_cast<uint8_t*>(sc + (size_t)G * SCS);
  int32_t* out = a.idx + (size_t)bh * K;
  const size_t bbase = (size_t)bh * CS * per;
  const __nv_bfloat16* kb = a.k + (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv) * N * D;

  if (K >= N) {   // everything is selected (same branch in every CTA)
    for (int i = tid; i < cnt; i += kCNT) out[j0 + i] = j0 + i;
    return;
  }

  // ---- stream this CTA's K rows in rounds of kRoundKeys (kSlots in flight)
  const uint32_t full0 = smem_u32(&sh.full[0]);
  const int nr = (cnt + kRoundKeys - 1) / kRoundKeys;
  if (tid == 0) {
    for (int sl = 0; sl < kSlots; ++sl) mbar_init(full0 + 8u * sl, 1);
    exchange_init<CS>(sh, G * 12);   // stats: one f32 max and one f64 sum per head
  }
  __syncthreads();
  cluster_arrive();   // matched before the first exchange, long after every CTA got here
  auto issue = [&](int r) {   // thread 0 only
    const int k0 = r * kRoundKeys, nk = min(kRoundKeys, cnt - k0);
    const uint32_t bytes = (uint32_t)nk * D * 2;
    const uint32_t bar = full0 + 8u * (uint32_t)(r % kSlots);
    const uint32_t dst = ring + (uint32_t)((r % kSlots) * L::RB);
    const char* src = reinterpret_cast<const char*>(kb + (size_t)(j0 + k0) * D);
    mbar_arrive_expect_tx(bar, bytes);
    for (uint32_t off = 0; off < bytes; off += 16384u) bulk_g2s(dst + off, src + off, min(16384u, bytes - off), bar);
  };
  if (tid == 0)
    for (int r = 0; r < kSlots && r < nr; ++r) issue(r);
  // query rows: fp32 copy for the fp64 band, MMA B fragments in registers
  // (lane (g, c) holds dims [32 s + 8 c, +8) of head g; heads >= G zero)
  for (int e = tid; e < G * D; e += kCNT) {
    const int gg = e / D, dd = e - gg * D;
    qf[e] = __bfloat162float(a.q[(size_t)(b * a.Hq + h * G + gg) * D + dd]);
  }
  uint4 qb[KS];
#pragma unroll
  for (int s = 0; s < KS; ++s)
    qb[s] = g < G ? *reinterpret_cast<const uint4*>(a.q + (size_t)(b * a.Hq + h * G + g) * D + 32 * s + 8 * c)
                  : make_uint4(0, 0, 0, 0);
  const float scale2 = kLog2e * rsqrtf((float)D);
  float mx0 = -INFINITY, mx1 = -INFINITY;   // heads 2c, 2c+1
  for (int r = 0; r < nr; ++r) {
    if (!mbar_wait_bounded(full0 + 8u * (uint32_t)(r % kSlots), (uint32_t)((r / kSlots) & 1)))
      raise_error(a.err, kErrTimeout);
    const int k0 = r * kRoundKeys, nk = min(kRoundKeys, cnt - k0);
    const uint32_t slot = ring + (uint32_t)((r % kSlots) * L::RB);
    const bool have = 16 * warp < nk;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (have) {
      const uint32_t row0 = slot + (uint32_t)((16 * warp + g) * D * 2 + 16 * c);
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        uint4 ka, kc;
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(ka.x), "=r"(ka.y), "=r"(ka.z), "=r"(ka.w)
                     : "r"(row0 + 64 * s));
        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(kc.x), "=r"(kc.y), "=r"(kc.z), "=r"(kc.w)
                     : "r"(row0 + 8 * D * 2 + 64 * s));
        const uint32_t a0[4] = {ka.x, kc.x, ka.y, kc.y};
        const uint32_t a1[4] = {ka.z, kc.z, ka.w, kc.w};
        mma_bf16_16816(acc, a0, qb[s].x, qb[s].y);
        mma_bf16_16816(acc, a1, qb[s].z, qb[s].w);
      }
    }
    __syncthreads();
    if (tid == 0 && r + kSlots < nr) {
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      issue(r + kSlots);
    }
    if (have) {
      const int i0 = k0 + 16 * warp + g, i1 = i0 + 8;   // local key indices
      if (i0 < cnt) {
        const float s0 = acc[0] * scale2, s1 = acc[1] * scale2;
        if (2 * c < G) sc[(2 * c) * SCS + i0] = s0;
        if (2 * c + 1 < G) sc[(2 * c + 1) * SCS + i0] = s1;
        mx0 = fmaxf(mx0, s0);
        mx1 = fmaxf(mx1, s1);
      }
      if (i1 < cnt) {
        const float s0 = acc[2] * scale2, s1 = acc[3] * scale2;
        if (2 * c < G) sc[(2 * c) * SCS + i1] = s0;
        if (2 * c + 1 < G) sc[(2 * c + 1) * SCS + i1] = s1;
        mx0 = fmaxf(mx0, s0);
        mx1 = fmaxf(mx1, s1);
      }
    }
  }
  __syncthreads();

  // ---- softmax statistics of every head over the cluster: each CTA
  // publishes its own (max, sum of exp2(s - max)); one exchange, partial sums
  // rescaled to the cluster max in fp64
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  if (g == 0) {
    sh.wmax[warp][2 * c] = mx0;
    sh.wmax[warp][2 * c + 1] = mx1;
  }
  __syncthreads();
  if (tid < G) {   // this CTA's max of each head, in its own exchange slot
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarpsC; ++w) m = fmaxf(m, sh.wmax[w][tid]);
    sh.rx_cmax[rank][tid] = m;
  }
  __syncthreads();
  // exp2(s - max) in place, four keys per thread per step (rows are 16-byte
  // aligned: SCS is a multiple of 4); lanes past cnt exponentiate slack
  // entries of the row and leave them out of the sums.  The head loop stays
  // rolled: this code runs once per launch from a cold instruction cache.
  const int n4 = (cnt + 3) >> 2;
#pragma unroll 1
  for (int hh = 0; hh < G; ++hh) {
    const float cmh = sh.rx_cmax[rank][hh];
    float ps = 0.f;
    for (int j = tid; j < n4; j += kCNT) {
      const int rem = cnt - 4 * j;
      float4* p = reinterpret_cast<float4*>(sc + hh * SCS + 4 * j);
      float4 x = *p;
      x.x = ex2_fast(x.x - cmh);   // kept for the pooled scores
      x.y = ex2_fast(x.y - cmh);
      x.z = ex2_fast(x.z - cmh);
      x.w = ex2_fast(x.w - cmh);
      *p = x;
      ps += rem > 3 ? (x.x + x.y) + (x.z + x.w) : (x.x + (rem > 1 ? x.y : 0.f)) + (rem > 2 ? x.z : 0.f);
    }
    double d = ps;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) sh.wsum[warp][hh] = d;
  }
  __syncthreads();
  if (tid < G) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kWarpsC; ++w) s += sh.wsum[w][tid];
    sh.rx_csum[rank][tid] = s;
  }
  __syncthreads();
  cluster_wait();   // every CTA's exchange barriers are initialised
  const uint32_t stats_bar = smem_u32(&sh.xbar[kBarStats]);
  if (tid < (CS - 1) * G) {
    const int hh = tid % G, pr = peer_of(rank, 1 + tid / G, CS);
    const uint32_t bar = mapa(stats_bar, pr);
    st_async_u32(mapa(smem_u32(&sh.rx_cmax[rank][hh]), pr), __float_as_uint(sh.rx_cmax[rank][hh]), bar);
    st_async_u64(mapa(smem_u32(&sh.rx_csum[rank][hh]), pr),
                 (unsigned long long)__double_as_longlong(sh.rx_csum[rank][hh]), bar);
  }
  if (!mbar_wait_cluster_bounded(stats_bar, 0)) raise_error(a.err, kErrTimeout);
  // warp hh (< G): lane r < CS takes CTA r's (max, sum) of head hh
  if (warp < G) {
    const float mr = lane < CS ? sh.rx_cmax[lane][warp] : -INFINITY;
    const double sr = lane < CS ? sh.rx_csum[lane][warp] : 0.0;
    float m = mr;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const double e = mr != -INFINITY ? exp2((double)mr - (double)m) : 0.0;   // CTA r's terms rescaled
    const double e_own = __shfl_sync(0xffffffffu, e, rank);
    double l = sr * e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      const double inv = 1.0 / l;
      sh.m2[warp] = m;
      sh.l[warp] = l;
      sh.inv_l[warp] = (float)inv;
      sh.wpool[warp] = (float)(e_own * inv);   // pooled weight of this CTA's stored terms exp2(s - cm)
    }
  }
  __syncthreads();

  // ---- pooled scores, in place of head 0's scores
  float* v = sc;
  const float invG = 1.0f / (float)G;
  for (int j = tid; j < n4; j += kCNT) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int hh = 0; hh < G; ++hh) {
      const float wh = sh.wpool[hh];
      const float4 x = *reinterpret_cast<const float4*>(sc + hh * SCS + 4 * j);
      acc.x += x.x * wh;
      acc.y += x.y * wh;
      acc.z += x.z * wh;
      acc.w += x.w * wh;
    }
    *reinterpret_cast<float4*>(v + 4 * j) =
        make_float4(acc.x * invG, acc.y * invG, acc.z * invG, acc.w * invG);
  }
  __syncthreads();
  // the ring is free: it receives the radix histograms
  cluster_topk<CS>(cluster, sh, reinterpret_cast<uint32_t*>(smem_raw + L::ring), v, st, cnt, j0, rank, K, out,
                   a.band_idx + bbase + (size_t)rank * per, a.band_val + bbase + (size_t)rank * per, qf, kb, G, D,
                   a.err);
}

int fused_per(int N, int cs) {
  const int per = (N + cs - 1) / cs;
  return (per + 63) / 64 * 64;
}

// How many clusters of `cs` CTAs of the fused kernel (one CTA per SM at
// these shared-memory sizes) the current device runs at once; 0 if none.
template <int CS, int D>
int fused_active_clusters(size_t smem) {
  if (cudaFuncSetAttribute(anchor_select_kernel<CS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return 0;
  if (CS > 8 &&
      cudaFuncSetAttribute(anchor_select_kernel<CS, D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(CS, 1, 1);
  cfg.blockDim = dim3(kCNT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, anchor_select_kernel<CS, D>, &cfg) != cudaSuccess) n = 0;
  return n;
}

// Cluster sizes the fused kernel is built for.  A cluster must sit inside
// one GPC, so how many clusters of each size run at once depends on the
// device's GPC layout rather than on the SM count alone (on a 148-SM B200:
// 15 of 8 or 9 CTAs, 11 of 10, 7 of 11 to 16).
constexpr int kFusedSizes[] = {16, 12, 10, 9, 8};
constexpr int kNumFusedSizes = 5;

// Cluster size of the fused kernel for this shape on the current device
// (fewest waves, then the most CTAs); 0 when the scores do not fit on chip
// or the problems take more than one wave (choose_fused_select_size).
template <int D>
int fused_cluster_size(const SelArgs& a) {
  static int cached[64][kNumFusedSizes] = {{0}};   // max active clusters (+1; 0 = unknown)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const size_t max_smem = 227 * 1024;
  if (!cached[dev][0]) {
    cached[dev][0] = 1 + fused_active_clusters<16, D>(max_smem);
    cached[dev][1] = 1 + fused_active_clusters<12, D>(max_smem);
    cached[dev][2] = 1 + fused_active_clusters<10, D>(max_smem);
    cached[dev][3] = 1 + fused_active_clusters<9, D>(max_smem);
    cached[dev][4] = 1 + fused_active_clusters<8, D>(max_smem);
    cudaGetLastError();
  }
  int active[kNumFusedSizes];
  bool fits[kNumFusedSizes];
  for (int i = 0; i < kNumFusedSizes; ++i) {
    active[i] = cached[dev][i] - 1;
    fits[i] = ASL<D>::bytes(a.G, fused_per(a.N, kFusedSizes[i])) <= max_smem;
  }
  return choose_fused_select_size((long long)a.B * a.Hp, kFusedSizes, active, fits, kNumFusedSizes);
}

template <int CS, int D>
cudaError_t launch_fused(const SelArgs& a, cudaStream_t stream) {
  const int per = fused_per(a.N, CS);
  const size_t smem = ASL<D>::bytes(a.G, per);
  const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(anchor_select_kernel<CS, D>), smem, CS > 8);
  if (e != cudaSuccess) return e;
  return launch_ex(anchor_select_kernel<CS, D>, dim3(CS, a.B * a.Hp), dim3(kCNT), smem, stream,
                   (a.flags & 1) != 0, CS, a, per);
}

}  // namespace

int select_decode_cluster_keys(int N) { return (N + kFallbackCS - 1) / kFallbackCS; }

bool select_decode_cluster_ok(int N) { return select_decode_cluster_keys(N) <= 16384; }

size_t select_decode_cluster_scratch(int B, int problems, int N) {
  // band entries for the fallback layout and both fused cluster sizes
  const size_t fb = (size_t)kFallbackCS * select_decode_cluster_keys(N);
  size_t m = fb;
  for (int i = 0; i < kNumFusedSizes; ++i) {
    const size_t f = (size_t)kFusedSizes[i] * fused_per(N, kFusedSizes[i]);
    m = f > m ? f : m;
  }
  return (size_t)B * problems * m;
}

cudaError_t launch_select_decode_cluster(const SelArgs& a, cudaStream_t stream) {
  const int per = select_decode_cluster_keys(a.N);
  const size_t smem = cluster_dyn_bytes(per);
  const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(select_decode_cluster_kernel), smem, false);
  if (e != cudaSuccess) return e;
  dim3 grid(kFallbackCS, a.B * a.Hp);
  return launch_ex(select_decode_cluster_kernel, grid, dim3(kCNT), smem, stream, (a.flags & 1) != 0, 1, a, per);
}

bool anchor_select_fused_ok(const SelArgs& a) {
  if (a.G > 8 || !(a.D == 64 || a.D == 128)) return false;
  return (a.D == 128 ? fused_cluster_size<128>(a) : fused_cluster_size<64>(a)) > 0;
}

cudaError_t launch_anchor_select_fused(const SelArgs& a, cudaStream_t stream) {
  if (a.D == 128) {
    switch (fused_cluster_size<128>(a)) {
      case 16: return launch_fused<16, 128>(a, stream);
      case 12: return launch_fused<12, 128>(a, stream);
      case 10: return launch_fused<10, 128>(a, stream);
      case 9: return launch_fused<9, 128>(a, stream);
      case 8: return launch_fused<8, 128>(a, stream);
      default: break;
    }
  } else {
    switch (fused_cluster_size<64>(a)) {
      case 16: return launch_fused<16, 64>(a, stream);
      case 12: return launch_fused<12, 64>(a, stream);
      case 10: return launch_fused<10, 64>(a, stream);
      case 9: return launch_fused<9, 64>(a, stream);
      case 8: return launch_fused<8, 64>(a, stream);
      default: break;
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace kascade
