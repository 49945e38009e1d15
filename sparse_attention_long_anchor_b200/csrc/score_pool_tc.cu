// Anchor prefill scoring and pooling on the 5th-generation tensor cores
// (Kascade README, Abstract and the post_softmax_pooled_prefill_topk
// strategy).  Same results as the warp-MMA version in score_pool.cu:
//   pass 1: S = Q K^T / sqrt(d), causal mask j <= i, per row the max m2_r and
//           l_r = sum_j exp2(s2_rj - m2_r) (base 2, fp32 terms, fp64 sum);
//   pass 2: S^T = K Q^T, so that every TMEM lane is one key and its columns
//           are the 32 G query rows of the tile; the pooled score
//           P_j = sum_r exp2(s2_rj - m2_r - log2 l_r) / (G rows_t) is a sum
//           along the lane.
// Exact post-softmax pooling needs each row's normaliser before any column
// sum, so K is read twice (the second time mostly from L2).
//
// Work item = (batch, kv head, query tile) with 128 rows = 4 heads x 32
// queries (G <= 4; rows of absent heads stay zero).  Persistent CTAs take
// items longest tile first.  Per CTA:
//   warp 0      TMA producer: the Q tile (32-row boxes, one per head) and a
//               ring of kStages K blocks of 128 keys, 128-byte swizzled;
//   warp 1      single-thread tcgen05.mma issue (M = N = 128, K = 16 steps);
//               owns TMEM;
//   warps 2..17 epilogue: four warpgroups take the K blocks in turn (four
//               128-column TMEM accumulators); tcgen05.ld of one TMEM lane
//               quarter per warp, online row statistics (pass 1, merged
//               across the groups per tile), masked column sums (pass 2).
// All hand-offs are mbarriers; every wait is bounded and a timeout stops the
// CTA's loops and records an error code.
#include "../../include/kascade.h"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace kascade {

namespace {

constexpr int kStages = 4;
constexpr int kKB = 128;          // keys per block
constexpr int kEpiGroups = 4;     // epilogue warpgroups, taking K blocks in turn
constexpr int kBufs = 4;          // TMEM accumulators of 128 columns
constexpr int kThreads = 64 + 128 * kEpiGroups;
constexpr int kErrTimeout = 2;

template <int D>
struct SPL {
  static constexpr int CB = D / 64;                 // 64-element (128-byte) column blocks
  static constexpr int QTILE = 128 * D * 2;
  static constexpr int KTILE = kKB * D * 2;
  static constexpr int CBYTES = 128 * 128;          // one column block of 128 rows
  static constexpr size_t q = 0;
  static constexpr size_t k = q + QTILE;
  static constexpr size_t bars = k + (size_t)kStages * KTILE;
  // q_full, q_empty, k_full[S], k_empty[S], acc_full[B], acc_empty[B], drain
  static constexpr int NBARS = 2 + 2 * kStages + 2 * kBufs + 1;
  static constexpr size_t tslot = bars + NBARS * 8;
  static constexpr size_t stop = (tslot + 8 + 15) / 16 * 16;
  static constexpr size_t bcol = stop + 16;         // [128] f32, read as float4
  static constexpr size_t rpos = bcol + 128 * 4;    // [128] int, read as int4
  static constexpr size_t pstat = rpos + 128 * 4;   // [groups][128] (m f32, l f64) row partials
  static constexpr size_t total = pstat + kEpiGroups * 128 * 16;
  static_assert(bcol % 16 == 0 && rpos % 16 == 0, "vector reads of bcol / rpos need 16-byte alignment");
  static_assert(bars % 8 == 0 && k % 1024 == 0, "mbarriers and swizzled tiles alignment");
  static constexpr size_t alloc = total + 1024;     // slack for 1024-byte alignment
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;\n" ::"n"(128 * kEpiGroups) : "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    score_pool_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                         const ScorePoolArgs a, int* err) {
  using L = SPL<D>;
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  char* sm = smem_raw + (base - raw);
  const uint32_t q_s = base + (uint32_t)L::q, k_s = base + (uint32_t)L::k;
  const uint32_t bar0 = base + (uint32_t)L::bars;
  const uint32_t q_full = bar0, q_empty = bar0 + 8;
  const uint32_t k_full0 = bar0 + 16, k_empty0 = k_full0 + 8 * kStages;
  const uint32_t acc_full0 = k_empty0 + 8 * kStages, acc_empty0 = acc_full0 + 8 * kBufs;
  const uint32_t drain = acc_empty0 + 8 * kBufs;
  volatile int* stop = reinterpret_cast<volatile int*>(sm + L::stop);
  float* bcol = reinterpret_cast<float*>(sm + L::bcol);
  int* rpos = reinterpret_cast<int*>(sm + L::rpos);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.G;
  const int T = (a.N + a.tile - 1) / a.tile;
  const int t0 = a.q0 / a.tile;   // first query tile of the call (rolling chunks)
  const int BH = a.B * a.Hkv;
  const int items = (T - t0) * BH;
  const uint32_t idesc = tc::idesc_bf16_f32(128, 128);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full0 + 8 * s, 1);
      mbar_init(k_empty0 + 8 * s, 1);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(acc_full0 + 8 * b, 1);
      mbar_init(acc_empty0 + 8 * b, 4);   // one arrival per warp of the consuming warpgroup
    }
    mbar_init(drain, 1);
    *stop = 0;
    mbar_fence_init();
  }
  // rows of absent heads (G < 4) stay zero for the whole kernel
  for (int i = threadIdx.x; i < L::CB * (4 - G) * 32 * 8; i += kThreads) {
    const int cb = i / ((4 - G) * 32 * 8), rem = i - cb * (4 - G) * 32 * 8;
    const int r = 32 * G + rem / 8, ch = rem % 8;
    *reinterpret_cast<uint4*>(sm + L::q + cb * L::CBYTES + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
  }
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  if (warp == 1) tc::tmem_alloc(base + (uint32_t)L::tslot, 128 * kBufs);
  pdl_wait();
  pdl_launch_dependents();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::tslot);

  auto fail = [&]() {
    *stop = 1;
    raise_error(err, kErrTimeout);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_map(&mq);
      tc::prefetch_map(&mk);
      int kcount = 0, qcount = 0;
      for (int it = blockIdx.x; it < items && !*stop; it += gridDim.x) {
        const int t = T - 1 - it / BH, bh = it % BH;
        const int b = bh / a.Hkv, h = bh - b * a.Hkv;
        const int i0 = t * a.tile;
        const int e_t = min(i0 + a.tile, a.N);
        const int nb = (e_t + kKB - 1) / kKB;
        if (qcount > 0 && !mbar_wait_bounded(q_empty, (qcount - 1) & 1)) { fail(); break; }
        mbar_arrive_expect_tx(q_full, (uint32_t)(L::CB * G * 32 * 128));
        // test switch: announce the first query tile but never load it, so
        // the waits on it give up and report through the error word
        if (!(qcount == 0 && (a.flags & KASCADE_FLAG_TEST_DROP_LOAD)))
          for (int cb = 0; cb < L::CB; ++cb)
            for (int g = 0; g < G; ++g)
              tc::tma_load_3d(q_s + cb * L::CBYTES + g * 4096, &mq, cb * 64, i0 - a.q0, b * a.Hq + h * G + g, q_full);
        ++qcount;
        for (int pass = 0; pass < 2; ++pass) {
          for (int blk = 0; blk < nb; ++blk) {
            const int s = kcount % kStages, use = kcount / kStages;
            if (use > 0 && !mbar_wait_bounded(k_empty0 + 8 * s, (use - 1) & 1)) { fail(); break; }
            mbar_arrive_expect_tx(k_full0 + 8 * s, (uint32_t)L::KTILE);
            for (int cb = 0; cb < L::CB; ++cb)
              tc::tma_load_3d(k_s + s * L::KTILE + cb * L::CBYTES, &mk, cb * 64, blk * kKB, bh, k_full0 + 8 * s);
            ++kcount;
          }
          if (*stop) break;
        }
      }
      // leave no copy in flight: the last fill of every stage has landed
      for (int s = 0; s < kStages && s < kcount; ++s) {
        const int last = (kcount - 1 - s) / kStages;
        if (!mbar_wait_bounded(k_full0 + 8 * s, last & 1)) raise_error(err, kErrTimeout);
      }
      if (qcount > 0 && !mbar_wait_bounded(q_full, (qcount - 1) & 1)) raise_error(err, kErrTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int kcount = 0, qcount = 0, acount = 0;
      for (int it = blockIdx.x; it < items && !*stop; it += gridDim.x) {
        const int t = T - 1 - it / BH;
        const int e_t = min(t * a.tile + a.tile, a.N);
        const int nb = (e_t + kKB - 1) / kKB;
        if (!mbar_wait_bounded(q_full, qcount & 1)) { fail(); break; }
        tc::fence_after();
        for (int pass = 0; pass < 2 && !*stop; ++pass) {
          for (int blk = 0; blk < nb; ++blk) {
            const int s = kcount % kStages, buf = acount % kBufs, ause = acount / kBufs;
            if (!mbar_wait_bounded(k_full0 + 8 * s, (kcount / kStages) & 1)) { fail(); break; }
            if (ause > 0 && !mbar_wait_bounded(acc_empty0 + 8 * buf, (ause - 1) & 1)) { fail(); break; }
            tc::fence_after();
            const uint32_t d = tmem + (uint32_t)(buf * 128);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (uint32_t)((kk >> 2) * L::CBYTES + (kk & 3) * 32);
              const uint64_t qd = tc::smem_desc_sw128(q_s + off);
              const uint64_t kd = tc::smem_desc_sw128(k_s + s * L::KTILE + off);
              if (pass == 0)
                tc::mma_bf16(d, qd, kd, idesc, kk > 0);
              else
                tc::mma_bf16(d, kd, qd, idesc, kk > 0);
            }
            tc::commit(k_empty0 + 8 * s);
            tc::commit(acc_full0 + 8 * buf);
            ++kcount;
            ++acount;
          }
        }
        tc::commit(q_empty);
        ++qcount;
      }
      // all issued MMAs complete before TMEM can be released
      tc::commit(drain);
      if (!mbar_wait_bounded(drain, 0)) raise_error(err, kErrTimeout);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warpgroup wg takes the K blocks with block sequence number = wg (mod kEpiGroups);
    // warp w reads TMEM lanes 32 (w % 4) .. +31
    const int ew = warp - 2;
    const int wg = ew >> 2;
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;       // pass 1: query row; pass 2: key within the block
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    const float scale2 = kLog2e * rsqrtf((float)D);
    float* pm = reinterpret_cast<float*>(sm + L::pstat);                   // [groups][128]
    double* pl = reinterpret_cast<double*>(sm + L::pstat + kEpiGroups * 128 * 4);
    int acount = 0;
    // the epilogue warps meet at named barriers, so their loops stay
    // uniform: after a failure the waits are skipped, never the structure
    auto wait_acc = [&](int buf, int par) -> bool {
      if (*stop) return false;
      if (mbar_wait_bounded(acc_full0 + 8 * buf, par)) return true;
      fail();
      return false;
    };
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      const int t = T - 1 - it / BH, bh = it % BH;
      const int b = bh / a.Hkv, h = bh - b * a.Hkv;
      const int i0 = t * a.tile;
      const int e_t = min(i0 + a.tile, a.N);
      const int rows_t = e_t - i0;
      const int nb = (e_t + kKB - 1) / kKB;
      const bool valid = quarter < G && lane < rows_t;
      const int pos = i0 + lane;
      // ---- pass 1: statistics of row r over this warpgroup's blocks.  The
      // running shift m2 is the fp32 value that gets stored, and every term is
      // exp2(fma(dot, scale2, -m2)) with a single rounding, so that the stored
      // (m2, l) pair is consistent term by term
      float m2 = -INFINITY;  // running max of dot * scale2 (fp32)
      double l = 0.0;        // sum of exp2(dot * scale2 - m2)
      for (int blk = 0; blk < nb; ++blk, ++acount) {
        if (acount % kEpiGroups != wg) continue;
        const int buf = acount % kBufs;
        wait_acc(buf, (acount / kBufs) & 1);
        tc::fence_after();
        const int j0 = blk * kKB;
        const bool diag = j0 + kKB - 1 > i0;   // block reaches the tile: mask j > pos
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          float v[32];
          tc::tmem_ld32(tmem + lane_addr + (uint32_t)(buf * 128 + ch * 32), v);
          if (!valid) continue;
          if (diag) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (j0 + ch * 32 + i > pos) v[i] = -INFINITY;
          }
          float cm = v[0];
#pragma unroll
          for (int i = 1; i < 32; ++i) cm = fmaxf(cm, v[i]);
          const float cm2 = cm * scale2;   // scale > 0 keeps the order
          if (cm2 > m2) {
            if (m2 != -INFINITY) l *= exp2((double)m2 - (double)cm2);
            m2 = cm2;
          }
          if (m2 != -INFINITY) {
            const float nm2 = -m2;
            float p0 = 0.f, p1 = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              p0 += ex2_fast(fmaf(v[i], scale2, nm2));
              p1 += ex2_fast(fmaf(v[i + 1], scale2, nm2));
            }
            l += (double)(p0 + p1);
          }
        }
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty0 + 8 * buf);
      }
      // merge the warpgroups' row statistics (after every reader of the
      // previous item's bcol / rpos is done)
      pm[wg * 128 + r] = m2;
      pl[wg * 128 + r] = l;
      epi_bar();
      if (wg == 0) {
        float M2 = -INFINITY;
#pragma unroll
        for (int e = 0; e < kEpiGroups; ++e) M2 = fmaxf(M2, pm[e * 128 + r]);
        double Ls = 0.0;
        if (M2 != -INFINITY) {
#pragma unroll
          for (int e = 0; e < kEpiGroups; ++e) {
            const float me = pm[e * 128 + r];
            if (me != -INFINITY) Ls += pl[e * 128 + r] * exp2((double)me - (double)M2);
          }
        }
        if (valid) {
          const size_t srow = (size_t)(b * a.Hq + h * G + quarter) * a.Lq + (pos - a.q0);
          a.row_m2[srow] = M2;
          a.row_l[srow] = Ls;
        }
        bcol[r] = valid ? (float)((double)M2 + log2(Ls)) : INFINITY;
        rpos[r] = valid ? pos : -1;
      }
      epi_bar();
      // ---- pass 2: pooled score of key j0 + r over this warpgroup's blocks
      const float inv_rows = 1.0f / (float)((a.per_head ? 1 : G) * rows_t);
      // pooled rows: one per kv head, or with per_head one per query head
      // (column chunk ch of the accumulator holds query head h G + ch)
      const size_t pooled_row = (size_t)chunk_pooled_len(a.N, t0, a.tile);
      float* pooled = a.pooled + (a.per_head ? (size_t)(b * a.Hq + h * G) : (size_t)bh) * pooled_row +
                      chunk_pooled_offset(t, t0, a.tile);
      for (int blk = 0; blk < nb; ++blk, ++acount) {
        if (acount % kEpiGroups != wg) continue;
        const int buf = acount % kBufs;
        wait_acc(buf, (acount / kBufs) & 1);
        tc::fence_after();
        const int j = blk * kKB + r;
        const bool diag = blk * kKB + kKB - 1 > i0;
        float c0 = 0.f, c1 = 0.f;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          float v[32];
          tc::tmem_ld32(tmem + lane_addr + (uint32_t)(buf * 128 + ch * 32), v);
          const float4* bc = reinterpret_cast<const float4*>(bcol + ch * 32);
          const int4* rp = reinterpret_cast<const int4*>(rpos + ch * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 bb = bc[q4];
            float e0 = ex2_fast(fmaf(v[q4 * 4 + 0], scale2, -bb.x));
            float e1 = ex2_fast(fmaf(v[q4 * 4 + 1], scale2, -bb.y));
            float e2 = ex2_fast(fmaf(v[q4 * 4 + 2], scale2, -bb.z));
            float e3 = ex2_fast(fmaf(v[q4 * 4 + 3], scale2, -bb.w));
            if (diag) {
              const int4 pp = rp[q4];
              e0 = j <= pp.x ? e0 : 0.f;
              e1 = j <= pp.y ? e1 : 0.f;
              e2 = j <= pp.z ? e2 : 0.f;
              e3 = j <= pp.w ? e3 : 0.f;
            }
            c0 += e0 + e1;
            c1 += e2 + e3;
          }
          if (a.per_head) {
            if (ch < G && j < e_t) pooled[(size_t)ch * pooled_row + j] = (c0 + c1) * inv_rows;
            c0 = c1 = 0.f;
          }
        }
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty0 + 8 * buf);
        if (!a.per_head && j < e_t) pooled[j] = (c0 + c1) * inv_rows;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, 128 * kBufs);
  }
}

}  // namespace

bool score_pool_tc_supported(const ScorePoolArgs& a) { return a.G <= 4 && (a.D == 64 || a.D == 128); }

cudaError_t launch_score_pool_tc(const ScorePoolArgs& a, int* err, int num_sms, cudaStream_t stream) {
  CUtensorMap mq, mk;
  if (!tc::make_map_3d(&mq, a.q, (uint64_t)a.D, (uint64_t)a.Lq, (uint64_t)a.B * a.Hq, 32) ||
      !tc::make_map_3d(&mk, a.k, (uint64_t)a.D, (uint64_t)a.N, (uint64_t)a.B * a.Hkv, kKB))
    return cudaErrorInvalidValue;
  const int T = (a.N + a.tile - 1) / a.tile - a.q0 / a.tile;   // the call's query tiles
  const long items = (long)T * a.B * a.Hkv;
  const int grid = (int)(items < num_sms ? items : num_sms);
  const bool pdl = (a.flags & 1) != 0;
  if (a.D == 128) {
    const cudaError_t e =
        ensure_func_attrs(reinterpret_cast<const void*>(score_pool_tc_kernel<128>), SPL<128>::alloc, false);
    if (e != cudaSuccess) return e;
    return launch_ex(score_pool_tc_kernel<128>, dim3(grid), dim3(kThreads), SPL<128>::alloc, stream, pdl, 1, mq, mk,
                     a, err);
  }
  const cudaError_t e =
      ensure_func_attrs(reinterpret_cast<const void*>(score_pool_tc_kernel<64>), SPL<64>::alloc, false);
  if (e != cudaSuccess) return e;
  return launch_ex(score_pool_tc_kernel<64>, dim3(grid), dim3(kThreads), SPL<64>::alloc, stream, pdl, 1, mq, mk, a,
                   err);
}

}  // namespace kascade
