// Gather-sparse prefill attention on the 5th-generation tensor cores, for
// the Kascade anchor and reuse layers (README, Abstract: reuse layers attend
// only over the anchor's Top-k indices; selection and attention are
// tile-level in prefill).  Same results as the warp-MMA kernel in
// sparse_attn.cu: for every query row i of tile t and every query head of
// the group, softmax over the tile's selected keys j <= i of q_i . k_j /
// sqrt(d), times V.  With an implicit key list [0, e_t) (causal) or [0, N)
// the same kernel is the dense reference.
//
// Work item = (query tile, row block, batch x kv head): 128 MMA rows = 4
// query heads x 32 queries (rows of absent heads are zero and never stored).
// Persistent CTAs take items head by head, longest tile first.  Each CTA
// runs two independent pipelines ("subs") on alternate items of its share,
// so that one pipeline's softmax overlaps the other's products and gathers.
// Per pipeline:
//   4 softmax warps   one TMEM lane (= one query row) per thread: read S
//                     with tcgen05.ld, mask causally by original key index,
//                     keep the running max and sum, write P (bf16) into TMEM
//                     as the A operand of the second product; finally read
//                     O, normalise and store it.  The running max used for
//                     the exponent is raised (and O, l rescaled in TMEM) only
//                     when a row's max grows by more than 2^8, which keeps
//                     the result exact and P within bf16 range;
//   2 gather warps    64 selected K and V rows per block, 16-byte cp.async
//                     into 128-byte-swizzled shared memory (kStages blocks),
//                     completion tracked per thread on the stage's mbarrier;
//                     one thread also TMA-loads the item's Q tile;
//   1 MMA thread      tcgen05.mma by readiness: S = Q K^T (M = 128, N = 64)
//                     and O += P V (M = 128, N = d, P from TMEM, V an MN-major
//                     shared-memory operand).
// All hand-offs are mbarriers; every wait is bounded and a timeout stops the
// CTA's waits and records an error code in the workspace error word.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace kascade {

namespace {

constexpr int kKB = 64;          // keys per block
constexpr int kSubs = 2;         // independent pipelines per CTA
constexpr int kStages = 2;       // K/V blocks in flight per pipeline
constexpr int kGather = 64;      // gather threads per pipeline
constexpr int kThreads = 448;    // 8 softmax warps, 4 gather warps, 2 MMA warps
constexpr int kErrTimeout = 4;
constexpr float kRescale = 8.0f; // log2 growth of a row max that forces a rescale
constexpr int kNoKey = 0x7fffffff;
// TMEM columns of pipeline `sub` start at 256 sub: S (kKB), P (kKB / 2, bf16
// pairs), O (128)
constexpr uint32_t kColS = 0, kColP = 64, kColO = 128;

template <int D>
struct PAL {
  static constexpr int QB = 128 * D * 2;            // Q tile
  static constexpr int QCB = 128 * 128;             // one 64-column block of the Q tile
  static constexpr int KB = kKB * D * 2;            // K (or V) of one block
  static constexpr int KVCB = kKB * 128;            // one 64-column block of K (or V)
  static constexpr size_t SUB = (size_t)QB + (size_t)kStages * 2 * KB;   // Q then the K/V stages
  static constexpr size_t bars = kSubs * SUB;
  static constexpr int NBARS = 10 + 2 * kStages;    // per pipeline
  static constexpr size_t tslot = bars + (size_t)kSubs * NBARS * 8;
  static constexpr size_t stop = tslot + 8;
  static constexpr size_t total = stop + 8;
  static constexpr size_t alloc = total + 1024;      // slack for 1024-byte alignment
  static_assert(SUB % 1024 == 0 && QB % 1024 == 0 && KB % 1024 == 0, "swizzled tiles");
  static_assert(bars % 8 == 0, "mbarrier alignment");
  static_assert(alloc <= 232448, "more than 227 KB of shared memory per block");
};

// barrier slots of one pipeline
constexpr int bQFull = 0, bQEmpty = 1, bSFull = 2, bSEmpty = 3, bPFull = 4, bPEmpty = 5, bODone = 6, bOEmpty = 7,
              bDrain = 8, bKVFull = 10, bKVEmpty = 10 + kStages;
static_assert(bKVEmpty + kStages == PAL<128>::NBARS, "barrier count");

// One work item: which rows, which key list.
struct Item {
  int b, h, hq0, i0, rows_t, list_len, nb;
  const int32_t* list;   // NULL: dense (keys 0, 1, ...)
};

__device__ __forceinline__ Item item_of(const AttnArgs& a, int it, int T, int RB) {
  // head-major, longest tile first within a head: the CTAs in flight share
  // one head's K and V, which then stay in L2
  Item I;
  const int t0 = a.q0 / a.tile;   // first query tile of the call (rolling chunks)
  const int Tc = T - t0;
  const int bh = it / (RB * Tc);
  const int rem = it - bh * (RB * Tc);
  const int t = T - 1 - rem / RB, rb = rem - (rem / RB) * RB;
  I.b = bh / a.Hp;
  I.h = bh - I.b * a.Hp;        // problem of the batch row
  I.hq0 = I.h * a.G + rb * 4;   // first query head of the row block
  I.i0 = t * a.tile;
  const int e_t = min(I.i0 + a.tile, a.N);
  I.rows_t = e_t - I.i0;
  I.list = nullptr;
  if (a.idx) {
    const int hm_raw = a.one_list ? 0 : (a.head_map ? a.head_map[I.h] : I.h);
    const bool hm_ok = hm_raw >= 0 && hm_raw < a.n_lists;
    const int hm = hm_ok ? hm_raw : 0;
    const int64_t row_len = chunk_row_len(a.N, t0, a.tile, a.num, a.den);
    I.list = a.idx + (size_t)(I.b * a.n_lists + hm) * row_len + chunk_list_offset(t, t0, a.tile, a.num, a.den);
    I.list_len = hm_ok ? topk_count(e_t, a.num, a.den) : 0;
  } else {
    I.list_len = a.causal ? e_t : a.N;
  }
  I.nb = (I.list_len + kKB - 1) / kKB;
  return I;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap mq, const AttnArgs a, int RB) {
  using L = PAL<D>;
  constexpr int CB = D / 64;
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  char* sm = smem_raw + (base - raw);
  volatile int* stop = reinterpret_cast<volatile int*>(sm + L::stop);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // roles: warps 0-3 / 4-7 softmax of pipeline 0 / 1, warps 8-9 / 10-11
  // gather, warps 12 / 13 MMA issue (warp 12 also owns TMEM)
  const int sub = warp < 8 ? warp >> 2 : (warp < 12 ? (warp - 8) >> 1 : warp - 12);
  const uint32_t q_s = base + (uint32_t)(sub * L::SUB), kv_s = q_s + (uint32_t)L::QB;
  const uint32_t bar0 = base + (uint32_t)(L::bars + (size_t)sub * L::NBARS * 8);
  auto bar = [&](int slot) { return bar0 + 8u * (uint32_t)slot; };
  const int G = a.G;
  const int T = (a.N + a.tile - 1) / a.tile;
  const int items = (T - a.q0 / a.tile) * RB * a.B * a.Hp;
  const bool causal = a.idx != nullptr || a.causal;
  const int heads_rb = min(4, G);   // query heads per row block
  // this pipeline's items: the CTA's share, alternating between pipelines
  const int it0 = blockIdx.x + sub * gridDim.x, istep = kSubs * gridDim.x;

  if (threadIdx.x == 0) {
    for (int p = 0; p < kSubs; ++p) {
      const uint32_t b0 = base + (uint32_t)(L::bars + (size_t)p * L::NBARS * 8);
      mbar_init(b0 + 8 * bQFull, 1);
      mbar_init(b0 + 8 * bQEmpty, 1);
      mbar_init(b0 + 8 * bSFull, 1);
      mbar_init(b0 + 8 * bSEmpty, 4);
      mbar_init(b0 + 8 * bPFull, 4);
      mbar_init(b0 + 8 * bPEmpty, 1);
      mbar_init(b0 + 8 * bODone, 1);
      mbar_init(b0 + 8 * bOEmpty, 4);
      mbar_init(b0 + 8 * bDrain, 1);
      for (int s = 0; s < kStages; ++s) {
        mbar_init(b0 + 8 * (bKVFull + s), kGather);
        mbar_init(b0 + 8 * (bKVEmpty + s), 1);
      }
    }
    *stop = 0;
    mbar_fence_init();
  }
  // rows of absent heads (G < 4) stay zero in both pipelines' Q tiles
  for (int i = threadIdx.x; i < kSubs * CB * (4 - heads_rb) * 32 * 8; i += kThreads) {
    const int per_sub = CB * (4 - heads_rb) * 32 * 8;
    const int p = i / per_sub, rem0 = i - p * per_sub;
    const int cb = rem0 / ((4 - heads_rb) * 32 * 8), rem = rem0 - cb * (4 - heads_rb) * 32 * 8;
    const int r = 32 * heads_rb + rem / 8, ch = rem % 8;
    *reinterpret_cast<uint4*>(sm + (size_t)p * L::SUB + cb * L::QCB + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
  }
  fence_async_smem();
  if (warp == 12) tc::tmem_alloc(base + (uint32_t)L::tslot, 512);
  pdl_wait();
  pdl_launch_dependents();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::tslot) + (uint32_t)(256 * sub);

  // bounded wait; after a timeout every later wait is skipped so that all
  // loops run to their (finite) ends
  auto wait = [&](int slot, int parity) {
    if (*stop) return;
    if (!mbar_wait_bounded(bar(slot), (uint32_t)(parity & 1))) {
      *stop = 1;
      raise_error(a.err, kErrTimeout);
    }
  };

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------ gather
    // thread -> 16-byte chunk c of rows r0, r0 + RPP, ...: one warp
    // instruction copies whole 256-byte rows.  The key indices of the next
    // block are loaded one block ahead, and every thread arrives on the
    // stage's barrier asynchronously when its copies land, so the gather
    // only ever waits for a free stage.
    constexpr int CH = D / 8, RPP = kGather / CH, KR = kKB / RPP;
    const int pt = threadIdx.x - 256 - kGather * sub;
    const int c = pt % CH, r0 = pt / CH;
    const int cb = c >> 3, cc = c & 7;
    auto load_keys = [&](const Item& I, int j, int (&kk)[KR]) {
#pragma unroll
      for (int u = 0; u < KR; ++u) {
        const int pos = j * kKB + r0 + RPP * u;
        kk[u] = pos < I.list_len ? (I.list ? __ldg(I.list + pos) : pos) : kNoKey;
      }
    };
    int cur[KR], nxt[KR];
    int pf_it = -1, pf_j = 0;   // block whose keys sit in cur
    int n = 0, qn = 0;
    if (it0 < items) {
      const Item I0 = item_of(a, it0, T, RB);
      if (I0.nb > 0) {
        load_keys(I0, 0, cur);
        pf_it = it0;
      }
    }
    for (int it = it0; it < items; it += istep, ++qn) {
      const Item I = item_of(a, it, T, RB);
      const int it2 = it + istep;
      const Item I2 = item_of(a, it2 < items ? it2 : it, T, RB);
      const bool have2 = it2 < items && I2.nb > 0;
      if (pt == 0) {
        if (qn >= 1) wait(bQEmpty, qn - 1);
        mbar_arrive_expect_tx(bar(bQFull), (uint32_t)(CB * heads_rb * 32 * 128));
        for (int b = 0; b < CB; ++b)
          for (int g = 0; g < heads_rb; ++g)
            tc::tma_load_3d(q_s + b * L::QCB + g * 4096, &mq, b * 64, I.i0 - a.q0, I.b * a.Hq + I.hq0 + g,
                            bar(bQFull));
      }
      const size_t bhoff = (size_t)kv_slab_of(I.b, I.h * a.G, a.Hkv, a.Gkv) * a.N * D;
      for (int j = 0; j < I.nb; ++j, ++n) {
        if (pf_it != it || pf_j != j) load_keys(I, j, cur);   // not prefetched (rare)
        int nx_it = -1, nx_j = 0;
        if (j + 1 < I.nb) {
          load_keys(I, j + 1, nxt);
          nx_it = it;
          nx_j = j + 1;
        } else if (have2) {
          load_keys(I2, 0, nxt);
          nx_it = it2;
        }
        const int s = n % kStages;
        if (n >= kStages) wait(bKVEmpty + s, n / kStages - 1);
        const uint32_t kd = kv_s + (uint32_t)(s * 2 * L::KB);
        const uint32_t vd = kd + L::KB;
#pragma unroll
        for (int u = 0; u < KR; ++u) {
          const int row = r0 + RPP * u;
          const bool ok = cur[u] != kNoKey;
          const size_t src = bhoff + (size_t)(ok ? cur[u] : 0) * D + c * 8;
          const uint32_t off = (uint32_t)(cb * L::KVCB + row * 128 + ((cc ^ (row & 7)) << 4));
          cp_async_16(kd + off, a.k + src, ok ? 16 : 0);
          cp_async_16(vd + off, a.v + src, ok ? 16 : 0);
        }
        cp_async_mbar_arrive(bar(bKVFull + s));
#pragma unroll
        for (int u = 0; u < KR; ++u) cur[u] = nxt[u];
        pf_it = nx_it;
        pf_j = nx_j;
      }
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    // no TMA copy may still be in flight when the CTA exits
    if (pt == 0 && qn > 0 && !mbar_wait_bounded(bar(bQFull), (qn - 1) & 1)) raise_error(a.err, kErrTimeout);
  } else if (warp >= 12) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16_f32(128, kKB);
      const uint32_t id2 = tc::idesc_bf16_f32_bmn(128, D);
      int n = 0, qn = 0;
      for (int it = it0; it < items; it += istep, ++qn) {
        const Item I = item_of(a, it, T, RB);
        wait(bQFull, qn);
        tc::fence_after();
        auto mma1 = [&](int m) {   // S = Q K_m^T
          const int s = m % kStages;
          tc::fence_after();
          const uint32_t ks = kv_s + (uint32_t)(s * 2 * L::KB);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = (uint32_t)((kk >> 2) * L::QCB + (kk & 3) * 32);
            const uint32_t koff = (uint32_t)((kk >> 2) * L::KVCB + (kk & 3) * 32);
            tc::mma_bf16(tmem + kColS, tc::smem_desc_sw128(q_s + qoff), tc::smem_desc_sw128(ks + koff), id1, kk > 0);
          }
          tc::commit(bar(bSFull));
        };
        auto mma2 = [&](int m, int j) {   // O += P V_m, P from TMEM
          const int s = m % kStages;
          tc::fence_after();
          const uint32_t vs = kv_s + (uint32_t)(s * 2 * L::KB + L::KB);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)
            tc::mma_bf16_ts(tmem + kColO, tmem + kColP + (uint32_t)(kk * 8),
                            tc::smem_desc_sw128_mn(vs + kk * 2048, L::KVCB), id2, (j > 0 || kk > 0) ? 1u : 0u);
          tc::commit(bar(bKVEmpty + s));
          tc::commit(bar(bPEmpty));
          tc::commit(bar(bODone));
        };
        // issue whichever product is ready: P V of the oldest published
        // block, else S of the next block (at most one ahead: S and P are
        // single buffers)
        int i1 = 0, i2 = 0;
        long long t_last = clock64();
        while (i2 < I.nb && !*stop) {
          bool did = false;
          if (i2 < i1) {
            const int m = n + i2;
            if (mbar_test(bar(bPFull), (uint32_t)(m & 1)) &&
                (i2 > 0 || qn < 1 || mbar_test(bar(bOEmpty), (uint32_t)((qn - 1) & 1)))) {
              mma2(m, i2);
              ++i2;
              did = true;
            }
          }
          if (!did && i1 < I.nb && i1 <= i2 + 1) {
            const int m = n + i1;
            if (mbar_test(bar(bKVFull + m % kStages), (uint32_t)((m / kStages) & 1)) &&
                (m < 1 || mbar_test(bar(bSEmpty), (uint32_t)((m - 1) & 1)))) {
              mma1(m);
              ++i1;
              did = true;
            }
          }
          if (did) {
            t_last = clock64();
          } else if (clock64() - t_last > (1ll << 32)) {
            *stop = 1;
            raise_error(a.err, kErrTimeout);
          }
        }
        tc::commit(bar(bQEmpty));
        n += I.nb;
      }
      // every issued MMA completes before TMEM is released
      tc::commit(bar(bDrain));
      if (!mbar_wait_bounded(bar(bDrain), 0)) raise_error(a.err, kErrTimeout);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x & 127;                  // TMEM lane = MMA row
    const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
    const float scale2 = kLog2e * rsqrtf((float)D);
    int n = 0, qn = 0;
    int ocnt = 0;                                     // completed MMA2 groups of this pipeline
    for (int it = it0; it < items; it += istep, ++qn) {
      const Item I = item_of(a, it, T, RB);
      const int g = r >> 5, qi = r & 31;
      const int pos = I.i0 + qi;
      const bool valid = g < heads_rb && qi < I.rows_t;
      float m_used = -INFINITY, l = 0.f;
      // last key of block j (lists are ascending), loaded one block ahead
      auto last_key = [&](int j) {
        const int q = min(j * kKB + kKB, I.list_len) - 1;
        return I.list ? __ldg(I.list + q) : q;
      };
      int last_next = I.nb > 0 ? last_key(0) : 0;
      for (int j = 0; j < I.nb; ++j) {
        const int m = n + j;
        // the block needs a per-key check if it holds keys past the list
        // end or (causal) keys after the tile start
        const int pos0 = j * kKB;
        const bool tail = pos0 + kKB > I.list_len;
        const int last = last_next;
        if (j + 1 < I.nb) last_next = last_key(j + 1);
        const bool check = tail || (causal && last > I.i0);
        wait(bSFull, m);
        tc::fence_after();
        float v[kKB];
        tc::tmem_ld32(tmem + lane_addr + kColS, *reinterpret_cast<float(*)[32]>(v));
        tc::tmem_ld32(tmem + lane_addr + kColS + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bSEmpty));
        if (check) {
#pragma unroll
          for (int c = 0; c < kKB; ++c) {
            const int q = pos0 + c;
            const int key = q < I.list_len ? (I.list ? __ldg(I.list + q) : q) : kNoKey;
            if (key == kNoKey || (causal && key > pos)) v[c] = -INFINITY;
          }
        }
        float mx4[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
        for (int c = 4; c < kKB; c += 4) {
          mx4[0] = fmaxf(mx4[0], v[c]);
          mx4[1] = fmaxf(mx4[1], v[c + 1]);
          mx4[2] = fmaxf(mx4[2], v[c + 2]);
          mx4[3] = fmaxf(mx4[3], v[c + 3]);
        }
        const float mx2 = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale2;   // scale > 0 keeps the order
        float m_new = m_used;
        bool resc = false;
        if (mx2 > m_used) {
          if (m_used == -INFINITY) {
            m_new = mx2;                 // no visible key so far: this row of O is zero
          } else if (mx2 > m_used + kRescale) {
            m_new = mx2;
            resc = true;
          }
        }
        if (__any_sync(0xffffffffu, resc)) {
          // rescale O (and l) once the previous block's P V has landed
          wait(bODone, ocnt + j - 1);
          tc::fence_after();
          const float alpha = resc ? exp2f(m_used - m_new) : 1.0f;
#pragma unroll 1
          for (int c32 = 0; c32 < D / 32; ++c32) {
            float o[32];
            const uint32_t ta = tmem + lane_addr + kColO + (uint32_t)(c32 * 32);
            tc::tmem_ld32(ta, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::tmem_st32(ta, o);
          }
          l *= alpha;
        }
        m_used = m_new;
        // P = exp2(s * scale2 - m_used) in bf16, row r of the block's A tile
        uint32_t pk[kKB / 2];
        if (m_used == -INFINITY) {
#pragma unroll
          for (int c = 0; c < kKB / 2; ++c) pk[c] = 0u;
        } else {
          const float nm = -m_used;
          float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < kKB; c += 4) {
            const float p0 = ex2_fast(fmaf(v[c], scale2, nm));
            const float p1 = ex2_fast(fmaf(v[c + 1], scale2, nm));
            const float p2 = ex2_fast(fmaf(v[c + 2], scale2, nm));
            const float p3 = ex2_fast(fmaf(v[c + 3], scale2, nm));
            ps[0] += p0;
            ps[1] += p1;
            ps[2] += p2;
            ps[3] += p3;
            pk[c / 2] = pack_bf16(p0, p1);
            pk[c / 2 + 1] = pack_bf16(p2, p3);
          }
          l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        }
        if (m >= 1) wait(bPEmpty, m - 1);
        tc::tmem_st16(tmem + lane_addr + kColP, *reinterpret_cast<uint32_t(*)[16]>(pk));
        tc::tmem_st16(tmem + lane_addr + kColP + 16, *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
        tc::fence_before();   // orders the P store and a TMEM rescale of O before the next P V
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bPFull));
      }
      // ---- output rows: O / l, bf16
      if (I.nb > 0) {
        wait(bODone, ocnt + I.nb - 1);
        tc::fence_after();
      }
      ocnt += I.nb;
      const float inv = l > 0.f ? 1.0f / l : 0.0f;
      __nv_bfloat16* orow = a.o + ((size_t)(I.b * a.Hq + I.hq0 + g) * a.Lq + (pos - a.q0)) * D;
#pragma unroll 1
      for (int c32 = 0; c32 < D / 32; ++c32) {
        float o[32];
        if (I.nb > 0) {
          tc::tmem_ld32(tmem + lane_addr + kColO + (uint32_t)(c32 * 32), o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack_bf16(o[i] * inv, o[i + 1] * inv);
            w.y = pack_bf16(o[i + 2] * inv, o[i + 3] * inv);
            w.z = pack_bf16(o[i + 4] * inv, o[i + 5] * inv);
            w.w = pack_bf16(o[i + 6] * inv, o[i + 7] * inv);
            *reinterpret_cast<uint4*>(orow + c32 * 32 + i) = w;
          }
        }
      }
      if (valid && a.lse)
        a.lse[(size_t)(I.b * a.Hq + I.hq0 + g) * a.Lq + (pos - a.q0)] =
            l > 0.f ? (m_used + log2f(l)) * (float)kLn2 : -INFINITY;
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bOEmpty));
      n += I.nb;
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before();
  __syncthreads();
  if (warp == 12) {
    tc::fence_after();
    tc::tmem_dealloc(*reinterpret_cast<volatile uint32_t*>(sm + L::tslot), 512);
  }
}

}  // namespace

bool prefill_attn_tc_supported(const AttnArgs& a) {
  return (a.D == 64 || a.D == 128) && a.tile == 32 && (a.G <= 4 || a.G % 4 == 0);
}

cudaError_t launch_prefill_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t stream) {
  CUtensorMap mq;
  if (!tc::make_map_3d(&mq, a.q, (uint64_t)a.D, (uint64_t)a.Lq, (uint64_t)a.B * a.Hq, 32)) return cudaErrorInvalidValue;
  const int T = (a.N + a.tile - 1) / a.tile - a.q0 / a.tile;   // the call's query tiles
  const int RB = a.G <= 4 ? 1 : a.G / 4;
  const long items = (long)T * RB * a.B * a.Hp;
  const long long ctas = (items + kSubs - 1) / kSubs;
  const int grid = (int)(ctas < num_sms ? ctas : num_sms);
  const bool pdl = (a.flags & 1) != 0;
  if (a.D == 128) {
    const cudaError_t e =
        ensure_func_attrs(reinterpret_cast<const void*>(prefill_attn_tc_kernel<128>), PAL<128>::alloc, false);
    if (e != cudaSuccess) return e;
    return launch_ex(prefill_attn_tc_kernel<128>, dim3(grid), dim3(kThreads), PAL<128>::alloc, stream, pdl, 1, mq,
                     a, RB);
  }
  const cudaError_t e =
      ensure_func_attrs(reinterpret_cast<const void*>(prefill_attn_tc_kernel<64>), PAL<64>::alloc, false);
  if (e != cudaSuccess) return e;
  return launch_ex(prefill_attn_tc_kernel<64>, dim3(grid), dim3(kThreads), PAL<64>::alloc, stream, pdl, 1, mq, a,
                   RB);
}

}  // namespace kascade
