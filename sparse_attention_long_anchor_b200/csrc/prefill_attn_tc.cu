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
// Persistent CTAs take items head by head, longest tile first.  Per CTA:
//   warps 0..3  softmax: one TMEM lane (= one query row) per thread; reads S
//               with tcgen05.ld, applies the causal mask by original key
//               index, keeps the running max and sum, writes P (bf16) into
//               shared memory as the A operand of the second product, and
//               finally reads O, normalises and stores it.  The running max
//               used for the exponent is raised (and O, l rescaled in TMEM)
//               only when a row's max grows by more than 2^8, which keeps
//               the result exact and P within bf16 range;
//   warps 4..7  gather: 64 selected K and V rows per block, 16-byte
//               cp.async into 128-byte-swizzled shared memory, a ring of
//               kStages blocks; one thread also issues the TMA loads of the
//               item's Q tile (double-buffered);
//   warp 8      single-thread tcgen05.mma issue and TMEM owner:
//               S = Q K^T (M = 128, N = 64, into one of two TMEM buffers),
//               O += P V (M = 128, N = d, V as an MN-major operand, into
//               one of two TMEM output buffers, one per item in flight).
// All hand-offs are mbarriers; every wait is bounded and a timeout stops the
// CTA's waits and records an error code in the workspace error word.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace kascade {

namespace {

constexpr int kKB = 64;          // keys per block
constexpr int kStages = 4;       // K/V ring; >= 3 keeps the MMA issue order deadlock-free
constexpr int kThreads = 288;    // 4 softmax warps, 4 gather warps, 1 MMA warp
constexpr int kErrTimeout = 4;
constexpr float kRescale = 8.0f; // log2 growth of a row max that forces a rescale
constexpr int kNoKey = 0x7fffffff;

template <int D>
struct PAL {
  static constexpr int QB = 128 * D * 2;            // Q tile
  static constexpr int QCB = 128 * 128;             // one 64-column block of the Q tile
  static constexpr int KB = kKB * D * 2;            // K (or V) of one block
  static constexpr int KVCB = kKB * 128;            // one 64-column block of K (or V)
  static constexpr int PB = 128 * kKB * 2;          // P of one block
  static constexpr size_t q = 0;                     // [2] Q
  static constexpr size_t kv = q + 2 * (size_t)QB;   // [S] K then V
  static constexpr size_t p = kv + (size_t)kStages * 2 * KB;   // [2] P
  static constexpr size_t keys = p + 2 * (size_t)PB; // [S][64] key index per row (kNoKey past the list)
  static constexpr size_t bars = keys + (size_t)kStages * kKB * 4;
  static constexpr int NBARS = 4 + 2 * kStages + 12 + 1;
  static constexpr size_t tslot = bars + NBARS * 8;
  static constexpr size_t stop = tslot + 8;
  static constexpr size_t total = stop + 8;
  static constexpr size_t alloc = total + 1024;      // slack for 1024-byte alignment
  static_assert(kv % 1024 == 0 && p % 1024 == 0 && KB % 1024 == 0 && PB % 1024 == 0, "swizzled tiles");
  static_assert(bars % 8 == 0, "mbarrier alignment");
  static_assert(alloc <= 232448, "more than 227 KB of shared memory per block");
};

// barrier slots
constexpr int bQFull = 0, bQEmpty = 2, bKVFull = 4, bKVEmpty = 4 + kStages, bSFull = 4 + 2 * kStages,
              bSEmpty = bSFull + 2, bPFull = bSEmpty + 2, bPEmpty = bPFull + 2, bODone = bPEmpty + 2,
              bOEmpty = bODone + 2, bDrain = bOEmpty + 2;
static_assert(bDrain + 1 == PAL<128>::NBARS, "barrier count");

// One work item: which rows, which key list.
struct Item {
  int b, h, hq0, i0, rows_t, list_len, nb;
  const int32_t* list;   // NULL: dense (keys 0, 1, ...)
};

__device__ __forceinline__ Item item_of(const AttnArgs& a, int it, int T, int RB) {
  // head-major, longest tile first within a head: the CTAs in flight share
  // one head's K and V, which then stay in L2
  Item I;
  const int bh = it / (RB * T);
  const int rem = it - bh * (RB * T);
  const int t = T - 1 - rem / RB, rb = rem - (rem / RB) * RB;
  I.b = bh / a.Hkv;
  I.h = bh - I.b * a.Hkv;
  I.hq0 = I.h * a.G + rb * 4;   // first query head of the row block
  I.i0 = t * a.tile;
  const int e_t = min(I.i0 + a.tile, a.N);
  I.rows_t = e_t - I.i0;
  I.list = nullptr;
  if (a.idx) {
    const int hm_raw = a.head_map ? a.head_map[I.h] : I.h;
    const bool hm_ok = hm_raw >= 0 && hm_raw < a.Hkv;
    const int hm = hm_ok ? hm_raw : 0;
    const int64_t row_len = tile_list_offset(T - 1, a.tile, a.num, a.den) + topk_count(a.N, a.num, a.den);
    I.list = a.idx + (size_t)(I.b * a.Hkv + hm) * row_len + tile_list_offset(t, a.tile, a.num, a.den);
    I.list_len = hm_ok ? topk_count(e_t, a.num, a.den) : 0;
  } else {
    I.list_len = a.causal ? e_t : a.N;
  }
  I.nb = (I.list_len + kKB - 1) / kKB;
  return I;
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap mq, const AttnArgs a, int RB) {
  using L = PAL<D>;
  constexpr int CB = D / 64;
  extern __shared__ __align__(1024) char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  char* sm = smem_raw + (base - raw);
  const uint32_t q_s = base + (uint32_t)L::q, kv_s = base + (uint32_t)L::kv, p_s = base + (uint32_t)L::p;
  int* keys_s = reinterpret_cast<int*>(sm + L::keys);
  const uint32_t bar0 = base + (uint32_t)L::bars;
  auto bar = [&](int slot) { return bar0 + 8u * (uint32_t)slot; };
  volatile int* stop = reinterpret_cast<volatile int*>(sm + L::stop);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.G;
  const int T = (a.N + a.tile - 1) / a.tile;
  const int items = T * RB * a.B * a.Hkv;
  const bool causal = a.idx != nullptr || a.causal;
  const int heads_rb = min(4, G);   // query heads per row block

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(bQFull + i), 1);
      mbar_init(bar(bQEmpty + i), 1);
      mbar_init(bar(bSFull + i), 1);
      mbar_init(bar(bSEmpty + i), 4);
      mbar_init(bar(bPFull + i), 4);
      mbar_init(bar(bPEmpty + i), 1);
      mbar_init(bar(bODone + i), 1);
      mbar_init(bar(bOEmpty + i), 4);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(bKVFull + s), 128);
      mbar_init(bar(bKVEmpty + s), 1);
    }
    mbar_init(bar(bDrain), 1);
    *stop = 0;
    mbar_fence_init();
  }
  // rows of absent heads (G < 4) stay zero in both Q buffers
  for (int i = threadIdx.x; i < 2 * CB * (4 - heads_rb) * 32 * 8; i += kThreads) {
    const int per_buf = CB * (4 - heads_rb) * 32 * 8;
    const int qb = i / per_buf, rem0 = i - qb * per_buf;
    const int cb = rem0 / ((4 - heads_rb) * 32 * 8), rem = rem0 - cb * (4 - heads_rb) * 32 * 8;
    const int r = 32 * heads_rb + rem / 8, ch = rem % 8;
    *reinterpret_cast<uint4*>(sm + L::q + (size_t)qb * L::QB + cb * L::QCB + r * 128 + ch * 16) =
        make_uint4(0, 0, 0, 0);
  }
  fence_async_smem();
  if (warp == 8) tc::tmem_alloc(base + (uint32_t)L::tslot, 512);
  pdl_wait();
  pdl_launch_dependents();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::tslot);

  // bounded wait; after a timeout every later wait is skipped so that all
  // loops run to their (finite) ends
  auto wait = [&](int slot, int parity) {
    if (*stop) return;
    if (!mbar_wait_bounded(bar(slot), (uint32_t)(parity & 1))) {
      *stop = 1;
      raise_error(a.err, kErrTimeout);
    }
  };

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ gather
    // thread -> 16-byte chunk c of rows r0, r0 + RPP, ...: one warp
    // instruction copies whole 256-byte rows
    constexpr int CH = D / 8, RPP = 128 / CH;
    const int pt = threadIdx.x - 128;
    const int c = pt % CH, r0 = pt / CH;
    const int cb = c >> 3, cc = c & 7;
    const __nv_bfloat16* kbase = a.k;
    const __nv_bfloat16* vbase = a.v;
    int n = 0, qn = 0, pend = -1;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++qn) {
      const Item I = item_of(a, it, T, RB);
      if (pt == 0) {
        const int qb = qn & 1;
        if (qn >= 2) wait(bQEmpty + qb, (qn >> 1) - 1);
        mbar_arrive_expect_tx(bar(bQFull + qb), (uint32_t)(CB * heads_rb * 32 * 128));
        for (int cb = 0; cb < CB; ++cb)
          for (int g = 0; g < heads_rb; ++g)
            tc::tma_load_3d(q_s + qb * L::QB + cb * L::QCB + g * 4096, &mq, cb * 64, I.i0,
                            I.b * a.Hq + I.hq0 + g, bar(bQFull + qb));
      }
      const size_t bhoff = (size_t)(I.b * a.Hkv + I.h) * a.N * D;
      for (int j = 0; j < I.nb; ++j, ++n) {
        const int s = n % kStages;
        if (n >= kStages) wait(bKVEmpty + s, n / kStages - 1);
        const uint32_t kd = kv_s + (uint32_t)(s * 2 * L::KB);
        const uint32_t vd = kd + L::KB;
#pragma unroll
        for (int u = 0; u < kKB / RPP; ++u) {
          const int row = r0 + RPP * u;
          const int pos = j * kKB + row;
          const bool ok = pos < I.list_len;
          const int key = ok ? (I.list ? __ldg(I.list + pos) : pos) : 0;
          if (c == 0) keys_s[s * kKB + row] = ok ? key : kNoKey;
          const size_t src = bhoff + (size_t)key * D + c * 8;
          const uint32_t off = (uint32_t)(cb * L::KVCB + row * 128 + ((cc ^ (row & 7)) << 4));
          cp_async_16(kd + off, kbase + src, ok ? 16 : 0);
          cp_async_16(vd + off, vbase + src, ok ? 16 : 0);
        }
        cp_async_commit();
        // the previous block of this thread has landed: publish it
        if (pend >= 0) {
          cp_async_wait<1>();
          fence_async_smem();
          mbar_arrive(bar(bKVFull + pend));
        }
        pend = s;
      }
    }
    cp_async_wait<0>();
    if (pend >= 0) {
      fence_async_smem();
      mbar_arrive(bar(bKVFull + pend));
    }
    // no TMA copy may still be in flight when the CTA exits
    if (pt == 0 && qn > 0 && !mbar_wait_bounded(bar(bQFull + ((qn - 1) & 1)), ((qn - 1) >> 1) & 1))
      raise_error(a.err, kErrTimeout);
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id1 = tc::idesc_bf16_f32(128, kKB);
      const uint32_t id2 = tc::idesc_bf16_f32_bmn(128, D);
      int n = 0, qn = 0;
      for (int it = blockIdx.x; it < items; it += gridDim.x, ++qn) {
        const Item I = item_of(a, it, T, RB);
        const int qb = qn & 1, ob = qn & 1;
        wait(bQFull + qb, qn >> 1);
        tc::fence_after();
        auto mma1 = [&](int m) {   // S[m & 1] = Q K_m^T
          const int s = m % kStages, sb = m & 1;
          wait(bKVFull + s, m / kStages);
          if (m >= 2) wait(bSEmpty + sb, (m >> 1) - 1);
          tc::fence_after();
          const uint32_t d = tmem + (uint32_t)(sb * kKB);
          const uint32_t ks = kv_s + (uint32_t)(s * 2 * L::KB);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = (uint32_t)((kk >> 2) * L::QCB + (kk & 3) * 32);
            const uint32_t koff = (uint32_t)((kk >> 2) * L::KVCB + (kk & 3) * 32);
            tc::mma_bf16(d, tc::smem_desc_sw128(q_s + qb * L::QB + qoff), tc::smem_desc_sw128(ks + koff), id1,
                         kk > 0);
          }
          tc::commit(bar(bSFull + sb));
        };
        auto mma2 = [&](int m, int j) {   // O[ob] += P[m & 1] V_m
          const int s = m % kStages, pb = m & 1;
          wait(bPFull + pb, m >> 1);
          if (j == 0 && qn >= 2) wait(bOEmpty + ob, (qn >> 1) - 1);
          tc::fence_after();
          const uint32_t d = tmem + 128u + (uint32_t)(ob * 128);
          const uint32_t vs = kv_s + (uint32_t)(s * 2 * L::KB + L::KB);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)
            tc::mma_bf16(d, tc::smem_desc_sw128(p_s + pb * L::PB + kk * 32),
                         tc::smem_desc_sw128_mn(vs + kk * 2048, L::KVCB), id2, (j > 0 || kk > 0) ? 1u : 0u);
          tc::commit(bar(bKVEmpty + s));
          tc::commit(bar(bPEmpty + pb));
          tc::commit(bar(bODone + ob));
        };
        if (I.nb > 0) mma1(n);
        for (int j = 0; j < I.nb; ++j) {
          if (j + 1 < I.nb) mma1(n + j + 1);
          mma2(n + j, j);
        }
        tc::commit(bar(bQEmpty + qb));
        n += I.nb;
      }
      // every issued MMA completes before TMEM is released
      tc::commit(bar(bDrain));
      if (!mbar_wait_bounded(bar(bDrain), 0)) raise_error(a.err, kErrTimeout);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;                        // TMEM lane = MMA row
    const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
    const float scale2 = kLog2e * rsqrtf((float)D);
    int n = 0, qn = 0;
    int ocnt[2] = {0, 0};                             // completed MMA2 groups per O buffer
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++qn) {
      const Item I = item_of(a, it, T, RB);
      const int ob = qn & 1;
      const int g = r >> 5, qi = r & 31;
      const int pos = I.i0 + qi;
      const bool valid = g < heads_rb && qi < I.rows_t;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < I.nb; ++j) {
        const int m = n + j;
        const int sb = m & 1, s = m % kStages, pb = m & 1;
        wait(bSFull + sb, m >> 1);
        wait(bKVFull + s, m / kStages);   // the block's key indices
        tc::fence_after();
        float v[kKB];
        tc::tmem_ld32(tmem + lane_addr + (uint32_t)(sb * kKB), *reinterpret_cast<float(*)[32]>(v));
        tc::tmem_ld32(tmem + lane_addr + (uint32_t)(sb * kKB + 32), *reinterpret_cast<float(*)[32]>(v + 32));
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bSEmpty + sb));
        // mask: lists are ascending with kNoKey past the end, so the last
        // entry tells whether any key of the block needs a check
        const int* kb = keys_s + s * kKB;
        const int last = kb[kKB - 1];
        if (causal ? last > I.i0 : last == kNoKey) {
#pragma unroll
          for (int c4 = 0; c4 < kKB; c4 += 4) {
            const int4 kk = *reinterpret_cast<const int4*>(kb + c4);
            if (causal) {
              if (kk.x > pos) v[c4] = -INFINITY;
              if (kk.y > pos) v[c4 + 1] = -INFINITY;
              if (kk.z > pos) v[c4 + 2] = -INFINITY;
              if (kk.w > pos) v[c4 + 3] = -INFINITY;
            } else {
              if (kk.x == kNoKey) v[c4] = -INFINITY;
              if (kk.y == kNoKey) v[c4 + 1] = -INFINITY;
              if (kk.z == kNoKey) v[c4 + 2] = -INFINITY;
              if (kk.w == kNoKey) v[c4 + 3] = -INFINITY;
            }
          }
        }
        float mx = v[0];
#pragma unroll
        for (int c = 1; c < kKB; ++c) mx = fmaxf(mx, v[c]);
        const float mx2 = mx * scale2;   // scale > 0 keeps the order; -inf stays -inf
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
          wait(bODone + ob, ocnt[ob] + j - 1);
          tc::fence_after();
          const float alpha = resc ? exp2f(m_used - m_new) : 1.0f;
#pragma unroll 1
          for (int c32 = 0; c32 < D / 32; ++c32) {
            float o[32];
            const uint32_t ta = tmem + lane_addr + 128u + (uint32_t)(ob * 128 + c32 * 32);
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
        float ps = 0.f;
        if (m_used == -INFINITY) {
#pragma unroll
          for (int c = 0; c < kKB / 2; ++c) pk[c] = 0u;
        } else {
          const float nm = -m_used;
#pragma unroll
          for (int c = 0; c < kKB; c += 2) {
            const float p0 = exp2f(fmaf(v[c], scale2, nm));
            const float p1 = exp2f(fmaf(v[c + 1], scale2, nm));
            ps += p0 + p1;
            pk[c / 2] = pack_bf16(p0, p1);
          }
        }
        l += ps;
        if (m >= 2) wait(bPEmpty + pb, (m >> 1) - 1);
        const uint32_t prow = p_s + (uint32_t)(pb * L::PB + r * 128);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          st_shared_v4(prow + ((cc ^ (r & 7)) << 4), pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        fence_async_smem();
        tc::fence_before();   // orders a TMEM rescale of O before the next P V
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bPFull + pb));
      }
      // ---- output rows: O / l, bf16
      if (I.nb > 0) {
        wait(bODone + ob, ocnt[ob] + I.nb - 1);
        tc::fence_after();
      }
      ocnt[ob] += I.nb;
      const float inv = l > 0.f ? 1.0f / l : 0.0f;
      __nv_bfloat16* orow = a.o + ((size_t)(I.b * a.Hq + I.hq0 + g) * a.N + pos) * D;
#pragma unroll 1
      for (int c32 = 0; c32 < D / 32; ++c32) {
        float o[32];
        if (I.nb > 0) {
          tc::tmem_ld32(tmem + lane_addr + 128u + (uint32_t)(ob * 128 + c32 * 32), o);
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
        a.lse[(size_t)(I.b * a.Hq + I.hq0 + g) * a.N + pos] =
            l > 0.f ? (m_used + log2f(l)) * (float)kLn2 : -INFINITY;
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(bOEmpty + ob));
      n += I.nb;
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before();
  __syncthreads();
  if (warp == 8) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool prefill_attn_tc_supported(const AttnArgs& a) {
  return (a.D == 64 || a.D == 128) && a.tile == 32 && (a.G <= 4 || a.G % 4 == 0);
}

cudaError_t launch_prefill_attn_tc(const AttnArgs& a, int num_sms, cudaStream_t stream) {
  CUtensorMap mq;
  if (!tc::make_map_3d(&mq, a.q, (uint64_t)a.D, (uint64_t)a.N, (uint64_t)a.B * a.Hq, 32)) return cudaErrorInvalidValue;
  const int T = (a.N + a.tile - 1) / a.tile;
  const int RB = a.G <= 4 ? 1 : a.G / 4;
  const long items = (long)T * RB * a.B * a.Hkv;
  const int grid = (int)(items < num_sms ? items : num_sms);
  const bool pdl = (a.flags & 1) != 0;
  if (a.D == 128) {
    cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)PAL<128>::alloc);
    if (e != cudaSuccess) return e;
    return launch_ex(prefill_attn_tc_kernel<128>, dim3(grid), dim3(kThreads), PAL<128>::alloc, stream, pdl, 1, mq,
                     a, RB);
  }
  cudaError_t e = cudaFuncSetAttribute(prefill_attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PAL<64>::alloc);
  if (e != cudaSuccess) return e;
  return launch_ex(prefill_attn_tc_kernel<64>, dim3(grid), dim3(kThreads), PAL<64>::alloc, stream, pdl, 1, mq, a,
                   RB);
}

}  // namespace kascade
