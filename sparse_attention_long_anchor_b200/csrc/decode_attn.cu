// Gather-sparse decode attention of the Kascade anchor and reuse layers
// (README, Abstract: reuse layers attend only over the anchor's Top-k
// indices; selection and reuse are head-aware).  With an implicit full key
// list the same kernel is the dense decode reference.
//
// One thread-block cluster per (batch, kv head); the index list is split
// evenly over the CTAs of the cluster and every warp owns the 16-key slices
// s = warp, warp + 8, ... of its CTA's share.  Each warp keeps its first two
// slices in flight from the start:
//   * K rows of its even slices go straight from global memory into the
//     registers of the 16x8x16 bf16 MMA (the contraction runs over d, so each
//     lane may take any permutation of d as long as q uses the same: lane
//     (g, c) loads dims [32s + 8c, +8) of key g, one 16-byte load per 32
//     dims); K rows of its odd slices go through a shared-memory slot and are
//     read back in the same permuted order;
//   * V rows go through a two-slot cp.async ring (16-byte chunks XOR-swizzled
//     by row, conflict-free for ldmatrix.trans);
//   * the G query rows sit in shared memory, read with 8-byte loads.
// With programmatic dependent launch and inputs the caller vouches for, all
// of that is issued before the kernel waits for its predecessor, so for the
// usual list lengths every byte a CTA needs lands while the previous layer
// is still running.
// S^T = K Q^T and O^T += V^T P^T with the keys, then the head dims, as the
// MMA rows and the query heads of the group as its columns; fp32 online
// softmax per head.
// The partial (max, sum, output) of each CTA is pushed with st.async into
// the shared memory of the CTA that owns each output element, completing on
// the owner's mbarrier; every CTA waits only for its own bytes and merges its
// slice.  No global scratch; the one wait is bounded.
#include <cooperative_groups.h>

#include <type_traits>

#include "cluster_choice.h"
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace kascade {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxCS = 16;
constexpr int kIdxStage = 512;      // index entries staged in shared memory, short-list mode
constexpr int kIdxStageB = 3584;    // the bulk mode's (a 2-CTA cluster's share of 64K at 10 %)
constexpr int kErrMergeTimeout = 3; // device error word: a merge wait gave up
constexpr int kErrGather = 6;       // device error word: a bulk-copied row never arrived

template <int D>
struct Lay {
  static constexpr int ROWB = D * 2;                       // K / V row bytes (chunks swizzled)
  static constexpr int SLAB = 16 * ROWB;                   // one 16-key slab
  static constexpr int WARPB = 3 * SLAB;                   // V slot 0, V slot 1, K slot
  static constexpr size_t slabs = 0;
  static constexpr int IDXN = kIdxStage;
  static constexpr size_t qs = slabs + (size_t)kWarps * WARPB;   // [8][D] bf16 query rows
  static constexpr size_t idx = qs + 8 * D * 2;
  static constexpr size_t recv_o = idx + IDXN * 4;         // [G*D] f32, written by the peers
  static constexpr size_t recv_ml = recv_o + (8 * D + 4 * kMaxCS) * 4;   // [16][8] (m, l)
  static constexpr size_t bar = recv_ml + kMaxCS * 8 * 8;  // mbarrier of the incoming partials
  static constexpr size_t total = bar + 16;
  // after the gather loop, inside the slabs
  static constexpr int RO = D + 4;                         // padded red_o row (floats)
  static constexpr size_t red_o = 0;                       // [W][8][RO]
  static constexpr size_t red_ml = red_o + (size_t)kWarps * 8 * RO * 4;   // [W][8] (m, l)
  static constexpr size_t wf = red_ml + kWarps * 8 * 8;    // [W][8] weight of each warp's partial
  static constexpr size_t pml = wf + kWarps * 8 * 4;       // [8] (m, l) of this CTA
  static constexpr size_t wts = pml + 8 * 8;               // [16][8] weight of each CTA's partial
  static constexpr size_t head = wts + kMaxCS * 8 * 4;     // [8] (m, l) of the whole list
  static_assert(head + 8 * 8 <= qs, "post-loop scratch must fit in the slabs");
  static_assert(recv_o % 16 == 0 && recv_ml % 8 == 0 && bar % 8 == 0, "alignment");
  // two CTAs per SM: 228 KB per SM less 1 KB reserved per CTA
  static_assert(total <= (228 * 1024 - 2 * 1024) / 2, "two CTAs per SM");
};

// Bulk mode (many keys per CTA, one CTA per SM): each warp owns kStagesB
// stages of one 16-key slice, K rows then V rows, every row landing by one
// untiled bulk copy at a padded pitch of 2 D + 16 bytes.  Rows at that pitch
// shift by one 16-byte bank group, so the ldmatrix.trans reads of V (8 rows,
// one chunk) and the K reads below (lane (g, c) takes chunks
// 8 (q>>1) + 2c + (q&1) of rows g and g + 8) are conflict-free.
constexpr int kStagesB = 3;

template <int D>
struct BLay {
  static constexpr int ROWB = D * 2;
  static constexpr int PITCH = ROWB + 16;
  static constexpr int TB = 16 * PITCH;                    // 16 rows of one tensor
  static constexpr int STAGE = 2 * TB;                     // K rows, then V rows
  static constexpr int WARPB = kStagesB * STAGE;
  static constexpr int SLAB = 16 * ROWB;                   // (the short-list mode's unit; not used here)
  static constexpr int IDXN = kIdxStageB;
  static constexpr size_t slabs = 0;
  static constexpr size_t qs = slabs + (size_t)kWarps * WARPB;
  static constexpr size_t idx = qs + 8 * D * 2;
  static constexpr size_t recv_o = idx + IDXN * 4;
  static constexpr size_t recv_ml = recv_o + (8 * D + 4 * kMaxCS) * 4;
  static constexpr size_t bar = recv_ml + kMaxCS * 8 * 8;
  static constexpr size_t sbar = bar + 16;                 // [warps][stages] mbarriers of the stages
  static constexpr size_t total = sbar + (size_t)kWarps * kStagesB * 8;
  static constexpr int RO = D + 4;
  static constexpr size_t red_o = 0;
  static constexpr size_t red_ml = red_o + (size_t)kWarps * 8 * RO * 4;
  static constexpr size_t wf = red_ml + kWarps * 8 * 8;
  static constexpr size_t pml = wf + kWarps * 8 * 4;
  static constexpr size_t wts = pml + 8 * 8;
  static constexpr size_t head = wts + kMaxCS * 8 * 4;
  static_assert(PITCH % 16 == 0 && (PITCH / 16) % 8 == 1, "pitch must shift rows by one 16-byte bank group");
  static_assert(head + 8 * 8 <= qs, "post-loop scratch must fit in the stages");
  static_assert(recv_o % 16 == 0 && recv_ml % 8 == 0 && bar % 8 == 0, "alignment");
  static_assert(total <= 227 * 1024, "one CTA per SM");
};

// kMode bits 0-1: 0 = every warp owns at most two slices, all issued up
// front by cp.async (two CTAs per SM); 2 = bulk-copied stages refilled as
// they are consumed (one CTA per SM).  Bit 2 (kPagedBit): rows addressed
// through a page table.
constexpr int kPagedBit = 4;
// kMode bit 4 (bulk mode, contiguous cache, no index list: the dense form):
// a slice's 16 consecutive rows arrive as one 128-byte-swizzled TMA tile per
// 64 columns of K and of V, instead of one request per row
constexpr int kDenseBit = 16;
template <int D>
constexpr int kDenseStage = 2 * 16 * D * 2;   // K (16 rows) then V, each as 2 KB tiles of 64 columns
template <int D, int kMode>
using LayOf = typename std::conditional<(kMode & 3) == 2, BLay<D>, Lay<D>>::type;

__device__ __forceinline__ float scale_from(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.0f : exp2f(m_old - m_new);
}

// Softmax-merge weights of n <= 32 partial results (m, l) of one head,
// strided by 8 entries: lane i < n takes exp2(m_i - M) against the max M and
// writes it to w[8 i]; lane 0 writes (M, sum of w_i l_i).  Whole warp.
__device__ __forceinline__ void merge_weights(int n, const float2* ml, float* w, float2* out, int lane) {
  const float2 v = lane < n ? ml[lane * 8] : make_float2(-INFINITY, 0.f);
  float M = v.x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float f = scale_from(v.x, M);
  float ls = f * v.y;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  if (lane < n) w[lane * 8] = f;
  if (lane == 0) *out = make_float2(M, ls);
}

// kMode & 3 == 0: every warp owns at most two slices (per <= 16 * 2 *
// kWarps), all issued up front; == 2: kStagesB bulk-copied stages per warp
// refilled as they are consumed (one CTA per SM, for many keys per CTA).
// kMode & kPagedBit: K and V rows through the page table.
template <int D, int kMode>
__global__ void __launch_bounds__(kThreads, (kMode & 3) == 2 ? 1 : 2)
    decode_attn_kernel(const AttnArgs a, int per, const __grid_constant__ CUtensorMap mk,
                       const __grid_constant__ CUtensorMap mv) {
  using L = LayOf<D, kMode>;
  constexpr bool kBulk = (kMode & 3) == 2;
  constexpr bool kPaged = (kMode & kPagedBit) != 0;
  constexpr bool kDense = (kMode & kDenseBit) != 0;
  static_assert(!kDense || (kBulk && !kPaged), "the tile form serves the contiguous bulk mode");
  static_assert(!kDense || 1023 + kWarps * kStagesB * kDenseStage<D> <= kWarps * BLay<D>::WARPB,
                "aligned tile stages fit the stage region");
  constexpr int KS = D / 32;          // 16-byte K loads per key row per lane
  constexpr int CH = D / 8;           // 16-byte chunks per row
  extern __shared__ __align__(128) char smem[];
  // with PDL the gathers may start before the previous kernel completes only
  // if the caller vouched for k, v, idx and head_map; otherwise wait first
  const bool early = (a.flags & 3) == 3;
  if (!early) {
    pdl_wait();
    pdl_launch_dependents();
  }
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int bh = blockIdx.y;   // problem: batch row b, problem h of the row
  const int b = bh / a.Hp, h = bh - b * a.Hp;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = a.G;
  const int E = G * D;
  // output elements owned by each CTA: en (a multiple of 4) for the first
  // ones, what is left for the last owner, none past it
  const int en = ((E + CS - 1) / CS + 3) & ~3;
  const int en_mine = max(0, min(en, E - rank * en));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + (uint32_t)L::bar;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
    // every CTA of the cluster sends this CTA's en_mine outputs and G (m, l) pairs
    mbar_arrive_expect_tx(bar, (uint32_t)(CS * en_mine * 4 + CS * G * 8));
  }
  cluster_arrive_release();   // the matching wait comes before the first push
  [[maybe_unused]] const uint32_t sbar0 =
      kBulk ? sbase + (uint32_t)(BLay<D>::sbar + warp * kStagesB * 8) : 0u;
  if constexpr (kBulk) {
    if (lane == 0) {
      for (int st = 0; st < kStagesB; ++st) mbar_init(sbar0 + 8 * st, 1);
      mbar_fence_init();
    }
    __syncwarp();
  }

  // an out-of-range head_map entry reads as an empty list (output 0, lse -inf)
  const int hm_raw = a.one_list ? 0 : (a.head_map ? a.head_map[h] : h);
  const bool hm_ok = hm_raw >= 0 && hm_raw < a.n_lists;
  const int hm = hm_ok ? hm_raw : 0;
  const int list_full = a.idx ? topk_count(a.N, a.num, a.den) : a.N;   // list stride
  // a varlen row attends over its own first ceil(frac N_b) entries (dense: N_b keys)
  const int n_b = a.kv_lens ? min(a.N, a.kv_lens[b]) : a.N;
  const int list_len = hm_ok ? (a.idx ? topk_count(n_b, a.num, a.den) : n_b) : 0;
  const int32_t* list = a.idx ? a.idx + (size_t)(b * a.n_lists + hm) * list_full : nullptr;
  const int c0 = min(list_len, rank * per);
  const int c1 = min(list_len, c0 + per);
  const int n_slices = (c1 - c0 + 15) / 16;
  int* idx_s = reinterpret_cast<int*>(smem + L::idx);
  const bool staged = list != nullptr && (c1 - c0) <= L::IDXN;
  const size_t slab = (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv);
  // contiguous cache: row key of the slab; paged cache: row key % P of page
  // page_table[b][key / P], pages [num_pages, Hkv, P, D]
  const int kvh = (int)(slab - (size_t)b * a.Hkv);
  const __nv_bfloat16* kb = kPaged ? a.k + (size_t)kvh * a.page_size * D : a.k + slab * a.N * D;
  const __nv_bfloat16* vb = kPaged ? a.v + (size_t)kvh * a.page_size * D : a.v + slab * a.N * D;
  [[maybe_unused]] const int32_t* ptab = kPaged ? a.page_table + (size_t)b * a.max_pages : nullptr;
  auto row_off = [&](int key) -> size_t {
    if constexpr (kPaged) {
      const int pg = __ldg(ptab + (key >> a.page_shift));
      return ((size_t)pg * a.Hkv * a.page_size + (key & (a.page_size - 1))) * D;
    } else {
      return (size_t)key * D;
    }
  };

  if (staged)
    for (int i = threadIdx.x; i < c1 - c0; i += kThreads) idx_s[i] = __ldg(list + c0 + i);
  __syncthreads();

  auto key_of = [&](int rel) -> int {
    return list ? (staged ? idx_s[rel] : __ldg(list + c0 + rel)) : c0 + rel;
  };
  const uint32_t wbase = sbase + (uint32_t)(L::slabs + warp * L::WARPB);
  const uint32_t kslot = wbase + 2 * L::SLAB;
  // 16 rows of slice s (K or V) into a slab; rows past the list zero-filled.
  // V chunks are swizzled by row & 7 (ldmatrix.trans), K chunks by
  // (row & 1) * 4 (the permuted 16-byte reads of two rows per quarter warp).
  auto issue_rows = [&](int s, uint32_t dst, const __nv_bfloat16* base, bool is_k) {
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {   // 16 rows x CH chunks over 32 lanes
      const int e = lane + 32 * i;
      const int r = e / CH, ch = e - r * CH;
      const int rel = s * 16 + r;
      const bool have = c0 + rel < c1;
      const int key = have ? key_of(rel) : 0;
      const int pch = is_k ? (ch ^ ((r & 1) << 2)) : (ch ^ (r & 7));
      cp_async_16(dst + r * L::ROWB + pch * 16, base + row_off(key) + ch * 8, have ? 16 : 0);
    }
  };
  // K rows g and 8+g of slice s into registers (zero past the list end)
  uint4 kr[2][KS];
  auto load_k = [&](int s) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int rel = s * 16 + t * 8 + g;
      const bool have = c0 + rel < c1;
      const __nv_bfloat16* row = kb + row_off(have ? key_of(rel) : 0) + 8 * c;
#pragma unroll
      for (int q = 0; q < KS; ++q) kr[t][q] = have ? ldg_nc_v4(row + 32 * q) : make_uint4(0, 0, 0, 0);
    }
  };

  // per lane: heads 2c and 2c+1 (running max in log2 units, partial sums
  // over this lane's keys) and O^T for dims 16i + g (+8) of those heads
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float oacc[D / 16][4];
#pragma unroll
  for (int i = 0; i < D / 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  const float scale2 = kLog2e * rsqrtf((float)D);
  const char* qrow = smem + L::qs + (size_t)(g * D + 8 * c) * 2;

  // bulk mode: this warp's slices warp, warp + kWarps, ..., the it-th in
  // stage it % kStagesB, rows past the list repeating its last key (finite
  // data, masked out).  The two tensors take different copy engines, which
  // each sustain only so many row-sized requests per SM: K rows by one bulk
  // copy each (lanes 0-15, completing on the stage's mbarrier), V rows by
  // 16-byte cp.async (every lane, one commit group per stage).
  const int n_my = warp < n_slices ? (n_slices - warp + kWarps - 1) / kWarps : 0;
  // the tile form: stages 1024-byte aligned (the swizzle repeats every 8
  // rows of 128 bytes), inside the stage region the index staging leaves free
  [[maybe_unused]] const uint32_t dbase =
      ((sbase + 1023u) & ~1023u) + (uint32_t)(warp * kStagesB * kDenseStage<D>);
  [[maybe_unused]] const int dslab = (int)slab;
  [[maybe_unused]] auto issue_bulk = [&](int it) {
    using B = BLay<D>;
    const int sl = warp + kWarps * it;
    const int st = it % kStagesB;
    const uint32_t sb = sbar0 + 8 * st;
    if constexpr (kDense) {
      if (lane == 0) {
        const uint32_t kd = dbase + (uint32_t)(st * kDenseStage<D>), vd = kd + kDenseStage<D> / 2;
        const int row = c0 + sl * 16;   // rows past the list are masked, past the slab read zeros
        mbar_arrive_expect_tx(sb, (uint32_t)(2 * 16 * D * 2));
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          tc::tma_load_3d(kd + (uint32_t)(bx * 2048), &mk, bx * 64, row, dslab, sb);
          tc::tma_load_3d(vd + (uint32_t)(bx * 2048), &mv, bx * 64, row, dslab, sb);
        }
      }
      return;
    }
    const uint32_t kdst = wbase + (uint32_t)(st * B::STAGE);
    if (lane == 0) mbar_arrive_expect_tx(sb, (uint32_t)(16 * B::ROWB));
    __syncwarp();
    const unsigned long long off = row_off(key_of(min(sl * 16 + (lane & 15), c1 - c0 - 1)));
    if (lane < 16) bulk_g2s(kdst + lane * B::PITCH, kb + off, (uint32_t)B::ROWB, sb);
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {   // 16 rows x CH chunks over 32 lanes
      const int e = lane + 32 * i;
      const int r = e / CH, ch = e - r * CH;
      const unsigned long long ro = __shfl_sync(0xffffffffu, off, r);
      cp_async_16(kdst + (uint32_t)(B::TB + r * B::PITCH + ch * 16), vb + ro + ch * 8, 16);
    }
  };

  if constexpr (kBulk) {
    for (int j = 0; j < kStagesB; ++j) {
      if (j < n_my) issue_bulk(j);
      cp_async_commit();   // one group per stage, empty past the warp's slices
    }
  } else {
    // prologue: this warp's first two slices
    if (warp < n_slices) issue_rows(warp, wbase, vb, false);
    if (warp + kWarps < n_slices) {
      issue_rows(warp + kWarps, wbase + L::SLAB, vb, false);
      issue_rows(warp + kWarps, kslot, kb, true);
    }
    cp_async_commit();
    if (warp < n_slices) load_k(warp);
  }
  if (early) {
    pdl_wait();
    pdl_launch_dependents();
  }
  // the G query rows of this kv head (rows G..7 zero)
  for (int i = threadIdx.x; i < 8 * CH; i += kThreads) {
    const int r = i / CH, ch = i - r * CH;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < G) val = *reinterpret_cast<const uint4*>(a.q + (size_t)(b * a.Hq + h * G + r) * D + ch * 8);
    *reinterpret_cast<uint4*>(smem + L::qs + (r * D + ch * 8) * 2) = val;
  }
  __syncthreads();

  // One slice, both products transposed so that the 16 keys (and then the
  // head dims) fill the MMA rows and the <= 8 query heads its columns:
  // S^T = K q^T (A = K rows, B = q^T), then O^T += V^T P^T (A = V^T by
  // ldmatrix.trans, B = P^T moved from accumulator to operand layout by
  // movmatrix).  K fragments come from registers (even iterations) or the
  // K slot (odd iterations).
  auto step = [&](int s, int slot, auto from_slot) {
    constexpr bool kSlot = decltype(from_slot)::value;
    // k-step 2q+t takes dims 32q + 8c + 4t + {0,1} (logical k 2c, 2c+1) and
    // + {2,3} (logical k 2c+8, 2c+9) of the key rows and the query rows
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < KS; ++q) {
      const uint2 qlo = *reinterpret_cast<const uint2*>(qrow + 64 * q);       // dims 32q+8c+0..3
      const uint2 qhi = *reinterpret_cast<const uint2*>(qrow + 64 * q + 8);   // dims 32q+8c+4..7
      uint4 k0, k1;
      if constexpr (kSlot) {
        const int pch = (4 * q + c) ^ ((g & 1) << 2);   // rows g and 8 + g share parity
        k0 = lds_v4(kslot + g * L::ROWB + pch * 16);
        k1 = lds_v4(kslot + (8 + g) * L::ROWB + pch * 16);
      } else {
        k0 = kr[0][q];
        k1 = kr[1][q];
      }
      const uint32_t a0[4] = {k0.x, k1.x, k0.y, k1.y};
      const uint32_t a1[4] = {k0.z, k1.z, k0.w, k1.w};
      mma_bf16_16816(q & 1 ? sb : sa, a0, qlo.x, qlo.y);
      mma_bf16_16816(q & 1 ? sb : sa, a1, qhi.x, qhi.y);
    }
    // sv: (key g, head 2c), (key g, head 2c+1), (key g+8, head 2c), (key g+8, head 2c+1)
    const int kbase = c0 + s * 16;
    const bool v_lo = kbase + g < c1, v_hi = kbase + 8 + g < c1;
    float sv[4];
    sv[0] = v_lo ? (sa[0] + sb[0]) * scale2 : -INFINITY;
    sv[1] = v_lo ? (sa[1] + sb[1]) * scale2 : -INFINITY;
    sv[2] = v_hi ? (sa[2] + sb[2]) * scale2 : -INFINITY;
    sv[3] = v_hi ? (sa[3] + sb[3]) * scale2 : -INFINITY;
    float mx0 = fmaxf(sv[0], sv[2]), mx1 = fmaxf(sv[1], sv[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    // key s*16 is always in the list, so the slice maxima are finite
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float al0 = scale_from(m_run[0], mn0), al1 = scale_from(m_run[1], mn1);
    const float p0 = exp2f(sv[0] - mn0), p1 = exp2f(sv[1] - mn1);
    const float p2 = exp2f(sv[2] - mn0), p3 = exp2f(sv[3] - mn1);
    l_run[0] = l_run[0] * al0 + (p0 + p2);
    l_run[1] = l_run[1] * al1 + (p1 + p3);
    m_run[0] = mn0;
    m_run[1] = mn1;
    // P^T rows (keys) x columns (heads) -> B fragments (k = keys, n = heads)
    const uint32_t b0 = movmatrix_trans(pack_bf16(p0, p1));   // keys 0..7
    const uint32_t b1 = movmatrix_trans(pack_bf16(p2, p3));   // keys 8..15
    const uint32_t vs = wbase + slot * L::SLAB;
    const int vrow = ((lane >> 4) << 3) + (lane & 7);         // key of this lane's ldmatrix row
    const int vch = (lane >> 3) & 1;                           // dims +0 / +8 of the tile
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      uint32_t r4[4];
      ldmatrix_x4_trans(r4, vs + vrow * L::ROWB + (((2 * i + vch) ^ (lane & 7)) * 16));
      float t[4] = {oacc[i][0] * al0, oacc[i][1] * al1, oacc[i][2] * al0, oacc[i][3] * al1};
      mma_bf16_16816(t, r4, b0, b1);
      oacc[i][0] = t[0];
      oacc[i][1] = t[1];
      oacc[i][2] = t[2];
      oacc[i][3] = t[3];
    }
  };

  // Both of a warp's slices as one 32-key block: four independent QK^T
  // accumulator chains, one online-softmax update, then both PV products, so
  // the two slices' latency chains overlap.
  auto step2 = [&](int s0, int s1) {
    float sa0[4] = {0.f, 0.f, 0.f, 0.f}, sb0[4] = {0.f, 0.f, 0.f, 0.f};
    float sa1[4] = {0.f, 0.f, 0.f, 0.f}, sb1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < KS; ++q) {
      const uint2 qlo = *reinterpret_cast<const uint2*>(qrow + 64 * q);
      const uint2 qhi = *reinterpret_cast<const uint2*>(qrow + 64 * q + 8);
      const int pch = (4 * q + c) ^ ((g & 1) << 2);
      const uint4 m0 = lds_v4(kslot + g * L::ROWB + pch * 16);
      const uint4 m1 = lds_v4(kslot + (8 + g) * L::ROWB + pch * 16);
      const uint4 k0 = kr[0][q], k1 = kr[1][q];
      const uint32_t a0[4] = {k0.x, k1.x, k0.y, k1.y}, a1[4] = {k0.z, k1.z, k0.w, k1.w};
      const uint32_t d0[4] = {m0.x, m1.x, m0.y, m1.y}, d1[4] = {m0.z, m1.z, m0.w, m1.w};
      mma_bf16_16816(q & 1 ? sb0 : sa0, a0, qlo.x, qlo.y);
      mma_bf16_16816(q & 1 ? sb1 : sa1, d0, qlo.x, qlo.y);
      mma_bf16_16816(q & 1 ? sb0 : sa0, a1, qhi.x, qhi.y);
      mma_bf16_16816(q & 1 ? sb1 : sa1, d1, qhi.x, qhi.y);
    }
    const int kb0 = c0 + s0 * 16, kb1 = c0 + s1 * 16;
    const bool v0l = kb0 + g < c1, v0h = kb0 + 8 + g < c1, v1l = kb1 + g < c1, v1h = kb1 + 8 + g < c1;
    float sv[8];
    sv[0] = v0l ? (sa0[0] + sb0[0]) * scale2 : -INFINITY;
    sv[1] = v0l ? (sa0[1] + sb0[1]) * scale2 : -INFINITY;
    sv[2] = v0h ? (sa0[2] + sb0[2]) * scale2 : -INFINITY;
    sv[3] = v0h ? (sa0[3] + sb0[3]) * scale2 : -INFINITY;
    sv[4] = v1l ? (sa1[0] + sb1[0]) * scale2 : -INFINITY;
    sv[5] = v1l ? (sa1[1] + sb1[1]) * scale2 : -INFINITY;
    sv[6] = v1h ? (sa1[2] + sb1[2]) * scale2 : -INFINITY;
    sv[7] = v1h ? (sa1[3] + sb1[3]) * scale2 : -INFINITY;
    float mx0 = fmaxf(fmaxf(sv[0], sv[2]), fmaxf(sv[4], sv[6]));
    float mx1 = fmaxf(fmaxf(sv[1], sv[3]), fmaxf(sv[5], sv[7]));
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float al0 = scale_from(m_run[0], mn0), al1 = scale_from(m_run[1], mn1);
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = exp2f(sv[i] - (i & 1 ? mn1 : mn0));
    l_run[0] = l_run[0] * al0 + ((p[0] + p[2]) + (p[4] + p[6]));
    l_run[1] = l_run[1] * al1 + ((p[1] + p[3]) + (p[5] + p[7]));
    m_run[0] = mn0;
    m_run[1] = mn1;
    const uint32_t b00 = movmatrix_trans(pack_bf16(p[0], p[1])), b01 = movmatrix_trans(pack_bf16(p[2], p[3]));
    const uint32_t b10 = movmatrix_trans(pack_bf16(p[4], p[5])), b11 = movmatrix_trans(pack_bf16(p[6], p[7]));
    const int vrow = ((lane >> 4) << 3) + (lane & 7);
    const int vch = (lane >> 3) & 1;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      uint32_t r0[4], r1[4];
      const uint32_t off = vrow * L::ROWB + (((2 * i + vch) ^ (lane & 7)) * 16);
      ldmatrix_x4_trans(r0, wbase + off);
      ldmatrix_x4_trans(r1, wbase + L::SLAB + off);
      float t[4] = {oacc[i][0] * al0, oacc[i][1] * al1, oacc[i][2] * al0, oacc[i][3] * al1};
      mma_bf16_16816(t, r0, b00, b01);
      mma_bf16_16816(t, r1, b10, b11);
      oacc[i][0] = t[0];
      oacc[i][1] = t[1];
      oacc[i][2] = t[2];
      oacc[i][3] = t[3];
    }
  };

  // bulk mode: one slice from stage st (K reads in the pitch-padded chunk
  // order above; the query rows read with the same chunk order)
  [[maybe_unused]] auto step_bulk = [&](int sl, int st) {
    using B = BLay<D>;
    const uint32_t kst = kDense ? dbase + (uint32_t)(st * kDenseStage<D>) : wbase + (uint32_t)(st * B::STAGE);
    const uint32_t vst = kDense ? kst + kDenseStage<D> / 2 : kst + (uint32_t)B::TB;
    // 16-byte chunk ch of row r: pitch-padded rows, or the tile form's
    // swizzled 64-column tiles
    auto chunk_at = [&](uint32_t base, int r, int ch) -> uint32_t {
      if constexpr (kDense)
        return base + (uint32_t)((ch >> 3) * 2048 + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
      else
        return base + (uint32_t)(r * B::PITCH + ch * 16);
    };
    const char* qg = smem + L::qs + (size_t)(g * D) * 2;
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < KS; ++q) {
      const int ch = 8 * (q >> 1) + 2 * c + (q & 1);
      const uint2 qlo = *reinterpret_cast<const uint2*>(qg + ch * 16);
      const uint2 qhi = *reinterpret_cast<const uint2*>(qg + ch * 16 + 8);
      const uint4 k0 = lds_v4(chunk_at(kst, g, ch));
      const uint4 k1 = lds_v4(chunk_at(kst, 8 + g, ch));
      const uint32_t a0[4] = {k0.x, k1.x, k0.y, k1.y};
      const uint32_t a1[4] = {k0.z, k1.z, k0.w, k1.w};
      mma_bf16_16816(q & 1 ? sb : sa, a0, qlo.x, qlo.y);
      mma_bf16_16816(q & 1 ? sb : sa, a1, qhi.x, qhi.y);
    }
    const int kbase = c0 + sl * 16;
    const bool v_lo = kbase + g < c1, v_hi = kbase + 8 + g < c1;
    float sv[4];
    sv[0] = v_lo ? (sa[0] + sb[0]) * scale2 : -INFINITY;
    sv[1] = v_lo ? (sa[1] + sb[1]) * scale2 : -INFINITY;
    sv[2] = v_hi ? (sa[2] + sb[2]) * scale2 : -INFINITY;
    sv[3] = v_hi ? (sa[3] + sb[3]) * scale2 : -INFINITY;
    float mx0 = fmaxf(sv[0], sv[2]), mx1 = fmaxf(sv[1], sv[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float al0 = scale_from(m_run[0], mn0), al1 = scale_from(m_run[1], mn1);
    const float p0 = exp2f(sv[0] - mn0), p1 = exp2f(sv[1] - mn1);
    const float p2 = exp2f(sv[2] - mn0), p3 = exp2f(sv[3] - mn1);
    l_run[0] = l_run[0] * al0 + (p0 + p2);
    l_run[1] = l_run[1] * al1 + (p1 + p3);
    m_run[0] = mn0;
    m_run[1] = mn1;
    const uint32_t b0 = movmatrix_trans(pack_bf16(p0, p1));
    const uint32_t b1 = movmatrix_trans(pack_bf16(p2, p3));
    const int vrow = ((lane >> 4) << 3) + (lane & 7);
    const int vch = (lane >> 3) & 1;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      uint32_t r4[4];
      ldmatrix_x4_trans(r4, chunk_at(vst, vrow, 2 * i + vch));
      float t[4] = {oacc[i][0] * al0, oacc[i][1] * al1, oacc[i][2] * al0, oacc[i][3] * al1};
      mma_bf16_16816(t, r4, b0, b1);
      oacc[i][0] = t[0];
      oacc[i][1] = t[1];
      oacc[i][2] = t[2];
      oacc[i][3] = t[3];
    }
  };

  if constexpr (kBulk) {
    int it = 0;
    bool failed = false;
    for (; it < n_my; ++it) {
      const int st = it % kStagesB;
      // warp-uniform verdict, so that no lane reaches a warp-wide step alone
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(sbar0 + 8 * st, (uint32_t)((it / kStagesB) & 1)))) {
        if (lane == 0) raise_error(a.err, kErrGather);
        failed = true;
        break;
      }
      cp_async_wait<kStagesB - 1>();   // this lane's V chunks of stage st
      __syncwarp();                    // ... and every other lane's
      step_bulk(warp + kWarps * it, st);
      __syncwarp();   // every lane is done with stage st
      if (it + kStagesB < n_my) issue_bulk(it + kStagesB);
      cp_async_commit();
    }
    // after a wait gave up: let the copies still in flight land (bounded)
    // before the stages become the merge's scratch
    if (failed)
      for (int j = it + 1; j < n_my && j < it + kStagesB; ++j)
        mbar_wait_bounded(sbar0 + 8 * (j % kStagesB), (uint32_t)((j / kStagesB) & 1));
  } else {
    cp_async_wait<0>();
    __syncwarp();
    if (warp + kWarps < n_slices) step2(warp, warp + kWarps);
    else if (warp < n_slices) step(warp, 0, std::false_type{});
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], o);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], o);
  }

  // ---------------- merge the warps into this CTA's partial
  __syncthreads();   // every warp is done with its slabs
  float* red_o = reinterpret_cast<float*>(smem + L::red_o);
  float2* red_ml = reinterpret_cast<float2*>(smem + L::red_ml);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int hh = 2 * c + j;
    if (hh < G) {
      float* ro = red_o + (warp * 8 + hh) * L::RO + g;
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        ro[16 * i] = oacc[i][j];
        ro[16 * i + 8] = oacc[i][2 + j];
      }
      if (g == 0) red_ml[warp * 8 + hh] = make_float2(m_run[j], l_run[j]);
    }
  }
  __syncthreads();
  // softmax-merge weights of the warps' partials, one warp per head
  float* wf = reinterpret_cast<float*>(smem + L::wf);
  float2* pml = reinterpret_cast<float2*>(smem + L::pml);
  if (warp < G) merge_weights(kWarps, red_ml + warp, wf + warp, pml + warp, lane);
  __syncthreads();
  cluster_wait_acquire();   // every peer's mbarrier is initialised
  const uint32_t recv_o = sbase + (uint32_t)L::recv_o;
  const uint32_t recv_ml = sbase + (uint32_t)L::recv_ml;
  // four consecutive output elements per thread, pushed to their owner e / en
  if (threadIdx.x * 4 < E) {
    const int e = threadIdx.x * 4;
    const int gg = e / D, dd = e - gg * D;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = wf[w * 8 + gg];
      const float4 v = *reinterpret_cast<const float4*>(red_o + (w * 8 + gg) * L::RO + dd);
      acc.x += f * v.x;
      acc.y += f * v.y;
      acc.z += f * v.z;
      acc.w += f * v.w;
    }
    const int q = e / en;
    const uint32_t off = (uint32_t)(rank * en + (e - q * en)) * 4;
    st_async_v4(mapa(recv_o + off, q), acc, mapa(bar, q));
  }
  // this CTA's (max, sum) of every head, to every CTA of the cluster
  if (threadIdx.x < CS * G) {
    const int r = threadIdx.x / G, gg = threadIdx.x - r * G;
    st_async_v2(mapa(recv_ml + (uint32_t)(rank * 8 + gg) * 8, r), pml[gg], mapa(bar, r));
  }

  // ---------------- merge this CTA's element slice once every peer's bytes landed
  if (!mbar_wait_cluster_bounded(bar, 0)) raise_error(a.err, kErrMergeTimeout);
  float* wts = reinterpret_cast<float*>(smem + L::wts);
  float2* head = reinterpret_cast<float2*>(smem + L::head);
  const float2* rml = reinterpret_cast<const float2*>(smem + L::recv_ml);
  if (warp < G) merge_weights(CS, rml + warp, wts + warp, head + warp, lane);
  __syncthreads();
  if ((int)threadIdx.x < en_mine) {
    const float* ro = reinterpret_cast<const float*>(smem + L::recv_o);
    const int e = rank * en + threadIdx.x;
    const int gg = e / D, dd = e - gg * D;
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxCS; ++r)
      if (r < CS) acc += wts[r * 8 + gg] * ro[r * en + threadIdx.x];
    const float2 ml = head[gg];
    const size_t orow = (size_t)(b * a.Hq + h * G + gg);
    a.o[orow * D + dd] = __float2bfloat16(ml.y > 0.f ? acc / ml.y : 0.f);
    if (dd == 0 && a.lse) a.lse[orow] = ml.y > 0.f ? (ml.x + log2f(ml.y)) * (float)kLn2 : -INFINITY;
  }
}

template <int D, int kMode>
cudaLaunchConfig_t make_cfg(int cs, int bh, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, bh, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = LayOf<D, kMode>::total;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Cluster sizes of the sparse decode, largest first; one cluster per
// (batch, list) problem.  Short lists (mode 0): the largest size at which a
// launch and its successor are resident together, else the largest with one
// wave (choose_overlap_cluster_size), among the sizes that keep every warp
// at two slices or fewer; on a 148-SM part 14 clusters of 16 fit at two
// CTAs per SM, so the Llama-shaped layer's 8 problems take 13 CTAs each.  Owners of the output elements
// get equal shares rounded to 4, so a size need not divide G d.  Long lists
// (the bulk mode, one CTA per SM): the fewest waves, pairs included, so 64
// problems still fit one wave.
constexpr int kDecSizes0[] = {16, 15, 14, 13, 12, 10, 8, 4};
constexpr int kNumDecSizes0 = 8;
constexpr int kDecSizesB[] = {16, 8, 4, 2};
constexpr int kNumDecSizesB = 4;
constexpr int kMaxDecSizes = 8;

// clusters of sizes[i] the device runs at once (cached per device)
template <int D, int kMode>
const int* decode_active(const int* sizes, int n) {
  static int cached[64][kMaxDecSizes + 1] = {{0}};   // [0]: 1 once filled
  static const int none[kMaxDecSizes] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return none;
  if (!cached[dev][0]) {
    for (int i = 0; i < n; ++i) {
      int m = 0;
      if (ensure_func_attrs(reinterpret_cast<const void*>(decode_attn_kernel<D, kMode>), LayOf<D, kMode>::total,
                            sizes[i] > 8) == cudaSuccess) {
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = make_cfg<D, kMode>(sizes[i], 1, nullptr, attr);
        if (cudaOccupancyMaxActiveClusters(&m, decode_attn_kernel<D, kMode>, &cfg) != cudaSuccess) m = 0;
      }
      cached[dev][1 + i] = m;
    }
    cudaGetLastError();
    cached[dev][0] = 1;
  }
  return &cached[dev][1];
}

template <int D, int kMode>
cudaError_t launch_cs(const AttnArgs& a, int cs, int per, cudaStream_t stream) {
  const size_t smem = LayOf<D, kMode>::total;
  const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(decode_attn_kernel<D, kMode>), smem, cs > 8);
  if (e != cudaSuccess) return e;
  // K and V as [B Hkv][N][D] in tiles of 16 rows x 64 columns (the tile
  // form reads them; the other forms get the maps unused)
  CUtensorMap mk{}, mv{};
  if constexpr ((kMode & kDenseBit) != 0) {
    if (!tc::make_map_3d(&mk, a.k, (uint64_t)D, (uint64_t)a.N, (uint64_t)a.B * a.Hkv, 16) ||
        !tc::make_map_3d(&mv, a.v, (uint64_t)D, (uint64_t)a.N, (uint64_t)a.B * a.Hkv, 16))
      return cudaErrorInvalidValue;
  }
  return launch_ex(decode_attn_kernel<D, kMode>, dim3(cs, a.B * a.Hp), dim3(kThreads), smem, stream,
                   (a.flags & 1) != 0, cs, a, per, mk, mv);
}

int share_of(int list_len, int cs) {
  int per = (list_len + cs - 1) / cs;
  per = (per + 15) / 16 * 16;
  return per < 16 ? 16 : per;
}

template <int D, int kPaged>
cudaError_t launch(const AttnArgs& a, cudaStream_t stream) {
  const long long problems = (long long)a.B * a.Hp;
  const int list_len = a.idx ? topk_count(a.N, a.num, a.den) : a.N;
  // few keys per CTA: every warp's slices issued up front, two CTAs per SM
  {
    const int* act = decode_active<D, 0 | kPaged>(kDecSizes0, kNumDecSizes0);
    bool fits[kNumDecSizes0];
    for (int i = 0; i < kNumDecSizes0; ++i) fits[i] = share_of(list_len, kDecSizes0[i]) <= 2 * 16 * kWarps;
    const int cs = choose_overlap_cluster_size(problems, kDecSizes0, act, fits, kNumDecSizes0);
    if (cs > 0) return launch_cs<D, 0 | kPaged>(a, cs, share_of(list_len, cs), stream);
  }
  // many keys per CTA: bulk-copied stages, one CTA per SM; the dense form
  // of a contiguous cache as whole tiles
  const int* act = decode_active<D, 2 | kPaged>(kDecSizesB, kNumDecSizesB);
  const bool fits[kNumDecSizesB] = {true, true, true, true};
  int csb = choose_cluster_size(problems, kDecSizesB, act, fits, kNumDecSizesB);
  if (csb <= 0) csb = 8;
  if constexpr (kPaged == 0) {
    if (!a.idx) return launch_cs<D, 2 | kDenseBit>(a, csb, share_of(list_len, csb), stream);
  }
  return launch_cs<D, 2 | kPaged>(a, csb, share_of(list_len, csb), stream);
}

}  // namespace

cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t stream) {
  if (a.page_table) return a.D == 128 ? launch<128, kPagedBit>(a, stream) : launch<64, kPagedBit>(a, stream);
  return a.D == 128 ? launch<128, 0>(a, stream) : launch<64, 0>(a, stream);
}

}  // namespace kascade
