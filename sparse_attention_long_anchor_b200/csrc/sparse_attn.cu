// Gather-sparse attention of the Kascade anchor and reuse layers (README,
// Abstract: reuse layers attend only over the anchor's Top-k indices; the
// selection and its reuse are head-aware).  The same kernels with an
// implicit full key list are the dense reference attention.
//
// Rows of the selected keys are gathered with 16-byte cp.async copies into
// XOR-swizzled shared memory (a conflict-free layout for ldmatrix) and fed to
// warp-level bf16 MMAs with an online softmax in fp32:
//   decode:  one CTA per (split of the index list, batch x kv head); every
//            warp owns 16-key slices with its own 2-stage pipeline; the G
//            query heads are the rows of a 16-row MMA tile; per-CTA partial
//            (max, sum, output) go to the workspace and the last CTA of a
//            (batch, kv head) -- found with an atomic ticket, no waiting --
//            merges them.
//   prefill: one CTA per (query tile, row block of 128 = 4 heads x 32
//            queries, batch x kv head), longest tiles first; all 8 warps share
//            a 3-stage pipeline of 64 gathered keys; causal mask j <= i.
#include "common.cuh"
#include "kernels.h"

namespace kascade {

namespace {

// ----------------------------------------------------------------- helpers

// shared-memory byte offset of 16-byte chunk `ch` of row `r` (rows of D bf16)
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return (uint32_t)(r * (D * 2) + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ float safe_exp2_scale(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.0f : exp2f(m_old - m_new);
}

// ----------------------------------------------------------------- decode

constexpr int kDecWarps = 4;
constexpr int kDecStages = 2;

template <int D>
__global__ void __launch_bounds__(kDecWarps * 32)
    decode_attn_kernel(const AttnArgs a) {
  constexpr int CH = D / 8;                   // 16-byte chunks per row
  constexpr int SLICE_BYTES = 16 * D * 2;     // one 16-key slab of K (or V)
  constexpr int WARP_BYTES = kDecStages * 2 * SLICE_BYTES;
  extern __shared__ __align__(128) char smem[];

  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = a.G;
  // an out-of-range head_map entry reads as an empty list (output 0, lse -inf)
  const int hm_raw = a.head_map ? a.head_map[h] : h;
  const bool hm_ok = hm_raw >= 0 && hm_raw < a.Hkv;
  const int hm = hm_ok ? hm_raw : 0;
  const int list_full = a.idx ? topk_count(a.N, a.num, a.den) : a.N;
  const int list_len = hm_ok ? list_full : 0;
  const int32_t* list = a.idx ? a.idx + (size_t)(b * a.Hkv + hm) * list_full : nullptr;
  const int c0 = split * a.keys_per_split;
  const int c1 = min(list_len, c0 + a.keys_per_split);
  const __nv_bfloat16* kb = a.k + (size_t)bh * a.N * D;
  const __nv_bfloat16* vb = a.v + (size_t)bh * a.N * D;

  // Q as the A operand: row g = query head g of the group (rows >= G are 0)
  uint32_t qa[D / 16][2];
  {
    const __nv_bfloat16* qrow = a.q + (size_t)(b * a.Hq + h * G + (g < G ? g : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * c) : 0u;
      qa[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * c + 8) : 0u;
    }
  }

  char* wsm = smem + warp * WARP_BYTES;
  const uint32_t wsm_u = smem_u32(wsm);
  const int n_slices = (c1 - c0 + 15) / 16;
  const float scale2 = kLog2e * rsqrtf((float)D);

  // each lane copies half of one row of K and of V per slice
  auto issue = [&](int slice, int stage) {
    const int pos = c0 + slice * 16 + (lane >> 1);
    const bool ok = pos < c1;
    const int key = ok ? (list ? list[pos] : pos) : 0;
    const uint32_t kdst = wsm_u + stage * 2 * SLICE_BYTES;
    const uint32_t vdst = kdst + SLICE_BYTES;
    const int r = lane >> 1;
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
      const int ch = (lane & 1) * (CH / 2) + i;
      cp_async_16(kdst + swz<D>(r, ch), kb + (size_t)key * D + ch * 8, ok ? 16 : 0);
      cp_async_16(vdst + swz<D>(r, ch), vb + (size_t)key * D + ch * 8, ok ? 16 : 0);
    }
  };

  float m_run = -INFINITY, l_run = 0.f;
  float oacc[D / 8][4];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.f;

  // slices of this warp: warp, warp + W, ...
  int s_issue = warp;
#pragma unroll
  for (int st = 0; st < kDecStages - 1; ++st) {
    if (s_issue < n_slices) issue(s_issue, st);
    cp_async_commit();
    s_issue += kDecWarps;
  }
  int stage = 0;
  for (int s = warp; s < n_slices; s += kDecWarps) {
    {
      const int st_next = (stage + kDecStages - 1) % kDecStages;
      if (s_issue < n_slices) issue(s_issue, st_next);
      cp_async_commit();
      s_issue += kDecWarps;
    }
    cp_async_wait<kDecStages - 1>();
    __syncwarp();
    const uint32_t ks = wsm_u + stage * 2 * SLICE_BYTES;
    const uint32_t vs = ks + SLICE_BYTES;

    // S = Q K^T for 16 keys (two n-tiles of 8)
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int kk = 0; kk < D / 16; kk += 2) {
        uint32_t r4[4];
        const int row = nt * 8 + (lane & 7);
        const int ch = 2 * kk + (lane >> 3);
        ldmatrix_x4(r4, ks + swz<D>(row, ch));
        const uint32_t a0[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
        mma_bf16_16816(sacc[nt], a0, r4[0], r4[1]);
        const uint32_t a1[4] = {qa[kk + 1][0], 0u, qa[kk + 1][1], 0u};
        mma_bf16_16816(sacc[nt], a1, r4[2], r4[3]);
      }
    }
    // online softmax for row g (keys beyond c1 are masked)
    const int kbase = c0 + s * 16;
    float sv[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = kbase + nt * 8 + 2 * c + e;
        sv[nt * 2 + e] = key < c1 ? sacc[nt][e] * scale2 : -INFINITY;
      }
    }
    float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = safe_exp2_scale(m_run, m_new);
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = exp2f(sv[e] - m_new);
    l_run = l_run * alpha + (p[0] + p[1] + p[2] + p[3]);
    m_run = m_new;
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      oacc[nd][0] *= alpha;
      oacc[nd][1] *= alpha;
    }
    const uint32_t pa[4] = {pack_bf16(p[0], p[1]), 0u, pack_bf16(p[2], p[3]), 0u};
    // O += P V
#pragma unroll
    for (int nd = 0; nd < D / 8; nd += 2) {
      uint32_t r4[4];
      const int mi = lane >> 3;
      const int row = (mi & 1) * 8 + (lane & 7);
      const int ch = nd + (mi >> 1);
      ldmatrix_x4_trans(r4, vs + swz<D>(row, ch));
      mma_bf16_16816(oacc[nd], pa, r4[0], r4[1]);
      mma_bf16_16816(oacc[nd + 1], pa, r4[2], r4[3]);
    }
    __syncwarp();
    stage = (stage + 1) % kDecStages;
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

  // merge the warps of this CTA (deterministic order) in shared memory
  __syncthreads();
  float* red_o = reinterpret_cast<float*>(smem);                    // [W][8][D]
  float* red_ml = red_o + kDecWarps * 8 * D;                        // [W][8][2]
  if (g < G) {
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      red_o[(warp * 8 + g) * D + nd * 8 + 2 * c] = oacc[nd][0];
      red_o[(warp * 8 + g) * D + nd * 8 + 2 * c + 1] = oacc[nd][1];
    }
    if (c == 0) {
      red_ml[(warp * 8 + g) * 2] = m_run;
      red_ml[(warp * 8 + g) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  const int splits = a.splits;
  float* part_o = a.part_o + ((size_t)bh * splits + split) * G * D;
  float* part_ml = a.part_ml + ((size_t)bh * splits + split) * G * 2;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int gg = e / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, red_ml[(w * 8 + gg) * 2]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float f = safe_exp2_scale(red_ml[(w * 8 + gg) * 2], M);
      acc += f * red_o[(w * 8 + gg) * D + (e - gg * D)];
      lsum += f * red_ml[(w * 8 + gg) * 2 + 1];
    }
    part_o[e] = acc;
    if (e - gg * D == 0) {
      part_ml[gg * 2] = M;
      part_ml[gg * 2 + 1] = lsum;
    }
  }

  // ticket: the last CTA of this (batch, kv head) merges all splits
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = splits > 1 ? atomicAdd(a.counters + bh, 1) : 0;
    s_last = (prev == splits - 1);
    if (s_last && splits > 1) a.counters[bh] = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* all_o = a.part_o + (size_t)bh * splits * G * D;
  const float* all_ml = a.part_ml + (size_t)bh * splits * G * 2;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int gg = e / D, dd = e - gg * D;
    float M = -INFINITY;
    for (int sp = 0; sp < splits; ++sp) M = fmaxf(M, __ldcg(all_ml + (sp * G + gg) * 2));
    float acc = 0.f, lsum = 0.f;
    for (int sp = 0; sp < splits; ++sp) {
      const float f = safe_exp2_scale(__ldcg(all_ml + (sp * G + gg) * 2), M);
      acc += f * __ldcg(all_o + (size_t)(sp * G + gg) * D + dd);
      lsum += f * __ldcg(all_ml + (sp * G + gg) * 2 + 1);
    }
    const size_t orow = (size_t)(b * a.Hq + h * G + gg);
    a.o[orow * D + dd] = __float2bfloat16(lsum > 0.f ? acc / lsum : 0.f);
    if (dd == 0 && a.lse) a.lse[orow] = lsum > 0.f ? (M + log2f(lsum)) * (float)kLn2 : -INFINITY;
  }
}

// ----------------------------------------------------------------- prefill

constexpr int kPreWarps = 8;
constexpr int kPreStages = 3;
constexpr int kPreKeys = 64;

template <int D>
__global__ void __launch_bounds__(kPreWarps * 32)
    prefill_attn_kernel(const AttnArgs a, int row_blocks) {
  constexpr int CH = D / 8;
  constexpr int MAT_BYTES = kPreKeys * D * 2;   // one stage of K (or V)
  constexpr int STAGE_BYTES = 2 * MAT_BYTES;
  extern __shared__ __align__(128) char smem[];
  int* key_s = reinterpret_cast<int*>(smem + kPreStages * STAGE_BYTES);   // [stages][64]

  const int T = (a.N + a.tile - 1) / a.tile;
  const int t = T - 1 - (int)(blockIdx.x / row_blocks);
  const int rb = blockIdx.x % row_blocks;
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = a.G;
  const int hm_raw = a.head_map ? a.head_map[h] : h;
  const bool hm_ok = hm_raw >= 0 && hm_raw < a.Hkv;
  const int hm = hm_ok ? hm_raw : 0;
  const int i0 = t * a.tile;
  const int e_t = min(i0 + a.tile, a.N);
  const int rows_t = e_t - i0;

  int list_len;
  const int32_t* list = nullptr;
  if (a.idx) {
    const int T_last = T - 1;
    const int64_t row_len = tile_list_offset(T_last, a.tile, a.num, a.den) + topk_count(a.N, a.num, a.den);
    list = a.idx + (size_t)(b * a.Hkv + hm) * row_len + tile_list_offset(t, a.tile, a.num, a.den);
    list_len = hm_ok ? topk_count(e_t, a.num, a.den) : 0;
  } else {
    list_len = a.causal ? e_t : a.N;
  }
  const bool need_mask = a.idx != nullptr || a.causal;

  // this thread's two rows (g and g+8 of the warp's 16)
  int qrow_i[2];
  bool qrow_ok[2];
  size_t qrow_off[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int r = rb * 128 + warp * 16 + g + hf * 8;
    const int gi = r / a.tile, il = r - gi * a.tile;
    qrow_ok[hf] = gi < G && il < rows_t;
    qrow_i[hf] = i0 + il;
    qrow_off[hf] = qrow_ok[hf] ? ((size_t)(b * a.Hq + h * G + gi) * a.N + i0 + il) * D : 0;
  }
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const __nv_bfloat16* qr = a.q + qrow_off[hf];
      qa[kk][hf] = qrow_ok[hf] ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * c) : 0u;
      qa[kk][hf + 2] = qrow_ok[hf] ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * c + 8) : 0u;
    }
  }

  const __nv_bfloat16* kb = a.k + (size_t)bh * a.N * D;
  const __nv_bfloat16* vb = a.v + (size_t)bh * a.N * D;
  const uint32_t sm_u = smem_u32(smem);
  const int n_blocks = (list_len + kPreKeys - 1) / kPreKeys;
  const float scale2 = kLog2e * rsqrtf((float)D);

  // 256 threads: thread -> row (tid / 4), 4 chunks of K and 4 of V (D = 128)
  auto issue = [&](int blk, int stage) {
    const int r = threadIdx.x >> 2;
    const int pos = blk * kPreKeys + r;
    const bool ok = pos < list_len;
    const int key = ok ? (list ? list[pos] : pos) : 0;
    if ((threadIdx.x & 3) == 0) key_s[stage * kPreKeys + r] = ok ? key : 0x7fffffff;
    const uint32_t kdst = sm_u + stage * STAGE_BYTES;
    const uint32_t vdst = kdst + MAT_BYTES;
#pragma unroll
    for (int i = 0; i < CH / 4; ++i) {
      const int ch = (threadIdx.x & 3) * (CH / 4) + i;
      cp_async_16(kdst + swz<D>(r, ch), kb + (size_t)key * D + ch * 8, ok ? 16 : 0);
      cp_async_16(vdst + swz<D>(r, ch), vb + (size_t)key * D + ch * 8, ok ? 16 : 0);
    }
  };

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float oacc[D / 8][4];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.f;

#pragma unroll
  for (int st = 0; st < kPreStages - 1; ++st) {
    if (st < n_blocks) issue(st, st);
    cp_async_commit();
  }
  for (int blk = 0; blk < n_blocks; ++blk) {
    const int stage = blk % kPreStages;
    {
      const int nb = blk + kPreStages - 1;
      if (nb < n_blocks) issue(nb, nb % kPreStages);
      cp_async_commit();
    }
    cp_async_wait<kPreStages - 1>();
    __syncthreads();
    const uint32_t ks = sm_u + stage * STAGE_BYTES;
    const uint32_t vs = ks + MAT_BYTES;
    const int* keys = key_s + stage * kPreKeys;

    float sacc[kPreKeys / 8][4];
#pragma unroll
    for (int nt = 0; nt < kPreKeys / 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < kPreKeys / 8; ++nt) {
#pragma unroll
      for (int kk = 0; kk < D / 16; kk += 2) {
        uint32_t r4[4];
        ldmatrix_x4(r4, ks + swz<D>(nt * 8 + (lane & 7), 2 * kk + (lane >> 3)));
        mma_bf16_16816(sacc[nt], qa[kk], r4[0], r4[1]);
        mma_bf16_16816(sacc[nt], qa[kk + 1], r4[2], r4[3]);
      }
    }
    // scale, mask (tail keys and j > i), online softmax for rows g and g+8
    const int last_pos = min(list_len, (blk + 1) * kPreKeys) - 1;
    const bool blk_mask = need_mask && (keys[last_pos - blk * kPreKeys] > i0 || last_pos < (blk + 1) * kPreKeys - 1);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < kPreKeys / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float s = sacc[nt][e] * scale2;
        if (blk_mask || blk * kPreKeys + nt * 8 + 2 * c + (e & 1) >= list_len) {
          const int kl = nt * 8 + 2 * c + (e & 1);
          const int key = keys[kl];
          if (key > qrow_i[e >> 1]) s = -INFINITY;   // also catches padding (INT_MAX)
        }
        sacc[nt][e] = s;
        mx[e >> 1] = fmaxf(mx[e >> 1], s);
      }
    }
    float alpha[2], mnew[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 1));
      mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 2));
      mnew[hf] = fmaxf(m_run[hf], mx[hf]);
      alpha[hf] = safe_exp2_scale(m_run[hf], mnew[hf]);
      m_run[hf] = mnew[hf];
      if (mnew[hf] == -INFINITY) mnew[hf] = 0.f;   // nothing visible yet: p = 0
    }
    float lsum[2] = {0.f, 0.f};
    uint32_t pa[kPreKeys / 16][4];
#pragma unroll
    for (int nt = 0; nt < kPreKeys / 8; ++nt) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p[e] = exp2f(sacc[nt][e] - mnew[e >> 1]);
        lsum[e >> 1] += p[e];
      }
      // A fragment of P for k16 step nt/2: regs {row g lo, row g+8 lo, row g hi, row g+8 hi}
      pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p[0], p[1]);
      pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p[2], p[3]);
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) l_run[hf] = l_run[hf] * alpha[hf] + lsum[hf];
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      oacc[nd][0] *= alpha[0];
      oacc[nd][1] *= alpha[0];
      oacc[nd][2] *= alpha[1];
      oacc[nd][3] *= alpha[1];
    }
#pragma unroll
    for (int ks16 = 0; ks16 < kPreKeys / 16; ++ks16) {
#pragma unroll
      for (int nd = 0; nd < D / 8; nd += 2) {
        uint32_t r4[4];
        const int mi = lane >> 3;
        const int row = ks16 * 16 + (mi & 1) * 8 + (lane & 7);
        ldmatrix_x4_trans(r4, vs + swz<D>(row, nd + (mi >> 1)));
        mma_bf16_16816(oacc[nd], pa[ks16], r4[0], r4[1]);
        mma_bf16_16816(oacc[nd + 1], pa[ks16], r4[2], r4[3]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    l_run[hf] += __shfl_xor_sync(0xffffffffu, l_run[hf], 1);
    l_run[hf] += __shfl_xor_sync(0xffffffffu, l_run[hf], 2);
  }
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (!qrow_ok[hf]) continue;
    const float inv = l_run[hf] > 0.f ? 1.f / l_run[hf] : 0.f;
    __nv_bfloat16* orow = a.o + qrow_off[hf];
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd) {
      *reinterpret_cast<uint32_t*>(orow + nd * 8 + 2 * c) =
          pack_bf16(oacc[nd][hf * 2] * inv, oacc[nd][hf * 2 + 1] * inv);
    }
    if (a.lse && c == 0)
      a.lse[qrow_off[hf] / D] = l_run[hf] > 0.f ? (m_run[hf] + log2f(l_run[hf])) * (float)kLn2 : -INFINITY;
  }
}

template <int D>
size_t decode_smem() {
  const size_t pipe = (size_t)kDecWarps * kDecStages * 2 * 16 * D * 2;
  const size_t red = (size_t)kDecWarps * 8 * (D + 2) * 4;
  return pipe > red ? pipe : red;
}

template <int D>
size_t prefill_smem() {
  return (size_t)kPreStages * 2 * kPreKeys * D * 2 + (size_t)kPreStages * kPreKeys * 4;
}

}  // namespace

void decode_attn_plan(int B, int Hkv, int list_len, int num_sms, int* splits, int* keys_per_split) {
  // aim for about 3 CTAs per SM in total, slices of 16 keys per warp
  const int bh = B * Hkv;
  const int target_ctas = 3 * num_sms;
  int per = (list_len * 1LL * bh + target_ctas - 1) / target_ctas;
  const int unit = 16 * kDecWarps;
  per = ((per + unit - 1) / unit) * unit;
  if (per < unit) per = unit;
  *keys_per_split = per;
  *splits = (list_len + per - 1) / per;
}

cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t stream) {
  dim3 grid(a.splits, a.B * a.Hkv);
  if (a.D == 128) {
    const size_t sm = decode_smem<128>();
    cudaFuncSetAttribute(decode_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    decode_attn_kernel<128><<<grid, kDecWarps * 32, sm, stream>>>(a);
  } else {
    const size_t sm = decode_smem<64>();
    cudaFuncSetAttribute(decode_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    decode_attn_kernel<64><<<grid, kDecWarps * 32, sm, stream>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_prefill_attn(const AttnArgs& a, cudaStream_t stream) {
  const int T = (a.N + a.tile - 1) / a.tile;
  const int row_blocks = (a.G * a.tile + 127) / 128;
  dim3 grid(T * row_blocks, a.B * a.Hkv);
  if (a.D == 128) {
    const size_t sm = prefill_smem<128>();
    cudaFuncSetAttribute(prefill_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    prefill_attn_kernel<128><<<grid, kPreWarps * 32, sm, stream>>>(a, row_blocks);
  } else {
    const size_t sm = prefill_smem<64>();
    cudaFuncSetAttribute(prefill_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    prefill_attn_kernel<64><<<grid, kPreWarps * 32, sm, stream>>>(a, row_blocks);
  }
  return cudaGetLastError();
}

}  // namespace kascade
