// Gather-sparse prefill attention of the Kascade anchor and reuse layers
// (README, Abstract: reuse layers attend only over the anchor's Top-k
// indices; tile-level operations in prefill).  With an implicit key list
// [0, e_t) (causal) or [0, N) the same kernel is the dense reference.
//
// One CTA per (query tile, row block of 128 = 4 heads x 32 queries, batch x
// kv head), longest tiles first.  The 8 warps share a 3-stage pipeline of 64
// gathered keys: rows of K and V are copied with 16-byte cp.async into
// XOR-swizzled shared memory (conflict-free for ldmatrix) and fed to
// warp-level bf16 MMAs with an fp32 online softmax and the causal mask
// j <= i applied by original key index.
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

// ----------------------------------------------------------------- prefill

constexpr int kPreWarps = 8;
constexpr int kPreStages = 3;
constexpr int kPreKeys = 64;

template <int D>
__global__ void __launch_bounds__(kPreWarps * 32)
    prefill_attn_kernel(const AttnArgs a, int row_blocks) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int CH = D / 8;
  constexpr int MAT_BYTES = kPreKeys * D * 2;   // one stage of K (or V)
  constexpr int STAGE_BYTES = 2 * MAT_BYTES;
  extern __shared__ __align__(128) char smem[];
  int* key_s = reinterpret_cast<int*>(smem + kPreStages * STAGE_BYTES);   // [stages][64]

  const int T = (a.N + a.tile - 1) / a.tile;
  const int t0 = a.q0 / a.tile;   // first query tile of the call (rolling chunks)
  const int t = T - 1 - (int)(blockIdx.x / row_blocks);
  const int rb = blockIdx.x % row_blocks;
  const int bh = blockIdx.y;
  const int b = bh / a.Hp, h = bh - b * a.Hp;   // problem h of batch row b
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = a.G;
  const int hm_raw = a.one_list ? 0 : (a.head_map ? a.head_map[h] : h);
  const bool hm_ok = hm_raw >= 0 && hm_raw < a.n_lists;
  const int hm = hm_ok ? hm_raw : 0;
  const int i0 = t * a.tile;
  const int e_t = min(i0 + a.tile, a.N);
  const int rows_t = e_t - i0;

  int list_len;
  const int32_t* list = nullptr;
  if (a.idx) {
    const int64_t row_len = chunk_row_len(a.N, t0, a.tile, a.num, a.den);
    list = a.idx + (size_t)(b * a.n_lists + hm) * row_len + chunk_list_offset(t, t0, a.tile, a.num, a.den);
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
    qrow_off[hf] = qrow_ok[hf] ? ((size_t)(b * a.Hq + h * G + gi) * a.Lq + (i0 - a.q0) + il) * D : 0;
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

  const size_t slab = (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv);
  const __nv_bfloat16* kb = a.k + slab * a.N * D;
  const __nv_bfloat16* vb = a.v + slab * a.N * D;
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
size_t prefill_smem() {
  return (size_t)kPreStages * 2 * kPreKeys * D * 2 + (size_t)kPreStages * kPreKeys * 4;
}

}  // namespace

cudaError_t launch_prefill_attn(const AttnArgs& a, cudaStream_t stream) {
  const int T = (a.N + a.tile - 1) / a.tile - a.q0 / a.tile;   // the call's query tiles
  const int row_blocks = (a.G * a.tile + 127) / 128;
  dim3 grid(T * row_blocks, a.B * a.Hp);
  if (a.D == 128) {
    const size_t sm = prefill_smem<128>();
    const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(prefill_attn_kernel<128>), sm, false);
    if (e != cudaSuccess) return e;
    return launch_ex(prefill_attn_kernel<128>, grid, dim3(kPreWarps * 32), sm, stream, (a.flags & 1) != 0, 1, a,
                     row_blocks);
  } else {
    const size_t sm = prefill_smem<64>();
    const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(prefill_attn_kernel<64>), sm, false);
    if (e != cudaSuccess) return e;
    return launch_ex(prefill_attn_kernel<64>, grid, dim3(kPreWarps * 32), sm, stream, (a.flags & 1) != 0, 1, a,
                     row_blocks);
  }
  return cudaGetLastError();
}

}  // namespace kascade
