// Anchor prefill scoring and pooling (Kascade README, Abstract and the
// post_softmax_pooled_prefill_topk strategy): for one (batch, kv head h,
// query tile t) the 32 queries of the tile in each of h's G query heads form
// the rows r; the candidates are the keys j < e_t.
//   pass 1: S = Q K^T / sqrt(d) with the causal mask j <= i; per row the max
//           m2_r and the sum l_r = sum_j exp2(s2_rj - m2_r) (base-2 domain,
//           fp32 terms, fp64 accumulation);
//   pass 2: S recomputed as K Q^T so that each MMA row is a key and each
//           lane holds whole key columns; the pooled score
//           P_j = sum_r exp2(s2_rj - m2_r - log2 l_r) / (G rows_t)
//           (masked entries count 0) is a per-lane column sum.
// Exact post-softmax pooling needs every row's normaliser before any column
// sum, hence the two passes over K (the second one mostly from L2).
//
// Warp-level bf16 MMA version: 8 warps own 16 rows (pass 1) or 16 keys
// (pass 2) each; K blocks of 128 keys go through a 2-stage cp.async pipeline.
#include "common.cuh"
#include "kernels.h"

namespace kascade {

namespace {

constexpr int kSpWarps = 8;
constexpr int kSpKeys = 128;
constexpr int kSpStages = 2;
constexpr int kSpMaxRows = 256;

template <int D>
__device__ __forceinline__ uint32_t sp_swz(int r, int ch) {
  return (uint32_t)(r * (D * 2) + ((ch ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kSpWarps * 32) score_pool_kernel(const ScorePoolArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int CH = D / 8;
  constexpr int KBLK_BYTES = kSpKeys * D * 2;
  extern __shared__ __align__(128) char smem[];
  char* q_sm = smem;                                                  // [RC*128][D]
  char* k_sm = smem + kSpMaxRows * D * 2;                             // [stages][128][D]
  float* bcol = reinterpret_cast<float*>(k_sm + kSpStages * KBLK_BYTES);   // [256]
  int* rpos = reinterpret_cast<int*>(bcol + kSpMaxRows);                   // [256]

  const int T = (a.N + a.tile - 1) / a.tile;
  const int t0 = a.q0 / a.tile;   // first query tile of the call (rolling chunks)
  const int t = T - 1 - (int)blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv;
  const int G = a.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int i0 = t * a.tile;
  const int e_t = min(i0 + a.tile, a.N);
  const int rows_t = e_t - i0;
  const int R = G * a.tile;
  const int RC = (R + 127) / 128;
  const uint32_t q_u = smem_u32(q_sm), k_u = smem_u32(k_sm);
  const float scale2 = kLog2e * rsqrtf((float)D);

  // Q tile -> shared (zero rows past the tile end), row positions
  for (int e = threadIdx.x; e < RC * 128 * CH; e += blockDim.x) {
    const int r = e / CH, ch = e - r * CH;
    const int gi = r / a.tile, il = r - gi * a.tile;
    const bool ok = r < R && il < rows_t;
    const __nv_bfloat16* src =
        a.q + ((size_t)(b * a.Hq + h * G + (ok ? gi : 0)) * a.Lq + (i0 - a.q0) + (ok ? il : 0)) * D + ch * 8;
    cp_async_16(q_u + sp_swz<D>(r, ch), src, ok ? 16 : 0);
  }
  cp_async_commit();
  for (int r = threadIdx.x; r < RC * 128; r += blockDim.x) {
    const int gi = r / a.tile, il = r - gi * a.tile;
    rpos[r] = (r < R && il < rows_t) ? i0 + il : -1;   // -1: padding row, sees nothing
  }

  const __nv_bfloat16* kb = a.k + (size_t)bh * a.N * D;
  const int n_blk = (e_t + kSpKeys - 1) / kSpKeys;
  auto issue = [&](int blk, int stage) {
    const int r = threadIdx.x >> 1;
    const int j = blk * kSpKeys + r;
    const bool ok = j < e_t;
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
      const int ch = (threadIdx.x & 1) * (CH / 2) + i;
      cp_async_16(k_u + stage * KBLK_BYTES + sp_swz<D>(r, ch), kb + (size_t)(ok ? j : 0) * D + ch * 8, ok ? 16 : 0);
    }
  };

  // ------------------------------------------------------------ pass 1
  for (int rc = 0; rc < RC; ++rc) {
    issue(0, 0);
    cp_async_commit();
    cp_async_wait<1>();   // Q tile (first round) has landed
    __syncthreads();
    const int rbase = rc * 128 + warp * 16;
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int mi = lane >> 3;
      ldmatrix_x4(qa[kk], q_u + sp_swz<D>(rbase + (mi & 1) * 8 + (lane & 7), 2 * kk + (mi >> 1)));
    }
    const int ipos[2] = {rpos[rbase + g], rpos[rbase + g + 8]};
    float m_run[2] = {-INFINITY, -INFINITY};
    double l_run[2] = {0.0, 0.0};
    for (int blk = 0; blk < n_blk; ++blk) {
      const int stage = blk % kSpStages;
      if (blk + 1 < n_blk) issue(blk + 1, (blk + 1) % kSpStages);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const uint32_t ks = k_u + stage * KBLK_BYTES;
      float sacc[kSpKeys / 8][4];
#pragma unroll
      for (int nt = 0; nt < kSpKeys / 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int nt = 0; nt < kSpKeys / 8; ++nt) {
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
          uint32_t r4[4];
          ldmatrix_x4(r4, ks + sp_swz<D>(nt * 8 + (lane & 7), 2 * kk + (lane >> 3)));
          mma_bf16_16816(sacc[nt], qa[kk], r4[0], r4[1]);
          mma_bf16_16816(sacc[nt], qa[kk + 1], r4[2], r4[3]);
        }
      }
      const int j0 = blk * kSpKeys;
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < kSpKeys / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j0 + nt * 8 + 2 * c + (e & 1);
          float s = sacc[nt][e] * scale2;
          if (j > ipos[e >> 1]) s = -INFINITY;   // causal (also j >= e_t and padding rows)
          sacc[nt][e] = s;
          mx[e >> 1] = fmaxf(mx[e >> 1], s);
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 1));
        mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 2));
        if (mx[hf] > m_run[hf]) {
          if (m_run[hf] != -INFINITY) l_run[hf] *= exp2((double)m_run[hf] - (double)mx[hf]);
          m_run[hf] = mx[hf];
        }
      }
      float part[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < kSpKeys / 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mm = m_run[e >> 1] == -INFINITY ? 0.f : m_run[e >> 1];
          part[e >> 1] += exp2f(sacc[nt][e] - mm);
        }
      }
      l_run[0] += (double)part[0];
      l_run[1] += (double)part[1];
      __syncthreads();
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      l_run[hf] += __shfl_xor_sync(0xffffffffu, l_run[hf], 1);
      l_run[hf] += __shfl_xor_sync(0xffffffffu, l_run[hf], 2);
      const int r = rbase + g + hf * 8;
      if (c == 0) {
        if (ipos[hf] >= 0) {
          const int gi = r / a.tile;
          const size_t srow = (size_t)(b * a.Hq + h * G + gi) * a.Lq + (ipos[hf] - a.q0);
          a.row_m2[srow] = m_run[hf];
          a.row_l[srow] = l_run[hf];
          bcol[r] = (float)((double)m_run[hf] + log2(l_run[hf]));
        } else {
          bcol[r] = INFINITY;
        }
      }
    }
    __syncthreads();
  }

  // ------------------------------------------------------------ pass 2
  const float inv_rows = 1.0f / (float)(G * rows_t);
  const float inv_rows_head = 1.0f / (float)rows_t;
  // pooled rows: one per kv head, or one per query head (per_head: the G
  // rows of this kv head's query heads, b Hq + h G + hh)
  const size_t pooled_row = (size_t)chunk_pooled_len(a.N, t0, a.tile);
  const size_t prow0 = a.per_head ? (size_t)(b * a.Hq + h * G) : (size_t)bh;
  float* pooled = a.pooled + prow0 * pooled_row + chunk_pooled_offset(t, t0, a.tile);
  issue(0, 0);
  cp_async_commit();
  for (int blk = 0; blk < n_blk; ++blk) {
    const int stage = blk % kSpStages;
    if (blk + 1 < n_blk) issue(blk + 1, (blk + 1) % kSpStages);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t ks = k_u + stage * KBLK_BYTES;
    // A = this warp's 16 keys
    uint32_t ka[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int mi = lane >> 3;
      ldmatrix_x4(ka[kk], ks + sp_swz<D>(warp * 16 + (mi & 1) * 8 + (lane & 7), 2 * kk + (mi >> 1)));
    }
    const int j0 = blk * kSpKeys + warp * 16;
    const int jk[2] = {j0 + g, j0 + g + 8};
    float colsum[2] = {0.f, 0.f};
    // the tile's 32 rows of head hh are rows [32 hh, 32 hh + 32)
    for (int hh = 0; hh < G; ++hh) {
      float hsum[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int rrow = hh * 32 + nt * 8;
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
          uint32_t r4[4];
          ldmatrix_x4(r4, q_u + sp_swz<D>(rrow + (lane & 7), 2 * kk + (lane >> 3)));
          mma_bf16_16816(acc, ka[kk], r4[0], r4[1]);
          mma_bf16_16816(acc, ka[kk + 1], r4[2], r4[3]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = rrow + 2 * c + (e & 1);
          const int j = jk[e >> 1];
          const float bb = bcol[r];
          const float p = (j <= rpos[r]) ? exp2f(acc[e] * scale2 - bb) : 0.f;
          hsum[e >> 1] += p;
        }
      }
      if (a.per_head) {
        // head hh alone: its own pooled row, mean over the tile's rows
        float* prow = pooled + (size_t)hh * pooled_row;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          hsum[hf] += __shfl_xor_sync(0xffffffffu, hsum[hf], 1);
          hsum[hf] += __shfl_xor_sync(0xffffffffu, hsum[hf], 2);
          if (c == 0 && jk[hf] < e_t) prow[jk[hf]] = hsum[hf] * inv_rows_head;
        }
      } else {
        colsum[0] += hsum[0];
        colsum[1] += hsum[1];
      }
    }
    if (!a.per_head) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        colsum[hf] += __shfl_xor_sync(0xffffffffu, colsum[hf], 1);
        colsum[hf] += __shfl_xor_sync(0xffffffffu, colsum[hf], 2);
        if (c == 0 && jk[hf] < e_t) pooled[jk[hf]] = colsum[hf] * inv_rows;
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
}

template <int D>
size_t score_pool_smem() {
  return (size_t)kSpMaxRows * D * 2 + (size_t)kSpStages * kSpKeys * D * 2 + kSpMaxRows * 8;
}

}  // namespace

cudaError_t launch_score_pool(const ScorePoolArgs& a, cudaStream_t stream) {
  const int T = (a.N + a.tile - 1) / a.tile - a.q0 / a.tile;   // the call's query tiles
  dim3 grid(T, a.B * a.Hkv);
  if (a.D == 128) {
    const size_t sm = score_pool_smem<128>();
    const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(score_pool_kernel<128>), sm, false);
    if (e != cudaSuccess) return e;
    return launch_ex(score_pool_kernel<128>, grid, dim3(kSpWarps * 32), sm, stream, (a.flags & 1) != 0, 1, a);
  } else {
    const size_t sm = score_pool_smem<64>();
    const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(score_pool_kernel<64>), sm, false);
    if (e != cudaSuccess) return e;
    return launch_ex(score_pool_kernel<64>, grid, dim3(kSpWarps * 32), sm, stream, (a.flags & 1) != 0, 1, a);
  }
  return cudaGetLastError();
}

}  // namespace kascade
