// Anchor decode scoring (Kascade README, Abstract: anchor layers compute
// exact attention scores over the whole context before selecting Top-k).
//
// For one decode query per query head and every cached key j < N:
//   s2[b, qh, j] = (q_qh . k_j) * log2(e) / sqrt(d)        (fp32, base-2 domain)
// plus per-split softmax statistics of each query head
//   m2[b, qh, split] = max_j s2,   l[b, qh, split] = sum_j exp2(s2 - m2)   (fp64)
//
// HBM-bound: every byte of K is read once with 16-byte coalesced loads that
// go straight into the registers of a warp-level bf16 MMA (K rows as the
// 16x16 A tile, the G <= 8 query heads of the kv head as the 8-wide B tile).
// Since the contraction runs over d, each lane may take any permutation of d
// as long as q uses the same one: lane (g, c) loads dims [32s + 8c, +8) of
// key rows g and g+8, which is exactly what a 16-byte load gives.
#include "common.cuh"
#include "kernels.h"

namespace kascade {

namespace {

constexpr int kScoreWarps = 4;
constexpr int kGroupsPerWarp = 8;  // 16 keys per group

template <int D>
__global__ void __launch_bounds__(kScoreWarps * 32)
    decode_score_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                        float* __restrict__ s2, float* __restrict__ m_part,
                        double* __restrict__ l_part, int N, int Hq, int Hkv, int G, int splits,
                        float scale2, const int32_t* __restrict__ cand, const int32_t* __restrict__ cand_map,
                        int cand_lists, int n_ctx, const int32_t* __restrict__ kv_lens) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int CH = D / 32;
  constexpr int KEYS = 16 * kScoreWarps * kGroupsPerWarp;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / Hkv, h = bh - b * Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;

  uint4 qf[CH];
  if (g < G) {
    const __nv_bfloat16* qrow = q + (size_t)(b * Hq + h * G + g) * D;
#pragma unroll
    for (int s = 0; s < CH; ++s) qf[s] = *reinterpret_cast<const uint4*>(qrow + 32 * s + 8 * c);
  } else {
#pragma unroll
    for (int s = 0; s < CH; ++s) qf[s] = make_uint4(0, 0, 0, 0);
  }

  const __nv_bfloat16* kbase = k + (size_t)bh * n_ctx * D;
  // scored position r is key r, or key clist[r] of the candidate list
  const int32_t* clist = nullptr;
  if (cand) {
    int hm = cand_map ? cand_map[h] : h;
    if (hm < 0 || hm >= cand_lists) hm = 0;
    clist = cand + (size_t)(b * cand_lists + hm) * N;
  }
  const int j0 = split * KEYS;
  const int j1 = min(kv_lens ? min(N, kv_lens[b]) : N, j0 + KEYS);   // a varlen row ends at its own length

  float sc[kGroupsPerWarp][4];
  uint4 ra[CH], rb[CH];
  auto load_group = [&](int it) {
    const int r0 = j0 + (it * kScoreWarps + warp) * 16 + g;
    const int r1 = r0 + 8;
    const int k0 = r0 < j1 ? (clist ? __ldg(clist + r0) : r0) : 0;
    const int k1 = r1 < j1 ? (clist ? __ldg(clist + r1) : r1) : 0;
#pragma unroll
    for (int s = 0; s < CH; ++s) {
      ra[s] = r0 < j1 ? ldg_nc_v4(kbase + (size_t)k0 * D + 32 * s + 8 * c) : make_uint4(0, 0, 0, 0);
      rb[s] = r1 < j1 ? ldg_nc_v4(kbase + (size_t)k1 * D + 32 * s + 8 * c) : make_uint4(0, 0, 0, 0);
    }
  };

  load_group(0);
#pragma unroll
  for (int it = 0; it < kGroupsPerWarp; ++it) {
    uint4 ca[CH], cb[CH];
#pragma unroll
    for (int s = 0; s < CH; ++s) {
      ca[s] = ra[s];
      cb[s] = rb[s];
    }
    if (it + 1 < kGroupsPerWarp) load_group(it + 1);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < CH; ++s) {
      const uint32_t a0[4] = {ca[s].x, cb[s].x, ca[s].y, cb[s].y};
      mma_bf16_16816(acc, a0, qf[s].x, qf[s].y);
      const uint32_t a1[4] = {ca[s].z, cb[s].z, ca[s].w, cb[s].w};
      mma_bf16_16816(acc, a1, qf[s].z, qf[s].w);
    }
    const int r0 = j0 + (it * kScoreWarps + warp) * 16 + g;
    const int r1 = r0 + 8;
    const bool v0 = r0 < j1, v1 = r1 < j1;
    sc[it][0] = v0 ? acc[0] * scale2 : -INFINITY;  // key r0, head 2c
    sc[it][1] = v0 ? acc[1] * scale2 : -INFINITY;  // key r0, head 2c+1
    sc[it][2] = v1 ? acc[2] * scale2 : -INFINITY;  // key r1, head 2c
    sc[it][3] = v1 ? acc[3] * scale2 : -INFINITY;  // key r1, head 2c+1
    const int h0 = 2 * c, h1 = 2 * c + 1;
    float* out0 = s2 + (size_t)(b * Hq + h * G + h0) * N;
    float* out1 = out0 + N;
    if (h0 < G) {
      if (v0) out0[r0] = sc[it][0];
      if (v1) out0[r1] = sc[it][2];
    }
    if (h1 < G) {
      if (v0) out1[r0] = sc[it][1];
      if (v1) out1[r1] = sc[it][3];
    }
  }

  // split statistics: max, then sum of exp2(s - max) (fp32 per lane, fp64 across lanes)
  __shared__ float red_m[kScoreWarps][8];
  __shared__ double red_l[kScoreWarps][8];
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int it = 0; it < kGroupsPerWarp; ++it) {
    mx0 = fmaxf(mx0, fmaxf(sc[it][0], sc[it][2]));
    mx1 = fmaxf(mx1, fmaxf(sc[it][1], sc[it][3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  if (g == 0) {
    red_m[warp][2 * c] = mx0;
    red_m[warp][2 * c + 1] = mx1;
  }
  __syncthreads();
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < kScoreWarps; ++w) {
    m0 = fmaxf(m0, red_m[w][2 * c]);
    m1 = fmaxf(m1, red_m[w][2 * c + 1]);
  }
  float su0 = 0.f, su1 = 0.f;
#pragma unroll
  for (int it = 0; it < kGroupsPerWarp; ++it) {
    if (m0 != -INFINITY) su0 += exp2f(sc[it][0] - m0) + exp2f(sc[it][2] - m0);   // a split past a
    if (m1 != -INFINITY) su1 += exp2f(sc[it][1] - m1) + exp2f(sc[it][3] - m1);   // varlen row's end: 0
  }
  double d0 = su0, d1 = su1;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    d0 += __shfl_xor_sync(0xffffffffu, d0, o);
    d1 += __shfl_xor_sync(0xffffffffu, d1, o);
  }
  if (g == 0) {
    red_l[warp][2 * c] = d0;
    red_l[warp][2 * c + 1] = d1;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int hh = threadIdx.x;
    double l = 0.0;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kScoreWarps; ++w) {
      l += red_l[w][hh];
      m = fmaxf(m, red_m[w][hh]);
    }
    const size_t row = (size_t)(b * Hq + h * G + hh) * splits + split;
    m_part[row] = m;
    l_part[row] = l;
  }
}

}  // namespace

int decode_score_keys_per_split() { return 16 * kScoreWarps * kGroupsPerWarp; }

cudaError_t launch_decode_score(const DecodeScoreArgs& a, cudaStream_t stream) {
  const int splits = (a.N + decode_score_keys_per_split() - 1) / decode_score_keys_per_split();
  dim3 grid(splits, a.B * a.Hkv);
  const float scale2 = kLog2e / sqrtf((float)a.D);
  const bool pdl = (a.flags & 1) != 0;
  const int n_ctx = a.cand ? a.n_ctx : a.N;
  if (a.D == 128)
    return launch_ex(decode_score_kernel<128>, grid, dim3(kScoreWarps * 32), 0, stream, pdl, 1, a.q, a.k, a.s2,
                     a.m_part, a.l_part, a.N, a.Hq, a.Hkv, a.G, splits, scale2, a.cand, a.cand_map, a.cand_lists,
                     n_ctx, a.kv_lens);
  return launch_ex(decode_score_kernel<64>, grid, dim3(kScoreWarps * 32), 0, stream, pdl, 1, a.q, a.k, a.s2,
                   a.m_part, a.l_part, a.N, a.Hq, a.Hkv, a.G, splits, scale2, a.cand, a.cand_map, a.cand_lists,
                   n_ctx, a.kv_lens);
}

}  // namespace kascade
