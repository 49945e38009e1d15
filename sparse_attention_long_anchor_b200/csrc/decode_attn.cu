// Gather-sparse decode attention of the Kascade anchor and reuse layers
// (README, Abstract: reuse layers attend only over the anchor's Top-k
// indices; selection and reuse are head-aware).  With an implicit full key
// list the same kernel is the dense decode reference.
//
// One thread-block cluster per (batch, kv head); the index list is split
// evenly over the CTAs of the cluster and every warp owns 16-key slices of
// its CTA's share.  All warps gather at once:
//   * K rows go straight from global memory into the registers of the
//     16x8x16 bf16 MMA (the contraction runs over d, so each lane may take
//     any permutation of d as long as q uses the same: lane (g, c) loads
//     dims [32s + 8c, +8) of key g, one 16-byte load per 32 dims);
//   * V rows go through a two-slot cp.async ring per warp (16-byte copies
//     into rows padded by 16 bytes, conflict-free for ldmatrix.trans);
//   * the G query rows sit in shared memory and are read with 8-byte loads
//     in the same permuted order.
// S = Q K^T (query heads as the MMA rows), fp32 online softmax, O += P V.
// The partial (max, sum, output) of each CTA is pushed over distributed
// shared memory to the CTA that owns each output element; after one cluster
// barrier every CTA merges its slice locally.  No global scratch, no
// spin-waits.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace kascade {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxCS = 16;
constexpr int kIdxStage = 2048;   // index entries staged in shared memory

template <int D>
struct Lay {
  static constexpr int ROW = D * 2 + 16;                  // padded V row bytes
  static constexpr int SLOT = 16 * ROW;                   // one 16-key V slab
  static constexpr size_t vslots = 0;                     // [W][2] slots
  static constexpr size_t qs = vslots + (size_t)kWarps * 2 * SLOT;   // [8][D] bf16 query rows
  static constexpr size_t idx = qs + 8 * D * 2;
  static constexpr size_t recv_o = idx + kIdxStage * 4;   // [G*D] f32, peers write here
  static constexpr size_t recv_ml = recv_o + 8 * D * 4;   // [16][8][2]
  static constexpr size_t total = recv_ml + kMaxCS * 8 * 2 * 4;
  // after the gather loop, inside the V slots
  static constexpr int RO = D + 8;                        // padded red_o row (floats)
  static constexpr size_t red_o = 0;                      // [W][8][RO]
  static constexpr size_t red_ml = red_o + (size_t)kWarps * 8 * RO * 4;
  static constexpr size_t wf = red_ml + kWarps * 8 * 2 * 4;
  static constexpr size_t pml = wf + kWarps * 8 * 4;
  static constexpr size_t wts = pml + 8 * 2 * 4;
  static constexpr size_t head = wts + kMaxCS * 8 * 4;
  static_assert(head + 64 <= qs, "post-loop scratch must fit in the V slots");
};

__device__ __forceinline__ float scale_from(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.0f : exp2f(m_old - m_new);
}

// Softmax-merge weights of n_slots partial results per head: for every
// (slot, head) the factor exp2(m - M) against the head's max M, and per head
// (M, sum of factor * l).  Called by one whole warp.  ml and w are laid out
// [slot][8][2] and [slot][8]; out is [8][2].
__device__ void merge_weights(int n_slots, int G, const float* ml, float* w, float* out, int lane) {
  if (32 % G == 0) {
    const int gg = lane % G;   // every pair a lane visits belongs to this head
    float M = -INFINITY;
    for (int i = lane; i < n_slots * G; i += 32) M = fmaxf(M, ml[((i / G) * 8 + gg) * 2]);
    for (int o = G; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float ls = 0.f;
    for (int i = lane; i < n_slots * G; i += 32) {
      const int sl = i / G;
      const float f = scale_from(ml[(sl * 8 + gg) * 2], M);
      w[sl * 8 + gg] = f;
      ls += f * ml[(sl * 8 + gg) * 2 + 1];
    }
    for (int o = G; o < 32; o <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    if (lane < G) {
      out[gg * 2] = M;
      out[gg * 2 + 1] = ls;
    }
  } else if (lane < G) {
    const int gg = lane;
    float M = -INFINITY;
    for (int sl = 0; sl < n_slots; ++sl) M = fmaxf(M, ml[(sl * 8 + gg) * 2]);
    float ls = 0.f;
    for (int sl = 0; sl < n_slots; ++sl) {
      const float f = scale_from(ml[(sl * 8 + gg) * 2], M);
      w[sl * 8 + gg] = f;
      ls += f * ml[(sl * 8 + gg) * 2 + 1];
    }
    out[gg * 2] = M;
    out[gg * 2 + 1] = ls;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2) decode_attn_kernel(const AttnArgs a, int per) {
  using L = Lay<D>;
  constexpr int KS = D / 32;          // 16-byte K loads per key row per lane
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
  const int bh = blockIdx.y;
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
  const int c0 = min(list_len, rank * per);
  const int c1 = min(list_len, c0 + per);
  const int n_slices = (c1 - c0 + 15) / 16;
  int* idx_s = reinterpret_cast<int*>(smem + L::idx);
  const bool staged = list != nullptr && (c1 - c0) <= kIdxStage;
  const __nv_bfloat16* kb = a.k + (size_t)bh * a.N * D;
  const __nv_bfloat16* vb = a.v + (size_t)bh * a.N * D;

  if (staged)
    for (int i = threadIdx.x; i < c1 - c0; i += kThreads) idx_s[i] = __ldg(list + c0 + i);
  __syncthreads();

  auto key_of = [&](int rel) -> int {
    return list ? (staged ? idx_s[rel] : __ldg(list + c0 + rel)) : c0 + rel;
  };
  // V rows of slice s into this warp's slot (s / W) & 1; missing rows zero-filled
  const uint32_t vbase = smem_u32(smem) + (uint32_t)(warp * 2 * L::SLOT);
  auto issue_v = [&](int s) {
    const uint32_t dst = vbase + ((s / kWarps) & 1) * L::SLOT;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {   // 16 rows x D/8 chunks over 32 lanes
      const int e = lane + 32 * i;
      const int r = e / (D / 8), ch = e - r * (D / 8);
      const int rel = s * 16 + r;
      const bool have = c0 + rel < c1;
      const int key = have ? key_of(rel) : 0;
      cp_async_16(dst + r * L::ROW + ch * 16, vb + (size_t)key * D + ch * 8, have ? 16 : 0);
    }
    cp_async_commit();
  };
  // K rows g and 8+g of slice s into registers (zero past the list end)
  uint4 kr[2][KS];
  auto load_k = [&](int s) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int rel = s * 16 + t * 8 + g;
      const bool have = c0 + rel < c1;
      const __nv_bfloat16* row = kb + (size_t)(have ? key_of(rel) : 0) * D + 8 * c;
#pragma unroll
      for (int q = 0; q < KS; ++q) kr[t][q] = have ? ldg_nc_v4(row + 32 * q) : make_uint4(0, 0, 0, 0);
    }
  };

  float m_run = -INFINITY, l_run = 0.f;
  float oacc[D / 8][2];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) oacc[nd][0] = oacc[nd][1] = 0.f;
  const float scale2 = kLog2e * rsqrtf((float)D);
  const char* qrow = smem + L::qs + (size_t)(g * D + 8 * c) * 2;

  // prologue: V of this warp's first two slices, K of its first slice
  int s = warp;
  if (s < n_slices) issue_v(s);
  if (s + kWarps < n_slices) issue_v(s + kWarps);
  if (s < n_slices) load_k(s);
  if (early) {
    pdl_wait();
    pdl_launch_dependents();
  }
  // the G query rows of this kv head (rows G..7 zero)
  for (int i = threadIdx.x; i < 8 * (D / 8); i += kThreads) {
    const int r = i / (D / 8), ch = i - r * (D / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < G) val = *reinterpret_cast<const uint4*>(a.q + (size_t)(b * a.Hq + h * G + r) * D + ch * 8);
    *reinterpret_cast<uint4*>(smem + L::qs + (r * D + ch * 8) * 2) = val;
  }
  __syncthreads();
  for (; s < n_slices; s += kWarps) {
    // S = Q K^T: k-step 2q+hf takes dims 32q + 8c + 4hf + {0,1} (a0/b0) and
    // + {2,3} (a2/b1) of the query rows and key rows
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < KS; ++q) {
      const uint2 qlo = *reinterpret_cast<const uint2*>(qrow + 64 * q);       // dims 32q+8c+0..3
      const uint2 qhi = *reinterpret_cast<const uint2*>(qrow + 64 * q + 8);   // dims 32q+8c+4..7
      const uint32_t a0[4] = {qlo.x, 0u, qlo.y, 0u};
      const uint32_t a1[4] = {qhi.x, 0u, qhi.y, 0u};
      mma_bf16_16816(s0, a0, kr[0][q].x, kr[0][q].y);
      mma_bf16_16816(s1, a0, kr[1][q].x, kr[1][q].y);
      mma_bf16_16816(s0, a1, kr[0][q].z, kr[0][q].w);
      mma_bf16_16816(s1, a1, kr[1][q].z, kr[1][q].w);
    }
    const int kbase = c0 + s * 16;
    float sv[4];
    sv[0] = kbase + 2 * c < c1 ? s0[0] * scale2 : -INFINITY;
    sv[1] = kbase + 2 * c + 1 < c1 ? s0[1] * scale2 : -INFINITY;
    sv[2] = kbase + 8 + 2 * c < c1 ? s1[0] * scale2 : -INFINITY;
    sv[3] = kbase + 9 + 2 * c < c1 ? s1[1] * scale2 : -INFINITY;
    float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = scale_from(m_run, m_new);
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = exp2f(sv[e] - m_new);
    l_run = l_run * alpha + (p[0] + p[1] + p[2] + p[3]);
    m_run = m_new;
    const uint32_t pa[4] = {pack_bf16(p[0], p[1]), 0u, pack_bf16(p[2], p[3]), 0u};
    // V of this slice: its copy group is the oldest one still pending
    if (s + kWarps < n_slices) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncwarp();
    const uint32_t vs = vbase + ((s / kWarps) & 1) * L::SLOT;
#pragma unroll
    for (int nd = 0; nd < D / 8; nd += 2) {
      uint32_t r4[4];
      const int mi = lane >> 3;
      ldmatrix_x4_trans(r4, vs + ((mi & 1) * 8 + (lane & 7)) * L::ROW + (nd + (mi >> 1)) * 16);
      float t0[4] = {oacc[nd][0] * alpha, oacc[nd][1] * alpha, 0.f, 0.f};
      float t1[4] = {oacc[nd + 1][0] * alpha, oacc[nd + 1][1] * alpha, 0.f, 0.f};
      mma_bf16_16816(t0, pa, r4[0], r4[1]);
      mma_bf16_16816(t1, pa, r4[2], r4[3]);
      oacc[nd][0] = t0[0];
      oacc[nd][1] = t0[1];
      oacc[nd + 1][0] = t1[0];
      oacc[nd + 1][1] = t1[1];
    }
    __syncwarp();
    if (s + 2 * kWarps < n_slices) issue_v(s + 2 * kWarps);   // refill the slot just read
    if (s + kWarps < n_slices) load_k(s + kWarps);
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

  // ---------------- merge the warps into this CTA's partial
  __syncthreads();
  float* red_o = reinterpret_cast<float*>(smem + L::red_o);
  float* red_ml = reinterpret_cast<float*>(smem + L::red_ml);
  if (g < G) {
#pragma unroll
    for (int nd = 0; nd < D / 8; ++nd)
      *reinterpret_cast<float2*>(red_o + (warp * 8 + g) * L::RO + nd * 8 + 2 * c) =
          make_float2(oacc[nd][0], oacc[nd][1]);
    if (c == 0) {
      red_ml[(warp * 8 + g) * 2] = m_run;
      red_ml[(warp * 8 + g) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  // per-head weights of the warps
  float* wf = reinterpret_cast<float*>(smem + L::wf);
  float* pml = reinterpret_cast<float*>(smem + L::pml);
  if (warp == 0) merge_weights(kWarps, G, red_ml, wf, pml, lane);
  __syncthreads();
  // push element e to CTA e / en (E is a multiple of the cluster size)
  float* recv_o = reinterpret_cast<float*>(smem + L::recv_o);
  float* recv_ml = reinterpret_cast<float*>(smem + L::recv_ml);
  const int E = G * D;
  const int en = E / CS;
  for (int e = threadIdx.x; e < E; e += kThreads) {
    const int gg = e / D, dd = e - gg * D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) acc += wf[w * 8 + gg] * red_o[(w * 8 + gg) * L::RO + dd];
    const int q = e / en;
    *cluster.map_shared_rank(recv_o + rank * en + (e - q * en), q) = acc;
  }
  if (threadIdx.x < CS * G) {
    const int r = threadIdx.x / G, gg = threadIdx.x - r * G;
    float* ml = cluster.map_shared_rank(recv_ml, r);
    ml[(rank * 8 + gg) * 2] = pml[gg * 2];
    ml[(rank * 8 + gg) * 2 + 1] = pml[gg * 2 + 1];
  }
  cluster.sync();

  // ---------------- merge this CTA's element slice from local shared memory
  float* wts = reinterpret_cast<float*>(smem + L::wts);
  float* head = reinterpret_cast<float*>(smem + L::head);
  if (warp == 0) merge_weights(CS, G, recv_ml, wts, head, lane);
  __syncthreads();
  const int e0 = rank * en, e1 = e0 + en;
  for (int e = e0 + (int)threadIdx.x; e < e1; e += kThreads) {
    const int gg = e / D, dd = e - gg * D;
    float acc = 0.f;
    for (int r = 0; r < CS; ++r) acc += wts[r * 8 + gg] * recv_o[r * en + (e - e0)];
    const float Ls = head[gg * 2 + 1];
    const size_t orow = (size_t)(b * a.Hq + h * G + gg);
    a.o[orow * D + dd] = __float2bfloat16(Ls > 0.f ? acc / Ls : 0.f);
    if (dd == 0 && a.lse) a.lse[orow] = Ls > 0.f ? (head[gg * 2] + log2f(Ls)) * (float)kLn2 : -INFINITY;
  }
}

template <int D>
cudaLaunchConfig_t make_cfg(int cs, int bh, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, bh, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Lay<D>::total;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// 16-CTA clusters when the device can co-schedule them, else 8
template <int D>
int cluster_size_for_device() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (cached[dev]) return cached[dev];
  int cs = 8;
  if (cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)Lay<D>::total) == cudaSuccess &&
      cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess) {
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = make_cfg<D>(kMaxCS, 1, nullptr, attr);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_attn_kernel<D>, &cfg) == cudaSuccess && n > 0) cs = kMaxCS;
  }
  cudaGetLastError();
  cached[dev] = cs;
  return cs;
}

template <int D>
cudaError_t launch(const AttnArgs& a, cudaStream_t stream) {
  const int cs = cluster_size_for_device<D>();
  const int list_len = a.idx ? topk_count(a.N, a.num, a.den) : a.N;
  int per = (list_len + cs - 1) / cs;
  per = (per + 15) / 16 * 16;
  if (per < 16) per = 16;
  if ((a.G * D) % cs != 0) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Lay<D>::total);
  if (e != cudaSuccess) return e;
  if (cs > 8) {
    e = cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  return launch_ex(decode_attn_kernel<D>, dim3(cs, a.B * a.Hkv), dim3(kThreads), Lay<D>::total, stream,
                   (a.flags & 1) != 0, cs, a, per);
}

}  // namespace

cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t stream) {
  return a.D == 128 ? launch<128>(a, stream) : launch<64>(a, stream);
}

}  // namespace kascade
