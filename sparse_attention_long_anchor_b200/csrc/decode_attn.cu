// Gather-sparse decode attention of the Kascade anchor and reuse layers
// (README, Abstract: reuse layers attend only over the anchor's Top-k
// indices; selection and reuse are head-aware).  With an implicit full key
// list the same kernel is the dense decode reference.
//
// One thread-block cluster per (batch, kv head): the index list is split
// evenly over the CTAs of the cluster, every warp gathers 16-key slices of
// K and V rows with 16-byte cp.async into XOR-swizzled shared memory
// (3-stage pipeline per warp) and runs bf16 MMAs with the G query heads as
// the rows of a 16-row tile and an fp32 online softmax.  The partial
// (max, sum, output) of each CTA stays in its shared memory; after a
// cluster barrier every CTA merges one slice of the output elements from
// all CTAs over distributed shared memory.  Nothing goes through global
// scratch and no CTA waits on anything but the cluster barrier.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace kascade {

namespace {

constexpr int kWarps = 4;
constexpr int kStages = 3;
constexpr int kMaxCS = 16;

template <int D>
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return (uint32_t)(r * (D * 2) + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ float scale_from(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.0f : exp2f(m_old - m_new);
}

template <int D>
constexpr size_t pipe_bytes() {
  return (size_t)kWarps * kStages * 2 * 16 * D * 2;
}

// shared-memory layout after the gather loop (inside the pipeline region):
//   red_o [W][8][D] | red_ml [W][8][2] | wts [16][8] | head [8][2]
// and, in a region of their own that peers may write at any time:
//   recv_o [G*D] f32 ([rank][slice] of this CTA's element slice) | recv_ml [16][8][2]
template <int D>
struct Post {
  static constexpr size_t red_o = 0;
  static constexpr size_t red_ml = red_o + (size_t)kWarps * 8 * D * 4;
  static constexpr size_t wts = red_ml + kWarps * 8 * 2 * 4;
  static constexpr size_t head = wts + kMaxCS * 8 * 4;
  static constexpr size_t end = head + 8 * 2 * 4;
};

constexpr int kIdxStage = 2048;   // index entries staged in shared memory

template <int D>
constexpr size_t main_bytes() {
  return pipe_bytes<D>() > Post<D>::end ? pipe_bytes<D>() : Post<D>::end;
}
template <int D>
constexpr size_t recv_off() {
  return main_bytes<D>() + kIdxStage * 4;
}
template <int D>
constexpr size_t smem_bytes() {
  return recv_off<D>() + 8 * D * 4 + kMaxCS * 8 * 2 * 4;
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) decode_attn_kernel(const AttnArgs a, int per) {
  constexpr int CH = D / 8;
  constexpr int SLICE = 16 * D * 2;   // one 16-key slab of K (or V)
  extern __shared__ __align__(128) char smem[];

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

  const uint32_t wsm = smem_u32(smem) + warp * (kStages * 2 * SLICE);
  const int n_slices = (c1 - c0 + 15) / 16;
  const float scale2 = kLog2e * rsqrtf((float)D);

  // this CTA's slice of the index list, staged once with coalesced loads
  int* idx_s = reinterpret_cast<int*>(smem + main_bytes<D>());
  const bool staged = list != nullptr && (c1 - c0) <= kIdxStage;
  if (staged) {
    for (int i = threadIdx.x; i < c1 - c0; i += blockDim.x) idx_s[i] = __ldg(list + c0 + i);
    __syncthreads();
  }

  // lanes 2r, 2r+1 copy row r; each instruction moves 32 contiguous bytes per row
  auto issue = [&](int slice, int stage) {
    const int rel = slice * 16 + (lane >> 1);
    const int pos = c0 + rel;
    const bool ok = pos < c1;
    const int key = !ok ? 0 : (list ? (staged ? idx_s[rel] : __ldg(list + pos)) : pos);
    const uint32_t kdst = wsm + stage * 2 * SLICE;
    const uint32_t vdst = kdst + SLICE;
    const int r = lane >> 1;
#pragma unroll
    for (int i = 0; i < CH / 2; ++i) {
      const int ch = 2 * i + (lane & 1);
      cp_async_16(kdst + swz<D>(r, ch), kb + (size_t)key * D + ch * 8, ok ? 16 : 0);
      cp_async_16(vdst + swz<D>(r, ch), vb + (size_t)key * D + ch * 8, ok ? 16 : 0);
    }
  };

  float m_run = -INFINITY, l_run = 0.f;
  float oacc[D / 8][2];
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) oacc[nd][0] = oacc[nd][1] = 0.f;

  // this warp's slices: warp, warp + W, ...; up to kStages - 1 in flight ahead
  int s_issue = warp;
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (s_issue < n_slices) issue(s_issue, st);
    cp_async_commit();
    s_issue += kWarps;
  }
  int stage = 0;
  for (int s = warp; s < n_slices; s += kWarps) {
    {
      const int st_next = (stage + kStages - 1) % kStages;
      if (s_issue < n_slices) issue(s_issue, st_next);
      cp_async_commit();
      s_issue += kWarps;
    }
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint32_t ks = wsm + stage * 2 * SLICE;
    const uint32_t vs = ks + SLICE;

    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int kk = 0; kk < D / 16; kk += 2) {
        uint32_t r4[4];
        ldmatrix_x4(r4, ks + swz<D>(nt * 8 + (lane & 7), 2 * kk + (lane >> 3)));
        const uint32_t a0[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
        mma_bf16_16816(sacc[nt], a0, r4[0], r4[1]);
        const uint32_t a1[4] = {qa[kk + 1][0], 0u, qa[kk + 1][1], 0u};
        mma_bf16_16816(sacc[nt], a1, r4[2], r4[3]);
      }
    }
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
    const float alpha = scale_from(m_run, m_new);
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
#pragma unroll
    for (int nd = 0; nd < D / 8; nd += 2) {
      uint32_t r4[4];
      const int mi = lane >> 3;
      ldmatrix_x4_trans(r4, vs + swz<D>((mi & 1) * 8 + (lane & 7), nd + (mi >> 1)));
      float t0[4] = {oacc[nd][0], oacc[nd][1], 0.f, 0.f};
      float t1[4] = {oacc[nd + 1][0], oacc[nd + 1][1], 0.f, 0.f};
      mma_bf16_16816(t0, pa, r4[0], r4[1]);
      mma_bf16_16816(t1, pa, r4[2], r4[3]);
      oacc[nd][0] = t0[0];
      oacc[nd][1] = t0[1];
      oacc[nd + 1][0] = t1[0];
      oacc[nd + 1][1] = t1[1];
    }
    __syncwarp();
    stage = (stage + 1) % kStages;
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

  // merge the warps of this CTA, then push the partial to the CTAs that own
  // each output element (remote stores do not stall the issuing thread)
  __syncthreads();
  using P = Post<D>;
  float* recv_o = reinterpret_cast<float*>(smem + recv_off<D>());
  float* recv_ml = recv_o + 8 * D;
  float* red_o = reinterpret_cast<float*>(smem + P::red_o);
  float* red_ml = reinterpret_cast<float*>(smem + P::red_ml);
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
  const int E = G * D;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int gg = e / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_ml[(w * 8 + gg) * 2]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = scale_from(red_ml[(w * 8 + gg) * 2], M);
      acc += f * red_o[(w * 8 + gg) * D + (e - gg * D)];
      lsum += f * red_ml[(w * 8 + gg) * 2 + 1];
    }
    // owner of element e and its slot: slices [E*q/CS, E*(q+1)/CS)
    int q = (int)(((long)e * CS) / E);
    while ((int)((long)E * (q + 1) / CS) <= e) ++q;
    while ((int)((long)E * q / CS) > e) --q;
    const int q0 = (int)((long)E * q / CS), qn = (int)((long)E * (q + 1) / CS) - q0;
    float* dst = cluster.map_shared_rank(recv_o, q);
    dst[rank * qn + (e - q0)] = acc;
    if (e - gg * D == 0) {
      for (int r = 0; r < CS; ++r) {
        float* ml = cluster.map_shared_rank(recv_ml, r);
        ml[(rank * 8 + gg) * 2] = M;
        ml[(rank * 8 + gg) * 2 + 1] = lsum;
      }
    }
  }
  cluster.sync();

  // merge this CTA's element slice from local shared memory
  float* wts = reinterpret_cast<float*>(smem + P::wts);    // [CS][8]
  float* head = reinterpret_cast<float*>(smem + P::head);  // [8]: M, L
  if (threadIdx.x < G) {
    const int gg = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < CS; ++r) M = fmaxf(M, recv_ml[(r * 8 + gg) * 2]);
    float L = 0.f;
    for (int r = 0; r < CS; ++r) {
      const float f = scale_from(recv_ml[(r * 8 + gg) * 2], M);
      wts[r * 8 + gg] = f;
      L += f * recv_ml[(r * 8 + gg) * 2 + 1];
    }
    head[gg * 2] = M;
    head[gg * 2 + 1] = L;
  }
  __syncthreads();
  const int e0 = (int)((long)E * rank / CS), e1 = (int)((long)E * (rank + 1) / CS);
  const int en = e1 - e0;
  for (int e = e0 + (int)threadIdx.x; e < e1; e += blockDim.x) {
    const int gg = e / D, dd = e - gg * D;
    float acc = 0.f;
    for (int r = 0; r < CS; ++r) acc += wts[r * 8 + gg] * recv_o[r * en + (e - e0)];
    const float L = head[gg * 2 + 1];
    const size_t orow = (size_t)(b * a.Hq + h * G + gg);
    a.o[orow * D + dd] = __float2bfloat16(L > 0.f ? acc / L : 0.f);
    if (dd == 0 && a.lse) a.lse[orow] = L > 0.f ? (head[gg * 2] + log2f(L)) * (float)kLn2 : -INFINITY;
  }
}

template <int D>
cudaError_t launch(const AttnArgs& a, cudaStream_t stream, int cs, int per) {
  const size_t sm = smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  if (cs > 8) {
    e = cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, a.B * a.Hkv, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_attn_kernel<D>, a, per);
}

}  // namespace

int decode_attn_cluster_size() { return kMaxCS; }

// 16-CTA clusters when the device can co-schedule them, else 8
template <int D>
int cluster_size_for_device() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (cached[dev]) return cached[dev];
  int cs = 8;
  const size_t sm = smem_bytes<D>();
  if (cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) ==
          cudaSuccess &&
      cudaFuncSetAttribute(decode_attn_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMaxCS, 1, 1);
    cfg.blockDim = dim3(kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = sm;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kMaxCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_attn_kernel<D>, &cfg) == cudaSuccess && n > 0) cs = kMaxCS;
  }
  cudaGetLastError();
  cached[dev] = cs;
  return cs;
}

cudaError_t launch_decode_attn(const AttnArgs& a, cudaStream_t stream) {
  const int list_len = a.idx ? topk_count(a.N, a.num, a.den) : a.N;
  const int cs = a.D == 128 ? cluster_size_for_device<128>() : cluster_size_for_device<64>();
  int per = (list_len + cs - 1) / cs;
  per = (per + 15) / 16 * 16;
  if (per < 16) per = 16;
  return a.D == 128 ? launch<128>(a, stream, cs, per) : launch<64>(a, stream, cs, per);
}

}  // namespace kascade
