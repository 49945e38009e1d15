// fp32- and fp16-input variants of the Kascade path: q, k, v and o in fp32
// (for callers that need outputs within 1e-4 of exact attention: bf16 inputs
// and outputs carry about 4e-3 relative rounding, TF32 tensor-core products
// about 1e-3) or in fp16 (the README's own kernels take fp16 only, Running
// Evaluations).  Same method as the bf16 kernels (README,
// Abstract: exact post-softmax pooled Top-k in anchor layers, reuse of the
// index sets in the layers between), on CUDA cores:
//
//   decode_score_f32  scores of every cached key, dot products in fp64,
//                     stored as fp32 s2 = q.k log2(e)/sqrt(d) with the
//                     per-split (max, sum of exp2) statistics (fp64 sums);
//   score_pool_f32    prefill row statistics and pooled scores per
//                     (batch, kv head, query tile), fp64 dot products, one
//                     thread per query row;
//   then the shared Top-k kernel (exact fp64 band, reading fp32 inputs);
//   sparse_decode_f32 / sparse_prefill_f32: fp32 online-softmax attention
//                     over the selected rows (dense with no list).
//
// The selection scores use fp64 products so that the stored statistics and
// the Top-k kernel's fp64 band recomputation agree to far better than the
// 1e-6 near-tie rule.  These kernels are correctness-first: they keep the
// bf16 kernels' layouts and problem mapping but not their data movement.
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace kascade {

namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
template <class T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

constexpr int kF32SplitKeys = 512;   // must match the bf16 scoring split (workspace layout)

// ------------------------------------------------------------ decode scoring

// grid (splits, B * Hkv), 256 threads; warp w scores keys j0 + w, j0 + w + 8, ...
template <int D, class T>
__global__ void __launch_bounds__(256) decode_score_f32_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                              float* __restrict__ s2, float* __restrict__ m_part,
                                                              double* __restrict__ l_part, int N, int Hq, int Hkv,
                                                              int G, int splits, const int32_t* __restrict__ cand,
                                                              const int32_t* __restrict__ cand_map, int cand_lists,
                                                              int n_ctx) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int PL = D / 32;   // dims per lane
  __shared__ float wmax[8][8];
  __shared__ float hmax[8];
  __shared__ double wsum[8][8];
  __shared__ double sc[8][kF32SplitKeys];   // fp64 scores of this split (base 2)
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / Hkv, h = bh - b * Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const double c2 = 1.4426950408889634 / sqrt((double)D);
  double qv[8][PL];
#pragma unroll
  for (int g = 0; g < 8; ++g)
#pragma unroll
    for (int e = 0; e < PL; ++e) qv[g][e] = g < G ? (double)to_f(q[(size_t)(b * Hq + h * G + g) * D + lane * PL + e]) : 0.0;
  const T* kb = k + (size_t)bh * n_ctx * D;
  const int32_t* clist = nullptr;   // scored position j is key j, or key clist[j]
  if (cand) {
    int hm = cand_map ? cand_map[h] : h;
    if (hm < 0 || hm >= cand_lists) hm = 0;
    clist = cand + (size_t)(b * cand_lists + hm) * N;
  }
  const int j0 = split * kF32SplitKeys, j1 = min(N, j0 + kF32SplitKeys);
  float mloc[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) mloc[g] = -INFINITY;
  for (int j = j0 + warp; j < j1; j += 8) {
    float kr[PL];
    const int key = clist ? clist[j] : j;
#pragma unroll
    for (int e = 0; e < PL; ++e) kr[e] = to_f(kb[(size_t)key * D + lane * PL + e]);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g >= G) break;
      double dot = 0.0;
#pragma unroll
      for (int e = 0; e < PL; ++e) dot = fma(qv[g][e], (double)kr[e], dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float sv = (float)(dot * c2);
      if (lane == 0) {
        s2[(size_t)(b * Hq + h * G + g) * N + j] = sv;
        sc[g][j - j0] = dot * c2;
      }
      mloc[g] = fmaxf(mloc[g], sv);
    }
  }
  if (lane == 0)
    for (int g = 0; g < G; ++g) wmax[warp][g] = mloc[g];
  __syncthreads();
  if (threadIdx.x < G) {
    float m = -INFINITY;
    for (int w = 0; w < 8; ++w) m = fmaxf(m, wmax[w][threadIdx.x]);
    hmax[threadIdx.x] = m;
  }
  __syncthreads();
  // sum of exp2(s - m2) over the fp64 scores against the stored fp32 shift,
  // the same terms the Top-k kernel's fp64 band recomputes
  double lsum[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) lsum[g] = 0.0;
  for (int j = j0 + threadIdx.x; j < j1; j += 256)
    for (int g = 0; g < G; ++g) lsum[g] += exp2(sc[g][j - j0] - (double)hmax[g]);
  for (int g = 0; g < G; ++g) {
    double x = lsum[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) wsum[warp][g] = x;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    double l = 0.0;
    for (int w = 0; w < 8; ++w) l += wsum[w][threadIdx.x];
    const size_t row = (size_t)(b * Hq + h * G + threadIdx.x) * splits + split;
    m_part[row] = hmax[threadIdx.x];
    l_part[row] = l;
  }
}

// ------------------------------------------------------------ prefill scoring

// grid (T, B * Hkv), one thread per query row of the tile's G heads (G * 32
// <= 256 rows); keys staged in shared memory 32 at a time.
template <int D, class T>
__global__ void __launch_bounds__(256) score_pool_f32_kernel(const ScorePoolArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int KB = 32;
  extern __shared__ __align__(16) char smem[];
  float* qs = reinterpret_cast<float*>(smem);             // [256][D + 1]
  float* ks = qs + 256 * (D + 1);                         // [KB][D]
  const T* q = reinterpret_cast<const T*>(a.q);
  const T* k = reinterpret_cast<const T*>(a.k);
  const int nT = (a.N + a.tile - 1) / a.tile;
  const int t0 = a.q0 / a.tile;   // first query tile of the call (rolling chunks)
  const int t = nT - 1 - (int)blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv;
  const int G = a.G;
  const int i0 = t * a.tile, e_t = min(i0 + a.tile, a.N), rows_t = e_t - i0;
  const int r = threadIdx.x, g = r >> 5, il = r & 31;
  const bool valid = g < G && il < rows_t;
  const int pos = i0 + il;
  const int lane = threadIdx.x & 31;
  const double c2 = 1.4426950408889634 / sqrt((double)D);
  for (int e = threadIdx.x; e < G * 32 * D; e += 256) {
    const int rr = e / D, dd = e - rr * D;
    const int gi = rr >> 5, li = rr & 31;
    qs[rr * (D + 1) + dd] =
        li < rows_t ? to_f(q[((size_t)(b * a.Hq + h * G + gi) * a.Lq + (i0 - a.q0) + li) * D + dd]) : 0.f;
  }
  const float* qrow = qs + r * (D + 1);
  const T* kb = k + (size_t)bh * a.N * D;
  auto dot_key = [&](int jj) -> double {
    double acc = 0.0;
#pragma unroll 8
    for (int d = 0; d < D; ++d) acc = fma((double)qrow[d], (double)ks[jj * D + d], acc);
    return acc;
  };
  auto stage = [&](int j0) {
    __syncthreads();
    for (int e = threadIdx.x; e < KB * D; e += 256) {
      const int jj = e / D;
      ks[e] = j0 + jj < e_t ? to_f(kb[(size_t)(j0 + jj) * D + (e - jj * D)]) : 0.f;
    }
    __syncthreads();
  };
  // pass 1: row max (fp64, then stored as fp32 m2) and sum of exp2
  double mx = -INFINITY, l = 0.0;
  for (int j0 = 0; j0 < e_t; j0 += KB) {
    stage(j0);
    if (!valid) continue;
    for (int jj = 0; jj < KB && j0 + jj <= pos; ++jj) {
      const double s = dot_key(jj) * c2;
      if (s > mx) {
        if (mx != -INFINITY) l *= exp2(mx - s);
        mx = s;
      }
      l += exp2(s - mx);
    }
  }
  // the stored shift is the fp32 value; rescale the sum to it
  const float m2 = (float)mx;
  const double lsum = valid ? l * exp2(mx - (double)m2) : 1.0;
  if (valid) {
    const size_t srow = (size_t)(b * a.Hq + h * G + g) * a.Lq + (pos - a.q0);
    a.row_m2[srow] = m2;
    a.row_l[srow] = lsum;
  }
  // pass 2: pooled score of each key, summed over the rows (per head with
  // per_head: a warp holds one head's 32 rows)
  __shared__ float part[8][KB];
  const size_t prow = (size_t)chunk_pooled_len(a.N, t0, a.tile);
  const float inv = 1.0f / (float)((a.per_head ? 1 : G) * rows_t);
  for (int j0 = 0; j0 < e_t; j0 += KB) {
    stage(j0);
    for (int jj = 0; jj < KB; ++jj) {
      const int j = j0 + jj;
      float p = 0.f;
      if (valid && j <= pos) p = (float)(exp2(dot_key(jj) * c2 - (double)m2) / lsum);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      if (lane == 0) part[g][jj] = p;
    }
    __syncthreads();
    if (threadIdx.x < KB && j0 + threadIdx.x < e_t) {
      const int j = j0 + threadIdx.x;
      if (a.per_head) {
        for (int gg = 0; gg < G; ++gg)
          a.pooled[(size_t)(b * a.Hq + h * G + gg) * prow + chunk_pooled_offset(t, t0, a.tile) + j] = part[gg][threadIdx.x] * inv;
      } else {
        float sum = 0.f;
        for (int gg = 0; gg < G; ++gg) sum += part[gg][threadIdx.x];
        a.pooled[(size_t)bh * prow + chunk_pooled_offset(t, t0, a.tile) + j] = sum * inv;
      }
    }
  }
}

// ------------------------------------------------------------ attention

// the list of problem h of batch row b (NULL: dense) and its length
struct ListRef {
  const int32_t* list;
  int len;
};

__device__ __forceinline__ ListRef list_ref(const AttnArgs& a, int b, int h, int t, int e_t, bool prefill) {
  ListRef r{nullptr, 0};
  if (!a.idx) {
    r.len = prefill ? (a.causal ? e_t : a.N) : a.N;
    return r;
  }
  const int hm_raw = a.one_list ? 0 : (a.head_map ? a.head_map[h] : h);
  const bool ok = hm_raw >= 0 && hm_raw < a.n_lists;
  const int hm = ok ? hm_raw : 0;
  if (prefill) {
    const int t0 = a.q0 / a.tile;
    const int64_t row_len = chunk_row_len(a.N, t0, a.tile, a.num, a.den);
    r.list = a.idx + (size_t)(b * a.n_lists + hm) * row_len + chunk_list_offset(t, t0, a.tile, a.num, a.den);
    r.len = ok ? topk_count(e_t, a.num, a.den) : 0;
  } else {
    const int K = topk_count(a.N, a.num, a.den);
    r.list = a.idx + (size_t)(b * a.n_lists + hm) * K;
    r.len = ok ? K : 0;
  }
  return r;
}

// decode: grid B * Hp, 8 warps; warp w takes list entries w, w + 8, ...;
// lanes split d; per-warp online softmax, merged across warps in shared memory
template <int D, class T>
__global__ void __launch_bounds__(256) sparse_decode_f32_kernel(const AttnArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int PL = D / 32;
  __shared__ float sm_m[8][8], sm_l[8][8];
  __shared__ float sm_o[8][8][D];
  const int bh = blockIdx.x;
  const int b = bh / a.Hp, h = bh - b * a.Hp;
  const int G = a.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const T* q = reinterpret_cast<const T*>(a.q);
  const T* kb = reinterpret_cast<const T*>(a.k) + (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv) * a.N * D;
  const T* vb = reinterpret_cast<const T*>(a.v) + (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv) * a.N * D;
  const ListRef L = list_ref(a, b, h, 0, a.N, false);
  const float scale2 = (float)(1.4426950408889634 / sqrt((double)D));
  float qv[8][PL], o[8][PL], m[8], l[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      qv[g][e] = g < G ? to_f(q[(size_t)(b * a.Hq + h * G + g) * D + lane * PL + e]) : 0.f;
      o[g][e] = 0.f;
    }
  }
  for (int i = warp; i < L.len; i += 8) {
    const int j = L.list ? L.list[i] : i;
    float kr[PL], vr[PL];
#pragma unroll
    for (int e = 0; e < PL; ++e) {
      kr[e] = to_f(kb[(size_t)j * D + lane * PL + e]);
      vr[e] = to_f(vb[(size_t)j * D + lane * PL + e]);
    }
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g >= G) break;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < PL; ++e) dot = fmaf(qv[g][e], kr[e], dot);
#pragma unroll
      for (int s = 16; s > 0; s >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, s);
      const float sv = dot * scale2;
      const float mn = fmaxf(m[g], sv);
      const float al = m[g] == -INFINITY ? 0.f : exp2f(m[g] - mn);
      const float p = exp2f(sv - mn);
      l[g] = l[g] * al + p;
#pragma unroll
      for (int e = 0; e < PL; ++e) o[g][e] = o[g][e] * al + p * vr[e];
      m[g] = mn;
    }
  }
  for (int g = 0; g < G; ++g) {
    if (lane == 0) {
      sm_m[warp][g] = m[g];
      sm_l[warp][g] = l[g];
    }
#pragma unroll
    for (int e = 0; e < PL; ++e) sm_o[warp][g][lane * PL + e] = o[g][e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += 256) {
    const int g = e / D, dd = e - g * D;
    float M = -INFINITY;
    for (int w = 0; w < 8; ++w) M = fmaxf(M, sm_m[w][g]);
    float Ls = 0.f, acc = 0.f;
    for (int w = 0; w < 8; ++w) {
      const float f = sm_m[w][g] == -INFINITY ? 0.f : exp2f(sm_m[w][g] - M);
      Ls += f * sm_l[w][g];
      acc += f * sm_o[w][g][dd];
    }
    const size_t orow = (size_t)(b * a.Hq + h * G + g);
    reinterpret_cast<T*>(a.o)[orow * D + dd] = from_f<T>(Ls > 0.f ? acc / Ls : 0.f);
    if (dd == 0 && a.lse) a.lse[orow] = Ls > 0.f ? (M + log2f(Ls)) * (float)kLn2 : -INFINITY;
  }
}

// prefill: grid (T * row blocks, B * Hp), 256 threads = 128 rows x 2 halves
// of d; keys of the tile's list staged 32 at a time in shared memory
template <int D, class T>
__global__ void __launch_bounds__(256) sparse_prefill_f32_kernel(const AttnArgs a, int row_blocks) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int KB = 32, HD = D / 2;
  __shared__ float ks[KB][D + 4], vs[KB][D + 4];
  __shared__ int keys[KB];
  const int nT = (a.N + a.tile - 1) / a.tile;
  const int t = nT - 1 - (int)(blockIdx.x / row_blocks);
  const int rb = blockIdx.x % row_blocks;
  const int bh = blockIdx.y;
  const int b = bh / a.Hp, h = bh - b * a.Hp;
  const int G = a.G;
  const int i0 = t * a.tile, e_t = min(i0 + a.tile, a.N), rows_t = e_t - i0;
  const int row = rb * 128 + (threadIdx.x >> 1), half = threadIdx.x & 1;
  const int g = row / a.tile, il = row - g * a.tile;
  const bool valid = g < G && il < rows_t;
  const int pos = i0 + il;
  const size_t slab = (size_t)kv_slab_of(b, h * G, a.Hkv, a.Gkv);
  const T* kb = reinterpret_cast<const T*>(a.k) + slab * a.N * D;
  const T* vb = reinterpret_cast<const T*>(a.v) + slab * a.N * D;
  const ListRef L = list_ref(a, b, h, t, e_t, true);
  const bool causal = a.idx != nullptr || a.causal;
  const float scale2 = (float)(1.4426950408889634 / sqrt((double)D));
  float qv[HD], o[HD];
  const T* qr = reinterpret_cast<const T*>(a.q) + ((size_t)(b * a.Hq + h * G + (valid ? g : 0)) * a.Lq +
                                                   (valid ? pos - a.q0 : 0)) * D + half * HD;
#pragma unroll
  for (int e = 0; e < HD; ++e) {
    qv[e] = valid ? to_f(qr[e]) : 0.f;
    o[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int c0 = 0; c0 < L.len; c0 += KB) {
    __syncthreads();
    if (threadIdx.x < KB) keys[threadIdx.x] = c0 + threadIdx.x < L.len ? (L.list ? L.list[c0 + threadIdx.x] : c0 + threadIdx.x) : -1;
    __syncthreads();
    for (int e = threadIdx.x; e < KB * D; e += 256) {
      const int jj = e / D, dd = e - jj * D;
      const int key = keys[jj];
      ks[jj][dd] = key >= 0 ? to_f(kb[(size_t)key * D + dd]) : 0.f;
      vs[jj][dd] = key >= 0 ? to_f(vb[(size_t)key * D + dd]) : 0.f;
    }
    __syncthreads();
    for (int jj = 0; jj < KB; ++jj) {
      const int key = keys[jj];
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < HD; ++e) dot = fmaf(qv[e], ks[jj][half * HD + e], dot);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      const bool vis = valid && key >= 0 && (!causal || key <= pos);
      if (!vis) continue;
      const float sv = dot * scale2;
      const float mn = fmaxf(m, sv);
      const float al = m == -INFINITY ? 0.f : exp2f(m - mn);
      const float p = exp2f(sv - mn);
      l = l * al + p;
#pragma unroll
      for (int e = 0; e < HD; ++e) o[e] = o[e] * al + p * vs[jj][half * HD + e];
      m = mn;
    }
  }
  if (!valid) return;
  const size_t orow = (size_t)(b * a.Hq + h * G + g) * a.Lq + (pos - a.q0);
  T* od = reinterpret_cast<T*>(a.o) + orow * D + half * HD;
#pragma unroll
  for (int e = 0; e < HD; ++e) od[e] = from_f<T>(l > 0.f ? o[e] / l : 0.f);
  if (half == 0 && a.lse) a.lse[orow] = l > 0.f ? (m + log2f(l)) * (float)kLn2 : -INFINITY;
}

// element type dispatch: fp16 or fp32 inputs
template <int D, class F>
cudaError_t by_type(bool half, F&& f) {
  return half ? f((__half*)nullptr) : f((float*)nullptr);
}

}  // namespace

cudaError_t launch_decode_score_f32(const DecodeScoreArgs& a, bool half, cudaStream_t stream) {
  const int splits = (a.N + kF32SplitKeys - 1) / kF32SplitKeys;
  const dim3 grid(splits, a.B * a.Hkv);
  const int n_ctx = a.cand ? a.n_ctx : a.N;
  auto go = [&](auto tag) -> cudaError_t {
    using T = std::remove_pointer_t<decltype(tag)>;
    const T* q = reinterpret_cast<const T*>(a.q);
    const T* k = reinterpret_cast<const T*>(a.k);
    if (a.D == 128)
      return launch_ex(decode_score_f32_kernel<128, T>, grid, dim3(256), 0, stream, (a.flags & 1) != 0, 1, q, k, a.s2,
                       a.m_part, a.l_part, a.N, a.Hq, a.Hkv, a.G, splits, a.cand, a.cand_map, a.cand_lists, n_ctx);
    return launch_ex(decode_score_f32_kernel<64, T>, grid, dim3(256), 0, stream, (a.flags & 1) != 0, 1, q, k, a.s2,
                     a.m_part, a.l_part, a.N, a.Hq, a.Hkv, a.G, splits, a.cand, a.cand_map, a.cand_lists, n_ctx);
  };
  return by_type<0>(half, go);
}

cudaError_t launch_score_pool_f32(const ScorePoolArgs& a, bool half, cudaStream_t stream) {
  const int T = (a.N + a.tile - 1) / a.tile - a.q0 / a.tile;   // the call's query tiles
  const dim3 grid(T, a.B * a.Hkv);
  auto go = [&](auto tag) -> cudaError_t {
    using E = std::remove_pointer_t<decltype(tag)>;
    if (a.D == 128) {
      const size_t smem = (size_t)(256 * 129 + 32 * 128) * 4;
      const cudaError_t e =
          ensure_func_attrs(reinterpret_cast<const void*>(score_pool_f32_kernel<128, E>), smem, false);
      if (e != cudaSuccess) return e;
      return launch_ex(score_pool_f32_kernel<128, E>, grid, dim3(256), smem, stream, (a.flags & 1) != 0, 1, a);
    }
    const size_t smem = (size_t)(256 * 65 + 32 * 64) * 4;
    const cudaError_t e = ensure_func_attrs(reinterpret_cast<const void*>(score_pool_f32_kernel<64, E>), smem, false);
    if (e != cudaSuccess) return e;
    return launch_ex(score_pool_f32_kernel<64, E>, grid, dim3(256), smem, stream, (a.flags & 1) != 0, 1, a);
  };
  return by_type<0>(half, go);
}

cudaError_t launch_sparse_decode_f32(const AttnArgs& a, bool half, cudaStream_t stream) {
  const dim3 grid(a.B * a.Hp);
  auto go = [&](auto tag) -> cudaError_t {
    using E = std::remove_pointer_t<decltype(tag)>;
    if (a.D == 128)
      return launch_ex(sparse_decode_f32_kernel<128, E>, grid, dim3(256), 0, stream, (a.flags & 1) != 0, 1, a);
    return launch_ex(sparse_decode_f32_kernel<64, E>, grid, dim3(256), 0, stream, (a.flags & 1) != 0, 1, a);
  };
  return by_type<0>(half, go);
}

cudaError_t launch_sparse_prefill_f32(const AttnArgs& a, bool half, cudaStream_t stream) {
  const int T = (a.N + a.tile - 1) / a.tile - a.q0 / a.tile;   // the call's query tiles
  const int row_blocks = (a.G * a.tile + 127) / 128;
  const dim3 grid(T * row_blocks, a.B * a.Hp);
  auto go = [&](auto tag) -> cudaError_t {
    using E = std::remove_pointer_t<decltype(tag)>;
    if (a.D == 128)
      return launch_ex(sparse_prefill_f32_kernel<128, E>, grid, dim3(256), 0, stream, (a.flags & 1) != 0, 1, a,
                       row_blocks);
    return launch_ex(sparse_prefill_f32_kernel<64, E>, grid, dim3(256), 0, stream, (a.flags & 1) != 0, 1, a,
                     row_blocks);
  };
  return by_type<0>(half, go);
}

}  // namespace kascade
