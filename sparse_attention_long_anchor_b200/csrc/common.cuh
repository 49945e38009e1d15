// Shared device helpers of the Kascade CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

namespace kascade {

constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLn2 = 0.6931471805599453;

// ---------------------------------------------------------------------------
// tile arithmetic (prefill): e_t = min(32 (t+1), N), k_t = ceil(num e_t / den)

__host__ __device__ inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

__host__ __device__ inline int topk_count(int64_t e, int num, int den) {
  return e <= 0 ? 0 : (int)ceil_div64((int64_t)num * e, den);
}

// sum_{i=0}^{n-1} floor((a i + b) / m) for a, b >= 0, m > 0, n >= 0.
// Reduces a and b modulo m, then counts lattice points under the line by
// exchanging the roles of the axes (Euclid-like recursion); O(log) steps.
__host__ __device__ inline int64_t floor_sum(int64_t n, int64_t m, int64_t a, int64_t b) {
  int64_t total = 0;
  while (n > 0) {
    if (a >= m) {
      total += (n * (n - 1) / 2) * (a / m);
      a %= m;
    }
    if (b >= m) {
      total += n * (b / m);
      b %= m;
    }
    const int64_t y = a * n + b;   // the line a x + b at x = n
    if (y < m) break;
    // points (x, j) with 1 <= j <= floor(y/m) - ... : swap axes
    n = y / m;
    b = y % m;
    const int64_t t = m;
    m = a;
    a = t;
  }
  return total;
}

// Start of tile t's list inside one (batch, kv head) index row: sum over
// the full tiles t' < t of ceil(num * tile (t'+1) / den).
__host__ __device__ inline int64_t tile_list_offset(int64_t t, int tile, int num, int den) {
  // ceil(A (i+1) / Q) = floor((A i + A + Q - 1) / Q), A = num * tile, Q = den
  const int64_t A = (int64_t)num * tile;
  return floor_sum(t, den, A, A + den - 1);
}

// Start of tile t's pooled-score row: sum_{t' < t} e_t' = tile * t (t+1) / 2.
__host__ __device__ inline int64_t tile_pooled_offset(int64_t t, int tile) {
  return (int64_t)tile * t * (t + 1) / 2;
}

// Rolling (chunked) prefill: the query rows are the last Lq positions
// [q0, N) of an N-key context, q0 a multiple of the tile, so the call covers
// tiles t0 = q0 / tile .. T - 1.  Index lists and pooled rows of such a call
// hold only those tiles; offsets are relative to tile t0 (t0 = 0 for a full
// prefill).
__host__ __device__ inline int64_t chunk_list_offset(int64_t t, int64_t t0, int tile, int num, int den) {
  return tile_list_offset(t, tile, num, den) - tile_list_offset(t0, tile, num, den);
}
__host__ __device__ inline int64_t chunk_pooled_offset(int64_t t, int64_t t0, int tile) {
  return tile_pooled_offset(t, tile) - tile_pooled_offset(t0, tile);
}
// length of one (batch row, list) index row / pooled row of the chunk
__host__ __device__ inline int64_t chunk_row_len(int N, int64_t t0, int tile, int num, int den) {
  const int64_t T = (N + tile - 1) / tile;
  return chunk_list_offset(T - 1, t0, tile, num, den) + topk_count(N, num, den);
}
__host__ __device__ inline int64_t chunk_pooled_len(int N, int64_t t0, int tile) {
  const int64_t T = (N + tile - 1) / tile;
  return chunk_pooled_offset(T - 1, t0, tile) + N;
}

// ---------------------------------------------------------------------------
// bf16 helpers

// 2^x as the single MUFU instruction ex2.approx.ftz.f32 (relative error
// about 2^-22; subnormal results flush to zero).  For epilogues that are
// bound by instruction issue; exp2f adds range handling around the same
// instruction.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// ---------------------------------------------------------------------------
// warp-level tensor-core MMA (m16n8k16, bf16 in, fp32 accumulate)

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t smem_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr));
}

// 8x8 b16 transpose across the warp: lane (g, c) passes row g, columns
// 2c and 2c+1, and receives row 2c and 2c+1 of column g
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(r) : "r"(x));
  return r;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared async copy; src_bytes = 0 zero-fills the line.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// block-wide inclusive scan of one int per thread (NT threads, NT % 32 == 0)

template <int NT>
__device__ __forceinline__ int block_inclusive_scan(int x, int* warp_buf /* >= NT/32 + 1 ints */,
                                                    int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? warp_buf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) warp_buf[lane] = w;
  }
  __syncthreads();
  if (warp > 0) x += warp_buf[warp - 1];
  if (total) *total = warp_buf[NT / 32 - 1];
  __syncthreads();
  return x;
}

}  // namespace kascade

namespace kascade {

// ---------------------------------------------------------------------------
// mbarriers and bulk (TMA) copies

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

// make barrier initialisation visible to the async proxy and the cluster
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of phase `parity` of an mbarrier (never suspends the
// thread, for polling several barriers).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier: gives up after about
// 2^32 SM clocks (~2 s) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << 32)) return false;
  }
  return true;
}

// Untiled bulk copy global -> this CTA's shared memory, completing on `bar`
// (both addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Arrive on `bar` once all of this thread's earlier cp.async copies have
// landed (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}

// ---------------------------------------------------------------------------
// distributed shared memory within a thread-block cluster

__device__ __forceinline__ uint32_t mapa(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// asynchronous store into another CTA's shared memory, completing on that
// CTA's mbarrier (both addresses in the shared::cluster window)
__device__ __forceinline__ void st_async_v4(uint32_t raddr, float4 v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];\n" ::"r"(raddr),
      "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t raddr, float2 v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];\n" ::"r"(raddr),
               "f"(v.x), "f"(v.y), "r"(rbar)
               : "memory");
}

__device__ __forceinline__ void st_async_u32(uint32_t raddr, uint32_t v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];\n" ::"r"(raddr), "r"(v),
               "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_u64(uint32_t raddr, unsigned long long v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];\n" ::"r"(raddr), "l"(v),
               "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_v4u(uint32_t raddr, uint4 v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];\n" ::"r"(
                   raddr),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(rbar)
               : "memory");
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// bounded wait (about 2^32 SM clocks) for data other CTAs of the cluster
// stored into this CTA
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (clock64() - t0 > (1ll << 32)) return false;
  }
  return true;
}

// Record a device-side failure (a bounded wait that gave up).
__device__ __forceinline__ void raise_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

}  // namespace kascade

namespace kascade {

// Programmatic dependent launch: wait for the previous kernel on the stream
// (and the visibility of its writes); allow the next one to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

}  // namespace kascade

namespace kascade {

// Set a kernel's dynamic shared-memory limit (and, for clusters above 8
// CTAs, the non-portable cluster size) once per device: the attributes stay
// with the function in the device's context, so repeating the driver calls
// on every launch only adds host latency.  The limit is raised when a launch
// needs more than any earlier one on the device.  (A device reset clears the
// attributes; the cache assumes none happens while the library is in use.)
inline cudaError_t ensure_func_attrs(const void* fn, size_t smem, bool nonportable_cluster) {
  struct Entry {
    const void* fn;
    int dev;
    long long smem;
    bool nonportable;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  size_t i = 0;
  while (i < done.size() && !(done[i].fn == fn && done[i].dev == dev)) ++i;
  if (i == done.size()) done.push_back({fn, dev, -1, false});
  if ((long long)smem > done[i].smem) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    done[i].smem = (long long)smem;
  }
  if (nonportable_cluster && !done[i].nonportable) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    done[i].nonportable = true;
  }
  return cudaSuccess;
}

// Host-side launch with optional programmatic dependent launch and a
// runtime cluster size (1 = none).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             bool pdl, int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace kascade
