// Shared device helpers: storage types, conversions, warp/block reductions.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <math.h>

#include <mutex>
#include <unordered_map>
#include <utility>

namespace fm {

typedef __nv_bfloat16 bf16;

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// (value, index) argmax with ties to the lowest index; NaN never wins
// because every comparison with NaN is false.
struct ArgMax {
  float v;
  int i;
};
__device__ __forceinline__ bool am_better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}
__device__ __forceinline__ ArgMax warp_argmax(ArgMax a) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float v = __shfl_xor_sync(0xffffffffu, a.v, o);
    int i = __shfl_xor_sync(0xffffffffu, a.i, o);
    if (am_better(v, i, a.v, a.i)) { a.v = v; a.i = i; }
  }
  return a;
}

// Block-wide reductions; `sh` needs 32 slots.  Every thread gets the result.
__device__ __forceinline__ float block_sum(float v, float* sh) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  v = (lane < nw) ? sh[lane] : 0.f;
  v = warp_sum(v);
  return v;
}
__device__ __forceinline__ double block_sum_d(double v, double* sh) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  v = (lane < nw) ? sh[lane] : 0.0;
  v = warp_sum_d(v);
  return v;
}
__device__ __forceinline__ float block_max(float v, float* sh) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  v = (lane < nw) ? sh[lane] : -INFINITY;
  v = warp_max(v);
  return v;
}
__device__ __forceinline__ ArgMax block_argmax(ArgMax a, float* shv, int* shi) {
  int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  a = warp_argmax(a);
  __syncthreads();
  if (lane == 0) { shv[w] = a.v; shi[w] = a.i; }
  __syncthreads();
  if (lane < nw) { a.v = shv[lane]; a.i = shi[lane]; } else { a.v = -INFINITY; a.i = 0x7fffffff; }
  a = warp_argmax(a);
  return a;
}

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may start while the previous kernel on the
// stream is still running: pdl_wait() blocks until that kernel has finished
// and its memory is visible; pdl_trigger() lets the next kernel launch once
// every CTA of this one has started.  Both are no-ops without the attribute.
// Every kernel here calls pdl_wait() before its first global write and
// before reading anything an earlier kernel produced.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Thread-block clusters (a launch without a cluster is a cluster of one CTA):
// this CTA's rank and the cluster's size, a barrier of every thread of the
// cluster, and distributed shared memory
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}
// All threads of every CTA of the cluster must reach it (in the GEMM, only
// at kernel start, before anything can give up).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t local, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local), "r"(rank));
  return a;
}
__device__ __forceinline__ float dsmem_ld(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
// Launch with the programmatic stream-serialization attribute.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// As launch_pdl, in clusters of `cluster` CTAs along x (grid.x a multiple).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t st, unsigned cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device):
// the call is host-side only and would otherwise cost host time per launch.
inline cudaError_t set_smem_once_ptr(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, unsigned long long> done;  // bit per device id < 64
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long& m = done[kernel];
  if (m & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) m |= bit;
  return e;
}
template <typename F>
inline cudaError_t set_smem_once(F* kernel, int bytes) {
  return set_smem_once_ptr((const void*)kernel, bytes);
}

// Cross-CTA handoffs: the writing CTA orders its threads' stores with a CTA
// barrier, then one thread publishes them with a release (cumulative over
// what the barrier ordered before it); the reading CTA's one thread acquires
// and a CTA barrier orders the other threads' reads after it.
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void red_add_release_gpu(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *(uint32_t*)&v;
}

// GELU, tanh form: 0.5 u (1 + tanh(z)) with z = sqrt(2/pi) (u + 0.044715 u^3).
// Since 1 + tanh(z) = 2 / (1 + e^{-2z}), this is u / (1 + e^{-2z}): one
// exponential and one fast division.  The exponent is clamped at 80
// (e^80 < 2^126, the fast division's range; the quotient there is below
// |u| * 2e-35 anyway).
__device__ __forceinline__ float gelu_tanh(float u) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float z = k0 * (u + 0.044715f * u * u * u);
  return __fdividef(u, 1.f + __expf(fminf(-2.f * z, 80.f)));
}
__device__ __forceinline__ float silu(float u) { return u / (1.f + expf(-u)); }

}  // namespace fm
