// Tensor-core weight GEMM for sm_100a: tcgen05.mma with TMEM accumulators,
// operands staged in shared memory by TMA.
//
// Y[M][N] = A[M][K] . W[N][K]^T with both operands K-major bf16 and fp32
// accumulation.  The drafter's GEMMs stream a large weight through a few
// activation rows (M = 16 at concurrency 1), so the weight takes the MMA's
// 128-row side ("swap-AB"): each tile is D[128 features][BN rows] =
// W_tile[128][K] . A_tile[BN][K]^T.  Few output tiles (x.E has 16 at d=2048)
// are spread over all SMs by splitting K; the last CTA to finish a tile
// (arrival counter, no waiting) sums the fp32 partials in split order and
// runs the epilogue, so results do not depend on scheduling.
//
// Roles per CTA (192 threads, one CTA per SM, persistent over work units):
//   warp 0     TMA producer (one lane) filling a ring of smem stages
//   warp 1     TMEM allocator and MMA issuer (one lane)
//   warps 2-5  epilogue: TMEM -> registers -> epilogue functor
// Two TMEM accumulators let the epilogue of one unit overlap the MMAs of the
// next.  Every mbarrier wait is bounded in time; on expiry the CTA records
// an error code, lets in-flight copies land, frees its TMEM and exits.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>

#include <type_traits>
#include <vector>

#include "fm_common.cuh"

namespace fm {

constexpr int TC_BM = 128;       // weight rows (output features) per tile
constexpr int TC_BK = 64;        // reduction elements per stage: one 128-byte swizzle row
constexpr int TC_THREADS = 192;
constexpr unsigned long long TC_TIMEOUT_NS = 2000000000ull;
constexpr int TC_ERR_TIMEOUT = 1;

// ------------------------------------------------------------------ host-side maps
struct TcMap {
  bool valid = false;
  CUtensorMap map;
  int N = 0, Kd = 0;
};
struct TcMaps {
  TcMap embed, lm, fc, kv_all;   // kv_all: every block's key and value weights stacked
  std::vector<TcMap> qkv, kv, o, up, down;
  int* err = nullptr;  // device error word shared by all tensor-core launches
};

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// As mbar_try, but a thread whose phase is not complete yet is suspended
// until the phase completes or about 20 us have passed (the time hint), so
// a waiting warp takes no issue slots from the warps that share its
// scheduler.
__device__ __forceinline__ bool mbar_try_suspend(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity; false when it timed out or
// another role of the CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = gtimer();
  while (!mbar_try_suspend(bar, parity)) {
    if (*abort) return false;
    if (gtimer() - t0 > TC_TIMEOUT_NS) {
      *abort = 1;
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(dst),
      "l"((unsigned long long)map), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// L2 prefetch of one tile of a 2D tensor map (no data reaches shared memory).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   (unsigned long long)map),
               "r"(c0), "r"(c1)
               : "memory");
}
// Untiled bulk copy global -> shared (addresses 16-byte aligned, bytes a
// multiple of 16), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"((unsigned long long)src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane; the wait is part of
// the same statement so the registers are complete when it returns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Shared-memory matrix descriptor: K-major operand written by TMA with the
// 128-byte swizzle, rows of 64 bf16, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128, N = BN.
template <int BN>
__host__ __device__ constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// ------------------------------------------------------------------ epilogue for the LM head
// Per activation row and 128-token tile: the largest logit and its lowest
// index.  The logits themselves never reach HBM.
struct EpiArgmax {
  float* part_v;  // [M][n_part]
  int* part_i;
  int n_part;
};
template <class E>
struct is_argmax : std::false_type {};
template <>
struct is_argmax<EpiArgmax> : std::true_type {};

struct TcArgs {
  int M, N, Kd;
  int n_tiles, m_tiles, splits, k_blocks, units;
  float* partial;       // [splits][tiles][128][BN] fp32 (splits > 1)
  unsigned* tile_cnt;   // [tiles], zero between launches
  int* err;
  // B operand computed in the kernel as LN0(x) (1 + scale) + shift (bf16)
  const float* ln_x;    // [M_ln][Kd] fp32
  const float* ln_shift;
  const float* ln_scale;
  int M_ln;             // rows [0, M_ln) come from x; rows [M_ln, M) are copied from ln_extra
  const bf16* ln_extra; // [M - M_ln][Kd] bf16, already normalised
  int b_kb;             // k-blocks of the shared-memory-resident B operand
  // > 1: the grid runs in clusters of this many CTAs, one unit each, that
  // are the K splits of one output tile (one activation tile); their partial
  // tiles are summed through distributed shared memory, not global memory
  int cluster = 0;
};

// Ring depth: "deep" (about 200 KB, one CTA per SM) for long weight streams
// per CTA; "shallow" (about 100 KB) for short ones, so that two CTAs -- the
// running GEMM's and the next GEMM's, launched early -- share an SM and the
// next weight stream starts while the current one drains.
template <int BN>
__host__ __device__ constexpr int tc_stages(bool deep) {
  return deep ? ((200 * 1024) / (TC_BM * TC_BK * 2 + BN * TC_BK * 2) > 12
                     ? 12
                     : (200 * 1024) / (TC_BM * TC_BK * 2 + BN * TC_BK * 2))
              : (100 * 1024) / (TC_BM * TC_BK * 2 + BN * TC_BK * 2);
}

// barriers and flags of a GEMM CTA (after the operand tiles)
constexpr int TC_BAR_BYTES = 256;

// Whether split-K GEMMs of one activation tile may run as clusters that
// reduce in distributed shared memory (diagnostic switch, set by the host).
inline bool tc_cluster_ok = true;

template <int BN, int STAGES_>
struct TcCfg {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;  // 16 KB
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = STAGES_;
  static constexpr int TMEM_COLS = (2 * BN) < 32 ? 32 : 2 * BN;
  static constexpr int SMEM = STAGES * STAGE + 1024 /*align*/ + TC_BAR_BYTES + 8 * BN * 4;
};

template <int BN, class Epi>
__device__ __forceinline__ void tc_finish_chunk(const Epi& epi, const TcArgs& a, int n0, int m0,
                                                int r, int j0, const float* v, float* red_v,
                                                int* red_i, int q) {
  const int n = n0 + r;
  if constexpr (is_argmax<Epi>::value) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      // a NaN logit enters as "no candidate", so it never wins (not even
      // against -inf) and cannot stick in the shuffle tree
      const bool ok = n < a.N && v[j] == v[j];
      ArgMax am{ok ? v[j] : -INFINITY, ok ? n : 0x7fffffff};
      am = warp_argmax(am);
      if (lane == 0) {
        red_v[q * BN + j0 + j] = am.v;
        red_i[q * BN + j0 + j] = am.i;
      }
    }
  } else if constexpr (has_chunk16<Epi>::value) {
    if (n >= a.N) return;
    const int mb = m0 + j0;
    epi.chunk16(mb, n, v, a.M - mb < 16 ? a.M - mb : 16);
  } else {
    if (n >= a.N) return;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int m = m0 + j0 + j;
      if (m < a.M) epi(m, n, v[j]);
    }
  }
}

// ---- cluster-scope barrier arrivals (the cluster helpers are in fm_common.cuh)
// One arrival, with release at cluster scope, on the barrier at `local` in
// CTA `rank`.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t local, uint32_t rank) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   dsmem_addr(local, rank))
               : "memory");
}
// Bounded wait, with acquire at cluster scope, for the phase of parity 0.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, unsigned long long limit_ns) {
  const unsigned long long t0 = gtimer();
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(0u), "r"(20000u)
        : "memory");
    if (ok) return true;
    if (gtimer() - t0 > limit_ns) return false;
  }
}

// Rows m .. m + count - 1 (count <= 16) of feature n0 + r through the
// epilogue (not the argmax epilogue).
template <class Epi>
__device__ __forceinline__ void tc_finish_rows(const Epi& epi, const TcArgs& a, int n0, int r, int m,
                                               int count, const float* v) {
  const int n = n0 + r;
  if (n >= a.N) return;
  if constexpr (has_chunk16<Epi>::value) {
    epi.chunk16(m, n, v, count);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < count) epi(m + j, n, v[j]);
  }
}

// Split-K reduction of one output tile inside its cluster (a.cluster CTAs,
// CTA z of the cluster holds K split z).  Every CTA stores its partial tile
// [BN][128] fp32 in its own shared memory `sP`, arrives on every CTA's
// `crdy`, waits for its own, then sums rows [z M / S, (z + 1) M / S) over
// the cluster's tiles in split order (as the global-memory reduction does)
// and finishes them; last, it arrives on every CTA's `cfree` and waits for
// its own, so no CTA leaves while another may still read its tile.  A CTA
// whose accumulator never arrived (`have` false) still makes every arrival,
// so the others' waits end; it returns false and writes nothing.
template <int BN, class Epi>
__device__ __forceinline__ bool tc_cluster_finish(const Epi& epi, const TcArgs& a, int n0, int r,
                                                  int et, uint32_t taddr, bool have, float* sP,
                                                  uint64_t* crdy, uint64_t* cfree,
                                                  volatile int* s_flag) {
  const uint32_t S = (uint32_t)a.cluster, z = cluster_rank();
  float v[16];
  if (have) {
    tc_fence_after();
    for (int j0 = 0; j0 < BN; j0 += 16) {
      tmem_ld16(taddr + j0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) sP[(j0 + j) * TC_BM + r] = v[j];
    }
    tc_fence_before();
  }
  named_sync(1, 128);   // every thread's stores before the releasing arrivals
  if (et == 0) {
    for (uint32_t p = 0; p < S; ++p) mbar_arrive_cluster(smem_u32(crdy), p);
    *s_flag = mbar_wait_cluster(smem_u32(crdy), TC_TIMEOUT_NS) ? 1 : 0;
  }
  named_sync(1, 128);
  const bool ok = have && *s_flag != 0;
  if (ok) {
    (void)mbar_wait_cluster(smem_u32(crdy), TC_TIMEOUT_NS);   // complete: acquire for this thread
    const int lo = (int)(z * (uint32_t)a.M / S), hi = (int)((z + 1) * (uint32_t)a.M / S);
    const uint32_t mine = smem_u32(sP) + (uint32_t)r * 4u;
    for (int m = lo; m < hi; m += 16) {
      const int count = hi - m < 16 ? hi - m : 16;
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.f;
      for (uint32_t p0 = 0; p0 < S; p0 += 4) {
        // four splits' loads in flight; sums stay in split order
        float t[4][16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t pa = dsmem_addr(mine, p0 + u < S ? p0 + u : 0);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            t[u][j] = (p0 + u < S && j < count) ? dsmem_ld(pa + (uint32_t)((m + j) * TC_BM * 4)) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (p0 + u < S)
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += t[u][j];
      }
      tc_finish_rows(epi, a, n0, r, m, count, v);
    }
  }
  named_sync(1, 128);   // this CTA's reads of the other tiles are done
  if (et == 0) {
    for (uint32_t p = 0; p < S; ++p) mbar_arrive_cluster(smem_u32(cfree), p);
    // longer than any wait before it, so a CTA that gave up late still
    // finds the others resident when it arrives
    if (!mbar_wait_cluster(smem_u32(cfree), 4ull * TC_TIMEOUT_NS)) *s_flag = 0;
  }
  named_sync(1, 128);
  return ok && *s_flag != 0;
}

// Modulated LayerNorm of the activation rows, written straight into the
// shared-memory B operand (128-byte swizzle, K-major, one BN x 64 tile per
// k-block) by the 128 epilogue threads before any accumulator is ready.
// Rows [0, M_ln) are LN0(x)(1 + scale) + shift with fp32 statistics (two
// passes, eight threads per row); rows [M_ln, M) are copied from ln_extra;
// rows past M are zero.
template <int BN>
__device__ __forceinline__ void tc_ln_fill(uint8_t* sB, const TcArgs& a, int kb0, int nkb, int et,
                                           float* s_stat) {
  const int Kd = a.Kd;
  const int part = et & 7;
  for (int r0 = 0; r0 < a.M_ln; r0 += 16) {
    const int row = r0 + (et >> 3);
    const bool valid = row < a.M_ln;
    const float* xr = a.ln_x + (size_t)row * Kd;
    float s = 0.f;
    if (valid)
      for (int c = part * 4; c < Kd; c += 32) {
        const float4 v = *(const float4*)(xr + c);
        s += (v.x + v.y) + (v.z + v.w);
      }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)Kd;
    float q = 0.f;
    if (valid)
      for (int c = part * 4; c < Kd; c += 32) {
        const float4 v = *(const float4*)(xr + c);
        const float a0 = v.x - mean, a1 = v.y - mean, a2 = v.z - mean, a3 = v.w - mean;
        q += (a0 * a0 + a1 * a1) + (a2 * a2 + a3 * a3);
      }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (part == 0 && valid) {
      s_stat[row] = mean;
      s_stat[BN + row] = rsqrtf(q / (float)Kd + 1e-6f);
    }
  }
  named_sync(1, 128);
  constexpr int B_BYTES = BN * TC_BK * 2;
  for (int idx = et; idx < nkb * BN * 8; idx += 128) {
    const int kbi = idx / (BN * 8), rem = idx - kbi * (BN * 8);
    const int row = rem >> 3, ch = rem & 7;
    const int col = (kb0 + kbi) * TC_BK + ch * 8;
    uint4 packed = make_uint4(0, 0, 0, 0);
    if (col < Kd) {
      if (row < a.M_ln) {
        const float mean = s_stat[row], rstd = s_stat[BN + row];
        const float* xr = a.ln_x + (size_t)row * Kd + col;
        const float4 x0 = *(const float4*)xr, x1 = *(const float4*)(xr + 4);
        const float4 c0 = *(const float4*)(a.ln_scale + col), c1 = *(const float4*)(a.ln_scale + col + 4);
        const float4 h0 = *(const float4*)(a.ln_shift + col), h1 = *(const float4*)(a.ln_shift + col + 4);
        packed.x = pack_bf16x2((x0.x - mean) * rstd * (1.f + c0.x) + h0.x, (x0.y - mean) * rstd * (1.f + c0.y) + h0.y);
        packed.y = pack_bf16x2((x0.z - mean) * rstd * (1.f + c0.z) + h0.z, (x0.w - mean) * rstd * (1.f + c0.w) + h0.w);
        packed.z = pack_bf16x2((x1.x - mean) * rstd * (1.f + c1.x) + h1.x, (x1.y - mean) * rstd * (1.f + c1.y) + h1.y);
        packed.w = pack_bf16x2((x1.z - mean) * rstd * (1.f + c1.z) + h1.z, (x1.w - mean) * rstd * (1.f + c1.w) + h1.w);
      } else if (row < a.M) {
        packed = *(const uint4*)(a.ln_extra + (size_t)(row - a.M_ln) * Kd + col);
      }
    }
    *(uint4*)(sB + kbi * B_BYTES + row * 128 + ((ch ^ (row & 7)) << 4)) = packed;
  }
  // generic-proxy writes must be visible to the tensor core's async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// CL: launched in clusters of a.cluster CTAs that reduce their split-K
// partials in distributed shared memory (a separate instantiation, so the
// other launches carry none of its code)
template <int BN, int STAGES, bool LNB, class Epi, bool CL = false>
__global__ void __launch_bounds__(TC_THREADS, 1)
k_tc_gemm(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapA,
          TcArgs a, Epi epi) {
  static_assert(!CL || (!LNB && !is_argmax<Epi>::value), "cluster reduction: plain epilogues only");
  using C = TcCfg<BN, STAGES>;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // ring of A (weight) tiles, then B: a ring of activation tiles, or with
  // LNB one resident tile per k-block computed in the kernel
  uint8_t* sA = base;
  uint8_t* sB = base + C::STAGES * C::A_BYTES;
  const int data_bytes = LNB ? C::STAGES * C::A_BYTES + a.b_kb * C::B_BYTES : C::STAGES * C::STAGE;
  uint64_t* bars = (uint64_t*)(base + data_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* bready = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(bready + 1);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  int* s_last = (int*)(tmem_slot + 2);
  volatile int* s_ok = (volatile int*)(tmem_slot + 3);  // two slots
  float* red_v = (float*)(base + data_bytes + TC_BAR_BYTES);
  // cluster reduction barriers: in the argmax scratch, which CL kernels
  // never use (8-byte aligned)
  uint64_t* crdy = (uint64_t*)red_v;
  uint64_t* cfree = crdy + 1;
  int* red_i = (int*)(red_v + 4 * BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 128);
    }
    mbar_init(smem_u32(bready), 128);
    if constexpr (CL) {
      mbar_init(smem_u32(crdy), (uint32_t)a.cluster);
      mbar_init(smem_u32(cfree), (uint32_t)a.cluster);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // every CTA's barriers are initialised before another CTA can arrive on them
  if constexpr (CL) cluster_sync_all();
  const uint32_t tmem = *tmem_slot;
  const int tiles = a.n_tiles * a.m_tiles;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&mapW) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&mapA) : "memory");
      int stage = 0;
      uint32_t phase = 0;
      // Weights do not depend on earlier kernels: the first unit's weight
      // tiles go out before the dependency wait, the activation tiles after.
      int npre = 0;
      {
        const int u = blockIdx.x;
        const int mt = u % a.m_tiles, rest = u / a.m_tiles;
        const int z = rest % a.splits, nt = rest / a.splits;
        const int kb0 = (int)((long)z * a.k_blocks / a.splits);
        const int kb1 = (int)((long)(z + 1) * a.k_blocks / a.splits);
        npre = min(C::STAGES, kb1 - kb0);
        for (int i = 0; i < npre; ++i) {
          const uint32_t fb = smem_u32(&full[i]);
          mbar_expect_tx(fb, LNB ? C::A_BYTES : C::STAGE);
          tma_load_2d(smem_u32(sA + i * C::A_BYTES), &mapW, (kb0 + i) * TC_BK, nt * TC_BM, fb);
        }
        pdl_wait();
        if (!LNB)
          for (int i = 0; i < npre; ++i)
            tma_load_2d(smem_u32(sB + i * C::B_BYTES), &mapA, (kb0 + i) * TC_BK, mt * BN,
                        smem_u32(&full[i]));
        stage = npre % C::STAGES;
        phase = (npre == C::STAGES) ? 1u : 0u;
      }
      for (int u = blockIdx.x; u < a.units && !*abort; u += gridDim.x) {
        const int mt = u % a.m_tiles, rest = u / a.m_tiles;
        const int z = rest % a.splits, nt = rest / a.splits;
        const int kb0 = (int)((long)z * a.k_blocks / a.splits) + (u == (int)blockIdx.x ? npre : 0);
        const int kb1 = (int)((long)(z + 1) * a.k_blocks / a.splits);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort)) break;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, LNB ? C::A_BYTES : C::STAGE);
          tma_load_2d(smem_u32(sA + stage * C::A_BYTES), &mapW, kb * TC_BK, nt * TC_BM, fb);
          if (!LNB) tma_load_2d(smem_u32(sB + stage * C::B_BYTES), &mapA, kb * TC_BK, mt * BN, fb);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16<BN>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      // resident B starts at the first unit's k-block (every unit of a CTA
      // shares it: one unit per CTA, or no split of K)
      const int kb_res0 = (int)((long)((blockIdx.x / a.m_tiles) % a.splits) * a.k_blocks / a.splits);
      bool b_ok = true;
      if (LNB) b_ok = mbar_wait(smem_u32(bready), 0, abort);
      for (int u = blockIdx.x; b_ok && u < a.units && !*abort; u += gridDim.x) {
        const int z = (u / a.m_tiles) % a.splits;
        const int kb0 = (int)((long)z * a.k_blocks / a.splits);
        const int kb1 = (int)((long)(z + 1) * a.k_blocks / a.splits);
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc_sw128(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd =
              desc_sw128(smem_u32(sB + (LNB ? kb - kb_res0 : stage) * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k)
            tc_mma(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          tc_commit(smem_u32(&empty[stage]));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5 = TMEM lane quadrants 2, 3, 0, 1)
    const int q = warp & 3;
    const int r = q * 32 + lane;          // feature row within the tile
    const int et = threadIdx.x - 64;      // 0..127
    pdl_wait();                           // epilogues read and write earlier kernels' data
    if constexpr (LNB) {
      const int u = blockIdx.x;
      const int z = (u / a.m_tiles) % a.splits;
      const int kb0 = (int)((long)z * a.k_blocks / a.splits);
      tc_ln_fill<BN>(sB, a, kb0, a.b_kb, et, red_v);
      mbar_arrive(smem_u32(bready));
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    int it = 0;
    // the loop condition must not read `abort`: all 128 threads leave together
    for (int u = blockIdx.x; u < a.units; u += gridDim.x, ++it) {
      const int mt = u % a.m_tiles, rest = u / a.m_tiles;
      const int z = rest % a.splits, nt = rest / a.splits;
      const int n0 = nt * TC_BM, m0 = mt * BN;
      const int tile = nt * a.m_tiles + mt;
      // one waiter, then a barrier the 128 threads always reach together; the
      // flag alternates between two slots so a late reader never sees the
      // next unit's value
      if (et == 0) s_ok[it & 1] = mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort) ? 1 : 0;
      named_sync(1, 128);
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * BN;
      if constexpr (CL) {
        // this CTA's only unit: the ring is idle (every MMA has completed)
        // and holds the partial tile the cluster reduces
        if (!tc_cluster_finish<BN>(epi, a, n0, r, et, taddr, s_ok[it & 1] != 0, (float*)sA, crdy,
                                   cfree, (volatile int*)s_last))
          *abort = 1;
        break;
      }
      if (!s_ok[it & 1]) break;
      tc_fence_after();
      float v[16];
      if (a.splits == 1) {
        for (int j0 = 0; j0 < BN; j0 += 16) {
          tmem_ld16(taddr + j0, v);
          tc_finish_chunk<BN>(epi, a, n0, m0, r, j0, v, red_v, red_i, q);
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&tempty[acc]));
      } else {
        // partial tile stored [activation row][feature]: stores and loads are
        // 128 contiguous bytes per warp
        float* mine = a.partial + ((size_t)z * tiles + tile) * TC_BM * BN + r;
        for (int j0 = 0; j0 < BN; j0 += 16) {
          tmem_ld16(taddr + j0, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) mine[(size_t)(j0 + j) * TC_BM] = v[j];
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&tempty[acc]));
        // the CTA barrier orders every thread's partial stores before the
        // one acq_rel arrival; the last arrival acquires the other splits'
        named_sync(1, 128);
        if (et == 0) {
          unsigned prev = atom_add_acq_rel_gpu(&a.tile_cnt[tile], 1u);
          *s_last = (prev == (unsigned)(a.splits - 1));
        }
        named_sync(1, 128);
        const int last = *s_last;
        if (last) {
          const size_t zstride = (size_t)tiles * TC_BM * BN;
          const float* p0 = a.partial + (size_t)tile * TC_BM * BN + r;
          for (int j0 = 0; j0 < BN; j0 += 16) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
            // four splits' loads in flight at a time; sums stay in split order
            for (int zz = 0; zz < a.splits; zz += 4) {
              float t[4][16];
#pragma unroll
              for (int u2 = 0; u2 < 4; ++u2)
                if (zz + u2 < a.splits)
#pragma unroll
                  for (int j = 0; j < 16; ++j)
                    t[u2][j] = __ldcg(p0 + (zz + u2) * zstride + (size_t)(j0 + j) * TC_BM);
#pragma unroll
              for (int u2 = 0; u2 < 4; ++u2)
                if (zz + u2 < a.splits)
#pragma unroll
                  for (int j = 0; j < 16; ++j) v[j] += t[u2][j];
            }
            tc_finish_chunk<BN>(epi, a, n0, m0, r, j0, v, red_v, red_i, q);
          }
          if (et == 0) a.tile_cnt[tile] = 0u;
        }
        if (!last) {
          if (++acc == 2) { acc = 0; acc_phase ^= 1; }
          continue;
        }
      }
      if constexpr (is_argmax<Epi>::value) {
        named_sync(1, 128);
        for (int j = et; j < BN; j += 128) {
          float bv = red_v[j];
          int bi = red_i[j];
          for (int qq = 1; qq < 4; ++qq)
            if (am_better(red_v[qq * BN + j], red_i[qq * BN + j], bv, bi)) {
              bv = red_v[qq * BN + j];
              bi = red_i[qq * BN + j];
            }
          const int m = m0 + j;
          if (m < a.M) {
            epi.part_v[(size_t)m * epi.n_part + nt] = bv;
            epi.part_i[(size_t)m * epi.n_part + nt] = bi;
          }
        }
        named_sync(1, 128);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort) {
    if (threadIdx.x == 0) atomicExch(a.err, TC_ERR_TIMEOUT);
    // let copies and MMAs already issued land before the memory goes away
    const unsigned long long t0 = gtimer();
    while (gtimer() - t0 < 50000ull) {
    }
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
inline PFN_cuTensorMapEncodeTiled_v12000 tc_encoder(char* err, size_t errlen) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
      snprintf(err, errlen, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(e));
      return nullptr;
    }
    fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

// 2-D K-major bf16 map of a [rows][ld] matrix with `Kd` used columns; box 64 x box_rows.
inline bool tc_encode(CUtensorMap* m, const void* ptr, int Kd, int rows, int ld, int box_rows,
                      char* err, size_t errlen) {
  auto enc = tc_encoder(err, errlen);
  if (!enc) return false;
  if (((uintptr_t)ptr & 15) || (ld % 8)) {
    snprintf(err, errlen, "tensor map: base %p / leading dim %d not 16-byte aligned", ptr, ld);
    return false;
  }
  cuuint64_t dims[2] = {(cuuint64_t)Kd, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)TC_BK, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d) for %d x %d ld %d", (int)r, rows, Kd, ld);
    return false;
  }
  return true;
}

inline bool tc_supported(int d, int mlp, int V, int in_fc) {
  return d % 128 == 0 && mlp % 128 == 0 && V % 128 == 0 && d % 8 == 0 && mlp % 8 == 0 &&
         V % 8 == 0 && in_fc % 8 == 0;
}

inline bool tc_weight_map(TcMap& t, const void* W, int N, int Kd, char* err, size_t errlen) {
  t.N = N;
  t.Kd = Kd;
  t.valid = tc_encode(&t.map, W, Kd, N, Kd, TC_BM, err, errlen);
  return t.valid;
}

inline bool tc_make_maps(TcMaps& m, const void* W_lm, const void* Et, const void* W_fc,
                         const void* const* wqkv, const void* const* wo, const void* const* wup,
                         const void* const* wdown, int nb, int d, int mlp, int V, int in_fc,
                         char* err, size_t errlen) {
  if (!tc_weight_map(m.lm, W_lm, V, d, err, errlen)) return false;
  if (!tc_weight_map(m.embed, Et, d, V, err, errlen)) return false;
  if (!tc_weight_map(m.fc, W_fc, d, in_fc, err, errlen)) return false;
  m.qkv.resize(nb);
  m.kv.resize(nb);
  m.o.resize(nb);
  m.up.resize(nb);
  m.down.resize(nb);
  for (int l = 0; l < nb; ++l) {
    if (!tc_weight_map(m.qkv[l], wqkv[l], 3 * d, d, err, errlen)) return false;
    if (!tc_weight_map(m.kv[l], (const bf16*)wqkv[l] + (size_t)d * d, 2 * d, d, err, errlen))
      return false;
    if (!tc_weight_map(m.o[l], wo[l], d, d, err, errlen)) return false;
    if (!tc_weight_map(m.up[l], wup[l], mlp, d, err, errlen)) return false;
    if (!tc_weight_map(m.down[l], wdown[l], d, mlp, err, errlen)) return false;
  }
  return true;
}
inline void tc_free_maps(TcMaps&) {}

inline int tc_pick_bn(int M, int n_tiles = 0, int sms = 0, int k_blocks = 0) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  // 256-row activation tiles unless they leave a quarter of the SMs idle
  // while 128-row tiles would still fit in one round (reductions up to
  // 32K deep; the vocabulary-deep X.E keeps 256 rows and splits K).
  // Measured: choosing 128-row tiles whenever they fill the rounds of tiles
  // better (QKV at 1,024 rows: 384 tiles instead of 192) was slower
  // (43.8 vs 38.6 us): the shorter activation tile halves the work per
  // weight tile streamed
  if (n_tiles > 0 && sms > 0 && k_blocks <= 512) {
    const long t256 = (long)n_tiles * ((M + 255) / 256), t128 = (long)n_tiles * ((M + 127) / 128);
    if (4 * t256 < 3L * sms && t128 <= sms) return 128;
  }
  return 256;
}

template <int BN, int STAGES, class Epi, bool LNB = false>
fm_status tc_launch_cfg(const TcMap& wm, const CUtensorMap& mapA, const TcArgs& a, int grid, Epi epi,
                        cudaStream_t st, char* err, size_t errlen, int* n_launch) {
  using C = TcCfg<BN, STAGES>;
  const int smem = LNB ? C::STAGES * C::A_BYTES + a.b_kb * C::B_BYTES + 1024 + TC_BAR_BYTES + 8 * BN * 4
                       : C::SMEM;
  cudaError_t e = cudaSuccess;
  bool launched = false;
  if constexpr (!LNB && !is_argmax<Epi>::value && BN <= 128) {
    if (a.cluster > 1) {
      if (BN * TC_BM * 4 > C::STAGES * C::A_BYTES || 8 * BN * 4 < 16) {
        snprintf(err, errlen, "tensor-core GEMM: no room for a cluster's partial tile");
        return FM_ERR_UNSUPPORTED;
      }
      e = set_smem_once(k_tc_gemm<BN, STAGES, LNB, Epi, true>, C::SMEM);
      // programmatic launch in clusters of a.cluster CTAs (the K splits of a tile)
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(grid);
      cfg.blockDim = dim3(TC_THREADS);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = st;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = (unsigned)a.cluster;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      if (e == cudaSuccess)
        e = cudaLaunchKernelEx(&cfg, k_tc_gemm<BN, STAGES, LNB, Epi, true>, wm.map, mapA, a, epi);
      launched = true;
    }
  }
  if (!launched) {
    if (a.cluster > 1) {
      snprintf(err, errlen, "tensor-core GEMM: this epilogue has no cluster reduction");
      return FM_ERR_UNSUPPORTED;
    }
    e = set_smem_once(k_tc_gemm<BN, STAGES, LNB, Epi>, LNB ? 227 * 1024 : C::SMEM);
    if (e == cudaSuccess)
      e = launch_pdl(k_tc_gemm<BN, STAGES, LNB, Epi>, dim3(grid), dim3(TC_THREADS), smem, st,
                     wm.map, mapA, a, epi);
  }
  if (e != cudaSuccess) {
    snprintf(err, errlen, "tensor-core GEMM launch: %s", cudaGetErrorString(e));
    return FM_ERR_CUDA;
  }
  if (n_launch) ++*n_launch;
  return FM_OK;
}

template <int BN, class Epi>
fm_status tc_launch(const TcMap& wm, const bf16* A, int lda, int M, Epi epi, float* partial,
                    size_t partial_elems, unsigned* tile_cnt, int tile_cnt_n, int sms, int* err_word,
                    cudaStream_t st, char* err, size_t errlen, int* n_launch) {
  TcArgs a;
  a.M = M;
  a.N = wm.N;
  a.Kd = wm.Kd;
  a.n_tiles = (wm.N + TC_BM - 1) / TC_BM;
  a.m_tiles = (M + BN - 1) / BN;
  a.k_blocks = (wm.Kd + TC_BK - 1) / TC_BK;
  const int tiles = a.n_tiles * a.m_tiles;
  // K splits only while tiles leave SMs idle (measured: more splits than
  // that lose to the serial reduction of their partial tiles), and no more
  // than balance a split's weight stream against the last arrival's pull of
  // all partial tiles: with per-split weight bytes W/S and S partial tiles of
  // P bytes, S ~ sqrt(W/P) (the O projection at 64 rows: 4 splits of its
  // 512 KB weight tile instead of 9, each partial 32 KB)
  int splits = 1, cluster = 0;
  if (tiles < sms) {
    splits = sms / tiles;
    splits = splits > a.k_blocks ? a.k_blocks : splits;
    const double w_tile = (double)a.k_blocks * TC_BK * TC_BM * 2.0;
    const double p_tile = (double)TC_BM * BN * 4.0;
    const int s_bal = (int)ceil(sqrt(w_tile / p_tile));
    // one activation tile: the K splits of a tile can form a cluster (at
    // most 8 CTAs) and sum their partials in distributed shared memory, in
    // parallel over the rows and with no global-memory round trip, so the
    // balance cap does not apply; taken when it keeps at least as many
    // splits as the global-memory reduction would (measured: the context fc
    // at 17 rows in 8 clustered splits instead of 9 was no faster)
    const int s_cl = splits < 8 ? splits : 8;
    const int s_gm = splits > s_bal ? s_bal : splits;
    if (tc_cluster_ok && !is_argmax<Epi>::value && a.m_tiles == 1 && BN <= 128 && s_cl >= 2 &&
        s_cl >= s_gm) {
      splits = s_cl;
      cluster = s_cl;
    } else {
      splits = s_gm;
      while (splits > 1 && (size_t)splits * tiles * TC_BM * BN > partial_elems) --splits;
    }
  }
  if (!cluster && splits > 1 && tiles > tile_cnt_n) splits = 1;
  a.splits = splits < 1 ? 1 : splits;
  a.cluster = cluster;
  a.units = tiles * a.splits;
  a.partial = partial;
  a.tile_cnt = tile_cnt;
  a.err = err_word;
  a.ln_x = a.ln_shift = a.ln_scale = nullptr;
  a.M_ln = 0;
  a.ln_extra = nullptr;
  a.b_kb = 0;
  CUtensorMap mapA;
  if (!tc_encode(&mapA, A, wm.Kd, M, lda, BN, err, errlen)) return FM_ERR_CUDA;
  const int grid = a.units < sms ? a.units : sms;
  // k-blocks one CTA streams: deep ring for long streams, shallow otherwise
  const long per_cta = (long)((a.units + grid - 1) / grid) * ((a.k_blocks + a.splits - 1) / a.splits);
  if constexpr (BN <= 64) {
    if (per_cta < 24)
      return tc_launch_cfg<BN, tc_stages<BN>(false)>(wm, mapA, a, grid, epi, st, err, errlen, n_launch);
  }
  return tc_launch_cfg<BN, tc_stages<BN>(true)>(wm, mapA, a, grid, epi, st, err, errlen, n_launch);
}

template <class Epi>
fm_status tc_gemm(const TcMaps& maps, const TcMap& wm, const bf16* A, int lda, int M, int N, int Kd,
                  Epi epi, float* partial, size_t partial_elems, unsigned* tile_cnt, int tile_cnt_n,
                  int sms, cudaStream_t st, char* err, size_t errlen, int* n_launch) {
  if (N != wm.N || Kd != wm.Kd) {
    snprintf(err, errlen, "tensor-core GEMM: shape %d x %d does not match its weight map %d x %d", N,
             Kd, wm.N, wm.Kd);
    return FM_ERR_ARG;
  }
  switch (tc_pick_bn(M, (wm.N + TC_BM - 1) / TC_BM, sms, (wm.Kd + TC_BK - 1) / TC_BK)) {
    case 16: return tc_launch<16>(wm, A, lda, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
    case 32: return tc_launch<32>(wm, A, lda, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
    case 64: return tc_launch<64>(wm, A, lda, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
    case 128: return tc_launch<128>(wm, A, lda, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
    default: return tc_launch<256>(wm, A, lda, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
  }
}

// y = (LN0(x) (1 + scale) + shift) . W^T with the normalisation done inside
// the GEMM (no separate LayerNorm kernel, no bf16 activation round trip).
// Needs M <= 32 (one activation tile) and every CTA's units sharing one
// k-range; returns FM_ERR_UNSUPPORTED otherwise so the caller can fall back.
template <int BN, class Epi>
fm_status tc_launch_ln(const TcMap& wm, const float* x, const float* shift, const float* scale,
                       int M_ln, const bf16* extra, int M, Epi epi, float* partial,
                       size_t partial_elems, unsigned* tile_cnt, int tile_cnt_n, int sms,
                       int* err_word, cudaStream_t st, char* err, size_t errlen, int* n_launch) {
  TcArgs a;
  a.M = M;
  a.M_ln = M_ln;
  a.ln_extra = extra;
  a.N = wm.N;
  a.Kd = wm.Kd;
  a.n_tiles = (wm.N + TC_BM - 1) / TC_BM;
  a.m_tiles = 1;
  a.k_blocks = (wm.Kd + TC_BK - 1) / TC_BK;
  const int tiles = a.n_tiles;
  int splits = 1;
  if (tiles < sms) {
    splits = sms / tiles;
    splits = splits > a.k_blocks ? a.k_blocks : splits;
    while (splits > 1 && (size_t)splits * tiles * TC_BM * BN > partial_elems) --splits;
  }
  if (splits > 1 && tiles > tile_cnt_n) splits = 1;
  a.splits = splits < 1 ? 1 : splits;
  a.units = tiles * a.splits;
  a.partial = partial;
  a.tile_cnt = tile_cnt;
  a.err = err_word;
  a.ln_x = x;
  a.ln_shift = shift;
  a.ln_scale = scale;
  const int grid = a.units < sms ? a.units : sms;
  if (a.units > grid && a.splits > 1) return FM_ERR_UNSUPPORTED;
  a.b_kb = (a.units <= grid) ? (a.k_blocks + a.splits - 1) / a.splits : a.k_blocks;
  const long per_cta = (long)((a.units + grid - 1) / grid) * ((a.k_blocks + a.splits - 1) / a.splits);
  const bool deep = per_cta >= 24;
  using CS = TcCfg<BN, 5>;
  using CD = TcCfg<BN, 8>;
  if ((deep ? 8 * CD::A_BYTES : 5 * CS::A_BYTES) + a.b_kb * CS::B_BYTES + 1024 + TC_BAR_BYTES + 8 * BN * 4 >
      227 * 1024)
    return FM_ERR_UNSUPPORTED;
  if (deep)
    return tc_launch_cfg<BN, 8, Epi, true>(wm, wm.map, a, grid, epi, st, err, errlen, n_launch);
  return tc_launch_cfg<BN, 5, Epi, true>(wm, wm.map, a, grid, epi, st, err, errlen, n_launch);
}

// Rows [0, M_ln) are LN(x) rows; rows [M_ln, M) come from `extra` (bf16,
// normalised context rows riding along in the same GEMM).
template <class Epi>
fm_status tc_gemm_ln(const TcMaps& maps, const TcMap& wm, const float* x, const float* shift,
                     const float* scale, int M_ln, const bf16* extra, int M, Epi epi,
                     float* partial, size_t partial_elems, unsigned* tile_cnt, int tile_cnt_n,
                     int sms, cudaStream_t st, char* err, size_t errlen, int* n_launch) {
  if (M_ln > 32 || M < M_ln || (M > M_ln && !extra)) return FM_ERR_UNSUPPORTED;
  if (M <= 16)
    return tc_launch_ln<16>(wm, x, shift, scale, M_ln, extra, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
  if (M <= 32)
    return tc_launch_ln<32>(wm, x, shift, scale, M_ln, extra, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
  if (M <= 64)
    return tc_launch_ln<64>(wm, x, shift, scale, M_ln, extra, M, epi, partial, partial_elems, tile_cnt, tile_cnt_n, sms, maps.err, st, err, errlen, n_launch);
  return FM_ERR_UNSUPPORTED;
}

inline fm_status tc_lm_head_argmax(const TcMaps& maps, const bf16* h, int lda, int M, int V,
                                   float* part_v, int* part_i, int n_part, int sms, cudaStream_t st,
                                   char* err, size_t errlen, int* n_launch) {
  EpiArgmax epi{part_v, part_i, n_part};
  // no split-K: the vocabulary supplies enough tiles
  return tc_gemm(maps, maps.lm, h, lda, M, V, maps.lm.Kd, epi, nullptr, 0, nullptr, 0, sms, st, err,
                 errlen, n_launch);
}

}  // namespace fm
