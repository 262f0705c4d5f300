// Persistent DiT pass for one 16-row block (concurrency 1, bf16, sm_100a).
//
// At 16 activation rows every DiT GEMM is a short weight stream (8-34 MB)
// and a kernel per GEMM spends more time starting, filling its pipeline and
// finishing than streaming.  Here one cooperative launch (one CTA per SM)
// runs the whole pass:
//
//   stats, then per block l: QKV, attention, O (+ gated residual),
//   MLP-up (+ GELU), MLP-down (+ gated residual); then the final modulated
//   LayerNorm that feeds the LM head,
//
// separated by grid barriers.  The producer warp never waits on a barrier:
// it streams the weight tiles of the next phase into the shared-memory ring
// while the current phase finishes, so the HBM weight stream runs
// back to back.  Activations (the B operand, at most 64 rows) are written
// straight into shared memory by the epilogue warps: the modulated
// LayerNorm LN0(x)(1 + scale) + shift for QKV and MLP-up, a copy for O and
// MLP-down.  LayerNorm statistics travel as per-128-feature partials (mean,
// sum of squared deviations) written by the producing epilogue and combined
// in a fixed order (Chan et al.'s pairwise update), so no phase re-reads
// whole rows.  Context rows appended since the last draft ride along in the
// QKV phases as extra B rows and get their keys and values written to the
// cache.  Split-K partials are reduced by the last arriving CTA of a tile;
// every wait (mbarrier or grid barrier) is bounded and an expired wait
// aborts the pass with an error code.
#pragma once
#include "fm_attn.cuh"
#include "fm_simt.cuh"
#include "fm_tc.cuh"

namespace fm {

constexpr int DIT_MAX_BLOCKS = 8;
constexpr int DIT_RING = 6;                            // weight stages of 16 KB
constexpr int DIT_M = 16;                              // block rows
constexpr int DIT_BROWS_MAX = 64;                      // block rows + context rows
constexpr int DIT_UNION = 109568;                      // B tiles or attention scratch
constexpr int DIT_SMEM = 1024 + DIT_RING * 16384 + DIT_UNION + 4096;

enum { DIT_QKV = 0, DIT_ATTN = 1, DIT_O = 2, DIT_UP = 3, DIT_DOWN = 4 };

struct DitParams {
  CUtensorMap w[DIT_MAX_BLOCKS][4];   // W_qkv, W_o, W_up, W_down (K-major, box 64 x 128)
  int n_blocks, d, F, M;              // M <= 16 block rows
  int splits[5];                      // per GEMM kind (index by DIT_*; [1] = attention splits)
  float* x;                           // residual stream [M][d] fp32
  float* stats;                       // [d/128 tiles][M][2]: tile mean, tile sum of squared deviations
  float* partial;                     // split-K partials
  unsigned* tile_cnt;                 // per tile, zero between uses
  unsigned* bar;                      // grid barrier counter, zeroed before the launch
  int* err;                           // error word
  int* abort_g;                       // set when any CTA gave up; zeroed before the launch
  bf16* qkv;                          // [M][3d]
  bf16* o;                            // [M][d]
  bf16* u;                            // [M][F]
  bf16* hf;                           // [M][d] final modulated LayerNorm (LM-head input)
  const float* mods;                  // [n_blocks][6][d] then final [2][d]
  bf16* Kc[DIT_MAX_BLOCKS];
  bf16* Vc[DIT_MAX_BLOCKS];
  const bf16* ctx_rows;               // [n_ctx][d] context rows whose keys/values are pending
  int n_ctx;
  int max_ctx;
  RowMap ctx_map;
  AttnMmaArgs attn;                   // one sequence, one noise draft
};

struct DitShared {                    // after the ring and the union region
  uint64_t full[DIT_RING], empty[DIT_RING], tfull[2], tempty[2], bready;
  uint32_t tmem;
  int abort, last, ok[2], attn_last;
  float stat[2 * DIT_BROWS_MAX];      // mean, rstd per row
  float red[4][DIT_M][2];             // per-warp row partials
};

__device__ __forceinline__ int dit_phase_kind(int p, int nb, int* l) {
  // p = 0: statistics of the embedded rows; p = 1 + 5 l + k: block l, kind k;
  // p = 1 + 5 nb: final LayerNorm
  if (p == 0) return -1;
  if (p == 1 + 5 * nb) return -2;
  *l = (p - 1) / 5;
  return (p - 1) % 5;
}

// GEMM shape of a phase kind.
__device__ __forceinline__ void dit_gemm_shape(const DitParams& P, int kind, int* N, int* Kd) {
  const int d = P.d;
  if (kind == DIT_QKV) { *N = 3 * d; *Kd = d; }
  else if (kind == DIT_O) { *N = d; *Kd = d; }
  else if (kind == DIT_UP) { *N = P.F; *Kd = d; }
  else { *N = d; *Kd = P.F; }
}

__device__ __forceinline__ int dit_brows(const DitParams& P, int kind) {
  if (kind == DIT_QKV && P.n_ctx > 0) return (P.M + P.n_ctx + 15) / 16 * 16;
  return 16;
}

// Bounded grid barrier wait (one thread): true when `target` arrivals are in.
__device__ __forceinline__ bool dit_grid_wait(const DitParams& P, unsigned target) {
  const unsigned long long t0 = gtimer();
  while (true) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(P.bar) : "memory");
    if (v >= target) return true;
    if (*(volatile int*)P.abort_g) return false;
    if (gtimer() - t0 > TC_TIMEOUT_NS) {
      atomicExch(P.abort_g, 1);
      return false;
    }
  }
}

// Per-row mean and sum of squared deviations over the 128 features held by
// the 128 epilogue threads (thread et holds feature et of every row).
__device__ __forceinline__ void dit_tile_stats(const float* v, int M, int et, DitShared* sh,
                                               float* out /* [M][2] */) {
  const int w = et >> 5, lane = et & 31;
  float s[DIT_M];
#pragma unroll
  for (int j = 0; j < DIT_M; ++j) s[j] = warp_sum(j < M ? v[j] : 0.f);
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < DIT_M; ++j) sh->red[w][j][0] = s[j];
  named_sync(1, 128);
  float mean[DIT_M];
#pragma unroll
  for (int j = 0; j < DIT_M; ++j)
    mean[j] = (sh->red[0][j][0] + sh->red[1][j][0] + sh->red[2][j][0] + sh->red[3][j][0]) / 128.f;
#pragma unroll
  for (int j = 0; j < DIT_M; ++j) {
    const float dv = j < M ? v[j] - mean[j] : 0.f;
    s[j] = warp_sum(dv * dv);
  }
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < DIT_M; ++j) sh->red[w][j][1] = s[j];
  named_sync(1, 128);
  if (et < M) {
    out[et * 2] = mean[et];
    out[et * 2 + 1] = sh->red[0][et][1] + sh->red[1][et][1] + sh->red[2][et][1] + sh->red[3][et][1];
  }
  named_sync(1, 128);
}

// Row mean / rstd from the 16 tile partials (fixed order; equal tile sizes).
__device__ __forceinline__ void dit_row_stats(const DitParams& P, int et, DitShared* sh) {
  if (et < P.M) {
    const float* st = P.stats;
    const int tiles = P.d / 128;
    float mean = 0.f;
    for (int t = 0; t < tiles; ++t) mean += __ldcg(st + ((size_t)t * P.M + et) * 2);
    mean /= (float)tiles;
    float m2 = 0.f;
    for (int t = 0; t < tiles; ++t) {
      const float mt = __ldcg(st + ((size_t)t * P.M + et) * 2);
      const float dv = mt - mean;
      m2 += __ldcg(st + ((size_t)t * P.M + et) * 2 + 1) + 128.f * dv * dv;
    }
    sh->stat[et] = mean;
    sh->stat[DIT_BROWS_MAX + et] = rsqrtf(m2 / (float)(tiles * 128) + 1e-6f);
  }
  named_sync(1, 128);
}

// B tiles of k-blocks [kb0, kb0 + nkb) for `brows` rows into `sB`
// (128-byte swizzle).  kind QKV/UP: rows < M are the modulated LayerNorm
// of x, QKV rows M .. M+n_ctx-1 are copied context rows; kind O/DOWN: rows
// < M are copied from o / u.  Other rows are zero.
__device__ __forceinline__ void dit_fill_b(const DitParams& P, int kind, int l, uint8_t* sB,
                                           int kb0, int nkb, int brows, int Kd, int et,
                                           DitShared* sh) {
  const bool ln = (kind == DIT_QKV || kind == DIT_UP);
  if (ln) dit_row_stats(P, et, sh);
  const float* shift = nullptr;
  const float* scale = nullptr;
  if (ln) {
    const float* ml = P.mods + (size_t)l * 6 * P.d;
    shift = kind == DIT_QKV ? ml : ml + 3 * P.d;
    scale = kind == DIT_QKV ? ml + P.d : ml + 4 * P.d;
  }
  const bf16* src = kind == DIT_O ? P.o : P.u;
  const int tile_bytes = brows * 128;
  for (int idx = et; idx < nkb * brows * 8; idx += 128) {
    const int kbi = idx / (brows * 8), rem = idx - kbi * (brows * 8);
    const int row = rem >> 3, ch = rem & 7;
    const int col = (kb0 + kbi) * TC_BK + ch * 8;
    uint4 packed = make_uint4(0, 0, 0, 0);
    if (row < P.M) {
      if (ln) {
        const float mean = sh->stat[row], rstd = sh->stat[DIT_BROWS_MAX + row];
        const float* xr = P.x + (size_t)row * P.d + col;
        const float4 x0 = __ldcg((const float4*)xr), x1 = __ldcg((const float4*)(xr + 4));
        const float4 c0 = *(const float4*)(scale + col), c1 = *(const float4*)(scale + col + 4);
        const float4 h0 = *(const float4*)(shift + col), h1 = *(const float4*)(shift + col + 4);
        packed.x = pack_bf16x2((x0.x - mean) * rstd * (1.f + c0.x) + h0.x, (x0.y - mean) * rstd * (1.f + c0.y) + h0.y);
        packed.y = pack_bf16x2((x0.z - mean) * rstd * (1.f + c0.z) + h0.z, (x0.w - mean) * rstd * (1.f + c0.w) + h0.w);
        packed.z = pack_bf16x2((x1.x - mean) * rstd * (1.f + c1.x) + h1.x, (x1.y - mean) * rstd * (1.f + c1.y) + h1.y);
        packed.w = pack_bf16x2((x1.z - mean) * rstd * (1.f + c1.z) + h1.z, (x1.w - mean) * rstd * (1.f + c1.w) + h1.w);
      } else {
        packed = __ldcg((const uint4*)(src + (size_t)row * Kd + col));
      }
    } else if (kind == DIT_QKV && row - P.M < P.n_ctx) {
      packed = __ldcg((const uint4*)(P.ctx_rows + (size_t)(row - P.M) * P.d + col));
    }
    *(uint4*)(sB + kbi * tile_bytes + row * 128 + ((ch ^ (row & 7)) << 4)) = packed;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Final epilogue of one 128-feature tile with the reduced accumulators v
// (column j of the chunk j0 .. j0+15 = B row j0 + j).
__device__ __forceinline__ void dit_epilogue_chunk(const DitParams& P, int kind, int l, int n,
                                                   int j0, const float* v, float* xn) {
  const int d = P.d;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int m = j0 + j;
    if (kind == DIT_QKV) {
      if (m < P.M) {
        P.qkv[(size_t)m * 3 * d + n] = __float2bfloat16_rn(v[j]);
      } else if (m - P.M < P.n_ctx && n >= d) {
        const int r = m - P.M;
        const int q = r / P.ctx_map.n_new, k = r - q * P.ctx_map.n_new;
        const size_t row = (size_t)P.ctx_map.slot[q] * P.max_ctx + P.ctx_map.pos0[q] + k;
        if (n < 2 * d) P.Kc[l][row * d + n - d] = __float2bfloat16_rn(v[j]);
        else P.Vc[l][row * d + n - 2 * d] = __float2bfloat16_rn(v[j]);
      }
    } else if (kind == DIT_UP) {
      if (m < P.M) P.u[(size_t)m * P.F + n] = __float2bfloat16_rn(gelu_tanh(v[j]));
    } else {  // residual: x += gate * y
      if (m < P.M) {
        const float* gate = P.mods + (size_t)l * 6 * d + (kind == DIT_O ? 2 : 5) * d;
        const float xv = __ldcg(P.x + (size_t)m * d + n) + gate[n] * v[j];
        P.x[(size_t)m * d + n] = xv;
        xn[m] = xv;
      }
    }
  }
}

__global__ void __launch_bounds__(TC_THREADS, 1) k_dit_persistent(const __grid_constant__ DitParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sU = base + DIT_RING * 16384;
  DitShared* sh = (DitShared*)(sU + DIT_UNION);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int nb = P.n_blocks, n_phases = 2 + 5 * nb;
  volatile int* abort = &sh->abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DIT_RING; ++s) {
      mbar_init(smem_u32(&sh->full[s]), 1);
      mbar_init(smem_u32(&sh->empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh->tfull[i]), 1);
      mbar_init(smem_u32(&sh->tempty[i]), 128);
    }
    mbar_init(smem_u32(&sh->bready), 128);
    sh->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh->tmem), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem;

  if (warp == 0) {
    // ---------------- weight producer: all phases, never waits on a barrier
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int p = 1; p < n_phases - 1 && !*abort; ++p) {
        int l = 0;
        const int kind = dit_phase_kind(p, nb, &l);
        if (kind == DIT_ATTN) continue;
        int N, Kd;
        dit_gemm_shape(P, kind, &N, &Kd);
        const int S = P.splits[kind], tiles = N / TC_BM, kbs = Kd / TC_BK;
        if (cta >= tiles * S) continue;
        const int nt = cta / S, z = cta % S;
        const int kb0 = z * kbs / S, kb1 = (z + 1) * kbs / S;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&sh->empty[stage]), phase ^ 1, abort)) break;
          const uint32_t fb = smem_u32(&sh->full[stage]);
          mbar_expect_tx(fb, 16384);
          tma_load_2d(smem_u32(sA + stage * 16384), &P.w[l][kind == DIT_QKV ? 0 : kind - 1],
                      kb * TC_BK, nt * TC_BM, fb);
          if (++stage == DIT_RING) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0, b_phase = 0;
      for (int p = 1; p < n_phases - 1 && !*abort; ++p) {
        int l = 0;
        const int kind = dit_phase_kind(p, nb, &l);
        if (kind == DIT_ATTN) continue;
        int N, Kd;
        dit_gemm_shape(P, kind, &N, &Kd);
        const int S = P.splits[kind], tiles = N / TC_BM, kbs = Kd / TC_BK;
        if (cta >= tiles * S) continue;
        const int z = cta % S;
        const int kb0 = z * kbs / S, kb1 = (z + 1) * kbs / S;
        const int brows = dit_brows(P, kind);
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(brows >> 3) << 17) |
                               ((uint32_t)(128 >> 4) << 24);
        if (!mbar_wait(smem_u32(&sh->bready), b_phase, abort)) break;
        b_phase ^= 1;
        if (!mbar_wait(smem_u32(&sh->tempty[acc]), acc_phase ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * 64;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(smem_u32(&sh->full[stage]), phase, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc_sw128(smem_u32(sA + stage * 16384));
          const uint64_t bd = desc_sw128(smem_u32(sU + (kb - kb0) * brows * 128));
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k)
            tc_mma(d_tmem, ad + 2 * k, bd + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          tc_commit(smem_u32(&sh->empty[stage]));
          if (++stage == DIT_RING) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(smem_u32(&sh->tfull[acc]));
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
    }
  } else {
    // ---------------- epilogue warps: barriers, B operands, epilogues, attention
    const int et = threadIdx.x - 64;
    const int q = warp & 3;
    const int r = q * 32 + lane;          // feature row within a 128-row weight tile
    int acc = 0;
    uint32_t acc_phase = 0;
    int it = 0;
    for (int p = 0; p < n_phases; ++p) {
      if (p > 0) {
        // wait until every CTA finished phase p - 1
        if (et == 0) sh->ok[it & 1] = dit_grid_wait(P, (unsigned)(p * G)) ? 1 : 0;
        named_sync(1, 128);
        if (!sh->ok[it & 1]) { *abort = 1; break; }
        ++it;
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
      }
      int l = 0;
      const int kind = dit_phase_kind(p, nb, &l);
      if (kind == -1 || kind == -2) {
        // statistics of the embedded rows (-1) or the final LayerNorm (-2):
        // CTA t < d/128 owns features [128 t, 128 t + 128)
        if (cta < P.d / 128) {
          const int n = cta * 128 + et;
          if (kind == -1) {
            float v[DIT_M];
#pragma unroll
            for (int j = 0; j < DIT_M; ++j) v[j] = j < P.M ? __ldcg(P.x + (size_t)j * P.d + n) : 0.f;
            dit_tile_stats(v, P.M, et, sh, P.stats + (size_t)cta * P.M * 2);
          } else {
            dit_row_stats(P, et, sh);
            const float* mf = P.mods + (size_t)nb * 6 * P.d;
            for (int j = 0; j < P.M; ++j) {
              const float y = (__ldcg(P.x + (size_t)j * P.d + n) - sh->stat[j]) * sh->stat[DIT_BROWS_MAX + j];
              P.hf[(size_t)j * P.d + n] = __float2bfloat16_rn(y * (1.f + mf[P.d + n]) + mf[n]);
            }
          }
        }
      } else if (kind == DIT_ATTN) {
        const int items = P.attn.n_heads * (P.attn.n_ctx_splits + 1);
        if (cta < items) {
          attn_item<1>(P.qkv, P.Kc[l], P.Vc[l], P.o, P.attn, cta % P.attn.n_heads,
                       cta / P.attn.n_heads, sU, &sh->attn_last, et,
                       [] __device__() { named_sync(1, 128); });
        }
      } else {
        int N, Kd;
        dit_gemm_shape(P, kind, &N, &Kd);
        const int S = P.splits[kind], tiles = N / TC_BM, kbs = Kd / TC_BK;
        if (cta < tiles * S) {
          const int nt = cta / S, z = cta % S;
          const int kb0 = z * kbs / S, kb1 = (z + 1) * kbs / S;
          const int brows = dit_brows(P, kind);
          dit_fill_b(P, kind, l, sU, kb0, kb1 - kb0, brows, Kd, et, sh);
          mbar_arrive(smem_u32(&sh->bready));
          // accumulator ready
          if (et == 0) sh->ok[it & 1] = mbar_wait(smem_u32(&sh->tfull[acc]), acc_phase, abort) ? 1 : 0;
          named_sync(1, 128);
          if (!sh->ok[it & 1]) {
            *abort = 1;
            if (et == 0) atomicExch(P.abort_g, 1);
            break;
          }
          ++it;
          tc_fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * 64;
          const int n = nt * TC_BM + r;
          float v[16];
          float xn[DIT_M];
#pragma unroll
          for (int j = 0; j < DIT_M; ++j) xn[j] = 0.f;
          if (S == 1) {
            for (int j0 = 0; j0 < brows; j0 += 16) {
              tmem_ld16(taddr + j0, v);
              dit_epilogue_chunk(P, kind, l, n, j0, v, xn);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sh->tempty[acc]));
          } else {
            float* mine = P.partial + (((size_t)z * tiles + nt) * TC_BM + r) * brows;
            for (int j0 = 0; j0 < brows; j0 += 16) {
              tmem_ld16(taddr + j0, v);
#pragma unroll
              for (int j = 0; j < 16; j += 4)
                *(float4*)(mine + j0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sh->tempty[acc]));
            __threadfence();
            named_sync(1, 128);
            if (et == 0) sh->last = (atomicAdd(&P.tile_cnt[nt], 1u) == (unsigned)(S - 1));
            named_sync(1, 128);
            if (sh->last) {
              __threadfence();
              const size_t zstride = (size_t)tiles * TC_BM * brows;
              const float* p0 = P.partial + ((size_t)nt * TC_BM + r) * brows;
              for (int j0 = 0; j0 < brows; j0 += 16) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
                for (int zz = 0; zz < S; zz += 4) {
                  float4 t4[4][4];
#pragma unroll
                  for (int u2 = 0; u2 < 4; ++u2)
                    if (zz + u2 < S)
#pragma unroll
                      for (int j = 0; j < 4; ++j)
                        t4[u2][j] = __ldcg((const float4*)(p0 + (zz + u2) * zstride + j0 + 4 * j));
#pragma unroll
                  for (int u2 = 0; u2 < 4; ++u2)
                    if (zz + u2 < S)
#pragma unroll
                      for (int j = 0; j < 4; ++j) {
                        v[4 * j] += t4[u2][j].x; v[4 * j + 1] += t4[u2][j].y;
                        v[4 * j + 2] += t4[u2][j].z; v[4 * j + 3] += t4[u2][j].w;
                      }
                }
                dit_epilogue_chunk(P, kind, l, n, j0, v, xn);
              }
              if (et == 0) P.tile_cnt[nt] = 0u;
            }
          }
          const bool finished = (S == 1) || sh->last;
          if ((kind == DIT_O || kind == DIT_DOWN) && finished)
            dit_tile_stats(xn, P.M, et, sh, P.stats + (size_t)nt * P.M * 2);
          named_sync(1, 128);
          if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
      }
      // this CTA is done with phase p
      if (p < n_phases - 1) {
        named_sync(1, 128);
        if (et == 0) {
          __threadfence();
          atomicAdd(P.bar, 1u);
        }
      }
    }
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort || *(volatile int*)P.abort_g) {
    if (threadIdx.x == 0) atomicExch(P.err, TC_ERR_TIMEOUT);
    const unsigned long long t0 = gtimer();
    while (gtimer() - t0 < 50000ull) {
    }
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace fm
