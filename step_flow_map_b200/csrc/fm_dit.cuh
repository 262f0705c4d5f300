// Persistent DiT pass for one 16-row block (concurrency 1, bf16, sm_100a).
//
// At 16 activation rows every DiT GEMM is a short weight stream (8-34 MB)
// and a kernel per GEMM spends more time starting, filling its pipeline and
// finishing than streaming.  Here one cooperative launch (one CTA per SM)
// runs the whole pass:
//
//   stats, then per block l: QKV, attention, O (+ gated residual),
//   MLP-up (+ GELU), MLP-down (+ gated residual); then the final modulated
//   LayerNorm that feeds the LM head.
//
// There is no grid barrier: each unit of a phase (an output tile x K split,
// or an attention item) waits only for the counters of the units whose
// outputs it reads (release/acquire handoffs; one epilogue warp polls a
// counter per lane).  The producer warp never waits on another CTA: it
// streams the weight tiles of the next units into the shared-memory ring
// while the current one finishes.  Activations (the B operand, at most 64
// rows) are written straight into shared memory by the epilogue warps —
// the modulated LayerNorm LN0(x)(1 + scale) + shift for QKV and MLP-up, a
// copy for O and MLP-down — and published to the MMA warp per 8 k-blocks.
// LayerNorm statistics travel as per-128-feature partials (mean, sum of
// squared deviations) written by the producing epilogue and combined in a
// fixed order (Chan et al.'s pairwise update), so no phase re-reads whole
// rows.  Context rows appended since the last draft ride along in the QKV
// phases as extra B rows and get their keys and values written to the
// cache.  Split-K partials are pulled by the last arriving CTA of a tile
// with bulk copies and reduced in shared memory.  Every wait (mbarrier or
// counter) is bounded and an expired wait aborts the pass with an error
// code.  Unrolled loops hold one code path each: rare cases inside them cost
// as much as common ones.
#pragma once
#include "fm_attn.cuh"
#include "fm_simt.cuh"
#include "fm_tc.cuh"

namespace fm {

constexpr int DIT_MAX_BLOCKS = 8;
constexpr int DIT_RING = 8;                            // weight stages of 16 KB
constexpr int DIT_M = 16;                              // block rows
constexpr int DIT_BROWS_MAX = 64;                      // block rows + context rows
constexpr int DIT_ATTN_ST = 2;                         // context chunks in flight in attention
// B tiles, split-K partial tiles, or attention scratch
constexpr int DIT_UNION = 87040;
constexpr int DIT_SMEM = 1024 + DIT_RING * 16384 + DIT_UNION + 12288;
static_assert(attn_mma_smem<1, DIT_ATTN_ST>() <= DIT_UNION, "attention scratch");
static_assert(DIT_SMEM <= 232448, "shared memory per CTA");

enum { DIT_QKV = 0, DIT_ATTN = 1, DIT_O = 2, DIT_UP = 3, DIT_DOWN = 4 };

struct DitParams {
  CUtensorMap w[DIT_MAX_BLOCKS][4];   // W_qkv, W_o, W_up, W_down (K-major, box 64 x 128)
  int n_blocks, d, F, M;              // M <= 16 block rows
  int splits[5];                      // per GEMM kind (index by DIT_*; [1] = attention splits)
  int l2_ahead;                       // weight k-blocks prefetched into L2 beyond the ring
  int skip_final;                     // the LM head applies the final LayerNorm itself
  int stall;                          // test hook: the first QKV wait targets a count never reached
  float* x;                           // residual stream [M][d] fp32
  float* stats;                       // [d/128 tiles][M][2]: tile mean, tile sum of squared deviations
  float* partial;                     // split-K partials, one region per GEMM kind
  size_t part_off[5];                 // float offset of each kind's region
  unsigned* tile_cnt;                 // [kind][1024] arrivals per output tile, zero between uses
  int* err;                           // error word
  int* abort_g;                       // set when any CTA gave up; zeroed before the launch
  // completion counters and flags, zeroed before the launch; a unit of a
  // phase waits only for the units whose outputs it reads
  unsigned* c_stats;                  // tiles of the embedded rows' statistics done (of d/128)
  unsigned* c_o;                      // [n_blocks] O-projection tiles done (of d/128)
  unsigned* c_down;                   // [n_blocks] down-projection tiles done (of d/128)
  unsigned* f_qkv;                    // [n_blocks][3d/128] QKV output tile done
  unsigned* f_head;                   // [n_blocks][n_heads] attention output of a head done
  unsigned* f_up;                     // [n_blocks][F/128] up-projection tile done
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
  int attn_safe;                      // context rows below this are not written by the pass
};

struct DitShared {                    // after the ring and the union region
  uint64_t full[DIT_RING], empty[DIT_RING], tfull[2], tempty[2], bready[2], rbar;
  uint32_t tmem;
  int abort, last, ok[2], attn_last;
  float stat[2 * DIT_BROWS_MAX];      // mean, rstd per row
  float ss[2][1024];                  // shift, scale of this CTA's column slice
  int ctx_row[DIT_BROWS_MAX];         // cache row (slot * max_ctx + position) of each appended context row
};

static_assert(sizeof(DitShared) + 16 <= 12288, "shared bookkeeping region");

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

// Position of the weight producer in this CTA's sequence of k-blocks over all
// GEMM phases.
struct DitCursor {
  int p, l, kind, nt, kb, kb1;
  bool valid;
};

// First k-block of the first phase >= p with GEMM work for this CTA.
__device__ __forceinline__ void dit_cursor_seek(const DitParams& P, int cta, int n_phases, int p,
                                                DitCursor& c) {
  for (; p < n_phases - 1; ++p) {
    int l = 0;
    const int kind = dit_phase_kind(p, P.n_blocks, &l);
    if (kind < 0 || kind == DIT_ATTN) continue;
    int N, Kd;
    dit_gemm_shape(P, kind, &N, &Kd);
    const int S = P.splits[kind], tiles = N / TC_BM, kbs = Kd / TC_BK;
    if (cta >= tiles * S) continue;
    const int z = cta % S;
    c.p = p;
    c.l = l;
    c.kind = kind;
    c.nt = cta / S;
    c.kb = z * kbs / S;
    c.kb1 = (z + 1) * kbs / S;
    if (c.kb >= c.kb1) continue;
    c.valid = true;
    return;
  }
  c.valid = false;
}

__device__ __forceinline__ void dit_cursor_next(const DitParams& P, int cta, int n_phases,
                                                DitCursor& c) {
  if (++c.kb < c.kb1) return;
  dit_cursor_seek(P, cta, n_phases, c.p + 1, c);
}

__device__ __forceinline__ const CUtensorMap* dit_wmap(const DitParams& P, const DitCursor& c) {
  return &P.w[c.l][c.kind == DIT_QKV ? 0 : c.kind - 1];
}

__device__ __forceinline__ int dit_brows(const DitParams& P, int kind) {
  if (kind == DIT_QKV && P.n_ctx > 0) return (P.M + P.n_ctx + 15) / 16 * 16;
  return 16;
}

// Bounded wait (one thread) until the counter reaches `target`.  The abort
// word and the clock are read every 32 polls only: a load after an acquire
// load cannot start before it, so checking them on every poll would double
// the poll's round trip.
__device__ __forceinline__ bool dit_wait(const DitParams& P, const unsigned* ctr, unsigned target) {
  const unsigned long long t0 = gtimer();
  for (unsigned n = 1;; ++n) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    if ((n & 31) == 0) {
      if (*(volatile int*)P.abort_g) return false;
      if (gtimer() - t0 > TC_TIMEOUT_NS) {
        atomicExch(P.abort_g, 1);
        return false;
      }
    }
  }
}

// Publish one completion (thread et == 0, after the CTA's writes are ordered
// before it by a CTA barrier).
__device__ __forceinline__ void dit_signal(unsigned* ctr) { red_add_release_gpu(ctr, 1u); }

// Waits for everything this CTA's unit of the phase reads:
//   QKV(l)   the residual stream after the last block (all down tiles) or the
//            embedded rows' statistics;
//   ATTN(l)  the Q, K and V tiles of its head;
//   O(l)     the attention outputs of the heads its k-slice covers;
//   UP(l)    the residual stream after O(l) (all O tiles);
//   DOWN(l)  the up-projection tiles its k-slice covers;
//   final    the residual stream after the last block.
// Every write-after-read hazard on the shared buffers is ordered through the
// same chain: a unit that overwrites a buffer depends, through full-row
// LayerNorm waits, on every unit that read the previous contents.
//
// One warp waits: each lane polls its own counters (a single counter on lane
// 0; attention's three tiles or a k-slice's heads / up tiles spread over the
// lanes), so their acquire loads are in flight together; the warp vote and
// the CTA barrier that follows order every thread after all of them.
__device__ bool dit_wait_deps_warp(const DitParams& P, int kind, int l, int cta, int lane) {
  const unsigned tiles_d = (unsigned)(P.d / TC_BM);
  const int H = P.attn.n_heads;
  bool ok = true;
  if (kind == -2) {
    if (lane == 0) ok = dit_wait(P, P.c_down + P.n_blocks - 1, tiles_d);
  } else if (kind == DIT_QKV) {
    if (lane == 0)
      ok = dit_wait(P, l == 0 ? P.c_stats : P.c_down + l - 1,
                    tiles_d + ((P.stall && l == 0) ? 1u : 0u));
  } else if (kind == DIT_UP) {
    if (lane == 0) ok = dit_wait(P, P.c_o + l, tiles_d);
  } else if (kind == DIT_ATTN) {
    const int h = cta % H;
    if (lane < 3) ok = dit_wait(P, P.f_qkv + (size_t)l * 3 * H + (size_t)lane * H + h, 1);
  } else if (kind == DIT_O || kind == DIT_DOWN) {
    int N, Kd;
    dit_gemm_shape(P, kind, &N, &Kd);
    const int S = P.splits[kind], kbs = Kd / TC_BK, z = cta % S;
    const int c0 = (z * kbs / S) * TC_BK, c1 = ((z + 1) * kbs / S) * TC_BK;
    // 128-column groups of the input this k-slice reads (a head, or an up tile)
    const int g0 = c0 / 128, g1 = (c1 - 1) / 128;
    const unsigned* f = kind == DIT_O ? P.f_head + (size_t)l * H : P.f_up + (size_t)l * (P.F / TC_BM);
    for (int g = g0 + lane; g <= g1 && ok; g += 32) ok = dit_wait(P, f + g, 1);
  }
  return __all_sync(0xffffffffu, ok);
}

// Per-row mean and sum of squared deviations over the 128 features held by
// the 128 epilogue threads (thread et holds feature et of every row):
// transposed through shared memory `buf` [16][136] (the row stride keeps the
// reads free of bank conflicts), then eight threads per row, each summing
// sixteen features, combine with three shuffles.  Ends with a CTA barrier.
constexpr int DIT_TS_LD = 136;
constexpr int DIT_TS_BYTES = DIT_M * DIT_TS_LD * 4;
__device__ __forceinline__ void dit_tile_stats(const float* v, int M, int et, float* buf,
                                               float* out /* [M][2] */) {
#pragma unroll
  for (int j = 0; j < DIT_M; ++j) buf[j * DIT_TS_LD + et] = j < M ? v[j] : 0.f;
  named_sync(1, 128);
  const int row = et >> 3, g = et & 7;
  float x[16];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    x[i] = buf[row * DIT_TS_LD + i * 8 + g];
    s += x[i];
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 4);
  const float mean = s * (1.f / 128.f);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float dv = x[i] - mean;
    q = fmaf(dv, dv, q);
  }
  q += __shfl_xor_sync(0xffffffffu, q, 1);
  q += __shfl_xor_sync(0xffffffffu, q, 2);
  q += __shfl_xor_sync(0xffffffffu, q, 4);
  if (g == 0 && row < M) {
    out[row * 2] = mean;
    out[row * 2 + 1] = q;
  }
  named_sync(1, 128);
}

// Row mean / rstd from the tile partials (fixed order; equal tile sizes):
// eight threads per row, each loading two tiles' (mean, M2), combined over
// the eight lanes with shuffles (Chan's update with equal counts).
__device__ __forceinline__ void dit_row_stats(const DitParams& P, int et, DitShared* sh) {
  const int row = et >> 3, g = et & 7;
  const int tiles = P.d / 128;  // <= 16
  float mt[2] = {0.f, 0.f}, m2t[2] = {0.f, 0.f};
  bool have[2] = {false, false};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int t = g + 8 * i;
    if (row < P.M && t < tiles) {
      const float2 v = __ldcg((const float2*)(P.stats + ((size_t)t * P.M + row) * 2));
      mt[i] = v.x;
      m2t[i] = v.y;
      have[i] = true;
    }
  }
  float s = (have[0] ? mt[0] : 0.f) + (have[1] ? mt[1] : 0.f);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / (float)tiles;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i)
    if (have[i]) q += m2t[i] + 128.f * (mt[i] - mean) * (mt[i] - mean);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (g == 0 && row < P.M) {
    sh->stat[row] = mean;
    sh->stat[DIT_BROWS_MAX + row] = rsqrtf(q / (float)(tiles * 128) + 1e-6f);
  }
  named_sync(1, 128);
}

// B tiles of k-blocks [kb0, kb0 + nkb) for `brows` rows into `sB`
// (128-byte swizzle).  kind QKV/UP: rows < M are the modulated LayerNorm
// of x, QKV rows M .. M+n_ctx-1 are copied context rows; kind O/DOWN: rows
// < M are copied from o / u.  Other rows are zero.
// Shift and scale of a LayerNorm phase for this CTA's columns [c0, c0 + ncol)
// into shared memory, all loads in flight at once (loaded by
// dit_mods_load, stored by dit_mods_store, so other loads can be issued in
// between).  The adaLN modulation is fixed for the whole pass, so this runs
// before the phase's wait.
__device__ __forceinline__ void dit_mods_load(const DitParams& P, int kind, int l, int c0,
                                              int ncol, int et, float (&hv)[8], float (&cv)[8]) {
  const float* ml = P.mods + (size_t)l * 6 * P.d;
  const float* shift = kind == DIT_QKV ? ml : ml + 3 * P.d;
  const float* scale = kind == DIT_QKV ? ml + P.d : ml + 4 * P.d;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = et + 128 * u;
    hv[u] = cv[u] = 0.f;
    if (c < ncol) {
      hv[u] = __ldg(shift + c0 + c);
      cv[u] = __ldg(scale + c0 + c);
    }
  }
}

__device__ __forceinline__ void dit_mods_store(int ncol, int et, const float (&hv)[8],
                                               const float (&cv)[8], DitShared* sh) {
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int c = et + 128 * u;
    if (c < ncol) {
      sh->ss[0][c] = hv[u];
      sh->ss[1][c] = cv[u];
    }
  }
}

// Rows M .. brows-1 of a QKV phase's B operand: the appended context rows
// (normalised before the pass), then zeros.  They depend on nothing the
// pass computes, so this runs before the phase's wait.
__device__ __forceinline__ void dit_fill_extra(const DitParams& P, uint8_t* sB, int kb0, int nkb,
                                               int brows, int Kd, int et) {
  const int tile_bytes = brows * 128;
  const int M = P.M, nr = P.n_ctx;                 // nr >= 1
  // the context rows, sixteen loads per thread in flight per batch (one
  // batch up to 16 rows x 16 k-blocks)
  const int items = nkb * nr * 8;
  for (int i0 = 0; i0 < items; i0 += 128 * 16) {
    uint4 cp[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = i0 + u * 128 + et;
      const int kbi = idx / (nr * 8), rem = idx - kbi * (nr * 8);
      const int r = rem >> 3, col = (kb0 + kbi) * TC_BK + (rem & 7) * 8;
      cp[u] = make_uint4(0, 0, 0, 0);
      if (idx < items && col < Kd) cp[u] = __ldcg((const uint4*)(P.ctx_rows + (size_t)r * P.d + col));
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = i0 + u * 128 + et;
      if (idx >= items) break;
      const int kbi = idx / (nr * 8), rem = idx - kbi * (nr * 8);
      const int row = M + (rem >> 3), ch = rem & 7;
      *(uint4*)(sB + kbi * tile_bytes + row * 128 + ((ch ^ (row & 7)) << 4)) = cp[u];
    }
  }
  // rows past the context rows up to the tile height: zeros
  const int pr = brows - M - nr;
  const int zitems = nkb * pr * 8;
  for (int idx = et; idx < zitems; idx += 128) {
    const int kbi = idx / (pr * 8), rem = idx - kbi * (pr * 8);
    const int row = M + nr + (rem >> 3), ch = rem & 7;
    *(uint4*)(sB + kbi * tile_bytes + row * 128 + ((ch ^ (row & 7)) << 4)) = make_uint4(0, 0, 0, 0);
  }
}

// B operand rows 0 .. M-1 (M = 16: 128 items per k-block, so each batch of
// 1024 items is 8 k-blocks).  Batch i is published on bready[i] (all 128
// threads arrive) as soon as it is stored, so the MMAs of its k-blocks, and
// the ring refills they free, overlap the rest of the fill.  One barrier per
// batch: each completes at most once per GEMM phase, and the MMA warp
// observes that completion before the epilogue can reach the next phase's
// fill (the epilogue first waits for this phase's accumulator), so a waiter
// polling by parity never misses a phase.  (With one barrier for both
// batches, two completions in quick succession could pass between two polls
// and leave the MMA warp waiting on the wrong phase.)
__device__ __forceinline__ void dit_fill_b(const DitParams& P, int kind, uint8_t* sB, int kb0,
                                           int nkb, int brows, int Kd, int et, DitShared* sh,
                                           const uint64_t* bready) {
  // one loop per kind of row, so each unrolled batch holds one code path
  const int tile_bytes = brows * 128;
  const int M = P.M;
  auto put = [&](int kbi, int row, int ch, uint4 packed) {
    *(uint4*)(sB + kbi * tile_bytes + row * 128 + ((ch ^ (row & 7)) << 4)) = packed;
  };
  if (kind == DIT_QKV || kind == DIT_UP) {
    // block rows: LN0(x)(1 + scale) + shift, eight items per thread and
    // batch with every load of the batch in flight before any is used
    const int items = nkb * M * 8;
    for (int i0 = 0; i0 < items; i0 += 128 * 8) {
      float4 xa[8], xb[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = i0 + u * 128 + et;
        const int kbi = idx / (M * 8), rem = idx - kbi * (M * 8);
        const int row = rem >> 3, col = (kb0 + kbi) * TC_BK + (rem & 7) * 8;
        xa[u] = xb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (idx < items && col < Kd) {
          const float* xr = P.x + (size_t)row * P.d + col;
          xa[u] = __ldcg((const float4*)xr);
          xb[u] = __ldcg((const float4*)(xr + 4));
        }
      }
      // the row statistics load while the first batch is in flight (ends
      // with a CTA barrier)
      if (i0 == 0) dit_row_stats(P, et, sh);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = i0 + u * 128 + et;
        if (idx >= items) break;
        const int kbi = idx / (M * 8), rem = idx - kbi * (M * 8);
        const int row = rem >> 3, ch = rem & 7;
        const int cc = kbi * TC_BK + ch * 8;  // column within this CTA's slice
        const float mean = sh->stat[row], rstd = sh->stat[DIT_BROWS_MAX + row];
        const float* h = sh->ss[0] + cc;
        const float* c = sh->ss[1] + cc;
        uint4 packed;
        packed.x = pack_bf16x2((xa[u].x - mean) * rstd * (1.f + c[0]) + h[0], (xa[u].y - mean) * rstd * (1.f + c[1]) + h[1]);
        packed.y = pack_bf16x2((xa[u].z - mean) * rstd * (1.f + c[2]) + h[2], (xa[u].w - mean) * rstd * (1.f + c[3]) + h[3]);
        packed.z = pack_bf16x2((xb[u].x - mean) * rstd * (1.f + c[4]) + h[4], (xb[u].y - mean) * rstd * (1.f + c[5]) + h[5]);
        packed.w = pack_bf16x2((xb[u].z - mean) * rstd * (1.f + c[6]) + h[6], (xb[u].w - mean) * rstd * (1.f + c[7]) + h[7]);
        put(kbi, row, ch, packed);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(smem_u32(&bready[i0 >> 10]));
    }
  } else {
    // copied rows: attention output (O) or MLP hidden (down); brows == M
    const bf16* src = kind == DIT_O ? P.o : P.u;
    const int items = nkb * brows * 8;
    uint4 cp[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = u * 128 + et;
      const int kbi = idx / (brows * 8), rem = idx - kbi * (brows * 8);
      const int row = rem >> 3, col = (kb0 + kbi) * TC_BK + (rem & 7) * 8;
      cp[u] = make_uint4(0, 0, 0, 0);
      if (idx < items && row < M && col < Kd)
        cp[u] = __ldcg((const uint4*)(src + (size_t)row * Kd + col));
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (half * 1024 >= items) break;
#pragma unroll
      for (int u = 8 * half; u < 8 * half + 8; ++u) {
        const int idx = u * 128 + et;
        if (idx >= items) break;
        const int kbi = idx / (brows * 8), rem = idx - kbi * (brows * 8);
        put(kbi, rem >> 3, rem & 7, cp[u]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(smem_u32(&bready[half]));
    }
  }
}

// Final epilogue of one 128-feature tile with the reduced accumulators v
// (column j of the chunk j0 .. j0+15 = B row j0 + j).
__device__ __forceinline__ void dit_epilogue_chunk(const DitParams& P, int kind, int l, int n,
                                                   int j0, const float* v, const int* ctx_row) {
  const int d = P.d;
  if (kind == DIT_QKV) {
    if (j0 < P.M) {
      // block rows (P.M = 16: the whole chunk)
      bf16* q = P.qkv + (size_t)j0 * 3 * d + n;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j0 + j < P.M) q[(size_t)j * 3 * d] = __float2bfloat16_rn(v[j]);
    } else if (n >= d) {
      // appended context rows: keys and values into the cache (queries dropped)
      bf16* c = n < 2 * d ? P.Kc[l] + (n - d) : P.Vc[l] + (n - 2 * d);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int r = j0 + j - P.M;
        if (r < P.n_ctx) c[(size_t)ctx_row[r] * d] = __float2bfloat16_rn(v[j]);
      }
    }
  } else {
    bf16* u = P.u + (size_t)j0 * P.F + n;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j0 + j < P.M) u[(size_t)j * P.F] = __float2bfloat16_rn(gelu_tanh(v[j]));
  }
}

// Residual epilogue of an O or down-projection tile (16 rows): x += gate * y,
// with x and the gate loaded before the accumulator was ready.
__device__ __forceinline__ void dit_epilogue_residual(const DitParams& P, int n, const float* v,
                                                      const float* xo, float gate, float* xn) {
#pragma unroll
  for (int j = 0; j < DIT_M; ++j) {
    if (j < P.M) {
      const float xv = xo[j] + gate * v[j];
      P.x[(size_t)j * P.d + n] = xv;
      xn[j] = xv;
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
  const int cta = blockIdx.x;
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
    mbar_init(smem_u32(&sh->bready[0]), 128);
    mbar_init(smem_u32(&sh->bready[1]), 128);
    mbar_init(smem_u32(&sh->rbar), 1);
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
    // ---------------- weight producer: all phases, never waits on a barrier.
    // Loads fill the shared-memory ring; while the ring is full, L2
    // prefetches run up to l2_ahead k-blocks further down the same sequence
    // so HBM keeps streaming through barriers, fills and attention.
    if (lane == 0) {
      DitCursor ld, pf;
      dit_cursor_seek(P, cta, n_phases, 1, ld);
      pf = ld;
      int ahead = 0;                    // k-blocks prefetched beyond ld
      int stage = 0;
      uint32_t phase = 0;
      unsigned long long t_prog = gtimer();
      while (ld.valid && !*abort) {
        // with no L2 prefetch to issue, the wait for a free stage suspends
        if (P.l2_ahead > 0 ? mbar_try(smem_u32(&sh->empty[stage]), phase ^ 1)
                           : mbar_try_suspend(smem_u32(&sh->empty[stage]), phase ^ 1)) {
          const uint32_t fb = smem_u32(&sh->full[stage]);
          mbar_expect_tx(fb, 16384);
          tma_load_2d(smem_u32(sA + stage * 16384), dit_wmap(P, ld), ld.kb * TC_BK, ld.nt * TC_BM, fb);
          if (++stage == DIT_RING) { stage = 0; phase ^= 1; }
          dit_cursor_next(P, cta, n_phases, ld);
          if (ahead > 0) --ahead;
          else pf = ld;
          t_prog = gtimer();
        } else if (pf.valid && ahead < P.l2_ahead) {
          tma_prefetch_2d(dit_wmap(P, pf), pf.kb * TC_BK, pf.nt * TC_BM);
          dit_cursor_next(P, cta, n_phases, pf);
          ++ahead;
          t_prog = gtimer();
        } else if (gtimer() - t_prog > TC_TIMEOUT_NS) {
          *abort = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0, b_phase[2] = {0u, 0u};
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
        if (!mbar_wait(smem_u32(&sh->tempty[acc]), acc_phase ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * 64;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (((kb - kb0) & 7) == 0) {
            // the next 8 k-blocks of the B operand are in shared memory
            const int bi = (kb - kb0) >> 3;   // batch 0 or 1 (at most 16 k-blocks)
            if (!mbar_wait(smem_u32(&sh->bready[bi]), b_phase[bi], abort)) { ok = false; break; }
            b_phase[bi] ^= 1;
            tc_fence_after();
          }
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
    if (et < P.n_ctx) {
      const int cq = et / P.ctx_map.n_new, ck = et - cq * P.ctx_map.n_new;
      sh->ctx_row[et] = P.ctx_map.slot[cq] * P.max_ctx + P.ctx_map.pos0[cq] + ck;
    }
    named_sync(1, 128);
    int acc = 0;
    uint32_t acc_phase = 0, r_phase = 0;
    int it = 0;
    for (int p = 0; p < n_phases; ++p) {
      int l = 0;
      const int kind = dit_phase_kind(p, nb, &l);
      if (kind == -2 && P.skip_final) continue;
      bool active;
      if (kind == -1 || kind == -2) active = cta < P.d / TC_BM;
      else if (kind == DIT_ATTN) active = cta < P.attn.n_heads * (P.attn.n_ctx_splits + 1);
      else {
        int N, Kd;
        dit_gemm_shape(P, kind, &N, &Kd);
        active = cta < (N / TC_BM) * P.splits[kind];
      }
      if (!active) continue;
      bool kv_pre = false;
      if (kind == DIT_ATTN) {
        // context chunks the pass does not write load while the QKV tiles
        // are still being produced
        const int h = cta % P.attn.n_heads, split = cta / P.attn.n_heads;
        if (split < P.attn.n_ctx_splits) {
          const AttnRange rg = attn_range(P.attn, 0, h, split);
          kv_pre = rg.k0 + min(AM_CHUNK * DIT_ATTN_ST, rg.k1 - rg.k0) <= P.attn_safe;
          if (kv_pre)
            attn_ctx_prologue<1, DIT_ATTN_ST, DIT_ATTN_ST>(P.Kc[l], P.Vc[l], P.attn, h, split, sU, et);
        }
      }
      if (kind == DIT_QKV || kind == DIT_UP) {
        // work that needs nothing this phase waits for: the adaLN shift and
        // scale of this CTA's columns, and (QKV) the appended context rows
        // of the B operand, their loads in flight together
        int N, Kd;
        dit_gemm_shape(P, kind, &N, &Kd);
        const int S = P.splits[kind], kbs = Kd / TC_BK, z = cta % S;
        const int kb0 = z * kbs / S, kb1 = (z + 1) * kbs / S;
        float hv[8], cv[8];
        dit_mods_load(P, kind, l, kb0 * TC_BK, (kb1 - kb0) * TC_BK, et, hv, cv);
        if (kind == DIT_QKV && P.n_ctx > 0)
          dit_fill_extra(P, sU, kb0, kb1 - kb0, dit_brows(P, kind), Kd, et);
        dit_mods_store((kb1 - kb0) * TC_BK, et, hv, cv, sh);
      }
      if (kind != -1) {
        // wait for the units whose outputs this one reads
        if (et < 32) {
          const bool ok = dit_wait_deps_warp(P, kind, l, cta, et);
          if (et == 0) sh->ok[it & 1] = ok ? 1 : 0;
        }
        named_sync(1, 128);
        if (!sh->ok[it & 1]) { *abort = 1; break; }
        ++it;
      }
      if (kind == -1 || kind == -2) {
        // statistics of the embedded rows (-1) or the final LayerNorm (-2):
        // CTA t < d/128 owns features [128 t, 128 t + 128)
        if (cta < P.d / 128) {
          const int n = cta * 128 + et;
          if (kind == -1) {
            float v[DIT_M];
#pragma unroll
            for (int j = 0; j < DIT_M; ++j) v[j] = j < P.M ? __ldcg(P.x + (size_t)j * P.d + n) : 0.f;
            dit_tile_stats(v, P.M, et, (float*)(sU + DIT_UNION - DIT_TS_BYTES),
                           P.stats + (size_t)cta * P.M * 2);
            if (et == 0) dit_signal(P.c_stats);
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
          attn_item<1, DIT_ATTN_ST, true>(P.qkv, P.Kc[l], P.Vc[l], P.o, P.attn, cta % P.attn.n_heads,
                                    cta / P.attn.n_heads, sU, &sh->attn_last, et,
                                    [] __device__() { named_sync(1, 128); },
                                    AttnBulkMerge{&sh->rbar, &r_phase, abort, (uint32_t)DIT_UNION},
                                    kv_pre);
          named_sync(1, 128);
          // the CTA that merged the head's splits publishes it
          if (et == 0 && sh->attn_last)
            dit_signal(P.f_head + (size_t)l * P.attn.n_heads + cta % P.attn.n_heads);
        }
      } else {
        int N, Kd;
        dit_gemm_shape(P, kind, &N, &Kd);
        const int S = P.splits[kind], tiles = N / TC_BM, kbs = Kd / TC_BK;
        if (cta < tiles * S) {
          const int nt = cta / S, z = cta % S;
          const int kb0 = z * kbs / S, kb1 = (z + 1) * kbs / S;
          const int brows = dit_brows(P, kind);
          dit_fill_b(P, kind, sU, kb0, kb1 - kb0, brows, Kd, et, sh, sh->bready);
          const int n = nt * TC_BM + r;
          // residual phases: x and the gate, loaded while the MMAs run
          const bool resid = (kind == DIT_O || kind == DIT_DOWN);
          float xo[DIT_M];
          float gate = 0.f;
          if (resid) {
            gate = __ldg(P.mods + (size_t)l * 6 * P.d + (kind == DIT_O ? 2 : 5) * P.d + n);
#pragma unroll
            for (int j = 0; j < DIT_M; ++j) xo[j] = j < P.M ? __ldcg(P.x + (size_t)j * P.d + n) : 0.f;
          }
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
          float v[16];
          float xn[DIT_M];
#pragma unroll
          for (int j = 0; j < DIT_M; ++j) xn[j] = 0.f;
          if (S == 1) {
            for (int j0 = 0; j0 < brows; j0 += 16) {
              tmem_ld16(taddr + j0, v);
              if (resid) dit_epilogue_residual(P, n, v, xo, gate, xn);
              else dit_epilogue_chunk(P, kind, l, n, j0, v, sh->ctx_row);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sh->tempty[acc]));
          } else {
            float* part = P.partial + P.part_off[kind];
            unsigned* cnt = P.tile_cnt + kind * 1024;
            // partial tile stored [row j][feature r]: every store and every
            // later shared-memory read is consecutive across the lanes
            float* mine = part + ((size_t)z * tiles + nt) * TC_BM * brows + r;
            for (int j0 = 0; j0 < brows; j0 += 16) {
              tmem_ld16(taddr + j0, v);
#pragma unroll
              for (int j = 0; j < 16; ++j) mine[(size_t)(j0 + j) * TC_BM] = v[j];
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sh->tempty[acc]));
            named_sync(1, 128);
            if (et == 0) sh->last = (atom_add_acq_rel_gpu(&cnt[nt], 1u) == (unsigned)(S - 1));
            named_sync(1, 128);
            if (sh->last) {
              // the S partial tiles of this output tile, one bulk copy each,
              // into the B region (the MMAs that read it have completed)
              const uint32_t tile_bytes = (uint32_t)(TC_BM * brows * 4);
              const uint32_t rb = smem_u32(&sh->rbar);
              if (et == 0) {
                asm volatile("fence.proxy.async.global;" ::: "memory");
                mbar_expect_tx(rb, tile_bytes * S);
                for (int zz = 0; zz < S; ++zz)
                  bulk_load(smem_u32(sU) + zz * tile_bytes,
                            part + ((size_t)zz * tiles + nt) * TC_BM * brows, tile_bytes, rb);
              }
              // one bounded waiter decides for all; then every thread observes
              // the completed phase itself (it cannot advance again here)
              if (et == 0) sh->ok[it & 1] = mbar_wait(rb, r_phase, abort) ? 1 : 0;
              named_sync(1, 128);
              if (!sh->ok[it & 1]) {
                *abort = 1;
                if (et == 0) atomicExch(P.abort_g, 1);
                break;
              }
              ++it;
              (void)mbar_wait(rb, r_phase, abort);   // returns at once
              r_phase ^= 1;
              const float* sp = (const float*)sU + r;
              for (int j0 = 0; j0 < brows; j0 += 16) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = 0.f;
                for (int zz = 0; zz < S; ++zz) {
                  const float* t = sp + ((size_t)zz * brows + j0) * TC_BM;
#pragma unroll
                  for (int j = 0; j < 16; ++j) v[j] += t[j * TC_BM];
                }
                if (resid) dit_epilogue_residual(P, n, v, xo, gate, xn);
                else dit_epilogue_chunk(P, kind, l, n, j0, v, sh->ctx_row);
              }
              if (et == 0) cnt[nt] = 0u;
            }
          }
          const bool finished = (S == 1) || sh->last;
          if ((kind == DIT_O || kind == DIT_DOWN) && finished)
            dit_tile_stats(xn, P.M, et, (float*)(sU + DIT_UNION - DIT_TS_BYTES),
                           P.stats + (size_t)nt * P.M * 2);
          named_sync(1, 128);
          if (finished && et == 0) {
            if (kind == DIT_QKV) dit_signal(P.f_qkv + (size_t)l * tiles + nt);
            else if (kind == DIT_O) dit_signal(P.c_o + l);
            else if (kind == DIT_UP) dit_signal(P.f_up + (size_t)l * tiles + nt);
            else dit_signal(P.c_down + l);
          }
          if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
      }
      named_sync(1, 128);
    }
  }

  // ---------------- teardown
  tc_fence_before();
  // one barrier that also ORs every thread's view of the abort words, so
  // every thread takes the same branch
  if (__syncthreads_or((*abort || *(volatile int*)P.abort_g) ? 1 : 0)) {
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
