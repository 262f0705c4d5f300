// Split-KV attention of the block queries (bf16, head width 128).
//
// For each (sequence, head) the N*16 block queries of the sequence's noise
// drafts attend, without a mask, over [context rows; the draft's own 16
// block rows] (the drafter's attention; the pages give 16 heads of a
// 2048-wide DiT -- page "FlashMap并行草拟加速大模型解码", section
// "一步生成整块，训练时做了什么").  The context rows are shared by every draft of
// the sequence, so one CTA streams a context slice once for all N drafts.
//
// Grid: (sequence*head, n_ctx_splits + 1).  Split s < n_ctx_splits covers a
// contiguous slice of context rows; the last split covers each draft's own
// block rows.  Every CTA keeps an online softmax in registers (mma.sync
// m16n8k16 bf16 -> fp32), merges its four warps in shared memory and writes
// an unnormalised partial (row max m, row sum l, O).  The last CTA of a
// (sequence, head) -- arrival counter, no waiting -- merges the partials in
// split order and writes O / l as bf16.
#pragma once
#include <type_traits>
#include "fm_common.cuh"
#include "fm_tc.cuh"

namespace fm {

constexpr int AM_DH = 128;            // head width
constexpr int AM_CHUNK = 64;          // context rows per smem stage
constexpr int AM_STAGES = 3;          // context chunks in flight per CTA
constexpr int AM_LD = AM_DH + 8;      // padded smem row (272 bytes): conflict-free ldmatrix
constexpr int AM_THREADS = 128;
constexpr int AM_PSTRIDE = AM_DH + 4;  // floats per partial row: O[128], m, l, pad (16-byte rows)

struct AttnMmaArgs {
  int n_seqs, n_noise, K, d, n_heads, max_ctx, n_ctx_splits;
  // split_rows == 0: the context splits divide [0, len) evenly.  split_rows
  // > 0 (one sequence, one noise draft): split s covers rows
  // [s split_rows, (s + 1) split_rows) of [0, tail0), and the block-row item
  // also takes the context rows [tail0, len) (at most 112 of them)
  int split_rows, tail0;
  float scale_log2;    // log2(e) / sqrt(dh)
  float* part;         // [pairs][n_ctx_splits + 1][N*16][AM_PSTRIDE]
  unsigned* cnt;       // [pairs], zero between launches
  int slot[256];
  int len[256];
};

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *(uint32_t*)&v;
}

// Online-softmax state of one warp: 16 query rows (this thread: rows g, g+8).
struct AttnState {
  float o[16][4];
  float m[2], l[2];
};

// Scores of one warp's 16 queries (A fragments qa) against `nk` keys at
// smem rows ks (row-major [key][AM_LD]), then the online update with the
// matching value rows vs.  NT = number of 8-key tiles (nk <= 8*NT).
template <int NT>
__device__ __forceinline__ void attn_block(AttnState& st, const uint32_t (&qa)[8][4],
                                           const bf16* ks, const bf16* vs, int nk, float sl2) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  float s[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < AM_DH / 16; ++kk) {
#pragma unroll
    for (int n = 0; n < NT; n += 2) {
      const int key = n * 8 + (lane & 7) + ((lane >> 4) << 3);
      const int col = kk * 16 + ((lane >> 3) & 1) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4((uint32_t)__cvta_generic_to_shared(ks + key * AM_LD + col), b0, b1, b2, b3);
      mma_bf16(s[n], qa[kk], b0, b1);
      mma_bf16(s[n + 1], qa[kk], b2, b3);
    }
  }
  // mask keys beyond nk, scale to log2 units, row maxima over the quad
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = n * 8 + 2 * t + (e & 1);
      s[n][e] = key < nk ? s[n][e] * sl2 : -INFINITY;
      mx[e >> 1] = fmaxf(mx[e >> 1], s[n][e]);
    }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
  }
  float corr[2], mnew[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    mnew[r] = fmaxf(st.m[r], mx[r]);
    corr[r] = (mnew[r] == -INFINITY) ? 1.f : exp2f(st.m[r] - mnew[r]);
    st.m[r] = mnew[r];
    st.l[r] *= corr[r];
  }
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    st.o[n][0] *= corr[0]; st.o[n][1] *= corr[0];
    st.o[n][2] *= corr[1]; st.o[n][3] *= corr[1];
  }
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mm = mnew[e >> 1];
      s[n][e] = (mm == -INFINITY) ? 0.f : exp2f(s[n][e] - mm);
      st.l[e >> 1] += s[n][e];
    }
  // O += P V, 16 keys per k-step
#pragma unroll
  for (int kb = 0; kb < NT / 2; ++kb) {
    uint32_t pa[4];
    pa[0] = pack_bf16(s[2 * kb][0], s[2 * kb][1]);
    pa[1] = pack_bf16(s[2 * kb][2], s[2 * kb][3]);
    pa[2] = pack_bf16(s[2 * kb + 1][0], s[2 * kb + 1][1]);
    pa[3] = pack_bf16(s[2 * kb + 1][2], s[2 * kb + 1][3]);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
      const int key = kb * 16 + (lane & 15);
      const int col = n * 8 + (lane >> 4) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t((uint32_t)__cvta_generic_to_shared(vs + key * AM_LD + col), b0, b1, b2, b3);
      mma_bf16(st.o[n], pa, b0, b1);
      mma_bf16(st.o[n + 1], pa, b2, b3);
    }
  }
}

// Loads rows [r0, r0+nr) of a [rows][ld] bf16 matrix (dh columns from col0)
// into smem [nr][AM_LD]; rows past nr up to `pad_to` are zero-filled.  Run by
// the AM_THREADS threads of an attention work item (tid 0..AM_THREADS-1).
__device__ __forceinline__ void load_rows(bf16* dst, const bf16* src, size_t ld, int nr, int pad_to,
                                          int tid) {
  for (int e = tid; e < pad_to * (AM_DH / 8); e += AM_THREADS) {
    const int r = e / (AM_DH / 8), c8 = (e % (AM_DH / 8)) * 8;
    bf16* dp = dst + r * AM_LD + c8;
    if (r < nr) cp_async16((uint32_t)__cvta_generic_to_shared(dp), src + (size_t)r * ld + c8);
    else *(uint4*)dp = make_uint4(0, 0, 0, 0);
  }
}

// Context rows [k0, k1) of split `split` of sequence b.
struct AttnRange {
  int k0, k1, n_chunks;
  size_t base;   // element offset of (slot, row 0, head h) in the K/V caches
};
__device__ __forceinline__ AttnRange attn_range(const AttnMmaArgs& a, int b, int h, int split) {
  AttnRange r;
  const int L = a.len[b];
  if (a.split_rows > 0) {
    r.k0 = min(split * a.split_rows, a.tail0);
    r.k1 = min(r.k0 + a.split_rows, a.tail0);
  } else {
    r.k0 = (int)((long)split * L / a.n_ctx_splits);
    r.k1 = (int)((long)(split + 1) * L / a.n_ctx_splits);
  }
  r.n_chunks = (r.k1 - r.k0 + AM_CHUNK - 1) / AM_CHUNK;
  r.base = (size_t)a.slot[b] * a.max_ctx * a.d + h * AM_DH;
  return r;
}

// Issue the first NPRE (ST - 1, or the whole ring: ST) context chunks of a
// split (one cp.async commit group each, empty past the end) into the K/V
// ring.  A caller may run this before the queries exist, when those rows are
// not written by the same pass.
template <int N, int ST, int NPRE = ST - 1>
__device__ __forceinline__ void attn_ctx_prologue(const bf16* __restrict__ Kc,
                                                  const bf16* __restrict__ Vc,
                                                  const AttnMmaArgs& a, int pair, int split,
                                                  uint8_t* smem_raw, int tid) {
  bf16* sK = (bf16*)smem_raw + N * 16 * AM_LD;
  bf16* sV = sK + ST * AM_CHUNK * AM_LD;
  const int b = pair / a.n_heads, h = pair - b * a.n_heads;
  const AttnRange rg = attn_range(a, b, h, split);
#pragma unroll
  for (int c = 0; c < NPRE; ++c) {
    if (c < rg.n_chunks) {
      const int r0 = rg.k0 + c * AM_CHUNK, nr = min(AM_CHUNK, rg.k1 - r0);
      load_rows(sK + c * AM_CHUNK * AM_LD, Kc + rg.base + (size_t)r0 * a.d, a.d, nr, AM_CHUNK, tid);
      load_rows(sV + c * AM_CHUNK * AM_LD, Vc + rg.base + (size_t)r0 * a.d, a.d, nr, AM_CHUNK, tid);
    }
    cp_commit();
  }
}

// Merge of a head's split partials through shared memory (BULK items): one
// bulk copy of all partials, completing on `bar` (phase parity `phase`,
// flipped on use); they must fit in `smem_bytes` (the caller checks; a
// merge that would not fit sets `abort` and is skipped); `abort` also bounds
// the wait.  Without BULK the merging CTA reads the partials from global
// memory directly.
struct AttnBulkMerge {
  uint64_t* bar;
  uint32_t* phase;
  volatile int* abort;
  uint32_t smem_bytes;
};

// One work item -- (sequence, head) pair `pair`, split `split` -- run by
// AM_THREADS threads (tid 0..AM_THREADS-1, four whole warps) that
// synchronise with `sync()`.  ST context chunks are in flight; `smem_raw`
// holds attn_mma_smem<N, ST>() bytes; `s_last` is one shared int.  BULK
// (the persistent pass): the prologue fills the whole ring (ST chunks, so a
// split of at most ST chunks needs no load after its queries exist) and the
// split partials are merged through one bulk copy.
template <int N, int ST, bool BULK, class Sync>
__device__ __forceinline__ void attn_item(const bf16* __restrict__ qkv, const bf16* __restrict__ Kc,
                                          const bf16* __restrict__ Vc, bf16* __restrict__ out,
                                          const AttnMmaArgs& a, int pair, int split,
                                          uint8_t* smem_raw, int* s_last_p, int tid, Sync sync,
                                          AttnBulkMerge bm = AttnBulkMerge{nullptr, nullptr, nullptr, 0},
                                          bool prologue_done = false) {
  bf16* sQ = (bf16*)smem_raw;                       // [N*16][AM_LD]
  bf16* sK = sQ + N * 16 * AM_LD;                   // [ST][AM_CHUNK][AM_LD]
  bf16* sV = sK + ST * AM_CHUNK * AM_LD;            // [ST][AM_CHUNK][AM_LD]
  int& s_last = *s_last_p;
  constexpr int WPM = 4 / N;                        // warps sharing one 16-query tile
  const int b = pair / a.n_heads, h = pair - b * a.n_heads;
  const int d3 = 3 * a.d, warp = tid >> 5, lane = tid & 31;
  const int mt = warp % N, sub = warp / N;          // query tile, key sub-slice
  const int row0 = b * a.n_noise * a.K;             // first block row of the sequence
  const int S_all = a.n_ctx_splits + 1;
  const int NQ = N * 16;

  AttnState st;
#pragma unroll
  for (int n = 0; n < 16; ++n) st.o[n][0] = st.o[n][1] = st.o[n][2] = st.o[n][3] = 0.f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.f;

  uint32_t qa[8][4];
  auto q_fragments = [&]() {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int r = mt * 16 + (lane & 15), c = kk * 16 + (lane >> 4) * 8;
      ldsm_x4((uint32_t)__cvta_generic_to_shared(sQ + r * AM_LD + c), qa[kk][0], qa[kk][1],
              qa[kk][2], qa[kk][3]);
    }
  };

  if (split < a.n_ctx_splits) {
    const AttnRange rg = attn_range(a, b, h, split);
    const int k0 = rg.k0, k1 = rg.k1, n_chunks = rg.n_chunks;
    const size_t base = rg.base;
    auto load_chunk = [&](int c) {
      const int r0 = k0 + c * AM_CHUNK, nr = min(AM_CHUNK, k1 - r0);
      const int buf = c % ST;
      load_rows(sK + buf * AM_CHUNK * AM_LD, Kc + base + (size_t)r0 * a.d, a.d, nr, AM_CHUNK, tid);
      load_rows(sV + buf * AM_CHUNK * AM_LD, Vc + base + (size_t)r0 * a.d, a.d, nr, AM_CHUNK, tid);
    };
    // one commit group per chunk (empty past the end) keeps the group count
    // fixed: ST - 1 chunks are always in flight ahead of the one used
    constexpr int NPRE = BULK ? ST : ST - 1;
    if (!prologue_done) attn_ctx_prologue<N, ST, NPRE>(Kc, Vc, a, pair, split, smem_raw, tid);
    // queries of all drafts of the sequence (the newest group)
    load_rows(sQ, qkv + (size_t)row0 * d3 + h * AM_DH, d3, NQ, NQ, tid);
    cp_commit();
    cp_wait<0>();
    sync();
    q_fragments();
    for (int c = 0; c < n_chunks; ++c) {
      if constexpr (!BULK) {
        if (c + ST - 1 < n_chunks) load_chunk(c + ST - 1);
        cp_commit();
      }
      // one commit group per iteration: chunk c's group is older than the
      // ST - 1 most recent ones
      cp_wait<ST - 1>();
      sync();
      const int buf = c % ST;
      const int nk_chunk = min(AM_CHUNK, k1 - (k0 + c * AM_CHUNK));
      constexpr int KW = AM_CHUNK / WPM;            // keys of this warp within the chunk
      const int kw0 = sub * KW;
      const int nk = max(0, min(KW, nk_chunk - kw0));
      const bf16* ks = sK + buf * AM_CHUNK * AM_LD + kw0 * AM_LD;
      const bf16* vs = sV + buf * AM_CHUNK * AM_LD + kw0 * AM_LD;
      if (nk > 0) attn_block<KW / 8>(st, qa, ks, vs, nk, a.scale_log2);
      sync();
      if constexpr (BULK) {
        // the whole ring was prefetched: chunk c + ST goes into the buffer
        // just read
        if (c + ST < n_chunks) load_chunk(c + ST);
        cp_commit();
      }
    }
  } else if (a.split_rows > 0) {
    // one sequence, one noise draft: the context rows [tail0, len) and the
    // block's own 16 rows, as one key range [tail rows; own rows] spread
    // over the four warps
    static_assert(N == 1 || BULK == false, "tail rows need one noise draft");
    const int L = a.len[b], nt = L - a.tail0, nkey = nt + 16;
    const size_t base = (size_t)a.slot[b] * a.max_ctx * a.d + h * AM_DH;
    load_rows(sQ, qkv + (size_t)row0 * d3 + h * AM_DH, d3, NQ, NQ, tid);
    load_rows(sK, Kc + base + (size_t)a.tail0 * a.d, a.d, nt, nt, tid);
    load_rows(sV, Vc + base + (size_t)a.tail0 * a.d, a.d, nt, nt, tid);
    const int pad = (nkey + 31) / 32 * 32;
    load_rows(sK + nt * AM_LD, qkv + (size_t)row0 * d3 + a.d + h * AM_DH, d3, 16, pad - nt, tid);
    load_rows(sV + nt * AM_LD, qkv + (size_t)row0 * d3 + 2 * a.d + h * AM_DH, d3, 16, pad - nt, tid);
    cp_commit();
    cp_wait<0>();
    sync();
    q_fragments();
    const int kw0 = warp * 32, nk = max(0, min(32, nkey - kw0));
    if (nk > 0) attn_block<4>(st, qa, sK + kw0 * AM_LD, sV + kw0 * AM_LD, nk, a.scale_log2);
    sync();
  } else {
    load_rows(sQ, qkv + (size_t)row0 * d3 + h * AM_DH, d3, NQ, NQ, tid);
    // each draft's own block rows: keys/values of rows row0 + mt*16 .. +16
    if (sub == 0) {
      // warps sub==0 (one per draft) load their 16 rows into their own slice
      bf16* kd = sK + mt * 16 * AM_LD;
      bf16* vd = sV + mt * 16 * AM_LD;
      const bf16* kg = qkv + (size_t)(row0 + mt * 16) * d3 + a.d + h * AM_DH;
      const bf16* vg = kg + a.d;
      for (int e = lane; e < 16 * (AM_DH / 8); e += 32) {
        const int r = e / (AM_DH / 8), c8 = (e % (AM_DH / 8)) * 8;
        cp_async16((uint32_t)__cvta_generic_to_shared(kd + r * AM_LD + c8), kg + (size_t)r * d3 + c8);
        cp_async16((uint32_t)__cvta_generic_to_shared(vd + r * AM_LD + c8), vg + (size_t)r * d3 + c8);
      }
    }
    cp_commit();
    cp_wait<0>();
    sync();
    q_fragments();
    if (sub == 0) attn_block<2>(st, qa, sK + mt * 16 * AM_LD, sV + mt * 16 * AM_LD, 16, a.scale_log2);
    sync();
  }

  // ---- merge the warps of each query tile: per-row (max, sum) of every warp
  // through shared memory; each warp rescales its own O in registers; the
  // partial is the sum of the rescaled warp tiles
  float l_tot[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_tot[r] = st.l[r];
    l_tot[r] += __shfl_xor_sync(0xffffffffu, l_tot[r], 1);
    l_tot[r] += __shfl_xor_sync(0xffffffffu, l_tot[r], 2);
  }
  constexpr int OLD = AM_DH + 4;                    // row stride of a warp's O tile (16-byte rows)
  float* sML = (float*)sK;                          // [4 warps][16][2]: row max, row sum
  float* sO = sML + 4 * 16 * 2;                     // [4 warps][16][OLD] rescaled O
  const int g = lane >> 2, t = lane & 3;
  if (t == 0) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      sML[(warp * 16 + g + 8 * r) * 2] = st.m[r];
      sML[(warp * 16 + g + 8 * r) * 2 + 1] = l_tot[r];
    }
  }
  sync();
  float Mrow[2], Lrow[2], f[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = g + 8 * r;
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < WPM; ++s2) M = fmaxf(M, sML[((s2 * N + mt) * 16 + row) * 2]);
    float L = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < WPM; ++s2) {
      const float mm = sML[((s2 * N + mt) * 16 + row) * 2];
      if (mm != -INFINITY) L += exp2f(mm - M) * sML[((s2 * N + mt) * 16 + row) * 2 + 1];
    }
    f[r] = (st.m[r] == -INFINITY) ? 0.f : exp2f(st.m[r] - M);
    Mrow[r] = M;
    Lrow[r] = L;
  }
  float* wo = sO + warp * 16 * OLD;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int c = n * 8 + 2 * t;
    *(float2*)(wo + g * OLD + c) = make_float2(st.o[n][0] * f[0], st.o[n][1] * f[0]);
    *(float2*)(wo + (g + 8) * OLD + c) = make_float2(st.o[n][2] * f[1], st.o[n][3] * f[1]);
  }
  sync();
  float* part = a.part + ((size_t)pair * S_all + split) * NQ * AM_PSTRIDE;
  for (int e = tid; e < NQ * (AM_DH / 4); e += AM_THREADS) {
    const int q = e / (AM_DH / 4), c4 = (e % (AM_DH / 4)) * 4;
    const int tile = q / 16, rr = q % 16;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s2 = 0; s2 < WPM; ++s2) {
      const float4 v = *(const float4*)(sO + ((s2 * N + tile) * 16 + rr) * OLD + c4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *(float4*)(part + (size_t)q * AM_PSTRIDE + c4) = acc;
  }
  if (sub == 0 && t == 0) {
    // one warp per query tile writes its rows' (max, sum)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int q = mt * 16 + g + 8 * r;
      *(float2*)(part + (size_t)q * AM_PSTRIDE + AM_DH) = make_float2(Mrow[r], Lrow[r]);
    }
  }
  sync();
  if (tid == 0) s_last = (atom_add_acq_rel_gpu(&a.cnt[pair], 1u) == (unsigned)(S_all - 1));
  sync();
  if (!s_last) return;
  // ---- last CTA of this (sequence, head): merge the splits in split order,
  // eight threads per query row, each with four float4 column groups 32
  // columns apart (the eight lanes of a row read 128 contiguous bytes)
  const float* pp = a.part + (size_t)pair * S_all * NQ * AM_PSTRIDE;
  const uint32_t merge_bytes = (uint32_t)((size_t)S_all * NQ * AM_PSTRIDE * 4);
  if constexpr (BULK) {
    if (merge_bytes > bm.smem_bytes) {
      if (tid == 0) {
        *bm.abort = 1;
        s_last = 0;   // nothing merged: the caller must not publish the head
      }
      return;
    }
    // all partials of the pair are contiguous: one copy into shared memory
    const uint32_t mb = (uint32_t)__cvta_generic_to_shared(bm.bar);
    if (tid == 0) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      mbar_expect_tx(mb, merge_bytes);
      bulk_load((uint32_t)__cvta_generic_to_shared(smem_raw), pp, merge_bytes, mb);
      if (!mbar_wait(mb, *bm.phase, bm.abort)) s_last = 0;
    }
    sync();
    if (!s_last) return;   // the wait gave up (abort is set)
    (void)mbar_wait(mb, *bm.phase, bm.abort);   // completed: returns at once
    *bm.phase ^= 1;
    pp = (const float*)smem_raw;
  }
  const int cg = (tid & 7) * 4;
  for (int q = tid >> 3; q < NQ; q += AM_THREADS / 8) {
    float o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = 0.f;
    float l = 0.f, M = -INFINITY;
    for (int s0 = 0; s0 < S_all; s0 += 4) {
      float2 ml[4];
      float4 os[4][4];
#pragma unroll
      for (int u2 = 0; u2 < 4; ++u2) {
        if (s0 + u2 < S_all) {
          const float* w = pp + ((size_t)(s0 + u2) * NQ + q) * AM_PSTRIDE;
          if constexpr (BULK) {
            ml[u2] = *(const float2*)(w + AM_DH);
#pragma unroll
            for (int i = 0; i < 4; ++i) os[u2][i] = *(const float4*)(w + cg + 32 * i);
          } else {
            ml[u2] = __ldcg((const float2*)(w + AM_DH));
#pragma unroll
            for (int i = 0; i < 4; ++i) os[u2][i] = __ldcg((const float4*)(w + cg + 32 * i));
          }
        } else {
          ml[u2] = make_float2(-INFINITY, 0.f);
        }
      }
#pragma unroll
      for (int u2 = 0; u2 < 4; ++u2) {
        if (ml[u2].x == -INFINITY) continue;
        if (ml[u2].x > M) {
          const float f = (M == -INFINITY) ? 0.f : exp2f(M - ml[u2].x);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= f;
          l *= f;
          M = ml[u2].x;
        }
        const float f = exp2f(ml[u2].x - M);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          o[4 * i] += f * os[u2][i].x; o[4 * i + 1] += f * os[u2][i].y;
          o[4 * i + 2] += f * os[u2][i].z; o[4 * i + 3] += f * os[u2][i].w;
        }
        l += f * ml[u2].y;
      }
    }
    const float inv = 1.f / l;
    const int j = q / 16, i = q % 16;
    bf16* dst = out + (size_t)(row0 + j * a.K + i) * a.d + h * AM_DH + cg;
#pragma unroll
    for (int g = 0; g < 4; ++g)
      *(uint2*)(dst + 32 * g) = make_uint2(pack_bf16x2(o[4 * g] * inv, o[4 * g + 1] * inv),
                                           pack_bf16x2(o[4 * g + 2] * inv, o[4 * g + 3] * inv));
  }
  if (tid == 0) a.cnt[pair] = 0u;
}

template <int N>
__global__ void __launch_bounds__(AM_THREADS)
k_attn_mma(const bf16* __restrict__ qkv, const bf16* __restrict__ Kc, const bf16* __restrict__ Vc,
           bf16* __restrict__ out, AttnMmaArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ int s_last;
  attn_item<N, AM_STAGES, false>(qkv, Kc, Vc, out, a, blockIdx.x, blockIdx.y, smem_raw, &s_last, threadIdx.x,
               [] __device__() { __syncthreads(); });
}

template <int N, int ST = AM_STAGES>
constexpr int attn_mma_smem() {
  return (N * 16 + 2 * ST * AM_CHUNK) * AM_LD * 2;
}

}  // namespace fm
