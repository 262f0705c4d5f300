// C ABI of the flow-map drafter and verifier: context management and the
// orchestration of the kernels of one draft / verify call.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <vector>

#include "flashmap.h"
#include "fm_simt.cuh"
#include "fm_misc.cuh"
#include "fm_verify.cuh"
#include "fm_tc.cuh"
#include "fm_attn.cuh"
#include "fm_dit.cuh"
#include "fm_tree.cuh"

using fm::bf16;

// ------------------------------------------------------------------ errors
static thread_local char g_err[1024] = "no error";

static fm_status set_err(fm_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

#define FM_CUDA(call)                                                               \
  do {                                                                              \
    cudaError_t e_ = (call);                                                        \
    if (e_ != cudaSuccess)                                                          \
      return set_err(FM_ERR_CUDA, "%s failed: %s (%s:%d)", #call,                   \
                     cudaGetErrorString(e_), __FILE__, __LINE__);                   \
  } while (0)
#define FM_LAUNCHED() FM_CUDA(cudaGetLastError())
#define FM_TRY(expr)                  \
  do {                                \
    fm_status s_ = (expr);            \
    if (s_ != FM_OK) return s_;       \
  } while (0)

extern "C" const char* fm_last_error(void) { return g_err; }

// ------------------------------------------------------------------ context
namespace {

constexpr int N_MOD_SLOTS = 8;

struct ModSlot {
  bool valid = false;
  float s = 0.f, t = 0.f;
  float* buf = nullptr;  // [n_blocks][6][d] then [2][d], fp32
  unsigned long long stamp = 0;
};

}  // namespace

struct fm_ctx {
  fm_config cfg;
  int dev = 0, sms = 148;
  size_t esz = 4;
  fm_weights w;
  std::vector<const void*> wqkv, wo, wup, wdown, wada;
  void* wkv_all = nullptr;       // every block's key and value weights stacked [nb][2d][d] (bf16)
  std::vector<void*> owned;  // every cudaMalloc of the context
  void* Et = nullptr;        // E transposed, [d][V]
  std::vector<void*> Kc, Vc; // per block [max_seqs][max_ctx][d]
  std::vector<int> ctx_len;  // host copy of each slot's context length
  ModSlot mods[N_MOD_SLOTS];
  unsigned long long clock = 0;
  float *P = nullptr, *phi = nullptr, *tv = nullptr;  // tv: 5 x d time-MLP scratch
  int M_max = 0, R_max = 0;
  float *x = nullptr, *z = nullptr, *logits = nullptr;
  void *h = nullptr, *qkv = nullptr, *o = nullptr, *u = nullptr, *D = nullptr;
  float* part_v = nullptr;
  int* part_i = nullptr;
  float* smp_max = nullptr;      // chunked sampling: chunk maxima and weight sums per row
  double* smp_sum = nullptr;
  int32_t* fac_tok = nullptr;    // factorised drafting: tokens and uniforms of all K drafts
  double* fac_u = nullptr;
  int n_part = 0;
  float* splitk = nullptr;
  size_t splitk_elems = 0;
  unsigned* tile_cnt = nullptr;
  int tile_cnt_n = 0;
  float* c_raw = nullptr;
  void* c_norm = nullptr;
  // context rows projected by fc + LN but whose keys/values are not yet in
  // the cache: the next draft computes them inside its QKV GEMMs (same
  // W_k, W_v), or they are flushed by separate GEMMs
  int pending_rows = 0;
  fm::RowMap pending_map;
  int v_chunks = 1;
  float* vg_pv = nullptr;
  int* vg_pi = nullptr;
  unsigned* vg_cnt = nullptr;
  int* tree_rowmap = nullptr;    // target row of each (sequence, draft, position) of a tree
  unsigned* dit_flags = nullptr; // persistent DiT pass: abort word, completion counters and
  size_t dit_flags_n = 0;        //   flags, LayerNorm tile statistics, final LayerNorm output
  float* dit_stats = nullptr;
  void* dit_hf = nullptr;
  bool dit_ok = false;           // the persistent pass fits this configuration and device
  bool dit_stall_once = false;   // test hook (FM_TEST_STALL=1): the next pass's first wait never ends
  int dit_l2_ahead = 0;          // weight k-blocks the persistent pass prefetches into L2 (measured: no gain)
  float* attn_part = nullptr;   // split-KV attention partials
  unsigned* attn_cnt = nullptr;
  size_t attn_part_elems = 0;
  int attn_pairs_max = 0;
  float* vs_pm = nullptr;
  double* vs_ps = nullptr;
  double* vs_resid = nullptr;
  // the tree's stochastic verify over many CTAs per sequence: per-chunk
  // partial sums [max_seqs][VT_MAX_CHUNKS], abort word + one barrier
  // counter per sequence, resident CTAs of that kernel per SM
  double* vt_part = nullptr;
  unsigned* vt_bar = nullptr;
  int vt_per_sm = 0;
  fm::Vs1Plan* vs1_plan = nullptr;   // one-draft stochastic verify: the draw of each sequence
  double* vs1_csum = nullptr;        //   and its per-chunk weight sums
  bool use_tc = false;
  // LayerNorm inside the consuming GEMM (measured slower than a LayerNorm
  // kernel followed by the GEMM at 16 rows; kept off)
  bool ln_in_gemm = false;
  fm::TcMaps tc;  // tensor maps of the weight operands (tensor-core path)
  // launch counts and optional device timing per kernel class
  long long launches[FM_PROF_N] = {};
  int prof_mask = 0;
  std::vector<cudaEvent_t> ev_a, ev_b;
  std::vector<int> ev_cls;
  size_t ev_used = 0;
};

namespace {

fm_status dalloc(fm_ctx* c, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return set_err(FM_ERR_OOM, "cudaMalloc(%zu bytes) failed: %s", bytes, cudaGetErrorString(e));
  }
  c->owned.push_back(*p);
  return FM_OK;
}
template <typename P>
fm_status dalloc_t(fm_ctx* c, P** p, size_t count) {
  void* v = nullptr;
  fm_status s = dalloc(c, &v, count * sizeof(P));
  *p = (P*)v;
  return s;
}

// Records an event pair around the launches of one operation when its class
// is being timed.
struct Prof {
  fm_ctx* c;
  cudaStream_t st;
  long slot = -1;
  Prof(fm_ctx* c_, int cls, cudaStream_t st_) : c(c_), st(st_) {
    if (((c->prof_mask >> cls) & 1) && c->ev_used < c->ev_a.size()) {
      slot = (long)c->ev_used++;
      c->ev_cls[slot] = cls;
      record(c->ev_a[slot]);
    }
  }
  ~Prof() {
    if (slot >= 0) record(c->ev_b[slot]);
  }
  // inside a stream capture only "external" records become timing records
  // of the graph; outside a capture the plain record is the valid one
  void record(cudaEvent_t e) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
      cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    else
      cudaEventRecord(e, st);
  }
};

// Every kernel goes out with programmatic stream serialization (see
// fm::pdl_wait): it may start while its predecessor drains.
#define FM_LAUNCH(c, cls, kernel, grid, block, smem, st, ...)                               \
  do {                                                                                   \
    cudaError_t e_ = fm::launch_pdl(kernel, dim3(grid), dim3(block), smem, st, __VA_ARGS__); \
    (c)->launches[cls]++;                                                                \
    if (e_ != cudaSuccess)                                                               \
      return set_err(FM_ERR_CUDA, "launch of %s failed: %s (%s:%d)", #kernel,            \
                     cudaGetErrorString(e_), __FILE__, __LINE__);                        \
  } while (0)

int grid_1d(size_t n, int threads, int cap = 148 * 16) {
  size_t b = (n + threads - 1) / threads;
  if (b > (size_t)cap) b = cap;
  return b < 1 ? 1 : (int)b;
}

// ------------------------------------------------------------------ GEMM dispatch
// Y[M][N] = A[M][Kd] . W(n,k), W K-major ([N][ldw]) or N-major ([Kd][ldw]).
template <typename TA, typename TW, class Epi>
fm_status gemm_simt(fm_ctx* c, int cls, const TA* A, int lda, const TW* W, int ldw, bool wk, int M,
                    int N, int Kd, Epi epi, cudaStream_t st) {
  Prof prof(c, cls, st);
  dim3 grid((N + fm::SG_BN - 1) / fm::SG_BN, (M + fm::SG_BM - 1) / fm::SG_BM, 1);
  long tiles = (long)grid.x * grid.y;
  int splits = 1;
  if (tiles < 2L * c->sms && Kd >= 512) {
    splits = (int)((2L * c->sms + tiles - 1) / tiles);
    splits = std::min(splits, Kd / 256);
    splits = std::min(splits, 64);
    while (splits > 1 && (size_t)splits * M * N > c->splitk_elems) --splits;
    if (splits < 1) splits = 1;
  }
  int k_split = Kd;
  if (splits > 1) {
    k_split = (Kd + splits - 1) / splits;
    k_split = (k_split + fm::SG_BK - 1) / fm::SG_BK * fm::SG_BK;
    splits = (Kd + k_split - 1) / k_split;
  }
  grid.z = splits;
  if (wk)
    FM_LAUNCH(c, cls, (fm::k_gemm_simt<TA, TW, true, Epi>), grid, 256, 0, st,
              A, lda, W, ldw, M, N, Kd, k_split, c->splitk, epi);
  else
    FM_LAUNCH(c, cls, (fm::k_gemm_simt<TA, TW, false, Epi>), grid, 256, 0, st,
              A, lda, W, ldw, M, N, Kd, k_split, c->splitk, epi);
  if (splits > 1)
    FM_LAUNCH(c, cls, (fm::k_splitk_apply<Epi>), grid_1d((size_t)M * N, 256), 256, 0, st,
              c->splitk, splits, M, N, epi);
  return FM_OK;
}

// Weight GEMM for the DiT, fc and LM head: tensor cores for bf16 when the
// shape allows, CUDA cores otherwise.
template <typename T, class Epi>
fm_status gemm_w(fm_ctx* c, int cls, const T* A, int lda, const T* W, int M, int N, int Kd,
                 Epi epi, cudaStream_t st, const fm::TcMap* map = nullptr) {
  if constexpr (sizeof(T) == 2) {
    if (c->use_tc && map && map->valid) {
      Prof prof(c, cls, st);
      int n_launch = 0;
      fm_status s = fm::tc_gemm(c->tc, *map, (const bf16*)A, lda, M, N, Kd, epi, c->splitk,
                                c->splitk_elems, c->tile_cnt, c->tile_cnt_n, c->sms, st, g_err,
                                sizeof(g_err), &n_launch);
      c->launches[cls] += n_launch;
      return s;
    }
  }
  return gemm_simt<T, T, Epi>(c, cls, A, lda, W, Kd, true, M, N, Kd, epi, st);
}

// GEMM whose input is the modulated LayerNorm of the residual stream,
// LN0(x)(1 + scale) + shift, computed inside the tensor-core kernel.  Sets
// *done = false (and launches nothing) when the shape needs the separate
// LayerNorm kernel instead.
template <class Epi>
fm_status gemm_ln(fm_ctx* c, int cls, const float* x, const float* shift, const float* scale,
                  int M, Epi epi, cudaStream_t st, const fm::TcMap* map, bool* done,
                  const bf16* extra = nullptr, int n_extra = 0, bool force = false) {
  *done = false;
  if (!c->use_tc || !map || !map->valid || M > 32 || !(c->ln_in_gemm || force)) return FM_OK;
  Prof prof(c, cls, st);
  int n_launch = 0;
  fm_status s = fm::tc_gemm_ln(c->tc, *map, x, shift, scale, M, extra, M + n_extra, epi, c->splitk,
                               c->splitk_elems, c->tile_cnt, c->tile_cnt_n, c->sms, st, g_err,
                               sizeof(g_err), &n_launch);
  c->launches[cls] += n_launch;
  if (s == FM_ERR_UNSUPPORTED) return FM_OK;
  if (s == FM_OK) *done = true;
  return s;
}

// ------------------------------------------------------------------ conditioning
template <typename T>
fm_status compute_mods(fm_ctx* c, float s, float t, float* out, cudaStream_t st) {
  const int d = c->cfg.d, nb = c->cfg.n_blocks;
  float* tv = c->tv;  // 5 slots of d
  auto gemv = [&](const void* W, int n_out, int n_in, const float* x, float* y, const float* add,
                  int act) -> fm_status {
    int threads = 256, blocks = (n_out * 32 + threads - 1) / threads;
    FM_LAUNCH(c, FM_PROF_OTHER, (fm::k_gemv<T>), blocks, threads, 0, st,
              (const T*)W, n_out, n_in, x, y, add, act);
    return FM_OK;
  };
  FM_LAUNCH(c, FM_PROF_OTHER, (fm::k_time_features), 1, 256, 0, st,
              (double)s, (double)t, c->phi);
  FM_TRY(gemv(c->w.W_ts1, d, 256, c->phi, tv, nullptr, 1));                // SiLU(W1 phi(s))
  FM_TRY(gemv(c->w.W_ts2, d, d, tv, tv + d, nullptr, 0));                 // TE_s(s)
  FM_TRY(gemv(c->w.W_tt1, d, 256, c->phi + 256, tv + 2 * d, nullptr, 1)); // SiLU(W1 phi(t))
  FM_TRY(gemv(c->w.W_tt2, d, d, tv + 2 * d, tv + 3 * d, tv + d, 0));      // c = TE_s + TE_t
  FM_LAUNCH(c, FM_PROF_OTHER, (fm::k_silu_vec), (d + 255) / 256, 256, 0, st,
              tv + 3 * d, tv + 4 * d, d);
  for (int l = 0; l < nb; ++l)
    FM_TRY(gemv(c->wada[l], 6 * d, d, tv + 4 * d, out + (size_t)l * 6 * d, nullptr, 0));
  FM_TRY(gemv(c->w.W_ada_f, 2 * d, d, tv + 4 * d, out + (size_t)nb * 6 * d, nullptr, 0));
  return FM_OK;
}

template <typename T>
fm_status get_mods(fm_ctx* c, float s, float t, const float** out, cudaStream_t st) {
  for (auto& m : c->mods)
    if (m.valid && m.s == s && m.t == t) {
      m.stamp = ++c->clock;
      *out = m.buf;
      return FM_OK;
    }
  ModSlot* victim = &c->mods[0];
  for (auto& m : c->mods) {
    if (!m.valid) { victim = &m; break; }
    if (m.stamp < victim->stamp) victim = &m;
  }
  victim->valid = false;
  FM_TRY(compute_mods<T>(c, s, t, victim->buf, st));
  victim->valid = true;
  victim->s = s;
  victim->t = t;
  victim->stamp = ++c->clock;
  *out = victim->buf;
  return FM_OK;
}

// ------------------------------------------------------------------ load
template <typename T>
fm_status load_impl(fm_ctx* c, cudaStream_t st) {
  const fm_config& g = c->cfg;
  const int d = g.d;
  FM_TRY(dalloc(c, &c->Et, (size_t)g.V * d * sizeof(T)));
  {
    dim3 grid((d + 31) / 32, (g.V + 31) / 32), block(32, 8);
    FM_LAUNCH(c, FM_PROF_OTHER, (fm::k_transpose<T>), grid, block, 0, st,
              (const T*)c->w.E, (T*)c->Et, g.V, d);
  }
  c->Kc.resize(g.n_blocks);
  c->Vc.resize(g.n_blocks);
  for (int l = 0; l < g.n_blocks; ++l) {
    size_t n = (size_t)g.max_seqs * g.max_ctx * d * sizeof(T);
    FM_TRY(dalloc(c, &c->Kc[l], n));
    FM_TRY(dalloc(c, &c->Vc[l], n));
  }
  c->ctx_len.assign(g.max_seqs, 0);
  for (auto& m : c->mods) FM_TRY(dalloc_t(c, &m.buf, (size_t)(g.n_blocks * 6 + 2) * d));
  FM_TRY(dalloc_t(c, &c->P, (size_t)g.K * d));
  FM_TRY(dalloc_t(c, &c->phi, 512));
  FM_TRY(dalloc_t(c, &c->tv, (size_t)5 * d));
  {
    std::vector<float> P((size_t)g.K * d);
    for (int i = 0; i < g.K; ++i)
      for (int k = 0; k < d / 2; ++k) {
        double w = pow(10000.0, -2.0 * k / d);
        P[(size_t)i * d + 2 * k] = (float)sin(i * w);
        P[(size_t)i * d + 2 * k + 1] = (float)cos(i * w);
      }
    FM_CUDA(cudaMemcpyAsync(c->P, P.data(), P.size() * sizeof(float), cudaMemcpyHostToDevice, st));
    FM_CUDA(cudaStreamSynchronize(st));
  }
  const int call_seqs = std::min(g.max_seqs, FM_MAX_CALL_SEQS);
  c->M_max = call_seqs * g.max_noise * g.K;
  c->R_max = call_seqs * g.max_new;
  const size_t M = c->M_max;
  FM_TRY(dalloc_t(c, &c->x, M * d));
  FM_TRY(dalloc_t(c, &c->z, M * d));
  FM_TRY(dalloc(c, &c->h, M * d * sizeof(T)));
  FM_TRY(dalloc(c, &c->qkv, M * 3 * d * sizeof(T)));
  FM_TRY(dalloc(c, &c->o, M * d * sizeof(T)));
  FM_TRY(dalloc(c, &c->u, M * g.mlp * sizeof(T)));
  FM_TRY(dalloc_t(c, &c->logits, M * g.V));
  FM_TRY(dalloc(c, &c->D, M * g.V * sizeof(T)));
  c->n_part = (g.V + 127) / 128;
  FM_TRY(dalloc_t(c, &c->smp_max, M * fm::SAMPLE_CHUNKS));
  FM_TRY(dalloc_t(c, &c->smp_sum, M * fm::SAMPLE_CHUNKS));
  FM_TRY(dalloc_t(c, &c->fac_tok, M));
  FM_TRY(dalloc_t(c, &c->fac_u, M));
  FM_TRY(dalloc_t(c, &c->part_v, M * c->n_part));
  FM_TRY(dalloc_t(c, &c->part_i, M * c->n_part));
  c->splitk_elems = std::max<size_t>((size_t)1 << 22, 8 * M * (size_t)std::max(3 * d, g.mlp));
  FM_TRY(dalloc_t(c, &c->splitk, c->splitk_elems));
  c->tile_cnt_n = 1 << 16;
  FM_TRY(dalloc_t(c, &c->tile_cnt, c->tile_cnt_n));
  FM_CUDA(cudaMemsetAsync(c->tile_cnt, 0, c->tile_cnt_n * sizeof(unsigned), st));
  c->attn_pairs_max = call_seqs * g.max_noise * g.n_heads;
  c->attn_part_elems = (size_t)(2 * c->sms + 2 * c->attn_pairs_max) * g.max_noise * 16 * fm::AM_PSTRIDE;
  FM_TRY(dalloc_t(c, &c->attn_part, c->attn_part_elems));
  FM_TRY(dalloc_t(c, &c->attn_cnt, (size_t)c->attn_pairs_max));
  FM_CUDA(cudaMemsetAsync(c->attn_cnt, 0, c->attn_pairs_max * sizeof(unsigned), st));
  // abort word, c_stats, c_o[nb], c_down[nb], f_qkv[nb][3d/128], f_head[nb][H], f_up[nb][F/128]
  c->dit_flags_n = 2 + 2 * (size_t)g.n_blocks +
                   (size_t)g.n_blocks * (3 * d / 128 + g.n_heads + g.mlp / 128);
  FM_TRY(dalloc_t(c, &c->dit_flags, c->dit_flags_n));
  FM_TRY(dalloc_t(c, &c->dit_stats, (size_t)(d / 128 + 1) * fm::DIT_M * 2));
  FM_TRY(dalloc(c, &c->dit_hf, (size_t)fm::DIT_M * d * sizeof(T)));
  FM_TRY(dalloc_t(c, &c->c_raw, (size_t)c->R_max * d));
  FM_TRY(dalloc(c, &c->c_norm, (size_t)c->R_max * d * sizeof(T)));
  // verify workspaces: rows = B*N*(K+1) target + B*N*K draft rows
  c->v_chunks = 64;
  const size_t vrows = (size_t)g.max_seqs * g.max_noise * (2 * g.K + 1);
  FM_TRY(dalloc_t(c, &c->vg_pv, vrows * c->v_chunks));
  FM_TRY(dalloc_t(c, &c->vg_pi, vrows * c->v_chunks));
  FM_TRY(dalloc_t(c, &c->vg_cnt, (size_t)g.max_seqs));
  FM_TRY(dalloc_t(c, &c->tree_rowmap, (size_t)g.max_seqs * g.max_noise * (g.K + 1)));
  FM_CUDA(cudaMemsetAsync(c->vg_cnt, 0, g.max_seqs * sizeof(unsigned), st));
  FM_TRY(dalloc_t(c, &c->vs_pm, vrows * c->v_chunks));
  FM_TRY(dalloc_t(c, &c->vs_ps, vrows * c->v_chunks));
  FM_TRY(dalloc_t(c, &c->vs_resid, (size_t)g.max_seqs * 2 * g.V));
  FM_TRY(dalloc_t(c, &c->vt_part, (size_t)g.max_seqs * fm::VT_MAX_CHUNKS));
  FM_TRY(dalloc_t(c, &c->vt_bar, (size_t)g.max_seqs + 1));
  {
    int coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c->dev);
    if (coop)
      FM_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c->vt_per_sm, fm::k_vtree,
                                                            fm::VT_THREADS, 0));
  }
  FM_TRY(dalloc_t(c, &c->vs1_plan, (size_t)g.max_seqs));
  FM_TRY(dalloc_t(c, &c->vs1_csum, (size_t)g.max_seqs * fm::VS1_CHUNKS * 2));
  FM_TRY(dalloc_t(c, &c->tc.err, 1));
  FM_CUDA(cudaMemsetAsync(c->tc.err, 0, sizeof(int), st));
  if constexpr (sizeof(T) == 2) {
    const char* off = getenv("FM_DISABLE_TC");  // diagnostic: force the CUDA-core GEMMs
    c->use_tc = fm::tc_supported(g.d, g.mlp, g.V, g.n_taps * g.target_hidden) && !(off && *off == '1');
    if (c->use_tc) {
      if (!fm::tc_make_maps(c->tc, c->w.W_lm, c->Et, c->w.W_fc, c->wqkv.data(), c->wo.data(),
                            c->wup.data(), c->wdown.data(), g.n_blocks, g.d, g.mlp, g.V,
                            g.n_taps * g.target_hidden, g_err, sizeof(g_err)))
        return FM_ERR_CUDA;
      // the keys and values of appended context rows for every block come
      // from one GEMM over the stacked key/value weights (one launch, and
      // enough output tiles to fill the SMs even for a few rows)
      if (g.n_blocks <= 8) {
        const size_t per = (size_t)2 * d * d;
        FM_TRY(dalloc(c, &c->wkv_all, (size_t)g.n_blocks * per * sizeof(T)));
        for (int l = 0; l < g.n_blocks; ++l)
          FM_CUDA(cudaMemcpyAsync((T*)c->wkv_all + (size_t)l * per, (const T*)c->wqkv[l] + (size_t)d * d,
                                  per * sizeof(T), cudaMemcpyDeviceToDevice, st));
        if (!fm::tc_weight_map(c->tc.kv_all, c->wkv_all, g.n_blocks * 2 * d, d, g_err, sizeof(g_err)))
          return FM_ERR_CUDA;
      }
    }
  }
  if constexpr (sizeof(T) == 2) {
    // diagnostic: split-K GEMMs reduce through global memory only
    const char* ncl = getenv("FM_DISABLE_TC_CLUSTER");
    fm::tc_cluster_ok = !(ncl && *ncl == '1');
    int coop = 0;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c->dev);
    const char* off = getenv("FM_DISABLE_PERSISTENT");  // diagnostic: per-kernel DiT path
    c->dit_ok = c->use_tc && coop && !(off && *off == '1') && g.n_blocks <= fm::DIT_MAX_BLOCKS &&
                d / g.n_heads == fm::AM_DH && g.K == fm::DIT_M && d % 128 == 0 && g.mlp % 128 == 0 &&
                d / 128 <= c->sms;
    if (c->dit_ok) {
      FM_CUDA(fm::set_smem_once(fm::k_dit_persistent, fm::DIT_SMEM));
      int per_sm = 0;
      FM_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fm::k_dit_persistent,
                                                            fm::TC_THREADS, fm::DIT_SMEM));
      c->dit_ok = per_sm >= 1;
    }
    // test hook: the next persistent pass waits for a count no phase
    // reaches, so its bounded wait runs out (failure-path test; no fault)
    const char* stall = getenv("FM_TEST_STALL");
    c->dit_stall_once = stall && *stall == '1';
    // diagnostic: L2 prefetch depth of the persistent pass (k-blocks, 0 = off)
    const char* ahead = getenv("FM_DIT_L2_AHEAD");
    if (ahead) c->dit_l2_ahead = std::max(0, std::min(256, atoi(ahead)));
  }
  // the grids every draft uses
  const float grids[3][2] = {{0.f, 1.f}, {0.f, 0.5f}, {0.5f, 1.f}};
  for (auto& gp : grids) {
    const float* tmp;
    FM_TRY(get_mods<T>(c, gp[0], gp[1], &tmp, st));
  }
  FM_CUDA(cudaStreamSynchronize(st));
  return FM_OK;
}

// ------------------------------------------------------------------ context projection
template <typename T>
fm_status flush_pending(fm_ctx* c, cudaStream_t st) {
  if (c->pending_rows == 0) return FM_OK;
  const fm_config& g = c->cfg;
  const int d = g.d, R = c->pending_rows;
  if constexpr (sizeof(T) == 2) {
   if (c->use_tc && c->tc.kv_all.valid) {
    fm::EpiCtxKVAll<T> ea;
    for (int l = 0; l < g.n_blocks; ++l) {
      ea.Kc[l] = (T*)c->Kc[l];
      ea.Vc[l] = (T*)c->Vc[l];
    }
    ea.d = d;
    ea.max_ctx = g.max_ctx;
    ea.map = c->pending_map;
    FM_TRY(gemm_w<T>(c, FM_PROF_CONTEXT, (const T*)c->c_norm, d, (const T*)c->wkv_all, R,
                     g.n_blocks * 2 * d, d, ea, st, &c->tc.kv_all));
    c->pending_rows = 0;
    return FM_OK;
   }
  }
  fm::EpiCtxKV<T> epi;
  epi.d = d;
  epi.max_ctx = g.max_ctx;
  epi.map = c->pending_map;
  for (int l = 0; l < g.n_blocks; ++l) {
    epi.Kc = (T*)c->Kc[l];
    epi.Vc = (T*)c->Vc[l];
    const T* Wkv = (const T*)c->wqkv[l] + (size_t)d * d;  // key and value thirds
    FM_TRY(gemm_w<T>(c, FM_PROF_CONTEXT, (const T*)c->c_norm, d, Wkv, R, 2 * d, d, epi, st,
                     &c->tc.kv[l]));
  }
  c->pending_rows = 0;
  return FM_OK;
}

// Rows that a following one-step draft of at most this many block rows can
// absorb into its QKV GEMMs (one 64-row activation tile).
constexpr int FUSED_CTX_ROWS = 64;

template <typename T>
fm_status project_impl(fm_ctx* c, const int32_t* seq_ids, int n_seqs, const void* hidden,
                       int n_new, const int32_t* pos0, cudaStream_t st) {
  const fm_config& g = c->cfg;
  const int d = g.d, R = n_seqs * n_new, in = g.n_taps * g.target_hidden;
  FM_TRY(flush_pending<T>(c, st));   // c_norm is about to be overwritten
  FM_TRY(gemm_w<T>(c, FM_PROF_CONTEXT, (const T*)hidden, in, (const T*)c->w.W_fc, R, d, in,
                   fm::EpiStoreF32{c->c_raw, d}, st, &c->tc.fc));
  {
    Prof prof(c, FM_PROF_CONTEXT, st);
    FM_LAUNCH(c, FM_PROF_CONTEXT, (fm::k_adaln<float, T>), R, 256, 0, st,
              c->c_raw, d, nullptr, nullptr, (T*)c->c_norm);
  }
  c->pending_map.n_seqs = n_seqs;
  c->pending_map.n_new = n_new;
  for (int q = 0; q < n_seqs; ++q) {
    c->pending_map.slot[q] = seq_ids[q];
    c->pending_map.pos0[q] = pos0[q];
  }
  c->pending_rows = R;
  // keys/values now unless a small draft can take them over
  // keys/values now unless a following draft can take them over: the
  // persistent pass (one 16-row draft) or an in-GEMM LayerNorm path
  const bool absorb = sizeof(T) == 2 && c->use_tc &&
                      ((c->ln_in_gemm && R < FUSED_CTX_ROWS) ||
                       (c->dit_ok && fm::DIT_M + R <= fm::DIT_BROWS_MAX));
  if (!absorb) FM_TRY(flush_pending<T>(c, st));
  for (int q = 0; q < n_seqs; ++q) c->ctx_len[seq_ids[q]] = pos0[q] + n_new;
  return FM_OK;
}

// ------------------------------------------------------------------ attention
template <int N>
fm_status attn_mma_launch(fm_ctx* c, const fm::AttnMmaArgs& am, dim3 grid, const bf16* qkv,
                          const bf16* Kc, const bf16* Vc, bf16* o, cudaStream_t st) {
  constexpr int smem = fm::attn_mma_smem<N>();
  FM_CUDA(fm::set_smem_once(fm::k_attn_mma<N>, smem));
  FM_LAUNCH(c, FM_PROF_ATTN, (fm::k_attn_mma<N>), grid, fm::AM_THREADS, smem, st,
              qkv, Kc, Vc, o, am);
  return FM_OK;
}

// Whether attn_mma can run every noise draft of n_seqs sequences as its own
// one-draft sequence.
static bool attn_split_drafts_ok(const fm_ctx* c, int n_seqs, int n_noise) {
  return n_seqs * n_noise <= 256 && n_seqs * n_noise * c->cfg.n_heads <= c->attn_pairs_max;
}

// Split count: about two CTAs per SM over all (sequence, head) pairs, at
// most one 64-row chunk per split when the context is short.
fm_status attn_mma(fm_ctx* c, int n_noise, fm::AttnMmaArgs am, const bf16* qkv, const bf16* Kc,
                   const bf16* Vc, bf16* o, int n_seqs, int max_len, cudaStream_t st) {
  // Few sequences with several noise drafts: one CTA per (draft, head,
  // split) instead of one per (sequence, head, split).  The drafts' rows are
  // consecutive [sequence][draft][K], so draft j of sequence b is "sequence"
  // b n_noise + j of one draft with b's context; the CTAs of a context slice
  // run together and share its reads in L2, and each head's merge covers
  // 16 query rows instead of n_noise * 16.
  const bool tiled = n_noise == 1 || n_noise == 2 || n_noise == 4;
  if (n_noise > 1 && attn_split_drafts_ok(c, n_seqs, n_noise) &&
      (!tiled || n_seqs * am.n_heads < c->sms)) {
    for (int q = n_seqs - 1; q >= 0; --q)
      for (int j = n_noise - 1; j >= 0; --j) {
        am.slot[q * n_noise + j] = am.slot[q];
        am.len[q * n_noise + j] = am.len[q];
      }
    n_seqs *= n_noise;
    n_noise = 1;
    am.n_seqs = n_seqs;
    am.n_noise = 1;
  }
  const int pairs = n_seqs * am.n_heads;
  // at most about two CTAs per SM, and at least four 64-row chunks per split:
  // every extra split adds a partial to the final merge
  int s_ctx = (2 * c->sms + pairs - 1) / pairs - 1;
  s_ctx = std::min(s_ctx, (max_len + 4 * fm::AM_CHUNK - 1) / (4 * fm::AM_CHUNK));
  s_ctx = std::max(s_ctx, 1);
  while (s_ctx > 1 &&
         (size_t)pairs * (s_ctx + 1) * n_noise * 16 * fm::AM_PSTRIDE > c->attn_part_elems)
    --s_ctx;
  am.n_ctx_splits = s_ctx;
  dim3 grid(pairs, s_ctx + 1);
  switch (n_noise) {
    case 1: return attn_mma_launch<1>(c, am, grid, qkv, Kc, Vc, o, st);
    case 2: return attn_mma_launch<2>(c, am, grid, qkv, Kc, Vc, o, st);
    default: return attn_mma_launch<4>(c, am, grid, qkv, Kc, Vc, o, st);
  }
}

// ------------------------------------------------------------------ persistent DiT pass
// One cooperative launch for all blocks of one 16-row draft (one sequence,
// one noise draft); leaves the final modulated LayerNorm in c->dit_hf.
// Returns FM_ERR_UNSUPPORTED (nothing launched) when a limit does not hold.
fm_status dit_persistent(fm_ctx* c, const float* mods, int slot, int ctx_len, bool with_ctx,
                         cudaStream_t st) {
  const fm_config& g = c->cfg;
  const int d = g.d, G = c->sms;
  fm::DitParams P;
  memset(&P, 0, sizeof(P));
  for (int l = 0; l < g.n_blocks; ++l) {
    P.w[l][0] = c->tc.qkv[l].map;
    P.w[l][1] = c->tc.o[l].map;
    P.w[l][2] = c->tc.up[l].map;
    P.w[l][3] = c->tc.down[l].map;
    P.Kc[l] = (bf16*)c->Kc[l];
    P.Vc[l] = (bf16*)c->Vc[l];
  }
  P.n_blocks = g.n_blocks;
  P.d = d;
  P.F = g.mlp;
  P.M = fm::DIT_M;
  P.l2_ahead = c->dit_l2_ahead;
  P.skip_final = 0;
  P.stall = c->dit_stall_once ? 1 : 0;
  // K splits per GEMM kind: about one unit per SM
  const int tiles[5] = {3 * d / 128, 0, d / 128, g.mlp / 128, d / 128};
  const int kbs[5] = {d / 64, 0, d / 64, d / 64, g.mlp / 64};
  for (int k : {fm::DIT_QKV, fm::DIT_O, fm::DIT_UP, fm::DIT_DOWN}) {
    if (tiles[k] > G) return FM_ERR_UNSUPPORTED;
    P.splits[k] = std::max(1, std::min(G / tiles[k], kbs[k]));
  }
  P.x = c->x;
  P.stats = c->dit_stats;
  P.partial = c->splitk;
  P.tile_cnt = c->tile_cnt;
  {
    unsigned* f = c->dit_flags;
    const int nb = g.n_blocks;
    P.abort_g = (int*)f;
    P.c_stats = f + 1;
    P.c_o = f + 2;
    P.c_down = P.c_o + nb;
    P.f_qkv = P.c_down + nb;
    P.f_head = P.f_qkv + (size_t)nb * (3 * d / 128);
    P.f_up = P.f_head + (size_t)nb * g.n_heads;
  }
  P.err = c->tc.err;
  P.qkv = (bf16*)c->qkv;
  P.o = (bf16*)c->o;
  P.u = (bf16*)c->u;
  P.hf = (bf16*)c->dit_hf;
  P.mods = mods;
  P.max_ctx = g.max_ctx;
  P.n_ctx = 0;
  if (with_ctx && c->pending_rows > 0) {
    P.n_ctx = c->pending_rows;
    P.ctx_rows = (const bf16*)c->c_norm;
    P.ctx_map = c->pending_map;
  }
  if (fm::DIT_M + P.n_ctx > fm::DIT_BROWS_MAX) return FM_ERR_UNSUPPORTED;
  // shared-memory and workspace limits of every phase; each GEMM kind keeps
  // its own split-K region and tile counters (consecutive phases overlap)
  size_t part_total = 0;
  for (int k : {fm::DIT_QKV, fm::DIT_O, fm::DIT_UP, fm::DIT_DOWN}) {
    const int brows = (k == fm::DIT_QKV && P.n_ctx) ? (fm::DIT_M + P.n_ctx + 15) / 16 * 16 : 16;
    const int nkb = (kbs[k] + P.splits[k] - 1) / P.splits[k];
    if ((size_t)nkb * brows * 128 > (size_t)fm::DIT_UNION) return FM_ERR_UNSUPPORTED;
    if (nkb * 64 > 1024) return FM_ERR_UNSUPPORTED;  // staged shift/scale slice
    // the B operand is published in at most two batches of 8 k-blocks on one
    // mbarrier, so the MMA issuer can never fall two phases behind
    if (nkb > 16) return FM_ERR_UNSUPPORTED;
    // staged partial tiles, below the tile-statistics scratch at the end
    if ((size_t)P.splits[k] * 128 * brows * 4 > (size_t)(fm::DIT_UNION - fm::DIT_TS_BYTES))
      return FM_ERR_UNSUPPORTED;
    if (tiles[k] > 1024 || 4 * 1024 > c->tile_cnt_n) return FM_ERR_UNSUPPORTED;
    P.part_off[k] = part_total;
    part_total += (size_t)P.splits[k] * tiles[k] * 128 * brows;
  }
  if (part_total > c->splitk_elems) return FM_ERR_UNSUPPORTED;
  fm::AttnMmaArgs& am = P.attn;
  am.n_seqs = 1;
  am.n_noise = 1;
  am.K = g.K;
  am.d = d;
  am.n_heads = g.n_heads;
  am.max_ctx = g.max_ctx;
  am.scale_log2 = (float)(1.4426950408889634 / sqrt((double)fm::AM_DH));
  am.part = c->attn_part;
  am.cnt = c->attn_cnt;
  am.slot[0] = slot;
  am.len[0] = ctx_len;
  // context rows this pass appends (keys/values written by its QKV phases)
  P.attn_safe = ctx_len;
  for (int q = 0; q < (P.n_ctx ? P.ctx_map.n_seqs : 0); ++q)
    if (P.ctx_map.slot[q] == slot) P.attn_safe = std::min(P.attn_safe, P.ctx_map.pos0[q]);
  // context splits of whole 64-row chunks below the appended rows, at least
  // a full ring (two chunks) each, so a split's first chunks load before its
  // queries exist; the rows from the last whole chunk on (appended rows
  // included) ride with the block's own rows
  const int s_max = G / g.n_heads - 1;
  if (s_max < 1) return FM_ERR_UNSUPPORTED;
  const int base = P.attn_safe / fm::AM_CHUNK * fm::AM_CHUNK;
  const int per = (base + s_max * fm::AM_CHUNK - 1) / (s_max * fm::AM_CHUNK) * fm::AM_CHUNK;
  am.split_rows = std::max(fm::DIT_ATTN_ST * fm::AM_CHUNK, per);
  am.tail0 = base;
  int s_ctx = std::max(1, (base + am.split_rows - 1) / am.split_rows);
  if (ctx_len - base + 16 > fm::DIT_ATTN_ST * fm::AM_CHUNK) return FM_ERR_UNSUPPORTED;
  if (g.n_heads * (s_ctx + 1) > G) return FM_ERR_UNSUPPORTED;
  if ((size_t)g.n_heads * (s_ctx + 1) * 16 * fm::AM_PSTRIDE > c->attn_part_elems)
    return FM_ERR_UNSUPPORTED;
  // a head's split partials are merged in shared memory
  if ((size_t)(s_ctx + 1) * 16 * fm::AM_PSTRIDE * 4 > (size_t)fm::DIT_UNION) return FM_ERR_UNSUPPORTED;
  am.n_ctx_splits = s_ctx;
  P.splits[fm::DIT_ATTN] = s_ctx;
  // Measured: a programmatic launch (the pass's weight stream starting
  // under x.E's tail, the LM head's under the pass's) with the flags cleared
  // by the pass's last CTA instead of this memset made the pass 3.6 us
  // slower and the end-to-end round 20-35 us slower
  FM_CUDA(cudaMemsetAsync(c->dit_flags, 0, c->dit_flags_n * sizeof(unsigned), st));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(fm::TC_THREADS);
  cfg.dynamicSmemBytes = fm::DIT_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    Prof prof(c, FM_PROF_DIT_GEMM, st);
    FM_CUDA(cudaLaunchKernelEx(&cfg, fm::k_dit_persistent, P));
  }
  c->launches[FM_PROF_DIT_GEMM]++;
  c->dit_stall_once = false;
  if (P.n_ctx) c->pending_rows = 0;
  return FM_OK;
}

// ------------------------------------------------------------------ draft
template <typename T>
fm_status draft_impl(fm_ctx* c, const int32_t* seq_ids, int n_seqs, const void* noise,
                     int n_noise, const float* t_grid, int num_steps, const float* temps,
                     const double* u_draft, int32_t* tokens, float* draft_logits,
                     cudaStream_t st) {
  const fm_config& g = c->cfg;
  const int d = g.d, K = g.K, V = g.V, nb = g.n_blocks, F = g.mlp;
  const int M = n_seqs * n_noise * K;
  T* h = (T*)c->h;
  T* qkv = (T*)c->qkv;
  T* o = (T*)c->o;
  T* u = (T*)c->u;
  fm::AttnArgs aa;
  aa.n_seqs = n_seqs;
  aa.n_noise = n_noise;
  aa.K = K;
  aa.d = d;
  aa.n_heads = g.n_heads;
  aa.max_ctx = g.max_ctx;
  aa.scale = (float)(1.0 / sqrt((double)(d / g.n_heads)));
  for (int q = 0; q < n_seqs; ++q) {
    aa.slot[q] = seq_ids[q];
    aa.len[q] = c->ctx_len[seq_ids[q]];
  }
  // tensor-core (mma.sync) split-KV attention for bf16, head width 128
  const bool use_mma_attn = sizeof(T) == 2 && d / g.n_heads == fm::AM_DH && K == 16 &&
                            (n_noise == 1 || n_noise == 2 || n_noise == 4 ||
                             attn_split_drafts_ok(c, n_seqs, n_noise));
  fm::AttnMmaArgs am;
  int max_len = 0;
  if (use_mma_attn) {
    am.split_rows = 0;
    am.tail0 = 0;
    am.n_seqs = n_seqs;
    am.n_noise = n_noise;
    am.K = K;
    am.d = d;
    am.n_heads = g.n_heads;
    am.max_ctx = g.max_ctx;
    am.scale_log2 = (float)(1.4426950408889634 / sqrt((double)fm::AM_DH));
    am.part = c->attn_part;
    am.cnt = c->attn_cnt;
    for (int q = 0; q < n_seqs; ++q) {
      am.slot[q] = seq_ids[q];
      am.len[q] = c->ctx_len[seq_ids[q]];
      max_len = std::max(max_len, am.len[q]);
    }
  }
  bool any_sample = false;
  fm::TempArgs ta;
  ta.n_noise = n_noise;
  ta.K = K;
  for (int q = 0; q < n_seqs; ++q) {
    ta.temp[q] = temps[q];
    any_sample |= temps[q] > 0.f;
  }
  float* logits = draft_logits ? draft_logits : c->logits;
  // context rows whose keys/values are still pending: the first step's QKV
  // GEMMs compute them when the rows fit one activation tile, else now
  bool fuse_ctx = false;
  const bool will_persist = sizeof(T) == 2 && c->dit_ok && M == fm::DIT_M && n_seqs == 1;
  if (c->pending_rows > 0) {
    if (sizeof(T) == 2 && c->use_tc && c->ln_in_gemm && M <= 32 &&
        M + c->pending_rows <= FUSED_CTX_ROWS)
      fuse_ctx = true;
    else if (!will_persist)   // the persistent pass takes them over
      FM_TRY(flush_pending<T>(c, st));
  }
  for (int k = 0; k < num_steps; ++k) {
    const float s = t_grid[k], t = t_grid[k + 1];
    const bool last = (k == num_steps - 1);
    const float* mods;
    FM_TRY(get_mods<T>(c, s, t, &mods, st));
    // input embedding (first step: x0 E; later: flow-map update through E)
    // the state entering step k moved by the previous step's flow-map update,
    // alpha = (t_k - t_{k-1}) / (1 - t_{k-1})
    float alpha = -1.f;
    if (k > 0) {
      const double sp = t_grid[k - 1], tp = t_grid[k];
      alpha = (float)((tp - sp) / (1.0 - sp));
    }
    fm::EpiEmbed emb{c->x, num_steps > 1 ? c->z : nullptr, c->P, d, K, alpha};
    const T* A = (k == 0) ? (const T*)noise : (const T*)c->D;
    if (c->use_tc && c->tc.embed.valid) {
      FM_TRY(gemm_w<T>(c, FM_PROF_EMBED, A, V, (const T*)c->Et, M, d, V, emb, st, &c->tc.embed));
    } else {
      FM_TRY((gemm_simt<T, T, fm::EpiEmbed>(c, FM_PROF_EMBED, A, V, (const T*)c->w.E, d, false, M,
                                             d, V, emb, st)));
    }
    bool persistent = false;
    if constexpr (sizeof(T) == 2) {
      if (will_persist) {
        fm_status ps = dit_persistent(c, mods, seq_ids[0], c->ctx_len[seq_ids[0]], k == 0, st);
        if (ps == FM_OK) persistent = true;
        else if (ps != FM_ERR_UNSUPPORTED) return ps;
      }
    }
    if (!persistent && c->pending_rows > 0 && !fuse_ctx) FM_TRY(flush_pending<T>(c, st));
    for (int l = 0; l < nb && !persistent; ++l) {
      const float* ml = mods + (size_t)l * 6 * d;
      bool fused = false;
      if constexpr (sizeof(T) == 2) {
        if (fuse_ctx) {
          // this step's QKV GEMM also projects the pending context rows
          fm::EpiQkvCtx<T> e;
          e.qkv = qkv;
          e.ld = 3 * d;
          e.M_draft = M;
          e.d = d;
          e.kv.Kc = (T*)c->Kc[l];
          e.kv.Vc = (T*)c->Vc[l];
          e.kv.d = d;
          e.kv.max_ctx = g.max_ctx;
          e.kv.map = c->pending_map;
          FM_TRY(gemm_ln(c, FM_PROF_DIT_GEMM, c->x, ml, ml + d, M, e, st, &c->tc.qkv[l], &fused,
                         (const bf16*)c->c_norm, c->pending_rows));
          if (!fused) {
            if (l > 0) return set_err(FM_ERR_CUDA, "fused context projection stopped at block %d", l);
            fuse_ctx = false;
            FM_TRY(flush_pending<T>(c, st));
          }
        }
      }
      if (!fused)
        FM_TRY(gemm_ln(c, FM_PROF_DIT_GEMM, c->x, ml, ml + d, M, fm::EpiStore<T>{qkv, 3 * d}, st,
                       &c->tc.qkv[l], &fused));
      if (!fused) {
        {
          Prof prof(c, FM_PROF_NORM, st);
          FM_LAUNCH(c, FM_PROF_NORM, (fm::k_adaln<float, T>), M, 256, 0, st,
                c->x, d, ml, ml + d, h);
        }
        FM_TRY(gemm_w<T>(c, FM_PROF_DIT_GEMM, h, d, (const T*)c->wqkv[l], M, 3 * d, d,
                         fm::EpiStore<T>{qkv, 3 * d}, st, &c->tc.qkv[l]));
      }
      {
        Prof prof(c, FM_PROF_ATTN, st);
        if (use_mma_attn) {
          FM_TRY(attn_mma(c, n_noise, am, (const bf16*)qkv, (const bf16*)c->Kc[l],
                          (const bf16*)c->Vc[l], (bf16*)o, n_seqs, max_len, st));
        } else {
          dim3 grid(n_seqs, g.n_heads, n_noise);
          FM_LAUNCH(c, FM_PROF_ATTN, (fm::k_attn_simt<T>), grid, 128, 0, st,
              qkv, (const T*)c->Kc[l], (const T*)c->Vc[l], o, aa);
        }
      }
      FM_TRY(gemm_w<T>(c, FM_PROF_DIT_GEMM, o, d, (const T*)c->wo[l], M, d, d,
                       fm::EpiResidual{c->x, ml + 2 * d, d}, st, &c->tc.o[l]));
      FM_TRY(gemm_ln(c, FM_PROF_DIT_GEMM, c->x, ml + 3 * d, ml + 4 * d, M, fm::EpiGelu<T>{u, F}, st,
                     &c->tc.up[l], &fused));
      if (!fused) {
        {
          Prof prof(c, FM_PROF_NORM, st);
          FM_LAUNCH(c, FM_PROF_NORM, (fm::k_adaln<float, T>), M, 256, 0, st,
                c->x, d, ml + 3 * d, ml + 4 * d, h);
        }
        FM_TRY(gemm_w<T>(c, FM_PROF_DIT_GEMM, h, d, (const T*)c->wup[l], M, F, d,
                         fm::EpiGelu<T>{u, F}, st, &c->tc.up[l]));
      }
      FM_TRY(gemm_w<T>(c, FM_PROF_DIT_GEMM, u, F, (const T*)c->wdown[l], M, d, F,
                       fm::EpiResidual{c->x, ml + 5 * d, d}, st, &c->tc.down[l]));
    }
    if (fuse_ctx) {
      c->pending_rows = 0;
      fuse_ctx = false;
    }
    const float* mf = mods + (size_t)nb * 6 * d;
    // LM head: greedy-only final steps keep the logits on chip when possible
    const bool need_logits = !last || any_sample || draft_logits != nullptr;
    bool have_partials = false, fused = false;
    if (persistent) {
      fused = true;
      if (need_logits) {
        FM_TRY(gemm_w<T>(c, FM_PROF_LM_HEAD, (const T*)c->dit_hf, d, (const T*)c->w.W_lm, M, V, d,
                         fm::EpiStoreF32{logits, V}, st, &c->tc.lm));
      } else {
        Prof prof(c, FM_PROF_LM_HEAD, st);
        int n_launch = 0;
        FM_TRY(fm::tc_lm_head_argmax(c->tc, (const bf16*)c->dit_hf, d, M, V, c->part_v, c->part_i,
                                     c->n_part, c->sms, st, g_err, sizeof(g_err), &n_launch));
        c->launches[FM_PROF_LM_HEAD] += n_launch;
        have_partials = true;
      }
    } else if (need_logits) {
      FM_TRY(gemm_ln(c, FM_PROF_LM_HEAD, c->x, mf, mf + d, M, fm::EpiStoreF32{logits, V}, st,
                     &c->tc.lm, &fused));
    } else {
      FM_TRY(gemm_ln(c, FM_PROF_LM_HEAD, c->x, mf, mf + d, M,
                     fm::EpiArgmax{c->part_v, c->part_i, c->n_part}, st, &c->tc.lm, &fused));
      have_partials = fused;
    }
    if (!fused) {
      {
        Prof prof(c, FM_PROF_NORM, st);
        FM_LAUNCH(c, FM_PROF_NORM, (fm::k_adaln<float, T>), M, 256, 0, st, c->x, d, mf, mf + d, h);
      }
      if (c->use_tc && c->tc.lm.valid && !need_logits) {
        Prof prof(c, FM_PROF_LM_HEAD, st);
        int n_launch = 0;
        FM_TRY(fm::tc_lm_head_argmax(c->tc, (const bf16*)h, d, M, V, c->part_v, c->part_i,
                                     c->n_part, c->sms, st, g_err, sizeof(g_err), &n_launch));
        c->launches[FM_PROF_LM_HEAD] += n_launch;
        have_partials = true;
      } else {
        FM_TRY(gemm_w<T>(c, FM_PROF_LM_HEAD, h, d, (const T*)c->w.W_lm, M, V, d,
                         fm::EpiStoreF32{logits, V}, st, &c->tc.lm));
      }
    }
    Prof prof(c, FM_PROF_NORM, st);
    if (!last) {
      // a cluster of CTAs per row, up to four, about two CTAs per SM; 512
      // threads, so registers admit two CTAs per SM (measured: 1,024 threads
      // of 44 registers fit one per SM and ran in two waves, 44 us)
      const int C = std::max(1, std::min(4, 2 * c->sms / std::max(1, M)));
      const cudaError_t e_ = fm::launch_pdl_cluster(fm::k_softmax_rows<T>, dim3(M * C), dim3(512),
                                                    0, st, (unsigned)C, (const float*)logits, V, M,
                                                    (T*)c->D);
      c->launches[FM_PROF_NORM]++;
      if (e_ != cudaSuccess)
        return set_err(FM_ERR_CUDA, "launch of k_softmax_rows failed: %s", cudaGetErrorString(e_));
    } else {
      // greedy rows (and, with few sampled rows, the sampled ones) one CTA
      // per row; many sampled rows through the chunked sampler
      const bool chunked = any_sample && !have_partials && M >= 64;
      FM_LAUNCH(c, FM_PROF_NORM, (fm::k_select_tokens), M, 1024, 0, st,
              have_partials ? nullptr : logits, V, have_partials ? c->part_v : nullptr,
                    have_partials ? c->part_i : nullptr, c->n_part, u_draft, ta, tokens,
                    chunked ? 1 : 0);
      if (chunked) {
        FM_LAUNCH(c, FM_PROF_NORM, fm::k_sample_chunk_max, M * fm::SAMPLE_CHUNKS, 256, 0, st,
                  (const float*)logits, V, ta, c->smp_max);
        FM_LAUNCH(c, FM_PROF_NORM, fm::k_sample_chunk_sum, M * fm::SAMPLE_CHUNKS, 256, 0, st,
                  (const float*)logits, V, ta, (const float*)c->smp_max, c->smp_sum);
        FM_LAUNCH(c, FM_PROF_NORM, fm::k_sample_pick, M, 512, 0, st, (const float*)logits, V,
                  u_draft, ta, (const float*)c->smp_max, (const double*)c->smp_sum, tokens);
      }
    }
  }
  return FM_OK;
}

fm_status check_cfg(const fm_config* g) {
  if (!g) return set_err(FM_ERR_ARG, "cfg is NULL");
  if (g->V < 2 || g->d < 2 || g->n_blocks < 1 || g->n_heads < 1 || g->mlp < 1 || g->K < 1 ||
      g->target_hidden < 1 || g->n_taps < 1 || g->max_ctx < 1 || g->max_seqs < 1 ||
      g->max_noise < 1 || g->max_new < 1)
    return set_err(FM_ERR_ARG, "config sizes must be positive");
  if (g->d % g->n_heads || (g->d / g->n_heads) > fm::SA_MAXDH || (g->d & 1))
    return set_err(FM_ERR_ARG, "d must be even and d/n_heads <= %d", fm::SA_MAXDH);
  if (g->K > fm::SA_MAXQ) return set_err(FM_ERR_UNSUPPORTED, "K must be <= %d", fm::SA_MAXQ);
  if (g->max_noise > 32) return set_err(FM_ERR_UNSUPPORTED, "max_noise must be <= 32");
  if (g->max_noise * (g->K + 1) > fm::VG_MAX_ROWS)
    return set_err(FM_ERR_UNSUPPORTED, "max_noise*(K+1) must be <= %d", fm::VG_MAX_ROWS);
  if (g->dtype != FM_F32 && g->dtype != FM_BF16) return set_err(FM_ERR_ARG, "bad dtype");
  return FM_OK;
}

}  // namespace

// ------------------------------------------------------------------ ABI
extern "C" fm_status fm_load_weights(fm_ctx** out, const fm_config* cfg, const fm_weights* w,
                                     fm_stream stream) {
  if (!out) return set_err(FM_ERR_ARG, "out is NULL");
  *out = nullptr;
  FM_TRY(check_cfg(cfg));
  if (!w || !w->E || !w->W_lm || !w->W_fc || !w->W_ts1 || !w->W_ts2 || !w->W_tt1 || !w->W_tt2 ||
      !w->W_ada_f || !w->W_qkv || !w->W_o || !w->W_up || !w->W_down || !w->W_ada)
    return set_err(FM_ERR_ARG, "a weight pointer is NULL");
  fm_ctx* c = new fm_ctx();
  c->cfg = *cfg;
  c->w = *w;
  c->esz = cfg->dtype == FM_BF16 ? 2 : 4;
  for (int l = 0; l < cfg->n_blocks; ++l) {
    if (!w->W_qkv[l] || !w->W_o[l] || !w->W_up[l] || !w->W_down[l] || !w->W_ada[l]) {
      delete c;
      return set_err(FM_ERR_ARG, "block %d weight pointer is NULL", l);
    }
    c->wqkv.push_back(w->W_qkv[l]);
    c->wo.push_back(w->W_o[l]);
    c->wup.push_back(w->W_up[l]);
    c->wdown.push_back(w->W_down[l]);
    c->wada.push_back(w->W_ada[l]);
  }
  c->w.W_qkv = c->w.W_o = c->w.W_up = c->w.W_down = c->w.W_ada = nullptr;
  cudaError_t e = cudaGetDevice(&c->dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->dev);
  if (e != cudaSuccess) {
    delete c;
    return set_err(FM_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
  }
  cudaStream_t st = (cudaStream_t)stream;
  fm_status s = cfg->dtype == FM_BF16 ? load_impl<bf16>(c, st) : load_impl<float>(c, st);
  if (s != FM_OK) {
    char keep[sizeof(g_err)];
    memcpy(keep, g_err, sizeof(keep));
    fm_free(c);
    memcpy(g_err, keep, sizeof(keep));
    return s;
  }
  *out = c;
  return FM_OK;
}

extern "C" void fm_free(fm_ctx* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  for (void* p : c->owned) cudaFree(p);
  for (auto e : c->ev_a) cudaEventDestroy(e);
  for (auto e : c->ev_b) cudaEventDestroy(e);
  fm::tc_free_maps(c->tc);
  delete c;
}

extern "C" fm_status fm_project_context(fm_ctx* c, const int32_t* seq_ids, int n_seqs,
                                        const void* hidden, int n_new, const int32_t* pos0,
                                        fm_stream stream) {
  if (!c || !seq_ids || !hidden || !pos0) return set_err(FM_ERR_ARG, "NULL argument");
  const fm_config& g = c->cfg;
  if (n_seqs < 1 || n_seqs > FM_MAX_CALL_SEQS || n_seqs > g.max_seqs)
    return set_err(FM_ERR_ARG, "n_seqs=%d out of range", n_seqs);
  if (n_new < 1 || n_new > g.max_new) return set_err(FM_ERR_ARG, "n_new=%d out of range", n_new);
  std::vector<char> seen(g.max_seqs, 0);
  for (int q = 0; q < n_seqs; ++q) {
    if (seq_ids[q] < 0 || seq_ids[q] >= g.max_seqs || seen[seq_ids[q]])
      return set_err(FM_ERR_ARG, "seq_ids[%d]=%d invalid or repeated", q, seq_ids[q]);
    seen[seq_ids[q]] = 1;
    if (pos0[q] < 0 || pos0[q] + n_new > g.max_ctx)
      return set_err(FM_ERR_ARG, "pos0[%d]=%d: rows exceed max_ctx=%d", q, pos0[q], g.max_ctx);
  }
  cudaStream_t st = (cudaStream_t)stream;
  return g.dtype == FM_BF16 ? project_impl<bf16>(c, seq_ids, n_seqs, hidden, n_new, pos0, st)
                            : project_impl<float>(c, seq_ids, n_seqs, hidden, n_new, pos0, st);
}

static fm_status check_draft(fm_ctx* c, const int32_t* seq_ids, int n_seqs, const void* noise,
                             int n_noise, const float* t_grid, int num_steps,
                             const float* temperature, const double* u_draft,
                             const int32_t* tokens) {
  if (!c || !seq_ids || !noise || !t_grid || !temperature || !tokens)
    return set_err(FM_ERR_ARG, "NULL argument");
  const fm_config& g = c->cfg;
  if (n_seqs < 1 || n_seqs > FM_MAX_CALL_SEQS || n_seqs > g.max_seqs)
    return set_err(FM_ERR_ARG, "n_seqs=%d out of range", n_seqs);
  if (n_noise < 1 || n_noise > g.max_noise)
    return set_err(FM_ERR_ARG, "n_noise=%d out of range", n_noise);
  if (num_steps < 1 || num_steps > FM_MAX_STEPS)
    return set_err(FM_ERR_ARG, "num_steps=%d out of range", num_steps);
  if (t_grid[0] != 0.f || t_grid[num_steps] != 1.f)
    return set_err(FM_ERR_ARG, "t_grid must start at 0 and end at 1");
  for (int k = 0; k < num_steps; ++k)
    if (!(t_grid[k] < t_grid[k + 1])) return set_err(FM_ERR_ARG, "t_grid must increase");
  for (int q = 0; q < n_seqs; ++q) {
    if (seq_ids[q] < 0 || seq_ids[q] >= g.max_seqs)
      return set_err(FM_ERR_ARG, "seq_ids[%d]=%d invalid", q, seq_ids[q]);
    if (!(temperature[q] >= 0.f)) return set_err(FM_ERR_ARG, "temperature[%d] < 0", q);
    if (temperature[q] > 0.f && !u_draft)
      return set_err(FM_ERR_ARG, "u_draft is NULL but sequence %d samples", q);
  }
  return FM_OK;
}

extern "C" fm_status fm_draft(fm_ctx* c, const int32_t* seq_ids, int n_seqs, const void* noise,
                              int n_noise, const float* t_grid, int num_steps,
                              const float* temperature, const double* u_draft, int32_t* tokens,
                              float* draft_logits, fm_stream stream) {
  FM_TRY(check_draft(c, seq_ids, n_seqs, noise, n_noise, t_grid, num_steps, temperature, u_draft,
                     tokens));
  const fm_config& g = c->cfg;
  cudaStream_t st = (cudaStream_t)stream;
  return g.dtype == FM_BF16
             ? draft_impl<bf16>(c, seq_ids, n_seqs, noise, n_noise, t_grid, num_steps, temperature,
                                u_draft, tokens, draft_logits, st)
             : draft_impl<float>(c, seq_ids, n_seqs, noise, n_noise, t_grid, num_steps,
                                 temperature, u_draft, tokens, draft_logits, st);
}

extern "C" fm_status fm_draft_factorised(fm_ctx* c, const int32_t* seq_ids, int n_seqs,
                                         const void* noise, const float* t_grid, int num_steps,
                                         const float* temperature, const double* u_draft,
                                         int32_t* tokens, float* draft_logits, fm_stream stream) {
  if (!c) return set_err(FM_ERR_ARG, "NULL argument");
  const fm_config& g = c->cfg;
  const int K = g.K, V = g.V;
  FM_TRY(check_draft(c, seq_ids, n_seqs, noise, 1, t_grid, num_steps, temperature, u_draft, tokens));
  if (g.max_noise < K)
    return set_err(FM_ERR_UNSUPPORTED, "factorised drafting needs max_noise >= K = %d", K);
  bool any_sample = false;
  for (int q = 0; q < n_seqs; ++q) any_sample |= temperature[q] > 0.f;
  cudaStream_t st = (cudaStream_t)stream;
  // position i of every draft uses the uniform of position i; only draft i's
  // position i is kept
  if (any_sample)
    FM_LAUNCH(c, FM_PROF_NORM, fm::k_repeat_u, grid_1d((size_t)n_seqs * K * K, 256), 256, 0, st,
              u_draft, c->fac_u, n_seqs, K);
  float* all_logits = draft_logits ? c->logits : nullptr;
  fm_status s = g.dtype == FM_BF16
                    ? draft_impl<bf16>(c, seq_ids, n_seqs, noise, K, t_grid, num_steps, temperature,
                                       any_sample ? c->fac_u : nullptr, c->fac_tok, all_logits, st)
                    : draft_impl<float>(c, seq_ids, n_seqs, noise, K, t_grid, num_steps, temperature,
                                        any_sample ? c->fac_u : nullptr, c->fac_tok, all_logits, st);
  FM_TRY(s);
  FM_LAUNCH(c, FM_PROF_NORM, fm::k_take_diagonal, n_seqs * K, 256, 0, st, (const int*)c->fac_tok,
            (const float*)all_logits, n_seqs, K, V, tokens, draft_logits);
  return FM_OK;
}

static fm_status check_verify(fm_ctx* c, const void* tgt, const void* draft, int B, int N, int K,
                              int V, const void* n_acc, const void* branch, const void* out) {
  if (!c || !tgt || !draft || !n_acc || !branch || !out) return set_err(FM_ERR_ARG, "NULL argument");
  const fm_config& g = c->cfg;
  if (B < 1 || B > g.max_seqs) return set_err(FM_ERR_ARG, "B=%d out of range", B);
  if (N < 1 || N > g.max_noise) return set_err(FM_ERR_ARG, "N=%d out of range", N);
  if (K != g.K || V != g.V) return set_err(FM_ERR_UNSUPPORTED, "K/V differ from the configuration");
  return FM_OK;
}

static int verify_chunks(fm_ctx* c, long rows, int V) {
  long want = (2L * c->sms + rows - 1) / rows;
  int ch = (int)std::min<long>(want, c->v_chunks);
  ch = std::min(ch, std::max(1, V / 1024));
  return std::max(ch, 1);
}

static fm_status verify_greedy_impl(fm_ctx* c, const float* target_logits, const int32_t* draft,
                                    int B, int N, int K, int V, int32_t* n_acc, int32_t* branch,
                                    int32_t* out_tokens, const int* rowmap, cudaStream_t st) {
  const long rows = (long)B * N * (K + 1);
  const int ch = verify_chunks(c, rows, V);
  Prof prof(c, FM_PROF_VERIFY, st);
  FM_LAUNCH(c, FM_PROF_VERIFY, (fm::k_verify_greedy), (unsigned)(rows * ch), fm::VG_THREADS, 0, st,
            target_logits, draft, B, N, K, V, ch, c->vg_pv, c->vg_pi, c->vg_cnt, n_acc, branch,
            out_tokens, rowmap);
  return FM_OK;
}

static fm_status verify_sample_impl(fm_ctx* c, const float* target_logits,
                                    const float* draft_logits, const int32_t* draft, int B, int N,
                                    int K, int V, float temperature, const double* u_accept,
                                    const double* u_res, int32_t* n_acc, int32_t* branch,
                                    int32_t* out_tokens, const int* rowmap, cudaStream_t st) {
  if (!(temperature > 0.f)) return set_err(FM_ERR_ARG, "temperature must be > 0");
  if (!u_accept || !u_res) return set_err(FM_ERR_ARG, "uniforms are NULL");
  const int n_tgt = B * N * (K + 1);
  const int n_rows = n_tgt + (draft_logits ? B * N * K : 0);
  const int ch = verify_chunks(c, n_rows, V);
  Prof prof(c, FM_PROF_VERIFY, st);
  FM_LAUNCH(c, FM_PROF_VERIFY, (fm::k_row_stats), (unsigned)((long)n_rows * ch), fm::VS_THREADS, 0, st,
            target_logits, draft_logits, n_tgt, n_rows, V, ch, temperature, c->vs_pm, c->vs_ps,
            rowmap);
  if (N == 1) {
    // one draft: a warp per sequence walks the depths, then the one draw is
    // summed and searched over many CTAs per sequence
    FM_LAUNCH(c, FM_PROF_VERIFY, fm::k_vs1_walk, (B + 3) / 4, 128, 0, st, target_logits, draft_logits,
              draft, B, K, V, temperature, u_accept, c->vs_pm, c->vs_ps, ch, c->vs1_plan, n_acc,
              branch, out_tokens, rowmap);
    FM_LAUNCH(c, FM_PROF_VERIFY, fm::k_vs1_sums, B * fm::VS1_CHUNKS, 256, 0, st, target_logits,
              draft_logits, V, temperature, (const fm::Vs1Plan*)c->vs1_plan, c->vs1_csum, rowmap);
    FM_LAUNCH(c, FM_PROF_VERIFY, fm::k_vs1_pick, B, 512, 0, st, target_logits, draft_logits, K, V,
              temperature, u_res, (const fm::Vs1Plan*)c->vs1_plan, (const double*)c->vs1_csum,
              out_tokens, rowmap);
    return FM_OK;
  }
  // the tree: C CTAs per sequence share each pass over the vocabulary
  // (cooperative launch, so the CTAs that wait on one another are resident)
  const long capacity = (long)c->sms * c->vt_per_sm;
  const int C = (int)std::min<long>({(long)fm::VT_MAX_CHUNKS, capacity / B, std::max(1, V / 1024)});
  if (C >= 2) {
    FM_CUDA(cudaMemsetAsync(c->vt_bar, 0, (size_t)(B + 1) * sizeof(unsigned), st));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(B * C));
    cfg.blockDim = dim3(fm::VT_THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    FM_CUDA(cudaLaunchKernelEx(&cfg, fm::k_vtree, target_logits, draft_logits, draft, B, N, K, V,
                               temperature, u_accept, u_res, (const float*)c->vs_pm,
                               (const double*)c->vs_ps, ch, c->vs_resid, C, c->vt_part, c->vt_bar,
                               c->tc.err, n_acc, branch, out_tokens, rowmap));
    c->launches[FM_PROF_VERIFY]++;
    return FM_OK;
  }
  FM_LAUNCH(c, FM_PROF_VERIFY, (fm::k_verify_sample_decide), B, fm::VS_DECIDE_THREADS, 0, st,
            target_logits, draft_logits, draft, B, N, K, V, temperature, u_accept, u_res, c->vs_pm,
            c->vs_ps, ch, c->vs_resid, n_acc, branch, out_tokens, rowmap);
  return FM_OK;
}

extern "C" fm_status fm_verify_greedy(fm_ctx* c, const float* target_logits, const int32_t* draft,
                                      int B, int N, int K, int V, int32_t* n_acc,
                                      int32_t* branch, int32_t* out_tokens, fm_stream stream) {
  FM_TRY(check_verify(c, target_logits, draft, B, N, K, V, n_acc, branch, out_tokens));
  return verify_greedy_impl(c, target_logits, draft, B, N, K, V, n_acc, branch, out_tokens, nullptr,
                            (cudaStream_t)stream);
}

extern "C" fm_status fm_verify_sample(fm_ctx* c, const float* target_logits,
                                      const float* draft_logits, const int32_t* draft, int B, int N,
                                      int K, int V, float temperature, const double* u_accept,
                                      const double* u_res, int32_t* n_acc, int32_t* branch,
                                      int32_t* out_tokens, fm_stream stream) {
  FM_TRY(check_verify(c, target_logits, draft, B, N, K, V, n_acc, branch, out_tokens));
  return verify_sample_impl(c, target_logits, draft_logits, draft, B, N, K, V, temperature, u_accept,
                            u_res, n_acc, branch, out_tokens, nullptr, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ tree of noise drafts
static fm_status check_tree_sizes(int B, int N, int K) {
  if (B < 1 || N < 1 || K < 1) return set_err(FM_ERR_ARG, "sizes must be positive");
  // each factor bounded before the product
  if (N > fm::TREE_MAX_DRAFTS || K > fm::TREE_MAX_NODES || N * K > fm::TREE_MAX_NODES)
    return set_err(FM_ERR_UNSUPPORTED, "a tree holds at most %d drafts and %d nodes",
                   fm::TREE_MAX_DRAFTS, fm::TREE_MAX_NODES);
  return FM_OK;
}

extern "C" fm_status fm_build_tree(const int32_t* draft, int B, int N, int K, int32_t* node_token,
                                   int32_t* node_parent, int32_t* node_depth, int32_t* n_nodes,
                                   int32_t* draft_node, uint64_t* anc_mask, fm_stream stream) {
  if (!draft || !node_token || !node_parent || !node_depth || !n_nodes || !draft_node || !anc_mask)
    return set_err(FM_ERR_ARG, "NULL argument");
  FM_TRY(check_tree_sizes(B, N, K));
  const int NN = N * K, W = (NN + 63) / 64;
  cudaError_t e = fm::launch_pdl(fm::k_build_tree, dim3(B), dim3(32), 0, (cudaStream_t)stream,
                                 (const int*)draft, N, K, NN, W, (int*)node_token,
                                 (int*)node_parent, (int*)node_depth, (int*)n_nodes,
                                 (int*)draft_node, anc_mask);
  if (e != cudaSuccess) return set_err(FM_ERR_CUDA, "tree build launch failed: %s", cudaGetErrorString(e));
  return FM_OK;
}

extern "C" fm_status fm_tree_attention(const float* q, const float* k_ctx, const float* v_ctx,
                                       const float* k_nodes, const float* v_nodes,
                                       const uint64_t* anc_mask, const int32_t* n_nodes, int B,
                                       int NN, int L, int n_heads, int dh, float* out,
                                       fm_stream stream) {
  if (!q || !k_nodes || !v_nodes || !anc_mask || !n_nodes || !out || (L > 0 && (!k_ctx || !v_ctx)))
    return set_err(FM_ERR_ARG, "NULL argument");
  if (B < 1 || NN < 1 || L < 0 || n_heads < 1 || dh < 1)
    return set_err(FM_ERR_ARG, "sizes must be positive");
  if (NN > fm::TREE_MAX_NODES || dh > 128 || n_heads > 1024)
    return set_err(FM_ERR_UNSUPPORTED, "at most %d nodes, head width 128", fm::TREE_MAX_NODES);
  const long warps = (long)B * NN * n_heads;
  if (warps > (1L << 31)) return set_err(FM_ERR_UNSUPPORTED, "too many (node, head) pairs");
  const int W = (NN + 63) / 64;
  cudaError_t e = fm::launch_pdl(fm::k_tree_attention, dim3((unsigned)((warps + 3) / 4)), dim3(128), 0,
                                 (cudaStream_t)stream, q, k_ctx, v_ctx, k_nodes, v_nodes, anc_mask,
                                 (const int*)n_nodes, B, NN, L, n_heads, dh, W,
                                 (float)(1.0 / sqrt((double)dh)), out);
  if (e != cudaSuccess) return set_err(FM_ERR_CUDA, "tree attention launch failed: %s", cudaGetErrorString(e));
  return FM_OK;
}

static fm_status tree_rowmap(fm_ctx* c, const int32_t* draft_node, int B, int N, int K, int R,
                             cudaStream_t st) {
  if (!draft_node) return set_err(FM_ERR_ARG, "NULL argument");
  if (R < 1 + N * K) return set_err(FM_ERR_ARG, "R=%d rows per sequence < 1 + N*K", R);
  FM_LAUNCH(c, FM_PROF_VERIFY, fm::k_tree_rowmap, grid_1d((size_t)B * N * (K + 1), 256), 256, 0, st,
            (const int*)draft_node, B, N, K, R, c->tree_rowmap);
  return FM_OK;
}

extern "C" fm_status fm_verify_greedy_tree(fm_ctx* c, const float* node_logits, int R,
                                           const int32_t* draft, const int32_t* draft_node, int B,
                                           int N, int K, int V, int32_t* n_acc, int32_t* branch,
                                           int32_t* out_tokens, fm_stream stream) {
  FM_TRY(check_verify(c, node_logits, draft, B, N, K, V, n_acc, branch, out_tokens));
  cudaStream_t st = (cudaStream_t)stream;
  FM_TRY(tree_rowmap(c, draft_node, B, N, K, R, st));
  return verify_greedy_impl(c, node_logits, draft, B, N, K, V, n_acc, branch, out_tokens,
                            c->tree_rowmap, st);
}

extern "C" fm_status fm_verify_sample_tree(fm_ctx* c, const float* node_logits, int R,
                                           const float* draft_logits, const int32_t* draft,
                                           const int32_t* draft_node, int B, int N, int K, int V,
                                           float temperature, const double* u_accept,
                                           const double* u_res, int32_t* n_acc, int32_t* branch,
                                           int32_t* out_tokens, fm_stream stream) {
  FM_TRY(check_verify(c, node_logits, draft, B, N, K, V, n_acc, branch, out_tokens));
  cudaStream_t st = (cudaStream_t)stream;
  FM_TRY(tree_rowmap(c, draft_node, B, N, K, R, st));
  return verify_sample_impl(c, node_logits, draft_logits, draft, B, N, K, V, temperature, u_accept,
                            u_res, n_acc, branch, out_tokens, c->tree_rowmap, st);
}

extern "C" fm_status fm_profile(fm_ctx* c, int mask) {
  if (!c) return set_err(FM_ERR_ARG, "NULL context");
  if (mask && c->ev_a.empty()) {
    const size_t n = 65536;
    c->ev_a.resize(n);
    c->ev_b.resize(n);
    c->ev_cls.assign(n, 0);
    for (size_t i = 0; i < n; ++i) {
      FM_CUDA(cudaEventCreate(&c->ev_a[i]));
      FM_CUDA(cudaEventCreate(&c->ev_b[i]));
    }
  }
  c->prof_mask = mask & ((1 << FM_PROF_N) - 1);
  c->ev_used = 0;
  return FM_OK;
}

extern "C" fm_status fm_profile_read(fm_ctx* c, double* ms, int64_t* launches, int reset) {
  if (!c) return set_err(FM_ERR_ARG, "NULL context");
  if (ms) {
    for (int k = 0; k < FM_PROF_N; ++k) ms[k] = 0.0;
    for (size_t i = 0; i < c->ev_used; ++i) {
      FM_CUDA(cudaEventSynchronize(c->ev_b[i]));
      float t = 0.f;
      FM_CUDA(cudaEventElapsedTime(&t, c->ev_a[i], c->ev_b[i]));
      ms[c->ev_cls[i]] += t;
    }
  }
  if (launches)
    for (int k = 0; k < FM_PROF_N; ++k) launches[k] = c->launches[k];
  if (reset) {
    for (int k = 0; k < FM_PROF_N; ++k) c->launches[k] = 0;
    c->ev_used = 0;
  }
  return FM_OK;
}

extern "C" fm_status fm_selftest_exp(const double* e, double* mine, double* ref, int n,
                                     fm_stream stream) {
  if (!e || !mine || !ref || n < 0) return set_err(FM_ERR_ARG, "NULL argument or n < 0");
  if (n == 0) return FM_OK;
  fm::k_selftest_exp<<<grid_1d((size_t)n, 256), 256, 0, (cudaStream_t)stream>>>(e, mine, ref, n);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return set_err(FM_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(err));
  return FM_OK;
}

extern "C" fm_status fm_device_status(fm_ctx* c, fm_stream stream) {
  if (!c) return set_err(FM_ERR_ARG, "NULL context");
  int v = 0;
  cudaStream_t st = (cudaStream_t)stream;
  FM_CUDA(cudaMemcpyAsync(&v, c->tc.err, sizeof(int), cudaMemcpyDeviceToHost, st));
  FM_CUDA(cudaStreamSynchronize(st));
  if (v) {
    // a kernel that gave up may have left arrival counters mid-count: they
    // return to zero here, so the context's next call starts clean (the
    // persistent pass's completion counters are zeroed before each launch)
    FM_CUDA(cudaMemsetAsync(c->tc.err, 0, sizeof(int), st));
    FM_CUDA(cudaMemsetAsync(c->tile_cnt, 0, c->tile_cnt_n * sizeof(unsigned), st));
    FM_CUDA(cudaMemsetAsync(c->attn_cnt, 0, c->attn_pairs_max * sizeof(unsigned), st));
    FM_CUDA(cudaMemsetAsync(c->vg_cnt, 0, c->cfg.max_seqs * sizeof(unsigned), st));
    FM_CUDA(cudaStreamSynchronize(st));
    return set_err(FM_ERR_TIMEOUT, "a bounded wait inside a tensor-core kernel gave up (code %d)", v);
  }
  return FM_OK;
}

// ------------------------------------------------------------------ greedy verify without allocation
// Some callers cannot allocate device memory at call time: inference servers
// that reserve the whole device in their own arena and forbid further
// cudaMalloc, and verify-only users who bring their own drafter and do not
// want a drafter context (fm_load_weights allocates the weight copy, caches
// and workspaces).  fm_verify_greedy_noalloc serves them: it runs the same
// greedy-verify kernel as fm_verify_greedy, with its scratch (per-chunk
// partial maxima and per-sequence arrival counters) in the file-scope device
// array below instead of a context's workspace.  Every GPU that loads the
// library holds this array (about 260 KB) until the process exits.
#define FM_NOALLOC_PARTIALS 32768  /* (row, vocabulary chunk) partials */
#define FM_NOALLOC_SEQS 1024       /* sequences per call */
#define FM_NOALLOC_MAX_V (1 << 28)  /* vocabulary entries per row */

namespace {
struct NoallocScratch {
  float pv[FM_NOALLOC_PARTIALS];
  int pi[FM_NOALLOC_PARTIALS];
  unsigned cnt[FM_NOALLOC_SEQS];
};
}  // namespace

static __device__ __align__(256) NoallocScratch g_noalloc_scratch;

// Device address of the scratch for the current device, looked up once per
// device (the name is only a host-side stand-in for the device symbol).
static fm_status noalloc_scratch(NoallocScratch** out, int* sms) {
  static std::mutex mu;
  static NoallocScratch* addr[64] = {};
  static int sm_count[64] = {};
  int dev = 0;
  FM_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return set_err(FM_ERR_UNSUPPORTED, "device id %d >= 64", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_err(FM_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    FM_CUDA(cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev));
    addr[dev] = (NoallocScratch*)p;
  }
  *out = addr[dev];
  *sms = sm_count[dev];
  return FM_OK;
}

extern "C" fm_status fm_verify_greedy_noalloc(const float* target_logits, const int32_t* draft,
                                              int B, int N, int K, int V, int32_t* n_acc,
                                              int32_t* branch, int32_t* out_tokens,
                                              fm_stream stream) {
  if (!target_logits || !draft || !n_acc || !branch || !out_tokens)
    return set_err(FM_ERR_ARG, "NULL argument");
  if (B < 1 || N < 1 || K < 1 || V < 1) return set_err(FM_ERR_ARG, "sizes must be positive");
  // each factor is bounded before any product is formed, and every product
  // is taken in 64 bits, so no size can wrap past these checks
  if (B > FM_NOALLOC_SEQS)
    return set_err(FM_ERR_UNSUPPORTED, "B=%d exceeds the no-allocation limit of %d sequences", B,
                   FM_NOALLOC_SEQS);
  if (N > fm::VG_MAX_ROWS || K > fm::VG_MAX_ROWS - 1)
    return set_err(FM_ERR_UNSUPPORTED, "N=%d or K=%d exceeds %d rows per sequence", N, K,
                   fm::VG_MAX_ROWS);
  if (V > FM_NOALLOC_MAX_V)
    return set_err(FM_ERR_UNSUPPORTED, "V=%d exceeds %d", V, FM_NOALLOC_MAX_V);
  const int64_t rows_b = (int64_t)N * ((int64_t)K + 1);
  if (rows_b > fm::VG_MAX_ROWS)
    return set_err(FM_ERR_UNSUPPORTED, "N*(K+1)=%lld exceeds %d rows per sequence",
                   (long long)rows_b, fm::VG_MAX_ROWS);
  const int64_t rows = (int64_t)B * rows_b;
  if (rows > FM_NOALLOC_PARTIALS)
    return set_err(FM_ERR_UNSUPPORTED, "B*N*(K+1)=%lld exceeds the no-allocation limit of %d rows",
                   (long long)rows, FM_NOALLOC_PARTIALS);
  NoallocScratch* s = nullptr;
  int sms = 148;
  FM_TRY(noalloc_scratch(&s, &sms));
  const int64_t want = (2 * (int64_t)sms + rows - 1) / rows;
  int ch = (int)std::min<int64_t>(want, 64);
  ch = std::min(ch, std::max(1, V / 1024));
  ch = (int)std::min<int64_t>(ch, FM_NOALLOC_PARTIALS / rows);
  ch = std::max(ch, 1);
  cudaStream_t st = (cudaStream_t)stream;
  // the counters start at zero (the kernel also returns them to zero)
  FM_CUDA(cudaMemsetAsync(s->cnt, 0, (size_t)B * sizeof(unsigned), st));
  cudaError_t e = fm::launch_pdl(fm::k_verify_greedy, dim3((unsigned)(rows * ch)),
                                 dim3(fm::VG_THREADS), 0, st, target_logits, draft, B, N, K, V, ch,
                                 s->pv, s->pi, s->cnt, n_acc, branch, out_tokens,
                                 (const int*)nullptr);
  if (e != cudaSuccess)
    return set_err(FM_ERR_CUDA, "greedy verify launch failed: %s", cudaGetErrorString(e));
  return FM_OK;
}
