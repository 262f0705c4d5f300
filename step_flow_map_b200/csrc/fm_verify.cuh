// Prefix verify of drafted blocks against target logits.
//
// Greedy: keep the drafted tokens while they equal the target argmax, then
// emit the target argmax (page "FlashMap Drafts 16 Dependent Tokens at
// Once…", section "Why drafting still costs time").  Stochastic: accept with
// probability min(1, p/q) and resample the normalised residual on
// rejection, trying the drafts of a tree in index order.
#pragma once
#include "fm_misc.cuh"
#include "fm_exp.cuh"
#include "fm_tc.cuh"

namespace fm {

// ------------------------------------------------------------------ greedy
// Grid: one CTA per (row, vocabulary chunk), rows = B*N*(K+1).  Each CTA
// writes its chunk's (max, lowest argmax); the last CTA of a sequence
// (arrival counter, no waiting) combines the chunks in order, counts the
// leading matches of every draft and writes the outputs.  The counter is
// returned to zero for the next launch.
constexpr int VG_THREADS = 256;
constexpr int VG_MAX_ROWS = 1024;  // N*(K+1) per sequence

__global__ void __launch_bounds__(VG_THREADS)
k_verify_greedy(const float* __restrict__ tgt, const int* __restrict__ draft, int B, int N,
                int K, int V, int chunks, float* __restrict__ pv, int* __restrict__ pi,
                unsigned* __restrict__ counter, int* __restrict__ n_acc,
                int* __restrict__ branch, int* __restrict__ out,
                const int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  __shared__ float shv[32];
  __shared__ int shi[32];
  __shared__ int amax[VG_MAX_ROWS];
  __shared__ int ydraft[VG_MAX_ROWS];   // N*K < N*(K+1) <= VG_MAX_ROWS
  __shared__ int is_last;
  const int rows_b = N * (K + 1);
  const int row = blockIdx.x / chunks, c = blockIdx.x - row * chunks;
  const int b = row / rows_b;
  const int per = (V + chunks - 1) / chunks;
  const int v0 = min(V, c * per), v1 = min(V, v0 + per);
  // a tree's rows come through its row map (shared prefixes share a row)
  const float* r = tgt + (size_t)(rowmap ? rowmap[row] : row) * V;
  ArgMax a{-INFINITY, 0x7fffffff};
  // 16-byte loads, four in flight per thread, compared in any order (ties go
  // to the lowest index)
  for_row_range(r, v0, v1, [&](int v, float x) {
    if (am_better(x, v, a.v, a.i)) { a.v = x; a.i = v; }
  });
  a = block_argmax(a, shv, shi);
  if (threadIdx.x == 0) {
    pv[(size_t)row * chunks + c] = a.v;
    pi[(size_t)row * chunks + c] = a.i;
    __threadfence();
    unsigned prev = atomicAdd(&counter[b], 1u);
    is_last = (prev == (unsigned)(rows_b * chunks - 1));
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // one warp per row: lanes take chunks (their loads in flight together),
  // the warp combines in chunk-index order of ties (lowest token wins)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int rr = warp; rr < rows_b; rr += nwarps) {
    const size_t base = ((size_t)b * rows_b + rr) * chunks;
    ArgMax m{-INFINITY, 0x7fffffff};
    for (int k0 = 0; k0 < chunks; k0 += 64) {
      float v[2];
      int i[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int k = k0 + u * 32 + lane;
        v[u] = k < chunks ? __ldcg(pv + base + k) : -INFINITY;
        i[u] = k < chunks ? __ldcg(pi + base + k) : 0x7fffffff;
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (am_better(v[u], i[u], m.v, m.i)) { m.v = v[u]; m.i = i[u]; }
    }
    m = warp_argmax(m);
    if (lane == 0) amax[rr] = (m.i == 0x7fffffff) ? 0 : m.i;
  }
  // the drafts of the sequence, staged by all threads
  for (int e = threadIdx.x; e < N * K; e += blockDim.x) ydraft[e] = draft[(size_t)b * N * K + e];
  __syncthreads();
  if (threadIdx.x == 0) {
    int best_n = -1, best_j = 0;
    for (int j = 0; j < N; ++j) {
      const int* y = ydraft + j * K;
      int n = 0;
      while (n < K && y[n] == amax[j * (K + 1) + n]) ++n;
      if (n > best_n) { best_n = n; best_j = j; }
    }
    const int* y = ydraft + best_j * K;
    int* o = out + (size_t)b * (K + 1);
    for (int i = 0; i < best_n; ++i) o[i] = y[i];
    o[best_n] = amax[best_j * (K + 1) + best_n];
    for (int i = best_n + 1; i <= K; ++i) o[i] = -1;
    n_acc[b] = best_n;
    branch[b] = best_j;
    counter[b] = 0u;
  }
}

// ------------------------------------------------------------------ stochastic
// Pass 1: per (row, chunk) the chunk max m_c and S_c = sum exp((l - m_c)/T)
// in fp64, for every target row and, when present, every draft row.  One
// read of the chunk: each thread keeps a running max and a sum relative to
// it (rescaled by exp((m_old - m_new)/T) when the max grows, which after
// the first few elements is rare), then the block takes the largest max
// and rescales every thread's sum to it.
constexpr int VS_THREADS = 256;

__global__ void __launch_bounds__(VS_THREADS)
k_row_stats(const float* __restrict__ tgt, const float* __restrict__ dlog, int n_tgt_rows,
            int n_rows, int V, int chunks, float T, float* __restrict__ pm,
            double* __restrict__ ps, const int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  __shared__ float shf[32];
  __shared__ double shd[32];
  const int row = blockIdx.x / chunks, c = blockIdx.x - row * chunks;
  const float* r = (row < n_tgt_rows) ? tgt + (size_t)(rowmap ? rowmap[row] : row) * V
                                      : dlog + (size_t)(row - n_tgt_rows) * V;
  const int per = (V + chunks - 1) / chunks;
  const int v0 = min(V, c * per), v1 = min(V, v0 + per);
  const double iT = 1.0 / (double)T;
  float mx = -INFINITY;
  double mxd = -INFINITY;   // mx as a double
  double s = 0.0;
  // one element: running max, the sum rescaled when the max grows
  auto one = [&](float x) {
    const double xd = (double)x;
    if (x > mx) {
      s = (mx == -INFINITY) ? 0.0 : s * exp_nonpos((mxd - xd) * iT);
      mx = x;
      mxd = xd;
    }
    if (x > -INFINITY) s += exp_nonpos((xd - mxd) * iT);
  };
  // the bulk: sixteen values per thread from four 16-byte loads in flight;
  // the max of the sixteen first (one rescale at most), then sixteen
  // independent exponentials into four partial sums (NaN never raises the
  // max -- fmaxf ignores it -- and adds nothing, as in `one`)
  int a = v0;
  while (a < v1 && ((reinterpret_cast<uintptr_t>(r + a) & 15) != 0)) {
    if (a - v0 == (int)threadIdx.x) one(r[a]);
    ++a;
  }
  const int nv = (v1 - a) >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(r + a);
  const int TT = blockDim.x;
  int i = threadIdx.x;
  for (; i + 3 * TT < nv; i += 4 * TT) {
    float x[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 q = __ldcs(r4 + i + k * TT);
      x[4 * k] = q.x; x[4 * k + 1] = q.y; x[4 * k + 2] = q.z; x[4 * k + 3] = q.w;
    }
    float bm = x[0];
#pragma unroll
    for (int k = 1; k < 16; ++k) bm = fmaxf(bm, x[k]);
    if (bm > mx) {
      const double bd = (double)bm;
      s = (mx == -INFINITY) ? 0.0 : s * exp_nonpos((mxd - bd) * iT);
      mx = bm;
      mxd = bd;
    }
    if (mx > -INFINITY) {
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (x[k] > -INFINITY) acc[k & 3] += exp_nonpos(((double)x[k] - mxd) * iT);
      s += (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
  }
  for (; i < nv; i += TT) {
    const float4 q = __ldcs(r4 + i);
    one(q.x); one(q.y); one(q.z); one(q.w);
  }
  for (int v = a + 4 * nv + (int)threadIdx.x; v < v1; v += TT) one(r[v]);
  const float M = block_max(mx, shf);
  double sc = (mx == -INFINITY) ? 0.0 : s * exp_nonpos(((double)mx - (double)M) * iT);
  sc = block_sum_d(sc, shd);
  if (threadIdx.x == 0) {
    pm[(size_t)row * chunks + c] = M;
    ps[(size_t)row * chunks + c] = sc;
  }
}

// Both exponentials of each argument, for the self-check entry point.
__global__ void k_selftest_exp(const double* __restrict__ e, double* __restrict__ mine,
                               double* __restrict__ ref, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    mine[i] = exp_nonpos(e[i]);
    ref[i] = exp(e[i]);
  }
}

struct RowStat {
  double m, S;
};
// Row statistics (max m, S = sum of exp((l - m)/T)) from the chunk partials,
// combined by one warp: lanes over chunks, a fixed shuffle tree
// (deterministic); every lane returns the result.
__device__ __forceinline__ RowStat warp_combine_stats(const float* pm, const double* ps, int row,
                                                      int chunks, double T, int lane) {
  double m = -INFINITY;
  for (int c = lane; c < chunks; c += 32) m = fmax(m, (double)pm[(size_t)row * chunks + c]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  double S = 0.0;
  for (int c = lane; c < chunks; c += 32) {
    const double mc = (double)pm[(size_t)row * chunks + c];
    if (mc > -INFINITY) S += ps[(size_t)row * chunks + c] * exp_nonpos((mc - m) / T);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  return RowStat{m, S};
}

// Pass 2: one CTA per sequence walks the depths.  Residual distributions
// are materialised, normalised, in a per-sequence fp64 ping-pong buffer
// [2][V]; a residual whose mass rounds to zero leaves p' unchanged.
constexpr int VS_DECIDE_THREADS = 512;

__global__ void __launch_bounds__(VS_DECIDE_THREADS)
k_verify_sample_decide(const float* __restrict__ tgt, const float* __restrict__ dlog,
                       const int* __restrict__ draft, int B, int N, int K, int V, float T,
                       const double* __restrict__ ua, const double* __restrict__ ures,
                       const float* __restrict__ pm, const double* __restrict__ ps, int chunks,
                       double* __restrict__ resid, int* __restrict__ n_acc,
                       int* __restrict__ branch, int* __restrict__ out,
                       const int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  __shared__ double shd[32];
  __shared__ int s_accept, s_mode, s_buf;
  __shared__ double s_mp, s_Sp, s_mq, s_Sq;
  const int b = blockIdx.x, tid = threadIdx.x;
  const double dT = (double)T, iT = 1.0 / dT;   // loops over V multiply by reciprocals
  const int n_tgt_rows = B * N * (K + 1);
  double* buf[2] = {resid + (size_t)b * 2 * V, resid + (size_t)b * 2 * V + V};
  int* o = out + (size_t)b * (K + 1);
  unsigned alive = (N >= 32) ? 0xffffffffu : ((1u << N) - 1u);
  int n_done = K;
  int r0 = 0;
  for (int i = 0; i < K; ++i) {
    r0 = __ffs(alive) - 1;
    const int trow = (b * N + r0) * (K + 1) + i;
    const float* tp = tgt + (size_t)(rowmap ? rowmap[trow] : trow) * V;
    if (tid < 32) {
      RowStat st = warp_combine_stats(pm, ps, trow, chunks, dT, tid);
      if (tid == 0) { s_mp = st.m; s_Sp = st.S; s_mode = 0; s_buf = 0; s_accept = -1; }
    }
    __syncthreads();
    for (int j = 0; j < N; ++j) {
      if (!((alive >> j) & 1u)) continue;
      const int y = draft[((size_t)b * N + j) * K + i];
      const int drow = (b * N + j) * K + i;
      const float* qp = dlog ? dlog + (size_t)drow * V : nullptr;
      if (tid < 32) {
        RowStat sq{0.0, 1.0};
        if (qp) sq = warp_combine_stats(pm, ps, n_tgt_rows + drow, chunks, dT, tid);
        if (tid == 0) {
          double qy = 1.0;
          if (qp) {
            s_mq = sq.m; s_Sq = sq.S;
            qy = exp(((double)qp[y] - sq.m) / dT) / sq.S;
          }
          double py = (s_mode == 0) ? exp(((double)tp[y] - s_mp) / dT) / s_Sp : buf[s_buf][y];
          s_accept = (ua[((size_t)b * N + j) * K + i] * qy < py) ? y : -1;
        }
      }
      __syncthreads();
      if (s_accept >= 0) break;
      // residual r = max(0, p' - q_j), then p' = r / sum(r)
      const int mode = s_mode, src = s_buf, dst = mode == 0 ? 0 : 1 - src;
      const double mp = s_mp, mq = s_mq;
      const double iSp = 1.0 / s_Sp, iSq = qp ? 1.0 / s_Sq : 0.0;
      double local = 0.0;
      for (int v = tid; v < V; v += blockDim.x) {
        double p = (mode == 0) ? exp_nonpos(((double)tp[v] - mp) * iT) * iSp : buf[src][v];
        double q = qp ? exp_nonpos(((double)qp[v] - mq) * iT) * iSq : (v == y ? 1.0 : 0.0);
        double r = fmax(p - q, 0.0);
        buf[dst][v] = r;
        local += r;
      }
      const double Z = block_sum_d(local, shd);
      if (Z > 0.0) {
        const double iZ = 1.0 / Z;
        for (int v = tid; v < V; v += blockDim.x) buf[dst][v] *= iZ;
        __syncthreads();
        if (tid == 0) { s_mode = 1; s_buf = dst; }
      } else if (mode == 0) {
        // p' stays the target row itself: materialise it for later steps
        for (int v = tid; v < V; v += blockDim.x) buf[dst][v] = exp_nonpos(((double)tp[v] - mp) * iT) * iSp;
        __syncthreads();
        if (tid == 0) { s_mode = 1; s_buf = dst; }
      }
      __syncthreads();
    }
    const int acc = s_accept;
    __syncthreads();
    if (acc < 0) {
      // sample the current p' at u_res
      const double u = ures[b];
      int tok;
      if (s_mode == 0) {
        const double mp = s_mp, iSp = 1.0 / s_Sp;
        auto wf = [&](int v) { return exp_nonpos(((double)tp[v] - mp) * iT) * iSp; };
        tok = block_sample(wf, V, u);
      } else {
        const double* pb = buf[s_buf];
        auto wf = [&](int v) { return pb[v]; };
        tok = block_sample(wf, V, u);
      }
      if (tid == 0) o[i] = tok;
      n_done = i;
      break;
    }
    if (tid == 0) o[i] = acc;
    unsigned keep = 0u;
    for (int j = 0; j < N; ++j)
      if (((alive >> j) & 1u) && draft[((size_t)b * N + j) * K + i] == acc) keep |= 1u << j;
    alive = keep;
  }
  if (n_done == K) {
    r0 = __ffs(alive) - 1;
    const int trow = (b * N + r0) * (K + 1) + K;
    const float* tp = tgt + (size_t)(rowmap ? rowmap[trow] : trow) * V;
    if (tid < 32) {
      RowStat st = warp_combine_stats(pm, ps, trow, chunks, dT, tid);
      if (tid == 0) { s_mp = st.m; s_Sp = st.S; }
    }
    __syncthreads();
    const double mp = s_mp, iSp = 1.0 / s_Sp, u = ures[b];
    auto wf = [&](int v) { return exp_nonpos(((double)tp[v] - mp) * iT) * iSp; };
    int tok = block_sample(wf, V, u);
    if (tid == 0) o[K] = tok;
  } else {
    r0 = __ffs(alive) - 1;
  }
  if (tid == 0) {
    for (int i = n_done + 1; i <= K; ++i) o[i] = -1;
    n_acc[b] = n_done;
    branch[b] = r0;
  }
}

// ------------------------------------------------------------------ stochastic, tree, many CTAs
// The same walk as k_verify_sample_decide, run by C CTAs per sequence
// (cooperative launch: every CTA resident).  Each CTA owns one vocabulary
// chunk of the sequence's residual buffers and computes every decision of
// the walk itself from the same inputs, so all of them take the same path;
// a full-vocabulary quantity (a residual's mass, the sampled distribution's
// chunk sums) is a per-chunk partial, summed by every CTA in chunk order
// after a barrier of the sequence's CTAs.  One barrier per pass, so a
// rejection costs two short passes over 1/C of the vocabulary instead of
// full-vocabulary passes on one SM.
constexpr int VT_THREADS = 256;
constexpr int VT_MAX_CHUNKS = 128;

// Barrier of the C CTAs of one sequence: the k-th call returns once all C
// have arrived for the k-th time (target C k on a counter zeroed before the
// launch), after at most TC_TIMEOUT_NS; false when it gave up or another
// CTA did (the abort word), with the error word set.
__device__ __forceinline__ bool vt_barrier(unsigned* bar, unsigned target, int* abort_g, int* err) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    red_add_release_gpu(bar, 1u);
    const unsigned long long t0 = gtimer();
    int ok = 1;
    for (unsigned n = 1;; ++n) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= target) break;
      if ((n & 31) == 0) {
        if (*(volatile int*)abort_g) { ok = 0; break; }
        if (gtimer() - t0 > TC_TIMEOUT_NS) {
          atomicExch(abort_g, 1);
          atomicExch(err, TC_ERR_TIMEOUT);
          ok = 0;
          break;
        }
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__global__ void __launch_bounds__(VT_THREADS)
k_vtree(const float* __restrict__ tgt, const float* __restrict__ dlog, const int* __restrict__ draft,
        int B, int N, int K, int V, float T, const double* __restrict__ ua,
        const double* __restrict__ ures, const float* __restrict__ pm, const double* __restrict__ ps,
        int chunks, double* __restrict__ resid, int C, double* __restrict__ vpart,
        unsigned* __restrict__ vbar, int* __restrict__ err, int* __restrict__ n_acc,
        int* __restrict__ branch, int* __restrict__ out, const int* __restrict__ rowmap) {
  __shared__ double shd[32];
  __shared__ int s_accept, s_own;
  __shared__ double s_mp, s_Sp, s_mq, s_Sq, s_Z, s_u;
  const int b = blockIdx.x / C, g = blockIdx.x - b * C, tid = threadIdx.x;
  int* abort_g = (int*)vbar;
  unsigned* bar = vbar + 1 + b;
  unsigned epoch = 0;
  const double dT = (double)T, iT = 1.0 / dT;
  const int n_tgt_rows = B * N * (K + 1);
  const int per = (V + C - 1) / C;
  const int v0 = min(V, g * per), v1 = min(V, v0 + per);
  double* part = vpart + (size_t)b * C;
  double* buf[2] = {resid + (size_t)b * 2 * V, resid + (size_t)b * 2 * V + V};
  int* o = out + (size_t)b * (K + 1);
  unsigned alive = (N >= 32) ? 0xffffffffu : ((1u << N) - 1u);
  int n_done = K, r0 = 0;
  bool ok = true;

  // draws a token from the current distribution p' (mode 0: the target row
  // given by (tp, mp, Sp); mode 1: buf[cur]) at u: chunk sums, a barrier,
  // then the chunk holding u * total (fixed chunk order) is searched by its
  // owner, which writes o[pos]
  auto sample = [&](const float* tp, int mode, int cur, double u, int pos) -> bool {
    const double mp = s_mp, iSp = 1.0 / s_Sp;
    double local = 0.0;
    for (int v = v0 + tid; v < v1; v += VT_THREADS)
      local += (mode == 0) ? exp_nonpos(((double)tp[v] - mp) * iT) * iSp : buf[cur][v];
    local = block_sum_d(local, shd);
    if (tid == 0) part[g] = local;
    if (!vt_barrier(bar, (unsigned)C * ++epoch, abort_g, err)) return false;
    if (tid == 0) {
      double tot = 0.0;
      for (int k = 0; k < C; ++k) tot += part[k];
      const double target = u * tot;
      double pre = 0.0;
      int own = -1, last_pos = 0;
      for (int k = 0; k < C; ++k) {
        const double sc = part[k];
        if (sc > 0.0) last_pos = k;
        if (own < 0 && pre + sc > target) own = k;
        else if (own < 0) pre += sc;
      }
      if (own < 0) {                       // rounding: the last chunk with mass
        own = last_pos;
        pre = 0.0;
        for (int k = 0; k < own; ++k) pre += part[k];
      }
      const double sc = part[own];
      s_own = own;
      s_u = sc > 0.0 ? fmin(fmax((target - pre) / sc, 0.0), 1.0) : 0.0;
    }
    __syncthreads();
    if (s_own == g) {
      int tok;
      if (mode == 0) {
        auto wf = [&](int v) { return exp_nonpos(((double)tp[v0 + v] - mp) * iT) * iSp; };
        tok = v0 + block_sample(wf, v1 - v0, s_u);
      } else {
        const double* pb = buf[cur] + v0;
        auto wf = [&](int v) { return pb[v]; };
        tok = v0 + block_sample(wf, v1 - v0, s_u);
      }
      if (tid == 0) o[pos] = tok;
    }
    return true;
  };

  for (int i = 0; i < K && ok; ++i) {
    r0 = __ffs(alive) - 1;
    const int trow = (b * N + r0) * (K + 1) + i;
    const float* tp = tgt + (size_t)(rowmap ? rowmap[trow] : trow) * V;
    if (tid < 32) {
      RowStat st = warp_combine_stats(pm, ps, trow, chunks, dT, tid);
      if (tid == 0) { s_mp = st.m; s_Sp = st.S; }
    }
    __syncthreads();
    int mode = 0, cur = 0, acc = -1;
    for (int j = 0; j < N; ++j) {
      if (!((alive >> j) & 1u)) continue;
      const int y = draft[((size_t)b * N + j) * K + i];
      const int drow = (b * N + j) * K + i;
      const float* qp = dlog ? dlog + (size_t)drow * V : nullptr;
      if (tid < 32) {
        RowStat sq{0.0, 1.0};
        if (qp) sq = warp_combine_stats(pm, ps, n_tgt_rows + drow, chunks, dT, tid);
        if (tid == 0) {
          double qy = 1.0;
          if (qp) {
            s_mq = sq.m; s_Sq = sq.S;
            qy = exp(((double)qp[y] - sq.m) / dT) / sq.S;
          }
          const double py = (mode == 0) ? exp(((double)tp[y] - s_mp) / dT) / s_Sp : buf[cur][y];
          s_accept = (ua[((size_t)b * N + j) * K + i] * qy < py) ? y : -1;
        }
      }
      __syncthreads();
      acc = s_accept;
      if (acc >= 0) break;
      // residual r = max(0, p' - q_j) on this CTA's chunk, its mass summed
      // over the chunks, then p' = r / mass
      const int dst = mode == 0 ? 0 : 1 - cur;
      const double mp = s_mp, mq = s_mq;
      const double iSp = 1.0 / s_Sp, iSq = qp ? 1.0 / s_Sq : 0.0;
      double local = 0.0;
      for (int v = v0 + tid; v < v1; v += VT_THREADS) {
        const double pv = (mode == 0) ? exp_nonpos(((double)tp[v] - mp) * iT) * iSp : buf[cur][v];
        const double qv = qp ? exp_nonpos(((double)qp[v] - mq) * iT) * iSq : (v == y ? 1.0 : 0.0);
        const double rv = fmax(pv - qv, 0.0);
        buf[dst][v] = rv;
        local += rv;
      }
      local = block_sum_d(local, shd);
      if (tid == 0) part[g] = local;
      if (!vt_barrier(bar, (unsigned)C * ++epoch, abort_g, err)) { ok = false; break; }
      if (tid == 0) {
        double Z = 0.0;
        for (int k = 0; k < C; ++k) Z += part[k];
        s_Z = Z;
      }
      __syncthreads();
      const double Z = s_Z;
      if (Z > 0.0) {
        const double iZ = 1.0 / Z;
        for (int v = v0 + tid; v < v1; v += VT_THREADS) buf[dst][v] *= iZ;
        mode = 1;
        cur = dst;
      } else if (mode == 0) {
        // p' stays the target row itself: materialise it for later steps
        for (int v = v0 + tid; v < v1; v += VT_THREADS)
          buf[dst][v] = exp_nonpos(((double)tp[v] - mp) * iT) * iSp;
        mode = 1;
        cur = dst;
      }
      // buf[cur] complete on every chunk before any CTA reads an entry of
      // another's (the next accept test), and the partials are free again
      if (!vt_barrier(bar, (unsigned)C * ++epoch, abort_g, err)) { ok = false; break; }
    }
    if (!ok) break;
    if (acc < 0) {
      if (!sample(tp, mode, cur, ures[b], i)) { ok = false; break; }
      n_done = i;
      break;
    }
    if (g == 0 && tid == 0) o[i] = acc;
    unsigned keep = 0u;
    for (int j = 0; j < N; ++j)
      if (((alive >> j) & 1u) && draft[((size_t)b * N + j) * K + i] == acc) keep |= 1u << j;
    alive = keep;
  }
  if (!ok) return;
  if (n_done == K) {
    r0 = __ffs(alive) - 1;
    const int trow = (b * N + r0) * (K + 1) + K;
    const float* tp = tgt + (size_t)(rowmap ? rowmap[trow] : trow) * V;
    if (tid < 32) {
      RowStat st = warp_combine_stats(pm, ps, trow, chunks, dT, tid);
      if (tid == 0) { s_mp = st.m; s_Sp = st.S; }
    }
    __syncthreads();
    if (!sample(tp, 0, 0, ures[b], K)) return;
  } else {
    r0 = __ffs(alive) - 1;
  }
  if (g == 0 && tid == 0) {
    for (int i = n_done + 1; i <= K; ++i) o[i] = -1;
    n_acc[b] = n_done;
    branch[b] = r0;
  }
}

// ------------------------------------------------------------------ stochastic, one draft
// With one draft per sequence the walk needs no materialised residual: the
// first rejected depth fixes what is sampled -- normalise(max(0, p - q)) at
// that depth, or p of row K when every depth is accepted -- so the walk is
// one warp per sequence, and the weights of that one draw are summed and
// searched by many CTAs per sequence (VS1_CHUNKS vocabulary chunks each)
// instead of one.
constexpr int VS1_CHUNKS = 16;

// Per sequence: 0 depth of the draw (n accepted), 1 rejected token (-1 when
// every depth accepted), 2 target row, 3 draft row (-1 without draft
// logits); and fp64 (m_p, S_p, m_q, S_q).
struct Vs1Plan {
  int n, y, trow, drow;
  double mp, Sp, mq, Sq;
};

// One warp per sequence: accept while u q(y) < p(y) (fp64), write the
// accepted tokens, the counts and the -1 padding, and the draw's plan.
__global__ void __launch_bounds__(128)
k_vs1_walk(const float* __restrict__ tgt, const float* __restrict__ dlog,
           const int* __restrict__ draft, int B, int K, int V, float T,
           const double* __restrict__ ua, const float* __restrict__ pm,
           const double* __restrict__ ps, int chunks, Vs1Plan* __restrict__ plan,
           int* __restrict__ n_acc, int* __restrict__ branch, int* __restrict__ out,
           const int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (b >= B) return;
  const double dT = (double)T;
  const int n_tgt_rows = B * (K + 1);
  int* o = out + (size_t)b * (K + 1);
  int i = 0;
  RowStat sp{0.0, 1.0}, sq{0.0, 1.0};
  int y = -1;
  for (; i < K; ++i) {
    const int trow = b * (K + 1) + i, drow = b * K + i;
    sp = warp_combine_stats(pm, ps, trow, chunks, dT, lane);
    if (dlog) sq = warp_combine_stats(pm, ps, n_tgt_rows + drow, chunks, dT, lane);
    y = draft[(size_t)b * K + i];
    int acc = 0;
    if (lane == 0) {
      const float* tp = tgt + (size_t)(rowmap ? rowmap[trow] : trow) * V;
      const double py = exp(((double)tp[y] - sp.m) / dT) / sp.S;
      const double qy = dlog ? exp(((double)dlog[(size_t)drow * V + y] - sq.m) / dT) / sq.S : 1.0;
      acc = (ua[(size_t)b * K + i] * qy < py) ? 1 : 0;
      if (acc) o[i] = y;
    }
    acc = __shfl_sync(0xffffffffu, acc, 0);
    if (!acc) break;
  }
  if (lane == 0) {
    Vs1Plan pl;
    pl.n = i;
    if (i < K) {
      pl.y = y;
      pl.trow = b * (K + 1) + i;
      pl.drow = dlog ? b * K + i : -1;
      pl.mp = sp.m; pl.Sp = sp.S; pl.mq = sq.m; pl.Sq = sq.S;
    } else {
      const int trow = b * (K + 1) + K;
      pl.y = -1;
      pl.trow = trow;
      pl.drow = -1;
      pl.mp = pl.Sp = pl.mq = pl.Sq = 0.0;
    }
    plan[b] = pl;
    for (int k = i + 1; k <= K; ++k) o[k] = -1;
    n_acc[b] = i;
    branch[b] = 0;
  }
  if (i == K) {
    // the bonus row's statistics
    RowStat st = warp_combine_stats(pm, ps, b * (K + 1) + K, chunks, dT, lane);
    if (lane == 0) { plan[b].mp = st.m; plan[b].Sp = st.S; }
  }
}

// Weight of token v in a draw: max(0, p - q) for a rejected depth (q the
// draft distribution, or the point mass on the rejected token), p itself
// for the bonus row; `use_p` forces p (a residual whose mass rounded to 0
// leaves p unchanged).
struct Vs1Weight {
  const float* tp;
  const float* qp;
  double mp, iSp, mq, iSq, iT;
  int y;
  bool resid;
  __device__ __forceinline__ double p(int v) const { return exp_nonpos(((double)tp[v] - mp) * iT) * iSp; }
  __device__ __forceinline__ double operator()(int v) const {
    const double pv = p(v);
    if (!resid) return pv;
    const double qv = qp ? exp_nonpos(((double)qp[v] - mq) * iT) * iSq : (v == y ? 1.0 : 0.0);
    return fmax(pv - qv, 0.0);
  }
};

__device__ __forceinline__ Vs1Weight vs1_weight(const Vs1Plan& pl, const float* tgt,
                                                const float* dlog, int V, float T,
                                                const int* rowmap) {
  Vs1Weight w;
  w.tp = tgt + (size_t)(rowmap ? rowmap[pl.trow] : pl.trow) * V;
  w.qp = pl.drow >= 0 ? dlog + (size_t)pl.drow * V : nullptr;
  w.mp = pl.mp;
  w.iSp = 1.0 / pl.Sp;
  w.mq = pl.mq;
  w.iSq = pl.drow >= 0 ? 1.0 / pl.Sq : 0.0;
  w.iT = 1.0 / (double)T;
  w.y = pl.y;
  w.resid = pl.y >= 0;
  return w;
}

// (sum of the draw's weights, sum of p) over chunk c of sequence b.
__global__ void __launch_bounds__(256)
k_vs1_sums(const float* __restrict__ tgt, const float* __restrict__ dlog, int V, float T,
           const Vs1Plan* __restrict__ plan, double* __restrict__ csum,
           const int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  __shared__ double shd[32];
  const int b = blockIdx.x / VS1_CHUNKS, c = blockIdx.x - b * VS1_CHUNKS;
  const Vs1Plan pl = plan[b];
  const Vs1Weight w = vs1_weight(pl, tgt, dlog, V, T, rowmap);
  const int per = (V + VS1_CHUNKS - 1) / VS1_CHUNKS;
  const int v0 = min(V, c * per), v1 = min(V, v0 + per);
  double sw = 0.0, sp = 0.0;
  for (int v = v0 + (int)threadIdx.x; v < v1; v += blockDim.x) {
    const double pv = w.p(v);
    sp += pv;
    if (w.resid) {
      const double qv = w.qp ? exp_nonpos(((double)w.qp[v] - w.mq) * w.iT) * w.iSq : (v == w.y ? 1.0 : 0.0);
      sw += fmax(pv - qv, 0.0);
    }
  }
  sw = block_sum_d(sw, shd);
  sp = block_sum_d(sp, shd);
  if (threadIdx.x == 0) {
    csum[((size_t)b * VS1_CHUNKS + c) * 2] = w.resid ? sw : sp;
    csum[((size_t)b * VS1_CHUNKS + c) * 2 + 1] = sp;
  }
}

// One CTA per sequence: the chunk holding u * total (chunk sums in fixed
// order), then the token inside it by inverse CDF; writes the drawn token.
__global__ void __launch_bounds__(512)
k_vs1_pick(const float* __restrict__ tgt, const float* __restrict__ dlog, int K, int V, float T,
           const double* __restrict__ ures, const Vs1Plan* __restrict__ plan,
           const double* __restrict__ csum, int* __restrict__ out,
           const int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_c;
  __shared__ double s_u;
  const int b = blockIdx.x;
  const Vs1Plan pl = plan[b];
  Vs1Weight w = vs1_weight(pl, tgt, dlog, V, T, rowmap);
  const double* cs = csum + (size_t)b * VS1_CHUNKS * 2;
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int c = 0; c < VS1_CHUNKS; ++c) tot += cs[c * 2];
    int col = 0;                           // the sums to use: the draw's weights, or p
    if (w.resid && !(tot > 0.0)) {
      col = 1;
      tot = 0.0;
      for (int c = 0; c < VS1_CHUNKS; ++c) tot += cs[c * 2 + 1];
    }
    const double target = ures[b] * tot;
    double pre = 0.0;
    int own = -1, last_pos = 0;
    for (int c = 0; c < VS1_CHUNKS; ++c) {
      const double sc = cs[c * 2 + col];
      if (sc > 0.0) last_pos = c;
      if (own < 0 && pre + sc > target) own = c;
      else if (own < 0) pre += sc;
    }
    if (own < 0) {                        // rounding: the last chunk with mass
      own = last_pos;
      pre = 0.0;
      for (int c = 0; c < own; ++c) pre += cs[c * 2 + col];
    }
    const double sc = cs[own * 2 + col];
    s_c = own | (col << 16);
    s_u = sc > 0.0 ? fmin(fmax((target - pre) / sc, 0.0), 1.0) : 0.0;
  }
  __syncthreads();
  const int own = s_c & 0xffff;
  if (s_c >> 16) w.resid = false;
  const int per = (V + VS1_CHUNKS - 1) / VS1_CHUNKS;
  const int v0 = min(V, own * per), v1 = min(V, v0 + per);
  auto wf = [&](int v) { return w(v0 + v); };
  const int tok = v0 + block_sample(wf, v1 - v0, s_u);
  if (threadIdx.x == 0) out[(size_t)b * (K + 1) + pl.n] = tok;
}

}  // namespace fm
