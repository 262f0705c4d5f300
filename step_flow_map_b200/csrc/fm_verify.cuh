// Prefix verify of drafted blocks against target logits.
//
// Greedy: keep the drafted tokens while they equal the target argmax, then
// emit the target argmax (page "FlashMap Drafts 16 Dependent Tokens at
// Once…", section "Why drafting still costs time").  Stochastic: accept with
// probability min(1, p/q) and resample the normalised residual on
// rejection, trying the drafts of a tree in index order.
#pragma once
#include "fm_misc.cuh"

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
                int* __restrict__ branch, int* __restrict__ out) {
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
  const float* r = tgt + (size_t)row * V;
  ArgMax a{-INFINITY, 0x7fffffff};
  // eight strided loads in flight per thread before they are compared (the
  // comparison is order-independent: ties go to the lowest index)
  for (int base = v0 + (int)threadIdx.x; base < v1; base += 8 * (int)blockDim.x) {
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = base + u * (int)blockDim.x;
      x[u] = v < v1 ? __ldcs(r + v) : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = base + u * (int)blockDim.x;
      if (v < v1 && am_better(x[u], v, a.v, a.i)) { a.v = x[u]; a.i = v; }
    }
  }
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
// in fp64, for every target row and, when present, every draft row.
constexpr int VS_THREADS = 256;

__global__ void __launch_bounds__(VS_THREADS)
k_row_stats(const float* __restrict__ tgt, const float* __restrict__ dlog, int n_tgt_rows,
            int n_rows, int V, int chunks, float T, float* __restrict__ pm,
            double* __restrict__ ps) {
  pdl_wait();
  pdl_trigger();
  __shared__ float shf[32];
  __shared__ double shd[32];
  const int row = blockIdx.x / chunks, c = blockIdx.x - row * chunks;
  const float* r = (row < n_tgt_rows) ? tgt + (size_t)row * V
                                      : dlog + (size_t)(row - n_tgt_rows) * V;
  const int per = (V + chunks - 1) / chunks;
  const int v0 = min(V, c * per), v1 = min(V, v0 + per);
  float mx = -INFINITY;
  for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) mx = fmaxf(mx, r[v]);
  mx = block_max(mx, shf);
  double s = 0.0;
  const double dm = (double)mx, iT = 1.0 / (double)T;
  for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) s += exp(((double)r[v] - dm) * iT);
  s = block_sum_d(s, shd);
  if (threadIdx.x == 0) {
    pm[(size_t)row * chunks + c] = mx;
    ps[(size_t)row * chunks + c] = s;
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
    if (mc > -INFINITY) S += ps[(size_t)row * chunks + c] * exp((mc - m) / T);
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
                       int* __restrict__ branch, int* __restrict__ out) {
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
    const float* tp = tgt + (size_t)trow * V;
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
        double p = (mode == 0) ? exp(((double)tp[v] - mp) * iT) * iSp : buf[src][v];
        double q = qp ? exp(((double)qp[v] - mq) * iT) * iSq : (v == y ? 1.0 : 0.0);
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
        for (int v = tid; v < V; v += blockDim.x) buf[dst][v] = exp(((double)tp[v] - mp) * iT) * iSp;
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
        auto wf = [&](int v) { return exp(((double)tp[v] - mp) * iT) * iSp; };
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
    const float* tp = tgt + (size_t)trow * V;
    if (tid < 32) {
      RowStat st = warp_combine_stats(pm, ps, trow, chunks, dT, tid);
      if (tid == 0) { s_mp = st.m; s_Sp = st.S; }
    }
    __syncthreads();
    const double mp = s_mp, iSp = 1.0 / s_Sp, u = ures[b];
    auto wf = [&](int v) { return exp(((double)tp[v] - mp) * iT) * iSp; };
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

}  // namespace fm
