// Row kernels of the drafter: time conditioning, modulated LayerNorm,
// softmax, token selection, and a tiled transpose.
#pragma once
#include "fm_common.cuh"

namespace fm {

// ------------------------------------------------------------------ conditioning
// 256-wide time features of s and t: [cos(1000 tau f_j), sin(1000 tau f_j)],
// f_j = 10000^(-j/128), evaluated in fp64.
__global__ void k_time_features(double s, double t, float* __restrict__ phi) {
  pdl_wait();
  pdl_trigger();
  int e = threadIdx.x;  // 0..255
  int j = e & 127;
  double f = exp(-log(10000.0) * (double)j / 128.0);
  for (int w = 0; w < 2; ++w) {
    double a = 1000.0 * (w == 0 ? s : t) * f;
    phi[w * 256 + e] = (float)(e < 128 ? cos(a) : sin(a));
  }
}

// y[o] = act(sum_i W[o][i] * x[i]) (+ add[o]); one warp per output row.
// act: 0 = identity, 1 = SiLU.  x may be pre-activated by the caller.
template <typename T>
__global__ void k_gemv(const T* __restrict__ W, int n_out, int n_in, const float* __restrict__ x,
                       float* __restrict__ y, const float* __restrict__ add, int act) {
  pdl_wait();
  pdl_trigger();
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n_out) return;
  const T* row = W + (size_t)warp * n_in;
  float s = 0.f;
  for (int i = lane; i < n_in; i += 32) s = fmaf(to_f(row[i]), x[i], s);
  s = warp_sum(s);
  if (lane == 0) {
    if (act == 1) s = silu(s);
    if (add) s += add[warp];
    y[warp] = s;
  }
}

__global__ void k_silu_vec(const float* __restrict__ x, float* __restrict__ y, int n) {
  pdl_wait();
  pdl_trigger();
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = silu(x[i]);
}

// ------------------------------------------------------------------ LayerNorm
// out[m] = LN0(x[m]) * (1 + scale) + shift, LN0 without affine part, eps 1e-6,
// mean and variance in fp32 by two passes over the row held in registers.
// shift/scale may be null (plain LN0).  One CTA of 256 threads per row.
template <typename TI, typename TO>
__global__ void __launch_bounds__(256)
k_adaln(const TI* __restrict__ x, int d, const float* __restrict__ shift,
        const float* __restrict__ scale, TO* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sh[32];
  const int m = blockIdx.x;
  const TI* row = x + (size_t)m * d;
  const int T = blockDim.x;
  // rows up to 16 T wide stay in registers: one read, all loads in flight
  constexpr int CACHE = 16;
  float xv[CACHE], cv[CACHE], hv[CACHE];
  const bool cached = d <= CACHE * T;
  float s = 0.f;
  if (cached) {
    // the row, and the modulation of this thread's columns, in one round trip
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
      const int c = threadIdx.x + i * T;
      xv[i] = c < d ? to_f(row[c]) : 0.f;
      cv[i] = (scale && c < d) ? scale[c] : 0.f;
      hv[i] = (scale && c < d) ? shift[c] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < CACHE; ++i) s += xv[i];
  } else {
    for (int c = threadIdx.x; c < d; c += T) s += to_f(row[c]);
  }
  const float mean = block_sum(s, sh) / (float)d;
  float v = 0.f;
  if (cached) {
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
      if (threadIdx.x + i * T < d) {
        const float t = xv[i] - mean;
        v = fmaf(t, t, v);
      }
    }
  } else {
    for (int c = threadIdx.x; c < d; c += T) {
      float t = to_f(row[c]) - mean;
      v = fmaf(t, t, v);
    }
  }
  const float var = block_sum(v, sh) / (float)d;
  const float rstd = rsqrtf(var + 1e-6f);
  if (cached) {
#pragma unroll
    for (int i = 0; i < CACHE; ++i) {
      const int c = threadIdx.x + i * T;
      if (c < d) {
        float y = (xv[i] - mean) * rstd;
        if (scale) y = y * (1.f + cv[i]) + hv[i];
        out[(size_t)m * d + c] = from_f<TO>(y);
      }
    }
  } else {
    for (int c = threadIdx.x; c < d; c += T) {
      float y = (to_f(row[c]) - mean) * rstd;
      if (scale) y = y * (1.f + scale[c]) + shift[c];
      out[(size_t)m * d + c] = from_f<TO>(y);
    }
  }
}

// Calls f(v, x) for every v in [v0, v1) of `row`, the bulk through 16-byte
// loads with four in flight per thread (elements before the first 16-byte
// boundary and after the last one one by one).  Visiting order differs from
// index order; callers combine order-independently or break ties by index.
template <class F>
__device__ __forceinline__ void for_row_range(const float* __restrict__ row, int v0, int v1, F f) {
  int a = v0;
  while (a < v1 && ((reinterpret_cast<uintptr_t>(row + a) & 15) != 0)) {
    if (a - v0 == (int)threadIdx.x) f(a, row[a]);
    ++a;
  }
  const int nv = (v1 - a) >> 2;                     // whole float4 groups
  const float4* r4 = reinterpret_cast<const float4*>(row + a);
  const int T = blockDim.x;
  int i = threadIdx.x;
  for (; i + 3 * T < nv; i += 4 * T) {
    float4 x[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) x[k] = __ldcs(r4 + i + k * T);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int v = a + 4 * (i + k * T);
      f(v, x[k].x); f(v + 1, x[k].y); f(v + 2, x[k].z); f(v + 3, x[k].w);
    }
  }
  for (; i < nv; i += T) {
    const float4 x = __ldcs(r4 + i);
    const int v = a + 4 * i;
    f(v, x.x); f(v + 1, x.y); f(v + 2, x.z); f(v + 3, x.w);
  }
  for (int v = a + 4 * nv + (int)threadIdx.x; v < v1; v += T) f(v, row[v]);
}

// ------------------------------------------------------------------ softmax rows
// D[m] = softmax(logits[m]) at temperature 1, stored as dtype (the flow-map
// denoiser output used by the next step's embedding).  Launched in clusters
// of C CTAs per row (C = 1 without a cluster; grid = rows x C): CTA z of a
// row takes the vocabulary slice [z V / C, (z + 1) V / C).  One pass keeps a
// running (max, sum of exp(x - max)) per thread; the CTA combines its
// threads' pairs, the cluster its CTAs' pairs through distributed shared
// memory, and a second pass writes exp(x - max) / sum.
template <typename TO>
__global__ void __launch_bounds__(1024)
k_softmax_rows(const float* __restrict__ logits, int V, int rows, TO* __restrict__ D) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sh[32];
  __shared__ float s_ms[2];               // this CTA's (max, sum), read by the cluster
  const uint32_t C = cluster_size(), z = cluster_rank();
  const int r = blockIdx.x / (int)C;
  if (r >= rows) return;                  // every CTA of the cluster: the same row
  const int v0 = (int)((long)z * V / C), v1 = (int)((long)(z + 1) * V / C);
  const float* row = logits + (size_t)r * V;
  float m = -INFINITY, s = 0.f;
  for_row_range(row, v0, v1, [&](int, float x) {
    if (x > m) {
      s = s * __expf(m - x) + 1.f;
      m = x;
    } else if (x != -INFINITY) {
      s += __expf(x - m);
    }
  });
  const float mb = block_max(m, sh);
  float sb = block_sum(m == -INFINITY ? 0.f : s * __expf(m - mb), sh);
  if (threadIdx.x == 0) {
    s_ms[0] = mb;
    s_ms[1] = sb;
  }
  cluster_sync_all();                     // every CTA's pair is written
  float mx = -INFINITY;
  for (uint32_t p = 0; p < C; ++p) mx = fmaxf(mx, dsmem_ld(dsmem_addr((uint32_t)__cvta_generic_to_shared(&s_ms[0]), p)));
  float tot = 0.f;
  for (uint32_t p = 0; p < C; ++p) {
    const float mp = dsmem_ld(dsmem_addr((uint32_t)__cvta_generic_to_shared(&s_ms[0]), p));
    const float sp = dsmem_ld(dsmem_addr((uint32_t)__cvta_generic_to_shared(&s_ms[1]), p));
    if (mp != -INFINITY) tot += sp * __expf(mp - mx);
  }
  cluster_sync_all();                     // no CTA leaves while another reads its pair
  const float inv = 1.f / tot;
  TO* out = D + (size_t)r * V;
  for_row_range(row, v0, v1, [&](int v, float x) { out[v] = from_f<TO>(__expf(x - mx) * inv); });
}

// ------------------------------------------------------------------ inverse CDF
// One pass over the row: the smallest v whose running sum of w(v), in
// vocabulary order, exceeds u * total, where total is the sum of all w(v);
// if rounding leaves none, the last v with w(v) > 0.  Warp i sums segment i
// of the row (its lanes strided, so loads are coalesced) while the total
// forms; only the segment holding u * total is read again, by its warp with
// each lane on a contiguous sub-chunk, and then the owning sub-chunk by its
// lane.  blockDim.x is a multiple of 32, at most 1024.  All threads return
// the answer.
template <class WF>
__device__ int block_sample(const WF& w, int V, double u) {
  __shared__ double seg_sum[32];
  __shared__ double s_base, s_target;
  __shared__ int s_last, s_owner, s_pick;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  const int seg = ((V + nw - 1) / nw + 31) / 32 * 32;   // a multiple of 32
  const int s0 = min(V, wid * seg), s1 = min(V, s0 + seg);
  if (tid == 0) {
    s_last = -1;
    s_pick = -1;
  }
  __syncthreads();
  double acc = 0.0;
  int last = -1;
  for (int v = s0 + lane; v < s1; v += 32) {
    const double x = w(v);
    acc += x;
    if (x > 0.0) last = v;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    acc += __shfl_xor_sync(0xffffffffu, acc, o);
    last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
  }
  if (lane == 0) {
    seg_sum[wid] = acc;
    if (last >= 0) atomicMax(&s_last, last);
  }
  __syncthreads();
  if (tid == 0) {
    double tot = 0.0;
    for (int i = 0; i < nw; ++i) tot += seg_sum[i];
    const double target = u * tot;
    double pre = 0.0;
    int own = -1;
    for (int i = 0; i < nw; ++i) {
      if (pre + seg_sum[i] > target) {
        own = i;
        break;
      }
      pre += seg_sum[i];
    }
    s_owner = own;
    s_base = pre;
    s_target = target;
  }
  __syncthreads();
  const int own = s_owner;
  if (own >= 0 && wid == own) {
    const int L = seg / 32;
    const int c0 = min(s1, s0 + lane * L), c1 = min(s1, c0 + L);
    double sub = 0.0;
    int lp = -1;
    for (int v = c0; v < c1; ++v) {
      const double x = w(v);
      sub += x;
      if (x > 0.0) lp = v;
    }
    double incl = sub;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const double base = s_base, target = s_target;
    const unsigned hit = __ballot_sync(0xffffffffu, base + incl > target);
    int seg_last = lp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) seg_last = max(seg_last, __shfl_xor_sync(0xffffffffu, seg_last, o));
    if (hit) {
      if (lane == __ffs(hit) - 1) {
        double r = base + incl - sub;   // mass before this sub-chunk
        int pick = -1, lq = -1;
        for (int v = c0; v < c1; ++v) {
          const double x = w(v);
          r += x;
          if (x > 0.0) lq = v;
          if (r > target) {
            pick = v;
            break;
          }
        }
        s_pick = pick >= 0 ? pick : (lq >= 0 ? lq : c0);   // rounding at the sub-chunk end
      }
    } else if (lane == 0) {
      s_pick = seg_last;   // rounding: the segment's strided sum said it holds the target
    }
  }
  __syncthreads();
  int ans = s_pick;
  if (ans < 0) ans = s_last >= 0 ? s_last : 0;
  __syncthreads();
  return ans;
}

// ------------------------------------------------------------------ token choice
struct TempArgs {
  int n_noise, K;
  float temp[256];  // per call-sequence; 0 = greedy
};

// One CTA per row.  Greedy rows: argmax of the fp32 logits (ties lowest) or,
// when `part_v` is given, of the per-tile partial maxima the LM-head
// epilogue left.  Sampled rows: inverse CDF of softmax(logits / T) at u.
__global__ void __launch_bounds__(1024)
k_select_tokens(const float* __restrict__ logits, int V, const float* __restrict__ part_v,
                const int* __restrict__ part_i, int n_part, const double* __restrict__ u,
                TempArgs ta, int* __restrict__ tokens, int skip_sampled) {
  pdl_wait();
  pdl_trigger();
  __shared__ float shv[32];
  __shared__ int shi[32];
  const int m = blockIdx.x;
  const int q = m / (ta.n_noise * ta.K);
  const float T = ta.temp[q];
  if (T > 0.f && skip_sampled) return;   // drawn by the chunked sampler below
  if (T == 0.f) {
    ArgMax a{-INFINITY, 0x7fffffff};
    if (part_v) {
      for (int p = threadIdx.x; p < n_part; p += blockDim.x) {
        float v = part_v[(size_t)m * n_part + p];
        int i = part_i[(size_t)m * n_part + p];
        if (am_better(v, i, a.v, a.i)) { a.v = v; a.i = i; }
      }
    } else {
      const float* row = logits + (size_t)m * V;
      for_row_range(row, 0, V, [&](int v, float x) {
        if (am_better(x, v, a.v, a.i)) { a.v = x; a.i = v; }
      });
    }
    a = block_argmax(a, shv, shi);
    if (threadIdx.x == 0) tokens[m] = (a.i == 0x7fffffff) ? 0 : a.i;
    return;
  }
  // weights exp((l - max)/T) in fp32, accumulated in fp64
  const float* row = logits + (size_t)m * V;
  float mx = -INFINITY;
  for (int v = threadIdx.x; v < V; v += blockDim.x) mx = fmaxf(mx, row[v]);
  mx = block_max(mx, shv);
  const float iT = 1.f / T;
  auto wf = [&](int v) { return (double)expf((row[v] - mx) * iT); };
  int tok = block_sample(wf, V, u[m]);
  if (threadIdx.x == 0) tokens[m] = tok;
}

// ------------------------------------------------------------------ chunked sampling
// Sampled rows (T > 0) of a batch, spread over SAMPLE_CHUNKS vocabulary
// chunks per row: the chunk maxima, then per chunk the sum of the row's fp32
// weights exp((l - max) / T) in fp64, then one CTA per row finds the chunk
// holding u * total (chunk sums in fixed order) and draws inside it by the
// inverse CDF -- the same weights and rule as one CTA per row, with every
// pass over the logits spread over the whole GPU.  Greedy rows return at
// once.
constexpr int SAMPLE_CHUNKS = 16;

__global__ void __launch_bounds__(256)
k_sample_chunk_max(const float* __restrict__ logits, int V, TempArgs ta, float* __restrict__ cmax) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sh[32];
  const int m = blockIdx.x / SAMPLE_CHUNKS, c = blockIdx.x - m * SAMPLE_CHUNKS;
  if (ta.temp[m / (ta.n_noise * ta.K)] == 0.f) return;
  const int per = (V + SAMPLE_CHUNKS - 1) / SAMPLE_CHUNKS;
  const int v0 = min(V, c * per), v1 = min(V, v0 + per);
  const float* row = logits + (size_t)m * V;
  float mx = -INFINITY;
  for_row_range(row, v0, v1, [&](int, float x) { mx = fmaxf(mx, x); });
  mx = block_max(mx, sh);
  if (threadIdx.x == 0) cmax[(size_t)m * SAMPLE_CHUNKS + c] = mx;
}

__global__ void __launch_bounds__(256)
k_sample_chunk_sum(const float* __restrict__ logits, int V, TempArgs ta,
                   const float* __restrict__ cmax, double* __restrict__ csum) {
  pdl_wait();
  pdl_trigger();
  __shared__ double sh[32];
  const int m = blockIdx.x / SAMPLE_CHUNKS, c = blockIdx.x - m * SAMPLE_CHUNKS;
  const float T = ta.temp[m / (ta.n_noise * ta.K)];
  if (T == 0.f) return;
  float mx = -INFINITY;
  for (int k = 0; k < SAMPLE_CHUNKS; ++k) mx = fmaxf(mx, cmax[(size_t)m * SAMPLE_CHUNKS + k]);
  const int per = (V + SAMPLE_CHUNKS - 1) / SAMPLE_CHUNKS;
  const int v0 = min(V, c * per), v1 = min(V, v0 + per);
  const float* row = logits + (size_t)m * V;
  const float iT = 1.f / T;
  double s = 0.0;
  for_row_range(row, v0, v1, [&](int, float x) { s += (double)expf((x - mx) * iT); });
  s = block_sum_d(s, sh);
  if (threadIdx.x == 0) csum[(size_t)m * SAMPLE_CHUNKS + c] = s;
}

__global__ void __launch_bounds__(512)
k_sample_pick(const float* __restrict__ logits, int V, const double* __restrict__ u, TempArgs ta,
              const float* __restrict__ cmax, const double* __restrict__ csum,
              int* __restrict__ tokens) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_c;
  __shared__ double s_u;
  const int m = blockIdx.x;
  const float T = ta.temp[m / (ta.n_noise * ta.K)];
  if (T == 0.f) return;
  const double* cs = csum + (size_t)m * SAMPLE_CHUNKS;
  float mx = -INFINITY;
  for (int k = 0; k < SAMPLE_CHUNKS; ++k) mx = fmaxf(mx, cmax[(size_t)m * SAMPLE_CHUNKS + k]);
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int k = 0; k < SAMPLE_CHUNKS; ++k) tot += cs[k];
    const double target = u[m] * tot;
    double pre = 0.0;
    int own = -1, last_pos = 0;
    for (int k = 0; k < SAMPLE_CHUNKS; ++k) {
      if (cs[k] > 0.0) last_pos = k;
      if (own < 0 && pre + cs[k] > target) own = k;
      else if (own < 0) pre += cs[k];
    }
    if (own < 0) {                        // rounding: the last chunk with mass
      own = last_pos;
      pre = 0.0;
      for (int k = 0; k < own; ++k) pre += cs[k];
    }
    s_c = own;
    s_u = cs[own] > 0.0 ? fmin(fmax((target - pre) / cs[own], 0.0), 1.0) : 0.0;
  }
  __syncthreads();
  const int per = (V + SAMPLE_CHUNKS - 1) / SAMPLE_CHUNKS;
  const int v0 = min(V, s_c * per), v1 = min(V, v0 + per);
  const float* row = logits + (size_t)m * V;
  const float iT = 1.f / T;
  auto wf = [&](int v) { return (double)expf((row[v0 + v] - mx) * iT); };
  const int tok = v0 + block_sample(wf, v1 - v0, s_u);
  if (threadIdx.x == 0) tokens[m] = tok;
}

// ------------------------------------------------------------------ factorised drafting
// u_full[b][j][i] = u[b][i]: every draft j of sequence b samples position i
// with that position's uniform.
__global__ void k_repeat_u(const double* __restrict__ u, double* __restrict__ u_full, int n_seqs,
                           int K) {
  pdl_wait();
  pdl_trigger();
  const size_t n = (size_t)n_seqs * K * K;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t b = e / ((size_t)K * K);
    const int i = (int)(e % K);
    u_full[e] = u[b * K + i];
  }
}

// tokens[b][i] = all_tok[b][i][i] and, when both are given, logits[b][i][:]
// = all_logits[b][i][i][:]: position i of the factorised block comes from
// the draft of noise block i.  One CTA per (b, i).
__global__ void k_take_diagonal(const int* __restrict__ all_tok, const float* __restrict__ all_logits,
                                int n_seqs, int K, int V, int* __restrict__ tokens,
                                float* __restrict__ logits) {
  pdl_wait();
  pdl_trigger();
  const int bi = blockIdx.x, b = bi / K, i = bi - b * K;
  const size_t src = ((size_t)b * K + i) * K + i;
  if (threadIdx.x == 0) tokens[bi] = all_tok[src];
  if (all_logits && logits) {
    const float* r = all_logits + src * V;
    float* o = logits + (size_t)bi * V;
    for (int v = threadIdx.x; v < V; v += blockDim.x) o[v] = r[v];
  }
}

// ------------------------------------------------------------------ transpose
// out[c][r] = in[r][c] for in [R][C]; 32 x 32 tiles.
template <typename T>
__global__ void k_transpose(const T* __restrict__ in, T* __restrict__ out, int R, int C) {
  pdl_wait();
  pdl_trigger();
  __shared__ T tile[32][33];
  int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    int r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C) tile[i][threadIdx.x] = in[(size_t)r * C + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    int c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C) out[(size_t)c * R + r] = tile[threadIdx.x][i];
  }
}

}  // namespace fm
