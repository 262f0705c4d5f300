// SIMT kernels: the fp32 path of the drafter (and a plain-CUDA-core form of
// each contraction, used for small shapes).  Epilogue functors are shared
// with the tensor-core GEMM.
#pragma once
#include <type_traits>
#include "fm_common.cuh"

namespace fm {

// ------------------------------------------------------------------ epilogues
// Every GEMM here computes Y[m][n] = sum_k A[m][k] W(n, k) in fp32 and hands
// each finished element to an epilogue functor exactly once.

template <typename TO>
struct EpiStore {  // Y -> out (dtype)
  TO* out;
  int ld;
  __device__ __forceinline__ void operator()(int m, int n, float v) const {
    out[(size_t)m * ld + n] = from_f<TO>(v);
  }
};

struct EpiStoreF32 {  // Y -> fp32 buffer
  float* out;
  int ld;
  __device__ __forceinline__ void operator()(int m, int n, float v) const {
    out[(size_t)m * ld + n] = v;
  }
};

// Input embedding of the vocabulary-space state.  First step: z = x0 E.
// Later steps: z <- (1 - alpha) z + alpha (D E), the flow-map update
// x_t = x_s + alpha (D - x_s) pushed through the linear map E.  Either way
// the residual stream starts as x = z + P[slot].
struct EpiEmbed {
  float* x;
  float* z;        // may be null on a one-step draft
  const float* P;  // [K][d]
  int d, K;
  float alpha;     // < 0: first step
  __device__ __forceinline__ void operator()(int m, int n, float v) const {
    size_t o = (size_t)m * d + n;
    float zz = v;
    if (alpha >= 0.f) zz = (1.f - alpha) * z[o] + alpha * v;
    if (z) z[o] = zz;
    x[o] = zz + P[(m % K) * d + n];
  }
};

// Gated residual: x += gate * Y (adaLN-Zero style gate of a DiT block).
struct EpiResidual {
  float* x;
  const float* gate;
  int d;
  __device__ __forceinline__ void operator()(int m, int n, float v) const {
    x[(size_t)m * d + n] += gate[n] * v;
  }
  // Rows m0 .. m0 + count - 1 (count <= 16) of feature n: every load is
  // issued before the first store, so the read-modify-writes do not
  // serialise on memory latency.
  __device__ __forceinline__ void chunk16(int m0, int n, const float* v, int count) const {
    const float g = gate[n];
    float xo[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) xo[j] = j < count ? __ldcg(x + (size_t)(m0 + j) * d + n) : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < count) x[(size_t)(m0 + j) * d + n] = xo[j] + g * v[j];
  }
};

// Epilogues with a whole-chunk form (chunk16) take it in the GEMM kernels.
template <class E>
struct has_chunk16 : std::false_type {};
template <>
struct has_chunk16<EpiResidual> : std::true_type {};

template <typename TO>
struct EpiGelu {
  TO* out;
  int ld;
  __device__ __forceinline__ void operator()(int m, int n, float v) const {
    out[(size_t)m * ld + n] = from_f<TO>(gelu_tanh(v));
  }
};

// Context keys/values: row r of the projected batch is row k = r % n_new of
// call-sequence q = r / n_new; it lands in cache slot slot[q] at position
// pos0[q] + k.  Columns [0, d) are keys, [d, 2d) values.
struct RowMap {
  int n_seqs, n_new;
  int slot[256];
  int pos0[256];
};
template <typename TO>
struct EpiCtxKV {
  TO* Kc;  // [max_seqs][max_ctx][d] of this block
  TO* Vc;
  int d, max_ctx;
  RowMap map;
  __device__ __forceinline__ void operator()(int r, int n, float v) const {
    int q = r / map.n_new, k = r - q * map.n_new;
    size_t row = (size_t)map.slot[q] * max_ctx + map.pos0[q] + k;
    if (n < d) Kc[row * d + n] = from_f<TO>(v);
    else Vc[row * d + (n - d)] = from_f<TO>(v);
  }
};

// Keys and values of every block in one GEMM over the blocks' stacked key
// and value weights (column n: block n / (2d), then keys [0, d), values
// [d, 2d) of that block); rows map to cache positions as in EpiCtxKV.
template <typename TO>
struct EpiCtxKVAll {
  TO* Kc[8];  // [max_seqs][max_ctx][d] of each block
  TO* Vc[8];
  int d, max_ctx;
  RowMap map;
  __device__ __forceinline__ void operator()(int r, int n, float v) const {
    const int l = n / (2 * d), nn = n - l * 2 * d;
    int q = r / map.n_new, k = r - q * map.n_new;
    size_t row = (size_t)map.slot[q] * max_ctx + map.pos0[q] + k;
    if (nn < d) Kc[l][row * d + nn] = from_f<TO>(v);
    else Vc[l][row * d + (nn - d)] = from_f<TO>(v);
  }
  // rows r0 .. r0 + count - 1 (count <= 16) of column n: the block, the
  // key/value half and the first row's sequence are found once, the later
  // rows step through the sequences' row ranges
  __device__ __forceinline__ void chunk16(int r0, int n, const float* v, int count) const {
    const int l = n / (2 * d), nn = n - l * 2 * d;
    TO* col = nn < d ? Kc[l] + nn : Vc[l] + (nn - d);
    int q = r0 / map.n_new, k = r0 - q * map.n_new;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < count) {
        col[((size_t)map.slot[q] * max_ctx + map.pos0[q] + k) * d] = from_f<TO>(v[j]);
        if (++k == map.n_new) {
          k = 0;
          ++q;
        }
      }
    }
  }
};

template <typename TO>
struct has_chunk16<EpiCtxKVAll<TO>> : std::true_type {};

// QKV of the block rows plus, in the same GEMM, the keys and values of
// context rows appended after them (rows >= M_draft; their query columns
// are not needed and are dropped).
template <typename TO>
struct EpiQkvCtx {
  TO* qkv;
  int ld, M_draft, d;
  EpiCtxKV<TO> kv;
  __device__ __forceinline__ void operator()(int m, int n, float v) const {
    if (m < M_draft) qkv[(size_t)m * ld + n] = from_f<TO>(v);
    else if (n >= d) kv(m - M_draft, n - d, v);
  }
};

// ------------------------------------------------------------------ SIMT GEMM
// Y[m][n] = sum_k A[m][k] * W(n,k), W(n,k) = W[n*ldw+k] (WK) or W[k*ldw+n].
// Tile 32 x 64 x 16, 256 threads, 2 x 4 outputs per thread.  With
// gridDim.z > 1 each z-slice covers k_split columns of the reduction and
// writes fp32 partials [z][M][N]; k_splitk_apply finishes them.
constexpr int SG_BM = 32, SG_BN = 64, SG_BK = 16;

template <typename TA, typename TW, bool WK, class Epi>
__global__ void __launch_bounds__(256)
k_gemm_simt(const TA* __restrict__ A, int lda, const TW* __restrict__ W, int ldw,
            int M, int N, int Kd, int k_split, float* __restrict__ partial, Epi epi) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[SG_BK][SG_BM];
  __shared__ float Ws[SG_BK][SG_BN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * SG_BM, n0 = blockIdx.x * SG_BN;
  const int kb = blockIdx.z * k_split, ke = min(Kd, kb + k_split);
  float acc[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = kb; k0 < ke; k0 += SG_BK) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {  // A tile: 32 x 16
      int e = tid + r * 256, mm = e / SG_BK, kk = e % SG_BK;
      int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < ke) ? to_f(A[(size_t)gm * lda + gk]) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {  // W tile: 64 x 16
      int e = tid + r * 256;
      int nn, kk;
      if (WK) { nn = e / SG_BK; kk = e % SG_BK; } else { kk = e / SG_BN; nn = e % SG_BN; }
      int gn = n0 + nn, gk = k0 + kk;
      float v = 0.f;
      if (gn < N && gk < ke) v = to_f(WK ? W[(size_t)gn * ldw + gk] : W[(size_t)gk * ldw + gn]);
      Ws[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a0 = As[kk][ty], a1 = As[kk][ty + 16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float w = Ws[kk][tx + 16 * j];
        acc[0][j] = fmaf(a0, w, acc[0][j]);
        acc[1][j] = fmaf(a1, w, acc[1][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    int m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      if (gridDim.z > 1) partial[((size_t)blockIdx.z * M + m) * N + n] = acc[i][j];
      else epi(m, n, acc[i][j]);
    }
  }
}

template <class Epi>
__global__ void k_splitk_apply(const float* __restrict__ partial, int splits, int M, int N, Epi epi) {
  pdl_wait();
  pdl_trigger();
  size_t total = (size_t)M * N;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < splits; ++z) s += partial[(size_t)z * total + e];
    epi((int)(e / N), (int)(e % N), s);
  }
}

// ------------------------------------------------------------------ SIMT attention
// One CTA per (sequence, head, noise draft): the K block queries attend,
// without a mask, over [context rows 0..L-1 of the sequence's slot; the
// draft's own K block rows], online softmax over key chunks of 16.
struct AttnArgs {
  int n_seqs, n_noise, K, d, n_heads, max_ctx;
  float scale;  // 1/sqrt(dh)
  int slot[256];
  int len[256];
};

constexpr int SA_KEYS = 16;
constexpr int SA_MAXQ = 16;
constexpr int SA_MAXDH = 128;

template <typename T>
__global__ void __launch_bounds__(128)
k_attn_simt(const T* __restrict__ qkv, const T* __restrict__ Kc, const T* __restrict__ Vc,
            T* __restrict__ out, AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x, h = blockIdx.y, j = blockIdx.z;
  const int dh = a.d / a.n_heads, K = a.K, d3 = 3 * a.d;
  const int L = a.len[b];
  const size_t ctx_base = (size_t)a.slot[b] * a.max_ctx * a.d;
  const int m0 = (b * a.n_noise + j) * K;
  __shared__ float Qs[SA_MAXQ][SA_MAXDH];
  __shared__ float Ks[SA_KEYS][SA_MAXDH + 1];
  __shared__ float Vs[SA_KEYS][SA_MAXDH];
  __shared__ float S[SA_MAXQ][SA_KEYS];
  __shared__ float Os[SA_MAXQ][SA_MAXDH];
  __shared__ float mrun[SA_MAXQ], lrun[SA_MAXQ], corr[SA_MAXQ];
  const int tid = threadIdx.x;
  for (int e = tid; e < K * dh; e += blockDim.x) {
    int q = e / dh, c = e % dh;
    Qs[q][c] = to_f(qkv[(size_t)(m0 + q) * d3 + h * dh + c]) * a.scale;
    Os[q][c] = 0.f;
  }
  if (tid < K) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; }
  __syncthreads();
  const int total = L + K;
  for (int k0 = 0; k0 < total; k0 += SA_KEYS) {
    const int nk = min(SA_KEYS, total - k0);
    for (int e = tid; e < nk * dh; e += blockDim.x) {
      int r = e / dh, c = e % dh, key = k0 + r;
      float kv, vv;
      if (key < L) {
        size_t o = ctx_base + (size_t)key * a.d + h * dh + c;
        kv = to_f(Kc[o]);
        vv = to_f(Vc[o]);
      } else {
        size_t o = (size_t)(m0 + key - L) * d3 + h * dh + c;
        kv = to_f(qkv[o + a.d]);
        vv = to_f(qkv[o + 2 * a.d]);
      }
      Ks[r][c] = kv;
      Vs[r][c] = vv;
    }
    __syncthreads();
    for (int e = tid; e < K * SA_KEYS; e += blockDim.x) {
      int q = e / SA_KEYS, r = e % SA_KEYS;
      float s = -INFINITY;
      if (r < nk) {
        s = 0.f;
        for (int c = 0; c < dh; ++c) s = fmaf(Qs[q][c], Ks[r][c], s);
      }
      S[q][r] = s;
    }
    __syncthreads();
    if (tid < K) {
      float mx = mrun[tid];
      for (int r = 0; r < nk; ++r) mx = fmaxf(mx, S[tid][r]);
      float cr = expf(mrun[tid] - mx), sum = 0.f;
      for (int r = 0; r < SA_KEYS; ++r) {
        float p = (r < nk) ? expf(S[tid][r] - mx) : 0.f;
        S[tid][r] = p;
        sum += p;
      }
      lrun[tid] = lrun[tid] * cr + sum;
      mrun[tid] = mx;
      corr[tid] = cr;
    }
    __syncthreads();
    for (int e = tid; e < K * dh; e += blockDim.x) {
      int q = e / dh, c = e % dh;
      float acc = Os[q][c] * corr[q];
      for (int r = 0; r < nk; ++r) acc = fmaf(S[q][r], Vs[r][c], acc);
      Os[q][c] = acc;
    }
    __syncthreads();
  }
  for (int e = tid; e < K * dh; e += blockDim.x) {
    int q = e / dh, c = e % dh;
    out[(size_t)(m0 + q) * a.d + h * dh + c] = from_f<T>(Os[q][c] / lrun[q]);
  }
}

}  // namespace fm
