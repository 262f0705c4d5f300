// Target-side tree scoring of a sequence's noise drafts: the prefix trie of
// the drafts, its ancestor masks, and the attention that scores every node
// in one pass.
//
// A tree of noise drafts adds speed (page "FlashMap并行草拟加速大模型解码",
// section "6.14 倍是最好成绩…": four noise drafts scored as a tree, +11 %
// mean speedup).  Drafts that share a prefix need the target's next-token
// distribution after that prefix once, so the target scores the unique
// prefixes -- the trie's nodes -- each attending to the context and to its
// own ancestors (the path of the draft that leads to it).
//
// Node order: breadth first (all nodes of depth i before depth i + 1), and
// within a depth in the order of the first draft that creates the node.
// Node n is a prefix of length depth(n) + 1 ending in token(n); parent(n) is
// that prefix without its last token (-1 at depth 0).  Target rows of a
// tree: row 0 is the root (the distribution of the first drafted position),
// row 1 + n is node n's.
#pragma once
#include "fm_common.cuh"

namespace fm {

constexpr int TREE_MAX_DRAFTS = 32;
constexpr int TREE_MAX_NODES = 1024;
constexpr int TREE_MAX_WORDS = TREE_MAX_NODES / 64;

// One warp per sequence; lane j is draft j.  Depth by depth, draft j's key
// is (its node at the previous depth, its token); it creates a node when no
// earlier draft has the same key, and new nodes are numbered in draft order
// after every node of the earlier depths.  Then the ancestor masks: bit m of
// node n's W words is set when m is n or one of its ancestors.  Entries past
// the sequence's node count are -1 (masks 0).
__global__ void __launch_bounds__(32)
k_build_tree(const int* __restrict__ draft, int N, int K, int NN, int W,
             int* __restrict__ node_token, int* __restrict__ node_parent,
             int* __restrict__ node_depth, int* __restrict__ n_nodes,
             int* __restrict__ draft_node, uint64_t* __restrict__ anc) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x, j = threadIdx.x;
  const bool live = j < N;
  int* tok_b = node_token + (size_t)b * NN;
  int* par_b = node_parent + (size_t)b * NN;
  int* dep_b = node_depth + (size_t)b * NN;
  int prev = -1, base = 0;
  for (int i = 0; i < K; ++i) {
    const int tok = live ? draft[((size_t)b * N + j) * K + i] : -1;
    // the earliest draft with the same key
    int first = j;
    for (int j2 = 0; j2 < N; ++j2) {
      const int p2 = __shfl_sync(0xffffffffu, prev, j2);
      const int t2 = __shfl_sync(0xffffffffu, tok, j2);
      if (j2 < first && p2 == prev && t2 == tok) first = j2;
    }
    const bool creator = live && first == j;
    const unsigned cm = __ballot_sync(0xffffffffu, creator);
    const int mine = base + __popc(cm & ((1u << j) - 1u));
    const int node = __shfl_sync(0xffffffffu, mine, first & 31);
    if (live) draft_node[((size_t)b * N + j) * K + i] = node;
    if (creator) {
      tok_b[node] = tok;
      par_b[node] = prev;
      dep_b[node] = i;
    }
    base += __popc(cm);
    prev = node;
  }
  __syncwarp();
  for (int n = base + j; n < NN; n += 32) {
    tok_b[n] = -1;
    par_b[n] = -1;
    dep_b[n] = -1;
  }
  if (j == 0) n_nodes[b] = base;
  __syncwarp();
  __threadfence_block();
  // ancestor masks: walk each node's parent chain (its parents were written
  // by this warp above)
  for (int n = j; n < NN; n += 32) {
    uint64_t w[TREE_MAX_WORDS];
#pragma unroll
    for (int k = 0; k < TREE_MAX_WORDS; ++k) w[k] = 0ull;
    if (n < base) {
      for (int u = n; u >= 0; u = par_b[u]) {
#pragma unroll
        for (int k = 0; k < TREE_MAX_WORDS; ++k)
          if (k == (u >> 6)) w[k] |= 1ull << (u & 63);
      }
    }
    uint64_t* dst = anc + ((size_t)b * NN + n) * W;
#pragma unroll
    for (int k = 0; k < TREE_MAX_WORDS; ++k)
      if (k < W) dst[k] = w[k];
  }
}

// Attention of every trie node over [context rows; its ancestors and
// itself], fp32, one warp per (sequence, node, head): the lanes hold the
// query's dh <= 128 values, every key is one warp dot product, with an online
// softmax.  Nodes past the sequence's count are skipped.
__global__ void __launch_bounds__(128)
k_tree_attention(const float* __restrict__ q, const float* __restrict__ k_ctx,
                 const float* __restrict__ v_ctx, const float* __restrict__ k_nodes,
                 const float* __restrict__ v_nodes, const uint64_t* __restrict__ anc,
                 const int* __restrict__ n_nodes, int B, int NN, int L, int H, int dh, int W,
                 float scale, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long gw = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= (long)B * NN * H) return;
  const int h = (int)(gw % H);
  const int n = (int)((gw / H) % NN);
  const int b = (int)(gw / ((long)H * NN));
  if (n >= n_nodes[b]) return;
  const int D = H * dh;
  float qv[4], acc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = lane + 32 * e;
    qv[e] = c < dh ? q[((size_t)b * NN + n) * D + h * dh + c] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto key = [&](const float* kr, const float* vr) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = lane + 32 * e;
      if (c < dh) s = fmaf(qv[e], kr[c], s);
    }
    s = warp_sum(s) * scale;
    const float mn = fmaxf(m, s);
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float p = expf(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = lane + 32 * e;
      acc[e] = acc[e] * corr + (c < dh ? p * vr[c] : 0.f);
    }
    m = mn;
  };
  for (int r = 0; r < L; ++r)
    key(k_ctx + ((size_t)b * L + r) * D + h * dh, v_ctx + ((size_t)b * L + r) * D + h * dh);
  const uint64_t* am = anc + ((size_t)b * NN + n) * W;
  for (int k = 0; k < W; ++k) {
    uint64_t bits = am[k];
    while (bits) {
      const int u = k * 64 + __ffsll((long long)bits) - 1;
      bits &= bits - 1;
      key(k_nodes + ((size_t)b * NN + u) * D + h * dh, v_nodes + ((size_t)b * NN + u) * D + h * dh);
    }
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = lane + 32 * e;
    if (c < dh) out[((size_t)b * NN + n) * D + h * dh + c] = acc[e] * inv;
  }
}

// Row map of a tree's target rows: draft j's position i of sequence b is
// scored by row b * R + (i == 0 ? 0 : 1 + draft_node[b][j][i - 1]).
__global__ void k_tree_rowmap(const int* __restrict__ draft_node, int B, int N, int K, int R,
                              int* __restrict__ rowmap) {
  pdl_wait();
  pdl_trigger();
  const long total = (long)B * N * (K + 1);
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < total;
       e += (long)gridDim.x * blockDim.x) {
    const int i = (int)(e % (K + 1));
    const long bj = e / (K + 1);
    const int b = (int)(bj / N);
    rowmap[e] = b * R + (i == 0 ? 0 : 1 + draft_node[bj * K + i - 1]);
  }
}

}  // namespace fm
