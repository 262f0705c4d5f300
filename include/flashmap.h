/*
 * flashmap.h -- C ABI of the B200 flow-map block drafter and prefix verifier.
 *
 * The library implements the hot path of FlashMap speculative decoding:
 * a flow-map drafter that maps one Gaussian noise block over the
 * vocabulary to a whole K-token block in one DiT pass, and the verifier
 * that keeps the longest valid prefix of that block against target logits.
 *
 * Sources, cited below by tag, title and section:
 *   P1  "FlashMap并行草拟加速大模型解码" (zh)
 *   P2  "Polymathic AI и исследователи из Princeton выпустили FlashMap —
 *        модель-черновик Flow Map для декодирования LLM в 6,14 раза быстрее" (ru)
 *   P5  "FlashMap Drafts 16 Dependent Tokens at Once, Hitting 6.1x Faster
 *        Decoding" (en)
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device memory of the current device (the
 *     device that was current at fm_load_weights).  Host pointers are
 *     ordinary host memory, read before the call returns.
 *   - Matrices are row-major.  Linear weights are [out, in] (y = x W^T).
 *   - "dtype" storage is fp32 (FM_F32) or bf16 bit patterns (FM_BF16),
 *     fixed per context by fm_config.dtype.  Logits are always fp32,
 *     uniforms fp64, tokens and counts int32.
 *   - The caller owns every buffer it passes.  Weights are borrowed and
 *     must outlive the context, except E, which the library copies once
 *     into its own transposed layout.
 *   - All work is queued on the given stream; no entry point synchronises
 *     the host with the device.  Argument errors are found on the host and
 *     return before anything is queued.  A CUDA error returns FM_ERR_CUDA;
 *     fm_last_error() then describes it.
 *   - Calls on one context must not overlap on the device: the context's
 *     workspaces are shared by all of its calls.
 */
#ifndef FLASHMAP_H
#define FLASHMAP_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fm_stream;   /* a cudaStream_t; NULL = legacy default stream */
typedef struct fm_ctx fm_ctx;            /* opaque, owned by the library */

typedef enum {
  FM_OK = 0,
  FM_ERR_ARG = -1,          /* a pointer, size or value is invalid */
  FM_ERR_CUDA = -2,         /* a CUDA call failed; see fm_last_error() */
  FM_ERR_OOM = -3,          /* device allocation failed */
  FM_ERR_TIMEOUT = -4,      /* a bounded device wait gave up */
  FM_ERR_UNSUPPORTED = -5   /* shape outside the loaded configuration */
} fm_status;

typedef enum { FM_F32 = 0, FM_BF16 = 1 } fm_dtype;

/* Largest number of sequences in one fm_project_context / fm_draft call. */
#define FM_MAX_CALL_SEQS 256
/* Largest number of flow-map steps in one fm_draft call. */
#define FM_MAX_STEPS 8

/* Model shape and capacities.
 *   V             vocabulary (151,936 for Qwen3; P1 "一步生成整块，训练时做了什么")
 *   d             DiT width (2048), n_heads heads (16), head width d/n_heads
 *                 must be 128 (bf16) or any divisor-friendly size (fp32);
 *                 n_blocks DiT blocks (6) (P1, same section; P2 "Как
 *                 работает FlashMap?")
 *   mlp           MLP hidden width
 *   K             block size (16; P1 "一次猜 16 个 token，为什么还会前后不搭")
 *   target_hidden width of each tapped target hidden state
 *   n_taps        number of tapped target layers (5: layers 1, 9, 17, 25, 33)
 *   dtype         FM_F32 or FM_BF16
 *   max_ctx       context rows per sequence slot
 *   max_seqs      sequence slots of the context cache
 *   max_noise     noise drafts per sequence in one fm_draft call
 *   max_new       context rows per sequence in one fm_project_context call */
typedef struct {
  int V, d, n_blocks, n_heads, mlp, K, target_hidden, n_taps;
  int dtype;
  int max_ctx, max_seqs, max_noise, max_new;
} fm_config;

/* Device pointers to the drafter weights, all of dtype fm_config.dtype.
 *   E        [V, d]        frozen embedding table: noise x [K, V] enters as x E
 *   W_lm     [V, d]        frozen LM head: logits = h W_lm^T
 *   W_fc     [d, n_taps*H] projection of the concatenated tapped states
 *   W_ts1    [d, 256], W_ts2 [d, d]   embedder of the start time s
 *   W_tt1    [d, 256], W_tt2 [d, d]   embedder of the end time t
 *   W_ada_f  [2d, d]       final (shift, scale)
 *   W_qkv[l] [3d, d]  W_o[l] [d, d]  W_up[l] [mlp, d]  W_down[l] [d, mlp]
 *   W_ada[l] [6d, d]       (shift1, scale1, gate1, shift2, scale2, gate2)
 * The per-block members are host arrays of n_blocks device pointers. */
typedef struct {
  const void *E, *W_lm, *W_fc;
  const void *W_ts1, *W_ts2, *W_tt1, *W_tt2, *W_ada_f;
  const void *const *W_qkv;
  const void *const *W_o;
  const void *const *W_up;
  const void *const *W_down;
  const void *const *W_ada;
} fm_weights;

/* Creates a context on the current device: checks the shape, allocates the
 * context cache and workspaces, copies E into the library's transposed
 * layout and precomputes the adaLN modulation of the one-step (0 -> 1) and
 * two-step (0 -> 0.5 -> 1) grids (P2 "Как развернуть FlashMap?": num_steps
 * 2 trades speed for acceptance).  *out is set only on FM_OK. */
fm_status fm_load_weights(fm_ctx **out, const fm_config *cfg, const fm_weights *w,
                          fm_stream stream);

/* Releases everything the context owns.  NULL is a no-op. */
void fm_free(fm_ctx *ctx);

/* Text of the last error seen by this thread (never NULL). */
const char *fm_last_error(void);

/* Appends target features to the context cache (the drafter reads target
 * hidden states of five layers; P1 "一步生成整块，训练时做了什么").
 *   seq_ids  host [n_seqs]  distinct slots in [0, max_seqs)
 *   hidden   device [n_seqs, n_new, n_taps, target_hidden] dtype
 *   pos0     host [n_seqs]  first row written per slot; rows pos0..pos0+n_new-1
 *            are (re)written and the slot's context length becomes pos0+n_new
 * Computes C = LN0(concat_taps(hidden) W_fc^T) and, for every block l, the
 * context keys and values C W_k,l^T, C W_v,l^T.  Requires
 * 1 <= n_seqs <= FM_MAX_CALL_SEQS, 1 <= n_new <= max_new,
 * 0 <= pos0, pos0 + n_new <= max_ctx. */
fm_status fm_project_context(fm_ctx *ctx, const int32_t *seq_ids, int n_seqs,
                             const void *hidden, int n_new, const int32_t *pos0,
                             fm_stream stream);

/* Drafts one block per noise sample (P2 "Что такое FlashMap?": Gaussian
 * noise to a whole token block in one step).
 *   seq_ids      host [n_seqs]  slots whose context the drafts attend to
 *   noise        device [n_seqs, n_noise, K, V] dtype
 *   t_grid       host [num_steps + 1], 0 = t0 < t1 < ... < t_S = 1
 *   num_steps    1 .. FM_MAX_STEPS (one step is the flow map's single jump)
 *   temperature  host [n_seqs]; 0 selects the argmax (lowest index on ties;
 *                a NaN logit never wins, a row of NaN gives token 0),
 *                T > 0 samples softmax(logits / T) by inverse CDF
 *   u_draft      device [n_seqs, n_noise, K] uniforms in [0, 1) for sampled
 *                sequences; may be NULL when every temperature is 0
 *   tokens       device [n_seqs, n_noise, K] out
 *   draft_logits device [n_seqs, n_noise, K, V] out (fp32, the last step's
 *                logits before temperature), or NULL
 * Each step s -> t embeds the vocabulary-space state (x E), runs the DiT
 * conditioned on (s, t) and, for t < 1, moves the state by
 * x + ((t - s)/(1 - s)) (softmax(logits) - x). */
fm_status fm_draft(fm_ctx *ctx, const int32_t *seq_ids, int n_seqs,
                   const void *noise, int n_noise,
                   const float *t_grid, int num_steps,
                   const float *temperature, const double *u_draft,
                   int32_t *tokens, float *draft_logits, fm_stream stream);

/* Factorised drafting, the foil of the joint draft (P2 "Почему
 * diffusion-драфтеры теряют в доле принятых токенов?": a drafter that picks
 * each position on its own mixes modes, "new diego" / "san york", half the
 * time): position i of the block comes from its own independent noise block,
 * as if each position were drafted by a separate flow-map pass.
 *   noise        device [n_seqs, K, K, V] dtype: noise block i for position i
 *   u_draft      device [n_seqs, K] uniforms (position i), or NULL when greedy
 *   tokens       device [n_seqs, K] out: token i of the draft of noise block i
 *   draft_logits device [n_seqs, K, V] out (that draft's row i), or NULL
 * Other arguments as for fm_draft.  Runs the K drafts of a sequence as one
 * batched draft, so it needs max_noise >= K (else FM_ERR_UNSUPPORTED). */
fm_status fm_draft_factorised(fm_ctx *ctx, const int32_t *seq_ids, int n_seqs,
                              const void *noise, const float *t_grid, int num_steps,
                              const float *temperature, const double *u_draft,
                              int32_t *tokens, float *draft_logits, fm_stream stream);

/* Greedy verify (P5 "Why drafting still costs time": keep the longest valid
 * prefix, resume from a target token; P2 "Что такое FlashMap?": the result
 * equals the target's own greedy output).
 *   target_logits device [B, N, K+1, V] fp32; row i of draft j scores
 *                 position i+1 after that draft's first i tokens
 *   draft         device [B, N, K]
 *   n_acc         device [B] out: accepted drafted tokens n (0..K)
 *   branch        device [B] out: the draft with the largest n (lowest on ties)
 *   out_tokens    device [B, K+1] out: the n accepted tokens, then the
 *                 target argmax at position n+1, then -1 padding
 * Argmax ties go to the lowest index; NaN never wins (it ranks below every
 * number, -inf included; a row of NaN gives token 0).  Bit-exact. */
fm_status fm_verify_greedy(fm_ctx *ctx, const float *target_logits, const int32_t *draft,
                           int B, int N, int K, int V,
                           int32_t *n_acc, int32_t *branch, int32_t *out_tokens,
                           fm_stream stream);

/* Stochastic verify at temperature T > 0 (P1 "能拿来做什么" and P2 "Как
 * развернуть FlashMap?": probabilistic draft sampling for T > 0; lossless
 * in distribution, P5 "Why drafting still costs time").
 *   p = softmax(target / T); q = softmax(draft_logits / T), or the point mass
 *   on the drafted token when draft_logits is NULL.
 *   At each depth the drafts still on the accepted prefix are tried in index
 *   order: draft j is accepted iff u_accept[b,j,i] * q(y) < p'(y), else
 *   p' <- normalise(max(0, p' - q)).  If none is accepted one token is drawn
 *   from p' by inverse CDF at u_res[b]; if all K depths accept, the bonus
 *   token is drawn from row K of the accepted branch.
 *   u_accept device [B, N, K] fp64, u_res device [B] fp64, both in [0, 1).
 * Sums are fp64; decisions match an fp64 evaluation except within ~1e-12
 * of a threshold.  Outputs as for fm_verify_greedy. */
fm_status fm_verify_sample(fm_ctx *ctx, const float *target_logits, const float *draft_logits,
                           const int32_t *draft, int B, int N, int K, int V, float temperature,
                           const double *u_accept, const double *u_res,
                           int32_t *n_acc, int32_t *branch, int32_t *out_tokens,
                           fm_stream stream);

/* ---- Target-side tree scoring of a sequence's noise drafts (P1 "6.14 倍是最好
 * 成绩…": four noise drafts scored as a tree add about 11 % mean speedup).
 * Drafts that share a prefix need the target's distribution after it once:
 * the target scores the nodes of the drafts' prefix trie in one pass, each
 * node attending to the context and to its ancestors.  Node order is breadth
 * first, and within a depth the order of the first draft that creates the
 * node.  Node n is a prefix of length depth + 1 ending in its token; parent
 * -1 at depth 0.  Target rows of a tree: row 0 is the root (the first
 * drafted position's distribution), row 1 + n node n's. */

/* Builds the trie of each sequence's N drafts.  No context, no allocation.
 *   draft        device [B, N, K]
 *   node_token, node_parent, node_depth  device [B, N*K] out; entries past
 *                the sequence's node count are -1
 *   n_nodes      device [B] out
 *   draft_node   device [B, N, K] out: the node of draft j's prefix of
 *                length i + 1
 *   anc_mask     device [B, N*K, W] out, W = ceil(N*K / 64): bit m of node
 *                n's words is set iff m is n or one of its ancestors
 * Requires N <= 32 and N*K <= 1024 (else FM_ERR_UNSUPPORTED).  Exact. */
fm_status fm_build_tree(const int32_t *draft, int B, int N, int K, int32_t *node_token,
                        int32_t *node_parent, int32_t *node_depth, int32_t *n_nodes,
                        int32_t *draft_node, uint64_t *anc_mask, fm_stream stream);

/* The attention that scores a tree's nodes in one pass: node n's query
 * attends over the context rows and over the rows of n and its ancestors
 * (softmax scale 1/sqrt(dh)), per head.  fp32, no context, no allocation;
 * a reference of the mask's meaning for a target's own attention.
 *   q, k_nodes, v_nodes device [B, NN, n_heads*dh]; k_ctx, v_ctx device
 *   [B, L, n_heads*dh] (L may be 0); anc_mask, n_nodes from fm_build_tree
 *   (NN = N*K); out device [B, NN, n_heads*dh], rows past n_nodes untouched.
 * Requires NN <= 1024 and dh <= 128. */
fm_status fm_tree_attention(const float *q, const float *k_ctx, const float *v_ctx,
                            const float *k_nodes, const float *v_nodes, const uint64_t *anc_mask,
                            const int32_t *n_nodes, int B, int NN, int L, int n_heads, int dh,
                            float *out, fm_stream stream);

/* Greedy and stochastic verify of a tree whose target rows are given per
 * node: node_logits device [B, R, V] fp32, R >= 1 + N*K (row 0 the root,
 * row 1 + n node n), draft_node from fm_build_tree.  Results are those of
 * fm_verify_greedy / fm_verify_sample on the per-draft rows the nodes stand
 * for (shared prefixes share rows). */
fm_status fm_verify_greedy_tree(fm_ctx *ctx, const float *node_logits, int R, const int32_t *draft,
                                const int32_t *draft_node, int B, int N, int K, int V,
                                int32_t *n_acc, int32_t *branch, int32_t *out_tokens,
                                fm_stream stream);
fm_status fm_verify_sample_tree(fm_ctx *ctx, const float *node_logits, int R,
                                const float *draft_logits, const int32_t *draft,
                                const int32_t *draft_node, int B, int N, int K, int V,
                                float temperature, const double *u_accept, const double *u_res,
                                int32_t *n_acc, int32_t *branch, int32_t *out_tokens,
                                fm_stream stream);

/* Greedy verify that allocates nothing and needs no context: same inputs,
 * outputs and bit-exact results as fm_verify_greedy (the pages have no
 * counterpart; this is a deployment variant).  It is for callers that
 * cannot allocate device memory -- servers whose arena owns the whole
 * device, or verify-only users without a drafter context.  Its scratch is a
 * fixed device array inside the library (about 260 KB on every GPU that
 * loads it, kept until exit), so: B <= 1024, N*(K+1) <= 1024,
 * B*N*(K+1) <= 32768 and V <= 2^28, else FM_ERR_UNSUPPORTED (checked on
 * the host before anything is queued).  The first call on a device
 * looks the array up (cudaGetSymbolAddress) and should come before any
 * stream capture.  Each call clears the scratch counters it uses; all calls
 * share the one array, so calls that overlap on the same GPU (issued on
 * different streams or from different host threads) race and must be
 * serialised by the caller.  No cudaMalloc, cudaFree or allocating library
 * call is made. */
fm_status fm_verify_greedy_noalloc(const float *target_logits, const int32_t *draft,
                                   int B, int N, int K, int V,
                                   int32_t *n_acc, int32_t *branch, int32_t *out_tokens,
                                   fm_stream stream);

/* Reads and clears the context's device error word: FM_OK, or
 * FM_ERR_TIMEOUT when a bounded wait inside a kernel gave up (about two
 * seconds; the kernel then stopped early and the outputs of the calls since
 * the last check are invalid).  On FM_ERR_TIMEOUT it also returns the
 * context's arrival counters to zero, so the next call starts clean; context
 * rows projected by the failed calls may be missing from the cache and are
 * projected again by the caller.  Waits for the work queued on `stream`. */
fm_status fm_device_status(fm_ctx *ctx, fm_stream stream);

/* Kernel classes for launch counting and optional device timing. */
#define FM_PROF_EMBED 0     /* soft-embedding GEMM x.E (and D.E of later steps) */
#define FM_PROF_DIT_GEMM 1  /* QKV, O, MLP GEMMs of the DiT blocks */
#define FM_PROF_ATTN 2      /* attention over [context; block] */
#define FM_PROF_NORM 3      /* modulated LayerNorm, softmax rows, token selection */
#define FM_PROF_LM_HEAD 4   /* LM-head GEMM (and its fused argmax) */
#define FM_PROF_CONTEXT 5   /* context projection (fc, LayerNorm, keys/values) */
#define FM_PROF_VERIFY 6    /* verify kernels */
#define FM_PROF_OTHER 7     /* conditioning, transposes (load time) */
#define FM_PROF_N 8

/* Device timing of chosen kernel classes.  `mask` is a bit set of
 * (1 << FM_PROF_*); while it is non-zero the library records a CUDA event
 * pair on the call's stream around every launch of a chosen class (up to
 * 65,536 pairs; later launches are counted but not timed).  Setting a mask
 * clears the previous records; 0 stops recording. */
fm_status fm_profile(fm_ctx *ctx, int mask);

/* Per class: total device milliseconds of the timed launches (ms, may be
 * NULL) and the number of kernel launches since the context was created
 * or since the last call with reset != 0 (launches, may be NULL).  Both
 * arrays have FM_PROF_N entries.  Waits for the recorded events. */
fm_status fm_profile_read(fm_ctx *ctx, double *ms, int64_t *launches, int reset);

/* Self-check of the fp64 exponential the stochastic verify sums with
 * (Tang's table-driven method; valid for arguments <= 0, the softmax
 * weights exp((l - max)/T)).  Device arrays: e[n] (arguments), mine[n]
 * (that function) and ref[n] (CUDA's exp of the same argument).  No
 * context needed; FM_ERR_ARG for NULL pointers or n < 0.  Asynchronous
 * on `stream`. */
fm_status fm_selftest_exp(const double *e, double *mine, double *ref, int n, fm_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* FLASHMAP_H */
