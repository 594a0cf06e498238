/*
 * medusa.h - C ABI of libmedusa.so: the per-step Medusa draft-and-verify
 * chain (heads -> top-s -> tree -> tree attention -> acceptance -> KV
 * compaction) as CUDA kernels for sm_100a (B200).
 *
 * Sources (page title, then section):
 *   [MD] "論文解説: Medusa — 複数デコーディングヘッドによるLLM推論高速化フレームワーク":
 *        "Medusa Headのアーキテクチャ" (head equation), "ツリーアテンションによる
 *        並列検証" (top-s, Cartesian-product tree, ancestor mask),
 *        "候補選択：Typical Acceptance" (typical and greedy acceptance).
 *   [EX] "メドゥーサ デコーディング ヘッド", "ディープダイブ" (accept the longest
 *        matching prefix).
 *   [FR] "Medusa" (glossaire), "Attention en arbre" (each node sees only its
 *        ancestors; the longest valid path is accepted).
 *   [ZH] "Medusa：基于多Token预测的LLM推理加速", "3.3 贪婪vs采样验证" (greedy
 *        versus sampling verification).
 *
 * Conventions shared by every call:
 *   - Return value: MEDUSA_OK (0) or a negative medusa_status.  On error
 *     medusa_last_error() (thread-local) describes the failure.  Nothing is
 *     launched when argument validation fails.  No C++ exception crosses
 *     the ABI.
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or retains them.  Layouts are row-major and
 *     contiguous as written in brackets, e.g. h [B][d].
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every compute call is asynchronous on that stream and never
 *     synchronizes the host.
 *   - `ws`/`ws_bytes` is caller-owned device scratch of at least the size the
 *     matching *_workspace_size() call returns, 256-byte aligned.  Its
 *     contents on entry are irrelevant; calls sharing one workspace must be
 *     ordered on the GPU (same stream, or synchronized).
 *   - Outputs are completely overwritten; no pre-zeroing is required.
 *   - dtype is MEDUSA_F32 or MEDUSA_BF16 and applies to every floating-point
 *     tensor argument of the call that is not explicitly typed float*.
 *   - Device-side waits are bounded.  A kernel whose wait runs out sets a
 *     device status word and returns early (its outputs are then undefined);
 *     medusa_device_status() reports MEDUSA_ERR_TIMEOUT.
 */
#ifndef MEDUSA_H_
#define MEDUSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MEDUSA_OK = 0,
  MEDUSA_ERR_INVALID_ARG = -1, /* null pointer, bad size, bad tree, ... */
  MEDUSA_ERR_UNSUPPORTED = -2, /* valid but not implemented (dtype/shape) */
  MEDUSA_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed */
  MEDUSA_ERR_TIMEOUT = -4,     /* a device-side bounded wait ran out */
  MEDUSA_ERR_BOUNDS = -5       /* a device-side index check failed (debug build) */
} medusa_status;

typedef enum { MEDUSA_F32 = 0, MEDUSA_BF16 = 1 } medusa_dtype;

/* Opaque, immutable tree plan (library-owned host + device copy). */
typedef struct medusa_tree medusa_tree_t;

/* Limits of this build. */
#define MEDUSA_MAX_K 8      /* Medusa heads = maximum tree depth */
#define MEDUSA_MAX_S 16     /* top-s per head */
#define MEDUSA_MAX_N 256    /* tree nodes, root included */

/* Thread-local message for the last failing call on this thread ("" if none). */
const char* medusa_last_error(void);

/* Library version string. */
const char* medusa_version(void);

/*
 * Reads (and with clear != 0 resets) the device status word of the current
 * device.  Synchronizes the device.  *status receives MEDUSA_OK,
 * MEDUSA_ERR_TIMEOUT or, from the debug build, MEDUSA_ERR_BOUNDS (then
 * medusa_last_error() names the first failing check site).  Returns
 * MEDUSA_ERR_CUDA if the device is unusable.
 *
 * Debug build (libmedusa_debug.so, compiled with MEDUSA_DEBUG; the Python
 * binding loads it when the environment has MEDUSA_DEBUG=1): every kernel
 * also checks the indices it derives from its inputs (tree slots against the
 * cache, nodes against N, tokens against V, plan entries against K s).  A
 * failed check records MEDUSA_ERR_BOUNDS in the status word and skips the
 * access (it never traps).  Sites: 1 tree expansion (head, rank) index,
 * 2 attention key tile, 3 attention key slot (SIMT kernel), 4 acceptance
 * parent, 5 acceptance tree token, 6 compaction node, 7 sampling node,
 * 8 shard-merge candidate id.  Results of the release build are identical.
 */
int medusa_device_status(int* status, int clear);

/*
 * Failure-detection self-test; the pages have no counterpart (it checks the
 * library's own bounded device waits).  Launches one CTA on `stream` (a
 * cudaStream_t, NULL = default stream) whose single thread waits, with the
 * same bounded wait every kernel of the library uses, for an mbarrier phase
 * that nothing completes, giving up after `limit_ms` milliseconds of global
 * time (1 <= limit_ms <= 2000).  The wait runs out, the kernel raises the
 * device status word and returns normally: afterwards medusa_device_status()
 * reports MEDUSA_ERR_TIMEOUT and the CUDA context stays usable.  Returns
 * MEDUSA_ERR_INVALID_ARG for a limit out of range, MEDUSA_ERR_CUDA if the
 * launch fails; asynchronous otherwise.
 */
int medusa_selftest_wait_timeout(int limit_ms, void* stream);

/* ------------------------------------------------------------------------
 * Tree plan.  [MD] "ツリーアテンションによる並列検証": each of the K heads
 * proposes its top-s tokens; their Cartesian product is pruned to a tree.
 * Pruning rule: keep the N rank tuples (r_1..r_D), 0 <= D <= K, 0-based
 * ranks, with the largest score prod_i 0.5^{r_i} * 0.8^D.  N includes the
 * root (the empty tuple).  Score ties break by (depth asc, tuple
 * lexicographic asc).  Node order is (depth asc, tuple lexicographic asc):
 * node 0 is the root and parent[n] < n.
 * ------------------------------------------------------------------------ */

/*
 * Host only (no CUDA call): fills caller-owned HOST arrays
 *   parent[N] (-1 for the root), depth[N], rank_path[N][K] (-1 padded),
 *   anc_mask[N][(N+31)/32] (bit j of row i set iff node j is node i or one
 *   of its ancestors).
 * Any output pointer may be NULL.  Errors: INVALID_ARG if K, s, N are out of
 * [1, MEDUSA_MAX_*] or N exceeds the number of tuples 1 + s + ... + s^K.
 */
int medusa_tree_plan_host(int K, int s, int N, int32_t* parent, int32_t* depth,
                          int32_t* rank_path, uint32_t* anc_mask);

/*
 * Builds the plan and uploads it to the CURRENT device (synchronous upload).
 * *out receives the handle; release it with medusa_tree_destroy.
 */
int medusa_tree_create(int K, int s, int N, medusa_tree_t** out);
int medusa_tree_destroy(medusa_tree_t* tree);

/* Host copies of a plan's shape and arrays (same layouts as plan_host). */
int medusa_tree_info(const medusa_tree_t* tree, int* K, int* s, int* N,
                     int32_t* parent, int32_t* depth, int32_t* rank_path,
                     uint32_t* anc_mask);

/* ------------------------------------------------------------------------
 * Medusa heads.  [MD] "Medusa Headのアーキテクチャ":
 *   logits_k[b] = W2_k (SiLU(W1_k h[b] + b1_k) + h[b]),  k = 0..K-1,
 * SiLU(x) = x * sigmoid(x).  Head k (0-based) predicts the token k+2 steps
 * ahead of the last verified token.
 * ------------------------------------------------------------------------ */

/* Scratch bytes needed by medusa_heads_forward for these sizes. */
size_t medusa_heads_workspace_size(int B, int d, int V, int K, int s, int dtype);

/*
 * h [B][d]; W1 [K][d][d] (row = output feature); b1 [K][d] or NULL (= 0);
 * W2 [K][V][d] (row = vocabulary entry); all of `dtype`.
 * Outputs (each may be NULL, not both):
 *   logits   [B][K][V] fp32;
 *   topk_idx [B][K][s] int32: the s best vocabulary ids of each (b, k),
 *            by logit descending, ties to the lower id;
 *   topk_val [B][K][s] fp32 (only written when topk_idx is non-NULL).
 * bf16: W1 and W2 are streamed by tcgen05 tensor-core GEMMs (TMA-fed, fp32
 * accumulation in TMEM) with the bias, SiLU and residual applied between
 * the two GEMMs and a partial top-s fused in the second's epilogue.  The
 * hidden activation u is passed to the second GEMM as a bf16 hi/lo pair (u =
 * hi + lo), so it keeps ~16 mantissa bits.  B <= 32: weight-streaming
 * kernels (activations as a narrow N operand, HBM-bound).  32 < B <=
 * MEDUSA_MAX_HEADS_B: compute-bound kernels with N = 256 activation columns
 * per tile (the second GEMM executes 2x the method's flops, for hi and lo).
 * fp32: SIMT kernels.
 * Limits: d % 8 == 0; B <= MEDUSA_MAX_HEADS_B (bf16) or 16 (fp32);
 * K <= MEDUSA_MAX_K; 1 <= s <= MEDUSA_MAX_S, s <= V.  Pointers 16-byte
 * aligned.
 */
#define MEDUSA_MAX_HEADS_B 4096
int medusa_heads_forward(const void* h, const void* W1, const void* b1,
                         const void* W2, int B, int d, int V, int K, int dtype,
                         float* logits, int s, int32_t* topk_idx,
                         float* topk_val, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * Top-s of each row of logits [R][V] (dtype): idx [R][s] int32 (value
 * descending, ties to the lower index); val [R][s] fp32 or NULL.
 * 1 <= s <= MEDUSA_MAX_S, s <= V.
 */
int medusa_topk(const void* logits, int dtype, int R, int V, int s,
                int32_t* idx, float* val, void* stream);

/* ------------------------------------------------------------------------
 * Tree expansion: node n with rank tuple (r_1..r_D) carries
 *   tree_tok[b][n] = root_tok[b]                      if D == 0
 *                  = topk_idx[b][D-1][r_D]            otherwise
 * (head D-1, 0-based, proposes the token at tree depth D), and
 *   tree_pos[b][n] = prefix_len[b] + D.
 * root_tok [B], topk_idx [B][K][s], prefix_len [B] int32 device arrays.
 * ------------------------------------------------------------------------ */
int medusa_build_tree(const medusa_tree_t* tree, const int32_t* root_tok,
                      const int32_t* topk_idx, const int32_t* prefix_len,
                      int B, int32_t* tree_tok, int32_t* tree_pos,
                      void* stream);

/* ------------------------------------------------------------------------
 * Tree attention.  [MD] Mask_ij = 1 iff j is an ancestor of i (the node
 * itself included).  For sequence b, tree node i and query head h:
 *   out[b][i][h] = softmax_j(scale * q[b][i][h] . k_j) v_j
 * over the keys j in {prefix slots 0..L_b-1} U {slot L_b + a : a is node i
 * or an ancestor of i}, where L_b = prefix_len[b] and the tree tokens' K/V
 * sit at slots L_b..L_b+N-1 of the cache.  kv-head of query head h is
 * h / (Hq/Hkv).
 * q [B][N][Hq][dh]; k_cache, v_cache [B][Lcap][Hkv][dh]; out [B][N][Hq][dh].
 * Requires L_b + N <= Lcap (checked on the device: rows of a sequence that
 * violates it are written as zeros and the status word is left untouched).
 * Slots 0..L_b+N-1 of sequence b must hold finite values; slots L_b+N and
 * beyond (unused capacity) may hold anything, NaN and Inf included: they get
 * weight exactly 0 and never reach the output.  Further requirements:
 * Hq % Hkv == 0, dh in {64, 128}, scale finite and > 0 (normally
 * 1/sqrt(dh)).  bf16 with dh = 128 and (Hq/Hkv) dividing 128 runs on the
 * tcgen05 tensor-core kernels (one or two 128-row query tiles per CTA, keys
 * split into chunks where that fills the device; the choice is reported by
 * the introspection calls below); other shapes on a SIMT kernel.
 * ------------------------------------------------------------------------ */
size_t medusa_tree_attention_workspace_size(const medusa_tree_t* tree, int B,
                                            int Hq, int Hkv, int dh, int Lcap);

/*
 * Number of key chunks medusa_tree_attention splits each (sequence, kv-head)
 * into for these sizes on the current device (>= 1).  With more than one,
 * the chunks' partial results are merged either inside the attention kernel
 * (bf16, dh = 128, at most 8 chunks, and every thread-block cluster of the
 * chunks of one query tile resident on the device at once: the chunks merge
 * through distributed shared memory) or by a combine kernel that follows it.
 * Negative status on bad arguments.  Introspection only.
 */
int medusa_tree_attention_chunks(const medusa_tree_t* tree, int B, int Hq,
                                 int Hkv, int dh, int Lcap, int dtype);

/*
 * Number of kernels one medusa_tree_attention call with these sizes launches
 * on the current device (0 for B = 0, else 1 or 2).  Negative status on bad
 * arguments.  Introspection only (used to count kernel launches).
 */
int medusa_tree_attention_launches(const medusa_tree_t* tree, int B, int Hq,
                                   int Hkv, int dh, int Lcap, int dtype);

/*
 * 128-row query tiles one CTA of medusa_tree_attention takes for these sizes
 * on the current device: 2 when the keys are not split, a (sequence,
 * kv-head) has at least two query tiles and pairing them saves enough waves
 * of CTAs on the device (both tiles then share every K/V tile the CTA
 * stages), else 1.
 * Negative status on bad arguments.  Introspection only.
 */
int medusa_tree_attention_tiles_per_cta(const medusa_tree_t* tree, int B,
                                        int Hq, int Hkv, int dh, int Lcap,
                                        int dtype);

int medusa_tree_attention(const void* q, const void* k_cache,
                          const void* v_cache, const int32_t* prefix_len,
                          const medusa_tree_t* tree, int B, int Hq, int Hkv,
                          int dh, int Lcap, float scale, int dtype, void* out,
                          void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Acceptance over verify logits vlogits [B][N][V] (dtype) for the tree
 * tokens tree_tok [B][N].
 *   greedy  ([MD], temperature 0): node n != 0 is accepted iff its parent is
 *           accepted and argmax(vlogits[b][parent]) == tree_tok[b][n]
 *           (argmax ties to the lowest id).
 *   typical ([MD] "候補選択：Typical Acceptance"): node n != 0 is accepted iff
 *           its parent is accepted and p(tok) > min(eps, delta*exp(-H(p)))
 *           with p = softmax(vlogits[b][parent] / temperature) and
 *           H(p) = -sum p ln p.
 * The deepest accepted node wins (ties: lowest node index) ([EX], [FR]).
 * Outputs: accept_len [B] (its depth, 0..K); accept_nodes [B][K+1] (node
 * ids on the root-to-node path, root first, -1 padded); next_tok [B] (argmax
 * of the winning node's verify row).
 * ------------------------------------------------------------------------ */
size_t medusa_accept_workspace_size(const medusa_tree_t* tree, int B, int V);

int medusa_accept_greedy(const void* vlogits, int dtype, const int32_t* tree_tok,
                         const medusa_tree_t* tree, int B, int V,
                         int32_t* accept_len, int32_t* accept_nodes,
                         int32_t* next_tok, void* ws, size_t ws_bytes,
                         void* stream);

int medusa_accept_typical(const void* vlogits, int dtype,
                          const int32_t* tree_tok, const medusa_tree_t* tree,
                          int B, int V, float temperature, float eps,
                          float delta, int32_t* accept_len,
                          int32_t* accept_nodes, int32_t* next_tok, void* ws,
                          size_t ws_bytes, void* stream);

/*
 * Greedy and typical acceptance of the same verify logits in one pass over
 * them (a workload that verifies under both rules, as the long-context
 * configuration does): writes exactly what medusa_accept_greedy (g_*) and
 * medusa_accept_typical (t_*) write for the same arguments.  One row
 * reduction serves both walks, since the typical pass keeps every row's
 * argmax.  Workspace: medusa_accept_workspace_size's.  Errors: those of
 * medusa_accept_typical, and MEDUSA_ERR_INVALID_ARG (nothing launched) when
 * a greedy output is NULL or the two output sets share a pointer.
 */
int medusa_accept_greedy_typical(const void* vlogits, int dtype,
                                 const int32_t* tree_tok,
                                 const medusa_tree_t* tree, int B, int V,
                                 float temperature, float eps, float delta,
                                 int32_t* g_accept_len, int32_t* g_accept_nodes,
                                 int32_t* g_next_tok, int32_t* t_accept_len,
                                 int32_t* t_accept_nodes, int32_t* t_next_tok,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * Typical acceptance with one temperature per head.  [ZH] "4.2 温度调优"
 * tunes a temperature per Medusa head; reading: head D proposes the
 * candidates of depth D, and each is verified on its parent's row at
 * temperatures[D-1] (a host array of K floats, each finite and > 0; the
 * workspace is medusa_accept_workspace_size's).  With all K equal this is
 * medusa_accept_typical.  next_tok is the argmax of the last accepted row.
 */
int medusa_accept_typical_per_head(const void* vlogits, int dtype,
                                   const int32_t* tree_tok,
                                   const medusa_tree_t* tree, int B, int V,
                                   const float* temperatures, float eps,
                                   float delta, int32_t* accept_len,
                                   int32_t* accept_nodes, int32_t* next_tok,
                                   void* ws, size_t ws_bytes, void* stream);

/*
 * medusa_accept_greedy without a workspace argument, for callers that cannot
 * allocate device memory: code that runs where cudaMalloc and allocating
 * libraries are off limits (for example a serving loop whose device memory
 * was partitioned up front, or a host language binding with no device
 * allocator of its own).  The paper has no counterpart; this is a library
 * convenience.  Same inputs, outputs and results as medusa_accept_greedy.
 * Its scratch is a fixed array inside the library of
 * MEDUSA_NOALLOC_ACCEPT_PARTS row-chunk records (24 bytes each, 1.5 MiB),
 * which every GPU that loads the library holds until the process exits.
 * Limit: B * N <= MEDUSA_NOALLOC_ACCEPT_PARTS, else MEDUSA_ERR_INVALID_ARG
 * and nothing is launched.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress, host side, once per device and
 * context: after a cudaDeviceReset the next call looks it up again in the
 * new context); make that first call before any stream capture.  All calls
 * share the array:
 * calls that may overlap on the GPU (different streams without ordering)
 * race and must be serialized by the caller.  No memory is allocated or
 * freed by this call.
 */
#define MEDUSA_NOALLOC_ACCEPT_PARTS 65536
int medusa_accept_greedy_noalloc(const void* vlogits, int dtype,
                                 const int32_t* tree_tok,
                                 const medusa_tree_t* tree, int B, int V,
                                 int32_t* accept_len, int32_t* accept_nodes,
                                 int32_t* next_tok, void* stream);

/* ------------------------------------------------------------------------
 * KV compaction of the accepted path (the accepted tokens' K/V become the
 * contiguous continuation of the sequence):
 *   for j = 1..accept_len[b]: slot L_b + j <- slot L_b + accept_nodes[b][j]
 * in k_cache and v_cache [B][Lcap][Hkv][dh] (in place, bit-exact), and
 *   new_len[b] = L_b + 1 + accept_len[b]   (root + accepted tokens).
 * accept_nodes [B][K+1] as written by the accept calls.  Entries with
 * accept_len outside [0, K] or nodes outside the cache are skipped.
 * ------------------------------------------------------------------------ */
int medusa_kv_compact(void* k_cache, void* v_cache, const int32_t* prefix_len,
                      const int32_t* accept_len, const int32_t* accept_nodes,
                      int B, int Hkv, int dh, int Lcap, int K, int dtype,
                      int32_t* new_len, void* stream);

/*
 * medusa_kv_compact over the caches of n_layers layers in one launch.
 * [MD] "ツリーアテンションによる並列検証": the tree is verified in one forward
 * pass of the base model, so every layer has written the tree's K/V at slots
 * L_b..L_b+N-1 of its own cache, and the accepted path is kept in each.
 * Layer l's caches start at k_caches + l * layer_stride and v_caches + l *
 * layer_stride (elements of dtype; layer_stride >= B * Lcap * Hkv * dh when
 * n_layers > 1), each [B][Lcap][Hkv][dh].  prefix_len, accept_len,
 * accept_nodes and new_len are shared by the layers (new_len written once).
 * Same rules and skipped entries as medusa_kv_compact; n_layers = 1 is
 * medusa_kv_compact.
 */
int medusa_kv_compact_layers(void* k_caches, void* v_caches, int n_layers,
                             long long layer_stride, const int32_t* prefix_len,
                             const int32_t* accept_len, const int32_t* accept_nodes,
                             int B, int Hkv, int dh, int Lcap, int K, int dtype,
                             int32_t* new_len, void* stream);

/* ------------------------------------------------------------------------
 * Merge of top-s candidate lists from G vocabulary shards (heads whose W2
 * rows are split across ranks: each rank's medusa_heads_forward top-s over
 * its slice, gathered, then merged).  [MD] "ツリーアテンションによる並列検証":
 * each head contributes its s most likely tokens.  Shard g's list for row
 * r is val[g * shard_stride + r * c + j] fp32 and idx[...] int32 with the
 * same offsets, j < c (index < 0: empty slot); shard_stride >= R * c
 * elements (R * c for dense [G][R][c] arrays; 2 * R * c for the [G][2][R][c]
 * buffer an all-gather of [values; ids] planes produces).  Shard g's indices
 * are offset by v0[g] (device int32 [G]; NULL = no offset).  Per row r
 * writes the s best candidates by value descending, ties to the lower
 * (offset) index: out_idx [R][s] and, if non-NULL, out_val [R][s]; -1 / NaN
 * where fewer than s candidates exist.  1 <= s <= MEDUSA_MAX_S.
 * ------------------------------------------------------------------------ */
int medusa_topk_merge(const float* val, const int32_t* idx,
                      long long shard_stride, const int32_t* v0, int G, int R,
                      int c, int s, int32_t* out_idx, float* out_val,
                      void* stream);

/* ------------------------------------------------------------------------
 * Sampled next token.  [ZH] "3.3 贪婪vs采样验证": greedy verification takes
 * the argmax, sampling verification draws from softmax(logits / T).  For
 * every sequence b the token is drawn from the verify row
 * vlogits[b][n_a][0..V) of its last accepted node n_a =
 * accept_nodes[b][accept_len[b]] (accept_len / accept_nodes [B][K+1] as the
 * accept calls write them; N = tree nodes).  temperature == 0: the argmax
 * (lowest index on ties).  temperature > 0: argmax_v of
 * fl(fl(l_v * (1/T)) + G_v) in fp32, G_v = -log(-log(U_v)) standard Gumbel
 * noise (Gumbel-max: a draw from softmax(l / T)), U_v = (t + 1/2) * 2^-23
 * with t the top 23 bits of output number ((offset * B) + b) * V + v of
 * SplitMix64 started at `seed` (Steele, Lea & Flood, OOPSLA 2014); offset =
 * `offset` + *offset_dev when offset_dev (a device uint64, read when the
 * kernel runs) is not NULL.  The result depends only on (seed, offset) and
 * the inputs: pass a new offset for every call that must draw fresh noise
 * (offset_dev lets a captured CUDA graph advance it on the device between
 * replays).  A sequence whose accept_len
 * is outside [0, K] or whose node is outside [0, N) gets next_tok = -1.
 * temperature must be finite and >= 0.  Writes next_tok [B] only.
 * ------------------------------------------------------------------------ */
int medusa_sample_next(const void* vlogits, int dtype, const int32_t* accept_len,
                       const int32_t* accept_nodes, int B, int N, int V, int K,
                       float temperature, uint64_t seed, uint64_t offset,
                       const uint64_t* offset_dev, int32_t* next_tok, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MEDUSA_H_ */
