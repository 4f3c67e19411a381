/*
 * medusa.h - C ABI of the Medusa decode-verify step on NVIDIA B200 (sm_100a).
 *
 * One decode-verify step of Medusa speculative decoding, in five stage calls:
 *
 *   medusa_heads_topk      K Medusa heads on the last hidden state, then a
 *                          top-k over the vocabulary per head;
 *   medusa_tree_build      candidate tree from those top-k lists: candidate
 *                          ids, position ids, ancestor mask, retrieve paths;
 *   medusa_tree_attention  attention of every tree node over the cached
 *                          prefix and its own ancestors;
 *   medusa_verify_accept   the longest branch the base model agrees with
 *                          (greedy match or typical acceptance);
 *   medusa_kv_compact      the kept branch's K/V moved into contiguous slots.
 *
 * Around them: medusa_lmhead_verify (the verification from the nodes' hidden
 * states, lm_head fused), medusa_next_step (inputs of the next step),
 * medusa_sample_bonus (a drawn bonus token), medusa_heads_topk_tree and
 * medusa_verify_accept_compact (the first two and the last two calls, each
 * pair in one), medusa_tree_from_accuracies
 * (the sparse tree of the most accurate combinations, host only), the
 * vocabulary-sharding calls (medusa_topk_merge, medusa_verify_records,
 * medusa_verify_from_records), medusa_verify_accept_noalloc and
 * medusa_wait_flag (a check of the bounded device waits).
 *
 * Sources (page title, then section):
 *   "Medusa Heads" glossary - "Comment les têtes prédisent les tokens
 *     suivants" (the head) and "Attention arborescente et acceptation" (tree,
 *     tree mask, greedy and typical acceptance, longest kept branch);
 *   "Medusa Decoding Heads" overview - "Diepe duik" (one-pass verification of
 *     the whole tree, losslessness);
 *   "Medusa no contexto de LLMs" - "o que significa medusa na prática de
 *     deploy" (accepted tokens enter the sequence without another pass; the
 *     conventionally generated token on rejection);
 *   "Medusa: Simple LLM Inference Acceleration Framework with Multiple
 *     Decoding Heads" - abstract (tree-based attention over candidate
 *     continuations, one decoding step).
 *
 * Conventions for every call
 *   - Pointers named as device pointers must point to memory of the current
 *     CUDA device; host pointers are read before the call returns.  The
 *     caller owns every buffer.  The library never allocates device memory
 *     and never synchronises: all work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - All arrays are dense, row-major, with the layouts given per call.
 *     bf16 arrays are IEEE bfloat16 bit patterns (uint16).
 *   - Errors the host can see (null pointer, unsupported size, misaligned
 *     pointer, workspace too small) are returned before anything is launched.
 *     MEDUSA_ERR_CUDA reports a failed launch; medusa_last_error() then holds
 *     the CUDA error text.
 *   - Errors only the device can see (an index out of range in a tree or an
 *     accepted path, a NaN logit, a bounded wait that ran out) are written
 *     into *dev_status (device int32, 0 = OK) with an atomic compare-and-swap,
 *     so the first error sticks.  The caller zeroes it once and reads it after
 *     its own synchronisation.  No kernel traps; outputs of a call that set a
 *     device error are unspecified but every write stays inside its buffer.
 *   - The library is re-entrant.  Calls on the same stream run in order; the
 *     caller orders calls on different streams.
 */
#ifndef MEDUSA_B200_H
#define MEDUSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MEDUSA_API __attribute__((visibility("default")))
#else
#define MEDUSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MEDUSA_OK = 0,
  MEDUSA_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, negative size      */
  MEDUSA_ERR_SHAPE = 2,        /* sizes outside the supported limits          */
  MEDUSA_ERR_UNSUPPORTED = 3,  /* valid request this build does not handle    */
  MEDUSA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed           */
  MEDUSA_ERR_TIMEOUT = 5,      /* device: a bounded wait ran out              */
  MEDUSA_ERR_DEVICE_CHECK = 6, /* device: index out of range, NaN input       */
  MEDUSA_ERR_WORKSPACE = 7,    /* workspace pointer null or too small         */
  MEDUSA_ERR_ALIGNMENT = 8     /* pointer not aligned as the call requires    */
} medusa_status_t;

typedef enum { MEDUSA_BF16 = 0, MEDUSA_F32 = 1 } medusa_dtype_t;
typedef enum { MEDUSA_ACCEPT_GREEDY = 0, MEDUSA_ACCEPT_TYPICAL = 1 } medusa_accept_t;

/* Limits of this build. */
#define MEDUSA_MAX_NODES 256   /* tree nodes, root included                  */
#define MEDUSA_MAX_KMAX 32     /* top-k width per head                       */
#define MEDUSA_MAX_HEADS 16    /* Medusa heads = deepest possible tree level */
#define MEDUSA_MAX_BATCH 128   /* sequences per call (bf16 heads)            */

/*
 * A candidate tree.  Nodes are in breadth-first order (parents before
 * children); node 0 is the root.  The struct lives in host memory; the three
 * arrays are DEVICE arrays of n_nodes int32 each:
 *   parent[i]  parent node (parent[0] = -1, 0 <= parent[i] < i otherwise);
 *   depth[i]   depth (depth[0] = 0, depth[i] = depth[parent[i]] + 1);
 *   rank[i]    for i > 0, which entry of head depth[i]'s top-k list the node
 *              carries (0 <= rank[i] < kmax).
 * max_depth is the largest depth[i]; n_leaves the number of nodes without a
 * child.  Kernels check these relations and report violations through
 * dev_status.
 */
typedef struct medusa_tree {
  int32_t n_nodes;
  int32_t max_depth;
  int32_t n_leaves;
  const int32_t* parent;
  const int32_t* depth;
  const int32_t* rank;
} medusa_tree_t;

/* Text for a status code (static storage). */
MEDUSA_API const char* medusa_status_string(medusa_status_t status);
/* Text of the last failing call on this host thread ("" if none). */
MEDUSA_API const char* medusa_last_error(void);
/* ABI version: major*10000 + minor*100 + patch. */
MEDUSA_API int medusa_version(void);

/* ------------------------------------------------------------------------
 * medusa_heads_topk
 *
 * "Medusa Heads" glossary, "Comment les têtes prédisent les tokens
 * suivants": head k is one feed-forward layer with a SiLU activation and a
 * residual connection, followed by a projection to the vocabulary; every
 * head reads the same last hidden state.  "Attention arborescente et
 * acceptation": the heads' top choices (top-2, top-3, ...) feed the tree.
 *
 *   y_k   = h + SiLU(W1_k h + b1_k)
 *   z_k   = W2_k y_k                      (no bias)
 *   top-kmax of z_k per (sequence, head): values descending, equal values by
 *   ascending token id.
 *
 * Inputs (device, dtype dt for h/W1/b1/W2):
 *   h  [B, d]        last hidden state per sequence
 *   W1 [K, d, d]     W1[k][j][:] = weights of output feature j (Linear layout)
 *   b1 [K, d]
 *   W2 [K, V, d]     W2[k][v][:] = weights of token v
 * Outputs (device):
 *   topk_ids  [B, K, kmax] int32
 *   topk_vals [B, K, kmax] float32
 *   logits    [B, K, V] float32, or NULL to skip (parity checks).
 * Workspace: ws of at least medusa_heads_topk_workspace_size(...) bytes,
 *   256-byte aligned; contents on entry are ignored.
 * Precision: bf16 inputs, fp32 accumulation; y is fed to the vocabulary
 *   projection as the sum of two bf16 terms (hi + lo) so its rounding stays
 *   far below the fp32 accumulation error.  dt = MEDUSA_F32 runs an fp32
 *   CUDA-core path (small shapes).
 * Limits: 1 <= B <= MEDUSA_MAX_BATCH, 1 <= K <= MEDUSA_MAX_HEADS,
 *   1 <= kmax <= min(MEDUSA_MAX_KMAX, V); bf16: d % 64 == 0, all pointers
 *   16-byte aligned.
 * ---------------------------------------------------------------------- */
MEDUSA_API size_t medusa_heads_topk_workspace_size(int B, int d, int V, int K, int kmax,
                                        medusa_dtype_t dt);
MEDUSA_API medusa_status_t medusa_heads_topk(const void* h, const void* W1, const void* b1,
                                  const void* W2, medusa_dtype_t dt, int B, int d,
                                  int V, int K, int kmax, int32_t* topk_ids,
                                  float* topk_vals, float* logits, void* ws,
                                  size_t ws_bytes, int32_t* dev_status,
                                  void* stream);

/* ------------------------------------------------------------------------
 * medusa_tree_build
 *
 * "Medusa Heads" glossary, "Attention arborescente et acceptation": the
 * heads' top choices combine into candidate continuations forming a tree
 * (a Cartesian product, or a sparse selection of it); head 2 proposes the
 * same tokens under every head-1 branch; a mask lets each token see only its
 * ancestors in the tree.
 *
 *   cand_ids[b][0] = root_tok[b] (the base model's own next token);
 *   cand_ids[b][i] = topk_ids[b][depth[i]-1][rank[i]] for i > 0;
 *   pos_ids[b][i]  = prefix_len[b] + depth[i];
 *   anc_mask[i][w] bit t set iff node 32*w+t is i or an ancestor of i;
 *   retrieve[p][t] = node at depth t on the path root -> p-th leaf (leaves in
 *                    node order), -1 past the leaf.
 *
 * Inputs (device): root_tok [B] int32, topk_ids [B, K, kmax] int32,
 *   prefix_len [B] int32; tree as above (depth[i] <= K required).
 * Outputs (device): cand_ids [B, N], pos_ids [B, N] int32;
 *   anc_mask [N, ceil(N/32)] uint32; retrieve [n_leaves, max_depth+1] int32.
 * Limits: N <= MEDUSA_MAX_NODES, max_depth <= K <= MEDUSA_MAX_HEADS,
 *   kmax <= MEDUSA_MAX_KMAX.
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_tree_build(const medusa_tree_t* tree, const int32_t* root_tok,
                                  const int32_t* topk_ids, int K, int kmax,
                                  const int32_t* prefix_len, int B, int32_t* cand_ids,
                                  int32_t* pos_ids, uint32_t* anc_mask,
                                  int32_t* retrieve, int32_t* dev_status,
                                  void* stream);

/* ------------------------------------------------------------------------
 * medusa_heads_topk_tree
 *
 * medusa_heads_topk followed by medusa_tree_build of its top-k lists, in the
 * launches of medusa_heads_topk alone: the thread block that finishes the
 * last of a sequence's K lists builds that sequence's candidates (the
 * sections cited at the two calls).  Every output equals that of the two
 * calls made one after the other on the same stream, with the tree build's
 * K and kmax the heads'.
 *
 * Arguments: those of medusa_heads_topk, then those of medusa_tree_build
 *   (tree, root_tok [B], prefix_len [B]; cand_ids, pos_ids [B, N]; anc_mask
 *   [N, ceil(N/32)]; retrieve [n_leaves, max_depth+1]).  Workspace as
 *   medusa_heads_topk.
 * Host checks: medusa_heads_topk's arguments, then the tree's (as
 *   medusa_tree_build), then the workspace; nothing is launched on an error.
 * Device checks: medusa_tree_build's.
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_heads_topk_tree(
    const void* h, const void* W1, const void* b1, const void* W2, medusa_dtype_t dt, int B, int d,
    int V, int K, int kmax, int32_t* topk_ids, float* topk_vals, float* logits, void* ws,
    size_t ws_bytes, const medusa_tree_t* tree, const int32_t* root_tok, const int32_t* prefix_len,
    int32_t* cand_ids, int32_t* pos_ids, uint32_t* anc_mask, int32_t* retrieve, int32_t* dev_status,
    void* stream);

/* ------------------------------------------------------------------------
 * medusa_tree_attention
 *
 * "Medusa Heads" glossary, "Attention arborescente et acceptation": every
 * candidate token is appended to the input at once and attends only to its
 * ancestors, so one forward pass scores every branch; abstract of the Medusa
 * paper: tree-based attention verifies all candidates in one step.
 *
 * The N tree tokens' K/V are written to cache slots prefix_len[b] + i.  Query
 * (node i, head hq) then attends with weights softmax(scale * q.k) to slots
 * [0, prefix_len[b]) and to slots prefix_len[b] + j for every j set in
 * anc_mask row i.  Query head hq reads kv head hq / (Hq / Hkv).  No
 * positional rotation is applied: q and k are taken as already positioned.
 *
 * Inputs (device, dtype dt): q [B, N, Hq, dh]; k_new, v_new [B, N, Hkv, dh];
 *   caches Kc, Vc [B, Hkv, cap, dh] (read, and written at the tree slots);
 *   prefix_len [B] int32 with prefix_len[b] <= max_prefix and
 *   prefix_len[b] + N <= cap; anc_mask from medusa_tree_build.
 * Output (device): out [B, N, Hq, dh] of dtype out_dt (bf16 or f32).
 * max_prefix: host-side upper bound on every prefix_len[b]; sizes the launch.
 * Workspace: medusa_tree_attention_workspace_size(...) bytes (partial
 *   results of key ranges, merged at the end), 256-byte aligned.
 * Precision: bf16 q/k/v, fp32 scores, fp32 softmax statistics; the softmax
 *   weights (at most 2^8 relative to the running maximum) enter the value
 *   product as fp16, with V converted to fp16 in shared memory.  A V tile
 *   that fp16 cannot carry (some |v| >= 65536, or every |v| < 2^-6, where fp16
 *   would lose mantissa bits) puts its kv head's query rows on a list that an
 *   exact pass recomputes afterwards on CUDA cores in fp32, so any finite bf16
 *   V is supported; with no such tile the pass only reads an empty list.  Inf
 *   or NaN in V is reported as MEDUSA_ERR_DEVICE_CHECK.
 *   dt = MEDUSA_F32 runs an fp32 CUDA-core path.
 * Limits: Hq % Hkv == 0; bf16: dh in {64, 128}, B <= 256, pointers 16-byte
 *   aligned; f32: dh <= 256 and dh % 32 == 0; N <= MEDUSA_MAX_NODES.
 * ---------------------------------------------------------------------- */
MEDUSA_API size_t medusa_tree_attention_workspace_size(int B, int N, int Hq, int Hkv, int dh,
                                            int max_prefix, medusa_dtype_t dt);
MEDUSA_API medusa_status_t medusa_tree_attention(const void* q, const void* k_new, const void* v_new,
                                      void* Kc, void* Vc, const int32_t* prefix_len,
                                      const uint32_t* anc_mask, medusa_dtype_t dt, int B,
                                      int N, int Hq, int Hkv, int dh, int cap,
                                      int max_prefix, float scale, void* out,
                                      medusa_dtype_t out_dt, void* ws, size_t ws_bytes,
                                      int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_verify_accept
 *
 * "Medusa Heads" glossary, "Attention arborescente et acceptation": the
 * longest branch the model agrees with is kept.  Greedy: a candidate is
 * accepted when it equals the model's first choice.  Typical: a candidate is
 * kept when its probability under the base model exceeds a threshold tied to
 * the entropy of the distribution; here thr = min(eps, delta * exp(-H(p))),
 * p = softmax(logits / temperature), H in nats, strict ">".  "Medusa no
 * contexto de LLMs": on rejection the conventionally generated token is
 * used (the bonus token).
 *
 *   g[i]   = argmax_v logits[b][i][v] (lowest v among equal maxima);
 *   node c > 0 passes iff g[parent[c]] == cand_ids[b][c] (greedy) or
 *          p_parent[c](cand_ids[b][c]) > thr_parent[c] (typical);
 *   the root is accepted; c is accepted iff it passes and parent[c] is;
 *   kept node = deepest accepted node, lowest index among equally deep;
 *   accept_len[b] = its depth; accepted_nodes[b] = root..kept node, then -1;
 *   accepted_tokens[b] = kept candidates' tokens (root excluded), then the
 *   bonus token, then -1; bonus[b] = g[kept node].
 *
 * Inputs (device): logits [B, N, V] of dtype dt; cand_ids [B, N] int32; tree.
 * Outputs (device): accept_len [B], accepted_nodes [B, max_depth+1],
 *   accepted_tokens [B, max_depth+1], bonus [B], all int32.
 * Workspace: medusa_verify_accept_workspace_size(...) bytes, 256-byte aligned.
 * Limits: N <= MEDUSA_MAX_NODES; temperature > 0 (typical); eps, delta >= 0.
 * Device checks: a NaN logit, a candidate id outside [0, V).
 * ---------------------------------------------------------------------- */
MEDUSA_API size_t medusa_verify_accept_workspace_size(int B, int N, int V);
MEDUSA_API medusa_status_t medusa_verify_accept(const void* logits, medusa_dtype_t dt,
                                     const int32_t* cand_ids, const medusa_tree_t* tree,
                                     int B, int V, medusa_accept_t mode, float temperature,
                                     float eps, float delta, int32_t* accept_len,
                                     int32_t* accepted_nodes, int32_t* accepted_tokens,
                                     int32_t* bonus, void* ws, size_t ws_bytes,
                                     int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_kv_compact
 *
 * "Medusa no contexto de LLMs": an accepted candidate enters the sequence
 * without another full pass; "Medusa Heads" glossary: only the longest
 * accepted branch is kept.  The cache therefore keeps the kept branch's K/V
 * in contiguous slots after the prefix and drops the rest of the tree.
 *
 *   for j = 0..L (L = accept_len[b], P = prefix_len[b]):
 *       slot P + j of Kc and Vc (every kv head) <- slot P + accepted_nodes[b][j]
 *   (as if done for ascending j; the kernel stages the sources first, so the
 *   result is the same whichever slots overlap);
 *   compact_src[b][j] = P + accepted_nodes[b][j] for j <= L, else -1;
 *   prefix_len[b] = P + L + 1.
 *
 * In/out (device): Kc, Vc [B, Hkv, cap, dh] of dtype dt; prefix_len [B] int32.
 * Inputs (device): accepted_nodes [B, max_depth+1], accept_len [B] int32.
 * Output (device): compact_src [B, max_depth+1] int32.
 * Limits: max_depth < MEDUSA_MAX_HEADS; bf16 pointers 16-byte aligned.
 * Device checks: accept_len outside [0, max_depth], a source slot outside
 *   [P, cap).
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_kv_compact(void* Kc, void* Vc, medusa_dtype_t dt, int32_t* prefix_len,
                                  const int32_t* accepted_nodes, const int32_t* accept_len,
                                  int B, int Hkv, int dh, int cap, int max_depth,
                                  int32_t* compact_src, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_verify_accept_compact
 *
 * medusa_verify_accept followed by medusa_kv_compact of its result, in the
 * same launches as medusa_verify_accept alone: the block that picks a
 * sequence's kept branch then moves that branch's K/V (the sections cited at
 * the two calls).  Results, in every output of both calls, equal those of
 * the two calls made one after the other on the same stream.
 *
 * Arguments: those of medusa_verify_accept, then the caches Kc, Vc
 *   [B, Hkv, cap, dh] of dtype kv_dt, prefix_len [B] (in/out) and
 *   compact_src [B, max_depth+1] (out) as in medusa_kv_compact; its B and
 *   max_depth are the verification's.  Workspace as medusa_verify_accept.
 * Host checks: medusa_verify_accept's, then medusa_kv_compact's, then the
 *   workspace; nothing is launched on an error.
 * Device checks: medusa_verify_accept's; a kept slot P + node outside
 *   [0, cap).  A sequence whose tree fails the device check, or whose kept
 *   slots fail it, is not compacted and its prefix_len is unchanged.
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_verify_accept_compact(
    const void* logits, medusa_dtype_t dt, const int32_t* cand_ids, const medusa_tree_t* tree,
    int B, int V, medusa_accept_t mode, float temperature, float eps, float delta,
    int32_t* accept_len, int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus,
    void* Kc, void* Vc, medusa_dtype_t kv_dt, int32_t* prefix_len, int Hkv, int dh, int cap,
    int32_t* compact_src, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_verify_accept_noalloc
 *
 * No counterpart on the Medusa pages: a service of this library for callers
 * that cannot provide device memory per call - a host framework that reserves
 * all device memory up front and forbids allocating more at run time, or hot
 * paths that must avoid cudaMalloc/cudaFree because those calls can
 * synchronise the device.
 *
 * Same arguments, results, checks and errors as medusa_verify_accept, without
 * ws/ws_bytes: the row statistics go to a 4 MiB array compiled into the
 * library (every GPU that loads the library holds it until the process
 * exits).  Requests needing more, i.e. B * n_nodes * ceil(V / 4096) * 16 bytes
 * > 4 MiB, are rejected with MEDUSA_ERR_WORKSPACE before any launch, after
 * the argument checks medusa_verify_accept makes (so a bad tree or shape gets
 * the same error as there).  Nothing is allocated.  Every call looks up the
 * array's device address (cudaGetSymbolAddress, a host-side query) with the
 * caller's device and context current, so the address stays right after a
 * device reset or in another context; the first call on a device may load
 * the library's device code there, so make it before any stream capture.
 * All calls share the one array and it keeps the last call's contents:
 * calls whose kernels overlap on the GPU (e.g. on two streams at once) race
 * and give wrong results.
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_verify_accept_noalloc(
    const void* logits, medusa_dtype_t dt, const int32_t* cand_ids, const medusa_tree_t* tree,
    int B, int V, medusa_accept_t mode, float temperature, float eps, float delta,
    int32_t* accept_len, int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus,
    int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_lmhead_verify
 *
 * "Medusa Heads" glossary, "Attention arborescente et acceptation": one
 * forward pass scores every tree node, and the longest branch the base model
 * agrees with is kept; "Comment les têtes prédisent les tokens suivants": the
 * base model's next-token scores at a node are its lm_head applied to the
 * node's last hidden state.
 *
 * The verification of medusa_verify_accept, with the verify logits never
 * materialised: logits[b][i][v] = sum_j lm_head[v][j] * hidden[b][i][j]
 * (bf16 inputs, fp32 accumulation on the tensor cores), reduced tile by tile
 * to each node's argmax (greedy) or to its log-sum-exp and entropy
 * (typical); then exactly the acceptance rules of medusa_verify_accept.  In
 * typical mode the candidate's logit at its parent is recomputed as one dot
 * product (fp32), so near the threshold its decision may differ from one
 * taken on the GEMM's own value by the rounding of the two sums.
 *
 * Inputs (device): hidden [B, N, d] bf16 (node rows in tree order); lm_head
 *   [V, d] bf16 (torch Linear layout, no bias); cand_ids [B, N] int32; tree.
 * Outputs (device): accept_len [B], accepted_nodes [B, max_depth+1],
 *   accepted_tokens [B, max_depth+1], bonus [B] (int32, as
 *   medusa_verify_accept).  logits: optional [B, N, V] fp32 copy of the
 *   logits for checking (NULL in normal use; it adds B*N*V*4 bytes of writes).
 * dt must be MEDUSA_BF16 (MEDUSA_ERR_UNSUPPORTED otherwise).
 * Workspace: medusa_lmhead_verify_workspace_size(...) bytes, 256-byte
 *   aligned; the size depends on the current device's multiprocessor count.
 * Limits: d a positive multiple of 64; N <= MEDUSA_MAX_NODES; B * N <= 65535;
 *   hidden and lm_head 16-byte aligned; temperature > 0 (typical).
 * Device checks: a NaN logit, a candidate id outside [0, V).
 * ---------------------------------------------------------------------- */
MEDUSA_API size_t medusa_lmhead_verify_workspace_size(int B, int N, int d, int V);
MEDUSA_API medusa_status_t medusa_lmhead_verify(
    const void* hidden, const void* lm_head, medusa_dtype_t dt, const int32_t* cand_ids,
    const medusa_tree_t* tree, int B, int d, int V, medusa_accept_t mode, float temperature,
    float eps, float delta, int32_t* accept_len, int32_t* accepted_nodes,
    int32_t* accepted_tokens, int32_t* bonus, float* logits, void* ws, size_t ws_bytes,
    int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_next_step
 *
 * "Medusa Heads" glossary, "Attention arborescente et acceptation": the
 * accepted candidates join the sequence, and the heads of the next round
 * read the base model's last hidden state - that of the kept node; "Medusa
 * no contexto de LLMs": the base model's own token at the kept node (the
 * bonus token) is the next generated token, the next tree's root.
 *
 *   kept = accepted_nodes[b][accept_len[b]];
 *   h_next[b][:] = node_hidden[b][kept][:];   root_next[b] = bonus[b].
 *
 * Inputs (device): node_hidden [B, N, d] of dtype dt (the base model's last
 *   hidden states of the tree nodes); accept_len [B], accepted_nodes
 *   [B, max_depth+1], bonus [B] (int32, as written by the verification).
 * Outputs (device): h_next [B, d] of dtype dt; root_next [B] int32.
 * Limits: d * element size a multiple of 16; N <= MEDUSA_MAX_NODES;
 *   node_hidden and h_next 16-byte aligned.
 * Device checks: accept_len outside [0, max_depth] or a kept node outside
 *   [0, N) (that sequence's outputs are left unwritten).
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_next_step(const void* node_hidden, medusa_dtype_t dt,
                                            const int32_t* accept_len,
                                            const int32_t* accepted_nodes, const int32_t* bonus,
                                            int B, int N, int d, int max_depth, void* h_next,
                                            int32_t* root_next, int32_t* dev_status,
                                            void* stream);

/* ------------------------------------------------------------------------
 * Vocabulary sharding (several GPUs, each holding a slice of the vocabulary)
 *
 * No counterpart on the pages; these calls split medusa_heads_topk and
 * medusa_verify_accept at their only reduction over the vocabulary, so that
 * a caller can keep W2 rows and verify logits for tokens [v_offset,
 * v_offset + V_shard) on each GPU and exchange a few KB between them (for
 * example one all-gather and one max all-reduce).  The arithmetic of every
 * shard and of the merge runs here; the exchange is the caller's.
 *
 * A row record summarises one row of logits over a set of tokens: its
 * largest logit, the lowest token id holding it, and for typical acceptance
 * s = sum exp(z/T - maxz/T) and t = sum exp(z/T - maxz/T) * z/T.
 * ---------------------------------------------------------------------- */
typedef struct medusa_row_record {
  float maxz;
  int32_t idx;
  float s;
  float t;
} medusa_row_record_t;

/* medusa_topk_merge: the best kmax of n_lists lists of list_len candidates
 * per row (values descending, equal values by ascending id).  Candidate j of
 * list g of row r is vals/ids[r * row_stride + g * list_stride + j] (device);
 * its id gains id_offsets[g] (device int32 [n_lists], or NULL).  With the
 * per-shard outputs of medusa_heads_topk all-gathered as [G][B*K][kmax]:
 * rows = B*K, n_lists = G, list_len = kmax, row_stride = kmax, list_stride =
 * B*K*kmax, id_offsets = each shard's first token.  Outputs (device):
 * topk_ids, topk_vals [rows, kmax].  Limits: kmax <= MEDUSA_MAX_KMAX and
 * <= n_lists * list_len; rows <= 65535. */
MEDUSA_API medusa_status_t medusa_topk_merge(const float* vals, const int32_t* ids, int rows,
                                             int n_lists, int list_len, long long row_stride,
                                             long long list_stride, const int32_t* id_offsets,
                                             int kmax, int32_t* topk_ids, float* topk_vals,
                                             void* stream);

/* medusa_verify_records: this shard's row records and candidate logits.
 * Inputs (device): logits [B, N, V_shard] of dtype dt (tokens v_offset ..
 * v_offset + V_shard - 1), cand_ids [B, N] (global token ids), tree.
 * Outputs (device): records [B*N] (token ids global); cand_logit [B*N]
 * float: node c's candidate token's logit at its parent when that token is in
 * this shard, else -inf (root: -inf).  Workspace:
 * medusa_verify_records_workspace_size(B, N, V_shard) bytes, 256-aligned. */
MEDUSA_API size_t medusa_verify_records_workspace_size(int B, int N, int V_shard);
MEDUSA_API medusa_status_t medusa_verify_records(const void* logits, medusa_dtype_t dt,
                                                 const int32_t* cand_ids,
                                                 const medusa_tree_t* tree, int B, int V_shard,
                                                 int v_offset, medusa_accept_t mode,
                                                 float temperature,
                                                 medusa_row_record_t* records, float* cand_logit,
                                                 void* ws, size_t ws_bytes, int32_t* dev_status,
                                                 void* stream);

/* medusa_verify_from_records: the verification of medusa_verify_accept from
 * the G shards' records, shard-major [G][B*N] (device), and the candidate
 * logits [B*N] maximised over the shards (device; typical mode only, may be
 * NULL for greedy).  V is the full vocabulary size.  Outputs as
 * medusa_verify_accept. */
MEDUSA_API medusa_status_t medusa_verify_from_records(
    const medusa_row_record_t* records, int G, const float* cand_logit, const int32_t* cand_ids,
    const medusa_tree_t* tree, int B, int V, medusa_accept_t mode, float temperature, float eps,
    float delta, int32_t* accept_len, int32_t* accepted_nodes, int32_t* accepted_tokens,
    int32_t* bonus, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * medusa_sample_bonus
 *
 * "Medusa no contexto de LLMs", "o que significa medusa na prática de
 * deploy": the token the base model generates itself at the kept node enters
 * the sequence after the kept candidates.  medusa_verify_accept writes its
 * first choice; this call replaces it with a draw from the base model's
 * distribution there, p = softmax(logits[b][kept] / temperature):
 *
 *   x = first word of Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 *       Random Numbers: As Easy as 1, 2, 3", SC 2011) with key
 *       (seed low 32 bits, seed high 32 bits) and counter (offset low,
 *       offset high, b, 0);  u = (x >> 8) * 2^-24 in [0, 1);
 *   token = the first v whose cumulative probability exceeds u.
 *
 * Call it after medusa_verify_accept on the same logits; it overwrites
 * bonus[b] and accepted_tokens[b][accept_len[b]].  Advance offset between
 * steps for fresh draws.  The cumulative sums are fp32 (chunked scan), so a u
 * within about 1e-6 of a boundary may select the neighbouring token of an
 * fp64 inverse CDF.
 * Inputs (device): logits [B, N, V] of dtype dt; accept_len [B] and
 *   accepted_nodes [B, max_depth+1] int32 from the verification.
 * Outputs (device): bonus [B], accepted_tokens [B, max_depth+1] (one entry).
 * Limits: temperature > 0.  Device checks: a kept node outside [0, N), a
 *   row with no probability mass (NaN logits).
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_sample_bonus(const void* logits, medusa_dtype_t dt,
                                               const int32_t* accept_len,
                                               const int32_t* accepted_nodes, int B, int N,
                                               int V, int max_depth, float temperature,
                                               uint64_t seed, uint64_t offset, int32_t* bonus,
                                               int32_t* accepted_tokens, int32_t* dev_status,
                                               void* stream);

/* ------------------------------------------------------------------------
 * medusa_tree_from_accuracies   (host only: no device memory, no launch)
 *
 * "Medusa Heads" glossary, "Attention arborescente et acceptation": a sparse
 * tree built from the most accurate combinations of the heads' top choices
 * beats a dense one.
 *
 * acc [n_heads * kmax] (host, row-major): acc[t-1][r] = probability that head
 * t's rank-r token is the base model's choice, in [0, 1].  A node with rank
 * path (r1..rt) is accepted with probability prod acc[i-1][r_i] (one rank at
 * most is right, heads independent); the tree holds the root and the
 * n_nodes - 1 paths of depth <= min(n_heads, max_depth) with the largest
 * products (equal products: lexicographically smaller path first), which
 * maximises the expected accept length (the sum of the products, returned in
 * *expected_accept_len when that pointer is not NULL).  Nodes are numbered by
 * depth, then lexicographic path: parent[0] = -1, parent[i] < i.
 * Outputs (host): parent, depth, rank [n_nodes] int32 - the arrays of a
 *   medusa_tree_t once copied to the device.
 * Errors: MEDUSA_ERR_SHAPE when fewer than n_nodes - 1 paths exist or a size
 *   is out of range; MEDUSA_ERR_INVALID_ARG for an accuracy outside [0, 1].
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_tree_from_accuracies(const float* acc, int n_heads, int kmax,
                                                       int n_nodes, int max_depth,
                                                       int32_t* parent, int32_t* depth,
                                                       int32_t* rank,
                                                       double* expected_accept_len);

/* ------------------------------------------------------------------------
 * medusa_wait_flag
 *
 * No counterpart on the pages: a check of this library's failure handling.
 * Every wait inside the library's kernels (on a shared-memory barrier, or on
 * a flag another block raises) is bounded: when it runs out it writes
 * MEDUSA_ERR_TIMEOUT into *dev_status and the kernel returns, instead of
 * holding the GPU.  This call runs that same bounded flag wait (the one the
 * heads' first GEMM uses for its stream-K partials) in one thread on a
 * caller's flag: it waits until *flag == value (acquire, device scope) or
 * until budget_cycles SM clock cycles have passed, and in the second case
 * writes MEDUSA_ERR_TIMEOUT into *dev_status.  The budget is checked every
 * 64 polls of about 64 ns, so the wait lasts at least a few microseconds.
 * budget_cycles <= 0 takes the library's own bound (2e9 cycles, one to two
 * seconds).  A flag that nothing sets thus shows, on a given device and
 * driver, that a stalled wait ends with a status the host can read and
 * leaves the context usable.
 * Inputs (device): flag, 4-byte aligned.  Output (device): dev_status.
 * Errors: MEDUSA_ERR_SHAPE for budget_cycles above the library's bound.
 * ---------------------------------------------------------------------- */
MEDUSA_API medusa_status_t medusa_wait_flag(const int32_t* flag, int32_t value,
                                            long long budget_cycles, int32_t* dev_status,
                                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MEDUSA_B200_H */
