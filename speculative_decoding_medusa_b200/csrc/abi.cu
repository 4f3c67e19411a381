// The C entry points: argument checks, then the per-stage launchers.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "abi_internal.h"

namespace medusa {

static thread_local char g_last_error[512] = "";

medusa_status_t fail(medusa_status_t code, const char* msg) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return code;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("MEDUSA_PDL");
    return v == nullptr || strcmp(v, "0") != 0;
  }();
  return on;
}

medusa_status_t check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MEDUSA_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
  return MEDUSA_ERR_CUDA;
}

}  // namespace medusa

using medusa::fail;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
bool valid_dtype(medusa_dtype_t d) { return d == MEDUSA_BF16 || d == MEDUSA_F32; }

medusa_status_t check_tree(const medusa_tree_t* t) {
  if (t == nullptr || t->parent == nullptr || t->depth == nullptr || t->rank == nullptr)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree: null pointer");
  if (t->n_nodes < 1 || t->n_nodes > MEDUSA_MAX_NODES)
    return fail(MEDUSA_ERR_SHAPE, "tree: n_nodes must be in [1, 256]");
  if (t->max_depth < 0 || t->max_depth >= t->n_nodes || t->max_depth > MEDUSA_MAX_HEADS)
    return fail(MEDUSA_ERR_SHAPE, "tree: max_depth out of range");
  if (t->n_leaves < 1 || t->n_leaves > t->n_nodes)
    return fail(MEDUSA_ERR_SHAPE, "tree: n_leaves out of range");
  return MEDUSA_OK;
}

}  // namespace

extern "C" {

const char* medusa_status_string(medusa_status_t s) {
  switch (s) {
    case MEDUSA_OK: return "ok";
    case MEDUSA_ERR_INVALID_ARG: return "invalid argument";
    case MEDUSA_ERR_SHAPE: return "unsupported shape";
    case MEDUSA_ERR_UNSUPPORTED: return "unsupported";
    case MEDUSA_ERR_CUDA: return "CUDA error";
    case MEDUSA_ERR_TIMEOUT: return "device wait timed out";
    case MEDUSA_ERR_DEVICE_CHECK: return "device-side check failed";
    case MEDUSA_ERR_WORKSPACE: return "workspace missing or too small";
    case MEDUSA_ERR_ALIGNMENT: return "misaligned pointer";
  }
  return "unknown status";
}

const char* medusa_last_error(void) { return medusa::g_last_error; }

int medusa_version(void) { return 10000; }

size_t medusa_heads_topk_workspace_size(int B, int d, int V, int K, int kmax, medusa_dtype_t dt) {
  if (B < 1 || d < 1 || V < 1 || K < 1 || kmax < 1 || !valid_dtype(dt)) return 0;
  return medusa::heads_topk_workspace_size(B, d, V, K, kmax, dt);
}

namespace {

medusa_status_t check_heads_args(const void* h, const void* W1, const void* b1, const void* W2,
                                 medusa_dtype_t dt, int B, int d, int V, int K, int kmax,
                                 int32_t* topk_ids, float* topk_vals) {
  if (!h || !W1 || !b1 || !W2 || !topk_ids || !topk_vals)
    return fail(MEDUSA_ERR_INVALID_ARG, "heads_topk: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "heads_topk: bad dtype");
  if (B < 1 || B > MEDUSA_MAX_BATCH || d < 1 || V < 1 || K < 1 || K > MEDUSA_MAX_HEADS)
    return fail(MEDUSA_ERR_SHAPE, "heads_topk: B, d, V or K out of range");
  if (kmax < 1 || kmax > MEDUSA_MAX_KMAX || kmax > V)
    return fail(MEDUSA_ERR_SHAPE, "heads_topk: kmax must be in [1, min(32, V)]");
  if ((long long)B * K > 65535 || (long long)V * K > (1LL << 31) / 2)
    return fail(MEDUSA_ERR_SHAPE, "heads_topk: B*K or K*V too large");
  if (dt == MEDUSA_BF16) {
    if (d % 64 != 0) return fail(MEDUSA_ERR_SHAPE, "heads_topk: bf16 needs d % 64 == 0");
    if (!aligned16(h) || !aligned16(W1) || !aligned16(b1) || !aligned16(W2))
      return fail(MEDUSA_ERR_ALIGNMENT, "heads_topk: inputs must be 16-byte aligned");
  }
  return MEDUSA_OK;
}

medusa_status_t check_heads_ws(int B, int d, int V, int K, int kmax, medusa_dtype_t dt,
                               const void* ws, size_t ws_bytes) {
  const size_t need = medusa::heads_topk_workspace_size(B, d, V, K, kmax, dt);
  if (ws == nullptr || ws_bytes < need || !aligned256(ws))
    return fail(MEDUSA_ERR_WORKSPACE, "heads_topk: workspace null, misaligned or too small");
  return MEDUSA_OK;
}

}  // namespace

medusa_status_t medusa_heads_topk(const void* h, const void* W1, const void* b1, const void* W2,
                                  medusa_dtype_t dt, int B, int d, int V, int K, int kmax,
                                  int32_t* topk_ids, float* topk_vals, float* logits, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream) {
  medusa_status_t st = check_heads_args(h, W1, b1, W2, dt, B, d, V, K, kmax, topk_ids, topk_vals);
  if (st != MEDUSA_OK) return st;
  st = check_heads_ws(B, d, V, K, kmax, dt, ws, ws_bytes);
  if (st != MEDUSA_OK) return st;
  return medusa::heads_topk(h, W1, b1, W2, dt, B, d, V, K, kmax, topk_ids, topk_vals, logits, ws,
                            dev_status, static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_heads_topk_tree(const void* h, const void* W1, const void* b1,
                                       const void* W2, medusa_dtype_t dt, int B, int d, int V,
                                       int K, int kmax, int32_t* topk_ids, float* topk_vals,
                                       float* logits, void* ws, size_t ws_bytes,
                                       const medusa_tree_t* tree, const int32_t* root_tok,
                                       const int32_t* prefix_len, int32_t* cand_ids,
                                       int32_t* pos_ids, uint32_t* anc_mask, int32_t* retrieve,
                                       int32_t* dev_status, void* stream) {
  medusa_status_t st = check_heads_args(h, W1, b1, W2, dt, B, d, V, K, kmax, topk_ids, topk_vals);
  if (st != MEDUSA_OK) return st;
  // the checks of medusa_tree_build
  st = check_tree(tree);
  if (st != MEDUSA_OK) return st;
  if (!root_tok || !prefix_len || !cand_ids || !pos_ids || !anc_mask || !retrieve)
    return fail(MEDUSA_ERR_INVALID_ARG, "heads_topk_tree: null pointer");
  if (tree->max_depth > K)
    return fail(MEDUSA_ERR_SHAPE, "heads_topk_tree: tree deeper than K heads");
  st = check_heads_ws(B, d, V, K, kmax, dt, ws, ws_bytes);
  if (st != MEDUSA_OK) return st;
  const medusa::TreeOut t{tree->parent, tree->depth, tree->rank, tree->n_nodes, tree->max_depth,
                          tree->n_leaves, K, kmax, root_tok, prefix_len, cand_ids, pos_ids,
                          anc_mask, retrieve, dev_status};
  return medusa::heads_topk(h, W1, b1, W2, dt, B, d, V, K, kmax, topk_ids, topk_vals, logits, ws,
                            dev_status, static_cast<cudaStream_t>(stream), &t);
}

medusa_status_t medusa_tree_build(const medusa_tree_t* tree, const int32_t* root_tok,
                                  const int32_t* topk_ids, int K, int kmax,
                                  const int32_t* prefix_len, int B, int32_t* cand_ids,
                                  int32_t* pos_ids, uint32_t* anc_mask, int32_t* retrieve,
                                  int32_t* dev_status, void* stream) {
  medusa_status_t st = check_tree(tree);
  if (st != MEDUSA_OK) return st;
  if (!root_tok || !topk_ids || !prefix_len || !cand_ids || !pos_ids || !anc_mask || !retrieve)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree_build: null pointer");
  if (B < 1 || B > 65535 || K < 1 || K > MEDUSA_MAX_HEADS || kmax < 1 || kmax > MEDUSA_MAX_KMAX)
    return fail(MEDUSA_ERR_SHAPE, "tree_build: B, K or kmax out of range");
  if (tree->max_depth > K) return fail(MEDUSA_ERR_SHAPE, "tree_build: tree deeper than K heads");
  return medusa::tree_build(*tree, root_tok, topk_ids, K, kmax, prefix_len, B, cand_ids, pos_ids,
                            anc_mask, retrieve, dev_status, static_cast<cudaStream_t>(stream));
}

size_t medusa_tree_attention_workspace_size(int B, int N, int Hq, int Hkv, int dh, int max_prefix,
                                            medusa_dtype_t dt) {
  if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || dh < 1 || max_prefix < 0 || !valid_dtype(dt))
    return 0;
  return medusa::tree_attention_workspace_size(B, N, Hq, Hkv, dh, max_prefix, dt);
}

medusa_status_t medusa_tree_attention(const void* q, const void* k_new, const void* v_new,
                                      void* Kc, void* Vc, const int32_t* prefix_len,
                                      const uint32_t* anc_mask, medusa_dtype_t dt, int B, int N,
                                      int Hq, int Hkv, int dh, int cap, int max_prefix, float scale,
                                      void* out, medusa_dtype_t out_dt, void* ws, size_t ws_bytes,
                                      int32_t* dev_status, void* stream) {
  if (!q || !k_new || !v_new || !Kc || !Vc || !prefix_len || !anc_mask || !out)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention: null pointer");
  if (!valid_dtype(dt) || !valid_dtype(out_dt))
    return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention: bad dtype");
  if (B < 1 || N < 1 || N > MEDUSA_MAX_NODES || Hq < 1 || Hkv < 1 || Hq % Hkv != 0)
    return fail(MEDUSA_ERR_SHAPE, "tree_attention: B, N, Hq or Hkv out of range");
  if (max_prefix < 0 || cap < N || max_prefix + N > cap)
    return fail(MEDUSA_ERR_SHAPE, "tree_attention: need 0 <= max_prefix and max_prefix + N <= cap");
  if ((long long)B * Hkv > 65535 || (long long)B * Hkv * cap * dh > (1LL << 40))
    return fail(MEDUSA_ERR_SHAPE, "tree_attention: cache too large");
  if (dt == MEDUSA_BF16) {
    if (dh != 64 && dh != 128) return fail(MEDUSA_ERR_SHAPE, "tree_attention: bf16 dh must be 64 or 128");
    if (B > 256) return fail(MEDUSA_ERR_SHAPE, "tree_attention: bf16 path takes at most 256 sequences");
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(Kc) ||
        !aligned16(Vc) || !aligned16(out))
      return fail(MEDUSA_ERR_ALIGNMENT, "tree_attention: pointers must be 16-byte aligned");
    const size_t need = medusa::tree_attention_workspace_size(B, N, Hq, Hkv, dh, max_prefix, dt);
    if (ws == nullptr || ws_bytes < need || !aligned256(ws))
      return fail(MEDUSA_ERR_WORKSPACE, "tree_attention: workspace null, misaligned or too small");
  } else {
    if (dh % 32 != 0 || dh > 256)
      return fail(MEDUSA_ERR_SHAPE, "tree_attention: f32 dh must be a multiple of 32, <= 256");
  }
  if (!(scale > 0.f)) return fail(MEDUSA_ERR_INVALID_ARG, "tree_attention: scale must be > 0");
  return medusa::tree_attention(q, k_new, v_new, Kc, Vc, prefix_len, anc_mask, dt, B, N, Hq, Hkv,
                                dh, cap, max_prefix, scale, out, out_dt, ws, dev_status,
                                static_cast<cudaStream_t>(stream));
}

size_t medusa_verify_accept_workspace_size(int B, int N, int V) {
  if (B < 1 || N < 1 || V < 1) return 0;
  return medusa::verify_accept_workspace_size(B, N, V);
}

}  // extern "C"

// Every check of medusa_verify_accept except the workspace's (shared with
// medusa_verify_accept_noalloc, whose scratch limit is checked after these).
medusa_status_t medusa::check_verify_accept_args(const void* logits, medusa_dtype_t dt,
                                                 const int32_t* cand_ids,
                                                 const medusa_tree_t* tree, int B, int V,
                                                 medusa_accept_t mode, float temperature,
                                                 float eps, float delta, const int32_t* accept_len,
                                                 const int32_t* accepted_nodes,
                                                 const int32_t* accepted_tokens,
                                                 const int32_t* bonus) {
  medusa_status_t st = check_tree(tree);
  if (st != MEDUSA_OK) return st;
  if (!logits || !cand_ids || !accept_len || !accepted_nodes || !accepted_tokens || !bonus)
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_accept: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "verify_accept: bad dtype");
  if (mode != MEDUSA_ACCEPT_GREEDY && mode != MEDUSA_ACCEPT_TYPICAL)
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_accept: bad mode");
  if (B < 1 || V < 1 || (long long)B * tree->n_nodes > 65535)
    return fail(MEDUSA_ERR_SHAPE, "verify_accept: B, V out of range");
  if (mode == MEDUSA_ACCEPT_TYPICAL && (!(temperature > 0.f) || !(eps >= 0.f) || !(delta >= 0.f)))
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_accept: need temperature > 0, eps >= 0, delta >= 0");
  if (!aligned16(logits)) return fail(MEDUSA_ERR_ALIGNMENT, "verify_accept: logits not 16-byte aligned");
  return MEDUSA_OK;
}

extern "C" {

medusa_status_t medusa_verify_accept(const void* logits, medusa_dtype_t dt,
                                     const int32_t* cand_ids, const medusa_tree_t* tree, int B,
                                     int V, medusa_accept_t mode, float temperature, float eps,
                                     float delta, int32_t* accept_len, int32_t* accepted_nodes,
                                     int32_t* accepted_tokens, int32_t* bonus, void* ws,
                                     size_t ws_bytes, int32_t* dev_status, void* stream) {
  medusa_status_t st = medusa::check_verify_accept_args(logits, dt, cand_ids, tree, B, V, mode,
                                                        temperature, eps, delta, accept_len,
                                                        accepted_nodes, accepted_tokens, bonus);
  if (st != MEDUSA_OK) return st;
  const size_t need = medusa::verify_accept_workspace_size(B, tree->n_nodes, V);
  if (ws == nullptr || ws_bytes < need || !aligned256(ws))
    return fail(MEDUSA_ERR_WORKSPACE, "verify_accept: workspace null, misaligned or too small");
  return medusa::verify_accept(logits, dt, cand_ids, *tree, B, V, mode, temperature, eps, delta,
                               accept_len, accepted_nodes, accepted_tokens, bonus, ws, dev_status,
                               static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_verify_accept_compact(
    const void* logits, medusa_dtype_t dt, const int32_t* cand_ids, const medusa_tree_t* tree,
    int B, int V, medusa_accept_t mode, float temperature, float eps, float delta,
    int32_t* accept_len, int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus,
    void* Kc, void* Vc, medusa_dtype_t kv_dt, int32_t* prefix_len, int Hkv, int dh, int cap,
    int32_t* compact_src, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  medusa_status_t st = medusa::check_verify_accept_args(logits, dt, cand_ids, tree, B, V, mode,
                                                        temperature, eps, delta, accept_len,
                                                        accepted_nodes, accepted_tokens, bonus);
  if (st != MEDUSA_OK) return st;
  // the checks of medusa_kv_compact
  if (!Kc || !Vc || !prefix_len || !compact_src)
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_accept_compact: null pointer");
  if (!valid_dtype(kv_dt)) return fail(MEDUSA_ERR_INVALID_ARG, "verify_accept_compact: bad dtype");
  if (Hkv < 1 || dh < 1 || cap < 1 || tree->max_depth >= MEDUSA_MAX_HEADS)
    return fail(MEDUSA_ERR_SHAPE, "verify_accept_compact: Hkv, dh, cap or max_depth out of range");
  const int row_bytes = dh * (kv_dt == MEDUSA_BF16 ? 2 : 4);
  if (row_bytes % 16 != 0)
    return fail(MEDUSA_ERR_SHAPE, "verify_accept_compact: a cache row must be a multiple of 16 bytes");
  if (!aligned16(Kc) || !aligned16(Vc))
    return fail(MEDUSA_ERR_ALIGNMENT, "verify_accept_compact: caches not 16-byte aligned");
  int heads_per_round = 0;
  size_t smem = 0;
  if (!medusa::compact_plan(kv_dt, dh, Hkv, tree->max_depth, &heads_per_round, &smem))
    return fail(MEDUSA_ERR_UNSUPPORTED, "verify_accept_compact: (max_depth+1) * row too large");
  const size_t need = medusa::verify_accept_workspace_size(B, tree->n_nodes, V);
  if (ws == nullptr || ws_bytes < need || !aligned256(ws))
    return fail(MEDUSA_ERR_WORKSPACE, "verify_accept_compact: workspace null, misaligned or too small");
  const medusa::CompactArgs ca{static_cast<uint8_t*>(Kc), static_cast<uint8_t*>(Vc), row_bytes,
                               prefix_len, Hkv, cap, heads_per_round, compact_src};
  return medusa::verify_accept(logits, dt, cand_ids, *tree, B, V, mode, temperature, eps, delta,
                               accept_len, accepted_nodes, accepted_tokens, bonus, ws, dev_status,
                               static_cast<cudaStream_t>(stream), ca, smem);
}

size_t medusa_lmhead_verify_workspace_size(int B, int N, int d, int V) {
  if (B < 1 || N < 1 || d < 1 || V < 1 || (long long)B * N > 65535) return 0;
  return medusa::lmhead_verify_workspace_size(B, N, d, V);
}

medusa_status_t medusa_lmhead_verify(const void* hidden, const void* lm_head, medusa_dtype_t dt,
                                     const int32_t* cand_ids, const medusa_tree_t* tree, int B,
                                     int d, int V, medusa_accept_t mode, float temperature,
                                     float eps, float delta, int32_t* accept_len,
                                     int32_t* accepted_nodes, int32_t* accepted_tokens,
                                     int32_t* bonus, float* logits, void* ws, size_t ws_bytes,
                                     int32_t* dev_status, void* stream) {
  medusa_status_t st = check_tree(tree);
  if (st != MEDUSA_OK) return st;
  if (!hidden || !lm_head || !cand_ids || !accept_len || !accepted_nodes || !accepted_tokens ||
      !bonus)
    return fail(MEDUSA_ERR_INVALID_ARG, "lmhead_verify: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "lmhead_verify: bad dtype");
  if (dt != MEDUSA_BF16) return fail(MEDUSA_ERR_UNSUPPORTED, "lmhead_verify: bf16 only");
  if (mode != MEDUSA_ACCEPT_GREEDY && mode != MEDUSA_ACCEPT_TYPICAL)
    return fail(MEDUSA_ERR_INVALID_ARG, "lmhead_verify: bad mode");
  if (B < 1 || V < 1 || d < 64 || d % 64 != 0 || (long long)B * tree->n_nodes > 65535 ||
      (long long)V * d > (1LL << 40))
    return fail(MEDUSA_ERR_SHAPE, "lmhead_verify: need d a multiple of 64, B*N <= 65535");
  if (mode == MEDUSA_ACCEPT_TYPICAL && (!(temperature > 0.f) || !(eps >= 0.f) || !(delta >= 0.f)))
    return fail(MEDUSA_ERR_INVALID_ARG, "lmhead_verify: need temperature > 0, eps >= 0, delta >= 0");
  if (!aligned16(hidden) || !aligned16(lm_head) ||
      (logits != nullptr && reinterpret_cast<uintptr_t>(logits) % 4 != 0))
    return fail(MEDUSA_ERR_ALIGNMENT, "lmhead_verify: hidden/lm_head not 16-byte aligned");
  const size_t need = medusa::lmhead_verify_workspace_size(B, tree->n_nodes, d, V);
  if (ws == nullptr || ws_bytes < need || !aligned256(ws))
    return fail(MEDUSA_ERR_WORKSPACE, "lmhead_verify: workspace null, misaligned or too small");
  return medusa::lmhead_verify(hidden, lm_head, cand_ids, *tree, B, d, V, mode, temperature, eps,
                               delta, accept_len, accepted_nodes, accepted_tokens, bonus, logits,
                               ws, dev_status, static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_next_step(const void* node_hidden, medusa_dtype_t dt,
                                 const int32_t* accept_len, const int32_t* accepted_nodes,
                                 const int32_t* bonus, int B, int N, int d, int max_depth,
                                 void* h_next, int32_t* root_next, int32_t* dev_status,
                                 void* stream) {
  if (!node_hidden || !accept_len || !accepted_nodes || !bonus || !h_next || !root_next)
    return fail(MEDUSA_ERR_INVALID_ARG, "next_step: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "next_step: bad dtype");
  if (B < 1 || B > 65535 || N < 1 || N > MEDUSA_MAX_NODES || d < 1 || max_depth < 0 ||
      max_depth >= MEDUSA_MAX_HEADS)
    return fail(MEDUSA_ERR_SHAPE, "next_step: B, N, d or max_depth out of range");
  const int eb = dt == MEDUSA_BF16 ? 2 : 4;
  if ((d * eb) % 16 != 0) return fail(MEDUSA_ERR_SHAPE, "next_step: d * element size % 16 != 0");
  if (!aligned16(node_hidden) || !aligned16(h_next))
    return fail(MEDUSA_ERR_ALIGNMENT, "next_step: hidden buffers must be 16-byte aligned");
  return medusa::next_step(node_hidden, eb, accept_len, accepted_nodes, bonus, B, N, d, max_depth,
                           h_next, root_next, dev_status, static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_tree_from_accuracies(const float* acc, int n_heads, int kmax,
                                            int n_nodes, int max_depth, int32_t* parent,
                                            int32_t* depth, int32_t* rank,
                                            double* expected_accept_len) {
  if (!acc || !parent || !depth || !rank)
    return fail(MEDUSA_ERR_INVALID_ARG, "tree_from_accuracies: null pointer");
  if (n_heads < 1 || n_heads > MEDUSA_MAX_HEADS || kmax < 1 || kmax > MEDUSA_MAX_KMAX ||
      n_nodes < 1 || n_nodes > MEDUSA_MAX_NODES || max_depth < 1)
    return fail(MEDUSA_ERR_SHAPE, "tree_from_accuracies: sizes out of range");
  for (int i = 0; i < n_heads * kmax; ++i)
    if (!(acc[i] >= 0.f && acc[i] <= 1.f))
      return fail(MEDUSA_ERR_INVALID_ARG, "tree_from_accuracies: accuracies must be in [0, 1]");
  return medusa::tree_from_accuracies(acc, n_heads, kmax, n_nodes, max_depth, parent, depth, rank,
                                      expected_accept_len);
}

medusa_status_t medusa_sample_bonus(const void* logits, medusa_dtype_t dt,
                                    const int32_t* accept_len, const int32_t* accepted_nodes,
                                    int B, int N, int V, int max_depth, float temperature,
                                    uint64_t seed, uint64_t offset, int32_t* bonus,
                                    int32_t* accepted_tokens, int32_t* dev_status, void* stream) {
  if (!logits || !accept_len || !accepted_nodes || !bonus || !accepted_tokens)
    return fail(MEDUSA_ERR_INVALID_ARG, "sample_bonus: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "sample_bonus: bad dtype");
  if (B < 1 || B > 65535 || N < 1 || N > MEDUSA_MAX_NODES || V < 1 || max_depth < 0 ||
      max_depth >= MEDUSA_MAX_HEADS)
    return fail(MEDUSA_ERR_SHAPE, "sample_bonus: B, N, V or max_depth out of range");
  if (!(temperature > 0.f))
    return fail(MEDUSA_ERR_INVALID_ARG, "sample_bonus: temperature must be > 0");
  return medusa::sample_bonus(logits, dt, accept_len, accepted_nodes, B, N, V, max_depth,
                              temperature, seed, offset, bonus, accepted_tokens, dev_status,
                              static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_topk_merge(const float* vals, const int32_t* ids, int rows, int n_lists,
                                  int list_len, long long row_stride, long long list_stride,
                                  const int32_t* id_offsets, int kmax, int32_t* topk_ids,
                                  float* topk_vals, void* stream) {
  if (!vals || !ids || !topk_ids || !topk_vals)
    return fail(MEDUSA_ERR_INVALID_ARG, "topk_merge: null pointer");
  if (rows < 1 || rows > 65535 || n_lists < 1 || list_len < 1 || kmax < 1 ||
      kmax > MEDUSA_MAX_KMAX || (long long)n_lists * list_len < kmax || row_stride < 0 ||
      list_stride < 0)
    return fail(MEDUSA_ERR_SHAPE, "topk_merge: sizes out of range");
  return medusa::topk_merge_lists(vals, ids, rows, n_lists, list_len, row_stride, list_stride,
                                  id_offsets, kmax, topk_ids, topk_vals,
                                  static_cast<cudaStream_t>(stream));
}

size_t medusa_verify_records_workspace_size(int B, int N, int V_shard) {
  if (B < 1 || N < 1 || V_shard < 1) return 0;
  return medusa::verify_records_workspace_size(B, N, V_shard);
}

medusa_status_t medusa_verify_records(const void* logits, medusa_dtype_t dt,
                                      const int32_t* cand_ids, const medusa_tree_t* tree, int B,
                                      int V_shard, int v_offset, medusa_accept_t mode,
                                      float temperature, medusa_row_record_t* records,
                                      float* cand_logit, void* ws, size_t ws_bytes,
                                      int32_t* dev_status, void* stream) {
  medusa_status_t st = check_tree(tree);
  if (st != MEDUSA_OK) return st;
  if (!logits || !cand_ids || !records || !cand_logit)
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_records: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "verify_records: bad dtype");
  if (mode != MEDUSA_ACCEPT_GREEDY && mode != MEDUSA_ACCEPT_TYPICAL)
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_records: bad mode");
  if (B < 1 || V_shard < 1 || v_offset < 0 || (long long)B * tree->n_nodes > 65535)
    return fail(MEDUSA_ERR_SHAPE, "verify_records: B, V_shard or v_offset out of range");
  if (mode == MEDUSA_ACCEPT_TYPICAL && !(temperature > 0.f))
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_records: temperature must be > 0");
  if (!aligned16(logits)) return fail(MEDUSA_ERR_ALIGNMENT, "verify_records: logits not 16-byte aligned");
  const size_t need = medusa::verify_records_workspace_size(B, tree->n_nodes, V_shard);
  if (ws == nullptr || ws_bytes < need || !aligned256(ws))
    return fail(MEDUSA_ERR_WORKSPACE, "verify_records: workspace null, misaligned or too small");
  return medusa::verify_records(logits, dt, cand_ids, *tree, B, V_shard, v_offset, mode,
                                temperature, reinterpret_cast<medusa::RowPart*>(records),
                                cand_logit, ws, dev_status, static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_verify_from_records(const medusa_row_record_t* records, int G,
                                           const float* cand_logit, const int32_t* cand_ids,
                                           const medusa_tree_t* tree, int B, int V,
                                           medusa_accept_t mode, float temperature, float eps,
                                           float delta, int32_t* accept_len,
                                           int32_t* accepted_nodes, int32_t* accepted_tokens,
                                           int32_t* bonus, int32_t* dev_status, void* stream) {
  medusa_status_t st = check_tree(tree);
  if (st != MEDUSA_OK) return st;
  if (!records || !cand_ids || !accept_len || !accepted_nodes || !accepted_tokens || !bonus ||
      (mode == MEDUSA_ACCEPT_TYPICAL && !cand_logit))
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_from_records: null pointer");
  if (mode != MEDUSA_ACCEPT_GREEDY && mode != MEDUSA_ACCEPT_TYPICAL)
    return fail(MEDUSA_ERR_INVALID_ARG, "verify_from_records: bad mode");
  if (B < 1 || V < 1 || G < 1 || G > 4096 || (long long)B * tree->n_nodes > 65535)
    return fail(MEDUSA_ERR_SHAPE, "verify_from_records: B, V or G out of range");
  if (mode == MEDUSA_ACCEPT_TYPICAL && (!(temperature > 0.f) || !(eps >= 0.f) || !(delta >= 0.f)))
    return fail(MEDUSA_ERR_INVALID_ARG,
                "verify_from_records: need temperature > 0, eps >= 0, delta >= 0");
  return medusa::verify_from_records(reinterpret_cast<const medusa::RowPart*>(records), G,
                                     cand_logit, cand_ids, *tree, B, V, mode, temperature, eps,
                                     delta, accept_len, accepted_nodes, accepted_tokens, bonus,
                                     dev_status, static_cast<cudaStream_t>(stream));
}

medusa_status_t medusa_kv_compact(void* Kc, void* Vc, medusa_dtype_t dt, int32_t* prefix_len,
                                  const int32_t* accepted_nodes, const int32_t* accept_len, int B,
                                  int Hkv, int dh, int cap, int max_depth, int32_t* compact_src,
                                  int32_t* dev_status, void* stream) {
  if (!Kc || !Vc || !prefix_len || !accepted_nodes || !accept_len || !compact_src)
    return fail(MEDUSA_ERR_INVALID_ARG, "kv_compact: null pointer");
  if (!valid_dtype(dt)) return fail(MEDUSA_ERR_INVALID_ARG, "kv_compact: bad dtype");
  if (B < 1 || B > 65535 || Hkv < 1 || dh < 1 || cap < 1 || max_depth < 0 ||
      max_depth >= MEDUSA_MAX_HEADS)
    return fail(MEDUSA_ERR_SHAPE, "kv_compact: B, Hkv, dh, cap or max_depth out of range");
  const int row_bytes = dh * (dt == MEDUSA_BF16 ? 2 : 4);
  if (row_bytes % 16 != 0) return fail(MEDUSA_ERR_SHAPE, "kv_compact: dh * element size % 16 != 0");
  if (!aligned16(Kc) || !aligned16(Vc))
    return fail(MEDUSA_ERR_ALIGNMENT, "kv_compact: caches must be 16-byte aligned");
  return medusa::kv_compact(Kc, Vc, dt, prefix_len, accepted_nodes, accept_len, B, Hkv, dh, cap,
                            max_depth, compact_src, dev_status, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
