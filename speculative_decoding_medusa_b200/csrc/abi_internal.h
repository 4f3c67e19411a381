// Internal host-side interface between the C entry points (abi.cu) and the
// per-stage launchers.  Every launcher assumes its arguments were validated.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/medusa.h"
#include "kv_compact.cuh"
#include "tree_build.cuh"

namespace medusa {

// record a message for medusa_last_error() and return `code`
medusa_status_t fail(medusa_status_t code, const char* msg);
// MEDUSA_OK, or MEDUSA_ERR_CUDA with the launch error text recorded
medusa_status_t check_launch(const char* what);

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// KV compaction staging: kv heads per round and the dynamic shared memory it
// takes (false when one head's kept rows do not fit)
bool compact_plan(medusa_dtype_t dt, int dh, int Hkv, int max_depth, int* heads_per_round,
                  size_t* smem);

// the argument checks of medusa_verify_accept, all but the workspace's
medusa_status_t check_verify_accept_args(const void* logits, medusa_dtype_t dt,
                                         const int32_t* cand_ids, const medusa_tree_t* tree,
                                         int B, int V, medusa_accept_t mode, float temperature,
                                         float eps, float delta, const int32_t* accept_len,
                                         const int32_t* accepted_nodes,
                                         const int32_t* accepted_tokens, const int32_t* bonus);

// bf16 tensor of `rank` dims (dims[0] contiguous; byte_strides[i] is the
// stride of dims[i+1]), tile `box`, 128-byte swizzle, zero fill outside
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* byte_strides, const uint32_t* box);
// multiprocessors of the current device
int device_sm_count();

size_t heads_topk_workspace_size(int B, int d, int V, int K, int kmax, medusa_dtype_t dt);
medusa_status_t heads_topk(const void* h, const void* W1, const void* b1, const void* W2,
                           medusa_dtype_t dt, int B, int d, int V, int K, int kmax,
                           int32_t* topk_ids, float* topk_vals, float* logits, void* ws,
                           int32_t* status, cudaStream_t stream, const TreeOut* tree = nullptr);

medusa_status_t tree_build(const medusa_tree_t& tree, const int32_t* root_tok,
                           const int32_t* topk_ids, int K, int kmax, const int32_t* prefix_len,
                           int B, int32_t* cand_ids, int32_t* pos_ids, uint32_t* anc_mask,
                           int32_t* retrieve, int32_t* status, cudaStream_t stream);

size_t tree_attention_workspace_size(int B, int N, int Hq, int Hkv, int dh, int max_prefix,
                                     medusa_dtype_t dt);
medusa_status_t tree_attention(const void* q, const void* k_new, const void* v_new, void* Kc,
                               void* Vc, const int32_t* prefix_len, const uint32_t* anc_mask,
                               medusa_dtype_t dt, int B, int N, int Hq, int Hkv, int dh, int cap,
                               int max_prefix, float scale, void* out, medusa_dtype_t out_dt,
                               void* ws, int32_t* status, cudaStream_t stream);

// Per-(row, chunk) statistics of verify logits: the chunk's largest logit,
// its lowest index, and for typical acceptance sum exp(z/T - maxz/T) and
// sum exp(z/T - maxz/T) * z/T.
struct RowPart {
  float maxz;
  int idx;
  float s;
  float t;
};
static_assert(sizeof(RowPart) == sizeof(medusa_row_record_t), "record layout");

// Merges B*N rows of n_chunks RowParts each ([row][chunk], row = b*N + node)
// and runs the path selection.  Typical acceptance reads the candidate's
// logit as lm_head[tok] . hidden[b, parent] (bf16, d a multiple of 64).
medusa_status_t verify_path_from_parts(const RowPart* part, int n_chunks,
                                       const __nv_bfloat16* hidden,
                                       const __nv_bfloat16* lm_head, int d,
                                       const int32_t* cand_ids, const medusa_tree_t& tree, int B,
                                       int V, medusa_accept_t mode, float temperature, float eps,
                                       float delta, int32_t* accept_len,
                                       int32_t* accepted_nodes, int32_t* accepted_tokens,
                                       int32_t* bonus, int32_t* status, cudaStream_t stream);

size_t verify_accept_workspace_size(int B, int N, int V);
// ca.Kc != nullptr: the path kernel also compacts the kept branch (ca_smem
// bytes of dynamic shared memory, from compact_plan)
medusa_status_t verify_accept(const void* logits, medusa_dtype_t dt, const int32_t* cand_ids,
                              const medusa_tree_t& tree, int B, int V, medusa_accept_t mode,
                              float temperature, float eps, float delta, int32_t* accept_len,
                              int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus,
                              void* ws, int32_t* status, cudaStream_t stream,
                              const CompactArgs& ca = CompactArgs{}, size_t ca_smem = 0);

size_t lmhead_verify_workspace_size(int B, int N, int d, int V);
medusa_status_t lmhead_verify(const void* hidden, const void* lm_head, const int32_t* cand_ids,
                              const medusa_tree_t& tree, int B, int d, int V,
                              medusa_accept_t mode, float temperature, float eps, float delta,
                              int32_t* accept_len, int32_t* accepted_nodes,
                              int32_t* accepted_tokens, int32_t* bonus, float* logits, void* ws,
                              int32_t* status, cudaStream_t stream);

medusa_status_t next_step(const void* node_hidden, int elem_bytes, const int32_t* accept_len,
                          const int32_t* accepted_nodes, const int32_t* bonus, int B, int N,
                          int d, int max_depth, void* h_next, int32_t* root_next,
                          int32_t* status, cudaStream_t stream);

medusa_status_t tree_from_accuracies(const float* acc, int n_heads, int kmax, int n_nodes,
                                     int max_depth, int32_t* parent, int32_t* depth,
                                     int32_t* rank, double* expected_accept_len);

medusa_status_t sample_bonus(const void* logits, medusa_dtype_t dt, const int32_t* accept_len,
                             const int32_t* accepted_nodes, int B, int N, int V, int max_depth,
                             float temperature, uint64_t seed, uint64_t offset, int32_t* bonus,
                             int32_t* accepted_tokens, int32_t* status, cudaStream_t stream);

// best kmax of n_lists lists of list_len (value, id) candidates per row;
// entry (r, g, j) at r * row_stride + g * list_stride + j; ids of list g
// gain id_offsets[g] (NULL: none)
medusa_status_t topk_merge_lists(const float* vals, const int32_t* ids, int rows, int n_lists,
                                 int list_len, long long row_stride, long long list_stride,
                                 const int32_t* id_offsets, int kmax, int32_t* out_ids,
                                 float* out_vals, cudaStream_t stream);

size_t verify_records_workspace_size(int B, int N, int V_shard);
medusa_status_t verify_records(const void* logits, medusa_dtype_t dt, const int32_t* cand_ids,
                               const medusa_tree_t& tree, int B, int V_shard, int v_offset,
                               medusa_accept_t mode, float temperature, RowPart* records,
                               float* cand_logit, void* ws, int32_t* status, cudaStream_t stream);
medusa_status_t verify_from_records(const RowPart* records, int G, const float* cand_logit,
                                    const int32_t* cand_ids, const medusa_tree_t& tree, int B,
                                    int V, medusa_accept_t mode, float temperature, float eps,
                                    float delta, int32_t* accept_len, int32_t* accepted_nodes,
                                    int32_t* accepted_tokens, int32_t* bonus, int32_t* status,
                                    cudaStream_t stream);

medusa_status_t kv_compact(void* Kc, void* Vc, medusa_dtype_t dt, int32_t* prefix_len,
                           const int32_t* accepted_nodes, const int32_t* accept_len, int B,
                           int Hkv, int dh, int cap, int max_depth, int32_t* compact_src,
                           int32_t* status, cudaStream_t stream);

}  // namespace medusa
