// sv_internal.h -- parameter blocks and launchers shared by the libsv sources.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sv.h"

namespace sv {

// Zero-filled scratch owned by the caller (see sv.h).  The same layout serves
// every entry point, so one workspace can be shared by calls in sequence.
struct Workspace {
  uint32_t* req_counter;   // [B]   rows of a request that have finished
  uint32_t* req_reject;    // [B]   max over rejected rows of (k - i); 0 = none yet
  uint32_t* glob_counter;  // [1]   requests that have finished
  uint32_t* work;          // [1]   next row item to hand out (persistent kernels)
  uint32_t* done;          // [1]   clusters that have run out of items
  int32_t* row_a;          // [B*R] per-row result code (0 = not yet written)
  int32_t* row_b;          // [B*R] per-row value + 1 (sampled token / argmax; 0 = none)
};

size_t workspace_bytes(int B, int rows_per_request);
Workspace workspace_carve(void* base, int B, int rows_per_request);

// Shared-memory layout of a row kernel: fixed block, then the staged chunk(s),
// then a scratch region.
struct RowLayout {
  int off_t;   // target/row chunk
  int off_d;   // draft chunk (pair kernels)
  int off_x;   // scratch (per-piece weight sums, scan values, top-K candidates)
  int bytes;   // total dynamic shared memory
};

struct RowPlan {
  int C;         // CTAs per cluster (chunks per row)
  int L;         // elements per chunk, multiple of 8
  int npieces;   // pieces of the longest chunk
  int use_bulk;  // 1: bulk copies (16-byte aligned rows); 0: scalar staging
  RowLayout lay;
};

struct ChainParams {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const float* u;
  int B, k, V, L;
  float c;  // log2(e) / T
  int use_bulk;
  RowLayout lay;
  int32_t* accepted_len;
  int32_t* out_tokens;
  // fused KD (K == 0: off)
  int K;
  float* topk_logp;
  int32_t* topk_idx;
  float* lse;
  float* kl;
  const float* reward;
  int wmode, group;
  float clip;
  float* loss;
  float* total;
  Workspace ws;
  int32_t* status;
};

struct ArgmaxParams {
  const void* logits;
  const int32_t* tokens;   // chain: draft tokens [B,k]; tree: node tokens [B,n]
  const int32_t* parents;  // tree only
  int B, R, V, L;          // R rows per request (chain: k+1, tree: n)
  int max_depth;           // tree only
  int use_bulk;
  RowLayout lay;
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* accepted_nodes;  // tree only
  Workspace ws;
  int32_t* status;
};

struct TopkParams {
  const void* logits;
  int rows, V, L, K;
  float c;
  int use_bulk;
  RowLayout lay;
  float* topk_logp;
  int32_t* topk_idx;
  float* lse;
  int32_t* status;
};

struct KlParams {
  const float* topk_logp;
  const int32_t* topk_idx;
  const void* draft;
  int B, k, K, V, L;
  float c;
  int use_bulk;
  RowLayout lay;
  const int32_t* accepted_len;
  const float* reward;
  int wmode, group;
  float clip;
  float* kl;
  float* loss;
  float* total;
  Workspace ws;
  int32_t* status;
};

// dtype codes: 0 = fp32, 1 = bf16; draft kind: 0 = logits, 1 = probs.
cudaError_t launch_chain_sample(const ChainParams& p, const RowPlan& plan, int t_dtype,
                                int d_dtype, int d_kind, bool kd, cudaStream_t s);
cudaError_t launch_chain_greedy(const ArgmaxParams& p, const RowPlan& plan, int dtype,
                                cudaStream_t s);
cudaError_t launch_tree_greedy(const ArgmaxParams& p, const RowPlan& plan, int dtype,
                               cudaStream_t s);
cudaError_t launch_topk(const TopkParams& p, const RowPlan& plan, int dtype, cudaStream_t s);
cudaError_t launch_kl(const KlParams& p, const RowPlan& plan, int d_dtype, int d_kind,
                      cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit (and allow clusters of more
// than 8 CTAs) once per device; later calls, including calls made while a
// stream is being captured into a CUDA graph, only look the setting up.
cudaError_t ensure_kernel_attrs(const void* kernel, int smem_bytes, bool nonportable_cluster);

// Clusters of `cluster` CTAs (kThreads each, smem_bytes of dynamic shared
// memory) that can be resident at once on the current device (cached).
cudaError_t max_active_clusters(const void* kernel, int smem_bytes, int cluster, int* out);

// Shared-memory layout for a chunk of L elements (bytes per element tb / db,
// db = 0 when there is no second row) with `fixed` bytes of fixed block.
RowLayout row_layout(int fixed, int L, int tb, int db, int npieces, int x_bytes);

}  // namespace sv
