// sv_internal.h -- plans shared by the libsv sources.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sv.h"

namespace sv {

// Shared-memory layout of a finishing kernel: fixed block, then the staged
// chunk(s) of one row pair, then a scratch region.
struct RowLayout {
  int off_rows;  // per-row records of the request (RowRec each)
  int off_t;   // target chunk
  int off_d;   // draft chunk
  int off_x;   // scratch (per-piece weight sums, scan values, KD merge buffers)
  int bytes;   // total dynamic shared memory
};

// Finishing plan for one row pair: C CTAs (a cluster) of L elements each.
struct RowPlan {
  int C;
  int L;         // multiple of 8
  int npieces;
  int use_bulk;  // 1: rows 16-byte aligned, bulk copies; 0: plain loads
  RowLayout lay;
};

// Workspace layout (all of it zero between calls).
struct WsLayout {
  size_t off_glob, off_reject, off_counter, off_rec, off_part, off_cand, bytes;
};

// Process-wide test and tuning knobs (sv_set_knob; 0 = the library's choice).
long long knob(int id);

// Per-device helpers shared by the launchers (sv_api.cu).
cudaError_t ensure_kernel_attrs(const void* kernel, int smem_bytes, bool nonportable);
cudaError_t sm_count(int* out);

// Chain verification in one persistent launch (sv_chain_*.cu): the
// arguments of sv_verify_chain after validation, the workspace carved by
// chain_ws_layout.
struct ChainArgs {
  const void* target;
  int t_dtype;
  const void* draft;
  int d_dtype;
  int d_kind;
  const int32_t* tokens;
  const float* u;
  const int32_t* klen;
  const int32_t* active;
  int B, k, V;
  float temperature;
  int32_t* accepted_len;
  int32_t* out_tokens;
  const sv_kd_args* kd;
  void* workspace;
  int32_t* status;
  cudaStream_t stream;
};
size_t chain_ws_bytes(int B, int k, int V, int K);
cudaError_t launch_chain_bf16(const ChainArgs& a);
cudaError_t launch_chain_f32(const ChainArgs& a);

}  // namespace sv
