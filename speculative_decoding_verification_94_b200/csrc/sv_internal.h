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

}  // namespace sv
