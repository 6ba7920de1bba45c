// sv_rowops.cuh -- block-level pieces of the finishing kernels, built on
// sv_device.cuh: the fixed shared-memory block, staging of one row pair's
// chunk, per-piece totals, reward weights and the request/batch finalizers.
#pragma once

#include "sv_device.cuh"
#include "sv_internal.h"

namespace sv {

// Fixed block at the start of dynamic shared memory.  Fields marked (x) are
// read by the other CTAs of the cluster through distributed shared memory.
struct RowShared {
  uint64_t bars[kMaxPieces];
  // (x) per-CTA partials of the current item
  float G_t, G_d;
  double S_t, S_d;
  float zx_t, zx_d;
  int has_x;
  int timeouts;
  int skip;       // this CTA skipped the item (an earlier row of the request rejected)
  int next_item;  // (rank 0) the item this cluster processes after the current one
  int first_item; // (rank 0) the first item of this cluster
  int pad0;
  double R;
  unsigned long long key;
  unsigned long long topk[kMaxK];
  // block-local
  double ptot[kMaxPieces];
  double wsum[kWarps][kMaxPieces];
  float redf[kWarps];
  double redd[kWarps];
  float2 redf2[2 * kWarps];
  double2 redd2[kWarps];
  unsigned long long redk[kWarps];
  float tmax[kWarps][32];
  float theta;
  int cand_count;
  unsigned long long keyth;
  // item decision, computed by warp 0 and broadcast
  float Gt, Gd;
  double St, Sd, Lt, Ld;
  int accept, need, err, owner, rowskip, item;
  double base, tt;
  int piece, first_thread, last_pos, tok;
  int last, fin_n, fin_tok, redo;
};

constexpr int kFixedBytes = (int)((sizeof(RowShared) + 127) / 128 * 128);

template <class T>
__device__ __forceinline__ const void* row_ptr(const void* base, size_t row, int V) {
  return reinterpret_cast<const unsigned char*>(base) + row * (size_t)V * T::bytes;
}

__device__ __forceinline__ uint32_t load_relaxed(const uint32_t* p) {
  return *reinterpret_cast<const volatile uint32_t*>(p);
}

// Once per kernel (thread 0): initialise the piece barriers.
__device__ __forceinline__ void init_piece_barriers(RowShared& sh, const ChunkGeom& g,
                                                    bool use_bulk) {
  if (use_bulk) {
    for (int p = 0; p < g.npieces; ++p) mbar_init(&sh.bars[p], 1);
    fence_mbar_init();
  }
}

// Thread 0: arm the piece barriers of this item and issue its bulk copies.
template <class TT, class DT, bool PAIR>
__device__ __forceinline__ void issue_item_copies(RowShared& sh, unsigned char* tbuf,
                                                  unsigned char* dbuf, const void* trow,
                                                  const void* drow, const ChunkGeom& g,
                                                  uint64_t policy) {
  for (int p = 0; p < g.npieces; ++p)
    mbar_arrive_expect_tx(&sh.bars[p],
                          piece_bytes<TT>(g, p) + (PAIR ? piece_bytes<DT>(g, p) : 0u));
  issue_row_copies<TT>(tbuf, trow, g, sh.bars, policy);
  if (PAIR) issue_row_copies<DT>(dbuf, drow, g, sh.bars, policy);
}

// Stage one or two rows' chunks into shared memory (single-item kernels).
// Collective.
template <class TT, class DT, bool PAIR>
__device__ __forceinline__ void stage_chunks(RowShared& sh, unsigned char* tbuf,
                                             unsigned char* dbuf, const void* trow,
                                             const void* drow, const ChunkGeom& g,
                                             bool use_bulk, bool dprobs) {
  if (threadIdx.x == 0) {
    sh.timeouts = 0;
    init_piece_barriers(sh, g, use_bulk);
    if (use_bulk)
      issue_item_copies<TT, DT, PAIR>(sh, tbuf, dbuf, trow, drow, g, policy_evict_first());
  }
  scalar_fill<TT>(tbuf, trow, g, use_bulk, false);
  if (PAIR) scalar_fill<DT>(dbuf, drow, g, use_bulk, dprobs);
  __syncthreads();
}

// Wait for piece p (bulk path) in phase `phase`; records a timeout.
__device__ __forceinline__ bool wait_piece(RowShared& sh, int p, bool use_bulk,
                                           uint32_t phase = 0) {
  if (!use_bulk) return true;
  if (mbar_wait_bounded(&sh.bars[p], phase)) return true;
  atomicAdd(&sh.timeouts, 1);
  return false;
}

// After a timed-out wait, wait once more (bounded) so that no bulk copy into
// shared memory is still in flight when the buffer is reused or the CTA exits.
__device__ __forceinline__ void drain_pieces(RowShared& sh, const ChunkGeom& g, bool use_bulk,
                                             uint32_t phase = 0) {
  if (!use_bulk || threadIdx.x != 0) return;
  if (sh.timeouts == 0) return;
  for (int p = 0; p < g.npieces; ++p) mbar_wait_bounded(&sh.bars[p], phase);
}

// Per-piece totals of per-thread sums sums[p * kThreads + t], in a fixed
// order (warp butterflies, then warps in index order).  Collective.
__device__ __forceinline__ void piece_totals(const float* sums, int npieces, RowShared& sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int p = 0; p < npieces; ++p) {
    const double v = warp_sum((double)sums[p * kThreads + threadIdx.x]);
    if (lane == 0) sh.wsum[w][p] = v;
  }
  __syncthreads();
  if ((int)threadIdx.x < npieces) {
    double t = 0.0;
#pragma unroll
    for (int q = 0; q < kWarps; ++q) t += sh.wsum[q][threadIdx.x];
    sh.ptot[threadIdx.x] = t;
  }
  __syncthreads();
}

// Reward weight of request b (fixed summation order over its group).
__device__ __forceinline__ double reward_weight(const float* reward, int b, int wmode, int group,
                                                float clip) {
  double w = (double)reward[b];
  if (wmode == SV_W_GROUP_NORM) {
    const int g0 = (b / group) * group;
    double gs = 0.0;
    for (int t = g0; t < g0 + group; ++t) gs += (double)reward[t];
    w = (gs == 0.0) ? 0.0 : (double)reward[b] / gs;
  }
  if (clip > 0.f) w = fmin(fmax(w, -(double)clip), (double)clip);
  return w;
}

// Count this row in its request; returns true (block-uniform) if it was the
// last one, after a fence that makes the other rows' results visible.  The
// caller's writes are made visible by the fence before the increment.
__device__ __forceinline__ bool arrive_last(uint32_t* counter, uint32_t total, RowShared& sh) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(counter, 1u);
    sh.last = (old == total - 1u);
    if (sh.last) __threadfence();
  }
  __syncthreads();
  return sh.last != 0;
}

// Loss of request b, then (if it is the last request) the total.  Called by
// the whole block that finalized request b.  kl rows are read through L2.
__device__ inline void kd_finalize(int b, int n, int B, int k, int kb, const float* kl,
                            const float* reward,
                            int wmode, int group, float clip, int positions, float* loss,
                            float* total, uint32_t* glob_counter, RowShared& sh) {
  if (threadIdx.x == 0) {
    // the KD positions: the accepted drafts, and with `positions` the first
    // rejected one as well (kb: the request's draft count)
    const int m = (positions && n >= 0 && n < kb) ? n + 1 : n;
    double s = 0.0;
    for (int i = 0; i < m; ++i) s += (double)__ldcg(&kl[(size_t)b * k + i]);
    const double w = (n < 0) ? 0.0 : reward_weight(reward, b, wmode, group, clip);
    loss[b] = (w == 0.0) ? 0.f : (float)(w * s);
  }
  if (!arrive_last(glob_counter, (uint32_t)B, sh)) return;
  double part = 0.0;
  for (int t = threadIdx.x; t < B; t += kThreads) part += (double)__ldcg(&loss[t]);
  const double tot = block_sum(part, sh.redd);
  if (threadIdx.x == 0) {
    *total = (float)tot;
    *glob_counter = 0u;
  }
}

}  // namespace sv
