// sv_rowops.cuh -- row-level collectives built on sv_device.cuh: the shared
// fixed block of every row kernel, chunk staging, CTA and cluster top-K, the
// inverse-CDF draw over a cluster-resident row, and the request finalizers.
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

// Row results kept in the workspace between a row and its request's
// finalizer (zero = not written; the finalizer zeroes them again).
enum RowResult : int { kRowAccepted = 1, kRowRejected = 2, kRowSkipped = 3, kRowError = 4 };

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

__device__ __forceinline__ unsigned long long block_max_key(unsigned long long v,
                                                            unsigned long long* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
    v = y > v ? y : v;
  }
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  unsigned long long r = red[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) r = red[i] > r ? red[i] : r;
  return r;
}

// CTA top-K of a staged chunk, sorted by (value desc, index asc) into sh.topk.
// A threshold (the K-th largest per-thread maximum) bounds the candidates: at
// least K elements reach it, so every top-K element does too.  Candidates are
// ranked exactly.  Massive ties overflow the candidate buffer and take K
// exact block-wide passes instead.  Collective.
template <class T>
__device__ void cta_topk(const unsigned char* buf, const ChunkGeom& g, float thread_max, int K,
                         RowShared& sh, unsigned long long* cand, int32_t* status) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float v = warp_sort_desc(thread_max);
  sh.tmax[w][lane] = v;
  __syncthreads();
  if (w == 0) {
    float a = sh.tmax[0][lane];
    for (int q = 1; q < kWarps; ++q) a = warp_merge_desc(a, sh.tmax[q][lane]);
    if (lane == K - 1) sh.theta = a;
    if (lane == 0) sh.cand_count = 0;
  }
  __syncthreads();
  const float th = sh.theta;
  for (int p = 0; p < g.npieces; ++p) {
    const int e = p * kRound + (int)threadIdx.x * kVec;
    if (e < g.nvec * kVec) {
      float x[8];
      const float m = load8_max<T>(buf, e, x);
      if (m >= th) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (e + q < g.len && x[q] >= th) {
            const int pos = atomicAdd(&sh.cand_count, 1);
            if (pos < kCandCap) cand[pos] = topk_key(x[q], g.j0 + e + q);
          }
        }
      }
    }
  }
  __syncthreads();
  const int n = sh.cand_count;
  if (n <= kCandCap) {
    rank_select(cand, n, K, sh.topk);
  } else {
    if (threadIdx.x == 0) set_status(status, SV_DEV_TOPK_SLOW);
    unsigned long long last = ~0ull;
    for (int r = 0; r < K; ++r) {
      unsigned long long best = kNoKey;
      for (int p = 0; p < g.npieces; ++p) {
        const int e = p * kRound + (int)threadIdx.x * kVec;
        if (e < g.nvec * kVec) {
          float x[8];
          load8<T>(buf, e, x);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (e + q < g.len) {
              const unsigned long long kk = topk_key(x[q], g.j0 + e + q);
              if (kk < last && kk > best) best = kk;
            }
          }
        }
      }
      best = block_max_key(best, sh.redk);
      if (threadIdx.x == 0) sh.topk[r] = best;
      last = best;
    }
  }
  __syncthreads();
}

// Merge the C CTA lists of a cluster into the row's top-K (rank 0, collective
// over its block).  Only keys at least as large as the largest per-CTA K-th
// key can be in the row's top K.
__device__ inline void cluster_topk_merge(cg::cluster_group& cluster, int C, int K, RowShared& sh,
                                   unsigned long long* cand, unsigned long long* out) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    unsigned long long th =
        lane < C ? cluster.map_shared_rank(&sh, lane)->topk[K - 1] : kNoKey;
    th = warp_max_u64(th);
    if (lane == 0) {
      sh.keyth = th;
      sh.cand_count = 0;
    }
  }
  __syncthreads();
  const unsigned long long th = sh.keyth;
  for (int t = threadIdx.x; t < C * K; t += kThreads) {
    const RowShared* o = cluster.map_shared_rank(&sh, t / K);
    const unsigned long long kk = o->topk[t % K];
    if (kk != kNoKey && kk >= th) cand[atomicAdd(&sh.cand_count, 1)] = kk;
  }
  __syncthreads();
  rank_select(cand, sh.cand_count, K, out);
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
__device__ inline void kd_finalize(int b, int n, int B, int k, const float* kl, const float* reward,
                            int wmode, int group, float clip, float* loss, float* total,
                            uint32_t* glob_counter, RowShared& sh) {
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += (double)__ldcg(&kl[(size_t)b * k + i]);
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
