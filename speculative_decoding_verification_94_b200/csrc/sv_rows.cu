// sv_rows.cu -- greedy tree verification, top-K extraction and the KD loss.
//
// Same row plan as the chain kernels: one C-CTA cluster per vocabulary row,
// chunks resident in shared memory, partials combined in a fixed order
// through distributed shared memory, and a last-arriver per request (and per
// batch for the loss total) instead of a second launch.
#include "sv_rowops.cuh"

namespace sv {

template <class TT>
__device__ __forceinline__ unsigned long long chunk_argmax_key_rows(RowShared& sh,
                                                                    const unsigned char* buf,
                                                                    const ChunkGeom& g,
                                                                    bool use_bulk) {
  float best = -INFINITY;
  int bidx = -1;
  for (int p = 0; p < g.npieces; ++p) {
    if (!wait_piece(sh, p, use_bulk)) break;
    const int e = p * kRound + (int)threadIdx.x * kVec;
    if (e < g.nvec * kVec) {
      float v[8];
      const float vm = load8_max<TT>(buf, e, v);
      if (vm > best || bidx < 0) {
        int q = 0;
#pragma unroll
        for (int t = 7; t >= 0; --t)
          if (v[t] == vm) q = t;
        best = vm;
        bidx = g.j0 + e + q;
      }
    }
  }
  const unsigned long long key = bidx < 0 ? kNoKey : topk_key(best, bidx);
  return block_max_key(key, sh.redk);
}

// ---------------------------------------------------------------------------
// Greedy tree verification.  Rows are node-major (node j of every request,
// then node j+1) and each cluster writes the argmax of its node row.  The
// last node of a request to finish walks the tree in index order (parents
// precede children) and writes the deepest accepted path.
// ---------------------------------------------------------------------------
template <class TT>
__global__ void __launch_bounds__(kThreads) tree_greedy_kernel(const ArgmaxParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* buf = smem + prm.lay.off_t;
  const int n = prm.R, B = prm.B, V = prm.V;
  const int row = (int)(blockIdx.x / (unsigned)C);
  const int j = row / B, b = row - j * B;
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const bool use_bulk = prm.use_bulk != 0;
  stage_chunks<TT, TT, false>(sh, buf, nullptr, row_ptr<TT>(prm.logits, (size_t)b * n + j, V),
                              nullptr, g, use_bulk, false);
  const unsigned long long key = chunk_argmax_key_rows<TT>(sh, buf, g, use_bulk);
  if (threadIdx.x == 0) sh.key = key;
  drain_pieces(sh, g, use_bulk);
  cluster.sync();
  if (rank == 0 && threadIdx.x < 32) {
    const int lane = threadIdx.x;
    unsigned long long best = kNoKey;
    int tmo = 0;
    if (lane < C) {
      const RowShared* o = cluster.map_shared_rank(&sh, lane);
      best = o->key;
      tmo = o->timeouts;
    }
    best = warp_max_u64(best);
    tmo = warp_sum_int(tmo);
    if (lane == 0) {
      if (tmo) set_status(prm.status, SV_DEV_TIMEOUT);
      prm.ws.row_a[(size_t)b * n + j] = tmo ? 0 : key_index(best) + 1;  // 0 = no argmax
    }
  }
  cluster.sync();
  if (rank != 0) return;
  if (!arrive_last(&prm.ws.req_counter[b], (uint32_t)n, sh)) return;

  int* garg = reinterpret_cast<int*>(smem + prm.lay.off_x);
  int* par = garg + n;
  int* tok = par + n;
  int* dep = tok + n;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    garg[t] = __ldcg(&prm.ws.row_a[(size_t)b * n + t]) - 1;
    prm.ws.row_a[(size_t)b * n + t] = 0;
    par[t] = prm.parents[(size_t)b * n + t];
    tok[t] = prm.tokens[(size_t)b * n + t];
  }
  __syncthreads();
  const int W = prm.max_depth + 1;
  if (threadIdx.x == 0) {
    int bad = (par[0] != -1) || (garg[0] < 0);
    int best = 0;
    // dep[t] >= 0: node t accepted at that depth; dep[t] < 0: rejected, at
    // depth -dep[t] - 1.  The root is accepted at depth 0.
    dep[0] = 0;
    for (int t = 1; t < n && !bad; ++t) {
      const int pj = par[t];
      if (pj < 0 || pj >= t) {
        bad = 1;
        break;
      }
      const int dp = dep[pj] >= 0 ? dep[pj] : -dep[pj] - 1;
      const int d = dp + 1;
      if (d > prm.max_depth) {
        bad = 1;
        break;
      }
      if (tok[t] < 0 || tok[t] >= V) {
        set_status(prm.status, SV_DEV_BAD_TOKEN);
        bad = 2;
        break;
      }
      if (garg[t] < 0) {
        bad = 1;
        break;
      }
      const bool a = dep[pj] >= 0 && tok[t] == garg[pj];
      dep[t] = a ? d : -(d + 1);
      if (a && d > dep[best]) best = t;
    }
    if (bad == 1) set_status(prm.status, SV_DEV_BAD_TREE);
    sh.fin_n = bad ? -1 : dep[best];
    sh.fin_tok = best;
    prm.accepted_len[b] = sh.fin_n;
    prm.ws.req_counter[b] = 0u;
  }
  __syncthreads();
  const int L = sh.fin_n, best = sh.fin_tok;
  if (threadIdx.x == 0) {
    int32_t* on = prm.accepted_nodes + (size_t)b * W;
    int32_t* ot = prm.out_tokens + (size_t)b * W;
    for (int d = 0; d < W; ++d) on[d] = ot[d] = -1;
    if (L >= 0) {
      for (int t = best, d = L; d >= 0; t = par[t], --d) on[d] = t;
      for (int d = 0; d < L; ++d) ot[d] = tok[on[d + 1]];
      ot[L] = garg[best];
    }
  }
}

// ---------------------------------------------------------------------------
// Top-K extraction: per row, the online softmax normaliser and the K largest
// logits; rank 0 writes log-probs z/T - lse for the merged top K.
// ---------------------------------------------------------------------------
template <class TT>
__global__ void __launch_bounds__(kThreads) topk_kernel(const TopkParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* buf = smem + prm.lay.off_t;
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + prm.lay.off_x);
  const int row = (int)(blockIdx.x / (unsigned)C);
  const ChunkGeom g = chunk_geom(rank, prm.L, prm.V);
  const bool use_bulk = prm.use_bulk != 0;
  const float c = prm.c;
  stage_chunks<TT, TT, false>(sh, buf, nullptr, row_ptr<TT>(prm.logits, (size_t)row, prm.V),
                              nullptr, g, use_bulk, false);
  ThreadStat st;
  stat_init(st);
  for (int p = 0; p < g.npieces; ++p) {
    if (!wait_piece(sh, p, use_bulk)) break;
    const int e = p * kRound + (int)threadIdx.x * kVec;
    if (e < g.nvec * kVec) {
      float v[8];
      const float vm = load8_max<TT>(buf, e, v);
      stat_update(st, v, vm, c);
    }
  }
  const CtaStat cs = stat_block(st, sh.redf, sh.redd);
  if (threadIdx.x == 0) {
    sh.G_t = cs.G;
    sh.S_t = cs.S;
  }
  cta_topk<TT>(buf, g, st.mz, prm.K, sh, cand, prm.status);
  drain_pieces(sh, g, use_bulk);
  cluster.sync();
  if (rank == 0) {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      float G = -INFINITY;
      double S = 0.0;
      int tmo = 0;
      if (lane < C) {
        const RowShared* o = cluster.map_shared_rank(&sh, lane);
        G = o->G_t;
        S = o->S_t;
        tmo = o->timeouts;
      }
      float Gm;
      double Sm;
      warp_stat_combine(G, S, &Gm, &Sm);
      tmo = warp_sum_int(tmo);
      if (lane == 0) {
        sh.Gt = Gm;
        sh.St = Sm;
        sh.Lt = (double)Gm + log2(Sm);
        sh.err = 0;
        if (Gm == -INFINITY) sh.err |= SV_DEV_NO_FINITE;
        if (tmo) sh.err |= SV_DEV_TIMEOUT;
        if (sh.err) set_status(prm.status, sh.err);
      }
    }
    unsigned long long* out = cand + kCandCap - kMaxK;
    cluster_topk_merge(cluster, C, prm.K, sh, cand, out);
    const double ln2 = 0.69314718055994530942;
    const int K = prm.K;
    if (threadIdx.x < K) {
      const unsigned long long kk = out[threadIdx.x];
      const float z = key_value(kk);
      const double lp = ((double)z * (double)c - sh.Lt) * ln2;
      prm.topk_logp[(size_t)row * K + threadIdx.x] = sh.err ? NAN : (float)lp;
      prm.topk_idx[(size_t)row * K + threadIdx.x] = key_index(kk);
    }
    if (threadIdx.x == 0) prm.lse[row] = sh.err ? NAN : (float)(sh.Lt * ln2);
  }
  cluster.sync();
}

// ---------------------------------------------------------------------------
// KD loss.  One cluster per draft row (b, i < k), position-major.  Logits
// drafts are streamed for their normaliser and stay resident for the K
// gathers; probability drafts need only the K gathers (one CTA).
// ---------------------------------------------------------------------------
template <class DT, int DKIND>
__global__ void __launch_bounds__(kThreads) kl_kernel(const KlParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* dbuf = smem + prm.lay.off_t;
  const int k = prm.k, P = k + 1, B = prm.B, V = prm.V, K = prm.K;
  const int row = (int)(blockIdx.x / (unsigned)C);
  const int i = row / B, b = row - i * B;
  const float c = prm.c;
  const bool use_bulk = prm.use_bulk != 0;
  const void* drow = row_ptr<DT>(prm.draft, (size_t)b * k + i, V);
  ChunkGeom g = chunk_geom(rank, prm.L, V);
  if (DKIND == kDraftLogits) {
    stage_chunks<DT, DT, false>(sh, dbuf, nullptr, drow, nullptr, g, use_bulk, false);
    ThreadStat st;
    stat_init(st);
    for (int p = 0; p < g.npieces; ++p) {
      if (!wait_piece(sh, p, use_bulk)) break;
      const int e = p * kRound + (int)threadIdx.x * kVec;
      if (e < g.nvec * kVec) {
        float v[8];
        const float vm = load8_max<DT>(dbuf, e, v);
        stat_update(st, v, vm, c);
      }
    }
    const CtaStat cs = stat_block(st, sh.redf, sh.redd);
    if (threadIdx.x == 0) {
      sh.G_d = cs.G;
      sh.S_d = cs.S;
    }
    drain_pieces(sh, g, use_bulk);
  } else if (threadIdx.x == 0) {
    sh.timeouts = 0;
  }
  cluster.sync();
  if (rank == 0) {
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      float G = -INFINITY;
      double S = 0.0;
      int tmo = 0;
      if (DKIND == kDraftLogits && lane < C) {
        const RowShared* o = cluster.map_shared_rank(&sh, lane);
        G = o->G_d;
        S = o->S_d;
        tmo = o->timeouts;
      }
      float Gm;
      double Sm;
      warp_stat_combine(G, S, &Gm, &Sm);
      tmo = warp_sum_int(tmo);
      if (lane == 0) {
        sh.err = 0;
        sh.Ld = 0.0;
        if (DKIND == kDraftLogits) {
          sh.Gd = Gm;
          sh.Sd = Sm;
          sh.Ld = (double)Gm + log2(Sm);
          if (Gm == -INFINITY) sh.err |= SV_DEV_NO_FINITE;
          if (tmo) sh.err |= SV_DEV_TIMEOUT;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      const double ln2 = 0.69314718055994530942;
      const size_t trow = (size_t)b * P + i;
      double lp = -INFINITY;
      int j = -1;
      if (lane < K) {
        lp = (double)prm.topk_logp[trow * K + lane];
        j = prm.topk_idx[trow * K + lane];
      }
      const int badj = (lane < K && (j < 0 || j >= V)) ? 1 : 0;
      const int anybad = __any_sync(0xffffffffu, badj);
      double m = lp;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
      double s = (lane < K) ? exp(lp - m) : 0.0;
      s = warp_sum(s);
      const double lse_k = m + log(s);
      double term = 0.0;
      if (lane < K && !anybad && !sh.err) {
        float zd;
        if (DKIND == kDraftLogits) {
          const int owner = j / prm.L;
          const unsigned char* rb = cluster.map_shared_rank(dbuf, owner);
          zd = load1<DT>(rb, j - owner * prm.L);
        } else {
          zd = reinterpret_cast<const float*>(drow)[j];
        }
        const double log_pt = lp - lse_k;
        const double pt = exp(log_pt);
        const double log_q = (DKIND == kDraftLogits) ? ((double)zd * (double)c - sh.Ld) * ln2
                                                     : log((double)zd);
        term = (pt == 0.0) ? 0.0 : pt * (log_pt - log_q);
      }
      term = warp_sum(term);
      if (lane == 0) {
        int err = sh.err | (anybad ? SV_DEV_BAD_INDEX : 0);
        if (err) set_status(prm.status, err);
        prm.kl[(size_t)b * k + i] = err ? NAN : (float)term;
      }
    }
  }
  cluster.sync();
  if (rank != 0) return;
  if (!arrive_last(&prm.ws.req_counter[b], (uint32_t)k, sh)) return;
  if (threadIdx.x == 0) {
    int n = prm.accepted_len[b];
    if (n < 0 || n > k) {
      set_status(prm.status, SV_DEV_BAD_INDEX);
      n = -1;
    }
    sh.fin_n = n;
    prm.ws.req_counter[b] = 0u;
  }
  __syncthreads();
  kd_finalize(b, sh.fin_n, B, k, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip, prm.loss,
              prm.total, prm.ws.glob_counter, sh);
}

// ---------------------------------------------------------------------------
// Launchers.
// ---------------------------------------------------------------------------
template <class Kern, class Prm>
static cudaError_t launch_rows(Kern kernel, const Prm& prm, const RowPlan& plan, int nclusters,
                               cudaStream_t s) {
  cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(kernel), plan.lay.bytes,
                                      plan.C > 8);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nclusters * (unsigned)plan.C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)plan.lay.bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)plan.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, prm);
}

cudaError_t launch_tree_greedy(const ArgmaxParams& p, const RowPlan& plan, int dtype,
                               cudaStream_t s) {
  const int n = p.B * p.R;
  if (dtype == SV_BF16) return launch_rows(tree_greedy_kernel<BF16>, p, plan, n, s);
  return launch_rows(tree_greedy_kernel<F32>, p, plan, n, s);
}

cudaError_t launch_topk(const TopkParams& p, const RowPlan& plan, int dtype, cudaStream_t s) {
  if (dtype == SV_BF16) return launch_rows(topk_kernel<BF16>, p, plan, p.rows, s);
  return launch_rows(topk_kernel<F32>, p, plan, p.rows, s);
}

cudaError_t launch_kl(const KlParams& p, const RowPlan& plan, int d_dtype, int d_kind,
                      cudaStream_t s) {
  const int n = p.B * p.k;
  if (d_kind == kDraftProbs) return launch_rows(kl_kernel<F32, kDraftProbs>, p, plan, n, s);
  if (d_dtype == SV_BF16) return launch_rows(kl_kernel<BF16, kDraftLogits>, p, plan, n, s);
  return launch_rows(kl_kernel<F32, kDraftLogits>, p, plan, n, s);
}

}  // namespace sv
