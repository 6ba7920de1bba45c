// sv_tree_sample.cuh -- sampling verification of candidate trees.
//
// The rule is the multi-step speculative sampling of SpecInfer (Miao et al.,
// "SpecInfer: Accelerating Large Language Model Serving with Tree-based
// Speculative Inference and Verification"), the recursive rejection sampling
// that EAGLE adopts; the ReSpec reading notes (section 3, "G1 解法") name the
// EAGLE trees (depth s, top-t branching, n nodes) it runs on.  From the root,
// at node v with target row p_v and draft row q_v, r = p_v and the children of
// v are tried in ascending index order: child c with token x is accepted iff
// u_c * q_v(x) < r(x); on a rejection r becomes max(0, r - q_v) normalised.
// The walk moves to the first accepted child; a node whose children are all
// rejected (or a leaf) draws one token from r.
//
// Residual form used here: after i rejections r is proportional to
// max(0, p - sigma_i q) with sigma_0 = 0 and sigma_{i+1} = sigma_i + M_i, where
// M_i = sum_j max(0, p_j - sigma_i q_j) (M_0 = 1).  So the test of the next
// child is u * q(x) * M_i < max(0, p(x) - sigma_i q(x)), and only a rejection
// costs a pass over the row pair.
//
// One cluster of C CTAs per request.  Each visited node's row pair is staged
// into the cluster's shared memory (CTA q holds vocabulary chunk q), the
// rows' log-partitions and every residual mass are combined across the
// cluster in rank order through distributed shared memory, so every CTA takes
// the same decisions; the CTA that owns the drawn token writes the outputs.
// Nothing is read for nodes off the accepted path.
#pragma once

#include "sv_finish.cuh"

namespace sv {

// Per-CTA values of one cluster combine.  Two slots, used alternately: a CTA
// writes slot s again only after every CTA has passed the barrier that ended
// the previous read of s.
struct TreePart {
  float Gt, Gd;
  double St, Sd;
  double R;  // chunk mass of the current weights
  int timeouts;
  int pad;
};

struct TreeShared {
  TreePart part[2];
  double Lt, Ld;     // log2-partitions of the staged rows
  double M, lo, hi;  // residual mass of the cluster, this CTA's share [lo, hi)
  double tt;         // the draw's target in [0, M)
  double t16[16];    // 2^(j/16), j = 0..15, for exp2_f64_tab
  int nkids, err, owner, tok, piece, first_thread, last_pos, pad;
};

// Residual weights max(0, p - sigma q) of 8 consecutive entries in float64:
// p = 2^(zt c - Gt) / St, q likewise (or the given probability), with the
// exponents, the powers and the difference in float64, so that the running
// residual mass and the tests against it carry float64 rounding only (the
// difference p - sigma q cancels where the two rows agree).
template <class TT, class DT, int DKIND>
__device__ __forceinline__ void tree_weights8(const unsigned char* tbuf, const unsigned char* dbuf,
                                              int e, double c, double Gt, double invSt,
                                              double Gd, double invSd, double sg,
                                              const double* t16, double w[8]) {
  float zt[8];
  load8<TT>(tbuf, e, zt);
  float q[8];
  if (DKIND == kDraftLogits) load8<DT>(dbuf, e, q);
  else load8<F32>(dbuf, e, q);
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const double p = exp2_f64_tab(fma((double)zt[t], c, -Gt), t16) * invSt;
    const double qq =
        DKIND == kDraftLogits ? exp2_f64_tab(fma((double)q[t], c, -Gd), t16) * invSd : (double)q[t];
    w[t] = fmax(fma(-sg, qq, p), 0.0);
  }
}

__device__ __forceinline__ double seq_sum8d(const double w[8]) {
  double s = w[0];
#pragma unroll
  for (int t = 1; t < 8; ++t) s += w[t];
  return s;
}

// Per-piece totals of per-thread float64 sums sums[p * kThreads + t], in a
// fixed order (warp butterflies, then warps in index order).  Collective.
__device__ __forceinline__ void piece_totals_d(const double* sums, int npieces, RowShared& sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int p = 0; p < npieces; ++p) {
    const double v = warp_sum(sums[p * kThreads + threadIdx.x]);
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

// Sampling tree verification: one cluster of C CTAs per request.
template <class TT, class DT, int DKIND>
__global__ void __launch_bounds__(kThreads) tree_sample_kernel(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  TreeShared& ts = *reinterpret_cast<TreeShared*>(smem + prm.lay.off_rows);
  const int n = prm.k, V = prm.V, W = prm.max_depth + 1;
  int* par = reinterpret_cast<int*>(&ts + 1);
  int* tok = par + n;
  int* kids = tok + n;
  int* pth = kids + n;
  float* kzt = reinterpret_cast<float*>(pth + n);  // the children's target logits
  float* kzd = kzt + n;                            // ... and draft logits (or probabilities)
  double* kpx = reinterpret_cast<double*>(kzd + n);  // p(x) and q(x) of each child
  double* kqx = kpx + n;
  float* ku = reinterpret_cast<float*>(kqx + n);     // each child's uniform
  unsigned char* tbuf = smem + prm.lay.off_t;
  unsigned char* dbuf = smem + prm.lay.off_d;
  const int b = (int)(blockIdx.x / (unsigned)C);
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  double* sums = reinterpret_cast<double*>(smem + prm.lay.off_x);
  double* incl_arr = sums + g.npieces * kThreads;
  const float c = prm.c;
  const double c64 = prm.c64;
  const bool use_bulk = prm.use_bulk != 0;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  pdl_wait();
  // the root's row pair is needed by every valid tree: its copies start first
  const void* root_t = row_ptr<TT>(prm.target, (size_t)b * n, V);
  const void* root_d = row_ptr<DT>(prm.draft, (size_t)b * n, V);
  if (threadIdx.x == 0) {
    init_piece_barriers(sh, g, use_bulk);
    sh.timeouts = 0;
    if (use_bulk)
      issue_item_copies<TT, DT, true>(sh, tbuf, dbuf, root_t, root_d, g, policy_evict_first());
  }

  if (threadIdx.x < 16) ts.t16[threadIdx.x] = exp2_f64((double)threadIdx.x * 0.0625);

  // 0. the tree, checked the same way in every CTA (its barriers also
  //    publish the table above)
  int bad_tree = 0, bad_tok = 0;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    const int pj = prm.parents[(size_t)b * n + t];
    const int x = prm.tokens[(size_t)b * n + t];
    par[t] = pj;
    tok[t] = x;
    if (t == 0 ? pj != -1 : (pj < 0 || pj >= t)) bad_tree = 1;
    if (t > 0 && (x < 0 || x >= V)) bad_tok = 1;
  }
  bad_tree = __syncthreads_or(bad_tree);
  if (!bad_tree) {
    // depth of every node <= max_depth (parents precede children, so every
    // walk up ends at the root; it stops early once too deep)
    for (int t = threadIdx.x; t < n; t += kThreads) {
      int j = t, d = 0;
      while (j > 0 && d <= prm.max_depth) {
        j = par[j];
        ++d;
      }
      if (d > prm.max_depth) bad_tree = 1;
    }
  }
  bad_tree = __syncthreads_or(bad_tree);
  bad_tok = __syncthreads_or(bad_tok);
  if (bad_tree || bad_tok) {
    if (rank == 0) {
      if (threadIdx.x == 0) {
        set_status(prm.status, bad_tree ? SV_DEV_BAD_TREE : SV_DEV_BAD_TOKEN);
        prm.accepted_len[b] = -1;
      }
      for (int d = threadIdx.x; d < W; d += kThreads) {
        prm.out_tokens[(size_t)b * W + d] = -1;
        prm.accepted_nodes[(size_t)b * W + d] = -1;
      }
    }
    // no CTA has touched another's shared memory; the root's copies land
    // before this CTA's shared memory is released
    if (use_bulk && threadIdx.x == 0)
      for (int p = 0; p < g.npieces; ++p) mbar_wait_bounded(&sh.bars[p], 0u);
    return;
  }
  if (threadIdx.x == 0) pth[0] = 0;
  __syncthreads();

  int red = 0;  // cluster combines so far (selects the slot)
  // Chunk masses of the weights max(0, p - sg q) into sums[] and ts.part,
  // then the cluster total M and this CTA's share [lo, hi).  Collective over
  // the cluster.
  auto residual_pass = [&](double sg, double Gt, double invSt, double Gd, double invSd) {
#pragma unroll 2
    for (int p = 0; p < kMaxPieces; ++p) {
      if (p >= g.npieces) break;
      const int e = p * kRound + (int)threadIdx.x * kVec;
      double s = 0.0;
      if (e < g.nvec * kVec) {
        double wv[8];
        tree_weights8<TT, DT, DKIND>(tbuf, dbuf, e, c64, Gt, invSt, Gd, invSd, sg, ts.t16, wv);
        s = seq_sum8d(wv);
      }
      sums[p * kThreads + threadIdx.x] = s;
    }
    piece_totals_d(sums, g.npieces, sh);
    const int slot = red & 1;
    ++red;
    if (threadIdx.x == 0) {
      double Rc = 0.0;
      for (int p = 0; p < g.npieces; ++p) Rc += sh.ptot[p];
      ts.part[slot].R = Rc;
    }
    cluster.sync();
    if (w == 0) {
      const double Rq = lane < C ? cluster.map_shared_rank(&ts.part[slot], lane)->R : 0.0;
      const double incl = warp_scan_incl(Rq);
      const double tot = __shfl_sync(0xffffffffu, incl, 31);
      const double lo = __shfl_sync(0xffffffffu, incl, rank > 0 ? rank - 1 : 0);
      const double hi = __shfl_sync(0xffffffffu, incl, rank);
      if (lane == 0) {
        ts.M = tot;
        ts.lo = rank > 0 ? lo : 0.0;
        ts.hi = hi;
      }
    }
    __syncthreads();
  };

  int v = 0, depth = 0, visit = 0, err = 0;
  bool drawn = false;
  for (;;) {
    // a. stage the row pair of node v (after every warp has left the previous
    //    node's tests, which read kids[] and ts.nkids)
    __syncthreads();
    const size_t row = (size_t)b * n + v;
    const void* trow = row_ptr<TT>(prm.target, row, V);
    const void* drow = row_ptr<DT>(prm.draft, row, V);
    if (visit > 0 && threadIdx.x == 0) {  // (the root's copies were issued at the start)
      sh.timeouts = 0;
      if (use_bulk) {
        fence_proxy_async_smem();  // earlier reads of the buffers precede the copies
        issue_item_copies<TT, DT, true>(sh, tbuf, dbuf, trow, drow, g, policy_evict_first());
      }
    }
    if (w == 1) {
      // the children of v in ascending order
      int m = 0;
      for (int base = v + 1; base < n; base += 32) {
        const int j = base + lane;
        const bool is = j < n && par[j] == v;
        const unsigned bal = __ballot_sync(0xffffffffu, is);
        if (is) kids[m + __popc(bal & ((1u << lane) - 1u))] = j;
        m += __popc(bal);
      }
      if (lane == 0) ts.nkids = m;
    }
    scalar_fill<TT>(tbuf, trow, g, use_bulk, false);
    scalar_fill<DT>(dbuf, drow, g, use_bulk, DKIND == kDraftProbs);
    __syncthreads();
    // the two values each child's test reads, fetched while the copies land
    for (int i = threadIdx.x; i < ts.nkids; i += kThreads) {
      const int x = tok[kids[i]];
      kzt[i] = load1<TT>(reinterpret_cast<const unsigned char*>(trow), x);
      kzd[i] = load1<DT>(reinterpret_cast<const unsigned char*>(drow), x);
      ku[i] = prm.u[(size_t)b * n + kids[i]];
    }
    for (int p = 0; p < g.npieces; ++p) wait_piece(sh, p, use_bulk, (uint32_t)(visit & 1));
    __syncthreads();

    // b. the rows' statistics, combined over the cluster
    // (two passes over the staged chunk: the maxima, then the exp2 terms
    //  against one reference, so that the iterations are independent)
    ThreadStat a, d;
    stat_init(a);
    stat_init(d);
    {
      float mt = -INFINITY, md = -INFINITY;
#pragma unroll 4
      for (int p = 0; p < kMaxPieces; ++p) {
        if (p >= g.npieces) break;
        const int e = p * kRound + (int)threadIdx.x * kVec;
        if (e < g.nvec * kVec) {
          mt = fmaxf(mt, max8<TT>(tbuf, e));
          if (DKIND == kDraftLogits) md = fmaxf(md, max8<DT>(dbuf, e));
        }
      }
      // integer references ceil(max z * c) in float64 (exact in fp32 too);
      // the terms 2^(z c - ref) in float64
      a.mz = mt;
      a.ref = mt == -INFINITY ? -INFINITY : (float)ceil((double)mt * c64);
      if (DKIND == kDraftLogits) {
        d.mz = md;
        d.ref = md == -INFINITY ? -INFINITY : (float)ceil((double)md * c64);
      }
      const bool fa = a.ref != -INFINITY, fd = DKIND == kDraftLogits && d.ref != -INFINITY;
#pragma unroll 2
      for (int p = 0; p < kMaxPieces; ++p) {
        if (p >= g.npieces) break;
        const int e = p * kRound + (int)threadIdx.x * kVec;
        if (e < g.nvec * kVec) {
          float z[8];
          if (fa) {
            load8<TT>(tbuf, e, z);
            double t = 0.0;
#pragma unroll
            for (int k = 0; k < 8; ++k) t += exp2_f64_tab(fma((double)z[k], c64, -(double)a.ref), ts.t16);
            a.S += t;
          }
          if (fd) {
            load8<DT>(dbuf, e, z);
            double t = 0.0;
#pragma unroll
            for (int k = 0; k < 8; ++k) t += exp2_f64_tab(fma((double)z[k], c64, -(double)d.ref), ts.t16);
            d.S += t;
          }
        }
      }
    }
    CtaStat ca, cd;
    stat_block2(a, d, sh.redf2, sh.redd2, &ca, &cd);
    {
      const int slot = red & 1;
      ++red;
      if (threadIdx.x == 0) {
        ts.part[slot].Gt = ca.G;
        ts.part[slot].St = ca.S;
        ts.part[slot].Gd = cd.G;
        ts.part[slot].Sd = cd.S;
        ts.part[slot].timeouts = sh.timeouts;
      }
      cluster.sync();
      if (w == 0) {
        const TreePart* q = cluster.map_shared_rank(&ts.part[slot], lane < C ? lane : 0);
        float Gt, Gd;
        double St, Sd;
        warp_stat_combine(lane < C ? q->Gt : -INFINITY, lane < C ? q->St : 0.0, &Gt, &St);
        warp_stat_combine(lane < C ? q->Gd : -INFINITY, lane < C ? q->Sd : 0.0, &Gd, &Sd);
        const int tmo = warp_sum_int(lane < C ? q->timeouts : 0);
        if (lane == 0) {
          sh.Gt = Gt;
          sh.St = St;
          sh.Gd = Gd;
          sh.Sd = Sd;
          ts.Lt = (double)Gt + log2(St);
          ts.Ld = (double)Gd + log2(Sd);
          ts.err = tmo ? SV_DEV_TIMEOUT
                       : ((Gt == -INFINITY || (DKIND == kDraftLogits && Gd == -INFINITY))
                              ? SV_DEV_NO_FINITE
                              : 0);
        }
      }
      __syncthreads();
    }
    if (ts.err) {
      err = ts.err;
      break;
    }

    // c. the children's tests against the running residual (p(x) and q(x) of
    //    every child first, in parallel)
    const double Gt = (double)sh.Gt, Gd = (double)sh.Gd;
    const double invSt = 1.0 / sh.St;
    const double invSd = DKIND == kDraftLogits ? 1.0 / sh.Sd : 1.0;
    {
      for (int i = threadIdx.x; i < ts.nkids; i += kThreads) {
        kpx[i] = exp2_f64_tab(fma((double)kzt[i], c64, -Gt), ts.t16) * invSt;
        kqx[i] = DKIND == kDraftLogits ? exp2_f64_tab(fma((double)kzd[i], c64, -Gd), ts.t16) * invSd
                                       : (double)kzd[i];
      }
      __syncthreads();
    }
    double sigma = 0.0, M = 1.0;
    bool have = false, fallback = false;
    int next = -1;
    for (int i = 0; i < ts.nkids; ++i) {
      const int node = kids[i];
      const double px = kpx[i], qx = kqx[i];
      const double rx = fmax(px - sigma * qx, 0.0);
      const double uc = (double)ku[i];
      if (uc * qx * M < rx) {  // accepted with probability min(1, r(x) / q(x))
        next = node;
        break;
      }
      sigma += M;
      residual_pass(sigma, Gt, invSt, Gd, invSd);
      M = ts.M;
      have = true;
      if (!(M > 0.0)) {  // zero residual mass: draw from the target row
        fallback = true;
        break;
      }
    }
    if (next >= 0) {
      ++depth;
      if (threadIdx.x == 0) pth[depth] = next;
      v = next;
      ++visit;
      continue;  // (depth <= max_depth: checked above)
    }

    // d. the draw from max(0, p - sigma q) (p itself at sigma = 0)
    if (fallback) {
      if (rank == 0 && threadIdx.x == 0) set_status(prm.status, SV_DEV_RESIDUAL_ZERO);
      sigma = 0.0;
      have = false;
    }
    if (!have) residual_pass(sigma, Gt, invSt, Gd, invSd);
    if (threadIdx.x == 0) {
      ts.tt = (double)prm.u[(size_t)b * n] * ts.M;
      ts.owner = (ts.M > 0.0 && ts.lo <= ts.tt && ts.tt < ts.hi) ? 1 : 0;
      ts.tok = -1;
      if (!(ts.M > 0.0)) ts.err = SV_DEV_NO_FINITE;
    }
    __syncthreads();
    err = ts.err;
    if (ts.owner) {
      if (threadIdx.x == 0) {
        double base = ts.lo;
        int pp = -1;
        for (int p = 0; p < g.npieces; ++p) {
          if (base + sh.ptot[p] > ts.tt) {
            pp = p;
            break;
          }
          base += sh.ptot[p];
        }
        if (pp < 0) {  // rounding pushed the target past this chunk: last piece with mass
          double b2 = ts.lo;
          base = ts.lo;
          for (int p = 0; p < g.npieces; ++p) {
            if (sh.ptot[p] > 0.0) {
              pp = p;
              base = b2;
            }
            b2 += sh.ptot[p];
          }
        }
        ts.piece = pp;
        ts.lo = base;
        ts.first_thread = kThreads;
        ts.last_pos = -1;
      }
      __syncthreads();
      const int pp = ts.piece;
      if (pp >= 0) {
        const double s = sums[pp * kThreads + threadIdx.x];
        double tot;
        const double incl = block_scan_incl(s, sh.redd, &tot);
        incl_arr[threadIdx.x] = incl;
        if (ts.lo + incl > ts.tt) atomicMin(&ts.first_thread, (int)threadIdx.x);
        if (s > 0.0) atomicMax(&ts.last_pos, (int)threadIdx.x);
        __syncthreads();
        int tsel = ts.first_thread;
        const bool fb = (tsel == kThreads);
        if (fb) tsel = ts.last_pos;
        if ((int)threadIdx.x == tsel) {
          const int e = pp * kRound + tsel * kVec;
          double wv[8];
          tree_weights8<TT, DT, DKIND>(tbuf, dbuf, e, c64, Gt, invSt, Gd, invSd, sigma, ts.t16, wv);
          const double b0 = ts.lo + (tsel > 0 ? incl_arr[tsel - 1] : 0.0);
          double acc = 0.0;
          int pick = -1, lastq = -1;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            acc += wv[q];
            if (wv[q] > 0.0) lastq = q;
            if (!fb && pick < 0 && b0 + acc > ts.tt) pick = q;
          }
          if (pick < 0) pick = lastq;
          ts.tok = pick < 0 ? -1 : g.j0 + e + pick;
        }
        __syncthreads();
      }
      drawn = true;
    }
    break;
  }

  // 4. outputs, by the owner of the drawn token (the first CTA on an error)
  const bool writer = err ? rank == 0 : drawn;
  if (writer) {
    const int tk = err ? -1 : ts.tok;
    const bool ok = !err && tk >= 0 && tk < V;
    if (threadIdx.x == 0) {
      if (err) set_status(prm.status, err);
      prm.accepted_len[b] = ok ? depth : -1;
    }
    for (int d = threadIdx.x; d < W; d += kThreads) {
      int on = -1, ot = -1;
      if (ok && d <= depth) {
        on = pth[d];
        ot = d < depth ? tok[pth[d + 1]] : tk;
      }
      prm.accepted_nodes[(size_t)b * W + d] = on;
      prm.out_tokens[(size_t)b * W + d] = ot;
    }
  }
  drain_pieces(sh, g, use_bulk, (uint32_t)(visit & 1));
  cluster.sync();  // no CTA leaves while another may still read its shared memory
}

}  // namespace sv
