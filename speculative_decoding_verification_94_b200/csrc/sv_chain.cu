// sv_chain.cu -- chain verification kernels (persistent clusters).
//
// Work items are rows (b, i): target row i of request b and, for i < k, draft
// row i.  Items are handed out in position-major order (every request's i = 0
// first) from a counter in the workspace to persistent C-CTA clusters; each
// CTA of a cluster stages its chunk of the item's rows into shared memory with
// bulk copies.  Verification is sequential within a request (a draft is only
// tested if all earlier ones were accepted), so an item whose request already
// rejected at an earlier position is skipped before any byte is loaded: rows
// after the first rejection are never read.  With many requests, positions run
// one after the other per request and no row is read in vain; with few
// requests, otherwise idle clusters work on later positions speculatively.
//
// Per item (sampling, T > 0):
//   1. skip check; bulk copies; online max / sum-of-exp2 per thread -> per
//      CTA; optional CTA top-K of the target chunk (fused KD)
//   2. cluster barrier; warp 0 of every CTA combines the C partials in the same
//      order (identical bits everywhere) and evaluates the acceptance test
//      u * q(x) < p(x) in float64
//   3. if this row must be sampled (a rejection, or the bonus row):
//      residual weights max(0, p - q) (or p) from shared memory, cluster
//      barrier, chunk offsets, inverse-CDF search inside the owning CTA
//   4. rank 0: fused KD (cluster top-K merge, lse, KL against the draft row
//      gathered from the resident chunks), row result
//   5. final cluster barrier; the last row of a request to finish writes the
//      request's outputs (and the KD loss; the last request the total).
#include "sv_rowops.cuh"

namespace sv {

enum { kModeResidual = 0, kModeP = 1 };

template <class TT, class DT, int DKIND>
__device__ __forceinline__ void weights8(const unsigned char* tbuf, const unsigned char* dbuf,
                                         int e, int mode, float c, float Gt, float invSt,
                                         float Gd, float invSd, float w[8]) {
  float zt[8];
  load8<TT>(tbuf, e, zt);
  float p[8];
  // explicitly rounded products: p - q must be exactly 0 when p == q
#pragma unroll
  for (int t = 0; t < 8; ++t) p[t] = __fmul_rn(ex2(fmaf(zt[t], c, -Gt)), invSt);
  if (mode == kModeResidual) {
    float q[8];
    if (DKIND == kDraftLogits) {
      float zd[8];
      load8<DT>(dbuf, e, zd);
#pragma unroll
      for (int t = 0; t < 8; ++t) q[t] = __fmul_rn(ex2(fmaf(zd[t], c, -Gd)), invSd);
    } else {
      load8<F32>(dbuf, e, q);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = fmaxf(__fsub_rn(p[t], q[t]), 0.f);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = p[t];
  }
}

__device__ __forceinline__ float seq_sum8(const float w[8]) {
  float s = w[0];
#pragma unroll
  for (int t = 1; t < 8; ++t) s = __fadd_rn(s, w[t]);
  return s;
}

// Request finalizer, run by the whole rank-0 block of the cluster that
// finished the request's last row.  Reads and clears the row results.
__device__ void chain_finalize(const ChainParams& prm, int b, bool kd, RowShared& sh,
                               int* scratch) {
  const int k = prm.k, P = k + 1, V = prm.V;
  int* fa = scratch;
  int* fc = scratch + kThreads;
  for (int t = threadIdx.x; t < P; t += kThreads) {
    const size_t r = (size_t)b * P + t;
    fa[t] = __ldcg(&prm.ws.row_a[r]);
    fc[t] = __ldcg(&prm.ws.row_b[r]);
    prm.ws.row_a[r] = 0;
    prm.ws.row_b[r] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = k;
    for (int t = 0; t < k; ++t)
      if (fa[t] == kRowRejected) {
        n = t;
        break;
      }
    int bad = 0;
    for (int t = 0; t <= n; ++t) bad |= (fa[t] != kRowAccepted && fa[t] != kRowRejected);
    const int tk = fc[n] - 1;
    if (tk < 0 || tk >= V) bad = 1;
    sh.fin_n = bad ? -1 : n;
    sh.fin_tok = tk;
    prm.accepted_len[b] = sh.fin_n;
    prm.ws.req_counter[b] = 0u;
    prm.ws.req_reject[b] = 0u;
  }
  __syncthreads();
  const int n = sh.fin_n;
  for (int t = threadIdx.x; t < P; t += kThreads) {
    int v = -1;
    if (n >= 0) v = (t < n) ? prm.tokens[(size_t)b * k + t] : (t == n ? sh.fin_tok : -1);
    prm.out_tokens[(size_t)b * P + t] = v;
  }
  if (!kd) return;
  // KD rows after the emitted position were never (or only speculatively)
  // read: define them as empty.
  const int K = prm.K;
  const int first_undef = n < 0 ? 0 : n + 1;
  for (int t = first_undef * K + (int)threadIdx.x; t < P * K; t += kThreads) {
    prm.topk_logp[(size_t)b * P * K + t] = NAN;
    prm.topk_idx[(size_t)b * P * K + t] = -1;
  }
  for (int t = first_undef + (int)threadIdx.x; t < P; t += kThreads)
    prm.lse[(size_t)b * P + t] = NAN;
  for (int t = first_undef + (int)threadIdx.x; t < k; t += kThreads)
    prm.kl[(size_t)b * k + t] = NAN;
  kd_finalize(b, n, prm.B, k, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip, prm.loss,
              prm.total, prm.ws.glob_counter, sh);
}

// Cluster bookkeeping when a cluster runs out of items: the last one resets
// the item counter for the next call.
__device__ __forceinline__ void cluster_retire(const Workspace& ws, int rank, int C) {
  if (rank == 0 && threadIdx.x == 0) {
    __threadfence();
    const uint32_t nclusters = gridDim.x / (uint32_t)C;
    if (atomicAdd(ws.done, 1u) == nclusters - 1u) {
      *ws.work = 0u;
      *ws.done = 0u;
    }
  }
}

template <class TT, class DT, int DKIND, bool KD>
__global__ void __launch_bounds__(kThreads, 4) chain_sample_kernel(const ChainParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* tbuf = smem + prm.lay.off_t;
  unsigned char* dbuf = smem + prm.lay.off_d;
  float* sums = reinterpret_cast<float*>(smem + prm.lay.off_x);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + prm.lay.off_x);

  const int k = prm.k, P = k + 1, B = prm.B, V = prm.V;
  const int total = B * P;
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const float c = prm.c;
  const bool use_bulk = prm.use_bulk != 0;
  uint64_t policy = 0;
  uint32_t phase = 0;

  if (threadIdx.x == 0) {
    init_piece_barriers(sh, g, use_bulk);
    if (use_bulk) policy = policy_evict_first();
    if (rank == 0) sh.first_item = (int)atomicAdd(prm.ws.work, 1u);
  }
  cluster.sync();
  if (threadIdx.x == 0) sh.item = cluster.map_shared_rank(&sh, 0)->first_item;
  __syncthreads();
  int item = sh.item;

  while (item < total) {
    const int i = item / B, b = item - i * B;
    const bool has_draft = i < k;
    const void* trow = row_ptr<TT>(prm.target, (size_t)b * P + i, V);
    const void* drow = has_draft ? row_ptr<DT>(prm.draft, (size_t)b * k + i, V) : nullptr;
    const int x = has_draft ? prm.tokens[(size_t)b * k + i] : -1;

    // 1. skip check, bulk copies, streaming statistics.
    if (threadIdx.x == 0) {
      if (rank == 0) sh.next_item = (int)atomicAdd(prm.ws.work, 1u);
      sh.skip = load_relaxed(&prm.ws.req_reject[b]) > (uint32_t)(k - i) ? 1 : 0;
      sh.timeouts = 0;
      if (use_bulk && !sh.skip) {
        if (has_draft)
          issue_item_copies<TT, DT, true>(sh, tbuf, dbuf, trow, drow, g, policy);
        else
          issue_item_copies<TT, DT, false>(sh, tbuf, dbuf, trow, drow, g, policy);
      }
    }
    __syncthreads();
    const bool skip = sh.skip != 0;
    if (!skip) {
      scalar_fill<TT>(tbuf, trow, g, use_bulk, false);
      if (has_draft) scalar_fill<DT>(dbuf, drow, g, use_bulk, DKIND == kDraftProbs);
    }
    __syncthreads();

    ThreadStat st_t, st_d;
    stat_init(st_t);
    stat_init(st_d);
    if (!skip) {
      for (int p = 0; p < g.npieces; ++p) {
        if (!wait_piece(sh, p, use_bulk, phase)) break;
        const int e = p * kRound + (int)threadIdx.x * kVec;
        if (e < g.nvec * kVec) {
          float v[8];
          float vm = load8_max<TT>(tbuf, e, v);
          stat_update(st_t, v, vm, c);
          if (DKIND == kDraftLogits && has_draft) {
            vm = load8_max<DT>(dbuf, e, v);
            stat_update(st_d, v, vm, c);
          }
        }
      }
    }
    if (DKIND == kDraftLogits && has_draft) {
      CtaStat ct, cd;
      stat_block2(st_t, st_d, sh.redf2, sh.redd2, &ct, &cd);
      if (threadIdx.x == 0) {
        sh.G_t = ct.G;
        sh.S_t = ct.S;
        sh.G_d = cd.G;
        sh.S_d = cd.S;
      }
    } else {
      const CtaStat cs = stat_block(st_t, sh.redf, sh.redd);
      if (threadIdx.x == 0) {
        sh.G_t = cs.G;
        sh.S_t = cs.S;
      }
    }
    if (!skip && use_bulk) {
      drain_pieces(sh, g, use_bulk, phase);
      phase ^= 1u;
    }
    if (threadIdx.x == 0) {
      sh.has_x = 0;
      if (!skip && has_draft && x >= g.j0 && x < g.j0 + g.len) {
        sh.has_x = 1;
        sh.zx_t = load1<TT>(tbuf, x - g.j0);
        sh.zx_d = load1<DT>(dbuf, x - g.j0);
      }
    }
    if (KD) {
      if (!skip) {
        cta_topk<TT>(tbuf, g, st_t.mz, prm.K, sh, cand, prm.status);
      } else {
        if ((int)threadIdx.x < kMaxK) sh.topk[threadIdx.x] = kNoKey;
        __syncthreads();
      }
    }
    cluster.sync();  // #1: partials visible

    // 2. combine + acceptance test: warp 0 of every CTA, lane q reading CTA q.
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      float Gt = -INFINITY, Gd = -INFINITY, zt = 0.f, zd = 0.f;
      double St = 0.0, Sd = 0.0;
      int hx = 0, tmo = 0, skp = 0;
      if (lane < C) {
        const RowShared* o = cluster.map_shared_rank(&sh, lane);
        Gt = o->G_t;
        St = o->S_t;
        if (DKIND == kDraftLogits && has_draft) {
          Gd = o->G_d;
          Sd = o->S_d;
        }
        hx = o->has_x;
        zt = o->zx_t;
        zd = o->zx_d;
        tmo = o->timeouts;
        skp = o->skip;
      }
      const int nxt = cluster.map_shared_rank(&sh, 0)->next_item;
      float Gm;
      double Sm;
      warp_stat_combine(Gt, St, &Gm, &Sm);
      const unsigned hmask = __ballot_sync(0xffffffffu, hx != 0);
      const int src = hmask ? __ffs(hmask) - 1 : 0;
      zt = __shfl_sync(0xffffffffu, zt, src);
      zd = __shfl_sync(0xffffffffu, zd, src);
      tmo = warp_sum_int(tmo);
      const bool rowskip = __any_sync(0xffffffffu, skp != 0);
      float Gdm = 0.f;
      double Sdm = 1.0;
      if (DKIND == kDraftLogits && has_draft) warp_stat_combine(Gd, Sd, &Gdm, &Sdm);
      if (lane == 0) {
        sh.item = nxt;
        sh.rowskip = rowskip ? 1 : 0;
        int err = 0;
        int accept = 1;
        sh.Gt = Gm;
        sh.St = Sm;
        sh.Lt = (double)Gm + log2(Sm);
        sh.Gd = Gdm;
        sh.Sd = Sdm;
        sh.Ld = 0.0;
        if (!rowskip) {
          if (Gm == -INFINITY) err |= SV_DEV_NO_FINITE;
          if (DKIND == kDraftLogits && has_draft) {
            if (Gdm == -INFINITY) err |= SV_DEV_NO_FINITE;
            sh.Ld = (double)Gdm + log2(Sdm);
          }
          if (has_draft && (x < 0 || x >= V || hmask == 0u)) err |= SV_DEV_BAD_TOKEN;
          if (tmo) err |= SV_DEV_TIMEOUT;
          if (has_draft && !err) {
            const double px = exp2((double)zt * (double)c - sh.Lt);
            const double qx = (DKIND == kDraftLogits) ? exp2((double)zd * (double)c - sh.Ld)
                                                      : (double)zd;
            const double u = (double)prm.u[(size_t)b * P + i];
            accept = (u * qx < px) ? 1 : 0;
          }
        }
        sh.accept = accept;
        sh.err = err;
        sh.need = (!rowskip && !err && (!has_draft || !accept)) ? 1 : 0;
        if (rank == 0) {
          if (err) set_status(prm.status, err);
          if (!rowskip && has_draft && !accept && !err)
            atomicMax(&prm.ws.req_reject[b], (uint32_t)(k - i));
        }
      }
    }
    __syncthreads();

    // 4a. fused KD (rank 0): merge the cluster's top-K while the other CTAs
    // compute their residual weights.
    if (KD && rank == 0 && !sh.rowskip) {
      unsigned long long* out = cand + kCandCap - kMaxK;
      cluster_topk_merge(cluster, C, prm.K, sh, cand, out);
      const int lane = threadIdx.x & 31;
      if (threadIdx.x < 32) {
        const int K = prm.K;
        const double ln2 = 0.69314718055994530942;
        const size_t orow = (size_t)b * P + i;
        double lp = -INFINITY;
        int j = -1;
        if (lane < K) {
          const unsigned long long kk = out[lane];
          j = key_index(kk);
          lp = ((double)key_value(kk) * (double)c - sh.Lt) * ln2;
          prm.topk_logp[orow * K + lane] = sh.err ? NAN : (float)lp;
          prm.topk_idx[orow * K + lane] = j;
        }
        if (lane == 0) prm.lse[orow] = sh.err ? NAN : (float)(sh.Lt * ln2);
        if (has_draft) {
          double m = lp;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
          double s = (lane < K) ? exp(lp - m) : 0.0;
          s = warp_sum(s);
          const double lse_k = m + log(s);
          double term = 0.0;
          if (lane < K && !sh.err && j >= 0 && j < V) {
            const int owner = j / prm.L;
            const unsigned char* rb = cluster.map_shared_rank(dbuf, owner);
            const float zdj = load1<DT>(rb, j - owner * prm.L);
            const double log_pt = lp - lse_k;
            const double pt = exp(log_pt);
            const double log_q = (DKIND == kDraftLogits)
                                     ? ((double)zdj * (double)c - sh.Ld) * ln2
                                     : log((double)zdj);
            term = (pt == 0.0) ? 0.0 : pt * (log_pt - log_q);
          }
          term = warp_sum(term);
          if (lane == 0) prm.kl[(size_t)b * k + i] = sh.err ? NAN : (float)term;
        }
      }
      __syncthreads();
    }

    // 3. sampling pass.
    if (sh.need) {
      int mode = has_draft ? kModeResidual : kModeP;
      const float Gt = sh.Gt, Gd = sh.Gd;
      const float invSt = (float)(1.0 / sh.St);
      const float invSd = (float)(1.0 / sh.Sd);
      for (int attempt = 0; attempt < 2; ++attempt) {
        for (int p = 0; p < g.npieces; ++p) {
          const int e = p * kRound + (int)threadIdx.x * kVec;
          float s = 0.f;
          if (e < g.nvec * kVec) {
            float w[8];
            weights8<TT, DT, DKIND>(tbuf, dbuf, e, mode, c, Gt, invSt, Gd, invSd, w);
            s = seq_sum8(w);
          }
          sums[p * kThreads + threadIdx.x] = s;
        }
        piece_totals(sums, g.npieces, sh);
        if (threadIdx.x == 0) {
          double Rc = 0.0;
          for (int p = 0; p < g.npieces; ++p) Rc += sh.ptot[p];
          sh.R = Rc;
        }
        cluster.sync();  // #2: chunk masses visible
        if (threadIdx.x < 32) {
          // chunk q owns [incl(q-1), incl(q)) of the row's cumulative mass; the
          // scan runs in the same order in every CTA.
          const int lane = threadIdx.x;
          const double Rq = lane < C ? cluster.map_shared_rank(&sh, lane)->R : 0.0;
          const double incl = warp_scan_incl(Rq);
          const double R = __shfl_sync(0xffffffffu, incl, 31);
          const double lo = __shfl_sync(0xffffffffu, incl, rank > 0 ? rank - 1 : 0);
          const double hi = __shfl_sync(0xffffffffu, incl, rank);
          if (lane == 0) {
            const double myO = rank > 0 ? lo : 0.0;
            const double tt = (double)prm.u[(size_t)b * P + k] * R;
            sh.tt = tt;
            sh.base = myO;
            sh.redo = (R == 0.0 && mode == kModeResidual) ? 1 : 0;
            sh.owner = (R > 0.0 && myO <= tt && tt < hi) ? 1 : 0;
          }
        }
        __syncthreads();
        if (!sh.redo) break;
        if (rank == 0 && threadIdx.x == 0) set_status(prm.status, SV_DEV_RESIDUAL_ZERO);
        mode = kModeP;
        cluster.sync();  // nobody still reads sh.R of the first attempt
      }
      if (sh.owner) {
        // Locate the piece, then the thread, then the element.
        if (threadIdx.x == 0) {
          double base = sh.base;
          int pp = -1;
          for (int p = 0; p < g.npieces; ++p) {
            if (base + sh.ptot[p] > sh.tt) {
              pp = p;
              break;
            }
            base += sh.ptot[p];
          }
          if (pp < 0) {  // rounding pushed the target past this chunk: last piece with mass
            double b2 = sh.base;
            base = sh.base;
            for (int p = 0; p < g.npieces; ++p) {
              if (sh.ptot[p] > 0.0) {
                pp = p;
                base = b2;
              }
              b2 += sh.ptot[p];
            }
          }
          sh.piece = pp;
          sh.base = base;
          sh.first_thread = kThreads;
          sh.last_pos = -1;
          sh.tok = -1;
        }
        __syncthreads();
        const int pp = sh.piece;
        if (pp >= 0) {
          const float s = sums[pp * kThreads + threadIdx.x];
          double tot;
          const double incl = block_scan_incl((double)s, sh.redd, &tot);
          double* incl_arr = reinterpret_cast<double*>(sums + g.npieces * kThreads);
          incl_arr[threadIdx.x] = incl;
          if (sh.base + incl > sh.tt) atomicMin(&sh.first_thread, (int)threadIdx.x);
          if (s > 0.f) atomicMax(&sh.last_pos, (int)threadIdx.x);
          __syncthreads();
          int ts = sh.first_thread;
          const bool fb = (ts == kThreads);
          if (fb) ts = sh.last_pos;
          if ((int)threadIdx.x == ts) {
            const int e = pp * kRound + ts * kVec;
            float w[8];
            weights8<TT, DT, DKIND>(tbuf, dbuf, e, mode, c, Gt, invSt, Gd, invSd, w);
            const double b0 = sh.base + (ts > 0 ? incl_arr[ts - 1] : 0.0);
            float a = 0.f;
            int pick = -1, lastq = -1;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              a = __fadd_rn(a, w[q]);
              if (w[q] > 0.f) lastq = q;
              if (!fb && pick < 0 && b0 + (double)a > sh.tt) pick = q;
            }
            if (pick < 0) pick = lastq;
            sh.tok = (pick < 0) ? -1 : g.j0 + e + pick;
          }
          __syncthreads();
        }
        if (threadIdx.x == 0 && sh.tok >= 0) {
          prm.ws.row_b[(size_t)b * P + i] = sh.tok + 1;
          __threadfence();
        }
      }
    }

    // 4b. row result (rank 0).
    if (rank == 0 && threadIdx.x == 0) {
      int res = kRowAccepted;
      if (sh.rowskip) res = kRowSkipped;
      else if (sh.err) res = kRowError;
      else if (has_draft && !sh.accept) res = kRowRejected;
      prm.ws.row_a[(size_t)b * P + i] = res;
    }
    cluster.sync();  // final: no CTA reads another's shared memory of this item after this

    // 5. request finalize by the last of its P rows.
    if (rank == 0 && arrive_last(&prm.ws.req_counter[b], (uint32_t)P, sh))
      chain_finalize(prm, b, KD, sh, reinterpret_cast<int*>(sums));
    item = sh.item;
  }
  cluster_retire(prm.ws, rank, C);
}

// ---------------------------------------------------------------------------
// Greedy chain (T == 0): argmax per target row, same persistent scheme.
// ---------------------------------------------------------------------------
template <class TT>
__device__ __forceinline__ unsigned long long chunk_argmax_key(RowShared& sh,
                                                               const unsigned char* buf,
                                                               const ChunkGeom& g,
                                                               bool use_bulk, uint32_t phase) {
  float best = -INFINITY;
  int bidx = -1;
  for (int p = 0; p < g.npieces; ++p) {
    if (!wait_piece(sh, p, use_bulk, phase)) break;
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

template <class TT>
__global__ void __launch_bounds__(kThreads) chain_greedy_kernel(const ArgmaxParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* tbuf = smem + prm.lay.off_t;
  const int P = prm.R, k = P - 1, B = prm.B, V = prm.V, total = B * P;
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const bool use_bulk = prm.use_bulk != 0;
  uint64_t policy = 0;
  uint32_t phase = 0;
  if (threadIdx.x == 0) {
    init_piece_barriers(sh, g, use_bulk);
    if (use_bulk) policy = policy_evict_first();
    if (rank == 0) sh.first_item = (int)atomicAdd(prm.ws.work, 1u);
  }
  cluster.sync();
  if (threadIdx.x == 0) sh.item = cluster.map_shared_rank(&sh, 0)->first_item;
  __syncthreads();
  int item = sh.item;
  while (item < total) {
    const int i = item / B, b = item - i * B;
    const void* trow = row_ptr<TT>(prm.logits, (size_t)b * P + i, V);
    if (threadIdx.x == 0) {
      if (rank == 0) sh.next_item = (int)atomicAdd(prm.ws.work, 1u);
      sh.skip = load_relaxed(&prm.ws.req_reject[b]) > (uint32_t)(k - i) ? 1 : 0;
      sh.timeouts = 0;
      if (use_bulk && !sh.skip)
        issue_item_copies<TT, TT, false>(sh, tbuf, nullptr, trow, nullptr, g, policy);
    }
    __syncthreads();
    const bool skip = sh.skip != 0;
    if (!skip) scalar_fill<TT>(tbuf, trow, g, use_bulk, false);
    __syncthreads();
    unsigned long long key = kNoKey;
    if (!skip) key = chunk_argmax_key<TT>(sh, tbuf, g, use_bulk, phase);
    if (threadIdx.x == 0) sh.key = key;
    if (!skip && use_bulk) {
      drain_pieces(sh, g, use_bulk, phase);
      phase ^= 1u;
    }
    cluster.sync();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      unsigned long long best = kNoKey;
      int tmo = 0, skp = 0;
      if (lane < C) {
        const RowShared* o = cluster.map_shared_rank(&sh, lane);
        best = o->key;
        tmo = o->timeouts;
        skp = o->skip;
      }
      const int nxt = cluster.map_shared_rank(&sh, 0)->next_item;
      best = warp_max_u64(best);
      tmo = warp_sum_int(tmo);
      const bool rowskip = __any_sync(0xffffffffu, skp != 0);
      if (lane == 0) {
        sh.item = nxt;
        if (rank == 0) {
          const int gi = key_index(best);
          int res, val = 0;
          if (rowskip) {
            res = kRowSkipped;
          } else if (tmo) {
            set_status(prm.status, SV_DEV_TIMEOUT);
            res = kRowError;
          } else if (i < k) {
            const int x = prm.tokens[(size_t)b * k + i];
            if (x < 0 || x >= V) {
              set_status(prm.status, SV_DEV_BAD_TOKEN);
              res = kRowError;
            } else {
              res = (x == gi) ? kRowAccepted : kRowRejected;
              if (x != gi) atomicMax(&prm.ws.req_reject[b], (uint32_t)(k - i));
            }
            val = gi + 1;
          } else {
            res = kRowAccepted;
            val = gi + 1;
          }
          prm.ws.row_a[(size_t)b * P + i] = res;
          prm.ws.row_b[(size_t)b * P + i] = val;
        }
      }
    }
    __syncthreads();
    cluster.sync();
    if (rank == 0 && arrive_last(&prm.ws.req_counter[b], (uint32_t)P, sh)) {
      // first rejection, then the argmax stored at that row
      int* fa = reinterpret_cast<int*>(smem + prm.lay.off_x);
      int* fc = fa + kThreads;
      for (int t = threadIdx.x; t < P; t += kThreads) {
        const size_t r = (size_t)b * P + t;
        fa[t] = __ldcg(&prm.ws.row_a[r]);
        fc[t] = __ldcg(&prm.ws.row_b[r]);
        prm.ws.row_a[r] = 0;
        prm.ws.row_b[r] = 0;
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int n = k;
        for (int t = 0; t < k; ++t)
          if (fa[t] == kRowRejected) {
            n = t;
            break;
          }
        int bad = 0;
        for (int t = 0; t <= n; ++t) bad |= (fa[t] != kRowAccepted && fa[t] != kRowRejected);
        const int tk = fc[n] - 1;
        if (tk < 0 || tk >= V) bad = 1;
        sh.fin_n = bad ? -1 : n;
        sh.fin_tok = tk;
        prm.accepted_len[b] = sh.fin_n;
        prm.ws.req_counter[b] = 0u;
        prm.ws.req_reject[b] = 0u;
      }
      __syncthreads();
      const int n = sh.fin_n;
      for (int t = threadIdx.x; t < P; t += kThreads) {
        int v = -1;
        if (n >= 0) v = (t < n) ? prm.tokens[(size_t)b * k + t] : (t == n ? sh.fin_tok : -1);
        prm.out_tokens[(size_t)b * P + t] = v;
      }
    }
    item = sh.item;
  }
  cluster_retire(prm.ws, rank, C);
}

// ---------------------------------------------------------------------------
// Launchers: as many clusters as can be resident (each loops over items).
// ---------------------------------------------------------------------------
template <class K, class Prm>
static cudaError_t launch_persistent(K kernel, const Prm& prm, const RowPlan& plan, int items,
                                     cudaStream_t s) {
  const void* kp = reinterpret_cast<const void*>(kernel);
  cudaError_t e = ensure_kernel_attrs(kp, plan.lay.bytes, plan.C > 8);
  if (e != cudaSuccess) return e;
  int nres = 0;
  e = max_active_clusters(kp, plan.lay.bytes, plan.C, &nres);
  if (e != cudaSuccess) return e;
  if (nres < 1) return cudaErrorInvalidConfiguration;
  const int ncl = nres < items ? nres : items;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ncl * (unsigned)plan.C, 1, 1);
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

template <class TT, class DT, int DKIND>
static cudaError_t launch_sample_t(const ChainParams& p, const RowPlan& plan, bool kd,
                                   cudaStream_t s) {
  const int n = p.B * (p.k + 1);
  if (kd) return launch_persistent(chain_sample_kernel<TT, DT, DKIND, true>, p, plan, n, s);
  return launch_persistent(chain_sample_kernel<TT, DT, DKIND, false>, p, plan, n, s);
}

cudaError_t launch_chain_sample(const ChainParams& p, const RowPlan& plan, int t_dtype,
                                int d_dtype, int d_kind, bool kd, cudaStream_t s) {
  if (d_kind == kDraftProbs) {
    if (t_dtype == SV_BF16) return launch_sample_t<BF16, F32, kDraftProbs>(p, plan, kd, s);
    return launch_sample_t<F32, F32, kDraftProbs>(p, plan, kd, s);
  }
  if (t_dtype == SV_BF16) {
    if (d_dtype == SV_BF16) return launch_sample_t<BF16, BF16, kDraftLogits>(p, plan, kd, s);
    return launch_sample_t<BF16, F32, kDraftLogits>(p, plan, kd, s);
  }
  if (d_dtype == SV_BF16) return launch_sample_t<F32, BF16, kDraftLogits>(p, plan, kd, s);
  return launch_sample_t<F32, F32, kDraftLogits>(p, plan, kd, s);
}

cudaError_t launch_chain_greedy(const ArgmaxParams& p, const RowPlan& plan, int dtype,
                                cudaStream_t s) {
  const int n = p.B * p.R;
  if (dtype == SV_BF16) return launch_persistent(chain_greedy_kernel<BF16>, p, plan, n, s);
  return launch_persistent(chain_greedy_kernel<F32>, p, plan, n, s);
}

}  // namespace sv
