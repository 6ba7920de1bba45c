// sv_chain.cu -- chain verification kernels.
//
// One C-CTA cluster per (request b, position i): target row i and, for
// i < k, draft row i, split into C chunks that stay resident in shared memory.
// Clusters are ordered position-major (all i = 0 first) so that a later
// position usually starts after the earlier ones of its request finished;
// a row that sees an earlier rejection of its request skips its resample.
//
// Per cluster (sampling, T > 0):
//   1. stage chunks; online max / sum-of-exp2 per thread -> per CTA;
//      optional CTA top-K of the target chunk (fused KD)
//   2. cluster barrier; every CTA combines the C partials in the same order
//      (identical bits everywhere) and evaluates the acceptance test
//      u * q(x) < p(x) in float64
//   3. if this row must be sampled (first rejection candidate, or the bonus
//      row): residual weights max(0, p - q) (or p) per piece from shared
//      memory, cluster barrier, chunk offsets, inverse-CDF search inside the
//      owning CTA
//   4. rank 0: fused KD (cluster top-K merge, lse, KL against the draft row
//      gathered from the resident chunks), row result
//   5. final cluster barrier; the last row of each request to finish writes
//      the request's outputs (and the KD loss; the last request the total).
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
#pragma unroll
  for (int t = 0; t < 8; ++t) p[t] = ex2(fmaf(zt[t], c, -Gt)) * invSt;
  if (mode == kModeResidual) {
    float q[8];
    if (DKIND == kDraftLogits) {
      float zd[8];
      load8<DT>(dbuf, e, zd);
#pragma unroll
      for (int t = 0; t < 8; ++t) q[t] = ex2(fmaf(zd[t], c, -Gd)) * invSd;
    } else {
      load8<F32>(dbuf, e, q);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = fmaxf(p[t] - q[t], 0.f);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) w[t] = p[t];
  }
}

__device__ __forceinline__ float seq_sum8(const float w[8]) {
  float s = w[0];
#pragma unroll
  for (int t = 1; t < 8; ++t) s += w[t];
  return s;
}

template <class TT, class DT, int DKIND, bool KD>
__global__ void __launch_bounds__(kThreads) chain_sample_kernel(const ChainParams prm) {
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
  const int pair = (int)(blockIdx.x / (unsigned)C);
  const int i = pair / B, b = pair - i * B;
  const bool has_draft = i < k;
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const float c = prm.c;
  const bool use_bulk = prm.use_bulk != 0;
  const void* trow = row_ptr<TT>(prm.target, (size_t)b * P + i, V);
  const void* drow = has_draft ? row_ptr<DT>(prm.draft, (size_t)b * k + i, V) : nullptr;
  const int x = has_draft ? prm.tokens[(size_t)b * k + i] : -1;

  // 1. stage and stream.
  if (has_draft)
    stage_chunks<TT, DT, true>(sh, tbuf, dbuf, trow, drow, g, use_bulk, DKIND == kDraftProbs);
  else
    stage_chunks<TT, DT, false>(sh, tbuf, dbuf, trow, drow, g, use_bulk, false);

  ThreadStat st_t, st_d;
  stat_init(st_t);
  stat_init(st_d);
  for (int p = 0; p < g.npieces; ++p) {
    if (!wait_piece(sh, p, use_bulk)) break;
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
  {
    const CtaStat cs = stat_block(st_t, sh.redf, sh.redd);
    if (threadIdx.x == 0) {
      sh.G_t = cs.G;
      sh.S_t = cs.S;
    }
  }
  if (DKIND == kDraftLogits && has_draft) {
    const CtaStat cs = stat_block(st_d, sh.redf, sh.redd);
    if (threadIdx.x == 0) {
      sh.G_d = cs.G;
      sh.S_d = cs.S;
    }
  }
  if (threadIdx.x == 0) {
    sh.has_x = 0;
    if (has_draft && x >= g.j0 && x < g.j0 + g.len) {
      sh.has_x = 1;
      sh.zx_t = load1<TT>(tbuf, x - g.j0);
      sh.zx_d = load1<DT>(dbuf, x - g.j0);
    }
    sh.skip = 0;
    if (rank == 0) {
      const uint32_t wrd = *reinterpret_cast<volatile uint32_t*>(&prm.ws.req_reject[b]);
      sh.skip = wrd > (uint32_t)(k - i) ? 1 : 0;
    }
  }
  if (KD) cta_topk<TT>(tbuf, g, st_t.mz, prm.K, sh, cand, prm.status);
  cluster.sync();  // #1: partials visible

  // 2. combine + acceptance test (thread 0 of every CTA, same bits everywhere).
  if (threadIdx.x == 0) {
    float Gs[kMaxCluster], Gd[kMaxCluster];
    double Ss[kMaxCluster], Sd[kMaxCluster];
    float zx_t = 0.f, zx_d = 0.f;
    int found = 0, tmo = 0;
    for (int q = 0; q < C; ++q) {
      const RowShared* o = cluster.map_shared_rank(&sh, q);
      Gs[q] = o->G_t;
      Ss[q] = o->S_t;
      if (DKIND == kDraftLogits && has_draft) {
        Gd[q] = o->G_d;
        Sd[q] = o->S_d;
      }
      if (o->has_x) {
        found = 1;
        zx_t = o->zx_t;
        zx_d = o->zx_d;
      }
      tmo += o->timeouts;
    }
    const RowShared* r0 = cluster.map_shared_rank(&sh, 0);
    const int skip = r0->skip;
    int err = 0;
    stat_combine(Gs, Ss, C, &sh.Gt, &sh.St);
    if (sh.Gt == -INFINITY) err |= SV_DEV_NO_FINITE;
    sh.Lt = (double)sh.Gt + log2(sh.St);
    if (DKIND == kDraftLogits && has_draft) {
      stat_combine(Gd, Sd, C, &sh.Gd, &sh.Sd);
      if (sh.Gd == -INFINITY) err |= SV_DEV_NO_FINITE;
      sh.Ld = (double)sh.Gd + log2(sh.Sd);
    } else {
      sh.Gd = 0.f;
      sh.Sd = 1.0;
      sh.Ld = 0.0;
    }
    if (has_draft && (x < 0 || x >= V || !found)) err |= SV_DEV_BAD_TOKEN;
    if (tmo) err |= SV_DEV_TIMEOUT;
    int accept = 1;
    if (has_draft && !err) {
      const double px = exp2((double)zx_t * (double)c - sh.Lt);
      const double qx = (DKIND == kDraftLogits) ? exp2((double)zx_d * (double)c - sh.Ld)
                                                : (double)zx_d;
      const double u = (double)prm.u[(size_t)b * P + i];
      accept = (u * qx < px) ? 1 : 0;
    }
    sh.accept = accept;
    sh.err = err;
    sh.need = (!err && !skip && (!has_draft || !accept)) ? 1 : 0;
    if (rank == 0) {
      if (err) set_status(prm.status, err);
      if (has_draft && !accept && !err) atomicMax(&prm.ws.req_reject[b], (uint32_t)(k - i));
    }
  }
  __syncthreads();

  // 4a. fused KD, part 1 (rank 0): merge the cluster's top-K while the other
  // CTAs compute their residual weights.
  if (KD && rank == 0) {
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
        const float z = key_value(kk);
        lp = ((double)z * (double)c - sh.Lt) * ln2;
        prm.topk_logp[orow * K + lane] = (float)lp;
        prm.topk_idx[orow * K + lane] = j;
      }
      if (lane == 0) prm.lse[orow] = (float)(sh.Lt * ln2);
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
          const float zd = load1<DT>(rb, j - owner * prm.L);
          const double log_pt = lp - lse_k;
          const double pt = exp(log_pt);
          const double log_q = (DKIND == kDraftLogits) ? ((double)zd * (double)c - sh.Ld) * ln2
                                                       : log((double)zd);
          term = (pt == 0.0) ? 0.0 : pt * (log_pt - log_q);
        }
        term = warp_sum(term);
        if (lane == 0) prm.kl[(size_t)b * k + i] = sh.err ? NAN : (float)term;
      }
    }
    __syncthreads();
  }

  // 3. sampling pass.
  int tok = -1;
  if (sh.need) {
    int mode = has_draft ? kModeResidual : kModeP;
    const float Gt = sh.Gt, Gd = sh.Gd;
    const float invSt = (float)(1.0 / sh.St);
    const float invSd = (float)(1.0 / sh.Sd);
    double myO = 0.0, tt = 0.0, Rc = 0.0;
    // Clear the row's token before barrier #2: the owning CTA writes it after.
    if (rank == 0 && threadIdx.x == 0) prm.ws.row_b[(size_t)b * P + i] = -1;
    for (int attempt = 0; attempt < 2; ++attempt) {
      Rc = 0.0;
      for (int p = 0; p < g.npieces; ++p) {
        const int e = p * kRound + (int)threadIdx.x * kVec;
        float s = 0.f;
        if (e < g.nvec * kVec) {
          float w[8];
          weights8<TT, DT, DKIND>(tbuf, dbuf, e, mode, c, Gt, invSt, Gd, invSd, w);
          s = seq_sum8(w);
        }
        sums[p * kThreads + threadIdx.x] = s;
        double tot;
        block_scan_incl((double)s, sh.redd, &tot);
        if (threadIdx.x == 0) sh.ptot[p] = tot;
        Rc += tot;
      }
      if (threadIdx.x == 0) sh.R = Rc;
      cluster.sync();  // #2: chunk masses visible
      if (threadIdx.x == 0) {
        double O = 0.0;
        for (int q = 0; q < C; ++q) {
          if (q == rank) myO = O;
          O += cluster.map_shared_rank(&sh, q)->R;
        }
        const double R = O;
        tt = (double)prm.u[(size_t)b * P + k] * R;
        sh.tt = tt;
        sh.base = myO;
        sh.redo = (R == 0.0 && mode == kModeResidual) ? 1 : 0;
        sh.owner = (R > 0.0 && myO <= tt && tt < myO + Rc) ? 1 : 0;
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
            a += w[q];
            if (w[q] > 0.f) lastq = q;
            if (!fb && pick < 0 && b0 + (double)a > sh.tt) pick = q;
          }
          if (pick < 0) pick = lastq;
          sh.tok = (pick < 0) ? -1 : g.j0 + e + pick;
        }
        __syncthreads();
      }
      if (threadIdx.x == 0) {
        tok = sh.tok;
        prm.ws.row_b[(size_t)b * P + i] = tok;
        __threadfence();
      }
    }
  }

  // 4b. row result (rank 0).
  if (rank == 0 && threadIdx.x == 0) {
    prm.ws.row_a[(size_t)b * P + i] = sh.err ? -1 : sh.accept;
    if (!sh.need) prm.ws.row_b[(size_t)b * P + i] = -1;
  }
  drain_pieces(sh, g, use_bulk);
  cluster.sync();  // final: no CTA reads another's shared memory after this
  if (rank != 0) return;

  // 5. request finalize by the last of its P rows.
  if (!arrive_last(&prm.ws.req_counter[b], (uint32_t)P, sh)) return;
  int* fa = reinterpret_cast<int*>(sums);
  int* fc = fa + kThreads;
  for (int t = threadIdx.x; t < P; t += kThreads) {
    fa[t] = __ldcg(&prm.ws.row_a[(size_t)b * P + t]);
    fc[t] = __ldcg(&prm.ws.row_b[(size_t)b * P + t]);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = k, bad = 0;
    for (int t = 0; t < P; ++t) bad |= (fa[t] < 0);
    for (int t = 0; t < k; ++t)
      if (fa[t] == 0) {
        n = t;
        break;
      }
    const int tk = fc[n];
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
  if (KD)
    kd_finalize(b, n, B, k, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip, prm.loss,
                prm.total, prm.ws.glob_counter, sh);
}

// ---------------------------------------------------------------------------
// Greedy chain (T == 0): argmax per target row.
// ---------------------------------------------------------------------------
template <class TT>
__device__ __forceinline__ unsigned long long chunk_argmax_key(RowShared& sh,
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

template <class TT>
__global__ void __launch_bounds__(kThreads) chain_greedy_kernel(const ArgmaxParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* tbuf = smem + prm.lay.off_t;
  const int P = prm.R, k = P - 1, B = prm.B, V = prm.V;
  const int row = (int)(blockIdx.x / (unsigned)C);
  const int i = row / B, b = row - i * B;
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const bool use_bulk = prm.use_bulk != 0;
  stage_chunks<TT, TT, false>(sh, tbuf, nullptr, row_ptr<TT>(prm.logits, (size_t)b * P + i, V),
                              nullptr, g, use_bulk, false);
  const unsigned long long key = chunk_argmax_key<TT>(sh, tbuf, g, use_bulk);
  if (threadIdx.x == 0) sh.key = key;
  drain_pieces(sh, g, use_bulk);
  cluster.sync();
  if (rank == 0 && threadIdx.x == 0) {
    unsigned long long best = kNoKey;
    int tmo = 0;
    for (int q = 0; q < C; ++q) {
      const RowShared* o = cluster.map_shared_rank(&sh, q);
      best = o->key > best ? o->key : best;
      tmo += o->timeouts;
    }
    const int gi = key_index(best);
    int res;
    if (tmo) {
      set_status(prm.status, SV_DEV_TIMEOUT);
      res = -1;
    } else if (i < k) {
      const int x = prm.tokens[(size_t)b * k + i];
      if (x < 0 || x >= V) {
        set_status(prm.status, SV_DEV_BAD_TOKEN);
        res = -1;
      } else {
        res = (x == gi) ? 1 : 0;
      }
    } else {
      res = 1;
    }
    prm.ws.row_a[(size_t)b * P + i] = res;
    prm.ws.row_b[(size_t)b * P + i] = gi;
  }
  cluster.sync();
  if (rank != 0) return;
  if (!arrive_last(&prm.ws.req_counter[b], (uint32_t)P, sh)) return;
  if (threadIdx.x == 0) {
    int n = k, bad = 0;
    for (int t = 0; t < P; ++t) bad |= (__ldcg(&prm.ws.row_a[(size_t)b * P + t]) < 0);
    for (int t = 0; t < k; ++t)
      if (__ldcg(&prm.ws.row_a[(size_t)b * P + t]) == 0) {
        n = t;
        break;
      }
    sh.fin_n = bad ? -1 : n;
    sh.fin_tok = __ldcg(&prm.ws.row_b[(size_t)b * P + n]);
    prm.accepted_len[b] = sh.fin_n;
    prm.ws.req_counter[b] = 0u;
  }
  __syncthreads();
  const int n = sh.fin_n;
  for (int t = threadIdx.x; t < P; t += kThreads) {
    int v = -1;
    if (n >= 0) v = (t < n) ? prm.tokens[(size_t)b * k + t] : (t == n ? sh.fin_tok : -1);
    prm.out_tokens[(size_t)b * P + t] = v;
  }
}

// ---------------------------------------------------------------------------
// Launchers.
// ---------------------------------------------------------------------------
template <class K, class Prm>
static cudaError_t launch_cluster(K kernel, const Prm& prm, const RowPlan& plan, int nclusters,
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

template <class TT, class DT, int DKIND>
static cudaError_t launch_sample_t(const ChainParams& p, const RowPlan& plan, bool kd,
                                   cudaStream_t s) {
  const int n = p.B * (p.k + 1);
  if (kd) return launch_cluster(chain_sample_kernel<TT, DT, DKIND, true>, p, plan, n, s);
  return launch_cluster(chain_sample_kernel<TT, DT, DKIND, false>, p, plan, n, s);
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
  if (dtype == SV_BF16) return launch_cluster(chain_greedy_kernel<BF16>, p, plan, n, s);
  return launch_cluster(chain_greedy_kernel<F32>, p, plan, n, s);
}

}  // namespace sv
