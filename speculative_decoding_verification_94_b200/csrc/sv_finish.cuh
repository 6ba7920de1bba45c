// sv_finish.cuh -- the finishing pass of every entry point (after the stream).
//
// Chain sampling: one C-CTA cluster per request reads the request's row
// records, finds the first rejection n (or n = k), and draws the emitted token
// from the one row pair that needs it: residual max(0, p_n - q_n) or, for
// n = k, the bonus row p_k, by inverse CDF in ascending vocabulary order.  The
// row pair is staged in shared memory (bulk copies), the CTA chunk masses are
// combined in a fixed order through distributed shared memory and the owning
// CTA locates the draw.  Fused KD rows were written by the stream; the
// finisher marks the rows after the emitted position as undefined and forms
// the reward-weighted losses.  Every finisher returns the row records it read
// to zero (the stream zeroes the partials), so the workspace stays zero
// between calls.
#include "sv_rowops.cuh"
#include "sv_stream.cuh"

namespace sv {

enum { kModeResidual = 0, kModeP = 1 };

struct FinishParams {
  // rows (chain: target [B, k+1, V], draft [B, k, V]; tree: logits [B, n, V])
  const void* target;
  const void* draft;
  const int32_t* tokens;   // chain: [B, k]; tree: node tokens [B, n]
  const int32_t* parents;  // tree
  const float* u;
  int B, k, V, L, nchunk, K;
  int max_depth;
  float c;
  int use_bulk;
  RowLayout lay;
  // outputs
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* accepted_nodes;
  float* topk_logp;
  int32_t* topk_idx;
  float* lse;
  float* kl;
  const float* reward;
  int wmode, group;
  float clip;
  float* loss;
  float* total;
  // KL-loss inputs (standalone)
  const float* in_topk_logp;
  const int32_t* in_topk_idx;
  const int32_t* in_accepted_len;
  int draft_probs;
  // stream scratch
  Partial* part;
  unsigned long long* cand;
  RowRec* rec;
  uint32_t* req_reject;
  uint32_t* glob_counter;
  int32_t* status;
  // the stream's parameters: rows it did not complete (sp.count == 0) are
  // completed here first
  StreamParams sp;
};

// Stream flags of the sampling chain (they fix what a row completion does).
template <int DKIND, bool KD>
constexpr int chain_sample_flags() {
  return kFStats0 | kFGather | (DKIND == kDraftLogits ? (kFRow1 | kFStats1) : 0) |
         (KD ? kFTopk0 : 0);
}

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

// First rejection of request b from its row records (one warp, all lanes
// return the same): n, and whether every row that decides the outcome
// (0..n) was verified.
__device__ __forceinline__ int warp_first_rejection(const RowRec* rec, int B, int k, int b,
                                                    bool* bad) {
  const int lane = threadIdx.x & 31;
  int n = k;
  for (int base = 0; base < k; base += 32) {
    const int t = base + lane;
    const int code = t < k ? __ldcg(&rec[(size_t)t * B + b].code) : 0;
    const unsigned m = __ballot_sync(0xffffffffu, t < k && code == kRowRejected);
    if (m) {
      n = base + __ffs(m) - 1;
      break;
    }
  }
  bool bd = false;
  for (int base = 0; base <= n; base += 32) {
    const int t = base + lane;
    const int code = t <= n ? __ldcg(&rec[(size_t)t * B + b].code) : kRowAccepted;
    bd |= __any_sync(0xffffffffu, code != kRowAccepted && code != kRowRejected);
  }
  *bad = bd;
  return n;
}

// Zero the row records of rows r0, r0 + stride_rows, ... (nr rows) with
// threads t0, t0 + nt, ...
__device__ __forceinline__ void zero_recs(const FinishParams& p, size_t r0, int stride_rows,
                                          int nr, int t0, int nt) {
  for (int q = t0; q < nr; q += nt) p.rec[r0 + (size_t)q * stride_rows] = RowRec{};
}

template <class TT, class DT, int DKIND, bool KD>
__global__ void __launch_bounds__(kThreads) chain_sample_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  unsigned char* tbuf = smem + prm.lay.off_t;
  unsigned char* dbuf = smem + prm.lay.off_d;
  float* sums = reinterpret_cast<float*>(smem + prm.lay.off_x);
  const int k = prm.k, P = k + 1, B = prm.B, V = prm.V;
  const int b = (int)(blockIdx.x / (unsigned)C);
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const float c = prm.c;
  const bool use_bulk = prm.use_bulk != 0;

  // 0. rows 0..k of the request, when the stream left them to this kernel
  if (!prm.sp.count) {
    const int w = threadIdx.x >> 5;
    for (int t = rank * kWarps + w; t < P; t += C * kWarps)
      row_complete<TT, DT, chain_sample_flags<DKIND, KD>()>(
          prm.sp, t * B + b, t < k ? prm.tokens[(size_t)b * k + t] : -1);
    if (threadIdx.x == 0) __threadfence();
    cluster.sync();
  }

  if (threadIdx.x < 32) {
    bool bad;
    const int n = warp_first_rejection(prm.rec, B, k, b, &bad);
    if (threadIdx.x == 0) {
      sh.fin_n = bad ? -1 : n;
      sh.need = bad ? 0 : 1;
      sh.err = 0;
      // cleared before the draw's first cluster barrier; the owning CTA writes it after
      if (rank == 0 && !bad) prm.out_tokens[(size_t)b * P + n] = -1;
      const RowRec* rn = &prm.rec[(size_t)n * B + b];
      sh.Gt = __ldcg(&rn->G0);
      sh.St = __ldcg(&rn->S0);
      sh.Gd = __ldcg(&rn->G1);
      sh.Sd = __ldcg(&rn->S1);
      sh.tok = -1;
    }
  }
  __syncthreads();
  const int n = sh.fin_n;

  // 1. the draw, from row pair n (residual) or the bonus row k (target only).
  if (sh.need) {
    const bool pair = n < k;
    const void* trow = row_ptr<TT>(prm.target, (size_t)b * P + n, V);
    const void* drow = pair ? row_ptr<DT>(prm.draft, (size_t)b * k + n, V) : nullptr;
    if (pair)
      stage_chunks<TT, DT, true>(sh, tbuf, dbuf, trow, drow, g, use_bulk, DKIND == kDraftProbs);
    else
      stage_chunks<TT, DT, false>(sh, tbuf, dbuf, trow, drow, g, use_bulk, false);
    for (int p = 0; p < g.npieces; ++p) wait_piece(sh, p, use_bulk);
    __syncthreads();
    int mode = pair ? kModeResidual : kModeP;
    const float Gt = sh.Gt, Gd = sh.Gd;
    const float invSt = (float)(1.0 / sh.St);
    const float invSd = (DKIND == kDraftLogits && pair) ? (float)(1.0 / sh.Sd) : 1.f;
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
      cluster.sync();  // chunk masses visible
      if (threadIdx.x < 32) {
        // chunk q owns [incl(q-1), incl(q)) of the cumulative mass; the scan
        // runs in the same order in every CTA.
        const int lane = threadIdx.x;
        const double Rq = lane < C ? cluster.map_shared_rank(&sh, lane)->R : 0.0;
        const double incl = warp_scan_incl(Rq);
        const double R = __shfl_sync(0xffffffffu, incl, 31);
        const double lo = __shfl_sync(0xffffffffu, incl, rank > 0 ? rank - 1 : 0);
        const double hi = __shfl_sync(0xffffffffu, incl, rank);
        const int tmo = warp_sum_int(lane < C ? cluster.map_shared_rank(&sh, lane)->timeouts : 0);
        if (lane == 0) {
          const double myO = rank > 0 ? lo : 0.0;
          const double tt = (double)prm.u[(size_t)b * P + k] * R;
          sh.tt = tt;
          sh.base = myO;
          sh.redo = (R == 0.0 && mode == kModeResidual && !tmo) ? 1 : 0;
          sh.owner = (R > 0.0 && !tmo && myO <= tt && tt < hi) ? 1 : 0;
          if (tmo && rank == 0) set_status(prm.status, SV_DEV_TIMEOUT);
          sh.err = tmo ? 1 : 0;
        }
      }
      __syncthreads();
      if (!sh.redo) break;
      if (rank == 0 && threadIdx.x == 0) set_status(prm.status, SV_DEV_RESIDUAL_ZERO);
      mode = kModeP;
      cluster.sync();  // nobody still reads sh.R of the first attempt
    }
    if (sh.owner) {
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
      if (threadIdx.x == 0) prm.out_tokens[(size_t)b * P + n] = sh.tok;
    }
  }

  // 2. fused KD: the stream wrote rows 0..n; later rows are not verified and
  // are defined as empty.
  if (KD) {
    // rows after the emitted position: not verified, defined as empty
    if (rank == 0) {
      const int first_undef = n < 0 ? 0 : n + 1;
      for (int t = first_undef * prm.K + (int)threadIdx.x; t < P * prm.K; t += kThreads) {
        prm.topk_logp[(size_t)b * P * prm.K + t] = NAN;
        prm.topk_idx[(size_t)b * P * prm.K + t] = -1;
      }
      for (int t = first_undef + (int)threadIdx.x; t < P; t += kThreads)
        prm.lse[(size_t)b * P + t] = NAN;
      for (int t = first_undef + (int)threadIdx.x; t < k; t += kThreads)
        prm.kl[(size_t)b * k + t] = NAN;
    }
  }
  if (threadIdx.x == 0) __threadfence();
  cluster.sync();  // draw, KD rows and every read of the records are done

  // 3. outputs (rank 0) and workspace hygiene (every CTA).
  zero_recs(prm, (size_t)b, B, P, rank * kThreads + (int)threadIdx.x, C * kThreads);
  if (rank != 0) return;
  if (threadIdx.x == 0) {
    int nn = n;
    if (nn >= 0 && sh.need && sh.err) nn = -1;
    if (nn >= 0) {
      const int tk = __ldcg(&prm.out_tokens[(size_t)b * P + nn]);
      if (tk < 0 || tk >= V) nn = -1;
    }
    sh.fin_n = nn;
    prm.accepted_len[b] = nn;
    prm.req_reject[b] = 0u;
  }
  __syncthreads();
  const int nf = sh.fin_n;
  for (int t = threadIdx.x; t < P; t += kThreads) {
    if (nf >= 0 && t == nf) continue;  // the drawn token, written by the owning CTA
    const int v = (nf >= 0 && t < nf) ? prm.tokens[(size_t)b * k + t] : -1;
    prm.out_tokens[(size_t)b * P + t] = v;
  }
  if (KD)
    kd_finalize(b, nf, B, k, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip, prm.loss,
                prm.total, prm.glob_counter, sh);
}

// Greedy chain: one block per request (its warps complete the request's rows
// when the stream left them; warp 0 takes the decision).
template <class T>
__global__ void __launch_bounds__(kThreads) chain_greedy_finish(const __grid_constant__ FinishParams prm) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int b = (int)blockIdx.x;
  const int k = prm.k, P = k + 1, B = prm.B;
  if (!prm.sp.count) {
    for (int t = w; t < P; t += kWarps)
      row_complete<T, T, kFArgmax0>(prm.sp, t * B + b, t < k ? prm.tokens[(size_t)b * k + t] : -1);
    __threadfence();
    __syncthreads();
  }
  if (w != 0) return;
  bool bad = false;
  const int n = warp_first_rejection(prm.rec, B, k, b, &bad);
  const int tok = __ldcg(&prm.rec[(size_t)n * B + b].argmax);
  if (tok < 0 || tok >= prm.V) bad = true;
  for (int t = lane; t < P; t += 32) {
    int v = -1;
    if (!bad) v = (t < n) ? prm.tokens[(size_t)b * k + t] : (t == n ? tok : -1);
    prm.out_tokens[(size_t)b * P + t] = v;
  }
  __syncwarp();
  zero_recs(prm, (size_t)b, B, P, lane, 32);
  if (lane == 0) {
    prm.accepted_len[b] = bad ? -1 : n;
    prm.req_reject[b] = 0u;
  }
}

// Greedy tree: one block per request; node rows are rows b * n + j.
template <class T>
__global__ void __launch_bounds__(kThreads) tree_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  const int n = prm.k, V = prm.V;
  const int b = (int)blockIdx.x;
  if (!prm.sp.count) {
    for (int t = threadIdx.x >> 5; t < n; t += kWarps)
      row_complete<T, T, kFArgmax0>(prm.sp, b * n + t, -1);
    __threadfence();
    __syncthreads();
  }
  int* garg = reinterpret_cast<int*>(smem + kFixedBytes);
  int* par = garg + n;
  int* tok = par + n;
  int* dep = tok + n;
  int err_any = 0;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    const RowRec* r = &prm.rec[(size_t)b * n + t];
    const int code = __ldcg(&r->code);
    garg[t] = code == kRowAccepted ? __ldcg(&r->argmax) : -1;
    err_any |= (code != kRowAccepted);
    par[t] = prm.parents[(size_t)b * n + t];
    tok[t] = prm.tokens[(size_t)b * n + t];
  }
  err_any = __syncthreads_or(err_any);
  const int W = prm.max_depth + 1;
  if (threadIdx.x == 0) {
    int bad = (par[0] != -1) || err_any;
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
      const bool a = dep[pj] >= 0 && tok[t] == garg[pj];
      dep[t] = a ? d : -(d + 1);
      if (a && d > dep[best]) best = t;
    }
    if (bad == 1 && !err_any) set_status(prm.status, SV_DEV_BAD_TREE);
    sh.fin_n = bad ? -1 : dep[best];
    sh.fin_tok = best;
    prm.accepted_len[b] = sh.fin_n;
  }
  __syncthreads();
  const int Lb = sh.fin_n, best = sh.fin_tok;
  if (threadIdx.x == 0) {
    int32_t* on = prm.accepted_nodes + (size_t)b * W;
    int32_t* ot = prm.out_tokens + (size_t)b * W;
    for (int d = 0; d < W; ++d) on[d] = ot[d] = -1;
    if (Lb >= 0) {
      for (int t = best, d = Lb; d >= 0; t = par[t], --d) on[d] = t;
      for (int d = 0; d < Lb; ++d) ot[d] = tok[on[d + 1]];
      ot[Lb] = garg[best];
    }
  }
  zero_recs(prm, (size_t)b * n, 1, n, threadIdx.x, kThreads);
}

// KD loss: one block per request, one warp per draft row (b, i < k).  Draft
// rows stream first (logits) so that rec holds their normalisers; probability
// drafts have no stream pass.
template <class DT>
__global__ void __launch_bounds__(kThreads) kl_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int b = (int)blockIdx.x;
  const int k = prm.k, P = k + 1, B = prm.B, V = prm.V, K = prm.K;
  if (!prm.draft_probs && !prm.sp.count) {
    for (int t = w; t < k; t += kWarps) row_complete<DT, DT, kFStats0>(prm.sp, b * k + t, -1);
    __threadfence();
    __syncthreads();
  }
  const double ln2 = 0.69314718055994530942;
  const double c = (double)prm.c;
  for (int i = w; i < k; i += kWarps) {
    const size_t trow = (size_t)b * P + i;
    const size_t drow = (size_t)b * k + i;
    double lp = -INFINITY;
    int j = -1;
    if (lane < K) {
      lp = (double)prm.in_topk_logp[trow * K + lane];
      j = prm.in_topk_idx[trow * K + lane];
    }
    const int badj = __any_sync(0xffffffffu, lane < K && (j < 0 || j >= V));
    double L1 = 0.0;
    int err = 0;
    if (!prm.draft_probs) {
      const int code = __ldcg(&prm.rec[drow].code);
      L1 = __ldcg(&prm.rec[drow].L0);
      if (code != kRowAccepted) err = 1;
    }
    double m = lp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    double s = (lane < K) ? exp(lp - m) : 0.0;
    s = warp_sum(s);
    const double lse_k = m + log(s);
    double term = 0.0;
    if (lane < K && !badj && !err) {
      const double log_pt = lp - lse_k;
      const double pt = exp(log_pt);
      double log_q;
      const float zd = load1<DT>(
          reinterpret_cast<const unsigned char*>(row_ptr<DT>(prm.draft, drow, V)), j);
      log_q = prm.draft_probs ? log((double)zd) : ((double)zd * c - L1) * ln2;
      term = (pt == 0.0) ? 0.0 : pt * (log_pt - log_q);
    }
    term = warp_sum(term);
    if (lane == 0) {
      if (badj) set_status(prm.status, SV_DEV_BAD_INDEX);
      prm.kl[drow] = (badj || err) ? NAN : (float)term;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = prm.in_accepted_len[b];
    if (n < 0 || n > k) {
      set_status(prm.status, SV_DEV_BAD_INDEX);
      n = -1;
    }
    sh.fin_n = n;
  }
  __syncthreads();
  if (!prm.draft_probs) zero_recs(prm, (size_t)b * k, 1, k, threadIdx.x, kThreads);
  kd_finalize(b, sh.fin_n, B, k, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip, prm.loss,
              prm.total, prm.glob_counter, sh);
}

}  // namespace sv
