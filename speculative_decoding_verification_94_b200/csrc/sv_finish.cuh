// sv_finish.cuh -- the finishing pass of every entry point (after the stream).
//
// Chain sampling: one C-CTA cluster per request folds (static schedule) or
// reads (dynamic schedule) the request's row records, finds the first
// rejection n (or n = k_b, the request's draft count), and draws the emitted
// token from the one row pair that needs it: residual max(0, p_n - q_n) or,
// for n = k_b, the bonus row p_{k_b}, by inverse CDF in ascending vocabulary
// order.  The row pair is staged in shared memory (bulk copies), the CTA
// chunk masses are combined in a fixed order through distributed shared
// memory and the owning CTA locates the draw.  Fused KD rows are written here
// (static schedule) or were written by the stream (dynamic); the finisher
// marks the rows after the emitted position as undefined and forms the
// reward-weighted losses.  Every finisher returns the stream state it read
// (the static schedule's records, or the dynamic schedule's row records) to
// zero, so the workspace stays zero between calls.
#pragma once

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
  double c64;  // log2(e) / T in float64 (sampling trees)
  int use_bulk;
  int nsplit;  // kd_grad_kernel: CTAs per draft row
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
  int positions;  // KD positions (sv_kd_args.positions)
  // KD gradient (sv_kd_grad)
  float* grad;
  float temperature;
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

// Eight consecutive elements j..j+7 of a row in global memory, widened to
// fp32; elements at or past jend read as `pad`.  vec: the row base is 16-byte
// aligned and j a multiple of 8, so a full vector is one 16-byte load (two for
// fp32).  The rows are read-only inputs, so the loads take the read-only path.
template <class T>
__device__ __forceinline__ void gload8(const void* row, int j, int jend, bool vec, float pad,
                                       float v[8]);

template <>
__device__ __forceinline__ void gload8<BF16>(const void* row, int j, int jend, bool vec, float pad,
                                             float v[8]) {
  const uint16_t* src = static_cast<const uint16_t*>(row) + j;
  if (vec && j + 8 <= jend) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src));
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t)
      v[t] = j + t < jend ? __uint_as_float((uint32_t)__ldg(src + t) << 16) : pad;
  }
}

template <>
__device__ __forceinline__ void gload8<F32>(const void* row, int j, int jend, bool vec, float pad,
                                            float v[8]) {
  const float* src = static_cast<const float*>(row) + j;
  if (vec && j + 8 <= jend) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(src));
    const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = j + t < jend ? __ldg(src + t) : pad;
  }
}

// Draw weights of eight vocabulary entries from their target values zt and
// draft values zd (draft logits, or draft probabilities): the residual
// max(0, p - q), or p itself (mode P, where zd is not read).
template <int DKIND>
__device__ __forceinline__ void weights8(const float zt[8], const float zd[8], int mode, float c,
                                         float Gt, float invSt, float Gd, float invSd,
                                         float w[8]) {
  float p[8];
  // explicitly rounded products: p - q must be exactly 0 when p == q
#pragma unroll
  for (int t = 0; t < 8; ++t) p[t] = __fmul_rn(ex2(fmaf(zt[t], c, -Gt)), invSt);
  if (mode == kModeResidual) {
    float q[8];
    if (DKIND == kDraftLogits) {
#pragma unroll
      for (int t = 0; t < 8; ++t) q[t] = __fmul_rn(ex2(fmaf(zd[t], c, -Gd)), invSd);
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) q[t] = zd[t];
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

// The request's rows in shared memory (rows[t] = row t of the request):
// folded here from the stream's records (static schedule), or read from the
// records the stream completed (dynamic schedule).  Warp w takes rows w, w + 8,
// ...; every caller in a cluster does this redundantly (no barrier needed).
// Returns nothing; rows[] is valid after the caller's __syncthreads.
template <class T0, class T1, int FLAGS>
__device__ __forceinline__ void load_rows(const FinishParams& prm, RowRec* rows, int nrows,
                                          int row0, int row_stride, const int32_t* xs, int nx,
                                          bool report) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const bool stat = !prm.sp.count;
  for (int t = w; t < nrows; t += kWarps) {
    const int r = row0 + t * row_stride;
    const int x = t < nx ? xs[t] : -1;
    RowRec rr;
    if (stat) {
      const RowSum s = row_combine<T0, T1, FLAGS>(prm.sp, r, x, true);
      int err = 0;
      rr = row_decide<FLAGS>(prm.sp, r, x, s, &err);
      if (err && report && lane == 0) set_status(prm.status, err);
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(prm.rec + r);
      uint4 q[3];
      q[0] = __ldcg(src);
      q[1] = __ldcg(src + 1);
      q[2] = __ldcg(src + 2);
      memcpy(&rr, q, sizeof(RowRec));
    }
    if (lane == 0) rows[t] = rr;
  }
}

// First rejection n of a chain (one warp; all lanes return the same) and
// whether every row that decides the outcome (0..n) was verified.
__device__ __forceinline__ int first_rejection(const RowRec* rows, int k, bool* bad) {
  const int lane = threadIdx.x & 31;
  int n = k;
  for (int base = 0; base < k; base += 32) {
    const int t = base + lane;
    const unsigned m = __ballot_sync(0xffffffffu, t < k && rows[t].code == kRowRejected);
    if (m) {
      n = base + __ffs(m) - 1;
      break;
    }
  }
  bool bd = false;
  for (int base = 0; base <= n; base += 32) {
    const int t = base + lane;
    const int code = t <= n ? rows[t].code : kRowAccepted;
    bd |= __any_sync(0xffffffffu, code != kRowAccepted && code != kRowRejected);
  }
  *bad = bd;
  return n;
}

// The rows' stream state back to zero: the records of the static schedule,
// or the row records of the dynamic one.  Rows t = t0, t0 + nt, ... (warps).
__device__ __forceinline__ void release_rows(const FinishParams& prm, int nrows, int row0,
                                             int row_stride, int t0, int nt) {
  const int lane = threadIdx.x & 31;
  for (int t = t0; t < nrows; t += nt) {
    const int r = row0 + t * row_stride;
    if (!prm.sp.count) {
      row_zero_records(prm.sp, r, true);
      if (lane == 0) prm.sp.row_counter[r] = 0u;  // the top-K floor of the row
    } else if (lane == 0) {
      prm.rec[r] = RowRec{};
    }
  }
}

// Chain sampling: one cluster of C CTAs per request.
//   0. rows 0..k in every CTA (load_rows); warp 0 finds the first rejection n;
//   1. fused KD (static schedule): the rows' top-K outputs for rows 0..n,
//      spread over the cluster's warps; later rows' lists are cleared;
//   2. the draw from the one row pair that needs it (residual at n < k, bonus
//      row at n = k), staged by bulk copies, chunk masses scanned in a fixed
//      order through distributed shared memory (the one cluster barrier);
//   3. the rows' stream state back to zero (after the barrier: no CTA still
//      reads it);
//   4. the CTA that owns the drawn token writes the request's outputs (the
//      first CTA when there is no draw: failed rows or timeouts).
// STAGED: the drawn row's chunk is copied to shared memory first (one CTA per
// SM, the registers it wants); otherwise it is read from global memory and
// four CTAs share an SM.
template <class TT, class DT, int DKIND, bool KD, bool STAGED>
__global__ void __launch_bounds__(kThreads, STAGED ? 1 : 4)
    chain_sample_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  RowRec* rows = reinterpret_cast<RowRec*>(smem + prm.lay.off_rows);
  unsigned char* tbuf = smem + prm.lay.off_t;
  unsigned char* dbuf = smem + prm.lay.off_d;
  float* sums = reinterpret_cast<float*>(smem + prm.lay.off_x);
  const int k = prm.k, P = k + 1, B = prm.B, V = prm.V;
  const int b = (int)(blockIdx.x / (unsigned)C);
  const ChunkGeom g = chunk_geom(rank, prm.L, V);
  const float c = prm.c;
  const bool use_bulk = prm.use_bulk != 0;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  constexpr int RF = chain_sample_flags<DKIND, KD>();
  if (threadIdx.x == 0) sh.tok = -1;
  pdl_wait();  // the stream's records are complete

  // 0. the request's rows 0..k_b and its first rejection (k_b < 0: an
  //    inactive request or an invalid draft count: no row)
  const int kb = req_kb(prm.sp, b);
  const int nld = kb < 0 ? 0 : kb + 1;
  load_rows<TT, DT, RF>(prm, rows, nld, b, B, prm.tokens + (size_t)b * k, nld - 1, rank == 0);
  __syncthreads();
  if (w == 0) {
    bool bad = true;
    const int n = kb < 0 ? 0 : first_rejection(rows, kb, &bad);
    if (lane == 0) {
      sh.fin_n = bad ? -1 : n;
      sh.need = bad ? 0 : 1;
      sh.err = 0;
      sh.owner = 0;
      if (!bad) {
        sh.Gt = rows[n].G0;
        sh.St = rows[n].S0;
        sh.Gd = rows[n].G1;
        sh.Sd = rows[n].S1;
      }
      if (kb == -2 && rank == 0) set_status(prm.status, SV_DEV_BAD_LEN);
    }
  }
  __syncthreads();
  const int n = sh.fin_n;
  // Direct reads: this CTA's chunk of the drawn row (pair) starts towards L2
  // now, so that its latency overlaps the KD rows below and the pass's loads
  // find it there.
  if (!STAGED && sh.need && use_bulk && threadIdx.x == 0 && g.len > 0) {
    const uint32_t tb = (uint32_t)(g.len * TT::bytes) & ~15u;
    if (tb) bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(
                                 row_ptr<TT>(prm.target, (size_t)b * P + n, V)) + (size_t)g.j0 * TT::bytes,
                             tb);
    const uint32_t dbytes = (uint32_t)(g.len * DT::bytes) & ~15u;
    if (n < kb && dbytes)
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(
                           row_ptr<DT>(prm.draft, (size_t)b * k + n, V)) + (size_t)g.j0 * DT::bytes,
                       dbytes);
  }

  // 2. the draw, from row pair n (residual) or the bonus row k_b (target only).
  //    Staged: the chunk is copied to shared memory first.  Otherwise (when
  //    staging would leave clusters waiting for a second wave) it is read
  //    straight from global memory into registers and only the per-thread
  //    piece sums are kept; the owner of the drawn token re-reads one vector.
  bool arrived = false;
  if (sh.need) {
    const bool pair = n < kb;
    const void* trow = row_ptr<TT>(prm.target, (size_t)b * P + n, V);
    const void* drow = pair ? row_ptr<DT>(prm.draft, (size_t)b * k + n, V) : nullptr;
    constexpr bool staged = STAGED;
    if (staged) {
      if (pair)
        stage_chunks<TT, DT, true>(sh, tbuf, dbuf, trow, drow, g, use_bulk, DKIND == kDraftProbs);
      else
        stage_chunks<TT, DT, false>(sh, tbuf, dbuf, trow, drow, g, use_bulk, false);
      for (int p = 0; p < g.npieces; ++p) wait_piece(sh, p, use_bulk);
    } else if (threadIdx.x == 0) {
      sh.timeouts = 0;
    }
    __syncthreads();
    const int jend = g.j0 + g.len;
    const float dpad = DKIND == kDraftProbs ? 0.f : -INFINITY;
    int mode = pair ? kModeResidual : kModeP;
    const float Gt = sh.Gt, Gd = sh.Gd;
    const float invSt = (float)(1.0 / sh.St);
    const float invSd = (DKIND == kDraftLogits && pair) ? (float)(1.0 / sh.Sd) : 1.f;
    // the weights of this thread's vector of piece p
    auto piece_weights = [&](int p, float wv[8]) -> bool {
      const int e = p * kRound + (int)threadIdx.x * kVec;
      if (e >= g.nvec * kVec) return false;
      float zt[8], zd[8];
      if (staged) {
        load8<TT>(tbuf, e, zt);
        if (mode == kModeResidual) load8<DT>(dbuf, e, zd);
      } else {
        gload8<TT>(trow, g.j0 + e, jend, use_bulk, -INFINITY, zt);
        if (mode == kModeResidual) gload8<DT>(drow, g.j0 + e, jend, use_bulk, dpad, zd);
      }
      weights8<DKIND>(zt, zd, mode, c, Gt, invSt, Gd, invSd, wv);
      return true;
    };
    for (int attempt = 0; attempt < 2; ++attempt) {
      // four pieces at a time: their loads are in flight together
      for (int p0 = 0; p0 < g.npieces; p0 += 4) {
        float s4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float wv[8];
          s4[u] = (p0 + u < g.npieces && piece_weights(p0 + u, wv)) ? seq_sum8(wv) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (p0 + u < g.npieces) sums[(p0 + u) * kThreads + threadIdx.x] = s4[u];
      }
      piece_totals(sums, g.npieces, sh);
      if (threadIdx.x == 0) {
        double Rc = 0.0;
        for (int p = 0; p < g.npieces; ++p) Rc += sh.ptot[p];
        sh.R = Rc;
      }
      cluster.sync();  // chunk masses visible; every CTA has read the rows' records
      if (w == 0) {
        // chunk q owns [incl(q-1), incl(q)) of the cumulative mass; the scan
        // runs in the same order in every CTA.
        const double Rq = lane < C ? cluster.map_shared_rank(&sh, lane)->R : 0.0;
        const double incl = warp_scan_incl(Rq);
        const double R = __shfl_sync(0xffffffffu, incl, 31);
        const double lo = __shfl_sync(0xffffffffu, incl, rank > 0 ? rank - 1 : 0);
        const double hi = __shfl_sync(0xffffffffu, incl, rank);
        const int tmo = warp_sum_int(lane < C ? cluster.map_shared_rank(&sh, lane)->timeouts : 0);
        if (lane == 0) {
          const double myO = rank > 0 ? lo : 0.0;
          const double tt = (double)prm.u[(size_t)b * P + kb] * R;
          sh.tt = tt;
          sh.base = myO;
          sh.redo = (R == 0.0 && mode == kModeResidual && !tmo) ? 1 : 0;
          sh.owner = (R > 0.0 && !tmo && myO <= tt && tt < hi) ? 1 : 0;
          if (tmo && rank == 0) set_status(prm.status, SV_DEV_TIMEOUT);
          sh.err = (tmo || !(R > 0.0)) ? 1 : 0;
        }
      }
      __syncthreads();
      cluster_arrive_release();  // done with the other CTAs' shared memory
      arrived = true;
      if (!sh.redo) break;
      if (rank == 0 && threadIdx.x == 0) set_status(prm.status, SV_DEV_RESIDUAL_ZERO);
      mode = kModeP;
      cluster_wait_acquire();  // nobody still reads sh.R of the first attempt
      arrived = false;
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
          float wv[8];
          piece_weights(pp, wv);
          const double b0 = sh.base + (ts > 0 ? incl_arr[ts - 1] : 0.0);
          float a = 0.f;
          int pick = -1, lastq = -1;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            a = __fadd_rn(a, wv[q]);
            if (wv[q] > 0.f) lastq = q;
            if (!fb && pick < 0 && b0 + (double)a > sh.tt) pick = q;
          }
          if (pick < 0) pick = lastq;
          sh.tok = (pick < 0) ? -1 : g.j0 + e + pick;
        }
        __syncthreads();
      }
    }
  } else {
    cluster.sync();  // every CTA has read the rows' records
  }

  // 3. fused KD outputs, by rank 0 after the draw, so that no CTA of the
  //    cluster waits at the scan for them: the top-K and KL of rows 0..n
  //    (static schedule; the dynamic schedule wrote them in the stream), the
  //    other rows' lists cleared, the rows after the emitted position filled
  //    as empty, and the request's loss.  The emitted position is the one the
  //    owner reports: n unless the request failed or the draw did (the owner
  //    rejects a located token outside [0, V) too, which a draw with positive
  //    mass cannot produce).
  if (KD && rank == 0) {
    const int nf = (n >= 0 && sh.need && !sh.err) ? n : -1;
    if (!prm.sp.count) {
      for (int t = w; t < P; t += kWarps) {
        const bool ld = t < nld;
        row_outputs<TT, DT, RF>(prm.sp, t * B + b, t < kb ? prm.tokens[(size_t)b * k + t] : -1,
                                ld ? rows[t].L0 : 0.0, ld ? rows[t].L1 : 0.0, 0,
                                n >= 0 && t <= n, true);
      }
      __syncthreads();
    }
    // rows after the emitted position are not verified: defined as empty
    const int first_undef = nf < 0 ? 0 : nf + 1;
    for (int t = first_undef * prm.K + (int)threadIdx.x; t < P * prm.K; t += kThreads) {
      prm.topk_logp[(size_t)b * P * prm.K + t] = NAN;
      prm.topk_idx[(size_t)b * P * prm.K + t] = -1;
    }
    for (int t = first_undef + (int)threadIdx.x; t < P; t += kThreads)
      prm.lse[(size_t)b * P + t] = NAN;
    // draft rows past the request's own drafts (k_b <= k) have no KL either
    const int kl_undef = min(first_undef, kb < 0 ? 0 : kb);
    for (int t = kl_undef + (int)threadIdx.x; t < k; t += kThreads)
      prm.kl[(size_t)b * k + t] = NAN;
    __syncthreads();
    kd_finalize(b, nf, B, k, kb, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip,
                prm.positions, prm.loss, prm.total, prm.glob_counter, sh);
  }

  // 4. the rows' stream state back to zero
  release_rows(prm, P, b, B, rank * kWarps + w, C * kWarps);

  // 5. outputs, by the owner of the drawn token (or the first CTA without a draw)
  const bool writer = sh.need ? (sh.owner != 0 || (sh.err && rank == 0)) : rank == 0;
  if (writer) {
    if (threadIdx.x == 0) {
      int nn = n;
      if (nn >= 0 && (!sh.need || sh.err)) nn = -1;
      if (nn >= 0 && (sh.tok < 0 || sh.tok >= V)) nn = -1;
      sh.fin_n = nn;
      prm.accepted_len[b] = kb == -1 ? 0 : nn;  // an inactive request accepts nothing
      prm.req_reject[b] = 0u;
    }
    __syncthreads();
    const int nf = sh.fin_n;
    for (int t = threadIdx.x; t < P; t += kThreads) {
      int v = -1;
      if (nf >= 0) v = t < nf ? prm.tokens[(size_t)b * k + t] : (t == nf ? sh.tok : -1);
      prm.out_tokens[(size_t)b * P + t] = v;
    }
  }
  if (arrived) cluster_wait_acquire();  // keep this CTA's shared memory until all have read it
}

// Greedy chain: one block per request.
template <class T>
__global__ void __launch_bounds__(kThreads) chain_greedy_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  RowRec* rows = reinterpret_cast<RowRec*>(smem + kFixedBytes);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int b = (int)blockIdx.x;
  const int k = prm.k, P = k + 1, B = prm.B;
  pdl_wait();
  const int kb = req_kb(prm.sp, b);  // rows 0..k_b (none when k_b < 0)
  const int nld = kb < 0 ? 0 : kb + 1;
  load_rows<T, T, kFArgmax0>(prm, rows, nld, b, B, prm.tokens + (size_t)b * k, nld - 1, true);
  __syncthreads();
  if (w == 0) {
    bool bad = true;
    const int n = kb < 0 ? 0 : first_rejection(rows, kb, &bad);
    const int tok = kb < 0 ? -1 : rows[n].argmax;
    if (tok < 0 || tok >= prm.V) bad = true;
    if (kb == -2 && lane == 0) set_status(prm.status, SV_DEV_BAD_LEN);
    for (int t = lane; t < P; t += 32) {
      int v = -1;
      if (!bad) v = (t < n) ? prm.tokens[(size_t)b * k + t] : (t == n ? tok : -1);
      prm.out_tokens[(size_t)b * P + t] = v;
    }
    if (lane == 0) {
      prm.accepted_len[b] = kb == -1 ? 0 : (bad ? -1 : n);
      prm.req_reject[b] = 0u;
    }
  }
  __syncthreads();  // (every warp has read the rows' state)
  release_rows(prm, P, b, B, w, kWarps);
}

// Greedy tree: one block per request; node rows are rows b * n + j.
template <class T>
__global__ void __launch_bounds__(kThreads) tree_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  const int n = prm.k, V = prm.V;
  // nsplit blocks per tree: each folds its share of the node rows (a warp a
  // row) into the row records in global memory; the last to finish walks
  // the tree.  One block folds every row itself.
  const int S = prm.nsplit > 1 ? prm.nsplit : 1;
  const int b = (int)blockIdx.x / S, s = (int)blockIdx.x - b * S;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  RowRec* rows = reinterpret_cast<RowRec*>(smem + kFixedBytes);
  int* garg = reinterpret_cast<int*>(smem + kFixedBytes + (size_t)n * sizeof(RowRec));
  int* par = garg + n;
  int* tok = par + n;
  int* dep = tok + n;
  pdl_wait();
  if (S == 1) {
    load_rows<T, T, kFArgmax0>(prm, rows, n, b * n, 1, nullptr, 0, true);
  } else {
    for (int t = s * kWarps + w; t < n; t += S * kWarps) {
      const int r = b * n + t;
      const RowSum rs = row_combine<T, T, kFArgmax0>(prm.sp, r, -1, true);
      int err = 0;
      const RowRec rr = row_decide<kFArgmax0>(prm.sp, r, -1, rs, &err);
      if (err && lane == 0) set_status(prm.status, err);
      row_zero_records(prm.sp, r, true);
      if (lane == 0) prm.rec[r] = rr;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();  // this block's row records before its arrival
      const int last = atomicAdd(&prm.req_reject[b], 1u) == (uint32_t)(S - 1) ? 1 : 0;
      if (last) __threadfence();  // the other blocks' records before the reads below
      sh.owner = last;
    }
    __syncthreads();
    if (!sh.owner) return;
    for (int t = threadIdx.x; t < n; t += kThreads) {
      const uint4* src = reinterpret_cast<const uint4*>(prm.rec + (size_t)b * n + t);
      uint4 q[3];
      q[0] = __ldcg(src);
      q[1] = __ldcg(src + 1);
      q[2] = __ldcg(src + 2);
      memcpy(&rows[t], q, sizeof(RowRec));
      prm.rec[(size_t)b * n + t] = RowRec{};  // the workspace back to zero
    }
    if (threadIdx.x == 0) prm.req_reject[b] = 0u;
  }
  __syncthreads();
  int err_any = 0;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    const int code = rows[t].code;
    garg[t] = code == kRowAccepted ? rows[t].argmax : -1;
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
  if (S == 1) release_rows(prm, n, b * n, 1, threadIdx.x >> 5, kWarps);
}

// KD loss: one block per request, one warp per draft row (b, i < k).  Draft
// logit rows are folded from the stream's records first; probability drafts
// have no stream pass.
template <class DT>
__global__ void __launch_bounds__(kThreads) kl_finish(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  RowRec* rows = reinterpret_cast<RowRec*>(smem + kFixedBytes);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int b = (int)blockIdx.x;
  const int k = prm.k, P = k + 1, B = prm.B, V = prm.V, K = prm.K;
  const double ln2 = 0.69314718055994530942;
  const double c = (double)prm.c;
  pdl_wait();
  if (!prm.draft_probs) load_rows<DT, DT, kFStats0>(prm, rows, k, b * k, 1, nullptr, 0, true);
  __syncthreads();
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
      L1 = rows[i].L0;
      if (rows[i].code != kRowAccepted) err = 1;
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
  if (!prm.draft_probs) release_rows(prm, k, b * k, 1, w, kWarps);
  kd_finalize(b, sh.fin_n, B, k, k, prm.kl, prm.reward, prm.wmode, prm.group, prm.clip,
              prm.positions, prm.loss, prm.total, prm.glob_counter, sh);
}

// Gradient of the reward-weighted KD loss with respect to the draft logits:
// one block per draft row (b, i).  grad = w_b (q - p~ [j in K]) / T for
// i < n_b (zero otherwise), q = softmax(z / T) from the row's folded
// statistics: q_j = 2^((z_j c - G) - log2 S), the exact integer reference G
// taken first so that the float argument stays small.
template <class DT>
__global__ void __launch_bounds__(kThreads) kd_grad_kernel(const __grid_constant__ FinishParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  // nsplit CTAs per draft row, each a range of whole 8-element vectors, so
  // that the grid has enough items to fill the last wave
  const int nsplit = prm.nsplit > 0 ? prm.nsplit : 1;
  const int row = (int)blockIdx.x / nsplit, part = (int)blockIdx.x - row * nsplit;
  const int k = prm.k, P = k + 1, V = prm.V, K = prm.K;
  const int b = row / k, i = row - b * k;
  const int Lp = ((V + nsplit - 1) / nsplit + kVec - 1) / kVec * kVec;
  const int lo = min(V, part * Lp), hi = min(V, lo + Lp);
  float* g = prm.grad + (size_t)row * V;
  pdl_wait();
  if (w == 0) {
    const int n = prm.in_accepted_len[b];
    const double wb = reward_weight(prm.reward, b, prm.wmode, prm.group, prm.clip);
    const int npos = (prm.positions && n >= 0 && n < k) ? n + 1 : n;  // KD positions
    int active = (n >= 0 && n <= k && i < npos && wb != 0.0) ? 1 : 0;
    if (n < 0 || n > k) {
      if (lane == 0 && i == 0) set_status(prm.status, SV_DEV_BAD_INDEX);
    }
    // the row's statistics (every draft row was streamed)
    const RowSum st = row_combine<DT, DT, kFStats0>(prm.sp, row, -1, true);
    // the last of the row's CTAs to have folded its records clears them
    // (the row's counter word counts the folds and returns to zero)
    int last = 1;
    if (nsplit > 1) {
      __syncwarp();
      if (lane == 0) {
        __threadfence();  // this CTA's reads of the records before its count
        last = atomicAdd(&prm.sp.row_counter[row], 1u) == (uint32_t)(nsplit - 1) ? 1 : 0;
        if (last) __threadfence();  // the other CTAs' reads before the clearing
      }
      last = __shfl_sync(0xffffffffu, last, 0);
    }
    if (last) {
      row_zero_records(prm.sp, row, true);
      if (lane == 0 && nsplit > 1) prm.sp.row_counter[row] = 0u;
    }
    int bad = st.G0 == -INFINITY || (st.flags & kPTimeout);
    if (active && bad && lane == 0)
      set_status(prm.status, (st.flags & kPTimeout) ? SV_DEV_TIMEOUT : SV_DEV_NO_FINITE);
    // p~ over the kept entries of target row (b, i)
    double lp = -INFINITY;
    int j = -1;
    if (lane < K) {
      lp = (double)prm.in_topk_logp[((size_t)b * P + i) * K + lane];
      j = prm.in_topk_idx[((size_t)b * P + i) * K + lane];
    }
    const int badj = __any_sync(0xffffffffu, lane < K && (j < 0 || j >= V));
    if (active && badj && lane == 0) set_status(prm.status, SV_DEV_BAD_INDEX);
    double m = lp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    double se = (lane < K) ? exp(lp - m) : 0.0;
    se = warp_sum(se);
    const double pt = (lane < K) ? exp(lp - (m + log(se))) : 0.0;
    if (lane == 0) {
      sh.need = active ? (bad || badj ? 2 : 1) : 0;  // 0: zeros, 1: gradient, 2: NaN
      sh.Gt = st.G0;
      sh.St = log2(st.S0);  // log2 S, the fractional part of the log2-partition
      sh.R = wb / (double)prm.temperature;
    }
    if (lane < 32) {  // the kept entries' p~, for the fix-up below
      sh.topk[lane] = (lane < K) ? ((unsigned long long)(uint32_t)j << 32) |
                                       (unsigned long long)__float_as_uint((float)pt)
                                 : 0ull;
    }
  }
  __syncthreads();
  const int mode = sh.need;
  const float c = prm.c, G = sh.Gt, l2s = (float)sh.St, scale = (float)sh.R;
  const typename DT::storage* z = reinterpret_cast<const typename DT::storage*>(
      row_ptr<DT>(prm.draft, (size_t)row, V));
  // 8 elements per thread and step: one 16- or 32-byte load, two 16-byte
  // streaming stores (when the row and the gradient row are 16-byte aligned)
  const bool vec = (reinterpret_cast<uintptr_t>(z) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(g) % 16 == 0);
  const int vend = vec ? lo + (hi - lo) / kVec * kVec : lo;  // end of the vector part
  const float fill = mode == 2 ? NAN : 0.f;
#pragma unroll 4
  for (int t = lo / kVec + (int)threadIdx.x; t < vend / kVec; t += kThreads) {
    float v[8];
    if (mode == 1) {
      load8<DT>(reinterpret_cast<const unsigned char*>(z), t * kVec, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = scale * ex2(fmaf(v[q], c, -G) - l2s);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = fill;
    }
    __stcs(reinterpret_cast<float4*>(g + (size_t)t * kVec), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(g + (size_t)t * kVec + 4), make_float4(v[4], v[5], v[6], v[7]));
  }
  for (int e = vend + (int)threadIdx.x; e < hi; e += kThreads) {
    float v = fill;
    if (mode == 1) {
      const float zf = load1<DT>(reinterpret_cast<const unsigned char*>(z), e);
      v = scale * ex2(fmaf(zf, c, -G) - l2s);
    }
    g[e] = v;
  }
  __syncthreads();  // the kept entries are rewritten after the plain writes
  if (mode == 1 && w == 0 && lane < K) {
    const unsigned long long t = sh.topk[lane];
    const int j = (int)(t >> 32);
    if (j >= lo && j < hi) {  // this CTA's range wrote g[j]
      const float pt = __uint_as_float((uint32_t)(t & 0xffffffffu));
      const float zf = load1<DT>(reinterpret_cast<const unsigned char*>(z), j);
      const float q = ex2(fmaf(zf, c, -G) - l2s);
      g[j] = scale * (q - pt);
    }
  }
}

}  // namespace sv
