// sv_stream.cuh -- the streaming pass shared by every entry point.
//
// Every warp is an independent worker.  Two schedules (chosen per call):
//  - static (kFStatic): warp g takes a contiguous range of 1024-element pieces
//    of the row-major piece space and writes one record per run of pieces
//    within a row; the finishing kernel folds each row's records;
//  - dynamic: work items are chunks of W vocabulary entries of one row (or of
//    a target/draft row pair, read together), handed out roughly in index
//    order (first items, then per-stripe counters; see stream_kernel), and
//    the stream itself completes the rows.
// Chain items are numbered position-major (every request's position 0
// first): an item whose request has already rejected at an earlier position
// (dynamic schedule), or whose row the request does not use (ragged batches,
// either schedule), is skipped before any byte is loaded.
//
// A warp streams its items through its own ring of kStages pieces of kPiece
// elements; lane 0 issues bulk copies (cp.async.bulk, no multicast) up to
// kStages pieces ahead, across item boundaries, and each piece completes on its
// own mbarrier.  Each lane moves its share of a piece to registers and keeps
// online softmax statistics (ThreadStat: exact power-of-two rescales), the
// element at the draft token, the argmax, and a sorted warp list of the K best
// keys; per item these are reduced with shuffles into one partial record.
// Dynamic schedule: items are counted into their row one item late (deferred
// counting); the warp whose count completes a row combines the row's partials
// in chunk order (so the result does not depend on which warp finished last)
// and records the row's normaliser and, for chain rows, the acceptance
// decision.
//
// No __syncthreads, no cluster barrier and no shared-memory residency: the
// only cross-warp communication is the counters and the records.
#pragma once

#include "sv_device.cuh"

namespace sv {

constexpr int kPiece = 1024;                  // elements per piece
constexpr int kLaneVecs = kPiece / (32 * kVec);  // 8-element vectors per lane per piece
constexpr int kStages = 2;                    // ring depth per warp
constexpr int kStreamWarps = 8;
constexpr int kStreamThreads = kStreamWarps * 32;
constexpr int kStripes = 32;                  // dynamic item counters (one per warp stripe)

// What an item computes.
enum StreamFlags : int {
  kFStats0 = 1,    // softmax statistics of row 0
  kFStats1 = 2,    // softmax statistics of row 1 (draft logits)
  kFRow1 = 4,      // row 1 exists (draft logits or probabilities) and is staged
  kFArgmax0 = 8,   // argmax of row 0
  kFTopk0 = 16,    // top-K keys of row 0
  kFGather = 32,   // the two rows' values at the row's draft token
  kFStatic = 64,   // static contiguous partition, no in-stream counting (the
                   // finishing kernel completes the rows); else dynamic items
                   // with in-stream counting and early exit
  kFRagged = 128,  // chain requests with their own draft counts or an active
                   // mask: rows a request does not use are skipped, and row
                   // k_b streams its target row only
};

// How items map to rows and what the row decision is.
enum StreamKind : int {
  kKindChainSample = 0,  // rows (i, b) position-major; target i [+ draft i]
  kKindChainGreedy = 1,  // rows (i, b) position-major; target i
  kKindRows = 2,         // plain rows (top-K, KL draft rows, tree nodes)
};

struct __align__(16) Partial {
  float G0, G1;
  double S0, S1;
  float zx0, zx1;
  int flags;  // kPHasX | kPSkipped | kPTimeout
  int pad;
  unsigned long long key;  // argmax key of row 0
};
enum : int { kPHasX = 1, kPSkipped = 2, kPTimeout = 4 };
static_assert(sizeof(Partial) == 48, "chunk record layout");

// Row record written by the warp that completes a row.
struct __align__(16) RowRec {
  int code;    // RowCode
  int argmax;  // argmax of row 0 (greedy kinds)
  float G0, G1;
  double S0, S1;  // normalisers relative to the references G
  double L0, L1;  // log2 of the partition functions: G + log2(S)
};
enum RowCode : int { kRowNone = 0, kRowAccepted = 1, kRowRejected = 2, kRowSkipped = 3,
                     kRowError = 4 };

// Where the bulk copies of an item come from (lane 0 of a warp, in shared
// memory): its two rows at the chunk start and the chunk length.
struct IssueDesc {
  const unsigned char* src0;
  const unsigned char* src1;  // nullptr: row 1 not streamed
  int len;
  int pad;
};

struct StreamParams {
  const void* rows0;      // row-0 array: target logits (chain, rows) or draft logits (KL)
  const void* rows1;      // row-1 array: draft logits / probabilities (chain sample)
  const int32_t* tokens;  // chain: draft tokens [B, k]
  const float* u;         // chain sample: uniforms [B, k+1]
  int kind;
  int B, k, V;            // chain: k drafts per request (k+1 rows)
  int nrows;              // rows streamed
  int row0_stride_rows;   // chain: rows per request in rows0 (k+1); rows: 1
  int W, nchunk;          // chunk length (multiple of kPiece) and chunks per row
  float c;                // log2(e) / T
  int use_bulk;
  int K;                  // top-K list length (kFTopk0)
  int stage_bytes;        // bytes per ring stage (row 0 then row 1), multiple of 128
  int stage_off1;         // offset of row 1 inside a stage
  Partial* part;          // [nrows * nchunk]
  unsigned long long* cand;  // [nrows * nchunk * K]
  // kFTopk0 outputs, written by the warp that completes a row: top-K log
  // probabilities and indices, log-partition (chain: rows b * (k + 1) + i) and,
  // for chain rows with a draft row, KL(renormalised top-K || draft).
  float* topk_logp;
  int32_t* topk_idx;
  float* lse;
  float* kl;
  RowRec* rec;            // [nrows]
  uint32_t* row_counter;  // [nrows]
  uint32_t* req_reject;   // [B] max over rejected chain rows of (k - i)
  int32_t* status;
  FastDiv div_nchunk;     // item -> row
  FastDiv div_B;          // chain row -> position
  uint32_t* sched;        // [kStripes] dynamic item counters (zero between calls)
  int nwarps_eff;         // static partition: warps with a range (<= the grid's warps)
  int count;              // 1: items are counted into rows and rows completed here
                          //    (required for skipping); 0: partials only, rows are
                          //    completed by the finishing kernel
  // Ragged chains (both may be null): request b drafted klen[b] <= k tokens
  // (rows 0..klen[b] are used, row klen[b] being its bonus row); a request
  // with active[b] == 0 uses no row.
  const int32_t* klen;
  const int32_t* active;
};

// Draft count k_b of chain request b: k, or klen[b]; -1 for an inactive
// request, -2 when klen[b] lies outside [0, k].  Rows i > k_b of the request
// are not read.  (The streaming loop asks only in its kFRagged variants.)
__device__ __forceinline__ int req_kb(const StreamParams& p, int b) {
  if (p.klen == nullptr && p.active == nullptr) return p.k;
  if (p.active != nullptr && __ldg(&p.active[b]) == 0) return -1;
  if (p.klen == nullptr) return p.k;
  const int kb = __ldg(&p.klen[b]);
  return (kb < 0 || kb > p.k) ? -2 : kb;
}

// Where row r of a stream lives.
struct RowLoc {
  int b, i;            // chain: request and position; rows: b = r, i = 0
  const unsigned char* row0;
  const unsigned char* row1;
  int x;               // chain: draft token of this row (-1 for the bonus row / none)
};

// A chunk record read through L2 in three 16-byte loads.
__device__ __forceinline__ Partial load_partial(const Partial* p) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  const uint4 a = __ldcg(q), b = __ldcg(q + 1), c = __ldcg(q + 2);
  Partial r;
  memcpy(reinterpret_cast<unsigned char*>(&r), &a, 16);
  memcpy(reinterpret_cast<unsigned char*>(&r) + 16, &b, 16);
  memcpy(reinterpret_cast<unsigned char*>(&r) + 32, &c, 16);
  return r;
}

// Row pointers of row r (the draft token is supplied separately).
template <class T0, class T1, int FLAGS>
__device__ __forceinline__ RowLoc locate_row(const StreamParams& p, int r, int x) {
  RowLoc L;
  L.x = x;
  if (p.kind == kKindRows) {
    L.b = r;
    L.i = 0;
    L.row0 = reinterpret_cast<const unsigned char*>(p.rows0) + (size_t)r * p.V * T0::bytes;
    L.row1 = nullptr;
    return L;
  }
  L.i = fast_div(r, p.div_B);
  L.b = r - L.i * p.B;
  const int P = p.k + 1;
  L.row0 = reinterpret_cast<const unsigned char*>(p.rows0) + ((size_t)L.b * P + L.i) * p.V * T0::bytes;
  L.row1 = nullptr;
  if (p.rows1 != nullptr && L.i < ((FLAGS & kFRagged) ? req_kb(p, L.b) : p.k))
    L.row1 = reinterpret_cast<const unsigned char*>(p.rows1) +
             ((size_t)L.b * p.k + L.i) * p.V * T1::bytes;
  return L;
}

// Acquire-release fence at device scope.
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Warp maximum of a float through the integer reduction unit.
__device__ __forceinline__ float warp_max_redux(float v) {
  return order_float(__reduce_max_sync(0xffffffffu, float_order(v)));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Insert a warp-uniform key into the sorted warp list (lane t holds entry t,
// best first; only lanes < K are meaningful).
__device__ __forceinline__ void warp_list_insert(unsigned long long& list, unsigned long long key,
                                                 unsigned kmask) {
  const int lane = threadIdx.x & 31;
  const int pos = __popc(__ballot_sync(0xffffffffu, list > key) & kmask);
  const unsigned long long up = __shfl_up_sync(0xffffffffu, list, 1);
  if (lane > pos) list = up;
  else if (lane == pos) list = key;
}

__device__ __forceinline__ uint32_t load_relaxed_u32(const uint32_t* p) {
  return *reinterpret_cast<const volatile uint32_t*>(p);
}

// The record slots of row r: one per chunk (dynamic schedule), or, for the
// static partition, one per run: the row start unless a warp range starts
// there, and every warp range start inside the row.  Warp w's range starts at
// floor(w * total / NWs) (total = rows * slots per row, NWs = prm.nwarps_eff).
// floor(num / den) for 0 <= num < 2^53, 0 < den: a float64 estimate, then an
// exact integer correction (avoids a 64-bit integer division).
__device__ __forceinline__ long long floor_div(long long num, long long den) {
  long long q = (long long)((double)num / (double)den);
  if (q * den > num) --q;
  else if ((q + 1) * den <= num) ++q;
  return q;
}

struct SlotMap {
  long long a;      // first slot of the row
  long long total;  // slots of the stream
  int nw;           // warps of the static partition (0: one slot per chunk)
  int wA;           // first warp whose range starts inside the row
  int head;         // 1: the row start is a slot of its own
  int nseg;         // slots of the row
};

__device__ __forceinline__ SlotMap slot_map(const StreamParams& p, int r, bool stat) {
  SlotMap m;
  m.a = (long long)r * p.nchunk;
  m.total = (long long)p.nrows * p.nchunk;
  if (!stat) {
    m.nw = 0;
    m.wA = 0;
    m.head = 1;
    m.nseg = p.nchunk;
    return m;
  }
  const long long nw = p.nwarps_eff;
  const long long e = m.a + p.nchunk;
  const long long wA = floor_div(m.a * nw + m.total - 1, m.total);  // ceil
  const long long wB = floor_div(e * nw + m.total - 1, m.total);
  m.nw = (int)nw;
  m.wA = (int)wA;
  m.head = (wA >= wB || floor_div(wA * m.total, nw) != m.a) ? 1 : 0;
  m.nseg = m.head + (int)(wB - wA);
  return m;
}

__device__ __forceinline__ long long slot_at(const SlotMap& m, int q) {
  if (m.nw == 0) return m.a + q;
  if (m.head && q == 0) return m.a;
  return floor_div((long long)(m.wA + q - m.head) * m.total, m.nw);
}

// Top K keys of a row from its slots' lists (each sorted, best first), best
// first in lanes 0..K-1.  The heads are merged first; a list whose head is not
// above the K-th best key so far holds nothing that can enter, so only the few
// lists with a larger head are read in full.
__device__ __forceinline__ unsigned long long row_topk_merge(const unsigned long long* cand,
                                                             const SlotMap& m, int K) {
  const int lane = threadIdx.x & 31;
  unsigned long long list = kNoKey;
  for (int q0 = 0; q0 < m.nseg; q0 += 32) {
    const int q = q0 + lane;
    const unsigned long long h = q < m.nseg ? __ldcg(&cand[slot_at(m, q) * K]) : kNoKey;
    list = warp_merge_desc(list, warp_sort_desc(h));
  }
  unsigned long long thr = __shfl_sync(0xffffffffu, list, K - 1);
  for (int q0 = 0; q0 < m.nseg; q0 += 32) {
    const int q = q0 + lane;
    const long long sq = q < m.nseg ? slot_at(m, q) : 0;
    const unsigned long long h = q < m.nseg ? __ldcg(&cand[sq * K]) : kNoKey;
    unsigned msk = __ballot_sync(0xffffffffu, h > thr);
    while (msk) {
      // up to four lists at a time: their keys 1..K-1 (the heads are merged)
      unsigned long long x[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        x[t] = kNoKey;
        if (msk) {
          const int src = __ffs(msk) - 1;
          msk &= msk - 1;
          const long long ss = __shfl_sync(0xffffffffu, sq, src);
          if (lane + 1 < K) x[t] = __ldcg(&cand[ss * K + lane + 1]);
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) list = warp_merge_desc(list, x[t]);
      thr = __shfl_sync(0xffffffffu, list, K - 1);
      msk &= __ballot_sync(0xffffffffu, h > thr);
    }
  }
  return list;
}

// A row's statistics folded from its records (every lane holds the same).
struct RowSum {
  float G0, G1;
  double S0, S1;
  double L0, L1;  // log2 of the partition functions: G + log2(S)
  float zx0, zx1;
  int flags;
  int hx;
  unsigned long long key;
};

// Fold row r's records (warp-collective, read-only).  Lane l folds slots l,
// l + 32, ... in order into a running (reference, sum) pair; the power-of-two
// rescales are exact, so the sums equal those of a fold at the final
// reference.  Two records per lane are loaded at a time.
template <class T0, class T1, int FLAGS>
__device__ __noinline__ RowSum row_combine(const StreamParams& prm, int r, int x, bool stat) {
  const int lane = threadIdx.x & 31;
  const SlotMap m = slot_map(prm, r, stat);
  float g0 = -INFINITY, g1 = -INFINITY, zx0 = 0.f, zx1 = 0.f;
  double s0 = 0.0, s1 = 0.0;
  int flags = 0, hx = 0;
  unsigned long long key = kNoKey;
  auto fold = [&](const Partial& pq) {
    if (pq.G0 > g0) {
      s0 = rescale_pow2(s0, g0, pq.G0);
      g0 = pq.G0;
    }
    s0 += rescale_pow2(pq.S0, pq.G0, g0);
    if (pq.G1 > g1) {
      s1 = rescale_pow2(s1, g1, pq.G1);
      g1 = pq.G1;
    }
    s1 += rescale_pow2(pq.S1, pq.G1, g1);
    flags |= pq.flags;
    if (pq.flags & kPHasX) {
      hx = 1;
      zx0 = pq.zx0;
      zx1 = pq.zx1;
    }
    key = pq.key > key ? pq.key : key;
  };
  for (int q = lane; q < m.nseg; q += 64) {
    const Partial pa = load_partial(prm.part + slot_at(m, q));
    const bool two = q + 32 < m.nseg;
    const Partial pb = two ? load_partial(prm.part + slot_at(m, q + 32)) : Partial{};
    fold(pa);
    if (two) fold(pb);
  }
  RowSum s;
  s.G0 = warp_max(g0);
  s.G1 = warp_max(g1);
  s.S0 = warp_sum(rescale_pow2(s0, g0, s.G0));
  s.S1 = warp_sum(rescale_pow2(s1, g1, s.G1));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) flags |= __shfl_xor_sync(0xffffffffu, flags, o);
  s.flags = flags;
  s.key = warp_max_u64(key);
  const unsigned hm = __ballot_sync(0xffffffffu, hx != 0);
  s.hx = hm != 0u;
  s.zx0 = s.zx1 = 0.f;
  if (hm) {
    const int src = __ffs(hm) - 1;
    s.zx0 = __shfl_sync(0xffffffffu, zx0, src);
    s.zx1 = __shfl_sync(0xffffffffu, zx1, src);
    // a draft row that is not streamed (probabilities): q(x) read directly
    if (!(FLAGS & kFRow1) && prm.rows1 != nullptr && prm.kind != kKindRows) {
      const RowLoc L = locate_row<T0, T1, FLAGS>(prm, r, x);
      if (L.row1 != nullptr) s.zx1 = load1<T1>(L.row1, x);
    }
  }
  s.L0 = (double)s.G0 + log2(s.S0);
  s.L1 = (double)s.G1 + log2(s.S1);
  return s;
}

// A completed row's record: code (RowCode) and error bits (lane-uniform, no
// side effects).  Chain sampling takes the ratio test u * q(x) < p(x) in
// float64 from the row's log-partitions; greedy chains compare the draft
// token with the argmax.
template <int FLAGS>
__device__ __forceinline__ RowRec row_decide(const StreamParams& prm, int r, int x,
                                             const RowSum& s, int* err_out) {
  RowRec rec;
  rec.G0 = s.G0;
  rec.G1 = s.G1;
  rec.S0 = s.S0;
  rec.S1 = s.S1;
  rec.L0 = s.L0;
  rec.L1 = s.L1;
  rec.argmax = key_index(s.key);
  int err = 0, code = kRowAccepted;
  if (s.flags & kPTimeout) err |= SV_DEV_TIMEOUT;
  if ((FLAGS & kFStats0) && s.G0 == -INFINITY) err |= SV_DEV_NO_FINITE;
  if (prm.kind != kKindRows) {
    const int i = fast_div(r, prm.div_B), b = r - i * prm.B, k = req_kb(prm, b);
    if ((FLAGS & kFStats1) && i < k && s.G1 == -INFINITY) err |= SV_DEV_NO_FINITE;
    if (s.flags & kPSkipped) {
      err = 0;
      code = kRowSkipped;
    } else if (prm.kind == kKindChainSample) {
      if (i < k && !s.hx) err |= SV_DEV_BAD_TOKEN;
      if (!err && i < k) {
        const double c = (double)prm.c;
        const double px = exp2((double)s.zx0 * c - s.L0);
        const double qx = (FLAGS & kFStats1) ? exp2((double)s.zx1 * c - s.L1) : (double)s.zx1;
        const double u = (double)prm.u[(size_t)b * (prm.k + 1) + i];
        code = (u * qx < px) ? kRowAccepted : kRowRejected;
      }
    } else {  // greedy: accept iff the draft token is the argmax
      if (i < k && (x < 0 || x >= prm.V)) err |= SV_DEV_BAD_TOKEN;
      if (!err && i < k) code = (x == rec.argmax) ? kRowAccepted : kRowRejected;
    }
  }
  if (err) code = kRowError;
  rec.code = code;
  *err_out = err;
  return rec;
}

// Top-K outputs of a completed row (kFTopk0; warp-collective): merge the
// row's lists and return them to zero; with `outputs`, write the row's top-K
// log-probabilities, indices and lse (and, for a chain row with a draft row,
// KL(p~ || q)).  L0/L1: the row's log2-partitions.  A failed row of a plain
// top-K call reads as NaN.
template <class T0, class T1, int FLAGS>
__device__ __noinline__ void row_outputs(const StreamParams& prm, int r, int x, double L0,
                                         double L1, int err, bool outputs, bool stat) {
  const int lane = threadIdx.x & 31;
  const SlotMap m = slot_map(prm, r, stat);
  const int K = prm.K;
  const unsigned long long kk = row_topk_merge(prm.cand, m, K);
  __syncwarp();
  for (int q = 0; q < m.nseg; ++q) {
    const long long sq = slot_at(m, q);
    if (lane < K) prm.cand[sq * K + lane] = 0ull;
  }
  if (!outputs) return;
  const RowLoc L = locate_row<T0, T1, FLAGS>(prm, r, x);
  const double ln2 = 0.69314718055994530942;
  const bool rows = prm.kind == kKindRows;
  const size_t orow = rows ? (size_t)r : (size_t)L.b * (prm.k + 1) + L.i;
  const bool nan_out = rows && err != 0;
  double lp = -INFINITY;
  int j = -1;
  if (lane < K) {
    j = key_index(kk);
    lp = ((double)key_value(kk) * (double)prm.c - L0) * ln2;
    prm.topk_logp[orow * K + lane] = nan_out ? NAN : (float)lp;
    prm.topk_idx[orow * K + lane] = j;
  }
  if (lane == 0) prm.lse[orow] = nan_out ? NAN : (float)(L0 * ln2);
  if (!rows && L.row1 != nullptr && L.i < req_kb(prm, L.b)) {
    // KL(p~ || q) over the renormalised top-K of the target row
    double mx = lp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double se = (lane < K) ? exp(lp - mx) : 0.0;
    se = warp_sum(se);
    const double lse_k = mx + log(se);
    double term = 0.0;
    if (lane < K && j >= 0 && j < prm.V) {
      const float zd = load1<T1>(L.row1, j);
      const double log_pt = lp - lse_k;
      const double pt = exp(log_pt);
      const double log_q =
          (FLAGS & kFStats1) ? ((double)zd * (double)prm.c - L1) * ln2 : log((double)zd);
      term = (pt == 0.0) ? 0.0 : pt * (log_pt - log_q);
    }
    term = warp_sum(term);
    if (lane == 0) prm.kl[(size_t)L.b * prm.k + L.i] = (float)term;
  }
}

// Return row r's records to zero (warp-collective).
__device__ __forceinline__ void row_zero_records(const StreamParams& prm, int r, bool stat) {
  const int lane = threadIdx.x & 31;
  const SlotMap m = slot_map(prm, r, stat);
  for (int q = lane; q < m.nseg; q += 32) prm.part[slot_at(m, q)] = Partial{};
}

// In-stream completion (dynamic schedule): the warp whose count completed row
// r decides it, publishes its record (and a rejection to the request's
// rejection word, so that later positions are skipped) and commits it.
template <class T0, class T1, int FLAGS>
__device__ __noinline__ void row_complete(const StreamParams& prm, int r, int x) {
  const int lane = threadIdx.x & 31;
  const RowSum s = row_combine<T0, T1, FLAGS>(prm, r, x, false);
  int err = 0;
  const RowRec rec = row_decide<FLAGS>(prm, r, x, s, &err);
  if (lane == 0) {
    if (rec.code == kRowRejected) {
      const int i = fast_div(r, prm.div_B), b = r - i * prm.B;
      atomicMax(&prm.req_reject[b], (uint32_t)(prm.k - i));
    }
    if (err) set_status(prm.status, err);
    // a plain top-K call has no second pass: no record
    if (!(prm.kind == kKindRows && (FLAGS & kFTopk0))) prm.rec[r] = rec;
    prm.row_counter[r] = 0u;
  }
  if (FLAGS & kFTopk0) row_outputs<T0, T1, FLAGS>(prm, r, x, s.L0, s.L1, err, rec.code != kRowSkipped, false);
  row_zero_records(prm, r, false);
}

// ---------------------------------------------------------------------------
// One lane's share of one row of a piece: kLaneVecs vectors of 8 elements,
// vector v holding piece elements (v * 32 + lane) * 8 .. + 7, in registers.
// Vectors past the end of the piece read as -inf (no mass, never a maximum).
// ---------------------------------------------------------------------------
template <class T>
struct LaneRow;
template <>
struct LaneRow<BF16> {
  uint4 w[kLaneVecs];
};
template <>
struct LaneRow<F32> {
  float4 w[2 * kLaneVecs];
};

__device__ __forceinline__ void lane_load(const unsigned char* st, int nv, LaneRow<BF16>& R) {
  const int lane = threadIdx.x & 31;
  if (nv == kLaneVecs * 32) {  // full piece (warp-uniform)
#pragma unroll
    for (int v = 0; v < kLaneVecs; ++v)
      R.w[v] = *reinterpret_cast<const uint4*>(st + (size_t)(v * 32 + lane) * 16);
    return;
  }
#pragma unroll
  for (int v = 0; v < kLaneVecs; ++v) {
    const int vi = v * 32 + lane;
    R.w[v] = vi < nv ? *reinterpret_cast<const uint4*>(st + (size_t)vi * 16)
                     : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
  }
}
__device__ __forceinline__ void lane_load(const unsigned char* st, int nv, LaneRow<F32>& R) {
  const int lane = threadIdx.x & 31;
  if (nv == kLaneVecs * 32) {  // full piece (warp-uniform)
#pragma unroll
    for (int v = 0; v < kLaneVecs; ++v) {
      R.w[2 * v] = *reinterpret_cast<const float4*>(st + (size_t)(v * 32 + lane) * 32);
      R.w[2 * v + 1] = *reinterpret_cast<const float4*>(st + (size_t)(v * 32 + lane) * 32 + 16);
    }
    return;
  }
  const float ni = -INFINITY;
#pragma unroll
  for (int v = 0; v < kLaneVecs; ++v) {
    const int vi = v * 32 + lane;
    if (vi < nv) {
      R.w[2 * v] = *reinterpret_cast<const float4*>(st + (size_t)vi * 32);
      R.w[2 * v + 1] = *reinterpret_cast<const float4*>(st + (size_t)vi * 32 + 16);
    } else {
      R.w[2 * v] = R.w[2 * v + 1] = make_float4(ni, ni, ni, ni);
    }
  }
}

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Maximum of vector v, and of all the lane's vectors.
__device__ __forceinline__ float vec_max(const LaneRow<BF16>& R, int v) {
  const uint32_t m = bmax2(bmax2(R.w[v].x, R.w[v].y), bmax2(R.w[v].z, R.w[v].w));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}
__device__ __forceinline__ float vec_max(const LaneRow<F32>& R, int v) {
  const float4 a = R.w[2 * v], b = R.w[2 * v + 1];
  return fmaxf(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), fmaxf(fmaxf(b.x, b.y), fmaxf(b.z, b.w)));
}
__device__ __forceinline__ float lane_max(const LaneRow<BF16>& R) {
  uint32_t m = bmax2(bmax2(R.w[0].x, R.w[0].y), bmax2(R.w[0].z, R.w[0].w));
#pragma unroll
  for (int v = 1; v < kLaneVecs; ++v)
    m = bmax2(m, bmax2(bmax2(R.w[v].x, R.w[v].y), bmax2(R.w[v].z, R.w[v].w)));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}
__device__ __forceinline__ float lane_max(const LaneRow<F32>& R) {
  float m = vec_max(R, 0);
#pragma unroll
  for (int v = 1; v < kLaneVecs; ++v) m = fmaxf(m, vec_max(R, v));
  return m;
}

// Element t (0..7) of vector v.
__device__ __forceinline__ float lane_elem(const LaneRow<BF16>& R, int v, int t) {
  const uint32_t w = (t >> 1) == 0 ? R.w[v].x : (t >> 1) == 1 ? R.w[v].y : (t >> 1) == 2 ? R.w[v].z
                                                                                       : R.w[v].w;
  return (t & 1) ? bf16_hi(w) : bf16_lo(w);
}
__device__ __forceinline__ float lane_elem(const LaneRow<F32>& R, int v, int t) {
  const float4 q = R.w[2 * v + (t >> 2)];
  const int u = t & 3;
  return u == 0 ? q.x : u == 1 ? q.y : u == 2 ? q.z : q.w;
}

// 2^(x c - ref) for the pair (lo, hi): one packed fma, two exp2.
__device__ __forceinline__ unsigned long long term2(float lo, float hi, unsigned long long cc,
                                                    unsigned long long nr) {
  float a, b;
  f2_unpack(f2_fma(f2_pack(lo, hi), cc, nr), a, b);
  return f2_pack(ex2(a), ex2(b));
}

// 2^a and 2^b on the FMA pipe instead of the special-function unit, for
// arguments a, b <= 0 (-inf allowed).  Cody-Waite reduction: n = rint(a),
// f = a - n in [-1/2, 1/2] (exact); 2^f = e^(f ln 2) by its Taylor polynomial
// through f^6, whose coefficients are (ln 2)^k / k! rounded to fp32
// (truncation error below 1.7e-7 relative, about that of ex2.approx),
// evaluated for both arguments at once with packed fp32 FMAs; then n is added
// to the exponent field.  Results below 2^-125 are 0 (ex2.approx.ftz flushes
// below 2^-126; the terms here are relative to a maximum of order 1).
__device__ __forceinline__ unsigned long long ex2_fma_pair(float a, float b) {
  a = fmaxf(a, -127.f);
  b = fmaxf(b, -127.f);
  const float na = rintf(a), nb = rintf(b);
  const unsigned long long f = f2_pack(a - na, b - nb);
  auto k2 = [](float v) { return f2_pack(v, v); };
  unsigned long long p = k2(1.540352969e-04f);  // (ln 2)^6 / 6!
  p = f2_fma(p, f, k2(1.333355787e-03f));        // (ln 2)^5 / 5!
  p = f2_fma(p, f, k2(9.618128650e-03f));        // (ln 2)^4 / 4!
  p = f2_fma(p, f, k2(5.550410971e-02f));        // (ln 2)^3 / 3!
  p = f2_fma(p, f, k2(2.402265072e-01f));        // (ln 2)^2 / 2!
  p = f2_fma(p, f, k2(6.931471825e-01f));        // ln 2
  p = f2_fma(p, f, k2(1.0f));
  float pa, pb;
  f2_unpack(p, pa, pb);
  const int ia = (int)na, ib = (int)nb;
  pa = ia < -125 ? 0.f : __uint_as_float(__float_as_uint(pa) + ((unsigned)ia << 23));
  pb = ib < -125 ? 0.f : __uint_as_float(__float_as_uint(pb) + ((unsigned)ib << 23));
  return f2_pack(pa, pb);
}

// term2 with the two powers on the FMA pipe.
__device__ __forceinline__ unsigned long long term2_fma(float lo, float hi, unsigned long long cc,
                                                        unsigned long long nr) {
  float a, b;
  f2_unpack(f2_fma(f2_pack(lo, hi), cc, nr), a, b);
  return ex2_fma_pair(a, b);
}

// Every SV_EXP2_FMA_EVERY-th element pair of a lane's piece takes its powers
// on the FMA pipe (0: none), to balance the special-function unit against
// the FMA pipe.
#ifndef SV_EXP2_FMA_EVERY
#define SV_EXP2_FMA_EVERY 0
#endif
__device__ __forceinline__ unsigned long long term2_sel(int j, float lo, float hi,
                                                        unsigned long long cc, unsigned long long nr) {
  if (SV_EXP2_FMA_EVERY > 0 && j % (SV_EXP2_FMA_EVERY > 0 ? SV_EXP2_FMA_EVERY : 1) ==
                                   (SV_EXP2_FMA_EVERY > 0 ? SV_EXP2_FMA_EVERY : 1) - 1)
    return term2_fma(lo, hi, cc, nr);
  return term2(lo, hi, cc, nr);
}

// Sum over the lane's elements of 2^(x c - ref), by a fixed tree of packed adds.
__device__ __forceinline__ float lane_terms(const LaneRow<BF16>& R, float c, float ref) {
  const unsigned long long cc = f2_pack(c, c), nr = f2_pack(-ref, -ref);
  unsigned long long e[4 * kLaneVecs];
#pragma unroll
  for (int v = 0; v < kLaneVecs; ++v) {
    e[4 * v + 0] = term2_sel(4 * v + 0, bf16_lo(R.w[v].x), bf16_hi(R.w[v].x), cc, nr);
    e[4 * v + 1] = term2_sel(4 * v + 1, bf16_lo(R.w[v].y), bf16_hi(R.w[v].y), cc, nr);
    e[4 * v + 2] = term2_sel(4 * v + 2, bf16_lo(R.w[v].z), bf16_hi(R.w[v].z), cc, nr);
    e[4 * v + 3] = term2_sel(4 * v + 3, bf16_lo(R.w[v].w), bf16_hi(R.w[v].w), cc, nr);
  }
#pragma unroll
  for (int w = 2 * kLaneVecs; w >= 1; w >>= 1)
#pragma unroll
    for (int t = 0; t < w; ++t) e[t] = f2_add(e[t], e[t + w]);
  float lo, hi;
  f2_unpack(e[0], lo, hi);
  return lo + hi;
}
__device__ __forceinline__ float lane_terms(const LaneRow<F32>& R, float c, float ref) {
  const unsigned long long cc = f2_pack(c, c), nr = f2_pack(-ref, -ref);
  unsigned long long e[4 * kLaneVecs];
#pragma unroll
  for (int v = 0; v < 2 * kLaneVecs; ++v) {
    e[2 * v + 0] = term2(R.w[v].x, R.w[v].y, cc, nr);
    e[2 * v + 1] = term2(R.w[v].z, R.w[v].w, cc, nr);
  }
#pragma unroll
  for (int w = 2 * kLaneVecs; w >= 1; w >>= 1)
#pragma unroll
    for (int t = 0; t < w; ++t) e[t] = f2_add(e[t], e[t + w]);
  float lo, hi;
  f2_unpack(e[0], lo, hi);
  return lo + hi;
}

// Fold one row of a piece into a lane's statistics (reference moved first).
template <class T>
__device__ __forceinline__ void lane_stats(ThreadStat& st, const LaneRow<T>& R, float pm, float c) {
  stat_cover(st, pm, c);
  if (pm != -INFINITY) st.S += (double)lane_terms(R, c, st.ref);
}

// ---------------------------------------------------------------------------
// The streaming kernel.
//
// Work distribution: warp g takes items g and g + NW first, then items
// 2 NW + 32 t + (g mod 32) in the order of the counter t of its stripe
// (g mod 32), so the items run roughly in index order (position-major for
// chains) and no warp waits on a slow neighbour; 32 counters keep the atomic
// traffic per address low.  A warp knows its next three items; the counter
// value, rejection word and draft token of each are read an item before they
// are used.  Every warp fetches until it draws an item past the end, so each
// counter receives a known number of fetches; the fetch that returns the last
// of them returns the counter to zero.
// ---------------------------------------------------------------------------
template <class T0, class T1, int FLAGS>
__global__ void __launch_bounds__(kStreamThreads, 3) stream_kernel(const __grid_constant__ StreamParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char* ring = smem + (size_t)warp * kStages * prm.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kStreamWarps * kStages * prm.stage_bytes) +
                   warp * kStages;
  IssueDesc* desc = reinterpret_cast<IssueDesc*>(smem + (size_t)kStreamWarps * kStages * prm.stage_bytes +
                                                 (size_t)kStreamWarps * kStages * 8) +
                    warp * 2;
  const bool use_bulk = prm.use_bulk != 0;
  const bool chain = prm.kind != kKindRows;
  constexpr bool stat = (FLAGS & kFStatic) != 0;
  constexpr int RF = FLAGS & ~kFStatic;  // what a row completion does
  const int V = prm.V, W = prm.W, nchunk = prm.nchunk;
  const int total = prm.nrows * nchunk;
  const int nwarps = (int)gridDim.x * kStreamWarps;
  const int gwarp = (int)blockIdx.x * kStreamWarps + warp;
  const float c = prm.c;
  const int K = prm.K;
  pdl_launch_dependents();  // the finisher may be scheduled as resources free up
  // Static schedule: this warp's pieces [lo, hi); an item is a run of them
  // within one row (the record slot is the run's first piece).
  const int nws = prm.nwarps_eff;
  // (floor_div: the exact floor by a float64 quotient and one correction,
  // cheaper than a 64-bit integer division)
  const long long lo = (stat && gwarp < nws) ? floor_div((long long)gwarp * total, nws) : 0;
  const long long hi = (stat && gwarp < nws) ? floor_div((long long)(gwarp + 1) * total, nws) : 0;
  auto run_end = [&](int item) -> long long {  // static: one past the run's last piece
    const long long re = (long long)(fast_div(item, prm.div_nchunk) + 1) * nchunk;
    return re < hi ? re : hi;
  };
  auto next_run = [&](int item) -> int {  // static: the run after the one starting at item
    if (item >= total) return total;
    const long long e = run_end(item);
    return e < hi ? (int)e : total;
  };
  // Elements of an item whose first piece is piece ch of its row.
  auto item_len = [&](int item, int ch) -> int {
    if (!stat) return min(W, V - ch * W);
    return (int)min((run_end(item) - item) * (long long)kPiece, (long long)(V - ch * kPiece));
  };
  if (lane == 0 && use_bulk) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // Lane 0: an item's request-rejection word and draft token (chain kinds).
  auto prefetch = [&](int item, uint32_t& rj, int& x) {
    rj = 0u;
    x = -1;
    if (!chain || item >= total) return;
    const int r = fast_div(item, prm.div_nchunk);
    const int i = fast_div(r, prm.div_B), b = r - i * prm.B;
    if (!stat) rj = load_relaxed_u32(&prm.req_reject[b]);
    if (FLAGS & kFRagged) {
      const int kb = req_kb(prm, b);
      if (i > kb) rj = 0xffffffffu;  // a row its request does not use
      if (i < kb) x = prm.tokens[(size_t)b * prm.k + i];
    } else if (i < prm.k) {
      x = prm.tokens[(size_t)b * prm.k + i];
    }
  };
  // Pieces of an item (lane-uniform); 0 when skipped: an earlier position of
  // its request rejected, or the request does not use the row.  Lane 0 records the item's copy sources in
  // descriptor `slot`.
  auto pieces_of = [&](int item, uint32_t rj, int slot) -> int {
    if (item >= total) return 0;
    const int r = fast_div(item, prm.div_nchunk);
    const int ch = item - r * nchunk;
    int skip = 0;
    if (chain) {
      const int i = fast_div(r, prm.div_B);
      skip = __shfl_sync(0xffffffffu, rj > (uint32_t)(prm.k - i) ? 1 : 0, 0);
    }
    const int len = item_len(item, ch);
    if (lane == 0 && !skip) {
      const RowLoc L = locate_row<T0, T1, FLAGS>(prm, r, -1);
      IssueDesc d;
      d.src0 = L.row0 + (size_t)ch * W * T0::bytes;
      d.src1 = ((FLAGS & kFRow1) && L.row1 != nullptr) ? L.row1 + (size_t)ch * W * T1::bytes : nullptr;
      d.len = len;
      d.pad = 0;
      desc[slot] = d;
    }
    return skip ? 0 : (len + kPiece - 1) / kPiece;
  };

  // Lane 0: bulk copies of piece p of the item in descriptor `slot` into ring
  // stage s.
  auto issue = [&](int slot, int p, int s) {
    const IssueDesc d = desc[slot];
    const int e0 = p * kPiece;
    const int n = min(kPiece, d.len - e0);
    const uint32_t nb0 = (uint32_t)(n * T0::bytes) & ~15u;
    const uint32_t nb1 = d.src1 != nullptr ? ((uint32_t)(n * T1::bytes) & ~15u) : 0u;
    unsigned char* st = ring + (size_t)s * prm.stage_bytes;
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[s], nb0 + nb1);
    if (nb0) bulk_g2s_plain(st, d.src0 + (size_t)e0 * T0::bytes, nb0, &bars[s]);
    if (nb1) bulk_g2s_plain(st + prm.stage_off1, d.src1 + (size_t)e0 * T1::bytes, nb1, &bars[s]);
  };
  int slot_cur = 0;  // descriptor of cur; nxt uses the other

  uint32_t n_issued = 0, n_consumed = 0;
  // Static mode (no in-stream counting): warp g takes the contiguous items
  // [g * total / NW, (g + 1) * total / NW) and merges consecutive items of one
  // row into one record.  Dynamic mode: first items g and g + NW, then the
  // stripe counters.
  int cur = stat ? (lo < hi ? (int)lo : total) : gwarp, cur_np, cur_x;
  int cur_x0 = -1;  // lane 0: the first item's draft token, read after the first copies are issued
  {
    uint32_t rj;
    if (lane == 0) prefetch(cur, rj, cur_x0);
    cur_np = pieces_of(cur, rj, 0);
  }
  int nxt = stat ? next_run(cur) : gwarp + nwarps, nxt_np = -1, nxt_x = -1;  // nxt_x: lane 0 only
  uint32_t nxt_rj = 0u;
  // Lane 0: the stripe counter and the number of fetches it will receive.
  const int stripe = gwarp % kStripes;
  uint32_t* const ctr = prm.sched + stripe;
  uint32_t fetches = 0u;
  {
    const long long rest = (long long)total - 2LL * nwarps - stripe;
    const long long valid = rest > 0 ? (rest + kStripes - 1) / kStripes : 0;
    const int warps = nwarps / kStripes + (stripe < nwarps % kStripes ? 1 : 0);
    fetches = (uint32_t)(valid + warps);
  }
  auto fetch = [&]() -> uint32_t {  // lane 0; the result is read an item later
    return atomicAdd(ctr, 1u);
  };
  // The item of a fetched counter value (read by every lane from lane 0).  The
  // lane that holds the last value of this call returns the counter to zero.
  auto take = [&](uint32_t t0) -> int {
    if (lane == 0 && t0 == fetches - 1u) *ctr = 0u;
    const uint32_t t = __shfl_sync(0xffffffffu, t0, 0);
    const long long d = 2LL * nwarps + (long long)t * kStripes + stripe;
    return d < total ? (int)d : total;
  };
  // Three items ahead are known: cur, nxt and nxt2.  nxt's rejection word and
  // token were read one item before they are needed; nxt2's are in flight;
  // pend (the counter value of the item after nxt2) was fetched one item
  // before it is read.
  int nxt2 = total, nxt2_x = -1;  // nxt2_x: lane 0 only
  uint32_t nxt2_rj = 0u;
  uint32_t pend = 0u;  // lane 0
  if (lane == 0) {
    prefetch(nxt, nxt_rj, nxt_x);
    if (!stat) pend = fetch();  // every warp fetches at least once
  }
  nxt2 = stat ? next_run(nxt) : take(pend);
  if (lane == 0) {
    prefetch(nxt2, nxt2_rj, nxt2_x);
    if (!stat && nxt2 < total) pend = fetch();
  }
  int iss_which = 0, iss_p = 0;
  int timeouts = 0;

  auto top_up = [&]() {
    while (n_issued - n_consumed < (uint32_t)kStages) {
      int it, pp;
      if (iss_which == 0) {
        if (iss_p < cur_np) {
          it = slot_cur;
          pp = iss_p++;
        } else {
          iss_which = 1;
          iss_p = 0;
          continue;
        }
      } else {
        if (nxt_np < 0) nxt_np = pieces_of(nxt, nxt_rj, slot_cur ^ 1);
        if (iss_p < nxt_np) {
          it = slot_cur ^ 1;
          pp = iss_p++;
        } else {
          break;
        }
      }
      if (use_bulk && lane == 0) issue(it, pp, (int)(n_issued % kStages));
      ++n_issued;
    }
  };

  // Deferred row counting.  sig_*: an item whose record is written but not
  // yet counted; res_*: a count added whose result (lane 0) is not yet read.
  int sig_r = -1, sig_x = -1, res_r = -1, res_x = -1;
  uint32_t res_old = 0u;
  auto resolve = [&]() {
    if (res_r < 0) return;
    const int last = __shfl_sync(0xffffffffu, res_old == (uint32_t)(nchunk - 1) ? 1 : 0, 0);
    if (last) {
      __threadfence();  // acquire: the other items' records
      __syncwarp();
      row_complete<T0, T1, RF>(prm, res_r, res_x);
    }
    res_r = -1;
  };
  auto signal = [&]() {
    if (sig_r < 0) return;
    __syncwarp();
    if (lane == 0) {
      fence_acq_rel_gpu();  // release: the record (and list) before its count
      res_old = atomicAdd(&prm.row_counter[sig_r], 1u);
    }
    res_r = sig_r;
    res_x = sig_x;
    sig_r = -1;
  };

  top_up();
  cur_x = __shfl_sync(0xffffffffu, cur_x0, 0);
  // The statistics of a run: the items merged into one record (one item in
  // dynamic mode).
  ThreadStat st0, st1;
  float best = -INFINITY;
  int bidx = -1;
  float zx0 = 0.f, zx1 = 0.f;
  int hx = 0;
  unsigned long long list = kNoKey;
  unsigned long long thr_key = kNoKey;
  unsigned long long thr_floor = kNoKey;  // lower bound of the run's K-th best key
  float thr_val = -INFINITY;
  bool seed = false;
  // Static schedule with top-K: the row's counter word (unused by the static
  // schedule) holds the largest K-th-best value any warp of the row has
  // published (order-preserving bits).  At least K elements of the row are
  // that large, so every warp of the row may drop what is below it.
  uint32_t pub = 0u;  // the largest value this run has published
  int run_first = -1;  // the item whose record slot the run writes
  while (cur < total) {
    const int r = fast_div(cur, prm.div_nchunk);
    const int ch = cur - r * nchunk;
    const RowLoc L = locate_row<T0, T1, FLAGS>(prm, r, cur_x);
    const int clen = item_len(cur, ch);
    const bool has1 = (FLAGS & kFRow1) && L.row1 != nullptr;
    if (run_first < 0) {
      run_first = cur;
      stat_init(st0);
      stat_init(st1);
      best = -INFINITY;
      bidx = -1;
      zx0 = zx1 = 0.f;
      hx = 0;
      list = kNoKey;
      thr_key = kNoKey;
      thr_floor = kNoKey;
      thr_val = -INFINITY;
      seed = true;
      pub = 0u;
    }

    for (int p = 0; p < cur_np; ++p) {
      // the row's shared floor, read now and used after the statistics
      uint32_t row_floor = 0u;
      if ((FLAGS & kFTopk0) && stat) row_floor = *reinterpret_cast<volatile uint32_t*>(&prm.row_counter[r]);
      const int s = (int)(n_consumed % kStages);
      const uint32_t ph = (n_consumed / kStages) & 1u;
      unsigned char* st = ring + (size_t)s * prm.stage_bytes;
      unsigned char* st1p = st + prm.stage_off1;
      const int e0 = ch * W + p * kPiece;  // row index of the piece's first element
      const int n = min(kPiece, clen - p * kPiece);
      if (use_bulk) {
        if (!mbar_wait_bounded(&bars[s], ph)) ++timeouts;
      }
      // Elements the bulk copy does not cover (the unaligned tail, or the whole
      // piece on the scalar path) and padding of the last vector.
      if (!use_bulk || n < kPiece) {
        const int a0 = use_bulk ? (int)(((uint32_t)(n * T0::bytes) & ~15u) / T0::bytes) : 0;
        const typename T0::storage* src = reinterpret_cast<const typename T0::storage*>(L.row0) + e0;
        for (int e = a0 + lane; e < n; e += 32)
          reinterpret_cast<typename T0::storage*>(st)[e] = src[e];
        for (int e = n + lane; e < ((n + kVec - 1) / kVec) * kVec; e += 32) store_pad<T0>(st, e, false);
        if (has1) {
          const int a1 = use_bulk ? (int)(((uint32_t)(n * T1::bytes) & ~15u) / T1::bytes) : 0;
          const typename T1::storage* src1 =
              reinterpret_cast<const typename T1::storage*>(L.row1) + e0;
          for (int e = a1 + lane; e < n; e += 32)
            reinterpret_cast<typename T1::storage*>(st1p)[e] = src1[e];
          for (int e = n + lane; e < ((n + kVec - 1) / kVec) * kVec; e += 32)
            store_pad<T1>(st1p, e, false);
        }
        __syncwarp();
      }
      const int nv = (n + kVec - 1) / kVec;
      // The draft token's values.
      if ((FLAGS & kFGather) && L.x >= e0 && L.x < e0 + n) {
        hx = 1;
        zx0 = load1<T0>(st, L.x - e0);
        if (has1) zx1 = load1<T1>(st1p, L.x - e0);
      }
      {
        LaneRow<T0> R;
        lane_load(st, nv, R);
        const float pm = lane_max(R);
        if (FLAGS & kFStats0) lane_stats(st0, R, pm, c);
        if (FLAGS & kFArgmax0) {
          if (pm > best || (bidx < 0 && nv > lane)) {
            int bi = -1;
#pragma unroll
            for (int v = kLaneVecs - 1; v >= 0; --v)
#pragma unroll
              for (int t = 7; t >= 0; --t)
                if (lane_elem(R, v, t) == pm) bi = (v * 32 + lane) * kVec + t;
            best = pm;
            bidx = e0 + bi;
          }
        }
        if (FLAGS & kFTopk0) {
          if (seed) {
            // The smallest lane maximum of the run's first piece: every lane
            // holds an element at least that large, so the run's K best (K <=
            // 32) are too; nothing below it needs to enter the list.
            const float t = order_float(__reduce_min_sync(0xffffffffu, float_order(pm)));
            thr_floor = (unsigned long long)float_order(t) << 32;
            thr_key = thr_floor > thr_key ? thr_floor : thr_key;
            thr_val = key_value(thr_key);
            seed = false;
          }
          if (stat) {
            // another warp's K-th best value of this row: a floor like the
            // lane maxima's (equal values may still enter)
            const unsigned long long ef = (unsigned long long)row_floor << 32;
            if (ef > thr_floor) {
              thr_floor = ef;
              if (thr_floor > thr_key) thr_key = thr_floor;
              thr_val = key_value(thr_key);
            }
          }
          // Candidates are found lane-parallel in registers: each round, every
          // lane offers its best key above the threshold that it has not yet
          // offered; the 32 offers are sorted and merged into the list.
          // This lane's vectors that can hold a candidate.  The list holds
          // only earlier pieces' keys here, so a value equal to the list's
          // K-th cannot enter (larger index); the floor admits equal values.
          unsigned pmask = 0;
          const bool strict = thr_key != thr_floor;
          if (pm > thr_val || (!strict && pm == thr_val)) {  // the lane maximum first
#pragma unroll
            for (int v = 0; v < kLaneVecs; ++v) {
              const float vm = vec_max(R, v);
              if (v * 32 + lane < nv && (vm > thr_val || (!strict && vm == thr_val))) pmask |= 1u << v;
            }
          }
          unsigned long long last = ~0ull;
          while (__any_sync(0xffffffffu, pmask != 0)) {
            unsigned long long cand = kNoKey;
            int more = 0;  // keys above the threshold besides the offer
            for (unsigned mm = pmask; mm; mm &= mm - 1) {
              const int vi = (__ffs(mm) - 1) * 32 + lane;
              float xs[8];
              load8<T0>(st, vi * kVec, xs);  // (the stage is still this piece's)
              // the elements whose value can give a key above the threshold
              // (a value below thr_val cannot); keys only for those
              unsigned em = 0;
#pragma unroll
              for (int t = 0; t < 8; ++t)
                if (vi * kVec + t < n && !(xs[t] < thr_val)) em |= 1u << t;
              for (; em; em &= em - 1) {
                const int t = __ffs(em) - 1;
                float xv = xs[0];
#pragma unroll
                for (int q = 1; q < 8; ++q)
                  if (t == q) xv = xs[q];
                const unsigned long long key = topk_key(xv, e0 + vi * kVec + t);
                if (key > thr_key && key < last) {
                  more += cand != kNoKey;
                  if (key > cand) cand = key;
                }
              }
            }
            if (cand == kNoKey || more == 0) pmask = 0;  // nothing left after this offer
            unsigned cm = __ballot_sync(0xffffffffu, cand != kNoKey);
            if (!cm) break;
            if (__popc(cm) <= 12) {  // few offers: one by one (a sort costs about ten inserts)
              while (cm) {
                const int src = __ffs(cm) - 1;
                cm &= cm - 1;
                warp_list_insert(list, __shfl_sync(0xffffffffu, cand, src), 0xffffffffu);
              }
            } else {
              list = warp_merge_desc(list, warp_sort_desc(cand));
            }
            const unsigned long long kth = __shfl_sync(0xffffffffu, list, K - 1);
            thr_key = kth > thr_floor ? kth : thr_floor;
            thr_val = thr_key == kNoKey ? -INFINITY : key_value(thr_key);
            if (cand != kNoKey) last = cand;
          }
          if (stat) {
            // publish this run's K-th best value once the list is full
            const unsigned long long kth = __shfl_sync(0xffffffffu, list, K - 1);
            const uint32_t kv = (uint32_t)(kth >> 32);
            if (kth != kNoKey && kv > pub) {
              if (lane == 0) atomicMax(&prm.row_counter[r], kv);
              pub = kv;
            }
          }
        }
      }
      if ((FLAGS & kFStats1) && has1) {
        // Row 1 moves to registers; the stage is refilled while its terms run.
        LaneRow<T1> R;
        lane_load(st1p, nv, R);
        const float pm1 = lane_max(R);
        __syncwarp();
        ++n_consumed;
        top_up();
        lane_stats(st1, R, pm1, c);
      } else {
        __syncwarp();
        ++n_consumed;
        top_up();
      }
    }

    // The run ends at a row boundary, at the end of the warp's range, and
    // after every item in dynamic mode.
    {
    // Per-run reduction and record.
    Partial pr;
    pr.G0 = pr.G1 = -INFINITY;
    pr.S0 = pr.S1 = 0.0;
    if (FLAGS & kFStats0) {
      pr.G0 = warp_max_redux(st0.ref);
      pr.S0 = warp_sum(rescale_pow2(st0.S, st0.ref, pr.G0));
    }
    if (FLAGS & kFStats1) {
      pr.G1 = warp_max_redux(st1.ref);
      pr.S1 = warp_sum(rescale_pow2(st1.S, st1.ref, pr.G1));
    }
    pr.key = kNoKey;
    if (FLAGS & kFArgmax0) pr.key = warp_max_u64(bidx < 0 ? kNoKey : topk_key(best, bidx));
    pr.zx0 = pr.zx1 = 0.f;
    int flags = 0;
    if (FLAGS & kFGather) {
      const unsigned hm = __ballot_sync(0xffffffffu, hx != 0);
      if (hm) {
        const int src = __ffs(hm) - 1;
        pr.zx0 = __shfl_sync(0xffffffffu, zx0, src);
        pr.zx1 = __shfl_sync(0xffffffffu, zx1, src);
        flags |= kPHasX;
      }
    }
    if (cur_np == 0) flags |= kPSkipped;
    if (__any_sync(0xffffffffu, timeouts != 0)) flags |= kPTimeout;
    pr.flags = flags;
    pr.pad = 0;
    // Counting is deferred: the count of an item is added one item later,
    // when its record has long been written, and the returned count is read
    // one item after that.
    if (!stat) {
      resolve();
      signal();
    }
    if ((FLAGS & kFTopk0) && lane < K) prm.cand[(size_t)run_first * K + lane] = list;
    if (lane == 0) prm.part[run_first] = pr;
    sig_r = r;
    sig_x = L.x;
    timeouts = 0;
    run_first = -1;
    }

    // Advance: nxt becomes current; the item after it comes from the counter.
    cur = nxt;
    if (nxt_np < 0) nxt_np = pieces_of(nxt, nxt_rj, slot_cur ^ 1);
    slot_cur ^= 1;
    cur_np = nxt_np;
    cur_x = __shfl_sync(0xffffffffu, nxt_x, 0);
    if (iss_which == 0) iss_p = 0;
    iss_which = 0;
    nxt = nxt2;
    nxt_np = -1;
    nxt_rj = nxt2_rj;
    nxt_x = nxt2_x;
    nxt2 = nxt2 < total ? (stat ? next_run(nxt2) : take(pend)) : total;
    if (lane == 0) {
      prefetch(nxt2, nxt2_rj, nxt2_x);
      if (!stat && nxt2 < total) pend = fetch();
    }
    top_up();
  }
  // Count the last item and read the outstanding results.
  if (!stat) {
    resolve();
    signal();
    resolve();
  }
  // Any copy still in flight (only after a timed-out wait) completes before exit.
  if (use_bulk && lane == 0)
    while (n_consumed < n_issued) {
      mbar_wait_bounded(&bars[n_consumed % kStages], (n_consumed / kStages) & 1u);
      ++n_consumed;
    }
}

}  // namespace sv
