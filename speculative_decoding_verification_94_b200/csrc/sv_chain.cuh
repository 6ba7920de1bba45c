// sv_chain.cuh -- chain verification in one persistent launch (sm_100a).
//
// One CTA per SM: a producer warp and kCW consumer warps around a ring of
// `stages` shared-memory stages, and a manager warp that runs the completion
// work the consumers hand it (so a completion never holds up the ring).  A stage holds one tile: kTileW consecutive
// vocabulary entries of target row i of request b and, when the draft is given
// as logits, of draft row i (the pair the acceptance test at position i
// compares).  The producer's elected lane claims tiles from one global counter
// in position-major order (every request's position 0 first), skips the tiles
// of rows that no longer matter, and fills the stage with bulk asynchronous
// copies (cp.async.bulk, no multicast) completing on the stage's mbarrier.
// Each consumer warp reduces its kSliceW-element slice of the tile (online
// softmax statistics with exact power-of-two rescales, the values at the
// draft token, the argmax, the top-K keys); the last warp of the stage folds
// the warps' partials into one tile record, returns the stage, and counts the
// tile into its row.
//
// The warp that counts a row's last tile hands the row to its CTA's manager
// warp, which completes it: it folds the
// tiles' records in tile order (so the result does not depend on which CTA
// streamed which tile), takes the ratio test u * q(x) < p(x) in float64 (or
// compares x with the argmax), and ORs the outcome into the request's state
// word.  Rows of a request complete in any order; the one OR that makes the
// outcome known (a decided prefix ending in a rejection, or every draft
// accepted and the bonus row done) names that warp the request's finisher.
// Rows after a known rejection are never loaded (the producer reads the state
// word before it issues a tile), so the bytes read approach the rows the
// outcome depends on.
//
// Draws: a bonus draw (or a greedy outcome) is finished at once from the
// stream's tile records.  A rejection at position n < k_b queues a draw job:
// its kTileW-entry tiles of the row pair n are spread over the CTAs' private
// draw queues (tile d of the job list goes to CTA d mod grid), so every CTA
// takes part without contention; the producers serve their queue before they
// claim stream tiles.  Each draw tile yields the residual mass
// sum max(0, p - q) of its slices; the warp that counts the job's last tile
// scans the masses in vocabulary order and locates the drawn token inside one
// slice.  Every wait is bounded (a time limit, after which the call reports
// SV_DEV_TIMEOUT and stops issuing work), so no CTA waits forever.
#pragma once

#include "sv_rowops.cuh"
#include "sv_stream.cuh"

namespace sv {

#ifndef SV_CHAIN_CW
#define SV_CHAIN_CW 16
#endif
constexpr int kCW = SV_CHAIN_CW;             // consumer warps per CTA
// + the producer warp, the counter warp and the completer warp
constexpr int kChainThreads = (kCW + 3) * 32;
constexpr int kTaskQ = 256;                  // completion tasks queued per CTA
constexpr int kTileW = 8192;                 // vocabulary entries per tile and row
constexpr int kRowW = kCW / 2;               // warps per row when a tile holds a row pair
constexpr int kSliceP = kTileW / kRowW;      // entries per warp, one row of a pair tile
constexpr int kVPLP = kSliceP / (32 * kVec); // 8-entry vectors per lane for those
constexpr int kSliceW = kTileW / kCW;        // entries per warp, target-only and draw tiles
constexpr int kVPL = kSliceW / (32 * kVec);  // 8-entry vectors per lane for those
constexpr int kClaim = 4;                    // stream tiles claimed per atomic (4 measured a little faster than 2)
constexpr int kMaxStagesC = 8;
constexpr int kChainMaxK = 30;               // drafts per request (state word: 31 rows)

enum ChainMode : int { kCMSample = 0, kCMProbs = 1, kCMGreedy = 2 };
enum TileKind : int { kTKStream = 0, kTKDraw = 1, kTKIdle = 2, kTKExit = 3 };
// Global counters (first 256 B of the workspace).
enum GlobSlot : int { kGNext = 0, kGJobTail = 1, kGDet = 2, kGExit = 3, kGKd = 4, kGAbort = 5 };
constexpr unsigned long long kFinalBit = 1ull << 63;  // request state: outputs written

struct __align__(16) TileRec {
  float G0, G1;
  double S0, S1;
  float zx0, zx1;
  int flags;  // kPHasX | kPTimeout
  int pad;
  unsigned long long key;  // argmax key of the target row
};
static_assert(sizeof(TileRec) == 48, "tile record layout");

struct __align__(16) WarpStat {  // one warp's slice of a bonus row
  float G;
  float pad;
  double S;
};

struct __align__(16) DrawRec {
  double mass;        // tile residual mass (slices in order)
  double wm[kCW];     // per-slice masses
};

struct __align__(16) DrawJob {
  int b, n, kb, pad;
  float Gt, Gd, invSt, invSd;
};

struct __align__(16) StageDesc {
  int kind;
  int row;    // stream: b * P + i; draw: job; idle: b
  int tile;
  int len;    // entries of the tile
  int b, i, kb;
  int flags;  // kSDDraft: draft row staged; kSDBonus: the request's bonus row
};
enum : int { kSDDraft = 1, kSDBonus = 2 };

// Completion work handed from the consumer warps to the CTA's manager warp,
// so that a row completion or a draw never holds up the stage ring.
enum TaskKind : int { kTaskTile = 0, kTaskDraw = 1, kTaskIdle = 2 };
struct TaskQueue {
  int tail;            // tasks pushed (shared-memory atomic)
  int head;            // tasks taken (manager)
  int consumers_done;  // consumer warps that saw the exit stage
  int pad;
  int ready[kTaskQ];
  int4 task[kTaskQ];   // kind, b or job, i, kb
};

struct __align__(16) WarpPart {
  float G0, G1;
  double S0, S1;
  float zx0, zx1;
  int hx, tmo;
  unsigned long long key;
};

struct ChainParams {
  const void* target;   // [B, P, V]
  const void* draft;    // [B, k, V] logits or fp32 probabilities
  const int32_t* tokens;  // [B, k]
  const float* u;       // [B, P]
  const int32_t* klen;  // ragged draft counts (or null)
  const int32_t* active;  // ragged active mask (or null)
  int B, k, V, P, NT, total, order;
  FastDiv div_NT, div_B;
  float c;
  int use_bulk;
  int stages, stage_bytes, stage_off1;
  int off_bars, off_desc, off_done, off_parts, off_lists, off_tasks;
  int K;
  int32_t* accepted_len;
  int32_t* out_tokens;
  float* topk_logp;
  int32_t* topk_idx;
  float* lse;
  float* kl;
  const float* reward;
  int wmode, group;
  float clip;
  float* loss;
  float* total_out;
  int positions;
  int32_t* status;
  // workspace
  uint32_t* glob;
  unsigned long long* req_state;  // [B]
  uint32_t* pair_cnt;             // [B * P]
  RowRec* rows;                   // [B * P]
  TileRec* tiles;                 // [B * P * NT]
  WarpStat* bonus;                // [B * NT * kCW]
  DrawJob* jobs;                  // [B]
  uint32_t* job_cnt;              // [B]
  uint32_t* drawq;                // [B * NT]
  DrawRec* draws;                 // [B * NT]
  unsigned long long* cand;       // [B * P * NT * K]
  unsigned long long* rowthr;     // [B * P]
  float* st_logp;                 // [B * P * K]
  int32_t* st_idx;                // [B * P * K]
  float* st_lse;                  // [B * P]
  float* st_kl;                   // [B * k]
  unsigned long long wait_ns;
  int stall;
  unsigned char* ws_base;  // the whole workspace (cleared after a timeout)
  size_t ws_bytes;
};

// ---------------------------------------------------------------------------
// Small helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long atom_or_acq_rel_u64(unsigned long long* p,
                                                              unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.or.b64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ void red_or_release_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.or.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void red_add_release_u32(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// A 16-byte-aligned record written by another SM, read through L2.
template <class T>
__device__ __forceinline__ T ldcg_rec(const T* src) {
  static_assert(sizeof(T) % 16 == 0, "record size");
  T r;
  const uint4* q = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(&r);
#pragma unroll
  for (int t = 0; t < (int)(sizeof(T) / 16); ++t) d[t] = __ldcg(q + t);
  return r;
}

// try_wait without a suspend-time hint (the instruction's own bounded wait).
__device__ __forceinline__ uint32_t mbar_try_wait_spin(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok;
}

// Non-blocking test of phase `parity` of an mbarrier.
__device__ __forceinline__ uint32_t mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok;
}

// Wait for phase `parity` of an mbarrier, giving up after limit_ns.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity,
                                                unsigned long long limit_ns) {
  if (mbar_try_wait_spin(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_spin(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Request draft count: k, or klen[b]; -1 idle; -2 a draft count outside [0, k].
__device__ __forceinline__ int chain_kb(const ChainParams& p, int b) {
  if (p.active != nullptr && __ldg(&p.active[b]) == 0) return -1;
  if (p.klen == nullptr) return p.k;
  const int kb = __ldg(&p.klen[b]);
  return (kb < 0 || kb > p.k) ? -2 : kb;
}

// Outcome of a request from its state word (decided rows in bits 0..30,
// rejected-or-failed rows in bits 32..62): the first rejected row n when rows
// 0..n are decided, kb when rows 0..kb are decided without a rejection before
// kb, else -1 (not known yet).
__device__ __forceinline__ int chain_outcome(unsigned long long s, int kb) {
  const uint32_t dec = (uint32_t)s & 0x7fffffffu;
  const uint32_t rej = (uint32_t)(s >> 32) & 0x7fffffffu;
  const int fu = __ffs(~dec) - 1;  // first undecided row (bit 31 of ~dec is set)
  const int fr = rej ? __ffs(rej) - 1 : 32;
  if (fr < fu) return fr;
  if (fu > kb) return kb;
  return -1;
}

// Tile t of the stream -> (position i, request b, tile tau).
__device__ __forceinline__ void chain_decode(const ChainParams& p, int t, int& i, int& b,
                                             int& tau) {
  if (p.order == 0) {  // request-major inside a position, tiles innermost
    const int rb = fast_div(t, p.div_NT);
    tau = t - rb * p.NT;
    i = fast_div(rb, p.div_B);
    b = rb - i * p.B;
  } else {  // tile-major inside a position, requests innermost
    const int it = fast_div(t, p.div_B);
    b = t - it * p.B;
    i = fast_div(it, p.div_NT);
    tau = it - i * p.NT;
  }
}

template <class T>
__device__ __forceinline__ const unsigned char* chain_row(const void* base, size_t row, int V) {
  return reinterpret_cast<const unsigned char*>(base) + row * (size_t)V * T::bytes;
}

// ---------------------------------------------------------------------------
// A lane's share of a warp slice: kVPL vectors of 8 entries, vector v holding
// slice entries (v * 32 + lane) * 8 .. + 7.  Entries at or past `n` (the
// slice length) read as `pad`.  From shared memory (bulk path, 16-byte
// aligned rows) or straight from global memory (scalar path).
// ---------------------------------------------------------------------------
template <class T, int NV>
struct Slice;
template <int NV>
struct Slice<BF16, NV> {
  uint4 w[NV];
};
template <int NV>
struct Slice<F32, NV> {
  float4 w[2 * NV];
};

template <int NV>
__device__ __forceinline__ void slice_load(const unsigned char* src, int n, bool smem, float pad,
                                           Slice<BF16, NV>& R) {
  const int lane = threadIdx.x & 31;
  const uint16_t pb = (uint16_t)(__float_as_uint(pad) >> 16);
  if (smem && n >= NV * 256) {
#pragma unroll
    for (int v = 0; v < NV; ++v)
      R.w[v] = *reinterpret_cast<const uint4*>(src + (size_t)(v * 32 + lane) * 16);
    return;
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int e = (v * 32 + lane) * kVec;
    if (smem && e + kVec <= n) {
      R.w[v] = *reinterpret_cast<const uint4*>(src + (size_t)e * 2);
      continue;
    }
    uint32_t h[kVec];
#pragma unroll
    for (int t = 0; t < kVec; ++t)
      h[t] = (e + t < n) ? (uint32_t)reinterpret_cast<const uint16_t*>(src)[e + t] : (uint32_t)pb;
    R.w[v] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                        h[6] | (h[7] << 16));
  }
}

template <int NV>
__device__ __forceinline__ void slice_load(const unsigned char* src, int n, bool smem, float pad,
                                           Slice<F32, NV>& R) {
  const int lane = threadIdx.x & 31;
  if (smem && n >= NV * 256) {
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      R.w[2 * v] = *reinterpret_cast<const float4*>(src + (size_t)(v * 32 + lane) * 32);
      R.w[2 * v + 1] = *reinterpret_cast<const float4*>(src + (size_t)(v * 32 + lane) * 32 + 16);
    }
    return;
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int e = (v * 32 + lane) * kVec;
    float h[kVec];
#pragma unroll
    for (int t = 0; t < kVec; ++t)
      h[t] = (e + t < n) ? reinterpret_cast<const float*>(src)[e + t] : pad;
    R.w[2 * v] = make_float4(h[0], h[1], h[2], h[3]);
    R.w[2 * v + 1] = make_float4(h[4], h[5], h[6], h[7]);
  }
}

template <int NV>
__device__ __forceinline__ float slice_elem(const Slice<BF16, NV>& R, int v, int t) {
  const uint32_t w = (t >> 1) == 0 ? R.w[v].x : (t >> 1) == 1 ? R.w[v].y : (t >> 1) == 2 ? R.w[v].z
                                                                                       : R.w[v].w;
  return (t & 1) ? bf16_hi(w) : bf16_lo(w);
}
template <int NV>
__device__ __forceinline__ float slice_elem(const Slice<F32, NV>& R, int v, int t) {
  const float4 q = R.w[2 * v + (t >> 2)];
  const int u = t & 3;
  return u == 0 ? q.x : u == 1 ? q.y : u == 2 ? q.z : q.w;
}

template <int NV>
__device__ __forceinline__ float slice_vmax(const Slice<BF16, NV>& R, int v) {
  const uint32_t m = bmax2(bmax2(R.w[v].x, R.w[v].y), bmax2(R.w[v].z, R.w[v].w));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}
template <int NV>
__device__ __forceinline__ float slice_vmax(const Slice<F32, NV>& R, int v) {
  const float4 a = R.w[2 * v], b = R.w[2 * v + 1];
  return fmaxf(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), fmaxf(fmaxf(b.x, b.y), fmaxf(b.z, b.w)));
}
template <int NV>
__device__ __forceinline__ float slice_max(const Slice<BF16, NV>& R) {
  uint32_t m = bmax2(bmax2(R.w[0].x, R.w[0].y), bmax2(R.w[0].z, R.w[0].w));
#pragma unroll
  for (int v = 1; v < NV; ++v)
    m = bmax2(m, bmax2(bmax2(R.w[v].x, R.w[v].y), bmax2(R.w[v].z, R.w[v].w)));
  return fmaxf(bf16_lo(m), bf16_hi(m));
}
template <int NV>
__device__ __forceinline__ float slice_max(const Slice<F32, NV>& R) {
  float m = slice_vmax(R, 0);
#pragma unroll
  for (int v = 1; v < NV; ++v) m = fmaxf(m, slice_vmax(R, v));
  return m;
}

// Sum over the lane's entries of 2^(z c - ref): packed fma, two exp2, and a
// fixed tree of packed adds.
template <int NV>
__device__ __forceinline__ float slice_terms(const Slice<BF16, NV>& R, float c, float ref) {
  const unsigned long long cc = f2_pack(c, c), nr = f2_pack(-ref, -ref);
  unsigned long long e[4 * NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    e[4 * v + 0] = term2(bf16_lo(R.w[v].x), bf16_hi(R.w[v].x), cc, nr);
    e[4 * v + 1] = term2(bf16_lo(R.w[v].y), bf16_hi(R.w[v].y), cc, nr);
    e[4 * v + 2] = term2(bf16_lo(R.w[v].z), bf16_hi(R.w[v].z), cc, nr);
    e[4 * v + 3] = term2(bf16_lo(R.w[v].w), bf16_hi(R.w[v].w), cc, nr);
  }
#pragma unroll
  for (int w = 2 * NV; w >= 1; w >>= 1)
#pragma unroll
    for (int t = 0; t < w; ++t) e[t] = f2_add(e[t], e[t + w]);
  float lo, hi;
  f2_unpack(e[0], lo, hi);
  return lo + hi;
}
template <int NV>
__device__ __forceinline__ float slice_terms(const Slice<F32, NV>& R, float c, float ref) {
  const unsigned long long cc = f2_pack(c, c), nr = f2_pack(-ref, -ref);
  unsigned long long e[4 * NV];
#pragma unroll
  for (int v = 0; v < 2 * NV; ++v) {
    e[2 * v + 0] = term2(R.w[v].x, R.w[v].y, cc, nr);
    e[2 * v + 1] = term2(R.w[v].z, R.w[v].w, cc, nr);
  }
#pragma unroll
  for (int w = 2 * NV; w >= 1; w >>= 1)
#pragma unroll
    for (int t = 0; t < w; ++t) e[t] = f2_add(e[t], e[t + w]);
  float lo, hi;
  f2_unpack(e[0], lo, hi);
  return lo + hi;
}

// One row of a slice into a warp partial, against one reference for the
// warp: G = ceil(c * the slice maximum) (an integer, so later rescales are
// exact powers of two) and S = sum 2^(z c - G), fp32 per lane, float64 across
// the warp.  pm: the lane's maximum.
template <class T, int NV>
__device__ __forceinline__ void slice_stats(const Slice<T, NV>& R, float pm, float c, float* G,
                                            double* S) {
  const float wm = warp_max_redux(pm);
  if (wm == -INFINITY) {
    *G = -INFINITY;
    *S = 0.0;
    return;
  }
  const float g = ceilf(wm * c);
  *G = g;
  *S = warp_sum((double)slice_terms(R, c, g));
}

// ---------------------------------------------------------------------------
// Eight consecutive entries e..e+7 of a row segment (shared or global memory)
// widened to fp32; entries at or past n read as `pad`.  `vec`: the segment
// start is 16-byte aligned, so a whole group is one or two vector loads.
// ---------------------------------------------------------------------------
template <class T>
__device__ __forceinline__ void load8g(const unsigned char* src, int e, int n, bool vec,
                                       float pad, float v[8]);
template <>
__device__ __forceinline__ void load8g<BF16>(const unsigned char* src, int e, int n, bool vec,
                                             float pad, float v[8]) {
  if (vec && e + 8 <= n) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + (size_t)e * 2);
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
    return;
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) v[t] = (e + t < n) ? load1<BF16>(src, e + t) : pad;
}
template <>
__device__ __forceinline__ void load8g<F32>(const unsigned char* src, int e, int n, bool vec,
                                            float pad, float v[8]) {
  if (vec && e + 8 <= n) {
    const float4 a = *reinterpret_cast<const float4*>(src + (size_t)e * 4);
    const float4 b = *reinterpret_cast<const float4*>(src + (size_t)e * 4 + 16);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    return;
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) v[t] = (e + t < n) ? load1<F32>(src, e + t) : pad;
}

// Residual weights of 8 consecutive entries (the same rounding in the mass
// pass and in the locate pass): p = 2^(zt c - Gt) / St and q alike, products
// explicitly rounded so that p - q is exactly 0 when p == q.  Entries past n
// weigh 0.
template <class TT, class DT, int MODE>
__device__ __forceinline__ void resid8(const unsigned char* tsrc, const unsigned char* dsrc, int e,
                                       int n, bool vec, float c, float Gt, float invSt, float Gd,
                                       float invSd, float w[8]) {
  float zt[8], zd[8];
  load8g<TT>(tsrc, e, n, vec, -INFINITY, zt);
  if (MODE == kCMProbs) load8g<F32>(dsrc, e, n, vec, 0.f, zd);
  else load8g<DT>(dsrc, e, n, vec, -INFINITY, zd);
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const float p = __fmul_rn(ex2(fmaf(zt[t], c, -Gt)), invSt);
    const float q = (MODE == kCMProbs) ? zd[t] : __fmul_rn(ex2(fmaf(zd[t], c, -Gd)), invSd);
    w[t] = (e + t < n) ? fmaxf(__fsub_rn(p, q), 0.f) : 0.f;
  }
}

// Unnormalised target terms 2^(z c - G) of 8 consecutive entries.
template <class TT>
__device__ __forceinline__ void pterm8(const unsigned char* tsrc, int e, int n, bool vec, float c,
                                       float G, float w[8]) {
  float z[8];
  load8g<TT>(tsrc, e, n, vec, -INFINITY, z);
#pragma unroll
  for (int t = 0; t < 8; ++t) w[t] = (e + t < n) ? ex2(fmaf(z[t], c, -G)) : 0.f;
}

__device__ __forceinline__ float seq8(const float w[8]) {
  float s = w[0];
#pragma unroll
  for (int t = 1; t < 8; ++t) s = __fadd_rn(s, w[t]);
  return s;
}

// Locate a draw inside one slice (warp-collective).  The slice's 8-entry
// groups are visited in vocabulary order; `base` is the mass before the
// slice and `target` the draw's position on the cumulative mass.  WF fills a
// group's weights.  Returns the slice entry, or the last entry with positive
// weight when rounding leaves the target past the slice's total, or -1.
template <class WF>
__device__ __forceinline__ int slice_locate(int n, double base, double target, WF wf) {
  const int lane = threadIdx.x & 31;
  int found = -1, lastpos = -1;
  for (int v = 0; v < kVPL; ++v) {
    const int e = (v * 32 + lane) * kVec;
    float w[8];
    wf(e, w);
    const float s = seq8(w);
    double incl = (double)s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const double before = base + incl - (double)s;
    const unsigned hit = __ballot_sync(0xffffffffu, base + incl > target && s > 0.f);
    const unsigned pos = __ballot_sync(0xffffffffu, s > 0.f);
    if (pos) {
      const int src = 31 - __clz(pos);
      int lp = -1;
      if (lane == src)
#pragma unroll
        for (int t = 0; t < 8; ++t)
          if (w[t] > 0.f) lp = e + t;
      lastpos = __shfl_sync(0xffffffffu, lp, src);
    }
    if (hit) {
      const int src = __ffs(hit) - 1;
      int pick = -1;
      if (lane == src) {
        float a = 0.f;
        int lq = -1;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          a = __fadd_rn(a, w[t]);
          if (w[t] > 0.f) lq = t;
          if (pick < 0 && before + (double)a > target) pick = t;
        }
        if (pick < 0) pick = lq;
        pick = pick < 0 ? -1 : e + pick;
      }
      found = __shfl_sync(0xffffffffu, pick, src);
      break;
    }
    base = __shfl_sync(0xffffffffu, incl, 31) + base;
  }
  (void)n;
  return found >= 0 ? found : lastpos;
}

// ---------------------------------------------------------------------------
// Returning records to zero (warp-collective).  Every record a call writes is
// cleared by its last reader, so the workspace is all zero between calls:
// a row's tile records and top-K lists by the warp that folds them; the
// bonus row's (kept for the draw) by the draw, or by whoever learns that the
// request ended earlier; row records and staged KD rows after the outputs are
// written; rows streamed in part and then skipped by the last CTA.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void zero_tiles(const ChainParams& p, int r) {
  const int lane = threadIdx.x & 31;
  for (int q = lane; q < p.NT; q += 32) p.tiles[(size_t)r * p.NT + q] = TileRec{};
}
__device__ __forceinline__ void zero_bonus(const ChainParams& p, int b) {
  const int lane = threadIdx.x & 31;
  for (int q = lane; q < p.NT * kCW; q += 32) p.bonus[(size_t)b * p.NT * kCW + q] = WarpStat{};
}
template <bool KD>
__device__ __forceinline__ void zero_lists(const ChainParams& p, int r) {
  if (!KD) return;
  const int lane = threadIdx.x & 31;
  const size_t n = (size_t)p.NT * p.K;
  for (size_t q = lane; q < n; q += 32) p.cand[(size_t)r * n + q] = 0ull;
  if (lane == 0) p.rowthr[r] = 0ull;
}
// The row record and staged KD outputs of row i of request b.
template <bool KD>
__device__ __forceinline__ void zero_row(const ChainParams& p, int b, int i) {
  const int lane = threadIdx.x & 31;
  const int r = b * p.P + i;
  if (lane == 0) p.rows[r] = RowRec{};
  if (KD) {
    if (lane < p.K) {
      p.st_logp[(size_t)r * p.K + lane] = 0.f;
      p.st_idx[(size_t)r * p.K + lane] = 0;
    }
    if (lane == 0) {
      p.st_lse[r] = 0.f;
      if (i < p.k) p.st_kl[(size_t)b * p.k + i] = 0.f;
    }
  }
}
// Row i of request b completed but is not part of the outcome: its record,
// staged rows and, for a sampling bonus row, the tile sums kept for the draw.
template <int MODE, bool KD>
__device__ __forceinline__ void drop_row(const ChainParams& p, int b, int i, int kb) {
  zero_row<KD>(p, b, i);
  if (MODE != kCMGreedy && i == kb) {
    zero_tiles(p, b * p.P + i);
    zero_bonus(p, b);
  }
}

// ---------------------------------------------------------------------------
// Outputs of a finished request (warp-collective).  nn: accepted drafts, or
// -1 for a failed request; kb == -1 (idle) reports 0 accepted.
// ---------------------------------------------------------------------------
template <bool KD>
__device__ __noinline__ void chain_write_outputs(const ChainParams& p, int b, int kb, int nn,
                                                 int tok, int nz) {
  const int lane = threadIdx.x & 31;
  const int P = p.P, k = p.k;
  if (nn >= 0 && (tok < 0 || tok >= p.V)) nn = -1;
  if (lane == 0) p.accepted_len[b] = kb == -1 ? 0 : nn;
  for (int t = lane; t < P; t += 32) {
    int v = -1;
    if (nn >= 0) v = t < nn ? __ldg(&p.tokens[(size_t)b * k + t]) : (t == nn ? tok : -1);
    p.out_tokens[(size_t)b * P + t] = v;
  }
  if (KD) {
    const int K = p.K;
    const int first_undef = nn < 0 ? 0 : nn + 1;
    for (int q = lane; q < P * K; q += 32) {
      const int t = q / K;
      const size_t o = (size_t)b * P * K + q;
      const bool def = t < first_undef;
      p.topk_logp[o] = def ? __ldcg(&p.st_logp[o]) : NAN;
      p.topk_idx[o] = def ? __ldcg(&p.st_idx[o]) : -1;
    }
    for (int t = lane; t < P; t += 32)
      p.lse[(size_t)b * P + t] = t < first_undef ? __ldcg(&p.st_lse[(size_t)b * P + t]) : NAN;
    const int kl_def = min(first_undef, kb < 0 ? 0 : kb);
    for (int t = lane; t < k; t += 32)
      p.kl[(size_t)b * k + t] = t < kl_def ? __ldcg(&p.st_kl[(size_t)b * k + t]) : NAN;
    // the request's loss over its KD positions, then (last request) the total
    int last = 0;
    if (lane == 0) {
      const int m = (p.positions && nn >= 0 && nn < kb) ? nn + 1 : nn;
      double s = 0.0;
      for (int i = 0; i < m; ++i) s += (double)__ldcg(&p.st_kl[(size_t)b * k + i]);
      const double w = (nn < 0) ? 0.0 : reward_weight(p.reward, b, p.wmode, p.group, p.clip);
      p.loss[b] = (w == 0.0) ? 0.f : (float)(w * s);
      fence_acq_rel_gpu();
      last = atomicAdd(&p.glob[kGKd], 1u) == (uint32_t)p.B - 1u;
      if (last) fence_acq_rel_gpu();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      double part = 0.0;
      for (int t = lane; t < p.B; t += 32) part += (double)__ldcg(&p.loss[t]);
      part = warp_sum(part);
      if (lane == 0) *p.total_out = (float)part;
    }
  }
  // the decided prefix's records are no longer read
  __syncwarp();
  for (int i = 0; i < nz; ++i) zero_row<KD>(p, b, i);
  __syncwarp();
  if (lane == 0) red_or_release_u64(&p.req_state[b], kFinalBit);
}

// ---------------------------------------------------------------------------
// Pick the segment holding `target` on a cumulative mass (warp-collective):
// segments 0..n-1 with masses m(q) (every lane evaluates its own q), scanned
// in order from `base`.  Returns the first segment whose cumulative mass
// exceeds the target and sets *before to the mass before it; when rounding
// leaves the target past the total, the last segment with positive mass.
// -1 when every mass is 0.
// ---------------------------------------------------------------------------
template <class MF>
__device__ __forceinline__ int scan_pick(int n, double base, double target, MF mf,
                                         double* before) {
  const int lane = threadIdx.x & 31;
  int lastpos = -1;
  double lastbase = 0.0;
  for (int q0 = 0; q0 < n; q0 += 32) {
    const int q = q0 + lane;
    const double m = q < n ? mf(q) : 0.0;
    const double incl = warp_scan_incl(m);
    const unsigned hit = __ballot_sync(0xffffffffu, q < n && m > 0.0 && base + incl > target);
    const unsigned pos = __ballot_sync(0xffffffffu, q < n && m > 0.0);
    if (hit) {
      const int src = __ffs(hit) - 1;
      *before = base + __shfl_sync(0xffffffffu, incl - m, src);
      return q0 + src;
    }
    if (pos) {
      const int src = 31 - __clz(pos);
      lastpos = q0 + src;
      lastbase = base + __shfl_sync(0xffffffffu, incl - m, src);
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  *before = lastbase;
  return lastpos;
}

// ---------------------------------------------------------------------------
// Draw from the target row r = b * P + i (unnormalised terms 2^(z c - Gt),
// target u * St), from the stream's tile sums: the tile by a scan of the
// tiles' sums, the slice by the bonus row's per-warp sums (or, without them,
// by recomputing the tile's slices), the entry by recomputing the slice.
// ---------------------------------------------------------------------------
template <class TT>
__device__ __noinline__ int chain_pdraw(const ChainParams& p, int b, int i, float uu,
                                        bool from_records) {
  const int lane = threadIdx.x & 31;
  const int r = b * p.P + i;
  const RowRec rr = ldcg_rec(&p.rows[r]);
  const float Gt = rr.G0;
  const double target = (double)uu * rr.S0;
  const float c = p.c;
  const int V = p.V, NT = p.NT;
  const bool vec = p.use_bulk != 0;
  const unsigned char* row = chain_row<TT>(p.target, (size_t)r, V);
  // mass of slice w of tile tau, recomputed from the logits (warp-collective)
  auto slice_mass = [&](int tau, int w) -> double {
    const int t0 = tau * kTileW + w * kSliceW;
    const int n = max(0, min(kSliceW, V - t0));
    double a = 0.0;
    for (int v = 0; v < kVPL; ++v) {
      float wv[8];
      pterm8<TT>(row + (size_t)t0 * TT::bytes, (v * 32 + lane) * kVec, n, vec, c, Gt, wv);
      a += (double)seq8(wv);
    }
    return warp_sum(a);
  };
  double base = 0.0;
  int tau = -1;
  double sm = 0.0;  // lane w: mass of slice w of tile tau
  if (from_records) {
    // the stream's tile sums, then the bonus row's per-warp sums
    tau = scan_pick(NT, 0.0, target, [&](int q) {
      const TileRec tr = ldcg_rec(&p.tiles[(size_t)r * NT + q]);
      return rescale_pow2(tr.S0, tr.G0, Gt);
    }, &base);
    if (tau < 0) return -1;
    const int nsl = (min(kTileW, V - tau * kTileW) + kSliceW - 1) / kSliceW;
    if (lane < nsl) {
      const WarpStat ws = ldcg_rec(&p.bonus[((size_t)b * NT + tau) * kCW + lane]);
      sm = rescale_pow2(ws.S, ws.G, Gt);
    }
  } else {
    // recomputed tile by tile (the rare zero-residual fallback)
    int lastpos = -1;
    double lastbase = 0.0;
    for (int q = 0; q < NT && tau < 0; ++q) {
      const int nsl = (min(kTileW, V - q * kTileW) + kSliceW - 1) / kSliceW;
      double tm = 0.0, mine = 0.0;
      for (int w = 0; w < nsl; ++w) {
        const double m = slice_mass(q, w);
        if (lane == w) mine = m;
        tm += m;
      }
      if (tm > 0.0 && base + tm > target) {
        tau = q;
        sm = mine;
      } else {
        if (tm > 0.0) {
          lastpos = q;
          lastbase = base;
        }
        base += tm;
      }
    }
    if (tau < 0 && lastpos >= 0) {
      tau = lastpos;
      base = lastbase;
      const int nsl = (min(kTileW, V - tau * kTileW) + kSliceW - 1) / kSliceW;
      for (int w = 0; w < nsl; ++w) {
        const double m = slice_mass(tau, w);
        if (lane == w) sm = m;
      }
    }
    if (tau < 0) return -1;
  }
  const int t0 = tau * kTileW;
  const int tlen = min(kTileW, V - t0);
  const int nsl = (tlen + kSliceW - 1) / kSliceW;
  double before = 0.0;
  // (one pass: nsl <= kCW <= 32, so lane q evaluates slice q)
  const int sl = scan_pick(nsl, base, target, [&](int) { return sm; }, &before);
  if (sl < 0) return -1;
  const int s0 = sl * kSliceW;
  const int n = min(kSliceW, tlen - s0);
  const unsigned char* src = row + (size_t)(t0 + s0) * TT::bytes;
  const int e = slice_locate(n, before, target, [&](int e8, float w8[8]) {
    pterm8<TT>(src, e8, n, vec, c, Gt, w8);
  });
  return e < 0 ? -1 : t0 + s0 + e;
}

// ---------------------------------------------------------------------------
// A request whose outcome is known (warp-collective): write its outputs, or
// queue its residual draw.  n: the outcome (chain_outcome).
// ---------------------------------------------------------------------------
template <class TT, class DT, int MODE, bool KD>
__device__ __noinline__ void chain_finish_request(const ChainParams& p, int b, int n,
                                                  unsigned long long st, const RowRec* known) {
  const int lane = threadIdx.x & 31;
  const int kb = chain_kb(p, b);
  // rows after the outcome that have completed already are not part of it
  const uint32_t dec = (uint32_t)st & 0x7fffffffu;
  for (int i = n + 1; i < p.P; ++i)
    if ((dec >> i) & 1u) drop_row<MODE, KD>(p, b, i, kb);
  const RowRec rn = known ? *known : ldcg_rec(&p.rows[b * p.P + n]);
  const bool failed = rn.code == kRowError;
  if (failed || MODE == kCMGreedy || n == kb) {
    int tok = -1;
    if (!failed && MODE == kCMGreedy) tok = rn.argmax;
    if (!failed && MODE != kCMGreedy) {
      const float uu = __ldg(&p.u[(size_t)b * p.P + kb]);
      tok = chain_pdraw<TT>(p, b, n, uu, true);
    }
    if (MODE != kCMGreedy && n == kb) {  // the tile sums kept for the draw
      __syncwarp();
      zero_tiles(p, b * p.P + kb);
      zero_bonus(p, b);
    }
    chain_write_outputs<KD>(p, b, kb, failed ? -1 : n, tok, n + 1);
  } else {
    // a rejection at n < kb: queue the residual draw over the row pair n
    int j = 0;
    if (lane == 0) {
      j = (int)atomicAdd(&p.glob[kGJobTail], 1u);
      DrawJob d;
      d.b = b;
      d.n = n;
      d.kb = kb;
      d.pad = 0;
      d.Gt = rn.G0;
      d.Gd = rn.G1;
      d.invSt = (float)(1.0 / rn.S0);
      d.invSd = (MODE == kCMSample) ? (float)(1.0 / rn.S1) : 1.f;
      p.jobs[j] = d;
    }
    __syncwarp();  // the job record before every lane's release of an entry
    j = __shfl_sync(0xffffffffu, j, 0);
    // each tile's queue entry names the row pair, so that a producer can
    // issue the copies as soon as it sees the entry
    const uint32_t flag = 1u + (uint32_t)(b * p.P + n);
    for (int q = lane; q < p.NT; q += 32) st_release_u32(&p.drawq[(size_t)j * p.NT + q], flag);
  }
  __syncwarp();
  if (lane == 0) red_add_release_u32(&p.glob[kGDet], 1u);
}

// ---------------------------------------------------------------------------
// Row completion (warp-collective): fold the row's tile records, decide the
// row, stage the KD outputs, publish the outcome to the request's state word,
// and finish the request when this row made its outcome known.
// ---------------------------------------------------------------------------
template <class TT, class DT, int MODE, bool KD>
__device__ __noinline__ void chain_complete_row(const ChainParams& p, int b, int i, int kb) {
  const int lane = threadIdx.x & 31;
  const int r = b * p.P + i, NT = p.NT, V = p.V;
  const bool has_draft = (MODE == kCMSample) && i < kb;
  // the loads the decision needs, issued with the records'
  const int x = i < kb ? __ldg(&p.tokens[(size_t)b * p.k + i]) : -1;
  const float u_i = (MODE != kCMGreedy && i < kb) ? __ldg(&p.u[(size_t)b * p.P + i]) : 0.f;
  float g0 = -INFINITY, g1 = -INFINITY, zx0 = 0.f, zx1 = 0.f;
  double s0 = 0.0, s1 = 0.0;
  int flags = 0, hx = 0;
  unsigned long long key = kNoKey;
  for (int q = lane; q < NT; q += 32) {
    const TileRec tr = ldcg_rec(&p.tiles[(size_t)r * NT + q]);
    if (tr.G0 > g0) {
      s0 = rescale_pow2(s0, g0, tr.G0);
      g0 = tr.G0;
    }
    s0 += rescale_pow2(tr.S0, tr.G0, g0);
    if (tr.G1 > g1) {
      s1 = rescale_pow2(s1, g1, tr.G1);
      g1 = tr.G1;
    }
    s1 += rescale_pow2(tr.S1, tr.G1, g1);
    flags |= tr.flags;
    if (tr.flags & kPHasX) {
      hx = 1;
      zx0 = tr.zx0;
      zx1 = tr.zx1;
    }
    key = tr.key > key ? tr.key : key;
  }
  RowRec rec;
  rec.G0 = warp_max(g0);
  rec.G1 = warp_max(g1);
  rec.S0 = warp_sum(rescale_pow2(s0, g0, rec.G0));
  rec.S1 = warp_sum(rescale_pow2(s1, g1, rec.G1));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) flags |= __shfl_xor_sync(0xffffffffu, flags, o);
  key = warp_max_u64(key);
  const unsigned hm = __ballot_sync(0xffffffffu, hx != 0);
  if (hm) {
    const int src = __ffs(hm) - 1;
    zx0 = __shfl_sync(0xffffffffu, zx0, src);
    zx1 = __shfl_sync(0xffffffffu, zx1, src);
  }
  rec.L0 = (double)rec.G0 + log2(rec.S0);
  rec.L1 = (double)rec.G1 + log2(rec.S1);
  rec.argmax = key_index(key);
  int err = 0, code = kRowAccepted;
  if (flags & kPTimeout) err |= SV_DEV_TIMEOUT;
  if (MODE != kCMGreedy && rec.G0 == -INFINITY) err |= SV_DEV_NO_FINITE;
  if (has_draft && rec.G1 == -INFINITY) err |= SV_DEV_NO_FINITE;
  if (i < kb) {
    if (x < 0 || x >= V || !hm) err |= SV_DEV_BAD_TOKEN;
    if (!err) {
      if (MODE == kCMGreedy) {
        code = (x == rec.argmax) ? kRowAccepted : kRowRejected;
      } else {
        const double cc = (double)p.c;
        const double px = exp2((double)zx0 * cc - rec.L0);
        const double qx =
            (MODE == kCMSample)
                ? exp2((double)zx1 * cc - rec.L1)
                : (double)__ldg(reinterpret_cast<const float*>(p.draft) + ((size_t)b * p.k + i) * V + x);
        const double uu = (double)u_i;
        code = (uu * qx < px) ? kRowAccepted : kRowRejected;
      }
    }
  } else if (MODE == kCMGreedy && key == kNoKey) {
    err |= SV_DEV_NO_FINITE;
  }
  if (MODE == kCMGreedy && i < kb && key == kNoKey) err |= SV_DEV_NO_FINITE;
  if (err) code = kRowError;
  rec.code = code;
  if (lane == 0) {
    p.rows[r] = rec;
    if (err) set_status(p.status, err);
  }
  if (KD) {
    // top-K of the target row from its tiles' lists (heads first), staged
    const int K = p.K;
    unsigned long long list = kNoKey;
    for (int q0 = 0; q0 < NT; q0 += 32) {
      const int q = q0 + lane;
      const unsigned long long h = q < NT ? __ldcg(&p.cand[((size_t)r * NT + q) * K]) : kNoKey;
      list = warp_merge_desc(list, warp_sort_desc(h));
    }
    unsigned long long thr = __shfl_sync(0xffffffffu, list, K - 1);
    for (int q0 = 0; q0 < NT; q0 += 32) {
      const int q = q0 + lane;
      const unsigned long long h = q < NT ? __ldcg(&p.cand[((size_t)r * NT + q) * K]) : kNoKey;
      unsigned msk = __ballot_sync(0xffffffffu, h > thr);
      while (msk) {
        const int src = __ffs(msk) - 1;
        msk &= msk - 1;
        const int qq = q0 + src;
        // entries 1..K-1 of that list (its head is merged), descending
        const unsigned long long y =
            (lane + 1 < K) ? __ldcg(&p.cand[((size_t)r * NT + qq) * K + lane + 1]) : kNoKey;
        list = warp_merge_desc(list, y);
        thr = __shfl_sync(0xffffffffu, list, K - 1);
        msk &= __ballot_sync(0xffffffffu, h > thr);
      }
    }
    const double ln2 = 0.69314718055994530942;
    double lp = -INFINITY;
    int j = -1;
    if (lane < K) {
      j = key_index(list);
      lp = ((double)key_value(list) * (double)p.c - rec.L0) * ln2;
      p.st_logp[(size_t)r * K + lane] = (float)lp;
      p.st_idx[(size_t)r * K + lane] = j;
    }
    if (lane == 0) p.st_lse[r] = (float)(rec.L0 * ln2);
    if (i < kb) {
      // KL(p~ || q) of draft row i over the renormalised top-K of target row i
      double mx = lp;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      double se = (lane < K) ? exp(lp - mx) : 0.0;
      se = warp_sum(se);
      const double lse_k = mx + log(se);
      double term = 0.0;
      if (lane < K && j >= 0 && j < V) {
        const double log_pt = lp - lse_k;
        const double pt = exp(log_pt);
        double log_q;
        if (MODE == kCMSample) {
          const float zd = load1<DT>(chain_row<DT>(p.draft, (size_t)b * p.k + i, V), j);
          log_q = ((double)zd * (double)p.c - rec.L1) * ln2;
        } else {
          log_q = log((double)__ldg(reinterpret_cast<const float*>(p.draft) +
                                    ((size_t)b * p.k + i) * V + j));
        }
        term = (pt == 0.0) ? 0.0 : pt * (log_pt - log_q);
      }
      term = warp_sum(term);
      if (lane == 0) p.st_kl[(size_t)b * p.k + i] = (float)term;
    }
  }
  // the tile records and lists are folded (a sampling bonus row keeps its
  // tile sums for the draw); the row's count is complete
  __syncwarp();
  if (!(MODE != kCMGreedy && i == kb)) zero_tiles(p, r);
  zero_lists<KD>(p, r);
  if (lane == 0) p.pair_cnt[r] = 0u;
  // publish the row's outcome (release: the row record and staged rows
  // first; acquire: the rows published before); the OR that makes the
  // request's outcome known names this warp its finisher
  __syncwarp();
  int before = -1, after = -1;
  unsigned long long now = 0ull;
  if (lane == 0) {
    const unsigned long long bits =
        (1ull << i) | ((code != kRowAccepted) ? (1ull << (32 + i)) : 0ull);
    const unsigned long long old = atom_or_acq_rel_u64(&p.req_state[b], bits);
    now = old | bits;
    before = chain_outcome(old, kb);
    after = chain_outcome(now, kb);
  }
  before = __shfl_sync(0xffffffffu, before, 0);
  after = __shfl_sync(0xffffffffu, after, 0);
  now = __shfl_sync(0xffffffffu, now, 0);
  if (before >= 0) drop_row<MODE, KD>(p, b, i, kb);  // completed after the outcome was known
  else if (after >= 0) chain_finish_request<TT, DT, MODE, KD>(p, b, after, now, after == i ? &rec : nullptr);
}

// ---------------------------------------------------------------------------
// Residual draw of job j after its last tile (warp-collective): the total
// residual mass R, the tile and then the slice holding u * R, and the entry
// inside the slice.  R == 0 (impossible when x ~ q) draws from p instead.
// ---------------------------------------------------------------------------
template <class TT, class DT, int MODE, bool KD>
__device__ __noinline__ void chain_locate(const ChainParams& p, int j) {
  const int lane = threadIdx.x & 31;
  const DrawJob d = ldcg_rec(&p.jobs[j]);
  const int b = d.b, n = d.n, kb = d.kb, NT = p.NT, V = p.V;
  const float uu = __ldg(&p.u[(size_t)b * p.P + kb]);
  const DrawRec* dr = p.draws + (size_t)j * NT;
  double R = 0.0;
  for (int q0 = 0; q0 < NT; q0 += 32) {
    const int q = q0 + lane;
    const double m = q < NT ? __ldcg(&dr[q].mass) : 0.0;
    R += __shfl_sync(0xffffffffu, warp_scan_incl(m), 31);
  }
  int tok = -1;
  if (!(R > 0.0)) {
    if (lane == 0) set_status(p.status, SV_DEV_RESIDUAL_ZERO);
    tok = chain_pdraw<TT>(p, b, n, uu, false);
  } else {
    const double target = (double)uu * R;
    double base = 0.0;
    const int tau = scan_pick(NT, 0.0, target, [&](int q) { return __ldcg(&dr[q].mass); }, &base);
    if (tau >= 0) {
      const int t0 = tau * kTileW;
      const int tlen = min(kTileW, V - t0);
      const int nsl = (tlen + kSliceW - 1) / kSliceW;
      const double sm = lane < nsl ? __ldcg(&dr[tau].wm[lane]) : 0.0;
      double before = 0.0;
      const int sl = scan_pick(nsl, base, target, [&](int) { return sm; }, &before);
      if (sl >= 0) {
        const int s0 = sl * kSliceW;
        const int ns = min(kSliceW, tlen - s0);
        const unsigned char* ts = chain_row<TT>(p.target, (size_t)b * p.P + n, V) +
                                  (size_t)(t0 + s0) * TT::bytes;
        const unsigned char* ds =
            (MODE == kCMProbs)
                ? chain_row<F32>(p.draft, (size_t)b * p.k + n, V) + (size_t)(t0 + s0) * 4
                : chain_row<DT>(p.draft, (size_t)b * p.k + n, V) + (size_t)(t0 + s0) * DT::bytes;
        const float c = p.c;
        const bool vec = p.use_bulk != 0;
        const int e = slice_locate(ns, before, target, [&](int e8, float w8[8]) {
          resid8<TT, DT, MODE>(ts, ds, e8, ns, vec, c, d.Gt, d.invSt, d.Gd, d.invSd, w8);
        });
        tok = e < 0 ? -1 : t0 + s0 + e;
      }
    }
  }
  chain_write_outputs<KD>(p, b, kb, n, tok, n + 1);
  // the job's records are read by nobody else now
  for (int q = lane; q < NT; q += 32) p.draws[(size_t)j * NT + q] = DrawRec{};
  if (lane == 0) {
    p.jobs[j] = DrawJob{};
    p.job_cnt[j] = 0u;
  }
}

// ---------------------------------------------------------------------------
// The kernel.
// ---------------------------------------------------------------------------

// Atomic add with release semantics (this thread's earlier writes, and those
// it has observed, are visible device-wide before the add); the returned
// value is read only when needed.
__device__ __forceinline__ uint32_t atom_add_release(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Push a task into a shared-memory queue (one thread; waits, bounded, for
// room).
__device__ __forceinline__ void queue_push(TaskQueue* q, int4 task, const ChainParams& p) {
  const int slot = atomicAdd(&q->tail, 1);
  const uint64_t t0 = globaltimer_ns();
  while (slot - *reinterpret_cast<volatile int*>(&q->head) >= kTaskQ) {
    if (globaltimer_ns() - t0 > p.wait_ns) {
      set_status(p.status, SV_DEV_TIMEOUT);
      atomicExch(&p.glob[kGAbort], 1u);
      break;
    }
    __nanosleep(128);
  }
  q->task[slot % kTaskQ] = task;
  __threadfence_block();
  *reinterpret_cast<volatile int*>(&q->ready[slot % kTaskQ]) = 1;
}

// One consumer warp's share of a stream tile: its slice of the target row or,
// for a tile holding a row pair, of the draft row.
template <class TT, class DT, int MODE, bool KD, int NV>
__device__ __forceinline__ void chain_slice(const ChainParams& p, const StageDesc& sd,
                                            const unsigned char* st, bool use_bulk, int warp,
                                            WarpPart& wp, unsigned long long* list_out) {
  const int lane = threadIdx.x & 31;
  constexpr int SW = NV * 256;
  const bool pair = (sd.flags & kSDDraft) != 0;
  const bool drow = pair && warp >= kRowW;       // this warp reduces the draft row
  const int wi = drow ? warp - kRowW : warp;     // slice index inside the row
  const int e0 = wi * SW;
  const int n = max(0, min(SW, sd.len - e0));
  const int t0e = sd.tile * kTileW + e0;
  const int x = sd.i < sd.kb ? __ldg(&p.tokens[(size_t)sd.b * p.k + sd.i]) : -1;
  const bool hasx = x >= t0e && x < t0e + n;
  if (!drow) {
    const unsigned char* src =
        use_bulk ? st + (size_t)e0 * TT::bytes
                 : chain_row<TT>(p.target, (size_t)sd.row, p.V) + (size_t)t0e * TT::bytes;
    Slice<TT, NV> R;
    slice_load(src, n, use_bulk, -INFINITY, R);
    const float pm = slice_max(R);
    if (MODE != kCMGreedy) {
      slice_stats(R, pm, p.c, &wp.G0, &wp.S0);
    } else {
      int bi = -1;
      if (pm != -INFINITY) {
#pragma unroll
        for (int v = NV - 1; v >= 0; --v)
#pragma unroll
          for (int t = kVec - 1; t >= 0; --t)
            if (slice_elem(R, v, t) == pm) bi = (v * 32 + lane) * kVec + t;
      }
      wp.key = warp_max_u64(bi < 0 ? kNoKey : topk_key(pm, t0e + bi));
    }
    if (KD) {
      // top-K keys of the slice above the row's running threshold and the
      // slice floor (the smallest lane maximum: every lane holds an entry at
      // least that large, so the slice's K best are too)
      const int K = p.K;
      const unsigned long long rthr = ld_relaxed_u64(&p.rowthr[sd.row]);
      const float fl = order_float(__reduce_min_sync(0xffffffffu, float_order(pm)));
      const unsigned long long floor_key =
          fl == -INFINITY ? kNoKey : ((unsigned long long)float_order(fl) << 32);
      unsigned long long thr = rthr;
      if (floor_key > 0ull && floor_key - 1ull > thr) thr = floor_key - 1ull;
      unsigned long long list = kNoKey;
      unsigned pmask = 0;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const float vm = slice_vmax(R, v);
        const unsigned long long vk = ((unsigned long long)float_order(vm) << 32) | 0xffffffffull;
        if (vm != -INFINITY && vk > thr) pmask |= 1u << v;
      }
      unsigned long long last = ~0ull;
      while (__any_sync(0xffffffffu, pmask != 0)) {
        unsigned long long cnd = kNoKey;
        int more = 0;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          if (!(pmask & (1u << v))) continue;
          const int ev = (v * 32 + lane) * kVec;
#pragma unroll
          for (int t = 0; t < kVec; ++t) {
            if (ev + t < n) {
              const unsigned long long kk = topk_key(slice_elem(R, v, t), t0e + ev + t);
              if (kk > thr && kk < last) {
                more += cnd != kNoKey;
                if (kk > cnd) cnd = kk;
              }
            }
          }
        }
        if (cnd == kNoKey || more == 0) pmask = 0;
        unsigned cm = __ballot_sync(0xffffffffu, cnd != kNoKey);
        if (!cm) break;
        if (__popc(cm) <= 4) {
          while (cm) {
            const int src2 = __ffs(cm) - 1;
            cm &= cm - 1;
            warp_list_insert(list, __shfl_sync(0xffffffffu, cnd, src2), 0xffffffffu);
          }
        } else {
          list = warp_merge_desc(list, warp_sort_desc(cnd));
        }
        const unsigned long long kth = __shfl_sync(0xffffffffu, list, K - 1);
        if (kth > thr) thr = kth;
        if (cnd != kNoKey) last = cnd;
      }
      *list_out = list;
    }
    if (hasx && lane == 0) {
      wp.hx = 1;
      wp.zx0 = load1<TT>(src, x - t0e);
    }
  } else {
    const unsigned char* src =
        use_bulk ? st + p.stage_off1 + (size_t)e0 * DT::bytes
                 : chain_row<DT>(p.draft, (size_t)sd.b * p.k + sd.i, p.V) + (size_t)t0e * DT::bytes;
    Slice<DT, NV> R;
    slice_load(src, n, use_bulk, -INFINITY, R);
    slice_stats(R, slice_max(R), p.c, &wp.G1, &wp.S1);
    if (hasx && lane == 0) {
      wp.hx = 2;
      wp.zx1 = load1<DT>(src, x - t0e);
    }
  }
}

template <class TT, class DT, int MODE, bool KD>
__global__ void __launch_bounds__(kChainThreads, 1) chain_kernel(const __grid_constant__ ChainParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint64_t* empty = full + kMaxStagesC;
  uint64_t* stall_bar = empty + kMaxStagesC;
  StageDesc* desc = reinterpret_cast<StageDesc*>(smem + p.off_desc);
  int* done = reinterpret_cast<int*>(smem + p.off_done);
  WarpPart* parts = reinterpret_cast<WarpPart*>(smem + p.off_parts);
  unsigned long long* lists = reinterpret_cast<unsigned long long*>(smem + p.off_lists);
  TaskQueue* tq = reinterpret_cast<TaskQueue*>(smem + p.off_tasks);  // consumers -> counter
  TaskQueue* cq = tq + 1;                                              // counter -> completer
  const bool use_bulk = p.use_bulk != 0;
  constexpr int DB = (MODE == kCMProbs) ? 4 : DT::bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
      done[s] = 0;
    }
    mbar_init(stall_bar, 1);
    fence_mbar_init();
    tq->tail = tq->head = tq->consumers_done = 0;
    cq->tail = cq->head = cq->consumers_done = 0;
  }
  for (int q = threadIdx.x; q < kTaskQ; q += blockDim.x) tq->ready[q] = cq->ready[q] = 0;
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // the previous grid on the stream (its outputs may be our inputs) is complete

  if (warp == kCW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const int G = (int)gridDim.x;
      const int nd = p.B * p.NT;  // draw tiles of the largest possible job list
      uint32_t it = 0;            // stages issued
      int m = 0;                  // this CTA's next draw entry: d = blockIdx.x + m * G
      bool abort = false;
      const uint64_t policy = policy_evict_first();
      auto get_stage = [&](int& s) -> bool {
        s = (int)(it % (uint32_t)S);
        const uint32_t ph = ((it / (uint32_t)S) & 1u) ^ 1u;
        if (!mbar_wait_limit(&empty[s], ph, p.wait_ns)) {
          set_status(p.status, SV_DEV_TIMEOUT);
          atomicExch(&p.glob[kGAbort], 1u);
          return false;
        }
        return true;
      };
      // Stream tiles are claimed kClaim at a time, two claims ahead, so the
      // atomic's latency overlaps the issue of the tiles before; the loads
      // that decide the next step (the request state of the next claim, this
      // CTA's draw-queue entry, the abort word) are issued one step ahead.  A
      // state read a little late only skips a little less.
      auto state_of = [&](int t) -> unsigned long long {
        if (t >= p.total) return 0ull;
        int i, b, tau;
        chain_decode(p, t, i, b, tau);
        return ld_relaxed_u64(&p.req_state[b]);
      };
      auto draw_flag = [&](int d) -> uint32_t { return d < nd ? ld_relaxed_u32(&p.drawq[d]) : 0u; };
      // Four claims are in flight: c0 (in use, its tiles' request states
      // loaded), c1 (its states loading), c2 and c3 (the atomics returning),
      // so a claim's value is first used two claims after its atomic.  The
      // draw-queue flag is read three passes after its load and the abort
      // word eight, so no pass waits on a load issued in the one before (a
      // register is only read, or copied, once its load is that old).
      int c0 = (int)atomicAdd(&p.glob[kGNext], (uint32_t)kClaim);
      int c1 = (int)atomicAdd(&p.glob[kGNext], (uint32_t)kClaim);
      int c2 = (int)atomicAdd(&p.glob[kGNext], (uint32_t)kClaim);
      int c3 = (int)atomicAdd(&p.glob[kGNext], (uint32_t)kClaim);
      int ci = 0;  // next tile of claim c0
      unsigned long long st0[kClaim], st1[kClaim];  // request state of each tile of c0, c1
#pragma unroll
      for (int q = 0; q < kClaim; ++q) st0[q] = state_of(c0 + q);
#pragma unroll
      for (int q = 0; q < kClaim; ++q) st1[q] = state_of(c1 + q);
      int dq = (int)blockIdx.x;   // the entry the flag was loaded for
      uint32_t fl = draw_flag(dq);  // its flag (in flight until fl_age reaches 3)
      uint32_t fl_age = 0;
      uint32_t pf_abort = 0u;
      uint32_t iter = 0;
      bool stream_done = false;
      uint64_t idle_t0 = 0;
      while (!abort) {
        if ((++iter & 7u) == 0u) {
          if (pf_abort) break;
          pf_abort = ld_relaxed_u32(&p.glob[kGAbort]);
        }
        // 1. this CTA's next draw tile, when its job is queued
        const int dn = (int)blockIdx.x + m * G;
        uint32_t pf_draw = 0u;
        if (++fl_age >= 3u) {
          pf_draw = dq == dn ? fl : 0u;
          fl = draw_flag(dn);
          dq = dn;
          fl_age = 0u;
        }
        if (dn < nd && pf_draw) {
          // the entry names the job's row pair; its record (read by the
          // consumers) was written before the entry
          fence_acq_rel_gpu();
          const int trow = (int)pf_draw - 1;
          const int db = trow / p.P, dnr = trow - db * p.P;
          p.drawq[dn] = 0u;
          ++m;
          // the next entry's flag: jobs come in bursts, so load it now
          dq = dn + G;
          fl = draw_flag(dq);
          fl_age = 0u;
          const int j = fast_div(dn, p.div_NT);
          const int tau = dn - j * p.NT;
          int s;
          if (!get_stage(s)) break;
          const int len = min(kTileW, p.V - tau * kTileW);
          StageDesc sd;
          sd.kind = kTKDraw;
          sd.row = j;
          sd.tile = tau;
          sd.len = len;
          sd.b = db;
          sd.i = dnr;
          sd.kb = 0;
          sd.flags = kSDDraft;
          desc[s] = sd;
          if (use_bulk) {
            const unsigned char* ts =
                chain_row<TT>(p.target, (size_t)trow, p.V) + (size_t)tau * kTileW * TT::bytes;
            const unsigned char* ds = reinterpret_cast<const unsigned char*>(p.draft) +
                                      (((size_t)db * p.k + dnr) * p.V + (size_t)tau * kTileW) * DB;
            unsigned char* st = smem + (size_t)s * p.stage_bytes;
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full[s], (uint32_t)(len * TT::bytes + len * DB));
            bulk_g2s(st, ts, (uint32_t)(len * TT::bytes), &full[s], policy);
            bulk_g2s(st + p.stage_off1, ds, (uint32_t)(len * DB), &full[s], policy);
          } else {
            mbar_arrive(&full[s]);
          }
          ++it;
          idle_t0 = 0;
          continue;
        }
        // 2. the next stream tile
        if (!stream_done) {
          if (c0 >= p.total) {
            stream_done = true;
            continue;
          }
          const int t = c0 + ci;
          unsigned long long stw = st0[0];
#pragma unroll
          for (int q = 1; q < kClaim; ++q)
            if (ci == q) stw = st0[q];
          if (++ci == kClaim || t + 1 >= p.total) {  // the claim is used up: move to the next
            c0 = c1;
            c1 = c2;
            c2 = c3;
            ci = 0;
            c3 = (int)atomicAdd(&p.glob[kGNext], (uint32_t)kClaim);
#pragma unroll
            for (int q = 0; q < kClaim; ++q) {
              st0[q] = st1[q];
              st1[q] = state_of(c1 + q);
            }
          }
          int i, b, tau;
          chain_decode(p, t, i, b, tau);
          const int kb = chain_kb(p, b);
          // a row that is not needed: with the tiles of a row consecutive,
          // move the claim counter past it (never past a row's first tile)
          auto skip_row = [&]() {
            if (p.order == 0 && tau + 1 < p.NT)
              atomicMax(&p.glob[kGNext], (uint32_t)(t - tau + p.NT));
          };
          if (kb < 0) {
            // an idle request, or an invalid draft count: finished by the
            // manager warp (once, at its first tile)
            if (!(i == 0 && tau == 0)) skip_row();
            if (i == 0 && tau == 0) {
              int s;
              if (!get_stage(s)) break;
              StageDesc sd = {};
              sd.kind = kTKIdle;
              sd.row = b;
              sd.b = b;
              sd.kb = kb;
              desc[s] = sd;
              mbar_arrive(&full[s]);
              ++it;
            }
            continue;
          }
          if (i > kb) {  // a row the request does not use
            skip_row();
            continue;
          }
          const uint32_t rej = (uint32_t)(stw >> 32) & 0x7fffffffu;
          if (rej && (__ffs(rej) - 1) < i) {  // an earlier position rejected
            skip_row();
            continue;
          }
          int s;
          if (!get_stage(s)) break;
          const int len = min(kTileW, p.V - tau * kTileW);
          const bool dr = (MODE == kCMSample) && i < kb;
          StageDesc sd;
          sd.kind = kTKStream;
          sd.row = b * p.P + i;
          sd.tile = tau;
          sd.len = len;
          sd.b = b;
          sd.i = i;
          sd.kb = kb;
          sd.flags = (dr ? kSDDraft : 0) | (i == kb ? kSDBonus : 0);
          desc[s] = sd;
          if (use_bulk) {
            const unsigned char* ts =
                chain_row<TT>(p.target, (size_t)b * p.P + i, p.V) + (size_t)tau * kTileW * TT::bytes;
            unsigned char* st = smem + (size_t)s * p.stage_bytes;
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&full[s], (uint32_t)(len * TT::bytes + (dr ? len * DT::bytes : 0)));
            bulk_g2s_plain(st, ts, (uint32_t)(len * TT::bytes), &full[s]);
            if (dr) {
              const unsigned char* ds =
                  chain_row<DT>(p.draft, (size_t)b * p.k + i, p.V) + (size_t)tau * kTileW * DT::bytes;
              bulk_g2s_plain(st + p.stage_off1, ds, (uint32_t)(len * DT::bytes), &full[s]);
            }
          } else {
            mbar_arrive(&full[s]);
          }
          ++it;
          idle_t0 = 0;
          continue;
        }
        // 3. nothing to issue: finished once every request's outcome is
        //    known and this CTA's queue holds no further job tile
        if (ld_acquire_u32(&p.glob[kGDet]) == (uint32_t)p.B) {
          const uint32_t jt = ld_acquire_u32(&p.glob[kGJobTail]);
          if (dn >= (int)(jt * (uint32_t)p.NT)) break;
        }
        const uint64_t now = globaltimer_ns();
        if (idle_t0 == 0) idle_t0 = now;
        else if (now - idle_t0 > p.wait_ns) {
          set_status(p.status, SV_DEV_TIMEOUT);
          atomicExch(&p.glob[kGAbort], 1u);
          abort = true;
          break;
        }
        __nanosleep(64);
        // idle: the flag loaded now is read at the next pass
        fl = draw_flag(dn);
        dq = dn;
        fl_age = 2u;
        pf_abort = ld_relaxed_u32(&p.glob[kGAbort]);
        if (pf_abort) break;
      }
      // the consumers stop at an exit stage
      int s;
      if (*reinterpret_cast<volatile uint32_t*>(&p.glob[kGAbort])) {
        // after a timeout a copy may still be landing: wait (bounded) for the
        // last phase of every stage issued, so no copy outlives the CTA
        for (uint32_t q = 0; q < (uint32_t)S && q < it; ++q) {
          const uint32_t uses = (it - 1u - q) / (uint32_t)S + 1u;  // times stage q was armed
          mbar_wait_limit(&full[q], (uses - 1u) & 1u, p.wait_ns);
        }
      }
      if (get_stage(s)) {
        StageDesc sd = {};
        sd.kind = kTKExit;
        desc[s] = sd;
        mbar_arrive(&full[s]);
        ++it;
      } else {
        // the ring did not drain in time: consumers give up on their own
        for (int q = 0; q < S; ++q) {
          StageDesc sd = {};
          sd.kind = kTKExit;
          desc[q] = sd;
        }
        __threadfence_block();
        for (int q = 0; q < S; ++q) mbar_arrive(&full[q]);
      }
    }
  } else if (warp == kCW + 1) {
    // ---------------- counter: tiles into rows, draw tiles into jobs ----------------
    // Up to 32 count tasks at a time, one release atomic per lane, all in
    // flight together; the counts that complete a row or a job become
    // completion tasks for the completer warp.
    int head = 0;
    uint64_t idle_t0 = 0;
    while (true) {
      int n = 0;
      if (lane == 0) {
        while (n < 32 && *reinterpret_cast<volatile int*>(&tq->ready[(head + n) % kTaskQ])) ++n;
        if (n == 0 && *reinterpret_cast<volatile int*>(&tq->consumers_done) == kCW &&
            *reinterpret_cast<volatile int*>(&tq->tail) == head)
          n = -1;
      }
      n = __shfl_sync(0xffffffffu, n, 0);
      if (n < 0) break;
      if (n == 0) {
        // idle; the consumers always finish (their waits are bounded), the
        // limit here is a last resort
        const uint64_t now = globaltimer_ns();
        if (idle_t0 == 0) idle_t0 = now;
        else if (now - idle_t0 > 8ull * p.wait_ns) break;
        __nanosleep(32);
        continue;
      }
      idle_t0 = 0;
      __threadfence_block();  // the tasks and the records they name (acquire, CTA scope)
      int4 t = make_int4(-1, 0, 0, 0);
      if (lane < n) {
        const int slot = (head + lane) % kTaskQ;
        t = tq->task[slot];
        tq->ready[slot] = 0;
      }
      __threadfence_block();
      __syncwarp();
      head += n;
      if (lane == 0) *reinterpret_cast<volatile int*>(&tq->head) = head;
      int fire = 0;
      if (t.x == kTaskTile) {
        fire = atom_add_release(&p.pair_cnt[t.y * p.P + t.z], 1u) == (uint32_t)p.NT - 1u;
      } else if (t.x == kTaskDraw) {
        fire = atom_add_release(&p.job_cnt[t.y], 1u) == (uint32_t)p.NT - 1u;
      } else if (t.x == kTaskIdle) {
        fire = 1;
      }
      unsigned todo = __ballot_sync(0xffffffffu, fire != 0);
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        if (lane == src) queue_push(cq, t, p);
      }
      __syncwarp();
    }
    if (lane == 0) {
      __threadfence_block();
      *reinterpret_cast<volatile int*>(&cq->consumers_done) = 1;
    }
  } else if (warp == kCW + 2) {
    // ---------------- completer: row completions, draws, idle requests ----------------
    int head = 0;
    uint64_t idle_t0 = 0;
    while (true) {
      int go = 0;
      int4 t = make_int4(0, 0, 0, 0);
      if (lane == 0) {
        const int slot = head % kTaskQ;
        if (*reinterpret_cast<volatile int*>(&cq->ready[slot])) {
          __threadfence_block();
          t = cq->task[slot];
          cq->ready[slot] = 0;
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&cq->head) = head + 1;
          go = 1;
        } else if (*reinterpret_cast<volatile int*>(&cq->consumers_done) != 0 &&
                   *reinterpret_cast<volatile int*>(&cq->tail) == head) {
          go = 2;
        }
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (go == 2) break;
      if (go == 0) {
        const uint64_t now = globaltimer_ns();
        if (idle_t0 == 0) idle_t0 = now;
        else if (now - idle_t0 > 8ull * p.wait_ns) break;
        __nanosleep(32);
        continue;
      }
      idle_t0 = 0;
      ++head;
      t.x = __shfl_sync(0xffffffffu, t.x, 0);
      t.y = __shfl_sync(0xffffffffu, t.y, 0);
      t.z = __shfl_sync(0xffffffffu, t.z, 0);
      t.w = __shfl_sync(0xffffffffu, t.w, 0);
      if (t.x == kTaskTile) {
        // the row's count is complete: acquire it (synchronising with every
        // tile's release), then complete the row
        const int r = t.y * p.P + t.z;
        if (lane == 0) (void)ld_acquire_u32(&p.pair_cnt[r]);
        __syncwarp();
        chain_complete_row<TT, DT, MODE, KD>(p, t.y, t.z, t.w);
      } else if (t.x == kTaskDraw) {
        if (lane == 0) (void)ld_acquire_u32(&p.job_cnt[t.y]);
        __syncwarp();
        chain_locate<TT, DT, MODE, KD>(p, t.y);
      } else {  // an idle request, or one with an invalid draft count
        if (t.w == -2 && lane == 0) set_status(p.status, SV_DEV_BAD_LEN);
        chain_write_outputs<KD>(p, t.y, t.w, -1, -1, 0);
        __syncwarp();
        if (lane == 0) red_add_release_u32(&p.glob[kGDet], 1u);
      }
    }
  } else {
    // ---------------- consumers ----------------
    // The warp that folds a tile hands its count to the counter warp.
    auto push_task = [&](int kind, int a, int b2, int c2) {
      if (lane == 0) queue_push(tq, make_int4(kind, a, b2, c2), p);
      __syncwarp();
    };
    bool stalled = false;
    int misses = 0;
    for (uint32_t it = 0;; ++it) {
      const int s = (int)(it % (uint32_t)S);
      const uint32_t ph = (it / (uint32_t)S) & 1u;
      const bool ok = mbar_wait_limit(&full[s], ph, p.wait_ns);
      const StageDesc sd = desc[s];
      if (sd.kind == kTKExit) break;
      if (!ok) {
        if (lane == 0) {
          set_status(p.status, SV_DEV_TIMEOUT);
          atomicExch(&p.glob[kGAbort], 1u);
        }
        // a producer that supplies nothing twice in a row is gone
        if (++misses >= 2) break;
      } else {
        misses = 0;
      }
      unsigned char* st = smem + (size_t)s * p.stage_bytes;
      WarpPart wp;
      wp.G0 = wp.G1 = -INFINITY;
      wp.S0 = wp.S1 = 0.0;
      wp.zx0 = wp.zx1 = 0.f;
      wp.hx = 0;
      wp.tmo = ok ? 0 : 1;
      wp.key = kNoKey;
      unsigned long long list = kNoKey;
      if (sd.kind == kTKStream) {
        if (p.stall && !stalled && warp == 0 && sd.row == 0 && sd.tile == 0) {
          // test hook: wait on a barrier nothing arrives on, as a copy that
          // never lands would; the bounded wait gives up (after a quarter of
          // the limit, so no other wait runs out meanwhile) and reports it
          stalled = true;
          if (!mbar_wait_limit(stall_bar, 0, p.wait_ns / 4)) wp.tmo = 1;
        }
        if (sd.flags & kSDDraft)
          chain_slice<TT, DT, MODE, KD, kVPLP>(p, sd, st, use_bulk, warp, wp, &list);
        else
          chain_slice<TT, DT, MODE, KD, kVPL>(p, sd, st, use_bulk, warp, wp, &list);
        if (KD && lane < p.K) lists[((size_t)s * kCW + warp) * p.K + lane] = list;
      } else if (sd.kind == kTKDraw) {
        // residual mass of the slice: p and q of the row pair sd.i
        const DrawJob dj = ldcg_rec(&p.jobs[sd.row]);
        const int e0 = warp * kSliceW;
        const int n = max(0, min(kSliceW, sd.len - e0));
        const int t0e = sd.tile * kTileW + e0;
        const unsigned char* ts =
            use_bulk ? st + (size_t)e0 * TT::bytes
                     : chain_row<TT>(p.target, (size_t)dj.b * p.P + dj.n, p.V) + (size_t)t0e * TT::bytes;
        const unsigned char* ds =
            use_bulk ? st + p.stage_off1 + (size_t)e0 * DB
                     : reinterpret_cast<const unsigned char*>(p.draft) +
                           (((size_t)dj.b * p.k + dj.n) * p.V + (size_t)t0e) * DB;
        double a = 0.0;
#pragma unroll
        for (int v = 0; v < kVPL; ++v) {
          float w8[8];
          resid8<TT, DT, MODE>(ts, ds, (v * 32 + lane) * kVec, n, use_bulk, p.c, dj.Gt,
                               dj.invSt, dj.Gd, dj.invSd, w8);
          a += (double)seq8(w8);
        }
        wp.S0 = warp_sum(a);
      }
      if (lane == 0) parts[s * kCW + warp] = wp;
      __syncwarp();
      // the last warp of the stage folds the partials and returns the stage
      int last = 0;
      if (lane == 0) {
        __threadfence_block();
        last = atomicAdd(&done[s], 1) == kCW - 1;
        if (last) {
          done[s] = 0;
          __threadfence_block();
        } else {
          mbar_arrive(&empty[s]);
        }
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (!last) continue;
      if (sd.kind == kTKStream) {
        const bool pair = (sd.flags & kSDDraft) != 0;
        const WarpPart q = lane < kCW ? parts[s * kCW + lane]
                                      : WarpPart{-INFINITY, -INFINITY, 0.0, 0.0, 0.f, 0.f, 0, 0, kNoKey};
        // target partials from the target warps, draft partials from the draft warps
        const bool tl_ = lane < (pair ? kRowW : kCW);
        const float g0 = tl_ ? q.G0 : -INFINITY, g1 = tl_ ? -INFINITY : q.G1;
        const double s0 = tl_ ? q.S0 : 0.0, s1 = tl_ ? 0.0 : q.S1;
        TileRec tr;
        tr.G0 = warp_max(g0);
        tr.G1 = warp_max(g1);
        tr.S0 = warp_sum(rescale_pow2(s0, g0, tr.G0));
        tr.S1 = warp_sum(rescale_pow2(s1, g1, tr.G1));
        const unsigned h0 = __ballot_sync(0xffffffffu, q.hx == 1);
        const unsigned h1 = __ballot_sync(0xffffffffu, q.hx == 2);
        tr.zx0 = h0 ? __shfl_sync(0xffffffffu, q.zx0, __ffs(h0) - 1) : 0.f;
        tr.zx1 = h1 ? __shfl_sync(0xffffffffu, q.zx1, __ffs(h1) - 1) : 0.f;
        int fl = __any_sync(0xffffffffu, q.tmo != 0) ? kPTimeout : 0;
        if (h0) fl |= kPHasX;
        tr.flags = fl;
        tr.pad = 0;
        tr.key = warp_max_u64(q.key);
        unsigned long long tl = kNoKey;
        if (KD) {
          const int K = p.K;
          const int nw = pair ? kRowW : kCW;
          for (int w = 0; w < nw; ++w)
            tl = warp_merge_desc(tl, lane < K ? lists[((size_t)s * kCW + w) * K + lane] : kNoKey);
        }
        const bool bonus = (MODE != kCMGreedy) && (sd.flags & kSDBonus);
        if (lane == 0) mbar_arrive(&empty[s]);  // partials and lists read
        const size_t ti = (size_t)sd.row * p.NT + sd.tile;
        if (lane == 0) p.tiles[ti] = tr;
        if (bonus && lane < kCW) {
          WarpStat ws;
          ws.G = q.G0;
          ws.pad = 0.f;
          ws.S = q.S0;
          p.bonus[((size_t)sd.b * p.NT + sd.tile) * kCW + lane] = ws;
        }
        if (KD) {
          const int K = p.K;
          if (lane < K) p.cand[ti * K + lane] = tl;
          const unsigned long long kth = __shfl_sync(0xffffffffu, tl, K - 1);
          if (lane == 0 && kth != kNoKey) atomicMax(&p.rowthr[sd.row], kth);
        }
        __threadfence_block();
        __syncwarp();
        push_task(kTaskTile, sd.b, sd.i, sd.kb);
      } else if (sd.kind == kTKDraw) {
        const double q = lane < kCW ? parts[s * kCW + lane].S0 : 0.0;
        if (lane == 0) mbar_arrive(&empty[s]);
        DrawRec* dr = &p.draws[(size_t)sd.row * p.NT + sd.tile];
        double tot = 0.0;
#pragma unroll
        for (int w = 0; w < kCW; ++w) tot += __shfl_sync(0xffffffffu, q, w);
        if (lane < kCW) dr->wm[lane] = q;
        if (lane == 0) dr->mass = tot;
        __threadfence_block();
        __syncwarp();
        push_task(kTaskDraw, sd.row, 0, 0);
      } else {  // kTKIdle
        if (lane == 0) mbar_arrive(&empty[s]);
        push_task(kTaskIdle, sd.b, 0, sd.kb);
      }
    }
    if (lane == 0) {
      __threadfence_block();
      atomicAdd(&tq->consumers_done, 1);
    }
  }

  // The last CTA out returns the call's counters and request state to zero
  // (and, after a timeout, writes the outputs of requests left unfinished).
  __syncthreads();
  __shared__ int last_cta;
  if (threadIdx.x == 0) {
    fence_acq_rel_gpu();
    last_cta = atomicAdd(&p.glob[kGExit], 1u) == gridDim.x - 1u;
    if (last_cta) fence_acq_rel_gpu();
  }
  __syncthreads();
  if (!last_cta) return;
  const bool aborted = __ldcg(&p.glob[kGAbort]) != 0u;
  if (aborted) {
    // outputs of the requests left unfinished, then the whole workspace
    if (warp < kCW)
      for (int b = warp; b < p.B; b += kCW) {
        const unsigned long long stw = __ldcg(&p.req_state[b]);
        if (!(stw & kFinalBit)) chain_write_outputs<false>(p, b, 0, -1, -1, 0);
      }
    if (KD && threadIdx.x == 0) *p.total_out = NAN;
    __syncthreads();
    uint4* w4 = reinterpret_cast<uint4*>(p.ws_base);
    for (size_t q = threadIdx.x; q < p.ws_bytes / 16; q += blockDim.x) w4[q] = make_uint4(0, 0, 0, 0);
    return;
  }
  // rows streamed in part and then skipped (their count stopped short)
  if (warp < kCW) {
    for (int r = warp; r < p.B * p.P; r += kCW) {
      const uint32_t c = __shfl_sync(0xffffffffu, lane == 0 ? __ldcg(&p.pair_cnt[r]) : 0u, 0);
      if (c == 0u) continue;
      zero_tiles(p, r);
      zero_lists<KD>(p, r);
      if (MODE != kCMGreedy) {
        const int b = r / p.P, i = r - b * p.P;
        if (i == chain_kb(p, b)) zero_bonus(p, b);
      }
      if (lane == 0) p.pair_cnt[r] = 0u;
    }
  }
  for (int q = threadIdx.x; q < p.B; q += blockDim.x) p.req_state[q] = 0ull;
  __syncthreads();
  if (threadIdx.x == 0) {
    p.glob[kGNext] = 0u;
    p.glob[kGJobTail] = 0u;
    p.glob[kGDet] = 0u;
    p.glob[kGKd] = 0u;
    p.glob[kGAbort] = 0u;
    p.glob[kGExit] = 0u;
  }
}

}  // namespace sv
