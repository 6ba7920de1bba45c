// sv_device.cuh -- device building blocks shared by the libsv kernels (sm_100a).
//
// Row plan: a vocabulary row (or a target/draft row pair) is split into C
// contiguous chunks of L elements, one CTA of a C-CTA thread-block cluster per
// chunk.  Each CTA stages its chunk into shared memory with bulk asynchronous
// copies (cp.async.bulk, no multicast), in pieces of kRound elements that
// complete on their own mbarrier, so that compute on piece p overlaps the
// landing of pieces p+1...  The chunk stays resident for the whole kernel:
// second passes (residual CDF, top-K candidates, KL gathers) read shared
// memory, never HBM.  Partial results are combined across the cluster through
// distributed shared memory in a fixed order, so every result is
// deterministic.
//
// Thread mapping inside a chunk: piece p covers elements [p*kRound, (p+1)*kRound);
// thread t owns the 8 consecutive elements p*kRound + 8t ... + 7 of every
// piece.  The inverse-CDF search relies on this mapping being the same in the
// pass that sums the weights and in the pass that locates the draw.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sv.h"

namespace sv {
namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kVec = 8;                     // elements per thread per piece
constexpr int kRound = kThreads * kVec;     // elements per piece
constexpr int kMaxPieces = 16;              // chunk length <= 32768 elements
constexpr int kMaxChunk = kRound * kMaxPieces;
constexpr int kMaxCluster = 16;
constexpr int kMaxK = 32;
constexpr int kCandCap = 1024;              // top-K candidate buffer per CTA
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per bounded wait
constexpr uint32_t kWaitHintNs = 1000000u;                  // sleep up to 1 ms per try

enum DraftKind { kDraftLogits = 0, kDraftProbs = 1 };

// ---------------------------------------------------------------------------
// Storage types.
// ---------------------------------------------------------------------------
struct F32 {
  using storage = float;
  static constexpr int bytes = 4;
};
// Division by a runtime divisor 1 <= d < 2^31 for dividends 0 <= n < 2^31:
// floor(n / d) = (n * m) >> (32 + s) with 2^s >= d and m = ceil(2^(32+s) / d)
// (m < 2^33, so the product fits 64 bits; the rounding excess of m adds less
// than n / 2^(32+s) < 1/(2d), which never crosses the next multiple of 1/d).
struct FastDiv {
  unsigned long long m;
  int s;
};
inline FastDiv make_fastdiv(int d) {
  int s = 0;
  while ((1LL << s) < d) ++s;
  const unsigned __int128 num = (unsigned __int128)1 << (32 + s);
  FastDiv f;
  f.m = (unsigned long long)((num + (unsigned)d - 1) / (unsigned)d);
  f.s = s;
  return f;
}
__device__ __forceinline__ int fast_div(int n, const FastDiv& f) {
  return (int)(((unsigned long long)(unsigned)n * f.m) >> (32 + f.s));
}

struct BF16 {
  using storage = uint16_t;
  static constexpr int bytes = 2;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Eight consecutive elements starting at element e (e % 8 == 0) of a chunk
// buffer in shared memory, widened to fp32.
template <class T>
__device__ __forceinline__ void load8(const unsigned char* buf, int e, float v[8]);

template <>
__device__ __forceinline__ void load8<BF16>(const unsigned char* buf, int e, float v[8]) {
  uint4 w = *reinterpret_cast<const uint4*>(buf + (size_t)e * 2);
  v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
  v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

template <>
__device__ __forceinline__ void load8<F32>(const unsigned char* buf, int e, float v[8]) {
  float4 a = *reinterpret_cast<const float4*>(buf + (size_t)e * 4);
  float4 b = *reinterpret_cast<const float4*>(buf + (size_t)e * 4 + 16);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Eight elements plus their maximum.  For bf16 the maximum is taken on the
// packed pairs (3 packed max + 1 scalar max instead of 7 scalar max).
template <class T>
__device__ __forceinline__ float load8_max(const unsigned char* buf, int e, float v[8]);

template <>
__device__ __forceinline__ float load8_max<BF16>(const unsigned char* buf, int e, float v[8]) {
  uint4 w = *reinterpret_cast<const uint4*>(buf + (size_t)e * 2);
  __nv_bfloat162 a = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.x),
                             *reinterpret_cast<__nv_bfloat162*>(&w.y));
  __nv_bfloat162 c = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.z),
                             *reinterpret_cast<__nv_bfloat162*>(&w.w));
  a = __hmax2(a, c);
  uint32_t m = *reinterpret_cast<uint32_t*>(&a);
  v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
  v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
  return fmaxf(bf16_lo(m), bf16_hi(m));
}

template <>
__device__ __forceinline__ float load8_max<F32>(const unsigned char* buf, int e, float v[8]) {
  load8<F32>(buf, e, v);
  return fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])),
               fmaxf(fmaxf(v[4], v[5]), fmaxf(v[6], v[7])));
}

// Maximum of eight elements without widening them all.
template <class T>
__device__ __forceinline__ float max8(const unsigned char* buf, int e);

template <>
__device__ __forceinline__ float max8<BF16>(const unsigned char* buf, int e) {
  uint4 w = *reinterpret_cast<const uint4*>(buf + (size_t)e * 2);
  __nv_bfloat162 a = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.x),
                             *reinterpret_cast<__nv_bfloat162*>(&w.y));
  __nv_bfloat162 c = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.z),
                             *reinterpret_cast<__nv_bfloat162*>(&w.w));
  a = __hmax2(a, c);
  const uint32_t m = *reinterpret_cast<uint32_t*>(&a);
  return fmaxf(bf16_lo(m), bf16_hi(m));
}

template <>
__device__ __forceinline__ float max8<F32>(const unsigned char* buf, int e) {
  const float4 a = *reinterpret_cast<const float4*>(buf + (size_t)e * 4);
  const float4 b = *reinterpret_cast<const float4*>(buf + (size_t)e * 4 + 16);
  return fmaxf(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), fmaxf(fmaxf(b.x, b.y), fmaxf(b.z, b.w)));
}

// Value of the element that fills the padding of a partial last vector:
// -inf for logits (no mass, never a maximum), 0 for probabilities.
template <class T>
__device__ __forceinline__ void store_pad(unsigned char* buf, int e, bool probs);
template <>
__device__ __forceinline__ void store_pad<BF16>(unsigned char* buf, int e, bool probs) {
  reinterpret_cast<uint16_t*>(buf)[e] = probs ? 0 : 0xff80u;
}
template <>
__device__ __forceinline__ void store_pad<F32>(unsigned char* buf, int e, bool probs) {
  reinterpret_cast<float*>(buf)[e] = probs ? 0.0f : __int_as_float(0xff800000);
}

template <class T>
__device__ __forceinline__ float load1(const unsigned char* buf, int e);
template <>
__device__ __forceinline__ float load1<BF16>(const unsigned char* buf, int e) {
  return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(buf)[e] << 16);
}
template <>
__device__ __forceinline__ float load1<F32>(const unsigned char* buf, int e) {
  return reinterpret_cast<const float*>(buf)[e];
}

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier, bulk copy, timers, fast exp2.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Global -> shared bulk copy completing on an mbarrier of this CTA.  Both
// addresses 16-byte aligned, bytes a multiple of 16.  L2 policy evict-first:
// the data is consumed from shared memory and never re-read through L2.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Same, default L2 policy (data that a later pass may read again).
__device__ __forceinline__ void bulk_g2s_plain(void* dst, const void* src, uint32_t bytes,
                                               uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bring [src, src + bytes) into L2 without a destination (src 16-byte
// aligned, bytes a multiple of 16); the copy completes on its own.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// try_wait with a suspend-time hint: the waiting warp sleeps in hardware until
// the phase completes (or the hint expires) instead of spinning.
__device__ __forceinline__ uint32_t mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
      : "memory");
  return ok;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of an mbarrier, giving up after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Packed pairs of fp32 in one 64-bit register (sm_100 f32x2 arithmetic: one
// instruction for two lanes of a pair).
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2_unpack(unsigned long long d, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Programmatic dependent launch: a kernel lets the next kernel on its stream
// be scheduled early; the next kernel waits here until this grid has
// completed and its memory operations are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Split cluster barrier (every thread of the cluster arrives, then waits).
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

// 2^x in float64 to a few units in the last place: x = k + f with k the
// nearest integer and |f| <= 1/2, 2^f = e^y with y = f ln 2 (|y| < 0.347)
// summed as its Taylor series through y^12 (truncation below 1e-16
// relative), then scaled by 2^k.  Results below 2^-1022 flush to 0 (every
// caller's terms are relative to a maximum of order 1).
__device__ __forceinline__ double exp2_f64(double x) {
  if (!(x > -1022.0)) return 0.0;  // also -inf and NaN-free underflow
  const double k = rint(x);
  const double y = (x - k) * 0.693147180559945309417232121458;
  double s = 1.0 / 479001600.0;             // 1/12!
  s = fma(s, y, 1.0 / 39916800.0);          // 1/11!
  s = fma(s, y, 1.0 / 3628800.0);           // 1/10!
  s = fma(s, y, 1.0 / 362880.0);            // 1/9!
  s = fma(s, y, 1.0 / 40320.0);             // 1/8!
  s = fma(s, y, 1.0 / 5040.0);              // 1/7!
  s = fma(s, y, 1.0 / 720.0);               // 1/6!
  s = fma(s, y, 1.0 / 120.0);               // 1/5!
  s = fma(s, y, 1.0 / 24.0);                // 1/4!
  s = fma(s, y, 1.0 / 6.0);                 // 1/3!
  s = fma(s, y, 0.5);                       // 1/2!
  s = fma(s, y, 1.0);                       // 1/1!
  s = fma(s, y, 1.0);                       // 1/0!
  return s * __longlong_as_double((long long)((int)k + 1023) << 52);
}

// 2^x in float64 with a shorter chain: x = k/16 + f with k = rint(16 x) and
// |f| <= 1/32, so 2^x = 2^(k div 16) * t16[k mod 16] * e^(f ln 2), where
// t16[j] = 2^(j/16) (filled by the caller, e.g. with exp2_f64) and e^y for
// |y| <= ln(2)/32 is its Taylor series through y^6 (truncation below 5e-16
// relative).  Results below 2^-1022 flush to 0.
__device__ __forceinline__ double exp2_f64_tab(double x, const double* t16) {
  if (!(x > -1022.0)) return 0.0;
  const double k16 = rint(x * 16.0);
  const double y = fma(-k16, 0.0625, x) * 0.693147180559945309417232121458;
  double s = 1.0 / 720.0;                   // 1/6!
  s = fma(s, y, 1.0 / 120.0);               // 1/5!
  s = fma(s, y, 1.0 / 24.0);                // 1/4!
  s = fma(s, y, 1.0 / 6.0);                 // 1/3!
  s = fma(s, y, 0.5);                       // 1/2!
  s = fma(s, y, 1.0);                       // 1/1!
  s = fma(s, y, 1.0);                       // 1/0!
  const long long ki = (long long)k16;
  const int j = (int)(ki & 15);
  const int n = (int)((ki - j) >> 4);       // floor(k / 16)
  return s * t16[j] * __longlong_as_double((long long)(n + 1023) << 52);
}

// 2^x on the special-function unit (ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void set_status(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------------------
// Deterministic block reductions (xor butterflies give every lane the same
// bits; warp partials are combined by warp 0 in a fixed tree).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide max (result broadcast).  `red` holds kWarps floats.
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) r = fmaxf(r, red[i]);
  return r;
}

// Block-wide sum in float64 (result broadcast).  `red` holds kWarps doubles.
__device__ __forceinline__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double r = red[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) r += red[i];
  return r;
}

// Block-wide inclusive scan in float64; returns this thread's inclusive value
// and writes the block total to *total.  `red` holds kWarps doubles.
__device__ __forceinline__ double block_scan_incl(double v, double* red, double* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  __syncthreads();
  if (lane == 31) red[w] = v;
  __syncthreads();
  double off = 0.0, tot = 0.0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    if (i < w) off += red[i];
    tot += red[i];
  }
  *total = tot;
  return off + v;
}

// ---------------------------------------------------------------------------
// Chunk staging.
// ---------------------------------------------------------------------------
struct ChunkGeom {
  int j0;        // first vocabulary index of this CTA's chunk
  int len;       // elements in the chunk (0..L)
  int npieces;   // pieces holding at least one element
  int nvec;      // 8-element vectors covering len (last may be partial)
};

__device__ __forceinline__ ChunkGeom chunk_geom(int rank, int L, int V) {
  ChunkGeom g;
  g.j0 = rank * L;
  g.len = max(0, min(L, V - g.j0));
  g.nvec = (g.len + kVec - 1) / kVec;
  g.npieces = (g.len + kRound - 1) / kRound;
  return g;
}

// Issue the bulk copies of one row's chunk (thread 0 only).  Piece p of the
// 16-byte-aligned prefix completes on bars[p]; the caller has armed bars[p]
// with the expected byte count of all rows sharing that barrier.
template <class T>
__device__ __forceinline__ uint32_t piece_bytes(const ChunkGeom& g, int p) {
  const int al = (g.len * T::bytes) & ~15;      // aligned prefix bytes
  const int b0 = p * kRound * T::bytes;
  return (uint32_t)max(0, min(kRound * T::bytes, al - b0));
}

template <class T>
__device__ __forceinline__ void issue_row_copies(unsigned char* buf, const void* row_base,
                                                 const ChunkGeom& g, uint64_t* bars,
                                                 uint64_t policy) {
  const unsigned char* src =
      reinterpret_cast<const unsigned char*>(row_base) + (size_t)g.j0 * T::bytes;
  for (int p = 0; p < g.npieces; ++p) {
    uint32_t nb = piece_bytes<T>(g, p);
    if (nb) bulk_g2s(buf + (size_t)p * kRound * T::bytes, src + (size_t)p * kRound * T::bytes, nb,
                     &bars[p], policy);
  }
}

// Elements the bulk copies do not cover: the unaligned tail (bulk path) or the
// whole chunk (scalar path), plus padding to a multiple of 8 elements.
template <class T>
__device__ __forceinline__ void scalar_fill(unsigned char* buf, const void* row_base,
                                            const ChunkGeom& g, bool use_bulk, bool probs) {
  const typename T::storage* src =
      reinterpret_cast<const typename T::storage*>(row_base) + g.j0;
  typename T::storage* dst = reinterpret_cast<typename T::storage*>(buf);
  const int start = use_bulk ? ((g.len * T::bytes) & ~15) / T::bytes : 0;
  for (int e = start + (int)threadIdx.x; e < g.len; e += kThreads) dst[e] = src[e];
  for (int e = g.len + (int)threadIdx.x; e < g.nvec * kVec; e += kThreads)
    store_pad<T>(buf, e, probs);
}

// ---------------------------------------------------------------------------
// Online softmax statistics.  With c = log2(e) / T, a thread keeps its largest
// raw logit mz, an integer-valued exponent reference ref >= c * mz (the
// ceiling of c times its running maximum), and S = sum 2^(fl(z*c - ref)) in
// float64 from 8-term fp32 partials.  Because ref is an integer, moving it
// rescales S by an exact power of two, and the largest terms have exponents in
// (-1, 0], where the fp32 argument is most precise.  CTA and cluster combines
// rescale the same way, so no transcendental runs outside the per-element exp2.
// ---------------------------------------------------------------------------
struct ThreadStat {
  float mz;
  float ref;
  double S;
};

__device__ __forceinline__ void stat_init(ThreadStat& s) {
  s.mz = -INFINITY;
  s.ref = -INFINITY;
  s.S = 0.0;
}

// 2^e as a binary64 for integer e in [-1022, 1023], built from the exponent field.
__device__ __forceinline__ double pow2i(int e) {
  return __longlong_as_double((long long)(e + 1023) << 52);
}

// S * 2^(from - to) for integer-valued from <= to: exact for normal results,
// in two steps below 2^-1022, 0 below 2^-2000.
__device__ __forceinline__ double rescale_pow2(double S, float from, float to) {
  if (S == 0.0) return 0.0;
  const float d = from - to;
  if (d < -2000.f) return 0.0;
  int e = (int)d;
  if (e > 1023) e = 1023;
  if (e < -1022) {
    S *= pow2i(-1022);
    e += 1022;
  }
  return S * pow2i(e);
}

__device__ __forceinline__ void stat_update(ThreadStat& s, const float v[8], float vmax, float c) {
  s.mz = fmaxf(s.mz, vmax);
  const float top = vmax * c;
  if (top > s.ref) {
    const float nref = ceilf(top);
    s.S = rescale_pow2(s.S, s.ref, nref);
    s.ref = nref;
  }
  if (vmax != -INFINITY) {
    float e[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) e[t] = ex2(fmaf(v[t], c, -s.ref));
    s.S += (double)(((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7])));
  }
}

// Move a thread's reference to cover a new maximum pm (before its terms).
__device__ __forceinline__ void stat_cover(ThreadStat& s, float pm, float c) {
  s.mz = fmaxf(s.mz, pm);
  const float top = pm * c;
  if (top > s.ref) {
    const float nref = ceilf(top);
    s.S = rescale_pow2(s.S, s.ref, nref);
    s.ref = nref;
  }
}

// Sum of the exp2 terms of NV vectors of 8 (relative to the current
// reference), by a fixed fp32 tree.
template <int NV>
__device__ __forceinline__ float stat_terms(const ThreadStat& s, const float (&x)[NV][8],
                                            float c) {
  float e[NV * 8];
#pragma unroll
  for (int v = 0; v < NV; ++v)
#pragma unroll
    for (int t = 0; t < 8; ++t) e[v * 8 + t] = ex2(fmaf(x[v][t], c, -s.ref));
#pragma unroll
  for (int w = NV * 8 / 2; w >= 1; w >>= 1)
#pragma unroll
    for (int t = 0; t < w; ++t) e[t] = e[t] + e[t + w];
  return e[0];
}

// CTA partial: exponent reference G (max over threads of ref) and
// S = sum over the chunk of 2^(z*c - G).  Collective over the block.
struct CtaStat {
  float G;
  float mz;
  double S;
};

__device__ __forceinline__ CtaStat stat_block(const ThreadStat& s, float* redf, double* redd) {
  CtaStat r;
  r.G = block_max(s.ref, redf);
  r.mz = block_max(s.mz, redf);
  r.S = block_sum(rescale_pow2(s.S, s.ref, r.G), redd);
  return r;
}

// Two rows at once (target and draft of a pair): one set of barriers.
__device__ __forceinline__ void stat_block2(const ThreadStat& a, const ThreadStat& b,
                                            float2* redf2, double2* redd2, CtaStat* ra,
                                            CtaStat* rb) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float ga = warp_max(a.ref), gb = warp_max(b.ref), ma = warp_max(a.mz), mb = warp_max(b.mz);
  __syncthreads();
  if (lane == 0) {
    redf2[w] = make_float2(ga, gb);
    redf2[kWarps + w] = make_float2(ma, mb);
  }
  __syncthreads();
  ga = redf2[0].x; gb = redf2[0].y; ma = redf2[kWarps].x; mb = redf2[kWarps].y;
#pragma unroll
  for (int i = 1; i < kWarps; ++i) {
    ga = fmaxf(ga, redf2[i].x);
    gb = fmaxf(gb, redf2[i].y);
    ma = fmaxf(ma, redf2[kWarps + i].x);
    mb = fmaxf(mb, redf2[kWarps + i].y);
  }
  double sa = warp_sum(rescale_pow2(a.S, a.ref, ga));
  double sb = warp_sum(rescale_pow2(b.S, b.ref, gb));
  if (lane == 0) redd2[w] = make_double2(sa, sb);
  __syncthreads();
  sa = redd2[0].x;
  sb = redd2[0].y;
#pragma unroll
  for (int i = 1; i < kWarps; ++i) {
    sa += redd2[i].x;
    sb += redd2[i].y;
  }
  ra->G = ga; ra->mz = ma; ra->S = sa;
  rb->G = gb; rb->mz = mb; rb->S = sb;
}

// Combine per-lane partials of warp 0 (lane q holds CTA q's, lanes >= C hold
// G = -inf, S = 0) into the row's exponent reference and normaliser.  The
// xor butterflies give every lane, and every CTA running the same code on
// the same values, identical bits.
__device__ __forceinline__ void warp_stat_combine(float G, double S, float* Gout, double* Sout) {
  const float Gm = warp_max(G);
  *Gout = Gm;
  *Sout = warp_sum(rescale_pow2(S, G, Gm));
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
    v = y > v ? y : v;
  }
  return v;
}

// Inclusive scan over the 32 lanes in a fixed order (lanes >= C add 0).
__device__ __forceinline__ double warp_scan_incl(double v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// ---------------------------------------------------------------------------
// Top-K keys: (value desc, index asc) as one 64-bit integer, larger = better.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t float_order(float v) {
  uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_float(uint32_t o) {
  uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return __uint_as_float(u);
}
__device__ __forceinline__ unsigned long long topk_key(float v, int idx) {
  return ((unsigned long long)float_order(v) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)idx);
}
__device__ __forceinline__ int key_index(unsigned long long k) {
  return (int)(0xffffffffu - (uint32_t)(k & 0xffffffffull));
}
__device__ __forceinline__ float key_value(unsigned long long k) {
  return order_float((uint32_t)(k >> 32));
}
constexpr unsigned long long kNoKey = 0ull;  // below every real key (even -inf)

// Bitonic sort of one key per lane, descending (lane 0 largest).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool take_max = ((lane & j) == 0) == ((lane & k) == 0);
      v = take_max ? (o > v ? o : v) : (o < v ? o : v);
    }
  }
  return v;
}

// Merge two descending lists held one key per lane; keeps the 32 largest,
// descending (reverse one list, take the lane-wise maxima, which form a
// bitonic sequence holding the 32 largest, and sort it with a half cleaner).
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long a,
                                                              unsigned long long b) {
  const int lane = threadIdx.x & 31;
  const unsigned long long br = __shfl_sync(0xffffffffu, b, 31 - lane);
  unsigned long long v = a > br ? a : br;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, j);
    v = ((lane & j) == 0) ? (o > v ? o : v) : (o < v ? o : v);
  }
  return v;
}

}  // namespace sv
