// sv_api.cu -- the C ABI of libsv: argument validation, plans, workspace
// layout and dispatch of the streaming pass and the finishing pass.  No entry
// point synchronises or allocates.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "sv_chain.cuh"
#include "sv_finish.cuh"
#include "sv_tree_sample.cuh"

namespace sv {

namespace {

constexpr int kMaxV = kMaxChunk * kMaxCluster;  // 524288: finishing plan limit
constexpr int kMaxSmem = 200 * 1024;            // hard per-CTA limit used by plans

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

enum : int { kKnobClusterCtas = 1, kKnobStreamCount = 2, kKnobStreamW = 3, kKnobPersistent = 8,
              kKnobKernelMarks = 9, kKnobFinishRead = 10, kKnobCount = 16 };
long long g_knobs[kKnobCount];

// Kernel timing marks.  With the knob set, every kernel launch of the library
// is bracketed by two events recorded on its stream, kept in a ring, and
// sv_kernel_times reads the durations of the launches since its last call.
// The records are external ones, which stream capture turns into event
// record nodes, so the calls of a captured graph are timed launch by launch
// at every replay.
enum : int { kMarkStream = 0, kMarkFinish = 1, kMarkChain = 2 };
constexpr int kMarkLaunches = 2048;
struct MarkRing {
  cudaEvent_t ev[2 * kMarkLaunches];
  int tag[kMarkLaunches];
  long long pos;  // launches bracketed since the last read
  int dev;        // device the events belong to, -1 before the first mark
};
MarkRing g_mark = {{}, {}, 0, -1};

bool marks_on() { return knob(kKnobKernelMarks) != 0; }

cudaError_t mark_events_ready() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || g_mark.dev == dev) return e;
  if (g_mark.dev >= 0) {
    int cur = dev;
    cudaSetDevice(g_mark.dev);
    for (auto& ev : g_mark.ev) cudaEventDestroy(ev);
    cudaSetDevice(cur);
  }
  g_mark.dev = -1;
  for (auto& ev : g_mark.ev)
    if ((e = cudaEventCreate(&ev)) != cudaSuccess) return e;
  g_mark.dev = dev;
  g_mark.pos = 0;
  return cudaSuccess;
}

cudaError_t mark_record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
             : cudaEventRecord(ev, s);
}

// Event before a launch (no-op without the knob).
cudaError_t mark_before(cudaStream_t s) {
  if (!marks_on()) return cudaSuccess;
  cudaError_t e = mark_events_ready();
  if (e != cudaSuccess) return e;
  return mark_record(g_mark.ev[2 * (g_mark.pos % kMarkLaunches)], s);
}

// Event after a launch, and the launch's tag; passes on the launch's error.
cudaError_t mark_after(cudaStream_t s, int tag, cudaError_t launched) {
  if (!marks_on() || launched != cudaSuccess || g_mark.dev < 0) return launched;
  const long long q = g_mark.pos % kMarkLaunches;
  g_mark.tag[q] = tag;
  ++g_mark.pos;
  return mark_record(g_mark.ev[2 * q + 1], s);
}

int forced_cluster() {
  const int c = (int)knob(kKnobClusterCtas);
  return (c >= 1 && c <= kMaxCluster) ? c : 0;
}

// Finishing plans: every cluster size C (1..16) whose chunk of
// ceil(V / C) elements fits the shared-memory limit, C ascending.
template <class XB>
int feasible_plans(int V, int tb, int db, XB x_bytes, bool bulk_ok, int rows_bytes, RowPlan* plans) {
  if (V < 1 || V > kMaxV) return 0;
  const int forced = forced_cluster();
  int n = 0;
  for (int C = 1; C <= kMaxCluster; ++C) {
    if (forced && C != forced) continue;
    const int L = (int)align_up((size_t)((V + C - 1) / C), kVec);
    if (L > kMaxChunk) continue;
    const int np = (L + kRound - 1) / kRound;
    RowLayout lay;
    lay.off_rows = kFixedBytes;
    lay.off_t = kFixedBytes + (int)align_up((size_t)rows_bytes, 128);
    lay.off_d = lay.off_t + (int)align_up((size_t)L * tb, 128);
    lay.off_x = lay.off_d + (int)align_up((size_t)L * db, 128);
    lay.bytes = lay.off_x + (int)align_up((size_t)x_bytes(L, np), 128);
    if (lay.bytes > kMaxSmem) continue;
    plans[n++] = RowPlan{C, L, np, bulk_ok ? 1 : 0, lay};
  }
  return n;
}

bool bulk_ok_row(const void* base, int V, int es) {
  return base != nullptr && aligned(base, 16) && ((size_t)V * es) % 16 == 0;
}

// The kernels scale logits by c = fl32(log2(e) / T); T must leave c finite.
bool scale_ok(float T) {
  return T > 0.f && isfinite(T) && isfinite((float)(1.4426950408889634 / (double)T));
}

int esize(sv_dtype d) { return d == SV_BF16 ? 2 : 4; }
bool dtype_ok(int d) { return d == SV_F32 || d == SV_BF16; }

sv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SV_OK : SV_ERR_CUDA; }

// ---------------------------------------------------------------------------
// Per-device caches of kernel attributes and occupancy.
// ---------------------------------------------------------------------------
struct AttrEntry {
  const void* kernel;
  int device, smem, extra, value;
};
constexpr int kSlots = 512;
AttrEntry g_attr[kSlots];
int g_attr_n = 0;
AttrEntry g_occ[kSlots];
int g_occ_n = 0;
int g_sms[64];
std::mutex g_mu;

}  // namespace

long long knob(int id) {
  if (id < 0 || id >= kKnobCount) return 0;
  return __atomic_load_n(&g_knobs[id], __ATOMIC_RELAXED);
}

cudaError_t ensure_kernel_attrs(const void* kernel, int smem_bytes, bool nonportable) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  AttrEntry* slot = nullptr;
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].kernel == kernel && g_attr[i].device == dev) slot = &g_attr[i];
  if (slot && slot->smem >= smem_bytes && (slot->extra || !nonportable)) return cudaSuccess;
  const int want = slot && slot->smem > smem_bytes ? slot->smem : smem_bytes;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
  if (e != cudaSuccess) return e;
  const bool np = nonportable || (slot && slot->extra);
  if (np) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  if (!slot) {
    if (g_attr_n == kSlots) return cudaSuccess;  // table full: set every time
    slot = &g_attr[g_attr_n++];
    slot->kernel = kernel;
    slot->device = dev;
  }
  slot->smem = want;
  slot->extra = np ? 1 : 0;
  return cudaSuccess;
}

static cudaError_t blocks_per_sm(const void* kernel, int threads, int smem, int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_occ_n; ++i)
    if (g_occ[i].kernel == kernel && g_occ[i].device == dev && g_occ[i].smem == smem &&
        g_occ[i].extra == threads) {
      *out = g_occ[i].value;
      return cudaSuccess;
    }
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, (size_t)smem);
  if (e != cudaSuccess) return e;
  if (g_occ_n < kSlots) g_occ[g_occ_n++] = AttrEntry{kernel, dev, smem, threads, n};
  *out = n;
  return cudaSuccess;
}

cudaError_t sm_count(int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_sms[dev] = n;
  }
  *out = g_sms[dev];
  return cudaSuccess;
}

// Chunk length of the stream (a multiple of the piece, at most 8 pieces):
// long enough to amortise the per-chunk record, short enough that a batch
// gives every warp of the device several chunks (about 16384 in all), which
// keeps the tail of the dynamic schedule short.  It
// depends on the sizes only, so workspace sizes are device independent.
static int stream_chunk(int V, long long nrows) {
  const int forced = (int)knob(kKnobStreamW);
  if (forced >= kPiece && forced % kPiece == 0) return forced;
  int w = kPiece;
  while (w < 8 * kPiece && (long long)V * nrows / (2 * w) >= 16384) w *= 2;
  const int cap = (int)align_up((size_t)V, kPiece);
  return w < cap ? w : cap;
}

// Record slots per row: one per piece, enough for either schedule (a record
// per chunk of W >= kPiece elements, or one per run of pieces).
static int record_slots(int V) { return (V + kPiece - 1) / kPiece; }

// Workspace: batch and item counters, per-request rejection words, per-row chunk
// counters, row records, chunk partials and (top-K) chunk lists.  Every byte
// is zero between calls.
static WsLayout ws_layout(int B, int nrows, int nchunk, int K) {
  WsLayout w;
  size_t o = 0;
  w.off_glob = o;
  o += 256;  // batch counter (word 0) and the stream's item counters (words 32..63)
  w.off_reject = o;
  o = align_up(o + 4 * (size_t)B, 16);
  w.off_counter = o;
  o = align_up(o + 4 * (size_t)nrows, 16);
  w.off_rec = o;
  o += sizeof(RowRec) * (size_t)nrows;
  w.off_part = o;
  o += sizeof(Partial) * (size_t)nrows * nchunk;
  w.off_cand = o;
  o += 8 * (size_t)nrows * nchunk * K;
  w.bytes = align_up(o, 256);
  return w;
}

struct WsPtrs {
  uint32_t* glob;
  uint32_t* reject;
  uint32_t* counter;
  RowRec* rec;
  Partial* part;
  unsigned long long* cand;
};

static WsPtrs ws_carve(void* base, const WsLayout& l) {
  unsigned char* p = static_cast<unsigned char*>(base);
  return WsPtrs{reinterpret_cast<uint32_t*>(p + l.off_glob),
                reinterpret_cast<uint32_t*>(p + l.off_reject),
                reinterpret_cast<uint32_t*>(p + l.off_counter),
                reinterpret_cast<RowRec*>(p + l.off_rec), reinterpret_cast<Partial*>(p + l.off_part),
                reinterpret_cast<unsigned long long*>(p + l.off_cand)};
}

// ---------------------------------------------------------------------------
// Streaming pass.
// ---------------------------------------------------------------------------
struct StreamGeom {
  int W, nchunk, stage_bytes, stage_off1, smem;
};

static StreamGeom stream_geom(int V, long long nrows, int te, int de) {
  StreamGeom g;
  g.W = stream_chunk(V, nrows);
  g.nchunk = (V + g.W - 1) / g.W;
  g.stage_off1 = (int)align_up((size_t)kPiece * te, 128);
  g.stage_bytes = g.stage_off1 + (int)align_up((size_t)kPiece * de, 128);
  g.smem = kStreamWarps * kStages * g.stage_bytes + kStreamWarps * kStages * 8 +
           kStreamWarps * 2 * (int)sizeof(IssueDesc);
  return g;
}

// In-stream row counting (count = -1: decide here).  It only pays when a
// chain's positions run one after another, letting rows after a rejection be
// skipped: every position must span at least three rounds of the resident
// warps.  Otherwise the finisher completes the rows and the stream spends
// nothing per item on counting.
static int stream_count_policy(const StreamParams& p, long long resident_warps) {
  const int forced = (int)knob(kKnobStreamCount);
  if (forced == 1 || forced == 2) return forced - 1;  // 1: off, 2: on
  return (long long)p.B * p.nchunk >= 3 * resident_warps ? 1 : 0;
}

template <class T0, class T1, int FLAGS>
static cudaError_t launch_stream(StreamParams& p, const StreamGeom& g, cudaStream_t s) {
  auto kd = stream_kernel<T0, T1, FLAGS>;             // dynamic items, in-stream counting
  auto ks = stream_kernel<T0, T1, FLAGS | kFStatic>;  // static partition
  cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(kd), g.smem, false);
  if (e != cudaSuccess) return e;
  if ((e = ensure_kernel_attrs(reinterpret_cast<const void*>(ks), g.smem, false)) != cudaSuccess)
    return e;
  int per_sm = 0, sms = 0;
  if ((e = blocks_per_sm(reinterpret_cast<const void*>(kd), kStreamThreads, g.smem, &per_sm)) !=
      cudaSuccess)
    return e;
  if ((e = sm_count(&sms)) != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  if (p.count < 0) p.count = stream_count_policy(p, (long long)per_sm * sms * kStreamWarps);
  if (p.count == 0) {  // static partition into pieces (one record slot each)
    p.W = kPiece;
    p.nchunk = record_slots(p.V);
    p.div_nchunk = make_fastdiv(p.nchunk);
  }
  const long long items = (long long)p.nrows * p.nchunk;
  long long grid = (long long)per_sm * sms;
  const long long need = (items + kStreamWarps - 1) / kStreamWarps;
  if (need < grid) grid = need;
  if (grid < 1) grid = 1;
  p.nwarps_eff = (int)(grid * kStreamWarps < items ? grid * kStreamWarps : items);
  if ((e = mark_before(s)) != cudaSuccess) return e;
  if (p.count == 0)
    ks<<<(unsigned)grid, kStreamThreads, g.smem, s>>>(p);
  else
    kd<<<(unsigned)grid, kStreamThreads, g.smem, s>>>(p);
  return mark_after(s, kMarkStream, cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Finishing pass.
// ---------------------------------------------------------------------------
template <class K, class Prm>
static cudaError_t launch_clusters(K kernel, const Prm& prm, const RowPlan& plan, int nclusters,
                                   cudaStream_t s) {
  cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(kernel), plan.lay.bytes,
                                      plan.C > 8);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nclusters * (unsigned)plan.C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)plan.lay.bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)plan.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps the stream's tail
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if ((e = mark_before(s)) != cudaSuccess) return e;
  return mark_after(s, kMarkFinish, cudaLaunchKernelEx(&cfg, kernel, prm));
}

template <class K, class Prm>
static cudaError_t launch_blocks(K kernel, const Prm& prm, int blocks, int smem, cudaStream_t s) {
  cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(kernel), smem, false);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlaps the stream's tail
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((e = mark_before(s)) != cudaSuccess) return e;
  return mark_after(s, kMarkFinish, cudaLaunchKernelEx(&cfg, kernel, prm));
}

// Clusters of plan.C CTAs of this kernel that the device holds at once.
template <class K>
static cudaError_t cluster_capacity(K kernel, const RowPlan& plan, int* out) {
  const void* kp = reinterpret_cast<const void*>(kernel);
  cudaError_t e = ensure_kernel_attrs(kp, plan.lay.bytes, plan.C > 8);
  if (e != cudaSuccess) return e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_occ_n; ++i)
      if (g_occ[i].kernel == kp && g_occ[i].device == dev && g_occ[i].smem == plan.lay.bytes &&
          g_occ[i].extra == -plan.C) {
        *out = g_occ[i].value;
        return cudaSuccess;
      }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)plan.C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)plan.lay.bytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)plan.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&n, kp, &cfg)) != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_occ_n < kSlots) g_occ[g_occ_n++] = AttrEntry{kp, dev, plan.lay.bytes, -plan.C, n};
  *out = n;
  return cudaSuccess;
}

// Cluster size for `nclusters` requests: the plan minimising
// waves * (chunk + a fixed latency worth of elements), where waves is the
// number of rounds of co-resident clusters the grid needs.  A smaller
// cluster (longer chunk) wins when it keeps the grid in one wave.  With
// `fractional`, a partial last wave counts by its share (the clusters of a
// multi-wave grid start as others finish).
template <class K>
static cudaError_t pick_plan(K kernel, const RowPlan* plans, int np, int nclusters,
                             RowPlan* out, long long* waves_out = nullptr,
                             bool fractional = false) {
  constexpr long long kLatencyElems = 8192;
  double best = -1.0;
  for (int i = 0; i < np; ++i) {
    int cap = 0;
    cudaError_t e = cluster_capacity(kernel, plans[i], &cap);
    if (e != cudaSuccess) return e;
    if (cap < 1) continue;
    const long long waves = (nclusters + cap - 1) / cap;
    const double w = fractional ? (double)nclusters / cap : (double)waves;
    const double cost = w * (double)(plans[i].L + kLatencyElems);
    if (best < 0.0 || cost < best) {
      best = cost;
      *out = plans[i];
      if (waves_out) *waves_out = waves;
    }
  }
  return best < 0.0 ? cudaErrorInvalidConfiguration : cudaSuccess;
}

// Finishing plans of the sampling chain: `staged` (the drawn row's chunk
// copied to shared memory) while every cluster is resident in one wave, else
// `direct` (read from global memory, little shared memory per CTA).
template <class TT, class DT, int DKIND>
static cudaError_t run_chain_sample(StreamParams sp, const StreamGeom& sg, FinishParams fp,
                                    const RowPlan* staged, int ns, const RowPlan* direct, int nd,
                                    bool kd, cudaStream_t s) {
  // probability drafts are not streamed: q(x) is read directly
  constexpr int base = kFStats0 | kFGather | (DKIND == kDraftLogits ? (kFRow1 | kFStats1) : 0);
  auto fin_s = kd ? chain_sample_finish<TT, DT, DKIND, true, true>
                  : chain_sample_finish<TT, DT, DKIND, false, true>;
  auto fin_d = kd ? chain_sample_finish<TT, DT, DKIND, true, false>
                  : chain_sample_finish<TT, DT, DKIND, false, false>;
  RowPlan plan;
  long long waves = 0;
  const long long force = knob(kKnobFinishRead);  // 1 staged, 2 direct
  cudaError_t e = ns > 0 && force != 2 ? pick_plan(fin_s, staged, ns, fp.B, &plan, &waves)
                                      : cudaErrorInvalidConfiguration;
  bool use_staged = true;
  if (e != cudaSuccess || (waves != 1 && force != 1)) {
    use_staged = false;
    e = pick_plan(fin_d, direct, nd, fp.B, &plan, nullptr, true);
  }
  if (e != cudaSuccess) return e;
  fp.L = plan.L;
  fp.use_bulk = plan.use_bulk;
  fp.lay = plan.lay;
  static_assert(base == chain_sample_flags<DKIND, false>(), "stream and finisher flags");
  const bool rg = sp.klen != nullptr || sp.active != nullptr;
  e = kd ? (rg ? launch_stream<TT, DT, base | kFTopk0 | kFRagged>(sp, sg, s)
               : launch_stream<TT, DT, base | kFTopk0>(sp, sg, s))
         : (rg ? launch_stream<TT, DT, base | kFRagged>(sp, sg, s)
               : launch_stream<TT, DT, base>(sp, sg, s));
  if (e != cudaSuccess) return e;
  fp.sp = sp;
  return use_staged ? launch_clusters(fin_s, fp, plan, fp.B, s)
                    : launch_clusters(fin_d, fp, plan, fp.B, s);
}

}  // namespace sv

using namespace sv;

// Chain calls take the two-kernel path; with the persistent knob set, chains
// of at most kChainMaxK drafts run as one persistent launch.
static bool chain_legacy(int k) { return k > kChainMaxK || knob(kKnobPersistent) == 0; }

extern "C" {

size_t sv_verify_chain_workspace_size(int B, int k, int V, int K) {
  if (B <= 0 || k < 1 || V < 1) return 256;
  if (!chain_legacy(k)) return chain_ws_bytes(B, k, V, K > 0 ? K : 0);
  return ws_layout(B, B * (k + 1), record_slots(V), K > 0 ? K : 0).bytes;
}
size_t sv_verify_tree_workspace_size(int B, int n, int V) {
  if (B <= 0 || n < 1 || V < 1) return 256;
  return ws_layout(B, B * n, record_slots(V), 0).bytes;
}
size_t sv_extract_topk_workspace_size(int rows, int V, int K) {
  if (rows <= 0 || V < 1) return 256;
  return ws_layout(rows, rows, record_slots(V), K > 0 ? K : 0).bytes;
}
size_t sv_kd_kl_loss_workspace_size(int B, int k, int V) {
  if (B <= 0 || k < 1 || V < 1) return 256;
  return ws_layout(B, B * k, record_slots(V), 0).bytes;
}

static sv_status check_workspace(void* ws, size_t bytes, size_t need) {
  if (!ws || !aligned(ws, 16) || bytes < need) return SV_ERR_WORKSPACE;
  return SV_OK;
}

}  // extern "C"

// Host-side checks of a chain call, before anything touches the workspace
// or the device (every chain entry point runs them first).
static sv_status validate_chain(const void* target_logits, sv_dtype t_dtype, const void* draft,
                                sv_dtype d_dtype, sv_draft_kind d_kind,
                                const int32_t* draft_tokens, const float* uniforms,
                                const int32_t* draft_len, const int32_t* active, int B, int k,
                                int V, float temperature, int32_t* accepted_len,
                                int32_t* out_tokens, const sv_kd_args* kd,
                                int32_t* device_status) {
  if (B < 0 || k < 1 || k > 255 || V < 1) return SV_ERR_INVALID_ARG;
  if ((draft_len && !aligned(draft_len, 4)) || (active && !aligned(active, 4)))
    return SV_ERR_INVALID_ARG;
  if (!(temperature >= 0.f) || !isfinite(temperature)) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(t_dtype)) return SV_ERR_INVALID_ARG;
  if (kd && (kd->K < 1 || kd->K > kMaxK || kd->K > V)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!target_logits || !draft_tokens || !accepted_len || !out_tokens) return SV_ERR_INVALID_ARG;
  if (!aligned(target_logits, esize(t_dtype)) || !aligned(draft_tokens, 4) ||
      !aligned(accepted_len, 4) || !aligned(out_tokens, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  const bool greedy = temperature == 0.f;
  if (greedy && kd) return SV_ERR_INVALID_ARG;
  if (!greedy) {
    if (!draft || !uniforms || !aligned(uniforms, 4)) return SV_ERR_INVALID_ARG;
    if (d_kind != SV_DRAFT_LOGITS && d_kind != SV_DRAFT_PROBS) return SV_ERR_INVALID_ARG;
    if (!dtype_ok(d_dtype)) return SV_ERR_INVALID_ARG;
    if (d_kind == SV_DRAFT_PROBS && d_dtype != SV_F32) return SV_ERR_INVALID_ARG;
    if (!aligned(draft, esize(d_dtype))) return SV_ERR_INVALID_ARG;
    if (!scale_ok(temperature)) return SV_ERR_INVALID_ARG;
  }
  if (kd) {
    if (!kd->topk_logp || !kd->topk_idx || !kd->lse || !kd->kl || !kd->reward || !kd->loss ||
        !kd->total)
      return SV_ERR_INVALID_ARG;
    if (kd->wmode != SV_W_RAW && kd->wmode != SV_W_GROUP_NORM) return SV_ERR_INVALID_ARG;
    if (kd->wmode == SV_W_GROUP_NORM && (kd->group < 1 || B % kd->group != 0))
      return SV_ERR_INVALID_ARG;
    if (!isfinite(kd->clip)) return SV_ERR_INVALID_ARG;
  }
  if (V > kMaxV) return SV_ERR_UNSUPPORTED;
  if ((long long)B * (k + 1) > 0x7fffffffLL / 64) return SV_ERR_UNSUPPORTED;
  return SV_OK;
}

// Chain verification, padded (draft_len == active == nullptr) or ragged.
static sv_status verify_chain_impl(const void* target_logits, sv_dtype t_dtype, const void* draft,
                                   sv_dtype d_dtype, sv_draft_kind d_kind,
                                   const int32_t* draft_tokens, const float* uniforms,
                                   const int32_t* draft_len, const int32_t* active, int B, int k,
                                   int V, float temperature, int32_t* accepted_len,
                                   int32_t* out_tokens, const sv_kd_args* kd, void* workspace,
                                   size_t workspace_bytes, int32_t* device_status, void* stream) {
  sv_status vst = validate_chain(target_logits, t_dtype, draft, d_dtype, d_kind, draft_tokens,
                                 uniforms, draft_len, active, B, k, V, temperature, accepted_len,
                                 out_tokens, kd, device_status);
  if (vst != SV_OK || B == 0) return vst;
  const bool greedy = temperature == 0.f;
  if (!chain_legacy(k)) {
    const sv_status st = check_workspace(
        workspace, workspace_bytes, sv_verify_chain_workspace_size(B, k, V, kd ? kd->K : 0));
    if (st != SV_OK) return st;
    ChainArgs ca;
    ca.target = target_logits;
    ca.t_dtype = t_dtype;
    ca.draft = greedy ? nullptr : draft;
    ca.d_dtype = d_dtype;
    ca.d_kind = d_kind;
    ca.tokens = draft_tokens;
    ca.u = uniforms;
    ca.klen = draft_len;
    ca.active = active;
    ca.B = B;
    ca.k = k;
    ca.V = V;
    ca.temperature = temperature;
    ca.accepted_len = accepted_len;
    ca.out_tokens = out_tokens;
    ca.kd = kd;
    ca.workspace = workspace;
    ca.status = device_status;
    ca.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mark_before(ca.stream);
    if (e != cudaSuccess) return SV_ERR_CUDA;
    return cuda_status(mark_after(ca.stream, kMarkChain,
                                  t_dtype == SV_BF16 ? launch_chain_bf16(ca) : launch_chain_f32(ca)));
  }
  const int P = k + 1;
  if ((long long)B * P > 0x7fffffffLL / 64) return SV_ERR_UNSUPPORTED;
  const int K = kd ? kd->K : 0;
  const int te = esize(t_dtype);
  const int de = greedy ? 0 : (d_kind == SV_DRAFT_PROBS ? 4 : esize(d_dtype));
  const StreamGeom sg = stream_geom(V, (long long)B * P, te, d_kind == SV_DRAFT_PROBS ? 0 : de);
  const WsLayout wl = ws_layout(B, B * P, record_slots(V), K);
  sv_status st = check_workspace(workspace, workspace_bytes, wl.bytes);
  if (st != SV_OK) return st;
  const WsPtrs w = ws_carve(workspace, wl);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  StreamParams sp = {};
  sp.count = -1;  // decided at launch
  sp.rows0 = target_logits;
  sp.rows1 = greedy ? nullptr : draft;
  sp.tokens = draft_tokens;
  sp.u = uniforms;
  sp.kind = greedy ? kKindChainGreedy : kKindChainSample;
  sp.B = B;
  sp.k = k;
  sp.V = V;
  sp.nrows = B * P;
  sp.W = sg.W;
  sp.nchunk = sg.nchunk;
  sp.div_nchunk = make_fastdiv(sg.nchunk);
  sp.div_B = make_fastdiv(sp.B);
  sp.c = greedy ? 0.f : (float)(1.4426950408889634 / (double)temperature);
  sp.use_bulk = bulk_ok_row(target_logits, V, te) && (greedy || bulk_ok_row(draft, V, de));
  sp.K = K > 0 ? K : 1;
  sp.stage_bytes = sg.stage_bytes;
  sp.stage_off1 = sg.stage_off1;
  sp.part = w.part;
  sp.cand = w.cand;
  sp.rec = w.rec;
  sp.row_counter = w.counter;
  sp.req_reject = w.reject;
  sp.sched = w.glob + 32;
  sp.status = device_status;
  sp.klen = draft_len;
  sp.active = active;

  FinishParams fp = {};
  fp.target = target_logits;
  fp.draft = draft;
  fp.tokens = draft_tokens;
  fp.u = uniforms;
  fp.B = B;
  fp.k = k;
  fp.V = V;
  fp.nchunk = sg.nchunk;
  fp.K = K;
  fp.c = sp.c;
  fp.accepted_len = accepted_len;
  fp.out_tokens = out_tokens;
  fp.part = w.part;
  fp.cand = w.cand;
  fp.rec = w.rec;
  fp.req_reject = w.reject;
  fp.glob_counter = w.glob;
  fp.status = device_status;
  if (kd) {
    fp.topk_logp = kd->topk_logp;
    fp.topk_idx = kd->topk_idx;
    fp.lse = kd->lse;
    fp.kl = kd->kl;
    fp.reward = kd->reward;
    fp.wmode = kd->wmode;
    fp.group = kd->group < 1 ? 1 : kd->group;
    fp.clip = kd->clip;
    fp.loss = kd->loss;
    fp.total = kd->total;
    fp.positions = kd->positions ? 1 : 0;
    sp.topk_logp = kd->topk_logp;
    sp.topk_idx = kd->topk_idx;
    sp.lse = kd->lse;
    sp.kl = kd->kl;
  }

  if (greedy) {
    const bool rg = draft_len != nullptr || active != nullptr;
    cudaError_t e =
        t_dtype == SV_BF16
            ? (rg ? launch_stream<BF16, BF16, kFArgmax0 | kFRagged>(sp, sg, s)
                  : launch_stream<BF16, BF16, kFArgmax0>(sp, sg, s))
            : (rg ? launch_stream<F32, F32, kFArgmax0 | kFRagged>(sp, sg, s)
                  : launch_stream<F32, F32, kFArgmax0>(sp, sg, s));
    if (e != cudaSuccess) return SV_ERR_CUDA;
    fp.sp = sp;
    const int gsm = kFixedBytes + P * (int)sizeof(RowRec);
    return cuda_status(t_dtype == SV_BF16 ? launch_blocks(chain_greedy_finish<BF16>, fp, B, gsm, s)
                                          : launch_blocks(chain_greedy_finish<F32>, fp, B, gsm, s));
  }

  // finishing plans with staging buffers for the drawn row's chunk, and
  // without (the chunk read from global memory)
  const auto x_bytes = [](int, int npc) {
    const int x = npc * kThreads * 4 + kThreads * 8;
    return x < 2 * kThreads * 4 ? 2 * kThreads * 4 : x;
  };
  const bool rows_aligned = bulk_ok_row(target_logits, V, te) && bulk_ok_row(draft, V, de);
  RowPlan plans[kMaxCluster], dplans[kMaxCluster];
  const int np = feasible_plans(V, te, de, x_bytes, rows_aligned, P * (int)sizeof(RowRec), plans);
  const int nd = feasible_plans(V, 0, 0, x_bytes, rows_aligned, P * (int)sizeof(RowRec), dplans);
  if (nd == 0) return SV_ERR_UNSUPPORTED;
  cudaError_t e;
  if (d_kind == SV_DRAFT_PROBS)
    e = t_dtype == SV_BF16 ? run_chain_sample<BF16, F32, kDraftProbs>(sp, sg, fp, plans, np, dplans, nd, kd, s)
                           : run_chain_sample<F32, F32, kDraftProbs>(sp, sg, fp, plans, np, dplans, nd, kd, s);
  else if (t_dtype == SV_BF16)
    e = d_dtype == SV_BF16
            ? run_chain_sample<BF16, BF16, kDraftLogits>(sp, sg, fp, plans, np, dplans, nd, kd, s)
            : run_chain_sample<BF16, F32, kDraftLogits>(sp, sg, fp, plans, np, dplans, nd, kd, s);
  else
    e = d_dtype == SV_BF16
            ? run_chain_sample<F32, BF16, kDraftLogits>(sp, sg, fp, plans, np, dplans, nd, kd, s)
            : run_chain_sample<F32, F32, kDraftLogits>(sp, sg, fp, plans, np, dplans, nd, kd, s);
  return cuda_status(e);
}

extern "C" {

sv_status sv_verify_chain(const void* target_logits, sv_dtype t_dtype, const void* draft,
                          sv_dtype d_dtype, sv_draft_kind d_kind, const int32_t* draft_tokens,
                          const float* uniforms, int B, int k, int V, float temperature,
                          int32_t* accepted_len, int32_t* out_tokens, const sv_kd_args* kd,
                          void* workspace, size_t workspace_bytes, int32_t* device_status,
                          void* stream) {
  return verify_chain_impl(target_logits, t_dtype, draft, d_dtype, d_kind, draft_tokens, uniforms,
                           nullptr, nullptr, B, k, V, temperature, accepted_len, out_tokens, kd,
                           workspace, workspace_bytes, device_status, stream);
}

sv_status sv_verify_chain_ragged(const void* target_logits, sv_dtype t_dtype, const void* draft,
                                 sv_dtype d_dtype, sv_draft_kind d_kind,
                                 const int32_t* draft_tokens, const float* uniforms,
                                 const int32_t* draft_len, const int32_t* active, int B, int k,
                                 int V, float temperature, int32_t* accepted_len,
                                 int32_t* out_tokens, const sv_kd_args* kd, void* workspace,
                                 size_t workspace_bytes, int32_t* device_status, void* stream) {
  return verify_chain_impl(target_logits, t_dtype, draft, d_dtype, d_kind, draft_tokens, uniforms,
                           draft_len, active, B, k, V, temperature, accepted_len, out_tokens, kd,
                           workspace, workspace_bytes, device_status, stream);
}

// Scratch of sv_verify_chain_noalloc: one fixed, zero-initialised array per
// device (every completed call returns it to zero).  Its device address is
// looked up on every call, in the calling thread's current context, so a
// context created after a device reset is served correctly.
static __device__ __align__(256) unsigned char g_noalloc_ws[SV_NOALLOC_MAX_BYTES];

sv_status sv_verify_chain_noalloc(const void* target_logits, sv_dtype t_dtype, const void* draft,
                                  sv_dtype d_dtype, sv_draft_kind d_kind,
                                  const int32_t* draft_tokens, const float* uniforms, int B, int k,
                                  int V, float temperature, int32_t* accepted_len,
                                  int32_t* out_tokens, const sv_kd_args* kd,
                                  int32_t* device_status, void* stream) {
  // the same argument checks and codes as sv_verify_chain, first
  const sv_status vst =
      validate_chain(target_logits, t_dtype, draft, d_dtype, d_kind, draft_tokens, uniforms,
                     nullptr, nullptr, B, k, V, temperature, accepted_len, out_tokens, kd,
                     device_status);
  if (vst != SV_OK || B == 0) return vst;
  const size_t need = sv_verify_chain_workspace_size(B, k, V, kd ? kd->K : 0);
  if (need > (size_t)SV_NOALLOC_MAX_BYTES) return SV_ERR_WORKSPACE;
  void* ws = nullptr;
  if (cudaGetSymbolAddress(&ws, g_noalloc_ws) != cudaSuccess || ws == nullptr) return SV_ERR_CUDA;
  const sv_status st =
      sv_verify_chain(target_logits, t_dtype, draft, d_dtype, d_kind, draft_tokens, uniforms, B, k,
                      V, temperature, accepted_len, out_tokens, kd, ws,
                      (size_t)SV_NOALLOC_MAX_BYTES, device_status, stream);
  // A launch that failed part way (the two-kernel path) can leave the
  // scratch in use: return it to zero on the same stream.
  if (st == SV_ERR_CUDA)
    cudaMemsetAsync(ws, 0, need, reinterpret_cast<cudaStream_t>(stream));
  return st;
}

sv_status sv_kernel_times(float* us, int32_t* tags, int cap, int32_t* n) {
  if (n == nullptr || (cap > 0 && (us == nullptr || tags == nullptr)) || cap < 0)
    return SV_ERR_INVALID_ARG;
  *n = 0;
  if (g_mark.dev < 0 || g_mark.pos == 0) return SV_OK;
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != g_mark.dev) return SV_ERR_INVALID_ARG;
  const long long total = g_mark.pos;
  const long long kept = total < kMarkLaunches ? total : kMarkLaunches;
  const long long first = total - kept;
  const long long last = (total - 1) % kMarkLaunches;
  if (cudaEventSynchronize(g_mark.ev[2 * last + 1]) != cudaSuccess) return SV_ERR_CUDA;
  int m = 0;
  for (long long j = first; j < total && m < cap; ++j, ++m) {
    const long long q = j % kMarkLaunches;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_mark.ev[2 * q], g_mark.ev[2 * q + 1]) != cudaSuccess)
      return SV_ERR_CUDA;
    us[m] = 1e3f * ms;
    tags[m] = g_mark.tag[q];
  }
  *n = m;
  g_mark.pos = 0;
  return SV_OK;
}

sv_status sv_set_knob(int knob_id, long long value) {
  if (knob_id < 1 || knob_id > kKnobFinishRead) return SV_ERR_INVALID_ARG;
  __atomic_store_n(&g_knobs[knob_id], value, __ATOMIC_RELAXED);
  return SV_OK;
}

sv_status sv_verify_tree_greedy(const void* logits, sv_dtype dt, const int32_t* node_tokens,
                                const int32_t* parents, int B, int n, int V, int max_depth,
                                int32_t* accepted_len, int32_t* out_tokens,
                                int32_t* accepted_nodes, void* workspace, size_t workspace_bytes,
                                int32_t* device_status, void* stream) {
  if (B < 0 || n < 1 || n > 1024 || V < 1 || max_depth < 0 || max_depth >= n)
    return SV_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!logits || !node_tokens || !parents || !accepted_len || !out_tokens || !accepted_nodes)
    return SV_ERR_INVALID_ARG;
  if (!aligned(logits, esize(dt)) || !aligned(node_tokens, 4) || !aligned(parents, 4) ||
      !aligned(accepted_len, 4) || !aligned(out_tokens, 4) || !aligned(accepted_nodes, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if ((long long)B * n > 0x7fffffffLL / 64) return SV_ERR_UNSUPPORTED;
  const StreamGeom sg = stream_geom(V, (long long)B * n, esize(dt), 0);
  const WsLayout wl = ws_layout(B, B * n, record_slots(V), 0);
  sv_status st = check_workspace(workspace, workspace_bytes, wl.bytes);
  if (st != SV_OK) return st;
  const WsPtrs w = ws_carve(workspace, wl);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  StreamParams sp = {};
  sp.rows0 = logits;
  sp.kind = kKindRows;
  sp.B = B * n;
  sp.k = 1;
  sp.V = V;
  sp.nrows = B * n;
  sp.W = sg.W;
  sp.nchunk = sg.nchunk;
  sp.div_nchunk = make_fastdiv(sg.nchunk);
  sp.div_B = make_fastdiv(sp.B);
  sp.use_bulk = bulk_ok_row(logits, V, esize(dt));
  sp.K = 1;
  sp.stage_bytes = sg.stage_bytes;
  sp.stage_off1 = sg.stage_off1;
  sp.part = w.part;
  sp.cand = w.cand;
  sp.rec = w.rec;
  sp.row_counter = w.counter;
  sp.req_reject = w.reject;
  sp.sched = w.glob + 32;
  sp.status = device_status;
  sp.count = 0;  // no skipping in a tree: the finisher completes the rows
  cudaError_t e = dt == SV_BF16 ? launch_stream<BF16, BF16, kFArgmax0>(sp, sg, s)
                                : launch_stream<F32, F32, kFArgmax0>(sp, sg, s);
  if (e != cudaSuccess) return SV_ERR_CUDA;
  FinishParams fp = {};
  fp.tokens = node_tokens;
  fp.parents = parents;
  fp.B = B;
  fp.k = n;
  fp.V = V;
  fp.nchunk = sg.nchunk;
  fp.max_depth = max_depth;
  fp.accepted_len = accepted_len;
  fp.out_tokens = out_tokens;
  fp.accepted_nodes = accepted_nodes;
  fp.part = w.part;
  fp.rec = w.rec;
  fp.req_reject = w.reject;
  fp.status = device_status;
  fp.sp = sp;
  const int tsm = kFixedBytes + n * (int)sizeof(RowRec) + 4 * n * 4;
  // blocks per tree: one warp per node row folds in parallel (at most 16)
  fp.nsplit = n > kWarps ? (n + kWarps - 1) / kWarps : 1;
  if (fp.nsplit > 16) fp.nsplit = 16;
  if ((long long)B * fp.nsplit > 0x7fffffffLL) fp.nsplit = 1;
  const int nb = B * fp.nsplit;
  return cuda_status(dt == SV_BF16 ? launch_blocks(tree_finish<BF16>, fp, nb, tsm, s)
                                   : launch_blocks(tree_finish<F32>, fp, nb, tsm, s));
}

}  // extern "C"

template <class TT, class DT, int DKIND>
static cudaError_t run_tree_sample(FinishParams fp, int te, int de, bool bulk_ok, cudaStream_t s) {
  RowPlan plans[kMaxCluster];
  // per node: 4 int, 2 float, 2 double, 1 float
  const int rows_bytes = (int)sizeof(TreeShared) + 44 * fp.k;
  const int np = feasible_plans(
      fp.V, te, de,
      [](int, int npc) { return npc * kThreads * 8 + kThreads * 8; },  // float64 sums, scan
      bulk_ok, rows_bytes, plans);
  if (np == 0) return cudaErrorInvalidConfiguration;
  auto kern = tree_sample_kernel<TT, DT, DKIND>;
  RowPlan plan;
  cudaError_t e = pick_plan(kern, plans, np, fp.B, &plan);
  if (e != cudaSuccess) return e;
  fp.L = plan.L;
  fp.use_bulk = plan.use_bulk;
  fp.lay = plan.lay;
  return launch_clusters(kern, fp, plan, fp.B, s);
}

extern "C" {

sv_status sv_verify_tree_sample(const void* target_logits, sv_dtype t_dtype, const void* draft,
                                sv_dtype d_dtype, sv_draft_kind d_kind, const int32_t* node_tokens,
                                const int32_t* parents, const float* uniforms, int B, int n, int V,
                                int max_depth, float temperature, int32_t* accepted_len,
                                int32_t* out_tokens, int32_t* accepted_nodes,
                                int32_t* device_status, void* stream) {
  if (B < 0 || n < 1 || n > 1024 || V < 1 || max_depth < 0 || max_depth >= n)
    return SV_ERR_INVALID_ARG;
  if (!dtype_ok(t_dtype) || !dtype_ok(d_dtype)) return SV_ERR_INVALID_ARG;
  if (d_kind != SV_DRAFT_LOGITS && d_kind != SV_DRAFT_PROBS) return SV_ERR_INVALID_ARG;
  if (d_kind == SV_DRAFT_PROBS && d_dtype != SV_F32) return SV_ERR_INVALID_ARG;
  if (!scale_ok(temperature)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!target_logits || !draft || !node_tokens || !parents || !uniforms || !accepted_len ||
      !out_tokens || !accepted_nodes)
    return SV_ERR_INVALID_ARG;
  const int te = esize(t_dtype), de = esize(d_dtype);
  if (!aligned(target_logits, te) || !aligned(draft, de) || !aligned(node_tokens, 4) ||
      !aligned(parents, 4) || !aligned(uniforms, 4) || !aligned(accepted_len, 4) ||
      !aligned(out_tokens, 4) || !aligned(accepted_nodes, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if (V > kMaxV) return SV_ERR_UNSUPPORTED;
  if ((long long)B * kMaxCluster > 0x7fffffffLL) return SV_ERR_UNSUPPORTED;
  FinishParams fp = {};
  fp.target = target_logits;
  fp.draft = draft;
  fp.tokens = node_tokens;
  fp.parents = parents;
  fp.u = uniforms;
  fp.B = B;
  fp.k = n;
  fp.V = V;
  fp.max_depth = max_depth;
  fp.c = (float)(1.4426950408889634 / (double)temperature);
  fp.c64 = 1.4426950408889634 / (double)temperature;
  fp.accepted_len = accepted_len;
  fp.out_tokens = out_tokens;
  fp.accepted_nodes = accepted_nodes;
  fp.status = device_status;
  const bool bulk = bulk_ok_row(target_logits, V, te) && bulk_ok_row(draft, V, de);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (d_kind == SV_DRAFT_PROBS)
    e = t_dtype == SV_BF16 ? run_tree_sample<BF16, F32, kDraftProbs>(fp, te, de, bulk, s)
                           : run_tree_sample<F32, F32, kDraftProbs>(fp, te, de, bulk, s);
  else if (t_dtype == SV_BF16)
    e = d_dtype == SV_BF16 ? run_tree_sample<BF16, BF16, kDraftLogits>(fp, te, de, bulk, s)
                           : run_tree_sample<BF16, F32, kDraftLogits>(fp, te, de, bulk, s);
  else
    e = d_dtype == SV_BF16 ? run_tree_sample<F32, BF16, kDraftLogits>(fp, te, de, bulk, s)
                           : run_tree_sample<F32, F32, kDraftLogits>(fp, te, de, bulk, s);
  if (e == cudaErrorInvalidConfiguration) return SV_ERR_UNSUPPORTED;
  return cuda_status(e);
}

sv_status sv_extract_topk_kd(const void* logits, sv_dtype dt, int rows, int V, int K,
                             float temperature, float* topk_logp, int32_t* topk_idx, float* lse,
                             void* workspace, size_t workspace_bytes, int32_t* device_status,
                             void* stream) {
  if (rows < 0 || V < 1 || K < 1 || K > kMaxK || K > V) return SV_ERR_INVALID_ARG;
  if (!scale_ok(temperature)) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return SV_ERR_INVALID_ARG;
  if (rows == 0) return SV_OK;
  if (!logits || !topk_logp || !topk_idx || !lse) return SV_ERR_INVALID_ARG;
  if (!aligned(logits, esize(dt)) || !aligned(topk_logp, 4) || !aligned(topk_idx, 4) ||
      !aligned(lse, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if (rows > 0x7fffffff / 64) return SV_ERR_UNSUPPORTED;
  const StreamGeom sg = stream_geom(V, rows, esize(dt), 0);
  const WsLayout wl = ws_layout(rows, rows, record_slots(V), K);
  sv_status st = check_workspace(workspace, workspace_bytes, wl.bytes);
  if (st != SV_OK) return st;
  const WsPtrs w = ws_carve(workspace, wl);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  StreamParams sp = {};
  sp.rows0 = logits;
  sp.kind = kKindRows;
  sp.B = rows;
  sp.k = 1;
  sp.V = V;
  sp.nrows = rows;
  sp.W = sg.W;
  sp.nchunk = sg.nchunk;
  sp.div_nchunk = make_fastdiv(sg.nchunk);
  sp.div_B = make_fastdiv(sp.B);
  sp.c = (float)(1.4426950408889634 / (double)temperature);
  sp.use_bulk = bulk_ok_row(logits, V, esize(dt));
  sp.K = K;
  sp.stage_bytes = sg.stage_bytes;
  sp.stage_off1 = sg.stage_off1;
  sp.part = w.part;
  sp.cand = w.cand;
  sp.rec = w.rec;
  sp.row_counter = w.counter;
  sp.req_reject = w.reject;
  sp.sched = w.glob + 32;
  sp.status = device_status;
  sp.topk_logp = topk_logp;
  sp.topk_idx = topk_idx;
  sp.lse = lse;
  sp.count = 1;  // no finishing kernel: rows complete in the stream
  // one pass: the warp that completes a row merges its chunk lists and writes it
  return cuda_status(dt == SV_BF16 ? launch_stream<BF16, BF16, kFStats0 | kFTopk0>(sp, sg, s)
                                   : launch_stream<F32, F32, kFStats0 | kFTopk0>(sp, sg, s));
}

sv_status sv_kd_kl_loss(const float* topk_logp, const int32_t* topk_idx, int B, int k, int K,
                        const void* draft, sv_dtype d_dtype, sv_draft_kind d_kind, int V,
                        float temperature, const int32_t* accepted_len, const float* reward,
                        sv_weight_mode wmode, int group, float clip, int positions, float* kl,
                        float* loss, float* total, void* workspace, size_t workspace_bytes,
                        int32_t* device_status, void* stream) {
  if (B < 0 || k < 1 || k > 255 || K < 1 || K > kMaxK || V < 1 || K > V) return SV_ERR_INVALID_ARG;
  if (!scale_ok(temperature)) return SV_ERR_INVALID_ARG;
  if (d_kind != SV_DRAFT_LOGITS && d_kind != SV_DRAFT_PROBS) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(d_dtype) || (d_kind == SV_DRAFT_PROBS && d_dtype != SV_F32))
    return SV_ERR_INVALID_ARG;
  if (wmode != SV_W_RAW && wmode != SV_W_GROUP_NORM) return SV_ERR_INVALID_ARG;
  if (wmode == SV_W_GROUP_NORM && (group < 1 || (B > 0 && B % group != 0)))
    return SV_ERR_INVALID_ARG;
  if (!isfinite(clip)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!topk_logp || !topk_idx || !draft || !accepted_len || !reward || !kl || !loss || !total)
    return SV_ERR_INVALID_ARG;
  if (!aligned(topk_logp, 4) || !aligned(topk_idx, 4) || !aligned(draft, esize(d_dtype)) ||
      !aligned(accepted_len, 4) || !aligned(reward, 4) || !aligned(kl, 4) || !aligned(loss, 4) ||
      !aligned(total, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if ((long long)B * k > 0x7fffffffLL / 64) return SV_ERR_UNSUPPORTED;
  const StreamGeom sg = stream_geom(V, (long long)B * k, esize(d_dtype), 0);
  const WsLayout wl = ws_layout(B, B * k, record_slots(V), 0);
  sv_status st = check_workspace(workspace, workspace_bytes, wl.bytes);
  if (st != SV_OK) return st;
  const WsPtrs w = ws_carve(workspace, wl);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const float c = (float)(1.4426950408889634 / (double)temperature);
  StreamParams sp = {};
  if (d_kind == SV_DRAFT_LOGITS) {
    sp.rows0 = draft;
    sp.kind = kKindRows;
    sp.B = B * k;
    sp.k = 1;
    sp.V = V;
    sp.nrows = B * k;
    sp.W = sg.W;
    sp.nchunk = sg.nchunk;
    sp.div_nchunk = make_fastdiv(sg.nchunk);
    sp.div_B = make_fastdiv(sp.B);
    sp.c = c;
    sp.use_bulk = bulk_ok_row(draft, V, esize(d_dtype));
    sp.K = 1;
    sp.stage_bytes = sg.stage_bytes;
    sp.stage_off1 = sg.stage_off1;
    sp.part = w.part;
    sp.cand = w.cand;
    sp.rec = w.rec;
    sp.row_counter = w.counter;
    sp.req_reject = w.reject;
    sp.sched = w.glob + 32;
    sp.status = device_status;
    sp.count = 0;  // the finisher completes the draft rows
    cudaError_t e = d_dtype == SV_BF16 ? launch_stream<BF16, BF16, kFStats0>(sp, sg, s)
                                       : launch_stream<F32, F32, kFStats0>(sp, sg, s);
    if (e != cudaSuccess) return SV_ERR_CUDA;
  }
  FinishParams fp = {};
  fp.draft = draft;
  fp.B = B;
  fp.k = k;
  fp.K = K;
  fp.V = V;
  fp.nchunk = sg.nchunk;
  fp.c = c;
  fp.in_topk_logp = topk_logp;
  fp.in_topk_idx = topk_idx;
  fp.in_accepted_len = accepted_len;
  fp.draft_probs = d_kind == SV_DRAFT_PROBS ? 1 : 0;
  fp.reward = reward;
  fp.wmode = wmode;
  fp.group = group < 1 ? 1 : group;
  fp.clip = clip;
  fp.positions = positions ? 1 : 0;
  fp.kl = kl;
  fp.loss = loss;
  fp.total = total;
  fp.part = w.part;
  fp.rec = w.rec;
  fp.req_reject = w.reject;
  fp.glob_counter = w.glob;
  fp.status = device_status;
  fp.sp = sp;
  const int ksm = kFixedBytes + k * (int)sizeof(RowRec);
  cudaError_t e = (d_dtype == SV_BF16) ? launch_blocks(kl_finish<BF16>, fp, B, ksm, s)
                                       : launch_blocks(kl_finish<F32>, fp, B, ksm, s);
  return cuda_status(e);
}

size_t sv_kd_grad_workspace_size(int B, int k, int V) { return sv_kd_kl_loss_workspace_size(B, k, V); }

sv_status sv_kd_grad(const float* topk_logp, const int32_t* topk_idx, int B, int k, int K,
                     const void* draft, sv_dtype d_dtype, int V, float temperature,
                     const int32_t* accepted_len, const float* reward, sv_weight_mode wmode,
                     int group, float clip, int positions, float* grad, void* workspace,
                     size_t workspace_bytes, int32_t* device_status, void* stream) {
  if (B < 0 || k < 1 || k > 255 || K < 1 || K > kMaxK || V < 1 || K > V) return SV_ERR_INVALID_ARG;
  if (!scale_ok(temperature) || !dtype_ok(d_dtype)) return SV_ERR_INVALID_ARG;
  if (wmode != SV_W_RAW && wmode != SV_W_GROUP_NORM) return SV_ERR_INVALID_ARG;
  if (wmode == SV_W_GROUP_NORM && (group < 1 || (B > 0 && B % group != 0)))
    return SV_ERR_INVALID_ARG;
  if (!isfinite(clip)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!topk_logp || !topk_idx || !draft || !accepted_len || !reward || !grad)
    return SV_ERR_INVALID_ARG;
  if (!aligned(topk_logp, 4) || !aligned(topk_idx, 4) || !aligned(draft, esize(d_dtype)) ||
      !aligned(accepted_len, 4) || !aligned(reward, 4) || !aligned(grad, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if ((long long)B * k > 0x7fffffffLL / 64 || (long long)B * k * V > (1LL << 40))
    return SV_ERR_UNSUPPORTED;
  const StreamGeom sg = stream_geom(V, (long long)B * k, esize(d_dtype), 0);
  const WsLayout wl = ws_layout(B, B * k, record_slots(V), 0);
  sv_status st = check_workspace(workspace, workspace_bytes, wl.bytes);
  if (st != SV_OK) return st;
  const WsPtrs w = ws_carve(workspace, wl);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const float c = (float)(1.4426950408889634 / (double)temperature);
  StreamParams sp = {};
  sp.rows0 = draft;
  sp.kind = kKindRows;
  sp.B = B * k;
  sp.k = 1;
  sp.V = V;
  sp.nrows = B * k;
  sp.W = sg.W;
  sp.nchunk = sg.nchunk;
  sp.div_nchunk = make_fastdiv(sg.nchunk);
  sp.div_B = make_fastdiv(sp.B);
  sp.c = c;
  sp.use_bulk = bulk_ok_row(draft, V, esize(d_dtype));
  sp.K = 1;
  sp.stage_bytes = sg.stage_bytes;
  sp.stage_off1 = sg.stage_off1;
  sp.part = w.part;
  sp.cand = w.cand;
  sp.rec = w.rec;
  sp.row_counter = w.counter;
  sp.req_reject = w.reject;
  sp.sched = w.glob + 32;
  sp.status = device_status;
  sp.count = 0;  // the gradient kernel folds the rows
  cudaError_t e = d_dtype == SV_BF16 ? launch_stream<BF16, BF16, kFStats0>(sp, sg, s)
                                     : launch_stream<F32, F32, kFStats0>(sp, sg, s);
  if (e != cudaSuccess) return SV_ERR_CUDA;
  FinishParams fp = {};
  fp.draft = draft;
  fp.B = B;
  fp.k = k;
  fp.K = K;
  fp.V = V;
  fp.c = c;
  fp.temperature = temperature;
  fp.in_topk_logp = topk_logp;
  fp.in_topk_idx = topk_idx;
  fp.in_accepted_len = accepted_len;
  fp.reward = reward;
  fp.wmode = wmode;
  fp.group = group < 1 ? 1 : group;
  fp.clip = clip;
  fp.positions = positions ? 1 : 0;
  fp.grad = grad;
  fp.part = w.part;
  fp.rec = w.rec;
  fp.status = device_status;
  fp.sp = sp;
  // CTAs per draft row: enough items for about four waves of resident CTAs
  // (so the last wave is nearly full), at most 8, at least 2048 entries each
  {
    const void* kern = d_dtype == SV_BF16 ? reinterpret_cast<const void*>(kd_grad_kernel<BF16>)
                                          : reinterpret_cast<const void*>(kd_grad_kernel<F32>);
    int per_sm = 0, sms = 0;
    if ((e = ensure_kernel_attrs(kern, kFixedBytes, false)) != cudaSuccess) return SV_ERR_CUDA;
    if ((e = blocks_per_sm(kern, kThreads, kFixedBytes, &per_sm)) != cudaSuccess) return SV_ERR_CUDA;
    if ((e = sm_count(&sms)) != cudaSuccess) return SV_ERR_CUDA;
    const long long rows = (long long)B * k, cap = (long long)per_sm * sms;
    long long ns = (4 * cap + rows - 1) / rows;
    ns = ns < 1 ? 1 : (ns > 8 ? 8 : ns);
    const long long by_len = V / 2048 < 1 ? 1 : V / 2048;
    if (ns > by_len) ns = by_len;
    if (rows * ns > 0x7fffffffLL) ns = 1;
    fp.nsplit = (int)ns;
  }
  e = (d_dtype == SV_BF16)
          ? launch_blocks(kd_grad_kernel<BF16>, fp, (int)((long long)B * k * fp.nsplit), kFixedBytes, s)
          : launch_blocks(kd_grad_kernel<F32>, fp, (int)((long long)B * k * fp.nsplit), kFixedBytes, s);
  return cuda_status(e);
}

sv_status sv_device_status_check(int32_t w) {
  if (w & SV_DEV_TIMEOUT) return SV_ERR_TIMEOUT;
  if (w & SV_DEV_ERROR_MASK) return SV_ERR_DEVICE_CHECK;
  return SV_OK;
}

sv_status sv_sched_select(const float* throughput, const int32_t* batches, int n_cfg,
                          int n_batch, int nonspec, int active_batch, int32_t* config,
                          float* predicted_speedup) {
  if (!throughput || !batches || !config || n_cfg < 1 || n_batch < 1 || nonspec < 0 ||
      nonspec >= n_cfg || active_batch < 1)
    return SV_ERR_INVALID_ARG;
  for (int j = 0; j < n_batch; ++j)
    if (batches[j] < 1 || (j > 0 && batches[j] <= batches[j - 1])) return SV_ERR_INVALID_ARG;
  for (long long i = 0; i < (long long)n_cfg * n_batch; ++i)
    if (!(throughput[i] >= 0.f) || !isfinite(throughput[i])) return SV_ERR_INVALID_ARG;
  // the two profiled sizes around the active batch and the weight of the upper one
  int j0 = 0, j1 = 0;
  double t = 0.0;
  if (active_batch >= batches[n_batch - 1]) {
    j0 = j1 = n_batch - 1;
  } else if (active_batch > batches[0]) {
    while (batches[j1] <= active_batch) ++j1;
    j0 = j1 - 1;
    t = (double)(active_batch - batches[j0]) / (double)(batches[j1] - batches[j0]);
  }
  auto at = [&](int c) {
    const double a = throughput[(size_t)c * n_batch + j0], b = throughput[(size_t)c * n_batch + j1];
    return a + t * (b - a);
  };
  const double base = at(nonspec);
  if (!(base > 0.0)) return SV_ERR_INVALID_ARG;
  int best = -1;
  double best_thr = 0.0;
  for (int c = 0; c < n_cfg; ++c) {
    if (c == nonspec) continue;
    const double v = at(c);
    if (best < 0 || v > best_thr) {
      best = c;
      best_thr = v;
    }
  }
  const double speedup = best < 0 ? 0.0 : best_thr / base;
  *config = (best < 0 || speedup < 1.0) ? nonspec : best;
  if (predicted_speedup) *predicted_speedup = (float)speedup;
  return SV_OK;
}

const char* sv_status_string(sv_status s) {
  switch (s) {
    case SV_OK: return "ok";
    case SV_ERR_INVALID_ARG: return "invalid argument";
    case SV_ERR_UNSUPPORTED: return "unsupported size or mode";
    case SV_ERR_CUDA: return "CUDA runtime error";
    case SV_ERR_DEVICE_CHECK: return "device-side input check failed";
    case SV_ERR_TIMEOUT: return "bounded device wait timed out";
    case SV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

int sv_version(void) { return 200; }

}  // extern "C"
