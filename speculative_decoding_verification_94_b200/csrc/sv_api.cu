// sv_api.cu -- the C ABI of libsv: argument validation, row plans, workspace
// layout and kernel dispatch.  No entry point synchronises or allocates.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "sv_rowops.cuh"

namespace sv {

namespace {

constexpr int kMaxV = kMaxChunk * kMaxCluster;  // 524288
constexpr int kTargetSmem = 48 * 1024;          // preferred per-CTA footprint
constexpr int kMaxSmem = 200 * 1024;            // hard per-CTA limit used by plans

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int forced_cluster() {
  const char* s = getenv("SV_CLUSTER_CTAS");
  if (!s) return 0;
  int c = atoi(s);
  return (c == 1 || c == 2 || c == 4 || c == 8 || c == 16) ? c : 0;
}

// Smallest power-of-two cluster whose chunk fits the preferred shared-memory
// footprint (or the largest cluster that fits at all).  `x_bytes(L, np)`
// sizes the scratch region.
template <class XB>
sv_status make_plan(int V, int tb, int db, XB x_bytes, bool bulk_ok, RowPlan* plan) {
  if (V < 1 || V > kMaxV) return SV_ERR_UNSUPPORTED;
  const int forced = forced_cluster();
  RowPlan best = {};
  bool have = false;
  for (int C = 1; C <= kMaxCluster; C *= 2) {
    if (forced && C != forced) continue;
    const int L = (int)align_up((size_t)((V + C - 1) / C), kVec);
    if (L > kMaxChunk) continue;
    const int np = (L + kRound - 1) / kRound;
    RowLayout lay = row_layout(kFixedBytes, L, tb, db, np, x_bytes(L, np));
    if (lay.bytes > kMaxSmem) continue;
    best = RowPlan{C, L, np, bulk_ok ? 1 : 0, lay};
    have = true;
    if (lay.bytes <= kTargetSmem) break;
  }
  if (!have) return SV_ERR_UNSUPPORTED;
  *plan = best;
  return SV_OK;
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

}  // namespace

RowLayout row_layout(int fixed, int L, int tb, int db, int npieces, int x_bytes) {
  (void)npieces;
  RowLayout l;
  l.off_t = fixed;
  l.off_d = l.off_t + (int)align_up((size_t)L * tb, 128);
  l.off_x = l.off_d + (int)align_up((size_t)L * db, 128);
  l.bytes = l.off_x + (int)align_up((size_t)x_bytes, 128);
  return l;
}

namespace {
struct AttrEntry {
  const void* kernel;
  int device;
  int smem;
  bool nonportable;
};
constexpr int kAttrSlots = 256;
AttrEntry g_attr[kAttrSlots];
int g_attr_n = 0;
std::mutex g_attr_mu;
}  // namespace

cudaError_t ensure_kernel_attrs(const void* kernel, int smem_bytes, bool nonportable) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  AttrEntry* slot = nullptr;
  for (int i = 0; i < g_attr_n; ++i)
    if (g_attr[i].kernel == kernel && g_attr[i].device == dev) slot = &g_attr[i];
  if (slot && slot->smem >= smem_bytes && (slot->nonportable || !nonportable)) return cudaSuccess;
  const int want = slot && slot->smem > smem_bytes ? slot->smem : smem_bytes;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
  if (e != cudaSuccess) return e;
  const bool np = nonportable || (slot && slot->nonportable);
  if (np) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  if (!slot) {
    if (g_attr_n == kAttrSlots) return cudaSuccess;  // table full: set every time
    slot = &g_attr[g_attr_n++];
    slot->kernel = kernel;
    slot->device = dev;
  }
  slot->smem = want;
  slot->nonportable = np;
  return cudaSuccess;
}

namespace {
struct OccEntry {
  const void* kernel;
  int device, smem, cluster, n;
};
constexpr int kOccSlots = 256;
OccEntry g_occ[kOccSlots];
int g_occ_n = 0;
std::mutex g_occ_mu;
}  // namespace

cudaError_t max_active_clusters(const void* kernel, int smem_bytes, int cluster, int* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_occ_mu);
  for (int i = 0; i < g_occ_n; ++i)
    if (g_occ[i].kernel == kernel && g_occ[i].device == dev && g_occ[i].smem == smem_bytes &&
        g_occ[i].cluster == cluster) {
      *out = g_occ[i].n;
      return cudaSuccess;
    }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cluster, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem_bytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
  if (e != cudaSuccess) return e;
  if (g_occ_n < kOccSlots) g_occ[g_occ_n++] = OccEntry{kernel, dev, smem_bytes, cluster, n};
  *out = n;
  return cudaSuccess;
}

// Workspace: [0,4) finished-request counter, [4,8) next work item, [8,12)
// retired clusters; [16, 16+4B) per-request row counters; [16+4B, 16+8B)
// per-request rejection words; then two int32 arrays of B*R per-row results.
// Every word is returned to zero by the call that used it.
size_t workspace_bytes(int B, int R) {
  if (B <= 0) return 256;
  size_t n = align_up(16 + 8 * (size_t)B, 16);
  n += 2 * align_up(4 * (size_t)B * (size_t)R, 16);
  return align_up(n, 256);
}

Workspace workspace_carve(void* base, int B, int R) {
  unsigned char* p = static_cast<unsigned char*>(base);
  Workspace w;
  w.glob_counter = reinterpret_cast<uint32_t*>(p);
  w.work = reinterpret_cast<uint32_t*>(p + 4);
  w.done = reinterpret_cast<uint32_t*>(p + 8);
  w.req_counter = reinterpret_cast<uint32_t*>(p + 16);
  w.req_reject = reinterpret_cast<uint32_t*>(p + 16 + 4 * (size_t)B);
  size_t off = align_up(16 + 8 * (size_t)B, 16);
  w.row_a = reinterpret_cast<int32_t*>(p + off);
  off += align_up(4 * (size_t)B * (size_t)R, 16);
  w.row_b = reinterpret_cast<int32_t*>(p + off);
  return w;
}

}  // namespace sv

using namespace sv;

extern "C" {

size_t sv_verify_chain_workspace_size(int B, int k) { return workspace_bytes(B, k + 1); }
size_t sv_verify_tree_workspace_size(int B, int n) { return workspace_bytes(B, n); }
size_t sv_kd_kl_loss_workspace_size(int B, int k) { return workspace_bytes(B, 0); }

static sv_status check_workspace(void* ws, size_t bytes, size_t need) {
  if (!ws || !aligned(ws, 16) || bytes < need) return SV_ERR_WORKSPACE;
  return SV_OK;
}

sv_status sv_verify_chain(const void* target_logits, sv_dtype t_dtype, const void* draft,
                          sv_dtype d_dtype, sv_draft_kind d_kind, const int32_t* draft_tokens,
                          const float* uniforms, int B, int k, int V, float temperature,
                          int32_t* accepted_len, int32_t* out_tokens, const sv_kd_args* kd,
                          void* workspace, size_t workspace_bytes_, int32_t* device_status,
                          void* stream) {
  if (B < 0 || k < 1 || k > 255 || V < 1) return SV_ERR_INVALID_ARG;
  if (!(temperature >= 0.f) || !isfinite(temperature)) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(t_dtype)) return SV_ERR_INVALID_ARG;
  if (B == 0 && (!kd || (kd->K >= 1 && kd->K <= kMaxK && kd->K <= V))) return SV_OK;
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
    if (kd->K < 1 || kd->K > kMaxK || kd->K > V) return SV_ERR_INVALID_ARG;
    if (!kd->topk_logp || !kd->topk_idx || !kd->lse || !kd->kl || !kd->reward || !kd->loss ||
        !kd->total)
      return SV_ERR_INVALID_ARG;
    if (kd->wmode != SV_W_RAW && kd->wmode != SV_W_GROUP_NORM) return SV_ERR_INVALID_ARG;
    if (kd->wmode == SV_W_GROUP_NORM && (kd->group < 1 || (B > 0 && B % kd->group != 0)))
      return SV_ERR_INVALID_ARG;
    if (!isfinite(kd->clip)) return SV_ERR_INVALID_ARG;
  }
  if (B == 0) return SV_OK;
  sv_status st = check_workspace(workspace, workspace_bytes_, workspace_bytes(B, k + 1));
  if (st != SV_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const Workspace ws = workspace_carve(workspace, B, k + 1);

  if (greedy) {
    RowPlan plan;
    st = make_plan(V, esize(t_dtype), 0, [](int, int) { return 2 * kThreads * 4; },
                   bulk_ok_row(target_logits, V, esize(t_dtype)), &plan);
    if (st != SV_OK) return st;
    if ((long long)B * (k + 1) * plan.C > 0x7fffffffLL) return SV_ERR_UNSUPPORTED;
    ArgmaxParams p = {};
    p.logits = target_logits;
    p.tokens = draft_tokens;
    p.B = B;
    p.R = k + 1;
    p.V = V;
    p.L = plan.L;
    p.use_bulk = plan.use_bulk;
    p.lay = plan.lay;
    p.accepted_len = accepted_len;
    p.out_tokens = out_tokens;
    p.ws = ws;
    p.status = device_status;
    return cuda_status(launch_chain_greedy(p, plan, t_dtype, s));
  }

  const int db = d_kind == SV_DRAFT_PROBS ? 4 : esize(d_dtype);
  const bool with_kd = kd != nullptr;
  RowPlan plan;
  st = make_plan(
      V, esize(t_dtype), db,
      [with_kd](int, int np) {
        int x = np * kThreads * 4 + kThreads * 8;
        if (x < 2 * kThreads * 4) x = 2 * kThreads * 4;
        if (with_kd && x < kCandCap * 8) x = kCandCap * 8;
        return x;
      },
      bulk_ok_row(target_logits, V, esize(t_dtype)) && bulk_ok_row(draft, V, db), &plan);
  if (st != SV_OK) return st;
  if ((long long)B * (k + 1) * plan.C > 0x7fffffffLL) return SV_ERR_UNSUPPORTED;
  ChainParams p = {};
  p.target = target_logits;
  p.draft = draft;
  p.tokens = draft_tokens;
  p.u = uniforms;
  p.B = B;
  p.k = k;
  p.V = V;
  p.L = plan.L;
  p.c = (float)(1.4426950408889634 / (double)temperature);
  p.use_bulk = plan.use_bulk;
  p.lay = plan.lay;
  p.accepted_len = accepted_len;
  p.out_tokens = out_tokens;
  if (kd) {
    p.K = kd->K;
    p.topk_logp = kd->topk_logp;
    p.topk_idx = kd->topk_idx;
    p.lse = kd->lse;
    p.kl = kd->kl;
    p.reward = kd->reward;
    p.wmode = kd->wmode;
    p.group = kd->group < 1 ? 1 : kd->group;
    p.clip = kd->clip;
    p.loss = kd->loss;
    p.total = kd->total;
  }
  p.ws = ws;
  p.status = device_status;
  return cuda_status(launch_chain_sample(p, plan, t_dtype, d_dtype, d_kind, with_kd, s));
}

sv_status sv_verify_tree_greedy(const void* logits, sv_dtype dt, const int32_t* node_tokens,
                                const int32_t* parents, int B, int n, int V, int max_depth,
                                int32_t* accepted_len, int32_t* out_tokens,
                                int32_t* accepted_nodes, void* workspace, size_t workspace_bytes_,
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
  if (B == 0) return SV_OK;
  sv_status st = check_workspace(workspace, workspace_bytes_, workspace_bytes(B, n));
  if (st != SV_OK) return st;
  RowPlan plan;
  st = make_plan(V, esize(dt), 0, [n](int, int) { return 4 * n * 4; },
                 bulk_ok_row(logits, V, esize(dt)), &plan);
  if (st != SV_OK) return st;
  if ((long long)B * n * plan.C > 0x7fffffffLL) return SV_ERR_UNSUPPORTED;
  ArgmaxParams p = {};
  p.logits = logits;
  p.tokens = node_tokens;
  p.parents = parents;
  p.B = B;
  p.R = n;
  p.V = V;
  p.L = plan.L;
  p.max_depth = max_depth;
  p.use_bulk = plan.use_bulk;
  p.lay = plan.lay;
  p.accepted_len = accepted_len;
  p.out_tokens = out_tokens;
  p.accepted_nodes = accepted_nodes;
  p.ws = workspace_carve(workspace, B, n);
  p.status = device_status;
  return cuda_status(launch_tree_greedy(p, plan, dt, reinterpret_cast<cudaStream_t>(stream)));
}

sv_status sv_extract_topk_kd(const void* logits, sv_dtype dt, int rows, int V, int K,
                             float temperature, float* topk_logp, int32_t* topk_idx, float* lse,
                             int32_t* device_status, void* stream) {
  if (rows < 0 || V < 1 || K < 1 || K > kMaxK || K > V) return SV_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !scale_ok(temperature)) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return SV_ERR_INVALID_ARG;
  if (rows == 0) return SV_OK;
  if (!logits || !topk_logp || !topk_idx || !lse) return SV_ERR_INVALID_ARG;
  if (!aligned(logits, esize(dt)) || !aligned(topk_logp, 4) || !aligned(topk_idx, 4) ||
      !aligned(lse, 4))
    return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if (rows == 0) return SV_OK;
  RowPlan plan;
  sv_status st = make_plan(V, esize(dt), 0, [](int, int) { return kCandCap * 8; },
                           bulk_ok_row(logits, V, esize(dt)), &plan);
  if (st != SV_OK) return st;
  if ((long long)rows * plan.C > 0x7fffffffLL) return SV_ERR_UNSUPPORTED;
  TopkParams p = {};
  p.logits = logits;
  p.rows = rows;
  p.V = V;
  p.L = plan.L;
  p.K = K;
  p.c = (float)(1.4426950408889634 / (double)temperature);
  p.use_bulk = plan.use_bulk;
  p.lay = plan.lay;
  p.topk_logp = topk_logp;
  p.topk_idx = topk_idx;
  p.lse = lse;
  p.status = device_status;
  return cuda_status(launch_topk(p, plan, dt, reinterpret_cast<cudaStream_t>(stream)));
}

sv_status sv_kd_kl_loss(const float* topk_logp, const int32_t* topk_idx, int B, int k, int K,
                        const void* draft, sv_dtype d_dtype, sv_draft_kind d_kind, int V,
                        float temperature, const int32_t* accepted_len, const float* reward,
                        sv_weight_mode wmode, int group, float clip, float* kl, float* loss,
                        float* total, void* workspace, size_t workspace_bytes_,
                        int32_t* device_status, void* stream) {
  if (B < 0 || k < 1 || k > 255 || K < 1 || K > kMaxK || V < 1 || K > V) return SV_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !scale_ok(temperature)) return SV_ERR_INVALID_ARG;
  if (d_kind != SV_DRAFT_LOGITS && d_kind != SV_DRAFT_PROBS) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(d_dtype) || (d_kind == SV_DRAFT_PROBS && d_dtype != SV_F32))
    return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!topk_logp || !topk_idx || !draft || !accepted_len || !reward || !kl || !loss || !total)
    return SV_ERR_INVALID_ARG;
  if (!aligned(topk_logp, 4) || !aligned(topk_idx, 4) || !aligned(draft, esize(d_dtype)) ||
      !aligned(accepted_len, 4) || !aligned(reward, 4) || !aligned(kl, 4) || !aligned(loss, 4) ||
      !aligned(total, 4))
    return SV_ERR_INVALID_ARG;
  if (wmode != SV_W_RAW && wmode != SV_W_GROUP_NORM) return SV_ERR_INVALID_ARG;
  if (wmode == SV_W_GROUP_NORM && (group < 1 || (B > 0 && B % group != 0)))
    return SV_ERR_INVALID_ARG;
  if (!isfinite(clip)) return SV_ERR_INVALID_ARG;
  if (device_status && !aligned(device_status, 4)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  sv_status st = check_workspace(workspace, workspace_bytes_, workspace_bytes(B, 0));
  if (st != SV_OK) return st;
  RowPlan plan;
  if (d_kind == SV_DRAFT_PROBS) {
    plan = RowPlan{1, 0, 0, 0, row_layout(kFixedBytes, 0, 0, 0, 0, 0)};
  } else {
    st = make_plan(V, esize(d_dtype), 0, [](int, int) { return 0; },
                   bulk_ok_row(draft, V, esize(d_dtype)), &plan);
    if (st != SV_OK) return st;
  }
  if ((long long)B * k * plan.C > 0x7fffffffLL) return SV_ERR_UNSUPPORTED;
  KlParams p = {};
  p.topk_logp = topk_logp;
  p.topk_idx = topk_idx;
  p.draft = draft;
  p.B = B;
  p.k = k;
  p.K = K;
  p.V = V;
  p.L = plan.L;
  p.c = (float)(1.4426950408889634 / (double)temperature);
  p.use_bulk = plan.use_bulk;
  p.lay = plan.lay;
  p.accepted_len = accepted_len;
  p.reward = reward;
  p.wmode = wmode;
  p.group = group < 1 ? 1 : group;
  p.clip = clip;
  p.kl = kl;
  p.loss = loss;
  p.total = total;
  p.ws = workspace_carve(workspace, B, 0);
  p.status = device_status;
  return cuda_status(
      launch_kl(p, plan, d_dtype, d_kind, reinterpret_cast<cudaStream_t>(stream)));
}

sv_status sv_device_status_check(int32_t w) {
  if (w & SV_DEV_TIMEOUT) return SV_ERR_TIMEOUT;
  if (w & SV_DEV_ERROR_MASK) return SV_ERR_DEVICE_CHECK;
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

int sv_version(void) { return 100; }

}  // extern "C"
