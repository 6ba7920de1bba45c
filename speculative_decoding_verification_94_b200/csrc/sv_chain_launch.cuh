// sv_chain_launch.cuh -- host side of the persistent chain kernel: workspace
// layout, shared-memory plan and launch.  Included by one source file per
// target dtype (the kernel's instantiations compile in parallel).
#pragma once

#include "sv_chain.cuh"
#include "sv_internal.h"

namespace sv {

enum : int { kKnobWaitNs = 4, kKnobStall = 5, kKnobStages = 6, kKnobOrder = 7 };

struct ChainWs {
  size_t glob, req_state, pair_cnt, job_cnt, drawq, rowthr, rows, tiles, bonus, jobs, draws, cand,
      st_logp, st_idx, st_lse, st_kl, bytes;
};

// Workspace of one call: counters and per-request/per-row state first (zero
// between calls), then records that every call writes before it reads them.
inline ChainWs chain_ws_layout(int B, int k, int V, int K) {
  auto al = [](size_t x) { return (x + 15) / 16 * 16; };
  const size_t P = (size_t)k + 1, NT = ((size_t)V + kTileW - 1) / kTileW, Bs = (size_t)B;
  ChainWs w;
  size_t o = 0;
  w.glob = o;
  o += 256;
  w.req_state = o;
  o = al(o + 8 * Bs);
  w.pair_cnt = o;
  o = al(o + 4 * Bs * P);
  w.job_cnt = o;
  o = al(o + 4 * Bs);
  w.drawq = o;
  o = al(o + 4 * Bs * NT);
  w.rowthr = o;
  o = al(o + (K > 0 ? 8 * Bs * P : 0));
  w.rows = o;
  o += sizeof(RowRec) * Bs * P;
  w.tiles = o;
  o += sizeof(TileRec) * Bs * P * NT;
  w.bonus = o;
  o += sizeof(WarpStat) * Bs * NT * kCW;
  w.jobs = o;
  o += sizeof(DrawJob) * Bs;
  w.draws = o;
  o += sizeof(DrawRec) * Bs * NT;
  w.cand = o;
  o += (K > 0 ? 8 * Bs * P * NT * (size_t)K : 0);
  w.st_logp = o;
  o = al(o + (K > 0 ? 4 * Bs * P * (size_t)K : 0));
  w.st_idx = o;
  o = al(o + (K > 0 ? 4 * Bs * P * (size_t)K : 0));
  w.st_lse = o;
  o = al(o + (K > 0 ? 4 * Bs * P : 0));
  w.st_kl = o;
  o = al(o + (K > 0 ? 4 * Bs * (size_t)k : 0));
  w.bytes = (o + 255) / 256 * 256;
  return w;
}

template <class TT, class DT, int MODE, bool KD>
cudaError_t launch_chain_t(const ChainArgs& a) {
  const int te = TT::bytes;
  const int de = MODE == kCMGreedy ? 0 : (MODE == kCMProbs ? 4 : DT::bytes);
  const int K = KD ? a.kd->K : 0;
  const ChainWs w = chain_ws_layout(a.B, a.k, a.V, K);
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  ChainParams p = {};
  p.target = a.target;
  p.draft = a.draft;
  p.tokens = a.tokens;
  p.u = a.u;
  p.klen = a.klen;
  p.active = a.active;
  p.B = a.B;
  p.k = a.k;
  p.V = a.V;
  p.P = a.k + 1;
  p.NT = (a.V + kTileW - 1) / kTileW;
  p.total = p.P * a.B * p.NT;
  const long long ko = knob(kKnobOrder);
  p.order = ko == 1 ? 0 : ko == 2 ? 1 : (KD ? 1 : 0);
  p.div_NT = make_fastdiv(p.NT);
  p.div_B = make_fastdiv(a.B);
  p.c = MODE == kCMGreedy ? 0.f : (float)(1.4426950408889634 / (double)a.temperature);
  auto row_ok = [](const void* base, int V, int es) {
    return base != nullptr && (reinterpret_cast<uintptr_t>(base) % 16) == 0 &&
           ((size_t)V * es) % 16 == 0;
  };
  p.use_bulk = row_ok(a.target, a.V, te) && (MODE == kCMGreedy || row_ok(a.draft, a.V, de));
  // shared memory: stages, then barriers, descriptors, counters, partials, lists
  const int stage_off1 = (kTileW * te + 127) / 128 * 128;
  const int stage_bytes = stage_off1 + (kTileW * de + 127) / 128 * 128;
  auto fixed_bytes = [&](int S) {
    int f = (2 * kMaxStagesC + 1) * 8;
    f = (f + 15) / 16 * 16 + S * (int)sizeof(StageDesc);
    f = (f + 15) / 16 * 16 + S * 4;
    f = (f + 15) / 16 * 16 + S * kCW * (int)sizeof(WarpPart);
    f = (f + 15) / 16 * 16 + (KD ? S * kCW * K * 8 : 0);
    f = (f + 15) / 16 * 16 + 2 * (int)sizeof(TaskQueue);
    return f;
  };
  int S = (int)knob(kKnobStages);
  if (S < 2 || S > kMaxStagesC) {
    S = (160 * 1024) / stage_bytes;
    S = S < 2 ? 2 : (S > 5 ? 5 : S);
  }
  while (S > 2 && S * stage_bytes + fixed_bytes(S) > 220 * 1024) --S;
  p.stages = S;
  p.stage_bytes = stage_bytes;
  p.stage_off1 = stage_off1;
  int o = S * stage_bytes;
  p.off_bars = o;
  o = (o + (2 * kMaxStagesC + 1) * 8 + 15) / 16 * 16;
  p.off_desc = o;
  o = (o + S * (int)sizeof(StageDesc) + 15) / 16 * 16;
  p.off_done = o;
  o = (o + S * 4 + 15) / 16 * 16;
  p.off_parts = o;
  o = (o + S * kCW * (int)sizeof(WarpPart) + 15) / 16 * 16;
  p.off_lists = o;
  o = (o + (KD ? S * kCW * K * 8 : 0) + 15) / 16 * 16;
  p.off_tasks = o;
  o += 2 * (int)sizeof(TaskQueue);
  const int smem = o;
  p.K = K > 0 ? K : 1;
  p.accepted_len = a.accepted_len;
  p.out_tokens = a.out_tokens;
  if (KD) {
    p.topk_logp = a.kd->topk_logp;
    p.topk_idx = a.kd->topk_idx;
    p.lse = a.kd->lse;
    p.kl = a.kd->kl;
    p.reward = a.kd->reward;
    p.wmode = a.kd->wmode;
    p.group = a.kd->group < 1 ? 1 : a.kd->group;
    p.clip = a.kd->clip;
    p.loss = a.kd->loss;
    p.total_out = a.kd->total;
    p.positions = a.kd->positions ? 1 : 0;
  }
  p.status = a.status;
  p.glob = reinterpret_cast<uint32_t*>(ws + w.glob);
  p.req_state = reinterpret_cast<unsigned long long*>(ws + w.req_state);
  p.pair_cnt = reinterpret_cast<uint32_t*>(ws + w.pair_cnt);
  p.rows = reinterpret_cast<RowRec*>(ws + w.rows);
  p.tiles = reinterpret_cast<TileRec*>(ws + w.tiles);
  p.bonus = reinterpret_cast<WarpStat*>(ws + w.bonus);
  p.jobs = reinterpret_cast<DrawJob*>(ws + w.jobs);
  p.job_cnt = reinterpret_cast<uint32_t*>(ws + w.job_cnt);
  p.drawq = reinterpret_cast<uint32_t*>(ws + w.drawq);
  p.draws = reinterpret_cast<DrawRec*>(ws + w.draws);
  p.cand = reinterpret_cast<unsigned long long*>(ws + w.cand);
  p.rowthr = reinterpret_cast<unsigned long long*>(ws + w.rowthr);
  p.st_logp = reinterpret_cast<float*>(ws + w.st_logp);
  p.st_idx = reinterpret_cast<int32_t*>(ws + w.st_idx);
  p.st_lse = reinterpret_cast<float*>(ws + w.st_lse);
  p.st_kl = reinterpret_cast<float*>(ws + w.st_kl);
  const long long wn = knob(kKnobWaitNs);
  p.wait_ns = wn > 0 ? (unsigned long long)wn : 1000000000ull;
  p.stall = knob(kKnobStall) ? 1 : 0;
  p.ws_base = ws;
  p.ws_bytes = w.bytes;

  auto kern = chain_kernel<TT, DT, MODE, KD>;
  cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(kern), smem, false);
  if (e != cudaSuccess) return e;
  int sms = 0;
  if ((e = sm_count(&sms)) != cudaSuccess) return e;
  const int grid = p.total < sms ? (p.total < 1 ? 1 : p.total) : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kChainThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  // the launch may overlap the previous kernel's tail; the kernel waits for
  // it (griddepcontrol.wait) before it touches global memory
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// Every mode of one target dtype.
template <class TT>
cudaError_t launch_chain_dtype(const ChainArgs& a) {
  const bool kd = a.kd != nullptr;
  if (a.temperature == 0.f) return launch_chain_t<TT, TT, kCMGreedy, false>(a);
  if (a.d_kind == SV_DRAFT_PROBS)
    return kd ? launch_chain_t<TT, F32, kCMProbs, true>(a) : launch_chain_t<TT, F32, kCMProbs, false>(a);
  if (a.d_dtype == SV_BF16)
    return kd ? launch_chain_t<TT, BF16, kCMSample, true>(a)
              : launch_chain_t<TT, BF16, kCMSample, false>(a);
  return kd ? launch_chain_t<TT, F32, kCMSample, true>(a) : launch_chain_t<TT, F32, kCMSample, false>(a);
}

}  // namespace sv
