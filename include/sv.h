/*
 * sv.h -- C ABI of libsv: batched speculative-sampling verification on B200.
 *
 * Pages this interface restates (no page gives an API; the operations are
 * theirs, the signatures are this library's):
 *  - "基于推测性解码的强化学习训练" (ReSpec blog), section "推测解码
 *    Speculative Decoding（SD）": the drafter proposes k tokens, the target
 *    runs one forward over prefix + k, target and draft logits are compared,
 *    the first bad token is resampled, else one more token is sampled from the
 *    target.
 *  - "ReSpec: Towards Optimizing Speculative Decoding in Reinforcement
 *    Learning Systems" (reading notes): section 2 (acceptance test min(1, p/q),
 *    residual max(0, p-q) / sum max(0, p-q)); section 3 (EAGLE candidate
 *    trees with depth s, branching t, n nodes); section 4 (top-K = 32 target
 *    log-probs of the V = 151936 row kept for distillation, KD target
 *    KL(softmax(log p) || q)); section 5 (reward weight w(r) = r, normalised
 *    and clipped).
 *  - ReSpec blog, section "奖励加权的适应机制": L_KD = w(r) sum_t KL(p~ || q).
 *
 * Conventions shared by every entry point
 *  - Every array argument is caller-owned DEVICE memory on the current CUDA
 *    device, dense and row-major in the layout given; scalars are host values.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls only enqueue work on it: they never synchronise, never allocate
 *    device memory, and outputs are valid once the stream reaches the call.
 *  - Logits are fp32 or bf16 and must be finite or -inf (no NaN / +inf); every
 *    row needs at least one finite logit.  Temperature T scales target and
 *    draft logits alike (softmax(z / T)); T == 0 selects greedy verification
 *    where the call allows it.
 *  - Ties in argmax and top-K go to the lowest vocabulary index.
 *  - Host-detectable errors (null or misaligned pointers, bad sizes, a
 *    workspace that is too small) return a non-OK status and enqueue nothing.
 *    Data-dependent errors found on the device are OR-ed as SV_DEV_* bits into
 *    the optional `device_status` word (one int32 in device memory, may be
 *    NULL); the caller zeroes it when it wants a fresh reading.  No kernel
 *    traps, asserts or waits without a time limit.
 *  - Workspace: the calls that take one need `*_workspace_size(...)` bytes of
 *    device memory, 16-byte aligned, ZERO-FILLED before its first use (counters
 *    and per-row results that the kernels hand between thread-block clusters).
 *    Every call that runs to completion returns all of it to zero, so one
 *    zeroing suffices for any later sequence of calls, of any entry point and
 *    any size that fits.  One workspace must not be used by two calls that can
 *    run at the same time.
 *  - Results are deterministic: the same inputs on the same device give
 *    bit-identical outputs.
 */
#ifndef SV_H_
#define SV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SV_API __attribute__((visibility("default")))
#else
#define SV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sv_status {
  SV_OK = 0,
  SV_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, size or mode out of range */
  SV_ERR_UNSUPPORTED = 2,  /* valid but beyond the library's limits (e.g. V too large for one row plan) */
  SV_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, attribute, device query) */
  SV_ERR_DEVICE_CHECK = 4, /* returned by sv_device_status_check() for SV_DEV_* error bits */
  SV_ERR_TIMEOUT = 5,      /* returned by sv_device_status_check() for SV_DEV_TIMEOUT */
  SV_ERR_WORKSPACE = 6     /* workspace pointer NULL, misaligned or smaller than required */
} sv_status;

typedef enum sv_dtype { SV_F32 = 0, SV_BF16 = 1 } sv_dtype;

/* The draft distribution is given either as logits (softmax at T) or as
 * fp32 probabilities used as given (not renormalised, T not applied). */
typedef enum sv_draft_kind { SV_DRAFT_LOGITS = 0, SV_DRAFT_PROBS = 1 } sv_draft_kind;

/* Reward weight w_b: RAW w = r_b; GROUP_NORM w = r_b / sum of r over the
 * request's group of `group` consecutive requests (0 when that sum is 0). */
typedef enum sv_weight_mode { SV_W_RAW = 0, SV_W_GROUP_NORM = 1 } sv_weight_mode;

/* Device status bits (OR-ed into *device_status). */
#define SV_DEV_BAD_TOKEN 0x1      /* a draft or node token outside [0, V) */
#define SV_DEV_NO_FINITE 0x2      /* a logit row with no finite value */
#define SV_DEV_TIMEOUT 0x4        /* a bounded wait for a bulk copy gave up */
#define SV_DEV_BAD_TREE 0x8       /* parents[] is not a tree in BFS order, or depth > max_depth */
#define SV_DEV_BAD_INDEX 0x10     /* a top-K index outside [0, V) given to sv_kd_kl_loss */
#define SV_DEV_BAD_LEN 0x20       /* a draft_len outside [0, k] given to sv_verify_chain_ragged */
#define SV_DEV_ERROR_MASK 0xff
#define SV_DEV_RESIDUAL_ZERO 0x100 /* info: a rejection met zero residual mass; the target row was sampled */
#define SV_DEV_TOPK_SLOW 0x200     /* info: massive ties sent a top-K through the slow exact path */

/* KD outputs fused into sv_verify_chain (all device pointers). */
typedef struct sv_kd_args {
  int K;                      /* kept entries per row, 1..32 (32 on the pages) */
  float* topk_logp;           /* [B, k+1, K] out: log p_j = z_j/T - lse, sorted (value desc, index asc) */
  int32_t* topk_idx;          /* [B, k+1, K] out: vocabulary indices of the kept entries */
  float* lse;                 /* [B, k+1]    out: log sum_j exp(z_j / T) of each target row */
  float* kl;                  /* [B, k]      out: KL(p~ || q) of draft row i vs target row i */
  const float* reward;        /* [B]         in:  scalar reward per request */
  sv_weight_mode wmode;       /* reward weighting */
  int group;                  /* GROUP_NORM group size (B % group == 0); ignored for RAW */
  float clip;                 /* > 0: clamp w to [-clip, clip]; <= 0: no clipping */
  float* loss;                /* [B]         out: w_b * sum_{i < m_b} kl[b, i] (0 if w_b == 0) */
  float* total;               /* [1]         out: sum_b loss[b], fixed summation order */
  int positions;              /* the KD positions: 0: m_b = accepted_len[b] (the accepted drafts);
                                 1: also the first rejected position, m_b = n + 1 when n < k (as
                                 drafters that learn from rejected proposals do, "Draft-OPD" page) */
} sv_kd_args;

/* Bytes of zero-filled workspace needed by each call (K = 0: no fused KD).
 * The workspace holds per-row chunk counters, row records and per-chunk
 * partial results of the streaming pass: at most rows * ceil(V / 1024) small records,
 * plus K keys per chunk when top-K lists are kept. */
SV_API size_t sv_verify_chain_workspace_size(int B, int k, int V, int K);
SV_API size_t sv_verify_tree_workspace_size(int B, int n, int V);
SV_API size_t sv_extract_topk_workspace_size(int rows, int V, int K);
SV_API size_t sv_kd_kl_loss_workspace_size(int B, int k, int V);

/*
 * sv_verify_chain -- verify k drafted tokens for each of B requests.
 *
 * Operation (ReSpec blog "推测解码" steps; reading notes section 2):
 *   p_i = softmax(target[b, i, :] / T), q_i = softmax(draft[b, i, :] / T)
 *   (or the given probabilities).  For i = 0..k-1 in order, draft token
 *   x_i = draft_tokens[b, i] is accepted iff uniforms[b, i] * q_i(x_i) <
 *   p_i(x_i) (probability min(1, p/q)).  At the first rejection i* the
 *   emitted token is drawn from max(0, p_i* - q_i*) by inverse CDF in
 *   ascending vocabulary order with uniforms[b, k]; if every draft is
 *   accepted, a bonus token is drawn the same way from p_k.  A zero residual
 *   mass (impossible when x ~ q) samples p_i* and sets SV_DEV_RESIDUAL_ZERO.
 *   T == 0: x_i is accepted iff it equals argmax target[b, i, :]; the argmax
 *   at the first mismatch (or at row k) is emitted; draft and uniforms may be
 *   NULL and kd must be NULL.
 *
 * Arguments
 *   target_logits [B, k+1, V] (t_dtype); row i is the target distribution for
 *                 draft slot i, row k the bonus position.
 *   draft         [B, k, V] logits (d_dtype) or fp32 probabilities (d_kind).
 *   draft_tokens  [B, k] int32 in [0, V).
 *   uniforms      [B, k+1] fp32 in [0, 1): column i < k tests draft i,
 *                 column k drives the single resample-or-bonus draw.
 *   B >= 0 (0 is a no-op), 1 <= k <= 255, 1 <= V <= 524288, T >= 0 finite.
 *   accepted_len  [B] int32 out: n = accepted drafts (0..k); -1 marks a
 *                 request whose inputs failed a device check.
 *   out_tokens    [B, k+1] int32 out: x_0..x_{n-1}, then the resampled or
 *                 bonus token, then -1 padding.
 *   kd            NULL, or the fused KD outputs (T > 0 only), for the rows of
 *                 the emitted sequence: top-K, lse of target rows 0..n and KL
 *                 of draft rows 0..min(n, k-1) against their target rows
 *                 (n = accepted_len[b]); the reward-weighted loss over the
 *                 accepted positions i < n.  Rows after the emitted position
 *                 are not verified (and not read when the rejection is known
 *                 in time): their top-K indices are -1 and their floats NaN.
 *   workspace     sv_verify_chain_workspace_size(B, k, V, kd ? kd->K : 0) bytes.
 *
 * Verification is sequential within a request: a draft after the first
 * rejection is never tested.  Rows are streamed position-major and a row whose
 * request has already rejected at an earlier position is skipped before it is
 * loaded, so the bytes read approach the rows the outcome depends on.  A call
 * is two kernel launches (a streaming pass, then per-request finishing
 * clusters); SV_KNOB_PERSISTENT makes chains of k <= 30 one persistent launch.
 *   device_status optional int32 status word (SV_DEV_* bits).
 */
SV_API sv_status sv_verify_chain(const void* target_logits, sv_dtype t_dtype, const void* draft,
                          sv_dtype d_dtype, sv_draft_kind d_kind, const int32_t* draft_tokens,
                          const float* uniforms, int B, int k, int V, float temperature,
                          int32_t* accepted_len, int32_t* out_tokens, const sv_kd_args* kd,
                          void* workspace, size_t workspace_bytes, int32_t* device_status,
                          void* stream);

/*
 * sv_verify_chain_ragged -- sv_verify_chain for a batch whose requests
 * drafted different numbers of tokens, some of which may be idle.
 *
 * Operation: that of sv_verify_chain with k replaced per request by
 *   k_b = draft_len[b] (0 <= k_b <= k; k itself is the padded length).  The
 *   pages verify each request's own draft chain; a batch that mixes chain
 *   lengths, or that holds finished requests, is padded to one k here, and
 *   the padding is never read.  Request b tests drafts 0..k_b-1 with
 *   uniforms[b, 0..k_b-1], draws the resample or the bonus token with
 *   uniforms[b, k_b], and takes the bonus from target row k_b.  k_b = 0
 *   draws one token from target row 0.  A request with active[b] == 0 is
 *   idle: none of its rows is read, accepted_len = 0 and every out_token is
 *   -1; with kd, its rows are empty and its loss is 0.
 *
 * Arguments: those of sv_verify_chain, plus
 *   draft_len  [B] int32 device, or NULL (k for every request).  A value
 *              outside [0, k] fails that request (accepted_len -1, outputs
 *              -1 / NaN) and sets SV_DEV_BAD_LEN.
 *   active     [B] int32 device, or NULL (every request active).
 *   Row and draft-token entries past k_b (and all entries of an idle request)
 *   are not read and need not be valid.  With kd and positions = 1, the first
 *   rejected position is added when n < k_b.
 *   Layouts, workspace size and errors are those of sv_verify_chain.
 */
SV_API sv_status sv_verify_chain_ragged(const void* target_logits, sv_dtype t_dtype,
                                        const void* draft, sv_dtype d_dtype,
                                        sv_draft_kind d_kind, const int32_t* draft_tokens,
                                        const float* uniforms, const int32_t* draft_len,
                                        const int32_t* active, int B, int k, int V,
                                        float temperature, int32_t* accepted_len,
                                        int32_t* out_tokens, const sv_kd_args* kd,
                                        void* workspace, size_t workspace_bytes,
                                        int32_t* device_status, void* stream);

/*
 * sv_verify_chain_noalloc -- sv_verify_chain without a caller-supplied
 * workspace.  The pages have no counterpart: this is a convenience of this
 * library for callers that cannot allocate device memory around a call, such
 * as host code running under another framework's allocator, or a plugin
 * interface that hands over only input and output pointers, so that they
 * cannot own a workspace buffer.
 *
 *   Arguments, results and errors are those of sv_verify_chain, and the
 *   argument checks run first, so a bad argument returns the same code.
 *   The scratch is a fixed array of SV_NOALLOC_MAX_BYTES per device inside
 *   libsv.  Every call looks up the array's device address in the calling
 *   thread's current context (a host-side lookup); the first call on a device
 *   also loads the library's device code there, so make it before any stream
 *   capture.
 *   A call whose sv_verify_chain_workspace_size(B, k, V, kd ? kd->K : 0)
 *   exceeds SV_NOALLOC_MAX_BYTES returns SV_ERR_WORKSPACE and launches
 *   nothing.  At V = 151936 (k = 3) that allows about B*(k+1) <= 580 target
 *   rows without KD and about 90 with K = 32 on the default path; about 1450
 *   and 520 with SV_KNOB_PERSISTENT set.
 *   The array starts zero-filled and every completed call returns it to zero,
 *   including calls whose requests fail a device check; a call that returns
 *   SV_ERR_CUDA after a partial launch clears it with an asynchronous memset
 *   on `stream`.  All calls on a device share the one array: calls that can
 *   run at the same time (on different streams, or from host threads without
 *   mutual ordering) race on it and must be ordered by the caller.
 */
#define SV_NOALLOC_MAX_BYTES (4u << 20)
SV_API sv_status sv_verify_chain_noalloc(const void* target_logits, sv_dtype t_dtype,
                                         const void* draft, sv_dtype d_dtype,
                                         sv_draft_kind d_kind, const int32_t* draft_tokens,
                                         const float* uniforms, int B, int k, int V,
                                         float temperature, int32_t* accepted_len,
                                         int32_t* out_tokens, const sv_kd_args* kd,
                                         int32_t* device_status, void* stream);

/*
 * sv_verify_tree_greedy -- greedy (T = 0) verification of B candidate trees
 * (reading notes section 3: EAGLE trees of depth s, top-t branching, n nodes).
 *
 *   logits      [B, n, V] (dt): row j is the target distribution after node j.
 *   node_tokens [B, n] int32: token of node j (node 0, the root, is unused).
 *   parents     [B, n] int32: parents[b, 0] = -1, 0 <= parents[b, j] < j.
 *   Node j >= 1 is accepted iff its parent is accepted and node_tokens[j] ==
 *   argmax logits[b, parents[j], :]; the root is always accepted.  The deepest
 *   accepted node wins (lowest index among equals); its depth d is
 *   accepted_len[b] (depth must never exceed max_depth).
 *   accepted_nodes [B, max_depth+1] out: the path root..best, then -1.
 *   out_tokens     [B, max_depth+1] out: the path's tokens (root excluded),
 *                  then argmax logits[b, best, :], then -1.
 *   1 <= n <= 1024, 0 <= max_depth < n, 1 <= V <= 524288.
 *   Invalid parents, depths or tokens set SV_DEV_BAD_TREE / SV_DEV_BAD_TOKEN
 *   and accepted_len[b] = -1.
 */
SV_API sv_status sv_verify_tree_greedy(const void* logits, sv_dtype dt, const int32_t* node_tokens,
                                const int32_t* parents, int B, int n, int V, int max_depth,
                                int32_t* accepted_len, int32_t* out_tokens,
                                int32_t* accepted_nodes, void* workspace, size_t workspace_bytes,
                                int32_t* device_status, void* stream);

/*
 * sv_verify_tree_sample -- sampling (T > 0) verification of B candidate
 * trees.  The reading notes (section 3) name the EAGLE trees but no sampling
 * rule; the rule is the multi-step speculative sampling of SpecInfer (Miao et
 * al., "SpecInfer: Accelerating Large Language Model Serving with Tree-based
 * Speculative Inference and Verification"), the recursive rejection sampling
 * EAGLE adopts.
 *
 * Operation: from the root, at node v (p_v = softmax(target[b, v, :] / T),
 *   q_v = softmax(draft[b, v, :] / T) or the given probabilities), r = p_v;
 *   the children of v are tried in ascending node order: child c with token
 *   x is accepted iff uniforms[b, c] * q_v(x) < r(x) (probability
 *   min(1, r(x)/q_v(x))), and the walk moves to c; otherwise r becomes
 *   max(0, r - q_v) normalised and the next child is tried.  A node with no
 *   accepted child (or none at all) draws one token from r by inverse CDF in
 *   ascending vocabulary order with uniforms[b, 0].  A zero residual mass
 *   (probability zero when children are drawn from q_v) draws from p_v and
 *   sets SV_DEV_RESIDUAL_ZERO.  The emitted tokens follow the target's
 *   distribution when the children of every node are drawn independently
 *   from its draft row.
 *
 * Arguments
 *   target_logits [B, n, V] (t_dtype): row j is the target distribution after
 *                 node j.
 *   draft         [B, n, V]: row j is the draft distribution node j's children
 *                 were drawn from: logits (d_dtype), or fp32 probabilities.
 *                 Rows of leaves are read only when the walk reaches them.
 *   node_tokens, parents, max_depth as in sv_verify_tree_greedy.
 *   uniforms      [B, n] fp32 in [0, 1): column j >= 1 tests node j, column 0
 *                 drives the final draw.
 *   T > 0.  1 <= n <= 1024, 0 <= max_depth < n, 1 <= V <= 524288.
 *   accepted_len, accepted_nodes, out_tokens as in sv_verify_tree_greedy
 *   (the token after the path is the drawn one).  Invalid trees or tokens set
 *   SV_DEV_BAD_TREE / SV_DEV_BAD_TOKEN, a row without a finite value
 *   SV_DEV_NO_FINITE; the request then has accepted_len -1 and -1 outputs.
 *   No workspace: each request's rows are read by one thread-block cluster,
 *   and only the rows of the nodes the walk visits.
 */
SV_API sv_status sv_verify_tree_sample(const void* target_logits, sv_dtype t_dtype,
                                       const void* draft, sv_dtype d_dtype,
                                       sv_draft_kind d_kind, const int32_t* node_tokens,
                                       const int32_t* parents, const float* uniforms, int B,
                                       int n, int V, int max_depth, float temperature,
                                       int32_t* accepted_len, int32_t* out_tokens,
                                       int32_t* accepted_nodes, int32_t* device_status,
                                       void* stream);

/*
 * sv_extract_topk_kd -- the distillation buffer of the reading notes,
 * section 4: for each of `rows` rows of V logits, the K largest logits
 * (value desc, index asc) as full-vocabulary log-probs at temperature T.
 *   logits [rows, V] (dt); topk_logp [rows, K] fp32 out; topk_idx [rows, K]
 *   int32 out; lse [rows] fp32 out (log sum_j exp(z_j / T)).
 *   1 <= K <= min(32, V), T > 0.  A [B, k+1, V] target is rows = B*(k+1).
 *   workspace: sv_extract_topk_workspace_size(rows, V, K) bytes.
 */
SV_API sv_status sv_extract_topk_kd(const void* logits, sv_dtype dt, int rows, int V, int K,
                                    float temperature, float* topk_logp, int32_t* topk_idx,
                                    float* lse, void* workspace, size_t workspace_bytes,
                                    int32_t* device_status, void* stream);

/*
 * sv_kd_kl_loss -- reward-weighted KD loss (ReSpec blog "奖励加权的适应机制";
 * reading notes sections 4-5).
 *   topk_logp, topk_idx [B, k+1, K] as produced by sv_extract_topk_kd on the
 *   [B, k+1, V] target; draft [B, k, V] logits (d_dtype) or fp32 probs.
 *   For each draft row (b, i < k): p~ = softmax of topk_logp[b, i, :] (the
 *   renormalised kept target mass), log q_j = log softmax(draft[b, i] / T)_j
 *   (or log of the given probability) at j = topk_idx[b, i, :],
 *   kl[b, i] = sum_j p~_j (log p~_j - log q_j) (+inf when q_j = 0 < p~_j).
 *   loss[b] = w_b * sum_{i < m_b} kl[b, i] (0 when w_b == 0), m_b as in
 *   sv_kd_args.positions (accepted_len[b], or one more at a rejection),
 *   total[0] = sum_b loss[b]; w_b as in sv_weight_mode, optionally clipped.
 *   accepted_len [B] int32 in [0, k]; reward [B] fp32; T > 0.
 */
SV_API sv_status sv_kd_kl_loss(const float* topk_logp, const int32_t* topk_idx, int B, int k, int K,
                        const void* draft, sv_dtype d_dtype, sv_draft_kind d_kind, int V,
                        float temperature, const int32_t* accepted_len, const float* reward,
                        sv_weight_mode wmode, int group, float clip, int positions, float* kl,
                        float* loss, float* total, void* workspace, size_t workspace_bytes,
                        int32_t* device_status, void* stream);

/*
 * sv_kd_grad -- gradient of the reward-weighted KD loss with respect to the
 * draft logits, the drafter update of the reading notes, section 4 (Algorithm
 * 1 step 3: the gradient flows into the current q_theta only) with the reward
 * weights of section 5.  With q = softmax(draft[b, i] / T) and p~ as in
 * sv_kd_kl_loss:
 *   grad[b, i, j] = w_b * (q_j - p~_j [j in topk_idx[b, i, :]]) / T  for i < m_b,
 *   grad[b, i, j] = 0                                                 otherwise,
 * which is d loss[b] / d draft[b, i, j] for the loss of sv_kd_kl_loss with
 * the same `positions` (m_b as in sv_kd_args).
 *   topk_logp, topk_idx [B, k+1, K]; draft [B, k, V] logits (d_dtype);
 *   accepted_len [B]; reward [B]; grad [B, k, V] fp32 out.  T > 0.
 *   A row whose statistics fail (no finite logit) or whose top-K indices are
 *   out of range is set to NaN, with the matching SV_DEV_* bit.
 *   workspace: sv_kd_grad_workspace_size(B, k, V) bytes.
 */
SV_API size_t sv_kd_grad_workspace_size(int B, int k, int V);
SV_API sv_status sv_kd_grad(const float* topk_logp, const int32_t* topk_idx, int B, int k, int K,
                            const void* draft, sv_dtype d_dtype, int V, float temperature,
                            const int32_t* accepted_len, const float* reward,
                            sv_weight_mode wmode, int group, float clip, int positions, float* grad,
                            void* workspace, size_t workspace_bytes, int32_t* device_status,
                            void* stream);

/*
 * sv_set_knob -- process-wide test and tuning settings (not needed for
 * normal use; the pages have no counterpart).  Every knob defaults to 0, the
 * library's own choice, and a value set applies to every later call from any
 * thread until it is set again.  Returns SV_ERR_INVALID_ARG for an unknown
 * knob; values outside a knob's range select the default.
 *   SV_KNOB_CLUSTER_CTAS  finishing cluster size of the two-kernel paths, 1..16
 *   SV_KNOB_STREAM_COUNT  two-kernel streaming pass: 1 static partition,
 *                         2 dynamic items with in-stream row completion
 *   SV_KNOB_STREAM_W      two-kernel streaming chunk, a multiple of 1024 entries
 *   SV_KNOB_WAIT_NS       time limit of every bounded wait of the chain kernel,
 *                         in ns (default 1 s); a wait that runs out sets
 *                         SV_DEV_TIMEOUT
 *   SV_KNOB_STALL         1: the chain kernel's warp that reduces the first
 *                         slice of request 0's first row waits on a barrier
 *                         nothing arrives on, for a quarter of the wait limit,
 *                         so that the wait runs out (a test of the timeout
 *                         path: request 0 fails with SV_DEV_TIMEOUT, everything
 *                         else completes)
 *   SV_KNOB_STAGES        chain kernel ring stages per CTA, 2..8
 *   SV_KNOB_ORDER         chain kernel tile order: 1 the tiles of a row
 *                         consecutive, 2 the requests innermost
 *   SV_KNOB_PERSISTENT    1: chain calls with k <= 30 run as one persistent
 *                         launch (streaming, early exit, residual and bonus
 *                         draws and request completion in one grid); 0, the
 *                         default, the two-kernel path (stream pass, then
 *                         finishing clusters), which is faster on B200 today
 *   SV_KNOB_KERNEL_MARKS  1: bracket every kernel launch with events (see
 *                         sv_kernel_times)
 *   SV_KNOB_FINISH_READ   two-kernel sampling chain, how the finishing clusters
 *                         read the drawn row: 1 staged in shared memory, 2 read
 *                         from global memory (default: staged when every
 *                         cluster fits in one wave)
 */
#define SV_KNOB_CLUSTER_CTAS 1
#define SV_KNOB_STREAM_COUNT 2
#define SV_KNOB_STREAM_W 3
#define SV_KNOB_WAIT_NS 4
#define SV_KNOB_STALL 5
#define SV_KNOB_STAGES 6
#define SV_KNOB_ORDER 7
#define SV_KNOB_PERSISTENT 8
#define SV_KNOB_KERNEL_MARKS 9
#define SV_KNOB_FINISH_READ 10
SV_API sv_status sv_set_knob(int knob, long long value);

/*
 * sv_kernel_times -- per-launch device times, for measurement.  While
 * SV_KNOB_KERNEL_MARKS is 1, the library records an event on the call's stream
 * before and after each kernel it launches (also inside stream capture, where
 * the events become graph nodes and are recorded at every replay); the events
 * are the library's own, created on the current device at the first marked
 * launch.  This call waits for the last marked launch, writes the duration in
 * microseconds of each launch marked since its previous call (at most the
 * last 2048, oldest first, at most `cap`) to us[] and its kind to tags[]
 * (SV_MARK_STREAM: a streaming pass; SV_MARK_FINISH: a finishing or
 * reduction kernel; SV_MARK_CHAIN: the persistent chain kernel), stores the
 * count in *n and starts a new count.  The marks add an event record between
 * launches, so a marked call can run slightly slower than an unmarked one.
 *   Errors: SV_ERR_INVALID_ARG for null pointers or a current device other
 *   than the marks' own; SV_ERR_CUDA if reading an event fails.
 */
#define SV_MARK_STREAM 0
#define SV_MARK_FINISH 1
#define SV_MARK_CHAIN 2
SV_API sv_status sv_kernel_times(float* us, int32_t* tags, int cap, int32_t* n);

/* Map a device status word (read back by the caller) to a host status:
 * SV_OK, SV_ERR_TIMEOUT if SV_DEV_TIMEOUT is set, else SV_ERR_DEVICE_CHECK
 * if any other error bit is set.  Informational bits are ignored. */
SV_API sv_status sv_device_status_check(int32_t device_status_word);

/* Static description of a status code. */
/*
 * sv_sched_select -- the runtime half of the adaptive speculative decoding
 * scheduler (reading notes, section 3 "G1 解法: Adaptive Speculative Decoding
 * Server": an offline solver profiles throughput over configurations x batch
 * sizes; at each decoding step the scheduler looks up the best configuration
 * for the current active batch and falls back to plain target decoding when
 * the predicted speedup is below 1).  Host code: no device memory, no stream.
 *
 * Arguments (all host memory, caller-owned):
 *   throughput  [n_cfg, n_batch] fp32: profiled throughput (tokens/s or any
 *               unit where higher is better) of configuration c at batch
 *               size batches[j]; finite, >= 0, and > 0 in row `nonspec`.
 *   batches     [n_batch] int32, strictly ascending, >= 1.
 *   nonspec     the row of plain (non-speculative) target decoding.
 *   active_batch >= 1: the current number of active requests.
 *   config      out: the configuration to run.
 *   predicted_speedup  out (may be NULL): the best speculative configuration's
 *               predicted throughput over plain decoding's at active_batch
 *               (the value compared with 1; 0 when n_cfg == 1).
 * Lookup model: each row is interpolated linearly in the batch size between
 * the two profiled sizes around active_batch, and held constant outside the
 * profiled range.  The best speculative row is the largest interpolated
 * throughput (lowest index on ties); it is chosen unless its speedup is
 * below 1.  Invalid arguments return SV_ERR_INVALID_ARG.
 */
SV_API sv_status sv_sched_select(const float* throughput, const int32_t* batches, int n_cfg,
                                 int n_batch, int nonspec, int active_batch, int32_t* config,
                                 float* predicted_speedup);

SV_API const char* sv_status_string(sv_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
SV_API int sv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SV_H_ */
