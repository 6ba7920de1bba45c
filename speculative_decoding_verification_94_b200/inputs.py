"""Seeded synthetic inputs for speculative-sampling verification.

This module holds random-number generation and dtype casting only: no
softmax, acceptance test, sampling rule or loss.  Both the CUDA path's tests
and benchmark and the oracle's tests draw their inputs from here, so that the
two sides see identical bytes.

Generator: numpy ``Generator(Philox)``.  Every target/draft row r has its own
stream ``Philox(SeedSequence([seed, 1, r]))``, drawn in the fixed order
target noise -> draft noise -> vocabulary permutation -> Gumbel uniforms for
the draft token; the batch-level stream ``Philox(SeedSequence([seed, 0]))``
then draws the verification uniforms and the rewards.

Logit models (the workloads of the configs; sizes follow the pages: Qwen2.5
vocabulary V=151936, k=3 draft tokens, GRPO groups of 16, (s,t,n) = (5,8,32)):
  * ``"gauss"``: z_t ~ N(0, sigma_t^2) (fp32 tiny case);
  * ``"zipf"``:  z_t = sigma_t * N(0,1) - s * ln(1 + pi(j)), pi a random
    permutation of the vocabulary per row (a Zipf(s) log-prior);
  * draft logits z_d = z_t + N(0, sigma_d^2), both rounded once to the storage
    dtype (bf16 round-to-nearest-even via torch).
Draft tokens are drawn from the draft distribution by the Gumbel-max trick on
the stored draft logits, x = argmax_j (z_d,j / T + G_j) (x = argmax z_d when
T = 0), which needs no normalisation.  Uniforms are 24-bit:
u = (32-bit draw >> 8) * 2^-24, exactly representable in fp32, in [0, 1).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

V_QWEN = 151936


def _row_rng(seed: int, r: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, 1, r])))


def _batch_rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, 0])))


def uniforms24(rng: np.random.Generator, shape) -> np.ndarray:
    draws = rng.integers(0, 2**32, size=shape, dtype=np.uint64).astype(np.uint32)
    return ((draws >> np.uint32(8)).astype(np.float64) * 2.0**-24).astype(np.float32)


def _cast(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def _gumbel_argmax(z: np.ndarray, T: float, rng: np.random.Generator) -> int:
    if T == 0.0:
        return int(np.argmax(z))
    g = -np.log(-np.log(rng.random(z.shape[0]) * (1 - 2.0**-53) + 2.0**-54))
    return int(np.argmax(z.astype(np.float64) / T + g))


@dataclass
class ChainInputs:
    target: torch.Tensor        # [B, k+1, V] bf16 / fp32 logits
    draft: torch.Tensor         # [B, k, V] logits (or fp32 probabilities)
    draft_tokens: torch.Tensor  # [B, k] int32
    uniforms: torch.Tensor      # [B, k+1] fp32 in [0, 1)
    reward: torch.Tensor        # [B] fp32
    temperature: float
    draft_kind: str = "logits"
    meta: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.target.shape[0]

    @property
    def k(self):
        return self.target.shape[1] - 1

    @property
    def V(self):
        return self.target.shape[2]


def make_chain(B: int, k: int, V: int, *, dtype: str = "bf16", model: str = "zipf",
               sigma_t: float = 3.0, sigma_d: float = 1.0, zipf_s: float = 1.1,
               temperature: float = 0.7, seed: int = 0) -> ChainInputs:
    """Target/draft logits, Gumbel-drawn draft tokens, uniforms and rewards."""
    P = k + 1
    tgt = np.empty((B, P, V), np.float32)
    dft = np.empty((B, k, V), np.float32)
    tokens = np.empty((B, k), np.int32)
    T = float(np.float32(temperature))
    for b in range(B):
        for i in range(P):
            rng = _row_rng(seed, b * P + i)
            noise_t = rng.standard_normal(V, dtype=np.float32)
            noise_d = rng.standard_normal(V, dtype=np.float32) if i < k else None
            if model == "zipf":
                perm = rng.permutation(V)
                prior = (-zipf_s * np.log1p(perm.astype(np.float64))).astype(np.float32)
                zt = np.float32(sigma_t) * noise_t + prior
            elif model == "gauss":
                zt = np.float32(sigma_t) * noise_t
            else:
                raise ValueError(model)
            tgt[b, i] = zt
            if i < k:
                dft[b, i] = zt + np.float32(sigma_d) * noise_d
                stored = _cast(dft[b, i], dtype).float().numpy()
                tokens[b, i] = _gumbel_argmax(stored, T, rng)
    tgt_t = _cast(tgt, dtype)
    dft_t = _cast(dft, dtype)
    brng = _batch_rng(seed)
    u = uniforms24(brng, (B, P))
    reward = brng.random(B).astype(np.float32)
    return ChainInputs(tgt_t, dft_t, torch.from_numpy(tokens), torch.from_numpy(u),
                       torch.from_numpy(reward), T,
                       meta=dict(B=B, k=k, V=V, dtype=dtype, model=model, sigma_t=sigma_t,
                                 sigma_d=sigma_d, zipf_s=zipf_s, seed=seed))


def make_chain_fixed(B: int, target_logits: np.ndarray, draft: np.ndarray, *,
                     draft_kind: str = "probs", temperature: float = 1.0, seed: int = 0,
                     dtype: str = "f32") -> ChainInputs:
    """The same target logits [k+1, V] and draft rows [k, V] (fp32
    probabilities, or logits in ``dtype``) for all B requests; per request,
    independent draft tokens x_i ~ q_i (Gumbel-max on log q, or on z_d / T)
    and fresh uniforms.  Used by the Monte-Carlo tests of the acceptance rule."""
    target_logits = np.asarray(target_logits, np.float32)
    P, V = target_logits.shape
    k = P - 1
    T = float(np.float32(temperature))
    tgt = _cast(target_logits, dtype)
    if draft_kind == "probs":
        dft = torch.from_numpy(np.ascontiguousarray(np.asarray(draft, np.float32)))
        score = np.log(dft.double().numpy())
    else:
        dft = _cast(np.asarray(draft, np.float32), dtype)
        score = dft.double().numpy() / T
    brng = _batch_rng(seed)
    g = -np.log(-np.log(brng.random((B, k, V)) * (1 - 2.0**-53) + 2.0**-54))
    tokens = np.argmax(score[None] + g, axis=-1).astype(np.int32)
    u = uniforms24(brng, (B, P))
    return ChainInputs(tgt.unsqueeze(0).expand(B, P, V).contiguous(),
                       dft.unsqueeze(0).expand(B, k, V).contiguous(), torch.from_numpy(tokens),
                       torch.from_numpy(u), torch.zeros(B), T, draft_kind=draft_kind,
                       meta=dict(B=B, k=k, V=V, seed=seed))


@dataclass
class TreeInputs:
    logits: torch.Tensor       # [B, n, V]
    node_tokens: torch.Tensor  # [B, n] int32 (root token unused)
    parents: torch.Tensor      # [B, n] int32, parents[:, 0] = -1
    max_depth: int
    meta: dict = field(default_factory=dict)


def _tree_shape(brng: np.random.Generator, par: np.ndarray, depth_counts, branching: int):
    """Fill par (BFS order: depth d holds depth_counts[d-1] nodes, each with a
    parent drawn among the previous depth's nodes that have fewer than
    ``branching`` children); return {parent: [children ascending]}."""
    prev = [0]
    nxt = 1
    for cnt in depth_counts:
        kids = {p: 0 for p in prev}
        level = []
        for _ in range(cnt):
            choices = [p for p in prev if kids[p] < branching]
            p = int(choices[brng.integers(len(choices))])
            kids[p] += 1
            par[nxt] = p
            level.append(nxt)
            nxt += 1
        prev = level
    children: dict[int, list[int]] = {}
    for j in range(1, len(par)):
        children.setdefault(int(par[j]), []).append(j)
    return children


@dataclass
class TreeSampleInputs:
    target: torch.Tensor       # [B, n, V] logits
    draft: torch.Tensor        # [B, n, V] logits (or fp32 probabilities)
    node_tokens: torch.Tensor  # [B, n] int32 (root token unused)
    parents: torch.Tensor      # [B, n] int32, parents[:, 0] = -1
    uniforms: torch.Tensor     # [B, n] fp32: column j >= 1 tests node j, column 0 the draw
    temperature: float
    max_depth: int
    draft_kind: str = "logits"
    meta: dict = field(default_factory=dict)


def make_tree_sample(B: int = 8, V: int = V_QWEN, *, depth_counts=(8, 8, 8, 4, 3),
                     branching: int = 8, dtype: str = "bf16", model: str = "zipf",
                     sigma_t: float = 3.0, sigma_d: float = 1.0, zipf_s: float = 1.1,
                     temperature: float = 0.7, seed: int = 0) -> TreeSampleInputs:
    """Candidate trees (shapes as make_tree) for sampling verification: target
    rows as make_chain's, draft logit rows z_t + sigma_d * N(0, 1), and the
    children of every node drawn independently (with replacement) from the
    stored draft row of their parent at temperature T, by Gumbel-max."""
    n = 1 + sum(depth_counts)
    T = float(np.float32(temperature))
    tgt = np.empty((B, n, V), np.float32)
    dft = np.empty((B, n, V), np.float32)
    tok = np.zeros((B, n), np.int32)
    par = np.full((B, n), -1, np.int32)
    brng = _batch_rng(seed)
    for b in range(B):
        children = _tree_shape(brng, par[b], depth_counts, branching)
        for j in range(n):
            rng = _row_rng(seed, b * n + j)
            noise_t = rng.standard_normal(V, dtype=np.float32)
            noise_d = rng.standard_normal(V, dtype=np.float32)
            if model == "zipf":
                perm = rng.permutation(V)
                prior = (-zipf_s * np.log1p(perm.astype(np.float64))).astype(np.float32)
                zt = np.float32(sigma_t) * noise_t + prior
            elif model == "gauss":
                zt = np.float32(sigma_t) * noise_t
            else:
                raise ValueError(model)
            tgt[b, j] = zt
            dft[b, j] = zt + np.float32(sigma_d) * noise_d
            kids = children.get(j, [])
            if not kids:
                continue
            score = _cast(dft[b, j], dtype).double().numpy() / T
            for c in kids:
                g = -np.log(-np.log(rng.random(V) * (1 - 2.0**-53) + 2.0**-54))
                tok[b, c] = int(np.argmax(score + g))
    u = uniforms24(_batch_rng(seed + 7919), (B, n))
    return TreeSampleInputs(_cast(tgt, dtype), _cast(dft, dtype), torch.from_numpy(tok),
                            torch.from_numpy(par), torch.from_numpy(u), T, len(depth_counts),
                            meta=dict(B=B, n=n, V=V, seed=seed))


def make_tree(B: int = 8, V: int = V_QWEN, *, depth_counts=(8, 8, 8, 4, 3), branching: int = 8,
              plant_prob: float = 0.6, plant_value: float = 40.0, dtype: str = "bf16",
              sigma_t: float = 3.0, zipf_s: float = 1.1, seed: int = 0) -> TreeInputs:
    """Candidate trees in BFS order: node 0 is the root, depth d holds
    depth_counts[d-1] nodes whose parents are drawn among depth d-1 nodes with
    at most ``branching`` children each; siblings carry distinct tokens.  With
    probability ``plant_prob`` one child of a parent gets a token whose logit in
    the parent's row is set to ``plant_value`` (above every generated logit),
    so that accepted depths span 0..len(depth_counts)."""
    n = 1 + sum(depth_counts)
    z = np.empty((B, n, V), np.float32)
    tok = np.zeros((B, n), np.int32)
    par = np.full((B, n), -1, np.int32)
    brng = _batch_rng(seed)
    for b in range(B):
        for j in range(n):
            rng = _row_rng(seed, b * n + j)
            noise = rng.standard_normal(V, dtype=np.float32)
            perm = rng.permutation(V)
            z[b, j] = sigma_t * noise + (-zipf_s * np.log1p(perm.astype(np.float64))).astype(np.float32)
        children = _tree_shape(brng, par[b], depth_counts, branching)
        for p, ch in children.items():
            toks = brng.choice(V, size=len(ch), replace=False)
            for j, t in zip(ch, toks):
                tok[b, j] = int(t)
            if brng.random() < plant_prob:
                j = ch[int(brng.integers(len(ch)))]
                z[b, p, tok[b, j]] = plant_value
    return TreeInputs(_cast(z, dtype), torch.from_numpy(tok), torch.from_numpy(par),
                      len(depth_counts), meta=dict(B=B, n=n, V=V, seed=seed))


def ragged_lengths(B: int, k: int, seed: int = 0, idle_frac: float = 0.15):
    """Per-request draft counts k_b uniform on 0..k and an active mask (a
    request is idle with probability idle_frac); the first min(B, k+1)
    requests are active with k_b = 0, 1, .., k so that every length occurs.
    Returns int32 tensors (draft_len, active)."""
    rng = _batch_rng(seed + 104729)
    klen = rng.integers(0, k + 1, B).astype(np.int32)
    act = (rng.random(B) >= idle_frac).astype(np.int32)
    m = min(B, k + 1)
    klen[:m] = np.arange(m, dtype=np.int32)
    act[:m] = 1
    return torch.from_numpy(klen), torch.from_numpy(act)


# The workloads, by what they are.
def tiny_chain(seed: int = 0) -> ChainInputs:
    """B=4, k=3, V=1024 fp32, z_t ~ N(0, 2^2), z_d = z_t + N(0, 0.5^2), T=1."""
    return make_chain(4, 3, 1024, dtype="f32", model="gauss", sigma_t=2.0, sigma_d=0.5,
                      temperature=1.0, seed=seed)


def qwen_chain(B: int = 32, k: int = 3, sigma_d: float = 1.0, seed: int = 0,
               temperature: float = 0.7) -> ChainInputs:
    """Qwen-vocabulary chain verify: V=151936 bf16, Zipf(1.1) log-prior."""
    return make_chain(B, k, V_QWEN, dtype="bf16", model="zipf", sigma_t=3.0, sigma_d=sigma_d,
                      zipf_s=1.1, temperature=temperature, seed=seed)


def kd_chain(B: int = 256, k: int = 3, seed: int = 0) -> ChainInputs:
    """Fused verify + KD: 16 prompts x 16 rollouts, V=151936 bf16, T=1, r ~ U[0,1]."""
    return qwen_chain(B=B, k=k, sigma_d=1.0, seed=seed, temperature=1.0)
