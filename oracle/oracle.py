"""Python binding of the float64 CPU oracle (``sv_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product path never
imports this module; the CUDA library and this oracle share no code.

Each function takes host arrays (torch CPU tensors or numpy arrays), widens
nothing itself (the C code widens bf16/fp32 to float64 exactly) and returns
numpy arrays.  See the header of ``sv_oracle.c`` for the definitions followed
and the pages they come from.  One function is plain Python: ``sched_select``,
the adaptive scheduler's table lookup (no float64 arithmetic to speak of).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_DIR = Path(__file__).resolve().parent
_SRC = _DIR / "sv_oracle.c"

F32, BF16 = 0, 1
DRAFT_LOGITS, DRAFT_PROBS = 0, 1
W_RAW, W_GROUP_NORM = 0, 1

_ERRORS = {
    -1: "bad argument",
    -2: "token id out of range",
    -3: "row without a finite logit",
    -4: "invalid tree",
    -5: "out of memory",
}


class OracleError(RuntimeError):
    pass


def lib_path(plant: int = 0) -> Path:
    return _DIR / ("libsv_oracle.so" if plant == 0 else f"libsv_oracle_plant{plant}.so")


def build(force: bool = False, plant: int = 0) -> Path:
    """Compile the oracle with gcc (IEEE float64, no contraction, OpenMP)."""
    out = lib_path(plant)
    if out.exists() and not force and out.stat().st_mtime >= _SRC.stat().st_mtime:
        return out
    tmp = out.with_suffix(f".{os.getpid()}.tmp")
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", f"-DOR_PLANT={plant}", "-o", str(tmp), str(_SRC), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_LIBS: dict[int, ctypes.CDLL] = {}


def _lib(plant: int = 0) -> ctypes.CDLL:
    if plant not in _LIBS:
        L = ctypes.CDLL(str(build(plant=plant)))
        vp, i32p, f32p, f64p = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32),
                                ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double))
        ci, cd = ctypes.c_int, ctypes.c_double
        L.oracle_verify_chain.argtypes = [vp, ci, vp, ci, ci, i32p, f32p, ci, ci, ci, cd, i32p, i32p,
                                          i32p, i32p, f64p, f64p, f64p, i32p, i32p, ci]
        L.oracle_tree_sample.argtypes = [vp, ci, vp, ci, ci, i32p, i32p, f32p, ci, ci, ci, cd, ci,
                                         i32p, i32p, i32p, f64p, f64p, i32p, i32p, ci]
        L.oracle_tree_greedy.argtypes = [vp, ci, i32p, i32p, ci, ci, ci, ci, i32p, i32p, i32p, ci]
        L.oracle_topk.argtypes = [vp, ci, ci, ci, ci, cd, f64p, i32p, f64p, ci]
        L.oracle_kl.argtypes = [f64p, i32p, ci, ci, ci, vp, ci, ci, ci, cd, f64p, f64p, ci]
        L.oracle_reward_loss.argtypes = [f64p, i32p, f64p, ci, ci, ci, ci, cd, ci, i32p, i32p,
                                         f64p, f64p,
                                         f64p]
        L.oracle_softmax.argtypes = [vp, ci, ci, ci, cd, f64p, f64p]
        L.oracle_kd_grad.argtypes = [f64p, i32p, ci, ci, ci, vp, ci, ci, cd, i32p, f64p, ci, ci,
                                     cd, ci, f64p, ci]
        L.oracle_max_threads.argtypes = []
        for name in ("oracle_verify_chain", "oracle_tree_greedy", "oracle_topk", "oracle_kl",
                     "oracle_reward_loss", "oracle_softmax", "oracle_kd_grad",
                     "oracle_max_threads"):
            getattr(L, name).restype = ci
        _LIBS[plant] = L
    return _LIBS[plant]


def max_threads() -> int:
    return int(_lib().oracle_max_threads())


def _raw(x):
    """Return (contiguous numpy array of raw element bits, dtype code)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"unsupported dtype {x.dtype}")


def _np(x, dtype):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=dtype)


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _opt_i32(x, n: int):
    """An optional int32 [n] argument (None passes NULL); the pointer keeps the
    converted array alive for the call."""
    if x is None:
        return None
    a = _np(x, np.int32).reshape(-1)
    if a.size != n:
        raise ValueError(f"expected {n} entries, got {a.size}")
    return _ptr(a, ctypes.c_int32)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: {_ERRORS.get(rc, rc)}")


def verify_chain(target, draft, draft_tokens, uniforms, temperature: float, *,
                 draft_kind: int = DRAFT_LOGITS, threads: int = 0, plant: int = 0,
                 allow_errors: bool = False, draft_len=None, active=None) -> dict:
    """Chain verification of B requests with k draft tokens each.

    target [B, k+1, V] and draft [B, k, V] (fp32 or bf16; draft may be fp32
    probabilities), draft_tokens [B, k] int32, uniforms [B, k+1] fp32.
    ``temperature`` is widened from fp32, as the CUDA path receives it.
    """
    t, tdt = _raw(target)
    B, P, V = t.shape
    k = P - 1
    x = _np(draft_tokens, np.int32).reshape(B, k)
    T = float(np.float32(temperature))
    if T > 0:
        d, ddt = _raw(draft)
        u = _np(uniforms, np.float32).reshape(B, P)
    else:
        d, ddt = (None, F32) if draft is None else _raw(draft)
        u = np.zeros((B, P), np.float32) if uniforms is None else _np(uniforms, np.float32)
    acc = np.zeros(B, np.int32)
    out = np.zeros((B, P), np.int32)
    px = np.zeros((B, k), np.float64)
    qx = np.zeros((B, k), np.float64)
    margin = np.zeros(B, np.float64)
    srow = np.zeros(B, np.int32)
    fb = np.zeros(B, np.int32)
    rc = _lib(plant).oracle_verify_chain(
        t.ctypes.data, tdt, None if d is None else d.ctypes.data, ddt, draft_kind,
        _ptr(x, ctypes.c_int32), _ptr(u, ctypes.c_float), B, k, V, T,
        _opt_i32(draft_len, B), _opt_i32(active, B),
        _ptr(acc, ctypes.c_int32), _ptr(out, ctypes.c_int32), _ptr(px, ctypes.c_double),
        _ptr(qx, ctypes.c_double), _ptr(margin, ctypes.c_double), _ptr(srow, ctypes.c_int32),
        _ptr(fb, ctypes.c_int32), threads)
    if not allow_errors:
        _check(rc, "verify_chain")
    return dict(accepted_len=acc, out_tokens=out, p_x=px, q_x=qx, cdf_margin=margin,
                sample_row=srow, fallback=fb, status=rc)


def tree_sample(target, draft, node_tokens, parents, uniforms, temperature: float,
                max_depth: int, *, draft_kind: int = DRAFT_LOGITS, threads: int = 0,
                plant: int = 0) -> dict:
    """Sampling verification of B candidate trees of n nodes by multi-step
    speculative sampling: target and draft [B, n, V], uniforms [B, n]."""
    t, tdt = _raw(target)
    d, ddt = _raw(draft)
    B, n, V = t.shape
    tok = _np(node_tokens, np.int32).reshape(B, n)
    par = _np(parents, np.int32).reshape(B, n)
    u = _np(uniforms, np.float32).reshape(B, n)
    W = max_depth + 1
    acc = np.zeros(B, np.int32)
    out = np.zeros((B, W), np.int32)
    nodes = np.zeros((B, W), np.int32)
    tm = np.zeros(B, np.float64)
    cm = np.zeros(B, np.float64)
    fb = np.zeros(B, np.int32)
    nt = np.zeros(B, np.int32)
    rc = _lib(plant).oracle_tree_sample(
        t.ctypes.data, tdt, d.ctypes.data, ddt, draft_kind, _ptr(tok, ctypes.c_int32),
        _ptr(par, ctypes.c_int32), _ptr(u, ctypes.c_float), B, n, V,
        float(np.float32(temperature)), max_depth, _ptr(acc, ctypes.c_int32),
        _ptr(out, ctypes.c_int32), _ptr(nodes, ctypes.c_int32), _ptr(tm, ctypes.c_double),
        _ptr(cm, ctypes.c_double), _ptr(fb, ctypes.c_int32), _ptr(nt, ctypes.c_int32), threads)
    _check(rc, "tree_sample")
    return dict(accepted_len=acc, out_tokens=out, accepted_nodes=nodes, test_margin=tm,
                cdf_margin=cm, fallback=fb, n_tests=nt)


def tree_greedy(logits, node_tokens, parents, max_depth: int, *, threads: int = 0) -> dict:
    """Greedy verification of B candidate trees of n nodes (logits [B, n, V])."""
    z, dt = _raw(logits)
    B, n, V = z.shape
    tok = _np(node_tokens, np.int32).reshape(B, n)
    par = _np(parents, np.int32).reshape(B, n)
    W = max_depth + 1
    acc = np.zeros(B, np.int32)
    out = np.zeros((B, W), np.int32)
    nodes = np.zeros((B, W), np.int32)
    rc = _lib().oracle_tree_greedy(z.ctypes.data, dt, _ptr(tok, ctypes.c_int32),
                                   _ptr(par, ctypes.c_int32), B, n, V, max_depth,
                                   _ptr(acc, ctypes.c_int32), _ptr(out, ctypes.c_int32),
                                   _ptr(nodes, ctypes.c_int32), threads)
    _check(rc, "tree_greedy")
    return dict(accepted_len=acc, out_tokens=out, accepted_nodes=nodes)


def topk(logits, K: int, temperature: float, *, threads: int = 0) -> dict:
    """Top-K log-probs of every row of logits [..., V] (rows flattened)."""
    z, dt = _raw(logits)
    V = z.shape[-1]
    rows = z.size // V
    lp = np.zeros((rows, K), np.float64)
    ix = np.zeros((rows, K), np.int32)
    lse = np.zeros(rows, np.float64)
    rc = _lib().oracle_topk(z.ctypes.data, dt, rows, V, K, float(np.float32(temperature)),
                            _ptr(lp, ctypes.c_double), _ptr(ix, ctypes.c_int32),
                            _ptr(lse, ctypes.c_double), threads)
    _check(rc, "topk")
    lead = z.shape[:-1]
    return dict(topk_logp=lp.reshape(*lead, K), topk_idx=ix.reshape(*lead, K),
                lse=lse.reshape(lead))


def kl(topk_logp, topk_idx, draft, temperature: float, *, draft_kind: int = DRAFT_LOGITS,
       threads: int = 0) -> dict:
    """KL(p~ || q) for every draft row; topk buffers are [B, k+1, K]."""
    lp = _np(topk_logp, np.float64)
    ix = _np(topk_idx, np.int32)
    B, P, K = lp.shape
    k = P - 1
    d, ddt = _raw(draft)
    V = d.shape[-1]
    out = np.zeros((B, k), np.float64)
    scale = np.zeros((B, k), np.float64)
    rc = _lib().oracle_kl(_ptr(lp, ctypes.c_double), _ptr(ix, ctypes.c_int32), B, k, K,
                          d.ctypes.data, ddt, draft_kind, V, float(np.float32(temperature)),
                          _ptr(out, ctypes.c_double), _ptr(scale, ctypes.c_double), threads)
    _check(rc, "kl")
    return dict(kl=out, scale=scale)


def reward_loss(kl_values, accepted_len, reward, *, mode: int = W_RAW, group: int = 1,
                clip: float = 0.0, positions: int = 0, draft_len=None, active=None) -> dict:
    """Reward-weighted KD loss per request and its sum."""
    klv = _np(kl_values, np.float64)
    B, k = klv.shape
    acc = _np(accepted_len, np.int32)
    r = _np(reward, np.float64)
    w = np.zeros(B, np.float64)
    loss = np.zeros(B, np.float64)
    total = np.zeros(1, np.float64)
    rc = _lib().oracle_reward_loss(_ptr(klv, ctypes.c_double), _ptr(acc, ctypes.c_int32),
                                   _ptr(r, ctypes.c_double), B, k, mode, group, float(clip),
                                   int(positions), _opt_i32(draft_len, B),
                                   _opt_i32(active, B), _ptr(w, ctypes.c_double),
                                   _ptr(loss, ctypes.c_double),
                                   _ptr(total, ctypes.c_double))
    _check(rc, "reward_loss")
    return dict(w=w, loss=loss, total=float(total[0]))


def kd_grad(topk_logp, topk_idx, draft, accepted_len, reward, temperature: float, *,
            mode: int = W_RAW, group: int = 1, clip: float = 0.0, positions: int = 0,
            threads: int = 0):
    """d loss / d draft logits [B, k, V] (float64) of the reward-weighted KD loss."""
    lp = _np(topk_logp, np.float64)
    ix = _np(topk_idx, np.int32)
    B, P, K = lp.shape
    k = P - 1
    d, ddt = _raw(draft)
    V = d.shape[-1]
    acc = _np(accepted_len, np.int32)
    r = _np(reward, np.float64)
    g = np.zeros((B, k, V), np.float64)
    rc = _lib().oracle_kd_grad(_ptr(lp, ctypes.c_double), _ptr(ix, ctypes.c_int32), B, k, K,
                               d.ctypes.data, ddt, V, float(np.float32(temperature)),
                               _ptr(acc, ctypes.c_int32), _ptr(r, ctypes.c_double), mode, group,
                               float(clip), int(positions), _ptr(g, ctypes.c_double), threads)
    _check(rc, "kd_grad")
    return g


def softmax(logits, temperature: float) -> dict:
    z, dt = _raw(logits)
    V = z.shape[-1]
    rows = z.size // V
    p = np.zeros((rows, V), np.float64)
    lz = np.zeros(rows, np.float64)
    rc = _lib().oracle_softmax(z.ctypes.data, dt, rows, V, float(np.float32(temperature)),
                               _ptr(p, ctypes.c_double), _ptr(lz, ctypes.c_double))
    _check(rc, "softmax")
    return dict(p=p.reshape(z.shape), log_partition=lz.reshape(z.shape[:-1]))


def verify_kd(target, draft, draft_tokens, uniforms, reward, temperature: float, K: int, *,
              mode: int = W_RAW, group: int = 1, clip: float = 0.0,
              draft_kind: int = DRAFT_LOGITS, positions: int = 0, threads: int = 0,
              draft_len=None, active=None) -> dict:
    """Chain verification followed by the KD quantities, each step as above."""
    v = verify_chain(target, draft, draft_tokens, uniforms, temperature,
                     draft_kind=draft_kind, threads=threads, draft_len=draft_len, active=active)
    tk = topk(target, K, temperature, threads=threads)
    d = kl(tk["topk_logp"], tk["topk_idx"], draft, temperature, draft_kind=draft_kind,
           threads=threads)
    rl = reward_loss(d["kl"], v["accepted_len"], reward, mode=mode, group=group, clip=clip,
                     positions=positions, draft_len=draft_len, active=active)
    return {**v, **tk, **d, **rl}


def sched_select(throughput, batches, nonspec: int, active_batch: int):
    """Adaptive scheduler lookup ("ReSpec ... (reading notes)", section 3 "G1
    解法: Adaptive Speculative Decoding Server": the solver's profiled
    throughput per configuration and batch size; the scheduler picks the best
    configuration for the active batch and falls back to plain decoding when
    the predicted speedup is below 1).  Reading: each configuration's
    throughput is interpolated linearly between the profiled batch sizes
    around the active batch (held at the end values outside them); the best
    speculative configuration is the largest (lowest index on ties).
    Returns (config, best speculative speedup), in float64 from the float32
    table."""
    thr = [[float(np.float32(v)) for v in row] for row in np.asarray(throughput)]
    bs = [int(b) for b in batches]
    n_cfg = len(thr)

    def interp(row):
        if active_batch <= bs[0]:
            return row[0]
        if active_batch >= bs[-1]:
            return row[-1]
        for j in range(len(bs) - 1):
            if bs[j] <= active_batch < bs[j + 1]:
                t = (active_batch - bs[j]) / (bs[j + 1] - bs[j])
                return row[j] + t * (row[j + 1] - row[j])
        raise AssertionError("unreachable")

    base = interp(thr[nonspec])
    best, best_thr = -1, 0.0
    for c in range(n_cfg):
        if c == nonspec:
            continue
        v = interp(thr[c])
        if best < 0 or v > best_thr:
            best, best_thr = c, v
    speedup = 0.0 if best < 0 else best_thr / base
    return (nonspec if best < 0 or speedup < 1.0 else best), speedup
