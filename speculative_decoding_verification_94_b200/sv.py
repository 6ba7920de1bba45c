"""Python binding of libsv (the C ABI declared in include/sv.h).

Argument marshalling only: every step of verification runs in the CUDA
kernels of libsv.so.  PyTorch provides device memory and the current stream.
There is no CPU fallback: if libsv.so is missing, every call raises.

Function names and argument order follow the C ABI; see include/sv.h for the
operation each call performs and the pages it restates.
"""
from __future__ import annotations

import ctypes
import threading
from pathlib import Path

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libsv.so"

SV_OK, SV_ERR_INVALID_ARG, SV_ERR_UNSUPPORTED, SV_ERR_CUDA = 0, 1, 2, 3
SV_ERR_DEVICE_CHECK, SV_ERR_TIMEOUT, SV_ERR_WORKSPACE = 4, 5, 6
SV_F32, SV_BF16 = 0, 1
SV_DRAFT_LOGITS, SV_DRAFT_PROBS = 0, 1
SV_W_RAW, SV_W_GROUP_NORM = 0, 1
SV_DEV_BAD_TOKEN, SV_DEV_NO_FINITE, SV_DEV_TIMEOUT, SV_DEV_BAD_TREE = 0x1, 0x2, 0x4, 0x8
SV_DEV_BAD_INDEX, SV_DEV_BAD_LEN, SV_DEV_ERROR_MASK = 0x10, 0x20, 0xFF
SV_DEV_RESIDUAL_ZERO, SV_DEV_TOPK_SLOW = 0x100, 0x200

SV_KNOB_CLUSTER_CTAS, SV_KNOB_STREAM_COUNT, SV_KNOB_STREAM_W, SV_KNOB_WAIT_NS = 1, 2, 3, 4
SV_KNOB_STALL, SV_KNOB_STAGES, SV_KNOB_ORDER, SV_KNOB_PERSISTENT = 5, 6, 7, 8
SV_KNOB_KERNEL_MARKS = 9
SV_KNOB_FINISH_READ = 10
SV_MARK_STREAM, SV_MARK_FINISH, SV_MARK_CHAIN = 0, 1, 2
MARK_NAMES = {SV_MARK_STREAM: "stream", SV_MARK_FINISH: "finish", SV_MARK_CHAIN: "chain"}

EXPORTS = ("sv_verify_chain", "sv_verify_chain_ragged", "sv_verify_chain_noalloc", "sv_set_knob",
           "sv_kernel_times",
           "sv_verify_tree_greedy", "sv_kd_grad", "sv_kd_grad_workspace_size",
           "sv_verify_tree_sample", "sv_extract_topk_kd", "sv_kd_kl_loss", "sv_sched_select",
           "sv_verify_chain_workspace_size", "sv_verify_tree_workspace_size",
           "sv_extract_topk_workspace_size", "sv_kd_kl_loss_workspace_size",
           "sv_device_status_check", "sv_status_string", "sv_version")


class SVError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class sv_kd_args(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int), ("topk_logp", ctypes.c_void_p),
                ("topk_idx", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("kl", ctypes.c_void_p), ("reward", ctypes.c_void_p),
                ("wmode", ctypes.c_int), ("group", ctypes.c_int), ("clip", ctypes.c_float),
                ("loss", ctypes.c_void_p), ("total", ctypes.c_void_p),
                ("positions", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def lib_path() -> Path:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libsv.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not _LIB_PATH.exists():
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                                   "`python -m speculative_decoding_verification_94_b200.build`")
            L = ctypes.CDLL(str(_LIB_PATH))
            vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            L.sv_verify_chain.argtypes = [vp, ci, vp, ci, ci, vp, vp, ci, ci, ci, cf, vp, vp,
                                          ctypes.POINTER(sv_kd_args), vp, sz, vp, vp]
            L.sv_verify_chain_ragged.argtypes = [vp, ci, vp, ci, ci, vp, vp, vp, vp, ci, ci, ci,
                                                 cf, vp, vp, ctypes.POINTER(sv_kd_args), vp, sz,
                                                 vp, vp]
            L.sv_verify_chain_ragged.restype = ci
            L.sv_verify_chain_noalloc.argtypes = [vp, ci, vp, ci, ci, vp, vp, ci, ci, ci, cf, vp,
                                                  vp, ctypes.POINTER(sv_kd_args), vp, vp]
            L.sv_verify_chain_noalloc.restype = ci
            L.sv_verify_tree_greedy.argtypes = [vp, ci, vp, vp, ci, ci, ci, ci, vp, vp, vp, vp, sz,
                                                vp, vp]
            L.sv_extract_topk_kd.argtypes = [vp, ci, ci, ci, ci, cf, vp, vp, vp, vp, sz, vp, vp]
            L.sv_kd_kl_loss.argtypes = [vp, vp, ci, ci, ci, vp, ci, ci, ci, cf, vp, vp, ci, ci, cf,
                                        ci, vp, vp, vp, vp, sz, vp, vp]
            L.sv_kd_grad.argtypes = [vp, vp, ci, ci, ci, vp, ci, ci, cf, vp, vp, ci, ci, cf, ci,
                                     vp, vp, sz, vp, vp]
            L.sv_kd_grad_workspace_size.argtypes = [ci, ci, ci]
            L.sv_kd_grad_workspace_size.restype = sz
            for f in ("sv_verify_chain", "sv_verify_tree_greedy", "sv_extract_topk_kd",
                      "sv_kd_kl_loss", "sv_kd_grad", "sv_device_status_check"):
                getattr(L, f).restype = ci
            L.sv_device_status_check.argtypes = [ctypes.c_int32]
            L.sv_verify_chain_workspace_size.argtypes = [ci, ci, ci, ci]
            L.sv_verify_tree_workspace_size.argtypes = [ci, ci, ci]
            L.sv_extract_topk_workspace_size.argtypes = [ci, ci, ci]
            L.sv_kd_kl_loss_workspace_size.argtypes = [ci, ci, ci]
            for f in ("sv_verify_chain_workspace_size", "sv_verify_tree_workspace_size",
                      "sv_extract_topk_workspace_size", "sv_kd_kl_loss_workspace_size"):
                getattr(L, f).restype = sz
            L.sv_verify_tree_sample.argtypes = [vp, ci, vp, ci, ci, vp, vp, vp, ci, ci, ci, ci,
                                                cf, vp, vp, vp, vp, vp]
            L.sv_verify_tree_sample.restype = ci
            L.sv_sched_select.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp]
            L.sv_sched_select.restype = ci
            L.sv_set_knob.argtypes = [ci, ctypes.c_longlong]
            L.sv_set_knob.restype = ci
            L.sv_kernel_times.argtypes = [vp, vp, ci, vp]
            L.sv_kernel_times.restype = ci
            L.sv_status_string.argtypes = [ci]
            L.sv_status_string.restype = ctypes.c_char_p
            L.sv_version.argtypes = []
            L.sv_version.restype = ci
            _lib = L
    return _lib


_KNOB_VALUES: dict = {}  # what this process last set, so that knobs() can restore it


def sv_set_knob(knob: int, value: int) -> None:
    """Process-wide test / tuning setting (see sv.h); 0 restores the default."""
    _check(lib().sv_set_knob(int(knob), int(value)), "sv_set_knob")
    _KNOB_VALUES[int(knob)] = int(value)


def sv_kernel_times(cap: int = 2048):
    """Durations (us) and kinds of the kernel launches marked since the last
    read (SV_KNOB_KERNEL_MARKS): a list of (kind name, microseconds)."""
    import ctypes
    us = (ctypes.c_float * cap)()
    tags = (ctypes.c_int32 * cap)()
    n = ctypes.c_int32(0)
    _check(lib().sv_kernel_times(us, tags, int(cap), ctypes.byref(n)), "sv_kernel_times")
    return [(MARK_NAMES.get(tags[j], str(tags[j])), float(us[j])) for j in range(n.value)]


class knobs:
    """Context manager: set knobs by name for the block, then put back the
    values they had before it (blocks nest)."""

    def __init__(self, **kw):
        self.kw = {globals()["SV_KNOB_" + k.upper()]: v for k, v in kw.items()}
        self.saved = {}

    def __enter__(self):
        for k, v in self.kw.items():
            self.saved[k] = _KNOB_VALUES.get(k, 0)
            sv_set_knob(k, v)
        return self

    def __exit__(self, *exc):
        for k, v in self.saved.items():
            sv_set_knob(k, v)
        return False


def status_string(status: int) -> str:
    return lib().sv_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != SV_OK:
        raise SVError(what, rc)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SV_BF16
    if t.dtype == torch.float32:
        return SV_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


# Workspaces: zero-filled once when allocated; every completed call returns
# all of it to zero, so a cached buffer serves any later call that fits.
_WS: dict = {}


def workspace(device: torch.device, B: int, nbytes: int) -> torch.Tensor:
    key = (device.index if device.index is not None else torch.cuda.current_device())
    cur = _WS.get(key)
    if cur is None or cur.numel() < nbytes:
        cur = torch.zeros(max(nbytes, cur.numel() if cur is not None else 0), dtype=torch.uint8,
                          device=device)
        _WS[key] = cur
    return cur


def sv_verify_chain_workspace_size(B: int, k: int, V: int, K: int = 0) -> int:
    return int(lib().sv_verify_chain_workspace_size(B, k, V, K))


def sv_verify_tree_workspace_size(B: int, n: int, V: int) -> int:
    return int(lib().sv_verify_tree_workspace_size(B, n, V))


def sv_sched_select(throughput, batches, nonspec: int, active_batch: int) -> tuple[int, float]:
    """Adaptive scheduler lookup (see sv.h): the configuration to run at
    `active_batch` from a profiled throughput table [n_cfg, n_batch] over
    ascending batch sizes, and the best speculative configuration's predicted
    speedup.  Host arrays; nothing touches the GPU."""
    import numpy as np
    thr = np.ascontiguousarray(throughput, dtype=np.float32)
    bs = np.ascontiguousarray(batches, dtype=np.int32)
    if thr.ndim != 2 or bs.ndim != 1 or thr.shape[1] != bs.shape[0]:
        raise ValueError("throughput must be [n_cfg, n_batch] and batches [n_batch]")
    cfg = ctypes.c_int32(-1)
    sp = ctypes.c_float(0.0)
    rc = lib().sv_sched_select(thr.ctypes.data, bs.ctypes.data, thr.shape[0], thr.shape[1],
                               int(nonspec), int(active_batch), ctypes.addressof(cfg),
                               ctypes.addressof(sp))
    _check(rc, "sv_sched_select")
    return int(cfg.value), float(sp.value)


def sv_extract_topk_workspace_size(rows: int, V: int, K: int) -> int:
    return int(lib().sv_extract_topk_workspace_size(rows, V, K))


def sv_kd_kl_loss_workspace_size(B: int, k: int, V: int) -> int:
    return int(lib().sv_kd_kl_loss_workspace_size(B, k, V))


def sv_verify_chain(target: torch.Tensor, draft: torch.Tensor | None, draft_tokens: torch.Tensor,
                    uniforms: torch.Tensor | None, temperature: float, *,
                    draft_kind: str = "logits", kd: dict | None = None, out: dict | None = None,
                    ws: torch.Tensor | None = None, device_status: torch.Tensor | None = None,
                    stream=None) -> dict:
    """Verify k drafted tokens for each of B requests (see sv.h).

    target [B, k+1, V], draft [B, k, V] (logits, or fp32 probabilities with
    draft_kind="probs"), draft_tokens [B, k] int32, uniforms [B, k+1] fp32.
    kd: None or dict(K=32, reward=[B] fp32, wmode="raw"|"group_norm",
    group=16, clip=0.0, positions=0) for the fused top-K / KL / loss outputs.
    Returns the output tensors (allocated unless given in `out`).
    """
    return _verify_chain(target, draft, draft_tokens, uniforms, temperature, None, None,
                         draft_kind, kd, out, ws, device_status, stream)


def sv_verify_chain_ragged(target: torch.Tensor, draft: torch.Tensor | None,
                           draft_tokens: torch.Tensor, uniforms: torch.Tensor | None,
                           temperature: float, *, draft_len: torch.Tensor | None = None,
                           active: torch.Tensor | None = None, draft_kind: str = "logits",
                           kd: dict | None = None, out: dict | None = None,
                           ws: torch.Tensor | None = None,
                           device_status: torch.Tensor | None = None, stream=None) -> dict:
    """sv_verify_chain for requests with their own draft counts (see sv.h).

    draft_len [B] int32 (k_b <= k; None: k) and active [B] int32 (0: an idle
    request; None: all active), both on the device; the rest as in
    sv_verify_chain, padded to k."""
    B = target.shape[0]
    for name, t in (("draft_len", draft_len), ("active", active)):
        if t is not None:
            _dev(t, name, torch.int32)
            if t.numel() != B:
                raise ValueError(f"{name} must have {B} entries")
    return _verify_chain(target, draft, draft_tokens, uniforms, temperature, draft_len, active,
                         draft_kind, kd, out, ws, device_status, stream)


def _verify_chain(target, draft, draft_tokens, uniforms, temperature, draft_len, active,
                  draft_kind, kd, out, ws, device_status, stream) -> dict:
    _dev(target, "target")
    B, P, V = target.shape
    k = P - 1
    dev = target.device
    _dev(draft_tokens, "draft_tokens", torch.int32)
    T = float(temperature)
    dk = SV_DRAFT_PROBS if draft_kind == "probs" else SV_DRAFT_LOGITS
    if draft is not None:
        _dev(draft, "draft")
    if uniforms is not None:
        _dev(uniforms, "uniforms", torch.float32)
    o = dict(out or {})
    o.setdefault("accepted_len", torch.empty(B, dtype=torch.int32, device=dev))
    o.setdefault("out_tokens", torch.empty(B, P, dtype=torch.int32, device=dev))
    kd_ptr = None
    if kd is not None:
        K = int(kd.get("K", 32))
        o.setdefault("topk_logp", torch.empty(B, P, K, dtype=torch.float32, device=dev))
        o.setdefault("topk_idx", torch.empty(B, P, K, dtype=torch.int32, device=dev))
        o.setdefault("lse", torch.empty(B, P, dtype=torch.float32, device=dev))
        o.setdefault("kl", torch.empty(B, k, dtype=torch.float32, device=dev))
        o.setdefault("loss", torch.empty(B, dtype=torch.float32, device=dev))
        o.setdefault("total", torch.empty(1, dtype=torch.float32, device=dev))
        reward = _dev(kd["reward"], "reward", torch.float32)
        wmode = SV_W_GROUP_NORM if kd.get("wmode", "raw") == "group_norm" else SV_W_RAW
        kd_ptr = ctypes.byref(sv_kd_args(K, o["topk_logp"].data_ptr(), o["topk_idx"].data_ptr(),
                                         o["lse"].data_ptr(), o["kl"].data_ptr(),
                                         reward.data_ptr(), wmode, int(kd.get("group", 1)),
                                         float(kd.get("clip", 0.0)), o["loss"].data_ptr(),
                                         o["total"].data_ptr(), int(kd.get("positions", 0))))
    nbytes = sv_verify_chain_workspace_size(B, k, V, int(kd.get("K", 32)) if kd else 0)
    w = ws if ws is not None else workspace(dev, B, nbytes)
    head = (_p(target), _dtype_code(target), _p(draft),
            _dtype_code(draft) if draft is not None else SV_F32, dk, _p(draft_tokens),
            _p(uniforms))
    tail = (B, k, V, T, _p(o["accepted_len"]), _p(o["out_tokens"]), kd_ptr, _p(w), w.numel(),
            _p(device_status), _stream(dev, stream))
    if draft_len is None and active is None:
        rc = lib().sv_verify_chain(*head, *tail)
        _check(rc, "sv_verify_chain")
    else:
        rc = lib().sv_verify_chain_ragged(*head, _p(draft_len), _p(active), *tail)
        _check(rc, "sv_verify_chain_ragged")
    return o


def sv_verify_chain_noalloc(target: torch.Tensor, draft: torch.Tensor | None,
                            draft_tokens: torch.Tensor, uniforms: torch.Tensor | None,
                            temperature: float, *, draft_kind: str = "logits",
                            kd: dict | None = None, out: dict | None = None,
                            device_status: torch.Tensor | None = None, stream=None) -> dict:
    """sv_verify_chain with the library's fixed per-device scratch instead of a
    workspace (see sv.h for its size limit and ordering rule).  Outputs are
    allocated here unless given in `out`; the C call itself allocates nothing."""
    _dev(target, "target")
    B, P, V = target.shape
    k = P - 1
    dev = target.device
    _dev(draft_tokens, "draft_tokens", torch.int32)
    dk = SV_DRAFT_PROBS if draft_kind == "probs" else SV_DRAFT_LOGITS
    if draft is not None:
        _dev(draft, "draft")
    if uniforms is not None:
        _dev(uniforms, "uniforms", torch.float32)
    o = dict(out or {})
    o.setdefault("accepted_len", torch.empty(B, dtype=torch.int32, device=dev))
    o.setdefault("out_tokens", torch.empty(B, P, dtype=torch.int32, device=dev))
    kd_ptr = None
    if kd is not None:
        K = int(kd.get("K", 32))
        o.setdefault("topk_logp", torch.empty(B, P, K, dtype=torch.float32, device=dev))
        o.setdefault("topk_idx", torch.empty(B, P, K, dtype=torch.int32, device=dev))
        o.setdefault("lse", torch.empty(B, P, dtype=torch.float32, device=dev))
        o.setdefault("kl", torch.empty(B, k, dtype=torch.float32, device=dev))
        o.setdefault("loss", torch.empty(B, dtype=torch.float32, device=dev))
        o.setdefault("total", torch.empty(1, dtype=torch.float32, device=dev))
        reward = _dev(kd["reward"], "reward", torch.float32)
        wmode = SV_W_GROUP_NORM if kd.get("wmode", "raw") == "group_norm" else SV_W_RAW
        kd_ptr = ctypes.byref(sv_kd_args(K, o["topk_logp"].data_ptr(), o["topk_idx"].data_ptr(),
                                         o["lse"].data_ptr(), o["kl"].data_ptr(),
                                         reward.data_ptr(), wmode, int(kd.get("group", 1)),
                                         float(kd.get("clip", 0.0)), o["loss"].data_ptr(),
                                         o["total"].data_ptr(), int(kd.get("positions", 0))))
    rc = lib().sv_verify_chain_noalloc(
        _p(target), _dtype_code(target), _p(draft),
        _dtype_code(draft) if draft is not None else SV_F32, dk, _p(draft_tokens), _p(uniforms),
        B, k, V, float(temperature), _p(o["accepted_len"]), _p(o["out_tokens"]), kd_ptr,
        _p(device_status), _stream(dev, stream))
    _check(rc, "sv_verify_chain_noalloc")
    return o


def sv_verify_tree_greedy(logits: torch.Tensor, node_tokens: torch.Tensor,
                          parents: torch.Tensor, max_depth: int, *, out: dict | None = None,
                          ws: torch.Tensor | None = None,
                          device_status: torch.Tensor | None = None, stream=None) -> dict:
    """Greedy verification of B candidate trees (logits [B, n, V])."""
    _dev(logits, "logits")
    B, n, V = logits.shape
    dev = logits.device
    _dev(node_tokens, "node_tokens", torch.int32)
    _dev(parents, "parents", torch.int32)
    W = max_depth + 1
    o = dict(out or {})
    o.setdefault("accepted_len", torch.empty(B, dtype=torch.int32, device=dev))
    o.setdefault("out_tokens", torch.empty(B, W, dtype=torch.int32, device=dev))
    o.setdefault("accepted_nodes", torch.empty(B, W, dtype=torch.int32, device=dev))
    nbytes = sv_verify_tree_workspace_size(B, n, V)
    w = ws if ws is not None else workspace(dev, B, nbytes)
    rc = lib().sv_verify_tree_greedy(_p(logits), _dtype_code(logits), _p(node_tokens),
                                     _p(parents), B, n, V, max_depth, _p(o["accepted_len"]),
                                     _p(o["out_tokens"]), _p(o["accepted_nodes"]), _p(w),
                                     w.numel(), _p(device_status), _stream(dev, stream))
    _check(rc, "sv_verify_tree_greedy")
    return o


def sv_verify_tree_sample(target: torch.Tensor, draft: torch.Tensor, node_tokens: torch.Tensor,
                          parents: torch.Tensor, uniforms: torch.Tensor, temperature: float,
                          max_depth: int, *, draft_kind: str = "logits", out: dict | None = None,
                          device_status: torch.Tensor | None = None, stream=None) -> dict:
    """Sampling verification of B candidate trees (see sv.h): target and draft
    [B, n, V] (draft logits, or fp32 probabilities with draft_kind="probs"),
    node_tokens and parents [B, n] int32, uniforms [B, n] fp32."""
    _dev(target, "target")
    _dev(draft, "draft")
    B, n, V = target.shape
    dev = target.device
    _dev(node_tokens, "node_tokens", torch.int32)
    _dev(parents, "parents", torch.int32)
    _dev(uniforms, "uniforms", torch.float32)
    W = max_depth + 1
    o = dict(out or {})
    o.setdefault("accepted_len", torch.empty(B, dtype=torch.int32, device=dev))
    o.setdefault("out_tokens", torch.empty(B, W, dtype=torch.int32, device=dev))
    o.setdefault("accepted_nodes", torch.empty(B, W, dtype=torch.int32, device=dev))
    dk = SV_DRAFT_PROBS if draft_kind == "probs" else SV_DRAFT_LOGITS
    rc = lib().sv_verify_tree_sample(_p(target), _dtype_code(target), _p(draft),
                                     _dtype_code(draft), dk, _p(node_tokens), _p(parents),
                                     _p(uniforms), B, n, V, max_depth, float(temperature),
                                     _p(o["accepted_len"]), _p(o["out_tokens"]),
                                     _p(o["accepted_nodes"]), _p(device_status),
                                     _stream(dev, stream))
    _check(rc, "sv_verify_tree_sample")
    return o


def sv_extract_topk_kd(logits: torch.Tensor, K: int, temperature: float, *,
                       out: dict | None = None, ws: torch.Tensor | None = None,
                       device_status: torch.Tensor | None = None, stream=None) -> dict:
    """Top-K log-probs of every row of logits [..., V]."""
    _dev(logits, "logits")
    V = logits.shape[-1]
    lead = tuple(logits.shape[:-1])
    rows = logits.numel() // V if V else 0
    dev = logits.device
    o = dict(out or {})
    o.setdefault("topk_logp", torch.empty(*lead, K, dtype=torch.float32, device=dev))
    o.setdefault("topk_idx", torch.empty(*lead, K, dtype=torch.int32, device=dev))
    o.setdefault("lse", torch.empty(*lead, dtype=torch.float32, device=dev))
    nbytes = sv_extract_topk_workspace_size(rows, V, K)
    w = ws if ws is not None else workspace(dev, rows, nbytes)
    rc = lib().sv_extract_topk_kd(_p(logits), _dtype_code(logits), rows, V, K, float(temperature),
                                  _p(o["topk_logp"]), _p(o["topk_idx"]), _p(o["lse"]), _p(w),
                                  w.numel(), _p(device_status), _stream(dev, stream))
    _check(rc, "sv_extract_topk_kd")
    return o


def sv_kd_kl_loss(topk_logp: torch.Tensor, topk_idx: torch.Tensor, draft: torch.Tensor,
                  temperature: float, accepted_len: torch.Tensor, reward: torch.Tensor, *,
                  draft_kind: str = "logits", wmode: str = "raw", group: int = 1,
                  clip: float = 0.0, positions: int = 0, out: dict | None = None,
                  ws: torch.Tensor | None = None, device_status: torch.Tensor | None = None,
                  stream=None) -> dict:
    """Reward-weighted KD loss from top-K buffers [B, k+1, K] and draft [B, k, V]."""
    _dev(topk_logp, "topk_logp", torch.float32)
    _dev(topk_idx, "topk_idx", torch.int32)
    _dev(draft, "draft")
    _dev(accepted_len, "accepted_len", torch.int32)
    _dev(reward, "reward", torch.float32)
    B, P, K = topk_logp.shape
    k = P - 1
    V = draft.shape[-1]
    dev = draft.device
    dk = SV_DRAFT_PROBS if draft_kind == "probs" else SV_DRAFT_LOGITS
    o = dict(out or {})
    o.setdefault("kl", torch.empty(B, k, dtype=torch.float32, device=dev))
    o.setdefault("loss", torch.empty(B, dtype=torch.float32, device=dev))
    o.setdefault("total", torch.empty(1, dtype=torch.float32, device=dev))
    nbytes = sv_kd_kl_loss_workspace_size(B, k, V)
    w = ws if ws is not None else workspace(dev, B, nbytes)
    wm = SV_W_GROUP_NORM if wmode == "group_norm" else SV_W_RAW
    rc = lib().sv_kd_kl_loss(_p(topk_logp), _p(topk_idx), B, k, K, _p(draft), _dtype_code(draft),
                             dk, V, float(temperature), _p(accepted_len), _p(reward), wm,
                             int(group), float(clip), int(positions), _p(o["kl"]), _p(o["loss"]),
                             _p(o["total"]),
                             _p(w), w.numel(), _p(device_status), _stream(dev, stream))
    _check(rc, "sv_kd_kl_loss")
    return o


def sv_device_status_check(word: int) -> int:
    return int(lib().sv_device_status_check(ctypes.c_int32(int(word))))


def sv_version() -> int:
    return int(lib().sv_version())


def sv_kd_grad(topk_logp: torch.Tensor, topk_idx: torch.Tensor, draft: torch.Tensor,
               accepted_len: torch.Tensor, reward: torch.Tensor, temperature: float, *,
               wmode: str = "raw", group: int = 1, clip: float = 0.0, positions: int = 0,
               out: torch.Tensor | None = None, ws: torch.Tensor | None = None,
               device_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """d loss / d draft logits [B, k, V] fp32 of the reward-weighted KD loss (see sv.h)."""
    _dev(topk_logp, "topk_logp", torch.float32)
    _dev(topk_idx, "topk_idx", torch.int32)
    _dev(draft, "draft")
    _dev(accepted_len, "accepted_len", torch.int32)
    _dev(reward, "reward", torch.float32)
    B, P, K = topk_logp.shape
    k = P - 1
    V = draft.shape[-1]
    dev = draft.device
    g = out if out is not None else torch.empty(B, k, V, dtype=torch.float32, device=dev)
    nbytes = int(lib().sv_kd_grad_workspace_size(B, k, V))
    w = ws if ws is not None else workspace(dev, B, nbytes)
    wm = SV_W_GROUP_NORM if wmode == "group_norm" else SV_W_RAW
    rc = lib().sv_kd_grad(_p(topk_logp), _p(topk_idx), B, k, K, _p(draft), _dtype_code(draft), V,
                          float(temperature), _p(accepted_len), _p(reward), wm, int(group),
                          float(clip), int(positions), _p(g), _p(w), w.numel(), _p(device_status),
                          _stream(dev, stream))
    _check(rc, "sv_kd_grad")
    return g
