"""Comparison rules between the CUDA path and the float64 oracle.

Integers (accepted lengths, token ids, top-K indices) must be bit-exact,
except for requests whose draws lie within 1e-6 of an acceptance boundary
(|u - p(x)/q(x)| < 1e-6 at a tested position) or of an inverse-CDF boundary
(min_j |u - C_j / W| < 1e-6).  Those are counted; their outputs must still be
well formed.

Floats are compared with a relative tolerance of 1e-5 applied to the
magnitude that sets their rounding: for log-probabilities and log-partitions
the larger of |ref| and 1 (they are differences of O(|z|/T) numbers, so
relative error is meaningless at 0); for KL the larger of |ref| and
sum_j p~_j |log q_j|; for losses the weighted sum of those.
"""
from __future__ import annotations

import numpy as np

REL = 1e-5
WINDOW = 1e-6


def chain_flags(ref: dict, uniforms: np.ndarray, temperature: float) -> np.ndarray:
    B = ref["accepted_len"].shape[0]
    if temperature == 0.0:
        return np.zeros(B, bool)
    k = ref["p_x"].shape[1]
    u = np.asarray(uniforms, np.float64)
    flagged = ref["cdf_margin"] < WINDOW
    for b in range(B):
        n = int(ref["accepted_len"][b])
        for i in range(min(n + 1, k)):
            px, qx = ref["p_x"][b, i], ref["q_x"][b, i]
            if qx > 0 and abs(u[b, i] - px / qx) < WINDOW:
                flagged[b] = True
    return flagged


def assert_chain_match(gpu: dict, ref: dict, uniforms, temperature: float, k: int,
                       max_flag_frac: float = 0.05) -> dict:
    acc = gpu["accepted_len"].cpu().numpy()
    out = gpu["out_tokens"].cpu().numpy()
    flags = chain_flags(ref, uniforms, temperature)
    same = (acc == ref["accepted_len"]) & (out == ref["out_tokens"]).all(axis=1)
    bad = np.nonzero(~same & ~flags)[0]
    assert bad.size == 0, (
        f"{bad.size} unflagged mismatches, first b={bad[0]}: gpu acc={acc[bad[0]]} "
        f"out={out[bad[0]]} ref acc={ref['accepted_len'][bad[0]]} out={ref['out_tokens'][bad[0]]}")
    # flagged requests: outputs must be well formed
    for b in np.nonzero(flags)[0]:
        n = acc[b]
        assert 0 <= n <= k
        assert (out[b, n + 1:] == -1).all() and out[b, n] >= 0
    assert flags.mean() <= max_flag_frac, f"{flags.sum()} of {flags.size} requests flagged"
    return dict(flagged=int(flags.sum()), flagged_mismatch=int((~same & flags).sum()),
                requests=int(acc.size))


def assert_close(got, ref, scale, what: str, rel: float = REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.broadcast_to(np.asarray(scale, np.float64), ref.shape)
    both_inf = np.isinf(ref) & (got == ref)
    tol = rel * np.maximum(np.abs(np.where(np.isinf(ref), 0, ref)), scale)
    err = np.abs(got - ref)
    ok = both_inf | (err <= tol)
    if not ok.all():
        i = np.argmax(np.where(ok, -1, err / np.maximum(tol, 1e-300)))
        raise AssertionError(f"{what}: {int((~ok).sum())} values out of tolerance; worst at "
                             f"{np.unravel_index(i, ref.shape)}: got {got.flat[i]!r} "
                             f"ref {ref.flat[i]!r} tol {tol.flat[i]!r}")


def kd_rows(accepted_len, k: int):
    """Masks of the KD rows the verifier defines: target rows 0..n and draft
    rows 0..min(n, k-1) of each request (n = accepted_len).  Rows after the
    emitted position are not read by the verifier and hold -1 / NaN."""
    acc = np.asarray(accepted_len)
    t = np.arange(k + 1)[None, :] <= acc[:, None]
    d = np.arange(k)[None, :] <= acc[:, None]
    return t, d


def assert_kd_match(got: dict, ref: dict, k: int):
    acc = got["accepted_len"].cpu().numpy()
    tmask, dmask = kd_rows(acc, k)
    idx = got["topk_idx"].cpu().numpy()
    assert np.array_equal(idx[tmask], ref["topk_idx"][tmask]), "topk_idx"
    assert (idx[~tmask] == -1).all()
    lp = got["topk_logp"].cpu().numpy()
    assert_close(lp[tmask], ref["topk_logp"][tmask], 1.0, "topk_logp")
    assert np.isnan(lp[~tmask]).all()
    lse = got["lse"].cpu().numpy()
    assert_close(lse[tmask], ref["lse"][tmask], 1.0, "lse")
    assert np.isnan(lse[~tmask]).all()
    kl = got["kl"].cpu().numpy()
    assert_close(kl[dmask], ref["kl"][dmask], ref["scale"][dmask], "kl")
    assert np.isnan(kl[~dmask]).all()
    # the error actually reached, relative to |KL| itself (the bar's scale
    # above is the larger of |KL| and sum p~ |ln q|)
    r, g = ref["kl"][dmask], kl[dmask].astype(np.float64)
    nz = np.abs(r) > 0
    if nz.any():
        print(f"kl: worst error {float(np.max(np.abs(g[nz] - r[nz]) / np.abs(r[nz]))):.3e} "
              f"of |KL| over {int(nz.sum())} rows")


def bitwise_equal(a, b) -> bool:
    """Equality of two tensors bit for bit (NaN == NaN)."""
    import torch
    if a.dtype != b.dtype or a.shape != b.shape:
        return False
    if a.dtype.is_floating_point:
        return torch.equal(a.view(torch.int32 if a.element_size() == 4 else torch.int16),
                           b.view(torch.int32 if b.element_size() == 4 else torch.int16))
    return torch.equal(a, b)
