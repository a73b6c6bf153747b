"""Comparison helpers for the GPU parity tests (test infrastructure).

The CUDA path and the fp64 oracle receive the same stored tensors; these
helpers run the oracle on them and compare, stage by stage:

  build   GPU planes vs oracle planes (tolerances derived from fp32 arithmetic
          on the stored inputs, plus the bf16 rounding of the stored slopes);
  route   the oracle's routing run on the GPU-stored planes must keep the same
          level-1 blocks as the GPU, except for heads where the oracle's trace
          has a boundary case (cumulative mass within delta of p at the cut) or
          a near-tie straddling the cut (estimates closer than the fp32 error
          bound of the GPU estimate) - those are counted and reported;
  attend  the oracle's attention over the GPU's kept blocks vs the GPU output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import numpy as np
import torch

import oracle.zha_oracle as zo

U32 = 2.0 ** -24


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def p32(p):
    """The threshold (or per-step thresholds) as the library sees it (C floats)."""
    if np.ndim(p) == 0:
        return float(np.float32(p))
    return [float(np.float32(x)) for x in p]


# --------------------------------------------------------------------------- build
def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def compare_planes(gpu_mu, gpu_bias, gpu_f, orc: zo.Planes, dtype: str, refs: np.ndarray, label: str = ""):
    """Assert GPU planes (numpy fp64, [n, R, d] / [n, R]) match the oracle's within derived bounds."""
    n = orc.f.shape[0]
    d = orc.mu.shape[-1]
    mu_o, f_o, b_o = orc.mu[:n], orc.f[:n], orc.bias[:n]
    g_o = f_o - b_o
    # f: fp32 logsumexp of fp32 scores: a few ulps of the score magnitudes
    scale_f = np.abs(f_o) + np.abs(g_o) + 1.0
    err_f = np.abs(gpu_f[:n] - f_o)
    assert np.all(err_f <= 2e-5 * scale_f), f"{label} f: max err {err_f.max():.3e}"
    err_b = np.abs(gpu_bias[:n] - b_o)
    assert np.all(err_b <= 2e-5 * scale_f), f"{label} bias: max err {err_b.max():.3e}"
    vec_scale = np.max(np.abs(mu_o), axis=-1, keepdims=True) + 1e-30
    err_mu = np.abs(gpu_mu[:n] - mu_o)
    if dtype == "bf16":
        tol = 1.0 * bf16_ulp(mu_o) + 1e-4 * vec_scale
    else:
        tol = 2e-5 * vec_scale
    bad = err_mu > tol
    assert not bad.any(), f"{label} mu: {bad.sum()} elements out of bound, max err {err_mu.max():.3e}"


# --------------------------------------------------------------------------- route
@dataclass
class RouteReport:
    heads: int = 0
    exact: int = 0
    flagged: int = 0
    failures: List[str] = field(default_factory=list)


def ehat_error_bound(mu: np.ndarray, bias: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Bound on |e_gpu - e| for fp32 evaluation of max_j (b_j + q.mu_j/sqrt d) on the stored planes."""
    d = mu.shape[-1]
    mag = np.einsum("nrd,d->nr", np.abs(mu), np.abs(q)) / math.sqrt(d) + np.abs(bias)
    return (d + 8) * U32 * mag.max(axis=1) + 1e-7


def trace_flags(trace: zo.RouteTrace, planes, q: np.ndarray, p, block: int) -> List[str]:
    """Boundary / near-tie cases along the oracle's path (the places where fp32 and fp64 may differ)."""
    flags = []
    for s, st in enumerate(trace.steps):
        p = st.p
        if p >= 1:
            continue
        n = len(st.cand)
        lv = np.array([c[0] for c in st.cand])
        ix = np.array([c[1] for c in st.cand])
        eps = np.empty(n)
        for level in np.unique(lv):
            sel = np.nonzero(lv == level)[0]
            mu, bias = planes(int(level), ix[sel])
            eps[sel] = ehat_error_bound(mu, bias, q)
        delta = max(1e-5, 4 * float(eps.max()) + 1e-6)
        k = st.k
        if abs(st.cum[k - 1] - p) <= delta or (k >= 2 and abs(st.cum[k - 2] - p) <= delta):
            flags.append(f"step {s}: boundary cum={st.cum[k - 1]:.8f}")
        if k < n:
            a, b = st.order[k - 1], st.order[k]
            if abs(st.ehat[a] - st.ehat[b]) <= eps[a] + eps[b]:
                flags.append(f"step {s}: near-tie {st.ehat[a]:.8f} / {st.ehat[b]:.8f}")
    return flags


def gpu_planes_fn(tree, kv_head: int, levels: int):
    """planes(level, idx) over the planes the GPU router reads (the stored bf16/fp32 slopes, or the FP4
    router copies' exact values), upcast to fp64, read lazily."""
    cache: Dict[int, Tuple[torch.Tensor, torch.Tensor]] = {}

    def fn(level, idx):
        if level not in cache:
            mu, bias = tree.router_planes(level)
            cache[level] = (mu[kv_head].cpu(), bias[kv_head].cpu())
        mu, bias = cache[level]
        idx_t = torch.as_tensor(np.asarray(idx), dtype=torch.long)
        return f64(mu[idx_t]), f64(bias[idx_t])

    return fn


def compare_route(tree, Q: torch.Tensor, kept: torch.Tensor, cnt: torch.Tensor, p, n_tokens: int,
                  block: int, levels: int, group: int, heads=None) -> RouteReport:
    """Oracle routing on the GPU planes vs the GPU kept sets, for every (sequence, head)."""
    rep = RouteReport()
    B, Hq = Q.shape[0], Q.shape[1]
    kept = kept.cpu()
    cnt = cnt.cpu()
    planes_by_kv = {}
    for bb in range(B):
        for h in (range(Hq) if heads is None else heads):
            kvh = h // group
            if kvh not in planes_by_kv:
                planes_by_kv[kvh] = gpu_planes_fn(tree, kvh, levels)
            planes = planes_by_kv[kvh]
            q = f64(Q[bb, h])
            trace = zo.route(planes, q, p, n_tokens, block, levels)
            gk = sorted(kept[bb, h, : int(cnt[bb, h])].tolist())
            rep.heads += 1
            if gk == trace.leaves:
                rep.exact += 1
                continue
            flags = trace_flags(trace, planes, q, p, block)
            if flags:
                rep.flagged += 1
            else:
                rep.failures.append(
                    f"seq {bb} head {h}: gpu {len(gk)} blocks, oracle {len(trace.leaves)}; "
                    f"only-gpu {sorted(set(gk) - set(trace.leaves))[:8]} only-oracle "
                    f"{sorted(set(trace.leaves) - set(gk))[:8]}")
    return rep


# --------------------------------------------------------------------------- attend
def oracle_attend_on_sets(K: torch.Tensor, V: torch.Tensor, Q: torch.Tensor, kept: torch.Tensor, cnt: torch.Tensor,
                          n_tokens: int, block: int, group: int, heads=None) -> np.ndarray:
    """Oracle attention of every head over the GPU's kept blocks (+ sink + tail)."""
    B, Hq, d = Q.shape
    out = np.zeros((B, Hq, d))
    kept = kept.cpu()
    cnt = cnt.cpu()
    Kc = {}
    for bb in range(B):
        for h in (range(Hq) if heads is None else heads):
            kvh = h // group
            if kvh not in Kc:
                Kc[kvh] = (f64(K[kvh, :n_tokens]), f64(V[kvh, :n_tokens]))
            Kh, Vh = Kc[kvh]
            leaves = kept[bb, h, : int(cnt[bb, h])].tolist()
            toks = zo.attended_tokens(leaves, n_tokens, block)
            out[bb, h] = zo.attend(Kh, Vh, f64(Q[bb, h]), toks)
    return out


def assert_close_out(gpu: np.ndarray, ref: np.ndarray, atol: float, label: str = ""):
    err = np.abs(gpu - ref)
    assert np.all(err <= atol), f"{label} max abs err {err.max():.3e} > {atol:.1e}"
