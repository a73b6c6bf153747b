"""Comparison helpers for the GPU parity tests (test infrastructure).

The CUDA path and the fp64 oracle receive the same stored tensors; these
helpers run the oracle on them and compare, stage by stage:

  build   GPU planes vs oracle planes (tolerances derived from fp32 arithmetic
          on the stored inputs, plus the bf16 rounding of the stored slopes);
  route   the oracle's routing run on the GPU-stored planes must keep the same
          level-1 blocks as the GPU; a head may differ only if its GPU set is
          exactly the oracle's route with one (or two) of the decisions that
          fp32 may take the other way flipped: a cut whose cumulative mass lies
          within delta of p (one candidate more or fewer kept), or a near-tie
          straddling the cut (estimates closer than the fp32 error bound of the
          GPU estimate; the two swapped) - those heads are counted and
          reported, separately for cuts within 1e-5 of p and the rest;
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
    flagged: int = 0          # heads whose GPU set is an excused alternative of the oracle's route
    flagged_tight: int = 0    # ... excused by a cut whose cumulative mass lies within 1e-5 of p
    flagged_wide: int = 0     # ... excused only by the widened fp32 bound or a near-tie across the cut
    failures: List[str] = field(default_factory=list)

    def summary(self) -> Dict[str, int]:
        return {"heads": self.heads, "exact": self.exact, "flagged": self.flagged,
                "flagged_tight": self.flagged_tight, "flagged_wide": self.flagged_wide,
                "failed": len(self.failures)}


def ehat_error_bound(mu: np.ndarray, bias: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Bound on |e_gpu - e| for fp32 evaluation of max_j (b_j + q.mu_j/sqrt d) on the stored planes."""
    d = mu.shape[-1]
    mag = np.einsum("nrd,d->nr", np.abs(mu), np.abs(q)) / math.sqrt(d) + np.abs(bias)
    return (d + 8) * U32 * mag.max(axis=1) + 1e-7


@dataclass
class Flag:
    """A decision of the oracle's route that fp32 arithmetic may legitimately take the other way."""

    step: int
    kind: str      # "keep_more" (cut mass just reached p), "keep_less" (one fewer just missed), "swap" (tie)
    tight: bool    # within 1e-5 of p (the stated boundary), not only within the widened fp32 bound
    text: str


def step_flags(s: int, st, planes, q: np.ndarray) -> List[Flag]:
    """Boundary and near-tie cases of one routing step of an oracle trace."""
    p = st.p
    if p >= 1:
        return []
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
    out = []
    if abs(st.cum[k - 1] - p) <= delta and k < n:
        out.append(Flag(s, "keep_more", abs(st.cum[k - 1] - p) <= 1e-5, f"step {s}: boundary cum={st.cum[k - 1]:.8f}"))
    if k >= 2 and abs(st.cum[k - 2] - p) <= delta:
        out.append(Flag(s, "keep_less", abs(st.cum[k - 2] - p) <= 1e-5, f"step {s}: boundary cum={st.cum[k - 2]:.8f}"))
    if k < n:
        a, b = st.order[k - 1], st.order[k]
        if abs(st.ehat[a] - st.ehat[b]) <= eps[a] + eps[b]:
            out.append(Flag(s, "swap", False, f"step {s}: near-tie {st.ehat[a]:.8f} / {st.ehat[b]:.8f}"))
    return out


def trace_flags(trace: zo.RouteTrace, planes, q: np.ndarray, p, block: int) -> List[str]:
    """Boundary / near-tie cases along the oracle's path (the places where fp32 and fp64 may differ)."""
    return [f.text for s, st in enumerate(trace.steps) for f in step_flags(s, st, planes, q)]


def route_overridden(planes, q: np.ndarray, p, n_tokens: int, block: int, levels: int,
                     overrides: Dict[int, str]) -> zo.RouteTrace:
    """The oracle's route with the decisions of some steps taken the other way: "keep_more" keeps one more
    candidate, "keep_less" one fewer, "swap" exchanges the last kept candidate with the first dropped one.
    Built from the oracle's own primitives (candidates, estimates, order, top-p count, children)."""
    trace = zo.RouteTrace()
    cand = zo.forest_roots(n_tokens, block, levels)
    s = 0
    while cand:
        ehat = np.empty(len(cand))
        lv = np.array([c[0] for c in cand])
        ix = np.array([c[1] for c in cand])
        for level in np.unique(lv):
            sel = np.nonzero(lv == level)[0]
            mu, bias = planes(int(level), ix[sel])
            ehat[sel] = zo.estimate(mu, bias, q)
        start = ix * np.array([block ** int(v) for v in lv])
        order = np.lexsort((start, -ehat))
        ps = zo.step_threshold(p, s)
        k, cum = zo.top_p_count(ehat, order, ps)
        ov = overrides.get(s)
        if ov == "keep_more":
            k = min(k + 1, len(order))
        elif ov == "keep_less":
            k = max(k - 1, 1)
        elif ov == "swap" and k < len(order):
            order = order.copy()
            order[k - 1], order[k] = order[k], order[k - 1]
        trace.steps.append(zo.RouteStep(cand, ehat, order, cum, k, ps))
        s += 1
        nxt = []
        for j in order[:k]:
            node = cand[j]
            if node[0] == 1:
                trace.leaves.append(node[1])
            else:
                nxt += zo.children(node, block)
        cand = nxt
    trace.leaves.sort()
    return trace


def excused(gk: List[int], trace: zo.RouteTrace, planes, q: np.ndarray, p, n_tokens: int, block: int,
            levels: int, depth: int = 2):
    """Whether the GPU's kept blocks equal the oracle's route with at most ``depth`` flagged decisions taken
    the other way (each flag found on the path being followed).  Returns the flags used, or None."""
    def search(tr, overrides, used):
        if tr.leaves == gk:
            return used
        if len(used) >= depth:
            return None
        last = max(overrides) if overrides else -1
        for s, st in enumerate(tr.steps):
            if s <= last:
                continue
            for f in step_flags(s, st, planes, q):
                ov = dict(overrides)
                ov[s] = f.kind
                alt = route_overridden(planes, q, p, n_tokens, block, levels, ov)
                r = search(alt, ov, used + [f])
                if r is not None:
                    return r
        return None

    return search(trace, {}, [])


def gpu_planes_fn(tree, kv_head: int, levels: int):
    """planes(level, idx) over the planes the GPU router reads, upcast to fp64, read lazily: the stored
    bf16/fp32 slopes, or, with FP4 router planes, the raw codes and scales the library stores, turned into
    slopes by the oracle's own decoder (``oracle.dequantize_fp4``)."""
    cache: Dict[int, Tuple[np.ndarray, np.ndarray]] = {}
    fp4 = tree.cfg.planes == 1

    def fn(level, idx):
        if level not in cache:
            if fp4:
                codes, scales, bias = tree.fp4_records(level)
                mu = zo.dequantize_fp4(codes[kv_head].cpu().numpy(), scales[kv_head].cpu().numpy())
                cache[level] = (mu, f64(bias[kv_head]))
            else:
                mu, bias, _ = tree.level_planes(level)
                cache[level] = (f64(mu[kv_head]), f64(bias[kv_head]))
        mu, bias = cache[level]
        ix = np.asarray(idx, dtype=np.int64)
        return mu[ix], bias[ix]

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
            used = excused(gk, trace, planes, q, p, n_tokens, block, levels)
            if used is not None:
                rep.flagged += 1
                if all(f.tight for f in used):
                    rep.flagged_tight += 1
                else:
                    rep.flagged_wide += 1
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


# --------------------------------------------------------------------------- end to end
@dataclass
class EndToEnd:
    """GPU decode vs the oracle's own decode (its tree built in fp64 from the raw keys): kept-set Jaccard per
    head and output error.  The GPU routes on planes stored in the element type, so where bf16 rounding of
    the slopes moves a cut the sets legitimately differ; heads whose sets match must agree within the
    output tolerance."""

    jaccard: List[float] = field(default_factory=list)
    err: List[float] = field(default_factory=list)
    err_matched: List[float] = field(default_factory=list)
    retained: List[float] = field(default_factory=list)  # the oracle route's retained estimated mass per head

    def summary(self) -> Dict[str, float]:
        return {"heads": len(self.jaccard), "jaccard_mean": float(np.mean(self.jaccard)) if self.jaccard else 1.0,
                "jaccard_min": float(np.min(self.jaccard)) if self.jaccard else 1.0,
                "matched_sets": len(self.err_matched),
                "max_abs_err_matched": float(np.max(self.err_matched)) if self.err_matched else 0.0,
                "max_abs_err": float(np.max(self.err)) if self.err else 0.0,
                "retained_mass_mean": float(np.mean(self.retained)) if self.retained else 1.0,
                "retained_mass_min": float(np.min(self.retained)) if self.retained else 1.0}


def end_to_end(K: torch.Tensor, V: torch.Tensor, refs: torch.Tensor, Q: torch.Tensor, O: torch.Tensor,
               kept: torch.Tensor, cnt: torch.Tensor, n_tokens: int, block: int, levels: int, p, group: int,
               kv_head: int, seqs, oracle_tree=None) -> EndToEnd:
    """Route and attend the query heads of one KV head with the oracle's own tree (built here from the raw
    keys unless given) and compare with the GPU's kept blocks and outputs."""
    Kh = f64(K[kv_head, :n_tokens])
    Vh = f64(V[kv_head, :n_tokens])
    tree = oracle_tree if oracle_tree is not None else zo.build_tree(Kh, f64(refs[kv_head]), n_tokens, block, levels)
    pfn = zo.tree_planes_fn(tree)
    kept, cnt, O = kept.cpu(), cnt.cpu(), O.cpu()
    rep = EndToEnd()
    for bb in seqs:
        for h in range(kv_head * group, (kv_head + 1) * group):
            o_ref, tr = zo.decode_head(Kh, Vh, pfn, f64(Q[bb, h]), p, n_tokens, block, levels)
            rep.retained.append(zo.retained_mass(tr))
            g = set(kept[bb, h, : int(cnt[bb, h])].tolist())
            o = set(tr.leaves)
            rep.jaccard.append(len(g & o) / max(1, len(g | o)))
            e = float(np.abs(O[bb, h].numpy().astype(np.float64) - o_ref).max())
            rep.err.append(e)
            if g == o:
                rep.err_matched.append(e)
    return rep
