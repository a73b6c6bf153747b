"""Planted mistakes in the oracle (on the CPU) must each be caught by at least one pin.

Each mutation replaces one oracle function, for the duration of the test,
with a copy that carries a plausible slip (a dropped 1/sqrt(d), a wrong sign,
an unnormalised merge weight, a wrong tie rule, a forgotten sink ...).  The
pins of tests/oracle_pins.py then run against the mutated module; the test
passes only if some pin fails.
"""
import math

import numpy as np
import pytest

import oracle.zha_oracle as zo
from oracle_pins import ALL_PINS

_orig = {name: getattr(zo, name) for name in dir(zo) if not name.startswith("__")}


def _leaf_no_scale(blocks, refs):
    s = np.einsum("nkd,rd->nrk", blocks, refs)
    f = zo._logsumexp(s, 2)
    w = np.exp(s - f[:, :, None])
    mu = np.einsum("nrk,nkd->nrd", w, blocks)
    return zo.Planes(f, mu, f - np.einsum("nrd,rd->nr", mu, refs) / math.sqrt(blocks.shape[-1]))


def _leaf_bias_sign(blocks, refs):
    pl = _orig["leaf_planes"](blocks, refs)
    return zo.Planes(pl.f, pl.mu, 2 * pl.f - pl.bias)


def _leaf_mean_mu(blocks, refs):
    pl = _orig["leaf_planes"](blocks, refs)
    mu = np.repeat(blocks.mean(1)[:, None, :], refs.shape[0], axis=1)
    return zo.Planes(pl.f, mu, pl.f - np.einsum("nrd,rd->nr", mu, refs) / math.sqrt(blocks.shape[-1]))


def _merge_unnormalised(child, refs, block):
    d = refs.shape[-1]
    R = refs.shape[0]
    n = child.f.shape[0] // block
    fc = child.f[: n * block].reshape(n, block, R)
    muc = child.mu[: n * block].reshape(n, block, R, d)
    f = zo._logsumexp(fc, 1)
    a = np.exp(fc - fc.max(1, keepdims=True))          # missing normalisation
    mu = np.einsum("pcr,pcrd->prd", a, muc)
    return zo.Planes(f, mu, f - np.einsum("prd,rd->pr", mu, refs) / math.sqrt(d))


def _merge_plain_mean(child, refs, block):
    d = refs.shape[-1]
    R = refs.shape[0]
    n = child.f.shape[0] // block
    fc = child.f[: n * block].reshape(n, block, R)
    muc = child.mu[: n * block].reshape(n, block, R, d)
    f = zo._logsumexp(fc, 1)
    mu = muc.mean(1)
    return zo.Planes(f, mu, f - np.einsum("prd,rd->pr", mu, refs) / math.sqrt(d))


def _merge_max_f(child, refs, block):
    pl = _orig["merge_planes"](child, refs, block)
    R = refs.shape[0]
    n = child.f.shape[0] // block
    f = child.f[: n * block].reshape(n, block, R).max(1)
    return zo.Planes(f, pl.mu, f - (pl.f - pl.bias))


def _estimate_min(mu, bias, q):
    return np.min(bias + np.einsum("nrd,d->nr", mu, q) / math.sqrt(mu.shape[-1]), axis=1)


def _estimate_no_scale(mu, bias, q):
    return np.max(bias + np.einsum("nrd,d->nr", mu, q), axis=1)


def _estimate_no_bias(mu, bias, q):
    return np.max(np.einsum("nrd,d->nr", mu, q) / math.sqrt(mu.shape[-1]), axis=1)


def _top_p_strict(ehat, order, p):
    m = ehat.max()
    pi = np.exp(ehat - m)
    pi /= pi.sum()
    cum = np.cumsum(pi[order])
    if p >= 1:
        return len(order), cum
    hit = np.nonzero(cum > p)[0]                         # ">" instead of ">="
    return (int(hit[0]) + 1 if hit.size else len(order)), cum


def _top_p_one_short(ehat, order, p):
    k, cum = _orig["top_p_count"](ehat, order, p)
    return max(1, k - 1), cum


def _top_p_one_extra(ehat, order, p):
    k, cum = _orig["top_p_count"](ehat, order, p)
    return min(len(order), k + 1), cum


def _children_off_by_one(node, block):
    level, idx = node
    return [(level - 1, block * idx + c + 1) for c in range(block)]


def _roots_top_only(n_tokens, block, levels):
    n = zo.level_counts(n_tokens, block, levels)
    return [(levels, i) for i in range(n[levels])]


def _attended_no_sink(leaves, n_tokens, block):
    n1 = n_tokens // block
    parts = [np.arange(i * block, (i + 1) * block) for i in leaves] + [np.arange(n1 * block, n_tokens)]
    return np.unique(np.concatenate(parts + [np.zeros(0)]).astype(np.int64))


def _attended_no_tail(leaves, n_tokens, block):
    parts = [np.arange(i * block, (i + 1) * block) for i in leaves] + [np.array([0])]
    return np.unique(np.concatenate(parts).astype(np.int64))


def _attend_no_scale(K, V, q, tokens):
    s = K[tokens] @ q
    w = np.exp(s - s.max())
    return (w / w.sum()) @ V[tokens]


def _e2m1_ties_up(y):
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    idx = np.zeros(a.shape, dtype=np.uint8)
    for i in range(1, 8):
        mid = (zo.E2M1_VALUES[i - 1] + zo.E2M1_VALUES[i]) / 2
        idx = np.where(a >= mid, np.uint8(i), idx)       # ties away from zero
    return np.where(idx == 0, 0, idx | np.where(y < 0, 8, 0)).astype(np.uint8)


def _quantize_scale_amax4(mu):
    m32 = np.asarray(mu, dtype=np.float32)
    g = m32.reshape(*m32.shape[:-1], m32.shape[-1] // 16, 16)
    amax = np.abs(g).max(axis=-1)
    sval, sbits = zo.e4m3_nearest((amax / np.float32(4)).astype(np.float32))
    s32 = sval.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (g / s32[..., None]).astype(np.float32)
    codes = np.where(s32[..., None] > 0, zo.e2m1_code(y), 0).astype(np.uint8)
    return codes.reshape(m32.shape), sbits


def _step_threshold_first(p, s):
    return float(p) if np.ndim(p) == 0 else float(p[0])


def _route_ties_high(planes, q, p, n_tokens, block, levels):
    trace = zo.RouteTrace()
    cand = zo.forest_roots(n_tokens, block, levels)
    s = 0
    while cand:
        lv = np.array([c[0] for c in cand])
        ix = np.array([c[1] for c in cand])
        ehat = np.empty(len(cand))
        for level in np.unique(lv):
            sel = np.nonzero(lv == level)[0]
            mu, bias = planes(int(level), ix[sel])
            ehat[sel] = zo.estimate(mu, bias, q)
        start = ix * np.array([block ** int(v) for v in lv])
        order = np.lexsort((-start, -ehat))            # higher start first on ties
        ps = zo.step_threshold(p, s)
        k, cum = zo.top_p_count(ehat, order, ps)
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


def _retained_without_last(trace):
    return float(np.prod([st.cum[st.k - 1] for st in trace.steps[:-1]]))


def _retained_one_past(trace):
    return float(np.prod([st.cum[min(st.k, len(st.cum) - 1)] for st in trace.steps]))


MUTATIONS = {
    "leaf scores without 1/sqrt(d)": ("leaf_planes", _leaf_no_scale),
    "leaf intercept sign flipped": ("leaf_planes", _leaf_bias_sign),
    "leaf mu as plain mean": ("leaf_planes", _leaf_mean_mu),
    "merge weights unnormalised": ("merge_planes", _merge_unnormalised),
    "merge mu as plain mean": ("merge_planes", _merge_plain_mean),
    "merge f as max instead of logsumexp": ("merge_planes", _merge_max_f),
    "estimate takes min over planes": ("estimate", _estimate_min),
    "estimate without 1/sqrt(d)": ("estimate", _estimate_no_scale),
    "estimate without intercept": ("estimate", _estimate_no_bias),
    "cut needs mass > p": ("top_p_count", _top_p_strict),
    "cut one short": ("top_p_count", _top_p_one_short),
    "cut one extra": ("top_p_count", _top_p_one_extra),
    "children index off by one": ("children", _children_off_by_one),
    "roots without partial subtrees": ("forest_roots", _roots_top_only),
    "sink forgotten": ("attended_tokens", _attended_no_sink),
    "tail forgotten": ("attended_tokens", _attended_no_tail),
    "attention without 1/sqrt(d)": ("attend", _attend_no_scale),
    "ties to the higher start": ("route", _route_ties_high),
    "step thresholds ignored after the first": ("step_threshold", _step_threshold_first),
    "e2m1 ties away from zero": ("e2m1_code", _e2m1_ties_up),
    "fp4 scale from amax / 4": ("quantize_fp4", _quantize_scale_amax4),
    "retained mass without the last step": ("retained_mass", _retained_without_last),
    "retained mass one past the cut": ("retained_mass", _retained_one_past),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(zo, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(zo)
        except (AssertionError, IndexError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake: {name}"
