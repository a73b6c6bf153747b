"""Seeded synthetic inputs for the ZHA decode path.

This module is the one place both sides of the parity check draw their
inputs from: the CUDA path (through the ctypes binding) and the fp64 oracle
receive the very same stored tensors.  It holds none of the method's
arithmetic - only random draws, casts and the shapes of the workloads.

The pages describe the workloads only by their geometry (block size, depth,
number of reference queries, threshold) and by the kind of data the method is
meant for: long documents whose attention mass concentrates on a few regions
(Zyphra blog, section "Why is efficient attention so hard?": the tokens that
hold a fixed share of attention grow sublinearly; tanhow.com summary, section
"How does ZHA compare with dense attention and MSA?": needle-style retrieval at
256K).  The evaluation suites named there are not available here; the
"topics" and "needles" below are synthetic stand-ins with the same structure
(contiguous segments about recurring topics, plus single planted keys that one
query head looks for).

Every tensor is drawn in fp32 from a seeded ``torch.Generator`` and then
rounded to nearest-even into the workload's storage dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict
from typing import Optional

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def levels_for_top(n_tokens: int, block: int, max_top: int = 4096) -> int:
    """Smallest depth L >= 1 whose top level holds at most ``max_top`` complete nodes."""
    L = 1
    while n_tokens // block ** L > max_top:
        L += 1
    return L


@dataclass
class Workload:
    """Geometry and generator settings of one decode workload."""

    name: str
    d: int
    n_q_heads: int
    n_kv_heads: int
    n_tokens: int
    block: int
    levels: int
    n_refs: int
    p: float
    batch: int
    dtype: str
    gen: str               # "needles" (tiny fp32 case) or "topics"
    seed: int
    n_query_sets: int = 16
    append: int = 0        # tokens appended after the initial build
    planes: str = "key"    # router planes: "key" (the stored slopes) or "fp4"
    # topic / needle constants (logit gains are in units of q.k/sqrt(d))
    n_topics: int = 64
    n_segments: int = 256
    topic_amp: float = 4.0     # |key/value shift along the topic direction|
    topic_gain: float = 9.0    # logits a matching topic adds to a key
    needle_gain: float = 18.0  # logits a head's needle adds for that head
    needle_query_amp: float = 0.0   # 0: sqrt(needle_gain*sqrt(d)), the same size as the key's needle shift
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def as_config(self) -> dict:
        c = asdict(self)
        c.pop("extra")
        return c


def workload(name: str, n_tokens: Optional[int] = None) -> Workload:
    """The named workloads (tiny fp32, deep and wide 256K trees, the deep tree at any size, the light
    sweep, build+batch)."""
    if name == "tiny4k_fp32":
        return Workload(name, d=64, n_q_heads=1, n_kv_heads=1, n_tokens=4096, block=4, levels=3,
                        n_refs=4, p=0.9, batch=8, dtype="f32", gen="needles", seed=0)
    if name == "deep256k_bf16":
        return Workload(name, d=128, n_q_heads=32, n_kv_heads=4, n_tokens=262144, block=4,
                        levels=6, n_refs=16, p=0.95, batch=1, dtype="bf16", gen="topics", seed=1)
    if name == "deep256k_fp4":  # the deep 256K tree, routed on FP4 router planes
        return Workload(name, d=128, n_q_heads=32, n_kv_heads=4, n_tokens=262144, block=4,
                        levels=6, n_refs=16, p=0.95, batch=1, dtype="bf16", gen="topics", seed=1, planes="fp4")
    if name == "deep_bf16":  # the deep tree's shape at another context length (profiling cases)
        n = n_tokens if n_tokens is not None else 262144
        return Workload(name, d=128, n_q_heads=32, n_kv_heads=4, n_tokens=n, block=4,
                        levels=levels_for_top(n, 4, max_top=64), n_refs=16, p=0.95, batch=1, dtype="bf16",
                        gen="topics", seed=1)
    if name == "wide256k_bf16":
        return Workload(name, d=128, n_q_heads=32, n_kv_heads=4, n_tokens=262144, block=256,
                        levels=1, n_refs=16, p=0.95, batch=1, dtype="bf16", gen="topics", seed=1)
    if name == "sweep_bf16":
        n = n_tokens if n_tokens is not None else 262144
        sweep = [32768, 65536, 131072, 262144, 524288, 1048576, 2097152, 4194304]
        seed = 3 + (sweep.index(n) if n in sweep else 0)
        return Workload(name, d=128, n_q_heads=32, n_kv_heads=4, n_tokens=n, block=8,
                        levels=levels_for_top(n, 8), n_refs=1, p=0.75, batch=1, dtype="bf16",
                        gen="topics", seed=seed)
    if name == "build1m_bf16":
        return Workload(name, d=128, n_q_heads=32, n_kv_heads=4, n_tokens=1048576, block=4,
                        levels=7, n_refs=16, p=0.95, batch=16, dtype="bf16", gen="topics", seed=4,
                        append=4096)
    raise KeyError(name)


def small_topics(n_tokens: int, *, d=128, n_q_heads=8, n_kv_heads=1, block=4, levels=3,
                 n_refs=4, p=0.95, batch=1, dtype="bf16", seed=11, n_topics=16,
                 n_segments=32) -> Workload:
    """A scaled-down topic workload for parity tests that the oracle finishes in seconds."""
    return Workload("small_topics", d=d, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads,
                    n_tokens=n_tokens, block=block, levels=levels, n_refs=n_refs, p=p,
                    batch=batch, dtype=dtype, gen="topics", seed=seed, n_topics=n_topics,
                    n_segments=n_segments)


@dataclass
class Inputs:
    """Stored tensors of one workload (all on the generator's device, storage dtype)."""

    K: torch.Tensor        # [Hkv, n_total, d]   keys (initial context followed by appended tokens)
    V: torch.Tensor        # [Hkv, n_total, d]
    refs: torch.Tensor     # [Hkv, R, d]         reference queries of each KV head's tree
    Q: torch.Tensor        # [n_query_sets, B, Hq, d]
    needle_pos: torch.Tensor  # positions of the planted needle keys
    meta: dict


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def generate(w: Workload, device: str = "cpu", n_total: Optional[int] = None) -> Inputs:
    """Draw the workload's tensors.

    The workload's own tokens (``n_tokens + append``) do not depend on
    ``n_total``: asking for fewer returns a prefix, asking for more draws the
    extra tokens from a second seeded stream (same distribution; under
    "topics" they continue the last segment's topic), so a benchmark's step
    count never changes the context it runs on.
    """
    n_base = w.n_tokens + w.append
    n_want = n_base if n_total is None else n_total
    n = n_base
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    f32 = torch.float32
    Hkv, Hq, d, G = w.n_kv_heads, w.n_q_heads, w.d, w.group
    meta: dict = {"seed": w.seed, "n_total": n}

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=device, dtype=f32)

    def randint(hi, shape):
        return torch.randint(0, hi, shape, generator=g, device=device)

    refs = randn(Hkv, w.n_refs, d)

    if w.gen == "needles":
        # Keys N(0, I/4), values N(0, I); 16 needle keys pointing along the queries.
        q = randn(w.batch, Hq, d)
        K = randn(Hkv, n, d) * 0.5
        V = randn(Hkv, n, d)
        n_needles = 16
        pos = (torch.randperm(max(n - 1, 1), generator=g, device=device)[:n_needles] + 1).clamp(max=n - 1)
        for m in range(min(n_needles, pos.numel())):
            i = m % w.batch
            qi = q[i, m % Hq]
            K[m % Hkv, pos[m]] = 3.0 * _unit(qi) * math.sqrt(d) + randn(d) * 0.5
        Q = torch.stack([q] + [randn(w.batch, Hq, d) for _ in range(w.n_query_sets - 1)])
        meta.update(needles=n_needles)
    elif w.gen == "topics":
        T = _unit(randn(Hkv, w.n_topics, d))                 # topic directions per KV head
        cuts = torch.randperm(max(n - 1, 1), generator=g, device=device)[: w.n_segments - 1] + 1
        cuts = torch.sort(cuts).values
        seg_topic = randint(w.n_topics, (w.n_segments,))
        seg_of = torch.zeros(n, dtype=torch.long, device=device)
        if n > 1:
            seg_of[cuts[cuts < n]] = 1
        seg_of = torch.cumsum(seg_of, 0).clamp(max=w.n_segments - 1)
        tok_topic = seg_topic[seg_of]                         # [n]
        K = randn(Hkv, n, d)
        V = randn(Hkv, n, d)
        for h in range(Hkv):
            shift = w.topic_amp * T[h, tok_topic]
            K[h] += shift
            V[h] += shift
        # needle directions: one per query head, planted once in its KV head's keys
        nu = _unit(randn(Hq, d))
        kappa = w.needle_query_amp or math.sqrt(w.needle_gain * math.sqrt(d))
        lam = w.needle_gain * math.sqrt(d) / kappa
        pos = torch.randperm(max(n - 1, 1), generator=g, device=device)[:Hq] + 1
        pos = pos.clamp(max=n - 1)
        for h in range(Hq):
            K[h // G, pos[h]] = randn(d) + lam * nu[h]
        beta = w.topic_gain * math.sqrt(d) / w.topic_amp
        sets = []
        for s in range(w.n_query_sets):
            z = randn(w.batch, Hq, d)
            topic = randint(w.n_topics, (w.batch, Hq))
            kvh = torch.arange(Hq, device=device) // G
            qs = z + beta * T[kvh[None, :].expand(w.batch, Hq), topic] + kappa * nu[None]
            sets.append(qs)
        Q = torch.stack(sets)
        meta.update(topic_beta=beta, needle_lambda=lam, needle_kappa=kappa, n_topics=w.n_topics,
                    n_segments=w.n_segments)
    else:
        raise KeyError(w.gen)

    if n_want < n:
        K, V = K[:, :n_want], V[:, :n_want]
    elif n_want > n:
        g2 = torch.Generator(device=device)
        g2.manual_seed(w.seed * 1000003 + 7919)
        m = n_want - n
        Kx = torch.randn(Hkv, m, d, generator=g2, device=device, dtype=f32)
        Vx = torch.randn(Hkv, m, d, generator=g2, device=device, dtype=f32)
        if w.gen == "needles":
            Kx *= 0.5
        else:
            last = int(tok_topic[-1])
            for h in range(Hkv):
                Kx[h] += w.topic_amp * T[h, last]
                Vx[h] += w.topic_amp * T[h, last]
        K, V = torch.cat([K, Kx], 1), torch.cat([V, Vx], 1)
    meta["n_total"] = n_want
    dt = DTYPES[w.dtype]
    return Inputs(K=K.to(dt).contiguous(), V=V.to(dt).contiguous(), refs=refs.to(dt).contiguous(),
                  Q=Q.to(dt).contiguous(), needle_pos=pos, meta=meta)


def random_tree_case(seed: int, *, n_tokens: int, d: int, n_q_heads: int, n_kv_heads: int,
                     n_refs: int, batch: int, dtype: str, key_scale: float = 1.0,
                     device: str = "cpu"):
    """Plain Gaussian K, V, refs and queries for small randomized parity cases."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    f32 = torch.float32
    K = torch.randn(n_kv_heads, n_tokens, d, generator=g, device=device, dtype=f32) * key_scale
    V = torch.randn(n_kv_heads, n_tokens, d, generator=g, device=device, dtype=f32)
    refs = torch.randn(n_kv_heads, n_refs, d, generator=g, device=device, dtype=f32)
    Q = torch.randn(batch, n_q_heads, d, generator=g, device=device, dtype=f32) * 1.5
    dt = DTYPES[dtype]
    return K.to(dt), V.to(dt), refs.to(dt), Q.to(dt)


def random_queries(seed: int, m: int, n_q_heads: int, d: int, dtype: str, topics_from: Optional[Inputs] = None):
    """m seeded query sets [m, Hq, d]: Gaussian, or, given a generated workload, drawn around its own query sets
    (a random one of them plus Gaussian noise of a quarter of their scale), so that routing stays selective."""
    g = torch.Generator()
    g.manual_seed(seed)
    if topics_from is None:
        Q = torch.randn(m, n_q_heads, d, generator=g) * 1.5
    else:
        base = topics_from.Q.reshape(-1, n_q_heads, d).float()
        pick = torch.randint(0, base.shape[0], (m,), generator=g)
        Q = base[pick] + 0.25 * base.std() * torch.randn(m, n_q_heads, d, generator=g)
    return Q.to(DTYPES[dtype])
