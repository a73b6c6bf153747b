"""Parity at the other full sizes: the build + batched decode workload (N = 1M, block append of 4096
tokens, batch 16) and the light sweep's largest point (N = 4M, b = 8, R = 1, p = 0.75), each in the
configuration the benchmark times.

As at 256K, the build is checked on sampled nodes against planes the oracle computes straight from the
raw keys they cover, routing on every head (the oracle's route on the GPU-stored planes), and attention on
sampled heads with the oracle reading only the attended keys.
"""
import numpy as np
import pytest
import torch

import oracle.zha_oracle as zo
from parity_helpers import assert_close_out, compare_planes, compare_route, end_to_end, f64, p32
from synth.workloads import generate, workload

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import tree_indexed_sparse_03_b200 as z


def _host_memory_gb() -> float:
    try:
        import psutil
        return psutil.virtual_memory().available / 2 ** 30
    except Exception:  # noqa: BLE001
        return 0.0


def _tree(w, inp, n_build, cap):
    cfg = z.make_config(d=w.d, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, block=w.block, levels=w.levels,
                        n_refs=w.n_refs, p=w.p, dtype=w.dtype, capacity=cap, max_batch=w.batch)
    K = torch.zeros(w.n_kv_heads, cap, w.d, dtype=inp.K.dtype, device="cuda")
    V = torch.zeros_like(K)
    K[:, :n_build] = inp.K[:, :n_build].cuda()
    V[:, :n_build] = inp.V[:, :n_build].cuda()
    tree = z.ZhaTree(cfg, K, V, inp.refs.cuda().contiguous())
    tree.build(n_build)
    torch.cuda.synchronize()
    tree.status()
    return tree


def _check_nodes(w, inp, tree, kvh, per_level, seed):
    rng = np.random.default_rng(seed)
    n = tree.size
    Kh = f64(inp.K[kvh, :n])
    refs = f64(inp.refs[kvh])
    for level in range(1, w.levels + 1):
        count = n // w.block ** level
        if count == 0:
            continue
        idx = np.unique(np.concatenate([[0, count - 1], rng.integers(0, count, per_level)]))
        mu, bias, f = tree.level_planes(level)
        direct = [zo.node_planes_direct(Kh, refs, (level, int(i)), w.block) for i in idx]
        orc = zo.Planes(np.concatenate([p.f for p in direct]), np.concatenate([p.mu for p in direct]),
                        np.concatenate([p.bias for p in direct]))
        it = torch.as_tensor(idx, dtype=torch.long)
        compare_planes(f64(mu[kvh].cpu()[it]), f64(bias[kvh].cpu()[it]), f64(f[kvh].cpu()[it]), orc, w.dtype, refs,
                       label=f"kv{kvh} level {level}")


def _check_decode(w, inp, tree, Q, attend_heads):
    O_bench = tree.decode(Q)
    O, (kept, cnt), stats = tree.decode(Q, want_kept=True, want_stats=True)
    torch.cuda.synchronize()
    tree.status()
    assert torch.equal(O_bench, O)
    n = tree.size
    group = w.n_q_heads // w.n_kv_heads
    rep = compare_route(tree, Q, kept, cnt, p32(w.p), n, w.block, w.levels, group)
    print(f"route at N={n}: {rep.summary()}")
    assert not rep.failures, "\n".join(rep.failures[:5])
    assert rep.flagged <= max(1, rep.heads // 64), rep.summary()
    kept, cnt = kept.cpu(), cnt.cpu()
    vmax = 0.0
    for bb, h in attend_heads:
        kvh = h // group
        toks = zo.attended_tokens(kept[bb, h, : int(cnt[bb, h])].tolist(), n, w.block)
        it = torch.as_tensor(np.asarray(toks), dtype=torch.long)
        Ks, Vs = f64(inp.K[kvh][it]), f64(inp.V[kvh][it])
        vmax = max(vmax, float(np.abs(Vs).max()))
        ref = zo.attend(Ks, Vs, f64(Q[bb, h]), np.arange(len(toks)))
        assert_close_out(O[bb, h].cpu().numpy()[None], ref[None], 2e-5 * float(inp.V[kvh].abs().max()) + 1e-6,
                         f"attend seq {bb} head {h}")
    return rep, O, kept, cnt


def test_build_append_batched_decode_1m():
    w = workload("build1m_bf16")  # N = 1M built, then the 4096-token block append, batch 16
    n_build, n0 = w.n_tokens, w.n_tokens + w.append
    inp = generate(w)
    tree = _tree(w, inp, n_build, n0)
    tree.append(inp.K[:, n_build:n0].contiguous().cuda(), inp.V[:, n_build:n0].contiguous().cuda())
    torch.cuda.synchronize()
    tree.status()
    assert tree.size == n0
    _check_nodes(w, inp, tree, kvh=1, per_level=12, seed=3)
    Q = inp.Q[0].cuda()
    heads = [(bb, h) for bb in (0, 7, 15) for h in (0, 9, 18, 31)]
    rep, O, kept, cnt = _check_decode(w, inp, tree, Q, heads)
    print(f"1M batch 16: {rep.exact}/{rep.heads} exact, {rep.flagged} flagged")
    # the whole path against the oracle's own tree of KV head 0 (fp64 planes from the raw keys, including the
    # appended block), for three of the sixteen sequences
    e2e = end_to_end(inp.K, inp.V, inp.refs, inp.Q[0], O, kept, cnt, n0, w.block, w.levels, p32(w.p), w.group, 0,
                     (0, 7, 15))
    s = e2e.summary()
    print(f"end to end 1M: {s}")
    assert s["jaccard_mean"] >= 0.97 and s["jaccard_min"] >= 0.85, s
    assert s["max_abs_err_matched"] <= 2e-2 and s["max_abs_err"] <= 0.25, s


@pytest.mark.skipif(not torch.cuda.is_available() or _host_memory_gb() < 48,
                    reason="the 4M-token workload needs about 30 GB of host memory to generate")
def test_light_sweep_4m():
    w = workload("sweep_bf16", 4194304)
    inp = generate(w)
    tree = _tree(w, inp, w.n_tokens, w.n_tokens)
    _check_nodes(w, inp, tree, kvh=0, per_level=8, seed=5)
    Q = inp.Q[0].cuda()
    rep, *_ = _check_decode(w, inp, tree, Q, [(0, h) for h in (0, 3, 5, 8)])
    print(f"4M sweep: {rep.exact}/{rep.heads} exact, {rep.flagged} flagged")
