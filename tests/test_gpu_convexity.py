"""The GPU-stored planes against the convexity bound.

Each stored node holds tangent planes of its log attention mass f_node(q) = log sum_k exp(q.k / sqrt d), a
convex function of q, at the reference queries r_j (tanhow.com summary, section "How does ZHA's tree indexer
work? / Building the tree"; Zyphra blog, section "Building the tree").  So the estimate
e(q) = max_j (b_j + q.mu_j / sqrt d) lies below f_node(q) for every q and touches it at each r_j.  Checked
on the planes the GPU build stored, against f_node computed in fp64 from the raw keys each node covers, for
sampled nodes of every level and queries near the references and far from them:
  fp32 configurations - e(q) <= f_node(q) within the fp32 rounding of the stored planes, and e(r_j) = f(r_j);
  bf16 configurations - the slopes are stored rounded to bf16, so e(q) may exceed f_node(q) by at most what
  that rounding can move q.mu_j / sqrt d; the share of (node, query) pairs above f_node and the largest excess
  are printed (the report) and the excess is asserted within that bound.
"""
import math

import numpy as np
import pytest
import torch

import oracle.zha_oracle as zo
from parity_helpers import bf16_ulp, f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import tree_indexed_sparse_03_b200 as z


def _tree(dtype, n, d, R, block, levels, seed):
    g = torch.Generator().manual_seed(seed)
    K = (torch.randn(1, n, d, generator=g) * 0.7).to(dtype)
    V = torch.randn(1, n, d, generator=g).to(dtype)
    refs = torch.randn(1, R, d, generator=g).to(dtype)
    cfg = z.make_config(d=d, n_q_heads=1, n_kv_heads=1, block=block, levels=levels, n_refs=R, p=0.9,
                        dtype="bf16" if dtype == torch.bfloat16 else "f32", capacity=n, max_batch=1)
    tree = z.ZhaTree(cfg, K.cuda(), V.cuda(), refs.cuda().contiguous())
    tree.build(n)
    torch.cuda.synchronize()
    tree.status()
    return tree, f64(K[0]), f64(refs[0])


@pytest.mark.parametrize("dtype,d,R", [(torch.float32, 64, 4), (torch.bfloat16, 128, 16)])
def test_stored_planes_lie_below_log_mass(dtype, d, R):
    n, block, levels = 4096, 4, 3
    tree, K, refs = _tree(dtype, n, d, R, block, levels, seed=7)
    rng = np.random.default_rng(11)
    pairs, above, worst, worst_bound = 0, 0, -np.inf, 0.0
    for level in range(1, levels + 1):
        count = n // block ** level
        mu_t, bias_t, _ = tree.level_planes(level)
        idx = np.unique(np.concatenate([[0, count - 1], rng.integers(0, count, 24)]))
        mu = f64(mu_t[0].cpu()[torch.as_tensor(idx)])        # [m, R, d]
        bias = f64(bias_t[0].cpu()[torch.as_tensor(idx)])    # [m, R]
        # queries: each reference (the tangent points), references plus noise, and draws far from them
        qs = [refs[j] for j in range(R)]
        qs += [refs[rng.integers(R)] + rng.normal(size=d) * 0.3 for _ in range(8)]
        qs += [rng.normal(size=d) * s for s in (0.5, 1.0, 2.0, 4.0)]
        for qi, q in enumerate(qs):
            e = zo.estimate(mu, bias, q)
            f = np.array([zo.log_mass(K, (level, int(i)), q, block) for i in idx])
            terms = np.abs(bias) + np.abs(np.einsum("mrd,d->mr", mu, q)) / math.sqrt(d)
            # fp32 rounding of the stored planes (bias and slopes computed in fp32 from the same keys)
            tol32 = 2e-5 * (terms.max(1) + np.abs(f) + 1.0)
            if dtype == torch.bfloat16:  # the slopes are stored rounded to bf16 (half an ulp each)
                shift = np.einsum("mrd,d->mr", bf16_ulp(mu) / 2, np.abs(q)) / math.sqrt(d)
                bound = tol32 + shift.max(1)
            else:
                bound = tol32
            excess = e - f
            pairs += excess.size
            above += int(np.sum(excess > 0))
            k = int(np.argmax(excess - bound))
            if excess[k] - bound[k] > worst - worst_bound:
                worst, worst_bound = float(excess[k]), float(bound[k])
            assert np.all(excess <= bound), (level, qi, float(excess.max()), float(bound[np.argmax(excess)]))
            if qi < R:  # at a tangent point the estimate equals the log mass
                assert np.all(np.abs(excess) <= bound), (level, qi, float(np.abs(excess).max()))
    print(f"convexity {dtype}: {above}/{pairs} (node, query) pairs above f_node; largest excess {worst:.3e} "
          f"(allowed there {worst_bound:.3e})")
