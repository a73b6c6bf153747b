"""zha_dense_decode_noalloc: dense decode with the library's fixed scratch instead of caller memory.

Some callers cannot allocate device memory once they are running - a serving
loop with a fixed, pre-partitioned memory budget, or a host framework that owns
the device arena.  This entry point serves them with a static array inside
libzha.so; here it is called through the C ABI and checked against the
ordinary entry point (caller-provided scratch) on two calls in a row.
"""
import ctypes

import pytest
import torch

from synth.workloads import random_tree_case

pytestmark = pytest.mark.gpu


def _call_noalloc(z, cfg, K, V, n, Q, O):
    L = z.lib()
    return L.zha_dense_decode_noalloc(ctypes.byref(cfg), K.data_ptr(), V.data_ptr(), K.shape[1], n, Q.data_ptr(),
                                      O.data_ptr(), Q.shape[0], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,d,hq,hkv,n,B", [("bf16", 128, 32, 4, 5003, 1), ("bf16", 128, 32, 4, 20000, 4),
                                                ("f32", 64, 4, 2, 777, 2)])
def test_noalloc_matches_caller_scratch(dtype, d, hq, hkv, n, B):
    import tree_indexed_sparse_03_b200 as z
    K, V, _, Q = random_tree_case(31, n_tokens=n, d=d, n_q_heads=hq, n_kv_heads=hkv, n_refs=1, batch=B, dtype=dtype)
    Kc, Vc, Qc = K.cuda(), V.cuda(), Q.cuda()
    cfg = z.make_config(d=d, n_q_heads=hq, n_kv_heads=hkv, block=4, levels=1, n_refs=1, p=1.0, dtype=dtype,
                        capacity=n, max_batch=B)
    ref = z.DenseDecoder(cfg, B, n)(Kc, Vc, n, Qc)
    torch.cuda.synchronize()
    # the same kernels with the same split plan run on both paths; only where the partials live differs,
    # so the outputs must be identical bit for bit (the oracle comparison is test_dense_decode's)
    for _ in range(2):
        O = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device="cuda")
        assert _call_noalloc(z, cfg, Kc, Vc, n, Qc, O) == 0, z.lib().zha_last_error()
        torch.cuda.synchronize()
        assert torch.equal(O, ref)


def test_noalloc_rejects_requests_beyond_the_fixed_scratch():
    import tree_indexed_sparse_03_b200 as z
    from tree_indexed_sparse_03_b200 import zha as zb
    # 1024 query heads x 148 splits x 130 floats is far beyond 2^20 floats
    cfg = z.make_config(d=128, n_q_heads=1024, n_kv_heads=1, block=4, levels=1, n_refs=1, p=1.0, dtype="bf16",
                        capacity=1 << 20, max_batch=1)
    K = torch.zeros(1, 1 << 16, 128, dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros(1, 1024, 128, dtype=torch.bfloat16, device="cuda")
    O = torch.zeros(1, 1024, 128, dtype=torch.float32, device="cuda")
    rc = _call_noalloc(z, cfg, K, K, 1 << 16, Q, O)
    assert rc == zb.ZHA_ERR_CAPACITY
    assert b"fixed scratch" in z.lib().zha_last_error()
