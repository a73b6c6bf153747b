"""ctypes binding of libzha.so (include/zha.h): argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; this module
allocates the caller-owned device buffers with PyTorch, passes raw pointers
and the current CUDA stream, and turns error codes into exceptions.  There is
no fallback: if libzha.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzha.so")

ZHA_OK, ZHA_ERR_INVALID, ZHA_ERR_CAPACITY, ZHA_ERR_UNSUPPORTED, ZHA_ERR_CUDA, ZHA_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
ZHA_F32, ZHA_BF16 = 0, 1
ZHA_PLANES_KEY, ZHA_PLANES_FP4 = 0, 1
PLANES_CODE = {"key": ZHA_PLANES_KEY, "fp4": ZHA_PLANES_FP4}
STAT_NODES_SCORED, STAT_LEAVES_KEPT, STAT_KEYS, STAT_STEPS, STAT_COUNT = 0, 1, 2, 3, 4

TORCH_DTYPE = {ZHA_F32: torch.float32, ZHA_BF16: torch.bfloat16}
DTYPE_CODE = {"f32": ZHA_F32, "bf16": ZHA_BF16, torch.float32: ZHA_F32, torch.bfloat16: ZHA_BF16}

# every function the header declares, with its ctypes signature
_c = ctypes
_SIGS = {
    "zha_tree_bytes": (_c.c_int, [_c.c_void_p, _c.POINTER(_c.c_size_t), _c.POINTER(_c.c_size_t)]),
    "zha_tree_layout": (_c.c_int, [_c.c_void_p, _c.c_int32, _c.POINTER(_c.c_size_t), _c.POINTER(_c.c_size_t),
                                   _c.POINTER(_c.c_int64), _c.POINTER(_c.c_size_t)]),
    "zha_tree_layout_fp4": (_c.c_int, [_c.c_void_p, _c.c_int32, _c.POINTER(_c.c_size_t), _c.POINTER(_c.c_size_t)]),
    "zha_tree_create": (_c.c_int, [_c.c_void_p] * 6 + [_c.POINTER(_c.c_void_p)]),
    "zha_tree_build": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_void_p]),
    "zha_tree_append": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "zha_tree_size": (_c.c_int64, [_c.c_void_p]),
    "zha_decode": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_void_p, _c.c_void_p,
                              _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "zha_route_multi": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_void_p, _c.c_void_p,
                                   _c.c_void_p]),
    "zha_decode_step_host": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                        _c.c_int32, _c.c_void_p]),
    "zha_dense_scratch_bytes": (_c.c_size_t, [_c.c_void_p, _c.c_int32, _c.c_int64]),
    "zha_dense_decode": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p,
                                    _c.c_void_p, _c.c_int32, _c.c_void_p, _c.c_void_p]),
    "zha_dense_decode_noalloc": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64,
                                            _c.c_void_p, _c.c_void_p, _c.c_int32, _c.c_void_p]),
    "zha_tree_status": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "zha_tree_set_step_p": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int32]),
    "zha_tree_destroy": (None, [_c.c_void_p]),
    "zha_last_error": (_c.c_char_p, []),
    "zha_launch_count": (_c.c_uint64, []),
}

_lib = None


class ZhaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"zha error {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libzha.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m tree_indexed_sparse_03_b200.build_lib`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != ZHA_OK:
        raise ZhaError(rc, lib().zha_last_error().decode())


class ZhaConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("block", ctypes.c_int32), ("levels", ctypes.c_int32), ("n_refs", ctypes.c_int32),
                ("p", ctypes.c_float), ("dtype", ctypes.c_int32), ("capacity", ctypes.c_int64),
                ("max_batch", ctypes.c_int32), ("planes", ctypes.c_int32)]


def make_config(*, d: int, n_q_heads: int, n_kv_heads: int, block: int, levels: int, n_refs: int, p: float,
                dtype, capacity: int, max_batch: int = 1, planes: str = "key") -> ZhaConfig:
    return ZhaConfig(d, n_q_heads, n_kv_heads, block, levels, n_refs, p, DTYPE_CODE[dtype], capacity, max_batch,
                     PLANES_CODE[planes])


def _stream(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def tree_bytes(cfg: ZhaConfig) -> Tuple[int, int]:
    nb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().zha_tree_bytes(ctypes.byref(cfg), ctypes.byref(nb), ctypes.byref(sb)))
    return nb.value, sb.value


@dataclass
class LevelLayout:
    rec_offset: int
    f_offset: int
    cap_nodes: int
    rec_bytes: int


def tree_layout(cfg: ZhaConfig, level: int) -> LevelLayout:
    ro, fo, rb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    cap = ctypes.c_int64()
    _check(lib().zha_tree_layout(ctypes.byref(cfg), level, ctypes.byref(ro), ctypes.byref(fo), ctypes.byref(cap),
                                 ctypes.byref(rb)))
    return LevelLayout(ro.value, fo.value, cap.value, rb.value)


def tree_layout_fp4(cfg: ZhaConfig, level: int) -> Tuple[int, int]:
    """(byte offset, bytes per record) of the FP4 router records of a level."""
    ro, rb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().zha_tree_layout_fp4(ctypes.byref(cfg), level, ctypes.byref(ro), ctypes.byref(rb)))
    return ro.value, rb.value


class ZhaTree:
    """A tree over a caller-owned KV cache K, V [Hkv, capacity, d] (CUDA tensors)."""

    def __init__(self, cfg: ZhaConfig, K: torch.Tensor, V: torch.Tensor, refs: torch.Tensor):
        self.cfg = cfg
        dt = TORCH_DTYPE[cfg.dtype]
        shape = (cfg.n_kv_heads, cfg.capacity, cfg.d)
        for name, t in (("K", K), ("V", V)):
            if tuple(t.shape) != shape or t.dtype != dt or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA {dt} tensor of shape {shape}")
        if (tuple(refs.shape) != (cfg.n_kv_heads, cfg.n_refs, cfg.d) or refs.dtype != dt or not refs.is_cuda
                or not refs.is_contiguous()):
            raise ValueError("refs must be a contiguous CUDA tensor [Hkv, R, d] of the cache dtype")
        self.K, self.V, self.refs = K, V, refs
        nb, sb = tree_bytes(cfg)
        self.nodes = torch.zeros(nb, dtype=torch.uint8, device=K.device)
        self.scratch = torch.zeros(sb, dtype=torch.uint8, device=K.device)
        h = ctypes.c_void_p()
        _check(lib().zha_tree_create(ctypes.byref(cfg), K.data_ptr(), V.data_ptr(), refs.data_ptr(),
                                     self.nodes.data_ptr(), self.scratch.data_ptr(), ctypes.byref(h)))
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.zha_tree_destroy(h)
            self._h = None

    @property
    def size(self) -> int:
        return int(lib().zha_tree_size(self._h))

    def build(self, n: int, stream=None) -> None:
        _check(lib().zha_tree_build(self._h, n, _stream(stream)))

    def append(self, K_new: torch.Tensor, V_new: torch.Tensor, stream=None) -> None:
        """Append tokens K_new, V_new [Hkv, m, d] (CUDA, cache dtype)."""
        c = self.cfg
        for name, t in (("K_new", K_new), ("V_new", V_new)):
            if (t.dim() != 3 or t.shape[0] != c.n_kv_heads or t.shape[2] != c.d or t.dtype != TORCH_DTYPE[c.dtype]
                    or not t.is_cuda):
                raise ValueError(f"{name} must be a CUDA {TORCH_DTYPE[c.dtype]} tensor [{c.n_kv_heads}, m, {c.d}]")
        if K_new.shape != V_new.shape:
            raise ValueError("K_new and V_new must have the same shape")
        m = K_new.shape[1]
        K_new = K_new.contiguous()
        V_new = V_new.contiguous()
        _check(lib().zha_tree_append(self._h, K_new.data_ptr(), V_new.data_ptr(), m, _stream(stream)))

    def decode(self, Q: torch.Tensor, *, want_kept: bool = False, want_stats: bool = False, out=None,
               scored_cap: int = 0, stream=None):
        """Decode queries Q [B, Hq, d].  Returns O [B, Hq, d] fp32 (and kept lists / stats when asked)."""
        c = self.cfg
        if Q.dim() != 3 or tuple(Q.shape[1:]) != (c.n_q_heads, c.d) or Q.dtype != TORCH_DTYPE[c.dtype] or not Q.is_cuda:
            raise ValueError(f"Q must be a CUDA {TORCH_DTYPE[c.dtype]} tensor [B, {c.n_q_heads}, {c.d}]")
        B = Q.shape[0]
        if out is not None and (tuple(out.shape) != (B, c.n_q_heads, c.d) or out.dtype != torch.float32
                                or not out.is_cuda or not out.is_contiguous()):
            raise ValueError(f"out must be a contiguous CUDA float32 tensor [{B}, {c.n_q_heads}, {c.d}]")
        Q = Q.contiguous()
        O = out if out is not None else torch.empty(B, self.cfg.n_q_heads, self.cfg.d, dtype=torch.float32,
                                                    device=Q.device)
        kept = cnt = stats = None
        if want_kept:
            kept = torch.full((B, self.cfg.n_q_heads, max(1, self.cfg.capacity // self.cfg.block)), -1,
                              dtype=torch.int32, device=Q.device)
            cnt = torch.zeros(B, self.cfg.n_q_heads, dtype=torch.int32, device=Q.device)
        if want_stats:
            stats = torch.zeros(B, self.cfg.n_q_heads, STAT_COUNT, dtype=torch.int64, device=Q.device)
        scored = None
        if scored_cap > 0:
            scored = torch.full((B, self.cfg.n_q_heads, scored_cap), -1, dtype=torch.int32, device=Q.device)
        _check(lib().zha_decode(self._h, Q.data_ptr(), O.data_ptr(), B, _ptr(kept), _ptr(cnt), _ptr(stats),
                                _ptr(scored), scored_cap, _stream(stream)))
        if not (want_kept or want_stats or scored is not None):
            return O
        res = [O]
        if want_kept:
            res.append((kept, cnt))
        if want_stats:
            res.append(stats)
        if scored is not None:
            res.append(scored)
        return tuple(res)

    def route_multi(self, Q: torch.Tensor, *, want_kept: bool = False, stream=None):
        """Route and attend m queries Q [m, Hq, d] of this context (zha_route_multi).  Returns O [m, Hq, d] fp32
        (and (kept, kept_cnt) when asked)."""
        c = self.cfg
        if Q.dim() != 3 or tuple(Q.shape[1:]) != (c.n_q_heads, c.d) or Q.dtype != TORCH_DTYPE[c.dtype] or not Q.is_cuda:
            raise ValueError(f"Q must be a CUDA {TORCH_DTYPE[c.dtype]} tensor [m, {c.n_q_heads}, {c.d}]")
        m = Q.shape[0]
        Q = Q.contiguous()
        O = torch.empty(m, c.n_q_heads, c.d, dtype=torch.float32, device=Q.device)
        kept = cnt = None
        if want_kept:
            kept = torch.full((m, c.n_q_heads, max(1, c.capacity // c.block)), -1, dtype=torch.int32, device=Q.device)
            cnt = torch.zeros(m, c.n_q_heads, dtype=torch.int32, device=Q.device)
        _check(lib().zha_route_multi(self._h, Q.data_ptr(), O.data_ptr(), m, _ptr(kept), _ptr(cnt), _stream(stream)))
        return (O, (kept, cnt)) if want_kept else O

    def decode_step_host(self, k_host: Optional[torch.Tensor], v_host: Optional[torch.Tensor], q_host: torch.Tensor,
                         o_host: torch.Tensor, stream=None) -> None:
        """One decode step from (pinned) host tensors; o_host [B, Hq, d] fp32 receives the output."""
        B = q_host.shape[0]
        _check(lib().zha_decode_step_host(self._h, _ptr(k_host), _ptr(v_host), q_host.data_ptr(), o_host.data_ptr(),
                                          B, _stream(stream)))

    def set_step_p(self, p) -> None:
        """Top-p threshold per routing step (p[s] for step s, the last value for later steps); [] or None
        returns to the configuration's p."""
        vals = [] if p is None else [float(x) for x in p]
        arr = (_c.c_float * max(len(vals), 1))(*vals)
        _check(lib().zha_tree_set_step_p(self._h, _c.cast(arr, _c.c_void_p) if vals else None, len(vals)))

    def status(self, stream=None) -> None:
        _check(lib().zha_tree_status(self._h, _stream(stream)))

    def level_planes(self, level: int):
        """Stored planes of one level: (mu [Hkv, cap, R, d], bias [Hkv, cap, R] fp32, f [Hkv, cap, R] fp32)."""
        c = self.cfg
        lay = tree_layout(c, level)
        es = 2 if c.dtype == ZHA_BF16 else 4
        n = c.n_kv_heads * lay.cap_nodes
        rec = self.nodes[lay.rec_offset: lay.rec_offset + n * lay.rec_bytes].view(c.n_kv_heads, lay.cap_nodes,
                                                                                lay.rec_bytes)
        mu_b = c.n_refs * c.d * es
        mu = rec[..., :mu_b].contiguous().view(TORCH_DTYPE[c.dtype]).view(c.n_kv_heads, lay.cap_nodes, c.n_refs, c.d)
        bias = rec[..., mu_b: mu_b + 4 * c.n_refs].contiguous().view(torch.float32)
        f = self.nodes[lay.f_offset: lay.f_offset + n * c.n_refs * 4].view(torch.float32).view(
            c.n_kv_heads, lay.cap_nodes, c.n_refs)
        return mu, bias, f

    def fp4_records(self, level: int):
        """FP4 router records of one level: (codes [Hkv, cap, R, d] uint8 (one code per dimension),
        scales [Hkv, cap, R, d/16] uint8 e4m3, bias [Hkv, cap, R] fp32)."""
        c = self.cfg
        off, rb = tree_layout_fp4(c, level)
        cap = tree_layout(c, level).cap_nodes
        rec = self.nodes[off: off + c.n_kv_heads * cap * rb].view(c.n_kv_heads, cap, rb)
        R, D = c.n_refs, c.d
        packed = rec[..., : R * D // 2].reshape(c.n_kv_heads, cap, R, D // 2)
        codes = torch.stack([packed & 15, packed >> 4], dim=-1).reshape(c.n_kv_heads, cap, R, D)
        scales = rec[..., R * D // 2: R * (D // 2 + D // 16)].reshape(c.n_kv_heads, cap, R, D // 16)
        b0 = R * (D // 2 + D // 16)
        bias = rec[..., b0: b0 + 4 * R].contiguous().view(torch.float32)
        return codes, scales, bias


def launch_count() -> int:
    """Kernels libzha.so has launched in this process."""
    return int(lib().zha_launch_count())


def dense_scratch_bytes(cfg: ZhaConfig, B: int, n: int) -> int:
    return int(lib().zha_dense_scratch_bytes(ctypes.byref(cfg), B, n))


class DenseDecoder:
    """Dense decode over tokens [0, n) of K, V [Hkv, ld, d] with a reusable zero-filled scratch."""

    def __init__(self, cfg: ZhaConfig, B: int, n_max: int, device="cuda"):
        self.cfg = cfg
        self.scratch = torch.zeros(max(256, dense_scratch_bytes(cfg, B, n_max)), dtype=torch.uint8, device=device)
        self.B = B

    def __call__(self, K: torch.Tensor, V: torch.Tensor, n: int, Q: torch.Tensor, out=None, stream=None):
        B = Q.shape[0]
        need = dense_scratch_bytes(self.cfg, B, n)
        if need > self.scratch.numel():
            self.scratch = torch.zeros(need, dtype=torch.uint8, device=Q.device)
        Q = Q.contiguous()
        O = out if out is not None else torch.empty(B, self.cfg.n_q_heads, self.cfg.d, dtype=torch.float32,
                                                    device=Q.device)
        _check(lib().zha_dense_decode(ctypes.byref(self.cfg), K.data_ptr(), V.data_ptr(), K.shape[1], n,
                                      Q.data_ptr(), O.data_ptr(), B, self.scratch.data_ptr(), _stream(stream)))
        return O


def dense_decode(cfg: ZhaConfig, K: torch.Tensor, V: torch.Tensor, n: int, Q: torch.Tensor, stream=None):
    return DenseDecoder(cfg, Q.shape[0], n, device=Q.device)(K, V, n, Q, stream=stream)
