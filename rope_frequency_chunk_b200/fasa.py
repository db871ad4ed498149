"""Python binding of the FASA C ABI (include/fasa.h): argument marshalling only.

Every call passes device pointers, sizes and the current CUDA stream to
libfasa.so; all arithmetic runs in the library's kernels. torch provides the
device memory and the stream. There is no fallback: if the library is missing
or a call fails, a FasaError is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfasa.so")

FASA_F32, FASA_BF16 = 0, 1
HEAD_DIM = 128
STATUS = {0: "FASA_OK", 1: "FASA_ERR_INVALID_ARG", 2: "FASA_ERR_UNSUPPORTED", 3: "FASA_ERR_CAPACITY",
          4: "FASA_ERR_WORKSPACE", 5: "FASA_ERR_CUDA", 6: "FASA_ERR_TIMEOUT", 7: "FASA_ERR_BAD_INDEX"}

_TORCH_DTYPE = {FASA_F32: torch.float32, FASA_BF16: torch.bfloat16}
_DTYPE_CODE = {"f32": FASA_F32, "bf16": FASA_BF16, torch.float32: FASA_F32, torch.bfloat16: FASA_BF16,
               FASA_F32: FASA_F32, FASA_BF16: FASA_BF16}


class FasaError(RuntimeError):
    def __init__(self, status: int, call: str):
        super().__init__(f"{call}: {STATUS.get(status, status)}")
        self.status = status


class fasa_cache(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_dom", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("sketch_stride", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("sketch", ctypes.c_void_p),
                ("dom_idx", ctypes.c_void_p)]


class fasa_varlen(ctypes.Structure):
    _fields_ = [("seq_len", ctypes.c_void_p), ("budget", ctypes.c_void_p), ("max_seq_len", ctypes.c_int32),
                ("max_budget", ctypes.c_int32), ("q_prerotated", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class fasa_paged(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("block_size", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("n_pages", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_CP = ctypes.POINTER(fasa_cache)

_SIGS = {
    "fasa_abi_version": (_I, []),
    "fasa_status_string": (ctypes.c_char_p, [_I]),
    "fasa_last_cuda_error": (ctypes.c_char_p, []),
    "fasa_sketch_stride": (_I, [_I, _I]),
    "fasa_check_dom_idx": (_I, [_P, _I, _I]),
    "fasa_append_kv": (_I, [_CP, _P, _P, _I, _I, _P]),
    "fasa_score": (_I, [_CP, _I, _P, _I, _P, _P]),
    "fasa_select_topk": (_I, [_P, _I, _I, _I, _P, _P]),
    "fasa_sparse_attend": (_I, [_CP, _I, _P, _I, _P, _I, _P, _P]),
    "fasa_decode_workspace_bytes": (ctypes.c_size_t, [_CP, _I, _I]),
    "fasa_decode_launches": (_I, [_CP, _I, _I]),
    "fasa_decode": (_I, [_CP, _I, _P, _I, _I, _P, _P, _P, ctypes.c_size_t, _P]),
    "fasa_decode_varlen_workspace_bytes": (ctypes.c_size_t, [_CP, ctypes.POINTER(fasa_varlen)]),
    "fasa_decode_varlen": (_I, [_CP, ctypes.POINTER(fasa_varlen), _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "fasa_append_kv_paged": (_I, [_CP, ctypes.POINTER(fasa_paged), _P, _P, _I, _P, _P]),
    "fasa_decode_paged_workspace_bytes": (ctypes.c_size_t, [_CP, ctypes.POINTER(fasa_paged),
                                                            ctypes.POINTER(fasa_varlen)]),
    "fasa_decode_paged": (_I, [_CP, ctypes.POINTER(fasa_paged), ctypes.POINTER(fasa_varlen), _P, _P, _P, _P,
                               ctypes.c_size_t, _P]),
    "fasa_decode_multi_workspace_bytes": (ctypes.c_size_t, [_CP, _I, _I, _I]),
    "fasa_decode_multi": (_I, [_CP, _I, _P, _I, _I, _I, _P, _P, _P, ctypes.c_size_t, _P]),
    "fasa_decode_static_scratch": (_I, [_CP, _I, _P, _I, _I, _P, _P, _P]),
    "fasa_dense_workspace_bytes": (ctypes.c_size_t, [_CP, _I]),
    "fasa_dense_decode": (_I, [_CP, _I, _P, _I, _P, _P, ctypes.c_size_t, _P]),
    "fasa_device_status": (_I, [_I]),
    "fasa_host_kv_pointer": (_I, [_P, ctypes.POINTER(ctypes.c_void_p)]),
    "fasa_set_decode_path": (_I, [_I]),
    "fasa_decode_path": (_I, [_CP, _I, _I]),
    "fasa_calibrate_workspace_bytes": (ctypes.c_size_t, [_CP, _I, _I, _I]),
    "fasa_calibrate_scores": (_I, [_CP, _I, _P, _I, _I, _P, _P]),
    "fasa_calibrate_counts": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, ctypes.c_size_t, _P]),
    "fasa_calibrate_dominant": (_I, [_P, _I, _I, _P, _P]),
    "fasa_calibrate": (_I, [_CP, _I, _P, _I, _I, _I, _I, _P, _P, _P, ctypes.c_size_t, _P]),
}


def lib() -> ctypes.CDLL:
    """Load libfasa.so (built in-tree by rope_frequency_chunk_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FasaError(5, f"libfasa.so not found at {LIB_PATH}; build it with "
                               "`python -m rope_frequency_chunk_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int, call: str):
    if status != 0:
        detail = ""
        if status == 5:
            detail = " (" + lib().fasa_last_cuda_error().decode() + ")"
        raise FasaError(status, call + detail)


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


# ------------------------------------------------------------------ cache

def fasa_sketch_stride(n_dom: int, dtype) -> int:
    return int(lib().fasa_sketch_stride(n_dom, _DTYPE_CODE[dtype]))


def fasa_check_dom_idx(dom_idx_host) -> None:
    import numpy as np
    a = np.ascontiguousarray(dom_idx_host, dtype=np.int32)
    _check(lib().fasa_check_dom_idx(a.ctypes.data, a.shape[0], a.shape[1]), "fasa_check_dom_idx")


class KVCache:
    """A layer's KV cache and dominant-FC key sketch, in caller-owned memory:
    all on the device (FASA-C), or, with kv_on_host, K and V in pinned host
    memory that the device reads across the host link and only the sketch on
    the device (FASA-M)."""

    def __init__(self, batch, n_q_heads, n_kv_heads, n_dom, max_len, dtype, rope_base, dom_idx,
                 device="cuda", kv_on_host=False):
        code = _DTYPE_CODE[dtype]
        tdt = _TORCH_DTYPE[code]
        stride = fasa_sketch_stride(n_dom, code)
        if stride < 0:
            raise FasaError(1, "fasa_sketch_stride")
        fasa_check_dom_idx(dom_idx)
        self.batch, self.n_q_heads, self.n_kv_heads = batch, n_q_heads, n_kv_heads
        self.n_dom, self.max_len, self.dtype, self.rope_base = n_dom, max_len, tdt, float(rope_base)
        shape = (batch, n_kv_heads, max_len, HEAD_DIM)
        self.kv_on_host = bool(kv_on_host)
        if self.kv_on_host:
            self.k = torch.empty(shape, dtype=tdt, pin_memory=True)
            self.v = torch.empty(shape, dtype=tdt, pin_memory=True)
            kp, vp = fasa_host_kv_pointer(self.k), fasa_host_kv_pointer(self.v)
        else:
            self.k = torch.empty(shape, dtype=tdt, device=device)
            self.v = torch.empty_like(self.k)
            kp, vp = self.k.data_ptr(), self.v.data_ptr()
        self.sketch = torch.empty(batch, n_kv_heads, max_len, stride, dtype=tdt, device=device)
        self.dom_idx = torch.as_tensor(dom_idx, dtype=torch.int32).to(device).contiguous()
        self.struct = fasa_cache(batch, n_q_heads, n_kv_heads, HEAD_DIM, n_dom, max_len, code, stride,
                                 float(rope_base), kp, vp, self.sketch.data_ptr(), self.dom_idx.data_ptr())
        self.sketch_stride = stride

    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads

    def device_bytes(self) -> int:
        """Bytes of this cache held in device memory."""
        n = self.sketch.numel() * self.sketch.element_size() + self.dom_idx.numel() * 4
        if not self.kv_on_host:
            n += (self.k.numel() + self.v.numel()) * self.k.element_size()
        return n

    def ref(self):
        return ctypes.byref(self.struct)


def fasa_host_kv_pointer(t: torch.Tensor) -> int:
    """Device address of a pinned host tensor's data (FASA-M K and V)."""
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned():
        raise TypeError("expected a pinned host tensor")
    out = ctypes.c_void_p()
    _check(lib().fasa_host_kv_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(out)), "fasa_host_kv_pointer")
    return int(out.value)


class PagedKVCache:
    """A layer's paged KV cache: K, V and sketch page pools [n_pages][Hkv]
    [block_size][...] on the device and a block table [B][max_blocks] (int32,
    device) mapping each sequence's logical blocks to pages. The caller
    assigns pages by writing block_table."""

    def __init__(self, batch, n_q_heads, n_kv_heads, n_dom, n_pages, block_size, max_blocks, dtype, rope_base,
                 dom_idx, device="cuda"):
        code = _DTYPE_CODE[dtype]
        tdt = _TORCH_DTYPE[code]
        stride = fasa_sketch_stride(n_dom, code)
        if stride < 0:
            raise FasaError(1, "fasa_sketch_stride")
        fasa_check_dom_idx(dom_idx)
        self.batch, self.n_q_heads, self.n_kv_heads = batch, n_q_heads, n_kv_heads
        self.n_dom, self.dtype, self.rope_base = n_dom, tdt, float(rope_base)
        self.n_pages, self.block_size, self.max_blocks = n_pages, block_size, max_blocks
        self.max_len = max_blocks * block_size
        self.k = torch.zeros(n_pages, n_kv_heads, block_size, HEAD_DIM, dtype=tdt, device=device)
        self.v = torch.zeros_like(self.k)
        self.sketch = torch.zeros(n_pages, n_kv_heads, block_size, stride, dtype=tdt, device=device)
        self.block_table = torch.zeros(batch, max_blocks, dtype=torch.int32, device=device)
        self.dom_idx = torch.as_tensor(dom_idx, dtype=torch.int32).to(device).contiguous()
        self.struct = fasa_cache(batch, n_q_heads, n_kv_heads, HEAD_DIM, n_dom, self.max_len, code, stride,
                                 float(rope_base), self.k.data_ptr(), self.v.data_ptr(), self.sketch.data_ptr(),
                                 self.dom_idx.data_ptr())
        self.pages = fasa_paged(self.block_table.data_ptr(), block_size, max_blocks, n_pages, 0)
        self.sketch_stride = stride

    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads

    def ref(self):
        return ctypes.byref(self.struct)

    def pref(self):
        return ctypes.byref(self.pages)

    def logical(self, pool, b: int, g: int, length: int):
        """Rows 0 .. length-1 of (b, g) gathered from a pool (k, v or sketch)."""
        t = torch.arange(length, device=pool.device)
        pg = self.block_table[b, (t // self.block_size)].long()
        return pool[pg, g, t % self.block_size]


def fasa_append_kv_paged(cache: PagedKVCache, k_new, v_new, pos0, stream=None) -> None:
    """Append n_new tokens to every sequence b at slots pos0[b] .. (pos0: int32 [B] on the device)."""
    _dev(k_new, "k_new", cache.dtype)
    _dev(v_new, "v_new", cache.dtype)
    _dev(pos0, "pos0", torch.int32)
    n_new = k_new.shape[2]
    if tuple(k_new.shape) != (cache.batch, cache.n_kv_heads, n_new, HEAD_DIM) or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new must be [B, Hkv, n_new, 128]")
    _check(lib().fasa_append_kv_paged(cache.ref(), cache.pref(), k_new.data_ptr(), v_new.data_ptr(), n_new,
                                      pos0.data_ptr(), _stream(stream)), "fasa_append_kv_paged")


def fasa_decode_paged(cache: PagedKVCache, seq_len, q, max_seq_len: int, max_budget: int, budget=None,
                      q_prerotated: bool = False, out=None, idx_out=None, workspace=None, stream=None):
    """fasa_decode_varlen over a paged cache."""
    _q(cache, q)
    vl = _varlen(seq_len, budget, max_seq_len, max_budget, q_prerotated)
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", cache.dtype)
    if idx_out is not None:
        _dev(idx_out, "idx_out", torch.int32)
    if workspace is None:
        need = int(lib().fasa_decode_paged_workspace_bytes(cache.ref(), cache.pref(), ctypes.byref(vl)))
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_decode_paged(cache.ref(), cache.pref(), ctypes.byref(vl), q.data_ptr(), out.data_ptr(),
                                   _ptr(idx_out), workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "fasa_decode_paged")
    return out


# ------------------------------------------------------------------ calls

def fasa_append_kv(cache: KVCache, k_new, v_new, pos0: int, stream=None) -> None:
    _dev(k_new, "k_new", cache.dtype)
    _dev(v_new, "v_new", cache.dtype)
    n_new = k_new.shape[2]
    if tuple(k_new.shape) != (cache.batch, cache.n_kv_heads, n_new, HEAD_DIM) or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new must be [B, Hkv, n_new, 128]")
    _check(lib().fasa_append_kv(cache.ref(), k_new.data_ptr(), v_new.data_ptr(), n_new, pos0,
                                _stream(stream)), "fasa_append_kv")


def _q(cache, q):
    _dev(q, "q", cache.dtype)
    if tuple(q.shape) != (cache.batch, cache.n_q_heads, HEAD_DIM):
        raise ValueError("q must be [B, Hq, 128]")
    return q


def fasa_score(cache: KVCache, length: int, q, q_pos: int, scores=None, stream=None):
    _q(cache, q)
    if scores is None:
        scores = torch.empty(cache.batch, cache.n_kv_heads, length, dtype=torch.float32, device=q.device)
    _dev(scores, "scores", torch.float32)
    _check(lib().fasa_score(cache.ref(), length, q.data_ptr(), q_pos, scores.data_ptr(), _stream(stream)),
           "fasa_score")
    return scores


def fasa_select_topk(scores, k: int, idx=None, stream=None):
    _dev(scores, "scores", torch.float32)
    length = scores.shape[-1]
    rows = scores.numel() // max(length, 1)
    k_eff = min(k, length)
    if idx is None:
        idx = torch.empty(*scores.shape[:-1], k_eff, dtype=torch.int32, device=scores.device)
    _dev(idx, "idx", torch.int32)
    _check(lib().fasa_select_topk(scores.data_ptr(), rows, length, k, idx.data_ptr(), _stream(stream)),
           "fasa_select_topk")
    return idx


def fasa_sparse_attend(cache: KVCache, length: int, q, q_pos: int, idx, out=None, stream=None):
    _q(cache, q)
    _dev(idx, "idx", torch.int32)
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", cache.dtype)
    _check(lib().fasa_sparse_attend(cache.ref(), length, q.data_ptr(), q_pos, idx.data_ptr(), idx.shape[-1],
                                    out.data_ptr(), _stream(stream)), "fasa_sparse_attend")
    return out


def fasa_decode_workspace_bytes(cache: KVCache, length: int, k: int) -> int:
    return int(lib().fasa_decode_workspace_bytes(cache.ref(), length, k))


def fasa_decode_workspace(cache: KVCache, length: int, k: int, device=None):
    """A decode workspace for this shape, zeroed as fasa_decode requires
    before its first use (every call leaves its semaphores zero again)."""
    dev = device if device is not None else cache.k.device
    return torch.zeros(max(fasa_decode_workspace_bytes(cache, length, k), 1), dtype=torch.uint8, device=dev)


def fasa_decode(cache: KVCache, length: int, q, q_pos: int, k: int, out=None, idx_out=None,
                workspace=None, stream=None):
    """One FASA decode step; returns out (and fills idx_out when given). A
    given workspace must have been zeroed once (fasa_decode_workspace)."""
    _q(cache, q)
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", cache.dtype)
    if idx_out is not None:
        _dev(idx_out, "idx_out", torch.int32)
    need = fasa_decode_workspace_bytes(cache, length, k)
    if workspace is None:
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_decode(cache.ref(), length, q.data_ptr(), q_pos, k, out.data_ptr(), _ptr(idx_out),
                             workspace.data_ptr(), workspace.numel(), _stream(stream)), "fasa_decode")
    return out


def _varlen(seq_len, budget, max_seq_len: int, max_budget: int, q_prerotated: bool):
    """The C description of a varlen call; seq_len [B] and budget [Hkv]
    (or None) are int32 device tensors."""
    if seq_len is not None:
        _dev(seq_len, "seq_len", torch.int32)
    if budget is not None:
        _dev(budget, "budget", torch.int32)
    return fasa_varlen(_ptr(seq_len), _ptr(budget), int(max_seq_len), int(max_budget),
                       1 if q_prerotated else 0, 0)


def fasa_decode_varlen_workspace_bytes(cache: KVCache, max_seq_len: int, max_budget: int) -> int:
    d = fasa_varlen(None, None, int(max_seq_len), int(max_budget), 0, 0)
    d.seq_len = 16  # any aligned non-null value: only the bounds size the workspace
    return int(lib().fasa_decode_varlen_workspace_bytes(cache.ref(), ctypes.byref(d)))


def fasa_decode_varlen_workspace(cache: KVCache, max_seq_len: int, max_budget: int, device=None):
    """A zeroed workspace for fasa_decode_varlen with these bounds."""
    dev = device if device is not None else cache.k.device
    need = fasa_decode_varlen_workspace_bytes(cache, max_seq_len, max_budget)
    return torch.zeros(max(need, 1), dtype=torch.uint8, device=dev)


def fasa_decode_varlen(cache: KVCache, seq_len, q, max_seq_len: int, max_budget: int, budget=None,
                       q_prerotated: bool = False, out=None, idx_out=None, workspace=None, stream=None):
    """One decode step over sequences of their own lengths (seq_len, int32
    [B] on the device; the query of sequence b sits at position seq_len[b])
    with per-KV-head budgets (budget, int32 [Hkv] on the device, or None for
    max_budget everywhere). idx_out, when given, is int32 [B][Hkv][max_budget]:
    each row's kept tokens ascending, then -1."""
    _q(cache, q)
    vl = _varlen(seq_len, budget, max_seq_len, max_budget, q_prerotated)
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", cache.dtype)
    if idx_out is not None:
        _dev(idx_out, "idx_out", torch.int32)
    if workspace is None:
        workspace = fasa_decode_varlen_workspace(cache, max_seq_len, max_budget, q.device)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_decode_varlen(cache.ref(), ctypes.byref(vl), q.data_ptr(), out.data_ptr(), _ptr(idx_out),
                                    workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "fasa_decode_varlen")
    return out


def fasa_decode_multi_workspace(cache: KVCache, length: int, n_q: int, k: int, device=None):
    """A zeroed workspace for fasa_decode_multi at this shape."""
    dev = device if device is not None else cache.k.device
    need = int(lib().fasa_decode_multi_workspace_bytes(cache.ref(), length, n_q, k))
    return torch.zeros(max(need, 1), dtype=torch.uint8, device=dev)


def fasa_decode_multi(cache: KVCache, length: int, q, q_pos0: int, k: int, out=None, idx_out=None,
                      workspace=None, stream=None):
    """Multi-query decode: q [B, n_q, Hq, 128], token j at position q_pos0 + j;
    the query rows of a KV head share one kept set (idx_out [B, Hkv, k_eff])."""
    _dev(q, "q", cache.dtype)
    if q.dim() != 4 or tuple(q.shape[::2]) != (cache.batch, cache.n_q_heads) or q.shape[3] != HEAD_DIM:
        raise ValueError("q must be [B, n_q, Hq, 128]")
    n_q = q.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", cache.dtype)
    if idx_out is not None:
        _dev(idx_out, "idx_out", torch.int32)
    if workspace is None:
        workspace = fasa_decode_multi_workspace(cache, length, n_q, k, q.device)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_decode_multi(cache.ref(), length, q.data_ptr(), q_pos0, n_q, k, out.data_ptr(),
                                   _ptr(idx_out), workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "fasa_decode_multi")
    return out


DECODE_AUTO, DECODE_FUSED, DECODE_STAGED = 0, 1, 2


def fasa_set_decode_path(path: int) -> None:
    """Launch plan of later fasa_decode calls (process-wide)."""
    _check(lib().fasa_set_decode_path(int(path)), "fasa_set_decode_path")


def fasa_decode_path(cache: KVCache, length: int, k: int) -> int:
    """The plan fasa_decode would run for this shape (DECODE_FUSED or DECODE_STAGED)."""
    r = int(lib().fasa_decode_path(cache.ref(), length, k))
    if r < 0:
        _check(-r, "fasa_decode_path")
    return r


def fasa_decode_launches(cache: KVCache, length: int, k: int) -> int:
    """Kernels of this library one fasa_decode call launches for this shape."""
    r = int(lib().fasa_decode_launches(cache.ref(), length, k))
    if r < 0:
        _check(-r, "fasa_decode_launches")
    return r


def fasa_dense_workspace(cache: KVCache, length: int, device=None):
    """A zeroed workspace for fasa_dense_decode at this length."""
    dev = device if device is not None else cache.k.device
    need = int(lib().fasa_dense_workspace_bytes(cache.ref(), length))
    return torch.zeros(max(need, 1), dtype=torch.uint8, device=dev)


def fasa_dense_decode(cache: KVCache, length: int, q, q_pos: int, out=None, workspace=None, stream=None):
    """Dense attention over all `length` cached rows (the comparison path). A
    given workspace must have been zeroed once (fasa_dense_workspace)."""
    _q(cache, q)
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", cache.dtype)
    if workspace is None:
        workspace = fasa_dense_workspace(cache, length, q.device)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_dense_decode(cache.ref(), length, q.data_ptr(), q_pos, out.data_ptr(), workspace.data_ptr(),
                                   workspace.numel(), _stream(stream)), "fasa_dense_decode")
    return out


def fasa_device_status(clear: bool = True) -> int:
    """Synchronizes; returns the device status word (0 = OK)."""
    return int(lib().fasa_device_status(1 if clear else 0))


# ------------------------------------------------------------ calibration

CAL_MAX_WIN = 8
CAL_PLANES = 65


def _q_win(cache, q_win):
    _dev(q_win, "q_win", cache.dtype)
    if q_win.dim() != 4 or q_win.shape[0] != cache.batch or q_win.shape[2] != cache.n_q_heads \
            or q_win.shape[3] != HEAD_DIM:
        raise ValueError("q_win must be [B, n_win, Hq, 128]")
    return q_win.shape[1]


def fasa_calibrate_workspace_bytes(cache: KVCache, length: int, n_win: int, budget: int) -> int:
    return int(lib().fasa_calibrate_workspace_bytes(cache.ref(), length, n_win, budget))


def fasa_calibrate_scores(cache: KVCache, length: int, q_win, q_pos0: int, planes=None, stream=None):
    """Score planes [B, Hkv, n_win, 65, len] float32 of the calibration queries."""
    n_win = _q_win(cache, q_win)
    if planes is None:
        planes = torch.empty(cache.batch, cache.n_kv_heads, n_win, CAL_PLANES, length, dtype=torch.float32,
                             device=q_win.device)
    _dev(planes, "planes", torch.float32)
    _check(lib().fasa_calibrate_scores(cache.ref(), length, q_win.data_ptr(), q_pos0, n_win, planes.data_ptr(),
                                       _stream(stream)), "fasa_calibrate_scores")
    return planes


def fasa_calibrate_counts(planes, n_kv_heads: int, budget: int, counts=None, workspace=None, stream=None):
    """Agreement counts [Hkv, 64] uint32 (as int32 storage) from planes [..., n_win, 65, len]."""
    _dev(planes, "planes", torch.float32)
    n_win, length = planes.shape[-3], planes.shape[-1]
    if planes.shape[-2] != CAL_PLANES:
        raise ValueError("planes must be [..., n_win, 65, len]")
    rows = planes.numel() // (n_win * CAL_PLANES * length)
    if counts is None:
        counts = torch.empty(n_kv_heads, 64, dtype=torch.int32, device=planes.device)
    _dev(counts, "counts", torch.int32)
    need = rows * n_win * CAL_PLANES * min(budget, length) * 4
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=planes.device)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_calibrate_counts(planes.data_ptr(), rows, n_kv_heads, n_win, length, budget,
                                       counts.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                       _stream(stream)), "fasa_calibrate_counts")
    return counts


def fasa_calibrate_dominant(counts, n_dom: int, dom_idx=None, stream=None):
    """I_dom [Hkv, n_dom] int32 from counts [Hkv, 64]."""
    _dev(counts, "counts", torch.int32)
    if dom_idx is None:
        dom_idx = torch.empty(counts.shape[0], n_dom, dtype=torch.int32, device=counts.device)
    _dev(dom_idx, "dom_idx", torch.int32)
    _check(lib().fasa_calibrate_dominant(counts.data_ptr(), counts.shape[0], n_dom, dom_idx.data_ptr(),
                                         _stream(stream)), "fasa_calibrate_dominant")
    return dom_idx


def fasa_calibrate(cache: KVCache, length: int, q_win, q_pos0: int, budget: int, n_dom: int,
                   counts=None, dom_idx=None, workspace=None, stream=None):
    """Offline calibration; returns (counts [Hkv, 64], dom_idx [Hkv, n_dom])."""
    n_win = _q_win(cache, q_win)
    dev = q_win.device
    if counts is None:
        counts = torch.empty(cache.n_kv_heads, 64, dtype=torch.int32, device=dev)
    if dom_idx is None:
        dom_idx = torch.empty(cache.n_kv_heads, n_dom, dtype=torch.int32, device=dev)
    _dev(counts, "counts", torch.int32)
    _dev(dom_idx, "dom_idx", torch.int32)
    need = fasa_calibrate_workspace_bytes(cache, length, n_win, budget)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8)
    _check(lib().fasa_calibrate(cache.ref(), length, q_win.data_ptr(), q_pos0, n_win, budget, n_dom,
                                counts.data_ptr(), dom_idx.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                _stream(stream)), "fasa_calibrate")
    return counts, dom_idx
