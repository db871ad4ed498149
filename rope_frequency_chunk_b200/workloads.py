"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

This module is the single source of inputs for both the CUDA path and the CPU
oracle. It draws pre-RoPE queries, keys and values, rounds them to the cache
dtype, and picks each KV head's dominant frequency-chunk set. It performs no
RoPE, no scoring, no selection and no attention.

Recipe (stated once, used everywhere):

* Every tensor comes from its own numpy PCG64 stream, keyed by
  ``SeedSequence([seed, tag, layer, b, g, step])``, so any single
  (layer, sequence, KV head) can be regenerated alone, and sequences are
  independent.
* Per (layer, KV head) a per-dimension scale vector ``s`` in R^128 is drawn
  log-normal(0, 1); it is shared by the group's query heads, the keys and the
  values (the weights of a real layer play this role).
* Queries and keys are N(0, 1) * s; values are N(0, 1) * s.
* Where a workload has outlier frequency chunks, each KV head gets
  ``n_outlier`` FCs chosen uniformly; on both dims of those FCs the query and
  key entries are Student-t(3) * 4 * s instead of N(0, 1) * s (heavy tails).
* The dominant set of a KV head stands in for the offline calibration step of
  "FASA: Frequency-aware Sparse Attention" (gist.science technical summary,
  §2, TIP "offline calibration"), which needs a trained model: it is the
  ``n_dom`` FCs with the largest expected energy
  ``c_i = m_i * (s_i^2 + s_{i+64}^2)`` (``m_i = 48`` = Var(4 * t_3) for an
  outlier FC, else 1), ties to the lower FC index, listed in that rank order.
* Values are drawn in float32 and rounded once to the cache dtype
  (bf16: round-to-nearest-even, via torch's float32->bfloat16 cast).
* The cache holds positions 0..L-1; the single query sits at position L.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HEAD_DIM = 128
N_FC = HEAD_DIM // 2

# stream tags (part of each SeedSequence key)
_TAG_SCALE, _TAG_OUTLIER, _TAG_Q, _TAG_K, _TAG_V = 1, 2, 3, 4, 5

# Budget numbers printed by the pages ("FASA: Frequency-aware Sparse
# Attention", English abstract): 256 kept tokens on LongBench-V1, and 18.9% of
# the cache on AIME24.
PAGE_TOKEN_BUDGET = 256
PAGE_CACHE_FRACTION = 0.189


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode-layer configuration."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    rope_base: float
    dtype: str            # "f32" or "bf16": cache, query and output dtype
    ctx_len: int          # L, cached tokens per sequence (positions 0..L-1)
    n_dom: int            # dominant FCs per KV head
    k: int                # kept tokens per (sequence, KV head)
    n_outlier: int = 0    # heavy-tailed outlier FCs per KV head
    seed: int = 0
    head_dim: int = HEAD_DIM

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def q_pos(self) -> int:
        return self.ctx_len

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def c4_budget(ctx_len: int) -> int:
    """Kept tokens for the long-CoT sweep: 18.9% of L, rounded half away from zero."""
    return int(math.floor(PAGE_CACHE_FRACTION * ctx_len + 0.5))


def _cfg(name, seed, **kw):
    return Workload(name=name, seed=seed, **kw)


# The five decode workloads (sizes as the headline configuration list states).
CONFIGS = {
    # 1 head, fp32, L 4096, 16 dominant FCs, top-256
    "c1": _cfg("c1", 101, batch=1, n_q_heads=1, n_kv_heads=1, rope_base=1e4,
               dtype="f32", ctx_len=4096, n_dom=16, k=256),
    # Llama-3-8B-shaped layer: B1, 32/8 heads, base 5e5, bf16, L 32768, top-256
    "c2": _cfg("c2", 202, batch=1, n_q_heads=32, n_kv_heads=8, rope_base=5e5,
               dtype="bf16", ctx_len=32768, n_dom=16, k=256, n_outlier=2),
    # same layer, B8, L 131072, top-2048
    "c3": _cfg("c3", 303, batch=8, n_q_heads=32, n_kv_heads=8, rope_base=5e5,
               dtype="bf16", ctx_len=131072, n_dom=16, k=2048, n_outlier=2),
    # long-CoT sweep point (B4, 28/4 heads); L and k vary per step, n_dom in {8,16,32}
    "c4": _cfg("c4", 404, batch=4, n_q_heads=28, n_kv_heads=4, rope_base=1e4,
               dtype="bf16", ctx_len=32768, n_dom=16, k=c4_budget(32768)),
    # high-batch serving: B64, 32/8, L 16384, k in {128,256,512,1024}
    "c5": _cfg("c5", 505, batch=64, n_q_heads=32, n_kv_heads=8, rope_base=5e5,
               dtype="bf16", ctx_len=16384, n_dom=16, k=256),
}

C4_APPEND_CHUNK = 1024
C4_STEPS = 32
C4_NDOMS = (8, 16, 32)
C5_KS = (128, 256, 512, 1024)


def _rng(wl: Workload, tag: int, layer: int, b: int = 0, g: int = 0, step: int = 0):
    ss = np.random.SeedSequence([wl.seed, tag, layer, b, g, step])
    return np.random.Generator(np.random.PCG64(ss))


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the storage dtype.

    Returns float32 for "f32" and the raw bfloat16 bit patterns (uint16) for
    "bf16" (round-to-nearest-even, torch's cast).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype != "bf16":
        raise ValueError(dtype)
    import torch

    t = torch.from_numpy(x).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def stored_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of stored elements (float32, or uint16 bf16 bits)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------- per layer

@dataclasses.dataclass
class LayerParams:
    scales: np.ndarray     # [Hkv, 128] float32
    outliers: np.ndarray   # [Hkv, n_outlier] int64 FC indices
    dom_idx: np.ndarray    # [Hkv, n_dom] int32


def layer_params(wl: Workload, layer: int = 0, n_dom: int | None = None) -> LayerParams:
    n_dom = wl.n_dom if n_dom is None else n_dom
    if not 1 <= n_dom <= N_FC:
        raise ValueError(f"n_dom={n_dom}")
    H = wl.n_kv_heads
    scales = np.empty((H, HEAD_DIM), np.float32)
    outl = np.zeros((H, wl.n_outlier), np.int64)
    dom = np.empty((H, n_dom), np.int32)
    for g in range(H):
        r = _rng(wl, _TAG_SCALE, layer, 0, g)
        scales[g] = np.exp(r.standard_normal(HEAD_DIM)).astype(np.float32)
        if wl.n_outlier:
            ro = _rng(wl, _TAG_OUTLIER, layer, 0, g)
            outl[g] = np.sort(ro.choice(N_FC, size=wl.n_outlier, replace=False))
        s2 = scales[g].astype(np.float64) ** 2
        energy = s2[:N_FC] + s2[N_FC:]
        if wl.n_outlier:
            energy[outl[g]] *= 48.0
        # rank descending by energy, ties to the lower FC index
        order = np.lexsort((np.arange(N_FC), -energy))
        dom[g] = order[:n_dom]
    return LayerParams(scales, outl, dom)


def _draw(wl, lp, tag, layer, b, g, n_rows, step=0, outliers=True, row0=0, n_total=None):
    """N(0,1)*s rows (with heavy-tailed outlier FCs when asked), float32.

    Rows ``row0 .. row0+n_rows-1`` of a stream of ``n_total`` rows; a stream is
    always drawn whole so that any slice is reproducible.
    """
    n_total = n_rows if n_total is None else n_total
    r = _rng(wl, tag, layer, b, g, step)
    x = np.empty((n_total, HEAD_DIM), np.float32)
    r.standard_normal(out=x, dtype=np.float32)
    if outliers and wl.n_outlier:
        t = r.standard_t(3, size=(n_total, 2 * wl.n_outlier)).astype(np.float32) * 4.0
        cols = np.concatenate([lp.outliers[g], lp.outliers[g] + N_FC])
        x[:, cols] = t
    x *= lp.scales[g]
    return x[row0:row0 + n_rows]


def head_q(wl: Workload, lp: LayerParams, layer: int, b: int, g: int, step: int = 0) -> np.ndarray:
    """Pre-RoPE queries of the G heads of KV group g, stored dtype, [G, 128]."""
    x = _draw(wl, lp, _TAG_Q, layer, b, g, wl.group, step=step)
    return round_to_dtype(x, wl.dtype)


def head_kv(wl: Workload, lp: LayerParams, layer: int, b: int, g: int,
            n_tokens: int | None = None):
    """Pre-RoPE keys and values of one (sequence, KV head), stored dtype, [L, 128] each."""
    L = wl.ctx_len if n_tokens is None else n_tokens
    k = _draw(wl, lp, _TAG_K, layer, b, g, L)
    v = _draw(wl, lp, _TAG_V, layer, b, g, L, outliers=False)
    return round_to_dtype(k, wl.dtype), round_to_dtype(v, wl.dtype)


def _threads() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    return max(1, min(32, n))


@dataclasses.dataclass
class LayerInputs:
    params: LayerParams
    q: np.ndarray      # [B, Hq, 128] stored dtype (pre-RoPE)
    k: np.ndarray      # [B, Hkv, L, 128] stored dtype (pre-RoPE)
    v: np.ndarray      # [B, Hkv, L, 128] stored dtype


def layer_inputs(wl: Workload, layer: int = 0, n_dom: int | None = None,
                 step: int = 0, with_kv: bool = True) -> LayerInputs:
    """All inputs of one layer, generated head by head on a thread pool."""
    lp = layer_params(wl, layer, n_dom)
    B, H, G, L = wl.batch, wl.n_kv_heads, wl.group, wl.ctx_len
    sdt = np.float32 if wl.dtype == "f32" else np.uint16
    q = np.empty((B, H * G, HEAD_DIM), sdt)
    k = np.empty((B, H, L, HEAD_DIM), sdt) if with_kv else None
    v = np.empty((B, H, L, HEAD_DIM), sdt) if with_kv else None

    def work(bg):
        b, g = divmod(bg, H)
        q[b, g * G:(g + 1) * G] = head_q(wl, lp, layer, b, g, step)
        if with_kv:
            k[b, g], v[b, g] = head_kv(wl, lp, layer, b, g)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(B * H)))
    return LayerInputs(lp, q, k, v)


def multi_queries(wl: Workload, n_q: int, layer: int = 0, n_dom: int | None = None) -> np.ndarray:
    """Queries of n_q tokens per sequence, [B][n_q][Hq][128] stored: token j
    is the layer's query of decode step j (token 0 = layer_inputs' q)."""
    lp = layer_params(wl, layer, n_dom)
    B, H, G = wl.batch, wl.n_kv_heads, wl.group
    sdt = np.float32 if wl.dtype == "f32" else np.uint16
    q = np.empty((B, n_q, H * G, HEAD_DIM), sdt)
    for j in range(n_q):
        for b in range(B):
            for g in range(H):
                q[b, j, g * G:(g + 1) * G] = head_q(wl, lp, layer, b, g, j)
    return q


def to_torch(a: np.ndarray, device="cpu"):
    """Stored array (float32, or uint16 bf16 bits) -> torch tensor of the cache dtype."""
    import torch

    if a.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device)


def from_torch(t) -> np.ndarray:
    """torch tensor (float32 or bfloat16) -> stored numpy array (float32 or uint16 bits)."""
    import torch

    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()
