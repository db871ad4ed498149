"""Shared helpers of the GPU parity tests: build a cache through the C ABI,
compare each stage with the CPU oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle.fasa_oracle as O
from rope_frequency_chunk_b200 import fasa as F
from rope_frequency_chunk_b200 import workloads as W

OUT_TOL = {"bf16": 2e-2, "f32": 1e-3}   # max-abs output tolerance
TIE_BAND = 1e-6                          # relative band around the k-th score
# The GPU's TIP scores are float32 sums in a fixed order: |error| is below
# TIP_REL * sum_j |c_j| |x_j| (coefficient c_j, sketch element x_j), with
# TIP_REL = 13.01 * 2^-24 for every sketch shape (n <= 12 roundings on any
# path of the sum, plus the float32 rounding of the coefficients). The
# float64 coefficients themselves differ from the oracle's by rounding only
# (ABS_SLACK).
TIP_REL = 13.01 * 2.0 ** -24
ABS_SLACK = 1e-12


def build(wl, layer=0, n_dom=None, max_len=None, chunks=None, inp=None, kv_on_host=False):
    """Generate a layer's inputs and append them to a fresh cache on the GPU
    (K and V in pinned host memory with kv_on_host)."""
    inp = inp or W.layer_inputs(wl, layer=layer, n_dom=n_dom)
    lp = inp.params
    cache = F.KVCache(wl.batch, wl.n_q_heads, wl.n_kv_heads, lp.dom_idx.shape[1],
                      max_len or wl.ctx_len, wl.dtype, wl.rope_base, lp.dom_idx, kv_on_host=kv_on_host)
    k = W.to_torch(inp.k, "cuda")
    v = W.to_torch(inp.v, "cuda")
    if chunks is None:
        F.fasa_append_kv(cache, k, v, 0)
    else:
        c0 = 0
        for n in chunks:
            F.fasa_append_kv(cache, k[:, :, c0:c0 + n].contiguous(), v[:, :, c0:c0 + n].contiguous(), c0)
            c0 += n
        assert c0 == wl.ctx_len
    q = W.to_torch(inp.q, "cuda")
    torch.cuda.synchronize()
    return inp, cache, q


def stored(t):
    return W.from_torch(t)


def ulp_diff_bf16(a_bits, b_bits):
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    # sign-magnitude -> monotone integer line
    a = np.where(a & 0x8000, -(a & 0x7FFF), a)
    b = np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(a - b)


def check_append(wl, inp, cache, heads, length=None):
    """K rotated at its slot, V copied, sketch = dominant dims of the stored key."""
    L = length or wl.ctx_len
    G = wl.group
    worst = 0
    for (b, g) in heads:
        dom = inp.params.dom_idx[g]
        k_or, v_or, sk_or = O.append_kv(inp.k[b, g, :L], inp.v[b, g, :L], 0, wl.rope_base, dom, wl.dtype)
        k_gpu = stored(cache.k[b, g, :L])
        v_gpu = stored(cache.v[b, g, :L])
        sk_gpu = stored(cache.sketch[b, g, :L])
        n2 = 2 * len(dom)
        if wl.dtype == "bf16":
            d = ulp_diff_bf16(k_gpu, k_or)
            worst = max(worst, int(d.max()))
            assert d.max() <= 1, f"K_rot differs by {d.max()} ulp"
            assert (d == 0).mean() > 0.9999
        else:
            assert np.array_equal(k_gpu, k_or) or np.max(np.abs(k_gpu - k_or) / (np.abs(k_or) + 1e-30)) < 2.4e-7
        assert np.array_equal(v_gpu, v_or)
        # the sketch is the stored key's dominant dims, bit for bit
        assert np.array_equal(sk_gpu[:, :n2], O.sketch_rows(k_gpu, dom))
        assert np.all(W.stored_to_f64(sk_gpu[:, n2:]) == 0)
        if wl.dtype == "bf16":
            assert ulp_diff_bf16(sk_gpu[:, :n2], sk_or).max() <= 1
    return worst


def oracle_scores(wl, inp, cache, b, g, length=None, q_rot=None):
    """The oracle's rotated group queries, TIP scores and sum_j |c_j| |x_j| of
    (b, g) over the first `length` slots; the query sits at position
    `length` (default: the workload's), or q_rot gives it already rotated."""
    L = length or wl.ctx_len
    dom = inp.params.dom_idx[g]
    G = wl.group
    if q_rot is None:
        q_rot = O.rotate_queries(inp.q[b, g * G:(g + 1) * G], wl.q_pos if length is None else length,
                                 wl.rope_base)
    sk = stored(cache.sketch[b, g, :L])[:, :2 * len(dom)]
    s = O.tip_scores(q_rot, sk, dom)
    qd = O.sketch_rows(q_rot, dom)
    abs_sum = np.abs(qd).sum(0) @ np.abs(O.to_f64(sk)).T
    return q_rot, s, abs_sum


def score_err(abs_sum):
    """Bound on |GPU score - exact score| per token; abs_sum >= sum_j |c_j| |x_j|."""
    return (TIP_REL + ABS_SLACK) * abs_sum + 1e-30


def check_scores(gpu, ref, abs_sum):
    gpu = gpu.astype(np.float64)
    tol = score_err(abs_sum)
    err = np.abs(gpu - ref)
    assert np.all(err <= tol), f"score error {np.max(err / tol)} x tolerance"


def check_idx_in_band(gpu_idx, ref_scores, k, err=None):
    """The kept set is an exact top-k_eff selection of some scores that lie
    within err (per token) of the oracle's, up to ties within TIE_BAND
    (relative) of the k-th score: a threshold separates every kept token's
    score + err from every dropped token's score - err. Returns how many
    tokens differ from the oracle's own selection."""
    L = len(ref_scores)
    k_eff = min(k, L)
    or_idx = O.select_critical_set(ref_scores, k)
    gpu_idx = np.asarray(gpu_idx)
    assert len(gpu_idx) == k_eff
    assert np.all(np.diff(gpu_idx) > 0), "indices must be strictly ascending"
    assert gpu_idx[0] >= 0 and gpu_idx[-1] < L, "index out of range"
    e = np.zeros(L) if err is None else np.asarray(err, np.float64)
    s_k = np.sort(ref_scores)[::-1][k_eff - 1]
    band = TIE_BAND * abs(s_k)
    kept = np.zeros(L, bool)
    kept[gpu_idx] = True
    if k_eff < L:
        lo_kept = np.min(ref_scores[kept] + e[kept])
        hi_drop = np.max(ref_scores[~kept] - e[~kept])
        assert lo_kept + band >= hi_drop, (
            f"a dropped token outscores a kept one by {hi_drop - lo_kept:.3e} beyond the error bounds")
    return len(set(gpu_idx.tolist()) ^ set(or_idx.tolist()))


def half_ulp(x, dtype):
    """Half a unit in the last place of |x| in the output dtype (normal range)."""
    mant = 8 if dtype == "bf16" else 24
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - mant)


def check_out(wl, gpu_out, ref_out):
    """Output parity. The output is stored in the cache dtype, so one final
    rounding (half an ulp of the value) is unavoidable; the tolerance (2e-2
    bf16, 1e-3 fp32, max-abs) bounds the error beyond it. A sharper check
    bounds that error by 1e-3 of the rms of the output row."""
    g = W.stored_to_f64(gpu_out)
    hu = half_ulp(np.maximum(np.abs(ref_out), np.abs(g)), wl.dtype)
    excess = float(np.max(np.abs(g - ref_out) - hu))
    assert excess <= OUT_TOL[wl.dtype], f"max abs error beyond rounding {excess}"
    # sharper: beyond the final rounding, float32 accumulation error is tiny
    # against the magnitude of each output row
    row = np.sqrt(np.mean(ref_out ** 2, axis=-1, keepdims=True))
    sharp = np.max((np.abs(g - ref_out) - hu) / (row + 1e-30))
    assert sharp <= 1e-3, f"error beyond rounding is {sharp} of the row's rms"
    return max(excess, 0.0)


def check_gpu_pair(wl, a_stored, b_stored):
    """Two GPU outputs of the same attention (different kernels or orders):
    each holds one final rounding, so they may differ by two half-ulps plus
    float32 accumulation error, which is bounded by 1e-3 of the row's rms."""
    a = W.stored_to_f64(a_stored)
    b = W.stored_to_f64(b_stored)
    hu = half_ulp(np.maximum(np.abs(a), np.abs(b)), wl.dtype)
    row = np.sqrt(np.mean(b ** 2, axis=-1, keepdims=True))
    excess = np.max((np.abs(a - b) - 2 * hu) / (row + 1e-30))
    assert excess <= 1e-3, f"outputs differ by {excess} of the row rms beyond rounding"


def check_decode_heads(wl, inp, cache, q, k, heads, out, idx_out, scores_gpu=None, length=None):
    """Fused decode vs oracle on the given heads; returns worst output error."""
    L = length or wl.ctx_len
    G = wl.group
    out_np = stored(out)
    idx_np = idx_out.cpu().numpy()
    worst = 0.0
    for (b, g) in heads:
        q_rot, s_ref, abs_sum = oracle_scores(wl, inp, cache, b, g, length)
        check_idx_in_band(idx_np[b, g], s_ref, k, score_err(abs_sum))
        if scores_gpu is not None:
            # staged: the selection is exactly the oracle's selection of the GPU's scores
            sg = scores_gpu[b, g].astype(np.float64)
            check_scores(scores_gpu[b, g], s_ref, abs_sum)
            assert np.array_equal(idx_np[b, g], O.select_critical_set(sg, k))
        ref = O.focused_attention(q_rot, stored(cache.k[b, g, :L]), stored(cache.v[b, g, :L]), idx_np[b, g])
        worst = max(worst, check_out(wl, out_np[b, g * G:(g + 1) * G], ref))
    return worst


def all_heads(wl):
    return [(b, g) for b in range(wl.batch) for g in range(wl.n_kv_heads)]


def sample_heads(wl, n, seed=0):
    r = np.random.default_rng(seed)
    hs = all_heads(wl)
    pick = r.choice(len(hs), size=min(n, len(hs)), replace=False)
    return [hs[i] for i in sorted(pick)]
