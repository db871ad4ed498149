"""CPU oracle of the FASA decode hot path: plain, slow, float64.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does, and this module imports nothing from the CUDA package.

It restates, step by step and in float64, what "FASA: Frequency-aware Sparse
Attention" computes at decode time (gist.science technical summary, §2
"Metodologia e Insight Central"; English abstract on the chatpaper.ai page):

1. RoPE splits a head vector into 2-D orthogonal subspaces, the frequency
   chunks (FCs), each rotated at its own angular frequency (§2 "A Descoberta").
   Pairing: FC i = dims (i, i + d/2) ("rotate-half"); theta_i = base^(-2i/d).
2. TIP, online prediction (§2, TIP second bullet): a token's importance is the
   sum of the contributions of the pre-calibrated dominant FCs only. A
   contribution is the FC's share of the query-key dot product,
   P_i(q', k') = q'[i] k'[i] + q'[i+64] k'[i+64]; with grouped-query attention
   the shares of the group's query heads are added.
3. FAC (§2, FAC bullets): take the critical set T_t of the k highest-scoring
   tokens (ties to the lower index; k_eff = min(k, L)) and run full softmax
   attention over exactly those rows, each kept at its original absolute
   position (its key was rotated at that position when it was cached).
4. Dense full-KV attention (the comparison): the same attention over all rows.
5. Multi-query decode (several query tokens per sequence in one step): the
   group sum of step 2 taken over every query row, one shared critical set,
   each row attending over the kept slots not after its position (the
   reading is stated at decode_multi_head).
6. Offline calibration (§2, TIP first bullet): the agreement of each single
   FC's token selection with the full head's over calibration queries picks
   the dominant FCs (the reading of "Contextual Agreement" is stated at the
   calibration functions).

Stored values (the KV cache, the dominant-FC key sketch) are rounded once to
the cache dtype, as the cache stores them. Every function takes and returns
plain numpy arrays.

Pins: every function here is checked by tests against closed forms,
invariants, library routines and brute force; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

D = 128          # head_dim
NFC = D // 2     # number of frequency chunks

# --------------------------------------------------------------- dtype


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 to bfloat16 (nearest, ties to even) in one step.

    Works on the IEEE-754 bit pattern: keep sign, exponent and the top 7
    mantissa bits, round on the 45 dropped bits. Zero maps to (signed) zero;
    values outside the bfloat16 normal range are rejected (the workloads never
    produce them).
    """
    x = np.asarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    sign = (bits >> np.uint64(63)).astype(np.uint32)
    mag = bits & np.uint64(0x7FFFFFFFFFFFFFFF)
    keep = mag >> np.uint64(45)                      # 11-bit exp + 7-bit mantissa
    rem = mag & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rem > half) | ((rem == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    exp64 = (keep >> np.uint64(7)).astype(np.int64)
    mant = (keep & np.uint64(0x7F)).astype(np.uint32)
    zero = mag == 0
    exp16 = exp64 - 1023 + 127
    bad = ~zero & ((exp16 < 1) | (exp16 > 254))
    if np.any(bad):
        raise ValueError("value outside the bfloat16 normal range")
    exp16 = np.where(zero, 0, exp16).astype(np.uint32)
    mant = np.where(zero, 0, mant).astype(np.uint32)
    out = (sign << 15) | (exp16 << 7) | mant
    return out.astype(np.uint16)


def bf16_bits_to_f64(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(stored: np.ndarray) -> np.ndarray:
    """Exact value of stored elements: float32, or bfloat16 given as uint16 bits."""
    stored = np.asarray(stored)
    if stored.dtype == np.uint16:
        return bf16_bits_to_f64(stored)
    return stored.astype(np.float64)


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the cache dtype; returns the stored representation."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == "bf16":
        return f64_to_bf16_bits(x)
    raise ValueError(dtype)


# ---------------------------------------------------------------- RoPE


def rope_frequencies(base: float, d: int = D) -> np.ndarray:
    """Angular frequency of each FC: theta_i = base^(-2i/d), i = 0 .. d/2-1."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def rope_rotate(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate each FC (x[i], x[i+d/2]) of x by the angle pos * theta_i.

    x: [..., d] float64; pos: integer position(s), broadcast against x[..., 0].
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_frequencies(base, d)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def fc_partials(qr: np.ndarray, kr: np.ndarray) -> np.ndarray:
    """P_i = qr[i] kr[i] + qr[i+h] kr[i+h] for every FC i; broadcasts over leading dims."""
    h = qr.shape[-1] // 2
    return qr[..., :h] * kr[..., :h] + qr[..., h:] * kr[..., h:]


# -------------------------------------------------------- append (cache)


def sketch_rows(k_rot: np.ndarray, dom: np.ndarray) -> np.ndarray:
    """Dominant-FC key sketch: for FC j of the dominant list, columns 2j, 2j+1
    hold the rotated key's two dims of that FC (k_rot[:, dom[j]], k_rot[:, dom[j]+h])."""
    h = k_rot.shape[-1] // 2
    dom = np.asarray(dom, dtype=np.int64)
    out = np.empty(k_rot.shape[:-1] + (2 * len(dom),), dtype=k_rot.dtype)
    out[..., 0::2] = k_rot[..., dom]
    out[..., 1::2] = k_rot[..., dom + h]
    return out


def append_kv(k_pre: np.ndarray, v: np.ndarray, pos0: int, base: float, dom, dtype: str):
    """What appending n new tokens at positions pos0.. stores for one KV head.

    k_pre, v: [n, d] stored-dtype inputs. Returns (k_rot, v, sketch) in the
    stored representation: keys rotated at their own positions then rounded;
    values copied unchanged; sketch gathered from the stored rotated keys.
    """
    k64 = to_f64(k_pre)
    pos = pos0 + np.arange(k64.shape[0])
    k_rot = store(rope_rotate(k64, pos, base), dtype)
    v_st = np.array(v, copy=True)
    sk = sketch_rows(k_rot, dom)
    return k_rot, v_st, sk


# ---------------------------------------------------------------- TIP


def rotate_queries(q_pre: np.ndarray, q_pos: int, base: float) -> np.ndarray:
    """Rotated queries in float64 (never rounded): [G, d]."""
    return rope_rotate(to_f64(q_pre), q_pos, base)


def tip_scores(q_rot: np.ndarray, sketch: np.ndarray, dom) -> np.ndarray:
    """Token importance over the dominant FCs, summed over the group's query heads.

    q_rot: [G, d] rotated queries (float64); sketch: [L, 2*n_dom] stored sketch
    rows (as written by append). s[t] = sum_h sum_j (q_h[dom_j] sk[t,2j] +
    q_h[dom_j + h] sk[t,2j+1]).
    """
    sk = to_f64(sketch)
    qd = sketch_rows(np.asarray(q_rot, dtype=np.float64), dom)      # [G, 2n]
    return np.einsum("gc,tc->t", qd, sk)


def select_critical_set(scores: np.ndarray, k: int) -> np.ndarray:
    """T_t: indices of the k_eff = min(k, L) highest scores; ties go to the
    lower token index; returned in ascending index order (int64)."""
    s = np.asarray(scores, dtype=np.float64)
    L = s.shape[0]
    k_eff = min(int(k), L)
    order = np.lexsort((np.arange(L), -s))   # primary: score desc; secondary: index asc
    return np.sort(order[:k_eff])


# ---------------------------------------------------------------- FAC


def focused_attention(q_rot: np.ndarray, k_rot: np.ndarray, v: np.ndarray, idx) -> np.ndarray:
    """Softmax attention of each query head over the rows idx only.

    q_rot [G, d] float64; k_rot, v [L, d] stored; idx [m] (m >= 1).
    Returns [G, d] float64: softmax(q K_idx^T / sqrt(d)) V_idx.
    """
    idx = np.asarray(idx, dtype=np.int64)
    K = to_f64(k_rot)[idx]
    V = to_f64(v)[idx]
    q = np.asarray(q_rot, dtype=np.float64)
    z = (q @ K.T) / np.sqrt(q.shape[-1])
    z = z - z.max(axis=-1, keepdims=True)
    p = np.exp(z)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ V


def dense_attention(q_rot: np.ndarray, k_rot: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Full-KV attention over all L cached rows."""
    return focused_attention(q_rot, k_rot, v, np.arange(np.asarray(k_rot).shape[0]))


# ------------------------------------------------------------ decode


def decode_head(q_pre: np.ndarray, q_pos: int, k_rot: np.ndarray, v: np.ndarray,
                sketch: np.ndarray, dom, k: int, base: float):
    """One (sequence, KV head) of a FASA decode step: TIP -> T_t -> FAC.

    Returns (idx, out [G, d] float64, scores [L] float64).
    """
    q_rot = rotate_queries(q_pre, q_pos, base)
    s = tip_scores(q_rot, sketch, dom)
    idx = select_critical_set(s, k)
    out = focused_attention(q_rot, k_rot, v, idx)
    return idx, out, s



def decode_multi_head(q_pre: np.ndarray, q_pos0: int, k_rot: np.ndarray, v: np.ndarray,
                      sketch: np.ndarray, dom, k: int, base: float):
    """One (sequence, KV head) of a multi-query decode step: n_q query tokens
    (speculative drafts or batched rows), token j at position q_pos0 + j,
    each with the group's G query heads.

    Reading (the pages treat one query at a time): TIP's group sum extends
    over every query row of the KV head, so the n_q * G rows share one
    critical set, T = top-k of s_t = sum_j sum_h sum_{i in D_g} P_i(q'_{j,h},
    k'_t). Each row then attends over the kept slots that are not after its
    own position (t <= q_pos0 + j; every slot when the cache ends before the
    queries, the usual decode). A row left with no slot gets a zero output.

    q_pre: [n_q, G, d] pre-RoPE queries. Returns (idx, out [n_q, G, d]
    float64, scores [L]).
    """
    q_pre = to_f64(q_pre)
    n_q = q_pre.shape[0]
    q_rot = np.stack([rotate_queries(q_pre[j], q_pos0 + j, base) for j in range(n_q)])
    s = tip_scores(q_rot.reshape(-1, q_rot.shape[-1]), sketch, dom)
    idx = select_critical_set(s, k)
    out = np.zeros(q_rot.shape)
    for j in range(n_q):
        seen = idx[idx <= q_pos0 + j]
        if len(seen):
            out[j] = focused_attention(q_rot[j], k_rot, v, seen)
    return idx, out, s


# ------------------------------------------------------- calibration
#
# Offline calibration of the dominant FCs (gist.science technical summary,
# §2, TIP first bullet): per attention head, the "Contextual Agreement" (CA)
# between the attention scores of a single FC and those of the full head,
# over a small calibration set, picks I_dom. The pages give no formula for
# CA. Reading taken here: the agreement of the token sets each one selects
# at the decode budget K, i.e. |Top_K(P_i) ∩ Top_K(full)| summed over the
# calibration queries, with scores and selection exactly as the decode does
# them (group-summed, rounded to float32, ties to the lower index).


def calibration_scores(q_pre_win: np.ndarray, pos_win, k_rot: np.ndarray, base: float) -> np.ndarray:
    """Score planes of one (sequence, KV head) for W calibration queries.

    q_pre_win: [W, G, d] stored pre-RoPE queries; pos_win: [W] positions;
    k_rot: [L, d] stored rotated keys. Returns float32 [W, 65, L]: plane i < 64
    is the single-FC score P_i(t) = qs[i] k[t][i] + qs[i+64] k[t][i+64] with
    qs the group's rotated queries added head by head (head 0 first), and
    plane 64 the full-head score, the 64 planes added in FC order. Every
    product and sum is one float64 operation, rounded to float32 at the end.
    """
    q = to_f64(q_pre_win)
    W, G, d = q.shape
    h = d // 2
    k = to_f64(k_rot)
    out = np.empty((W, NFC + 1, k.shape[0]), np.float32)
    for w in range(W):
        qr = rope_rotate(q[w], int(pos_win[w]), base)           # [G, d]
        qs = qr[0].copy()
        for g in range(1, G):
            qs = qs + qr[g]
        acc = None
        for i in range(h):
            p = qs[i] * k[:, i] + qs[i + h] * k[:, i + h]
            out[w, i] = p.astype(np.float32)
            acc = p if acc is None else acc + p
        out[w, NFC] = acc.astype(np.float32)
    return out


def calibration_counts(planes: np.ndarray, budget: int) -> np.ndarray:
    """Agreement counts of one (sequence, KV head): for each FC i, the number
    of tokens its top-K set shares with the full head's, summed over the W
    calibration queries (K_eff = min(K, L); selection as select_critical_set
    on the float32 planes). planes: [W, 65, L]. Returns int64 [64]."""
    W = planes.shape[0]
    counts = np.zeros(NFC, np.int64)
    for w in range(W):
        full = select_critical_set(planes[w, NFC], budget)
        for i in range(NFC):
            counts[i] += np.intersect1d(select_critical_set(planes[w, i], budget), full).size
    return counts


def dominant_from_counts(counts: np.ndarray, n_dom: int) -> np.ndarray:
    """I_dom: the n_dom FCs of largest agreement, ties to the lower FC index,
    listed in that order (int32)."""
    c = np.asarray(counts, dtype=np.int64)
    order = np.lexsort((np.arange(c.shape[0]), -c))
    return order[:n_dom].astype(np.int32)
