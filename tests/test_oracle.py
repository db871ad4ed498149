"""Pins of the CPU oracle to facts fixed outside it.

Each ``check_*`` function compares the oracle with something it does not
share code with: a library routine (torch's bfloat16 cast, the RoPE of
transformers' Llama, torch's scaled_dot_product_attention and topk), a closed
form (complex rotation, relative-position dependence of an FC's share), an
invariant (orthogonal FC decomposition sums to the dot product, GQA
linearity, norm preservation) or brute force on tiny inputs. The mutation test
at the bottom plants plausible mistakes in the oracle and checks that at least
one pin fails for each.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.fasa_oracle as O

RNG = np.random.default_rng(12345)


def _close(a, b, rtol=1e-12, atol=1e-12):
    return np.allclose(a, b, rtol=rtol, atol=atol)


# ------------------------------------------------------------ bf16 storage

def check_bf16_vs_torch(m):
    x = (RNG.standard_normal(20000) * np.exp(RNG.uniform(-20, 20, 20000))).astype(np.float32)
    x[:4] = [0.0, -0.0, 1.0, -3.5]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = m.f64_to_bf16_bits(x.astype(np.float64))
    return np.array_equal(got, want)


def _exact_bf16(v: Fraction) -> Fraction:
    """Nearest bfloat16 (8 significant bits), ties to even, by exact arithmetic."""
    if v == 0:
        return Fraction(0)
    sgn = -1 if v < 0 else 1
    a = abs(v)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    scaled = a * 128                      # in [128, 256)
    lo = scaled.numerator // scaled.denominator
    frac = scaled - lo
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sgn * Fraction(lo, 128) * Fraction(2) ** e


def check_bf16_halfway_exact(m):
    # values exactly at, and a hair (below float32 resolution) around, bf16 ties
    vals = []
    for mant in [128, 129, 200, 255]:
        for e in [-10, 0, 3]:
            tie = Fraction(2 * mant + 1, 256) * Fraction(2) ** e
            for eps in [Fraction(0), Fraction(1, 2 ** 40), -Fraction(1, 2 ** 40)]:
                vals.append(tie + eps * Fraction(2) ** e)
    xs = np.array([float(v) for v in vals], dtype=np.float64)
    got = m.to_f64(m.f64_to_bf16_bits(xs))
    want = np.array([float(_exact_bf16(Fraction(float(v)))) for v in vals])
    return np.array_equal(got, want)


# ------------------------------------------------------------------- RoPE

def check_rope_vs_complex(m):
    base = 5e5
    x = RNG.standard_normal((6, 128))
    pos = np.array([0, 1, 5, 4096, 32768, 131071])
    got = m.rope_rotate(x, pos, base)
    theta = 1.0 / base ** (np.arange(0, 128, 2, dtype=np.float64) / 128)
    z = (x[:, :64] + 1j * x[:, 64:]) * np.exp(1j * pos[:, None] * theta)
    want = np.concatenate([z.real, z.imag], axis=1)
    return _close(got, want, rtol=1e-9, atol=1e-9)


_HF = {}


def _hf_rope(base):
    if base not in _HF:
        from transformers import LlamaConfig
        from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb
        cfg = LlamaConfig(hidden_size=256, num_attention_heads=2, head_dim=128,
                          rope_theta=float(base), max_position_embeddings=1 << 20)
        _HF[base] = (LlamaRotaryEmbedding(cfg), apply_rotary_pos_emb)
    return _HF[base]


def check_rope_vs_transformers(m):
    ok = True
    for base in (1e4, 5e5):
        rot, apply = _hf_rope(base)
        # the library evaluates angles in float32, so compare at small positions
        pos = torch.tensor([[0, 1, 2, 3, 17, 63, 100]])
        x = torch.from_numpy(RNG.standard_normal((1, 1, 7, 128)))
        cos, sin = rot(x, pos)
        want, _ = apply(x, x, cos, sin)
        got = m.rope_rotate(x.numpy()[0, 0], pos.numpy()[0], base)
        ok &= _close(got, want.numpy()[0, 0], rtol=0, atol=2e-5)
        ok &= _close(m.rope_frequencies(base), rot.inv_freq.double().numpy(), rtol=2e-6, atol=0)
    return bool(ok)


def check_rope_invariants(m):
    x = RNG.standard_normal((9, 128))
    ok = _close(m.rope_rotate(x, 0, 1e4), x)                      # identity at 0
    r = m.rope_rotate(x, 777, 1e4)
    n0 = x[:, :64] ** 2 + x[:, 64:] ** 2
    n1 = r[:, :64] ** 2 + r[:, 64:] ** 2
    ok &= _close(n0, n1, rtol=1e-12)                               # per-FC norm kept
    ok &= _close(m.rope_rotate(m.rope_rotate(x, 300, 1e4), 477, 1e4), r, rtol=1e-9, atol=1e-9)
    return bool(ok)


# -------------------------------------------------------------- FC shares

def check_fc_partials_sum_to_dot(m):
    q = RNG.standard_normal((5, 128))
    k = RNG.standard_normal((5, 128))
    P = m.fc_partials(q, k)
    return P.shape == (5, 64) and _close(P.sum(-1), np.einsum("ij,ij->i", q, k))


def check_fc_partial_closed_form(m):
    base = 1e4
    q = RNG.standard_normal(128)
    k = RNG.standard_normal(128)
    ok = True
    th = 1.0 / base ** (np.arange(0, 128, 2) / 128.0)
    qc = q[:64] + 1j * q[64:]
    kc = k[:64] + 1j * k[64:]
    for p, t in [(4096, 0), (4096, 4095), (100, 37), (37, 100)]:
        P = m.fc_partials(m.rope_rotate(q, p, base), m.rope_rotate(k, t, base))
        want = np.real(qc * np.conj(kc) * np.exp(1j * (p - t) * th))
        ok &= _close(P, want, rtol=1e-9, atol=1e-9)
        # only the relative position matters
        P2 = m.fc_partials(m.rope_rotate(q, p + 500, base), m.rope_rotate(k, t + 500, base))
        ok &= _close(P, P2, rtol=1e-8, atol=1e-8)
    return bool(ok)


# -------------------------------------------------------------------- TIP

def _head(L=40, G=3, base=1e4, seed=0, dtype="f32"):
    r = np.random.default_rng(seed)
    qpre = r.standard_normal((G, 128)).astype(np.float32)
    kpre = r.standard_normal((L, 128)).astype(np.float32)
    v = r.standard_normal((L, 128)).astype(np.float32)
    if dtype == "bf16":
        qpre = O.f64_to_bf16_bits(qpre.astype(np.float64))
        kpre = O.f64_to_bf16_bits(kpre.astype(np.float64))
        v = O.f64_to_bf16_bits(v.astype(np.float64))
    return qpre, kpre, v


def check_tip_all_fcs_is_dot(m):
    qpre, kpre, v = _head()
    dom = np.arange(64)
    k_rot, _, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
    qr = m.rotate_queries(qpre, 40, 1e4)
    s = m.tip_scores(qr, sk, dom)
    want = (qr @ m.to_f64(k_rot).T).sum(0)
    return _close(s, want, rtol=1e-10, atol=1e-10)


def check_tip_subset_is_partial_sum(m):
    qpre, kpre, v = _head(seed=1)
    dom = np.array([5, 63, 0, 17, 40])
    k_rot, _, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
    qr = m.rotate_queries(qpre, 40, 1e4)
    P = m.fc_partials(qr[:, None, :], m.to_f64(k_rot)[None, :, :])   # [G, L, 64]
    want = P[:, :, dom].sum(axis=(0, 2))
    return _close(m.tip_scores(qr, sk, dom), want, rtol=1e-10, atol=1e-10)


def check_tip_gqa_linear(m):
    qpre, kpre, v = _head(seed=2, G=4)
    dom = np.array([3, 9, 27])
    _, _, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
    qr = m.rotate_queries(qpre, 40, 1e4)
    s_group = m.tip_scores(qr, sk, dom)
    s_sum = m.tip_scores(qr.sum(0, keepdims=True), sk, dom)
    return _close(s_group, s_sum, rtol=1e-10, atol=1e-10)


def check_tip_brute_force(m):
    qpre, kpre, v = _head(L=12, G=2, seed=3)
    dom = [7, 1, 50]
    k_rot, _, sk = m.append_kv(kpre, v, 0, 1e4, np.array(dom), "f32")
    qr = m.rotate_queries(qpre, 12, 1e4)
    kr = m.to_f64(k_rot)
    want = []
    for t in range(12):
        acc = 0.0
        for h in range(2):
            for i in dom:
                acc += qr[h][i] * kr[t][i] + qr[h][i + 64] * kr[t][i + 64]
        want.append(acc)
    return _close(m.tip_scores(qr, sk, np.array(dom)), np.array(want), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- select

def check_select_brute_force(m):
    ok = True
    r = np.random.default_rng(4)
    for L, k in [(1, 1), (7, 3), (20, 5), (33, 33), (10, 25), (40, 1)]:
        s = r.integers(-3, 4, L).astype(np.float64)          # many exact ties
        want = []
        for t in range(L):
            rank = sum(1 for u in range(L) if s[u] > s[t] or (s[u] == s[t] and u < t))
            if rank < min(k, L):
                want.append(t)
        got = m.select_critical_set(s, k)
        ok &= list(got) == want
    return bool(ok)


def check_select_permutation(m):
    r = np.random.default_rng(5)
    s = r.standard_normal(200)
    perm = r.permutation(200)
    a = set(m.select_critical_set(s, 17).tolist())
    b = set(perm[m.select_critical_set(s[perm], 17)].tolist())
    return a == b and len(a) == 17


# -------------------------------------------------------------------- FAC

def _sdpa(q, K, V):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()


def check_dense_vs_sdpa(m):
    r = np.random.default_rng(6)
    q = r.standard_normal((4, 128)) * 0.3
    K = r.standard_normal((50, 128))
    V = r.standard_normal((50, 128))
    return _close(m.dense_attention(q, K, V), _sdpa(q, K, V), rtol=1e-10, atol=1e-12)


def check_focused_special_cases(m):
    r = np.random.default_rng(7)
    q = r.standard_normal((3, 128)) * 0.3
    K = r.standard_normal((30, 128))
    V = r.standard_normal((30, 128))
    ok = _close(m.focused_attention(q, K, V, np.arange(30)), m.dense_attention(q, K, V))
    idx = np.array([2, 9, 11, 20])
    o = m.focused_attention(q, K, V, idx)
    ok &= _close(o, _sdpa(q, K[idx], V[idx]), rtol=1e-10, atol=1e-12)
    ok &= bool(np.all(o <= V[idx].max(0) + 1e-12) and np.all(o >= V[idx].min(0) - 1e-12))
    one = m.focused_attention(q, K, V, np.array([13]))
    ok &= _close(one, np.repeat(V[13][None], 3, 0))
    return bool(ok)


# ------------------------------------------------------------- end to end

def check_e2e_all_fc_full_k_is_dense(m):
    qpre, kpre, v = _head(L=64, G=2, seed=8)
    dom = np.arange(64)
    k_rot, v_st, sk = m.append_kv(kpre, v, 0, 5e5, dom, "f32")
    idx, out, _ = m.decode_head(qpre, 64, k_rot, v_st, sk, dom, 64, 5e5)
    qr = m.rope_rotate(m.to_f64(qpre), 64, 5e5)
    want = _sdpa(qr, m.to_f64(k_rot), m.to_f64(v_st))
    return list(idx) == list(range(64)) and _close(out, want, rtol=1e-9, atol=1e-12)


def check_e2e_all_fc_topk_exact(m):
    qpre, kpre, v = _head(L=64, G=1, seed=9)
    dom = np.arange(64)
    k_rot, v_st, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
    idx, out, _ = m.decode_head(qpre, 64, k_rot, v_st, sk, dom, 9, 1e4)
    qr = m.rope_rotate(m.to_f64(qpre), 64, 1e4)
    logits = torch.from_numpy(qr @ m.to_f64(k_rot).T)[0]
    top = np.sort(torch.topk(logits, 9).indices.numpy())
    want = _sdpa(qr, m.to_f64(k_rot)[top], m.to_f64(v_st)[top])
    return list(idx) == list(top) and _close(out, want, rtol=1e-9, atol=1e-12)


def _multi_case(L=40, n_q=4, G=2, seed=30, base=1e4):
    r = np.random.default_rng(seed)
    qpre = r.standard_normal((n_q, G, 128)).astype(np.float32)
    kpre = r.standard_normal((L, 128)).astype(np.float32)
    v = r.standard_normal((L, 128)).astype(np.float32)
    return qpre, kpre, v


def check_multi_one_query_is_decode(m):
    qpre, kpre, v = _multi_case(n_q=1, seed=31)
    dom = np.array([4, 17, 60])
    k_rot, v_st, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
    a = m.decode_multi_head(qpre, 40, k_rot, v_st, sk, dom, 9, 1e4)
    b = m.decode_head(qpre[0], 40, k_rot, v_st, sk, dom, 9, 1e4)
    return list(a[0]) == list(b[0]) and np.array_equal(a[1][0], b[1]) and np.array_equal(a[2], b[2])


def check_multi_scores_add_over_positions(m):
    # the shared score is the sum of the per-token group scores, each token
    # rotated at its own position (dominant dims by brute force)
    qpre, kpre, v = _multi_case(L=30, n_q=3, G=2, seed=32)
    dom = [9, 2, 33]
    k_rot, v_st, sk = m.append_kv(kpre, v, 0, 1e4, np.array(dom), "f32")
    _, _, s = m.decode_multi_head(qpre, 30, k_rot, v_st, sk, np.array(dom), 5, 1e4)
    kr = m.to_f64(k_rot)
    want = np.zeros(30)
    for j in range(3):
        ang = (30 + j) * 1e4 ** (-2.0 * np.arange(64) / 128)
        for h in range(2):
            z = (qpre[j, h, :64] + 1j * qpre[j, h, 64:]).astype(np.complex128) * np.exp(1j * ang)
            for i in dom:
                want += z[i].real * kr[:, i] + z[i].imag * kr[:, i + 64]
    return _close(s, want, rtol=1e-10, atol=1e-10)


def check_multi_causal_vs_sdpa(m):
    # drafts already in the cache: query j at position 36 + j sees slots
    # 0 .. 36 + j; all FCs and k = L reduce it to masked dense attention
    qpre, kpre, v = _multi_case(L=40, n_q=4, G=2, seed=33)
    dom = np.arange(64)
    k_rot, v_st, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
    idx, out, _ = m.decode_multi_head(qpre, 36, k_rot, v_st, sk, dom, 40, 1e4)
    ok = list(idx) == list(range(40))
    for j in range(4):
        qr = m.rope_rotate(m.to_f64(qpre[j]), 36 + j, 1e4)
        mask = torch.from_numpy(np.arange(40) <= 36 + j)[None].expand(2, 40)
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr)[None], torch.from_numpy(m.to_f64(k_rot))[None],
            torch.from_numpy(m.to_f64(v_st))[None], attn_mask=mask[None])[0].numpy()
        ok &= _close(out[j], want, rtol=1e-9, atol=1e-12)
    return bool(ok)


def check_multi_masked_row_without_slots_is_zero(m):
    # one kept token after the first query's position: that row is zero, the
    # rows that see it get its V row (the first seed where the best token is
    # slot 10 or 11 of 12)
    dom = np.arange(64)
    for seed in range(34, 400):
        qpre, kpre, v = _multi_case(L=12, n_q=3, G=1, seed=seed)
        k_rot, v_st, sk = m.append_kv(kpre, v, 0, 1e4, dom, "f32")
        idx, out, s = m.decode_multi_head(qpre, 9, k_rot, v_st, sk, dom, 1, 1e4)
        if idx[0] > 9:
            break
    else:
        return False
    t = int(idx[0])
    ok = int(np.argmax(s)) == t and np.all(out[0] == 0.0)
    for j in (1, 2):
        want = m.to_f64(v_st)[t][None] if t <= 9 + j else np.zeros((1, 128))
        ok &= _close(out[j], want)
    return bool(ok)


def check_append_positions(m):
    qpre, kpre, v = _head(L=30, seed=10, dtype="bf16")
    dom = np.array([0, 2, 4])
    a = m.append_kv(kpre, v, 0, 1e4, dom, "bf16")
    b1 = m.append_kv(kpre[:11], v[:11], 0, 1e4, dom, "bf16")
    b2 = m.append_kv(kpre[11:], v[11:], 11, 1e4, dom, "bf16")
    ok = all(np.array_equal(x, np.concatenate([y, z])) for x, y, z in zip(a, b1, b2))
    # slot t holds the key rotated at absolute position t
    t = 23
    ok &= np.array_equal(a[0][t], m.store(m.rope_rotate(m.to_f64(kpre[t]), t, 1e4), "bf16"))
    return bool(ok)


# ------------------------------------------------------------ calibration

def _calib_case(L=40, G=3, W=3, seed=21, dtype="f32", base=1e4):
    r = np.random.default_rng(seed)
    q = (r.standard_normal((W, G, 128)) * np.exp(r.standard_normal(128))).astype(np.float32)
    kpre = (r.standard_normal((L, 128)) * np.exp(r.standard_normal(128))).astype(np.float32)
    q = O.store(q, dtype)
    k_rot = O.store(O.rope_rotate(O.to_f64(O.store(kpre, dtype)), np.arange(L), base), dtype)
    pos = L + np.arange(W) * 7
    return q, pos, k_rot, base


def _complex_planes(q, pos, k_rot, base):
    """Group-summed FC shares by complex rotation: z = (x_i + j x_{i+64}) e^{j p theta_i}."""
    qq = O.to_f64(q)
    kk = O.to_f64(k_rot)
    theta = np.power(float(base), -np.arange(64) / 64.0)
    kz = kk[:, :64] + 1j * kk[:, 64:]
    out = []
    for w in range(qq.shape[0]):
        z = (qq[w, :, :64] + 1j * qq[w, :, 64:]) * np.exp(1j * pos[w] * theta)   # [G, 64]
        share = np.real(z.sum(0)[None, :] * np.conj(kz))                           # [L, 64]
        out.append(np.concatenate([share.T, share.sum(1)[None, :]], axis=0))      # [65, L]
    return np.stack(out)


def check_calib_planes_closed_form(m):
    q, pos, k_rot, base = _calib_case(dtype="bf16")
    got = m.calibration_scores(q, pos, k_rot, base).astype(np.float64)
    want = _complex_planes(q, pos, k_rot, base)
    scale = np.abs(want).max()
    return got.shape == (3, 65, 40) and np.abs(got - want).max() <= 1e-6 * scale


def check_calib_planes_match_tip(m):
    q, pos, k_rot, base = _calib_case(L=33, G=2, W=2, seed=22)
    planes = m.calibration_scores(q, pos, k_rot, base)
    ok = True
    for w in range(2):
        qr = m.rotate_queries(q[w], int(pos[w]), base)
        full = m.tip_scores(qr, m.sketch_rows(k_rot, np.arange(64)), np.arange(64))
        ok &= np.allclose(planes[w, 64], full, rtol=2e-7, atol=1e-6 * np.abs(full).max())
        for i in (0, 17, 63):
            one = m.tip_scores(qr, m.sketch_rows(k_rot, np.array([i])), np.array([i]))
            ok &= np.allclose(planes[w, i], one, rtol=2e-7, atol=1e-6 * np.abs(one).max() + 1e-30)
    return bool(ok)


def check_calib_counts_brute_force(m):
    r = np.random.default_rng(23)
    W, L, K = 3, 24, 5
    planes = r.standard_normal((W, 65, L)).astype(np.float32)
    planes[0, 3, 7] = planes[0, 3, 11] = np.sort(planes[0, 3])[-5]   # a tie at the boundary
    planes[1, 64, 2] = planes[1, 64, 20] = np.sort(planes[1, 64])[-5]
    want = np.zeros(64, np.int64)
    for w in range(W):
        rank = lambda row: {t for _, t in sorted((-float(row[t]), t) for t in range(L))[:K]}
        full = rank(planes[w, 64])
        for i in range(64):
            want[i] += len(rank(planes[w, i]) & full)
    return np.array_equal(m.calibration_counts(planes, K), want)


def check_calib_single_fc_query(m):
    q, pos, k_rot, base = _calib_case(L=60, G=2, W=2, seed=24)
    j = 37
    mask = np.zeros(128, bool)
    mask[[j, j + 64]] = True
    q = np.where(mask, q, np.float32(0))
    planes = m.calibration_scores(q, pos, k_rot, base)
    c = m.calibration_counts(planes, 8)
    others = np.delete(c, j)
    return (np.array_equal(planes[:, j], planes[:, 64]) and c[j] == 2 * 8 and others.max() < c[j]
            and m.dominant_from_counts(c, 1)[0] == j)


def check_calib_budget_covers_all(m):
    q, pos, k_rot, base = _calib_case(L=12, G=1, W=2, seed=25)
    c = m.calibration_counts(m.calibration_scores(q, pos, k_rot, base), 50)
    return np.array_equal(c, np.full(64, 2 * 12)) and list(m.dominant_from_counts(c, 4)) == [0, 1, 2, 3]


def check_dominant_ties(m):
    c = np.zeros(64, np.int64)
    c[[1, 2, 4]] = 7
    c[0] = 5
    c[3] = 1
    return (list(m.dominant_from_counts(c, 3)) == [1, 2, 4]
            and list(m.dominant_from_counts(c, 6)) == [1, 2, 4, 0, 3, 5])


PINS = [check_bf16_vs_torch, check_bf16_halfway_exact, check_rope_vs_complex,
        check_rope_vs_transformers, check_rope_invariants, check_fc_partials_sum_to_dot,
        check_fc_partial_closed_form, check_tip_all_fcs_is_dot, check_tip_subset_is_partial_sum,
        check_tip_gqa_linear, check_tip_brute_force, check_select_brute_force,
        check_select_permutation, check_dense_vs_sdpa, check_focused_special_cases,
        check_e2e_all_fc_full_k_is_dense, check_e2e_all_fc_topk_exact, check_append_positions,
        check_calib_planes_closed_form, check_calib_planes_match_tip, check_calib_counts_brute_force,
        check_calib_single_fc_query, check_calib_budget_covers_all, check_dominant_ties,
        check_multi_one_query_is_decode, check_multi_scores_add_over_positions, check_multi_causal_vs_sdpa,
        check_multi_masked_row_without_slots_is_zero]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    assert pin(O)


def test_golden_fixture_matches_oracle():
    """Regression fixture written by tests/golden/make_golden.py (oracle only)."""
    import json, os
    from tests.golden.make_golden import compute_golden
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_decode.json")
    with open(path) as f:
        stored = json.load(f)
    fresh = compute_golden()
    assert stored["idx"] == fresh["idx"]
    np.testing.assert_allclose(stored["out"], fresh["out"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(stored["scores"], fresh["scores"], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- mutations

def _mut_rope_sign(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * O.rope_frequencies(base, x.shape[-1])
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :64], x[..., 64:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)


def _mut_rope_adjacent(x, pos, base):
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * O.rope_frequencies(base, x.shape[-1])
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _mut_freq(base, d=128):
    return np.power(float(base), -1.0 * np.arange(d // 2) / d)


def _mut_partials(qr, kr):
    return qr[..., :64] * kr[..., :64]


def _mut_tip_head0(q_rot, sketch, dom):
    return _orig_tip(q_rot[:1], sketch, dom)


def _mut_select_high_tie(scores, k):
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((-np.arange(len(s)), -s))
    return np.sort(order[:min(k, len(s))])


def _mut_no_scale(q_rot, k_rot, v, idx):
    idx = np.asarray(idx)
    K, V = O.to_f64(k_rot)[idx], O.to_f64(v)[idx]
    z = q_rot @ K.T
    p = np.exp(z - z.max(-1, keepdims=True))
    return (p / p.sum(-1, keepdims=True)) @ V


def _mut_sketch(k_rot, dom):
    dom = np.asarray(dom)
    out = np.empty(k_rot.shape[:-1] + (2 * len(dom),), dtype=k_rot.dtype)
    out[..., 0::2] = k_rot[..., dom]
    out[..., 1::2] = k_rot[..., (dom + 1) % 128]
    return out


def _mut_append_pos(k_pre, v, pos0, base, dom, dtype):
    return _orig_append(k_pre, v, pos0 + 1, base, dom, dtype)


def _mut_bf16_trunc(x):
    x = np.asarray(x, np.float64).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _mut_calib_adjacent(q_pre_win, pos_win, k_rot, base):
    perm = np.empty(128, np.int64)
    perm[0::2], perm[1::2] = np.arange(64), np.arange(64, 128)
    return _orig_calib_scores(q_pre_win[..., perm], pos_win, k_rot[..., perm], base)


def _mut_calib_head0(q_pre_win, pos_win, k_rot, base):
    return _orig_calib_scores(q_pre_win[:, :1], pos_win, k_rot, base)


def _mut_calib_abs(planes, budget):
    return _orig_calib_counts(np.abs(planes), budget)


def _mut_dominant_high_tie(counts, n_dom):
    c = np.asarray(counts, dtype=np.int64)
    return np.lexsort((-np.arange(c.shape[0]), -c))[:n_dom].astype(np.int32)


_orig_calib_scores = O.calibration_scores
_orig_calib_counts = O.calibration_counts


_orig_append = O.append_kv
_orig_tip = O.tip_scores

def _mut_multi_one_position(q_pre, q_pos0, k_rot, v, sketch, dom, k, base):
    q = O.to_f64(q_pre)
    qr = np.stack([O.rotate_queries(q[j], q_pos0, base) for j in range(q.shape[0])])
    s = O.tip_scores(qr.reshape(-1, 128), sketch, dom)
    idx = O.select_critical_set(s, k)
    return idx, np.stack([O.focused_attention(qr[j], k_rot, v, idx) for j in range(q.shape[0])]), s


def _mut_multi_no_mask(q_pre, q_pos0, k_rot, v, sketch, dom, k, base):
    q = O.to_f64(q_pre)
    qr = np.stack([O.rotate_queries(q[j], q_pos0 + j, base) for j in range(q.shape[0])])
    s = O.tip_scores(qr.reshape(-1, 128), sketch, dom)
    idx = O.select_critical_set(s, k)
    return idx, np.stack([O.focused_attention(qr[j], k_rot, v, idx) for j in range(q.shape[0])]), s


MUTANTS = {
    "multi_rotates_every_token_at_first_position": ("decode_multi_head", _mut_multi_one_position),
    "multi_without_causal_mask": ("decode_multi_head", _mut_multi_no_mask),
    "rope_rotates_backwards": ("rope_rotate", _mut_rope_sign),
    "rope_adjacent_pairs": ("rope_rotate", _mut_rope_adjacent),
    "rope_theta_exponent": ("rope_frequencies", _mut_freq),
    "fc_partial_drops_half": ("fc_partials", _mut_partials),
    "tip_drops_group_heads": ("tip_scores", _mut_tip_head0),
    "select_ties_to_higher_index": ("select_critical_set", _mut_select_high_tie),
    "attention_without_scale": ("focused_attention", _mut_no_scale),
    "sketch_wrong_pair": ("sketch_rows", _mut_sketch),
    "append_position_off_by_one": ("append_kv", _mut_append_pos),
    "bf16_truncates": ("f64_to_bf16_bits", _mut_bf16_trunc),
    "calib_adjacent_pairs": ("calibration_scores", _mut_calib_adjacent),
    "calib_drops_group_heads": ("calibration_scores", _mut_calib_head0),
    "calib_selects_magnitude": ("calibration_counts", _mut_calib_abs),
    "calib_dominant_ties_to_higher_fc": ("dominant_from_counts", _mut_dominant_high_tie),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in PINS:
        try:
            ok = pin(O)
        except Exception:
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
