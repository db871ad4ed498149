"""GPU parity: every stage of the CUDA path against the CPU oracle, through the C ABI.

Stages are checked both alone (each fed the GPU's own output of the previous
stage) and fused (fasa_decode). Small cases span several tiles with ragged
tails; the full workload sizes are checked on sampled heads.
"""
import numpy as np
import pytest
import torch

import oracle.fasa_oracle as O
from rope_frequency_chunk_b200 import fasa as F
from rope_frequency_chunk_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

C = W.CONFIGS


@pytest.fixture(autouse=True)
def _clean_status():
    F.fasa_device_status(clear=True)
    yield
    assert F.fasa_device_status(clear=True) == 0


# small variants: ragged lengths, every group size and n_dom family
SMALL = {
    "c1": C["c1"],
    "c2_ragged": C["c2"].replace(ctx_len=5003),
    "c4_g7": C["c4"].replace(ctx_len=3001, batch=2, k=567, n_dom=8),
    "g16_f32": C["c1"].replace(name="g16", n_q_heads=32, n_kv_heads=2, ctx_len=1500, n_dom=5, k=100),
    "g1_bf16_ndom64": C["c2"].replace(name="g1", n_q_heads=3, n_kv_heads=3, ctx_len=777, n_dom=64, k=64),
    "bf16_ndom1": C["c2"].replace(name="nd1", batch=2, n_q_heads=8, n_kv_heads=2, ctx_len=2049, n_dom=1, k=31),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_append_matches_oracle(name):
    wl = SMALL[name]
    inp, cache, q = U.build(wl, chunks=None)
    U.check_append(wl, inp, cache, U.all_heads(wl))


def test_append_in_ragged_chunks_equals_one_shot():
    wl = SMALL["c2_ragged"]
    inp = W.layer_inputs(wl)
    _, a, _ = U.build(wl, inp=inp)
    _, b, _ = U.build(wl, inp=inp, chunks=[1, 2, 1000, 7, 3993], max_len=6000)
    L = wl.ctx_len
    assert torch.equal(a.k[:, :, :L], b.k[:, :, :L]) and torch.equal(a.v[:, :, :L], b.v[:, :, :L])
    assert torch.equal(a.sketch[:, :, :L], b.sketch[:, :, :L])


@pytest.mark.parametrize("name", list(SMALL))
def test_score_matches_oracle(name):
    wl = SMALL[name]
    inp, cache, q = U.build(wl)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    for (b, g) in U.all_heads(wl):
        _, ref, abs_sum = U.oracle_scores(wl, inp, cache, b, g)
        U.check_scores(s[b, g], ref, abs_sum)


def _select_cases():
    r = np.random.default_rng(7)
    cases = []
    for rows, L, k in [(1, 1, 1), (1, 7, 3), (3, 100, 100), (3, 100, 250), (2, 4096, 256), (5, 40001, 1),
                       (4, 40001, 5000), (1, 300000, 2048), (64, 16384, 1024), (2, 2 ** 19, 9000)]:
        s = r.standard_normal((rows, L)).astype(np.float32)
        cases.append((f"normal_{rows}x{L}_k{k}", s, k))
    ties = r.integers(-3, 3, (3, 20000)).astype(np.float32)
    ties[0, :50] = -0.0
    ties[0, 50:100] = 0.0
    cases.append(("many_ties", ties, 777))
    cases.append(("all_equal", np.full((2, 5000), 1.5, np.float32), 300))
    cases.append(("zeros_signed", np.where(r.random((1, 3000)) < 0.5, -0.0, 0.0).astype(np.float32), 10))
    neg = -np.abs(r.standard_normal((2, 9999))).astype(np.float32)
    cases.append(("all_negative", neg, 4000))
    return cases


@pytest.mark.parametrize("name,scores,k", _select_cases(), ids=[c[0] for c in _select_cases()])
def test_select_is_exact(name, scores, k):
    idx = F.fasa_select_topk(torch.from_numpy(scores).cuda(), k).cpu().numpy()
    for r in range(scores.shape[0]):
        want = O.select_critical_set(scores[r].astype(np.float64), k)
        assert np.array_equal(idx[r], want), name


@pytest.mark.parametrize("name", list(SMALL))
def test_sparse_attend_matches_oracle(name):
    wl = SMALL[name]
    inp, cache, q = U.build(wl)
    r = np.random.default_rng(3)
    n_idx = min(wl.k, wl.ctx_len)
    idx = np.stack([np.stack([r.choice(wl.ctx_len, n_idx, replace=False) for _ in range(wl.n_kv_heads)])
                    for _ in range(wl.batch)]).astype(np.int32)
    idx[0, 0, :3] = idx[0, 0, 0]  # duplicates count twice; order is free
    out = F.fasa_sparse_attend(cache, wl.ctx_len, q, wl.q_pos, torch.from_numpy(idx).cuda())
    out_np = U.stored(out)
    G = wl.group
    for (b, g) in U.all_heads(wl):
        q_rot = O.rotate_queries(inp.q[b, g * G:(g + 1) * G], wl.q_pos, wl.rope_base)
        ref = O.focused_attention(q_rot, U.stored(cache.k[b, g]), U.stored(cache.v[b, g]), idx[b, g])
        U.check_out(wl, out_np[b, g * G:(g + 1) * G], ref)


def test_sparse_attend_skips_bad_index():
    wl = SMALL["c2_ragged"]
    inp, cache, q = U.build(wl)
    idx = np.tile(np.arange(0, 40, dtype=np.int32), (1, wl.n_kv_heads, 1))
    idx[0, 1, 5] = wl.ctx_len        # out of range -> skipped, status recorded
    idx[0, 2, 7] = -3
    out = F.fasa_sparse_attend(cache, wl.ctx_len, q, wl.q_pos, torch.from_numpy(idx).cuda())
    assert F.fasa_device_status(clear=True) == 7
    G = wl.group
    for g in (1, 2):
        keep = [t for t in idx[0, g] if 0 <= t < wl.ctx_len]
        q_rot = O.rotate_queries(inp.q[0, g * G:(g + 1) * G], wl.q_pos, wl.rope_base)
        ref = O.focused_attention(q_rot, U.stored(cache.k[0, g]), U.stored(cache.v[0, g]), keep)
        U.check_out(wl, U.stored(out)[0, g * G:(g + 1) * G], ref)


@pytest.mark.parametrize("name", list(SMALL))
def test_dense_matches_oracle(name):
    wl = SMALL[name]
    inp, cache, q = U.build(wl)
    out = U.stored(F.fasa_dense_decode(cache, wl.ctx_len, q, wl.q_pos))
    G = wl.group
    for (b, g) in U.all_heads(wl):
        q_rot = O.rotate_queries(inp.q[b, g * G:(g + 1) * G], wl.q_pos, wl.rope_base)
        ref = O.dense_attention(q_rot, U.stored(cache.k[b, g]), U.stored(cache.v[b, g]))
        U.check_out(wl, out[b, g * G:(g + 1) * G], ref)


PATHS = {"fused": F.DECODE_FUSED, "staged": F.DECODE_STAGED}


@pytest.fixture(params=list(PATHS))
def path(request):
    """Runs a decode test under each launch plan of fasa_decode."""
    F.fasa_set_decode_path(PATHS[request.param])
    yield request.param
    F.fasa_set_decode_path(F.DECODE_AUTO)


def _skip_unless_plan(wl, path):
    if path == "fused" and wl.dtype != "bf16":
        pytest.skip("the fused decode takes bf16 caches only")


def _decode(wl, cache, q, k, length=None):
    L = length or wl.ctx_len
    idx = torch.empty(wl.batch, wl.n_kv_heads, min(k, L), dtype=torch.int32, device="cuda")
    out = F.fasa_decode(cache, L, q, L, k, idx_out=idx)
    return out, idx


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_matches_oracle(name, path):
    wl = SMALL[name]
    _skip_unless_plan(wl, path)
    inp, cache, q = U.build(wl)
    out, idx = _decode(wl, cache, q, wl.k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, wl.k, U.all_heads(wl), out, idx, scores_gpu=s)


@pytest.mark.parametrize("k_of_L", ["one", "equal", "more", "half"])
def test_decode_budget_edges(k_of_L, path):
    wl = SMALL["c2_ragged"].replace(ctx_len=1999)
    L = wl.ctx_len
    k = {"one": 1, "equal": L, "more": L + 500, "half": L // 2}[k_of_L]
    inp, cache, q = U.build(wl)
    out, idx = _decode(wl, cache, q, k)
    U.check_decode_heads(wl, inp, cache, q, k, U.all_heads(wl), out, idx)
    if k >= L:  # keeping every token is dense attention
        dense = F.fasa_dense_decode(cache, L, q, L)
        U.check_gpu_pair(wl, U.stored(out), U.stored(dense))


def test_decode_single_token_cache(path):
    wl = C["c2"].replace(ctx_len=1, batch=2)
    inp, cache, q = U.build(wl)
    out, idx = _decode(wl, cache, q, 256)
    assert idx.cpu().numpy().ravel().tolist() == [0] * (2 * 8)
    U.check_decode_heads(wl, inp, cache, q, 256, U.all_heads(wl), out, idx)


def test_decode_all_fc_full_budget_is_dense(path):
    """With every FC dominant and k = L, FASA is dense attention."""
    wl = C["c2"].replace(ctx_len=3000, n_dom=64, k=3000)
    inp, cache, q = U.build(wl)
    out, idx = _decode(wl, cache, q, wl.k)
    dense = F.fasa_dense_decode(cache, wl.ctx_len, q, wl.q_pos)
    U.check_gpu_pair(wl, U.stored(out), U.stored(dense))


def test_decode_with_tied_tokens(path):
    """Tokens whose dominant dims are zero all score exactly 0; the budget is
    placed inside that tie, so ties must go to the lower index."""
    wl = C["c2"].replace(n_q_heads=4, n_kv_heads=1, ctx_len=4000)
    inp = W.layer_inputs(wl)
    dom = inp.params.dom_idx[0]
    cols = np.concatenate([dom, dom + 64])
    for c in cols:
        inp.k[0, 0, 1000:3000, c] = 0          # +0.0
    _, cache, q = U.build(wl, inp=inp)
    _, s_ref, _ = U.oracle_scores(wl, inp, cache, 0, 0)
    assert np.sum(s_ref == 0) >= 2000
    k = int(np.sum(s_ref > 0)) + 37
    out, idx = _decode(wl, cache, q, k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, k, [(0, 0)], out, idx, scores_gpu=s)
    kept_zero = [t for t in idx.cpu().numpy()[0, 0] if s_ref[t] == 0]
    assert kept_zero == list(range(1000, 1037))


def test_decode_with_small_tie_at_budget_edge(path):
    """Six scattered tokens score exactly 0 and the budget ends inside them:
    the threshold bin holds only the tie (a small union, resolved by
    ranking), and the three lowest indices of it are kept."""
    wl = C["c2"].replace(n_q_heads=4, n_kv_heads=1, ctx_len=4000)
    inp = W.layer_inputs(wl)
    dom = inp.params.dom_idx[0]
    tied = [17, 400, 401, 1999, 2500, 3999]
    for t in tied:
        inp.k[0, 0, t, np.concatenate([dom, dom + 64])] = 0   # +0.0
    _, cache, q = U.build(wl, inp=inp)
    _, s_ref, _ = U.oracle_scores(wl, inp, cache, 0, 0)
    assert np.sum(s_ref == 0) == len(tied)
    k = int(np.sum(s_ref > 0)) + 3
    out, idx = _decode(wl, cache, q, k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, k, [(0, 0)], out, idx, scores_gpu=s)
    kept_zero = [t for t in idx.cpu().numpy()[0, 0] if s_ref[t] == 0]
    assert kept_zero == tied[:3]


@pytest.mark.parametrize("case", ["all_tied", "k_beyond_union"])
def test_decode_exact_fallbacks(case, path):
    """Shapes that take the exact radix selects: every token tied (the
    boundary bin holds the whole row, far beyond the shared-memory tie list)
    and a budget of half a 40000-token row (every CTA publishes all of its
    tokens; the kept list goes to the split-K attention)."""
    if case == "all_tied":
        wl = C["c2"].replace(n_q_heads=4, n_kv_heads=1, ctx_len=8192, k=100)
        inp = W.layer_inputs(wl)
        dom = inp.params.dom_idx[0]
        inp.k[0, 0][:, np.concatenate([dom, dom + 64])] = 0
    else:
        wl = C["c2"].replace(n_q_heads=4, n_kv_heads=1, ctx_len=40000, k=20000)
        inp = W.layer_inputs(wl)
    _, cache, q = U.build(wl, inp=inp)
    out, idx = _decode(wl, cache, q, wl.k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, wl.k, [(0, 0)], out, idx, scores_gpu=s)
    if case == "all_tied":
        assert idx.cpu().numpy()[0, 0].tolist() == list(range(wl.k))


def test_decode_with_clustered_top_scores(path):
    """The highest scores sit in a few hundred consecutive tokens, inside one
    or two of the fused plan's CTA slices: such a CTA holds far more of the
    kept set than it publishes, and the selection must still be exact (the
    fused plan falls back to every key of the row)."""
    wl = C["c2"].replace(ctx_len=8192, k=256)
    inp = W.layer_inputs(wl)
    for g in range(wl.n_kv_heads):
        dom = inp.params.dom_idx[g]
        cols = np.concatenate([dom, dom + 64])
        blk = W.stored_to_f64(inp.k[0, g, 100:700][:, cols]) * 16.0  # exact: a power of two
        inp.k[0, g, 100:700][:, cols] = W.round_to_dtype(blk.astype(np.float32), wl.dtype)
    _, cache, q = U.build(wl, inp=inp)
    out, idx = _decode(wl, cache, q, wl.k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, wl.k, U.all_heads(wl), out, idx, scores_gpu=s)
    kept = idx.cpu().numpy()
    # the cluster holds most of each kept set, so at least one CTA slice
    # (about 480 tokens at this shape) holds far more than it publishes
    assert ((kept >= 100) & (kept < 700)).mean() > 0.5


def test_decode_is_deterministic_and_capturable(path):
    wl = SMALL["c2_ragged"]
    inp, cache, q = U.build(wl)
    ws = F.fasa_decode_workspace(cache, wl.ctx_len, wl.k)
    out1 = torch.empty_like(q)
    F.fasa_decode(cache, wl.ctx_len, q, wl.q_pos, wl.k, out=out1, workspace=ws)
    s = torch.cuda.Stream()
    out2 = torch.empty_like(q)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        F.fasa_decode(cache, wl.ctx_len, q, wl.q_pos, wl.k, out=out2, workspace=ws)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def _both_paths(wl, cache, q, k):
    res = {}
    for name, pth in PATHS.items():
        F.fasa_set_decode_path(pth)
        try:
            res[name] = _decode(wl, cache, q, k)
        finally:
            F.fasa_set_decode_path(F.DECODE_AUTO)
    return res


def _check_paths_agree(wl, res):
    """Every plan scores bit-identically and selects exactly: the same kept
    sets; outputs differ only by float32 summation order."""
    o_s, i_s = res["staged"]
    for name in ("fused",):
        o_x, i_x = res[name]
        assert torch.equal(i_x, i_s), name
        U.check_gpu_pair(wl, U.stored(o_x), U.stored(o_s))


def test_decode_path_setting_and_choice():
    wl = C["c2"].replace(ctx_len=4096)
    _, cache, _ = U.build(wl)
    assert F.fasa_decode_path(cache, wl.ctx_len, wl.k) == F.DECODE_FUSED
    # a budget above 1024 takes the staged plan
    assert F.fasa_decode_path(cache, wl.ctx_len, 1024) == F.DECODE_FUSED
    assert F.fasa_decode_path(cache, wl.ctx_len, 1025) == F.DECODE_STAGED
    assert F.fasa_decode_launches(cache, wl.ctx_len, 1025) in (4, 5)
    F.fasa_set_decode_path(F.DECODE_STAGED)
    try:
        assert F.fasa_decode_path(cache, wl.ctx_len, wl.k) == F.DECODE_STAGED
    finally:
        F.fasa_set_decode_path(F.DECODE_AUTO)
    with pytest.raises(F.FasaError):
        F.fasa_set_decode_path(7)


def test_one_workspace_serves_smaller_lengths_and_budgets():
    """A workspace zeroed once and sized for the largest len and k serves
    decodes at smaller len and k on the same cache, in either plan: the parts
    that must stay zero between calls sit at offsets fixed by the row count.
    Each decode equals the same decode with a fresh workspace."""
    wl = C["c2"].replace(name="wsr", batch=2, ctx_len=3000)
    _, cache, q = U.build(wl)
    ws = F.fasa_decode_workspace(cache, 3000, 700)
    rows = wl.batch * wl.n_kv_heads
    for path in (F.DECODE_STAGED, F.DECODE_FUSED):
        F.fasa_set_decode_path(path)
        try:
            for L, k in [(3000, 700), (1000, 190), (2500, 300), (640, 640), (3000, 257), (3000, 700)]:
                idx = torch.empty((wl.batch, wl.n_kv_heads, k), dtype=torch.int32, device="cuda")
                out = F.fasa_decode(cache, L, q, L, k, idx_out=idx, workspace=ws)
                idx_f = torch.empty_like(idx)
                out_f = F.fasa_decode(cache, L, q, L, k, idx_out=idx_f, workspace=F.fasa_decode_workspace(cache, L, k))
                torch.cuda.synchronize()
                assert F.fasa_device_status(clear=True) == 0, (path, L, k)
                assert torch.equal(idx, idx_f), (path, L, k)
                assert torch.equal(out, out_f), (path, L, k)
                assert idx.reshape(rows, k).max().item() < L
        finally:
            F.fasa_set_decode_path(F.DECODE_AUTO)


def test_fused_decode_rejects_f32_when_forced():
    wl = SMALL["c1"]
    _, cache, q = U.build(wl)
    F.fasa_set_decode_path(F.DECODE_FUSED)
    try:
        with pytest.raises(F.FasaError) as e:
            _decode(wl, cache, q, wl.k)
        assert e.value.status == 2
    finally:
        F.fasa_set_decode_path(F.DECODE_AUTO)


# ------------------------------------------------------------ full sizes

def test_full_c1():
    wl = C["c1"]
    inp, cache, q = U.build(wl)
    U.check_append(wl, inp, cache, U.all_heads(wl))
    out, idx = _decode(wl, cache, q, wl.k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, wl.k, U.all_heads(wl), out, idx, scores_gpu=s)


def test_full_c2():
    wl = C["c2"]
    inp, cache, q = U.build(wl)
    U.check_append(wl, inp, cache, U.sample_heads(wl, 2))
    out, idx = _decode(wl, cache, q, wl.k)
    s = F.fasa_score(cache, wl.ctx_len, q, wl.q_pos).cpu().numpy()
    U.check_decode_heads(wl, inp, cache, q, wl.k, U.all_heads(wl), out, idx, scores_gpu=s)
    assert F.fasa_decode_path(cache, wl.ctx_len, wl.k) == F.DECODE_FUSED
    _check_paths_agree(wl, _both_paths(wl, cache, q, wl.k))
    dense = U.stored(F.fasa_dense_decode(cache, wl.ctx_len, q, wl.q_pos))
    G = wl.group
    for (b, g) in U.sample_heads(wl, 2, seed=1):
        q_rot = O.rotate_queries(inp.q[b, g * G:(g + 1) * G], wl.q_pos, wl.rope_base)
        ref = O.dense_attention(q_rot, U.stored(cache.k[b, g]), U.stored(cache.v[b, g]))
        U.check_out(wl, dense[b, g * G:(g + 1) * G], ref)


def test_full_c3():
    """Every (sequence, KV head) row of c3 against the oracle."""
    wl = C["c3"]
    inp, cache, q = U.build(wl)
    U.check_append(wl, inp, cache, U.sample_heads(wl, 1))
    out, idx = _decode(wl, cache, q, wl.k)
    U.check_decode_heads(wl, inp, cache, q, wl.k, U.all_heads(wl), out, idx)
    _check_paths_agree(wl, _both_paths(wl, cache, q, wl.k))


@pytest.fixture(scope="module")
def c5_state():
    state = U.build(C["c5"])
    yield state
    del state
    torch.cuda.empty_cache()


@pytest.mark.parametrize("k", W.C5_KS)
def test_full_c5(k, c5_state):
    """Every row of c5 at each budget against the oracle."""
    wl = C["c5"]
    inp, cache, q = c5_state
    out, idx = _decode(wl, cache, q, k)
    U.check_decode_heads(wl, inp, cache, q, k, U.all_heads(wl), out, idx)
    if k == W.C5_KS[0]:
        _check_paths_agree(wl, _both_paths(wl, cache, q, k))
    if k == W.C5_KS[-1]:
        dense = U.stored(F.fasa_dense_decode(cache, wl.ctx_len, q, wl.q_pos))
        G = wl.group
        for (b, g) in U.sample_heads(wl, 2, seed=5):
            q_rot = O.rotate_queries(inp.q[b, g * G:(g + 1) * G], wl.q_pos, wl.rope_base)
            ref = O.dense_attention(q_rot, U.stored(cache.k[b, g]), U.stored(cache.v[b, g]))
            U.check_out(wl, dense[b, g * G:(g + 1) * G], ref)


@pytest.mark.parametrize("n_dom", W.C4_NDOMS)
def test_full_c4_sweep(n_dom):
    """Long-CoT sweep: 1K appends up to 32K; decode with k = 18.9% of L at
    several steps, every row against the oracle."""
    wl = C["c4"]
    inp = W.layer_inputs(wl, n_dom=n_dom)
    lp = inp.params
    cache = F.KVCache(wl.batch, wl.n_q_heads, wl.n_kv_heads, n_dom, wl.ctx_len, wl.dtype, wl.rope_base,
                      lp.dom_idx)
    k_all = W.to_torch(inp.k, "cuda")
    v_all = W.to_torch(inp.v, "cuda")
    heads = U.all_heads(wl)
    for step in range(W.C4_STEPS):
        c0 = step * W.C4_APPEND_CHUNK
        c1 = c0 + W.C4_APPEND_CHUNK
        F.fasa_append_kv(cache, k_all[:, :, c0:c1].contiguous(), v_all[:, :, c0:c1].contiguous(), c0)
        L = c1
        if step in (0, 7, W.C4_STEPS - 1):
            k = W.c4_budget(L)
            q_np = np.stack([np.concatenate([W.head_q(wl, lp, 0, b, g, step=step) for g in range(wl.n_kv_heads)])
                             for b in range(wl.batch)])
            q = W.to_torch(q_np, "cuda")
            sub = W.LayerInputs(lp, q_np, inp.k, inp.v)
            out, idx = _decode(wl, cache, q, k, length=L)
            U.check_decode_heads(wl, sub, cache, q, k, heads, out, idx, length=L)
    U.check_append(wl, inp, cache, U.sample_heads(wl, 1, seed=n_dom))
