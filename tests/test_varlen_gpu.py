"""GPU parity of the varlen decode (per-sequence lengths, per-head budgets)
and of pre-rotated queries, against the CPU oracle run on each sequence
alone at its own length and budget, through the C ABI."""
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


def check_row(wl, inp, cache, b, g, L, k, idx_row, out_rows, q_rot=None):
    """(b, g) of a varlen call against the oracle at length L and budget k:
    the kept set (then -1 padding) and the group's output."""
    q_rot, s_ref, abs_sum = U.oracle_scores(wl, inp, cache, b, g, L, q_rot=q_rot)
    ke = min(k, L)
    assert np.all(idx_row[ke:] == -1), "rows shorter than the bound are padded with -1"
    U.check_idx_in_band(idx_row[:ke], s_ref, k, U.score_err(abs_sum))
    ref = O.focused_attention(q_rot, U.stored(cache.k[b, g, :L]), U.stored(cache.v[b, g, :L]), idx_row[:ke])
    return U.check_out(wl, out_rows, ref)


def run_varlen(wl, cache, q, seq_len, budget, max_budget, q_prerotated=False, max_seq_len=None):
    B, H = wl.batch, wl.n_kv_heads
    sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
    bd = None if budget is None else torch.tensor(budget, dtype=torch.int32, device="cuda")
    idx = torch.full((B, H, max_budget), -7, dtype=torch.int32, device="cuda")
    out = F.fasa_decode_varlen(cache, sl, q, max_seq_len or wl.ctx_len, max_budget, budget=bd,
                               q_prerotated=q_prerotated, idx_out=idx)
    torch.cuda.synchronize()
    return U.stored(out), idx.cpu().numpy()


# name: (workload, seq_len per sequence, budget per KV head or None, max_budget)
CASES = {
    # mixed lengths (a single token, ragged tails) and budgets; the kept sets
    # exceed 256, so the split-K attention launch follows the fused kernel
    "mixed_split": (C["c2"].replace(name="vl1", batch=6, ctx_len=5003),
                    [5003, 1, 257, 4096, 3000, 17], [256, 1, 100, 512, 256, 64, 7, 300], 512),
    # every kept set within 256: the attention runs inside the fused kernel
    "mixed_direct": (C["c2"].replace(name="vl2", batch=3, ctx_len=3001),
                     [2049, 150, 3001], None, 200),
    # group 7, eight dominant FCs, a budget above some lengths
    "g7": (C["c4"].replace(name="vl3", batch=2, ctx_len=3001, k=567, n_dom=8),
           [3001, 1234], [567, 1, 100, 2000], 2000),
    # group 1, every FC dominant
    "g1_ndom64": (C["c2"].replace(name="vl4", n_q_heads=3, n_kv_heads=3, batch=2, ctx_len=777, n_dom=64, k=64),
                  [777, 300], [64, 300, 5], 300),
}


@pytest.mark.parametrize("name", list(CASES))
def test_varlen_matches_oracle_per_sequence(name):
    wl, seq_len, budget, mb = CASES[name]
    inp, cache, q = U.build(wl)
    out, idx = run_varlen(wl, cache, q, seq_len, budget, mb)
    G = wl.group
    for (b, g) in U.all_heads(wl):
        k = mb if budget is None else budget[g]
        check_row(wl, inp, cache, b, g, seq_len[b], k, idx[b, g], out[b, g * G:(g + 1) * G])


def test_varlen_serving_batch_full_size():
    """64 sequences of lengths spread over 1 .. 16384 and budgets of 128 ..
    1024 per head, at the serving batch's full cache size; sampled rows."""
    wl = C["c5"]
    r = np.random.default_rng(11)
    seq_len = r.integers(1, wl.ctx_len + 1, wl.batch).tolist()
    seq_len[0], seq_len[1] = wl.ctx_len, 1
    budget = [int(x) for x in r.choice(W.C5_KS, wl.n_kv_heads)]
    inp, cache, q = U.build(wl)
    out, idx = run_varlen(wl, cache, q, seq_len, budget, max(W.C5_KS))
    G = wl.group
    heads = sorted(set(U.sample_heads(wl, 20, seed=3)) | {(0, 0), (1, 3)})
    for (b, g) in heads:
        check_row(wl, inp, cache, b, g, seq_len[b], budget[g], idx[b, g], out[b, g * G:(g + 1) * G])
    # every row's list: ascending kept tokens, then -1
    for b in range(wl.batch):
        for g in range(wl.n_kv_heads):
            ke = min(budget[g], seq_len[b])
            row = idx[b, g]
            assert np.all(np.diff(row[:ke]) > 0) and row[0] >= 0 and row[ke - 1] < seq_len[b]
            assert np.all(row[ke:] == -1)


def test_varlen_uniform_equals_decode():
    """Equal lengths and no budgets: the same kept sets and outputs as
    fasa_decode at that length (the fused plan on both sides)."""
    wl = C["c2"].replace(name="vl5", batch=2, ctx_len=9000, k=300)
    inp, cache, q = U.build(wl)
    F.fasa_set_decode_path(F.DECODE_FUSED)
    try:
        idx_u = torch.empty((wl.batch, wl.n_kv_heads, wl.k), dtype=torch.int32, device="cuda")
        out_u = F.fasa_decode(cache, wl.ctx_len, q, wl.q_pos, wl.k, idx_out=idx_u)
        torch.cuda.synchronize()
    finally:
        F.fasa_set_decode_path(F.DECODE_AUTO)
    out, idx = run_varlen(wl, cache, q, [wl.ctx_len] * wl.batch, None, wl.k)
    iu = idx_u.cpu().numpy()
    # the angle comes from the device's float64 sincos instead of the host's:
    # a coefficient may round differently once in many millions, so allow a
    # single swapped token per row
    for (b, g) in U.all_heads(wl):
        assert len(set(iu[b, g].tolist()) ^ set(idx[b, g].tolist())) <= 2
    U.check_gpu_pair(wl, out, U.stored(out_u))


def test_varlen_out_of_range_lengths_are_clamped_and_flagged():
    wl = C["c2"].replace(name="vl6", batch=3, ctx_len=2000)
    inp, cache, q = U.build(wl)
    out, idx = run_varlen(wl, cache, q, [0, 2000, 5000], [0, 64, 64, 64, 64, 64, 64, 99999], 128)
    assert F.fasa_device_status(clear=True) == 7
    G = wl.group
    # clamped: length 0 -> 1, 5000 -> 2000; budget 0 -> 1, 99999 -> 128
    for (b, g) in [(0, 0), (0, 7), (1, 0), (1, 7), (2, 3), (2, 7)]:
        L = [1, 2000, 2000][b]
        k = [1, 64, 64, 64, 64, 64, 64, 128][g]
        check_row(wl, inp, cache, b, g, L, k, idx[b, g], out[b, g * G:(g + 1) * G])


def _prerotated(wl, inp, pos_of_b):
    """The workload's queries rotated by the oracle at each sequence's
    position and stored in the cache dtype; returns (stored, float64)."""
    q = W.stored_to_f64(inp.q)
    qr = np.stack([O.rope_rotate(q[b], pos_of_b[b], wl.rope_base) for b in range(wl.batch)])
    st = W.round_to_dtype(qr.astype(np.float32), wl.dtype)
    return st, W.stored_to_f64(st)


@pytest.mark.parametrize("path", [F.DECODE_FUSED, F.DECODE_STAGED])
def test_decode_with_prerotated_queries(path):
    """q_pos = FASA_Q_PREROTATED: the queries are used as given (the oracle
    takes the stored rotated queries as q' directly)."""
    wl = C["c2"].replace(name="pr1", batch=2, ctx_len=4001, k=300)
    inp, cache, _ = U.build(wl)
    st, qr = _prerotated(wl, inp, [wl.q_pos] * wl.batch)
    q = W.to_torch(st, "cuda")
    idx = torch.empty((wl.batch, wl.n_kv_heads, wl.k), dtype=torch.int32, device="cuda")
    F.fasa_set_decode_path(path)
    try:
        out = F.fasa_decode(cache, wl.ctx_len, q, -1, wl.k, idx_out=idx)
        torch.cuda.synchronize()
    finally:
        F.fasa_set_decode_path(F.DECODE_AUTO)
    out, idx = U.stored(out), idx.cpu().numpy()
    G = wl.group
    for (b, g) in U.all_heads(wl):
        check_row(wl, inp, cache, b, g, wl.ctx_len, wl.k, idx[b, g], out[b, g * G:(g + 1) * G],
                  q_rot=qr[b, g * G:(g + 1) * G])


def test_varlen_with_prerotated_queries():
    wl = C["c2"].replace(name="pr2", batch=3, ctx_len=3000)
    seq_len = [3000, 999, 40]
    inp, cache, _ = U.build(wl)
    st, qr = _prerotated(wl, inp, seq_len)
    q = W.to_torch(st, "cuda")
    out, idx = run_varlen(wl, cache, q, seq_len, None, 256, q_prerotated=True)
    G = wl.group
    for (b, g) in U.all_heads(wl):
        check_row(wl, inp, cache, b, g, seq_len[b], 256, idx[b, g], out[b, g * G:(g + 1) * G],
                  q_rot=qr[b, g * G:(g + 1) * G])


def test_varlen_workspace_reuse_without_zeroing():
    """One workspace, zeroed once, across calls of different lengths and
    budgets: every call leaves its semaphores and counters zero again."""
    wl = C["c2"].replace(name="vl7", batch=4, ctx_len=6000)
    inp, cache, q = U.build(wl)
    ws = F.fasa_decode_varlen_workspace(cache, wl.ctx_len, 600)
    G = wl.group
    for seq_len, budget in [([6000, 5, 3000, 4500], [600] * 8), ([1, 6000, 6000, 77], [3, 300, 600, 1, 9, 256, 257, 500]),
                            ([2500] * 4, None)]:
        sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
        bd = None if budget is None else torch.tensor(budget, dtype=torch.int32, device="cuda")
        idx = torch.empty((wl.batch, wl.n_kv_heads, 600), dtype=torch.int32, device="cuda")
        out = F.fasa_decode_varlen(cache, sl, q, wl.ctx_len, 600, budget=bd, idx_out=idx, workspace=ws)
        torch.cuda.synchronize()
        out, idx = U.stored(out), idx.cpu().numpy()
        for (b, g) in U.sample_heads(wl, 8, seed=len(seq_len) + seq_len[0]):
            k = 600 if budget is None else budget[g]
            check_row(wl, inp, cache, b, g, seq_len[b], k, idx[b, g], out[b, g * G:(g + 1) * G])
