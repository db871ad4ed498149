"""GPU parity of the multi-query decode (n_q query tokens per sequence, one
shared critical set per KV head, attention on the tensor cores) against the
CPU oracle, through the C ABI."""
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


def check_multi(wl, inp, cache, qm, q_pos0, k, idx, out, heads, length=None, q_rot_all=None):
    """Every (b, g) in heads against the oracle: the kept set is an exact
    top-k_eff of scores within the TIP error bound of the oracle's, and each
    query row's output equals the oracle's masked attention over the GPU's
    kept set."""
    L = length or wl.ctx_len
    G, n_q = wl.group, qm.shape[1]
    worst = 0.0
    for (b, g) in heads:
        dom = inp.params.dom_idx[g]
        if q_rot_all is None:
            q_rot = np.stack([O.rotate_queries(qm[b, j, g * G:(g + 1) * G], q_pos0 + j, wl.rope_base)
                              for j in range(n_q)])
        else:
            q_rot = q_rot_all[b, :, g * G:(g + 1) * G]
        sk = U.stored(cache.sketch[b, g, :L])[:, :2 * len(dom)]
        rows = q_rot.reshape(-1, 128)
        s_ref = O.tip_scores(rows, sk, dom)
        abs_sum = np.abs(O.sketch_rows(rows, dom)).sum(0) @ np.abs(O.to_f64(sk)).T
        U.check_idx_in_band(idx[b, g], s_ref, k, U.score_err(abs_sum))
        kr, vr = U.stored(cache.k[b, g, :L]), U.stored(cache.v[b, g, :L])
        for j in range(n_q):
            seen = idx[b, g][idx[b, g] <= (q_pos0 + j if q_rot_all is None else 1 << 40)]
            got = out[b, j, g * G:(g + 1) * G]
            if len(seen) == 0:
                assert np.all(W.stored_to_f64(got) == 0.0)
                continue
            ref = O.focused_attention(q_rot[j], kr, vr, seen)
            worst = max(worst, U.check_out(wl, got, ref))
    return worst


def run_multi(wl, cache, qm, q_pos0, k, length=None):
    L = length or wl.ctx_len
    q = W.to_torch(qm, "cuda")
    idx = torch.empty((wl.batch, wl.n_kv_heads, min(k, L)), dtype=torch.int32, device="cuda")
    out = F.fasa_decode_multi(cache, L, q, q_pos0, k, idx_out=idx)
    torch.cuda.synchronize()
    return U.stored(out), idx.cpu().numpy()


# name: (workload, n_q, k)
CASES = {
    "nq4_k300_ragged": (C["c2"].replace(name="mq1", batch=2, ctx_len=5003), 4, 300),
    "nq8_k256": (C["c2"].replace(name="mq2", batch=2, ctx_len=3001), 8, 256),
    "nq16_k1000_splits": (C["c2"].replace(name="mq3", batch=1, ctx_len=9000), 16, 1000),
    "g7_nq9": (C["c4"].replace(name="mq4", batch=2, ctx_len=3001, n_dom=8), 9, 567),
    "nq1_k128": (C["c2"].replace(name="mq5", batch=2, ctx_len=2000), 1, 128),
    "g1_nq2_ndom64": (C["c2"].replace(name="mq6", n_q_heads=3, n_kv_heads=3, batch=1, ctx_len=777, n_dom=64),
                      2, 777),
}


@pytest.mark.parametrize("name", list(CASES))
def test_multi_matches_oracle(name):
    wl, n_q, k = CASES[name]
    inp, cache, _ = U.build(wl)
    qm = W.multi_queries(wl, n_q)
    out, idx = run_multi(wl, cache, qm, wl.q_pos, k)
    check_multi(wl, inp, cache, qm, wl.q_pos, k, idx, out, U.all_heads(wl))


def test_multi_full_c2_layer():
    """The c2 layer (B1, 32/8, L 32768, k 256) with 8 query tokens: all heads."""
    wl = C["c2"]
    inp, cache, _ = U.build(wl)
    qm = W.multi_queries(wl, 8)
    out, idx = run_multi(wl, cache, qm, wl.q_pos, wl.k)
    check_multi(wl, inp, cache, qm, wl.q_pos, wl.k, idx, out, U.all_heads(wl))


@pytest.mark.parametrize("k", [100, 2000])
def test_multi_drafts_in_cache_are_masked(k):
    """Draft tokens already appended at slots 1996 .. 1999: query j at
    position 1996 + j sees only the kept slots up to its own position
    (k = L: masked dense attention)."""
    wl = C["c2"].replace(name="mq7", batch=2, ctx_len=2000)
    inp, cache, _ = U.build(wl)
    qm = W.multi_queries(wl, 4)
    out, idx = run_multi(wl, cache, qm, 1996, k)
    check_multi(wl, inp, cache, qm, 1996, k, idx, out, U.all_heads(wl))


def test_multi_row_without_visible_slot_is_zero():
    """k = 1 with queries placed before most of the cache: rows whose
    position precedes the kept token are zero."""
    wl = C["c2"].replace(name="mq8", batch=1, ctx_len=600)
    inp, cache, _ = U.build(wl)
    qm = W.multi_queries(wl, 4)
    out, idx = run_multi(wl, cache, qm, 10, 1)
    check_multi(wl, inp, cache, qm, 10, 1, idx, out, U.all_heads(wl))
    assert (idx > 13).any(), "expected a kept token after every query's position"


def test_multi_prerotated_queries():
    wl = C["c2"].replace(name="mq9", batch=2, ctx_len=3000)
    inp, cache, _ = U.build(wl)
    qm = W.multi_queries(wl, 4)
    qr = np.stack([np.stack([O.rope_rotate(W.stored_to_f64(qm[b, j]), wl.q_pos + j, wl.rope_base)
                             for j in range(4)]) for b in range(wl.batch)])
    st = W.round_to_dtype(qr.astype(np.float32), wl.dtype)
    out, idx = run_multi(wl, cache, st, -1, 256)
    check_multi(wl, inp, cache, st, -1, 256, idx, out, U.all_heads(wl), q_rot_all=W.stored_to_f64(st))


def test_multi_one_token_agrees_with_decode():
    """n_q = 1: the same kept sets as fasa_decode (up to a rare coefficient
    rounding from the device's angle) and outputs within rounding."""
    wl = C["c2"].replace(name="mq10", batch=2, ctx_len=7000)
    inp, cache, q = U.build(wl)
    idx_d = torch.empty((wl.batch, wl.n_kv_heads, 300), dtype=torch.int32, device="cuda")
    out_d = F.fasa_decode(cache, wl.ctx_len, q, wl.q_pos, 300, idx_out=idx_d)
    torch.cuda.synchronize()
    out, idx = run_multi(wl, cache, inp.q[:, None], wl.q_pos, 300)
    idd = idx_d.cpu().numpy()
    for (b, g) in U.all_heads(wl):
        assert len(set(idd[b, g].tolist()) ^ set(idx[b, g].tolist())) <= 2
    U.check_gpu_pair(wl, out[:, 0], U.stored(out_d))


def test_multi_workspace_reuse_and_determinism():
    wl = C["c2"].replace(name="mq11", batch=2, ctx_len=6000)
    inp, cache, _ = U.build(wl)
    qm = W.to_torch(W.multi_queries(wl, 8), "cuda")
    ws = F.fasa_decode_multi_workspace(cache, wl.ctx_len, 8, 700)
    outs = []
    for k in (700, 300, 700):
        idx = torch.empty((wl.batch, wl.n_kv_heads, k), dtype=torch.int32, device="cuda")
        o = F.fasa_decode_multi(cache, wl.ctx_len, qm, wl.q_pos, k, idx_out=idx, workspace=ws)
        torch.cuda.synchronize()
        outs.append((o.clone(), idx.clone()))
    assert torch.equal(outs[0][0], outs[2][0]) and torch.equal(outs[0][1], outs[2][1])
