"""GPU parity of the offline FC calibration, through the C ABI.

Stage by stage: the score planes against the oracle's (float tolerance), then
the agreement counts and the dominant sets against the oracle fed the GPU's
own planes (integers: exact), then the one-call calibration against the
stages. Small cases span several token tiles with ragged tails; the headline
layer shape is checked on sampled heads.
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


def calib_queries(wl, n_win, seed_step=100):
    """Calibration queries [B, n_win, Hq, 128] (stored dtype): the workload's
    query law, one draw per calibration step."""
    lp = W.layer_params(wl, 0)
    G = wl.group
    sdt = np.float32 if wl.dtype == "f32" else np.uint16
    q = np.empty((wl.batch, n_win, wl.n_q_heads, 128), sdt)
    for b in range(wl.batch):
        for w in range(n_win):
            for g in range(wl.n_kv_heads):
                q[b, w, g * G:(g + 1) * G] = W.head_q(wl, lp, 0, b, g, step=seed_step + w)
    return q


def oracle_planes(wl, inp, cache, q_win, b, g, q_pos0, length=None):
    """The oracle's planes over the GPU's own stored keys (the append stage is
    checked on its own by the decode parity tests)."""
    L = length or wl.ctx_len
    k_rot = U.stored(cache.k[b, g, :L])
    G = wl.group
    pos = q_pos0 + np.arange(q_win.shape[1])
    return O.calibration_scores(q_win[b, :, g * G:(g + 1) * G], pos, k_rot, wl.rope_base)


def check_planes(gpu, ref):
    """Each plane within float32 rounding of the oracle's (both round a float64
    value once; their float64 values differ only by the host's and numpy's
    cos/sin ulps)."""
    scale = np.abs(ref).max(axis=-1, keepdims=True) + 1e-30
    err = np.abs(gpu.astype(np.float64) - ref.astype(np.float64)) / scale
    assert err.max() <= 1e-6, f"plane mismatch {err.max():.3e}"


def counts_from_planes(planes_np, n_kv, budget):
    """Oracle counts summed over sequences, from planes [B, Hkv, W, 65, L]."""
    B = planes_np.shape[0]
    out = np.zeros((n_kv, 64), np.int64)
    for b in range(B):
        for g in range(n_kv):
            out[g] += O.calibration_counts(planes_np[b, g], budget)
    return out


SMALL = {
    "bf16_g4": (C["c2"].replace(name="cal_g4", batch=2, n_q_heads=8, n_kv_heads=2, ctx_len=1000), 3, 37),
    "f32_g1": (C["c1"].replace(name="cal_f32", ctx_len=777), 2, 50),
    "bf16_g7_win8": (C["c4"].replace(name="cal_g7", batch=1, ctx_len=513), 8, 64),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_calibration_stages_match_oracle(name):
    wl, n_win, budget = SMALL[name]
    inp, cache, _ = U.build(wl)
    qw = calib_queries(wl, n_win)
    q_t = W.to_torch(qw, "cuda")
    q_pos0 = wl.ctx_len
    planes = F.fasa_calibrate_scores(cache, wl.ctx_len, q_t, q_pos0)
    pn = planes.cpu().numpy()
    for b in range(wl.batch):
        for g in range(wl.n_kv_heads):
            check_planes(pn[b, g], oracle_planes(wl, inp, cache, qw, b, g, q_pos0))
    counts = F.fasa_calibrate_counts(planes, wl.n_kv_heads, budget)
    want = counts_from_planes(pn, wl.n_kv_heads, budget)
    assert np.array_equal(counts.cpu().numpy().astype(np.int64), want)
    n_dom = 16
    dom = F.fasa_calibrate_dominant(counts, n_dom)
    for g in range(wl.n_kv_heads):
        assert list(dom[g].cpu().numpy()) == list(O.dominant_from_counts(want[g], n_dom))
    # the one-call calibration equals the stages
    c2, d2 = F.fasa_calibrate(cache, wl.ctx_len, q_t, q_pos0, budget, n_dom)
    assert torch.equal(c2, counts) and torch.equal(d2, dom)


def test_calibration_budget_covering_the_cache():
    wl = C["c2"].replace(name="cal_all", batch=2, n_q_heads=4, n_kv_heads=2, ctx_len=300)
    _, cache, _ = U.build(wl)
    q_t = W.to_torch(calib_queries(wl, 3), "cuda")
    counts, dom = F.fasa_calibrate(cache, wl.ctx_len, q_t, wl.ctx_len, 10_000, 5)
    assert (counts.cpu().numpy() == 2 * 3 * 300).all()
    assert (dom.cpu().numpy() == np.arange(5)).all()


def test_calibration_finds_a_single_carrier_fc():
    """Queries with energy in one FC only: that FC's plane is the full head's,
    so it agrees on every token and is ranked first."""
    wl = C["c2"].replace(name="cal_one", batch=1, n_q_heads=8, n_kv_heads=2, ctx_len=2000)
    _, cache, _ = U.build(wl)
    qw = calib_queries(wl, 4)
    carrier = [23, 5]           # per KV head
    G = wl.group
    for g, j in enumerate(carrier):
        keep = np.zeros(128, bool)
        keep[[j, j + 64]] = True
        qw[:, :, g * G:(g + 1) * G, ~keep] = 0
    q_t = W.to_torch(qw, "cuda")
    counts, dom = F.fasa_calibrate(cache, wl.ctx_len, q_t, wl.ctx_len, 128, 4)
    c = counts.cpu().numpy()
    for g, j in enumerate(carrier):
        assert c[g, j] == 4 * 128 and int(dom[g, 0]) == j


def test_calibration_full_layer_sampled():
    """The headline layer shape (B1, 32/8 heads, L 32768), 8 calibration
    queries at the decode budget 256: planes of two heads against the oracle,
    counts of every head against the oracle fed the GPU's planes."""
    wl = C["c2"]
    inp, cache, _ = U.build(wl)
    n_win, budget = 8, 256
    qw = calib_queries(wl, n_win)
    q_t = W.to_torch(qw, "cuda")
    planes = F.fasa_calibrate_scores(cache, wl.ctx_len, q_t, wl.ctx_len)
    counts, dom = F.fasa_calibrate(cache, wl.ctx_len, q_t, wl.ctx_len, budget, wl.n_dom)
    pn = planes.cpu().numpy()
    for g in (0, 5):
        check_planes(pn[0, g, :2], oracle_planes(wl, inp, cache, qw, 0, g, wl.ctx_len)[:2])
    want = counts_from_planes(pn, wl.n_kv_heads, budget)
    assert np.array_equal(counts.cpu().numpy().astype(np.int64), want)
    for g in range(wl.n_kv_heads):
        assert list(dom[g].cpu().numpy()) == list(O.dominant_from_counts(want[g], wl.n_dom))
