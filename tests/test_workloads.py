"""The seeded input generator: shapes, determinism, per-head independence."""
import numpy as np

from rope_frequency_chunk_b200 import workloads as W


def test_configs_match_the_stated_shapes():
    c = W.CONFIGS
    assert (c["c1"].n_q_heads, c["c1"].dtype, c["c1"].ctx_len, c["c1"].k, c["c1"].rope_base) == (1, "f32", 4096, 256, 1e4)
    assert (c["c2"].batch, c["c2"].n_q_heads, c["c2"].n_kv_heads, c["c2"].ctx_len, c["c2"].k) == (1, 32, 8, 32768, 256)
    assert c["c2"].rope_base == 5e5 and c["c2"].n_outlier == 2 and c["c2"].group == 4
    assert (c["c3"].batch, c["c3"].ctx_len, c["c3"].k) == (8, 131072, 2048)
    assert (c["c4"].batch, c["c4"].n_q_heads, c["c4"].n_kv_heads) == (4, 28, 4)
    assert (c["c5"].batch, c["c5"].ctx_len) == (64, 16384)
    assert all(w.q_pos == w.ctx_len for w in c.values())


def test_c4_budget_is_18_9_percent():
    assert W.c4_budget(1000) == 189
    assert W.c4_budget(32768) == 6193       # 6193.152
    assert W.c4_budget(1024) == 194         # 193.536


def test_layer_generation_is_deterministic_and_per_head():
    wl = W.CONFIGS["c2"].replace(ctx_len=300)
    a = W.layer_inputs(wl, layer=1)
    b = W.layer_inputs(wl, layer=1)
    assert np.array_equal(a.k, b.k) and np.array_equal(a.q, b.q) and np.array_equal(a.v, b.v)
    assert a.k.shape == (1, 8, 300, 128) and a.k.dtype == np.uint16
    assert a.q.shape == (1, 32, 128)
    # a single head regenerates alone, identically
    lp = W.layer_params(wl, 1)
    k5, v5 = W.head_kv(wl, lp, 1, 0, 5)
    assert np.array_equal(k5, a.k[0, 5]) and np.array_equal(v5, a.v[0, 5])
    assert np.array_equal(W.head_q(wl, lp, 1, 0, 5), a.q[0, 20:24])
    c = W.layer_inputs(wl, layer=2)
    assert not np.array_equal(a.k, c.k)


def test_sequences_are_independent():
    wl = W.CONFIGS["c3"].replace(ctx_len=64, batch=2)
    x = W.layer_inputs(wl)
    assert not np.array_equal(x.k[0], x.k[1])


def test_dominant_set_is_top_energy_and_distinct():
    wl = W.CONFIGS["c2"]
    lp = W.layer_params(wl, 0)
    for g in range(wl.n_kv_heads):
        d = lp.dom_idx[g]
        assert len(set(d.tolist())) == wl.n_dom and d.min() >= 0 and d.max() < 64
        s2 = lp.scales[g].astype(np.float64) ** 2
        e = s2[:64] + s2[64:]
        e[lp.outliers[g]] *= 48
        assert e[d].min() >= np.delete(e, d).max()
        assert list(e[d]) == sorted(e[d], reverse=True)


def test_bf16_inputs_are_exact_round_to_nearest_even():
    x = np.array([1.0, 1.00390625, 1.005859375, -2.0e-3], np.float32)
    bits = W.round_to_dtype(x, "bf16")
    back = W.stored_to_f64(bits)
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0078125


def test_outlier_fcs_are_heavy_tailed():
    wl = W.CONFIGS["c2"].replace(ctx_len=4000)
    lp = W.layer_params(wl)
    k, _ = W.head_kv(wl, lp, 0, 0, 0)
    kf = W.stored_to_f64(k) / lp.scales[0]
    i = lp.outliers[0][0]
    normal_cols = [j for j in range(64) if j not in lp.outliers[0]]
    kurt = lambda a: np.mean(a ** 4) / np.mean(a ** 2) ** 2
    assert kurt(kf[:, i]) > 6 > kurt(kf[:, normal_cols[0]])
