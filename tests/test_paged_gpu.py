"""GPU parity of paged caches (a block table maps each sequence's logical
blocks to pages of shared pools): appends land in the right page rows, and a
paged decode gives the same kept sets and outputs as the varlen decode of a
contiguous cache holding the same slots, and matches the CPU oracle."""
import numpy as np
import pytest
import torch

from rope_frequency_chunk_b200 import fasa as F
from rope_frequency_chunk_b200 import workloads as W
from tests import gpu_util as U
from tests.test_varlen_gpu import check_row, run_varlen

pytestmark = pytest.mark.gpu

C = W.CONFIGS


@pytest.fixture(autouse=True)
def _clean_status():
    F.fasa_device_status(clear=True)
    yield
    assert F.fasa_device_status(clear=True) == 0


def paged_cache(wl, inp, bs, seq_len, spare=7, seed=0, chunks=None):
    """A paged cache holding the first seq_len[b] slots of each sequence of
    inp, pages drawn at random from a shared pool (spare pages unused); the
    appends go in chunks (uniform n_new per call, each sequence at its own
    position)."""
    B, H = wl.batch, wl.n_kv_heads
    max_blocks = -(-wl.ctx_len // bs)
    need = [-(-L // bs) for L in seq_len]
    n_pages = sum(need) + spare
    r = np.random.default_rng(seed)
    perm = r.permutation(n_pages)
    table = np.full((B, max_blocks), n_pages + 5, np.int32)  # entries beyond a sequence stay out of range
    o = 0
    for b in range(B):
        table[b, :need[b]] = perm[o:o + need[b]]
        o += need[b]
    cache = F.PagedKVCache(B, wl.n_q_heads, H, inp.params.dom_idx.shape[1], n_pages, bs, max_blocks, wl.dtype,
                           wl.rope_base, inp.params.dom_idx)
    cache.block_table.copy_(torch.from_numpy(table))
    k = W.to_torch(inp.k, "cuda")
    v = W.to_torch(inp.v, "cuda")
    # every sequence receives chunks of the same size at its own position,
    # until its length is reached (sequences that are full take a position
    # whose range leaves the cache: the kernel skips them and flags it)
    if chunks is None:  # the gaps between the distinct lengths: every sequence ends exactly full
        ends = sorted(set(seq_len))
        chunks = [e - s for s, e in zip([0] + ends[:-1], ends)]
    pos = np.zeros(B, np.int64)
    for n in chunks:
        p0 = torch.tensor([int(x) if x + n <= seq_len[b] else -1 for b, x in enumerate(pos)], dtype=torch.int32,
                          device="cuda")
        kk = torch.stack([k[b, :, int(pos[b]):int(pos[b]) + n] if pos[b] + n <= seq_len[b]
                          else torch.zeros_like(k[b, :, :n]) for b in range(B)]).contiguous()
        vv = torch.stack([v[b, :, int(pos[b]):int(pos[b]) + n] if pos[b] + n <= seq_len[b]
                          else torch.zeros_like(v[b, :, :n]) for b in range(B)]).contiguous()
        F.fasa_append_kv_paged(cache, kk, vv, p0)
        skipped = any(int(x) < 0 for x in p0.tolist())
        torch.cuda.synchronize()
        st = F.fasa_device_status(clear=True)
        assert st == (7 if skipped else 0)
        pos = np.array([x + n if x + n <= seq_len[b] else x for b, x in enumerate(pos)])
    assert list(pos) == list(seq_len)
    torch.cuda.synchronize()
    return cache


def test_paged_append_matches_contiguous():
    wl = C["c2"].replace(name="pg1", batch=3, ctx_len=3001)
    seq_len = [3001, 1000, 1000]
    inp = W.layer_inputs(wl)
    _, ref, _ = U.build(wl, inp=inp)
    cache = paged_cache(wl, inp, 16, seq_len, chunks=[1000, 1000, 1000, 1])
    for b in range(wl.batch):
        L = seq_len[b]
        for g in range(wl.n_kv_heads):
            assert torch.equal(cache.logical(cache.k, b, g, L), ref.k[b, g, :L])
            assert torch.equal(cache.logical(cache.v, b, g, L), ref.v[b, g, :L])
            assert torch.equal(cache.logical(cache.sketch, b, g, L), ref.sketch[b, g, :L])


def test_decode_style_appends_one_token_per_sequence():
    """A serving step appends one token per sequence at its own position."""
    wl = C["c2"].replace(name="pg2", batch=4, ctx_len=300)
    seq_len = [300, 257, 16, 1]
    inp = W.layer_inputs(wl)
    cache = paged_cache(wl, inp, 16, seq_len, chunks=[1] * 300)
    _, ref, _ = U.build(wl, inp=inp)
    for b in range(wl.batch):
        for g in range(wl.n_kv_heads):
            L = seq_len[b]
            assert torch.equal(cache.logical(cache.k, b, g, L), ref.k[b, g, :L])
            assert torch.equal(cache.logical(cache.sketch, b, g, L), ref.sketch[b, g, :L])


CASES = {
    # block size 16, kept sets beyond 256 (split-K attention launch)
    "bs16_split": (C["c2"].replace(name="pg3", batch=4, ctx_len=5003), 16, [5003, 1, 4000, 777],
                   [256, 1, 100, 512, 256, 64, 7, 300], 512),
    # block size 64, attention inside the fused kernel
    "bs64_direct": (C["c2"].replace(name="pg4", batch=3, ctx_len=4096), 64, [4096, 65, 2500], None, 200),
    # group 7, eight dominant FCs, large pages
    "bs1024_g7": (C["c4"].replace(name="pg5", batch=2, ctx_len=3001, k=567, n_dom=8), 1024, [3001, 1500],
                  [567, 1, 100, 2000], 2000),
}


@pytest.mark.parametrize("name", list(CASES))
def test_paged_decode_equals_contiguous_and_oracle(name):
    wl, bs, seq_len, budget, mb = CASES[name]
    inp = W.layer_inputs(wl)
    _, ref, q = U.build(wl, inp=inp)
    cache = paged_cache(wl, inp, bs, seq_len, seed=len(name))
    out_c, idx_c = run_varlen(wl, ref, q, seq_len, budget, mb)
    sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
    bd = None if budget is None else torch.tensor(budget, dtype=torch.int32, device="cuda")
    idx = torch.full((wl.batch, wl.n_kv_heads, mb), -7, dtype=torch.int32, device="cuda")
    out = F.fasa_decode_paged(cache, sl, q, wl.ctx_len, mb, budget=bd, idx_out=idx)
    torch.cuda.synchronize()
    out, idx = U.stored(out), idx.cpu().numpy()
    assert np.array_equal(idx, idx_c) and np.array_equal(out, out_c)
    G = wl.group
    for (b, g) in U.all_heads(wl):
        k = mb if budget is None else budget[g]
        check_row(wl, inp, ref, b, g, seq_len[b], k, idx[b, g], out[b, g * G:(g + 1) * G])


def test_paged_decode_serving_batch_full_size():
    """64 sequences of mixed lengths up to 16384 in 16-token pages, budgets
    128 .. 1024 per head; every row against the contiguous varlen decode,
    sampled rows against the oracle."""
    wl = C["c5"]
    r = np.random.default_rng(21)
    seq_len = r.integers(1, wl.ctx_len + 1, wl.batch).tolist()
    seq_len[0], seq_len[1] = wl.ctx_len, 1
    budget = [int(x) for x in r.choice(W.C5_KS, wl.n_kv_heads)]
    inp = W.layer_inputs(wl)
    _, ref, q = U.build(wl, inp=inp)
    cache = paged_cache(wl, inp, 16, seq_len, seed=4)
    out_c, idx_c = run_varlen(wl, ref, q, seq_len, budget, max(W.C5_KS))
    sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
    bd = torch.tensor(budget, dtype=torch.int32, device="cuda")
    idx = torch.empty((wl.batch, wl.n_kv_heads, max(W.C5_KS)), dtype=torch.int32, device="cuda")
    out = F.fasa_decode_paged(cache, sl, q, wl.ctx_len, max(W.C5_KS), budget=bd, idx_out=idx)
    torch.cuda.synchronize()
    out, idx = U.stored(out), idx.cpu().numpy()
    assert np.array_equal(idx, idx_c) and np.array_equal(out, out_c)
    G = wl.group
    for (b, g) in sorted(set(U.sample_heads(wl, 12, seed=9)) | {(0, 1), (1, 2)}):
        check_row(wl, inp, ref, b, g, seq_len[b], budget[g], idx[b, g], out[b, g * G:(g + 1) * G])


def test_out_of_pool_page_is_skipped_and_flagged():
    """A table entry outside the pool inside a sequence's length: its rows
    are neither read nor written, and the status word says so."""
    wl = C["c2"].replace(name="pg6", batch=2, ctx_len=512)
    seq_len = [512, 512]
    inp = W.layer_inputs(wl)
    cache = paged_cache(wl, inp, 16, seq_len, seed=2)
    cache.block_table[1, 5] = cache.n_pages + 100
    cache.block_table[1, 9] = -3
    sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
    idx = torch.empty((2, wl.n_kv_heads, 256), dtype=torch.int32, device="cuda")
    out = F.fasa_decode_paged(cache, sl, W.to_torch(inp.q, "cuda"), wl.ctx_len, 256, idx_out=idx)
    torch.cuda.synchronize()
    assert F.fasa_device_status(clear=True) == 7
    assert torch.isfinite(out.float()).all()
    # sequence 0 does not reach the bad entries: its results are exact
    _, ref, q = U.build(wl, inp=inp)
    out_c, idx_c = run_varlen(wl, ref, q, seq_len, None, 256)
    assert np.array_equal(idx.cpu().numpy()[0], idx_c[0])
    assert np.array_equal(U.stored(out)[0], out_c[0])
