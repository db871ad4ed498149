"""The C-ABI library: it loads, exports every symbol the header declares, and
rejects bad arguments on the host (no GPU needed: nothing is launched)."""
import ctypes
import os
import re

import pytest

from rope_frequency_chunk_b200 import fasa as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fasa.h")


@pytest.fixture(scope="module")
def L():
    from rope_frequency_chunk_b200 import build
    build.build()
    return F.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fasa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["fasa_append_kv", "fasa_score", "fasa_select_topk", "fasa_sparse_attend", "fasa_decode",
                 "fasa_dense_decode", "fasa_decode_workspace_bytes", "fasa_device_status"]:
        assert want in names


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing


def test_version_and_strings(L):
    assert L.fasa_abi_version() == 1
    assert F.lib().fasa_status_string(0) == b"FASA_OK"
    assert F.lib().fasa_status_string(7) == b"FASA_ERR_BAD_INDEX"
    assert F.lib().fasa_status_string(99) == b"FASA_ERR_UNKNOWN"


def test_sketch_stride(L):
    s = F.fasa_sketch_stride
    assert [s(n, "bf16") for n in (1, 4, 5, 8, 16, 32, 64)] == [8, 8, 16, 16, 32, 64, 128]
    assert [s(n, "f32") for n in (1, 2, 3, 16, 64)] == [4, 4, 8, 32, 128]
    assert s(0, "bf16") == -1 and s(65, "bf16") == -1
    assert L.fasa_sketch_stride(16, 7) == -1
    assert s(16, F.FASA_BF16) == s(16, "bf16") == s(16, __import__("torch").bfloat16) == 32


def test_check_dom_idx(L):
    F.fasa_check_dom_idx([[0, 5, 63], [1, 2, 3]])
    for bad in ([[0, 0, 1]], [[0, 64, 1]], [[-1, 2, 3]]):
        with pytest.raises(F.FasaError):
            F.fasa_check_dom_idx(bad)


def _fake_cache(**kw):
    c = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, n_dom=16, max_len=1024, dtype=1,
             sketch_stride=32, rope_base=1e4, k=0x10000, v=0x20000, sketch=0x30000, dom_idx=0x40000)
    c.update(kw)
    return F.fasa_cache(**c)


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, 2), ("dtype", 3, 2), ("n_q_heads", 3, 1), ("n_q_heads", 64, 2), ("n_dom", 0, 1),
    ("sketch_stride", 16, 1), ("max_len", 0, 1), ("rope_base", 1.0, 1), ("k", 0x10008, 1), ("v", 0, 1),
])
def test_cache_validation(L, field, value, status):
    c = _fake_cache(**{field: value})
    st = L.fasa_score(ctypes.byref(c), 10, 0x50000, 10, 0x60000, None)
    assert st == status


def test_call_validation_without_launch(L):
    c = ctypes.byref(_fake_cache())
    assert L.fasa_append_kv(c, 0x50000, 0x60000, 10, 1020, None) == 3          # beyond max_len
    assert L.fasa_append_kv(c, 0x50000, 0x60000, 0, 5, None) == 0              # no-op
    assert L.fasa_append_kv(c, 0x50008, 0x60000, 4, 0, None) == 1              # misaligned input
    assert L.fasa_score(c, 2000, 0x50000, 0, 0x60000, None) == 3               # len > max_len
    assert L.fasa_score(c, 0, 0x50000, 0, 0x60000, None) == 0                  # empty
    assert L.fasa_select_topk(None, 1, 10, 2, 0x60000, None) == 1
    assert L.fasa_select_topk(0x50000, 1, 10, 0, 0x60000, None) == 1           # k < 1
    assert L.fasa_select_topk(0x50000, 1, (1 << 19) + 1, 5, 0x60000, None) == 2
    assert L.fasa_sparse_attend(c, 10, 0x50000, 10, 0x60000, 0, 0x70000, None) == 1   # n_idx < 1
    assert L.fasa_decode(c, 0, 0x50000, 0, 8, 0x70000, None, 0x80000, 1 << 20, None) == 1
    assert L.fasa_decode(c, 100, 0x50000, 100, 8, 0x70000, None, None, 1 << 20, None) == 4
    need = L.fasa_decode_workspace_bytes(c, 100, 8)
    assert need >= 2 * 100 * 4
    assert L.fasa_decode(c, 100, 0x50000, 100, 8, 0x70000, None, 0x80000, need - 1, None) == 4
    assert L.fasa_dense_decode(c, 0, 0x50000, 0, 0x70000, 0x80000, 1 << 20, None) == 1
    dneed = L.fasa_dense_workspace_bytes(c, 100)
    assert dneed > 0
    assert L.fasa_dense_decode(c, 100, 0x50000, 100, 0x70000, 0x80000, dneed - 1, None) == 4
    assert L.fasa_dense_decode(c, 100, 0x50000, 100, 0x70000, None, dneed, None) == 4


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(F, "_lib", None)
    monkeypatch.setattr(F, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(F.FasaError):
        F.lib()


def test_decode_path_setting_is_validated_on_the_host(L):
    for bad in (3, 4, -1):
        assert L.fasa_set_decode_path(bad) == 1
    for p in (1, 2, 0):
        assert L.fasa_set_decode_path(p) == 0
    assert L.fasa_decode_path(None, 10, 10) < 0
    assert L.fasa_decode_launches(None, 10, 10) < 0


def test_calibration_validation_without_launch(L):
    c = ctypes.byref(_fake_cache())
    ws = L.fasa_calibrate_workspace_bytes
    assert ws(c, 100, 0, 8) == 0 and ws(c, 100, 9, 8) == 0 and ws(c, 0, 2, 8) == 0 and ws(c, 100, 2, 0) == 0
    rows = 2
    need = ws(c, 100, 2, 8)
    assert need >= rows * 2 * 65 * (100 + 8) * 4 and need % 256 == 0
    assert L.fasa_calibrate_scores(c, 100, 0x50000, 0, 0, 0x60000, None) == 1       # n_win 0
    assert L.fasa_calibrate_scores(c, 100, 0x50000, 0, 9, 0x60000, None) == 1       # n_win > 8
    assert L.fasa_calibrate_scores(c, 100, 0x50000, -1, 2, 0x60000, None) == 1      # q_pos0 < 0
    assert L.fasa_calibrate_scores(c, 2000, 0x50000, 0, 2, 0x60000, None) == 3      # len > max_len
    assert L.fasa_calibrate_scores(c, 100, 0x50008, 0, 2, 0x60000, None) == 1       # misaligned q
    cnt = L.fasa_calibrate_counts
    assert cnt(0x50000, 3, 2, 2, 100, 8, 0x60000, 0x70000, 1 << 20, None) == 1      # rows % Hkv
    assert cnt(0x50000, 2, 2, 2, 100, 0, 0x60000, 0x70000, 1 << 20, None) == 1      # budget 0
    assert cnt(0x50000, 2, 2, 2, (1 << 19) + 1, 8, 0x60000, 0x70000, 1 << 30, None) == 2
    assert cnt(0x50000, 2, 2, 2, 100, 8, 0x60000, 0x70000, 2 * 2 * 65 * 8 * 4 - 1, None) == 4
    assert cnt(0x50000, 2, 2, 2, 100, 8, 0x60000, None, 1 << 20, None) == 4
    assert L.fasa_calibrate_dominant(0x60000, 2, 0, 0x70000, None) == 1
    assert L.fasa_calibrate_dominant(0x60000, 2, 65, 0x70000, None) == 1
    assert L.fasa_calibrate_dominant(0x60000, 0, 4, 0x70000, None) == 1
    assert L.fasa_calibrate(c, 100, 0x50000, 0, 2, 8, 4, 0x60000, 0x70000, None, need, None) == 4
    assert L.fasa_calibrate(c, 100, 0x50000, 0, 2, 8, 4, 0x60000, 0x70000, 0x80000, need - 1, None) == 4
    assert L.fasa_calibrate(c, 100, 0x50000, 0, 2, 8, 0, 0x60000, 0x70000, 0x80000, need, None) == 1


def test_varlen_validation_without_launch(L):
    c = ctypes.byref(_fake_cache())

    def vl(**kw):
        d = dict(seq_len=0x90000, budget=None, max_seq_len=100, max_budget=8, q_prerotated=0, reserved=0)
        d.update(kw)
        return ctypes.byref(F.fasa_varlen(**d))

    ws = L.fasa_decode_varlen_workspace_bytes
    need = ws(c, vl())
    assert need > 0 and need % 256 == 0
    # the bounds size the workspace like a uniform call at those bounds
    assert need == L.fasa_decode_workspace_bytes(c, 100, 8)
    assert ws(c, None) == 0 and ws(c, vl(seq_len=None)) == 0 and ws(c, vl(max_seq_len=0)) == 0
    run = L.fasa_decode_varlen
    args = (0x50000, 0x70000, None, 0x80000, need, None)
    assert run(c, None, *args) == 1                                  # no description
    assert run(c, vl(seq_len=None), *args) == 1                      # no lengths
    assert run(c, vl(seq_len=0x90002), *args) == 1                   # misaligned lengths
    assert run(c, vl(budget=0x90001), *args) == 1                    # misaligned budgets
    assert run(c, vl(max_seq_len=0), *args) == 1
    assert run(c, vl(max_budget=0), *args) == 1
    assert run(c, vl(q_prerotated=2), *args) == 1
    assert run(c, vl(max_seq_len=2000), *args) == 3                  # beyond the cache
    assert run(c, vl(max_budget=(1 << 17) + 1), *args) == 2
    assert run(ctypes.byref(_fake_cache(dtype=0)), vl(), *args) == 2  # f32 caches: fused plan only
    assert run(c, vl(), 0x50008, 0x70000, None, 0x80000, need, None) == 1   # misaligned q
    assert run(c, vl(), 0x50000, 0x70000, 0x60002, 0x80000, need, None) == 1
    assert run(c, vl(), 0x50000, 0x70000, None, None, need, None) == 4
    assert run(c, vl(), 0x50000, 0x70000, None, 0x80000, need - 1, None) == 4
    assert run(c, vl(), 0x50000, 0x70000, None, 0x80010, need, None) == 4  # workspace alignment


def test_paged_validation_without_launch(L):
    # a paged cache: max_len = max_blocks * block_size
    c = ctypes.byref(_fake_cache(max_len=64 * 16))

    def pg(**kw):
        d = dict(block_table=0xA0000, block_size=16, max_blocks=64, n_pages=100, reserved=0)
        d.update(kw)
        return ctypes.byref(F.fasa_paged(**d))

    vl = ctypes.byref(F.fasa_varlen(seq_len=0x90000, budget=None, max_seq_len=1000, max_budget=8,
                                    q_prerotated=0, reserved=0))
    ws = L.fasa_decode_paged_workspace_bytes
    need = ws(c, pg(), vl)
    assert need > 0 and need == L.fasa_decode_varlen_workspace_bytes(c, vl)
    for bad in (dict(block_table=None), dict(block_table=0xA0002), dict(block_size=8), dict(block_size=48),
                dict(block_size=1 << 17), dict(max_blocks=0), dict(n_pages=0), dict(max_blocks=63)):
        assert ws(c, pg(**bad), vl) == 0, bad
        assert L.fasa_decode_paged(c, pg(**bad), vl, 0x50000, 0x70000, None, 0x80000, need, None) == 1, bad
    assert ws(c, None, vl) == 0
    big = ctypes.byref(_fake_cache(max_len=64 * 65536))
    assert L.fasa_decode_paged(big, pg(block_size=65536, n_pages=20000), vl, 0x50000, 0x70000, None, 0x80000,
                               1 << 40, None) == 2                      # pool rows beyond 32-bit indices
    run = L.fasa_decode_paged
    assert run(c, pg(), None, 0x50000, 0x70000, None, 0x80000, need, None) == 1
    assert run(c, pg(), vl, 0x50000, 0x70000, None, 0x80000, need - 1, None) == 4
    assert run(ctypes.byref(_fake_cache(max_len=64 * 16, dtype=0)), pg(), vl, 0x50000, 0x70000, None, 0x80000,
               need, None) == 2
    app = L.fasa_append_kv_paged
    assert app(c, pg(), 0x50000, 0x60000, 4, None, None) == 1                  # no positions
    assert app(c, pg(), 0x50000, 0x60000, 4, 0x90002, None) == 1               # misaligned positions
    assert app(c, pg(), 0x50000, 0x60000, -1, 0x90000, None) == 1
    assert app(c, pg(), 0x50000, 0x60000, 2000, 0x90000, None) == 3           # more than a sequence holds
    assert app(c, pg(), 0x50000, 0x60000, 0, 0x90000, None) == 0              # no-op
    assert app(c, pg(), 0x50008, 0x60000, 4, 0x90000, None) == 1              # misaligned input
    assert app(c, pg(block_size=24), 0x50000, 0x60000, 4, 0x90000, None) == 1


def test_multi_validation_without_launch(L):
    c = ctypes.byref(_fake_cache())  # G = 2
    ws = L.fasa_decode_multi_workspace_bytes
    need = ws(c, 100, 4, 8)
    assert need > L.fasa_decode_workspace_bytes(c, 100, 8) and need % 256 == 0
    assert ws(c, 0, 4, 8) == 0 and ws(c, 100, 0, 8) == 0 and ws(c, 100, 4, 0) == 0
    run = L.fasa_decode_multi
    tail = (0x70000, None, 0x80000, need, None)
    assert run(c, 100, 0x50000, 100, 0, 8, *tail) == 1          # n_q < 1
    assert run(c, 100, 0x50000, 100, 17, 8, *tail) == 2         # more than 16 tokens
    assert run(ctypes.byref(_fake_cache(n_q_heads=32, n_kv_heads=2)), 100, 0x50000, 100, 5, 8, *tail) == 2
    assert run(c, 100, 0x50000, -2, 4, 8, *tail) == 1           # bad position
    assert run(c, 100, 0x50000, 2 ** 31 - 2, 4, 8, *tail) == 1  # positions overflow
    assert run(c, 2000, 0x50000, 100, 4, 8, *tail) == 3
    assert run(ctypes.byref(_fake_cache(dtype=0)), 100, 0x50000, 100, 4, 8, *tail) == 2
    assert run(c, 100, 0x50008, 100, 4, 8, *tail) == 1
    assert run(c, 100, 0x50000, 100, 4, 8, 0x70000, None, 0x80000, need - 1, None) == 4
    assert run(c, 100, 0x50000, 100, 4, 8, 0x70000, None, None, need, None) == 4
