"""GPU parity of FASA-M, the memory-optimised variant: K and V in pinned
host memory read across the host link, only the dominant-FC sketch on the
device. The kept sets must be identical to the device-resident cache's, and
so must the outputs wherever both caches run the same attention kernel; the
fused plan attends a host-resident cache's kept rows with the split-K
launch even where a device-resident cache is attended inside the fused
kernel, and those outputs agree within the two kernels' rounding. Every
result is also checked against the CPU oracle."""
import ctypes

import numpy as np
import pytest
import torch

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


def pair(wl, chunks=None):
    """The same layer in a device-resident and a host-resident cache."""
    inp = W.layer_inputs(wl)
    _, dev, q = U.build(wl, inp=inp)
    _, host, _ = U.build(wl, inp=inp, chunks=chunks, kv_on_host=True)
    return inp, dev, host, q


def test_host_resident_cache_layout_and_append():
    wl = C["c2"].replace(name="m1", batch=2, ctx_len=3001)
    inp, dev, host, q = pair(wl, chunks=[1, 1000, 7, 1993])
    assert not host.k.is_cuda and host.k.is_pinned() and host.sketch.is_cuda
    L = wl.ctx_len
    assert torch.equal(dev.k[:, :, :L].cpu(), host.k[:, :, :L])
    assert torch.equal(dev.v[:, :, :L].cpu(), host.v[:, :, :L])
    assert torch.equal(dev.sketch[:, :, :L], host.sketch[:, :, :L])
    # the device holds the sketch alone: 2 * 128 / 32 + 1 = 9x less than FASA-C at n_dom 16
    assert dev.device_bytes() / host.device_bytes() > 8.9


@pytest.mark.parametrize("path", [F.DECODE_FUSED, F.DECODE_STAGED])
@pytest.mark.parametrize("k", [256, 700])
def test_decode_on_host_resident_cache(path, k):
    wl = C["c2"].replace(name="m2", batch=2, ctx_len=9000, k=k)
    inp, dev, host, q = pair(wl)
    res = []
    F.fasa_set_decode_path(path)
    try:
        for cache in (dev, host):
            idx = torch.empty((wl.batch, wl.n_kv_heads, k), dtype=torch.int32, device="cuda")
            out = F.fasa_decode(cache, wl.ctx_len, q, wl.q_pos, k, idx_out=idx)
            torch.cuda.synchronize()
            res.append((idx, out))
    finally:
        F.fasa_set_decode_path(F.DECODE_AUTO)
    assert torch.equal(res[0][0], res[1][0])
    if path == F.DECODE_FUSED and k <= 256:  # in-CTA attention on the device cache, split-K on the host one
        assert F.fasa_decode_launches(dev, wl.ctx_len, k) == 1 and F.fasa_decode_launches(host, wl.ctx_len, k) > 1
        U.check_gpu_pair(wl, U.stored(res[0][1]), U.stored(res[1][1]))
    else:
        assert torch.equal(res[0][1], res[1][1])
    U.check_decode_heads(wl, inp, host, q, k, U.all_heads(wl), res[1][1], res[1][0])


def test_varlen_on_host_resident_cache():
    wl = C["c2"].replace(name="m3", batch=3, ctx_len=5000)
    inp, dev, host, q = pair(wl)
    sl = torch.tensor([5000, 31, 2222], dtype=torch.int32, device="cuda")
    bd = torch.tensor([256, 1, 64, 300, 300, 17, 128, 5], dtype=torch.int32, device="cuda")
    res = []
    for cache in (dev, host):
        idx = torch.empty((wl.batch, wl.n_kv_heads, 300), dtype=torch.int32, device="cuda")
        out = F.fasa_decode_varlen(cache, sl, q, wl.ctx_len, 300, budget=bd, idx_out=idx)
        torch.cuda.synchronize()
        res.append((idx, out))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


def test_sparse_attend_f32_on_host_resident_cache():
    wl = C["c1"].replace(name="m4", ctx_len=2500)
    inp, dev, host, q = pair(wl)
    r = np.random.default_rng(5)
    idx = torch.tensor(np.sort(r.choice(wl.ctx_len, (1, 1, 300), replace=False), axis=-1), dtype=torch.int32,
                       device="cuda")
    a = F.fasa_sparse_attend(dev, wl.ctx_len, q, wl.q_pos, idx)
    b = F.fasa_sparse_attend(host, wl.ctx_len, q, wl.q_pos, idx)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # and the fused decode of the f32 cache (staged plan)
    oa = F.fasa_decode(dev, wl.ctx_len, q, wl.q_pos, wl.k)
    ob = F.fasa_decode(host, wl.ctx_len, q, wl.q_pos, wl.k)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob)


def test_dense_on_host_resident_cache():
    wl = C["c2"].replace(name="m5", batch=1, ctx_len=4000)
    inp, dev, host, q = pair(wl)
    a = F.fasa_dense_decode(dev, wl.ctx_len, q, wl.q_pos)
    b = F.fasa_dense_decode(host, wl.ctx_len, q, wl.q_pos)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # the f32 dense kernel stages rows with bulk copies: refused on host memory
    wl1 = C["c1"].replace(name="m6", ctx_len=1000)
    _, host1, q1 = U.build(wl1, kv_on_host=True)
    with pytest.raises(F.FasaError) as e:
        F.fasa_dense_decode(host1, wl1.ctx_len, q1, wl1.q_pos)
    assert e.value.status == 2


def test_host_pointer_rejects_unpinned_memory():
    t = torch.empty(1024, dtype=torch.uint8)
    out = ctypes.c_void_p()
    assert F.lib().fasa_host_kv_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(out)) == 1
    assert F.lib().fasa_host_kv_pointer(None, ctypes.byref(out)) == 1
    with pytest.raises(TypeError):
        F.fasa_host_kv_pointer(t)
