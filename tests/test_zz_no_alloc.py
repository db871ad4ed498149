"""fasa_decode_static_scratch: the decode for callers that cannot allocate.

Some callers have no device allocator to hand the library a workspace (a
plugin inside a framework that owns the device memory pool, or a path that
must not call cudaMalloc). This entry point uses a fixed scratch array inside
the library instead. It must give the same kept indices and outputs as
fasa_decode with a caller workspace, on consecutive calls that reuse the same
shared scratch. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from rope_frequency_chunk_b200 import fasa as F
from rope_frequency_chunk_b200 import workloads as W

pytestmark = pytest.mark.gpu


PLANS = {"fused": F.DECODE_FUSED, "staged": F.DECODE_STAGED}


@pytest.mark.parametrize("plan", list(PLANS))
def test_static_scratch_decode_matches_workspace_decode(plan):
    """Two calls in a row with different lengths and budgets, under each
    launch plan: the plans keep histograms, counters, semaphores and
    candidate lists in the scratch, so anything the first call left behind
    and the second call read would change its kept set or output."""
    wl = W.CONFIGS["c2"].replace(ctx_len=6007, batch=2, k=300)
    inp = W.layer_inputs(wl)
    cache = F.KVCache(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.n_dom, wl.ctx_len, wl.dtype, wl.rope_base,
                      inp.params.dom_idx)
    F.fasa_append_kv(cache, W.to_torch(inp.k, "cuda"), W.to_torch(inp.v, "cuda"), 0)
    lib = F.lib()
    F.fasa_set_decode_path(PLANS[plan])
    try:
        for step, (L, k) in enumerate([(6007, 300), (4099, 77)]):
            assert lib.fasa_decode_workspace_bytes(cache.ref(), L, k) <= (64 << 20)
            q = W.to_torch(np.stack([np.concatenate([W.head_q(wl, inp.params, 0, b, g, step=step)
                                                     for g in range(wl.n_kv_heads)]) for b in range(wl.batch)]),
                           "cuda")
            idx_ref = torch.empty(wl.batch, wl.n_kv_heads, k, dtype=torch.int32, device="cuda")
            out_ref = F.fasa_decode(cache, L, q, L, k, idx_out=idx_ref)
            idx = torch.full_like(idx_ref, -1)
            out = torch.zeros_like(out_ref)
            st = lib.fasa_decode_static_scratch(cache.ref(), L, q.data_ptr(), L, k, out.data_ptr(),
                                                idx.data_ptr(), torch.cuda.current_stream().cuda_stream)
            assert st == 0, F.STATUS.get(st, st)
            torch.cuda.synchronize()
            assert F.fasa_device_status(clear=True) == 0
            # the same kernels on the same inputs: bit-identical results
            assert torch.equal(idx, idx_ref)
            assert torch.equal(out, out_ref)
    finally:
        F.fasa_set_decode_path(F.DECODE_AUTO)


def test_static_scratch_rejects_oversized_calls():
    wl = W.CONFIGS["c2"].replace(ctx_len=16)
    lp = W.layer_params(wl)
    cache = F.KVCache(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.n_dom, 16, wl.dtype, wl.rope_base, lp.dom_idx)
    big = F.fasa_cache.from_buffer_copy(cache.struct)
    big.batch = 4096          # 4096 x 8 x 1024 tokens of scores need 128 MiB > 64 MiB
    big.max_len = 1024
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    st = F.lib().fasa_decode_static_scratch(ctypes.byref(big), 1024, q.data_ptr(), 1024, 8, q.data_ptr(), None,
                                            None)
    assert st == 4  # FASA_ERR_WORKSPACE, nothing launched
