"""The multi-GPU path is replicas only: every rank decodes its own copy of the
workload with no data-path collective. What the ranks share is the timing
(the slowest rank's step time, all-reduced) and the whole-job value. Those
host-side pieces run here as two gloo ranks on CPU; the oracle checks that a
split of the (batch, KV head) units over ranks reproduces the unsplit run."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle.fasa_oracle as O
from rope_frequency_chunk_b200 import workloads as W

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, fn, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        out[rank] = fn(rank)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run(fn):
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(_free_port(), fn, out), nprocs=WORLD, join=True)
    return [out[r] for r in range(WORLD)]


def _max_fn(rank):
    return bench.max_over_ranks([3.5, 7.25][rank], dist, "cpu")


def test_step_time_is_the_max_over_ranks():
    assert _run(_max_fn) == [7.25, 7.25]


def test_single_process_time_is_its_own():
    assert bench.max_over_ranks(4.0, None) == 4.0


def test_whole_job_value_counts_every_rank():
    # 2 ranks x 1 GB per step in 0.5 ms (the slower rank) = 4000 GB/s
    assert bench.job_gbs(1e9, 0.5, 2) == pytest.approx(4000.0)
    assert bench.job_gbs(1e9, 0.5, 1) == pytest.approx(2000.0)


SMALL = W.CONFIGS["c2"].replace(batch=2, n_q_heads=8, n_kv_heads=2, ctx_len=300, k=40)


def _units(wl):
    return [(b, g) for b in range(wl.batch) for g in range(wl.n_kv_heads)]


def _decode_unit(wl, lp, b, g):
    kk, vv = W.head_kv(wl, lp, 0, b, g)
    k_rot, v_st, sk = O.append_kv(kk, vv, 0, wl.rope_base, lp.dom_idx[g], wl.dtype)
    qq = W.head_q(wl, lp, 0, b, g)
    idx, out, _ = O.decode_head(qq, wl.q_pos, k_rot, v_st, sk, lp.dom_idx[g], wl.k, wl.rope_base)
    return np.asarray(out), np.asarray(idx)


def _shard_fn(rank):
    wl = SMALL
    lp = W.layer_params(wl, 0)
    mine = _units(wl)[rank::WORLD]
    res = {u: _decode_unit(wl, lp, *u) for u in mine}
    gathered = [None] * WORLD
    dist.all_gather_object(gathered, res)
    merged = {}
    for part in gathered:
        merged.update(part)
    return {k: (v[0].tolist(), v[1].tolist()) for k, v in merged.items()}


def test_units_split_over_ranks_reproduce_the_single_run():
    per_rank = _run(_shard_fn)
    assert per_rank[0] == per_rank[1]
    wl = SMALL
    lp = W.layer_params(wl, 0)
    for u in _units(wl):
        out, idx = _decode_unit(wl, lp, *u)
        got_out, got_idx = per_rank[0][u]
        assert got_idx == idx.tolist()
        np.testing.assert_array_equal(np.asarray(got_out), out)


def test_reference_arm_prints_on_rank_zero_only(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.build_parser().parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args, W.CONFIGS["c1"]) == 0
    assert capsys.readouterr().out == ""


def test_profiled_traffic_is_gated_by_workload_and_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu record (JSON) only for the
    captured kernel and workload, and only while the kernel's sources are the
    captured ones."""
    import json
    wl = bench.W.CONFIGS["c2"]
    sig = bench.workload_sig(wl, wl.k)
    assert sig == "c2-B1-H32/8-L32768-n16-k256-bf16"
    srcs = ["decode_wide.cuh", "tip.cuh"]
    rec = {f"decode_wide_kernel@{sig}": {"bytes_per_launch": 123, "sources": srcs,
                                         "csrc_sha256": bench.csrc_sha256(srcs)}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.profiled_traffic("decode_wide_kernel", sig) == 123
    assert bench.profiled_traffic("decode_wide_kernel", bench.workload_sig(wl, 512)) is None
    assert bench.profiled_traffic("score_kernel", sig) is None
    # the digest covers the named sources only; any change there voids the figure
    assert bench.csrc_sha256(srcs) != bench.csrc_sha256(["decode_wide.cuh"])
    monkeypatch.setattr(bench, "csrc_sha256", lambda files=None: "0" * 64)
    assert bench.profiled_traffic("decode_wide_kernel", sig) is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.profiled_traffic("decode_wide_kernel", sig) is None
