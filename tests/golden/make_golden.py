"""Writes tests/golden/tiny_decode.json: a regression fixture computed by the
CPU oracle alone (the pages print no worked numeric example).

Inputs: numpy PCG64 seed 2026, one KV head with G = 2 query heads, L = 48
cached bf16 tokens at positions 0..47, query at position 48, RoPE base 1e4,
dominant FCs [3, 60, 11, 0, 33], k = 7.

Run:  python -m tests.golden.make_golden
"""
import json
import os

import numpy as np

import oracle.fasa_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def compute_golden():
    r = np.random.default_rng(2026)
    L, G, base, k = 48, 2, 1e4, 7
    dom = np.array([3, 60, 11, 0, 33])
    q_pre = O.store(r.standard_normal((G, 128)), "bf16")
    k_pre = O.store(r.standard_normal((L, 128)), "bf16")
    v = O.store(r.standard_normal((L, 128)), "bf16")
    k_rot, v_st, sk = O.append_kv(k_pre, v, 0, base, dom, "bf16")
    idx, out, s = O.decode_head(q_pre, L, k_rot, v_st, sk, dom, k, base)
    return {"idx": [int(i) for i in idx], "out": out.tolist(), "scores": s.tolist()}


if __name__ == "__main__":
    g = compute_golden()
    g["_about"] = ("FASA decode of one KV head by the CPU oracle; see make_golden.py "
                   "for the inputs. Regression fixture only.")
    with open(os.path.join(HERE, "tiny_decode.json"), "w") as f:
        json.dump(g, f)
    print("wrote", len(g["idx"]), "indices")
