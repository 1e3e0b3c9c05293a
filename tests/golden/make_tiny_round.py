"""Writes tiny_fp32_round.json: the oracle's draft round on the tiny fp32 workload.

The pages print no worked example of a round, so this file holds no values of
theirs: every number in it is computed here by ``oracle/`` alone (fp64) from the
seeded inputs of ``synthetic/`` (tiny fp32 round: 1 layer, hidden 256, 4 q-heads
x head_dim 64, 1 kv head with k = v, intermediate 512, vocab 1024, markov rank 8,
gamma 4, one row of 32 context positions 0..31, seed 0). It is a regression
snapshot of the oracle, not a pin: ``tests/test_oracle_golden.py`` checks that
the oracle still reproduces it, so a change to the oracle's arithmetic shows up
and has to be justified where it is made. Run from the repository root:

    python tests/golden/make_tiny_round.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_round.json")


def tiny_round():
    from oracle import dspark as O
    from synthetic import WORKLOADS, make_round_inputs, make_weights

    wl = WORKLOADS["tiny_fp32"]
    cpu = make_weights(wl.model, wl.seed)
    inp = make_round_inputs(wl)
    lens = inp["ctx_len"].tolist()
    W = O.OracleWeights(cpu, wl.model)
    kv = O.project_context_kv(W, inp["hidden"], inp["pos0"].tolist(), lengths=lens)
    ref = O.draft_rows(W, kv, inp["anchors"].tolist(), inp["block_pos"].tolist())
    U = np.asarray(ref["base_logits"], dtype=np.float64)          # [A, gamma, V]
    top = np.argsort(-U, axis=-1, kind="stable")[..., :5]
    k0, v0 = kv[0][0]
    return {
        "workload": "tiny fp32 round (1 layer, hidden 256, 4x64 heads, 1 kv head, vocab 1024, rank 8, gamma 4, "
                    "32 context rows, seed 0)",
        "source": "oracle/dspark.py via tests/golden/make_tiny_round.py",
        "anchors": inp["anchors"].tolist(),
        "tokens": np.asarray(ref["tokens"]).astype(int).tolist(),
        "lengths": np.asarray(ref["lengths"]).astype(int).tolist(),
        "conf": np.asarray(ref["conf"], dtype=np.float64).tolist() if "conf" in ref else None,
        "logits_top5_index": top.astype(int).tolist(),
        "logits_top5_value": np.take_along_axis(U, top, axis=-1).tolist(),
        "logits_row_sum": U.sum(axis=-1).tolist(),
        "k_ctx_layer0_row0": np.asarray(k0, dtype=np.float64).reshape(-1, np.asarray(k0).shape[-1])[0].tolist(),
        "v_ctx_layer0_row0": np.asarray(v0, dtype=np.float64).reshape(-1, np.asarray(v0).shape[-1])[0].tolist(),
    }


if __name__ == "__main__":
    with open(OUT, "w") as fh:
        json.dump(tiny_round(), fh, indent=1)
    print("wrote", OUT)
