"""Writes tiny_oracle.json: the oracle's passing blocks and a few output rows of
the tiny layer (H=2, 4 q / 2 kv heads, d=64, 2048 tokens, seed 0).  Calls only
oracle/ and the seeded input generator; run it again only for a change of the
oracle that names the passage or reading that justifies it."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "..", ".."))

import oracle  # noqa: E402
from sequence_sparse_attention_b200.synth import WORKLOADS, bf16_bits, chunk_offsets, make_inputs  # noqa: E402

ROWS = [0, 63, 64, 551, 1040, 1528, 2015, 2016, 2047]  # anchor, chunk edges, query block


def compute():
    w = WORKLOADS["tiny"]
    Q, K, V, _ = make_inputs(w)
    p = oracle.Problem(H=w.H, Hq=w.Hq, Hkv=w.Hkv, d=w.d, N=w.N, a=w.a, q=w.q,
                       offsets=chunk_offsets(w), l=w.l, local_pair_full=w.local_pair_full)
    Qb, Kb, Vb = bf16_bits(Q), bf16_bits(K), bf16_bits(V)
    scores, idx = oracle.scores_and_select(p, Qb, Kb)
    O, lse = oracle.prefill_rows(p, Qb, Kb, Vb, idx, np.array(ROWS), list(range(w.Hq)))
    return {"workload": "tiny", "rows": ROWS, "idx": idx.tolist(),
            "score_sums": scores.sum(axis=1).tolist(),
            "O": O.round(12).tolist(), "lse": lse.round(12).tolist()}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(compute(), f, separators=(",", ":"))
    print("written")
