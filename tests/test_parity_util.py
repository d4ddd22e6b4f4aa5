"""The selection check of the end-to-end parity tests (host logic, no GPU):
which selections it accepts, what it counts, and that the expected outputs
follow the selection that was accepted."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import OracleRun, check_selection, expected_rows, problem
from sequence_sparse_attention_b200.synth import Workload, chunk_offsets, make_inputs

W = Workload("sel", H=2, Hq=4, Hkv=2, d=64, N=700, a=60, q=40, l=20, frame=32, seed=3)


@pytest.fixture(scope="module")
def ref():
    Q, K, V, _ = make_inputs(W)
    return OracleRun(W, Q, K, V)


def test_oracle_selection_is_accepted_as_exact(ref):
    rep = check_selection(W, ref.scores, ref.idx, range(W.Hkv), ref.idx)
    assert rep["differ"] == 0
    assert rep["exact"] + rep["band"] == (2 * W.H - 1) * W.Hkv


def test_swap_across_a_clear_gap_is_rejected(ref):
    off = chunk_offsets(W)
    bad = ref.idx.copy()
    # replace the best key of chunk 0, group 0 by the worst one
    S = ref.scores[0, : off[1] - off[0]]
    best, worst = off[0] + int(np.argmax(S)), off[0] + int(np.argmin(S))
    sel = [x for x in bad[0, 0] if x != best] + [worst]
    bad[0, 0] = np.sort(sel)
    with pytest.raises(AssertionError):
        check_selection(W, ref.scores, bad, range(W.Hkv), ref.idx)


def test_swap_inside_a_tie_band_is_accepted_and_counted(ref):
    off = chunk_offsets(W)
    u, g, k = 1, 1, W.l
    s0 = int(off[u] - W.a)
    n = int(off[u + 1] - off[u])
    scores = ref.scores.copy()
    S = scores[g, s0:s0 + n]
    order = np.argsort(-S, kind="stable")
    # plant a tie between the l-th and (l+1)-th key of this chunk
    S[order[k]] = S[order[k - 1]]
    idx_o = oracle.select_top_l(S, int(off[u]), W.l)
    idx_alt = np.sort(np.concatenate([np.setdiff1d(idx_o, [off[u] + order[k - 1]]),
                                      [off[u] + order[k]]])).astype(np.int32)
    assert not np.array_equal(idx_o, idx_alt)
    want = ref.idx.copy()
    want[u, g] = idx_o
    got = want.copy()
    got[u, g] = idx_alt
    rep = check_selection(W, scores, got, range(W.Hkv), want)
    assert rep["differ"] == 1 and rep["band"] >= 1 and min(rep["band_keys"]) >= 2


def test_expected_rows_follow_the_accepted_selection(ref):
    rows = np.arange(W.N)
    heads = list(range(W.Hq))
    cached = ref.rows(rows, heads)
    assert expected_rows(ref, ref.idx, rows, heads, cached) is cached
    off = chunk_offsets(W)
    other = ref.idx.copy()
    unused = np.setdiff1d(np.arange(off[0], off[1]), other[0, 0])[0]
    other[0, 0, -1] = unused               # chunk 0, KV group 0: one key swapped
    other[0, 0] = np.sort(other[0, 0])
    O2, lse2 = expected_rows(ref, other, rows, heads, cached)
    O_direct, lse_direct = oracle.prefill_rows(problem(W), ref.Qb, ref.Kb, ref.Vb, other, rows, heads)
    np.testing.assert_array_equal(O2, O_direct)
    # rows of chunk 1.. of KV group 0 read that passing block; chunk 0 does not
    g0 = [h for h in heads if h // 2 == 0]
    later = (rows >= off[2]) & (rows < W.N - W.q)
    assert np.abs(O2[later][:, g0] - cached[0][later][:, g0]).max() > 0
    early = rows < off[1]
    np.testing.assert_array_equal(O2[early], cached[0][early])
