"""The tie-aware output comparison of the end-to-end parity tests (host logic,
no GPU): which outputs are unique when a selection broke a tie differently."""
import numpy as np
import pytest
import torch

from parity_util import check_convex, unique_mask
from sequence_sparse_attention_b200.synth import Workload, chunk_offsets


def test_unique_mask_marks_later_chunks_of_that_group():
    w = Workload("m", H=2, Hq=4, Hkv=2, d=64, N=700, a=60, q=40, l=20, frame=32, seed=0)
    off = chunk_offsets(w)
    ref = np.arange(3 * 2 * 20, dtype=np.int32).reshape(3, 2, 20)
    gpu = ref.copy()
    gpu[1, 0, 5] += 1                     # chunk 1, KV group 0 took another key
    rows = np.arange(w.N)
    m = unique_mask(w, gpu, ref, rows, [0, 1, 2, 3])
    v = np.searchsorted(off, rows, side="right") - 1
    context = (rows >= w.a) & (rows < w.N - w.q)
    for t in rows:
        for h in range(4):
            tied = context[t] and h // 2 == 0 and v[t] >= 2
            assert m[t, h] == (not tied), (t, h)
    assert unique_mask(w, ref, ref, rows, [0, 1, 2, 3]).all()


def test_check_convex_bounds():
    # two KV groups with different ranges; heads 0, 1 -> group 0, heads 2, 3 -> group 1
    V = torch.tensor([[[0.0, -1.0], [10.0, 10.0]], [[2.0, 1.0], [12.0, 11.0]]])  # [N, Hkv, d]
    O = np.array([[[1.0, 0.0], [2.0, -1.0], [11.0, 10.5], [12.0, 11.0]]])     # [1, 4 heads, d]
    everything = np.ones((1, 4), dtype=bool)
    check_convex(O, V, [0, 1, 2, 3], 2, everything)
    bad = O.copy()
    bad[0, 2, 0] = 2.5                    # inside group 0's range, below group 1's
    with pytest.raises(AssertionError):
        check_convex(bad, V, [0, 1, 2, 3], 2, everything)
    skip = everything.copy()
    skip[0, 2] = False                    # entries outside the mask are not checked
    check_convex(bad, V, [0, 1, 2, 3], 2, skip)
    bad[0, 0, 1] = np.nan
    with pytest.raises(AssertionError):
        check_convex(bad, V, [0, 1, 2, 3], 2, skip)
