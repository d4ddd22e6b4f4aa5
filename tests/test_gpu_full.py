"""Parity at the full layer sizes of the long-video study (16K, 64K, 128K and
256K tokens), in the launch configuration bench.py times (the four C-ABI steps
on one stream), checked on what the oracle can compute one by one: the scores
and passing blocks of every KV group, and the outputs of sampled rows
(first/last rows of every chunk and of every 128-row tile edge, random rows,
anchor and query rows) for every query head.  Every selection
of every group is also checked for validity (ascending, inside its chunk,
-1 padded)."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (LSE_ABS, O_MAX_ABS, O_MEAN_ABS, SCORE_REL, check_outputs, check_selection,
                         problem, sample_rows, to_np)
from sequence_sparse_attention_b200.api import Layout, Spava
from sequence_sparse_attention_b200.synth import WORKLOADS, bf16_bits, chunk_offsets, make_inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def run_layer_like_bench(sp: Spava, Q, K, V):
    w = sp.lay
    scores = torch.zeros((w.Hkv, w.context), dtype=torch.float32, device=Q.device)
    idx = torch.empty((2 * w.H - 1, w.Hkv, w.l), dtype=torch.int32, device=Q.device)
    sp.score(Q, K, scores)
    sp.topk_select(scores, idx)
    pk, pv = sp.pack_passing(K, V, idx)
    O, lse = sp.attn(Q, K, V, pk, pv)
    torch.cuda.synchronize()
    return scores, idx, O, lse


def checked_groups(w):
    """KV groups compared with the oracle: every one of them, on every layer."""
    return list(range(w.Hkv))


@pytest.mark.parametrize("name", ["16k", "64k", "128k", "256k"])
def test_full_size_layer(name):
    w = WORKLOADS[name]
    Q, K, V, off = make_inputs(w, "cuda")
    sp = Spava(Layout.from_workload(w))
    scores, idx, O, lse = run_layer_like_bench(sp, Q, K, V)
    assert sp.device_status() == 0
    idx_h = idx.cpu().numpy()

    # the layer entry point (fused selection + gather) gives the same bytes
    O2, lse2, idx2 = sp.prefill_attention(Q, K, V, want_idx=True)
    torch.cuda.synchronize()
    assert sp.device_status() == 0
    assert torch.equal(idx2, idx)
    assert torch.equal(O2.view(torch.int16), O.view(torch.int16))
    assert torch.equal(lse2, lse)
    del O2, lse2, idx2

    # every selection is well formed
    for u in range(2 * w.H - 1):
        k = min(w.l, int(off[u + 1] - off[u]))
        sel = idx_h[u, :, :k]
        assert (np.diff(sel, axis=1) > 0).all()
        assert ((sel >= off[u]) & (sel < off[u + 1])).all()
        assert (idx_h[u, :, k:] == -1).all()

    groups = checked_groups(w)
    p = problem(w, off)
    Qb, Kb, Vb = bf16_bits(Q), bf16_bits(K), bf16_bits(V)
    sc_ref, idx_ref = oracle.scores_and_select(p, Qb, Kb, groups)
    sc = to_np(scores)
    last0 = int(off[-2] - w.a)
    for g in groups:
        np.testing.assert_allclose(sc[g, :last0], sc_ref[g, :last0], rtol=SCORE_REL,
                                   atol=1e-7 * w.q * w.Hq / w.Hkv)
    rep = check_selection(w, sc_ref, idx_h, groups, idx_ref)
    # Every selection of every KV group is, bit for bit, the top-l of the GPU's
    # own fp32 scores (ties to the lower index): the selection step is exact
    # even where the oracle's fp64 scores leave a band of valid choices.
    for u in range(2 * w.H - 1):
        s0, n = int(off[u] - w.a), int(off[u + 1] - off[u])
        for g in range(w.Hkv):
            want = oracle.select_top_l(sc[g, s0:s0 + n].astype(np.float64), int(off[u]), w.l)
            np.testing.assert_array_equal(idx_h[u, g], want, err_msg=f"{name} u={u} g={g}")

    # Every sampled row and head against the oracle's attention over the key
    # sets of the GPU's (accepted) selection: nothing is exempt.
    G = w.Hq // w.Hkv
    heads = [h for g in groups for h in range(g * G, (g + 1) * G)]
    rows = sample_rows(w, per_chunk=8, seed=1)
    O_ref, lse_ref = oracle.prefill_rows(p, Qb, Kb, Vb, idx_h, rows, heads)
    O_got = to_np(O[torch.from_numpy(rows).cuda()][:, heads])
    mx, mean = check_outputs(O_got, O_ref, name)
    lse_got = to_np(lse[heads][:, torch.from_numpy(rows).cuda()]).T
    lse_err = float(np.abs(lse_got - lse_ref).max())
    assert lse_err <= LSE_ABS, f"{name}: lse {lse_err:.3e}"
    keys = rep["band_keys"]
    print(f"{name}: groups {groups}; selections exact {rep['exact']}, in band {rep['band']} "
          f"(keys in band: min {min(keys) if keys else 0}, max {max(keys) if keys else 0}, "
          f"total {sum(keys)}), differing from the oracle's {rep['differ']}; "
          f"{len(rows)} rows x {len(heads)} heads: O max-abs {mx:.2e} ({mx / O_MAX_ABS:.0%} of gate), "
          f"mean-abs {mean:.2e} ({mean / O_MEAN_ABS:.0%} of gate), lse {lse_err:.2e}")
