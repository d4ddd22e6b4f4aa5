"""Shared helpers of the GPU parity tests: run the oracle and compare.

Expected values come only from the oracle (tests/ may call it); the GPU path is
the libspava C ABI through sequence_sparse_attention_b200.api.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sequence_sparse_attention_b200.synth import Workload, bf16_bits, chunk_offsets

# Output gates: bf16 outputs against the fp64 oracle.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 2e-3
# Selection band: a selection may differ from the oracle's only among keys
# whose oracle score is within this relative distance of the l-th score.
SEL_BAND = 1e-3
# Scores: fp32 accumulation of ex2.approx terms vs fp64.
SCORE_REL = 1e-3


def problem(w: Workload, off=None) -> oracle.Problem:
    return oracle.Problem(H=w.H, Hq=w.Hq, Hkv=w.Hkv, d=w.d, N=w.N, a=w.a, q=w.q,
                          offsets=chunk_offsets(w) if off is None else off, l=w.l,
                          local_pair_full=w.local_pair_full, score_norm=w.score_norm,
                          score_pool=w.score_pool)


class OracleRun:
    """The oracle on one layer's inputs (host bf16 bit patterns)."""

    def __init__(self, w: Workload, Q, K, V, groups=None):
        self.w = w
        self.p = problem(w)
        self.Qb, self.Kb, self.Vb = bf16_bits(Q), bf16_bits(K), bf16_bits(V)
        self.groups = list(range(w.Hkv)) if groups is None else list(groups)
        self.scores, self.idx = oracle.scores_and_select(self.p, self.Qb, self.Kb, self.groups)

    def rows(self, rows, heads, idx=None):
        return oracle.prefill_rows(self.p, self.Qb, self.Kb, self.Vb,
                                   self.idx if idx is None else idx, rows, heads)


def check_selection(w: Workload, scores_oracle: np.ndarray, idx_gpu: np.ndarray, groups,
                    idx_oracle: np.ndarray | None = None) -> dict:
    """Every (chunk, group) selection is a valid top-l of the oracle scores (or
    of their window sums, with pooling): the same set wherever the l-th /
    (l+1)-th gap exceeds SEL_BAND relative, otherwise the same outside the band
    around the l-th value.

    Returns counts for the record: ``exact`` selections decided by a clear gap
    (or trivially: l = 0 or l >= n), ``band`` selections whose l-th and
    (l+1)-th scores lie within the band, ``band_keys`` the number of keys
    inside each such band, and ``differ`` the selections that are not the
    oracle's own (possible only inside a band)."""
    scores_oracle = oracle.selection_scores(problem(w), scores_oracle)
    off = chunk_offsets(w)
    rep = {"exact": 0, "band": 0, "band_keys": [], "differ": 0}
    for u in range(2 * w.H - 1):
        n = int(off[u + 1] - off[u])
        k = min(w.l, n)
        s0 = int(off[u] - w.a)
        for g in groups:
            got = idx_gpu[u, g]
            assert (got[k:] == -1).all(), (u, g, "padding")
            sel = got[:k]
            assert (np.diff(sel) > 0).all(), (u, g, "not ascending")
            assert ((sel >= off[u]) & (sel < off[u + 1])).all(), (u, g, "outside chunk")
            if idx_oracle is not None and not np.array_equal(got, idx_oracle[u, g]):
                rep["differ"] += 1
            if k == 0 or k == n:
                rep["exact"] += 1
                continue
            S = scores_oracle[g, s0:s0 + n]
            srt = np.sort(S)[::-1]
            sl, sl1 = srt[k - 1], srt[k]
            chosen = np.zeros(n, dtype=bool)
            chosen[sel - off[u]] = True
            if (sl - sl1) > SEL_BAND * abs(sl):
                want = S >= sl
                assert (chosen == want).all(), (u, g, "set differs with a clear gap")
                rep["exact"] += 1
            else:
                hi, lo = sl + SEL_BAND * abs(sl), sl - SEL_BAND * abs(sl)
                assert chosen[S > hi].all(), (u, g, "missed a key above the band")
                assert not chosen[S < lo].any(), (u, g, "took a key below the band")
                rep["band"] += 1
                rep["band_keys"].append(int(((S >= lo) & (S <= hi)).sum()))
    return rep


def expected_rows(ref: "OracleRun", idx_gpu: np.ndarray, rows, heads, cached=None):
    """The oracle's outputs for the GPU's own selection.

    Once `check_selection` has accepted ``idx_gpu`` as a correct top-l (equal
    to the oracle's wherever the scores leave no choice, inside the band where
    they tie), every row has exactly one expected output: the oracle's
    attention over the key set that selection gives.  Where the two
    selections are identical that is the oracle's own result (``cached``, if
    given, is returned)."""
    if cached is not None and np.array_equal(idx_gpu, ref.idx):
        return cached
    return ref.rows(rows, heads, idx=idx_gpu)


def check_outputs(O_gpu: np.ndarray, O_ref: np.ndarray, what=""):
    err = np.abs(O_gpu.astype(np.float64) - O_ref)
    assert np.isfinite(O_gpu).all(), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= O_MAX_ABS, f"{what}: max-abs {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean-abs {mean:.3e} > {O_MEAN_ABS}"
    return mx, mean


def sample_rows(w: Workload, per_chunk=6, seed=0):
    """First and last rows of every chunk, a few random rows, some anchor and
    query rows."""
    off = chunk_offsets(w)
    rng = np.random.default_rng(seed)
    rows = set()
    if w.a:
        rows.update([0, w.a - 1, min(w.a - 1, 127), min(w.a - 1, 128)])
        rows.update(rng.integers(0, w.a, 2).tolist())
    for v in range(2 * w.H):
        lo, hi = int(off[v]), int(off[v + 1])
        rows.update([lo, lo + 1, hi - 1, min(hi - 1, lo + 127), min(hi - 1, lo + 128)])
        rows.update(rng.integers(lo, hi, max(0, per_chunk - 5)).tolist())
    rows.update([w.N - w.q, w.N - 1])
    rows.update(rng.integers(w.N - w.q, w.N, 4).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def gpu_tensors(Q, K, V, device="cuda"):
    return Q.to(device), K.to(device), V.to(device)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()
