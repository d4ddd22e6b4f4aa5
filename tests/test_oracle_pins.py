"""Pins of the CPU oracle against facts fixed outside the oracle itself.

The pages ("Riepilogo Tecnico: APB-V", gist.science) print no worked example,
so every pin is a closed form, an invariant, a special case that reduces to a
library routine (torch fp64 scaled_dot_product_attention / softmax), or a
brute-force enumeration on tiny inputs.  Each is chosen so that a plausible
mistake (a dropped segment, a wrong partner index, a wrong tie order, a
transposed operand, a missing normaliser) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from sequence_sparse_attention_b200.synth import Workload, bf16_bits, chunk_offsets, make_inputs


def problem(w: Workload, l=None, lpf=None) -> oracle.Problem:
    return oracle.Problem(H=w.H, Hq=w.Hq, Hkv=w.Hkv, d=w.d, N=w.N, a=w.a, q=w.q,
                          offsets=chunk_offsets(w), l=w.l if l is None else l,
                          local_pair_full=w.local_pair_full if lpf is None else lpf)


def small(**kw) -> Workload:
    base = dict(name="pin", H=2, Hq=4, Hkv=2, d=32, N=420, a=20, q=16, l=24, frame=16, seed=7)
    base.update(kw)
    return Workload(**base)


def bits(w):
    Q, K, V, off = make_inputs(w)
    return Q, K, V, bf16_bits(Q), bf16_bits(K), bf16_bits(V)


def sdpa_rows(Q, K, V, key_pos, rows, h, G, causal_pos=None):
    """Library reference: fp64 SDPA of the given query rows over the given keys."""
    g = h // G
    q = Q[rows, h].double()[None, None]                  # [1,1,R,d]
    k = K[key_pos, g].double()[None, None]
    v = V[key_pos, g].double()[None, None]
    mask = None
    if causal_pos is not None:
        mask = (torch.as_tensor(key_pos)[None, :] <= torch.as_tensor(causal_pos)[:, None])[None, None]
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=1.0 / math.sqrt(Q.shape[-1]))
    s = (q @ k.transpose(-1, -2)) / math.sqrt(Q.shape[-1])
    if mask is not None:
        s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o[0, 0].numpy(), lse[0, 0].numpy()


def run_oracle(w, p, Qb, Kb, Vb, rows, heads):
    _, idx = oracle.scores_and_select(p, Qb, Kb)
    return oracle.prefill_rows(p, Qb, Kb, Vb, idx, rows, heads), idx


# ---------------------------------------------------------------- dense cases

def test_one_host_is_dense_causal():
    """Limitazioni: with one host the method degenerates to standard attention."""
    w = small(H=1, N=300, a=12, q=10, l=5)
    p = problem(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    rows = np.arange(w.N)
    (O, lse), _ = run_oracle(w, p, Qb, Kb, Vb, rows, list(range(w.Hq)))
    G = w.Hq // w.Hkv
    for h in range(w.Hq):
        o_ref, l_ref = sdpa_rows(Q, K, V, np.arange(w.N), rows, h, G, causal_pos=rows)
        np.testing.assert_allclose(O[:, h], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], l_ref, rtol=0, atol=1e-12)


def test_full_passing_blocks_is_dense_causal():
    """l >= every chunk: the passing blocks carry whole chunks -> dense causal."""
    w = small(H=3, N=400, a=16, q=12, l=10_000, Hq=6, Hkv=2)
    p = problem(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    rows = np.arange(w.N)
    (O, lse), idx = run_oracle(w, p, Qb, Kb, Vb, rows, list(range(w.Hq)))
    G = w.Hq // w.Hkv
    for h in range(w.Hq):
        o_ref, l_ref = sdpa_rows(Q, K, V, np.arange(w.N), rows, h, G, causal_pos=rows)
        np.testing.assert_allclose(O[:, h], o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], l_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("lpf", [1, 0])
def test_query_and_anchor_rows_exact(lpf):
    """Forward Fuso di Contesto e Query: query rows are exact; anchor rows causal."""
    w = small(H=2, l=3)
    p = problem(w, lpf=lpf)
    Q, K, V, Qb, Kb, Vb = bits(w)
    rows = np.r_[np.arange(w.a), np.arange(w.N - w.q, w.N)]
    (O, lse), _ = run_oracle(w, p, Qb, Kb, Vb, rows, list(range(w.Hq)))
    for h in range(w.Hq):
        o_ref, l_ref = sdpa_rows(Q, K, V, np.arange(w.N), rows, h, 2, causal_pos=rows)
        np.testing.assert_allclose(O[:, h], o_ref, atol=1e-12)
        np.testing.assert_allclose(lse[:, h], l_ref, atol=1e-12)


# ------------------------------------------------------------ key-set segments

def seg(off, v):
    return np.arange(off[v], off[v + 1])


@pytest.mark.parametrize("lpf", [1, 0])
def test_no_passing_blocks_reduces_to_subsequence_attention(lpf):
    """l = 0: a chunk row sees anchor, (partner chunk), and its own chunk
    causally -- i.e. dense causal attention over a gathered subsequence."""
    w = small(H=2, l=0)
    p = problem(w, lpf=lpf)
    off = chunk_offsets(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    A = np.arange(w.a)
    partner = {0: None, 1: None, 2: 1, 3: 0} if lpf else {v: None for v in range(4)}
    G = w.Hq // w.Hkv
    for v in range(4):
        rows = seg(off, v)
        keys = np.r_[A, seg(off, partner[v]) if partner[v] is not None else [], rows].astype(np.int64)
        (O, lse), _ = run_oracle(w, p, Qb, Kb, Vb, rows, list(range(w.Hq)))
        for h in range(w.Hq):
            o_ref, l_ref = sdpa_rows(Q, K, V, keys, rows, h, G, causal_pos=rows)
            np.testing.assert_allclose(O[:, h], o_ref, atol=1e-12)
            np.testing.assert_allclose(lse[:, h], l_ref, atol=1e-12)


@pytest.mark.parametrize("lpf", [1, 0])
def test_passing_blocks_enter_the_key_set(lpf):
    """With l > 0 a chunk row equals dense attention over
    [anchor | earlier chunks' passing blocks (other hosts) | partner | own causal]."""
    w = small(H=3, l=9, N=500, Hq=6, Hkv=3)
    p = problem(w, lpf=lpf)
    off = chunk_offsets(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    _, idx = oracle.scores_and_select(p, Qb, Kb)
    H, G = w.H, w.Hq // w.Hkv
    pair = lambda v: v if v < H else 2 * H - 1 - v
    for v in range(2 * H):
        rows = seg(off, v)
        for h in range(w.Hq):
            g = h // G
            parts = [np.arange(w.a)]
            for u in range(v):
                if lpf and pair(u) == pair(v):
                    continue
                parts.append(idx[u, g][idx[u, g] >= 0])
            if lpf and v >= H:
                parts.append(seg(off, 2 * H - 1 - v))
            parts.append(rows)
            keys = np.sort(np.concatenate(parts).astype(np.int64))
            O, lse = oracle.prefill_rows(p, Qb, Kb, Vb, idx, rows, [h])
            o_ref, l_ref = sdpa_rows(Q, K, V, keys, rows, h, G, causal_pos=rows)
            np.testing.assert_allclose(O[:, 0], o_ref, atol=1e-12)
            np.testing.assert_allclose(lse[:, 0], l_ref, atol=1e-12)


def test_key_set_counts_one_host_vs_zigzag():
    """Passing blocks per row: each physical host receives 2H-2 blocks in total
    (Bilanciamento del Carico dell'Attenzione Approssimata), counted from the
    oracle's own key sets with exact integers."""
    for H in (2, 3, 4):
        w = small(H=H, N=16 + 8 + 2 * H * 30, a=16, q=8, l=4)
        p = problem(w)
        off = chunk_offsets(w)
        idx = np.zeros((2 * H - 1, w.Hkv, w.l), dtype=np.int32)
        for u in range(2 * H - 1):
            idx[u, :, :] = off[u] + np.arange(w.l)       # any valid selection
        per_host = {}
        for v in range(2 * H):
            t = int(off[v])                                # first row: local = 1 key
            n = len(oracle.key_set(p, idx, t, 0))
            partner = 30 if v >= H else 0
            n_blocks = (n - w.a - 1 - partner) // w.l
            host = oracle.pair(H, v)
            per_host[host] = per_host.get(host, 0) + n_blocks
            # total attended pairs of the chunk
        assert set(per_host.values()) == {2 * H - 2}, per_host


def test_zigzag_equal_work_per_physical_host():
    """Equal chunks -> every physical host attends exactly the same number of
    (row, key) pairs (ZigZag load balance), exact integers."""
    H = 3
    w = small(H=H, N=10 + 6 + 2 * H * 24, a=10, q=6, l=5)
    p = problem(w)
    off = chunk_offsets(w)
    idx = np.zeros((2 * H - 1, w.Hkv, w.l), dtype=np.int32)
    for u in range(2 * H - 1):
        idx[u, :, :] = off[u] + 2 * np.arange(w.l)
    work = {}
    for v in range(2 * H):
        pairs = sum(len(oracle.key_set(p, idx, t, 1)) for t in range(off[v], off[v + 1]))
        work[oracle.pair(H, v)] = work.get(oracle.pair(H, v), 0) + pairs
    assert len(set(work.values())) == 1, work
    for v in range(2 * H):
        assert oracle.pair(H, v) == oracle.pair(H, 2 * H - 1 - v)


# ---------------------------------------------------------------------- scores

def test_scores_match_library_softmax():
    """S_u[g, j] = sum over query rows and group heads of softmax over chunk u."""
    w = small(H=2, Hq=6, Hkv=2)
    p = problem(w)
    off = chunk_offsets(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    G = w.Hq // w.Hkv
    for u in range(2 * w.H - 1):
        for g in range(w.Hkv):
            S = oracle.chunk_scores(p, Qb, Kb, u, g)
            qr = Q[w.N - w.q:, g * G:(g + 1) * G].double()           # [q, G, d]
            k = K[off[u]:off[u + 1], g].double()                       # [n, d]
            x = torch.einsum("igc,jc->gij", qr, k) / math.sqrt(w.d)
            ref = torch.softmax(x, dim=-1).sum(dim=(0, 1)).numpy()
            np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-14)


def test_score_mass_closed_form():
    """Every softmax row sums to one -> the chunk's scores sum to G*q."""
    w = small(H=2, Hq=6, Hkv=3, q=11)
    p = problem(w)
    _, _, _, Qb, Kb, _ = bits(w)
    G = w.Hq // w.Hkv
    for u in range(2 * w.H - 1):
        for g in range(w.Hkv):
            S = oracle.chunk_scores(p, Qb, Kb, u, g)
            assert abs(S.sum() - G * w.q) < 1e-10
            assert (S > 0).all()


def test_scores_uniform_for_identical_keys():
    w = small(H=2)
    p = problem(w)
    off = chunk_offsets(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    K[:] = K[0:1, 0:1]
    Kb = bf16_bits(K)
    G = w.Hq // w.Hkv
    for u in range(3):
        S = oracle.chunk_scores(p, Qb, Kb, u, 1)
        n = off[u + 1] - off[u]
        np.testing.assert_allclose(S, G * w.q / n, rtol=1e-13)


# ------------------------------------------------------------------- selection

def test_selection_matches_bruteforce_sort():
    rng = np.random.default_rng(3)
    for n, l in [(37, 5), (64, 64), (50, 80), (200, 17), (9, 0)]:
        S = rng.integers(0, 6, size=n).astype(np.float64) / 7.0   # many exact ties
        got = oracle.select_top_l(S, 1000, l)
        order = sorted(range(n), key=lambda j: (-S[j], j))
        keep = sorted(order[: min(l, n)])
        want = np.array([1000 + j for j in keep] + [-1] * (l - min(l, n)), dtype=np.int32)
        np.testing.assert_array_equal(got, want)


def test_zero_keys_select_first_positions():
    """K = 0: every score ties, so the lower-index rule keeps the first l_eff."""
    w = small(H=2, l=7)
    p = problem(w)
    off = chunk_offsets(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    K.zero_()
    _, idx = oracle.scores_and_select(p, Qb, bf16_bits(K))
    for u in range(3):
        for g in range(w.Hkv):
            np.testing.assert_array_equal(idx[u, g], off[u] + np.arange(7))


def test_planted_key_is_selected():
    """A key aligned with the query block's mean gets the largest score."""
    w = small(H=2, l=1, Hq=4, Hkv=2)
    p = problem(w)
    off = chunk_offsets(w)
    Q, K, V, Qb, Kb, Vb = bits(w)
    G = w.Hq // w.Hkv
    plant = {}
    for u in range(3):
        for g in range(w.Hkv):
            j = int(off[u] + (7 * u + 3 * g) % (off[u + 1] - off[u]))
            K[j, g] = (Q[w.N - w.q:, g * G:(g + 1) * G].float().mean(dim=(0, 1)) * 40).to(K.dtype)
            plant[(u, g)] = j
    _, idx = oracle.scores_and_select(p, Qb, bf16_bits(K))
    for (u, g), j in plant.items():
        assert idx[u, g, 0] == j


def test_validation_rejects_bad_splits():
    w = small()
    good = problem(w)
    assert oracle.validate(good)
    off = chunk_offsets(w)
    bad = [off.copy() for _ in range(3)]
    bad[0][0] += 1          # anchor boundary
    bad[1][-1] -= 1         # query boundary
    bad[2][2] = bad[2][1]   # empty chunk
    for b in bad:
        p = problem(w)
        p.offsets = b
        assert not oracle.validate(p)
    p = problem(w)
    p.Hq = 5
    assert not oracle.validate(p)


# ---------------------------------------------------------------- selection variants

def row_softmax_scores(Q, K, w, u, g, norm_over_all):
    """Library reference for the scores of chunk u: torch fp64 softmax of each
    query row over the chunk, or over every key the row attends ([0, t]),
    summed over the query rows and the query heads of KV head g."""
    G = w.Hq // w.Hkv
    off = chunk_offsets(w)
    j0, j1 = int(off[u]), int(off[u + 1])
    S = torch.zeros(j1 - j0, dtype=torch.float64)
    for h in range(g * G, (g + 1) * G):
        for i in range(w.q):
            t = w.N - w.q + i
            q = Q[t, h].double()
            k0, k1 = (0, t + 1) if norm_over_all else (j0, j1)
            x = (K[k0:k1, g].double() @ q) / math.sqrt(w.d)
            p = torch.softmax(x, dim=0)
            S += p[j0 - k0:j1 - k0]
    return S.numpy()


@pytest.mark.parametrize("norm", [0, 1])
def test_scores_against_library_softmax(norm):
    """Both normalisations against torch's softmax, row by row."""
    w = small(H=2, N=260, a=12, q=6, l=8, Hq=4, Hkv=2, d=16)
    Q, K, V, Qb, Kb, Vb = bits(w)
    p = problem(w)
    p.score_norm = norm
    for u in range(2 * w.H - 1):
        for g in range(w.Hkv):
            np.testing.assert_allclose(oracle.chunk_scores(p, Qb, Kb, u, g),
                                       row_softmax_scores(Q, K, w, u, g, norm == 1), rtol=1e-12, atol=1e-15)


def test_row_normalised_scores_of_identical_keys():
    """score_norm 1 with every key equal: each query row spreads 1/(t+1) over
    its t+1 keys, so every key of every chunk scores sum_{h in g, i} 1/(t_i+1)."""
    w = small(H=2, N=300, a=10, q=8, l=4)
    Q, K, V, Qb, Kb, Vb = bits(w)
    Kb = np.ascontiguousarray(np.broadcast_to(Kb[:1], Kb.shape))
    p = problem(w)
    p.score_norm = 1
    G = w.Hq // w.Hkv
    want = G * sum(1.0 / (w.N - w.q + i + 1) for i in range(w.q))
    for u in range(2 * w.H - 1):
        np.testing.assert_allclose(oracle.chunk_scores(p, Qb, Kb, u, 0), want, rtol=1e-12)


def test_row_normalised_scores_sum_to_the_context_mass():
    """score_norm 1: the scores of all producing chunks add up to each row's
    attention mass on those chunks -- G*q minus the mass on the anchor, the
    last chunk and the query block, computed here with torch."""
    w = small(H=2, N=240, a=10, q=6, l=4, d=16)
    Q, K, V, Qb, Kb, Vb = bits(w)
    p = problem(w)
    p.score_norm = 1
    off = chunk_offsets(w)
    G = w.Hq // w.Hkv
    for g in range(w.Hkv):
        total = sum(oracle.chunk_scores(p, Qb, Kb, u, g).sum() for u in range(2 * w.H - 1))
        mass = 0.0
        for h in range(g * G, (g + 1) * G):
            for i in range(w.q):
                t = w.N - w.q + i
                x = (K[:t + 1, g].double() @ Q[t, h].double()) / math.sqrt(w.d)
                pr = torch.softmax(x, dim=0)
                mass += float(pr[int(off[0]):int(off[2 * w.H - 1])].sum())
        np.testing.assert_allclose(total, mass, rtol=1e-12)


def test_pool_sums_brute_force():
    """Window sums against numpy's convolution with a box of w ones (zero
    outside), float64 and float32, and w <= 1 as the identity."""
    rng = np.random.default_rng(3)
    for n in (1, 2, 5, 37):
        S = rng.random(n)
        for wdw in (1, 3, 5, 7):
            want = np.convolve(S, np.ones(wdw), mode="same") if wdw <= n else None
            got = oracle.pool_sums(S, wdw)
            if want is not None:
                np.testing.assert_allclose(got, want, rtol=1e-13)
            # clipped window, summed directly
            h = wdw // 2
            direct = np.array([S[max(0, j - h):j + h + 1].sum() for j in range(n)])
            np.testing.assert_allclose(got, direct, rtol=1e-13)
            got32 = oracle.pool_sums(S.astype(np.float32), wdw)
            ref32 = np.zeros(n, dtype=np.float32)
            for j in range(n):
                acc = np.float32(0)
                for k in range(max(0, j - h), min(n, j + h + 1)):
                    acc = np.float32(acc + np.float32(S[k]))
                ref32[j] = acc
            assert np.array_equal(got32, ref32)
    np.testing.assert_array_equal(oracle.pool_sums(np.arange(4.0), 1), np.arange(4.0))


def test_pooled_selection_takes_the_window_of_a_spike():
    """One dominant score: with pooling of width w and l = w the passing block
    is exactly the w keys centred on it (a plausible off-by-one in the window
    fails this)."""
    n, spike, wdw = 40, 17, 5
    S = np.full(n, 1e-3)
    S[spike] = 10.0
    idx = oracle.select_top_l(oracle.pool_sums(S, wdw), 100, wdw)
    np.testing.assert_array_equal(idx, 100 + np.arange(spike - 2, spike + 3))


def test_variant_flags_are_validated():
    w = small()
    Q, K, V, Qb, Kb, Vb = bits(w)
    for norm, pool in ((2, 0), (0, 4), (-1, 0), (0, -3)):
        p = problem(w)
        p.score_norm, p.score_pool = norm, pool
        with pytest.raises(ValueError):
            oracle.chunk_scores(p, Qb, Kb, 0, 0)


def _compositions(n, k):
    """Every way of writing n as an ordered sum of k positive integers."""
    if k == 1:
        yield (n,)
        return
    for first in range(1, n - k + 2):
        for rest in _compositions(n - first, k - 1):
            yield (first,) + rest


@pytest.mark.parametrize("H,n_frames", [(1, 2), (1, 5), (2, 4), (2, 7), (2, 11), (3, 6), (3, 13)])
def test_plan_chunks_brute_force(H, n_frames):
    """Visual load balancing, pinned by enumeration: over EVERY split of the
    frame list into 2H runs of consecutive whole frames, the ones whose frame
    counts differ by at most one and never grow from one virtual host to the
    next are a single split, and it is the oracle's; the offsets add up the
    tokens of each run after the anchor."""
    rng = np.random.default_rng(100 * H + n_frames)
    ft = rng.integers(1, 50, n_frames)
    nc = 2 * H
    even = [c for c in _compositions(n_frames, nc)
            if max(c) - min(c) <= 1 and all(c[v] >= c[v + 1] for v in range(nc - 1))]
    assert len(even) == 1
    counts = even[0]
    a = int(rng.integers(0, 30))
    want = [a]
    f = 0
    for c in counts:
        want.append(want[-1] + int(sum(ft[f:f + c])))
        f += c
    np.testing.assert_array_equal(oracle.plan_chunks(H, ft, a), want)


def test_plan_chunks_equal_frames_are_equal_chunks():
    """Closed form: n_frames = 2H m frames of F tokens give chunks of m F tokens."""
    off = oracle.plan_chunks(4, [256] * 64, 1024)
    np.testing.assert_array_equal(off, 1024 + 256 * 8 * np.arange(9))


@pytest.mark.parametrize("args", [(2, [5, 5, 5], 0), (1, [5, 0], 0), (1, [5, 5], -1), (0, [5, 5], 0)])
def test_plan_chunks_rejects_impossible_splits(args):
    with pytest.raises(ValueError):
        oracle.plan_chunks(*args)


@pytest.mark.parametrize("lpf", [0, 1])
@pytest.mark.parametrize("H,a,l,jitter", [(1, 16, 4, 0.0), (2, 0, 7, 0.0), (3, 10, 5, 0.2),
                                          (4, 9, 100, 0.0), (2, 12, 0, 0.3)])
def test_attended_pairs_closed_form_counts_the_key_sets(lpf, H, a, l, jitter):
    """The closed-form pair count equals the sizes of the key sets listed one
    row at a time (any valid selection: every passing block has l_eff keys)."""
    w = small(H=H, N=a + 8 + 2 * H * 32, a=a, q=8, l=l, frame=8, jitter=jitter,
              local_pair_full=lpf)
    p = problem(w)
    off = chunk_offsets(w)
    idx = np.full((2 * H - 1, w.Hkv, max(l, 1)), -1, dtype=np.int32)[:, :, :l]
    for u in range(2 * H - 1):
        k = min(l, int(off[u + 1] - off[u]))
        idx[u, :, :k] = off[u] + np.arange(k)
    counts = [0, 0, 0]
    for t in range(w.N):
        cls = 0 if t < w.a else (2 if t >= w.N - w.q else 1)
        counts[cls] += len(oracle.key_set(p, idx, t, 0))
    assert oracle.attended_pairs(p) == tuple(counts)
