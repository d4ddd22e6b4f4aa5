"""The ZigZag sequence-parallel shards on the host (no GPU): which chunks and
rows each rank holds, the slots of its exchange messages, and -- with two gloo
ranks exchanging real messages -- that every rank ends up with exactly what its
rows' key sets need, checked against the oracle.

Shard rule under test: rank r of `world` holds the physical hosts p in
[r*m, (r+1)*m), m = H/world, i.e. chunks p and 2H-1-p of each ("Disposizione
ZigZag"), in local buffers [anchor | its chunks ascending | query block]; the
anchor and the query block are on every rank."""
import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sequence_sparse_attention_b200 import native
from sequence_sparse_attention_b200.api import Layout, local_positions, shard_layout, shard_sizes
from sequence_sparse_attention_b200.synth import WORKLOADS, Workload, bf16_bits, chunk_offsets, make_inputs


def pair(H, v):
    return v if v < H else 2 * H - 1 - v


@pytest.mark.parametrize("name,world", [("tiny", 1), ("tiny", 2), ("16k", 2), ("16k", 4),
                                        ("128k", 8), ("256k", 4), ("256k", 16)])
def test_ranks_partition_the_chunks_by_physical_host(name, world):
    w = WORKLOADS[name]
    lay = Layout.from_workload(w)
    off = chunk_offsets(w)
    m = w.H // world
    seen = []
    for r in range(world):
        first, n_local, slots = shard_layout(lay, r, world)
        held = [v for v in range(2 * w.H) if first[1 + v] >= 0]
        assert held == sorted(slots.tolist())
        assert all(pair(w.H, v) // m == r for v in held)
        assert len(held) == 2 * m
        pos = local_positions(lay, first)
        assert len(pos) == n_local == w.a + sum(int(off[v + 1] - off[v]) for v in held) + w.q
        assert (np.diff(pos) > 0).all()                      # regions in global order
        assert first[0] == 0 and first[-1] == n_local - w.q  # anchor first, query block last
        seen += held
    assert sorted(seen) == list(range(2 * w.H))             # every chunk on exactly one rank


def test_message_sizes_do_not_depend_on_the_rank():
    lay = Layout.from_workload(WORKLOADS["16k"])
    ws, pm, qm = shard_sizes(lay, 4)
    w = WORKLOADS["16k"]
    m = w.H // 4
    assert pm >= 2 * m * w.Hkv * w.l * (4 + 2 * 2 * w.d)
    assert qm >= 2 * m * w.Hq * w.q * (w.d + 1) * 4
    assert pm % 256 == 0 and qm % 256 == 0


@pytest.mark.parametrize("change,world,expect", [
    ({}, 3, 2),                     # world does not divide H = 4
    ({}, 0, 1),
    (dict(score_norm=1), 2, 2),     # row-normalised scores need every chunk's statistics
])
def test_shard_rejects(change, world, expect):
    lay = Layout.from_workload(WORKLOADS["16k"])
    for k, v in change.items():
        setattr(lay, k, v)
    cfg = lay.c()
    n = ctypes.c_int64()
    rc = native.load().spava_shard_layout(ctypes.byref(cfg), 0, world, None, ctypes.byref(n), None)
    assert rc == expect
    rc = native.load().spava_shard_layout(ctypes.byref(cfg), 5, 2, None, ctypes.byref(n), None)
    assert rc in (1, 2)


# ---------------------------------------------------------------- two gloo ranks
W = Workload("shard", H=4, Hq=4, Hkv=2, d=64, N=96 + 8 * 40 + 24, a=96, q=24, l=12, frame=16, seed=9)
NAN_BF16 = np.uint16(0x7FC0)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(w):
    return oracle.Problem(H=w.H, Hq=w.Hq, Hkv=w.Hkv, d=w.d, N=w.N, a=w.a, q=w.q,
                          offsets=chunk_offsets(w), l=w.l)


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W
        lay = Layout.from_workload(w)
        p = _problem(w)
        off = chunk_offsets(w)
        first, n_local, slots = shard_layout(lay, rank, world)
        pos = local_positions(lay, first)
        Q, K, V, _ = make_inputs(w)
        Qb, Kb, Vb = bf16_bits(Q), bf16_bits(K), bf16_bits(V)
        # What this rank holds: every other row is poisoned with NaN, so any
        # use of a row the rank does not hold shows up in the results.
        held = np.zeros(w.N, dtype=bool)
        held[pos] = True
        Qr, Kr, Vr = Qb.copy(), Kb.copy(), Vb.copy()
        Qr[~held], Kr[~held], Vr[~held] = NAN_BF16, NAN_BF16, NAN_BF16

        # (1) this rank's passing blocks, from its own rows only
        n_slots = len(slots)
        m_idx = np.full((n_slots, w.Hkv, w.l), -1, dtype=np.int32)
        m_k = np.zeros((n_slots, w.Hkv, w.l, w.d), dtype=np.int16)
        m_v = np.zeros_like(m_k)
        for s, u in enumerate(slots.tolist()):
            if u == 2 * w.H - 1:
                continue                                   # the last chunk passes nothing
            for g in range(w.Hkv):
                S = oracle.chunk_scores(p, Qr, Kr, int(u), g)
                assert np.isfinite(S).all()
                sel = oracle.select_top_l(S, int(off[u]), w.l)
                m_idx[s, g] = sel
                k = int((sel >= 0).sum())
                m_k[s, g, :k] = Kb[sel[:k], g].view(np.int16)
                m_v[s, g, :k] = Vb[sel[:k], g].view(np.int16)

        # (2) the exchange: fixed-size byte messages, gathered rank-major
        def gather(a):
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.uint8))
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t)
            return [x.numpy().view(a.dtype).reshape(a.shape) for x in parts]
        g_idx, g_k, g_v = gather(m_idx), gather(m_k), gather(m_v)

        # (3) unpack: full selection, and the received passing-block rows
        idx = np.full((2 * w.H - 1, w.Hkv, w.l), -3, dtype=np.int32)
        Kx, Vx = Kr.copy(), Vr.copy()
        for r2 in range(world):
            _, _, slots2 = shard_layout(lay, r2, world)
            for s, u in enumerate(slots2.tolist()):
                if u == 2 * w.H - 1:
                    continue
                idx[u] = g_idx[r2][s]
                for g in range(w.Hkv):
                    sel = g_idx[r2][s, g]
                    k = int((sel >= 0).sum())
                    Kx[sel[:k], g] = g_k[r2][s, g, :k].view(np.uint16)
                    Vx[sel[:k], g] = g_v[r2][s, g, :k].view(np.uint16)
        _, idx_ref = oracle.scores_and_select(p, Qb, Kb)
        same_idx = bool((idx == idx_ref).all())

        # (4) this rank's context rows from what it holds + what it received
        rows = np.concatenate([np.arange(off[v], off[v + 1]) for v in range(2 * w.H) if first[1 + v] >= 0])
        heads = list(range(w.Hq))
        O, lse = oracle.prefill_rows(p, Qr, Kx, Vx, idx, rows, heads)
        O_ref, lse_ref = oracle.prefill_rows(p, Qb, Kb, Vb, idx_ref, rows, heads)
        exact = bool(np.isfinite(O).all() and (O == O_ref).all() and (lse == lse_ref).all())

        # (5) query-row partial segments computed here: anchor and query block on
        # every rank, chunk v where it is held
        segs = [1 + v for v in range(2 * w.H) if first[1 + v] >= 0]
        all_segs = [None] * world
        dist.all_gather_object(all_segs, segs)
        out.put((rank, same_idx, exact, sorted(s for x in all_segs for s in x)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_what_their_rows_need():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=300)
    assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, same_idx, exact, segs in res:
        assert same_idx, f"rank {rank}: gathered selection differs from the oracle's"
        assert exact, f"rank {rank}: its rows need data it neither holds nor received"
        assert segs == list(range(1, 2 * W.H + 1))       # every chunk's partial exactly once


def test_shard_calls_reject_bad_arguments_before_any_launch():
    """Missing or misaligned pointers and a missing or misaligned workspace are
    refused by every shard call before anything is launched (no GPU needed)."""
    lay = Layout.from_workload(WORKLOADS["16k"])
    cfg = lay.c()
    lib = native.load()
    ws_b, _, _ = shard_sizes(lay, 2)
    good = 1 << 20          # an aligned, never dereferenced address
    odd = good + 8          # 16-byte misaligned
    ws = 1 << 24            # 256-byte aligned
    c = ctypes.byref(cfg)
    # front: q, k, v, pass_send, ws
    assert lib.spava_shard_front(c, 0, 2, None, good, good, good, ws, ws_b, None) == 1
    assert lib.spava_shard_front(c, 0, 2, good, good, good, odd, ws, ws_b, None) == 3
    assert lib.spava_shard_front(c, 0, 2, good, good, good, good, None, ws_b, None) == 4
    assert lib.spava_shard_front(c, 0, 2, good, good, good, good, ws + 16, ws_b, None) == 3
    assert lib.spava_shard_front(c, 0, 2, good, good, good, good, ws, ws_b - 256, None) == 4
    assert lib.spava_shard_front(c, 2, 2, good, good, good, good, ws, ws_b, None) == 1
    # local attention: o, lse (optional), part_send
    assert lib.spava_shard_local_attn(c, 1, 2, good, good, good, None, None, good, ws, ws_b, None) == 1
    assert lib.spava_shard_local_attn(c, 1, 2, good, good, good, good, odd, good, ws, ws_b, None) == 3
    # context attention: pass_all required, idx_out optional but aligned
    assert lib.spava_shard_context_attn(c, 0, 2, good, good, good, None, good, None, None, ws, ws_b, None) == 1
    assert lib.spava_shard_context_attn(c, 0, 2, good, good, good, good, good, None, odd, ws, ws_b, None) == 3
    # merge: part_all required
    assert lib.spava_shard_merge(c, 0, 2, None, good, None, ws, ws_b, None) == 1


def test_noalloc_status_rejects_a_missing_output():
    assert native.load().spava_score_noalloc_status(None, None) == 1
