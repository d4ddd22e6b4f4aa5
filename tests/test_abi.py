"""The C-ABI library on the host: it loads without a GPU, exports every entry
point include/spava.h declares, rejects bad arguments before touching the
device, and its work plan attends exactly the oracle's key sets."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from sequence_sparse_attention_b200 import native
from sequence_sparse_attention_b200.api import Layout, attended_pairs, packed_len, workspace_size
from sequence_sparse_attention_b200.synth import WORKLOADS, Workload, chunk_offsets

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "spava.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spava_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = native.load()
    declared = header_functions()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(native.EXPORTS)


def test_status_strings():
    lib = native.load()
    for s in range(7):
        assert lib.spava_status_string(s)
    assert lib.spava_status_string(0) == b"ok"


def lay_of(w, **kw):
    lay = Layout.from_workload(w)
    for k, v in kw.items():
        setattr(lay, k, v)
    return lay


def status(fn, lay, *args):
    cfg = lay.c()
    return getattr(native.load(), fn)(ctypes.byref(cfg), *args)


@pytest.mark.parametrize("change,expect", [
    (dict(Hq=5), 1),                      # Hq not a multiple of Hkv
    (dict(d=96), 2),                      # head dim not built
    (dict(H=40), 2),                      # more chunks than the plan holds
    (dict(q=0), 1),
    (dict(l=-1), 1),
    (dict(local_pair_full=2), 1),
    (dict(score_norm=2), 1),              # selection variants: unknown normalisation
    (dict(score_pool=4), 1),              # even window
    (dict(score_pool=-3), 1),
    (dict(score_pool=257), 2),            # wider than the kernel offers
])
def test_bad_config_rejected(change, expect):
    w = WORKLOADS["tiny"]
    lay = lay_of(w, **change)
    n = ctypes.c_size_t()
    assert status("spava_workspace_size", lay, ctypes.byref(n)) == expect


def test_bad_offsets_rejected():
    w = WORKLOADS["tiny"]
    for k in range(3):
        off = chunk_offsets(w).copy()
        if k == 0:
            off[0] += 1
        elif k == 1:
            off[-1] -= 1
        else:
            off[2] = off[1]
        lay = lay_of(w, offsets=off)
        n = ctypes.c_size_t()
        assert status("spava_workspace_size", lay, ctypes.byref(n)) == 1


def test_pointer_and_workspace_checks_before_launch():
    """Null / misaligned pointers and short workspaces fail before any CUDA call,
    so these statuses come back even without a GPU."""
    lay = Layout.from_workload(WORKLOADS["tiny"])
    ws_bytes = workspace_size(lay)
    buf = ctypes.create_string_buffer(ws_bytes + 512)
    base = (ctypes.addressof(buf) + 255) // 256 * 256
    fake = base  # aligned address never dereferenced on these paths
    # null required pointer
    assert status("spava_attn", lay, None, fake, fake, fake, fake, fake, None, base, ws_bytes, None) == 1
    # misaligned q
    assert status("spava_attn", lay, fake + 2, fake, fake, fake, fake, fake, None, base, ws_bytes, None) == 3
    # workspace too small / missing / misaligned
    assert status("spava_attn", lay, fake, fake, fake, fake, fake, fake, None, base, ws_bytes - 1, None) == 4
    assert status("spava_attn", lay, fake, fake, fake, fake, fake, fake, None, None, ws_bytes, None) == 4
    assert status("spava_attn", lay, fake, fake, fake, fake, fake, fake, None, base + 16, ws_bytes, None) == 3
    assert status("spava_prefill_attention", lay, fake, fake, None, fake, None, None, base, ws_bytes, None) == 1
    assert status("spava_score", lay, fake, fake, fake, base, 16, None) == 4
    # selection and gather: missing scores, misaligned indices, misaligned packed rows
    assert status("spava_topk_select", lay, None, fake, None) == 1
    assert status("spava_topk_select", lay, fake, fake + 4, None) == 3
    assert status("spava_pack_passing", lay, fake, fake, fake, fake + 8, fake, None) == 3
    assert status("spava_pack_passing", lay, fake, None, fake, fake, fake, None) == 1
    # host-buffer entry point: host and device pointers, then the workspace, all
    # checked before the first copy or stream is made
    host = fake  # any non-null host address; never read on these paths
    args = [host, host, host, host, None, fake, fake, fake, fake, None, base, ws_bytes, None, None]
    bad = list(args); bad[1] = None                      # k_host missing
    assert status("spava_prefill_attention_host", lay, *bad) == 1
    bad = list(args); bad[5] = fake + 2                  # q misaligned
    assert status("spava_prefill_attention_host", lay, *bad) == 3
    bad = list(args); bad[11] = ws_bytes - 1             # workspace short
    assert status("spava_prefill_attention_host", lay, *bad) == 4
    bad = list(args); bad[10] = None                     # workspace missing
    assert status("spava_prefill_attention_host", lay, *bad) == 4


def test_workspace_and_packed_sizes():
    for name, w in WORKLOADS.items():
        lay = Layout.from_workload(w)
        off = chunk_offsets(w)
        L = w.a + sum(min(w.l, int(off[u + 1] - off[u])) for u in range(2 * w.H - 1))
        assert packed_len(lay) == L
        assert workspace_size(lay) >= 2 * w.Hkv * L * w.d * 2


def _oracle_pair_counts(w, lpf):
    p = oracle.Problem(H=w.H, Hq=w.Hq, Hkv=w.Hkv, d=w.d, N=w.N, a=w.a, q=w.q,
                       offsets=chunk_offsets(w), l=w.l, local_pair_full=lpf)
    off = chunk_offsets(w)
    idx = np.full((2 * w.H - 1, w.Hkv, w.l), -1, dtype=np.int32)
    for u in range(2 * w.H - 1):
        n = int(off[u + 1] - off[u])
        k = min(w.l, n)
        idx[u, :, :k] = off[u] + np.arange(k)
    anchor = sum(len(oracle.key_set(p, idx, t, 0)) for t in range(w.a))
    ctx = sum(len(oracle.key_set(p, idx, t, 0)) for t in range(w.a, w.N - w.q))
    query = sum(len(oracle.key_set(p, idx, t, 0)) for t in range(w.N - w.q, w.N))
    host = [0] * w.H
    for v in range(2 * w.H):
        host[oracle.pair(w.H, v)] += sum(len(oracle.key_set(p, idx, t, 0))
                                         for t in range(off[v], off[v + 1]))
    return (anchor, ctx, query), host


@pytest.mark.parametrize("w", [
    Workload("a", H=2, Hq=4, Hkv=2, d=64, N=700, a=40, q=30, l=50, frame=16),
    Workload("b", H=3, Hq=6, Hkv=3, d=128, N=900, a=0, q=200, l=17, frame=16),
    Workload("c", H=1, Hq=2, Hkv=1, d=64, N=500, a=130, q=131, l=1000, frame=16),
    Workload("d", H=4, Hq=4, Hkv=1, d=64, N=1600, a=300, q=5, l=0, frame=16),
    Workload("e", H=3, Hq=4, Hkv=2, d=64, N=48 * 64 + 100, a=64, q=36, l=40, frame=64, jitter=0.1),
])
@pytest.mark.parametrize("lpf", [1, 0])
def test_plan_attends_exactly_the_oracle_key_sets(w, lpf):
    """Integer, exact: the segment plan of the kernels covers the same number of
    (row, key) pairs per class and per physical host as the oracle's key sets."""
    lay = lay_of(w, local_pair_full=lpf)
    pairs, host = attended_pairs(lay)
    o_pairs, o_host = _oracle_pair_counts(w, lpf)
    assert tuple(pairs) == o_pairs
    assert list(host) == o_host


def test_zigzag_host_balance_on_equal_chunks():
    """Bilanciamento del Carico dell'Attenzione Approssimata: equal chunks ->
    every physical host attends the same number of context pairs."""
    for name in ("16k", "64k", "128k"):
        _, host = attended_pairs(Layout.from_workload(WORKLOADS[name]))
        assert len(set(host)) == 1, (name, host)


def test_variant_configs_accepted_and_noalloc_refuses_row_norm():
    """The selection variants are valid configurations; the allocation-free
    scoring entry (whose fixed scratch holds per-chunk statistics only) refuses
    the row-normalised one before any CUDA call."""
    w = WORKLOADS["tiny"]
    for kw in (dict(score_norm=1), dict(score_pool=1), dict(score_pool=5), dict(score_norm=1, score_pool=255)):
        n = ctypes.c_size_t()
        assert status("spava_workspace_size", lay_of(w, **kw), ctypes.byref(n)) == 0
    buf = ctypes.create_string_buffer(4096)
    fake = (ctypes.addressof(buf) + 255) // 256 * 256
    assert status("spava_score_noalloc", lay_of(w, score_norm=1), fake, fake, fake, None) == 2


def test_plan_chunks_matches_the_oracle():
    """Visual load balancing: the library's chunk offsets equal the oracle's
    (whole consecutive frames dealt evenly over the 2H virtual hosts) on random
    frame lists, and form a valid layer."""
    from sequence_sparse_attention_b200.api import plan_chunks
    rng = np.random.default_rng(5)
    for H, n_frames in ((1, 2), (2, 9), (4, 64), (8, 1006), (3, 37), (16, 1024), (32, 64)):
        for trial in range(3):
            ft = rng.integers(1 if trial == 0 else 100, 300, n_frames)
            a = int(rng.integers(0, 2000))
            off = plan_chunks(H, ft, a)
            np.testing.assert_array_equal(off, oracle.plan_chunks(H, ft, a))
            lay = Layout(H, 4, 2, 64, int(off[-1]) + 16, a, 16, off, 8)
            n = ctypes.c_size_t()
            assert status("spava_workspace_size", lay, ctypes.byref(n)) == 0


def test_plan_chunks_equal_frames_divide_evenly():
    """Equal frames whose count divides by 2H: every chunk gets the same number
    of whole frames."""
    from sequence_sparse_attention_b200.api import plan_chunks
    off = plan_chunks(4, [256] * 64, 1024)
    np.testing.assert_array_equal(off, 1024 + 256 * 8 * np.arange(9))


@pytest.mark.parametrize("args", [
    (0, [5, 5], 0), (33, [1] * 66, 0),    # H out of range
    (2, [5, 5, 5], 0),                    # fewer frames than chunks
    (1, [5, 0], 0),                       # a frame without tokens
    (1, [5, 5], -1),                      # negative anchor
    (1, [2 ** 30, 2 ** 30], 0),           # past 2^31 tokens
])
def test_plan_chunks_rejects(args):
    from sequence_sparse_attention_b200.api import plan_chunks
    from sequence_sparse_attention_b200.native import SpavaError
    with pytest.raises(SpavaError):
        plan_chunks(*args)
