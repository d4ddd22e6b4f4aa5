"""GPU parity of every step of the path against the fp64 oracle, element by
element, on sizes the oracle finishes in seconds that still span several 128
tiles and ragged tails (chunk, anchor and query lengths not multiples of 128,
GQA groups of 2 and 7, d = 64 and 128, uneven chunks, a = 0, one host, full
passing blocks, local_pair_full = 0)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from parity_util import (LSE_ABS, SCORE_REL, OracleRun, check_outputs, check_selection,
                         expected_rows, to_np)
from sequence_sparse_attention_b200.api import Layout, Spava, plan_chunks
from sequence_sparse_attention_b200.synth import (WORKLOADS, Workload, chunk_offsets, make_inputs,
                                                  uneven_frames)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],
    "g7": Workload("g7", H=2, Hq=14, Hkv=2, d=128, N=1500, a=100, q=150, l=100, frame=32, seed=11),
    "g7_pure": Workload("g7_pure", H=2, Hq=14, Hkv=2, d=128, N=1500, a=100, q=150, l=100, frame=32,
                        seed=11, local_pair_full=0),
    "no_anchor": Workload("no_anchor", H=3, Hq=8, Hkv=4, d=128, N=1300, a=0, q=64, l=64, frame=32,
                          seed=12),
    "one_host": Workload("one_host", H=1, Hq=4, Hkv=2, d=128, N=1000, a=64, q=40, l=30, frame=32,
                         seed=13),
    "full_l": Workload("full_l", H=3, Hq=4, Hkv=1, d=64, N=1200, a=200, q=130, l=100000, frame=32,
                       seed=14),
    "jitter_heavy": Workload("jitter_heavy", H=3, Hq=6, Hkv=2, d=64, N=64 * 30 + 70 + 90, a=70, q=90,
                             l=45, frame=64, jitter=0.1, heavy_frac=0.05, seed=15),
    "long_anchor": Workload("long_anchor", H=2, Hq=4, Hkv=4, d=128, N=1800, a=300, q=257, l=160,
                            frame=32, seed=16),
    # no passing blocks at all: anchor + partner + own chunk only
    "no_passing": Workload("no_passing", H=3, Hq=6, Hkv=2, d=128, N=1400, a=96, q=70, l=0,
                           frame=32, seed=17),
    # no anchor and no passing blocks: zero packed rows
    "empty_packed": Workload("empty_packed", H=2, Hq=4, Hkv=2, d=64, N=900, a=0, q=40, l=0,
                             frame=32, seed=18),
    # chunks shorter than one 128-row tile
    "short_chunks": Workload("short_chunks", H=4, Hq=4, Hkv=2, d=128, N=600, a=30, q=20, l=20,
                             frame=16, seed=19),
    # multi-head (G = 1) and a wide GQA group (G = 16)
    "mha": Workload("mha", H=2, Hq=3, Hkv=3, d=64, N=1100, a=50, q=60, l=40, frame=32, seed=20),
    "wide_group": Workload("wide_group", H=2, Hq=16, Hkv=1, d=128, N=1000, a=64, q=130, l=64,
                           frame=32, seed=21),
    # selection variants: row-normalised scores, pooled ranking, both
    "rownorm": Workload("rownorm", H=3, Hq=6, Hkv=2, d=128, N=1500, a=80, q=150, l=60, frame=32,
                        seed=22, score_norm=1),
    "pooled": Workload("pooled", H=2, Hq=4, Hkv=2, d=64, N=1200, a=40, q=70, l=50, frame=32,
                       seed=23, score_pool=5),
    "rownorm_pooled": Workload("rownorm_pooled", H=2, Hq=8, Hkv=2, d=128, N=1300, a=0, q=90, l=40,
                               frame=32, seed=24, score_norm=1, score_pool=7),
    # sixteen chunks shorter than one row tile, and the pure-virtual pairing on d = 64
    "many_hosts": Workload("many_hosts", H=8, Hq=6, Hkv=2, d=128, N=2150, a=100, q=60, l=30,
                           frame=16, seed=25),
    "pure_d64": Workload("pure_d64", H=3, Hq=4, Hkv=1, d=64, N=1400, a=50, q=100, l=70, frame=32,
                         seed=26, local_pair_full=0),
    "variants_d64": Workload("variants_d64", H=3, Hq=6, Hkv=3, d=64, N=1500, a=64, q=140, l=50,
                             frame=32, seed=27, score_norm=1, score_pool=3),
    # the most hosts the library takes (H = 32: 64 chunks, a full 64-bit host mask)
    "max_hosts": Workload("max_hosts", H=32, Hq=4, Hkv=2, d=64, N=64 + 64 * 41 + 40, a=64, q=40, l=16,
                          frame=16, seed=29),
    # the smallest query block and anchor: one row each
    "one_row_query": Workload("one_row_query", H=2, Hq=4, Hkv=2, d=128, N=1 + 4 * 200 + 1, a=1, q=1,
                              l=50, frame=16, seed=30),
}



def visual_balance_case() -> Workload:
    """A layer whose chunks come from the library's visual load balancer
    (spava_plan_chunks) on 29 frames of uneven token counts (40..80): whole
    frames dealt evenly over the 6 virtual hosts, so the chunks' token counts
    differ.  The oracle's own planner must give the same offsets."""
    H, a, q = 3, 70, 90
    ft = uneven_frames(29, 40, 81, seed=28)
    off = plan_chunks(H, ft, a)
    assert np.array_equal(off, oracle.plan_chunks(H, ft, a))
    return Workload("visual_balance", H=H, Hq=6, Hkv=2, d=128, N=int(off[-1]) + q, a=a, q=q, l=48,
                    seed=28, frame_tokens=ft, offsets=tuple(int(x) for x in off))


CASES["visual_balance"] = visual_balance_case()

_cache = {}


def setup_case(name):
    if name not in _cache:
        w = CASES[name]
        Q, K, V, off = make_inputs(w)          # CPU generator, copied to the GPU below
        ref = OracleRun(w, Q, K, V)
        rows = np.arange(w.N)
        O_ref, lse_ref = ref.rows(rows, list(range(w.Hq)))
        _cache[name] = (w, Q, K, V, ref, O_ref, lse_ref)
    return _cache[name]


def device_clean(sp: Spava):
    assert sp.device_status() == 0, "a kernel wait timed out"


@pytest.mark.parametrize("name", list(CASES))
def test_scores(name):
    w, Q, K, V, ref, _, _ = setup_case(name)
    sp = Spava(Layout.from_workload(w))
    scores = to_np(sp.score(Q.cuda(), K.cuda()))
    device_clean(sp)
    off = chunk_offsets(w)
    G = w.Hq // w.Hkv
    last0 = int(off[-2] - w.a)          # the last chunk produces no passing block
    want = ref.scores[:, :last0]
    got = scores[:, :last0]
    np.testing.assert_allclose(got, want, rtol=SCORE_REL, atol=1e-7 * G * w.q)
    if w.score_norm == 0:
        for u in range(2 * w.H - 1):    # closed form: each chunk's scores sum to G*q
            s0, s1 = int(off[u] - w.a), int(off[u + 1] - w.a)
            np.testing.assert_allclose(got[:, s0:s1].sum(axis=1), G * w.q, rtol=1e-4)


@pytest.mark.parametrize("name", list(CASES))
def test_topk_bit_exact_on_fp32_scores(name):
    """Selection from the same fp32 scores: index sets bit-exact (ties to the
    lower index), against the oracle's sort run on those fp32 values."""
    w, Q, K, V, ref, _, _ = setup_case(name)
    sp = Spava(Layout.from_workload(w))
    off = chunk_offsets(w)
    s32 = ref.scores.astype(np.float32)
    # plant exact ties across a chunk so the tie rule decides
    s32[:, 5:40] = s32[:, 3:4]
    idx = to_np(sp.topk_select(torch.from_numpy(s32).cuda())).astype(np.int32)
    for u in range(2 * w.H - 1):
        s0 = int(off[u] - w.a)
        n = int(off[u + 1] - off[u])
        for g in range(w.Hkv):
            ranked = s32[g, s0:s0 + n]
            if w.score_pool > 1:            # window sums in the kernel's fp32 order
                ranked = oracle.pool_sums(ranked, w.score_pool)
            want = oracle.select_top_l(ranked.astype(np.float64), int(off[u]), w.l)
            np.testing.assert_array_equal(idx[u, g], want, err_msg=f"{name} u={u} g={g}")


@pytest.mark.parametrize("name", ["tiny", "g7", "no_anchor", "long_anchor", "short_chunks"])
def test_pack_exact(name):
    w, Q, K, V, ref, _, _ = setup_case(name)
    sp = Spava(Layout.from_workload(w))
    Kd, Vd = K.cuda(), V.cuda()
    idx = torch.from_numpy(ref.idx).cuda()
    pk, pv = sp.pack_passing(Kd, Vd, idx)
    torch.cuda.synchronize()
    off = chunk_offsets(w)
    for g in range(w.Hkv):
        rows = list(range(w.a))
        for u in range(2 * w.H - 1):
            k = min(w.l, int(off[u + 1] - off[u]))
            rows += ref.idx[u, g, :k].tolist()
        r = torch.tensor(rows, dtype=torch.long)
        assert torch.equal(pk[g].cpu().view(torch.int16), K[r, g].view(torch.int16))
        assert torch.equal(pv[g].cpu().view(torch.int16), V[r, g].view(torch.int16))


@pytest.mark.parametrize("name", list(CASES))
def test_attn_given_oracle_selection(name):
    """spava_attn on passing blocks packed from the oracle's own selection:
    every row and head against the oracle."""
    w, Q, K, V, ref, O_ref, lse_ref = setup_case(name)
    sp = Spava(Layout.from_workload(w))
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    pk, pv = sp.pack_passing(Kd, Vd, torch.from_numpy(ref.idx).cuda())
    O, lse = sp.attn(Qd, Kd, Vd, pk, pv)
    device_clean(sp)
    check_outputs(to_np(O), O_ref, name)
    np.testing.assert_allclose(to_np(lse).T, lse_ref, atol=LSE_ABS, rtol=0)


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_end_to_end(name):
    """The whole layer entry point.  The selection must be a correct top-l of
    the oracle's scores (bit-exact outside the tie band); then EVERY row and
    head is compared with the oracle's attention over the key sets of that
    selection -- no output is exempt."""
    w, Q, K, V, ref, O_ref, lse_ref = setup_case(name)
    sp = Spava(Layout.from_workload(w))
    O, lse, idx = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda(), want_idx=True)
    device_clean(sp)
    idx_h = idx.cpu().numpy()
    rep = check_selection(w, ref.scores, idx_h, range(w.Hkv), ref.idx)
    heads = list(range(w.Hq))
    O_want, lse_want = expected_rows(ref, idx_h, np.arange(w.N), heads, cached=(O_ref, lse_ref))
    mx, mean = check_outputs(to_np(O), O_want, name)
    np.testing.assert_allclose(to_np(lse).T, lse_want, atol=LSE_ABS, rtol=0)
    print(f"{name}: selections exact {rep['exact']}, in band {rep['band']} "
          f"(keys in band {rep['band_keys']}), differing from the oracle's {rep['differ']}; "
          f"O max-abs {mx:.2e} mean-abs {mean:.2e}")


def test_values_one_give_ones():
    """V = 1 everywhere: every softmax-weighted average is exactly one up to
    the bf16 rounding of P."""
    w = CASES["g7"]
    Q, K, V, _ = make_inputs(w)
    V = torch.ones_like(V)
    sp = Spava(Layout.from_workload(w))
    O, _, _ = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda())
    device_clean(sp)
    err = (O.float() - 1).abs()
    assert err.max().item() < 1e-2 and err.mean().item() < 2e-3


def test_repeat_calls_bit_identical():
    w = CASES["g7"]
    Q, K, V, _ = make_inputs(w)
    sp = Spava(Layout.from_workload(w))
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    O1, l1, i1 = sp.prefill_attention(Qd, Kd, Vd, want_idx=True)
    O2, l2, i2 = sp.prefill_attention(Qd, Kd, Vd, want_idx=True)
    device_clean(sp)
    assert torch.equal(i1, i2)
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16))
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("name", ["tiny", "g7", "no_anchor", "long_anchor", "short_chunks",
                                  "one_host", "many_hosts", "rownorm_pooled"])
@pytest.mark.parametrize("pipelined", [False, True])
def test_host_buffers_entry_point(name, pipelined):
    """Host buffers in and out, on one stream or with the copies on a second
    stream overlapping the kernels group by group: bit-identical to the
    device-buffer entry point."""
    w = CASES[name]
    Q, K, V, _ = make_inputs(w)
    sp = Spava(Layout.from_workload(w))
    qh, kh, vh = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    oh = torch.full_like(Q, 7.0).pin_memory()
    lh = torch.full((w.Hq, w.N), 7.0, dtype=torch.float32).pin_memory()
    # device buffers start as NaN: a kernel that read a row before its upload
    # landed would show it
    qd, kd, vd = (torch.full_like(x, float("nan"), device="cuda") for x in (Q, K, V))
    od = torch.full_like(qd, float("nan"))
    ld = torch.empty((w.Hq, w.N), dtype=torch.float32, device="cuda")
    cs = torch.cuda.Stream() if pipelined else None
    sp.prefill_attention_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, copy_stream=cs)
    torch.cuda.current_stream().synchronize()   # the call's work ends on this stream
    oh_c, lh_c = oh.clone(), lh.clone()
    torch.cuda.synchronize()
    device_clean(sp)
    O_dev, lse_dev, _ = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda())
    assert torch.equal(oh_c.view(torch.int16), O_dev.cpu().view(torch.int16))
    assert torch.equal(lh_c, lse_dev.cpu())


def test_host_buffers_back_to_back():
    """Two pipelined host calls in a row on the same device buffers with
    different inputs: the second call's uploads must wait for the first call's
    kernels, so each host output matches the device path for its own inputs."""
    w = WORKLOADS["16k"]
    ins = [make_inputs(w), make_inputs(dataclasses.replace(w, seed=w.seed + 100))]
    sp = Spava(Layout.from_workload(w))
    qd = torch.full(ins[0][0].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    kd = torch.full(ins[0][1].shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    vd = torch.full_like(kd, float("nan"))
    od = torch.full_like(qd, float("nan"))
    cs = torch.cuda.Stream()
    outs = []
    hosts = []
    for Q, K, V, _ in ins:
        hosts.append((Q.pin_memory(), K.pin_memory(), V.pin_memory(), torch.empty_like(Q).pin_memory()))
    for qh, kh, vh, oh in hosts:
        sp.prefill_attention_host(qh, kh, vh, oh, None, qd, kd, vd, od, None, copy_stream=cs)
    torch.cuda.synchronize()
    device_clean(sp)
    for (Q, K, V, _), (_, _, _, oh) in zip(ins, hosts):
        O_dev, _, _ = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda())
        assert torch.equal(oh.view(torch.int16), O_dev.cpu().view(torch.int16))


def test_host_buffers_on_a_caller_stream():
    """The caller computes on its own (non-default) stream: the pipelined host
    call ends on that stream, so synchronising it alone is enough to read the
    host outputs, which equal the device entry point's bytes."""
    w = CASES["g7"]
    Q, K, V, _ = make_inputs(w)
    sp = Spava(Layout.from_workload(w))
    qh, kh, vh = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    oh = torch.full_like(Q, 7.0).pin_memory()
    lh = torch.full((w.Hq, w.N), 7.0, dtype=torch.float32).pin_memory()
    qd, kd, vd = (torch.full_like(x, float("nan"), device="cuda") for x in (Q, K, V))
    od = torch.full_like(qd, float("nan"))
    ld = torch.empty((w.Hq, w.N), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    compute, copies = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(compute):
        for _ in range(2):
            sp.prefill_attention_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, copy_stream=copies)
    compute.synchronize()
    oh_c, lh_c = oh.clone(), lh.clone()
    torch.cuda.synchronize()
    device_clean(sp)
    O_dev, lse_dev, _ = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda())
    assert torch.equal(oh_c.view(torch.int16), O_dev.cpu().view(torch.int16))
    assert torch.equal(lh_c, lse_dev.cpu())
