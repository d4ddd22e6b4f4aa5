"""The ZigZag sequence-parallel layer, its ranks emulated one after another on
one GPU: each rank gets only its local rows ([anchor | its chunks | query
block]), its exchange messages are gathered by device copies (what the NCCL
all-gather does across GPUs), and the assembled outputs must be BIT-identical
to the single-GPU layer entry point -- every kernel computes the same work
items from the same bytes, only the rows' home differs."""
import numpy as np
import pytest
import torch

from sequence_sparse_attention_b200.api import Layout, Spava, SpavaShard
from sequence_sparse_attention_b200.synth import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "base": Workload("base", H=4, Hq=8, Hkv=2, d=128, N=100 + 8 * 301 + 7 + 150, a=100, q=150, l=64,
                     frame=32, seed=31),
    "pure": Workload("pure", H=4, Hq=8, Hkv=2, d=128, N=100 + 8 * 301 + 7 + 150, a=100, q=150, l=64,
                     frame=32, seed=32, local_pair_full=0),
    "no_anchor_d64": Workload("no_anchor_d64", H=2, Hq=6, Hkv=3, d=64, N=4 * 260 + 90, a=0, q=90,
                              l=40, frame=32, seed=33),
    "no_passing": Workload("no_passing", H=4, Hq=4, Hkv=2, d=128, N=64 + 8 * 200 + 70, a=64, q=70,
                           l=0, frame=32, seed=34),
    "pooled": Workload("pooled", H=2, Hq=4, Hkv=2, d=64, N=40 + 4 * 290 + 70, a=40, q=70, l=50,
                       frame=32, seed=35, score_pool=5),
    "heavy_jitter": Workload("heavy_jitter", H=4, Hq=4, Hkv=1, d=128, N=80 + 64 * 40 + 60, a=80, q=60,
                             l=70, frame=64, jitter=0.1, heavy_frac=0.05, seed=36),
    "max_hosts": Workload("max_hosts", H=32, Hq=4, Hkv=2, d=64, N=64 + 64 * 41 + 40, a=64, q=40, l=16,
                          frame=16, seed=37),
}


def ws_status(sh: SpavaShard) -> int:
    torch.cuda.synchronize()
    return int(sh.ws[:4].view(torch.int32).item())


def run_emulated(w: Workload, world: int, Q, K, V):
    """Every rank's calls in order, the all-gathers done by device copies.
    Returns the full-size O, lse, idx assembled from the ranks' own rows, and
    every rank's local outputs."""
    lay = Layout.from_workload(w)
    shards = [SpavaShard(lay, r, world) for r in range(world)]
    loc = []
    for sh in shards:
        pos = torch.from_numpy(sh.positions).cuda()
        q, k, v = Q[pos].contiguous(), K[pos].contiguous(), V[pos].contiguous()
        o, lse = sh.new_outputs()
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        idx = torch.full((2 * w.H - 1, w.Hkv, w.l), -7, dtype=torch.int32, device="cuda")
        loc.append((q, k, v, o, lse, idx))
    for sh, (q, k, v, o, lse, idx) in zip(shards, loc):
        sh.front(q, k, v)
    gathered = torch.cat([sh.pass_send for sh in shards])
    for sh in shards:
        sh.pass_all.copy_(gathered)
    for sh, (q, k, v, o, lse, idx) in zip(shards, loc):
        sh.local_attn(q, k, v, o, lse)
    gathered = torch.cat([sh.part_send for sh in shards])
    for sh in shards:
        sh.part_all.copy_(gathered)
    for sh, (q, k, v, o, lse, idx) in zip(shards, loc):
        sh.context_attn(q, k, v, o, lse, idx)
    for sh, (q, k, v, o, lse, idx) in zip(shards, loc):
        sh.merge(o, lse)
    torch.cuda.synchronize()
    for sh in shards:
        assert ws_status(sh) == 0, "a kernel wait timed out"
    return shards, loc


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("name", list(CASES))
def test_sharded_layer_is_bit_identical(name, world):
    w = CASES[name]
    if w.H % world:
        pytest.skip("world does not divide H")
    Q, K, V, _ = make_inputs(w, "cuda")
    O_ref, lse_ref, idx_ref = Spava(Layout.from_workload(w)).prefill_attention(Q, K, V, want_idx=True)
    shards, loc = run_emulated(w, world, Q, K, V)
    O_ref16 = O_ref.view(torch.int16)
    for sh, (q, k, v, o, lse, idx) in zip(shards, loc):
        pos = torch.from_numpy(sh.positions).cuda()
        # every local row: own chunks, and the anchor and query rows every rank computes
        assert torch.equal(o.view(torch.int16), O_ref16[pos]), f"rank {sh.rank}: O differs"
        assert torch.equal(lse, lse_ref[:, pos]), f"rank {sh.rank}: lse differs"
        if w.l > 0:
            assert torch.equal(idx, idx_ref), f"rank {sh.rank}: passing-block indices differ"


def test_sharded_16k_layer_four_ranks():
    """The 16K layer of the study (H = 4) as four ranks, one physical host each."""
    w = WORKLOADS["16k"]
    Q, K, V, _ = make_inputs(w, "cuda")
    O_ref, lse_ref, idx_ref = Spava(Layout.from_workload(w)).prefill_attention(Q, K, V, want_idx=True)
    shards, loc = run_emulated(w, 4, Q, K, V)
    covered = torch.zeros(w.N, dtype=torch.bool, device="cuda")
    for sh, (q, k, v, o, lse, idx) in zip(shards, loc):
        pos = torch.from_numpy(sh.positions).cuda()
        assert torch.equal(o.view(torch.int16), O_ref.view(torch.int16)[pos])
        assert torch.equal(lse, lse_ref[:, pos])
        assert torch.equal(idx, idx_ref)
        covered[pos] = True
    assert bool(covered.all())


def test_one_rank_layer_with_a_comm_stream():
    """SpavaShard.layer on one rank (the all-gather is a copy) with the
    exchanges on a second stream: same bytes as the layer entry point."""
    w = CASES["base"]
    Q, K, V, _ = make_inputs(w, "cuda")
    O_ref, lse_ref, _ = Spava(Layout.from_workload(w)).prefill_attention(Q, K, V)
    sh = SpavaShard(Layout.from_workload(w), 0, 1)
    o, lse = sh.new_outputs()
    cs = torch.cuda.Stream()
    for _ in range(2):
        sh.layer(Q, K, V, o, lse, lambda out, inp: out.copy_(inp), comm_stream=cs)
    torch.cuda.synchronize()
    assert ws_status(sh) == 0
    assert torch.equal(o.view(torch.int16), O_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)
