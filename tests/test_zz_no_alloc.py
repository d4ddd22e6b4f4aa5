"""spava_score_noalloc: the scoring entry point for callers that cannot
allocate device memory (a plug-in handed only its input and output buffers, or
code that must not allocate after start-up).  Its scratch is a fixed array
inside the library instead of a caller workspace.

Called through the C ABI twice in a row, on two different layers.  Each result
must be bit-identical to spava_score with a workspace (the same kernels run in
the same order) and match the oracle's scores; the status word of the fixed
array must read clean after each call.  A third layer that does not fit the
fixed array must be refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity_util import SCORE_REL, problem
from sequence_sparse_attention_b200 import native
from sequence_sparse_attention_b200.api import Layout, Spava
from sequence_sparse_attention_b200.synth import Workload, bf16_bits, make_inputs

pytestmark = pytest.mark.gpu

FIRST = Workload("noalloc_a", H=2, Hq=14, Hkv=2, d=128, N=1500, a=100, q=150, l=100, frame=32, seed=21)
SECOND = Workload("noalloc_b", H=3, Hq=4, Hkv=2, d=64, N=2100, a=64, q=40, l=50, frame=32, seed=22)


def scores_noalloc(w, Q, K):
    lay = Layout.from_workload(w)
    cfg = lay.c()
    out = torch.full((w.Hkv, lay.context), float("nan"), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    lib = native.load()
    rc = lib.spava_score_noalloc(ctypes.byref(cfg), Q.data_ptr(), K.data_ptr(), out.data_ptr(), stream)
    assert rc == 0, native.STATUS_NAMES.get(rc, rc)
    flags = ctypes.c_int32(-1)
    rc = lib.spava_score_noalloc_status(stream, ctypes.byref(flags))
    assert rc == 0 and flags.value == 0, (rc, flags.value)
    return out


def scores_with_workspace(w, Q, K):
    sp = Spava(Layout.from_workload(w))
    out = torch.full((w.Hkv, sp.lay.context), float("nan"), dtype=torch.float32, device="cuda")
    sp.score(Q, K, out)
    assert sp.device_status() == 0
    return out


def test_noalloc_scores_match_workspace_scores_on_two_calls():
    for w in (FIRST, SECOND):
        Q, K, _, off = make_inputs(w)
        last0 = int(off[-2] - w.a)      # columns of the producing chunks
        got = scores_noalloc(w, Q.cuda(), K.cuda())[:, :last0].cpu().numpy()
        want = scores_with_workspace(w, Q.cuda(), K.cuda())[:, :last0].cpu().numpy()
        assert np.isfinite(got).all()
        np.testing.assert_array_equal(got, want)   # same kernels, same order: same bits
        ref, _ = oracle.scores_and_select(problem(w), bf16_bits(Q), bf16_bits(K))
        np.testing.assert_allclose(got, ref[:, :last0], rtol=SCORE_REL,
                                   atol=1e-7 * w.q * w.Hq / w.Hkv)


def test_noalloc_refuses_layers_beyond_the_fixed_scratch():
    # 4 * (2H-1) * Hq * q bytes of statistics: 4*63*64*512 = 8 MiB > 4 MiB.
    w = Workload("too_big", H=32, Hq=64, Hkv=8, d=128, N=64 * 4 + 512 + 8, a=8, q=512, l=4, frame=4)
    lay = Layout.from_workload(w)
    cfg = lay.c()
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    rc = native.load().spava_score_noalloc(ctypes.byref(cfg), dummy.data_ptr(), dummy.data_ptr(),
                                           dummy.data_ptr(), None)
    assert native.STATUS_NAMES[rc] == "SPAVA_ERR_WORKSPACE"
