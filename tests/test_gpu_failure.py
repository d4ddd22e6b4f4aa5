"""Failure detection on the GPU without a GPU fault: a kernel wait that can
never complete gives up after its bound, the status word reports it, and the
context stays usable for the next layer."""
import ctypes

import numpy as np
import pytest
import torch

from sequence_sparse_attention_b200 import native
from sequence_sparse_attention_b200.api import Layout, Spava
from sequence_sparse_attention_b200.synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    w = WORKLOADS["tiny"]
    sp = Spava(Layout.from_workload(w))
    assert sp.device_status() == 0
    lib = native.load()
    rc = lib.spava_selftest_wait_timeout(sp.ws.data_ptr(), sp.ws.numel(),
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    flags = ctypes.c_int32()
    rc = lib.spava_device_status(sp.ws.data_ptr(), sp.ws.numel(),
                                 torch.cuda.current_stream().cuda_stream, ctypes.byref(flags))
    assert native.STATUS_NAMES[rc] == "SPAVA_ERR_TIMEOUT" and flags.value & 1
    assert sp.device_status() == 0          # the bit was cleared
    # the context is intact: a full layer still runs and is deterministic
    Q, K, V, _ = make_inputs(w)
    O1, _, _ = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda())
    O2, _, _ = sp.prefill_attention(Q.cuda(), K.cuda(), V.cuda())
    torch.cuda.synchronize()
    assert sp.device_status() == 0
    assert torch.equal(O1.view(torch.int16), O2.view(torch.int16))
    assert torch.isfinite(O1.float()).all()
