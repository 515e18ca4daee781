"""Failure detection on the GPU without a fault: a bounded wait made to run out.

Every mbarrier wait of the kernels gives up after about one second, records SVDQ_ERR_TIMEOUT
in a device status word and lets the kernel return.  svdq_selftest_wait_timeout runs that wait
code on a barrier at which nothing arrives (no copy or MMA in flight); the status must read 5,
clear, and the context must stay usable for a normal layer call afterwards on the same stream.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import svdq
from parity_util import check_output

pytestmark = pytest.mark.gpu


def test_a_bounded_wait_that_runs_out_reports_timeout_and_leaves_the_context_usable(cuda_lib):
    P = cuda_lib
    assert P.svdq_device_status(clear=True) == 0
    stream = torch.cuda.current_stream()
    assert P.LIB.svdq_selftest_wait_timeout(ctypes.c_void_p(stream.cuda_stream)) == 0
    torch.cuda.synchronize()                      # returns: the wait gave up instead of hanging
    assert P.svdq_device_status(clear=False) == 5
    assert P.svdq_device_status(clear=True) == 5  # read, then cleared
    assert P.svdq_device_status() == 0
    # a layer call on the same stream afterwards is unaffected
    w = synth.svdq_workload(256, 512, 512)
    layer = P.SvdqW4A4Linear(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2), synth.bf16_bits(w.bias),
                             synth.bf16_bits(w.smooth_inv), w.g_a, device="cuda")
    X = torch.from_numpy(w.X).to(torch.bfloat16).cuda()
    Y = layer(X)
    torch.cuda.synchronize()
    check_output(Y.float().cpu().numpy(), svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a))
    assert P.svdq_device_status() == 0
