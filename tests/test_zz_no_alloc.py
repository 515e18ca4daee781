"""svdq_act_amax_noalloc, the amax call for callers that cannot allocate device memory (an
engine or plugin whose device memory the host application plans up front, a real-time path
that must not enter the allocator): its scratch is a static array inside the library, so the
caller passes only the input and the 4-byte result word.

Checked through the C ABI against svdq_act_amax, which takes its scratch from the caller's
buffer: the same amax bit for bit on two calls in a row (a batch with a large value, then a
smaller batch, so a stale scratch from the first call would show in the second), and an empty
batch.  The amax is exact (bf16 x bf16 products in fp32, order-free maximum), so equality is
the tolerance.  This file is collected last so that a run stopping at its first failure has
run every other test before it.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def test_noalloc_amax_matches_the_caller_scratch_call_on_consecutive_calls(cuda_lib):
    L = cuda_lib.LIB
    K = 3072
    w = synth.svdq_workload(1024, K, 256)
    smooth = _bf16(w.smooth_inv)
    big = synth.to_bf16(w.X * 64.0)                       # first call: the larger amax
    small = synth.to_bf16(w.X[:300])                      # second call: smaller batch and amax
    ref_buf = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    seen = []
    for X in (big, small):
        Xd = _bf16(X)
        M = X.shape[0]
        assert L.svdq_act_amax(_p(Xd), _p(smooth), M, K, _p(ref_buf), _stream()) == 0
        out.fill_(-1.0)
        assert L.svdq_act_amax_noalloc(_p(Xd), _p(smooth), M, K, _p(out), _stream()) == 0
        torch.cuda.synchronize()
        got = int(out.view(torch.int32).item())
        assert got == int(ref_buf[0].item())
        seen.append(float(out.item()))
    assert seen[0] > seen[1] > 0.0
    # an empty batch writes 0
    out.fill_(-1.0)
    assert L.svdq_act_amax_noalloc(None, None, 0, K, _p(out), _stream()) == 0
    torch.cuda.synchronize()
    assert float(out.item()) == 0.0
    assert cuda_lib.svdq_device_status() == 0
