"""The torch.library operators and nn.Module layers on the GPU: the same results as the
direct calls (bit for bit), the oracle's parity bar, torch.compile(fullgraph=True), and
torch.library's own consistency checks of the fake implementations."""

import numpy as np
import pytest
import torch

import synth
from oracle import awq as oawq
from oracle import svdq
from parity_util import check_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P(cuda_lib):
    return cuda_lib


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def svdq_layer(P):
    w = synth.svdq_workload(256, 512, 512)
    layer = P.SvdqLinear.from_exported(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2), synth.bf16_bits(w.bias),
                                       synth.bf16_bits(w.smooth_inv), w.g_a)
    return w, layer


def test_svdq_layer_matches_direct_calls_and_oracle(P, svdq_layer):
    w, layer = svdq_layer
    X = _bf(w.X)
    Y = layer(X.reshape(2, 128, 512))
    assert Y.shape == (2, 128, 512)
    old = P.SvdqW4A4Linear(w.R, synth.bf16_bits(w.L1), synth.bf16_bits(w.L2), synth.bf16_bits(w.bias),
                           synth.bf16_bits(w.smooth_inv), w.g_a)
    assert torch.equal(Y.reshape(256, 512), old(X))
    y_ref = svdq.forward(w.X, w.smooth_inv, w.R, w.L1, w.L2, w.bias, w.g_a)
    check_output(Y.reshape(256, 512).float().cpu().numpy(), y_ref)


def test_svdq_layer_under_compile_fullgraph(svdq_layer):
    w, layer = svdq_layer
    X = _bf(w.X)
    compiled = torch.compile(layer, fullgraph=True, backend="aot_eager")
    assert torch.equal(compiled(X), layer(X))


@pytest.mark.parametrize("M", [8, 24])
def test_awq_layer_matches_direct_calls_and_oracle(P, M):
    a = synth.awq_workload(M, 1024, 384)
    bias = synth.to_bf16(np.random.default_rng(5).standard_normal(384) * 0.1)
    layer = P.AwqLinear(torch.from_numpy(a.qweight).cuda(), _bf(a.scales), _bf(a.zeros), _bf(bias))
    X = _bf(a.X)
    Y = layer(X.reshape(1, M, 1024))
    assert torch.equal(Y.reshape(M, 384), P.awq_w4a16_linear(X, layer.qweight, layer.scales, layer.zeros, layer.bias))
    check_output(Y.reshape(M, 384).float().cpu().numpy(), oawq.forward(a.X, a.q, a.scales, a.zeros, bias))
    compiled = torch.compile(layer, fullgraph=True, backend="aot_eager")
    assert torch.equal(compiled(X), Y.reshape(M, 384))


def test_opcheck_fake_implementations(P, svdq_layer):
    w, layer = svdq_layer
    X = _bf(w.X[:130])
    torch.library.opcheck(torch.ops.svdq.quantize_act_lowrank_down.default,
                          (X, layer.smooth_inv, layer.packed_w, layer.act_global_scale, 32))
    codes, scales, low = torch.ops.svdq.quantize_act_lowrank_down(X, layer.smooth_inv, layer.packed_w,
                                                                  layer.act_global_scale, 32)
    torch.library.opcheck(torch.ops.svdq.w4a4_nvfp4_linear.default,
                          (codes, scales, low, layer.act_global_scale, layer.packed_w, layer.w_global_scale, 512, 32))
    a = synth.awq_workload(12, 512, 256)
    torch.library.opcheck(torch.ops.svdq.awq_w4a16_linear.default,
                          (_bf(a.X), torch.from_numpy(a.qweight).cuda(), _bf(a.scales), _bf(a.zeros), None))
    assert P.svdq_device_status() == 0
