"""torch.library registration of the device calls and the nn.Module layers (host side:
registration, fake implementations, tracing by torch.export, the nn.Linear swap)."""

import pytest
import torch
from torch import nn

import bit_diffusion_transformer_act_b200 as P
from bit_diffusion_transformer_act_b200 import torch_ops as T


def test_operators_registered():
    for name in ("quantize_act_lowrank_down", "w4a4_nvfp4_linear", "awq_w4a16_linear"):
        assert hasattr(torch.ops.svdq, name), name


@pytest.mark.parametrize("M,K", [(1, 64), (5, 512), (128, 3072), (129, 3072), (4096, 3072)])
def test_fake_scale_bytes_match_the_library(M, K):
    X = torch.empty((M, K), dtype=torch.bfloat16, device="meta")
    codes, scales, low = torch.ops.svdq.quantize_act_lowrank_down(X, torch.empty((K,), dtype=torch.bfloat16,
                                                                                 device="meta"),
                                                                  torch.empty((8,), dtype=torch.uint8, device="meta"),
                                                                  0.5, 32)
    assert codes.shape == (M, K // 2) and codes.dtype == torch.uint8
    assert scales.shape == (P.svdq_act_scale_bytes(M, K),) and scales.dtype == torch.uint8
    assert low.shape == (M, 64) and low.dtype == torch.bfloat16


def _awq_layer(N=128, K=512, bias=False):
    return T.AwqLinear(torch.zeros((N, K // 2), dtype=torch.uint8), torch.zeros((N, K // 64), dtype=torch.bfloat16),
                       torch.zeros((N, K // 64), dtype=torch.bfloat16),
                       torch.zeros((N,), dtype=torch.bfloat16) if bias else None)


def test_export_traces_awq_layer_without_breaks():
    ep = torch.export.export(_awq_layer(bias=True), (torch.zeros((2, 3, 512), dtype=torch.bfloat16),))
    targets = [str(n.target) for n in ep.graph.nodes if n.op == "call_function"]
    assert "svdq.awq_w4a16_linear.default" in targets
    out = [n for n in ep.graph.nodes if n.op == "output"][0].args[0][0]
    assert tuple(out.meta["val"].shape) == (2, 3, 128)


def test_export_traces_svdq_layer_without_breaks():
    layer = T.SvdqLinear(512, 256, 32, torch.zeros(1024, dtype=torch.uint8), torch.zeros(512, dtype=torch.bfloat16),
                         0.5, 0.25)
    ep = torch.export.export(layer, (torch.zeros((7, 512), dtype=torch.bfloat16),))
    targets = [str(n.target) for n in ep.graph.nodes if n.op == "call_function"]
    assert targets.count("svdq.quantize_act_lowrank_down.default") == 1
    assert targets.count("svdq.w4a4_nvfp4_linear.default") == 1
    out = [n for n in ep.graph.nodes if n.op == "output"][0].args[0][0]
    assert tuple(out.meta["val"].shape) == (7, 256)


def test_wrong_in_features_raises():
    with pytest.raises(ValueError):
        _awq_layer()(torch.zeros((2, 256), dtype=torch.bfloat16))


def test_swap_linears_replaces_selected_layers():
    model = nn.Sequential(nn.Linear(512, 128), nn.GELU(), nn.Sequential(nn.Linear(128, 512), nn.Linear(512, 64)))
    names = []

    def factory(name, lin):
        names.append(name)
        return _awq_layer(lin.out_features, lin.in_features) if lin.in_features % 256 == 0 else None

    assert T.swap_linears(model, factory) == 2
    assert names == ["0", "2.0", "2.1"]
    assert isinstance(model[0], T.AwqLinear) and isinstance(model[2][1], T.AwqLinear)
    assert isinstance(model[2][0], nn.Linear)


def test_svdq_layer_state_dict_round_trip_keeps_the_scales():
    a = T.SvdqLinear(512, 256, 32, torch.arange(1024, dtype=torch.int32).to(torch.uint8),
                     torch.ones(512, dtype=torch.bfloat16), 0.5, 0.25)
    b = T.SvdqLinear(64, 128, 32, torch.zeros(1024, dtype=torch.uint8), torch.zeros(512, dtype=torch.bfloat16),
                     1.0, 1.0)
    b.load_state_dict(a.state_dict())
    assert (b.in_features, b.out_features, b.rank) == (512, 256, 32)
    assert (b.act_global_scale, b.w_global_scale) == (0.5, 0.25)
    assert torch.equal(b.packed_w, a.packed_w) and torch.equal(b.smooth_inv, a.smooth_inv)
