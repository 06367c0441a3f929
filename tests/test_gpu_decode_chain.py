"""The dependency-ordered decode step (chain.DecodeChain): each layer's
projections read the previous launch's output, through SubLN before o and
down and the ReLU^2-gated FFN, twelve layers of the 125M shapes in one
CUDA graph.  Checked layer by layer against the oracle run on that layer's
input as the GPU produced it: every x_q and s bit for bit, every int32
accumulator exactly, every Y within 1e-6 relative -- up to the last layer's
output."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ternary_quantized_linear_bitlinear_b200 import api, workloads
from ternary_quantized_linear_bitlinear_b200.chain import PROJ, DecodeChain
from _parity import check_y, np32

pytestmark = pytest.mark.gpu


def _build(M, nlayers, record=True):
    items = workloads.decode125m(seed=5, M=M, layers=nlayers)
    layers, refs, gains = [], [], []
    per = len(PROJ)
    for li in range(nlayers):
        lay, ref = {}, {}
        for j, name in enumerate(PROJ):
            _, W, _ = items[li * per + j]
            packed, gamma = api.bl_quant_weights(W.cuda())
            lay[name] = (packed, gamma, W.shape[0], W.shape[1])
            _, g_ref, wq = oracle.quant_weights(np32(W))
            ref[name] = (wq, g_ref)
        layers.append(lay)
        refs.append(ref)
        gains.append((workloads.uniform((768,), 0.9, 1.1, 30 + li).cuda(),
                      workloads.uniform((2048,), 0.9, 1.1, 60 + li).cuda()))
    chain = DecodeChain(layers, gains, M, record=record)
    chain.x0.copy_(items[0][2].float().cuda() * 3.0)
    return chain, refs, gains


def _check_proj(b, X, gain, ref):
    xq_ref, s_ref = oracle.quant_act(X, None if gain is None else np32(gain), 1e-6)
    assert np.array_equal(b["x_q"].cpu().numpy(), xq_ref)
    assert np.array_equal(b["s"].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    wq, g = ref
    acc_ref = oracle.contract(xq_ref, wq)
    assert np.array_equal(b["acc"].cpu().numpy(), acc_ref)
    check_y(b["Y"].cpu().numpy(), acc_ref, g, s_ref[:, None])


@pytest.mark.parametrize("M", [1, 4])
def test_decode_chain_layer_by_layer(M):
    nlayers = 12
    chain, refs, gains = _build(M, nlayers)
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    chain.run(stream.cuda_stream)  # eager once (one-time set-up), then the graph
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        chain.run(stream.cuda_stream)
    g.replay()
    torch.cuda.synchronize()
    api.bl_check_device_error()
    for li, (b, ref, (g_o, g_d)) in enumerate(zip(chain.layers, refs, gains)):
        x_in = np32(b["x_in"])
        for name in ("q", "k", "v"):
            _check_proj(b[name], x_in, None, ref[name])
        _check_proj(b["o"], np32(b["q"]["Y"]), g_o, ref["o"])
        y_o = np32(b["o"]["Y"])
        for name in ("gate", "up"):
            _check_proj(b[name], y_o, None, ref[name])
        xq_ref, s_ref = oracle.ffn_act_quant(np32(b["gate"]["Y"]), np32(b["up"]["Y"]), np32(g_d), 1e-6)
        assert np.array_equal(b["ffn_xq"].cpu().numpy(), xq_ref), f"layer {li}: FFN x_q"
        assert np.array_equal(b["ffn_s"].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        wq, gd = ref["down"]
        acc_ref = oracle.contract(xq_ref, wq)
        assert np.array_equal(b["down"]["acc"].cpu().numpy(), acc_ref), f"layer {li}: down acc"
        check_y(b["down"]["Y"].cpu().numpy(), acc_ref, gd, s_ref[:, None])
    assert chain.out.data_ptr() == chain.layers[-1]["down"]["Y"].data_ptr()
    assert torch.isfinite(chain.out).all() and chain.out.abs().max() > 0
