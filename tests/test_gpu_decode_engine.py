"""The decode engine's work partition, against the CPU oracle element by
element: the host cuts the groups of 32 weight rows of all problems into
one byte-balanced range per CTA and splits ranges at problem boundaries for
the activation staging; inside a CTA the chunks of 32 rows x 512 k stream
through a ring and the warps' partial sums meet in per-group accumulator
slots.  These cases drive the corners of that: many tiny problems in one
range, one group of many chunks, chunks with only part of their 512 k in
range, slot reuse over hundreds of one-chunk groups, and launches repeated
on the same buffers (the slots must come back clean).
"""
from __future__ import annotations

import pytest
import torch

from ternary_quantized_linear_bitlinear_b200 import api, workloads
from _parity import check_act, check_forward_full, check_weights, gpu_quant_weights

pytestmark = pytest.mark.gpu


def _xq_path(shapes, M, seed, repeat=1):
    """shapes: [(N, K)]; x_q path (bl_quant_act_grouped + bl_forward_grouped)."""
    dev, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W = workloads.normal((N, K), 0.02, seed + 3 * i)
        X = workloads.with_outlier_channels(workloads.normal((M, K), 1.0, seed + 3 * i + 1, torch.bfloat16),
                                            max(1, K // 128), 20.0, seed + 3 * i + 2)
        packed, gamma = gpu_quant_weights(W)
        x_q, s = api.bl_quant_act(X.cuda())
        Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
        dev.append((packed, gamma, x_q, s, Y, acc, N, K))
        refs.append((W, X))
    arr = api.make_problems(dev)
    for _ in range(repeat):
        api.bl_forward_grouped(arr, len(dev), M)
    api.bl_check_device_error()
    for (packed, gamma, x_q, s, Y, acc, N, K), (W, X) in zip(dev, refs):
        wq_ref, g_ref = check_weights(W, packed, gamma)
        xq_ref, s_ref = check_act(X, x_q, s)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, Y, acc)


def test_many_tiny_problems_share_a_range():
    """120 small problems (one group each, ragged N, K from 64 to 512) ahead
    of one large one: the first byte-balanced range holds all of them and is
    split at problem boundaries (at most eight problems' activations per
    CTA)."""
    shapes = [(1 + (7 * i) % 64, 64 * (1 + i % 8)) for i in range(120)] + [(8192, 4096)]
    _xq_path(shapes, 4, 1000)


def test_one_group_of_many_chunks():
    """K = 32768 at M = 1: 64 chunks per group, N ragged (three groups, the
    last with 4 rows)."""
    _xq_path([(68, 32768)], 1, 1100)


def test_partial_chunks_and_slot_reuse():
    """K = 256 and K = 832: chunks with 64 or 80 of their 128 bytes in range;
    N = 8192 gives hundreds of one-chunk groups per launch, each CTA reusing
    every accumulator slot many times; run twice on the same buffers."""
    _xq_path([(8192, 256), (333, 832)], 3, 1200, repeat=2)


def test_m16_wide_activations_one_problem_per_cta():
    """M = 16, K = 2048 (32 KiB of staged activations per problem): ranges
    hold one problem each; fused act quant with SubLN."""
    M = 16
    dev, refs = [], []
    for i in range(5):
        N, K = 700 + 37 * i, 2048
        W = workloads.normal((N, K), 0.02, 1300 + i)
        X = workloads.normal((M, K), 1.0, 1310 + i, torch.bfloat16)
        gain = workloads.uniform((K,), 0.9, 1.1, 1320 + i)
        packed, gamma = gpu_quant_weights(W)
        Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        s = torch.empty(M, dtype=torch.float32, device="cuda")
        acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
        dev.append((packed, gamma, X.cuda(), gain.cuda(), Y, xq, s, acc, N, K))
        refs.append((W, X, gain))
    arr = api.make_decode_problems(dev)
    api.bl_linear_decode_grouped(arr, len(dev), M, torch.bfloat16, 1e-6)
    api.bl_check_device_error()
    for d, (W, X, gain) in zip(dev, refs):
        wq_ref, g_ref = check_weights(W, d[0], d[1])
        xq_ref, s_ref = check_act(X, d[5], d[6], gain)
        check_forward_full(xq_ref, s_ref, wq_ref, g_ref, d[4], d[7])
