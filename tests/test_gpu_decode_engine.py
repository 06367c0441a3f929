"""The decode engine's work split, against the CPU oracle element by
element: a CTA stages T = 8 / G whole 32-row groups of one problem (G warps
per group split its k steps; partial sums meet in a shared-memory table),
groups too long for shared memory are staged in 2 KiB chunks of their rows,
launches too small to fill the GPU take one group per CTA, and a call is
split into several launches when it holds more CTAs than one launch maps,
or when a problem would take the third CTA slot per SM from the others
(the host-side planner's cases are in test_decode_plan.py).  These cases
drive the corners of that: many tiny problems, one group of many chunks,
steps with only part of their 256 k in range, whole groups up to 96 KiB,
the splits, and launches repeated on the same buffers.
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
    of one large one: 121 problems in one launch, most of them one CTA of a
    single partial group."""
    shapes = [(1 + (7 * i) % 64, 64 * (1 + i % 8)) for i in range(120)] + [(8192, 4096)]
    _xq_path(shapes, 4, 1000)


def test_one_group_of_many_chunks():
    """K = 32768 at M = 1: a group of whole rows (256 KiB) exceeds shared
    memory, so each CTA stages its group in 4 chunks of 2 KiB per row; N
    ragged (three groups, the last with 4 rows)."""
    _xq_path([(68, 32768)], 1, 1100)


def test_partial_chunks_and_slot_reuse():
    """K = 256 and K = 832: one-step rows, and a last step with 64 of its
    256 k in range (the lanes past the row read the next row's bytes against
    zero x_q); N = 8192 gives 32 CTAs of eight groups; run twice on the same
    buffers (the sums table must come back clean)."""
    _xq_path([(8192, 256), (333, 832)], 3, 1200, repeat=2)


def test_m16_wide_activations_one_problem_per_cta():
    """M = 16, K = 2048 (32 KiB of staged activations per CTA), two token
    tiles; fused act quant with SubLN."""
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


def test_whole_and_chunked_groups_in_one_launch():
    """K = 6144 at M = 4: whole groups of 48 KiB; K = 8640 and 12288 chunked
    (2160- and 3072-byte rows); K = 32768 (128 KiB of x_q at M = 4) beside
    them: the largest layouts share one launch (a few CTAs, one group each)."""
    _xq_path([(70, 8640), (65, 12288), (40, 32768), (33, 768), (50, 6144)], 4, 1400)


def test_more_ctas_than_one_launch_maps():
    """N = 600,000 rows of K = 64 at M = 2: 2344 CTAs of eight groups, more
    than the 2048 one launch maps, so the problem is split by row ranges
    over two launches."""
    _xq_path([(600000, 64)], 2, 1500)
