"""The decode engine's launch planner (host logic, no GPU): how a decode call
over a list of (N, K) problems is cut into launches, CTAs of whole 32-row
groups and row slices, checked through bl_debug_decode_plan."""
from __future__ import annotations

import pytest

from ternary_quantized_linear_bitlinear_b200 import api, workloads

SMEM_ATTR = 226 * 1024
SMEM_3 = 228 * 1024 // 3 - 2 * 1024  # a CTA layout that still fits three to an SM


def _check_cover(shapes, launches):
    """Every row of every problem in exactly one slice; a slice's CTAs are
    consecutive, each of T = 8 >> glog groups (one with K chunks); launch
    limits hold."""
    seen = {j: [] for j in range(len(shapes))}
    for L in launches:
        assert 1 <= L["ctas"] <= 2048
        assert len(L["problems"]) <= 128
        assert 0 < L["smem"] <= SMEM_ATTR
        cta = 0
        for p in L["problems"]:
            N, K = shapes[p["job"]]
            T = 8 >> p["glog"]
            assert p["cta_begin"] == cta
            if p["kch"] > 1:
                assert p["glog"] == 3 and p["kch"] == -(-(K // 4) // 2048)
            cta += -(-p["rows"] // (T * 32))
            seen[p["job"]].append((p["row0"], p["rows"]))
        assert cta == L["ctas"]
    for j, (N, K) in enumerate(shapes):
        row = 0
        for r0, n in sorted(seen[j]):
            assert r0 == row and n > 0
            row += n
        assert row == N, f"problem {j}: rows {row} of {N}"


@pytest.mark.parametrize("M", [1, 4, 8, 16])
def test_decode125m_step_is_one_launch(M):
    shapes = [(N, K) for _ in range(12) for (_, N, K, _) in workloads.decode125m_layer_shapes()]
    launches = api.bl_debug_decode_plan(shapes, M)
    _check_cover(shapes, launches)
    assert len(launches) == 1 and launches[0]["ctas"] == 432
    if M <= 8:
        assert launches[0]["smem"] <= SMEM_3  # three CTAs per SM


def test_layer3b_m1():
    shapes = [(N, K) for (_, N, K, _) in workloads.layer3b_shapes()]
    launches = api.bl_debug_decode_plan(shapes, 1)
    _check_cover(shapes, launches)
    assert len(launches) == 1 and launches[0]["ctas"] == 570
    down = [p for p in launches[0]["problems"] if shapes[p["job"]][1] == 8640]
    assert down and all(p["kch"] == 2 for p in down)  # 2160-byte rows: chunked
    assert launches[0]["smem"] <= SMEM_3


def test_more_ctas_than_one_launch_maps():
    shapes = [(600000, 64)]
    launches = api.bl_debug_decode_plan(shapes, 2)
    _check_cover(shapes, launches)
    assert len(launches) == 2 and launches[0]["ctas"] == 2048


def test_largest_layouts_fit_one_launch():
    # chunked 32768-wide rows (64 KiB of weights, 128 KiB of x_q at M = 4)
    # beside whole and chunked groups: the largest layouts the limits allow
    # still fit one launch's shared memory
    shapes = [(70, 8640), (65, 12288), (40, 32768), (33, 768), (50, 6144)]
    launches = api.bl_debug_decode_plan(shapes, 4)
    _check_cover(shapes, launches)
    assert len(launches) == 1
    assert [p["kch"] for p in launches[0]["problems"]] == [2, 2, 4, 1, 1]


def test_third_cta_slot_kept():
    # problems whose CTAs fit three to an SM (256 of them) ahead of one whose
    # layout (M = 8, 32 KiB of x_q) would not: a second launch for it
    shapes = [(32768, 768), (32768, 768), (64, 4096)]
    launches = api.bl_debug_decode_plan(shapes, 8)
    _check_cover(shapes, launches)
    assert len(launches) == 2
    assert launches[0]["smem"] <= SMEM_3  # (the combined layout would not be)
    assert [p["job"] for p in launches[1]["problems"]] == [2]


def test_too_few_ctas_take_a_group_each():
    shapes = [(300, 768)]
    launches = api.bl_debug_decode_plan(shapes, 1)
    _check_cover(shapes, launches)
    assert launches[0]["ctas"] == 10 and launches[0]["problems"][0]["glog"] == 3


@pytest.mark.parametrize("shapes,M", [([], 1), ([(64, 768)], 0), ([(64, 768)], 17), ([(64, 100)], 1),
                                      ([(0, 768)], 1), ([(64, 32768)], 5)])
def test_rejected_calls(shapes, M):
    with pytest.raises(api.BitLinearError):
        api.bl_debug_decode_plan(shapes, M)
