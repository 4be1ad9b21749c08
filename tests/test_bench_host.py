"""Host logic of bench.py that needs no GPU: the end-to-end copy groups and the
roofline peak of each kernel kind."""
import pytest

import bench
import workloads


@pytest.mark.parametrize("w", workloads.WORKLOADS, ids=lambda w: w.name)
def test_e2e_groups_partition_the_set_by_shape(w):
    groups = bench.e2e_groups(w)
    assert sorted(i for g in groups for i in g) == list(range(w.count))
    for g in groups:
        assert 1 <= len(g) <= 16
        assert len({(min(w.shapes[i]), max(w.shapes[i])) for i in g}) == 1
    smallest = min(r * c for r, c in w.shapes)
    if sum(r * c == smallest for r, c in w.shapes) > 4:
        # the groups whose copies overlap nothing hold two of the smallest matrices
        for g in (groups[0], groups[-1]):
            assert len(g) == 2 and all(w.shapes[i][0] * w.shapes[i][1] == smallest for i in g)


def test_roofline_peak_by_kernel_kind():
    peaks = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
    # FFMA kernels: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz
    for kind in ("chain_ffma", "gram_ffma", "apply_ffma", "chain_small"):
        bound, unit, peak, basis = bench.roofline_peak(kind, True, peaks, 148, 1965.0)
        assert (bound, unit, peak) == ("alu", "TFLOP/s", 74.4) and "148 SMs" in basis
    assert bench.roofline_peak("chain_ffma", True, peaks, 148, None)[2] == 74.4
    assert bench.roofline_peak("apply_tc", True, peaks, 148, 1965.0) == ("tensor", "TFLOP/s", 1400.0, None)
    assert bench.roofline_peak("chain_tc", True, {"hbm_gbs": 1.0, "bf16_tflops": 1590.0}, 148, None)[2] == 1590.0
    assert bench.roofline_peak("momentum", False, peaks, 148, 1965.0) == ("hbm", "GB/s", 6650.0, None)
