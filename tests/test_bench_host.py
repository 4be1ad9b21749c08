"""Host logic of bench.py that needs no GPU: the end-to-end copy groups."""
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
