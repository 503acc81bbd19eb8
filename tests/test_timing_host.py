"""Host-only checks of the measurement helpers: the busy-interval union of the timing build's
MMA-group log, and the no-alloc status reader's argument check."""
import pytest

from matrix_memory_rnn_b200 import build as gbuild
from matrix_memory_rnn_b200 import gdr
from matrix_memory_rnn_b200.phase_timing import union_length


@pytest.mark.parametrize("spans,expect", [
    ([], 0),
    ([(3, 3)], 0),
    ([(0, 10)], 10),
    ([(0, 10), (20, 25)], 15),                 # disjoint
    ([(0, 10), (5, 15)], 15),                  # overlapping
    ([(0, 30), (5, 10), (12, 20)], 30),        # nested
    ([(20, 25), (0, 10), (10, 12)], 17),       # unsorted, touching
    ([(0, 10), (0, 10)], 10),                  # identical
])
def test_union_length(spans, expect):
    assert union_length(spans) == expect


def test_union_length_matches_a_cell_count():
    """Against counting covered unit cells on a grid (an independent formulation)."""
    import random
    rng = random.Random(7)
    for _ in range(200):
        spans = []
        for _ in range(rng.randint(1, 8)):
            a = rng.randint(0, 60)
            spans.append((a, a + rng.randint(0, 15)))
        cells = set()
        for a, b in spans:
            cells.update(range(a, b))
        assert union_length(spans) == len(cells)


def test_noalloc_read_status_rejects_a_null_output():
    gbuild.build()
    lib = gdr.library()
    fn = lib.gdr_noalloc_read_status
    fn.restype = gdr._c_int
    assert fn(None, None) == 1   # GDR_ERR_INVALID_ARG, before any CUDA call
