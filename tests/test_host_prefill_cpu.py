"""Host logic of pipeline.HostPrefill: its slice boundaries (no GPU)."""
import pytest

from long_context_rope_b200.pipeline import slice_bounds


@pytest.mark.parametrize("q_len,chunk,cps", [(65536, 64, 64), (1500, 64, 10), (1244, 64, 10),
                                             (64, 64, 8), (100, 64, 8), (8192, 128, 3),
                                             (4096, 64, 1000), (2000, 64, 1)])
def test_slice_bounds_cover_the_span_on_chunk_boundaries(q_len, chunk, cps):
    nqc = (q_len + chunk - 1) // chunk
    b = slice_bounds(nqc, chunk, q_len, cps)
    assert b[0] == 0 and b[-1] == q_len
    assert all(x < y for x, y in zip(b, b[1:]))                 # non-empty, ascending
    assert all(x % chunk == 0 for x in b[:-1])                   # every slice starts a chunk
    sizes = [(y - x + chunk - 1) // chunk for x, y in zip(b, b[1:])]  # query chunks per slice
    assert sum(sizes) == nqc
    assert min(sizes) >= min(cps, nqc)                           # never fewer than asked
    if nqc >= cps:
        assert max(sizes) < 2 * cps                              # and not much more


def test_slice_bounds_examples():
    assert slice_bounds(24, 64, 1500, 10) == [0, 768, 1500]
    assert slice_bounds(1024, 64, 65536, 64) == [64 * 64 * i for i in range(16)] + [65536]
    assert slice_bounds(3, 64, 150, 8) == [0, 150]
