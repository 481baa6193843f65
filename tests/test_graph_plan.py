"""Host-side logic of the decode graph runner (CPU only): the captured batch sizes
follow the engine's list ("Architektur im Überblick", CUDA Graph Optimierung:
[1, 2, 4, 8] + multiples of 16 up to the maximum batch), and a batch is padded to
the smallest captured size that holds it."""
import bisect

import pytest

from paged_kv_cache_331_b200.graphs import graph_batch_sizes


def test_graph_batch_sizes_follow_the_engine():
    assert graph_batch_sizes(64) == [1, 2, 4, 8, 16, 32, 48, 64]
    assert graph_batch_sizes(20) == [1, 2, 4, 8, 16]
    assert graph_batch_sizes(1) == [1]
    assert graph_batch_sizes(512)[-1] == 512 and len(graph_batch_sizes(512)) == 4 + 32


@pytest.mark.parametrize("n,want", [(1, 1), (3, 4), (8, 8), (9, 16), (17, 32), (64, 64)])
def test_padding_takes_the_smallest_captured_size(n, want):
    sizes = graph_batch_sizes(64)
    assert sizes[bisect.bisect_left(sizes, n)] == want
