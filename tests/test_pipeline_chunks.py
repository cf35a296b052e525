"""Host logic of the streamed (copy-overlapped) pipeline: the chunks of a
[B, heads, ...] call are contiguous, disjoint and cover every (b, head)."""

import pytest

from block_sparse_attention_34_b200.pipeline import chunk_ranges


@pytest.mark.parametrize("B,heads,chunks", [(1, 40, 8), (1, 3, 8), (1, 12, 5), (2, 12, 8),
                                            (5, 4, 2), (1, 1, 1), (3, 7, 3)])
def test_chunks_cover_every_head_once(B, heads, chunks):
    r = chunk_ranges(B, heads, chunks)
    assert 1 <= len(r) <= chunks
    seen = set()
    for b0, b1, h0, h1 in r:
        assert 0 <= b0 < b1 <= B and 0 <= h0 < h1 <= heads
        # contiguous in a [B, heads, N, d] tensor: one batch element's head
        # range, or whole batch elements
        assert b1 - b0 == 1 or (h0, h1) == (0, heads)
        for b in range(b0, b1):
            for h in range(h0, h1):
                assert (b, h) not in seen
                seen.add((b, h))
    assert len(seen) == B * heads
    sizes = [(b1 - b0) * (h1 - h0) for b0, b1, h0, h1 in r]
    assert max(sizes) - min(sizes) <= (heads if B > 1 else 1)  # balanced
