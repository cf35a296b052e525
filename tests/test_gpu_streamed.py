"""The host-memory API with copies overlapped with the work
(pipeline.StreamedPipeline) gives the one-shot Pipeline's output bit for
bit: every step of the path is per head, so splitting the heads (or batch
elements) into chunks on their own streams changes no arithmetic."""

import pytest
import torch

from block_sparse_attention_34_b200.pipeline import Pipeline, StreamedPipeline

from helpers import custom, inputs, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    (custom("streamed_6h", 1, 6, 128, (5, 18, 20), 128, "bf16", 0.3,
            perms=(0, 3, 6, 8, 5, 1)), 4, {}),
    (custom("streamed_b2", 2, 3, 128, (6, 10, 13), 128, "bf16", 0.5, perms=(4, 0, 2)), 8, {}),
    (custom("streamed_int8", 1, 4, 128, (5, 7, 9), 128, "bf16", 0.67, perms=(0, 1, 2, 3)), 3,
     {"int8": True}),
    (custom("streamed_int4", 1, 4, 128, (5, 7, 9), 128, "bf16", 0.67, perms=(0, 1, 2, 3)), 2,
     {"int4_pv": True}),
]


@pytest.mark.parametrize("w,chunks,kw", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_streamed_equals_one_shot(w, chunks, kw):
    q, k, v, perms = inputs(w)
    grid = (w.F, w.H, w.W)
    one = Pipeline(w.B, w.heads, grid, w.d, w.block, perms, w.density, **kw)
    want = one.run(*to_dev(q, k, v)).clone()
    torch.cuda.synchronize()
    assert one.status.item() == 0
    sp = StreamedPipeline(w.B, w.heads, grid, w.d, w.block, perms, w.density, chunks=chunks,
                          **kw)
    host = [x.to(torch.bfloat16).contiguous().pin_memory() for x in (q, k, v)]
    host_out = torch.full(want.shape, float("nan"), dtype=want.dtype).pin_memory()
    for _ in range(2):  # twice: buffers are reused across calls
        sp.run(*host, host_out)
        torch.cuda.synchronize()
        assert sp.status() == 0
        assert torch.equal(host_out, want.cpu())
