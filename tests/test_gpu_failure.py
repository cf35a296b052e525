"""The failure path of the tcgen05 attention kernel, driven on the GPU
without a fault: a host-set test hook (pa_test_inject_v_stall) makes the
V-tile loader of one CTA skip one kept tile, so the MMA issuer's bounded
wait for it runs out after a host-set limit of 1 ms.  The kernel must record
PA_ERR_TIMEOUT, unwind (every role leaves its loop, copies and MMAs drained,
tensor memory released), return quickly, and leave the context usable: a
normal call afterwards on the same context is checked against the oracle.
No trap, no bad address, nothing left waiting."""

import time

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_ref as ref

from helpers import compare, custom, inputs, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("permuted", [True, False], ids=["tma_tiles", "gathered_rows"])
def test_bounded_wait_runs_out_and_context_stays_usable(permuted):
    w = custom("stall_1024", 1, 2, 128, (4, 16, 16), 128, "bf16", 1.0, perms=(0, 3))
    q, k, v, perms = inputs(w)
    pr = paro.Problem(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms)
    qd, kd, vd = to_dev(q, k, v)
    if permuted:
        qd, kd, vd = (paro.reorder(x, pr) for x in (qd, kd, vd))
    idx = torch.arange(w.NB, dtype=torch.int32, device="cuda").expand(1, w.heads, w.NB, w.NB)
    idx = idx.contiguous()
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block,
                         idx.cpu().numpy())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call():
        out = paro.block_sparse_attn(qd, kd, vd, pr, idx, status=status, permuted=permuted)
        torch.cuda.synchronize()
        return out

    out = call()  # warm: module load, attribute set-up
    assert status.item() == 0
    compare(out, want)

    paro.test_inject_v_stall(query_block=3, batch_head=1, tile=2, wait_limit_ns=1_000_000)
    try:
        t0 = time.perf_counter()
        call()
        elapsed = time.perf_counter() - t0
    finally:
        paro.test_inject_v_stall(-1, -1, -1, 0)
    assert status.item() == paro.PA_ERR_TIMEOUT
    assert elapsed < 1.0, elapsed

    # the same context, the hook off, the status cleared: a normal call
    paro.clear_status(status)
    out = call()
    assert status.item() == 0
    compare(out, want)

