"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The batch-1 heads kernel waits, between its residual block and its
vocabulary projection, until every CTA has published its part of u.  The
test hook makes that wait expect one more CTA than the launch has and gives
every wait of the kernel a 1 ms limit, so the wait runs out: the kernel must
record MEDUSA_ERR_TIMEOUT with the detail of that wait in the device status
word, let its copies in flight land, and return.  The context stays usable:
after the workspace is zeroed again, the next call without the hook must be
exact against the oracle.  Nothing here traps, faults or hangs the GPU.
"""

import numpy as np
import pytest
import torch

import oracle.medusa_oracle as O
from helpers import SMALL, check_logits, pick_sub_h

pytestmark = pytest.mark.gpu

DETAIL_HEADS_S1_WAIT = 1


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


def _heads(mb, t, w, ws):
    ids = torch.full((w.B, w.K, w.topk), -7, dtype=torch.int32, device="cuda")
    vals = torch.zeros((w.B, w.K, w.topk), device="cuda")
    logits = torch.zeros((w.B, w.K, w.V), device="cuda")
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, ids, vals, ws, head_logits=logits)
    return ids, vals, logits


@pytest.mark.parametrize("name", ["v7b_small", "tiny_f32"])
def test_wait_runs_out_and_the_next_call_is_exact(mb, name):
    from synth import device
    w = SMALL[name]
    assert w.B == 1            # the batch-1 kernel holds the grid-wide wait
    sub_h, _, z = pick_sub_h(w)
    ref_ids, _ = O.topk_desc(z, w.topk)
    t = device.materialise(w, sub_h=sub_h)
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    mb.device_status(clear=True)
    try:
        mb.medusa_test_heads_wait(1, 1_000_000)          # one CTA too many, 1 ms
        ids, _, _ = _heads(mb, t, w, ws)
        torch.cuda.synchronize()
    finally:
        mb.medusa_test_heads_wait(0, 0)
    st, det = mb.device_status(clear=True)
    assert (st, det) == (mb.MEDUSA_ERR_TIMEOUT, DETAIL_HEADS_S1_WAIT)
    assert (ids == -7).all(), "an aborted launch writes no top-k"
    # The context is still usable; with the workspace zeroed again the next call is exact.
    ws.zero_()
    ids, vals, logits = _heads(mb, t, w, ws)
    torch.cuda.synchronize()
    assert mb.device_status(clear=True) == (0, 0)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    check_logits(logits.cpu().numpy(), z)
    # ... and so is a second call on the same workspace (its counters reset themselves).
    ids2, _, _ = _heads(mb, t, w, ws)
    torch.cuda.synchronize()
    assert torch.equal(ids2, ids) and mb.device_status(clear=True) == (0, 0)


def test_hook_rejects_bad_values(mb):
    for bad in [(-1, 0), (2000, 0), (0, -5)]:
        with pytest.raises(mb.MedusaError):
            mb.medusa_test_heads_wait(*bad)
