"""medusa_heads_topk_noalloc: the heads + top-k call for callers that cannot
allocate device memory (a host that reserves all device memory up front and
gives this library no allocator, or code where allocating is not allowed).

It must give the same results as medusa_heads_topk with a caller workspace,
call after call, because it keeps its scratch in one fixed array that every
call reuses.  The file name makes pytest collect it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from helpers import LOGIT_RTOL, SMALL, check_logits, pick_sub_h

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


def _run_with_workspace(mb, t, w):
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    ids = torch.full((w.B, w.K, w.topk), -1, dtype=torch.int32, device="cuda")
    vals = torch.zeros((w.B, w.K, w.topk), dtype=torch.float32, device="cuda")
    logits = torch.zeros((w.B, w.K, w.V), dtype=torch.float32, device="cuda")
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, ids, vals, ws, head_logits=logits)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), vals.cpu().numpy(), logits.cpu().numpy()


@pytest.mark.parametrize("name", ["v7b_small", "tiny_f32", "v13b_small"])
def test_noalloc_matches_workspace_call(mb, name):
    from synth import device
    w = SMALL[name]
    sub_h, _, _ = pick_sub_h(w)
    t = device.materialise(w, sub_h=sub_h)
    ref_ids, ref_vals, ref_logits = _run_with_workspace(mb, t, w)
    for call in range(2):                      # the array keeps the previous call's contents
        ids = torch.full((w.B, w.K, w.topk), -3, dtype=torch.int32, device="cuda")
        vals = torch.zeros((w.B, w.K, w.topk), dtype=torch.float32, device="cuda")
        logits = torch.zeros((w.B, w.K, w.V), dtype=torch.float32, device="cuda")
        mb.medusa_heads_topk_noalloc(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, ids, vals,
                                     head_logits=logits)
        torch.cuda.synchronize()
        assert np.array_equal(ids.cpu().numpy(), ref_ids), f"call {call}"
        check_logits(vals.cpu().numpy(), ref_vals.astype(np.float64), LOGIT_RTOL)
        check_logits(logits.cpu().numpy(), ref_logits.astype(np.float64), LOGIT_RTOL)
    st, det = mb.device_status()
    assert (st, det) == (0, 0)


def test_noalloc_rejects_shapes_above_its_fixed_scratch(mb):
    # u alone needs B*K*d*4 bytes: 64 * 16 * 8192 * 4 = 32 MiB > 4 MiB
    B, d, V, K, topk = 64, 8192, 1000, 16, 8
    h = torch.zeros((B, d), dtype=torch.bfloat16, device="cuda")
    Wout = torch.zeros((K, V, d), dtype=torch.bfloat16, device="cuda")
    ids = torch.full((B, K, topk), -3, dtype=torch.int32, device="cuda")
    vals = torch.zeros((B, K, topk), dtype=torch.float32, device="cuda")
    # Straight through the C ABI: the size check comes before any pointer is
    # used, so h stands in for W1 and b1 here (the binding would refuse their shapes).
    p = lambda x: ctypes.c_void_p(x.data_ptr())
    with pytest.raises(mb.MedusaError) as ei:
        mb._check(mb._lib.medusa_heads_topk_noalloc(p(h), p(h), p(h), p(Wout), B, d, V, K, topk, mb.MEDUSA_BF16,
                                                    None, p(ids), p(vals), None))
    assert ei.value.code == mb.MEDUSA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (ids == -3).all()
