"""Failure detection without a GPU fault: a kernel wait that can never
complete runs out after its bound, the kernel records a timeout in the
workspace status word and returns, hyb_check_status reports HYB_ERR_TIMEOUT,
and the context keeps working (the next product is correct)."""
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, case, dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(orc):
    ws = hyb.new_workspace(256, dev())
    hyb.selftest_wait_timeout(ws, wait_limit=256)
    with pytest.raises(hyb.HybError) as ei:
        hyb.check_status(ws)
    assert ei.value.status == hyb.HYB_ERR_TIMEOUT
    assert ei.value.flags & hyb.STATUS_TIMEOUT
    assert hyb.check_status(ws) == 0  # the word was cleared
    # the context is intact: a product right after is correct
    n, k, b1, b2 = 512, 1024, 128, 128
    tmap = inputs.tile_map_bernoulli((n // b1) * (k // b2), 0.5, inputs.seed_of("after_timeout"))
    W, tmap, X, _ = case(n, k, b1, b2, tmap, batch=2, name="after_timeout")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    Y = hyb.spmm_skinny(P, X.to(dev()))
    torch.cuda.synchronize()
    y_ref, env = orc.spmv(n, k, b1, b2, tmap, orc.pack(inputs.bits(W), b1, b2, tmap),
                          inputs.bits(X))
    assert_within(Y.cpu().numpy(), y_ref, env, what="after timeout")
