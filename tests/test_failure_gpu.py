"""Failure detection without a fault: a bounded device-side wait that gives up is
reported as KDA_ERR_TIMEOUT by kda_check_status, cleared, and the context stays
usable.  The wait runs on a barrier that nothing completes (kda_selftest_timeout);
no GPU is faulted, trapped or hung.
"""
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import inputs as I


def test_selftest_rejects_bad_wait_before_launch():
    lib = kda.load()
    assert lib.kda_selftest_timeout(0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_selftest_timeout(10001, None) == kda.KDA_ERR_INVALID_ARG


@pytest.mark.gpu
def test_bounded_wait_gives_up_is_reported_and_cleared():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kda.check_status()                       # nothing pending
    kda.selftest_timeout(50)
    with pytest.raises(kda.KDAError) as err:
        kda.check_status()
    assert err.value.status == kda.KDA_ERR_TIMEOUT
    kda.check_status()                       # reading the status cleared it
    # the context is still usable: a prefill on both paths runs and matches the oracle
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=1, H=2, T=200, seed=91)
    x = I.make_inputs(w, "cuda")
    args = [x[n] for n in ("q", "k", "v", "log_alpha", "beta")] + [x["initial_state"]]
    o_ref, s_ref = oracle.forward(*args)
    for ws in (None, kda.make_workspace(w.B, w.T, w.H, 128, 128)):
        out, sT = kda.forward(*args, workspace=ws)
        torch.cuda.synchronize()
        kda.check_status()
        assert oracle.parity_error(out.cpu().numpy(), o_ref) <= 2e-3
        assert oracle.parity_error(sT.cpu().numpy(), s_ref) <= 2e-3
