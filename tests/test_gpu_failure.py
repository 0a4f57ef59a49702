"""Failure detection on the device, without a GPU fault.

The self-test kernel waits, through the forward kernel's bounded wait, on a
barrier that nothing arrives on (the shape of a lost arrival). The wait gives up
after its time limit, the kernel records the timeout in the device status word
and returns normally; the host reads BSFA_ERR_DEVICE_TIMEOUT, the word clears,
and the context keeps working.
"""
import time

import numpy as np
import pytest
import torch

from oracle import bsfa_oracle as O
from threshold_gated_block_b200 import bsfa
from threshold_gated_block_b200.build import build
from threshold_gated_block_b200.inputs import custom_config, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build()
    bsfa.load()


def test_lost_arrival_times_out_reports_and_leaves_the_context_usable():
    assert bsfa.bsfa_get_status(None) == bsfa.BSFA_OK
    t0 = time.time()
    assert bsfa.bsfa_selftest_lost_arrival(None) == bsfa.BSFA_OK
    status = bsfa.bsfa_get_status(None)
    elapsed = time.time() - t0
    assert status == bsfa.BSFA_ERR_DEVICE_TIMEOUT, bsfa.bsfa_status_string(status)
    assert "bounded wait" in bsfa.bsfa_last_error()
    assert 1.0 < elapsed < 60.0
    assert bsfa.bsfa_get_status(None) == bsfa.BSFA_OK          # the word was cleared

    cfg = custom_config(N=256, D=64, Hq=2, Hkv=2, Bq=64, Bk=64, causal=True, seed=31)
    x = make_inputs(cfg)
    tau = [np.inf, -np.inf]
    dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    out, lse, mask = bsfa.forward(dev(x["q"]), dev(x["k"]), dev(x["v"]), torch.tensor(tau, device="cuda"),
                                  Bq=64, Bk=64, causal=True, want_mask=True)
    torch.cuda.synchronize()
    assert bsfa.bsfa_get_status(None) == bsfa.BSFA_OK
    ref = O.forward(x["q"], x["k"], x["v"], tau, 64, 64, True)
    assert np.array_equal(mask.cpu().numpy(), ref["codes"])
    assert np.abs(out.float().cpu().numpy() - ref["out"]).max() <= 2e-2
