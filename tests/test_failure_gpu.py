"""Failure reporting without a GPU fault: a bounded device-side wait that runs
out (on a barrier nothing completes) is reported as KDA_ERR_TIMEOUT by
kda_device_status, the flag is cleared by reading it, and the context stays
usable for the real kernels."""
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert K.device_status() == 0            # nothing pending
    K.selftest_timeout(limit_us=2000)        # the wait gives up after 2 ms
    assert K.device_status() == 5            # KDA_ERR_TIMEOUT
    assert K.device_status() == 0            # reading clears the flag
    d = W.draw((1, 130), 2, 128, 128, io="bf16", n_states=1, device="cuda",
               seed=1)
    out, fin = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], None, chunk=64)
    assert K.device_status() == 0
    ref, _ = PY.oracle_dense(d)
    PY.check("out after timeout", PY.host64(out), ref, PY.TOL_BF16)


def test_timeout_probe_rejects_bad_limits():
    for bad in (0, -5, 200000):
        with pytest.raises(K.KdaError):
            K.selftest_timeout(limit_us=bad)
    torch.cuda.synchronize()
