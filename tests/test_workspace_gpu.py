"""The stream-ordered workspace is cached by the device's memory pool: after
the first call of a given size, repeated calls of the staged pipeline, the
packed fused path and the backward pass reserve no new device memory
(kda_workspace_pool), and their results do not change from call to call."""
import numpy as np
import pytest
import torch

import kda_workloads as W
import parity as PY
from gated_delta_rule_156_b200 import kda as K

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _calls(fn, n=5):
    outs, reserved = [], []
    for _ in range(n):
        outs.append(fn())
        torch.cuda.synchronize()
        reserved.append(K.workspace_pool()[0])
    return outs, reserved


def test_repeated_calls_reserve_nothing_new():
    d = W.make(1, device=DEV)
    _, _, ws = K.chunk_fwd_plan(1, 2048, 4, 64, 64, 64, torch.bfloat16,
                                staged=True)

    def staged():
        o, f = K.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                           d["initial_state"], None, chunk=64, staged=True)
        return PY.host64(o)

    outs, reserved = _calls(staged)
    assert reserved[0] >= ws, (reserved, ws)
    assert all(r == reserved[0] for r in reserved), reserved
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])

    lengths = [300, 0, 77, 200]
    dp = W.draw((1, sum(lengths)), 2, 128, 128, io="bf16",
                n_states=len(lengths), device=DEV, seed=5)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]),
                      dtype=torch.int32, device=DEV)

    def packed():
        o, f = K.chunk_fwd(dp["q"], dp["k"], dp["v"], dp["log_alpha"],
                           dp["beta"], dp["initial_state"], cu, chunk=64)
        return PY.host64(o)

    outs, reserved = _calls(packed)
    assert all(r == reserved[0] for r in reserved), reserved

    db = W.draw((1, 200), 2, 64, 64, io="f32", n_states=1, device=DEV, seed=6)
    do = torch.randn(db["v"].shape, device=DEV)

    def backward():
        g = K.chunk_bwd(db["q"], db["k"], db["v"], db["log_alpha"], db["beta"],
                        db["initial_state"], None, do, None, chunk=32)
        return PY.host64(g[0])

    outs, reserved = _calls(backward)
    assert all(r == reserved[0] for r in reserved), reserved
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
